"""Pins for the gate-projection oracle: the pages' rank table, a one-hot case
whose every gate output is known in closed form (so a swapped or shifted rank
slice fails), the zero-input special case, and identities of the activations
that hold independently of how they are evaluated."""
import math
import os

import numpy as np

from oracle import gate_proj_oracle as gpo

HERE = os.path.dirname(os.path.abspath(__file__))


def test_ranks_match_the_pages_table():
    table = {}
    for line in open(os.path.join(HERE, "golden", "gate_ranks.txt")):
        if line.strip() and not line.startswith("#"):
            k, v = line.split()
            table[k] = int(v)
    assert gpo.RANKS == (table["decay"], table["erase"], table["output"], table["write"], table["read"])
    assert sum(gpo.RANKS) == table["total"] == gpo.TOTAL_RANK
    assert gpo.rank_slices() == [(0, 64), (64, 128), (128, 256), (256, 384), (384, 512)]


def _identity_ups(Ok, Ov):
    """U_j that copy slice entry r to output column r (and leave the rest at 0)."""
    ups = []
    for r, o in zip(gpo.RANKS, (Ok, Ok, Ov, Ov, Ok)):
        U = np.zeros((r, o))
        n = min(r, o)
        U[np.arange(n), np.arange(n)] = 1.0
        ups.append(U)
    return ups


def test_one_hot_rows_select_each_gates_own_slice():
    """x = e_i picks row i of W_down; with copying up-projections gate j's first
    r_j outputs are act(W_down[i, slice_j]) and the rest act(0)."""
    rng = np.random.default_rng(3)
    D, Ok, Ov = 6, 160, 144
    w_down = rng.normal(size=(D, 512))
    ups = _identity_ups(Ok, Ov)
    x = np.eye(D)[[2, 5, 0]]
    la, e, z, w, g = gpo.gate_proj(x, w_down, *ups)
    outs = [la, e, z, w, g]
    for j, ((a, b), out) in enumerate(zip(gpo.rank_slices(), outs)):
        for row, i in enumerate([2, 5, 0]):
            hj = w_down[i, a:b]
            n = b - a
            want_sig = 1.0 / (1.0 + np.exp(-hj))
            if j == 0:
                np.testing.assert_allclose(np.exp(out[row, :n]), want_sig, rtol=1e-13)
                np.testing.assert_allclose(out[row, n:], -math.log(2.0), rtol=1e-15)
            else:
                np.testing.assert_allclose(out[row, :n], want_sig, rtol=1e-13)
                np.testing.assert_allclose(out[row, n:], 0.5, rtol=1e-15)


def test_zero_input_gives_half_gates():
    rng = np.random.default_rng(4)
    D, Ok, Ov = 8, 64, 128
    ups = [rng.normal(size=(r, o)) for r, o in zip(gpo.RANKS, (Ok, Ok, Ov, Ov, Ok))]
    la, e, z, w, g = gpo.gate_proj(np.zeros((3, D)), rng.normal(size=(D, 512)), *ups)
    np.testing.assert_allclose(la, -math.log(2.0), rtol=1e-15)
    for t in (e, z, w, g):
        np.testing.assert_allclose(t, 0.5, rtol=1e-15)


def test_activation_identities():
    u = np.concatenate([np.linspace(-40, 40, 801), [-700.0, -60.0, 60.0, 700.0]])
    s, ls = gpo.sigmoid(u), gpo.log_sigmoid(u)
    np.testing.assert_allclose(s + gpo.sigmoid(-u), 1.0, rtol=1e-15)  # symmetry
    np.testing.assert_allclose(ls - gpo.log_sigmoid(-u), u, rtol=1e-12, atol=1e-12)  # log-odds
    mid = np.abs(u) <= 40
    np.testing.assert_allclose(np.exp(ls[mid]), s[mid], rtol=1e-14)
    assert abs(gpo.log_sigmoid(np.array([-700.0]))[0] + 700.0) < 1e-12  # log sigmoid(u) -> u for u << 0
    assert np.all(np.isfinite(ls)) and np.all((s >= 0) & (s <= 1)) and np.all(ls <= 0)


def test_linear_in_x_before_the_activation():
    """Inverting the activations recovers h_j U_j, which is linear in x."""
    rng = np.random.default_rng(5)
    D, Ok, Ov = 10, 32, 48
    wd = rng.normal(size=(D, 512)) * 0.05
    ups = [rng.normal(size=(r, o)) * 0.05 for r, o in zip(gpo.RANKS, (Ok, Ok, Ov, Ov, Ok))]
    x1, x2 = rng.normal(size=(4, D)), rng.normal(size=(4, D))

    def logits(x):
        la, e, z, w, g = gpo.gate_proj(x, wd, *ups)
        return [la - np.log1p(-np.exp(la))] + [np.log(t / (1.0 - t)) for t in (e, z, w, g)]

    for a, b, c in zip(logits(x1), logits(x2), logits(x1 + 2.0 * x2)):
        np.testing.assert_allclose(c, a + 2.0 * b, rtol=1e-9, atol=1e-12)
