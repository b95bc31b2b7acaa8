"""Pins for the fp64 oracle: each test checks it against something other than
itself (a closed form, a brute-force sum, a textbook special case, finite
differences, an independent autograd transcription, a figure from the pages)."""
import os

import numpy as np
import pytest

from gated_delta_rule_muir_b200.inputs import make_inputs, DECODE
from oracle import muir_oracle as orc

HERE = os.path.dirname(os.path.abspath(__file__))


def _inp(B=1, T=12, H=2, dk=4, dv=3, seed=0, **kw):
    return make_inputs(B, T, H, dk, dv, dtype="f32", seed=seed, **kw)


def _args(d):
    return (d["q"], d["k"], d["v"], d["e"], d["w"], d["g"], d["z"], d["log_alpha"], d["r"])


def test_linear_attention_closed_form():
    """alpha = 1, e = 0, w = 1: causal linear attention with query qt = r*g*q,
    O = tril(Qt K^T) V and S_T = S0 + K^T V."""
    d = _inp(B=2, T=17, H=3, dk=5, dv=4, with_state=True)
    d["log_alpha"][:] = 0.0
    d["e"][:] = 0.0
    d["w"][:] = 1.0
    y, S = orc.forward(*_args(d), S0=d["S0"])
    for b in range(2):
        for h in range(3):
            Q = d["r"][h] * d["g"][b, :, h] * d["q"][b, :, h]
            K, V = d["k"][b, :, h], d["v"][b, :, h]
            O = np.tril(Q @ K.T) @ V + Q @ d["S0"][b, h]
            np.testing.assert_allclose(y[b, :, h], d["z"][b, :, h] * O, rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(S[b, h], d["S0"][b, h] + K.T @ V, rtol=1e-12, atol=1e-12)


def test_gated_linear_attention_brute_force():
    """e = 0, w = 1: no erase, so o_t = sum_{s<=t} sum_i qt_ti k_si prod_{u=s+1..t} alpha_ui v_s
    (+ the decayed initial state), with every decay product multiplied out explicitly."""
    d = _inp(B=1, T=9, H=2, dk=3, dv=2, seed=3, with_state=True)
    d["e"][:] = 0.0
    d["w"][:] = 1.0
    y, _ = orc.forward(*_args(d), S0=d["S0"])
    al = np.exp(d["log_alpha"])
    T = 9
    for h in range(2):
        for t in range(T):
            qt = d["r"][h] * d["g"][0, t, h] * d["q"][0, t, h]
            o = np.zeros(2)
            for s in range(t + 1):
                for i in range(3):
                    prod = 1.0
                    for u in range(s + 1, t + 1):
                        prod *= al[0, u, h, i]
                    o += qt[i] * d["k"][0, s, h, i] * prod * d["v"][0, s, h]
            for i in range(3):
                prod = 1.0
                for u in range(0, t + 1):
                    prod *= al[0, u, h, i]
                o += qt[i] * prod * d["S0"][0, h, i]
            np.testing.assert_allclose(y[0, t, h], d["z"][0, t, h] * o, rtol=1e-12, atol=1e-13)


def test_one_hot_keys_decouple_rows():
    """k_t = unit vector on row i_t: every row decays by its alpha; the keyed row then
    becomes (1 - e_i) * alpha_i * S_i + w*v (erase then write), the others stay decayed."""
    rng = np.random.default_rng(5)
    B, T, H, dk, dv = 1, 20, 1, 4, 3
    d = _inp(B, T, H, dk, dv, seed=5, with_state=True)
    idx = rng.integers(0, dk, size=T)
    d["k"][:] = 0.0
    d["k"][0, np.arange(T), 0, idx] = 1.0
    _, S = orc.forward(*_args(d), S0=d["S0"])
    Sref = d["S0"][0, 0].copy()
    al = np.exp(d["log_alpha"][0, :, 0])
    for t in range(T):
        Sref = al[t][:, None] * Sref
        i = idx[t]
        Sref[i] = (1.0 - d["e"][0, t, 0, i]) * Sref[i] + d["w"][0, t, 0] * d["v"][0, t, 0]
    np.testing.assert_allclose(S[0, 0], Sref, rtol=1e-13, atol=1e-13)


def test_single_token_identities():
    """S0 = 0, q = k unit, r = g = z = 1: the readout after the write returns w*v.
    S0 = k c^T, alpha = 1, e = 1: the erase removes the old association entirely, S1 = k (w*v)^T."""
    d = _inp(B=1, T=1, H=1, dk=6, dv=4, seed=9)
    d["q"] = d["k"].copy()
    d["r"][:] = 1.0
    d["g"][:] = 1.0
    d["z"][:] = 1.0
    y, S = orc.forward(*_args(d))
    u = d["w"][0, 0, 0] * d["v"][0, 0, 0]
    np.testing.assert_allclose(y[0, 0, 0], u * (d["k"][0, 0, 0] @ d["k"][0, 0, 0]), rtol=1e-13)
    np.testing.assert_allclose(y[0, 0, 0], u, rtol=1e-6)   # |k| = 1 up to its fp32 rounding
    k = d["k"][0, 0, 0] / np.linalg.norm(d["k"][0, 0, 0])
    d["k"][0, 0, 0] = k
    c = np.arange(4.0) - 1.5
    d["log_alpha"][:] = 0.0
    d["e"][:] = 1.0
    _, S = orc.forward(*_args(d), S0=np.outer(k, c)[None, None])
    np.testing.assert_allclose(S[0, 0], np.outer(k, u), rtol=1e-12, atol=1e-13)


def test_scalar_gates_reduce_to_textbook_gated_delta_rule():
    """alpha scalar per token, e = w = beta (scalars): S_t = alpha (I - beta k k^T) S + beta k v^T."""
    rng = np.random.default_rng(11)
    B, T, H, dk, dv = 1, 15, 1, 5, 4
    d = _inp(B, T, H, dk, dv, seed=11, with_state=True)
    la = -rng.uniform(0.01, 0.5, size=T)
    beta = rng.uniform(0.1, 0.9, size=T)
    d["log_alpha"][0, :, 0, :] = la[:, None]
    d["e"][0, :, 0, :] = beta[:, None]
    d["w"][0, :, 0, :] = beta[:, None]
    _, S = orc.forward(*_args(d), S0=d["S0"])
    St = d["S0"][0, 0].copy()
    for t in range(T):
        k = d["k"][0, t, 0]
        St = np.exp(la[t]) * (np.eye(dk) - beta[t] * np.outer(k, k)) @ St + beta[t] * np.outer(k, d["v"][0, t, 0])
    np.testing.assert_allclose(S[0, 0], St, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("T,C,sub,dk", [(32, 8, 4, 4), (48, 16, 4, 8), (64, 16, 8, 4), (24, 8, 2, 5)])
def test_chunk_algebra_equals_recurrence(T, C, sub, dk):
    d = _inp(B=1, T=T, H=2, dk=dk, dv=3, seed=T + C, with_state=True)
    y0, S0 = orc.forward(*_args(d), S0=d["S0"])
    y1, S1, fac = orc.chunk_forward(*_args(d), chunk=C, sub=sub, S0=d["S0"], return_factors=True)
    np.testing.assert_allclose(y1, y0, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(S1, S0, rtol=1e-11, atol=1e-12)
    f = np.concatenate([np.ravel(x) for x in fac])
    assert np.all(f >= 0.0) and np.all(f <= 1.0)


def test_chunk_algebra_under_extreme_decay():
    """Bimodal stress decay (rates up to 8 per token): every pivoted factor stays in
    [0, 1], nothing overflows, and the chunk form still equals the recurrence."""
    d = make_inputs(1, 64, 1, 8, 4, dtype="f32", bimodal=True, seed=4)
    y0, S0 = orc.forward(*_args(d))
    y1, S1, fac = orc.chunk_forward(*_args(d), chunk=64, sub=8, return_factors=True)
    f = np.concatenate([np.ravel(x) for x in fac])
    assert np.all(np.isfinite(f)) and np.all(f >= 0.0) and np.all(f <= 1.0)
    # the stress is real: whole-chunk decay products fall below fp32's smallest normal
    assert np.exp(d["log_alpha"].sum(1)).min() < np.finfo(np.float32).tiny
    np.testing.assert_allclose(y1, y0, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(S1, S0, rtol=1e-10, atol=1e-12)


def test_identity_padding_tokens_leave_state_unchanged():
    """Tokens with log_alpha = 0, k = 0, e = 0, w = 0 are exact no-ops on the state."""
    d = _inp(B=1, T=10, H=2, dk=4, dv=3, seed=2, with_state=True)
    _, S_a = orc.forward(*_args(d), S0=d["S0"])
    for n in ("log_alpha", "k", "e"):
        d[n][:, 5:] = 0.0
    d["w"][:, 5:] = 0.0
    _, S_b = orc.forward(*[x[:, :5] if x.ndim == 4 else x for x in _args(d)], S0=d["S0"])
    _, S_c = orc.forward(*_args(d), S0=d["S0"])
    np.testing.assert_array_equal(S_b, S_c)
    assert not np.allclose(S_a, S_c)


def _loss_and_grads(d, dy, dS_T):
    y, S = orc.forward(*_args(d), S0=d["S0"])
    return float((y * dy).sum() + (S * dS_T).sum())


def test_backward_central_differences():
    d = _inp(B=1, T=7, H=2, dk=3, dv=2, seed=21, with_state=True, with_grads=True)
    dy, dS_T = d["dy"], d["dS_T"]
    gr = orc.backward(*_args(d), dy, S0=d["S0"], dS_T=dS_T, checkpoint_every=3)
    eps = 1e-6
    names = {"q": "dq", "k": "dk", "v": "dv", "e": "de", "w": "dw", "g": "dg", "z": "dz",
             "log_alpha": "dlog_alpha", "S0": "dS0", "r": "dr"}
    for n, gname in names.items():
        base = d[n]
        num = np.zeros_like(base)
        it = np.nditer(base, flags=["multi_index"])
        for _ in it:
            i = it.multi_index
            old = base[i]
            base[i] = old + eps
            lp = _loss_and_grads(d, dy, dS_T)
            base[i] = old - eps
            lm = _loss_and_grads(d, dy, dS_T)
            base[i] = old
            num[i] = (lp - lm) / (2 * eps)
        err = np.max(np.abs(num - gr[gname])) / max(np.max(np.abs(num)), 1e-30)
        assert err < 1e-6, (n, err)


def test_backward_matches_independent_autograd():
    """A separate transcription of the recurrence in torch (CPU, float64) differentiated
    by autograd agrees with the hand-written reverse recurrence."""
    torch = pytest.importorskip("torch")
    d = _inp(B=2, T=13, H=2, dk=4, dv=3, seed=31, with_state=True, with_grads=True)
    names = ["q", "k", "v", "e", "w", "g", "z", "log_alpha", "r", "S0"]
    tt = {n: torch.tensor(d[n], dtype=torch.float64, requires_grad=True) for n in names}

    S = tt["S0"]
    ys = []
    for t in range(13):
        al = torch.exp(tt["log_alpha"][:, t])                     # [B,H,dk]
        k = tt["k"][:, t]
        X = al.unsqueeze(-1) * S
        pred = torch.einsum("bhi,bhij->bhj", k, X)
        S = X - torch.einsum("bhi,bhj->bhij", tt["e"][:, t] * k, pred) \
            + torch.einsum("bhi,bhj->bhij", k, tt["w"][:, t] * tt["v"][:, t])
        qq = tt["r"].unsqueeze(0) * tt["g"][:, t] * tt["q"][:, t]
        ys.append(tt["z"][:, t] * torch.einsum("bhi,bhij->bhj", qq, S))
    Y = torch.stack(ys, 1)
    loss = (Y * torch.tensor(d["dy"])).sum() + (S * torch.tensor(d["dS_T"])).sum()
    loss.backward()
    gr = orc.backward(*_args(d), d["dy"], S0=d["S0"], dS_T=d["dS_T"], checkpoint_every=5)
    m = {"q": "dq", "k": "dk", "v": "dv", "e": "de", "w": "dw", "g": "dg", "z": "dz",
         "log_alpha": "dlog_alpha", "r": "dr", "S0": "dS0"}
    for n, gname in m.items():
        np.testing.assert_allclose(gr[gname], tt[n].grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(orc.forward(*_args(d), S0=d["S0"])[0], Y.detach().numpy(), rtol=1e-12)


def test_backward_checkpoint_interval_irrelevant():
    d = _inp(B=1, T=11, H=1, dk=3, dv=3, seed=41, with_state=True, with_grads=True)
    g1 = orc.backward(*_args(d), d["dy"], S0=d["S0"], dS_T=d["dS_T"], checkpoint_every=1)
    g2 = orc.backward(*_args(d), d["dy"], S0=d["S0"], dS_T=d["dS_T"], checkpoint_every=4)
    for n in g1:
        np.testing.assert_allclose(g1[n], g2[n], rtol=1e-13, atol=1e-14)


def test_decode_step_is_one_token_of_forward():
    d = _inp(B=3, T=1, H=2, dk=4, dv=5, seed=7, with_state=True)
    y, S = orc.decode_step(d["S0"], *[d[n][:, 0] for n in ("q", "k", "v", "e", "w", "g", "z", "log_alpha")], d["r"])
    y2, S2 = orc.forward(*_args(d), S0=d["S0"])
    np.testing.assert_array_equal(y, y2[:, 0])
    np.testing.assert_array_equal(S, S2)


def test_state_size_matches_pages():
    """The decode workload's state is the pages' 25 MB (24 layers x 16 heads x 128 x 128 fp32)."""
    vals = {}
    for line in open(os.path.join(HERE, "golden", "state_size.txt")):
        if line.strip() and not line.startswith("#"):
            key, val = line.split()
            vals[key] = int(val)
    nbytes = vals["layers"] * vals["heads"] * vals["dk"] * vals["dv"] * vals["bytes_per_element"]
    assert nbytes == 25_165_824 and round(nbytes / 1e6) == vals["approx_total_MB"]
    assert (DECODE.extra["layers"], DECODE.H, DECODE.dk, DECODE.dv) == \
        (vals["layers"], vals["heads"], vals["dk"], vals["dv"])


def test_row_scale_matches_the_stationary_energy_of_a_decaying_row():
    """A row that decays by abar per token and receives unit-variance writes has
    stationary energy 1 / (1 - abar^2); with exponent 0.5 the measured scale is
    its inverse square root, sqrt(1 - abar^2), the static scale the input recipe
    uses up to the constant (1 + abar)^0.5. Rows of constant magnitude c give c^-1
    exactly."""
    rng = np.random.default_rng(7)
    abar = np.array([0.5, 0.9, 0.99])
    n_chain, T = 256, 3000
    s = np.zeros((n_chain, abar.size))
    samples = []
    for t in range(T):
        s = abar * s + rng.standard_normal(s.shape)
        if t >= 1000 and t % 10 == 0:
            samples.append(s.copy())
    S = np.stack(samples)[:, None, :, :].transpose(0, 1, 3, 2)  # [N, H=1, dk=3, dv=n_chain]
    r = orc.row_scale(S, exponent=0.5)[0]
    np.testing.assert_allclose(r, np.sqrt(1 - abar ** 2), rtol=0.08)
    c = np.array([0.5, 2.0, 3.0])
    S2 = np.broadcast_to(c[None, None, :, None], (4, 1, 3, 5)) * np.where(np.arange(5) % 2, 1.0, -1.0)
    np.testing.assert_allclose(orc.row_scale(S2, exponent=0.5, eps=0.0)[0], 1.0 / c, rtol=1e-12)
