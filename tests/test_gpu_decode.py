"""Decode step (one token, in place) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import gated_delta_rule_muir_b200 as muir
from gated_delta_rule_muir_b200.inputs import make_inputs
from oracle import muir_oracle as orc
from tests.gpu_util import to_dev, rel_err

pytestmark = pytest.mark.gpu

STEP = ("q", "k", "v", "e", "w", "g", "z", "log_alpha")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("n,H,dk,dv", [(1, 2, 32, 32), (3, 4, 64, 128), (5, 16, 128, 128), (2, 3, 128, 64)])
def test_decode_single_step(cuda_ok, dtype, n, H, dk, dv):
    d = make_inputs(n, 1, H, dk, dv, dtype=dtype, seed=dk + dv + n, with_state=True)
    t = to_dev(d, dtype)
    S = t["S0"].clone()
    y = muir.decode_step(S, *[t[k][:, 0].contiguous() for k in STEP], t["r"])
    y_ref, S_ref = orc.decode_step(d["S0"], *[d[k][:, 0] for k in STEP], d["r"])
    tol_y = 1e-4 if dtype == "f32" else 2e-2
    assert rel_err(y, y_ref) < tol_y
    assert rel_err(S, S_ref) < 1e-5
    assert muir.device_status() == 0


def test_decode_many_steps_track_recurrence(cuda_ok):
    """256 consecutive decode steps equal the token recurrence over the same inputs."""
    B, T, H, dk, dv = 2, 256, 4, 128, 128
    d = make_inputs(B, T, H, dk, dv, dtype="bf16", rate_lo=1e-4, rate_hi=0.7, seed=3, with_state=True)
    t = to_dev(d, "bf16")
    S = t["S0"].clone()
    ys = []
    for s in range(T):
        ys.append(muir.decode_step(S, *[t[k][:, s].contiguous() for k in STEP], t["r"]))
    y = torch.stack(ys, 1)
    y_ref, S_ref = orc.forward(*[d[k] for k in STEP], d["r"], S0=d["S0"])
    assert rel_err(y, y_ref) < 2e-2
    assert rel_err(S, S_ref) < 1e-4


def test_decode_per_row_readout_scale_and_no_output_gate(cuda_ok):
    n, H, dk, dv = 6, 2, 64, 64
    d = make_inputs(n, 1, H, dk, dv, dtype="f32", seed=8, with_state=True)
    t = to_dev(d, "f32")
    rr = np.random.default_rng(0).uniform(0.1, 1.0, size=(n, H, dk)).astype(np.float32).astype(np.float64)
    S = t["S0"].clone()
    y = muir.decode_step(S, *[t[k][:, 0].contiguous() if k != "z" else None for k in STEP],
                         torch.tensor(rr, dtype=torch.float32, device="cuda"))
    for i in range(n):
        yr, Sr = orc.decode_step(d["S0"][i:i + 1], *[d[k][i:i + 1, 0] if k != "z" else None for k in STEP], rr[i])
        assert rel_err(y[i:i + 1], yr) < 1e-4
        assert rel_err(S[i:i + 1], Sr) < 1e-5


def test_state_init(cuda_ok):
    S = torch.randn(3, 2, 64, 32, device="cuda")
    src = torch.randn(3, 2, 64, 32, device="cuda")
    muir.state_init(S)
    assert torch.count_nonzero(S).item() == 0
    muir.state_init(S, src)
    assert torch.equal(S, src)


def test_decode_empty(cuda_ok):
    S = torch.zeros(0, 2, 32, 32, device="cuda")
    z = torch.zeros(0, 2, 32, device="cuda")
    y = muir.decode_step(S, z, z, z, z, z, z, z, z, torch.zeros(2, 32, device="cuda"))
    assert y.shape == (0, 2, 32)


def test_row_scale_matches_oracle(cuda_ok):
    """Static row scale from measured energies: states of a decode run, all rows."""
    g = torch.Generator().manual_seed(9)
    S = (torch.randn(6, 3, 64, 32, generator=g, dtype=torch.float64) *
         torch.rand(1, 3, 64, 1, generator=g, dtype=torch.float64) * 3)
    r = muir.row_scale(S.float().cuda(), exponent=0.5, eps=1e-6)
    r_ref = orc.row_scale(S.float().double().numpy(), exponent=0.5, eps=1e-6)
    assert rel_err(r, r_ref) < 1e-5
