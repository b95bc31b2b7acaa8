"""Chunkwise backward (libmuir) against the oracle's reverse-mode recurrence."""
import pytest
import torch

import gated_delta_rule_muir_b200 as muir
from gated_delta_rule_muir_b200.inputs import make_inputs
from oracle import muir_oracle as orc
from tests.gpu_util import INPUT_NAMES, to_dev, rel_err

pytestmark = pytest.mark.gpu

GRADS = ("dq", "dk", "dv", "de", "dw", "dg", "dz", "dlog_alpha", "dS0")
# Gradient tolerance (max-normalised relative error): 5e-3; the fp32 path is held to 1e-3.
TOL = {"f32": 1e-3, "bf16": 5e-3}


def _check(B, T, H, dk, dv, chunk, dtype, with_z=True, with_s0=True, with_dst=True, seed=0):
    d = make_inputs(B, T, H, dk, dv, dtype=dtype, rate_lo=1e-3 if dtype == "f32" else 1e-4,
                    rate_hi=0.5 if dtype == "f32" else 0.7, seed=seed, with_state=True, with_grads=True)
    t = to_dev(d, dtype)
    args = [t[n] if (n != "z" or with_z) else None for n in INPUT_NAMES]
    gr = muir.chunk_bwd(*args, t["dy"], chunk=chunk, S0=t["S0"] if with_s0 else None,
                        dS_T=t["dS_T"] if with_dst else None, want_dr=True)
    assert muir.device_status() == 0
    oargs = [d[n] if (n != "z" or with_z) else None for n in INPUT_NAMES]
    ref = orc.backward(*oargs, d["dy"], S0=d["S0"] if with_s0 else None, dS_T=d["dS_T"] if with_dst else None)
    errs = {}
    for n in GRADS + ("dr",):
        if n == "dz" and not with_z:
            continue
        errs[n] = rel_err(gr[n], ref[n])
    bad = {n: e for n, e in errs.items() if not e < TOL[dtype]}
    assert not bad, errs


@pytest.mark.parametrize("B,T,H,dk,dv,chunk,dtype", [
    (1, 256, 2, 32, 32, 64, "f32"),
    (2, 256, 1, 64, 128, 128, "f32"),
    (1, 512, 1, 128, 128, 256, "f32"),
    (1, 256, 2, 128, 64, 64, "f32"),
    (1, 256, 2, 128, 128, 128, "bf16"),
    (2, 384, 1, 64, 64, 128, "bf16"),
])
def test_chunk_bwd_matches_reverse_recurrence(cuda_ok, B, T, H, dk, dv, chunk, dtype):
    _check(B, T, H, dk, dv, chunk, dtype, seed=T + dk + chunk)


def test_chunk_bwd_optional_inputs_absent(cuda_ok):
    _check(1, 256, 2, 64, 64, 128, "f32", with_z=False, with_s0=False, with_dst=False, seed=3)


def test_chunk_bwd_extreme_decay(cuda_ok):
    d = make_inputs(1, 256, 1, 128, 128, dtype="f32", bimodal=True, seed=4, with_state=True, with_grads=True)
    t = to_dev(d, "f32")
    gr = muir.chunk_bwd(*[t[n] for n in INPUT_NAMES], t["dy"], chunk=128, S0=t["S0"], dS_T=t["dS_T"])
    ref = orc.backward(*[d[n] for n in INPUT_NAMES], d["dy"], S0=d["S0"], dS_T=d["dS_T"])
    for n in GRADS:
        assert torch.isfinite(gr[n]).all(), n
        assert rel_err(gr[n], ref[n]) < 1e-3, (n, rel_err(gr[n], ref[n]))
