"""Chunkwise forward (libmuir, tcgen05 path) against the fp64 token recurrence."""
import numpy as np
import pytest
import torch

import gated_delta_rule_muir_b200 as muir
from gated_delta_rule_muir_b200.inputs import make_inputs
from oracle import muir_oracle as orc
from tests.gpu_util import INPUT_NAMES, to_dev, rel_err

pytestmark = pytest.mark.gpu

# Tolerances (max |x - ref| / max |ref| per tensor): fp32 path 1e-4; bf16 inputs:
# outputs 2e-2, final state 1e-3.
TOL = {"f32": (1e-4, 1e-4), "bf16": (2e-2, 1e-3)}


def _run(d, dtype, chunk, with_z=True, with_s0=True):
    t = to_dev(d, dtype)
    args = [t[n] if (n != "z" or with_z) else None for n in INPUT_NAMES]
    y, S = muir.chunk_fwd(*args, chunk=chunk, S0=t["S0"] if with_s0 else None)
    assert muir.device_status() == 0
    oargs = [d[n] if (n != "z" or with_z) else None for n in INPUT_NAMES]
    y_ref, S_ref = orc.forward(*oargs, S0=d["S0"] if with_s0 else None)
    return y, S, y_ref, S_ref


@pytest.mark.parametrize("B,T,H,dk,dv,chunk,dtype", [
    (1, 256, 2, 32, 32, 64, "f32"),      # the tiny correctness workload
    (1, 512, 2, 32, 32, 128, "f32"),
    (1, 512, 2, 32, 32, 256, "f32"),
    (2, 256, 1, 64, 128, 128, "f32"),
    (1, 256, 2, 128, 64, 64, "f32"),
    (1, 512, 1, 128, 128, 256, "f32"),
    (2, 512, 2, 128, 128, 128, "bf16"),
    (1, 384, 3, 128, 128, 128, "bf16"),
    (1, 256, 2, 64, 32, 64, "bf16"),
])
def test_chunk_fwd_matches_recurrence(cuda_ok, B, T, H, dk, dv, chunk, dtype):
    d = make_inputs(B, T, H, dk, dv, dtype=dtype, rate_lo=1e-3 if dtype == "f32" else 1e-4,
                    rate_hi=0.5 if dtype == "f32" else 0.7, seed=B * 7 + T + dk + chunk, with_state=True)
    y, S, y_ref, S_ref = _run(d, dtype, chunk)
    ty, ts = TOL[dtype]
    ey, es = rel_err(y, y_ref), rel_err(S, S_ref)
    assert ey < ty and es < ts, (ey, es)


def test_chunk_fwd_without_output_gate_or_initial_state(cuda_ok):
    d = make_inputs(1, 256, 2, 64, 64, dtype="f32", seed=5, with_state=True)
    y, S, y_ref, S_ref = _run(d, "f32", 128, with_z=False, with_s0=False)
    assert rel_err(y, y_ref) < 1e-4 and rel_err(S, S_ref) < 1e-4


@pytest.mark.parametrize("chunk", [64, 128, 256])
def test_chunk_fwd_extreme_decay_stays_finite(cuda_ok, chunk):
    """Bimodal decay (rates up to ~8 per token): whole-chunk decay products
    underflow fp32, yet nothing becomes NaN/Inf and the result still matches."""
    d = make_inputs(1, 512, 2, 128, 128, dtype="f32", bimodal=True, seed=4, with_state=True)
    y, S, y_ref, S_ref = _run(d, "f32", chunk)
    assert torch.isfinite(y).all() and torch.isfinite(S).all()
    assert rel_err(y, y_ref) < 1e-4 and rel_err(S, S_ref) < 1e-4


def test_chunk_fwd_identity_padding(cuda_ok):
    """Padding a sequence with identity tokens leaves the final state unchanged."""
    d = make_inputs(1, 192, 2, 32, 32, dtype="f32", seed=12, with_state=True)
    pad = {n: np.concatenate([x, np.zeros_like(x[:, :64])], 1) if x.ndim == 4 else x for n, x in d.items()}
    t = to_dev(d, "f32")
    tp = to_dev(pad, "f32")
    _, S_a = muir.chunk_fwd(*[t[n] for n in INPUT_NAMES], chunk=64, S0=t["S0"])
    _, S_b = muir.chunk_fwd(*[tp[n] for n in INPUT_NAMES], chunk=64, S0=t["S0"])
    # exact in arithmetic; the extra chunk's identity map goes through 3-pass bf16
    # tensor-core products, whose relative rounding is about 2^-17
    assert rel_err(S_b, S_a.double().cpu().numpy()) < 2e-5


def test_chunk_fwd_deterministic(cuda_ok):
    d = make_inputs(1, 256, 2, 128, 128, dtype="bf16", seed=1, with_state=True)
    t = to_dev(d, "bf16")
    a = [t[n] for n in INPUT_NAMES]
    y1, S1 = muir.chunk_fwd(*a, chunk=128, S0=t["S0"])
    y2, S2 = muir.chunk_fwd(*a, chunk=128, S0=t["S0"])
    assert torch.equal(y1, y2) and torch.equal(S1, S2)


def test_chunk_sizes_agree(cuda_ok):
    d = make_inputs(1, 512, 2, 64, 64, dtype="f32", seed=77, with_state=True)
    t = to_dev(d, "f32")
    a = [t[n] for n in INPUT_NAMES]
    outs = [muir.chunk_fwd(*a, chunk=c, S0=t["S0"]) for c in (64, 128, 256)]
    for y, S in outs[1:]:
        assert rel_err(y, outs[0][0].double().cpu().numpy()) < 1e-5
        assert rel_err(S, outs[0][1].double().cpu().numpy()) < 1e-5
