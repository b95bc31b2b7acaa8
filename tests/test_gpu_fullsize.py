"""Full-size workloads: the GPU computes every head; the fp64 oracle recomputes
sampled (batch, head) chains, which are independent of all other chains."""
import pytest
import torch

import gated_delta_rule_muir_b200 as muir
from gated_delta_rule_muir_b200.inputs import TRAIN_FWD, TRAIN_FWD_BWD, STRESS, device_inputs
from oracle import muir_oracle as orc
from tests.gpu_util import INPUT_NAMES, rel_err

pytestmark = pytest.mark.gpu


def _gen(wl, dev, with_grads=False, B=None, T=None):
    return device_inputs(B or wl.B, T or wl.T, wl.H, wl.dk, wl.dv, dtype=wl.dtype, rate_lo=wl.rate_lo,
                         rate_hi=wl.rate_hi, bimodal=wl.bimodal, seed=wl.seed, device=dev, with_grads=with_grads)


def _chain(d, b, h):
    """Host float64 copy of one (b, h) chain, shaped [1, T, 1, d] / r [1, dk]."""
    out = {}
    for n, x in d.items():
        if n == "r":
            out[n] = x[h:h + 1].double().cpu().numpy()
        elif n == "dS_T":
            out[n] = x[b:b + 1, h:h + 1].double().cpu().numpy()
        else:
            out[n] = x[b:b + 1, :, h:h + 1].double().cpu().numpy()
    return out


@pytest.mark.parametrize("chunk", [64, 128, 256])
def test_train_forward_full_size(cuda_ok, chunk):
    """B=8, T=4096, H=16, d=128, bf16: every chunk size; chains (0,0) and (7,15) checked."""
    dev = torch.device("cuda")
    d = _gen(TRAIN_FWD, dev)
    y, S = muir.chunk_fwd(*[d[n] for n in INPUT_NAMES], chunk=chunk)
    assert muir.device_status() == 0
    assert torch.isfinite(y).all() and torch.isfinite(S).all()
    for b, h in ((0, 0), (7, 15)):
        c = _chain(d, b, h)
        y_ref, S_ref = orc.forward(*[c[n] for n in INPUT_NAMES])
        assert rel_err(y[b:b + 1, :, h:h + 1], y_ref) < 2e-2
        assert rel_err(S[b:b + 1, h:h + 1], S_ref) < 1e-3


@pytest.mark.parametrize("saved", [False, True])
def test_train_forward_backward_full_size(cuda_ok, saved):
    """B=1, T=32768, H=16, d=128, chunk 128, bf16, dy ~ N(0,1): head 5 checked for y,
    the final state and every gradient; with and without the forward saving for the
    backward (the saving path is the one the benchmark times)."""
    dev = torch.device("cuda")
    d = _gen(TRAIN_FWD_BWD, dev, with_grads=True)
    a = [d[n] for n in INPUT_NAMES]
    if saved:
        ws = torch.empty(muir.chunk_bwd_workspace_bytes(*a, 128), dtype=torch.uint8, device=dev)
        y, S = muir.chunk_fwd(*a, chunk=128, workspace=ws, save_for_bwd=True)
        gr = muir.chunk_bwd(*a, d["dy"], chunk=128, dS_T=d["dS_T"], want_dr=True, workspace=ws, use_saved=True)
    else:
        y, S = muir.chunk_fwd(*a, chunk=128)
        gr = muir.chunk_bwd(*a, d["dy"], chunk=128, dS_T=d["dS_T"], want_dr=True)
    assert muir.device_status() == 0
    h = 5
    c = _chain(d, 0, h)
    y_ref, S_ref = orc.forward(*[c[n] for n in INPUT_NAMES])
    assert rel_err(y[:, :, h:h + 1], y_ref) < 2e-2
    assert rel_err(S[:, h:h + 1], S_ref) < 1e-3
    ref = orc.backward(*[c[n] for n in INPUT_NAMES], c["dy"], dS_T=c["dS_T"], checkpoint_every=256)
    for n in ("dq", "dk", "dv", "de", "dw", "dg", "dz", "dlog_alpha"):
        assert rel_err(gr[n][:, :, h:h + 1], ref[n]) < 5e-3, n
    assert rel_err(gr["dS0"][:, h:h + 1], ref["dS0"]) < 5e-3
    assert rel_err(gr["dr"][h:h + 1], ref["dr"]) < 5e-3


def test_stress_forward_full_size(cuda_ok):
    """B=2, T=32768, H=16, d=128, chunk 256, fp32, bimodal decay: no NaN/Inf anywhere,
    chain (1, 3) matches the oracle to 1e-4."""
    dev = torch.device("cuda")
    d = _gen(STRESS, dev)
    y, S = muir.chunk_fwd(*[d[n] for n in INPUT_NAMES], chunk=256)
    assert muir.device_status() == 0
    assert torch.isfinite(y).all() and torch.isfinite(S).all()
    c = _chain(d, 1, 3)
    y_ref, S_ref = orc.forward(*[c[n] for n in INPUT_NAMES])
    assert rel_err(y[1:2, :, 3:4], y_ref) < 1e-4
    assert rel_err(S[1:2, 3:4], S_ref) < 1e-4

