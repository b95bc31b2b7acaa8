"""Static-only readout (g = NULL: the query is scaled by the static row scale r
alone, the variant the openai-hub article's matched-filter section compares with
the dynamic readout): chunk forward, backward (with and without the saved maps)
and decode against the oracle with g absent, and against the kernels run with an
explicit all-ones g."""
import pytest
import torch

import gated_delta_rule_muir_b200 as muir
from gated_delta_rule_muir_b200.inputs import make_inputs
from oracle import muir_oracle as orc
from tests.gpu_util import INPUT_NAMES, to_dev, rel_err

pytestmark = pytest.mark.gpu
GI = INPUT_NAMES.index("g")


@pytest.mark.parametrize("dtype,chunk,dk,dv", [("f32", 64, 32, 64), ("bf16", 128, 128, 128), ("f32", 256, 64, 32)])
def test_chunk_static_readout(cuda_ok, dtype, chunk, dk, dv):
    d = make_inputs(1, 512, 2, dk, dv, dtype=dtype, rate_lo=1e-4, rate_hi=0.7, seed=chunk + dk,
                    with_state=True, with_grads=True)
    t = to_dev(d, dtype)
    args = [t[n] for n in INPUT_NAMES]
    args[GI] = None
    ones = list(args)
    ones[GI] = torch.ones_like(t["q"])
    y, S = muir.chunk_fwd(*args, chunk=chunk, S0=t["S0"])
    y1, S1 = muir.chunk_fwd(*ones, chunk=chunk, S0=t["S0"])
    gr = muir.chunk_bwd(*args, t["dy"], chunk=chunk, S0=t["S0"], dS_T=t["dS_T"], want_dr=True)
    gr1 = muir.chunk_bwd(*ones, t["dy"], chunk=chunk, S0=t["S0"], dS_T=t["dS_T"], want_dr=True)
    assert muir.device_status() == 0
    assert gr["dg"] is None
    assert torch.equal(y, y1) and torch.equal(S, S1)
    for n in ("dq", "dk", "dv", "de", "dw", "dz", "dlog_alpha", "dS0"):
        assert torch.equal(gr[n], gr1[n]), n
    oargs = [d[n] for n in INPUT_NAMES]
    oargs[GI] = None
    y_ref, S_ref = orc.forward(*oargs, S0=d["S0"])
    assert rel_err(y, y_ref) < (1e-4 if dtype == "f32" else 2e-2)
    assert rel_err(S, S_ref) < (1e-4 if dtype == "f32" else 1e-3)
    ref = orc.backward(*oargs, d["dy"], S0=d["S0"], dS_T=d["dS_T"])
    assert ref["dg"] is None
    tol = 1e-3 if dtype == "f32" else 5e-3
    for n in ("dq", "dk", "dv", "de", "dw", "dz", "dlog_alpha", "dS0", "dr"):
        assert rel_err(gr[n], ref[n]) < tol, n
    # the saved-maps path
    ws = torch.empty(muir.chunk_bwd_workspace_bytes(*args, chunk, S0=t["S0"]), dtype=torch.uint8, device="cuda")
    muir.chunk_fwd(*args, chunk=chunk, S0=t["S0"], workspace=ws, save_for_bwd=True)
    gs = muir.chunk_bwd(*args, t["dy"], chunk=chunk, S0=t["S0"], dS_T=t["dS_T"], want_dr=True, workspace=ws,
                        use_saved=True)
    for n in ("dq", "dk", "dv", "de", "dw", "dz", "dlog_alpha", "dS0"):
        assert rel_err(gs[n], gr[n].double().cpu().numpy()) < 1e-5, n


def test_decode_static_readout(cuda_ok):
    d = make_inputs(3, 4, 2, 64, 64, dtype="bf16", seed=5, with_state=True)
    t = to_dev(d, "bf16")
    S = t["S0"].clone()
    ys = []
    for s in range(4):
        tok = [t[n][:, s].contiguous() if n != "g" else None for n in INPUT_NAMES[:8]]
        ys.append(muir.decode_step(S, *tok, t["r"]))
    assert muir.device_status() == 0
    oargs = [d[n] for n in INPUT_NAMES]
    oargs[GI] = None
    y_ref, S_ref = orc.forward(*oargs, S0=d["S0"])
    assert rel_err(torch.stack(ys, 1), y_ref) < 2e-2
    assert rel_err(S, S_ref) < 1e-3
