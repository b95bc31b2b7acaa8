"""Outputs at addresses that are 16-byte aligned but not 32-byte aligned.

The C ABI asks 16-byte alignment of every pointer. The kernels store fp32 state
rows (the final state S_T, the state cotangent dS0, the segment maps Phi and Psi)
with 32-byte vector stores where the address allows it and with two 16-byte
stores where it does not. Each output here is a view 16 bytes past a 256-byte
boundary, and must come out bit for bit as it does at an aligned address."""
import ctypes as C

import pytest
import torch

import gated_delta_rule_muir_b200 as muir
from gated_delta_rule_muir_b200 import _native as N
from gated_delta_rule_muir_b200.inputs import make_inputs
from tests.gpu_util import INPUT_NAMES, to_dev

pytestmark = pytest.mark.gpu


def _offset_like(x):
    buf = torch.empty(x.numel() + 4, dtype=x.dtype, device=x.device)
    v = buf[4:].view_as(x)
    assert v.data_ptr() % 32 == 16
    return v


@pytest.mark.parametrize("dtype,chunk", [("f32", 64), ("bf16", 128)])
def test_state_outputs_at_16_byte_offsets(cuda_ok, dtype, chunk):
    d = make_inputs(1, 256, 2, 64, 64, dtype=dtype, seed=5, with_state=True, with_grads=True)
    t = to_dev(d, dtype)
    a = [t[n] for n in INPUT_NAMES]
    y0, S0 = muir.chunk_fwd(*a, chunk=chunk, S0=t["S0"])
    y1, S1 = muir.chunk_fwd(*a, chunk=chunk, S0=t["S0"], S_T=_offset_like(S0))
    g0 = muir.chunk_bwd(*a, t["dy"], chunk=chunk, S0=t["S0"], dS_T=t["dS_T"])
    outs = {k: (torch.empty_like(v) if v is not None else None) for k, v in g0.items()}
    outs["dS0"] = _offset_like(g0["dS0"])
    g1 = muir.chunk_bwd(*a, t["dy"], chunk=chunk, S0=t["S0"], dS_T=t["dS_T"], outputs=outs)
    torch.cuda.synchronize()
    assert muir.device_status() == 0
    assert torch.equal(y0, y1) and torch.equal(S0, S1)
    for k, v in g0.items():
        if v is not None:
            assert torch.equal(v, g1[k]), k


def test_segment_maps_at_16_byte_offsets(cuda_ok):
    d = make_inputs(1, 512, 2, 64, 64, dtype="f32", seed=6)
    t = to_dev(d, "f32")
    a = [t[n] for n in INPUT_NAMES]
    Phi0, Psi0 = muir.chunk_segment_map(*a, chunk=64)
    Phi1, Psi1 = _offset_like(Phi0), _offset_like(Psi0)
    lib = N.load()
    args, _ = muir._chunk_args(*a, 64, None)
    nbytes = int(lib.muir_chunk_segment_map_workspace(C.byref(args)))
    ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device="cuda")
    N.check(lib.muir_chunk_segment_map(C.byref(args), C.c_void_p(Phi1.data_ptr()), C.c_void_p(Psi1.data_ptr()),
                                       C.c_void_p(ws.data_ptr()), nbytes,
                                       C.c_void_p(torch.cuda.current_stream().cuda_stream)),
            "muir_chunk_segment_map")
    torch.cuda.synchronize()
    assert muir.device_status() == 0
    assert torch.equal(Phi0, Phi1) and torch.equal(Psi0, Psi1)
