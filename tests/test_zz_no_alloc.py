"""The allocation-free forward entry point (muir_chunk_fwd_noalloc).

Callers that cannot allocate device memory (a plug-in host that owns every
allocation, or a latency-critical loop that must not call cudaMalloc/cudaFree
because those can synchronise the device) use this entry point: it runs the
chunkwise forward on a scratch area compiled into the library. These tests call
it through the C ABI and compare it with muir_chunk_fwd, which takes a
caller-provided workspace. This file is collected last on purpose.
"""
import ctypes as C

import pytest
import torch

import gated_delta_rule_muir_b200 as muir
from gated_delta_rule_muir_b200 import _native as N
from gated_delta_rule_muir_b200.inputs import make_inputs
from tests.gpu_util import INPUT_NAMES, to_dev, rel_err


def _args(t, chunk, S0):
    B, T, H, dk = t["q"].shape
    dv = t["v"].shape[-1]
    p = lambda x: C.c_void_p(x.data_ptr()) if x is not None else None
    return N.ChunkArgs(B=B, T=T, H=H, dk=dk, dv=dv, chunk=chunk,
                       dtype=N.MUIR_BF16 if t["q"].dtype == torch.bfloat16 else N.MUIR_F32, flags=0,
                       q=p(t["q"]), k=p(t["k"]), v=p(t["v"]), e=p(t["e"]), w=p(t["w"]), g=p(t["g"]), z=p(t["z"]),
                       log_alpha=p(t["log_alpha"]), r=p(t["r"]), S0=p(S0))


def _noalloc(t, chunk):
    lib = N.load()
    a = _args(t, chunk, t["S0"])
    y = torch.empty_like(t["v"])
    S = torch.empty_like(t["S0"])
    stream = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    N.check(lib.muir_chunk_fwd_noalloc(C.byref(a), C.c_void_p(y.data_ptr()), C.c_void_p(S.data_ptr()), stream),
            "muir_chunk_fwd_noalloc")
    return y, S


@pytest.mark.gpu
def test_noalloc_forward_matches_workspace_forward_twice(cuda_ok):
    # two calls in a row on different inputs and shapes: the second call must not
    # see anything the first one left in the shared scratch
    cases = [(1, 512, 2, 128, 128, 128, "f32", 11), (1, 256, 2, 64, 32, 64, "bf16", 12)]
    for B, T, H, dk, dv, chunk, dtype, seed in cases:
        d = make_inputs(B, T, H, dk, dv, dtype=dtype, seed=seed, with_state=True)
        t = to_dev(d, dtype)
        y0, S0 = muir.chunk_fwd(*[t[n] for n in INPUT_NAMES], chunk=chunk, S0=t["S0"])
        y1, S1 = _noalloc(t, chunk)
        torch.cuda.synchronize()
        # the same kernels on the same inputs, with no atomics in the forward:
        # the results must agree bit for bit, so that stale scratch contents
        # from the previous call could not hide inside a tolerance
        assert torch.equal(y1, y0), rel_err(y1, y0.double().cpu().numpy())
        assert torch.equal(S1, S0), rel_err(S1, S0.double().cpu().numpy())
    assert muir.device_status() == 0


def test_noalloc_rejects_problems_beyond_the_scratch():
    from gated_delta_rule_muir_b200 import build
    build.build()
    lib = N.load()
    fake = C.c_void_p(1 << 20)
    a = N.ChunkArgs(B=4, T=8192, H=16, dk=128, dv=128, chunk=128, dtype=N.MUIR_BF16, flags=0,
                    q=fake, k=fake, v=fake, e=fake, w=fake, g=fake, z=None, log_alpha=fake, r=fake, S0=None)
    assert lib.muir_chunk_fwd_workspace(C.byref(a)) > (32 << 20)
    assert lib.muir_chunk_fwd_noalloc(C.byref(a), fake, None, None) == N.MUIR_ERR_UNSUPPORTED
    assert b"scratch" in lib.muir_last_error()
