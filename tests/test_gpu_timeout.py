"""The give-up path of the library's bounded device waits, made to run out on purpose.

Every wait in the kernels (bulk-copy and tensor-core completions on an mbarrier)
is bounded: when its limit passes, the kernel records a timeout in a device status
word and returns instead of spinning forever, and muir_device_status() reports
MUIR_ERR_TIMEOUT. Here a one-warp diagnostic kernel waits, through the same wait
routine, on an mbarrier that nothing ever completes (a flag nobody sets), with a
short limit. No copy or tensor-core operation is in flight, so nothing is left
behind on the GPU, and the context stays usable afterwards."""
import ctypes as C
import time

import numpy as np
import pytest
import torch

import gated_delta_rule_muir_b200 as muir
from gated_delta_rule_muir_b200 import _native as N

pytestmark = pytest.mark.gpu


def _wait(limit_ns, arrive):
    lib = N.load()
    out = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    stream = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    N.check(lib.muir_selftest_wait(C.c_uint64(limit_ns), C.c_int32(arrive), C.c_void_p(out.data_ptr()), stream),
            "muir_selftest_wait")
    return out


def test_wait_that_nothing_completes_times_out_and_returns(cuda_ok):
    assert muir.device_status() == N.MUIR_OK  # start from a clear status word
    t0 = time.perf_counter()
    out = _wait(2_000_000, 0)  # 2 ms limit
    status = muir.device_status()  # synchronises: the kernel has returned
    elapsed = time.perf_counter() - t0
    assert int(out.item()) == 0
    assert status == N.MUIR_ERR_TIMEOUT
    assert elapsed < 5.0  # given up after the short limit, not after the library's one second per wait
    # the status word was cleared by the read, and the context still works
    assert muir.device_status() == N.MUIR_OK
    x = torch.arange(8, device="cuda", dtype=torch.float32)
    assert float((x * 2).sum().item()) == 56.0


def test_wait_that_completes_reports_ok(cuda_ok):
    out = _wait(2_000_000, 1)
    assert muir.device_status() == N.MUIR_OK
    assert int(out.item()) == 1


def test_timeout_does_not_leak_into_later_operator_calls(cuda_ok):
    """After a timeout has been read and cleared, an ordinary operator call
    reports a clean status again."""
    _wait(1_000_000, 0)
    assert muir.device_status() == N.MUIR_ERR_TIMEOUT
    from gated_delta_rule_muir_b200.inputs import make_inputs
    from tests.gpu_util import INPUT_NAMES, to_dev
    d = make_inputs(1, 128, 2, 32, 32, dtype="f32", seed=3, with_state=True)
    t = to_dev(d, "f32")
    y, S = muir.chunk_fwd(*[t[n] for n in INPUT_NAMES], chunk=64, S0=t["S0"])
    torch.cuda.synchronize()
    assert muir.device_status() == N.MUIR_OK
    assert np.all(np.isfinite(y.cpu().numpy()))

