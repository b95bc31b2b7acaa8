"""The tensor-core operand layouts (K-major / MN-major no-swizzle tiles, 1- and
3-pass bf16) against an fp64 matmul, through the library's diagnostic export."""
import ctypes as C

import numpy as np
import pytest
import torch

from gated_delta_rule_muir_b200 import _native as N

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("a_mn", [0, 1, 2, 3])
@pytest.mark.parametrize("b_mn", [0, 1, 2, 3])
@pytest.mark.parametrize("N_,K", [(16, 16), (64, 128), (128, 64), (256, 128), (48, 32)])
@pytest.mark.parametrize("nsplit", [1, 3])
def test_selftest_gemm(cuda_ok, a_mn, b_mn, N_, K, nsplit):
    lib = N.load()
    g = torch.Generator().manual_seed(N_ * 1000 + K * 10 + a_mn * 2 + b_mn)
    A = torch.randn(128, K, generator=g)
    B = torch.randn(K, N_, generator=g)
    Ad, Bd = A.cuda(), B.cuda()
    D = torch.full((128, N_), float("nan"), device="cuda")
    N.check(lib.muir_selftest_gemm(C.c_void_p(Ad.data_ptr()), C.c_void_p(Bd.data_ptr()), C.c_void_p(D.data_ptr()),
                                   N_, K, a_mn, b_mn, nsplit, C.c_void_p(torch.cuda.current_stream().cuda_stream)),
            "selftest")
    torch.cuda.synchronize()
    ref = (A.double() @ B.double()).numpy()
    err = np.max(np.abs(D.double().cpu().numpy() - ref)) / np.max(np.abs(ref))
    assert err < (1e-2 if nsplit == 1 else 5e-5), err


@pytest.mark.parametrize("mode", [0, 1, 2])
@pytest.mark.parametrize("N_,K", [(64, 64), (128, 64), (256, 128), (64, 128)])
def test_selftest_sw128(cuda_ok, mode, N_, K):
    """128-byte-swizzled operands: A K-major, B MN-major, written by the threads
    (mode 0) or loaded by TMA boxes (mode 1); mode 2 stores A transposed and reads
    it as the MN-major operand. bf16 products are exact, so only the fp32
    accumulation order separates the result from the fp64 matmul of the same bf16
    values."""
    use_tma = mode
    lib = N.load()
    g = torch.Generator().manual_seed(7 * N_ + K + 1000 * use_tma)
    A = torch.randn(128, K, generator=g).bfloat16()
    B = torch.randn(K, N_, generator=g).bfloat16()
    Ad, Bd = A.cuda(), B.cuda()
    D = torch.full((128, N_), float("nan"), device="cuda")
    N.check(lib.muir_selftest_sw128(C.c_void_p(Ad.data_ptr()), C.c_void_p(Bd.data_ptr()), C.c_void_p(D.data_ptr()),
                                    N_, K, use_tma, C.c_void_p(torch.cuda.current_stream().cuda_stream)),
            "selftest_sw128")
    torch.cuda.synchronize()
    from gated_delta_rule_muir_b200 import device_status
    assert device_status() == 0
    ref = (A.double() @ B.double()).numpy()
    err = np.max(np.abs(D.double().cpu().numpy() - ref)) / np.max(np.abs(ref))
    assert err < 1e-5, err
