"""The benchmark's algorithmic work model against the per-head-token figures the
survey of the pages prints for the measurement (its "Algorithmic work" paragraph):
forward flops 1.98e5 / 2.68e5 / 4.15e5 at chunk 64 / 128 / 256 (d = 128),
backward 7.26e5 at chunk 128, fwd+bwd 993,962 flops over 8,448 bytes, and bytes
2,560 forward / 5,888 backward on the bf16 path, 4,608 forward on the fp32 path.
The roofline fractions bench.py reports divide by these."""
import pytest

import bench


@pytest.mark.parametrize("C,printed", [(64, 1.98e5), (128, 2.68e5), (256, 4.15e5)])
def test_forward_flops_per_head_token(C, printed):
    ff, _, _, _ = bench.pass_work(C, 128, 2)
    assert abs(ff - printed) / printed < 5e-3


def test_backward_and_step_work_at_chunk_128():
    ff, fb, bf, bb = bench.pass_work(128, 128, 2)
    assert abs(bf - 7.26e5) / 7.26e5 < 5e-3
    assert int(ff + bf) == 993_962
    assert (fb, bb) == (2560, 5888)
    assert fb + bb == 8448


def test_fp32_forward_bytes():
    _, fb, _, _ = bench.pass_work(256, 128, 4)
    assert fb == 4608


def test_flop_split_is_a_split():
    fs = bench.flop_split(128, 128, 128)
    assert abs(fs["mma_share"] + fs["alu_share"] - 1.0) < 1e-3
    assert 0.9 < fs["mma_share"] < 1.0
    assert all(v > 0 for v in fs["alu_terms_per_unit"].values())
