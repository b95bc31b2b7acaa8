"""The division-based chunk decay (tests/unpivoted_foil.py, fp32, no pivoting)
against the pivoted chunk algebra on the same inputs: equal where the decay is
mild, and non-finite where fast-decaying channels meet a long chunk, while the
pivoted form stays finite and equal to the token recurrence."""
import numpy as np

from gated_delta_rule_muir_b200.inputs import make_inputs
from oracle import muir_oracle as orc
from tests.unpivoted_foil import forward_unpivoted_fp32

NAMES = ("q", "k", "v", "e", "w", "g", "z", "log_alpha", "r")


def _rel(x, ref):
    return float(np.max(np.abs(x - ref)) / np.max(np.abs(ref)))


def test_foil_agrees_with_the_recurrence_on_mild_decay():
    d = make_inputs(1, 128, 2, 16, 16, dtype="f32", rate_lo=1e-3, rate_hi=0.05, seed=11)
    a = [d[n] for n in NAMES]
    y_ref, S_ref = orc.forward(*a)
    y, S = forward_unpivoted_fp32(*a, chunk=64)
    assert np.isfinite(y).all() and np.isfinite(S).all()
    assert _rel(y, y_ref) < 1e-4 and _rel(S, S_ref) < 1e-4


def test_foil_breaks_on_fast_decay_where_pivoting_holds():
    """Bimodal decay as in the stress workload (half the rows of each head decay with
    rates in [2, 8] per token) over a 128-token chunk: the reciprocal prefix
    products overflow fp32, and the foil's outputs turn non-finite in every head."""
    H = 4
    d = make_inputs(1, 128, H, 16, 16, dtype="f32", bimodal=True, seed=12)
    a = [d[n] for n in NAMES]
    y, S = forward_unpivoted_fp32(*a, chunk=128)
    bad_heads = [h for h in range(H) if not np.isfinite(y[:, :, h]).all()]
    assert len(bad_heads) >= 1, "the unpivoted form should fail on this decay"
    y_p, S_p = orc.chunk_forward(*a, chunk=128, sub=16)
    y_ref, S_ref = orc.forward(*a)
    assert np.isfinite(y_p).all() and np.isfinite(S_p).all()
    assert _rel(y_p, y_ref) < 1e-10 and _rel(S_p, S_ref) < 1e-10


def test_foil_breaks_at_chunk_256_on_the_training_decays():
    """The training workloads' decay rates (log-uniform in [1e-4, 0.7] per row): over
    128 tokens the fastest rows' prefix products stay inside fp32 and the foil is
    finite; over 256 tokens they underflow and every head turns non-finite. The
    pivoted kernels run these workloads at chunk 256 (tests/test_gpu_fullsize.py)."""
    d = make_inputs(1, 256, 8, 16, 16, dtype="f32", rate_lo=1e-4, rate_hi=0.7, seed=2)
    a = [d[n] for n in NAMES]
    y128, _ = forward_unpivoted_fp32(*a, chunk=128)
    y256, _ = forward_unpivoted_fp32(*a, chunk=256)
    assert np.isfinite(y128).all()
    assert not np.isfinite(y256).all()
    y_ref, _ = orc.forward(*a)
    assert _rel(y128, y_ref) < 1e-3
