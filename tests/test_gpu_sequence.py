"""Sequence segments on one GPU: the forward of a segment is the affine map
(Phi, Psi) of its start state, so a sequence split into consecutive segments,
each started from its predecessors' maps applied to the initial state, gives the
same outputs and final state as the whole-sequence forward (and the oracle)."""
import pytest
import torch

import gated_delta_rule_muir_b200 as muir
from gated_delta_rule_muir_b200.inputs import make_inputs
from oracle import muir_oracle as orc
from tests.gpu_util import INPUT_NAMES, to_dev, rel_err

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype,chunk,dk,dv,cuts", [
    ("f32", 64, 32, 64, (192, 448)),
    ("bf16", 128, 128, 128, (256, 640)),
    ("f32", 256, 64, 32, (256, 512)),
])
def test_segments_compose_to_the_whole_sequence(cuda_ok, dtype, chunk, dk, dv, cuts):
    T = 768
    d = make_inputs(2, T, 2, dk, dv, dtype=dtype, rate_lo=1e-4, rate_hi=0.7, seed=T + chunk, with_state=True)
    t = to_dev(d, dtype)
    args = [t[n] for n in INPUT_NAMES]
    y_full, S_full = muir.chunk_fwd(*args, chunk=chunk, S0=t["S0"])
    bounds = (0,) + cuts + (T,)
    seg = lambda a, lo, hi: a if a is None or a.dim() == 2 else a[:, lo:hi].contiguous()
    maps = [muir.chunk_segment_map(*[seg(a, lo, hi) for a in args], chunk=chunk)
            for lo, hi in zip(bounds[:-1], bounds[1:])]
    S, ys = t["S0"], []
    for (lo, hi), (Phi, Psi) in zip(zip(bounds[:-1], bounds[1:]), maps):
        y_i, S_end = muir.chunk_fwd(*[seg(a, lo, hi) for a in args], chunk=chunk, S0=S)
        S_map = muir.apply_map(Phi, Psi, S)  # the map reproduces the segment's own end state
        assert rel_err(S_map, S_end.double().cpu().numpy()) < (1e-5 if dtype == "f32" else 1e-4)
        ys.append(y_i)
        S = S_map
    assert muir.device_status() == 0
    y = torch.cat(ys, 1)
    assert rel_err(y, y_full.double().cpu().numpy()) < (1e-5 if dtype == "f32" else 1e-2)
    assert rel_err(S, S_full.double().cpu().numpy()) < (1e-5 if dtype == "f32" else 1e-4)
    y_ref, S_ref = orc.forward(*[d[n] for n in INPUT_NAMES], S0=d["S0"])
    assert rel_err(S, S_ref) < (1e-4 if dtype == "f32" else 1e-3)
    assert rel_err(y, y_ref) < (1e-4 if dtype == "f32" else 2e-2)


def test_empty_segment_is_the_identity_map(cuda_ok):
    d = make_inputs(1, 64, 2, 32, 32, dtype="f32", seed=1)
    t = to_dev(d, "f32")
    args = [a[:, :0].contiguous() if a.dim() == 4 else a for a in (t[n] for n in INPUT_NAMES)]
    Phi, Psi = muir.chunk_segment_map(*args, chunk=64)
    eye = torch.eye(32, device="cuda").expand(1, 2, 32, 32)
    assert torch.equal(Phi, eye) and torch.equal(Psi, torch.zeros_like(Psi))


def test_empty_sequence_forward_and_backward(cuda_ok):
    """T = 0: the forward returns the start state, the backward passes dS_T to dS0."""
    d = make_inputs(1, 64, 2, 32, 32, dtype="f32", seed=2, with_state=True, with_grads=True)
    t = to_dev(d, "f32")
    args = [a[:, :0].contiguous() if a.dim() == 4 else a for a in (t[n] for n in INPUT_NAMES)]
    y, S = muir.chunk_fwd(*args, chunk=64, S0=t["S0"])
    assert y.numel() == 0 and torch.equal(S, t["S0"])
    gr = muir.chunk_bwd(*args, t["dy"][:, :0].contiguous(), chunk=64, S0=t["S0"], dS_T=t["dS_T"], want_dr=True)
    assert torch.equal(gr["dS0"], t["dS_T"]) and torch.equal(gr["dr"], torch.zeros_like(gr["dr"]))
