"""Sequence parallelism for the chunkwise forward: a sequence split along T
across the ranks of a process group, with one exchange.

The forward over a segment is an affine map of the segment's start state,
S_end = Phi S_start + Psi (every chunk map is affine and their composition is
too). Rank i holds the i-th consecutive segment. Each rank composes its
segment's map (muir_chunk_segment_map), the maps are all-gathered (NCCL on GPUs;
dk x (dk + dv) floats per (batch, head)), rank i applies the maps of ranks
0..i-1 to the initial state to obtain its own start state, and then runs the
ordinary forward from it. Argument marshalling only: the maps, their
application and the forward run in libmuir's kernels (the `ops` hook exists so
that the exchange can be exercised without a GPU).
"""
from __future__ import annotations

import torch
import torch.distributed as dist


class _LibOps:
    """The library's kernels (default `ops`)."""

    @staticmethod
    def segment_map(args, chunk):
        from . import chunk_segment_map
        return chunk_segment_map(*args, chunk=chunk)

    @staticmethod
    def apply_map(Phi, Psi, S):
        from . import apply_map
        return apply_map(Phi, Psi, S)

    @staticmethod
    def forward(args, chunk, S0):
        from . import chunk_fwd
        return chunk_fwd(*args, chunk=chunk, S0=S0)


def chunk_fwd_sequence_parallel(q, k, v, e, w, g, z, log_alpha, r, *, chunk=128, S0=None, group=None, ops=None):
    """Forward of this rank's segment [B, T_i, H, d] of a sequence split along T
    across `group` (rank order = segment order). S0 is the sequence's initial
    state (the same on every rank, or None for zeros). Returns (y_i, S_end_i);
    the last rank's S_end is the sequence's final state."""
    ops = ops or _LibOps
    args = (q, k, v, e, w, g, z, log_alpha, r)
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    Phi, Psi = ops.segment_map(args, chunk)
    phis = [torch.empty_like(Phi) for _ in range(world)]
    psis = [torch.empty_like(Psi) for _ in range(world)]
    dist.all_gather(phis, Phi.contiguous(), group=group)
    dist.all_gather(psis, Psi.contiguous(), group=group)
    S = S0
    for i in range(rank):  # the predecessors' segments, in order
        S = ops.apply_map(phis[i], psis[i], S)
    return ops.forward(args, chunk, S)
