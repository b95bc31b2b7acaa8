"""The exchange of gated_delta_rule_muir_b200.sequence on CPU with three gloo
ranks: each rank's segment map, all-gathered, composed over its predecessors,
gives every rank its start state, and the segments' outputs and the last
rank's final state equal the whole-sequence recurrence. The segment maps and
their application are the oracle's here (the GPU kernels are tested in
test_gpu_sequence.py)."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from gated_delta_rule_muir_b200.inputs import make_inputs
from gated_delta_rule_muir_b200.sequence import chunk_fwd_sequence_parallel
from oracle import muir_oracle as orc

NAMES = ("q", "k", "v", "e", "w", "g", "z", "log_alpha", "r")


class OracleOps:
    """Segment maps by probing the oracle's forward (the map is affine in S0)."""

    @staticmethod
    def segment_map(args, chunk):
        a = [None if x is None else x.numpy() for x in args]
        B, H, dk, dv = a[0].shape[0], a[0].shape[2], a[0].shape[3], a[2].shape[3]
        _, Psi = orc.forward(*a, S0=np.zeros((B, H, dk, dv)))
        Phi = np.zeros((B, H, dk, dk))
        for c in range(dk):
            S0 = np.zeros((B, H, dk, dv))
            S0[:, :, c, 0] = 1.0
            _, S_T = orc.forward(*a, S0=S0)
            Phi[:, :, :, c] = (S_T - Psi)[:, :, :, 0]
        return torch.from_numpy(Phi), torch.from_numpy(Psi)

    @staticmethod
    def apply_map(Phi, Psi, S):
        return Psi.clone() if S is None else Phi @ S + Psi

    @staticmethod
    def forward(args, chunk, S0):
        a = [None if x is None else x.numpy() for x in args]
        y, S_T = orc.forward(*a, S0=None if S0 is None else S0.numpy())
        return torch.from_numpy(y), torch.from_numpy(S_T)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, bounds, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        d = make_inputs(1, bounds[-1], 2, 4, 3, dtype="f32", rate_lo=1e-2, rate_hi=0.5, seed=21, with_state=True)
        lo, hi = bounds[rank], bounds[rank + 1]
        args = [torch.from_numpy(d[n]) if n == "r" else torch.from_numpy(d[n][:, lo:hi]) for n in NAMES]
        y, S_end = chunk_fwd_sequence_parallel(*args, chunk=8, S0=torch.from_numpy(d["S0"]), ops=OracleOps)
        out[rank] = (y.numpy(), S_end.numpy())
    finally:
        dist.destroy_process_group()


def test_three_gloo_ranks_split_the_sequence():
    bounds = (0, 16, 24, 40)
    world = len(bounds) - 1
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(world, _free_port(), bounds, out), nprocs=world, start_method="spawn")
        res = dict(out)
    d = make_inputs(1, bounds[-1], 2, 4, 3, dtype="f32", rate_lo=1e-2, rate_hi=0.5, seed=21, with_state=True)
    y_ref, S_ref = orc.forward(*[d[n] for n in NAMES], S0=d["S0"])
    y = np.concatenate([res[i][0] for i in range(world)], axis=1)
    np.testing.assert_allclose(y, y_ref, rtol=0, atol=1e-10)
    np.testing.assert_allclose(res[world - 1][1], S_ref, rtol=0, atol=1e-10)
