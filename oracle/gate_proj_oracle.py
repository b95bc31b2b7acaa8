"""fp64 CPU oracle for Muir's fused low-rank gate projection.

TEST INFRASTRUCTURE ONLY. Nothing in the product path (the CUDA library, its
Python binding, the benchmark's GPU arm) may import or call this module; only
the tests and the benchmark's CPU-baseline arm do. It shares no code with the
CUDA path.

Source: openai-hub article "Google Research 提出 Muir：25MB 固定状态跑完千万 Token",
section "五套门控被压进一个低秩投影" and its table, and the liuch.name post, second
bullet ("13x write-vs-erase sensitivity"): the five gates (decay, erase,
output, write, dynamic read) share one down-projection of total rank 512 and
each gets its own up-projection, with ranks 64, 64, 128, 128 and 128 in the
table's order.

Readings where the pages are silent (listed in the design notes):
  * h = x W_down is split into consecutive rank slices in the table's order:
    decay [0, 64), erase [64, 128), output [128, 256), write [256, 384),
    read [384, 512);
  * u_j = h_j U_j, no biases;
  * the decay gate is emitted as log alpha = log sigmoid(u) (so alpha is in
    (0, 1)), the other four as sigmoid(u).

Layout: x [N, D]; W_down [D, 512]; U_decay, U_erase [64, Ok]; U_out, U_write
[128, Ov]; U_read [128, Ok]; outputs [N, Ok] (log_alpha, e, g) and [N, Ov]
(z, w), Ok = H d_k and Ov = H d_v, i.e. the operator's [B, T, H, d] layout with
the tokens flattened. Everything is computed in float64.
"""
from __future__ import annotations

import numpy as np

RANKS = (64, 64, 128, 128, 128)  # decay, erase, output, write, read
TOTAL_RANK = 512


def rank_slices():
    """[start, end) of each gate's slice of h, in the table's order."""
    out, s = [], 0
    for r in RANKS:
        out.append((s, s + r))
        s += r
    return out


def sigmoid(u):
    u = np.asarray(u, dtype=np.float64)
    out = np.empty_like(u)
    pos = u >= 0
    out[pos] = 1.0 / (1.0 + np.exp(-u[pos]))
    eu = np.exp(u[~pos])
    out[~pos] = eu / (1.0 + eu)
    return out


def log_sigmoid(u):
    """log(1 / (1 + exp(-u))) = -log(1 + exp(-u)), evaluated without overflow."""
    u = np.asarray(u, dtype=np.float64)
    return -np.logaddexp(0.0, -u)


def gate_proj(x, w_down, u_decay, u_erase, u_out, u_write, u_read):
    """The five gate tensors of a token batch: (log_alpha, e, z, w, g)."""
    x = np.asarray(x, dtype=np.float64)
    h = x @ np.asarray(w_down, dtype=np.float64)
    ups = [u_decay, u_erase, u_out, u_write, u_read]
    u = [h[:, a:b] @ np.asarray(U, dtype=np.float64) for (a, b), U in zip(rank_slices(), ups)]
    return log_sigmoid(u[0]), sigmoid(u[1]), sigmoid(u[2]), sigmoid(u[3]), sigmoid(u[4])
