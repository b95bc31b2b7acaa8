"""Seeded synthetic inputs for the Muir gated delta-rule operator.

This module only draws random numbers and shapes them; it holds none of the
operator's arithmetic. Both the CUDA path (benchmarks, GPU tests) and the fp64
oracle (tests) consume what it produces, so the two sides see identical inputs.

Value recipe (the pages describe the 1.34B model only in prose; the recipe below
is the plainest reading of the workload descriptions):

* q, k: standard normal, then SiLU, then L2-normalised over the head dimension
  (the operator receives already-activated, unit-norm keys and queries; the
  arXiv abstract names "key activation and unit normalization").
* v: standard normal.
* e, w, g, z (erase, write, dynamic read, output gates): sigmoid of a standard
  normal, i.e. values in (0, 1).
* channel decay: each (head, key-row) pair gets a base rate c drawn
  log-uniformly from a range; each token then jitters the rate in log space,
  rate = c * exp(eps), eps ~ N(0, 0.1), and log_alpha = -rate <= 0 (alpha is in
  (0, 1]). Jitter in log space keeps the rate positive even for c = 1e-3.
* static readout scale: r_i = (1 - alpha_bar_i) ** 0.5 with alpha_bar_i =
  exp(-c_i), the jitter-free decay of the row: an inverse square root of the
  row's expected energy (the pages call it an inverse fractional power law).
* bimodal stress decay: half the rows of every head (a seeded permutation) get
  c in [1e-5, 1e-4], the other half c in [2, 8].

All tensors use the layout the library takes: [B, T, H, d] token-major, r [H, dk].
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    """One synthetic operator workload (sizes + value distribution)."""

    name: str
    B: int
    T: int
    H: int
    dk: int
    dv: int
    chunk: int
    dtype: str  # "f32" or "bf16": dtype of q,k,v,e,w,g,z,y; log_alpha and state stay fp32
    rate_lo: float = 1e-3
    rate_hi: float = 0.5
    bimodal: bool = False
    seed: int = 0
    extra: dict = field(default_factory=dict)


# The five workloads the operator is specified on.
TINY = Workload("tiny_f32_B1_T256_H2_d32_C64", 1, 256, 2, 32, 32, 64, "f32", 1e-3, 0.5, False, 0)
TRAIN_FWD = Workload("train_fwd_bf16_B8_T4096_H16_d128", 8, 4096, 16, 128, 128, 128, "bf16", 1e-4, 0.7, False, 1)
TRAIN_FWD_BWD = Workload("train_fwdbwd_bf16_B1_T32768_H16_d128_C128", 1, 32768, 16, 128, 128, 128, "bf16", 1e-4, 0.7, False, 2)
DECODE = Workload("decode_f32state_L24_H16_d128", 1, 1, 16, 128, 128, 128, "bf16", 1e-4, 0.7, False, 3,
                  {"layers": 24, "batches": (1, 8, 64), "prefill": 4096, "steps": 1 << 20, "drift_every": 1 << 16})
STRESS = Workload("stress_f32_B2_T32768_H16_d128_C256", 2, 32768, 16, 128, 128, 256, "f32", 0, 0, True, 4)

WORKLOADS = {w.name: w for w in (TINY, TRAIN_FWD, TRAIN_FWD_BWD, DECODE, STRESS)}


def _rng(seed: int, stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64([seed, stream]))


def base_rates(H: int, dk: int, rate_lo: float, rate_hi: float, bimodal: bool, seed: int) -> np.ndarray:
    """Per (head, key row) base decay rate c, float64 [H, dk]."""
    rng = _rng(seed, 100)
    if bimodal:
        c = np.empty((H, dk))
        for h in range(H):
            perm = rng.permutation(dk)
            slow, fast = perm[: dk // 2], perm[dk // 2:]
            c[h, slow] = np.exp(rng.uniform(np.log(1e-5), np.log(1e-4), size=slow.size))
            c[h, fast] = rng.uniform(2.0, 8.0, size=fast.size)
        return c
    return np.exp(rng.uniform(np.log(rate_lo), np.log(rate_hi), size=(H, dk)))


def _unit_silu(x: np.ndarray) -> np.ndarray:
    s = x / (1.0 + np.exp(-x))
    n = np.sqrt((s * s).sum(-1, keepdims=True))
    return s / np.maximum(n, 1e-12)


def _sigmoid(x: np.ndarray) -> np.ndarray:
    return 1.0 / (1.0 + np.exp(-x))


def round_to(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round to the storage dtype and return float64 holding exactly those values."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    if dtype == "bf16":
        t = t.to(torch.bfloat16)
    return t.to(torch.float64).numpy()


def make_inputs(B: int, T: int, H: int, dk: int, dv: int, *, dtype: str = "f32",
                rate_lo: float = 1e-3, rate_hi: float = 0.5, bimodal: bool = False,
                seed: int = 0, with_state: bool = False, with_grads: bool = False) -> dict:
    """Draw one seeded input set. Returns float64 numpy arrays holding values that
    are exactly representable in the storage dtype (bf16 or fp32), so the oracle
    and the kernel see the same numbers."""
    c = base_rates(H, dk, rate_lo, rate_hi, bimodal, seed)
    rng = _rng(seed, 1)
    out = {}
    out["q"] = round_to(_unit_silu(rng.standard_normal((B, T, H, dk))), dtype)
    out["k"] = round_to(_unit_silu(rng.standard_normal((B, T, H, dk))), dtype)
    out["v"] = round_to(rng.standard_normal((B, T, H, dv)), dtype)
    out["e"] = round_to(_sigmoid(rng.standard_normal((B, T, H, dk))), dtype)
    out["w"] = round_to(_sigmoid(rng.standard_normal((B, T, H, dv))), dtype)
    out["g"] = round_to(_sigmoid(rng.standard_normal((B, T, H, dk))), dtype)
    out["z"] = round_to(_sigmoid(rng.standard_normal((B, T, H, dv))), dtype)
    eps = 0.1 * rng.standard_normal((B, T, H, dk))
    out["log_alpha"] = round_to(-(c[None, None] * np.exp(eps)), "f32")
    out["r"] = round_to(np.sqrt(1.0 - np.exp(-c)), "f32")
    if with_state:
        out["S0"] = round_to(0.5 * rng.standard_normal((B, H, dk, dv)), "f32")
    if with_grads:
        out["dy"] = round_to(rng.standard_normal((B, T, H, dv)), dtype)
        out["dS_T"] = round_to(0.1 * rng.standard_normal((B, H, dk, dv)), "f32")
    return out


def workload_inputs(wl: Workload, **kw) -> dict:
    return make_inputs(wl.B, wl.T, wl.H, wl.dk, wl.dv, dtype=wl.dtype, rate_lo=wl.rate_lo,
                       rate_hi=wl.rate_hi, bimodal=wl.bimodal, seed=wl.seed, **kw)


def device_inputs(B: int, T: int, H: int, dk: int, dv: int, *, dtype: str, rate_lo: float,
                  rate_hi: float, bimodal: bool, seed: int, device, with_grads: bool = False) -> dict:
    """Same distributions drawn directly on a device with torch's generator (used
    for large benchmark tensors; parity tests use make_inputs)."""
    c = torch.from_numpy(base_rates(H, dk, rate_lo, rate_hi, bimodal, seed)).to(device=device, dtype=torch.float32)
    gen = torch.Generator(device=device)
    gen.manual_seed(seed * 1000003 + 7)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32

    def normal(*shape):
        return torch.randn(*shape, generator=gen, device=device, dtype=torch.float32)

    def unit_silu(x):
        s = torch.nn.functional.silu(x)
        return s / s.norm(dim=-1, keepdim=True).clamp_min(1e-12)

    out = {
        "q": unit_silu(normal(B, T, H, dk)).to(tdt),
        "k": unit_silu(normal(B, T, H, dk)).to(tdt),
        "v": normal(B, T, H, dv).to(tdt),
        "e": torch.sigmoid(normal(B, T, H, dk)).to(tdt),
        "w": torch.sigmoid(normal(B, T, H, dv)).to(tdt),
        "g": torch.sigmoid(normal(B, T, H, dk)).to(tdt),
        "z": torch.sigmoid(normal(B, T, H, dv)).to(tdt),
    }
    out["log_alpha"] = -(c[None, None] * torch.exp(0.1 * normal(B, T, H, dk)))
    out["r"] = torch.sqrt(1.0 - torch.exp(-c)).contiguous()
    if with_grads:
        out["dy"] = normal(B, T, H, dv).to(tdt)
        out["dS_T"] = 0.1 * normal(B, H, dk, dv)
    return out


def stream_inputs(rows: int, T: int, H: int, dk: int, dv: int, *, c: torch.Tensor, dtype: str, seed: int,
                  device, token_major: bool = True, out: dict | None = None) -> dict:
    """One window of a decode stream with fixed per-(head, key row) base decay
    rates c [H, dk] (fp32, on `device`): the same distributions as device_inputs,
    with only the per-token jitter redrawn. token_major=True gives [T, rows, H, d]
    (token t of every row is one contiguous slice, as a decode step takes it);
    otherwise [rows, T, H, d]. With `out`, the tensors are written into those
    buffers (same shapes and dtypes) instead of new ones."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed * 1000003 + 11)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    shape = (lambda d: (T, rows, H, d)) if token_major else (lambda d: (rows, T, H, d))

    def normal(d):
        return torch.randn(*shape(d), generator=gen, device=device, dtype=torch.float32)

    def unit_silu(x):
        s = torch.nn.functional.silu(x)
        return s / s.norm(dim=-1, keepdim=True).clamp_min(1e-12)

    vals = {
        "q": lambda: unit_silu(normal(dk)).to(tdt),
        "k": lambda: unit_silu(normal(dk)).to(tdt),
        "v": lambda: normal(dv).to(tdt),
        "e": lambda: torch.sigmoid(normal(dk)).to(tdt),
        "w": lambda: torch.sigmoid(normal(dv)).to(tdt),
        "g": lambda: torch.sigmoid(normal(dk)).to(tdt),
        "z": lambda: torch.sigmoid(normal(dv)).to(tdt),
        "log_alpha": lambda: -(c * torch.exp(0.1 * normal(dk))),
    }
    res = {}
    for n, f in vals.items():
        x = f()
        if out is not None:
            out[n].copy_(x)
            res[n] = out[n]
        else:
            res[n] = x
        del x
    res["r"] = torch.sqrt(1.0 - torch.exp(-c)).contiguous()
    return res
