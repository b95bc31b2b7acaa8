"""Helpers shared by the GPU parity tests (no operator arithmetic here)."""
import numpy as np
import torch

INPUT_NAMES = ("q", "k", "v", "e", "w", "g", "z", "log_alpha", "r")


def to_dev(d, dtype, device="cuda"):
    """numpy float64 inputs (already exactly representable) -> CUDA tensors in the
    storage dtypes the library takes."""
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    out = {}
    for n, x in d.items():
        keep32 = n in ("log_alpha", "r", "S0", "dS_T")
        out[n] = torch.tensor(x, dtype=torch.float32).to(torch.float32 if keep32 else tdt).to(device).contiguous()
    return out


def rel_err(a, b):
    """max |a - b| / max |b| (b = oracle, float64)."""
    if isinstance(a, torch.Tensor):
        a = a.detach().double().cpu().numpy()
    b = np.asarray(b, dtype=np.float64)
    den = max(float(np.max(np.abs(b))), 1e-30)
    return float(np.max(np.abs(a - b))) / den
