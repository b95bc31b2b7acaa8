"""Parity of the fused gate projection (muir_gate_proj, through the C ABI) with the
fp64 oracle, element by element: small sizes spanning several 128-token tiles and
a ragged tail, the degenerate sizes, and the full-size launch on sampled token
rows (each token's gates depend on its own row of x only)."""
import numpy as np
import pytest
import torch

import gated_delta_rule_muir_b200 as muir
from oracle import gate_proj_oracle as gpo

pytestmark = pytest.mark.gpu

NAMES = ("log_alpha", "e", "z", "w", "g")


def _weights(rng, D, Ok, Ov):
    """h ~ N(0, 1) and u ~ N(0, 1) for x ~ N(0, 1): gates spread over (0, 1)."""
    wd = rng.normal(size=(D, 512)) / np.sqrt(D)
    ups = [rng.normal(size=(r, o)) / np.sqrt(r) for r, o in zip(gpo.RANKS, (Ok, Ok, Ov, Ov, Ok))]
    return wd, ups


def _run(x, wd, ups, dtype):
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to("cuda", dtype)
    out = muir.gate_proj(dev(x), dev(wd), *[dev(u) for u in ups])
    torch.cuda.synchronize()
    assert muir.device_status() == 0
    return {k: v.double().cpu().numpy() for k, v in out.items()}


def _as_dtype(a, dtype):
    """The inputs as the device holds them (bf16 rounding), in float64."""
    return torch.from_numpy(np.ascontiguousarray(a)).to(dtype).double().numpy()


def _check(got, ref, dtype):
    # fp32: h and u carry fp32 accuracy (3-pass hi/lo products). bf16 outputs are
    # rounded to 8 significant bits: half an ulp of a value in (0, 1) is <= 2^-9.
    for name, r in zip(NAMES, ref):
        g = got[name]
        assert np.all(np.isfinite(g)), name
        if name == "log_alpha":  # fp32 output in both dtypes
            tol = 2e-5 + 1e-4 * np.abs(r) if dtype == torch.float32 else 2e-4 + 1e-3 * np.abs(r)
        else:
            tol = 1e-5 if dtype == torch.float32 else 2.5e-3
        err = np.abs(g - r)
        assert np.all(err <= tol), (name, float(err.max()))


@pytest.mark.parametrize("dtype,N,D,Ok,Ov", [
    (torch.float32, 300, 128, 256, 256),
    # fp32 with several K steps and several U chunks per gate (the prefetch of
    # the next chunk and the reuse of the staged h), and a ragged last tile
    (torch.float32, 389, 256, 512, 768),
    (torch.bfloat16, 333, 256, 512, 256),
    (torch.bfloat16, 5, 64, 256, 512),
])
def test_gate_proj_matches_oracle(dtype, N, D, Ok, Ov):
    rng = np.random.default_rng(11 + N)
    x = rng.normal(size=(N, D))
    wd, ups = _weights(rng, D, Ok, Ov)
    x, wd, ups = _as_dtype(x, dtype), _as_dtype(wd, dtype), [_as_dtype(u, dtype) for u in ups]
    got = _run(x, wd, ups, dtype)
    _check(got, gpo.gate_proj(x, wd, *ups), dtype)


def test_gate_proj_empty_batch_launches_nothing():
    dev = lambda *s: torch.zeros(*s, dtype=torch.bfloat16, device="cuda")
    before = muir.launch_count()
    out = muir.gate_proj(dev(0, 64), dev(64, 512), dev(64, 256), dev(64, 256), dev(128, 256), dev(128, 256),
                         dev(128, 256))
    assert muir.launch_count() == before
    assert all(v.shape[0] == 0 for v in out.values())


def test_gate_proj_full_size_sampled_rows():
    """The benchmark's launch: 32,768 tokens, d_model 2048, H*d = 2048, bf16."""
    N, D, Ok, Ov = 32768, 2048, 2048, 2048
    g = torch.Generator(device="cuda").manual_seed(7)
    x = torch.randn(N, D, device="cuda", generator=g).to(torch.bfloat16)
    wd = (torch.randn(D, 512, device="cuda", generator=g) / D ** 0.5).to(torch.bfloat16)
    ups = [(torch.randn(r, o, device="cuda", generator=g) / r ** 0.5).to(torch.bfloat16)
           for r, o in zip(gpo.RANKS, (Ok, Ok, Ov, Ov, Ok))]
    out = muir.gate_proj(x, wd, *ups)
    torch.cuda.synchronize()
    assert muir.device_status() == 0
    rows = np.r_[0:3, 127:130, np.random.default_rng(0).integers(0, N, 40), N - 3:N]
    ref = gpo.gate_proj(x[rows].double().cpu().numpy(), wd.double().cpu().numpy(),
                        *[u.double().cpu().numpy() for u in ups])
    got = {k: v[rows].double().cpu().numpy() for k, v in out.items()}
    _check(got, ref, torch.bfloat16)
