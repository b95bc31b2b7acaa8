"""The streaming-decode workload in full: 24 layers x 16 heads x 128x128 fp32 state
(25 MB per sequence), prefilled by the chunked forward over 4096 tokens, then
stepped one token at a time by muir_decode_step (all 24 layers of every sequence
in one launch) for 1,048,576 tokens at batch 1 and 8, and for two 65,536-token
windows at batch 64.

Drift check (reading D12): at the end of every 65,536-token window the decoded
state is compared with a chunked recompute of the same window (muir_chunk_fwd,
chunk 128) from the same start state, final-state metric <= 1e-3; the decoded
outputs are compared with the recompute's outputs, <= 2e-2. The next window
starts both from the decoded state. Once per window one (layer, head) chain of
the window's last stretch is also recomputed by the fp64 oracle from the decoded
state at the stretch's start.

Decay rates stay fixed per (head, key row) along the stream (only the per-token
jitter is redrawn), the recipe of the training workloads. The decode steps of a
stretch run as one CUDA graph replay (the launches are the library's own)."""
import numpy as np
import pytest
import torch

import gated_delta_rule_muir_b200 as muir
from gated_delta_rule_muir_b200.inputs import DECODE, base_rates, stream_inputs
from oracle import muir_oracle as orc
from tests.gpu_util import INPUT_NAMES, rel_err

pytestmark = pytest.mark.gpu

STEP_NAMES = INPUT_NAMES[:8]  # q k v e w g z log_alpha; r is shared


def _rel_dev(a, b):
    """max |a - b| / max |b| on the device (b the reference)."""
    a, b = a.double(), b.double()
    return float(((a - b).abs().max() / b.abs().max().clamp_min(1e-30)).item())


def _run_stream(batch, windows, sub, seed0):
    dev = torch.device("cuda")
    L, H, dk, dv = DECODE.extra["layers"], DECODE.H, DECODE.dk, DECODE.dv
    rows = L * batch
    win = DECODE.extra["drift_every"]
    assert win % sub == 0
    c = torch.from_numpy(base_rates(H, dk, DECODE.rate_lo, DECODE.rate_hi, False, DECODE.seed)).to(dev, torch.float32)
    # token-major stretch buffers, and the same stretches row-major for the chunked forward
    tdt = torch.bfloat16
    buf = {n: torch.empty(sub, rows, H, dk if n in ("q", "k", "e", "g", "log_alpha") else dv,
                          dtype=torch.float32 if n == "log_alpha" else tdt, device=dev) for n in STEP_NAMES}
    rm = {n: torch.empty_like(buf[n].transpose(0, 1), memory_format=torch.contiguous_format) for n in STEP_NAMES}
    r = torch.sqrt(1.0 - torch.exp(-c)).contiguous()
    ws = torch.empty(muir.chunk_fwd_workspace_bytes(*[rm[n] for n in STEP_NAMES], r, 128), dtype=torch.uint8,
                     device=dev)
    # prefill: the chunked forward over 4096 tokens from a zero state, one stretch at a time
    S_dec = None
    for j in range(DECODE.extra["prefill"] // sub):
        stream_inputs(rows, sub, H, dk, dv, c=c, dtype="bf16", seed=seed0 + 500000 + j, device=dev,
                      token_major=False, out=rm)
        _, S_dec = muir.chunk_fwd(*[rm[n] for n in STEP_NAMES], r, chunk=128, S0=S_dec, workspace=ws)
    ybuf = torch.empty(sub, rows, H, dv, dtype=tdt, device=dev)
    stream_inputs(rows, sub, H, dk, dv, c=c, dtype="bf16", seed=seed0 + 1, device=dev, out=buf)
    S_warm = S_dec.clone()
    calls = lambda S: [muir.decode_step(S, *[buf[n][t] for n in STEP_NAMES], r, y=ybuf[t]) for t in range(sub)]
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        calls(S_warm)  # warm-up outside the capture (on a scratch copy of the state)
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        calls(S_dec)
    del S_warm
    report = []
    for w in range(windows):
        S_chk = S_dec.clone()  # the recompute starts from the decoded state (D12)
        y_err = 0.0
        nsub = win // sub
        for j in range(nsub):
            seed = seed0 + 2 + w * nsub + j
            stream_inputs(rows, sub, H, dk, dv, c=c, dtype="bf16", seed=seed, device=dev, out=buf)
            for n in STEP_NAMES:  # [rows, sub, H, d] for the chunked recompute
                rm[n].copy_(buf[n].transpose(0, 1))
            y_c, S_chk = muir.chunk_fwd(*[rm[n] for n in STEP_NAMES], r, chunk=128, S0=S_chk, workspace=ws)
            last = j == nsub - 1
            if last:  # oracle spot check of this stretch: one (layer, head) chain
                row, h = (5 * w + 3) % rows, (7 * w + 2) % H
                S_at = S_dec[row:row + 1, h:h + 1].double().cpu().numpy()
                chain = {n: rm[n][row:row + 1, :, h:h + 1].double().cpu().numpy() for n in STEP_NAMES}
                chain["r"] = r[h:h + 1].double().cpu().numpy()
            graph.replay()
            y_err = max(y_err, _rel_dev(ybuf.transpose(0, 1), y_c))
        s_err = _rel_dev(S_dec, S_chk)
        y_ref, S_ref = orc.forward(*[chain[n] for n in INPUT_NAMES], S0=S_at)
        o_y = rel_err(ybuf[:, row:row + 1, h:h + 1].transpose(0, 1), y_ref)
        o_s = rel_err(S_dec[row:row + 1, h:h + 1], S_ref)
        report.append((w, s_err, y_err, o_s, o_y))
        assert s_err < 1e-3, report
        assert y_err < 2e-2, report
        assert o_s < 1e-3 and o_y < 2e-2, report
    del graph
    assert muir.device_status() == 0
    assert bool(torch.isfinite(S_dec).all())
    return report


@pytest.mark.parametrize("batch,windows,sub", [(1, 16, 4096), (8, 16, 1024), (64, 2, 128)])
def test_decode_stream_drift(cuda_ok, batch, windows, sub):
    """batch 1 and 8: 16 windows = 1,048,576 decode steps; batch 64: two windows."""
    report = _run_stream(batch, windows, sub, seed0=1000 * batch)
    print(f"decode stream batch {batch}: (window, state err, y err, oracle state err, oracle y err)")
    for line in report:
        print("  ", line)
