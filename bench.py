#!/usr/bin/env python
"""Benchmark of the Muir gated delta-rule hot path on B200.

One step = the chunkwise forward and backward pass (libmuir.so) over the
training-shape workload B=1, T=32768, H=16, dk=dv=128, chunk=128, bf16 inputs,
fp32 state, random upstream gradient. The same run measures the streaming decode
step (24 layers x 16 heads x 128x128 fp32 state, batch 1/8/64) as GB/s of state
traffic. Prints one JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl muir|reference]

N > 1 runs under torch.distributed (one process per GPU, NCCL): every rank runs
its own replica of the workload (the operator has no cross-GPU exchange at this
shape), the timed region is bracketed by barriers and the slowest rank's time
is reported. --impl reference times the fp64 CPU oracle on a bounded sample of
the same workload on the host cores (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "chunk fwd+bwd tokens/s (H=16,d=128) & % TC peak; decode GB/s % HBM"
WL = dict(name="train_fwdbwd_bf16_B1_T32768_H16_d128_C128", B=1, T=32768, H=16, dk=128, dv=128, chunk=128,
          dtype="bf16", rate_lo=1e-4, rate_hi=0.7, seed=2)
DECODE = dict(layers=24, H=16, dk=128, dv=128, batches=(1, 8, 64))
CPU_SAMPLE_T = 1024  # oracle sample: all 16 heads, first 1024 tokens, fwd + bwd
REF_SAMPLE_T = 256   # per-step sample of the reference arm


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return dict(hbm=p["hbm_gbs"], bf16=p["bf16_tflops"], bf16_sus=p["bf16_tflops_sustained"], src="measured")
    except Exception:
        return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


# ---------------------------------------------------------------------------
# Algorithmic work per unit (one chunk of C tokens of one (batch, head)) for each
# kernel: (flops, bytes). Flops count each multiply-add as 2, triangles once,
# and the math once (the 3-pass bf16 split is an implementation cost, not work).
# Bytes are the kernel's compulsory global traffic for its interface.
# ---------------------------------------------------------------------------
def kernel_model(C, dk, dv, es):
    f4 = 4
    tri = C * C / 2
    m = {}
    m["decay"] = (0.0, C * dk * f4 + 4 * C * dk * f4)
    # off-diagonal blocks (tensor cores) + the exact 8x8 diagonal blocks (CUDA cores)
    m["gram"] = (4 * 2 * (tri - C * 4) * dk + 4 * 2 * C * 4.5 * dk,
                     4 * C * dk * es + 3 * C * dk * f4 + 4 * C * C * f4)
    m["solve"] = (C ** 3 / 3.0, 2 * C * C * f4)
    maps_fl = 2 * (tri * dk + tri * dv + tri * dv + C * dk * dk + tri * dk + 2 * tri * dv + 2 * C * dk * dv)
    m["maps"] = (maps_fl, 4 * C * C * f4 + 6 * C * dk * es + 2 * C * dk * f4 + (dk + C) * (dk + dv) * f4)
    m["scan"] = (2 * (dk + C) * dk * dv, (dk + C) * (dk + dv) * f4 + 2 * C * dv * es)
    m["scan_recompute"] = (2 * (dk + C) * dk * dv, (dk + C) * (dk + dv) * f4 + dk * dv * f4 + 2 * C * dv * es)
    m["rscan"] = (2 * (dk + C) * dk * dv, (dk + C) * dk * f4 + 2 * dk * dv * f4 + 2 * C * dv * es)
    m["out"] = (2 * C * dk * dv, C * dk * f4 + dk * dv * f4 + C * dv * f4 + 2 * C * dv * es)
    m["bwd_pe"] = (3 * 2 * C * dk * dv, 2 * C * dk * f4 + 2 * dk * dv * f4 + 3 * C * dv * f4 + 3 * C * dv * es)
    m["bwd_dz"] = (2 * (tri * dv + C * dk * dv + tri * dv + tri * dv + C * dk * dv + tri * dv),
                   3 * C * C * f4 + 2 * C * dv * es + dk * dv * f4 + 2 * C * dk * es + 2 * C * dv * f4)
    m["bwd_grads"] = (2 * (4 * C * dk * dv + 4 * tri * dv),
                      4 * C * dv * f4 + 2 * dk * dv * f4 + 2 * C * dv * es + 4 * C * dk * f4 + 4 * C * C * f4)
    m["bwd_gram"] = (4 * 2 * 2 * (tri - C * 8) * dk + 4 * 2 * 2 * C * 8.5 * dk, 4 * C * C * f4 + 4 * C * dk * es + 2 * C * dk * f4 + 4 * C * dk * f4)
    m["bwd_final"] = (0.0, 14 * C * dk * f4 + 6 * C * dk * es + C * dv * f4 + 4 * C * dv * es)
    return m


def flop_split(C, dk, dv):
    """Modelled share of the step's flops issued on the tensor cores. The CUDA-core
    share counts every vector step of the kernels per unit (one chunk of one head):
    the exact diagonal Gram blocks (8x8 forward, 16x16 backward), the 16x16 leaves of
    the triangular solve, the decay products, the elementwise decay scaling of the
    staged operands and epilogues, the state additions of the scans, the output
    gate, and the chain rule of the final backward kernel (an exponential counts as
    one flop). The tensor-core share is the algorithmic MMA work of the model (each
    multiply-add 2 flops, math counted once). The instruction counts behind the
    measured split are in the ncu summary of the step's kernels."""
    m = kernel_model(C, dk, dv, 2)
    nb = C // 16
    alu = {
        "diag_blocks": 4 * 2 * C * 4.5 * dk + 4 * 2 * 2 * C * 8.5 * dk,
        "solve_leaves": nb * 16 * (16 * 15 / 2) * 2,
        "decay": 4 * C * dk,
        "operand_scaling": (12 + 8 + 3) * C * dk + 2.5 * (12 + 8 + 3) * C * dk,
        "scan_adds": 2 * dk * dv,
        "output_gate": 2 * C * dv,
        "final_chain_rule": 35 * C * dk + 4 * C * dv,
    }
    fwd = ("gram", "solve", "maps", "scan", "out")
    bwd = ("bwd_pe", "rscan", "bwd_dz", "bwd_grads", "bwd_gram")
    mma = sum(m[k][0] for k in fwd + bwd) - alu["diag_blocks"] - alu["solve_leaves"]
    tot_alu = sum(alu.values())
    return {"mma_share": round(mma / (mma + tot_alu), 4), "alu_share": round(tot_alu / (mma + tot_alu), 4),
            "alu_terms_per_unit": {k: round(v) for k, v in alu.items()},
            "note": "modelled per unit of the step's kernels; the pages report 98% on matrix units"}


def pass_work(C, d, es):
    """Algorithmic work per head-token of the forward and the backward pass (the
    survey's measurement section): flops count a multiply-add as 2, triangles once
    and no zero tile; bytes are the compulsory HBM traffic of the pass's inputs and
    outputs (es = bytes per input element; log_alpha and the state are fp32).
    Returns (fwd_flops, fwd_bytes, bwd_flops, bwd_bytes)."""
    fwd_fl = 8 * C * d + C * C / 3 + 8 * d * d
    bwd_fl = 22 * C * d + C * C / 3 + 22 * d * d
    fwd_by = 7 * d * es + 4 * d + d * es          # q k v e w g z, log_alpha, y
    bwd_by = (7 * d * es + 4 * d) + d * es + 7 * d * es + 4 * d + 2 * 4 * d  # inputs, dy, grads, dlog_alpha, states
    return fwd_fl, fwd_by, bwd_fl, bwd_by


def algorithmic_step():
    """Work of one fwd+bwd step of the whole path at the benchmark's shape: flops and bytes."""
    ht = WL["B"] * WL["T"] * WL["H"]
    ff, fb, bf, bb = pass_work(WL["chunk"], WL["dk"], 2)
    return ht * (ff + bf), ht * (fb + bb)


class ClockSampler:
    """nvidia-smi clock/throttle samples during the timed region."""

    FIELDS = "index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown," \
             "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown," \
             "clocks_event_reasons.sw_power_cap"

    def __init__(self, index):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "200", "-i", str(self.index)], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.3)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]
        return False

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def make_workload(dev):
    import torch
    from gated_delta_rule_muir_b200.inputs import device_inputs
    d = device_inputs(WL["B"], WL["T"], WL["H"], WL["dk"], WL["dv"], dtype=WL["dtype"], rate_lo=WL["rate_lo"],
                      rate_hi=WL["rate_hi"], bimodal=False, seed=WL["seed"], device=dev, with_grads=True)
    torch.cuda.synchronize()
    return d


NAMES = ("q", "k", "v", "e", "w", "g", "z", "log_alpha", "r")


class Step:
    """Preallocated fwd+bwd step through the public binding."""

    fwd_only = False

    def __init__(self, d):
        import torch
        import gated_delta_rule_muir_b200 as muir
        self.muir = muir
        self.d = d
        self.args = [d[n] for n in NAMES]
        C = WL["chunk"]
        self.y = torch.empty_like(d["v"])
        self.S = torch.empty(WL["B"], WL["H"], WL["dk"], WL["dv"], device=d["q"].device)
        nf = muir.chunk_fwd_workspace_bytes(*self.args, C)
        nb = muir.chunk_bwd_workspace_bytes(*self.args, C)
        self.ws = torch.empty(max(nf, nb), dtype=torch.uint8, device=d["q"].device)
        if not self.fwd_only:
            # the forward keeps its chunk maps for the backward (no recomputation)
            muir.chunk_fwd(*self.args, chunk=C, y=self.y, S_T=self.S, workspace=self.ws, save_for_bwd=True)
            self.grads = muir.chunk_bwd(*self.args, d["dy"], chunk=C, workspace=self.ws, use_saved=True)

    def fwd(self):
        self.muir.chunk_fwd(*self.args, chunk=WL["chunk"], y=self.y, S_T=self.S, workspace=self.ws,
                            save_for_bwd=not self.fwd_only)

    def bwd(self):
        if not self.fwd_only:
            self.muir.chunk_bwd(*self.args, self.d["dy"], chunk=WL["chunk"], workspace=self.ws, outputs=self.grads,
                                use_saved=True)

    def __call__(self):
        self.fwd()
        self.bwd()


def max_over_ranks(ms, device):
    """The slowest rank's time: every rank contributes its own device time and
    gets back the maximum (the whole job is done when the last replica is)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(ms)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, tokens_per_rank, ms_per_step):
    """Whole-job tokens/s of `world` replicas that each process `tokens_per_rank`
    tokens per step, timed by the slowest rank."""
    return world * tokens_per_rank / (ms_per_step * 1e-3)


def time_step_passes(step, steps, dist_on):
    """Time `steps` calls of step() as time_steps does, and also each call's forward
    and backward pass with CUDA events recorded between them on the launching
    stream. Returns (total ms, mean forward ms, mean backward ms)."""
    import torch
    import torch.distributed as dist
    if dist_on:
        dist.barrier()
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    for e in ev:
        e[0].record()
        step.fwd()
        e[1].record()
        step.bwd()
        e[2].record()
    torch.cuda.synchronize()
    ms = ev[0][0].elapsed_time(ev[-1][2])
    f = sum(e[0].elapsed_time(e[1]) for e in ev) / steps
    b = sum(e[1].elapsed_time(e[2]) for e in ev) / steps
    if dist_on:
        ms = max_over_ranks(ms, "cuda")
        f = max_over_ranks(f, "cuda")
        b = max_over_ranks(b, "cuda")
        dist.barrier()
    return ms, f, b


def time_steps(fn, steps, dist_on):
    import torch
    import torch.distributed as dist
    if dist_on:
        dist.barrier()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(steps):
        fn()
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b)
    if dist_on:
        ms = max_over_ranks(ms, "cuda")
        dist.barrier()
    return ms


GATE_WL = {"N": 32768, "D": 2048, "Ok": 2048, "Ov": 2048}  # tokens of the fwd+bwd workload, d_model = H*d


def bench_gate_proj(dev, steps, warmup, pk):
    """The fused gate projection (muir_gate_proj) over the fwd+bwd workload's tokens:
    x [32768, 2048] bf16 -> log_alpha (fp32), e, z, w, g (bf16). Inputs and outputs
    exceed L2. Algorithmic work: 2N(512 D + 64 Ok + 64 Ok + 128 Ov + 128 Ov + 128 Ok)
    flops; bytes = x + weights + outputs."""
    import torch
    import gated_delta_rule_muir_b200 as muir
    N, D, Ok, Ov = GATE_WL["N"], GATE_WL["D"], GATE_WL["Ok"], GATE_WL["Ov"]
    g = torch.Generator(device=dev)
    g.manual_seed(5)
    x = torch.randn(N, D, device=dev, generator=g).bfloat16()
    wd = (torch.randn(D, 512, device=dev, generator=g) / D ** 0.5).bfloat16()
    ups = [(torch.randn(r, o, device=dev, generator=g) / r ** 0.5).bfloat16()
           for r, o in zip(muir.GATE_RANKS, (Ok, Ok, Ov, Ov, Ok))]
    out = muir.gate_proj(x, wd, *ups)
    fn = lambda: muir.gate_proj(x, wd, *ups, out=out)
    for _ in range(max(warmup, 3)):
        fn()
    reps = max(steps, 10)
    ms = time_steps(fn, reps, False) / reps
    flops = 2.0 * N * (512 * D + 64 * Ok * 2 + 128 * Ov * 2 + 128 * Ok)
    byts = 2.0 * (N * D + D * 512 + sum(u.numel() for u in ups)) + N * Ok * 4 + 2.0 * N * (Ok + 2 * Ov + Ok)
    t = ms * 1e-3
    roof_ms = 1e3 * max(flops / (pk["bf16"] * 1e12), byts / (pk["hbm"] * 1e9))
    return {"workload": f"gate_proj_bf16_N{N}_D{D}_Ok{Ok}_Ov{Ov}", "ms": round(ms, 4), "tokens_s": round(N / t, 1),
            "algorithmic_TFLOP_s": round(flops / t / 1e12, 2), "frac_tc_peak": round(flops / t / 1e12 / pk["bf16"], 4),
            "algorithmic_GB_s": round(byts / t / 1e9, 1), "frac_hbm": round(byts / t / 1e9 / pk["hbm"], 4),
            "roofline_ms": round(roof_ms, 4), "frac_roofline": round(roof_ms / ms, 4), "gpu_launches": reps}


FWD_WORKLOADS = [
    # the training shape's forward alone (no saving), then the training-forward workload at every chunk
    # size, then the fp32 stress workload
    dict(name="fwd_bf16_B1_T32768_H16_d128_C128", B=1, T=32768, C=128, dtype="bf16", lo=1e-4, hi=0.7, bimodal=False,
         seed=2),
    dict(name="train_fwd_bf16_B8_T4096_H16_d128_C64", B=8, T=4096, C=64, dtype="bf16", lo=1e-4, hi=0.7,
         bimodal=False, seed=1),
    dict(name="train_fwd_bf16_B8_T4096_H16_d128_C128", B=8, T=4096, C=128, dtype="bf16", lo=1e-4, hi=0.7,
         bimodal=False, seed=1),
    dict(name="train_fwd_bf16_B8_T4096_H16_d128_C256", B=8, T=4096, C=256, dtype="bf16", lo=1e-4, hi=0.7,
         bimodal=False, seed=1),
    dict(name="stress_fwd_f32_B2_T32768_H16_d128_C256", B=2, T=32768, C=256, dtype="f32", lo=0, hi=0, bimodal=True,
         seed=4),
]


def bench_forwards(dev, steps, warmup, pk):
    """Forward-only throughput (muir_chunk_fwd, nothing saved) on each forward
    workload, against the survey's per-head-token forward work: % of the measured
    bf16 tensor peak (burst and sustained; for the fp32 workload also against the
    tf32 peak, taken as half the bf16 figure, the nominal ratio), % of the measured
    HBM bandwidth, and the fraction of the max(flops, bytes) roofline."""
    import torch
    import gated_delta_rule_muir_b200 as muir
    from gated_delta_rule_muir_b200.inputs import device_inputs
    H, d = WL["H"], WL["dk"]
    out = {}
    for wl in FWD_WORKLOADS:
        x = device_inputs(wl["B"], wl["T"], H, d, d, dtype=wl["dtype"], rate_lo=wl["lo"], rate_hi=wl["hi"],
                          bimodal=wl["bimodal"], seed=wl["seed"], device=dev)
        a = [x[n] for n in NAMES]
        y = torch.empty_like(x["v"])
        S = torch.empty(wl["B"], H, d, d, device=dev)
        ws = torch.empty(muir.chunk_fwd_workspace_bytes(*a, wl["C"]), dtype=torch.uint8, device=dev)
        fn = lambda: muir.chunk_fwd(*a, chunk=wl["C"], y=y, S_T=S, workspace=ws)
        for _ in range(max(warmup, 3)):
            fn()
        reps = max(steps, 10)
        ms = time_steps(fn, reps, False) / reps
        es = 2 if wl["dtype"] == "bf16" else 4
        ff, fb, _, _ = pass_work(wl["C"], d, es)
        ht = wl["B"] * wl["T"] * H
        t = ms * 1e-3
        tf, gb = ht * ff / t / 1e12, ht * fb / t / 1e9
        roof_ms = 1e3 * max(ht * ff / (pk["bf16"] * 1e12), ht * fb / (pk["hbm"] * 1e9))
        r = {"ms": round(ms, 4), "tokens_s": round(wl["B"] * wl["T"] / t, 1), "algorithmic_TFLOP_s": round(tf, 2),
             "frac_tc_peak": round(tf / pk["bf16"], 4), "frac_tc_peak_sustained": round(tf / pk["bf16_sus"], 4),
             "algorithmic_GB_s": round(gb, 1), "frac_hbm": round(gb / pk["hbm"], 4),
             "roofline_ms": round(roof_ms, 4), "frac_roofline": round(roof_ms / ms, 4),
             "per_head_token": {"flops": round(ff), "bytes": fb}}
        if es == 4:
            r["frac_tf32_peak"] = round(tf / (pk["bf16"] / 2), 4)
        out[wl["name"]] = r
        del x, a, y, S, ws
        torch.cuda.empty_cache()
    return out


def bench_decode(dev, steps, warmup, pk, graph=True):
    """Decode GB/s of one token through all 24 layers: one launch over the 24 x batch
    rows (per-row readout scale), and (graph=True) a CUDA graph of 24 per-layer
    launches."""
    import torch
    import gated_delta_rule_muir_b200 as muir
    out = {}
    L, H, dk, dv = DECODE["layers"], DECODE["H"], DECODE["dk"], DECODE["dv"]
    g = torch.Generator(device=dev)
    g.manual_seed(3)
    for nb in DECODE["batches"]:
        n = L * nb
        S = 0.1 * torch.randn(n, H, dk, dv, device=dev, generator=g)
        mk = lambda d: torch.randn(n, H, d, device=dev, generator=g)
        q = torch.nn.functional.normalize(torch.nn.functional.silu(mk(dk)), dim=-1).bfloat16()
        k = torch.nn.functional.normalize(torch.nn.functional.silu(mk(dk)), dim=-1).bfloat16()
        v = mk(dv).bfloat16()
        e, gg = torch.sigmoid(mk(dk)).bfloat16(), torch.sigmoid(mk(dk)).bfloat16()
        w, z = torch.sigmoid(mk(dv)).bfloat16(), torch.sigmoid(mk(dv)).bfloat16()
        la = -0.01 * torch.rand(n, H, dk, device=dev, generator=g)
        r = torch.rand(n, H, dk, device=dev, generator=g)
        y = torch.empty(n, H, dv, device=dev, dtype=torch.bfloat16)
        fn = lambda: muir.decode_step(S, q, k, v, e, w, gg, z, la, r, y=y)
        for _ in range(max(warmup, 3)):
            fn()
        reps = max(steps, 20) if graph else steps
        ms = time_steps(fn, reps, False) / reps
        state_bytes = 2.0 * n * H * dk * dv * 4
        io_bytes = n * H * (5 * dk * 2 + dk * 4 + dk * 4 + 3 * dv * 2 + dv * 2)
        gbs = (state_bytes + io_bytes) / (ms * 1e-3) / 1e9
        if not graph:
            out[f"batch{nb}"] = {"ms_per_token": round(ms, 4), "GB_s": round(gbs, 1), "frac_hbm": round(gbs / pk["hbm"], 3),
                                 "state_MB": round(n * H * dk * dv * 4 / 1e6, 1)}
            del S, q, k, v, e, gg, w, z, la, r, y
            continue
        # the same token as a CUDA graph of 24 per-layer launches (batch rows each)
        sl = [slice(l * nb, (l + 1) * nb) for l in range(L)]
        layer_calls = lambda: [muir.decode_step(S[i], q[i], k[i], v[i], e[i], w[i], gg[i], z[i], la[i], r[i], y=y[i])
                               for i in sl]
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            layer_calls()  # warm-up outside the capture
        torch.cuda.current_stream().wait_stream(side)
        cg = torch.cuda.CUDAGraph()
        with torch.cuda.graph(cg):
            layer_calls()
        for _ in range(max(warmup, 3)):
            cg.replay()
        ms_g = time_steps(cg.replay, reps, False) / reps
        del cg
        gbs_g = (state_bytes + io_bytes) / (ms_g * 1e-3) / 1e9
        out[f"batch{nb}"] = {"ms_per_token": round(ms, 4), "GB_s": round(gbs, 1), "frac_hbm": round(gbs / pk["hbm"], 3),
                             "graph24_ms_per_token": round(ms_g, 4), "graph24_GB_s": round(gbs_g, 1),
                             "state_MB": round(n * H * dk * dv * 4 / 1e6, 1),
                             "note": "state fits in L2: effective bandwidth" if n * H * dk * dv * 4 < 100e6 else "HBM"}
        del S, q, k, v, e, gg, w, z, la, r, y
    return out


def e2e_pass(d, steps, warmup):
    """Same fwd+bwd through the public API with host (pinned) inputs copied in and
    all outputs copied back inside the timed region."""
    import torch
    import gated_delta_rule_muir_b200 as muir
    dev = d["q"].device
    host = {n: d[n].cpu().pin_memory() for n in NAMES + ("dy",)}
    dbuf = {n: torch.empty_like(d[n]) for n in NAMES + ("dy",)}
    st = Step({**dbuf})
    outs_h = {"y": torch.empty_like(st.y, device="cpu").pin_memory(),
              "S_T": torch.empty_like(st.S, device="cpu").pin_memory()}
    for n, t in st.grads.items():
        if t is not None:
            outs_h[n] = torch.empty_like(t, device="cpu").pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = sum(t.numel() * t.element_size() for t in outs_h.values())

    def one():
        for n in host:
            dbuf[n].copy_(host[n], non_blocking=True)
        st()
        outs_h["y"].copy_(st.y, non_blocking=True)
        outs_h["S_T"].copy_(st.S, non_blocking=True)
        for n, t in st.grads.items():
            if t is not None:
                outs_h[n].copy_(t, non_blocking=True)

    for _ in range(warmup):
        one()
    ms = time_steps(one, steps, False) / steps
    tok = WL["B"] * WL["T"]
    return {"value": round(tok / (ms * 1e-3), 1), "unit": "tokens/s", "ms_per_step": round(ms, 3),
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)}


def oracle_sample(T_sample):
    """fwd + bwd of the fp64 oracle on all heads of the first T_sample tokens."""
    from gated_delta_rule_muir_b200.inputs import make_inputs
    from oracle import muir_oracle as orc
    d = make_inputs(WL["B"], T_sample, WL["H"], WL["dk"], WL["dv"], dtype=WL["dtype"], rate_lo=WL["rate_lo"],
                    rate_hi=WL["rate_hi"], seed=WL["seed"], with_grads=True)
    a = [d[n] for n in NAMES]
    t0 = time.perf_counter()
    orc.forward(*a)
    orc.backward(*a, d["dy"])
    return time.perf_counter() - t0


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        return 1


def oracle_forward_sample(T_sample):
    """Forward only of the fp64 oracle on all heads of the first T_sample tokens."""
    from gated_delta_rule_muir_b200.inputs import make_inputs
    from oracle import muir_oracle as orc
    d = make_inputs(WL["B"], T_sample, WL["H"], WL["dk"], WL["dv"], dtype=WL["dtype"], rate_lo=WL["rate_lo"],
                    rate_hi=WL["rate_hi"], seed=WL["seed"])
    t0 = time.perf_counter()
    orc.forward(*[d[n] for n in NAMES])
    return time.perf_counter() - t0


def oracle_decode_sample(steps):
    """Decode steps of the fp64 oracle for one sequence through all 24 layers (384 heads)."""
    from gated_delta_rule_muir_b200.inputs import make_inputs
    from oracle import muir_oracle as orc
    L, H = DECODE["layers"], DECODE["H"]
    d = make_inputs(L, steps, H, DECODE["dk"], DECODE["dv"], dtype="bf16", rate_lo=1e-4, rate_hi=0.7, seed=3,
                    with_state=True)
    S = d["S0"]
    t0 = time.perf_counter()
    for t in range(steps):
        tok = [d[n][:, t] if d[n] is not None else None for n in NAMES[:8]]
        _, S = orc.decode_step(S, *tok, d["r"])
    return time.perf_counter() - t0


def cpu_baseline():
    sec = oracle_sample(CPU_SAMPLE_T)
    tok = WL["B"] * CPU_SAMPLE_T
    sec_f = oracle_forward_sample(CPU_SAMPLE_T)
    dec_steps = 32
    sec_d = oracle_decode_sample(dec_steps)
    return {"value": round(tok / sec, 2), "unit": "tokens/s", "cores": blas_threads(), "host_cpus": os.cpu_count(),
            "kind": "oracle",
            "sample": f"fp64 numpy oracle fwd+bwd, all {WL['H']} heads, first {CPU_SAMPLE_T} of {WL['T']} tokens "
                      f"({sec:.1f} s)",
            "forward_tokens_s": round(tok / sec_f, 2),
            "decode_tokens_s": round(dec_steps / sec_d, 2),
            "detail": f"forward only on the same sample ({sec_f:.1f} s); decode: one sequence, 24 layers x "
                      f"{DECODE['H']} heads, {dec_steps} tokens ({sec_d:.1f} s)"}


def run_reference(args, rank):
    if rank != 0:
        return
    for _ in range(args.warmup):
        oracle_sample(REF_SAMPLE_T)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_sample(REF_SAMPLE_T)
    sec = time.perf_counter() - t0
    tok = WL["B"] * REF_SAMPLE_T * args.steps
    v = round(tok / sec, 2)
    line = {"metric": METRIC, "value": v, "unit": "tokens/s", "impl": "reference", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * sec / args.steps, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WL["name"], "B": WL["B"], "T": WL["T"], "H": WL["H"], "dk": WL["dk"],
                       "dv": WL["dv"], "chunk": WL["chunk"], "sample_tokens_per_step": REF_SAMPLE_T},
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                             "sample": f"fp64 numpy oracle fwd+bwd, all {WL['H']} heads, {REF_SAMPLE_T} tokens per step"},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="muir", choices=["muir", "reference"])
    ap.add_argument("--skip-extras", action="store_true", help="only the timed step (for profiling)")
    ap.add_argument("--T", type=int, default=None, help="override the sequence length (profiling runs)")
    ap.add_argument("--fwd-only", action="store_true", help="time the forward pass only (profiling runs)")
    ap.add_argument("--gate-only", action="store_true", help="only the gate projection's measurement (profiling runs)")
    ap.add_argument("--decode-only", action="store_true",
                    help="only the decode step at batch 1, 8, 64: W warm-up and K timed launches each, no graph "
                         "(profiling runs)")
    args = ap.parse_args()
    if args.T:
        WL["T"] = args.T
        WL["name"] = f"train_fwdbwd_bf16_B1_T{args.T}_H16_d128_C128"
    args.warmup = max(args.warmup, 3)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if args.impl == "reference":
        run_reference(args, rank)
        return

    import torch
    import torch.distributed as dist
    import gated_delta_rule_muir_b200 as muir

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist_on = world > 1
    if dist_on:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    pk = peaks()
    if args.gate_only:
        if rank == 0:
            print(json.dumps(bench_gate_proj(dev, args.steps, args.warmup, pk)))
        return
    if args.decode_only:
        if rank == 0:
            print(json.dumps(bench_decode(dev, args.steps, args.warmup, pk, graph=False)))
        return
    Step.fwd_only = args.fwd_only
    d = make_workload(dev)
    step = Step(d)
    with ClockSampler(local) as clk:  # started before the warm-up so its start-up stays outside the timing
        for _ in range(args.warmup):
            step()
        n0 = muir.launch_count()
        ms_tot, ms_f, ms_b = time_step_passes(step, args.steps, dist_on)
        ms = ms_tot / args.steps
        launches = (muir.launch_count() - n0)
    tok = WL["B"] * WL["T"]
    value = job_throughput(world, tok, ms)
    line = {"metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": WL["name"], "B": WL["B"], "T": WL["T"], "H": WL["H"], "dk": WL["dk"],
                       "dv": WL["dv"], "chunk": WL["chunk"], "global_batch": world * WL["B"], "seq_len": WL["T"],
                       "parallelism": "replicas" if world > 1 else "single",
                       "l2": "inputs larger than L2 (about 1.3 GB read per step)",
                       "state": "fp32", "tensor_core": "tcgen05 kind::f16, 3-pass bf16 split, fp32 accumulate",
                       "step": "forward only" if Step.fwd_only else
                       "forward (saving its chunk maps) + backward (using them)"},
            "gpu_launches": int(launches), "clocks": clk.summary()}
    # Roofline of the dominant pass against the survey's algorithmic work per head-token
    # (fwd 2,560 B, bwd 5,888 B at bf16, d = 128): both passes are HBM-bound by that model
    # (flops / bytes below the bf16 ridge). Each pass is one C-ABI call of several kernel
    # launches, timed live by the events around it on the launching stream.
    C, dk, dv = WL["chunk"], WL["dk"], WL["dv"]
    ht = WL["B"] * WL["T"] * WL["H"]
    ff, fb, bf, bb = pass_work(C, dk, 2)
    passes = {"muir_chunk_fwd": (ms_f, ff, fb), "muir_chunk_bwd": (ms_b, bf, bb)}
    if Step.fwd_only:
        passes.pop("muir_chunk_bwd")
    pname, (p_ms, p_fl, p_by) = max(passes.items(), key=lambda kv: kv[1][0])
    t_p = p_ms * 1e-3
    ach = ht * p_by / t_p / 1e9
    roof = {"bound": "hbm", "achieved": round(ach, 1), "peak": pk["hbm"], "unit": "GB/s",
            "frac": round(ach / pk["hbm"], 4), "traffic": None, "kernel": pname,
            "ms_per_launch": round(p_ms, 4), "algorithmic_bytes_per_head_token": p_by,
            "head_tokens_per_launch": ht, "frac_tc_peak": round(ht * p_fl / t_p / 1e12 / pk["bf16_sus"], 4),
            "peak_source": pk["src"]}
    line["roofline"] = roof
    line["passes_ms"] = {k: round(v[0], 4) for k, v in passes.items()}
    # per-kernel device times (library events on the launch stream), same workload
    with muir.KernelTimer() as kt:
        for _ in range(args.steps):
            step()
    kern = {k: {"launches": c, "ms_per_step": round(t / args.steps, 4)} for k, (c, t) in kt.result.items()}
    line["kernels"] = kern
    # the slowest single kernel, with its modelled algorithmic flops (vs the tensor peak) and its
    # interface bytes (the intermediates it exchanges with the other kernels, vs HBM)
    model = kernel_model(C, dk, dv, 2)
    units = WL["B"] * WL["H"] * (WL["T"] // C)
    name, (cnt, tot) = max(kt.result.items(), key=lambda kv: kv[1][1])
    base = name.split(":")[-1]
    if base in model:
        fl, by = model[base]
        t_k = tot / cnt * 1e-3
        lps = cnt / args.steps
        line["slowest_kernel"] = {
            "kernel": name, "ms_per_launch": round(tot / cnt, 4),
            "algorithmic_TFLOP_s": round(fl * units / lps / t_k / 1e12, 2),
            "frac_tc_peak": round(fl * units / lps / t_k / 1e12 / pk["bf16_sus"], 4),
            "interface_GB_s": round(by * units / lps / t_k / 1e9, 1),
            "frac_hbm_interface": round(by * units / lps / t_k / 1e9 / pk["hbm"], 4)}
    line["flop_split"] = flop_split(C, dk, dv)
    sfl, sby = algorithmic_step()
    t_step = ms * 1e-3
    line["step_roofline"] = {"algorithmic_TFLOP_s": round(sfl / t_step / 1e12, 2),
                             "frac_tc_peak": round(sfl / t_step / 1e12 / pk["bf16_sus"], 4),
                             "algorithmic_GB_s": round(sby / t_step / 1e9, 1),
                             "frac_hbm_peak": round(sby / t_step / 1e9 / pk["hbm"], 4),
                             "roofline_ms": round(1e3 * max(sfl / (pk["bf16_sus"] * 1e12), sby / (pk["hbm"] * 1e9)), 3)}
    if not args.skip_extras and rank == 0:
        line["forward"] = bench_forwards(dev, args.steps, args.warmup, pk)
        line["decode"] = bench_decode(dev, args.steps, args.warmup, pk)
        line["gate_proj"] = bench_gate_proj(dev, args.steps, args.warmup, pk)
        line["e2e"] = e2e_pass(d, max(2, min(args.steps, 5)), 1)
        if world == 1:
            line["cpu_baseline"] = cpu_baseline()
    if dist_on:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
