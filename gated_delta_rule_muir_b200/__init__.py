"""Muir gated delta-rule operator on NVIDIA B200: Python binding of libmuir.so.

Each function only checks tensor shapes/dtypes, allocates outputs and workspace
with torch (device memory plumbing), and calls the C ABI (include/muir.h) on the
current CUDA stream. All arithmetic runs in the library's CUDA kernels; there is
no CPU or PyTorch fallback.
"""
from __future__ import annotations

import ctypes as C

import torch

from . import _native as N

__all__ = ["chunk_fwd", "chunk_bwd", "decode_step", "state_init", "device_status", "chunk_fwd_workspace_bytes",
           "chunk_bwd_workspace_bytes", "MuirError", "KernelTimer", "launch_count", "gate_proj", "GATE_RANKS"]

MuirError = N.MuirError


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return C.c_void_p(s.cuda_stream)


def _dtype_code(dt):
    if dt == torch.float32:
        return N.MUIR_F32
    if dt == torch.bfloat16:
        return N.MUIR_BF16
    raise TypeError(f"unsupported dtype {dt}")


def _need(t, name, shape, dtype=None):
    if t.shape != torch.Size(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name}: must be a contiguous CUDA tensor")


def _chunk_args(q, k, v, e, w, g, z, log_alpha, r, chunk, S0, flags=0):
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    for n, t, d in (("q", q, dk), ("k", k, dk), ("e", e, dk), ("v", v, dv), ("w", w, dv)):
        _need(t, n, (B, T, H, d), dt)
    if g is not None:  # g = None: static-only readout (g = 1)
        _need(g, "g", (B, T, H, dk), dt)
    if z is not None:
        _need(z, "z", (B, T, H, dv), dt)
    _need(log_alpha, "log_alpha", (B, T, H, dk), torch.float32)
    _need(r, "r", (H, dk), torch.float32)
    if S0 is not None:
        _need(S0, "S0", (B, H, dk, dv), torch.float32)
    a = N.ChunkArgs(B=B, T=T, H=H, dk=dk, dv=dv, chunk=chunk, dtype=_dtype_code(dt), flags=flags,
                    q=_ptr(q), k=_ptr(k), v=_ptr(v), e=_ptr(e), w=_ptr(w), g=_ptr(g), z=_ptr(z),
                    log_alpha=_ptr(log_alpha), r=_ptr(r), S0=_ptr(S0))
    return a, (B, T, H, dk, dv, dt)


def chunk_fwd_workspace_bytes(q, k, v, e, w, g, z, log_alpha, r, chunk, S0=None, save_for_bwd=False) -> int:
    a, _ = _chunk_args(q, k, v, e, w, g, z, log_alpha, r, chunk, S0, N.MUIR_SAVE_FOR_BWD if save_for_bwd else 0)
    return int(N.load().muir_chunk_fwd_workspace(C.byref(a)))


def chunk_bwd_workspace_bytes(q, k, v, e, w, g, z, log_alpha, r, chunk, S0=None) -> int:
    a, _ = _chunk_args(q, k, v, e, w, g, z, log_alpha, r, chunk, S0)
    return int(N.load().muir_chunk_bwd_workspace(C.byref(a)))


def _workspace(nbytes, device, ws):
    if ws is not None:
        if ws.numel() * ws.element_size() < nbytes:
            raise ValueError("workspace too small")
        return ws
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def chunk_fwd(q, k, v, e, w, g, z, log_alpha, r, *, chunk=128, S0=None, want_state=True, y=None, S_T=None,
              workspace=None, save_for_bwd=False, stream=None):
    """Chunkwise forward pass. Inputs [B,T,H,d] (fp32 or bf16; log_alpha fp32), r [H,dk] fp32.
    Returns (y [B,T,H,dv], S_T [B,H,dk,dv] fp32 or None). With save_for_bwd=True the
    workspace (pass one, of chunk_bwd_workspace_bytes) keeps what chunk_bwd(use_saved=True)
    needs."""
    lib = N.load()
    flags = N.MUIR_SAVE_FOR_BWD if save_for_bwd else 0
    a, (B, T, H, dk, dv, dt) = _chunk_args(q, k, v, e, w, g, z, log_alpha, r, chunk, S0, flags)
    if y is None:
        y = torch.empty(B, T, H, dv, dtype=dt, device=q.device)
    if want_state and S_T is None:
        S_T = torch.empty(B, H, dk, dv, dtype=torch.float32, device=q.device)
    nbytes = int(lib.muir_chunk_fwd_workspace(C.byref(a)))
    if save_for_bwd and workspace is None:
        raise ValueError("save_for_bwd needs a workspace to keep (chunk_bwd_workspace_bytes)")
    ws = _workspace(nbytes, q.device, workspace)
    N.check(lib.muir_chunk_fwd(C.byref(a), _ptr(y), _ptr(S_T if want_state else None), _ptr(ws), nbytes,
                               _stream(stream)), "muir_chunk_fwd")
    return y, (S_T if want_state else None)


def chunk_bwd(q, k, v, e, w, g, z, log_alpha, r, dy, *, chunk=128, S0=None, dS_T=None, want_dS0=True,
              want_dr=False, workspace=None, outputs=None, use_saved=False, stream=None):
    """Backward pass of chunk_fwd. Returns a dict of gradients (dq, dk, dv, de, dw, dg, dz, dlog_alpha,
    dS0, dr), each shaped like its input. `outputs` (a dict from an earlier call) is reused if given.
    use_saved=True: `workspace` is the one a chunk_fwd(save_for_bwd=True) of the same inputs filled."""
    lib = N.load()
    if use_saved and workspace is None:
        raise ValueError("use_saved needs the workspace of chunk_fwd(save_for_bwd=True)")
    flags = N.MUIR_USE_SAVED if use_saved else 0
    a, (B, T, H, dk, dv, dt) = _chunk_args(q, k, v, e, w, g, z, log_alpha, r, chunk, S0, flags)
    _need(dy, "dy", (B, T, H, dv), dt)
    if dS_T is not None:
        _need(dS_T, "dS_T", (B, H, dk, dv), torch.float32)
    dev = q.device
    if outputs is not None:
        out = outputs
        gr = N.ChunkGrads(dy=_ptr(dy), dS_T=_ptr(dS_T), dq=_ptr(out["dq"]), dk=_ptr(out["dk"]), dv=_ptr(out["dv"]),
                          de=_ptr(out["de"]), dw=_ptr(out["dw"]), dg=_ptr(out["dg"]), dz=_ptr(out["dz"]),
                          dlog_alpha=_ptr(out["dlog_alpha"]), dS0=_ptr(out["dS0"]), dr=_ptr(out["dr"]))
        nbytes = int(lib.muir_chunk_bwd_workspace(C.byref(a)))
        ws = _workspace(nbytes, dev, workspace)
        N.check(lib.muir_chunk_bwd(C.byref(a), C.byref(gr), _ptr(ws), nbytes, _stream(stream)), "muir_chunk_bwd")
        return out
    out = {n: torch.empty(B, T, H, dk, dtype=dt, device=dev) for n in ("dq", "dk", "de", "dg")}
    if g is None:
        out["dg"] = None
    out.update({n: torch.empty(B, T, H, dv, dtype=dt, device=dev) for n in ("dv", "dw")})
    out["dz"] = torch.empty(B, T, H, dv, dtype=dt, device=dev) if z is not None else None
    out["dlog_alpha"] = torch.empty(B, T, H, dk, dtype=torch.float32, device=dev)
    out["dS0"] = torch.empty(B, H, dk, dv, dtype=torch.float32, device=dev) if want_dS0 else None
    out["dr"] = torch.empty(H, dk, dtype=torch.float32, device=dev) if want_dr else None
    gr = N.ChunkGrads(dy=_ptr(dy), dS_T=_ptr(dS_T), dq=_ptr(out["dq"]), dk=_ptr(out["dk"]), dv=_ptr(out["dv"]),
                      de=_ptr(out["de"]), dw=_ptr(out["dw"]), dg=_ptr(out["dg"]), dz=_ptr(out["dz"]),
                      dlog_alpha=_ptr(out["dlog_alpha"]), dS0=_ptr(out["dS0"]), dr=_ptr(out["dr"]))
    nbytes = int(lib.muir_chunk_bwd_workspace(C.byref(a)))
    ws = _workspace(nbytes, dev, workspace)
    N.check(lib.muir_chunk_bwd(C.byref(a), C.byref(gr), _ptr(ws), nbytes, _stream(stream)), "muir_chunk_bwd")
    return out


def decode_step(S, q, k, v, e, w, g, z, log_alpha, r, *, y=None, stream=None):
    """One recurrent token for n rows: S [n,H,dk,dv] fp32 updated in place; inputs [n,H,d];
    r [H,dk] (shared) or [n,H,dk] (per row). Returns y [n,H,dv]."""
    lib = N.load()
    n, H, dk, dv = S.shape
    dt = q.dtype
    _need(S, "S", (n, H, dk, dv), torch.float32)
    for nm, t, d in (("q", q, dk), ("k", k, dk), ("e", e, dk), ("v", v, dv), ("w", w, dv)):
        _need(t, nm, (n, H, d), dt)
    if g is not None:
        _need(g, "g", (n, H, dk), dt)
    if z is not None:
        _need(z, "z", (n, H, dv), dt)
    _need(log_alpha, "log_alpha", (n, H, dk), torch.float32)
    if r.dim() == 2:
        _need(r, "r", (H, dk), torch.float32)
        rs = 0
    else:
        _need(r, "r", (n, H, dk), torch.float32)
        rs = H * dk
    if y is None:
        y = torch.empty(n, H, dv, dtype=dt, device=S.device)
    a = N.DecodeArgs(n_seq=n, H=H, dk=dk, dv=dv, dtype=_dtype_code(dt), S=_ptr(S), q=_ptr(q), k=_ptr(k),
                     v=_ptr(v), e=_ptr(e), w=_ptr(w), g=_ptr(g), z=_ptr(z), log_alpha=_ptr(log_alpha), r=_ptr(r),
                     r_seq_stride=rs, y=_ptr(y))
    N.check(lib.muir_decode_step(C.byref(a), _stream(stream)), "muir_decode_step")
    return y


def state_init(S, S_src=None, *, stream=None):
    """S := S_src (or zeros), S [n,H,dk,dv] fp32."""
    lib = N.load()
    n, H, dk, dv = S.shape
    _need(S, "S", (n, H, dk, dv), torch.float32)
    if S_src is not None:
        _need(S_src, "S_src", (n, H, dk, dv), torch.float32)
    N.check(lib.muir_state_init(_ptr(S), _ptr(S_src), n, H, dk, dv, _stream(stream)), "muir_state_init")
    return S


def chunk_segment_map(q, k, v, e, w, g, z, log_alpha, r, *, chunk=128, workspace=None, stream=None):
    """The segment's chunkwise forward as an affine map of its start state,
    S_end = Phi S0 + Psi: returns (Phi [B,H,dk,dk], Psi [B,H,dk,dv]) fp32."""
    lib = N.load()
    a, (B, T, H, dk, dv, dt) = _chunk_args(q, k, v, e, w, g, z, log_alpha, r, chunk, None)
    Phi = torch.empty(B, H, dk, dk, dtype=torch.float32, device=q.device)
    Psi = torch.empty(B, H, dk, dv, dtype=torch.float32, device=q.device)
    nbytes = int(lib.muir_chunk_segment_map_workspace(C.byref(a)))
    ws = _workspace(nbytes, q.device, workspace)
    N.check(lib.muir_chunk_segment_map(C.byref(a), _ptr(Phi), _ptr(Psi), _ptr(ws), nbytes, _stream(stream)),
            "muir_chunk_segment_map")
    return Phi, Psi


def apply_map(Phi, Psi, S_in=None, *, S_out=None, stream=None):
    """S_out = Phi S_in + Psi for [n,H] maps (S_in None: S_out = Psi), fp32."""
    lib = N.load()
    n, H, dk, _ = Phi.shape
    dv = Psi.shape[-1]
    _need(Phi, "Phi", (n, H, dk, dk), torch.float32)
    _need(Psi, "Psi", (n, H, dk, dv), torch.float32)
    if S_in is not None:
        _need(S_in, "S_in", (n, H, dk, dv), torch.float32)
    if S_out is None:
        S_out = torch.empty_like(Psi)
    N.check(lib.muir_apply_map(_ptr(Phi), _ptr(Psi), _ptr(S_in), _ptr(S_out), n, H, dk, dv, _stream(stream)),
            "muir_apply_map")
    return S_out


def row_scale(S, *, exponent=0.5, eps=1e-12, r=None, stream=None):
    """Static matched-filter row scale from measured row energies of states
    S [n,H,dk,dv] fp32: r[h,i] = (mean_{n,j} S[n,h,i,j]^2 + eps)^(-exponent), [H,dk]."""
    lib = N.load()
    n, H, dk, dv = S.shape
    _need(S, "S", (n, H, dk, dv), torch.float32)
    if r is None:
        r = torch.empty(H, dk, dtype=torch.float32, device=S.device)
    _need(r, "r", (H, dk), torch.float32)
    N.check(lib.muir_row_scale(_ptr(S), n, H, dk, dv, float(exponent), float(eps), _ptr(r), _stream(stream)),
            "muir_row_scale")
    return r


GATE_RANKS = (64, 64, 128, 128, 128)  # decay, erase, output, write, read (total rank 512)


def gate_proj(x, w_down, u_decay, u_erase, u_out, u_write, u_read, *, out=None, stream=None):
    """Fused low-rank gate projection (muir_gate_proj): x [N, D] and weights of x's
    dtype (w_down [D, 512], u_decay / u_erase [64, Ok], u_out / u_write [128, Ov],
    u_read [128, Ok]) -> dict of log_alpha [N, Ok] fp32 and e, z, w, g in x's dtype
    (e, g [N, Ok]; z, w [N, Ov]). `out` may hold preallocated outputs."""
    lib = N.load()
    n, D = x.shape
    Ok, Ov = u_decay.shape[1], u_out.shape[1]
    dt = x.dtype
    _need(x, "x", (n, D), dt)
    _need(w_down, "w_down", (D, 512), dt)
    for name, t, shape in (("u_decay", u_decay, (64, Ok)), ("u_erase", u_erase, (64, Ok)),
                           ("u_out", u_out, (128, Ov)), ("u_write", u_write, (128, Ov)),
                           ("u_read", u_read, (128, Ok))):
        _need(t, name, shape, dt)
    out = dict(out or {})
    shapes = {"log_alpha": ((n, Ok), torch.float32), "e": ((n, Ok), dt), "z": ((n, Ov), dt),
              "w": ((n, Ov), dt), "g": ((n, Ok), dt)}
    for name, (shape, odt) in shapes.items():
        if name not in out:
            out[name] = torch.empty(shape, dtype=odt, device=x.device)
        _need(out[name], name, shape, odt)
    N.check(lib.muir_gate_proj(_ptr(x), _ptr(w_down), _ptr(u_decay), _ptr(u_erase), _ptr(u_out), _ptr(u_write),
                               _ptr(u_read), _ptr(out["log_alpha"]), _ptr(out["e"]), _ptr(out["z"]), _ptr(out["w"]),
                               _ptr(out["g"]), n, D, Ok, Ov, _dtype_code(dt), _stream(stream)), "muir_gate_proj")
    return out


def launch_count() -> int:
    """Number of kernels libmuir has launched in this process."""
    return int(N.load().muir_launch_count())


class KernelTimer:
    """Per-kernel device time from CUDA events the library records around each of
    its launches (on the launch stream). Use as a context manager; .result maps
    'phase:kernel' -> (launches, total_ms)."""

    def __enter__(self):
        N.load().muir_profile_begin()
        return self

    def __exit__(self, *exc):
        lib = N.load()
        cap, maxn = 1 << 14, 64
        buf = C.create_string_buffer(cap)
        ms = (C.c_float * maxn)()
        cnt = (C.c_int64 * maxn)()
        n = lib.muir_profile_end(buf, cap, ms, cnt, maxn)
        if n < 0:
            raise MuirError(N.MUIR_ERR_CUDA, "muir_profile_end", "event timing failed")
        names = buf.value.decode().split("\n")[:n]
        self.result = {nm: (int(cnt[i]), float(ms[i])) for i, nm in enumerate(names)}
        return False


def device_status(stream=None) -> int:
    """Synchronise and return the library's device status code (0 = OK)."""
    return int(N.load().muir_device_status(_stream(stream)))
