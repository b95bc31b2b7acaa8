"""ctypes view of libmuir.so (the C ABI in include/muir.h). Marshalling only."""
from __future__ import annotations

import ctypes as C
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
# MUIR_LIBRARY selects another in-tree build of the same library (the checking
# build, libmuir_check.so, in its test); there is still no fallback.
LIB_PATH = os.environ.get("MUIR_LIBRARY") or os.path.join(_PKG, "libmuir.so")
CHECK_LIB_PATH = os.path.join(_PKG, "libmuir_check.so")

(MUIR_OK, MUIR_ERR_INVALID_ARG, MUIR_ERR_UNSUPPORTED, MUIR_ERR_WORKSPACE, MUIR_ERR_CUDA, MUIR_ERR_TIMEOUT,
 MUIR_ERR_BOUNDS) = range(7)
MUIR_F32, MUIR_BF16 = 0, 1
MUIR_SAVE_FOR_BWD, MUIR_USE_SAVED = 1, 2

ERROR_NAMES = {MUIR_ERR_INVALID_ARG: "invalid argument", MUIR_ERR_UNSUPPORTED: "unsupported",
               MUIR_ERR_WORKSPACE: "workspace", MUIR_ERR_CUDA: "CUDA error", MUIR_ERR_TIMEOUT: "device timeout",
               MUIR_ERR_BOUNDS: "bounds check"}

vp = C.c_void_p


class ChunkArgs(C.Structure):
    _fields_ = [("B", C.c_int64), ("T", C.c_int64), ("H", C.c_int32), ("dk", C.c_int32), ("dv", C.c_int32),
                ("chunk", C.c_int32), ("dtype", C.c_int32), ("flags", C.c_int32),
                ("q", vp), ("k", vp), ("v", vp), ("e", vp), ("w", vp), ("g", vp), ("z", vp),
                ("log_alpha", vp), ("r", vp), ("S0", vp)]


class ChunkGrads(C.Structure):
    _fields_ = [("dy", vp), ("dS_T", vp), ("dq", vp), ("dk", vp), ("dv", vp), ("de", vp), ("dw", vp),
                ("dg", vp), ("dz", vp), ("dlog_alpha", vp), ("dS0", vp), ("dr", vp)]


class DecodeArgs(C.Structure):
    _fields_ = [("n_seq", C.c_int64), ("H", C.c_int32), ("dk", C.c_int32), ("dv", C.c_int32), ("dtype", C.c_int32),
                ("S", vp), ("q", vp), ("k", vp), ("v", vp), ("e", vp), ("w", vp), ("g", vp), ("z", vp),
                ("log_alpha", vp), ("r", vp), ("r_seq_stride", C.c_int64), ("y", vp)]


# Every symbol include/muir.h declares, with its ctypes signature.
SIGNATURES = {
    "muir_chunk_fwd_workspace": (C.c_size_t, [C.POINTER(ChunkArgs)]),
    "muir_chunk_fwd": (C.c_int, [C.POINTER(ChunkArgs), vp, vp, vp, C.c_size_t, vp]),
    "muir_chunk_fwd_noalloc": (C.c_int, [C.POINTER(ChunkArgs), vp, vp, vp]),
    "muir_chunk_bwd_workspace": (C.c_size_t, [C.POINTER(ChunkArgs)]),
    "muir_chunk_bwd": (C.c_int, [C.POINTER(ChunkArgs), C.POINTER(ChunkGrads), vp, C.c_size_t, vp]),
    "muir_decode_step": (C.c_int, [C.POINTER(DecodeArgs), vp]),
    "muir_state_init": (C.c_int, [vp, vp, C.c_int64, C.c_int32, C.c_int32, C.c_int32, vp]),
    "muir_row_scale": (C.c_int, [vp, C.c_int64, C.c_int32, C.c_int32, C.c_int32, C.c_float, C.c_float, vp, vp]),
    "muir_chunk_segment_map_workspace": (C.c_size_t, [C.POINTER(ChunkArgs)]),
    "muir_chunk_segment_map": (C.c_int, [C.POINTER(ChunkArgs), vp, vp, vp, C.c_size_t, vp]),
    "muir_apply_map": (C.c_int, [vp, vp, vp, vp, C.c_int64, C.c_int32, C.c_int32, C.c_int32, vp]),
    "muir_gate_proj": (C.c_int, [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, C.c_int64, C.c_int32, C.c_int32,
                                 C.c_int32, C.c_int32, vp]),
    "muir_device_status": (C.c_int, [vp]),
    "muir_last_error": (C.c_char_p, []),
    "muir_version": (C.c_int, []),
}

# Diagnostic exports declared in include/muir_profile.h.
EXTRA_SIGNATURES = {
    "muir_selftest_gemm": (C.c_int, [vp, vp, vp, C.c_int32, C.c_int32, C.c_int32, C.c_int32, C.c_int32, vp]),
    "muir_selftest_wait": (C.c_int, [C.c_uint64, C.c_int32, vp, vp]),
    "muir_selftest_sw128": (C.c_int, [vp, vp, vp, C.c_int32, C.c_int32, C.c_int32, vp]),
    "muir_profile_begin": (None, []),
    "muir_profile_end": (C.c_int, [C.c_char_p, C.c_size_t, C.POINTER(C.c_float), C.POINTER(C.c_int64), C.c_int]),
    "muir_launch_count": (C.c_int64, []),
}

_lib = None


def load(path: str = LIB_PATH) -> C.CDLL:
    """Load libmuir.so (built in-tree by build.py). Raises if it is missing: there is
    no fallback implementation."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"libmuir.so not found at {path}; build it with "
                           f"`python -m gated_delta_rule_muir_b200.build`")
    lib = C.CDLL(path)
    for name, (res, args) in {**SIGNATURES, **EXTRA_SIGNATURES}.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


class MuirError(RuntimeError):
    def __init__(self, code: int, where: str, msg: str):
        super().__init__(f"{where}: {ERROR_NAMES.get(code, code)}: {msg}")
        self.code = code


def check(code: int, where: str) -> None:
    if code != MUIR_OK:
        raise MuirError(code, where, load().muir_last_error().decode())
