"""ctypes view of include/fused_norm.h and libfused_norm.so.

Argument marshalling only: every step of the operation runs in the library's CUDA
kernels. Loading fails loudly when the library has not been built; there is no
other implementation to fall back to.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfused_norm.so")

FN_OK = 0
FN_ERR_INVALID_ARG = 1
FN_ERR_UNSUPPORTED = 2
FN_ERR_MISALIGNED = 3
FN_ERR_CUDA = 4
STATUS_NAMES = {0: "FN_OK", 1: "FN_ERR_INVALID_ARG", 2: "FN_ERR_UNSUPPORTED",
                3: "FN_ERR_MISALIGNED", 4: "FN_ERR_CUDA"}

# Every function include/fused_norm.h declares.
EXPORTED = ("fused_norm_create", "fused_norm_validate", "fused_norm_launch", "fused_norm_destroy",
            "fused_norm_get_config", "fused_norm_plan", "fused_norm_status_string",
            "fused_norm_last_cuda_error", "fused_norm_version")


class fn_config(ctypes.Structure):
    _fields_ = [("D", ctypes.c_int), ("is_rms", ctypes.c_int), ("has_gate", ctypes.c_int),
                ("has_weight", ctypes.c_int), ("has_bias", ctypes.c_int),
                ("norm_only", ctypes.c_int), ("affine_fp32", ctypes.c_int),
                ("eps", ctypes.c_double)]


class fn_operand(ctypes.Structure):
    _fields_ = [("ptr", ctypes.c_void_p), ("stride_b", ctypes.c_int64),
                ("stride_f", ctypes.c_int64), ("stride_l", ctypes.c_int64)]


class fn_args(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int64), ("L", ctypes.c_int64), ("tokens_per_frame", ctypes.c_int64),
                ("x", fn_operand), ("residual", fn_operand), ("gate", fn_operand),
                ("scale", fn_operand), ("shift", fn_operand),
                ("weight", ctypes.c_void_p), ("bias", ctypes.c_void_p),
                ("y", ctypes.c_void_p), ("y_stride_b", ctypes.c_int64), ("y_stride_l", ctypes.c_int64),
                ("r", ctypes.c_void_p), ("r_stride_b", ctypes.c_int64), ("r_stride_l", ctypes.c_int64)]


class FusedNormError(RuntimeError):
    def __init__(self, status: int, what: str, detail: str = ""):
        self.status = status
        msg = f"{what}: {STATUS_NAMES.get(status, status)} ({detail})" if detail else \
            f"{what}: {STATUS_NAMES.get(status, status)}"
        super().__init__(msg)


_lib = None


def load() -> ctypes.CDLL:
    """The loaded library; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m rmsnorm_row_b200.build` "
            "(there is no fallback implementation)")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.POINTER
    lib.fused_norm_create.argtypes = [P(ctypes.c_void_p), P(fn_config)]
    lib.fused_norm_validate.argtypes = [ctypes.c_void_p, P(fn_args)]
    lib.fused_norm_launch.argtypes = [ctypes.c_void_p, P(fn_args), ctypes.c_void_p]
    lib.fused_norm_destroy.argtypes = [ctypes.c_void_p]
    lib.fused_norm_get_config.argtypes = [ctypes.c_void_p, P(fn_config)]
    lib.fused_norm_plan.argtypes = [ctypes.c_void_p, P(fn_args), P(ctypes.c_int64),
                                    P(ctypes.c_int), P(ctypes.c_size_t)]
    lib.fused_norm_status_string.argtypes = [ctypes.c_int]
    lib.fused_norm_status_string.restype = ctypes.c_char_p
    lib.fused_norm_last_cuda_error.argtypes = []
    lib.fused_norm_version.argtypes = []
    for name in ("fused_norm_create", "fused_norm_validate", "fused_norm_launch",
                 "fused_norm_destroy", "fused_norm_get_config", "fused_norm_plan",
                 "fused_norm_last_cuda_error", "fused_norm_version"):
        getattr(lib, name).restype = ctypes.c_int
    _lib = lib
    return lib


# ---------------------------------------------------------------------------
# The C entry points under their own names (status codes returned as ints).
# ---------------------------------------------------------------------------

def fused_norm_create(cfg: fn_config):
    """Returns (status, handle); handle is None unless status == FN_OK."""
    h = ctypes.c_void_p()
    st = load().fused_norm_create(ctypes.byref(h), ctypes.byref(cfg))
    return st, (h.value if st == FN_OK else None)


def fused_norm_validate(h, args: fn_args) -> int:
    return load().fused_norm_validate(h, ctypes.byref(args))


def fused_norm_launch(h, args: fn_args, stream: int) -> int:
    return load().fused_norm_launch(h, ctypes.byref(args), ctypes.c_void_p(stream))


def fused_norm_destroy(h) -> int:
    return load().fused_norm_destroy(h)


def fused_norm_get_config(h):
    cfg = fn_config()
    st = load().fused_norm_get_config(h, ctypes.byref(cfg))
    return st, cfg


def fused_norm_plan(h, args: fn_args):
    """Returns (status, grid, block, smem_bytes)."""
    g, b, s = ctypes.c_int64(), ctypes.c_int(), ctypes.c_size_t()
    st = load().fused_norm_plan(h, ctypes.byref(args), ctypes.byref(g), ctypes.byref(b),
                                ctypes.byref(s))
    return st, g.value, b.value, s.value


def fused_norm_status_string(status: int) -> str:
    return load().fused_norm_status_string(status).decode()


def fused_norm_last_cuda_error() -> int:
    return load().fused_norm_last_cuda_error()


def fused_norm_version() -> int:
    return load().fused_norm_version()
