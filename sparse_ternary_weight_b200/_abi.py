"""ctypes declarations of the C ABI in include/sherry.h (argument marshalling only)."""
from __future__ import annotations

import ctypes
import os
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
SO_PATH = os.path.join(HERE, "libsherry.so")

OK = 0
ERR_NULL, ERR_SHAPE, ERR_GRANULARITY, ERR_GROUP, ERR_DTYPE = 1, 2, 3, 4, 5
ERR_ALIGN, ERR_WORKSPACE, ERR_CUDA, ERR_TIMEOUT, ERR_UNSUPPORTED = 6, 7, 8, 9, 10
PER_TENSOR, PER_CHANNEL, PER_GROUP = 0, 1, 2
F32, BF16 = 0, 1
OP_QUANTIZE_PACK, OP_LINEAR, OP_UNPACK = 0, 1, 2
MAX_K = 262144
MAX_BATCH = 256
NOALLOC_SCRATCH_BYTES = 16 << 20
TEQUILA_ONES, TEQUILA_SIGN = 0, 1

vp, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t


class LinearDesc(ctypes.Structure):
    """Mirror of ``sherry_linear_desc``."""
    _fields_ = [("X", vp), ("idx", vp), ("sgn", vp), ("scales", vp), ("Y", vp),
                ("N", i64), ("K", i64), ("granularity", ctypes.c_int32), ("group", ctypes.c_int32)]


class QuantizeDesc(ctypes.Structure):
    """Mirror of ``sherry_quantize_desc``."""
    _fields_ = [("W", vp), ("idx", vp), ("sgn", vp), ("scales", vp), ("Wq", vp), ("N", i64), ("K", i64),
                ("w_dtype", ctypes.c_int32), ("granularity", ctypes.c_int32), ("group", ctypes.c_int32),
                ("wq_dtype", ctypes.c_int32)]


class UnpackDesc(ctypes.Structure):
    """Mirror of ``sherry_unpack_desc``."""
    _fields_ = [("idx", vp), ("sgn", vp), ("scales", vp), ("N", i64), ("K", i64),
                ("granularity", ctypes.c_int32), ("group", ctypes.c_int32), ("W_out", vp)]


SIGNATURES = {
    "sherry_idx_bytes": (sz, [i64, i64]),
    "sherry_sgn_bytes": (sz, [i64, i64]),
    "sherry_num_scales": (i64, [i64, i64, i32, i32]),
    "sherry_workspace_bytes": (sz, [i32, i64, i64, i64, i32, i32]),
    "sherry_quantize_pack": (i32, [vp, i32, i64, i64, i32, i32, vp, vp, vp, vp, sz, vp]),
    "sherry_fake_quant": (i32, [vp, i32, i64, i64, i32, i32, vp, i32, vp, vp, vp, vp, sz, vp]),
    "sherry_quantize_pack_batched": (i32, [ctypes.POINTER(QuantizeDesc), i32, vp, sz, vp]),
    "sherry_quantize_pack_batched_workspace_bytes": (sz, [ctypes.POINTER(QuantizeDesc), i32]),
    "sherry_quantize_pack_tequila": (i32, [vp, i32, i64, i64, i32, i32, ctypes.c_float, vp, vp, vp, vp, vp, vp, sz,
                                           vp]),
    "sherry_linear_tequila": (i32, [vp, i64, i64, i64, vp, vp, vp, i32, i32, vp, vp, i32, vp, i32, vp, sz, vp]),
    "sherry_linear_tequila_workspace_bytes": (sz, [i64, i64, i64, i32, i32, i32]),
    "sherry_arenas_linear": (i32, [vp, i64, i64, i64, vp, vp, vp, i32, i32, vp, ctypes.c_float, vp, i32, vp]),
    "sherry_arenas_lambda": (ctypes.c_float, [i64, i64, ctypes.c_float]),
    "sherry_linear": (i32, [vp, i64, i64, i64, vp, vp, vp, i32, i32, vp, i32, vp, sz, vp]),
    "sherry_linear_batched": (i32, [ctypes.POINTER(LinearDesc), i32, i64, i32, vp, sz, vp]),
    "sherry_linear_batched_workspace_bytes": (sz, [ctypes.POINTER(LinearDesc), i32, i64]),
    "sherry_linear_chain": (i32, [ctypes.POINTER(LinearDesc), i32, ctypes.POINTER(ctypes.c_int), i32, i64, i32, vp,
                                  sz, vp]),
    "sherry_linear_chain_workspace_bytes": (sz, [ctypes.POINTER(LinearDesc), i32, ctypes.POINTER(ctypes.c_int), i32,
                                                 i64]),
    "sherry_unpack": (i32, [vp, vp, vp, i64, i64, i32, i32, vp, vp]),
    "sherry_unpack_batched": (i32, [ctypes.POINTER(UnpackDesc), i32, vp]),
    "sherry_linear_noalloc": (i32, [vp, i64, i64, i64, vp, vp, vp, i32, i32, vp, i32, vp]),
    "sherry_status_string": (ctypes.c_char_p, [i32]),
    "sherry_last_cuda_error": (i32, []),
    "sherry_device_status": (i32, [vp]),
    "sherry_timeout_count": (i64, []),
    "sherry_set_wait_budget": (i64, [i64]),
    "sherry_version": (i32, []),
}

_lock = threading.Lock()
_lib = None


class SherryError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        msg = lib().sherry_status_string(status).decode()
        if status == ERR_CUDA:
            msg += f" (cudaError {lib().sherry_last_cuda_error()})"
        super().__init__(f"{what}: status {status}: {msg}" if what else f"status {status}: {msg}")


def lib() -> ctypes.CDLL:
    """The in-tree CUDA library.  Raises if it has not been built: there is no
    fallback implementation."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(SO_PATH):
                raise RuntimeError(f"{SO_PATH} is missing; build it with "
                                   "`python -m sparse_ternary_weight_b200.build`")
            L = ctypes.CDLL(SO_PATH)
            for name, (res, args) in SIGNATURES.items():
                f = getattr(L, name)
                f.restype = res
                f.argtypes = args
            _lib = L
        return _lib


def check(status: int, what: str = "") -> None:
    if status != OK:
        raise SherryError(status, what)
