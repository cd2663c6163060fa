"""CPU oracle for Sherry 3:4-sparse ternary quantise+pack, unpack and linear.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The product library
(``sparse_ternary_weight_b200``) never imports it and shares no code with it.

Two independent statements of the same definitions live here:

* ``sherry_ref.c`` -- plain C99, loaded through ctypes (:func:`lib`).  Built
  single-threaded, and with OpenMP over independent rows for the all-cores
  timing; both builds give identical results.
* ``sherry_np.py`` -- a NumPy restatement that follows the pages' tensor code
  path (block reshape, mask of the kept top-3 magnitudes, sign, sum of |kept|
  over the granularity's domain, divide by the kept count).  Used on small
  inputs to cross-check the C file bit for bit.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sherry_ref.c")
_HDR = os.path.join(_HERE, "sherry_ref.h")
_CFLAGS = ["-std=c99", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fPIC", "-shared"]

OK, ERR_NULL, ERR_SHAPE, ERR_GRANULARITY, ERR_GROUP, ERR_DTYPE = 0, 1, 2, 3, 4, 5
PER_TENSOR, PER_CHANNEL, PER_GROUP = 0, 1, 2
F32, BF16 = 0, 1

_lock = threading.Lock()
_libs: dict = {}


def so_path(omp: bool = False) -> str:
    return os.path.join(_HERE, "libsherry_ref_omp.so" if omp else "libsherry_ref.so")


def build(omp: bool = False, src: str = _SRC, out: str | None = None, force: bool = False) -> str:
    """Compile the C oracle with gcc (no fast-math, no FP contraction)."""
    out = out or so_path(omp)
    if not force and os.path.exists(out):
        newest = max(os.path.getmtime(src), os.path.getmtime(_HDR))
        if os.path.getmtime(out) >= newest:
            return out
    cmd = ["gcc", *_CFLAGS, "-I", _HERE, src, "-o", out + ".tmp", "-lm"]
    if omp:
        cmd.insert(1, "-fopenmp")
    subprocess.run(cmd, check=True)
    os.replace(out + ".tmp", out)
    return out


def _declare(L: ctypes.CDLL) -> ctypes.CDLL:
    vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    L.sherry_ref_pairsum.argtypes = [vp, i64]
    L.sherry_ref_pairsum.restype = ctypes.c_float
    L.sherry_ref_num_scales.argtypes = [i64, i64, i32, i32]
    L.sherry_ref_num_scales.restype = i64
    L.sherry_ref_quantize_pack.argtypes = [vp, i32, i64, i64, i32, i32, vp, vp, vp]
    L.sherry_ref_quantize_pack.restype = i32
    for f in (L.sherry_ref_unpack_f32, L.sherry_ref_unpack_bf16):
        f.argtypes = [vp, vp, vp, i64, i64, i32, i32, vp]
        f.restype = i32
    L.sherry_ref_linear.argtypes = [vp, i64, vp, i64, vp, vp, vp, i64, i64, i32, i32, vp]
    L.sherry_ref_linear.restype = i32
    L.sherry_ref_fake_quant.argtypes = [vp, i32, i64, i64, i32, i32, vp, vp]
    L.sherry_ref_fake_quant.restype = i32
    L.sherry_ref_tequila_dead.argtypes = [vp, i32, i64, i64, ctypes.c_float, vp, vp]
    L.sherry_ref_tequila_dead.restype = i32
    L.sherry_ref_tequila_term.argtypes = [vp, i64, vp, vp, vp, i64, i64, i32, vp]
    L.sherry_ref_tequila_term.restype = i32
    L.sherry_ref_arenas_linear.argtypes = [vp, i64, vp, vp, vp, vp, ctypes.c_float, i64, i64, i32, i32, vp]
    L.sherry_ref_arenas_linear.restype = i32
    L.sherry_ref_arenas_lambda.argtypes = [i64, i64, ctypes.c_double]
    L.sherry_ref_arenas_lambda.restype = ctypes.c_double
    L.sherry_ref_threads.argtypes = []
    L.sherry_ref_threads.restype = i32
    return L


def load_so(path: str) -> ctypes.CDLL:
    return _declare(ctypes.CDLL(path))


def lib(omp: bool = False) -> ctypes.CDLL:
    """The compiled oracle (built on first use)."""
    with _lock:
        if omp not in _libs:
            _libs[omp] = load_so(build(omp))
        return _libs[omp]


def _p(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


class Oracle:
    """NumPy-array front end over one compiled oracle library."""

    def __init__(self, L: ctypes.CDLL):
        self.L = L

    def num_scales(self, N, K, gran, group=128) -> int:
        return int(self.L.sherry_ref_num_scales(N, K, gran, group))

    def pairsum(self, v) -> np.float32:
        v = np.ascontiguousarray(v, dtype=np.float32)
        return np.float32(self.L.sherry_ref_pairsum(_p(v), v.size))

    def quantize_pack(self, W, gran=PER_GROUP, group=128, w_dtype=None):
        """W: float32 [N,K] or uint16 bf16 bits [N,K] -> (idx u32, sgn u8, scales f32)."""
        W = np.ascontiguousarray(W)
        if w_dtype is None:
            w_dtype = BF16 if W.dtype == np.uint16 else F32
        N, K = W.shape
        ns = self.num_scales(N, K, gran, group)
        if ns < 0:
            raise ValueError("invalid shape/granularity/group")
        idx = np.zeros((N, K // 32), np.uint32)
        sgn = np.zeros((N, K // 32), np.uint8)
        scales = np.zeros(max(ns, 1), np.float32)
        st = self.L.sherry_ref_quantize_pack(_p(W), w_dtype, N, K, gran, group, _p(idx), _p(sgn), _p(scales))
        if st:
            raise ValueError(f"oracle quantize_pack status {st}")
        return idx, sgn, scales[:ns]

    def unpack_f32(self, idx, sgn, scales, N, K, gran=PER_GROUP, group=128):
        out = np.empty((N, K), np.float32)
        st = self.L.sherry_ref_unpack_f32(_p(idx), _p(sgn), _p(np.ascontiguousarray(scales, np.float32)),
                                          N, K, gran, group, _p(out))
        if st:
            raise ValueError(f"oracle unpack status {st}")
        return out

    def unpack_bf16(self, idx, sgn, scales, N, K, gran=PER_GROUP, group=128):
        out = np.empty((N, K), np.uint16)
        st = self.L.sherry_ref_unpack_bf16(_p(idx), _p(sgn), _p(np.ascontiguousarray(scales, np.float32)),
                                           N, K, gran, group, _p(out))
        if st:
            raise ValueError(f"oracle unpack status {st}")
        return out

    def linear(self, X_bf16, idx, sgn, scales, N, K, gran=PER_GROUP, group=128, rows=None):
        """Y (float64) = X Wq^T for all token rows of X, or only for ``rows``."""
        X = np.ascontiguousarray(X_bf16, np.uint16)
        M = X.shape[0]
        r = None if rows is None else np.ascontiguousarray(rows, np.int64)
        nr = M if r is None else r.size
        Y = np.zeros((nr, N), np.float64)
        st = self.L.sherry_ref_linear(_p(X), M, _p(r), nr, _p(idx), _p(sgn),
                                      _p(np.ascontiguousarray(scales, np.float32)), N, K, gran, group, _p(Y))
        if st:
            raise ValueError(f"oracle linear status {st}")
        return Y

    def fake_quant(self, W, gran=PER_GROUP, group=128, w_dtype=None):
        """The quantiser's forward output: (Wq float32 [N,K], Wq as bf16 bits [N,K])."""
        W = np.ascontiguousarray(W)
        if w_dtype is None:
            w_dtype = BF16 if W.dtype == np.uint16 else F32
        N, K = W.shape
        Wq = np.empty((N, K), np.float32)
        Wb = np.empty((N, K), np.uint16)
        st = self.L.sherry_ref_fake_quant(_p(W), w_dtype, N, K, gran, group, _p(Wq), _p(Wb))
        if st:
            raise ValueError(f"oracle fake_quant status {st}")
        return Wq, Wb

    def tequila_dead(self, W, eps, w_dtype=None):
        """(D bf16 bits [N, K/4], bias float32 [N]): the zeroed weight of every block times eps."""
        W = np.ascontiguousarray(W)
        if w_dtype is None:
            w_dtype = BF16 if W.dtype == np.uint16 else F32
        N, K = W.shape
        D = np.empty((N, K // 4), np.uint16)
        bias = np.empty(N, np.float32)
        st = self.L.sherry_ref_tequila_dead(_p(W), w_dtype, N, K, float(eps), _p(D), _p(bias))
        if st:
            raise ValueError(f"oracle tequila_dead status {st}")
        return D, bias

    def tequila_term(self, X_bf16, idx, D, bias, N, K, mode):
        """The dead-weight term T [M, N] (float64); mode 0: bias, 1: sign(X) D^T."""
        X = np.ascontiguousarray(X_bf16, np.uint16)
        M = X.shape[0]
        T = np.zeros((M, N), np.float64)
        st = self.L.sherry_ref_tequila_term(_p(X), M, _p(np.ascontiguousarray(idx)), _p(np.ascontiguousarray(D)),
                                            _p(np.ascontiguousarray(bias, np.float32)), N, K, mode, _p(T))
        if st:
            raise ValueError(f"oracle tequila_term status {st}")
        return T

    def arenas_linear(self, X_bf16, idx, sgn, scales, Wd_bf16, lam, N, K, gran=PER_GROUP, group=128):
        """Y (float64) = X (T alpha)^T + lam * X Wd^T (Wd: the latent weight as bf16 bits [N,K])."""
        X = np.ascontiguousarray(X_bf16, np.uint16)
        M = X.shape[0]
        Y = np.zeros((M, N), np.float64)
        st = self.L.sherry_ref_arenas_linear(_p(X), M, _p(idx), _p(sgn), _p(np.ascontiguousarray(scales, np.float32)),
                                             _p(np.ascontiguousarray(Wd_bf16, np.uint16)), float(lam), N, K, gran,
                                             group, _p(Y))
        if st:
            raise ValueError(f"oracle arenas_linear status {st}")
        return Y

    def arenas_lambda(self, step, total, lam0) -> float:
        return float(self.L.sherry_ref_arenas_lambda(step, total, lam0))

    def threads(self) -> int:
        return int(self.L.sherry_ref_threads())


def oracle(omp: bool = False) -> Oracle:
    return Oracle(lib(omp))
