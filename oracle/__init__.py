"""Oracle for the weight-only 4-bit codebook linear layer -- TEST INFRASTRUCTURE.

A ctypes wrapper around ``q4_oracle.c``, the plain single-threaded C
reference.  Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may import this package.  The CUDA library never does, and
this package imports nothing from it.

Every function takes and returns numpy arrays:
  w       float32 [N, K]
  cb      uint16  [16]        binary16 bit patterns
  codes   uint8   [N, K/2]    k = 2j in the low nibble of byte j
  scales  uint16  [N, K/64]   binary16 bit patterns
  x       uint16  [M, K]      bfloat16 bit patterns
  y       float32 [M, N]

``Oracle(path)`` wraps any build of the source; ``build_variant`` compiles an
edited copy of it, which the tests use to plant mistakes and check that the
pins catch them.  The module-level functions use the committed source.
"""
from __future__ import annotations

import ctypes
import hashlib
import os
import subprocess
import tempfile

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "q4_oracle.c")
HEADER = os.path.join(_HERE, "q4_oracle.h")
LIBRARY = os.path.join(_HERE, "libq4oracle.so")
GROUP = 64
CFLAGS = ["-std=c99", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]


def _compile(src: str, out: str) -> None:
    tmp = out + f".tmp{os.getpid()}"
    subprocess.run(["gcc", *CFLAGS, "-I", _HERE, src, "-lm", "-o", tmp], check=True)
    os.replace(tmp, out)


def build(force: bool = False) -> str:
    """Compile the committed oracle (plain IEEE binary32, no FMA contraction)."""
    stale = (not os.path.exists(LIBRARY)
             or os.path.getmtime(LIBRARY) < max(os.path.getmtime(SOURCE), os.path.getmtime(HEADER)))
    if force or stale:
        _compile(SOURCE, LIBRARY)
    return LIBRARY


def build_variant(source_text: str) -> "Oracle":
    """Compile an edited copy of the oracle source into a temporary library."""
    tag = hashlib.sha1(source_text.encode()).hexdigest()[:12]
    d = os.path.join(tempfile.gettempdir(), "q4oracle_variants")
    os.makedirs(d, exist_ok=True)
    src = os.path.join(d, f"v_{tag}.c")
    lib = os.path.join(d, f"libv_{tag}.so")
    if not os.path.exists(lib):
        with open(src, "w") as fh:
            fh.write(source_text)
        _compile(src, lib)
    return Oracle(lib)


def _ptr(a):
    return None if a is None else a.ctypes.data


def _c(a, dtype) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != dtype:
        raise TypeError(f"expected {np.dtype(dtype)}, got {a.dtype}")
    return a


class Oracle:
    def __init__(self, path: str):
        lib = ctypes.CDLL(path)
        P, I64 = ctypes.c_void_p, ctypes.c_int64
        lib.oracle_h2f.restype = ctypes.c_float
        lib.oracle_h2f.argtypes = [ctypes.c_uint16]
        lib.oracle_f2h_rne.restype = ctypes.c_uint16
        lib.oracle_f2h_rne.argtypes = [ctypes.c_float]
        lib.oracle_bf2f.restype = ctypes.c_float
        lib.oracle_bf2f.argtypes = [ctypes.c_uint16]
        for name in ("oracle_f2h_rne_array", "oracle_h2f_array", "oracle_bf2f_array"):
            getattr(lib, name).restype = None
            getattr(lib, name).argtypes = [P, P, I64]
        lib.oracle_nf4_codebook.restype = None
        lib.oracle_nf4_codebook.argtypes = [P]
        lib.oracle_inv_phi.restype = ctypes.c_double
        lib.oracle_inv_phi.argtypes = [ctypes.c_double]
        lib.oracle_pack.restype = ctypes.c_int
        lib.oracle_pack.argtypes = [P, P, P, P, I64, I64]
        lib.oracle_weight.restype = ctypes.c_float
        lib.oracle_weight.argtypes = [P, P, P, I64, I64, I64]
        lib.oracle_dequant.restype = ctypes.c_int
        lib.oracle_dequant.argtypes = [P, P, P, P, I64, I64]
        lib.oracle_matmul.restype = ctypes.c_int
        lib.oracle_matmul.argtypes = [P, P, P, P, I64, I64, I64, P, I64, P, P]
        lib.oracle_embed_rows.restype = ctypes.c_int
        lib.oracle_embed_rows.argtypes = [P, P, P, P, I64, I64, I64, P]
        lib.oracle_pack2.restype = ctypes.c_int
        lib.oracle_pack2.argtypes = [P, P, P, P, I64, I64]
        lib.oracle_weight2.restype = ctypes.c_float
        lib.oracle_weight2.argtypes = [P, P, P, I64, I64, I64]
        lib.oracle_dequant2.restype = ctypes.c_int
        lib.oracle_dequant2.argtypes = [P, P, P, P, I64, I64]
        lib.oracle_matmul2.restype = ctypes.c_int
        lib.oracle_matmul2.argtypes = [P, P, P, P, I64, I64, I64, P, P]
        self.lib = lib
        self.path = path

    # ---- number formats ---------------------------------------------------
    def h2f(self, h) -> np.ndarray:
        h = _c(np.asarray(h, dtype=np.uint16), np.uint16)
        out = np.empty(h.shape, np.float32)
        self.lib.oracle_h2f_array(_ptr(h), _ptr(out), h.size)
        return out

    def f2h_rne(self, f) -> np.ndarray:
        f = _c(np.asarray(f, dtype=np.float32), np.float32)
        out = np.empty(f.shape, np.uint16)
        self.lib.oracle_f2h_rne_array(_ptr(f), _ptr(out), f.size)
        return out

    def bf2f(self, b) -> np.ndarray:
        b = _c(np.asarray(b, dtype=np.uint16), np.uint16)
        out = np.empty(b.shape, np.float32)
        self.lib.oracle_bf2f_array(_ptr(b), _ptr(out), b.size)
        return out

    def inv_phi(self, p: float) -> float:
        return float(self.lib.oracle_inv_phi(float(p)))

    def nf4_codebook(self) -> np.ndarray:
        out = np.empty(16, np.uint16)
        self.lib.oracle_nf4_codebook(_ptr(out))
        return out

    # ---- the method ---------------------------------------------------------
    def pack(self, w, cb):
        """Quantize fp32 W [N, K] -> (codes uint8 [N, K/2], scales uint16 [N, K/64])."""
        w = _c(w, np.float32)
        cb = _c(cb, np.uint16)
        N, K = w.shape
        codes = np.empty((N, K // 2), np.uint8)
        scales = np.empty((N, K // GROUP), np.uint16)
        rc = self.lib.oracle_pack(_ptr(w), _ptr(cb), _ptr(codes), _ptr(scales), N, K)
        if rc != 0:
            raise ValueError(f"oracle_pack: bad shape N={N} K={K}")
        return codes, scales

    def weight(self, codes, scales, cb, n: int, k: int) -> float:
        codes, scales, cb = _c(codes, np.uint8), _c(scales, np.uint16), _c(cb, np.uint16)
        K = codes.shape[1] * 2
        return float(self.lib.oracle_weight(_ptr(codes), _ptr(scales), _ptr(cb), K, n, k))

    def dequant(self, codes, scales, cb) -> np.ndarray:
        codes, scales, cb = _c(codes, np.uint8), _c(scales, np.uint16), _c(cb, np.uint16)
        N, K = codes.shape[0], codes.shape[1] * 2
        out = np.empty((N, K), np.float32)
        rc = self.lib.oracle_dequant(_ptr(codes), _ptr(scales), _ptr(cb), _ptr(out), N, K)
        if rc != 0:
            raise ValueError("oracle_dequant: bad shape")
        return out

    def embed_rows(self, codes, scales, cb, ids) -> np.ndarray:
        """Rows ``ids`` (int32) of the dequantized matrix, fp32 [n, K]; ids
        outside [0, N) give rows of zeros."""
        codes, scales, cb = _c(codes, np.uint8), _c(scales, np.uint16), _c(cb, np.uint16)
        ids = _c(np.asarray(ids, dtype=np.int32), np.int32)
        N, K = codes.shape[0], codes.shape[1] * 2
        out = np.empty((ids.size, K), np.float32)
        rc = self.lib.oracle_embed_rows(_ptr(codes), _ptr(scales), _ptr(cb), _ptr(ids), ids.size,
                                        N, K, _ptr(out))
        if rc != 0:
            raise ValueError("oracle_embed_rows: bad shape")
        return out

    # ---- the two-bit variant: cb4 uint16 [4], codes uint8 [N, K/4] ------------
    def pack2(self, w, cb4):
        w, cb4 = _c(w, np.float32), _c(cb4, np.uint16)
        N, K = w.shape
        codes = np.empty((N, K // 4), np.uint8)
        scales = np.empty((N, K // GROUP), np.uint16)
        if self.lib.oracle_pack2(_ptr(w), _ptr(cb4), _ptr(codes), _ptr(scales), N, K) != 0:
            raise ValueError(f"oracle_pack2: bad shape N={N} K={K}")
        return codes, scales

    def weight2(self, codes, scales, cb4, n: int, k: int) -> float:
        codes, scales, cb4 = _c(codes, np.uint8), _c(scales, np.uint16), _c(cb4, np.uint16)
        return float(self.lib.oracle_weight2(_ptr(codes), _ptr(scales), _ptr(cb4),
                                             codes.shape[1] * 4, n, k))

    def dequant2(self, codes, scales, cb4) -> np.ndarray:
        codes, scales, cb4 = _c(codes, np.uint8), _c(scales, np.uint16), _c(cb4, np.uint16)
        N, K = codes.shape[0], codes.shape[1] * 4
        out = np.empty((N, K), np.float32)
        if self.lib.oracle_dequant2(_ptr(codes), _ptr(scales), _ptr(cb4), _ptr(out), N, K) != 0:
            raise ValueError("oracle_dequant2: bad shape")
        return out

    def matmul2(self, codes, scales, cb4, x):
        codes, scales, cb4 = _c(codes, np.uint8), _c(scales, np.uint16), _c(cb4, np.uint16)
        x = _c(x, np.uint16)
        N, K = codes.shape[0], codes.shape[1] * 4
        M = x.shape[0]
        if x.shape[1] != K:
            raise ValueError("x has the wrong K")
        y = np.empty((M, N), np.float32)
        a = np.empty((M, N), np.float64)
        if self.lib.oracle_matmul2(_ptr(codes), _ptr(scales), _ptr(cb4), _ptr(x), M, N, K,
                                   _ptr(y), _ptr(a)) != 0:
            raise ValueError("oracle_matmul2: bad arguments")
        return y, a

    def matmul(self, codes, scales, cb, x, rows=None, with_abs: bool = True):
        """y [M, n_out] (fp32) and sum|W*x| [M, n_out] (fp64, or None).

        ``rows`` (indices into N) restricts the output to those rows of W."""
        codes, scales, cb = _c(codes, np.uint8), _c(scales, np.uint16), _c(cb, np.uint16)
        x = _c(x, np.uint16)
        N, K = codes.shape[0], codes.shape[1] * 2
        M = x.shape[0]
        if x.shape[1] != K:
            raise ValueError("x has the wrong K")
        if rows is None:
            nout, rptr, nrows = N, None, 0
        else:
            rows = _c(np.asarray(rows, dtype=np.int64), np.int64)
            nout, rptr, nrows = rows.size, _ptr(rows), rows.size
        y = np.empty((M, nout), np.float32)
        a = np.empty((M, nout), np.float64) if with_abs else None
        rc = self.lib.oracle_matmul(_ptr(codes), _ptr(scales), _ptr(cb), _ptr(x), M, N, K,
                                    rptr, nrows, _ptr(y), _ptr(a))
        if rc != 0:
            raise ValueError("oracle_matmul: bad arguments")
        return y, a


_default = None


def default() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle(build())
    return _default


def h2f(h): return default().h2f(h)
def f2h_rne(f): return default().f2h_rne(f)
def bf2f(b): return default().bf2f(b)
def inv_phi(p): return default().inv_phi(p)
def nf4_codebook(): return default().nf4_codebook()
def pack(w, cb): return default().pack(w, cb)
def weight(codes, scales, cb, n, k): return default().weight(codes, scales, cb, n, k)
def dequant(codes, scales, cb): return default().dequant(codes, scales, cb)
def matmul(codes, scales, cb, x, rows=None, with_abs=True):
    return default().matmul(codes, scales, cb, x, rows, with_abs)
def embed_rows(codes, scales, cb, ids): return default().embed_rows(codes, scales, cb, ids)
def pack2(w, cb4): return default().pack2(w, cb4)
def weight2(codes, scales, cb4, n, k): return default().weight2(codes, scales, cb4, n, k)
def dequant2(codes, scales, cb4): return default().dequant2(codes, scales, cb4)
def matmul2(codes, scales, cb4, x): return default().matmul2(codes, scales, cb4, x)
