"""Python binding of the sm_100a 4-bit codebook linear-layer library (libq4.so).

Argument marshalling only: every step of pack, dequant and the matmuls runs in
the CUDA kernels of libq4.so, on the tensors' device, on the current torch
stream.  PyTorch supplies device memory and streams.  There is no CPU path:
if the library cannot be loaded, every call raises.

Q4_LIBRARY=debug in the environment loads libq4_debug.so instead: the same
kernels built with -DQ4_DEBUG, in which each global load and store checks its
index range first and a failed check sets a bit of bounds_flags() and skips
the access.  It is slower and meant for tests only.

Tensor conventions (all contiguous, on one CUDA device):
  w        float32            [N, K]
  codebook float16 or uint16  [16]       (binary16 bits)
  codes    uint8              [N, K/2]   low nibble = even k
  scales   float16 or uint16  [N, K/64]  (binary16 bits)
  x        bfloat16 or uint16 [M, K]     (bfloat16 bits)
  y        float32            [M, N]
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

from . import build as _build

GROUP = 64
_HERE = os.path.dirname(os.path.abspath(__file__))
HEADER = os.path.join(os.path.dirname(_HERE), "include", "q4.h")

STATUS = {0: "Q4_OK", 1: "Q4_ERR_NULL", 2: "Q4_ERR_SHAPE", 3: "Q4_ERR_ALIGN", 4: "Q4_ERR_ARCH",
          5: "Q4_ERR_CUDA", 6: "Q4_ERR_TOO_LARGE"}


class Q4Error(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(message)
        self.status = status


_lib = None


class Q4Linear(ctypes.Structure):
    """struct q4_linear of q4.h: one linear of a recorded step."""
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("codebook", ctypes.c_void_p), ("x", ctypes.c_void_p), ("y", ctypes.c_void_p),
                ("M", ctypes.c_int64), ("N", ctypes.c_int64), ("K", ctypes.c_int64)]


def debug_selected() -> bool:
    """True when Q4_LIBRARY=debug selects the bounds-checked build."""
    v = os.environ.get("Q4_LIBRARY", "").strip().lower()
    if v not in ("", "release", "debug"):
        raise RuntimeError(f"Q4_LIBRARY must be 'release' or 'debug', not {v!r}")
    return v == "debug"


def library_path() -> str:
    return _build.DEBUG_LIBRARY if debug_selected() else _build.LIBRARY


def load(build_if_missing: bool = True) -> ctypes.CDLL:
    """Load libq4.so, or libq4_debug.so under Q4_LIBRARY=debug (building it
    with nvcc first if it is missing or stale)."""
    global _lib
    if _lib is not None:
        return _lib
    debug = debug_selected()
    path = library_path()
    if build_if_missing and _build.stale(path):
        _build.build(debug=debug)
    if not os.path.exists(path):
        raise RuntimeError(f"{os.path.basename(path)} not found at {path}; run "
                           "python -m weight_only_bit_gemv_b200.build" + (" --debug" if debug else ""))
    lib = ctypes.CDLL(path)
    P, I64, S = ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p
    lib.q4_pack.argtypes = [P, P, P, P, I64, I64, S]
    lib.q4_dequant.argtypes = [P, P, P, P, I64, I64, S]
    lib.q4_gemv.argtypes = [P, P, P, P, P, I64, I64, I64, S]
    lib.q4_gemm.argtypes = [P, P, P, P, P, I64, I64, I64, S]
    lib.q4_gemm_noalloc.argtypes = [P, P, P, P, P, I64, I64, I64, S]
    lib.q4_embed_rows.argtypes = [P, P, P, P, P, I64, I64, I64, S]
    lib.q4_pack2.argtypes = [P, P, P, P, I64, I64, S]
    lib.q4_dequant2.argtypes = [P, P, P, P, I64, I64, S]
    lib.q4_gemv2.argtypes = [P, P, P, P, P, I64, I64, S]
    for f in ("q4_pack", "q4_dequant", "q4_gemv", "q4_gemm", "q4_gemm_noalloc", "q4_embed_rows",
              "q4_pack2", "q4_dequant2", "q4_gemv2"):
        getattr(lib, f).restype = ctypes.c_int
    lib.q4_status_string.argtypes = [ctypes.c_int]
    lib.q4_status_string.restype = ctypes.c_char_p
    lib.q4_last_cuda_error.argtypes = []
    lib.q4_last_cuda_error.restype = ctypes.c_int
    lib.q4_abi_version.argtypes = []
    lib.q4_abi_version.restype = ctypes.c_int
    lib.q4_timeout_flags.argtypes = [ctypes.POINTER(ctypes.c_uint32)]
    lib.q4_timeout_flags.restype = ctypes.c_int
    lib.q4_ring_create.argtypes = [I64, ctypes.POINTER(ctypes.c_void_p)]
    lib.q4_ring_create.restype = ctypes.c_int
    lib.q4_ring_gemm.argtypes = [P, P, P, P, P, P, I64, I64, I64, S]
    lib.q4_ring_gemm.restype = ctypes.c_int
    lib.q4_ring_destroy.argtypes = [P]
    lib.q4_ring_destroy.restype = ctypes.c_int
    lib.q4_step_create.argtypes = [ctypes.POINTER(Q4Linear), I64, ctypes.POINTER(ctypes.c_void_p)]
    lib.q4_step_create.restype = ctypes.c_int
    lib.q4_step_launch.argtypes = [P, S]
    lib.q4_step_launch.restype = ctypes.c_int
    lib.q4_step_destroy.argtypes = [P]
    lib.q4_step_destroy.restype = ctypes.c_int
    lib.q4_wait_selftest.argtypes = [ctypes.c_uint32, ctypes.c_int, ctypes.POINTER(ctypes.c_uint32)]
    lib.q4_wait_selftest.restype = ctypes.c_int
    lib.q4_bounds_flags.argtypes = [ctypes.POINTER(ctypes.c_uint32)]
    lib.q4_bounds_flags.restype = ctypes.c_int
    lib.q4_bounds_checked.argtypes = []
    lib.q4_bounds_checked.restype = ctypes.c_int
    _lib = lib
    return lib


def header_functions() -> list:
    """Names of the functions include/q4.h declares."""
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(q4_[a-z0-9_]+)\s*\(", text)))


def status_string(status: int) -> str:
    return load().q4_status_string(int(status)).decode()


def _check(status: int, what: str) -> None:
    if status != 0:
        lib = load()
        msg = f"{what}: {status_string(status)}"
        if status == 5:
            msg += f" (cudaError {lib.q4_last_cuda_error()})"
        raise Q4Error(status, msg)


def _stream(t: torch.Tensor, stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream(t.device)
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _need(t: torch.Tensor, name: str, dtypes, shape=None) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype not in dtypes:
        raise TypeError(f"{name}: dtype {t.dtype} not in {dtypes}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)} != {tuple(shape)}")


_H16 = (torch.float16, torch.uint16, torch.int16)
_BF16 = (torch.bfloat16, torch.uint16, torch.int16)


def _packed_dims(codes: torch.Tensor):
    if codes.dim() != 2:
        raise ValueError("codes must be [N, K/2]")
    return codes.shape[0], codes.shape[1] * 2


def q4_pack(w: torch.Tensor, codebook: torch.Tensor, codes: torch.Tensor = None,
            scales: torch.Tensor = None, stream=None):
    """Quantize w [N, K] fp32 into (codes, scales); allocates them with torch if not given."""
    if w.dim() != 2:
        raise ValueError("w must be [N, K]")
    N, K = w.shape
    if codes is None:
        codes = torch.empty((N, K // 2), dtype=torch.uint8, device=w.device)
    if scales is None:
        scales = torch.empty((N, K // GROUP), dtype=torch.float16, device=w.device)
    _need(w, "w", (torch.float32,))
    _need(codebook, "codebook", _H16, (16,))
    _need(codes, "codes", (torch.uint8,), (N, K // 2))
    _need(scales, "scales", _H16, (N, K // GROUP))
    st = load().q4_pack(w.data_ptr(), codebook.data_ptr(), codes.data_ptr(), scales.data_ptr(),
                        N, K, _stream(w, stream))
    _check(st, "q4_pack")
    return codes, scales


def q4_dequant(codes: torch.Tensor, scales: torch.Tensor, codebook: torch.Tensor,
               w_out: torch.Tensor = None, stream=None) -> torch.Tensor:
    N, K = _packed_dims(codes)
    if w_out is None:
        w_out = torch.empty((N, K), dtype=torch.float32, device=codes.device)
    _need(codes, "codes", (torch.uint8,))
    _need(scales, "scales", _H16, (N, K // GROUP))
    _need(codebook, "codebook", _H16, (16,))
    _need(w_out, "w_out", (torch.float32,), (N, K))
    st = load().q4_dequant(codes.data_ptr(), scales.data_ptr(), codebook.data_ptr(),
                           w_out.data_ptr(), N, K, _stream(codes, stream))
    _check(st, "q4_dequant")
    return w_out


def q4_embed_rows(codes: torch.Tensor, scales: torch.Tensor, codebook: torch.Tensor,
                  ids: torch.Tensor, out: torch.Tensor = None, stream=None) -> torch.Tensor:
    """out [n, K] fp32 = rows ids [n] (int32) of the packed matrix, dequantized
    exactly; ids outside [0, N) give rows of zeros."""
    N, K = _packed_dims(codes)
    if ids.dim() != 1:
        raise ValueError("ids must be [n]")
    n = ids.shape[0]
    if out is None:
        out = torch.empty((n, K), dtype=torch.float32, device=codes.device)
    _need(codes, "codes", (torch.uint8,))
    _need(scales, "scales", _H16, (N, K // GROUP))
    _need(codebook, "codebook", _H16, (16,))
    _need(ids, "ids", (torch.int32,))
    _need(out, "out", (torch.float32,), (n, K))
    st = load().q4_embed_rows(codes.data_ptr(), scales.data_ptr(), codebook.data_ptr(),
                              ids.data_ptr(), out.data_ptr(), n, N, K, _stream(codes, stream))
    _check(st, "q4_embed_rows")
    return out


def _matmul(fn: str, codes, scales, codebook, x, y, stream):
    N, K = _packed_dims(codes)
    if x.dim() != 2 or x.shape[1] != K:
        raise ValueError(f"x must be [M, {K}]")
    M = x.shape[0]
    if y is None:
        y = torch.empty((M, N), dtype=torch.float32, device=codes.device)
    _need(codes, "codes", (torch.uint8,))
    _need(scales, "scales", _H16, (N, K // GROUP))
    _need(codebook, "codebook", _H16, (16,))
    _need(x, "x", _BF16)
    _need(y, "y", (torch.float32,), (M, N))
    st = getattr(load(), fn)(codes.data_ptr(), scales.data_ptr(), codebook.data_ptr(),
                             x.data_ptr(), y.data_ptr(), M, N, K, _stream(codes, stream))
    _check(st, fn)
    return y


# ---- the two-bit variant: codes [N, K/4], a 4-entry codebook ---------------

def q4_pack2(w: torch.Tensor, codebook4: torch.Tensor, codes: torch.Tensor = None,
             scales: torch.Tensor = None, stream=None):
    """Quantize w [N, K] fp32 into 2-bit (codes [N, K/4], scales [N, K/64])."""
    if w.dim() != 2:
        raise ValueError("w must be [N, K]")
    N, K = w.shape
    if codes is None:
        codes = torch.empty((N, K // 4), dtype=torch.uint8, device=w.device)
    if scales is None:
        scales = torch.empty((N, K // GROUP), dtype=torch.float16, device=w.device)
    _need(w, "w", (torch.float32,))
    _need(codebook4, "codebook4", _H16, (4,))
    _need(codes, "codes", (torch.uint8,), (N, K // 4))
    _need(scales, "scales", _H16, (N, K // GROUP))
    st = load().q4_pack2(w.data_ptr(), codebook4.data_ptr(), codes.data_ptr(), scales.data_ptr(),
                         N, K, _stream(w, stream))
    _check(st, "q4_pack2")
    return codes, scales


def _packed2_dims(codes: torch.Tensor):
    if codes.dim() != 2:
        raise ValueError("codes must be [N, K/4]")
    return codes.shape[0], codes.shape[1] * 4


def q4_dequant2(codes: torch.Tensor, scales: torch.Tensor, codebook4: torch.Tensor,
                w_out: torch.Tensor = None, stream=None) -> torch.Tensor:
    N, K = _packed2_dims(codes)
    if w_out is None:
        w_out = torch.empty((N, K), dtype=torch.float32, device=codes.device)
    _need(codes, "codes", (torch.uint8,))
    _need(scales, "scales", _H16, (N, K // GROUP))
    _need(codebook4, "codebook4", _H16, (4,))
    _need(w_out, "w_out", (torch.float32,), (N, K))
    st = load().q4_dequant2(codes.data_ptr(), scales.data_ptr(), codebook4.data_ptr(),
                            w_out.data_ptr(), N, K, _stream(codes, stream))
    _check(st, "q4_dequant2")
    return w_out


def q4_gemv2(codes, scales, codebook4, x, y=None, stream=None) -> torch.Tensor:
    """y [1, N] = x [1, K] @ W^T with W rebuilt from the 2-bit codes in the kernel."""
    N, K = _packed2_dims(codes)
    if x.dim() != 2 or tuple(x.shape) != (1, K):
        raise ValueError(f"x must be [1, {K}]")
    if y is None:
        y = torch.empty((1, N), dtype=torch.float32, device=codes.device)
    _need(codes, "codes", (torch.uint8,))
    _need(scales, "scales", _H16, (N, K // GROUP))
    _need(codebook4, "codebook4", _H16, (4,))
    _need(x, "x", _BF16)
    _need(y, "y", (torch.float32,), (1, N))
    st = load().q4_gemv2(codes.data_ptr(), scales.data_ptr(), codebook4.data_ptr(),
                         x.data_ptr(), y.data_ptr(), N, K, _stream(codes, stream))
    _check(st, "q4_gemv2")
    return y


def q4_gemv(codes, scales, codebook, x, y=None, stream=None) -> torch.Tensor:
    """y [1, N] = x [1, K] @ W^T with W rebuilt from codes/scales/codebook in the kernel."""
    return _matmul("q4_gemv", codes, scales, codebook, x, y, stream)


def q4_gemm(codes, scales, codebook, x, y=None, stream=None) -> torch.Tensor:
    """y [M, N] = x [M, K] @ W^T for any M (M <= 24: verify batches and short
    chunks on the CUDA-core decode kernels; M > 24: prefill on tensor cores)."""
    return _matmul("q4_gemm", codes, scales, codebook, x, y, stream)


def q4_gemm_noalloc(codes, scales, codebook, x, y, stream=None) -> torch.Tensor:
    """q4_gemm without any device allocation by the library: for M > 16 the
    binary16 copy of x lives in the library's fixed 8 MiB device array, so
    2 * M * K must fit in it (else Q4Error Q4_ERR_TOO_LARGE), and calls that
    overlap on the GPU race on that array.  y must be passed in."""
    if y is None:
        raise ValueError("q4_gemm_noalloc writes into a caller-provided y")
    return _matmul("q4_gemm_noalloc", codes, scales, codebook, x, y, stream)


def ring_slot_bytes(N: int, K: int) -> int:
    """Bytes a CopyRing slot needs for one [N, K] matrix (codes padded to 256
    bytes, then scales)."""
    return (N * (K // 2) + 255) // 256 * 256 + N * (K // GROUP) * 2


class Ring:
    """Two device slots fed from host memory ("CopyRing"): ``gemm`` copies a
    matrix's packed codes and scales from (pinned) host tensors into the next
    slot on the ring's copy stream and runs q4_gemm on it, so that the copy of
    one call overlaps the matmul of the previous one."""

    def __init__(self, slot_bytes: int):
        self._h = ctypes.c_void_p()
        _check(load().q4_ring_create(int(slot_bytes), ctypes.byref(self._h)), "q4_ring_create")

    def gemm(self, codes_host: torch.Tensor, scales_host: torch.Tensor, codebook: torch.Tensor,
             x: torch.Tensor, y: torch.Tensor = None, stream=None) -> torch.Tensor:
        if self._h.value is None:
            raise RuntimeError("ring is closed")
        if codes_host.dim() != 2:
            raise ValueError("codes must be [N, K/2]")
        N, K = codes_host.shape[0], codes_host.shape[1] * 2
        for t, name in ((codes_host, "codes_host"), (scales_host, "scales_host")):
            if t.is_cuda or not t.is_contiguous():
                raise ValueError(f"{name} must be a contiguous host tensor")
        if codes_host.dtype != torch.uint8 or scales_host.dtype not in _H16 or \
                tuple(scales_host.shape) != (N, K // GROUP):
            raise TypeError("codes_host uint8 [N, K/2], scales_host binary16 [N, K/64]")
        if x.dim() != 2 or x.shape[1] != K:
            raise ValueError(f"x must be [M, {K}]")
        M = x.shape[0]
        if y is None:
            y = torch.empty((M, N), dtype=torch.float32, device=x.device)
        _need(codebook, "codebook", _H16, (16,))
        _need(x, "x", _BF16)
        _need(y, "y", (torch.float32,), (M, N))
        st = load().q4_ring_gemm(self._h, codes_host.data_ptr(), scales_host.data_ptr(),
                                 codebook.data_ptr(), x.data_ptr(), y.data_ptr(), M, N, K,
                                 _stream(x, stream))
        _check(st, "q4_ring_gemm")
        return y

    def close(self) -> None:
        if self._h.value is not None:
            _check(load().q4_ring_destroy(self._h), "q4_ring_destroy")
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class Step:
    """A decode step recorded once as a CUDA graph (q4_step_create) and
    replayed per token (``launch``).  ``linears`` is a sequence of
    (codes, scales, codebook, x, y) device tensors with the q4_gemm
    conventions; the graph keeps their addresses, so the caller keeps the
    tensors alive and writes each token's activations into the same x."""

    def __init__(self, linears):
        self._keep = []
        arr = (Q4Linear * len(linears))()
        for i, (codes, scales, codebook, x, y) in enumerate(linears):
            N, K = _packed_dims(codes)
            if x.dim() != 2 or x.shape[1] != K:
                raise ValueError(f"linear {i}: x must be [M, {K}]")
            M = x.shape[0]
            _need(codes, "codes", (torch.uint8,))
            _need(scales, "scales", _H16, (N, K // GROUP))
            _need(codebook, "codebook", _H16, (16,))
            _need(x, "x", _BF16)
            _need(y, "y", (torch.float32,), (M, N))
            arr[i] = Q4Linear(codes.data_ptr(), scales.data_ptr(), codebook.data_ptr(),
                              x.data_ptr(), y.data_ptr(), M, N, K)
            self._keep.append((codes, scales, codebook, x, y))
        self._device = self._keep[0][0].device if self._keep else None
        self._h = ctypes.c_void_p()
        _check(load().q4_step_create(arr, len(linears), ctypes.byref(self._h)), "q4_step_create")

    def launch(self, stream=None) -> None:
        if self._h.value is None:
            raise RuntimeError("step is closed")
        if stream is None:
            stream = torch.cuda.current_stream(self._device)
        s = int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)
        _check(load().q4_step_launch(self._h, s), "q4_step_launch")

    def close(self) -> None:
        if self._h.value is not None:
            _check(load().q4_step_destroy(self._h), "q4_step_destroy")
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def wait_selftest(limit_us: int, arrive: bool) -> int:
    """Run the bounded-wait self-test kernel (synchronizes the device); returns
    the microseconds the wait took.  Without ``arrive`` the wait runs out and
    sets bit 7 of timeout_flags()."""
    out = ctypes.c_uint32(0)
    _check(load().q4_wait_selftest(int(limit_us), 1 if arrive else 0, ctypes.byref(out)),
           "q4_wait_selftest")
    return int(out.value)


def timeout_flags() -> int:
    """Synchronize the current device; return and clear the kernels' bounded-wait timeout bits."""
    out = ctypes.c_uint32(0)
    _check(load().q4_timeout_flags(ctypes.byref(out)), "q4_timeout_flags")
    return int(out.value)


def bounds_flags() -> int:
    """Synchronize the current device; return and clear the bits of the
    kernels' failed index checks (always 0 from the release build)."""
    out = ctypes.c_uint32(0)
    _check(load().q4_bounds_flags(ctypes.byref(out)), "q4_bounds_flags")
    return int(out.value)


def bounds_checked() -> bool:
    """True when the loaded library is the bounds-checked build."""
    return bool(load().q4_bounds_checked())


def abi_version() -> int:
    return load().q4_abi_version()


# ---- the C names, one Python function per entry point of include/q4.h ------

def q4_status_string(status: int) -> str:
    return status_string(status)


def q4_last_cuda_error() -> int:
    """The CUDA error code behind the calling thread's last Q4_ERR_CUDA."""
    return int(load().q4_last_cuda_error())


def q4_abi_version() -> int:
    return abi_version()


def q4_timeout_flags() -> int:
    return timeout_flags()


def q4_ring_create(slot_bytes: int) -> Ring:
    return Ring(slot_bytes)


def q4_ring_gemm(ring: Ring, codes_host, scales_host, codebook, x, y=None, stream=None):
    return ring.gemm(codes_host, scales_host, codebook, x, y, stream)


def q4_ring_destroy(ring: Ring) -> None:
    ring.close()


def q4_step_create(linears) -> Step:
    return Step(linears)


def q4_step_launch(step: Step, stream=None) -> None:
    step.launch(stream)


def q4_step_destroy(step: Step) -> None:
    step.close()


def q4_wait_selftest(limit_us: int, arrive: bool) -> int:
    return wait_selftest(limit_us, arrive)


def q4_bounds_flags() -> int:
    return bounds_flags()


def q4_bounds_checked() -> bool:
    return bounds_checked()
