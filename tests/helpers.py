"""Shared test helpers: independent decoders and the parity tolerance."""
from __future__ import annotations

import numpy as np
import torch

GROUP = 64


def f16_bits_to_f64(bits) -> np.ndarray:
    """binary16 patterns -> float64 via numpy's own float16 type."""
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def bf16_bits_to_f64(bits) -> np.ndarray:
    """bfloat16 patterns -> float64 via torch's bfloat16 type."""
    t = torch.from_numpy(np.ascontiguousarray(np.asarray(bits, dtype=np.uint16)).view(np.int16))
    return t.view(torch.bfloat16).to(torch.float64).numpy()


def f32_to_f16_bits_torch(f) -> np.ndarray:
    """float32 -> binary16 (nearest-even) via torch's conversion."""
    t = torch.from_numpy(np.ascontiguousarray(np.asarray(f, dtype=np.float32)))
    return t.to(torch.float16).view(torch.int16).numpy().view(np.uint16)


def unpack_codes(codes: np.ndarray) -> np.ndarray:
    """uint8 [N, K/2] -> codes [N, K] by the layout convention (low nibble = even k)."""
    codes = np.asarray(codes, dtype=np.uint8)
    out = np.empty((codes.shape[0], codes.shape[1] * 2), np.uint8)
    out[:, 0::2] = codes & 0x0F
    out[:, 1::2] = codes >> 4
    return out


def pack_codes(c: np.ndarray) -> np.ndarray:
    """codes [N, K] in 0..15 -> uint8 [N, K/2] by the layout convention."""
    c = np.asarray(c, dtype=np.uint8)
    return (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)


def within_tolerance(y_test, y_ref, absacc, rel=1e-4, abs_=1e-6):
    """|y_test - y_ref| <= rel * sum_k |w_k x_k| + abs_ elementwise; returns (ok, worst ratio)."""
    y_test = np.asarray(y_test, dtype=np.float64)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    bound = rel * np.asarray(absacc, dtype=np.float64) + abs_
    err = np.abs(y_test - y_ref)
    ok = bool(np.all(err <= bound)) and bool(np.all(np.isfinite(y_test)))
    worst = float(np.max(err / bound)) if err.size else 0.0
    return ok, worst


def oracle_matmul_parallel(codes, scales, cb, x, rows=None, workers=None):
    """oracle.matmul on the given rows of W (all rows if None), split into
    chunks run on host threads.  The oracle is a C library called through
    ctypes, which releases the GIL for the call, so the chunks run on as many
    cores as there are workers; each chunk is the oracle's own serial loop.
    Returns (y [M, n_rows] fp32, sum|W x| [M, n_rows] fp64)."""
    import os
    from concurrent.futures import ThreadPoolExecutor

    import oracle

    N = codes.shape[0]
    rows = np.arange(N, dtype=np.int64) if rows is None else np.asarray(rows, dtype=np.int64)
    workers = workers or max(1, min(32, os.cpu_count() or 1))
    chunks = [c for c in np.array_split(rows, workers) if c.size]
    with ThreadPoolExecutor(max_workers=len(chunks)) as ex:
        parts = list(ex.map(lambda c: oracle.matmul(codes, scales, cb, x, rows=c), chunks))
    return (np.concatenate([p[0] for p in parts], axis=1),
            np.concatenate([p[1] for p in parts], axis=1))
