"""Pins for the oracle: checks against things other than the oracle itself.

Each ``pin_*`` function takes an ``oracle.Oracle`` and raises AssertionError
when the build under test disagrees with an independent fact: a library
routine (numpy float16, torch bfloat16, scipy's normal quantile, numpy fp64
matmul), an exact-arithmetic special case, an invariant of the method, or the
size identity the "deep-fold" page states ("Method": about 3.76x smaller than
BF16).  ``test_mutants_are_caught`` plants mistakes in copies of the oracle
source and checks that every one of them fails at least one pin.
"""
from __future__ import annotations

import os
import re
import concurrent.futures as cf

import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import (GROUP, bf16_bits_to_f64, f16_bits_to_f64, f32_to_f16_bits_torch,
                     pack_codes, unpack_codes)

NF4 = synth.codebook()
RNG = np.random.default_rng(12345)


def _codes_with_extremes(rng, N, K, lo_code=0, hi_code=15):
    """Random codes where every group holds the end code lo_code or hi_code."""
    c = rng.integers(0, 16, size=(N, K), dtype=np.uint8)
    G = K // GROUP
    for n in range(N):
        for g in range(G):
            j = rng.integers(0, GROUP)
            c[n, g * GROUP + j] = hi_code if rng.integers(0, 2) else lo_code
    return c


def _f16_bits(vals):
    return np.asarray(vals, dtype=np.float16).view(np.uint16)


# ---------------------------------------------------------------------------
# number formats
# ---------------------------------------------------------------------------

def pin_h2f_all_patterns(o):
    h = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = o.h2f(h)
    ref = h.view(np.float16).astype(np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def pin_f2h_structured(o):
    """Every binary16 rounding boundary and its neighbours, plus random patterns,
    against torch's float -> half conversion."""
    h = np.arange(0, 0x7C00, dtype=np.uint32)
    v = h.astype(np.uint16).view(np.float16).astype(np.float64)
    nxt = np.append(v[1:], 65520.0)
    mids = ((v + nxt) / 2).astype(np.float32)          # exact midpoints (all fit in fp32)
    base = mids.view(np.uint32).astype(np.int64)
    cand = [base + d for d in (-2, -1, 0, 1, 2)]
    cand.append(v.astype(np.float32).view(np.uint32).astype(np.int64))
    cand.append(RNG.integers(0, 2**32, size=1 << 20, dtype=np.int64))
    u = np.concatenate(cand) & 0x7FFFFFFF
    u = np.concatenate([u, u | 0x80000000]).astype(np.uint32)
    f = u.view(np.float32)
    got = o.f2h_rne(f)
    ref = f32_to_f16_bits_torch(f)
    nan = np.isnan(f)
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.all((got[nan] & 0x7C00) == 0x7C00) and np.all((got[nan] & 0x3FF) != 0)


def pin_bf2f_all_patterns(o):
    b = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    with np.errstate(invalid="ignore"):
        got = o.bf2f(b).astype(np.float64)
    ref = bf16_bits_to_f64(b)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


# ---------------------------------------------------------------------------
# codebook
# ---------------------------------------------------------------------------

def pin_nf4_against_scipy(o):
    """The NormalFloat construction redone with scipy's normal quantile."""
    from scipy.stats import norm
    p_max = 1.0 - 0.5 * (1.0 / 30.0 + 1.0 / 32.0)
    pos = norm.ppf(np.linspace(p_max, 0.5, 9)[:-1])
    neg = -norm.ppf(np.linspace(p_max, 0.5, 8)[:-1])
    v = np.sort(np.concatenate([pos, [0.0], neg])) / norm.ppf(p_max)
    ref = v.astype(np.float16).view(np.uint16)   # direct float64 -> float16
    got = o.nf4_codebook()
    assert np.array_equal(got, ref), (got, ref)
    vals = f16_bits_to_f64(got)
    assert vals[0] == -1.0 and vals[7] == 0.0 and vals[15] == 1.0
    assert np.all(np.diff(vals) > 0)


def pin_inv_phi(o):
    from scipy.stats import norm
    for p in (0.5, 0.6, 0.9, 0.9677083333, 0.99, 1e-3):
        assert abs(o.inv_phi(p) - norm.ppf(p)) < 1e-12


# ---------------------------------------------------------------------------
# dequant
# ---------------------------------------------------------------------------

def pin_dequant_nibble_order(o):
    """A hand-built byte 0x21 holds code 1 at even k and code 2 at odd k."""
    codes = np.zeros((1, 32), np.uint8)
    codes[0, 0] = 0x21
    scales = _f16_bits([0.5])[None, :]
    w = o.dequant(codes, scales, NF4)
    cbv = f16_bits_to_f64(NF4)
    assert w[0, 0] == cbv[1] * 0.5 and w[0, 1] == cbv[2] * 0.5
    assert w[0, 2] == cbv[0] * 0.5
    assert o.weight(codes, scales, NF4, 0, 1) == cbv[2] * 0.5


def pin_dequant_is_codebook_times_scale(o):
    """Uniform code i with a unit scale gives cb[i] itself; power-of-two scales
    scale it exactly; each group uses its own scale; a zero scale gives zero."""
    cbv = f16_bits_to_f64(NF4)
    K = 4 * GROUP
    codes = np.zeros((16, K // 2), np.uint8)
    for i in range(16):
        codes[i, :] = i | (i << 4)
    pows = np.array([1.0, 0.25, 8.0, 0.0])
    scales = np.tile(_f16_bits(pows), (16, 1))
    w = o.dequant(codes, scales, NF4).astype(np.float64)
    for i in range(16):
        for g in range(4):
            assert np.all(w[i, g * GROUP:(g + 1) * GROUP] == cbv[i] * pows[g])


def pin_dequant_exact_product(o):
    """W = cb[c] * s is exact in binary32: it equals the fp64 product of the
    numpy-decoded binary16 operands, for random codes and scales (subnormal
    scales included)."""
    rng = np.random.default_rng(7)
    N, K = 8, 4 * GROUP
    codes = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    sbits = rng.integers(0, 0x7C00, size=(N, K // GROUP)).astype(np.uint16)
    cb = rng.integers(0, 0x7C00, size=16).astype(np.uint16) | (rng.integers(0, 2, size=16) << 15).astype(np.uint16)
    w = o.dequant(codes, sbits, cb).astype(np.float64)
    c = unpack_codes(codes)
    ref = f16_bits_to_f64(cb)[c] * np.repeat(f16_bits_to_f64(sbits), GROUP, axis=1)
    assert np.array_equal(w, ref)


# ---------------------------------------------------------------------------
# pack
# ---------------------------------------------------------------------------

def pin_pack_round_trip(o):
    """Weights lying exactly on cb * s, with a +-1 entry in every group (so the
    group's absmax is s), re-quantize to the same codes and scales."""
    rng = np.random.default_rng(11)
    N, K = 6, 8 * GROUP
    for cb in (NF4, NF4[rng.permutation(16)]):
        cbv = f16_bits_to_f64(cb)
        lo, hi = int(np.argmin(cbv)), int(np.argmax(cbv))
        c = _codes_with_extremes(rng, N, K, lo, hi)
        s = rng.uniform(0.001, 2.0, size=(N, K // GROUP)).astype(np.float16)
        w = (cbv[c] * np.repeat(s.astype(np.float64), GROUP, axis=1)).astype(np.float32)
        codes, scales = o.pack(w, cb)
        assert np.array_equal(scales, s.view(np.uint16))
        assert np.array_equal(codes, pack_codes(c))


def pin_pack_scale_is_f16_absmax(o):
    rng = np.random.default_rng(3)
    w = (rng.standard_normal((5, 6 * GROUP)) * rng.uniform(1e-6, 30, size=(5, 1))).astype(np.float32)
    w[0, :GROUP] *= 1e-4    # subnormal binary16 scales
    _, scales = o.pack(w, NF4)
    amax = np.abs(w.reshape(5, -1, GROUP)).max(axis=2)
    assert np.array_equal(scales, f32_to_f16_bits_torch(amax))


def pin_pack_nearest(o):
    """Brute force: every code is a nearest codebook entry to w/s (fp64 distances,
    with slack for the binary32 division), and dequantization error is bounded
    by half the widest codebook gap times s."""
    rng = np.random.default_rng(5)
    N, K = 16, 4 * GROUP
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    codes, scales = o.pack(w, NF4)
    c = unpack_codes(codes)
    s = np.repeat(f16_bits_to_f64(scales), GROUP, axis=1)
    r = w.astype(np.float64) / s
    cbv = f16_bits_to_f64(NF4)
    d = np.abs(r[..., None] - cbv[None, None, :])
    chosen = np.take_along_axis(d, c[..., None].astype(np.int64), axis=2)[..., 0]
    assert np.all(chosen <= d.min(axis=2) + 1e-6)
    wq = cbv[c] * s
    assert np.all(np.abs(wq - w) <= 0.5 * np.max(np.diff(cbv)) * s * (1 + 1e-6))


def pin_pack_monotone(o):
    """With a sorted codebook and a fixed scale the code is nondecreasing in w."""
    w = np.linspace(-1.0, 1.0, 4 * GROUP).astype(np.float32)[None, :]
    for g in range(4):
        w[0, g * GROUP] = -1.0     # pin every group's absmax to 1
    codes, scales = o.pack(w, NF4)
    assert np.all(f16_bits_to_f64(scales) == 1.0)
    c = unpack_codes(codes)[0]
    for g in range(4):
        cg = c[g * GROUP + 1:(g + 1) * GROUP]
        assert np.all(np.diff(cg.astype(int)) >= 0)
    assert c[0] == 0 and c[-1] == 15


def pin_pack_ties_to_lowest_index(o):
    """Integer codebook {-8..7}, group absmax 8: w/s = +-0.5 lies exactly
    between two entries; the lower index wins."""
    cb = synth.integer_codebook()
    w = np.zeros((1, GROUP), np.float32)
    w[0, 0] = 8.0
    w[0, 1] = 4.0      # r = 0.5: entries 0 (index 8) and 1 (index 9)
    w[0, 2] = -4.0     # r = -0.5: entries -1 (index 7) and 0 (index 8)
    w[0, 3] = 12.0 / 8  # r = 0.1875: nearest 0 (index 8)
    codes, scales = o.pack(w, cb)
    c = unpack_codes(codes)[0]
    assert f16_bits_to_f64(scales)[0, 0] == 8.0
    assert c[0] == 9 and c[1] == 8 and c[2] == 7 and c[3] == 8


def pin_pack_zero_groups(o):
    """An all-zero group, and one too small for a binary16 scale, get scale 0
    and the index of the zero entry; they dequantize to zero rows."""
    w = np.zeros((2, 2 * GROUP), np.float32)
    w[1, GROUP:] = 1e-9
    w[1, :GROUP] = np.linspace(-1, 1, GROUP)
    codes, scales = o.pack(w, NF4)
    assert scales[0, 0] == 0 and scales[0, 1] == 0 and scales[1, 1] == 0
    c = unpack_codes(codes)
    assert np.all(c[0] == 7) and np.all(c[1, GROUP:] == 7)
    wq = o.dequant(codes, scales, NF4)
    assert np.all(wq[0] == 0) and np.all(wq[1, GROUP:] == 0)


def pin_pack_codebook_permutation(o):
    """Permuting the codebook permutes the codes and leaves W unchanged."""
    rng = np.random.default_rng(9)
    w = (rng.standard_normal((8, 4 * GROUP)) * 0.02).astype(np.float32)
    perm = rng.permutation(16)
    cb_p = NF4[perm]
    c1, s1 = o.pack(w, NF4)
    c2, s2 = o.pack(w, cb_p)
    assert np.array_equal(s1, s2)
    inv = np.argsort(perm)
    assert np.array_equal(inv[unpack_codes(c1)], unpack_codes(c2))
    assert np.array_equal(o.dequant(c1, s1, NF4), o.dequant(c2, s2, cb_p))


def pin_size_identity(o):
    """Packed payload = N*K/2 code bytes + N*K/64 binary16 scales, which is
    64/17 = 3.7647x smaller than BF16: the page's "about 3.76x"."""
    N, K = 12, 4096
    codes, scales = o.pack(np.zeros((N, K), np.float32), NF4)
    payload = codes.nbytes + scales.nbytes
    assert payload == N * K // 2 + N * K // 32
    ratio = (2 * N * K) / payload
    assert abs(ratio - 64 / 17) < 1e-12 and round(ratio, 2) == 3.76


# ---------------------------------------------------------------------------
# matmul
# ---------------------------------------------------------------------------

def pin_matmul_bruteforce(o):
    """fp64 numpy matmul of the explicitly dequantized matrix (checked above)
    by x decoded with torch, on tiny shapes."""
    rng = np.random.default_rng(21)
    for M, N, K in ((1, 5, 64), (3, 7, 192), (4, 128, 256)):
        codes = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
        scales = synth.f32_to_f16_bits(rng.uniform(0.005, 0.05, size=(N, K // GROUP)).astype(np.float32))
        x = synth.f32_to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
        y, a = o.matmul(codes, scales, NF4, x)
        W = o.dequant(codes, scales, NF4).astype(np.float64)
        X = bf16_bits_to_f64(x)
        ref = X @ W.T
        assert y.shape == (M, N)
        assert np.all(np.abs(y - ref) <= np.abs(ref) * 2.0 ** -24 + 1e-300)
        assert np.allclose(a, np.abs(X) @ np.abs(W).T, rtol=1e-12, atol=0)


def pin_matmul_one_hot(o):
    """x = e_k selects column k of W exactly."""
    rng = np.random.default_rng(2)
    N, K = 9, 3 * GROUP
    codes = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    scales = synth.f32_to_f16_bits(rng.uniform(0.005, 0.05, size=(N, K // GROUP)).astype(np.float32))
    W = o.dequant(codes, scales, NF4)
    ks = [0, 1, 63, 64, 130, K - 1]
    x = np.zeros((len(ks), K), np.uint16)
    for i, k in enumerate(ks):
        x[i, k] = 0x3F80          # bfloat16 1.0
    y, _ = o.matmul(codes, scales, NF4, x)
    for i, k in enumerate(ks):
        assert np.array_equal(y[i], W[:, k])


def pin_matmul_integer_exact(o):
    """Integer codebook, power-of-two scales, small-integer x: the result is an
    exact integer that numpy's int64 matmul reproduces."""
    rng = np.random.default_rng(4)
    M, N, K = 3, 11, 5 * GROUP
    cb = synth.integer_codebook()
    c = rng.integers(0, 16, size=(N, K), dtype=np.uint8)
    e = rng.integers(0, 3, size=(N, K // GROUP))
    scales = _f16_bits(2.0 ** e)
    xi = rng.integers(-4, 5, size=(M, K))
    x = synth.f32_to_bf16_bits(xi.astype(np.float32))
    y, _ = o.matmul(pack_codes(c), scales, cb, x)
    Wi = (c.astype(np.int64) - 8) * np.repeat(2 ** e, GROUP, axis=1)
    assert np.all(np.isfinite(y)) and np.all(y == np.round(y)) and np.all(np.abs(y) < 2.0 ** 62)
    assert np.array_equal(y.astype(np.int64), xi @ Wi.T)


def pin_matmul_zero_scales(o):
    rng = np.random.default_rng(6)
    codes = rng.integers(0, 256, size=(4, GROUP), dtype=np.uint8)
    scales = np.zeros((4, 2), np.uint16)
    x = synth.f32_to_bf16_bits(rng.standard_normal((2, 2 * GROUP)).astype(np.float32))
    y, a = o.matmul(codes, scales, NF4, x)
    assert np.all(y == 0) and np.all(a == 0)


def pin_matmul_linear_in_x(o):
    """y(x1 + x2) = y(x1) + y(x2): small-integer x keep the sums exact in bf16,
    and fp64 accumulation keeps the identity to the last binary32 rounding."""
    rng = np.random.default_rng(8)
    N, K = 13, 4 * GROUP
    codes = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    scales = synth.f32_to_f16_bits(rng.uniform(0.005, 0.05, size=(N, K // GROUP)).astype(np.float32))
    x1 = rng.integers(-8, 9, size=(1, K)).astype(np.float32)
    x2 = rng.integers(-8, 9, size=(1, K)).astype(np.float32)
    b = synth.f32_to_bf16_bits
    y1, _ = o.matmul(codes, scales, NF4, b(x1))
    y2, _ = o.matmul(codes, scales, NF4, b(x2))
    y12, _ = o.matmul(codes, scales, NF4, b(x1 + x2))
    s = y1.astype(np.float64) + y2.astype(np.float64)
    assert np.all(np.abs(y12 - s) <= 2.0 ** -23 * (np.abs(y1) + np.abs(y2)) + 1e-12)


def pin_matmul_row_subset(o):
    rng = np.random.default_rng(10)
    N, K = 20, 2 * GROUP
    codes = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    scales = synth.f32_to_f16_bits(rng.uniform(0.005, 0.05, size=(N, K // GROUP)).astype(np.float32))
    x = synth.f32_to_bf16_bits(rng.standard_normal((3, K)).astype(np.float32))
    y, a = o.matmul(codes, scales, NF4, x)
    rows = np.array([19, 0, 7, 7])
    ys, as_ = o.matmul(codes, scales, NF4, x, rows=rows)
    assert np.array_equal(ys, y[:, rows]) and np.array_equal(as_, a[:, rows])


def pin_embed_rows_definition(o):
    """Embedding rows ("deep-fold", introduction and Figure 1: only the
    requested rows are decoded): each output row equals cb[code] * scale of
    that row, computed here from the bytes with numpy's own binary16 ->
    binary32 conversion and binary32 product; ids outside [0, N) give zeros;
    repeated ids repeat the row."""
    rng = np.random.default_rng(12)
    N, K = 23, 3 * GROUP
    codes = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    scales = synth.f32_to_f16_bits(rng.uniform(0.005, 0.05, size=(N, K // GROUP)).astype(np.float32))
    ids = np.array([5, 0, 22, -1, 23, 5, 1 << 30, 11], np.int32)
    got = o.embed_rows(codes, scales, NF4, ids)
    cbf = NF4.view(np.float16).astype(np.float32)
    sf = scales.view(np.float16).astype(np.float32)
    lo, hi = codes & 0x0F, codes >> 4
    nib = np.empty((N, K), np.uint8)
    nib[:, 0::2], nib[:, 1::2] = lo, hi
    w = cbf[nib] * np.repeat(sf, GROUP, axis=1)
    for i, n in enumerate(ids):
        want = w[n] if 0 <= n < N else np.zeros(K, np.float32)
        assert np.array_equal(got[i], want), f"row {i} (id {n})"


# ---- the two-bit variant (4-entry codebook, four codes per byte) -----------

CB4 = synth.codebook2()


def _decode2_numpy(codes, scales, cb4):
    """W of the two-bit format straight from the bytes, with numpy's own
    binary16 -> binary32 conversion and binary32 product."""
    N, K = codes.shape[0], codes.shape[1] * 4
    cbf = cb4.view(np.float16).astype(np.float32)
    sf = scales.view(np.float16).astype(np.float32)
    idx = np.empty((N, K), np.uint8)
    for i in range(4):
        idx[:, i::4] = (codes >> (2 * i)) & 3
    return cbf[idx] * np.repeat(sf, GROUP, axis=1)


def pin_two_bit_bit_order(o):
    """Byte 0xE4 = 0b11_10_01_00 holds codes 0, 1, 2, 3 for k = 0..3."""
    codes = np.full((1, GROUP // 4), 0xE4, np.uint8)
    scales = np.array([[0x3C00]], np.uint16)                 # scale 1
    cbf = CB4.view(np.float16).astype(np.float32)
    for k in range(4):
        assert o.weight2(codes, scales, CB4, 0, k) == cbf[k]


def pin_two_bit_dequant_definition(o):
    rng = np.random.default_rng(21)
    N, K = 9, 3 * GROUP
    codes = rng.integers(0, 256, size=(N, K // 4), dtype=np.uint8)
    scales = synth.f32_to_f16_bits(rng.uniform(0.005, 0.05, size=(N, K // GROUP)).astype(np.float32))
    assert np.array_equal(o.dequant2(codes, scales, CB4), _decode2_numpy(codes, scales, CB4))


def pin_two_bit_pack_round_trip(o):
    """W built on the grid (each group holds a code of magnitude 1, so the
    absmax is the scale) packs back to the same codes and scales."""
    rng = np.random.default_rng(22)
    N, K = 6, 4 * GROUP
    idx = rng.integers(0, 4, size=(N, K)).astype(np.uint8)
    idx[:, ::GROUP] = 3                                       # cb4[3] = +1 in every group
    s = np.asarray(2.0 ** rng.integers(-8, -3, size=(N, K // GROUP)), np.float16)
    w = CB4.view(np.float16).astype(np.float32)[idx] * np.repeat(s.astype(np.float32), GROUP, axis=1)
    codes, scales = o.pack2(w, CB4)
    assert np.array_equal(scales, s.view(np.uint16))
    assert np.array_equal(_decode2_numpy(codes, scales, CB4), w)


def pin_two_bit_pack_brute_force(o):
    """Each code is the nearest entry to w / scale in binary32, ties to the
    lowest index; scale = binary16(absmax); zero groups take the entry of
    smallest magnitude (index 1: |-1/3| ties |1/3|, lowest index)."""
    rng = np.random.default_rng(23)
    N, K = 7, 2 * GROUP
    w = (rng.standard_normal((N, K)) * 0.03).astype(np.float32)
    w[2, :GROUP] = 0.0
    codes, scales = o.pack2(w, CB4)
    cbf = CB4.view(np.float16).astype(np.float32)
    amax = np.abs(w.reshape(N, K // GROUP, GROUP)).max(axis=2)
    assert np.array_equal(scales, amax.astype(np.float16).view(np.uint16))
    sf = np.repeat(scales.view(np.float16).astype(np.float32), GROUP, axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        r = (w / sf).astype(np.float32)
    want = np.argmin(np.abs(r[..., None] - cbf), axis=-1)
    want[sf == 0] = 1
    got = np.empty((N, K), np.int64)
    for i in range(4):
        got[:, i::4] = (codes >> (2 * i)) & 3
    assert np.array_equal(got, want)


def pin_two_bit_pack_ties(o):
    """Values exactly halfway between two entries take the lower index:
    0 sits between -1/3 and 1/3 (index 1), the midpoints of the binary16
    entries (exact in binary32) go to indices 0, 1 and 2."""
    cbf = CB4.view(np.float16).astype(np.float32)
    mids = [(cbf[0] + cbf[1]) / 2, np.float32(0.0), (cbf[2] + cbf[3]) / 2]
    w = np.zeros((1, GROUP), np.float32)
    w[0, 0] = 0.25                                            # absmax, a power of two
    w[0, 1:4] = np.array(mids, np.float32) * np.float32(0.25)
    codes, scales = o.pack2(w, CB4)
    assert scales[0, 0] == 0x3400
    got = [(codes[0, k // 4] >> (2 * (k % 4))) & 3 for k in range(4)]
    assert got == [3, 0, 1, 2]


def pin_two_bit_codebook_permutation(o):
    """Permuting the codebook and inverse-permuting the codes leaves W, and
    so y, unchanged (the codebook is looked up, never assumed sorted)."""
    rng = np.random.default_rng(25)
    N, K = 5, 2 * GROUP
    codes = rng.integers(0, 256, size=(N, K // 4), dtype=np.uint8)
    scales = synth.f32_to_f16_bits(rng.uniform(0.005, 0.05, size=(N, K // GROUP)).astype(np.float32))
    perm = np.array([2, 0, 3, 1])                       # new entry j = old entry perm[j]
    inv = np.argsort(perm)                              # old index c -> new index inv[c]
    cb_p = CB4[perm]
    codes_p = np.zeros_like(codes)
    for i in range(4):
        codes_p |= (inv[(codes >> (2 * i)) & 3].astype(np.uint8) << (2 * i))
    assert np.array_equal(o.dequant2(codes_p, scales, cb_p), o.dequant2(codes, scales, CB4))
    x = synth.f32_to_bf16_bits(rng.standard_normal((1, K)).astype(np.float32))
    assert np.array_equal(o.matmul2(codes_p, scales, cb_p, x)[0], o.matmul2(codes, scales, CB4, x)[0])


def pin_two_bit_matmul_one_hot(o):
    """x = e_k picks column k of W exactly."""
    rng = np.random.default_rng(26)
    N, K = 9, 3 * GROUP
    codes = rng.integers(0, 256, size=(N, K // 4), dtype=np.uint8)
    scales = synth.f32_to_f16_bits(rng.uniform(0.005, 0.05, size=(N, K // GROUP)).astype(np.float32))
    W = _decode2_numpy(codes, scales, CB4)
    for k in (0, 1, 63, 64, K - 1):
        x = np.zeros((1, K), np.uint16)
        x[0, k] = 0x3F80                                  # bf16 1.0
        assert np.array_equal(o.matmul2(codes, scales, CB4, x)[0][0], W[:, k])


def pin_two_bit_matmul_brute_force(o):
    rng = np.random.default_rng(24)
    N, K, M = 11, 2 * GROUP, 3
    codes = rng.integers(0, 256, size=(N, K // 4), dtype=np.uint8)
    scales = synth.f32_to_f16_bits(rng.uniform(0.005, 0.05, size=(N, K // GROUP)).astype(np.float32))
    x = synth.f32_to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    y, a = o.matmul2(codes, scales, CB4, x)
    W = _decode2_numpy(codes, scales, CB4).astype(np.float64)
    xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    ref = np.array([[sum(W[n, k] * xf[m, k] for k in range(K)) for n in range(N)] for m in range(M)])
    assert np.array_equal(y, ref.astype(np.float32))
    assert np.allclose(a, np.abs(xf) @ np.abs(W).T, rtol=1e-13, atol=0)


PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(orc, pin):
    pin(orc)


def test_fixture_matches_oracle(orc):
    assert np.array_equal(synth.codebook(), orc.nf4_codebook())


# ---------------------------------------------------------------------------
# exhaustive binary32 -> binary16 check (all 2^32 patterns, in parallel)
# ---------------------------------------------------------------------------

def _f2h_chunk(start: int) -> int:
    import numpy as _np
    import torch as _t
    import oracle as _o
    u = _np.arange(start, start + (1 << 24), dtype=_np.uint64).astype(_np.uint32)
    f = u.view(_np.float32)
    got = _o.f2h_rne(f)
    ref = _t.from_numpy(f).to(_t.float16).view(_t.int16).numpy().view(_np.uint16)
    nan = _np.isnan(f)
    bad = (got != ref) & ~nan
    bad |= nan & (((got & 0x7C00) != 0x7C00) | ((got & 0x3FF) == 0))
    return int(bad.sum())


def test_f2h_exhaustive(orc):
    starts = [i << 24 for i in range(256)]
    workers = min(8, os.cpu_count() or 1)
    ctx = __import__("multiprocessing").get_context("spawn")
    with cf.ProcessPoolExecutor(max_workers=workers, mp_context=ctx) as ex:
        bad = sum(ex.map(_f2h_chunk, starts))
    assert bad == 0


# ---------------------------------------------------------------------------
# planted mistakes: each must fail at least one pin
# ---------------------------------------------------------------------------

MUTANTS = {
    "weight_nibble_swap": ("(byte & 0x0F) : (byte >> 4)", "(byte >> 4) : (byte & 0x0F)"),
    "pack_nibble_swap": ("c[2 * j] | (c[2 * j + 1] << 4)", "c[2 * j + 1] | (c[2 * j] << 4)"),
    "scale_dropped": ("return v * s;", "return v;"),
    "scale_wrong_group": ("+ k / ORACLE_GROUP]);", "+ (k / ORACLE_GROUP) / 2]);"),
    "x_transposed": ("oracle_bf2f(x[m * K + k])", "oracle_bf2f(x[k * M + m])"),
    "last_k_dropped": ("for (int64_t k = 0; k < K; ++k) {\n                double p",
                       "for (int64_t k = 0; k < K - 1; ++k) {\n                double p"),
    "tie_to_highest": ("if (d < bestd) {", "if (d <= bestd) {"),
    "f2h_truncates": ("q = rint(ldexp(a, 10 - E));", "q = floor(ldexp(a, 10 - E));"),
    "f2h_subnormal_scale": ("q = rint(ldexp(a, 24));", "q = rint(ldexp(a, 23));"),
    "h2f_sign": ("return (float)(sign ? -v : v);", "return (float)(sign ? v : -v);"),
    "h2f_subnormal": ("v = ldexp((double)frac, -24);", "v = ldexp((double)frac, -25);"),
    "h2f_bias": ("frac + 1024), e - 25)", "frac + 1024), e - 24)"),
    "absmax_signed": ("float m = fabsf(wg[j]);", "float m = wg[j];"),
    "bf2f_shift": ("(uint32_t)b << 16", "(uint32_t)b << 15"),
    "zero_code_first": ("c[j] = zero_code;", "c[j] = 0;"),
    "nf4_neg_spacing": ("(double)i / 7.0", "(double)i / 8.0"),
    "divide_becomes_multiply": ("float r = wg[j] / s;", "float r = wg[j] * s;"),
    "abs_sum_signed": ("aacc += fabs(p);", "aacc += p;"),
    "embed_out_of_range_clamped": ("(n >= 0 && n < N) ? oracle_weight(codes, scales, cb, K, n, k) : 0.0f",
                                   "oracle_weight(codes, scales, cb, K, n < 0 ? 0 : (n >= N ? N - 1 : n), k)"),
    "embed_row_off_by_one": ("? oracle_weight(codes, scales, cb, K, n, k)",
                             "? oracle_weight(codes, scales, cb, K, n > 0 ? n - 1 : 0, k)"),
    "two_bit_order_reversed": ("int code = (b >> (2 * (k % 4))) & 3;", "int code = (b >> (2 * (3 - k % 4))) & 3;"),
    "two_bit_pack_order_reversed": ("(code << (2 * (j % 4)))", "(code << (2 * (3 - j % 4)))"),
    "two_bit_tie_to_highest": ("if (di < dist) {", "if (di <= dist) {"),
    "two_bit_scale_wrong_group": ("+ (k / ORACLE_GROUP)]);", "+ (k / ORACLE_GROUP) / 2]);"),
    "two_bit_zero_scale_first": ("(sv == 0.0f) ? least :", "(sv == 0.0f) ? 0 :"),
    "two_bit_abs_sum_signed": ("abs_sum += fabs(prod);", "abs_sum += prod;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutants_are_caught(name):
    with open(oracle.SOURCE) as fh:
        src = fh.read()
    old, new = MUTANTS[name]
    assert src.count(old) == 1, f"mutation site for {name} not unique"
    mutant = oracle.build_variant(src.replace(old, new))
    failed = []
    for pin in PINS:
        try:
            pin(mutant)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"mutant {name} passed every pin"
