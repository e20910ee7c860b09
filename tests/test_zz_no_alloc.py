"""q4_gemm_noalloc: the entry point for callers that may not allocate device
memory (engines whose memory is all reserved up front, hosts that forbid hidden
allocations).  It must give what q4_gemm gives, within the parity tolerance,
while keeping the binary16 copy of x in the library's fixed device array.

Two calls in a row on different inputs check that what the first call leaves in
the shared array does not leak into the second.  This file sorts last so that a
run stopping at the first failure has run every other test before it; it also
passes on its own in a fresh process.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import synth
import weight_only_bit_gemv_b200 as q4
from helpers import GROUP, oracle_matmul_parallel, within_tolerance

pytestmark = pytest.mark.gpu

NF4 = synth.codebook()
SCRATCH = 8 << 20   # Q4_NOALLOC_SCRATCH_BYTES


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    q4.load()


def _dev16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()


def _call(name, codes, scales, cb, x, y):
    """One call through the C ABI; returns the status."""
    M, K = x.shape
    st = getattr(q4.load(), name)(codes.data_ptr(), scales.data_ptr(), cb.data_ptr(), x.data_ptr(),
                                  y.data_ptr(), M, codes.shape[0], K,
                                  torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    return st


def _case(seed, M, N, K):
    rng = np.random.default_rng(seed)
    codes = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    scales = synth.f32_to_f16_bits(rng.uniform(0.005, 0.05, size=(N, K // GROUP)).astype(np.float32))
    x = synth.activations(seed + 1, M, K)
    return codes, scales, x


def _compare(seed, M, N, K, cb):
    """q4_gemm_noalloc against the oracle's y and against q4_gemm's y, both
    within the parity tolerance."""
    codes, scales, x = _case(seed, M, N, K)
    c, s, xd = torch.from_numpy(codes).cuda(), _dev16(scales), _dev16(x)
    y_gemm = torch.full((M, N), float("nan"), device="cuda")
    y_new = torch.full((M, N), float("nan"), device="cuda")
    assert _call("q4_gemm", c, s, cb, xd, y_gemm) == 0
    assert _call("q4_gemm_noalloc", c, s, cb, xd, y_new) == 0
    y_ref, absacc = oracle_matmul_parallel(codes, scales, NF4, x)
    new, old = y_new.cpu().numpy(), y_gemm.cpu().numpy()
    ok, worst = within_tolerance(new, y_ref, absacc)
    assert ok, f"M={M} N={N} K={K}: against the oracle, worst err/bound = {worst:.3g}"
    ok, worst = within_tolerance(new, old, absacc)
    assert ok, f"M={M} N={N} K={K}: against q4_gemm, worst err/bound = {worst:.3g}"


def test_matches_oracle_on_two_calls_in_a_row():
    cb = _dev16(NF4)
    # the second call is smaller and has other data: stale scratch must not matter
    for seed, (M, N, K) in ((21, (96, 300, 4096)), (22, (40, 130, 1088))):
        _compare(seed, M, N, K, cb)
    assert q4.timeout_flags() == 0


def test_verify_sizes_and_exact_fit():
    """M = 20 (the M <= 24 kernel, which needs no scratch) and the largest
    input that fits: 2 * M * K equal to the array's size (M = 512, K = 8192),
    which would expose an access one past its end."""
    cb = _dev16(NF4)
    _compare(24, 20, 257, 4160, cb)
    assert 2 * 512 * 8192 == SCRATCH
    _compare(25, 512, 130, 8192, cb)
    assert q4.timeout_flags() == 0


def test_small_m_and_size_limit():
    cb = _dev16(NF4)
    codes, scales, x = _case(23, 8, 64, 512)          # M <= 16: no scratch used
    c, s, xd = torch.from_numpy(codes).cuda(), _dev16(scales), _dev16(x)
    y_ref = torch.empty((8, 64), device="cuda")
    y_new = torch.empty((8, 64), device="cuda")
    assert _call("q4_gemm", c, s, cb, xd, y_ref) == 0
    assert _call("q4_gemm_noalloc", c, s, cb, xd, y_new) == 0
    y_or, absacc = oracle_matmul_parallel(codes, scales, NF4, x)
    assert within_tolerance(y_new.cpu().numpy(), y_or, absacc)[0]
    assert within_tolerance(y_new.cpu().numpy(), y_ref.cpu().numpy(), absacc)[0]
    # one token past the limit is refused before anything runs
    K = 4096
    M = SCRATCH // (2 * K) + 1
    big_x = torch.zeros((M, K), dtype=torch.int16, device="cuda")
    codes2 = torch.zeros((64, K // 2), dtype=torch.uint8, device="cuda")
    scales2 = torch.zeros((64, K // GROUP), dtype=torch.int16, device="cuda")
    y = torch.empty((M, 64), device="cuda")
    assert _call("q4_gemm_noalloc", codes2, scales2, cb, big_x, y) == 6   # Q4_ERR_TOO_LARGE
    assert q4.timeout_flags() == 0
