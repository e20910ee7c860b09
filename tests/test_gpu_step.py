"""Recorded decode steps (q4_step_create / q4_step_launch) and the bounded-wait
self-test, on the GPU through the C ABI.

A step records its linears' launches once as a CUDA graph and replays them per
token ("deep-fold", "Method" table: a full greedy decode step as one CUDA graph).
Every replayed output is compared with the oracle.  Inputs come from ``synth``
(seeded); expected values come only from the oracle.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import synth
import weight_only_bit_gemv_b200 as q4
from helpers import GROUP, within_tolerance

pytestmark = pytest.mark.gpu

NF4 = synth.codebook()


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    q4.load()


def dev16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()


def check(y, codes, scales, x, rows=None, label=""):
    y_ref, a = oracle.matmul(codes, scales, NF4, x, rows=rows)
    ys = y if rows is None else y[:, rows]
    ok, worst = within_tolerance(ys, y_ref, a)
    assert ok, f"{label}: worst err/bound = {worst:.3g}"


def test_step_replays_every_path():
    """One step over all kernel families -- M = 1 (decode GEMV), 3 and 8
    (verify batches), 20 (the M <= 24 kernel) and 40 (tensor cores) -- and an
    empty linear; replayed twice with new activations written into the same x
    buffers in between, every output against the oracle each time."""
    shapes = [(1, 300, 4096), (3, 129, 1088), (8, 1000, 2048), (20, 257, 4160), (40, 300, 640),
              (0, 64, 256), (1, 33, 11008)]
    cb = dev16(NF4)
    lins, host = [], []
    for i, (M, N, K) in enumerate(shapes):
        codes, scales = synth.tiny_codes_scales(700 + i, N, K)
        x = torch.zeros((M, K), dtype=torch.int16, device="cuda")
        y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        c, s = torch.from_numpy(codes).cuda(), dev16(scales)
        lins.append((c, s, cb, x, y))
        host.append((codes, scales))
    step = q4.Step(lins)
    try:
        for rep in range(2):
            xs = []
            for i, (M, N, K) in enumerate(shapes):
                xh = synth.activations(7100 + 10 * i + rep, M, K)
                lins[i][3].copy_(dev16(xh))
                xs.append(xh)
            step.launch()
            torch.cuda.synchronize()
            for i, (M, N, K) in enumerate(shapes):
                if M == 0:
                    continue
                codes, scales = host[i]
                check(lins[i][4].cpu().numpy(), codes, scales, xs[i], label=f"rep {rep} M={M} N={N} K={K}")
    finally:
        step.close()
    assert q4.timeout_flags() == 0


def test_llama31_8b_step_graph():
    """The Llama-3.1-8B decode step as one recorded graph: 32 layers x (qkv,
    o, gate_up, down) + lm_head, 129 launches at M = 1, each layer's packed
    weights drawn from its own seed (codes uniform over the 16 entries,
    scales U[0.005, 0.05]: the packed operands a group-64 quantizer of N(0,
    0.02) weights produces, without quantizing 4 GB on the host).  After a
    replay, every one of the 129 outputs is compared with the oracle on 64
    seeded rows plus its first and last row; a second replay with new x
    must follow the new x."""
    wl = synth.WORKLOADS["llama31_8b_step"]
    cb = dev16(NF4)
    layer_lins = [l for l in wl.linears if l.name != "lm_head"]
    head = [l for l in wl.linears if l.name == "lm_head"][0]
    plan = [(layer, l) for layer in range(wl.layers) for l in layer_lins] + [(0, head)]
    lins, meta = [], []
    for layer, l in plan:
        seed = synth.seed_for(wl.index, layer, l.name)
        codes, scales = synth.tiny_codes_scales(seed, l.N, l.K)
        x = torch.zeros((1, l.K), dtype=torch.int16, device="cuda")
        y = torch.full((1, l.N), float("nan"), dtype=torch.float32, device="cuda")
        lins.append((torch.from_numpy(codes).cuda(), dev16(scales), cb, x, y))
        rows = np.unique(np.concatenate([[0, l.N - 1],
                                         np.random.default_rng(seed).choice(l.N, 64, replace=False)]))
        meta.append((seed, codes[rows], scales[rows], rows, l))
        del codes, scales
    assert len(lins) == 129
    step = q4.Step(lins)
    try:
        for rep in range(2):
            xs = []
            for (seed, _, _, _, l), lin in zip(meta, lins):
                xh = synth.activations(synth.x_seed(seed) + rep, 1, l.K)
                lin[3].copy_(dev16(xh))
                xs.append(xh)
            step.launch()
            torch.cuda.synchronize()
            for (seed, codes_r, scales_r, rows, l), lin, xh in zip(meta, lins, xs):
                y = lin[4].cpu().numpy()[:, rows]
                y_ref, a = oracle.matmul(codes_r, scales_r, NF4, xh)
                ok, worst = within_tolerance(y, y_ref, a)
                assert ok, f"rep {rep} {l.name} seed {seed}: worst err/bound = {worst:.3g}"
    finally:
        step.close()
    assert q4.timeout_flags() == 0


def test_step_rejects_a_bad_linear_before_recording():
    cb = dev16(NF4)
    c = torch.zeros((64, 128), dtype=torch.uint8, device="cuda")
    s = torch.zeros((64, 4), dtype=torch.int16, device="cuda")
    x = torch.zeros((1, 256), dtype=torch.int16, device="cuda")
    y = torch.zeros((1, 64), dtype=torch.float32, device="cuda")
    bad_y = torch.zeros((1, 65), dtype=torch.float32, device="cuda")[:, 1:]   # not 16-byte aligned
    arr = (q4.Q4Linear * 2)(q4.Q4Linear(c.data_ptr(), s.data_ptr(), cb.data_ptr(), x.data_ptr(),
                                        y.data_ptr(), 1, 64, 256),
                            q4.Q4Linear(c.data_ptr(), s.data_ptr(), cb.data_ptr(), x.data_ptr(),
                                        bad_y.data_ptr(), 1, 64, 256))
    import ctypes
    h = ctypes.c_void_p()
    assert q4.load().q4_step_create(arr, 2, ctypes.byref(h)) == 3     # Q4_ERR_ALIGN
    assert h.value is None


def test_bounded_wait_runs_out_and_reports():
    """Failure detection without a fault: a wait on an mbarrier nobody
    arrives at gives up after its limit, sets its bit in q4_timeout_flags,
    and reading the flags clears it; a wait whose arrival comes returns at
    once and sets nothing."""
    assert q4.timeout_flags() == 0
    waited = q4.wait_selftest(1000, arrive=False)
    assert 1000 <= waited < 200000, waited
    assert q4.timeout_flags() == 0x80
    assert q4.timeout_flags() == 0
    waited = q4.wait_selftest(1000, arrive=True)
    assert waited < 1000, waited
    assert q4.timeout_flags() == 0
    # the device is still usable: a matmul right after gives the oracle's y
    codes, scales = synth.tiny_codes_scales(5, 100, 512)
    x = synth.activations(6, 1, 512)
    y = q4.q4_gemv(torch.from_numpy(codes).cuda(), dev16(scales), dev16(NF4), dev16(x))
    torch.cuda.synchronize()
    check(y.cpu().numpy(), codes, scales, x, label="after self-test")
