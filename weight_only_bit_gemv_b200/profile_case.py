"""Runs one quantized linear repeatedly on cuda:0: the target of ncu captures.

    python -m weight_only_bit_gemv_b200.profile_case --workload llama2_7b_layer \
        --linear gate_up --M 1 --iters 6 [--copies 4] [--bits 2]

Weights are drawn on the GPU (seeded N(0, std)) and packed with q4_pack; each
iteration runs q4_gemm (q4_gemv when M = 1) on the next of ``--copies``
copies of the packed weights, then the run synchronizes and prints the mean
device time per launch.  ``--bits 2`` runs the two-bit variant instead
(q4_pack2 with the 4-entry codebook, then q4_gemv2; M must be 1).
"""
from __future__ import annotations

import argparse
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402
import weight_only_bit_gemv_b200 as q4  # noqa: E402


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="llama2_7b_layer")
    ap.add_argument("--linear", default="gate_up")
    ap.add_argument("--M", type=int, default=1)
    ap.add_argument("--iters", type=int, default=6)
    ap.add_argument("--copies", type=int, default=4)
    ap.add_argument("--bits", type=int, default=4, choices=(2, 4))
    a = ap.parse_args()
    if a.bits == 2 and a.M != 1:
        ap.error("--bits 2 runs the one-token GEMV only (M = 1)")
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    wl = synth.WORKLOADS[a.workload]
    lin = {l.name: l for l in wl.linears}[a.linear]
    book = synth.codebook2() if a.bits == 2 else synth.codebook()
    cb = torch.from_numpy(book.view(np.int16)).to(dev)
    seed = synth.seed_for(wl.index, 0, lin.name)
    w = synth.weights_device(seed, lin.N, lin.K, wl.w_std or 0.02, dev)
    codes, scales = (q4.q4_pack2 if a.bits == 2 else q4.q4_pack)(w, cb)
    del w
    copies = [(codes, scales)] + [(codes.clone(), scales.clone()) for _ in range(a.copies - 1)]
    x = synth.activations_device(synth.x_seed(seed), a.M, lin.K, dev)
    y = torch.empty((a.M, lin.N), dtype=torch.float32, device=dev)
    fn = q4.q4_gemv2 if a.bits == 2 else (q4.q4_gemv if a.M == 1 else q4.q4_gemm)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(a.iters):
        c, s = copies[i % a.copies]
        fn(c, s, cb, x, y)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / a.iters
    code_bytes = lin.N * lin.K * a.bits // 8
    nbytes = code_bytes + lin.N * lin.K // 32 + a.M * lin.K * 2 + a.M * lin.N * 4
    print(f"{a.workload}/{a.linear} M={a.M}: {ms * 1e3:.2f} us/launch, "
          f"{nbytes / ms / 1e6:.1f} GB/s algorithmic, {2 * a.M * lin.N * lin.K / ms / 1e9:.2f} TFLOP/s")


if __name__ == "__main__":
    main()
