#!/usr/bin/env python
"""Benchmark of the fused 4-bit codebook GEMV / GEMM on B200.

A step is one Llama-2-7B decoder layer's four linears at M = 1 through
q4_gemv (qkv 4096->12288, o 4096->4096, gate_up 4096->22016, down
11008->4096), weights quantized from seeded N(0, 0.02) by q4_pack.  Eight
distinct copies of the layer's packed weights (862 MB, several times the
126 MB L2) rotate from step to step, so every step streams its weights from
HBM.  The timed region replays CUDA graphs of these launches.

The JSON line reports:
  value         algorithmic GB/s = (code + scale + x + y + codebook bytes) per
                step / device time per step, summed over ranks
  roofline      the gate_up launch (largest share of the step), its algorithmic
                bytes / its mean CUDA-event duration, against the measured HBM peak
  e2e           the same metric through the Python API per step, with x copied
                from pinned host memory and y read back every step (the step's
                calls replayed from a CUDA graph)
  cpu_baseline  the oracle (single-threaded C) on the same layer, on the host
  gemm_prefill  q4_gemm at M = 256 on the Llama-2-70B linears: TFLOP/s

``--impl reference`` times the oracle instead (the reference arm).
Multi-GPU (torchrun): independent replicas, one per rank (weak scaling); the
timed region is bracketed by barriers and the max over ranks is reported.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

L2_BYTES = 126 * 1024 * 1024
COPIES = 8
GROUP = 64


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            d = json.load(fh)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


# DRAM bytes (read + write) of one q4_gemv launch on the gate_up linear
# (4096 -> 22016) from an ncu capture, with the SHA-1 of the kernel source it
# was taken on; when the source changes the figure no longer applies and the
# bench reports null.
GEMV_TRAFFIC = {"bytes": 47952896,
                "source_sha1": "96e7038247d1cef1a06a1c422a6ee1555db83a0f",
                "capture": "ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum,gpu__time_duration.sum "
                           "--clock-control none -k regex:gemv_m1 -s 2 -c 1 python -m "
                           "weight_only_bit_gemv_b200.profile_case --workload llama2_7b_layer "
                           "--linear gate_up --M 1 --iters 5 --copies 2"}


def gemv_traffic():
    import hashlib
    path = os.path.join(ROOT, "weight_only_bit_gemv_b200", "csrc", "q4_gemv_m1.cu")
    try:
        sha = hashlib.sha1(open(path, "rb").read()).hexdigest()
    except OSError:
        return None
    return GEMV_TRAFFIC["bytes"] if sha == GEMV_TRAFFIC["source_sha1"] else None


def algo_bytes(M, N, K):
    """Algorithmic bytes of one q4 matmul: codes + scales + x + y + codebook."""
    return N * K // 2 + N * (K // GROUP) * 2 + M * K * 2 + M * N * 4 + 32


class Clocks:
    """Samples nvidia-smi during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        import tempfile
        self.path = tempfile.mktemp(suffix=".csv")
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


def setup_dist():
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def barrier(world):
    """Every rank reaches this point, and this rank's GPU work is done."""
    import torch
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    if torch.cuda.is_available():
        torch.cuda.synchronize()


def max_over_ranks(v, world):
    """The largest of the ranks' values (device time: the slowest rank sets the
    step).  The tensor lives where the process group's backend works: on the
    GPU for NCCL, on the host for gloo."""
    import torch
    if world == 1:
        return v
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(units_per_rank, ms_per_step, world):
    """Whole-job throughput of independent replicas (weak scaling): every rank
    processes ``units_per_rank`` per step, and the step takes the slowest
    rank's time."""
    return world * units_per_rank / (ms_per_step * 1e-3)


# ---------------------------------------------------------------------------
# the layer on the GPU
# ---------------------------------------------------------------------------

def pcts(ms_list):
    """[p10, median, p90] of a list of durations in ms, in µs."""
    med = statistics.median(ms_list)
    if len(ms_list) < 2:
        return [round(med * 1e3, 3)] * 3
    q = statistics.quantiles(ms_list, n=10, method="inclusive")
    return [round(q[0] * 1e3, 3), round(med * 1e3, 3), round(q[8] * 1e3, 3)]


def build_layer(dev, cb):
    import torch
    import weight_only_bit_gemv_b200 as q4
    wl = synth.WORKLOADS["llama2_7b_layer"]
    lins = []
    for lin in wl.linears:
        seed = synth.seed_for(wl.index, 0, lin.name)
        w = synth.weights_device(seed, lin.N, lin.K, wl.w_std, dev)
        codes, scales = q4.q4_pack(w, cb)
        del w
        copies = [(codes, scales)] + [(codes.clone(), scales.clone()) for _ in range(COPIES - 1)]
        x = synth.activations_device(synth.x_seed(seed), 1, lin.K, dev)
        y = torch.empty((1, lin.N), dtype=torch.float32, device=dev)
        lins.append(dict(lin=lin, copies=copies, x=x, y=y, seed=seed))
    torch.cuda.synchronize()
    return lins


def capture_graphs(lins, cb, stream, with_events):
    """One CUDA graph per weight copy: the step's four launches, optionally
    with an event recorded after each launch."""
    import torch
    import weight_only_bit_gemv_b200 as q4
    graphs, events = [], []
    for c in range(COPIES):
        g = torch.cuda.CUDAGraph()
        evs = ([torch.cuda.Event(enable_timing=True, external=True) for _ in range(len(lins) + 1)]
               if with_events else [])
        with torch.cuda.graph(g, stream=stream):
            if with_events:
                evs[0].record()
            for i, L in enumerate(lins):
                codes, scales = L["copies"][c]
                q4.q4_gemv(codes, scales, cb, L["x"], L["y"])
                if with_events:
                    evs[i + 1].record()
        graphs.append(g)
        events.append(evs)
    return graphs, events


def run_ours(args, world, rank, local):
    import torch
    import weight_only_bit_gemv_b200 as q4
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    q4.load()
    hbm_peak, tc_peak, peak_src = peaks()
    cb = torch.from_numpy(synth.codebook().view(np.int16)).to(dev)
    lins = build_layer(dev, cb)
    bytes_step = sum(algo_bytes(1, L["lin"].N, L["lin"].K) for L in lins)
    stream = torch.cuda.Stream(device=dev)

    # warm-up outside capture (sets kernel attributes), then capture
    with torch.cuda.stream(stream):
        for _ in range(2):
            for L in lins:
                q4.q4_gemv(L["copies"][0][0], L["copies"][0][1], cb, L["x"], L["y"])
    stream.synchronize()
    graphs, _ = capture_graphs(lins, cb, stream, with_events=False)
    egraphs, eevents = capture_graphs(lins, cb, stream, with_events=True)
    # One graph of COPIES consecutive steps (one per weight copy): a replay
    # submits 4 * COPIES launches, so host submission never paces the GPU.
    g_multi = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_multi, stream=stream):
        for c in range(COPIES):
            for L in lins:
                q4.q4_gemv(L["copies"][c][0], L["copies"][c][1], cb, L["x"], L["y"])

    K, W = args.steps, args.warmup
    with torch.cuda.stream(stream):
        for i in range(W):
            graphs[i % COPIES].replay()
        g_multi.replay()
    stream.synchronize()

    # ---- timed region: exactly K steps -------------------------------------
    clocks = Clocks(local)
    clocks.start()
    time.sleep(0.3)
    barrier(world)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        t0.record()
        for i in range(K // COPIES):
            g_multi.replay()
        for i in range(K % COPIES):
            graphs[i].replay()
        t1.record()
    t1.synchronize()
    barrier(world)
    clk = clocks.stop()
    ms_total = max_over_ranks(t0.elapsed_time(t1), world)
    ms_step = ms_total / K

    # ---- per-launch durations (graphs with an event after each launch) -------
    per = [[] for _ in lins]
    reps = max(COPIES, min(K, 400))
    with torch.cuda.stream(stream):
        for i in range(reps):
            egraphs[i % COPIES].replay()
            if i % COPIES == COPIES - 1:
                stream.synchronize()
                for c in range(COPIES):
                    evs = eevents[c]
                    for j in range(len(lins)):
                        per[j].append(evs[j].elapsed_time(evs[j + 1]))
    stream.synchronize()
    per_ms = [statistics.mean(p) for p in per]
    dom = max(range(len(lins)), key=lambda j: algo_bytes(1, lins[j]["lin"].N, lins[j]["lin"].K))
    dom_bytes = algo_bytes(1, lins[dom]["lin"].N, lins[dom]["lin"].K)
    # Each linear timed on its own: one graph of COPIES back-to-back launches
    # over the rotating weight copies, events around the graph (an event
    # between launches would also time the launch gap it creates).  The
    # dominant one is the roofline kernel.
    def alone_ms(L):
        g_one = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_one, stream=stream):
            for c in range(COPIES):
                q4.q4_gemv(L["copies"][c][0], L["copies"][c][1], cb, L["x"], L["y"])
        reps_one = max(4, min(K, 200))
        d0 = torch.cuda.Event(enable_timing=True)
        d1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            for _ in range(3):
                g_one.replay()
            d0.record()
            for _ in range(reps_one):
                g_one.replay()
            d1.record()
        d1.synchronize()
        return d0.elapsed_time(d1) / (reps_one * COPIES)

    alone = [alone_ms(L) for L in lins]
    dom_ms = alone[dom]
    dom_gbs = dom_bytes / (dom_ms * 1e-3) / 1e9

    # ---- end to end through the Python API with host buffers -----------------
    # The step's inputs (x of the four linears) sit in one pinned host buffer
    # and its results (the four y) in one device buffer: every step copies x
    # host -> device, runs the four q4_gemv calls and copies y device -> host.
    # Each step is replayed from a CUDA graph captured over those API calls
    # (one graph per weight copy).
    xs_len = [L["lin"].K for L in lins]
    ys_len = [L["lin"].N for L in lins]
    xh_all = torch.empty(sum(xs_len), dtype=torch.bfloat16).pin_memory()
    yh_all = torch.empty(sum(ys_len), dtype=torch.float32).pin_memory()
    xd_all = torch.empty(sum(xs_len), dtype=torch.bfloat16, device=dev)
    yd_all = torch.empty(sum(ys_len), dtype=torch.float32, device=dev)
    xh_all.copy_(torch.cat([L["x"].reshape(-1).cpu() for L in lins]))
    xd_views = [v.view(1, -1) for v in torch.split(xd_all, xs_len)]
    yd_views = [v.view(1, -1) for v in torch.split(yd_all, ys_len)]
    h2d = xh_all.numel() * 2
    d2h = yh_all.numel() * 4
    e2e_steps = min(K, 2000)

    def e2e_step(c):
        xd_all.copy_(xh_all, non_blocking=True)
        for j, L in enumerate(lins):
            q4.q4_gemv(L["copies"][c][0], L["copies"][c][1], cb, xd_views[j], yd_views[j])
        yh_all.copy_(yd_all, non_blocking=True)

    with torch.cuda.stream(stream):
        for c in range(COPIES):
            e2e_step(c)  # eager once per copy (first-call set-up outside the graph)
    stream.synchronize()
    g_e2e = []
    for c in range(COPIES):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            e2e_step(c)
        g_e2e.append(g)
    with torch.cuda.stream(stream):
        for i in range(max(W, 3) * COPIES):
            g_e2e[i % COPIES].replay()
    stream.synchronize()
    barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record()
        for i in range(e2e_steps):
            g_e2e[i % COPIES].replay()
        e1.record()
    e1.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world) / e2e_steps
    # the last step's y arrived on the host: it must equal the device-timed y
    e2e_match = bool(torch.equal(yh_all, torch.cat([L["y"].reshape(-1).cpu() for L in lins])))
    del g_e2e

    # ---- prefill q4_gemm, M = 256, Llama-2-70B linears --------------------------
    gemm = None
    if not args.no_gemm:
        gemm = bench_prefill(dev, cb, stream, tc_peak, hbm_peak)

    # ---- other workloads: a full 8B decode step, small-M verify batches --------
    step8b = None if args.no_step else bench_decode_step(dev, cb, stream, hbm_peak)
    smallm = None if args.no_smallm else bench_small_m(dev, cb, stream, hbm_peak)
    embed = None if args.no_smallm else bench_embed_rows(dev, cb, stream, hbm_peak)
    ring = None if args.no_smallm else bench_ring(dev, cb, stream, lins)
    two_bit = None if args.no_smallm else bench_gemv2(dev, stream, hbm_peak)
    bf16_base = None
    if not args.no_gemm:
        try:
            bf16_base = bench_bf16_baseline(dev, cb, stream, lins, hbm_peak, tc_peak, ms_step, gemm)
        except Exception as exc:  # a baseline must not cost the bench line
            bf16_base = {"error": f"{type(exc).__name__}: {exc}"[:300]}

    # ---- CPU baseline: the oracle on the host --------------------------------
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_baseline(lins, cb, args.cpu_seconds)
        cpu["coverage"] = cpu_coverage()

    # per-linear launch time, each linear back to back on its own, as a fixed
    # cost plus bytes over a streaming rate (least squares over the four)
    xb = np.array([algo_bytes(1, L["lin"].N, L["lin"].K) for L in lins], dtype=np.float64)
    tb = np.array([a * 1e3 for a in alone], dtype=np.float64)  # us
    slope, fixed = np.polyfit(xb, tb, 1)
    fit = f"{fixed:.2f} us fixed + bytes at {1e-3 / slope:.0f} GB/s" if slope > 0 else "n/a"

    value = aggregate(bytes_step, ms_step, world) / 1e9
    line = {
        "metric": "q4_gemv HBM GB/s (% of B200 peak) at M=1; q4_gemm TFLOP/s at M>=16",
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": K,
        "warmup": W,
        "ms_per_step": round(ms_step, 6),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "u4 codes x bf16 -> f16 mma, f32 accumulate",
        "data": "synthetic (seeded N(0,0.02) weights quantized by q4_pack; x ~ N(0,1) bf16)",
        "config": {
            "workload": "llama2_7b_layer: qkv 4096->12288, o 4096->4096, gate_up 4096->22016, "
                        "down 11008->4096; M=1; one q4_gemv per linear",
            "bytes_per_step": bytes_step,
            "l2": f"inputs larger than L2: {COPIES} rotating copies of the packed layer "
                  f"({COPIES * sum(L['copies'][0][0].numel() + 2 * L['copies'][0][1].numel() for L in lins) / 1e6:.0f} MB)",
            "launch": "CUDA graphs of the step's four launches",
            "hbm_frac_of_" + peak_src: round(value / world / hbm_peak, 4),
            "per_linear_us_in_step_events": {L["lin"].name: round(per_ms[j] * 1e3, 3) for j, L in enumerate(lins)},
            "per_linear_us_p10_p50_p90": {L["lin"].name: pcts(per[j]) for j, L in enumerate(lins)},
            "decode_tok_s_equiv_32_layers": round(1e3 / (ms_step * 32), 1),
            "per_linear_us_back_to_back": "; ".join(
                f"{L['lin'].name} {alone[j] * 1e3:.2f}" for j, L in enumerate(lins)),
            "per_linear_us_in_step_p10_p50_p90": "; ".join(
                f"{L['lin'].name} " + "/".join(f"{v:.2f}" for v in pcts(per[j])) for j, L in enumerate(lins)),
            "per_linear_fit": fit,
        },
        "roofline": {
            "kernel": f"q4_gemv gate_up {lins[dom]['lin'].K}->{lins[dom]['lin'].N}",
            "bound": "hbm",
            "achieved": round(dom_gbs, 2),
            "peak": hbm_peak,
            "peak_source": peak_src,
            "unit": "GB/s",
            "frac": round(dom_gbs / hbm_peak, 4),
            "traffic": gemv_traffic(),
            "algorithmic_bytes": dom_bytes,
            "us_per_launch": round(dom_ms * 1e3, 3),
            "timing": f"{COPIES} back-to-back launches in one CUDA graph over rotating weight copies",
        },
        "e2e": {
            "value": round(aggregate(bytes_step, e2e_ms, world) / 1e9, 2),
            "unit": "GB/s",
            "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h,
            "ms_per_step": round(e2e_ms, 6),
            "y_matches_device_path": e2e_match,
            "api": "weight_only_bit_gemv_b200.q4_gemv per linear; per step one pinned host-to-device "
                   "copy of the four x and one device-to-host copy of the four y, the step's API "
                   "calls captured in a CUDA graph",
        },
        "gpu_launches": 4 * K,
        "clocks": clk,
    }
    cfg = line["config"]
    if gemm is not None:
        sw = gemm["sweep"]
        cfg["prefill_llama2_70b_M256_tflops"] = gemm["tflops"]
        cfg["prefill_llama2_70b_M256_frac_of_bf16_peak"] = gemm["frac_of_bf16_peak"]
        cfg["prefill_llama2_70b_tflops_M32_128_256_512"] = " / ".join(
            f"{sw[k]['tflops']:.1f}" for k in sorted(sw, key=lambda k: int(k[2:])))
        cfg["prefill_llama2_70b_frac_of_roofline_M32_128_256_512"] = " / ".join(
            f"{sw[k]['frac_of_roofline']:.3f}" for k in sorted(sw, key=lambda k: int(k[2:])))
    if step8b is not None:
        cfg["decode_step_llama31_8b_tok_s"] = step8b["tok_s"]
        cfg["decode_step_llama31_8b_hbm_frac"] = step8b["hbm_frac_of_measured"]
    if smallm is not None:
        cfg["verify_llama31_8b_gbs_M2_4_8_16"] = " / ".join(
            f"{smallm[k]['gbs']:.0f}" for k in ("M=2", "M=4", "M=8", "M=16") if k in smallm)
        cfg["verify_llama31_8b_hbm_frac_M2_4_8_16"] = " / ".join(
            f"{smallm[k]['hbm_frac_of_measured']:.3f}" for k in ("M=2", "M=4", "M=8", "M=16") if k in smallm)
    if two_bit is not None and "gbs" in two_bit:
        cfg["two_bit_llama2_70b_layer_gbs"] = two_bit["gbs"]
        cfg["two_bit_llama2_70b_layer_hbm_frac"] = two_bit["hbm_frac_of_measured"]
    if embed is not None:
        cfg["embed_rows_gbs"] = embed["gbs"]
    if ring is not None:
        cfg["copy_ring_frac_of_h2d_copy"] = ring["frac_of_h2d_copy"]
    if bf16_base is not None and "decode_llama2_7b_layer_m1" in bf16_base:
        cfg["torch_bf16_decode_gbs"] = bf16_base["decode_llama2_7b_layer_m1"]["gbs_at_2B_per_weight"]
        cfg["torch_bf16_prefill_M256_tflops"] = bf16_base["prefill_llama2_70b_layer_m256"]["tflops"]
    if gemm is not None:
        line["gemm_prefill"] = gemm
    if step8b is not None:
        line["decode_step_llama31_8b"] = step8b
    if smallm is not None:
        line["small_m_verify"] = smallm
    if embed is not None:
        line["embed_rows"] = embed
    if ring is not None:
        line["copy_ring"] = ring
    if two_bit is not None:
        line["two_bit_gemv_llama2_70b"] = two_bit
    if bf16_base is not None:
        line["torch_bf16_baseline"] = bf16_base
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if rank == 0:
        print(json.dumps(line), flush=True)


def bench_prefill(dev, cb, stream, tc_peak, hbm_peak, Ms=(32, 128, 256, 512), main_M=256):
    """q4_gemm on the Llama-2-70B linears at each M of ``Ms``: each linear is
    packed once and timed from a CUDA graph of 4 back-to-back calls."""
    import torch
    import weight_only_bit_gemv_b200 as q4
    wl = synth.WORKLOADS["llama2_70b_prefill"]
    per_m = {M: {"flop": 0.0, "bytes": 0.0, "ms": 0.0, "roof_ms": 0.0, "lin": {}} for M in Ms}
    for lin in wl.linears:
        seed = synth.seed_for(wl.index, 0, lin.name)
        w = synth.weights_device(seed, lin.N, lin.K, wl.w_std, dev)
        codes, scales = q4.q4_pack(w, cb)
        del w
        for M in Ms:
            x = synth.activations_device(synth.x_seed(seed) + M, M, lin.K, dev)
            y = torch.empty((M, lin.N), dtype=torch.float32, device=dev)
            with torch.cuda.stream(stream):
                for _ in range(3):
                    q4.q4_gemm(codes, scales, cb, x, y)
                stream.synchronize()
                # a CUDA graph of `per` calls: the device time of the calls,
                # without the host's per-call work (tensor-map encoding, checks)
                per = 4
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream):
                    for _ in range(per):
                        q4.q4_gemm(codes, scales, cb, x, y)
                g.replay()
                stream.synchronize()
                reps = 5
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record()
                for _ in range(reps):
                    g.replay()
                e1.record()
            e1.synchronize()
            ms = e0.elapsed_time(e1) / (reps * per)
            del g
            flop = 2.0 * M * lin.N * lin.K
            nbytes = algo_bytes(M, lin.N, lin.K)
            r = per_m[M]
            r["lin"][lin.name] = {"us": round(ms * 1e3, 2), "tflops": round(flop / (ms * 1e-3) / 1e12, 2)}
            r["flop"] += flop
            r["bytes"] += nbytes
            r["ms"] += ms
            # roofline time of this linear: the slower of its flops at the
            # tensor peak and its bytes at the HBM peak
            r["roof_ms"] += max(flop / (tc_peak * 1e12), nbytes / (hbm_peak * 1e9)) * 1e3
            del x, y
        del codes, scales
        torch.cuda.empty_cache()
    sweep = {}
    for M in Ms:
        r = per_m[M]
        tf = r["flop"] / (r["ms"] * 1e-3) / 1e12
        gbs = r["bytes"] / (r["ms"] * 1e-3) / 1e9
        hbm_bound = r["bytes"] / (hbm_peak * 1e9) > r["flop"] / (tc_peak * 1e12)
        sweep[f"M={M}"] = {"tflops": round(tf, 2), "gbs": round(gbs, 1),
                           "bound": "hbm" if hbm_bound else "tensor",
                           "frac_of_roofline": round(r["roof_ms"] / r["ms"], 4),
                           "us": round(r["ms"] * 1e3, 2)}
    m = per_m[main_M]
    tf = m["flop"] / (m["ms"] * 1e-3) / 1e12
    return {"workload": f"llama2_70b_prefill layer (4 linears), M={main_M}", "tflops": round(tf, 2),
            "frac_of_bf16_peak": round(tf / tc_peak, 4), "per_linear": m["lin"],
            "sweep": sweep,
            "timing": "per linear and M: CUDA graph of 4 back-to-back q4_gemm calls (y zeroing when "
                      "K is split, and the tensor-core GEMM, which converts x inside), replayed 5 times",
            "note": "no L2 flush: each linear is 37-253 MB of packed weights, read once per launch; "
                    "frac_of_roofline = sum over the linears of max(flop / tensor peak, bytes / HBM "
                    "peak) over the measured time"}


def bench_decode_step(dev, cb, stream, hbm_peak, reps=20):
    """Llama-3.1-8B decode step at M = 1: 32 layers x (qkv, o, gate_up, down) +
    lm_head, one q4_gemv per linear (129 launches) in one CUDA graph, every
    layer with its own seeded weights (3.99 GB packed, resident in HBM)."""
    import torch
    import weight_only_bit_gemv_b200 as q4
    wl = synth.WORKLOADS["llama31_8b_step"]
    layers = [lin for lin in wl.linears if lin.name != "lm_head"]
    head = [lin for lin in wl.linears if lin.name == "lm_head"][0]
    order = [(layer, lin) for layer in range(32) for lin in layers] + [(0, head)]
    packs, xs, ys = [], {}, []
    for layer, lin in order:
        seed = synth.seed_for(wl.index, layer, lin.name)
        w = synth.weights_device(seed, lin.N, lin.K, wl.w_std, dev)
        codes, scales = q4.q4_pack(w, cb)
        del w
        packs.append((codes, scales, lin))
        if lin.K not in xs:
            xs[lin.K] = synth.activations_device(synth.x_seed(seed), 1, lin.K, dev)
        ys.append(torch.empty((1, lin.N), dtype=torch.float32, device=dev))
    torch.cuda.synchronize()
    nbytes = sum(algo_bytes(1, lin.N, lin.K) for _, _, lin in packs)
    # the library records the 129 launches as one CUDA graph (q4_step_create)
    step = q4.Step([(codes, scales, cb, xs[lin.K], y) for (codes, scales, lin), y in zip(packs, ys)])
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        for _ in range(3):
            step.launch(stream)
        e0.record()
        for _ in range(reps):
            step.launch(stream)
        e1.record()
    e1.synchronize()
    ms = e0.elapsed_time(e1) / reps
    step.close()
    del packs, xs, ys
    torch.cuda.empty_cache()
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"workload": "llama31_8b_step: 32 x (qkv 4096->6144, o 4096->4096, gate_up 4096->28672, "
                        "down 14336->4096) + lm_head 4096->128256, M=1, 129 q4_gemv launches recorded "
                        "by q4_step_create as one CUDA graph, replayed by q4_step_launch",
            "bytes_per_step": nbytes, "ms_per_step": round(ms, 4), "tok_s": round(1e3 / ms, 1),
            "gbs": round(gbs, 1), "hbm_frac_of_measured": round(gbs / hbm_peak, 4)}


def bench_small_m(dev, cb, stream, hbm_peak, Ms=(2, 4, 8, 16), reps=20):
    """Verify batches on the Llama-3.1-8B linears + lm_head (396 MB packed, more
    than L2, so each step streams its weights from HBM): q4_gemm of the five
    linears at M tokens in one CUDA graph."""
    import torch
    import weight_only_bit_gemv_b200 as q4
    wl = synth.WORKLOADS["small_m_verify"]
    packs = []
    for lin in wl.linears:
        seed = synth.seed_for(wl.index, 0, lin.name)
        w = synth.weights_device(seed, lin.N, lin.K, wl.w_std, dev)
        codes, scales = q4.q4_pack(w, cb)
        del w
        packs.append((codes, scales, lin, seed))
    out = {}
    for M in Ms:
        xs = [synth.activations_device(synth.x_seed(seed) + M, M, lin.K, dev) for _, _, lin, seed in packs]
        ys = [torch.empty((M, lin.N), dtype=torch.float32, device=dev) for _, _, lin, _ in packs]
        with torch.cuda.stream(stream):
            for (codes, scales, lin, _), x, y in zip(packs, xs, ys):
                q4.q4_gemm(codes, scales, cb, x, y)
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for (codes, scales, lin, _), x, y in zip(packs, xs, ys):
                q4.q4_gemm(codes, scales, cb, x, y)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            for _ in range(3):
                g.replay()
            e0.record()
            for _ in range(reps):
                g.replay()
            e1.record()
        e1.synchronize()
        ms = e0.elapsed_time(e1) / reps
        nbytes = sum(algo_bytes(M, lin.N, lin.K) for _, _, lin, _ in packs)
        flops = sum(2.0 * M * lin.N * lin.K for _, _, lin, _ in packs)
        out[f"M={M}"] = {"us": round(ms * 1e3, 2), "gbs": round(nbytes / (ms * 1e-3) / 1e9, 1),
                         "hbm_frac_of_measured": round(nbytes / (ms * 1e-3) / 1e9 / hbm_peak, 4),
                         "tflops": round(flops / (ms * 1e-3) / 1e12, 2)}
        del g, xs, ys
    del packs
    torch.cuda.empty_cache()
    return {"workload": "small_m_verify: Llama-3.1-8B qkv, o, gate_up, down + lm_head, q4_gemm per "
                        "linear, 5 launches in one CUDA graph", **out}


def bench_embed_rows(dev, cb, stream, hbm_peak, n_ids=4096, reps=20):
    """q4_embed_rows on the Llama-3.1-8B embedding table (128256 x 4096,
    packed: 279 MB, more than L2): a prefill chunk of ``n_ids`` seeded token
    ids, four calls per CUDA graph."""
    import torch
    import weight_only_bit_gemv_b200 as q4
    N, K = 128256, 4096
    w = synth.weights_device(synth.seed_for(9, 0, "embed"), N, K, 0.02, dev)
    codes, scales = q4.q4_pack(w, cb)
    del w
    g_ids = torch.Generator(device="cpu").manual_seed(12345)
    ids = torch.randint(0, N, (4, n_ids), generator=g_ids, dtype=torch.int32).to(dev)
    outs = [torch.empty((n_ids, K), dtype=torch.float32, device=dev) for _ in range(4)]
    with torch.cuda.stream(stream):
        for j in range(4):
            q4.q4_embed_rows(codes, scales, cb, ids[j], outs[j])
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for j in range(4):
            q4.q4_embed_rows(codes, scales, cb, ids[j], outs[j])
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        for _ in range(3):
            g.replay()
        e0.record()
        for _ in range(reps):
            g.replay()
        e1.record()
    e1.synchronize()
    ms = e0.elapsed_time(e1) / (reps * 4)
    # algorithmic bytes: each id's code row and scales read, its fp32 row
    # written, the id itself and the codebook
    nbytes = n_ids * (K // 2 + (K // GROUP) * 2 + 4 * K + 4) + 32
    gbs = nbytes / (ms * 1e-3) / 1e9
    del g, codes, scales, outs
    torch.cuda.empty_cache()
    return {"workload": f"llama31_8b embedding table {N}x{K}, {n_ids} seeded token ids per call",
            "us": round(ms * 1e3, 2), "gbs": round(gbs, 1),
            "hbm_frac_of_measured": round(gbs / hbm_peak, 4),
            "timing": "CUDA graph of 4 calls on different ids, replayed 20 times"}


def _graph_time_ms(fn, stream, per=4, reps=10):
    """Device time of one ``fn()`` call: a CUDA graph of ``per`` calls,
    replayed ``reps`` times after an eager warm-up."""
    import torch
    with torch.cuda.stream(stream):
        for _ in range(3):
            fn()
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for _ in range(per):
            fn()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        g.replay()
        e0.record()
        for _ in range(reps):
            g.replay()
        e1.record()
    e1.synchronize()
    del g
    return e0.elapsed_time(e1) / (reps * per)


def bench_bf16_baseline(dev, cb, stream, lins, hbm_peak, tc_peak, ours_ms_step, gemm):
    """The same shapes in plain torch: y = x @ W_bf16^T through cuBLAS, with
    W_bf16 = bf16(dequantized W), i.e. 2 B per weight.  Decode: the
    Llama-2-7B layer at M = 1 against the q4_gemv step; prefill: the
    Llama-2-70B layer at M = 256 against q4_gemm."""
    import torch
    import weight_only_bit_gemv_b200 as q4
    # decode, M = 1
    ws = [q4.q4_dequant(L["copies"][0][0], L["copies"][0][1], cb).to(torch.bfloat16) for L in lins]
    ys = [torch.empty((1, L["lin"].N), dtype=torch.bfloat16, device=dev) for L in lins]
    torch.cuda.synchronize()  # the weights were made on the default stream

    def step():
        for L, w, y in zip(lins, ws, ys):
            torch.matmul(L["x"], w.t(), out=y)

    ms = _graph_time_ms(step, stream, per=4, reps=20)
    nbytes = sum(2 * L["lin"].N * L["lin"].K + 2 * L["lin"].K + 2 * L["lin"].N for L in lins)
    gbs = nbytes / (ms * 1e-3) / 1e9
    out = {"decode_llama2_7b_layer_m1": {
        "us_per_step": round(ms * 1e3, 2), "gbs_at_2B_per_weight": round(gbs, 1),
        "hbm_frac_of_measured": round(gbs / hbm_peak, 4),
        "q4_gemv_speedup": round(ms / ours_ms_step, 3)}}
    del ws, ys
    torch.cuda.empty_cache()
    # prefill, M = 256
    M = 256
    wl = synth.WORKLOADS["llama2_70b_prefill"]
    tot_ms, tot_flop, per_lin = 0.0, 0.0, {}
    for lin in wl.linears:
        seed = synth.seed_for(wl.index, 0, lin.name)
        w = synth.weights_device(seed, lin.N, lin.K, wl.w_std, dev)
        codes, scales = q4.q4_pack(w, cb)
        del w
        wb = q4.q4_dequant(codes, scales, cb).to(torch.bfloat16)
        del codes, scales
        x = synth.activations_device(synth.x_seed(seed) + M, M, lin.K, dev)
        y = torch.empty((M, lin.N), dtype=torch.bfloat16, device=dev)
        torch.cuda.synchronize()
        lms = _graph_time_ms(lambda: torch.matmul(x, wb.t(), out=y), stream, per=4, reps=5)
        flop = 2.0 * M * lin.N * lin.K
        per_lin[lin.name] = {"us": round(lms * 1e3, 2), "tflops": round(flop / (lms * 1e-3) / 1e12, 2)}
        tot_ms += lms
        tot_flop += flop
        del wb, x, y
        torch.cuda.empty_cache()
    tf = tot_flop / (tot_ms * 1e-3) / 1e12
    pre = {"tflops": round(tf, 2), "frac_of_bf16_peak": round(tf / tc_peak, 4),
           "us_per_layer": round(tot_ms * 1e3, 2), "per_linear": per_lin}
    if gemm is not None:
        pre["q4_gemm_speedup"] = round(gemm["tflops"] / tf, 3)
    out["prefill_llama2_70b_layer_m256"] = pre
    out["timing"] = ("CUDA graphs of 4 calls (decode: 4 steps of the 4 linears), replayed 20 (decode) "
                     "or 5 (prefill) times; bf16 output; W_bf16 = bf16(q4_dequant(codes, scales))")
    return out


def bench_gemv2(dev, stream, hbm_peak, reps=20):
    """The two-bit variant: the Llama-2-70B decoder layer's four linears at
    M = 1 (q4_gemv2; uniform random 2-bit codes and U[0.005, 0.05] scales,
    241 MB per layer, more than L2), one CUDA graph of the four calls."""
    import torch
    import weight_only_bit_gemv_b200 as q4
    cb4 = torch.from_numpy(synth.codebook2().view(np.int16)).to(dev)
    lins = []
    for lin in synth.WORKLOADS["llama2_70b_prefill"].linears:
        g = torch.Generator(device=dev)
        g.manual_seed(synth.seed_for(5, 0, lin.name))
        codes = torch.randint(0, 256, (lin.N, lin.K // 4), generator=g, device=dev, dtype=torch.uint8)
        scales = (torch.rand((lin.N, lin.K // GROUP), generator=g, device=dev) * 0.045 + 0.005).half()
        x = synth.activations_device(synth.x_seed(synth.seed_for(5, 0, lin.name)), 1, lin.K, dev)
        y = torch.empty((1, lin.N), dtype=torch.float32, device=dev)
        lins.append((lin, codes, scales, x, y))
    torch.cuda.synchronize()  # inputs drawn on the default stream
    with torch.cuda.stream(stream):
        for lin, c, sc, x, y in lins:
            q4.q4_gemv2(c, sc, cb4, x, y)
    stream.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for lin, c, sc, x, y in lins:
            q4.q4_gemv2(c, sc, cb4, x, y)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        for _ in range(3):
            graph.replay()
        e0.record()
        for _ in range(reps):
            graph.replay()
        e1.record()
    e1.synchronize()
    ms = e0.elapsed_time(e1) / reps
    # algorithmic bytes: codes, scales, x and y of each linear, the codebook
    nbytes = sum(l.N * l.K // 4 + l.N * (l.K // GROUP) * 2 + 2 * l.K + 4 * l.N + 8 for l, *_ in lins)
    per = {}
    for lin, c, sc, x, y in lins:
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            t0.record()
            for _ in range(reps):
                q4.q4_gemv2(c, sc, cb4, x, y)
            t1.record()
        t1.synchronize()
        us = t0.elapsed_time(t1) * 1e3 / reps
        b = lin.N * lin.K // 4 + lin.N * (lin.K // GROUP) * 2 + 2 * lin.K + 4 * lin.N + 8
        per[lin.name] = {"N": lin.N, "K": lin.K, "us": round(us, 2),
                         "gbs": round(b / (us * 1e-6) / 1e9, 1)}
    gbs = nbytes / (ms * 1e-3) / 1e9
    del graph, lins
    torch.cuda.empty_cache()
    return {"workload": "llama2_70b decoder layer in 2 bits (4-entry codebook), M=1, "
                        "4 q4_gemv2 calls (qkv 8192->10240, o, gate_up 8192->57344, down)",
            "us_per_layer": round(ms * 1e3, 2), "gbs": round(gbs, 1),
            "hbm_frac_of_measured": round(gbs / hbm_peak, 4), "bytes_per_layer": nbytes,
            "per_linear_back_to_back": per,
            "timing": "CUDA graph of the 4 calls (each a y memset and one kernel), replayed 20 times; "
                      "per linear: 20 back-to-back calls"}


def bench_ring(dev, cb, stream, lins, steps=20):
    """CopyRing: the Llama-2-7B layer's four linears with their packed weights
    in pinned host memory, streamed through the ring's two device slots (one
    q4_ring_gemm per linear, M = 1).  The bound is the host link: the figure
    is set against a plain pinned host-to-device copy of the same bytes."""
    import torch
    import weight_only_bit_gemv_b200 as q4
    host = [(L["copies"][0][0].cpu().pin_memory(), L["copies"][0][1].cpu().pin_memory()) for L in lins]
    slot = max(q4.ring_slot_bytes(L["lin"].N, L["lin"].K) for L in lins)
    ring = q4.Ring(slot)
    try:
        with torch.cuda.stream(stream):
            for (ch, sh), L in zip(host, lins):
                ring.gemm(ch, sh, cb, L["x"], L["y"])
        stream.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record()
            for _ in range(steps):
                for (ch, sh), L in zip(host, lins):
                    ring.gemm(ch, sh, cb, L["x"], L["y"])
            e1.record()
        e1.synchronize()
        ms = e0.elapsed_time(e1) / steps
    finally:
        ring.close()
    wbytes = sum(ch.numel() + sh.numel() * 2 for ch, sh in host)
    # the host link alone: the same bytes as one pinned copy per matrix
    dst = torch.empty(max(ch.numel() for ch, _ in host), dtype=torch.uint8, device=dev)
    with torch.cuda.stream(stream):
        c0 = torch.cuda.Event(enable_timing=True)
        c1 = torch.cuda.Event(enable_timing=True)
        c0.record()
        for _ in range(5):
            for ch, sh in host:
                dst[:ch.numel()].copy_(ch.view(-1), non_blocking=True)
                dst[:sh.numel() * 2].view(torch.int16).copy_(sh.view(torch.int16).view(-1), non_blocking=True)
        c1.record()
    c1.synchronize()
    copy_ms = c0.elapsed_time(c1) / 5
    del dst, host
    gbs = wbytes / (ms * 1e-3) / 1e9
    h2d = wbytes / (copy_ms * 1e-3) / 1e9
    return {"workload": "llama2_7b_layer, M=1, packed weights in pinned host memory, two device slots",
            "us_per_step": round(ms * 1e3, 1), "gbs": round(gbs, 1), "h2d_copy_gbs": round(h2d, 1),
            "frac_of_h2d_copy": round(gbs / h2d, 4),
            "timing": f"{steps} steps of four q4_ring_gemm calls, eager; the copy alone timed the same way"}


def cpu_baseline(lins, cb, seconds):
    """The oracle, as it stands, single-threaded, on a bounded sample: the first
    rows of each linear of the same layer (same weights, copied to the host)."""
    import oracle
    cbn = synth.codebook()
    # estimate: the oracle's matmul at M=1 costs ~30 ns/weight on these hosts
    total_w = sum(L["lin"].N * L["lin"].K for L in lins)
    frac = min(1.0, seconds / (total_w * 30e-9))
    packs = []
    for L in lins:
        n = max(16, int(L["lin"].N * frac))
        seed = L["seed"]
        import torch
        w = synth.weights_device(seed, L["lin"].N, L["lin"].K, 0.02, L["x"].device)[:n].cpu().numpy()
        codes, scales = oracle.pack(w, cbn)
        x = L["x"].cpu().view(torch.int16).numpy().view(np.uint16)
        packs.append((codes, scales, x, n, L["lin"].K))
    t = time.perf_counter()
    byt = 0
    for codes, scales, x, n, K in packs:
        oracle.matmul(codes, scales, cbn, x, with_abs=False)
        byt += algo_bytes(1, n, K)
    dt = time.perf_counter() - t
    return {"value": round(byt / dt / 1e9, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"first {frac:.1%} of the rows of each of the 4 linears (same seeded "
                      f"weights, packed by the oracle), M=1, one pass; {dt:.1f} s single-threaded",
            "host_cpus": os.cpu_count()}


def cpu_coverage(seconds_per_case=1.5):
    """The oracle (as it stands, single-threaded) on a bounded row sample of
    each workload, with the time of the whole workload extrapolated from the
    sample (labelled as such).  Packed operands are seeded random codes and
    scales of the workload's shapes: the oracle's time does not depend on the
    values.  Samples are sized by a cost model of the oracle's loops (about
    27 ns per weight to rebuild a row, plus 2.7 ns per weight and token)."""
    import oracle
    cbn = synth.codebook()
    out = {}

    def run(label, seed, N, K, M, extra=None):
        n = int(min(N, max(16, seconds_per_case / (K * (27e-9 + 2.7e-9 * M)))))
        codes, scales = synth.tiny_codes_scales(seed, n, K)
        x = synth.activations(seed + 1, M, K)
        t = time.perf_counter()
        oracle.matmul(codes, scales, cbn, x, with_abs=False)
        dt = time.perf_counter() - t
        full_s = dt * N / n
        r = {"sample_rows": n, "rows": N, "M": M, "K": K, "sample_s": round(dt, 3),
             "ns_per_weight_token": round(dt / (n * K * M) * 1e9, 3),
             "full_ms_extrapolated": round(full_s * 1e3, 1),
             "gbs_extrapolated": round(algo_bytes(M, N, K) / full_s / 1e9, 4)}
        if extra:
            r.update(extra)
        out[label] = r
        return full_s

    lin = synth.WORKLOADS["tiny"].linears[0]
    run("tiny 256->128 M=1", 7, lin.N, lin.K, 1)
    wl = synth.WORKLOADS["llama31_8b_step"]
    layer_s = 0.0
    for l in wl.linears:
        s_l = run(f"llama31_8b {l.name} {l.K}->{l.N} M=1", synth.seed_for(wl.index, 0, l.name), l.N, l.K, 1)
        layer_s += 0.0 if l.name == "lm_head" else s_l
    head_s = out[f"llama31_8b lm_head 4096->128256 M=1"]["full_ms_extrapolated"] / 1e3
    out["llama31_8b step (32 layers + lm_head), extrapolated from one layer"] = {
        "ms_per_step": round((32 * layer_s + head_s) * 1e3, 1),
        "tok_s": round(1.0 / (32 * layer_s + head_s), 4)}
    run("small_m_verify o 4096->4096 M=16", 3001, 4096, 4096, 16)
    run("llama2_70b_prefill o 8192->8192 M=32", 4001, 8192, 8192, 32,
        {"tflops_extrapolated": None})
    r = out["llama2_70b_prefill o 8192->8192 M=32"]
    r["tflops_extrapolated"] = round(2 * 32 * 8192 * 8192 / (r["full_ms_extrapolated"] * 1e-3) / 1e12, 6)
    return out


def run_reference(args, world, rank):
    """The reference arm: the oracle, single-threaded, on the host cores."""
    if rank != 0:
        return
    import oracle
    cbn = synth.codebook()
    wl = synth.WORKLOADS["llama2_7b_layer"]
    steps = args.steps + args.warmup
    budget = args.ref_seconds
    total_w = sum(l.N * l.K for l in wl.linears)
    frac = min(1.0, budget / steps / (total_w * 30e-9))
    packs = []
    for lin in wl.linears:
        n = max(8, int(lin.N * frac))
        seed = synth.seed_for(wl.index, 0, lin.name)
        rng = np.random.Generator(np.random.PCG64(seed))
        w = (rng.standard_normal((n, lin.K), dtype=np.float32) * np.float32(wl.w_std))
        codes, scales = oracle.pack(w, cbn)
        x = synth.activations(synth.x_seed(seed), 1, lin.K)
        packs.append((codes, scales, x, n, lin.K))
    byt = sum(algo_bytes(1, n, K) for _, _, _, n, K in packs)

    def step():
        for codes, scales, x, n, K in packs:
            oracle.matmul(codes, scales, cbn, x, with_abs=False)

    for _ in range(args.warmup):
        step()
    t = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t) / args.steps
    v = byt / dt / 1e9
    sample = (f"first {frac:.2%} of the rows of each Llama-2-7B linear per step "
              f"({byt / 1e6:.2f} MB algorithmic), M=1, single-threaded C oracle")
    print(json.dumps({
        "impl": "reference",
        "metric": "q4_gemv HBM GB/s (% of B200 peak) at M=1; q4_gemm TFLOP/s at M>=16",
        "value": round(v, 4), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle)", "data": "synthetic",
        "config": {"workload": "llama2_7b_layer: qkv 4096->12288, o 4096->4096, gate_up "
                               "4096->22016, down 11008->4096; M=1 (row sample)"},
        "cpu_baseline": {"value": round(v, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(v, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-gemm", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-step", action="store_true", help="skip the Llama-3.1-8B decode step")
    ap.add_argument("--no-smallm", action="store_true", help="skip the small-M verify batches")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--ref-seconds", type=float, default=90.0)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, world, rank)
        return
    world, rank, local = setup_dist()
    try:
        run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
