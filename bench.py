#!/usr/bin/env python
"""KDA recurrence benchmark: one JSON line on rank 0.

Default workload (the step): one chunked prefill over the layer-shape batch
(B=1, H=96, T=8192, dk=dv=128, bf16 q/k/v/g/beta, fp32 state, chunk 64), all of
it in the library's kernels, inputs resident in HBM. The same line carries the
decode step (256 requests x 96 heads, fp32 states in place) as a second
measurement, the end-to-end figure through host buffers, the roofline of the
dominant kernel, the SM clocks seen while timing, and the fp64 oracle timed on
the host cores as the CPU baseline.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload prefill|varlen|b2|decode] [--path auto|simt|tc]

Multi-GPU (torchrun, one rank per GPU): (sequence, head) units are independent,
so every rank runs its own batch (weak scaling, no collective on the data path);
value = all ranks' tokens / the slowest rank's time.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "KDA prefill tokens/s (H=96,d=128) & % tensor peak; decode GB/s vs HBM"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
NOMINAL_HBM_GBS = 7700.0  # HGX B200 HBM3e, for context beside the measured / fallback copy bandwidth
WORKLOAD_ALIASES = {"prefill": "prefill_h96_T8192_d128_bf16", "varlen": "varlen_h96_8seq_d128_bf16",
                    "b2": "b2_h4_T2048_d128_bf16", "small": "small_f32_T256_d32",
                    "decode": "decode_n256_h96_d128", "long": "long_h8_T65536_d128_bf16"}


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--workload", default="prefill", choices=sorted(WORKLOAD_ALIASES))
    p.add_argument("--path", default="auto", choices=["auto", "simt", "tc", "tc_single", "tc_split", "tc_pipe"])
    p.add_argument("--snap-every", type=int, default=1024,
                   help="prefill leg saving the state every N tokens (0: skip)")
    p.add_argument("--draft-tokens", type=int, default=4,
                   help="draft tokens per request in the speculative decode leg (0: skip)")
    p.add_argument("--decode-steps", type=int, default=0,
                   help="decode steps timed (0: the decode workload's own count, 1000)")
    p.add_argument("--no-varlen", action="store_true",
                   help="skip the packed-sequence leg of the default run")
    p.add_argument("--tokens", type=int, default=0,
                   help="override T of the dense prefill workload (smaller only for profiling captures)")
    p.add_argument("--decode-requests", type=int, default=256,
                   help="requests in the decode batch (smaller only for profiling captures)")
    p.add_argument("--no-decode", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--e2e-piece", type=int, default=1024,
                   help="tokens per piece of kda_forward_host in the end-to-end leg (0: library default)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU-baseline sample time")
    return p.parse_args()


# ----------------------------------------------------------------- helpers

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return dict(FALLBACK_PEAKS, source="fallback")


def source_sha(relpath):
    with open(os.path.join(ROOT, relpath), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def traffic_for(kernel_src, workload_name):
    """DRAM bytes per launch from the committed ncu summary, or None if the
    summary is missing or was taken on a different version of the kernel."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        e = d[workload_name]
        if e.get("source_sha") != source_sha(kernel_src):
            return None
        return float(e["dram_bytes_per_launch"])
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi clock/throttle samples every 200 ms while timing."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.idx = str(device_index)
        self.proc = None
        self.out = None

    def __enter__(self):
        try:
            self.out = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if self.proc is None or self.out is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.out.flush()
        rows = []
        with open(self.out.name) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9 and parts[0] == self.idx:
                    rows.append(parts)
        os.unlink(self.out.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def prefill_algorithmic(w, elem):
    """Algorithmic bytes and flops of one prefill over workload w.

    bytes: q, k, g (dk each), v and o (dv each), beta, per token-head, in the
    storage dtype; plus the fp32 initial state read (when present) and the
    final state written, once per (sequence, head).
    flops per token-head (chunk C): 6 dk dv for the three state contractions
    (W S, (Gamma q) S, Kh^T U), C (3 dk + 2 dv) for the lower-triangular chunk
    products (A and P Grams, W, Ut, P U), C^2/3 for the triangular solve."""
    th = w.total_tokens * w.H
    units = w.num_seqs * w.H
    b = th * ((3 * w.dk + 2 * w.dv) * elem + elem) + units * w.dk * w.dv * 4 * (2 if w.s0_std > 0 else 1)
    C = w.chunk
    f = th * (6 * w.dk * w.dv + C * (3 * w.dk + 2 * w.dv) + C * C / 3.0)
    return float(b), float(f)


def decode_algorithmic(N, H, dk, dv, elem):
    per_head = 2 * dk * dv * 4 + (3 * dk + dv) * elem + elem + dv * elem
    return float(N * H * per_head), float(N * H * 7 * dk * dv)


# ----------------------------------------------------- multi-rank helpers

def rank_workload(w, rank: int):
    """Each rank runs its own batch of independent sequences (weak scaling):
    the same shapes and distributions, a rank-specific seed."""
    import dataclasses
    return dataclasses.replace(w, seed=w.seed + 7919 * rank)


def max_over_ranks(x: float, world: int, device) -> float:
    """The slowest rank's time: an all-reduce MAX (no-op for one rank)."""
    if world == 1:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(units_per_rank: float, steps: int, ms_total_max: float, world: int) -> float:
    """Whole-job throughput: all ranks' units over the slowest rank's time."""
    return world * units_per_rank * steps / (ms_total_max / 1e3)


# --------------------------------------------------------------- our arm

def run_ours(args, rank, world, device):
    import torch
    from linear_attention_recurrence_11_b200 import kda
    from linear_attention_recurrence_11_b200.inputs import WORKLOADS, workload_inputs
    import dataclasses
    wname = WORKLOAD_ALIASES[args.workload]
    w = WORKLOADS[wname]
    if args.tokens and not w.seqlens and not w.decode_steps:
        w = dataclasses.replace(w, T=args.tokens)
        wname = f"{wname}@T{args.tokens}"
    peaks = load_peaks()
    res = {}
    stream = torch.cuda.current_stream(device)

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    def max_ranks(x):
        return max_over_ranks(x, world, device)

    if w.decode_steps:
        return run_decode_main(args, rank, world, device, w, peaks, barrier, max_ranks)

    # every rank draws its own batch (independent sequences)
    inp = workload_inputs(rank_workload(w, rank), device=device)
    B = 1 if w.seqlens else w.B
    T = w.total_tokens if w.seqlens else w.T
    N = w.num_seqs
    dt = inp["k"].dtype
    elem = inp["k"].element_size()
    o = torch.empty((B, T, w.H, w.dv), dtype=dt, device=device)
    ST = torch.empty((N, w.H, w.dv, w.dk), dtype=torch.float32, device=device)
    cu = inp.get("cu_seqlens")
    seg = w.seg_len if (w.seg_len and not w.seqlens) else 0
    if seg:  # long sequences with few heads: segment-parallel (pairs, scan, replay)
        ws_n = kda.kda_forward_segmented_workspace_size(B, T, w.H, w.dk, w.dv, w.chunk, dt, seg)
        launches = kda.kda_forward_segmented_launches(B, T, w.H, w.dk, w.dv, w.chunk, dt, seg, args.path)
    else:
        ws_n = kda.kda_forward_workspace_size(B, T, w.H, w.dk, w.dv, w.chunk, N, dt)
        launches = kda.kda_forward_launches(B, T, w.H, w.dk, w.dv, w.chunk, dt, cu is not None, N, args.path)
    ws = torch.empty(max(ws_n, 1), dtype=torch.uint8, device=device)
    tc_ok = kda.kda_forward_launches(B, T, w.H, w.dk, w.dv, w.chunk, dt, cu is not None, N, "tc") > 0
    path_used = "tc" if (args.path != "simt" and tc_ok) else "simt"

    def forward(q, k, v, g, beta, S0):
        if seg:
            kda.kda_forward_segmented(q, k, v, g, beta, S0, seg_len=seg, chunk=w.chunk, o=o, S_T=ST,
                                      workspace=ws, path=args.path)
        else:
            kda.kda_forward(q, k, v, g, beta, S0, chunk=w.chunk, cu_seqlens=cu, o=o, S_T=ST,
                            workspace=ws, path=args.path)

    def step():
        forward(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["S0"])

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    barrier()
    torch.cuda.synchronize(device)
    K = args.steps
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(device.index) as clk:
        t0.record(stream)
        for i in range(K):
            evs[i][0].record(stream)
            step()
            evs[i][1].record(stream)
        t1.record(stream)
        torch.cuda.synchronize(device)
    barrier()
    torch.cuda.synchronize(device)
    ms_total = max_ranks(t0.elapsed_time(t1))
    kern_ms = statistics.mean(a.elapsed_time(b) for a, b in evs)
    ms_step = ms_total / K
    tokens = w.total_tokens
    value = weak_scaling_value(tokens, K, ms_total, world)
    alg_bytes, alg_flops = prefill_algorithmic(w, elem)
    if path_used == "tc" and seg:  # segments: records once, three chain passes, a scan
        kern_src = "linear_attention_recurrence_11_b200/csrc/kda_prefill_split.cu"
        path_used = "tc_segmented"
    elif path_used == "tc":  # AUTO: the split form up to three units per SM, else the single kernel
        sms = torch.cuda.get_device_properties(device).multi_processor_count
        if args.path in ("tc_split", "tc_pipe", "tc_single"):
            path_used = args.path
        else:
            path_used = "tc_split" if N * w.H <= 3 * sms else "tc_single"
        kern_src = ("linear_attention_recurrence_11_b200/csrc/kda_prefill_tc.cu" if path_used == "tc_single"
                    else "linear_attention_recurrence_11_b200/csrc/kda_prefill_split.cu")
    else:
        kern_src = "linear_attention_recurrence_11_b200/csrc/kda_prefill_simt.cu"
    achieved = alg_bytes / (kern_ms / 1e3) / 1e9
    traffic = traffic_for(kern_src, f"{wname}/{path_used}")
    res.update({
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if path_used.startswith("tc") else ("f32" if elem == 4 else "bf16-storage/f32-compute"),
        "data": "synthetic (seeded: q,k unit-norm N(0,1); v N(0,1); beta sigmoid(N); g -5*sigmoid(N))",
        "config": {"workload": wname, "B": B, "T": T, "H": w.H, "dk": w.dk, "dv": w.dv,
                   "chunk": w.chunk, "num_seqs": N, "kernel_path": path_used,
                   **({"seg_len": seg, "segments": -(-T // seg) * B} if seg else {}),
                   "l2": f"inputs larger than L2 ({(inp['q'].numel() * elem * 4) / 1e6:.0f} MB read per step)",
                   "parallelism": f"dp{world} over independent (sequence, head) units"
                                  + (" (segments of a sequence run as units: KCP pairs, scan, replay)" if seg else "")},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "traffic": traffic,
                     "kernel": os.path.basename(kern_src), "kernel_ms": kern_ms,
                     "algorithmic_bytes_per_launch": alg_bytes, "peak_source": peaks["source"] + " (hbm_gbs)"},
        "tensor": {"achieved_tflops": alg_flops / (kern_ms / 1e3) / 1e12,
                   "peak_tflops": peaks["bf16_tflops"],
                   "frac": alg_flops / (kern_ms / 1e3) / 1e12 / peaks["bf16_tflops"],
                   "algorithmic_flops_per_launch": alg_flops, "peak_source": peaks["source"] + " (bf16_tflops)"},
        "gpu_launches": K * launches,
        "clocks": clk.summary(),
    })

    if seg:  # context: the plain prefill on the same workload (one unit per (sequence, head))
        ws_p = torch.empty(max(kda.kda_forward_workspace_size(B, T, w.H, w.dk, w.dv, w.chunk, N, dt), 1),
                           dtype=torch.uint8, device=device)

        def plain():
            kda.kda_forward(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["S0"], chunk=w.chunk,
                            o=o, S_T=ST, workspace=ws_p, path=args.path)
        plain()
        torch.cuda.synchronize(device)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(3):
            plain()
        b.record(stream)
        torch.cuda.synchronize(device)
        res["plain_prefill"] = {"ms_per_step": a.elapsed_time(b) / 3,
                                "tokens_per_s": tokens / (a.elapsed_time(b) / 3 / 1e3),
                                "note": "kda_forward on the same inputs, one unit per (sequence, head); outside the timed region"}
    if args.snap_every > 0 and not seg and not w.seqlens and T >= args.snap_every and args.path != "tc_pipe":
        # the same prefill saving the state every snap_every tokens (prefix cache)
        Ssn = torch.empty((B, T // args.snap_every, w.H, w.dv, w.dk), dtype=torch.float32, device=device)

        def snap():
            kda.kda_forward_snapshots(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["S0"],
                                      snap_every=args.snap_every, chunk=w.chunk, o=o, S_T=ST, S_snap=Ssn,
                                      workspace=ws, path=args.path)
        for _ in range(2):
            snap()
        torch.cuda.synchronize(device)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(5):
            snap()
        b.record(stream)
        torch.cuda.synchronize(device)
        ms_snap = a.elapsed_time(b) / 5
        res["snapshots"] = {"snap_every": args.snap_every, "snapshots_per_unit": T // args.snap_every,
                            "ms_per_step": ms_snap, "overhead_vs_step": ms_snap / kern_ms - 1.0,
                            "snapshot_bytes_per_step": Ssn.numel() * 4,
                            "note": "kda_forward_snapshots on the same inputs, outside the timed region"}
    if not seg and not w.seqlens and args.path != "tc_pipe":  # the pipe form has no fused variant
        # the same step with the fused pre-operations (q, k normalised per row and g computed from
        # gate logits inside the kernels; the synthetic g read as logits, for timing only)
        def fused():
            kda.kda_forward(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["S0"], chunk=w.chunk, o=o,
                            S_T=ST, workspace=ws, path=args.path,
                            fuse=kda.KDA_FUSE_NORM_QK | kda.KDA_FUSE_GATE_LOGITS)
        for _ in range(2):
            fused()
        torch.cuda.synchronize(device)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(5):
            fused()
        b.record(stream)
        torch.cuda.synchronize(device)
        ms_fused = a.elapsed_time(b) / 5
        res["fused"] = {"ms_per_step": ms_fused, "overhead_vs_step": ms_fused / kern_ms - 1.0,
                        "note": "kda_forward with KDA_FUSE_NORM_QK | KDA_FUSE_GATE_LOGITS on the same inputs, "
                                "outside the timed region"}
    if not args.no_e2e:
        res["e2e"] = e2e_prefill(args, device, inp, w, forward, o, ST, world, barrier, max_ranks,
                                 dense=not seg and not w.seqlens)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline_prefill(inp, w, args.cpu_seconds)
        res["cpu_baseline_all_cores"] = cpu_baseline_all_cores(inp, w)
    default_run = args.workload == "prefill" and not args.tokens
    del inp, o, ST, ws
    torch.cuda.empty_cache()
    if default_run and not args.no_varlen:
        res["varlen"] = varlen_measure(args, device, peaks, barrier, max_ranks, world, rank)
        torch.cuda.empty_cache()
    if not args.no_decode and args.workload == "prefill":
        res["decode"] = decode_measure(args, device, peaks, barrier, max_ranks, world,
                                       steps=args.decode_steps)
    return res


def varlen_measure(args, device, peaks, barrier, max_ranks, world, rank):
    """The packed long-context workload (8 sequences, log-uniform lengths in
    [4096, 131072], 96 heads) through kda_forward with cu_seqlens, inputs
    resident in HBM; and, for the chain-bound question, the longest sequence
    alone through the same entry point (its time over the batch's time)."""
    import torch
    from linear_attention_recurrence_11_b200 import kda
    from linear_attention_recurrence_11_b200.inputs import WORKLOADS, workload_inputs
    w = rank_workload(WORKLOADS["varlen_h96_8seq_d128_bf16"], rank)
    inp = workload_inputs(w, device=device)
    T, N = w.total_tokens, w.num_seqs
    dt = inp["k"].dtype
    o = torch.empty((1, T, w.H, w.dv), dtype=dt, device=device)
    ST = torch.empty((N, w.H, w.dv, w.dk), dtype=torch.float32, device=device)
    ws = torch.empty(max(1, kda.kda_forward_workspace_size(1, T, w.H, w.dk, w.dv, w.chunk, N, dt)),
                     dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)

    def step():
        kda.kda_forward(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["S0"], chunk=w.chunk,
                        cu_seqlens=inp["cu_seqlens"], o=o, S_T=ST, workspace=ws, path=args.path)

    def timed(fn, K):
        for _ in range(2):
            fn()
        torch.cuda.synchronize(device)
        barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(K):
            fn()
        b.record(stream)
        torch.cuda.synchronize(device)
        return max_ranks(a.elapsed_time(b)) / K

    K = max(3, min(args.steps, 5))
    with ClockSampler(device.index) as clk:
        ms = timed(step, K)
    # the longest sequence alone (dense B = 1), the same kernels
    cu = w.cu_seqlens()
    nl = max(range(N), key=lambda n: w.seqlens[n])
    sl = {x: inp[x][:, cu[nl]:cu[nl + 1]].contiguous() for x in ("q", "k", "v", "g", "beta")}
    o1 = torch.empty_like(sl["v"])
    ST1 = torch.empty((1, w.H, w.dv, w.dk), dtype=torch.float32, device=device)

    ws1 = torch.empty(max(1, kda.kda_forward_workspace_size(1, w.seqlens[nl], w.H, w.dk, w.dv, w.chunk, 1, dt,
                                                           path=args.path)), dtype=torch.uint8, device=device)

    def longest():
        kda.kda_forward(sl["q"], sl["k"], sl["v"], sl["g"], sl["beta"], None, chunk=w.chunk, o=o1, S_T=ST1,
                        workspace=ws1, path=args.path)
    ms_long = timed(longest, K)
    del o1, ST1, ws1, sl
    # the same batch through the segment-parallel prefill (sequences cut every seg_len
    # tokens; the short ones stay one segment each)
    seg_len = 16384
    wss = torch.empty(max(1, kda.kda_forward_segmented_varlen_workspace_size(T, w.H, w.dk, w.dv, w.chunk, dt, N,
                                                                             seg_len)),
                      dtype=torch.uint8, device=device)

    def segmented():
        kda.kda_forward_segmented(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["S0"], seg_len=seg_len,
                                  chunk=w.chunk, cu_seqlens=inp["cu_seqlens"], o=o, S_T=ST, workspace=wss,
                                  path=args.path)
    ms_seg = timed(segmented, 3)
    del wss
    alg_bytes, alg_flops = prefill_algorithmic(w, dt.itemsize)
    gbs = alg_bytes / (ms / 1e3) / 1e9
    return {"workload": w.name, "tokens": T, "sequences": N, "lengths": list(w.seqlens),
            "ms_per_step": ms, "tokens_per_s": world * T / (ms / 1e3),
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / peaks["hbm_gbs"], "algorithmic_bytes_per_step": alg_bytes,
                         "peak_source": peaks["source"] + " (hbm_gbs)"},
            "tensor_frac": alg_flops / (ms / 1e3) / 1e12 / peaks["bf16_tflops"],
            "longest_sequence": {"tokens": w.seqlens[nl], "ms": ms_long, "ratio_to_batch": ms_long / ms,
                                 "note": "the longest sequence alone (all 96 heads) through kda_forward; "
                                         "near 1 means the batch is bound by that sequence's chain"},
            "segmented": {"seg_len": seg_len, "ms_per_step": ms_seg, "tokens_per_s": world * T / (ms_seg / 1e3),
                          "launches": kda.kda_forward_segmented_varlen_launches(T, w.H, w.dk, w.dv, w.chunk, dt, N,
                                                                                seg_len, args.path),
                          "note": "kda_forward_segmented with cu_seqlens: segment pairs, scan, replay; three "
                                  "passes over the inputs, outside the leg's timed steps"},
            "gpu_launches": K * kda.kda_forward_launches(1, T, w.H, w.dk, w.dv, w.chunk, dt, True, N, args.path),
            "steps": K, "clocks": clk.summary(),
            "l2": f"inputs larger than L2 ({4 * inp['q'].numel() * dt.itemsize / 1e9:.1f} GB read per step)"}


def e2e_prefill(args, device, inp, w, forward, o, ST, world, barrier, max_ranks, dense):
    """Same metric from pinned host buffers, host<->device copies inside the
    timed region: per step the inputs q,k,v,g,beta(,S0) go up and o and S_T come
    back. Dense batches go through the C ABI's host entry point
    (kda_forward_host: pieces of --e2e-piece tokens, uploads, launches and
    downloads overlapped); packed or segmented workloads copy whole tensors
    around the device call. For dense batches the serial form (whole-tensor
    copies around kda_forward) is timed too, for comparison."""
    import torch
    from linear_attention_recurrence_11_b200 import kda
    names = [n for n in ("q", "k", "v", "g", "beta", "S0") if inp.get(n) is not None]
    host = {n: inp[n].to("cpu").pin_memory() for n in names}
    dev = {n: torch.empty_like(inp[n]) for n in names}
    o_h = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
    S_h = torch.empty(ST.shape, dtype=ST.dtype, pin_memory=True)
    h2d = sum(host[n].numel() * host[n].element_size() for n in names)
    d2h = o_h.numel() * o_h.element_size() + S_h.numel() * S_h.element_size()
    stream = torch.cuda.current_stream(device)

    def serial_step():
        for n in names:
            dev[n].copy_(host[n], non_blocking=True)
        forward(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], dev.get("S0"))
        o_h.copy_(o, non_blocking=True)
        S_h.copy_(ST, non_blocking=True)

    if dense:
        B, T, H, dk = inp["k"].shape
        ws = torch.empty(kda.kda_forward_host_workspace_size(B, T, H, dk, inp["v"].shape[-1], w.chunk,
                                                             inp["k"].dtype, args.e2e_piece),
                         dtype=torch.uint8, device=device)

        def host_step():
            kda.kda_forward_host(host["q"], host["k"], host["v"], host["g"], host["beta"], host.get("S0"),
                                 chunk=w.chunk, piece_len=args.e2e_piece, o=o_h, S_T=S_h, workspace=ws,
                                 device=device, stream=stream, path=args.path)

    def timed(step):
        K = max(3, min(args.steps, 10))
        for _ in range(2):
            step()
        torch.cuda.synchronize(device)
        barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(K):
            step()
        b.record(stream)
        torch.cuda.synchronize(device)
        return max_ranks(a.elapsed_time(b)), K

    ms, K = timed(host_step if dense else serial_step)
    res = {"value": world * w.total_tokens * K / (ms / 1e3), "unit": "tokens/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": K,
           "ms_per_step": ms / K}
    if dense:
        ms_serial, K_s = timed(serial_step)
        res["api"] = f"kda_forward_host (pieces of {args.e2e_piece or 'T/8'} tokens)"
        res["serial_ms_per_step"] = ms_serial / K_s
    else:
        res["api"] = "whole-tensor copies around the device call"
    return res


def decode_measure(args, device, peaks, barrier, max_ranks, world, steps):
    """Decode steps over 256 requests x 96 heads (1.61 GB of fp32 state, larger
    than L2), states updated in place, for the workload's step count (1000)
    unless --decode-steps says otherwise; every step has its own seeded inputs
    (drawn before the timed region)."""
    import torch
    from linear_attention_recurrence_11_b200 import kda
    from linear_attention_recurrence_11_b200.inputs import WORKLOADS, workload_inputs
    import dataclasses
    w = WORKLOADS["decode_n256_h96_d128"]
    if args.decode_requests != w.B:
        w = dataclasses.replace(w, B=args.decode_requests)
    steps = steps or w.decode_steps
    S = workload_inputs(w, device=device, step=0)["S0"]
    warm = max(3, args.warmup)
    sets = []
    for s in range(warm + steps):
        d = workload_inputs(w, device=device, step=s)
        sets.append({k: d[k][:, 0].contiguous() for k in ("q", "k", "v", "g", "beta")})
    o = torch.empty((w.B, w.H, w.dv), dtype=sets[0]["k"].dtype, device=device)
    stream = torch.cuda.current_stream(device)

    def step(i):
        d = sets[i]
        kda.kda_decode_step(d["q"], d["k"], d["v"], d["g"], d["beta"], S, o)

    for i in range(warm):
        step(i)
    torch.cuda.synchronize(device)
    barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(device.index) as clk:
        a.record(stream)
        for i in range(steps):
            step(warm + i)
        b.record(stream)
        torch.cuda.synchronize(device)
    ms = max_ranks(a.elapsed_time(b)) / steps
    # speculative rounds on the states as the timed steps left them
    multi = multi_decode_measure(args, device, peaks, max_ranks, world, w, S) if args.draft_tokens > 0 else None
    # the same steps captured once in a CUDA graph and replayed (launch cost off the host)
    graph_ms = None
    try:
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(device)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            with torch.cuda.graph(g, stream=side):
                for i in range(steps):
                    step(warm + i)
        stream.wait_stream(side)
        g.replay()
        torch.cuda.synchronize(device)
        barrier()
        a.record(stream)
        g.replay()
        b.record(stream)
        torch.cuda.synchronize(device)
        graph_ms = max_ranks(a.elapsed_time(b)) / steps
        del g
    except RuntimeError:
        graph_ms = None
    elem = sets[0]["k"].element_size()
    del sets
    alg_bytes, _ = decode_algorithmic(w.B, w.H, w.dk, w.dv, elem)
    gbs = alg_bytes / (ms / 1e3) / 1e9
    res = {"metric": f"KDA decode step GB/s ({w.B} req x {w.H} heads, fp32 state)",
            "value": gbs * world, "unit": "GB/s", "ms_per_step": ms,
            "tokens_per_s": world * w.B / (ms / 1e3), "steps": steps,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / peaks["hbm_gbs"], "kernel": "kda_decode.cu",
                         # the committed capture is scaled to the full 256-request batch only
                         "traffic": traffic_for("linear_attention_recurrence_11_b200/csrc/kda_decode.cu",
                                                "decode_n256_h96_d128") if w.B == 256 else None,
                         "algorithmic_bytes_per_launch": alg_bytes,
                         "peak_source": peaks["source"] + " (hbm_gbs)"},
            "gpu_launches": steps, "clocks": clk.summary(),
            "graph_ms_per_step": graph_ms,
            "frac_of_nominal_hbm": gbs / NOMINAL_HBM_GBS,
            "requests": w.B, "l2": f"state {w.B * w.H * w.dk * w.dv * 4 / 1e9:.2f} GB per step, larger than L2"}
    if multi is not None:
        res["multi_token"] = multi
    return res


def multi_decode_algorithmic(B, H, T, dk, dv, accepted):
    """Bytes one speculative round must move (bf16 inputs and outputs, fp32 states):
    the verification reads every state and the inputs of all T tokens and writes all
    outputs; the commit reads and writes the states of the requests with an accepted
    token and reads the accepted tokens' inputs."""
    state = dk * dv * 4
    per_tok = (3 * dk + dv + 1) * 2
    written = sum(1 for a in accepted if a > 0)
    return ((B + 2 * written) * H * state + (B * T + sum(accepted)) * H * per_tok
            + B * T * H * dv * 2)


def multi_decode_measure(args, device, peaks, max_ranks, world, w, S, rounds=10):
    """Speculative decoding rounds on the same states: T draft tokens per request,
    a verification call (outputs of all T, states untouched) then a commit call
    (the state after each request's accepted prefix, no outputs). Acceptance
    counts are seeded draws in [0, T]."""
    import torch
    from linear_attention_recurrence_11_b200 import kda
    from linear_attention_recurrence_11_b200.inputs import make_inputs
    T = args.draft_tokens
    inp = make_inputs(w.B, T, w.H, w.dk, w.dv, "bf16", seed=w.seed + 77, device=device)
    gen = torch.Generator().manual_seed(w.seed + 78)
    acc = torch.randint(0, T + 1, (w.B,), generator=gen, dtype=torch.int32).to(device)
    zeros = torch.zeros_like(acc)
    o = torch.empty((w.B, T, w.H, w.dv), dtype=inp["k"].dtype, device=device)
    stream = torch.cuda.current_stream(device)

    def round_():
        kda.kda_decode_multi(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], S, o, n_accept=zeros)
        kda.kda_decode_multi(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], S, None, n_accept=acc,
                             outputs=False)

    for _ in range(3):
        round_()
    torch.cuda.synchronize(device)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(rounds):
        round_()
    b.record(stream)
    torch.cuda.synchronize(device)
    ms = max_ranks(a.elapsed_time(b)) / rounds
    # each call alone: the verification (repeatable, states untouched), then the commit
    parts = {}
    for name, call in (("verify", lambda: kda.kda_decode_multi(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                                                               S, o, n_accept=zeros)),
                       ("commit", lambda: kda.kda_decode_multi(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                                                               S, None, n_accept=acc, outputs=False))):
        torch.cuda.synchronize(device)
        a.record(stream)
        for _ in range(rounds):
            call()
        b.record(stream)
        torch.cuda.synchronize(device)
        parts[name + "_ms"] = max_ranks(a.elapsed_time(b)) / rounds
    accepted = int(acc.sum().item())
    bytes_round = multi_decode_algorithmic(w.B, w.H, T, w.dk, w.dv, acc.tolist())
    gbs = bytes_round / (ms / 1e3) / 1e9
    return {"draft_tokens": T, "ms_per_round": ms, "accepted_tokens_per_round": accepted * world,
            "accepted_tokens_per_s": world * accepted / (ms / 1e3),
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / peaks["hbm_gbs"], "kernel": "kda_decode_multi.cu",
                         "algorithmic_bytes_per_round": bytes_round, "peak_source": peaks["source"] + " (hbm_gbs)"},
            **parts, "gpu_launches": 2 * rounds,
            "note": "per round: verify (outputs of all draft tokens) + commit (accepted prefixes); "
                    "kda_decode_step would move the state twice per accepted token instead"}


def run_decode_main(args, rank, world, device, w, peaks, barrier, max_ranks):
    d = decode_measure(args, device, peaks, barrier, max_ranks, world, steps=args.steps)
    return {"metric": d["metric"], "value": d["value"], "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": d["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic", "config": {"workload": w.name, "N": d["requests"], "H": w.H, "dk": w.dk,
                                            "dv": w.dv, "l2": d["l2"]},
            "roofline": d["roofline"], "gpu_launches": d["gpu_launches"], "clocks": d["clocks"]}


# ---------------------------------------------------------- CPU baseline

def _oracle_sample(inp, w, seconds, max_heads=None):
    """Time the fp64 oracle (sequential form, one host core) on whole heads of
    the workload until about ``seconds`` have elapsed. Returns
    (token-heads processed, elapsed seconds, heads)."""
    import oracle
    from linear_attention_recurrence_11_b200.inputs import to_f64
    oracle.build()
    T = w.total_tokens if w.seqlens else w.T
    T = min(T, 8192)
    done, el, heads = 0, 0.0, 0
    h = 0
    while el < seconds and (max_heads is None or heads < max_heads):
        a = [to_f64(inp[x][0, :T, h % w.H]) for x in ("q", "k", "v", "g", "beta")]
        t = time.perf_counter()
        oracle.forward(*a)
        el += time.perf_counter() - t
        done += T
        heads += 1
        h += 1
    return done, el, heads, T


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def cpu_baseline_prefill(inp, w, seconds):
    done, el, heads, T = _oracle_sample(inp, w, seconds)
    return {"value": done / w.H / el, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{heads} of {w.H} heads x {T} tokens of {w.name}, sequential fp64 oracle, "
                      f"one thread; tokens/s = token-heads/s / {w.H}",
            "host_cpus": os.cpu_count(), "cpu_model": cpu_model(), "seconds": el}


def cpu_baseline_all_cores(inp, w):
    """The same oracle over all host cores: one whole head per task on a thread
    pool (the oracle is a C library called through ctypes, which releases the
    GIL, so the heads run in parallel), every head of the workload at up to 8192
    tokens; the wall time includes each head's copy to fp64."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    from linear_attention_recurrence_11_b200.inputs import to_f64
    oracle.build()
    T = min(w.total_tokens if w.seqlens else w.T, 8192)
    host = {x: inp[x][0, :T].cpu() for x in ("q", "k", "v", "g", "beta")}
    cores = os.cpu_count() or 1

    def one(h):
        a = [to_f64(host[x][:, h]) for x in ("q", "k", "v", "g", "beta")]
        oracle.forward(*a)

    t = time.perf_counter()
    with ThreadPoolExecutor(max_workers=cores) as ex:
        list(ex.map(one, range(w.H)))
    el = time.perf_counter() - t
    return {"value": T * w.H / w.H / el, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "label": "CPU baseline, all cores",
            "sample": f"all {w.H} heads x {T} tokens of {w.name}, sequential fp64 oracle per head, "
                      f"{cores} threads (one head per task); tokens/s = token-heads/s / {w.H}",
            "seconds": el}


def run_reference(args, rank, world):
    """The reference arm: the oracle as it stands, on host cores, on a bounded
    sample of the same workload per step."""
    if rank != 0:
        return None
    import torch
    from linear_attention_recurrence_11_b200.inputs import WORKLOADS, workload_inputs
    w = WORKLOADS[WORKLOAD_ALIASES[args.workload]]
    if w.decode_steps:
        w_in = workload_inputs(w, device="cpu", step=0)
    else:
        import dataclasses
        small = dataclasses.replace(w, T=min(w.T or 8192, 8192), seqlens=(), B=1, H=2)
        w_in = workload_inputs(small, device="cpu")
    per_step = max(1.0, min(8.0, 150.0 / max(1, args.steps + args.warmup)))
    tot_done, tot_el = 0, 0.0
    heads = T = 0
    for i in range(args.warmup + args.steps):
        if w.decode_steps:
            import numpy as np
            import oracle
            from linear_attention_recurrence_11_b200.inputs import to_f64
            d = {k: to_f64(w_in[k][:, 0]) for k in ("q", "k", "v", "g", "beta")}
            S = to_f64(w_in["S0"])
            t = time.perf_counter()
            n_units = 0
            while time.perf_counter() - t < per_step:
                n, h = n_units % w.B, (n_units // w.B) % w.H
                St = np.ascontiguousarray(S[n, h])
                oracle.decode_step(d["q"][n, h], d["k"][n, h], d["v"][n, h], d["g"][n, h],
                                   d["beta"][n, h], St)
                n_units += 1
            done, el = n_units, time.perf_counter() - t
        else:
            done, el, heads, T = _oracle_sample(w_in, small, per_step, max_heads=2)
        if i >= args.warmup:
            tot_done += done
            tot_el += el
    if w.decode_steps:
        alg, _ = decode_algorithmic(1, 1, w.dk, w.dv, 2)
        value, unit = tot_done * alg / tot_el / 1e9, "GB/s"
        metric = "KDA decode step GB/s (256 req x 96 heads, fp32 state)"
        sample = f"(request, head) units of one decode step, fp64 oracle, one thread, ~{per_step:.0f} s per step"
    else:
        value, unit = tot_done / w.H / tot_el, "tokens/s"
        metric = METRIC
        sample = (f"up to 2 heads x {T} tokens per step (same distributions as {w.name}), "
                  f"sequential fp64 oracle, one thread; tokens/s = token-heads/s / {w.H}")
    ms = tot_el / max(1, args.steps) * 1e3
    return {"impl": "reference", "metric": metric, "value": value, "unit": unit, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name},
            "cpu_baseline": {"value": value, "unit": unit, "cores": 1, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    args = parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return 0
    import torch
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=device)
    try:
        res = run_ours(args, rank, world, device)
    finally:
        if world > 1:
            torch.distributed.barrier()
            torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
