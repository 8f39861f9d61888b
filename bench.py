#!/usr/bin/env python
"""Benchmark of the HSA hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl hsa|reference]

Headline step: one ``hsa_fwd`` (pool -> select -> chunk attention + fusion)
over the 64K-token workload (B=1, L=65536, S=64, K=8, h_q=16, h_kv=2, d=128,
bf16, per-chunk key offsets), inputs resident in HBM, L2 flushed (256 MB
write) before every timed step.  Prints ONE JSON line on rank 0.

Also measured in the same run (keys "decode" and "train"): the decode step at
B=16 with a 16K-token cache (median of CUDA-graph replays) and one
forward+backward step of the B=4, L=16K training workload.

Multi-GPU (torchrun): each rank runs its own sequence (the (batch, group)
units are independent: no collective on the data path), weak scaling; time is
the max over ranks of the device time.

``--impl reference`` times the fp64 CPU oracle (the only reference this
method has) on a bounded row sample of the same workload, on rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "HSA fwd tokens/s at L=64K and fraction of roofline; decode step latency at B=16"
FLUSH_BYTES = 256 << 20
# B200 datasheet figures (dense bf16 tensor throughput, HBM3e bandwidth of the HGX part),
# reported beside the fractions of the measured peaks
DATASHEET = {"bf16_tflops": 2250.0, "hbm_gbs": 7700.0}


# --------------------------------------------------------------------------- helpers
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return {"hbm_gbs": j["hbm_gbs"], "bf16_tflops": j["bf16_tflops"],
                "bf16_tflops_sustained": j.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def selected_pairs(wl) -> int:
    """sum over (b, t, g) of min(K, eligible chunks): the (token, group, slot) triples."""
    t = np.arange(wl.L)
    ne = np.minimum(t // wl.S, wl.n_c)
    return int(wl.B * wl.h_kv * np.minimum(ne, wl.K).sum())


def eligible_pairs(wl) -> int:
    t = np.arange(wl.L)
    return int(wl.B * wl.h_kv * np.minimum(t // wl.S, wl.n_c).sum())


def fwd_work(wl):
    """Algorithmic FLOPs and compulsory bytes of one forward (selected pairs only)."""
    G = wl.h_q // wl.h_kv
    att_flops = selected_pairs(wl) * G * 4 * wl.S * wl.d
    sel_flops = eligible_pairs(wl) * 2 * wl.d
    eb = 2 if wl.dtype == "bf16" else 4
    tok = wl.B * wl.L
    kv = 2 * wl.B * wl.h_kv * wl.L * wl.d * eb
    q = tok * wl.h_q * wl.d * eb
    qs = tok * wl.h_kv * wl.d * eb
    kbar = wl.B * wl.h_kv * wl.n_c * wl.d * 4
    byt = q + qs + kv + q + 2 * kbar  # q, q_slc, k, v read; o written; kbar written + read
    return att_flops, sel_flops, byt


def source_hash(files):
    """sha256 prefix of the files' code: comments, trailing blanks and empty lines removed,
    so an edit to comments alone leaves the key of a measurement in place."""
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), encoding="utf-8") as fh:
            src = fh.read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        code = "\n".join(ln.rstrip() for ln in src.splitlines() if ln.strip())
        h.update(code.encode())
    return h.hexdigest()[:12]


def read_traffic(kernel_file: str):
    """Per-launch DRAM bytes of the dominant kernel from the committed ncu
    summary, if it was taken on the current source (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(p):
        return None
    # the kernel's behaviour also depends on the library's shared headers
    want = source_hash([kernel_file, "chunked_hierarchical_sparse_b200/csrc/hsa_internal.cuh",
                        "chunked_hierarchical_sparse_b200/csrc/sm100.cuh"])
    for ln in open(p):
        m = re.match(r"\s*(\S+)\s+source=(\w+)\s+bytes_per_launch=(\d+)", ln)
        if m and m.group(1) == os.path.basename(kernel_file) and m.group(2) == want:
            return int(m.group(3))
    return None


class ClockSampler:
    """SM clocks and throttle reasons sampled through NVML every few ms while
    the timed region runs."""

    def __init__(self, index: int, period_s: float = 0.005):
        self.index = index
        self.period = period_s
        self.samples = []
        self.stop = threading.Event()
        self.err = None

    def _run(self):
        try:
            import pynvml as nv
            nv.nvmlInit()
            h = nv.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
            bits = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
                    "sw_power_cap": 0x4}
            while not self.stop.is_set():
                mhz = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((mhz, [n for n, b in bits.items() if r & b]))
                time.sleep(self.period)
        except Exception as e:  # pragma: no cover - reported in the JSON line
            self.err = repr(e)

    def __enter__(self):
        self.max_mhz = None
        self.t = threading.Thread(target=self._run, daemon=True)
        self.t.start()
        time.sleep(0.05)
        return self

    def __exit__(self, *a):
        self.stop.set()
        self.t.join(timeout=5)

    def summary(self):
        sm = [m for m, _ in self.samples]
        reasons = sorted({r for _, rs in self.samples for r in rs})
        out = {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": self.max_mhz,
               "reasons": reasons, "samples": len(sm), "source": "nvml"}
        if self.err:
            out["error"] = self.err
        return out


# --------------------------------------------------------------------------- reference arm
def run_reference(args, rank, world):
    if rank != 0:
        return
    import oracle
    from chunked_hierarchical_sparse_b200 import synth
    wl = synth.WORKLOADS[args.workload]
    x = synth.make_inputs(wl)
    kbar = oracle.pool(x["k"], wl.S)
    rng = np.random.default_rng(0)
    n_rows = args.ref_rows
    times = []
    for i in range(args.warmup + args.steps):
        rows = np.sort(rng.choice(wl.B * wl.L, size=n_rows, replace=False))
        t0 = time.perf_counter()
        oracle.fwd(x["q"], x["k"], x["v"], x["q_slc"], kbar, wl.S, wl.K, rows=rows)
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            times.append(dt)
    tot = sum(times)
    value = n_rows * len(times) / tot
    cores = oracle.num_threads()
    sample = f"{n_rows} uniformly sampled token rows of the {args.workload} workload per step (pool once per run)"
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "impl": "reference",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * tot / len(times), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.workload, "B": wl.B, "L": wl.L, "S": wl.S, "K": wl.K,
                       "h_q": wl.h_q, "h_kv": wl.h_kv, "d": wl.d, "global_batch": wl.B,
                       "seq_len": wl.L},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------- hsa arm
def cpu_baseline(wl, x, budget_s: float):
    """Time the oracle as it stands on a bounded row sample of the workload."""
    import oracle
    kbar = oracle.pool(x["k"], wl.S)
    rng = np.random.default_rng(1)
    probe = np.sort(rng.choice(wl.B * wl.L, size=64, replace=False))
    t0 = time.perf_counter()
    oracle.fwd(x["q"], x["k"], x["v"], x["q_slc"], kbar, wl.S, wl.K, rows=probe)
    per_row = (time.perf_counter() - t0) / 64
    n = int(min(wl.B * wl.L, max(64, budget_s / max(per_row, 1e-9))))
    rows = np.sort(rng.choice(wl.B * wl.L, size=n, replace=False))
    t0 = time.perf_counter()
    oracle.fwd(x["q"], x["k"], x["v"], x["q_slc"], kbar, wl.S, wl.K, rows=rows)
    dt = time.perf_counter() - t0
    return {"value": n / dt, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{n} uniformly sampled token rows of the 64K workload ({dt:.1f} s)"}


def to_dev(a, dev, bf16=True):
    import torch
    return torch.from_numpy(a).to(dev, torch.bfloat16 if bf16 else torch.float32)


def bench_decode(hsa, dev, reps=1000):
    import torch
    from chunked_hierarchical_sparse_b200 import synth
    wl = synth.WORKLOADS["decode16k"]
    x = synth.make_inputs(wl)
    q, qs, kc, vc = (to_dev(x[n], dev) for n in ("q", "q_slc", "k", "v"))
    kbar = hsa.hsa_pool(kc)
    o = torch.empty_like(q)
    n = hsa.hsa_workspace_size(wl.B, wl.L, wl.h_q, wl.h_kv, wl.d, wl.S, wl.K, torch.bfloat16,
                               hsa.OP_DECODE)
    ws = torch.empty(n, dtype=torch.uint8, device=dev)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for _ in range(3):
            hsa.hsa_decode(q, qs, kc, vc, kbar, wl.K, o=o, ws=ws, want_sel=False)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        hsa.hsa_decode(q, qs, kc, vc, kbar, wl.K, o=o, ws=ws, want_sel=False)
    for _ in range(20):
        g.replay()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    for a, b in ev:
        a.record()
        g.replay()
        b.record()
    torch.cuda.synchronize()
    warm = sorted(a.elapsed_time(b) * 1e3 for a, b in ev)
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    cold = []
    for i in range(50):
        flush.fill_(float(i))
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        g.replay()
        b.record()
        torch.cuda.synchronize()
        cold.append(a.elapsed_time(b) * 1e3)
    cold.sort()
    del g
    # the launch floor of this measurement: a graph of one trivial kernel, replayed the same way
    tiny = torch.zeros(1, dtype=torch.float32, device=dev)
    g0 = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g0):
        tiny.add_(1.0)
    floor = _median_us(g0.replay, 1000)
    del g0
    # steps captured back to back in one graph (a serving loop): time per step
    n_in = 16
    gn = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gn):
        for _ in range(n_in):
            hsa.hsa_decode(q, qs, kc, vc, kbar, wl.K, o=o, ws=ws, want_sel=False)
    per_step = _median_us(gn.replay, 200) / n_in
    del gn
    # kernel-only time of the decode kernel (timing facility, warm)
    hsa.hsa_timing_enable(True)
    for _ in range(50):
        hsa.hsa_decode(q, qs, kc, vc, kbar, wl.K, o=o, ws=ws, want_sel=False)
    torch.cuda.synchronize()
    kms, kn = hsa.hsa_timing_read("decode")
    hsa.hsa_timing_enable(False)
    eb = 2
    sel_bytes = wl.B * wl.h_kv * wl.K * 2 * wl.S * wl.d * eb
    byt = (x["q"].size + x["q_slc"].size) * eb + wl.B * wl.h_kv * wl.n_c * wl.d * 4 + sel_bytes + x["q"].size * eb
    return {"workload": "decode16k", "B": wl.B, "P": wl.L, "unit": "us",
            "median_us_warm_graph": warm[len(warm) // 2], "p10_us_warm": warm[len(warm) // 10],
            "p90_us_warm": warm[9 * len(warm) // 10], "median_us_cold_l2": cold[len(cold) // 2],
            "replays": reps, "kernel_us": 1e3 * kms / max(kn, 1),
            "graph_floor_us": floor, "per_step_us_16_in_graph": per_step,
            "compulsory_bytes": int(byt), "roofline_us": byt / (load_peaks()["hbm_gbs"] * 1e9) * 1e6}


def _median_us(fn, reps):
    import torch
    for _ in range(5):
        fn()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    for a, b in ev:
        a.record()
        fn()
        b.record()
    torch.cuda.synchronize()
    t = sorted(a.elapsed_time(b) * 1e3 for a, b in ev)
    return t[len(t) // 2]


def bench_decode_offload(hsa, dev, layers=(1, 4), reps=200):
    """The decode16k step with the KV cache in page-locked host memory: only the
    K selected chunks per (sequence, group) cross the host link.  For n_layers
    layers sharing one selection (hsa_decode_multi) against n_layers separate
    hsa_decode calls (each selecting and reading its chunks again)."""
    import torch
    from chunked_hierarchical_sparse_b200 import synth
    wl = synth.WORKLOADS["decode16k"]
    x = synth.make_inputs(wl)
    qs = to_dev(x["q_slc"], dev)
    kh = torch.from_numpy(x["k"]).to(torch.bfloat16).pin_memory()
    vh = torch.from_numpy(x["v"]).to(torch.bfloat16).pin_memory()
    kbar = hsa.hsa_pool(kh.to(dev))
    n = hsa.hsa_workspace_size(wl.B, wl.L, wl.h_q, wl.h_kv, wl.d, wl.S, wl.K, torch.bfloat16, hsa.OP_DECODE)
    ws = torch.empty(n, dtype=torch.uint8, device=dev)
    # host-to-device copy bandwidth of this box's link (the bound of the offloaded step)
    dst = torch.empty(kh.numel(), dtype=torch.bfloat16, device=dev)
    link_us = _median_us(lambda: dst.copy_(kh.view(-1), non_blocking=True), 10)
    link_gbs = kh.numel() * 2 / (link_us * 1e-6) / 1e9
    del dst
    sel_bytes = wl.B * wl.h_kv * wl.K * 2 * wl.S * wl.d * 2
    out = {"workload": "decode16k, KV cache in page-locked host memory", "unit": "us",
           "host_link_h2d_gbs": link_gbs, "selected_bytes_per_step": sel_bytes,
           "link_bound_us": sel_bytes / (link_gbs * 1e9) * 1e6}
    for NL in layers:
        q = to_dev(synth.layer_queries(wl, NL), dev)
        o = torch.empty_like(q)
        shared = _median_us(lambda: hsa.hsa_decode_multi(q, qs, kh, vh, kbar, wl.K, o=o, ws=ws, want_sel=False),
                            reps)
        ol = [torch.empty_like(q[l]) for l in range(NL)]
        ql = [q[l].contiguous() for l in range(NL)]

        def separate():
            for l in range(NL):
                hsa.hsa_decode(ql[l], qs, kh, vh, kbar, wl.K, o=ol[l], ws=ws, want_sel=False)
        sep = _median_us(separate, reps)
        out[f"layers{NL}"] = {"shared_us": shared, "separate_us": sep,
                              "achieved_link_gbs": sel_bytes / (shared * 1e-6) / 1e9}
    return out


def bench_train(hsa, dev, steps=3):
    import torch
    from chunked_hierarchical_sparse_b200 import synth
    wl = synth.WORKLOADS["train16k"]
    x = synth.make_inputs(wl)
    t = {n: to_dev(x[n], dev) for n in ("q", "k", "v", "q_slc", "dO")}
    del x
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    def step():
        o, lse, idx, w, kbar = hsa.hsa_fwd(t["q"], t["k"], t["v"], t["q_slc"], wl.K)
        return hsa.hsa_bwd(t["q"], t["k"], t["v"], t["q_slc"], t["dO"], lse, idx, w, kbar, wl.K)

    step()
    torch.cuda.synchronize()
    times = []
    hsa.hsa_timing_enable(True)
    for i in range(steps):
        flush.fill_(float(i))
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        step()
        b.record()
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b))
    per_kernel = {k: round(hsa.hsa_timing_read(k)[0] / steps, 4) for k in hsa.KERNELS
                  if hsa.hsa_timing_read(k)[1] > 0}
    hsa.hsa_timing_enable(False)
    att, sel, _ = fwd_work(wl)
    G = wl.h_q // wl.h_kv
    bwd_flops = selected_pairs(wl) * G * 12 * wl.S * wl.d
    ms = float(np.median(times))
    flops = att + sel + bwd_flops
    return {"workload": "train16k", "ms_per_step": ms, "tokens_per_s": wl.B * wl.L / (ms / 1e3),
            "algorithmic_tflop": flops / 1e12,
            "roofline_ms": flops / (load_peaks()["bf16_tflops"] * 1e12) * 1e3,
            "kernel_ms_per_step": per_kernel}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="hsa", choices=["hsa", "reference"])
    ap.add_argument("--ref-rows", type=int, default=4096)
    ap.add_argument("--cpu-budget-s", type=float, default=12.0)
    ap.add_argument("--no-extras", action="store_true", help="skip the decode and train measurements")
    ap.add_argument("--no-cpu", action="store_true", help="skip the oracle CPU baseline")
    ap.add_argument("--decode-only", action="store_true",
                    help="time only the decode16k step (one GPU; the case used for ncu captures of the decode kernel)")
    ap.add_argument("--train-only", action="store_true",
                    help="time only the train16k step (one GPU; the case used for ncu captures of the backward)")
    ap.add_argument("--workload", default="fwd64k", choices=["fwd64k", "fwd16k"],
                    help="forward workload (fwd16k: the smaller case used for ncu captures)")
    args = ap.parse_args()
    assert args.warmup >= 3 or args.impl == "reference", "at least 3 warm-up steps"

    from chunked_hierarchical_sparse_b200 import dist_util
    world, rank, local = dist_util.env_ranks()

    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    import torch
    import chunked_hierarchical_sparse_b200 as hsa
    from chunked_hierarchical_sparse_b200 import synth

    if world > 1:
        torch.cuda.set_device(local)
        dist_util.init(world, "nccl")
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    hsa.load_library()
    if args.decode_only or args.train_only:
        if rank == 0:
            key, fn = ("decode", bench_decode) if args.decode_only else ("train", bench_train)
            print(json.dumps({key: fn(hsa, dev)}), flush=True)
        dist_util.finish(world)
        return

    base = synth.WORKLOADS[args.workload]
    wl = base.scaled(seed=dist_util.rank_seed(base.seed, rank))  # one independent sequence per rank
    x = synth.make_inputs(wl)
    q, k, v, qs = (to_dev(x[n], dev) for n in ("q", "k", "v", "q_slc"))
    o = torch.empty_like(q)
    nws = hsa.hsa_workspace_size(wl.B, wl.L, wl.h_q, wl.h_kv, wl.d, wl.S, wl.K, torch.bfloat16, hsa.OP_FWD)
    ws = torch.empty(nws, dtype=torch.uint8, device=dev)
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    def fwd():
        hsa.hsa_fwd(q, k, v, qs, wl.K, want_lse=False, want_sel=False, o=o, ws=ws)

    for i in range(args.warmup):
        flush.fill_(float(i))
        fwd()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    dist_util.barrier(world)
    torch.cuda.synchronize()
    hsa.hsa_timing_enable(True)
    with ClockSampler(dev.index) as clocks:
        for i, (a, b) in enumerate(ev):
            flush.fill_(float(i))
            a.record()
            fwd()
            b.record()
        torch.cuda.synchronize()
    dist_util.barrier(world)
    torch.cuda.synchronize()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    kern = {name: hsa.hsa_timing_read(name) for name in hsa.KERNELS}
    hsa.hsa_timing_enable(False)
    assert hsa.hsa_device_status(ws) == 0, "device status set during the timed region"
    max_ms = dist_util.max_over_ranks(sum(step_ms), world, dev)
    value = dist_util.job_throughput(wl.B * wl.L, world, args.steps, max_ms)

    # dominant kernel: the chunk attention (whichever path ran)
    att_name = "attend_tc" if kern["attend_tc"][1] > 0 else "attend_simt"
    att_ms, att_n = kern[att_name]
    att_flops, sel_flops, comp_bytes = fwd_work(wl)
    peaks = load_peaks()
    achieved = att_flops / (att_ms / att_n / 1e3) / 1e12 if att_n else 0.0
    att_src = ("chunked_hierarchical_sparse_b200/csrc/k_attend_tc.cu" if att_name == "attend_tc"
               else "chunked_hierarchical_sparse_b200/csrc/k_attend_simt.cu")
    roof_us = max((att_flops + sel_flops) / (peaks["bf16_tflops"] * 1e12),
                  comp_bytes / (peaks["hbm_gbs"] * 1e9)) * 1e6
    roof_ds_us = max((att_flops + sel_flops) / (DATASHEET["bf16_tflops"] * 1e12),
                     comp_bytes / (DATASHEET["hbm_gbs"] * 1e9)) * 1e6
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": max_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": args.workload, "B": wl.B, "L": wl.L, "S": wl.S, "K": wl.K, "h_q": wl.h_q,
                   "h_kv": wl.h_kv, "d": wl.d, "global_batch": wl.B * world, "seq_len": wl.L,
                   "parallelism": f"dp{world} (independent sequences)",
                   "l2": "flushed (256 MB write) before every timed step"},
        "q_heads_per_s": value * wl.h_q,
        "roofline_fraction_step": roof_us / (max_ms / args.steps * 1e3),
        "roofline_step_us": roof_us,
        "roofline_fraction_step_datasheet": roof_ds_us / (max_ms / args.steps * 1e3),
        "roofline": {"bound": "tensor", "kernel": att_name, "achieved": achieved,
                     "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": achieved / peaks["bf16_tflops"],
                     "traffic": read_traffic(att_src),
                     "peak_source": f"{peaks['source']} bf16 dense (burst)",
                     "frac_of_datasheet": achieved / DATASHEET["bf16_tflops"],
                     "datasheet_peak": DATASHEET["bf16_tflops"],
                     "algorithmic_flops_per_launch": att_flops,
                     "avg_launch_us": 1e3 * att_ms / max(att_n, 1)},
        "kernel_us_per_step": {n: round(1e3 * ms / args.steps, 2) for n, (ms, c) in kern.items() if c},
        "gpu_launches": int(sum(c for _, c in kern.values())),
        "clocks": clocks.summary(),
    }

    # end to end through the public API: pinned host inputs -> device -> hsa_fwd -> host output,
    # as a pipeline over consecutive steps (two device buffer sets, three streams): step i's
    # upload, step i-1's forward and step i-2's read-back overlap, as a caller streaming
    # sequences through the library would run them.  Each step includes its own copies; the
    # value is the steps' tokens over the time from the first upload to the last read-back.
    hq = {n: torch.from_numpy(x[n]).to(torch.bfloat16).pin_memory() for n in ("q", "k", "v", "q_slc")}
    ho = [torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for _ in range(2)]
    sets = [dict(q=q, k=k, v=v, q_slc=qs, o=o, ws=ws)]
    sets.append({n: torch.empty_like(t_) for n, t_ in sets[0].items()})
    s_up, s_fw, s_dn = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    n_e2e = 12  # the pipeline's fill (first upload) and drain (last read-back) spread over 12 steps

    def pipeline(n):
        ev = lambda: torch.cuda.Event(enable_timing=True)
        up, fw, dn = [ev() for _ in range(n)], [ev() for _ in range(n)], [ev() for _ in range(n)]
        t0, t1 = ev(), ev()
        torch.cuda.synchronize()
        t0.record(s_up)
        for i in range(n):
            bs = sets[i % 2]
            with torch.cuda.stream(s_up):
                if i >= 2:
                    s_up.wait_event(fw[i - 2])  # the forward of step i - 2 no longer reads this set
                for name in ("q", "k", "v", "q_slc"):
                    bs[name].copy_(hq[name], non_blocking=True)
                up[i].record(s_up)
            with torch.cuda.stream(s_fw):
                s_fw.wait_event(up[i])
                if i >= 2:
                    s_fw.wait_event(dn[i - 2])  # step i - 2's output has been read back
                hsa.hsa_fwd(bs["q"], bs["k"], bs["v"], bs["q_slc"], wl.K, want_lse=False, want_sel=False,
                            o=bs["o"], ws=bs["ws"], stream=s_fw)
                fw[i].record(s_fw)
            with torch.cuda.stream(s_dn):
                s_dn.wait_event(fw[i])
                ho[i % 2].copy_(bs["o"], non_blocking=True)
                dn[i].record(s_dn)
        s_dn.wait_event(dn[n - 1])
        t1.record(s_dn)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1)

    pipeline(2)  # warm-up
    e2e_ms = pipeline(n_e2e)
    for st_ in sets:
        assert hsa.hsa_device_status(st_["ws"]) == 0, "device status set in the end-to-end run"
    h2d = sum(t_.numel() * t_.element_size() for t_ in hq.values())
    e2e_max = dist_util.max_over_ranks(e2e_ms, world, dev)
    line["e2e"] = {"value": dist_util.job_throughput(wl.B * wl.L, world, n_e2e, e2e_max), "unit": "tokens/s",
                   "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(ho[0].numel() * ho[0].element_size()),
                   "steps": n_e2e, "pipelined": "upload, forward and read-back of consecutive steps overlap"}
    del hq, ho, sets

    if not args.no_extras:
        line["decode"] = bench_decode(hsa, dev)
        line["decode_offload"] = bench_decode_offload(hsa, dev)
        line["train"] = bench_train(hsa, dev)
    if rank == 0 and world == 1 and not args.no_cpu:
        line["cpu_baseline"] = cpu_baseline(wl, x, args.cpu_budget_s)
    dist_util.finish(world)
    if rank == 0:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
