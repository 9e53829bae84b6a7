#!/usr/bin/env python
"""Benchmark of the KDA core on B200: chunkwise prefill tokens/s (headline) and the
decode step's state GB/s, each against the roofline, plus the fp64 oracle as the
CPU baseline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One JSON line on rank 0.  The headline workload is the bf16 prefill batch
B=4 x T=4096 tokens, H=32 heads, dk=dv=128, head-wise RMSNorm * sigmoid gate, fp32
final states.  A step is one kda_chunk_fwd call over that batch (every prefill row of
the path: staging, decay prep, decayed Gram blocks, UT inverse, W/U, state carry,
output and the fused epilogue).  The decode workload (N=512 sequences x H=32, fp32
states updated in place, 1,000 consecutive steps over a ring of 16 input sets) is
timed in its own loop and reported under "decode".  With N GPUs every rank runs its
own batch (different seed): weak scaling, no collective on the data path.
"""
from __future__ import annotations

import argparse
import ctypes
import datetime
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "KDA chunk-fwd tokens/s & TC util; decode-step state HBM GB/s vs peak"
UNIT = "tokens/s"
WORKLOAD = "prefill_bf16"
DECODE = "decode_bf16"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# Algorithmic bytes and useful FLOPs per head-token of the prefill (dk = dv = 128):
# q, k, v, g, gate, out at 256 B each plus beta 2 B; FLOPs 6 dk dv + C (3 dk + 2 dv) + C^2 / 3
# with C = 64 (the canonical chunk count, triangular products at half).
BYTES_PER_HEAD_TOKEN = 6 * 256 + 2
FLOPS_PER_HEAD_TOKEN = 6 * 128 * 128 + 64 * (3 * 128 + 2 * 128) + 64 * 64 // 3
STATE_BYTES = 128 * 128 * 4


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--decode-steps", type=int, default=1000)
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-snapshots", action="store_true")
    ap.add_argument("--no-preprocess", action="store_true")
    ap.add_argument("--no-unbounded", action="store_true")
    ap.add_argument("--no-varlen", action="store_true")
    ap.add_argument("--no-long", action="store_true")
    ap.add_argument("--long-tokens", type=int, default=1 << 20,
                    help="tokens of the long-context sequence (default 2^20, the full workload)")
    return ap.parse_args()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 20 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.path = None
        self.windows = []

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def mark(self, on: bool):
        self.windows.append((time.time(), on))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        if self.path and os.path.exists(self.path):
            with open(self.path) as f:
                for line in f:
                    parts = [x.strip() for x in line.split(",")]
                    if len(parts) >= 9:
                        rows.append(parts)
            os.unlink(self.path)
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        loaded = [s for s in sm if mx and s > 0.5 * max(mx)] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------ helpers
def kernel_traffic(kernel_tag: str, src_files):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on the current
    kernel source (sha1 of the listed files); else None."""
    h = hashlib.sha1()
    for fpath in src_files:
        with open(os.path.join(ROOT, fpath), "rb") as f:
            h.update(f.read())
    sha = h.hexdigest()[:12]
    prof = os.path.join(ROOT, "profiles", f"{kernel_tag}.md")
    if not os.path.exists(prof):
        return None, sha
    text = open(prof).read()
    m = re.search(r"traffic_bytes_per_launch:\s*([0-9]+)\s+source_sha1:\s*([0-9a-f]+)", text)
    if m and m.group(2) == sha:
        return int(m.group(1)), sha
    return None, sha


def gpu_uuid(dev):
    import torch
    props = torch.cuda.get_device_properties(dev)
    u = getattr(props, "uuid", None)
    return f"GPU-{u}" if u is not None else str(dev.index)


def dist_setup(n_gpus, backend="nccl"):
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    return rank, world, local


def max_over_ranks(x: float, world: int, device) -> float:
    """The slowest rank's time: every rank's number is reduced with MAX."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(base_seed: int, rank: int) -> int:
    """Each rank draws its own batch (weak scaling: the work per GPU is fixed)."""
    return base_seed + 1000 * rank


def whole_job_rate(world: int, units_per_rank_step: float, steps: int, max_ms: float) -> float:
    """Units processed by all ranks divided by the slowest rank's time."""
    return world * units_per_rank_step * steps / (max_ms / 1e3)


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------------------ oracle timing
def oracle_sample_tokens_per_s(inp, H, units, num_threads=0):
    """Time the fp64 oracle on the listed (n, h) units of `inp`; returns (tokens/s, seconds,
    head-tokens).  One token = one position over all H heads, as in the GPU metric."""
    import numpy as np
    import oracle
    cu = inp.cu_seqlens
    h = lambda t: t.float().cpu().numpy()
    parts = {n: [] for n in ("q", "k", "v", "g", "beta", "gate")}
    lens = []
    for n, hd in units:
        sl = slice(int(cu[n]), int(cu[n + 1]))
        for name in parts:
            parts[name].append(h(getattr(inp, name)[sl, hd:hd + 1]))
        lens.append(int(cu[n + 1] - cu[n]))
    a = {n: np.concatenate(v) for n, v in parts.items()}
    cuu = np.concatenate([[0], np.cumsum(lens)])
    t0 = time.perf_counter()
    oracle.forward(a["q"], a["k"], a["v"], a["g"], a["beta"], cu_seqlens=cuu, gate=a["gate"],
                   num_threads=num_threads, return_final_state=True)
    dt = time.perf_counter() - t0
    ht = int(cuu[-1])
    return ht / H / dt, dt, ht


def cpu_sample_units(B, H, cores):
    """The whole batch: the oracle takes about a second for all B x H units on a 16-core host,
    well inside the bounded CPU sample the benchmark allows."""
    return [(u // H, u % H) for u in range(B * H)]


# ------------------------------------------------------------------ reference arm
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    from linear_attention_serving_rule_b200 import synth
    oracle.build()
    cores = oracle.max_threads()
    w = synth.WORKLOADS[WORKLOAD]
    inp = synth.make_workload(WORKLOAD, device="cpu")
    units = cpu_sample_units(w["B"], w["H"], cores)
    rates, secs = [], []
    for i in range(args.warmup + args.steps):
        r, dt, ht = oracle_sample_tokens_per_s(inp, w["H"], units)
        if i >= args.warmup:
            rates.append(r)
            secs.append(dt)
    value = statistics.median(rates)
    sample = (f"{len(units)} (sequence, head) units x {w['T']} tokens of the B{w['B']} H{w['H']} "
              f"T{w['T']} d128 bf16 batch per step; fp64 oracle, OpenMP over units")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * statistics.median(secs),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": "KDA prefill bf16 B4 H32 T4096 dk=dv=128 (oracle sample)",
                       "global_batch": w["B"], "seq_len": w["T"], "heads": w["H"],
                       "parallelism": "host cores (OpenMP), rank 0 only"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ our arm
def run_ours(args):
    import numpy as np
    import torch

    import linear_attention_serving_rule_b200 as kda
    from linear_attention_serving_rule_b200 import binding as B
    from linear_attention_serving_rule_b200 import synth

    rank, world, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    kda.lib()
    L = kda.lib()
    peaks, peak_src = load_peaks()
    stream = torch.cuda.current_stream(dev)
    sptr = stream.cuda_stream

    # ---------------- prefill workload (own batch per rank)
    w = synth.WORKLOADS[WORKLOAD]
    inp = synth.make_workload(WORKLOAD, device=dev, seed=rank_seed(w["seed"], rank))
    Bq, T, H, dk, dv = w["B"], w["T"], w["H"], w["dk"], w["dv"]
    out = torch.empty_like(inp.v)
    fin = torch.empty((Bq, H, dk, dv), dtype=torch.float32, device=dev)
    a, keep = kda.make_chunk_args(inp.q, inp.k, inp.v, inp.g, inp.beta, gate=inp.gate,
                                  cu_seqlens=inp.cu_seqlens, out=out, final_state=fin)
    ws_bytes = kda.kda_chunk_fwd_workspace_size(a)
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device=dev)
    a.workspace, a.workspace_bytes = ws.data_ptr(), ws_bytes
    # 128 (sequence, head) units on 148 SMs: the automatic split only cuts sequences when the units
    # fill less than half the GPU, so this batch runs as one kernel per call
    launches_per_call = 1
    input_bytes = sum(t.numel() * t.element_size() for t in (inp.q, inp.k, inp.v, inp.g, inp.beta, inp.gate))

    def call():
        rc = L.kda_chunk_fwd(ctypes.byref(a), sptr)
        if rc != 0:
            raise B.KdaError(rc, "kda_chunk_fwd")

    clocks = ClockSampler(gpu_uuid(dev))
    clocks.start()
    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize(dev)
    st = kda.kda_read_device_error(ws)
    if st != 0:
        raise RuntimeError(f"device error in warm-up: {kda.kda_status_string(st)}")

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize(dev)
    g0.record(stream)
    for i in range(args.steps):
        ev[i][0].record(stream)
        call()
        ev[i][1].record(stream)
    g1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    elapsed_ms = g0.elapsed_time(g1)
    kern_ms = statistics.mean(e0.elapsed_time(e1) for e0, e1 in ev)
    elapsed_ms = max_over_ranks(elapsed_ms, world, dev)
    st = kda.kda_read_device_error(ws)
    if st != 0:
        raise RuntimeError(f"device error in timed region: {kda.kda_status_string(st)}")

    tokens_per_step = Bq * T
    value = whole_job_rate(world, tokens_per_step, args.steps, elapsed_ms)
    head_tokens = Bq * T * H
    alg_bytes = head_tokens * BYTES_PER_HEAD_TOKEN + Bq * H * STATE_BYTES  # final states written
    alg_flops = head_tokens * FLOPS_PER_HEAD_TOKEN
    achieved = alg_bytes / (kern_ms / 1e3) / 1e9
    tc_tflops = alg_flops / (kern_ms / 1e3) / 1e12
    traffic, sha = kernel_traffic("chunk_prefill_bf16", ["linear_attention_serving_rule_b200/csrc/kda_chunk_tc.cu",
                                                         "linear_attention_serving_rule_b200/csrc/kda_chunk_simt.cu"])
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "traffic": traffic,
                "peak_source": peak_src, "alg_bytes_per_launch": alg_bytes,
                "kernel_ms": kern_ms, "kernel_source_sha1": sha,
                "tc_util": {"useful_tflops": tc_tflops, "peak": peaks["bf16_tflops"],
                            "frac": tc_tflops / peaks["bf16_tflops"],
                            "useful_flops_per_launch": alg_flops}}

    # ---------------- the same launch writing chunk-boundary state snapshots (prefix caching)
    snaps = None
    if not args.no_snapshots:
        snaps = run_snapshots(args, L, a, sptr, stream, dev, ws, kern_ms, Bq, T, H, dk, dv)

    # ---------------- the same batch as raw projections, pre-processed inside the kernel
    prep = None
    if not args.no_preprocess:
        prep = run_preprocess(args, L, stream, dev, kern_ms, rank, w, peaks)

    # ---------------- what the decay bound buys: the batch with unbounded (negative-softplus) decay
    unb = None
    if not args.no_unbounded:
        unb = run_unbounded(args, L, stream, dev, kern_ms, rank, w)

    # ---------------- decode workload
    decode = None
    decode_multi = None
    if not args.no_decode:
        decode = run_decode(args, dev, stream, rank, world, peaks, peak_src, clocks)
        decode_multi = run_decode_multi(args, dev, stream, rank, peaks, decode["roofline"]["kernel_ms"])

    # ---------------- the varlen and long-context prefill workloads (their own legs)
    cpu_ok = rank == 0 and world == 1 and not args.no_cpu_baseline
    varlen = None
    if not args.no_varlen:
        varlen = run_varlen(args, L, stream, dev, rank, world, peaks, peak_src, cpu_ok)
    longctx = None
    if not args.no_long:
        longctx = run_long(args, L, stream, dev, rank, world, peaks, peak_src, cpu_ok)
    clocks.stop()
    clk = clocks.summary()

    # ---------------- end to end through the C ABI with host buffers (pinned)
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, inp, out, fin, a, L, sptr, stream, dev, world, Bq * T)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        oracle.build()
        cores = oracle.max_threads()
        units = cpu_sample_units(Bq, H, cores)
        r, dt, ht = oracle_sample_tokens_per_s(inp, H, units)
        cpu = {"value": r, "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": f"{len(units)} (sequence, head) units x {T} tokens of this batch "
                         f"({ht} head-tokens, {dt:.1f} s), fp64, OpenMP over units"}

    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "KDA prefill bf16 B4 H32 T4096 dk=dv=128, gate + RMSNorm, fp32 final states",
                       "global_batch": Bq * world, "seq_len": T, "heads": H, "dk": dk, "dv": dv,
                       "parallelism": f"dp{world} (independent batch per GPU)",
                       "l2": f"inputs {input_bytes / 2**20:.0f} MiB per step > 126 MiB L2; no flush"},
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": launches_per_call * args.steps, "clocks": clk, "decode": decode,
            "snapshots": snaps, "preprocess": prep, "decode_multi": decode_multi,
            "unbounded_decay": unb, "varlen": varlen, "long_context": longctx}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_snapshots(args, L, a, sptr, stream, dev, ws, base_ms, Bq, T, H, dk, dv, interval=1024):
    """The prefill launch with a state snapshot every `interval` tokens: kernel time and its
    overhead over the launch without snapshots (CUDA events on the launching stream)."""
    import torch
    import linear_attention_serving_rule_b200 as kda
    from linear_attention_serving_rule_b200 import binding as B
    rows = Bq * (T // interval)
    buf = torch.empty((rows, H, dk, dv), dtype=torch.float32, device=dev)
    a.snapshots, a.snapshot_interval = buf.data_ptr(), interval
    try:
        def call():
            rc = L.kda_chunk_fwd(ctypes.byref(a), sptr)
            if rc != 0:
                raise B.KdaError(rc, "kda_chunk_fwd")
        for _ in range(args.warmup):
            call()
        n = max(5, min(args.steps, 50))
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
        torch.cuda.synchronize(dev)
        for i in range(n):
            ev[i][0].record(stream)
            call()
            ev[i][1].record(stream)
        torch.cuda.synchronize(dev)
        st = kda.kda_read_device_error(ws)
        if st != 0:
            raise RuntimeError(f"device error with snapshots: {kda.kda_status_string(st)}")
        ms = statistics.mean(e0.elapsed_time(e1) for e0, e1 in ev)
    finally:
        a.snapshots, a.snapshot_interval = None, 0
    return {"interval": interval, "rows": rows, "launches": n, "kernel_ms": ms,
            "overhead_frac": ms / base_ms - 1.0,
            "snapshot_bytes_per_launch": rows * H * dk * dv * 4}


def run_preprocess(args, L, stream, dev, base_ms, rank, w, peaks):
    """The headline batch given as raw projections (unnormalised q, k; decay and beta logits)
    with KDA_FLAG_G_LOGITS | KDA_FLAG_BETA_LOGITS | KDA_FLAG_QK_L2NORM: kernel time, its overhead
    over the launch on pre-processed inputs, and the HBM bytes a separate pre-processing pass
    (read the raw q, k, g, beta; write them back) would move per step."""
    import torch
    import linear_attention_serving_rule_b200 as kda
    from linear_attention_serving_rule_b200 import binding as B
    from linear_attention_serving_rule_b200 import synth
    raw = synth.make_workload(WORKLOAD, device=dev, seed=rank_seed(w["seed"], rank), raw=True)
    flags = kda.KDA_FLAG_G_LOGITS | kda.KDA_FLAG_BETA_LOGITS | kda.KDA_FLAG_QK_L2NORM
    out = torch.empty_like(raw.v)
    fin = torch.empty((w["B"], w["H"], w["dk"], w["dv"]), dtype=torch.float32, device=dev)
    a, keep = kda.make_chunk_args(raw.q, raw.k, raw.v, raw.g, raw.beta, gate=raw.gate,
                                  cu_seqlens=raw.cu_seqlens, out=out, final_state=fin, flags=flags)
    nb = kda.kda_chunk_fwd_workspace_size(a)
    ws = torch.zeros(nb, dtype=torch.uint8, device=dev)
    a.workspace, a.workspace_bytes = ws.data_ptr(), nb
    sptr = stream.cuda_stream

    def call():
        rc = L.kda_chunk_fwd(ctypes.byref(a), sptr)
        if rc != 0:
            raise B.KdaError(rc, "kda_chunk_fwd")
    for _ in range(args.warmup):
        call()
    n = max(5, min(args.steps, 50))
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    torch.cuda.synchronize(dev)
    for i in range(n):
        ev[i][0].record(stream)
        call()
        ev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    st = kda.kda_read_device_error(ws)
    if st != 0:
        raise RuntimeError(f"device error with pre-processing: {kda.kda_status_string(st)}")
    ms = statistics.mean(e0.elapsed_time(e1) for e0, e1 in ev)
    del keep
    esz = raw.q.element_size()
    pass_bytes = 2 * sum(t.numel() * esz for t in (raw.q, raw.k, raw.g, raw.beta))
    return {"flags": "G_LOGITS|BETA_LOGITS|QK_L2NORM", "launches": n, "kernel_ms": ms,
            "overhead_frac": ms / base_ms - 1.0, "separate_pass_bytes_per_step": pass_bytes,
            "separate_pass_ms_at_peak": pass_bytes / (peaks["hbm_gbs"] * 1e9) * 1e3}


def run_e2e(args, inp, out, fin, a, L, sptr, stream, dev, world, tokens_per_step):
    """The headline step with its inputs in pinned host memory: every step copies all of its
    inputs to the device, runs kda_chunk_fwd through the C ABI and copies its outputs and final
    states back, all inside the timed region.  Steps are double-buffered the way a serving loop
    runs them: the host-to-device copies of step i + 1 (one stream), the kernel of step i (the
    compute stream) and the device-to-host copies of step i - 1 (a third stream) overlap, ordered
    by events so that no buffer is overwritten before the copy or kernel reading it is done."""
    import torch
    names = ("q", "k", "v", "g", "beta", "gate")
    dev_in = [[getattr(inp, n) for n in names]]
    dev_in.append([torch.empty_like(t) for t in dev_in[0]])
    dev_out = [(out, fin), (torch.empty_like(out), torch.empty_like(fin))]
    args_set = [a, type(a).from_buffer_copy(a)]
    a1 = args_set[1]
    a1.q, a1.k, a1.v, a1.g, a1.beta, a1.gate = (t.data_ptr() for t in dev_in[1])
    a1.out, a1.final_state = dev_out[1][0].data_ptr(), dev_out[1][1].data_ptr()
    host_in = []
    for t in dev_in[0]:
        hbuf = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
        hbuf.copy_(t)
        host_in.append(hbuf)
    host_out = [(torch.empty(out.shape, dtype=out.dtype, pin_memory=True),
                 torch.empty(fin.shape, dtype=fin.dtype, pin_memory=True)) for _ in range(2)]
    h2d = sum(h.numel() * h.element_size() for h in host_in)
    d2h = sum(x.numel() * x.element_size() for x in host_out[0])
    steps = max(1, min(args.steps, 20))
    s_h2d, s_d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: [torch.cuda.Event() for _ in range(2)]
    in_ready, k_done, out_copied = ev(), ev(), ev()
    used = [False, False]

    def step(i):
        b = i & 1
        with torch.cuda.stream(s_h2d):
            if used[b]:
                s_h2d.wait_event(k_done[b])  # the kernel two steps back has read set b
            for hbuf, dbuf in zip(host_in, dev_in[b]):
                dbuf.copy_(hbuf, non_blocking=True)
            in_ready[b].record(s_h2d)
        stream.wait_event(in_ready[b])
        if used[b]:
            stream.wait_event(out_copied[b])  # set b's outputs of two steps back are on the host
        rc = L.kda_chunk_fwd(ctypes.byref(args_set[b]), sptr)
        if rc != 0:
            raise RuntimeError(f"kda_chunk_fwd failed: {rc}")
        k_done[b].record(stream)
        with torch.cuda.stream(s_d2h):
            s_d2h.wait_event(k_done[b])
            host_out[b][0].copy_(dev_out[b][0], non_blocking=True)
            host_out[b][1].copy_(dev_out[b][1], non_blocking=True)
            out_copied[b].record(s_d2h)
        used[b] = True

    for i in range(2):
        step(i)
    torch.cuda.synchronize(dev)
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    s_h2d.wait_event(e0)
    s_d2h.wait_event(e0)
    for i in range(steps):
        step(i)
    stream.wait_stream(s_d2h)  # the last step's outputs are on the host before the end event
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    return {"value": world * tokens_per_step * steps / (ms / 1e3), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "ms_per_step": ms / steps, "pipelining": "double-buffered: H2D, kernel and D2H of consecutive steps overlap"}


def run_decode(args, dev, stream, rank, world, peaks, peak_src, clocks):
    import torch
    import linear_attention_serving_rule_b200 as kda
    from linear_attention_serving_rule_b200 import binding as B
    from linear_attention_serving_rule_b200 import synth
    w = synth.WORKLOADS[DECODE]
    N, H, dk, dv, ring = w["N"], w["H"], w["dk"], w["dv"], w["ring"]
    seed = rank_seed(w["seed"], rank)
    state = synth.make_states(slots=N, H=H, dk=dk, dv=dv, seed=seed, device=dev)
    toks = [synth.make_decode_token(N=N, H=H, dk=dk, dv=dv, seed=seed + 1 + i, device=dev)
            for i in range(ring)]
    out = torch.empty((N, H, dv), dtype=torch.bfloat16, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    L = kda.lib()
    args_ring = []
    for t in toks:
        d = B.KdaDecodeArgs()
        d.N, d.H, d.dk, d.dv, d.dtype = N, H, dk, dv, B.KDA_BF16
        d.q, d.k, d.v, d.g, d.beta, d.gate = (x.data_ptr() for x in (t.q, t.k, t.v, t.g, t.beta, t.gate))
        d.norm_weight = None
        d.state, d.num_slots, d.state_indices = state.data_ptr(), N, None
        d.out, d.scale, d.eps, d.flags, d.error_word = out.data_ptr(), 0.0, 1e-6, 0, err.data_ptr()
        args_ring.append(d)
    sptr = stream.cuda_stream
    steps = args.decode_steps
    for i in range(5):
        L.kda_decode_step(ctypes.byref(args_ring[i % ring]), sptr)
    torch.cuda.synchronize(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    barrier(world)
    torch.cuda.synchronize(dev)
    g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    g0.record(stream)
    for i in range(steps):
        ev[i][0].record(stream)
        rc = L.kda_decode_step(ctypes.byref(args_ring[i % ring]), sptr)
        ev[i][1].record(stream)
        if rc != 0:
            raise RuntimeError(f"kda_decode_step failed: {rc}")
    g1.record(stream)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(g0.elapsed_time(g1), world, dev)
    kern_ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    st = kda.kda_read_device_error(err)
    if st != 0:
        raise RuntimeError(f"decode device error: {kda.kda_status_string(st)}")
    state_bytes = 2 * N * H * dk * dv * 4
    achieved = state_bytes / (kern_ms / 1e3) / 1e9
    traffic, sha = kernel_traffic("decode_bf16", ["linear_attention_serving_rule_b200/csrc/kda_decode.cu"])
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = decode_cpu_baseline(state, toks, N, H, dk, dv, ring)
    return {"metric": "decode-step state HBM GB/s", "cpu_baseline": cpu,
            "workload": f"decode bf16 N{N} x H{H} dk=dv={dk}, "
            f"fp32 states in place, {steps} steps, ring of {ring} input sets",
            "value": world * state_bytes * steps / (ms / 1e3) / 1e9, "unit": "GB/s",
            "ms_per_step": ms / steps, "tokens_per_s": world * N * steps / (ms / 1e3),
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / peaks["hbm_gbs"], "traffic": traffic, "peak_source": peak_src,
                         "alg_bytes_per_launch": state_bytes, "kernel_ms": kern_ms,
                         "kernel_source_sha1": sha},
            "gpu_launches": steps}


def decode_cpu_baseline(state, toks, N, H, dk, dv, ring, n_seq=512, steps=32):
    """The fp64 oracle's decode step on a sample of the batch (n_seq sequences, all heads, `steps`
    consecutive steps over the same input ring), on the host cores: state GB/s in the GPU metric's
    unit (fp32 state bytes read + written per step) and tokens/s."""
    import numpy as np
    import oracle
    oracle.build()
    cores = oracle.max_threads()
    s64 = state[:n_seq].double().cpu().numpy()
    h = lambda t: t.float().cpu().numpy()
    sub = [{n: h(getattr(t, n)[:n_seq]) for n in ("q", "k", "v", "g", "beta", "gate")} for t in toks]
    t0 = time.perf_counter()
    for i in range(steps):
        a = sub[i % ring]
        oracle.decode_step(a["q"], a["k"], a["v"], a["g"], a["beta"], s64, gate=a["gate"])
    dt = time.perf_counter() - t0
    state_bytes = 2 * n_seq * H * dk * dv * 4 * steps
    return {"value": state_bytes / dt / 1e9, "unit": "GB/s", "tokens_per_s": n_seq * steps / dt,
            "cores": cores, "kind": "oracle",
            "sample": f"{n_seq} sequences x H{H} (all heads) x {steps} consecutive steps of this decode "
                      f"batch ({dt:.1f} s), fp64, OpenMP over (sequence, head) units"}


def _time_calls(call, n, warmup, stream, dev):
    """Mean CUDA-event time of `call` (ms) on `stream` after `warmup` untimed calls."""
    import torch
    for _ in range(warmup):
        call()
    torch.cuda.synchronize(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    for i in range(n):
        ev[i][0].record(stream)
        call()
        ev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    return statistics.mean(e0.elapsed_time(e1) for e0, e1 in ev)


def _prefill_leg(args, L, stream, dev, world, peaks, peak_src, inp, H, n_calls, warmup, label,
                 state_io_units, state_io_count):
    """Time kda_chunk_fwd on `inp` (inputs resident in HBM): tokens/s and the HBM roofline on the
    algorithmic bytes (1,538 B per head-token plus the fp32 states read and written)."""
    import torch
    import linear_attention_serving_rule_b200 as kda
    from linear_attention_serving_rule_b200 import binding as B
    out = torch.empty_like(inp.v)
    N = inp.num_seqs
    fin = torch.empty((N, H, 128, 128), dtype=torch.float32, device=dev)
    a, keep = kda.make_chunk_args(inp.q, inp.k, inp.v, inp.g, inp.beta, gate=inp.gate,
                                  cu_seqlens=inp.cu_seqlens, initial_state=inp.initial_state,
                                  out=out, final_state=fin)
    nb = kda.kda_chunk_fwd_workspace_size(a)
    ws = torch.zeros(nb, dtype=torch.uint8, device=dev)
    a.workspace, a.workspace_bytes = ws.data_ptr(), nb
    sptr = stream.cuda_stream

    def call():
        rc = L.kda_chunk_fwd(ctypes.byref(a), sptr)
        if rc != 0:
            raise B.KdaError(rc, "kda_chunk_fwd")
    barrier(world)
    ms = _time_calls(call, n_calls, warmup, stream, dev)
    ms = max_over_ranks(ms, world, dev)
    st = kda.kda_read_device_error(ws)
    if st != 0:
        raise RuntimeError(f"device error in the {label} leg: {kda.kda_status_string(st)}")
    del keep
    tokens = inp.total_tokens
    head_tokens = tokens * H
    alg_bytes = head_tokens * BYTES_PER_HEAD_TOKEN + state_io_count * state_io_units * STATE_BYTES
    achieved = alg_bytes / (ms / 1e3) / 1e9
    tc = head_tokens * FLOPS_PER_HEAD_TOKEN / (ms / 1e3) / 1e12
    return {"value": world * tokens / (ms / 1e3), "unit": UNIT, "tokens_per_call": tokens,
            "head_tokens": head_tokens, "calls": n_calls, "kernel_ms": ms, "workspace_bytes": nb,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / peaks["hbm_gbs"], "peak_source": peak_src,
                         "alg_bytes_per_call": alg_bytes,
                         "tc_util": {"useful_tflops": tc, "frac": tc / peaks["bf16_tflops"]}}}


def run_varlen(args, L, stream, dev, rank, world, peaks, peak_src, cpu_ok):
    """64 packed sequences of U[128, 8192] tokens, H32, fp32 initial states read and final states
    written: one kda_chunk_fwd call per step."""
    import numpy as np
    import torch
    from linear_attention_serving_rule_b200 import synth
    w = synth.WORKLOADS["varlen_bf16"]
    inp = synth.make_workload("varlen_bf16", device=dev, seed=rank_seed(w["seed"], rank))
    H = w["H"]
    N = inp.num_seqs
    res = _prefill_leg(args, L, stream, dev, world, peaks, peak_src, inp, H, n_calls=10, warmup=3,
                       label="varlen", state_io_units=N * H, state_io_count=2)
    lens = np.diff(inp.cu_seqlens)
    res["workload"] = (f"KDA varlen packed prefill bf16: {N} sequences, lengths U[128, 8192] "
                       f"({int(lens.min())}..{int(lens.max())}, {inp.total_tokens} tokens), H{H} d128, "
                       f"gate + RMSNorm, fp32 initial and final states")
    if cpu_ok:
        import oracle
        oracle.build()
        cores = oracle.max_threads()
        rng = np.random.default_rng(5)
        units = [(int(n), int(h)) for n, h in zip(rng.integers(N, size=512), rng.integers(H, size=512))]
        r, dt, ht = oracle_sample_tokens_per_s(inp, H, units)
        res["cpu_baseline"] = {"value": r, "unit": UNIT, "cores": cores, "kind": "oracle",
                               "sample": f"{len(units)} random (sequence, head) units of this batch "
                                         f"({ht} head-tokens, {dt:.1f} s), fp64, OpenMP over units"}
    del inp
    torch.cuda.empty_cache()
    return res


def run_long(args, L, stream, dev, rank, world, peaks, peak_src, cpu_ok):
    """One 2^20-token sequence, H16: 16 units for 148 SMs, so the library splits the sequence
    (pass 1 per segment, the combine, pass 2); one kda_chunk_fwd call per step."""
    import numpy as np
    import torch
    from linear_attention_serving_rule_b200 import synth
    w = synth.WORKLOADS["long_bf16"]
    T = int(args.long_tokens)
    inp = synth.make_workload("long_bf16", device=dev, seed=rank_seed(w["seed"], rank), T=T)
    H = w["H"]
    res = _prefill_leg(args, L, stream, dev, world, peaks, peak_src, inp, H, n_calls=3, warmup=1,
                       label="long-context", state_io_units=H, state_io_count=1)
    res["workload"] = (f"KDA long-context prefill bf16: B1 H{H} T={T} d128, gate + RMSNorm, zero initial "
                       f"state, fp32 final state; automatic sequence split")
    if cpu_ok:
        import oracle
        oracle.build()
        cores = oracle.max_threads()
        P = min(T, 65536)
        pre = synth.PrefillInputs(inp.q[:P], inp.k[:P], inp.v[:P], inp.g[:P], inp.beta[:P], inp.gate[:P],
                                  None, np.array([0, P]))
        units = [(0, h) for h in range(H)]
        r, dt, ht = oracle_sample_tokens_per_s(pre, H, units)
        res["cpu_baseline"] = {"value": r, "unit": UNIT, "cores": cores, "kind": "oracle",
                               "sample": f"the first {P} tokens of all {H} heads ({ht} head-tokens, "
                                         f"{dt:.1f} s), fp64, OpenMP over the {H} heads"}
    del inp
    torch.cuda.empty_cache()
    return res


def run_unbounded(args, L, stream, dev, bounded_ms, rank, w):
    """The headline batch with g = -softplus(a) (no lower bound) through KDA_FLAG_UNBOUNDED_DECAY:
    the exact fp32 path with pairwise Gram blocks.  Its time over the bounded tensor-core launch
    is what the g >= -5 bound buys."""
    import torch
    import linear_attention_serving_rule_b200 as kda
    from linear_attention_serving_rule_b200 import binding as B
    from linear_attention_serving_rule_b200 import synth
    inp = synth.make_workload(WORKLOAD, device=dev, seed=rank_seed(w["seed"], rank), decay="softplus")
    out = torch.empty_like(inp.v)
    fin = torch.empty((w["B"], w["H"], w["dk"], w["dv"]), dtype=torch.float32, device=dev)
    a, keep = kda.make_chunk_args(inp.q, inp.k, inp.v, inp.g, inp.beta, gate=inp.gate,
                                  cu_seqlens=inp.cu_seqlens, out=out, final_state=fin,
                                  flags=kda.KDA_FLAG_UNBOUNDED_DECAY)
    nb = kda.kda_chunk_fwd_workspace_size(a)
    ws = torch.zeros(nb, dtype=torch.uint8, device=dev)
    a.workspace, a.workspace_bytes = ws.data_ptr(), nb
    sptr = stream.cuda_stream

    def call():
        rc = L.kda_chunk_fwd(ctypes.byref(a), sptr)
        if rc != 0:
            raise B.KdaError(rc, "kda_chunk_fwd")
    call()
    n = 3
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    torch.cuda.synchronize(dev)
    for i in range(n):
        ev[i][0].record(stream)
        call()
        ev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    st = kda.kda_read_device_error(ws)
    if st != 0:
        raise RuntimeError(f"device error on the unbounded path: {kda.kda_status_string(st)}")
    ms = statistics.mean(e0.elapsed_time(e1) for e0, e1 in ev)
    del keep
    return {"decay": "g = -softplus(a), a ~ N(0,1)", "path": "fp32 CUDA cores, pairwise Gram blocks",
            "launches": n, "kernel_ms": ms, "bounded_kernel_ms": bounded_ms,
            "speedup_of_bound": ms / bounded_ms}


def run_decode_multi(args, dev, stream, rank, peaks, single_ms, K=4):
    """The decode batch verifying K draft tokens per sequence in one call (state read once and
    written once): kernel time, tokens/s and state GB/s, and the per-token cost against K
    single-token steps."""
    import numpy as np
    import torch
    import linear_attention_serving_rule_b200 as kda
    from linear_attention_serving_rule_b200 import synth
    w = synth.WORKLOADS[DECODE]
    N, H, dk, dv = w["N"], w["H"], w["dk"], w["dv"]
    seed = rank_seed(w["seed"], rank) + 100
    state = synth.make_states(slots=N, H=H, dk=dk, dv=dv, seed=seed, device=dev)
    p = synth.make_prefill(H=H, dk=dk, dv=dv, dtype="bf16", seed=seed + 1, device=dev,
                           lengths=np.full(N, K, dtype=np.int64), gate=True)
    t = [getattr(p, n).reshape((N, K) + tuple(getattr(p, n).shape[1:])).contiguous()
         for n in ("q", "k", "v", "g", "beta", "gate")]
    out = torch.empty((N, K, H, dv), dtype=torch.bfloat16, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)

    def call():
        kda.kda_decode_step(*t[:5], state, gate=t[5], out=out, error_word=err, stream=stream)
    for _ in range(5):
        call()
    n = 50
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    torch.cuda.synchronize(dev)
    for i in range(n):
        ev[i][0].record(stream)
        call()
        ev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    st = kda.kda_read_device_error(err)
    if st != 0:
        raise RuntimeError(f"multi-token decode device error: {kda.kda_status_string(st)}")
    ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    state_bytes = 2 * N * H * dk * dv * 4
    return {"workload": f"decode bf16 N{N} x H{H} dk=dv={dk}, K={K} tokens per sequence per call",
            "tokens_per_call": K, "launches": n, "kernel_ms": ms, "tokens_per_s": N * K / (ms / 1e3),
            "state_gbs": state_bytes / (ms / 1e3) / 1e9,
            "state_frac_of_peak": state_bytes / (ms / 1e3) / 1e9 / peaks["hbm_gbs"],
            "ms_per_token_vs_single_step": ms / K / single_ms}


def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
