#!/usr/bin/env python
"""Benchmark of the KDA hot path on B200: chunked prefill + decode step, one JSON line.

A step is one pass of the whole hot path over one batch of synthetic input:
  * prefill: kda_forward_chunked over the K3-shaped workload B=4, T=8192, H=96,
    dk=dv=128, bf16 inputs, fp32 state (S0 ~ N(0, 0.02^2), decay logits z ~ N(-2, 1));
  * decode: one kda_decode_step over 256 sequences x 96 heads of 128x128 fp32 states,
    updated in place (fresh bf16 token each step, from a ring of pre-drawn inputs).
`value` is prefill tokens/s (B*T per prefill / device time of the prefill launches,
summed over ranks for N > 1: weak scaling, every rank runs its own batch, no collective
on the data path).  Decode states/s, the roofline of each kernel, the end-to-end figure
through the public API with host buffers, the oracle's CPU baseline and the clocks seen
during the timed region are reported in the same line.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "KDA prefill tokens/s (K3 shape, H=96, d=128) and decode states/s; % of roofline"
PREFILL = dict(name="k3_b4_t8k", B=4, T=8192, H=96, dk=128, dv=128, dtype="bf16", s0_std=0.02, zg_mean=-2.0)
DECODE = dict(name="decode_b256_h96", batch=256, H=96, dk=128, dv=128, dtype="bf16")
LONG = dict(name="k3_t64k", B=1, T=65536, H=96, dk=128, dv=128, dtype="bf16")
# the recorded ncu traffic (profiles/) is per launch of these two workloads
DEFAULT_PREFILL_NAME, DEFAULT_DECODE_NAME = PREFILL["name"], DECODE["name"]
DECODE_RING = 8


def prefill_alg_bytes(B, T, H, dk, dv, elem=2, with_s0=True, with_st=True):
    """Algorithmic HBM bytes of one prefill launch: every input read once, every output written once."""
    per_token_head = elem * (3 * dk + dv) + elem + elem * dv   # q, k, g, v, beta in; o out
    per_head = 4 * dk * dv * (int(with_s0) + int(with_st))        # S0 in, S_T out (fp32)
    return B * T * H * per_token_head + B * H * per_head


def decode_alg_bytes(batch, H, dk, dv, elem=2):
    """Per step: the fp32 state read and written once, plus the token's inputs and o."""
    return batch * H * (2 * 4 * dk * dv + elem * (3 * dk + dv) + elem + elem * dv)


# Contraction work of the chunked prefill per token-head (d = 128, chunk 64): the three state
# products at 2 d^2 each, plus five 64 x 64 x d products counted causally (half) or as whole tiles.
PREFILL_FLOP_CAUSAL = 6 * 128 * 128 + 5 * 64 * 128
PREFILL_FLOP_DENSE = 6 * 128 * 128 + 10 * 64 * 128


def measured_bf16_tflops():
    """Measured dense bf16 tensor throughput (burst), or the fallback figure."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        if "bf16_tflops" in d:
            return float(d["bf16_tflops"]), "measured"
    return 1590.0, "fallback"


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


KERNEL_SOURCES = {
    "prefill_tc": ("kda_prefill_tc.cu", "sm100_ptx.cuh", "kda_internal.cuh"),
    "prefill_simt": ("kda_prefill_simt.cu", "kda_internal.cuh"),
    "decode": ("kda_decode.cu", "kda_internal.cuh"),
}


def kernel_source_sha(kernel_tag):
    """Short hash of the source files a kernel is built from (a recorded ncu figure is valid only
    while they are unchanged)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "linear_attention_recurrence_forward_b200", "csrc")
    for name in KERNEL_SOURCES[kernel_tag]:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel_tag):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on the current sources."""
    prof = os.path.join(ROOT, "profiles")
    if not os.path.isdir(prof):
        return None
    sha = kernel_source_sha(kernel_tag)
    for name in sorted(os.listdir(prof)):
        if not name.endswith(".md"):
            continue
        text = open(os.path.join(prof, name)).read()
        m = re.search(r"traffic_record:\s*kernel=(\S+)\s+sources=(\S+)\s+dram_bytes_per_launch=(\d+)", text)
        if m and m.group(1) == kernel_tag and m.group(2) == sha:
            return int(m.group(3))
    return None


def measure_long_split(kda, LC, lq, lo, lst, stream, reps, l_ms):
    """The long-context workload cut at T/2 the way context parallelism cuts it over ranks, all on one
    GPU: one launch of 3 x B*H half-length runs (the first halves from S0 = 0; the second halves from
    a zero state; the second halves with v = 0 and S0 = I, whose outputs are the correction operands
    and whose final states are the state maps), then the incoming state's composition and the
    output correction.  Measured to show whether filling the idle SMs this way pays."""
    import torch

    B, T, H, dk, dv = LC["B"], LC["T"], LC["H"], LC["dk"], LC["dv"]
    h = T // 2
    q, k, v, g, beta = lq[:5]
    cat = lambda x, y, z: torch.cat([x, y, z], 0).contiguous()
    q3 = cat(q[:, :h], q[:, h:], q[:, h:])
    k3 = cat(k[:, :h], k[:, h:], k[:, h:])
    g3 = cat(g[:, :h], g[:, h:], g[:, h:])
    b3 = cat(beta[:, :h], beta[:, h:], beta[:, h:])
    v3 = cat(v[:, :h], v[:, h:], torch.zeros_like(v[:, h:]))
    S03 = torch.zeros((3 * B, H, dk, dv), dtype=torch.float32, device=q.device)
    S03[2 * B:] = torch.eye(dk, dtype=torch.float32, device=q.device)
    o3 = torch.empty((3 * B, h, H, dv), dtype=q.dtype, device=q.device)
    st3 = torch.empty((3 * B, H, dk, dv), dtype=torch.float32, device=q.device)
    final = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)

    def step(whole):
        kda.kda_forward_chunked(q3, k3, v3, g3, b3, S03, o=o3, S_T=st3, stream=stream)
        if whole:   # S_in = N of the first half (it started from 0); o2 += S_in^T C; S_T = M2 S_in + N2
            kda.kda_output_correct(o3[2 * B:], st3[:B], o3[B:2 * B], out=o3[B:2 * B], stream=stream)
            kda.kda_state_compose(st3[2 * B:], st3[:B], st3[B:2 * B], out=final, stream=stream)

    times = {}
    for whole in (False, True):
        step(whole)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        torch.cuda.synchronize()
        for e0, e1 in ev:
            e0.record(stream)
            step(whole)
            e1.record(stream)
        torch.cuda.synchronize()
        times[whole] = sum(e0.elapsed_time(e1) for e0, e1 in ev) / reps
    if kda.kda_get_device_status() != 0:
        raise RuntimeError("device status after the split long-context run")
    o_split = torch.cat([o3[:B], o3[B:2 * B]], 1).float()
    ref = lo.float()
    rel = lambda x, r: float((x - r).abs().max() / r.abs().max())
    out = {"segments": 2, "ctas": 3 * B * H, "forward_ms": times[False],
           "correct_and_compose_ms": times[True] - times[False], "total_ms": times[True],
           "vs_single_pass": times[True] / l_ms,
           "o_first_half_bitwise_equal": bool(torch.equal(o3[:B], lo[:, :h])),
           "max_rel_diff_o_vs_single_pass": rel(o_split, ref),
           "max_rel_diff_state_vs_single_pass": rel(final, lst)}
    del q3, k3, g3, b3, v3, S03, o3, st3, final, o_split, ref
    return out


def measure_batching(kda, dev, stream, rank, args, H=96, d=128, nseq=64, max_len=2048, batch=256, n_slots=512):
    """Continuous batching, the paged / variable-length row: (1) one packed prefill over 64 sequences
    whose lengths are drawn uniformly from 1..2048 (seeded), H = 96, d = 128, each from its own S0;
    (2) the decode step with the 256 x 96 states in a pool of 512 slots, the sequences on a random
    permutation of slots.  CUDA events per launch, the same algorithmic byte counts as the dense
    workloads (tokens x heads x 1282 B plus 128 KiB of S0/S_T per sequence-head; 132,354 B per
    head-step)."""
    import torch
    from linear_attention_recurrence_forward_b200.inputs import make_prefill_inputs, make_decode_inputs

    gen = torch.Generator()
    gen.manual_seed(5000 + rank)
    lengths = torch.randint(1, max_len + 1, (nseq,), generator=gen)
    cu = torch.zeros(nseq + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(lengths, 0).to(torch.int32)
    total = int(cu[-1])
    q, k, v, g, beta, S0 = make_prefill_inputs(1, total, H, d, d, "bf16", seed=5000 + rank, s0_std=0.02,
                                               zg_mean=-2.0, device=str(dev))
    q, k, v, g, beta = (x[0].contiguous() for x in (q, k, v, g, beta))
    S0n = (torch.randn((nseq, H, d, d), generator=gen) * 0.02).to(dev)
    cu_d = cu.to(dev)
    o = torch.empty((total, H, d), dtype=q.dtype, device=dev)
    ST = torch.empty((nseq, H, d, d), dtype=torch.float32, device=dev)
    reps = max(3, min(args.steps, 10))

    def timed(fn):
        for _ in range(2):
            fn()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        torch.cuda.synchronize()
        for e0, e1 in ev:
            e0.record(stream)
            fn()
            e1.record(stream)
        torch.cuda.synchronize()
        if kda.kda_get_device_status() != 0:
            raise RuntimeError("device status after a continuous-batching run")
        return sum(e0.elapsed_time(e1) for e0, e1 in ev) / reps

    peak, peak_kind = measured_peaks()
    p_ms = timed(lambda: kda.kda_forward_varlen(q, k, v, g, beta, cu_d, S0n, o=o, S_T=ST, stream=stream))
    p_bytes = total * H * (2 * (3 * d + d) + 2 + 2 * d) + nseq * H * 2 * d * d * 4   # 1282 B per token-head at d = 128
    packed = {"sequences": nseq, "tokens": total, "H": H, "lengths": f"uniform on 1..{max_len} (seeded)",
              "longest": int(lengths.max()), "launch_ms": p_ms, "tokens_per_s": total / (p_ms / 1e3),
              "roofline": {"bound": "hbm", "achieved": p_bytes / (p_ms / 1e3) / 1e9, "peak": peak, "unit": "GB/s",
                           "frac": p_bytes / (p_ms / 1e3) / 1e9 / peak, "alg_bytes_per_launch": p_bytes,
                           "peak_kind": peak_kind},
              "grid": f"{nseq * H} CTAs (one per sequence and head)"}
    del q, k, v, g, beta, S0, S0n, o, ST

    B = batch
    perm = torch.randperm(n_slots, generator=gen)[:B].to(torch.int32).to(dev)
    pool = torch.zeros((n_slots, H, d, d), dtype=torch.float32, device=dev)
    ring = [make_decode_inputs(B, H, d, d, "bf16", gen=None, seed=6000 + i, device=str(dev))[:5] for i in range(4)]
    step = [0]

    def paged():
        kda.kda_decode_step_paged(*ring[step[0] % 4], pool, perm, stream=stream)
        step[0] += 1

    d_ms = timed(paged)
    d_bytes = decode_alg_bytes(B, H, d, d)
    paged_line = {"sequences": B, "slots": n_slots, "ms_per_step": d_ms, "states_per_s": B * H / (d_ms / 1e3),
                  "roofline": {"bound": "hbm", "achieved": d_bytes / (d_ms / 1e3) / 1e9, "peak": peak,
                               "unit": "GB/s", "frac": d_bytes / (d_ms / 1e3) / 1e9 / peak,
                               "alg_bytes_per_launch": d_bytes, "peak_kind": peak_kind}}
    del pool, ring
    return {"packed_prefill": packed, "paged_decode": paged_line,
            "timed": "separately, after the headline region, CUDA events per launch"}


class ClockSampler:
    """nvidia-smi clocks/throttle reasons sampled every 200 ms during the timed region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu_index = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"kda_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu_index}", f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, ValueError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        sms, maxes, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sms.append(float(parts[1])); maxes.append(float(parts[2]))
            except ValueError:
                continue
            for n, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sms) if sms else None, "sm_max_mhz": max(maxes) if maxes else None,
                "reasons": sorted(reasons), "samples": len(sms)}


def cpu_model():
    """The host CPU's model name (Linux), or None."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def oracle_baseline(budget_s=15.0, seed=0):
    """Time the fp64 oracle (as it stands) on a bounded sample of the prefill workload.

    The sample is n_heads full-length heads of the K3 workload (T = 8192, d = 128); the
    result is scaled to the metric's unit: tokens/s = (token-heads/s) / H.
    """
    import torch
    import oracle
    from linear_attention_recurrence_forward_b200.inputs import make_prefill_inputs
    cores = len(os.sched_getaffinity(0))
    T, H, d = PREFILL["T"], PREFILL["H"], PREFILL["dk"]
    # calibrate on one short head
    cal = make_prefill_inputs(1, 512, 1, d, d, "bf16", seed=seed + 1, zg_mean=PREFILL["zg_mean"])
    t0 = time.perf_counter()
    oracle.forward(*cal[:5], None, nthreads=1)
    per_token_head = (time.perf_counter() - t0) / 512
    n_heads = max(cores, int(budget_s * cores / (per_token_head * T)))
    n_heads = max(cores, (n_heads // cores) * cores)
    n_heads = min(n_heads, 4 * 96)
    q, k, v, g, beta, S0 = make_prefill_inputs(1, T, n_heads, d, d, "bf16", seed=seed, s0_std=0.02,
                                               zg_mean=PREFILL["zg_mean"])
    t0 = time.perf_counter()
    oracle.forward(q, k, v, g, beta, S0, nthreads=cores)
    dt = time.perf_counter() - t0
    token_heads_per_s = n_heads * T / dt
    # one thread on one head of the 4096-token, 32-head workload
    T1, H1 = 4096, 32
    one = make_prefill_inputs(1, T1, 1, d, d, "bf16", seed=seed + 2)
    t1 = time.perf_counter()
    oracle.forward(*one[:5], None, nthreads=1)
    dt1 = time.perf_counter() - t1
    return {"value": token_heads_per_s / H, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{n_heads} heads x {T} tokens of the K3 prefill workload (d=128), fp64, {dt:.1f} s; "
                      f"tokens/s = token-heads/s / {H}",
            "cpu_model": cpu_model(),
            "single_thread": {"value": T1 / dt1 / H1, "unit": "tokens/s", "threads": 1,
                              "sample": f"1 head x {T1} tokens of the h32_t4k workload (B1 T4096 H32 d128), "
                                        f"fp64, {dt1:.2f} s; tokens/s = token-heads/s / {H1}"},
            "seconds": dt, "token_heads_per_s": token_heads_per_s}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    per_step = []
    base = None
    for i in range(args.warmup + args.steps):
        r = oracle_baseline(budget_s=8.0, seed=i)
        if i >= args.warmup:
            per_step.append(r)
        base = r
    value = statistics.mean(r["value"] for r in per_step)
    secs = statistics.mean(r["seconds"] for r in per_step)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": PREFILL["name"], "B": PREFILL["B"], "T": PREFILL["T"], "H": PREFILL["H"],
                       "dk": PREFILL["dk"], "dv": PREFILL["dv"]},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": base["cores"], "kind": "oracle",
                             "sample": base["sample"], "cpu_model": base["cpu_model"],
                             "single_thread": base["single_thread"]},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def max_over_ranks(values, device, world):
    """Element-wise max of per-rank timings (every rank gets the result); identity for one rank."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def weak_scaling_throughput(units_per_rank, world, steps, seconds):
    """Whole-job throughput: every rank processed units_per_rank per step; time is the max over ranks."""
    return world * units_per_rank * steps / seconds


def measure_e2e(kda, dist, world, dev, stream, args, q, k, v, g, beta, S0, o):
    """Prefill through the host-buffer entry point, per step: pinned host inputs and S0 copied in,
    o copied out (the library overlaps copy-in, kernels and copy-out segment by segment)."""
    import torch
    P = PREFILL
    host_in = [t.to("cpu").pin_memory() for t in (q, k, v, g, beta)]
    host_s0 = S0.to("cpu").pin_memory()
    host_o = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    ws = torch.empty(kda.host_workspace_bytes(P["T"], P["H"], P["dk"], P["dv"], q.dtype), dtype=torch.uint8,
                     device=dev)
    e2e_steps = max(1, min(args.steps, 3))

    def step():
        kda.kda_forward_chunked_host(*host_in, host_s0, o=host_o, return_state=False, workspace=ws, stream=stream)

    step()   # untimed: first touch of the workspace
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    (e2e_ms,) = max_over_ranks([e0.elapsed_time(e1) / e2e_steps], dev, world)
    h2d = sum(t.numel() * t.element_size() for t in host_in) + host_s0.numel() * 4
    d2h = host_o.numel() * host_o.element_size()
    return {"value": weak_scaling_throughput(P["B"] * P["T"], world, 1, e2e_ms / 1e3), "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "note": "prefill through kda_forward_chunked_host: pinned host inputs and S0 in, o out, "
                    "copies overlapped with the kernels in 2048-token segments"}


def run_ours(args):
    import torch
    import torch.distributed as dist
    import linear_attention_recurrence_forward_b200 as kda
    from linear_attention_recurrence_forward_b200.inputs import make_prefill_inputs, make_decode_inputs, fingerprint

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local_rank)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local_rank))
    dev = torch.device("cuda", local_rank)

    P = PREFILL
    q, k, v, g, beta, S0 = make_prefill_inputs(P["B"], P["T"], P["H"], P["dk"], P["dv"], P["dtype"],
                                               seed=1000 + rank, s0_std=P["s0_std"], zg_mean=P["zg_mean"],
                                               device=str(dev))
    o = torch.empty((P["B"], P["T"], P["H"], P["dv"]), dtype=q.dtype, device=dev)
    ST = torch.empty((P["B"], P["H"], P["dk"], P["dv"]), dtype=torch.float32, device=dev)
    D = DECODE
    gen = torch.Generator(device=str(dev))
    gen.manual_seed(2000 + rank)
    ring = [make_decode_inputs(D["batch"], D["H"], D["dk"], D["dv"], D["dtype"], gen=gen, device=str(dev))
            for _ in range(DECODE_RING)]
    S = torch.zeros((D["batch"], D["H"], D["dk"], D["dv"]), dtype=torch.float32, device=dev)
    od = torch.empty((D["batch"], D["H"], D["dv"]), dtype=q.dtype, device=dev)
    stream = torch.cuda.current_stream()
    # the exact input bytes of this rank's workloads (before any timing)
    inputs_sha256 = {"prefill": fingerprint(q, k, v, g, beta, S0),
                     "decode_ring": fingerprint(*[t for r in ring for t in r])}

    nvtx = torch.cuda.nvtx   # ranges for profilers (ncu --nvtx); no-ops otherwise

    def step(i, ev=None):
        if ev is not None:
            ev[0].record(stream)
        nvtx.range_push("kda.prefill")
        kda.kda_forward_chunked(q, k, v, g, beta, S0, o=o, S_T=ST, stream=stream)
        nvtx.range_pop()
        if ev is not None:
            ev[1].record(stream)
        x = ring[i % DECODE_RING]
        nvtx.range_push("kda.decode")
        kda.kda_decode_step(*x, S, o=od, stream=stream)
        nvtx.range_pop()
        if ev is not None:
            ev[2].record(stream)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    status = kda.kda_get_device_status()
    if status != 0:
        raise RuntimeError(f"device status after warm-up: {kda.kda_status_string(status)}")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    visible = os.environ.get("CUDA_VISIBLE_DEVICES")
    sampler = ClockSampler(visible.split(",")[local_rank].strip() if visible else str(local_rank))
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    t_start.record(stream)
    for i in range(args.steps):
        step(i, evs[i])
    t_end.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if world > 1:
        dist.barrier()
    status = kda.kda_get_device_status()
    if status != 0:
        raise RuntimeError(f"device status after timing: {kda.kda_status_string(status)}")

    total_ms = t_start.elapsed_time(t_end)
    prefill_ms = [e[0].elapsed_time(e[1]) for e in evs]
    decode_ms = [e[1].elapsed_time(e[2]) for e in evs]
    total_ms, prefill_sum, decode_sum = max_over_ranks([total_ms, sum(prefill_ms), sum(decode_ms)], dev, world)

    # ---- the same prefill writing the state every 512 tokens (prefix-cache boundaries), timed alone
    states_line = None
    if not args.no_states:
        interval = 512
        n_mid = P["T"] // interval
        S_mid = torch.empty((P["B"], P["H"], n_mid, P["dk"], P["dv"]), dtype=torch.float32, device=dev)
        for _ in range(2):
            kda.kda_forward_chunked_states(q, k, v, g, beta, S0, interval=interval, o=o, S_T=ST, S_mid=S_mid,
                                           stream=stream)
        reps = max(3, min(args.steps, 10))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(reps):
            kda.kda_forward_chunked_states(q, k, v, g, beta, S0, interval=interval, o=o, S_T=ST, S_mid=S_mid,
                                           stream=stream)
        e1.record(stream)
        torch.cuda.synchronize()
        if kda.kda_get_device_status() != 0:
            raise RuntimeError("device status after the state-emission run")
        st_ms = e0.elapsed_time(e1) / reps
        extra = P["B"] * P["H"] * n_mid * P["dk"] * P["dv"] * 4
        st_bytes = prefill_alg_bytes(P["B"], P["T"], P["H"], P["dk"], P["dv"]) + extra
        states_line = {"interval": interval, "states_per_head": n_mid, "launch_ms": st_ms,
                       "tokens_per_s": P["B"] * P["T"] / (st_ms / 1e3), "extra_bytes": extra,
                       "achieved_gbs": st_bytes / (st_ms / 1e3) / 1e9, "launches": reps,
                       "timed": "separately, after the headline region (rank 0's own device)"}
        del S_mid

    # ---- the same prefill with the gate / normalisation prologue in the kernel, on raw inputs
    fused_line = None
    if not args.no_states:
        from linear_attention_recurrence_forward_b200.inputs import make_prefill_raw_inputs
        raw = make_prefill_raw_inputs(P["B"], P["T"], P["H"], P["dk"], P["dv"], P["dtype"], seed=3000 + rank,
                                      s0_std=P["s0_std"], zg_mean=P["zg_mean"], device=str(dev))
        for _ in range(2):
            kda.kda_forward_chunked_fused(*raw[:5], raw[5], o=o, S_T=ST, stream=stream)
        reps = max(3, min(args.steps, 10))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(reps):
            kda.kda_forward_chunked_fused(*raw[:5], raw[5], o=o, S_T=ST, stream=stream)
        e1.record(stream)
        torch.cuda.synchronize()
        if kda.kda_get_device_status() != 0:
            raise RuntimeError("device status after the prologue-fused run")
        f_ms = e0.elapsed_time(e1) / reps
        fb = prefill_alg_bytes(P["B"], P["T"], P["H"], P["dk"], P["dv"])
        fused_line = {"launch_ms": f_ms, "tokens_per_s": P["B"] * P["T"] / (f_ms / 1e3),
                      "achieved_gbs": fb / (f_ms / 1e3) / 1e9, "launches": reps,
                      "note": "raw q, k and gate logits in; g, beta and the q/k norms formed in the kernel "
                              "(an unfused pipeline also reads and writes them once more in a separate pass)"}
        del raw

    # ---- continuous batching: packed prefill of mixed lengths and the paged decode step, timed alone
    batching_line = None if args.no_batching else measure_batching(kda, dev, stream, rank, args)

    # ---- the long-context workload (B1 T65536 H96, S0 = 0, 1024 chunks carried in sequence), timed alone
    long_line = None
    if not args.no_long:
        LC = LONG
        lq = make_prefill_inputs(LC["B"], LC["T"], LC["H"], LC["dk"], LC["dv"], LC["dtype"], seed=4000 + rank,
                                 device=str(dev))
        lo = torch.empty((LC["B"], LC["T"], LC["H"], LC["dv"]), dtype=lq[0].dtype, device=dev)
        lst = torch.empty((LC["B"], LC["H"], LC["dk"], LC["dv"]), dtype=torch.float32, device=dev)
        for _ in range(2):
            kda.kda_forward_chunked(*lq[:5], None, o=lo, S_T=lst, stream=stream)
        reps = max(3, min(args.steps, 10))
        lev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        torch.cuda.synchronize()
        for e0, e1 in lev:
            e0.record(stream)
            kda.kda_forward_chunked(*lq[:5], None, o=lo, S_T=lst, stream=stream)
            e1.record(stream)
        torch.cuda.synchronize()
        if kda.kda_get_device_status() != 0:
            raise RuntimeError("device status after the long-context run")
        l_ms = sum(e0.elapsed_time(e1) for e0, e1 in lev) / reps
        lb = prefill_alg_bytes(LC["B"], LC["T"], LC["H"], LC["dk"], LC["dv"], with_s0=False)
        lpeak, lpeak_kind = measured_peaks()
        l_ach = lb / (l_ms / 1e3) / 1e9
        long_line = {"workload": LC["name"], "B": LC["B"], "T": LC["T"], "H": LC["H"], "launch_ms": l_ms,
                     "tokens_per_s": LC["B"] * LC["T"] / (l_ms / 1e3), "launches": reps,
                     "roofline": {"bound": "hbm", "achieved": l_ach, "peak": lpeak, "unit": "GB/s",
                                  "frac": l_ach / lpeak, "alg_bytes_per_launch": lb, "peak_kind": lpeak_kind},
                     "grid": f"{LC['B'] * LC['H']} CTAs (one per head) on the SMs",
                     "timed": "separately, after the headline region, CUDA events per launch"}
        long_line["split_in_two"] = measure_long_split(kda, LC, lq, lo, lst, stream, reps, l_ms)
        del lq, lo, lst

    # ---- end to end through the public API with host buffers (pinned), copies inside the timed region
    if args.no_e2e:
        e2e = None
    else:
        e2e = measure_e2e(kda, dist, world, dev, stream, args, q, k, v, g, beta, S0, o)
    tokens_per_prefill = P["B"] * P["T"]
    value = weak_scaling_throughput(tokens_per_prefill, world, args.steps, prefill_sum / 1e3)
    states = D["batch"] * D["H"]
    decode_states_per_s = weak_scaling_throughput(states, world, args.steps, decode_sum / 1e3)
    peak, peak_kind = measured_peaks()
    pb = prefill_alg_bytes(P["B"], P["T"], P["H"], P["dk"], P["dv"])
    prefill_launch_ms = prefill_sum / args.steps
    achieved = pb / (prefill_launch_ms / 1e3) / 1e9
    db_ = decode_alg_bytes(D["batch"], D["H"], D["dk"], D["dv"])
    decode_launch_ms = decode_sum / args.steps
    dec_achieved = db_ / (decode_launch_ms / 1e3) / 1e9
    impl_tag = "prefill_tc" if kda.lib().kda_forward_chunked_impl(None, None, None, None, None, None, None,
                                                                    None, 1, 0, 1, 128, 128, 0, 1, None) == 0 \
        else "prefill_simt"

    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return 0
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        cpu = oracle_baseline(budget_s=args.cpu_budget)
        cpu = {k_: cpu[k_] for k_ in ("value", "unit", "cores", "kind", "sample", "cpu_model", "single_thread")}
    tc_peak, tc_kind = measured_bf16_tflops()
    token_heads = P["B"] * P["T"] * P["H"]
    tensor_line = {"unit": "TFLOP/s", "peak": tc_peak, "peak_kind": tc_kind,
                   "causal": token_heads * PREFILL_FLOP_CAUSAL / (prefill_launch_ms * 1e-3) / 1e12,
                   "dense_tiles": token_heads * PREFILL_FLOP_DENSE / (prefill_launch_ms * 1e-3) / 1e12,
                   "note": "contraction work per launch / launch time (139,264 flop per token-head causal, "
                           "180,224 as whole tiles); the kernel is HBM-bound, so this is context"}
    tensor_line["frac_causal"] = tensor_line["causal"] / tc_peak
    tensor_line["frac_dense_tiles"] = tensor_line["dense_tiles"] / tc_peak
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"{P['name']} prefill + {D['name']} decode step",
                   "B": P["B"], "T": P["T"], "H": P["H"], "dk": P["dk"], "dv": P["dv"],
                   "decode_batch": D["batch"], "l2": "inputs larger than L2 (4.1 GB prefill, 1.6 GB decode state)",
                   "parallelism": f"replicas x{world} (independent batches, no collective)",
                   "inputs_sha256": inputs_sha256},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak,
                     "traffic": recorded_traffic(impl_tag) if P["name"] == DEFAULT_PREFILL_NAME else None,
                     "kernel": impl_tag, "alg_bytes_per_launch": pb, "launch_ms": prefill_launch_ms,
                     "peak_kind": peak_kind, "tensor": tensor_line},
        "decode": {"states_per_s": decode_states_per_s, "tokens_per_s": decode_states_per_s / D["H"],
                   "ms_per_step": decode_launch_ms,
                   "roofline": {"bound": "hbm", "achieved": dec_achieved, "peak": peak, "unit": "GB/s",
                                "frac": dec_achieved / peak, "alg_bytes_per_launch": db_,
                                "traffic": recorded_traffic("decode") if D["name"] == DEFAULT_DECODE_NAME else None}},
        "long_context": long_line,
        "state_emission": states_line,
        "fused_prologue": fused_line,
        "continuous_batching": batching_line,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": 2 * args.steps,
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def run_decode_only(args):
    """Decode steps back to back on one GPU (profiling: consecutive launches of the decode kernel, so that
    the state lines one launch leaves dirty in L2 are written back during the next)."""
    import torch
    import linear_attention_recurrence_forward_b200 as kda
    from linear_attention_recurrence_forward_b200.inputs import make_decode_inputs
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    D = DECODE
    gen = torch.Generator(device=str(dev))
    gen.manual_seed(2000)
    ring = [make_decode_inputs(D["batch"], D["H"], D["dk"], D["dv"], D["dtype"], gen=gen, device=str(dev))
            for _ in range(DECODE_RING)]
    S = torch.zeros((D["batch"], D["H"], D["dk"], D["dv"]), dtype=torch.float32, device=dev)
    od = torch.empty((D["batch"], D["H"], D["dv"]), dtype=ring[0][0].dtype, device=dev)
    stream = torch.cuda.current_stream()
    for i in range(args.warmup):
        kda.kda_decode_step(*ring[i % DECODE_RING], S, o=od, stream=stream)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    t0.record(stream)
    for i in range(args.steps):
        kda.kda_decode_step(*ring[i % DECODE_RING], S, o=od, stream=stream)
    t1.record(stream)
    torch.cuda.synchronize()
    if kda.kda_get_device_status() != 0:
        raise RuntimeError("device status after the decode steps")
    ms = t0.elapsed_time(t1) / args.steps
    db_ = decode_alg_bytes(D["batch"], D["H"], D["dk"], D["dv"])
    print(json.dumps({"mode": "decode-only (profiling)", "workload": D["name"], "ms_per_step": ms,
                      "alg_bytes_per_launch": db_, "achieved_gbs": db_ / (ms / 1e3) / 1e9}), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--prefill-shape", default=None, metavar="B,T,H",
                    help="override the prefill workload (profiling small cases); the line is then not the headline")
    ap.add_argument("--decode-batch", type=int, default=None, help="override the decode batch (profiling)")
    ap.add_argument("--head-dims", default=None, metavar="DK,DV",
                    help="override the prefill head sizes (64 or 128 each; timing other shapes), not the headline")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end measurement")
    ap.add_argument("--no-states", action="store_true", help="skip the state-emission (every 512 tokens) timing")
    ap.add_argument("--no-long", action="store_true", help="skip the long-context (T = 65536) timing")
    ap.add_argument("--no-batching", action="store_true",
                    help="skip the continuous-batching timings (packed prefill, paged decode)")
    ap.add_argument("--decode-only", action="store_true",
                    help="profiling: run only decode steps back to back (no prefill between them) and print their "
                         "timing; not the benchmark line")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.prefill_shape:
        B, T, H = (int(x) for x in args.prefill_shape.split(","))
        PREFILL.update(B=B, T=T, H=H, name=f"prefill_b{B}_t{T}_h{H}")
    if args.head_dims:
        dk, dv = (int(x) for x in args.head_dims.split(","))
        PREFILL.update(dk=dk, dv=dv, name=f"{PREFILL['name']}_dk{dk}_dv{dv}")
    if args.decode_batch:
        DECODE.update(batch=args.decode_batch, name=f"decode_b{args.decode_batch}_h{DECODE['H']}")
    if args.impl == "reference":
        return run_reference(args)
    if args.decode_only:
        return run_decode_only(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
