"""Benchmark of the attention sub-block on B200: prefill attention TFLOP/s and decode
KV-read GB/s, each against its roofline.

One step = one pass of the whole hot path over one batch of synthetic inputs:
  * prefill, the long-context workload (B=1, T=32768, H=64, Hkv=8, D=128), the
    largest single-GPU prefill: k-hat prologue (RMSNorm + RoPE of K) then the fused
    q-prologue + causal GQA attention kernel;
  * decode, batched workload (64 sequences, cache lengths U[1024, 32768], H=32,
    Hkv=8, D=128): split-KV kernel then the log-sum-exp merge.
The large prefill (B=4, T=4096, H=32, Hkv=8, inputs x0.5), the decode step with cache
append and the paged-cache decode are timed in regions of their own and reported as
extra keys.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun (N > 1) every rank runs the same step on its own GPU (independent
replicas: weak scaling, no collective on the data path); the time is the max over
ranks and the value counts the work of all ranks.  `--impl reference` times the
fp64 CPU oracle on bounded samples of the same workloads on the host cores.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from grouped_query_causal_b200 import synthetic  # noqa: E402

METRIC = "prefill attn TFLOPS and decode KV-read GB/s on 1 B200, % of roofline"
PREFILL = "long_context_prefill"
PREFILL_EXTRA = "large_prefill"
DECODE = "batched_decode"
WORKLOAD_TEXT = {
    "long_context_prefill": "long-context prefill (B1 T32768 H64 Hkv8 D128, causal)",
    "large_prefill": "large prefill (B4 T4096 H32 Hkv8 D128, inputs x0.5, causal)",
    "batched_decode": "batched decode (64 seqs, cache len U[1024,32768], H32 Hkv8 D128)",
}
L2_FLUSH_BYTES = 256 << 20   # written between timed calls whose inputs may still sit in L2 (126 MB)
DECODE_APPEND = "batched_decode_append"
# The sources each kernel is compiled from; its ncu traffic figures are stale once they change.
KERNEL_SOURCES = {
    "attn_fwd_kernel": ["prefill.cuh", "ptx.cuh", "rope.cuh", "gqa_attn.cu"],   # the schedule is set on the host
    "decode_split_kernel": ["decode.cuh", "ptx.cuh", "rope.cuh"],
    "decode_split_kernel<paged>": ["decode.cuh", "ptx.cuh", "rope.cuh"],
}
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------------------- workload sizes
def prefill_flops(B, T, H, D=128):
    """Algorithmic FLOPs of causal attention: QK^T and PV over the visible (i, j <= i)
    pairs only, 2*D each: B*H*T(T+1)/2 pairs * 4D."""
    return B * H * 2 * D * T * (T + 1)


def decode_bytes(seqlens, H, Hkv, D=128):
    """Algorithmic bytes of decode: every cached K and V row read once (bf16), plus the
    bf16 query and the fp32 output."""
    B = len(seqlens)
    return int(sum(int(s) for s in seqlens)) * Hkv * D * 2 * 2 + B * H * D * 2 + B * H * D * 4


def max_over_ranks(values, device, world):
    """Element-wise maximum of `values` (durations) over all ranks of the process group;
    the values themselves when there is one rank."""
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.tolist()


def whole_job_rate(units_per_rank, world, seconds):
    """Throughput of the whole job: every rank processed `units_per_rank` in at most
    `seconds` (the maximum over ranks)."""
    return world * units_per_rank / seconds


def decode_append_bytes(seqlens, H, Hkv, D=128):
    """Algorithmic bytes of the append step: the new K/V rows read (bf16) and written into
    the cache, then decode over seqlens[b] + 1 rows."""
    B = len(seqlens)
    return decode_bytes([int(s) + 1 for s in seqlens], H, Hkv, D) + 2 * B * Hkv * D * 2 * 2


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def _code_only(text: str) -> str:
    """C++ source with comments and blank lines removed, so that editing a comment does
    not mark a kernel's counters stale."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    lines = (re.sub(r"//.*$", "", line).rstrip() for line in text.splitlines())
    return "\n".join(line for line in lines if line)


def kernel_source_hash(kernel):
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "grouped_query_causal_b200", "csrc", name), encoding="utf-8") as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def traffic_from_profiles(kernel, workload):
    """DRAM bytes per launch of `kernel` on `workload` from the committed ncu summary
    (profiles/traffic.json), or None when there is none or the kernel's sources changed
    since the counters were taken."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)
    except (OSError, ValueError):
        return None
    e = t.get(kernel)
    if not e or kernel not in KERNEL_SOURCES or e.get("source_hash") != kernel_source_hash(kernel):
        return None
    w = e.get("workloads", {}).get(workload)
    return None if w is None else w.get("dram_bytes_per_launch")


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax.append(float(parts[2]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- our arm
def run_ours(args, rank, world, local_rank):
    from grouped_query_causal_b200 import binding as gqa
    lib = gqa.load()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    sh = stream.cuda_stream

    pin = synthetic.make(PREFILL)
    dec = synthetic.make(DECODE)
    B, T, H, D = pin.q.shape
    Hkv = pin.k.shape[2]
    dB, dH, _ = dec.q.shape
    dHkv = dec.k_cache.shape[1]
    max_len = dec.max_len
    flops = prefill_flops(B, T, H, D)
    dbytes = decode_bytes(dec.seqlens.tolist(), dH, dHkv, D)

    # device-resident inputs, outputs, workspaces
    q, k, v, pos = pin.q.to(dev), pin.k.to(dev), pin.v.to(dev), pin.pos.to(dev)
    wq, wk = pin.wq.to(dev), pin.wk.to(dev)
    khat = torch.empty_like(k)
    rope_cs = torch.empty(gqa.rope_table_numel(B * T, D), dtype=torch.float32, device=dev)
    out = torch.empty((B, T, H, D), dtype=torch.float32, device=dev)
    dq, kc, vc = dec.q.to(dev), dec.k_cache.to(dev), dec.v_cache.to(dev)
    offs, sl, dwq = dec.offsets.to(dev), dec.seqlens.to(dev), dec.wq.to(dev)
    dout = torch.empty((dB, dH, D), dtype=torch.float32, device=dev)
    dws = torch.empty(gqa.decode_workspace_size(dB, dH, dHkv, max_len, D), dtype=torch.uint8, device=dev)
    ptr = lambda t: t.data_ptr()  # noqa: E731

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        st = lib.gqa_attn_k_norm_rope(ptr(k), ptr(pos), ptr(wk), pin.theta, pin.eps, ptr(khat), ptr(rope_cs), B * T,
                                      Hkv, D, sh)
        if ev:
            ev[1].record(stream)
        st |= lib.gqa_attn_prefill_khat(ptr(q), ptr(khat), ptr(v), ptr(pos), ptr(rope_cs), ptr(wq), pin.theta,
                                        pin.eps, ptr(out), B, T, H, Hkv, D, sh)
        if ev:
            ev[2].record(stream)
        st |= lib.gqa_attn_decode(ptr(dq), ptr(kc), ptr(vc), ptr(offs), ptr(sl), None, ptr(dwq), dec.theta, dec.eps,
                                  ptr(dout), dB, dH, dHkv, D, max_len, ptr(dws), dws.numel(), sh)
        if ev:
            ev[3].record(stream)
        if st != 0:
            raise RuntimeError(f"library call failed with status {st}")

    launches_per_step = 2 + 2   # k prologue + attention, decode split + merge

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if gqa.device_status() != 0:
        raise RuntimeError("device status error after warm-up")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    sampler = ClockSampler(local_rank) if rank == 0 else None
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(args.steps):
        step(evs[i])
    t1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop() if sampler else None
    if gqa.device_status() != 0:
        raise RuntimeError("device status error in the timed region")

    total_ms = t0.elapsed_time(t1)
    pro_ms = sum(e[0].elapsed_time(e[1]) for e in evs)
    attn_ms = sum(e[1].elapsed_time(e[2]) for e in evs)
    dec_ms = sum(e[2].elapsed_time(e[3]) for e in evs)
    # max over ranks of every duration
    total_ms, pro_ms, attn_ms, dec_ms = max_over_ranks([total_ms, pro_ms, attn_ms, dec_ms], dev, world)
    K = args.steps
    prefill_s = (pro_ms + attn_ms) / 1e3
    dec_s = dec_ms / 1e3

    # ---- end to end through the public API with host buffers (pinned), copies timed
    e2e = run_e2e(gqa, pin, dec, dev, stream, rank, world, max(3, min(K, 10)))

    # ---- the large prefill (its own timed region)
    extra = run_prefill_leg(gqa, PREFILL_EXTRA, dev, stream, world, K, args.warmup)
    # ---- packed variable-length and chunked prefill, the projections (own timed regions)
    varlen = run_packed_leg(gqa, "varlen_prefill", dev, stream, world, K, args.warmup)
    chunked = run_packed_leg(gqa, "chunked_prefill", dev, stream, world, K, args.warmup)
    chunked_paged = run_packed_leg(gqa, "chunked_prefill", dev, stream, world, K, args.warmup, page_size=16)
    proj = run_projection_leg(gqa, dev, stream, world, K, args.warmup)
    block = run_block_leg(gqa, dev, stream, world, K, args.warmup)
    # ---- the decode step that appends the new token first, and the plain decode, each in
    # its own timed region (the in-step decode runs after the long prefill)
    app = run_decode_append(gqa, dev, stream, world, K, args.warmup)
    dalone = run_decode_alone(gqa, dec, dq, kc, vc, offs, sl, dwq, dws, dout, dev, stream, world, K, args.warmup)
    # ---- the batched decode on a paged copy of the same cache (its own timed region)
    paged = run_decode_paged(gqa, dec, dq, kc, vc, sl, dwq, dev, stream, world, K, args.warmup)

    if rank != 0:
        return None
    pk, pk_kind = peaks()
    hbm = float(pk["hbm_gbs"])
    # The burst figure when the step runs at the maximum SM clock, like the burst cuBLAS
    # measurement; the sustained (power-capped) figure when the clocks show the step ran
    # under the power cap, like the seconds-long cuBLAS loop.
    capped = clocks is not None and ("sw_power_cap" in clocks.get("reasons", []) or (
        clocks.get("sm_mhz") and clocks.get("sm_max_mhz") and clocks["sm_mhz"] < 0.97 * clocks["sm_max_mhz"]))
    tc_kind = "bf16_tflops_sustained" if capped and "bf16_tflops_sustained" in pk else "bf16_tflops"
    tc = float(pk[tc_kind])
    attn_tflops = flops * K / (attn_ms / 1e3) / 1e12
    total_tflops = flops * K / prefill_s / 1e12
    dec_gbs = dbytes * K / dec_s / 1e9
    traffic_attn = traffic_from_profiles("attn_fwd_kernel", PREFILL)
    traffic_dec = traffic_from_profiles("decode_split_kernel", DECODE)
    for key, legd in (("large_prefill", extra), ("varlen_prefill", varlen), ("chunked_prefill", chunked),
                      ("chunked_prefill_paged", chunked_paged), ("projections", proj), ("attn_block", block),
                      ("decode_append", app), ("decode_paged", paged), ("decode_alone", dalone)):
        legd["clocks"] = LEG_CLOCKS.get(key)
    hbm_line = lambda leg: dict(leg, roofline=dict(leg["roofline"], peak=hbm,  # noqa: E731
                                                   frac=round(leg["roofline"]["achieved"] / hbm, 4),
                                                   peak_source=f"hbm_gbs of {pk_kind}"))
    tcb = float(pk["bf16_tflops"])
    tc_line = lambda leg: dict(leg, roofline=dict(leg["roofline"], peak=tcb,  # noqa: E731
                                                  frac=round(leg["roofline"]["achieved"] / tcb, 4),
                                                  peak_source=f"bf16_tflops (burst) of {pk_kind}",
                                                  **({"frac_incl_k_prologue": round(leg["value"] / world / tcb, 4)}
                                                     if "k_prologue_ms" in leg else {})))
    line = {
        "metric": METRIC,
        "value": round(whole_job_rate(flops * K, world, prefill_s) / 1e12, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": round(total_ms / K, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {
            "workload": f"{WORKLOAD_TEXT[PREFILL]} + {WORKLOAD_TEXT[DECODE]}",
            "prefill": {"B": B, "T": T, "H": H, "Hkv": Hkv, "D": D, "flops_per_step": flops},
            "decode": {"B": dB, "H": dH, "Hkv": dHkv, "D": D, "cached_tokens": int(dec.seqlens.sum()),
                       "bytes_per_step": dbytes},
            "l2": "inputs larger than L2 (prefill q/k/v/out 1.75 GB; decode KV cache 3.9 GB); no flush in the "
                  "step; the extra legs write 256 MB between timed calls",
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
        },
        "prefill_ms": round(1e3 * prefill_s / K, 4),
        "decode": {
            "value": round(whole_job_rate(dbytes * K, world, dec_s) / 1e9, 1),
            "unit": "GB/s",
            "ms": round(1e3 * dec_s / K, 4),
            "roofline": {"bound": "hbm", "achieved": round(dec_gbs, 1), "peak": hbm, "unit": "GB/s",
                         "frac": round(dec_gbs / hbm, 4), "traffic": traffic_dec,
                         "kernel": "decode_split_kernel + decode_merge_kernel (one call)",
                         "peak_source": f"hbm_gbs of {pk_kind}"},
            "e2e": e2e["decode"],
        },
        # value counts the k-hat prologue and the attention kernel; roofline is the
        # attention kernel alone (the dominant kernel), frac_incl_k_prologue both.
        "roofline": {"bound": "tensor", "achieved": round(attn_tflops, 2), "peak": tc, "unit": "TFLOP/s",
                     "frac": round(attn_tflops / tc, 4), "frac_incl_k_prologue": round(total_tflops / tc, 4),
                     "traffic": traffic_attn, "kernel": "attn_fwd_kernel",
                     "attn_ms": round(attn_ms / K, 4), "k_prologue_ms": round(pro_ms / K, 4),
                     "peak_source": f"{tc_kind} of {pk_kind}",
                     "peak_burst": float(pk["bf16_tflops"]),
                     "peak_sustained": float(pk.get("bf16_tflops_sustained", pk["bf16_tflops"]))},
        "e2e": e2e["prefill"],
        "large_prefill": tc_line(extra),
        "varlen_prefill": tc_line(varlen),
        "chunked_prefill": tc_line(chunked),
        "chunked_prefill_paged": tc_line(chunked_paged),
        "projections": tc_line(proj),
        "attn_block": tc_line(block),
        "decode_append": hbm_line(app),
        "decode_alone": hbm_line(dalone),
        "decode_paged": hbm_line(paged),
        "gpu_launches": launches_per_step * K,
        "clocks": clocks,
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(pin, dec, budget_s=args.cpu_seconds)
    return line


LEG_CLOCKS = {}   # clocks sampled during each extra leg's timed calls, by leg name


def timed_calls(call, stream, world, dev, K, W, flush=None, leg=None):
    """W untimed calls, then K calls each between its own pair of CUDA events on `stream`
    (with `flush`, a 256 MB write between calls, outside the events); returns the summed
    seconds per event pair (a list), maximum over ranks.  With `leg`, the SM clocks seen
    during the timed calls go to LEG_CLOCKS[leg] (rank 0)."""
    sampler = ClockSampler(dev.index or 0) if (leg and int(os.environ.get("RANK", "0")) == 0) else None
    if sampler:   # started ahead of the warm-up so that nvidia-smi is sampling by the timed calls
        sampler.start()
        time.sleep(0.3)
    for _ in range(W):
        call(None)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    evs = []
    for i in range(K):
        if flush is not None:
            flush.fill_(i & 255)
        evs.append(call(stream))
    torch.cuda.synchronize()
    if sampler:
        LEG_CLOCKS[leg] = sampler.stop()
    n = len(evs[0]) - 1
    ms = [sum(e[j].elapsed_time(e[j + 1]) for e in evs) for j in range(n)]
    return [x / 1e3 for x in max_over_ranks(ms, dev, world)]


def run_prefill_leg(gqa, name, dev, stream, world, K, W):
    """The k-hat prologue and attention kernel on the prefill workload `name`, inputs
    resident, each call between CUDA events (prologue and attention separately), L2
    flushed between calls."""
    lib = gqa.load()
    sh = stream.cuda_stream
    w = synthetic.make(name)
    B, T, H, D = w.q.shape
    Hkv = w.k.shape[2]
    q, k, v, pos, wq, wk = (x.to(dev) for x in (w.q, w.k, w.v, w.pos, w.wq, w.wk))
    khat = torch.empty_like(k)
    rope_cs = torch.empty(gqa.rope_table_numel(B * T, D), dtype=torch.float32, device=dev)
    out = torch.empty((B, T, H, D), dtype=torch.float32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    ptr = lambda t: t.data_ptr()  # noqa: E731

    def call(st_):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)] if st_ is not None else None
        if ev:
            ev[0].record(st_)
        st = lib.gqa_attn_k_norm_rope(ptr(k), ptr(pos), ptr(wk), w.theta, w.eps, ptr(khat), ptr(rope_cs), B * T,
                                      Hkv, D, sh)
        if ev:
            ev[1].record(st_)
        st |= lib.gqa_attn_prefill_khat(ptr(q), ptr(khat), ptr(v), ptr(pos), ptr(rope_cs), ptr(wq), w.theta, w.eps,
                                        ptr(out), B, T, H, Hkv, D, sh)
        if ev:
            ev[2].record(st_)
        if st != 0:
            raise RuntimeError(f"{name}: library call failed with status {st}")
        return ev

    pro_s, attn_s = timed_calls(call, stream, world, dev, K, W, flush, leg=name)
    if gqa.device_status() != 0:
        raise RuntimeError(f"device status error in the {name} timing")
    flops = prefill_flops(B, T, H, D)
    del q, k, v, pos, khat, rope_cs, out, flush
    return {"value": round(whole_job_rate(flops * K, world, pro_s + attn_s) / 1e12, 2), "unit": "TFLOP/s",
            "ms": round(1e3 * (pro_s + attn_s) / K, 4), "attn_ms": round(1e3 * attn_s / K, 4),
            "k_prologue_ms": round(1e3 * pro_s / K, 4), "workload": WORKLOAD_TEXT[name],
            "flops_per_call": flops, "gpu_launches": 2 * K,
            "roofline": {"bound": "tensor", "achieved": round(flops * K / attn_s / 1e12, 2), "unit": "TFLOP/s",
                         "traffic": traffic_from_profiles("attn_fwd_kernel", name), "kernel": "attn_fwd_kernel"}}


def packed_flops(lens, prefix, H, D=128):
    """Algorithmic FLOPs of causal attention over packed sequences: chunk row t of
    sequence b sees prefix[b] + t + 1 keys, 4 D FLOP each (QK^T and PV)."""
    return sum(4 * D * H * (n * p + n * (n + 1) // 2) for n, p in zip(lens, prefix))


def run_packed_leg(gqa, name, dev, stream, world, K, W, page_size=None):
    """gqa_attn_prefill_varlen (no prefix) or gqa_attn_prefill_chunk (each sequence has
    cached rows; the chunk is appended to the cache first) on a packed workload, inputs
    resident, CUDA events around each call, L2 flushed between calls.  With page_size, the
    chunk workload's cache in shuffled pages of that many rows (gqa_attn_prefill_chunk_paged)."""
    lib = gqa.load()
    sh = stream.cuda_stream
    w = synthetic.make(name)
    N, H, D = w.q.shape
    Hkv = w.k.shape[1]
    B = len(w.lens)
    chunk = w.prefix is not None
    t = {n: getattr(w, n).to(dev) for n in ("q", "k", "v", "pos", "cu", "wq", "wk")}
    paged = chunk and page_size is not None
    leg = name + ("_paged" if paged else "")
    if paged:
        caps = [p + n for p, n in zip(w.prefix.tolist(), w.lens)]
        pc = synthetic.page_cache(w.k_cache, w.v_cache, w.cache_offsets, caps, page_size, seed=31)
        t.update(k_pages=pc.k_pages.to(dev), v_pages=pc.v_pages.to(dev), table=pc.page_table.to(dev),
                 prefix=w.prefix.to(dev))
        ws_n = lib.gqa_attn_prefill_chunk_paged_workspace_size(N, D)
        del pc
    elif chunk:
        t.update({n: getattr(w, n).to(dev) for n in ("k_cache", "v_cache", "cache_offsets", "prefix")})
        ws_n = lib.gqa_attn_prefill_chunk_workspace_size(N, D)
    else:
        ws_n = lib.gqa_attn_prefill_varlen_workspace_size(N, Hkv, D)
    ws = torch.empty(ws_n, dtype=torch.uint8, device=dev)
    out = torch.empty((N, H, D), dtype=torch.float32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    rope = gqa.RopeConfig.make(theta=w.theta)
    maxlen = max(w.lens)
    ptr = lambda x: x.data_ptr()  # noqa: E731

    def call(st_):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)] if st_ is not None else None
        if ev:
            ev[0].record(st_)
        if paged:
            st = lib.gqa_attn_prefill_chunk_paged(
                ptr(t["q"]), ptr(t["k"]), ptr(t["v"]), ptr(t["pos"]), ptr(t["cu"]), ptr(t["k_pages"]),
                ptr(t["v_pages"]), ptr(t["table"]), t["k_pages"].shape[0], page_size, t["table"].shape[1],
                ptr(t["prefix"]), ptr(t["wq"]), ptr(t["wk"]), ctypes.byref(rope), w.eps, ptr(out), B, N, H, Hkv, D,
                maxlen, ptr(ws), ws.numel(), sh)
        elif chunk:
            st = lib.gqa_attn_prefill_chunk(ptr(t["q"]), ptr(t["k"]), ptr(t["v"]), ptr(t["pos"]), ptr(t["cu"]),
                                            ptr(t["k_cache"]), ptr(t["v_cache"]), ptr(t["cache_offsets"]),
                                            ptr(t["prefix"]), t["k_cache"].shape[0], ptr(t["wq"]), ptr(t["wk"]),
                                            ctypes.byref(rope), w.eps, ptr(out), B, N, H, Hkv, D, maxlen, ptr(ws),
                                            ws.numel(), sh)
        else:
            st = lib.gqa_attn_prefill_varlen(ptr(t["q"]), ptr(t["k"]), ptr(t["v"]), ptr(t["pos"]), ptr(t["cu"]),
                                             ptr(t["wq"]), ptr(t["wk"]), ctypes.byref(rope), w.eps, ptr(out), B, N,
                                             H, Hkv, D, maxlen, ptr(ws), ws.numel(), sh)
        if ev:
            ev[1].record(st_)
        if st != 0:
            raise RuntimeError(f"{leg}: library call failed with status {st}")
        return ev

    sec = timed_calls(call, stream, world, dev, K, W, flush, leg=leg)[0]
    if gqa.device_status() != 0:
        raise RuntimeError(f"device status error in the {leg} timing")
    prefix = w.prefix.tolist() if chunk else [0] * B
    flops = packed_flops(w.lens, prefix, H, D)
    del t, ws, out, flush
    what = (f"{B} sequences, {prefix[0]} cached rows + a {w.lens[0]}-token chunk each, H{H} Hkv{Hkv} D{D}"
            + (f", cache in shuffled {page_size}-row pages" if paged else "")
            if chunk else f"{B} packed sequences, lengths U[256,8192] (N={N}), H{H} Hkv{Hkv} D{D}")
    return {"value": round(whole_job_rate(flops * K, world, sec) / 1e12, 2), "unit": "TFLOP/s",
            "ms": round(1e3 * sec / K, 4), "workload": what, "flops_per_call": flops, "gpu_launches": 3 * K,
            "roofline": {"bound": "tensor", "achieved": round(flops * K / sec / 1e12, 2), "unit": "TFLOP/s",
                         "traffic": None,
                         "kernel": "k_prologue_kernel + unit_list_kernel + attn_fwd_kernel (one call)"}}


def run_projection_leg(gqa, dev, stream, world, K, W):
    """gqa_linear as the fused QKV projection (16384 x 4096 -> 6144, bf16 out) and as the
    output projection (16384 x 4096 -> 4096, fp32 out), each call between CUDA events, L2
    flushed between calls."""
    lib = gqa.load()
    sh = stream.cuda_stream
    w = synthetic.make("projections")
    x, wqkv, wo = w.x.to(dev), w.w_qkv.to(dev), w.w_o.to(dev)
    M, hidden = x.shape
    Nq = wqkv.shape[0]
    qkv = torch.empty((M, Nq), dtype=torch.bfloat16, device=dev)
    y = torch.empty((M, hidden), dtype=torch.float32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def call(st_):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)] if st_ is not None else None
        if ev:
            ev[0].record(st_)
        st = lib.gqa_linear(x.data_ptr(), wqkv.data_ptr(), qkv.data_ptr(), 0, M, Nq, hidden, sh)
        if ev:
            ev[1].record(st_)
        # the output projection reads an [M, H D] bf16 operand (H D = hidden here); x stands
        # in for the attention output (same shape and dtype)
        st |= lib.gqa_linear(x.data_ptr(), wo.data_ptr(), y.data_ptr(), 1, M, hidden, hidden, sh)
        if ev:
            ev[2].record(st_)
        if st != 0:
            raise RuntimeError(f"gqa_linear failed with status {st}")
        return ev

    s_qkv, s_o = timed_calls(call, stream, world, dev, K, W, flush, leg="projections")
    if gqa.device_status() != 0:
        raise RuntimeError("device status error in the projection timing")
    f_qkv, f_o = 2 * M * Nq * hidden, 2 * M * hidden * hidden
    del x, wqkv, wo, qkv, y, flush
    return {"value": round(whole_job_rate((f_qkv + f_o) * K, world, s_qkv + s_o) / 1e12, 2), "unit": "TFLOP/s",
            "workload": f"qkv_proj {M}x{hidden} -> {Nq} (bf16 out) and o_proj {M}x{hidden} -> {hidden} (fp32 out)",
            "qkv_ms": round(1e3 * s_qkv / K, 4), "o_proj_ms": round(1e3 * s_o / K, 4),
            "qkv_tflops": round(f_qkv * K / s_qkv / 1e12, 2), "o_proj_tflops": round(f_o * K / s_o / 1e12, 2),
            "gpu_launches": 2 * K,
            "roofline": {"bound": "tensor", "achieved": round((f_qkv + f_o) * K / (s_qkv + s_o) / 1e12, 2),
                         "unit": "TFLOP/s", "traffic": None, "kernel": "gemm_kernel"}}


def run_block_leg(gqa, dev, stream, world, K, W):
    """gqa_attn_block_prefill, the whole attention sub-block (qkv projection, q/k norm,
    RoPE, causal GQA attention, output projection) on the large prefill's shape with
    hidden 4096, CUDA events around each call, L2 flushed between calls."""
    lib = gqa.load()
    sh = stream.cuda_stream
    B, T, H, Hkv, D, hidden = 4, 4096, 32, 8, 128, 4096
    w = synthetic.projection_inputs(B * T, hidden, H, Hkv, seed=40)
    x, wqkv, wo = w.x.to(dev), w.w_qkv.to(dev), w.w_o.to(dev)
    pos = torch.arange(T, dtype=torch.int32, device=dev).repeat(B, 1).contiguous()
    g = torch.Generator().manual_seed(41)
    wq = (torch.rand(D, generator=g) + 0.5).to(dev)
    wk = (torch.rand(D, generator=g) + 0.5).to(dev)
    y = torch.empty((B * T, hidden), dtype=torch.float32, device=dev)
    ws = torch.empty(lib.gqa_attn_block_prefill_workspace_size(B, T, hidden, H, Hkv, D), dtype=torch.uint8,
                     device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    rope = gqa.RopeConfig.make(theta=synthetic.THETA)

    def call(st_):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)] if st_ is not None else None
        if ev:
            ev[0].record(st_)
        st = lib.gqa_attn_block_prefill(x.data_ptr(), wqkv.data_ptr(), wo.data_ptr(), pos.data_ptr(), wq.data_ptr(),
                                        wk.data_ptr(), ctypes.byref(rope), synthetic.EPS, y.data_ptr(), B, T, hidden,
                                        H, Hkv, D, ws.data_ptr(), ws.numel(), sh)
        if ev:
            ev[1].record(st_)
        if st != 0:
            raise RuntimeError(f"gqa_attn_block_prefill failed with status {st}")
        return ev

    sec = timed_calls(call, stream, world, dev, K, W, flush, leg="attn_block")[0]
    if gqa.device_status() != 0:
        raise RuntimeError("device status error in the attention-block timing")
    N = B * T
    flops = 2 * N * (H + 2 * Hkv) * D * hidden + prefill_flops(B, T, H, D) + 2 * N * hidden * H * D
    del x, wqkv, wo, y, ws, flush
    return {"value": round(whole_job_rate(flops * K, world, sec) / 1e12, 2), "unit": "TFLOP/s",
            "ms": round(1e3 * sec / K, 4), "flops_per_call": flops,
            "workload": f"attention sub-block B{B} T{T} hidden {hidden} H{H} Hkv{Hkv} D{D}: qkv_proj, q/k norm, "
                        "RoPE, causal GQA attention, o_proj", "gpu_launches": 4 * K,
            "roofline": {"bound": "tensor", "achieved": round(flops * K / sec / 1e12, 2), "unit": "TFLOP/s",
                         "traffic": None, "kernel": "gemm_kernel, k_prologue_kernel, attn_fwd_kernel, gemm_kernel"}}


def run_decode_alone(gqa, dec, dq, kc, vc, offs, sl, dwq, dws, dout, dev, stream, world, K, W):
    """gqa_attn_decode on the batched decode workload in its own timed region (CUDA events
    around each call, L2 flushed between calls), away from the prefill of the step."""
    lib = gqa.load()
    sh = stream.cuda_stream
    B, H, D = dec.q.shape
    Hkv = dec.k_cache.shape[1]
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    ptr = lambda t: t.data_ptr()  # noqa: E731

    def call(st_):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)] if st_ is not None else None
        if ev:
            ev[0].record(st_)
        st = lib.gqa_attn_decode(ptr(dq), ptr(kc), ptr(vc), ptr(offs), ptr(sl), None, ptr(dwq), dec.theta, dec.eps,
                                 ptr(dout), B, H, Hkv, D, dec.max_len, ptr(dws), dws.numel(), sh)
        if ev:
            ev[1].record(st_)
        if st != 0:
            raise RuntimeError(f"gqa_attn_decode failed with status {st}")
        return ev

    sec = timed_calls(call, stream, world, dev, K, W, flush, leg="decode_alone")[0]
    if gqa.device_status() != 0:
        raise RuntimeError("device status error in the decode timing")
    nbytes = decode_bytes(dec.seqlens.tolist(), H, Hkv, D)
    del flush
    return {"value": round(whole_job_rate(nbytes * K, world, sec) / 1e9, 1), "unit": "GB/s",
            "ms": round(1e3 * sec / K, 4), "workload": WORKLOAD_TEXT[DECODE], "bytes_per_call": nbytes,
            "gpu_launches": 2 * K, "l2": "256 MB written between timed calls",
            "roofline": {"bound": "hbm", "achieved": round(nbytes * K / sec / 1e9, 1), "unit": "GB/s",
                         "traffic": traffic_from_profiles("decode_split_kernel", DECODE),
                         "kernel": "decode_split_kernel + decode_merge_kernel (one call)"}}


def run_decode_append(gqa, dev, stream, world, K, W):
    """gqa_attn_decode_append on the batched append workload (64 sequences with
    1023..32767 cached rows, one new token each), inputs resident, CUDA events around each
    of K calls after W warm-up calls, L2 flushed between calls.  Every call writes the
    same rows with the same values."""
    lib = gqa.load()
    sh = stream.cuda_stream
    w = synthetic.make(DECODE_APPEND)
    B, H, D = w.q.shape
    Hkv = w.k_cache.shape[1]
    t = {n: getattr(w, n).to(dev) for n in ("q", "k_new", "v_new", "k_cache", "v_cache", "offsets", "seqlens",
                                               "wq", "wk")}
    out = torch.empty((B, H, D), dtype=torch.float32, device=dev)
    ws = torch.empty(gqa.decode_workspace_size(B, H, Hkv, w.max_len, D), dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    ptr = lambda x: x.data_ptr()  # noqa: E731

    def call(st_):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)] if st_ is not None else None
        if ev:
            ev[0].record(st_)
        st = lib.gqa_attn_decode_append(ptr(t["q"]), ptr(t["k_new"]), ptr(t["v_new"]), ptr(t["k_cache"]),
                                        ptr(t["v_cache"]), ptr(t["offsets"]), ptr(t["seqlens"]), None, ptr(t["wq"]),
                                        ptr(t["wk"]), w.theta, w.eps, ptr(out), B, H, Hkv, D, w.max_len, ptr(ws),
                                        ws.numel(), sh)
        if ev:
            ev[1].record(st_)
        if st != 0:
            raise RuntimeError(f"gqa_attn_decode_append failed with status {st}")
        return ev

    sec = timed_calls(call, stream, world, dev, K, W, flush, leg="decode_append")[0]
    if gqa.device_status() != 0:
        raise RuntimeError("device status error in the append-step timing")
    nbytes = decode_append_bytes(w.seqlens.tolist(), H, Hkv, D)
    gbs = nbytes * K / sec / 1e9
    del t, out, ws, flush
    return {"value": round(whole_job_rate(nbytes * K, world, sec) / 1e9, 1), "unit": "GB/s",
            "ms": round(1e3 * sec / K, 4),
            "workload": "64 sequences, cached rows U[1023,32767] + 1 appended, H32 Hkv8 D128",
            "bytes_per_call": nbytes, "gpu_launches": 3 * K, "l2": "256 MB written between timed calls",
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "unit": "GB/s",
                         "traffic": traffic_from_profiles("decode_split_kernel", DECODE_APPEND),
                         "kernel": "decode_append_kernel + decode_split_kernel + decode_merge_kernel (one call)"}}


def paged_layout(lens, offs, page_size, seed=30):
    """Page table [B, max pages] (int32, -1 unused) and, for every row of every page, the
    contiguous cache row it holds (-1: past the end of its sequence), with the pages of all
    sequences handed out in a seeded random order."""
    B = len(lens)
    need = [(int(n) + page_size - 1) // page_size for n in lens]
    num_pages = sum(need)
    perm = torch.randperm(num_pages, generator=torch.Generator().manual_seed(seed))
    table = torch.full((B, max(1, max(need))), -1, dtype=torch.int32)
    src = torch.full((num_pages * page_size,), -1, dtype=torch.int64)
    start = 0
    for b in range(B):
        pids = perm[start:start + need[b]]
        start += need[b]
        table[b, :need[b]] = pids.to(torch.int32)
        rows = torch.arange(int(lens[b]), dtype=torch.int64)
        src[pids.repeat_interleave(page_size)[:int(lens[b])] * page_size + rows % page_size] = int(offs[b]) + rows
    return table, src


def run_decode_paged(gqa, dec, dq, kc, vc, sl, dwq, dev, stream, world, K, W, page_size=64):
    """gqa_attn_decode_paged on the batched decode workload, its cache copied on the
    device into pages of page_size rows handed out in a seeded random order; CUDA events
    around each of K calls after W warm-up calls, L2 flushed between calls."""
    lib = gqa.load()
    sh = stream.cuda_stream
    B, H, D = dec.q.shape
    Hkv = dec.k_cache.shape[1]
    lens = dec.seqlens.tolist()
    table, src = paged_layout(lens, dec.offsets.tolist(), page_size)
    num_pages = src.numel() // page_size
    src = src.to(dev)
    ok = (src >= 0).view(-1, 1, 1)
    kp = torch.where(ok, kc[src.clamp(min=0)], 0).view(num_pages, page_size, Hkv, D)
    vp = torch.where(ok, vc[src.clamp(min=0)], 0).view(num_pages, page_size, Hkv, D)
    del src, ok
    tab = table.to(dev)
    out = torch.empty((B, H, D), dtype=torch.float32, device=dev)
    ws = torch.empty(gqa.decode_workspace_size(B, H, Hkv, dec.max_len, D), dtype=torch.uint8, device=dev)
    rope = gqa.RopeConfig.make(theta=dec.theta)

    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def call(st_):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)] if st_ is not None else None
        if ev:
            ev[0].record(st_)
        st = lib.gqa_attn_decode_paged(dq.data_ptr(), kp.data_ptr(), vp.data_ptr(), tab.data_ptr(), num_pages,
                                       page_size, tab.shape[1], sl.data_ptr(), None, dwq.data_ptr(),
                                       ctypes.byref(rope), dec.eps, out.data_ptr(), B, H, Hkv, D, dec.max_len,
                                       ws.data_ptr(), ws.numel(), sh)
        if ev:
            ev[1].record(st_)
        if st != 0:
            raise RuntimeError(f"gqa_attn_decode_paged failed with status {st}")
        return ev

    sec = timed_calls(call, stream, world, dev, K, W, flush, leg="decode_paged")[0]
    if gqa.device_status() != 0:
        raise RuntimeError("device status error in the paged-decode timing")
    nbytes = decode_bytes(lens, H, Hkv, D)
    gbs = nbytes * K / sec / 1e9
    del kp, vp, tab, out, ws, flush
    return {"value": round(whole_job_rate(nbytes * K, world, sec) / 1e9, 1), "unit": "GB/s",
            "ms": round(1e3 * sec / K, 4), "page_size": page_size, "num_pages": num_pages,
            "workload": "the batched decode (64 seqs, cache len U[1024,32768], H32 Hkv8 D128) in shuffled pages",
            "bytes_per_call": nbytes, "gpu_launches": 2 * K, "l2": "256 MB written between timed calls",
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "unit": "GB/s",
                         "traffic": traffic_from_profiles("decode_split_kernel<paged>", "batched_decode_paged64"),
                         "kernel": "decode_split_kernel (paged) + decode_merge_kernel (one call)"}}


def run_e2e(gqa, pin, dec, dev, stream, rank, world, steps):
    """Same metrics through the public API with host (pinned) buffers: every step copies
    that step's inputs host->device, runs the call, and reads the result back.  The steps
    are pipelined as a serving loop would run them: copies in on one stream, the calls on
    the compute stream, copies out on a third, with two device buffer sets, so that step
    i+1's inputs and step i-1's result cross PCIe while step i computes (events order
    each buffer set's reuse)."""
    lib = gqa.load()
    sh = stream.cuda_stream
    B, T, H, D = pin.q.shape
    Hkv = pin.k.shape[2]
    dB, dH, _ = dec.q.shape
    dHkv = dec.k_cache.shape[1]
    max_len = dec.max_len
    hp = {n: getattr(pin, n).pin_memory() for n in ("q", "k", "v", "pos", "wq", "wk")}
    hd = {"q": dec.q.pin_memory(), "k_cache": dec.k_cache.pin_memory(), "v_cache": dec.v_cache.pin_memory(),
          "offsets": dec.offsets.pin_memory(), "seqlens": dec.seqlens.pin_memory(), "wq": dec.wq.pin_memory()}
    hout = torch.empty((B, T, H, D), dtype=torch.float32).pin_memory()
    hdout = torch.empty((dB, dH, D), dtype=torch.float32).pin_memory()
    pws = torch.empty(gqa.prefill_workspace_size(B, T, H, Hkv, D), dtype=torch.uint8, device=dev)
    dws = torch.empty(gqa.decode_workspace_size(dB, dH, dHkv, max_len, D), dtype=torch.uint8, device=dev)
    ptr = lambda t: t.data_ptr()  # noqa: E731
    p_in = sum(t.numel() * t.element_size() for t in hp.values())
    d_in = sum(t.numel() * t.element_size() for t in hd.values())
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def prefill_set():
        d = {n: torch.empty_like(t, device=dev) for n, t in hp.items()}
        d["out"] = torch.empty((B, T, H, D), dtype=torch.float32, device=dev)
        return d

    def prefill_call(d):
        return lib.gqa_attn_prefill(ptr(d["q"]), ptr(d["k"]), ptr(d["v"]), ptr(d["pos"]), ptr(d["wq"]),
                                    ptr(d["wk"]), pin.theta, pin.eps, ptr(d["out"]), B, T, H, Hkv, D, ptr(pws),
                                    pws.numel(), sh)

    def decode_set():
        d = {n: torch.empty_like(t, device=dev) for n, t in hd.items()}
        d["out"] = torch.empty((dB, dH, D), dtype=torch.float32, device=dev)
        return d

    def decode_call(d):
        return lib.gqa_attn_decode(ptr(d["q"]), ptr(d["k_cache"]), ptr(d["v_cache"]), ptr(d["offsets"]),
                                   ptr(d["seqlens"]), None, ptr(d["wq"]), dec.theta, dec.eps, ptr(d["out"]), dB, dH,
                                   dHkv, D, max_len, ptr(dws), dws.numel(), sh)

    def run(host_in, host_out, sets, call, n):
        """n pipelined steps; returns the device time from the first copy in to the last copy out."""
        ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
        computed, copied = [None, None], [None, None]
        start, end = ev(), ev()
        start.record(s_in)
        for i in range(n):
            d = sets[i % 2]
            with torch.cuda.stream(s_in):
                if computed[i % 2] is not None:
                    s_in.wait_event(computed[i % 2])       # the call two steps back has read this set
                for k in host_in:
                    d[k].copy_(host_in[k], non_blocking=True)
                loaded = ev()
                loaded.record(s_in)
            stream.wait_event(loaded)
            if copied[i % 2] is not None:
                stream.wait_event(copied[i % 2])           # this set's previous result has been read out
            if call(d) != 0:
                raise RuntimeError("e2e call failed")
            computed[i % 2] = ev()
            computed[i % 2].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(computed[i % 2])
                host_out.copy_(d["out"], non_blocking=True)
                copied[i % 2] = ev()
                copied[i % 2].record(s_out)
        end.record(s_out)
        torch.cuda.synchronize()
        return start.elapsed_time(end) / 1e3

    res = {}
    for name, make_set, call, host_in, host_out, units, unit, scale, b_in in (
            ("prefill", prefill_set, prefill_call, hp, hout, prefill_flops(B, T, H, D), "TFLOP/s", 1e12, p_in),
            ("decode", decode_set, decode_call, hd, hdout, decode_bytes(dec.seqlens.tolist(), dH, dHkv, D), "GB/s",
             1e9, d_in)):
        sets = [make_set(), make_set()]
        run(host_in, host_out, sets, call, 2)   # warm-up
        if world > 1:
            torch.distributed.barrier()
        sec = max_over_ranks([run(host_in, host_out, sets, call, steps) * 1e3], dev, world)[0] / 1e3
        res[name] = {"value": round(whole_job_rate(units * steps, world, sec) / scale, 3), "unit": unit,
                     "h2d_bytes_per_step": int(b_in), "d2h_bytes_per_step": int(host_out.numel() * 4),
                     "steps": steps, "pipelined": "copies in, calls and copies out on three streams, "
                                                  "two device buffer sets"}
        del sets
    return res


# ----------------------------------------------------------------------------- oracle (CPU)
def _prefill_sample_rows(T, H, B, n, seed):
    rng = np.random.default_rng(seed)
    return np.stack([rng.integers(0, B, n), rng.integers(0, H, n), rng.integers(0, T, n)], 1).astype(np.int64)


def oracle_prefill_sample(pin, rows):
    from oracle import oracle
    b = synthetic.bf16_bits
    t0 = time.perf_counter()
    oracle.prefill_rows(b(pin.q), b(pin.k), b(pin.v), pin.pos.numpy(), pin.wq.numpy(), pin.wk.numpy(), pin.theta,
                        pin.eps, rows)
    sec = time.perf_counter() - t0
    D = pin.q.shape[-1]
    return float(np.sum(rows[:, 2] + 1) * 4 * D), sec   # 4*D FLOP per visible (i, j) pair


def oracle_decode_sample(dec, idx):
    from oracle import oracle
    b = synthetic.bf16_bits
    offs = dec.offsets.numpy()
    sl = dec.seqlens.numpy()
    H, D = dec.q.shape[1], dec.q.shape[2]
    Hkv = dec.k_cache.shape[1]
    lo, hi = int(offs[idx].min()), int((offs[idx] + sl[idx]).max())
    kc = b(dec.k_cache[lo:hi])
    vc = b(dec.v_cache[lo:hi])
    t0 = time.perf_counter()
    oracle.decode(b(dec.q)[idx], kc, vc, np.append(offs[idx], hi) - lo, sl[idx], None, dec.wq.numpy(), dec.theta,
                  dec.eps)
    sec = time.perf_counter() - t0
    return float(decode_bytes(sl[idx].tolist(), H, Hkv, D)), sec


def cpu_baseline(pin, dec, budget_s=20.0):
    """The oracle as it stands on the host cores, on bounded samples of both workloads."""
    from oracle import oracle
    B, T, H, D = pin.q.shape
    oracle.num_threads()   # build + load before timing
    # prefill: random rows of the large workload, doubled until about half the budget
    n = 64
    fl, sec = oracle_prefill_sample(pin, _prefill_sample_rows(T, H, B, n, 0))
    while sec < budget_s / 4 and n < 1 << 16:
        n *= 2
        fl, sec = oracle_prefill_sample(pin, _prefill_sample_rows(T, H, B, n, n))
    # decode: whole sequences (all heads), shortest first, about the other half
    order = np.argsort(dec.seqlens.numpy())
    m = 1
    by, dsec = oracle_decode_sample(dec, order[:m])
    while dsec < budget_s / 4 and m < len(order):
        m = min(len(order), m * 2)
        by, dsec = oracle_decode_sample(dec, np.sort(order[:m]))
    return {"value": round(fl / sec / 1e12, 6), "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"prefill: {n} random output rows (b, head, i) of the {WORKLOAD_TEXT[PREFILL]}, "
                      f"{sec:.1f} s; fp64 C, OpenMP",
            "decode": {"value": round(by / dsec / 1e9, 4), "unit": "GB/s",
                       "sample": f"decode: the {m} shortest sequences of the batched decode, all heads, {dsec:.1f} s"}}


def run_reference(args, rank, world):
    """The reference arm: the fp64 oracle as it stands, on the host cores; each step is a
    bounded sample (prefill rows + one decode sequence) of the same workloads."""
    if rank != 0:
        return None
    from oracle import oracle
    pin = synthetic.make(PREFILL)
    dec = synthetic.make(DECODE)
    B, T, H, D = pin.q.shape
    order = np.argsort(dec.seqlens.numpy())
    rows_per_step = 16
    fl_t = sec_t = by_t = dsec_t = 0.0
    for i in range(args.warmup + args.steps):
        rows = _prefill_sample_rows(T, H, B, rows_per_step, 1000 + i)
        fl, sec = oracle_prefill_sample(pin, rows)
        by, dsec = oracle_decode_sample(dec, order[i % 4:i % 4 + 1])
        if i >= args.warmup:
            fl_t += fl
            sec_t += sec
            by_t += by
            dsec_t += dsec
    value = fl_t / sec_t / 1e12
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * (sec_t + dsec_t) / args.steps, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{WORKLOAD_TEXT[PREFILL]} + {WORKLOAD_TEXT[DECODE]}",
                   "sample_per_step": f"{rows_per_step} prefill output rows + 1 decode sequence (all heads)"},
        "decode": {"value": round(by_t / dsec_t / 1e9, 4), "unit": "GB/s"},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": f"{rows_per_step} random prefill rows + 1 decode sequence per step"},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=20.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        ap.error("--warmup must be at least 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and args.impl == "ours":
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    try:
        line = run_reference(args, rank, world) if args.impl == "reference" else run_ours(args, rank, world,
                                                                                          local_rank)
    finally:
        if world > 1 and args.impl == "ours":
            torch.distributed.destroy_process_group()
    if rank == 0 and line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
