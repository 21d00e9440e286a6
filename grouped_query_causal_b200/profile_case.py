"""Run one prefill, decode, paged-decode or projection workload a few times on cuda:0 (for
profilers such as ncu).

    python -m grouped_query_causal_b200.profile_case prefill --B 2 --T 4096 --H 32 --Hkv 8 --iters 2
    python -m grouped_query_causal_b200.profile_case decode --B 16 --len 16384 --H 32 --Hkv 8 --iters 2
    python -m grouped_query_causal_b200.profile_case paged --B 16 --len 16384 --H 32 --Hkv 8 --iters 2
    python -m grouped_query_causal_b200.profile_case linear --M 4096 --N 6144 --K 4096 --iters 2
    python -m grouped_query_causal_b200.profile_case workload --name long_context_prefill --iters 2

`workload` runs one of the named synthetic workloads exactly as the benchmark does (same
inputs and launch), so that counters taken on it are per bench launch.

Inputs are random on the device (their values do not matter for timing or counters);
each iteration is one full library call: k-hat prologue + attention for prefill,
split + merge for decode, one GEMM for linear.  Prints the CUDA-event time of each iteration.
"""
from __future__ import annotations

import argparse

import torch

from . import binding


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("kind", choices=["prefill", "decode", "paged", "linear", "workload"])
    ap.add_argument("--name", default="long_context_prefill", help="workload: a name from synthetic.WORKLOADS")
    ap.add_argument("--M", type=int, default=4096)
    ap.add_argument("--N", type=int, default=6144)
    ap.add_argument("--K", type=int, default=4096)
    ap.add_argument("--page", type=int, default=64, help="paged: rows per page")
    ap.add_argument("--B", type=int, default=2)
    ap.add_argument("--T", type=int, default=4096)
    ap.add_argument("--len", type=int, default=16384, help="decode: cached tokens per sequence")
    ap.add_argument("--H", type=int, default=32)
    ap.add_argument("--Hkv", type=int, default=8)
    ap.add_argument("--iters", type=int, default=2)
    a = ap.parse_args(argv)
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    g = torch.Generator(device=dev)
    g.manual_seed(0)
    D = 128
    wq = torch.rand(D, device=dev, generator=g) + 0.5
    wk = torch.rand(D, device=dev, generator=g) + 0.5
    if a.kind == "prefill":
        q = torch.randn(a.B, a.T, a.H, D, device=dev, generator=g).to(torch.bfloat16)
        k = torch.randn(a.B, a.T, a.Hkv, D, device=dev, generator=g).to(torch.bfloat16)
        v = torch.randn(a.B, a.T, a.Hkv, D, device=dev, generator=g).to(torch.bfloat16)
        pos = torch.arange(a.T, dtype=torch.int32, device=dev).repeat(a.B, 1).contiguous()
        out = torch.empty(a.B, a.T, a.H, D, device=dev)
        ws = torch.empty(binding.prefill_workspace_size(a.B, a.T, a.H, a.Hkv), dtype=torch.uint8, device=dev)
        run = lambda: binding.prefill(q, k, v, pos, wq, wk, out=out, workspace=ws)  # noqa: E731
        flops = a.B * a.H * 2 * D * a.T * (a.T + 1)
        unit, scale = "TFLOP/s", 1e12
    elif a.kind == "workload":
        from . import synthetic
        w = synthetic.make(a.name)
        kind = synthetic.WORKLOADS[a.name]["kind"]
        if kind == "prefill":
            t = [x.to(dev) for x in (w.q, w.k, w.v, w.pos, w.wq, w.wk)]
            B, T, H, D = w.q.shape
            Hkv = w.k.shape[2]
            out = torch.empty(B, T, H, D, device=dev)
            ws = torch.empty(binding.prefill_workspace_size(B, T, H, Hkv), dtype=torch.uint8, device=dev)
            run = lambda: binding.prefill(*t, w.theta, w.eps, out=out, workspace=ws)  # noqa: E731
            flops = B * H * 2 * D * T * (T + 1)
            unit, scale = "TFLOP/s", 1e12
        elif kind == "decode":
            q, kc, vc, offs, sl, dwq = (x.to(dev) for x in (w.q, w.k_cache, w.v_cache, w.offsets, w.seqlens, w.wq))
            B, H, D = w.q.shape
            Hkv = w.k_cache.shape[1]
            out = torch.empty(B, H, D, device=dev)
            ws = torch.empty(binding.decode_workspace_size(B, H, Hkv, w.max_len), dtype=torch.uint8, device=dev)
            run = lambda: binding.decode(q, kc, vc, offs, sl, dwq, w.max_len, out=out, workspace=ws)  # noqa: E731
            flops = int(w.seqlens.sum()) * Hkv * D * 2 * 2
            unit, scale = "GB/s", 1e9
        else:
            raise SystemExit(f"workload {a.name}: kind {kind} is not run here")
    elif a.kind == "linear":
        x = torch.randn(a.M, a.K, device=dev, generator=g).to(torch.bfloat16)
        w = (torch.randn(a.N, a.K, device=dev, generator=g) / a.K ** 0.5).to(torch.bfloat16)
        out = torch.empty(a.M, a.N, dtype=torch.bfloat16, device=dev)
        run = lambda: binding.linear(x, w, out=out)  # noqa: E731
        flops = 2 * a.M * a.N * a.K
        unit, scale = "TFLOP/s", 1e12
    elif a.kind == "paged":
        # every sequence's pages in a shuffled order over one pool
        npg = (a.len + a.page - 1) // a.page
        q = torch.randn(a.B, a.H, D, device=dev, generator=g).to(torch.bfloat16)
        kp = torch.randn(a.B * npg, a.page, a.Hkv, D, device=dev, generator=g).to(torch.bfloat16)
        vp = torch.randn(a.B * npg, a.page, a.Hkv, D, device=dev, generator=g).to(torch.bfloat16)
        table = torch.randperm(a.B * npg, device=dev, generator=g).to(torch.int32).view(a.B, npg)
        sl = torch.full((a.B,), a.len, dtype=torch.int32, device=dev)
        out = torch.empty(a.B, a.H, D, device=dev)
        ws = torch.empty(binding.decode_workspace_size(a.B, a.H, a.Hkv, a.len), dtype=torch.uint8, device=dev)
        rope = binding.RopeConfig.make()
        run = lambda: binding.decode_paged(q, kp, vp, table, sl, wq, a.len, rope=rope, out=out,  # noqa: E731
                                           workspace=ws)
        flops = a.B * a.len * a.Hkv * D * 2 * 2   # bytes, for decode
        unit, scale = "GB/s", 1e9
    else:
        rows = a.B * a.len
        q = torch.randn(a.B, a.H, D, device=dev, generator=g).to(torch.bfloat16)
        kc = torch.randn(rows, a.Hkv, D, device=dev, generator=g).to(torch.bfloat16)
        vc = torch.randn(rows, a.Hkv, D, device=dev, generator=g).to(torch.bfloat16)
        offs = torch.arange(a.B + 1, dtype=torch.int64, device=dev) * a.len
        sl = torch.full((a.B,), a.len, dtype=torch.int32, device=dev)
        out = torch.empty(a.B, a.H, D, device=dev)
        ws = torch.empty(binding.decode_workspace_size(a.B, a.H, a.Hkv, a.len), dtype=torch.uint8, device=dev)
        run = lambda: binding.decode(q, kc, vc, offs, sl, wq, a.len, out=out, workspace=ws)  # noqa: E731
        flops = rows * a.Hkv * D * 2 * 2   # bytes, for decode
        unit, scale = "GB/s", 1e9
    for i in range(a.iters):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        run()
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1)
        print(f"{a.kind} iter {i}: {ms:.4f} ms, {flops / (ms / 1e3) / scale:.1f} {unit}")
    binding.check_device_status()


if __name__ == "__main__":
    main()
