"""Shared helpers for the GPU parity tests (oracle comparison, tolerances)."""
import numpy as np
import torch

from grouped_query_causal_b200 import synthetic

# Tolerance on every output element against the fp64 oracle: bf16 inputs, fp32
# accumulation, q-hat/k-hat/P rounded to bf16 for the tensor cores.
MAX_ABS = 2e-2
MEAN_ABS = 2e-3


def bits(t):
    return synthetic.bf16_bits(t)


def assert_close(got, ref, what=""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    err = np.abs(got - ref)
    mx, mean = float(err.max()) if err.size else 0.0, float(err.mean()) if err.size else 0.0
    assert mx <= MAX_ABS and mean <= MEAN_ABS, f"{what}: max-abs {mx:.3e}, mean-abs {mean:.3e}"
    return mx, mean


def to_dev(inp: synthetic.PrefillInputs, dev="cuda"):
    return dict(q=inp.q.to(dev), k=inp.k.to(dev), v=inp.v.to(dev), pos=inp.pos.to(dev),
                qnorm_w=inp.wq.to(dev), knorm_w=inp.wk.to(dev), theta=inp.theta, eps=inp.eps)


def oracle_prefill_args(inp: synthetic.PrefillInputs):
    return (bits(inp.q), bits(inp.k), bits(inp.v), inp.pos.numpy(), inp.wq.numpy(), inp.wk.numpy(),
            inp.theta, inp.eps)


def strided_rows(B, T, H, stride, edges=(), tail_heads=(), tail=0, whole_heads=()):
    """(b, hq, i) rows for a full-size prefill check: every `stride`-th row of every head
    (the phase shifts from head to head, so that together the heads cover every row
    offset inside a 128-row tile), the rows `edges` of every head, the last `tail` rows
    of every head in `tail_heads`, and every row of the (b, hq) heads in `whole_heads`."""
    rows = set()
    for b in range(B):
        for hq in range(H):
            phase = (7 * hq + 3 * b) % stride
            rows.update((b, hq, i) for i in range(phase, T, stride))
            rows.update((b, hq, i) for i in edges if 0 <= i < T)
            if hq in tail_heads:
                rows.update((b, hq, i) for i in range(max(0, T - tail), T))
    for b, hq in whole_heads:
        rows.update((b, hq, i) for i in range(T))
    return np.array(sorted(rows), dtype=np.int64)


def decode_to_dev(inp: synthetic.DecodeInputs, dev="cuda"):
    return dict(q=inp.q.to(dev), k_cache=inp.k_cache.to(dev), v_cache=inp.v_cache.to(dev),
                cache_offsets=inp.offsets.to(dev), seqlens=inp.seqlens.to(dev), qnorm_w=inp.wq.to(dev),
                theta=inp.theta, eps=inp.eps)
