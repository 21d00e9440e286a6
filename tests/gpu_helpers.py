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


def sample_rows(B, T, H, n_random, seed=0):
    """(b, hq, i) rows: tile edges, the first and last rows, and random ones."""
    rng = np.random.default_rng(seed)
    rows = set()
    edges = [0, 1, 126, 127, 128, 129, 255, 256, T // 2, T - 129, T - 128, T - 2, T - 1]
    for b in range(B):
        for i in edges:
            if 0 <= i < T:
                rows.add((b, int(rng.integers(H)), i))
                rows.add((b, H - 1, i))
    for _ in range(n_random):
        rows.add((int(rng.integers(B)), int(rng.integers(H)), int(rng.integers(T))))
    return np.array(sorted(rows), dtype=np.int64)


def decode_to_dev(inp: synthetic.DecodeInputs, dev="cuda"):
    return dict(q=inp.q.to(dev), k_cache=inp.k_cache.to(dev), v_cache=inp.v_cache.to(dev),
                cache_offsets=inp.offsets.to(dev), seqlens=inp.seqlens.to(dev), qnorm_w=inp.wq.to(dev),
                theta=inp.theta, eps=inp.eps)
