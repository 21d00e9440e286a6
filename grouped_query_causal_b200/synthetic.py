"""Seeded synthetic inputs for the attention sub-block.

Holds none of the method's arithmetic: only seeded random tensors with the
shapes, value distributions and structure of the documented workloads.  Every
tensor is produced on the CPU with its own ``torch.Generator`` (seed, seed+1, ...)
so that a CPU check and the GPU path see the same bits.

* q, k, v: fp32 N(0, 1) (times an optional scale), rounded to bf16 (round to
  nearest even, torch's conversion).
* q/k norm weights: fp32 U(0.5, 1.5).
* positions: 0 .. T-1 per sequence (int32).
* decode: per-sequence cache lengths uniform on [len_lo, len_hi]; K and V cache
  rows N(0, 1) bf16, packed sequence after sequence as [rows, Hkv, D].
* packed prefill: sequence lengths uniform on [len_lo, len_hi], tokens packed; a
  chunk after a cached prefix adds a cache whose prefix rows are N(0, 1) bf16.
* projections: hidden states N(0, 1) bf16, weights N(0, 1/fan-in) bf16.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

EPS = 1e-6
THETA = 1.0e6
HEAD_DIM = 128


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def _normal_bf16(shape, seed: int, scale: float = 1.0, chunk: int = 1 << 26) -> torch.Tensor:
    """N(0,1)*scale rounded to bf16, drawn in chunks to bound host memory."""
    n = int(np.prod(shape)) if len(shape) else 1
    out = torch.empty(n, dtype=torch.bfloat16)
    g = _gen(seed)
    for s in range(0, n, chunk):
        e = min(n, s + chunk)
        x = torch.randn(e - s, generator=g, dtype=torch.float32)
        if scale != 1.0:
            x.mul_(scale)
        out[s:e] = x.to(torch.bfloat16)
    return out.view(*shape)


def _uniform(shape, seed: int, lo: float, hi: float) -> torch.Tensor:
    return torch.rand(*shape, generator=_gen(seed), dtype=torch.float32) * (hi - lo) + lo


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """Raw bf16 bit patterns of a CPU bf16 tensor as a uint16 numpy array."""
    assert t.dtype == torch.bfloat16
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


@dataclass
class PrefillInputs:
    q: torch.Tensor      # bf16 [B,T,H,D]
    k: torch.Tensor      # bf16 [B,T,Hkv,D]
    v: torch.Tensor      # bf16 [B,T,Hkv,D]
    pos: torch.Tensor    # int32 [B,T]
    wq: torch.Tensor     # fp32 [D]
    wk: torch.Tensor     # fp32 [D]
    theta: float = THETA
    eps: float = EPS


def prefill_inputs(B: int, T: int, H: int, Hkv: int, D: int = HEAD_DIM, seed: int = 0,
                   scale: float = 1.0) -> PrefillInputs:
    q = _normal_bf16((B, T, H, D), seed, scale)
    k = _normal_bf16((B, T, Hkv, D), seed + 1, scale)
    v = _normal_bf16((B, T, Hkv, D), seed + 2, scale)
    wq = _uniform((D,), seed + 3, 0.5, 1.5)
    wk = _uniform((D,), seed + 4, 0.5, 1.5)
    pos = torch.arange(T, dtype=torch.int32).repeat(B, 1).contiguous()
    return PrefillInputs(q, k, v, pos, wq, wk)


@dataclass
class DecodeInputs:
    q: torch.Tensor        # bf16 [B,H,D]
    k_cache: torch.Tensor  # bf16 [rows,Hkv,D]
    v_cache: torch.Tensor  # bf16 [rows,Hkv,D]
    offsets: torch.Tensor  # int64 [B+1], rows of sequence b: offsets[b] .. offsets[b+1]-1
    seqlens: torch.Tensor  # int32 [B]
    wq: torch.Tensor       # fp32 [D]
    theta: float = THETA
    eps: float = EPS

    @property
    def max_len(self) -> int:
        return int(self.seqlens.max()) if self.seqlens.numel() else 0


def decode_inputs(B: int = 64, H: int = 32, Hkv: int = 8, D: int = HEAD_DIM, seed: int = 0,
                  len_lo: int = 1024, len_hi: int = 32768, seqlens=None) -> DecodeInputs:
    if seqlens is None:
        seqlens = torch.randint(len_lo, len_hi + 1, (B,), generator=_gen(seed + 10),
                                dtype=torch.int64)
    seqlens = torch.as_tensor(seqlens, dtype=torch.int64).reshape(B)
    offsets = torch.zeros(B + 1, dtype=torch.int64)
    offsets[1:] = torch.cumsum(seqlens, 0)
    rows = int(offsets[-1])
    q = _normal_bf16((B, H, D), seed)
    k_cache = _normal_bf16((rows, Hkv, D), seed + 1)
    v_cache = _normal_bf16((rows, Hkv, D), seed + 2)
    wq = _uniform((D,), seed + 3, 0.5, 1.5)
    return DecodeInputs(q, k_cache, v_cache, offsets, seqlens.to(torch.int32), wq)


@dataclass
class DecodeAppendInputs:
    q: torch.Tensor        # bf16 [B,H,D], the new token's raw query
    k_new: torch.Tensor    # bf16 [B,Hkv,D], the new token's raw key
    v_new: torch.Tensor    # bf16 [B,Hkv,D], the new token's value
    k_cache: torch.Tensor  # bf16 [rows,Hkv,D]; rows past a sequence's length hold stale data
    v_cache: torch.Tensor  # bf16 [rows,Hkv,D]
    offsets: torch.Tensor  # int64 [B+1]; sequence b owns rows offsets[b] .. offsets[b+1]-1
    seqlens: torch.Tensor  # int32 [B], cached rows before the step (>= 0)
    wq: torch.Tensor       # fp32 [D]
    wk: torch.Tensor       # fp32 [D]
    theta: float = THETA
    eps: float = EPS

    @property
    def max_len(self) -> int:
        """Keys attended after the append: the longest length + 1."""
        return int(self.seqlens.max()) + 1 if self.seqlens.numel() else 0


def decode_append_inputs(B: int = 64, H: int = 32, Hkv: int = 8, D: int = HEAD_DIM, seed: int = 0,
                         len_lo: int = 1023, len_hi: int = 32767, seqlens=None,
                         spare: int = 1) -> DecodeAppendInputs:
    """A cache with `spare` free rows after each sequence's cached rows, plus one new token
    per sequence.  Lengths U{len_lo..len_hi} unless given; every other value as in
    decode_inputs."""
    if seqlens is None:
        seqlens = torch.randint(len_lo, len_hi + 1, (B,), generator=_gen(seed + 10), dtype=torch.int64)
    seqlens = torch.as_tensor(seqlens, dtype=torch.int64).reshape(B)
    offsets = torch.zeros(B + 1, dtype=torch.int64)
    offsets[1:] = torch.cumsum(seqlens + spare, 0)
    rows = int(offsets[-1])
    q = _normal_bf16((B, H, D), seed)
    k_cache = _normal_bf16((rows, Hkv, D), seed + 1)
    v_cache = _normal_bf16((rows, Hkv, D), seed + 2)
    wq = _uniform((D,), seed + 3, 0.5, 1.5)
    wk = _uniform((D,), seed + 4, 0.5, 1.5)
    k_new = _normal_bf16((B, Hkv, D), seed + 5)
    v_new = _normal_bf16((B, Hkv, D), seed + 6)
    return DecodeAppendInputs(q, k_new, v_new, k_cache, v_cache, offsets, seqlens.to(torch.int32), wq, wk)


@dataclass
class PagedCache:
    k_pages: torch.Tensor     # bf16 [num_pages, page_size, Hkv, D]
    v_pages: torch.Tensor     # bf16 [num_pages, page_size, Hkv, D]
    page_table: torch.Tensor  # int32 [B, max_pages]; unused entries -1
    page_size: int


def page_cache(k_rows: torch.Tensor, v_rows: torch.Tensor, offsets, capacities, page_size: int, seed: int = 0,
               spare_pages: int = 3) -> PagedCache:
    """Scatter per-sequence rows (sequence b: rows offsets[b] .. + capacities[b]) into
    pages of page_size rows, pages handed out in a seeded random order with a few unused
    ones; the tail of a sequence's last page is zero."""
    B = len(capacities)
    Hkv, D = k_rows.shape[1], k_rows.shape[2]
    need = [(int(c) + page_size - 1) // page_size for c in capacities]
    max_pages = max(1, max(need))
    num_pages = sum(need) + spare_pages
    order = torch.randperm(num_pages, generator=_gen(seed + 20)).tolist()
    kp = torch.zeros(num_pages, page_size, Hkv, D, dtype=k_rows.dtype)
    vp = torch.zeros_like(kp)
    table = torch.full((B, max_pages), -1, dtype=torch.int32)
    nxt = 0
    for b in range(B):
        o = int(offsets[b])
        for j in range(need[b]):
            pid = order[nxt]
            nxt += 1
            table[b, j] = pid
            lo = j * page_size
            n = min(page_size, int(capacities[b]) - lo)
            kp[pid, :n] = k_rows[o + lo:o + lo + n]
            vp[pid, :n] = v_rows[o + lo:o + lo + n]
    return PagedCache(kp, vp, table, page_size)


@dataclass
class PackedInputs:
    """Sequences packed token after token: q [N,H,D], k/v [N,Hkv,D] raw bf16, positions
    [N] (each sequence from prefix[b] on), cu [B+1] token offsets; for a chunk after a
    cached prefix also the cache (k-hat / v rows of the prefix, room for the chunk)."""
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    pos: torch.Tensor
    cu: torch.Tensor
    wq: torch.Tensor
    wk: torch.Tensor
    prefix: torch.Tensor = None      # int32 [B] cached rows (chunk workloads)
    k_cache: torch.Tensor = None     # bf16 [rows, Hkv, D]
    v_cache: torch.Tensor = None
    cache_offsets: torch.Tensor = None   # int64 [B+1]
    theta: float = THETA
    eps: float = EPS

    @property
    def lens(self):
        return (self.cu[1:] - self.cu[:-1]).tolist()


def packed_inputs(lens, H: int, Hkv: int, D: int = HEAD_DIM, seed: int = 0, prefix=None) -> PackedInputs:
    """Packed sequences of the given lengths, N(0,1) bf16 q/k/v, U(0.5, 1.5) norm weights.
    With prefix (rows already cached per sequence), a cache of prefix[b] + lens[b] rows
    per sequence is added whose first prefix[b] rows hold N(0,1) bf16 values (they stand
    in for cached k-hat and v, as in the decode workloads)."""
    B = len(lens)
    N = int(sum(lens))
    cu = torch.zeros(B + 1, dtype=torch.int64)
    cu[1:] = torch.cumsum(torch.as_tensor(lens, dtype=torch.int64), 0)
    pre = [0] * B if prefix is None else [int(p) for p in prefix]
    pos = torch.cat([torch.arange(p, p + n, dtype=torch.int32) for p, n in zip(pre, lens)]) if N else \
        torch.zeros(0, dtype=torch.int32)
    out = PackedInputs(_normal_bf16((N, H, D), seed), _normal_bf16((N, Hkv, D), seed + 1),
                       _normal_bf16((N, Hkv, D), seed + 2), pos, cu, _uniform((D,), seed + 3, 0.5, 1.5),
                       _uniform((D,), seed + 4, 0.5, 1.5))
    if prefix is not None:
        caps = torch.as_tensor([p + n for p, n in zip(pre, lens)], dtype=torch.int64)
        offs = torch.zeros(B + 1, dtype=torch.int64)
        offs[1:] = torch.cumsum(caps, 0)
        out.prefix = torch.as_tensor(pre, dtype=torch.int32)
        out.k_cache = _normal_bf16((int(offs[-1]), Hkv, D), seed + 5)
        out.v_cache = _normal_bf16((int(offs[-1]), Hkv, D), seed + 6)
        out.cache_offsets = offs
    return out


@dataclass
class ProjectionInputs:
    """Hidden states x [N, hidden] bf16 N(0,1) and projection weights scaled by
    1/sqrt(fan-in): w_qkv [(H + 2 Hkv) D, hidden], w_o [hidden, H D]."""
    x: torch.Tensor
    w_qkv: torch.Tensor
    w_o: torch.Tensor
    H: int
    Hkv: int


def projection_inputs(N: int, hidden: int, H: int, Hkv: int, D: int = HEAD_DIM, seed: int = 0) -> ProjectionInputs:
    x = _normal_bf16((N, hidden), seed)
    w_qkv = _normal_bf16(((H + 2 * Hkv) * D, hidden), seed + 1, 1.0 / hidden ** 0.5)
    w_o = _normal_bf16((hidden, H * D), seed + 2, 1.0 / (H * D) ** 0.5)
    return ProjectionInputs(x, w_qkv, w_o, H, Hkv)


# The documented workloads, by name.
WORKLOADS = {
    "prefill_correctness": dict(kind="prefill", B=1, T=128, H=16, Hkv=8),
    "gqa_sweep_mha": dict(kind="prefill", B=2, T=512, H=16, Hkv=16),
    "gqa_sweep_hkv8": dict(kind="prefill", B=2, T=512, H=16, Hkv=8),
    "gqa_sweep_hkv4": dict(kind="prefill", B=2, T=512, H=16, Hkv=4),
    "gqa_sweep_mqa": dict(kind="prefill", B=2, T=512, H=16, Hkv=1),
    "large_prefill": dict(kind="prefill", B=4, T=4096, H=32, Hkv=8, scale=0.5),
    "batched_decode": dict(kind="decode", B=64, H=32, Hkv=8, len_lo=1024, len_hi=32768),
    "long_context_prefill": dict(kind="prefill", B=1, T=32768, H=64, Hkv=8),
    "batched_decode_append": dict(kind="decode_append", B=64, H=32, Hkv=8, len_lo=1023, len_hi=32767),
    # 16 packed sequences, lengths U{256..8192}
    "varlen_prefill": dict(kind="packed", B=16, H=32, Hkv=8, len_lo=256, len_hi=8192),
    # 8 sequences with 8192 cached rows each and a new chunk of 2048 tokens
    "chunked_prefill": dict(kind="chunk", B=8, H=32, Hkv=8, prefix=8192, chunk=2048),
    # the projections around the large prefill's attention: 16384 tokens, hidden 4096
    "projections": dict(kind="projection", N=16384, hidden=4096, H=32, Hkv=8),
}


def make(name: str, seed: int = 0):
    w = dict(WORKLOADS[name])
    kind = w.pop("kind")
    if kind == "prefill":
        return prefill_inputs(seed=seed, **w)
    if kind == "decode_append":
        return decode_append_inputs(seed=seed, **w)
    if kind == "packed":
        lens = torch.randint(w["len_lo"], w["len_hi"] + 1, (w["B"],), generator=_gen(seed + 10)).tolist()
        return packed_inputs(lens, w["H"], w["Hkv"], seed=seed)
    if kind == "chunk":
        return packed_inputs([w["chunk"]] * w["B"], w["H"], w["Hkv"], seed=seed, prefix=[w["prefix"]] * w["B"])
    if kind == "projection":
        return projection_inputs(w["N"], w["hidden"], w["H"], w["Hkv"], seed=seed)
    return decode_inputs(seed=seed, **w)
