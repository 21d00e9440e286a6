"""ctypes front end of the fp64 CPU oracle (``gqa_oracle.c``).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU
baseline leg are the only callers.  The product path (the CUDA library and its
Python binding) never imports this module, and this module never imports the
product path.

Inputs are numpy arrays: bf16 tensors travel as their raw ``uint16`` bit
patterns, positions as ``int32``, norm weights as ``float32``; every output is
``float64``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gqa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ``gqa_oracle.c`` into ``liboracle.so`` beside it (gcc, OpenMP)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c11", "-Wall",
           "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            I, L, Dd = ctypes.c_int, ctypes.c_int64, ctypes.c_double
            lib.oracle_rmsnorm.argtypes = [P, P, Dd, I, P]
            lib.oracle_rope.argtypes = [P, Dd, Dd, I, P]
            lib.oracle_qk_transform.argtypes = [P, P, P, Dd, Dd, L, I, I, P]
            lib.oracle_sdpa_gqa.argtypes = [P, P, P, I, I, I, I, I, I, P, P]
            lib.oracle_prefill.argtypes = [P, P, P, P, P, P, Dd, Dd, I, I, I, I, I, P]
            lib.oracle_prefill_rows.argtypes = [P, P, P, P, P, P, Dd, Dd, I, I, I, I, I,
                                                L, P, P]
            lib.oracle_decode.argtypes = [P, P, P, P, P, P, P, Dd, Dd, I, I, I, I, P]
            lib.oracle_decode_append.argtypes = [P, P, P, P, P, P, P, P, P, P, Dd, Dd, I, I, I, I,
                                                 P, P]
            lib.oracle_rope_inv_freq.argtypes = [Dd, I, I, Dd, I, Dd, Dd, P]
            lib.oracle_rope_logit_mult.argtypes = [I, Dd]
            lib.oracle_rope_logit_mult.restype = Dd
            lib.oracle_rope_ex.argtypes = [P, Dd, P, I, I, P]
            lib.oracle_qk_transform_ex.argtypes = [P, P, P, P, I, Dd, L, I, I, P]
            lib.oracle_prefill_rows_ex.argtypes = [P, P, P, P, P, P, P, I, Dd, Dd, I, I, I, I, I, L,
                                                   P, P]
            lib.oracle_decode_ex.argtypes = [P, P, P, P, P, P, P, P, I, Dd, Dd, I, I, I, I, P]
            lib.oracle_decode_append_ex.argtypes = [P, P, P, P, P, P, P, P, P, P, P, I, Dd, Dd, I, I,
                                                    I, I, P, P]
            lib.oracle_prefill_chunk_ex.argtypes = [P, P, P, P, P, P, P, P, P, P, P, I, Dd, Dd, I, I, I,
                                                    I, I, P, P]
            lib.oracle_prefill_chunk_rows_ex.argtypes = [P, P, P, P, P, P, P, P, P, P, P, I, Dd, Dd, I, I, I,
                                                         I, I, L, P, P, P]
            lib.oracle_prefill_varlen_ex.argtypes = [P, P, P, P, P, P, P, P, I, Dd, Dd, I, I, I, I, P]
            lib.oracle_linear.argtypes = [P, P, L, L, L, P]
            lib.oracle_num_threads.restype = I
            _lib = lib
    return _lib


def _c(a: np.ndarray, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


def _p(a) -> ctypes.c_void_p:
    return ctypes.c_void_p(0) if a is None else ctypes.c_void_p(a.ctypes.data)


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def rmsnorm(x, w, eps: float) -> np.ndarray:
    x = _c(x, np.float64)
    w = _c(w, np.float64)
    out = np.empty_like(x)
    _load().oracle_rmsnorm(_p(x), _p(w), eps, x.shape[-1], _p(out))
    return out


def rope(x, pos: float, theta: float) -> np.ndarray:
    x = _c(x, np.float64)
    out = np.empty_like(x)
    _load().oracle_rope(_p(x), float(pos), float(theta), x.shape[-1], _p(out))
    return out


def qk_transform(x_bits, pos, w, theta: float, eps: float) -> np.ndarray:
    """x_bits [N, nheads, D] uint16 (bf16 bits), pos [N] -> fp64 [N, nheads, D]."""
    x_bits = _c(x_bits, np.uint16)
    N, nh, D = x_bits.shape
    pos = _c(pos, np.int32).reshape(N)
    w = _c(w, np.float32)
    out = np.empty((N, nh, D), np.float64)
    _load().oracle_qk_transform(_p(x_bits), _p(pos), _p(w), theta, eps, N, nh, D, _p(out))
    return out


def sdpa_gqa(q, k, v, causal: bool = True, return_weights: bool = False):
    """fp64 q [B,T,H,D], k/v [B,T,Hkv,D] (already normed and rotated)."""
    q = _c(q, np.float64)
    k = _c(k, np.float64)
    v = _c(v, np.float64)
    B, T, H, D = q.shape
    Hkv = k.shape[2]
    assert H % Hkv == 0
    out = np.empty((B, T, H, D), np.float64)
    w = np.empty((B, H, T, T), np.float64) if return_weights else None
    _load().oracle_sdpa_gqa(_p(q), _p(k), _p(v), B, T, H, Hkv, D, int(bool(causal)),
                            _p(out), _p(w))
    return (out, w) if return_weights else out


def prefill(q_bits, k_bits, v_bits, pos, wq, wk, theta: float, eps: float) -> np.ndarray:
    """Whole prefill sub-block: bf16 bits q [B,T,H,D], k/v [B,T,Hkv,D]; pos [B,T]."""
    q_bits = _c(q_bits, np.uint16)
    k_bits = _c(k_bits, np.uint16)
    v_bits = _c(v_bits, np.uint16)
    B, T, H, D = q_bits.shape
    Hkv = k_bits.shape[2]
    assert H % Hkv == 0
    pos = _c(pos, np.int32).reshape(B, T)
    wq = _c(wq, np.float32)
    wk = _c(wk, np.float32)
    out = np.empty((B, T, H, D), np.float64)
    _load().oracle_prefill(_p(q_bits), _p(k_bits), _p(v_bits), _p(pos), _p(wq), _p(wk),
                           theta, eps, B, T, H, Hkv, D, _p(out))
    return out


def prefill_rows(q_bits, k_bits, v_bits, pos, wq, wk, theta: float, eps: float,
                 rows) -> np.ndarray:
    """Selected output rows of prefill; rows is an int array [n, 3] of (b, hq, i)."""
    q_bits = _c(q_bits, np.uint16)
    k_bits = _c(k_bits, np.uint16)
    v_bits = _c(v_bits, np.uint16)
    B, T, H, D = q_bits.shape
    Hkv = k_bits.shape[2]
    pos = _c(pos, np.int32).reshape(B, T)
    wq = _c(wq, np.float32)
    wk = _c(wk, np.float32)
    rows = _c(rows, np.int64).reshape(-1, 3)
    assert (rows[:, 0] < B).all() and (rows[:, 1] < H).all() and (rows[:, 2] < T).all()
    out = np.empty((rows.shape[0], D), np.float64)
    _load().oracle_prefill_rows(_p(q_bits), _p(k_bits), _p(v_bits), _p(pos), _p(wq),
                                _p(wk), theta, eps, B, T, H, Hkv, D, rows.shape[0],
                                _p(rows), _p(out))
    return out


def decode(q_bits, k_cache_bits, v_cache_bits, offsets, seqlens, qpos, wq, theta: float,
           eps: float) -> np.ndarray:
    """Decode: q [B,H,D] bf16 bits; caches [rows,Hkv,D] bf16 bits; offsets [B(+1)] int64;
    seqlens [B] int32 (>= 1); qpos [B] int32 or None (then qpos = seqlens)."""
    q_bits = _c(q_bits, np.uint16)
    k_cache_bits = _c(k_cache_bits, np.uint16)
    v_cache_bits = _c(v_cache_bits, np.uint16)
    B, H, D = q_bits.shape
    Hkv = k_cache_bits.shape[1]
    offsets = _c(offsets, np.int64)
    seqlens = _c(seqlens, np.int32)
    assert (seqlens >= 1).all()
    qpos_a = None if qpos is None else _c(qpos, np.int32)
    wq = _c(wq, np.float32)
    out = np.empty((B, H, D), np.float64)
    _load().oracle_decode(_p(q_bits), _p(k_cache_bits), _p(v_cache_bits), _p(offsets),
                          _p(seqlens), _p(qpos_a), _p(wq), theta, eps, B, H, Hkv, D,
                          _p(out))
    return out


def decode_append(q_bits, k_new_bits, v_new_bits, k_cache_bits, v_cache_bits, offsets, seqlens,
                  qpos, wq, wk, theta: float, eps: float):
    """Decode step that appends the new token first: q [B,H,D], k_new / v_new [B,Hkv,D] bf16
    bits; caches [rows,Hkv,D] bf16 bits; offsets [B(+1)] int64; seqlens [B] int32 (>= 0);
    qpos [B] int32 or None (then qpos = seqlens).  Returns (out [B,H,D], k-hat of the
    appended rows [B,Hkv,D]), both fp64."""
    q_bits = _c(q_bits, np.uint16)
    k_new_bits = _c(k_new_bits, np.uint16)
    v_new_bits = _c(v_new_bits, np.uint16)
    k_cache_bits = _c(k_cache_bits, np.uint16)
    v_cache_bits = _c(v_cache_bits, np.uint16)
    B, H, D = q_bits.shape
    Hkv = k_new_bits.shape[1]
    assert k_new_bits.shape == (B, Hkv, D) and v_new_bits.shape == (B, Hkv, D)
    offsets = _c(offsets, np.int64)
    seqlens = _c(seqlens, np.int32)
    assert (seqlens >= 0).all()
    qpos_a = None if qpos is None else _c(qpos, np.int32)
    wq = _c(wq, np.float32)
    wk = _c(wk, np.float32)
    out = np.empty((B, H, D), np.float64)
    khat = np.empty((B, Hkv, D), np.float64)
    _load().oracle_decode_append(_p(q_bits), _p(k_new_bits), _p(v_new_bits), _p(k_cache_bits),
                                 _p(v_cache_bits), _p(offsets), _p(seqlens), _p(qpos_a), _p(wq),
                                 _p(wk), theta, eps, B, H, Hkv, D, _p(out), _p(khat))
    return out, khat


# ---- RoPE variants -------------------------------------------------------------------
SCALINGS = {"none": 0, "linear": 1, "ntk": 2, "yarn": 3}
PAIRINGS = {"adjacent": 0, "half": 1}


class Rope:
    """A RoPE variant: base theta, pairing ("adjacent" or "half"), scaling ("none",
    "linear", "ntk", "yarn") with factor s, and YaRN's training length and ramp bounds."""

    def __init__(self, theta=1.0e6, pairing="adjacent", scaling="none", factor=1.0,
                 original_max_position=4096, beta_fast=32.0, beta_slow=1.0):
        self.theta, self.pairing, self.scaling, self.factor = float(theta), pairing, scaling, float(factor)
        self.original_max_position = int(original_max_position)
        self.beta_fast, self.beta_slow = float(beta_fast), float(beta_slow)

    def inv_freq(self, D: int) -> np.ndarray:
        out = np.empty(D // 2, np.float64)
        _load().oracle_rope_inv_freq(self.theta, D, SCALINGS[self.scaling], self.factor,
                                     self.original_max_position, self.beta_fast, self.beta_slow,
                                     _p(out))
        return out

    def logit_mult(self) -> float:
        return float(_load().oracle_rope_logit_mult(SCALINGS[self.scaling], self.factor))

    def pair_code(self) -> int:
        return PAIRINGS[self.pairing]


def rope_ex(x, pos: float, rope: Rope) -> np.ndarray:
    x = _c(x, np.float64)
    D = x.shape[-1]
    f = rope.inv_freq(D)
    out = np.empty_like(x)
    _load().oracle_rope_ex(_p(x), float(pos), _p(f), rope.pair_code(), D, _p(out))
    return out


def qk_transform_ex(x_bits, pos, w, rope: Rope, eps: float) -> np.ndarray:
    x_bits = _c(x_bits, np.uint16)
    N, nh, D = x_bits.shape
    pos = _c(pos, np.int32).reshape(N)
    w = _c(w, np.float32)
    f = rope.inv_freq(D)
    out = np.empty((N, nh, D), np.float64)
    _load().oracle_qk_transform_ex(_p(x_bits), _p(pos), _p(w), _p(f), rope.pair_code(), eps, N, nh, D,
                                   _p(out))
    return out


def prefill_rows_ex(q_bits, k_bits, v_bits, pos, wq, wk, rope: Rope, eps: float, rows) -> np.ndarray:
    q_bits = _c(q_bits, np.uint16)
    k_bits = _c(k_bits, np.uint16)
    v_bits = _c(v_bits, np.uint16)
    B, T, H, D = q_bits.shape
    Hkv = k_bits.shape[2]
    pos = _c(pos, np.int32).reshape(B, T)
    rows = _c(rows, np.int64).reshape(-1, 3)
    assert (rows[:, 0] < B).all() and (rows[:, 1] < H).all() and (rows[:, 2] < T).all()
    f = rope.inv_freq(D)
    out = np.empty((rows.shape[0], D), np.float64)
    _load().oracle_prefill_rows_ex(_p(q_bits), _p(k_bits), _p(v_bits), _p(pos), _p(_c(wq, np.float32)),
                                   _p(_c(wk, np.float32)), _p(f), rope.pair_code(), rope.logit_mult(), eps,
                                   B, T, H, Hkv, D, rows.shape[0], _p(rows), _p(out))
    return out


def decode_ex(q_bits, k_cache_bits, v_cache_bits, offsets, seqlens, qpos, wq, rope: Rope,
              eps: float) -> np.ndarray:
    q_bits = _c(q_bits, np.uint16)
    k_cache_bits = _c(k_cache_bits, np.uint16)
    v_cache_bits = _c(v_cache_bits, np.uint16)
    B, H, D = q_bits.shape
    Hkv = k_cache_bits.shape[1]
    seqlens = _c(seqlens, np.int32)
    assert (seqlens >= 1).all()
    qpos_a = None if qpos is None else _c(qpos, np.int32)
    f = rope.inv_freq(D)
    out = np.empty((B, H, D), np.float64)
    _load().oracle_decode_ex(_p(q_bits), _p(k_cache_bits), _p(v_cache_bits), _p(_c(offsets, np.int64)),
                             _p(seqlens), _p(qpos_a), _p(_c(wq, np.float32)), _p(f), rope.pair_code(),
                             rope.logit_mult(), eps, B, H, Hkv, D, _p(out))
    return out


def decode_append_ex(q_bits, k_new_bits, v_new_bits, k_cache_bits, v_cache_bits, offsets, seqlens,
                     qpos, wq, wk, rope: Rope, eps: float):
    q_bits = _c(q_bits, np.uint16)
    k_new_bits = _c(k_new_bits, np.uint16)
    v_new_bits = _c(v_new_bits, np.uint16)
    B, H, D = q_bits.shape
    Hkv = k_new_bits.shape[1]
    seqlens = _c(seqlens, np.int32)
    assert (seqlens >= 0).all()
    qpos_a = None if qpos is None else _c(qpos, np.int32)
    f = rope.inv_freq(D)
    out = np.empty((B, H, D), np.float64)
    khat = np.empty((B, Hkv, D), np.float64)
    _load().oracle_decode_append_ex(_p(q_bits), _p(k_new_bits), _p(v_new_bits), _p(_c(k_cache_bits, np.uint16)),
                                    _p(_c(v_cache_bits, np.uint16)), _p(_c(offsets, np.int64)), _p(seqlens),
                                    _p(qpos_a), _p(_c(wq, np.float32)), _p(_c(wk, np.float32)), _p(f),
                                    rope.pair_code(), rope.logit_mult(), eps, B, H, Hkv, D, _p(out), _p(khat))
    return out, khat


# ---- paged KV cache: the same attention on rows gathered through a page table --------
def _gather_pages(pages_bits, table, page_size, nrows):
    """Rows 0..nrows-1 of one sequence from [num_pages, page_size, Hkv, D] pages."""
    idx = np.arange(nrows)
    return pages_bits[table[idx // page_size], idx % page_size]


def decode_paged_ex(q_bits, k_pages_bits, v_pages_bits, page_table, page_size, seqlens, qpos, wq,
                    rope: Rope, eps: float) -> np.ndarray:
    """Decode on a paged cache: row r of sequence b is row r % page_size of page
    page_table[b, r // page_size]; the attention is decode_ex on the gathered rows."""
    k_pages_bits = _c(k_pages_bits, np.uint16)
    v_pages_bits = _c(v_pages_bits, np.uint16)
    table = np.asarray(page_table)
    sl = np.asarray(seqlens, np.int64)
    kc = np.concatenate([_gather_pages(k_pages_bits, table[b], page_size, sl[b]) for b in range(len(sl))])
    vc = np.concatenate([_gather_pages(v_pages_bits, table[b], page_size, sl[b]) for b in range(len(sl))])
    offsets = np.concatenate([[0], np.cumsum(sl)]).astype(np.int64)
    return decode_ex(q_bits, kc, vc, offsets, sl.astype(np.int32), qpos, wq, rope, eps)


def decode_append_paged_ex(q_bits, k_new_bits, v_new_bits, k_pages_bits, v_pages_bits, page_table, page_size,
                           seqlens, qpos, wq, wk, rope: Rope, eps: float):
    """decode_append_ex on a paged cache (the cached rows gathered through the table)."""
    k_pages_bits = _c(k_pages_bits, np.uint16)
    v_pages_bits = _c(v_pages_bits, np.uint16)
    table = np.asarray(page_table)
    sl = np.asarray(seqlens, np.int64)
    Hkv, D = k_pages_bits.shape[2], k_pages_bits.shape[3]
    ks, vs = [], []
    for b in range(len(sl)):   # the cached rows, then one free row for the appended token
        ks += [_gather_pages(k_pages_bits, table[b], page_size, sl[b]), np.zeros((1, Hkv, D), np.uint16)]
        vs += [_gather_pages(v_pages_bits, table[b], page_size, sl[b]), np.zeros((1, Hkv, D), np.uint16)]
    offsets = np.concatenate([[0], np.cumsum(sl + 1)]).astype(np.int64)
    return decode_append_ex(q_bits, k_new_bits, v_new_bits, np.concatenate(ks), np.concatenate(vs), offsets,
                            sl.astype(np.int32), qpos, wq, wk, rope, eps)


def prefill_chunk_ex(q_bits, k_bits, v_bits, k_cache_bits, v_cache_bits, offsets, prefix_len, pos, wq, wk,
                     rope: Rope, eps: float):
    """Chunked prefill against a cache prefix: q [B,C,H,D], k/v [B,C,Hkv,D] raw bf16 bits of
    the chunk at positions pos [B,C]; the cache [rows,Hkv,D] holds prefix_len[b] rows of
    sequence b from offsets[b] on (k-hat, v).  Returns (out [B,C,H,D], chunk k-hat
    [B,C,Hkv,D]), both fp64."""
    q_bits = _c(q_bits, np.uint16)
    k_bits = _c(k_bits, np.uint16)
    v_bits = _c(v_bits, np.uint16)
    B, C, H, D = q_bits.shape
    Hkv = k_bits.shape[2]
    assert k_bits.shape == (B, C, Hkv, D) and v_bits.shape == k_bits.shape
    pl = _c(prefix_len, np.int32)
    assert (pl >= 0).all()
    f = rope.inv_freq(D)
    out = np.empty((B, C, H, D), np.float64)
    khat = np.empty((B, C, Hkv, D), np.float64)
    _load().oracle_prefill_chunk_ex(_p(q_bits), _p(k_bits), _p(v_bits), _p(_c(k_cache_bits, np.uint16)),
                                    _p(_c(v_cache_bits, np.uint16)), _p(_c(offsets, np.int64)), _p(pl),
                                    _p(_c(pos, np.int32).reshape(B, C)), _p(_c(wq, np.float32)),
                                    _p(_c(wk, np.float32)), _p(f), rope.pair_code(), rope.logit_mult(), eps, B, C,
                                    H, Hkv, D, _p(out), _p(khat))
    return out, khat


def prefill_chunk_rows_ex(q_bits, k_bits, v_bits, k_cache_bits, v_cache_bits, offsets, prefix_len, pos, wq, wk,
                          rope: Rope, eps: float, rows) -> np.ndarray:
    """The rows (b, hq, i) of prefill_chunk_ex listed in rows [n, 3] (chunk row i of query
    head hq of sequence b), for launches too large to compute whole.  Returns (out [n, D],
    chunk k-hat [B,C,Hkv,D]), both fp64."""
    q_bits = _c(q_bits, np.uint16)
    k_bits = _c(k_bits, np.uint16)
    v_bits = _c(v_bits, np.uint16)
    B, C, H, D = q_bits.shape
    Hkv = k_bits.shape[2]
    assert k_bits.shape == (B, C, Hkv, D) and v_bits.shape == k_bits.shape
    pl = _c(prefix_len, np.int32)
    assert (pl >= 0).all()
    rows = _c(rows, np.int64).reshape(-1, 3)
    assert (rows[:, 0] < B).all() and (rows[:, 1] < H).all() and (rows[:, 2] < C).all() and (rows >= 0).all()
    f = rope.inv_freq(D)
    out = np.empty((rows.shape[0], D), np.float64)
    khat = np.empty((B, C, Hkv, D), np.float64)
    _load().oracle_prefill_chunk_rows_ex(_p(q_bits), _p(k_bits), _p(v_bits), _p(_c(k_cache_bits, np.uint16)),
                                         _p(_c(v_cache_bits, np.uint16)), _p(_c(offsets, np.int64)), _p(pl),
                                         _p(_c(pos, np.int32).reshape(B, C)), _p(_c(wq, np.float32)),
                                         _p(_c(wk, np.float32)), _p(f), rope.pair_code(), rope.logit_mult(), eps, B,
                                         C, H, Hkv, D, rows.shape[0], _p(rows), _p(out), _p(khat))
    return out, khat


def prefill_chunk_paged_ex(q_bits, k_bits, v_bits, k_pages_bits, v_pages_bits, page_table, page_size, prefix_len,
                           pos, wq, wk, rope: Rope, eps: float):
    """Chunked prefill against a paged cache prefix: cached row r of sequence b is row
    r % page_size of page page_table[b, r // page_size]; the attention is prefill_chunk_ex
    on the gathered prefix rows.  Returns (out [B,C,H,D], chunk k-hat [B,C,Hkv,D]), fp64."""
    k_pages_bits = _c(k_pages_bits, np.uint16)
    v_pages_bits = _c(v_pages_bits, np.uint16)
    table = np.asarray(page_table)
    pl = np.asarray(prefix_len, np.int64)
    Hkv, D = k_pages_bits.shape[2], k_pages_bits.shape[3]
    none = np.zeros((0, Hkv, D), np.uint16)
    kc = np.concatenate([none] + [_gather_pages(k_pages_bits, table[b], page_size, pl[b]) for b in range(len(pl))])
    vc = np.concatenate([none] + [_gather_pages(v_pages_bits, table[b], page_size, pl[b]) for b in range(len(pl))])
    offsets = np.concatenate([[0], np.cumsum(pl)]).astype(np.int64)
    return prefill_chunk_ex(q_bits, k_bits, v_bits, kc, vc, offsets, pl.astype(np.int32), pos, wq, wk, rope, eps)


def prefill_varlen_ex(q_bits, k_bits, v_bits, cu_seqlens, pos, wq, wk, rope: Rope, eps: float) -> np.ndarray:
    """Packed variable-length prefill: q [N,H,D], k/v [N,Hkv,D] bf16 bits, sequence b on
    tokens cu_seqlens[b] .. cu_seqlens[b+1]-1, positions pos [N]; causal within each
    sequence.  Returns out [N,H,D] fp64."""
    q_bits = _c(q_bits, np.uint16)
    k_bits = _c(k_bits, np.uint16)
    v_bits = _c(v_bits, np.uint16)
    N, H, D = q_bits.shape
    Hkv = k_bits.shape[1]
    cu = _c(cu_seqlens, np.int64)
    B = cu.shape[0] - 1
    assert cu[0] == 0 and cu[-1] == N and (np.diff(cu) >= 0).all()
    f = rope.inv_freq(D)
    out = np.empty((N, H, D), np.float64)
    _load().oracle_prefill_varlen_ex(_p(q_bits), _p(k_bits), _p(v_bits), _p(cu), _p(_c(pos, np.int32).reshape(N)),
                                     _p(_c(wq, np.float32)), _p(_c(wk, np.float32)), _p(f), rope.pair_code(),
                                     rope.logit_mult(), eps, B, H, Hkv, D, _p(out))
    return out


def linear(x_bits, w_bits) -> np.ndarray:
    """Projection without bias: y = x W^T over the last axis of x (nn.Linear; the pages
    give Qwen3's projections no bias).  x [..., K] and w [N, K] bf16 bits -> y [..., N]
    fp64."""
    x_bits = _c(x_bits, np.uint16)
    w_bits = _c(w_bits, np.uint16)
    K = x_bits.shape[-1]
    N = w_bits.shape[0]
    assert w_bits.shape == (N, K)
    M = x_bits.size // K if K else 0
    y = np.empty(x_bits.shape[:-1] + (N,), np.float64)
    _load().oracle_linear(_p(x_bits), _p(w_bits), M, N, K, _p(y))
    return y


def qkv_proj(x_bits, w_qkv_bits, H: int, Hkv: int, D: int):
    """Fused QKV projection, then the split and the per-head view of the "Qwen3"
    walkthrough's forward steps 1-3: qkv = x W_qkv^T with W_qkv = [W_q; W_k; W_v]
    ((H + 2 Hkv) D rows), split into H D, Hkv D, Hkv D columns and viewed as
    q [N, H, D], k [N, Hkv, D], v [N, Hkv, D] (fp64)."""
    y = linear(x_bits, w_qkv_bits)
    N = y.size // ((H + 2 * Hkv) * D)
    y = y.reshape(N, H + 2 * Hkv, D)
    return y[:, :H], y[:, H:H + Hkv], y[:, H + Hkv:]


def o_proj(o_bits, w_o_bits) -> np.ndarray:
    """Output projection of the "Qwen3" walkthrough's forward step 7: the heads of the
    attention output o [N, H, D] (bf16 bits) flattened to [N, H D], times W_o^T
    (W_o [hidden, H D]) -> [N, hidden] fp64."""
    o_bits = _c(o_bits, np.uint16)
    N = o_bits.shape[0]
    return linear(o_bits.reshape(N, -1), w_o_bits)


def round_bf16_bits(a) -> np.ndarray:
    """fp64 values rounded to the nearest bfloat16 (ties to even), returned as bf16 bit
    patterns: the dtype boundary where a bf16 model stores a tensor.  Written from the
    format (8 significant bits, 8 exponent bits) for finite normal-range values."""
    a = np.asarray(a, np.float64)
    m, e = np.frexp(a)                     # a = m 2^e, 0.5 <= |m| < 1
    r = np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)   # 8 significant bits, ties to even
    return (r.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)


def attn_block_prefill(x_bits, w_qkv_bits, w_o_bits, pos, wq, wk, rope: Rope, eps: float, H: int, Hkv: int,
                       D: int, rows=None) -> np.ndarray:
    """The attention sub-block of a prefill in the order of the "Qwen3" walkthrough's
    forward steps: qkv projection (steps 1-3), q/k RMSNorm (4), RoPE (5), causal GQA
    attention (6), output projection over the concatenated heads (7).  x [B, T, hidden]
    bf16 bits; q, k, v and the attention output are stored as bf16 between the steps
    (the tensors' dtype in a bf16 model), every step computed in fp64.  Returns y
    [B, T, hidden] fp64, or, with rows (an array of (b, t)), only those rows (the
    attention rows of every head of those tokens are evaluated one by one)."""
    x_bits = _c(x_bits, np.uint16)
    B, T, hidden = x_bits.shape
    q, k, v = qkv_proj(x_bits.reshape(B * T, hidden), w_qkv_bits, H, Hkv, D)
    qb = round_bf16_bits(q).reshape(B, T, H, D)
    kb = round_bf16_bits(k).reshape(B, T, Hkv, D)
    vb = round_bf16_bits(v).reshape(B, T, Hkv, D)
    if rows is None:
        rs = np.array([(b, h, t) for b in range(B) for t in range(T) for h in range(H)], np.int64)
    else:
        rs = np.array([(b, h, t) for b, t in rows for h in range(H)], np.int64)
    o = prefill_rows_ex(qb, kb, vb, pos, wq, wk, rope, eps, rs)
    ob = round_bf16_bits(o).reshape(-1, H, D)
    y = o_proj(ob, w_o_bits)
    return y.reshape(B, T, hidden) if rows is None else y
