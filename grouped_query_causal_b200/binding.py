"""Python binding of ``libgqa_attn.so`` (the C ABI in ``include/gqa_attn.h``).

Argument marshalling only: torch tensors supply device memory and the current
CUDA stream; every step of the computation runs in the library's kernels.  There
is no fallback: if the library is missing or a call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgqa_attn.so")

GQA_OK = 0
STATUS_NAMES = {
    0: "GQA_OK", -1: "GQA_ERR_INVALID_ARG", -2: "GQA_ERR_UNSUPPORTED", -3: "GQA_ERR_WORKSPACE",
    -4: "GQA_ERR_CUDA", -5: "GQA_ERR_DEVICE_TIMEOUT", -6: "GQA_ERR_DEVICE_INPUT",
}
# Every symbol the header declares.
EXPORTS = ("gqa_status_string", "gqa_attn_prefill_workspace_size", "gqa_attn_prefill",
           "gqa_attn_k_norm_rope", "gqa_attn_prefill_khat", "gqa_attn_decode_workspace_size",
           "gqa_attn_decode", "gqa_attn_decode_append", "gqa_attn_decode_noalloc",
           "gqa_attn_device_status", "gqa_attn_prefill_ex", "gqa_attn_k_norm_rope_ex",
           "gqa_attn_prefill_khat_ex", "gqa_attn_decode_ex", "gqa_attn_decode_append_ex",
           "gqa_attn_decode_paged", "gqa_attn_decode_append_paged", "gqa_attn_prefill_varlen_workspace_size",
           "gqa_attn_prefill_varlen", "gqa_attn_prefill_chunk_workspace_size", "gqa_attn_prefill_chunk",
           "gqa_attn_prefill_chunk_paged_workspace_size", "gqa_attn_prefill_chunk_paged",
           "gqa_linear", "gqa_attn_block_prefill_workspace_size", "gqa_attn_block_prefill",
           "gqa_attn_test_stall")


def _header_scratch_bytes() -> int:
    """GQA_NOALLOC_SCRATCH_BYTES as include/gqa_attn.h defines it (the library is compiled
    from the same header), so the two cannot drift apart."""
    import re
    path = os.path.join(os.path.dirname(_PKG), "include", "gqa_attn.h")
    with open(path, encoding="utf-8") as f:
        m = re.search(r"#define\s+GQA_NOALLOC_SCRATCH_BYTES\s+\((\d+)u\s*<<\s*(\d+)\)", f.read())
    if m is None:
        raise RuntimeError(f"GQA_NOALLOC_SCRATCH_BYTES not found in {path}")
    return int(m.group(1)) << int(m.group(2))


# Size of the library's built-in scratch used by gqa_attn_decode_noalloc.
NOALLOC_SCRATCH_BYTES = _header_scratch_bytes()


class RopeConfig(ctypes.Structure):
    """gqa_rope_config: a RoPE variant (pairing "adjacent"/"half"; scaling "none",
    "linear", "ntk" or "yarn" with factor s; YaRN's training length and ramp bounds)."""
    _fields_ = [("theta", ctypes.c_double), ("pairing", ctypes.c_int), ("scaling", ctypes.c_int),
                ("factor", ctypes.c_double), ("original_max_position", ctypes.c_int),
                ("beta_fast", ctypes.c_double), ("beta_slow", ctypes.c_double)]

    PAIRINGS = {"adjacent": 0, "half": 1}
    SCALINGS = {"none": 0, "linear": 1, "ntk": 2, "yarn": 3}

    @classmethod
    def make(cls, theta: float = 1.0e6, pairing: str = "adjacent", scaling: str = "none",
             factor: float = 1.0, original_max_position: int = 4096, beta_fast: float = 32.0,
             beta_slow: float = 1.0) -> "RopeConfig":
        return cls(float(theta), cls.PAIRINGS[pairing], cls.SCALINGS[scaling], float(factor),
                   int(original_max_position), float(beta_fast), float(beta_slow))


def _rope_call(lib, name: str, rope: Optional["RopeConfig"], theta: float):
    """The entry point to call and the argument that goes where theta sits: the plain
    symbol with theta, or its _ex form with a pointer to the RoPE configuration."""
    if rope is None:
        return getattr(lib, name), float(theta)
    return getattr(lib, name + "_ex"), ctypes.byref(rope)


class GqaError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)}")
        self.status = status


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the library and declare its C signatures (raises if it is missing)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with `python -m grouped_query_causal_b200.build`")
    lib = ctypes.CDLL(path)
    P, I, F, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.gqa_status_string.argtypes = [I]
    lib.gqa_status_string.restype = ctypes.c_char_p
    lib.gqa_attn_prefill_workspace_size.argtypes = [I, I, I, I, I]
    lib.gqa_attn_prefill_workspace_size.restype = Z
    lib.gqa_attn_prefill.argtypes = [P, P, P, P, P, P, F, F, P, I, I, I, I, I, P, Z, P]
    lib.gqa_attn_prefill.restype = I
    lib.gqa_attn_k_norm_rope.argtypes = [P, P, P, F, F, P, P, ctypes.c_int64, I, I, P]
    lib.gqa_attn_k_norm_rope.restype = I
    lib.gqa_attn_prefill_khat.argtypes = [P, P, P, P, P, P, F, F, P, I, I, I, I, I, P]
    lib.gqa_attn_prefill_khat.restype = I
    lib.gqa_attn_decode_workspace_size.argtypes = [I, I, I, I, I]
    lib.gqa_attn_decode_workspace_size.restype = Z
    lib.gqa_attn_decode.argtypes = [P, P, P, P, P, P, P, F, F, P, I, I, I, I, I, P, Z, P]
    lib.gqa_attn_decode.restype = I
    lib.gqa_attn_decode_append.argtypes = [P, P, P, P, P, P, P, P, P, P, F, F, P, I, I, I, I, I, P, Z, P]
    lib.gqa_attn_decode_append.restype = I
    lib.gqa_attn_decode_noalloc.argtypes = [P, P, P, P, P, P, P, F, F, P, I, I, I, I, I, P]
    lib.gqa_attn_decode_noalloc.restype = I
    lib.gqa_attn_device_status.argtypes = [P]
    lib.gqa_attn_device_status.restype = I
    R = ctypes.POINTER(RopeConfig)
    lib.gqa_attn_prefill_ex.argtypes = [P, P, P, P, P, P, R, F, P, I, I, I, I, I, P, Z, P]
    lib.gqa_attn_k_norm_rope_ex.argtypes = [P, P, P, R, F, P, P, ctypes.c_int64, I, I, P]
    lib.gqa_attn_prefill_khat_ex.argtypes = [P, P, P, P, P, P, R, F, P, I, I, I, I, I, P]
    lib.gqa_attn_decode_ex.argtypes = [P, P, P, P, P, P, P, R, F, P, I, I, I, I, I, P, Z, P]
    lib.gqa_attn_decode_append_ex.argtypes = [P, P, P, P, P, P, P, P, P, P, R, F, P, I, I, I, I, I, P, Z, P]
    lib.gqa_attn_decode_paged.argtypes = [P, P, P, P, I, I, I, P, P, P, R, F, P, I, I, I, I, I, P, Z, P]
    lib.gqa_attn_decode_append_paged.argtypes = [P, P, P, P, P, P, I, I, I, P, P, P, P, R, F, P, I, I, I, I, I, P, Z,
                                                 P]
    L = ctypes.c_int64
    lib.gqa_attn_prefill_varlen_workspace_size.argtypes = [L, I, I]
    lib.gqa_attn_prefill_varlen_workspace_size.restype = Z
    lib.gqa_attn_prefill_varlen.argtypes = [P, P, P, P, P, P, P, R, F, P, I, L, I, I, I, I, P, Z, P]
    lib.gqa_attn_prefill_chunk_workspace_size.argtypes = [L, I]
    lib.gqa_attn_prefill_chunk_workspace_size.restype = Z
    lib.gqa_attn_prefill_chunk.argtypes = [P, P, P, P, P, P, P, P, P, L, P, P, R, F, P, I, L, I, I, I, I, P, Z, P]
    lib.gqa_attn_prefill_chunk_paged_workspace_size.argtypes = [L, I]
    lib.gqa_attn_prefill_chunk_paged_workspace_size.restype = Z
    lib.gqa_attn_prefill_chunk_paged.argtypes = [P, P, P, P, P, P, P, P, I, I, I, P, P, P, R, F, P, I, L, I, I, I, I, P,
                                                 Z, P]
    lib.gqa_attn_test_stall.argtypes = [I]
    lib.gqa_attn_test_stall.restype = None
    lib.gqa_linear.argtypes = [P, P, P, I, L, I, I, P]
    lib.gqa_linear.restype = I
    lib.gqa_attn_block_prefill_workspace_size.argtypes = [I, I, I, I, I, I]
    lib.gqa_attn_block_prefill_workspace_size.restype = Z
    lib.gqa_attn_block_prefill.argtypes = [P, P, P, P, P, P, R, F, P, I, I, I, I, I, I, P, Z, P]
    lib.gqa_attn_block_prefill.restype = I
    for n in ("gqa_attn_prefill_ex", "gqa_attn_k_norm_rope_ex", "gqa_attn_prefill_khat_ex", "gqa_attn_decode_ex",
              "gqa_attn_decode_append_ex", "gqa_attn_decode_paged", "gqa_attn_decode_append_paged",
              "gqa_attn_prefill_varlen", "gqa_attn_prefill_chunk"):
        getattr(lib, n).restype = I
    _lib = lib
    return lib


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream_handle(stream: Optional[torch.cuda.Stream]) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _check(t: torch.Tensor, name: str, dtype: torch.dtype, dim: int):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.dim() != dim:
        raise ValueError(f"{name} must have {dim} dims, got {tuple(t.shape)}")


def _raise(status: int, what: str):
    if status != GQA_OK:
        raise GqaError(status, what)


def rope_table_numel(n_tokens: int, D: int = 128) -> int:
    """fp32 elements of the RoPE cos/sin table for n_tokens (GQA_ROPE_TABLE_BYTES / 4)."""
    return (n_tokens + 127) // 128 * 128 * D


def rope_table_entry(table: torch.Tensor, n: int, pair: int):
    """(cos, sin) of RoPE pair `pair` of flattened token n in a table k_norm_rope wrote."""
    i2, k = divmod(pair, 2)
    base = (((n >> 7) * 32 + i2) * 128 + (n & 127)) * 4 + 2 * k
    return float(table[base]), float(table[base + 1])


def prefill_workspace_size(B: int, T: int, H: int, Hkv: int, D: int = 128) -> int:
    return int(load().gqa_attn_prefill_workspace_size(B, T, H, Hkv, D))


def decode_workspace_size(B: int, H: int, Hkv: int, max_len: int, D: int = 128) -> int:
    return int(load().gqa_attn_decode_workspace_size(B, H, Hkv, D, max_len))


def prefill(q, k, v, pos, qnorm_w, knorm_w, theta: float = 1.0e6, eps: float = 1e-6,
            out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
            stream: Optional[torch.cuda.Stream] = None, rope: Optional[RopeConfig] = None) -> torch.Tensor:
    """Causal GQA prefill with fused q/k RMSNorm + RoPE.  q [B,T,H,D] bf16, k/v
    [B,T,Hkv,D] bf16, pos [B,T] int32, norm weights [D] fp32 -> out [B,T,H,D] fp32.
    rope (a RopeConfig) selects a RoPE variant in place of theta."""
    lib = load()
    _check(q, "q", torch.bfloat16, 4)
    _check(k, "k", torch.bfloat16, 4)
    _check(v, "v", torch.bfloat16, 4)
    _check(pos, "pos", torch.int32, 2)
    _check(qnorm_w, "qnorm_w", torch.float32, 1)
    _check(knorm_w, "knorm_w", torch.float32, 1)
    B, T, H, D = q.shape
    Hkv = k.shape[2]
    if k.shape != (B, T, Hkv, D) or v.shape != k.shape or pos.shape != (B, T):
        raise ValueError("shape mismatch between q, k, v, pos")
    if qnorm_w.shape != (D,) or knorm_w.shape != (D,):
        raise ValueError("norm weights must be [D]")
    if out is None:
        out = torch.empty((B, T, H, D), dtype=torch.float32, device=q.device)
    _check(out, "out", torch.float32, 4)
    need = int(lib.gqa_attn_prefill_workspace_size(B, T, H, Hkv, D))
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    fn, th = _rope_call(lib, "gqa_attn_prefill", rope, theta)
    st = fn(_ptr(q), _ptr(k), _ptr(v), _ptr(pos), _ptr(qnorm_w), _ptr(knorm_w), th, float(eps), _ptr(out), B, T,
            H, Hkv, D, _ptr(workspace), workspace.numel() * workspace.element_size(), _stream_handle(stream))
    _raise(st, "gqa_attn_prefill")
    return out


def k_norm_rope(k, pos, knorm_w, theta: float = 1.0e6, eps: float = 1e-6,
                out: Optional[torch.Tensor] = None, rope_cs: Optional[torch.Tensor] = None,
                stream: Optional[torch.cuda.Stream] = None, rope: Optional[RopeConfig] = None) -> torch.Tensor:
    """k-hat = RoPE(RMSNorm(k)) in bf16.  k [..., Hkv, D] bf16 with one position per
    token (pos has the leading shape of k) -> k_hat of k's shape (a decode cache).
    rope_cs (fp32, rope_table_numel(N) elements), when given, receives the tokens' RoPE
    cos/sin (an opaque blocked table) for prefill_khat to reuse."""
    lib = load()
    if k.dtype != torch.bfloat16 or not k.is_cuda or not k.is_contiguous() or k.dim() < 2:
        raise ValueError("k must be a contiguous CUDA bf16 tensor [..., Hkv, D]")
    _check(knorm_w, "knorm_w", torch.float32, 1)
    Hkv, D = k.shape[-2], k.shape[-1]
    N = k.numel() // (Hkv * D) if k.numel() else 0
    if pos.dtype != torch.int32 or not pos.is_cuda or not pos.is_contiguous() or pos.numel() != N:
        raise ValueError("pos must be a contiguous CUDA int32 tensor with one entry per token")
    if rope_cs is not None and (rope_cs.dtype != torch.float32 or not rope_cs.is_cuda or not rope_cs.is_contiguous()
                                or rope_cs.numel() < rope_table_numel(N)):
        raise ValueError("rope_cs must be a contiguous CUDA fp32 tensor of rope_table_numel(N) elements")
    if out is None:
        out = torch.empty_like(k)
    fn, th = _rope_call(lib, "gqa_attn_k_norm_rope", rope, theta)
    st = fn(_ptr(k), _ptr(pos), _ptr(knorm_w), th, float(eps), _ptr(out), _ptr(rope_cs), N, Hkv, D,
            _stream_handle(stream))
    _raise(st, "gqa_attn_k_norm_rope")
    return out


def prefill_khat(q, k_hat, v, pos, qnorm_w, theta: float = 1.0e6, eps: float = 1e-6,
                 out: Optional[torch.Tensor] = None, rope_cs: Optional[torch.Tensor] = None,
                 stream: Optional[torch.cuda.Stream] = None, rope: Optional[RopeConfig] = None) -> torch.Tensor:
    """Attention stage of prefill on already normed + rotated keys (k_hat [B,T,Hkv,D]);
    rope_cs is the cos/sin table k_norm_rope wrote for the same tokens, or None."""
    lib = load()
    _check(q, "q", torch.bfloat16, 4)
    _check(k_hat, "k_hat", torch.bfloat16, 4)
    _check(v, "v", torch.bfloat16, 4)
    _check(pos, "pos", torch.int32, 2)
    _check(qnorm_w, "qnorm_w", torch.float32, 1)
    B, T, H, D = q.shape
    Hkv = k_hat.shape[2]
    if k_hat.shape != (B, T, Hkv, D) or v.shape != k_hat.shape or pos.shape != (B, T):
        raise ValueError("shape mismatch between q, k_hat, v, pos")
    if out is None:
        out = torch.empty((B, T, H, D), dtype=torch.float32, device=q.device)
    _check(out, "out", torch.float32, 4)
    if rope_cs is not None and (rope_cs.dtype != torch.float32 or not rope_cs.is_cuda or not rope_cs.is_contiguous()
                                or rope_cs.numel() < rope_table_numel(B * T)):
        raise ValueError("rope_cs must be a contiguous CUDA fp32 tensor of rope_table_numel(B * T) elements")
    fn, th = _rope_call(lib, "gqa_attn_prefill_khat", rope, theta)
    st = fn(_ptr(q), _ptr(k_hat), _ptr(v), _ptr(pos), _ptr(rope_cs), _ptr(qnorm_w), th, float(eps), _ptr(out), B,
            T, H, Hkv, D, _stream_handle(stream))
    _raise(st, "gqa_attn_prefill_khat")
    return out


def prefill_varlen(q, k, v, pos, cu_seqlens, qnorm_w, knorm_w, max_seqlen: int, eps: float = 1e-6,
                   rope: Optional[RopeConfig] = None, out: Optional[torch.Tensor] = None,
                   workspace: Optional[torch.Tensor] = None,
                   stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Packed variable-length causal prefill.  q [N,H,D], k/v [N,Hkv,D] bf16, pos [N]
    int32, cu_seqlens [B+1] int64 (device) -> out [N,H,D] fp32; each sequence attends
    causally within itself.  rope defaults to the plain RoPE of base 1e6."""
    lib = load()
    _check(q, "q", torch.bfloat16, 3)
    _check(k, "k", torch.bfloat16, 3)
    _check(v, "v", torch.bfloat16, 3)
    _check(pos, "pos", torch.int32, 1)
    _check(cu_seqlens, "cu_seqlens", torch.int64, 1)
    _check(qnorm_w, "qnorm_w", torch.float32, 1)
    _check(knorm_w, "knorm_w", torch.float32, 1)
    N, H, D = q.shape
    Hkv = k.shape[1]
    B = cu_seqlens.numel() - 1
    if k.shape != (N, Hkv, D) or v.shape != k.shape or pos.shape != (N,) or B < 0:
        raise ValueError("shape mismatch between q, k, v, pos, cu_seqlens")
    rope = rope if rope is not None else RopeConfig.make()
    if out is None:
        out = torch.empty((N, H, D), dtype=torch.float32, device=q.device)
    _check(out, "out", torch.float32, 3)
    need = int(lib.gqa_attn_prefill_varlen_workspace_size(N, Hkv, D))
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    st = lib.gqa_attn_prefill_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(pos), _ptr(cu_seqlens), _ptr(qnorm_w),
                                     _ptr(knorm_w), ctypes.byref(rope), float(eps), _ptr(out), B, N, H, Hkv, D,
                                     int(max_seqlen), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                     _stream_handle(stream))
    _raise(st, "gqa_attn_prefill_varlen")
    return out


def prefill_chunk(q, k, v, pos, cu_seqlens, k_cache, v_cache, cache_offsets, prefix_len, qnorm_w, knorm_w,
                  max_chunk_len: int, eps: float = 1e-6, rope: Optional[RopeConfig] = None,
                  out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                  stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Chunked prefill after a cached prefix: the N chunk tokens (q [N,H,D], k/v
    [N,Hkv,D] raw, pos [N], packed per cu_seqlens [B+1]) are appended to the cache
    (k_cache/v_cache [rows,Hkv,D], sequence b at cache_offsets[b] with prefix_len[b] rows
    cached) and attend to it -> out [N,H,D] fp32."""
    lib = load()
    for t, n, dt, d in ((q, "q", torch.bfloat16, 3), (k, "k", torch.bfloat16, 3), (v, "v", torch.bfloat16, 3),
                        (pos, "pos", torch.int32, 1), (cu_seqlens, "cu_seqlens", torch.int64, 1),
                        (k_cache, "k_cache", torch.bfloat16, 3), (v_cache, "v_cache", torch.bfloat16, 3),
                        (cache_offsets, "cache_offsets", torch.int64, 1), (prefix_len, "prefix_len", torch.int32, 1),
                        (qnorm_w, "qnorm_w", torch.float32, 1), (knorm_w, "knorm_w", torch.float32, 1)):
        _check(t, n, dt, d)
    N, H, D = q.shape
    Hkv = k.shape[1]
    B = cu_seqlens.numel() - 1
    if (k.shape != (N, Hkv, D) or v.shape != k.shape or pos.shape != (N,) or k_cache.shape[1:] != (Hkv, D)
            or v_cache.shape != k_cache.shape or cache_offsets.shape != (B + 1,) or prefix_len.shape != (B,)):
        raise ValueError("shape mismatch")
    rope = rope if rope is not None else RopeConfig.make()
    if out is None:
        out = torch.empty((N, H, D), dtype=torch.float32, device=q.device)
    _check(out, "out", torch.float32, 3)
    need = int(lib.gqa_attn_prefill_chunk_workspace_size(N, D))
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    st = lib.gqa_attn_prefill_chunk(_ptr(q), _ptr(k), _ptr(v), _ptr(pos), _ptr(cu_seqlens), _ptr(k_cache),
                                    _ptr(v_cache), _ptr(cache_offsets), _ptr(prefix_len), k_cache.shape[0],
                                    _ptr(qnorm_w), _ptr(knorm_w), ctypes.byref(rope), float(eps), _ptr(out), B, N, H,
                                    Hkv, D, int(max_chunk_len), _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), _stream_handle(stream))
    _raise(st, "gqa_attn_prefill_chunk")
    return out


def prefill_chunk_paged(q, k, v, pos, cu_seqlens, k_pages, v_pages, page_table, prefix_len, qnorm_w, knorm_w,
                        max_chunk_len: int, eps: float = 1e-6, rope: Optional[RopeConfig] = None,
                        out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                        stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Chunked prefill on a paged cache: as prefill_chunk, with the cache in pages
    (k_pages/v_pages [num_pages, page_size, Hkv, D], page_table [B, max_pages] int32)."""
    lib = load()
    for t, n, dt, d in ((q, "q", torch.bfloat16, 3), (k, "k", torch.bfloat16, 3), (v, "v", torch.bfloat16, 3),
                        (pos, "pos", torch.int32, 1), (cu_seqlens, "cu_seqlens", torch.int64, 1),
                        (k_pages, "k_pages", torch.bfloat16, 4), (v_pages, "v_pages", torch.bfloat16, 4),
                        (page_table, "page_table", torch.int32, 2), (prefix_len, "prefix_len", torch.int32, 1),
                        (qnorm_w, "qnorm_w", torch.float32, 1), (knorm_w, "knorm_w", torch.float32, 1)):
        _check(t, n, dt, d)
    N, H, D = q.shape
    Hkv = k.shape[1]
    B = cu_seqlens.numel() - 1
    num_pages, page_size = k_pages.shape[0], k_pages.shape[1]
    if (k.shape != (N, Hkv, D) or v.shape != k.shape or pos.shape != (N,) or k_pages.shape[2:] != (Hkv, D)
            or v_pages.shape != k_pages.shape or page_table.shape[0] != B or prefix_len.shape != (B,)):
        raise ValueError("shape mismatch")
    rope = rope if rope is not None else RopeConfig.make()
    if out is None:
        out = torch.empty((N, H, D), dtype=torch.float32, device=q.device)
    _check(out, "out", torch.float32, 3)
    need = int(lib.gqa_attn_prefill_chunk_paged_workspace_size(N, D))
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    st = lib.gqa_attn_prefill_chunk_paged(_ptr(q), _ptr(k), _ptr(v), _ptr(pos), _ptr(cu_seqlens), _ptr(k_pages),
                                          _ptr(v_pages), _ptr(page_table), num_pages, page_size, page_table.shape[1],
                                          _ptr(prefix_len), _ptr(qnorm_w), _ptr(knorm_w), ctypes.byref(rope),
                                          float(eps), _ptr(out), B, N, H, Hkv, D, int(max_chunk_len), _ptr(workspace),
                                          workspace.numel() * workspace.element_size(), _stream_handle(stream))
    _raise(st, "gqa_attn_prefill_chunk_paged")
    return out


def linear(x, w, out_dtype: torch.dtype = torch.bfloat16, out: Optional[torch.Tensor] = None,
           stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Projection without bias, y = x W^T: x [..., K] bf16, w [N, K] bf16 -> y [..., N]
    in bf16 or fp32 (fp32 accumulation)."""
    lib = load()
    if x.dtype != torch.bfloat16 or not x.is_cuda or not x.is_contiguous() or x.dim() < 1:
        raise ValueError("x must be a contiguous CUDA bf16 tensor [..., K]")
    _check(w, "w", torch.bfloat16, 2)
    N, K = w.shape
    if x.shape[-1] != K:
        raise ValueError("x and w disagree on K")
    M = x.numel() // K if K else 0
    if out_dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("out_dtype must be bf16 or fp32")
    if out is None:
        out = torch.empty(x.shape[:-1] + (N,), dtype=out_dtype, device=x.device)
    if out.dtype != out_dtype or not out.is_contiguous() or out.numel() != M * N:
        raise ValueError("out must be a contiguous tensor of the output shape and dtype")
    st = lib.gqa_linear(_ptr(x), _ptr(w), _ptr(out), 1 if out_dtype == torch.float32 else 0, M, N, K,
                        _stream_handle(stream))
    _raise(st, "gqa_linear")
    return out


def attn_block_prefill(x, w_qkv, w_o, pos, qnorm_w, knorm_w, H: int, Hkv: int, eps: float = 1e-6,
                       rope: Optional[RopeConfig] = None, out: Optional[torch.Tensor] = None,
                       workspace: Optional[torch.Tensor] = None,
                       stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """The attention sub-block for a prefill: x [B,T,hidden] bf16, w_qkv [(H+2Hkv)D,
    hidden], w_o [hidden, H D] bf16, pos [B,T] -> y [B,T,hidden] fp32 (qkv projection,
    q/k norm, RoPE, causal GQA attention, output projection)."""
    lib = load()
    _check(x, "x", torch.bfloat16, 3)
    _check(w_qkv, "w_qkv", torch.bfloat16, 2)
    _check(w_o, "w_o", torch.bfloat16, 2)
    _check(pos, "pos", torch.int32, 2)
    _check(qnorm_w, "qnorm_w", torch.float32, 1)
    _check(knorm_w, "knorm_w", torch.float32, 1)
    B, T, hidden = x.shape
    D = qnorm_w.shape[0]
    if w_qkv.shape != ((H + 2 * Hkv) * D, hidden) or w_o.shape != (hidden, H * D) or pos.shape != (B, T):
        raise ValueError("shape mismatch between x, w_qkv, w_o, pos")
    rope = rope if rope is not None else RopeConfig.make()
    if out is None:
        out = torch.empty((B, T, hidden), dtype=torch.float32, device=x.device)
    _check(out, "out", torch.float32, 3)
    need = int(lib.gqa_attn_block_prefill_workspace_size(B, T, hidden, H, Hkv, D))
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=x.device)
    st = lib.gqa_attn_block_prefill(_ptr(x), _ptr(w_qkv), _ptr(w_o), _ptr(pos), _ptr(qnorm_w), _ptr(knorm_w),
                                    ctypes.byref(rope), float(eps), _ptr(out), B, T, hidden, H, Hkv, D,
                                    _ptr(workspace), workspace.numel() * workspace.element_size(),
                                    _stream_handle(stream))
    _raise(st, "gqa_attn_block_prefill")
    return out


def decode(q, k_cache, v_cache, cache_offsets, seqlens, qnorm_w, max_len: int,
           q_pos: Optional[torch.Tensor] = None, theta: float = 1.0e6, eps: float = 1e-6,
           out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
           stream: Optional[torch.cuda.Stream] = None, rope: Optional[RopeConfig] = None) -> torch.Tensor:
    """Split-KV decode.  q [B,H,D] bf16 (raw), caches [rows,Hkv,D] bf16 (normed/rotated
    K, raw V), cache_offsets [B+1] int64, seqlens [B] int32, q_pos [B] int32 or None
    (then the query sits at position seqlens[b]) -> out [B,H,D] fp32."""
    lib = load()
    _check(q, "q", torch.bfloat16, 3)
    _check(k_cache, "k_cache", torch.bfloat16, 3)
    _check(v_cache, "v_cache", torch.bfloat16, 3)
    _check(cache_offsets, "cache_offsets", torch.int64, 1)
    _check(seqlens, "seqlens", torch.int32, 1)
    _check(qnorm_w, "qnorm_w", torch.float32, 1)
    if q_pos is not None:
        _check(q_pos, "q_pos", torch.int32, 1)
    B, H, D = q.shape
    Hkv = k_cache.shape[1]
    if k_cache.shape[2] != D or v_cache.shape != k_cache.shape:
        raise ValueError("cache shape mismatch")
    if cache_offsets.shape != (B + 1,) or seqlens.shape != (B,):
        raise ValueError("cache_offsets must be [B+1] and seqlens [B]")
    if out is None:
        out = torch.empty((B, H, D), dtype=torch.float32, device=q.device)
    _check(out, "out", torch.float32, 3)
    need = int(lib.gqa_attn_decode_workspace_size(B, H, Hkv, D, int(max_len)))
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    fn, th = _rope_call(lib, "gqa_attn_decode", rope, theta)
    st = fn(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(cache_offsets), _ptr(seqlens), _ptr(q_pos), _ptr(qnorm_w),
            th, float(eps), _ptr(out), B, H, Hkv, D, int(max_len), _ptr(workspace),
            workspace.numel() * workspace.element_size(), _stream_handle(stream))
    _raise(st, "gqa_attn_decode")
    return out


def decode_append(q, k_new, v_new, k_cache, v_cache, cache_offsets, seqlens, qnorm_w, knorm_w,
                  max_len: int, q_pos: Optional[torch.Tensor] = None, theta: float = 1.0e6,
                  eps: float = 1e-6, out: Optional[torch.Tensor] = None,
                  workspace: Optional[torch.Tensor] = None,
                  stream: Optional[torch.cuda.Stream] = None, rope: Optional[RopeConfig] = None) -> torch.Tensor:
    """Decode step that appends the new token first: k-hat of k_new [B,Hkv,D] (normed
    with knorm_w, rotated at q_pos or seqlens[b]) and v_new [B,Hkv,D] go to row seqlens[b]
    of each sequence in k_cache / v_cache (written in place), then q [B,H,D] attends to
    rows 0..seqlens[b].  max_len bounds seqlens[b] + 1.  seqlens is not advanced."""
    lib = load()
    _check(q, "q", torch.bfloat16, 3)
    _check(k_new, "k_new", torch.bfloat16, 3)
    _check(v_new, "v_new", torch.bfloat16, 3)
    _check(k_cache, "k_cache", torch.bfloat16, 3)
    _check(v_cache, "v_cache", torch.bfloat16, 3)
    _check(cache_offsets, "cache_offsets", torch.int64, 1)
    _check(seqlens, "seqlens", torch.int32, 1)
    _check(qnorm_w, "qnorm_w", torch.float32, 1)
    _check(knorm_w, "knorm_w", torch.float32, 1)
    if q_pos is not None:
        _check(q_pos, "q_pos", torch.int32, 1)
    B, H, D = q.shape
    Hkv = k_cache.shape[1]
    if k_cache.shape[2] != D or v_cache.shape != k_cache.shape:
        raise ValueError("cache shape mismatch")
    if k_new.shape != (B, Hkv, D) or v_new.shape != (B, Hkv, D):
        raise ValueError("k_new and v_new must be [B, Hkv, D]")
    if cache_offsets.shape != (B + 1,) or seqlens.shape != (B,):
        raise ValueError("cache_offsets must be [B+1] and seqlens [B]")
    if out is None:
        out = torch.empty((B, H, D), dtype=torch.float32, device=q.device)
    _check(out, "out", torch.float32, 3)
    need = int(lib.gqa_attn_decode_workspace_size(B, H, Hkv, D, int(max_len)))
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    fn, th = _rope_call(lib, "gqa_attn_decode_append", rope, theta)
    st = fn(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache), _ptr(cache_offsets), _ptr(seqlens),
            _ptr(q_pos), _ptr(qnorm_w), _ptr(knorm_w), th, float(eps), _ptr(out), B, H, Hkv, D, int(max_len),
            _ptr(workspace), workspace.numel() * workspace.element_size(), _stream_handle(stream))
    _raise(st, "gqa_attn_decode_append")
    return out


def _check_pages(k_pages, v_pages, page_table, B):
    _check(k_pages, "k_pages", torch.bfloat16, 4)
    _check(v_pages, "v_pages", torch.bfloat16, 4)
    _check(page_table, "page_table", torch.int32, 2)
    if v_pages.shape != k_pages.shape:
        raise ValueError("k_pages and v_pages must have one shape [num_pages, page_size, Hkv, D]")
    if page_table.shape[0] != B:
        raise ValueError("page_table must be [B, max_pages_per_seq]")
    return k_pages.shape[0], k_pages.shape[1], k_pages.shape[2], page_table.shape[1]


def decode_paged(q, k_pages, v_pages, page_table, seqlens, qnorm_w, max_len: int,
                 q_pos: Optional[torch.Tensor] = None, rope: Optional[RopeConfig] = None, eps: float = 1e-6,
                 out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                 stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Decode on a paged cache: k_pages / v_pages [num_pages, page_size, Hkv, D] bf16,
    page_table [B, max_pages] int32 (row r of sequence b: row r % page_size of page
    page_table[b, r // page_size]).  rope defaults to the plain RoPE of base 1e6."""
    lib = load()
    _check(q, "q", torch.bfloat16, 3)
    _check(seqlens, "seqlens", torch.int32, 1)
    _check(qnorm_w, "qnorm_w", torch.float32, 1)
    if q_pos is not None:
        _check(q_pos, "q_pos", torch.int32, 1)
    B, H, D = q.shape
    num_pages, page_size, Hkv, _ = _check_pages(k_pages, v_pages, page_table, B)
    rope = rope if rope is not None else RopeConfig.make()
    if out is None:
        out = torch.empty((B, H, D), dtype=torch.float32, device=q.device)
    _check(out, "out", torch.float32, 3)
    need = int(lib.gqa_attn_decode_workspace_size(B, H, Hkv, D, int(max_len)))
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    st = lib.gqa_attn_decode_paged(_ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(page_table), num_pages, page_size,
                                   page_table.shape[1], _ptr(seqlens), _ptr(q_pos), _ptr(qnorm_w), ctypes.byref(rope),
                                   float(eps), _ptr(out), B, H, Hkv, D, int(max_len), _ptr(workspace),
                                   workspace.numel() * workspace.element_size(), _stream_handle(stream))
    _raise(st, "gqa_attn_decode_paged")
    return out


def decode_append_paged(q, k_new, v_new, k_pages, v_pages, page_table, seqlens, qnorm_w, knorm_w,
                        max_len: int, q_pos: Optional[torch.Tensor] = None, rope: Optional[RopeConfig] = None,
                        eps: float = 1e-6, out: Optional[torch.Tensor] = None,
                        workspace: Optional[torch.Tensor] = None,
                        stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """decode_append on a paged cache: the new token's k-hat and v go to row seqlens[b]
    (in its page), then the query attends to rows 0..seqlens[b]."""
    lib = load()
    _check(q, "q", torch.bfloat16, 3)
    _check(k_new, "k_new", torch.bfloat16, 3)
    _check(v_new, "v_new", torch.bfloat16, 3)
    _check(seqlens, "seqlens", torch.int32, 1)
    _check(qnorm_w, "qnorm_w", torch.float32, 1)
    _check(knorm_w, "knorm_w", torch.float32, 1)
    if q_pos is not None:
        _check(q_pos, "q_pos", torch.int32, 1)
    B, H, D = q.shape
    num_pages, page_size, Hkv, _ = _check_pages(k_pages, v_pages, page_table, B)
    if k_new.shape != (B, Hkv, D) or v_new.shape != (B, Hkv, D):
        raise ValueError("k_new and v_new must be [B, Hkv, D]")
    rope = rope if rope is not None else RopeConfig.make()
    if out is None:
        out = torch.empty((B, H, D), dtype=torch.float32, device=q.device)
    _check(out, "out", torch.float32, 3)
    need = int(lib.gqa_attn_decode_workspace_size(B, H, Hkv, D, int(max_len)))
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    st = lib.gqa_attn_decode_append_paged(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_pages), _ptr(v_pages),
                                          _ptr(page_table), num_pages, page_size, page_table.shape[1], _ptr(seqlens),
                                          _ptr(q_pos), _ptr(qnorm_w), _ptr(knorm_w), ctypes.byref(rope), float(eps),
                                          _ptr(out), B, H, Hkv, D, int(max_len), _ptr(workspace),
                                          workspace.numel() * workspace.element_size(), _stream_handle(stream))
    _raise(st, "gqa_attn_decode_append_paged")
    return out


def decode_noalloc(q, k_cache, v_cache, cache_offsets, seqlens, qnorm_w, max_len: int,
                   q_pos: Optional[torch.Tensor] = None, theta: float = 1.0e6, eps: float = 1e-6,
                   out: Optional[torch.Tensor] = None,
                   stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """decode() without a workspace, for callers that cannot allocate one: the library's
    built-in scratch (NOALLOC_SCRATCH_BYTES per GPU) holds the partial results.  Calls
    that overlap on the GPU share that scratch and must be serialized."""
    lib = load()
    _check(q, "q", torch.bfloat16, 3)
    _check(k_cache, "k_cache", torch.bfloat16, 3)
    _check(v_cache, "v_cache", torch.bfloat16, 3)
    _check(cache_offsets, "cache_offsets", torch.int64, 1)
    _check(seqlens, "seqlens", torch.int32, 1)
    _check(qnorm_w, "qnorm_w", torch.float32, 1)
    if q_pos is not None:
        _check(q_pos, "q_pos", torch.int32, 1)
    B, H, D = q.shape
    Hkv = k_cache.shape[1]
    if out is None:
        out = torch.empty((B, H, D), dtype=torch.float32, device=q.device)
    _check(out, "out", torch.float32, 3)
    st = lib.gqa_attn_decode_noalloc(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(cache_offsets), _ptr(seqlens),
                                     _ptr(q_pos), _ptr(qnorm_w), float(theta), float(eps), _ptr(out), B, H, Hkv, D,
                                     int(max_len), _stream_handle(stream))
    _raise(st, "gqa_attn_decode_noalloc")
    return out


def device_status(stream: Optional[torch.cuda.Stream] = None) -> int:
    """Synchronize `stream`, read and clear the device error word; returns a status code."""
    return int(load().gqa_attn_device_status(_stream_handle(stream)))


def check_device_status(stream: Optional[torch.cuda.Stream] = None):
    _raise(device_status(stream), "device status")
