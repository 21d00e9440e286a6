"""The zero-allocation decode entry point, gqa_attn_decode_noalloc.

Some callers cannot allocate device memory or pass a workspace: a plugin inside a
host framework that owns the whole device memory pool, or a serving loop that must
never call cudaMalloc.  For them the library keeps the decode scratch in a fixed
array of its own.  These tests call that entry point through the C ABI and check it
against gqa_attn_decode (which takes a caller-provided workspace), twice in a row with
different inputs, since every call reuses the same scratch.  The file is named so
that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

from grouped_query_causal_b200 import synthetic
from tests.gpu_helpers import MAX_ABS, MEAN_ABS, decode_to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for the gpu tests")
    from grouped_query_causal_b200 import binding
    return binding.load()


def _call_noalloc(lib, d, B, H, Hkv, max_len, out):
    return lib.gqa_attn_decode_noalloc(
        d["q"].data_ptr(), d["k_cache"].data_ptr(), d["v_cache"].data_ptr(), d["cache_offsets"].data_ptr(),
        d["seqlens"].data_ptr(), None, d["qnorm_w"].data_ptr(), d["theta"], d["eps"], out.data_ptr(), B, H, Hkv,
        128, max_len, torch.cuda.current_stream().cuda_stream)


def _call_with_workspace(lib, d, B, H, Hkv, max_len, out):
    ws = torch.empty(lib.gqa_attn_decode_workspace_size(B, H, Hkv, 128, max_len), dtype=torch.uint8, device="cuda")
    st = lib.gqa_attn_decode(
        d["q"].data_ptr(), d["k_cache"].data_ptr(), d["v_cache"].data_ptr(), d["cache_offsets"].data_ptr(),
        d["seqlens"].data_ptr(), None, d["qnorm_w"].data_ptr(), d["theta"], d["eps"], out.data_ptr(), B, H, Hkv,
        128, max_len, ws.data_ptr(), ws.numel(), torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    return st


def test_noalloc_matches_workspace_decode_on_two_calls_in_a_row(lib):
    cases = [  # the first call leaves its partials in the shared scratch; the second must not see them
        synthetic.decode_inputs(8, 32, 8, seed=41, seqlens=[8192, 1, 5000, 513, 777, 4096, 2048, 8000]),
        synthetic.decode_inputs(5, 16, 4, seed=42, seqlens=[300, 2500, 1, 1024, 64]),
    ]
    for inp in cases:
        B, H, _ = inp.q.shape
        Hkv = inp.k_cache.shape[1]
        max_len = inp.max_len
        d = decode_to_dev(inp)
        out = torch.full((B, H, 128), float("nan"), device="cuda")
        assert _call_noalloc(lib, d, B, H, Hkv, max_len, out) == 0
        torch.cuda.synchronize()
        ref = torch.empty_like(out)
        assert _call_with_workspace(lib, d, B, H, Hkv, max_len, ref) == 0
        assert lib.gqa_attn_device_status(None) == 0
        got, want = out.cpu().numpy().astype(np.float64), ref.cpu().numpy().astype(np.float64)
        assert np.isfinite(got).all()
        err = np.abs(got - want)
        assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (err.max(), err.mean())


def test_noalloc_rejects_problems_beyond_its_scratch(lib):
    from grouped_query_causal_b200 import binding
    # 64 sequences x 32 heads with up to 32768 cached tokens needs about 68 MB of partials
    need = lib.gqa_attn_decode_workspace_size(64, 32, 8, 128, 32768)
    assert need > binding.NOALLOC_SCRATCH_BYTES
    dummy = torch.zeros(16, dtype=torch.uint8, device="cuda")
    p = dummy.data_ptr()
    st = lib.gqa_attn_decode_noalloc(p, p, p, p, p, None, p, 1e6, 1e-6, p, 64, 32, 8, 128, 32768, None)
    assert st == -3   # GQA_ERR_WORKSPACE, returned before anything is launched
