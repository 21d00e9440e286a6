"""The zero-allocation decode entry point, gqa_attn_decode_noalloc.

Some callers cannot allocate device memory or pass a workspace: a plugin inside a
host framework that owns the whole device memory pool, or a serving loop that must
never call cudaMalloc.  For them the library keeps the decode scratch in a fixed
array of its own.  These tests call that entry point through the C ABI and check it
against gqa_attn_decode (which takes a caller-provided workspace; the two run the same
kernels with the same launch geometry, so the results must be bit-identical) and
against the fp64 oracle, on several calls in a row, since every call reuses the same
scratch.  The file is named so that pytest collects it last.
"""
import numpy as np
import pytest
import torch

from oracle import oracle
from grouped_query_causal_b200 import synthetic
from tests.gpu_helpers import assert_close, bits, decode_to_dev

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


def _oracle(inp):
    return oracle.decode(bits(inp.q), bits(inp.k_cache), bits(inp.v_cache), inp.offsets.numpy(),
                         inp.seqlens.numpy(), None, inp.wq.numpy(), inp.theta, inp.eps)


def _check_one(lib, inp, max_len=None):
    B, H, _ = inp.q.shape
    Hkv = inp.k_cache.shape[1]
    max_len = max_len or inp.max_len
    d = decode_to_dev(inp)
    out = torch.full((B, H, 128), float("nan"), device="cuda")
    assert _call_noalloc(lib, d, B, H, Hkv, max_len, out) == 0
    torch.cuda.synchronize()
    ref = torch.empty_like(out)
    assert _call_with_workspace(lib, d, B, H, Hkv, max_len, ref) == 0
    assert lib.gqa_attn_device_status(None) == 0
    got = out.cpu().numpy()
    np.testing.assert_array_equal(got, ref.cpu().numpy())
    assert_close(got, _oracle(inp), f"noalloc decode B={B} H={H} Hkv={Hkv}")


def test_noalloc_matches_workspace_decode_and_oracle_on_calls_in_a_row(lib):
    # small, then larger (its merge reads scratch slots the first call wrote, so stale
    # partials would show), then small again after the large one
    _check_one(lib, synthetic.decode_inputs(5, 16, 4, seed=42, seqlens=[300, 2500, 1, 1024, 64]))
    _check_one(lib, synthetic.decode_inputs(8, 32, 8, seed=41, seqlens=[8192, 1, 5000, 513, 777, 4096, 2048, 8000]))
    _check_one(lib, synthetic.decode_inputs(3, 8, 2, seed=43, seqlens=[1025, 3, 2049]))


def test_noalloc_limit_is_the_header_size(lib):
    """The largest problem whose partials fit GQA_NOALLOC_SCRATCH_BYTES (as the header
    defines it) runs; one chunk more is rejected before any launch."""
    from grouped_query_causal_b200 import binding
    B, H, Hkv = 63, 1, 1
    size = lambda mc: lib.gqa_attn_decode_workspace_size(B, H, Hkv, 128, mc * 1024)  # noqa: E731
    mc = 1
    while size(mc + 1) <= binding.NOALLOC_SCRATCH_BYTES:
        mc += 1
    assert size(mc) <= binding.NOALLOC_SCRATCH_BYTES < size(mc + 1)
    inp = synthetic.decode_inputs(B, H, Hkv, seed=44, seqlens=[1 + (7 * b) % 40 for b in range(B)])
    _check_one(lib, inp, max_len=mc * 1024)           # uses all but the tail of the scratch
    d = decode_to_dev(inp)
    out = torch.empty((B, H, 128), device="cuda")
    assert _call_noalloc(lib, d, B, H, Hkv, mc * 1024 + 1, out) == -3   # GQA_ERR_WORKSPACE


def test_noalloc_argument_errors_come_before_the_size_limit(lib):
    from grouped_query_causal_b200 import binding
    # 64 sequences x 32 heads with up to 32768 cached tokens needs about 68 MB of partials
    need = lib.gqa_attn_decode_workspace_size(64, 32, 8, 128, 32768)
    assert need > binding.NOALLOC_SCRATCH_BYTES
    dummy = torch.zeros(16, dtype=torch.uint8, device="cuda")
    p = dummy.data_ptr()
    st = lib.gqa_attn_decode_noalloc(p, p, p, p, p, None, p, 1e6, 1e-6, p, 64, 32, 8, 128, 32768, None)
    assert st == -3   # GQA_ERR_WORKSPACE, returned before anything is launched
    # a null query pointer on the same oversize problem is an argument error
    st = lib.gqa_attn_decode_noalloc(None, p, p, p, p, None, p, 1e6, 1e-6, p, 64, 32, 8, 128, 32768, None)
    assert st == -1   # GQA_ERR_INVALID_ARG
    st = lib.gqa_attn_decode_noalloc(p, p, p, p, p, None, p, -1.0, 1e-6, p, 64, 32, 8, 128, 32768, None)
    assert st == -1
