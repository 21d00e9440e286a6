"""GPU parity of the projection GEMM (gqa_linear: y = x W^T, the fused QKV projection
and the output projection of the "Qwen3" walkthrough's attention forward) against the
fp64 oracle, through the C ABI via the ctypes binding.  Tolerance: max-abs 2e-2,
mean-abs 2e-3 per element, on outputs of unit scale (weights scaled by 1/sqrt(K))."""
import numpy as np
import pytest
import torch

from oracle import oracle
from grouped_query_causal_b200 import synthetic
from tests.gpu_helpers import assert_close, bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gqa():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for the gpu tests")
    from grouped_query_causal_b200 import binding
    binding.load()
    return binding


def _inputs(M, N, K, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(M, K, generator=g).to(torch.bfloat16)
    w = (torch.randn(N, K, generator=g) / K ** 0.5).to(torch.bfloat16)
    return x, w


@pytest.mark.parametrize("M,N,K", [(1, 32, 8), (128, 256, 64), (129, 288, 200), (300, 1536, 512),
                                   (1000, 96, 4096), (257, 6144, 128)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_linear_against_oracle(gqa, M, N, K, dtype):
    """Ragged M (partial 128-row tiles), N not a multiple of the 256-column tile, K not a
    multiple of the 64-deep stage (zero-filled tail), one and many K stages."""
    x, w = _inputs(M, N, K, seed=M + N + K)
    y = gqa.linear(x.cuda(), w.cuda(), out_dtype=dtype)
    torch.cuda.synchronize()
    gqa.check_device_status()
    ref = oracle.linear(bits(x), bits(w))
    assert_close(y.float().cpu().numpy(), ref, f"linear M={M} N={N} K={K} {dtype}")


def test_linear_persistent_many_tiles(gqa):
    """More tiles than SMs (every CTA walks several tiles and reuses both accumulators);
    rows sampled across the whole output."""
    M, N, K = 4096, 2048, 1024
    x, w = _inputs(M, N, K, seed=7)
    y = gqa.linear(x.cuda(), w.cuda(), out_dtype=torch.float32)
    torch.cuda.synchronize()
    gqa.check_device_status()
    rows = np.unique(np.concatenate([np.arange(0, M, 37), [0, 127, 128, M - 1]]))
    ref = oracle.linear(bits(x)[rows], bits(w))
    assert_close(y.cpu().numpy()[rows], ref, "linear 4096x2048x1024")


def test_linear_deterministic(gqa):
    x, w = _inputs(300, 512, 320, seed=8)
    a = gqa.linear(x.cuda(), w.cuda())
    b = gqa.linear(x.cuda(), w.cuda())
    torch.cuda.synchronize()
    assert torch.equal(a, b)


@pytest.mark.parametrize("B,T,hidden,H,Hkv", [(2, 300, 512, 8, 2), (1, 129, 256, 4, 4), (1, 640, 1024, 16, 8)])
def test_attention_block_against_oracle(gqa, B, T, hidden, H, Hkv):
    """The whole sub-block: qkv projection, q/k norm, RoPE, causal GQA attention on the
    q/k/v sections read in place, bf16 attention output, output projection."""
    D = 128
    g = torch.Generator().manual_seed(B * 1000 + T)
    x = torch.randn(B, T, hidden, generator=g).to(torch.bfloat16)
    w_qkv = (torch.randn((H + 2 * Hkv) * D, hidden, generator=g) / hidden ** 0.5).to(torch.bfloat16)
    w_o = (torch.randn(hidden, H * D, generator=g) / (H * D) ** 0.5).to(torch.bfloat16)
    pos = torch.arange(T, dtype=torch.int32).repeat(B, 1)
    wq = torch.rand(D, generator=g) + 0.5
    wk = torch.rand(D, generator=g) + 0.5
    y = gqa.attn_block_prefill(x.cuda(), w_qkv.cuda(), w_o.cuda(), pos.cuda(), wq.cuda(), wk.cuda(), H, Hkv,
                               eps=1e-6, rope=gqa.RopeConfig.make(theta=1e6))
    torch.cuda.synchronize()
    gqa.check_device_status()
    ref = oracle.attn_block_prefill(bits(x), bits(w_qkv), bits(w_o), pos.numpy(), wq.numpy(), wk.numpy(),
                                    oracle.Rope(theta=1e6), 1e-6, H, Hkv, D)
    assert_close(y.cpu().numpy(), ref, f"attention block B={B} T={T} hidden={hidden} H={H} Hkv={Hkv}")
