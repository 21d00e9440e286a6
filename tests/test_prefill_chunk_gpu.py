"""GPU parity of gqa_attn_prefill_chunk (a chunk of C tokens against a cached prefix of P
rows) against the fp64 oracle.  Tolerance: max-abs 2e-2, mean-abs 2e-3 per element."""
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


def _run(gqa, B, P, C, H, Hkv, seed, rope_kw=None):
    """GPU: k-hat of all P + C tokens from gqa_attn_k_norm_rope_ex (the prefix as a cache
    would hold it), then the chunked attention.  Oracle: its own bf16 prefix cache and the
    chunk's raw tokens."""
    rope_kw = rope_kw or {}
    inp = synthetic.prefill_inputs(B, P + C, H, Hkv, seed=seed)
    rc = gqa.RopeConfig.make(theta=inp.theta, **rope_kw)
    ro = oracle.Rope(theta=inp.theta, **rope_kw)
    k, v, q = inp.k.cuda(), inp.v.cuda(), inp.q.cuda()
    pos = inp.pos.cuda()
    wq, wk = inp.wq.cuda(), inp.wk.cuda()
    kh = gqa.k_norm_rope(k, pos, wk, eps=inp.eps, rope=rc)          # [B, P+C, Hkv, D], every token
    qc = q[:, P:].contiguous()
    pc = pos[:, P:].contiguous()
    out = gqa.prefill_chunk(qc, kh, v, pc, wq, eps=inp.eps, rope=rc)
    torch.cuda.synchronize()
    gqa.check_device_status()
    # the oracle's prefix cache: its own k-hat of the first P tokens, stored as bf16
    kpre = oracle.qk_transform_ex(bits(inp.k)[:, :P].reshape(B * P, Hkv, 128), inp.pos.numpy()[:, :P].reshape(B * P),
                                  inp.wk.numpy(), ro, inp.eps)
    kc = torch.from_numpy(kpre).to(torch.bfloat16)
    vc = inp.v[:, :P].reshape(B * P, Hkv, 128)
    offsets = np.arange(B + 1, dtype=np.int64) * P
    ref, _ = oracle.prefill_chunk_ex(bits(inp.q)[:, P:], bits(inp.k)[:, P:], bits(inp.v)[:, P:], bits(kc), bits(vc),
                                     offsets, np.full(B, P, np.int32), inp.pos.numpy()[:, P:], inp.wq.numpy(),
                                     inp.wk.numpy(), ro, inp.eps)
    return out.cpu().numpy(), ref, (q, kh, v, pos, wq, rc, inp)


@pytest.mark.parametrize("B,P,C,H,Hkv", [(2, 200, 300, 16, 4), (1, 128, 128, 8, 8), (1, 37, 5, 8, 1),
                                         (2, 1000, 77, 32, 8), (1, 1, 257, 12, 4)])
def test_chunk_against_oracle(gqa, B, P, C, H, Hkv):
    got, ref, _ = _run(gqa, B, P, C, H, Hkv, seed=90 + P)
    assert_close(got, ref, f"chunk B={B} P={P} C={C} H={H} Hkv={Hkv}")


def test_chunk_with_rope_variant(gqa):
    got, ref, _ = _run(gqa, 1, 300, 200, 16, 4, seed=91,
                       rope_kw=dict(pairing="half", scaling="yarn", factor=8.0, original_max_position=256))
    assert_close(got, ref, "chunk, rotate-half + YaRN")


def test_empty_prefix_is_plain_prefill(gqa):
    inp = synthetic.prefill_inputs(2, 300, 8, 2, seed=92)
    q, k, v, pos = inp.q.cuda(), inp.k.cuda(), inp.v.cuda(), inp.pos.cuda()
    wq, wk = inp.wq.cuda(), inp.wk.cuda()
    rc = gqa.RopeConfig.make(theta=inp.theta)
    kh = gqa.k_norm_rope(k, pos, wk, eps=inp.eps, rope=rc)
    a = gqa.prefill_khat(q, kh, v, pos, wq, eps=inp.eps, rope=rc)
    b = gqa.prefill_chunk(q, kh, v, pos, wq, eps=inp.eps, rope=rc)
    torch.cuda.synchronize()
    gqa.check_device_status()
    assert torch.equal(a, b)
