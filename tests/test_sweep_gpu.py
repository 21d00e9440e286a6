"""Seeded sweep of small random problems through the C ABI against the fp64 oracle, every
output row: dense prefill, packed variable-length prefill, chunked prefill on a paged cache,
contiguous and paged decode, over
random batch sizes, lengths (ragged tails, single tokens), head groupings (MHA to MQA, odd
heads per group), positions and RoPE variants.  The draws are fixed by the seed, so a failure
names a reproducible case.  Tolerance: max-abs 2e-2, mean-abs 2e-3 per element."""
import numpy as np
import pytest
import torch

from oracle import oracle
from grouped_query_causal_b200 import synthetic
from tests.gpu_helpers import assert_close, bits

pytestmark = pytest.mark.gpu

ROPES = [
    dict(),
    dict(pairing="half"),
    dict(scaling="linear", factor=2.0),
    dict(scaling="ntk", factor=4.0),
    dict(scaling="yarn", factor=8.0, original_max_position=512),
    dict(pairing="half", scaling="yarn", factor=4.0, original_max_position=1024),
]
GROUPS = [(1, 1), (2, 1), (2, 2), (3, 1), (4, 2), (5, 1), (8, 8), (6, 2), (4, 4), (12, 3), (16, 2)]   # (H, Hkv)


@pytest.fixture(scope="module")
def gqa():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for the gpu tests")
    from grouped_query_causal_b200 import binding
    binding.load()
    return binding


def _draw(case):
    rng = np.random.default_rng(9000 + case)
    H, Hkv = GROUPS[rng.integers(len(GROUPS))]
    return rng, H, Hkv, ROPES[rng.integers(len(ROPES))]


@pytest.mark.parametrize("case", range(16))
def test_prefill_sweep(gqa, case):
    rng, H, Hkv, kw = _draw(case)
    B = int(rng.integers(1, 4))
    T = int(rng.choice([1, 2, 63, 128, 129, int(rng.integers(3, 700))]))
    inp = synthetic.prefill_inputs(B, T, H, Hkv, seed=9100 + case)
    if rng.random() < 0.5:   # positions spread over a long context; the mask stays on the token index
        inp.pos = torch.from_numpy(np.sort(rng.integers(0, 50000, (B, T)), axis=1).astype(np.int32))
    theta = float(rng.choice([1.0e4, 1.0e6]))
    d = [t.cuda() for t in (inp.q, inp.k, inp.v, inp.pos, inp.wq, inp.wk)]
    out = gqa.prefill(*d, eps=inp.eps, rope=gqa.RopeConfig.make(theta=theta, **kw))
    torch.cuda.synchronize()
    gqa.check_device_status()
    rows = np.array([(b, h, i) for b in range(B) for h in range(H) for i in range(T)], np.int64)
    ref = oracle.prefill_rows_ex(bits(inp.q), bits(inp.k), bits(inp.v), inp.pos.numpy(), inp.wq.numpy(),
                                 inp.wk.numpy(), oracle.Rope(theta=theta, **kw), inp.eps, rows)
    got = out.cpu().numpy()[rows[:, 0], rows[:, 2], rows[:, 1]]
    assert_close(got, ref, f"prefill case {case}: B{B} T{T} H{H} Hkv{Hkv} {kw}")


@pytest.mark.parametrize("case", range(8))
def test_varlen_sweep(gqa, case):
    rng, H, Hkv, kw = _draw(100 + case)
    lens = [int(x) for x in rng.choice([0, 1, 2, 127, 128, 129, 200, 300, 450], size=int(rng.integers(1, 7)))]
    lens.append(int(rng.integers(1, 400)))   # at least one token
    N = int(sum(lens))
    inp = synthetic.prefill_inputs(1, max(N, 1), H, Hkv, seed=9200 + case)
    q, k, v = inp.q[0, :N].contiguous(), inp.k[0, :N].contiguous(), inp.v[0, :N].contiguous()
    pos = torch.cat([torch.arange(n, dtype=torch.int32) for n in lens])
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int64)
    out = gqa.prefill_varlen(q.cuda(), k.cuda(), v.cuda(), pos.cuda(), cu.cuda(), inp.wq.cuda(), inp.wk.cuda(),
                             max_seqlen=max(lens), eps=inp.eps, rope=gqa.RopeConfig.make(theta=inp.theta, **kw))
    torch.cuda.synchronize()
    gqa.check_device_status()
    ref = oracle.prefill_varlen_ex(bits(q), bits(k), bits(v), cu.numpy(), pos.numpy(), inp.wq.numpy(),
                                   inp.wk.numpy(), oracle.Rope(theta=inp.theta, **kw), inp.eps)
    assert_close(out.cpu().numpy(), ref, f"varlen case {case}: lens {lens} H{H} Hkv{Hkv} {kw}")


@pytest.mark.parametrize("case", range(10))
def test_decode_sweep(gqa, case):
    rng, H, Hkv, kw = _draw(200 + case)
    B = int(rng.integers(1, 7))
    seqlens = [int(x) for x in rng.integers(1, 3000, size=B)]
    d = synthetic.decode_inputs(B, H, Hkv, seed=9300 + case, seqlens=seqlens)
    qpos = torch.from_numpy(rng.integers(0, 60000, size=B).astype(np.int32)) if rng.random() < 0.5 else None
    rc, ro = gqa.RopeConfig.make(theta=d.theta, **kw), oracle.Rope(theta=d.theta, **kw)
    ref = oracle.decode_ex(bits(d.q), bits(d.k_cache), bits(d.v_cache), d.offsets.numpy(), d.seqlens.numpy(),
                           None if qpos is None else qpos.numpy(), d.wq.numpy(), ro, d.eps)
    qp = None if qpos is None else qpos.cuda()
    out = gqa.decode(d.q.cuda(), d.k_cache.cuda(), d.v_cache.cuda(), d.offsets.cuda(), d.seqlens.cuda(),
                     d.wq.cuda(), max_len=d.max_len, q_pos=qp, eps=d.eps, rope=rc)
    page = int(rng.choice([16, 32, 64, 128]))
    pc = synthetic.page_cache(d.k_cache, d.v_cache, d.offsets, seqlens, page, seed=9400 + case)
    paged = gqa.decode_paged(d.q.cuda(), pc.k_pages.cuda(), pc.v_pages.cuda(), pc.page_table.cuda(),
                             d.seqlens.cuda(), d.wq.cuda(), max_len=d.max_len, q_pos=qp, eps=d.eps, rope=rc)
    torch.cuda.synchronize()
    gqa.check_device_status()
    what = f"decode case {case}: seqlens {seqlens} H{H} Hkv{Hkv} {kw}"
    assert_close(out.cpu().numpy(), ref, what)
    assert_close(paged.cpu().numpy(), ref, f"paged ({page}-row pages) " + what)


@pytest.mark.parametrize("case", range(8))
def test_paged_chunk_sweep(gqa, case):
    rng, H, Hkv, kw = _draw(300 + case)
    B = int(rng.integers(1, 5))
    prefix = [int(x) for x in rng.choice([0, 1, 15, 16, 127, 128, 300, 1000], size=B)]
    chunk = [int(x) for x in rng.choice([1, 2, 64, 129, 200, 384], size=B)]
    page = int(rng.choice([16, 32, 64, 128, 256]))
    N = int(sum(chunk))
    inp = synthetic.prefill_inputs(1, N, H, Hkv, seed=9500 + case)
    q, k, v = inp.q[0].contiguous(), inp.k[0].contiguous(), inp.v[0].contiguous()
    pos = torch.cat([torch.arange(p, p + c, dtype=torch.int32) for p, c in zip(prefix, chunk)])
    cu = torch.tensor(np.concatenate([[0], np.cumsum(chunk)]), dtype=torch.int64)
    ro, rc = oracle.Rope(theta=inp.theta, **kw), gqa.RopeConfig.make(theta=inp.theta, **kw)
    # the cached prefix: the oracle's k-hat of random raw keys at positions 0 .. P-1, random values
    g = torch.Generator().manual_seed(9600 + case)
    caps = [p + c for p, c in zip(prefix, chunk)]
    offs = np.concatenate([[0], np.cumsum(caps)]).astype(np.int64)
    kc = torch.zeros(int(offs[-1]), Hkv, 128, dtype=torch.bfloat16)
    vc = torch.randn(int(offs[-1]), Hkv, 128, generator=g).to(torch.bfloat16)
    for b, p in enumerate(prefix):
        if p:
            raw = torch.randn(p, Hkv, 128, generator=g).to(torch.bfloat16)
            kh = oracle.qk_transform_ex(bits(raw), np.arange(p, dtype=np.int32), inp.wk.numpy(), ro, inp.eps)
            kc[offs[b]:offs[b] + p] = torch.from_numpy(kh).to(torch.bfloat16)
    pc = synthetic.page_cache(kc, vc, offs, caps, page, seed=9700 + case)
    out = gqa.prefill_chunk_paged(q.cuda(), k.cuda(), v.cuda(), pos.cuda(), cu.cuda(), pc.k_pages.cuda(),
                                  pc.v_pages.cuda(), pc.page_table.cuda(), torch.tensor(prefix, dtype=torch.int32).cuda(),
                                  inp.wq.cuda(), inp.wk.cuda(), max_chunk_len=max(chunk), eps=inp.eps, rope=rc)
    torch.cuda.synchronize()
    gqa.check_device_status()
    got = out.cpu().numpy()
    table = pc.page_table.numpy()
    for b, (p, c) in enumerate(zip(prefix, chunk)):
        lo, hi = int(cu[b]), int(cu[b + 1])
        ref, _ = oracle.prefill_chunk_paged_ex(
            bits(q[lo:hi]).reshape(1, c, H, 128), bits(k[lo:hi]).reshape(1, c, Hkv, 128),
            bits(v[lo:hi]).reshape(1, c, Hkv, 128), bits(pc.k_pages), bits(pc.v_pages), table[b:b + 1], page,
            np.array([p], np.int32), pos[lo:hi].numpy().reshape(1, c), inp.wq.numpy(), inp.wk.numpy(), ro, inp.eps)
        assert_close(got[lo:hi], ref[0], f"paged chunk case {case}, sequence {b}: P={prefix} C={chunk} "
                                         f"page {page} H{H} Hkv{Hkv} {kw}")
