"""GPU parity of the packed variable-length prefill (gqa_attn_prefill_varlen) and the
chunked prefill against a cached prefix (gqa_attn_prefill_chunk) with the fp64 oracle,
through the C ABI via the ctypes binding.  Tolerance: max-abs 2e-2, mean-abs 2e-3 per
element; cache rows the chunk writes are within one bf16 rounding of the oracle's k-hat
(values bit-exact), every other cache row is untouched."""
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


def _packed(lens, H, Hkv, seed, pos_of=None):
    """Raw q/k/v of sum(lens) tokens packed [N, heads, D], positions 0..len-1 per sequence
    (or pos_of(b, len)), cu_seqlens, norm weights."""
    N = int(sum(lens))
    inp = synthetic.prefill_inputs(1, max(N, 1), H, Hkv, seed=seed)
    q, k, v = inp.q[0, :N].contiguous(), inp.k[0, :N].contiguous(), inp.v[0, :N].contiguous()
    pos = torch.cat([torch.arange(n, dtype=torch.int32) if pos_of is None else pos_of(b, n)
                     for b, n in enumerate(lens)] or [torch.zeros(0, dtype=torch.int32)])
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int64)
    return q, k, v, pos, cu, inp.wq, inp.wk, inp.theta, inp.eps


@pytest.mark.parametrize("H,Hkv", [(16, 4), (8, 8), (12, 4), (16, 1)])
def test_varlen_against_oracle(gqa, H, Hkv):
    lens = [300, 0, 1, 127, 128, 129, 513, 77, 1000]
    q, k, v, pos, cu, wq, wk, theta, eps = _packed(lens, H, Hkv, seed=100 + H + Hkv)
    out = gqa.prefill_varlen(q.cuda(), k.cuda(), v.cuda(), pos.cuda(), cu.cuda(), wq.cuda(), wk.cuda(),
                             max_seqlen=max(lens), eps=eps, rope=gqa.RopeConfig.make(theta=theta))
    torch.cuda.synchronize()
    gqa.check_device_status()
    ref = oracle.prefill_varlen_ex(bits(q), bits(k), bits(v), cu.numpy(), pos.numpy(), wq.numpy(), wk.numpy(),
                                   oracle.Rope(theta=theta), eps)
    assert_close(out.cpu().numpy(), ref, f"varlen H={H} Hkv={Hkv}")


def test_varlen_with_rope_variant(gqa):
    lens = [700, 5, 260]
    kw = dict(pairing="half", scaling="yarn", factor=8.0, original_max_position=256)
    q, k, v, pos, cu, wq, wk, theta, eps = _packed(lens, 16, 4, seed=120,
                                                   pos_of=lambda b, n: torch.arange(n, dtype=torch.int32) * 3 + b)
    out = gqa.prefill_varlen(q.cuda(), k.cuda(), v.cuda(), pos.cuda(), cu.cuda(), wq.cuda(), wk.cuda(),
                             max_seqlen=max(lens), eps=eps, rope=gqa.RopeConfig.make(theta=theta, **kw))
    torch.cuda.synchronize()
    gqa.check_device_status()
    ref = oracle.prefill_varlen_ex(bits(q), bits(k), bits(v), cu.numpy(), pos.numpy(), wq.numpy(), wk.numpy(),
                                   oracle.Rope(theta=theta, **kw), eps)
    assert_close(out.cpu().numpy(), ref, "varlen, rotate-half + YaRN")


def test_equal_lengths_equal_dense_prefill(gqa):
    """B sequences of one length packed = the dense [B, T] prefill, bit for bit."""
    B, T, H, Hkv = 3, 300, 8, 2
    inp = synthetic.prefill_inputs(B, T, H, Hkv, seed=121)
    d = [t.cuda() for t in (inp.q, inp.k, inp.v, inp.pos, inp.wq, inp.wk)]
    dense = gqa.prefill(*d, theta=inp.theta, eps=inp.eps)
    cu = (torch.arange(B + 1, dtype=torch.int64) * T).cuda()
    packed = gqa.prefill_varlen(d[0].reshape(B * T, H, 128), d[1].reshape(B * T, Hkv, 128),
                                d[2].reshape(B * T, Hkv, 128), d[3].reshape(B * T), cu, d[4], d[5], max_seqlen=T,
                                eps=inp.eps, rope=gqa.RopeConfig.make(theta=inp.theta))
    torch.cuda.synchronize()
    gqa.check_device_status()
    assert torch.equal(dense.reshape(B * T, H, 128), packed)


def _cache_with_prefix(prefix, chunk, Hkv, wk, theta, eps, rope_kw, seed, spare=3):
    """A cache holding, per sequence, the oracle's bf16 k-hat and raw v of `prefix[b]`
    earlier tokens, room for the chunk and `spare` rows of random filler after it.
    Returns (k_cache, v_cache, offsets, prefix raw keys' positions)."""
    g = torch.Generator().manual_seed(seed)
    caps = [p + c + spare for p, c in zip(prefix, chunk)]
    rows = int(sum(caps))
    kc = (torch.randn(rows, Hkv, 128, generator=g)).to(torch.bfloat16)
    vc = (torch.randn(rows, Hkv, 128, generator=g)).to(torch.bfloat16)
    offs = np.concatenate([[0], np.cumsum(caps)]).astype(np.int64)
    ro = oracle.Rope(theta=theta, **rope_kw)
    for b, p in enumerate(prefix):
        if p == 0:
            continue
        raw = (torch.randn(p, Hkv, 128, generator=g)).to(torch.bfloat16)
        kh = oracle.qk_transform_ex(bits(raw), np.arange(p, dtype=np.int32), wk.numpy(), ro, eps)
        kc[offs[b]:offs[b] + p] = torch.from_numpy(kh).to(torch.bfloat16)
    return kc, vc, torch.from_numpy(offs)


def _chunk_case(gqa, prefix, chunk, H, Hkv, seed, rope_kw=None):
    rope_kw = rope_kw or {}
    q, k, v, _, cu, wq, wk, theta, eps = _packed(chunk, H, Hkv, seed)
    pos = torch.cat([torch.arange(p, p + c, dtype=torch.int32) for p, c in zip(prefix, chunk)])
    kc, vc, offs = _cache_with_prefix(prefix, chunk, Hkv, wk, theta, eps, rope_kw, seed + 1)
    pl = torch.tensor(prefix, dtype=torch.int32)
    kcd, vcd = kc.cuda(), vc.cuda()
    out = gqa.prefill_chunk(q.cuda(), k.cuda(), v.cuda(), pos.cuda(), cu.cuda(), kcd, vcd, offs.cuda(), pl.cuda(),
                            wq.cuda(), wk.cuda(), max_chunk_len=max(chunk), eps=eps,
                            rope=gqa.RopeConfig.make(theta=theta, **rope_kw))
    torch.cuda.synchronize()
    gqa.check_device_status()
    got = out.cpu().numpy()
    kcd, vcd = kcd.cpu(), vcd.cpu()
    ro = oracle.Rope(theta=theta, **rope_kw)
    written = torch.zeros(kc.shape[0], dtype=torch.bool)
    for b, (p, c) in enumerate(zip(prefix, chunk)):
        lo, hi = int(cu[b]), int(cu[b + 1])
        o = int(offs[b])
        ref, khat = oracle.prefill_chunk_ex(
            bits(q[lo:hi]).reshape(1, c, H, 128), bits(k[lo:hi]).reshape(1, c, Hkv, 128),
            bits(v[lo:hi]).reshape(1, c, Hkv, 128), bits(kc[o:o + max(p, 1)]), bits(vc[o:o + max(p, 1)]),
            np.array([0, p], np.int64), np.array([p], np.int32), pos[lo:hi].numpy().reshape(1, c), wq.numpy(),
            wk.numpy(), ro, eps)
        assert_close(got[lo:hi], ref[0], f"chunk seq {b} (P={p}, C={c})")
        gk = kcd[o + p:o + p + c].double().numpy()
        assert (np.abs(gk - khat[0]) <= 2.0 ** -8 * np.abs(khat[0]) + 1e-5).all(), f"k-hat rows of sequence {b}"
        assert torch.equal(vcd[o + p:o + p + c], v[lo:hi]), f"value rows of sequence {b}"
        written[o + p:o + p + c] = True
    assert torch.equal(kcd[~written], kc[~written]) and torch.equal(vcd[~written], vc[~written])


@pytest.mark.parametrize("prefix,chunk,H,Hkv", [
    ([256], [256], 8, 2),                       # prefix and chunk whole tiles
    ([200, 0], [300, 77], 16, 4),               # ragged prefix; a sequence without prefix
    ([1000, 1, 37], [77, 257, 5], 32, 8),
    ([128, 4096], [1, 128], 12, 4),             # one-token chunk; long prefix; odd heads per group
    ([300], [300], 16, 1),                      # MQA
])
def test_chunk_against_oracle(gqa, prefix, chunk, H, Hkv):
    _chunk_case(gqa, prefix, chunk, H, Hkv, seed=130 + sum(prefix) % 97)


def test_chunk_with_rope_variant(gqa):
    _chunk_case(gqa, [300, 64], [200, 129], 16, 4, seed=140,
                rope_kw=dict(pairing="half", scaling="yarn", factor=8.0, original_max_position=256))


def test_chunks_in_sequence_equal_one_prefill(gqa):
    """A prompt prefilled as three chunks into one cache (prefix_len advanced by the
    caller between calls) gives the rows of a single causal prefill over the whole
    prompt, checked against the oracle's prefill."""
    T, H, Hkv = 700, 16, 4
    inp = synthetic.prefill_inputs(1, T, H, Hkv, seed=150)
    q, k, v, pos = inp.q[0].cuda(), inp.k[0].cuda(), inp.v[0].cuda(), inp.pos[0].cuda()
    wq, wk = inp.wq.cuda(), inp.wk.cuda()
    kc = torch.zeros(T, Hkv, 128, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    offs = torch.tensor([0, T], dtype=torch.int64, device="cuda")
    rope = gqa.RopeConfig.make(theta=inp.theta)
    outs = []
    for lo, hi in ((0, 250), (250, 256), (256, 700)):
        cu = torch.tensor([0, hi - lo], dtype=torch.int64, device="cuda")
        pl = torch.tensor([lo], dtype=torch.int32, device="cuda")
        outs.append(gqa.prefill_chunk(q[lo:hi].contiguous(), k[lo:hi].contiguous(), v[lo:hi].contiguous(),
                                      pos[lo:hi].contiguous(), cu, kc, vc, offs, pl, wq, wk, max_chunk_len=hi - lo,
                                      eps=inp.eps, rope=rope))
    torch.cuda.synchronize()
    gqa.check_device_status()
    got = torch.cat(outs).cpu().numpy()
    ref = oracle.prefill(bits(inp.q), bits(inp.k), bits(inp.v), inp.pos.numpy(), inp.wq.numpy(), inp.wk.numpy(),
                         inp.theta, inp.eps)[0]
    assert_close(got, ref, "three chunks")


def test_chunk_overflowing_its_rows_is_a_device_input_error(gqa):
    """A chunk that does not fit its sequence's cache rows writes nothing outside them and
    raises the device input status."""
    q, k, v, _, cu, wq, wk, theta, eps = _packed([40, 40], 8, 2, seed=160)
    pos = torch.arange(80, dtype=torch.int32)
    kc = torch.zeros(100, 2, 128, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    offs = torch.tensor([0, 50, 100], dtype=torch.int64, device="cuda")   # 50 rows each
    pl = torch.tensor([5, 20], dtype=torch.int32, device="cuda")        # sequence 1: 20 + 40 > 50
    gqa.prefill_chunk(q.cuda(), k.cuda(), v.cuda(), pos.cuda(), cu.cuda(), kc, vc, offs, pl, wq.cuda(), wk.cuda(),
                      max_chunk_len=40, eps=eps, rope=gqa.RopeConfig.make(theta=theta))
    torch.cuda.synchronize()
    assert gqa.device_status() == -6
    kcpu = kc.cpu()
    assert (kcpu[:5] == 0).all() and (kcpu[45:70] == 0).all()   # nothing before the rows it may write
    assert gqa.device_status() == 0


def test_varlen_sequence_longer_than_max_is_a_device_input_error(gqa):
    """A sequence longer than max_seqlen gets no work (the unit list leaves it out) and
    raises the device input status; the other sequences are still right."""
    lens = [300, 200, 50]
    q, k, v, pos, cu, wq, wk, theta, eps = _packed(lens, 8, 2, seed=170)
    out = gqa.prefill_varlen(q.cuda(), k.cuda(), v.cuda(), pos.cuda(), cu.cuda(), wq.cuda(), wk.cuda(),
                             max_seqlen=256, eps=eps, rope=gqa.RopeConfig.make(theta=theta))
    torch.cuda.synchronize()
    assert gqa.device_status() == -6
    assert gqa.device_status() == 0
    ref = oracle.prefill_varlen_ex(bits(q), bits(k), bits(v), cu.numpy(), pos.numpy(), wq.numpy(), wk.numpy(),
                                   oracle.Rope(theta=theta), eps)
    assert_close(out.cpu().numpy()[300:], ref[300:], "the sequences within max_seqlen")


def test_varlen_overlapping_sequences_cannot_overrun_the_unit_list(gqa):
    """cu_seqlens that is not ascending describes overlapping sequences whose units can
    outnumber the list's room (one entry per 128 tokens plus one per sequence of N tokens):
    the list keeps to its room and the call raises the device input status."""
    N, B = 10, 40
    q, k, v, pos, _, wq, wk, theta, eps = _packed([N], 4, 2, seed=171)
    cu = torch.tensor([0 if i % 2 == 0 else N for i in range(B + 1)], dtype=torch.int64)   # 0, N, 0, N, ...
    gqa.prefill_varlen(q.cuda(), k.cuda(), v.cuda(), pos.cuda(), cu.cuda(), wq.cuda(), wk.cuda(), max_seqlen=N,
                       eps=eps, rope=gqa.RopeConfig.make(theta=theta))
    torch.cuda.synchronize()
    assert gqa.device_status() == -6
    assert gqa.device_status() == 0
