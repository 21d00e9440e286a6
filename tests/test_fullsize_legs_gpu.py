"""GPU parity at the full sizes of the benchmark's packed variable-length, chunked, paged
chunked and projection workloads, in the launch configuration the benchmark times, on
sampled outputs against the fp64 oracle (max-abs 2e-2, mean-abs 2e-3 per element), and
on what holds at any size: every k-hat / v row the chunk writes (k-hat within one bf16
rounding of the oracle's, v exact), the rows it must not touch, and the paged chunk equal
to the contiguous one bit for bit."""
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


def _sample_rows(n, rng, extra):
    """Token rows of a sequence of n tokens: the first and last, the tile edges 127 / 128
    where present, and `extra` random ones."""
    fixed = [i for i in (0, 127, 128, n - 1) if 0 <= i < n]
    return sorted(set(fixed) | set(int(i) for i in rng.integers(0, n, extra)))


def test_varlen_workload_sampled_rows(gqa):
    """16 packed sequences of U[256, 8192] tokens, H32 Hkv8: every head of every sequence on
    its first and last rows, its tile edges and two random rows."""
    w = synthetic.make("varlen_prefill")
    N, H, D = w.q.shape
    lens = w.lens
    out = gqa.prefill_varlen(w.q.cuda(), w.k.cuda(), w.v.cuda(), w.pos.cuda(), w.cu.cuda(), w.wq.cuda(),
                             w.wk.cuda(), max_seqlen=max(lens), eps=w.eps, rope=gqa.RopeConfig.make(theta=w.theta))
    torch.cuda.synchronize()
    gqa.check_device_status()
    got = out.cpu().numpy()
    rng = np.random.default_rng(501)
    ro = oracle.Rope(theta=w.theta)
    for b, n in enumerate(lens):
        lo = int(w.cu[b])
        rows = np.array([(0, h, i) for h in range(H) for i in _sample_rows(n, rng, 2)], np.int64)
        ref = oracle.prefill_rows_ex(bits(w.q[lo:lo + n]).reshape(1, n, H, D),
                                     bits(w.k[lo:lo + n]).reshape(1, n, -1, D),
                                     bits(w.v[lo:lo + n]).reshape(1, n, -1, D), w.pos[lo:lo + n].numpy().reshape(1, n),
                                     w.wq.numpy(), w.wk.numpy(), ro, w.eps, rows)
        assert_close(got[lo + rows[:, 2], rows[:, 1]], ref, f"varlen sequence {b} (length {n})")


def _chunk_rows(w, H, rng):
    C = w.lens[0]
    return np.array([(b, h, i) for b in range(len(w.lens)) for h in range(H)
                     for i in _sample_rows(C, rng, 2)], np.int64)


def test_chunk_workloads_sampled_rows(gqa):
    """8 sequences with 8192 cached rows and a 2048-token chunk, H32 Hkv8: the chunk on the
    contiguous cache against the oracle on sampled rows of every head, every written cache
    row against the oracle's k-hat and the raw v, the other rows untouched; then the same
    chunk on the cache cut into shuffled 16-row pages, equal to it bit for bit (outputs and
    written rows)."""
    w = synthetic.make("chunked_prefill")
    N, H, D = w.q.shape
    Hkv = w.k.shape[1]
    B, C = len(w.lens), w.lens[0]
    rope = gqa.RopeConfig.make(theta=w.theta)
    dev = [t.cuda() for t in (w.q, w.k, w.v, w.pos, w.cu)]
    kc, vc = w.k_cache.cuda(), w.v_cache.cuda()
    out = gqa.prefill_chunk(*dev, kc, vc, w.cache_offsets.cuda(), w.prefix.cuda(), w.wq.cuda(), w.wk.cuda(),
                            max_chunk_len=C, eps=w.eps, rope=rope)
    caps = [int(p) + n for p, n in zip(w.prefix.tolist(), w.lens)]
    pc = synthetic.page_cache(w.k_cache, w.v_cache, w.cache_offsets, caps, 16, seed=31)
    kp, vp = pc.k_pages.cuda(), pc.v_pages.cuda()
    outp = gqa.prefill_chunk_paged(*dev, kp, vp, pc.page_table.cuda(), w.prefix.cuda(), w.wq.cuda(), w.wk.cuda(),
                                   max_chunk_len=C, eps=w.eps, rope=rope)
    torch.cuda.synchronize()
    gqa.check_device_status()
    got = out.cpu()
    assert torch.equal(outp.cpu(), got), "paged and contiguous chunk differ"
    rows = _chunk_rows(w, H, np.random.default_rng(502))
    ref, khat = oracle.prefill_chunk_rows_ex(
        bits(w.q).reshape(B, C, H, D), bits(w.k).reshape(B, C, Hkv, D), bits(w.v).reshape(B, C, Hkv, D),
        bits(w.k_cache), bits(w.v_cache), w.cache_offsets.numpy(), w.prefix.numpy(), w.pos.numpy().reshape(B, C),
        w.wq.numpy(), w.wk.numpy(), oracle.Rope(theta=w.theta), w.eps, rows)
    assert_close(got.numpy()[rows[:, 0] * C + rows[:, 2], rows[:, 1]], ref, f"chunk, {len(rows)} rows")
    kcd, vcd = kc.cpu(), vc.cpu()
    written = torch.zeros(kcd.shape[0], dtype=torch.bool)
    table = pc.page_table.numpy()
    kpd, vpd = kp.cpu(), vp.cpu()
    for b in range(B):
        o, p = int(w.cache_offsets[b]), int(w.prefix[b])
        gk = kcd[o + p:o + p + C].double().numpy()
        assert (np.abs(gk - khat[b]) <= 2.0 ** -8 * np.abs(khat[b]) + 1e-5).all(), f"k-hat rows of sequence {b}"
        assert torch.equal(vcd[o + p:o + p + C], w.v[b * C:(b + 1) * C]), f"value rows of sequence {b}"
        written[o + p:o + p + C] = True
        r = np.arange(p, p + C)
        pg, pr = table[b, r // 16].astype(np.int64), r % 16
        assert torch.equal(kpd[pg, pr], kcd[o + p:o + p + C]), f"paged k-hat rows, sequence {b}"
        assert torch.equal(vpd[pg, pr], vcd[o + p:o + p + C]), f"paged value rows, sequence {b}"
    assert torch.equal(kcd[~written], w.k_cache[~written]) and torch.equal(vcd[~written], w.v_cache[~written])


def test_projection_workload_sampled_rows(gqa):
    """The QKV projection (16384 x 4096 -> 6144, bf16 out) and the output projection
    (16384 x 4096 -> 4096, fp32 out) on the benchmark's inputs, about 70 rows sampled across
    the whole output (tile edges among them) against the oracle."""
    w = synthetic.make("projections")
    x = w.x.cuda()
    qkv = gqa.linear(x, w.w_qkv.cuda())
    y = gqa.linear(x, w.w_o.cuda(), out_dtype=torch.float32)
    torch.cuda.synchronize()
    gqa.check_device_status()
    M = w.x.shape[0]
    rng = np.random.default_rng(503)
    rows = np.unique(np.concatenate([[0, 127, 128, 255, 256, M // 2, M - 129, M - 128, M - 1],
                                     rng.integers(0, M, 61)]))
    xb = bits(w.x)[rows]
    assert_close(qkv.float().cpu().numpy()[rows], oracle.linear(xb, bits(w.w_qkv)), "QKV projection rows")
    assert_close(y.cpu().numpy()[rows], oracle.linear(xb, bits(w.w_o)), "output projection rows")
