"""GPU parity of chunked prefill on a paged KV cache (gqa_attn_prefill_chunk_paged) through
the C ABI: outputs against the fp64 oracle (max-abs 2e-2, mean-abs 2e-3 per element) and
bit for bit against the contiguous-cache chunk on the same rows; the chunk's k-hat and v
land in the pages the table names, bit for bit as the contiguous chunk writes them, and
every other page row is untouched.  Page sizes 16 to 512 (384 included), pages handed out
in a shuffled order, prefixes that end inside a page."""
import numpy as np
import pytest
import torch

from oracle import oracle
from grouped_query_causal_b200 import synthetic
from tests.gpu_helpers import assert_close, bits
from tests.test_prefill_ragged_gpu import _cache_with_prefix, _packed

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gqa():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for the gpu tests")
    from grouped_query_causal_b200 import binding
    binding.load()
    return binding


def _page_rows(table, page_size, b, lo, hi):
    """(page, row-in-page) of rows lo .. hi-1 of sequence b."""
    r = np.arange(lo, hi)
    return table[b, r // page_size].astype(np.int64), r % page_size


def _paged_chunk_case(gqa, prefix, chunk, H, Hkv, page_size, seed, rope_kw=None):
    rope_kw = rope_kw or {}
    q, k, v, _, cu, wq, wk, theta, eps = _packed(chunk, H, Hkv, seed)
    pos = torch.cat([torch.arange(p, p + c, dtype=torch.int32) for p, c in zip(prefix, chunk)])
    kc, vc, offs = _cache_with_prefix(prefix, chunk, Hkv, wk, theta, eps, rope_kw, seed + 1)
    caps = [p + c for p, c in zip(prefix, chunk)]
    pc = synthetic.page_cache(kc, vc, offs, caps, page_size, seed=seed + 2)
    pl = torch.tensor(prefix, dtype=torch.int32)
    rope = gqa.RopeConfig.make(theta=theta, **rope_kw)
    dev = [t.cuda() for t in (q, k, v, pos, cu)]
    kp, vp = pc.k_pages.cuda(), pc.v_pages.cuda()
    out = gqa.prefill_chunk_paged(*dev, kp, vp, pc.page_table.cuda(), pl.cuda(), wq.cuda(), wk.cuda(),
                                  max_chunk_len=max(chunk), eps=eps, rope=rope)
    kcd, vcd = kc.cuda(), vc.cuda()
    flat = gqa.prefill_chunk(*dev, kcd, vcd, offs.cuda(), pl.cuda(), wq.cuda(), wk.cuda(), max_chunk_len=max(chunk),
                             eps=eps, rope=rope)
    torch.cuda.synchronize()
    gqa.check_device_status()
    got, kp, vp, kcd, vcd = out.cpu(), kp.cpu(), vp.cpu(), kcd.cpu(), vcd.cpu()
    what = f"P={prefix} C={chunk} H{H} Hkv{Hkv} page {page_size} {rope_kw}"
    assert torch.equal(got, flat.cpu()), "paged and contiguous chunk differ: " + what
    table = pc.page_table.numpy()
    ro = oracle.Rope(theta=theta, **rope_kw)
    written = torch.zeros(kp.shape[0], kp.shape[1], dtype=torch.bool)
    for b, (p, c) in enumerate(zip(prefix, chunk)):
        lo, hi = int(cu[b]), int(cu[b + 1])
        ref, _ = oracle.prefill_chunk_paged_ex(
            bits(q[lo:hi]).reshape(1, c, H, 128), bits(k[lo:hi]).reshape(1, c, Hkv, 128),
            bits(v[lo:hi]).reshape(1, c, Hkv, 128), bits(pc.k_pages), bits(pc.v_pages), table[b:b + 1], page_size,
            np.array([p], np.int32), pos[lo:hi].numpy().reshape(1, c), wq.numpy(), wk.numpy(), ro, eps)
        assert_close(got[lo:hi].numpy(), ref[0], f"sequence {b}: " + what)
        pg, r = _page_rows(table, page_size, b, p, p + c)
        o = int(offs[b])
        assert torch.equal(kp[pg, r], kcd[o + p:o + p + c]), f"k-hat rows of sequence {b}: " + what
        assert torch.equal(vp[pg, r], vcd[o + p:o + p + c]), f"value rows of sequence {b}: " + what
        written[pg, r] = True
    assert torch.equal(kp[~written], pc.k_pages[~written]) and torch.equal(vp[~written], pc.v_pages[~written])


@pytest.mark.parametrize("prefix,chunk,H,Hkv,page_size", [
    ([256], [256], 8, 2, 128),                   # prefix and chunk whole tiles and pages
    ([200, 0], [300, 77], 16, 4, 16),            # prefix ends inside a page; a sequence without prefix
    ([1000, 1, 37], [77, 257, 5], 32, 8, 32),
    ([1000, 1, 37], [77, 257, 5], 32, 8, 256),   # a 128-key tile inside a page
    ([128, 4096], [1, 128], 12, 4, 64),          # one-token chunk; long prefix; odd heads per group
    ([300], [300], 16, 1, 512),                  # MQA; one page holds the sequence
    ([2000, 77], [700, 129], 16, 4, 384),        # pages of three tiles
])
def test_paged_chunk_against_oracle(gqa, prefix, chunk, H, Hkv, page_size):
    _paged_chunk_case(gqa, prefix, chunk, H, Hkv, page_size, seed=400 + page_size)


def _pages_in_order(kc, vc, offs, caps, ps, order):
    """Cache rows cut into pages of ps rows, handed out in the given order of page ids (a
    permutation of the pool), sequence after sequence; two spare pages at the end."""
    need = [(c + ps - 1) // ps for c in caps]
    npg = sum(need) + 2
    ids = list(order) + [i for i in range(npg) if i not in set(order)]
    Hkv, D = kc.shape[1], kc.shape[2]
    kp = torch.zeros(npg, ps, Hkv, D, dtype=kc.dtype)
    vp = torch.zeros_like(kp)
    table = torch.full((len(caps), max(need)), -1, dtype=torch.int32)
    nxt = 0
    for b, c in enumerate(caps):
        o = int(offs[b])
        for j in range(need[b]):
            pid = ids[nxt]
            nxt += 1
            table[b, j] = pid
            n = min(ps, c - j * ps)
            kp[pid, :n] = kc[o + j * ps:o + j * ps + n]
            vp[pid, :n] = vc[o + j * ps:o + j * ps + n]
    return kp, vp, table


@pytest.mark.parametrize("ps,layout", [(16, "in_order"), (32, "in_order"), (64, "in_order"), (16, "runs"),
                                       (32, "runs"), (16, "descending")])
def test_paged_chunk_page_layouts(gqa, ps, layout):
    """Page layouts other than a random shuffle: pages in order, runs of 8 consecutive pages
    in shuffled order (tiles straddle runs at some prefixes and not at others), and pages in
    descending order.  Outputs bit for bit equal to the contiguous chunk's and within
    tolerance of the oracle; the chunk's rows land in the right pages."""
    prefix, chunk, H, Hkv = [500, 0, 1000], [300, 129, 77], 16, 4
    q, k, v, _, cu, wq, wk, theta, eps = _packed(chunk, H, Hkv, seed=520 + ps)
    pos = torch.cat([torch.arange(p, p + c, dtype=torch.int32) for p, c in zip(prefix, chunk)])
    kc, vc, offs = _cache_with_prefix(prefix, chunk, Hkv, wk, theta, eps, {}, seed=521 + ps)
    caps = [p + c for p, c in zip(prefix, chunk)]
    npg = sum((c + ps - 1) // ps for c in caps)
    if layout == "in_order":
        order = list(range(npg))
    elif layout == "descending":
        order = list(range(npg - 1, -1, -1))
    else:
        runs = [list(range(r, min(r + 8, npg))) for r in range(0, npg, 8)]
        rng = np.random.default_rng(522)
        order = [i for r in rng.permutation(len(runs)) for i in runs[r]]
    kp, vp, table = _pages_in_order(kc, vc, offs, caps, ps, order)
    pl = torch.tensor(prefix, dtype=torch.int32)
    rope = gqa.RopeConfig.make(theta=theta)
    dev = [t.cuda() for t in (q, k, v, pos, cu)]
    kpd, vpd = kp.cuda(), vp.cuda()
    out = gqa.prefill_chunk_paged(*dev, kpd, vpd, table.cuda(), pl.cuda(), wq.cuda(), wk.cuda(),
                                  max_chunk_len=max(chunk), eps=eps, rope=rope)
    kcd, vcd = kc.cuda(), vc.cuda()
    flat = gqa.prefill_chunk(*dev, kcd, vcd, offs.cuda(), pl.cuda(), wq.cuda(), wk.cuda(), max_chunk_len=max(chunk),
                             eps=eps, rope=rope)
    torch.cuda.synchronize()
    gqa.check_device_status()
    assert torch.equal(out.cpu(), flat.cpu()), f"paged ({layout}, {ps}-row pages) and contiguous chunk differ"
    kpd, vpd, kcd, vcd = kpd.cpu(), vpd.cpu(), kcd.cpu(), vcd.cpu()
    t = table.numpy()
    for b, (p, c) in enumerate(zip(prefix, chunk)):
        lo, hi = int(cu[b]), int(cu[b + 1])
        r = np.arange(p, p + c)
        pg = t[b, r // ps].astype(np.int64)
        o = int(offs[b])
        assert torch.equal(kpd[pg, r % ps], kcd[o + p:o + p + c]) and torch.equal(vpd[pg, r % ps], vcd[o + p:o + p + c])
        ref, _ = oracle.prefill_chunk_paged_ex(
            bits(q[lo:hi]).reshape(1, c, H, 128), bits(k[lo:hi]).reshape(1, c, Hkv, 128),
            bits(v[lo:hi]).reshape(1, c, Hkv, 128), bits(kp), bits(vp), t[b:b + 1], ps, np.array([p], np.int32),
            pos[lo:hi].numpy().reshape(1, c), wq.numpy(), wk.numpy(), oracle.Rope(theta=theta), eps)
        assert_close(out.cpu().numpy()[lo:hi], ref[0], f"{layout} {ps}-row pages, sequence {b}")


def test_paged_chunk_with_rope_variant(gqa):
    _paged_chunk_case(gqa, [333, 90], [200, 130], 16, 4, 32, seed=460,
                      rope_kw=dict(pairing="half", scaling="yarn", factor=4.0, original_max_position=256))


def test_paged_chunks_in_sequence_equal_one_prefill(gqa):
    """A prompt prefilled as three chunks into shuffled 64-row pages (prefix_len advanced by
    the caller between calls) gives the rows of one causal prefill over the prompt."""
    T, H, Hkv, ps = 700, 16, 4, 64
    inp = synthetic.prefill_inputs(1, T, H, Hkv, seed=470)
    q, k, v, pos = inp.q[0].cuda(), inp.k[0].cuda(), inp.v[0].cuda(), inp.pos[0].cuda()
    wq, wk = inp.wq.cuda(), inp.wk.cuda()
    need = (T + ps - 1) // ps
    order = torch.randperm(need + 4, generator=torch.Generator().manual_seed(471))
    table = order[:need].to(torch.int32).reshape(1, need).cuda()
    kp = torch.zeros(need + 4, ps, Hkv, 128, dtype=torch.bfloat16, device="cuda")
    vp = torch.zeros_like(kp)
    rope = gqa.RopeConfig.make(theta=inp.theta)
    outs = []
    for lo, hi in ((0, 250), (250, 256), (256, 700)):
        cu = torch.tensor([0, hi - lo], dtype=torch.int64, device="cuda")
        pl = torch.tensor([lo], dtype=torch.int32, device="cuda")
        outs.append(gqa.prefill_chunk_paged(q[lo:hi].contiguous(), k[lo:hi].contiguous(), v[lo:hi].contiguous(),
                                            pos[lo:hi].contiguous(), cu, kp, vp, table, pl, wq, wk,
                                            max_chunk_len=hi - lo, eps=inp.eps, rope=rope))
    torch.cuda.synchronize()
    gqa.check_device_status()
    got = torch.cat(outs).cpu().numpy()
    ref = oracle.prefill(bits(inp.q), bits(inp.k), bits(inp.v), inp.pos.numpy(), inp.wq.numpy(), inp.wk.numpy(),
                         inp.theta, inp.eps)[0]
    assert_close(got, ref, "three chunks through pages")


def test_paged_chunk_bad_page_id_is_a_device_input_error(gqa):
    """A page id out of range, for a cached row (read side) in one sequence and for a chunk
    row (write side) in another, writes no page memory through it and raises the device
    input status; the sequence with a clean table is still right."""
    prefix, chunk, H, Hkv, ps = [100, 40, 70], [60, 50, 90], 8, 2, 16
    q, k, v, _, cu, wq, wk, theta, eps = _packed(chunk, H, Hkv, seed=480)
    pos = torch.cat([torch.arange(p, p + c, dtype=torch.int32) for p, c in zip(prefix, chunk)])
    kc, vc, offs = _cache_with_prefix(prefix, chunk, Hkv, wk, theta, eps, {}, seed=481)
    pc = synthetic.page_cache(kc, vc, offs, [p + c for p, c in zip(prefix, chunk)], ps, seed=482)
    table = pc.page_table.clone()
    npages = pc.k_pages.shape[0]
    table[0, 2] = npages + 3      # rows 32..47 of sequence 0: cached keys
    table[1, 4] = -7              # rows 64..79 of sequence 1: chunk rows
    kp, vp = pc.k_pages.cuda(), pc.v_pages.cuda()
    out = gqa.prefill_chunk_paged(q.cuda(), k.cuda(), v.cuda(), pos.cuda(), cu.cuda(), kp, vp, table.cuda(),
                                  torch.tensor(prefix, dtype=torch.int32).cuda(), wq.cuda(), wk.cuda(),
                                  max_chunk_len=max(chunk), eps=eps, rope=gqa.RopeConfig.make(theta=theta))
    torch.cuda.synchronize()
    assert gqa.device_status() == -6
    assert gqa.device_status() == 0
    kp = kp.cpu()
    bad = pc.page_table[1, 4]     # the page the clean table gives those rows keeps its contents
    assert torch.equal(kp[bad], pc.k_pages[bad])
    lo, hi = int(cu[2]), int(cu[3])
    ref, _ = oracle.prefill_chunk_paged_ex(
        bits(q[lo:hi]).reshape(1, 90, H, 128), bits(k[lo:hi]).reshape(1, 90, Hkv, 128),
        bits(v[lo:hi]).reshape(1, 90, Hkv, 128), bits(pc.k_pages), bits(pc.v_pages), pc.page_table.numpy()[2:3], ps,
        np.array([70], np.int32), pos[lo:hi].numpy().reshape(1, 90), wq.numpy(), wk.numpy(), oracle.Rope(theta=theta),
        eps)
    assert_close(out.cpu().numpy()[lo:hi], ref[0], "the sequence with a clean table")
