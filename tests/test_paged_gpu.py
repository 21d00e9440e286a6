"""GPU parity of the paged-cache decode entry points (gqa_attn_decode_paged,
gqa_attn_decode_append_paged) against the fp64 oracle on the rows gathered through the
page table.  Tolerance: max-abs 2e-2, mean-abs 2e-3 per element."""
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


@pytest.mark.parametrize("page_size", [16, 64, 256])
@pytest.mark.parametrize("H,Hkv", [(32, 8), (16, 16), (16, 1)])
def test_paged_decode(gqa, page_size, H, Hkv):
    seqlens = [1, 15, 16, 17, 1023, 1024, 1025, 2500]
    d = synthetic.decode_inputs(len(seqlens), H, Hkv, seed=70, seqlens=seqlens)
    pc = synthetic.page_cache(d.k_cache, d.v_cache, d.offsets, seqlens, page_size, seed=71)
    out = gqa.decode_paged(d.q.cuda(), pc.k_pages.cuda(), pc.v_pages.cuda(), pc.page_table.cuda(), d.seqlens.cuda(),
                           d.wq.cuda(), max_len=d.max_len, eps=d.eps, rope=gqa.RopeConfig.make(theta=d.theta))
    torch.cuda.synchronize()
    gqa.check_device_status()
    ref = oracle.decode(bits(d.q), bits(d.k_cache), bits(d.v_cache), d.offsets.numpy(), d.seqlens.numpy(), None,
                        d.wq.numpy(), d.theta, d.eps)
    assert_close(out.cpu().numpy(), ref, f"paged decode P={page_size} H={H} Hkv={Hkv}")


def test_paged_decode_with_rope_variant(gqa):
    seqlens = [300, 2049]
    d = synthetic.decode_inputs(2, 16, 4, seed=72, seqlens=seqlens)
    pc = synthetic.page_cache(d.k_cache, d.v_cache, d.offsets, seqlens, 32, seed=73)
    kw = dict(pairing="half", scaling="yarn", factor=8.0, original_max_position=1024)
    qpos = torch.tensor([40000, 2049], dtype=torch.int32)
    out = gqa.decode_paged(d.q.cuda(), pc.k_pages.cuda(), pc.v_pages.cuda(), pc.page_table.cuda(), d.seqlens.cuda(),
                           d.wq.cuda(), max_len=d.max_len, q_pos=qpos.cuda(), eps=d.eps, rope=gqa.RopeConfig.make(**kw))
    torch.cuda.synchronize()
    gqa.check_device_status()
    ref = oracle.decode_paged_ex(bits(d.q), bits(pc.k_pages), bits(pc.v_pages), pc.page_table.numpy(), 32,
                                 d.seqlens.numpy(), qpos.numpy(), d.wq.numpy(), oracle.Rope(**kw), d.eps)
    assert_close(out.cpu().numpy(), ref, "paged decode, YaRN + rotate-half")


@pytest.mark.parametrize("page_size", [16, 128])
def test_paged_append(gqa, page_size):
    seqlens = [0, 15, 16, 127, 128, 1500]
    a = synthetic.decode_append_inputs(len(seqlens), 16, 4, seed=74, seqlens=seqlens, spare=1)
    caps = [s + 1 for s in seqlens]
    pc = synthetic.page_cache(a.k_cache, a.v_cache, a.offsets, caps, page_size, seed=75)
    kp, vp = pc.k_pages.cuda(), pc.v_pages.cuda()
    out = gqa.decode_append_paged(a.q.cuda(), a.k_new.cuda(), a.v_new.cuda(), kp, vp, pc.page_table.cuda(),
                                  a.seqlens.cuda(), a.wq.cuda(), a.wk.cuda(), max_len=a.max_len, eps=a.eps,
                                  rope=gqa.RopeConfig.make(theta=a.theta))
    torch.cuda.synchronize()
    gqa.check_device_status()
    ref, khat = oracle.decode_append_paged_ex(bits(a.q), bits(a.k_new), bits(a.v_new), bits(pc.k_pages),
                                              bits(pc.v_pages), pc.page_table.numpy(), page_size, a.seqlens.numpy(),
                                              None, a.wq.numpy(), a.wk.numpy(), oracle.Rope(theta=a.theta), a.eps)
    assert_close(out.cpu().numpy(), ref, f"paged append P={page_size}")
    kp, vp = kp.cpu(), vp.cpu()
    written = torch.zeros(kp.shape[:2], dtype=torch.bool)
    for b, n in enumerate(seqlens):
        pid, slot = int(pc.page_table[b, n // page_size]), n % page_size
        written[pid, slot] = True
        got = kp[pid, slot].double().numpy()
        assert (np.abs(got - khat[b]) <= 2.0 ** -8 * np.abs(khat[b]) + 1e-5).all(), f"k-hat row of sequence {b}"
        assert torch.equal(vp[pid, slot], a.v_new[b])
    assert torch.equal(kp[~written], pc.k_pages[~written]) and torch.equal(vp[~written], pc.v_pages[~written])


def test_bad_page_id_gives_nan_and_status(gqa):
    seqlens = [100, 200, 300]
    d = synthetic.decode_inputs(3, 8, 2, seed=76, seqlens=seqlens)
    pc = synthetic.page_cache(d.k_cache, d.v_cache, d.offsets, seqlens, 16, seed=77)
    table = pc.page_table.clone()
    table[1, 3] = pc.k_pages.shape[0] + 5        # sequence 1 points past the last page
    out = gqa.decode_paged(d.q.cuda(), pc.k_pages.cuda(), pc.v_pages.cuda(), table.cuda(), d.seqlens.cuda(),
                           d.wq.cuda(), max_len=d.max_len, eps=d.eps, rope=gqa.RopeConfig.make(theta=d.theta))
    torch.cuda.synchronize()
    assert gqa.device_status() == -6
    got = out.cpu().numpy()
    assert np.isnan(got[1]).all()
    ref = oracle.decode(bits(d.q), bits(d.k_cache), bits(d.v_cache), d.offsets.numpy(), d.seqlens.numpy(), None,
                        d.wq.numpy(), d.theta, d.eps)
    assert_close(got[[0, 2]], ref[[0, 2]], "sequences with valid pages")


def test_paged_batched_decode_config(gqa):
    """The batched decode workload (64 sequences, 1K-32K cached rows, H=32, Hkv=8) in
    shuffled 64-row pages, the paged launch the benchmark times: every sequence and head
    against the oracle on the contiguous rows (paged and contiguous caches give the same
    oracle result, exactly)."""
    d = synthetic.make("batched_decode")
    lens = d.seqlens.tolist()
    pc = synthetic.page_cache(d.k_cache, d.v_cache, d.offsets, lens, 64, seed=78)
    out = gqa.decode_paged(d.q.cuda(), pc.k_pages.cuda(), pc.v_pages.cuda(), pc.page_table.cuda(), d.seqlens.cuda(),
                           d.wq.cuda(), max_len=d.max_len, eps=d.eps, rope=gqa.RopeConfig.make(theta=d.theta))
    torch.cuda.synchronize()
    gqa.check_device_status()
    ref = oracle.decode(bits(d.q), bits(d.k_cache), bits(d.v_cache), d.offsets.numpy(), d.seqlens.numpy(), None,
                        d.wq.numpy(), d.theta, d.eps)
    assert_close(out.cpu().numpy(), ref, "paged batched decode, all 64 sequences")
