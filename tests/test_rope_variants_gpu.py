"""GPU parity of the RoPE variants (rotate-half pairing; linear, NTK-aware and YaRN
frequency scaling with YaRN's logit temperature) through the _ex entry points, against
the fp64 oracle.  Tolerance as elsewhere: max-abs 2e-2, mean-abs 2e-3 per element."""
import numpy as np
import pytest
import torch

from oracle import oracle
from grouped_query_causal_b200 import synthetic
from tests.gpu_helpers import assert_close, bits, to_dev

pytestmark = pytest.mark.gpu

VARIANTS = {
    "half": dict(pairing="half"),
    "linear4": dict(scaling="linear", factor=4.0),
    "ntk8": dict(scaling="ntk", factor=8.0),
    "yarn16": dict(scaling="yarn", factor=16.0, original_max_position=4096),
    "yarn16_half": dict(pairing="half", scaling="yarn", factor=16.0, original_max_position=2048, beta_fast=16.0,
                        beta_slow=2.0),
}


@pytest.fixture(scope="module")
def gqa():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for the gpu tests")
    from grouped_query_causal_b200 import binding
    binding.load()
    return binding


def _cfgs(gqa, name, theta=1.0e6):
    kw = VARIANTS[name]
    return gqa.RopeConfig.make(theta=theta, **kw), oracle.Rope(theta=theta, **kw)


def _prefill_inputs(seed, T=300):
    inp = synthetic.prefill_inputs(1, T, 8, 2, seed=seed)
    rng = np.random.default_rng(seed)
    # positions spread over a long context (the mask stays on the token index)
    inp.pos = torch.from_numpy(np.sort(rng.integers(0, 60000, (1, T))).astype(np.int32))
    return inp


@pytest.mark.parametrize("name", list(VARIANTS))
def test_prefill_variants(gqa, name):
    rc, ro = _cfgs(gqa, name)
    inp = _prefill_inputs(50)
    d = to_dev(inp)
    out = gqa.prefill(d["q"], d["k"], d["v"], d["pos"], d["qnorm_w"], d["knorm_w"], eps=inp.eps, rope=rc)
    torch.cuda.synchronize()
    gqa.check_device_status()
    B, T, H = 1, inp.q.shape[1], inp.q.shape[2]
    rows = np.array([(0, h, i) for h in range(H) for i in range(T)], np.int64)
    ref = oracle.prefill_rows_ex(bits(inp.q), bits(inp.k), bits(inp.v), inp.pos.numpy(), inp.wq.numpy(),
                                 inp.wk.numpy(), ro, inp.eps, rows).reshape(H, T, 128).transpose(1, 0, 2)
    assert_close(out.cpu().numpy()[0], ref, f"prefill {name}")
    # the two stages with and without the cos/sin table give the one-call result
    tab = torch.empty(gqa.rope_table_numel(T), dtype=torch.float32, device="cuda")
    kh = gqa.k_norm_rope(d["k"], d["pos"], d["knorm_w"], eps=inp.eps, rope_cs=tab, rope=rc)
    o2 = gqa.prefill_khat(d["q"], kh, d["v"], d["pos"], d["qnorm_w"], eps=inp.eps, rope_cs=tab, rope=rc)
    o3 = gqa.prefill_khat(d["q"], kh, d["v"], d["pos"], d["qnorm_w"], eps=inp.eps, rope=rc)
    torch.cuda.synchronize()
    gqa.check_device_status()
    assert torch.equal(o2, out)
    assert_close(o3.cpu().numpy()[0], ref, f"prefill {name} without the table")
    # k-hat itself against the oracle's, within bf16 rounding
    kref = oracle.qk_transform_ex(bits(inp.k)[0], inp.pos.numpy()[0], inp.wk.numpy(), ro, inp.eps)
    got = kh[0].double().cpu().numpy()
    assert (np.abs(got - kref) <= 2.0 ** -8 * np.abs(kref) + 1e-5).all()


def test_default_config_is_the_plain_entry_point(gqa):
    inp = _prefill_inputs(51, T=200)
    d = to_dev(inp)
    a = gqa.prefill(d["q"], d["k"], d["v"], d["pos"], d["qnorm_w"], d["knorm_w"], theta=inp.theta, eps=inp.eps)
    b = gqa.prefill(d["q"], d["k"], d["v"], d["pos"], d["qnorm_w"], d["knorm_w"], eps=inp.eps,
                    rope=gqa.RopeConfig.make(theta=inp.theta))
    dec = synthetic.decode_inputs(3, 8, 2, seed=52, seqlens=[1, 700, 1500])
    args = (dec.q.cuda(), dec.k_cache.cuda(), dec.v_cache.cuda(), dec.offsets.cuda(), dec.seqlens.cuda(), dec.wq.cuda())
    c = gqa.decode(*args, max_len=dec.max_len, theta=dec.theta, eps=dec.eps)
    e = gqa.decode(*args, max_len=dec.max_len, eps=dec.eps, rope=gqa.RopeConfig.make(theta=dec.theta))
    torch.cuda.synchronize()
    gqa.check_device_status()
    assert torch.equal(a, b) and torch.equal(c, e)


@pytest.mark.parametrize("name", list(VARIANTS))
def test_decode_variants(gqa, name):
    rc, ro = _cfgs(gqa, name)
    seqlens = [1, 900, 2049, 37]
    dec = synthetic.decode_inputs(len(seqlens), 16, 4, seed=53, seqlens=seqlens)
    qpos = np.array([5, 40000, 2049, 65000], np.int32)
    out = gqa.decode(dec.q.cuda(), dec.k_cache.cuda(), dec.v_cache.cuda(), dec.offsets.cuda(), dec.seqlens.cuda(),
                     dec.wq.cuda(), max_len=dec.max_len, q_pos=torch.from_numpy(qpos).cuda(), eps=dec.eps, rope=rc)
    torch.cuda.synchronize()
    gqa.check_device_status()
    ref = oracle.decode_ex(bits(dec.q), bits(dec.k_cache), bits(dec.v_cache), dec.offsets.numpy(),
                           dec.seqlens.numpy(), qpos, dec.wq.numpy(), ro, dec.eps)
    assert_close(out.cpu().numpy(), ref, f"decode {name}")


@pytest.mark.parametrize("name", list(VARIANTS))
def test_decode_append_variants(gqa, name):
    rc, ro = _cfgs(gqa, name)
    a = synthetic.decode_append_inputs(4, 16, 4, seed=54, seqlens=[0, 3, 1023, 1500], spare=1)
    kc, vc = a.k_cache.cuda(), a.v_cache.cuda()
    out = gqa.decode_append(a.q.cuda(), a.k_new.cuda(), a.v_new.cuda(), kc, vc, a.offsets.cuda(), a.seqlens.cuda(),
                            a.wq.cuda(), a.wk.cuda(), max_len=a.max_len, eps=a.eps, rope=rc)
    torch.cuda.synchronize()
    gqa.check_device_status()
    ref, khat = oracle.decode_append_ex(bits(a.q), bits(a.k_new), bits(a.v_new), bits(a.k_cache), bits(a.v_cache),
                                        a.offsets.numpy(), a.seqlens.numpy(), None, a.wq.numpy(), a.wk.numpy(), ro,
                                        a.eps)
    assert_close(out.cpu().numpy(), ref, f"decode_append {name}")
    kc = kc.cpu()
    for b in range(4):
        r = int(a.offsets[b]) + int(a.seqlens[b])
        got = kc[r].double().numpy()
        assert (np.abs(got - khat[b]) <= 2.0 ** -8 * np.abs(khat[b]) + 1e-5).all(), f"k-hat row {b}"
