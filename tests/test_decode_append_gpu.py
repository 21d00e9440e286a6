"""GPU parity of gqa_attn_decode_append (the decode step that writes the new token's
k-hat and v into the cache, then attends) against the fp64 oracle, through the C ABI via
the ctypes binding.  Output tolerance: max-abs 2e-2, mean-abs 2e-3 per element; the
written key row is within bf16 rounding of the oracle's k-hat, the written value row and
every other cache row are bit-exact."""
import numpy as np
import pytest
import torch

from oracle import oracle
from grouped_query_causal_b200 import synthetic
from tests.gpu_helpers import assert_close, bits, oracle_prefill_args, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gqa():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for the gpu tests")
    from grouped_query_causal_b200 import binding
    binding.load()
    return binding


def _run(gqa, inp, q_pos=None, max_len=None):
    """One append step on the device; returns (out, k_cache, v_cache) on the host."""
    kc, vc = inp.k_cache.cuda(), inp.v_cache.cuda()
    qp = None if q_pos is None else torch.as_tensor(q_pos, dtype=torch.int32).cuda()
    out = gqa.decode_append(inp.q.cuda(), inp.k_new.cuda(), inp.v_new.cuda(), kc, vc, inp.offsets.cuda(),
                            inp.seqlens.cuda(), inp.wq.cuda(), inp.wk.cuda(), max_len=max_len or inp.max_len,
                            q_pos=qp, theta=inp.theta, eps=inp.eps)
    torch.cuda.synchronize()
    return out.cpu().numpy(), kc.cpu(), vc.cpu()


def _oracle(inp, idx=None, q_pos=None):
    B = inp.q.shape[0]
    idx = np.arange(B) if idx is None else np.asarray(idx)
    offs = inp.offsets.numpy()
    qp = None if q_pos is None else np.asarray(q_pos, np.int32)[idx]
    return oracle.decode_append(bits(inp.q)[idx], bits(inp.k_new)[idx], bits(inp.v_new)[idx], bits(inp.k_cache),
                                bits(inp.v_cache), np.append(offs[idx], offs[-1]), inp.seqlens.numpy()[idx], qp,
                                inp.wq.numpy(), inp.wk.numpy(), inp.theta, inp.eps)


def _check_cache(inp, kc, vc, khat_ref, idx=None, q_pos=None):
    """Row seqlens[b] of each sequence holds the new k-hat (bf16-rounded) and v_new; every
    other row is unchanged."""
    B = inp.q.shape[0]
    idx = range(B) if idx is None else idx
    written = np.zeros(inp.k_cache.shape[0], bool)
    for n, b in enumerate(idx):
        r = int(inp.offsets[b]) + int(inp.seqlens[b])
        written[r] = True
        got_k = kc[r].double().numpy()
        ref_k = khat_ref[n]
        assert (np.abs(got_k - ref_k) <= 2.0 ** -8 * np.abs(ref_k) + 1e-5).all(), f"k-hat row of sequence {b}"
        assert torch.equal(vc[r], inp.v_new[b]), f"value row of sequence {b}"
    keep = torch.from_numpy(~written)
    assert torch.equal(kc[keep], inp.k_cache[keep]) and torch.equal(vc[keep], inp.v_cache[keep])


@pytest.mark.parametrize("H,Hkv", [(16, 8), (16, 1), (12, 4), (32, 8), (16, 16)])
def test_ragged_lengths(gqa, H, Hkv):
    """Lengths 0 (empty cache: the token attends only to itself), 1, chunk edges and a
    ragged tail; two spare rows per sequence."""
    seqlens = [0, 1, 511, 512, 1023, 1024, 1500, 37, 2047]
    inp = synthetic.decode_append_inputs(len(seqlens), H, Hkv, seed=31, seqlens=seqlens, spare=2)
    out, kc, vc = _run(gqa, inp)
    gqa.check_device_status()
    ref, khat = _oracle(inp)
    assert_close(out, ref, f"decode_append H={H} Hkv={Hkv}")
    _check_cache(inp, kc, vc, khat)


def test_explicit_positions(gqa):
    seqlens = [5, 700, 64]
    inp = synthetic.decode_append_inputs(3, 16, 4, seed=32, seqlens=seqlens, spare=1)
    qpos = [100000, 3, 70000]
    out, kc, vc = _run(gqa, inp, q_pos=qpos)
    gqa.check_device_status()
    ref, khat = _oracle(inp, q_pos=qpos)
    assert_close(out, ref, "decode_append q_pos")
    _check_cache(inp, kc, vc, khat)


def test_batched_decode_append_config(gqa):
    """64 sequences with 1023..32767 cached rows, H=32, Hkv=8: the append-step workload
    the benchmark times.  Every sequence's output and every cache row checked."""
    inp = synthetic.make("batched_decode_append")
    out, kc, vc = _run(gqa, inp)
    gqa.check_device_status()
    assert np.isfinite(out).all()
    ref, kh = _oracle(inp)
    assert_close(out, ref, "batched_decode_append, all 64 sequences")
    # the written keys: k-hat of every new key at its position (the sequence length)
    _check_cache(inp, kc, vc, kh)


def test_prefill_then_append_steps_continue_the_sequence(gqa):
    """Prefill T0 tokens (k-hat from gqa_attn_k_norm_rope into a cache with room for three
    more), then three append steps: step s must equal row T0 + s of causal attention over
    the whole T0 + 3 tokens."""
    B, T0, H, Hkv, steps = 2, 300, 16, 4, 3
    T = T0 + steps
    inp = synthetic.prefill_inputs(B, T, H, Hkv, seed=33)
    d = to_dev(inp)
    kh = gqa.k_norm_rope(d["k"][:, :T0].contiguous(), d["pos"][:, :T0].contiguous(), d["knorm_w"],
                         theta=inp.theta, eps=inp.eps)
    kc = torch.zeros(B, T, Hkv, 128, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    kc[:, :T0] = kh
    vc[:, :T0] = d["v"][:, :T0]
    kc, vc = kc.reshape(B * T, Hkv, 128), vc.reshape(B * T, Hkv, 128)
    offsets = (torch.arange(B + 1, dtype=torch.int64) * T).cuda()
    seqlens = torch.full((B,), T0, dtype=torch.int32, device="cuda")
    for s in range(steps):
        t = T0 + s
        out = gqa.decode_append(d["q"][:, t].contiguous(), d["k"][:, t].contiguous(), d["v"][:, t].contiguous(),
                                kc, vc, offsets, seqlens, d["qnorm_w"], d["knorm_w"], max_len=T,
                                theta=inp.theta, eps=inp.eps)
        torch.cuda.synchronize()
        gqa.check_device_status()
        rows = np.array([(b, hq, t) for b in range(B) for hq in range(H)], np.int64)
        ref = oracle.prefill_rows(*oracle_prefill_args(inp), rows).reshape(B, H, 128)
        assert_close(out.cpu().numpy(), ref, f"append step {s}")
        seqlens += 1


def test_full_cache_is_rejected_on_the_device(gqa):
    """A sequence with no free row is not written, gets NaN output and raises the device
    input status; the other sequences are unaffected."""
    seqlens = [10, 20, 30]
    inp = synthetic.decode_append_inputs(3, 8, 2, seed=34, seqlens=seqlens, spare=1)
    sl_bad = inp.seqlens.clone()
    sl_bad[1] = 21                        # capacity of sequence 1 is 21 rows: no room left
    bad = synthetic.DecodeAppendInputs(inp.q, inp.k_new, inp.v_new, inp.k_cache, inp.v_cache, inp.offsets, sl_bad,
                                       inp.wq, inp.wk)
    out, kc, vc = _run(gqa, bad, max_len=32)
    assert gqa.device_status() == -6
    assert np.isnan(out[1]).all()
    ref, khat = _oracle(inp, [0, 2])
    assert_close(out[[0, 2]], ref, "other sequences")
    _check_cache(inp, kc, vc, khat, idx=[0, 2])
