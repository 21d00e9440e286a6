"""GPU parity of gqa_attn_decode against the fp64 oracle (through the C ABI via the
ctypes binding).  Tolerance: max-abs 2e-2 and mean-abs 2e-3 per element."""
import numpy as np
import pytest
import torch

from oracle import oracle
from grouped_query_causal_b200 import synthetic
from tests.gpu_helpers import assert_close, bits, decode_to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gqa():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for the gpu tests")
    from grouped_query_causal_b200 import binding
    binding.load()
    return binding


def _run(gqa, inp, q_pos=None, max_len=None):
    d = decode_to_dev(inp)
    qp = None if q_pos is None else torch.as_tensor(q_pos, dtype=torch.int32).cuda()
    out = gqa.decode(d["q"], d["k_cache"], d["v_cache"], d["cache_offsets"], d["seqlens"], d["qnorm_w"],
                     max_len=max_len or inp.max_len, q_pos=qp, theta=d["theta"], eps=d["eps"])
    torch.cuda.synchronize()
    return out.cpu().numpy()


def _oracle(inp, idx=None, q_pos=None):
    """Oracle outputs of the sequences idx (all by default)."""
    B = inp.q.shape[0]
    idx = np.arange(B) if idx is None else np.asarray(idx)
    offs = inp.offsets.numpy()
    sl = inp.seqlens.numpy()
    qp = None if q_pos is None else np.asarray(q_pos, np.int32)[idx]
    return oracle.decode(bits(inp.q)[idx], bits(inp.k_cache), bits(inp.v_cache),
                         np.append(offs[idx], offs[-1]), sl[idx], qp, inp.wq.numpy(), inp.theta, inp.eps)


def test_batched_decode_config(gqa):
    """64 sequences, len ~ U[1024, 32768], H=32, Hkv=8, query at position len: the
    launch the benchmark times, every sequence and every head against the oracle."""
    inp = synthetic.make("batched_decode")
    got = _run(gqa, inp)
    gqa.check_device_status()
    assert np.isfinite(got).all()
    assert_close(got, _oracle(inp), "batched_decode, all 64 sequences")


@pytest.mark.parametrize("H,Hkv", [(16, 16), (16, 8), (16, 4), (16, 1), (12, 4), (10, 2), (32, 8)])
def test_group_sizes(gqa, H, Hkv):
    # chunk edges (1024-key chunks, 16-row load batches) and ragged tails
    seqlens = [1, 511, 512, 513, 1500, 37, 1023, 1024, 1025, 2049, 16, 17]
    inp = synthetic.decode_inputs(len(seqlens), H, Hkv, seed=H * 100 + Hkv, seqlens=seqlens)
    got = _run(gqa, inp)
    gqa.check_device_status()
    assert_close(got, _oracle(inp), f"H{H} Hkv{Hkv}")


def test_explicit_query_positions_and_spare_capacity(gqa):
    """q_pos given explicitly; sequences own more rows than they use (capacity > len)."""
    B, H, Hkv = 4, 8, 2
    cap = [700, 1100, 64, 2048]
    lens = [650, 1024, 1, 2000]
    full = synthetic.decode_inputs(B, H, Hkv, seed=9, seqlens=cap)
    inp = synthetic.DecodeInputs(full.q, full.k_cache, full.v_cache, full.offsets,
                                 torch.tensor(lens, dtype=torch.int32), full.wq)
    q_pos = [5, 30000, 0, 2000]
    got = _run(gqa, inp, q_pos=q_pos, max_len=2048)
    gqa.check_device_status()
    assert_close(got, _oracle(inp, q_pos=q_pos), "q_pos / capacity")


def test_bad_device_lengths_give_nan_and_status(gqa):
    B, H, Hkv = 3, 8, 2
    inp = synthetic.decode_inputs(B, H, Hkv, seed=10, seqlens=[100, 200, 300])
    bad = synthetic.DecodeInputs(inp.q, inp.k_cache, inp.v_cache, inp.offsets,
                                 torch.tensor([100, 0, 301], dtype=torch.int32), inp.wq)
    got = _run(gqa, bad, max_len=512)
    st = gqa.device_status()
    assert st == -6, st  # GQA_ERR_DEVICE_INPUT
    assert np.isnan(got[1]).all() and np.isnan(got[2]).all()
    assert_close(got[0], _oracle(inp, [0])[0], "valid sequence beside bad ones")
    assert gqa.device_status() == 0   # the word was cleared


def test_deterministic(gqa):
    inp = synthetic.decode_inputs(5, 16, 4, seed=3, seqlens=[3000, 10, 777, 4096, 1])
    a = _run(gqa, inp)
    b = _run(gqa, inp)
    np.testing.assert_array_equal(a, b)
