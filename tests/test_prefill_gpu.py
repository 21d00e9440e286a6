"""GPU parity of gqa_attn_prefill against the fp64 oracle (called through the C ABI
via the ctypes binding).  Tolerance: max-abs 2e-2 and mean-abs 2e-3 per element."""
import numpy as np
import pytest
import torch

from oracle import oracle
from grouped_query_causal_b200 import synthetic
from tests.gpu_helpers import (assert_close, bits as bits_of, oracle_prefill_args, strided_rows, to_dev)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gqa():
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for the gpu tests")
    from grouped_query_causal_b200 import binding
    binding.load()
    return binding


def _run(gqa, inp):
    d = to_dev(inp)
    out = gqa.prefill(d["q"], d["k"], d["v"], d["pos"], d["qnorm_w"], d["knorm_w"], d["theta"], d["eps"])
    torch.cuda.synchronize()
    gqa.check_device_status()
    return out.cpu().numpy()


def test_prefill_correctness_config(gqa):
    """B=1, T=128, H=16, Hkv=8 (one query block, one diagonal tile) in full."""
    inp = synthetic.make("prefill_correctness")
    got = _run(gqa, inp)
    ref = oracle.prefill(*oracle_prefill_args(inp))
    assert_close(got, ref, "prefill_correctness")


@pytest.mark.parametrize("name", ["gqa_sweep_mha", "gqa_sweep_hkv8", "gqa_sweep_hkv4", "gqa_sweep_mqa"])
def test_gqa_degeneracy_sweep(gqa, name):
    """B=2, T=512, H=16 with Hkv in {16 (MHA), 8, 4, 1 (MQA)}, every output element."""
    inp = synthetic.make(name)
    got = _run(gqa, inp)
    ref = oracle.prefill(*oracle_prefill_args(inp))
    assert_close(got, ref, name)


@pytest.mark.parametrize("B,T,H,Hkv", [(1, 1, 2, 1), (2, 7, 4, 2), (1, 129, 6, 2), (2, 200, 3, 1),
                                       (1, 383, 8, 8), (3, 130, 10, 2), (1, 257, 16, 2)])
def test_ragged_and_odd_groups(gqa, B, T, H, Hkv):
    """Ragged T (partial last query/key tile), odd heads per group, single token."""
    inp = synthetic.prefill_inputs(B, T, H, Hkv, seed=B * 1000 + T)
    got = _run(gqa, inp)
    ref = oracle.prefill(*oracle_prefill_args(inp))
    assert_close(got, ref, f"B{B} T{T} H{H} Hkv{Hkv}")


def test_positions_drive_rope_only(gqa):
    """Arbitrary (non-contiguous, large) positions: RoPE uses pos, the mask uses the index."""
    inp = synthetic.prefill_inputs(2, 160, 8, 2, seed=77)
    g = torch.Generator().manual_seed(78)
    inp.pos = torch.randint(0, 32768, (2, 160), generator=g, dtype=torch.int32)
    got = _run(gqa, inp)
    ref = oracle.prefill(*oracle_prefill_args(inp))
    assert_close(got, ref, "random positions")


def test_deterministic(gqa):
    inp = synthetic.prefill_inputs(1, 300, 8, 2, seed=5)
    a = _run(gqa, inp)
    b = _run(gqa, inp)
    np.testing.assert_array_equal(a, b)


def test_large_prefill_strided_rows(gqa):
    """B=4, T=4096, H=32, Hkv=8, inputs x0.5, in the launch configuration the benchmark
    times.  Checked element by element against the oracle on every 16th row of every
    head (phase shifted per head, so every row offset of a tile is covered), the tile
    edges of every head, and every row of three whole heads (among them the last KV
    head of the last sequence and its last query block)."""
    inp = synthetic.make("large_prefill")
    got = _run(gqa, inp)
    assert np.isfinite(got).all()
    T = 4096
    rows = strided_rows(4, T, 32, 16, edges=(0, 1, 126, 127, 128, 129, 2047, 2048, T - 129, T - 128, T - 1),
                        whole_heads=((3, 31), (0, 0), (2, 13)))
    ref = oracle.prefill_rows(*oracle_prefill_args(inp), rows)
    assert_close(got[rows[:, 0], rows[:, 2], rows[:, 1]], ref, f"large_prefill, {len(rows)} rows")


def test_long_context_prefill_strided_rows(gqa):
    """B=1, T=32768, H=64, Hkv=8, in the benchmark's launch configuration: every 64th
    row of every head (phase shifted per head), tile and half-sequence edges of every
    head, and the last 256 rows of every head of the last KV group (the longest causal
    sweeps, over all 256 key tiles)."""
    inp = synthetic.make("long_context_prefill")
    got = _run(gqa, inp)
    assert np.isfinite(got).all()
    T = 32768
    rows = strided_rows(1, T, 64, 64, edges=(0, 1, 127, 128, 129, 16383, 16384, T - 129, T - 128, T - 1),
                        tail_heads=range(56, 64), tail=256)
    ref = oracle.prefill_rows(*oracle_prefill_args(inp), rows)
    assert_close(got[rows[:, 0], rows[:, 2], rows[:, 1]], ref, f"long_context, {len(rows)} rows")


def test_unequal_bands_odd_groups_strided_rows(gqa):
    """B=1, T=24539 (a ragged last tile), H=21, Hkv=7: each KV group's K/V (12.6 MB) lets six
    groups share L2, so the seven groups run as two bands of 4 and 3, and with 3 query heads
    per group the second head pair of every group has a single head.  Every 128th row of
    every head (phase shifted per head), tile edges, and the last 128 rows of the heads of
    the last group (the short second band's longest sweeps)."""
    B, T, H, Hkv = 1, 24539, 21, 7
    inp = synthetic.prefill_inputs(B, T, H, Hkv, seed=5)
    got = _run(gqa, inp)
    assert np.isfinite(got).all()
    rows = strided_rows(B, T, H, 128, edges=(0, 1, 127, 128, 129, 12287, 12288, T - 129, T - 128, T - 1),
                        tail_heads=range(18, 21), tail=128)
    ref = oracle.prefill_rows(*oracle_prefill_args(inp), rows)
    assert_close(got[rows[:, 0], rows[:, 2], rows[:, 1]], ref, f"unequal bands, {len(rows)} rows")


def _aligned_keys_inputs(T, H, Hkv, seed):
    """Queries all near one direction u; keys random for the first 256 tokens, then turning
    towards u tile by tile, so a row's scores keep rising past its first tile's maximum."""
    inp = synthetic.prefill_inputs(1, T, H, Hkv, seed=seed)
    g = torch.Generator().manual_seed(seed + 7)
    u = torch.randn(128, generator=g)
    inp.q = (u + 0.1 * torch.randn(1, T, H, 128, generator=g)).to(torch.bfloat16)
    k = torch.randn(1, T, Hkv, 128, generator=g)
    t = torch.arange(T, dtype=torch.float32)
    ang = ((t - 256).clamp(min=0) / max(1, T - 256) * (np.pi / 2)).view(1, T, 1, 1)
    inp.k = (torch.cos(ang) * k + torch.sin(ang) * 3.0 * u).to(torch.bfloat16)
    return inp


def test_running_max_growth_rescales(gqa):
    """Scores that grow along the keys by more than 2^8 (base 2) over a row's first tile drive
    the softmax's exact-maximum pass and the rescale of l and O; every row against the
    oracle.  The inputs are checked to reach that case for many rows."""
    T, H, Hkv = 640, 4, 2
    inp = _aligned_keys_inputs(T, H, Hkv, seed=190)
    ro = oracle.Rope(theta=inp.theta)
    qh = oracle.qk_transform_ex(bits_of(inp.q[0]), inp.pos[0].numpy(), inp.wq.numpy(), ro, inp.eps)
    kh = oracle.qk_transform_ex(bits_of(inp.k[0]), inp.pos[0].numpy(), inp.wk.numpy(), ro, inp.eps)
    grows = 0
    for h in range(H):
        sc = qh[:, h, :] @ kh[:, h // (H // Hkv), :].T / np.sqrt(128.0) * np.log2(np.e)
        for i in range(128, T):
            first = sc[i, :128].max()
            later = sc[i, 128:i + 1].max()
            grows += later > first + 8.0
    assert grows > 500, grows
    got = _run(gqa, inp)
    ref = oracle.prefill(*oracle_prefill_args(inp))
    assert_close(got, ref, "scores growing along the keys")


def test_empty_problem_is_noop(gqa):
    dev = "cuda"
    q = torch.empty((0, 5, 4, 128), dtype=torch.bfloat16, device=dev)
    k = torch.empty((0, 5, 2, 128), dtype=torch.bfloat16, device=dev)
    pos = torch.empty((0, 5), dtype=torch.int32, device=dev)
    w = torch.ones(128, device=dev)
    out = gqa.prefill(q, k, k, pos, w, w)
    assert out.shape == (0, 5, 4, 128)


def test_k_norm_rope_matches_oracle_k_hat(gqa):
    """The k-hat stage on its own (the decode-cache writer): bf16 output within one bf16
    rounding of the oracle's k-hat, at positions up to 32767."""
    inp = synthetic.prefill_inputs(2, 300, 4, 4, seed=31)
    g = torch.Generator().manual_seed(32)
    inp.pos = torch.randint(0, 32768, (2, 300), generator=g, dtype=torch.int32)
    khat = gqa.k_norm_rope(inp.k.cuda(), inp.pos.cuda(), inp.wk.cuda(), inp.theta, inp.eps)
    torch.cuda.synchronize()
    ntok = 2 * 300
    ref = oracle.qk_transform(bits_of(inp.k).reshape(ntok, 4, 128), inp.pos.numpy().reshape(ntok), inp.wk.numpy(),
                              inp.theta, inp.eps).reshape(2, 300, 4, 128)
    got = khat.float().cpu().numpy()
    # one bf16 rounding (2^-9 relative) plus fp32 arithmetic
    assert (np.abs(got - ref) <= np.abs(ref) * 2.0 ** -8 + 1e-5).all()


def test_two_stage_prefill_equals_one_call(gqa):
    inp = synthetic.prefill_inputs(2, 190, 8, 2, seed=33)
    d = to_dev(inp)
    one = gqa.prefill(d["q"], d["k"], d["v"], d["pos"], d["qnorm_w"], d["knorm_w"], d["theta"], d["eps"])
    table = torch.empty(gqa.rope_table_numel(2 * 190), dtype=torch.float32, device="cuda")
    khat = gqa.k_norm_rope(d["k"], d["pos"], d["knorm_w"], d["theta"], d["eps"], rope_cs=table)
    two = gqa.prefill_khat(d["q"], khat, d["v"], d["pos"], d["qnorm_w"], d["theta"], d["eps"], rope_cs=table)
    torch.cuda.synchronize()
    assert torch.equal(one, two)


def test_q_rope_without_table_matches_oracle(gqa):
    """The attention stage alone, evaluating the query cos/sin itself (no table)."""
    inp = synthetic.prefill_inputs(1, 300, 8, 4, seed=34)
    g = torch.Generator().manual_seed(35)
    inp.pos = torch.randint(0, 32768, (1, 300), generator=g, dtype=torch.int32)
    d = to_dev(inp)
    khat = gqa.k_norm_rope(d["k"], d["pos"], d["knorm_w"], d["theta"], d["eps"])
    got = gqa.prefill_khat(d["q"], khat, d["v"], d["pos"], d["qnorm_w"], d["theta"], d["eps"])
    torch.cuda.synchronize()
    gqa.check_device_status()
    assert_close(got.cpu().numpy(), oracle.prefill(*oracle_prefill_args(inp)), "no table")


def test_rope_table_matches_closed_form(gqa):
    """The cos/sin table the K prologue writes: cos/sin(pos * theta^(-2i/D))."""
    g = torch.Generator().manual_seed(36)
    pos = torch.cat([torch.tensor([0, 1, 7, 4095, 32767]), torch.randint(0, 32768, (200,), generator=g)]).to(torch.int32)
    n = pos.numel()
    k = torch.zeros((n, 1, 128), dtype=torch.bfloat16)
    table = torch.empty(gqa.rope_table_numel(n), dtype=torch.float32, device="cuda")
    gqa.k_norm_rope(k.cuda(), pos.cuda(), torch.ones(128, device="cuda"), 1e6, 1e-6, rope_cs=table)
    torch.cuda.synchronize()
    tab = table.cpu()
    worst = 0.0
    for i in range(n):
        for pair in (0, 1, 31, 62, 63):
            c, s_ = gqa.rope_table_entry(tab, i, pair)
            ang = float(pos[i]) * 1e6 ** (-2.0 * pair / 128)
            worst = max(worst, abs(c - np.cos(ang)), abs(s_ - np.sin(ang)))
    assert worst < 2e-6, worst
