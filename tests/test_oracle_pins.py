"""Pins of the fp64 CPU oracle to things other than itself.

Each test ties one part of the oracle to what the pages and the mathematics fix:
worked examples with closed-form answers, invariants, degenerate cases that reduce
to a library routine (torch fp64 on the CPU), and brute force on tiny inputs.
Together they are chosen so that a plausible slip anywhere in the oracle (a dropped
term, a wrong sign or index, a transposed operand, the wrong softmax axis, the
wrong RoPE pairing or frequency) fails at least one of them.

Sources: "Qwen3系列1-理论基础&真实结构" D1-2, D1-4, D1-5, D2-1, D2-2, D2-3;
"深入剖析Qwen3模型架构" 3.1.2, 3.4.1; "Qwen3学习日志" section 一;
"Qwen3" (nano-vllm walkthrough) "Attention 的 Forward 流程".
"""
import math
import os

import numpy as np
import pytest
import torch

from oracle import oracle
from grouped_query_causal_b200 import synthetic

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
pytestmark = pytest.mark.filterwarnings("ignore")


def _read_golden(name):
    rows = {}
    with open(os.path.join(GOLDEN, name), encoding="utf-8") as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, rest = line.split(None, 1)
            if ";" in rest:
                rows[key] = np.array([[float(t) for t in r.split()] for r in rest.split(";")])
            else:
                rows[key] = np.array([float(t) for t in rest.split()])
    return rows


# --------------------------------------------------------------------------------------
# Worked examples (closed forms)
# --------------------------------------------------------------------------------------

def test_sdpa_worked_example_3_tokens_dim_2():
    """D1-4 / D1-5 pen-and-paper task: scores / sqrt(2), causal mask, row softmax, P V."""
    g = _read_golden("sdpa_3tok_d2.txt")
    Q, K, V = g["Q"], g["K"], g["V"]
    out, w = oracle.sdpa_gqa(Q[None, :, None, :], K[None, :, None, :], V[None, :, None, :],
                             causal=True, return_weights=True)
    out = out[0, :, 0, :]
    w = w[0, 0]
    a = math.exp(1.0 / math.sqrt(2.0))
    # row 0 sees only key 0 (score 1/sqrt 2): weight 1
    w0 = np.array([1.0, 0.0, 0.0])
    # row 1: scores (0, 1/sqrt 2) -> (1, a) / (1 + a)
    w1 = np.array([1.0, a, 0.0]) / (1.0 + a)
    # row 2: scores (1/sqrt 2, 1/sqrt 2, 2/sqrt 2) -> (a, a, a^2) / (2a + a^2) = (1, 1, a) / (2 + a)
    w2 = np.array([1.0, 1.0, a]) / (2.0 + a)
    W = np.stack([w0, w1, w2])
    np.testing.assert_allclose(w, W, rtol=0, atol=1e-15)
    np.testing.assert_allclose(out, W @ V, rtol=0, atol=1e-14)
    # the numbers the closed forms give, to 6 places, for a reader checking by hand
    np.testing.assert_allclose(out[1], [2.339524, 3.339524], atol=1e-6)
    np.testing.assert_allclose(out[2], [3.510470, 4.510470], atol=1e-6)


def test_rmsnorm_then_rope_worked_example_2d():
    """D2-1 formula and D2-2 pen-and-paper task (RMSNorm of a 2-D query, RoPE, dot)."""
    g = _read_golden("rmsnorm_rope_2d.txt")
    x, w, eps, pos, key = g["x"], g["w"], float(g["eps"][0]), float(g["pos"][0]), g["key"]
    normed = oracle.rmsnorm(x, w, eps)
    # mean(x^2) + eps = (9 + 16)/2 + 3.5 = 16 -> divide by 4 exactly
    np.testing.assert_allclose(normed, x / 4.0, rtol=0, atol=1e-15)
    rotated = oracle.rope(normed, pos, 1.0e6)
    # counter-clockwise quarter turn, R = [[cos, -sin], [sin, cos]]: (a, b) -> (-b, a)
    np.testing.assert_allclose(rotated, [-normed[1], normed[0]], rtol=0, atol=1e-15)
    assert abs(float(rotated @ key) - (-1.0 * 2 + 0.75 * -1)) < 1e-15


def test_rmsnorm_weight_multiplies_and_eps_inside_root():
    x = np.array([3.0, 4.0])
    np.testing.assert_allclose(oracle.rmsnorm(x, [2.0, 0.5], 0.0), [6 / math.sqrt(12.5), 2 / math.sqrt(12.5)],
                               rtol=1e-15)
    # mean, not sum, of squares: D = 4 with two zeros -> mean = 25/4
    x4 = np.array([3.0, 0.0, 4.0, 0.0])
    np.testing.assert_allclose(oracle.rmsnorm(x4, np.ones(4), 0.0), x4 / 2.5, rtol=1e-15)


def test_rope_adjacent_pairs_and_frequency():
    """Pairs are (x[2i], x[2i+1]) ("深入剖析Qwen3模型架构" 3.1.2, D2-2 R(pos)); the angle of
    pair i is pos * base^(-2i/D) (3.4.1)."""
    base = 1.0e6
    D = 4
    # pair 0 has frequency 1: pos = pi/2 turns e0 into e1 (adjacent), not into e2 (half split)
    np.testing.assert_allclose(oracle.rope([1.0, 0, 0, 0], math.pi / 2, base), [0, 1.0, 0, 0], atol=1e-15)
    # pair 1 has frequency base^(-2/4) = 1e-3: pos = 500 pi is a quarter turn of (x2, x3)
    np.testing.assert_allclose(oracle.rope([0, 0, 1.0, 0], 500 * math.pi, base), [0, 0, 0, 1.0], atol=1e-12)
    # pos 0 is the identity
    r = np.random.default_rng(0).standard_normal(128)
    np.testing.assert_array_equal(oracle.rope(r, 0.0, base), r)
    # with D = 128 the last pair has frequency base^(-126/128)
    D = 128
    x = np.zeros(D)
    x[D - 2] = 1.0
    pos = (math.pi / 2) / base ** (-(D - 2) / D)
    y = oracle.rope(x, pos, base)
    assert abs(y[D - 1] - 1.0) < 1e-9 and abs(y[D - 2]) < 1e-9


def test_rope_preserves_norm_and_depends_on_relative_position():
    """D2-2: rotation keeps the norm; q_m . k_n after RoPE depends only on m - n."""
    rng = np.random.default_rng(1)
    q = rng.standard_normal(128)
    k = rng.standard_normal(128)
    for pos in [0, 1, 7, 127, 4095, 32767]:
        assert abs(np.linalg.norm(oracle.rope(q, pos, 1e6)) - np.linalg.norm(q)) < 1e-12
    for m, n in [(5, 3), (100, 0), (4000, 3999), (32767, 1)]:
        ref = oracle.rope(q, m, 1e6) @ oracle.rope(k, n, 1e6)
        for s in [1, 17, 1000, 20000]:
            got = oracle.rope(q, m + s, 1e6) @ oracle.rope(k, n + s, 1e6)
            assert abs(got - ref) < 1e-9 * max(1.0, abs(ref))


# --------------------------------------------------------------------------------------
# Softmax and mask invariants (D1-2, D1-4, D1-5)
# --------------------------------------------------------------------------------------

def test_softmax_rows_sum_to_one_and_masked_weights_are_zero():
    rng = np.random.default_rng(2)
    B, T, H, Hkv, D = 2, 9, 4, 2, 16
    q = rng.standard_normal((B, T, H, D)) * 3
    k = rng.standard_normal((B, T, Hkv, D)) * 3
    v = rng.standard_normal((B, T, Hkv, D))
    _, w = oracle.sdpa_gqa(q, k, v, causal=True, return_weights=True)
    np.testing.assert_allclose(w.sum(-1), 1.0, rtol=0, atol=1e-12)
    upper = np.triu(np.ones((T, T), bool), 1)
    assert (w[..., upper] == 0.0).all()
    assert (w[..., ~upper] > 0.0).all()
    # V = one-hot rows: the output row is exactly the weight row (V is not transposed)
    T2, D2 = 6, 8
    q2 = rng.standard_normal((1, T2, 1, D2))
    k2 = rng.standard_normal((1, T2, 1, D2))
    v2 = np.eye(D2)[:T2][None, :, None, :]
    out2, w2 = oracle.sdpa_gqa(q2, k2, v2, causal=True, return_weights=True)
    np.testing.assert_allclose(out2[0, :, 0, :T2], w2[0, 0], atol=1e-15)
    # all-ones V -> output 1 everywhere
    out3 = oracle.sdpa_gqa(q, k, np.ones_like(v), causal=True)
    np.testing.assert_allclose(out3, 1.0, atol=1e-14)


def test_output_is_linear_in_v():
    rng = np.random.default_rng(3)
    B, T, H, Hkv, D = 1, 7, 4, 2, 8
    q = rng.standard_normal((B, T, H, D))
    k = rng.standard_normal((B, T, Hkv, D))
    v1 = rng.standard_normal((B, T, Hkv, D))
    v2 = rng.standard_normal((B, T, Hkv, D))
    lhs = oracle.sdpa_gqa(q, k, 2.0 * v1 - 0.5 * v2)
    rhs = 2.0 * oracle.sdpa_gqa(q, k, v1) - 0.5 * oracle.sdpa_gqa(q, k, v2)
    np.testing.assert_allclose(lhs, rhs, atol=1e-13)


# --------------------------------------------------------------------------------------
# GQA structure ("Qwen3学习日志" section 一; "深入剖析Qwen3模型架构" 3.1.2)
# --------------------------------------------------------------------------------------

def _torch_sdpa_repeat_interleave(q, k, v, causal=True):
    """torch fp64 on the CPU with K/V repeat_interleave'd to every query head (the
    structure of the GQA snippet in 3.1.2), a library routine independent of the oracle."""
    qt = torch.from_numpy(q).permute(0, 2, 1, 3)           # [B,H,T,D]
    kt = torch.from_numpy(k).permute(0, 2, 1, 3)           # [B,Hkv,T,D]
    vt = torch.from_numpy(v).permute(0, 2, 1, 3)
    rep = q.shape[2] // k.shape[2]
    kt = kt.repeat_interleave(rep, dim=1)
    vt = vt.repeat_interleave(rep, dim=1)
    scores = torch.matmul(qt, kt.transpose(-2, -1)) / math.sqrt(q.shape[-1])
    if causal:
        T = q.shape[1]
        mask = torch.triu(torch.ones(T, T, dtype=torch.bool), 1)
        scores = scores.masked_fill(mask, float("-inf"))
    out = torch.matmul(torch.softmax(scores, dim=-1), vt)
    return out.permute(0, 2, 1, 3).numpy()


@pytest.mark.parametrize("H,Hkv", [(16, 16), (16, 8), (16, 4), (16, 1), (6, 2), (3, 1)])
def test_group_map_matches_torch_repeat_interleave(H, Hkv):
    rng = np.random.default_rng(4 + H + Hkv)
    B, T, D = 2, 13, 16
    q = rng.standard_normal((B, T, H, D))
    k = rng.standard_normal((B, T, Hkv, D))
    v = rng.standard_normal((B, T, Hkv, D))
    np.testing.assert_allclose(oracle.sdpa_gqa(q, k, v), _torch_sdpa_repeat_interleave(q, k, v),
                               rtol=0, atol=1e-12)


def test_explicit_repetition_equals_grouped_indexing_bit_for_bit():
    rng = np.random.default_rng(5)
    B, T, H, Hkv, D = 1, 11, 8, 2, 16
    q = rng.standard_normal((B, T, H, D))
    k = rng.standard_normal((B, T, Hkv, D))
    v = rng.standard_normal((B, T, Hkv, D))
    rep = H // Hkv
    grouped = oracle.sdpa_gqa(q, k, v)
    repeated = oracle.sdpa_gqa(q, np.repeat(k, rep, axis=2), np.repeat(v, rep, axis=2))
    np.testing.assert_array_equal(grouped, repeated)


def test_mha_and_mqa_degeneracies():
    """G = H is MHA (each head alone); G = 1 is MQA (every head on one shared K/V)."""
    rng = np.random.default_rng(6)
    B, T, H, D = 1, 10, 4, 8
    q = rng.standard_normal((B, T, H, D))
    k = rng.standard_normal((B, T, H, D))
    v = rng.standard_normal((B, T, H, D))
    mha = oracle.sdpa_gqa(q, k, v)
    for h in range(H):
        alone = oracle.sdpa_gqa(q[:, :, h:h + 1], k[:, :, h:h + 1], v[:, :, h:h + 1])
        np.testing.assert_array_equal(mha[:, :, h:h + 1], alone)
    mqa = oracle.sdpa_gqa(q, k[:, :, :1], v[:, :, :1])
    for h in range(H):
        alone = oracle.sdpa_gqa(q[:, :, h:h + 1], k[:, :, :1], v[:, :, :1])
        np.testing.assert_array_equal(mqa[:, :, h:h + 1], alone)


# --------------------------------------------------------------------------------------
# The whole sub-block on bf16 inputs
# --------------------------------------------------------------------------------------

def _torch_prefill_fp64(inp: synthetic.PrefillInputs):
    """The sub-block in torch fp64 following the pages' PyTorch structure: RMSNorm per
    head ("Qwen3系列1" D2-1/D2-2), RoPE on (x[..., ::2], x[..., 1::2]) with
    inv_freq = base^(-arange(0, D, 2)/D) (3.1.2 / 3.4.1), repeat_interleave GQA (3.1.2)."""
    q = inp.q.double()
    k = inp.k.double()
    v = inp.v.double()
    D = q.shape[-1]

    def rms(x, w):
        return w.double() * x / torch.sqrt(x.pow(2).mean(-1, keepdim=True) + inp.eps)

    inv_freq = 1.0 / (inp.theta ** (torch.arange(0, D, 2, dtype=torch.float64) / D))
    ang = inp.pos.double()[..., None] * inv_freq            # [B,T,D/2]
    cos = torch.cos(ang)[:, :, None, :]
    sin = torch.sin(ang)[:, :, None, :]

    def rope(x):
        xr, xi = x[..., ::2], x[..., 1::2]
        return torch.stack([xr * cos - xi * sin, xr * sin + xi * cos], dim=-1).flatten(-2)

    qh = rope(rms(q, inp.wq))
    kh = rope(rms(k, inp.wk))
    return _torch_sdpa_repeat_interleave(qh.numpy(), kh.numpy(), v.numpy())


def _bits(t):
    return synthetic.bf16_bits(t)


@pytest.mark.parametrize("B,T,H,Hkv", [(1, 128, 16, 8), (2, 37, 6, 3), (1, 5, 2, 1)])
def test_prefill_matches_torch_fp64_pipeline(B, T, H, Hkv):
    inp = synthetic.prefill_inputs(B, T, H, Hkv, seed=11)
    got = oracle.prefill(_bits(inp.q), _bits(inp.k), _bits(inp.v), inp.pos.numpy(), inp.wq.numpy(),
                         inp.wk.numpy(), inp.theta, inp.eps)
    np.testing.assert_allclose(got, _torch_prefill_fp64(inp), rtol=0, atol=1e-11)


def test_prefill_rows_match_full_prefill():
    inp = synthetic.prefill_inputs(2, 40, 4, 2, seed=12)
    args = (_bits(inp.q), _bits(inp.k), _bits(inp.v), inp.pos.numpy(), inp.wq.numpy(), inp.wk.numpy(),
            inp.theta, inp.eps)
    full = oracle.prefill(*args)
    rows = np.array([(b, h, i) for b in range(2) for h in range(4) for i in range(40)])
    got = oracle.prefill_rows(*args, rows)
    np.testing.assert_allclose(got, full[rows[:, 0], rows[:, 2], rows[:, 1]], rtol=0, atol=1e-13)


def test_norm_scale_invariance():
    """RMSNorm removes a positive scale of q or k (eps = 0): scaling the bf16 inputs
    by 2 (exact in bf16) leaves the output unchanged."""
    inp = synthetic.prefill_inputs(1, 24, 4, 2, seed=13)
    args = dict(pos=inp.pos.numpy(), wq=inp.wq.numpy(), wk=inp.wk.numpy(), theta=inp.theta, eps=0.0)
    a = oracle.prefill(_bits(inp.q), _bits(inp.k), _bits(inp.v), **args)
    b = oracle.prefill(_bits(inp.q * 2), _bits(inp.k * 4), _bits(inp.v), **args)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


def _bruteforce_prefill(qb, kb, vb, pos, wq, wk, theta, eps):
    """Pure-Python loops on tiny inputs: widen bits, RMSNorm, rotate pairs, causal softmax."""
    def widen(bits):
        return float(np.array([int(bits) << 16], np.uint32).view(np.float32)[0])

    B, T, H, D = qb.shape
    Hkv = kb.shape[2]
    rep = H // Hkv

    def transform(vec_bits, w, p):
        x = [widen(t) for t in vec_bits]
        r = math.sqrt(sum(t * t for t in x) / D + eps)
        y = [float(w[d]) * x[d] / r for d in range(D)]
        z = list(y)
        for i in range(D // 2):
            ang = p * theta ** (-2.0 * i / D)
            c, s = math.cos(ang), math.sin(ang)
            z[2 * i] = y[2 * i] * c - y[2 * i + 1] * s
            z[2 * i + 1] = y[2 * i] * s + y[2 * i + 1] * c
        return z

    out = np.zeros((B, T, H, D))
    for b in range(B):
        for hq in range(H):
            g = hq // rep
            for i in range(T):
                qi = transform(qb[b, i, hq], wq, int(pos[b, i]))
                s = []
                for j in range(i + 1):
                    kj = transform(kb[b, j, g], wk, int(pos[b, j]))
                    s.append(sum(qi[d] * kj[d] for d in range(D)) / math.sqrt(D))
                m = max(s)
                e = [math.exp(t - m) for t in s]
                z = sum(e)
                for d in range(D):
                    out[b, i, hq, d] = sum(e[j] / z * widen(vb[b, j, g, d]) for j in range(i + 1))
    return out


@pytest.mark.parametrize("B,T,H,Hkv,D", [(1, 3, 2, 1, 2), (2, 5, 4, 2, 4), (1, 6, 3, 3, 8), (1, 4, 4, 1, 8)])
def test_prefill_bruteforce_tiny(B, T, H, Hkv, D):
    inp = synthetic.prefill_inputs(B, T, H, Hkv, D=D, seed=14)
    args = (_bits(inp.q), _bits(inp.k), _bits(inp.v), inp.pos.numpy(), inp.wq.numpy(), inp.wk.numpy(),
            1.0e4, 1e-6)
    np.testing.assert_allclose(oracle.prefill(*args), _bruteforce_prefill(*args), rtol=0, atol=1e-12)


def test_decode_equals_the_last_row_of_prefill():
    """Decode attends the new token (at position L) to cache rows 0..L; with the cache
    holding k-hat (normed, rotated K) and raw V it must equal row L of the causal
    computation ("Qwen3系列1" D2-3: K/V are written to the cache before attention)."""
    B, L, H, Hkv, D = 3, 20, 8, 2, 32
    inp = synthetic.prefill_inputs(B, L + 1, H, Hkv, D=D, seed=15)
    ntok = B * (L + 1)
    kh = oracle.qk_transform(_bits(inp.k).reshape(ntok, Hkv, D), inp.pos.numpy().reshape(ntok),
                             inp.wk.numpy(), inp.theta, inp.eps)
    kh_bf16 = torch.from_numpy(kh).to(torch.bfloat16)       # the cache stores bf16
    qh = oracle.qk_transform(_bits(inp.q).reshape(ntok, H, D), inp.pos.numpy().reshape(ntok),
                             inp.wq.numpy(), inp.theta, inp.eps)
    ref = oracle.sdpa_gqa(qh.reshape(B, L + 1, H, D), kh_bf16.double().numpy().reshape(B, L + 1, Hkv, D),
                          inp.v.double().numpy())[:, L]
    offsets = np.arange(B + 1, dtype=np.int64) * (L + 1)
    seqlens = np.full(B, L + 1, np.int32)
    qdec = _bits(inp.q)[:, L]                                # raw query of the last token
    got = oracle.decode(qdec, _bits(kh_bf16).reshape(ntok, Hkv, D), _bits(inp.v).reshape(ntok, Hkv, D),
                        offsets, seqlens, np.full(B, L, np.int32), inp.wq.numpy(), inp.theta, inp.eps)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)
    # qpos omitted -> the query sits at position len: here len = L + 1
    got2 = oracle.decode(qdec, _bits(kh_bf16).reshape(ntok, Hkv, D), _bits(inp.v).reshape(ntok, Hkv, D),
                         offsets, seqlens, None, inp.wq.numpy(), inp.theta, inp.eps)
    got3 = oracle.decode(qdec, _bits(kh_bf16).reshape(ntok, Hkv, D), _bits(inp.v).reshape(ntok, Hkv, D),
                         offsets, seqlens, np.full(B, L + 1, np.int32), inp.wq.numpy(), inp.theta, inp.eps)
    np.testing.assert_array_equal(got2, got3)


def test_decode_matches_torch_fp64_on_ragged_cache():
    rng = np.random.default_rng(16)
    B, H, Hkv, D = 4, 8, 2, 16
    seqlens = np.array([1, 5, 17, 3], np.int32)
    inp = synthetic.decode_inputs(B, H, Hkv, D, seed=16, seqlens=seqlens)
    qpos = rng.integers(0, 1000, B).astype(np.int32)
    got = oracle.decode(_bits(inp.q), _bits(inp.k_cache), _bits(inp.v_cache), inp.offsets.numpy(),
                        inp.seqlens.numpy(), qpos, inp.wq.numpy(), inp.theta, inp.eps)
    q = inp.q.double()
    qn = inp.wq.double() * q / torch.sqrt(q.pow(2).mean(-1, keepdim=True) + inp.eps)
    inv_freq = 1.0 / (inp.theta ** (torch.arange(0, D, 2, dtype=torch.float64) / D))
    ang = torch.from_numpy(qpos).double()[:, None, None] * inv_freq
    c, s = torch.cos(ang), torch.sin(ang)
    qh = torch.stack([qn[..., ::2] * c - qn[..., 1::2] * s, qn[..., ::2] * s + qn[..., 1::2] * c], -1).flatten(-2)
    for b in range(B):
        o0, n = int(inp.offsets[b]), int(seqlens[b])
        kc = inp.k_cache[o0:o0 + n].double().permute(1, 0, 2).repeat_interleave(H // Hkv, 0)   # [H,n,D]
        vc = inp.v_cache[o0:o0 + n].double().permute(1, 0, 2).repeat_interleave(H // Hkv, 0)
        p = torch.softmax((kc @ qh[b][:, :, None])[..., 0] / math.sqrt(D), -1)                # [H,n]
        ref = (p[:, :, None] * vc).sum(1)
        np.testing.assert_allclose(got[b], ref.numpy(), rtol=0, atol=1e-12)


# --------------------------------------------------------------------------------------
# Decode step with the new token appended to the cache first
# --------------------------------------------------------------------------------------

def test_decode_append_equals_the_last_row_of_prefill():
    """Appending token L (normed, rotated K at position L; raw V) to a cache holding the
    k-hat / v of tokens 0..L-1, then attending, is row L of the causal computation over
    L + 1 tokens ("Qwen3系列1" D2-3: the new K/V enter the cache before attention)."""
    B, L, H, Hkv, D = 3, 20, 8, 2, 32
    inp = synthetic.prefill_inputs(B, L + 1, H, Hkv, D=D, seed=21)
    ntok = B * (L + 1)
    pos = inp.pos.numpy().reshape(ntok)
    kh = oracle.qk_transform(_bits(inp.k).reshape(ntok, Hkv, D), pos, inp.wk.numpy(), inp.theta, inp.eps)
    qh = oracle.qk_transform(_bits(inp.q).reshape(ntok, H, D), pos, inp.wq.numpy(), inp.theta, inp.eps)
    kh = kh.reshape(B, L + 1, Hkv, D)
    kh_cache = torch.from_numpy(kh[:, :L].copy()).to(torch.bfloat16)   # the cache stores bf16
    # reference keys: cached rows as stored, the appended row exact
    k_ref = np.concatenate([kh_cache.double().numpy(), kh[:, L:]], axis=1)
    ref = oracle.sdpa_gqa(qh.reshape(B, L + 1, H, D), k_ref, inp.v.double().numpy())[:, L]
    # the cache has one free row after each sequence
    kc = torch.zeros(B, L + 1, Hkv, D, dtype=torch.bfloat16)
    kc[:, :L] = kh_cache
    vc = torch.zeros(B, L + 1, Hkv, D, dtype=torch.bfloat16)
    vc[:, :L] = inp.v[:, :L]
    offsets = np.arange(B + 1, dtype=np.int64) * (L + 1)
    seqlens = np.full(B, L, np.int32)
    got, khat = oracle.decode_append(_bits(inp.q)[:, L], _bits(inp.k)[:, L], _bits(inp.v)[:, L],
                                     _bits(kc).reshape(-1, Hkv, D), _bits(vc).reshape(-1, Hkv, D),
                                     offsets, seqlens, None, inp.wq.numpy(), inp.wk.numpy(), inp.theta, inp.eps)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)
    np.testing.assert_array_equal(khat, kh[:, L])
    # an explicit query position equal to the length is the default
    got2, _ = oracle.decode_append(_bits(inp.q)[:, L], _bits(inp.k)[:, L], _bits(inp.v)[:, L],
                                   _bits(kc).reshape(-1, Hkv, D), _bits(vc).reshape(-1, Hkv, D),
                                   offsets, seqlens, seqlens, inp.wq.numpy(), inp.wk.numpy(), inp.theta,
                                   inp.eps)
    np.testing.assert_array_equal(got, got2)


def test_decode_append_to_an_empty_cache_returns_the_new_value():
    """With no cached rows the token attends only to itself: one key, weight 1, so every
    query head of a group returns that group's new value exactly."""
    B, H, Hkv, D = 3, 6, 3, 16
    inp = synthetic.decode_append_inputs(B, H, Hkv, D, seed=22, seqlens=[0, 0, 0])
    got, _ = oracle.decode_append(_bits(inp.q), _bits(inp.k_new), _bits(inp.v_new), _bits(inp.k_cache),
                                  _bits(inp.v_cache), inp.offsets.numpy(), inp.seqlens.numpy(), None,
                                  inp.wq.numpy(), inp.wk.numpy(), inp.theta, inp.eps)
    v = inp.v_new.double().numpy()
    for hq in range(H):
        np.testing.assert_array_equal(got[:, hq], v[:, hq // (H // Hkv)])


def test_decode_append_matches_torch_fp64_on_ragged_cache():
    rng = np.random.default_rng(23)
    B, H, Hkv, D = 4, 8, 2, 16
    seqlens = np.array([0, 5, 17, 2], np.int32)
    inp = synthetic.decode_append_inputs(B, H, Hkv, D, seed=23, seqlens=seqlens, spare=3)
    qpos = rng.integers(0, 1000, B).astype(np.int32)
    got, khat = oracle.decode_append(_bits(inp.q), _bits(inp.k_new), _bits(inp.v_new), _bits(inp.k_cache),
                                     _bits(inp.v_cache), inp.offsets.numpy(), inp.seqlens.numpy(), qpos,
                                     inp.wq.numpy(), inp.wk.numpy(), inp.theta, inp.eps)
    inv_freq = 1.0 / (inp.theta ** (torch.arange(0, D, 2, dtype=torch.float64) / D))

    def norm_rope(x, w, p):   # x [..., D] at positions p (broadcast over leading dims)
        x = x.double()
        xn = w.double() * x / torch.sqrt(x.pow(2).mean(-1, keepdim=True) + inp.eps)
        ang = p[..., None] * inv_freq
        c, s = torch.cos(ang), torch.sin(ang)
        return torch.stack([xn[..., ::2] * c - xn[..., 1::2] * s, xn[..., ::2] * s + xn[..., 1::2] * c], -1).flatten(-2)

    pq = torch.from_numpy(qpos).double()
    qh = norm_rope(inp.q, inp.wq, pq[:, None])          # [B,H,D]
    kn = norm_rope(inp.k_new, inp.wk, pq[:, None])      # [B,Hkv,D]
    np.testing.assert_allclose(khat, kn.numpy(), rtol=0, atol=1e-13)
    for b in range(B):
        o0, n = int(inp.offsets[b]), int(seqlens[b])
        kc = torch.cat([inp.k_cache[o0:o0 + n].double(), kn[b][None]], 0)          # [n+1,Hkv,D]
        vc = torch.cat([inp.v_cache[o0:o0 + n].double(), inp.v_new[b][None].double()], 0)
        kc = kc.permute(1, 0, 2).repeat_interleave(H // Hkv, 0)
        vc = vc.permute(1, 0, 2).repeat_interleave(H // Hkv, 0)
        p = torch.softmax((kc @ qh[b][:, :, None])[..., 0] / math.sqrt(D), -1)
        np.testing.assert_allclose(got[b], (p[:, :, None] * vc).sum(1).numpy(), rtol=0, atol=1e-12)


def test_decode_append_ignores_rows_past_the_length():
    """Stale rows after a sequence's cached rows (where the append writes) play no part."""
    B, H, Hkv, D = 2, 4, 2, 16
    inp = synthetic.decode_append_inputs(B, H, Hkv, D, seed=24, seqlens=[7, 3], spare=4)
    args = (inp.offsets.numpy(), inp.seqlens.numpy(), None, inp.wq.numpy(), inp.wk.numpy(), inp.theta, inp.eps)
    a, _ = oracle.decode_append(_bits(inp.q), _bits(inp.k_new), _bits(inp.v_new), _bits(inp.k_cache),
                                _bits(inp.v_cache), *args)
    kc, vc = inp.k_cache.clone(), inp.v_cache.clone()
    for b in range(B):
        lo = int(inp.offsets[b]) + int(inp.seqlens[b])
        kc[lo:int(inp.offsets[b + 1])] = 7.0
        vc[lo:int(inp.offsets[b + 1])] = -3.0
    b_, _ = oracle.decode_append(_bits(inp.q), _bits(inp.k_new), _bits(inp.v_new), _bits(kc), _bits(vc), *args)
    np.testing.assert_array_equal(a, b_)


# --------------------------------------------------------------------------------------
# RoPE variants: rotate-half pairing and scaled frequencies (linear, NTK, YaRN)
# --------------------------------------------------------------------------------------

def _interleave(x, D):
    """y[2i] = x[i], y[2i+1] = x[i + D/2] along the last axis."""
    y = np.empty_like(x)
    y[..., 0::2] = x[..., :D // 2]
    y[..., 1::2] = x[..., D // 2:]
    return y


def _deinterleave(y, D):
    x = np.empty_like(y)
    x[..., :D // 2] = y[..., 0::2]
    x[..., D // 2:] = y[..., 1::2]
    return x


def test_rope_defaults_equal_the_plain_rope():
    rng = np.random.default_rng(40)
    D = 16
    x = rng.standard_normal(D)
    r = oracle.Rope(theta=1e6)
    np.testing.assert_array_equal(r.inv_freq(D), 1e6 ** (-np.arange(0, D, 2) / D))
    for pos in (0, 3, 1000, 32767):
        np.testing.assert_array_equal(oracle.rope_ex(x, pos, r), oracle.rope(x, pos, 1e6))
    assert r.logit_mult() == 1.0
    for sc in ("linear", "ntk", "yarn"):   # factor 1 is the plain RoPE for every method
        np.testing.assert_allclose(oracle.Rope(scaling=sc, factor=1.0).inv_freq(D), r.inv_freq(D), rtol=1e-15)
        assert oracle.Rope(scaling=sc, factor=1.0).logit_mult() == 1.0


def test_half_pairing_is_adjacent_pairing_of_the_interleaved_vector():
    """Rotating (x[i], x[i+D/2]) is rotating the adjacent pairs of the vector whose
    halves are interleaved: half(x) = deinterleave(adjacent(interleave(x)))."""
    rng = np.random.default_rng(41)
    D = 32
    x = rng.standard_normal(D)
    for pos in (1, 77, 30000):
        half = oracle.rope_ex(x, pos, oracle.Rope(pairing="half"))
        adj = oracle.rope_ex(_interleave(x, D), pos, oracle.Rope())
        np.testing.assert_allclose(half, _deinterleave(adj, D), rtol=0, atol=1e-15)
        # it rotates: norm preserved, and pair 0 of (x0, x_{D/2}) turns by exactly pos radians
        assert abs(np.linalg.norm(half) - np.linalg.norm(x)) < 1e-12
        c, s = math.cos(pos), math.sin(pos)
        assert abs(half[0] - (x[0] * c - x[D // 2] * s)) < 1e-12


def test_linear_scaling_is_the_position_divided_by_the_factor():
    rng = np.random.default_rng(42)
    D = 16
    x = rng.standard_normal(D)
    for s in (2.0, 4.0, 8.0):
        for p in (0, 5, 1000):
            got = oracle.rope_ex(x, s * p, oracle.Rope(scaling="linear", factor=s))
            np.testing.assert_allclose(got, oracle.rope(x, p, 1e6), rtol=0, atol=1e-12)


def test_ntk_keeps_the_highest_frequency_and_divides_the_lowest_by_the_factor():
    D = 128
    base = oracle.Rope().inv_freq(D)
    for s in (2.0, 8.0, 32.0):
        f = oracle.Rope(scaling="ntk", factor=s).inv_freq(D)
        assert f[0] == 1.0
        assert abs(f[-1] / base[-1] - 1.0 / s) < 1e-12
        ratio = f / base
        assert (np.diff(ratio) < 0).all() and (ratio <= 1.0).all()   # interpolation grows with wavelength


def test_yarn_by_parts_and_temperature():
    """Pairs whose wavelength fits the training length more than beta_fast times keep their
    frequency, pairs with fewer than beta_slow wavelengths are divided by s, the ones in
    between blend linearly in the number of wavelengths; logits scale by (0.1 ln s + 1)^2."""
    D, L = 128, 4096
    base = oracle.Rope().inv_freq(D)
    r = L * base / (2 * math.pi)           # wavelengths per training context
    for s in (4.0, 16.0):
        f = oracle.Rope(scaling="yarn", factor=s, original_max_position=L).inv_freq(D)
        hi, lo = r > 32.0, r < 1.0
        assert hi.any() and lo.any() and (~hi & ~lo).any()
        np.testing.assert_array_equal(f[hi], base[hi])
        np.testing.assert_allclose(f[lo], base[lo] / s, rtol=1e-15)
        mid = ~hi & ~lo
        gamma = (f[mid] - base[mid] / s) / (base[mid] - base[mid] / s)
        np.testing.assert_allclose(gamma, (r[mid] - 1.0) / 31.0, rtol=1e-9)
    assert abs(oracle.Rope(scaling="yarn", factor=math.exp(10.0)).logit_mult() - 4.0) < 1e-12
    assert oracle.Rope(scaling="linear", factor=8.0).logit_mult() == 1.0


def test_pipeline_defaults_equal_the_plain_pipeline():
    B, T, H, Hkv, D = 2, 9, 4, 2, 16
    inp = synthetic.prefill_inputs(B, T, H, Hkv, D=D, seed=43)
    rows = np.array([(b, h, i) for b in range(B) for h in range(H) for i in range(T)], np.int64)
    a = oracle.prefill_rows(_bits(inp.q), _bits(inp.k), _bits(inp.v), inp.pos.numpy(), inp.wq.numpy(),
                            inp.wk.numpy(), inp.theta, inp.eps, rows)
    b = oracle.prefill_rows_ex(_bits(inp.q), _bits(inp.k), _bits(inp.v), inp.pos.numpy(), inp.wq.numpy(),
                               inp.wk.numpy(), oracle.Rope(theta=inp.theta), inp.eps, rows)
    np.testing.assert_array_equal(a, b)
    d = synthetic.decode_inputs(3, H, Hkv, D, seed=44, seqlens=[1, 4, 9])
    args = (_bits(d.q), _bits(d.k_cache), _bits(d.v_cache), d.offsets.numpy(), d.seqlens.numpy(), None, d.wq.numpy())
    np.testing.assert_array_equal(oracle.decode(*args, d.theta, d.eps),
                                  oracle.decode_ex(*args, oracle.Rope(theta=d.theta), d.eps))


def test_half_pairing_through_the_pipeline_is_adjacent_on_interleaved_heads():
    """Scores depend on q-hat . k-hat only, which is unchanged when both vectors (and the
    norm weights) have their head dimension interleaved the same way; V is untouched."""
    B, T, H, Hkv, D = 1, 12, 4, 2, 16
    inp = synthetic.prefill_inputs(B, T, H, Hkv, D=D, seed=45)
    rows = np.array([(0, h, i) for h in range(H) for i in range(T)], np.int64)
    il = lambda t: torch.from_numpy(_interleave(t.numpy(), D).copy())   # noqa: E731
    got = oracle.prefill_rows_ex(_bits(inp.q), _bits(inp.k), _bits(inp.v), inp.pos.numpy(), inp.wq.numpy(),
                                 inp.wk.numpy(), oracle.Rope(pairing="half"), inp.eps, rows)
    ref = oracle.prefill_rows_ex(_bits(il(inp.q.float()).to(torch.bfloat16)), _bits(il(inp.k.float()).to(torch.bfloat16)),
                                 _bits(inp.v), inp.pos.numpy(), il(inp.wq).numpy(), il(inp.wk).numpy(), oracle.Rope(),
                                 inp.eps, rows)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_yarn_pipeline_matches_numpy_fp64():
    """Decode with YaRN: q-hat from the (pinned) variant RoPE, logits times the temperature
    factor, plain softmax, in numpy."""
    B, H, Hkv, D = 2, 4, 2, 16
    d = synthetic.decode_inputs(B, H, Hkv, D, seed=46, seqlens=[5, 11])
    rope = oracle.Rope(scaling="yarn", factor=8.0, original_max_position=64)
    got = oracle.decode_ex(_bits(d.q), _bits(d.k_cache), _bits(d.v_cache), d.offsets.numpy(), d.seqlens.numpy(),
                           None, d.wq.numpy(), rope, d.eps)
    m = rope.logit_mult()
    assert m > 1.0
    for b in range(B):
        n, o0 = int(d.seqlens[b]), int(d.offsets[b])
        for hq in range(H):
            x = d.q[b, hq].double().numpy()
            xn = d.wq.double().numpy() * x / np.sqrt((x * x).mean() + d.eps)
            qh = oracle.rope_ex(xn, n, rope)
            kc = d.k_cache[o0:o0 + n, hq // (H // Hkv)].double().numpy()
            vc = d.v_cache[o0:o0 + n, hq // (H // Hkv)].double().numpy()
            s = kc @ qh * m / math.sqrt(D)
            p = np.exp(s - s.max())
            p /= p.sum()
            np.testing.assert_allclose(got[b, hq], p @ vc, rtol=0, atol=1e-12)


# --------------------------------------------------------------------------------------
# Paged KV cache: a storage layout, so the attention must not change
# --------------------------------------------------------------------------------------

def test_paged_decode_equals_contiguous_decode():
    B, H, Hkv, D = 3, 4, 2, 16
    seqlens = [5, 33, 16]
    d = synthetic.decode_inputs(B, H, Hkv, D, seed=60, seqlens=seqlens)
    ref = oracle.decode(_bits(d.q), _bits(d.k_cache), _bits(d.v_cache), d.offsets.numpy(), d.seqlens.numpy(), None,
                        d.wq.numpy(), d.theta, d.eps)
    for ps in (16, 32):
        pc = synthetic.page_cache(d.k_cache, d.v_cache, d.offsets, seqlens, ps, seed=61)
        # pages handed out in a shuffled order: the table is not the identity
        assert not np.array_equal(pc.page_table.numpy()[0, :2], [0, 1])
        got = oracle.decode_paged_ex(_bits(d.q), _bits(pc.k_pages), _bits(pc.v_pages), pc.page_table.numpy(), ps,
                                     d.seqlens.numpy(), None, d.wq.numpy(), oracle.Rope(theta=d.theta), d.eps)
        np.testing.assert_array_equal(got, ref)


def test_paged_append_equals_contiguous_append():
    B, H, Hkv, D = 3, 4, 2, 16
    seqlens = [0, 15, 40]
    a = synthetic.decode_append_inputs(B, H, Hkv, D, seed=62, seqlens=seqlens, spare=1)
    ref, kref = oracle.decode_append(_bits(a.q), _bits(a.k_new), _bits(a.v_new), _bits(a.k_cache), _bits(a.v_cache),
                                     a.offsets.numpy(), a.seqlens.numpy(), None, a.wq.numpy(), a.wk.numpy(), a.theta,
                                     a.eps)
    pc = synthetic.page_cache(a.k_cache, a.v_cache, a.offsets, [s + 1 for s in seqlens], 16, seed=63)
    got, kh = oracle.decode_append_paged_ex(_bits(a.q), _bits(a.k_new), _bits(a.v_new), _bits(pc.k_pages),
                                            _bits(pc.v_pages), pc.page_table.numpy(), 16, a.seqlens.numpy(), None,
                                            a.wq.numpy(), a.wk.numpy(), oracle.Rope(theta=a.theta), a.eps)
    np.testing.assert_array_equal(got, ref)
    np.testing.assert_array_equal(kh, kref)


# --------------------------------------------------------------------------------------
# Chunked prefill against a cache prefix
# --------------------------------------------------------------------------------------

def _chunk_setup(B, P, C, H, Hkv, D, seed):
    """Prefill inputs for P + C tokens; the cache holds the bf16 k-hat / v of the first P."""
    inp = synthetic.prefill_inputs(B, P + C, H, Hkv, D=D, seed=seed)
    ntok = B * (P + C)
    pos = inp.pos.numpy().reshape(ntok)
    kh = oracle.qk_transform(_bits(inp.k).reshape(ntok, Hkv, D), pos, inp.wk.numpy(), inp.theta, inp.eps)
    kh = kh.reshape(B, P + C, Hkv, D)
    kc = torch.from_numpy(kh[:, :P].copy()).to(torch.bfloat16).reshape(B * P, Hkv, D)
    vc = inp.v[:, :P].reshape(B * P, Hkv, D)
    offsets = np.arange(B + 1, dtype=np.int64) * P
    return inp, kh, kc, vc, offsets


def test_chunk_after_a_prefix_equals_the_tail_of_prefill():
    """The last C rows of causal attention over P + C tokens, with the prefix keys as the
    cache stores them (bf16 k-hat), are the chunked prefill of those C tokens."""
    B, P, C, H, Hkv, D = 2, 13, 7, 4, 2, 16
    inp, kh, kc, vc, offsets = _chunk_setup(B, P, C, H, Hkv, D, seed=80)
    ntok = B * (P + C)
    qh = oracle.qk_transform(_bits(inp.q).reshape(ntok, H, D), inp.pos.numpy().reshape(ntok), inp.wq.numpy(),
                             inp.theta, inp.eps).reshape(B, P + C, H, D)
    k_ref = np.concatenate([kc.double().numpy().reshape(B, P, Hkv, D), kh[:, P:]], axis=1)
    ref = oracle.sdpa_gqa(qh, k_ref, inp.v.double().numpy())[:, P:]
    got, khat = oracle.prefill_chunk_ex(_bits(inp.q)[:, P:], _bits(inp.k)[:, P:], _bits(inp.v)[:, P:], _bits(kc),
                                        _bits(vc), offsets, np.full(B, P, np.int32), inp.pos.numpy()[:, P:],
                                        inp.wq.numpy(), inp.wk.numpy(), oracle.Rope(theta=inp.theta), inp.eps)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)
    np.testing.assert_array_equal(khat, kh[:, P:])


def test_paged_chunk_equals_contiguous_chunk():
    """The chunk against a prefix kept in pages handed out in a shuffled order is, bit for
    bit, the chunk against the same prefix kept contiguously."""
    B, P, C, H, Hkv, D = 2, 37, 9, 4, 2, 16
    inp, kh, kc, vc, offsets = _chunk_setup(B, P, C, H, Hkv, D, seed=84)
    args = (_bits(inp.q)[:, P:], _bits(inp.k)[:, P:], _bits(inp.v)[:, P:])
    rest = (inp.pos.numpy()[:, P:], inp.wq.numpy(), inp.wk.numpy(), oracle.Rope(theta=inp.theta), inp.eps)
    ref, kref = oracle.prefill_chunk_ex(*args, _bits(kc), _bits(vc), offsets, np.full(B, P, np.int32), *rest)
    for ps in (16, 32):
        pc = synthetic.page_cache(kc, vc, torch.from_numpy(offsets), [P] * B, ps, seed=85)
        assert not np.array_equal(pc.page_table.numpy()[0, :2], [0, 1])   # not the identity
        got, kgot = oracle.prefill_chunk_paged_ex(*args, _bits(pc.k_pages), _bits(pc.v_pages), pc.page_table.numpy(),
                                                  ps, np.full(B, P, np.int32), *rest)
        np.testing.assert_array_equal(got, ref)
        np.testing.assert_array_equal(kgot, kref)


def test_chunk_rows_equal_the_whole_chunk():
    """The sampled-rows chunk oracle returns, bit for bit, the listed rows (b, hq, i) of the
    whole-chunk oracle: every row in order, and a shuffled subset with repeats."""
    B, P, C, H, Hkv, D = 2, 37, 9, 4, 2, 16
    inp, kh, kc, vc, offsets = _chunk_setup(B, P, C, H, Hkv, D, seed=86)
    args = (_bits(inp.q)[:, P:], _bits(inp.k)[:, P:], _bits(inp.v)[:, P:], _bits(kc), _bits(vc), offsets,
            np.array([P, 5], np.int32), inp.pos.numpy()[:, P:], inp.wq.numpy(), inp.wk.numpy(),
            oracle.Rope(theta=inp.theta, pairing="half"), inp.eps)
    ref, _ = oracle.prefill_chunk_ex(*args)
    every = np.array([(b, h, i) for b in range(B) for h in range(H) for i in range(C)], np.int64)
    got, khat = oracle.prefill_chunk_rows_ex(*args, every)
    np.testing.assert_array_equal(got, ref[every[:, 0], every[:, 2], every[:, 1]])
    np.testing.assert_array_equal(khat, oracle.prefill_chunk_ex(*args)[1])
    rng = np.random.default_rng(87)
    some = every[rng.integers(0, len(every), 25)]
    got, _ = oracle.prefill_chunk_rows_ex(*args, some)
    np.testing.assert_array_equal(got, ref[some[:, 0], some[:, 2], some[:, 1]])


def test_chunk_without_prefix_is_plain_prefill():
    B, C, H, Hkv, D = 2, 9, 4, 2, 16
    inp = synthetic.prefill_inputs(B, C, H, Hkv, D=D, seed=81)
    empty = np.zeros((0, Hkv, D), np.uint16)
    got, _ = oracle.prefill_chunk_ex(_bits(inp.q), _bits(inp.k), _bits(inp.v), empty, empty,
                                     np.zeros(B + 1, np.int64), np.zeros(B, np.int32), inp.pos.numpy(), inp.wq.numpy(),
                                     inp.wk.numpy(), oracle.Rope(theta=inp.theta), inp.eps)
    ref = oracle.prefill(_bits(inp.q), _bits(inp.k), _bits(inp.v), inp.pos.numpy(), inp.wq.numpy(), inp.wk.numpy(),
                         inp.theta, inp.eps)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_chunk_of_one_token_is_the_append_step():
    B, H, Hkv, D = 3, 4, 2, 16
    seqlens = [0, 6, 11]
    a = synthetic.decode_append_inputs(B, H, Hkv, D, seed=82, seqlens=seqlens, spare=1)
    rope = oracle.Rope(theta=a.theta, scaling="yarn", factor=4.0, original_max_position=8)
    qpos = np.array([3, 40, 7], np.int32)
    ref, kref = oracle.decode_append_ex(_bits(a.q), _bits(a.k_new), _bits(a.v_new), _bits(a.k_cache),
                                        _bits(a.v_cache), a.offsets.numpy(), a.seqlens.numpy(), qpos, a.wq.numpy(),
                                        a.wk.numpy(), rope, a.eps)
    got, khat = oracle.prefill_chunk_ex(_bits(a.q)[:, None], _bits(a.k_new)[:, None], _bits(a.v_new)[:, None],
                                        _bits(a.k_cache), _bits(a.v_cache), a.offsets.numpy(), a.seqlens.numpy(),
                                        qpos[:, None], a.wq.numpy(), a.wk.numpy(), rope, a.eps)
    np.testing.assert_array_equal(got[:, 0], ref)
    np.testing.assert_array_equal(khat[:, 0], kref)


# --------------------------------------------------------------------------------------
# Variable-length packed prefill
# --------------------------------------------------------------------------------------

def test_varlen_prefill_is_each_sequence_on_its_own():
    """Packing sequences end to end changes nothing: each token attends causally within
    its own sequence, so every sequence's rows equal its own prefill, and no key of a
    neighbouring sequence leaks in."""
    H, Hkv, D = 4, 2, 16
    lens = [5, 1, 12, 0, 7]
    seqs = [synthetic.prefill_inputs(1, n, H, Hkv, D=D, seed=100 + i) for i, n in enumerate(lens) if n > 0]
    q = torch.cat([s.q[0] for s in seqs])
    k = torch.cat([s.k[0] for s in seqs])
    v = torch.cat([s.v[0] for s in seqs])
    pos = torch.cat([s.pos[0] + 1000 * i for i, s in enumerate(seqs)])
    wq, wk = seqs[0].wq, seqs[0].wk
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    got = oracle.prefill_varlen_ex(_bits(q), _bits(k), _bits(v), cu, pos.numpy(), wq.numpy(), wk.numpy(),
                                   oracle.Rope(), 1e-6)
    o = 0
    for i, s in enumerate(seqs):
        n = s.q.shape[1]
        ref = oracle.prefill(_bits(s.q), _bits(s.k), _bits(s.v), (s.pos + 1000 * i).numpy(), wq.numpy(), wk.numpy(),
                             1e6, 1e-6)[0]
        np.testing.assert_allclose(got[o:o + n], ref, rtol=0, atol=1e-12)
        o += n
    assert o == q.shape[0]


# ----------------------------------------------------------------------------- projections
# "Qwen3系列1" D1-2 (a linear layer is Y = XW + b; Qwen3's projections have no b), D1-4
# Q4/Q5 (heads concatenated, then W_O); "深入剖析Qwen3模型架构" 3.1.2 (no QKV bias); the
# "Qwen3" walkthrough's forward steps 1-3 (qkv_proj, split, per-head view) and 7 (o_proj).

def _bf(a):
    return synthetic.bf16_bits(torch.as_tensor(np.asarray(a, np.float32)).to(torch.bfloat16))


def test_linear_worked_example():
    """y = x W^T by hand: x = [[1,2,3],[4,5,6]], W = [[1,0,-1],[2,1,0]] gives
    [[1-3, 2+2], [4-6, 8+5]] = [[-2, 4], [-2, 13]].  A transposed W (3x2) or x W
    instead of x W^T cannot produce this shape and these values."""
    y = oracle.linear(_bf([[1, 2, 3], [4, 5, 6]]), _bf([[1, 0, -1], [2, 1, 0]]))
    np.testing.assert_array_equal(y, [[-2.0, 4.0], [-2.0, 13.0]])


def test_linear_identity_scaling_and_permutation():
    g = torch.Generator().manual_seed(200)
    x = torch.randn(5, 64, generator=g).to(torch.bfloat16)
    xb = synthetic.bf16_bits(x)
    # identity weights return the input exactly (every bf16 value is a double)
    np.testing.assert_array_equal(oracle.linear(xb, _bf(np.eye(64))), x.double().numpy())
    w = torch.randn(48, 64, generator=g).to(torch.bfloat16)
    y = oracle.linear(xb, synthetic.bf16_bits(w))
    # doubling the weights doubles the output exactly
    np.testing.assert_array_equal(oracle.linear(xb, synthetic.bf16_bits(w * 2)), 2 * y)
    # permuting the output rows of W permutes the output columns
    perm = torch.randperm(48, generator=g)
    np.testing.assert_array_equal(oracle.linear(xb, synthetic.bf16_bits(w[perm])), y[:, perm.numpy()])
    # linear in x: inputs with disjoint supports add
    mask = torch.arange(64) % 3 == 0
    x1, x2 = torch.where(mask, x, 0), torch.where(mask, 0, x)
    y12 = oracle.linear(synthetic.bf16_bits(x1), synthetic.bf16_bits(w)) + \
        oracle.linear(synthetic.bf16_bits(x2), synthetic.bf16_bits(w))
    np.testing.assert_allclose(y12, y, rtol=1e-12, atol=1e-12)


def test_linear_matches_torch_fp64_matmul():
    g = torch.Generator().manual_seed(201)
    x = torch.randn(7, 3, 96, generator=g).to(torch.bfloat16)
    w = torch.randn(40, 96, generator=g).to(torch.bfloat16)
    ref = (x.double() @ w.double().T).numpy()
    got = oracle.linear(synthetic.bf16_bits(x), synthetic.bf16_bits(w))
    assert got.shape == (7, 3, 40)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-11)


def test_qkv_proj_splits_into_the_three_projections():
    """The fused projection's q, k and v sections are the separate q/k/v projections
    (W_qkv = [W_q; W_k; W_v]) viewed per head, bit for bit."""
    H, Hkv, D, hidden = 4, 2, 16, 32
    g = torch.Generator().manual_seed(202)
    x = synthetic.bf16_bits(torch.randn(6, hidden, generator=g).to(torch.bfloat16))
    wq, wk, wv = (torch.randn(n * D, hidden, generator=g).to(torch.bfloat16) for n in (H, Hkv, Hkv))
    q, k, v = oracle.qkv_proj(x, synthetic.bf16_bits(torch.cat([wq, wk, wv])), H, Hkv, D)
    np.testing.assert_array_equal(q, oracle.linear(x, synthetic.bf16_bits(wq)).reshape(6, H, D))
    np.testing.assert_array_equal(k, oracle.linear(x, synthetic.bf16_bits(wk)).reshape(6, Hkv, D))
    np.testing.assert_array_equal(v, oracle.linear(x, synthetic.bf16_bits(wv)).reshape(6, Hkv, D))


def test_o_proj_is_concat_then_w_o():
    """Concatenating the heads and applying W_O equals summing each head's share of W_O:
    o_proj(o) = sum_h o[:, h] W_O[:, h D:(h+1) D]^T."""
    H, D, hidden = 3, 8, 20
    g = torch.Generator().manual_seed(203)
    o = torch.randn(5, H, D, generator=g).to(torch.bfloat16)
    w = torch.randn(hidden, H * D, generator=g).to(torch.bfloat16)
    got = oracle.o_proj(synthetic.bf16_bits(o), synthetic.bf16_bits(w))
    ref = sum(o[:, h].double() @ w[:, h * D:(h + 1) * D].double().T for h in range(H)).numpy()
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-11)


def test_round_bf16_ties_to_even_and_matches_torch():
    # 1 + 2^-8 lies halfway between 1 and 1 + 2^-7: the even neighbour is 1;
    # 1 + 3 * 2^-8 lies halfway between 1 + 2^-7 and 1 + 2^-6: the even one is 1 + 2^-6
    got = oracle.round_bf16_bits([1.0, 1 + 2 ** -8, 1 + 3 * 2 ** -8, -2.5, 0.0, 3.0e-3])
    assert got[0] == 0x3F80 and got[1] == 0x3F80 and got[2] == 0x3F82
    assert got[3] == 0xC020 and got[4] == 0
    g = torch.Generator().manual_seed(204)
    x = torch.randn(10000, generator=g) * 10.0 ** torch.randint(-3, 4, (10000,), generator=g)
    ref = synthetic.bf16_bits(x.to(torch.bfloat16))
    np.testing.assert_array_equal(oracle.round_bf16_bits(x.double().numpy()), ref)


def test_attention_block_with_identity_projections_is_the_prefill():
    """With W_qkv = [I; I_kv; I_kv] (hidden = H D, k and v the first Hkv D features) and
    W_o = I, the sub-block reduces to the prefill on q = x, k = v = x[:, :Hkv D], rounded
    to bf16 at the end: steps in the pages' order, split at the right boundaries."""
    B, T, H, Hkv, D = 1, 40, 4, 2, 16
    hidden = H * D
    inp = synthetic.prefill_inputs(B, T, H, Hkv, D=D, seed=205)
    x = inp.q.reshape(B, T, hidden)
    eye = torch.eye(hidden)
    w_qkv = torch.cat([eye, eye[:Hkv * D], eye[:Hkv * D]]).to(torch.bfloat16)
    w_o = eye.to(torch.bfloat16)
    rope = oracle.Rope(theta=inp.theta)
    y = oracle.attn_block_prefill(synthetic.bf16_bits(x), synthetic.bf16_bits(w_qkv), synthetic.bf16_bits(w_o),
                                  inp.pos.numpy(), inp.wq.numpy(), inp.wk.numpy(), rope, inp.eps, H, Hkv, D)
    xk = x.reshape(B, T, H, D)[:, :, :Hkv].contiguous()
    o = oracle.prefill(synthetic.bf16_bits(inp.q), synthetic.bf16_bits(xk), synthetic.bf16_bits(xk),
                       inp.pos.numpy(), inp.wq.numpy(), inp.wk.numpy(), inp.theta, inp.eps)
    ref = oracle.round_bf16_bits(o).view(np.uint16)
    ref = torch.from_numpy(ref.astype(np.int16)).view(torch.bfloat16).double().numpy().reshape(B, T, hidden)
    np.testing.assert_array_equal(y, ref)


def test_attention_block_rows_equal_the_full_block():
    B, T, H, Hkv, D, hidden = 2, 24, 4, 2, 16, 48
    g = torch.Generator().manual_seed(206)
    x = torch.randn(B, T, hidden, generator=g).to(torch.bfloat16)
    w_qkv = (torch.randn((H + 2 * Hkv) * D, hidden, generator=g) / hidden ** 0.5).to(torch.bfloat16)
    w_o = (torch.randn(hidden, H * D, generator=g) / (H * D) ** 0.5).to(torch.bfloat16)
    pos = torch.arange(T, dtype=torch.int32).repeat(B, 1).numpy()
    wq = np.linspace(0.5, 1.5, D).astype(np.float32)
    wk = wq[::-1].copy()
    args = (synthetic.bf16_bits(x), synthetic.bf16_bits(w_qkv), synthetic.bf16_bits(w_o), pos, wq, wk,
            oracle.Rope(theta=1e6), 1e-6, H, Hkv, D)
    full = oracle.attn_block_prefill(*args)
    rows = [(1, 0), (0, 23), (1, 17)]
    part = oracle.attn_block_prefill(*args, rows=rows)
    np.testing.assert_array_equal(part, np.stack([full[b, t] for b, t in rows]))
