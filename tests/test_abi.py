"""The C-ABI library loads, exports every symbol its header declares, and rejects bad
arguments on the host before anything reaches a GPU (no compute calls: CPU only)."""
import ctypes
import os
import re
import subprocess

import pytest

from grouped_query_causal_b200 import binding, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gqa_attn.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return binding.load()


def _declared():
    text = open(HEADER, encoding="utf-8").read()
    return sorted(set(re.findall(r"\b(gqa_\w+)\s*\(", text)))


def test_header_declares_what_the_binding_names():
    assert _declared() == sorted(binding.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", binding.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for name in _declared():
        assert name in exported, name
        assert getattr(lib, name) is not None
    # nothing but the C ABI is exported
    assert {n for n in exported if n.startswith("gqa")} == set(_declared())


def test_status_strings(lib):
    for code, name in binding.STATUS_NAMES.items():
        assert lib.gqa_status_string(code).decode() == name


def test_workspace_sizes(lib):
    # k-hat (bf16 [B,T,Hkv,D], rounded to 256 B) + RoPE table (round_up(B*T, 128) tokens x 512 B)
    assert lib.gqa_attn_prefill_workspace_size(4, 4096, 32, 8, 128) == 4 * 4096 * 8 * 128 * 2 + 4 * 4096 * 128 * 4
    assert lib.gqa_attn_prefill_workspace_size(1, 3, 2, 1, 128) == 3 * 128 * 2 + 128 * 128 * 4
    assert lib.gqa_attn_prefill_workspace_size(1, 128, 16, 8, 64) == 0
    assert lib.gqa_attn_prefill_workspace_size(1, 128, 16, 3, 128) == 0
    assert lib.gqa_attn_prefill_workspace_size(0, 128, 16, 8, 128) == 0
    slots = 64 * 32 * 32   # sequences x 1024-key chunks of 32768 keys x query heads
    assert lib.gqa_attn_decode_workspace_size(64, 32, 8, 128, 32768) == slots * 128 * 4 + slots * 2 * 4
    assert lib.gqa_attn_decode_workspace_size(2, 8, 2, 128, 1) == 2 * 8 * 128 * 4 + 256
    assert lib.gqa_attn_decode_workspace_size(2, 8, 3, 128, 100) == 0
    assert lib.gqa_attn_decode_workspace_size(2, 8, 2, 128, 0) == 0


def _prefill(lib, **kw):
    a = dict(q=16, k=16, v=16, pos=16, wq=16, wk=16, theta=1e6, eps=1e-6, out=16, B=1, T=8, H=4, Hkv=2, D=128,
             ws=256, wsb=1 << 20, stream=None)
    a.update(kw)
    return lib.gqa_attn_prefill(a["q"], a["k"], a["v"], a["pos"], a["wq"], a["wk"], a["theta"], a["eps"],
                                a["out"], a["B"], a["T"], a["H"], a["Hkv"], a["D"], a["ws"], a["wsb"],
                                a["stream"])


def test_prefill_argument_errors_are_caught_on_the_host(lib):
    # these return before any CUDA call (the pointers are never dereferenced)
    assert _prefill(lib, D=64) == -2
    assert _prefill(lib, D=0) == -1
    assert _prefill(lib, H=5, Hkv=2) == -1
    assert _prefill(lib, Hkv=0) == -1
    assert _prefill(lib, B=-1) == -1
    assert _prefill(lib, theta=0.0) == -1
    assert _prefill(lib, theta=float("nan")) == -1
    assert _prefill(lib, eps=-1.0) == -1
    assert _prefill(lib, q=None) == -1
    assert _prefill(lib, out=None) == -1
    assert _prefill(lib, k=24) == -1        # misaligned
    assert _prefill(lib, ws=None) == -3
    assert _prefill(lib, ws=128) == -3      # workspace not 256-aligned
    assert _prefill(lib, wsb=100) == -3     # too small
    assert _prefill(lib, B=0) == 0          # empty: no-op
    assert _prefill(lib, T=0, q=None) == 0


def _decode(lib, **kw):
    a = dict(q=16, kc=16, vc=16, offs=16, sl=16, qpos=None, wq=16, theta=1e6, eps=1e-6, out=16, B=2, H=8,
             Hkv=2, D=128, max_len=100, ws=256, wsb=1 << 20, stream=None)
    a.update(kw)
    return lib.gqa_attn_decode(a["q"], a["kc"], a["vc"], a["offs"], a["sl"], a["qpos"], a["wq"], a["theta"],
                               a["eps"], a["out"], a["B"], a["H"], a["Hkv"], a["D"], a["max_len"], a["ws"],
                               a["wsb"], a["stream"])


def test_decode_argument_errors_are_caught_on_the_host(lib):
    assert _decode(lib, D=256) == -2
    assert _decode(lib, H=8, Hkv=3) == -1
    assert _decode(lib, max_len=0) == -1
    assert _decode(lib, max_len=1 << 30) == -1   # more chunks than a grid dimension holds
    assert _decode(lib, kc=None) == -1
    assert _decode(lib, offs=20) == -1          # int64 offsets must be 8-byte aligned
    assert _decode(lib, qpos=18) == -1
    assert _decode(lib, eps=float("inf")) == -1
    assert _decode(lib, wsb=10) == -3
    assert _decode(lib, B=0) == 0


def _decode_append(lib, **kw):
    a = dict(q=16, kn=16, vn=16, kc=16, vc=16, offs=16, sl=16, qpos=None, wq=16, wk=16, theta=1e6, eps=1e-6,
             out=16, B=2, H=8, Hkv=2, D=128, max_len=100, ws=256, wsb=1 << 20, stream=None)
    a.update(kw)
    return lib.gqa_attn_decode_append(a["q"], a["kn"], a["vn"], a["kc"], a["vc"], a["offs"], a["sl"], a["qpos"],
                                      a["wq"], a["wk"], a["theta"], a["eps"], a["out"], a["B"], a["H"], a["Hkv"],
                                      a["D"], a["max_len"], a["ws"], a["wsb"], a["stream"])


def test_decode_append_argument_errors_are_caught_on_the_host(lib):
    assert _decode_append(lib, kn=None) == -1
    assert _decode_append(lib, vn=None) == -1
    assert _decode_append(lib, wk=None) == -1
    assert _decode_append(lib, kn=20) == -1     # new rows must be 8-byte aligned
    assert _decode_append(lib, wk=24) == -1     # knorm_w must be 16-byte aligned
    assert _decode_append(lib, D=256) == -2
    assert _decode_append(lib, H=8, Hkv=3) == -1
    assert _decode_append(lib, max_len=0) == -1
    assert _decode_append(lib, wsb=10) == -3
    assert _decode_append(lib, B=0) == 0


def _rope(**kw):
    return binding.RopeConfig.make(**kw)


def test_rope_config_errors_are_caught_on_the_host(lib):
    def pre(rope):
        return lib.gqa_attn_prefill_ex(16, 16, 16, 16, 16, 16, rope, 1e-6, 16, 1, 8, 4, 2, 128, 256, 1 << 20, None)
    assert pre(None) == -1
    bad = [_rope(theta=0.0), _rope(theta=float("inf")), _rope(scaling="linear", factor=0.5),
           _rope(scaling="ntk", factor=float("nan")), _rope(scaling="yarn", factor=4.0, original_max_position=0),
           _rope(scaling="yarn", factor=4.0, beta_fast=1.0, beta_slow=1.0)]
    c = _rope()
    c.pairing = 2
    bad.append(c)
    c = _rope()
    c.scaling = 7
    bad.append(c)
    for r in bad:
        assert pre(ctypes.byref(r)) == -1
        assert lib.gqa_attn_decode_ex(16, 16, 16, 16, 16, None, 16, ctypes.byref(r), 1e-6, 16, 2, 8, 2, 128, 100, 256,
                                      1 << 20, None) == -1
    ok = _rope(pairing="half", scaling="yarn", factor=8.0)
    assert lib.gqa_attn_prefill_ex(16, 16, 16, 16, 16, 16, ctypes.byref(ok), 1e-6, 16, 0, 8, 4, 2, 128, 256, 1 << 20,
                                   None) == 0          # B = 0: valid configuration, nothing to do
    assert lib.gqa_attn_k_norm_rope_ex(16, 16, 16, ctypes.byref(ok), 1e-6, 16, None, 0, 2, 128, None) == 0
    assert lib.gqa_attn_k_norm_rope_ex(16, 16, 16, ctypes.byref(ok), -1.0, 16, None, 0, 2, 128, None) == -1


def test_paged_decode_argument_errors_are_caught_on_the_host(lib):
    r = ctypes.byref(_rope())

    def dec(**kw):
        a = dict(q=16, kp=16, vp=16, tab=16, npages=10, ps=16, maxp=4, sl=16, qpos=None, wq=16, rope=r, eps=1e-6,
                 out=16, B=2, H=8, Hkv=2, D=128, max_len=64, ws=256, wsb=1 << 20)
        a.update(kw)
        return lib.gqa_attn_decode_paged(a["q"], a["kp"], a["vp"], a["tab"], a["npages"], a["ps"], a["maxp"], a["sl"],
                                         a["qpos"], a["wq"], a["rope"], a["eps"], a["out"], a["B"], a["H"], a["Hkv"],
                                         a["D"], a["max_len"], a["ws"], a["wsb"], None)
    assert dec(ps=8) == -1          # page size must be a multiple of 16
    assert dec(ps=24) == -1
    assert dec(npages=0) == -1
    assert dec(maxp=0) == -1
    assert dec(tab=None) == -1
    assert dec(tab=18) == -1        # int32 table must be 4-byte aligned
    assert dec(rope=None) == -1
    assert dec(D=64) == -2
    assert dec(B=0) == 0
    assert lib.gqa_attn_decode_append_paged(16, None, 16, 16, 16, 16, 10, 16, 4, 16, None, 16, 16, r, 1e-6, 16, 2, 8,
                                            2, 128, 64, 256, 1 << 20, None) == -1


def test_paged_chunk_argument_errors_are_caught_on_the_host(lib):
    r = ctypes.byref(_rope())

    def chunk(**kw):
        a = dict(q=16, k=16, v=16, pos=16, cu=16, kp=16, vp=16, tab=16, npages=10, ps=16, maxp=4, pl=16, wq=16,
                 wk=16, rope=r, eps=1e-6, out=16, B=2, N=40, H=8, Hkv=2, D=128, mcl=32, ws=256, wsb=1 << 20)
        a.update(kw)
        return lib.gqa_attn_prefill_chunk_paged(a["q"], a["k"], a["v"], a["pos"], a["cu"], a["kp"], a["vp"], a["tab"],
                                                a["npages"], a["ps"], a["maxp"], a["pl"], a["wq"], a["wk"], a["rope"],
                                                a["eps"], a["out"], a["B"], a["N"], a["H"], a["Hkv"], a["D"],
                                                a["mcl"], a["ws"], a["wsb"], None)
    assert chunk(ps=8) == -1        # page size must be a multiple of 16
    assert chunk(ps=48) == -2       # ... that divides 128 or is a multiple of it
    assert chunk(ps=160) == -2
    assert chunk(npages=0) == -1
    assert chunk(maxp=0) == -1
    assert chunk(npages=1 << 27, ps=16) == -1   # page rows must stay below 2^31 - 256
    assert chunk(tab=None) == -1
    assert chunk(tab=18) == -1      # int32 table must be 4-byte aligned
    assert chunk(kp=24) == -1
    assert chunk(cu=20) == -1
    assert chunk(rope=None) == -1
    assert chunk(D=64) == -2
    assert chunk(H=8, Hkv=3) == -1
    assert chunk(wsb=10) == -3
    assert chunk(ws=128) == -3
    assert chunk(B=0) == 0
    assert chunk(N=0, q=None) == 0
    assert lib.gqa_attn_prefill_chunk_paged_workspace_size(40, 128) == lib.gqa_attn_prefill_chunk_workspace_size(40, 128)


def test_binding_fails_loudly_without_the_library(tmp_path):
    saved = binding._lib
    binding._lib = None
    try:
        with pytest.raises(RuntimeError):
            binding.load(str(tmp_path / "missing.so"))
    finally:
        binding._lib = saved
