"""Host-side checks of the C ABI that need no GPU.

* The shared library loads and exports every function include/attn.h declares.
* Status strings exist for every status code.
* Argument validation returns the documented code before anything is launched. Each
  case below carries at least one invalid argument, so even on a GPU host no kernel
  can run on the fake pointers these tests pass.
* The workspace size query is pure host arithmetic.
"""
from __future__ import annotations

import os
import re

import pytest
import torch

import tiled_attention_19_b200 as ta

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn.h")

P = 0x10000  # a 16-byte-aligned fake address (never dereferenced: every call is invalid)


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(attn_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_expected_entry_points():
    names = declared_functions()
    for n in ("attn_fwd", "attn_fwd_window", "attn_fwd_paged", "attn_paged_workspace_size",
              "attn_error_string", "attn_get_device_status"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = ta.load()
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in attn.h but not exported"
        assert name in ta.SIGNATURES, f"{name} has no binding signature"


def declared_arities():
    """Parameter count of every attn_* function the header declares."""
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    out = {}
    for name, params in re.findall(r"\b(attn_[a-z_0-9]+)\s*\(([^;{]*?)\)\s*;", text, flags=re.S):
        params = params.strip()
        out[name] = 0 if params in ("", "void") else params.count(",") + 1
    return out


def test_binding_signatures_match_the_header():
    """Each ctypes signature has as many arguments as the C declaration: a parameter
    added to the header without the binding (or the reverse) fails here, on the CPU."""
    arity = declared_arities()
    assert set(arity) == set(declared_functions())
    for name, n in arity.items():
        assert len(ta.SIGNATURES[name][1]) == n, (name, n, len(ta.SIGNATURES[name][1]))


def test_error_strings():
    for code in ta.STATUS:
        s = ta.error_string(code)
        assert s and s != "unknown status"
    assert ta.error_string(12345) == "unknown status"


def fwd_args(**kw):
    a = dict(q=P, k=P, v=P, out=P, lse=P, B=1, Hq=2, Hkv=1, Lq=8, Lk=8, D=64, scale=0.125,
             causal=0, dtype=0, stream=None)
    a.update(kw)
    return a


FWD_BAD = [
    ("null_q", dict(q=None), -1),
    ("null_out", dict(out=None), -1),
    ("null_k_with_keys", dict(k=None), -1),
    ("neg_B", dict(B=-1), -1),
    ("zero_Hq", dict(Hq=0), -1),
    ("zero_Hkv", dict(Hkv=0), -1),
    ("neg_Lq", dict(Lq=-3), -1),
    ("neg_Lk", dict(Lk=-3), -1),
    ("group_not_divisible", dict(Hq=3, Hkv=2), -1),
    ("scale_zero", dict(scale=0.0), -1),
    ("scale_negative", dict(scale=-0.5), -1),
    ("scale_nan", dict(scale=float("nan")), -1),
    ("scale_inf", dict(scale=float("inf")), -1),
    ("D_96", dict(D=96), -2),
    ("D_256", dict(D=256), -2),
    ("dtype_fp32", dict(dtype=7), -2),
    ("Lq_too_long", dict(Lq=(1 << 22) + 1), -2),
    ("misaligned_q", dict(q=P + 2), -3),
    ("misaligned_v", dict(v=P + 8), -3),
    ("misaligned_lse", dict(lse=P + 2), -3),
]


@pytest.mark.parametrize("name,kw,code", FWD_BAD, ids=[c[0] for c in FWD_BAD])
def test_attn_fwd_validation(name, kw, code):
    a = fwd_args(**kw)
    rc = ta.load().attn_fwd(a["q"], a["k"], a["v"], a["out"], a["lse"], a["B"], a["Hq"], a["Hkv"],
                            a["Lq"], a["Lk"], a["D"], a["scale"], a["causal"], a["dtype"],
                            a["stream"])
    assert rc == code, (rc, ta.STATUS.get(rc))


def paged_args(**kw):
    a = dict(q=P, kc=P, vc=P, bt=P, sl=P, bs=16, out=P, lse=P, S=4, Hq=12, Hkv=2, D=128, MB=256,
             NB=1024, scale=0.088, dtype=1, ws=P, ws_n=1 << 30, stream=None)
    a.update(kw)
    return a


PAGED_BAD = [
    ("null_block_table", dict(bt=None), -1),
    ("null_seq_lens", dict(sl=None), -1),
    ("neg_seqs", dict(S=-1), -1),
    ("group_not_divisible", dict(Hq=12, Hkv=5), -1),
    ("neg_blocks", dict(NB=-1), -1),
    ("scale_nan", dict(scale=float("nan")), -1),
    ("block_size_32", dict(bs=32), -2),
    ("D_80", dict(D=80), -2),
    ("group_too_large", dict(Hq=32, Hkv=1), -2),
    ("misaligned_cache", dict(kc=P + 4), -3),
    ("misaligned_table", dict(bt=P + 2), -3),
    ("workspace_missing", dict(ws=None, ws_n=0), -7),
    ("workspace_small", dict(ws_n=1024), -7),
    ("workspace_misaligned", dict(ws=P + 16), -3),
]


@pytest.mark.parametrize("name,kw,code", PAGED_BAD, ids=[c[0] for c in PAGED_BAD])
def test_attn_fwd_paged_validation(name, kw, code):
    a = paged_args(**kw)
    rc = ta.load().attn_fwd_paged(a["q"], a["kc"], a["vc"], a["bt"], a["sl"], a["bs"], a["out"],
                                  a["lse"], a["S"], a["Hq"], a["Hkv"], a["D"], a["MB"], a["NB"],
                                  a["scale"], a["dtype"], a["ws"], a["ws_n"], a["stream"])
    assert rc == code, (rc, ta.STATUS.get(rc))


def test_attn_fwd_window_validation():
    lib = ta.load()
    a = fwd_args()
    base = (a["q"], a["k"], a["v"], a["out"], a["lse"], a["B"], a["Hq"], a["Hkv"], a["Lq"], a["Lk"],
            a["D"], a["scale"], 0)
    assert lib.attn_fwd_window(*base, -2, 5, 0, None) == -1       # bound below -1
    assert lib.attn_fwd_window(*base, 5, -3, 0, None) == -1
    bad = list(base)
    bad[10] = 96                                                   # D: unsupported
    assert lib.attn_fwd_window(*bad, 4, 4, 0, None) == -2


@pytest.mark.skipif(torch.cuda.is_available(), reason="only meaningful without a GPU")
def test_valid_call_without_gpu_reports_device_error():
    # Arguments are valid, so validation passes and the device check must refuse: there
    # is no CPU fallback.
    a = fwd_args()
    rc = ta.load().attn_fwd(a["q"], a["k"], a["v"], a["out"], a["lse"], a["B"], a["Hq"], a["Hkv"],
                            a["Lq"], a["Lk"], a["D"], a["scale"], a["causal"], a["dtype"], None)
    assert rc == -4
    assert ta.load().attn_get_device_status(None) == -4


def test_empty_problems_are_noops_with_null_pointers():
    lib = ta.load()
    # B == 0 or Lq == 0: nothing to do, every pointer may be NULL (returns before any
    # device access, so this is safe on any host)
    assert lib.attn_fwd(None, None, None, None, None, 0, 2, 1, 8, 8, 64, 0.1, 1, 0, None) == 0
    assert lib.attn_fwd(None, None, None, None, None, 1, 2, 1, 0, 8, 64, 0.1, 1, 0, None) == 0
    assert lib.attn_fwd_paged(None, None, None, None, None, 16, None, None, 0, 12, 2, 128, 256,
                              10, 0.1, 1, None, 0, None) == 0


def test_workspace_size():
    ws = ta.paged_workspace_size
    assert ws(16, 12, 2, 128, 1) == 0          # one block per sequence: never split, no workspace
    # 32 units -> 296 CTAs (chunks); counters + per-chunk lse + per-chunk O, each 256-B aligned
    grid, G = 296, 6
    expect = 256 + (grid * G * 4 + 255) // 256 * 256 + (grid * G * 128 * 4 + 255) // 256 * 256
    assert ws(16, 12, 2, 128, 256) == expect
    # more units than half the default grid: two chunks per unit on average
    assert ws(320, 32, 2, 128, 256) > ws(16, 32, 2, 128, 256)
    assert ws(16, 12, 2, 128, 256, 32) == 0    # unsupported block size -> 0
    assert ws(0, 12, 2, 128, 256) == 0
    assert ws(1, 4, 4, 64, 9) > 0
    assert ws(1024, 8, 2, 128, 256) == 0       # > 1024 units: one CTA per unit, no split


def bwd_args(**kw):
    a = dict(q=P, k=P, v=P, out=P, dout=P, lse=P, dq=P, dk=P, dv=P, B=1, Hq=2, Hkv=1, Lq=8, Lk=8,
             D=64, scale=0.125, causal=0, dtype=0, ws=P, ws_n=1 << 20, stream=None)
    a.update(kw)
    return a


BWD_BAD = [
    ("null_dout", dict(dout=None), -1),
    ("null_lse", dict(lse=None), -1),
    ("null_dq", dict(dq=None), -1),
    ("null_dk", dict(dk=None), -1),
    ("neg_Lk", dict(Lk=-1), -1),
    ("group_not_divisible", dict(Hq=3, Hkv=2), -1),
    ("scale_nan", dict(scale=float("nan")), -1),
    ("D_32", dict(D=32), -2),
    ("dtype_fp32", dict(dtype=7), -2),
    ("misaligned_dout", dict(dout=P + 2), -3),
    ("misaligned_dv", dict(dv=P + 8), -3),
    ("misaligned_lse", dict(lse=P + 1), -3),
    ("workspace_missing", dict(ws=None, ws_n=0), -7),
    ("workspace_small", dict(ws_n=8 * 2 * 128 - 1), -7),
]


def call_bwd(a, window=None):
    lib = ta.load()
    args = (a["q"], a["k"], a["v"], a["out"], a["dout"], a["lse"], a["dq"], a["dk"], a["dv"],
            a["B"], a["Hq"], a["Hkv"], a["Lq"], a["Lk"], a["D"], a["scale"], a["causal"])
    if window is None:
        return lib.attn_bwd(*args, a["dtype"], a["ws"], a["ws_n"], a["stream"])
    return lib.attn_bwd_window(*args, window[0], window[1], a["dtype"], a["ws"], a["ws_n"],
                               a["stream"])


@pytest.mark.parametrize("name,kw,code", BWD_BAD, ids=[c[0] for c in BWD_BAD])
def test_attn_bwd_validation(name, kw, code):
    rc = call_bwd(bwd_args(**kw))
    assert rc == code, (rc, ta.STATUS.get(rc))


def test_attn_bwd_window_validation():
    assert call_bwd(bwd_args(), window=(-2, 3)) == -1
    assert call_bwd(bwd_args(), window=(3, -5)) == -1
    assert call_bwd(bwd_args(D=80), window=(3, 3)) == -2


def test_attn_bwd_strided_validation():
    lib = ta.load()
    S = ta.Strides

    def call(st=(None,) * 8, **kw):
        a = bwd_args(**kw)
        return lib.attn_bwd_strided(a["q"], st[0], a["k"], st[1], a["v"], st[2], a["out"], st[3],
                                    a["dout"], st[4], a["lse"], a["dq"], st[5], a["dk"], st[6],
                                    a["dv"], st[7], a["B"], a["Hq"], a["Hkv"], a["Lq"], a["Lk"],
                                    a["D"], a["scale"], a["causal"], -1, -1, a["dtype"], a["ws"],
                                    a["ws_n"], a["stream"])
    bad_row = S(8 * 64 * 2, 64, 64 * 2 + 4)                       # 16-byte rule broken
    for i in range(8):                                            # every tensor's strides checked
        st = [None] * 8
        st[i] = bad_row
        assert call(st=st) == -3, i
    assert call(st=[None] * 6 + [S(-8, 512, 64), None], B=2) == -1   # negative dk stride
    assert call(st=[S(1 << 38, 512, 64)] + [None] * 7, B=2) == -1    # oversized q view
    assert call(ws_n=16) == -7                                       # strides do not excuse it
    assert call(st=[S(0, 0, 0)] * 8, B=1, Hq=1, Hkv=1, Lq=1, Lk=1, D=96) == -2


def test_bwd_empty_problems_and_workspace_size():
    lib = ta.load()
    # B == 0, or no queries and no keys: nothing to write, pointers may be NULL
    assert lib.attn_bwd(None, None, None, None, None, None, None, None, None, 0, 2, 1, 8, 8, 64,
                        0.1, 1, 0, None, 0, None) == 0
    assert lib.attn_bwd(None, None, None, None, None, None, None, None, None, 1, 2, 1, 0, 0, 64,
                        0.1, 1, 0, None, 0, None) == 0
    ws = ta.bwd_workspace_size
    assert ws(1, 16, 8192) == 8 * 16 * 8192
    assert ws(2, 3, 1) == 8 * 6 * 128          # rows padded to a multiple of 128
    assert ws(32, 12, 196) == 8 * 384 * 256
    assert ws(0, 4, 100) == 0 and ws(1, 4, 0) == 0


def test_attn_fwd_strided_validation():
    lib = ta.load()
    S = ta.Strides

    def call(qs=None, ks=None, vs=None, os_=None, **kw):
        a = fwd_args(**kw)
        return lib.attn_fwd_strided(a["q"], qs, a["k"], ks, a["v"], vs, a["out"], os_, a["lse"],
                                    a["B"], a["Hq"], a["Hkv"], a["Lq"], a["Lk"], a["D"],
                                    a["scale"], a["causal"], -1, -1, a["dtype"], None)
    assert call(qs=S(8 * 64 * 2, 64, 64 * 2 + 4)) == -3          # seq stride not a multiple of 8
    assert call(ks=S(-8, 512, 64), B=2) == -1                    # negative stride of a used dim
    assert call(os_=S(1 << 38, 512, 64), B=2) == -1              # oversized
    assert call(qs=S(0, 0, 0), B=1, Hq=1, Hkv=1, Lq=1, D=96) == -2  # unused strides; D refused


def test_attn_fwd_paged_prefill_validation():
    lib = ta.load()

    def call(**kw):
        a = dict(q=P, kc=P, vc=P, bt=P, sl=P, ql=None, bs=16, out=P, lse=P, S=2, Hq=4, Hkv=2,
                 Lq=64, D=128, MB=8, NB=16, scale=0.088, causal=1, dtype=1)
        a.update(kw)
        return lib.attn_fwd_paged_prefill(a["q"], None, a["kc"], a["vc"], a["bt"], a["sl"], a["ql"],
                                          a["bs"], a["out"], None, a["lse"], a["S"], a["Hq"],
                                          a["Hkv"], a["Lq"], a["D"], a["MB"], a["NB"], a["scale"],
                                          a["causal"], a["dtype"], None)
    assert call(sl=None) == -1
    assert call(bt=None) == -1
    assert call(Hq=3) == -1
    assert call(NB=0) == -1
    assert call(bs=32) == -2
    assert call(D=80) == -2
    assert call(bt=P + 2) == -3
    assert call(ql=P + 1) == -3
    assert call(S=0, q=None, out=None) == 0      # nothing to do: NULL pointers allowed


def test_attn_fwd_fp8_validation():
    lib = ta.load()
    S = ta.Strides

    def call(qs=None, D=128, scale=0.088, dq=1.0, dk=1.0, dv=1.0, **kw):
        a = fwd_args(**kw)
        return lib.attn_fwd_fp8(a["q"], qs, a["k"], None, a["v"], None, a["out"], None, a["lse"],
                                a["B"], a["Hq"], a["Hkv"], a["Lq"], a["Lk"], D, scale, dq, dk, dv,
                                a["causal"], None)
    assert call(D=64) == -2                        # 8-bit path: D = 128 only
    assert call(dv=0.0) == -1
    assert call(dq=float("nan")) == -1
    assert call(q=None) == -1
    assert call(qs=S(16 * 128, 8 * 128, 136)) == -3  # 136-byte rows: not a multiple of 16


def test_binding_refuses_tensors_off_the_current_device(monkeypatch):
    """The library launches on the calling thread's current device: the binding checks
    every tensor's and stream's device against it before any call."""
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    ta._on_current_device(torch.device("cuda", 0), "q")          # the current device: fine
    with pytest.raises(ValueError, match="cuda:1"):
        ta._on_current_device(torch.device("cuda", 1), "k")
    with pytest.raises(ValueError, match="CUDA tensor"):        # host tensors never get that far
        ta.fwd(torch.zeros(1, 1, 8, 64), torch.zeros(1, 1, 8, 64), torch.zeros(1, 1, 8, 64))
