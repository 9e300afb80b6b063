"""attn_fwd_paged_noalloc: paged decode for callers that cannot allocate device memory.

Such a caller (for example a plugin handed only its input and output buffers by a host
framework that owns the allocator) cannot provide the split-KV workspace that
attn_fwd_paged takes. The no-allocation entry point uses a fixed 4 MiB scratch array
inside the library instead. These tests call it through the C ABI and check that two
calls in a row match the fp64 oracle and attn_fwd_paged with a caller workspace, within
the parity tolerances, that a call after the array was overwritten with junk (as an
interrupted call can leave it) still matches the oracle, and that a problem too large
for the fixed array is refused.

This file is collected last on purpose; it must pass both on its own in a fresh
process and after every other test.
"""
from __future__ import annotations

import ctypes

import pytest
import torch

import oracle
import tiled_attention_19_b200 as ta
from tiled_attention_19_b200 import inputs
from tests.parity import LSE_REL, O_TOL, check_parity

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
SCRATCH_LIMIT = 4 << 20


def call_noalloc(x, s, out, lse):
    lib = ta.load()
    rc = lib.attn_fwd_paged_noalloc(
        x["q"].data_ptr(), x["k_cache"].data_ptr(), x["v_cache"].data_ptr(),
        x["block_table"].data_ptr(), x["seq_lens"].data_ptr(), s.block_size, out.data_ptr(),
        lse.data_ptr(), s.num_seqs, s.Hq, s.Hkv, s.D, s.max_blocks, s.num_blocks,
        ctypes.c_float(s.scale), 1 if s.dtype == torch.bfloat16 else 0,
        torch.cuda.current_stream().cuda_stream)
    return rc


@pytest.mark.parametrize("name", ["paged_decode_s16_hq12_hkv2_d128_bf16", "short_f16"])
def test_noalloc_matches_workspace_entry_point(name):
    if name == "short_f16":
        s = inputs.PagedSpec("short", 5, 8, 2, 64, 16, 1024, torch.float16, 0.125, seed=21,
                             fixed_lens=(0, 1, 129, 700, 1024))
    else:
        s = inputs.WORKLOADS[name]
    need = ta.paged_workspace_size(s.num_seqs, s.Hq, s.Hkv, s.D, s.max_blocks)
    assert 0 < need <= SCRATCH_LIMIT
    xh = inputs.make(s)
    x = {k: v.to(DEV) for k, v in xh.items()}
    oro, orl = oracle.attn_paged(xh["q"], xh["k_cache"], xh["v_cache"], xh["block_table"],
                                 xh["seq_lens"], s.scale)
    ref_out, ref_lse = ta.fwd_paged(x["q"], x["k_cache"], x["v_cache"], x["block_table"],
                                    x["seq_lens"], scale=s.scale)
    for _ in range(2):  # two calls in a row share (and must leave clean) the scratch
        out = torch.full_like(ref_out, 7.0)
        lse = torch.full_like(ref_lse, 7.0)
        assert call_noalloc(x, s, out, lse) == 0
        torch.cuda.synchronize()
        assert ta.device_status() == 0
        check_parity(out, lse, oro, orl, s.dtype, f"{name} no-alloc vs oracle")
        err = (out.double() - ref_out.double()).abs().max().item()
        assert err <= O_TOL[s.dtype], err
        fin = torch.isfinite(ref_lse)
        assert torch.equal(torch.isfinite(lse), fin)
        assert torch.all(lse[~fin] == ref_lse[~fin])
        rel = ((lse[fin] - ref_lse[fin]).abs() / ref_lse[fin].abs().clamp_min(1.0)).max().item()
        assert rel <= LSE_REL, rel


@pytest.mark.parametrize("fill", [0x07, 0xFF])
def test_noalloc_does_not_depend_on_what_the_scratch_held(fill):
    # An interrupted call can leave the completion counters non-zero and stale partials
    # in the fixed array. Every byte is overwritten first (0x07070707 or -1 as counters):
    # without the per-call counter clear no CTA would see its unit's count complete and
    # no split sequence would be merged.
    s = inputs.WORKLOADS["paged_decode_s16_hq12_hkv2_d128_bf16"]
    xh = inputs.make(s)
    x = {k: v.to(DEV) for k, v in xh.items()}
    oro, orl = oracle.attn_paged(xh["q"], xh["k_cache"], xh["v_cache"], xh["block_table"],
                                 xh["seq_lens"], s.scale)
    lib = ta.load()
    stream = torch.cuda.current_stream().cuda_stream
    for _ in range(2):
        assert lib.attn_selftest_fill_noalloc_scratch(fill, stream) == 0
        out = torch.full((s.num_seqs, s.Hq, s.D), 7.0, dtype=s.dtype, device=DEV)
        lse = torch.full((s.num_seqs, s.Hq), 7.0, device=DEV)
        assert call_noalloc(x, s, out, lse) == 0
        torch.cuda.synchronize()
        assert ta.device_status() == 0
        check_parity(out, lse, oro, orl, s.dtype, f"no-alloc after filling the scratch with {fill:#x}")


def test_noalloc_refuses_problems_past_the_scratch_limit():
    # 160 sequences with 32 query heads over 2 K/V heads need about 5.3 MB of scratch:
    # refused before anything is enqueued (no kernel runs, so the pointers are never read).
    s = inputs.PagedSpec("big", 160, 32, 2, 128, 16, 4096, torch.bfloat16, 0.088, seed=22)
    assert ta.paged_workspace_size(s.num_seqs, s.Hq, s.Hkv, s.D, s.max_blocks) > SCRATCH_LIMIT
    q = torch.empty(s.num_seqs, s.Hq, s.D, dtype=s.dtype, device=DEV)
    cache = torch.empty(16, s.Hkv, 16, s.D, dtype=s.dtype, device=DEV)
    bt = torch.zeros(s.num_seqs, s.max_blocks, dtype=torch.int32, device=DEV)
    sl = torch.zeros(s.num_seqs, dtype=torch.int32, device=DEV)
    out = torch.empty_like(q)
    lse = torch.empty(s.num_seqs, s.Hq, device=DEV)
    x = {"q": q, "k_cache": cache, "v_cache": cache, "block_table": bt, "seq_lens": sl}
    rc = call_noalloc(x, s, out, lse)
    assert rc == -9 and ta.STATUS[rc] == "ATTN_ERR_SCRATCH_LIMIT"
