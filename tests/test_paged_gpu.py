"""Parity of attn_fwd_paged (paged-KV decode kernel) with the fp64 oracle, on the GPU.

Calls go through the C ABI (ctypes). The decode workload is compared on every output;
a sweep covers sequence lengths around the 16-token block and the 128-token chunk
edges, empty sequences, group sizes 1..16, both head dims and both dtypes. Out-of-range
block-table entries and sequence lengths must be caught by the kernel's own checks and
reported through the status word.
"""
from __future__ import annotations

import math

import pytest
import torch

import oracle
import tiled_attention_19_b200 as ta
from tiled_attention_19_b200 import inputs
from tests.parity import check_parity, guarded_empty, guards_intact

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def to_dev(x):
    return {k: v.to(DEV) for k, v in x.items()}


def run_paged(x, scale, guard=False, workspace=None):
    d = to_dev(x)
    S, Hq, D = x["q"].shape
    if guard:
        ob, out, og = guarded_empty((S, Hq, D), x["q"].dtype, DEV)
        lb, lse, lg = guarded_empty((S, Hq), torch.float32, DEV)
        ta.fwd_paged(d["q"], d["k_cache"], d["v_cache"], d["block_table"], d["seq_lens"],
                     scale=scale, out=out, lse=lse, workspace=workspace)
        torch.cuda.synchronize()
        assert guards_intact(ob, og) and guards_intact(lb, lg)
    else:
        out, lse = ta.fwd_paged(d["q"], d["k_cache"], d["v_cache"], d["block_table"],
                                d["seq_lens"], scale=scale, workspace=workspace)
        torch.cuda.synchronize()
    return out.cpu(), lse.cpu()


def test_decode_workload_all_outputs():
    s = inputs.WORKLOADS["paged_decode_s16_hq12_hkv2_d128_bf16"]
    x = inputs.make(s)
    out, lse = run_paged(x, s.scale, guard=True)
    assert ta.device_status() == 0
    ro, rl = oracle.attn_paged(x["q"], x["k_cache"], x["v_cache"], x["block_table"],
                               x["seq_lens"], s.scale)
    check_parity(out, lse, ro, rl, s.dtype, "decode workload")


LENS = (0, 1, 15, 16, 17, 127, 128, 129, 255, 256, 257, 1000, 4096)
CASES = [
    (12, 2, 128, torch.bfloat16),
    (8, 8, 64, torch.float16),
    (16, 1, 128, torch.float16),
    (4, 2, 64, torch.bfloat16),
    (3, 3, 128, torch.bfloat16),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"Hq{c[0]}_Hkv{c[1]}_D{c[2]}_{str(c[3]).split('.')[-1]}")
def test_decode_length_sweep(case):
    Hq, Hkv, D, dtype = case
    s = inputs.PagedSpec("t", len(LENS), Hq, Hkv, D, 16, 4096, dtype, 1 / math.sqrt(D),
                         seed=D + Hq, fixed_lens=LENS)
    x = inputs.make(s)
    out, lse = run_paged(x, s.scale, guard=True)
    assert ta.device_status() == 0
    ro, rl = oracle.attn_paged(x["q"], x["k_cache"], x["v_cache"], x["block_table"],
                               x["seq_lens"], s.scale)
    check_parity(out, lse, ro, rl, dtype, str(case))


def test_workspace_reused_and_left_clean():
    s = inputs.WORKLOADS["paged_decode_s16_hq12_hkv2_d128_bf16"]
    x = inputs.make(s)
    n = ta.paged_workspace_size(s.num_seqs, s.Hq, s.Hkv, s.D, s.max_blocks)
    ws = torch.zeros(n, dtype=torch.uint8, device=DEV)
    o1, l1 = run_paged(x, s.scale, workspace=ws)
    o2, l2 = run_paged(x, s.scale, workspace=ws)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    # the completion counters (first bytes of the workspace) are back at zero
    assert torch.all(ws[: 4 * s.num_seqs * s.Hkv] == 0)


def test_bad_table_entry_is_reported_not_faulted():
    s = inputs.PagedSpec("t", 2, 4, 1, 64, 16, 256, torch.float16, 0.125, seed=3,
                         fixed_lens=(200, 40))
    x = inputs.make(s)
    x["block_table"][0, 3] = s.num_blocks + 5   # out of range
    x["block_table"][1, 1] = -1                 # negative
    run_paged(x, s.scale)
    assert ta.device_status() == -8
    assert ta.device_status() == 0              # reading clears it


def test_bad_seq_len_is_reported_not_faulted():
    s = inputs.PagedSpec("t", 2, 4, 1, 64, 16, 256, torch.float16, 0.125, seed=4,
                         fixed_lens=(10, 20))
    x = inputs.make(s)
    x["seq_lens"][1] = 10 ** 6  # past the table
    run_paged(x, s.scale)
    assert ta.device_status() == -8


def test_decode_skewed_lengths_balanced_schedule():
    # one long sequence among many short and empty ones: the long one is cut into many
    # chunks merged through the workspace, the short ones finish in one chunk
    lens = (4096,) + (0, 1, 3, 16, 17) * 6 + (31,)
    s = inputs.PagedSpec("t", len(lens), 8, 2, 128, 16, 4096, torch.bfloat16, 1 / math.sqrt(128),
                         seed=31, fixed_lens=lens)
    x = inputs.make(s)
    out, lse = run_paged(x, s.scale, guard=True)
    assert ta.device_status() == 0
    ro, rl = oracle.attn_paged(x["q"], x["k_cache"], x["v_cache"], x["block_table"],
                               x["seq_lens"], s.scale)
    check_parity(out, lse, ro, rl, s.dtype, "skewed")


def test_decode_one_sequence_of_a_million_tokens():
    """One sequence of 2^20 tokens (65,536 blocks through the table) and one of 5 tokens,
    H_q 8 / H_kv 1: the long unit is cut into about 290 chunks, too many partial outputs
    to stage in shared memory, so its merge reads them from L2; the other unit has one
    chunk and writes directly."""
    lens = (1 << 20, 5)
    s = inputs.PagedSpec("t", 2, 8, 1, 128, 16, 1 << 20, torch.bfloat16, 1 / math.sqrt(128),
                         seed=33, fixed_lens=lens)
    x = inputs.make(s)
    out, lse = run_paged(x, s.scale, guard=True)
    assert ta.device_status() == 0
    ro, rl = oracle.attn_paged(x["q"], x["k_cache"], x["v_cache"], x["block_table"],
                               x["seq_lens"], s.scale)
    check_parity(out, lse, ro, rl, s.dtype, "one long sequence")


def test_decode_many_units_one_cta_each():
    # more than 1024 (sequence, K/V head) units: each CTA takes a whole unit, no split
    s = inputs.PagedSpec("t", 520, 4, 2, 64, 16, 160, torch.float16, 0.125, seed=32, min_len=0)
    assert s.num_seqs * s.Hkv > 1024
    assert ta.paged_workspace_size(s.num_seqs, s.Hq, s.Hkv, s.D, s.max_blocks) == 0
    x = inputs.make(s)
    out, lse = run_paged(x, s.scale, guard=True)
    assert ta.device_status() == 0
    ro, rl = oracle.attn_paged(x["q"], x["k_cache"], x["v_cache"], x["block_table"],
                               x["seq_lens"], s.scale)
    check_parity(out, lse, ro, rl, s.dtype, "many units")


def test_rows_past_the_sequence_end_are_masked_even_if_nan():
    """Cache rows of a sequence's last block past its length are read with the block but
    must weigh nothing, whatever they hold: fill them with NaN in K and V."""
    s = inputs.PagedSpec("t", 4, 12, 2, 128, 16, 512, torch.bfloat16, 1 / math.sqrt(128), seed=31,
                         fixed_lens=(1, 17, 130, 511))
    x = inputs.make(s)
    for sq, n in enumerate(s.fixed_lens):
        blk = int(x["block_table"][sq][(n - 1) // 16])
        x["k_cache"][blk, :, n % 16 or 16:] = float("nan")
        x["v_cache"][blk, :, n % 16 or 16:] = float("nan")
    out, lse = run_paged(to_dev(x), s.scale)
    torch.cuda.synchronize()
    assert ta.device_status() == 0
    ro, rl = oracle.attn_paged(x["q"], x["k_cache"], x["v_cache"], x["block_table"],
                               x["seq_lens"], s.scale)
    check_parity(out.cpu(), lse.cpu(), ro, rl, s.dtype, "nan rows past the end")
