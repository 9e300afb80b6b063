"""Parity of sliding-window attention (attn_fwd_window) with the fp64 oracle, on the GPU.

window_size = (left, right) as in the "Flash Attention" skill page, Scenario 2 step 3:
query i (shifted to i' = i + Lk - Lq) sees keys i'-left .. i'+right, -1 = unbounded, and
causal caps the right side at i'. Windows narrower than a tile, wider than the sequence,
one-sided, with causal, GQA, Lq != Lk and ragged lengths are all compared element by
element; the unbounded window must reproduce attn_fwd exactly (same kernel path).
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

CASES = [
    # B, Hq, Hkv, Lq, Lk, D, dtype, causal, (left, right)
    (1, 2, 2, 700, 700, 64, torch.float16, True, (256, -1)),      # the pages' example, causal
    (1, 2, 1, 700, 700, 128, torch.bfloat16, False, (256, 256)),
    (1, 2, 2, 300, 300, 64, torch.float16, False, (0, 0)),         # each row sees one key
    (1, 2, 2, 300, 300, 128, torch.bfloat16, False, (5, 17)),      # narrower than a tile
    (2, 4, 2, 513, 513, 64, torch.bfloat16, True, (127, -1)),      # tile-edge width
    (1, 2, 2, 257, 257, 128, torch.float16, False, (-1, 40)),      # right bound only
    (1, 2, 2, 257, 257, 64, torch.float16, False, (40, -1)),       # left bound only
    (1, 3, 1, 100, 400, 64, torch.float16, True, (64, -1)),        # Lq < Lk
    (1, 2, 2, 400, 100, 128, torch.bfloat16, False, (10, 10)),     # Lq > Lk: empty rows
    (1, 2, 2, 1000, 1000, 128, torch.bfloat16, True, (5000, -1)),  # wider than the sequence
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "Lq{}_Lk{}_D{}_{}_{}_w{}_{}".format(
    c[3], c[4], c[5], str(c[6]).split(".")[-1], "causal" if c[7] else "full", *c[8]))
def test_window_parity(case):
    B, Hq, Hkv, Lq, Lk, D, dtype, causal, win = case
    s = inputs.DenseSpec("w", B, Hq, Hkv, Lq, Lk, D, dtype, causal, 1 / math.sqrt(D),
                         seed=Lq + 3 * Lk + win[0] + 7)
    x = inputs.make(s)
    q, k, v = (x[n].to(DEV) for n in ("q", "k", "v"))
    ob, out, og = guarded_empty((B, Hq, Lq, D), dtype, DEV)
    lb, lse, lg = guarded_empty((B, Hq, Lq), torch.float32, DEV)
    ta.fwd(q, k, v, causal=causal, scale=s.scale, out=out, lse=lse, window=win)
    torch.cuda.synchronize()
    assert guards_intact(ob, og) and guards_intact(lb, lg)
    assert ta.device_status() == 0
    ro, rl = oracle.attn_fwd_window(x["q"], x["k"], x["v"], s.scale, causal, win)
    check_parity(out.cpu(), lse.cpu(), ro, rl, dtype, str(case))


def test_unbounded_window_is_attn_fwd():
    s = inputs.DenseSpec("w", 1, 4, 2, 333, 333, 128, torch.bfloat16, True, 1 / math.sqrt(128), 5)
    x = inputs.make(s)
    q, k, v = (x[n].to(DEV) for n in ("q", "k", "v"))
    for causal in (False, True):
        o1, l1 = ta.fwd(q, k, v, causal=causal, scale=s.scale)
        o2, l2 = ta.fwd(q, k, v, causal=causal, scale=s.scale, window=(-1, -1))
        torch.cuda.synchronize()
        assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_long_prefill_with_window_sampled_rows():
    # the long prefill shape with the pages' 256-token causal window
    s = inputs.WORKLOADS["prefill_causal_b1_h16_l8192_d128_bf16"]
    x = inputs.make(s)
    q, k, v = (x[n].to(DEV) for n in ("q", "k", "v"))
    out, lse = ta.fwd(q, k, v, causal=True, scale=s.scale, window=(256, -1))
    torch.cuda.synchronize()
    g = torch.Generator().manual_seed(5)
    rows = []
    for h in range(s.Hq):
        picks = [0, 1, 255, 256, 257, 1000, 4095, 8191] + torch.randint(0, s.Lq, (24,), generator=g).tolist()
        rows += [h * s.Lq + i for i in picks]
    # the oracle row by row: with the window (256, causal) row i sees exactly keys
    # max(0, i-256) .. i, so its result is the oracle's unmasked attention over that slice
    outs, lses = [], []
    for r in rows:
        h, i = divmod(r, s.Lq)
        lo = max(0, i - 256)
        o_r, l_r = oracle.attn_fwd(x["q"][:, h:h + 1, i:i + 1], x["k"][:, h:h + 1, lo:i + 1],
                                   x["v"][:, h:h + 1, lo:i + 1], s.scale, False)
        outs.append(o_r.reshape(-1))
        lses.append(l_r.reshape(-1))
    rows_t = torch.tensor(rows)
    check_parity(out.reshape(-1, s.D)[rows_t].cpu(), lse.reshape(-1)[rows_t].cpu(),
                 torch.stack(outs), torch.cat(lses), s.dtype, "long prefill window")
