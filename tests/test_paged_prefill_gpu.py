"""Parity of prefill over a paged KV cache (attn_fwd_paged_prefill) on the GPU.

Each sequence's chunk of queries sits at its last positions and reads its keys through
the block table ("Fast attention kernels and operator fusion", section on
FlashAttention-style and paged attention). Checks:
* a whole-sequence chunk over a scattered cache equals attn_fwd on the gathered dense
  K/V bit for bit (the same tiles reach the same kernel),
* chunks of mixed lengths, grouped heads, both dtypes and head sizes, causal or not,
  element by element against the fp64 oracle,
* empty sequences and chunks, chunks longer than the context, strided q/out,
* a table entry outside the pool is reported (ATTN_ERR_BAD_INDEX) without a fault.
"""
from __future__ import annotations

import math

import pytest
import torch

import oracle
import tiled_attention_19_b200 as ta
from tests.parity import check_parity

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def make_cache(seed, S, Hq, Hkv, Lq, D, dtype, seq_lens, spare_blocks=3):
    g = torch.Generator().manual_seed(seed)
    mb = max(1, max(-(-int(n) // 16) for n in seq_lens))
    nb = S * mb + spare_blocks
    kc = torch.randn(nb, Hkv, 16, D, generator=g).to(dtype)
    vc = torch.randn(nb, Hkv, 16, D, generator=g).to(dtype)
    q = torch.randn(S, Hq, Lq, D, generator=g).to(dtype)
    bt = torch.randperm(nb, generator=g)[:S * mb].reshape(S, mb).to(torch.int32)
    return q, kc, vc, bt, torch.tensor(seq_lens, dtype=torch.int32)


def test_full_sequence_equals_dense_kernel():
    # 40 heads: the dense grid (2 x 40 heads x 4 pairs of query tiles) is more than one
    # wave, so the dense kernel keeps two query tiles per CTA like the paged one and the
    # results must agree bit for bit (a smaller grid splits each tile's key tiles between
    # the softmax warpgroups, which rounds differently).
    S, H, L, D, dtype = 2, 40, 1000, 128, torch.bfloat16
    q, kc, vc, bt, sl = make_cache(1, S, H, H, L, D, dtype, [L, L])
    out, lse = ta.fwd_paged_prefill(q.to(DEV), kc.to(DEV), vc.to(DEV), bt.to(DEV), sl.to(DEV),
                                    causal=True)
    t = torch.arange(L)
    K = torch.stack([kc[bt[s][t // 16].long(), :, t % 16].permute(1, 0, 2) for s in range(S)])
    V = torch.stack([vc[bt[s][t // 16].long(), :, t % 16].permute(1, 0, 2) for s in range(S)])
    ref_out, ref_lse = ta.fwd(q.to(DEV), K.to(DEV), V.to(DEV), causal=True)
    torch.cuda.synchronize()
    assert ta.device_status() == 0
    assert torch.equal(out, ref_out) and torch.equal(lse, ref_lse)


CASES = [
    # S, Hq, Hkv, Lq, D, dtype, causal, seq_lens, q_lens
    (3, 4, 2, 300, 128, torch.bfloat16, True, [700, 300, 1], [300, 129, 1]),
    (2, 8, 8, 256, 64, torch.float16, True, [2048, 257], [256, 200]),
    (4, 6, 1, 130, 64, torch.bfloat16, False, [130, 33, 500, 0], [130, 17, 64, 0]),
    (2, 2, 2, 200, 128, torch.float16, True, [150, 1000], None),    # chunk longer than context
    (1, 4, 4, 513, 128, torch.bfloat16, True, [513], [513]),
    (2, 2, 1, 600, 64, torch.float16, True, [900, 40], [100, 40]),   # CTAs wholly past a chunk
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "S{}_H{}-{}_Lq{}_D{}_{}_{}".format(
    *c[:5], str(c[5]).split(".")[-1], "causal" if c[6] else "full"))
def test_paged_prefill_parity(case):
    S, Hq, Hkv, Lq, D, dtype, causal, seq_lens, q_lens = case
    q, kc, vc, bt, sl = make_cache(Lq + D + S, S, Hq, Hkv, Lq, D, dtype, seq_lens)
    ql = None if q_lens is None else torch.tensor(q_lens, dtype=torch.int32)
    out, lse = ta.fwd_paged_prefill(q.to(DEV), kc.to(DEV), vc.to(DEV), bt.to(DEV), sl.to(DEV),
                                    q_lens=None if ql is None else ql.to(DEV), causal=causal)
    torch.cuda.synchronize()
    assert ta.device_status() == 0
    ro, rl = oracle.attn_paged_prefill(q, kc, vc, bt, sl, 1 / math.sqrt(D), causal, q_lens=ql)
    check_parity(out.cpu(), lse.cpu(), ro, rl, dtype, str(case))


def test_strided_chunk_layout():
    """q and out in the [S, Lq, H, D] layout of flash_attn's varlen-free interface."""
    S, H, Lq, D, dtype = 2, 4, 257, 128, torch.bfloat16
    q, kc, vc, bt, sl = make_cache(5, S, H, H, Lq, D, dtype, [900, 257])
    qb = q.transpose(1, 2).contiguous().to(DEV)               # storage [S, Lq, H, D]
    ob = torch.full_like(qb, 3.0)
    out, lse = ta.fwd_paged_prefill(qb.transpose(1, 2), kc.to(DEV), vc.to(DEV), bt.to(DEV),
                                    sl.to(DEV), causal=True, out=ob.transpose(1, 2))
    torch.cuda.synchronize()
    ro, rl = oracle.attn_paged_prefill(q, kc, vc, bt, sl, 1 / math.sqrt(D), True)
    check_parity(ob.transpose(1, 2).cpu(), lse.cpu(), ro, rl, dtype, "strided")


def test_bad_table_entry_is_reported():
    S, H, Lq, D = 1, 2, 64, 64
    q, kc, vc, bt, sl = make_cache(6, S, H, H, Lq, D, torch.float16, [64])
    bt[0, 1] = kc.shape[0] + 5                                # outside the pool
    ta.device_status()
    out, lse = ta.fwd_paged_prefill(q.to(DEV), kc.to(DEV), vc.to(DEV), bt.to(DEV), sl.to(DEV))
    torch.cuda.synchronize()
    assert ta.device_status() == -8
    assert torch.isfinite(out).all()
