"""Parity of the FP8 forward (attn_fwd_fp8) with the fp64 oracle, on the GPU.

The "Flash Attention" skill page, Scenario 3, casts q, k, v to float8_e4m3fn and runs
the forward pass in 8 bits. The oracle computes the definition on the exact e4m3
values (times the descale factors) in fp64.

Tolerance. The kernel's products are exact (8-bit operands, fp32 accumulation). It
rounds the attention weights P to e4m3 before P.V: relative error up to u = 2^-4 per
weight in the normal range, and an absolute error up to 2^-10 of the reference weight
for weights below e4m3's smallest normal (2^-6). Then it rounds O to bf16. So each
element is held to
    |O_gpu - O_ref| <= 2u m + 2^-8 |O_ref| + 2^-7,
with m = sum_j P_ij |v_jd| (the oracle on |V|) and the last term covering the
sub-normal weights. Per (batch, head) the relative Frobenius error must also stay below
u, which a wrong tile or mask would break. lse uses the unrounded fp32 weights and keeps
the 16-bit path's bound, 1e-4 * max(1, |lse|).
"""
from __future__ import annotations

import math

import pytest
import torch

import oracle
import tiled_attention_19_b200 as ta
from tiled_attention_19_b200 import inputs

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
U8 = 2.0 ** -4


def fp8_inputs(B, Hq, Hkv, Lq, Lk, D, seed, spread=1.0):
    g = torch.Generator().manual_seed(seed)
    q = (torch.randn(B, Hq, Lq, D, generator=g) * spread).to(torch.float8_e4m3fn)
    k = (torch.randn(B, Hkv, Lk, D, generator=g) * spread).to(torch.float8_e4m3fn)
    v = (torch.randn(B, Hkv, Lk, D, generator=g) * spread).to(torch.float8_e4m3fn)
    return q, k, v


def check_fp8(out, lse, q, k, v, scale, causal, descale, what):
    dq, dk, dv = descale
    q64, k64, v64 = (t.to(torch.float64) * d for t, d in ((q, dq), (k, dk), (v, dv)))
    ro, rl = oracle.attn_fwd(q64, k64, v64, scale, causal)
    m, _ = oracle.attn_fwd(q64, k64, v64.abs(), scale, causal)
    o = out.detach().to("cpu", torch.float64)
    assert torch.isfinite(o).all(), what
    err = (o - ro).abs()
    bound = 2 * U8 * m + 2.0 ** -8 * ro.abs() + 2.0 ** -7
    assert bool((err <= bound).all()), f"{what}: max err/bound {float((err / bound).max()):.3f}"
    num = err.pow(2).sum(dim=(-1, -2)).sqrt()
    den = ro.pow(2).sum(dim=(-1, -2)).sqrt().clamp_min(1e-30)
    rel = float((num / den).max())
    assert rel <= U8, f"{what}: relative Frobenius error {rel:.3e}"
    print(f"{what}: max err/bound {float((err / bound).max()):.3f}, relative Frobenius error {rel:.3e}")
    lg = lse.detach().to("cpu", torch.float64)
    fin = torch.isfinite(rl)
    assert torch.equal(torch.isfinite(lg), fin)
    if fin.any():
        lrel = float(((lg[fin] - rl[fin]).abs() / rl[fin].abs().clamp_min(1.0)).max())
        assert lrel <= 1e-4, f"{what}: lse error {lrel:.3e}"
    return rel


CASES = [
    # B, Hq, Hkv, Lq, Lk, causal, descale
    (1, 2, 2, 300, 300, False, (1.0, 1.0, 1.0)),
    (1, 4, 2, 513, 513, True, (1.0, 1.0, 1.0)),
    (2, 3, 1, 200, 700, True, (0.5, 2.0, 0.25)),     # Lq < Lk, grouped heads, descales
    (1, 2, 2, 129, 64, True, (1.0, 1.0, 1.0)),       # Lq > Lk: rows with no key
    (1, 1, 1, 1, 1, False, (1.0, 1.0, 1.0)),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B{}_H{}-{}_Lq{}_Lk{}_{}".format(
    *c[:5], "causal" if c[5] else "full"))
def test_fp8_parity(case):
    B, Hq, Hkv, Lq, Lk, causal, descale = case
    q, k, v = fp8_inputs(B, Hq, Hkv, Lq, Lk, 128, seed=Lq + Lk)
    scale = 1 / math.sqrt(128)
    out, lse = ta.fwd_fp8(q.to(DEV), k.to(DEV), v.to(DEV), causal=causal, scale=scale,
                          descale=descale)
    torch.cuda.synchronize()
    assert ta.device_status() == 0
    check_fp8(out, lse, q, k, v, scale, causal, descale, str(case))


def test_fp8_blhd_layout_matches_contiguous():
    q, k, v = fp8_inputs(2, 4, 4, 257, 257, 128, seed=3)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    ref, ref_lse = ta.fwd_fp8(qd, kd, vd, causal=True)
    qb, kb, vb = (t.transpose(1, 2).contiguous() for t in (qd, kd, vd))
    ob = torch.zeros(2, 257, 4, 128, dtype=torch.bfloat16, device=DEV)
    out, lse = ta.fwd_fp8(qb.transpose(1, 2), kb.transpose(1, 2), vb.transpose(1, 2), causal=True,
                          out=ob.transpose(1, 2))
    torch.cuda.synchronize()
    assert torch.equal(ob.transpose(1, 2), ref) and torch.equal(lse, ref_lse)


def test_fp8_long_causal_prefill_all_rows():
    """The long causal prefill shape (B1 H16 L8192 D128) with e4m3 inputs: every row
    against the oracle on the exact e4m3 values, under the same element bound, plus the
    per-head relative Frobenius bound."""
    s = inputs.WORKLOADS["prefill_causal_b1_h16_l8192_d128_bf16"]
    x = inputs.make(s)
    q, k, v = (x[n].to(torch.float32).to(torch.float8_e4m3fn) for n in ("q", "k", "v"))
    out, lse = ta.fwd_fp8(q.to(DEV), k.to(DEV), v.to(DEV), causal=True, scale=s.scale)
    torch.cuda.synchronize()
    assert ta.device_status() == 0
    check_fp8(out, lse, q, k, v, s.scale, True, (1.0, 1.0, 1.0), "long causal prefill, all rows")
