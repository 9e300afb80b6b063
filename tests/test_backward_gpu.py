"""Parity of the attention backward pass (attn_bwd, attn_bwd_window) with the fp64 oracle.

The forward pass runs on the GPU (attn_fwd / attn_fwd_window) and its O and lse feed
the backward pass, as in training; the oracle computes dQ, dK, dV from q, k, v and dO
alone, by the chain rule through the definition.

Tolerance. The pages give none for gradients; this one follows from the rounding the
kernels do. They round P and dS to the input dtype (relative error u = 2^-9 for bf16,
2^-11 for f16) before the tensor-core products that form dV, dK and dQ. They compute
delta_i = dO_i . O_i from the rounded output. They accumulate in fp32 and round each
gradient to the dtype (another u). To first order every gradient element g is then
off by at most u (m + |g|). Here m is the element's rounding sensitivity, which the
oracle returns beside the gradient (for dQ_i: scale sum_j (|dS_ij| + P_ij sum_d
|dO_id O_id|) |k_j|). fp32 accumulation over up to 8192 terms adds at most about
2^-11 m. So each element is checked against
    |g_gpu - g_ref| <= 3 u (m + |g_ref|).
A second check does not use the kernel's rounding model at all: per gradient tensor, the
relative Frobenius error ||g_gpu - g_ref|| / ||g_ref|| must stay within 2u. The rounding
errors of P, dS and the stored gradient are each at most u in relative terms and, on
these random inputs, independent from element to element, so the error norm stays near u
of the gradient's norm (measured 0.6u for f16 and 1.2-1.3u for bf16 on every case here,
the long prefill included).
"""
from __future__ import annotations

import math

import pytest
import torch

import oracle
import tiled_attention_19_b200 as ta
from tiled_attention_19_b200 import inputs
from tests.parity import check_grad, guarded_empty, guards_intact

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
def check_frobenius(got, ref, dtype, what):
    """||got - ref||_F <= 2u ||ref||_F, u the dtype's unit roundoff. A gradient that is
    exactly zero (one visible key per row: dS = 0) has no relative error to speak of; the
    per-element bound covers it."""
    g = got.detach().to("cpu", torch.float64)
    r = ref.to(torch.float64)
    n = float(r.norm())
    if n == 0.0:
        return
    e = float((g - r).norm())
    u = 2.0 ** -11 if dtype == torch.float16 else 2.0 ** -9
    assert e <= 2 * u * n + 1e-30, f"{what}: relative Frobenius error {e / n:.3e} > 2u = {2 * u:.3e}"


def run_case(B, Hq, Hkv, Lq, Lk, D, dtype, causal, window, seed):
    s = inputs.DenseSpec("bwd", B, Hq, Hkv, Lq, Lk, D, dtype, causal, 1 / math.sqrt(D), seed)
    x = inputs.make(s)
    do = inputs.dense_grad_output(s)
    q, k, v = (x[n].to(DEV) for n in ("q", "k", "v"))
    dout = do.to(DEV)
    out, lse = ta.fwd(q, k, v, causal=causal, scale=s.scale, window=window)
    qb, dq, qg = guarded_empty((B, Hq, Lq, D), dtype, DEV)
    kb, dk, kg = guarded_empty((B, Hkv, Lk, D), dtype, DEV)
    vb, dv, vg = guarded_empty((B, Hkv, Lk, D), dtype, DEV)
    ta.bwd(q, k, v, out, dout, lse, causal=causal, scale=s.scale, window=window, dq=dq, dk=dk,
           dv=dv)
    torch.cuda.synchronize()
    assert guards_intact(qb, qg) and guards_intact(kb, kg) and guards_intact(vb, vg)
    assert ta.device_status() == 0
    return s, x, do, (dq, dk, dv)


CASES = [
    # B, Hq, Hkv, Lq, Lk, D, dtype, causal, window
    (1, 2, 2, 300, 300, 64, torch.float16, False, None),
    (1, 2, 2, 300, 300, 128, torch.bfloat16, True, None),
    (2, 4, 2, 200, 333, 64, torch.bfloat16, True, None),     # grouped heads, Lq < Lk
    (1, 2, 1, 260, 130, 128, torch.float16, True, None),      # Lq > Lk: rows that see no key
    (1, 1, 1, 1, 1, 64, torch.float16, False, None),
    (1, 2, 2, 65, 129, 128, torch.bfloat16, False, None),     # ragged sub-tiles and tiles
    (1, 3, 3, 512, 512, 128, torch.float16, False, None),
    (1, 4, 1, 256, 256, 64, torch.float16, True, None),       # group of 4
    (1, 2, 2, 400, 400, 64, torch.bfloat16, False, (64, 32)),
    (1, 2, 1, 333, 333, 128, torch.float16, True, (100, -1)),
    (1, 2, 2, 300, 300, 128, torch.bfloat16, False, (0, 0)),  # each row sees one key
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B{}_H{}-{}_Lq{}_Lk{}_D{}_{}_{}_w{}".format(
    *c[:6], str(c[6]).split(".")[-1], "causal" if c[7] else "full", c[8]))
def test_backward_parity(case):
    B, Hq, Hkv, Lq, Lk, D, dtype, causal, window = case
    s, x, do, got = run_case(*case, seed=11 * Lq + Lk + D)
    ref = oracle.attn_bwd(x["q"], x["k"], x["v"], do, s.scale, causal,
                          window if window is not None else (-1, -1), sensitivity=True)
    for i, name in enumerate(("dq", "dk", "dv")):
        check_grad(got[i], ref[i], ref[3 + i], dtype, f"{case} {name}")
        check_frobenius(got[i], ref[i], dtype, f"{case} {name}")


@pytest.mark.parametrize("case", [
    (1, 4, 2, 333, 333, 128, torch.bfloat16, True, None),
    # windows whose dQ tiles stream three key sub-tiles: the softmax warps of one tile may
    # drift a sub-tile apart there, which the dS hand-off to the MMA must tolerate
    (1, 2, 2, 400, 400, 64, torch.bfloat16, False, (64, 32)),
    (1, 4, 2, 400, 400, 128, torch.float16, False, (64, 16)),
], ids=["causal_gqa", "window_d64", "window_gqa_d128"])
def test_backward_is_deterministic(case):
    runs = [run_case(*case, seed=3)[3] for _ in range(3)]
    for other in runs[1:]:
        for t, u in zip(runs[0], other):
            assert torch.isfinite(t).all()
            assert torch.equal(t, u)


def test_backward_empty_sides():
    q = torch.randn(1, 2, 5, 64, device=DEV).to(torch.float16)
    k = torch.empty(1, 1, 0, 64, device=DEV, dtype=torch.float16)
    out, lse = ta.fwd(q, k, k, causal=False)
    dq = torch.full_like(q, 3.0)
    ta.bwd(q, k, k, out, torch.ones_like(q), lse, dq=dq, dk=k.clone(), dv=k.clone())
    torch.cuda.synchronize()
    assert torch.count_nonzero(dq) == 0          # no keys: dQ = 0
    q0 = torch.empty(1, 2, 0, 64, device=DEV, dtype=torch.float16)
    kk = torch.randn(1, 1, 7, 64, device=DEV).to(torch.float16)
    dk = torch.full_like(kk, 3.0)
    dv = torch.full_like(kk, 3.0)
    lse0 = torch.empty(1, 2, 0, device=DEV)
    ta.bwd(q0, kk, kk, q0, q0, lse0, dq=q0.clone(), dk=dk, dv=dv)
    torch.cuda.synchronize()
    assert torch.count_nonzero(dk) == 0 and torch.count_nonzero(dv) == 0  # no queries
    assert ta.device_status() == 0


def test_backward_long_causal_prefill_all():
    """The long causal prefill workload (B1 H16 L8192 D128 bf16) end to end on the GPU:
    every element of dQ, dK and dV against the oracle's full backward pass (about a
    minute of host time on 16 cores), under the per-element bound."""
    s = inputs.WORKLOADS["prefill_causal_b1_h16_l8192_d128_bf16"]
    x = inputs.make(s)
    do = inputs.dense_grad_output(s)
    q, k, v = (x[n].to(DEV) for n in ("q", "k", "v"))
    out, lse = ta.fwd(q, k, v, causal=True, scale=s.scale)
    dq, dk, dv = ta.bwd(q, k, v, out, do.to(DEV), lse, causal=True, scale=s.scale)
    torch.cuda.synchronize()
    assert ta.device_status() == 0
    ref = oracle.attn_bwd(x["q"], x["k"], x["v"], do, s.scale, True, sensitivity=True)
    for i, (name, got) in enumerate((("dq", dq), ("dk", dk), ("dv", dv))):
        check_grad(got.cpu(), ref[i], ref[3 + i], s.dtype, f"long causal prefill {name}, all")
        check_frobenius(got, ref[i], s.dtype, f"long causal prefill {name}")
