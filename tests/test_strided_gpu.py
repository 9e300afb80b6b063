"""Parity of attn_fwd_strided (tensors with arbitrary strides over batch, head and
sequence) with the fp64 oracle, on the GPU.

The layouts are flash_attn_func's [B, L, H, D] tensors ("Flash Attention" skill page,
Scenario 2), q/k/v sliced from one packed [B, L, 3, H, D] projection, and an output
written into a slice of a larger buffer. Results must equal the contiguous path's
bit for bit (the same kernel runs; only the addresses differ), and match the oracle.
"""
from __future__ import annotations

import math

import pytest
import torch

import oracle
import tiled_attention_19_b200 as ta
from tiled_attention_19_b200 import inputs
from tests.parity import check_grad, check_parity

pytestmark = pytest.mark.gpu
DEV = "cuda:0"

CASES = [
    # B, Hq, Hkv, Lq, Lk, D, dtype, causal, window
    (2, 4, 2, 300, 300, 128, torch.bfloat16, True, None),
    (1, 8, 8, 513, 513, 64, torch.float16, False, None),
    (3, 6, 2, 130, 257, 64, torch.bfloat16, True, None),
    (1, 4, 4, 400, 400, 128, torch.float16, False, (64, 16)),
]


def dense(case):
    B, Hq, Hkv, Lq, Lk, D, dtype, causal, window = case
    s = inputs.DenseSpec("strided", B, Hq, Hkv, Lq, Lk, D, dtype, causal, 1 / math.sqrt(D),
                         seed=Lq + Lk + D)
    return s, inputs.make(s)


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B{}_H{}-{}_Lq{}_Lk{}_D{}_{}".format(
    *c[:6], "causal" if c[7] else "full"))
def test_blhd_layout(case):
    """flash_attn's layout: q [B, Lq, Hq, D], k/v [B, Lk, Hkv, D], out [B, Lq, Hq, D]."""
    s, x = dense(case)
    window = case[8]
    q, k, v = (x[n].to(DEV) for n in ("q", "k", "v"))
    qb, kb, vb = (t.transpose(1, 2).contiguous() for t in (q, k, v))   # [B, L, H, D] storage
    out_b = torch.full_like(qb, 7.0)
    out, lse = ta.fwd(qb.transpose(1, 2), kb.transpose(1, 2), vb.transpose(1, 2), causal=s.causal,
                      scale=s.scale, out=out_b.transpose(1, 2), window=window)
    ref_out, ref_lse = ta.fwd(q, k, v, causal=s.causal, scale=s.scale, window=window)
    torch.cuda.synchronize()
    assert ta.device_status() == 0
    assert torch.equal(out_b.transpose(1, 2), ref_out) and torch.equal(lse, ref_lse)
    ro, rl = oracle.attn_fwd_window(x["q"], x["k"], x["v"], s.scale, s.causal,
                                    window if window is not None else (-1, -1))
    check_parity(out.cpu(), lse.cpu(), ro, rl, s.dtype, str(case))


def test_packed_qkv_and_output_slice():
    """q, k, v as views of one packed [B, L, 3, H, D] tensor; out written into the first
    H heads of a wider [B, L, H + 2, D] buffer whose other heads must stay untouched."""
    B, H, L, D, dtype = 2, 4, 333, 128, torch.bfloat16
    s = inputs.DenseSpec("packed", B, H, H, L, L, D, dtype, True, 1 / math.sqrt(D), seed=9)
    x = inputs.make(s)
    qkv = torch.stack([x[n].transpose(1, 2) for n in ("q", "k", "v")], dim=2).contiguous().to(DEV)
    q, k, v = (qkv[:, :, i].transpose(1, 2) for i in range(3))           # [B, H, L, D] views
    wide = torch.full((B, L, H + 2, D), 5.0, dtype=dtype, device=DEV)
    out = wide[:, :, :H].transpose(1, 2)
    ta.fwd(q, k, v, causal=True, scale=s.scale, out=out)
    torch.cuda.synchronize()
    assert ta.device_status() == 0
    assert torch.all(wide[:, :, H:] == 5.0)
    ro, rl = oracle.attn_fwd(x["q"], x["k"], x["v"], s.scale, True)
    check_parity(out.cpu(), None, ro, rl, dtype, "packed qkv")


def test_no_keys_strided_output():
    q = torch.randn(1, 3, 2, 64, device=DEV).to(torch.float16)
    k = torch.empty(1, 3, 0, 64, device=DEV, dtype=torch.float16)
    wide = torch.full((1, 3, 4, 64), 9.0, dtype=torch.float16, device=DEV)
    out = wide[:, :, :2]                                                   # rows 2, 3 untouched
    _, lse = ta.fwd(q, k, k, out=out)
    torch.cuda.synchronize()
    assert torch.count_nonzero(wide[:, :, :2]) == 0 and torch.all(wide[:, :, 2:] == 9.0)
    assert torch.all(lse == -math.inf)


def test_bad_strides_rejected():
    q = torch.randn(1, 2, 16, 64, device=DEV).to(torch.float16)
    odd = torch.empty(1, 2, 16, 68, device=DEV, dtype=torch.float16)[..., :64]  # row stride 68
    with pytest.raises(ta.AttnError) as e:
        ta.fwd(odd, q, q)
    assert e.value.code == -3


BWD_CASES = [
    # B, Hq, Hkv, Lq, Lk, D, dtype, causal, window
    (2, 4, 2, 300, 300, 128, torch.bfloat16, True, None),
    (1, 4, 4, 257, 390, 64, torch.float16, False, None),
    (1, 4, 2, 400, 400, 128, torch.float16, False, (64, 16)),
]


@pytest.mark.parametrize("case", BWD_CASES, ids=lambda c: "B{}_H{}-{}_Lq{}_Lk{}_D{}_{}".format(
    *c[:6], "causal" if c[7] else "full"))
def test_backward_blhd_layout(case):
    """attn_bwd_strided on flash_attn's [B, L, H, D] tensors: q, k, v, out, dout read in that
    layout and dq, dk, dv written into the first heads of wider [B, L, H + 1, D] buffers,
    whose last head must stay untouched. Equal bit for bit to the contiguous backward
    (same kernels, other addresses) and within the gradient tolerance of the oracle."""
    B, Hq, Hkv, Lq, Lk, D, dtype, causal, window = case
    s, x = dense(case)
    do = inputs.dense_grad_output(s)
    q, k, v, dout = (t.to(DEV) for t in (x["q"], x["k"], x["v"], do))
    out, lse = ta.fwd(q, k, v, causal=causal, scale=s.scale, window=window)
    ref = ta.bwd(q, k, v, out, dout, lse, causal=causal, scale=s.scale, window=window)
    blhd = [t.transpose(1, 2).contiguous().transpose(1, 2) for t in (q, k, v, out, dout)]
    wides = [torch.full((B, L, H + 1, D), 3.0, dtype=dtype, device=DEV)
             for H, L in ((Hq, Lq), (Hkv, Lk), (Hkv, Lk))]
    grads = [w[:, :, :-1].transpose(1, 2) for w in wides]
    ta.bwd(*blhd, lse, causal=causal, scale=s.scale, window=window, dq=grads[0], dk=grads[1],
           dv=grads[2])
    torch.cuda.synchronize()
    assert ta.device_status() == 0
    for w in wides:
        assert torch.all(w[:, :, -1] == 3.0)
    for g, r in zip(grads, ref):
        assert torch.equal(g, r)
    want = oracle.attn_bwd(x["q"], x["k"], x["v"], do, s.scale, causal,
                           window if window is not None else (-1, -1), sensitivity=True)
    for i, name in enumerate(("dq", "dk", "dv")):
        check_grad(grads[i].cpu(), want[i], want[3 + i], dtype, f"{case} {name}")


def test_backward_default_gradients_take_input_strides():
    """Without dq/dk/dv, ta.bwd allocates them like q, k, v: [B, L, H, D] storage in,
    [B, L, H, D] storage out."""
    case = (1, 2, 1, 130, 130, 64, torch.bfloat16, True, None)
    s, x = dense(case)
    q, k, v = (x[n].to(DEV).transpose(1, 2).contiguous().transpose(1, 2) for n in ("q", "k", "v"))
    out, lse = ta.fwd(q, k, v, causal=True, scale=s.scale)
    dout = torch.ones_like(out)
    dq, dk, dv = ta.bwd(q, k, v, out, dout, lse, causal=True, scale=s.scale)
    torch.cuda.synchronize()
    assert dq.stride() == q.stride() and dk.stride() == k.stride()
    ref = ta.bwd(*(t.contiguous() for t in (q, k, v, out, dout)), lse, causal=True,
                 scale=s.scale)
    for g, r in zip((dq, dk, dv), ref):
        assert torch.equal(g, r)


def test_backward_empty_side_strided():
    """No keys: dQ = 0 written through its strides, neighbouring rows untouched."""
    q = torch.randn(1, 2, 3, 64, device=DEV).to(torch.float16)
    k = torch.empty(1, 1, 0, 64, device=DEV, dtype=torch.float16)
    out, lse = ta.fwd(q, k, k)
    wide = torch.full((1, 2, 5, 64), 4.0, dtype=torch.float16, device=DEV)
    dq = wide[:, :, 1:4]
    ta.bwd(q, k, k, out, torch.ones_like(q), lse, dq=dq, dk=k.clone(), dv=k.clone())
    torch.cuda.synchronize()
    assert torch.count_nonzero(dq) == 0
    assert torch.all(wide[:, :, 0] == 4.0) and torch.all(wide[:, :, 4] == 4.0)
