"""Shared parity helpers for the GPU tests.

Tolerances (fp32 accumulation, f16/bf16 outputs), compared element by element against
the fp64 oracle on the same inputs:
  O:   max |O_gpu - O_ref| <= 2e-3 (f16 outputs), <= 1.6e-2 (bf16 outputs)
  lse: |lse_gpu - lse_ref| <= 1e-4 * max(1, |lse_ref|); -inf exactly where the oracle has it
Gradients (backward pass): |g_gpu - g_ref| <= 3 u (m + |g_ref|) element by element, with
u the dtype's unit roundoff and m the element's first-order rounding sensitivity from the
oracle (the derivation is in tests/test_backward_gpu.py).
"""
from __future__ import annotations

import math

import torch

O_TOL = {torch.float16: 2e-3, torch.bfloat16: 1.6e-2}
LSE_REL = 1e-4
SENTINEL = 0x7BCD  # 16-bit pattern written around outputs to catch stray writes


def check_parity(out_gpu, lse_gpu, out_ref, lse_ref, dtype, what=""):
    o = out_gpu.detach().to("cpu", torch.float64)
    assert o.shape == out_ref.shape, (o.shape, out_ref.shape)
    assert torch.isfinite(o).all(), f"{what}: non-finite output"
    err = (o - out_ref).abs()
    tol = O_TOL[dtype]
    mx = float(err.max()) if err.numel() else 0.0
    assert mx <= tol, f"{what}: max |O err| {mx:.3e} > {tol} at {tuple(int(i) for i in torch.nonzero(err == err.max())[0])}"
    if lse_gpu is not None:
        lg = lse_gpu.detach().to("cpu", torch.float64)
        fin = torch.isfinite(lse_ref)
        assert torch.equal(torch.isfinite(lg), fin), f"{what}: lse finiteness differs"
        assert torch.all(lg[~fin] == lse_ref[~fin]), f"{what}: lse -inf rows differ"
        if fin.any():
            rel = ((lg[fin] - lse_ref[fin]).abs() / lse_ref[fin].abs().clamp_min(1.0)).max()
            assert float(rel) <= LSE_REL, f"{what}: lse error {float(rel):.3e} > {LSE_REL}"
    return mx


def check_rounding_bound(out_gpu, lse_gpu, out_ref, lse_ref, m, dtype, what=""):
    """O against a bound from the kernel's roundings instead of the fixed tolerance.

    P is rounded to the 16-bit input type (unit roundoff u) before P.V and O is rounded
    to it at the end; the accumulation is fp32. To first order the error of an element is
    at most u * m + u * |O| with m = sum_j p_j |v_j| / l (the oracle on |V|); the factor 2
    covers the exponential's own error and the fp32 accumulation. For rows dominated by
    a few keys m approaches max |v|, which the fixed tolerance does not allow for.
    lse keeps its relative tolerance."""
    u = GRAD_U[dtype]
    o = out_gpu.detach().to("cpu", torch.float64)
    assert o.shape == out_ref.shape, (o.shape, out_ref.shape)
    assert torch.isfinite(o).all(), f"{what}: non-finite output"
    err = (o - out_ref).abs()
    bound = 2 * u * (m.to(torch.float64) + out_ref.abs()) + 1e-6
    ok = err <= bound
    if not bool(ok.all()):
        at = tuple(int(i) for i in torch.nonzero(~ok)[0])
        raise AssertionError(f"{what}: {int((~ok).sum())} elements over the bound; first at {at}: "
                             f"|err| {float(err[at]):.3e} > {float(bound[at]):.3e}")
    check_parity(o, lse_gpu, o, lse_ref, dtype, what)  # lse only (O against itself)
    return float((err / bound).max())


def guarded_empty(shape, dtype, device, guard=4096):
    """A tensor whose storage sits between two guard bands filled with a sentinel."""
    n = math.prod(shape)
    el = torch.tensor([], dtype=dtype).element_size()
    g = guard // el
    buf = torch.empty(n + 2 * g, dtype=dtype, device=device)
    buf.view(torch.int16 if el == 2 else torch.int32).fill_(SENTINEL)
    return buf, buf[g:g + n].view(shape), g


def guards_intact(buf, g):
    el = buf.element_size()
    raw = buf.view(torch.int16 if el == 2 else torch.int32)
    return bool((raw[:g] == SENTINEL).all() and (raw[-g:] == SENTINEL).all())


GRAD_U = {torch.float16: 2.0 ** -11, torch.bfloat16: 2.0 ** -9}


def check_grad(got, ref, sens, dtype, what):
    g = got.detach().to("cpu", torch.float64)
    ref = ref.to(torch.float64)
    assert g.shape == ref.shape, (what, g.shape, ref.shape)
    assert torch.isfinite(g).all(), f"{what}: non-finite gradient"
    err = (g - ref).abs()
    bound = 3 * GRAD_U[dtype] * (sens.to(torch.float64) + ref.abs())
    ok = err <= bound
    if not bool(ok.all()):
        at = tuple(int(i) for i in torch.nonzero(~ok)[0])
        raise AssertionError(f"{what}: {int((~ok).sum())} elements over the bound; first at {at}: "
                             f"|err| {float(err[at]):.3e} > {float(bound[at]):.3e}")
    ratio = float((err / bound.clamp_min(1e-300)).max()) if err.numel() else 0.0
    print(f"{what}: max |err| / bound = {ratio:.3f}")
    return ratio
