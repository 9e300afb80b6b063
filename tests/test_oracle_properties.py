"""Randomised invariants of the fp64 oracle over many small shapes.

The pins in test_oracle.py fix the oracle on chosen shapes and worked examples. These
properties hold for every shape, so hypothesis draws the shapes (batch, grouped heads,
Lq != Lk, empty sides, causal and sliding-window bands) and the seeds; the draws are
derandomized, so the suite is reproducible. Each property follows from the definition
of attention in "Self-attention, CUDA kernels and FlashAttention" (russian.itimpress.au),
section 1, with the band of the "Flash Attention" skill page (hermes-agent-app.ru),
Scenario 2 (window_size):
  - O_i is a convex combination of the visible value rows, so every element lies between
    the smallest and the largest visible value of its column;
  - lse_i = log sum_j exp(s_ij) over the visible keys lies between max_j s_ij and
    max_j s_ij + ln(#visible);
  - a row that sees no key has O_i = 0 and lse_i = -inf;
  - the rows of P sum to 1 and P is zero outside the band.
"""
from __future__ import annotations

import math

import numpy as np
import torch
from hypothesis import given, settings, strategies as st

import oracle

SETTINGS = settings(max_examples=60, deadline=None, derandomize=True)


def visible(i: int, Lq: int, Lk: int, causal: bool, left: int, right: int) -> np.ndarray:
    """Keys query i sees: the band around i' = i + Lk - Lq (bottom-right alignment),
    right clipped to 0 when causal, -1 = unbounded."""
    ii = i + Lk - Lq
    j = np.arange(Lk)
    ok = np.ones(Lk, bool)
    if causal or right >= 0:
        ok &= j <= ii + (0 if causal else right)
    if left >= 0:
        ok &= j >= ii - left
    return j[ok]


@st.composite
def problems(draw):
    B = draw(st.integers(1, 2))
    Hkv = draw(st.integers(1, 2))
    G = draw(st.integers(1, 3))
    Lq = draw(st.integers(0, 24))
    Lk = draw(st.integers(0, 24))
    D = draw(st.integers(1, 12))
    causal = draw(st.booleans())
    left = draw(st.integers(-1, 8))
    right = draw(st.integers(-1, 8))
    scale = draw(st.sampled_from([0.125, 0.5, 1.0 / math.sqrt(max(D, 1))]))
    seed = draw(st.integers(0, 2**31 - 1))
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, Hkv * G, Lq, D, generator=g, dtype=torch.float64)
    k = torch.randn(B, Hkv, Lk, D, generator=g, dtype=torch.float64)
    v = torch.randn(B, Hkv, Lk, D, generator=g, dtype=torch.float64)
    return q, k, v, scale, causal, left, right


@SETTINGS
@given(problems())
def test_outputs_are_convex_and_lse_is_bounded(p):
    q, k, v, scale, causal, left, right = p
    B, Hq, Lq, D = q.shape
    Hkv, Lk = k.shape[1], k.shape[2]
    out, lse = oracle.attn_fwd_window(q, k, v, scale, causal, (left, right))
    out, lse = out.numpy(), lse.numpy()
    qn, kn, vn = q.numpy(), k.numpy(), v.numpy()
    G = Hq // Hkv
    for b in range(B):
        for h in range(Hq):
            hk = h // G
            for i in range(Lq):
                js = visible(i, Lq, Lk, causal, left, right)
                if js.size == 0:
                    assert np.all(out[b, h, i] == 0.0)
                    assert lse[b, h, i] == -math.inf
                    continue
                s = scale * (kn[b, hk, js] @ qn[b, h, i])
                m = s.max()
                assert m - 1e-12 <= lse[b, h, i] <= m + math.log(js.size) + 1e-12
                lo = vn[b, hk, js].min(axis=0) - 1e-12
                hi = vn[b, hk, js].max(axis=0) + 1e-12
                assert np.all(out[b, h, i] >= lo) and np.all(out[b, h, i] <= hi)


@SETTINGS
@given(problems())
def test_probability_rows_sum_to_one_inside_the_causal_band(p):
    q, k, v, scale, causal, _, _ = p
    Lq, Lk = q.shape[2], k.shape[2]
    probs = oracle.attn_probs(q, k, v, scale, causal).numpy()
    for i in range(Lq):
        js = visible(i, Lq, Lk, causal, -1, -1)
        row = probs[:, :, i, :]
        outside = np.setdiff1d(np.arange(Lk), js)
        assert np.all(row[..., outside] == 0.0)
        total = row.sum(axis=-1)
        if js.size == 0:
            assert np.all(total == 0.0)
        else:
            assert np.allclose(total, 1.0, atol=1e-12, rtol=0)
            assert np.all(row[..., js] > 0.0)  # every visible key weighs something
