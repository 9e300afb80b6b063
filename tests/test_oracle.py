"""Pins for the oracle: each check ties it to something other than itself.

* A brute force in 60-digit decimal arithmetic (exact products, Decimal.exp/ln, no
  max subtraction) on tiny random shapes.
* Closed-form worked examples derived by hand (tests/golden/).
* Invariants fixed by the definition: probability rows sum to 1, constant V, identical
  keys, the argmax limit, causal row 0, shift invariance, permutation equivariance,
  grouped-query heads equal repeated heads, paged equals the gathered dense problem,
  fully masked rows.
* Restatements of the algebra the GPU kernels use (a tiled online softmax with lazy
  rescaling, and a split-KV log-sum-exp combine), checked against the oracle.
* Backward pass: torch autograd in float64 through a plain statement of the forward,
  central finite differences of the forward oracle, hand-derived examples
  (tests/golden/backward_closed_form.json), and invariants of the definition (key
  gradients sum to zero, value gradients sum to dO, identical keys and single-key
  rows give dQ = 0, grouped heads equal summed repeated heads).

Every ``pin_*`` function takes an optional oracle library handle so that
test_pins_catch_planted_mistakes can run the same pins on deliberately broken builds
of the oracle and show that each planted mistake fails at least one of them.
"""
from __future__ import annotations

import json
import math
import os
import shutil
import subprocess
import sys
import tempfile
from decimal import Decimal, localcontext

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "closed_form_examples.json")


# --------------------------------------------------------------------------- helpers
def brute_attention(q, k, v, scale, causal, window=(-1, -1)):
    """Independent brute force: exact decimal products, Decimal exp/ln at 60 digits,
    no max subtraction. Returns (out, lse) as float64 arrays. window = (left, right):
    query i (shifted to i + Lk - Lq) sees keys within left before and right after it,
    -1 meaning unbounded; causal caps the right side at 0."""
    q, k, v = (np.asarray(t, dtype=np.float64) for t in (q, k, v))
    B, Hq, Lq, D = q.shape
    Hkv, Lk = k.shape[1], k.shape[2]
    G = Hq // Hkv
    out = np.zeros((B, Hq, Lq, D))
    lse = np.zeros((B, Hq, Lq))
    with localcontext() as ctx:
        ctx.prec = 60
        sc = Decimal(float(scale))
        for b in range(B):
            for h in range(Hq):
                hk = h // G
                for i in range(Lq):
                    ii = i + Lk - Lq
                    right = 0 if causal else window[1]
                    vis = [j for j in range(Lk)
                           if (right < 0 or j <= ii + right) and (window[0] < 0 or j >= ii - window[0])]
                    if not vis:
                        lse[b, h, i] = -math.inf
                        continue
                    w = []
                    for j in vis:
                        dot = sum(Decimal(float(q[b, h, i, d])) * Decimal(float(k[b, hk, j, d]))
                                  for d in range(D))
                        w.append((sc * dot).exp())
                    z = sum(w)
                    for d in range(D):
                        num = sum(wj * Decimal(float(v[b, hk, j, d])) for wj, j in zip(w, vis))
                        out[b, h, i, d] = float(num / z)
                    lse[b, h, i] = float(z.ln())
    return out, lse


def close(a, b, tol=1e-12):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, (a.shape, b.shape)
    fin = np.isfinite(b)
    assert np.array_equal(np.isfinite(a), fin) and np.array_equal(a[~fin], b[~fin])
    err = np.abs(a[fin] - b[fin]) / np.maximum(1.0, np.abs(b[fin]))
    assert err.size == 0 or err.max() <= tol, f"max scaled error {err.max():.3e} > {tol}"


def rand(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g, dtype=torch.float64) * scale).numpy()


def online_softmax_attention(q, K, V, n_vis, scale, tile, thr=0.0):
    """fp64 restatement of the tiled recurrence the prefill kernel runs for one row:
    per key tile, a running reference max m (moved only when the tile max exceeds it
    by more than ``thr``, natural-log units), a running sum l and an accumulator that
    is rescaled by exp(m_old - m_new) whenever m moves."""
    Lk, D = K.shape
    m, l, acc = -math.inf, 0.0, np.zeros(D)
    for t0 in range(0, Lk, tile):
        s = scale * (K[t0:t0 + tile] @ q)
        idx = np.arange(t0, min(t0 + tile, Lk))
        s = np.where(idx < n_vis, s, -math.inf)
        mx = s.max()
        m_new = mx if (m == -math.inf or mx > m + thr) else m
        if m_new == -math.inf:
            continue
        alpha = 0.0 if m == -math.inf else math.exp(m - m_new)
        p = np.exp(s - m_new)
        l = alpha * l + p.sum()
        acc = alpha * acc + p @ V[t0:t0 + tile]
        m = m_new
    if l == 0.0:
        return np.zeros(D), -math.inf
    return acc / l, m + math.log(l)


# ------------------------------------------------------------------------------ pins
def pin_brute_force(lib=None):
    cases = [
        # B, Hq, Hkv, Lq, Lk, D, causal, scale
        (1, 1, 1, 1, 1, 1, False, 1.0),
        (1, 2, 1, 3, 5, 4, False, 0.5),
        (2, 2, 2, 4, 4, 3, True, 0.7),
        (1, 4, 2, 5, 3, 8, True, 0.35),   # Lq > Lk causal: some rows fully masked
        (1, 3, 1, 2, 7, 5, True, 1.3),    # Lq < Lk causal: bottom-right alignment
        (2, 4, 1, 3, 6, 2, False, 0.25),
    ]
    for n, (B, Hq, Hkv, Lq, Lk, D, causal, scale) in enumerate(cases):
        q = rand((B, Hq, Lq, D), 100 + n)
        k = rand((B, Hkv, Lk, D), 200 + n)
        v = rand((B, Hkv, Lk, D), 300 + n)
        o_ref, l_ref = brute_attention(q, k, v, scale, causal)
        o, l = oracle.attn_fwd(q, k, v, scale, causal, lib=lib)
        close(o, o_ref)
        close(l, l_ref)


def pin_golden(lib=None):
    with open(GOLDEN) as f:
        examples = json.load(f)["examples"]
    for ex in examples:
        if ex["kind"] == "dense":
            o, l = oracle.attn_fwd(np.array(ex["q"]), np.array(ex["k"]), np.array(ex["v"]),
                                   ex["scale"], ex["causal"], lib=lib)
        elif ex["kind"] == "paged_prefill":
            o, l = oracle.attn_paged_prefill(np.array(ex["q"]), np.array(ex["k_cache"]),
                                             np.array(ex["v_cache"]),
                                             torch.tensor(ex["block_table"], dtype=torch.int32),
                                             torch.tensor(ex["seq_lens"], dtype=torch.int32),
                                             ex["scale"], ex["causal"], lib=lib)
        else:
            o, l = oracle.attn_paged(np.array(ex["q"]), np.array(ex["k_cache"]),
                                     np.array(ex["v_cache"]),
                                     torch.tensor(ex["block_table"], dtype=torch.int32),
                                     torch.tensor(ex["seq_lens"], dtype=torch.int32),
                                     ex["scale"], lib=lib)
        close(o, np.array(ex["out"]), 1e-14)
        close(l, np.array(ex["lse"]), 1e-14)


def pin_probability_rows(lib=None):
    for causal in (False, True):
        q = rand((1, 2, 6, 4), 1)
        k = rand((1, 2, 6, 4), 2)
        P = oracle.attn_probs(q, k, k, 0.6, causal, lib=lib).numpy()
        assert (P >= 0).all()
        close(P.sum(-1), np.ones(P.shape[:-1]))
        if causal:  # masked entries are exactly zero
            assert np.all(np.triu(P[0, 0], 1) == 0.0) and np.all(np.triu(P[0, 1], 1) == 0.0)
        # P must be the softmax of the scaled scores (pins P itself, not just O)
        s = 0.6 * np.einsum("bhid,bhjd->bhij", q, k)
        if causal:
            s = np.where(np.triu(np.ones((6, 6), bool), 1), -np.inf, s)
        e = np.exp(s - s.max(-1, keepdims=True))
        close(P, e / e.sum(-1, keepdims=True))


def pin_constant_values(lib=None):
    q = rand((2, 3, 5, 4), 3)
    k = rand((2, 3, 9, 4), 4)
    c = rand((4,), 5)
    v = np.broadcast_to(c, (2, 3, 9, 4)).copy()
    for causal in (False, True):
        o, _ = oracle.attn_fwd(q, k, v, 0.5, causal, lib=lib)
        close(o, np.broadcast_to(c, o.shape))


def pin_identical_keys(lib=None):
    q = rand((1, 2, 4, 3), 6)
    k = np.broadcast_to(rand((3,), 7), (1, 2, 4, 3)).copy()
    v = rand((1, 2, 4, 3), 8)
    o, l = oracle.attn_fwd(q, k, v, 0.9, True, lib=lib)
    s = 0.9 * np.einsum("bhid,bhjd->bhij", q, k)[..., 0]  # every key scores the same
    for i in range(4):  # causal: row i averages the first i+1 values uniformly
        close(o[:, :, i], v[:, :, : i + 1].mean(axis=2))
        close(l[:, :, i], s[:, :, i] + math.log(i + 1))


def pin_argmax_limit(lib=None):
    D, Lk = 4, 6
    k = rand((1, 1, Lk, D), 9)
    d = 2
    k[0, 0, :, d] = np.arange(Lk, dtype=np.float64)  # unique argmax (key 5) with margin 1
    q = np.zeros((1, 1, 1, D))
    q[0, 0, 0, d] = 1e4
    v = rand((1, 1, Lk, D), 10)
    o, l = oracle.attn_fwd(q, k, v, 0.1, False, lib=lib)  # scale * margin = 1000 nats
    close(o[0, 0, 0], v[0, 0, Lk - 1], 1e-9)
    close(l[0, 0, 0], 0.1 * 1e4 * (Lk - 1), 1e-12)


def pin_causal_row0(lib=None):
    q = rand((2, 2, 7, 5), 11)
    k = rand((2, 2, 7, 5), 12)
    v = rand((2, 2, 7, 5), 13)
    o, l = oracle.attn_fwd(q, k, v, 0.4, True, lib=lib)
    assert np.array_equal(o[:, :, 0].numpy(), v[:, :, 0])
    close(l[:, :, 0], 0.4 * np.einsum("bhd,bhd->bh", q[:, :, 0], k[:, :, 0]))


def pin_shift_invariance(lib=None):
    # adding u to every key shifts each row's scores by scale*(q.u): P, O unchanged,
    # lse shifted by the same amount
    q = rand((1, 2, 5, 4), 14)
    k = rand((1, 2, 8, 4), 15)
    v = rand((1, 2, 8, 4), 16)
    u = rand((4,), 17, 3.0)
    for causal in (False, True):
        o1, l1 = oracle.attn_fwd(q, k, v, 0.7, causal, lib=lib)
        o2, l2 = oracle.attn_fwd(q, k + u, v, 0.7, causal, lib=lib)
        close(o2, o1, 1e-10)
        close(l2, l1.numpy() + 0.7 * np.einsum("bhid,d->bhi", q, u), 1e-10)


def pin_permutation_equivariance(lib=None):
    q = rand((1, 1, 3, 4), 18)
    k = rand((1, 1, 9, 4), 19)
    v = rand((1, 1, 9, 4), 20)
    perm = np.random.default_rng(0).permutation(9)
    o1, l1 = oracle.attn_fwd(q, k, v, 0.5, False, lib=lib)
    o2, l2 = oracle.attn_fwd(q, k[:, :, perm], v[:, :, perm], 0.5, False, lib=lib)
    close(o2, o1)
    close(l2, l1)


def pin_gqa_equals_repeat(lib=None):
    B, Hq, Hkv, L, D = 2, 6, 2, 5, 4
    q = rand((B, Hq, L, D), 21)
    k = rand((B, Hkv, L, D), 22)
    v = rand((B, Hkv, L, D), 23)
    for causal in (False, True):
        o1, l1 = oracle.attn_fwd(q, k, v, 0.5, causal, lib=lib)
        kr = np.repeat(k, Hq // Hkv, axis=1)  # consecutive query heads share a K/V head
        vr = np.repeat(v, Hq // Hkv, axis=1)
        o2, l2 = oracle.attn_fwd(q, kr, vr, 0.5, causal, lib=lib)
        assert torch.equal(o1, o2) and torch.equal(l1, l2)
        # and it really is the grouped mapping, not a coincidence of the inputs
        o3, _ = oracle.attn_fwd(q, np.tile(k, (1, Hq // Hkv, 1, 1)),
                                np.tile(v, (1, Hq // Hkv, 1, 1)), 0.5, causal, lib=lib)
        assert not torch.allclose(o1, o3)


def pin_paged_equals_dense(lib=None):
    g = np.random.default_rng(1)
    S, Hq, Hkv, D, bs, MB = 3, 4, 2, 8, 4, 5
    NB = S * MB + 2
    kc = g.standard_normal((NB, Hkv, bs, D))
    vc = g.standard_normal((NB, Hkv, bs, D))
    q = g.standard_normal((S, Hq, D))
    bt = g.permutation(NB)[: S * MB].reshape(S, MB).astype(np.int32)
    lens = np.array([1, 7, MB * bs], np.int32)
    o, l = oracle.attn_paged(q, kc, vc, torch.from_numpy(bt), torch.from_numpy(lens), 0.3,
                             lib=lib)
    for s in range(S):
        t = np.arange(lens[s])
        kd = kc[bt[s, t // bs], :, t % bs]  # [len, Hkv, D]
        vd = vc[bt[s, t // bs], :, t % bs]
        od, ld = oracle.attn_fwd(q[s][None, :, None], kd.transpose(1, 0, 2)[None],
                                 vd.transpose(1, 0, 2)[None], 0.3, False, lib=lib)
        assert torch.equal(o[s], od[0, :, 0]) and torch.equal(l[s], ld[0, :, 0])


def pin_fully_masked_rows(lib=None):
    q = rand((1, 1, 6, 3), 24)
    k = rand((1, 1, 2, 3), 25)
    v = rand((1, 1, 2, 3), 26)
    o, l = oracle.attn_fwd(q, k, v, 1.0, True, lib=lib)  # rows 0..3 see no key
    assert np.all(o[0, 0, :4].numpy() == 0.0) and np.all(np.isneginf(l[0, 0, :4].numpy()))
    assert np.all(np.isfinite(l[0, 0, 4:].numpy()))
    # empty key set, and empty sequences in paged decode
    o, l = oracle.attn_fwd(q, k[:, :, :0], v[:, :, :0], 1.0, False, lib=lib)
    assert np.all(o.numpy() == 0.0) and np.all(np.isneginf(l.numpy()))
    o, l = oracle.attn_paged(q[0, 0][:1, None, :], np.zeros((1, 1, 16, 3)), np.zeros((1, 1, 16, 3)),
                             torch.zeros((1, 1), dtype=torch.int32),
                             torch.zeros((1,), dtype=torch.int32), 1.0, lib=lib)
    assert np.all(o.numpy() == 0.0) and np.all(np.isneginf(l.numpy()))


def pin_online_softmax(lib=None):
    # the tiled recurrence (any tile size, with or without lazy rescaling) reaches the
    # two-pass definition; threshold 8*ln2 is the kernel's lazy-rescale margin
    D, Lq, Lk = 6, 5, 37
    q = rand((1, 1, Lq, D), 27, 2.0)
    k = rand((1, 1, Lk, D), 28, 2.0)
    v = rand((1, 1, Lk, D), 29)
    for causal in (False, True):
        o, l = oracle.attn_fwd(q, k, v, 0.8, causal, lib=lib)
        for tile in (1, 4, 16, 128):
            for thr in (0.0, 8 * math.log(2)):
                for i in range(Lq):
                    n_vis = min(Lk, i + Lk - Lq + 1) if causal else Lk
                    oi, li = online_softmax_attention(q[0, 0, i], k[0, 0], v[0, 0], n_vis, 0.8,
                                                      tile, thr)
                    close(oi, o[0, 0, i])
                    close(li, l[0, 0, i])


def pin_split_combine(lib=None):
    # partial results over disjoint key chunks, merged with log-sum-exp weights,
    # equal the result over all keys (the decode kernel's split-KV combine)
    q = rand((1, 3, 1, 8), 30)
    k = rand((1, 3, 50, 8), 31)
    v = rand((1, 3, 50, 8), 32)
    o, l = oracle.attn_fwd(q, k, v, 0.5, False, lib=lib)
    for bounds in ([0, 50], [0, 16, 32, 48, 50], [0, 1, 2, 49, 50], [0, 0, 25, 50]):
        parts = [oracle.attn_fwd(q, k[:, :, a:b], v[:, :, a:b], 0.5, False, lib=lib)
                 for a, b in zip(bounds[:-1], bounds[1:])]
        lses = np.stack([p[1].numpy() for p in parts])
        m = lses.max(0)
        w = np.exp(lses - m)
        lse = m + np.log(w.sum(0))
        out = sum(np.exp(p[1].numpy() - lse)[..., None] * p[0].numpy() for p in parts)
        close(out, o)
        close(lse, l)


def pin_window(lib=None):
    # brute force with windows, GQA, Lq != Lk
    cases = [
        (1, 2, 1, 6, 6, 4, False, (1, 1), 0.6),
        (1, 2, 2, 5, 9, 3, True, (2, -1), 0.8),     # causal + left window
        (2, 2, 1, 7, 4, 2, False, (0, 2), 1.1),     # Lq > Lk: some rows see nothing
        (1, 1, 1, 8, 8, 5, False, (-1, 1), 0.4),
    ]
    for n, (B, Hq, Hkv, Lq, Lk, D, causal, win, scale) in enumerate(cases):
        q = rand((B, Hq, Lq, D), 400 + n)
        k = rand((B, Hkv, Lk, D), 410 + n)
        v = rand((B, Hkv, Lk, D), 420 + n)
        o_ref, l_ref = brute_attention(q, k, v, scale, causal, win)
        o, l = oracle.attn_fwd_window(q, k, v, scale, causal, win, lib=lib)
        close(o, o_ref)
        close(l, l_ref)
    # exact equivalences with the unwindowed definition
    q = rand((1, 2, 9, 4), 430)
    k = rand((1, 2, 13, 4), 431)
    v = rand((1, 2, 13, 4), 432)
    full = oracle.attn_fwd(q, k, v, 0.5, False, lib=lib)
    causal = oracle.attn_fwd(q, k, v, 0.5, True, lib=lib)
    for got, want in [(oracle.attn_fwd_window(q, k, v, 0.5, False, (-1, -1), lib=lib), full),
                      (oracle.attn_fwd_window(q, k, v, 0.5, False, (-1, 0), lib=lib), causal),
                      (oracle.attn_fwd_window(q, k, v, 0.5, True, (-1, 7), lib=lib), causal),
                      (oracle.attn_fwd_window(q, k, v, 0.5, False, (50, 50), lib=lib), full)]:
        assert torch.equal(got[0], want[0]) and torch.equal(got[1], want[1])
    # window (0, 0): row i attends to key i + (Lk - Lq) alone
    o, l = oracle.attn_fwd_window(q, k, v, 0.5, False, (0, 0), lib=lib)
    for i in range(9):
        close(o[0, :, i], v[0, :, i + 4])
        close(l[0, :, i], 0.5 * np.einsum("hd,hd->h", q[0, :, i], k[0, :, i + 4]))


# ------------------------------------------------------------------- backward pins
BWD_GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "backward_closed_form.json")


def autograd_grads(q, k, v, dout, scale, causal, window=(-1, -1)):
    """Independent derivation: torch autograd in float64 through a plain statement of
    the forward (einsum scores, a boolean band mask, softmax, einsum with V)."""
    q, k, v, do = (torch.tensor(np.asarray(t), dtype=torch.float64) for t in (q, k, v, dout))
    q.requires_grad_(True)
    k.requires_grad_(True)
    v.requires_grad_(True)
    G = q.shape[1] // k.shape[1]
    K = k.repeat_interleave(G, dim=1)
    V = v.repeat_interleave(G, dim=1)
    Lq, Lk = q.shape[2], k.shape[2]
    i = torch.arange(Lq)[:, None] + (Lk - Lq)
    j = torch.arange(Lk)[None, :]
    right = 0 if causal else window[1]
    vis = torch.ones(Lq, Lk, dtype=torch.bool)
    if right >= 0:
        vis &= j <= i + right
    if window[0] >= 0:
        vis &= j >= i - window[0]
    s = torch.einsum("bhid,bhjd->bhij", q, K) * scale
    s = s.masked_fill(~vis, -math.inf)
    p = torch.softmax(s, dim=-1).nan_to_num(0.0)  # rows with no visible key: P = 0
    o = torch.einsum("bhij,bhjd->bhid", p, V)
    (o * do).sum().backward()
    return q.grad.numpy(), k.grad.numpy(), v.grad.numpy()


BWD_CASES = [
    # B, Hq, Hkv, Lq, Lk, D, causal, scale, window
    (1, 1, 1, 1, 1, 1, False, 1.0, (-1, -1)),
    (1, 2, 1, 5, 6, 4, True, 0.5, (-1, -1)),     # grouped heads, Lq < Lk causal
    (2, 2, 2, 4, 4, 3, False, 0.7, (-1, -1)),
    (1, 4, 2, 6, 3, 5, True, 0.35, (-1, -1)),    # Lq > Lk causal: fully masked rows
    (1, 2, 2, 7, 7, 4, False, 0.6, (2, 1)),      # sliding window
    (1, 2, 1, 6, 8, 3, True, 0.9, (3, -1)),      # causal window
]


def pin_bwd_autograd(lib=None):
    for n, (B, Hq, Hkv, Lq, Lk, D, causal, scale, win) in enumerate(BWD_CASES):
        q = rand((B, Hq, Lq, D), 500 + n)
        k = rand((B, Hkv, Lk, D), 600 + n)
        v = rand((B, Hkv, Lk, D), 700 + n)
        do = rand((B, Hq, Lq, D), 800 + n)
        ref = autograd_grads(q, k, v, do, scale, causal, win)
        got = oracle.attn_bwd(q, k, v, do, scale, causal, win, lib=lib)
        for a, b in zip(got, ref):
            close(a, b)


def pin_bwd_finite_differences(lib=None):
    """Central differences of Loss = sum(dO * O) through the forward oracle, on every
    coordinate of q, k and v (h = 1e-6; truncation and rounding stay below 1e-8)."""
    B, Hq, Hkv, Lq, Lk, D, scale = 1, 2, 1, 4, 5, 3, 0.8
    for causal, win in ((True, (-1, -1)), (False, (1, 2))):
        q = rand((B, Hq, Lq, D), 901)
        k = rand((B, Hkv, Lk, D), 902)
        v = rand((B, Hkv, Lk, D), 903)
        do = rand((B, Hq, Lq, D), 904)

        def loss(qq, kk, vv):
            o, _ = oracle.attn_fwd_window(qq, kk, vv, scale, causal, win, lib=lib)
            return float((o.numpy() * do).sum())

        got = oracle.attn_bwd(q, k, v, do, scale, causal, win, lib=lib)
        for which, x in enumerate((q, k, v)):
            fd = np.zeros_like(x)
            for idx in np.ndindex(*x.shape):
                xp, xm = x.copy(), x.copy()
                xp[idx] += 1e-6
                xm[idx] -= 1e-6
                args_p = [q, k, v]
                args_m = [q, k, v]
                args_p[which], args_m[which] = xp, xm
                fd[idx] = (loss(*args_p) - loss(*args_m)) / 2e-6
            close(got[which].numpy(), fd, 1e-7)


def pin_bwd_golden(lib=None):
    with open(BWD_GOLDEN) as f:
        examples = json.load(f)["examples"]
    for ex in examples:
        got = oracle.attn_bwd(np.array(ex["q"]), np.array(ex["k"]), np.array(ex["v"]),
                              np.array(ex["dout"]), ex["scale"], ex["causal"], lib=lib)
        for a, key in zip(got, ("dq", "dk", "dv")):
            close(a, np.array(ex[key]), 1e-14)


def pin_bwd_invariants(lib=None):
    """Facts fixed by the definition. (1) Scores move by the same amount for every
    key when a constant vector is added to all keys, which changes nothing, so the
    key gradients of a head sum to zero. (2) Probability rows sum to 1, so the value
    gradients sum to the sum of dO over rows that see any key. (3) Identical keys give
    dQ = 0. (4) A row that sees a single key (causal row 0) has dQ = 0."""
    q = rand((2, 4, 6, 5), 910)
    k = rand((2, 2, 6, 5), 911)
    v = rand((2, 2, 6, 5), 912)
    do = rand((2, 4, 6, 5), 913)
    for causal in (False, True):
        dq, dk, dv = (t.numpy() for t in oracle.attn_bwd(q, k, v, do, 0.7, causal, lib=lib))
        close(dk.sum(axis=2), np.zeros((2, 2, 5)), 1e-12)
        close(dv.sum(axis=2), do.reshape(2, 2, 2, 6, 5).sum(axis=(2, 3)), 1e-12)
        if causal:
            close(dq[:, :, 0], np.zeros((2, 4, 5)), 1e-12)
    kk = np.repeat(rand((1, 1, 1, 5), 914), 6, axis=2)
    dq, _, _ = oracle.attn_bwd(q[:1, :2], kk, v[:1, :1], do[:1, :2], 0.7, False, lib=lib)
    close(dq.numpy(), np.zeros((1, 2, 6, 5)), 1e-12)


def pin_bwd_gqa_equals_repeat(lib=None):
    q = rand((1, 6, 5, 4), 920)
    k = rand((1, 2, 7, 4), 921)
    v = rand((1, 2, 7, 4), 922)
    do = rand((1, 6, 5, 4), 923)
    dq, dk, dv = oracle.attn_bwd(q, k, v, do, 0.5, True, lib=lib)
    dq2, dk2, dv2 = oracle.attn_bwd(q, np.repeat(k, 3, axis=1), np.repeat(v, 3, axis=1), do,
                                    0.5, True, lib=lib)
    close(dq, dq2)
    close(dk, dk2.numpy().reshape(1, 2, 3, 7, 4).sum(axis=2))
    close(dv, dv2.numpy().reshape(1, 2, 3, 7, 4).sum(axis=2))


def pin_bwd_selected_outputs(lib=None):
    """The selected-row and selected-key entry points give the full result's rows."""
    q = rand((2, 4, 9, 4), 930)
    k = rand((2, 2, 11, 4), 931)
    v = rand((2, 2, 11, 4), 932)
    do = rand((2, 4, 9, 4), 933)
    for causal in (False, True):
        dq, dk, dv = oracle.attn_bwd(q, k, v, do, 0.6, causal, lib=lib)
        rows = np.array([0, 8, 17, 40, 71], np.int64)
        close(oracle.attn_bwd_dq_rows(q, k, v, do, rows, 0.6, causal, lib=lib),
              dq.reshape(-1, 4)[rows])
        keys = np.array([3, 0, 30, 12, 43, 10], np.int64)
        sk, sv = oracle.attn_bwd_dkv_keys(q, k, v, do, keys, 0.6, causal, lib=lib)
        close(sk, dk.reshape(-1, 4)[keys])
        close(sv, dv.reshape(-1, 4)[keys])


def pin_bwd_sensitivity(lib=None):
    """The rounding sensitivities the GPU tests scale their tolerances with: a numpy
    statement from the oracle's probability matrix, the triangle inequality |g| <= m,
    and the selected-output entry points agreeing with the whole."""
    q = rand((1, 4, 7, 5), 940)
    k = rand((1, 2, 9, 5), 941)
    v = rand((1, 2, 9, 5), 942)
    do = rand((1, 4, 7, 5), 943)
    sc = 0.45
    for causal in (False, True):
        dq, dk, dv, mq, mk, mv = (t.numpy() for t in oracle.attn_bwd(
            q, k, v, do, sc, causal, lib=lib, sensitivity=True))
        P = oracle.attn_probs(q, k, v, sc, causal, lib=lib).numpy()
        K, V = np.repeat(k, 2, axis=1), np.repeat(v, 2, axis=1)
        dP = np.einsum("bhid,bhjd->bhij", do, V)
        dS = P * (dP - (P * dP).sum(-1, keepdims=True))
        A = np.abs(do * np.einsum("bhij,bhjd->bhid", P, V)).sum(-1)
        W = np.abs(dS) + P * A[..., None]
        close(mq, sc * np.einsum("bhij,bhjd->bhid", W, np.abs(K)))
        close(mk, sc * np.einsum("bhij,bhid->bhjd", W, np.abs(q)).reshape(1, 2, 2, 9, 5).sum(2))
        close(mv, np.einsum("bhij,bhid->bhjd", P, np.abs(do)).reshape(1, 2, 2, 9, 5).sum(2))
        for g, m in ((dq, mq), (dk, mk), (dv, mv)):
            assert (np.abs(g) <= m * (1 + 1e-12) + 1e-300).all()
        rows = np.array([0, 6, 13, 27], np.int64)
        _, mr = oracle.attn_bwd_dq_rows(q, k, v, do, rows, sc, causal, lib=lib, sensitivity=True)
        close(mr, mq.reshape(-1, 5)[rows])
        keys = np.array([0, 8, 9, 17], np.int64)
        _, _, mkr, mvr = oracle.attn_bwd_dkv_keys(q, k, v, do, keys, sc, causal, lib=lib,
                                                  sensitivity=True)
        close(mkr, mk.reshape(-1, 5)[keys])
        close(mvr, mv.reshape(-1, 5)[keys])


def pin_paged_prefill(lib=None):
    """Paged prefill equals the dense oracle on the gathered cache (Lq = q_len, Lk =
    seq_len, bottom-right causal), for every sequence and head; rows past a sequence's
    chunk are empty rows; one query per sequence is the paged decode."""
    g = torch.Generator().manual_seed(950)
    S, Hq, Hkv, Lq, D, bs, MB = 3, 4, 2, 6, 5, 4, 5
    NB = S * MB + 2
    kc = rand((NB, Hkv, bs, D), 951)
    vc = rand((NB, Hkv, bs, D), 952)
    q = rand((S, Hq, Lq, D), 953)
    bt = torch.randperm(NB, generator=g)[:S * MB].reshape(S, MB).to(torch.int32)
    sl = torch.tensor([17, 6, 1], dtype=torch.int32)
    ql = torch.tensor([6, 4, 1], dtype=torch.int32)
    for causal in (True, False):
        o, l = oracle.attn_paged_prefill(q, kc, vc, bt, sl, 0.6, causal, q_lens=ql, lib=lib)
        for s_ in range(S):
            n, m = int(sl[s_]), int(ql[s_])
            t = torch.arange(n)
            rows = bt[s_][t // bs].long()
            K = torch.from_numpy(kc)[rows, :, t % bs].permute(1, 0, 2).unsqueeze(0).numpy()
            V = torch.from_numpy(vc)[rows, :, t % bs].permute(1, 0, 2).unsqueeze(0).numpy()
            od, ld = oracle.attn_fwd(q[s_:s_ + 1, :, :m], K, V, 0.6, causal, lib=lib)
            close(o[s_:s_ + 1, :, :m], od)
            close(l[s_:s_ + 1, :, :m], ld)
            close(o[s_, :, m:], np.zeros((Hq, Lq - m, D)))
            assert bool((l[s_, :, m:] == -math.inf).all())
    o1, l1 = oracle.attn_paged_prefill(q[:, :, :1], kc, vc, bt, sl, 0.6, True, lib=lib)
    od, ld = oracle.attn_paged(q[:, :, 0], kc, vc, bt, sl, 0.6, lib=lib)
    close(o1[:, :, 0], od)
    close(l1[:, :, 0], ld)


PINS = [pin_brute_force, pin_golden, pin_probability_rows, pin_constant_values,
        pin_identical_keys, pin_argmax_limit, pin_causal_row0, pin_shift_invariance,
        pin_permutation_equivariance, pin_gqa_equals_repeat, pin_paged_equals_dense,
        pin_fully_masked_rows, pin_online_softmax, pin_split_combine, pin_window,
        pin_bwd_autograd, pin_bwd_finite_differences, pin_bwd_golden, pin_bwd_invariants,
        pin_bwd_gqa_equals_repeat, pin_bwd_selected_outputs, pin_bwd_sensitivity,
        pin_paged_prefill]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_oracle_pin(pin):
    pin()


def test_rows_subset_matches_full():
    q = rand((2, 4, 9, 8), 33)
    k = rand((2, 2, 11, 8), 34)
    v = rand((2, 2, 11, 8), 35)
    o, l = oracle.attn_fwd(q, k, v, 0.5, True)
    rows = np.array([0, 5, 17, 35, 71, 40], np.int64)
    orr, lr = oracle.attn_fwd_rows(q, k, v, rows, 0.5, True)
    assert torch.equal(orr, o.reshape(-1, 8)[rows]) and torch.equal(lr, l.reshape(-1)[rows])


def test_threads_do_not_change_results():
    q = rand((1, 4, 33, 16), 36)
    k = rand((1, 4, 33, 16), 37)
    v = rand((1, 4, 33, 16), 38)
    a = oracle.attn_fwd(q, k, v, 0.25, True, threads=1)
    b = oracle.attn_fwd(q, k, v, 0.25, True, threads=7)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_oracle_rejects_bad_table():
    with pytest.raises(ValueError):
        oracle.attn_paged(np.zeros((1, 1, 4)), np.zeros((2, 1, 4, 4)), np.zeros((2, 1, 4, 4)),
                          torch.tensor([[0, 5]], dtype=torch.int32),
                          torch.tensor([6], dtype=torch.int32), 1.0)


# Plausible mistakes, each planted in a temporary copy of the oracle source.
MUTANTS = {
    "scale_dropped": ("s[j] = scale * dot;", "s[j] = dot;"),
    "causal_off_by_one": ("int64_t last = i + (Lk - Lq);", "int64_t last = i + (Lk - Lq) - 1;"),
    "causal_top_left": ("int64_t last = i + (Lk - Lq);", "int64_t last = i;"),
    "gqa_modulo_mapping": ("int64_t hkv = h / group;", "int64_t hkv = h % J->Hkv;"),
    "keys_used_as_values": ("o[d] += p * V[j * D + d];", "o[d] += p * K[j * D + d];"),
    "values_used_as_keys": ("dot += qi[d] * K[j * D + d];", "dot += qi[d] * V[j * D + d];"),
    "max_not_subtracted_in_sum": ("l += exp(s[j] - m);", "l += exp(s[j]);"),
    "lse_log2": ("*lse = m + log(l);", "*lse = m + log2(l);"),
    "lse_without_max": ("*lse = m + log(l);", "*lse = log(l);"),
    "paged_row_index": ("t % J->block_size) * J->D;", "t / J->block_size) * J->D;"),
    "paged_head_index": ("((phys * J->Hkv + hkv) * J->block_size", "((phys * J->Hkv) * J->block_size"),
    "paged_len_plus_one": ("int64_t len = J->seq_lens[sq];", "int64_t len = J->seq_lens[sq] + 1;"),
    "window_left_off_by_one": ("if (left >= 0 && last - left > a) a = last - left;",
                               "if (left >= 0 && last - left + 1 > a) a = last - left + 1;"),
    "window_right_off_by_one": ("if (right >= 0 && last + right + 1 < b) b = last + right + 1;",
                                "if (right >= 0 && last + right < b) b = last + right;"),
    "bwd_delta_dropped": ("for (j = lo; j < hi; ++j) ds[j] = p[j] * (ds[j] - delta);",
                          "for (j = lo; j < hi; ++j) ds[j] = p[j] * ds[j];"),
    "bwd_delta_sign": ("for (j = lo; j < hi; ++j) ds[j] = p[j] * (ds[j] - delta);",
                       "for (j = lo; j < hi; ++j) ds[j] = p[j] * (ds[j] + delta);"),
    "bwd_dq_scale_dropped": ("for (d = 0; d < D; ++d) dqi[d] *= scale;", ""),
    "bwd_dk_scale_dropped": ("dK[j * D + d] += scale * ds[j] * qi[d];",
                             "dK[j * D + d] += ds[j] * qi[d];"),
    "bwd_dk_uses_keys": ("dK[j * D + d] += scale * ds[j] * qi[d];",
                         "dK[j * D + d] += scale * ds[j] * K[j * D + d];"),
    "bwd_dv_uses_ds": ("dV[j * D + d] += p[j] * doi[d];", "dV[j * D + d] += ds[j] * doi[d];"),
    "bwd_dp_uses_keys": ("for (d = 0; d < D; ++d) dot += doi[d] * V[j * D + d];\n        ds[j] = dot;",
                         "for (d = 0; d < D; ++d) dot += doi[d] * K[j * D + d];\n        ds[j] = dot;"),
    "bwd_dq_uses_values": ("for (d = 0; d < D; ++d) dqi[d] += ds[j] * K[j * D + d];",
                           "for (d = 0; d < D; ++d) dqi[d] += ds[j] * V[j * D + d];"),
    "bwd_gqa_heads_not_summed": ("for (int64_t g = 0; g < group; ++g) {\n            const int64_t h = hkv * group + g;\n            for (int64_t i = 0; i < J->Lq; ++i) {\n                const int64_t id = (b * J->Hq + h) * J->Lq + i;",
                                 "for (int64_t g = 0; g < group; ++g) {\n            const int64_t h = hkv * group + g;\n            if (g) for (int64_t x = 0; x < J->Lk * J->D; ++x) dK[x] = dV[x] = 0.0;\n            for (int64_t i = 0; i < J->Lq; ++i) {\n                const int64_t id = (b * J->Hq + h) * J->Lq + i;"),
    "bwd_keys_lse_sign": ("exp(J->scale * dot - J->lse[g * J->Lq + i])",
                          "exp(J->scale * dot + J->lse[g * J->Lq + i])"),
    "bwd_keys_delta_dropped": ("pij * (dpv - J->delta[g * J->Lq + i])", "pij * dpv"),
    "bwd_keys_mask_ignored": ("if (j < lo || j >= hi) continue;\n                const int64_t id",
                              "const int64_t id"),
    "paged_prefill_top_left": ("if (i < ql) visible_range(i, ql, len, J->causal, -1, -1, &lo, &hi);",
                               "if (i < ql) visible_range(i, len, len, J->causal, -1, -1, &lo, &hi);"),
    "paged_prefill_rows_past_chunk": ("int64_t lo = 0, hi = 0; /* rows past the chunk see no key */\n                if (i < ql)",
                                      "int64_t lo = 0, hi = 0; /* rows past the chunk see no key */\n                if (1)"),
    "masked_row_nan": ("if (m == -INFINITY) { /* no visible key */",
                       "if (0) { /* no visible key */"),
}


@pytest.fixture(scope="module")
def mutant_results():
    """Builds every mutant and runs the pins on each in a process of its own (a mutant
    may overrun a buffer; a crash counts as caught). The processes run side by side."""
    src = open(os.path.join(os.path.dirname(oracle.__file__), "attn_oracle.c")).read()
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    tmp = tempfile.mkdtemp(prefix="oracle_mutants_")
    results = {}
    try:
        pending = []
        for name, (old, new) in sorted(MUTANTS.items()):
            if src.count(old) < 1:  # a shared pattern is planted everywhere it occurs
                results[name] = None
                continue
            c = os.path.join(tmp, name + ".c")
            so = os.path.join(tmp, name + ".so")
            with open(c, "w") as f:
                f.write(src.replace(old, new))
            subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fPIC", "-shared",
                                   "-pthread", "-o", so, c, "-lm"])
            pending.append((name, so))
        width = max(1, min(8, (os.cpu_count() or 2) // 2))
        running = []
        while pending or running:
            while pending and len(running) < width:
                name, so = pending.pop(0)
                proc = subprocess.Popen([sys.executable, "-c", _CHILD, so], cwd=root,
                                        stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                        text=True)
                running.append((name, proc))
            name, proc = running.pop(0)
            out, _ = proc.communicate(timeout=600)
            results[name] = out.split() if proc.returncode == 0 else [f"crash:{proc.returncode}"]
    finally:
        shutil.rmtree(tmp, ignore_errors=True)
    return results


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistakes(name, mutant_results):
    caught = mutant_results[name]
    assert caught is not None, f"mutation anchor for {name} not found"
    assert caught, f"no pin caught the planted mistake {name}"


_CHILD = """
import sys
import oracle
from tests import test_oracle as t
lib = oracle.load(sys.argv[1])
for pin in t.PINS:
    try:
        pin(lib)
    except (AssertionError, ValueError):
        print(pin.__name__)
"""
