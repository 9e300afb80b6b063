"""Oracle: plain fp64 CPU attention. TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg may
import this package. The library under ``tiled_attention_19_b200`` never does, and the
two share no code. The arithmetic lives in ``attn_oracle.c``: a literal, row-by-row
statement of softmax(Q K^T * scale [+ causal mask]) V in double precision, and of
its gradients by the chain rule (see that file's header for the definition each step
follows). This module only builds the
shared object and marshals arrays into it.

Inputs may be any floating torch tensor (or numpy array); they are widened to fp64
exactly, so the oracle sees the same fp16/bf16 values the GPU sees.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_libs: dict = {}

_dp = ctypes.POINTER(ctypes.c_double)
_i32p = ctypes.POINTER(ctypes.c_int32)
_i64p = ctypes.POINTER(ctypes.c_int64)
_i64 = ctypes.c_int64


def build(force: bool = False) -> str:
    """Compile attn_oracle.c into liboracle.so (IEEE double, no fast-math)."""
    stale = (not os.path.exists(_LIB_PATH)) or (
        os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
                               "-shared", "-pthread", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def load(path: str | None = None):
    """The oracle library handle (built on first use). ``path`` loads another build of
    the same source, which only the pin-sensitivity tests use."""
    key = path or _LIB_PATH
    if key not in _libs:
        if path is None:
            build()
        lib = ctypes.CDLL(key)
        lib.oracle_attn_fwd.argtypes = [_dp, _dp, _dp, _dp, _dp, _i64, _i64, _i64, _i64, _i64,
                                        _i64, ctypes.c_double, ctypes.c_int, ctypes.c_int]
        lib.oracle_attn_fwd_window.argtypes = [_dp, _dp, _dp, _dp, _dp, _i64, _i64, _i64, _i64,
                                               _i64, _i64, ctypes.c_double, ctypes.c_int, _i64,
                                               _i64, ctypes.c_int]
        lib.oracle_attn_fwd_rows.argtypes = [_dp, _dp, _dp, _i64p, _i64, _dp, _dp, _i64, _i64,
                                             _i64, _i64, _i64, _i64, ctypes.c_double,
                                             ctypes.c_int, ctypes.c_int]
        lib.oracle_attn_probs.argtypes = [_dp, _dp, _dp, _dp, _i64, _i64, _i64, _i64, _i64,
                                          _i64, ctypes.c_double, ctypes.c_int]
        lib.oracle_attn_paged.argtypes = [_dp, _dp, _dp, _i32p, _i32p, _i64, _dp, _dp, _i64,
                                          _i64, _i64, _i64, _i64, _i64, ctypes.c_double,
                                          ctypes.c_int]
        lib.oracle_attn_bwd.argtypes = [_dp, _dp, _dp, _dp, _dp, _dp, _dp, _dp, _dp, _dp, _i64,
                                        _i64, _i64, _i64, _i64, _i64, ctypes.c_double,
                                        ctypes.c_int, _i64, _i64, ctypes.c_int]
        lib.oracle_attn_bwd_dq_rows.argtypes = [_dp, _dp, _dp, _dp, _i64p, _i64, _dp, _dp, _i64,
                                                _i64, _i64, _i64, _i64, _i64, ctypes.c_double,
                                                ctypes.c_int, ctypes.c_int]
        lib.oracle_attn_bwd_dkv_keys.argtypes = [_dp, _dp, _dp, _dp, _i64p, _i64, _dp, _dp, _dp,
                                                 _dp, _i64, _i64, _i64, _i64, _i64, _i64,
                                                 ctypes.c_double, ctypes.c_int, ctypes.c_int]
        lib.oracle_attn_paged_prefill.argtypes = [_dp, _dp, _dp, _i32p, _i32p, _i32p, _i64, _dp,
                                                  _dp, _i64, _i64, _i64, _i64, _i64, _i64, _i64,
                                                  ctypes.c_double, ctypes.c_int, ctypes.c_int]
        lib.oracle_attn_paged_prefill.restype = ctypes.c_int
        for f in (lib.oracle_attn_fwd, lib.oracle_attn_fwd_rows, lib.oracle_attn_probs,
                  lib.oracle_attn_paged, lib.oracle_attn_fwd_window, lib.oracle_attn_bwd,
                  lib.oracle_attn_bwd_dq_rows, lib.oracle_attn_bwd_dkv_keys):
            f.restype = ctypes.c_int
        _libs[key] = lib
    return _libs[key]


def _f64(x) -> np.ndarray:
    if isinstance(x, torch.Tensor):
        x = x.detach().to("cpu", torch.float64).contiguous().numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(a: np.ndarray, ty=_dp):
    return a.ctypes.data_as(ty)


def default_threads() -> int:
    return max(1, os.cpu_count() or 1)


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise ValueError(f"oracle {what} failed with code {rc}")


def attn_fwd(q, k, v, scale: float, causal: bool = False, threads: int | None = None,
             lib=None):
    """Full attention. q[B,Hq,Lq,D], k/v[B,Hkv,Lk,D] -> (out[B,Hq,Lq,D], lse[B,Hq,Lq]) fp64."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, Lq, D = q.shape
    Hkv, Lk = k.shape[1], k.shape[2]
    assert k.shape == (B, Hkv, Lk, D) and v.shape == k.shape
    out = np.zeros((B, Hq, Lq, D), np.float64)
    lse = np.zeros((B, Hq, Lq), np.float64)
    rc = (lib or load()).oracle_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv,
                                 Lq, Lk, D, float(scale), int(bool(causal)),
                                 threads or default_threads())
    _check(rc, "attn_fwd")
    return torch.from_numpy(out), torch.from_numpy(lse)


def attn_fwd_window(q, k, v, scale: float, causal: bool = False, window=(-1, -1),
                    threads: int | None = None, lib=None):
    """Sliding-window attention, window = (left, right) with -1 = unbounded on that side."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, Lq, D = q.shape
    Hkv, Lk = k.shape[1], k.shape[2]
    out = np.zeros((B, Hq, Lq, D), np.float64)
    lse = np.zeros((B, Hq, Lq), np.float64)
    rc = (lib or load()).oracle_attn_fwd_window(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse),
                                                B, Hq, Hkv, Lq, Lk, D, float(scale),
                                                int(bool(causal)), int(window[0]), int(window[1]),
                                                threads or default_threads())
    _check(rc, "attn_fwd_window")
    return torch.from_numpy(out), torch.from_numpy(lse)


def attn_fwd_rows(q, k, v, rows, scale: float, causal: bool = False,
                  threads: int | None = None, lib=None):
    """Selected rows only. rows: flattened ids (b*Hq + h)*Lq + i -> (out[n,D], lse[n])."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, Lq, D = q.shape
    Hkv, Lk = k.shape[1], k.shape[2]
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1))
    n = rows.shape[0]
    out = np.zeros((n, D), np.float64)
    lse = np.zeros((n,), np.float64)
    rc = (lib or load()).oracle_attn_fwd_rows(_ptr(q), _ptr(k), _ptr(v), _ptr(rows, _i64p), n,
                                      _ptr(out), _ptr(lse), B, Hq, Hkv, Lq, Lk, D,
                                      float(scale), int(bool(causal)),
                                      threads or default_threads())
    _check(rc, "attn_fwd_rows")
    return torch.from_numpy(out), torch.from_numpy(lse)


def attn_probs(q, k, v, scale: float, causal: bool = False, lib=None):
    """The softmax matrix P[B,Hq,Lq,Lk] in fp64 (small problems only)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, Lq, D = q.shape
    Hkv, Lk = k.shape[1], k.shape[2]
    probs = np.zeros((B, Hq, Lq, Lk), np.float64)
    rc = (lib or load()).oracle_attn_probs(_ptr(q), _ptr(k), _ptr(v), _ptr(probs), B, Hq, Hkv, Lq, Lk,
                                   D, float(scale), int(bool(causal)))
    _check(rc, "attn_probs")
    return torch.from_numpy(probs)


def attn_paged(q, k_cache, v_cache, block_table, seq_lens, scale: float,
               threads: int | None = None, lib=None):
    """Paged decode. q[S,Hq,D]; caches [NB,Hkv,bs,D]; block_table[S,MB] int32;
    seq_lens[S] int32 -> (out[S,Hq,D], lse[S,Hq]) fp64."""
    q, kc, vc = _f64(q), _f64(k_cache), _f64(v_cache)
    bt = np.ascontiguousarray(torch.as_tensor(block_table).to(torch.int32).numpy())
    sl = np.ascontiguousarray(torch.as_tensor(seq_lens).to(torch.int32).numpy())
    S, Hq, D = q.shape
    NB, Hkv, bs, _ = kc.shape
    MB = bt.shape[1] if bt.ndim == 2 else 0
    out = np.zeros((S, Hq, D), np.float64)
    lse = np.zeros((S, Hq), np.float64)
    rc = (lib or load()).oracle_attn_paged(_ptr(q), _ptr(kc), _ptr(vc), _ptr(bt, _i32p),
                                   _ptr(sl, _i32p), bs, _ptr(out), _ptr(lse), S, Hq, Hkv, D,
                                   MB, NB, float(scale), threads or default_threads())
    _check(rc, "attn_paged")
    return torch.from_numpy(out), torch.from_numpy(lse)


def attn_bwd(q, k, v, dout, scale: float, causal: bool = False, window=(-1, -1),
             threads: int | None = None, lib=None, sensitivity: bool = False):
    """Gradients of attention given dout = dLoss/dO: (dq[B,Hq,Lq,D], dk[B,Hkv,Lk,D],
    dv[B,Hkv,Lk,D]) in fp64. window = (left, right) as in attn_fwd_window. With
    sensitivity=True, also (mq, mk, mv): each element's first-order rounding
    sensitivity (see attn_oracle.c), which the tests' tolerances scale with."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, Hq, Lq, D = q.shape
    Hkv, Lk = k.shape[1], k.shape[2]
    assert k.shape == (B, Hkv, Lk, D) and v.shape == k.shape and do.shape == q.shape
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    m = (np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)) if sensitivity else None
    mp = (_ptr(m[0]), _ptr(m[1]), _ptr(m[2])) if m else (None, None, None)
    rc = (lib or load()).oracle_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(do), _ptr(dq), _ptr(dk),
                                         _ptr(dv), *mp, B, Hq, Hkv, Lq, Lk, D, float(scale),
                                         int(bool(causal)), int(window[0]), int(window[1]),
                                         threads or default_threads())
    _check(rc, "attn_bwd")
    g = (torch.from_numpy(dq), torch.from_numpy(dk), torch.from_numpy(dv))
    return g + tuple(torch.from_numpy(a) for a in m) if m else g


def attn_bwd_dq_rows(q, k, v, dout, rows, scale: float, causal: bool = False,
                     threads: int | None = None, lib=None, sensitivity: bool = False):
    """dq of selected query rows, ids (b*Hq + h)*Lq + i -> dq[n, D] fp64 (and mq[n, D]
    with sensitivity=True)."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, Hq, Lq, D = q.shape
    Hkv, Lk = k.shape[1], k.shape[2]
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1))
    dq = np.zeros((rows.shape[0], D), np.float64)
    mq = np.zeros_like(dq) if sensitivity else None
    rc = (lib or load()).oracle_attn_bwd_dq_rows(_ptr(q), _ptr(k), _ptr(v), _ptr(do),
                                                 _ptr(rows, _i64p), rows.shape[0], _ptr(dq),
                                                 _ptr(mq) if mq is not None else None, B, Hq,
                                                 Hkv, Lq, Lk, D, float(scale), int(bool(causal)),
                                                 threads or default_threads())
    _check(rc, "attn_bwd_dq_rows")
    if sensitivity:
        return torch.from_numpy(dq), torch.from_numpy(mq)
    return torch.from_numpy(dq)


def attn_bwd_dkv_keys(q, k, v, dout, keys, scale: float, causal: bool = False,
                      threads: int | None = None, lib=None, sensitivity: bool = False):
    """dk, dv of selected keys, ids (b*Hkv + h_kv)*Lk + j -> (dk[n, D], dv[n, D]) fp64
    (and mk, mv with sensitivity=True)."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, Hq, Lq, D = q.shape
    Hkv, Lk = k.shape[1], k.shape[2]
    keys = np.ascontiguousarray(np.asarray(keys, dtype=np.int64).reshape(-1))
    dk = np.zeros((keys.shape[0], D), np.float64)
    dv = np.zeros((keys.shape[0], D), np.float64)
    m = (np.zeros_like(dk), np.zeros_like(dv)) if sensitivity else None
    rc = (lib or load()).oracle_attn_bwd_dkv_keys(_ptr(q), _ptr(k), _ptr(v), _ptr(do),
                                                  _ptr(keys, _i64p), keys.shape[0], _ptr(dk),
                                                  _ptr(dv), _ptr(m[0]) if m else None,
                                                  _ptr(m[1]) if m else None, B, Hq, Hkv, Lq, Lk,
                                                  D, float(scale), int(bool(causal)),
                                                  threads or default_threads())
    _check(rc, "attn_bwd_dkv_keys")
    g = (torch.from_numpy(dk), torch.from_numpy(dv))
    return g + tuple(torch.from_numpy(a) for a in m) if m else g


def attn_paged_prefill(q, k_cache, v_cache, block_table, seq_lens, scale: float,
                       causal: bool = True, q_lens=None, threads: int | None = None, lib=None):
    """Prefill over a paged cache. q[S,Hq,Lq,D]: each sequence's chunk of queries, its
    last q_lens[s] positions (all Lq if q_lens is None); caches [NB,Hkv,bs,D];
    block_table[S,MB]; seq_lens[S] -> (out[S,Hq,Lq,D], lse[S,Hq,Lq]) fp64. Rows past a
    sequence's chunk come out as rows with no key (0, -inf)."""
    q, kc, vc = _f64(q), _f64(k_cache), _f64(v_cache)
    bt = np.ascontiguousarray(torch.as_tensor(block_table).to(torch.int32).numpy())
    sl = np.ascontiguousarray(torch.as_tensor(seq_lens).to(torch.int32).numpy())
    ql = None if q_lens is None else np.ascontiguousarray(
        torch.as_tensor(q_lens).to(torch.int32).numpy())
    S, Hq, Lq, D = q.shape
    NB, Hkv, bs, _ = kc.shape
    MB = bt.shape[1] if bt.ndim == 2 else 0
    out = np.zeros((S, Hq, Lq, D), np.float64)
    lse = np.zeros((S, Hq, Lq), np.float64)
    rc = (lib or load()).oracle_attn_paged_prefill(
        _ptr(q), _ptr(kc), _ptr(vc), _ptr(bt, _i32p), _ptr(sl, _i32p),
        _ptr(ql, _i32p) if ql is not None else None, bs, _ptr(out), _ptr(lse), S, Hq, Hkv, Lq, D,
        MB, NB, float(scale), int(bool(causal)), threads or default_threads())
    _check(rc, "attn_paged_prefill")
    return torch.from_numpy(out), torch.from_numpy(lse)
