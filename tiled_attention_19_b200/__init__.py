"""Python binding of libattn_b200: exact tiled attention forward and backward, and
paged-KV decode on B200 (sm_100a).

The binding only marshals arguments: tensors become raw device pointers and sizes, the
stream is torch's current stream, and every step of the computation runs in the CUDA
kernels behind the C ABI in ``include/attn.h``. There is no CPU fallback: if the
library is missing or the device is not sm_100, calls raise.

    out, lse = fwd(q, k, v, causal=True)                  # q [B,Hq,Lq,D], k/v [B,Hkv,Lk,D]
    dq, dk, dv = bwd(q, k, v, out, dout, lse, causal=True)
    out, lse = fwd_paged(q, k_cache, v_cache, block_table, seq_lens)
"""
from __future__ import annotations

import ctypes
import math
import os
import threading

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libattn_b200.so")

ATTN_F16, ATTN_BF16 = 0, 1
STATUS = {
    0: "ATTN_OK", -1: "ATTN_ERR_INVALID", -2: "ATTN_ERR_UNSUPPORTED", -3: "ATTN_ERR_MISALIGNED",
    -4: "ATTN_ERR_DEVICE", -5: "ATTN_ERR_CUDA", -6: "ATTN_ERR_TIMEOUT", -7: "ATTN_ERR_WORKSPACE",
    -8: "ATTN_ERR_BAD_INDEX", -9: "ATTN_ERR_SCRATCH_LIMIT",
}


class Strides(ctypes.Structure):
    """attn_strides_t: element strides over (batch, head, seq); D is contiguous."""
    _fields_ = [("batch", ctypes.c_int64), ("head", ctypes.c_int64), ("seq", ctypes.c_int64)]


# Every function include/attn.h declares, with its ctypes signature.
_vp, _i, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
_sp = ctypes.POINTER(Strides)
SIGNATURES = {
    "attn_fwd": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _i, _i, _vp]),
    "attn_fwd_window": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _i, _i, _i, _i,
                             _vp]),
    "attn_fwd_strided": (_i, [_vp, _sp, _vp, _sp, _vp, _sp, _vp, _sp, _vp, _i, _i, _i, _i, _i, _i,
                              _f, _i, _i, _i, _i, _vp]),
    "attn_fwd_paged_prefill": (_i, [_vp, _sp, _vp, _vp, _vp, _vp, _vp, _i, _vp, _sp, _vp, _i, _i,
                                    _i, _i, _i, _i, _i, _f, _i, _i, _vp]),
    "attn_fwd_fp8": (_i, [_vp, _sp, _vp, _sp, _vp, _sp, _vp, _sp, _vp, _i, _i, _i, _i, _i, _i, _f,
                          _f, _f, _f, _i, _vp]),
    "attn_paged_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i]),
    "attn_fwd_paged": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _vp, _vp, _i, _i, _i, _i, _i, _i, _f,
                            _i, _vp, _sz, _vp]),
    "attn_fwd_paged_noalloc": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _vp, _vp, _i, _i, _i, _i, _i,
                                    _i, _f, _i, _vp]),
    "attn_bwd_workspace_size": (_sz, [_i, _i, _i]),
    "attn_bwd": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _i,
                      _i, _vp, _sz, _vp]),
    "attn_bwd_window": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i,
                             _f, _i, _i, _i, _i, _vp, _sz, _vp]),
    "attn_bwd_strided": (_i, [_vp, _sp, _vp, _sp, _vp, _sp, _vp, _sp, _vp, _sp, _vp, _vp, _sp,
                              _vp, _sp, _vp, _sp, _i, _i, _i, _i, _i, _i, _f, _i, _i, _i, _i,
                              _vp, _sz, _vp]),
    "attn_error_string": (ctypes.c_char_p, [_i]),
    "attn_get_device_status": (_i, [_vp]),
    "attn_selftest_bounded_wait": (_i, [_vp]),
    "attn_selftest_fill_noalloc_scratch": (_i, [_i, _vp]),
}

_lib = None
_lock = threading.Lock()


class AttnError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {STATUS.get(code, code)} ({error_string(code)})")


def load(path: str = LIB_PATH):
    """The loaded C library. Raises if it has not been built (no fallback)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(path):
                raise RuntimeError(f"{path} is missing: build it with "
                                   "`python -m tiled_attention_19_b200.build`")
            lib = ctypes.CDLL(path)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
    return _lib


def error_string(code: int) -> str:
    return load().attn_error_string(int(code)).decode()


def _dtype_code(dt: torch.dtype) -> int:
    if dt == torch.float16:
        return ATTN_F16
    if dt == torch.bfloat16:
        return ATTN_BF16
    raise TypeError(f"unsupported dtype {dt}: float16 or bfloat16 only")


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        _on_current_device(stream.device, "stream")
        return stream.cuda_stream
    return int(stream)


def _on_current_device(device: torch.device, name: str) -> None:
    """The library launches its kernels on the calling thread's current CUDA device, so
    every tensor and stream of a call must live there."""
    cur = torch.cuda.current_device()
    if device.index != cur:
        raise ValueError(f"{name} is on {device} but the current CUDA device is cuda:{cur} "
                         "(select it with torch.cuda.set_device or torch.cuda.device)")


def _dev(t: torch.Tensor, name: str) -> int:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    _on_current_device(t.device, name)
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise AttnError(rc, what)


def _strides(t: torch.Tensor, name: str) -> Strides:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    _on_current_device(t.device, name)
    if t.dim() != 4 or t.stride(3) != 1:
        raise ValueError(f"{name} must be a 4-D view [B, H, L, D] with contiguous D")
    return Strides(t.stride(0), t.stride(1), t.stride(2))


def fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False,
        scale: float | None = None, out: torch.Tensor | None = None,
        lse: torch.Tensor | None = None, return_lse: bool = True, stream=None,
        window: tuple | None = None):
    """softmax(q k^T * scale [+ causal / window mask]) v.  q [B,Hq,Lq,D]; k, v [B,Hkv,Lk,D].
    window = (left, right) restricts query i to keys i'-left..i'+right (i' = i + Lk - Lq,
    -1 = unbounded). Returns (out [B,Hq,Lq,D], lse [B,Hq,Lq] fp32 or None). scale defaults
    to 1/sqrt(D). q, k, v and out may be any views with a contiguous last dimension (for
    example x.transpose(1, 2) of flash_attn's [B, L, H, D] tensors); those go through
    attn_fwd_strided, and a default out takes q's strides."""
    B, Hq, Lq, D = q.shape
    Hkv, Lk = k.shape[1], k.shape[2]
    if k.shape != (B, Hkv, Lk, D) or v.shape != k.shape:
        raise ValueError(f"shape mismatch q{tuple(q.shape)} k{tuple(k.shape)} v{tuple(v.shape)}")
    if q.dtype != k.dtype or q.dtype != v.dtype:
        raise TypeError("q, k, v must share a dtype")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty((B, Hq, Lq), dtype=torch.float32, device=q.device)
    if not all(t.is_contiguous() for t in (q, k, v, out)):
        st = [_strides(t, n) for t, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out"))]
        w = window if window is not None else (-1, -1)
        rc = load().attn_fwd_strided(q.data_ptr(), st[0], k.data_ptr(), st[1], v.data_ptr(), st[2],
                                     out.data_ptr(), st[3],
                                     _dev(lse, "lse") if lse is not None else None, B, Hq, Hkv,
                                     Lq, Lk, D, float(scale), int(bool(causal)), int(w[0]),
                                     int(w[1]), _dtype_code(q.dtype), _stream(stream))
        _check(rc, "attn_fwd_strided")
        return out, lse
    args = (_dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(out, "out"),
            _dev(lse, "lse") if lse is not None else None, B, Hq, Hkv, Lq, Lk, D, float(scale),
            int(bool(causal)))
    if window is None:
        rc = load().attn_fwd(*args, _dtype_code(q.dtype), _stream(stream))
        _check(rc, "attn_fwd")
    else:
        rc = load().attn_fwd_window(*args, int(window[0]), int(window[1]), _dtype_code(q.dtype),
                                    _stream(stream))
        _check(rc, "attn_fwd_window")
    return out, lse


def bwd_workspace_size(B: int, Hq: int, Lq: int) -> int:
    return int(load().attn_bwd_workspace_size(B, Hq, Lq))


def bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: torch.Tensor,
        dout: torch.Tensor, lse: torch.Tensor, causal: bool = False, scale: float | None = None,
        window: tuple | None = None, dq: torch.Tensor | None = None,
        dk: torch.Tensor | None = None, dv: torch.Tensor | None = None,
        workspace: torch.Tensor | None = None, stream=None):
    """Gradients (dq, dk, dv) of attention given dout = dLoss/dO, from the forward pass's
    inputs, output and lse (fwd with the same causal / window / scale). dk, dv have the
    K/V heads' shape. The workspace (attn_bwd_workspace_size bytes) is allocated when not
    given. Tensors may be any views with a contiguous last dimension (as fwd); those go
    through attn_bwd_strided, and default gradients take their inputs' strides."""
    B, Hq, Lq, D = q.shape
    Hkv, Lk = k.shape[1], k.shape[2]
    if k.shape != (B, Hkv, Lk, D) or v.shape != k.shape or out.shape != q.shape or \
            dout.shape != q.shape or tuple(lse.shape) != (B, Hq, Lq):
        raise ValueError("shape mismatch")
    if len({q.dtype, k.dtype, v.dtype, out.dtype, dout.dtype}) != 1:
        raise TypeError("q, k, v, out, dout must share a dtype")
    if lse.dtype != torch.float32:
        raise TypeError("lse must be float32")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if dq.shape != q.shape or dk.shape != k.shape or dv.shape != v.shape or \
            len({q.dtype, dq.dtype, dk.dtype, dv.dtype}) != 1:
        raise ValueError("dq, dk, dv must match q, k, v in shape and dtype")
    n = bwd_workspace_size(B, Hq, Lq)
    if workspace is None:
        workspace = torch.empty(max(n, 16), dtype=torch.uint8, device=q.device)
    ws_n = workspace.numel() * workspace.element_size()
    if not all(t.is_contiguous() for t in (q, k, v, out, dout, dq, dk, dv)):
        names = ("q", "k", "v", "out", "dout", "dq", "dk", "dv")
        st = [_strides(t, n) for t, n in zip((q, k, v, out, dout, dq, dk, dv), names)]
        w = window if window is not None else (-1, -1)
        rc = load().attn_bwd_strided(q.data_ptr(), st[0], k.data_ptr(), st[1], v.data_ptr(), st[2],
                                     out.data_ptr(), st[3], dout.data_ptr(), st[4],
                                     _dev(lse, "lse"), dq.data_ptr(), st[5], dk.data_ptr(), st[6],
                                     dv.data_ptr(), st[7], B, Hq, Hkv, Lq, Lk, D, float(scale),
                                     int(bool(causal)), int(w[0]), int(w[1]),
                                     _dtype_code(q.dtype), _dev(workspace, "workspace"), ws_n,
                                     _stream(stream))
        _check(rc, "attn_bwd_strided")
        return dq, dk, dv
    args = (_dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(out, "out"), _dev(dout, "dout"),
            _dev(lse, "lse"), _dev(dq, "dq"), _dev(dk, "dk"), _dev(dv, "dv"), B, Hq, Hkv, Lq, Lk,
            D, float(scale), int(bool(causal)))
    if window is None:
        rc = load().attn_bwd(*args, _dtype_code(q.dtype), _dev(workspace, "workspace"), ws_n,
                             _stream(stream))
        _check(rc, "attn_bwd")
    else:
        rc = load().attn_bwd_window(*args, int(window[0]), int(window[1]), _dtype_code(q.dtype),
                                    _dev(workspace, "workspace"), ws_n, _stream(stream))
        _check(rc, "attn_bwd_window")
    return dq, dk, dv


def fwd_fp8(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False,
            scale: float | None = None, descale=(1.0, 1.0, 1.0), out: torch.Tensor | None = None,
            lse: torch.Tensor | None = None, return_lse: bool = True, stream=None):
    """Attention on e4m3 inputs (torch.float8_e4m3fn views [B,H,L,D] with contiguous D);
    the values are q*descale[0], k*descale[1], v*descale[2]. Returns (out bf16, lse)."""
    B, Hq, Lq, D = q.shape
    Hkv, Lk = k.shape[1], k.shape[2]
    if k.shape != (B, Hkv, Lk, D) or v.shape != k.shape:
        raise ValueError("shape mismatch")
    if not all(t.dtype == torch.float8_e4m3fn for t in (q, k, v)):
        raise TypeError("q, k, v must be float8_e4m3fn")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty((B, Hq, Lq, D), dtype=torch.bfloat16, device=q.device)
    if out.dtype != torch.bfloat16:
        raise TypeError("out must be bfloat16")
    if lse is None and return_lse:
        lse = torch.empty((B, Hq, Lq), dtype=torch.float32, device=q.device)
    rc = load().attn_fwd_fp8(q.data_ptr(), _strides(q, "q"), k.data_ptr(), _strides(k, "k"),
                             v.data_ptr(), _strides(v, "v"), out.data_ptr(), _strides(out, "out"),
                             _dev(lse, "lse") if lse is not None else None, B, Hq, Hkv, Lq, Lk, D,
                             float(scale), float(descale[0]), float(descale[1]), float(descale[2]),
                             int(bool(causal)), _stream(stream))
    _check(rc, "attn_fwd_fp8")
    return out, lse


def paged_workspace_size(num_seqs: int, Hq: int, Hkv: int, D: int, max_blocks_per_seq: int,
                         block_size: int = 16) -> int:
    return int(load().attn_paged_workspace_size(num_seqs, Hq, Hkv, D, max_blocks_per_seq,
                                                block_size))


_workspaces: dict = {}


def paged_workspace(num_seqs: int, Hq: int, Hkv: int, D: int, max_blocks_per_seq: int,
                    device, block_size: int = 16) -> torch.Tensor | None:
    """A zero-filled workspace for these sizes, cached per device. Completed calls leave
    its counters at zero, so it is reused as is."""
    n = paged_workspace_size(num_seqs, Hq, Hkv, D, max_blocks_per_seq, block_size)
    if n == 0:
        return None
    device = torch.device(device)
    key = (device.index, n)
    ws = _workspaces.get(key)
    if ws is None:
        ws = torch.zeros(n, dtype=torch.uint8, device=device)
        _workspaces[key] = ws
    return ws


def fwd_paged(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
              block_table: torch.Tensor, seq_lens: torch.Tensor, scale: float | None = None,
              out: torch.Tensor | None = None, lse: torch.Tensor | None = None,
              return_lse: bool = True, workspace: torch.Tensor | None = None, stream=None):
    """Decode attention over a paged cache. q [S,Hq,D]; k_cache, v_cache [NB,Hkv,16,D];
    block_table [S,MB] int32; seq_lens [S] int32. Returns (out [S,Hq,D], lse [S,Hq])."""
    S, Hq, D = q.shape
    NB, Hkv, bs, D2 = k_cache.shape
    if v_cache.shape != k_cache.shape or D2 != D:
        raise ValueError("cache shape mismatch")
    if block_table.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise TypeError("block_table and seq_lens must be int32")
    MB = block_table.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty((S, Hq), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = paged_workspace(S, Hq, Hkv, D, MB, q.device, bs)
    ws_ptr = _dev(workspace, "workspace") if workspace is not None else None
    ws_n = workspace.numel() * workspace.element_size() if workspace is not None else 0
    rc = load().attn_fwd_paged(_dev(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
                               _dev(block_table, "block_table"), _dev(seq_lens, "seq_lens"), bs,
                               _dev(out, "out"), _dev(lse, "lse") if lse is not None else None,
                               S, Hq, Hkv, D, MB, NB, float(scale), _dtype_code(q.dtype), ws_ptr,
                               ws_n, _stream(stream))
    _check(rc, "attn_fwd_paged")
    return out, lse


def fwd_paged_prefill(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                      block_table: torch.Tensor, seq_lens: torch.Tensor,
                      q_lens: torch.Tensor | None = None, causal: bool = True,
                      scale: float | None = None, out: torch.Tensor | None = None,
                      lse: torch.Tensor | None = None, return_lse: bool = True, stream=None):
    """Prefill over a paged cache. q [S,Hq,Lq,D] (any view with contiguous D): sequence
    s's chunk is its first q_lens[s] rows (all Lq if q_lens is None), at the sequence's
    last positions; caches [NB,Hkv,16,D]; block_table [S,MB] int32; seq_lens [S] int32
    (keys, including the chunk's). Returns (out [S,Hq,Lq,D], lse [S,Hq,Lq])."""
    S, Hq, Lq, D = q.shape
    NB, Hkv, bs, D2 = k_cache.shape
    if v_cache.shape != k_cache.shape or D2 != D:
        raise ValueError("cache shape mismatch")
    if block_table.dtype != torch.int32 or seq_lens.dtype != torch.int32 or \
            (q_lens is not None and q_lens.dtype != torch.int32):
        raise TypeError("block_table, seq_lens and q_lens must be int32")
    MB = block_table.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty((S, Hq, Lq), dtype=torch.float32, device=q.device)
    rc = load().attn_fwd_paged_prefill(
        q.data_ptr(), _strides(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
        _dev(block_table, "block_table"), _dev(seq_lens, "seq_lens"),
        _dev(q_lens, "q_lens") if q_lens is not None else None, bs, out.data_ptr(),
        _strides(out, "out"), _dev(lse, "lse") if lse is not None else None, S, Hq, Hkv, Lq, D, MB,
        NB, float(scale), int(bool(causal)), _dtype_code(q.dtype), _stream(stream))
    _check(rc, "attn_fwd_paged_prefill")
    return out, lse


def device_status(stream=None) -> int:
    """Read and clear the device-side status word (0 = nothing reported)."""
    return int(load().attn_get_device_status(_stream(stream)))
