"""Seeded synthetic inputs, shared by the tests and the benchmark.

This module holds no attention arithmetic: it only draws random tensors with the
shapes, dtypes and structure of the workloads on the pages, and knows nothing about
how attention is computed. Every draw comes from a CPU ``torch.Generator`` seeded
per workload, in fp32, then rounded once (round-to-nearest-even) to fp16/bf16, so
the oracle and the CUDA path see bit-identical inputs.

Workloads (shapes from the pages; sizes in the names):

* ``sdpa_b1_h8_l512_d64_f16`` -- q, k, v ~ N(0,1) ``[1,8,512,64]``, scale 1/8, full.
  Shape of the accuracy check in "Flash Attention" (hermes-agent-app.ru), Scenario 1
  step 4.
* ``vit_b32_h12_n196_d64_f16`` -- ViT-B/16 self-attention: X ~ N(0,1) ``[32,196,768]``,
  W_Q, W_K, W_V ~ N(0, 1/768); Q = X W_Q etc. in fp32, split into 12 heads of 64,
  laid out ``[B,H,N,d]``. "Self-attention, CUDA kernels and FlashAttention", section 1
  (224x224 image, 16x16 patches -> N = 196, D = 768, 12 heads).
* ``sdpa_causal_b2_h8_l2048_d64_f16`` -- q, k, v ~ N(0,1) ``[2,8,2048,64]``, scale 1/8,
  causal. Shape of the benchmark in "Flash Attention", Scenario 1 step 3.
* ``prefill_causal_b1_h16_l8192_d128_bf16`` -- q, k, v ~ N(0,1) ``[1,16,8192,128]``,
  scale 1/sqrt(128), causal: a long-context prefill.
* ``paged_decode_s16_hq12_hkv2_d128_bf16`` -- 16 sequences, one query token each,
  12 query heads sharing 2 K/V heads, block size 16 ("Fast attention kernels and
  operator fusion", section on paged attention). seq_lens ~ U{1..4096}; a pool of
  16*256 physical blocks; block_table = one random permutation of the pool;
  k_cache, v_cache ~ N(0,1) ``[4096,2,16,128]``; q ~ N(0,1) ``[16,12,128]``.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

F16 = torch.float16
BF16 = torch.bfloat16


@dataclass(frozen=True)
class DenseSpec:
    name: str
    B: int
    Hq: int
    Hkv: int
    Lq: int
    Lk: int
    D: int
    dtype: torch.dtype
    causal: bool
    scale: float
    seed: int
    gen: str = "iid"  # "iid" or "vit"

    @property
    def kind(self) -> str:
        return "dense"

    def flops(self) -> float:
        """Algorithmic FLOPs 4*B*Hq*Lq*Lk*D, halved for causal (the usual convention)."""
        f = 4.0 * self.B * self.Hq * self.Lq * self.Lk * self.D
        return f / 2 if self.causal else f


@dataclass(frozen=True)
class PagedSpec:
    name: str
    num_seqs: int
    Hq: int
    Hkv: int
    D: int
    block_size: int
    max_len: int
    dtype: torch.dtype
    scale: float
    seed: int
    min_len: int = 1
    fixed_lens: tuple = field(default=())  # if given, seq_lens are these values

    @property
    def kind(self) -> str:
        return "paged"

    @property
    def max_blocks(self) -> int:
        return (self.max_len + self.block_size - 1) // self.block_size

    @property
    def num_blocks(self) -> int:
        return self.num_seqs * self.max_blocks


WORKLOADS = {
    s.name: s
    for s in [
        DenseSpec("sdpa_b1_h8_l512_d64_f16", 1, 8, 8, 512, 512, 64, F16, False, 1 / 8, 1),
        DenseSpec("vit_b32_h12_n196_d64_f16", 32, 12, 12, 196, 196, 64, F16, False, 1 / 8, 2,
                  gen="vit"),
        DenseSpec("sdpa_causal_b2_h8_l2048_d64_f16", 2, 8, 8, 2048, 2048, 64, F16, True, 1 / 8, 3),
        DenseSpec("prefill_causal_b1_h16_l8192_d128_bf16", 1, 16, 16, 8192, 8192, 128, BF16, True,
                  1 / math.sqrt(128), 4),
        PagedSpec("paged_decode_s16_hq12_hkv2_d128_bf16", 16, 12, 2, 128, 16, 4096, BF16,
                  1 / math.sqrt(128), 5),
    ]
}


def _randn(g: torch.Generator, shape) -> torch.Tensor:
    return torch.randn(tuple(shape), generator=g, dtype=torch.float32)


def dense_inputs(spec: DenseSpec) -> dict:
    """q[B,Hq,Lq,D], k/v[B,Hkv,Lk,D] on the CPU in spec.dtype. Draw order: q, k, v."""
    g = torch.Generator().manual_seed(spec.seed)
    if spec.gen == "iid":
        q = _randn(g, (spec.B, spec.Hq, spec.Lq, spec.D))
        k = _randn(g, (spec.B, spec.Hkv, spec.Lk, spec.D))
        v = _randn(g, (spec.B, spec.Hkv, spec.Lk, spec.D))
    elif spec.gen == "vit":
        assert spec.Hq == spec.Hkv and spec.Lq == spec.Lk
        dm = spec.Hq * spec.D
        x = _randn(g, (spec.B, spec.Lq, dm))
        ws = [_randn(g, (dm, dm)) * (1.0 / math.sqrt(dm)) for _ in range(3)]

        def heads(t):  # [B,N,H*d] -> [B,H,N,d]
            return t.reshape(spec.B, spec.Lq, spec.Hq, spec.D).permute(0, 2, 1, 3).contiguous()

        q, k, v = (heads(x @ w) for w in ws)
    else:
        raise ValueError(spec.gen)
    return {"q": q.to(spec.dtype), "k": k.to(spec.dtype), "v": v.to(spec.dtype)}


def dense_grad_output(spec: DenseSpec) -> torch.Tensor:
    """dO = dLoss/dO for the backward pass: N(0,1) of q's shape in spec.dtype, from its
    own generator (seed + 1000003) so the forward inputs are unchanged."""
    g = torch.Generator().manual_seed(spec.seed + 1000003)
    return _randn(g, (spec.B, spec.Hq, spec.Lq, spec.D)).to(spec.dtype)


def backward_flops(spec: DenseSpec) -> float:
    """Algorithmic FLOPs of the backward pass: five D-deep products (S, dP, dV, dK, dQ)
    over the visible (query, key) pairs, 2.5 times the forward's."""
    return 2.5 * spec.flops()


def paged_inputs(spec: PagedSpec) -> dict:
    """Paged-decode inputs on the CPU. Draw order: seq_lens, block_table, k_cache,
    v_cache, q."""
    g = torch.Generator().manual_seed(spec.seed)
    if spec.fixed_lens:
        assert len(spec.fixed_lens) == spec.num_seqs
        seq_lens = torch.tensor(spec.fixed_lens, dtype=torch.int32)
    else:
        seq_lens = torch.randint(spec.min_len, spec.max_len + 1, (spec.num_seqs,), generator=g,
                                 dtype=torch.int64).to(torch.int32)
    nb, mb = spec.num_blocks, spec.max_blocks
    block_table = torch.randperm(nb, generator=g).to(torch.int32).reshape(spec.num_seqs, mb)
    k_cache = _randn(g, (nb, spec.Hkv, spec.block_size, spec.D)).to(spec.dtype)
    v_cache = _randn(g, (nb, spec.Hkv, spec.block_size, spec.D)).to(spec.dtype)
    q = _randn(g, (spec.num_seqs, spec.Hq, spec.D)).to(spec.dtype)
    return {"q": q, "k_cache": k_cache, "v_cache": v_cache, "block_table": block_table,
            "seq_lens": seq_lens}


def make(spec) -> dict:
    if isinstance(spec, str):
        spec = WORKLOADS[spec]
    return dense_inputs(spec) if spec.kind == "dense" else paged_inputs(spec)


def paged_bytes(spec: PagedSpec, seq_lens: torch.Tensor) -> int:
    """Minimum HBM bytes one paged-decode call must move: the K and V rows of every
    valid token, q, out, lse, the block-table entries in use and seq_lens."""
    el = torch.tensor([], dtype=spec.dtype).element_size()
    lens = seq_lens.to(torch.int64)
    tokens = int(lens.sum())
    blocks = int(((lens + spec.block_size - 1) // spec.block_size).sum())
    kv = tokens * spec.Hkv * spec.D * el * 2
    qo = 2 * spec.num_seqs * spec.Hq * spec.D * el
    return kv + qo + spec.num_seqs * spec.Hq * 4 + blocks * 4 + spec.num_seqs * 4


def dense_bytes(spec: DenseSpec) -> int:
    """Minimum HBM bytes of one dense call: q, k, v read once, out and lse written."""
    el = torch.tensor([], dtype=spec.dtype).element_size()
    q = spec.B * spec.Hq * spec.Lq * spec.D * el
    kv = 2 * spec.B * spec.Hkv * spec.Lk * spec.D * el
    return 2 * q + kv + spec.B * spec.Hq * spec.Lq * 4
