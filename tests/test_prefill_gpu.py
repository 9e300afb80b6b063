"""Parity of attn_fwd (tcgen05 prefill kernel) with the fp64 oracle, on the GPU.

Every call goes through the C ABI (ctypes) of the in-tree library. Inputs are the
seeded generators' tensors; the oracle sees the identical f16/bf16 values widened to
fp64. Small shapes are compared element by element over every output; the full-size
workloads are run in the benchmark's launch configuration and compared on all outputs;
only the longest sequences the library accepts (2^22 keys or queries) are compared on
sampled rows.
"""
from __future__ import annotations

import math

import pytest
import torch

import oracle
import tiled_attention_19_b200 as ta
from tiled_attention_19_b200 import inputs
from tests.parity import check_parity, check_rounding_bound, guarded_empty, guards_intact

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def run(q, k, v, causal, scale, guard=False):
    B, Hq, Lq, D = q.shape
    qd, kd, vd = (t.to(DEV) for t in (q, k, v))
    if guard:
        ob, out, og = guarded_empty((B, Hq, Lq, D), q.dtype, DEV)
        lb, lse, lg = guarded_empty((B, Hq, Lq), torch.float32, DEV)
        ta.fwd(qd, kd, vd, causal=causal, scale=scale, out=out, lse=lse)
        torch.cuda.synchronize()
        assert guards_intact(ob, og), "write outside out"
        assert guards_intact(lb, lg), "write outside lse"
    else:
        out, lse = ta.fwd(qd, kd, vd, causal=causal, scale=scale)
        torch.cuda.synchronize()
    assert ta.device_status() == 0
    return out.cpu(), lse.cpu()


def spec(B, Hq, Hkv, Lq, Lk, D, dtype, causal, seed, scale=None):
    return inputs.DenseSpec("t", B, Hq, Hkv, Lq, Lk, D, dtype, causal,
                            scale if scale is not None else 1 / math.sqrt(D), seed)


SWEEP = []
for L in (1, 2, 15, 16, 17, 63, 64, 65, 127, 128, 129, 196, 255, 257, 1000):
    SWEEP.append((1, 2, 2, L, L, 64, torch.float16, False))
    SWEEP.append((1, 2, 1, L, L, 128, torch.bfloat16, True))
SWEEP += [
    (2, 4, 4, 300, 300, 64, torch.bfloat16, True),
    (2, 4, 4, 300, 300, 128, torch.float16, False),
    (1, 12, 2, 200, 200, 128, torch.bfloat16, True),   # GQA group 6
    (1, 8, 1, 130, 130, 64, torch.float16, True),      # MQA group 8
    (1, 4, 2, 257, 257, 64, torch.bfloat16, False),    # group 2
    (1, 2, 2, 100, 300, 64, torch.float16, True),      # Lq < Lk: bottom-right causal
    (1, 2, 2, 300, 100, 128, torch.float16, True),     # Lq > Lk: fully masked rows
    (1, 2, 2, 129, 700, 128, torch.bfloat16, False),   # Lq != Lk, ragged both
    (3, 3, 1, 1, 513, 64, torch.float16, True),        # single query row (decode-like)
    # grids of more than one wave (two query tiles per CTA); the small problems above run
    # with one query tile per CTA and the key tiles split between the softmax warpgroups
    (1, 160, 160, 300, 300, 64, torch.float16, True),
    (2, 96, 48, 257, 385, 128, torch.bfloat16, False),
]


@pytest.mark.parametrize("case", SWEEP, ids=lambda c: "B{}_H{}x{}_Lq{}_Lk{}_D{}_{}_{}".format(
    c[0], c[1], c[2], c[3], c[4], c[5], str(c[6]).split(".")[-1], "causal" if c[7] else "full"))
def test_prefill_sweep(case):
    B, Hq, Hkv, Lq, Lk, D, dtype, causal = case
    s = spec(B, Hq, Hkv, Lq, Lk, D, dtype, causal, seed=Lq * 7 + Lk + D)
    x = inputs.make(s)
    out, lse = run(x["q"], x["k"], x["v"], causal, s.scale, guard=True)
    ro, rl = oracle.attn_fwd(x["q"], x["k"], x["v"], s.scale, causal)
    check_parity(out, lse, ro, rl, dtype, str(case))


def test_lse_optional_and_deterministic():
    s = spec(1, 4, 2, 333, 333, 128, torch.bfloat16, True, seed=9)
    x = inputs.make(s)
    q, k, v = (t.to(DEV) for t in (x["q"], x["k"], x["v"]))
    o1, l1 = ta.fwd(q, k, v, causal=True, scale=s.scale)
    o2, l2 = ta.fwd(q, k, v, causal=True, scale=s.scale)
    o3, l3 = ta.fwd(q, k, v, causal=True, scale=s.scale, return_lse=False)
    torch.cuda.synchronize()
    assert l3 is None
    assert torch.equal(o1, o2) and torch.equal(l1, l2) and torch.equal(o1, o3)


@pytest.mark.parametrize("L,D,causal", [(400, 64, True), (1500, 64, False), (1100, 128, True),
                                         (2100, 128, False)])
def test_extreme_scores_stay_finite(L, D, causal):
    # Large-magnitude scores exercise the lazy rescaling path (the max moves by far
    # more than the threshold from tile to tile), over many key tiles per softmax
    # warpgroup in the longer cases.
    s = spec(1, 2, 2, L, L, D, torch.float16, causal, seed=10 + L)
    x = inputs.make(s)
    q = (x["q"].float() * 6).to(torch.float16)
    k = x["k"]
    ramp = torch.linspace(0, 8, L).view(1, 1, L, 1)
    k = (k.float() + ramp).to(torch.float16)  # later keys score ever higher
    out, lse = run(q, k, x["v"], causal, 0.5)
    ro, rl = oracle.attn_fwd(q, k, x["v"], 0.5, causal)
    m, _ = oracle.attn_fwd(q, k, x["v"].abs(), 0.5, causal)
    check_rounding_bound(out, lse, ro, rl, m, torch.float16, "extreme")
    if L == 400:  # a short case that also meets the fixed tolerance
        check_parity(out, lse, ro, rl, torch.float16, "extreme")


def test_empty_problems():
    q = torch.randn(1, 2, 0, 64, device=DEV, dtype=torch.float16)
    k = torch.randn(1, 2, 5, 64, device=DEV, dtype=torch.float16)
    out, lse = ta.fwd(q, k, k)  # Lq == 0: no-op
    assert out.numel() == 0
    q = torch.randn(2, 2, 37, 128, device=DEV, dtype=torch.bfloat16)
    k = torch.empty(2, 2, 0, 128, device=DEV, dtype=torch.bfloat16)
    out = torch.full_like(q, 3.0)
    out, lse = ta.fwd(q, k, k, out=out)  # no keys: O = 0, lse = -inf
    torch.cuda.synchronize()
    assert torch.all(out == 0) and torch.all(torch.isneginf(lse))


def test_rejects_bad_arguments_on_device():
    q = torch.randn(1, 2, 64, 96, device=DEV, dtype=torch.float16)
    with pytest.raises(ta.AttnError) as e:
        ta.fwd(q, q, q)
    assert e.value.code == -2
    raw = torch.empty(1 * 2 * 64 * 64 + 1, device=DEV, dtype=torch.float16)
    mis = raw[1:].view(1, 2, 64, 64)  # 2-byte offset: not 16-byte aligned
    ok = torch.randn(1, 2, 64, 64, device=DEV, dtype=torch.float16)
    with pytest.raises(ta.AttnError) as e:
        ta.fwd(mis, ok, ok)
    assert e.value.code == -3


# --------------------------------------------------------------- full-size workloads
FULL = ["sdpa_b1_h8_l512_d64_f16", "vit_b32_h12_n196_d64_f16", "sdpa_causal_b2_h8_l2048_d64_f16"]


@pytest.mark.parametrize("name", FULL)
def test_full_workload_all_outputs(name):
    s = inputs.WORKLOADS[name]
    x = inputs.make(s)
    out, lse = run(x["q"], x["k"], x["v"], s.causal, s.scale)
    ro, rl = oracle.attn_fwd(x["q"], x["k"], x["v"], s.scale, s.causal)
    check_parity(out, lse, ro, rl, s.dtype, name)


def test_long_prefill_all_rows():
    """The long causal prefill workload (B1 H16 L8192 D128 bf16) in the benchmark's launch
    configuration, compared with the oracle on every one of its 131,072 rows: every
    element of O and every lse (the oracle takes about 15 s of host time on 16 cores)."""
    s = inputs.WORKLOADS["prefill_causal_b1_h16_l8192_d128_bf16"]
    x = inputs.make(s)
    out, lse = run(x["q"], x["k"], x["v"], s.causal, s.scale)
    ro, rl = oracle.attn_fwd(x["q"], x["k"], x["v"], s.scale, s.causal)
    mx = check_parity(out, lse, ro, rl, s.dtype, "long prefill, all rows")
    print(f"long prefill: max |O err| {mx:.3e} over {ro.numel()} elements")
    # |O| never exceeds the largest |V| entry of its head (a convex combination of
    # value rows), up to the output rounding
    vmax = x["v"].float().abs().amax(dim=(2, 3)).view(1, s.Hq, 1, 1)
    assert torch.all(out.float().abs() <= vmax * (1 + 2 ** -7) + 1e-6)


@pytest.mark.parametrize("Lq,Lk,causal", [(256, 1 << 22, False), (1 << 22, 384, False),
                                          (1 << 22, 384, True)],
                         ids=["max_keys", "max_queries", "max_queries_causal"])
def test_maximum_sequence_lengths_sampled_rows(Lq, Lk, causal):
    """The longest sequences attn_fwd accepts (2^22 queries or keys; one head, D 64, bf16):
    32k key tiles streamed by one CTA, or 16k query tiles. With Lq > Lk the causal band
    is bottom-right aligned, so all but the last Lk rows see no key (O = 0, lse = -inf).
    The oracle checks sampled rows, including both sides of that edge."""
    s = inputs.DenseSpec("maxlen", 1, 1, 1, Lq, Lk, 64, torch.bfloat16, causal, 0.125,
                         seed=Lq % 1000 + Lk % 1000)
    x = inputs.make(s)
    out, lse = run(x["q"], x["k"], x["v"], causal, s.scale)
    g = torch.Generator().manual_seed(5)
    edge = Lq - Lk  # first row that sees a key under the causal mask
    picks = {0, 1, 127, 128, Lq - 1} | set(torch.randint(0, Lq, (3,), generator=g).tolist())
    if causal:
        picks |= {edge - 1, edge, edge + 1, edge + 127, edge + 128}
    rows = sorted(picks)
    ro, rl = oracle.attn_fwd_rows(x["q"], x["k"], x["v"], rows, s.scale, causal)
    rows_t = torch.tensor(rows)
    check_parity(out.reshape(-1, 64)[rows_t], lse.reshape(-1)[rows_t], ro, rl, s.dtype,
                 f"Lq {Lq} Lk {Lk} causal {causal}")
    if causal:
        assert torch.count_nonzero(out[0, 0, :edge]) == 0
        assert torch.all(lse[0, 0, :edge] == -math.inf)
        assert torch.isfinite(lse[0, 0, edge:]).all()
    else:
        assert torch.isfinite(lse).all()
