"""Many back-to-back launches per kernel form, inputs rotating through copies larger than
the L2, so that loads land late and out of order in every way the hand-offs between the
kernels' roles must survive. After the run the device status word must be clear (no
bounded wait expired, no index was out of range) and the outputs of the first input copy
must equal, bit for bit, those of its first launch: the kernels are deterministic, so any
difference would come from a hand-off race.
"""
from __future__ import annotations

import dataclasses

import pytest
import torch

import tiled_attention_19_b200 as ta
from tiled_attention_19_b200 import inputs

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
L2_BYTES = 126 * 1000 * 1000

# (name, spec, window, launches): each exercises one form of the prefill kernel
CASES = [
    # one query tile per CTA, key tiles split between the warpgroups, three S buffers
    ("split_d64_short", inputs.DenseSpec("r1", 1, 8, 8, 512, 512, 64, torch.float16, False, 0.125, 31),
     None, 3000),
    # the causal SDPA shape: split CTAs with and without the third S buffer
    ("split_d64_causal", inputs.DenseSpec("r2", 2, 8, 8, 2048, 2048, 64, torch.float16, True, 0.125, 32),
     None, 1500),
    # split at D = 128 (two S buffers)
    ("split_d128", inputs.DenseSpec("r3", 1, 4, 4, 2048, 2048, 128, torch.bfloat16, True, 0.088, 33),
     None, 1000),
    # two query tiles per CTA, paired K/V barriers
    ("paired_d128", inputs.DenseSpec("r4", 2, 48, 16, 1024, 1024, 128, torch.bfloat16, True, 0.088, 34),
     None, 300),
    # sliding window (the general issue loop)
    ("window_d64", inputs.DenseSpec("r5", 1, 80, 80, 1024, 1024, 64, torch.float16, False, 0.125, 35),
     (200, 30), 300),
]


def _copies(x, per):
    n = max(2, -(-2 * L2_BYTES // per))
    return [{k: v.clone() for k, v in x.items()} for _ in range(n)]


@pytest.mark.parametrize("name,spec,window,launches", CASES, ids=[c[0] for c in CASES])
def test_dense_repeated_launches(name, spec, window, launches):
    x = {k: v.to(DEV) for k, v in inputs.make(spec).items()}
    per = sum(t.numel() * t.element_size() for t in x.values())
    cps = _copies(x, per)
    outs = [torch.empty_like(x["q"]) for _ in cps]
    lses = [torch.empty(spec.B, spec.Hq, spec.Lq, device=DEV) for _ in cps]
    first = None
    for i in range(launches):
        c = i % len(cps)
        ta.fwd(cps[c]["q"], cps[c]["k"], cps[c]["v"], causal=spec.causal, scale=spec.scale,
               out=outs[c], lse=lses[c], window=window)
        if i == 0:
            torch.cuda.synchronize()
            first = (outs[0].clone(), lses[0].clone())
    torch.cuda.synchronize()
    assert ta.device_status() == 0, f"{name}: a bounded wait expired or an index was skipped"
    assert torch.equal(outs[0], first[0]) and torch.equal(lses[0], first[1]), name


def test_fp8_repeated_launches():
    spec = inputs.DenseSpec("r6", 1, 32, 8, 2048, 2048, 128, torch.bfloat16, True, 0.088, 36)
    x = inputs.make(spec)
    x8 = {k: v.to(DEV).to(torch.float8_e4m3fn) for k, v in x.items()}
    per = sum(t.numel() for t in x8.values())
    cps = _copies(x8, per)
    outs = [torch.empty(spec.B, spec.Hq, spec.Lq, spec.D, dtype=torch.bfloat16, device=DEV) for _ in cps]
    first = None
    for i in range(400):
        c = i % len(cps)
        ta.fwd_fp8(cps[c]["q"], cps[c]["k"], cps[c]["v"], causal=True, scale=spec.scale,
                   out=outs[c], return_lse=False)
        if i == 0:
            torch.cuda.synchronize()
            first = outs[0].clone()
    torch.cuda.synchronize()
    assert ta.device_status() == 0
    assert torch.equal(outs[0], first)


def test_paged_decode_repeated_launches():
    s = dataclasses.replace(inputs.WORKLOADS["paged_decode_s16_hq12_hkv2_d128_bf16"], seed=37)
    x = {k: v.to(DEV) for k, v in inputs.make(s).items()}
    per = sum(t.numel() * t.element_size() for t in x.values())
    cps = _copies(x, per)
    ws = ta.paged_workspace(s.num_seqs, s.Hq, s.Hkv, s.D, s.max_blocks, DEV)
    outs = [torch.empty_like(x["q"]) for _ in cps]
    lses = [torch.empty(s.num_seqs, s.Hq, device=DEV) for _ in cps]
    first = None
    for i in range(3000):
        c = i % len(cps)
        d = cps[c]
        ta.fwd_paged(d["q"], d["k_cache"], d["v_cache"], d["block_table"], d["seq_lens"],
                     scale=s.scale, out=outs[c], lse=lses[c], workspace=ws)
        if i == 0:
            torch.cuda.synchronize()
            first = (outs[0].clone(), lses[0].clone())
    torch.cuda.synchronize()
    assert ta.device_status() == 0
    assert torch.equal(outs[0], first[0]) and torch.equal(lses[0], first[1])
