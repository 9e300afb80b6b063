"""Launches that depend on the previous kernel's output, back to back on one stream.

The prefill and decode kernels are launched with programmatic stream serialisation:
each may start while the previous kernel of the stream is still running, and must wait
(griddepcontrol.wait) before it reads global memory. Here every call takes the previous
call's output as its query, with no synchronisation in between; the chain must give the
same bits as the same chain with a device synchronisation after every call.
"""
from __future__ import annotations

import dataclasses

import pytest
import torch

import tiled_attention_19_b200 as ta
from tiled_attention_19_b200 import inputs

pytestmark = pytest.mark.gpu
DEV = "cuda:0"

DENSE = [
    # split key tiles at D = 64 (set-up before the wait), three S buffers
    inputs.DenseSpec("c1", 1, 8, 8, 512, 512, 64, torch.float16, False, 0.125, 41),
    # the causal SDPA shape (split, mixed buffer counts)
    inputs.DenseSpec("c3", 2, 8, 8, 2048, 2048, 64, torch.float16, True, 0.125, 42),
    # two query tiles per CTA at D = 128, more CTAs than SMs
    inputs.DenseSpec("c4s", 1, 16, 16, 2304, 2304, 128, torch.bfloat16, True, 0.088, 43),
]


def _dense_chain(spec, x, sync, n=8):
    q = x["q"]
    outs = []
    for _ in range(n):
        q, _ = ta.fwd(q, x["k"], x["v"], causal=spec.causal, scale=spec.scale)
        if sync:
            torch.cuda.synchronize()
        outs.append(q)
    torch.cuda.synchronize()
    return outs


@pytest.mark.parametrize("spec", DENSE, ids=[s.name for s in DENSE])
def test_prefill_chain_reads_the_previous_output(spec):
    x = {k: v.to(DEV) for k, v in inputs.make(spec).items()}
    if spec.Hq != spec.Hkv:
        pytest.skip("the output is the next query only when the head counts match")
    ref = _dense_chain(spec, x, sync=True)
    got = _dense_chain(spec, x, sync=False)
    assert ta.device_status() == 0
    for i, (a, b) in enumerate(zip(got, ref)):
        assert torch.equal(a, b), f"{spec.name}: call {i} differs from the synchronised chain"


def _decode_chain(s, x, ws, sync, n=8):
    q = x["q"]
    outs = []
    for _ in range(n):
        q, _ = ta.fwd_paged(q, x["k_cache"], x["v_cache"], x["block_table"], x["seq_lens"],
                            scale=s.scale, workspace=ws)
        if sync:
            torch.cuda.synchronize()
        outs.append(q)
    torch.cuda.synchronize()
    return outs


def test_decode_chain_reads_the_previous_output():
    s = dataclasses.replace(inputs.WORKLOADS["paged_decode_s16_hq12_hkv2_d128_bf16"], seed=44)
    x = {k: v.to(DEV) for k, v in inputs.make(s).items()}
    ws = ta.paged_workspace(s.num_seqs, s.Hq, s.Hkv, s.D, s.max_blocks, DEV)
    ref = _decode_chain(s, x, ws, sync=True)
    got = _decode_chain(s, x, ws, sync=False)
    assert ta.device_status() == 0
    for i, (a, b) in enumerate(zip(got, ref)):
        assert torch.equal(a, b), f"decode call {i} differs from the synchronised chain"
