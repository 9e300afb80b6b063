"""Failure detection on the GPU without a fault.

Every wait in the kernels is bounded: a wait that runs out reports ATTN_ERR_TIMEOUT in a
device status word and the kernel returns (no trap, no hang). The self-test entry point
makes such a wait run out on purpose (a barrier nothing completes); the host reads the
status, and the context must stay usable for the next call.
"""
from __future__ import annotations

import math

import pytest
import torch

import oracle
import tiled_attention_19_b200 as ta
from tiled_attention_19_b200 import inputs
from tests.parity import check_parity

pytestmark = pytest.mark.gpu


@pytest.mark.timeout(60)
def test_bounded_wait_reports_timeout_and_context_survives():
    assert ta.device_status() == 0
    assert ta.load().attn_selftest_bounded_wait(torch.cuda.current_stream().cuda_stream) == 0
    torch.cuda.synchronize()
    assert ta.device_status() == -6      # ATTN_ERR_TIMEOUT, read ...
    assert ta.device_status() == 0       # ... and cleared
    # the context is intact: an ordinary call still matches the oracle
    s = inputs.DenseSpec("after", 1, 2, 1, 130, 130, 64, torch.float16, True, 1 / math.sqrt(64), 41)
    x = inputs.make(s)
    out, lse = ta.fwd(x["q"].cuda(), x["k"].cuda(), x["v"].cuda(), causal=True, scale=s.scale)
    torch.cuda.synchronize()
    ro, rl = oracle.attn_fwd(x["q"], x["k"], x["v"], s.scale, True)
    check_parity(out.cpu(), lse.cpu(), ro, rl, s.dtype, "after timeout")
    assert ta.device_status() == 0
