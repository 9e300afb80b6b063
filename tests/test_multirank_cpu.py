"""The multi-GPU bench path on CPU: two gloo ranks on 127.0.0.1.

bench.py runs independent replicas (the hot path shards with no exchange): each rank
times its own step, the job time is the slowest rank's (max over ranks), and the job
throughput is all ranks' work over that time. These tests run that host-side logic
with world_size 2 on the gloo backend.
"""
from __future__ import annotations

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, ws: int, port: int, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(ws), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=ws)
    try:
        got_ws, got_rank, got_local = bench.dist_env()
        bench.barrier(ws)
        mine = 10.0 + 5.0 * rank            # this rank's step time (ms)
        mx = bench.reduce_max(mine, ws, "cpu")
        rate = bench.job_rate(2.0e12, mx, ws, 1e12)  # 2 TFLOP per rank per step
        bench.barrier(ws)
        out[rank] = (got_ws, got_rank, got_local, mx, rate)
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_gloo_ranks_take_the_slowest_rank_and_sum_the_work():
    ws = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(ws, _free_port(), out), nprocs=ws, join=True)
        res = dict(out)
    for rank in range(ws):
        got_ws, got_rank, got_local, mx, rate = res[rank]
        assert (got_ws, got_rank, got_local) == (2, rank, rank)
        assert mx == 15.0                       # max over ranks, not the rank's own
        assert rate == pytest.approx(2 * 2.0e12 / 15e-3 / 1e12)


def test_job_rate_single_rank_and_degenerate_times():
    assert bench.job_rate(1e12, 1.0, 1, 1e12) == pytest.approx(1000.0)
    assert bench.job_rate(1e12, 0.0, 1, 1e12) is None
    assert bench.job_rate(1e12, float("nan"), 1, 1e12) is None


def test_reference_arm_prints_only_on_rank_zero(monkeypatch):
    class A:
        steps, warmup, cpu_seconds = 1, 3, 0.1
    assert bench.run_reference(A(), 2, 1) is None   # rank 1: no work, exits quietly


def test_decode_seqs_option_scales_the_decode_workload(monkeypatch, capsys):
    """--decode-seqs N swaps in the decode workload with N sequences (same heads, length
    distribution and seed); the reference arm, which runs on the host, reports it."""
    import json
    monkeypatch.setattr(bench, "DECODE", bench.DECODE)    # main() rebinds the workloads
    monkeypatch.setattr(bench, "PREFILL", bench.PREFILL)
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert bench.main(["--impl", "reference", "--decode-seqs", "4", "--steps", "1",
                       "--warmup", "3", "--cpu-seconds", "0.2"]) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert "paged_decode_s4_hq12_hkv2_d128_bf16" in line["config"]["workload"]
    assert bench.DECODE.num_seqs == 4 and bench.DECODE.Hq == 12 and bench.DECODE.seed == 5
    with pytest.raises(SystemExit):
        bench.main(["--decode-seqs", "0"])


def test_peaks_file_missing_keys_and_nesting(tmp_path):
    # No file: every figure is the fallback.
    peaks, src = bench.load_peaks(str(tmp_path / "absent.json"))
    assert src == "fallback" and peaks == bench.PEAKS_FALLBACK
    # Nested objects are searched; a key the file lacks takes its fallback, and the
    # label names it.
    p = tmp_path / "peaks.json"
    p.write_text('{"hbm": {"hbm_gbs": 6530.0}, "gemm": {"bf16_tflops": 1626.0}}')
    peaks, src = bench.load_peaks(str(p))
    assert peaks["hbm_gbs"] == 6530.0 and peaks["bf16_tflops"] == 1626.0
    assert peaks["bf16_tflops_sustained"] == bench.PEAKS_FALLBACK["bf16_tflops_sustained"]
    assert src == "measured (fallback for bf16_tflops_sustained)"
    p.write_text('{"hbm_gbs": 6530, "bf16_tflops": 1626, "bf16_tflops_sustained": 1402}')
    peaks, src = bench.load_peaks(str(p))
    assert src == "measured" and peaks["bf16_tflops_sustained"] == 1402.0
    # An unreadable file is the fallback, not a crash.
    p.write_text("{not json")
    assert bench.load_peaks(str(p))[1] == "fallback"
