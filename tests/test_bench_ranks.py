"""Host logic of the multi-GPU benchmark, run as two gloo ranks on the CPU.

The path shards by independent prompts (replicas, weak scaling): every rank draws
its own prompts and noise, nothing is exchanged on the data path, and the only
collective is the maximum of the per-rank timings.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime

    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # rank r "took" 10*(r+1) ms and 7 - r ms on its two timings
        got = bench.max_over_ranks([10.0 * (rank + 1), 7.0 - rank], torch.device("cpu"), world)
        emb, null, noise, lengths = bench.rank_inputs(rank)
        q.put((rank, got, float(emb.sum()), float(noise.sum()), float(np.abs(null).sum()), lengths.tolist()))
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_and_distinct_inputs():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = {}
    for _ in procs:
        r, *rest = q.get(timeout=120)
        res[r] = rest
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in (0, 1):
        assert res[r][0] == [20.0, 7.0]           # max over ranks, element-wise
        assert res[r][3] == 0.0                    # null embedding is zero
        assert res[r][4] == [bench.WORKLOAD["frames"]] * bench.WORKLOAD["batch"]
    assert res[0][1] != res[1][1] and res[0][2] != res[1][2]   # distinct prompts and noise per rank


def test_single_rank_is_identity():
    import torch
    assert bench.max_over_ranks([3.5, 1.25], torch.device("cpu"), 1) == [3.5, 1.25]


@pytest.mark.parametrize("n", [1, 2, 4, 8])
def test_whole_job_throughput_scales_with_ranks(n):
    # weak scaling: each rank generates `batch` clips per step; value counts all ranks
    per_rank = bench.clips_per_min(1, 10, 5.0)
    assert bench.clips_per_min(n, 10, 5.0) == pytest.approx(n * per_rank)
    assert bench.workload_config(n)["global_batch"] == n * bench.WORKLOAD["batch"]


def test_step_roofline_counts():
    """One prompt with CFG at 180 frames: 2 x 181 tokens per network forward."""
    r = bench.step_roofline(2, 181, 1.0)
    tokens = 2 * 181
    # projections: QKV 3, O 1, FFN 2 + 2 (x 1024^2 MACs) per token, 16 layers, 2 FLOP per MAC
    assert bench.PROJ_FLOP_PER_TOKEN == 16 * 2 * (3 + 1 + 2 + 2) * 1024 * 1024
    # attention per sequence and layer: QK^T and PV, 2 x 2 x S^2 x 1024 FLOP
    assert r["flop"] == 2 * (tokens * bench.PROJ_FLOP_PER_TOKEN + 16 * 2 * 4 * 181 * 181 * 1024)
    # bytes: bf16 layer weights of both networks, and the activation model's 18,432 bf16
    # values per token and layer, for both networks
    assert bench.ACT_BYTES_PER_TOKEN_LAYER == 2 * 18432
    assert r["bytes"] == 2 * 16 * (8 * 1024 * 1024) * 2 + 2 * 16 * 36864 * tokens
    peaks, _ = bench._measured_peaks()
    t_flop = r["flop"] / (float(peaks["bf16_tflops"]) * 1e12)
    t_byte = r["bytes"] / (float(peaks["hbm_gbs"]) * 1e9)
    assert r["floor_us"] == round(max(t_flop, t_byte) * 1e6, 2)
    assert r["bound"] == ("tensor" if t_flop >= t_byte else "hbm")
    assert r["frac"] == round(max(t_flop, t_byte) / 1e-3, 4)
    assert abs(bench.step_roofline(2, 181, 2.0)["frac"] - r["frac"] / 2) < 1e-4
