"""Host-side logic of the multi-GPU bench on CPU ranks (gloo, world size 2):
token-parallel replicas share the weights, draw their own token batches, and
report the whole-job rate from the slowest rank's time."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import moe_inputs as mi


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cfg = mi.CONFIGS["tiny"]
        x = bench.rank_tokens(cfg, rank)
        wr, b = mi.make_router(cfg)
        # fake per-rank step times: rank 1 is slower
        ms = 10.0 + 5.0 * rank
        mx = bench.max_over_ranks(ms, dist)
        rate = bench.whole_job_tokens_per_s(cfg.T, world, mx)
        digest = torch.tensor([float(x.astype(np.float64).sum()), float(wr.astype(np.float64).sum())],
                              dtype=torch.float64)
        allx = [torch.zeros(2, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(allx, digest)
        out[rank] = (mx, rate, [t.tolist() for t in allx])
    finally:
        dist.destroy_process_group()


def test_token_parallel_replicas_gloo_world2():
    world = 2
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
    cfg = mi.CONFIGS["tiny"]
    for r in range(world):
        mx, rate, digests = out[r]
        assert mx == 15.0  # the slowest rank's time
        assert rate == pytest.approx(world * cfg.T / 0.015)
        assert digests[0][1] == digests[1][1]  # same router weights
        assert digests[0][0] != digests[1][0]  # different token batches


def test_layer_roofline_time_and_fractions():
    peaks = {"bf16_tflops_sustained": 1000.0, "hbm_gbs": 5000.0}
    # compute-bound: 2 TFLOP at 1000 TF/s = 2 ms; 1 GB at 5 TB/s = 0.2 ms
    r = bench.layer_roofline(2e12, 1e9, 4.0, peaks, 1.0, 8)
    assert r["bound"] == "tensor" and abs(r["roofline_ms"] - 2.0) < 1e-12
    assert abs(r["roofline_frac"] - 0.5) < 1e-12 and abs(r["tflops_frac"] - 0.5) < 1e-12
    assert abs(r["gbs"] - 250.0) < 1e-9 and r["touched_experts"] == 8
    # the FP8 / FP4 ratio doubles the tensor roof
    assert abs(bench.layer_roofline(2e12, 1e9, 4.0, peaks, 2.0, 8)["roofline_ms"] - 1.0) < 1e-12
    # memory-bound: 10 GB at 5 TB/s = 2 ms
    r = bench.layer_roofline(1e9, 1e10, 2.5, peaks, 1.0, 3)
    assert r["bound"] == "hbm" and abs(r["roofline_ms"] - 2.0) < 1e-12
    assert abs(r["roofline_frac"] - 0.8) < 1e-12 and abs(r["gbs_frac"] - 0.8) < 1e-12


def test_cpu_model_is_read_from_the_host():
    m = bench.cpu_model()
    assert m is None or (isinstance(m, str) and m and "\n" not in m)
