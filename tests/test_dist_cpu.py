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


def _cfg(**kw):
    return mi.CONFIGS["tiny"].with_(**kw)


def test_rooflines_layer_time_and_fractions():
    peaks = {"bf16_tflops": 1000.0, "bf16_tflops_sustained": 800.0, "hbm_gbs": 5000.0}
    # T*k*H*I chosen so 6*T*k*H*I = 2e12 FLOP; one expert of 4 touched with rows
    cfg = _cfg(T=1000, k=1, H=1000, I=1000 * 1000 // 3, E=4)
    off = np.array([0, 1000, 1000, 1000, 1000], dtype=np.int32)
    flops = 6.0 * cfg.T * cfg.k * cfg.H * cfg.I
    stage = np.array([0.0, 0.0, 2.0, 1.0, 0.0])
    roof, lay, wbytes = bench.rooflines(cfg, off, 4.0, stage, 200.0, peaks, "measured")
    assert wbytes == 3 * cfg.H * cfg.I * 2 and lay["touched_experts"] == 1
    # a region under a second is compared with the burst peak
    assert roof["peak"] == 1000.0 and "burst" in roof["peak_source"]
    assert abs(roof["achieved"] - 4.0 * cfg.T * cfg.H * cfg.I / 2e-3 / 1e12) < 1e-9
    assert abs(roof["frac_of_sustained"] - roof["achieved"] / 800.0) < 1e-12
    assert lay["bound"] == "tensor"
    assert abs(lay["roofline_ms"] - flops / 1e15 * 1e3) < 1e-9
    assert abs(lay["roofline_frac"] - lay["roofline_ms"] / 4.0) < 1e-12
    # a long region takes the sustained peak
    roof2, lay2, _ = bench.rooflines(cfg, off, 4.0, stage, 5000.0, peaks, "measured")
    assert roof2["peak"] == 800.0 and "sustained" in roof2["peak_source"]
    # FP8 doubles the tensor roof
    r8, l8, _ = bench.rooflines(cfg.with_(fp8=True), off, 4.0, stage, 200.0, peaks, "measured",
                                e4m3_tflops=1800.0)
    assert r8["peak"] == 2000.0 and abs(r8["frac_of_cublas_e4m3"] - r8["achieved"] / 1800) < 1e-12


def test_rooflines_decode_is_hbm_bound():
    peaks = {"bf16_tflops": 1000.0, "hbm_gbs": 5000.0}
    cfg = _cfg(T=16, k=2, H=4096, I=14336, E=8)
    off = np.array([0, 4, 8, 12, 16, 20, 24, 28, 32], dtype=np.int32)
    stage = np.array([0.0, 0.0, 0.2, 0.1, 0.0])
    roof, lay, wbytes = bench.rooflines(cfg, off, 0.5, stage, 10.0, peaks, "fallback")
    g1 = 8 * 2 * cfg.H * cfg.I * 2.0
    assert roof["bound"] == "hbm" and abs(roof["achieved"] - g1 / 0.2e-3 / 1e9) < 1e-6
    assert lay["bound"] == "hbm"


def test_cpu_model_is_read_from_the_host():
    m = bench.cpu_model()
    assert m is None or (isinstance(m, str) and m and "\n" not in m)
