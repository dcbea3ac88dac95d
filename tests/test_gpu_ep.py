"""Expert parallelism on a B200 with its CUDA steps: one NCCL rank (the only
GPU a run gets here), so the exchanges are identities and every other step is
the library's kernels, against the oracle; plus the row gather that does the
regroup, on the layouts a multi-rank regroup produces. The multi-rank
exchange logic is covered on CPU ranks by tests/test_dist_ep_cpu.py."""
import socket

import numpy as np
import pytest

import moe_inputs as mi
import oracle
from helpers import BF16_TOL, check_close, dev, dev_bf16, host_bf16

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import torch.distributed as dist  # noqa: E402

import mixture_experts_layer_tcgen05_b200 as moe  # noqa: E402
from mixture_experts_layer_tcgen05_b200.ep import (CudaExpertOps, ExpertParallelMoE,  # noqa: E402
                                                   inverse_permutation, regroup_plan)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("row_bytes", [8192, 4100, 4])
def test_gather_rows_bit_exact_and_bad_index(row_bytes):
    rng = np.random.default_rng(row_bytes)
    src = rng.integers(0, 256, (300, row_bytes), dtype=np.uint8)
    idx = rng.integers(0, 300, 517).astype(np.int32)
    s, d = dev(src), torch.empty(517, row_bytes, dtype=torch.uint8, device="cuda")
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    moe.moe_gather_rows(s, 300, dev(idx), 517, row_bytes, d, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == 0
    np.testing.assert_array_equal(d.cpu().numpy(), src[idx])
    idx[5] = 300  # out of range: skipped and recorded
    d.zero_()
    moe.moe_gather_rows(s, 300, dev(idx), 517, row_bytes, d, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == (moe.MOE_ERR_INVALID_ARG << 8) | 6
    assert not d[5].any()


def test_regroup_round_trip_on_device():
    """The regroup and its inverse as a 3-rank exchange would leave the rows."""
    recv = np.array([[3, 0, 5], [1, 7, 2], [0, 4, 4]])
    src_idx, off = regroup_plan(recv)
    R, H = int(recv.sum()), 256
    x = mi.normal_bf16(0, 31, 1.0, 1, R, H).reshape(R, H)
    ops = CudaExpertOps(dev_bf16(np.zeros((H, 6), np.uint16)), None,
                        dev_bf16(np.zeros((3, 256, H), np.uint16)),
                        dev_bf16(np.zeros((3, H, 128), np.uint16)), 6, 2)
    loc = ops.gather(dev_bf16(x), src_idx)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host_bf16(loc), x[src_idx])
    back = ops.gather(loc, inverse_permutation(src_idx))
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host_bf16(back), x)
    assert off.tolist() == [0, 4, 15, 26]


@pytest.mark.parametrize("kw", [dict(T=200, E=8, k=2), dict(T=48, E=6, k=3, H=256, I=384)])
def test_expert_parallel_single_rank_matches_oracle(kw):
    cfg = mi.CONFIGS["tiny"].with_(bias="normal", **kw)
    L = mi.make_layer(cfg)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                            world_size=1)
    try:
        ops = CudaExpertOps(dev_bf16(L["wr"]), dev(L["bias"]), dev_bf16(L["w13"]),
                            dev_bf16(L["w2"]), cfg.E, cfg.k)
        out = ExpertParallelMoE(ops, cfg.E).forward(dev_bf16(L["x"]))
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    ref = oracle.moe_forward(L["x"], L["wr"], L["bias"], L["w13"], L["w2"], k=cfg.k)["out"]
    check_close(mi.bf16_to_f32(host_bf16(out)), ref, BF16_TOL)
