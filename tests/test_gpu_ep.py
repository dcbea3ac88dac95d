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
from mixture_experts_layer_tcgen05_b200.ep import (CudaExpertOps,  # noqa: E402
                                                   DeviceExpertParallelMoE, ExpertParallelMoE,
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


def _route_permute(cfg, L, x):
    """This (virtual) rank's routing and permutation on the library's kernels."""
    T = x.shape[0]
    ops = CudaExpertOps(dev_bf16(L["wr"]), dev(L["bias"]), dev_bf16(L["w13"][:1]),
                        dev_bf16(L["w2"][:1]), cfg.E, cfg.k)
    ops.H, ops.I = cfg.H, cfg.I
    ids, w = ops.route(dev_bf16(x))
    offsets, inv_perm, x_perm = ops.permute(ids, dev_bf16(x))
    return ids, w, offsets, inv_perm, x_perm


@pytest.mark.parametrize("G,Ts", [(3, [70, 33, 100]), (2, [1, 257]), (4, [16, 16, 16, 16])])
def test_device_exchange_emulated_ranks(G, Ts):
    """The exchange's kernels for G ranks, emulated on one GPU: every virtual
    rank's plan, dispatch and return run one after another on one stream (no
    kernel waits for another), into G separate buffers that stand for the ranks'
    receive and y_perm buffers. The receive buffers must hold exactly the
    expert-major concatenation of the sources' rows (bit-exact), the plan's local
    offsets their boundaries, and each rank's combined output the oracle layer."""
    E, k = 4 * G, 3
    cfg = mi.CONFIGS["tiny"].with_(H=256, I=256, E=E, k=k, bias="normal")
    L = mi.make_layer(cfg)
    El, H = E // G, cfg.H
    xs = [mi.make_x(cfg.with_(T=T, seed=10 + r)) for r, T in enumerate(Ts)]
    rr = [_route_permute(cfg.with_(T=T), L, x) for T, x in zip(Ts, xs)]
    counts_all = torch.stack([(o[2][1:] - o[2][:-1]).to(torch.int32) for o in rr]).contiguous()
    cap = G * max(Ts) * min(k, El)
    recv = [torch.zeros(cap, H, dtype=torch.bfloat16, device="cuda") for _ in range(G)]
    yperm = [torch.zeros(T * k, H, dtype=torch.bfloat16, device="cuda") for T in Ts]
    recv_ptrs = torch.tensor([b.data_ptr() for b in recv], dtype=torch.int64, device="cuda")
    yperm_ptrs = torch.tensor([b.data_ptr() for b in yperm], dtype=torch.int64, device="cuda")
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    plans = [torch.full((moe.moe_ep_plan_bytes(E, G) // 4,), -7, dtype=torch.int32, device="cuda")
             for _ in range(G)]
    for r in range(G):
        moe.moe_ep_plan(counts_all, G, r, E, plans[r])
        moe.moe_ep_dispatch(rr[r][4], rr[r][2], plans[r], E, G, Ts[r] * k, H * 2, recv_ptrs, cap, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == 0
    cnt = counts_all.cpu().numpy()
    offs = [o[2].cpu().numpy() for o in rr]
    xperm = [host_bf16(o[4]) for o in rr]
    for g in range(G):
        exp_rows = [xperm[s][offs[s][e]:offs[s][e + 1]] for e in range(g * El, (g + 1) * El)
                    for s in range(G)]
        exp = np.concatenate(exp_rows)
        got = host_bf16(recv[g])
        np.testing.assert_array_equal(got[:len(exp)], exp)
        loc_off = plans[g][:El + 1].cpu().numpy()
        np.testing.assert_array_equal(
            loc_off, np.concatenate([[0], np.cumsum(cnt[:, g * El:(g + 1) * El].sum(0))]))
    # local experts on each rank's receive buffer, then the return path and the combine
    w13, w2 = dev_bf16(L["w13"]), dev_bf16(L["w2"])
    y_loc = [torch.zeros(cap, H, dtype=torch.bfloat16, device="cuda") for _ in range(G)]
    h = torch.empty(cap, cfg.I, dtype=torch.bfloat16, device="cuda")
    big = torch.zeros(64 << 20, dtype=torch.uint8, device="cuda")
    for g in range(G):
        loc_off = plans[g][:El + 1]
        moe.moe_grouped_gemm(recv[g], w13[g * El:(g + 1) * El], loc_off, cap, El, cfg.I, H,
                             moe.MOE_DTYPE_BF16, moe.MOE_EPILOGUE_SWIGLU, h, ws=big)
        moe.moe_grouped_gemm(h, w2[g * El:(g + 1) * El], loc_off, cap, El, H, cfg.I,
                             moe.MOE_DTYPE_BF16, moe.MOE_EPILOGUE_NONE, y_loc[g], ws=big)
        moe.moe_ep_return(y_loc[g], plans[g], E, G, cap, H * 2, yperm_ptrs, max(Ts) * k, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == 0 and moe.moe_get_device_status(big) == 0
    for r in range(G):
        out = torch.empty(Ts[r], H, dtype=torch.bfloat16, device="cuda")
        moe.moe_combine(yperm[r], rr[r][1], rr[r][3], (Ts[r], H, cfg.I, E, k), out)
        torch.cuda.synchronize()
        ref = oracle.moe_forward(xs[r], L["wr"], L["bias"], L["w13"], L["w2"], k=k)["out"]
        check_close(mi.bf16_to_f32(host_bf16(out)), ref, BF16_TOL, f"rank {r}")


def test_device_exchange_records_rows_past_the_buffer():
    """A destination buffer shorter than the plan needs: the rows that do not fit are
    skipped and recorded in the status word; nothing is written outside the buffer."""
    G, E, k, T, H = 2, 4, 2, 40, 128
    cnt = torch.tensor([[20, 20, 20, 20], [20, 20, 20, 20]], dtype=torch.int32, device="cuda")
    offsets = torch.tensor([0, 20, 40, 60, 80], dtype=torch.int32, device="cuda")
    plan = torch.zeros(moe.moe_ep_plan_bytes(E, G) // 4, dtype=torch.int32, device="cuda")
    moe.moe_ep_plan(cnt, G, 1, E, plan)
    x_perm = torch.ones(T * k, H, dtype=torch.bfloat16, device="cuda")
    buf = torch.zeros(2, 60 + 8, H, dtype=torch.bfloat16, device="cuda")  # 60 rows each + guard
    ptrs = torch.tensor([buf[0].data_ptr(), buf[1].data_ptr()], dtype=torch.int64, device="cuda")
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    moe.moe_ep_dispatch(x_perm, offsets, plan, E, G, T * k, H * 2, ptrs, 60, ws)
    torch.cuda.synchronize()
    # rank 1's rows for each destination start at row 20 (rank 0's 20 come first) and
    # run to 60 for the first expert ... the second expert's rows land at 60..80: past 60
    assert moe.moe_get_device_status(ws) == (moe.MOE_ERR_INVALID_ARG << 8) | 6
    assert not buf[:, 60:].float().any()


@pytest.mark.parametrize("kw", [dict(T=200, E=8, k=2), dict(T=48, E=6, k=3, H=256, I=384)])
def test_device_expert_parallel_single_rank_matches_oracle(kw):
    """The device-side layer on one NCCL rank (symmetric-memory buffers of one
    rank, the exchange's kernels and collectives all running), against the oracle."""
    cfg = mi.CONFIGS["tiny"].with_(bias="normal", **kw)
    L = mi.make_layer(cfg)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                            world_size=1, device_id=torch.device("cuda", 0))
    try:
        ops = CudaExpertOps(dev_bf16(L["wr"]), dev(L["bias"]), dev_bf16(L["w13"]),
                            dev_bf16(L["w2"]), cfg.E, cfg.k)
        layer = DeviceExpertParallelMoE(ops, cfg.E, T_max=cfg.T)
        outs = [layer.forward(dev_bf16(L["x"])) for _ in range(2)]  # twice: buffers are reused
        torch.cuda.synchronize()
        assert int(layer.status[0].item()) == 0
    finally:
        dist.destroy_process_group()
    ref = oracle.moe_forward(L["x"], L["wr"], L["bias"], L["w13"], L["w2"], k=cfg.k)["out"]
    for out in outs:
        check_close(mi.bf16_to_f32(host_bf16(out)), ref, BF16_TOL)
