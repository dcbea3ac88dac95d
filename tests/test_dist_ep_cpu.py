"""Expert-parallel dispatch / combine on CPU ranks (gloo, world sizes 2 and 3).

`ExpertParallelMoE` runs the exchanges and the regroup; its per-rank compute
steps come from an object. Here that object works on the CPU in fp64
(routing and permutation by the oracle, the local experts' gated MLP by
numpy), so the counts exchange, the row all-to-alls, the regroup plan and the
return path are checked end to end without a GPU: every token's output must
equal the single-process oracle layer. The CUDA steps are checked on a GPU by
tests/test_gpu_ep.py."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import moe_inputs as mi
import oracle
from mixture_experts_layer_tcgen05_b200.ep import ExpertParallelMoE, regroup_plan


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleExpertOps:
    """Per-rank steps on the CPU in fp64; rows travel as fp64 copies of bf16 values."""

    def __init__(self, wr, bias, w13_local, w2_local, E, k):
        self.wr, self.bias, self.E, self.k = wr, bias, E, k
        self.w13 = mi.bf16_to_f32(w13_local).astype(np.float64)
        self.w2 = mi.bf16_to_f32(w2_local).astype(np.float64)
        self.I = self.w13.shape[1] // 2

    def route(self, x):
        bits = mi.f32_to_bf16(x.numpy().astype(np.float32))  # exact: x holds bf16 values
        ids, w = oracle.topk(oracle.router_logits(bits, self.wr, self.bias), self.k)
        return torch.from_numpy(ids), torch.from_numpy(w)

    def permute(self, ids, x):
        offsets, perm_token, _, inv_perm = oracle.permute(ids.numpy(), self.E)
        return (torch.from_numpy(offsets), torch.from_numpy(inv_perm),
                x[torch.from_numpy(perm_token).long()])

    def gather(self, src, idx):
        return src[torch.from_numpy(np.asarray(idx, dtype=np.int64))]

    def experts(self, x_loc, offsets):
        X = x_loc.numpy()
        y = np.zeros((X.shape[0], self.w2.shape[1]))
        for j in range(len(offsets) - 1):
            lo, hi = offsets[j], offsets[j + 1]
            g = X[lo:hi] @ self.w13[j, :self.I].T
            u = X[lo:hi] @ self.w13[j, self.I:].T
            y[lo:hi] = (g / (1 + np.exp(-g)) * u) @ self.w2[j].T
        return torch.from_numpy(y)

    def combine(self, y_perm, w, inv_perm):
        Y, W, P = y_perm.numpy(), w.numpy().astype(np.float64), inv_perm.numpy()
        out = np.zeros((W.shape[0], Y.shape[1]))
        for j in range(W.shape[1]):
            out += W[:, j:j + 1] * Y[P[:, j]]
        return torch.from_numpy(out)


def _layer(E, bias=None):
    cfg = mi.CONFIGS["tiny"].with_(T=96, H=128, I=256, E=E, k=2, bias="normal")
    L = mi.make_layer(cfg)
    if bias is not None:
        L["bias"] = np.asarray(bias, dtype=np.float32)
    return cfg, L


def _worker(rank, world, port, E, splits, bias, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cfg, L = _layer(E, bias)
        El = E // world
        lo = sum(splits[:rank])
        x = torch.from_numpy(mi.bf16_to_f32(L["x"][lo:lo + splits[rank]]).astype(np.float64))
        ops = OracleExpertOps(L["wr"], L["bias"], L["w13"][rank * El:(rank + 1) * El],
                              L["w2"][rank * El:(rank + 1) * El], E, cfg.k)
        layer = ExpertParallelMoE(ops, E)
        out[rank] = layer.forward(x).numpy()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,E,splits,bias", [
    (2, 8, [40, 56], None),
    (3, 6, [30, 1, 65], None),
    # experts 0-2 never chosen: rank 0 receives no rows and still takes every collective step
    (2, 6, [50, 46], [-40.0, -40.0, -40.0, 0.0, 0.0, 0.0]),
])
def test_expert_parallel_equals_single_process_layer(world, E, splits, bias):
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, E, splits, bias, out), nprocs=world, join=True,
                       start_method="spawn")
    cfg, L = _layer(E, bias)
    ref = oracle.moe_forward(L["x"], L["wr"], L["bias"], L["w13"], L["w2"], k=cfg.k)["out"]
    got = np.concatenate([out[r] for r in range(world)])
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-6 * np.abs(ref).max())


def test_regroup_plan_is_expert_major_then_source():
    # 2 sources x 3 local experts; received order: source 0 (e0: 2, e1: 0, e2: 1), source 1 (1, 2, 0)
    src_idx, off = regroup_plan([[2, 0, 1], [1, 2, 0]])
    # received rows: s0e0 = 0,1; s0e2 = 2; s1e0 = 3; s1e1 = 4,5
    assert src_idx.tolist() == [0, 1, 3, 4, 5, 2]
    assert off.tolist() == [0, 3, 5, 6]
    src_idx, off = regroup_plan(np.zeros((3, 2), dtype=np.int64))
    assert len(src_idx) == 0 and off.tolist() == [0, 0, 0]


def test_regroup_plan_properties_on_random_count_tables():
    """For any table of received row counts: the plan is a permutation of the
    received rows, each local expert's rows are one contiguous block in
    source order (sources ascending, each source's own order kept), and
    inverse_permutation undoes it."""
    from mixture_experts_layer_tcgen05_b200.ep import inverse_permutation
    rng = np.random.default_rng(17)
    for _ in range(200):
        G, El = int(rng.integers(1, 6)), int(rng.integers(1, 7))
        rc = rng.integers(0, 5, size=(G, El)) * (rng.random((G, El)) < 0.7)
        src_idx, off = regroup_plan(rc)
        n = int(rc.sum())
        assert sorted(src_idx.tolist()) == list(range(n))
        assert off[0] == 0 and off[-1] == n and np.all(np.diff(off) == rc.sum(0))
        # label each received row with (source, expert, position within that block)
        labels = [(s, j, i) for s in range(G) for j in range(El) for i in range(rc[s, j])]
        got = [labels[r] for r in src_idx]
        for j in range(El):
            block = got[off[j]:off[j + 1]]
            assert all(lab[1] == j for lab in block)
            assert block == sorted(block)  # sources ascending, then the source's own order
        inv = inverse_permutation(src_idx.astype(np.int64))
        assert np.array_equal(src_idx[inv], np.arange(n)) if n else len(inv) == 0
