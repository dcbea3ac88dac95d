"""Expert parallelism across ranks (one process per GPU, torch.distributed).

"Experts backends" (HF Transformers docs), backend table, `deepgemm_megamoe`
row: expert-parallel dispatch, the gated expert MLP and the combine, with the
token exchange over NVLink. Each of G ranks owns E / G consecutive experts
(rank g: experts [g*E/G, (g+1)*E/G)) and routes its own tokens:

1. route and permute locally (rows ordered by global expert, so the rows
   for rank g are one contiguous block);
2. exchange the per-expert row counts (all-to-all of E/G counts per pair);
3. dispatch: all-to-all of the rows, block g to rank g; a rank receives its
   rows source-major, then by local expert;
4. regroup them expert-major (a row gather with a plan built on the host from
   the counts) and run the grouped GEMMs of the local experts;
5. undo the regroup, send every row back to its source (the reverse
   all-to-all) and combine there with the routing weights.

The per-rank compute steps are the library's CUDA kernels (`CudaExpertOps`);
the exchanges are NCCL all-to-alls through torch.distributed. The class takes
the compute steps as an object so that the exchange and regroup logic can be
exercised by processes without a GPU. Its split sizes come to the host once
per forward (NCCL's variable all-to-all takes them there).

`DeviceExpertParallelMoE` keeps the whole exchange on the device: the counts
are all-gathered into a device [G, E] matrix, `moe_ep_plan` turns it into
every row's destination, `moe_ep_dispatch` stores the rows straight into the
owners' receive buffers (expert-major there, so the grouped GEMMs run on them
with no regroup) and `moe_ep_return` stores the expert outputs back into the
sources' y_perm. The receive and y_perm buffers are symmetric memory (every
rank maps every other rank's), the only host work is launching, and two NCCL
all-reduces of one word order the stores before the reads.
"""
from __future__ import annotations

import numpy as np
import torch
import torch.distributed as dist

from . import (MOE_DTYPE_BF16, MOE_EPILOGUE_NONE, MOE_EPILOGUE_SWIGLU, moe_combine, moe_ep_dispatch,
               moe_ep_plan, moe_ep_plan_bytes, moe_ep_return, moe_gather_rows, moe_grouped_gemm,
               moe_permute, moe_route_topk, moe_workspace_size)


def regroup_plan(recv_counts) -> tuple[np.ndarray, np.ndarray]:
    """Rows arrive source-major, then by local expert: recv_counts[s, j] rows
    from source s for local expert j. Returns (src_idx, offsets): local row i
    of the expert-major order (expert j, then source s ascending, then the
    source's own order) is received row src_idx[i]; expert j owns local rows
    [offsets[j], offsets[j+1])."""
    rc = np.asarray(recv_counts, dtype=np.int64)
    G, El = rc.shape
    flat = rc.reshape(-1)
    starts = (np.cumsum(flat) - flat).reshape(G, El)  # first received row of block (s, j)
    parts = [np.arange(starts[s, j], starts[s, j] + rc[s, j], dtype=np.int64)
             for j in range(El) for s in range(G)]
    src_idx = np.concatenate(parts) if parts else np.zeros(0, dtype=np.int64)
    offsets = np.concatenate([[0], np.cumsum(rc.sum(0))]).astype(np.int64)
    return src_idx.astype(np.int32), offsets.astype(np.int32)


def inverse_permutation(p: np.ndarray) -> np.ndarray:
    inv = np.empty_like(p)
    inv[p] = np.arange(len(p), dtype=p.dtype)
    return inv


class CudaExpertOps:
    """The per-rank steps of an expert-parallel bf16 layer on the library's kernels.

    wr [H, E] bf16 and bias [E] fp32 (or None) cover all E experts; w13_local
    [E/G, 2I, H] and w2_local [E/G, H, I] (bf16, K-major as for moe_forward)
    are this rank's experts."""

    def __init__(self, wr, bias, w13_local, w2_local, E: int, k: int):
        self.wr, self.bias, self.w13, self.w2 = wr, bias, w13_local, w2_local
        self.E, self.k = E, k
        self.El, two_i, self.H = w13_local.shape
        self.I = two_i // 2
        self.device = wr.device
        self._ws = {}

    def _workspace(self, T: int):
        if T not in self._ws:
            n = moe_workspace_size((T, self.H, self.I, self.E, self.k), MOE_DTYPE_BF16)
            self._ws[T] = torch.zeros(max(n, 64 << 20), dtype=torch.uint8, device=self.device)
        return self._ws[T]

    def route(self, x):
        T = x.shape[0]
        d = (T, self.H, self.I, self.E, self.k)
        logits = torch.empty(T, self.E, dtype=torch.float32, device=self.device)
        ids = torch.empty(T, self.k, dtype=torch.int32, device=self.device)
        w = torch.empty(T, self.k, dtype=torch.float32, device=self.device)
        moe_route_topk(x, self.wr, self.bias, d, logits, ids, w)
        return ids, w

    def permute(self, ids, x):
        T = x.shape[0]
        d = (T, self.H, self.I, self.E, self.k)
        offsets = torch.empty(self.E + 1, dtype=torch.int32, device=self.device)
        perm_token = torch.empty(T * self.k, dtype=torch.int32, device=self.device)
        inv_perm = torch.empty(T, self.k, dtype=torch.int32, device=self.device)
        x_perm = torch.empty(T * self.k, self.H, dtype=x.dtype, device=self.device)
        moe_permute(ids, d, offsets, perm_token, inv_perm, x, x_perm, self._workspace(T))
        return offsets, inv_perm, x_perm

    def gather(self, src, idx: np.ndarray):
        out = torch.empty(len(idx), *src.shape[1:], dtype=src.dtype, device=self.device)
        if len(idx):
            rows = torch.from_numpy(np.ascontiguousarray(idx, dtype=np.int32)).to(self.device)
            moe_gather_rows(src, src.shape[0], rows, len(idx), src[0].numel() * src.element_size(),
                            out)
        return out

    def experts(self, x_loc, offsets: np.ndarray):
        R = x_loc.shape[0]
        y = torch.empty(R, self.H, dtype=x_loc.dtype, device=self.device)
        if R == 0:
            return y
        off = torch.from_numpy(np.ascontiguousarray(offsets, dtype=np.int32)).to(self.device)
        hint = int(np.diff(offsets).max())
        h = torch.empty(R, self.I, dtype=x_loc.dtype, device=self.device)
        ws = self._workspace(1)
        moe_grouped_gemm(x_loc, self.w13, off, R, self.El, self.I, self.H, MOE_DTYPE_BF16,
                         MOE_EPILOGUE_SWIGLU, h, max_rows_per_expert=hint, ws=ws)
        moe_grouped_gemm(h, self.w2, off, R, self.El, self.H, self.I, MOE_DTYPE_BF16,
                         MOE_EPILOGUE_NONE, y, max_rows_per_expert=hint, ws=ws)
        return y

    def combine(self, y_perm, w, inv_perm):
        T = w.shape[0]
        out = torch.empty(T, self.H, dtype=y_perm.dtype, device=self.device)
        moe_combine(y_perm, w, inv_perm, (T, self.H, self.I, self.E, self.k), out)
        return out


class ExpertParallelMoE:
    """The layer with its experts spread over the ranks of `group`."""

    def __init__(self, ops, E: int, group=None):
        self.ops, self.E, self.group = ops, E, group
        self.G = dist.get_world_size(group)
        if E % self.G:
            raise ValueError(f"E={E} does not split over {self.G} ranks")
        self.El = E // self.G

    def forward(self, x):
        """x [T, H] this rank's tokens (T >= 1); returns out [T, H]."""
        ops, G, El = self.ops, self.G, self.El
        ids, w = ops.route(x)
        offsets, inv_perm, x_perm = ops.permute(ids, x)
        counts = (offsets[1:] - offsets[:-1]).to(torch.int32).contiguous()
        # every rank learns how many rows each source sends for each of its experts
        recv_counts = torch.empty_like(counts)
        dist.all_to_all_single(recv_counts, counts, group=self.group)
        send = counts.cpu().numpy().reshape(G, El)
        recv = recv_counts.cpu().numpy().reshape(G, El)
        send_split = [int(v) for v in send.sum(1)]
        recv_split = [int(v) for v in recv.sum(1)]
        # dispatch
        x_recv = x_perm.new_empty(sum(recv_split), x_perm.shape[1])
        dist.all_to_all_single(x_recv, x_perm, recv_split, send_split, group=self.group)
        # local experts, expert-major
        src_idx, loc_off = regroup_plan(recv)
        y_loc = ops.experts(ops.gather(x_recv, src_idx), loc_off)
        y_recv = ops.gather(y_loc, inverse_permutation(src_idx))
        # combine: rows back to their sources, in the order they were sent
        y_perm = y_recv.new_empty(x_perm.shape[0], y_recv.shape[1])
        dist.all_to_all_single(y_perm, y_recv, send_split, recv_split, group=self.group)
        return ops.combine(y_perm, w, inv_perm)


class DeviceExpertParallelMoE:
    """The bf16 layer with its experts spread over the ranks of `group`, the
    exchange planned and moved on the device (no count reaches the host).

    ops: this rank's `CudaExpertOps`. T_max: the most tokens a rank passes to
    forward. Buffers are sized for the worst case: a rank receives at most
    G * T_max * min(k, E / G) rows (a token holds each expert once)."""

    def __init__(self, ops: CudaExpertOps, E: int, T_max: int, group=None):
        import torch.distributed._symmetric_memory as symm_mem

        self.ops, self.E, self.group = ops, E, group
        self.G = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        if E % self.G:
            raise ValueError(f"E={E} does not split over {self.G} ranks")
        self.El = E // self.G
        self.T_max = T_max
        k, H, dev = ops.k, ops.H, ops.device
        self.cap = self.G * T_max * min(k, self.El)   # receive rows, worst case
        self.R_max = T_max * k                         # a rank's own routed rows
        gname = group.group_name if group is not None else dist.group.WORLD.group_name
        self.x_recv = symm_mem.empty(self.cap, H, dtype=torch.bfloat16, device=dev)
        self.y_perm = symm_mem.empty(self.R_max, H, dtype=torch.bfloat16, device=dev)
        hx = symm_mem.rendezvous(self.x_recv, gname)
        hy = symm_mem.rendezvous(self.y_perm, gname)
        self.recv_ptrs = torch.tensor(list(hx.buffer_ptrs), dtype=torch.int64, device=dev)
        self.yperm_ptrs = torch.tensor(list(hy.buffer_ptrs), dtype=torch.int64, device=dev)
        self._handles = (hx, hy)
        self.counts_all = torch.zeros(self.G, E, dtype=torch.int32, device=dev)
        self.plan = torch.zeros(moe_ep_plan_bytes(E, self.G) // 4, dtype=torch.int32, device=dev)
        self.h = torch.empty(self.cap, ops.I, dtype=torch.bfloat16, device=dev)
        self.y_loc = torch.empty(self.cap, H, dtype=torch.bfloat16, device=dev)
        self.status = torch.zeros(64, dtype=torch.int32, device=dev)
        self._sync = torch.zeros(1, dtype=torch.int32, device=dev)

    def _order(self):
        """Every rank's stores so far are visible to every rank's later reads: an
        all-reduce of one word on the stream (the host does not wait)."""
        dist.all_reduce(self._sync, group=self.group)

    def forward(self, x):
        """x [T, H] bf16, this rank's tokens (1 <= T <= T_max); returns out [T, H]."""
        ops, G, E, El = self.ops, self.G, self.E, self.El
        T, H = x.shape
        if not 1 <= T <= self.T_max:
            raise ValueError(f"T={T} outside [1, {self.T_max}]")
        ids, w = ops.route(x)
        offsets, inv_perm, x_perm = ops.permute(ids, x)
        counts = (offsets[1:] - offsets[:-1]).to(torch.int32).contiguous()
        dist.all_gather_into_tensor(self.counts_all, counts, group=self.group)
        moe_ep_plan(self.counts_all, G, self.rank, E, self.plan)
        row_bytes = H * 2
        moe_ep_dispatch(x_perm, offsets, self.plan, E, G, T * ops.k, row_bytes, self.recv_ptrs,
                        self.cap, self.status)
        self._order()
        loc_off = self.plan[:El + 1]
        ws = ops._workspace(1)
        moe_grouped_gemm(self.x_recv, ops.w13, loc_off, self.cap, El, ops.I, H, MOE_DTYPE_BF16,
                         MOE_EPILOGUE_SWIGLU, self.h, ws=ws)
        moe_grouped_gemm(self.h, ops.w2, loc_off, self.cap, El, H, ops.I, MOE_DTYPE_BF16,
                         MOE_EPILOGUE_NONE, self.y_loc, ws=ws)
        moe_ep_return(self.y_loc, self.plan, E, G, self.cap, row_bytes, self.yperm_ptrs,
                      self.R_max, self.status)
        self._order()
        return ops.combine(self.y_perm[:T * ops.k], w, inv_perm)
