"""moe_permute_noalloc: the permutation with the library's own fixed scratch
array, for callers that cannot allocate device memory when they call into the
library (a memory plan fixed at start-up, or a context where cudaMalloc is
not allowed). It must give exactly what moe_permute gives with a workspace.

Kept in its own file, collected last, and independent of every other test:
it passes in a fresh process and after the rest of the suite."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import mixture_experts_layer_tcgen05_b200 as moe  # noqa: E402
import moe_inputs as mi  # noqa: E402


def _ids(T, E, k, seed):
    rng = np.random.default_rng(seed)
    return np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)


def _with_workspace(ids, d, x):
    T, H, _, E, k = d
    ws = torch.zeros(moe.moe_workspace_size(d), dtype=torch.uint8, device="cuda")
    off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    pt = torch.empty(T * k, dtype=torch.int32, device="cuda")
    ip = torch.empty(T * k, dtype=torch.int32, device="cuda")
    xp = torch.empty(T * k, H, dtype=torch.bfloat16, device="cuda")
    moe.moe_permute(ids, d, off, pt, ip, x, xp, ws)
    return off, pt, ip, xp


def _no_alloc(ids, d, x):
    T, H, _, E, k = d
    off = torch.full((E + 1,), -1, dtype=torch.int32, device="cuda")
    pt = torch.full((T * k,), -1, dtype=torch.int32, device="cuda")
    ip = torch.full((T * k,), -1, dtype=torch.int32, device="cuda")
    xp = torch.zeros(T * k, H, dtype=torch.bfloat16, device="cuda")
    moe.moe_permute_noalloc(ids, d, off, pt, ip, x, xp)
    return off, pt, ip, xp


def test_no_alloc_permute_matches_workspace_permute_twice():
    # two calls in a row with different shapes: the second must not see the
    # first one's leftovers in the shared scratch array
    for T, E, k, seed in [(8192, 256, 8, 1), (4096, 8, 2, 2)]:
        H = 128
        d = (T, H, 128, E, k)
        ids = torch.from_numpy(_ids(T, E, k, seed)).cuda()
        x = torch.from_numpy(mi.normal_bf16(0, 91, 1.0, 1, T, H).view(np.int16)).view(
            torch.bfloat16).cuda().reshape(T, H)
        ref = _with_workspace(ids, d, x)
        got = _no_alloc(ids, d, x)
        torch.cuda.synchronize()
        for a, b in zip(got, ref):
            assert torch.equal(a, b)


def test_no_alloc_permute_rejects_oversize():
    d = (16384, 128, 128, 256, 8)  # needs just over MOE_NOALLOC_SCRATCH_BYTES
    ids = torch.zeros(16384, 8, dtype=torch.int32, device="cuda")
    buf = torch.empty(16384 * 8 + 257, dtype=torch.int32, device="cuda")
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_permute_noalloc(ids, d, buf, buf, buf)
    assert ei.value.status == moe.MOE_ERR_INVALID_ARG and "scratch" in str(ei.value)
