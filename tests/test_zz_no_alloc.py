"""moe_permute_noalloc: the permutation with the library's own fixed scratch
array, for callers that cannot allocate device memory when they call into the
library (a memory plan fixed at start-up, or a context where cudaMalloc is
not allowed). For valid ids it must give exactly what moe_permute gives with
a workspace, and what the CPU oracle's permutation gives.

Kept in its own file, collected last, and independent of every other test:
it passes in a fresh process and after the rest of the suite."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import mixture_experts_layer_tcgen05_b200 as moe  # noqa: E402
import moe_inputs as mi  # noqa: E402
import oracle  # noqa: E402

BAD_INDEX = (moe.MOE_ERR_INVALID_ARG << 8) | 6


def _ids(T, E, k, seed):
    rng = np.random.default_rng(seed)
    return np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)


def _x(T, H):
    return torch.from_numpy(mi.normal_bf16(0, 91, 1.0, 1, T, H).view(np.int16)).view(
        torch.bfloat16).cuda().reshape(T, H)


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


@pytest.mark.parametrize("shapes", [
    # two calls in a row with different shapes: the second must not see the first one's
    # leftovers in the shared array
    [(8192, 256, 8, 1), (4096, 8, 2, 2)],
    # decode-sized (moe_permute takes its one-launch kernel there), then T not a multiple of 32
    [(64, 256, 8, 3), (1000, 37, 3, 4)],
])
def test_no_alloc_permute_matches_workspace_permute_and_oracle(shapes):
    assert moe.moe_permute_noalloc_status(clear=True) in (0, BAD_INDEX)
    for T, E, k, seed in shapes:
        H = 128
        d = (T, H, 128, E, k)
        ids_h = _ids(T, E, k, seed)
        ids = torch.from_numpy(ids_h).cuda()
        x = _x(T, H)
        ref = _with_workspace(ids, d, x)
        got = _no_alloc(ids, d, x)
        torch.cuda.synchronize()
        for a, b in zip(got, ref):
            assert torch.equal(a, b)
        off, pt, _, ip = oracle.permute(ids_h, E)
        np.testing.assert_array_equal(got[0].cpu().numpy(), off)
        np.testing.assert_array_equal(got[1].cpu().numpy(), pt)
        np.testing.assert_array_equal(got[2].cpu().numpy(), ip.reshape(-1))
        xh = x.view(torch.int16).cpu().numpy()
        np.testing.assert_array_equal(got[3].view(torch.int16).cpu().numpy(), xh[pt])
    assert moe.moe_permute_noalloc_status() == 0


def test_no_alloc_permute_records_bad_ids_in_its_status_word():
    assert moe.moe_permute_noalloc_status(clear=True) in (0, BAD_INDEX)
    T, E, k, H = 300, 16, 2, 128
    d = (T, H, 128, E, k)
    ids_h = _ids(T, E, k, 5)
    ids_h[7, 1] = E  # out of range
    _no_alloc(torch.from_numpy(ids_h).cuda(), d, _x(T, H))
    assert moe.moe_permute_noalloc_status(clear=True) == BAD_INDEX
    assert moe.moe_permute_noalloc_status() == 0  # cleared
    ids_h = _ids(T, E, k, 6)
    ids_h[11, 1] = ids_h[11, 0]  # an expert repeated within a token
    _no_alloc(torch.from_numpy(ids_h).cuda(), d, _x(T, H))
    assert moe.moe_permute_noalloc_status(clear=True) == BAD_INDEX
    # valid ids afterwards: correct results, status stays clear
    ids_h = _ids(T, E, k, 7)
    got = _no_alloc(torch.from_numpy(ids_h).cuda(), d, _x(T, H))
    np.testing.assert_array_equal(got[1].cpu().numpy(), oracle.permute(ids_h, E)[1])
    assert moe.moe_permute_noalloc_status() == 0


def test_no_alloc_permute_rejects_oversize():
    d = (16384, 128, 128, 256, 8)  # needs just over the fixed array's scratch
    ids = torch.zeros(16384, 8, dtype=torch.int32, device="cuda")
    buf = torch.empty(16384 * 8 + 257, dtype=torch.int32, device="cuda")
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_permute_noalloc(ids, d, buf, buf, buf)
    assert ei.value.status == moe.MOE_ERR_INVALID_ARG and "scratch" in str(ei.value)
