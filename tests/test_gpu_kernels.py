"""Per-kernel parity on a B200, through the C ABI, against the CPU oracle.

Integer work (ids, offsets, permutation) must be bit-exact; the logits too,
because the kernel accumulates in the same pinned fp32 order; routing weights
within 1e-6; GEMM outputs within the layer's bf16 tolerance."""
import numpy as np
import pytest

import moe_inputs as mi
import oracle
from helpers import BF16_TOL, check_close, dev, dev_bf16, host_bf16

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import mixture_experts_layer_tcgen05_b200 as moe  # noqa: E402


def _route(cfg, x, wr, b):
    T, E, k = cfg.T, cfg.E, cfg.k
    logits = torch.empty(T, E, dtype=torch.float32, device="cuda")
    ids = torch.empty(T, k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, k, dtype=torch.float32, device="cuda")
    moe.moe_route_topk(dev_bf16(x), dev_bf16(wr), None if b is None else dev(b), (T, cfg.H, 128, E, k),
                       logits, ids, w)
    torch.cuda.synchronize()
    return logits.cpu().numpy(), ids.cpu().numpy(), w.cpu().numpy()


ROUTER_CASES = [
    ("tiny", {}),
    ("tiny", dict(T=1)),
    ("tiny", dict(T=77, E=5, k=5, bias="normal")),
    ("tiny", dict(T=33, E=1, k=1)),
    ("tiny", dict(T=50, E=40, k=16, H=384)),
    ("tiny", dict(T=20, E=1024, k=8, H=256, bias="normal")),
    ("mixtral_decode", {}),
    ("mixtral_prefill", {}),
    ("fine_grained", dict(T=1024)),
    # many experts: odd expert counts (scalar Wr loads), several passes per block
    ("tiny", dict(T=333, E=300, k=8, H=128, bias="normal")),
    ("tiny", dict(T=8192, E=1024, k=4, H=128)),
    # few experts: one fused logits + top-k kernel, every block shape and pair count
    ("tiny", dict(T=37, E=2, k=2, bias="normal")),
    ("tiny", dict(T=300, E=3, k=2)),
    ("tiny", dict(T=129, E=7, k=3, bias="normal")),
    ("tiny", dict(T=250, E=16, k=4)),
    ("tiny", dict(T=70, E=32, k=16, bias="normal")),
    ("tiny", dict(T=10000, E=8, k=2, H=256)),
    ("tiny", dict(T=5000, E=24, k=6, H=128)),
    # many tokens, few experts: the tall kernel (whole Wr in shared memory), its largest table
    ("tiny", dict(T=1100, E=1, k=1, H=384)),
    ("tiny", dict(T=1500, E=32, k=8, H=1536, bias="normal")),
    ("tiny", dict(T=2222, E=13, k=5, H=640, bias="normal")),
    # Wr too large for shared memory: the narrow kernel at many tokens
    ("tiny", dict(T=1200, E=16, k=4, H=4096)),
]


@pytest.mark.parametrize("name,kw", ROUTER_CASES)
def test_router_bit_exact(name, kw):
    cfg = mi.CONFIGS[name].with_(**kw)
    x = mi.make_x(cfg)
    wr, b = mi.make_router(cfg)
    logits, ids, w = _route(cfg, x, wr, b)
    ref_l = oracle.router_logits(x, wr, b)
    np.testing.assert_array_equal(logits.view(np.uint32), ref_l.view(np.uint32))
    ref_ids, ref_w = oracle.topk(ref_l, cfg.k)
    np.testing.assert_array_equal(ids, ref_ids)
    np.testing.assert_allclose(w, ref_w, rtol=0, atol=1e-6)


@pytest.mark.parametrize("T", [90, 1200])
@pytest.mark.parametrize("E,k", [(8, 2), (5, 5), (32, 16), (2, 1)])
def test_router_exact_ties(E, k, T):
    """Equal logits from duplicated router columns and all-zero tokens: the
    lowest expert index wins every tie, in the fused small-E kernels too."""
    cfg = mi.CONFIGS["tiny"].with_(T=T, E=E, k=k)
    x = mi.make_x(cfg)
    x[::4] = 0  # every logit of these tokens is exactly zero
    wr, _ = mi.make_router(cfg)
    wr[:, E - 1] = wr[:, 0]
    if E > 3:
        wr[:, 2] = wr[:, 1]
    logits, ids, w = _route(cfg, x, wr, None)
    ref_l = oracle.router_logits(x, wr, None)
    np.testing.assert_array_equal(logits.view(np.uint32), ref_l.view(np.uint32))
    ref_ids, ref_w = oracle.topk(ref_l, k)
    np.testing.assert_array_equal(ids, ref_ids)
    np.testing.assert_allclose(w, ref_w, rtol=0, atol=1e-6)


def test_topk_from_logits_ties_and_extremes():
    rng = np.random.default_rng(7)
    T, E, k = 300, 64, 6
    logits = rng.standard_normal((T, E)).astype(np.float32)
    logits[::3, :20] = 0.5  # exact ties
    logits[1::5] = -3.0  # all equal rows
    ids = torch.empty(T, k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, k, dtype=torch.float32, device="cuda")
    moe.moe_topk_from_logits(dev(logits), (T, 128, 128, E, k), ids, w)
    ref_ids, ref_w = oracle.topk(logits, k)
    np.testing.assert_array_equal(ids.cpu().numpy(), ref_ids)
    np.testing.assert_allclose(w.cpu().numpy(), ref_w, rtol=0, atol=1e-6)


def _ids_cases():
    rng = np.random.default_rng(11)
    cases = []
    # R = T*k <= 1024 takes the one-launch small-batch permutation, larger R the
    # chunked one; (512, 8, 2) and (205, 64, 5) sit on either side of the switch
    for T, E, k, skew in [(64, 8, 2, None), (1, 4, 4, None), (100, 1, 1, None), (1000, 256, 8, 1),
                          (4096, 8, 2, 3), (257, 16, 16, None), (8192, 256, 8, None),
                          (512, 8, 2, 5), (205, 64, 5, None), (64, 1024, 8, None)]:
        ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
        if skew is not None:  # one expert in every token (slot 0): one expert holds all T
            for t in range(T):
                row = list(ids[t])
                if skew in row:
                    i = row.index(skew)
                    row[0], row[i] = row[i], row[0]
                else:
                    row[0] = skew
                ids[t] = row
        cases.append((T, E, k, ids))
    return cases


@pytest.mark.parametrize("case,H", [(c, 128) for c in range(10)] +
                         # rows of several 4-vector steps per lane, the last one partial
                         [(3, 1152), (5, 7168), (6, 3200),
                          # rows above 16 KB: the vector-store scatter instead of bulk copies
                          (3, 8320)])
def test_permute_bit_exact(case, H):
    T, E, k, ids = _ids_cases()[case]
    d = (T, H, 128, E, k)
    ws = torch.zeros(moe.moe_workspace_size(d), dtype=torch.uint8, device="cuda")
    off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    pt = torch.empty(T * k, dtype=torch.int32, device="cuda")
    ip = torch.empty(T * k, dtype=torch.int32, device="cuda")
    x = mi.normal_bf16(0, 21, 1.0, 1, T, H).reshape(T, H)
    xp = torch.empty(T * k, H, dtype=torch.bfloat16, device="cuda")
    moe.moe_permute(dev(ids), d, off, pt, ip, dev_bf16(x), xp, ws)
    torch.cuda.synchronize()
    r_off, r_pt, _, r_ip = oracle.permute(ids, E)
    np.testing.assert_array_equal(off.cpu().numpy(), r_off)
    np.testing.assert_array_equal(pt.cpu().numpy(), r_pt)
    np.testing.assert_array_equal(ip.cpu().numpy().reshape(T, k), r_ip)
    np.testing.assert_array_equal(host_bf16(xp), x[r_pt])


def _grouped_problem(counts, N2, K, tag):
    E = len(counts)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    M = int(offsets[-1])
    A = mi.normal_bf16(0, tag, 1.0, 1, M, K).reshape(M, K)
    B = mi.normal_bf16(0, tag + 1, 0.05, E, N2, K).reshape(E, N2, K)
    return E, offsets, M, A, B


GEMM_CASES = [
    # counts, N (output cols), K, max_rows hint (0: rows kernel)
    ([0, 1, 130, 300], 256, 384, 0),
    ([128, 0, 0, 256, 5], 128, 256, 0),
    ([1000], 384, 128, 0),
    ([0, 1, 17, 64], 256, 256, 64),
    ([3, 0, 16], 128, 512, 16),
    ([31, 2, 32, 0, 9], 384, 256, 32),
    # large experts: many m-tiles per expert, banded raster
    ([1500, 0, 700], 256, 384, 0),
    # partial m-tiles of many sizes (1 row short of a 16-row step, on one, one past),
    # alone and after full tiles
    ([95, 96, 97, 15, 16, 17, 33, 112, 127, 128, 129, 224, 352], 256, 384, 0),
    # K >= 4096: the plain GEMM takes two-half (256-row) tiles as the gated one always
    # does; halves with no rows, a half with one row, several 256-row tiles
    ([0, 1, 130, 300, 513, 256], 256, 4096, 0),
    ([2048, 1, 255], 512, 256, 0),
]


@pytest.mark.parametrize("counts,N,K,hint", GEMM_CASES)
def test_grouped_gemm_swiglu(counts, N, K, hint):
    E, offsets, M, A, B = _grouped_problem(counts, 2 * N, K, 31)
    C = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    moe.moe_grouped_gemm(dev_bf16(A), dev_bf16(B), dev(offsets), M, E, N, K, moe.MOE_DTYPE_BF16,
                         moe.MOE_EPILOGUE_SWIGLU, C, max_rows_per_expert=hint, ws=ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == 0
    got = mi.bf16_to_f32(host_bf16(C))
    for e in range(E):
        lo, hi = offsets[e], offsets[e + 1]
        if hi > lo:
            ref = oracle.expert_swiglu_rows(A[lo:hi], B[e])
            check_close(got[lo:hi], ref, BF16_TOL, f"expert {e}")


@pytest.mark.parametrize("counts,N,K,hint", GEMM_CASES)
def test_grouped_gemm_plain(counts, N, K, hint):
    E, offsets, M, A, B = _grouped_problem(counts, N, K, 41)
    C = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    moe.moe_grouped_gemm(dev_bf16(A), dev_bf16(B), dev(offsets), M, E, N, K, moe.MOE_DTYPE_BF16,
                         moe.MOE_EPILOGUE_NONE, C, max_rows_per_expert=hint, ws=ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == 0
    got = mi.bf16_to_f32(host_bf16(C))
    for e in range(E):
        lo, hi = offsets[e], offsets[e + 1]
        if hi > lo:
            ref = oracle.expert_down_rows(A[lo:hi], B[e])
            check_close(got[lo:hi], ref, BF16_TOL, f"expert {e}")


@pytest.mark.parametrize("swiglu", [False, True])
@pytest.mark.parametrize("N,K", [(256, 128), (512, 384)])
def test_grouped_gemm_last_wave_split_over_k(N, K, swiglu):
    """Enough 128 x 256 tiles that the last wave of the 148-CTA grid is at most
    half full: for the plain GEMM those tiles run as two units over the halves
    of K, whose fp32 partials a second kernel adds -- given scratch for them;
    the gated GEMM keeps whole tiles with the same scratch."""
    counts = [20000, 300, 0, 180]
    E, offsets, M, A, B = _grouped_problem(counts, 2 * N if swiglu else N, K, 81)
    C = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(32 << 20, dtype=torch.uint8, device="cuda")
    ep = moe.MOE_EPILOGUE_SWIGLU if swiglu else moe.MOE_EPILOGUE_NONE
    moe.moe_grouped_gemm(dev_bf16(A), dev_bf16(B), dev(offsets), M, E, N, K, moe.MOE_DTYPE_BF16,
                         ep, C, ws=ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == 0
    got = mi.bf16_to_f32(host_bf16(C))
    for e in range(E):
        lo, hi = offsets[e], offsets[e + 1]
        if hi > lo:
            ref = (oracle.expert_swiglu_rows(A[lo:hi], B[e]) if swiglu
                   else oracle.expert_down_rows(A[lo:hi], B[e]))
            check_close(got[lo:hi], ref, BF16_TOL, f"expert {e}")


@pytest.mark.parametrize("k", [1, 3, 4, 6, 9, 16])  # routed rows are read four at a time
def test_combine_exact_given_y(k):
    rng = np.random.default_rng(5)
    T, H = 37, 256
    R = T * k
    y = mi.normal_bf16(0, 51, 1.0, 1, R, H).reshape(R, H)
    w = rng.random((T, k)).astype(np.float32)
    inv = rng.permutation(R).astype(np.int32).reshape(T, k)
    out = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
    moe.moe_combine(dev_bf16(y), dev(w), dev(inv), (T, H, 128, 16, k), out)
    torch.cuda.synchronize()
    yf = mi.bf16_to_f32(y)
    got = mi.bf16_to_f32(host_bf16(out))
    # against the definition in fp64: only the fp32 sum and one bf16 rounding differ
    exact = sum(w[:, j:j + 1].astype(np.float64) * yf[inv[:, j]] for j in range(k))
    check_close(got, exact, (2 ** -7, 2 ** -8), "combine")


@pytest.mark.parametrize("counts,N,K", [([0, 1, 130, 300], 256, 384), ([700, 5], 128, 256),
                                        ([129, 0, 257], 384, 128)])
def test_grouped_gemm_swiglu_row_gather(counts, N, K):
    """A's routed rows fetched by index from a source matrix inside the GEMM
    (the permutation's gather fused into the producer); rows of the tail past
    M_total and every other row must match the dense computation."""
    E = len(counts)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    M = int(offsets[-1])
    Tsrc = 97
    X = mi.normal_bf16(0, 33, 1.0, 1, Tsrc, K).reshape(Tsrc, K)
    rows = np.random.default_rng(9).integers(0, Tsrc, size=M).astype(np.int32)
    B = mi.normal_bf16(0, 34, 0.05, E, 2 * N, K).reshape(E, 2 * N, K)
    C = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    moe.moe_grouped_gemm(dev_bf16(X), dev_bf16(B), dev(offsets), M, E, N, K, moe.MOE_DTYPE_BF16,
                         moe.MOE_EPILOGUE_SWIGLU, C, ws=ws, a_rows=dev(rows), a_src_rows=Tsrc)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == 0
    got = mi.bf16_to_f32(host_bf16(C))
    for e in range(E):
        lo, hi = offsets[e], offsets[e + 1]
        if hi > lo:
            ref = oracle.expert_swiglu_rows(X[rows[lo:hi]], B[e])
            check_close(got[lo:hi], ref, BF16_TOL, f"expert {e}")


@pytest.mark.parametrize("swiglu", [True, False])
@pytest.mark.parametrize("counts,N,K,hint", [([3, 0, 16], 128, 4096, 16), ([31, 2, 32, 0, 9], 384, 2048, 32)])
def test_small_m_split_k(swiglu, counts, N, K, hint):
    """With workspace to spare, the small-M kernel splits K into ranges that
    fill whole waves; the fp32 partials are summed in a fixed order."""
    E, offsets, M, A, B = _grouped_problem(counts, (2 if swiglu else 1) * N, K, 51)
    C = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(64 << 20, dtype=torch.uint8, device="cuda")
    args = (dev_bf16(A), dev_bf16(B), dev(offsets), M, E, N, K, moe.MOE_DTYPE_BF16,
            moe.MOE_EPILOGUE_SWIGLU if swiglu else moe.MOE_EPILOGUE_NONE, C)
    moe.moe_grouped_gemm(*args, max_rows_per_expert=hint, ws=ws)
    torch.cuda.synchronize()
    first = C.clone()
    moe.moe_grouped_gemm(*args, max_rows_per_expert=hint, ws=ws)
    torch.cuda.synchronize()
    assert torch.equal(first, C)  # deterministic
    assert moe.moe_get_device_status(ws) == 0
    got = mi.bf16_to_f32(host_bf16(C))
    for e in range(E):
        lo, hi = offsets[e], offsets[e + 1]
        if hi > lo:
            ref = (oracle.expert_swiglu_rows(A[lo:hi], B[e]) if swiglu
                   else oracle.expert_down_rows(A[lo:hi], B[e]))
            check_close(got[lo:hi], ref, BF16_TOL, f"expert {e}")
