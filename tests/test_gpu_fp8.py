"""Fine-grained FP8 path on a B200 through the C ABI, against the CPU oracle.

Quantisation is integer/byte work decided in fp32 on both sides, so codes and
scales must match bit for bit. The FP8 layer is compared with the oracle run
on the dequantised values within the FP8 tolerance (6e-2 max, 2e-2 mean)."""
import numpy as np
import pytest

import moe_inputs as mi
import oracle
from helpers import FP8_TOL, check_close, dev, dev_bf16, dev_u8, host_bf16, layer_host

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import mixture_experts_layer_tcgen05_b200 as moe  # noqa: E402


def _dec_table():
    return np.array([oracle.e4m3_decode(q) for q in range(256)])


@pytest.mark.parametrize("ue8m0", [False, True])
@pytest.mark.parametrize("rows,cols", [(1, 128), (37, 512), (300, 7168)])
def test_act_quant_bit_exact(rows, cols, ue8m0):
    x = mi.normal_bf16(0, 61, 1.0, 1, rows, cols).reshape(rows, cols)
    x[0, :128] = 0  # an all-zero group
    q = torch.empty(rows, cols, dtype=torch.uint8, device="cuda")
    s = torch.empty(rows, cols // 128, dtype=torch.float32, device="cuda")
    moe.moe_quantize_act_fp8_fmt(dev_bf16(x), rows, cols, q, s,
                                 moe.MOE_SCALE_UE8M0 if ue8m0 else moe.MOE_SCALE_F32)
    torch.cuda.synchronize()
    rq, rs = oracle.quant_act_fp8(x, ue8m0=ue8m0)
    np.testing.assert_array_equal(q.cpu().numpy(), rq)
    np.testing.assert_array_equal(s.cpu().numpy().view(np.uint32), rs.view(np.uint32))


@pytest.mark.parametrize("ue8m0", [False, True])
@pytest.mark.parametrize("nb,rows,cols", [(1, 128, 128), (3, 256, 384), (2, 512, 1024)])
def test_weight_quant_bit_exact(nb, rows, cols, ue8m0):
    w = mi.normal_bf16(0, 62, 0.02, nb, rows, cols).reshape(nb, rows, cols)
    w[0, :128, :128] = 0
    q = torch.empty(nb, rows, cols, dtype=torch.uint8, device="cuda")
    s = torch.empty(nb, rows // 128, cols // 128, dtype=torch.float32, device="cuda")
    moe.moe_quantize_weight_fp8_fmt(dev_bf16(w), nb, rows, cols, q, s,
                                    moe.MOE_SCALE_UE8M0 if ue8m0 else moe.MOE_SCALE_F32)
    torch.cuda.synchronize()
    rq, rs = oracle.quant_weight_fp8(w, ue8m0=ue8m0)
    np.testing.assert_array_equal(q.cpu().numpy(), rq)
    np.testing.assert_array_equal(s.cpu().numpy().view(np.uint32), rs.view(np.uint32))


def _fp8_problem(counts, NB, K, tag):
    E = len(counts)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    M = int(offsets[-1])
    A = mi.normal_bf16(0, tag, 1.0, 1, M, K).reshape(M, K)
    B = mi.normal_bf16(0, tag + 1, 0.05, E, NB, K).reshape(E, NB, K)
    aq, as_ = oracle.quant_act_fp8(A)
    bq, bs = oracle.quant_weight_fp8(B)
    return E, offsets, M, aq, as_, bq, bs


FP8_GEMM_CASES = [([0, 1, 130, 300], 256, 384), ([128, 0, 5], 512, 256), ([700], 256, 1024)]


@pytest.mark.parametrize("counts,N,K", FP8_GEMM_CASES)
def test_fp8_grouped_gemm_swiglu_quantised_out(counts, N, K):
    E, offsets, M, aq, as_, bq, bs = _fp8_problem(counts, 2 * N, K, 71)
    C = torch.empty(M, N, dtype=torch.uint8, device="cuda")
    cs = torch.empty(M, N // 128, dtype=torch.float32, device="cuda")
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    moe.moe_grouped_gemm(dev_u8(aq), dev_u8(bq), dev(offsets), M, E, N, K, moe.MOE_DTYPE_FP8_E4M3,
                         moe.MOE_EPILOGUE_SWIGLU, C, dev(as_), dev(bs), cs, ws=ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == 0
    dec = _dec_table()
    A = dec[aq] * np.repeat(as_, 128, 1)
    Bd = dec[bq] * np.repeat(np.repeat(bs, 128, 1), 128, 2)
    got = dec[C.cpu().numpy()] * np.repeat(cs.cpu().numpy(), 128, 1)
    for e in range(E):
        lo, hi = offsets[e], offsets[e + 1]
        if hi == lo:
            continue
        g = A[lo:hi] @ Bd[e, :N].T
        u = A[lo:hi] @ Bd[e, N:].T
        h = (g / (1 + np.exp(-g)) * u).astype(np.float32)
        # the oracle's own re-quantisation of h (per row, 128-group)
        hq, hs = _quant_f32(h)
        ref = dec[hq] * np.repeat(hs, 128, 1)
        check_close(got[lo:hi], ref, FP8_TOL, f"expert {e}")
        # codes agree except at rounding boundaries
        assert np.mean(C.cpu().numpy()[lo:hi] != hq) < 0.02


def _quant_f32(h):
    """Per row, per 128 group of fp32 values: s = amax/448, q = e4m3(h/s) (torch's RNE cast)."""
    rows, cols = h.shape
    g = h.reshape(rows, cols // 128, 128)
    amax = np.abs(g).max(2)
    s = np.where(amax > 0, amax.astype(np.float32) / np.float32(448), np.float32(1)).astype(np.float32)
    q = torch.from_numpy((g / s[:, :, None]).astype(np.float32).reshape(rows, cols)).to(
        torch.float8_e4m3fn).view(torch.uint8).numpy()
    return q, s


# The plain GEMM stores 32-row groups of its output tile as whole boxes when all
# 32 rows belong to the expert and row by row otherwise: experts ending exactly
# on a 32-row group next to other experts' rows, groups of 1 and 31 rows, a
# tile whose last groups hold no rows of its expert.
@pytest.mark.parametrize("counts,N,K", [([0, 1, 130, 300], 256, 384), ([256, 7], 512, 256),
                                        ([32, 33, 95, 64, 1, 31, 160], 256, 256)])
def test_fp8_grouped_gemm_plain(counts, N, K):
    E, offsets, M, aq, as_, bq, bs = _fp8_problem(counts, N, K, 81)
    C = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    moe.moe_grouped_gemm(dev_u8(aq), dev_u8(bq), dev(offsets), M, E, N, K, moe.MOE_DTYPE_FP8_E4M3,
                         moe.MOE_EPILOGUE_NONE, C, dev(as_), dev(bs), None, ws=ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == 0
    dec = _dec_table()
    A = dec[aq] * np.repeat(as_, 128, 1)
    Bd = dec[bq] * np.repeat(np.repeat(bs, 128, 1), 128, 2)
    got = mi.bf16_to_f32(host_bf16(C))
    for e in range(E):
        lo, hi = offsets[e], offsets[e + 1]
        if hi > lo:
            # exact products of dequantised values; only fp32 accumulation and bf16 output differ
            check_close(got[lo:hi], A[lo:hi] @ Bd[e].T, (2e-2, 5e-3), f"expert {e}")


def run_fp8_forward(cfg, L):
    d = (cfg.T, cfg.H, cfg.I, cfg.E, cfg.k)
    w13 = dev_bf16(L["w13"])
    w2 = dev_bf16(L["w2"])
    w13q = torch.empty(cfg.E, 2 * cfg.I, cfg.H, dtype=torch.uint8, device="cuda")
    w13s = torch.empty(cfg.E, 2 * cfg.I // 128, cfg.H // 128, dtype=torch.float32, device="cuda")
    w2q = torch.empty(cfg.E, cfg.H, cfg.I, dtype=torch.uint8, device="cuda")
    w2s = torch.empty(cfg.E, cfg.H // 128, cfg.I // 128, dtype=torch.float32, device="cuda")
    moe.moe_quantize_weight_fp8(w13, cfg.E, 2 * cfg.I, cfg.H, w13q, w13s)
    moe.moe_quantize_weight_fp8(w2, cfg.E, cfg.H, cfg.I, w2q, w2s)
    del w13, w2
    ws = torch.zeros(moe.moe_workspace_size(d, moe.MOE_DTYPE_FP8_E4M3), dtype=torch.uint8, device="cuda")
    out = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device="cuda")
    moe.moe_forward_fp8(dev_bf16(L["x"]), dev_bf16(L["wr"]), dev(L["bias"]), w13q, w13s, w2q, w2s, d,
                        out, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == 0
    lay = moe.moe_workspace_layout(d, moe.MOE_DTYPE_FP8_E4M3)
    ids = ws[lay.topk_ids:lay.topk_ids + 4 * cfg.T * cfg.k].cpu().numpy().view(np.int32)
    return mi.bf16_to_f32(host_bf16(out)), ids.reshape(cfg.T, cfg.k)


def check_fp8_layer(cfg, L):
    got, ids = run_fp8_forward(cfg, L)
    toks = mi.token_subset(cfg)
    w13q, w13s = oracle.quant_weight_fp8(L["w13"])
    w2q, w2s = oracle.quant_weight_fp8(L["w2"])
    ref = oracle.moe_forward(L["x"], L["wr"], L["bias"], k=cfg.k, tokens=toks,
                             fp8=(w13q, w13s, w2q, w2s))
    np.testing.assert_array_equal(ids[toks], ref["ids"])
    return check_close(got[toks], ref["out"], FP8_TOL, cfg.name)


@pytest.mark.parametrize("kw", [dict(T=200, H=512, I=256, E=16, k=4, subset=0),
                                # T*k > 1024: permuted first, each token quantised into its k rows
                                dict(T=300, H=512, I=256, E=16, k=4, subset=0),
                                dict(T=33, H=256, I=384, E=8, k=2, subset=0),
                                dict(T=16, H=1024, I=2048, E=8, k=2, bias="zero", subset=0)])
def test_fp8_layer_small(kw):
    cfg = mi.CONFIGS["fine_grained_fp8"].with_(**kw)
    check_fp8_layer(cfg, mi.make_layer(cfg))


@pytest.mark.slow
def test_fp8_decode_full_size_all_tokens():
    cfg, L = layer_host("mixtral_decode_fp8")
    check_fp8_layer(cfg, L)


@pytest.mark.slow
def test_fp8_layer_full_size_sampled():
    cfg, L = layer_host("fine_grained_fp8")
    check_fp8_layer(cfg, L)


def test_fp8_grouped_gemm_row_gather():
    """FP8 GEMM-1 fetching its routed rows (and their activation scales) by index."""
    counts, N, K, Tsrc = [0, 3, 200, 129], 256, 384, 61
    E = len(counts)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    M = int(offsets[-1])
    X = mi.normal_bf16(0, 75, 1.0, 1, Tsrc, K).reshape(Tsrc, K)
    xq, xs = oracle.quant_act_fp8(X)
    rows = np.random.default_rng(3).integers(0, Tsrc, size=M).astype(np.int32)
    B = mi.normal_bf16(0, 76, 0.05, E, 2 * N, K).reshape(E, 2 * N, K)
    bq, bs = oracle.quant_weight_fp8(B)
    C = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    moe.moe_grouped_gemm(dev_u8(xq), dev_u8(bq), dev(offsets), M, E, N, K, moe.MOE_DTYPE_FP8_E4M3,
                         moe.MOE_EPILOGUE_SWIGLU, C, dev(xs), dev(bs), None, ws=ws,
                         a_rows=dev(rows), a_src_rows=Tsrc)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == 0
    dec = _dec_table()
    A = (dec[xq] * np.repeat(xs, 128, 1))[rows]
    Bd = dec[bq] * np.repeat(np.repeat(bs, 128, 1), 128, 2)
    got = mi.bf16_to_f32(host_bf16(C))
    for e in range(E):
        lo, hi = offsets[e], offsets[e + 1]
        if hi > lo:
            g = A[lo:hi] @ Bd[e, :N].T
            u = A[lo:hi] @ Bd[e, N:].T
            check_close(got[lo:hi], g / (1 + np.exp(-g)) * u, (2e-2, 5e-3), f"expert {e}")


@pytest.mark.parametrize("ue8m0", [False, True])
@pytest.mark.parametrize("H", [512, 768])  # 4 scale groups a row, and 6 (not 16-byte scale rows)
def test_fp8_forward_scattered_codes_bit_exact(H, ue8m0):
    """With more than 1024 routed rows the FP8 forwards quantise each token once and write its
    codes and scales to the token's k permuted rows; every permuted row must hold exactly the
    oracle's quantisation of its token (codes and scales byte for byte)."""
    cfg = mi.CONFIGS["tiny"].with_(T=300, H=H, I=256, E=16, k=4, bias="normal")
    L = mi.make_layer(cfg)
    T, E, k = cfg.T, cfg.E, cfg.k
    R = T * k
    d = (T, H, cfg.I, E, k)
    fmt = moe.MOE_SCALE_UE8M0 if ue8m0 else moe.MOE_SCALE_F32
    w13q = torch.empty(E, 2 * cfg.I, H, dtype=torch.uint8, device="cuda")
    w13s = torch.empty(E, 2 * cfg.I // 128, H // 128, dtype=torch.float32, device="cuda")
    w2q = torch.empty(E, H, cfg.I, dtype=torch.uint8, device="cuda")
    w2s = torch.empty(E, H // 128, cfg.I // 128, dtype=torch.float32, device="cuda")
    moe.moe_quantize_weight_fp8_fmt(dev_bf16(L["w13"]), E, 2 * cfg.I, H, w13q, w13s, fmt)
    moe.moe_quantize_weight_fp8_fmt(dev_bf16(L["w2"]), E, H, cfg.I, w2q, w2s, fmt)
    ws = torch.zeros(moe.moe_workspace_size(d, moe.MOE_DTYPE_FP8_E4M3), dtype=torch.uint8,
                     device="cuda")
    out = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
    args = (dev_bf16(L["x"]), dev_bf16(L["wr"]), dev(L["bias"]), w13q, w13s, w2q, w2s, d)
    if ue8m0:
        moe.moe_forward_fp8_ue8m0(*args, moe.MOE_EPILOGUE_SWIGLU, out, ws)
    else:
        moe.moe_forward_fp8(*args, out, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == 0
    lay = moe.moe_workspace_layout(d, moe.MOE_DTYPE_FP8_E4M3)
    wsh = ws.cpu().numpy()
    ids = wsh[lay.topk_ids:lay.topk_ids + 4 * R].view(np.int32).reshape(T, k)
    xq = wsh[lay.xq_perm:lay.xq_perm + R * H].reshape(R, H)
    xs = wsh[lay.xs_perm:lay.xs_perm + R * (H // 128) * 4].view(np.uint32).reshape(R, H // 128)
    _, perm_token, _, _ = oracle.permute(ids, E)
    rq, rs = oracle.quant_act_fp8(L["x"], ue8m0=ue8m0)
    np.testing.assert_array_equal(xq, rq[perm_token])
    np.testing.assert_array_equal(xs, rs.view(np.uint32)[perm_token])
