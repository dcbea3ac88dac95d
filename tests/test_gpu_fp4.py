"""FP4 (e2m1) expert weights with UE8M0 scales per (row, 32 K) on a B200,
through the C ABI, against the CPU oracle.

"Experts backends", "FP8 and FP4 quantized experts": FP4 expert weights packed
two per byte with UE8M0 weight scales, run on the block-scaled MMA with e4m3
activations. Weight quantisation is integer work (codes and scale bytes) and
must match the oracle bit for bit; the GEMMs are compared with the dense
product of the dequantised operands and the layers with the oracle run on the
same quantised weights, within the FP8 tolerance."""
import numpy as np
import pytest

import moe_inputs as mi
import oracle
from helpers import (FP8_TOL, check_close, dev, dev_bf16, dev_u8, host_bf16, layer_host,
                     quant_pow2_e4m3)

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import mixture_experts_layer_tcgen05_b200 as moe  # noqa: E402

_E2M1 = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6, -0.0, -0.5, -1, -1.5, -2, -3, -4, -6])


def _dequant_fp4(q, sc):
    codes = np.stack([q & 15, q >> 4], axis=-1).reshape(*q.shape[:-1], 2 * q.shape[-1])
    return _E2M1[codes] * np.repeat(2.0 ** (sc.astype(np.float64) - 127), 32, axis=-1)


def _chunks(sc):
    """e8m0 bytes [nb, rows, K/32] -> the chunk layout the GEMM reads: per 128
    rows and 128 K a 512-byte chunk, byte 16 r + 4 g + j = row 32 g + r, K step j."""
    nb, rows, kb32 = sc.shape
    return np.ascontiguousarray(
        sc.reshape(nb, rows // 128, 4, 32, kb32 // 4, 4).transpose(0, 1, 4, 3, 2, 5)).reshape(-1)


def _dequant_e4m3(q, s):
    dec = np.array([oracle.e4m3_decode(c) for c in range(256)])
    return dec[q] * np.repeat(s, 128, axis=-1)


def _quant_fp4_dev(w, nb, rows, cols):
    q = torch.empty(nb, rows, cols // 2, dtype=torch.uint8, device="cuda")
    sc = torch.empty(nb, rows, cols // 32, dtype=torch.uint8, device="cuda")
    moe.moe_quantize_weight_fp4(dev_bf16(w), nb, rows, cols, q, sc)
    return q, sc


@pytest.mark.parametrize("nb,rows,cols", [(1, 128, 128), (3, 128, 384), (2, 256, 1024)])
def test_quantize_weight_fp4_bit_exact(nb, rows, cols):
    rng = np.random.default_rng(rows * cols)
    w = (rng.standard_normal((nb, rows, cols)) * 0.02).astype(np.float32)
    w[0, 0, 32:64] = 0                                   # an all-zero block: scale 1
    w[0, 0, 64:96] *= 1e-3                               # tiny values, many rounding to -0 / +0
    w[-1, -1, -32:] = np.linspace(-6, 6, 32) * 2.0 ** -9  # every grid point and midpoints
    wb = mi.f32_to_bf16(w)
    q, sc = _quant_fp4_dev(wb, nb, rows, cols)
    torch.cuda.synchronize()
    rq, rs = oracle.quant_weight_fp4(wb)
    np.testing.assert_array_equal(sc.cpu().numpy().reshape(-1), _chunks(rs))
    np.testing.assert_array_equal(q.cpu().numpy(), rq)


def _problem(counts, NB, K, tag):
    E = len(counts)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    M = int(offsets[-1])
    A = mi.normal_bf16(0, tag, 1.0, 1, M, K).reshape(M, K)
    B = mi.normal_bf16(0, tag + 1, 0.05, E, NB, K).reshape(E, NB, K)
    aq, as_ = oracle.quant_act_fp8(A, ue8m0=True)
    bq, bs = oracle.quant_weight_fp4(B)
    return E, offsets, M, aq, as_, bq, bs


@pytest.mark.parametrize("counts,N,K,hint", [
    ([0, 1, 130, 300], 256, 384, 0), ([128, 0, 5], 512, 256, 0), ([700], 256, 1024, 0),
    ([3, 0, 16, 9], 256, 384, 16), ([1, 30, 2], 384, 256, 32), ([50, 64, 0, 33], 128, 512, 64)])
def test_fp4_grouped_gemm_plain(counts, N, K, hint):
    E, offsets, M, aq, as_, bq, bs = _problem(counts, N, K, 101)
    C = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    moe.moe_grouped_gemm_fp4(dev_u8(aq), dev(as_), dev_u8(bq), dev_u8(_chunks(bs)), dev(offsets), M,
                             E, N, K, moe.MOE_EPILOGUE_NONE, C, None, ws, max_rows_per_expert=hint)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == 0
    A, Bd = _dequant_e4m3(aq, as_), _dequant_fp4(bq, bs)
    got = mi.bf16_to_f32(host_bf16(C))
    for e in range(E):
        lo, hi = offsets[e], offsets[e + 1]
        if hi > lo:
            check_close(got[lo:hi], A[lo:hi] @ Bd[e].T, (2e-2, 5e-3), f"expert {e}")


@pytest.mark.parametrize("counts,N,K,hint", [([0, 1, 130, 300], 256, 384, 0), ([256, 7], 512, 256, 0),
                                             ([3, 0, 16, 9], 256, 384, 16), ([40, 1], 384, 256, 64)])
def test_fp4_grouped_gemm_swiglu_quantised_out(counts, N, K, hint):
    E, offsets, M, aq, as_, bq, bs = _problem(counts, 2 * N, K, 103)
    C = torch.empty(M, N, dtype=torch.uint8, device="cuda")
    cs = torch.empty(M, N // 128, dtype=torch.float32, device="cuda")
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    moe.moe_grouped_gemm_fp4(dev_u8(aq), dev(as_), dev_u8(bq), dev_u8(_chunks(bs)), dev(offsets), M,
                             E, N, K, moe.MOE_EPILOGUE_SWIGLU, C, cs, ws, max_rows_per_expert=hint)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == 0
    A, Bd = _dequant_e4m3(aq, as_), _dequant_fp4(bq, bs)
    got = _dequant_e4m3(C.cpu().numpy(), cs.cpu().numpy())
    for e in range(E):
        lo, hi = offsets[e], offsets[e + 1]
        if hi == lo:
            continue
        g, u = A[lo:hi] @ Bd[e, :N].T, A[lo:hi] @ Bd[e, N:].T
        # the reference output goes through the same power-of-two e4m3 quantisation
        hq, hs = quant_pow2_e4m3((g / (1 + np.exp(-g)) * u).astype(np.float32))
        check_close(got[lo:hi], _dequant_e4m3(hq, hs), FP8_TOL, f"expert {e}")
        assert np.mean(C.cpu().numpy()[lo:hi] != hq) < 0.02


def run_fp4_forward(cfg, L, ep=moe.MOE_EPILOGUE_SWIGLU):
    d = (cfg.T, cfg.H, cfg.I, cfg.E, cfg.k)
    w13q, w13s = _quant_fp4_dev(L["w13"], cfg.E, 2 * cfg.I, cfg.H)
    w2q, w2s = _quant_fp4_dev(L["w2"], cfg.E, cfg.H, cfg.I)
    ws = torch.zeros(moe.moe_workspace_size(d, moe.MOE_DTYPE_FP4_E2M1), dtype=torch.uint8,
                     device="cuda")
    out = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device="cuda")
    moe.moe_forward_fp4(dev_bf16(L["x"]), dev_bf16(L["wr"]), dev(L["bias"]), w13q, w13s, w2q, w2s,
                        d, ep, out, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == 0
    lay = moe.moe_workspace_layout(d, moe.MOE_DTYPE_FP4_E2M1)
    ids = ws[lay.topk_ids:lay.topk_ids + 4 * cfg.T * cfg.k].cpu().numpy().view(np.int32)
    return mi.bf16_to_f32(host_bf16(out)), ids.reshape(cfg.T, cfg.k)


def check_fp4_layer(cfg, L, act=oracle.ACT_SILU, ep=moe.MOE_EPILOGUE_SWIGLU):
    got, ids = run_fp4_forward(cfg, L, ep)
    toks = mi.token_subset(cfg)
    f4 = oracle.quant_weight_fp4(L["w13"]) + oracle.quant_weight_fp4(L["w2"])
    ref = oracle.moe_forward(L["x"], L["wr"], L["bias"], k=cfg.k, tokens=toks, fp4=f4, act=act)
    np.testing.assert_array_equal(ids[toks], ref["ids"])
    return check_close(got[toks], ref["out"], FP8_TOL, cfg.name)


@pytest.mark.parametrize("kw", [dict(T=200, H=512, I=256, E=16, k=4, subset=0),
                                # T*k > 1024: permuted first, each token quantised into its k rows
                                dict(T=300, H=512, I=256, E=16, k=4, subset=0),
                                dict(T=33, H=256, I=384, E=8, k=2, subset=0),
                                dict(T=16, H=1024, I=2048, E=8, k=2, bias="zero", subset=0)])
def test_fp4_layer_small(kw):
    cfg = mi.CONFIGS["fine_grained_fp4"].with_(**kw)
    check_fp4_layer(cfg, mi.make_layer(cfg))


def test_fp4_layer_geglu():
    cfg = mi.CONFIGS["fine_grained_fp4"].with_(T=100, H=256, I=256, E=8, k=2, subset=0)
    check_fp4_layer(cfg, mi.make_layer(cfg), oracle.ACT_GELU, moe.MOE_EPILOGUE_GEGLU)


def test_fp4_rejects_misaligned_weights():
    cfg = mi.CONFIGS["fine_grained_fp4"].with_(T=8, H=256, I=256, E=2, k=1)
    d = (cfg.T, cfg.H, cfg.I, cfg.E, cfg.k)
    z = torch.zeros(4 << 20, dtype=torch.uint8, device="cuda")
    with pytest.raises(moe.MoeError):
        moe.moe_forward_fp4(z, z, None, z[16:], z, z, z, d, moe.MOE_EPILOGUE_SWIGLU, z, z)


@pytest.mark.slow
def test_fp4_layer_full_size_sampled():
    cfg, L = layer_host("fine_grained_fp4")
    check_fp4_layer(cfg, L)
