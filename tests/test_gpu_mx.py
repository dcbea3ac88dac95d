"""FP8 with power-of-two (UE8M0) scales on the block-scaled tensor-core path,
on a B200 through the C ABI, against the CPU oracle.

"Experts backends", "FP8 and FP4 quantized experts" / "UE8M0 scale format":
scales stored as 8-bit exponents, which the block-scaled MMA applies itself.
The GEMM tests compare with the dense product of the dequantised operands
(exact products; only the fp32 accumulation order and the output rounding
differ); the layer tests with the oracle run on the same power-of-two
quantisation, within the FP8 tolerance."""
import numpy as np
import pytest

import moe_inputs as mi
import oracle
from helpers import (FP8_TOL, check_close, dev, dev_bf16, dev_u8, host_bf16, layer_host,
                     quant_pow2_e4m3)

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import mixture_experts_layer_tcgen05_b200 as moe  # noqa: E402

DT = moe.MOE_DTYPE_FP8_E4M3_UE8M0


def _dec_table():
    return np.array([oracle.e4m3_decode(q) for q in range(256)])


def _problem(counts, NB, K, tag, unit_scales=False):
    E = len(counts)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    M = int(offsets[-1])
    A = mi.normal_bf16(0, tag, 1.0, 1, M, K).reshape(M, K)
    B = mi.normal_bf16(0, tag + 1, 0.05, E, NB, K).reshape(E, NB, K)
    aq, as_ = oracle.quant_act_fp8(A, ue8m0=True)
    bq, bs = oracle.quant_weight_fp8(B, ue8m0=True)
    if unit_scales:
        as_, bs = np.ones_like(as_), np.ones_like(bs)
    return E, offsets, M, aq, as_, bq, bs


def _dense(aq, as_, bq, bs):
    dec = _dec_table()
    A = dec[aq] * np.repeat(as_, 128, 1)
    Bd = dec[bq] * np.repeat(np.repeat(bs, 128, 1), 128, 2)
    return A, Bd


@pytest.mark.parametrize("unit", [True, False])
@pytest.mark.parametrize("counts,N,K,hint", [
    ([0, 1, 130, 300], 256, 384, 0), ([128, 0, 5], 512, 256, 0), ([700], 256, 1024, 0),
    # decode sizes: weights in M, 16 / 32 / 64 token columns
    ([3, 0, 16, 9], 256, 384, 16), ([1, 30, 2], 384, 256, 32), ([50, 64, 0, 33], 128, 512, 64)])
def test_mx_grouped_gemm_plain(counts, N, K, hint, unit):
    """unit: every scale 1 (the MMA alone); else power-of-two scales per row,
    per 128-row weight block and per 128-K block (the scale-factor layout)."""
    if hint == 0 and N % 256:
        pytest.skip("the tokens-in-M form tiles N by 256")
    E, offsets, M, aq, as_, bq, bs = _problem(counts, N, K, 91, unit)
    C = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    moe.moe_grouped_gemm(dev_u8(aq), dev_u8(bq), dev(offsets), M, E, N, K, DT,
                         moe.MOE_EPILOGUE_NONE, C, dev(as_), dev(bs), max_rows_per_expert=hint, ws=ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == 0
    A, Bd = _dense(aq, as_, bq, bs)
    got = mi.bf16_to_f32(host_bf16(C))
    for e in range(E):
        lo, hi = offsets[e], offsets[e + 1]
        if hi > lo:
            check_close(got[lo:hi], A[lo:hi] @ Bd[e].T, (2e-2, 5e-3), f"expert {e}")


@pytest.mark.parametrize("counts,N,K,hint", [([0, 1, 130, 300], 256, 384, 0), ([256, 7], 512, 256, 0),
                                             ([3, 0, 16, 9], 256, 384, 16), ([40, 1], 384, 256, 64)])
def test_mx_grouped_gemm_swiglu_quantised_out(counts, N, K, hint):
    E, offsets, M, aq, as_, bq, bs = _problem(counts, 2 * N, K, 93)
    C = torch.empty(M, N, dtype=torch.uint8, device="cuda")
    cs = torch.empty(M, N // 128, dtype=torch.float32, device="cuda")
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    moe.moe_grouped_gemm(dev_u8(aq), dev_u8(bq), dev(offsets), M, E, N, K, DT,
                         moe.MOE_EPILOGUE_SWIGLU, C, dev(as_), dev(bs), cs, max_rows_per_expert=hint,
                         ws=ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == 0
    dec = _dec_table()
    A, Bd = _dense(aq, as_, bq, bs)
    csn = cs.cpu().numpy()
    m, _ = np.frexp(csn[np.concatenate([np.arange(offsets[e], offsets[e + 1]) for e in range(E)])])
    assert np.all(m == 0.5), "output scales are powers of two"
    got = dec[C.cpu().numpy()] * np.repeat(csn, 128, 1)
    for e in range(E):
        lo, hi = offsets[e], offsets[e + 1]
        if hi == lo:
            continue
        g = A[lo:hi] @ Bd[e, :N].T
        u = A[lo:hi] @ Bd[e, N:].T
        h = (g / (1 + np.exp(-g)) * u).astype(np.float32)
        hq, hs = quant_pow2_e4m3(h)
        ref = dec[hq] * np.repeat(hs, 128, 1)
        check_close(got[lo:hi], ref, FP8_TOL, f"expert {e}")
        assert np.mean(C.cpu().numpy()[lo:hi] != hq) < 0.02


def run_mx_forward(cfg, L, ep=moe.MOE_EPILOGUE_SWIGLU):
    d = (cfg.T, cfg.H, cfg.I, cfg.E, cfg.k)
    w13q = torch.empty(cfg.E, 2 * cfg.I, cfg.H, dtype=torch.uint8, device="cuda")
    w13s = torch.empty(cfg.E, 2 * cfg.I // 128, cfg.H // 128, dtype=torch.float32, device="cuda")
    w2q = torch.empty(cfg.E, cfg.H, cfg.I, dtype=torch.uint8, device="cuda")
    w2s = torch.empty(cfg.E, cfg.H // 128, cfg.I // 128, dtype=torch.float32, device="cuda")
    moe.moe_quantize_weight_fp8_fmt(dev_bf16(L["w13"]), cfg.E, 2 * cfg.I, cfg.H, w13q, w13s,
                                    moe.MOE_SCALE_UE8M0)
    moe.moe_quantize_weight_fp8_fmt(dev_bf16(L["w2"]), cfg.E, cfg.H, cfg.I, w2q, w2s,
                                    moe.MOE_SCALE_UE8M0)
    ws = torch.zeros(moe.moe_workspace_size(d, DT), dtype=torch.uint8, device="cuda")
    out = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device="cuda")
    moe.moe_forward_fp8_ue8m0(dev_bf16(L["x"]), dev_bf16(L["wr"]), dev(L["bias"]), w13q, w13s, w2q,
                              w2s, d, ep, out, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == 0
    lay = moe.moe_workspace_layout(d, DT)
    ids = ws[lay.topk_ids:lay.topk_ids + 4 * cfg.T * cfg.k].cpu().numpy().view(np.int32)
    return mi.bf16_to_f32(host_bf16(out)), ids.reshape(cfg.T, cfg.k)


def check_mx_layer(cfg, L, act=oracle.ACT_SILU, ep=moe.MOE_EPILOGUE_SWIGLU):
    got, ids = run_mx_forward(cfg, L, ep)
    toks = mi.token_subset(cfg)
    fq = oracle.quant_weight_fp8(L["w13"], ue8m0=True) + oracle.quant_weight_fp8(L["w2"], ue8m0=True)
    ref = oracle.moe_forward(L["x"], L["wr"], L["bias"], k=cfg.k, tokens=toks, fp8=fq, act=act,
                             ue8m0=True)
    np.testing.assert_array_equal(ids[toks], ref["ids"])
    return check_close(got[toks], ref["out"], FP8_TOL, cfg.name)


@pytest.mark.parametrize("kw", [dict(T=200, H=512, I=256, E=16, k=4, subset=0),
                                # T*k > 1024: permuted first, each token quantised into its k rows
                                dict(T=300, H=512, I=256, E=16, k=4, subset=0),
                                dict(T=33, H=256, I=384, E=8, k=2, subset=0),
                                dict(T=16, H=1024, I=2048, E=8, k=2, bias="zero", subset=0)])
def test_mx_layer_small(kw):
    cfg = mi.CONFIGS["fine_grained_fp8"].with_(**kw)
    check_mx_layer(cfg, mi.make_layer(cfg))


def test_mx_layer_geglu():
    cfg = mi.CONFIGS["fine_grained_fp8"].with_(T=100, H=256, I=256, E=8, k=2, subset=0)
    check_mx_layer(cfg, mi.make_layer(cfg), oracle.ACT_GELU, moe.MOE_EPILOGUE_GEGLU)


@pytest.mark.slow
def test_mx_layer_full_size_sampled():
    cfg, L = layer_host("fine_grained_fp8")
    check_mx_layer(cfg, L)
