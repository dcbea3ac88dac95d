"""Gated expert activations other than SwiGLU (GeGLU, ReGLU) on a B200,
through the C ABI, against the CPU oracle.

"Experts backends" lists experts whose gated activation is silu, gelu or
relu; the GEMM-1 epilogue computes act(g) * u for each. Every kernel that
carries the epilogue is covered: the tokens-in-M GEMM, the small-M (weights
in M) GEMM with and without split-K, the FP8 GEMM, and both whole layers."""
import numpy as np
import pytest

import moe_inputs as mi
import oracle
from helpers import BF16_TOL, FP8_TOL, check_close, dev, dev_bf16, host_bf16

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import mixture_experts_layer_tcgen05_b200 as moe  # noqa: E402

ACTS = [(moe.MOE_EPILOGUE_SWIGLU, oracle.ACT_SILU), (moe.MOE_EPILOGUE_GEGLU, oracle.ACT_GELU),
        (moe.MOE_EPILOGUE_REGLU, oracle.ACT_RELU)]


def _problem(counts, N2, K, tag):
    E = len(counts)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    M = int(offsets[-1])
    A = mi.normal_bf16(0, tag, 1.0, 1, M, K).reshape(M, K)
    B = mi.normal_bf16(0, tag + 1, 0.05, E, N2, K).reshape(E, N2, K)
    return E, offsets, M, A, B


@pytest.mark.parametrize("ep,act", ACTS[1:])
@pytest.mark.parametrize("counts,N,K,hint,ws_bytes", [
    ([0, 1, 130, 300], 256, 384, 0, 4096),          # tokens-in-M kernel
    ([0, 1, 17, 64], 256, 256, 64, 4096),           # small-M kernel
    ([3, 0, 16], 128, 4096, 16, 64 << 20),          # small-M kernel with split-K
    ([0, 1, 130, 300, 257], 256, 4096, 0, 4096),    # K >= 4096: two-half (256-row) tiles
])
def test_grouped_gemm_gated(ep, act, counts, N, K, hint, ws_bytes):
    E, offsets, M, A, B = _problem(counts, 2 * N, K, 71)
    C = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device="cuda")
    moe.moe_grouped_gemm(dev_bf16(A), dev_bf16(B), dev(offsets), M, E, N, K, moe.MOE_DTYPE_BF16,
                         ep, C, max_rows_per_expert=hint, ws=ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == 0
    got = mi.bf16_to_f32(host_bf16(C))
    for e in range(E):
        lo, hi = offsets[e], offsets[e + 1]
        if hi > lo:
            check_close(got[lo:hi], oracle.expert_gated_rows(A[lo:hi], B[e], act), BF16_TOL,
                        f"expert {e}")


def _routing(cfg, L):
    logits = oracle.router_logits(L["x"], L["wr"], L["bias"])
    return oracle.topk(logits, cfg.k)


@pytest.mark.parametrize("ep,act", ACTS)
@pytest.mark.parametrize("kw", [dict(T=64), dict(T=40, H=256, I=128),          # small-M path
                                dict(T=300, E=16, k=1, H=256, I=384, bias="normal")])
def test_forward_gated(ep, act, kw):
    cfg = mi.CONFIGS["tiny"].with_(**kw)
    L = mi.make_layer(cfg)
    d = (cfg.T, cfg.H, cfg.I, cfg.E, cfg.k)
    ws = torch.zeros(moe.moe_workspace_size(d), dtype=torch.uint8, device="cuda")
    out = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device="cuda")
    moe.moe_forward_gated(dev_bf16(L["x"]), dev_bf16(L["wr"]), dev(L["bias"]), dev_bf16(L["w13"]),
                          dev_bf16(L["w2"]), d, ep, out, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == 0
    lay = moe.moe_workspace_layout(d)
    ids_dev = ws[lay.topk_ids:lay.topk_ids + 4 * cfg.T * cfg.k].cpu().numpy().view(np.int32)
    ids, w = _routing(cfg, L)
    np.testing.assert_array_equal(ids_dev.reshape(cfg.T, cfg.k), ids)
    toks = np.arange(cfg.T, dtype=np.int32)
    ref = oracle.experts_combine(L["x"], toks, ids, w, L["w13"], L["w2"], act=act)
    check_close(mi.bf16_to_f32(host_bf16(out)), ref, BF16_TOL, f"act {act}")


@pytest.mark.parametrize("ep,act", ACTS[1:])
def test_forward_fp8_gated(ep, act):
    cfg = mi.CONFIGS["fine_grained_fp8"].with_(T=200, H=512, I=256, E=16, k=4, subset=0)
    L = mi.make_layer(cfg)
    d = (cfg.T, cfg.H, cfg.I, cfg.E, cfg.k)
    w13q = torch.empty(cfg.E, 2 * cfg.I, cfg.H, dtype=torch.uint8, device="cuda")
    w13s = torch.empty(cfg.E, 2 * cfg.I // 128, cfg.H // 128, dtype=torch.float32, device="cuda")
    w2q = torch.empty(cfg.E, cfg.H, cfg.I, dtype=torch.uint8, device="cuda")
    w2s = torch.empty(cfg.E, cfg.H // 128, cfg.I // 128, dtype=torch.float32, device="cuda")
    moe.moe_quantize_weight_fp8(dev_bf16(L["w13"]), cfg.E, 2 * cfg.I, cfg.H, w13q, w13s)
    moe.moe_quantize_weight_fp8(dev_bf16(L["w2"]), cfg.E, cfg.H, cfg.I, w2q, w2s)
    ws = torch.zeros(moe.moe_workspace_size(d, moe.MOE_DTYPE_FP8_E4M3), dtype=torch.uint8,
                     device="cuda")
    out = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device="cuda")
    moe.moe_forward_fp8_gated(dev_bf16(L["x"]), dev_bf16(L["wr"]), dev(L["bias"]), w13q, w13s, w2q,
                              w2s, d, ep, out, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == 0
    toks = np.arange(cfg.T, dtype=np.int32)
    fq = oracle.quant_weight_fp8(L["w13"]) + oracle.quant_weight_fp8(L["w2"])
    ref = oracle.moe_forward(L["x"], L["wr"], L["bias"], k=cfg.k, tokens=toks, fp8=fq, act=act)
    check_close(mi.bf16_to_f32(host_bf16(out)), ref["out"], FP8_TOL, f"act {act}")


def test_forward_gated_rejects_plain_epilogue():
    cfg = mi.CONFIGS["tiny"]
    d = (cfg.T, cfg.H, cfg.I, cfg.E, cfg.k)
    z = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
    with pytest.raises(moe.MoeError):
        moe.moe_forward_gated(z, z, None, z, z, d, moe.MOE_EPILOGUE_NONE, z, z)
