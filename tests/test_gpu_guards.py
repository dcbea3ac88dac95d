"""Guard regions around every buffer the kernels write, on a B200.

No sanitizer runs on these GPUs, so out-of-bounds writes are looked for with
canary bytes: each output and workspace buffer sits between two 4 KB guards
holding a known byte, and after the call both guards must be unchanged. The
shapes are ragged (experts whose rows end mid-tile, a last tile hanging past
the last row, empty experts) so that every masked edge is exercised: the
row scatter, the split router's block sums, the GEMM epilogues and their
split-K / K-split partials, the quantised copies and the combine. Its calls
repeat ones the parity tests make."""
import numpy as np
import pytest

import moe_inputs as mi
from helpers import Guarded, dev, dev_bf16

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import mixture_experts_layer_tcgen05_b200 as moe  # noqa: E402
from test_gpu_fp4 import _quant_fp4_dev  # noqa: E402
from test_gpu_kernels import _grouped_problem  # noqa: E402


def _check(ws, *bufs):
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws.t) == 0
    assert ws.intact(), "workspace guards"
    for i, b in enumerate(bufs):
        assert b.intact(), f"guards of output {i}"


@pytest.mark.parametrize("name,kw", [
    ("tiny", dict(T=40, E=8, k=2, H=256, I=128)),            # decode-sized: weights-in-M, split-K
    ("tiny", dict(T=513, E=32, k=4, H=384, I=256)),          # several tiles per expert, ragged tail
    ("fine_grained", dict(T=512, H=512, I=256, E=64)),       # split router, empty experts
])
def test_bf16_forward_stays_inside_its_buffers(name, kw):
    cfg = mi.CONFIGS[name].with_(**kw)
    L = mi.make_layer(cfg)
    d = (cfg.T, cfg.H, cfg.I, cfg.E, cfg.k)
    ws = Guarded((moe.moe_workspace_size(d),), torch.uint8, fill=0)
    out = Guarded((cfg.T, cfg.H), torch.bfloat16)
    moe.moe_forward(dev_bf16(L["x"]), dev_bf16(L["wr"]), dev(L["bias"]), dev_bf16(L["w13"]),
                    dev_bf16(L["w2"]), d, out.t, ws.t)
    _check(ws, out)


@pytest.mark.parametrize("kw", [dict(T=300, H=512, I=256, E=16, k=4, subset=0),
                                dict(T=16, H=1024, I=2048, E=8, k=2, bias="zero", subset=0)])
@pytest.mark.parametrize("layer", ["fp8", "fp8_ue8m0", "fp4"])
def test_quantised_forward_stays_inside_its_buffers(layer, kw):
    cfg = mi.CONFIGS["fine_grained_fp4" if layer == "fp4" else "fine_grained_fp8"].with_(**kw)
    L = mi.make_layer(cfg)
    d = (cfg.T, cfg.H, cfg.I, cfg.E, cfg.k)
    if layer == "fp4":
        dt = moe.MOE_DTYPE_FP4_E2M1
        w13q, w13s = _quant_fp4_dev(L["w13"], cfg.E, 2 * cfg.I, cfg.H)
        w2q, w2s = _quant_fp4_dev(L["w2"], cfg.E, cfg.H, cfg.I)
    else:
        ue = layer == "fp8_ue8m0"
        dt = moe.MOE_DTYPE_FP8_E4M3_UE8M0 if ue else moe.MOE_DTYPE_FP8_E4M3
        fmt = moe.MOE_SCALE_UE8M0 if ue else moe.MOE_SCALE_F32
        w13q = torch.empty(cfg.E, 2 * cfg.I, cfg.H, dtype=torch.uint8, device="cuda")
        w13s = torch.empty(cfg.E, 2 * cfg.I // 128, cfg.H // 128, dtype=torch.float32, device="cuda")
        w2q = torch.empty(cfg.E, cfg.H, cfg.I, dtype=torch.uint8, device="cuda")
        w2s = torch.empty(cfg.E, cfg.H // 128, cfg.I // 128, dtype=torch.float32, device="cuda")
        moe.moe_quantize_weight_fp8_fmt(dev_bf16(L["w13"]), cfg.E, 2 * cfg.I, cfg.H, w13q, w13s, fmt)
        moe.moe_quantize_weight_fp8_fmt(dev_bf16(L["w2"]), cfg.E, cfg.H, cfg.I, w2q, w2s, fmt)
    ws = Guarded((moe.moe_workspace_size(d, dt),), torch.uint8, fill=0)
    out = Guarded((cfg.T, cfg.H), torch.bfloat16)
    x, wr, b = dev_bf16(L["x"]), dev_bf16(L["wr"]), dev(L["bias"])
    if layer == "fp4":
        moe.moe_forward_fp4(x, wr, b, w13q, w13s, w2q, w2s, d, moe.MOE_EPILOGUE_SWIGLU, out.t, ws.t)
    elif layer == "fp8_ue8m0":
        moe.moe_forward_fp8_ue8m0(x, wr, b, w13q, w13s, w2q, w2s, d, moe.MOE_EPILOGUE_SWIGLU,
                                  out.t, ws.t)
    else:
        moe.moe_forward_fp8(x, wr, b, w13q, w13s, w2q, w2s, d, out.t, ws.t)
    _check(ws, out)


@pytest.mark.parametrize("swiglu", [False, True])
@pytest.mark.parametrize("counts,N,K,hint,ws_bytes", [
    ([0, 1, 130, 300], 256, 384, 0, 4096),        # tokens-in-M tiles, last tile past the last row
    ([31, 2, 32, 0, 9], 384, 256, 32, 4096),      # weights-in-M, 32 token columns
    ([20000, 300, 0, 180], 256, 128, 0, 32 << 20),  # last wave split over K (plain GEMM)
])
def test_grouped_gemm_stays_inside_its_buffers(counts, N, K, hint, ws_bytes, swiglu):
    E, offsets, M, A, B = _grouped_problem(counts, 2 * N if swiglu else N, K, 61)
    C = Guarded((M, N), torch.bfloat16)
    ws = Guarded((ws_bytes,), torch.uint8, fill=0)
    moe.moe_grouped_gemm(dev_bf16(A), dev_bf16(B), dev(offsets), M, E, N, K, moe.MOE_DTYPE_BF16,
                         moe.MOE_EPILOGUE_SWIGLU if swiglu else moe.MOE_EPILOGUE_NONE, C.t,
                         max_rows_per_expert=hint, ws=ws.t)
    _check(ws, C)


@pytest.mark.parametrize("T,E,k,H", [(1000, 256, 8, 384),   # chunked permutation + row scatter
                                     (64, 8, 2, 256)])      # one-launch small-batch permutation
def test_permute_and_combine_stay_inside_their_buffers(T, E, k, H):
    rng = np.random.default_rng(T + E)
    ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    x = mi.normal_bf16(0, 71, 1.0, 1, T, H).reshape(T, H)
    d = (T, H, 128, E, k)
    ws = Guarded((moe.moe_workspace_size(d),), torch.uint8, fill=0)
    off = Guarded((E + 1,), torch.int32)
    pt = Guarded((T * k,), torch.int32)
    ip = Guarded((T * k,), torch.int32)
    xp = Guarded((T * k, H), torch.bfloat16)
    moe.moe_permute(dev(ids), d, off.t, pt.t, ip.t, dev_bf16(x), xp.t, ws.t)
    _check(ws, off, pt, ip, xp)
    w = rng.random((T, k)).astype(np.float32)
    out = Guarded((T, H), torch.bfloat16)
    moe.moe_combine(xp.t, dev(w), ip.t, d, out.t)
    torch.cuda.synchronize()
    assert out.intact() and xp.intact() and ip.intact()
