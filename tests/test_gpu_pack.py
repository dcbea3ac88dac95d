"""moe_pack_weights on a B200: logical expert weights (Wg, Wu [E, H, I],
Wd [E, I, H]) packed into the K-major w13 / w2 the forward reads, compared
byte for byte with the generator's own K-major draw of the same values, and a
forward on the packed weights against the CPU oracle."""
import numpy as np
import pytest

import moe_inputs as mi
from helpers import dev_bf16, host_bf16

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import mixture_experts_layer_tcgen05_b200 as moe  # noqa: E402
from test_gpu_forward import check_layer  # noqa: E402


def _logical(cfg):
    """Wg, Wu [E, H, I] and Wd [E, I, H] as raw bf16 bits, drawn in their logical layout."""
    E, H, I = cfg.E, cfg.H, cfg.I
    wg = mi.normal_bf16(cfg.seed, mi.TAG_WG, cfg.w_sigma, E, H, I).reshape(E, H, I)
    wu = mi.normal_bf16(cfg.seed, mi.TAG_WU, cfg.w_sigma, E, H, I).reshape(E, H, I)
    wd = mi.normal_bf16(cfg.seed, mi.TAG_WD, cfg.w_sigma, E, I, H).reshape(E, I, H)
    return wg, wu, wd


def _pack(cfg):
    wg, wu, wd = (dev_bf16(a) for a in _logical(cfg))
    w13 = torch.full((cfg.E, 2 * cfg.I, cfg.H), float("nan"), dtype=torch.bfloat16, device="cuda")
    w2 = torch.full((cfg.E, cfg.H, cfg.I), float("nan"), dtype=torch.bfloat16, device="cuda")
    moe.moe_pack_weights(wg, wu, wd, cfg.E, cfg.H, cfg.I, w13, w2)
    torch.cuda.synchronize()
    return host_bf16(w13), host_bf16(w2)


@pytest.mark.parametrize("kw", [dict(E=3, H=256, I=384), dict(E=8, H=1024, I=2048),
                                dict(E=1, H=128, I=128)])
def test_pack_weights_bit_exact(kw):
    cfg = mi.CONFIGS["tiny"].with_(**kw)
    w13, w2 = _pack(cfg)
    np.testing.assert_array_equal(w13, mi.make_w13(cfg))
    np.testing.assert_array_equal(w2, mi.make_w2(cfg))


def test_forward_on_packed_weights_matches_oracle():
    cfg = mi.CONFIGS["tiny"].with_(T=300, E=16, k=4, H=512, I=384, bias="normal")
    L = mi.make_layer(cfg)
    w13, w2 = _pack(cfg)
    check_layer(cfg, L, w13=w13, w2=w2)
