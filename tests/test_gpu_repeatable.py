"""Bitwise repeatability of the whole layer on a B200.

The C ABI promises results that are identical run to run: every sum runs in
a fixed order (router blocks, GEMM K steps, split-K and K-split reduces, the
combine's slots) and no atomic decides an order. Two forwards on the same
inputs, each with a fresh workspace, must agree bit for bit in the output
and in every routing intermediate they expose."""
import numpy as np
import pytest

import moe_inputs as mi

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from test_gpu_forward import run_forward  # noqa: E402
from test_gpu_fp4 import run_fp4_forward  # noqa: E402
from test_gpu_fp8 import run_fp8_forward  # noqa: E402
from test_gpu_mx import run_mx_forward  # noqa: E402


def _same_bytes(a, b):
    return np.ascontiguousarray(a).tobytes() == np.ascontiguousarray(b).tobytes()


@pytest.mark.parametrize("name,kw", [
    ("tiny", dict(T=40, E=8, k=2, H=256, I=128)),            # decode-sized: weights-in-M GEMMs
    ("tiny", dict(T=513, E=32, k=4, H=384, I=256)),          # row scatter, several tiles per expert
    ("fine_grained", dict(T=512, H=512, I=256, E=64)),       # split router, skewed experts
])
def test_bf16_layer_is_bitwise_repeatable(name, kw):
    cfg = mi.CONFIGS[name].with_(**kw)
    L = mi.make_layer(cfg)
    a, ia = run_forward(cfg, L)
    b, ib = run_forward(cfg, L)
    assert _same_bytes(a, b), "output"
    for key in ("logits", "ids", "w", "offsets", "perm_token", "inv_perm"):
        assert _same_bytes(ia[key], ib[key]), key


QUANT_SHAPES = [dict(T=300, H=512, I=256, E=16, k=4, subset=0),                  # T*k > 1024
                dict(T=16, H=1024, I=2048, E=8, k=2, bias="zero", subset=0)]     # decode-sized


@pytest.mark.parametrize("kw", QUANT_SHAPES)
@pytest.mark.parametrize("layer", ["fp8", "fp8_ue8m0", "fp4"])
def test_quantised_layers_are_bitwise_repeatable(layer, kw):
    base, run = {"fp8": ("fine_grained_fp8", run_fp8_forward),
                 "fp8_ue8m0": ("fine_grained_fp8", run_mx_forward),
                 "fp4": ("fine_grained_fp4", run_fp4_forward)}[layer]
    cfg = mi.CONFIGS[base].with_(**kw)
    L = mi.make_layer(cfg)
    a, ida = run(cfg, L)
    b, idb = run(cfg, L)
    assert _same_bytes(ida, idb), "ids"
    assert _same_bytes(a, b), "output"
