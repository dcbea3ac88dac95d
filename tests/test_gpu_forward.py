"""The whole layer on a B200 through the C ABI, against the CPU oracle.

Routing (ids, offsets, permutation) is compared on every token, bit-exact;
outputs on every token for small layers and on a seeded 512-token subset at
full size (each token's output depends on that token only)."""
import numpy as np
import pytest

import moe_inputs as mi
import oracle
from helpers import BF16_TOL, check_close, dev, dev_bf16, host_bf16, layer_host

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import mixture_experts_layer_tcgen05_b200 as moe  # noqa: E402


def run_forward(cfg, L, w13=None, w2=None):
    d = (cfg.T, cfg.H, cfg.I, cfg.E, cfg.k)
    nbytes = moe.moe_workspace_size(d)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    out = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device="cuda")
    moe.moe_forward(dev_bf16(L["x"]), dev_bf16(L["wr"]), dev(L["bias"]),
                    dev_bf16(L["w13"] if w13 is None else w13), dev_bf16(L["w2"] if w2 is None else w2),
                    d, out, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == 0
    lay = moe.moe_workspace_layout(d)
    R = cfg.T * cfg.k

    def view(off, n, dt):
        return ws[off:off + n * np.dtype(dt).itemsize].cpu().numpy().view(dt)

    inter = {
        "ids": view(lay.topk_ids, R, np.int32).reshape(cfg.T, cfg.k),
        "w": view(lay.topk_w, R, np.float32).reshape(cfg.T, cfg.k),
        "offsets": view(lay.offsets, cfg.E + 1, np.int32),
        "perm_token": view(lay.perm_token, R, np.int32),
        "inv_perm": view(lay.inv_perm, R, np.int32).reshape(cfg.T, cfg.k),
        "logits": view(lay.logits, cfg.T * cfg.E, np.float32).reshape(cfg.T, cfg.E),
    }
    return mi.bf16_to_f32(host_bf16(out)), inter


def check_layer(cfg, L, w13=None, w2=None, tokens=None):
    got, inter = run_forward(cfg, L, w13, w2)
    # routing on all tokens, bit-exact
    ref_l = oracle.router_logits(L["x"], L["wr"], L["bias"])
    np.testing.assert_array_equal(inter["logits"].view(np.uint32), ref_l.view(np.uint32))
    ids, w = oracle.topk(ref_l, cfg.k)
    np.testing.assert_array_equal(inter["ids"], ids)
    np.testing.assert_allclose(inter["w"], w, rtol=0, atol=1e-6)
    off, pt, _, ip = oracle.permute(ids, cfg.E)
    np.testing.assert_array_equal(inter["offsets"], off)
    np.testing.assert_array_equal(inter["perm_token"], pt)
    np.testing.assert_array_equal(inter["inv_perm"], ip)
    # outputs on the sample
    toks = mi.token_subset(cfg) if tokens is None else tokens
    ref = oracle.experts_combine(L["x"], toks, ids[toks], w[toks],
                                 L["w13"] if w13 is None else w13, L["w2"] if w2 is None else w2)
    return check_close(got[toks], ref, BF16_TOL, cfg.name), off


def test_tiny_layer_all_tokens():
    cfg, L = layer_host("tiny")
    check_layer(cfg, L)


def test_mixtral_decode_all_tokens():
    cfg, L = layer_host("mixtral_decode")
    check_layer(cfg, L)


@pytest.mark.parametrize("kw", [
    dict(T=1),                                   # one token
    dict(T=100, E=1, k=1),                       # one expert, ragged T
    dict(T=45, E=4, k=4, bias="normal"),         # k = E
    dict(T=300, E=16, k=1, H=256, I=384),        # Switch top-1, I not a multiple of 256
    dict(T=513, E=32, k=4, H=384, I=256),        # rows spanning several tiles + ragged tail
    dict(T=40, E=8, k=2, H=256, I=128),          # decode-sized (small-M path)
    # E > 32: the wide router with its h blocks as separate CTAs (H % 256 == 0) or not
    dict(T=200, E=40, k=4, H=256, I=256, bias="normal"),
    dict(T=77, E=37, k=3, H=512, I=128),         # E not a multiple of 8
    dict(T=150, E=48, k=2, H=384, I=256),        # H % 256 != 0: blocks in one CTA
])
def test_edge_shapes(kw):
    cfg = mi.CONFIGS["tiny"].with_(**kw)
    check_layer(cfg, mi.make_layer(cfg))


def test_one_expert_takes_every_token():
    cfg = mi.CONFIGS["tiny"].with_(T=300, E=8, k=2)
    L = mi.make_layer(cfg)
    L["bias"] = L["bias"].copy()
    L["bias"][3] = 100.0  # expert 3 wins slot 0 everywhere
    _, off = check_layer(cfg, L)
    assert off[4] - off[3] == cfg.T


def test_empty_experts_skewed_routing():
    cfg = mi.CONFIGS["fine_grained"].with_(T=512, H=512, I=256, E=64)
    L = mi.make_layer(cfg)
    _, off = check_layer(cfg, L)
    assert np.sum(np.diff(off) == 0) >= 1, "expected at least one empty expert"


@pytest.mark.slow
def test_mixtral_prefill_full_size_sampled():
    cfg, L = layer_host("mixtral_prefill")
    check_layer(cfg, L)


@pytest.mark.slow
def test_fine_grained_full_size_sampled():
    cfg, L = layer_host("fine_grained")
    _, off = check_layer(cfg, L)
    counts = np.diff(off)
    # Zipf-skewed load: the largest expert holds many times the mean, and some experts get no
    # token at all
    assert counts.max() > 8 * counts.mean()
    assert np.sum(counts == 0) >= 1, "expected at least one empty expert at full size"
