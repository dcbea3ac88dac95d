"""Pins of the CPU oracle to things other than itself (CPU only).

Each test checks one oracle function against a closed form, a rigorous error
bound, brute force on tiny inputs, an invariant, a library routine, or the
hand-worked example in tests/golden/. Together they are chosen so that a
dropped term, a wrong sign or index, a transposed operand or a wrong tie rule
in the oracle fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import moe_inputs as mi
import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _small(name="tiny", **kw):
    return mi.CONFIGS[name].with_(**kw)


def _logical_weights(cfg):
    """Wg, Wu [E,H,I], Wd [E,I,H] in fp64 drawn in their logical layout (no packing)."""
    E, H, I = cfg.E, cfg.H, cfg.I
    wg = mi.bf16_to_f32(mi.normal_bf16(cfg.seed, mi.TAG_WG, cfg.w_sigma, E, H, I)).reshape(E, H, I)
    wu = mi.bf16_to_f32(mi.normal_bf16(cfg.seed, mi.TAG_WU, cfg.w_sigma, E, H, I)).reshape(E, H, I)
    wd = mi.bf16_to_f32(mi.normal_bf16(cfg.seed, mi.TAG_WD, cfg.w_sigma, E, I, H)).reshape(E, I, H)
    return wg.astype(np.float64), wu.astype(np.float64), wd.astype(np.float64)


def _bf16(a):
    return mi.f32_to_bf16(np.asarray(a, dtype=np.float32))


# --------------------------------------------------------------------------
# the hand-worked example (closed forms)
# --------------------------------------------------------------------------
def _golden_layer():
    g = json.load(open(os.path.join(GOLDEN, "hand_worked_layer.json")))
    d = g["dims"]
    E, H, I = d["E"], d["H"], d["I"]
    wg = np.array(g["wg_EHI"], dtype=np.float32)
    wu = np.array(g["wu_EHI"], dtype=np.float32)
    wd = np.array(g["wd_EIH"], dtype=np.float32)
    w13 = np.concatenate([wg.transpose(0, 2, 1), wu.transpose(0, 2, 1)], axis=1)  # [E,2I,H]
    w2 = wd.transpose(0, 2, 1)  # [E,H,I]
    return g, dict(x=_bf16(g["x"]), wr=_bf16(g["wr_HE"]), bias=np.array(g["bias"], np.float32),
                   w13=_bf16(w13), w2=_bf16(w2), k=d["k"], E=E)


def test_hand_worked_layer():
    g, L = _golden_layer()
    exp = g["expected"]
    r = oracle.moe_forward(L["x"], L["wr"], L["bias"], L["w13"], L["w2"], k=L["k"])
    np.testing.assert_array_equal(r["logits"], np.array(exp["logits"], np.float32))
    np.testing.assert_array_equal(r["ids"], np.array(exp["ids"]))
    np.testing.assert_allclose(r["w"], np.array(exp["w"]), rtol=0, atol=2 ** -24)
    np.testing.assert_allclose(r["out"], np.array(exp["out"]), rtol=2 ** -22, atol=0)
    offsets, perm_token, _, inv_perm = oracle.permute(r["ids"], L["E"])
    np.testing.assert_array_equal(offsets, exp["offsets"])
    np.testing.assert_array_equal(perm_token, exp["perm_token"])
    np.testing.assert_array_equal(inv_perm, exp["inv_perm"])


# --------------------------------------------------------------------------
# router logits: rigorous fp32 summation bound against an fp64 recomputation
# --------------------------------------------------------------------------
@pytest.mark.parametrize("H,E,T", [(128, 8, 64), (1024, 32, 16), (96, 5, 7)])
def test_logits_within_higham_bound(H, E, T):
    cfg = _small(H=H, E=E, T=T, bias="normal")
    x = mi.make_x(cfg)
    wr, b = mi.make_router(cfg)
    l32 = oracle.router_logits(x, wr, b)
    xf = mi.bf16_to_f32(x).astype(np.float64)
    wf = mi.bf16_to_f32(wr).astype(np.float64)
    l64 = xf @ wf + b.astype(np.float64)
    # recursive summation of H exact products: |err| <= gamma_{H-1} sum|x w| (Higham Thm 3.1),
    # plus one rounding of the bias add
    u = 2.0 ** -24
    gam = (H - 1) * u / (1 - (H - 1) * u)
    bound = gam * (np.abs(xf) @ np.abs(wf)) + u * (np.abs(l64) + 1e-30) * 2
    err = np.abs(l32.astype(np.float64) - l64)
    assert np.all(err <= bound), float((err - bound).max())
    # sensitivity: a sum missing one product (a dropped term) breaks the bound almost everywhere
    dropped = l64 - xf[:, :1] @ wf[:1, :]
    assert np.mean(np.abs(dropped - l64) > bound) > 0.75


def test_logits_blocked_order_closed_form():
    """The fixed fp32 order: 8 contiguous h blocks, each summed from 0 in h
    order, block sums added left to right. With x = 1, a column of Wr holding
    2^24 then 0 (block 0) and pairs of ones (blocks 1..7) sums to 2^24 + 14
    exactly: each block of ones gives 2, and 2^24 + 2 is representable. Summed
    h-sequentially every +1 after 2^24 would round away (2^24 + 1 is a tie to
    even), and with 4 blocks the answer would be 2^24 + 12."""
    H, E = 16, 2
    x = _bf16(np.ones((1, H), np.float32))
    col = np.array([2.0 ** 24, 0.0] + [1.0, 1.0] * 7, np.float32)
    wr = np.stack([col, col[::-1]], axis=1)  # expert 1: the big term last
    got = oracle.router_logits(x, _bf16(wr), None)
    np.testing.assert_array_equal(got, np.full((1, E), 2.0 ** 24 + 14, np.float32))


def test_logits_subset_rows_match_full():
    cfg = _small(T=40)
    x = mi.make_x(cfg)
    wr, b = mi.make_router(cfg)
    full = oracle.router_logits(x, wr, b)
    toks = np.array([3, 17, 39], dtype=np.int32)
    np.testing.assert_array_equal(oracle.router_logits(x, wr, b, tokens=toks), full[toks])


# --------------------------------------------------------------------------
# top-k selection and weights
# --------------------------------------------------------------------------
def _brute_topk(logits, k):
    ids = np.empty((logits.shape[0], k), np.int32)
    for t, l in enumerate(logits):
        order = np.lexsort((np.arange(len(l)), -l.astype(np.float64)))  # logit desc, index asc
        ids[t] = order[:k]
    return ids


@pytest.mark.parametrize("E,k", [(8, 2), (256, 8), (5, 5), (7, 1), (1, 1), (64, 16)])
def test_topk_matches_lexsort_and_softmax(E, k):
    rng = np.random.default_rng(E * 100 + k)
    T = 50
    logits = rng.standard_normal((T, E)).astype(np.float32)
    logits[::7, : E // 2] = 0.25  # planted exact ties
    ids, w = oracle.topk(logits, k)
    np.testing.assert_array_equal(ids, _brute_topk(logits, k))
    # renormalised weights = softmax over the selected logits (library routine, fp64)
    sel = np.take_along_axis(logits, ids, 1).astype(np.float64)
    ref = torch.softmax(torch.from_numpy(sel), dim=1).numpy()
    np.testing.assert_allclose(w, ref, rtol=0, atol=2 ** -24)
    assert np.all(np.abs(w.astype(np.float64).sum(1) - 1) <= k * 2 ** -24)
    # every selected logit >= every unselected one
    for t in range(T):
        mask = np.ones(E, bool)
        mask[ids[t]] = False
        if mask.any():
            assert logits[t, ids[t]].min() >= logits[t, mask].max()


def test_topk_all_equal_is_first_k_with_uniform_weights():
    logits = np.full((3, 16), -1.5, np.float32)
    ids, w = oracle.topk(logits, 4)
    np.testing.assert_array_equal(ids, np.tile(np.arange(4), (3, 1)))
    np.testing.assert_array_equal(w, np.full((3, 4), 0.25, np.float32))


def test_topk_k_equals_E_is_full_softmax():
    rng = np.random.default_rng(1)
    logits = rng.standard_normal((20, 8)).astype(np.float32)
    ids, w = oracle.topk(logits, 8)
    full = torch.softmax(torch.from_numpy(logits.astype(np.float64)), 1).numpy()
    np.testing.assert_allclose(w, np.take_along_axis(full, ids, 1), rtol=0, atol=2 ** -24)


def test_topk_k1_weight_is_one():
    rng = np.random.default_rng(2)
    logits = rng.standard_normal((30, 8)).astype(np.float32)
    ids, w = oracle.topk(logits, 1)
    np.testing.assert_array_equal(w, np.ones((30, 1), np.float32))
    np.testing.assert_array_equal(ids[:, 0], np.argmax(logits, 1))


# --------------------------------------------------------------------------
# permutation
# --------------------------------------------------------------------------
@pytest.mark.parametrize("T,E,k", [(64, 8, 2), (33, 256, 8), (1, 4, 4), (100, 1, 1), (17, 3, 2)])
def test_permute_is_stable_sort_by_expert(T, E, k):
    rng = np.random.default_rng(T * 7 + E)
    ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    if E > 2:  # skew: expert 1 in slot 0 for the first half (swapped in, no duplicates)
        for t in range(T // 2):
            row = list(ids[t])
            if 1 in row:
                i = row.index(1)
                row[0], row[i] = row[i], row[0]
            else:
                row[0] = 1
            ids[t] = row
    offsets, perm_token, perm_slot, inv_perm = oracle.permute(ids, E)
    flat = ids.reshape(-1)
    tok = np.repeat(np.arange(T), k)
    order = np.argsort(flat.astype(np.int64) * T + tok, kind="stable")  # library stable sort
    np.testing.assert_array_equal(perm_token, tok[order])
    np.testing.assert_array_equal(perm_slot, np.tile(np.arange(k), T)[order])
    counts = np.bincount(flat, minlength=E)
    np.testing.assert_array_equal(offsets, np.concatenate([[0], np.cumsum(counts)]))
    assert offsets[-1] == T * k and np.all(np.diff(offsets) >= 0)
    # bijection, and inv_perm inverts it
    assert sorted(inv_perm.reshape(-1).tolist()) == list(range(T * k))
    for t in range(T):
        for j in range(k):
            p = inv_perm[t, j]
            assert perm_token[p] == t and perm_slot[p] == j


# --------------------------------------------------------------------------
# experts + combine
# --------------------------------------------------------------------------
_TORCH_ACT = {
    oracle.ACT_SILU: torch.nn.functional.silu,
    oracle.ACT_GELU: lambda z: torch.nn.functional.gelu(z, approximate="none"),
    oracle.ACT_RELU: torch.nn.functional.relu,
}


def _dense_masked(cfg, L, ids, w, act=oracle.ACT_SILU):
    """Every expert on every token (fp64, logical weights), then masked by top-k."""
    wg, wu, wd = _logical_weights(cfg)
    x = mi.bf16_to_f32(L["x"]).astype(np.float64)
    out = np.zeros((cfg.T, cfg.H))
    for e in range(cfg.E):
        g = x @ wg[e]
        u = x @ wu[e]
        y = (_TORCH_ACT[act](torch.from_numpy(g)).numpy() * u) @ wd[e]
        for j in range(cfg.k):
            m = ids[:, j] == e
            out[m] += w[m, j:j + 1].astype(np.float64) * y[m]
    return out


@pytest.mark.parametrize("act", [oracle.ACT_SILU, oracle.ACT_GELU, oracle.ACT_RELU])
@pytest.mark.parametrize("name,kw", [("tiny", {}), ("tiny", dict(T=19, E=5, k=3, H=64, I=96,
                                                                   bias="normal"))])
def test_forward_matches_dense_masked_brute_force(name, kw, act):
    cfg = _small(name, **kw)
    L = mi.make_layer(cfg)
    r = oracle.moe_forward(L["x"], L["wr"], L["bias"], L["w13"], L["w2"], k=cfg.k, act=act)
    ref = _dense_masked(cfg, L, r["ids"], r["w"], act)
    np.testing.assert_allclose(r["out"], ref, rtol=1e-6, atol=1e-7 * np.abs(ref).max())


def test_one_hot_identical_experts_equal_one_dense_ffn():
    cfg = _small(T=24, E=4, k=1, H=64, I=128)
    L = mi.make_layer(cfg)
    w13 = np.repeat(L["w13"][:1], cfg.E, axis=0)
    w2 = np.repeat(L["w2"][:1], cfg.E, axis=0)
    r = oracle.moe_forward(L["x"], L["wr"], L["bias"], w13, w2, k=1)
    x = torch.from_numpy(mi.bf16_to_f32(L["x"]).astype(np.float64))
    W13 = torch.from_numpy(mi.bf16_to_f32(L["w13"][0]).astype(np.float64))
    W2 = torch.from_numpy(mi.bf16_to_f32(L["w2"][0]).astype(np.float64))
    g = torch.nn.functional.linear(x, W13[: cfg.I])
    u = torch.nn.functional.linear(x, W13[cfg.I:])
    ref = torch.nn.functional.linear(torch.nn.functional.silu(g) * u, W2).numpy()
    np.testing.assert_allclose(r["out"], ref, rtol=1e-6, atol=1e-7 * np.abs(ref).max())


def test_gated_activations_closed_forms():
    """One token x = e_0 and gate weights g_i on channel 0, up weights 1: the
    expert hidden row is act(g_i) exactly, against textbook values:
    silu(z) = z sigma(z), gelu(z) = z Phi(z) with Phi the normal CDF
    (Phi(1) = 0.8413447460685429, Phi(2) = 0.9772498680518208,
    Phi(-0.5) = 0.3085375387259869), relu(z) = max(z, 0)."""
    g = np.array([1.0, -1.0, 2.0, -0.5, 0.0], np.float32)
    I, H = len(g), 16
    a = np.zeros((1, H), np.float32)
    a[0, 0] = 1.0
    w13 = np.zeros((2 * I, H), np.float32)
    w13[:I, 0] = g
    w13[I:, 0] = 1.0
    A, W = _bf16(a), _bf16(w13)
    sig1 = 1.0 / (1.0 + np.exp(-1.0))
    want = {
        oracle.ACT_SILU: [sig1, -(1.0 - sig1), 2.0 / (1.0 + np.exp(-2.0)),
                          -0.5 / (1.0 + np.exp(0.5)), 0.0],
        oracle.ACT_GELU: [0.8413447460685429, -(1.0 - 0.8413447460685429), 2 * 0.9772498680518208,
                          -0.5 * 0.3085375387259869, 0.0],
        oracle.ACT_RELU: [1.0, 0.0, 2.0, 0.0, 0.0],
    }
    for act, ref in want.items():
        got = oracle.expert_gated_rows(A, W, act)[0]
        np.testing.assert_allclose(got, np.array(ref), rtol=1e-7, atol=1e-12, err_msg=str(act))
    # swapping gate and up halves changes the answer (the activation is on the gate)
    Wsw = np.concatenate([W[I:], W[:I]])
    assert not np.allclose(oracle.expert_gated_rows(A, Wsw, oracle.ACT_GELU)[0],
                           oracle.expert_gated_rows(A, W, oracle.ACT_GELU)[0])


def test_identical_experts_k2_equal_one_dense_ffn():
    cfg = _small(T=16, E=6, k=2, H=64, I=64, bias="normal")
    L = mi.make_layer(cfg)
    w13 = np.repeat(L["w13"][2:3], cfg.E, axis=0)
    w2 = np.repeat(L["w2"][2:3], cfg.E, axis=0)
    r = oracle.moe_forward(L["x"], L["wr"], L["bias"], w13, w2, k=2)
    one = oracle.moe_forward(L["x"], L["wr"], L["bias"], w13, w2, k=1)
    np.testing.assert_allclose(r["out"], one["out"], rtol=1e-6, atol=1e-7)


def test_stage_pieces_match_dense():
    cfg = _small(T=10, E=3, k=2, H=64, I=32)
    L = mi.make_layer(cfg)
    wg, wu, wd = _logical_weights(cfg)
    x = mi.bf16_to_f32(L["x"]).astype(np.float64)
    h = oracle.expert_swiglu_rows(L["x"], L["w13"][1])
    g, u = x @ wg[1], x @ wu[1]
    np.testing.assert_allclose(h, g / (1 + np.exp(-g)) * u, rtol=1e-6, atol=1e-9)
    hb = mi.f32_to_bf16(h)
    y = oracle.expert_down_rows(hb, L["w2"][1])
    np.testing.assert_allclose(y, mi.bf16_to_f32(hb).astype(np.float64) @ wd[1], rtol=1e-6,
                               atol=1e-9)


def test_subset_forward_equals_full_forward_rows():
    cfg = _small(T=48)
    L = mi.make_layer(cfg)
    full = oracle.moe_forward(L["x"], L["wr"], L["bias"], L["w13"], L["w2"], k=cfg.k)
    toks = np.array([0, 5, 47], np.int32)
    sub = oracle.moe_forward(L["x"], L["wr"], L["bias"], L["w13"], L["w2"], k=cfg.k, tokens=toks)
    np.testing.assert_array_equal(sub["out"], full["out"][toks])
    np.testing.assert_array_equal(sub["ids"], full["ids"][toks])


# --------------------------------------------------------------------------
# FP8 e4m3 codec and block quantisation
# --------------------------------------------------------------------------
def test_e4m3_decode_all_codes_match_torch():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mine = np.array([oracle.e4m3_decode(q) for q in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(mine), nan) and nan.sum() == 2
    np.testing.assert_array_equal(mine[~nan], ref[~nan])


def test_e4m3_encode_roundtrip_and_rne_vs_torch():
    for q in range(256):
        v = oracle.e4m3_decode(q)
        if not math.isnan(v):
            assert oracle.e4m3_encode(v) == q
    rng = np.random.default_rng(3)
    vals = np.concatenate([rng.standard_normal(4000) * s for s in (1e-3, 0.05, 1, 30, 200)])
    vals = np.clip(vals, -448, 448).astype(np.float32)
    # exact midpoints between neighbouring codes exercise ties-to-even
    finite = sorted({oracle.e4m3_decode(q) for q in range(128) if not math.isnan(oracle.e4m3_decode(q))})
    mids = np.array([(a + b) / 2 for a, b in zip(finite[:-1], finite[1:])], np.float32)
    vals = np.concatenate([vals, mids, -mids])
    ref = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    mine = np.array([oracle.e4m3_encode(v) for v in vals], np.uint8)
    np.testing.assert_array_equal(mine, ref)


def test_act_quant_bounds_and_closed_forms():
    cfg = _small(T=8, H=512)
    x = mi.make_x(cfg)
    x[3, 128:256] = 0  # an all-zero group
    q, s = oracle.quant_act_fp8(x)
    xf = mi.bf16_to_f32(x).astype(np.float64)
    dq = np.vectorize(oracle.e4m3_decode)(q) * np.repeat(s, 128, axis=1)
    assert s[3, 1] == 1.0 and np.all(q[3, 128:256] == 0)
    amax = np.abs(xf).reshape(8, 4, 128).max(2)
    nz = amax > 0
    np.testing.assert_array_equal(s[nz], (amax[nz].astype(np.float32) / np.float32(448)))
    # the element holding the group max encodes to +-448 (code 0x7E / 0xFE)
    for r in range(8):
        for g in range(4):
            if nz[r, g]:
                c = np.argmax(np.abs(xf[r, g * 128:(g + 1) * 128]))
                assert q[r, g * 128 + c] & 0x7F == 0x7E
    err = np.abs(dq - xf)
    sfull = np.repeat(s, 128, axis=1).astype(np.float64)
    assert np.all(err <= np.maximum(2.0 ** -4 * np.abs(xf), 2.0 ** -10 * sfull) * (1 + 1e-6))


def test_ue8m0_scales_closed_forms():
    """Power-of-two (UE8M0) scales: the smallest 2^p >= amax/448. Rows built so
    amax/448 is exactly 1 (scale 1), just above 1 (scale 2), exactly 1/2
    (scale 1/2) and 300/448 (scale 1); every scaled group max lands in
    (224, 448], and the scales are exact powers of two (e8m0 codes 127 + p)."""
    H = 128
    rows = np.zeros((5, H), np.float32)
    rows[0, 7] = 448.0
    rows[1, 9] = 450.0
    rows[2, 0] = -224.0
    rows[3, 100] = 300.0  # row 4 stays all zero: scale 1
    q, s = oracle.quant_act_fp8(_bf16(rows), ue8m0=True)
    np.testing.assert_array_equal(s[:, 0], np.array([1.0, 2.0, 0.5, 1.0, 1.0], np.float32))
    np.testing.assert_array_equal(oracle.e8m0_code(s[:, 0]), [127, 128, 126, 127, 127])
    assert q[0, 7] == 0x7E and q[2, 0] == 0xFE  # 448 and -448 after scaling
    assert q[1, 9] == oracle.e4m3_encode(225.0)  # 450 / 2
    x = mi.make_x(_small(T=16, H=512))
    q, s = oracle.quant_act_fp8(x, ue8m0=True)
    amax = np.abs(mi.bf16_to_f32(x)).reshape(16, 4, 128).max(2)
    ratio = amax / s
    assert np.all((ratio > 224) & (ratio <= 448))
    # same codes as the fp32-scale path would give for the scaled values
    sf = np.repeat(s, 128, axis=1)
    direct = np.vectorize(oracle.e4m3_encode)((mi.bf16_to_f32(x) / sf).astype(np.float32))
    np.testing.assert_array_equal(q, direct)


def test_ue8m0_weight_blocks_and_forward():
    cfg = _small(T=12, E=3, k=2, H=256, I=256)
    L = mi.make_layer(cfg)
    q13, s13 = oracle.quant_weight_fp8(L["w13"], ue8m0=True)
    q2, s2 = oracle.quant_weight_fp8(L["w2"], ue8m0=True)
    for s in (s13, s2):
        m, _ = np.frexp(s)
        assert np.all(m == 0.5)
    # the forward on power-of-two scales equals the dense layer on the dequantised values
    r = oracle.moe_forward(L["x"], L["wr"], L["bias"], k=cfg.k, fp8=(q13, s13, q2, s2), ue8m0=True)
    dec = np.vectorize(oracle.e4m3_decode)
    W13 = dec(q13) * np.repeat(np.repeat(s13, 128, 1), 128, 2)
    W2 = dec(q2) * np.repeat(np.repeat(s2, 128, 1), 128, 2)
    xq, xs = oracle.quant_act_fp8(L["x"], ue8m0=True)
    X = dec(xq) * np.repeat(xs, 128, 1)
    ref = np.zeros((cfg.T, cfg.H))
    for t in range(cfg.T):
        for j in range(cfg.k):
            e = r["ids"][t, j]
            g, u = W13[e, :cfg.I] @ X[t], W13[e, cfg.I:] @ X[t]
            h = (g / (1 + np.exp(-g)) * u).astype(np.float32)
            # h is re-quantised from fp32 (not bf16) per 128-group with a power-of-two scale
            amax = np.abs(h).reshape(-1, 128).max(1)
            sc = np.array([2.0 ** np.ceil(np.log2(np.float32(a) / np.float32(448))) if a > 0 else 1.0
                           for a in amax])
            hd = dec(np.vectorize(oracle.e4m3_encode)((h / np.repeat(sc, 128)).astype(np.float32)))
            ref[t] += r["w"][t, j] * (W2[e] @ (hd * np.repeat(sc, 128)))
    np.testing.assert_allclose(r["out"], ref, rtol=2e-5, atol=2e-5 * np.abs(ref).max())


def test_weight_quant_blocks():
    rng = np.random.default_rng(4)
    w = mi.f32_to_bf16(rng.standard_normal((2, 256, 384)).astype(np.float32) * 0.02)
    w[1, :128, 128:256] = 0
    q, s = oracle.quant_weight_fp8(w.reshape(2, 256, 384))
    assert s.shape == (2, 2, 3) and s[1, 0, 1] == 1.0
    wf = mi.bf16_to_f32(w).astype(np.float64)
    for b in range(2):
        for rb in range(2):
            for cb in range(3):
                blk = wf[b, rb * 128:(rb + 1) * 128, cb * 128:(cb + 1) * 128]
                amax = np.abs(blk).max()
                if amax > 0:
                    assert s[b, rb, cb] == np.float32(amax) / np.float32(448)
                dq = np.vectorize(oracle.e4m3_decode)(
                    q[b, rb * 128:(rb + 1) * 128, cb * 128:(cb + 1) * 128]) * s[b, rb, cb]
                assert np.all(np.abs(dq - blk) <= np.maximum(2.0 ** -4 * np.abs(blk),
                                                              2.0 ** -10 * s[b, rb, cb]) * (1 + 1e-6))


def test_fp8_forward_matches_dense_on_dequantised_values():
    cfg = _small(T=12, E=3, k=2, H=256, I=256)
    L = mi.make_layer(cfg)
    w13q, w13s = oracle.quant_weight_fp8(L["w13"])
    w2q, w2s = oracle.quant_weight_fp8(L["w2"])
    r = oracle.moe_forward(L["x"], L["wr"], L["bias"], k=2, fp8=(w13q, w13s, w2q, w2s))
    dec = np.vectorize(oracle.e4m3_decode)
    W13 = dec(w13q) * np.repeat(np.repeat(w13s, 128, 1), 128, 2)
    W2 = dec(w2q) * np.repeat(np.repeat(w2s, 128, 1), 128, 2)
    xq, xs = oracle.quant_act_fp8(L["x"])
    X = dec(xq) * np.repeat(xs, 128, 1)
    out = np.zeros((cfg.T, cfg.H))
    for t in range(cfg.T):
        for j in range(2):
            e = r["ids"][t, j]
            g = W13[e, :cfg.I] @ X[t]
            u = W13[e, cfg.I:] @ X[t]
            a = (g / (1 + np.exp(-g)) * u).astype(np.float32)
            # quantise a (fp32) per 128 group exactly as the layer states
            ah = np.empty(cfg.I)
            for g0 in range(0, cfg.I, 128):
                grp = a[g0:g0 + 128]
                sc = np.float32(np.abs(grp).max()) / np.float32(448) if np.abs(grp).max() > 0 else 1.0
                codes = torch.from_numpy((grp / np.float32(sc)).astype(np.float32)).to(
                    torch.float8_e4m3fn).to(torch.float64).numpy()
                ah[g0:g0 + 128] = codes * float(sc)
            out[t] += float(r["w"][t, j]) * (W2[e] @ ah)
    np.testing.assert_allclose(r["out"], out, rtol=1e-5, atol=1e-6 * np.abs(out).max())


# --------------------------------------------------------------------------
# FP4 e2m1 experts with e8m0 scales per (row, 32 elements)
# --------------------------------------------------------------------------
def _ml_dtypes():
    return pytest.importorskip("ml_dtypes")


def test_e2m1_decode_all_codes_match_ml_dtypes():
    md = _ml_dtypes()
    ref = np.arange(16, dtype=np.uint8).view(md.float4_e2m1fn).astype(np.float64)
    got = np.array([oracle.e2m1_decode(q) for q in range(16)])
    np.testing.assert_array_equal(got, ref)
    np.testing.assert_array_equal(np.signbit(got), np.signbit(ref))


def test_e2m1_encode_rne_vs_ml_dtypes():
    """Every grid point, every midpoint (ties to the even code), points just
    beside the midpoints and random values in [-6, 6]."""
    md = _ml_dtypes()
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], dtype=np.float64)
    mids = ((grid[1:] + grid[:-1]) / 2).astype(np.float32)
    pts = np.concatenate([grid.astype(np.float32), mids, np.nextafter(mids, np.float32(0)),
                          np.nextafter(mids, np.float32(10))])
    rng = np.random.default_rng(11)
    pts = np.concatenate([pts, -pts, rng.uniform(-6, 6, 4000).astype(np.float32)])
    ref = pts.astype(md.float4_e2m1fn).view(np.uint8) & 15
    got = np.array([oracle.e2m1_encode(v) for v in pts], dtype=np.uint8)
    nz = (pts != 0) & (np.abs(pts) > 0.25)  # results of +-0 carry the input's sign, checked below
    np.testing.assert_array_equal(got[nz], ref[nz])
    assert oracle.e2m1_encode(0.2) == 0 and oracle.e2m1_encode(-0.2) == 8
    assert oracle.e2m1_encode(5.0) == 6 and oracle.e2m1_encode(0.25) == 0  # ties -> even code
    assert oracle.e2m1_encode(1.75) == 4 and oracle.e2m1_encode(2.5) == 4


def _unpack_fp4(q, sc):
    """Dense fp64 values of packed e2m1 codes with e8m0 scales per (row, 32),
    decoded by ml_dtypes."""
    md = _ml_dtypes()
    codes = np.stack([q & 15, q >> 4], axis=-1).reshape(*q.shape[:-1], 2 * q.shape[-1])
    vals = codes.astype(np.uint8).view(md.float4_e2m1fn).astype(np.float64)
    scale = sc.astype(np.uint8).view(md.float8_e8m0fnu).astype(np.float64)
    return vals * np.repeat(scale, 32, axis=-1)


def test_fp4_weight_quant_closed_forms():
    """Block scale = smallest power of two >= amax/6, one per (row, 32);
    element 2i in the low nibble of byte i; an all-zero block has scale 1."""
    rng = np.random.default_rng(5)
    w = (rng.standard_normal((1, 2, 128)) * 0.01).astype(np.float32)
    w[0, 0, 3] = 6 * 2.0 ** -5          # block 0: amax / 6 is exactly 2^-5
    w[0, 0, :3] = w[0, 0, 4:32] = 0.01
    w[0, 0, 32:64] = 0                  # block 1: all zero
    w[0, 0, 64:96] = np.clip(w[0, 0, 64:96], -0.09, 0.09)
    w[0, 0, 70] = -0.1                  # block 2: bf16(0.1) / 6 rounds up to 2^-5
    wb16 = _bf16(w)
    q, sc = oracle.quant_weight_fp4(wb16)
    assert q.shape == (1, 2, 64) and sc.shape == (1, 2, 4)
    assert sc[0, 0, 0] == 127 - 5 and sc[0, 0, 1] == 127 and sc[0, 0, 2] == 127 - 5
    assert q[0, 0, 1] >> 4 == 7                   # element 3: +6 in the high nibble of byte 1
    assert q[0, 0, 0] == (1 | (1 << 4))           # 0.01 / 2^-5 = 0.32 -> 0.5 (code 1), twice
    assert np.all(q[0, 0, 16:32] == 0)
    assert (q[0, 0, 35] & 15) == 8 | 5            # element 70: -0.1001 / 2^-5 = -3.2 -> -3
    wf = mi.bf16_to_f32(wb16).astype(np.float64)
    deq = _unpack_fp4(q, sc)
    s = np.repeat(2.0 ** (sc.astype(np.float64) - 127), 32, axis=-1)
    assert np.all(np.abs(wf) <= 6 * s)
    err = np.abs(deq - wf)
    assert np.all(err <= s * (1 + 1e-12))                               # largest gap (4..6) / 2
    small = np.abs(wf) <= 2 * s
    assert np.all(err[small] <= 0.25 * s[small] * (1 + 1e-12))           # gap 0.5 below 2


def _pow2_quant_e4m3(v):
    """Per 128-group: scale = smallest power of two >= amax/448 (fp32), e4m3 by torch."""
    v = np.asarray(v, dtype=np.float32).reshape(-1, 128)
    out = np.empty(v.shape)
    for i, grp in enumerate(v):
        amax = np.float32(np.abs(grp).max())
        sc = 2.0 ** np.ceil(np.log2(np.float32(amax / np.float32(448)))) if amax > 0 else 1.0
        codes = torch.from_numpy((grp / np.float32(sc)).astype(np.float32)).to(torch.float8_e4m3fn)
        out[i] = codes.to(torch.float64).numpy() * sc
    return out.reshape(-1)


def test_fp4_forward_matches_dense_on_dequantised_values():
    cfg = _small(T=12, E=3, k=2, H=256, I=256)
    L = mi.make_layer(cfg)
    q13, s13 = oracle.quant_weight_fp4(L["w13"])
    q2, s2 = oracle.quant_weight_fp4(L["w2"])
    r = oracle.moe_forward(L["x"], L["wr"], L["bias"], k=cfg.k, fp4=(q13, s13, q2, s2))
    W13, W2 = _unpack_fp4(q13, s13), _unpack_fp4(q2, s2)
    xf = mi.bf16_to_f32(L["x"])
    ref = np.zeros((cfg.T, cfg.H))
    for t in range(cfg.T):
        X = _pow2_quant_e4m3(xf[t])
        for j in range(cfg.k):
            e = r["ids"][t, j]
            g, u = W13[e, :cfg.I] @ X, W13[e, cfg.I:] @ X
            h = (g / (1 + np.exp(-g)) * u).astype(np.float32)
            ref[t] += float(r["w"][t, j]) * (W2[e] @ _pow2_quant_e4m3(h))
    np.testing.assert_allclose(r["out"], ref, rtol=2e-5, atol=2e-5 * np.abs(ref).max())


def test_fp4_forward_on_fp4_exact_weights_equals_ue8m0_fp8_forward():
    """Weights already on the e2m1 grid (times 2^-7) quantise without error in
    both formats, so the FP4 layer must equal the power-of-two FP8 layer."""
    cfg = _small(T=20, E=4, k=2, H=256, I=384)
    L = mi.make_layer(cfg)
    rng = np.random.default_rng(9)
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6, -0.5, -1, -1.5, -2, -3, -4, -6])
    w13 = _bf16(rng.choice(grid, size=L["w13"].shape) * 2.0 ** -7)
    w2 = _bf16(rng.choice(grid, size=L["w2"].shape) * 2.0 ** -7)
    q13, s13 = oracle.quant_weight_fp4(w13)
    q2, s2 = oracle.quant_weight_fp4(w2)
    np.testing.assert_array_equal(_unpack_fp4(q13, s13), mi.bf16_to_f32(w13))
    f8 = oracle.quant_weight_fp8(w13, ue8m0=True) + oracle.quant_weight_fp8(w2, ue8m0=True)
    r4 = oracle.moe_forward(L["x"], L["wr"], L["bias"], k=cfg.k, fp4=(q13, s13, q2, s2))
    r8 = oracle.moe_forward(L["x"], L["wr"], L["bias"], k=cfg.k, fp8=f8, ue8m0=True)
    np.testing.assert_array_equal(r4["ids"], r8["ids"])
    np.testing.assert_array_equal(r4["out"], r8["out"])


# --------------------------------------------------------------------------
# the input generator itself
# --------------------------------------------------------------------------
def test_generator_splitmix_reference_value():
    # SplitMix64 (Steele, Lea & Flood 2014) seeded with 0: first output
    assert mi.splitmix64(0) == 0xE220A8397B1DCDAF


def test_generator_streams_of_different_seeds_are_unrelated():
    a = mi.normal_bf16(0, mi.TAG_X, 1.0, 1, 64, 128)
    b = mi.normal_bf16(1, mi.TAG_X, 1.0, 1, 64, 128)
    assert np.sort(a).tolist() != np.sort(b).tolist()


def test_generator_transposed_store_draws_same_values():
    cfg = _small(E=3, H=64, I=32)
    L = mi.make_layer(cfg)
    wg, wu, wd = _logical_weights(cfg)
    np.testing.assert_array_equal(mi.bf16_to_f32(L["w13"][:, :cfg.I, :]), wg.transpose(0, 2, 1))
    np.testing.assert_array_equal(mi.bf16_to_f32(L["w13"][:, cfg.I:, :]), wu.transpose(0, 2, 1))
    np.testing.assert_array_equal(mi.bf16_to_f32(L["w2"]), wd.transpose(0, 2, 1))


def test_generator_moments():
    v = mi.bf16_to_f32(mi.normal_bf16(0, 99, 0.02, 1, 1000, 1000)).astype(np.float64)
    assert abs(v.mean()) < 1e-4 and abs(v.std() - 0.02) < 2e-4
    z = v / 0.02
    assert 0.040 < np.mean(np.abs(z) > 2) < 0.051  # two-sided normal tail 4.55 %


def test_zipf_bias_is_log_pmf_of_a_rank_permutation():
    cfg = mi.CONFIGS["fine_grained"]
    _, b = mi.make_router(cfg.with_(H=8))
    sigma_l = 1.0 * 0.02 * np.sqrt(8)  # x ~ N(0,1), Wr ~ N(0,0.02): the logits' spread
    ranks = np.exp(-b.astype(np.float64) / (1.1 * sigma_l))
    np.testing.assert_allclose(np.sort(ranks), np.arange(1, 257), rtol=1e-5)


def test_fine_grained_workload_is_skewed_with_empty_experts():
    # The fine-grained workload promises Zipf-skewed expert loads "including some empty
    # experts": route the full-size seed-0 batch with the oracle and check both properties.
    cfg = mi.CONFIGS["fine_grained"]
    wr, b = mi.make_router(cfg)
    ids, _ = oracle.topk(oracle.router_logits(mi.make_x(cfg), wr, b), cfg.k)
    counts = np.bincount(ids.ravel(), minlength=cfg.E)
    assert counts.sum() == cfg.T * cfg.k
    assert np.sum(counts == 0) >= 1
    assert counts.max() > 8 * counts.mean()
