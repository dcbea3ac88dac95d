"""The C ABI library on the CPU: it loads, exports every symbol include/moe.h
declares, and its host-side validation rejects bad calls before any launch.
No GPU is touched (pointers below are never dereferenced: every call fails
validation or the device check first)."""
import ctypes
import os
import re

import pytest

import mixture_experts_layer_tcgen05_b200 as moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FAKE = 0x7F0000001000  # 16-byte aligned address, never dereferenced


def _declared():
    text = open(os.path.join(ROOT, "include", "moe.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    L = moe.lib()
    names = _declared()
    assert len(names) >= 18
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(moe.EXPORTED)
    assert moe.moe_abi_version() == 1


def test_workspace_size_and_layout():
    d = (64, 128, 256, 8, 2)
    n = moe.moe_workspace_size(d, moe.MOE_DTYPE_BF16)
    L = moe.moe_workspace_layout(d, moe.MOE_DTYPE_BF16)
    assert n == L.total > 0
    R, H, I = 128, 128, 256
    assert L.y_perm >= L.h + R * I * 2 and L.h >= L.x_perm + R * H * 2
    for f in ("logits", "topk_ids", "topk_w", "offsets", "perm_token", "inv_perm", "x_perm", "h",
              "y_perm"):
        assert getattr(L, f) % 256 == 0
    L8 = moe.moe_workspace_layout(d, moe.MOE_DTYPE_FP8_E4M3)
    assert L8.x_perm == -1 and L8.h == -1 and L8.xq_perm > 0 and L8.hs > 0
    assert moe.moe_workspace_size((64, 100, 256, 8, 2), moe.MOE_DTYPE_BF16) == 0


@pytest.mark.parametrize("d,msg", [
    ((0, 128, 256, 8, 2), "T must be"),
    ((4, 100, 256, 8, 2), "H must be"),
    ((4, 128, 200, 8, 2), "I must be"),
    ((4, 128, 256, 2000, 2), "E must be"),
    ((4, 128, 256, 8, 9), "k must be"),
    ((4, 128, 256, 8, 17), "k must be"),
])
def test_forward_rejects_bad_dims(d, msg):
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_forward(FAKE, FAKE, None, FAKE, FAKE, d, FAKE, FAKE, 1 << 30, stream=0)
    assert ei.value.status == moe.MOE_ERR_INVALID_ARG and msg in str(ei.value)


def test_forward_rejects_null_and_misaligned_pointers():
    d = (4, 128, 256, 8, 2)
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_forward(None, FAKE, None, FAKE, FAKE, d, FAKE, FAKE, 1 << 30, stream=0)
    assert ei.value.status == moe.MOE_ERR_INVALID_ARG and "x is NULL" in str(ei.value)
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_forward(FAKE + 2, FAKE, None, FAKE, FAKE, d, FAKE, FAKE, 1 << 30, stream=0)
    assert "aligned" in str(ei.value)


def test_forward_rejects_small_workspace():
    d = (4, 128, 256, 8, 2)
    need = moe.moe_workspace_size(d)
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_forward(FAKE, FAKE, None, FAKE, FAKE, d, FAKE, FAKE, need - 1, stream=0)
    assert ei.value.status == moe.MOE_ERR_WORKSPACE


def test_wrong_architecture_is_refused(monkeypatch):
    monkeypatch.setenv("MOE_FAKE_CC", "90")
    d = (4, 128, 256, 8, 2)
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_forward(FAKE, FAKE, None, FAKE, FAKE, d, FAKE, FAKE, 1 << 30, stream=0)
    assert ei.value.status == moe.MOE_ERR_UNSUPPORTED_DEVICE and "9.0" in str(ei.value)


def test_grouped_gemm_validation():
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_grouped_gemm(FAKE, FAKE, FAKE, 10, 4, 100, 128, moe.MOE_DTYPE_BF16,
                             moe.MOE_EPILOGUE_NONE, FAKE, ws=FAKE, ws_bytes=4096, stream=0)
    assert ei.value.status == moe.MOE_ERR_INVALID_ARG
    with pytest.raises(moe.MoeError) as ei:  # FP8 needs scales
        moe.moe_grouped_gemm(FAKE, FAKE, FAKE, 10, 4, 128, 128, moe.MOE_DTYPE_FP8_E4M3,
                             moe.MOE_EPILOGUE_NONE, FAKE, ws=FAKE, ws_bytes=4096, stream=0)
    assert "a_scales" in str(ei.value)


def test_permute_requires_x_and_x_perm_together():
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_permute(FAKE, (4, 128, 256, 8, 2), FAKE, FAKE, FAKE, FAKE, None, FAKE, 1 << 30,
                        stream=0)
    assert "both" in str(ei.value)


def test_stage_events_need_six():
    with pytest.raises(moe.MoeError):
        moe.moe_set_stage_events([1, 2, 3])
    moe.moe_set_stage_events(None)


def test_last_error_is_thread_local_and_cleared():
    moe.moe_set_stage_events(None)
    assert moe.moe_last_error() == ""


def test_fp4_entry_points_validate_before_launch():
    d = (16, 256, 256, 4, 2)
    assert moe.moe_workspace_size(d, moe.MOE_DTYPE_FP4_E2M1) == \
        moe.moe_workspace_size(d, moe.MOE_DTYPE_FP8_E4M3_UE8M0) > 0
    swi = moe.MOE_EPILOGUE_SWIGLU
    with pytest.raises(moe.MoeError) as ei:  # packed weights must be 32-byte aligned (TMA 4-bit map)
        moe.moe_forward_fp4(FAKE, FAKE, None, FAKE + 16, FAKE, FAKE, FAKE, d, swi, FAKE, FAKE,
                            1 << 30, stream=0)
    assert ei.value.status == moe.MOE_ERR_INVALID_ARG and "32-byte" in str(ei.value)
    with pytest.raises(moe.MoeError) as ei:  # scale chunks are bulk-copied: 16-byte aligned
        moe.moe_forward_fp4(FAKE, FAKE, None, FAKE, FAKE + 4, FAKE, FAKE, d, swi, FAKE, FAKE,
                            1 << 30, stream=0)
    assert ei.value.status == moe.MOE_ERR_INVALID_ARG and "w13s" in str(ei.value)
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_forward_fp4(FAKE, FAKE, None, FAKE, FAKE, FAKE, FAKE, d, moe.MOE_EPILOGUE_NONE,
                            FAKE, FAKE, 1 << 30, stream=0)
    assert ei.value.status == moe.MOE_ERR_INVALID_ARG
    with pytest.raises(moe.MoeError) as ei:  # the plain FP4 GEMM tiles N by 256
        moe.moe_grouped_gemm_fp4(FAKE, FAKE, FAKE, FAKE, FAKE, 10, 4, 384, 128,
                                 moe.MOE_EPILOGUE_NONE, FAKE, None, FAKE, 4096, stream=0)
    assert "256" in str(ei.value)
    with pytest.raises(moe.MoeError) as ei:  # FP4 B scales are bytes: the generic entry refuses
        moe.moe_grouped_gemm(FAKE, FAKE, FAKE, 10, 4, 256, 128, moe.MOE_DTYPE_FP4_E2M1,
                             moe.MOE_EPILOGUE_NONE, FAKE, FAKE, FAKE, ws=FAKE, ws_bytes=4096,
                             stream=0)
    assert "moe_grouped_gemm_fp4" in str(ei.value)
    with pytest.raises(moe.MoeError) as ei:  # scale chunks cover 128 rows
        moe.moe_quantize_weight_fp4(FAKE, 1, 100, 256, FAKE, FAKE, stream=0)
    assert ei.value.status == moe.MOE_ERR_INVALID_ARG


def test_product_path_never_reaches_the_oracle():
    """The package (binding, expert-parallel layer, CUDA sources, build script)
    neither imports the CPU oracle nor links or loads its C library: every step
    of the layer runs in the CUDA kernels, with no CPU fallback."""
    pkg = os.path.join(ROOT, "mixture_experts_layer_tcgen05_b200")
    seen = 0
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if not f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                continue
            src = open(os.path.join(dirpath, f)).read()
            seen += 1
            assert not re.search(r"^\s*(import|from)\s+oracle\b", src, re.M), f
            assert "moe_oracle" not in src and "liboracle" not in src, f
    assert seen > 5


def test_binding_fails_loudly_without_the_library(tmp_path, monkeypatch):
    """With the shared library absent the binding raises instead of computing
    anything another way."""
    import importlib.util
    src = os.path.join(ROOT, "mixture_experts_layer_tcgen05_b200", "__init__.py")
    fake_pkg = tmp_path / "mixture_experts_layer_tcgen05_b200"
    fake_pkg.mkdir()
    (fake_pkg / "__init__.py").write_text(open(src).read())
    spec = importlib.util.spec_from_file_location("moe_nolib", fake_pkg / "__init__.py")
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    with pytest.raises(ImportError, match="missing"):
        mod.lib()


@pytest.mark.parametrize("dtype,shape", [("bfloat16", (3, 5)), ("float32", (7,)), ("uint8", (2, 3, 4)),
                                         ("int32", (1, 9))])
def test_guarded_buffer_detects_writes_past_either_end(dtype, shape):
    """The GPU tests' canary buffers, checked here on CPU tensors."""
    import torch
    from helpers import GUARD_BYTES, Guarded
    dt = getattr(torch, dtype)
    g = Guarded(shape, dt, device="cpu", fill=0)
    assert g.t.shape == shape and g.t.dtype == dt and g.t.is_contiguous()
    assert g.t.data_ptr() - g.buf.data_ptr() == GUARD_BYTES
    assert g.t.data_ptr() % 256 == g.buf.data_ptr() % 256  # alignment carried over
    assert bool((g.t.view(torch.uint8) == 0).all()) and g.intact()
    g.t.view(torch.uint8).fill_(0x3C)  # writes inside the view leave the guards alone
    assert g.intact()
    g.buf[GUARD_BYTES - 1] = 0
    assert not g.intact()
    g2 = Guarded(shape, dt, device="cpu")
    g2.buf[GUARD_BYTES + g2.n] = 0
    assert not g2.intact()


def test_every_device_wait_is_bounded():
    """The kernels wait only through ptx::mbar_wait, which gives up after a
    clock64 budget (or as soon as another thread has recorded a failure) and
    records the site in the status word; there is no other spin loop, and no
    trap or device assert anywhere in the CUDA sources."""
    csrc = os.path.join(ROOT, "mixture_experts_layer_tcgen05_b200", "csrc")
    files = sorted(f for f in os.listdir(csrc) if f.endswith((".cu", ".cuh")))
    assert "ptx.cuh" in files and len(files) > 5
    for f in files:
        src = open(os.path.join(csrc, f)).read()
        code = re.sub(r"//[^\n]*|/\*.*?\*/", "", src, flags=re.S)
        if f != "ptx.cuh":
            assert "mbarrier.try_wait" not in code and "mbar_try_wait" not in code, f
        assert not re.search(r"while\s*\(\s*(1|true)\s*\)|for\s*\(\s*;\s*;\s*\)", code), f
        assert "__trap" not in code and not re.search(r"\btrap\s*;", code), f
        assert not re.search(r"\bassert\s*\(", code), f
    ptx = open(os.path.join(csrc, "ptx.cuh")).read()
    body = ptx[ptx.index("bool mbar_wait("):]
    body = body[:body.index("\n}\n")]
    for needed in ("clock64()", "budget", "record_timeout", "return false"):
        assert needed in body, needed


@pytest.mark.parametrize("dt", ["MOE_DTYPE_BF16", "MOE_DTYPE_FP8_E4M3", "MOE_DTYPE_FP8_E4M3_UE8M0",
                                "MOE_DTYPE_FP4_E2M1"])
def test_workspace_layout_at_the_largest_accepted_dims(dt):
    """Sizes far past 2^32 bytes: the layout arithmetic is 64-bit, every region
    is 256-byte aligned, no two regions overlap at their nominal sizes, and the
    total covers them all. T = 2^27 - 1 with k = 16 is just under the 2^31
    routed-row limit of the dims check."""
    dtype = getattr(moe, dt)
    T, H, I, E, k = (1 << 27) - 1, 7168, 2048, 1024, 16
    R = T * k
    L = moe.moe_workspace_layout((T, H, I, E, k), dtype)
    assert L.total == moe.moe_workspace_size((T, H, I, E, k), dtype) > R * H
    q = dtype != moe.MOE_DTYPE_BF16
    size = {"logits": T * E * 4, "topk_ids": R * 4, "topk_w": R * 4, "offsets": (E + 1) * 4,
            "perm_token": R * 4, "inv_perm": R * 4, "y_perm": R * H * 2}
    if q:
        size.update(xq=T * H, xs=T * (H // 128) * 4, xq_perm=R * H, xs_perm=R * (H // 128) * 4,
                    hq=R * I, hs=R * (I // 128) * 4)
    else:
        size.update(x_perm=R * H * 2, h=R * I * 2)
    regions = sorted((getattr(L, f), getattr(L, f) + n, f) for f, n in size.items())
    for lo, hi, f in regions:
        assert lo % 256 == 0, f
    for (lo0, hi0, f0), (lo1, hi1, f1) in zip(regions, regions[1:]):
        assert hi0 <= lo1, (f0, f1)  # no two regions overlap
    assert regions[-1][1] <= L.total


def _noalloc_scratch(T, E):
    # the permutation's scratch: chunk masks and chunk bases (ceil(T/32) x E words each, each
    # part rounded up to 256 bytes) and E counts (rounded up to 256)
    def up(n):
        return (n + 255) // 256 * 256
    c = (T + 31) // 32
    return 2 * up(c * E * 4) + up(E * 4)


@pytest.mark.parametrize("E", [256, 8])
def test_noalloc_rejects_exactly_past_its_fixed_array(E, monkeypatch):
    """The size check runs before the device check: the largest accepted T gets as far as
    the (faked, refused) device check; one token more is rejected as too large. The
    array's first 256 bytes are its status word."""
    monkeypatch.setenv("MOE_FAKE_CC", "90")
    cap = 1048576 - 256
    T = max(t for t in range(1, 600000) if _noalloc_scratch(t, E) <= cap) if E == 8 else \
        max(t for t in range(1, 20000) if _noalloc_scratch(t, E) <= cap)
    assert T == {256: 16352, 8: 524032}[E]  # the bounds include/moe.h states
    k = 2
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_permute_noalloc(FAKE, (T, 128, 128, E, k), FAKE, FAKE, FAKE, stream=0)
    assert ei.value.status == moe.MOE_ERR_UNSUPPORTED_DEVICE
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_permute_noalloc(FAKE, (T + 1, 128, 128, E, k), FAKE, FAKE, FAKE, stream=0)
    assert ei.value.status == moe.MOE_ERR_INVALID_ARG and "scratch" in str(ei.value)


def test_noalloc_status_validates():
    assert moe.lib().moe_permute_noalloc_status(None, 0) == moe.MOE_ERR_INVALID_ARG
    assert "NULL" in moe.moe_last_error()


def test_pack_weights_validates_before_launch(monkeypatch):
    monkeypatch.setenv("MOE_FAKE_CC", "90")
    E, H, I = 4, 256, 384
    n = E * H * I * 2
    wg, wu, wd = FAKE, FAKE + n, FAKE + 2 * n
    w13, w2 = FAKE + 3 * n, FAKE + 5 * n
    for bad, msg in [((0, H, I), "E must"), ((E, 100, I), "H must"), ((E, H, 64), "I must")]:
        with pytest.raises(moe.MoeError) as ei:
            moe.moe_pack_weights(wg, wu, wd, *bad, w13, w2, stream=0)
        assert ei.value.status == moe.MOE_ERR_INVALID_ARG and msg in str(ei.value)
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_pack_weights(None, wu, wd, E, H, I, w13, w2, stream=0)
    assert "wg is NULL" in str(ei.value)
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_pack_weights(wg, wu, wd + 8, E, H, I, w13, w2, stream=0)
    assert "aligned" in str(ei.value)
    with pytest.raises(moe.MoeError) as ei:  # w13 spans 2n bytes: it would run into w2 at 4n
        moe.moe_pack_weights(wg, wu, wd, E, H, I, FAKE + 3 * n, FAKE + 4 * n, stream=0)
    assert "overlap" in str(ei.value)
    with pytest.raises(moe.MoeError) as ei:  # output written over an input
        moe.moe_pack_weights(wg, wu, wd, E, H, I, FAKE + n, w2, stream=0)
    assert "overlap" in str(ei.value)
    with pytest.raises(moe.MoeError) as ei:  # valid: gets as far as the device check
        moe.moe_pack_weights(wg, wu, wd, E, H, I, w13, w2, stream=0)
    assert ei.value.status == moe.MOE_ERR_UNSUPPORTED_DEVICE


def test_expert_parallel_exchange_validates_before_launch(monkeypatch):
    monkeypatch.setenv("MOE_FAKE_CC", "90")
    assert moe.moe_ep_plan_bytes(12, 3) == 4 * (8 + 12 + 13 + 12)  # loc_off padded to 4 ints
    for E, G in [(10, 3), (0, 1), (2048, 2), (64, 0), (64, 65)]:
        assert moe.moe_ep_plan_bytes(E, G) == 0
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_ep_plan(FAKE, 3, 3, 12, FAKE, stream=0)  # rank outside [0, G)
    assert ei.value.status == moe.MOE_ERR_INVALID_ARG and "rank" in str(ei.value)
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_ep_dispatch(FAKE, FAKE, FAKE, 12, 3, 10, 100, FAKE, 64, stream=0)
    assert ei.value.status == moe.MOE_ERR_INVALID_ARG and "row_bytes" in str(ei.value)
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_ep_return(FAKE, FAKE, 12, 3, 64, 256, None, 64, stream=0)
    assert "src_bufs is NULL" in str(ei.value)
    with pytest.raises(moe.MoeError) as ei:  # valid: as far as the device check
        moe.moe_ep_dispatch(FAKE, FAKE, FAKE, 12, 3, 10, 256, FAKE, 64, stream=0)
    assert ei.value.status == moe.MOE_ERR_UNSUPPORTED_DEVICE
