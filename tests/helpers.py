"""Shared test helpers: device transfer of raw bf16 bits, the output tolerance
check, and cached full-size layer inputs."""
from __future__ import annotations

import functools

import numpy as np

import moe_inputs as mi

# Output tolerance for bf16 inputs with fp32 accumulation (the layer's stated bar):
#   max |out - ref| <= 2e-2 * max |ref|   and   sum |out - ref| / sum |ref| <= 5e-3
BF16_TOL = (2e-2, 5e-3)
# FP8 path, against the oracle run on the dequantised values
FP8_TOL = (6e-2, 2e-2)


def check_close(out, ref, tol=BF16_TOL, what="output"):
    out = np.asarray(out, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert out.shape == ref.shape, (out.shape, ref.shape)
    assert np.all(np.isfinite(out)), f"{what}: non-finite values"
    err = np.abs(out - ref)
    max_rel = err.max() / max(np.abs(ref).max(), 1e-30)
    l1_rel = err.sum() / max(np.abs(ref).sum(), 1e-30)
    assert max_rel <= tol[0] and l1_rel <= tol[1], (
        f"{what}: max|err|/max|ref| = {max_rel:.3e} (<= {tol[0]}), "
        f"sum|err|/sum|ref| = {l1_rel:.3e} (<= {tol[1]})")
    return max_rel, l1_rel


def quant_pow2_e4m3(h):
    """Per row, per 128 group: s = smallest power of two >= amax/448 (fp32),
    q = e4m3(h/s) by torch's cast. Returns (codes uint8, scales fp32)."""
    import torch
    rows, cols = h.shape
    g = h.reshape(rows, cols // 128, 128)
    amax = np.abs(g).max(2).astype(np.float32)
    m, e = np.frexp(amax / np.float32(448))
    s = np.where(amax > 0, np.ldexp(np.float32(1), np.where(m == 0.5, e - 1, e)), 1.0).astype(np.float32)
    q = torch.from_numpy((g / s[:, :, None]).astype(np.float32).reshape(rows, cols)).to(
        torch.float8_e4m3fn).view(torch.uint8).numpy()
    return q, s


def dev_bf16(a: np.ndarray):
    import torch
    a = np.ascontiguousarray(a, dtype=np.uint16)
    return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()


def host_bf16(t) -> np.ndarray:
    import torch
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def dev(a: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def dev_u8(a: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).cuda()


@functools.lru_cache(maxsize=2)
def layer_host(name: str, **over) -> tuple:
    cfg = mi.CONFIGS[name].with_(**over) if over else mi.CONFIGS[name]
    return cfg, mi.make_layer(cfg)


def dims(cfg):
    return (cfg.T, cfg.H, cfg.I, cfg.E, cfg.k)


# Canary bytes on both sides of a buffer: with no sanitizer on the GPU, a
# kernel that writes past either end of its output or workspace shows up as
# a changed guard byte.
GUARD_BYTES = 4096
GUARD_FILL = 0xA5


class Guarded:
    """`t` is a `shape`/`dtype` view starting GUARD_BYTES into a byte buffer
    whose guard bytes hold GUARD_FILL; `intact()` checks both guards. `fill`
    sets every byte of the view (e.g. 0 for a workspace)."""

    def __init__(self, shape, dtype, device="cuda", fill=None):
        import torch
        self.n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        self.buf = torch.full((2 * GUARD_BYTES + self.n,), GUARD_FILL, dtype=torch.uint8,
                              device=device)
        inner = self.buf[GUARD_BYTES:GUARD_BYTES + self.n]
        if fill is not None:
            inner.fill_(fill)
        self.t = inner.view(dtype).view(tuple(shape))

    def intact(self) -> bool:
        lo, hi = self.buf[:GUARD_BYTES], self.buf[GUARD_BYTES + self.n:]
        return bool((lo == GUARD_FILL).all().item()) and bool((hi == GUARD_FILL).all().item())
