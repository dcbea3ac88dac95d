"""CPU oracle for the sparse MoE FFN layer forward (ctypes wrapper of moe_oracle.c).

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s ``cpu_baseline`` leg (and its ``--impl reference`` arm) may
import this package. The product path (``mixture_experts_layer_tcgen05_b200``)
never imports it and shares no code with it.

What it computes, and the passages each step follows, are documented beside
each C function in ``moe_oracle.c``. All arrays are numpy; bf16 tensors are
``uint16`` arrays of raw bits, e4m3 tensors ``uint8`` arrays of codes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")

# -O3 vectorises the side-by-side rows; -ffp-contract=off keeps every
# multiply and add separately rounded; no fast-math (no reassociation).
CFLAGS = ["-O3", "-mavx2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]


def build(force: bool = False) -> str:
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _L():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        sig = {
            "oracle_router_logits": [vp, vp, vp, vp, i64, i64, i64, vp, i32],
            "oracle_topk": [vp, i64, i64, i32, vp, vp],
            "oracle_permute": [vp, i64, i64, i32, vp, vp, vp, vp],
            "oracle_expert_gated_rows": [vp, i64, vp, i64, i64, i32, vp],
            "oracle_expert_down_rows": [vp, i64, vp, i64, i64, vp],
            "oracle_quant_act_fp8": [vp, i64, i64, vp, vp, i32],
            "oracle_quant_weight_fp8": [vp, i64, i64, i64, vp, vp, i32, i32],
            "oracle_experts_combine": [vp, vp, i64, i64, i64, i64, i32, vp, vp, vp, vp, i32, vp,
                                       i32],
            "oracle_experts_combine_fp8": [vp, vp, i64, i64, i64, i64, i32, vp, vp, vp, vp, vp, vp,
                                           i32, i32, vp, i32],
            "oracle_moe_forward": [vp, vp, i64, i64, i64, i64, i32, vp, vp, vp, vp, vp, vp, vp, vp,
                                   i32, i32, vp, vp, vp, vp, i32],
            "oracle_quant_weight_fp4": [vp, i64, i64, i64, vp, vp, i32],
            "oracle_experts_combine_fp4": [vp, vp, i64, i64, i64, i64, i32, vp, vp, vp, vp, vp, vp,
                                           i32, vp, i32],
            "oracle_moe_forward_fp4": [vp, vp, i64, i64, i64, i64, i32, vp, vp, vp, vp, vp, vp,
                                       i32, vp, vp, vp, vp, i32],
        }
        for name, args in sig.items():
            f = getattr(lib, name)
            f.argtypes = args
            f.restype = None
        lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_decode.restype = ctypes.c_double
        lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        lib.oracle_e4m3_encode.restype = ctypes.c_uint8
        lib.oracle_e2m1_decode.argtypes = [ctypes.c_uint8]
        lib.oracle_e2m1_decode.restype = ctypes.c_double
        lib.oracle_e2m1_encode.argtypes = [ctypes.c_float]
        lib.oracle_e2m1_encode.restype = ctypes.c_uint8
        _lib = lib
    return _lib


def threads() -> int:
    return max(1, min(256, os.cpu_count() or 1))


def _p(a):
    if a is None:
        return None
    assert isinstance(a, np.ndarray) and a.flags["C_CONTIGUOUS"], "contiguous numpy array required"
    return a.ctypes.data


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def router_logits(x, wr, bias=None, tokens=None, nthreads=None):
    x, wr = _c(x, np.uint16), _c(wr, np.uint16)
    H, E = wr.shape
    if tokens is not None:
        tokens = _c(tokens, np.int32)
    nt = x.shape[0] if tokens is None else len(tokens)
    out = np.empty((nt, E), dtype=np.float32)
    b = None if bias is None else _c(bias, np.float32)
    _L().oracle_router_logits(_p(x), _p(wr), _p(b), _p(tokens), nt, H, E, _p(out),
                              nthreads or threads())
    return out


def topk(logits, k):
    logits = _c(logits, np.float32)
    T, E = logits.shape
    ids = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float32)
    _L().oracle_topk(_p(logits), T, E, k, _p(ids), _p(w))
    return ids, w


def permute(ids, E):
    ids = _c(ids, np.int32)
    T, k = ids.shape
    offsets = np.empty(E + 1, dtype=np.int32)
    perm_token = np.empty(T * k, dtype=np.int32)
    perm_slot = np.empty(T * k, dtype=np.int32)
    inv_perm = np.empty(T * k, dtype=np.int32)
    _L().oracle_permute(_p(ids), T, E, k, _p(offsets), _p(perm_token), _p(perm_slot), _p(inv_perm))
    return offsets, perm_token, perm_slot, inv_perm.reshape(T, k)


# gated activations of the expert MLP (values of the C ABI's epilogue enum)
ACT_SILU, ACT_GELU, ACT_RELU = 1, 2, 3


def expert_gated_rows(a_rows, w13e, act=ACT_SILU):
    """act(A Wg) * (A Wu) for bf16 rows A [n, H] and one expert's w13 [2I, H]."""
    a_rows, w13e = _c(a_rows, np.uint16), _c(w13e, np.uint16)
    n, H = a_rows.shape
    I = w13e.shape[0] // 2
    out = np.empty((n, I), dtype=np.float32)
    _L().oracle_expert_gated_rows(_p(a_rows), n, _p(w13e), H, I, int(act), _p(out))
    return out


def expert_swiglu_rows(a_rows, w13e):
    """silu(A Wg) * (A Wu) for bf16 rows A [n, H] and one expert's w13 [2I, H]."""
    return expert_gated_rows(a_rows, w13e, ACT_SILU)


def expert_down_rows(h_rows, w2e):
    """h Wd for bf16 rows h [n, I] and one expert's w2 [H, I]."""
    h_rows, w2e = _c(h_rows, np.uint16), _c(w2e, np.uint16)
    n, I = h_rows.shape
    H = w2e.shape[0]
    out = np.empty((n, H), dtype=np.float32)
    _L().oracle_expert_down_rows(_p(h_rows), n, _p(w2e), H, I, _p(out))
    return out


def e4m3_decode(q: int) -> float:
    return _L().oracle_e4m3_decode(int(q))


def e4m3_encode(f: float) -> int:
    return int(_L().oracle_e4m3_encode(float(f)))


def quant_act_fp8(x, ue8m0=False):
    """Per row, per 128-column group: s = amax/448 (1 if amax == 0), q = e4m3(x/s).
    ue8m0: s is the smallest power of two >= amax/448 instead."""
    x = _c(x, np.uint16)
    rows, cols = x.shape
    q = np.empty((rows, cols), dtype=np.uint8)
    s = np.empty((rows, cols // 128), dtype=np.float32)
    _L().oracle_quant_act_fp8(_p(x), rows, cols, _p(q), _p(s), int(bool(ue8m0)))
    return q, s


def quant_weight_fp8(w, nthreads=None, ue8m0=False):
    """128 x 128 blocks of w [nb, rows, cols]: q [nb, rows, cols], s [nb, rows/128, cols/128]."""
    w = _c(w, np.uint16)
    nb, rows, cols = w.shape
    q = np.empty((nb, rows, cols), dtype=np.uint8)
    s = np.empty((nb, rows // 128, cols // 128), dtype=np.float32)
    _L().oracle_quant_weight_fp8(_p(w), nb, rows, cols, _p(q), _p(s), int(bool(ue8m0)),
                                 nthreads or threads())
    return q, s


def e2m1_decode(q: int) -> float:
    return _L().oracle_e2m1_decode(int(q))


def e2m1_encode(f: float) -> int:
    return int(_L().oracle_e2m1_encode(float(f)))


def quant_weight_fp4(w, nthreads=None):
    """Per row, per 32 consecutive columns of w [nb, rows, cols] (bf16 bits):
    s = smallest power of two >= amax/6 (1 if amax == 0), q = e2m1(w/s).
    Returns q [nb, rows, cols/2] (element 2i in the low nibble of byte i) and
    the e8m0 codes of s [nb, rows, cols/32]."""
    w = _c(w, np.uint16)
    nb, rows, cols = w.shape
    q = np.empty((nb, rows, cols // 2), dtype=np.uint8)
    sc = np.empty((nb, rows, cols // 32), dtype=np.uint8)
    _L().oracle_quant_weight_fp4(_p(w), nb, rows, cols, _p(q), _p(sc), nthreads or threads())
    return q, sc


def experts_combine_fp4(x, tokens, ids, w, w13q, w13s, w2q, w2s, nthreads=None, act=ACT_SILU):
    x, tokens = _c(x, np.uint16), _c(tokens, np.int32)
    ids, w = _c(ids, np.int32), _c(w, np.float32)
    w13q, w2q, w13s, w2s = (_c(a, np.uint8) for a in (w13q, w2q, w13s, w2s))
    E, I2, H2 = w13q.shape
    nt, k = ids.shape
    H = 2 * H2
    out = np.empty((nt, H), dtype=np.float32)
    _L().oracle_experts_combine_fp4(_p(x), _p(tokens), nt, H, I2 // 2, E, k, _p(ids), _p(w),
                                    _p(w13q), _p(w13s), _p(w2q), _p(w2s), int(act), _p(out),
                                    nthreads or threads())
    return out


def e8m0_code(s):
    """The float8_e8m0fnu byte of power-of-two scales s (2^(code - 127))."""
    s = np.asarray(s, dtype=np.float32)
    m, e = np.frexp(s)
    assert np.all(m == 0.5), "not powers of two"
    return (e - 1 + 127).astype(np.uint8)


def experts_combine(x, tokens, ids, w, w13, w2, nthreads=None, act=ACT_SILU):
    x, tokens = _c(x, np.uint16), _c(tokens, np.int32)
    ids, w = _c(ids, np.int32), _c(w, np.float32)
    w13, w2 = _c(w13, np.uint16), _c(w2, np.uint16)
    E, I2, H = w13.shape
    nt, k = ids.shape
    out = np.empty((nt, H), dtype=np.float32)
    _L().oracle_experts_combine(_p(x), _p(tokens), nt, H, I2 // 2, E, k, _p(ids), _p(w), _p(w13),
                                _p(w2), int(act), _p(out), nthreads or threads())
    return out


def experts_combine_fp8(x, tokens, ids, w, w13q, w13s, w2q, w2s, nthreads=None, act=ACT_SILU,
                        ue8m0=False):
    x, tokens = _c(x, np.uint16), _c(tokens, np.int32)
    ids, w = _c(ids, np.int32), _c(w, np.float32)
    w13q, w2q = _c(w13q, np.uint8), _c(w2q, np.uint8)
    w13s, w2s = _c(w13s, np.float32), _c(w2s, np.float32)
    E, I2, H = w13q.shape
    nt, k = ids.shape
    out = np.empty((nt, H), dtype=np.float32)
    _L().oracle_experts_combine_fp8(_p(x), _p(tokens), nt, H, I2 // 2, E, k, _p(ids), _p(w),
                                    _p(w13q), _p(w13s), _p(w2q), _p(w2s), int(act),
                                    int(bool(ue8m0)), _p(out), nthreads or threads())
    return out


def moe_forward(x, wr, bias, w13=None, w2=None, k=2, tokens=None, fp8=None, nthreads=None,
                act=ACT_SILU, ue8m0=False, fp4=None):
    """The whole layer for ``tokens`` (all when None).

    ``fp8`` = (w13q, w13s, w2q, w2s) selects the FP8 experts (x is quantised
    inside); ``fp4`` = the packed e2m1 codes and e8m0 scale codes of
    ``quant_weight_fp4`` selects the FP4 experts. Returns dict(out [nt,H]
    f32, ids, w, logits).
    """
    x, wr = _c(x, np.uint16), _c(wr, np.uint16)
    T, H = x.shape
    E = wr.shape[1]
    tokens = np.arange(T, dtype=np.int32) if tokens is None else _c(tokens, np.int32)
    nt = len(tokens)
    if fp4 is not None:
        w13q, w13s, w2q, w2s = (_c(a, np.uint8) for a in fp4)
        I = w13q.shape[1] // 2
        b = None if bias is None else _c(bias, np.float32)
        out = np.empty((nt, H), dtype=np.float32)
        ids = np.empty((nt, k), dtype=np.int32)
        w = np.empty((nt, k), dtype=np.float32)
        logits = np.empty((nt, E), dtype=np.float32)
        _L().oracle_moe_forward_fp4(_p(x), _p(tokens), nt, H, I, E, k, _p(wr), _p(b), _p(w13q),
                                    _p(w13s), _p(w2q), _p(w2s), int(act), _p(out), _p(ids), _p(w),
                                    _p(logits), nthreads or threads())
        return {"out": out, "ids": ids, "w": w, "logits": logits}
    if fp8 is not None:
        w13q, w13s, w2q, w2s = (_c(fp8[0], np.uint8), _c(fp8[1], np.float32),
                                _c(fp8[2], np.uint8), _c(fp8[3], np.float32))
        I = w13q.shape[1] // 2
    else:
        w13, w2 = _c(w13, np.uint16), _c(w2, np.uint16)
        w13q = w13s = w2q = w2s = None
        I = w13.shape[1] // 2
    b = None if bias is None else _c(bias, np.float32)
    out = np.empty((nt, H), dtype=np.float32)
    ids = np.empty((nt, k), dtype=np.int32)
    w = np.empty((nt, k), dtype=np.float32)
    logits = np.empty((nt, E), dtype=np.float32)
    _L().oracle_moe_forward(_p(x), _p(tokens), nt, H, I, E, k, _p(wr), _p(b),
                            _p(w13) if fp8 is None else None, _p(w2) if fp8 is None else None,
                            _p(w13q), _p(w13s), _p(w2q), _p(w2s), int(act), int(bool(ue8m0)),
                            _p(out), _p(ids), _p(w), _p(logits), nthreads or threads())
    return {"out": out, "ids": ids, "w": w, "logits": logits}
