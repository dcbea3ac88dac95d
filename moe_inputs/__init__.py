"""Seeded synthetic inputs for the sparse MoE FFN layer.

This module is the one source of input bits shared by the CPU oracle and the
CUDA path. It holds random draws only (see ``gen.c`` for the generator's
definition) and none of the layer's arithmetic: no routing, no expert
projection, no quantisation.

Layer shapes follow the workloads the layer is exercised on: a tiny layer,
a Mixtral-shaped layer (prefill and decode), and a fine-grained
many-expert layer (bf16 and FP8). Every tensor is drawn from its LOGICAL index
(``x[T,H]``, ``Wr[H,E]``, ``Wg/Wu[E,H,I]``, ``Wd[E,I,H]``) and stored in the
layout the library consumes:

* ``x``    ``[T, H]`` bf16, N(0, 1)
* ``wr``   ``[H, E]`` bf16, N(0, 0.02)
* ``bias`` ``[E]`` fp32: zero, N(0, 0.5), or the Zipf(s=1.1) log-pmf of a seeded
  rank permutation in units of the logits' own spread,
  ``-1.1 * sigma_l * ln(rank)`` with ``sigma_l = x_sigma * w_sigma * sqrt(H)``
* ``w13``  ``[E, 2I, H]`` bf16, K-major: rows ``[0, I)`` are ``Wg[e]^T``, rows
  ``[I, 2I)`` are ``Wu[e]^T``; N(0, 0.02)
* ``w2``   ``[E, H, I]`` bf16, K-major: ``Wd[e]^T``; N(0, 0.02)

bf16 tensors are returned as ``numpy.uint16`` arrays holding the raw bits.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gen.c")
_LIB = os.path.join(_HERE, "libmoe_inputs.so")

# Stream tags: one independent stream per tensor.
TAG_X, TAG_WR, TAG_BIAS, TAG_WG, TAG_WU, TAG_WD, TAG_SUBSET, TAG_ZIPF = 1, 2, 3, 4, 5, 6, 7, 8


def build(force: bool = False) -> str:
    """Compile gen.c into a shared library next to it (gcc, -O2, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fno-fast-math", "-o", tmp,
                               _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _L():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        i64, u64, u32, f32, i32 = (ctypes.c_int64, ctypes.c_uint64, ctypes.c_uint32,
                                   ctypes.c_float, ctypes.c_int)
        vp = ctypes.c_void_p
        lib.gen_normal_bf16.argtypes = [u64, u32, f32, i64, i64, i64, i32, i64, vp, i32]
        lib.gen_normal_f32.argtypes = [u64, u32, f32, i64, i64, i64, i32, i64, vp, i32]
        lib.gen_permutation.argtypes = [u64, u32, i64, vp]
        lib.gen_raw_u64.argtypes = [u64, u32, i64, vp]
        lib.gen_splitmix64.argtypes = [u64]
        lib.gen_splitmix64.restype = u64
        for f in (lib.gen_normal_bf16, lib.gen_normal_f32, lib.gen_permutation, lib.gen_raw_u64):
            f.restype = None
        _lib = lib
    return _lib


def _threads() -> int:
    return max(1, min(256, os.cpu_count() or 1))


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def splitmix64(z: int) -> int:
    return int(_L().gen_splitmix64(z))


def raw_u64(seed: int, tag: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.uint64)
    _L().gen_raw_u64(seed, tag, n, _ptr(out))
    return out


def normal_bf16(seed, tag, sigma, nb, R, C, transpose=False, bstride=None, out=None):
    """Draw logical ``[nb, R, C]``; store ``[nb, C, R]`` when ``transpose``."""
    if bstride is None:
        bstride = R * C
    if out is None:
        out = np.empty(nb * bstride, dtype=np.uint16)
    _L().gen_normal_bf16(seed, tag, sigma, nb, R, C, int(transpose), bstride, _ptr(out), _threads())
    return out


def normal_f32(seed, tag, sigma, nb, R, C, transpose=False):
    out = np.empty(nb * R * C, dtype=np.float32)
    _L().gen_normal_f32(seed, tag, sigma, nb, R, C, int(transpose), R * C, _ptr(out), _threads())
    return out


def permutation(seed: int, tag: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.int32)
    _L().gen_permutation(seed, tag, n, _ptr(out))
    return out


@dataclass(frozen=True)
class LayerConfig:
    name: str
    T: int
    H: int
    I: int
    E: int
    k: int
    bias: str = "zero"          # "zero" | "normal" | "zipf"
    bias_sigma: float = 0.5
    zipf_s: float = 1.1
    fp8: bool = False
    ue8m0: bool = False         # FP8 scales as powers of two (block-scaled tensor-core path)
    fp4: bool = False           # FP4 (e2m1) expert weights with e8m0 scales per (row, 32)
    x_sigma: float = 1.0
    w_sigma: float = 0.02
    seed: int = 0
    subset: int = 0             # 0: compare every token; else a seeded sorted subset
    desc: str = field(default="", compare=False)

    @property
    def R(self) -> int:
        return self.T * self.k

    def with_(self, **kw) -> "LayerConfig":
        d = dict(self.__dict__)
        d.update(kw)
        return LayerConfig(**d)


CONFIGS = {
    "tiny": LayerConfig("tiny", 64, 128, 256, 8, 2,
                        desc="tiny layer: T=64 H=128 I=256 E=8 k=2 bf16"),
    "mixtral_prefill": LayerConfig("mixtral_prefill", 4096, 4096, 14336, 8, 2, bias="normal",
                                   subset=512,
                                   desc="Mixtral-shaped prefill: T=4096 H=4096 I=14336 E=8 k=2 "
                                        "bf16, router bias N(0,0.5)"),
    "mixtral_decode": LayerConfig("mixtral_decode", 16, 4096, 14336, 8, 2,
                                  desc="Mixtral-shaped decode: T=16 H=4096 I=14336 E=8 k=2 bf16"),
    "fine_grained": LayerConfig("fine_grained", 8192, 7168, 2048, 256, 8, bias="zipf", subset=512,
                                desc="fine-grained prefill: T=8192 H=7168 I=2048 E=256 k=8 bf16, "
                                     "Zipf(1.1) router bias"),
    "fine_grained_fp8": LayerConfig("fine_grained_fp8", 8192, 7168, 2048, 256, 8, bias="zipf",
                                    subset=512, fp8=True,
                                    desc="fine-grained prefill, FP8 experts (128x128 weight "
                                         "blocks, 1x128 activation groups)"),
    "fine_grained_fp8_ue8m0": LayerConfig("fine_grained_fp8_ue8m0", 8192, 7168, 2048, 256, 8,
                                          bias="zipf", subset=512, fp8=True, ue8m0=True,
                                          desc="fine-grained prefill, FP8 experts with power-of-two "
                                               "(UE8M0) scales on the block-scaled MMA"),
    "fine_grained_fp4": LayerConfig("fine_grained_fp4", 8192, 7168, 2048, 256, 8, bias="zipf",
                                    subset=512, fp4=True,
                                    desc="fine-grained prefill, FP4 (e2m1) expert weights with "
                                         "UE8M0 scales per 32, e4m3 activations"),
    "mixtral_decode_fp4": LayerConfig("mixtral_decode_fp4", 16, 4096, 14336, 8, 2, fp4=True,
                                      desc="Mixtral-shaped decode, FP4 expert weights: T=16 "
                                           "H=4096 I=14336 E=8 k=2"),
    "mixtral_decode_fp8_ue8m0": LayerConfig("mixtral_decode_fp8_ue8m0", 16, 4096, 14336, 8, 2,
                                            fp8=True, ue8m0=True,
                                            desc="Mixtral-shaped decode, FP8 experts with "
                                                 "power-of-two scales: T=16 H=4096 I=14336 E=8 k=2"),
    "mixtral_decode_fp8": LayerConfig("mixtral_decode_fp8", 16, 4096, 14336, 8, 2, fp8=True,
                                      desc="Mixtral-shaped decode, FP8 experts: T=16 H=4096 "
                                           "I=14336 E=8 k=2"),
}


def make_x(cfg: LayerConfig) -> np.ndarray:
    return normal_bf16(cfg.seed, TAG_X, cfg.x_sigma, 1, cfg.T, cfg.H).reshape(cfg.T, cfg.H)


def make_router(cfg: LayerConfig):
    wr = normal_bf16(cfg.seed, TAG_WR, cfg.w_sigma, 1, cfg.H, cfg.E).reshape(cfg.H, cfg.E)
    if cfg.bias == "zero":
        b = np.zeros(cfg.E, dtype=np.float32)
    elif cfg.bias == "normal":
        b = normal_f32(cfg.seed, TAG_BIAS, cfg.bias_sigma, 1, 1, cfg.E).reshape(cfg.E)
    elif cfg.bias == "zipf":
        # The Zipf(s) log-pmf of each expert's rank, -s*ln(rank) up to a constant, measured
        # in the logits' own standard deviation sigma_l (the nominal spread of x.Wr), so the
        # skew it imposes does not shrink as H grows. In plain logit units the router's
        # own spread (1.69 at H = 7168) flattens it and every expert keeps some tokens.
        perm = permutation(cfg.seed, TAG_ZIPF, cfg.E)
        rank = np.empty(cfg.E, dtype=np.int64)
        rank[perm] = np.arange(1, cfg.E + 1)
        sigma_l = cfg.x_sigma * cfg.w_sigma * math.sqrt(cfg.H)
        b = np.array([-cfg.zipf_s * sigma_l * math.log(r) for r in rank], dtype=np.float32)
    else:
        raise ValueError(cfg.bias)
    return wr, b


def make_w13(cfg: LayerConfig) -> np.ndarray:
    E, H, I = cfg.E, cfg.H, cfg.I
    w13 = np.empty(E * 2 * I * H, dtype=np.uint16)
    # gate block of expert e starts at e*2I*H, up block at e*2I*H + I*H
    normal_bf16(cfg.seed, TAG_WG, cfg.w_sigma, E, H, I, transpose=True, bstride=2 * I * H,
                out=w13)
    normal_bf16(cfg.seed, TAG_WU, cfg.w_sigma, E, H, I, transpose=True, bstride=2 * I * H,
                out=w13[I * H:])
    return w13.reshape(E, 2 * I, H)


def make_w2(cfg: LayerConfig) -> np.ndarray:
    E, H, I = cfg.E, cfg.H, cfg.I
    return normal_bf16(cfg.seed, TAG_WD, cfg.w_sigma, E, I, H, transpose=True).reshape(E, H, I)


def token_subset(cfg: LayerConfig, n: int | None = None) -> np.ndarray:
    """Seeded sorted subset of token indices (all tokens when no subset applies)."""
    n = cfg.subset if n is None else n
    if n <= 0 or n >= cfg.T:
        return np.arange(cfg.T, dtype=np.int32)
    perm = permutation(cfg.seed, TAG_SUBSET, cfg.T)
    return np.sort(perm[:n]).astype(np.int32)


def make_layer(cfg: LayerConfig) -> dict:
    wr, b = make_router(cfg)
    return {"x": make_x(cfg), "wr": wr, "bias": b, "w13": make_w13(cfg), "w2": make_w2(cfg)}


def bf16_to_f32(a: np.ndarray) -> np.ndarray:
    """Widen raw bf16 bits to float32 (exact)."""
    return (a.astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 bits, nearest even (finite inputs)."""
    b = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    b = b + 0x7FFF + ((b >> 16) & 1)
    return (b >> 16).astype(np.uint16)
