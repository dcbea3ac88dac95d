"""B200 (sm_100a) sparse Mixture-of-Experts FFN layer forward.

A thin ctypes binding of ``libmoe_b200.so`` (the C ABI in ``include/moe.h``):
every function here has the C entry point's name and arguments and only
marshals them (tensor -> device pointer, current torch stream -> cudaStream_t).
Every step of the layer runs in the library's CUDA kernels; there is no
fallback. If the library is missing, importing the binding's functions fails
loudly (build it with ``python -m mixture_experts_layer_tcgen05_b200.build``
or ``__graft_entry__.build()``).

Arguments that are device buffers accept a ``torch.Tensor`` (its
``data_ptr()``), a raw integer address, or ``None`` where the C function
allows NULL. ``stream`` defaults to torch's current CUDA stream.
"""
from __future__ import annotations

import ctypes
import os

__all__ = [
    "MoeError", "Dims", "WsLayout", "lib", "lib_path", "MOE_OK", "MOE_ERR_INVALID_ARG",
    "MOE_ERR_UNSUPPORTED_DEVICE", "MOE_ERR_WORKSPACE", "MOE_ERR_CUDA", "MOE_ERR_TIMEOUT",
    "MOE_DTYPE_BF16", "MOE_DTYPE_FP8_E4M3", "MOE_EPILOGUE_NONE", "MOE_EPILOGUE_SWIGLU",
    "MOE_EPILOGUE_GEGLU", "MOE_EPILOGUE_REGLU", "moe_forward_gated", "moe_forward_fp8_gated",
    "MOE_SCALE_F32", "MOE_SCALE_UE8M0", "moe_quantize_act_fp8_fmt", "moe_quantize_weight_fp8_fmt",
    "MOE_DTYPE_FP8_E4M3_UE8M0", "moe_forward_fp8_ue8m0",
    "MOE_DTYPE_FP4_E2M1", "moe_forward_fp4", "moe_grouped_gemm_fp4", "moe_quantize_weight_fp4",
    "moe_last_error", "moe_abi_version", "moe_launch_count", "moe_workspace_size",
    "moe_workspace_layout", "moe_route_topk", "moe_topk_from_logits", "moe_permute",
    "moe_permute_noalloc", "moe_permute_noalloc_status",
    "moe_grouped_gemm", "moe_combine", "moe_gather_rows", "moe_forward", "moe_forward_fp8", "moe_forward_hostio",
    "moe_quantize_act_fp8", "moe_quantize_weight_fp8", "moe_pack_weights", "moe_get_device_status",
    "moe_ep_plan_bytes", "moe_ep_plan", "moe_ep_dispatch", "moe_ep_return",
    "moe_clear_device_status", "moe_set_stage_events", "moe_check_wait_timeout", "EXPORTED",
]

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED_DEVICE = 0, 1, 2
MOE_ERR_WORKSPACE, MOE_ERR_CUDA, MOE_ERR_TIMEOUT = 3, 4, 5
MOE_DTYPE_BF16, MOE_DTYPE_FP8_E4M3, MOE_DTYPE_FP8_E4M3_UE8M0, MOE_DTYPE_FP4_E2M1 = 0, 1, 2, 3
MOE_EPILOGUE_NONE, MOE_EPILOGUE_SWIGLU, MOE_EPILOGUE_GEGLU, MOE_EPILOGUE_REGLU = 0, 1, 2, 3
MOE_SCALE_F32, MOE_SCALE_UE8M0 = 0, 1

_HERE = os.path.dirname(os.path.abspath(__file__))
lib_path = os.path.join(_HERE, "libmoe_b200.so")


class MoeError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"moe status {status}: {msg}")
        self.status = status


class Dims(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("H", ctypes.c_int32), ("I", ctypes.c_int32),
                ("E", ctypes.c_int32), ("k", ctypes.c_int32)]


class WsLayout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in (
        "status", "logits", "topk_ids", "topk_w", "offsets", "perm_token", "inv_perm", "x_perm",
        "xq", "xs", "xq_perm", "xs_perm", "h", "hq", "hs", "splitk", "y_perm", "scratch", "total")]


_vp, _i32, _i64, _sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
# C signatures: name -> (restype, argtypes)
_SIGS = {
    "moe_last_error": (ctypes.c_char_p, []),
    "moe_abi_version": (_i32, []),
    "moe_launch_count": (_i64, []),
    "moe_workspace_size": (_sz, [Dims, _i32]),
    "moe_workspace_layout": (_i32, [Dims, _i32, ctypes.POINTER(WsLayout)]),
    "moe_route_topk": (_i32, [_vp, _vp, _vp, Dims, _vp, _vp, _vp, _vp, _sz, _vp]),
    "moe_topk_from_logits": (_i32, [_vp, Dims, _vp, _vp, _vp]),
    "moe_permute": (_i32, [_vp, Dims, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "moe_permute_noalloc": (_i32, [_vp, Dims, _vp, _vp, _vp, _vp, _vp, _vp]),
    "moe_permute_noalloc_status": (_i32, [ctypes.POINTER(_i32), _i32]),
    "moe_grouped_gemm": (_i32, [_vp, _vp, _i32, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _vp,
                                _vp, _vp, _vp, _i32, _vp, _sz, _vp]),
    "moe_combine": (_i32, [_vp, _vp, _vp, Dims, _vp, _vp]),
    "moe_gather_rows": (_i32, [_vp, _i64, _vp, _i64, _i64, _vp, _vp, _vp]),
    "moe_forward": (_i32, [_vp, _vp, _vp, _vp, _vp, Dims, _vp, _vp, _sz, _vp]),
    "moe_forward_fp8": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, Dims, _vp, _vp, _sz, _vp]),
    "moe_forward_hostio": (_i32, [_vp, _vp, _vp, _vp, _vp, Dims, _vp, _vp, _sz, _vp]),
    "moe_forward_gated": (_i32, [_vp, _vp, _vp, _vp, _vp, Dims, _i32, _vp, _vp, _sz, _vp]),
    "moe_forward_fp8_gated": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, Dims, _i32, _vp, _vp, _sz,
                                     _vp]),
    "moe_forward_fp8_ue8m0": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, Dims, _i32, _vp, _vp, _sz,
                                     _vp]),
    "moe_forward_fp4": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, Dims, _i32, _vp, _vp, _sz, _vp]),
    "moe_grouped_gemm_fp4": (_i32, [_vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _vp,
                                    _vp, _i32, _vp, _sz, _vp]),
    "moe_quantize_weight_fp4": (_i32, [_vp, _i64, _i64, _i64, _vp, _vp, _vp]),
    "moe_quantize_act_fp8": (_i32, [_vp, _i64, _i64, _vp, _vp, _vp]),
    "moe_quantize_weight_fp8": (_i32, [_vp, _i64, _i64, _i64, _vp, _vp, _vp]),
    "moe_quantize_act_fp8_fmt": (_i32, [_vp, _i64, _i64, _vp, _vp, _i32, _vp]),
    "moe_quantize_weight_fp8_fmt": (_i32, [_vp, _i64, _i64, _i64, _vp, _vp, _i32, _vp]),
    "moe_pack_weights": (_i32, [_vp, _vp, _vp, _i32, _i32, _i32, _vp, _vp, _vp]),
    "moe_ep_plan_bytes": (_sz, [_i32, _i32]),
    "moe_ep_plan": (_i32, [_vp, _i32, _i32, _i32, _vp, _vp]),
    "moe_ep_dispatch": (_i32, [_vp, _vp, _vp, _i32, _i32, _i32, _i64, _vp, _i64, _vp, _vp]),
    "moe_ep_return": (_i32, [_vp, _vp, _i32, _i32, _i64, _i64, _vp, _i64, _vp, _vp]),
    "moe_get_device_status": (_i32, [_vp, ctypes.POINTER(_i32)]),
    "moe_clear_device_status": (_i32, [_vp, _vp]),
    "moe_check_wait_timeout": (_i32, [_vp, _i64, _vp]),
    "moe_set_stage_events": (_i32, [ctypes.POINTER(_vp), _i32]),
}
EXPORTED = tuple(_SIGS)

_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(lib_path):
            raise ImportError(f"{lib_path} is missing: build it with "
                              "`python -m mixture_experts_layer_tcgen05_b200.build`")
        L = ctypes.CDLL(lib_path)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype, f.argtypes = res, args
        _lib = L
    return _lib


def _p(a):
    """Device (or host) address of a tensor / int / None."""
    if a is None:
        return None
    if isinstance(a, int):
        return a
    if hasattr(a, "data_ptr"):
        return a.data_ptr()
    if hasattr(a, "ctypes"):  # numpy
        return a.ctypes.data
    raise TypeError(f"cannot take the address of {type(a)}")


def _s(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _nbytes(ws, ws_bytes):
    if ws_bytes is not None:
        return ws_bytes
    if hasattr(ws, "numel"):
        return ws.numel() * ws.element_size()
    raise ValueError("ws_bytes is required for a raw workspace address")


def _check(st: int):
    if st != MOE_OK:
        raise MoeError(st, moe_last_error())


def _dims(d) -> Dims:
    if isinstance(d, Dims):
        return d
    if isinstance(d, dict):
        return Dims(d["T"], d["H"], d["I"], d["E"], d["k"])
    return Dims(*d)


def moe_last_error() -> str:
    return lib().moe_last_error().decode()


def moe_abi_version() -> int:
    return lib().moe_abi_version()


def moe_launch_count() -> int:
    return lib().moe_launch_count()


def moe_workspace_size(d, dt: int = MOE_DTYPE_BF16) -> int:
    return lib().moe_workspace_size(_dims(d), dt)


def moe_workspace_layout(d, dt: int = MOE_DTYPE_BF16) -> WsLayout:
    out = WsLayout()
    _check(lib().moe_workspace_layout(_dims(d), dt, ctypes.byref(out)))
    return out


def moe_route_topk(x, wr, bias, d, logits, ids, w, ws=None, ws_bytes=None, stream=None):
    nb = _nbytes(ws, ws_bytes) if ws is not None else 0
    _check(lib().moe_route_topk(_p(x), _p(wr), _p(bias), _dims(d), _p(logits), _p(ids), _p(w),
                                _p(ws), nb, _s(stream)))


def moe_topk_from_logits(logits, d, ids, w, stream=None):
    _check(lib().moe_topk_from_logits(_p(logits), _dims(d), _p(ids), _p(w), _s(stream)))


def moe_permute(ids, d, offsets, perm_token, inv_perm, x, x_perm, ws, ws_bytes=None, stream=None):
    _check(lib().moe_permute(_p(ids), _dims(d), _p(offsets), _p(perm_token), _p(inv_perm), _p(x),
                             _p(x_perm), _p(ws), _nbytes(ws, ws_bytes), _s(stream)))


def moe_permute_noalloc(ids, d, offsets, perm_token, inv_perm, x=None, x_perm=None, stream=None):
    """moe_permute with the library's fixed scratch array (no workspace, no allocation)."""
    _check(lib().moe_permute_noalloc(_p(ids), _dims(d), _p(offsets), _p(perm_token), _p(inv_perm),
                                     _p(x), _p(x_perm), _s(stream)))


def moe_permute_noalloc_status(clear: bool = False) -> int:
    v = ctypes.c_int32(0)
    _check(lib().moe_permute_noalloc_status(ctypes.byref(v), int(bool(clear))))
    return v.value


def moe_grouped_gemm(A, B, offsets, M_total, E, N, K, dt, ep, C, a_scales=None, b_scales=None,
                     c_scales=None, max_rows_per_expert=0, ws=None, ws_bytes=None, stream=None,
                     a_rows=None, a_src_rows=0):
    _check(lib().moe_grouped_gemm(_p(A), _p(a_rows), a_src_rows, _p(B), _p(offsets), M_total, E, N,
                                  K, dt, ep, _p(C),
                                  _p(a_scales), _p(b_scales), _p(c_scales), max_rows_per_expert,
                                  _p(ws), _nbytes(ws, ws_bytes), _s(stream)))


def moe_gather_rows(src, src_rows, rows, n, row_bytes, dst, ws=None, stream=None):
    _check(lib().moe_gather_rows(_p(src), int(src_rows), _p(rows), int(n), int(row_bytes), _p(dst),
                                 _p(ws), _s(stream)))


def moe_combine(y_perm, w, inv_perm, d, out, stream=None):
    _check(lib().moe_combine(_p(y_perm), _p(w), _p(inv_perm), _dims(d), _p(out), _s(stream)))


def moe_forward(x, wr, bias, w13, w2, d, out, ws, ws_bytes=None, stream=None):
    _check(lib().moe_forward(_p(x), _p(wr), _p(bias), _p(w13), _p(w2), _dims(d), _p(out), _p(ws),
                             _nbytes(ws, ws_bytes), _s(stream)))


def moe_forward_fp8(x, wr, bias, w13q, w13s, w2q, w2s, d, out, ws, ws_bytes=None, stream=None):
    _check(lib().moe_forward_fp8(_p(x), _p(wr), _p(bias), _p(w13q), _p(w13s), _p(w2q), _p(w2s),
                                 _dims(d), _p(out), _p(ws), _nbytes(ws, ws_bytes), _s(stream)))


def moe_forward_gated(x, wr, bias, w13, w2, d, act, out, ws, ws_bytes=None, stream=None):
    _check(lib().moe_forward_gated(_p(x), _p(wr), _p(bias), _p(w13), _p(w2), _dims(d), int(act),
                                   _p(out), _p(ws), _nbytes(ws, ws_bytes), _s(stream)))


def moe_forward_fp8_gated(x, wr, bias, w13q, w13s, w2q, w2s, d, act, out, ws, ws_bytes=None,
                          stream=None):
    _check(lib().moe_forward_fp8_gated(_p(x), _p(wr), _p(bias), _p(w13q), _p(w13s), _p(w2q),
                                       _p(w2s), _dims(d), int(act), _p(out), _p(ws),
                                       _nbytes(ws, ws_bytes), _s(stream)))


def moe_forward_fp8_ue8m0(x, wr, bias, w13q, w13s, w2q, w2s, d, act, out, ws, ws_bytes=None,
                          stream=None):
    _check(lib().moe_forward_fp8_ue8m0(_p(x), _p(wr), _p(bias), _p(w13q), _p(w13s), _p(w2q),
                                       _p(w2s), _dims(d), int(act), _p(out), _p(ws),
                                       _nbytes(ws, ws_bytes), _s(stream)))


def moe_forward_fp4(x, wr, bias, w13q, w13s, w2q, w2s, d, act, out, ws, ws_bytes=None,
                    stream=None):
    _check(lib().moe_forward_fp4(_p(x), _p(wr), _p(bias), _p(w13q), _p(w13s), _p(w2q), _p(w2s),
                                 _dims(d), int(act), _p(out), _p(ws), _nbytes(ws, ws_bytes),
                                 _s(stream)))


def moe_grouped_gemm_fp4(A, a_scales, B, b_scales, offsets, M_total, E, N, K, ep, C,
                         c_scales=None, ws=None, ws_bytes=None, stream=None, max_rows_per_expert=0):
    _check(lib().moe_grouped_gemm_fp4(_p(A), _p(a_scales), _p(B), _p(b_scales), _p(offsets),
                                      M_total, E, N, K, int(ep), _p(C), _p(c_scales),
                                      int(max_rows_per_expert), _p(ws), _nbytes(ws, ws_bytes),
                                      _s(stream)))


def moe_quantize_weight_fp4(w, nb, rows, cols, q, s, stream=None):
    _check(lib().moe_quantize_weight_fp4(_p(w), nb, rows, cols, _p(q), _p(s), _s(stream)))


def moe_forward_hostio(x_host, wr, bias, w13, w2, d, out_host, ws, ws_bytes=None, stream=None):
    _check(lib().moe_forward_hostio(_p(x_host), _p(wr), _p(bias), _p(w13), _p(w2), _dims(d),
                                    _p(out_host), _p(ws), _nbytes(ws, ws_bytes), _s(stream)))


def moe_quantize_act_fp8(x, rows, cols, q, s, stream=None):
    _check(lib().moe_quantize_act_fp8(_p(x), rows, cols, _p(q), _p(s), _s(stream)))


def moe_quantize_weight_fp8(w, nb, rows, cols, q, s, stream=None):
    _check(lib().moe_quantize_weight_fp8(_p(w), nb, rows, cols, _p(q), _p(s), _s(stream)))


def moe_quantize_act_fp8_fmt(x, rows, cols, q, s, fmt, stream=None):
    _check(lib().moe_quantize_act_fp8_fmt(_p(x), rows, cols, _p(q), _p(s), int(fmt), _s(stream)))


def moe_quantize_weight_fp8_fmt(w, nb, rows, cols, q, s, fmt, stream=None):
    _check(lib().moe_quantize_weight_fp8_fmt(_p(w), nb, rows, cols, _p(q), _p(s), int(fmt),
                                             _s(stream)))


def moe_pack_weights(wg, wu, wd, E, H, I, w13, w2, stream=None):
    _check(lib().moe_pack_weights(_p(wg), _p(wu), _p(wd), E, H, I, _p(w13), _p(w2), _s(stream)))


def moe_ep_plan_bytes(E, G) -> int:
    return int(lib().moe_ep_plan_bytes(E, G))


def moe_ep_plan(counts_all, G, rank, E, plan, stream=None):
    _check(lib().moe_ep_plan(_p(counts_all), G, rank, E, _p(plan), _s(stream)))


def moe_ep_dispatch(x_perm, offsets, plan, E, G, R, row_bytes, dst_bufs, dst_rows, ws=None,
                    stream=None):
    _check(lib().moe_ep_dispatch(_p(x_perm), _p(offsets), _p(plan), E, G, R, row_bytes,
                                 _p(dst_bufs), dst_rows, _p(ws), _s(stream)))


def moe_ep_return(y_loc, plan, E, G, cap_rows, row_bytes, src_bufs, src_rows, ws=None, stream=None):
    _check(lib().moe_ep_return(_p(y_loc), _p(plan), E, G, cap_rows, row_bytes, _p(src_bufs),
                               src_rows, _p(ws), _s(stream)))


def moe_get_device_status(ws) -> int:
    v = ctypes.c_int32(0)
    _check(lib().moe_get_device_status(_p(ws), ctypes.byref(v)))
    return v.value


def moe_clear_device_status(ws, stream=None):
    _check(lib().moe_clear_device_status(_p(ws), _s(stream)))


def moe_check_wait_timeout(ws, budget_cycles, stream=None):
    _check(lib().moe_check_wait_timeout(_p(ws), int(budget_cycles), _s(stream)))


def moe_set_stage_events(events):
    """events: list of 6 torch.cuda.Event (recorded by later forwards) or None to stop."""
    if events is None:
        _check(lib().moe_set_stage_events(None, 0))
        return
    handles = []
    for e in events:
        if hasattr(e, "cuda_event"):
            if not e.cuda_event:  # torch creates the CUDA event lazily, on first record
                e.record()
            handles.append(e.cuda_event)
        else:
            handles.append(int(e))
    arr = (_vp * len(handles))(*handles)
    _check(lib().moe_set_stage_events(arr, len(handles)))
