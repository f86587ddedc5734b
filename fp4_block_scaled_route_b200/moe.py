"""Thin ctypes binding of ``libmoe.so`` (include/moe.h).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  The entry points keep the C names (``moe_create``, ``moe_forward``
...).  :class:`MoeLayer` wraps a context for torch tensors: it passes
``data_ptr()`` values and the current CUDA stream handle, nothing else.

There is no fallback: if the library is missing, or a call fails, this module
raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_UNSUPPORTED = 2
MOE_ERR_CUDA = 3
MOE_ERR_NO_MEMORY = 4
MOE_ERR_TIMEOUT = 5
MOE_ERR_BAD_ROUTING = 6

MOE_WFMT_FP8_E4M3_B128 = 0
MOE_WFMT_MXFP4_E2M1_E8M0_K32 = 1
MOE_WFMT_NVFP4_E2M1_E4M3_K16 = 2
MOE_WFMT_MXFP4_W4A4 = 3
MOE_WFMT_MXFP8_E4M3_E8M0_K32 = 4

# Every entry point declared in include/moe.h: name -> (restype, argtypes)
_vp = ctypes.c_void_p
_i = ctypes.c_int
SIGNATURES = {
    "moe_create": (_i, [_i, _i, _i, _i, _i, ctypes.POINTER(_vp)]),
    "moe_create_ex": (_i, [_i, _i, _i, _i, _i, _i, _i, ctypes.POINTER(_vp)]),
    "moe_destroy": (None, [_vp]),
    "moe_forward": (_i, [_vp, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "moe_forward_nvfp4": (_i, [_vp, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "moe_forward_partial": (_i, [_vp, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "moe_finalize_bf16": (_i, [_vp, _vp, ctypes.c_longlong, _vp]),
    "moe_pack_mxfp4_scales": (_i, [_vp, _vp, _i, _i, _vp]),
    "moe_pack_nvfp4_scales": (_i, [_vp, _vp, _i, _i, _vp]),
    "moe_declare_packed_scales": (_i, [_vp, ctypes.c_longlong, _i]),
    "moe_get_routing": (_i, [_vp, _vp, _vp, _vp, _vp, _vp]),
    "moe_get_activations": (_i, [_vp, _vp, _vp, _vp, _vp, _vp]),
    "moe_get_block_scales": (_i, [_vp, _vp, _vp, _vp]),
    "moe_get_device_status": (_i, [_vp, _vp]),
    "moe_last_config": (_i, [_vp, ctypes.POINTER(_i), ctypes.POINTER(_i)]),
    "moe_set_fault_injection": (_i, [_vp, _i]),
    "moe_profile_enable": (_i, [_vp, _i]),
    "moe_profile_read": (_i, [_vp, ctypes.POINTER(ctypes.c_float), ctypes.POINTER(_i)]),
    "moe_forward_noalloc": (_i, [_i, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "moe_router_topk": (_i, [_vp, _i, _vp, _vp, _vp, _vp, _vp]),
    "moe_set_green_ctx": (_i, [_vp, _i]),
    "moe_green_ctx_sms": (_i, [_vp, ctypes.POINTER(_i), ctypes.POINTER(_i)]),
    "moe_set_dispatch_overlap": (_i, [_vp, _i]),
    "moe_dispatch_overlap_ctas": (_i, [_vp, ctypes.POINTER(_i)]),
    "moe_status_string": (ctypes.c_char_p, [_i]),
}

_lib: Optional[ctypes.CDLL] = None


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


def lib() -> ctypes.CDLL:
    """Load libmoe.so (built by ``python -m fp4_block_scaled_route_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m fp4_block_scaled_route_b200.build` (no CPU fallback exists)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().moe_status_string(status).decode()


def _check(status: int, where: str) -> None:
    if status != MOE_OK:
        raise MoeError(status, where)


# ---- C entry points under their own names --------------------------------
def moe_create(H, I, E, k, wfmt):
    ctx = _vp()
    _check(lib().moe_create(H, I, E, k, wfmt, ctypes.byref(ctx)), "moe_create")
    return ctx


def moe_create_ex(H, I, E, k, wfmt, max_T, n_shared):
    ctx = _vp()
    _check(lib().moe_create_ex(H, I, E, k, wfmt, max_T, n_shared, ctypes.byref(ctx)), "moe_create_ex")
    return ctx


def moe_destroy(ctx) -> None:
    lib().moe_destroy(ctx)


def moe_forward(ctx, T, x, topk_ids, topk_w, w13, s13, w2, s2, out, stream) -> int:
    return lib().moe_forward(ctx, T, x, topk_ids, topk_w, w13, s13, w2, s2, out, stream)


def moe_forward_nvfp4(ctx, T, x, topk_ids, topk_w, w13, s13, g13, w2, s2, g2, out, stream) -> int:
    return lib().moe_forward_nvfp4(ctx, T, x, topk_ids, topk_w, w13, s13, g13, w2, s2, g2, out, stream)


def moe_forward_partial(ctx, T, x, topk_ids, topk_w, w13, s13, g13, w2, s2, g2, out_f32, stream) -> int:
    return lib().moe_forward_partial(ctx, T, x, topk_ids, topk_w, w13, s13, g13, w2, s2, g2, out_f32, stream)


def moe_finalize_bf16(inp, out, n, stream) -> int:
    return lib().moe_finalize_bf16(inp, out, n, stream)


def moe_forward_noalloc(H, I, E, k, wfmt, n_shared, T, x, topk_ids, topk_w, w13, s13, w2, s2, out, d_status,
                        stream) -> int:
    return lib().moe_forward_noalloc(H, I, E, k, wfmt, n_shared, T, x, topk_ids, topk_w, w13, s13, w2, s2, out,
                                     d_status, stream)


def moe_pack_mxfp4_scales(src, dst, rows, K, stream) -> int:
    return lib().moe_pack_mxfp4_scales(src, dst, rows, K, stream)


def moe_pack_nvfp4_scales(src, dst, rows, K, stream) -> int:
    return lib().moe_pack_nvfp4_scales(src, dst, rows, K, stream)


def moe_declare_packed_scales(p, nbytes, wfmt) -> int:
    return lib().moe_declare_packed_scales(p, nbytes, wfmt)


def moe_get_block_scales(ctx, xsc, hsc, stream) -> int:
    return lib().moe_get_block_scales(ctx, xsc, hsc, stream)


def moe_get_routing(ctx, counts, offsets, perm, inv, stream) -> int:
    return lib().moe_get_routing(ctx, counts, offsets, perm, inv, stream)


def moe_get_activations(ctx, xq, xs, hq, hs, stream) -> int:
    return lib().moe_get_activations(ctx, xq, xs, hq, hs, stream)


def moe_get_device_status(ctx, stream) -> int:
    return lib().moe_get_device_status(ctx, stream)


def moe_last_config(ctx):
    bn, grid = _i(), _i()
    _check(lib().moe_last_config(ctx, ctypes.byref(bn), ctypes.byref(grid)), "moe_last_config")
    return bn.value, grid.value


MOE_NUM_STAGES = 5
STAGE_NAMES = ("route", "quant", "gemm1_swiglu_requant", "gemm2_combine", "finalize")


def moe_set_fault_injection(ctx, mode) -> int:
    return lib().moe_set_fault_injection(ctx, mode)


def moe_router_topk(ctx, T, x, wr, topk_ids, topk_w, stream) -> int:
    return lib().moe_router_topk(ctx, T, x, wr, topk_ids, topk_w, stream)


def moe_set_green_ctx(ctx, dispatch_sms) -> int:
    return lib().moe_set_green_ctx(ctx, dispatch_sms)


def moe_green_ctx_sms(ctx):
    d, g = _i(), _i()
    _check(lib().moe_green_ctx_sms(ctx, ctypes.byref(d), ctypes.byref(g)), "moe_green_ctx_sms")
    return d.value, g.value


def moe_set_dispatch_overlap(ctx, dispatch_ctas) -> int:
    return lib().moe_set_dispatch_overlap(ctx, dispatch_ctas)


def moe_dispatch_overlap_ctas(ctx) -> int:
    d = _i()
    _check(lib().moe_dispatch_overlap_ctas(ctx, ctypes.byref(d)), "moe_dispatch_overlap_ctas")
    return d.value


def moe_profile_enable(ctx, on) -> int:
    return lib().moe_profile_enable(ctx, on)


def moe_profile_read(ctx):
    """Mean milliseconds per stage over the recorded calls, and their number."""
    arr = (ctypes.c_float * MOE_NUM_STAGES)()
    n = _i()
    _check(lib().moe_profile_read(ctx, arr, ctypes.byref(n)), "moe_profile_read")
    return list(arr), n.value


# ---- torch convenience wrapper (marshalling only) ------------------------
def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream_handle(stream=None) -> int:
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


class MoeLayer:
    """One context of the library; tensors are torch CUDA tensors."""

    def __init__(self, H, I, E, k, wfmt=MOE_WFMT_FP8_E4M3_B128, max_T=4096, n_shared=0):
        self.H, self.I, self.E, self.k, self.wfmt = H, I, E, k, wfmt
        self.max_T, self.n_shared = max_T, n_shared
        self.ctx = moe_create_ex(H, I, E, k, wfmt, max_T, n_shared)

    def close(self):
        if self.ctx:
            moe_destroy(self.ctx)
            self.ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def forward(self, x, topk_ids, topk_w, w13, s13, w2, s2, out=None, stream=None, g13=None, g2=None):
        """One layer; NVFP4 contexts also take the global scales g13 / g2 (moe_forward_nvfp4)."""
        import torch
        T = x.shape[0]
        if out is None:
            out = torch.empty((T, self.H), dtype=torch.bfloat16, device=x.device)
        nv = self.wfmt == MOE_WFMT_NVFP4_E2M1_E4M3_K16
        ts = (x, topk_ids, topk_w, w13, s13, w2, s2, out) + ((g13, g2) if nv else ())
        for t in ts:
            if t is None or not t.is_cuda or not t.is_contiguous():
                raise ValueError("MoeLayer.forward needs contiguous CUDA tensors")
        if nv:
            _check(moe_forward_nvfp4(self.ctx, T, _ptr(x), _ptr(topk_ids), _ptr(topk_w), _ptr(w13), _ptr(s13),
                                     _ptr(g13), _ptr(w2), _ptr(s2), _ptr(g2), _ptr(out), _stream_handle(stream)),
                   "moe_forward_nvfp4")
        else:
            _check(moe_forward(self.ctx, T, _ptr(x), _ptr(topk_ids), _ptr(topk_w), _ptr(w13), _ptr(s13),
                               _ptr(w2), _ptr(s2), _ptr(out), _stream_handle(stream)), "moe_forward")
        return out

    def forward_partial(self, x, topk_ids, topk_w, w13, s13, w2, s2, out=None, stream=None, g13=None, g2=None):
        """fp32 [T, H] partial combine result of this context's I slice (moe_forward_partial)."""
        import torch
        T = x.shape[0]
        if out is None:
            out = torch.empty((T, self.H), dtype=torch.float32, device=x.device)
        for t in (x, topk_ids, topk_w, w13, s13, w2, s2, out):
            if not t.is_cuda or not t.is_contiguous():
                raise ValueError("MoeLayer.forward_partial needs contiguous CUDA tensors")
        _check(moe_forward_partial(self.ctx, T, _ptr(x), _ptr(topk_ids), _ptr(topk_w), _ptr(w13), _ptr(s13),
                                   _ptr(g13), _ptr(w2), _ptr(s2), _ptr(g2), _ptr(out), _stream_handle(stream)),
               "moe_forward_partial")
        return out

    def routing(self, T, stream=None):
        """(counts, offsets, perm, inv) of the last forward, as host int32 numpy arrays."""
        import numpy as np
        P = T * self.k + self.n_shared * T
        NG = self.E + self.n_shared
        counts = np.zeros(NG, np.int32)
        offsets = np.zeros(NG + 1, np.int32)
        perm = np.zeros(max(P, 1), np.int32)
        inv = np.zeros(max(P, 1), np.int32)
        _check(moe_get_routing(self.ctx, counts.ctypes.data, offsets.ctypes.data, perm.ctypes.data,
                               inv.ctypes.data, _stream_handle(stream)), "moe_get_routing")
        return counts, offsets, perm[:P], inv[:P]

    def activations(self, T, stream=None):
        """(xq, xs, hq, hs) of the last forward, host numpy arrays in routing-position order
        (NVFP4: xq / hq packed, two codes per byte)."""
        import numpy as np
        P = T * self.k + self.n_shared * T
        cw = 2 if self.wfmt in (MOE_WFMT_NVFP4_E2M1_E4M3_K16, MOE_WFMT_MXFP4_W4A4) else 1
        xq = np.zeros((max(P, 1), self.H // cw), np.uint8)
        xs = np.zeros((max(P, 1), self.H // 128), np.float32)
        hq = np.zeros((max(P, 1), self.I // cw), np.uint8)
        hs = np.zeros((max(P, 1), self.I // 128), np.float32)
        _check(moe_get_activations(self.ctx, xq.ctypes.data, xs.ctypes.data, hq.ctypes.data, hs.ctypes.data,
                                   _stream_handle(stream)), "moe_get_activations")
        return xq[:P], xs[:P], hq[:P], hs[:P]

    def block_scales(self, T, stream=None):
        """4-bit activations: (xsc, hsc) block codes of the last forward, host numpy
        (NVFP4: E4M3 [P, H/16], [P, I/16]; MXFP4 x MXFP4: E8M0 [P, H/32], [P, I/32])."""
        import numpy as np
        P = T * self.k + self.n_shared * T
        bs = 16 if self.wfmt == MOE_WFMT_NVFP4_E2M1_E4M3_K16 else 32
        xsc = np.zeros((max(P, 1), self.H // bs), np.uint8)
        hsc = np.zeros((max(P, 1), self.I // bs), np.uint8)
        _check(moe_get_block_scales(self.ctx, xsc.ctypes.data, hsc.ctypes.data, _stream_handle(stream)),
               "moe_get_block_scales")
        return xsc[:P], hsc[:P]

    def device_status(self, stream=None) -> int:
        return moe_get_device_status(self.ctx, _stream_handle(stream))

    def last_config(self):
        return moe_last_config(self.ctx)

    def router(self, x, wr, ids=None, w=None, stream=None):
        """Fused router: (topk_ids int32 [T,k], topk_w fp32 [T,k]) from x bf16 [T,H] and wr bf16 [E,H]."""
        import torch
        T = x.shape[0]
        if ids is None:
            ids = torch.empty((T, self.k), dtype=torch.int32, device=x.device)
        if w is None:
            w = torch.empty((T, self.k), dtype=torch.float32, device=x.device)
        for t in (x, wr, ids, w):
            if not t.is_cuda or not t.is_contiguous():
                raise ValueError("MoeLayer.router needs contiguous CUDA tensors")
        _check(moe_router_topk(self.ctx, T, _ptr(x), _ptr(wr), _ptr(ids), _ptr(w), _stream_handle(stream)),
               "moe_router_topk")
        return ids, w

    def set_green_ctx(self, dispatch_sms):
        """Green-Context partition: dispatch kernels on >= dispatch_sms SMs, GEMMs on the rest (0 = off)."""
        _check(moe_set_green_ctx(self.ctx, dispatch_sms), "moe_set_green_ctx")
        return moe_green_ctx_sms(self.ctx)

    def set_dispatch_overlap(self, dispatch_ctas):
        """Dispatch overlap: the last dispatch_ctas CTAs of the GEMM1 launch quantise first (0 = off)."""
        _check(moe_set_dispatch_overlap(self.ctx, dispatch_ctas), "moe_set_dispatch_overlap")
        return moe_dispatch_overlap_ctas(self.ctx)


def pack_nvfp4_scales(s, stream=None):
    """Plain E4M3 block codes [NE, rows, K/16] (uint8 CUDA tensor) -> the layout moe_forward_nvfp4 reads."""
    NE, rows, kg = s.shape
    dst = __import__("torch").empty_like(s)
    _check(moe_pack_nvfp4_scales(_ptr(s.contiguous()), _ptr(dst), NE * rows, kg * 16, _stream_handle(stream)),
           "moe_pack_nvfp4_scales")
    return dst


def pack_mxfp4_scales(s, stream=None):
    """Plain E8M0 scales [NE, rows, K/32] (uint8 CUDA tensor) -> the layout moe_forward reads."""
    import torch
    NE, rows, kg = s.shape
    dst = torch.empty_like(s)
    _check(moe_pack_mxfp4_scales(_ptr(s.contiguous()), _ptr(dst), NE * rows, kg * 32, _stream_handle(stream)),
           "moe_pack_mxfp4_scales")
    return dst


def finalize_bf16(acc, out=None, stream=None):
    """bf16 rounding of a summed fp32 [T, H] result (moe_finalize_bf16)."""
    import torch
    if out is None:
        out = torch.empty(acc.shape, dtype=torch.bfloat16, device=acc.device)
    _check(moe_finalize_bf16(_ptr(acc.contiguous()), _ptr(out), acc.numel(), _stream_handle(stream)),
           "moe_finalize_bf16")
    return out
