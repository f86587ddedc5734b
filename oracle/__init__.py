"""CPU oracle for the decode-regime MoE layer (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its binding) never imports, links or calls it.

The arithmetic lives in ``moe_oracle.c`` (plain C, OpenMP); this module only
compiles it with gcc and marshals numpy arrays through ctypes.  See
``moe_oracle.h`` for the passages each function follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_HDR = os.path.join(_HERE, "moe_oracle.h")
_SO = os.path.join(_HERE, "libmoe_oracle.so")
_lock = threading.Lock()
_lib = None

WFMT_FP8 = 0
WFMT_MXFP4 = 1
WFMT_NVFP4 = 2
WFMT_MXFP4_A4 = 3
WFMT_MXFP8 = 4


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/libmoe_oracle.so`` (gcc, OpenMP)."""
    newest = max(os.path.getmtime(_SRC), os.path.getmtime(_HDR))
    if not force and os.path.exists(_SO) and os.path.getmtime(_SO) >= newest:
        return _SO
    tmp = _SO + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
           "-ffp-contract=off", "-fno-fast-math", "-Wall", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _SO)
    return _SO


class _Dims(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int), ("H", ctypes.c_int), ("I", ctypes.c_int),
                ("E", ctypes.c_int), ("k", ctypes.c_int), ("wfmt", ctypes.c_int),
                ("n_shared", ctypes.c_int)]


def lib() -> ctypes.CDLL:
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(_SO)
            vp = ctypes.c_void_p
            L.orc_e4m3_decode.restype = ctypes.c_float
            L.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
            L.orc_e4m3_encode.restype = ctypes.c_uint8
            L.orc_e4m3_encode.argtypes = [ctypes.c_float]
            L.orc_e2m1_decode.restype = ctypes.c_float
            L.orc_e2m1_decode.argtypes = [ctypes.c_uint8]
            L.orc_e8m0_decode.restype = ctypes.c_float
            L.orc_e8m0_decode.argtypes = [ctypes.c_uint8]
            L.orc_bf16_decode.restype = ctypes.c_float
            L.orc_bf16_decode.argtypes = [ctypes.c_uint16]
            L.orc_bf16_encode.restype = ctypes.c_uint16
            L.orc_bf16_encode.argtypes = [ctypes.c_float]
            L.orc_e2m1_encode.restype = ctypes.c_uint8
            L.orc_e2m1_encode.argtypes = [ctypes.c_float]
            for name in ("orc_e4m3_decode_n", "orc_e4m3_encode_n", "orc_e2m1_decode_n", "orc_e2m1_encode_n"):
                getattr(L, name).restype = None
                getattr(L, name).argtypes = [vp, vp, ctypes.c_int64]
            L.orc_route.restype = ctypes.c_int
            L.orc_route.argtypes = [ctypes.c_int] * 4 + [vp] * 5
            L.orc_quant_act.restype = None
            L.orc_quant_act.argtypes = [ctypes.c_int, ctypes.c_int, vp, vp, vp]
            L.orc_quant_row_f32.restype = None
            L.orc_quant_row_f32.argtypes = [ctypes.c_int, vp, vp, vp]
            L.orc_quant_row_nvfp4.restype = None
            L.orc_quant_row_nvfp4.argtypes = [ctypes.c_int, vp, vp, vp, vp]
            L.orc_quant_act_nvfp4.restype = None
            L.orc_quant_act_nvfp4.argtypes = [ctypes.c_int, ctypes.c_int, vp, vp, vp, vp]
            L.orc_quant_row_mxfp4.restype = None
            L.orc_quant_row_mxfp4.argtypes = [ctypes.c_int, vp, vp, vp]
            L.orc_quant_act_mxfp4.restype = None
            L.orc_quant_act_mxfp4.argtypes = [ctypes.c_int, ctypes.c_int, vp, vp, vp]
            L.orc_quant_row_mxfp8.restype = None
            L.orc_quant_row_mxfp8.argtypes = [ctypes.c_int, vp, vp, vp]
            L.orc_quant_act_mxfp8.restype = None
            L.orc_quant_act_mxfp8.argtypes = [ctypes.c_int, ctypes.c_int, vp, vp, vp]
            L.orc_forward.restype = ctypes.c_int
            L.orc_forward.argtypes = [ctypes.POINTER(_Dims)] + [vp] * 13
            L.orc_forward_ex.restype = ctypes.c_int
            L.orc_forward_ex.argtypes = [ctypes.POINTER(_Dims)] + [vp] * 17
            L.orc_router.restype = ctypes.c_int
            L.orc_router.argtypes = [ctypes.c_int] * 4 + [vp] * 5
            L.orc_num_threads.restype = ctypes.c_int
            L.orc_num_threads.argtypes = []
            _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    a = np.ascontiguousarray(a)
    assert a.dtype == dtype, (a.dtype, dtype)
    return a


def num_threads() -> int:
    return lib().orc_num_threads()


# ---- codecs ---------------------------------------------------------------
def e4m3_decode(codes) -> np.ndarray:
    c = _c(np.asarray(codes, dtype=np.uint8), np.uint8)
    out = np.empty(c.shape, np.float32)
    lib().orc_e4m3_decode_n(_p(c), _p(out), c.size)
    return out


def e4m3_encode(values) -> np.ndarray:
    v = _c(np.asarray(values, dtype=np.float32), np.float32)
    out = np.empty(v.shape, np.uint8)
    lib().orc_e4m3_encode_n(_p(v), _p(out), v.size)
    return out


def e2m1_decode(nibbles) -> np.ndarray:
    c = _c(np.asarray(nibbles, dtype=np.uint8), np.uint8)
    out = np.empty(c.shape, np.float32)
    lib().orc_e2m1_decode_n(_p(c), _p(out), c.size)
    return out


def e2m1_encode(values) -> np.ndarray:
    """fp32 values -> E2M1 codes (one per byte, low nibble)."""
    v = _c(np.asarray(values, dtype=np.float32), np.float32)
    out = np.empty(v.shape, np.uint8)
    lib().orc_e2m1_encode_n(_p(v), _p(out), v.size)
    return out


def e8m0_decode(code: int) -> float:
    return float(lib().orc_e8m0_decode(code))


def bf16_decode(bits: int) -> float:
    return float(lib().orc_bf16_decode(bits))


def bf16_encode(v: float) -> int:
    return int(lib().orc_bf16_encode(v))


# ---- steps ----------------------------------------------------------------
def route(ids: np.ndarray, E: int, n_shared: int = 0):
    """Counting sort of slots by expert.  Returns (counts, offsets, perm, inv, dropped)."""
    ids = _c(ids, np.int32)
    T, k = ids.shape
    S = T * k
    P = S + n_shared * T
    counts = np.empty(E + n_shared, np.int32)
    offsets = np.empty(E + n_shared + 1, np.int32)
    perm = np.empty(max(P, 1), np.int32)
    inv = np.empty(max(P, 1), np.int32)
    dropped = lib().orc_route(T, k, E, n_shared, _p(ids), _p(counts), _p(offsets),
                              _p(perm), _p(inv))
    return counts, offsets, perm[:P], inv[:P], dropped


def quant_act(x_bf16_bits: np.ndarray):
    """x as uint16 bf16 bits [T,H] -> (xq uint8 [T,H], xs float32 [T,H/128])."""
    x = _c(x_bf16_bits, np.uint16)
    T, H = x.shape
    xq = np.empty((T, H), np.uint8)
    xs = np.empty((T, H // 128), np.float32)
    lib().orc_quant_act(T, H, _p(x), _p(xq), _p(xs))
    return xq, xs


def quant_row_f32(v: np.ndarray):
    v = _c(v, np.float32)
    (K,) = v.shape
    q = np.empty(K, np.uint8)
    s = np.empty(K // 128, np.float32)
    lib().orc_quant_row_f32(K, _p(v), _p(q), _p(s))
    return q, s


def quant_row_nvfp4(v: np.ndarray):
    """fp32 row [K] -> (q packed uint8 [K/2], block codes uint8 [K/16], s float32 [K/128])."""
    v = _c(v, np.float32)
    (K,) = v.shape
    q = np.empty(K // 2, np.uint8)
    sc = np.empty(K // 16, np.uint8)
    s = np.empty(K // 128, np.float32)
    lib().orc_quant_row_nvfp4(K, _p(v), _p(q), _p(sc), _p(s))
    return q, sc, s


def quant_act_nvfp4(x_bf16_bits: np.ndarray):
    """x as bf16 bits [T,H] -> (xq packed [T,H/2], xsc [T,H/16], xs [T,H/128])."""
    x = _c(x_bf16_bits, np.uint16)
    T, H = x.shape
    xq = np.empty((T, H // 2), np.uint8)
    xsc = np.empty((T, H // 16), np.uint8)
    xs = np.empty((T, H // 128), np.float32)
    lib().orc_quant_act_nvfp4(T, H, _p(x), _p(xq), _p(xsc), _p(xs))
    return xq, xsc, xs


def quant_row_mxfp4(v: np.ndarray):
    """fp32 row [K] -> (q packed uint8 [K/2], E8M0 codes uint8 [K/32])."""
    v = _c(v, np.float32)
    (K,) = v.shape
    q = np.empty(K // 2, np.uint8)
    sc = np.empty(K // 32, np.uint8)
    lib().orc_quant_row_mxfp4(K, _p(v), _p(q), _p(sc))
    return q, sc


def quant_act_mxfp4(x_bf16_bits: np.ndarray):
    """x as bf16 bits [T,H] -> (xq packed [T,H/2], xsc E8M0 [T,H/32])."""
    x = _c(x_bf16_bits, np.uint16)
    T, H = x.shape
    xq = np.empty((T, H // 2), np.uint8)
    xsc = np.empty((T, H // 32), np.uint8)
    lib().orc_quant_act_mxfp4(T, H, _p(x), _p(xq), _p(xsc))
    return xq, xsc


def quant_row_mxfp8(v: np.ndarray):
    """fp32 row [K] -> (E4M3 codes [K], E8M0 codes [K/32])."""
    v = _c(np.asarray(v, dtype=np.float32), np.float32)
    K = v.shape[-1]
    q = np.empty(K, np.uint8)
    sc = np.empty(K // 32, np.uint8)
    lib().orc_quant_row_mxfp8(K, _p(v), _p(q), _p(sc))
    return q, sc


def quant_act_mxfp8(x_bf16_bits: np.ndarray):
    """bf16 [T,H] -> (E4M3 codes [T,H], E8M0 codes [T,H/32])."""
    x = _c(x_bf16_bits, np.uint16)
    T, H = x.shape
    xq = np.empty((T, H), np.uint8)
    xsc = np.empty((T, H // 32), np.uint8)
    lib().orc_quant_act_mxfp8(T, H, _p(x), _p(xq), _p(xsc))
    return xq, xsc


def forward(x_bf16_bits, ids, topk_w, w13, s13, w2, s2, *, H, I, E, wfmt,
            n_shared=0, token_mask=None, debug=False, g13=None, g2=None):
    """Whole layer on the CPU.

    Returns a dict with ``out_f32`` [T,H], ``out_bf16`` (uint16 bits) [T,H],
    ``dropped`` and, with ``debug``, ``xq``/``xs`` per token and ``hq``/``hs``
    per routed position (NVFP4: packed codes, plus ``xsc``/``hsc`` block
    codes).  ``g13``/``g2`` are the NVFP4 per-expert global scales.  Rows of
    unselected tokens are NaN / 0.
    """
    x = _c(x_bf16_bits, np.uint16)
    ids = _c(ids, np.int32)
    topk_w = _c(topk_w, np.float32)
    T, k = ids.shape
    assert x.shape == (T, H)
    S = T * k
    P = S + n_shared * T
    d = _Dims(T, H, I, E, k, wfmt, n_shared)
    w13 = np.ascontiguousarray(w13)
    s13 = np.ascontiguousarray(s13)
    w2 = np.ascontiguousarray(w2)
    s2 = np.ascontiguousarray(s2)
    mask = None
    if token_mask is not None:
        mask = _c(np.asarray(token_mask, dtype=np.uint8), np.uint8)
        assert mask.shape == (T,)
    nv = wfmt == WFMT_NVFP4
    if nv:
        g13 = _c(np.asarray(g13, dtype=np.float32), np.float32)
        g2 = _c(np.asarray(g2, dtype=np.float32), np.float32)
        assert g13.shape == (E + n_shared,) and g2.shape == (E + n_shared,)
    else:
        g13 = g2 = None
    out_f32 = np.full((T, H), np.nan, np.float32)
    out_bf16 = np.zeros((T, H), np.uint16)
    dbg = {}
    if debug:
        a4 = wfmt in (WFMT_NVFP4, WFMT_MXFP4_A4)
        cw = 2 if a4 else 1
        dbg = dict(xq=np.zeros((T, H // cw), np.uint8), xs=np.zeros((T, H // 128), np.float32),
                   hq=np.zeros((max(P, 1), I // cw), np.uint8),
                   hs=np.zeros((max(P, 1), I // 128), np.float32))
        if a4 or wfmt == WFMT_MXFP8:
            bs = 16 if nv else 32
            dbg.update(xsc=np.zeros((T, H // bs), np.uint8), hsc=np.zeros((max(P, 1), I // bs), np.uint8))
    rc = lib().orc_forward_ex(ctypes.byref(d), _p(x), _p(ids), _p(topk_w), _p(w13), _p(s13), _p(g13),
                              _p(w2), _p(s2), _p(g2), _p(mask), _p(out_f32), _p(out_bf16),
                              _p(dbg.get("xq")), _p(dbg.get("xsc")), _p(dbg.get("xs")),
                              _p(dbg.get("hq")), _p(dbg.get("hsc")), _p(dbg.get("hs")))
    if rc < 0:
        raise ValueError("oracle rejected the arguments")
    res = dict(out_f32=out_f32, out_bf16=out_bf16, dropped=rc)
    if debug:
        for key in ("hq", "hs", "hsc"):
            if key in dbg:
                dbg[key] = dbg[key][:P]
        res.update(dbg)
    return res


def router(x_bf16_bits, wr_bf16_bits, k: int, *, with_logits: bool = False):
    """Fused router oracle: (ids [T,k] int32, w [T,k] fp32[, logits [T,E] fp32])."""
    x = np.ascontiguousarray(x_bf16_bits, dtype=np.uint16)
    wr = np.ascontiguousarray(wr_bf16_bits, dtype=np.uint16)
    T, H = x.shape
    E = wr.shape[0]
    assert wr.shape[1] == H
    ids = np.zeros((T, k), np.int32)
    w = np.zeros((T, k), np.float32)
    lg = np.zeros((T, E), np.float32) if with_logits else None
    L = lib()
    vp = ctypes.c_void_p
    r = L.orc_router(T, H, E, k, x.ctypes.data_as(vp), wr.ctypes.data_as(vp),
                     lg.ctypes.data_as(vp) if lg is not None else None, ids.ctypes.data_as(vp),
                     w.ctypes.data_as(vp))
    if r != 0:
        raise ValueError("orc_router: bad arguments")
    return (ids, w, lg) if with_logits else (ids, w)
