"""Independent fp64 restatement of the MoE layer for pinning the oracle.

Used only by tests on tiny shapes.  It shares no code with the oracle: the
FP8 encode/decode steps go through torch's ``float8_e4m3fn`` dtype, E2M1
decoding through the OCP MX table in ``tests/golden`` (and E2M1 encoding by
brute-force nearest search over that table), matrix products through numpy
``einsum`` in float64, and tokens are processed densely per expert.
"""
from __future__ import annotations

import os

import numpy as np
import torch

_GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def load_table(name: str) -> dict:
    tab = {}
    with open(os.path.join(_GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            code, val = line.split()
            tab[int(code, 16)] = float(val)
    return tab


E2M1 = load_table("e2m1_ocp_mx.txt")
_E2M1_ARR = np.array([E2M1[c] for c in range(16)], dtype=np.float64)


def e4m3_values(codes: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8)).view(torch.float8_e4m3fn)
    return t.to(torch.float64).numpy()


def quant128(v: np.ndarray):
    """fp32 rows [..., K] -> (code values float64 [..., K], scales float32 [..., K/128]).

    Scale amax/448 (1 for an all-zero group), codes by torch's RNE cast of v/s."""
    t = torch.from_numpy(np.ascontiguousarray(v, dtype=np.float32))
    K = t.shape[-1]
    g = t.reshape(*t.shape[:-1], K // 128, 128)
    amax = g.abs().amax(dim=-1)
    s = torch.where(amax == 0, torch.ones_like(amax), amax / 448.0)
    q = (g / s[..., None]).to(torch.float8_e4m3fn)
    return q.to(torch.float64).reshape(t.shape).numpy(), s.numpy()


def e2m1_nearest(v: np.ndarray) -> np.ndarray:
    """E2M1 codes by brute force over the OCP table: the nearest value, ties to
    the code with mantissa bit 0, magnitudes beyond 6 to 6, sign bit kept."""
    vals = _E2M1_ARR[:8]
    a = np.minimum(np.abs(np.asarray(v, dtype=np.float64)), 6.0)
    dist = np.abs(a[..., None] - vals)
    cand = dist == dist.min(axis=-1, keepdims=True)
    even = cand & (np.arange(8) % 2 == 0)
    code = np.where(even.any(axis=-1), even.argmax(axis=-1), cand.argmax(axis=-1)).astype(np.uint8)
    return np.where(np.signbit(v), code | 8, code).astype(np.uint8)


def unpack_e2m1(w: np.ndarray, K: int) -> np.ndarray:
    codes = np.empty(w.shape[:-1] + (K,), dtype=np.uint8)
    codes[..., 0::2] = w & 0xF
    codes[..., 1::2] = w >> 4
    return codes


def quant_nvfp4(v: np.ndarray):
    """fp32 rows [..., K] -> (element x block-scale values float64 [..., K],
    per-128 scales float32 [..., K/128], E2M1 codes [..., K], E4M3 block codes
    [..., K/16]).  S = amax128/2688 (1 if zero), block code from torch's RNE
    cast of amax16/6/S, element codes by brute-force nearest of v/d."""
    t = torch.from_numpy(np.ascontiguousarray(v, dtype=np.float32))
    K = t.shape[-1]
    g = t.reshape(*t.shape[:-1], K // 128, 128)
    amax = g.abs().amax(dim=-1)
    S = torch.where(amax == 0, torch.ones_like(amax), amax / 2688.0)
    b = t.reshape(*t.shape[:-1], K // 16, 16)
    S16 = S.repeat_interleave(8, dim=-1)
    c = ((b.abs().amax(dim=-1) / 6.0) / S16).to(torch.float8_e4m3fn)
    d = c.float() * S16
    ratio = (b / torch.where(d == 0, torch.ones_like(d), d)[..., None]).numpy()
    q = e2m1_nearest(ratio)
    q = np.where((d == 0).numpy()[..., None], 0, q).astype(np.uint8)
    vals = _E2M1_ARR[q] * c.to(torch.float64).numpy()[..., None]
    shape = t.shape
    return vals.reshape(shape), S.numpy(), q.reshape(shape), c.view(torch.uint8).numpy()


def quant_mxfp4(v: np.ndarray):
    """fp32 rows [..., K] -> (element x 2^X values float64 [..., K], unit per-128
    scales float32 [..., K/128], E2M1 codes [..., K], E8M0 codes [..., K/32]).
    X = floor(log2 amax32) - 2 from numpy's frexp (exact), clamped to
    [-127, 127], -127 for an all-zero block; elements by brute-force nearest."""
    a = np.ascontiguousarray(v, dtype=np.float32)
    K = a.shape[-1]
    g = a.reshape(*a.shape[:-1], K // 32, 32)
    amax = np.abs(g).max(axis=-1)
    _, ex = np.frexp(amax.astype(np.float64))        # amax = m * 2^ex with m in [0.5, 1)
    X = np.where(amax == 0, -127, ex - 1 - 2)
    X = np.clip(X, -127, 127)
    scale = np.ldexp(1.0, X).astype(np.float32)       # exact powers of two
    q = e2m1_nearest((g / scale[..., None]).astype(np.float32))
    vals = _E2M1_ARR[q] * scale.astype(np.float64)[..., None]
    ones = np.ones(a.shape[:-1] + (K // 128,), np.float32)
    return vals.reshape(a.shape), ones, q.reshape(a.shape), (X + 127).astype(np.uint8)


def quant_mxfp8(v: np.ndarray):
    """fp32 rows [..., K] -> (element x 2^X values float64 [..., K], unit per-128
    scales float32 [..., K/128], E4M3 codes uint8 [..., K], E8M0 codes [..., K/32]).
    X = floor(log2 amax32) - 8 from numpy's frexp (exact), clamped to
    [-127, 127], -127 for an all-zero block; elements by torch's RNE cast to
    float8_e4m3fn of v / 2^X clamped to +-448 (the cast itself does not
    saturate)."""
    a = np.ascontiguousarray(v, dtype=np.float32)
    K = a.shape[-1]
    g = a.reshape(*a.shape[:-1], K // 32, 32)
    amax = np.abs(g).max(axis=-1)
    _, ex = np.frexp(amax.astype(np.float64))        # amax = m * 2^ex with m in [0.5, 1)
    X = np.where(amax == 0, -127, ex - 1 - 8)
    X = np.clip(X, -127, 127)
    scale = np.ldexp(1.0, X)
    r = np.clip(g.astype(np.float64) / scale[..., None], -448.0, 448.0).astype(np.float32)
    q = torch.from_numpy(np.ascontiguousarray(r)).to(torch.float8_e4m3fn)
    vals = q.to(torch.float64).numpy() * scale[..., None]
    ones = np.ones(a.shape[:-1] + (K // 128,), np.float32)
    return vals.reshape(a.shape), ones, q.view(torch.uint8).numpy().reshape(a.shape), (X + 127).astype(np.uint8)


def dequant_weights(w: np.ndarray, s: np.ndarray, wfmt: int, K: int) -> np.ndarray:
    """One expert's weights [R, K] as float64 code values, with the MXFP4 E8M0
    scale (NVFP4: the E4M3 block scale) folded in.  FP8 block scales and the
    NVFP4 global scale are applied separately."""
    if wfmt == 0:
        return e4m3_values(w)
    if wfmt == 4:  # MXFP8: E4M3 elements, E8M0 scale per 32
        return e4m3_values(w) * np.repeat(np.exp2(s.astype(np.float64) - 127.0), 32, axis=1)
    vals = _E2M1_ARR[unpack_e2m1(w, K)]
    if wfmt == 2:
        return vals * np.repeat(e4m3_values(s), 16, axis=1)
    scale = np.exp2(s.astype(np.float64) - 127.0)
    return vals * np.repeat(scale, 32, axis=1)


def grouped_gemm(ad: np.ndarray, as_: np.ndarray, wd: np.ndarray, ws, wfmt: int, wg=None) -> np.ndarray:
    """ad [n,K] code values, as_ [n,K/128]; wd [R,K]; ws [R/128,K/128] (FP8);
    wg the NVFP4 global scale -> [n,R] fp64."""
    n, K = ad.shape
    R = wd.shape[0]
    KB = K // 128
    part = np.einsum("nkc,rkc->nrk", ad.reshape(n, KB, 128), wd.reshape(R, KB, 128))
    part = part * as_.astype(np.float64)[:, None, :]
    if wfmt == 0:
        part = part * np.repeat(ws.astype(np.float64), 128, axis=0)[None, :, :]
    if wfmt == 2:
        part = part * float(wg)
    return part.sum(axis=2)


def expert_ffn(xd, xs, w13, s13, w2, s2, wfmt, H, I, g13=None, g2=None):
    """Tokens of one expert: quantised activations -> fp64 expert output [n,H]."""
    if wfmt == 4:  # MXFP8: every scale is folded into the values on both sides
        G = grouped_gemm(xd, xs, dequant_weights(w13, s13, 4, H), s13, 1)
        g, u = G[:, :I], G[:, I:]
        h = g / (1.0 + np.exp(-g)) * u
        hd, hs = quant_mxfp8(h.astype(np.float32))[:2]
        return grouped_gemm(hd, hs, dequant_weights(w2, s2, 4, I), s2, 1)
    if wfmt == 3:  # MXFP4 weights: the E8M0 scales are folded in by dequant_weights
        wfmt_w = 1
        G = grouped_gemm(xd, xs, dequant_weights(w13, s13, 1, H), s13, 1)
        g, u = G[:, :I], G[:, I:]
        h = g / (1.0 + np.exp(-g)) * u
        hd, hs = quant_mxfp4(h.astype(np.float32))[:2]
        return grouped_gemm(hd, hs, dequant_weights(w2, s2, wfmt_w, I), s2, 1)
    G = grouped_gemm(xd, xs, dequant_weights(w13, s13, wfmt, H), s13, wfmt, g13)
    g, u = G[:, :I], G[:, I:]
    h = g / (1.0 + np.exp(-g)) * u
    if wfmt == 2:
        hd, hs = quant_nvfp4(h.astype(np.float32))[:2]
    elif wfmt == 3:
        hd, hs = quant_mxfp4(h.astype(np.float32))[:2]
    else:
        hd, hs = quant128(h.astype(np.float32))
    return grouped_gemm(hd, hs, dequant_weights(w2, s2, wfmt, I), s2, wfmt, g2)


def moe_layer(x_bits, ids, topk_w, w13, s13, w2, s2, *, H, I, E, wfmt, n_shared=0, g13=None, g2=None):
    """Whole layer, token by token and slot by slot, in fp64."""
    x = (x_bits.astype(np.uint32) << 16).view(np.float32)
    xd, xs = (quant_nvfp4(x)[:2] if wfmt == 2 else quant_mxfp4(x)[:2] if wfmt == 3
              else quant_mxfp8(x)[:2] if wfmt == 4 else quant128(x))
    T, k = ids.shape
    out = np.zeros((T, H), dtype=np.float64)

    def gs(g, e):
        return None if g is None else g[e]

    for t in range(T):
        for j in range(k):
            e = int(ids[t, j])
            if not 0 <= e < E:
                continue
            y = expert_ffn(xd[t:t + 1], xs[t:t + 1], w13[e], s13[e], w2[e], s2[e], wfmt, H, I,
                           gs(g13, e), gs(g2, e))
            out[t] += float(topk_w[t, j]) * y[0]
        if n_shared:
            y = expert_ffn(xd[t:t + 1], xs[t:t + 1], w13[E], s13[E], w2[E], s2[E], wfmt, H, I,
                           gs(g13, E), gs(g2, E))
            out[t] += y[0]
    return out


def unquantised_layer(x_bits, ids, topk_w, w13, s13, w2, s2, *, H, I, E, wfmt):
    """The same layer with no activation quantisation (dequantised weights)."""
    x = (x_bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    T, k = ids.shape
    out = np.zeros((T, H))

    def full(w, s, R, K):
        d = dequant_weights(w, s, wfmt, K)
        if wfmt == 0:
            d = d * np.repeat(np.repeat(s.astype(np.float64), 128, 0), 128, 1)
        return d

    for t in range(T):
        for j in range(k):
            e = int(ids[t, j])
            W13 = full(w13[e], s13[e], 2 * I, H)
            W2 = full(w2[e], s2[e], H, I)
            G = W13 @ x[t]
            h = G[:I] / (1 + np.exp(-G[:I])) * G[I:]
            out[t] += float(topk_w[t, j]) * (W2 @ h)
    return out
