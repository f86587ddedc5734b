"""Independent fp64 restatement of the MoE layer for pinning the oracle.

Used only by tests on tiny shapes.  It shares no code with the oracle: the
FP8 encode/decode steps go through torch's ``float8_e4m3fn`` dtype, E2M1
decoding through the OCP MX table in ``tests/golden``, matrix products through
numpy ``einsum`` in float64, and tokens are processed densely per expert.
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


def dequant_weights(w: np.ndarray, s: np.ndarray, wfmt: int, K: int) -> np.ndarray:
    """One expert's weights [R, K] as float64 code values, with the MXFP4 E8M0
    scale folded in.  FP8 block scales are applied separately per K block."""
    if wfmt == 0:
        return e4m3_values(w)
    lo = w & 0xF
    hi = w >> 4
    codes = np.empty((w.shape[0], K), dtype=np.uint8)
    codes[:, 0::2] = lo
    codes[:, 1::2] = hi
    vals = _E2M1_ARR[codes]
    scale = np.exp2(s.astype(np.float64) - 127.0)
    return vals * np.repeat(scale, 32, axis=1)


def grouped_gemm(ad: np.ndarray, as_: np.ndarray, wd: np.ndarray, ws, wfmt: int) -> np.ndarray:
    """ad [n,K] code values, as_ [n,K/128]; wd [R,K]; ws [R/128,K/128] (FP8) -> [n,R] fp64."""
    n, K = ad.shape
    R = wd.shape[0]
    KB = K // 128
    part = np.einsum("nkc,rkc->nrk", ad.reshape(n, KB, 128), wd.reshape(R, KB, 128))
    part = part * as_.astype(np.float64)[:, None, :]
    if wfmt == 0:
        part = part * np.repeat(ws.astype(np.float64), 128, axis=0)[None, :, :]
    return part.sum(axis=2)


def expert_ffn(xd, xs, w13, s13, w2, s2, wfmt, H, I):
    """Tokens of one expert: quantised activations -> fp64 expert output [n,H]."""
    G = grouped_gemm(xd, xs, dequant_weights(w13, s13, wfmt, H), s13, wfmt)
    g, u = G[:, :I], G[:, I:]
    h = g / (1.0 + np.exp(-g)) * u
    hd, hs = quant128(h.astype(np.float32))
    return grouped_gemm(hd, hs, dequant_weights(w2, s2, wfmt, I), s2, wfmt)


def moe_layer(x_bits, ids, topk_w, w13, s13, w2, s2, *, H, I, E, wfmt, n_shared=0):
    """Whole layer, token by token and slot by slot, in fp64."""
    x = (x_bits.astype(np.uint32) << 16).view(np.float32)
    xd, xs = quant128(x)
    T, k = ids.shape
    out = np.zeros((T, H), dtype=np.float64)
    for t in range(T):
        for j in range(k):
            e = int(ids[t, j])
            if not 0 <= e < E:
                continue
            y = expert_ffn(xd[t:t + 1], xs[t:t + 1], w13[e], s13[e], w2[e], s2[e], wfmt, H, I)
            out[t] += float(topk_w[t, j]) * y[0]
        if n_shared:
            y = expert_ffn(xd[t:t + 1], xs[t:t + 1], w13[E], s13[E], w2[E], s2[E], wfmt, H, I)
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
