"""Checks of the GPU's SwiGLU-output requantisation codes (step 5).

Test infrastructure.  The GPU sums GEMM1 in another order than the oracle
(tensor cores, fp32 partial sums per 128-wide K block), so its SwiGLU output
h differs from the oracle's in the last bits, and a code can round the other
way where h / scale lies next to a rounding midpoint.  These helpers separate
that from a defect:

- every GPU code must equal the nearest code of the exact value
  h64 / (the GPU's own scale), where h64 is the SwiGLU output recomputed in
  fp64 from the same quantised operands, or be its neighbour on the other
  side of a midpoint that h64 / scale lies within the summation-order bound
  of;
- every GPU scale must equal the oracle's within the same bound, and a
  scale code (NVFP4 E4M3 block code, MXFP4 E8M0 exponent) may differ only by
  one step, at a midpoint (or a power of two) within that bound;
- the fraction of codes equal to the oracle's is returned for the caller to
  bound.

The summation-order bound per element is
    GAMMA * (|dh/dg| * A_g + |dh/du| * A_u)
where A_g, A_u are the sums of the absolute values of the terms of the gate
and up dot products (exactly the products the MMA adds, with every scale
applied) and GAMMA = 2^-24 * (128 + K/128 + 8): one fp32 rounding per
addition inside a 128-wide block and per promoted block, plus the SwiGLU's own
few roundings.  A plain defect (a wrong channel, row, block or lane) moves
values by whole code steps and fails these checks.

The recomputation reuses the independent fp64 restatement in dense_ref.py
(torch's float8 cast, the OCP E2M1 table, numpy einsum), never the oracle.
"""
from __future__ import annotations

import numpy as np
import torch

from tests import dense_ref

E2M1_VALUES = np.array([dense_ref.E2M1[c] for c in range(16)], np.float64)


def gamma(K: int) -> float:
    return 2.0 ** -24 * (128 + K // 128 + 8)


# ---- positions -> (token, expert) -------------------------------------------------
def position_map(perm, offsets, T, k):
    """Token and group (expert, or E for the shared expert) of every routing position."""
    P = int(offsets[-1])
    S = T * k
    p = np.asarray(perm[:P])
    tok = np.where(p < S, p // k, p - S)
    grp = np.searchsorted(np.asarray(offsets), np.arange(P), side="right") - 1
    return tok, grp


# ---- fp64 SwiGLU output and its error bound -------------------------------------------
def swiglu64(L, tokens, groups):
    """h64 [n, I] and its summation-order bound [n, I] for (token, group) pairs,
    from the same quantised activations and weights the layer uses."""
    H, I = L.H, L.I
    x = (torch_bits(L.x).astype(np.uint32) << 16).view(np.float32)
    wfmt = L.wfmt
    if wfmt == 2:
        xd_all, xs_all = dense_ref.quant_nvfp4(x[tokens])[:2]
    elif wfmt == 3:
        xd_all, xs_all = dense_ref.quant_mxfp4(x[tokens])[:2]
    elif wfmt == 4:
        xd_all, xs_all = dense_ref.quant_mxfp8(x[tokens])[:2]
    else:
        xd_all, xs_all = dense_ref.quant128(x[tokens])
    h = np.zeros((len(tokens), I))
    bound = np.zeros((len(tokens), I))
    g13 = L.g13.cpu().numpy() if getattr(L, "g13", None) is not None else None
    for e in np.unique(groups):
        rows = np.nonzero(groups == e)[0]
        w13 = L.w13[int(e)].cpu().numpy()
        s13 = L.s13[int(e)].cpu().numpy()
        wf = 1 if wfmt == 3 else wfmt
        wd = dense_ref.dequant_weights(w13, s13, wf, H)
        wg = None if g13 is None else g13[int(e)]
        G = dense_ref.grouped_gemm(xd_all[rows], xs_all[rows], wd, s13, wf, wg)
        A = dense_ref.grouped_gemm(np.abs(xd_all[rows]), xs_all[rows], np.abs(wd), s13, wf, wg)
        g, u = G[:, :I], G[:, I:]
        sig = 1.0 / (1.0 + np.exp(-g))
        h[rows] = g * sig * u
        dg = np.abs((sig + g * sig * (1.0 - sig)) * u)     # |d h / d g|
        du = np.abs(g * sig)                                # |d h / d u|
        bound[rows] = gamma(H) * (dg * A[:, :I] + du * A[:, I:]) + 4 * 2.0 ** -24 * np.abs(h[rows])
    return h, bound


def torch_bits(x: torch.Tensor) -> np.ndarray:
    return x.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


# ---- code grids -----------------------------------------------------------------------
def e4m3_values(codes) -> np.ndarray:
    return dense_ref.e4m3_values(np.asarray(codes, np.uint8))


def _signed_rank(codes, mag_mask):
    c = np.asarray(codes).astype(np.int64)
    mag = c & mag_mask
    return np.where(c & (mag_mask + 1), -mag, mag)


def _grid_check(v, code_gpu, values_of, rank_of, nearest_of, tol):
    """GPU codes against the exact ratios v (same shape): equal to the nearest
    code, or the neighbour across a midpoint that v lies within tol of.
    Returns the boolean array of violations."""
    near = nearest_of(v)
    same = (rank_of(near) == rank_of(code_gpu))
    adj = np.abs(rank_of(near) - rank_of(code_gpu)) == 1
    mid = 0.5 * (values_of(near) + values_of(code_gpu))
    ok = same | (adj & (np.abs(v - mid) <= tol))
    return ~ok


def e4m3_nearest(v):
    # ratios are computed in fp64; torch casts from fp32, so round v to fp32 first and
    # let the midpoint tolerance absorb that rounding; saturate at the E4M3 maximum
    t = torch.from_numpy(np.ascontiguousarray(np.clip(np.asarray(v, np.float64), -448.0, 448.0).astype(np.float32)))
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def e2m1_nearest(v):
    return dense_ref.e2m1_nearest(np.asarray(v, np.float64))


# ---- format-specific checks --------------------------------------------------------
class CodeReport(dict):
    """agreement (fraction of codes equal to the oracle's), scale agreement,
    the largest relative scale difference, and the number of violations."""


def check_fp8_requant(hq_g, hs_g, hq_o, hs_o, h64, bound):
    """FP8 E4M3 codes, one fp32 scale amax/448 per 128 channels."""
    n, I = h64.shape
    G = I // 128
    s_g = np.repeat(hs_g.astype(np.float64), 128, axis=1)
    v = h64 / s_g
    tol = bound / s_g + 4 * 2.0 ** -24 * np.abs(v)
    bad = _grid_check(v, hq_g, e4m3_values, lambda c: _signed_rank(c, 0x7F), e4m3_nearest, tol)
    # scales: amax / 448 of values that differ by at most the bound
    amax64 = np.abs(h64).reshape(n, G, 128).max(axis=2)
    sb = bound.reshape(n, G, 128).max(axis=2) / 448.0 + 2 * 2.0 ** -24 * amax64 / 448.0
    s_ref = np.where(amax64 == 0, 1.0, amax64 / 448.0)
    bad_s = np.abs(hs_g - s_ref) > sb
    rel = np.abs(hs_g.astype(np.float64) / hs_o - 1.0)
    return CodeReport(agreement=float((hq_g == hq_o).mean()), violations=int(bad.sum()),
                      scale_violations=int(bad_s.sum()), max_scale_rel=float(rel.max()) if rel.size else 0.0,
                      scale_agreement=float((hs_g == hs_o).mean()))


def _unpack(q, K):
    return dense_ref.unpack_e2m1(np.asarray(q, np.uint8), K)


def check_nvfp4_requant(hq_g, hsc_g, hs_g, hq_o, hsc_o, hs_o, h64, bound):
    """NVFP4: S = amax128/2688 per 128, E4M3 block code e4m3(amax16/6/S) per 16,
    E2M1 elements of h / (e4m3(code) * S)."""
    n, I = h64.shape
    S_g = hs_g.astype(np.float64)
    amax128 = np.abs(h64).reshape(n, I // 128, 128).max(axis=2)
    b128 = bound.reshape(n, I // 128, 128).max(axis=2)
    S_ref = np.where(amax128 == 0, 1.0, amax128 / 2688.0)
    bad_S = np.abs(S_g - S_ref) > b128 / 2688.0 + 2 * 2.0 ** -24 * S_ref
    # block codes against the exact amax16 / 6 / S_gpu
    amax16 = np.abs(h64).reshape(n, I // 16, 16).max(axis=2)
    b16 = bound.reshape(n, I // 16, 16).max(axis=2)
    S16 = np.repeat(S_g, 8, axis=1)
    vb = amax16 / 6.0 / S16
    tolb = b16 / 6.0 / S16 + 4 * 2.0 ** -24 * vb
    bad_c = _grid_check(vb, hsc_g, e4m3_values, lambda c: _signed_rank(c, 0x7F), e4m3_nearest, tolb)
    # elements against h / (code value * S), with the GPU's own code and S
    d = np.repeat(e4m3_values(hsc_g) * S16, 16, axis=1)
    q_g = _unpack(hq_g, I)
    zero_blk = d == 0
    v = np.where(zero_blk, 0.0, h64 / np.where(zero_blk, 1.0, d))
    tol = np.where(zero_blk, 0.0, bound / np.where(zero_blk, 1.0, d)) + 4 * 2.0 ** -24 * np.abs(v)
    bad = _grid_check(v, q_g, lambda c: E2M1_VALUES[np.asarray(c) & 15], lambda c: _signed_rank(c, 7),
                      e2m1_nearest, tol)
    bad &= ~(zero_blk & ((q_g & 7) == 0))
    rel = np.abs(S_g / hs_o - 1.0)
    return CodeReport(agreement=float((hq_g == hq_o).mean()), block_agreement=float((hsc_g == hsc_o).mean()),
                      violations=int(bad.sum()), block_violations=int(bad_c.sum()),
                      scale_violations=int(bad_S.sum()), max_scale_rel=float(rel.max()) if rel.size else 0.0)


def check_mxfp4_requant(hq_g, hsc_g, hq_o, hsc_o, h64, bound):
    """MXFP4 activations: X = floor(log2 amax32) - 2 (clamped to [-127, 127],
    -127 for a zero block), E8M0 code X + 127, E2M1 elements of h / 2^X."""
    n, I = h64.shape
    amax32 = np.abs(h64).reshape(n, I // 32, 32).max(axis=2)
    b32 = bound.reshape(n, I // 32, 32).max(axis=2)
    X_g = hsc_g.astype(np.int64) - 127
    # the GPU's exponent must bracket the exact amax, up to the bound at a power of two
    lo = np.ldexp(1.0, X_g + 2)
    hi = np.ldexp(1.0, X_g + 3)
    ok_x = ((amax32 >= lo - b32) & (amax32 < hi + b32)) | ((amax32 <= b32) & (X_g == -127))
    ok_x |= (X_g == -127) & (amax32 < hi + b32)
    ok_x |= (X_g == 127) & (amax32 >= lo - b32)
    scale = np.repeat(np.ldexp(1.0, X_g), 32, axis=1)
    v = h64 / scale
    tol = bound / scale + 4 * 2.0 ** -24 * np.abs(v)
    q_g = _unpack(hq_g, I)
    bad = _grid_check(v, q_g, lambda c: E2M1_VALUES[np.asarray(c) & 15], lambda c: _signed_rank(c, 7),
                      e2m1_nearest, tol)
    return CodeReport(agreement=float((hq_g == hq_o).mean()), block_agreement=float((hsc_g == hsc_o).mean()),
                      violations=int(bad.sum()), block_violations=int((~ok_x).sum()))


# Bounds the tests hold the GPU to.  Measured on B200 over the small parity
# shapes and H = 7168 / I = 2048 decode shapes of every format: code
# agreement >= 0.99998, requantisation scales within 7.5e-7 relative, and no
# code off the midpoint rule.
MIN_AGREEMENT = 0.9995
SCALE_RTOL = 1e-5


def check_mxfp8_requant(hq_g, hsc_g, hq_o, hsc_o, h64, bound):
    """MXFP8 activations: X = floor(log2 amax32) - 8 (clamped to [-127, 127],
    -127 for a zero block), E8M0 code X + 127, E4M3 elements of h / 2^X."""
    n, I = h64.shape
    amax32 = np.abs(h64).reshape(n, I // 32, 32).max(axis=2)
    b32 = bound.reshape(n, I // 32, 32).max(axis=2)
    X_g = hsc_g.astype(np.int64) - 127
    lo = np.ldexp(1.0, X_g + 8)
    hi = np.ldexp(1.0, X_g + 9)
    ok_x = ((amax32 >= lo - b32) & (amax32 < hi + b32)) | ((X_g == -127) & (amax32 < hi + b32))
    scale = np.repeat(np.ldexp(1.0, X_g), 32, axis=1)
    v = h64 / scale
    tol = bound / scale + 4 * 2.0 ** -24 * np.abs(v)
    bad = _grid_check(v, hq_g, e4m3_values, lambda c: _signed_rank(c, 0x7F), e4m3_nearest, tol)
    return CodeReport(agreement=float((hq_g == hq_o).mean()), block_agreement=float((hsc_g == hsc_o).mean()),
                      violations=int(bad.sum()), block_violations=int((~ok_x).sum()))


def check_requant(L, layer, ref, positions=None):
    """Runs the check of L's format on the routing positions `positions` (all
    by default) of the last forward of `layer`.  `ref` holds the oracle's
    debug outputs for the same positions (its routing order equals the
    GPU's, bit for bit), or None to check against the fp64 recomputation
    alone.  Returns the CodeReport."""
    T = L.T
    _, offsets, perm, _ = layer.routing(T)
    tok, grp = position_map(perm, offsets, T, L.k)
    P = len(tok)
    pos = np.arange(P) if positions is None else np.asarray(positions)
    _, _, hq, hs = layer.activations(T)
    h64, bound = swiglu64(L, tok[pos], grp[pos])
    if ref is None:
        # no oracle codes: compare the GPU with itself for the agreement fields
        ref = dict(hq=hq, hs=hs)
        if L.wfmt in (2, 3, 4):
            ref["hsc"] = layer.block_scales(T)[1]
    if L.wfmt in (0, 1):
        return check_fp8_requant(hq[pos], hs[pos], ref["hq"][pos], ref["hs"][pos], h64, bound)
    _, hsc = layer.block_scales(T)
    if L.wfmt == 4:
        return check_mxfp8_requant(hq[pos], hsc[pos], ref["hq"][pos], ref["hsc"][pos], h64, bound)
    if L.wfmt == 2:
        return check_nvfp4_requant(hq[pos], hsc[pos], hs[pos], ref["hq"][pos], ref["hsc"][pos], ref["hs"][pos],
                                   h64, bound)
    return check_mxfp4_requant(hq[pos], hsc[pos], ref["hq"][pos], ref["hsc"][pos], h64, bound)


def edge_positions(layer, L, n_experts: int, seed: int = 0):
    """The first and last routing position of n_experts touched experts (the
    shared expert always among them when there is one), for checks at full
    size where the fp64 recomputation of every position would take too long."""
    counts, offsets, _, _ = layer.routing(L.T)
    touched = np.nonzero(counts > 0)[0]
    rng = np.random.default_rng(seed)
    pick = rng.choice(touched, min(n_experts, len(touched)), replace=False)
    if L.n_shared:
        pick = np.unique(np.append(pick, len(counts) - 1))
    return np.unique(np.concatenate([offsets[pick], offsets[pick + 1] - 1]))


def assert_requant(rep: CodeReport, what: str = ""):
    """The bounds above: no violation of the midpoint rule, agreement with the
    oracle's codes and scales within the measured summation-order effect."""
    print(f"{what}: requant codes {dict(rep)}")
    assert rep["violations"] == 0, (what, dict(rep))
    assert rep.get("block_violations", 0) == 0, (what, dict(rep))
    assert rep.get("scale_violations", 0) == 0, (what, dict(rep))
    assert rep["agreement"] >= MIN_AGREEMENT, (what, dict(rep))
    assert rep.get("block_agreement", 1.0) >= MIN_AGREEMENT, (what, dict(rep))
    assert rep.get("max_scale_rel", 0.0) <= SCALE_RTOL, (what, dict(rep))
