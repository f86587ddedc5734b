"""Seeded synthetic inputs for the MoE layer.

This module is shared by the CUDA path's tests/benchmark and by the CPU
oracle's tests: both sides receive the very same bytes.  It holds none of the
layer's own arithmetic (no routing, activation quantisation, GEMM, SwiGLU or
combine).  It only draws random numbers and stores the expert weights in the
layer's input formats, using torch library casts (``float8_e4m3fn``) and a
rounding-to-grid helper for E2M1.

Workloads (the layer shapes of the pages' decode benchmarks, with seeded
synthetic data standing in for the model layers, which are not available):

==  =========================================  =====  =====  ===  ==  =====  ======
#   name                                        T      H      E    k   I      wfmt
==  =========================================  =====  =====  ===  ==  =====  ======
0   tiny                                        4      256    8    2   128    fp8
1   decode, FP8                                 32     7168   256  8   2048   fp8
2   decode, MXFP4                               128    7168   256  8   2048   mxfp4
3   skewed decode + shared expert (Zipf 1.2)    8      4096   160  8   1536   fp8
4   prefill                                     4096   7168   256  8   2048   fp8
==  =========================================  =====  =====  ===  ==  =====  ======

Recipe: x ~ N(0,1) rounded to bf16; expert ids k distinct per token, uniform
without replacement (config 3: sequential draws without replacement from a
Zipf(s=1.2) popularity over a seeded permutation of the experts); combine
weights = softmax over the k chosen of N(0,1) logits (fp32); expert weights
~ N(0, 0.02), stored as FP8 E4M3 with one fp32 scale amax/448 per 128x128
block, or as MXFP4 (E2M1 nibbles, element 2c in the low nibble, one E8M0
scale per 32 elements along K with exponent floor(log2 amax) - 2), or as
MXFP8 (E4M3 codes, one E8M0 scale per 32 elements along K with exponent
floor(log2 amax) - 8, elements saturated at 448), or as
NVFP4 (the same nibbles, one E4M3 scale per 16 elements along K and one fp32
global scale per expert matrix: g = amax / (448 * 6), block scale
e4m3(amax16 / 6 / g), element e2m1(w / (block scale * g))).

The NVFP4 decode workloads and an MXFP4-weights-and-activations workload
use the decode shapes, and an MXFP8 workload the prefill shape (not rows of
the table), in ``EXTRA_CONFIGS``.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np
import torch

WFMT_FP8 = 0
WFMT_MXFP4 = 1
WFMT_NVFP4 = 2
WFMT_MXFP4_A4 = 3  # MXFP4 weights (the WFMT_MXFP4 bytes) with MXFP4 activations
WFMT_MXFP8 = 4     # MXFP8: E4M3 weights and activations, E8M0 scale per 32 along K

CONFIGS = [
    dict(name="tiny_T4_H256_E8_k2_I128_fp8", T=4, H=256, E=8, k=2, I=128,
         wfmt=WFMT_FP8, routing="uniform", n_shared=0),
    dict(name="decode_T32_H7168_E256_k8_I2048_fp8", T=32, H=7168, E=256, k=8, I=2048,
         wfmt=WFMT_FP8, routing="uniform", n_shared=0),
    dict(name="decode_T128_H7168_E256_k8_I2048_mxfp4", T=128, H=7168, E=256, k=8, I=2048,
         wfmt=WFMT_MXFP4, routing="uniform", n_shared=0),
    dict(name="zipf_T8_H4096_E160_k8_I1536_fp8_shared", T=8, H=4096, E=160, k=8, I=1536,
         wfmt=WFMT_FP8, routing="zipf1.2", n_shared=1),
    dict(name="prefill_T4096_H7168_E256_k8_I2048_fp8", T=4096, H=7168, E=256, k=8, I=2048,
         wfmt=WFMT_FP8, routing="uniform", n_shared=0),
]


# Workloads beyond the five above: the NVFP4 weight format and MXFP4
# activations on the decode shapes, and the prefill shape in MXFP8.
EXTRA_CONFIGS = [
    dict(name="decode_T128_H7168_E256_k8_I2048_nvfp4", T=128, H=7168, E=256, k=8, I=2048,
         wfmt=WFMT_NVFP4, routing="uniform", n_shared=0),
    dict(name="decode_T32_H7168_E256_k8_I2048_nvfp4", T=32, H=7168, E=256, k=8, I=2048,
         wfmt=WFMT_NVFP4, routing="uniform", n_shared=0),
    dict(name="decode_T128_H7168_E256_k8_I2048_mxfp4_a4", T=128, H=7168, E=256, k=8, I=2048,
         wfmt=WFMT_MXFP4_A4, routing="uniform", n_shared=0),
    dict(name="prefill_T4096_H7168_E256_k8_I2048_mxfp8", T=4096, H=7168, E=256, k=8, I=2048,
         wfmt=WFMT_MXFP8, routing="uniform", n_shared=0),
]


def config_seed(idx: int) -> int:
    return 1000 + idx


# ---------------------------------------------------------------------------
def make_routing(T: int, E: int, k: int, kind: str, seed: int):
    """(ids int32 [T,k], topk_w float32 [T,k])."""
    rng = np.random.default_rng(seed)
    if kind == "uniform":
        keys = rng.random((T, E))
        ids = np.argsort(keys, axis=1, kind="stable")[:, :k]
    elif kind.startswith("zipf"):
        s = float(kind[4:])
        order = rng.permutation(E)                    # expert holding popularity rank r
        pop = (np.arange(E, dtype=np.float64) + 1.0) ** (-s)
        p = np.empty(E)
        p[order] = pop / pop.sum()
        ids = np.stack([rng.choice(E, size=k, replace=False, p=p) for _ in range(T)])
    else:
        raise ValueError(kind)
    logits = rng.standard_normal((T, k))
    ex = np.exp(logits - logits.max(axis=1, keepdims=True))
    w = (ex / ex.sum(axis=1, keepdims=True)).astype(np.float32)
    return ids.astype(np.int32), w


def make_x(T: int, H: int, gen: torch.Generator, device) -> torch.Tensor:
    return torch.randn(T, H, generator=gen, device=device, dtype=torch.float32).to(torch.bfloat16)


def _fp8_block(w: torch.Tensor):
    """w f32 [R, K] -> (codes uint8 [R, K], scales f32 [R/128, K/128])."""
    R, K = w.shape
    blk = w.reshape(R // 128, 128, K // 128, 128)
    amax = blk.abs().amax(dim=(1, 3))
    scale = amax / 448.0
    q = (blk / scale[:, None, :, None]).to(torch.float8_e4m3fn)
    return q.reshape(R, K).view(torch.uint8), scale.to(torch.float32)


_E2M1_MIDS = (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0)


def _e2m1_round(v: torch.Tensor) -> torch.Tensor:
    """Nearest E2M1 code (ties to the even code, magnitude clamped to 6)."""
    mids = torch.tensor(_E2M1_MIDS, dtype=v.dtype, device=v.device)
    a = v.abs()
    idx = torch.bucketize(a, mids)                    # ties land on the lower code
    at_mid = (idx < 7) & (a == mids[idx.clamp(max=6)])
    idx = torch.where(at_mid & (idx % 2 == 1), idx + 1, idx)
    code = idx.to(torch.uint8)
    return torch.where(torch.signbit(v), code | 8, code)


def _mxfp4_group(w: torch.Tensor):
    """w f32 [R, K] -> (packed uint8 [R, K/2], e8m0 uint8 [R, K/32])."""
    R, K = w.shape
    grp = w.reshape(R, K // 32, 32)
    amax = grp.abs().amax(dim=2)
    e = torch.floor(torch.log2(amax)) - 2.0           # OCP MX: emax(E2M1) = 2
    e = e.clamp(-127, 127)
    codes = _e2m1_round(grp / torch.exp2(e)[:, :, None]).reshape(R, K)
    packed = codes[:, 0::2] | (codes[:, 1::2] << 4)
    return packed.contiguous(), (e + 127).to(torch.uint8)


def _mxfp8_group(w: torch.Tensor):
    """w f32 [R, K] -> (E4M3 codes uint8 [R, K], e8m0 uint8 [R, K/32])."""
    R, K = w.shape
    grp = w.reshape(R, K // 32, 32)
    amax = grp.abs().amax(dim=2)
    e = torch.floor(torch.log2(amax)) - 8.0           # OCP MX: emax(E4M3) = 8
    e = e.clamp(-127, 127)
    scaled = (grp / torch.exp2(e)[:, :, None]).clamp(-448.0, 448.0)  # the cast does not saturate
    codes = scaled.to(torch.float8_e4m3fn).view(torch.uint8).reshape(R, K)
    return codes.contiguous(), (e + 127).to(torch.uint8)


def _nvfp4_matrix(w: torch.Tensor):
    """w f32 [R, K] -> (packed uint8 [R, K/2], E4M3 block codes uint8 [R, K/16], g f32 scalar)."""
    R, K = w.shape
    g = w.abs().amax() / 2688.0                       # 2688 = E4M3 max 448 x E2M1 max 6
    blk = w.reshape(R, K // 16, 16)
    amax16 = blk.abs().amax(dim=2)
    sc = ((amax16 / 6.0) / g).clamp(max=448.0).to(torch.float8_e4m3fn)
    d = sc.float() * g
    safe = torch.where(d == 0, torch.ones_like(d), d)
    codes = _e2m1_round(blk / safe[:, :, None])
    codes = torch.where((d == 0)[:, :, None], torch.zeros_like(codes), codes).reshape(R, K)
    packed = codes[:, 0::2] | (codes[:, 1::2] << 4)
    return packed.contiguous(), sc.view(torch.uint8), g.to(torch.float32)


def make_weights_nvfp4(NE: int, rows: int, K: int, gen: torch.Generator, device, std: float = 0.02):
    """NVFP4 expert weights: (packed [NE, rows, K/2], block codes [NE, rows, K/16], g [NE])."""
    w = torch.empty(NE, rows, K // 2, dtype=torch.uint8, device=device)
    s = torch.empty(NE, rows, K // 16, dtype=torch.uint8, device=device)
    g = torch.empty(NE, dtype=torch.float32, device=device)
    for e in range(NE):
        dense = torch.randn(rows, K, generator=gen, device=device, dtype=torch.float32) * std
        w[e], s[e], g[e] = _nvfp4_matrix(dense)
    return w, s, g


def make_weights(NE: int, rows: int, K: int, wfmt: int, gen: torch.Generator, device,
                 std: float = 0.02):
    """Expert weights [NE, rows, K] in the layer's storage format."""
    if wfmt == WFMT_FP8:
        w = torch.empty(NE, rows, K, dtype=torch.uint8, device=device)
        s = torch.empty(NE, rows // 128, K // 128, dtype=torch.float32, device=device)
    elif wfmt == WFMT_MXFP8:
        w = torch.empty(NE, rows, K, dtype=torch.uint8, device=device)
        s = torch.empty(NE, rows, K // 32, dtype=torch.uint8, device=device)
    else:
        w = torch.empty(NE, rows, K // 2, dtype=torch.uint8, device=device)
        s = torch.empty(NE, rows, K // 32, dtype=torch.uint8, device=device)
    for e in range(NE):
        dense = torch.randn(rows, K, generator=gen, device=device, dtype=torch.float32) * std
        if wfmt == WFMT_FP8:
            w[e], s[e] = _fp8_block(dense)
        elif wfmt == WFMT_MXFP8:
            w[e], s[e] = _mxfp8_group(dense)
        else:
            w[e], s[e] = _mxfp4_group(dense)
    return w, s


@dataclasses.dataclass
class Layer:
    T: int
    H: int
    I: int
    E: int
    k: int
    wfmt: int
    n_shared: int
    x: torch.Tensor        # bf16 [T, H]
    ids: torch.Tensor      # int32 [T, k]
    topk_w: torch.Tensor   # float32 [T, k]
    w13: torch.Tensor      # uint8, see module docstring
    s13: torch.Tensor
    w2: torch.Tensor
    s2: torch.Tensor
    g13: Optional[torch.Tensor] = None   # NVFP4: fp32 [NE] global scales of w13
    g2: Optional[torch.Tensor] = None    # NVFP4: fp32 [NE] global scales of w2

    @property
    def S(self) -> int:
        return self.T * self.k

    def host(self) -> "Layer":
        fields = ["x", "ids", "topk_w", "w13", "s13", "w2", "s2"]
        if self.g13 is not None:
            fields += ["g13", "g2"]
        return dataclasses.replace(self, **{f: getattr(self, f).cpu() for f in fields})


def make_layer(cfg: dict, seed: int, device="cpu", T: Optional[int] = None,
               routing: Optional[str] = None) -> Layer:
    """Seeded layer inputs for ``cfg`` (a CONFIGS entry or the same keys)."""
    T = cfg["T"] if T is None else T
    H, I, E, k = cfg["H"], cfg["I"], cfg["E"], cfg["k"]
    wfmt, nsh = cfg["wfmt"], cfg.get("n_shared", 0)
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    x = make_x(T, H, gen, device)
    ids, w = make_routing(T, E, k, routing or cfg.get("routing", "uniform"), seed)
    g13 = g2 = None
    if wfmt == WFMT_NVFP4:
        w13, s13, g13 = make_weights_nvfp4(E + nsh, 2 * I, H, gen, device)
        w2, s2, g2 = make_weights_nvfp4(E + nsh, H, I, gen, device)
    else:
        wf = WFMT_MXFP4 if wfmt == WFMT_MXFP4_A4 else wfmt  # the same MXFP4 weight bytes
        w13, s13 = make_weights(E + nsh, 2 * I, H, wf, gen, device)
        w2, s2 = make_weights(E + nsh, H, I, wf, gen, device)
    return Layer(T, H, I, E, k, wfmt, nsh, x, torch.from_numpy(ids).to(device),
                 torch.from_numpy(w).to(device), w13, s13, w2, s2, g13, g2)


def bf16_bits(x: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> numpy uint16 bit patterns (host)."""
    return x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def make_router(T: int, H: int, E: int, seed: int, device="cpu"):
    """Seeded router inputs: x ~ N(0,1) and router weights ~ N(0, 1/H), both
    rounded to bf16, so that the logits x . Wr^T have about unit variance."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    x = torch.randn(T, H, generator=g).to(torch.bfloat16)
    wr = (torch.randn(E, H, generator=g) / float(np.sqrt(H))).to(torch.bfloat16)
    return x.to(device), wr.to(device)
