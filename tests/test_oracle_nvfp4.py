"""Pins for the oracle's NVFP4 path, checked against things other than itself.

NVFP4 (named on the onnxruntime QMoE offload PR page; definition: NVIDIA's
E2M1 elements + one E4M3 scale per 16 + an fp32 second-level scale):
- E2M1 encoding against brute-force nearest search over the OCP MX table;
- groups whose values are exactly representable round-trip exactly (closed
  form), which fixes the nibble order, the block-scale index and S;
- the encoding error stays within half an E2M1 step of each block;
- zero groups and underflowing blocks;
- the layer against the independent fp64 restatement in tests/dense_ref.py,
  the dense-FFN reduction and linearity in the combine weights.
"""
import numpy as np
import pytest
import torch

import oracle
from fp4_block_scaled_route_b200 import synth
from tests import dense_ref

E2M1_POS = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


# ---- E2M1 encoding -----------------------------------------------------------
def test_e2m1_encode_matches_brute_force_nearest():
    rng = np.random.default_rng(0)
    grid = np.concatenate([
        np.linspace(-8, 8, 20001, dtype=np.float32),
        rng.standard_normal(20000).astype(np.float32) * 3,
        np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, 7.0, 1e30, -0.0, 0.0], np.float32),
    ])
    grid = np.concatenate([grid, -grid])
    assert np.array_equal(oracle.e2m1_encode(grid), dense_ref.e2m1_nearest(grid))


def test_e2m1_encode_midpoints_and_saturation():
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    # ties go to the neighbour whose code is even (mantissa bit 0)
    assert oracle.e2m1_encode(mids).tolist() == [0x0, 0x2, 0x2, 0x4, 0x4, 0x6, 0x6]
    assert oracle.e2m1_encode([6.0, 6.5, 7.0, 100.0, np.inf]).tolist() == [7] * 5
    assert oracle.e2m1_encode([-100.0, -0.1, -0.0]).tolist() == [0xF, 0x8, 0x8]


def test_e2m1_encode_roundtrips_every_code():
    codes = np.arange(16, dtype=np.uint8)
    assert np.array_equal(oracle.e2m1_encode(oracle.e2m1_decode(codes)), codes)


# ---- NVFP4 row quantisation ------------------------------------------------------
def _representable_group(rng):
    """128 values exactly representable as e2m1 * e4m3 * S with S = 1: every
    16-block has a chosen E4M3 scale c and a maximum element of 6 * c, and the
    first block's scale is 448, so amax128 = 2688."""
    e4m3 = oracle.e4m3_decode(np.arange(0x08, 0x7F, dtype=np.uint8))   # normal positive values
    v = np.empty(128, np.float32)
    codes = np.empty(128, np.uint8)
    scales = np.empty(8, np.float32)
    for b in range(8):
        c = 448.0 if b == 0 else float(rng.choice(e4m3))
        q = rng.integers(0, 16, 16).astype(np.uint8)
        q[rng.integers(0, 16)] = 0x7 if rng.random() < 0.5 else 0xF     # block maximum 6c
        codes[b * 16:(b + 1) * 16] = q
        scales[b] = c
        v[b * 16:(b + 1) * 16] = oracle.e2m1_decode(q) * np.float32(c)
    return v, codes, scales


def _unpack(q, K):
    return dense_ref.unpack_e2m1(q, K)


def test_representable_groups_roundtrip_exactly():
    rng = np.random.default_rng(1)
    for _ in range(20):
        v, codes, scales = _representable_group(rng)
        for mult in (1.0, 2.0 ** -20, 2.0 ** 10):                      # S scales exactly by powers of two
            q, sc, s = oracle.quant_row_nvfp4((v * mult).astype(np.float32))
            assert s[0] == np.float32(mult)
            assert np.array_equal(oracle.e4m3_decode(sc), scales)
            got = _unpack(q, 128)
            # -0 may come back as +0 where the value is zero; compare values and
            # the codes of every nonzero element
            nz = (codes & 7) != 0
            assert np.array_equal(got[nz], codes[nz])
            deq = oracle.e2m1_decode(got) * np.repeat(oracle.e4m3_decode(sc), 16) * s[0]
            assert np.array_equal(deq, v * np.float32(mult))


def test_nibble_order_and_block_index():
    # one nonzero element at column c: byte c // 2, nibble c % 2; block c // 16
    for c in (0, 1, 17, 126, 127):
        v = np.zeros(128, np.float32)
        v[c] = 3.0
        q, sc, s = oracle.quant_row_nvfp4(v)
        byte, nib = divmod(c, 2)
        assert q[byte] == (0x7 << (4 * nib)) and np.count_nonzero(q) == 1
        assert np.count_nonzero(sc) == 1 and oracle.e4m3_decode(sc[c // 16]) == 448.0
        assert s[0] == np.float32(3.0) / np.float32(2688.0)


def test_encoding_error_is_within_half_a_step():
    rng = np.random.default_rng(2)
    v = (rng.standard_normal(4096) * np.exp(rng.uniform(-3, 3, 4096))).astype(np.float32)
    q, sc, s = oracle.quant_row_nvfp4(v)
    d = (np.repeat(oracle.e4m3_decode(sc).astype(np.float64), 16)
         * np.repeat(s.astype(np.float64), 128))
    deq = oracle.e2m1_decode(_unpack(q, 4096)).astype(np.float64) * d
    r = np.abs(v.astype(np.float64)) / d
    # spacing of the E2M1 grid around |v|/d: 0.5 below 2, 1 in [2, 4), 2 above;
    # beyond 6 (block scale rounded down) the value saturates at 6
    step = np.where(r < 2, 0.5, np.where(r < 4, 1.0, 2.0))
    bound = np.where(r <= 6, 0.5 * step * d * (1 + 1e-6), (r - 6) * d * (1 + 1e-6))
    assert (np.abs(deq - v) <= bound).all()
    # block scales stay within the E4M3 range and S within a rounding of amax/2688
    assert oracle.e4m3_decode(sc).max() <= 448.0
    amax = np.abs(v).reshape(-1, 128).max(axis=1)
    assert np.array_equal(s, (amax / np.float32(2688.0)).astype(np.float32))


def test_zero_group_and_underflowing_block():
    v = np.zeros(256, np.float32)
    v[128] = 1000.0                          # group 1: one huge value ...
    v[144:160] = 1e-9                        # ... and a block whose scale underflows to code 0
    q, sc, s = oracle.quant_row_nvfp4(v)
    assert s[0] == 1.0 and not q[:64].any() and not sc[:8].any()       # all-zero group
    assert sc[9] == 0 and not q[72:80].any()                           # underflowed block stores zeros
    assert oracle.e2m1_decode(_unpack(q[64:65], 2))[0] == 6.0


def test_quant_act_nvfp4_matches_independent_restatement():
    gen = torch.Generator().manual_seed(3)
    x = synth.make_x(7, 512, gen, "cpu")
    x[2, 128:256] = 0
    xq, xsc, xs = oracle.quant_act_nvfp4(synth.bf16_bits(x))
    vals, S, q, c = dense_ref.quant_nvfp4(x.float().numpy())
    assert np.array_equal(xs, S)
    assert np.array_equal(xsc, c)
    assert np.array_equal(_unpack(xq, 512), q)


# ---- the layer ---------------------------------------------------------------
def _tiny(nsh, T=3, H=256, I=256, E=4, k=2, seed=7):
    cfg = dict(T=T, H=H, I=I, E=E, k=k, wfmt=2, n_shared=nsh, routing="uniform")
    return synth.make_layer(cfg, seed)


def _run(L, ids, w=None, x=None, **kw):
    return oracle.forward(synth.bf16_bits(L.x if x is None else x), ids,
                          L.topk_w.numpy() if w is None else w,
                          L.w13.numpy(), L.s13.numpy(), L.w2.numpy(), L.s2.numpy(),
                          H=L.H, I=L.I, E=L.E, wfmt=2, n_shared=L.n_shared,
                          g13=L.g13.numpy(), g2=L.g2.numpy(), **kw)


def _close(a, b, rel):
    scale = np.abs(b).max()
    err = np.abs(a - b).max()
    cos = float((a * b).sum() / (np.linalg.norm(a) * np.linalg.norm(b)))
    return err <= rel * scale, err / scale, cos


@pytest.mark.parametrize("nsh", [0, 1])
def test_layer_matches_fp64_brute_force(nsh):
    L = _tiny(nsh)
    ids = np.array([[0, 2], [1, 1], [2, 0]], np.int32)      # duplicate id, expert 3 empty
    got = _run(L, ids)["out_f32"].astype(np.float64)
    ref = dense_ref.moe_layer(synth.bf16_bits(L.x), ids, L.topk_w.numpy(), L.w13.numpy(), L.s13.numpy(),
                              L.w2.numpy(), L.s2.numpy(), H=L.H, I=L.I, E=L.E, wfmt=2, n_shared=nsh,
                              g13=L.g13.numpy(), g2=L.g2.numpy())
    ok, rel, cos = _close(got, ref, 2e-5)
    assert ok and cos > 1 - 1e-9, (rel, cos)


def test_one_expert_weight_one_is_dense_ffn():
    L = _tiny(0, T=6, H=384, I=256, E=2, k=1, seed=11)
    ids = np.zeros((6, 1), np.int32)
    w = np.ones((6, 1), np.float32)
    got = _run(L, ids, w=w)["out_f32"].astype(np.float64)
    xd, xs = dense_ref.quant_nvfp4((synth.bf16_bits(L.x).astype(np.uint32) << 16).view(np.float32))[:2]
    ref = dense_ref.expert_ffn(xd, xs, L.w13.numpy()[0], L.s13.numpy()[0], L.w2.numpy()[0], L.s2.numpy()[0],
                               2, L.H, L.I, L.g13.numpy()[0], L.g2.numpy()[0])
    ok, rel, cos = _close(got, ref, 2e-5)
    assert ok and cos > 1 - 1e-9, (rel, cos)


def test_linear_in_combine_weights_and_global_scales():
    L = _tiny(0)
    ids = L.ids.numpy()
    w = L.topk_w.numpy()
    a = _run(L, ids, w=w)
    b = _run(L, ids, w=2 * w)
    assert np.array_equal(b["out_f32"], 2 * a["out_f32"])
    # doubling the GEMM2 global scales doubles the output exactly (powers of two)
    L2 = synth.Layer(**{**L.__dict__, "g2": L.g2 * 2})
    assert np.array_equal(_run(L2, ids)["out_f32"], 2 * a["out_f32"])


def test_zero_input_gives_zero_output():
    L = _tiny(1)
    r = _run(L, L.ids.numpy(), x=torch.zeros_like(L.x), debug=True)
    assert not r["out_f32"].any()
    assert (r["xs"] == 1.0).all() and (r["hs"] == 1.0).all()
    assert not r["xsc"].any() and not r["hsc"].any()


def test_debug_outputs_match_row_quantiser():
    L = _tiny(1)
    r = _run(L, L.ids.numpy(), debug=True)
    xq, xsc, xs = oracle.quant_act_nvfp4(synth.bf16_bits(L.x))
    assert np.array_equal(r["xq"], xq) and np.array_equal(r["xsc"], xsc) and np.array_equal(r["xs"], xs)
    assert r["hq"].shape == (3 * 2 + 3, L.I // 2) and r["hsc"].shape == (9, L.I // 16)


def test_quantisation_error_is_fp4_sized():
    # informational: W4A4 NVFP4 against the unquantised layer is well under 30 %
    L = _tiny(0, T=4, H=512, I=256, E=4, k=2, seed=5)
    ids = L.ids.numpy()
    got = _run(L, ids)["out_f32"].astype(np.float64)
    x = (synth.bf16_bits(L.x).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    out = np.zeros_like(got)
    for t in range(L.T):
        for j in range(L.k):
            e = int(ids[t, j])
            W13 = dense_ref.dequant_weights(L.w13.numpy()[e], L.s13.numpy()[e], 2, L.H) * float(L.g13[e])
            W2 = dense_ref.dequant_weights(L.w2.numpy()[e], L.s2.numpy()[e], 2, L.I) * float(L.g2[e])
            G = W13 @ x[t]
            h = G[:L.I] / (1 + np.exp(-G[:L.I])) * G[L.I:]
            out[t] += float(L.topk_w[t, j]) * (W2 @ h)
    rel = np.linalg.norm(got - out) / np.linalg.norm(out)
    assert 1e-3 < rel < 0.3, rel
