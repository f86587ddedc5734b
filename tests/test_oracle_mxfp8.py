"""Pins for the oracle's MXFP8 path (E4M3 weights and activations, one E8M0
scale per 32 elements along K on both operands), checked against things
other than itself.

OCP MX v1.0 conversion with E4M3 elements: shared exponent
X = floor(log2 amax32) - 8 (8 = the largest E4M3 exponent; E8M0 code X + 127,
clamped to [-127, 127]), elements e4m3(v / 2^X), saturating at 448.
- the exponent rule in closed form for amax in [2^j, 2^(j+1)) and at the clamps;
- groups of representable values round-trip exactly (fixes the block index,
  the exponent and the code order);
- the per-element error bound (half an E4M3 step, or saturation above 448);
- codes bit-equal to an independent restatement (numpy frexp, torch's cast);
- the layer against the fp64 restatement, the dense-FFN reduction,
  linearity in the combine weights, zero input.
"""
import numpy as np
import pytest
import torch

import oracle
from fp4_block_scaled_route_b200 import synth
from tests import dense_ref

WFMT = 4


@pytest.mark.parametrize("j", [-149, -140, -127, -119, -118, -20, -1, 0, 1, 7, 20, 100, 126, 127])
def test_exponent_rule_closed_form(j):
    # amax anywhere in [2^j, 2^(j+1)) gives X = j - 8, clamped to [-127, 127]
    for frac in (1.0, 1.25, 1.999):
        a = np.float32(np.ldexp(frac, j))
        if not np.isfinite(a) or a == 0:
            continue
        v = np.zeros(32, np.float32)
        v[7] = -a
        _, sc = oracle.quant_row_mxfp8(v)
        X = int(np.clip(j - 8, -127, 127))
        assert sc[0] == X + 127, (j, frac, sc[0])


def test_zero_block_and_clamps():
    q, sc = oracle.quant_row_mxfp8(np.zeros(64, np.float32))
    assert sc.tolist() == [0, 0] and not (q & 0x7F).any()
    big = np.full(32, 3.0e38, np.float32)           # floor(log2) = 127 -> X = 119
    q, sc = oracle.quant_row_mxfp8(big)
    # 3.0e38 / 2^119 = 451.4: above the largest element, so it saturates to 448 (code 0x7E)
    assert sc[0] == 119 + 127 and (q == 0x7E).all()


def test_representable_groups_roundtrip_exactly():
    rng = np.random.default_rng(14)
    for _ in range(50):
        X = int(rng.integers(-110, 110))
        codes = rng.integers(0, 256, 32).astype(np.uint8)
        codes = np.where((codes & 0x7F) == 0x7F, codes & 0xF8, codes).astype(np.uint8)  # no NaN codes
        # the group's largest magnitude in [256, 448] (exponent field 15): floor(log2 amax) = X + 8
        big = np.uint8(0x78 + int(rng.integers(0, 7)))
        codes[rng.integers(0, 32)] = big | np.uint8(rng.integers(0, 2) << 7)
        vals = dense_ref.e4m3_values(codes)
        codes = np.where(np.abs(vals) > 448, 0, codes).astype(np.uint8)
        v = (dense_ref.e4m3_values(codes) * np.ldexp(1.0, X)).astype(np.float32)
        q, sc = oracle.quant_row_mxfp8(v)
        assert sc[0] == X + 127
        nz = (codes & 0x7F) != 0
        assert np.array_equal(q[nz], codes[nz])
        assert np.array_equal(dense_ref.e4m3_values(q) * np.ldexp(1.0, X), v.astype(np.float64))


def test_error_bound():
    rng = np.random.default_rng(15)
    v = (rng.standard_normal(8192) * np.exp(rng.uniform(-8, 8, 8192))).astype(np.float32)
    q, sc = oracle.quant_row_mxfp8(v)
    s = np.repeat(np.ldexp(1.0, sc.astype(np.int64) - 127), 32)
    deq = dense_ref.e4m3_values(q) * s
    r = np.abs(v.astype(np.float64)) / s
    e = np.floor(np.log2(np.maximum(r, 2.0 ** -6)))
    step = np.ldexp(1.0, (e - 3).astype(np.int64))         # 3 mantissa bits; subnormals step 2^-9
    bound = np.where(r <= 448, 0.5 * step * s, (r - 448) * s) * (1 + 1e-9)
    assert (np.abs(deq - v) <= bound).all()
    assert (r < 512).all()                                  # amax / 2^X < 512 by the exponent rule


def test_codes_match_independent_restatement():
    gen = torch.Generator().manual_seed(16)
    x = synth.make_x(9, 512, gen, "cpu")
    x[3, 64:96] = 0
    x[5, 128:160] *= 1e-30                                    # tiny values: the lower clamp region
    xq, xsc = oracle.quant_act_mxfp8(synth.bf16_bits(x))
    _, _, q, c = dense_ref.quant_mxfp8(x.float().numpy())
    assert np.array_equal(xsc, c)
    nz = (q & 0x7F) != 0                                      # a zero may keep or drop its sign
    assert np.array_equal(xq[nz], q[nz]) and not (xq[~nz] & 0x7F).any()
    assert xsc[3, 2] == 0


def _tiny(nsh, T=3, H=256, I=256, E=4, k=2, seed=17):
    cfg = dict(T=T, H=H, I=I, E=E, k=k, wfmt=WFMT, n_shared=nsh, routing="uniform")
    return synth.make_layer(cfg, seed)


def _run(L, ids, w=None, x=None, **kw):
    return oracle.forward(synth.bf16_bits(L.x if x is None else x), ids,
                          L.topk_w.numpy() if w is None else w,
                          L.w13.numpy(), L.s13.numpy(), L.w2.numpy(), L.s2.numpy(),
                          H=L.H, I=L.I, E=L.E, wfmt=WFMT, n_shared=L.n_shared, **kw)


def _close(a, b, rel):
    scale = np.abs(b).max()
    err = np.abs(a - b).max()
    cos = float((a * b).sum() / (np.linalg.norm(a) * np.linalg.norm(b)))
    return err <= rel * scale, err / scale, cos


@pytest.mark.parametrize("nsh", [0, 1])
def test_layer_matches_fp64_brute_force(nsh):
    L = _tiny(nsh)
    ids = np.array([[0, 2], [1, 1], [2, 0]], np.int32)
    got = _run(L, ids)["out_f32"].astype(np.float64)
    ref = dense_ref.moe_layer(synth.bf16_bits(L.x), ids, L.topk_w.numpy(), L.w13.numpy(), L.s13.numpy(),
                              L.w2.numpy(), L.s2.numpy(), H=L.H, I=L.I, E=L.E, wfmt=WFMT, n_shared=nsh)
    ok, rel, cos = _close(got, ref, 2e-5)
    assert ok and cos > 1 - 1e-9, (rel, cos)


def test_one_expert_weight_one_is_dense_ffn():
    L = _tiny(0, T=6, H=384, I=256, E=2, k=1, seed=21)
    ids = np.zeros((6, 1), np.int32)
    w = np.ones((6, 1), np.float32)
    got = _run(L, ids, w=w)["out_f32"].astype(np.float64)
    xd, xs = dense_ref.quant_mxfp8((synth.bf16_bits(L.x).astype(np.uint32) << 16).view(np.float32))[:2]
    ref = dense_ref.expert_ffn(xd, xs, L.w13.numpy()[0], L.s13.numpy()[0], L.w2.numpy()[0], L.s2.numpy()[0],
                               WFMT, L.H, L.I)
    ok, rel, cos = _close(got, ref, 2e-5)
    assert ok and cos > 1 - 1e-9, (rel, cos)


def test_linear_in_combine_weights_and_zero_input():
    L = _tiny(1)
    ids = L.ids.numpy()
    w = L.topk_w.numpy()
    a = _run(L, ids, w=w)
    b = _run(L, ids, w=2 * w)
    sh = _run(L, ids, w=np.zeros_like(w))["out_f32"]
    assert np.allclose(b["out_f32"] - sh, 2 * (a["out_f32"] - sh), rtol=0, atol=1e-6 * np.abs(a["out_f32"]).max())
    z = _run(L, ids, x=torch.zeros_like(L.x), debug=True)
    assert not z["out_f32"].any() and not z["xsc"].any() and not z["hsc"].any()


def test_planted_mistakes_fail_the_pins():
    """A copy of the exponent rule with the wrong offset, or a wrong block
    index, is caught by the pins above (checked here on the restatement)."""
    rng = np.random.default_rng(18)
    v = (rng.standard_normal(256) * 0.1).astype(np.float32)
    q, sc = oracle.quant_row_mxfp8(v)
    _, _, _, c = dense_ref.quant_mxfp8(v[None, :])
    assert np.array_equal(sc, c[0])
    assert not np.array_equal(sc, c[0] + 1)                 # an offset of 7 instead of 8
    assert not np.array_equal(sc, np.roll(c[0], 1))         # a shifted block index
