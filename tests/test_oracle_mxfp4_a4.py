"""Pins for the oracle's MXFP4-activation path (MXFP4 weights x MXFP4
activations), checked against things other than itself.

OCP MX v1.0 conversion with E2M1 elements: shared exponent
X = floor(log2 amax32) - 2 (E8M0 code X + 127, clamped to [-127, 127]),
elements e2m1(v / 2^X).
- the exponent rule in closed form for amax in [2^j, 2^(j+1)) and at the clamps;
- groups of representable values round-trip exactly (fixes nibble order,
  block index and exponent);
- the per-element error bound (half an E2M1 step, or saturation above 6);
- codes bit-equal to an independent numpy restatement (frexp, brute force);
- the layer against the fp64 restatement, the dense-FFN reduction,
  linearity in the combine weights, zero input.
"""
import numpy as np
import pytest
import torch

import oracle
from fp4_block_scaled_route_b200 import synth
from tests import dense_ref


def _unpack(q, K):
    return dense_ref.unpack_e2m1(q, K)


@pytest.mark.parametrize("j", [-130, -127, -126, -20, -1, 0, 1, 7, 20, 100, 126, 127])
def test_exponent_rule_closed_form(j):
    # amax anywhere in [2^j, 2^(j+1)) gives X = j - 2 (clamped to [-127, 127])
    for frac in (1.0, 1.25, 1.999):
        a = np.float32(np.ldexp(frac, j))
        if not np.isfinite(a) or a == 0:
            continue
        v = np.zeros(32, np.float32)
        v[5] = -a
        q, sc = oracle.quant_row_mxfp4(v)
        X = int(np.clip(j - 2, -127, 127))
        if j < -126:  # a subnormal: floor(log2 a) is still j
            X = -127
        assert sc[0] == X + 127, (j, frac, sc[0])


def test_zero_block_and_clamps():
    q, sc = oracle.quant_row_mxfp4(np.zeros(64, np.float32))
    assert sc.tolist() == [0, 0] and not q.any()
    big = np.full(32, 3.0e38, np.float32)           # floor(log2) = 127 -> X = 125
    q, sc = oracle.quant_row_mxfp4(big)
    # 3.0e38 / 2^125 = 7.05: above the largest element, so it saturates to 6 (code 7)
    assert sc[0] == 125 + 127 and (_unpack(q, 32) == 7).all()


def test_representable_groups_roundtrip_exactly():
    rng = np.random.default_rng(4)
    for _ in range(50):
        X = int(rng.integers(-120, 120))
        codes = rng.integers(0, 16, 32).astype(np.uint8)
        codes[rng.integers(0, 32)] = rng.choice([0x6, 0x7, 0xE, 0xF])  # max |e2m1| in {4, 6}: floor(log2) = X + 2
        v = (oracle.e2m1_decode(codes).astype(np.float64) * np.ldexp(1.0, X)).astype(np.float32)
        q, sc = oracle.quant_row_mxfp4(v)
        assert sc[0] == X + 127
        got = _unpack(q, 32)
        nz = (codes & 7) != 0
        assert np.array_equal(got[nz], codes[nz])
        assert np.array_equal(oracle.e2m1_decode(got) * np.float32(np.ldexp(1.0, X)), v)


def test_error_bound():
    rng = np.random.default_rng(5)
    v = (rng.standard_normal(4096) * np.exp(rng.uniform(-6, 6, 4096))).astype(np.float32)
    q, sc = oracle.quant_row_mxfp4(v)
    s = np.repeat(np.ldexp(1.0, sc.astype(np.int64) - 127), 32)
    deq = oracle.e2m1_decode(_unpack(q, 4096)).astype(np.float64) * s
    r = np.abs(v.astype(np.float64)) / s
    step = np.where(r < 2, 0.5, np.where(r < 4, 1.0, 2.0))
    bound = np.where(r <= 6, 0.5 * step * s, (r - 6) * s) * (1 + 1e-9)
    assert (np.abs(deq - v) <= bound).all()
    assert (r < 8).all()                             # amax / 2^X < 8 by the exponent rule


def test_codes_match_independent_restatement():
    gen = torch.Generator().manual_seed(6)
    x = synth.make_x(9, 512, gen, "cpu")
    x[3, 64:96] = 0
    xq, xsc = oracle.quant_act_mxfp4(synth.bf16_bits(x))
    vals, ones, q, c = dense_ref.quant_mxfp4(x.float().numpy())
    assert np.array_equal(xsc, c)
    assert np.array_equal(_unpack(xq, 512), q)
    assert xsc[3, 2] == 0


def _tiny(nsh, T=3, H=256, I=256, E=4, k=2, seed=7):
    cfg = dict(T=T, H=H, I=I, E=E, k=k, wfmt=3, n_shared=nsh, routing="uniform")
    return synth.make_layer(cfg, seed)


def _run(L, ids, w=None, x=None, **kw):
    return oracle.forward(synth.bf16_bits(L.x if x is None else x), ids,
                          L.topk_w.numpy() if w is None else w,
                          L.w13.numpy(), L.s13.numpy(), L.w2.numpy(), L.s2.numpy(),
                          H=L.H, I=L.I, E=L.E, wfmt=3, n_shared=L.n_shared, **kw)


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
                              L.w2.numpy(), L.s2.numpy(), H=L.H, I=L.I, E=L.E, wfmt=3, n_shared=nsh)
    ok, rel, cos = _close(got, ref, 2e-5)
    assert ok and cos > 1 - 1e-9, (rel, cos)


def test_one_expert_weight_one_is_dense_ffn():
    L = _tiny(0, T=6, H=384, I=256, E=2, k=1, seed=11)
    ids = np.zeros((6, 1), np.int32)
    w = np.ones((6, 1), np.float32)
    got = _run(L, ids, w=w)["out_f32"].astype(np.float64)
    xd, xs = dense_ref.quant_mxfp4((synth.bf16_bits(L.x).astype(np.uint32) << 16).view(np.float32))[:2]
    ref = dense_ref.expert_ffn(xd, xs, L.w13.numpy()[0], L.s13.numpy()[0], L.w2.numpy()[0], L.s2.numpy()[0],
                               3, L.H, L.I)
    ok, rel, cos = _close(got, ref, 2e-5)
    assert ok and cos > 1 - 1e-9, (rel, cos)


def test_linear_in_combine_weights_and_zero_input():
    L = _tiny(1)
    ids = L.ids.numpy()
    w = L.topk_w.numpy()
    a = _run(L, ids, w=w)
    b = _run(L, ids, w=2 * w)
    # the shared expert enters at weight 1: the routed part doubles exactly
    sh = _run(L, ids, w=np.zeros_like(w))["out_f32"]
    assert np.allclose(b["out_f32"] - sh, 2 * (a["out_f32"] - sh), rtol=0, atol=1e-6 * np.abs(a["out_f32"]).max())
    z = _run(L, ids, x=torch.zeros_like(L.x), debug=True)
    assert not z["out_f32"].any() and not z["xsc"].any() and not z["hsc"].any()
