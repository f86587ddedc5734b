"""Pins for the CPU oracle, checked against things other than itself.

Codecs against torch's float8 dtype and the OCP tables under tests/golden;
routing against numpy's stable argsort; the layer against an independent
fp64 restatement on tiny shapes (tests/dense_ref.py), against the dense
SwiGLU FFN it must reduce to when every token goes to one expert with weight
1, against linearity in the combine weights and a zero input.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from fp4_block_scaled_route_b200 import synth
from tests import dense_ref

ALL = np.arange(256, dtype=np.uint8)


# ---- codecs ---------------------------------------------------------------
def test_e4m3_decode_matches_torch_dtype():
    ours = oracle.e4m3_decode(ALL)
    ref = torch.from_numpy(ALL.copy()).view(torch.float8_e4m3fn).float().numpy()
    nan = np.isnan(ref)
    assert list(np.nonzero(nan)[0]) == [0x7F, 0xFF]
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan].view(np.uint32), ref[~nan].view(np.uint32))  # incl. -0


def test_e4m3_decode_golden_points():
    tab = dense_ref.load_table("e4m3_ocp_fp8.txt")
    for code, val in tab.items():
        got = float(oracle.e4m3_decode(np.array([code]))[0])
        if math.isnan(val):
            assert math.isnan(got)
        else:
            assert got == val and math.copysign(1, got) == math.copysign(1, val), hex(code)


def _e4m3_probe_values():
    vals = oracle.e4m3_decode(ALL)
    fin = np.sort(np.unique(vals[np.isfinite(vals)]))
    mids = (fin[1:].astype(np.float64) + fin[:-1]) / 2          # exact ties
    rng = np.random.default_rng(0)
    rnd = rng.uniform(-448, 448, 200_000).astype(np.float32)
    small = rng.uniform(-0.02, 0.02, 100_000).astype(np.float32)
    near = np.concatenate([np.nextafter(mids.astype(np.float32), np.float32(np.inf)),
                           np.nextafter(mids.astype(np.float32), np.float32(-np.inf))])
    return np.concatenate([fin, mids.astype(np.float32), near, rnd, small]).astype(np.float32)


def test_e4m3_encode_matches_torch_cast():
    v = _e4m3_probe_values()
    v = v[np.abs(v) <= 448]
    ours = oracle.e4m3_encode(v)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    # torch keeps the sign of a value that rounds to zero; so does the oracle
    assert np.array_equal(ours, ref)


def test_e4m3_encode_saturates_and_roundtrips():
    assert oracle.e4m3_encode(np.float32([449, 500, 1e30, np.inf])).tolist() == [0x7E] * 4
    assert oracle.e4m3_encode(np.float32([-449, -1e30, -np.inf])).tolist() == [0xFE] * 3
    assert oracle.e4m3_encode(np.float32([np.nan]))[0] & 0x7F == 0x7F
    fin = ALL[(ALL & 0x7F) != 0x7F]
    assert np.array_equal(oracle.e4m3_encode(oracle.e4m3_decode(fin)), fin)


def test_e4m3_ties_go_to_even_code():
    # 1.0 (0x38) and 1.125 (0x39): midpoint goes to 0x38; 1.125..1.25 midpoint to 0x3A
    assert oracle.e4m3_encode(np.float32([1.0625, 1.1875, -1.0625])).tolist() == [0x38, 0x3A, 0xB8]
    # binade boundary: 0.875*2^-6 (0x07) .. 2^-6 (0x08); midpoint -> 0x08 (even)
    assert oracle.e4m3_encode(np.float32([0.9375 * 2 ** -6]))[0] == 0x08


def test_e2m1_decode_golden_table():
    ours = oracle.e2m1_decode(np.arange(16, dtype=np.uint8))
    for c in range(16):
        assert ours[c] == dense_ref.E2M1[c] and math.copysign(1, ours[c]) == math.copysign(1, dense_ref.E2M1[c])


def test_e8m0_decode():
    for c in range(255):
        assert oracle.e8m0_decode(c) == math.ldexp(1.0, c - 127)
    assert math.isnan(oracle.e8m0_decode(255))


def test_bf16_roundtrip_matches_torch():
    rng = np.random.default_rng(1)
    v = np.concatenate([rng.standard_normal(50_000).astype(np.float32),
                        (rng.integers(0, 2 ** 16, 5000).astype(np.uint32) << 16 | 0x8000).view(np.float32)])
    v = v[np.isfinite(v)]
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    ours = np.array([oracle.bf16_encode(float(a)) for a in v[:20000]], dtype=np.uint16)
    assert np.array_equal(ours, ref[:20000])
    for b in [0x0000, 0x8000, 0x3F80, 0xC2F7, 0x7F7F]:
        assert oracle.bf16_decode(b) == float(torch.from_numpy(np.array([b], np.uint16).view(np.int16)).view(torch.bfloat16).float())


# ---- step 1: routing --------------------------------------------------------
@pytest.mark.parametrize("T,k,E,nsh", [(1, 1, 1, 0), (5, 3, 4, 0), (64, 8, 256, 0),
                                       (33, 8, 160, 1), (7, 2, 3, 1)])
def test_route_matches_stable_argsort(T, k, E, nsh):
    rng = np.random.default_rng(T * 31 + E)
    ids = rng.integers(0, E, (T, k)).astype(np.int32)   # duplicates allowed
    counts, offsets, perm, inv, dropped = oracle.route(ids, E, nsh)
    S = T * k
    flat = ids.reshape(-1)
    assert dropped == 0
    assert np.array_equal(counts[:E], np.bincount(flat, minlength=E))
    assert offsets[0] == 0 and np.array_equal(np.diff(offsets), counts)
    assert np.array_equal(perm[:S], np.argsort(flat, kind="stable"))
    assert np.array_equal(inv[perm], np.arange(S + nsh * T))        # round trip
    if nsh:
        assert counts[E] == T and np.array_equal(perm[S:], S + np.arange(T))


def test_route_drops_out_of_range_ids():
    ids = np.array([[0, 5], [-1, 1], [1, 2]], dtype=np.int32)
    counts, offsets, perm, inv, dropped = oracle.route(ids, 3)
    assert dropped == 2
    assert counts.tolist() == [1, 2, 1] and offsets.tolist() == [0, 1, 3, 4]
    assert perm[:4].tolist() == [0, 3, 4, 5]
    assert inv.tolist() == [0, -1, -1, 1, 2, 3]


# ---- step 2: activation quantisation ---------------------------------------
def test_quant_act_matches_torch_cast():
    gen = torch.Generator().manual_seed(3)
    x = synth.make_x(9, 512, gen, "cpu")
    x[2, 128:256] = 0                                    # all-zero group -> s = 1
    xq, xs = oracle.quant_act(synth.bf16_bits(x))
    xf = x.float().reshape(9, 4, 128)
    amax = xf.abs().amax(-1)
    s = torch.where(amax == 0, torch.ones_like(amax), amax / 448.0)
    ref = (xf / s[..., None]).to(torch.float8_e4m3fn).view(torch.uint8).reshape(9, 512)
    assert np.array_equal(xs, s.numpy())
    assert np.array_equal(xq, ref.numpy())
    assert xs[2, 1] == 1.0 and not xq[2, 128:256].any()
    # the group maximum maps to +-448 exactly
    assert set(np.unique(np.abs(oracle.e4m3_decode(xq)).max(axis=1))) == {448.0}


# ---- the layer --------------------------------------------------------------
def _tiny(wfmt, nsh, T=3, H=256, I=256, E=4, k=2, seed=7, ids=None):
    cfg = dict(T=T, H=H, I=I, E=E, k=k, wfmt=wfmt, n_shared=nsh, routing="uniform")
    L = synth.make_layer(cfg, seed)
    ids_np = L.ids.numpy() if ids is None else np.asarray(ids, np.int32)
    return L, ids_np


def _run(L, ids, w=None, x=None, **kw):
    return oracle.forward(synth.bf16_bits(L.x if x is None else x), ids,
                          L.topk_w.numpy() if w is None else w,
                          L.w13.numpy(), L.s13.numpy(), L.w2.numpy(), L.s2.numpy(),
                          H=L.H, I=L.I, E=L.E, wfmt=L.wfmt, n_shared=L.n_shared, **kw)


def _close(a, b, rel):
    scale = np.abs(b).max()
    err = np.abs(a - b).max()
    cos = float((a * b).sum() / (np.linalg.norm(a) * np.linalg.norm(b)))
    return err <= rel * scale, err / scale, cos


@pytest.mark.parametrize("wfmt,nsh", [(0, 0), (0, 1), (1, 0), (1, 1)])
def test_layer_matches_fp64_brute_force(wfmt, nsh):
    # duplicate id in token 1, expert 3 empty
    L, ids = _tiny(wfmt, nsh, ids=[[0, 2], [1, 1], [2, 0]])
    got = _run(L, ids)["out_f32"].astype(np.float64)
    ref = dense_ref.moe_layer(synth.bf16_bits(L.x), ids, L.topk_w.numpy(), L.w13.numpy(),
                              L.s13.numpy(), L.w2.numpy(), L.s2.numpy(), H=L.H, I=L.I, E=L.E,
                              wfmt=wfmt, n_shared=nsh)
    ok, rel, cos = _close(got, ref, 2e-5)
    assert ok and cos > 1 - 1e-9, (rel, cos)


def test_one_expert_weight_one_is_dense_ffn():
    # every token to expert 0 with weight 1 (k = 1): a dense SwiGLU FFN over all tokens
    L, _ = _tiny(0, 0, T=6, H=384, I=256, E=2, k=1, seed=11)
    ids = np.zeros((6, 1), np.int32)
    w = np.ones((6, 1), np.float32)
    got = _run(L, ids, w=w)["out_f32"].astype(np.float64)
    xd, xs = dense_ref.quant128((synth.bf16_bits(L.x).astype(np.uint32) << 16).view(np.float32))
    ref = dense_ref.expert_ffn(xd, xs, L.w13.numpy()[0], L.s13.numpy()[0], L.w2.numpy()[0],
                               L.s2.numpy()[0], 0, L.H, L.I)
    ok, rel, cos = _close(got, ref, 2e-5)
    assert ok and cos > 1 - 1e-9, (rel, cos)


@pytest.mark.parametrize("wfmt", [0, 1])
def test_linear_in_combine_weights(wfmt):
    L, ids = _tiny(wfmt, 0)
    w = L.topk_w.numpy()
    a = _run(L, ids, w=w)
    b = _run(L, ids, w=2 * w)
    assert np.array_equal(b["out_f32"], 2 * a["out_f32"])
    c = _run(L, ids, w=np.zeros_like(w))
    assert not c["out_f32"].any()


def test_zero_input_gives_zero_output():
    L, ids = _tiny(0, 1)
    r = _run(L, ids, x=torch.zeros_like(L.x), debug=True)
    assert not r["out_f32"].any() and not r["out_bf16"].any()
    assert (r["xs"] == 1.0).all() and (r["hs"] == 1.0).all()


def test_token_mask_selects_rows():
    L, ids = _tiny(0, 1, T=5)
    full = _run(L, ids)
    part = _run(L, ids, token_mask=[0, 1, 0, 0, 1])
    assert np.array_equal(part["out_f32"][[1, 4]], full["out_f32"][[1, 4]])
    assert np.isnan(part["out_f32"][[0, 2, 3]]).all()


def test_bf16_output_is_rounded_f32():
    L, ids = _tiny(1, 0)
    r = _run(L, ids)
    ref = torch.from_numpy(r["out_f32"]).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(r["out_bf16"], ref)


def test_quantisation_error_is_fp8_sized():
    # informational bound: vs the unquantised layer the error is a few percent
    L, ids = _tiny(0, 0, T=4, H=512, I=256, E=4, k=2, seed=5)
    got = _run(L, ids)["out_f32"].astype(np.float64)
    ref = dense_ref.unquantised_layer(synth.bf16_bits(L.x), ids, L.topk_w.numpy(), L.w13.numpy(),
                                      L.s13.numpy(), L.w2.numpy(), L.s2.numpy(), H=L.H, I=L.I,
                                      E=L.E, wfmt=0)
    rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert 1e-3 < rel < 0.08, rel


def test_debug_hq_positions_follow_routing():
    L, ids = _tiny(0, 1)
    r = _run(L, ids, debug=True)
    counts, offsets, perm, inv, _ = oracle.route(ids, L.E, 1)
    assert r["hq"].shape[0] == len(perm)
    assert (r["hs"] > 0).all()
