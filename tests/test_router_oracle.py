"""Pins of the fused-router oracle (CPU only).

The oracle (oracle.router / orc_router in C) computes logits = x . Wr^T with
fp64 accumulation rounded once to fp32, takes the k largest per token (ties to
the lower expert index, descending order) and the softmax over the chosen
logits.  Reading of the DeepGEMM 26/09 news page ("Mega Gate": routing GEMM +
MoE routing ops in one kernel), which names the fusion but gives no formula.
The pins below check it against independent numpy arithmetic, closed forms and
invariants, not against a retyped copy of its loops.
"""
import numpy as np
import pytest

import oracle
from fp4_block_scaled_route_b200 import synth


def _bf16_to_f64(bits):
    return (np.asarray(bits, np.uint32) << 16).view(np.float32).astype(np.float64)


def _ref(xb, wb, k):
    """numpy: fp64 matmul, fp32 rounding, stable descending selection, fp64 softmax."""
    lg = (_bf16_to_f64(xb) @ _bf16_to_f64(wb).T).astype(np.float32)
    T, E = lg.shape
    ids = np.zeros((T, k), np.int64)
    for t in range(T):
        order = np.lexsort((np.arange(E), -lg[t].astype(np.float64)))  # by -logit, then index
        ids[t] = order[:k]
    sel = np.take_along_axis(lg.astype(np.float64), ids, axis=1)
    ex = np.exp(sel - sel[:, :1])
    w = ex / ex.sum(axis=1, keepdims=True)
    return lg, ids, w


@pytest.mark.parametrize("T,H,E,k,seed", [(7, 256, 16, 4, 1), (3, 384, 256, 8, 2), (5, 128, 8, 8, 3)])
def test_router_oracle_against_numpy(T, H, E, k, seed):
    x, wr = synth.make_router(T, H, E, seed)
    xb, wb = synth.bf16_bits(x), synth.bf16_bits(wr)
    ids, w, lg = oracle.router(xb, wb, k, with_logits=True)
    rlg, rids, rw = _ref(xb, wb, k)
    np.testing.assert_allclose(lg, rlg, rtol=1e-6, atol=1e-7)
    assert np.array_equal(ids, rids)
    np.testing.assert_allclose(w, rw, rtol=2e-6, atol=1e-7)


def test_router_oracle_invariants():
    x, wr = synth.make_router(64, 512, 64, 11)
    ids, w, lg = oracle.router(synth.bf16_bits(x), synth.bf16_bits(wr), 6, with_logits=True)
    assert (w > 0).all()
    np.testing.assert_allclose(w.sum(axis=1), 1.0, atol=1e-6)
    for t in range(ids.shape[0]):
        assert len(set(ids[t].tolist())) == 6
        sel = lg[t, ids[t]]
        assert (np.diff(sel) <= 0).all()                     # descending
        rest = np.delete(lg[t], ids[t])
        assert rest.max() <= sel.min()                       # nothing unselected beats a selected logit
        assert (np.diff(w[t]) <= 0).all()                    # weights follow the logits


def test_router_oracle_k_equals_E_is_the_full_softmax():
    x, wr = synth.make_router(4, 128, 8, 5)
    ids, w, lg = oracle.router(synth.bf16_bits(x), synth.bf16_bits(wr), 8, with_logits=True)
    for t in range(4):
        assert sorted(ids[t].tolist()) == list(range(8))
        full = np.exp(lg[t].astype(np.float64) - lg[t].max())
        full /= full.sum()
        np.testing.assert_allclose(w[t], full[ids[t]], rtol=1e-6)


def test_router_oracle_ties_take_the_lower_index():
    """All-zero router weights: every logit is 0, so the choice is experts 0..k-1 at 1/k."""
    x, _ = synth.make_router(3, 128, 32, 7)
    wb = np.zeros((32, 128), np.uint16)
    ids, w = oracle.router(synth.bf16_bits(x), wb, 5)
    assert (ids == np.arange(5)).all()
    assert (w == np.float32(1.0 / 5)).all()


def test_router_oracle_one_hot_closed_form():
    """x = unit vector at column h: the logits are column h of Wr, known exactly."""
    H, E, k = 128, 16, 3
    h = 17
    x = np.zeros((1, H), np.float32)
    x[0, h] = 1.0
    vals = np.array([0.5, -1.0, 2.0, 0.25, 1.5, -0.5, 3.0, 0.0, 1.0, -2.0, 0.75, 2.5, -0.25, 1.25, -3.0, 0.125],
                    np.float32)  # all exact in bf16
    wr = np.zeros((E, H), np.float32)
    wr[:, h] = vals
    to_bits = lambda a: (a.view(np.uint32) >> 16).astype(np.uint16)
    ids, w, lg = oracle.router(to_bits(x), to_bits(wr), k, with_logits=True)
    assert np.array_equal(lg[0], vals)
    assert ids[0].tolist() == [6, 11, 2]                      # 3.0, 2.5, 2.0
    e = np.exp(np.array([3.0, 2.5, 2.0]) - 3.0)
    np.testing.assert_allclose(w[0], e / e.sum(), rtol=1e-6)
