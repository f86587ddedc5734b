"""CPU checks of the requantisation-code checker (tests/code_checks.py).

The oracle's own SwiGLU-output codes stand in for the GPU's: they must pass
(the oracle's fp32 sums differ from the fp64 recomputation only in the last
bits), and planted defects of the kinds a kernel could have must fail: two
channels swapped, whole rows shifted by one channel, a scale off by 0.1 %.
"""
import numpy as np
import pytest

import oracle
from fp4_block_scaled_route_b200 import synth
from tests import code_checks


class _Stand:
    """Duck-typed stand-in for the GPU layer: routing and activations from the oracle."""

    def __init__(self, L, ref, mutate=None):
        self.k = L.k
        self.r = oracle.route(L.ids.numpy(), L.E, L.n_shared)
        self.ref, self.mutate = ref, mutate

    def routing(self, T):
        return self.r[:4]

    def activations(self, T):
        hq, hs = self.ref["hq"].copy(), self.ref["hs"].copy()
        if self.mutate:
            hq, hs = self.mutate(hq, hs)
        return None, None, hq, hs

    def block_scales(self, T):
        return None, self.ref["hsc"].copy()


def _swap(hq, hs):
    hq[:, [0, 1]] = hq[:, [1, 0]]
    return hq, hs


def _roll(hq, hs):
    hq[::7] = np.roll(hq[::7], 1, axis=1)
    return hq, hs


def _scale(hq, hs):
    hs[3, 0] *= 1.001
    return hq, hs


CASES = [(dict(T=40, H=512, I=256, E=8, k=2, wfmt=0), 3), (dict(T=40, H=512, I=256, E=8, k=2, wfmt=1), 4),
         (dict(T=20, H=512, I=384, E=8, k=2, wfmt=2, n_shared=1), 5), (dict(T=20, H=512, I=384, E=8, k=2, wfmt=3), 6),
         (dict(T=20, H=512, I=384, E=8, k=2, wfmt=4, n_shared=1), 7)]


@pytest.mark.parametrize("cfg,seed", CASES, ids=["fp8", "mxfp4", "nvfp4_shared", "mxfp4_a4", "mxfp8_shared"])
def test_checker_passes_the_oracle_and_fails_planted_defects(cfg, seed):
    L = synth.make_layer(dict(cfg, routing="uniform"), seed, device="cpu")
    g = dict(g13=L.g13.numpy(), g2=L.g2.numpy()) if L.wfmt == 2 else {}
    ref = oracle.forward(synth.bf16_bits(L.x), L.ids.numpy(), L.topk_w.numpy(), L.w13.numpy(), L.s13.numpy(),
                         L.w2.numpy(), L.s2.numpy(), H=L.H, I=L.I, E=L.E, wfmt=L.wfmt, n_shared=L.n_shared,
                         debug=True, **g)
    code_checks.assert_requant(code_checks.check_requant(L, _Stand(L, ref), ref), "oracle")
    for mutate in (_swap, _roll):
        rep = code_checks.check_requant(L, _Stand(L, ref, mutate), ref)
        assert rep["violations"] > 0, (mutate.__name__, dict(rep))
    if L.wfmt in (0, 2):  # formats with an fp32 requantisation scale
        rep = code_checks.check_requant(L, _Stand(L, ref, _scale), ref)
        assert rep["scale_violations"] > 0, dict(rep)
