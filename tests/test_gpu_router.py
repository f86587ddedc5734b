"""GPU parity of the fused router (moe_router_topk) against its oracle.

Both sides select on fp32 logits, but the GPU sums the H products in another
order (tensor cores, K splits added with fp32 reductions), so a logit can
differ from the oracle's exact value in its last bits.  Where the oracle's k-th
and (k+1)-th logits are further apart than that, the chosen experts must match
exactly (as a set; the order must be non-increasing in the oracle's logits up
to the same margin) and the weights within 2e-5.  Where they are closer (a
near-tie), either choice is correct: the chosen set must still be a valid
top-k of the oracle's logits, and in every case the weights must be the
softmax of the oracle's logits of the chosen set.
"""
import numpy as np
import pytest
import torch

import oracle
from fp4_block_scaled_route_b200 import moe, synth

pytestmark = pytest.mark.gpu

EPS = 5e-4  # logit margin that the summation order can cross (fp32 sum error ~1e-5 here)
W_ATOL = 2e-5  # combine weights: a logit error of ~1e-5 moves a softmax weight by about as much


def _check(ids_g, w_g, ids_o, w_o, lg_o):
    T, k = ids_o.shape
    E = lg_o.shape[1]
    ambiguous = 0
    for t in range(T):
        order = np.argsort(-lg_o[t], kind="stable")
        kth = lg_o[t, order[k - 1]]
        nxt = lg_o[t, order[k]] if E > k else -np.inf
        g = ids_g[t]
        assert len(set(g.tolist())) == k and g.min() >= 0 and g.max() < E
        assert np.all(np.diff(lg_o[t, g]) <= EPS)                   # descending up to the margin
        np.testing.assert_allclose(w_g[t].sum(), 1.0, atol=1e-5)
        # whatever set was chosen, its weights are the softmax of the oracle's
        # logits of that set (measured on B200: within 1.4e-6)
        sel = lg_o[t, g].astype(np.float64)
        ex = np.exp(sel - sel.max())
        np.testing.assert_allclose(w_g[t], ex / ex.sum(), atol=W_ATOL)
        if kth - nxt > EPS:
            assert set(g.tolist()) == set(ids_o[t].tolist()), (t, g, ids_o[t])
            wo = dict(zip(ids_o[t].tolist(), w_o[t].tolist()))
            np.testing.assert_allclose(w_g[t], [wo[e] for e in g.tolist()], atol=W_ATOL)
        else:
            ambiguous += 1
            assert lg_o[t, g].min() >= kth - EPS                     # still a valid top-k
    return ambiguous


CASES = [("tiny", 4, 256, 8, 2), ("decode", 32, 7168, 256, 8), ("zipf_shape", 8, 4096, 160, 8),
         ("ragged", 300, 512, 64, 6), ("prefill", 4096, 7168, 256, 8)]


@pytest.mark.parametrize("name,T,H,E,k", CASES, ids=[c[0] for c in CASES])
def test_router_matches_oracle(name, T, H, E, k):
    assert torch.cuda.is_available(), "needs a CUDA device"
    x, wr = synth.make_router(T, H, E, 100 + T, device="cuda")
    layer = moe.MoeLayer(H, 128, E, k, 0, max_T=T)
    ids_o, w_o, lg_o = oracle.router(synth.bf16_bits(x), synth.bf16_bits(wr), k, with_logits=True)
    for _ in range(2):  # the second call also checks that the workspace was left zeroed
        ids, w = layer.router(x, wr)
        torch.cuda.synchronize()
        assert layer.device_status() == moe.MOE_OK
        amb = _check(ids.cpu().numpy(), w.cpu().numpy(), ids_o, w_o, lg_o)
        assert amb <= T // 8 + 2, amb
    layer.close()


def test_router_feeds_the_layer():
    """Router outputs drive moe_forward; the layer matches the oracle given the same routing."""
    cfg = dict(T=24, H=512, I=256, E=16, k=4, wfmt=0)
    L = synth.make_layer(cfg, 81, device="cuda")
    _, wr = synth.make_router(cfg["T"], cfg["H"], cfg["E"], 82, device="cuda")
    layer = moe.MoeLayer(cfg["H"], cfg["I"], cfg["E"], cfg["k"], 0, max_T=cfg["T"])
    ids, w = layer.router(L.x, wr)
    out = layer.forward(L.x, ids, w, L.w13, L.s13, L.w2, L.s2)
    torch.cuda.synchronize()
    ref = oracle.forward(synth.bf16_bits(L.x), ids.cpu().numpy(), w.cpu().numpy(), L.w13.cpu().numpy(),
                         L.s13.cpu().numpy(), L.w2.cpu().numpy(), L.s2.cpu().numpy(), H=cfg["H"], I=cfg["I"],
                         E=cfg["E"], wfmt=0)["out_f32"]
    got = out.float().cpu().numpy()
    assert np.abs(got - ref).max() <= 2e-2 * np.abs(ref).max() + 1e-3
    layer.close()


def test_router_rejects_unsupported_expert_counts():
    layer = moe.MoeLayer(256, 128, 6, 2, 0, max_T=8)  # E not a multiple of 4
    x = torch.zeros(8, 256, dtype=torch.bfloat16, device="cuda")
    wr = torch.zeros(6, 256, dtype=torch.bfloat16, device="cuda")
    ids = torch.empty(8, 2, dtype=torch.int32, device="cuda")
    w = torch.empty(8, 2, dtype=torch.float32, device="cuda")
    st = moe.moe_router_topk(layer.ctx, 8, x.data_ptr(), wr.data_ptr(), ids.data_ptr(), w.data_ptr(),
                             torch.cuda.current_stream().cuda_stream)
    assert st == moe.MOE_ERR_UNSUPPORTED
    layer.close()
