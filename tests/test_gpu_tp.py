"""Tensor parallelism over I on one GPU: the slices of G ranks run one after
another through moe_forward_partial in one process (no collective: the sum
is taken here, as the all-reduce would), then moe_finalize_bf16.  Each
partial must match the oracle's partial for its slice, and the finished
layer the oracle's whole layer, with the layer tolerance."""
import numpy as np
import pytest
import torch

import oracle
from fp4_block_scaled_route_b200 import moe, synth, tp

pytestmark = pytest.mark.gpu

RTOL = 2e-2
ATOL = 1e-3


def _close(got, ref, what):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    bound = RTOL * np.abs(ref).max() + ATOL
    err = np.abs(got - ref).max()
    assert err <= bound, f"{what}: {err:.3e} > {bound:.3e}"
    cos = float((got * ref).sum() / (np.linalg.norm(got) * np.linalg.norm(ref)))
    assert cos >= 0.9999, f"{what}: cosine {cos:.6f}"


def _oracle(L, w13, s13, w2, s2, I, g13=None, g2=None):
    kw = dict(g13=g13.cpu().numpy(), g2=g2.cpu().numpy()) if g13 is not None else {}
    return oracle.forward(synth.bf16_bits(L.x), L.ids.cpu().numpy(), L.topk_w.cpu().numpy(), w13.cpu().numpy(),
                          s13.cpu().numpy(), w2.cpu().numpy(), s2.cpu().numpy(), H=L.H, I=I, E=L.E, wfmt=L.wfmt,
                          n_shared=L.n_shared, **kw)["out_f32"]


CASES = [("fp8_shared", dict(T=24, H=512, I=512, E=8, k=2, wfmt=0, n_shared=1), 2),
         ("fp8_g4", dict(T=9, H=256, I=512, E=6, k=3, wfmt=0), 4),
         ("nvfp4", dict(T=16, H=512, I=512, E=8, k=2, wfmt=2), 2),
         ("mxfp4_a4", dict(T=16, H=512, I=512, E=8, k=2, wfmt=3, n_shared=1), 2),
         ("mxfp4", dict(T=12, H=512, I=512, E=8, k=2, wfmt=1), 2),
         ("mxfp8_shared", dict(T=20, H=512, I=512, E=8, k=2, wfmt=4, n_shared=1), 2)]


@pytest.mark.parametrize("name,cfg,G", CASES, ids=[c[0] for c in CASES])
def test_slices_sum_to_the_layer(name, cfg, G):
    L = synth.make_layer(dict(cfg, routing="uniform"), 95, device="cuda")
    Is = L.I // G
    total = torch.zeros(L.T, L.H, dtype=torch.float32, device="cuda")
    for r in range(G):
        sh = tp.shard_weights(L.w13, L.s13, L.w2, L.s2, L.wfmt, L.I, r, G, L.g13, L.g2)
        layer = moe.MoeLayer(L.H, Is, L.E, L.k, L.wfmt, max_T=L.T, n_shared=L.n_shared)
        pk = tp.pack_shard(sh, L.wfmt)
        part = layer.forward_partial(L.x, L.ids, L.topk_w, pk["w13"], pk["s13"], pk["w2"], pk["s2"],
                                     g13=pk.get("g13"), g2=pk.get("g2"))
        torch.cuda.synchronize()
        assert layer.device_status() == moe.MOE_OK
        _close(part.cpu().numpy(), _oracle(L, sh["w13"], sh["s13"], sh["w2"], sh["s2"], Is, sh.get("g13"),
                                           sh.get("g2")), f"{name} rank {r}")
        total += part
        layer.close()
    out = moe.finalize_bf16(total)
    torch.cuda.synchronize()
    _close(out.float().cpu().numpy(), _oracle(L, L.w13, L.s13, L.w2, L.s2, L.I, L.g13, L.g2), f"{name} sum")
    # the finalize step is the bf16 rounding of the summed fp32 result
    assert torch.equal(out, total.to(torch.bfloat16))


def test_partial_entry_point_checks():
    L = synth.make_layer(dict(T=4, H=256, I=256, E=4, k=2, wfmt=0), 96, device="cuda")
    layer = moe.MoeLayer(L.H, L.I, L.E, L.k, 0, max_T=4)
    st = torch.cuda.current_stream().cuda_stream
    args = (layer.ctx, 4, L.x.data_ptr(), L.ids.data_ptr(), L.topk_w.data_ptr(), L.w13.data_ptr(),
            L.s13.data_ptr(), None, L.w2.data_ptr(), L.s2.data_ptr(), None)
    assert moe.moe_forward_partial(*args, None, st) == moe.MOE_ERR_INVALID_ARG      # no output buffer
    buf = torch.empty(4 * 256 + 1, dtype=torch.float32, device="cuda")
    assert moe.moe_forward_partial(*args, buf.data_ptr() + 4, st) == moe.MOE_ERR_INVALID_ARG  # misaligned
    assert moe.moe_finalize_bf16(buf.data_ptr(), buf.data_ptr(), 6, st) == moe.MOE_ERR_INVALID_ARG  # n % 4
    torch.cuda.synchronize()
