"""moe_forward inside a CUDA graph: the layer is captured once on a stream
and replayed with new inputs written into the captured buffers.  Every
replay must give the oracle's layer for those inputs (routing bit-exact,
outputs within the layer tolerance), as the eager call does."""
import numpy as np
import pytest
import torch

import oracle
from fp4_block_scaled_route_b200 import moe, synth

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


def _inputs(T, H, E, k, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    x = torch.randn(T, H, generator=g).to(torch.bfloat16)
    ids, w = synth.make_routing(T, E, k, "uniform", seed)
    return x, torch.from_numpy(ids), torch.from_numpy(w)


CASES = [("fp8_shared", dict(T=24, H=512, I=256, E=8, k=2, wfmt=0, n_shared=1)),
         ("mxfp4", dict(T=40, H=1024, I=512, E=8, k=2, wfmt=1)),
         ("nvfp4", dict(T=16, H=512, I=256, E=6, k=2, wfmt=2))]


@pytest.mark.parametrize("name,cfg", CASES, ids=[c[0] for c in CASES])
def test_forward_replays_from_a_cuda_graph(name, cfg):
    L = synth.make_layer(dict(cfg, routing="uniform"), 81, device="cuda")
    layer = moe.MoeLayer(L.H, L.I, L.E, L.k, L.wfmt, max_T=L.T, n_shared=L.n_shared)
    s13, s2, gsc = L.s13, L.s2, {}
    if L.wfmt == synth.WFMT_MXFP4:
        s13, s2 = moe.pack_mxfp4_scales(s13), moe.pack_mxfp4_scales(s2)
    elif L.wfmt == synth.WFMT_NVFP4:
        s13, s2 = moe.pack_nvfp4_scales(s13), moe.pack_nvfp4_scales(s2)
        gsc = dict(g13=L.g13, g2=L.g2)
    x, ids, w = L.x.clone(), L.ids.clone(), L.topk_w.clone()
    out = torch.empty(L.T, L.H, dtype=torch.bfloat16, device="cuda")
    st = torch.cuda.Stream()
    st.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(st):  # first call encodes the tensor maps outside the capture
        layer.forward(x, ids, w, L.w13, s13, L.w2, s2, out=out, stream=st, **gsc)
    st.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=st):
        layer.forward(x, ids, w, L.w13, s13, L.w2, s2, out=out, stream=st, **gsc)

    kw = dict(g13=L.g13.cpu().numpy(), g2=L.g2.cpu().numpy()) if L.g13 is not None else {}
    for seed in (82, 83):
        xn, idn, wn = _inputs(L.T, L.H, L.E, L.k, seed)
        x.copy_(xn.cuda())
        ids.copy_(idn.cuda())
        w.copy_(wn.cuda())
        graph.replay()
        torch.cuda.synchronize()
        assert layer.device_status() == moe.MOE_OK
        counts, offsets, perm, inv = layer.routing(L.T)
        rc, ro, rp, ri, dropped = oracle.route(idn.numpy(), L.E, L.n_shared)
        assert dropped == 0
        assert np.array_equal(counts, rc) and np.array_equal(offsets, ro)
        assert np.array_equal(perm, rp) and np.array_equal(inv, ri)
        ref = oracle.forward(synth.bf16_bits(xn), idn.numpy(), wn.numpy(), L.w13.cpu().numpy(), L.s13.cpu().numpy(),
                             L.w2.cpu().numpy(), L.s2.cpu().numpy(), H=L.H, I=L.I, E=L.E, wfmt=L.wfmt,
                             n_shared=L.n_shared, **kw)["out_f32"]
        _close(out.float().cpu().numpy(), ref, f"{name} replay {seed}")
    del graph
    layer.close()
