"""GPU parity at the limits moe_create_ex accepts: the largest K (H = I =
8192, 64 K blocks per GEMM, the most the kernels' per-unit scale tables hold)
in every weight format, and the most experts (E = 1024) with the largest
top-k (32).  Every output element against the oracle with the layer's
tolerance; the routing bit-exact."""
import numpy as np
import pytest
import torch

import oracle
from fp4_block_scaled_route_b200 import moe, synth

pytestmark = pytest.mark.gpu

RTOL = 2e-2
ATOL = 1e-3
MIN_COS = 0.9999


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from fp4_block_scaled_route_b200 import build
    build.build()
    yield


def assert_close(gpu, ref, what=""):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    scale = np.abs(ref).max()
    err = np.abs(gpu - ref).max()
    assert err <= RTOL * scale + ATOL, f"{what}: max err {err:.3e} vs bound {RTOL * scale + ATOL:.3e}"
    den = np.linalg.norm(gpu) * np.linalg.norm(ref)
    cos = 1.0 if den == 0 else float((gpu * ref).sum() / den)
    assert cos >= MIN_COS, f"{what}: cosine {cos:.6f}"


def run_layer(L):
    layer = moe.MoeLayer(L.H, L.I, L.E, L.k, L.wfmt, max_T=L.T, n_shared=L.n_shared)
    s13, s2 = L.s13, L.s2
    if L.wfmt in (synth.WFMT_MXFP4, synth.WFMT_MXFP4_A4):
        s13, s2 = moe.pack_mxfp4_scales(s13), moe.pack_mxfp4_scales(s2)
    elif L.wfmt == synth.WFMT_NVFP4:
        s13, s2 = moe.pack_nvfp4_scales(s13), moe.pack_nvfp4_scales(s2)
    out = layer.forward(L.x, L.ids, L.topk_w, L.w13, s13, L.w2, s2, g13=L.g13, g2=L.g2)
    torch.cuda.synchronize()
    return layer, out


def oracle_out(L):
    kw = dict(g13=L.g13.cpu().numpy(), g2=L.g2.cpu().numpy()) if L.g13 is not None else {}
    return oracle.forward(synth.bf16_bits(L.x), L.ids.cpu().numpy(), L.topk_w.cpu().numpy(), L.w13.cpu().numpy(),
                          L.s13.cpu().numpy(), L.w2.cpu().numpy(), L.s2.cpu().numpy(), H=L.H, I=L.I, E=L.E,
                          wfmt=L.wfmt, n_shared=L.n_shared, **kw)["out_f32"]


FORMATS = [("fp8", synth.WFMT_FP8), ("mxfp4", synth.WFMT_MXFP4),
           ("nvfp4", synth.WFMT_NVFP4), ("mxfp4_a4", synth.WFMT_MXFP4_A4)]


@pytest.mark.parametrize("name,wfmt", FORMATS, ids=[f[0] for f in FORMATS])
def test_largest_K(name, wfmt):
    """H = I = 8192: GEMM1 and GEMM2 both run 64 K blocks per unit."""
    cfg = dict(T=5, H=8192, I=8192, E=3, k=2, wfmt=wfmt, n_shared=1, routing="uniform")
    L = synth.make_layer(cfg, 3100 + wfmt, device="cuda")
    layer, out = run_layer(L)
    assert layer.device_status() == moe.MOE_OK
    assert_close(out.float().cpu().numpy(), oracle_out(L), f"{name} H=I=8192")
    layer.close()


def test_most_experts_largest_k():
    """E = 1024 experts and top-k = 32: routing bit-exact, every output element."""
    cfg = dict(T=40, H=256, I=128, E=1024, k=32, wfmt=0, routing="uniform")
    L = synth.make_layer(cfg, 3200, device="cuda")
    layer, out = run_layer(L)
    assert layer.device_status() == moe.MOE_OK
    counts, offsets, perm, inv = layer.routing(L.T)
    rc, ro, rp, ri, dropped = oracle.route(L.ids.cpu().numpy(), L.E)
    assert dropped == 0
    assert np.array_equal(counts, rc) and np.array_equal(offsets, ro)
    assert np.array_equal(perm, rp) and np.array_equal(inv, ri)
    assert_close(out.float().cpu().numpy(), oracle_out(L), "E=1024 k=32")
    layer.close()

