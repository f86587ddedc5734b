"""moe_forward_noalloc: the layer for callers that cannot allocate device memory.

Such callers (code under a host framework that owns all device allocations,
or a memory-pool-locked process) get one entry point that
keeps its scratch in a fixed file-scope device array instead of a context's
workspace.  These tests call it through the C ABI and compare its output with
moe_forward's (the entry point that allocates a workspace), within the
layer's tolerance, on two calls in a row, so that scratch left behind by one
call cannot leak into the next.  The file is named to be collected last.
"""
import numpy as np
import pytest
import torch

from fp4_block_scaled_route_b200 import build as moe_build
from fp4_block_scaled_route_b200 import moe, synth

RTOL, ATOL, MIN_COS = 2e-2, 1e-3, 0.9999


def _close(a, b, what):
    a = a.float().cpu().numpy().astype(np.float64)
    b = b.float().cpu().numpy().astype(np.float64)
    bound = RTOL * np.abs(b).max() + ATOL
    err = np.abs(a - b).max()
    cos = float((a * b).sum() / (np.linalg.norm(a) * np.linalg.norm(b)))
    assert err <= bound and cos >= MIN_COS, (what, err, bound, cos)


def test_noalloc_rejects_shapes_beyond_the_scratch():
    moe_build.build()
    # T=4096 at H=7168, k=8 needs ~300 MB of scratch: refused before any device work
    rc = moe.moe_forward_noalloc(7168, 2048, 256, 8, 0, 0, 4096, None, None, None, None, None, None, None,
                                 None, None, None)
    assert rc == moe.MOE_ERR_UNSUPPORTED
    rc = moe.moe_forward_noalloc(100, 2048, 256, 8, 0, 0, 4, None, None, None, None, None, None, None,
                                 None, None, None)
    assert rc == moe.MOE_ERR_UNSUPPORTED
    # the formats with 4-bit activations, and MXFP8, are not offered here
    for wfmt in (moe.MOE_WFMT_NVFP4_E2M1_E4M3_K16, moe.MOE_WFMT_MXFP4_W4A4, moe.MOE_WFMT_MXFP8_E4M3_E8M0_K32):
        rc = moe.moe_forward_noalloc(512, 256, 8, 2, wfmt, 0, 4, None, None, None, None, None, None, None,
                                     None, None, None)
        assert rc == moe.MOE_ERR_UNSUPPORTED


# Each case reaches one token-tile width, which this entry point chooses and
# builds tensor maps for on its own: 16 (decode), 32, 64 (FP8 and MXFP4) and
# the 128-token token-major kernel (FP8).
CASES = [
    ("decode_fp8_T32_H7168_E256_k8_I2048", dict(T=32, H=7168, E=256, k=8, I=2048, wfmt=0), 501),
    ("mxfp4_shared_T12_H512_E8_k2_I256", dict(T=12, H=512, E=8, k=2, I=256, wfmt=1, n_shared=1), 502),
    ("fp8_bn32_T48_H512_E8_k2_I256", dict(T=48, H=512, E=8, k=2, I=256, wfmt=0), 503),
    ("fp8_bn64_T120_H512_E8_k2_I256", dict(T=120, H=512, E=8, k=2, I=256, wfmt=0), 504),
    ("fp8_bn128_T1024_H512_E8_k2_I256", dict(T=1024, H=512, E=8, k=2, I=256, wfmt=0), 505),
    ("mxfp4_bn64_T160_H512_E8_k2_I256", dict(T=160, H=512, E=8, k=2, I=256, wfmt=1), 506),
]


@pytest.mark.gpu
@pytest.mark.parametrize("name,cfg,seed", CASES, ids=[c[0] for c in CASES])
def test_noalloc_matches_moe_forward_twice(name, cfg, seed):
    assert torch.cuda.is_available(), "needs a CUDA device"
    moe_build.build()
    L = synth.make_layer(cfg, seed, device="cuda")
    gen = torch.Generator(device="cuda").manual_seed(seed + 1)
    x2 = synth.make_x(L.T, L.H, gen, "cuda")
    nsh = cfg.get("n_shared", 0)
    if L.wfmt == synth.WFMT_MXFP4:
        s13, s2 = moe.pack_mxfp4_scales(L.s13), moe.pack_mxfp4_scales(L.s2)
    else:
        s13, s2 = L.s13, L.s2
    layer = moe.MoeLayer(L.H, L.I, L.E, L.k, L.wfmt, max_T=L.T, n_shared=nsh)
    stream = torch.cuda.current_stream().cuda_stream
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    for call, x in enumerate((L.x, x2)):
        ref = layer.forward(x, L.ids, L.topk_w, L.w13, s13, L.w2, s2).clone()
        out = torch.full((L.T, L.H), float("nan"), dtype=torch.bfloat16, device="cuda")
        rc = moe.moe_forward_noalloc(L.H, L.I, L.E, L.k, L.wfmt, nsh, L.T, x.data_ptr(), L.ids.data_ptr(),
                                     L.topk_w.data_ptr(), L.w13.data_ptr(), s13.data_ptr(), L.w2.data_ptr(),
                                     s2.data_ptr(), out.data_ptr(), status.data_ptr(), stream)
        assert rc == moe.MOE_OK, moe.status_string(rc)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert torch.isfinite(out.float()).all()
        _close(out, ref, f"{name} call {call}")
    layer.close()
