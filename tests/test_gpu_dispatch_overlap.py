"""GPU parity of the dispatch-overlap option (moe_set_dispatch_overlap).

The activations are quantised inside the GEMM1 launch by its last D CTAs,
which publish per-expert ready counters that the other CTAs' token loads and
scale reads wait on (one cooperative launch).  Against the oracle:
- routing (counts, offsets, perm, inv) and the activation codes and scales
  bit for bit: the dispatch warps take every decision of step 2 in the same
  fp32 operations as the quantisation kernel;
- SwiGLU-output codes by the midpoint rule of tests/code_checks.py;
- outputs within the layer's tolerance;
at every token-tile width the option supports (16, 32, 64 and the 128-token
token-major kernel), with MXFP4 weights, the shared expert, the partial
(tensor-parallel) entry point, dispatch partitions from one CTA to all of
them, and the full-size FP8 decode layer.  A withheld ready count (fault
injection mode 2) must run out into MOE_ERR_TIMEOUT without a fault, and the
next call must be correct again.
"""
import time

import numpy as np
import pytest
import torch

import oracle
from fp4_block_scaled_route_b200 import moe, synth
from tests import code_checks

pytestmark = pytest.mark.gpu

RTOL, ATOL, MIN_COS = 2e-2, 1e-3, 0.9999


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from fp4_block_scaled_route_b200 import build
    build.build()
    yield


def _close(gpu, ref, what):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    err = np.abs(gpu - ref).max()
    assert err <= RTOL * np.abs(ref).max() + ATOL, (what, err)
    cos = float((gpu * ref).sum() / (np.linalg.norm(gpu) * np.linalg.norm(ref)))
    assert cos >= MIN_COS, (what, cos)


def _weights(L):
    if L.wfmt == synth.WFMT_MXFP4:
        return L.w13, moe.pack_mxfp4_scales(L.s13), L.w2, moe.pack_mxfp4_scales(L.s2)
    return L.w13, L.s13, L.w2, L.s2


def _oracle(L, debug=False):
    return oracle.forward(synth.bf16_bits(L.x), L.ids.cpu().numpy(), L.topk_w.cpu().numpy(), L.w13.cpu().numpy(),
                          L.s13.cpu().numpy(), L.w2.cpu().numpy(), L.s2.cpu().numpy(), H=L.H, I=L.I, E=L.E,
                          wfmt=L.wfmt, n_shared=L.n_shared, debug=debug)


SMS = None


def _sms():
    global SMS
    if SMS is None:
        SMS = torch.cuda.get_device_properties(0).multi_processor_count
    return SMS


# name, layer, dispatch CTAs (-1: every CTA of the grid), expected tile width
CASES = [
    ("bn16_fp8", dict(T=20, H=512, I=256, E=8, k=2, wfmt=0), 4, 16),
    ("bn16_one_cta", dict(T=20, H=512, I=256, E=8, k=2, wfmt=0), 1, 16),
    ("bn16_all_ctas", dict(T=20, H=512, I=256, E=8, k=2, wfmt=0), -1, 16),
    ("bn32_ragged", dict(T=64, H=512, I=256, E=8, k=2, wfmt=0), 8, 32),
    ("bn64_ragged", dict(T=90, H=384, I=384, E=6, k=3, wfmt=0), 8, 64),
    ("bn128_token_major", dict(T=300, H=256, I=256, E=4, k=2, wfmt=0), 8, 128),
    ("shared_fp8", dict(T=10, H=256, I=256, E=6, k=2, wfmt=0, n_shared=1), 2, 16),
    ("mxfp4", dict(T=20, H=512, I=256, E=8, k=2, wfmt=1), 4, 16),
    ("mxfp4_bn64_shared", dict(T=90, H=256, I=384, E=6, k=3, wfmt=1, n_shared=1), 6, 64),
]


@pytest.mark.parametrize("name,cfg,disp,bn", CASES, ids=[c[0] for c in CASES])
def test_dispatch_overlap_matches_oracle(name, cfg, disp, bn):
    L = synth.make_layer(dict(cfg, routing="uniform"), 300 + len(name), device="cuda")
    layer = moe.MoeLayer(L.H, L.I, L.E, L.k, L.wfmt, max_T=L.T, n_shared=L.n_shared)
    d = _sms() if disp < 0 else disp
    assert layer.set_dispatch_overlap(d) == d
    w13, s13, w2, s2 = _weights(L)
    ref = _oracle(L, debug=True)
    for call in range(2):  # twice: the ready counters are cleared for every call
        out = layer.forward(L.x, L.ids, L.topk_w, w13, s13, w2, s2)
        torch.cuda.synchronize()
        assert layer.device_status() == moe.MOE_OK
        _close(out.float().cpu().numpy(), ref["out_f32"], f"{name} call {call}")
    assert layer.last_config()[0] == bn
    counts, offsets, perm, inv = layer.routing(L.T)
    rc, ro, rp, ri, _ = oracle.route(L.ids.cpu().numpy(), L.E, L.n_shared)
    assert np.array_equal(counts, rc) and np.array_equal(offsets, ro)
    assert np.array_equal(perm, rp) and np.array_equal(inv, ri)
    # step 2, done by the dispatch warps: bit for bit per routed position
    P = int(offsets[-1])
    tok, _ = code_checks.position_map(perm, offsets, L.T, L.k)
    xq, xs, _, _ = layer.activations(L.T)
    assert np.array_equal(xq[:P], ref["xq"][tok])
    assert np.array_equal(xs[:P], ref["xs"][tok])
    code_checks.assert_requant(code_checks.check_requant(L, layer, ref), name)
    # and off again on the same context
    assert layer.set_dispatch_overlap(0) == 0
    out = layer.forward(L.x, L.ids, L.topk_w, w13, s13, w2, s2)
    torch.cuda.synchronize()
    _close(out.float().cpu().numpy(), ref["out_f32"], f"{name} off")
    layer.close()


def test_dispatch_overlap_partial_entry_point():
    """moe_forward_partial (tensor-parallel slices) with the dispatch warps clearing the caller's fp32 buffer."""
    L = synth.make_layer(dict(T=24, H=512, I=256, E=8, k=2, wfmt=0, routing="uniform"), 321, device="cuda")
    layer = moe.MoeLayer(L.H, L.I, L.E, L.k, 0, max_T=L.T)
    layer.set_dispatch_overlap(4)
    acc = torch.full((L.T, L.H), 7.0, dtype=torch.float32, device="cuda")  # must be overwritten, not added to
    layer.forward_partial(L.x, L.ids, L.topk_w, L.w13, L.s13, L.w2, L.s2, out=acc)
    torch.cuda.synchronize()
    assert layer.device_status() == moe.MOE_OK
    _close(acc.cpu().numpy(), _oracle(L)["out_f32"], "partial")
    layer.close()


def test_dispatch_overlap_full_size_decode():
    """The FP8 decode layer T=32, H=7168, E=256, k=8, I=2048, every token against the oracle."""
    L = synth.make_layer(synth.CONFIGS[1], synth.config_seed(1), device="cuda")
    layer = moe.MoeLayer(L.H, L.I, L.E, L.k, L.wfmt, max_T=L.T)
    layer.set_dispatch_overlap(16)
    out = layer.forward(L.x, L.ids, L.topk_w, L.w13, L.s13, L.w2, L.s2)
    torch.cuda.synchronize()
    assert layer.device_status() == moe.MOE_OK
    from tests.test_gpu_parity import oracle_sampled
    tokens = np.arange(L.T)
    _close(out.float().cpu().numpy(), oracle_sampled(L, tokens), "decode full size")
    layer.close()


def test_dispatch_overlap_option_checks():
    nv = moe.MoeLayer(256, 256, 4, 2, moe.MOE_WFMT_NVFP4_E2M1_E4M3_K16, max_T=8)
    assert moe.moe_set_dispatch_overlap(nv.ctx, 4) == moe.MOE_ERR_UNSUPPORTED  # FP8 activations only
    nv.close()
    fp8 = moe.MoeLayer(256, 256, 4, 2, 0, max_T=8)
    assert moe.moe_set_dispatch_overlap(fp8.ctx, -1) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_set_dispatch_overlap(fp8.ctx, _sms() + 1) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_set_dispatch_overlap(fp8.ctx, 4) == moe.MOE_OK
    assert moe.moe_set_green_ctx(fp8.ctx, 16) == moe.MOE_ERR_UNSUPPORTED  # one form of the split at a time
    assert moe.moe_dispatch_overlap_ctas(fp8.ctx) == 4
    fp8.close()


def test_dispatch_overlap_timeout_is_reported_and_context_recovers():
    """Fault injection mode 2: routing position 0 is never published, so the
    consumers of its expert's counter run out of time (about a second), the
    kernel drains and returns, and MOE_ERR_TIMEOUT is reported; nothing
    faults, and the next call is correct."""
    L = synth.make_layer(dict(T=8, H=512, I=256, E=8, k=2, wfmt=0, routing="uniform"), 92, device="cuda")
    layer = moe.MoeLayer(L.H, L.I, L.E, L.k, 0, max_T=L.T)
    layer.set_dispatch_overlap(4)
    assert moe.moe_set_fault_injection(layer.ctx, 2) == moe.MOE_OK
    t0 = time.time()
    layer.forward(L.x, L.ids, L.topk_w, L.w13, L.s13, L.w2, L.s2)
    torch.cuda.synchronize()
    dt = time.time() - t0
    assert layer.device_status() == moe.MOE_ERR_TIMEOUT
    assert dt < 30.0, dt
    assert moe.moe_set_fault_injection(layer.ctx, 0) == moe.MOE_OK
    out = layer.forward(L.x, L.ids, L.topk_w, L.w13, L.s13, L.w2, L.s2)
    torch.cuda.synchronize()
    assert layer.device_status() == moe.MOE_OK
    _close(out.float().cpu().numpy(), _oracle(L)["out_f32"], "after timeout")
    layer.close()
