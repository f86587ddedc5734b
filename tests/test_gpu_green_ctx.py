"""GPU parity of the Green-Context partition option (moe_set_green_ctx): the
dispatch kernels run in a green context of a few SMs and the grouped GEMMs in
one of the remaining SMs; results must match the oracle exactly as the
single-partition path does (indices bit-exact, outputs within the layer's
tolerance)."""
import numpy as np
import pytest
import torch

import oracle
from fp4_block_scaled_route_b200 import moe, synth

pytestmark = pytest.mark.gpu

RTOL, ATOL, MIN_COS = 2e-2, 1e-3, 0.9999


def _close(gpu, ref):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    err = np.abs(gpu - ref).max()
    assert err <= RTOL * np.abs(ref).max() + ATOL, err
    cos = float((gpu * ref).sum() / (np.linalg.norm(gpu) * np.linalg.norm(ref)))
    assert cos >= MIN_COS, cos


def _oracle(L):
    return oracle.forward(synth.bf16_bits(L.x), L.ids.cpu().numpy(), L.topk_w.cpu().numpy(), L.w13.cpu().numpy(),
                          L.s13.cpu().numpy(), L.w2.cpu().numpy(), L.s2.cpu().numpy(), H=L.H, I=L.I, E=L.E,
                          wfmt=L.wfmt, n_shared=L.n_shared)["out_f32"]


@pytest.mark.parametrize("cfg,seed", [(dict(T=20, H=512, I=256, E=8, k=2, wfmt=0, n_shared=1), 71),
                                      (dict(T=300, H=256, I=256, E=16, k=4, wfmt=0), 72),
                                      (dict(T=20, H=512, I=256, E=8, k=2, wfmt=1), 73)],
                         ids=["decode_tiles_shared", "token_major_tiles", "mxfp4"])
def test_green_ctx_matches_oracle(cfg, seed):
    assert torch.cuda.is_available(), "needs a CUDA device"
    L = synth.make_layer(cfg, seed, device="cuda")
    layer = moe.MoeLayer(L.H, L.I, L.E, L.k, L.wfmt, max_T=L.T, n_shared=L.n_shared)
    d, g = layer.set_green_ctx(16)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert d >= 16 and g >= 8 and d + g <= sms
    w13, s13, w2, s2 = L.w13, L.s13, L.w2, L.s2
    if L.wfmt == synth.WFMT_MXFP4:
        s13, s2 = moe.pack_mxfp4_scales(L.s13), moe.pack_mxfp4_scales(L.s2)
    for _ in range(2):  # twice: the partition's events and streams are reused
        out = layer.forward(L.x, L.ids, L.topk_w, w13, s13, w2, s2)
        torch.cuda.synchronize()
        assert layer.device_status() == moe.MOE_OK
        _close(out.float().cpu().numpy(), _oracle(L))
    assert layer.last_config()[1] == g  # the GEMMs ran on the large partition's SMs
    counts, offsets, perm, inv = layer.routing(L.T)
    rc, ro, rp, ri, _ = oracle.route(L.ids.cpu().numpy(), L.E, L.n_shared)
    assert np.array_equal(counts, rc) and np.array_equal(perm, rp) and np.array_equal(inv, ri)
    # back to one partition on the same context
    assert layer.set_green_ctx(0) == (0, 0)
    out = layer.forward(L.x, L.ids, L.topk_w, w13, s13, w2, s2)
    torch.cuda.synchronize()
    _close(out.float().cpu().numpy(), _oracle(L))
    layer.close()


def test_green_ctx_full_decode_sampled():
    """The FP8 decode layer T=32, H=7168, E=256, k=8, I=2048 on the partition, sampled tokens."""
    cfg = synth.CONFIGS[1]
    L = synth.make_layer(cfg, synth.config_seed(1), device="cuda")
    layer = moe.MoeLayer(L.H, L.I, L.E, L.k, L.wfmt, max_T=L.T)
    layer.set_green_ctx(8)
    out = layer.forward(L.x, L.ids, L.topk_w, L.w13, L.s13, L.w2, L.s2)
    torch.cuda.synchronize()
    assert layer.device_status() == moe.MOE_OK
    from tests.test_gpu_parity import oracle_sampled
    tokens = np.array([0, 7, 19, 31])
    _close(out.float().cpu().numpy()[tokens], oracle_sampled(L, tokens))
    layer.close()
