"""Failure detection on the GPU without a fault: a pipeline wait that runs out.

The fault-injection hook makes one GEMM1 stage expect 16 bytes that never
arrive.  The bounded wait must give up (about a second), the kernel must
drain and return, the host must read MOE_ERR_TIMEOUT, and the very next call
on the same context must be correct again.
"""
import time

import numpy as np
import pytest
import torch

import oracle
from fp4_block_scaled_route_b200 import moe, synth

pytestmark = pytest.mark.gpu


def test_pipeline_timeout_is_reported_and_context_recovers():
    assert torch.cuda.is_available(), "needs a CUDA device"
    L = synth.make_layer(dict(T=8, H=512, I=256, E=8, k=2, wfmt=0), 91, device="cuda")
    layer = moe.MoeLayer(L.H, L.I, L.E, L.k, 0, max_T=L.T)
    assert moe.moe_set_fault_injection(layer.ctx, 1) == moe.MOE_OK
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
    ref = oracle.forward(synth.bf16_bits(L.x), L.ids.cpu().numpy(), L.topk_w.cpu().numpy(), L.w13.cpu().numpy(),
                         L.s13.cpu().numpy(), L.w2.cpu().numpy(), L.s2.cpu().numpy(), H=L.H, I=L.I, E=L.E,
                         wfmt=0)["out_f32"]
    got = out.float().cpu().numpy()
    assert np.abs(got - ref).max() <= 2e-2 * np.abs(ref).max() + 1e-3
    layer.close()
