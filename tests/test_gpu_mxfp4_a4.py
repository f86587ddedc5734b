"""GPU parity of MXFP4 weights with MXFP4 activations (MOE_WFMT_MXFP4_W4A4,
tcgen05 kind::mxf4 with UE8M0 scales on both operands) against the oracle.

- Activation quantisation: packed E2M1 codes and E8M0 block codes compared
  bit for bit (both sides take every decision in the same fp32 operations).
- SwiGLU-output codes: not bit-exact (the tensor cores sum in another order,
  which can move a value across a rounding or exponent boundary) but nearly
  all equal.
- Layer outputs element by element with the layer's tolerance
  |gpu - oracle| <= 2e-2 * max|oracle| + 1e-3 and cosine >= 0.9999; the
  full-size decode shape on sampled tokens in the benchmark's launch
  configuration.
"""
import numpy as np
import pytest
import torch

import oracle
from fp4_block_scaled_route_b200 import moe, synth
from tests import code_checks

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


def run_gpu(L):
    layer = moe.MoeLayer(L.H, L.I, L.E, L.k, moe.MOE_WFMT_MXFP4_W4A4, max_T=max(L.T, 1), n_shared=L.n_shared)
    out = layer.forward(L.x, L.ids, L.topk_w, L.w13, moe.pack_mxfp4_scales(L.s13), L.w2,
                        moe.pack_mxfp4_scales(L.s2))
    torch.cuda.synchronize()
    return layer, out


def oracle_ref(L, debug=False, tokens=None):
    ids = L.ids.cpu().numpy()
    if tokens is None:
        return oracle.forward(synth.bf16_bits(L.x), ids, L.topk_w.cpu().numpy(), L.w13.cpu().numpy(),
                              L.s13.cpu().numpy(), L.w2.cpu().numpy(), L.s2.cpu().numpy(), H=L.H, I=L.I, E=L.E,
                              wfmt=3, n_shared=L.n_shared, debug=debug)
    tokens = np.asarray(tokens)
    sub = ids[tokens]
    used = np.unique(sub)
    remap = np.full(L.E, -1, np.int64)
    remap[used] = np.arange(len(used))
    sel = list(used) + ([L.E] if L.n_shared else [])
    idx = torch.tensor(sel, device=L.w13.device, dtype=torch.long)
    pick = lambda t: t.index_select(0, idx).cpu().numpy()
    tsel = torch.tensor(tokens, device=L.x.device, dtype=torch.long)
    return oracle.forward(synth.bf16_bits(L.x.index_select(0, tsel)), remap[sub].astype(np.int32),
                          L.topk_w.index_select(0, tsel).cpu().numpy(), pick(L.w13), pick(L.s13), pick(L.w2),
                          pick(L.s2), H=L.H, I=L.I, E=len(used), wfmt=3, n_shared=L.n_shared)


SMALL = [
    # name, cfg, seed, token-tile width the layer picks (from T*k/E, at most 32)
    ("tiny", dict(T=4, H=256, I=256, E=8, k=2), 71, 16),
    ("ragged_k4_bn32", dict(T=37, H=512, I=384, E=16, k=4), 72, 32),
    ("ragged_bn32", dict(T=70, H=384, I=256, E=6, k=2), 73, 32),
    ("shared", dict(T=9, H=256, I=384, E=5, k=3, n_shared=1), 74, 16),
    ("odd_kblocks", dict(T=21, H=640, I=384, E=7, k=2), 75, 16),
    ("one_token_k8", dict(T=1, H=1024, I=512, E=32, k=8), 76, 16),
]


@pytest.mark.parametrize("name,cfg,seed,bn", SMALL, ids=[s[0] for s in SMALL])
def test_mxfp4_a4_layer_small_all_elements(name, cfg, seed, bn):
    cfg = dict(cfg, wfmt=synth.WFMT_MXFP4_A4, routing="uniform")
    L = synth.make_layer(cfg, seed, device="cuda")
    layer, out = run_gpu(L)
    assert layer.device_status() == moe.MOE_OK
    assert layer.last_config()[0] == bn
    ref = oracle_ref(L, debug=True)
    assert_close(out.float().cpu().numpy(), ref["out_f32"], name)

    counts, offsets, perm, inv = layer.routing(L.T)
    P = int(offsets[-1])
    S = L.T * L.k
    tok = np.where(perm[:P] < S, perm[:P] // L.k, perm[:P] - S)
    xq, _, hq, _ = layer.activations(L.T)
    xsc, hsc = layer.block_scales(L.T)
    # step 2 (MXFP4): bit-exact per routed position
    assert np.array_equal(xsc[:P], ref["xsc"][tok])
    assert np.array_equal(xq[:P], ref["xq"][tok])
    # SwiGLU-output codes and exponents: equal to the oracle's except where the
    # summation order moves a value across a rounding midpoint or a power of two
    code_checks.assert_requant(code_checks.check_requant(L, layer, ref), name)


@pytest.mark.parametrize("bn", ["16", "32"])
def test_mxfp4_a4_both_tile_widths(bn, monkeypatch):
    monkeypatch.setenv("MOE_TILE_N", bn)
    L = synth.make_layer(dict(T=90, H=384, I=256, E=6, k=3, wfmt=3), 77, device="cuda")
    layer, out = run_gpu(L)
    assert layer.last_config()[0] == int(bn)
    assert layer.device_status() == moe.MOE_OK
    assert_close(out.float().cpu().numpy(), oracle_ref(L)["out_f32"], f"tile {bn}")


def test_mxfp4_a4_zero_input():
    L = synth.make_layer(dict(T=5, H=256, I=256, E=4, k=2, wfmt=3, n_shared=1), 78, device="cuda")
    layer = moe.MoeLayer(L.H, L.I, L.E, L.k, moe.MOE_WFMT_MXFP4_W4A4, max_T=8, n_shared=1)
    out = layer.forward(torch.zeros_like(L.x), L.ids, L.topk_w, L.w13, moe.pack_mxfp4_scales(L.s13), L.w2,
                        moe.pack_mxfp4_scales(L.s2))
    torch.cuda.synchronize()
    assert layer.device_status() == moe.MOE_OK
    assert not out.float().abs().max().item()


def test_mxfp4_a4_full_size_sampled():
    cfg = synth.EXTRA_CONFIGS[2]
    L = synth.make_layer(cfg, 2100, device="cuda")
    layer, out = run_gpu(L)
    assert layer.device_status() == moe.MOE_OK
    # every token (so every touched expert's every tile) against the oracle
    tokens = np.arange(L.T)
    ref = oracle_ref(L, tokens=tokens)["out_f32"]
    assert_close(out.float().cpu().numpy()[tokens], ref, cfg["name"])
    assert torch.isfinite(out.float()).all()
    # SwiGLU-output codes of the first and last position of a few experts
    code_checks.assert_requant(code_checks.check_requant(L, layer, None, code_checks.edge_positions(layer, L, 6)),
                               cfg["name"])
