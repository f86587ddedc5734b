"""GPU parity of the NVFP4 path (moe_forward_nvfp4) against the CPU oracle.

- Activation quantisation (step 2, NVFP4 form): packed E2M1 codes, E4M3
  block codes and per-128 scales compared bit for bit (both sides take every
  decision in the same fp32 operations).
- SwiGLU-output codes: not bit-exact (the tensor cores sum in another order,
  which can move a value across a rounding boundary) but nearly all equal.
- Layer outputs element by element with the layer's tolerance
  |gpu - oracle| <= 2e-2 * max|oracle| + 1e-3 and cosine >= 0.9999; the
  full-size decode shapes on sampled tokens in the benchmark's launch
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


def run_gpu(L, ids=None, max_T=None):
    layer = moe.MoeLayer(L.H, L.I, L.E, L.k, L.wfmt, max_T=max_T or max(L.T, 1), n_shared=L.n_shared)
    s13, s2 = moe.pack_nvfp4_scales(L.s13), moe.pack_nvfp4_scales(L.s2)
    out = layer.forward(L.x, L.ids if ids is None else ids, L.topk_w, L.w13, s13, L.w2, s2, g13=L.g13, g2=L.g2)
    torch.cuda.synchronize()
    return layer, out


def oracle_ref(L, ids=None, debug=False, tokens=None):
    """Oracle output rows (all tokens, or `tokens` on the experts they use)."""
    ids = (L.ids if ids is None else ids).cpu().numpy()
    if tokens is None:
        return oracle.forward(synth.bf16_bits(L.x), ids, L.topk_w.cpu().numpy(), L.w13.cpu().numpy(),
                              L.s13.cpu().numpy(), L.w2.cpu().numpy(), L.s2.cpu().numpy(), H=L.H, I=L.I, E=L.E,
                              wfmt=2, n_shared=L.n_shared, g13=L.g13.cpu().numpy(), g2=L.g2.cpu().numpy(),
                              debug=debug)
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
                          pick(L.s2), H=L.H, I=L.I, E=len(used), wfmt=2, n_shared=L.n_shared, g13=pick(L.g13),
                          g2=pick(L.g2))


SMALL = [
    # name, cfg, seed, token-tile width the layer picks (from T*k/E, at most 32)
    ("tiny", dict(T=4, H=256, I=256, E=8, k=2), 51, 16),
    ("ragged_k4_bn32", dict(T=37, H=512, I=384, E=16, k=4), 52, 32),
    ("ragged_bn32", dict(T=70, H=384, I=256, E=6, k=2), 53, 32),
    ("shared", dict(T=9, H=256, I=384, E=5, k=3, n_shared=1), 54, 16),
    ("odd_kblocks", dict(T=21, H=640, I=384, E=7, k=2), 55, 16),      # H/128 = 5: last token-code box half past the row
    ("one_token_k8", dict(T=1, H=1024, I=512, E=32, k=8), 56, 16),
]


@pytest.mark.parametrize("name,cfg,seed,bn", SMALL, ids=[s[0] for s in SMALL])
def test_nvfp4_layer_small_all_elements(name, cfg, seed, bn):
    cfg = dict(cfg, wfmt=synth.WFMT_NVFP4, routing="uniform")
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
    xq, xs, hq, hs = layer.activations(L.T)
    xsc, hsc = layer.block_scales(L.T)
    # step 2 (NVFP4): bit-exact per routed position
    assert np.array_equal(xs[:P], ref["xs"][tok])
    assert np.array_equal(xsc[:P], ref["xsc"][tok])
    assert np.array_equal(xq[:P], ref["xq"][tok])
    # SwiGLU-output codes, block codes and scales: equal to the oracle's except
    # where the summation order moves a value across a rounding midpoint
    code_checks.assert_requant(code_checks.check_requant(L, layer, ref), name)


@pytest.mark.parametrize("bn", ["16", "32"])
def test_nvfp4_both_tile_widths(bn, monkeypatch):
    monkeypatch.setenv("MOE_TILE_N", bn)
    L = synth.make_layer(dict(T=90, H=384, I=256, E=6, k=3, wfmt=2), 57, device="cuda")
    layer, out = run_gpu(L)
    assert layer.last_config()[0] == int(bn)
    assert layer.device_status() == moe.MOE_OK
    assert_close(out.float().cpu().numpy(), oracle_ref(L)["out_f32"], f"tile {bn}")


def test_nvfp4_zero_input_and_entry_point_checks():
    L = synth.make_layer(dict(T=5, H=256, I=256, E=4, k=2, wfmt=2, n_shared=1), 58, device="cuda")
    layer = moe.MoeLayer(L.H, L.I, L.E, L.k, 2, max_T=8, n_shared=1)
    s13, s2 = moe.pack_nvfp4_scales(L.s13), moe.pack_nvfp4_scales(L.s2)
    out = layer.forward(torch.zeros_like(L.x), L.ids, L.topk_w, L.w13, s13, L.w2, s2, g13=L.g13, g2=L.g2)
    torch.cuda.synchronize()
    assert not out.float().abs().max().item()
    st = torch.cuda.current_stream().cuda_stream
    args = [L.x.data_ptr(), L.ids.data_ptr(), L.topk_w.data_ptr(), L.w13.data_ptr(), s13.data_ptr(),
            L.w2.data_ptr(), s2.data_ptr(), out.data_ptr(), st]
    # an NVFP4 context needs the global scales: moe_forward refuses it
    assert moe.moe_forward(layer.ctx, 5, *args) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_forward_nvfp4(layer.ctx, 5, L.x.data_ptr(), L.ids.data_ptr(), L.topk_w.data_ptr(),
                                 L.w13.data_ptr(), s13.data_ptr(), None, L.w2.data_ptr(), s2.data_ptr(),
                                 L.g2.data_ptr(), out.data_ptr(), st) == moe.MOE_ERR_INVALID_ARG
    fp8 = moe.MoeLayer(256, 256, 4, 2, 0, max_T=8)
    assert moe.moe_forward_nvfp4(fp8.ctx, 5, L.x.data_ptr(), L.ids.data_ptr(), L.topk_w.data_ptr(),
                                 L.w13.data_ptr(), s13.data_ptr(), L.g13.data_ptr(), L.w2.data_ptr(),
                                 s2.data_ptr(), L.g2.data_ptr(), out.data_ptr(), st) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_get_block_scales(fp8.ctx, None, None, st) == moe.MOE_ERR_UNSUPPORTED
    torch.cuda.synchronize()


NV_FULL = [c for c in synth.EXTRA_CONFIGS if c["wfmt"] == synth.WFMT_NVFP4]


@pytest.mark.parametrize("cfg", NV_FULL, ids=[c["name"] for c in NV_FULL])
def test_nvfp4_full_size_sampled(cfg):
    L = synth.make_layer(cfg, 2000 + cfg["T"], device="cuda")
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
