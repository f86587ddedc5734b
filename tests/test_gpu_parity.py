"""GPU parity: the CUDA library through its C ABI against the CPU oracle.

Routing (counts, offsets, perm, inv) and the activation FP8 codes/scales are
compared bit for bit; layer outputs element by element with the layer's
tolerance |gpu - oracle| <= 2e-2 * max|oracle| + 1e-3 and cosine >= 0.9999.
Full-size workloads run in the launch configuration the benchmark times and
are checked on sampled tokens (an output row depends only on its own token).
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


def _need_gpu():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")


@pytest.fixture(scope="module", autouse=True)
def _setup():
    _need_gpu()
    from fp4_block_scaled_route_b200 import build
    build.build()
    yield


def assert_close(gpu, ref, what=""):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    assert gpu.shape == ref.shape
    scale = np.abs(ref).max()
    err = np.abs(gpu - ref).max()
    assert err <= RTOL * scale + ATOL, f"{what}: max err {err:.3e} vs bound {RTOL * scale + ATOL:.3e}"
    den = np.linalg.norm(gpu) * np.linalg.norm(ref)
    cos = 1.0 if den == 0 else float((gpu * ref).sum() / den)
    assert cos >= MIN_COS, f"{what}: cosine {cos:.6f}"
    return err / max(scale, 1e-30), cos


def gpu_weights(L):
    if L.wfmt == synth.WFMT_MXFP4:
        return L.w13, moe.pack_mxfp4_scales(L.s13), L.w2, moe.pack_mxfp4_scales(L.s2)
    return L.w13, L.s13, L.w2, L.s2


def run_gpu(L, ids=None, x=None, w=None, max_T=None):
    layer = moe.MoeLayer(L.H, L.I, L.E, L.k, L.wfmt, max_T=max_T or max(L.T, 1), n_shared=L.n_shared)
    w13, s13, w2, s2 = gpu_weights(L)
    ids = L.ids if ids is None else ids
    x = L.x if x is None else x
    w = L.topk_w if w is None else w
    out = layer.forward(x, ids, w, w13, s13, w2, s2)
    torch.cuda.synchronize()
    return layer, out


def oracle_full(L, ids=None, x=None, w=None, **kw):
    ids = (L.ids if ids is None else ids).cpu().numpy()
    x = L.x if x is None else x
    w = (L.topk_w if w is None else w).cpu().numpy()
    return oracle.forward(synth.bf16_bits(x), ids, w, L.w13.cpu().numpy(), L.s13.cpu().numpy(),
                          L.w2.cpu().numpy(), L.s2.cpu().numpy(), H=L.H, I=L.I, E=L.E, wfmt=L.wfmt,
                          n_shared=L.n_shared, **kw)


def oracle_sampled(L, tokens):
    """Oracle rows for `tokens` only, on the experts those tokens use."""
    tokens = np.asarray(tokens)
    ids = L.ids.cpu().numpy()[tokens]
    valid = (ids >= 0) & (ids < L.E)
    used = np.unique(ids[valid])
    remap = np.full(L.E, -1, np.int64)
    remap[used] = np.arange(len(used))
    ids_sub = np.where(valid, remap[np.clip(ids, 0, L.E - 1)], -1).astype(np.int32)
    sel = list(used) + ([L.E] if L.n_shared else [])
    idx = torch.tensor(sel, device=L.w13.device, dtype=torch.long)
    pick = lambda t: t.index_select(0, idx).cpu().numpy()
    tsel = torch.tensor(tokens, device=L.x.device, dtype=torch.long)
    res = oracle.forward(synth.bf16_bits(L.x.index_select(0, tsel)), ids_sub,
                         L.topk_w.index_select(0, tsel).cpu().numpy(), pick(L.w13), pick(L.s13),
                         pick(L.w2), pick(L.s2), H=L.H, I=L.I, E=max(len(used), 1), wfmt=L.wfmt,
                         n_shared=L.n_shared)
    return res["out_f32"]


def bf16_to_f32(t):
    return t.float().cpu().numpy()


# ---- step 1: routing, bit-exact -------------------------------------------------
ROUTE_CASES = [(c["T"], c["E"], c["k"], c["routing"], c.get("n_shared", 0), synth.config_seed(i))
               for i, c in enumerate(synth.CONFIGS)]
ROUTE_CASES += [(1, 256, 8, "uniform", 0, 1), (1, 1, 1, "uniform", 1, 2), (257, 7, 3, "uniform", 1, 3),
                (4096, 1024, 32, "uniform", 0, 4), (1000, 160, 8, "zipf1.2", 1, 5)]


@pytest.mark.parametrize("T,E,k,kind,nsh,seed", ROUTE_CASES)
def test_routing_bit_exact(T, E, k, kind, nsh, seed):
    ids, w = synth.make_routing(T, E, k, kind, seed)
    dev = "cuda"
    w13 = torch.zeros(E + nsh, 256, 128, dtype=torch.uint8, device=dev)
    s13 = torch.ones(E + nsh, 2, 1, dtype=torch.float32, device=dev)
    w2 = torch.zeros(E + nsh, 128, 128, dtype=torch.uint8, device=dev)
    s2 = torch.ones(E + nsh, 1, 1, dtype=torch.float32, device=dev)
    layer = moe.MoeLayer(128, 128, E, k, 0, max_T=T, n_shared=nsh)
    x = torch.zeros(T, 128, dtype=torch.bfloat16, device=dev)
    layer.forward(x, torch.from_numpy(ids).to(dev), torch.from_numpy(w).to(dev), w13, s13, w2, s2)
    counts, offsets, perm, inv = layer.routing(T)
    rc, ro, rp, ri, dropped = oracle.route(ids, E, nsh)
    assert dropped == 0
    assert np.array_equal(counts, rc)
    assert np.array_equal(offsets, ro)
    assert np.array_equal(perm, rp)
    assert np.array_equal(inv, ri)
    assert layer.device_status() == moe.MOE_OK


def test_routing_drops_bad_ids_and_reports():
    T, E, k = 6, 5, 2
    ids = np.array([[0, 5], [1, 1], [-1, 4], [2, 3], [4, 4], [7, 0]], np.int32)
    L = synth.make_layer(dict(T=T, H=256, I=128, E=E, k=k, wfmt=0), 77, device="cuda")
    layer, out = run_gpu(L, ids=torch.from_numpy(ids).cuda())
    counts, offsets, perm, inv = layer.routing(T)
    rc, ro, rp, ri, dropped = oracle.route(ids, E)
    assert dropped == 3
    assert np.array_equal(counts, rc) and np.array_equal(offsets, ro)
    assert np.array_equal(perm, rp) and np.array_equal(inv, ri)
    assert layer.device_status() == moe.MOE_ERR_BAD_ROUTING
    assert layer.device_status() == moe.MOE_OK  # cleared by the read
    ref = oracle_full(L, ids=torch.from_numpy(ids))
    assert_close(bf16_to_f32(out), ref["out_f32"], "dropped slots")


# ---- step 2: activation quantisation, bit-exact ------------------------------------
@pytest.mark.parametrize("T,H,E,k,nsh", [(4, 256, 8, 2, 0), (33, 7168, 256, 8, 0), (8, 4096, 160, 8, 1)])
def test_activation_codes_bit_exact(T, H, E, k, nsh):
    L = synth.make_layer(dict(T=T, H=H, I=128, E=E, k=k, wfmt=0, n_shared=nsh), 5 + T, device="cuda")
    layer, _ = run_gpu(L)
    counts, offsets, perm, inv = layer.routing(T)
    xq, xs, _, _ = layer.activations(T)
    rq, rs = oracle.quant_act(synth.bf16_bits(L.x))
    S = T * k
    P = offsets[-1]
    tok = np.where(perm[:P] < S, perm[:P] // k, perm[:P] - S)
    assert np.array_equal(xs[:P], rs[tok])
    assert np.array_equal(xq[:P], rq[tok])


# ---- the whole layer, small shapes, every output element ------------------------
SMALL = [
    # name, cfg, seed, token-tile width the layer picks (from T*k/E)
    ("config0_tiny", synth.CONFIGS[0], synth.config_seed(0), 16),
    ("ragged_bn32", dict(T=64, H=512, I=256, E=8, k=2, wfmt=0), 21, 32),
    ("ragged_bn64", dict(T=90, H=384, I=384, E=6, k=3, wfmt=0), 29, 64),
    ("ragged_k3_bn128", dict(T=100, H=384, I=384, E=6, k=3, wfmt=0), 22, 128),
    ("ragged_bn128", dict(T=300, H=256, I=256, E=16, k=4, wfmt=0), 23, 128),
    ("one_token", dict(T=1, H=1024, I=512, E=32, k=8, wfmt=0), 24, 16),
    ("shared_fp8", dict(T=10, H=256, I=256, E=6, k=2, wfmt=0, n_shared=1), 25, 16),
    ("mxfp4_small", dict(T=20, H=512, I=256, E=8, k=2, wfmt=1), 26, 16),
    ("mxfp4_ragged_bn64", dict(T=90, H=256, I=384, E=6, k=3, wfmt=1), 27, 64),
    ("mxfp4_shared", dict(T=7, H=384, I=256, E=5, k=2, wfmt=1, n_shared=1), 28, 16),
]


@pytest.mark.parametrize("name,cfg,seed,bn", SMALL, ids=[s[0] for s in SMALL])
def test_layer_small_all_elements(name, cfg, seed, bn):
    L = synth.make_layer(cfg, seed, device="cuda")
    layer, out = run_gpu(L)
    assert layer.device_status() == moe.MOE_OK
    assert layer.last_config()[0] == bn
    ref = oracle_full(L, debug=True)
    assert_close(bf16_to_f32(out), ref["out_f32"], name)
    # SwiGLU-output codes and scales: equal to the oracle's except where the
    # summation order moves a value across a rounding midpoint (code_checks)
    code_checks.assert_requant(code_checks.check_requant(L, layer, ref), name)


def test_all_tokens_to_one_expert_spans_tiles():
    T = 70
    L = synth.make_layer(dict(T=T, H=256, I=256, E=4, k=1, wfmt=0), 31, device="cuda")
    ids = torch.full((T, 1), 2, dtype=torch.int32, device="cuda")
    w = torch.ones(T, 1, dtype=torch.float32, device="cuda")
    layer, out = run_gpu(L, ids=ids, w=w)
    bn, _ = layer.last_config()
    assert T > bn
    ref = oracle_full(L, ids=ids, w=w)
    assert_close(bf16_to_f32(out), ref["out_f32"], "one expert")


def test_zero_input_and_zero_weights():
    L = synth.make_layer(dict(T=5, H=256, I=128, E=4, k=2, wfmt=0, n_shared=1), 32, device="cuda")
    _, out = run_gpu(L, x=torch.zeros_like(L.x))
    assert not out.float().abs().max().item()
    _, out = run_gpu(L, w=torch.zeros_like(L.topk_w))
    ref = oracle_full(L, w=torch.zeros_like(L.topk_w))
    assert_close(bf16_to_f32(out), ref["out_f32"], "shared only")


def test_token_count_limits():
    L = synth.make_layer(dict(T=8, H=256, I=128, E=4, k=2, wfmt=0), 33, device="cuda")
    layer = moe.MoeLayer(L.H, L.I, L.E, L.k, 0, max_T=8)
    out = torch.empty(8, 256, dtype=torch.bfloat16, device="cuda")
    args = [L.x.data_ptr(), L.ids.data_ptr(), L.topk_w.data_ptr(), L.w13.data_ptr(), L.s13.data_ptr(),
            L.w2.data_ptr(), L.s2.data_ptr(), out.data_ptr(), torch.cuda.current_stream().cuda_stream]
    assert moe.moe_forward(layer.ctx, 0, *args) == moe.MOE_OK
    assert moe.moe_forward(layer.ctx, 9, *args) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_forward(layer.ctx, 8, *args) == moe.MOE_OK
    torch.cuda.synchronize()


def test_repeated_calls_reuse_workspace():
    cfg = dict(T=16, H=256, I=256, E=8, k=2, wfmt=0)
    L1 = synth.make_layer(cfg, 41, device="cuda")
    L2 = synth.make_layer(cfg, 42, device="cuda")
    layer = moe.MoeLayer(256, 256, 8, 2, 0, max_T=16)
    o1 = layer.forward(L1.x, L1.ids, L1.topk_w, L1.w13, L1.s13, L1.w2, L1.s2).clone()
    o2 = layer.forward(L2.x[:9], L2.ids[:9], L2.topk_w[:9], L2.w13, L2.s13, L2.w2, L2.s2).clone()
    o3 = layer.forward(L1.x, L1.ids, L1.topk_w, L1.w13, L1.s13, L1.w2, L1.s2).clone()
    torch.cuda.synchronize()
    assert_close(bf16_to_f32(o1), oracle_full(L1)["out_f32"], "first")
    assert_close(bf16_to_f32(o3), oracle_full(L1)["out_f32"], "third")
    ref2 = oracle_full(L2, ids=L2.ids[:9], x=L2.x[:9], w=L2.topk_w[:9])
    # oracle_full with a 9-token slice
    assert_close(bf16_to_f32(o2), ref2["out_f32"], "second")


# ---- full-size workloads, sampled tokens ---------------------------------------------
FULL = [1, 2, 3, 4]


@pytest.mark.parametrize("cfg_idx", FULL, ids=[synth.CONFIGS[i]["name"] for i in FULL])
def test_full_size_sampled(cfg_idx):
    cfg = synth.CONFIGS[cfg_idx]
    L = synth.make_layer(cfg, synth.config_seed(cfg_idx), device="cuda")
    layer, out = run_gpu(L)
    assert layer.device_status() == moe.MOE_OK
    counts, offsets, perm, inv = layer.routing(L.T)
    if L.T <= 128:
        tokens = np.arange(L.T)  # every token, so every touched expert's every tile
    else:
        # the tokens holding each touched expert's first and last routing
        # position: every expert's first tile and its last (short) tile
        tok, grp = code_checks.position_map(perm, offsets, L.T, L.k)
        firsts = offsets[:-1][counts > 0]
        lasts = offsets[1:][counts > 0] - 1
        tokens = np.unique(np.concatenate([tok[firsts], tok[lasts], [L.T - 1]]))
        assert len(np.unique(grp[np.isin(tok, tokens)])) == int((counts > 0).sum())
    ref = oracle_sampled(L, tokens)
    got = bf16_to_f32(out)[tokens]
    assert_close(got, ref, cfg["name"])
    # properties at full size: every row finite; routing round trip
    assert torch.isfinite(out.float()).all()
    P = L.T * L.k + L.n_shared * L.T
    assert np.array_equal(inv[perm[:P]], np.arange(P))
    assert counts.sum() == P
    # SwiGLU-output codes of the first and last position of a few experts
    code_checks.assert_requant(code_checks.check_requant(L, layer, None, code_checks.edge_positions(layer, L, 6)),
                               cfg["name"])


# ---- both combine paths (fused fp32 reductions / stored rows + combine pass) ----
@pytest.mark.parametrize("mode", ["atomic", "rows"])
def test_combine_paths(mode, monkeypatch):
    monkeypatch.setenv("MOE_COMBINE", mode)
    cfg = dict(T=150, H=256, I=256, E=8, k=4, wfmt=0, n_shared=1)
    L = synth.make_layer(cfg, 61, device="cuda")
    layer, out = run_gpu(L)
    assert layer.device_status() == moe.MOE_OK
    assert_close(bf16_to_f32(out), oracle_full(L)["out_f32"], f"combine {mode}")


@pytest.mark.parametrize("bn", ["16", "32", "64", "128"])
def test_every_tile_width(bn, monkeypatch):
    monkeypatch.setenv("MOE_TILE_N", bn)
    cfg = dict(T=90, H=384, I=256, E=6, k=3, wfmt=0)
    L = synth.make_layer(cfg, 62, device="cuda")
    layer, out = run_gpu(L)
    assert layer.last_config()[0] == int(bn)
    assert_close(bf16_to_f32(out), oracle_full(L)["out_f32"], f"tile {bn}")


# ---- MXFP4 weights at every GEMM2 weight-tile count per stage -----------------
# 16-token tiles take four 128-row W2 tiles per stage where H % 512 == 0,
# else two where H % 256 == 0, else one; 32-token tiles two where
# H % 256 == 0.  GEMM1 keeps one gate/up pair per stage.
MX_TILES = [
    ("bn16_g2x4", "16", dict(T=40, H=1024, I=512, E=8, k=2, wfmt=1)),
    ("bn16_g2x2_shared", "16", dict(T=40, H=768, I=256, E=8, k=2, wfmt=1, n_shared=1)),
    ("bn16_g2x1", "16", dict(T=40, H=640, I=384, E=8, k=2, wfmt=1)),
    ("bn32_g2x2", "32", dict(T=90, H=768, I=256, E=6, k=3, wfmt=1)),
]


@pytest.mark.parametrize("name,bn,cfg", MX_TILES, ids=[m[0] for m in MX_TILES])
def test_mxfp4_weight_tiles_per_stage(name, bn, cfg, monkeypatch):
    monkeypatch.setenv("MOE_TILE_N", bn)
    L = synth.make_layer(dict(cfg, routing="uniform"), 63, device="cuda")
    layer, out = run_gpu(L)
    assert layer.last_config()[0] == int(bn)
    assert layer.device_status() == moe.MOE_OK
    assert_close(bf16_to_f32(out), oracle_full(L)["out_f32"], name)


# ---- 4-bit scales: only the packed layout is accepted ---------------------------
def test_mxfp4_refuses_scales_not_packed():
    """moe_forward with MXFP4 weights refuses scale buffers that no pack call
    wrote (plain [rows, K/32] scales would give wrong results silently), and
    accepts them once declared packed."""
    L = synth.make_layer(dict(T=6, H=256, I=256, E=4, k=2, wfmt=1), 64, device="cuda")
    layer = moe.MoeLayer(L.H, L.I, L.E, L.k, 1, max_T=8)
    out = torch.empty(L.T, L.H, dtype=torch.bfloat16, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    w13, s13, w2, s2 = gpu_weights(L)
    plain13, plain2 = L.s13.clone(), L.s2.clone()

    def call(a13, a2):
        return moe.moe_forward(layer.ctx, L.T, L.x.data_ptr(), L.ids.data_ptr(), L.topk_w.data_ptr(),
                               w13.data_ptr(), a13.data_ptr(), w2.data_ptr(), a2.data_ptr(), out.data_ptr(), st)

    assert call(plain13, s2) == moe.MOE_ERR_INVALID_ARG
    assert call(s13, plain2) == moe.MOE_ERR_INVALID_ARG
    assert call(s13, s2) == moe.MOE_OK
    torch.cuda.synchronize()
    assert_close(bf16_to_f32(out), oracle_full(L)["out_f32"], "packed")
    # a copy of packed scales (as if loaded from storage) is accepted once declared
    c13, c2 = s13.clone(), s2.clone()
    assert call(c13, c2) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_declare_packed_scales(c13.data_ptr(), c13.numel(), 1) == moe.MOE_OK
    assert moe.moe_declare_packed_scales(c2.data_ptr(), c2.numel(), 1) == moe.MOE_OK
    out.zero_()
    assert call(c13, c2) == moe.MOE_OK
    torch.cuda.synchronize()
    assert_close(bf16_to_f32(out), oracle_full(L)["out_f32"], "declared")
    assert layer.device_status() == moe.MOE_OK
