"""GPU parity of the CTA-pair GEMM1 (MOE_PAIR_MMA=1: MXFP4 weights, FP8
activations, 16-token tiles, tcgen05 MMAs with M = 256 over two SMs)
against the oracle.

- Routing and activation codes bit for bit (the dispatch kernels are the
  same as without the option).
- SwiGLU-output codes and scales by the midpoint rule (tests/code_checks.py).
- Layer outputs element by element with the layer tolerance
  |gpu - oracle| <= 2e-2 * max|oracle| + 1e-3 and cosine >= 0.9999; the
  full-size MXFP4 decode layer on the tokens holding each expert's first and
  last routing position.
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


@pytest.fixture(autouse=True)
def _pair(monkeypatch):
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from fp4_block_scaled_route_b200 import build
    build.build()
    monkeypatch.setenv("MOE_PAIR_MMA", "1")
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


def run(L, calls=1):
    layer = moe.MoeLayer(L.H, L.I, L.E, L.k, L.wfmt, max_T=L.T, n_shared=L.n_shared)
    s13, s2 = moe.pack_mxfp4_scales(L.s13), moe.pack_mxfp4_scales(L.s2)
    outs = []
    for _ in range(calls):
        outs.append(layer.forward(L.x, L.ids, L.topk_w, L.w13, s13, L.w2, s2).float().cpu().numpy())
        torch.cuda.synchronize()
        assert layer.device_status() == moe.MOE_OK
    return layer, outs


def oracle_ref(L, tokens=None):
    ids = L.ids.cpu().numpy()
    if tokens is None:
        return oracle.forward(synth.bf16_bits(L.x), ids, L.topk_w.cpu().numpy(), L.w13.cpu().numpy(),
                              L.s13.cpu().numpy(), L.w2.cpu().numpy(), L.s2.cpu().numpy(), H=L.H, I=L.I, E=L.E,
                              wfmt=L.wfmt, n_shared=L.n_shared, debug=True)
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
                          pick(L.s2), H=L.H, I=L.I, E=len(used), wfmt=L.wfmt, n_shared=L.n_shared)["out_f32"]


SMALL = [
    ("tiny", dict(T=4, H=256, I=256, E=8, k=2), 91),
    ("ragged", dict(T=21, H=640, I=384, E=7, k=2), 92),            # tiles of 1..16 positions, odd K blocks
    ("shared", dict(T=12, H=512, I=512, E=8, k=2, n_shared=1), 93),  # a 12-position shared-expert tile
    ("dense", dict(T=64, H=512, I=256, E=16, k=2), 94),            # ~8 positions per expert, some tiles near full
    ("many_units", dict(T=32, H=1024, I=2048, E=64, k=4), 95),     # several units per pair, deep K
]


@pytest.mark.parametrize("name,cfg,seed", SMALL, ids=[s[0] for s in SMALL])
def test_pair_gemm1_small_all_elements(name, cfg, seed):
    L = synth.make_layer(dict(cfg, wfmt=synth.WFMT_MXFP4, routing="uniform"), seed, device="cuda")
    layer, outs = run(L, calls=2)
    assert layer.last_config()[0] == 16
    ref = oracle_ref(L)
    for i, out in enumerate(outs):
        assert_close(out, ref["out_f32"], f"{name} call {i}")
    counts, offsets, perm, inv = layer.routing(L.T)
    rc, ro, rp, ri, _ = oracle.route(L.ids.cpu().numpy(), L.E, L.n_shared)
    assert np.array_equal(counts, rc) and np.array_equal(perm, rp) and np.array_equal(inv, ri)
    code_checks.assert_requant(code_checks.check_requant(L, layer, ref), name)


def test_pair_gemm1_full_size_decode():
    """MXFP4 decode T=128, H=7168, E=256, k=8, I=2048: the tokens holding each
    expert's first and last routing position, every row finite, SwiGLU-output
    codes of a few experts' edges."""
    cfg = synth.CONFIGS[2]
    L = synth.make_layer(cfg, synth.config_seed(2), device="cuda")
    layer, outs = run(L)
    assert layer.last_config()[0] == 16
    counts, offsets, perm, inv = layer.routing(L.T)
    tok, _ = code_checks.position_map(perm, offsets, L.T, L.k)
    firsts = offsets[:-1][counts > 0]
    lasts = offsets[1:][counts > 0] - 1
    tokens = np.unique(np.concatenate([tok[firsts], tok[lasts], [L.T - 1]]))
    assert_close(outs[0][tokens], oracle_ref(L, tokens), cfg["name"])
    assert np.isfinite(outs[0]).all()
    code_checks.assert_requant(code_checks.check_requant(L, layer, None, code_checks.edge_positions(layer, L, 6)),
                               cfg["name"])
