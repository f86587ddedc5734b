"""The byte and FLOP counts behind bench.py's roofline fractions, pinned to
something other than their own formulas (CPU only).

- Weight bytes per expert: the sizes of the weight and scale tensors the
  seeded generator makes for a layer (what a forward call reads for one
  expert), for every weight format.  GEMM1's share: the W13 tensors alone.
- Touched experts: a set of the valid ids, with dropped and duplicate ids.
- FLOPs: two per multiply-add of every routed position through GEMM1
  (2I x H) and GEMM2 (H x I), counted position by position.
"""
import numpy as np
import pytest

import bench
from fp4_block_scaled_route_b200 import synth

FORMATS = [synth.WFMT_FP8, synth.WFMT_MXFP4, synth.WFMT_NVFP4, synth.WFMT_MXFP4_A4, synth.WFMT_MXFP8]


def _nbytes(*ts):
    return sum(int(t.numel()) * t.element_size() for t in ts if t is not None)


@pytest.mark.parametrize("wfmt", FORMATS)
@pytest.mark.parametrize("nsh", [0, 1])
def test_weight_bytes_equal_the_generated_tensors(wfmt, nsh):
    L = synth.make_layer(dict(T=3, H=384, I=256, E=5, k=2, wfmt=wfmt, n_shared=nsh), 31 + wfmt)
    NE = L.E + L.n_shared
    assert L.w13.shape[0] == NE and L.w2.shape[0] == NE
    whole = _nbytes(L.w13, L.s13, L.w2, L.s2, L.g13, L.g2)
    gemm1 = _nbytes(L.w13, L.s13, L.g13)
    assert whole % NE == 0 and gemm1 % NE == 0
    assert bench.weight_bytes_per_expert(L) == whole // NE
    assert bench.gemm1_weight_bytes_per_expert(L) == gemm1 // NE


def test_touched_experts_counts_distinct_valid_ids():
    ids = np.array([[0, 5], [1, 1], [-1, 9], [2, 3], [4, 4], [7, 0]], np.int32)
    assert bench.touched_experts(ids, 5) == len({int(v) for v in ids.ravel() if 0 <= v < 5})
    assert bench.touched_experts(np.full((4, 2), -1, np.int32), 5) == 0


@pytest.mark.parametrize("wfmt", FORMATS)
def test_workload_stats_counts(wfmt):
    L = synth.make_layer(dict(T=6, H=256, I=384, E=7, k=3, wfmt=wfmt, n_shared=1), 41 + wfmt)
    ids = L.ids.numpy()
    st = bench.workload_stats(L, ids)
    used = {int(v) for v in ids.ravel()}
    assert st["experts_touched"] == len(used) + 1
    assert st["weight_bytes"] == st["experts_touched"] * bench.weight_bytes_per_expert(L)
    positions = [(t, j) for t in range(L.T) for j in range(L.k)] + [(t, "shared") for t in range(L.T)]
    assert st["positions"] == len(positions)
    flops = 0
    for _ in positions:
        flops += 2 * (2 * L.I) * L.H   # GEMM1: gate and up rows over K = H
        flops += 2 * L.H * L.I         # GEMM2: H rows over K = I
    assert st["flops"] == flops
    # GEMM1's bytes: its weights, plus activations in and SwiGLU outputs out
    assert st["gemm1_bytes"] > st["experts_touched"] * bench.gemm1_weight_bytes_per_expert(L)


def test_decode_fp8_gemm1_bytes_closed_form():
    """FP8 decode T=32, H=7168, E=256, k=8, I=2048 with the seeded routing:
    per touched expert 2I x H weight bytes plus one fp32 scale per 128 x 128
    block; per routed position H + I code bytes and one fp32 scale per 128."""
    cfg = synth.CONFIGS[1]
    ids, _ = synth.make_routing(cfg["T"], cfg["E"], cfg["k"], cfg.get("routing", "uniform"), synth.config_seed(1))

    class Shape:
        T, H, E, k, I, wfmt, n_shared = cfg["T"], cfg["H"], cfg["E"], cfg["k"], cfg["I"], cfg["wfmt"], 0

    st = bench.workload_stats(Shape, ids)
    n = len(np.unique(ids))
    H, I, P = 7168, 2048, 32 * 8
    assert st["gemm1_bytes"] == n * (2 * I * H + (2 * I // 128) * (H // 128) * 4) + P * (H + I + (H // 128 + I // 128) * 4)
    # the figures the bench line reports for this layer (165 experts touched)
    assert (n, st["gemm1_bytes"], st["weight_bytes"]) == (165, 4_848_036_864, 7_268_405_760)


def test_small_layers_are_timed_l2_cold():
    """The bench flushes the L2 between timed calls of a layer whose weight
    stream is under 8 x the 126 MB L2: the tiny and Zipf decode layers
    (their weights fit, wholly or mostly, in the L2); the others stream
    gigabytes per call and are not flushed."""
    flushed = {}
    for i, cfg in enumerate(synth.CONFIGS + synth.EXTRA_CONFIGS):
        ids, _ = synth.make_routing(cfg["T"], cfg["E"], cfg["k"], cfg.get("routing", "uniform"), synth.config_seed(i))

        class Shape:
            T, H, E, k, I, wfmt = cfg["T"], cfg["H"], cfg["E"], cfg["k"], cfg["I"], cfg["wfmt"]
            n_shared = cfg.get("n_shared", 0)

        flushed[cfg["name"]] = bench.workload_stats(Shape, ids)["weight_bytes"] < bench.FLUSH_BELOW_BYTES
    assert {n for n, f in flushed.items() if f} == {synth.CONFIGS[0]["name"], synth.CONFIGS[3]["name"]}
    assert bench.FLUSH_BELOW_BYTES == 8 * bench.L2_BYTES and bench.L2_BYTES >= 126 * 10**6
