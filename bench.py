#!/usr/bin/env python
"""Benchmark of the decode-regime MoE layer on B200.

One step = one full MoE layer (route, activation quant, GEMM1 + SwiGLU +
requant, GEMM2 + weighted combine, bf16 output) over one batch of seeded
synthetic inputs, through the C ABI.  Default workload: the FP8 decode layer
T=32, H=7168, E=256, top-k=8, I=2048.  Metric: weight-stream GB/s (bytes of
the weights and scales of every expert the step touches, divided by the step
time); microseconds per layer and TFLOP/s ride along.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload IDX] [--impl reference]

With N > 1 (launched by torchrun) every rank runs an independent replica of
the layer on its own GPU (the single-GPU path has no exchange step); the
value is the sum over ranks of the bytes streamed divided by the slowest
rank's time.  Rank 0 prints one JSON line on stdout.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE layer µs and weight-stream HBM GB/s (vs ~8 TB/s) at T=1–256; TFLOP/s at T=4096"
L2_BYTES = 126 * 1000 * 1000
# a workload whose weights streamed per step are below this is timed with the
# L2 flushed between steps (a 2 x L2 buffer written outside the timed events)
FLUSH_BELOW_BYTES = 8 * L2_BYTES
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
CSRC = "fp4_block_scaled_route_b200/csrc/"
# sources of the decode GEMM kernel (moe_gemm_kernel); a traffic record may
# name its own list (the token-major kernel: moe_gemm_tm.cu + moe_ptx.cuh)
GEMM_SOURCES = [CSRC + "moe_gemm.cu", CSRC + "moe_ptx.cuh"]


def log(*a):
    print(*a, file=sys.stderr, flush=True)


# ---------------------------------------------------------------------------
def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", type=int, default=1,
                    help="index into synth.CONFIGS (0-4), then synth.EXTRA_CONFIGS (5: NVFP4 T=128, 6: NVFP4 T=32, "
                         "7: MXFP4 weights and activations T=128, 8: MXFP8 prefill T=4096)")
    ap.add_argument("--shape", default=None,
                    help="custom layer T,H,E,k,I,fmt[,n_shared] (fmt fp8|mxfp4|nvfp4|mxfp4a4|mxfp8) instead of --workload")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--router", action="store_true",
                    help="also time the fused router (moe_router_topk) on seeded router weights of this shape")
    ap.add_argument("--green-ctx", type=int, default=0,
                    help="run the dispatch kernels in a green context of >= N SMs and the GEMMs on the rest")
    ap.add_argument("--dispatch-ctas", type=int, default=0,
                    help="dispatch overlap: the last N CTAs of the GEMM1 launch quantise the activations and "
                         "publish per-expert ready counters (one cooperative launch); 0 = off")
    ap.add_argument("--workloads", default=None,
                    help="comma-separated workload indices also timed (one GPU only) and reported under "
                         "'workloads' in the same JSON line; default: every other workload when the headline is "
                         "the default one, none otherwise; 'none' for none")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


def gemm_source_hash(sources=None) -> str:
    h = hashlib.sha256()
    for rel in sources or GEMM_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload_name: str):
    """Per-launch DRAM bytes of the GEMM1 kernel from the committed ncu summary,
    or None when there is none or the kernel sources changed since."""
    path = os.path.join(ROOT, "profiles", f"gemm1_{workload_name}_traffic.txt")
    if not os.path.exists(path):
        return None
    vals = {}
    with open(path) as f:
        for line in f:
            if ":" in line and not line.startswith("#"):
                k, v = line.split(":", 1)
                vals[k.strip()] = v.strip()
    sources = [CSRC + n for n in vals["kernel_sources"].split()] if "kernel_sources" in vals else None
    if vals.get("kernel_source_sha256_16") != gemm_source_hash(sources):
        return None
    try:
        return float(vals["dram_bytes_per_launch_full_size"])
    except (KeyError, ValueError):
        return None


# ---------------------------------------------------------------------------
class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str | None):
        self.lines = []
        self.proc = None
        try:
            cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "50"]
            if gpu_id:
                cmd += ["-i", gpu_id]
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.th = threading.Thread(target=self._read, daemon=True)
            self.th.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def wait_first(self, timeout=3.0):
        t0 = time.time()
        while self.proc and not self.lines and time.time() - t0 < timeout:
            time.sleep(0.01)

    def mark(self):
        return time.time()

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=2)
            except Exception:
                self.proc.kill()

    def summary(self, t0, t1):
        rows = [l for (t, l) in self.lines if t0 <= t <= t1]
        if not rows:
            rows = [l for (t, l) in self.lines if t0 - 0.1 <= t <= t1 + 0.1]
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            parts = [p.strip() for p in r.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for name, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def gpu_uuid(dev):
    import torch
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return None


# ---------------------------------------------------------------------------
WFMT_NAMES = ["fp8_e4m3_b128", "mxfp4_e2m1_e8m0_k32", "nvfp4_e2m1_e4m3_k16", "mxfp4_w4a4_e2m1_e8m0_k32",
              "mxfp8_e4m3_e8m0_k32"]
DTYPES = ["fp8_e4m3", "mxfp4_e2m1 x fp8_e4m3", "nvfp4_e2m1 x nvfp4_e2m1", "mxfp4_e2m1 x mxfp4_e2m1",
          "mxfp8_e4m3 x mxfp8_e4m3"]


def weight_bytes_per_expert(L) -> int:
    H, I = L.H, L.I
    if L.wfmt == 0:
        return 2 * I * H + (2 * I // 128) * (H // 128) * 4 + H * I + (H // 128) * (I // 128) * 4
    if L.wfmt == 2:  # E2M1 nibbles, one E4M3 code per 16, one fp32 global scale per matrix
        return 2 * I * H // 2 + 2 * I * H // 16 + 4 + H * I // 2 + H * I // 16 + 4
    if L.wfmt == 4:  # E4M3 bytes, one E8M0 code per 32
        return 2 * I * H + 2 * I * H // 32 + H * I + H * I // 32
    return 2 * I * H // 2 + 2 * I * H // 32 + H * I // 2 + H * I // 32


def gemm1_weight_bytes_per_expert(L) -> int:
    H, I = L.H, L.I
    if L.wfmt == 0:
        return 2 * I * H + (2 * I // 128) * (H // 128) * 4
    if L.wfmt == 2:
        return 2 * I * H // 2 + 2 * I * H // 16 + 4
    if L.wfmt == 4:
        return 2 * I * H + 2 * I * H // 32
    return 2 * I * H // 2 + 2 * I * H // 32


def touched_experts(ids: np.ndarray, E: int) -> int:
    v = ids[(ids >= 0) & (ids < E)]
    return int(np.unique(v).size)


def workload_stats(L, ids_np):
    n_exp = touched_experts(ids_np, L.E) + L.n_shared
    P = L.T * L.k + L.n_shared * L.T
    wbytes = n_exp * weight_bytes_per_expert(L)
    flops = 2.0 * P * 3 * L.I * L.H
    if L.wfmt == 2:  # activations in and out as NVFP4: nibbles, block codes, per-128 scales
        act = P * (L.H // 2 + L.H // 16 + (L.H // 128) * 4 + L.I // 2 + L.I // 16 + (L.I // 128) * 4)
    elif L.wfmt == 3:  # activations in and out as MXFP4: nibbles and E8M0 codes
        act = P * (L.H // 2 + L.H // 32 + L.I // 2 + L.I // 32)
    elif L.wfmt == 4:  # activations in and out as MXFP8: bytes and E8M0 codes
        act = P * (L.H + L.H // 32 + L.I + L.I // 32)
    else:
        act = P * L.H + P * (L.H // 128) * 4 + P * L.I + P * (L.I // 128) * 4
    g1 = n_exp * gemm1_weight_bytes_per_expert(L) + act
    return dict(experts_touched=n_exp, weight_bytes=wbytes, flops=flops, gemm1_bytes=g1, positions=P)


def build_layer(args, device):
    from fp4_block_scaled_route_b200 import synth
    if args.shape:
        f = args.shape.split(",")
        T, H, E, k, I = (int(v) for v in f[:5])
        wfmt = {"fp8": synth.WFMT_FP8, "mxfp4": synth.WFMT_MXFP4, "nvfp4": synth.WFMT_NVFP4,
                "mxfp4a4": synth.WFMT_MXFP4_A4, "mxfp8": synth.WFMT_MXFP8}[f[5]]
        nsh = int(f[6]) if len(f) > 6 else 0
        cfg = dict(name=f"custom_T{T}_H{H}_E{E}_k{k}_I{I}_{f[5]}" + ("_shared" if nsh else ""), T=T, H=H, E=E,
                   k=k, I=I, wfmt=wfmt, routing="uniform", n_shared=nsh)
        return cfg, synth.make_layer(cfg, 2000, device=device)
    allc = synth.CONFIGS + synth.EXTRA_CONFIGS
    cfg = allc[args.workload]
    L = synth.make_layer(cfg, synth.config_seed(args.workload), device=device)
    return cfg, L


def launches_per_call(L, dispatch_overlap: bool = False) -> int:
    """Kernels one moe_forward call launches: the route (from 4096 routed
    slots on two kernels, per-chunk expert counts and then the scatter), the
    quantisation (none with dispatch overlap, where GEMM1 quantises), GEMM1,
    GEMM2 and the bf16 output pass."""
    route = 2 if L.T * L.k >= 4096 else 1
    return route + (0 if dispatch_overlap else 1) + 3


def gpu_operands(L):
    """The layer's weights in the form moe_forward reads (MXFP4 / NVFP4 scales
    packed once, as at weight-load time) and the NVFP4 global scales."""
    from fp4_block_scaled_route_b200 import moe, synth
    if L.wfmt in (synth.WFMT_MXFP4, synth.WFMT_MXFP4_A4, synth.WFMT_MXFP8):  # E8M0 atoms
        w = (L.w13, moe.pack_mxfp4_scales(L.s13), L.w2, moe.pack_mxfp4_scales(L.s2))
    elif L.wfmt == synth.WFMT_NVFP4:
        w = (L.w13, moe.pack_nvfp4_scales(L.s13), L.w2, moe.pack_nvfp4_scales(L.s2))
    else:
        w = (L.w13, L.s13, L.w2, L.s2)
    gsc = dict(g13=L.g13, g2=L.g2) if L.wfmt == synth.WFMT_NVFP4 else {}
    return w, gsc


def l2_label(weight_bytes: int, flush: bool) -> str:
    if flush:
        return (f"L2 flushed between timed steps ({2 * L2_BYTES // 10**6} MB written outside the per-step events; "
                f"weights streamed per step {weight_bytes / 1e6:.1f} MB)")
    return (f"inputs larger than L2 (weights streamed per step {weight_bytes / 1e9:.2f} GB, more than 8 x the "
            f"126 MB L2); no flush")


def time_steps(step, steps: int, stream, flush_buf=None) -> float:
    """Device milliseconds of `steps` calls of step() on `stream` (CUDA events).
    With flush_buf, every call has its own event pair and the buffer (larger
    than the L2) is rewritten between calls, outside the pairs."""
    import torch
    if flush_buf is None:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            step()
        e1.record(stream)
        e1.synchronize()
        return e0.elapsed_time(e1)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    with torch.cuda.stream(stream):
        for i in range(steps):
            flush_buf.fill_(i & 0xFF)
            evs[i][0].record(stream)
            step()
            evs[i][1].record(stream)
    evs[-1][1].synchronize()
    return sum(a.elapsed_time(b) for a, b in evs)


def workload_record(idx: int, args, dev, stream, sampler):
    """One workload of synth.CONFIGS + synth.EXTRA_CONFIGS timed on this GPU:
    microseconds per layer, weight GB/s, TFLOP/s, the fraction of the
    roofline max(weight bytes / HBM peak, FLOP / dense tensor peak), GEMM1's
    own rate from per-kernel events, and the clocks seen."""
    import torch
    from fp4_block_scaled_route_b200 import moe, synth
    allc = synth.CONFIGS + synth.EXTRA_CONFIGS
    cfg = allc[idx]
    L = synth.make_layer(cfg, synth.config_seed(idx), device=dev)
    st = workload_stats(L, L.ids.cpu().numpy())
    layer = moe.MoeLayer(L.H, L.I, L.E, L.k, L.wfmt, max_T=L.T, n_shared=L.n_shared)
    (w13, s13, w2, s2), gsc = gpu_operands(L)
    out = torch.empty(L.T, L.H, dtype=torch.bfloat16, device=dev)

    def step():
        layer.forward(L.x, L.ids, L.topk_w, w13, s13, w2, s2, out=out, stream=stream, **gsc)

    flush = st["weight_bytes"] < FLUSH_BELOW_BYTES
    flush_buf = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev) if flush else None
    steps = max(args.steps, 100) if flush else args.steps
    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize(dev)
    t0 = time.time()
    ms = time_steps(step, steps, stream, flush_buf)
    t1 = time.time()
    moe.moe_profile_enable(layer.ctx, 1)
    time_steps(step, steps, stream, flush_buf)
    stage_ms, _ = moe.moe_profile_read(layer.ctx)
    moe.moe_profile_enable(layer.ctx, 0)
    if layer.device_status() != moe.MOE_OK:
        raise RuntimeError(f"device status not OK after workload {cfg['name']}")
    hbm, bf16, src = peaks()
    ratio = 4.0 if L.wfmt in (synth.WFMT_NVFP4, synth.WFMT_MXFP4_A4) else 2.0
    tpeak = ratio * bf16
    us = ms / steps * 1e3
    floor_us = max(st["weight_bytes"] / (hbm * 1e9), st["flops"] / (tpeak * 1e12)) * 1e6
    g1 = stage_ms[2]
    g1_flops = 2.0 * st["positions"] * 2 * L.I * L.H
    rec = {
        "workload": cfg["name"], "T": L.T, "H": L.H, "E": L.E, "k": L.k, "I": L.I, "wfmt": WFMT_NAMES[L.wfmt],
        "n_shared": L.n_shared, "dtype": DTYPES[L.wfmt], "experts_touched": st["experts_touched"],
        "weight_bytes_per_step": st["weight_bytes"], "flop_per_step": st["flops"],
        "us_per_layer": us, "weight_GBps": st["weight_bytes"] / (us * 1e-6) / 1e9,
        "hbm_frac": st["weight_bytes"] / (us * 1e-6) / 1e9 / hbm,
        "tflops": st["flops"] / (us * 1e-6) / 1e12, "tensor_frac": st["flops"] / (us * 1e-6) / 1e12 / tpeak,
        "roofline_us": floor_us, "roofline_frac": floor_us / us,
        "roofline_bound": "hbm" if st["weight_bytes"] / hbm >= st["flops"] / (tpeak * 1e3) else "tensor",
        "gemm1": {"ms": g1, "GBps": st["gemm1_bytes"] / (g1 * 1e-3) / 1e9 if g1 > 0 else None,
                  "hbm_frac": st["gemm1_bytes"] / (g1 * 1e-3) / 1e9 / hbm if g1 > 0 else None,
                  "tflops": g1_flops / (g1 * 1e-3) / 1e12 if g1 > 0 else None,
                  "tensor_frac": g1_flops / (g1 * 1e-3) / 1e12 / tpeak if g1 > 0 else None,
                  "traffic": recorded_traffic(cfg["name"]), "algorithmic_bytes_per_launch": st["gemm1_bytes"]},
        "stage_ms": dict(zip(moe.STAGE_NAMES, stage_ms)),
        "peaks": {"hbm_gbs": hbm, "tensor_tflops": tpeak,
                  "source": f"{src} hbm_gbs; {src} bf16_tflops x {ratio:g} ({'FP4' if ratio == 4 else 'FP8'}/bf16 "
                            f"nominal ratio)"},
        "l2": l2_label(st["weight_bytes"], flush), "steps": steps, "warmup": max(args.warmup, 3),
        "gpu_launches": launches_per_call(L) * steps, "clocks": sampler.summary(t0, t1),
    }
    layer.close()
    del L, out, flush_buf, w13, s13, w2, s2, gsc
    torch.cuda.empty_cache()
    return rec


# ---------------------------------------------------------------------------
def replica_throughput(dist, device, local_ms: float, local_bytes: float, steps: int):
    """Whole-job rate of independent replicas: the slowest rank's device time
    (max over ranks) and the bytes all ranks streamed (sum over ranks).
    Returns (ms_max, bytes_total, GB/s)."""
    ms, nbytes = float(local_ms), float(local_bytes)
    if dist is not None:
        import torch
        t = torch.tensor([ms], device=device, dtype=torch.float64)
        b = torch.tensor([nbytes], device=device, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        dist.all_reduce(b, op=dist.ReduceOp.SUM)
        ms, nbytes = float(t.item()), float(b.item())
    return ms, nbytes, nbytes / (ms / steps * 1e-3) / 1e9


# ---------------------------------------------------------------------------
def cpu_baseline(L, min_seconds=10.0, max_slots=None):
    """The oracle on a bounded sample of the workload, repeated until about
    min_seconds of CPU time: the first n (token, expert) slots, n doubling from
    8 until one pass takes >= 1 s or covers every slot."""
    S = L.T * L.k
    n = min(8, S)
    while True:
        dt, nbytes, nexp, cores = cpu_baseline_sample(L, n)
        if dt >= 1.0 or n >= S or (max_slots and n >= max_slots):
            break
        n = min(S, 2 * n)
    reps, tot_t, tot_b = 1, dt, nbytes
    while tot_t < min_seconds:
        dt, nbytes, _, _ = cpu_baseline_sample(L, n)
        reps += 1
        tot_t += dt
        tot_b += nbytes
    return {"value": tot_b / tot_t / 1e9, "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"first {n} of {S} (token, expert) slots of the workload ({nexp} expert FFNs, "
                      f"{nbytes / 1e9:.2f} GB of weights per pass), {reps} passes, {tot_t:.1f} s",
            "seconds": tot_t}


def cpu_baseline_sample(L, n_slots: int):
    """Oracle on the first n_slots (token, expert) pairs of the workload."""
    import oracle
    import torch
    from fp4_block_scaled_route_b200 import synth
    ids = L.ids.cpu().numpy()
    w = L.topk_w.cpu().numpy()
    slots = [(t, j) for t in range(L.T) for j in range(L.k)][:n_slots]
    experts = sorted({int(ids[t, j]) for (t, j) in slots})
    idx = torch.tensor(experts, device=L.w13.device)
    pick = lambda a: a.index_select(0, idx).cpu().numpy()
    w13, s13, w2, s2 = pick(L.w13), pick(L.s13), pick(L.w2), pick(L.s2)
    gs = dict(g13=pick(L.g13), g2=pick(L.g2)) if L.g13 is not None else {}
    remap = {e: i for i, e in enumerate(experts)}
    toks = sorted({t for (t, _) in slots})
    x = synth.bf16_bits(L.x[toks])
    ids_s = np.full((len(toks), L.k), -1, np.int32)
    w_s = np.zeros((len(toks), L.k), np.float32)
    for (t, j) in slots:
        ids_s[toks.index(t), j] = remap[int(ids[t, j])]
        w_s[toks.index(t), j] = w[t, j]
    t0 = time.perf_counter()
    oracle.forward(x, ids_s, w_s, w13, s13, w2, s2, H=L.H, I=L.I, E=len(experts), wfmt=L.wfmt, n_shared=0, **gs)
    dt = time.perf_counter() - t0
    nbytes = len(experts) * weight_bytes_per_expert(L)
    return dt, nbytes, len(experts), oracle.num_threads()


def run_reference(args):
    """The oracle, as it stands, on the host cores (rank 0 only)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import torch
    from fp4_block_scaled_route_b200 import synth
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    cfg, L = build_layer(args, dev)
    # per step: one (token, expert) slot, the smallest unit of the workload
    times, nb = [], 0
    for i in range(args.warmup + args.steps):
        dt, nbytes, _, cores = cpu_baseline_sample(L, 1)
        if i >= args.warmup:
            times.append(dt)
            nb += nbytes
    total = sum(times)
    value = nb / total / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded)",
        "config": {"workload": cfg["name"], "T": cfg["T"], "H": cfg["H"], "E": cfg["E"], "k": cfg["k"],
                   "I": cfg["I"], "wfmt": WFMT_NAMES[cfg["wfmt"]], "parallelism": "replicas"},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": "per step one (token, expert) slot of the workload: one expert FFN on one token"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
def time_router(args, L, layer, dev, stream):
    """The fused router (logits GEMM + top-k + softmax, one kernel) on seeded
    bf16 router weights of the layer's shape, timed with CUDA events; the
    roofline is the larger of its HBM time (x and router weights read once)
    and its bf16 tensor time."""
    import torch
    from fp4_block_scaled_route_b200 import synth
    _, wr = synth.make_router(L.T, L.H, L.E, 4242, device=dev)
    ids = torch.empty(L.T, L.k, dtype=torch.int32, device=dev)
    w = torch.empty(L.T, L.k, dtype=torch.float32, device=dev)
    for _ in range(5):
        layer.router(L.x, wr, ids, w, stream=stream)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        layer.router(L.x, wr, ids, w, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / args.steps
    hbm, bf16, src = peaks()
    nbytes = L.T * L.H * 2 + L.E * L.H * 2 + L.T * L.k * 8
    flops = 2.0 * L.T * L.H * L.E
    floor_ms = max(nbytes / (hbm * 1e9), flops / (bf16 * 1e12)) * 1e3
    return {"us": ms * 1e3, "bytes": nbytes, "GBps": nbytes / (ms * 1e-3) / 1e9, "tflops": flops / (ms * 1e-3) / 1e12,
            "roofline_us": floor_ms * 1e3, "frac": floor_ms / ms, "peak_source": f"{src} hbm_gbs / bf16_tflops",
            "launches_per_call": 1}


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
        return

    import torch
    from fp4_block_scaled_route_b200 import build as moe_build
    from fp4_block_scaled_route_b200 import moe, synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    if rank == 0:
        moe_build.build()
    if dist:
        dist.barrier()

    cfg, L = build_layer(args, dev)
    ids_np = L.ids.cpu().numpy()
    st = workload_stats(L, ids_np)
    layer = moe.MoeLayer(L.H, L.I, L.E, L.k, L.wfmt, max_T=L.T, n_shared=L.n_shared)
    green = layer.set_green_ctx(args.green_ctx) if args.green_ctx else None
    disp = layer.set_dispatch_overlap(args.dispatch_ctas) if args.dispatch_ctas else None
    (w13, s13, w2, s2), gsc = gpu_operands(L)
    out = torch.empty(L.T, L.H, dtype=torch.bfloat16, device=dev)
    flush = st["weight_bytes"] < FLUSH_BELOW_BYTES
    flush_buf = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev) if flush else None
    stream = torch.cuda.current_stream(dev)

    def step():
        layer.forward(L.x, L.ids, L.topk_w, w13, s13, w2, s2, out=out, stream=stream, **gsc)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize(dev)
    if layer.device_status() != moe.MOE_OK:
        raise RuntimeError("device status not OK after warm-up")

    # ---- timed region (device events, max over ranks) ----
    sampler = ClockSampler(gpu_uuid(dev))
    sampler.wait_first()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    if dist:
        dist.barrier()
    torch.cuda.synchronize(dev)
    tw0 = time.time()
    ms = time_steps(step, args.steps, stream, flush_buf)
    torch.cuda.synchronize(dev)
    tw1 = time.time()
    if dist:
        dist.barrier()
    clocks = sampler.summary(tw0, tw1)

    # ---- second timed region: the same K steps with CUDA events around each
    # kernel of the layer (on the launching stream), for the per-kernel times ----
    moe.moe_profile_enable(layer.ctx, 1)
    torch.cuda.synchronize(dev)
    ms_prof = time_steps(step, args.steps, stream, flush_buf)
    torch.cuda.synchronize(dev)
    stage_ms, ncalls = moe.moe_profile_read(layer.ctx)
    moe.moe_profile_enable(layer.ctx, 0)
    if layer.device_status() != moe.MOE_OK:
        raise RuntimeError("device status not OK after the timed region")
    ms, _, value = replica_throughput(dist, dev, ms, st["weight_bytes"], args.steps)
    ms_step = ms / args.steps

    # ---- end to end through the C ABI with host buffers ----
    # Every step uploads its inputs from pinned host memory and reads its
    # output back, all inside the timed region.  The copies run on their own
    # streams with two buffer sets, as a serving loop overlaps them: step
    # i+1's inputs upload and step i's output reads back while the layer
    # computes.
    e2e = None
    if not args.no_e2e:
        x_h = L.x.cpu().pin_memory()
        ids_h = L.ids.cpu().pin_memory()
        w_h = L.topk_w.cpu().pin_memory()
        out_h = [torch.empty(L.T, L.H, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        x_d = [torch.empty_like(L.x) for _ in range(2)]
        ids_d = [torch.empty_like(L.ids) for _ in range(2)]
        w_d = [torch.empty_like(L.topk_w) for _ in range(2)]
        out_d = [torch.empty_like(out) for _ in range(2)]
        up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_done = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]
        used = [False, False]

        def step_e2e(i):
            b = i % 2
            with torch.cuda.stream(up):
                if used[b]:
                    up.wait_event(ev_done[b])  # the layer of step i-2 has read buffer set b
                x_d[b].copy_(x_h, non_blocking=True)
                ids_d[b].copy_(ids_h, non_blocking=True)
                w_d[b].copy_(w_h, non_blocking=True)
                ev_in[b].record(up)
            stream.wait_event(ev_in[b])
            if used[b]:
                stream.wait_event(ev_out[b])  # step i-2's output has been read back
            layer.forward(x_d[b], ids_d[b], w_d[b], w13, s13, w2, s2, out=out_d[b], stream=stream, **gsc)
            ev_done[b].record(stream)
            with torch.cuda.stream(down):
                down.wait_event(ev_done[b])
                out_h[b].copy_(out_d[b], non_blocking=True)
                ev_out[b].record(down)
            used[b] = True

        def drain():  # the launching stream waits for every outstanding read-back
            for b in range(2):
                if used[b]:
                    stream.wait_event(ev_out[b])

        for i in range(3):
            step_e2e(i)
        drain()
        torch.cuda.synchronize(dev)
        if dist:
            dist.barrier()
        ev0.record(stream)
        up.wait_event(ev0)  # the first upload starts inside the timed region
        for i in range(args.steps):
            step_e2e(i)
        drain()
        ev1.record(stream)
        torch.cuda.synchronize(dev)
        ms_e, _, e2e_value = replica_throughput(dist, dev, ev0.elapsed_time(ev1), st["weight_bytes"], args.steps)
        h2d = x_h.numel() * 2 + ids_h.numel() * 4 + w_h.numel() * 4
        e2e = {"value": e2e_value, "unit": "GB/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": out_h[0].numel() * 2,
               "ms_per_step": ms_e / args.steps,
               "copies": "pinned host buffers, uploads and read-backs on their own streams, double-buffered"}

    # ---- roofline of the dominant kernel (GEMM1 + SwiGLU + requant) ----
    hbm_peak, bf16_peak, peak_src = peaks()
    g1_ms = stage_ms[2]
    g1_gbs = st["gemm1_bytes"] / (g1_ms * 1e-3) / 1e9 if g1_ms > 0 else None
    # the same launch against the dense tensor peak of its operand type (measured
    # bf16 x the nominal ratio: 2 for FP8, 4 for FP4 x FP4)
    g1_flops = 2.0 * st["positions"] * 2 * L.I * L.H
    g1_tflops = g1_flops / (g1_ms * 1e-3) / 1e12 if g1_ms > 0 else None
    ratio = 4.0 if L.wfmt in (synth.WFMT_NVFP4, synth.WFMT_MXFP4_A4) else 2.0
    fp8_peak = ratio * bf16_peak
    req = {synth.WFMT_NVFP4: "NVFP4", synth.WFMT_MXFP4_A4: "MXFP4", synth.WFMT_MXFP8: "MXFP8"}.get(L.wfmt, "FP8")
    roofline = {"kernel": f"GEMM1 (grouped GEMM1 + SwiGLU + {req} requant)", "bound": "hbm",
                "achieved": g1_gbs, "peak": hbm_peak, "unit": "GB/s",
                "frac": (g1_gbs / hbm_peak) if g1_gbs else None,
                "traffic": recorded_traffic(cfg["name"]),
                "algorithmic_bytes_per_launch": st["gemm1_bytes"], "avg_launch_ms": g1_ms,
                "peak_source": f"{peak_src} hbm_gbs (copy bandwidth)",
                "tensor_tflops": g1_tflops, "tensor_peak_tflops": fp8_peak,
                "tensor_frac": (g1_tflops / fp8_peak) if g1_tflops else None,
                "tensor_peak_source": f"{peak_src} bf16_tflops x {ratio:g} ({'FP4' if ratio == 4 else 'FP8'}/bf16 "
                                      f"nominal ratio)",
                "launches_timed": ncalls}

    if dist:
        dist.barrier()
    if rank != 0:
        sampler.stop()
        if dist:
            dist.destroy_process_group()
        return

    router = time_router(args, L, layer, dev, stream) if args.router else None

    # ---- the other workloads, each timed on its own (one GPU only) ----
    extra = []
    if world == 1:
        if args.workloads is None:
            default = args.shape is None and args.workload == 1
            extra = [i for i in range(len(synth.CONFIGS) + len(synth.EXTRA_CONFIGS)) if i != 1] if default else []
        elif args.workloads != "none":
            extra = [int(v) for v in args.workloads.split(",") if v.strip()]
    workloads = None
    if extra:
        # free the headline layer's device memory first (the prefill layer holds 11 GB of weights)
        layer.close()
        del w13, s13, w2, s2, gsc, out, flush_buf
        torch.cuda.empty_cache()
        workloads = {}
        for i in extra:
            rec = workload_record(i, args, dev, stream, sampler)
            workloads[rec["workload"]] = rec
            log(f"workload {rec['workload']}: {rec['us_per_layer']:.1f} us, {rec['weight_GBps']:.0f} GB/s, "
                f"{rec['tflops']:.1f} TFLOP/s, roofline frac {rec['roofline_frac']:.3f}")
    sampler.stop()

    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(L)

    frac_step = value / world / hbm_peak
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": DTYPES[L.wfmt],
        "data": "synthetic (seeded: x~N(0,1) bf16, uniform/zipf top-k, weights N(0,0.02) quantised)",
        "config": {"workload": cfg["name"], "T": L.T, "H": L.H, "E": L.E, "k": L.k, "I": L.I,
                   "wfmt": WFMT_NAMES[L.wfmt], "n_shared": L.n_shared,
                   "experts_touched": st["experts_touched"], "weight_bytes_per_step": st["weight_bytes"],
                   "l2": l2_label(st["weight_bytes"], flush),
                   "parallelism": "replicas" if world > 1 else "single GPU",
                   "green_ctx": {"dispatch_sms": green[0], "gemm_sms": green[1]} if green else None,
                   "dispatch_overlap_ctas": disp},
        "us_per_layer": ms_step * 1e3,
        "tflops": st["flops"] / (ms_step * 1e-3) / 1e12,
        "hbm_frac_of_step": frac_step,
        "stage_ms": dict(zip(moe.STAGE_NAMES, stage_ms)),
        "ms_per_step_profiled": ms_prof / args.steps,
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": launches_per_call(L, bool(disp)) * args.steps,  # per timed region
        "clocks": clocks,
    }
    if workloads:
        line["workloads"] = workloads
    if router:
        line["router"] = router
    print(json.dumps(line), flush=True)
    if dist:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
