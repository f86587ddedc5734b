// moe_route.cu -- routing, activation quantisation and output kernels.
//
// route_kernel   step 1: per-expert token counts, exclusive prefix sum,
//                stable scatter of slots into expert-contiguous positions
//                (perm) and its inverse (inv), plus the GEMM tile list.
//                GC-MoE abstract (token dispatch); FusedDeepMoE page
//                (per-expert counts, group list, expand index, prefix-summed
//                ranges in OpCombineSend).
// quant_kernel   step 2: per token, per 128 columns, s = amax/448 and
//                q = e4m3(x/s), written to every position the token is routed
//                to.  FusedDeepMoE QuantToken, with the E4M3 maximum in
//                place of the int8 127.
// finalize       fp32 combine accumulator -> bf16 output.
#include <cuda_bf16.h>

#include "moe_internal.h"
#include "moe_mxfp8.cuh"
#include "moe_ptx.cuh"

namespace moe {

// ---------------------------------------------------------------------------
// One CTA of 1024 threads.  Warp w owns the contiguous slot range
// [w*chunk, (w+1)*chunk); a ballot match groups equal expert ids within a
// 32-slot step, so a slot's position is
//   offsets[e] + (slots of e in earlier warps) + (earlier steps of this warp)
//   + (lower lanes with the same id in this step),
// which is exactly the stable counting-sort position.
constexpr int kRouteBatch = 8;  // 32-slot steps whose ids are loaded together

// Lanes of the warp holding the same key as this lane, from one ballot per
// key bit (the warp-ballot form of a match): key < 2^nbits.
__device__ __forceinline__ unsigned ballot_match(int key, int nbits) {
  unsigned peers = 0xFFFFFFFFu;
  for (int b = 0; b < nbits; ++b) {
    const bool bit = (key >> b) & 1;
    const unsigned m = __ballot_sync(0xFFFFFFFFu, bit);
    peers &= bit ? m : ~m;
  }
  return peers;
}

__global__ void __launch_bounds__(kRouteThreads, 1) route_kernel(RouteParams p) {
  // The next kernel (a quantisation kernel, or GEMM1 with dispatch overlap,
  // when launched as a programmatic dependent) may be scheduled now; it waits
  // for this grid's completion before it reads the routing.
  griddep_launch_dependents();
  extern __shared__ int sm[];
  const int E = p.E, NG = p.E + p.n_shared;
  const int S = p.T * p.k, P = S + p.n_shared * p.T;
  int* cnt = sm;                 // [NG]
  int* off = cnt + NG;           // [NG + 1]
  int* toff = off + NG + 1;      // [NG + 1]
  int* wc = toff + NG + 1;       // [32][NG]: per-warp counts, then per-warp bases
  int* cbase = wc + 32 * NG;     // [NG]: positions of each group in earlier CTAs' chunks
  __shared__ int s_bad;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // This CTA's slots (all of them with one CTA; with several, chunk
  // blockIdx.x of p.chunk slots, the later chunks after it in every group).
  const bool lead = blockIdx.x == 0;
  const int c0 = min(S, (int)blockIdx.x * p.chunk), c1 = min(S, c0 + p.chunk);

  for (int i = tid; i < 32 * NG; i += kRouteThreads) wc[i] = 0;
  if (p.ready && lead)  // dispatch-overlap counters of the GEMM1 launch that follows
    for (int g = tid; g < NG; g += kRouteThreads) p.ready[g] = 0;
  if (tid == 0) s_bad = 0;
  __syncthreads();

  const int chunk = ((((c1 - c0) + 31) / 32) + 31) & ~31;
  const int kbits = 32 - __clz(E);  // bits of the largest key, E (a dropped id)
  const int beg = min(c1, c0 + warp * chunk), end = min(c1, beg + chunk);

  // The expert ids of kRouteBatch consecutive 32-slot steps, loaded before
  // any of them is used, so a warp waits for one load latency per batch
  // rather than one per step (out-of-range ids read as -1).
  auto load_batch = [&](int b0, int (&ev)[kRouteBatch], bool& bad) {
#pragma unroll
    for (int r = 0; r < kRouteBatch; ++r) {
      const int s = b0 + r * 32 + lane;
      ev[r] = (s < end) ? p.ids[s] : -1;
    }
#pragma unroll
    for (int r = 0; r < kRouteBatch; ++r) {
      const int s = b0 + r * 32 + lane;
      if (s < end && (ev[r] < 0 || ev[r] >= E)) {
        ev[r] = -1;
        bad = true;
      }
    }
  };

  // pass A: per-warp, per-expert counts
  bool bad = false;
  for (int b0 = beg; b0 < end; b0 += 32 * kRouteBatch) {
    int ev[kRouteBatch];
    load_batch(b0, ev, bad);
#pragma unroll
    for (int r = 0; r < kRouteBatch; ++r) {
      if (b0 + r * 32 >= end) break;  // uniform across the warp
      const int e = ev[r];
      const unsigned peers = ballot_match(e >= 0 ? e : E, kbits);
      if (e >= 0 && lane == __ffs(peers) - 1) wc[warp * NG + e] += __popc(peers);
      __syncwarp();
    }
  }
  if (bad) s_bad = 1;
  __syncthreads();

  // per expert: total count, and counts of earlier warps (exclusive over
  // warps); with several CTAs the totals and this chunk's base come from the
  // per-chunk counts of route_count_kernel
  for (int e = tid; e < E; e += kRouteThreads) {
    int run = 0;
    for (int w = 0; w < 32; ++w) {
      const int c = wc[w * NG + e];
      wc[w * NG + e] = run;
      run += c;
    }
    int total = run, base = 0;
    if (p.nparts > 1) {
      total = 0;
      for (int b = 0; b < p.nparts; ++b) {
        const int c = p.part[b * E + e];
        if (b < (int)blockIdx.x) base += c;
        total += c;
      }
    }
    cnt[e] = total;
    cbase[e] = base;
  }
  if (p.n_shared && tid == 0) {
    cnt[E] = p.T;
    cbase[E] = 0;
  }
  __syncthreads();

  // exclusive scans: group offsets, and tile offsets (ceil(count / BN) tiles)
  if (warp == 0 || warp == 1) {
    const int per = (NG + 31) / 32;
    const int b = min(NG, lane * per), en = min(NG, b + per);
    int local = 0;
    for (int i = b; i < en; ++i) local += (warp == 0) ? cnt[i] : (cnt[i] + p.BN - 1) / p.BN;
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += v;
    }
    int run = incl - local;
    int* dst = (warp == 0) ? off : toff;
    for (int i = b; i < en; ++i) {
      dst[i] = run;
      run += (warp == 0) ? cnt[i] : (cnt[i] + p.BN - 1) / p.BN;
    }
    if (lane == 31) dst[NG] = incl;
  }
  __syncthreads();

  if (lead) {
    for (int g = tid; g < NG; g += kRouteThreads) p.counts[g] = cnt[g];
    for (int g = tid; g <= NG; g += kRouteThreads) p.offsets[g] = off[g];
    if (p.tile_off)
      for (int g = tid; g <= NG; g += kRouteThreads) p.tile_off[g] = toff[g];
  }

  // pass B: stable scatter
  for (int b0 = beg; b0 < end; b0 += 32 * kRouteBatch) {
    int ev[kRouteBatch];
    load_batch(b0, ev, bad);
#pragma unroll
    for (int r = 0; r < kRouteBatch; ++r) {
      if (b0 + r * 32 >= end) break;  // uniform across the warp
      const int s = b0 + r * 32 + lane;
      const int e = ev[r];
      const unsigned peers = ballot_match(e >= 0 ? e : E, kbits);
      const int rank = __popc(peers & ((1u << lane) - 1u));
      if (s < end) {
        if (e >= 0) {
          const int pos = off[e] + cbase[e] + wc[warp * NG + e] + rank;
          p.perm[pos] = s;
          p.inv[s] = pos;
        } else {
          p.inv[s] = -1;
        }
      }
      __syncwarp();
      if (e >= 0 && lane == __ffs(peers) - 1) wc[warp * NG + e] += __popc(peers);
      __syncwarp();
    }
  }

  if (!lead) {
    if (tid == 0 && s_bad) atomicOr(p.status, DEV_BAD_ROUTING);
    return;
  }
  // shared expert: every token, as virtual slot S + t, after the routed groups
  if (p.n_shared) {
    for (int t = tid; t < p.T; t += kRouteThreads) {
      const int pos = off[E] + t;
      p.perm[pos] = S + t;
      p.inv[S + t] = pos;
    }
  }
  for (int i = off[NG] + tid; i < P; i += kRouteThreads) p.perm[i] = -1;  // tail left by dropped slots

  // tile list: tiles[toff[g] + j] covers positions off[g] + j*BN ..
  for (int g = tid; g < NG; g += kRouteThreads) {
    const int n = cnt[g];
    for (int j = 0; j * p.BN < n; ++j)
      p.tiles[toff[g] + j] = make_int4(g, off[g] + j * p.BN, min(p.BN, n - j * p.BN), 0);
  }
  if (tid == 0) {
    *p.num_tiles = toff[NG];
    if (s_bad) atomicOr(p.status, DEV_BAD_ROUTING);
  }
}

size_t route_smem_bytes(int n_groups) { return sizeof(int) * (4 * (size_t)n_groups + 2 + 32 * (size_t)n_groups); }

// Per-chunk expert counts for the multi-CTA route: CTA b counts the valid
// expert ids of slots [b * chunk, (b + 1) * chunk) into part[b][e].
__global__ void __launch_bounds__(kRouteThreads) route_count_kernel(RouteParams p) {
  extern __shared__ int hist[];  // [E]
  const int S = p.T * p.k, E = p.E;
  for (int e = threadIdx.x; e < E; e += kRouteThreads) hist[e] = 0;
  __syncthreads();
  const int c0 = min(S, (int)blockIdx.x * p.chunk), c1 = min(S, c0 + p.chunk);
  for (int s = c0 + threadIdx.x; s < c1; s += kRouteThreads) {
    const int e = p.ids[s];
    if (e >= 0 && e < E) atomicAdd(&hist[e], 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += kRouteThreads) p.part[blockIdx.x * E + e] = hist[e];
}

// Slots per CTA of the multi-CTA route, and the slot count from which it is used
constexpr int kRouteChunk = 2048;
constexpr int kRouteMultiSlots = 4096;

// ---------------------------------------------------------------------------
// Routing for a few slots (S <= kRouteSmallUpTo): one CTA of 256 threads.
// The same counting sort and the same outputs as route_kernel, in fewer
// steps: the ids go to shared memory once, a shared-memory histogram gives
// the counts, one block scan the group and tile offsets, and warp 0 walks
// the slots in 32-slot steps in order, a slot's position being its group's
// offset plus the slots of the group already placed plus its rank among the
// lanes with the same id (a warp-ballot match), which is the stable
// counting-sort position.  Decode layers route 8 to a few hundred slots,
// where the 32-warp kernel spends its time in block barriers and in
// fetching its larger code.  Its scatter is one warp walking all S slots
// in order: at 1024 slots the kernel measured slower than the 32-warp one,
// whose warps scatter their slot ranges side by side (19.5-21.4 us against
// 12.6-14.4 us), at 256 and fewer faster, so it is used up to 256 slots.
constexpr int kRouteSmallSlots = 1024;  // capacity of its shared id array
constexpr int kRouteSmallUpTo = 256;    // slot count up to which launch_route picks it
constexpr int kRouteSmallThreads = 256;

__global__ void __launch_bounds__(kRouteSmallThreads, 1) route_small_kernel(RouteParams p) {
  griddep_launch_dependents();  // see route_kernel
  __shared__ int ids_s[kRouteSmallSlots];
  __shared__ int cnt[kMaxGroups], run[kMaxGroups];
  __shared__ int off[kMaxGroups + 1], toff[kMaxGroups + 1];
  __shared__ int wtot[2][kRouteSmallThreads / 32];
  __shared__ int s_bad;
  const int E = p.E, NG = p.E + p.n_shared;
  const int S = p.T * p.k, P = S + p.n_shared * p.T;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  for (int g = tid; g < NG; g += kRouteSmallThreads) {
    cnt[g] = (g == E) ? p.T : 0;  // the shared expert takes every token
    if (p.ready) p.ready[g] = 0;  // dispatch-overlap counters of the GEMM1 launch that follows
  }
  if (tid == 0) s_bad = 0;
  __syncthreads();
  for (int s = tid; s < S; s += kRouteSmallThreads) {
    int e = p.ids[s];
    if (e < 0 || e >= E) {
      e = -1;
      s_bad = 1;
    } else {
      atomicAdd(&cnt[e], 1);
    }
    ids_s[s] = e;
  }
  __syncthreads();

  // exclusive scans of the counts and of the tiles per group (ceil(count / BN));
  // thread tid owns groups [tid * per, tid * per + per)
  {
    const int per = (NG + kRouteSmallThreads - 1) / kRouteSmallThreads;
    const int b = min(NG, tid * per), en = min(NG, b + per);
    int lc = 0, lt = 0;
    for (int g = b; g < en; ++g) {
      lc += cnt[g];
      lt += (cnt[g] + p.BN - 1) / p.BN;
    }
    int ic = lc, it = lt;  // inclusive within the warp
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int vc = __shfl_up_sync(0xFFFFFFFFu, ic, o), vt = __shfl_up_sync(0xFFFFFFFFu, it, o);
      if (lane >= o) {
        ic += vc;
        it += vt;
      }
    }
    if (lane == 31) {
      wtot[0][warp] = ic;
      wtot[1][warp] = it;
    }
    __syncthreads();
    int bc = 0, bt = 0;  // totals of the earlier warps
    for (int w = 0; w < warp; ++w) {
      bc += wtot[0][w];
      bt += wtot[1][w];
    }
    int rc = bc + ic - lc, rt = bt + it - lt;
    for (int g = b; g < en; ++g) {
      off[g] = rc;
      toff[g] = rt;
      run[g] = rc;
      rc += cnt[g];
      rt += (cnt[g] + p.BN - 1) / p.BN;
    }
    if (tid == kRouteSmallThreads - 1) {
      off[NG] = rc;
      toff[NG] = rt;
    }
  }
  __syncthreads();

  for (int g = tid; g < NG; g += kRouteSmallThreads) p.counts[g] = cnt[g];
  for (int g = tid; g <= NG; g += kRouteSmallThreads) {
    p.offsets[g] = off[g];
    if (p.tile_off) p.tile_off[g] = toff[g];
  }
  if (warp == 0) {
    // stable scatter of the routed slots, in order
    const int kbits = 32 - __clz(E);  // bits of the largest key, E (a dropped id)
    for (int b0 = 0; b0 < S; b0 += 32) {
      const int s = b0 + lane;
      const int e = (s < S) ? ids_s[s] : -1;
      const unsigned peers = ballot_match(e >= 0 ? e : E, kbits);
      if (s < S) {
        if (e >= 0) {
          const int pos = run[e] + __popc(peers & ((1u << lane) - 1u));
          p.perm[pos] = s;
          p.inv[s] = pos;
        } else {
          p.inv[s] = -1;
        }
      }
      __syncwarp();
      if (e >= 0 && lane == __ffs(peers) - 1) run[e] += __popc(peers);
      __syncwarp();
    }
  } else {
    // shared expert: every token, as virtual slot S + t, after the routed groups
    const int t0 = tid - 32, nt = kRouteSmallThreads - 32;
    if (p.n_shared)
      for (int t = t0; t < p.T; t += nt) {
        const int pos = off[E] + t;
        p.perm[pos] = S + t;
        p.inv[S + t] = pos;
      }
    for (int i = off[NG] + t0; i < P; i += nt) p.perm[i] = -1;  // tail left by dropped slots
    // tile list: tiles[toff[g] + j] covers positions off[g] + j*BN ..
    for (int g = t0; g < NG; g += nt) {
      const int n = cnt[g];
      for (int j = 0; j * p.BN < n; ++j)
        p.tiles[toff[g] + j] = make_int4(g, off[g] + j * p.BN, min(p.BN, n - j * p.BN), 0);
    }
    if (t0 == 0) {
      *p.num_tiles = toff[NG];
      if (s_bad) atomicOr(p.status, DEV_BAD_ROUTING);
    }
  }
}

cudaError_t launch_route(const RouteParams& p0, cudaStream_t s) {
  RouteParams p = p0;
  const int S = p.T * p.k;
  p.nparts = 1;
  p.chunk = S;
  if (p.part && S >= kRouteMultiSlots) {
    p.nparts = min(kMaxRouteParts, (S + kRouteChunk - 1) / kRouteChunk);
    p.chunk = (S + p.nparts - 1) / p.nparts;
  }
  const size_t smem = route_smem_bytes(p.E + p.n_shared);
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(route_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)route_smem_bytes(kMaxGroups));
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  static_assert(kRouteSmallUpTo <= kRouteSmallSlots, "the small route kernel holds every id in shared memory");
  if (S <= kRouteSmallUpTo) {
    route_small_kernel<<<1, kRouteSmallThreads, 0, s>>>(p);
    return cudaGetLastError();
  }
  if (p.nparts > 1) {
    route_count_kernel<<<p.nparts, kRouteThreads, sizeof(int) * p.E, s>>>(p);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  route_kernel<<<p.nparts, kRouteThreads, smem, s>>>(p);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// One CTA per token, 8 warps; warp w quantises column groups w, w+8, ...
// Each lane holds 4 consecutive bf16 values of the 128-column group.
constexpr int kQuantThreads = 256;
constexpr int kQuantGroups = 64 / (kQuantThreads / 32);  // H <= 8192: at most 8 groups per warp

// The token's 128-column groups of this warp (g = warp, warp + 8, ...), all
// loads issued at once and before the routing rows are known: x does not
// depend on the route kernel, and a warp then waits for one load latency
// instead of one per group.
__device__ __forceinline__ void load_token_groups(const QuantParams& p, int t, uint2 (&raw)[kQuantGroups]) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint16_t* xr = p.x + (size_t)t * p.H;
#pragma unroll
  for (int i = 0; i < kQuantGroups; ++i) {
    const int g = warp + i * (kQuantThreads / 32);
    raw[i] = (g < p.H / 128) ? *reinterpret_cast<const uint2*>(xr + g * 128 + lane * 4) : make_uint2(0u, 0u);
  }
}

// Launched as a programmatic dependent of the route kernel (QuantParams::pdl),
// a quantisation kernel loads its token while the routing is computed and
// then waits for it; otherwise the wait returns at once.  GEMM1 may be
// scheduled only after that point: it reads the tile list before its own
// wait, and its weight prefetch then starts as the quantisation begins.
__device__ __forceinline__ void after_route() {
  griddep_wait();
  griddep_launch_dependents();
}

// One CTA per token; a programmatic dependent of the route kernel when p.pdl.
template <typename K>
static cudaError_t launch_quant_kernel(K kernel, const QuantParams& p, cudaStream_t s) {
  if (!p.pdl) {
    kernel<<<p.T, kQuantThreads, 0, s>>>(p);
    return cudaGetLastError();
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.T);
  cfg.blockDim = dim3(kQuantThreads);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, p);
}

// Drops raw[0] and moves the rest down (static indices: registers).
__device__ __forceinline__ void next_group(uint2 (&raw)[kQuantGroups]) {
#pragma unroll
  for (int i = 0; i + 1 < kQuantGroups; ++i) raw[i] = raw[i + 1];
}

// The token's routed positions in routing order (slot j of the token in
// lane j, the shared expert's position last), gathered by warp 0 in one
// round of loads: rows[0 .. *nrows).
__device__ __forceinline__ void gather_rows(const QuantParams& p, int t, int* rows, int* nrows) {
  const int lane = threadIdx.x & 31;
  const int S = p.T * p.k;
  const int r = (lane < p.k) ? p.inv[t * p.k + lane] : -1;
  const int rs = (lane == 0 && p.n_shared) ? p.inv[S + t] : -1;
  const unsigned valid = __ballot_sync(0xFFFFFFFFu, r >= 0);
  if (r >= 0) rows[__popc(valid & ((1u << lane) - 1u))] = r;
  if (lane == 0) {
    int n = __popc(valid);
    if (p.n_shared) rows[n++] = rs;
    *nrows = n;
  }
}

__global__ void __launch_bounds__(kQuantThreads) quant_kernel(QuantParams p) {
  const int t = blockIdx.x;
  const int H = p.H, HB = p.H / 128;
  __shared__ int rows[kMaxK + 1];
  __shared__ int nrows;
  uint2 raws[kQuantGroups];
  load_token_groups(p, t, raws);
  after_route();
  if (threadIdx.x < 32) gather_rows(p, t, rows, &nrows);
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll 1
  for (int g = warp; g < HB; g += kQuantThreads / 32, next_group(raws)) {
    const uint2 raw = raws[0];
    float sc;
    const uint32_t packed = quant_group_e4m3(raw, &sc);
    for (int r = 0; r < nrows; ++r) {
      *reinterpret_cast<uint32_t*>(p.xq + (size_t)rows[r] * H + g * 128 + lane * 4) = packed;
      if (lane == 0) p.xs[(size_t)g * p.xs_ld + rows[r]] = sc;
    }
  }
  if (p.out_acc) {
    float4* acc = reinterpret_cast<float4*>(p.out_acc + (size_t)t * H);
    for (int i = threadIdx.x; i < H / 4; i += kQuantThreads) acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

cudaError_t launch_quant(const QuantParams& p, cudaStream_t s) {
  return launch_quant_kernel(quant_kernel, p, s);
}

// ---------------------------------------------------------------------------
// NVFP4 form of step 2 (NVIDIA NVFP4: E2M1 elements, E4M3 scale per 16, fp32
// second-level scale; the second level per token per 128 columns, the FP8
// activation group of the FusedDeepMoE QuantToken step):
//   S = amax128 / 2688 (1 for an all-zero group), block code
//   c = e4m3((amax16 / 6) / S), element code q = e2m1(v / (e4m3_value(c) * S))
//   (q = 0 when c = 0), every operation one IEEE fp32 operation.
// Same grid as quant_kernel; a lane holds 4 consecutive columns, so a 16-
// column block is 4 neighbouring lanes and a 64-column MMA step 16 lanes.
// Outputs per routed position: packed codes (element 2c in the low nibble of
// byte c), the four block codes of each step as one 32-bit word (layout of
// QuantParams::xsc), S.
__global__ void __launch_bounds__(kQuantThreads) quant_nvfp4_kernel(QuantParams p) {
  const int t = blockIdx.x;
  const int H = p.H, HB = p.H / 128;
  __shared__ int rows[kMaxK + 1];
  __shared__ int nrows;
  uint2 raws[kQuantGroups];
  load_token_groups(p, t, raws);
  after_route();
  if (threadIdx.x < 32) gather_rows(p, t, rows, &nrows);
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll 1
  for (int g = warp; g < HB; g += kQuantThreads / 32, next_group(raws)) {
    const uint2 raw = raws[0];
    float f[4];
    f[0] = __uint_as_float((raw.x & 0xFFFFu) << 16);
    f[1] = __uint_as_float(raw.x & 0xFFFF0000u);
    f[2] = __uint_as_float((raw.y & 0xFFFFu) << 16);
    f[3] = __uint_as_float(raw.y & 0xFFFF0000u);
    float a16 = fmaxf(fmaxf(fabsf(f[0]), fabsf(f[1])), fmaxf(fabsf(f[2]), fabsf(f[3])));
    a16 = fmaxf(a16, __shfl_xor_sync(0xFFFFFFFFu, a16, 1));
    a16 = fmaxf(a16, __shfl_xor_sync(0xFFFFFFFFu, a16, 2));
    float amax = a16;
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
    const float sg = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 2688.0f);
    const uint32_t code = f32_to_e4m3(__fdiv_rn(__fdiv_rn(a16, 6.0f), sg));
    const float d = __fmul_rn(e4m3_code_value(code), sg);
    uint32_t packed = 0;
    if (code != 0)
      packed = f32x4_to_e2m1x4(__fdiv_rn(f[0], d), __fdiv_rn(f[1], d), __fdiv_rn(f[2], d), __fdiv_rn(f[3], d));
    // the step's four codes into one word (lanes 0 and 16 hold steps 2g, 2g+1)
    uint32_t word = ((lane & 3) == 0) ? code << (8 * ((lane >> 2) & 3)) : 0u;
    word |= __shfl_xor_sync(0xFFFFFFFFu, word, 4);
    word |= __shfl_xor_sync(0xFFFFFFFFu, word, 8);
    const size_t step = (size_t)(2 * g + (lane >> 4));
    for (int r = 0; r < nrows; ++r) {
      *reinterpret_cast<uint16_t*>(p.xq + (size_t)rows[r] * (H / 2) + g * 64 + lane * 2) = (uint16_t)packed;
      if ((lane & 15) == 0) *reinterpret_cast<uint32_t*>(p.xsc + (step * p.xs_ld + rows[r]) * 16) = word;
      if (lane == 0) p.xs[(size_t)g * p.xs_ld + rows[r]] = sg;
    }
  }
  if (p.out_acc) {
    float4* acc = reinterpret_cast<float4*>(p.out_acc + (size_t)t * H);
    for (int i = threadIdx.x; i < H / 4; i += kQuantThreads) acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

cudaError_t launch_quant_nvfp4(const QuantParams& p, cudaStream_t s) {
  return launch_quant_kernel(quant_nvfp4_kernel, p, s);
}

// ---------------------------------------------------------------------------
// MXFP4 form of step 2, for MXFP4 weights with MXFP4 activations (OCP MX
// v1.0 conversion with E2M1 elements): per 32 columns X = floor(log2 amax) - 2
// clamped to [-127, 127] (-127 for an all-zero block), code X + 127 (E8M0),
// elements e2m1(v / 2^X).  Same grid as quant_kernel; a lane holds 4
// consecutive columns, so a 32-column block is 8 lanes and the 128-column
// K block is the warp.  Outputs per routed position: packed codes and the
// K block's four E8M0 codes as one 32-bit word (layout of QuantParams::xsc).
__global__ void __launch_bounds__(kQuantThreads) quant_mxfp4_kernel(QuantParams p) {
  const int t = blockIdx.x;
  const int H = p.H, HB = p.H / 128;
  __shared__ int rows[kMaxK + 1];
  __shared__ int nrows;
  uint2 raws[kQuantGroups];
  load_token_groups(p, t, raws);
  after_route();
  if (threadIdx.x < 32) gather_rows(p, t, rows, &nrows);
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll 1
  for (int g = warp; g < HB; g += kQuantThreads / 32, next_group(raws)) {
    const uint2 raw = raws[0];
    float f[4];
    f[0] = __uint_as_float((raw.x & 0xFFFFu) << 16);
    f[1] = __uint_as_float(raw.x & 0xFFFF0000u);
    f[2] = __uint_as_float((raw.y & 0xFFFFu) << 16);
    f[3] = __uint_as_float(raw.y & 0xFFFF0000u);
    float a32 = fmaxf(fmaxf(fabsf(f[0]), fabsf(f[1])), fmaxf(fabsf(f[2]), fabsf(f[3])));
    a32 = fmaxf(a32, __shfl_xor_sync(0xFFFFFFFFu, a32, 1));
    a32 = fmaxf(a32, __shfl_xor_sync(0xFFFFFFFFu, a32, 2));
    a32 = fmaxf(a32, __shfl_xor_sync(0xFFFFFFFFu, a32, 4));
    float sc;
    const int X = mx_e2m1_exponent(a32, &sc);
    const uint32_t packed =
        f32x4_to_e2m1x4(__fdiv_rn(f[0], sc), __fdiv_rn(f[1], sc), __fdiv_rn(f[2], sc), __fdiv_rn(f[3], sc));
    // the K block's four codes into one word (lane 0)
    uint32_t word = ((lane & 7) == 0) ? static_cast<uint32_t>(X + 127) << (8 * (lane >> 3)) : 0u;
    word |= __shfl_xor_sync(0xFFFFFFFFu, word, 8);
    word |= __shfl_xor_sync(0xFFFFFFFFu, word, 16);
    for (int r = 0; r < nrows; ++r) {
      *reinterpret_cast<uint16_t*>(p.xq + (size_t)rows[r] * (H / 2) + g * 64 + lane * 2) = (uint16_t)packed;
      if (lane == 0) *reinterpret_cast<uint32_t*>(p.xsc + ((size_t)g * p.xs_ld + rows[r]) * 16) = word;
    }
  }
  if (p.out_acc) {
    float4* acc = reinterpret_cast<float4*>(p.out_acc + (size_t)t * H);
    for (int i = threadIdx.x; i < H / 4; i += kQuantThreads) acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

cudaError_t launch_quant_mxfp4(const QuantParams& p, cudaStream_t s) {
  return launch_quant_kernel(quant_mxfp4_kernel, p, s);
}

// ---------------------------------------------------------------------------
// MXFP8 form of step 2 (OCP MX v1.0 with E4M3 elements): per 32 columns
// X = floor(log2 amax) - 8 (clamped to [-127, 127], -127 for an all-zero
// block), E8M0 code X + 127, elements e4m3(v / 2^X) with round-to-nearest-
// even and saturation.  Same grid as quant_kernel; a lane holds 4
// consecutive columns, so a 32-column block is 8 neighbouring lanes.  Codes
// go to every routed position of the token (rows in routing order); the
// E8M0 codes go straight into the token-major kernel's A-operand scale
// atoms: the position's tile ti = tile_off[g] + (pos - offsets[g]) / 128 and
// row r = (pos - offsets[g]) % 128 within it.
__global__ void __launch_bounds__(kQuantThreads) quant_mxfp8_kernel(QuantParams p) {
  const int t = blockIdx.x;
  const int H = p.H, HB = p.H / 128, S = p.T * p.k;
  __shared__ int rows[kMaxK + 1];
  __shared__ int atom[kMaxK + 1];  // byte offset of the position's row in its tile's atoms
  __shared__ int nrows;
  uint2 raws[kQuantGroups];
  load_token_groups(p, t, raws);
  after_route();
  if (threadIdx.x < 32) {
    // slot j of the token in lane j, the shared expert's position in lane 0
    const int lane = threadIdx.x;
    auto atom_of = [&](int r, int g) {
      const int within = r - p.offsets[g];
      const int ti = p.tile_off[g] + within / 128, rr = within % 128;
      return ti * HB * 512 + (rr % 32) * 16 + (rr / 32) * 4;
    };
    const int r = (lane < p.k) ? p.inv[t * p.k + lane] : -1;
    const int rs = (lane == 0 && p.n_shared) ? p.inv[S + t] : -1;
    const unsigned valid = __ballot_sync(0xFFFFFFFFu, r >= 0);
    if (r >= 0) {
      const int i = __popc(valid & ((1u << lane) - 1u));
      rows[i] = r;
      atom[i] = atom_of(r, p.ids[t * p.k + lane]);
    }
    if (lane == 0) {
      int n = __popc(valid);
      if (p.n_shared) {
        rows[n] = rs;
        atom[n] = atom_of(rs, p.E);
        ++n;
      }
      nrows = n;
    }
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll 1
  for (int g = warp; g < HB; g += kQuantThreads / 32, next_group(raws)) {
    const uint2 raw = raws[0];
    float f[4];
    f[0] = __uint_as_float((raw.x & 0xFFFFu) << 16);
    f[1] = __uint_as_float(raw.x & 0xFFFF0000u);
    f[2] = __uint_as_float((raw.y & 0xFFFFu) << 16);
    f[3] = __uint_as_float(raw.y & 0xFFFF0000u);
    float amax = fmaxf(fmaxf(fabsf(f[0]), fabsf(f[1])), fmaxf(fabsf(f[2]), fabsf(f[3])));
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
    float sc;
    const int X = mx_e4m3_exponent(amax, &sc);
    const uint32_t packed = f32x2_to_e4m3x2(__fdiv_rn(f[0], sc), __fdiv_rn(f[1], sc)) |
                            (f32x2_to_e4m3x2(__fdiv_rn(f[2], sc), __fdiv_rn(f[3], sc)) << 16);
    for (int r = 0; r < nrows; ++r) {
      *reinterpret_cast<uint32_t*>(p.xq + (size_t)rows[r] * H + g * 128 + lane * 4) = packed;
      if ((lane & 7) == 0) p.sf_atoms[(size_t)atom[r] + (size_t)g * 512 + (lane >> 3)] = static_cast<uint8_t>(X + 127);
    }
  }
  if (p.out_acc) {
    float4* acc = reinterpret_cast<float4*>(p.out_acc + (size_t)t * H);
    for (int i = threadIdx.x; i < H / 4; i += kQuantThreads) acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

cudaError_t launch_quant_mxfp8(const QuantParams& p, cudaStream_t s) {
  return launch_quant_kernel(quant_mxfp8_kernel, p, s);
}

// ---------------------------------------------------------------------------
__global__ void finalize_kernel(const float4* __restrict__ acc, uint2* __restrict__ out, long long n4) {
  griddep_wait();  // the combine buffer is complete once GEMM2 has finished
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n4; i += (long long)gridDim.x * blockDim.x) {
    const float4 v = acc[i];
    const __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y);
    const __nv_bfloat162 b = __floats2bfloat162_rn(v.z, v.w);
    out[i] = make_uint2(*reinterpret_cast<const uint32_t*>(&a), *reinterpret_cast<const uint32_t*>(&b));
  }
}

cudaError_t launch_finalize(const float* acc, uint16_t* out, long long n, cudaStream_t s) {
  const long long n4 = n / 4;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  long long blocks = (n4 + 255) / 256;
  if (blocks > 4LL * sms) blocks = 4LL * sms;
  if (blocks < 1) blocks = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)blocks);
  cfg.blockDim = dim3(256);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, finalize_kernel, reinterpret_cast<const float4*>(acc), reinterpret_cast<uint2*>(out),
                            n4);
}

// ---------------------------------------------------------------------------
// Unfused combine (step 7) for large token counts: one CTA per token,
// out[t] = sum_j w[t,j] * y[inv[t*k+j]] (ascending j) + y[inv[S+t]] (shared
// expert, weight 1), in fp32, then bf16.  FusedDeepMoE ReducePermute
// (accumulate the expert outputs of each token), in the same order as the
// CPU reference and without atomics.
__global__ void __launch_bounds__(256) combine_kernel(CombineParams p) {
  griddep_wait();  // the expert output rows are complete once GEMM2 has finished
  const int t = blockIdx.x, S = p.T * p.k;
  __shared__ int rows[kMaxK + 1];
  __shared__ float wts[kMaxK + 1];
  __shared__ int nrows;
  if (threadIdx.x == 0) {
    int n = 0;
    for (int j = 0; j < p.k; ++j) {
      const int r = p.inv[t * p.k + j];
      if (r >= 0) {
        rows[n] = r;
        wts[n] = p.topk_w[t * p.k + j];
        ++n;
      }
    }
    if (p.n_shared) {
      rows[n] = p.inv[S + t];
      wts[n] = 1.0f;
      ++n;
    }
    nrows = n;
  }
  __syncthreads();
  for (int h = threadIdx.x * 4; h < p.H; h += 256 * 4) {
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int r = 0; r < nrows; ++r) {
      const float4 y = *reinterpret_cast<const float4*>(p.y_rows + (size_t)rows[r] * p.H + h);
      const float w = wts[r];
      o.x += w * y.x;
      o.y += w * y.y;
      o.z += w * y.z;
      o.w += w * y.w;
    }
    const __nv_bfloat162 a = __floats2bfloat162_rn(o.x, o.y);
    const __nv_bfloat162 b = __floats2bfloat162_rn(o.z, o.w);
    *reinterpret_cast<uint2*>(p.out + (size_t)t * p.H + h) =
        make_uint2(*reinterpret_cast<const uint32_t*>(&a), *reinterpret_cast<const uint32_t*>(&b));
  }
}

cudaError_t launch_combine(const CombineParams& p, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)p.T);
  cfg.blockDim = dim3(256);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, combine_kernel, p);
}

// ---------------------------------------------------------------------------
// Block scales, plain layout [rows, kgroups] (one byte per scale group along
// K: E8M0 per 32 elements for MXFP4, E4M3 per 16 for NVFP4) -> the
// block-scaled MMA layout: for each 128-row block and each run of four
// groups (one 128-wide K block of MXFP4, one K = 64 MMA step of NVFP4), one
// 512-byte atom with row m's 4 scales at byte
// (m % 32) * 16 + (m / 32) * 4 + (group within the run).
__global__ void pack_e8m0_kernel(const uint8_t* __restrict__ src, uint8_t* __restrict__ dst, int rows, int kgroups) {
  const long long total = (long long)rows * kgroups;
  const int kblocks = kgroups / 4;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total; i += (long long)gridDim.x * blockDim.x) {
    const int r = (int)(i / kgroups), kg = (int)(i % kgroups);
    const int rb = r / 128, m = r % 128, kb = kg / 4, kk = kg % 4;
    const long long o = ((long long)rb * kblocks + kb) * 512 + (m % 32) * 16 + (m / 32) * 4 + kk;
    dst[o] = src[i];
  }
}

cudaError_t launch_pack_e8m0(const uint8_t* src, uint8_t* dst, int rows, int kgroups, cudaStream_t s) {
  const long long total = (long long)rows * kgroups;
  long long blocks = (total + 255) / 256;
  if (blocks > 65535) blocks = 65535;
  if (blocks < 1) blocks = 1;
  pack_e8m0_kernel<<<(int)blocks, 256, 0, s>>>(src, dst, rows, kgroups);
  return cudaGetLastError();
}

}  // namespace moe
