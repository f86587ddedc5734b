// moe_router.cu -- fused router ("Mega Gate"): the routing GEMM and the MoE
// routing step in one kernel (DeepGEMM 26/09 news page: the router GEMM and
// the MoE routing operations fused into a single kernel).
//
//   logits[t, e] = sum_h x[t, h] * Wr[e, h]      x bf16 [T, H], Wr bf16 [E, H]
//   ids[t, :]    = the k largest logits of token t, descending, ties to the
//                  lower expert index
//   w[t, j]      = softmax over the k chosen logits
//
// One launch.  CTA (token tile of 128, K split): TMA streams 64-element K
// blocks of x and Wr into shared memory, tcgen05.mma kind::f16 (bf16 x bf16,
// fp32 accumulate; M = 128 tokens, N = E experts) accumulates the CTA's K
// range in TMEM, and the epilogue adds its partial logits into an fp32 buffer
// with vector reductions.  The CTA that finishes a tile last (atomic counter;
// nobody waits for anybody) reads the tile's logits into shared memory, selects
// and normalises the top k per token (one thread per token), and returns the
// buffer rows and the counter to zero for the next call.
#include <cuda_bf16.h>

#include "moe_internal.h"
#include "moe_ptx.cuh"

namespace moe {

namespace {

constexpr int kRtStages = 4;
constexpr int kRtThreads = 192;  // warp 0 TMA, warp 1 MMA + TMEM, warps 2-5 epilogue
constexpr int kRtA = 128 * 128;  // token tile: 128 rows x 64 bf16
constexpr int kRtBMax = 256 * 128;

// Instruction descriptor, kind::f16 with bf16 A and B, fp32 accumulate, K-major.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Bounded wait that ignores the abort word (drain of in-flight copies / MMAs).
__device__ __forceinline__ void rt_drain_wait(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kWaitCycles) break;
  }
}

// Top k (k <= 8) of one logit row in a single scan.  Each (value, index)
// pair becomes one 64-bit key that orders like "larger logit first, then
// lower index": the float's order-preserving bit pattern in the high word and
// the complemented index in the low word.  A sorted list of eight keys lives
// in named registers; an element enters when its key exceeds the k-th entry
// and moves down the list by plain 64-bit comparisons.  Then the softmax over
// the chosen logits.
__device__ __forceinline__ uint64_t rank_key(float v, int e) {
  const uint32_t b = __float_as_uint(v == 0.0f ? 0.0f : v);  // -0 and +0 tie, as values do
  const uint32_t ord = (b & 0x80000000u) ? ~b : (b | 0x80000000u);  // monotone in v
  return (static_cast<uint64_t>(ord) << 32) | (0xFFFFFFFFu - static_cast<uint32_t>(e));
}
__device__ __forceinline__ float key_value(uint64_t key) {
  const uint32_t ord = static_cast<uint32_t>(key >> 32);
  return __uint_as_float((ord & 0x80000000u) ? (ord & 0x7FFFFFFFu) : ~ord);
}
__device__ __forceinline__ int key_index(uint64_t key) {
  return static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(key));
}

__device__ __forceinline__ void topk8_row(const float* __restrict__ r, int E, int k, int32_t* ids, float* w) {
  uint64_t l0 = 0, l1 = 0, l2 = 0, l3 = 0, l4 = 0, l5 = 0, l6 = 0, l7 = 0;  // 0 ranks after every key
  uint64_t thr = 0;                                                         // key of the k-th entry
  for (int e = 0; e < E; ++e) {
    const uint64_t cv = rank_key(r[e], e);
    if (cv > thr) {
      // insertion slot = number of entries ranking before cv (the list is
      // sorted, so these are independent comparisons); entries from the slot
      // on move down by one
      const bool g0 = l0 > cv, g1 = l1 > cv, g2 = l2 > cv, g3 = l3 > cv, g4 = l4 > cv, g5 = l5 > cv,
                 g6 = l6 > cv, g7 = l7 > cv;
      l7 = g7 ? l7 : (g6 ? cv : l6);
      l6 = g6 ? l6 : (g5 ? cv : l5);
      l5 = g5 ? l5 : (g4 ? cv : l4);
      l4 = g4 ? l4 : (g3 ? cv : l3);
      l3 = g3 ? l3 : (g2 ? cv : l2);
      l2 = g2 ? l2 : (g1 ? cv : l1);
      l1 = g1 ? l1 : (g0 ? cv : l0);
      l0 = g0 ? l0 : cv;
      thr = (k == 1) ? l0 : (k == 2) ? l1 : (k == 3) ? l2 : (k == 4) ? l3 : (k == 5) ? l4 : (k == 6) ? l5
          : (k == 7) ? l6 : l7;
    }
  }
  const uint64_t ls[8] = {l0, l1, l2, l3, l4, l5, l6, l7};
  const float m = key_value(l0);
  float z = 0.0f;
#pragma unroll
  for (int s = 0; s < 8; ++s)
    if (s < k) z += expf(key_value(ls[s]) - m);
#pragma unroll
  for (int s = 0; s < 8; ++s)
    if (s < k) {
      ids[s] = key_index(ls[s]);
      w[s] = __fdiv_rn(expf(key_value(ls[s]) - m), z);
    }
}

// k > 8: k scans, each taking the largest logit ordered after the previous pick.
__device__ void topk_row_scan(const float* __restrict__ r, int E, int k, int32_t* ids, float* w) {
  float pv = 0.0f, m = 0.0f, z = 0.0f;
  int pe = -1;
  for (int j = 0; j < k; ++j) {
    float bv = 0.0f;
    int be = -1;
    for (int e = 0; e < E; ++e) {
      const float v = r[e];
      const bool after = (pe < 0) || (v < pv) || (v == pv && e > pe);
      if (after && (be < 0 || v > bv)) {
        bv = v;
        be = e;
      }
    }
    ids[j] = be;
    w[j] = bv;
    if (j == 0) m = bv;
    z += expf(bv - m);
    pv = bv;
    pe = be;
  }
  for (int j = 0; j < k; ++j) w[j] = __fdiv_rn(expf(w[j] - m), z);
}

}  // namespace

__global__ void __launch_bounds__(kRtThreads, 1)
    router_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                  const RouterParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int NP = p.N;                                   // MMA N: E rounded up to 16
  const int b_bytes = NP * 128;
  const int stage_bytes = kRtA + ((b_bytes + 1023) / 1024) * 1024;
  __shared__ uint64_t full[kRtStages], empty[kRtStages], mma_done;
  __shared__ uint32_t tmem_holder;
  __shared__ int s_last;
  __shared__ int abort_w;
  volatile int* abort = &abort_w;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x / p.splits, sp = blockIdx.x % p.splits;
  const int kb0 = (int)((long long)sp * p.kblocks / p.splits), kb1 = (int)((long long)(sp + 1) * p.kblocks / p.splits);
  const int nkb = kb1 - kb0;
  const int t0 = tile * 128;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kRtStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(&mma_done, 1);
    abort_w = 0;
    mbar_fence_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_holder, p.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_holder;

  if (warp == 0) {
    // TMA: lane 0 the token tile, lane 1 the router weight rows.
    const uint64_t pol = policy_evict_last();
    bool ok = true;
    int issued = 0;
    for (int i = 0; i < nkb; ++i) {
      const int s = i % kRtStages;
      if (lane == 0 && i >= kRtStages) ok = mbar_wait(&empty[s], (uint32_t)((i / kRtStages) - 1) & 1u, abort);
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      if (!ok) break;
      if (lane == 0) mbar_arrive_expect_tx(&full[s], (uint32_t)(kRtA + p.wbox_rows * 128));
      __syncwarp();
      uint8_t* st = smem + s * stage_bytes;
      if (lane == 0) tma_load_2d(&tmX, &full[s], st, (kb0 + i) * 64, t0, pol);
      if (lane == 1) tma_load_2d(&tmW, &full[s], st + kRtA, (kb0 + i) * 64, 0, pol);
      issued = i + 1;
    }
    // After an abort, wait (bounded) for the copies still in flight before the
    // CTA's shared memory is released.
    if (lane == 0 && *abort)
      for (int i = (issued > kRtStages ? issued - kRtStages : 0); i < issued; ++i)
        rt_drain_wait(&full[i % kRtStages], (uint32_t)(i / kRtStages) & 1u);
  } else if (warp == 1) {
    bool ok = true;
    const uint32_t idesc = idesc_bf16(128, NP);
    for (int i = 0; i < nkb && ok; ++i) {
      const int s = i % kRtStages;
      ok = mbar_wait(&full[s], (uint32_t)(i / kRtStages) & 1u, abort);
      ok = __all_sync(0xFFFFFFFFu, ok);
      if (!ok) break;
      tc_fence_after();
      if (lane == 0) {
        uint8_t* st = smem + s * stage_bytes;
        const uint64_t ad = sdesc_k_sw128(smem_u32(st));
        const uint64_t bd = sdesc_k_sw128(smem_u32(st + kRtA));
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)  // K = 16 bf16 (32 bytes) per MMA
          mma_bf16(tmem, ad + 2 * kk, bd + 2 * kk, idesc, (i > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&empty[s]);
      }
      __syncwarp();
    }
    if (lane == 0) mma_commit(&mma_done);
    __syncwarp();
    rt_drain_wait(&mma_done, 0);  // every MMA of this CTA has finished before TMEM is freed
  } else {
    // ---- epilogue: partial logits of this K range -> fp32 reductions ----
    const int q = warp & 3;
    const int row = q * 32 + lane;  // token row of this TMEM lane
    const int t = t0 + row;
    const bool ok = mbar_wait(&mma_done, 0, abort);
    tc_fence_after();
    if (ok && nkb > 0) {
      const uint32_t tl = tmem + ((uint32_t)(q * 32) << 16);
      for (int c0 = 0; c0 < NP; c0 += 16) {
        float v[16];
        tmem_ld16(tl + c0, v);
        tmem_wait_ld();
        if (t < p.T) {
          float* dst = p.logits + (size_t)t * p.E + c0;
#pragma unroll
          for (int j = 0; j < 16; j += 4)
            if (c0 + j < p.E) atomicAdd(reinterpret_cast<float4*>(dst + j), make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]));
        }
      }
    }
    __threadfence();
    named_sync(1, 128);
    if (threadIdx.x == 64) s_last = (atomicAdd(p.counters + tile, 1) == p.splits - 1);
    named_sync(1, 128);
    if (s_last) {
      // ---- last CTA of the tile: top-k + softmax per token ----
      __threadfence();
      const int nrows = min(128, p.T - t0);
      const int ld = p.E + 1;  // padded row: conflict-free column reads
      float* lg = reinterpret_cast<float*>(smem);  // the pipeline stages are idle now
      const int et = threadIdx.x - 64;
      // The tile's rows are one contiguous block of nrows * E floats (E % 4 == 0):
      // float4 loads, several in flight per thread, into padded shared rows;
      // then a second pass returns the block to zero.
      const int n4 = nrows * p.E / 4;
      float4* blk = reinterpret_cast<float4*>(p.logits + (size_t)t0 * p.E);
#pragma unroll 16
      for (int i = et; i < n4; i += 128) {
        const float4 v = __ldcg(blk + i);
        const int idx = i * 4, r = idx / p.E, c = idx - r * p.E;
        float* d = lg + r * ld + c;
        d[0] = v.x;
        d[1] = v.y;
        d[2] = v.z;
        d[3] = v.w;
      }
      named_sync(1, 128);
#pragma unroll 16
      for (int i = et; i < n4; i += 128) blk[i] = make_float4(0.f, 0.f, 0.f, 0.f);
      // one thread per token
      if (et < nrows) {
        const float* r = lg + et * ld;
        const size_t o = (size_t)(t0 + et) * p.k;
        if (p.k <= 8)
          topk8_row(r, p.E, p.k, p.ids + o, p.w + o);
        else
          topk_row_scan(r, p.E, p.k, p.ids + o, p.w + o);
      }
      if (threadIdx.x == 64) p.counters[tile] = 0;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, p.tmem_cols);
  }
  if (threadIdx.x == 0 && *abort) atomicOr(p.status, DEV_TIMEOUT);
}

size_t router_smem_bytes(int E) {
  const int NP = (E + 15) / 16 * 16;
  const int stage = kRtA + ((NP * 128 + 1023) / 1024) * 1024;
  const size_t pipe = (size_t)kRtStages * stage;
  const size_t topk = (size_t)128 * (E + 1) * 4;
  return 1024 + (pipe > topk ? pipe : topk);
}

cudaError_t router_setup(int E) {
  return cudaFuncSetAttribute(router_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)router_smem_bytes(E));
}

cudaError_t launch_router(const CUtensorMap& tx, const CUtensorMap& tw, const RouterParams& p, cudaStream_t s) {
  const int tiles = (p.T + 127) / 128;
  router_kernel<<<tiles * p.splits, kRtThreads, router_smem_bytes(p.E), s>>>(tx, tw, p);
  return cudaGetLastError();
}

}  // namespace moe
