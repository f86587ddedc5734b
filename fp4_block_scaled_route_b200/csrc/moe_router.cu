// moe_router.cu -- fused router ("Mega Gate"): the routing GEMM and the MoE
// routing step behind one call (DeepGEMM 26/09 news page: the router GEMM and
// the MoE routing operations fused).
//
//   logits[t, e] = sum_h x[t, h] * Wr[e, h]      x bf16 [T, H], Wr bf16 [E, H]
//   ids[t, :]    = the k largest logits of token t, descending, ties to the
//                  lower expert index
//   w[t, j]      = softmax over the k chosen logits
//
// Two kernels, the second a programmatic dependent launch of the first:
//   router_kernel       CTA (token tile of 128, K split): TMA streams 64-
//                       element K blocks of x and Wr into shared memory,
//                       tcgen05.mma kind::f16 (bf16 x bf16, fp32 accumulate;
//                       M = 128 tokens, N = E experts) accumulates the CTA's
//                       K range in TMEM, and the epilogue adds its partial
//                       logits into an fp32 buffer with vector reductions.
//   router_topk_kernel  one warp per token: top k + softmax from the summed
//                       logits, then the token's buffer row back to zero for
//                       the next call.
// (Selecting in the CTA that finishes a tile last kept one CTA busy with 128
// tokens while the rest of the GPU idled: 36 us of a 68 us call at T = 128.)
#include <cuda_bf16.h>

#include "moe_internal.h"
#include "moe_ptx.cuh"

namespace moe {

namespace {

constexpr int kRtStages = 4;
constexpr int kRtThreads = 192;  // warp 0 TMA, warp 1 MMA + TMEM, warps 2-5 epilogue
constexpr int kRtA = 128 * 128;  // token tile: 128 rows x 64 bf16

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

// Each (value, index) pair becomes one 64-bit key that orders like "larger
// logit first, then lower index": the float's order-preserving bit pattern in
// the high word and the complemented index in the low word, so all keys of a
// row are distinct and plain 64-bit comparisons select.
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

// Top-8 of two lists sorted in descending key order, left in `a` (sorted):
// the element-wise larger of a[i] and b[7-i] is a bitonic sequence holding
// exactly the 8 largest keys of both lists, and three half-cleaner stages
// (distances 4, 2, 1) sort it.  Keys are distinct (the expert index is part
// of the key), so both partners of an exchange end with the same list.
__device__ __forceinline__ void merge_top8(uint64_t (&a)[8], const uint64_t (&b)[8]) {
  uint64_t m[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) m[i] = a[i] > b[7 - i] ? a[i] : b[7 - i];
#pragma unroll
  for (int d = 4; d > 0; d >>= 1)
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if ((i & d) == 0) {
        const uint64_t x = m[i], y = m[i + d];
        m[i] = x > y ? x : y;
        m[i + d] = x > y ? y : x;
      }
#pragma unroll
  for (int i = 0; i < 8; ++i) a[i] = m[i];
}

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
  // the selection kernel may be scheduled now; it waits for this grid's
  // completion before it reads the logits
  griddep_launch_dependents();

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
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, p.tmem_cols);
  }
  if (threadIdx.x == 0 && *abort) atomicOr(p.status, DEV_TIMEOUT);
}

// Eight keys sorted in descending order (bitonic network: blocks of 2, 4, 8).
__device__ __forceinline__ void sort8_desc(uint64_t (&m)[8]) {
#pragma unroll
  for (int kk = 2; kk <= 8; kk <<= 1)
#pragma unroll
    for (int j = kk >> 1; j > 0; j >>= 1)
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int l = i ^ j;
        if (l > i) {
          const uint64_t x = m[i], y = m[l];
          const bool desc = (i & kk) == 0;
          const bool keep = desc ? x > y : x < y;
          m[i] = keep ? x : y;
          m[l] = keep ? y : x;
        }
      }
}

// One warp per token t < T: lane l takes logits l, l + 32, ... (E <= 256, at
// most 8), sorts its keys, and five shuffle rounds merge the lanes' lists
// into the token's top 8; lane 0 writes the k ids and softmax weights (k > 8:
// lane 0 scans the row k times).  The warp then zeroes the row.
constexpr int kTopkWarps = 4;
__global__ void __launch_bounds__(32 * kTopkWarps) router_topk_kernel(const RouterParams p) {
  griddep_wait();  // the logits are complete once the GEMM grid has finished
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * kTopkWarps + warp;
  if (t >= p.T) return;  // warp-uniform
  float* row = p.logits + (size_t)t * p.E;
  int32_t* ids = p.ids + (size_t)t * p.k;
  float* w = p.w + (size_t)t * p.k;
  if (p.k <= 8) {
    uint64_t ls[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = lane + 32 * j;
      ls[j] = (e < p.E) ? rank_key(__ldcg(row + e), e) : 0;  // 0 ranks after every key
    }
    sort8_desc(ls);
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      uint64_t other[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) other[i] = __shfl_xor_sync(0xFFFFFFFFu, ls[i], off);
      merge_top8(ls, other);
    }
    if (lane == 0) {
      const float m = key_value(ls[0]);
      float z = 0.0f;
#pragma unroll
      for (int s = 0; s < 8; ++s)
        if (s < p.k) z += expf(key_value(ls[s]) - m);
#pragma unroll
      for (int s = 0; s < 8; ++s)
        if (s < p.k) {
          ids[s] = key_index(ls[s]);
          w[s] = __fdiv_rn(expf(key_value(ls[s]) - m), z);
        }
    }
  } else if (lane == 0) {
    topk_row_scan(row, p.E, p.k, ids, w);
  }
  __syncwarp();
  for (int e = lane * 4; e < p.E; e += 128) *reinterpret_cast<float4*>(row + e) = make_float4(0.f, 0.f, 0.f, 0.f);
}

size_t router_smem_bytes(int E) {
  const int NP = (E + 15) / 16 * 16;
  const int stage = kRtA + ((NP * 128 + 1023) / 1024) * 1024;
  return 1024 + (size_t)kRtStages * stage;
}

cudaError_t router_setup(int E) {
  return cudaFuncSetAttribute(router_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)router_smem_bytes(E));
}

cudaError_t launch_router(const CUtensorMap& tx, const CUtensorMap& tw, const RouterParams& p, cudaStream_t s) {
  const int tiles = (p.T + 127) / 128;
  router_kernel<<<tiles * p.splits, kRtThreads, router_smem_bytes(p.E), s>>>(tx, tw, p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((p.T + kTopkWarps - 1) / kTopkWarps));
  cfg.blockDim = dim3(32 * kTopkWarps);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, router_topk_kernel, p);
}

}  // namespace moe
