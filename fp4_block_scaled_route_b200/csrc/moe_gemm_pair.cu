// moe_gemm_pair.cu -- GEMM1 (steps 3-5) for MXFP4 weights with FP8
// activations on CTA pairs: tcgen05 MMAs with cta_group::2.
//
// Why: with 4-bit weights in 8-bit containers the block-scaled MMA takes
// K = 32 per instruction, so the single-CTA kernel (moe_gemm.cu) issues 8
// MMAs, 2 scale copies and a commit per 16 KB of weights, and the tensor
// pipe's issue rate, not HBM, bounds it.  Here one MMA with M = 256 covers
// the gate rows (in the even CTA of a cluster of two) and the up rows of the
// same 128 channels (in the odd CTA): per 16 KB of weights the even CTA
// issues 4 MMAs, one scale copy and a commit to each CTA for both SMs.
//
// Measured, it is slower than the single-CTA kernel (decode T = 128: 1.42-
// 1.52 ms against 1.12-1.18 ms per layer): an SM takes one tcgen05
// instruction per ~90 cycles whoever issues it, and only the even CTA of a
// pair issues, so 7 instructions per 16 KB on one SM of two lose to 11 per
// 16 KB on each SM.  The kernel stays as an option (MOE_PAIR_MMA=1).
//
// Sources: GC-MoE abstract (operand-swapped tcgen05 block-scaled MMA on FP4
// weights, fused SwiGLU + requantisation); FusedDeepMoE page (GmmDeqSwigluQuant
// and the BlockEpilogue order: dequantise, SwiGLU, block quantisation).  The
// operand split of a cta_group::2 MMA (A: M/2 rows per CTA, B: N/2 rows per
// CTA, D: M/2 rows x N in each CTA's TMEM) and the forms of the pair
// instructions follow the PTX ISA as used by CUTLASS's sm100 2-SM atoms.
//
// Work unit = (expert token tile of <= 16 positions, 128 output channels).
// Cluster c takes units c, c + clusters, ...; in each, CTA rank 0 holds the
// gate rows, rank 1 the up rows, each loads its own 128 weight rows, its 8
// token rows (rank 0: positions 0-7 of the tile, rank 1: 8-15) and its
// rows' E8M0 scale atom, and every load completes on the even CTA's stage
// barrier.  The even CTA's MMA warp issues the pair MMAs and commits them to
// the stage-done barriers of both CTAs.  Each CTA's epilogue promotes its
// accumulator rows (the activation scale per token and K block, as in the
// single-CTA kernel); at the end of a unit the CTAs swap half of their
// columns through distributed shared memory (gate for positions 8-15 to the
// odd CTA, up for positions 0-7 to the even one), and each computes SwiGLU
// and the FP8 requantisation of its 8 positions.
//
// Every wait is bounded; a CTA that gives up raises its abort word and
// reports MOE_ERR_TIMEOUT, and its partner's waits then run out as well.
#include <cuda_bf16.h>

#include "moe_internal.h"
#include "moe_ptx.cuh"

namespace moe {
namespace {

// ---- pair / cluster PTX ------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// shared::cluster address of the same shared-memory location in CTA `rank`
__device__ __forceinline__ uint32_t mapa_rank(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}
// 2-D TMA load into this CTA's shared memory that completes its bytes on a
// barrier of either CTA of the pair (cluster address)
__device__ __forceinline__ void tma_load_2d_pair(const CUtensorMap* map, uint32_t bar_cluster, void* dst, int c0,
                                                 int c1, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar_cluster), "l"(policy)
      : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void mma_pair_mxf8f6f4(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t sfa,
                                                  uint32_t sfb, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale.scale_vec::1X [%0], %1, %2, %3, [%5], [%6], p;\n\t}\n" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}
// each CTA's shared memory at the descriptor's address -> its own TMEM
__device__ __forceinline__ void tmem_cp_pair_32x128b_warpx4(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}
// arrive on the barrier at a cluster address once the pair MMAs issued so
// far by this thread completed (one commit per CTA whose barrier is signalled)
__device__ __forceinline__ void mma_commit_pair(uint32_t bar_cluster) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar_cluster)
               : "memory");
}
// arrive on a barrier of either CTA: release at cluster scope (data written
// to the partner's shared memory before it), or default semantics (only an
// ordering signal, e.g. after TMEM reads that tcgen05.wait::ld completed)
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar_cluster) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster) : "memory");
}
__device__ __forceinline__ void mbar_arrive_remote(uint32_t bar_cluster) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_acq_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// bounded wait, acquire at cluster scope (for data the partner CTA wrote)
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, volatile int* abort) {
  if (mbar_try_wait_acq_cluster(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_try_wait_acq_cluster(bar, parity)) return true;
    if (*abort) return false;
    if (clock64() - t0 > kWaitCycles) {
      *abort = 1;
      return false;
    }
  }
}
__device__ __forceinline__ void st_cluster_v4(uint32_t addr, float a, float b, float c, float d) {
  asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}
__device__ __forceinline__ void drain_wait_pair(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kWaitCycles) break;
  }
}

struct PairCfg {
  static constexpr int BN = 16;                  // tokens per tile (MMA N; 8 per CTA)
  static constexpr int BH = BN / 2;
  static constexpr int W_BYTES = 128 * 128;      // 128 weight rows, E2M1 in 8-bit containers
  static constexpr int W_TX = W_BYTES / 2;       // bytes read from global memory (packed)
  static constexpr int B_BYTES = BH * 128;       // this CTA's 8 token rows of the K block
  static constexpr int SF_BYTES = 512;           // the weight rows' E8M0 atom of the K block
  static constexpr int STAGE_BYTES = 18432;      // W | B | SF, 1024-byte aligned
  static constexpr int STAGES = 11;
  static constexpr int NBUF = 8;                 // TMEM accumulators in flight
  static constexpr int NMD = STAGES + NBUF;      // MMA-done ring: every waiter within one phase
  static constexpr int KB_MAX = 64;
  static constexpr int NPROD = 2;
  static constexpr int NMMA = 2;                 // MMA warps (even CTA), iterations dealt in turn
  static constexpr int MMA_WARP = 2;
  static constexpr int EPI_WARP0 = 4;
  static constexpr int THREADS = 256;
  static constexpr int ACC_COLS = NBUF * BN;     // 128
  static constexpr int SFA_COL = ACC_COLS;       // 4 columns per accumulator buffer
  static constexpr int SFB_COL = SFA_COL + NBUF * 4;
  static constexpr int TMEM_COLS = 256;
  // transaction bytes of one stage of the pair (both CTAs' loads complete on
  // the even CTA's barrier)
  static constexpr int TX_PAIR = 2 * (W_TX + B_BYTES + SF_BYTES);
  static constexpr int AUX_FLOATS = BN * KB_MAX + 2 * BN + 4 * BN + 2 * 128 * BH;  // asc, cs, red, xbuf
  static constexpr int NBARS = STAGES + NMD + NBUF + 2 + 2 + 1;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + AUX_FLOATS * 4 + NBARS * 8 + 16;
  static_assert(SFB_COL + 4 <= TMEM_COLS, "TMEM");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
  static_assert(STAGES >= NPROD, "a producer could pass a stale MMA-done phase");
  // an MMA warp's parity wait on a stage is exact when every iteration that
  // shares the stage is its own or already released (see moe_gemm.cu)
  static_assert(STAGES % NMMA == 0 || NBUF <= STAGES, "an MMA warp could pass a stage's stale phase");
  static_assert(W_BYTES + B_BYTES + SF_BYTES <= STAGE_BYTES && STAGE_BYTES % 1024 == 0, "stage layout");
};

__global__ void __launch_bounds__(PairCfg::THREADS, 1)
    moe_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                         const __grid_constant__ CUtensorMap tmS, const GemmParams p) {
  using C = PairCfg;
  constexpr int STAGES = C::STAGES, NBUF = C::NBUF, NMD = C::NMD, BN = C::BN, BH = C::BH, KB_MAX = C::KB_MAX;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* asc = reinterpret_cast<float*>(smem + STAGES * C::STAGE_BYTES);  // [KB_MAX][BN] activation scales
  float* cs = asc + BN * KB_MAX;                                          // [2][BN] scale of K blocks kb, kb+1
  float* red = cs + 2 * BN;                                               // [4][BN] per-quarter amax
  float* xbuf = red + 4 * BN;                                             // [2][128][BH] received half
  uint64_t* bars = reinterpret_cast<uint64_t*>(xbuf + 2 * 128 * BH);
  uint64_t* full = bars;                // [STAGES] (used in the even CTA)
  uint64_t* mdone = full + STAGES;      // [NMD] (both CTAs, a commit to each)
  uint64_t* tempty = mdone + NMD;       // [NBUF] (even CTA: 4 local + 4 remote warp arrivals)
  uint64_t* xfull = tempty + NBUF;      // [2] partner's half landed (4 remote warp arrivals)
  uint64_t* xempty = xfull + 2;         // [2] partner consumed our half (4 remote warp arrivals)
  uint64_t* done = xempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool lead = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int KB = p.kblocks;
  const int num_tiles = *p.num_tiles;
  const int rows_e = 2 * p.I;
  const int NRT = p.I / 128;
  const int total = num_tiles * NRT;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) mbar_init(&full[s], 1);
    for (int i = 0; i < NMD; ++i) mbar_init(&mdone[i], 1);
    for (int b = 0; b < NBUF; ++b) mbar_init(&tempty[b], 8);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&xfull[b], 4);
      mbar_init(&xempty[b], 4);
    }
    mbar_init(done, C::NMMA);
    *abort = 0;
    mbar_fence_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_map(&tmW);
    tma_prefetch_map(&tmX);
    tma_prefetch_map(&tmS);
  }
  if (warp == C::MMA_WARP) tmem_alloc_pair(tmem_holder, C::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  if (warp == C::MMA_WARP) tmem_relinquish_pair();
  // B-side scales: all 1.0 (E8M0 127); the activation scales are promoted
  // in the epilogue
  if (warp >= C::EPI_WARP0) {
    const uint32_t q = warp & 3;
    tmem_st4(tmem + ((q * 32) << 16) + C::SFB_COL, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu);
    tmem_wait_st();
  }
  tc_fence_before();
  // both CTAs' barriers exist and TMEM is allocated before any cross-CTA signal
  cluster_sync_all();
  tc_fence_after();
  griddep_launch_dependents();

  const uint32_t full0 = mapa_rank(full, 0);  // the even CTA's stage barriers (+ 8 bytes per stage)

  if (warp < C::NPROD) {
    // ---------------- TMA producers (both CTAs) ----------------
    // Warp pr fills the stages of pipeline iterations it % NPROD == pr: lane
    // 0 the weight tile, lane 1 the token rows, lane 2 the scale atom.  The
    // even CTA's lane 0 posts the pair's transaction bytes.  The weights of
    // the first ring pass go out before the previous kernel (the
    // quantisation) has finished; their token rows follow after the wait.
    const int pr = warp;
    const uint64_t pol_w = policy_evict_first();
    const uint64_t pol_a = policy_evict_last();
    uint32_t issued = 0, last_par = 0;
    bool ok = true, waited = false;
    constexpr int NPEND = (STAGES + C::NPROD - 1) / C::NPROD;
    int npend = 0;
    int pend_kb[NPEND], pend_p0[NPEND], pend_st[NPEND];
    auto load_tokens = [&](int st, int kb, int p0) {
      tma_load_2d_pair(&tmX, full0 + 8u * st, smem + st * C::STAGE_BYTES + C::W_BYTES, kb * 128,
                       p0 + (int)rank * BH, pol_a);
    };
    int it = 0;
    for (int u = pair; u < total; u += npairs) {
      const int rt = u / num_tiles, ti = u % num_tiles;
      const int4 tile = p.tiles[ti];
      const int e = tile.x, p0 = tile.y;
      const int row = e * rows_e + ((int)rank * NRT + rt) * 128;  // gate rows (rank 0) or up rows (rank 1)
      for (int kb = 0; kb < KB; ++kb, ++it) {
        if (it % C::NPROD != pr) continue;
        const int stage = it % STAGES;
        const uint32_t phase = (uint32_t)(it / STAGES) & 1u;
        if (lane == 1 && !waited && it >= STAGES) {
          griddep_wait();
          for (int i = 0; i < npend; ++i) load_tokens(pend_st[i], pend_kb[i], pend_p0[i]);
          waited = true;
        }
        if (lane == 0 && ok && it >= STAGES) {  // the stage's previous iteration has been consumed
          const int prev = it - STAGES;
          ok = mbar_wait(&mdone[prev % NMD], (uint32_t)(prev / NMD) & 1u, abort);
        }
        ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
        if (!ok) continue;
        if (lane == 0) {
          if (lead) mbar_arrive_expect_tx(&full[stage], C::TX_PAIR);
          issued |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
        }
        __syncwarp();
        uint8_t* st = smem + stage * C::STAGE_BYTES;
        if (lane == 0) {
          tma_load_2d_pair(&tmW, full0 + 8u * stage, st, kb * 128, row, pol_w);
        } else if (lane == 1) {
          if (waited) {
            load_tokens(stage, kb, p0);
          } else {
            pend_kb[npend] = kb;
            pend_p0[npend] = p0;
            pend_st[npend] = stage;
            ++npend;
          }
        } else if (lane == 2) {
          // the atom of these 128 rows and K block: two 256-byte rows of the
          // scale map ([row / 128][KB][512] bytes)
          tma_load_2d_pair(&tmS, full0 + 8u * stage, st + C::W_BYTES + C::B_BYTES, 0,
                           2 * ((row / 128) * KB + kb), pol_w);
        }
      }
    }
    if (lane == 1 && !waited) {
      griddep_wait();
      for (int i = 0; i < npend; ++i) load_tokens(pend_st[i], pend_kb[i], pend_p0[i]);
    }
    __syncwarp();
    // after an abort, the even CTA waits (bounded) for the stages it armed;
    // those phases carry the odd CTA's bytes as well
    if (lane == 0 && lead && *abort)
      for (int s = 0; s < STAGES; ++s)
        if (issued & (1u << s)) drain_wait_pair(&full[s], (last_par >> s) & 1u);
  } else if (warp < C::MMA_WARP + C::NMMA) {
    // ---------------- pair MMA issuers (even CTA) ----------------
    if (lead) {
      const int mw = warp - C::MMA_WARP;
      const uint32_t mdone1 = mapa_rank(mdone, 1);  // the odd CTA's stage-done barriers
      bool ok = true;
      int mit = 0;
      for (int u = pair; u < total; u += npairs) {
        for (int kb = 0; kb < KB; ++kb, ++mit) {
          if (mit % C::NMMA != mw) continue;
          const int stage = mit % STAGES, buf = mit % NBUF;
          const uint32_t phase = (uint32_t)(mit / STAGES) & 1u, tphase = (uint32_t)(mit / NBUF) & 1u;
          if (ok) ok = mbar_wait(&tempty[buf], tphase ^ 1u, abort);
          if (ok) ok = mbar_wait(&full[stage], phase, abort);
          ok = __all_sync(0xFFFFFFFFu, ok);
          if (!ok) continue;
          tc_fence_after();
          if (lane == 0) {
            uint8_t* st = smem + stage * C::STAGE_BYTES;
            const uint64_t ad = sdesc_k_sw128(smem_u32(st));
            const uint64_t bd = sdesc_k_sw128(smem_u32(st + C::W_BYTES));
            const uint32_t sfa = tmem + C::SFA_COL + buf * 4;
            uint64_t sd = 0;
            sd |= static_cast<uint64_t>((smem_u32(st + C::W_BYTES + C::B_BYTES) & 0x3FFFFu) >> 4);
            sd |= static_cast<uint64_t>(128 >> 4) << 32;  // 8 rows x 16 bytes per core group
            sd |= static_cast<uint64_t>(1) << 46;
            tmem_cp_pair_32x128b_warpx4(sfa, sd);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_pair_mxf8f6f4(tmem + buf * BN, ad + 2 * kk, bd + 2 * kk, idesc_mxf8f6f4(256, BN, 5, 0, kk, 0), sfa,
                                tmem + C::SFB_COL, kk > 0);
            mma_commit_pair(smem_u32(&mdone[mit % NMD]));
            mma_commit_pair(mdone1 + 8u * (mit % NMD));
          }
          __syncwarp();
        }
      }
      if (lane == 0) mma_commit(done);
      __syncwarp();
      drain_wait_pair(done, 0);
    }
  } else if (warp >= C::EPI_WARP0) {
    // ---------------- epilogue (both CTAs) ----------------
    const int q = warp & 3;          // TMEM lane quarter
    const int row = q * 32 + lane;   // weight row within the tile = TMEM lane = channel
    const int etid = threadIdx.x - 32 * C::EPI_WARP0;
    const uint32_t tempty0 = mapa_rank(tempty, 0);
    const uint32_t other = rank ^ 1u;
    const uint32_t xbuf_peer = mapa_rank(xbuf, other);
    const uint32_t xfull_peer = mapa_rank(xfull, other);
    const uint32_t xempty_peer = mapa_rank(xempty, other);
    bool ok = true;
    int eit = 0, ju = 0;
    griddep_wait();  // activation scales come from the quantisation kernel
    for (int u = pair; u < total; u += npairs, ++ju) {
      const int rt = u / num_tiles, ti = u % num_tiles;
      const int4 tile = p.tiles[ti];
      const int p0 = tile.y, nv = tile.z;
      {
        // the unit's activation scales [KB][BN], every load in flight at once
        constexpr int NPA = BN * KB_MAX / 128;
        float v[NPA];
#pragma unroll
        for (int r = 0; r < NPA; ++r) {
          const int i = etid + r * 128;
          v[r] = (i < BN * KB) ? p.ascale[(size_t)(i / BN) * p.scale_ld + p0 + (i % BN)] : 0.0f;
        }
#pragma unroll
        for (int r = 0; r < NPA; ++r) asc[etid + r * 128] = v[r];
      }
      named_sync(1, 128);
      float acc[BN];
#pragma unroll
      for (int c = 0; c < BN; ++c) acc[c] = 0.0f;
      for (int kb = 0; kb < KB; ++kb, ++eit) {
        const int buf = eit % NBUF;
        if (ok) ok = mbar_wait(&mdone[eit % NMD], (uint32_t)(eit / NMD) & 1u, abort);
        ok = __all_sync(0xFFFFFFFFu, ok);
        if (ok) {
          tc_fence_after();
          float d[BN];
          tmem_ld16(tmem + ((uint32_t)(q * 32) << 16) + buf * BN, d);
          tmem_wait_ld();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            if (lead) mbar_arrive(&tempty[buf]);
            else mbar_arrive_remote(tempty0 + 8u * buf);
          }
#pragma unroll
          for (int c = 0; c < BN; ++c) acc[c] = fmaf(d[c], asc[kb * BN + c], acc[c]);
        }
      }
      // ---- swap halves with the partner: rank 0 keeps positions 0-7 (gate
      // here, up from rank 1), rank 1 keeps positions 8-15 ----
      const int xb = ju & 1;
      const uint32_t xphase = (uint32_t)(ju >> 1) & 1u;
      if (ju >= 2 && ok) ok = mbar_wait_cluster(&xempty[xb], xphase ^ 1u, abort);
      ok = __all_sync(0xFFFFFFFFu, ok);
      {
        const int c0 = lead ? BH : 0;  // the half the partner keeps
        const uint32_t dst = xbuf_peer + (uint32_t)((xb * 128 + row) * BH) * 4u;
        st_cluster_v4(dst, acc[c0], acc[c0 + 1], acc[c0 + 2], acc[c0 + 3]);
        st_cluster_v4(dst + 16u, acc[c0 + 4], acc[c0 + 5], acc[c0 + 6], acc[c0 + 7]);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(xfull_peer + 8u * xb);
      if (ok) ok = mbar_wait_cluster(&xfull[xb], xphase, abort);
      ok = __all_sync(0xFFFFFFFFu, ok);
      float h[BH];
      {
        const float* rx = xbuf + (xb * 128 + row) * BH;
        const int m0 = lead ? 0 : BH;  // this CTA's positions
#pragma unroll
        for (int i = 0; i < BH; ++i) {
          const float g = lead ? acc[m0 + i] : rx[i];
          const float up = lead ? rx[i] : acc[m0 + i];
          const float sig = __fdiv_rn(1.0f, 1.0f + expf(-g));
          h[i] = g * sig * up;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(xempty_peer + 8u * xb);
      // ---- FP8 requantisation per position over the tile's 128 channels ----
      const int ct = rt;
      const int ch = ct * 128 + row;
      const int m0 = lead ? 0 : BH;
#pragma unroll
      for (int i = 0; i < BH; ++i) {
        float m = fabsf(h[i]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
        if (lane == 0) red[q * BN + i] = m;
      }
      named_sync(1, 128);
      if (ok) {
#pragma unroll
        for (int i = 0; i < BH; ++i) {
          const int j = m0 + i;  // position within the tile
          const float amax = fmaxf(fmaxf(red[i], red[BN + i]), fmaxf(red[2 * BN + i], red[3 * BN + i]));
          const float sc = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 448.0f);
          if (j < nv) {
            p.hq[(size_t)(p0 + j) * p.I + ch] = static_cast<uint8_t>(f32_to_e4m3(__fdiv_rn(h[i], sc)));
            if (row == 0) p.hs[(size_t)ct * p.scale_ld + p0 + j] = sc;
          }
        }
      }
      named_sync(1, 128);  // red and asc are reused by the next unit
    }
  }

  tc_fence_before();
  __syncthreads();
  // neither CTA releases its TMEM or shared memory while the partner may
  // still signal it
  cluster_sync_all();
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, C::TMEM_COLS);
  }
  if (threadIdx.x == 0 && *abort) atomicOr(p.status, DEV_TIMEOUT);
}

}  // namespace

// Clusters of two CTAs that can be resident at once (one CTA per SM).
static int g_pair_clusters = -1;

cudaError_t gemm_pair_setup() {
  cudaError_t e = cudaFuncSetAttribute(moe_gemm_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       PairCfg::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(moe_gemm_pair_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 0);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * (sms / 2));
  cfg.blockDim = dim3(PairCfg::THREADS);
  cfg.dynamicSmemBytes = PairCfg::SMEM_BYTES;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int clusters = 0;
  if ((e = cudaOccupancyMaxActiveClusters(&clusters, moe_gemm_pair_kernel, &cfg)) != cudaSuccess) return e;
  g_pair_clusters = clusters < sms / 2 ? clusters : sms / 2;
  return g_pair_clusters > 0 ? cudaSuccess : cudaErrorInvalidConfiguration;
}

int gemm_pair_clusters() { return g_pair_clusters; }

cudaError_t launch_gemm1_pair(const CUtensorMap& tw, const CUtensorMap& tx8, const CUtensorMap& tsf,
                              const GemmParams& p, cudaStream_t s) {
  if (g_pair_clusters <= 0) return cudaErrorInvalidConfiguration;
  if (p.kblocks > PairCfg::KB_MAX) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * g_pair_clusters);
  cfg.blockDim = dim3(PairCfg::THREADS);
  cfg.dynamicSmemBytes = PairCfg::SMEM_BYTES;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, moe_gemm_pair_kernel, tw, tx8, tsf, p);
}

}  // namespace moe
