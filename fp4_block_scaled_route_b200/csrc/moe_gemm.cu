// moe_gemm.cu -- grouped expert GEMMs on tcgen05 tensor cores (sm_100a).
//
// One persistent kernel template serves both GEMMs of the layer:
//   GEMM1 (steps 3-5): per expert, G = Xq_e * W13[e]^T over K = H, then
//          SwiGLU (gate = first I rows) and FP8 requantisation per token per
//          128 channels, written as the GEMM2 activations hq / hs.
//   GEMM2 (steps 6-7): per expert, Y = Hq_e * W2[e]^T over K = I, then the
//          top-k weighted combine: out_acc[token] += w * Y (fp32 atomics).
// Sources: GC-MoE abstract (operand-swapped tcgen05 block-scaled MMA, fused
// SwiGLU + requantisation, optional shared experts); FusedDeepMoE page
// (GmmDeqSwigluQuant and GmmDeq with the combine as epilogue callback;
// BlockEpilogue order: dequant by weight scale and per-token scale, SwiGLU,
// block quant).
//
// Operand swap: the expert's weight rows fill the 128-row M side of the MMA
// and the (few) tokens of the expert are the N side (BN = 16 .. 128), so a
// decode step with 1-16 tokens per expert still issues full-height MMAs while
// the weights stream through shared memory exactly once.
//
// Work unit = (row tile rt of 128 weight rows [GEMM1: 128 gate + 128 up
// rows], token tile of <= BN positions of one expert).  Units are spread over
// a grid of one CTA per SM; every CTA walks units u = blockIdx.x + i*grid.
// For tiles of 64 or more tokens the order is token-tile major
// (u = tile * row_tiles + rt): all row tiles of an expert run at the same
// time and read that expert's token tile from L2, and its sibling token tiles
// read its weight tiles from L2.  Decode tiles run row-tile major.
//
// Warp roles (one CTA per SM):
//   warp 0     TMA producer: weight tiles (128 rows x 128 K bytes, 128-byte
//              swizzle, L2 evict-first) and the token tile, STAGES deep.
//   warp 1     allocates TMEM; one lane issues tcgen05.mma (K = 32 per
//              instruction, 4 per 128-wide K block) into one of two TMEM
//              accumulators per K block and commits to mbarriers.
//   warps 2..  epilogue: per K block, tcgen05.ld the block's fp32 partial and
//              promote it with the block's scales (FP8: weight block scale x
//              per-token activation scale; MXFP4: the E8M0 weight scales are
//              applied by the MMA and only the activation scale is promoted),
//              then the fused SwiGLU/requant or combine tail.
// Per-128-K promotion is required because the fp32 FP8 scales (amax/448) are
// not powers of two and so cannot be fed to the block-scaled MMA.
#include <cuda_bf16.h>

#include "moe_dispatch.cuh"
#include "moe_internal.h"
#include "moe_ptx.cuh"

namespace moe {

// NT: 128-row weight tiles per stage and unit.  GEMM1: pairs of a gate and
// an up tile of the same channels (NT = 2: one 128-channel tile, NT = 4: two
// neighbouring ones); GEMM2: NT neighbouring 128-row tiles of W2.  More tiles
// per stage share one token tile, its block-scale copies and one commit.
template <int KIND, int BN, int WFMT, int NT = (KIND == 1 ? 2 : 1)>
struct GemmCfg {
  static constexpr int NA = NT;                           // weight tiles per stage
  static_assert(KIND != 1 || NT % 2 == 0, "GEMM1 tiles come in gate/up pairs");
  // NVFP4 (WFMT 2): both operands packed E2M1, 64 bytes per row per 128-wide
  // K block, 64-byte swizzle; the block scales of a K block travel with the
  // stage as 512-byte atoms, two per weight tile and two for the token tile
  // (one per K = 64 MMA step each).
  // MXFP4 x MXFP4 (WFMT 3): the same packed operands with E8M0 scales per
  // 32, one 512-byte atom per weight tile and one for the token tile per K
  // block (its two K = 64 steps use scale bytes 0-1 and 2-3); every scale is
  // applied by the MMA.
  static constexpr bool NV = WFMT == 2;
  static constexpr bool MXA = WFMT == 3;
  static constexpr bool P4 = NV || MXA;                   // packed E2M1 on both operands
  static constexpr int KBYTES = P4 ? 64 : 128;            // smem bytes per row per K block
  static constexpr int A_BYTES = 128 * KBYTES;            // FP8 / E2M1 padded to 8 bits: 128 B rows
  static constexpr int B_BYTES = BN * KBYTES;
  static constexpr int SFA_BYTES = (WFMT == 1 || MXA) ? 512 : NV ? 1024 : 0;  // per weight tile
  static constexpr int SFB_BYTES = NV ? 1024 : MXA ? 512 : 0;
  static constexpr int SF_BYTES = NA * SFA_BYTES + SFB_BYTES;
  static constexpr int STAGE_BYTES = NA * A_BYTES + B_BYTES + SF_BYTES;
  static constexpr int KB_MAX = 64;                       // K <= 8192
  // Epilogue column groups (warpgroups, each taking CPT of the BN columns):
  // two for stages of four tiles, whose per-unit SwiGLU + requant tail would
  // otherwise stall the MMAs (only NBUF K blocks fit ahead of it).
  static constexpr int CG = (BN > 64) ? BN / 64 : (NT == 4) ? 2 : 1;
  static constexpr int CPT = BN / CG;                     // columns per epilogue thread
  static constexpr int EPI_THREADS = 128 * CG;
  // Warpgroup 0: NPROD TMA producer warps (warp p issues all loads of the
  // pipeline iterations it with it % NPROD == p) and NMMA MMA warps (MMA warp
  // m issues all MMAs of the iterations with it % NMMA == m, each iteration
  // into its own TMEM accumulator).  One issuing thread fills shared memory
  // through TMA at only ~47 GB/s, and one thread issues a tcgen05.mma only
  // every ~100 cycles whatever N is, which for 4-bit weights is below the
  // HBM rate; two of each double both.  Warpgroups 1..CG: the epilogue.
  // The epilogue warps need not start at a warpgroup boundary: TMEM lane
  // access depends only on the warp index mod 4, and any 4 consecutive warps
  // cover the 4 lane quarters.  Tiles of 64 tokens or more keep two producers
  // so that the epilogue's accumulators fit in the per-thread registers.
  static constexpr int NPROD = (BN >= 64) ? 2 : 3;
  static constexpr int NMMA = 2;
  // Unit order: wide token tiles (prefill) run token-tile major so an
  // expert's token tile is shared through L2 by its row tiles; decode runs
  // row-tile major (measured ~3% faster there).
  static constexpr bool TILE_MAJOR = BN >= 64;
  static constexpr int MMA_WARP = NPROD;  // first MMA warp; allocates TMEM
  static constexpr int EPI_WARP0 = NPROD + NMMA;
  static constexpr int THREADS = 32 * EPI_WARP0 + EPI_THREADS;
  static constexpr int MAX_STAGES = P4 ? 24 : 12;
  static constexpr int NBARS = 2 * MAX_STAGES + 2 * 8 + 1;
  static constexpr int AUX_BYTES =
      ((BN * KB_MAX + NA * KB_MAX + 6 * BN + 2 * NA * BN) * 4 + NBARS * 8 + 16 + 15) / 16 * 16;
  static constexpr int SMEM_LIMIT = 232448;
  static constexpr int FIT = (SMEM_LIMIT - 1024 - AUX_BYTES) / STAGE_BYTES;
  static constexpr int STAGES = FIT > MAX_STAGES ? MAX_STAGES : FIT;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + AUX_BYTES;
  // TMEM accumulators in flight: the MMA warps may run NBUF K blocks ahead of
  // the promoting epilogue (short K steps would otherwise be latency bound).
  //
  // Bound on NBUF from the stage ring.  The MMA warps take the iterations in
  // turn and are not ordered among themselves.  When warp m waits for the
  // stage of iteration it, the epilogue has released it - NBUF (so every
  // iteration up to it - NBUF has landed), and warp m has consumed its own
  // earlier iterations; an iteration it - d of another MMA warp (d not a
  // multiple of NMMA, d < NBUF) may still be waiting for its bytes.  If it
  // shares the stage (d a multiple of STAGES), warp m's parity wait sees that
  // stage's phase before last as complete and passes before its own bytes
  // land, and the producer can then post a second transaction count on a
  // phase that has not completed.  So either STAGES is a multiple of NMMA
  // (every iteration sharing warp m's stage is warp m's own) or NBUF <= STAGES.
  static constexpr int NBUF_RAW = 256 / (NA * BN);
  static constexpr int NBUF_WANT = NBUF_RAW < 2 ? 2 : (NBUF_RAW > 8 ? 8 : NBUF_RAW);
  static constexpr int NBUF = (STAGES % NMMA == 0 || STAGES >= NBUF_WANT) ? NBUF_WANT : STAGES;
  static_assert(STAGES % NMMA == 0 || NBUF <= STAGES, "an MMA warp could pass a stage's stale phase");
  // The producers take the iterations in turn as well; a producer's wait for
  // the MMAs of it - STAGES is exact when its previous iteration it - NPROD
  // is no older than that (its own wait then implies the phase before).
  static_assert(STAGES >= NPROD, "a producer could pass a stale MMA-done phase");
  static constexpr int ACC_COLS = NBUF * NA * BN;         // NBUF accumulators
  // Scale-factor columns per accumulator buffer: MXFP4 one 4-column atom per
  // weight tile (B: 4 shared columns of unit scales); NVFP4 two atoms per
  // weight tile and two for the token tile.  An MMA's scale operand starts
  // at a 4-column atom boundary.
  static constexpr int SFA_PER_BUF = NV ? NA * 8 : NA * 4;
  static constexpr int SFA_COL = ACC_COLS;
  static constexpr int SFB_COL = SFA_COL + NBUF * SFA_PER_BUF;
  static constexpr int SFB_PER_BUF = NV ? 8 : 4;
  static constexpr int USED_COLS = (WFMT == 1) ? SFB_COL + 4 : P4 ? SFB_COL + NBUF * SFB_PER_BUF : ACC_COLS;
  static constexpr int TMEM_COLS = USED_COLS <= 32 ? 32 : USED_COLS <= 64 ? 64 : USED_COLS <= 128 ? 128
                                 : USED_COLS <= 256 ? 256 : 512;
  // Transaction bytes per stage: a packed-E2M1 weight tile moves 64 bytes per
  // row from global memory although it lands as 128 padded bytes in smem.
  static constexpr int A_TX = (WFMT == 1) ? A_BYTES / 2 : A_BYTES;
  static constexpr int TX_BYTES = NA * A_TX + B_BYTES + SF_BYTES;
  static_assert(STAGES >= 2, "shared memory too small");
  static_assert(USED_COLS <= 512, "TMEM too small");
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 64, "BN");
  static_assert(CPT % 8 == 0, "columns per epilogue thread");
  // NVFP4 token scales: an atom is one box of 32 positions, token n of the
  // tile in row n (TMEM lane n, the atom's first column).
  static_assert(!P4 || BN <= 32, "4-bit activation tiles hold at most 32 tokens");
};

// Moves entries CH..N-1 of a register array to 0..N-CH-1 (the last CH are
// left for the caller); with static indices the array stays in registers.
template <int N, int CH>
__device__ __forceinline__ void rotl(float* a) {
#pragma unroll
  for (int i = 0; i + CH < N; ++i) a[i] = a[i + CH];
}

// Bounded wait that ignores the abort word (used to drain in-flight copies
// and MMAs before the CTA releases its shared memory and TMEM).
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kWaitCycles) break;
  }
}

// DISP: the GEMM1 launch with dispatch overlap (moe_dispatch.cuh); the other
// instantiations hold none of its code.
template <int KIND, int BN, int WFMT, int NT, bool DISP>
__global__ void __launch_bounds__(GemmCfg<KIND, BN, WFMT, NT>::THREADS, 1)
    moe_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmS, const GemmParams p) {
  using C = GemmCfg<KIND, BN, WFMT, NT>;
  constexpr int NA = C::NA, STAGES = C::STAGES, KB_MAX = C::KB_MAX, CPT = C::CPT;
  constexpr bool NV = C::NV;
  constexpr bool MXA = C::MXA;
  constexpr bool P4 = C::P4;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + STAGES * NA * C::A_BYTES;
  uint8_t* sSF = sB + STAGES * C::B_BYTES;
  float* asc = reinterpret_cast<float*>(sSF + STAGES * C::SF_BYTES);  // [KB_MAX][BN] activation scales
  float* wsc = asc + BN * KB_MAX;                                     // [NA][KB_MAX] FP8 weight scales (NVFP4: [0] global)
  float* red = wsc + NA * KB_MAX;                                     // [4][BN] per-quarter amax
  int* slot_tok = reinterpret_cast<int*>(red + 4 * BN);               // [BN] GEMM2: token of column
  float* slot_w = reinterpret_cast<float*>(slot_tok + BN);            // [BN] GEMM2: combine weight
  float* cs = slot_w + BN;                                            // [2][NA][BN] combined scales ring
  uint64_t* bars = reinterpret_cast<uint64_t*>(cs + 2 * NA * BN);
  // full[s]: TMA bytes of stage s landed.  mdone[i % NMD]: the MMAs of
  // pipeline iteration i completed -- one tcgen05.commit per iteration tells
  // the producers that the stage is free and the epilogue that the TMEM
  // accumulator is ready (each commit costs the tensor pipe several hundred
  // cycles, so a second one per iteration would halve the decode rate).
  // tempty[b]: the epilogue has read TMEM accumulator b.  NMD = STAGES +
  // NBUF keeps every waiter within one phase of the barrier it polls.
  constexpr int NBUF = C::NBUF;
  constexpr int NMD = STAGES + NBUF;
  uint64_t* full = bars;
  uint64_t* mdone = bars + STAGES;
  uint64_t* tempty = mdone + NMD;
  uint64_t* done = tempty + NBUF;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int KB = p.kblocks;
  // dispatch overlap: launched as a programmatic dependent of the route
  // kernel, whose tile list and counts it needs from the start
  if constexpr (DISP) griddep_wait();
  const int num_tiles = *p.num_tiles;
  const int rows_e = (KIND == 1) ? 2 * p.I : p.H;      // weight rows per expert
  constexpr int CT = (KIND == 1) ? NA / 2 : NA;        // 128-channel output tiles per unit
  const int NRT = ((KIND == 1) ? p.I : p.H) / 128 / CT;  // units per expert and token tile
  const int RB = rows_e / 128;                          // 128-row scale blocks per expert
  const int total = num_tiles * NRT;
  // 128-row block (within the expert) of weight tile a of unit row index rt:
  // GEMM1 tile 2c = gate, 2c + 1 = up of output tile rt * CT + c.
  auto tile_rb = [&](int rt, int a) {
    return (KIND == 1) ? (a & 1) * (p.I / 128) + rt * CT + (a >> 1) : rt * CT + a;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) mbar_init(&full[s], 1);
    for (int i = 0; i < NMD; ++i) mbar_init(&mdone[i], 1);
    for (int b = 0; b < NBUF; ++b) mbar_init(&tempty[b], C::EPI_THREADS);
    mbar_init(done, C::NMMA);
    *abort = 0;
    mbar_fence_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_map(&tmA);
    tma_prefetch_map(&tmB);
    if constexpr (P4) tma_prefetch_map(&tmS);
  }
  if (warp == C::MMA_WARP) {
    tmem_alloc(tmem_holder, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  // The next kernel may be scheduled as soon as SMs free up; it waits for this
  // grid's completion before it reads anything this grid writes.
  griddep_launch_dependents();

  if constexpr (WFMT == 1) {
    // B-side scale factors: all 1.0 (E8M0 127); the activation scales are
    // promoted in the epilogue instead.
    if (warp >= C::EPI_WARP0 && warp < C::EPI_WARP0 + 4) {
      const uint32_t q = warp & 3;
      tmem_st4(tmem + ((q * 32) << 16) + C::SFB_COL, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu);
      tmem_wait_st();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }

  if (warp < C::NPROD) {
    // ---------------- TMA producers ----------------
    // Producer warp pr fills the stages of the pipeline iterations it (one per
    // (unit, K block)) with it % NPROD == pr: stage it % STAGES, phase
    // (it / STAGES) & 1; the MMA warps consume the iterations in order.  One
    // issuing thread moves only ~47 GB/s through TMA, so within a warp the
    // loads of an iteration are split over lanes: lane 0 the gate (GEMM2: the
    // only) weight tile [+ its E8M0 atom], lane 1 the GEMM1 up tile [+ atom],
    // lane NJ-1 the token tile.  Lane 0 waits for the stage and posts the
    // transaction bytes before any lane issues.
    constexpr int NJ = NA + 1;
    const int pr = warp;
    const uint64_t pol_w = policy_evict_first();
    const uint64_t pol_a = policy_evict_last();
    const bool tok_lane = (lane == NJ - 1);
    uint32_t issued = 0, last_par = 0;  // lane 0: per-stage bitmasks for the abort drain
    bool ok = true;
    // The weights (and the tile list, written before the previous kernel
    // started) do not depend on the previous kernel: the first ring pass of
    // weight tiles is issued before waiting for it; the token tiles of that
    // pass follow once the previous kernel's output is visible.
    bool waited = false;
    constexpr int NPEND = (STAGES + C::NPROD - 1) / C::NPROD;
    int npend = 0;
    int pend_kb[NPEND], pend_p0[NPEND], pend_st[NPEND];
    // Dispatch overlap: the kernel follows the route kernel in plain stream
    // order, and a token tile is loaded once its group's ready counter is
    // complete (the load is issued even after that wait ran out, so that
    // the stage completes and the pipeline drains; the call then reports
    // MOE_ERR_TIMEOUT).
    constexpr int NPD = DISP ? NPEND : 1;
    int pend_e[NPD], pend_ti[NPD];
    int ready_ti = -1;  // token lane: the last tile whose group was seen ready
    auto tokens_ready = [&](int e, int ti) {
      if constexpr (DISP) {
        if (ti != ready_ti) {
          dispatch_ready(p, e, abort);
          ready_ti = ti;
        }
      }
    };
    // token tile of K block kb at positions p0.. (NVFP4: plus the block-code
    // atoms of its two MMA steps, rows ks * scale_ld + p0 .. + 31)
    auto load_tokens = [&](int st, int kb, int p0) {
      tma_load_2d(&tmB, &full[st], sB + st * C::B_BYTES, kb * C::KBYTES, p0, pol_a);
      if constexpr (NV) {
        uint8_t* dst = sSF + st * C::SF_BYTES + NA * C::SFA_BYTES;
        tma_load_2d(&tmS, &full[st], dst, 0, (2 * kb) * p.scale_ld + p0, pol_a);
        tma_load_2d(&tmS, &full[st], dst + 512, 0, (2 * kb + 1) * p.scale_ld + p0, pol_a);
      }
      if constexpr (MXA)
        tma_load_2d(&tmS, &full[st], sSF + st * C::SF_BYTES + NA * C::SFA_BYTES, 0, kb * p.scale_ld + p0, pol_a);
    };
    int it = 0;
    for (int u = blockIdx.x; u < total; u += gridDim.x) {
      const int rt = C::TILE_MAJOR ? u % NRT : u / num_tiles, ti = C::TILE_MAJOR ? u / NRT : u % num_tiles;
      const int4 tile = p.tiles[ti];
      const int e = tile.x, p0 = tile.y;
      const int row = e * rows_e + tile_rb(rt, lane < NA ? lane : 0) * 128;  // this lane's weight tile
      for (int kb = 0; kb < KB; ++kb, ++it) {
        if (it % C::NPROD != pr) continue;
        const int stage = it % STAGES;
        const uint32_t phase = (uint32_t)(it / STAGES) & 1u;
        if (tok_lane && !waited && it >= STAGES) {
          griddep_wait();
          for (int i = 0; i < npend; ++i) {
            if constexpr (DISP) tokens_ready(pend_e[i], pend_ti[i]);
            load_tokens(pend_st[i], pend_kb[i], pend_p0[i]);
          }
          waited = true;
        }
        if (lane == 0 && ok && it >= STAGES) {  // the stage's previous iteration has been consumed
          const int prev = it - STAGES;
          ok = mbar_wait(&mdone[prev % NMD], (uint32_t)(prev / NMD) & 1u, abort);
        }
        ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
        if (ok) {
          if (lane == 0) {
            // Failure-injection hook: CTA 0's first stage expects 16 bytes that
            // never arrive, so the MMA warp's bounded wait runs out (the load
            // itself completes; nothing is left in flight).
            const uint32_t extra = (p.inject == 1 && KIND == 1 && it == 0 && blockIdx.x == 0) ? 16u : 0u;
            mbar_arrive_expect_tx(&full[stage], C::TX_BYTES + extra);
            issued |= 1u << stage;
            last_par = (last_par & ~(1u << stage)) | (phase << stage);
          }
          __syncwarp();
          if (lane < NJ - 1) {
            tma_load_2d(&tmA, &full[stage], sA + (stage * NA + lane) * C::A_BYTES, kb * C::KBYTES, row, pol_w);
            if constexpr (WFMT == 1 || P4) {
              // the K block's block-scale atoms of these 128 rows (packed layout)
              const uint8_t* sf = reinterpret_cast<const uint8_t*>(p.wscale);
              bulk_load(sSF + stage * C::SF_BYTES + lane * C::SFA_BYTES,
                        sf + ((size_t)(row / 128) * KB + kb) * C::SFA_BYTES, C::SFA_BYTES, &full[stage], pol_w);
            }
          } else if (tok_lane) {
            if (waited) {
              tokens_ready(e, ti);
              load_tokens(stage, kb, p0);
            } else {
              pend_kb[npend] = kb;
              pend_p0[npend] = p0;
              pend_st[npend] = stage;
              if constexpr (DISP) {
                pend_e[npend] = e;
                pend_ti[npend] = ti;
              }
              ++npend;
            }
          }
        }
      }
    }
    if (tok_lane && !waited) {
      griddep_wait();
      for (int i = 0; i < npend; ++i) {
        if constexpr (DISP) tokens_ready(pend_e[i], pend_ti[i]);
        load_tokens(pend_st[i], pend_kb[i], pend_p0[i]);
      }
    }
    // Without an abort every issued load was consumed by the MMA warps.  After
    // one, wait (bounded) for this warp's last loads into each stage; a later
    // phase issued by another producer warp only shortens that wait.
    __syncwarp();
    if (lane == 0 && *abort)
      for (int s = 0; s < STAGES; ++s)
        if (issued & (1u << s)) drain_wait(&full[s], (last_par >> s) & 1u);
  } else if (warp < C::MMA_WARP + C::NMMA) {
    // ---------------- MMA issuers ----------------
    constexpr int AF = (WFMT == 1) ? 5 : 0;  // E2M1 : E4M3
    const int mw = warp - C::MMA_WARP;
    bool ok = true;
    int mit = 0;  // pipeline iteration
    for (int u = blockIdx.x; u < total; u += gridDim.x) {
      for (int kb = 0; kb < KB; ++kb, ++mit) {
        if (mit % C::NMMA != mw) continue;
        const int stage = mit % STAGES, buf = mit % NBUF;
        const uint32_t phase = (uint32_t)(mit / STAGES) & 1u, tphase = (uint32_t)(mit / NBUF) & 1u;
        if (ok) ok = mbar_wait(&tempty[buf], tphase ^ 1u, abort);
        if (ok) ok = mbar_wait(&full[stage], phase, abort);
        ok = __all_sync(0xFFFFFFFFu, ok);
        if (ok) {
          tc_fence_after();
          if (lane == 0) {
            const uint32_t d0 = tmem + buf * (NA * BN);
            const uint64_t ad = P4 ? sdesc_k_sw64(smem_u32(sA + stage * NA * C::A_BYTES))
                                   : sdesc_k_sw128(smem_u32(sA + stage * NA * C::A_BYTES));
            const uint64_t bd = P4 ? sdesc_k_sw64(smem_u32(sB + stage * C::B_BYTES))
                                   : sdesc_k_sw128(smem_u32(sB + stage * C::B_BYTES));
            constexpr uint32_t ATILE = C::A_BYTES >> 4;  // descriptor step between weight tiles
            if constexpr (NV) {
              // Scale atoms of this K block, smem -> TMEM (columns of buffer
              // buf): per weight tile a, atoms of K steps 0 and 1 at sfa + 8a
              // and sfa + 8a + 4; the token atoms at sfb and sfb + 4.
              const uint32_t sfa = tmem + C::SFA_COL + buf * C::SFA_PER_BUF;
              const uint32_t sfb = tmem + C::SFB_COL + buf * C::SFB_PER_BUF;
              uint8_t* sfs = sSF + stage * C::SF_BYTES;
              auto cp_atom = [&](uint32_t taddr, const uint8_t* src) {
                uint64_t sd = 0;
                sd |= static_cast<uint64_t>((smem_u32(src) & 0x3FFFFu) >> 4);
                sd |= static_cast<uint64_t>(128 >> 4) << 32;  // 8 rows x 16 bytes per core group
                sd |= static_cast<uint64_t>(1) << 46;
                tmem_cp_32x128b_warpx4(taddr, sd);
              };
#pragma unroll
              for (int a = 0; a < NA; ++a) {
                cp_atom(sfa + a * 8, sfs + a * 1024);
                cp_atom(sfa + a * 8 + 4, sfs + a * 1024 + 512);
              }
              cp_atom(sfb, sfs + NA * 1024);
              cp_atom(sfb + 4, sfs + NA * 1024 + 512);
              constexpr uint32_t idesc = idesc_mxf4nvf4(128, BN);
#pragma unroll
              for (int ks = 0; ks < 2; ++ks)
#pragma unroll
                for (int a = 0; a < NA; ++a)
                  mma_mxf4nvf4(d0 + a * BN, ad + a * ATILE + 2 * ks, bd + 2 * ks, idesc, sfa + a * 8 + ks * 4,
                               sfb + ks * 4, ks > 0);
            } else if constexpr (MXA) {
              // scale atoms of this K block, smem -> TMEM: weight tile a at
              // sfa + 4a, the token tile at sfb; K step ks uses scale bytes
              // 2ks and 2ks + 1 of each row's column (scale id 2ks)
              const uint32_t sfa = tmem + C::SFA_COL + buf * C::SFA_PER_BUF;
              const uint32_t sfb = tmem + C::SFB_COL + buf * C::SFB_PER_BUF;
              uint8_t* sfs = sSF + stage * C::SF_BYTES;
              auto cp_atom = [&](uint32_t taddr, const uint8_t* src) {
                uint64_t sd = 0;
                sd |= static_cast<uint64_t>((smem_u32(src) & 0x3FFFFu) >> 4);
                sd |= static_cast<uint64_t>(128 >> 4) << 32;  // 8 rows x 16 bytes per core group
                sd |= static_cast<uint64_t>(1) << 46;
                tmem_cp_32x128b_warpx4(taddr, sd);
              };
#pragma unroll
              for (int a = 0; a < NA; ++a) cp_atom(sfa + a * 4, sfs + a * 512);
              cp_atom(sfb, sfs + NA * 512);
#pragma unroll
              for (int ks = 0; ks < 2; ++ks) {
                const uint32_t idesc = idesc_mxf4(128, BN, 2 * ks, 2 * ks);
#pragma unroll
                for (int a = 0; a < NA; ++a)
                  mma_mxf4(d0 + a * BN, ad + a * ATILE + 2 * ks, bd + 2 * ks, idesc, sfa + a * 4, sfb, ks > 0);
              }
            } else if constexpr (WFMT == 0) {
              constexpr uint32_t idesc = idesc_f8f6f4(128, BN, AF, 0);
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
#pragma unroll
                for (int a = 0; a < NA; ++a) mma_f8f6f4(d0 + a * BN, ad + a * ATILE + 2 * kk, bd + 2 * kk, idesc, kk > 0);
            } else {
              // scale factors of this K block: smem atoms -> TMEM (parity buf)
              const uint32_t sfa = tmem + C::SFA_COL + buf * (NA * 4);  // per accumulator buffer
              const uint32_t sfb = tmem + C::SFB_COL;
              uint8_t* sfs = sSF + stage * C::SF_BYTES;
#pragma unroll
              for (int a = 0; a < NA; ++a) {
                uint64_t sd = 0;
                sd |= static_cast<uint64_t>((smem_u32(sfs + a * 512) & 0x3FFFFu) >> 4);
                sd |= static_cast<uint64_t>(128 >> 4) << 32;  // 8 rows x 16 bytes per core group
                sd |= static_cast<uint64_t>(1) << 46;
                tmem_cp_32x128b_warpx4(sfa + a * 4, sd);
              }
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint32_t idesc = idesc_mxf8f6f4(128, BN, AF, 0, kk, 0);
#pragma unroll
                for (int a = 0; a < NA; ++a)
                  mma_mxf8f6f4(d0 + a * BN, ad + a * ATILE + 2 * kk, bd + 2 * kk, idesc, sfa + a * 4, sfb, kk > 0);
              }
            }
            mma_commit(&mdone[mit % NMD]);
          }
          __syncwarp();
        }
      }
    }
    if (lane == 0) mma_commit(done);
    __syncwarp();
    drain_wait(done, 0);
  } else if (warp >= C::EPI_WARP0) {
    // ---------------- epilogue ----------------
    const int ew = warp - C::EPI_WARP0;
    const int q = warp & 3;        // TMEM lane quarter this warp may access
    const int cg = ew >> 2;        // column group
    const int row = q * 32 + lane; // weight row within the tile = TMEM lane
    const int etid = threadIdx.x - 32 * C::EPI_WARP0;
    const int S = p.S;
    int buf = 0;
    uint32_t tphase = 0;
    bool ok = true;
    int eit = 0;  // pipeline iteration
    auto unit_rt = [&](int uu) { return C::TILE_MAJOR ? uu % NRT : uu / num_tiles; };
    auto unit_ti = [&](int uu) { return C::TILE_MAJOR ? uu / NRT : uu % num_tiles; };
    // Inputs of unit u that do not come from the previous kernel: the weight
    // block scales (NVFP4: the expert's global scale) and, in GEMM2, the
    // combine target of every column (route outputs and the top-k weights).
    auto load_static = [&](int u, const int4& tile) {
      const int e = tile.x, p0 = tile.y, nv = tile.z, rt = unit_rt(u);
      (void)e; (void)p0; (void)nv; (void)rt;
      if constexpr (WFMT == 0) {
        for (int i = etid; i < NA * KB; i += C::EPI_THREADS) {
          const int a = i / KB, kb = i % KB;
          wsc[a * KB_MAX + kb] = p.wscale[((size_t)e * RB + tile_rb(rt, a)) * KB + kb];
        }
      }
      if constexpr (NV) {
        if (etid == 0) wsc[0] = p.wglobal[e];
      }
      if constexpr (KIND == 2) {
        for (int j = etid; j < BN; j += C::EPI_THREADS) {
          int tok = 0;
          float w = 0.0f;
          if (j < nv) {
            const int slot = p.perm[p0 + j];
            tok = (slot < S) ? slot / p.k : slot - S;
            w = (slot < S) ? p.topk_w[slot] : 1.0f;
          }
          slot_tok[j] = tok;
          slot_w[j] = w;
        }
      }
    };
    // The first unit's are read before waiting for the previous kernel (the
    // memory system is still quiet then), so that after the wait only its
    // activation scales remain to be read.
    const int u0 = blockIdx.x;
    int4 tile0 = make_int4(0, 0, 0, 0);
    if (u0 < total) {
      tile0 = p.tiles[unit_ti(u0)];
      load_static(u0, tile0);
    }
    griddep_wait();  // activation scales / combine buffer come from earlier kernels
    if constexpr (DISP) {
      // dispatch overlap: the last p.disp CTAs' epilogue warps quantise first
      const int dc = blockIdx.x - (int)(gridDim.x - p.disp);
      if (dc >= 0) dispatch_quant_fp8(p, dc * (C::EPI_THREADS / 32) + ew, p.disp * (C::EPI_THREADS / 32));
    }
    // Per-unit inputs of the epilogue: the activation scales of the tile's
    // columns [KB][BN], the weight block scales [NA][KB] and (GEMM2) the
    // combine target of every column.  In GEMM1 with tiles of up to 32 tokens
    // the next unit's tile record and scales are loaded into registers during
    // the current unit's K loop (record at K block 0, scales at K block 1), so
    // a unit starts without waiting on memory.  (Doing the same in GEMM2,
    // routing slot and combine weight included, made it slower.)
    constexpr bool PREF = BN <= 32 && KIND == 1 && !DISP;  // (dispatch overlap: scales read after the ready wait)
    constexpr int NPA = PREF ? (BN * KB_MAX + C::EPI_THREADS - 1) / C::EPI_THREADS : 1;
    int4 tile_n = make_int4(0, 0, 0, 0);
    float pa[NPA];
    float pw = 0.0f;
    bool have_next = false;
    auto pref_tile = [&](int un) {
      have_next = PREF && un < total;
      if (have_next) tile_n = p.tiles[unit_ti(un)];
    };
    auto pref_scales = [&](int un) {
      if (!have_next) return;
      const int rtn = unit_rt(un);
      (void)rtn;
      if constexpr (!MXA) {
#pragma unroll
        for (int r = 0; r < NPA; ++r) {
          const int i = etid + r * C::EPI_THREADS;
          pa[r] = (i < BN * KB) ? p.ascale[(size_t)(i / BN) * p.scale_ld + tile_n.y + (i % BN)] : 0.0f;
        }
      }
      if constexpr (WFMT == 0) {
        if (etid < NA * KB) {
          const int a = etid / KB, kb = etid % KB;
          pw = p.wscale[((size_t)tile_n.x * RB + tile_rb(rtn, a)) * KB + kb];
        }
      }
      if constexpr (NV) {
        if (etid == 0) pw = p.wglobal[tile_n.x];
      }
    };
    bool from_regs = false;
    if constexpr (PREF) {
      // the first unit's activation scales, all loads in flight together
      if (u0 < total) {
        tile_n = tile0;
        if constexpr (!MXA) {
#pragma unroll
          for (int r = 0; r < NPA; ++r) {
            const int i = etid + r * C::EPI_THREADS;
            pa[r] = (i < BN * KB) ? p.ascale[(size_t)(i / BN) * p.scale_ld + tile0.y + (i % BN)] : 0.0f;
          }
        }
        from_regs = true;
      }
    }
    for (int u = blockIdx.x; u < total; u += gridDim.x) {
      const int rt = unit_rt(u), ti = unit_ti(u);
      const int4 tile = from_regs ? tile_n : p.tiles[ti];  // (the first unit's: a cache hit)
      const int e = tile.x, p0 = tile.y, nv = tile.z;
      if constexpr (DISP) {
        if (ok) ok = dispatch_ready(p, e, abort);
      }
      if (from_regs) {
        if constexpr (!MXA) {
#pragma unroll
          for (int r = 0; r < NPA; ++r) {
            const int i = etid + r * C::EPI_THREADS;
            if (i < BN * KB) asc[i] = pa[r];
          }
        }
        if (u != u0) {  // the first unit's came from load_static
          if constexpr (WFMT == 0) {
            if (etid < NA * KB) wsc[(etid / KB) * KB_MAX + etid % KB] = pw;
          }
          if constexpr (NV) {
            if (etid == 0) wsc[0] = pw;
          }
        }
      } else {
        if constexpr (!MXA) {
          // four loads in flight per thread and round
          for (int i0 = etid; i0 < BN * KB; i0 += 4 * C::EPI_THREADS) {
            float v[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) {
              const int i = i0 + r * C::EPI_THREADS;
              v[r] = (i < BN * KB) ? p.ascale[(size_t)(i / BN) * p.scale_ld + p0 + (i % BN)] : 0.0f;
            }
#pragma unroll
            for (int r = 0; r < 4; ++r) {
              const int i = i0 + r * C::EPI_THREADS;
              if (i < BN * KB) asc[i] = v[r];
            }
          }
        }
        if (u != u0) load_static(u, tile);
      }
      named_sync(1, C::EPI_THREADS);
      const int un = u + gridDim.x;

      float acc[NA][CPT];  // one fp32 accumulator row per weight tile
#pragma unroll
      for (int a = 0; a < NA; ++a)
#pragma unroll
        for (int c = 0; c < CPT; ++c) acc[a][c] = 0.0f;
      // Combined scale of K block kb per tile column, shared by all 128 rows:
      // cs[kb & 1][a][j] = activation scale (column j, kb) x weight block
      // scale (tile a, kb) (MXFP4: the activation scale alone; NVFP4: x the
      // expert's global scale).  Filled one K block ahead by the epilogue
      // threads, one named barrier per K block.
      auto fill_cs = [&](int kb) {
        float* dst = cs + (kb & 1) * (NA * BN);
        for (int i = etid; i < NA * BN; i += C::EPI_THREADS) {
          const int a = i / BN, j = i - (i / BN) * BN;
          dst[i] = (WFMT == 0) ? asc[kb * BN + j] * wsc[a * KB_MAX + kb]
                   : NV        ? asc[kb * BN + j] * wsc[0]
                   : MXA       ? 1.0f  // every scale was applied by the MMA
                               : asc[kb * BN + j];
        }
      };
      fill_cs(0);
      named_sync(1, C::EPI_THREADS);
      for (int kb = 0; kb < KB; ++kb, ++eit) {
        if (kb + 1 < KB) fill_cs(kb + 1);
        if (kb == 0) pref_tile(un);
        if (kb == (KB > 1 ? 1 : 0)) pref_scales(un);
        if (ok) ok = mbar_wait(&mdone[eit % NMD], (uint32_t)(eit / NMD) & 1u, abort);
        ok = __all_sync(0xFFFFFFFFu, ok);
        if (ok) {
          tc_fence_after();
          const uint32_t tb = tmem + ((uint32_t)(q * 32) << 16) + buf * (NA * BN) + cg * CPT;
          const float* csb = cs + (kb & 1) * (NA * BN) + cg * CPT;
          // acc += D_kb * combined scale, two columns per paired fp32 FMA
          if constexpr (KIND == 1 && CPT >= 64) {
            // wide tiles (one gate/up pair): gate and up chunks one after the
            // other, so only 16 loaded values are live next to the 2 x CPT
            // accumulators
            static_assert(NA == 2, "wide tiles use one gate/up pair");
#pragma unroll
            for (int c0 = 0; c0 < 2 * CPT; c0 += 16) {
              float d[16];
              const int a = c0 >= CPT ? 1 : 0;
              const int cc = c0 - a * CPT;
              tmem_ld16(tb + a * BN + cc, d);
              tmem_wait_ld();
              if (c0 + 16 >= 2 * CPT) {
                tc_fence_before();
                mbar_arrive(&tempty[buf]);
              }
              const float2* s2 = reinterpret_cast<const float2*>(csb + a * BN + cc);
              float2* a2 = reinterpret_cast<float2*>(&acc[a][cc]);
#pragma unroll
              for (int i = 0; i < 8; ++i) a2[i] = __ffma2_rn(make_float2(d[2 * i], d[2 * i + 1]), s2[i], a2[i]);
            }
          } else {
            constexpr int LD = CPT >= 16 ? 16 : 8;  // columns per TMEM load
#pragma unroll
            for (int c0 = 0; c0 < CPT; c0 += LD) {
              float d[NA][LD];
#pragma unroll
              for (int a = 0; a < NA; ++a) {
                if constexpr (LD == 16) tmem_ld16(tb + a * BN + c0, d[a]);
                else tmem_ld8(tb + a * BN + c0, d[a]);
              }
              tmem_wait_ld();
              if (c0 + LD >= CPT) {
                tc_fence_before();
                mbar_arrive(&tempty[buf]);
              }
#pragma unroll
              for (int a = 0; a < NA; ++a) {
                const float2* s2 = reinterpret_cast<const float2*>(csb + a * BN + c0);
                float2* a2 = reinterpret_cast<float2*>(&acc[a][c0]);
#pragma unroll
                for (int i = 0; i < LD / 2; ++i)
                  a2[i] = __ffma2_rn(make_float2(d[a][2 * i], d[a][2 * i + 1]), s2[i], a2[i]);
              }
            }
          }
        }
        named_sync(1, C::EPI_THREADS);  // cs slot kb+1 written, slot kb consumed
        if (++buf == NBUF) {
          buf = 0;
          tphase ^= 1u;
        }
      }

      if constexpr (KIND == 1) {
        // Per gate/up pair (gate rows 0..I-1 of W13, up rows I..2I-1: same
        // channels): SwiGLU, then requantisation per token over the output
        // tile's 128 channels -- FP8, NVFP4 (the rule of quant_nvfp4_kernel:
        // lanes 16i .. 16i+15 of a warp hold one 16-channel block, the four
        // warps one 128 group) or MXFP4 (the rule of quant_mxfp4_kernel: a
        // 32-channel block is one warp).  h overwrites the gate accumulator.
        //
        // The columns are taken CH at a time in rolled loops, and the
        // register arrays rotate left by CH per step (static indices keep
        // them in registers).  Fully unrolled, this tail is tens of KB of
        // code per kernel, and the first unit of every launch then waits on
        // instruction fetches from a memory system that the weight stream
        // keeps saturated.
        // (CH chosen per shape to keep the tail free of register spills:
        // NVFP4 at 32 columns stays unrolled)
        constexpr int CH = CPT <= 8 ? CPT : CPT >= 64 ? 8 : CPT < 32 ? 2 : NV ? CPT : WFMT == 1 ? 8 : 4;
#pragma unroll
        for (int pr = 0; pr < NA / 2; ++pr) {
          float* h = acc[2 * pr];
          float* up = acc[2 * pr + 1];
          const int ct = rt * CT + pr;  // output channel tile
          const int ch = ct * 128 + row;
          if constexpr (MXA) {
            // one pass: SwiGLU, the block's amax (a warp reduction), lane 0
            // writes the block's E8M0 code (byte q of the tile's entry)
#pragma unroll 1
            for (int c0 = 0; c0 < CPT; c0 += CH) {
#pragma unroll
              for (int i = 0; i < CH; ++i) {
                const int j = cg * CPT + c0 + i;
                const float g = h[i];
                const float sig = __fdiv_rn(1.0f, 1.0f + expf(-g));
                const float hv = g * sig * up[i];
                float m = fabsf(hv);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
                float sc;
                const int X = mx_e2m1_exponent(m, &sc);
                const uint32_t nib = f32_to_e2m1(__fdiv_rn(hv, sc));
                uint32_t word = nib << (4 * (lane & 7));
                word |= __shfl_xor_sync(0xFFFFFFFFu, word, 1);
                word |= __shfl_xor_sync(0xFFFFFFFFu, word, 2);
                word |= __shfl_xor_sync(0xFFFFFFFFu, word, 4);
                if (ok && j < nv) {
                  if ((lane & 7) == 0)
                    *reinterpret_cast<uint32_t*>(p.hq + (size_t)(p0 + j) * (p.I / 2) + ch / 2) = word;
                  if (lane == 0)
                    p.hsc[((size_t)ct * p.scale_ld + p0 + j) * 16 + q] = static_cast<uint8_t>(X + 127);
                }
              }
              rotl<CPT, CH>(h);
              rotl<CPT, CH>(up);
            }
          } else {
            // pass 1: SwiGLU and the per-quarter amax of each column; h takes
            // the SwiGLU outputs and (NVFP4) up the 16-channel block amaxes
#pragma unroll 1
            for (int c0 = 0; c0 < CPT; c0 += CH) {
              float hv[CH], bv[CH];
#pragma unroll
              for (int i = 0; i < CH; ++i) {
                const float g = h[i];
                const float sig = __fdiv_rn(1.0f, 1.0f + expf(-g));
                hv[i] = g * sig * up[i];
                float m = fabsf(hv[i]);
#pragma unroll
                for (int o = 8; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
                bv[i] = m;
                m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 16));
                if (lane == 0) red[q * BN + cg * CPT + c0 + i] = m;
              }
              rotl<CPT, CH>(h);
              rotl<CPT, CH>(up);
#pragma unroll
              for (int i = 0; i < CH; ++i) {
                h[CPT - CH + i] = hv[i];
                up[CPT - CH + i] = bv[i];
              }
            }
            const float* a16 = up;
            named_sync(1, C::EPI_THREADS);
            // pass 2: the per-token scale of the 128 channels, the codes
            if (ok) {
#pragma unroll 1
              for (int c0 = 0; c0 < CPT; c0 += CH) {
#pragma unroll
                for (int i = 0; i < CH; ++i) {
                  const int j = cg * CPT + c0 + i;
                  const float amax = fmaxf(fmaxf(red[j], red[BN + j]), fmaxf(red[2 * BN + j], red[3 * BN + j]));
                  if constexpr (NV) {
                    const float sg = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 2688.0f);
                    const uint32_t code = f32_to_e4m3(__fdiv_rn(__fdiv_rn(a16[i], 6.0f), sg));
                    const float d = __fmul_rn(e4m3_code_value(code), sg);
                    const uint32_t nib = code ? f32_to_e2m1(__fdiv_rn(h[i], d)) : 0u;
                    // eight neighbouring channels -> one 32-bit word of packed codes
                    uint32_t word = nib << (4 * (lane & 7));
                    word |= __shfl_xor_sync(0xFFFFFFFFu, word, 1);
                    word |= __shfl_xor_sync(0xFFFFFFFFu, word, 2);
                    word |= __shfl_xor_sync(0xFFFFFFFFu, word, 4);
                    if (j < nv) {
                      if ((lane & 7) == 0)
                        *reinterpret_cast<uint32_t*>(p.hq + (size_t)(p0 + j) * (p.I / 2) + ch / 2) = word;
                      if ((lane & 15) == 0)
                        p.hsc[((size_t)(ch / 64) * p.scale_ld + p0 + j) * 16 + (ch / 16) % 4] =
                            static_cast<uint8_t>(code);
                      if (row == 0) p.hs[(size_t)ct * p.scale_ld + p0 + j] = sg;
                    }
                  } else {
                    const float sc = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 448.0f);
                    if (j < nv) {
                      p.hq[(size_t)(p0 + j) * p.I + ch] = static_cast<uint8_t>(f32_to_e4m3(__fdiv_rn(h[i], sc)));
                      if (row == 0) p.hs[(size_t)ct * p.scale_ld + p0 + j] = sc;
                    }
                  }
                }
                rotl<CPT, CH>(h);
                if constexpr (NV) rotl<CPT, CH>(up);
              }
            }
            if (pr + 1 < NA / 2) named_sync(1, C::EPI_THREADS);  // red is reused by the next pair
          }
        }
      } else {
        if (ok) {
#pragma unroll
          for (int a = 0; a < NA; ++a) {
            const int ch = (rt * CT + a) * 128 + row;
            if (p.y_rows) {
              // unfused combine: keep this position's expert output row
#pragma unroll
              for (int c = 0; c < CPT; ++c) {
                const int j = cg * CPT + c;
                if (j < nv) p.y_rows[(size_t)(p0 + j) * p.H + ch] = acc[a][c];
              }
            } else {
              // fused combine: out_acc[token] += w * y (fp32 reductions in L2)
#pragma unroll
              for (int c = 0; c < CPT; ++c) {
                const int j = cg * CPT + c;
                if (j < nv) atomicAdd(p.out_acc + (size_t)slot_tok[j] * p.H + ch, slot_w[j] * acc[a][c]);
              }
            }
          }
        }
      }
      named_sync(1, C::EPI_THREADS);
      from_regs = have_next;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
  if (threadIdx.x == 0 && *abort) atomicOr(p.status, DEV_TIMEOUT);
}

// ---------------------------------------------------------------------------
template <int KIND, int BN, int WFMT, int NT, bool DISP = false>
static cudaError_t set_attr() {
  using C = GemmCfg<KIND, BN, WFMT, NT>;
  return cudaFuncSetAttribute(moe_gemm_kernel<KIND, BN, WFMT, NT, DISP>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
}

template <int KIND, int BN, int WFMT, int NT = (KIND == 1 ? 2 : 1)>
static cudaError_t launch(int grid, const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& ts,
                          const GemmParams& p, cudaStream_t s) {
  using C = GemmCfg<KIND, BN, WFMT, NT>;
  constexpr bool CAN_DISP = KIND == 1 && WFMT <= 1;  // FP8 activations: the dispatch-overlap variant exists
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(C::THREADS);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  // dispatch overlap: CTAs wait for other CTAs' ready counters, so all of
  // them must be resident at once
  attr[1].id = cudaLaunchAttributeCooperative;
  attr[1].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = p.disp ? 2 : 1;
  if constexpr (CAN_DISP) {
    if (p.disp) return cudaLaunchKernelEx(&cfg, moe_gemm_kernel<KIND, BN, WFMT, NT, true>, ta, tb, ts, p);
  } else {
    if (p.disp) return cudaErrorInvalidValue;
  }
  return cudaLaunchKernelEx(&cfg, moe_gemm_kernel<KIND, BN, WFMT, NT, false>, ta, tb, ts, p);
}

// Weight tiles per stage with 4-bit weights: a stage of one or two 128-row
// tiles carries only 8-16 KB of weights, and per stage the tensor pipe also
// copies the block-scale atoms and commits, which at that size issues slower
// than HBM delivers.  16-token tiles therefore take four tiles per stage
// (32 KB) where the channel count divides: GEMM1 two gate/up pairs
// (I % 256 == 0; 4-bit activations only -- MXFP4 weights with FP8
// activations measured faster with one pair, whose padded tiles leave room
// for twice the stages), GEMM2 four output tiles (H % 512 == 0), else two
// (H % 256 == 0), else one.
static int fp4_tiles(int kind, int BN, const GemmParams& p) {
  if (kind == 1) return (BN == 16 && p.I % 256 == 0) ? 4 : 2;
  if (BN == 16 && p.H % 512 == 0) return 4;
  return (p.H % 256 == 0) ? 2 : 1;
}

cudaError_t gemm_setup(int wfmt) {
  cudaError_t e = cudaSuccess;
#define MOE_SET(K, B, W) \
  if (e == cudaSuccess) e = set_attr<K, B, W, (K == 1 ? 2 : 1)>();
#define MOE_SET_DISP(B, W) \
  if (e == cudaSuccess) e = set_attr<1, B, W, 2, true>();
#define MOE_SET_NT(K, B, W, N) \
  if (e == cudaSuccess) e = set_attr<K, B, W, N>();
  if (wfmt == 0) {
    MOE_SET(1, 16, 0) MOE_SET(1, 32, 0) MOE_SET(1, 64, 0)
    MOE_SET_DISP(16, 0) MOE_SET_DISP(32, 0) MOE_SET_DISP(64, 0)
    MOE_SET(2, 16, 0) MOE_SET(2, 32, 0) MOE_SET(2, 64, 0)
    MOE_SET_NT(2, 16, 0, 2) MOE_SET_NT(2, 32, 0, 2)
    if (e == cudaSuccess) e = gemm_tm_setup();
  } else if (wfmt == 1) {
    MOE_SET(1, 16, 1) MOE_SET(1, 32, 1) MOE_SET(1, 64, 1)
    MOE_SET_DISP(16, 1) MOE_SET_DISP(32, 1) MOE_SET_DISP(64, 1)
    MOE_SET_NT(2, 16, 1, 4) MOE_SET_NT(2, 16, 1, 2) MOE_SET(2, 16, 1)
    MOE_SET_NT(2, 32, 1, 2) MOE_SET(2, 32, 1) MOE_SET(2, 64, 1)
  } else if (wfmt == 2) {
    MOE_SET_NT(1, 16, 2, 4) MOE_SET_NT(1, 16, 2, 2) MOE_SET_NT(1, 32, 2, 2)
    MOE_SET_NT(2, 16, 2, 4) MOE_SET_NT(2, 16, 2, 2) MOE_SET_NT(2, 16, 2, 1)
    MOE_SET_NT(2, 32, 2, 2) MOE_SET_NT(2, 32, 2, 1)
  } else {
    MOE_SET_NT(1, 16, 3, 4) MOE_SET_NT(1, 16, 3, 2) MOE_SET_NT(1, 32, 3, 2)
    MOE_SET_NT(2, 16, 3, 4) MOE_SET_NT(2, 16, 3, 2) MOE_SET_NT(2, 16, 3, 1)
    MOE_SET_NT(2, 32, 3, 2) MOE_SET_NT(2, 32, 3, 1)
  }
#undef MOE_SET
#undef MOE_SET_DISP
#undef MOE_SET_NT
  return e;
}

cudaError_t launch_gemm1(int wfmt, int BN, int grid, const CUtensorMap& tw, const CUtensorMap& tx,
                         const CUtensorMap& tsf, const GemmParams& p, cudaStream_t s) {
  if (wfmt == 0) {
    switch (BN) {
      case 16: return launch<1, 16, 0>(grid, tw, tx, tsf, p, s);
      case 32: return launch<1, 32, 0>(grid, tw, tx, tsf, p, s);
      case 64: return launch<1, 64, 0>(grid, tw, tx, tsf, p, s);
      case 128: return launch_gemm1_tm(grid, tw, tx, p, s);
    }
  } else if (wfmt == 1) {
    switch (BN) {
      case 16: return launch<1, 16, 1>(grid, tw, tx, tsf, p, s);
      case 32: return launch<1, 32, 1>(grid, tw, tx, tsf, p, s);
      case 64: return launch<1, 64, 1>(grid, tw, tx, tsf, p, s);
    }
  } else if (wfmt == 2) {
    const int nt = fp4_tiles(1, BN, p);
    if (BN == 16) return nt == 4 ? launch<1, 16, 2, 4>(grid, tw, tx, tsf, p, s) : launch<1, 16, 2, 2>(grid, tw, tx, tsf, p, s);
    if (BN == 32) return launch<1, 32, 2, 2>(grid, tw, tx, tsf, p, s);
  } else {
    const int nt = fp4_tiles(1, BN, p);
    if (BN == 16) return nt == 4 ? launch<1, 16, 3, 4>(grid, tw, tx, tsf, p, s) : launch<1, 16, 3, 2>(grid, tw, tx, tsf, p, s);
    if (BN == 32) return launch<1, 32, 3, 2>(grid, tw, tx, tsf, p, s);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_gemm2(int wfmt, int BN, int grid, const CUtensorMap& tw, const CUtensorMap& th,
                         const CUtensorMap& tsf, const GemmParams& p, cudaStream_t s) {
  if (wfmt == 0) {
    // decode tiles: two 128-row W2 tiles per stage and unit (one token tile,
    // one commit and one unit prologue / combine per 256 output channels)
    const bool two = p.H % 256 == 0;
    switch (BN) {
      case 16: return two ? launch<2, 16, 0, 2>(grid, tw, th, tsf, p, s) : launch<2, 16, 0>(grid, tw, th, tsf, p, s);
      case 32: return two ? launch<2, 32, 0, 2>(grid, tw, th, tsf, p, s) : launch<2, 32, 0>(grid, tw, th, tsf, p, s);
      case 64: return launch<2, 64, 0>(grid, tw, th, tsf, p, s);
      case 128: return launch_gemm2_tm(grid, tw, th, p, s);
    }
  } else if (wfmt == 1) {
    const int nt = fp4_tiles(2, BN, p);
    switch (BN) {
      case 16:
        if (nt == 4) return launch<2, 16, 1, 4>(grid, tw, th, tsf, p, s);
        if (nt == 2) return launch<2, 16, 1, 2>(grid, tw, th, tsf, p, s);
        return launch<2, 16, 1>(grid, tw, th, tsf, p, s);
      case 32: return nt == 2 ? launch<2, 32, 1, 2>(grid, tw, th, tsf, p, s) : launch<2, 32, 1>(grid, tw, th, tsf, p, s);
      case 64: return launch<2, 64, 1>(grid, tw, th, tsf, p, s);
    }
  } else if (wfmt == 2) {
    const int nt = fp4_tiles(2, BN, p);
    if (BN == 16) {
      if (nt == 4) return launch<2, 16, 2, 4>(grid, tw, th, tsf, p, s);
      if (nt == 2) return launch<2, 16, 2, 2>(grid, tw, th, tsf, p, s);
      return launch<2, 16, 2, 1>(grid, tw, th, tsf, p, s);
    }
    if (BN == 32) return nt == 2 ? launch<2, 32, 2, 2>(grid, tw, th, tsf, p, s) : launch<2, 32, 2, 1>(grid, tw, th, tsf, p, s);
  } else {
    const int nt = fp4_tiles(2, BN, p);
    if (BN == 16) {
      if (nt == 4) return launch<2, 16, 3, 4>(grid, tw, th, tsf, p, s);
      if (nt == 2) return launch<2, 16, 3, 2>(grid, tw, th, tsf, p, s);
      return launch<2, 16, 3, 1>(grid, tw, th, tsf, p, s);
    }
    if (BN == 32) return nt == 2 ? launch<2, 32, 3, 2>(grid, tw, th, tsf, p, s) : launch<2, 32, 3, 1>(grid, tw, th, tsf, p, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace moe
