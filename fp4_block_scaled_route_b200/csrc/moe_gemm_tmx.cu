// moe_gemm_tmx.cu -- token-major grouped expert GEMMs for MXFP8 (E4M3 weights
// and activations, one E8M0 scale per 32 elements along K on both operands).
//
// The two GEMMs of the layer (GEMM1 + SwiGLU + requantisation, GEMM2 +
// weighted combine; GC-MoE abstract: block-scaled grouped GEMM with fused
// SwiGLU + requantisation; FusedDeepMoE page: GmmDeqSwigluQuant, GmmDeq with
// the combine as epilogue callback) with every scale a power of two, so the
// tensor cores apply them: tcgen05.mma kind::mxf8f6f4.block_scale, E8M0
// scales per 32 K on both sides (DeepGEMM 26/09 news page: Mega MoE's FP8
// layouts with power-of-two scales, in place of per-128-K promotion).  The
// fp32 accumulator of a unit therefore stays in TMEM for the whole K loop and
// is read out once, at the end of the unit.
//
// Operands as in moe_gemm_tm.cu:
//   M = 128 positions of one expert (A operand, TMEM lane = token),
//   N = 256 weight rows           (B operand): GEMM1 128 gate rows then the
//       matching 128 up rows, GEMM2 256 rows of W2 (128 for a trailing half).
// Scale factors: per stage the A operand's 512-byte atom of the tile and K
// block (written by quant_mxfp8_kernel / by GEMM1's tail for GEMM2) and one
// 512-byte atom per 128-row weight box (the packed E8M0 layout of
// moe_pack_mxfp4_scales), copied into TMEM by tcgen05.cp: row n of an
// operand at lane n % 32 (in every lane quarter), column n / 32, byte k =
// the k-th 32-wide K sub-block, which MMA step k selects by its scale id.
//
// Warp roles (one CTA per SM, persistent over the work units):
//   warps 0-1   TMA producers (pipeline iterations alternate between them;
//               lane 0 the token tile and its scale atom, lanes 1-2 the
//               weight boxes and their atoms)
//   warp 2      MMA issuer: all iterations in order, since consecutive K
//               blocks accumulate into one TMEM accumulator (allocates TMEM)
//   warp 3      idle
//   warps 4-11  epilogue, two warpgroups = two halves of the 256 columns:
//               once per unit, tcgen05.ld of the accumulator, then the tail.
#include <cuda_bf16.h>

#include "moe_internal.h"
#include "moe_mxfp8.cuh"
#include "moe_ptx.cuh"

namespace moe {

template <int KIND>
struct TmxCfg {
  static constexpr int BM = 128;                 // tokens per tile: MMA M = TMEM lanes
  static constexpr int BW = 256;                 // weight rows per unit: MMA N
  static constexpr int A_BYTES = BM * 128;       // token tile: 128 rows x 128 K bytes
  static constexpr int W_BOX = 128 * 128;        // one 128-row weight box
  static constexpr int SF_ATOM = 512;            // one scale atom (128 rows x 4 E8M0 codes)
  static constexpr int SF_BYTES = 3 * SF_ATOM;   // A atom + two weight atoms
  static constexpr int STAGE_BYTES = A_BYTES + 2 * W_BOX + SF_BYTES;
  static constexpr int STAGES = 4;
  static constexpr int NMD = STAGES + 1;         // MMA-done barrier ring (one MMA warp, in order)
  static constexpr int NPROD = 2;
  static constexpr int MMA_WARP = 2;
  static constexpr int EPI_WARP0 = 4;
  static constexpr int CG = 2;                   // epilogue warpgroups (column halves)
  static constexpr int EPI_THREADS = 128 * CG;
  static constexpr int THREADS = 32 * EPI_WARP0 + EPI_THREADS;
  static constexpr int CPT = BW / CG;            // accumulator columns per epilogue thread
  static constexpr int LAUNCH_REGS = 168;        // registers per thread at launch (launch bounds)
  static constexpr int REGS_LOW = 40;            // producer / MMA warpgroup after the split
  static constexpr int REGS_HIGH = 232;          // epilogue warpgroups after the split
  // TMEM: the accumulator (256 columns), then per stage a scale slot of 12
  // columns: the A atom (4) and the two weight atoms (8; B rows 128..255 in
  // the second four).  Every scale operand starts on a 4-column boundary.
  static constexpr int SF_COL = BW;
  static constexpr int SF_SLOT = 12;
  static constexpr int TMEM_COLS = 512;
  static constexpr int NBARS = STAGES + NMD + 1 + 1 + 1;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + NBARS * 8 + 16;
  // A producer's wait for the MMAs of it - STAGES is exact when its previous
  // iteration it - NPROD is no older than that.
  static_assert(STAGES >= NPROD, "a producer could pass a stale MMA-done phase");
  static_assert(SF_COL + STAGES * SF_SLOT <= TMEM_COLS, "TMEM");
  static_assert(128 * REGS_LOW + EPI_THREADS * REGS_HIGH <= THREADS * LAUNCH_REGS, "register split");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
  static_assert((A_BYTES + 2 * W_BOX) % 1024 == 0, "tile areas stay 1024-byte aligned (128-byte swizzle)");
};

// Bounded wait that ignores the abort word (drain of in-flight work).
__device__ __forceinline__ void tmx_drain_wait(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kWaitCycles) break;
  }
}

// Shared-memory descriptor of one 512-byte scale atom for tcgen05.cp
// .32x128b.warpx4 (8 rows x 16 bytes per core group, 128-byte stride).
__device__ __forceinline__ uint64_t sf_atom_desc(const void* src) {
  uint64_t sd = 0;
  sd |= static_cast<uint64_t>((smem_u32(src) & 0x3FFFFu) >> 4);
  sd |= static_cast<uint64_t>(128 >> 4) << 32;
  sd |= static_cast<uint64_t>(1) << 46;
  return sd;
}

template <int KIND>
__global__ void __launch_bounds__(TmxCfg<KIND>::THREADS, 1)
    moe_gemm_tmx_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                        const GemmParams p) {
  using C = TmxCfg<KIND>;
  constexpr int STAGES = C::STAGES, NMD = C::NMD;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // Stage s: token tile and weight boxes in the 1024-aligned tile area
  // (s * TILE_BYTES), scale atoms in a separate area after all stages.
  constexpr int TILE_BYTES = C::A_BYTES + 2 * C::W_BOX;
  uint8_t* sfs = smem + STAGES * TILE_BYTES;                                 // [STAGES][3][512]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sfs + STAGES * C::SF_BYTES);
  uint64_t* full = bars;             // [STAGES] TMA bytes landed
  uint64_t* mdone = full + STAGES;   // [NMD] MMAs of an iteration completed (the stage is free)
  // The accumulator of a unit is complete: a barrier of its own, one phase
  // per unit.  (Waiting on the ring barrier of the unit's last iteration
  // would be ambiguous: with more K blocks than ring slots that barrier's
  // wanted phase is not its next one, and a parity wait would pass on an
  // earlier phase.)  The MMA warp cannot complete the next unit's phase
  // before the epilogue has released the accumulator, so every wait on it
  // is exact.
  uint64_t* afull = mdone + NMD;
  uint64_t* tempty = afull + 1;      // the epilogue has read the accumulator
  uint64_t* done = tempty + 1;       // all MMAs of the CTA completed
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int KB = p.kblocks;
  const int num_tiles = *p.num_tiles;
  const int NRT = (KIND == 1) ? p.I / 128 : (p.H + 255) / 256;
  const int rows_e = (KIND == 1) ? 2 * p.I : p.H;   // weight rows per expert
  const int total = num_tiles * NRT;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) mbar_init(&full[s], 1);
    for (int i = 0; i < NMD; ++i) mbar_init(&mdone[i], 1);
    mbar_init(afull, 1);
    mbar_init(tempty, C::EPI_THREADS);
    mbar_init(done, 1);
    *abort = 0;
    mbar_fence_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_map(&tmW);
    tma_prefetch_map(&tmX);
  }
  if (warp == C::MMA_WARP) {
    tmem_alloc(tmem_holder, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  griddep_launch_dependents();

  auto weight_rows = [&](int rt) { return (KIND == 1) ? 256 : min(256, p.H - rt * 256); };
  const uint8_t* wsf = reinterpret_cast<const uint8_t*>(p.wscale);  // packed weight atoms [rows/128][KB][512]

  if (warp < C::EPI_WARP0) {
    regs_shrink<C::REGS_LOW>();
    if (warp < C::NPROD) {
      // ---------------- TMA producers ----------------
      const int pr = warp;
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_a = policy_evict_last();
      uint32_t issued = 0, last_par = 0;
      bool ok = true;
      // The weights and their scale atoms do not depend on the previous
      // kernel: the first ring pass of them is issued before waiting for it,
      // its token tiles and their atoms after.
      bool waited = false;
      constexpr int NPEND = (STAGES + C::NPROD - 1) / C::NPROD;
      int npend = 0;
      int pend_kb[NPEND], pend_p0[NPEND], pend_st[NPEND], pend_ti[NPEND];
      auto load_tokens = [&](int st, int kb, int p0, int ti) {
        tma_load_2d(&tmX, &full[st], smem + st * TILE_BYTES, kb * 128, p0, pol_a);
        bulk_load(sfs + st * C::SF_BYTES, p.act_sf + ((size_t)ti * KB + kb) * C::SF_ATOM, C::SF_ATOM, &full[st],
                  pol_a);
      };
      int it = 0;
      for (int u = blockIdx.x; u < total; u += gridDim.x) {
        const int ti = u / NRT, rt = u % NRT;
        const int4 tile = p.tiles[ti];
        const int e = tile.x, p0 = tile.y;
        const int nw = weight_rows(rt);
        // lane 1: first weight box (GEMM1 gate rows), lane 2: second (up rows)
        const int wrow = (KIND == 1) ? e * rows_e + (lane == 2 ? p.I : 0) + rt * 128
                                     : e * rows_e + rt * 256 + (lane == 2 ? 128 : 0);
        const bool w_lane = (lane == 1) || (lane == 2 && nw == 256);
        const uint32_t tx = C::A_BYTES + (uint32_t)nw * 128 + C::SF_ATOM * (1 + nw / 128);
        for (int kb = 0; kb < KB; ++kb, ++it) {
          if (it % C::NPROD != pr) continue;
          const int stage = it % STAGES;
          const uint32_t phase = (uint32_t)(it / STAGES) & 1u;
          if (lane == 0 && !waited && it >= STAGES) {
            griddep_wait();
            for (int i = 0; i < npend; ++i) load_tokens(pend_st[i], pend_kb[i], pend_p0[i], pend_ti[i]);
            waited = true;
          }
          if (lane == 0 && ok && it >= STAGES) {
            const int prev = it - STAGES;
            ok = mbar_wait(&mdone[prev % NMD], (uint32_t)(prev / NMD) & 1u, abort);
          }
          ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
          if (ok) {
            if (lane == 0) {
              mbar_arrive_expect_tx(&full[stage], tx);
              issued |= 1u << stage;
              last_par = (last_par & ~(1u << stage)) | (phase << stage);
            }
            __syncwarp();
            uint8_t* st = smem + stage * TILE_BYTES;
            if (w_lane) {
              const int box = lane - 1;
              tma_load_2d(&tmW, &full[stage], st + C::A_BYTES + box * C::W_BOX, kb * 128, wrow, pol_w);
              bulk_load(sfs + stage * C::SF_BYTES + (1 + box) * C::SF_ATOM,
                        wsf + ((size_t)(wrow / 128) * KB + kb) * C::SF_ATOM, C::SF_ATOM, &full[stage], pol_w);
            } else if (lane == 0) {
              if (waited) {
                load_tokens(stage, kb, p0, ti);
              } else {
                pend_kb[npend] = kb;
                pend_p0[npend] = p0;
                pend_st[npend] = stage;
                pend_ti[npend] = ti;
                ++npend;
              }
            }
          }
        }
      }
      if (lane == 0 && !waited) {
        griddep_wait();
        for (int i = 0; i < npend; ++i) load_tokens(pend_st[i], pend_kb[i], pend_p0[i], pend_ti[i]);
      }
      __syncwarp();
      if (lane == 0 && *abort)
        for (int s = 0; s < STAGES; ++s)
          if (issued & (1u << s)) tmx_drain_wait(&full[s], (last_par >> s) & 1u);
    } else if (warp == C::MMA_WARP) {
      // ---------------- MMA issuer ----------------
      // One warp issues every iteration in order: the K blocks of a unit
      // accumulate into the one accumulator.  Per iteration the stage's three
      // scale atoms are copied into its TMEM scale slot (free: the producer
      // refilled the stage only after the MMAs that read the slot last time
      // completed), then four K = 32 MMAs with scale ids 0..3.
      bool ok = true;
      int mit = 0, j = 0;  // pipeline iteration, unit count of this CTA
      for (int u = blockIdx.x; u < total; u += gridDim.x, ++j) {
        const int nw = weight_rows(u % NRT);
        for (int kb = 0; kb < KB; ++kb, ++mit) {
          const int stage = mit % STAGES;
          const uint32_t phase = (uint32_t)(mit / STAGES) & 1u;
          if (kb == 0 && ok) ok = mbar_wait(tempty, (uint32_t)(j & 1) ^ 1u, abort);  // accumulator read out
          if (ok) ok = mbar_wait(&full[stage], phase, abort);
          ok = __all_sync(0xFFFFFFFFu, ok);
          if (ok) {
            tc_fence_after();
            if (lane == 0) {
              const uint32_t sfa = tmem + C::SF_COL + stage * C::SF_SLOT;
              const uint32_t sfb = sfa + 4;
              const uint8_t* ss = sfs + stage * C::SF_BYTES;
              tmem_cp_32x128b_warpx4(sfa, sf_atom_desc(ss));
              tmem_cp_32x128b_warpx4(sfb, sf_atom_desc(ss + C::SF_ATOM));
              if (nw == 256) tmem_cp_32x128b_warpx4(sfb + 4, sf_atom_desc(ss + 2 * C::SF_ATOM));
              const uint64_t ad = sdesc_k_sw128(smem_u32(smem + stage * TILE_BYTES));
              const uint64_t bd = sdesc_k_sw128(smem_u32(smem + stage * TILE_BYTES + C::A_BYTES));
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                mma_mxf8f6f4(tmem, ad + 2 * kk, bd + 2 * kk, idesc_mxf8f6f4(128, nw, 0, 0, kk, kk), sfa, sfb,
                             (kb > 0 || kk > 0) ? 1u : 0u);
              mma_commit(&mdone[mit % NMD]);
              if (kb == KB - 1) mma_commit(afull);  // the unit's accumulator
            }
            __syncwarp();
          }
        }
      }
      if (lane == 0) mma_commit(done);
      __syncwarp();
      tmx_drain_wait(done, 0);
    }
  } else {
    // ---------------- epilogue ----------------
    regs_grow<C::REGS_HIGH>();
    const int ew = warp - C::EPI_WARP0;
    const int q = warp & 3;                 // TMEM lane quarter = token quarter
    const int cg = ew >> 2;                 // column half
    const int tok = q * 32 + lane;          // token row within the tile
    const uint32_t tlane = tmem + ((uint32_t)(q * 32) << 16);
    const int S = p.S;
    bool ok = true;
    int j = 0;
    griddep_wait();  // routing / combine buffer come from earlier kernels
    for (int u = blockIdx.x; u < total; u += gridDim.x, ++j) {
      const int ti = u / NRT, rt = u % NRT;
      const int4 tile = p.tiles[ti];
      const int p0 = tile.y, nv = tile.z;
      const int nw = weight_rows(rt);
      const bool has_cols = cg * C::CPT < nw;
      int out_tok = 0;
      float out_w = 0.0f;
      if (KIND == 2 && tok < nv) {
        const int slot = p.perm[p0 + tok];
        out_tok = (slot < S) ? slot / p.k : slot - S;
        out_w = (slot < S) ? p.topk_w[slot] : 1.0f;
      }
      if (ok) ok = mbar_wait(afull, (uint32_t)(j & 1), abort);
      ok = __all_sync(0xFFFFFFFFu, ok);
      float acc[C::CPT];
      if (ok) {
        tc_fence_after();
        // GEMM1: gate columns cg*64 .. +64 and the matching up columns
        // 128 + cg*64 ..; GEMM2: columns cg*128 .. +128
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const uint32_t clo = (KIND == 1) ? cg * 64 + r * 32 : cg * 128 + r * 64;
          const uint32_t chi = (KIND == 1) ? 128 + cg * 64 + r * 32 : clo + 32;
          if (has_cols) {
            tmem_ld32(tlane + clo, acc + ((KIND == 1) ? r * 32 : r * 64));
            tmem_ld32(tlane + chi, acc + ((KIND == 1) ? 64 + r * 32 : r * 64 + 32));
          }
        }
        tmem_wait_ld();
      }
      tc_fence_before();
      mbar_arrive(tempty);  // the accumulator may take the next unit

      if constexpr (KIND == 1) {
        // SwiGLU (gate = W13 rows 0..I-1, up = rows I..2I-1 of the same
        // channel), then MXFP8 requantisation per 32 channels, all in this
        // thread: the codes to hq, the E8M0 codes into GEMM2's A-operand
        // scale atom of this tile and K block rt.
        if (ok && tok < nv) {
#pragma unroll
          for (int c = 0; c < 64; ++c) {
            const float g = acc[c];
            const float sig = __fdiv_rn(1.0f, 1.0f + expf(-g));
            acc[c] = g * sig * acc[64 + c];
          }
          uint4* dst = reinterpret_cast<uint4*>(p.hq + (size_t)(p0 + tok) * p.I + rt * 128 + cg * 64);
          uint8_t* sf = p.hsc + ((size_t)ti * (p.I / 128) + rt) * C::SF_ATOM + (tok % 32) * 16 + (tok / 32) * 4;
#pragma unroll
          for (int b = 0; b < 2; ++b) {
            float amax = 0.0f;
#pragma unroll
            for (int c = 0; c < 32; ++c) amax = fmaxf(amax, fabsf(acc[b * 32 + c]));
            float sc;
            const int X = mx_e4m3_exponent(amax, &sc);
#pragma unroll
            for (int v = 0; v < 2; ++v) {
              uint32_t w[4];
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const int c = b * 32 + v * 16 + i * 4;
                w[i] = f32x2_to_e4m3x2(__fdiv_rn(acc[c], sc), __fdiv_rn(acc[c + 1], sc)) |
                       (f32x2_to_e4m3x2(__fdiv_rn(acc[c + 2], sc), __fdiv_rn(acc[c + 3], sc)) << 16);
              }
              dst[b * 2 + v] = make_uint4(w[0], w[1], w[2], w[3]);
            }
            sf[cg * 2 + b] = static_cast<uint8_t>(X + 127);
          }
        }
      } else {
        if (ok && has_cols && tok < nv) {
          const int col0 = rt * 256 + cg * 128;
          if (p.y_rows) {
            // unfused combine: keep this position's expert output row
            float4* dst = reinterpret_cast<float4*>(p.y_rows + (size_t)(p0 + tok) * p.H + col0);
#pragma unroll
            for (int c = 0; c < C::CPT; c += 4) dst[c / 4] = make_float4(acc[c], acc[c + 1], acc[c + 2], acc[c + 3]);
          } else {
            // fused combine: out_acc[token] += w * y (fp32 vector reductions in L2)
            float4* dst = reinterpret_cast<float4*>(p.out_acc + (size_t)out_tok * p.H + col0);
#pragma unroll
            for (int c = 0; c < C::CPT; c += 4)
              atomicAdd(dst + c / 4, make_float4(out_w * acc[c], out_w * acc[c + 1], out_w * acc[c + 2],
                                                 out_w * acc[c + 3]));
          }
        }
      }
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
template <int KIND>
static cudaError_t tmx_set_attr() {
  using C = TmxCfg<KIND>;
  cudaError_t e = cudaFuncSetAttribute(moe_gemm_tmx_kernel<KIND>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  // The register split (setmaxnreg) is only safe if the block is launched
  // with the registers it was laid out for.
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, moe_gemm_tmx_kernel<KIND>);
  if (e != cudaSuccess) return e;
  if (fa.numRegs < C::LAUNCH_REGS) return cudaErrorInvalidConfiguration;
  return cudaSuccess;
}

cudaError_t gemm_tmx_setup() {
  cudaError_t e = tmx_set_attr<1>();
  if (e == cudaSuccess) e = tmx_set_attr<2>();
  return e;
}

template <int KIND>
static cudaError_t tmx_launch(int grid, const CUtensorMap& tw, const CUtensorMap& tx, const GemmParams& p,
                              cudaStream_t s) {
  using C = TmxCfg<KIND>;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(C::THREADS);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, moe_gemm_tmx_kernel<KIND>, tw, tx, p);
}

cudaError_t launch_gemm1_tmx(int grid, const CUtensorMap& tw, const CUtensorMap& tx, const GemmParams& p,
                             cudaStream_t s) {
  return tmx_launch<1>(grid, tw, tx, p, s);
}

cudaError_t launch_gemm2_tmx(int grid, const CUtensorMap& tw, const CUtensorMap& th, const GemmParams& p,
                             cudaStream_t s) {
  return tmx_launch<2>(grid, tw, th, p, s);
}

}  // namespace moe
