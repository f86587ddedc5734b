// moe_gemm_tm.cu -- token-major grouped expert GEMMs for wide token tiles
// (about 50 or more tokens per expert: prefill-sized batches), FP8 weights.
//
// Same two GEMMs as moe_gemm.cu (GEMM1 + SwiGLU + requantisation, GEMM2 +
// weighted combine), same sources (GC-MoE abstract: block-scaled FP8 grouped
// GEMM with fused SwiGLU + requantisation; FusedDeepMoE page: GmmDeqSwigluQuant,
// GmmDeq with the combine as epilogue callback, and the BlockEpilogue order
// dequant -> SwiGLU -> block quant), but with the operands the other way
// round.  When an expert holds ~128 tokens the MMA's M side is full of tokens
// anyway, so here
//   M = 128 tokens of one expert (A operand, TMEM lane = token),
//   N = 256 weight rows        (B operand, TMEM column = weight row):
//       GEMM1: 128 gate rows followed by the matching 128 up rows,
//       GEMM2: 256 consecutive rows of W2 (128 for a trailing half tile).
// One N = 256 MMA does the work of two N = 128 ones, and every epilogue
// thread owns one token: the activation scale of a K block is a register,
// the SwiGLU partner of a gate column sits in the same thread, the 128-channel
// amax of the requantisation needs one exchange between the two column
// halves, and the token's FP8 row and fp32 combine row are written with
// 16-byte stores / reductions.
//
// Per-128-K promotion is required because the fp32 FP8 block scales
// (amax/448) are not powers of two.  Every K block's fp32 partial leaves TMEM
// (tcgen05.ld) and is added into registers with the block's combined scale
// (activation scale of the token x weight block scale of the column half).
//
// Warp roles (one CTA per SM, persistent over the work units):
//   warps 0-1   TMA producers (pipeline iterations alternate between them;
//               lane 0 the token tile, lanes 1-2 the two 128-row weight boxes)
//   warps 2-3   MMA issuers (iterations alternate; warp 2 allocates TMEM)
//   warps 4-11  epilogue, two warpgroups = two halves of the 256 columns.
// The producer/MMA warpgroup gives registers to the epilogue warpgroups
// (setmaxnreg), which hold 128 fp32 accumulators per thread.
#include <cuda_bf16.h>

#include "moe_dispatch.cuh"
#include "moe_internal.h"
#include "moe_ptx.cuh"

namespace moe {

template <int KIND>
struct TmCfg {
  static constexpr int BM = 128;                 // tokens per tile: MMA M = TMEM lanes
  static constexpr int BW = 256;                 // weight rows per unit: MMA N
  static constexpr int A_BYTES = BM * 128;       // token tile: 128 rows x 128 K bytes
  static constexpr int W_BOX = 128 * 128;        // one 128-row weight box
  static constexpr int STAGE_BYTES = A_BYTES + 2 * W_BOX;
  static constexpr int STAGES = 4;
  static constexpr int NBUF = 2;                 // TMEM accumulators (2 x 256 columns)
  static constexpr int NMD = STAGES + NBUF;      // MMA-done barrier ring
  static constexpr int NPROD = 2, NMMA = 2;
  // The MMA warps and the producers take the iterations in turn without
  // ordering among themselves; their parity waits are exact when every
  // iteration sharing a warp's stage is its own or already released (the
  // stage-ring bound of the decode kernel).
  static_assert(STAGES % NMMA == 0 || NBUF <= STAGES, "an MMA warp could pass a stage's stale phase");
  static_assert(STAGES >= NPROD, "a producer could pass a stale MMA-done phase");
  static constexpr int MMA_WARP = NPROD;
  static constexpr int EPI_WARP0 = NPROD + NMMA; // = 4: warpgroup 0 is producers + MMA
  static constexpr int CG = 2;                   // epilogue warpgroups (column halves)
  static constexpr int EPI_THREADS = 128 * CG;
  static constexpr int THREADS = 32 * EPI_WARP0 + EPI_THREADS;
  static constexpr int CPT = BW / CG;            // accumulator columns per epilogue thread
  static constexpr int LAUNCH_REGS = 168;        // registers per thread at launch (launch bounds)
  static constexpr int REGS_LOW = 40;            // producer / MMA warpgroup after the split
  static constexpr int REGS_HIGH = 232;          // epilogue warpgroups after the split
  static constexpr int NBARS = STAGES + NMD + NBUF + 1;
  static constexpr int RED_FLOATS = 2 * CG * BM; // amax exchange, double-buffered by unit parity
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + RED_FLOATS * 4 + NBARS * 8 + 16;
  static constexpr int TMEM_COLS = NBUF * BW;
  static_assert(EPI_WARP0 == 4, "producer and MMA warps must form warpgroup 0");
  static_assert(128 * REGS_LOW + EPI_THREADS * REGS_HIGH <= THREADS * LAUNCH_REGS, "register split");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
  static_assert(TMEM_COLS <= 512, "TMEM");
};

// Bounded wait that ignores the abort word (drain of in-flight work).
__device__ __forceinline__ void tm_drain_wait(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kWaitCycles) break;
  }
}

// DISP: GEMM1 launched with dispatch overlap (moe_dispatch.cuh); the other
// instantiations hold none of its code.
template <int KIND, bool DISP>
__global__ void __launch_bounds__(TmCfg<KIND>::THREADS, 1)
    moe_gemm_tm_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                       const GemmParams p) {
  using C = TmCfg<KIND>;
  constexpr int STAGES = C::STAGES, NBUF = C::NBUF, NMD = C::NMD;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // stage s: [token tile 16 KB][weight box 0 16 KB][weight box 1 16 KB]
  float* red = reinterpret_cast<float*>(smem + STAGES * C::STAGE_BYTES);  // [2][CG][BM]
  uint64_t* bars = reinterpret_cast<uint64_t*>(red + C::RED_FLOATS);
  uint64_t* full = bars;             // [STAGES] TMA bytes landed
  uint64_t* mdone = full + STAGES;   // [NMD] MMAs of an iteration completed (stage free + accumulator ready)
  uint64_t* tempty = mdone + NMD;    // [NBUF] epilogue has read the accumulator
  uint64_t* done = tempty + NBUF;    // all MMAs of the CTA completed
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int KB = p.kblocks;
  // dispatch overlap: launched as a programmatic dependent of the route
  // kernel, whose tile list and counts it needs from the start
  if constexpr (DISP) griddep_wait();
  const int num_tiles = *p.num_tiles;
  // Row tiles per token tile: GEMM1 128 channels (gate + up rows), GEMM2 256
  // output rows (the last one 128 when H is an odd multiple of 128).
  const int NRT = (KIND == 1) ? p.I / 128 : (p.H + 255) / 256;
  const int rows_e = (KIND == 1) ? 2 * p.I : p.H;   // weight rows per expert
  const int RB = rows_e / 128;                       // 128-row scale blocks per expert
  const int total = num_tiles * NRT;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) mbar_init(&full[s], 1);
    for (int i = 0; i < NMD; ++i) mbar_init(&mdone[i], 1);
    for (int b = 0; b < NBUF; ++b) mbar_init(&tempty[b], C::EPI_THREADS);
    mbar_init(done, C::NMMA);
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

  // Unit u -> (token tile, row tile), token-tile major: the row tiles of one
  // token tile run side by side and share its tokens through L2, and the
  // tiles of one expert (adjacent in the tile list) share its weights.
  auto weight_rows = [&](int rt) { return (KIND == 1) ? 256 : min(256, p.H - rt * 256); };

  if (warp < C::EPI_WARP0) {
    regs_shrink<C::REGS_LOW>();
    if (warp < C::NPROD) {
      // ---------------- TMA producers ----------------
      const int pr = warp;
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_a = policy_evict_last();
      uint32_t issued = 0, last_par = 0;
      bool ok = true;
      // The weights do not depend on the previous kernel: the first ring pass
      // of weight boxes is issued before waiting for it, its token tiles after.
      bool waited = false;
      constexpr int NPEND = (STAGES + C::NPROD - 1) / C::NPROD;
      int npend = 0;
      int pend_k[NPEND], pend_p0[NPEND], pend_st[NPEND];
      constexpr int NPD = DISP ? NPEND : 1;
      int pend_e[NPD], pend_ti[NPD];
      // Dispatch overlap: plain stream order after the route kernel; a token
      // tile is loaded once its group's ready counter is complete (issued
      // even after that wait ran out, so the stage completes and the
      // pipeline drains; the call then reports MOE_ERR_TIMEOUT).
      int ready_ti = -1;  // lane 0: the last tile whose group was seen ready
      auto tokens_ready = [&](int e, int ti) {
        if constexpr (DISP) {
          if (ti != ready_ti) {
            dispatch_ready(p, e, abort);
            ready_ti = ti;
          }
        }
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
        const uint32_t tx = C::A_BYTES + (uint32_t)nw * 128;
        for (int kb = 0; kb < KB; ++kb, ++it) {
          if (it % C::NPROD != pr) continue;
          const int stage = it % STAGES;
          const uint32_t phase = (uint32_t)(it / STAGES) & 1u;
          if (lane == 0 && !waited && it >= STAGES) {
            griddep_wait();
            for (int i = 0; i < npend; ++i) {
              if constexpr (DISP) tokens_ready(pend_e[i], pend_ti[i]);
              tma_load_2d(&tmX, &full[pend_st[i]], smem + pend_st[i] * C::STAGE_BYTES, pend_k[i], pend_p0[i],
                          pol_a);
            }
            waited = true;
          }
          if (lane == 0 && ok && it >= STAGES) {
            const int prev = it - STAGES;
            ok = mbar_wait(&mdone[prev % NMD], (uint32_t)(prev / NMD) & 1u, abort);
          }
          ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
          if (ok) {
            if (lane == 0) {
              // Failure-injection hook (see moe_set_fault_injection): CTA 0's
              // first GEMM1 stage expects 16 bytes that never arrive.
              const uint32_t extra = (p.inject == 1 && KIND == 1 && it == 0 && blockIdx.x == 0) ? 16u : 0u;
              mbar_arrive_expect_tx(&full[stage], tx + extra);
              issued |= 1u << stage;
              last_par = (last_par & ~(1u << stage)) | (phase << stage);
            }
            __syncwarp();
            uint8_t* st = smem + stage * C::STAGE_BYTES;
            if (w_lane) {
              tma_load_2d(&tmW, &full[stage], st + C::A_BYTES + (lane - 1) * C::W_BOX, kb * 128, wrow, pol_w);
            } else if (lane == 0) {
              if (waited) {
                tokens_ready(e, ti);
                tma_load_2d(&tmX, &full[stage], st, kb * 128, p0, pol_a);
              } else {
                pend_k[npend] = kb * 128;
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
      if (lane == 0 && !waited) {
        griddep_wait();
        for (int i = 0; i < npend; ++i) {
          if constexpr (DISP) tokens_ready(pend_e[i], pend_ti[i]);
          tma_load_2d(&tmX, &full[pend_st[i]], smem + pend_st[i] * C::STAGE_BYTES, pend_k[i], pend_p0[i], pol_a);
        }
      }
      __syncwarp();
      if (lane == 0 && *abort)
        for (int s = 0; s < STAGES; ++s)
          if (issued & (1u << s)) tm_drain_wait(&full[s], (last_par >> s) & 1u);
    } else {
      // ---------------- MMA issuers ----------------
      const int mw = warp - C::MMA_WARP;
      bool ok = true;
      int mit = 0;
      for (int u = blockIdx.x; u < total; u += gridDim.x) {
        const int nw = weight_rows(u % NRT);
        const uint32_t idesc = idesc_f8f6f4(128, nw, 0, 0);
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
              const uint32_t d = tmem + buf * C::BW;
              const uint64_t ad = sdesc_k_sw128(smem_u32(smem + stage * C::STAGE_BYTES));
              const uint64_t bd = sdesc_k_sw128(smem_u32(smem + stage * C::STAGE_BYTES + C::A_BYTES));
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) mma_f8f6f4(d, ad + 2 * kk, bd + 2 * kk, idesc, kk > 0);
              mma_commit(&mdone[mit % NMD]);
            }
            __syncwarp();
          }
        }
      }
      if (lane == 0) mma_commit(done);
      __syncwarp();
      tm_drain_wait(done, 0);
    }
  } else {
    // ---------------- epilogue ----------------
    regs_grow<C::REGS_HIGH>();
    const int ew = warp - C::EPI_WARP0;
    const int q = warp & 3;                 // TMEM lane quarter = token quarter
    const int cg = ew >> 2;                 // column half
    const int tok = q * 32 + lane;          // token row within the tile
    const uint32_t tlane = tmem + ((uint32_t)(q * 32) << 16);
    const int S = p.S, ld = p.scale_ld;
    bool ok = true;
    int eit = 0, uparity = 0;
    griddep_wait();  // activation scales / combine buffer come from earlier kernels
    if constexpr (DISP) {
      // dispatch overlap: the last p.disp CTAs' epilogue warps quantise first
      const int dc = blockIdx.x - (int)(gridDim.x - p.disp);
      if (dc >= 0) dispatch_quant_fp8(p, dc * (C::EPI_THREADS / 32) + ew, p.disp * (C::EPI_THREADS / 32));
    }

    // Scale prefetch, two pipeline iterations ahead: the activation scale of
    // this thread's token and the weight block scales of its columns.
    struct Cursor {
      int u, kb, e, p0;
    };
    auto cursor_at = [&](int u) {
      Cursor c{u, 0, 0, 0};
      if (u < total) {
        const int4 t = p.tiles[u / NRT];
        c.e = t.x;
        c.p0 = t.y;
      }
      return c;
    };
    auto advance = [&](Cursor& c) {
      if (++c.kb == KB) c = cursor_at(c.u + gridDim.x);
    };
    // GEMM1: w0 = gate block scale, w1 = up block scale.
    // GEMM2: w0 = scale of this thread's 128-row half (w1 unused).
    auto load_scales = [&](const Cursor& c, float& a, float& w0, float& w1) {
      a = 0.0f;
      w0 = 0.0f;
      w1 = 0.0f;
      if (c.u >= total) return;
      const int rt = c.u % NRT;
      if constexpr (DISP) {
        if (c.kb == 0 && ok) ok = dispatch_ready(p, c.e, abort);  // the unit's activation scales
      }
      a = p.ascale[(size_t)c.kb * ld + c.p0 + tok];
      const float* ws = p.wscale + (size_t)c.e * RB * KB + c.kb;
      if (KIND == 1) {
        w0 = ws[(size_t)rt * KB];
        w1 = ws[(size_t)(p.I / 128 + rt) * KB];
      } else {
        const int rb = min(2 * rt + cg, RB - 1);
        w0 = ws[(size_t)rb * KB];
      }
    };
    Cursor pc = cursor_at(blockIdx.x);
    float a0, g0, h0, a1, g1, h1;
    load_scales(pc, a0, g0, h0);
    advance(pc);
    load_scales(pc, a1, g1, h1);
    advance(pc);

    for (int u = blockIdx.x; u < total; u += gridDim.x, uparity ^= 1) {
      const int ti = u / NRT, rt = u % NRT;
      const int4 tile = p.tiles[ti];
      const int p0 = tile.y, nv = tile.z;
      const int nw = weight_rows(rt);
      const bool has_cols = cg * C::CPT < nw;
      // GEMM2: a lane quarter past the tile's last valid position (the short
      // last tile of an expert) skips its TMEM reads and promotion; it still
      // takes every barrier step.  Less TMEM read traffic leaves the tensor
      // pipe less contended for the quarters that do have positions
      // (measured: GEMM2 -8 %; the same skip in GEMM1 measured slower).
      const bool live = has_cols && (KIND == 1 || q * 32 < nv);
      // GEMM2: the combine target of this thread's token (used after the K loop)
      int out_tok = 0;
      float out_w = 0.0f;
      if (KIND == 2 && tok < nv) {
        const int slot = p.perm[p0 + tok];
        out_tok = (slot < S) ? slot / p.k : slot - S;
        out_w = (slot < S) ? p.topk_w[slot] : 1.0f;
      }

      float acc[C::CPT];
#pragma unroll
      for (int c = 0; c < C::CPT; ++c) acc[c] = 0.0f;

      for (int kb = 0; kb < KB; ++kb, ++eit) {
        const int buf = eit % NBUF;
        const float slo = a0 * g0, shi = (KIND == 1) ? a0 * h0 : slo;
        a0 = a1;
        g0 = g1;
        h0 = h1;
        load_scales(pc, a1, g1, h1);
        advance(pc);
        if (ok) ok = mbar_wait(&mdone[eit % NMD], (uint32_t)(eit / NMD) & 1u, abort);
        ok = __all_sync(0xFFFFFFFFu, ok);
        if (ok) {
          tc_fence_after();
          const uint32_t tb = tlane + buf * C::BW;
          // Two rounds of 64 columns: GEMM1 round r = gate columns
          // cg*64 + r*32 .. +32 and the matching up columns 128 + ...;
          // GEMM2 round r = columns cg*128 + r*64 .. +64.
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            float dlo[32], dhi[32];
            const uint32_t clo = (KIND == 1) ? cg * 64 + r * 32 : cg * 128 + r * 64;
            const uint32_t chi = (KIND == 1) ? 128 + cg * 64 + r * 32 : clo + 32;
            if (live) {
              tmem_ld32(tb + clo, dlo);
              tmem_ld32(tb + chi, dhi);
              tmem_wait_ld();
            }
            if (r == 1) {
              tc_fence_before();
              mbar_arrive(&tempty[buf]);
            }
            if (live) {
              constexpr int olo0 = 0;
              float2* alo = reinterpret_cast<float2*>(acc + ((KIND == 1) ? r * 32 : r * 64) + olo0);
              float2* ahi = reinterpret_cast<float2*>(acc + ((KIND == 1) ? 64 + r * 32 : r * 64 + 32));
              const float2 sl = make_float2(slo, slo), sh = make_float2(shi, shi);
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                alo[i] = __ffma2_rn(make_float2(dlo[2 * i], dlo[2 * i + 1]), sl, alo[i]);
                ahi[i] = __ffma2_rn(make_float2(dhi[2 * i], dhi[2 * i + 1]), sh, ahi[i]);
              }
            }
          }
        }
      }

      if constexpr (KIND == 1) {
        // SwiGLU (gate = W13 rows 0..I-1, up = rows I..2I-1 of the same
        // channel), then FP8 requantisation of the token's 128 channels.
        float amax = 0.0f;
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const float g = acc[c];
          const float sig = __fdiv_rn(1.0f, 1.0f + expf(-g));
          acc[c] = g * sig * acc[64 + c];
          amax = fmaxf(amax, fabsf(acc[c]));
        }
        float* rb = red + uparity * (C::CG * C::BM);
        rb[cg * C::BM + tok] = amax;
        named_sync(1, C::EPI_THREADS);
        amax = fmaxf(rb[tok], rb[C::BM + tok]);
        const float sc = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 448.0f);
        if (ok && tok < nv) {
          uint4* dst = reinterpret_cast<uint4*>(p.hq + (size_t)(p0 + tok) * p.I + rt * 128 + cg * 64);
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint32_t w[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int c = v * 16 + j * 4;
              w[j] = f32x2_to_e4m3x2(__fdiv_rn(acc[c], sc), __fdiv_rn(acc[c + 1], sc)) |
                     (f32x2_to_e4m3x2(__fdiv_rn(acc[c + 2], sc), __fdiv_rn(acc[c + 3], sc)) << 16);
            }
            dst[v] = make_uint4(w[0], w[1], w[2], w[3]);
          }
          if (cg == 0) p.hs[(size_t)rt * ld + p0 + tok] = sc;
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
template <int KIND, bool DISP = false>
static cudaError_t tm_set_attr() {
  using C = TmCfg<KIND>;
  cudaError_t e = cudaFuncSetAttribute(moe_gemm_tm_kernel<KIND, DISP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  // The register split (setmaxnreg) is only safe if the block is launched
  // with the registers it was laid out for.
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, moe_gemm_tm_kernel<KIND, DISP>);
  if (e != cudaSuccess) return e;
  if (fa.numRegs < C::LAUNCH_REGS) return cudaErrorInvalidConfiguration;
  return cudaSuccess;
}

cudaError_t gemm_tm_setup() {
  cudaError_t e = tm_set_attr<1>();
  if (e == cudaSuccess) e = tm_set_attr<1, true>();
  if (e == cudaSuccess) e = tm_set_attr<2>();
  return e;
}

template <int KIND>
static cudaError_t tm_launch(int grid, const CUtensorMap& tw, const CUtensorMap& tx, const GemmParams& p,
                             cudaStream_t s) {
  using C = TmCfg<KIND>;
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
  if constexpr (KIND == 1) {
    if (p.disp) return cudaLaunchKernelEx(&cfg, moe_gemm_tm_kernel<1, true>, tw, tx, p);
  } else {
    if (p.disp) return cudaErrorInvalidValue;
  }
  return cudaLaunchKernelEx(&cfg, moe_gemm_tm_kernel<KIND, false>, tw, tx, p);
}

cudaError_t launch_gemm1_tm(int grid, const CUtensorMap& tw, const CUtensorMap& tx, const GemmParams& p,
                            cudaStream_t s) {
  return tm_launch<1>(grid, tw, tx, p, s);
}

cudaError_t launch_gemm2_tm(int grid, const CUtensorMap& tw, const CUtensorMap& th, const GemmParams& p,
                            cudaStream_t s) {
  return tm_launch<2>(grid, tw, th, p, s);
}

}  // namespace moe
