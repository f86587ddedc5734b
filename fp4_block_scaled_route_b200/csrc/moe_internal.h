// moe_internal.h -- parameter blocks and launchers shared by the library's
// translation units (not part of the public C ABI).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace moe {

constexpr int kMaxK = 32;        // largest top-k accepted
constexpr int kMaxGroups = 1025; // routed experts + shared expert
constexpr int kRouteThreads = 1024;

struct RouteParams {
  int T, k, E, n_shared, BN;
  const int32_t* ids;     // [T*k]
  int32_t* counts;        // [E + n_shared]
  int32_t* offsets;       // [E + n_shared + 1]
  int32_t* perm;          // [P]   position -> slot (shared: S + t)
  int32_t* inv;           // [P]   slot -> position (-1: dropped)
  int4* tiles;            // (group, first position, valid rows, 0)
  int32_t* num_tiles;     // [1]
  int32_t* status;        // [1]
  int32_t* ready;         // [E + n_shared] dispatch-overlap counters, zeroed here (null: not used)
  int32_t* tile_off;      // [E + n_shared + 1] first tile of each group (null: not exported)
  // Multi-CTA routing for many slots: part [kMaxRouteParts][E] per-chunk
  // expert counts (null: always one CTA).  nparts and chunk are set by
  // launch_route.
  int32_t* part;
  int nparts, chunk;
};
constexpr int kMaxRouteParts = 64;

struct QuantParams {
  int T, H, k, n_shared;
  const uint16_t* x;      // bf16 [T, H]
  const int32_t* inv;     // [P]
  uint8_t* xq;            // E4M3 [S_pad, H]   rows in routing order
  float* xs;              // [H/128, xs_ld]    K-block major: one row of position scales per K block
  int xs_ld;              // = S_pad
  float* out_acc;         // [T, H] zeroed here (null: not needed)
  int pdl;                // launched as a programmatic dependent of the route kernel (see quant_pdl)
  // 4-bit activations: xq holds packed E2M1 [S_pad, H/2] and xsc the block
  // codes in 16-byte entries, four codes in bytes 0..3 (bytes 4..15 stay
  // zero), so that 32 consecutive positions form a block-scale atom of the
  // MMA's B operand:
  //   NVFP4 (quant_nvfp4_kernel): E4M3 codes, [H/64][xs_ld][16], one entry
  //     per 64-column MMA step;
  //   MXFP4 (quant_mxfp4_kernel): E8M0 codes, [H/128][xs_ld][16], one entry
  //     per 128-column K block (its two MMA steps use bytes 0-1 and 2-3).
  uint8_t* xsc;
  // MXFP8 (quant_mxfp8_kernel): E8M0 codes per 32 columns written straight
  // into the MMA's A-operand scale atoms of the token-major kernel: per tile
  // of 128 positions and 128-column K block one 512-byte atom, position row
  // r's four codes at bytes (r % 32) * 16 + (r / 32) * 4 + 0..3.
  uint8_t* sf_atoms;      // [tiles][H/128][512]
  const int32_t* ids;     // [T*k] expert ids (group of a routed position)
  const int32_t* offsets; // [NG + 1] first position of each group
  const int32_t* tile_off;// [NG + 1] first tile of each group
  int E;
};

struct GemmParams {
  int H, I, k, S;         // S = T*k routed slots
  int kblocks;            // K / 128
  const float* wscale;    // FP8: fp32 [NE, rows/128, K/128]; MXFP4: packed E8M0 atoms
  const float* ascale;    // activation scales [K/128, scale_ld], K-block major
  int scale_ld;           // = S_pad (row length of ascale and hs)
  uint8_t* hq;            // GEMM1: E4M3 [S_pad, I]
  float* hs;              // GEMM1: [I/128, scale_ld]
  const int32_t* perm;    // GEMM2: position -> slot
  const float* topk_w;    // GEMM2: [T*k]
  float* out_acc;         // GEMM2: fp32 [T, H]
  const int4* tiles;
  const int32_t* num_tiles;
  int32_t* status;
  float* y_rows;          // GEMM2: non-null = store fp32 rows [S_pad, H] instead of the fused combine
  int inject;             // failure-injection test hook (0 in normal use), see moe_set_fault_injection
  // NVFP4: wscale = packed E4M3 block-scale atoms; wglobal = fp32 [NE] global
  // scales; GEMM1 writes hq as packed E2M1 [S_pad, I/2] plus hsc block codes.
  const float* wglobal;
  uint8_t* hsc;           // GEMM1: block codes of hq (layout of QuantParams::xsc for the format)
  // Dispatch overlap (GEMM1 with FP8 activations, one cooperative launch):
  // the epilogue warps of the last `disp` CTAs first quantise the
  // activations (step 2) in routing-position order and add each finished
  // position to ready[group]; a token tile and the activation scales of
  // group g are read only once ready[g] == counts[g].  disp = 0: the
  // activations come from the quantisation kernel launched before.
  int disp;
  int32_t* ready;         // [NG] finished positions per group (zeroed by the route kernel)
  const int32_t* counts;  // [NG]
  const int32_t* offsets; // [NG + 1]
  const uint16_t* x;      // bf16 [T, H]
  uint8_t* xq;            // E4M3 [S_pad, H], written by the dispatch warps
  float* xs;              // [H/128, scale_ld], written by the dispatch warps (= ascale)
  float* zero_acc;        // fp32 [T, H] combine buffer the dispatch warps clear (null: none)
  int T, NG;
  // MXFP8 token-major kernels (moe_gemm_tmx.cu): the A operand's E8M0
  // scale atoms ([tiles][K/128][512], the layout of QuantParams::sf_atoms);
  // GEMM1 writes GEMM2's into hsc in the same layout.
  const uint8_t* act_sf;
};

struct CombineParams {
  int T, H, k, n_shared;
  const float* y_rows;    // [S_pad, H] expert output per routing position
  const int32_t* inv;     // slot -> position (-1: dropped)
  const float* topk_w;    // [T*k]
  uint16_t* out;          // bf16 [T, H]
};

struct RouterParams {
  int T, H, E, k;
  int N;                  // MMA N: E rounded up to a multiple of 16 (<= 256)
  int kblocks;            // H / 64
  int splits;             // K splits per token tile (grid = tiles x splits)
  int wbox_rows;          // rows of one router-weight TMA box (= N)
  int tmem_cols;
  float* logits;          // fp32 [tiles*128, E], zero between calls
  int32_t* ids;           // [T, k]
  float* w;               // [T, k]
  int32_t* status;
};

size_t router_smem_bytes(int E);
cudaError_t router_setup(int E);
cudaError_t launch_router(const CUtensorMap& tx, const CUtensorMap& tw, const RouterParams& p, cudaStream_t s);

size_t route_smem_bytes(int n_groups);
cudaError_t launch_route(const RouteParams& p, cudaStream_t s);
// Whether the quantisation kernel overlaps the route kernel (a programmatic
// dependent of it, QuantParams::pdl): only when the layer's weight stream is
// short.  GEMM1 may then be scheduled only once the routing is complete, so
// its first ring of weight loads no longer runs during the routing; for a
// long weight stream that costs more than the hidden launch gap saves.
// Bound: min(E, T*k) routed experts plus the shared one, 3*H*I bytes each.
inline bool quant_pdl(int T, int k, int E, int n_shared, int H, int I) {
  const long long routed = (long long)T * k < E ? (long long)T * k : E;
  return (routed + n_shared) * 3LL * H * I <= (32LL << 20);
}
cudaError_t launch_quant(const QuantParams& p, cudaStream_t s);
cudaError_t launch_quant_nvfp4(const QuantParams& p, cudaStream_t s);
cudaError_t launch_quant_mxfp4(const QuantParams& p, cudaStream_t s);
cudaError_t launch_finalize(const float* acc, uint16_t* out, long long n, cudaStream_t s);
cudaError_t gemm_setup(int wfmt);  // raise shared-memory limits once per process
// GEMM1 for MXFP4 weights with FP8 activations and 16-token tiles on CTA
// pairs (moe_gemm_pair.cu): set-up, the number of pairs it launches, launch
// (tx8: the activations with 8-row boxes; tsf: the packed weight scales as
// [atoms * 2][256] bytes).
cudaError_t gemm_pair_setup();
int gemm_pair_clusters();
cudaError_t launch_gemm1_pair(const CUtensorMap& tw, const CUtensorMap& tx8, const CUtensorMap& tsf,
                              const GemmParams& p, cudaStream_t s);
// tw: weight tiles; tx / th: token tiles.
// tsf: NVFP4 token block-scale codes, map over [K/64 * S_pad rows, 16 bytes]
// with boxes of 32 rows; unused otherwise.
cudaError_t launch_gemm1(int wfmt, int BN, int grid, const CUtensorMap& tw, const CUtensorMap& tx,
                         const CUtensorMap& tsf, const GemmParams& p, cudaStream_t s);
cudaError_t launch_gemm2(int wfmt, int BN, int grid, const CUtensorMap& tw, const CUtensorMap& th,
                         const CUtensorMap& tsf, const GemmParams& p, cudaStream_t s);
// Token-major kernels for 128-token tiles (FP8 weights), moe_gemm_tm.cu.
cudaError_t gemm_tm_setup();
cudaError_t launch_gemm1_tm(int grid, const CUtensorMap& tw, const CUtensorMap& tx, const GemmParams& p,
                            cudaStream_t s);
cudaError_t launch_gemm2_tm(int grid, const CUtensorMap& tw, const CUtensorMap& th, const GemmParams& p,
                            cudaStream_t s);
// MXFP8 token-major kernels (block-scaled MMA, no promotion), moe_gemm_tmx.cu.
cudaError_t gemm_tmx_setup();
cudaError_t launch_gemm1_tmx(int grid, const CUtensorMap& tw, const CUtensorMap& tx, const GemmParams& p,
                             cudaStream_t s);
cudaError_t launch_gemm2_tmx(int grid, const CUtensorMap& tw, const CUtensorMap& th, const GemmParams& p,
                             cudaStream_t s);
cudaError_t launch_quant_mxfp8(const QuantParams& p, cudaStream_t s);
cudaError_t launch_combine(const CombineParams& p, cudaStream_t s);
cudaError_t launch_pack_e8m0(const uint8_t* src, uint8_t* dst, int rows, int kgroups, cudaStream_t s);

// Packed block-scale registry (moe_api.cu): device ranges written by
// moe_pack_mxfp4_scales / moe_pack_nvfp4_scales or declared with
// moe_declare_packed_scales, by format (MOE_WFMT_MXFP4_E2M1_E8M0_K32 for
// E8M0 atoms, MOE_WFMT_NVFP4_E2M1_E4M3_K16 for E4M3 atoms).  True when
// [p, p + bytes) lies inside one registered range of that format.
bool packed_scales_known(const void* p, size_t bytes, int fmt);

}  // namespace moe
