/*
 * moe.h -- C ABI of the B200 (sm_100a) decode-regime MoE layer library
 * (libmoe.so).
 *
 * The operation (one MoE layer, single GPU):
 *   given hidden states x[T,H] (bf16) and the router's top-k choice per token
 *   (expert ids [T,k], combine weights [T,k]), compute
 *     out[t] = sum_j topk_w[t,j] * FFN_{ids[t,j]}(x[t])  (+ FFN_shared(x[t]))
 *   with FFN_e(x) = W2_e * (silu(W1_e x) * (W3_e x)) evaluated in the layer's
 *   quantised form: activations quantised to FP8 E4M3 per token per 128
 *   columns (scale amax/448), FP8 (128x128 block-scaled) or MXFP4 expert
 *   weights, fp32 accumulation, SwiGLU output requantised to FP8 per token per
 *   128 channels, fp32 combine, bf16 output.
 * Sources:
 *   - "GC-MoE: Overlapping Expert-Parallel Token Dispatch with FP8/FP4 Grouped
 *     GEMM via CUDA Green Contexts", abstract: dispatch -> grouped GEMMs ->
 *     combine; operand-swapped tcgen05 block-scaled MMA; fused SwiGLU and
 *     requantisation; optional shared experts.
 *   - FusedDeepMoE execution-flow page (Ascend fused family): the step math
 *     (QuantToken, OpDequant, OpSwiglu with gate = first half, OpBlockQuant,
 *     prefix-summed expert ranges, ReducePermute combine, shared expert as one
 *     group of all tokens).
 *   - OCP FP8 (E4M3) and OCP MX v1.0 (E2M1 + E8M0 per 32) define the formats.
 *
 * Conventions for every entry point:
 *   - Pointers named d_* or documented as "device" are CUDA device pointers on
 *     the context's device; the library never frees memory it did not allocate.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  All work is
 *     enqueued asynchronously on it; no entry point synchronises the device
 *     unless documented.
 *   - Errors detectable on the host are returned synchronously and nothing is
 *     enqueued.  Errors detected on the device (bad expert id, a pipeline wait
 *     that gave up) are OR-ed into a device status word that
 *     moe_get_device_status() reads.
 *   - The calls are not thread-safe on one context; use one context per
 *     host thread or serialise.
 */
#ifndef FP4_BLOCK_SCALED_ROUTE_B200_MOE_H
#define FP4_BLOCK_SCALED_ROUTE_B200_MOE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct moe_ctx moe_ctx;

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,  /* null pointer, bad size, misaligned pointer */
  MOE_ERR_UNSUPPORTED = 2,  /* shape/format outside what the kernels handle, or not an sm_100 GPU */
  MOE_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed */
  MOE_ERR_NO_MEMORY = 4,    /* workspace allocation failed */
  MOE_ERR_TIMEOUT = 5,      /* device: a pipeline wait gave up (no hang; outputs invalid) */
  MOE_ERR_BAD_ROUTING = 6   /* device: an expert id outside [0,E); that slot was dropped */
} moe_status;

/* Expert weight formats. */
enum {
  /* w13 u8 E4M3 [NE, 2I, H], rows 0..I-1 = gate (W1), I..2I-1 = up (W3);
   * s13 f32 [NE, 2I/128, H/128] one scale per 128x128 block;
   * w2 u8 E4M3 [NE, H, I]; s2 f32 [NE, H/128, I/128]. */
  MOE_WFMT_FP8_E4M3_B128 = 0,
  /* w13 u8 [NE, 2I, H/2]: E2M1 nibbles, element 2c in the low nibble of byte c;
   * w2 u8 [NE, H, I/2]; scales are E8M0 (2^(e-127)) per 32 elements along K,
   * plain layout [NE, rows, K/32], converted once with moe_pack_mxfp4_scales()
   * into the layout moe_forward() reads: the shared-memory image of the
   * block-scale atoms that the tensor cores' scale copy takes, which a plain
   * [rows, K/32] array cannot be loaded into by TMA (4 bytes per row and K
   * block, below TMA's 16-byte minimum).  moe_forward() refuses, with
   * MOE_ERR_INVALID_ARG, scale pointers that no moe_pack_mxfp4_scales() call
   * wrote and no moe_declare_packed_scales() call declared. */
  MOE_WFMT_MXFP4_E2M1_E8M0_K32 = 1,
  /* NVFP4 (named among the 4-bit expert layouts of the onnxruntime QMoE
   * offload PR page; NVIDIA's definition): w13 u8 [NE, 2I, H/2] and w2 u8
   * [NE, H, I/2] E2M1 nibbles as for MXFP4; s13 / s2 E4M3 scale codes per 16
   * elements along K, plain layout [NE, rows, K/16], converted once with
   * moe_pack_nvfp4_scales(); g13 / g2 fp32 [NE] per-expert global scales.
   * Weight value = e2m1 * e4m3(scale) * g.  The tensor cores take NVFP4 only
   * with FP4 on both sides, so the activations are quantised to NVFP4 too
   * (see moe_forward_nvfp4).  Used through moe_forward_nvfp4(), which, like
   * moe_forward() for MXFP4, refuses scale pointers that no
   * moe_pack_nvfp4_scales() call wrote and none was declared packed. */
  MOE_WFMT_NVFP4_E2M1_E4M3_K16 = 2,
  /* MXFP4 weights (the MOE_WFMT_MXFP4_E2M1_E8M0_K32 layout and packed scales)
   * with MXFP4 activations: x and the SwiGLU output are quantised per 32
   * columns to E2M1 with an E8M0 scale 2^X, X = floor(log2 amax) - 2 clamped
   * to [-127, 127] (OCP MX v1.0; -127 for an all-zero block), so that the
   * tensor cores (kind::mxf4, UE8M0 scales on both operands) apply every
   * scale and no fp32 scale is promoted.  Used through moe_forward(); tiles
   * hold at most 32 tokens. */
  MOE_WFMT_MXFP4_W4A4 = 3,
  /* MXFP8 (OCP MX v1.0 with E4M3 elements; the power-of-two-scaled FP8
   * layouts the DeepGEMM 26/09 news page names for Mega MoE): w13 u8 E4M3
   * [NE, 2I, H], w2 u8 E4M3 [NE, H, I]; scales E8M0 (2^(e-127)) per 32
   * elements along K, plain layout [NE, rows, K/32], converted once with
   * moe_pack_mxfp4_scales() (the same E8M0 atom layout).  The activations
   * (x, and the SwiGLU output) are quantised to MXFP8 per 32 columns: X =
   * floor(log2 amax) - 8 clamped to [-127, 127] (-127 for an all-zero
   * block), elements e4m3(v / 2^X) saturating at 448; the tensor cores
   * (kind::mxf8f6f4 with E8M0 scales on both operands) apply every scale, so
   * no fp32 scale is promoted and the accumulator of a whole K loop stays in
   * tensor memory.  Used through moe_forward(); always in tiles of 128
   * tokens (the token-major kernels). */
  MOE_WFMT_MXFP8_E4M3_E8M0_K32 = 4
};

/* moe_create -- context for a layer with hidden size H, expert intermediate
 * size I, E routed experts, top-k = k, weight format wfmt (MOE_WFMT_*), no
 * shared expert, up to 4096 tokens per call (the layer of the GC-MoE
 * abstract: token dispatch to E experts, grouped GEMMs on FP8/FP4
 * block-scaled expert weights, combine; the decode regime it targets is 1 to
 * 256 tokens).  Same as moe_create_ex(H, I, E, k, wfmt, 4096, 0, out). */
moe_status moe_create(int H, int I, int E, int k, int wfmt, moe_ctx** out);

/* moe_create_ex -- as moe_create, with the token capacity max_T (>= 1) and
 * n_shared (0 or 1) always-on shared experts at combine weight 1.0 (GC-MoE
 * abstract "optional shared experts"; FusedDeepMoE: the shared expert takes
 * every token as one group).  The shared expert's weights are expert index E
 * of the weight arrays (NE = E + n_shared) and share I.
 * Requirements: H and I multiples of 128, 128 <= H, I <= 8192; 1 <= E <= 1024;
 * 1 <= k <= 32.  The GPU must be sm_100 (B200).  The context owns its
 * workspace (device memory sized by max_T) on the current device; *out is
 * set to NULL on failure.  Tuning: the environment variable MOE_TILE_N
 * (16, 32, 64, or 128 for FP8), read here, fixes the token-tile width the
 * GEMMs use instead of the automatic choice from T*k/E, and MOE_COMBINE
 * ("atomic" or "rows") fixes how the top-k combine is done: fused into GEMM2
 * as fp32 reductions (default), or from stored per-position fp32 expert
 * outputs in a separate, deterministic pass that sums each token's experts
 * in ascending j (the context then holds an extra [positions, H] fp32
 * buffer).  MOE_PAIR_MMA=1 (MXFP4 weights with FP8 activations only) runs
 * GEMM1 of 16-token tiles on pairs of CTAs (tcgen05 MMAs with M = 256 over
 * two SMs, gate rows on one, up rows on the other); same results within the
 * layer tolerance, measured slower than the default on B200. */
moe_status moe_create_ex(int H, int I, int E, int k, int wfmt, int max_T, int n_shared, moe_ctx** out);

/* moe_destroy -- frees the context and its workspace (synchronises the
 * device first).  NULL is a no-op. */
void moe_destroy(moe_ctx* ctx);

/* moe_forward -- one MoE layer, the step sequence of the GC-MoE abstract
 * (dispatch, grouped GEMM1, fused SwiGLU + requantisation, grouped GEMM2,
 * combine) with the step math of the FusedDeepMoE execution-flow page:
 * QuantToken (per-token activation quantisation), OpDequant (accumulator x
 * weight block scale x token scale), OpSwiglu (gate = first half of the
 * GEMM1 rows), OpBlockQuant (requantisation of the SwiGLU output) and
 * ReducePermute (per-token sum of the top-k expert outputs, times their
 * weights).
 *   T          tokens, 0 <= T <= max_T (T = 0 enqueues nothing)
 *   x          device bf16 [T, H], 16-byte aligned
 *   topk_ids   device int32 [T, k]; ids outside [0, E) drop their slot and
 *              raise MOE_ERR_BAD_ROUTING in the device status
 *   topk_w     device fp32 [T, k], used as given (no renormalisation)
 *   w13, s13, w2, s2   device expert weights in the context's format (see
 *              MOE_WFMT_*), weights 128-byte aligned, scales 16-byte aligned
 *   out        device bf16 [T, H], overwritten, 16-byte aligned
 * Steps, all in this library's CUDA kernels on `stream`: route (counts,
 * prefix sum, stable permutation + inverse), activation FP8 quantisation,
 * GEMM1 with fused SwiGLU + requantisation, GEMM2 with fused weighted
 * combine, bf16 output.  The workspace is reused by the next call on the same
 * context, so calls on one context must be stream-ordered. */
moe_status moe_forward(moe_ctx* ctx, int T, const void* x, const int32_t* topk_ids, const float* topk_w,
                       const void* w13, const void* s13, const void* w2, const void* s2, void* out,
                       void* stream);

/* moe_forward_nvfp4 -- one MoE layer with NVFP4 weights (a context created
 * with MOE_WFMT_NVFP4_E2M1_E4M3_K16; other contexts: MOE_ERR_INVALID_ARG).
 * Arguments as moe_forward(), plus the per-expert global scales g13, g2
 * (device fp32 [NE], 4-byte aligned); s13 / s2 in the packed layout of
 * moe_pack_nvfp4_scales().  Activations (x, and the SwiGLU output) are
 * quantised to NVFP4 per token: for every 128 columns S = amax / 2688 (1 for
 * an all-zero group), for every 16 columns an E4M3 code
 * c = e4m3((amax16 / 6) / S), elements e2m1(v / (e4m3(c) * S)) (0 where
 * c = 0).  Each 128-wide K block's MMA sum (E2M1 x E4M3 block scales of both
 * operands, in the tensor cores) is scaled by S x g[expert] and accumulated
 * in fp32.  Tiles hold at most 32 tokens. */
moe_status moe_forward_nvfp4(moe_ctx* ctx, int T, const void* x, const int32_t* topk_ids, const float* topk_w,
                             const void* w13, const void* s13, const float* g13, const void* w2, const void* s2,
                             const float* g2, void* out, void* stream);

/* moe_forward_partial -- the layer up to its fp32 combine result, for tensor
 * parallelism over the intermediate size I: every rank holds
 * an I/G slice of each expert (its gate and up rows of w13, the matching
 * columns of w2 and their scales; I/G a multiple of 128, so no quantisation
 * group straddles two ranks), and the layer output is the sum over ranks of
 * these partial results.  Arguments as moe_forward() / moe_forward_nvfp4()
 * (g13, g2 required for NVFP4 contexts, ignored otherwise), with the
 * context's I the slice size; out_f32 is device fp32 [T, H], 16-byte aligned,
 * overwritten with this rank's partial out[t] = sum_j w[t,j] * Y_slice(t, j)
 * (+ the shared expert's slice).  Sum the ranks' buffers (for example an
 * NCCL all-reduce on `stream`), then convert with moe_finalize_bf16(). */
moe_status moe_forward_partial(moe_ctx* ctx, int T, const void* x, const int32_t* topk_ids, const float* topk_w,
                               const void* w13, const void* s13, const float* g13, const void* w2, const void* s2,
                               const float* g2, float* out_f32, void* stream);

/* moe_finalize_bf16 -- out[i] = bf16_rn(in[i]) for n values (n % 4 == 0; in
 * 16-byte and out 8-byte aligned, device pointers), on `stream`: the layer's
 * output step applied to summed partial results. */
moe_status moe_finalize_bf16(const float* in, void* out, long long n, void* stream);

/* moe_pack_mxfp4_scales -- converts E8M0 scales from the plain layout
 * [rows, K/32] (rows = NE*2I for s13, NE*H for s2) into the 128x128 atom
 * layout moe_forward() reads for MOE_WFMT_MXFP4_E2M1_E8M0_K32 (same byte
 * count).  src and dst are distinct device buffers; rows % 128 == 0 and
 * K % 128 == 0.  Weight-load-time step, asynchronous on `stream`. */
moe_status moe_pack_mxfp4_scales(const uint8_t* src, uint8_t* dst, int rows, int K, void* stream);

/* moe_pack_nvfp4_scales -- converts NVFP4 E4M3 block-scale codes from the
 * plain layout [rows, K/16] into the layout moe_forward_nvfp4() reads (same
 * byte count): per 128 rows and per 64 elements along K one 512-byte atom,
 * row m's four codes at bytes (m % 32) * 16 + (m / 32) * 4 + 0..3.  src and
 * dst are distinct device buffers; rows % 128 == 0 and K % 128 == 0.
 * Weight-load-time step, asynchronous on `stream`. */
moe_status moe_pack_nvfp4_scales(const uint8_t* src, uint8_t* dst, int rows, int K, void* stream);

/* moe_declare_packed_scales -- declares that the device range [p, p + bytes)
 * holds block scales already in the packed layout of format wfmt
 * (MOE_WFMT_MXFP4_E2M1_E8M0_K32, MOE_WFMT_MXFP4_W4A4 or
 * MOE_WFMT_MXFP8_E4M3_E8M0_K32: the E8M0 atom layout of
 * moe_pack_mxfp4_scales(); MOE_WFMT_NVFP4_E2M1_E4M3_K16: that of
 * moe_pack_nvfp4_scales()), for scales packed earlier and loaded from
 * storage.  The forward entry points accept only scale pointers inside a
 * range so declared or written by a pack call; a later pack or declaration
 * that overlaps a range replaces it.  The record is process-wide and
 * host-side (thread-safe); it does not follow frees, so declare again after
 * reusing memory.  Returns MOE_ERR_INVALID_ARG for a NULL pointer, bytes <= 0
 * or another format. */
moe_status moe_declare_packed_scales(const void* p, long long bytes, int wfmt);

/* moe_get_routing -- copies the routing of the last moe_forward() (after a
 * stream synchronisation) into caller buffers (host or device):
 *   counts  int32 [E + n_shared]     tokens per expert (shared expert: T)
 *   offsets int32 [E + n_shared + 1] exclusive prefix sum of counts
 *   perm    int32 [T*k + n_shared*T] position -> slot t*k+j (shared: T*k + t), -1 past the end
 *   inv     int32 [T*k + n_shared*T] slot -> position, -1 for a dropped slot
 * Any pointer may be NULL.  Debug / test entry point. */
moe_status moe_get_routing(moe_ctx* ctx, int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* inv,
                           void* stream);

/* moe_get_activations -- copies the quantised activations of the last call
 * (after a stream synchronisation), rows in routing-position order:
 *   xq u8 E4M3 [P, H], xs fp32 [P, H/128]  (GEMM1 input, P = T*k + n_shared*T)
 *   hq u8 E4M3 [P, I], hs fp32 [P, I/128]  (GEMM2 input)
 * (NVFP4 contexts: xq [P, H/2] and hq [P, I/2] packed E2M1, xs / hs the
 * per-128 scales S; MXFP4 x MXFP4 contexts: the same packed codes, xs / hs
 * unspecified; MXFP8 contexts: E4M3 codes as for FP8, xs / hs unspecified,
 * the E8M0 codes through moe_get_block_scales.)  Rows of dropped positions
 * are unspecified.  Any pointer may be NULL. */
moe_status moe_get_activations(moe_ctx* ctx, uint8_t* xq, float* xs, uint8_t* hq, float* hs, void* stream);

/* moe_get_block_scales -- contexts with 4-bit activations only (else
 * MOE_ERR_UNSUPPORTED): the block codes of the last call's activations,
 * after a stream synchronisation, rows in routing-position order.  NVFP4:
 * E4M3 codes xsc u8 [P, H/16], hsc u8 [P, I/16]; MXFP4 x MXFP4: E8M0 codes
 * xsc u8 [P, H/32], hsc u8 [P, I/32]; MXFP8: the E8M0 codes, xsc u8
 * [P, H/32], hsc u8 [P, I/32].  Either pointer may be NULL.  Debug / test
 * entry point. */
moe_status moe_get_block_scales(moe_ctx* ctx, uint8_t* xsc, uint8_t* hsc, void* stream);

/* moe_get_device_status -- synchronises `stream`, returns MOE_OK,
 * MOE_ERR_TIMEOUT or MOE_ERR_BAD_ROUTING (timeout wins) for all calls since
 * the last status read, and clears the status word. */
moe_status moe_get_device_status(moe_ctx* ctx, void* stream);

/* moe_last_config -- tile width (tokens per MMA N tile) and grid size the
 * last moe_forward() used; debug / benchmark entry point. */
moe_status moe_last_config(moe_ctx* ctx, int* tile_n, int* grid);

/* moe_set_fault_injection -- failure-detection test hook.  mode 1: every
 * following moe_forward() on this context makes one pipeline wait of its
 * GEMM1 run out (CTA 0's first stage expects 16 bytes that never arrive), so
 * the bounded wait gives up after about a second, the kernel drains, frees
 * its tensor memory and returns, and moe_get_device_status() reports
 * MOE_ERR_TIMEOUT; that call's output is invalid.  mode 2 (with dispatch
 * overlap on, see moe_set_dispatch_overlap): the dispatch warps never
 * publish routing position 0, so the consumers of its expert's ready counter
 * run out of time the same way.  mode 0 (default) turns it off; the context
 * stays usable.  Nothing faults, traps or hangs. */
moe_status moe_set_fault_injection(moe_ctx* ctx, int mode);

/* moe_router_topk -- fused router ("Mega Gate", DeepGEMM 26/09 news page:
 * the router GEMM and the MoE routing operations in one kernel), producing
 * the inputs of moe_forward():
 *   logits[t, e] = sum_h x[t, h] * wr[e, h]  (bf16 inputs, fp32 accumulation)
 *   topk_ids[t, :] = the k largest logits of token t, in descending order,
 *                    ties to the lower expert index
 *   topk_w[t, j]   = softmax over the k chosen logits
 * (the page names the fusion but no formula; this is the plainest reading).
 *   x        device bf16 [T, H] row-major (16-byte aligned)
 *   wr       device bf16 [E, H] row-major router weights (16-byte aligned)
 *   topk_ids device int32 [T, k] (output), topk_w device fp32 [T, k] (output)
 * H, E, k and the largest T are the context's.  Two kernels on `stream`:
 * the logits GEMM, then (a programmatic dependent launch) one warp per token
 * for the top k and the softmax.  Asynchronous, no host synchronisation; the
 * context's router workspace is left zeroed for the next call, so calls on
 * one context must be stream-ordered.  The fp32 partial logits of the K splits are added with
 * atomic reductions, so a logit can differ from call to call in its last bits
 * and a near-tie between the k-th and (k+1)-th expert can resolve either way.
 * Returns MOE_ERR_UNSUPPORTED when E > 256 or E is not a multiple of 4,
 * MOE_ERR_INVALID_ARG for null or misaligned pointers or T > max_T. */
moe_status moe_router_topk(moe_ctx* ctx, int T, const void* x, const void* wr, int32_t* topk_ids, float* topk_w,
                           void* stream);

/* moe_set_green_ctx -- optional Green-Context partition of the GPU, the
 * single-GPU form of the GC-MoE abstract's split into a small dispatch
 * partition and a large compute partition (CUDA Green Contexts).
 * dispatch_sms > 0: every following moe_forward() on this context runs the
 * dispatch kernels (route, quant) in a green context of at least
 * dispatch_sms SMs (the driver rounds up; a multiple of 8 on this GPU) and
 * the grouped GEMMs and the output kernel in a green context of the
 * remaining SMs, each on its own stream; events order them after the
 * caller's stream and make the caller's stream wait for the result, so the
 * call keeps its stream semantics.  The two partitions are ordered by events,
 * not by flags polled across kernels: the driver does not guarantee that
 * kernels of two green contexts run at the same time, so no kernel waits for
 * another one while running.  dispatch_sms == 0 removes the partition
 * (the default; the environment variable MOE_GREEN_CTX=<n> sets it at
 * create time).  Synchronises the device.  Returns MOE_ERR_UNSUPPORTED when
 * the driver has no green contexts or the split fails.  A measured option:
 * the library's default is off. */
moe_status moe_set_green_ctx(moe_ctx* ctx, int dispatch_sms);

/* moe_green_ctx_sms -- SM counts of the current partition (0, 0 when off). */
moe_status moe_green_ctx_sms(moe_ctx* ctx, int* dispatch_sms, int* gemm_sms);

/* moe_set_dispatch_overlap -- optional dispatch/GEMM overlap through ready
 * flags, the GC-MoE abstract's split of the GPU into a small dispatch
 * partition and a large GEMM partition whose GEMM starts on the tokens that
 * are ready.  Green contexts cannot carry it here: a kernel that spins on
 * flags another, separately launched kernel sets may wait on work that is
 * never scheduled beside it.  So both partitions are CTAs of ONE cooperative
 * launch (all CTAs resident at once): with dispatch_ctas > 0, every
 * following moe_forward() / moe_forward_partial() on this context launches
 * no quantisation kernel; instead the epilogue warps of the last
 * dispatch_ctas CTAs of the GEMM1 grid (one CTA per SM) first quantise the
 * activations (step 2, bit for bit the quantisation kernel's codes) in
 * routing-position order and add each finished position to its expert's
 * ready counter (release), then take their GEMM1 work; every CTA streams its
 * weight tiles from the start and loads an expert's token tile and scales
 * once that counter reaches the expert's token count (acquire; bounded wait,
 * MOE_ERR_TIMEOUT in the device status when it runs out).  The route kernel
 * clears the counters.  1 <= dispatch_ctas <= the SM count; 0 turns it off
 * (the default; the environment variable MOE_DISPATCH_CTAS=<n> sets it at
 * create time).  FP8 activations only (MOE_WFMT_FP8_E4M3_B128 and
 * MOE_WFMT_MXFP4_E2M1_E8M0_K32; other contexts: MOE_ERR_UNSUPPORTED), not
 * together with moe_set_green_ctx (MOE_ERR_UNSUPPORTED), and the GPU must
 * support cooperative launches.  The profiling stage MOE_STAGE_QUANT then
 * measures zero.  A measured option: the library's default is off. */
moe_status moe_set_dispatch_overlap(moe_ctx* ctx, int dispatch_ctas);

/* moe_dispatch_overlap_ctas -- the dispatch CTA count in use (0 when off). */
moe_status moe_dispatch_overlap_ctas(moe_ctx* ctx, int* dispatch_ctas);

/* Kernel stages of one moe_forward(), in launch order (profiling index). */
enum {
  MOE_STAGE_ROUTE = 0,     /* counts, prefix sum, permutation, tile list */
  MOE_STAGE_QUANT = 1,     /* activation FP8 quantisation (+ clears the fp32 combine buffer) */
  MOE_STAGE_GEMM1 = 2,     /* grouped GEMM1 + SwiGLU + FP8 requantisation */
  MOE_STAGE_GEMM2 = 3,     /* grouped GEMM2 + top-k weighted combine */
  MOE_STAGE_FINALIZE = 4,  /* fp32 -> bf16 output (or the unfused combine + bf16 output) */
  MOE_NUM_STAGES = 5
};

/* moe_profile_enable -- on != 0: every following moe_forward() also records
 * CUDA events around each of its kernels on the caller's stream (up to 4096
 * calls are kept); on == 0: stop and discard.  Profiling entry point. */
moe_status moe_profile_enable(moe_ctx* ctx, int on);

/* moe_profile_read -- synchronises the recorded events and writes the mean
 * duration in milliseconds of each stage over the calls recorded since
 * profiling was enabled (or last read) into avg_ms[MOE_NUM_STAGES]; *calls
 * receives their number.  Resets the record. */
moe_status moe_profile_read(moe_ctx* ctx, float* avg_ms, int* calls);

/* Size of the fixed device scratch array used by moe_forward_noalloc(). */
#define MOE_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)

/* moe_forward_noalloc -- the same layer as moe_forward(), for callers that
 * cannot allocate device memory: code running under a host framework that
 * owns every device allocation (its allocator may not be bypassed), or a
 * memory-pool-locked process.  No context is needed and nothing is
 * allocated: no cudaMalloc, cudaFree or allocating library routine.  The
 * scratch (routing arrays, tile list, quantised activations, fp32 combine
 * buffer) is one file-scope device array of MOE_NOALLOC_SCRATCH_BYTES that
 * every GPU which loads the library keeps until the process exits.  The
 * method's sources describe no counterpart of this entry point; it exists
 * only for such callers.
 *   H, I, E, k, n_shared   the layer, as in moe_create_ex()
 *   wfmt       MOE_WFMT_FP8_E4M3_B128 or MOE_WFMT_MXFP4_E2M1_E8M0_K32 (scales
 *              packed with moe_pack_mxfp4_scales()); the other formats
 *              (NVFP4, MXFP4_W4A4, MXFP8) return MOE_ERR_UNSUPPORTED
 *   T, x, topk_ids, topk_w, w13, s13, w2, s2, out   as in moe_forward()
 *   d_status   optional device int32 (caller memory): cleared, then receives
 *              the device status bits of this call (1 = expert id out of
 *              range, 2 = pipeline wait timed out); NULL keeps them in the
 *              scratch, where they are not readable.
 * The scratch needed grows with T*(k + n_shared)*(H + I) plus T*H*4 bytes
 * (FP8 decode T=32, H=7168, I=2048, k=8 needs about 5 MB; T=128 about
 * 15 MB); a shape that needs more than MOE_NOALLOC_SCRATCH_BYTES returns
 * MOE_ERR_UNSUPPORTED before any device work.
 * The first call on a device performs a one-time set-up on the current
 * device (looks up the array's device address, sets kernel attributes).
 * That set-up is thread-safe: host threads making their first calls at the
 * same time wait for one another.  A device index of 64 or more returns
 * MOE_ERR_UNSUPPORTED.  Every call, on every stream, shares the one array
 * and leaves its contents behind: calls whose execution overlaps on the GPU
 * race and corrupt each other's results, so order them (one stream, or
 * events). */
moe_status moe_forward_noalloc(int H, int I, int E, int k, int wfmt, int n_shared, int T, const void* x,
                               const int32_t* topk_ids, const float* topk_w, const void* w13, const void* s13,
                               const void* w2, const void* s2, void* out, int32_t* d_status, void* stream);

/* moe_status_string -- static description of a status code. */
const char* moe_status_string(int status);

#ifdef __cplusplus
}
#endif
#endif
