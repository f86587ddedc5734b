/*
 * moe_oracle.h -- plain, slow CPU oracle for the decode-regime MoE layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may include, link or
 * call this file: only the tests, the smoke check and the benchmark's CPU
 * baseline leg use it.  It shares no code, header, table or constant with the
 * CUDA library.
 *
 * What it computes (sources):
 *  - "GC-MoE: Overlapping Expert-Parallel Token Dispatch with FP8/FP4 Grouped
 *    GEMM via CUDA Green Contexts", abstract: per layer, token dispatch to
 *    experts, grouped GEMMs on FP8/FP4 block-scaled weights, fused SwiGLU with
 *    requantisation, optional shared experts, and a combine step.
 *  - FusedDeepMoE unified-execution-flow page (Ascend fused family analysis):
 *    QuantToken (per-token dynamic activation quantisation), OpDequant
 *    (accumulator x weight scale x per-token scale), OpSwiglu (gate = first
 *    half, x_left * sigmoid(x_left) * x_right), OpBlockQuant (abs -> max ->
 *    scale -> quant of the SwiGLU output), OpCombineSend / ReducePermute
 *    (prefix-summed per-expert ranges, accumulate expert outputs per token),
 *    and the shared-expert rank that treats all tokens as one group.
 *  - Number formats, which the pages name but do not define: OCP 8-bit
 *    floating point spec (E4M3, "e4m3fn": bias 7, no infinities, S.1111.111 is
 *    NaN, max 448) and OCP Microscaling (MX) v1.0 (E2M1 elements, E8M0 shared
 *    scale per 32 elements, 0xFF = NaN).
 *  - NVFP4, named among the 4-bit expert layouts of the onnxruntime QMoE
 *    offload PR page (with a per-tensor global scale folded into its FP4
 *    lookup table) but not defined there; the definition taken is NVIDIA's
 *    public one: E2M1 elements, one E4M3 scale per 16 consecutive elements,
 *    and an fp32 second-level scale.  See orc_quant_row_nvfp4 for the
 *    encoding rule and orc_forward_ex for where each scale applies.
 *
 * Precision: fp32 arithmetic throughout (the layer's own accumulate and
 * scale precision), partial sums of one 128-wide K block in ascending k,
 * blocks promoted in ascending order.  No blocking or reordering beyond that.
 *
 * Parity pins live in tests/test_oracle_pins.py (codec tables against torch's
 * float8 dtype and the OCP tables, routing against numpy's stable argsort,
 * the one-expert/dense-FFN reduction, fp64 brute force on tiny shapes,
 * linearity in the combine weights, zero input) and, for NVFP4, in
 * tests/test_oracle_nvfp4.py (E2M1 rounding against the OCP table by brute
 * force, exact round trips of representable groups, error bounds, the fp64
 * restatement of the layer) and, for MXFP4 activations, in
 * tests/test_oracle_mxfp4_a4.py.
 */
#ifndef MOE_ORACLE_H
#define MOE_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { ORC_WFMT_FP8 = 0, ORC_WFMT_MXFP4 = 1, ORC_WFMT_NVFP4 = 2, ORC_WFMT_MXFP4_A4 = 3, ORC_WFMT_MXFP8 = 4 };

/* ---- codecs (OCP FP8 / OCP MX v1.0) ---------------------------------- */
float   orc_e4m3_decode(uint8_t code);          /* exact value, NaN for S.1111.111 */
uint8_t orc_e4m3_encode(float v);               /* round-to-nearest-even, saturate to +-448 */
float   orc_e2m1_decode(uint8_t nibble);        /* low 4 bits used */
uint8_t orc_e2m1_encode(float v);               /* round-to-nearest-even, saturate to +-6, sign kept */
float   orc_e8m0_decode(uint8_t code);          /* 2^(code-127), NaN for 0xFF */
float   orc_bf16_decode(uint16_t bits);
uint16_t orc_bf16_encode(float v);              /* round-to-nearest-even */

/* Vector forms for the tests (n elements). */
void orc_e4m3_decode_n(const uint8_t* in, float* out, int64_t n);
void orc_e4m3_encode_n(const float* in, uint8_t* out, int64_t n);
void orc_e2m1_decode_n(const uint8_t* in, float* out, int64_t n);
void orc_e2m1_encode_n(const float* in, uint8_t* out, int64_t n);

/* ---- step 1: routing (counting sort of slots by expert) -------------- */
/* ids [T*k] expert ids, slot s = t*k + j.  With n_shared == 1 the shared
 * expert is group E holding every token t as virtual slot S + t.
 * Outputs: counts [E+n_shared], offsets [E+n_shared+1] (exclusive scan,
 * routed groups first), perm [S + n_shared*T] (position -> slot),
 * inv [S + n_shared*T] (slot -> position, -1 for a dropped slot).
 * Returns the number of slots dropped because their id is outside [0,E). */
int orc_route(int T, int k, int E, int n_shared, const int32_t* ids,
              int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* inv);

/* ---- step 2: per-token, per-128-column activation quantisation ------- */
/* x bf16 [T,H] -> xq E4M3 [T,H], xs fp32 [T,H/128] with s = amax/448
 * (s = 1 when the group is all zero) and q = e4m3(x / s). */
void orc_quant_act(int T, int H, const uint16_t* x, uint8_t* xq, float* xs);

/* Same rule on an fp32 row (used for the SwiGLU output requantisation). */
void orc_quant_row_f32(int K, const float* v, uint8_t* q, float* s);

/* NVFP4 form of steps 2 and 5 (activations meet NVFP4 weights as FP4 x FP4).
 * One fp32 row of K (multiple of 128) values -> q packed E2M1 [K/2] (element
 * 2c in the low nibble of byte c), sc E4M3 block codes [K/16], s fp32 [K/128]:
 *   per 128-group:  S = amax128 / 2688  (2688 = 448 * 6; S = 1 if all zero)
 *   per 16-block:   c = e4m3(amax16 / 6 / S),  d = e4m3_value(c) * S
 *   per element:    q = e2m1(v / d)  (q = 0 when c == 0)
 * so that v ~ e2m1_value(q) * e4m3_value(c) * S. */
void orc_quant_row_nvfp4(int K, const float* v, uint8_t* q, uint8_t* sc, float* s);
void orc_quant_act_nvfp4(int T, int H, const uint16_t* x, uint8_t* xq, uint8_t* xsc, float* xs);

/* MXFP4 form of steps 2 and 5 (OCP MX v1.0, "MX-compliant" conversion, with
 * E2M1 elements and an E8M0 shared scale per 32 consecutive elements):
 *   X = floor(log2(amax32)) - 2 (2 = the largest E2M1 exponent), clamped to
 *   [-127, 127]; an all-zero block takes X = -127;
 *   code = X + 127 (E8M0), q = e2m1(v / 2^X)  (round-to-nearest-even,
 *   saturating at +-6).
 * One fp32 row of K (multiple of 32) values -> q packed E2M1 [K/2] (element
 * 2c in the low nibble of byte c) and sc E8M0 codes [K/32]. */
void orc_quant_row_mxfp4(int K, const float* v, uint8_t* q, uint8_t* sc);
void orc_quant_act_mxfp4(int T, int H, const uint16_t* x, uint8_t* xq, uint8_t* xsc);

/* MXFP8 form of steps 2 and 5 (OCP MX v1.0, "MX-compliant" conversion, with
 * E4M3 elements and an E8M0 shared scale per 32 consecutive elements):
 *   X = floor(log2(amax32)) - 8 (8 = the largest E4M3 exponent), clamped to
 *   [-127, 127]; an all-zero block takes X = -127;
 *   code = X + 127 (E8M0), q = e4m3(v / 2^X)  (round-to-nearest-even,
 *   saturating at +-448).
 * One fp32 row of K (multiple of 32) values -> q E4M3 [K] and sc E8M0 codes
 * [K/32]. */
void orc_quant_row_mxfp8(int K, const float* v, uint8_t* q, uint8_t* sc);
void orc_quant_act_mxfp8(int T, int H, const uint16_t* x, uint8_t* xq, uint8_t* xsc);

/* ---- steps 1-8: the whole layer -------------------------------------- */
typedef struct {
  int T, H, I, E, k;
  int wfmt;       /* ORC_WFMT_FP8, ORC_WFMT_MXFP4, ORC_WFMT_NVFP4 or ORC_WFMT_MXFP4_A4 */
  int n_shared;   /* 0 or 1: shared expert stored as expert index E */
} orc_dims;

/* Weight layouts (row-major, K contiguous), NE = E + n_shared experts:
 *  FP8:   w13 u8 [NE, 2I, H] (rows 0..I-1 gate, I..2I-1 up), s13 f32 [NE, 2I/128, H/128]
 *         w2  u8 [NE, H, I],                               s2  f32 [NE, H/128, I/128]
 *  MXFP4: w13 u8 [NE, 2I, H/2] (element 2c in the low nibble of byte c),
 *         s13 u8 E8M0 [NE, 2I, H/32]; w2 u8 [NE, H, I/2], s2 u8 [NE, H, I/32]
 * token_mask [T] (1 = compute this token) or NULL for all tokens.
 * Outputs for masked-in tokens: out_f32 [T,H] fp32 combine result and
 * out_bf16 [T,H] its bf16 rounding (either may be NULL).  Other rows are
 * left untouched.  Optional debug outputs (NULL to skip): xq/xs per token
 * [T,H] / [T,H/128]; hq/hs per slot position (routing order of orc_route)
 * [S + n_shared*T, I] / [.., I/128].
 * Returns the number of dropped slots (as orc_route), or -1 on bad arguments. */
int orc_forward(const orc_dims* d, const uint16_t* x, const int32_t* ids,
                const float* topk_w, const void* w13, const void* s13,
                const void* w2, const void* s2, const uint8_t* token_mask,
                float* out_f32, uint16_t* out_bf16,
                uint8_t* dbg_xq, float* dbg_xs, uint8_t* dbg_hq, float* dbg_hs);

/* All five formats.  ORC_WFMT_MXFP8 (E4M3 weights and activations, one E8M0
 * scale per 32 elements along K on both operands, the OCP MXFP8 format):
 *   w13 u8 E4M3 [NE, 2I, H], s13 u8 E8M0 [NE, 2I, H/32]
 *   w2  u8 E4M3 [NE, H, I],  s2  u8 E8M0 [NE, H, I/32]
 * weight value = e4m3(q) * 2^(s - 127); the activations (x and the SwiGLU
 * output) are quantised with orc_quant_row_mxfp8; every product is then
 * (element x 2^X) x (element x 2^X), summed per 128-wide K block in
 * ascending k and the blocks added in ascending order with no further
 * scale.  Its debug outputs: xq [T, H], xsc [T, H/32]; hq [P, I], hsc
 * [P, I/32] (xs / hs unused).
 * ORC_WFMT_MXFP4_A4 takes the MXFP4 weight layout above
 * and quantises the activations (x and the SwiGLU output) to MXFP4 with
 * orc_quant_row_mxfp4; every product is then (element x 2^X) x (element x
 * 2^X), summed per 128-wide K block in ascending k and the blocks added in
 * ascending order with no further scale.  Its debug outputs: xq [T, H/2],
 * xsc [T, H/32]; hq [P, I/2], hsc [P, I/32] (xs / hs unused).
 * For ORC_WFMT_NVFP4 (g13, g2 required; ignored otherwise):
 *   w13 u8 [NE, 2I, H/2] packed E2M1, s13 u8 E4M3 [NE, 2I, H/16], g13 f32 [NE]
 *   w2  u8 [NE, H, I/2],              s2  u8 E4M3 [NE, H, I/16],  g2  f32 [NE]
 * weight value = e2m1(q) * e4m3(s) * g[expert].  Activations are quantised
 * with orc_quant_row_nvfp4; each 128-wide K block's partial sum of
 * (element x block scale) products is scaled by S_act[kb] * g[expert] and
 * added in ascending block order.  NVFP4 debug outputs: xq [T, H/2],
 * xsc [T, H/16], xs [T, H/128]; hq [P, I/2], hsc [P, I/16], hs [P, I/128]
 * (dbg_xsc / dbg_hsc are unused for the other formats). */
int orc_forward_ex(const orc_dims* d, const uint16_t* x, const int32_t* ids,
                   const float* topk_w, const void* w13, const void* s13, const float* g13,
                   const void* w2, const void* s2, const float* g2, const uint8_t* token_mask,
                   float* out_f32, uint16_t* out_bf16,
                   uint8_t* dbg_xq, uint8_t* dbg_xsc, float* dbg_xs,
                   uint8_t* dbg_hq, uint8_t* dbg_hsc, float* dbg_hs);

/* ---- fused router (a "Mega Gate": routing GEMM + top-k in one step) ----
 * DeepGEMM 26/09 news page: the router GEMM and the MoE routing ops fused
 * into one kernel.  The page gives no formula; reading taken (plainest form
 * consistent with the layer's inputs): logits = x . Wr^T with x bf16 [T,H]
 * and Wr bf16 [E,H]; the k largest logits per token, ties to the lower expert
 * index, in descending order; combine weights = softmax over the k chosen
 * logits (equal to the full softmax renormalised over the chosen experts).
 * Logits are the exact dot products (fp64 accumulation, one rounding to
 * fp32); the selection compares those fp32 values; the weights are computed
 * in fp64 from them and rounded to fp32.
 * Outputs: logits [T,E] (may be NULL), ids [T,k], w [T,k].  Returns -1 on bad
 * arguments (k > E, E > 1024), else 0. */
int orc_router(int T, int H, int E, int k, const uint16_t* x, const uint16_t* wr,
               float* logits, int32_t* ids, float* w);

/* OpenMP threads the oracle will use (1 when built without OpenMP). */
int orc_num_threads(void);

#ifdef __cplusplus
}
#endif
#endif
