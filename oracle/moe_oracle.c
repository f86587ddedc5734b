/*
 * moe_oracle.c -- plain CPU oracle for the decode-regime MoE layer.
 *
 * TEST INFRASTRUCTURE ONLY (tests, smoke check, CPU-baseline leg of the
 * benchmark).  The product path never includes, links or calls it, and it
 * shares nothing with the CUDA library.  The sources each function follows
 * are listed in moe_oracle.h and at each function below.
 *
 * Built with -O2 -ffp-contract=off and no fast-math, so every float
 * operation below is one IEEE fp32 operation in the order written.
 */
#include "moe_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ----------------------------------------------------------------------- */
/* Codecs.  The pages name E4M3 / E2M1 / E8M0 ("FP8", "FP4", "MXFP4") but do
 * not define them; the definitions are the OCP FP8 spec (E4M3: 1 sign bit,
 * 4 exponent bits with bias 7, 3 mantissa bits, no infinities, S.1111.111 =
 * NaN) and OCP MX v1.0 (E2M1: bias 1, 1 mantissa bit; E8M0: 2^(e-127),
 * 0xFF = NaN).                                                              */

float orc_e4m3_decode(uint8_t code) {
  int sign = code >> 7;
  int e = (code >> 3) & 0xF;
  int m = code & 0x7;
  float mag;
  if (e == 0xF && m == 0x7) return NAN;
  if (e == 0)
    mag = ldexpf((float)m / 8.0f, -6);            /* subnormal: 2^-6 * m/8 */
  else
    mag = ldexpf(1.0f + (float)m / 8.0f, e - 7);  /* normal: 2^(e-7) * (1 + m/8) */
  return sign ? -mag : mag;
}

/* Round-to-nearest, ties to the even code, saturating at the largest finite
 * magnitude (448 = code 0x7E).  Positive codes 0x00..0x7E are increasing in
 * value, so the two neighbours of |v| are found by binary search. */
uint8_t orc_e4m3_encode(float v) {
  uint8_t sign;
  float a;
  int lo, hi;
  if (isnan(v)) return 0x7F;
  sign = signbit(v) ? 0x80 : 0x00;
  a = fabsf(v);
  if (a >= 448.0f) return sign | 0x7E;
  lo = 0;
  hi = 0x7E;
  while (lo < hi) { /* largest code whose value is <= a */
    int mid = (lo + hi + 1) / 2;
    if (orc_e4m3_decode((uint8_t)mid) <= a) lo = mid; else hi = mid - 1;
  }
  if (orc_e4m3_decode((uint8_t)lo) == a) return sign | (uint8_t)lo;
  {
    int up = lo + 1; /* <= 0x7E because a < 448 */
    double d_lo = (double)a - (double)orc_e4m3_decode((uint8_t)lo);
    double d_up = (double)orc_e4m3_decode((uint8_t)up) - (double)a;
    int c;
    if (d_lo < d_up) c = lo;
    else if (d_up < d_lo) c = up;
    else c = (lo & 1) ? up : lo; /* tie: the code with an even mantissa */
    return sign | (uint8_t)c;
  }
}

float orc_e2m1_decode(uint8_t nibble) {
  int sign = (nibble >> 3) & 1;
  int e = (nibble >> 1) & 3;
  int m = nibble & 1;
  float mag = (e == 0) ? 0.5f * (float)m                    /* subnormal: 0 or 0.5 */
                       : ldexpf(1.0f + 0.5f * (float)m, e - 1);
  return sign ? -mag : mag;
}

/* Round-to-nearest, ties to the even code (the one with mantissa bit 0),
 * saturating at 6 (code 0x7).  The sign bit is kept, also when the magnitude
 * rounds to zero (code 0x8 = -0), as for E4M3 above.  NaN is never produced
 * by the layer; it maps to +6. */
uint8_t orc_e2m1_encode(float v) {
  uint8_t sign;
  float a;
  int lo;
  if (isnan(v)) return 0x7;
  sign = signbit(v) ? 0x8 : 0x0;
  a = fabsf(v);
  if (a >= 6.0f) return sign | 0x7;
  lo = 0; /* largest code whose value is <= a (codes 0..7 increase in value) */
  while (lo < 7 && orc_e2m1_decode((uint8_t)(lo + 1)) <= a) ++lo;
  if (orc_e2m1_decode((uint8_t)lo) == a) return sign | (uint8_t)lo;
  {
    int up = lo + 1; /* <= 7 because a < 6 */
    double d_lo = (double)a - (double)orc_e2m1_decode((uint8_t)lo);
    double d_up = (double)orc_e2m1_decode((uint8_t)up) - (double)a;
    int c;
    if (d_lo < d_up) c = lo;
    else if (d_up < d_lo) c = up;
    else c = (lo & 1) ? up : lo;
    return sign | (uint8_t)c;
  }
}

float orc_e8m0_decode(uint8_t code) {
  if (code == 0xFF) return NAN;
  return ldexpf(1.0f, (int)code - 127);
}

float orc_bf16_decode(uint16_t bits) {
  uint32_t u = (uint32_t)bits << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

uint16_t orc_bf16_encode(float v) {
  uint32_t u;
  memcpy(&u, &v, 4);
  if ((u & 0x7FFFFFFFu) > 0x7F800000u) return (uint16_t)((u >> 16) | 0x40); /* quiet NaN */
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

void orc_e4m3_decode_n(const uint8_t* in, float* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_decode(in[i]);
}
void orc_e4m3_encode_n(const float* in, uint8_t* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_encode(in[i]);
}
void orc_e2m1_decode_n(const uint8_t* in, float* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_e2m1_decode(in[i]);
}
void orc_e2m1_encode_n(const float* in, uint8_t* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_e2m1_encode(in[i]);
}

int orc_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* ----------------------------------------------------------------------- */
/* Step 1, routing.  GC-MoE abstract (token dispatch to experts) and the
 * FusedDeepMoE page (per-expert token counts, group list, expand index;
 * OpCombineSend takes each range from a prefix sum of the counts).  Reading:
 * within an expert, slots keep ascending slot order (a stable counting
 * sort); ids outside [0,E) are dropped.  The shared expert (FusedDeepMoE
 * shared-expert rank: all tokens as one group) is group E, after the routed
 * groups, with token t as virtual slot S + t. */
int orc_route(int T, int k, int E, int n_shared, const int32_t* ids,
              int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* inv) {
  const int S = T * k;
  const int NG = E + n_shared;
  const int P = S + n_shared * T;
  int dropped = 0;
  int32_t* fill = (int32_t*)malloc(sizeof(int32_t) * (size_t)(NG + 1));
  for (int g = 0; g < NG; ++g) counts[g] = 0;
  for (int s = 0; s < S; ++s) {
    int e = ids[s];
    if (e >= 0 && e < E) counts[e] += 1; else dropped += 1;
  }
  if (n_shared) counts[E] = T;
  offsets[0] = 0;
  for (int g = 0; g < NG; ++g) offsets[g + 1] = offsets[g] + counts[g];
  for (int g = 0; g <= NG; ++g) fill[g] = offsets[g];
  for (int p = 0; p < P; ++p) { perm[p] = -1; inv[p] = -1; }
  for (int s = 0; s < S; ++s) {
    int e = ids[s];
    if (e >= 0 && e < E) {
      int p = fill[e]++;
      perm[p] = s;
      inv[s] = p;
    }
  }
  if (n_shared) {
    for (int t = 0; t < T; ++t) {
      int p = fill[E]++;
      perm[p] = S + t;
      inv[S + t] = p;
    }
  }
  free(fill);
  return dropped;
}

/* ----------------------------------------------------------------------- */
/* Steps 2 and 5, group quantisation.  FusedDeepMoE QuantToken (abs, row max,
 * scale, stored dequant scale, round) and OpBlockQuant (abs -> max -> scale
 * -> quant), with the FP8 E4M3 maximum 448 in place of the int8 127 and one
 * group per 128 columns (the layer's FP8 per-token per-128-column format).
 * Readings: s = amax / 448 in fp32; q = e4m3(v / s) with RNE and
 * saturation; an all-zero group gets s = 1. */
void orc_quant_row_f32(int K, const float* v, uint8_t* q, float* s) {
  for (int g = 0; g < K / 128; ++g) {
    const float* vg = v + (size_t)g * 128;
    float amax = 0.0f;
    float sc;
    for (int c = 0; c < 128; ++c) {
      float a = fabsf(vg[c]);
      if (a > amax) amax = a;
    }
    sc = amax / 448.0f;
    if (amax == 0.0f) sc = 1.0f;
    s[g] = sc;
    for (int c = 0; c < 128; ++c) q[(size_t)g * 128 + c] = orc_e4m3_encode(vg[c] / sc);
  }
}

void orc_quant_act(int T, int H, const uint16_t* x, uint8_t* xq, float* xs) {
  float* row = (float*)malloc(sizeof(float) * (size_t)H);
  for (int t = 0; t < T; ++t) {
    for (int c = 0; c < H; ++c) row[c] = orc_bf16_decode(x[(size_t)t * H + c]);
    orc_quant_row_f32(H, row, xq + (size_t)t * H, xs + (size_t)t * (H / 128));
  }
  free(row);
}

/* NVFP4 (NVIDIA's definition; the onnxruntime QMoE page lists the layout and
 * a global scale but no rule) with the second-level scale taken per 128
 * columns, the layer's activation group.  Readings: S = amax128 / 2688 in
 * fp32 (2688 = E4M3 max 448 x E2M1 max 6, so the largest block scale code
 * is ~448), S = 1 for an all-zero group; block code c = e4m3((amax16 / 6) /
 * S) with two fp32 divisions; element code q = e2m1(v / d) with d =
 * e4m3_value(c) * S; a block whose code underflows to 0 stores q = 0. */
void orc_quant_row_nvfp4(int K, const float* v, uint8_t* q, uint8_t* sc, float* s) {
  for (int c = 0; c < K / 2; ++c) q[c] = 0;
  for (int g = 0; g < K / 128; ++g) {
    const float* vg = v + (size_t)g * 128;
    float amax = 0.0f;
    float S;
    for (int c = 0; c < 128; ++c) {
      float a = fabsf(vg[c]);
      if (a > amax) amax = a;
    }
    S = amax / 2688.0f;
    if (amax == 0.0f) S = 1.0f;
    s[g] = S;
    for (int b = 0; b < 8; ++b) {
      const float* vb = vg + b * 16;
      float amax16 = 0.0f;
      uint8_t code;
      float d;
      for (int c = 0; c < 16; ++c) {
        float a = fabsf(vb[c]);
        if (a > amax16) amax16 = a;
      }
      code = orc_e4m3_encode((amax16 / 6.0f) / S);
      sc[g * 8 + b] = code;
      d = orc_e4m3_decode(code) * S;
      for (int c = 0; c < 16; ++c) {
        const int col = g * 128 + b * 16 + c;
        uint8_t nib = (code == 0) ? 0 : orc_e2m1_encode(vb[c] / d);
        q[col / 2] |= (uint8_t)((col % 2 == 0) ? nib : (nib << 4));
      }
    }
  }
}

void orc_quant_act_nvfp4(int T, int H, const uint16_t* x, uint8_t* xq, uint8_t* xsc, float* xs) {
  float* row = (float*)malloc(sizeof(float) * (size_t)H);
  for (int t = 0; t < T; ++t) {
    for (int c = 0; c < H; ++c) row[c] = orc_bf16_decode(x[(size_t)t * H + c]);
    orc_quant_row_nvfp4(H, row, xq + (size_t)t * (H / 2), xsc + (size_t)t * (H / 16), xs + (size_t)t * (H / 128));
  }
  free(row);
}

/* MXFP4 activations (OCP MX v1.0 conversion with E2M1 elements): shared
 * exponent X = floor(log2(amax32)) - 2, clamped to the E8M0 range [-127, 127]
 * (an all-zero block: X = -127); elements e2m1(v / 2^X).  floor(log2 a) of a
 * positive float is read from its exponent field (normal) or its leading one
 * (subnormal), so it is exact. */
static int floor_log2f(float a) {
  uint32_t u;
  int e;
  memcpy(&u, &a, 4);
  e = (int)((u >> 23) & 0xFF);
  if (e != 0) return e - 127;
  {
    uint32_t m = u & 0x7FFFFFu;
    int p = 22;
    while (p >= 0 && !(m & (1u << p))) --p;
    return p - 149; /* subnormal: 2^-149 * m */
  }
}

void orc_quant_row_mxfp4(int K, const float* v, uint8_t* q, uint8_t* sc) {
  for (int c = 0; c < K / 2; ++c) q[c] = 0;
  for (int g = 0; g < K / 32; ++g) {
    const float* vg = v + (size_t)g * 32;
    float amax = 0.0f;
    int X;
    float s;
    for (int c = 0; c < 32; ++c) {
      float a = fabsf(vg[c]);
      if (a > amax) amax = a;
    }
    X = (amax == 0.0f) ? -127 : floor_log2f(amax) - 2;
    if (X < -127) X = -127;
    if (X > 127) X = 127;
    sc[g] = (uint8_t)(X + 127);
    s = ldexpf(1.0f, X); /* exact: 2^-127 is a subnormal float */
    for (int c = 0; c < 32; ++c) {
      const int col = g * 32 + c;
      uint8_t nib = orc_e2m1_encode(vg[c] / s);
      q[col / 2] |= (uint8_t)((col % 2 == 0) ? nib : (nib << 4));
    }
  }
}

void orc_quant_act_mxfp4(int T, int H, const uint16_t* x, uint8_t* xq, uint8_t* xsc) {
  float* row = (float*)malloc(sizeof(float) * (size_t)H);
  for (int t = 0; t < T; ++t) {
    for (int c = 0; c < H; ++c) row[c] = orc_bf16_decode(x[(size_t)t * H + c]);
    orc_quant_row_mxfp4(H, row, xq + (size_t)t * (H / 2), xsc + (size_t)t * (H / 32));
  }
  free(row);
}

/* MXFP8 (OCP MX v1.0 with E4M3 elements): X = floor(log2(amax32)) - 8,
 * clamped to [-127, 127] (an all-zero block: X = -127); elements
 * e4m3(v / 2^X), which saturates at 448 where v / 2^X reaches [448, 512). */
void orc_quant_row_mxfp8(int K, const float* v, uint8_t* q, uint8_t* sc) {
  for (int g = 0; g < K / 32; ++g) {
    const float* vg = v + (size_t)g * 32;
    float amax = 0.0f;
    int X;
    float s;
    for (int c = 0; c < 32; ++c) {
      float a = fabsf(vg[c]);
      if (a > amax) amax = a;
    }
    X = (amax == 0.0f) ? -127 : floor_log2f(amax) - 8;
    if (X < -127) X = -127;
    if (X > 127) X = 127;
    sc[g] = (uint8_t)(X + 127);
    s = ldexpf(1.0f, X); /* exact */
    for (int c = 0; c < 32; ++c) q[g * 32 + c] = orc_e4m3_encode(vg[c] / s);
  }
}

void orc_quant_act_mxfp8(int T, int H, const uint16_t* x, uint8_t* xq, uint8_t* xsc) {
  float* row = (float*)malloc(sizeof(float) * (size_t)H);
  for (int t = 0; t < T; ++t) {
    for (int c = 0; c < H; ++c) row[c] = orc_bf16_decode(x[(size_t)t * H + c]);
    orc_quant_row_mxfp8(H, row, xq + (size_t)t * H, xsc + (size_t)t * (H / 32));
  }
  free(row);
}

/* One MXFP8 row (E4M3 codes + E8M0 codes per 32) -> element x 2^X values
 * (exact in fp32). */
static void decode_mxfp8_row(const uint8_t* q, const uint8_t* sc, int K, float* out) {
  for (int c = 0; c < K; ++c) out[c] = orc_e4m3_decode(q[c]) * orc_e8m0_decode(sc[c / 32]);
}

/* One MXFP4 row (packed E2M1 + E8M0 codes per 32) -> element x 2^X values
 * (exact in fp32). */
static void decode_mxfp4_row(const uint8_t* q, const uint8_t* sc, int K, float* out) {
  for (int c = 0; c < K; ++c) {
    uint8_t nib = (c % 2 == 0) ? (q[c / 2] & 0xF) : (q[c / 2] >> 4);
    out[c] = orc_e2m1_decode(nib) * orc_e8m0_decode(sc[c / 32]);
  }
}

/* One NVFP4 row (packed E2M1 + E4M3 block codes) -> element x block scale
 * values (exact in fp32: 2 x 4 significant bits); the second-level scale is
 * applied per K block by the caller. */
static void decode_nvfp4_row(const uint8_t* q, const uint8_t* sc, int K, float* out) {
  for (int c = 0; c < K; ++c) {
    uint8_t nib = (c % 2 == 0) ? (q[c / 2] & 0xF) : (q[c / 2] >> 4);
    out[c] = orc_e2m1_decode(nib) * orc_e4m3_decode(sc[c / 16]);
  }
}

/* ----------------------------------------------------------------------- */
/* One weight row, decoded to fp32 without its FP8 block scale (FP8 path) or
 * with its E8M0 per-32 scale folded in (MXFP4 path: OCP MX element value =
 * shared scale x element). */
static void decode_row(int wfmt, const uint8_t* wrow, const uint8_t* srow_e8m0, int K,
                       const float* e4m3_tab, float* out) {
  if (wfmt == ORC_WFMT_FP8) {
    for (int c = 0; c < K; ++c) out[c] = e4m3_tab[wrow[c]];
  } else if (wfmt == ORC_WFMT_MXFP8) {
    decode_mxfp8_row(wrow, srow_e8m0, K, out);
  } else if (wfmt == ORC_WFMT_NVFP4) {
    decode_nvfp4_row(wrow, srow_e8m0 /* E4M3 block codes here */, K, out);
  } else {
    for (int c = 0; c < K; ++c) {
      uint8_t byte = wrow[c / 2];
      uint8_t nib = (c % 2 == 0) ? (byte & 0xF) : (byte >> 4); /* reading: low nibble first */
      out[c] = orc_e2m1_decode(nib) * orc_e8m0_decode(srow_e8m0[c / 32]);
    }
  }
}

/* Steps 3 and 6, one grouped-GEMM row against n activation rows.
 * FusedDeepMoE OpDequant / BlockEpilogue: accumulator x weight scale x
 * per-token scale.  With 128-wide K blocks carrying their own scales, each
 * block's partial sum is scaled and added in ascending block order.
 *   FP8:   acc = sum_kb ( sum_{c in kb} a[c] * w[c] ) * (as[kb] * ws[kb])
 *   MXFP4: acc = sum_kb ( sum_{c in kb} a[c] * w[c] ) * as[kb]  (w carries its E8M0 scale)
 *   NVFP4: as FP8 with ws[kb] = the expert's global scale, a and w carrying
 *          their E4M3 block scales */
static float row_dot(int K, const float* a, const float* as, const float* w,
                     const float* ws /* NULL for MXFP4 */) {
  float acc = 0.0f;
  for (int kb = 0; kb < K / 128; ++kb) {
    float part = 0.0f;
    for (int c = kb * 128; c < kb * 128 + 128; ++c) part += a[c] * w[c];
    if (ws) acc += part * (as[kb] * ws[kb]);
    else acc += part * as[kb];
  }
  return acc;
}

/* Step 4, SwiGLU.  FusedDeepMoE OpSwiglu: left half is the gate, result
 * left * sigmoid(left) * right. */
static float swiglu(float g, float u) {
  float sig = 1.0f / (1.0f + expf(-g));
  return g * sig * u;
}

int orc_forward_ex(const orc_dims* d, const uint16_t* x, const int32_t* ids,
                   const float* topk_w, const void* w13v, const void* s13v, const float* g13,
                   const void* w2v, const void* s2v, const float* g2, const uint8_t* token_mask,
                   float* out_f32, uint16_t* out_bf16,
                   uint8_t* dbg_xq, uint8_t* dbg_xsc, float* dbg_xs,
                   uint8_t* dbg_hq, uint8_t* dbg_hsc, float* dbg_hs) {
  const int T = d->T, H = d->H, I = d->I, E = d->E, k = d->k;
  const int wfmt = d->wfmt, nsh = d->n_shared;
  const int S = T * k, NG = E + nsh, P = S + nsh * T;
  const int HB = H / 128, IB = I / 128;
  const int nv = (wfmt == ORC_WFMT_NVFP4);
  const int mx4 = (wfmt == ORC_WFMT_MXFP4_A4);      /* MXFP4 weights and MXFP4 activations */
  const int mx8 = (wfmt == ORC_WFMT_MXFP8);          /* MXFP8 weights and MXFP8 activations */
  const int a4 = nv || mx4;                          /* 4-bit activations */
  const int wsc = mx4 ? ORC_WFMT_MXFP4 : wfmt;       /* weight decoding */
  const int byte_w = (wfmt == ORC_WFMT_FP8) || mx8;  /* one byte per weight */
  const uint8_t* w13 = (const uint8_t*)w13v;
  const uint8_t* w2 = (const uint8_t*)w2v;
  /* per-expert strides in bytes (weights) */
  const size_t w13_e = byte_w ? (size_t)2 * I * H : (size_t)2 * I * H / 2;
  const size_t w2_e = byte_w ? (size_t)H * I : (size_t)H * I / 2;
  const size_t w13_r = byte_w ? (size_t)H : (size_t)H / 2;
  const size_t w2_r = byte_w ? (size_t)I : (size_t)I / 2;
  /* activation codes per row: E4M3 bytes, or packed E2M1 (+ block codes) */
  const size_t xq_r = a4 ? (size_t)H / 2 : (size_t)H;
  const size_t hq_r = a4 ? (size_t)I / 2 : (size_t)I;
  const int bs = (mx4 || mx8) ? 32 : 16;             /* elements per block code */
  int32_t *counts, *offsets, *perm, *inv, *cidx;
  uint8_t *xq, *xsc = NULL;
  float *xs, *xd, *Y, e4m3_tab[256];
  int dropped, ncomp = 0;

  if (T < 0 || H <= 0 || I <= 0 || E <= 0 || k <= 0 || H % 128 || I % 128 ||
      (wfmt != ORC_WFMT_FP8 && wfmt != ORC_WFMT_MXFP4 && wfmt != ORC_WFMT_NVFP4 && !mx4 && !mx8) || nsh < 0 ||
      nsh > 1 ||
      (nv && (!g13 || !g2)))
    return -1;
  if (T == 0) return 0;
  for (int c = 0; c < 256; ++c) e4m3_tab[c] = orc_e4m3_decode((uint8_t)c);

  counts = (int32_t*)malloc(sizeof(int32_t) * (size_t)NG);
  offsets = (int32_t*)malloc(sizeof(int32_t) * (size_t)(NG + 1));
  perm = (int32_t*)malloc(sizeof(int32_t) * (size_t)P);
  inv = (int32_t*)malloc(sizeof(int32_t) * (size_t)P);
  cidx = (int32_t*)malloc(sizeof(int32_t) * (size_t)P);
  dropped = orc_route(T, k, E, nsh, ids, counts, offsets, perm, inv);

  /* step 2 for every token (cheap), then code values without their
   * per-128 scale (NVFP4: element x E4M3 block scale) */
  xq = (uint8_t*)malloc((size_t)T * xq_r);
  xs = (float*)malloc(sizeof(float) * (size_t)T * HB);
  xd = (float*)malloc(sizeof(float) * (size_t)T * H);
  if (nv) {
    xsc = (uint8_t*)malloc((size_t)T * (H / 16));
    orc_quant_act_nvfp4(T, H, x, xq, xsc, xs);
    for (int t = 0; t < T; ++t)
      decode_nvfp4_row(xq + (size_t)t * xq_r, xsc + (size_t)t * (H / 16), H, xd + (size_t)t * H);
    if (dbg_xsc) memcpy(dbg_xsc, xsc, (size_t)T * (H / 16));
  } else if (mx4) {
    xsc = (uint8_t*)malloc((size_t)T * (H / 32));
    orc_quant_act_mxfp4(T, H, x, xq, xsc);
    for (size_t i = 0; i < (size_t)T * HB; ++i) xs[i] = 1.0f;  /* every scale is in the codes */
    for (int t = 0; t < T; ++t)
      decode_mxfp4_row(xq + (size_t)t * xq_r, xsc + (size_t)t * (H / 32), H, xd + (size_t)t * H);
    if (dbg_xsc) memcpy(dbg_xsc, xsc, (size_t)T * (H / 32));
  } else if (mx8) {
    xsc = (uint8_t*)malloc((size_t)T * (H / 32));
    orc_quant_act_mxfp8(T, H, x, xq, xsc);
    for (size_t i = 0; i < (size_t)T * HB; ++i) xs[i] = 1.0f;  /* every scale is in the codes */
    for (int t = 0; t < T; ++t)
      decode_mxfp8_row(xq + (size_t)t * xq_r, xsc + (size_t)t * (H / 32), H, xd + (size_t)t * H);
    if (dbg_xsc) memcpy(dbg_xsc, xsc, (size_t)T * (H / 32));
  } else {
    orc_quant_act(T, H, x, xq, xs);
    for (size_t i = 0; i < (size_t)T * H; ++i) xd[i] = e4m3_tab[xq[i]];
  }
  if (dbg_xq) memcpy(dbg_xq, xq, (size_t)T * xq_r);
  if (dbg_xs) memcpy(dbg_xs, xs, sizeof(float) * (size_t)T * HB);

  /* compact index of the positions whose token is selected */
  for (int p = 0; p < P; ++p) {
    int s = perm[p], t;
    cidx[p] = -1;
    if (s < 0) continue;
    t = (s < S) ? s / k : s - S;
    if (!token_mask || token_mask[t]) cidx[p] = ncomp++;
  }
  Y = (float*)malloc(sizeof(float) * (size_t)(ncomp > 0 ? ncomp : 1) * H);

  for (int g = 0; g < NG; ++g) {
    const int p0 = offsets[g], p1 = offsets[g + 1];
    int n = 0;
    int *pos, *tok;
    float *G, *hd, *hs;
    uint8_t *hq, *hsc;
    for (int p = p0; p < p1; ++p) n += (cidx[p] >= 0);
    if (n == 0) continue;
    pos = (int*)malloc(sizeof(int) * (size_t)n);
    tok = (int*)malloc(sizeof(int) * (size_t)n);
    n = 0;
    for (int p = p0; p < p1; ++p) {
      if (cidx[p] < 0) continue;
      pos[n] = p;
      tok[n] = (perm[p] < S) ? perm[p] / k : perm[p] - S;
      ++n;
    }
    G = (float*)malloc(sizeof(float) * (size_t)n * 2 * I);
    hd = (float*)malloc(sizeof(float) * (size_t)n * I);
    hs = (float*)malloc(sizeof(float) * (size_t)n * IB);
    hq = (uint8_t*)malloc((size_t)n * hq_r);
    hsc = (uint8_t*)malloc((size_t)n * (I / bs));

    /* step 3: GEMM1, G[i][r] for gate rows r < I and up rows r >= I */
#pragma omp parallel
    {
      float* wrow = (float*)malloc(sizeof(float) * (size_t)H);
      float* ws = (float*)malloc(sizeof(float) * (size_t)HB);
#pragma omp for schedule(static)
      for (int r = 0; r < 2 * I; ++r) {
        const uint8_t* wr = w13 + (size_t)g * w13_e + (size_t)r * w13_r;
        const uint8_t* sr = NULL;
        if (wfmt == ORC_WFMT_FP8) {
          const float* s13 = (const float*)s13v;
          for (int kb = 0; kb < HB; ++kb)
            ws[kb] = s13[((size_t)g * (2 * I / 128) + (size_t)(r / 128)) * HB + kb];
        } else if (nv) {
          sr = (const uint8_t*)s13v + ((size_t)g * 2 * I + (size_t)r) * (H / 16);
          for (int kb = 0; kb < HB; ++kb) ws[kb] = g13[g];
        } else {
          sr = (const uint8_t*)s13v + ((size_t)g * 2 * I + (size_t)r) * (H / 32);
        }
        decode_row(wsc, wr, sr, H, e4m3_tab, wrow);
        for (int i = 0; i < n; ++i)
          G[(size_t)i * 2 * I + r] = row_dot(H, xd + (size_t)tok[i] * H, xs + (size_t)tok[i] * HB,
                                             wrow, (wsc == ORC_WFMT_MXFP4 || mx8) ? NULL : ws);
      }
      free(wrow);
      free(ws);
    }

    /* steps 4 and 5: SwiGLU, then requantise per 128 channels */
    {
      float* h = (float*)malloc(sizeof(float) * (size_t)I);
      for (int i = 0; i < n; ++i) {
        uint8_t* hqi = hq + (size_t)i * hq_r;
        for (int c = 0; c < I; ++c)
          h[c] = swiglu(G[(size_t)i * 2 * I + c], G[(size_t)i * 2 * I + I + c]);
        if (nv) {
          orc_quant_row_nvfp4(I, h, hqi, hsc + (size_t)i * (I / 16), hs + (size_t)i * IB);
          decode_nvfp4_row(hqi, hsc + (size_t)i * (I / 16), I, hd + (size_t)i * I);
          if (dbg_hsc) memcpy(dbg_hsc + (size_t)pos[i] * (I / 16), hsc + (size_t)i * (I / 16), (size_t)(I / 16));
        } else if (mx4) {
          orc_quant_row_mxfp4(I, h, hqi, hsc + (size_t)i * (I / 32));
          for (int kb = 0; kb < IB; ++kb) hs[(size_t)i * IB + kb] = 1.0f;
          decode_mxfp4_row(hqi, hsc + (size_t)i * (I / 32), I, hd + (size_t)i * I);
          if (dbg_hsc) memcpy(dbg_hsc + (size_t)pos[i] * (I / 32), hsc + (size_t)i * (I / 32), (size_t)(I / 32));
        } else if (mx8) {
          orc_quant_row_mxfp8(I, h, hqi, hsc + (size_t)i * (I / 32));
          for (int kb = 0; kb < IB; ++kb) hs[(size_t)i * IB + kb] = 1.0f;
          decode_mxfp8_row(hqi, hsc + (size_t)i * (I / 32), I, hd + (size_t)i * I);
          if (dbg_hsc) memcpy(dbg_hsc + (size_t)pos[i] * (I / 32), hsc + (size_t)i * (I / 32), (size_t)(I / 32));
        } else {
          orc_quant_row_f32(I, h, hqi, hs + (size_t)i * IB);
          for (int c = 0; c < I; ++c) hd[(size_t)i * I + c] = e4m3_tab[hqi[c]];
        }
        if (dbg_hq) memcpy(dbg_hq + (size_t)pos[i] * hq_r, hqi, hq_r);
        if (dbg_hs) memcpy(dbg_hs + (size_t)pos[i] * IB, hs + (size_t)i * IB, sizeof(float) * IB);
      }
      free(h);
    }

    /* step 6: GEMM2, Y[position][r] for output channels r < H */
#pragma omp parallel
    {
      float* wrow = (float*)malloc(sizeof(float) * (size_t)I);
      float* ws = (float*)malloc(sizeof(float) * (size_t)IB);
#pragma omp for schedule(static)
      for (int r = 0; r < H; ++r) {
        const uint8_t* wr = w2 + (size_t)g * w2_e + (size_t)r * w2_r;
        const uint8_t* sr = NULL;
        if (wfmt == ORC_WFMT_FP8) {
          const float* s2 = (const float*)s2v;
          for (int kb = 0; kb < IB; ++kb)
            ws[kb] = s2[((size_t)g * (H / 128) + (size_t)(r / 128)) * IB + kb];
        } else if (nv) {
          sr = (const uint8_t*)s2v + ((size_t)g * H + (size_t)r) * (I / 16);
          for (int kb = 0; kb < IB; ++kb) ws[kb] = g2[g];
        } else {
          sr = (const uint8_t*)s2v + ((size_t)g * H + (size_t)r) * (I / 32);
        }
        decode_row(wsc, wr, sr, I, e4m3_tab, wrow);
        for (int i = 0; i < n; ++i)
          Y[(size_t)cidx[pos[i]] * H + r] = row_dot(I, hd + (size_t)i * I, hs + (size_t)i * IB,
                                                    wrow, (wsc == ORC_WFMT_MXFP4 || mx8) ? NULL : ws);
      }
      free(wrow);
      free(ws);
    }
    free(pos); free(tok); free(G); free(hd); free(hs); free(hq); free(hsc);
  }

  /* step 7: top-k weighted combine (FusedDeepMoE ReducePermute: accumulate the
   * expert outputs of each token), ascending j, then the shared expert at
   * weight 1 (GC-MoE abstract, optional shared experts), then bf16. */
  for (int t = 0; t < T; ++t) {
    if (token_mask && !token_mask[t]) continue;
    for (int c = 0; c < H; ++c) {
      float o = 0.0f;
      for (int j = 0; j < k; ++j) {
        int p = inv[t * k + j];
        if (p < 0) continue;
        o += topk_w[t * k + j] * Y[(size_t)cidx[p] * H + c];
      }
      if (nsh) o += 1.0f * Y[(size_t)cidx[inv[S + t]] * H + c];
      if (out_f32) out_f32[(size_t)t * H + c] = o;
      if (out_bf16) out_bf16[(size_t)t * H + c] = orc_bf16_encode(o);
    }
  }

  free(counts); free(offsets); free(perm); free(inv); free(cidx);
  free(xq); free(xsc); free(xs); free(xd); free(Y);
  return dropped;
}

int orc_forward(const orc_dims* d, const uint16_t* x, const int32_t* ids,
                const float* topk_w, const void* w13, const void* s13,
                const void* w2, const void* s2, const uint8_t* token_mask,
                float* out_f32, uint16_t* out_bf16,
                uint8_t* dbg_xq, float* dbg_xs, uint8_t* dbg_hq, float* dbg_hs) {
  if (d && d->wfmt == ORC_WFMT_NVFP4) return -1; /* needs the global scales: orc_forward_ex */
  return orc_forward_ex(d, x, ids, topk_w, w13, s13, NULL, w2, s2, NULL, token_mask, out_f32, out_bf16,
                        dbg_xq, NULL, dbg_xs, dbg_hq, NULL, dbg_hs);
}

/* ----------------------------------------------------------------------- */
/* Fused router: DeepGEMM 26/09 news page ("Mega Gate": routing GEMM + MoE
 * routing ops in one kernel).  Reading: see moe_oracle.h.                   */
int orc_router(int T, int H, int E, int k, const uint16_t* x, const uint16_t* wr,
               float* logits, int32_t* ids, float* w) {
  if (T < 0 || H <= 0 || E <= 0 || E > 1024 || k <= 0 || k > E) return -1;
  int t;
#pragma omp parallel for schedule(static)
  for (t = 0; t < T; ++t) {
    float lg[1024];
    for (int e = 0; e < E; ++e) {
      double acc = 0.0;
      for (int h = 0; h < H; ++h)
        acc += (double)orc_bf16_decode(x[(size_t)t * H + h]) * (double)orc_bf16_decode(wr[(size_t)e * H + h]);
      lg[e] = (float)acc;
      if (logits) logits[(size_t)t * E + e] = lg[e];
    }
    /* k rounds of "largest remaining, lowest index first" */
    unsigned char taken[1024];
    memset(taken, 0, sizeof(taken));
    for (int j = 0; j < k; ++j) {
      int best = -1;
      for (int e = 0; e < E; ++e) {
        if (taken[e]) continue;
        if (best < 0 || lg[e] > lg[best]) best = e;
      }
      taken[best] = 1;
      ids[(size_t)t * k + j] = best;
    }
    /* softmax over the chosen logits (max subtracted) */
    const double m = (double)lg[ids[(size_t)t * k]];
    double z = 0.0;
    for (int j = 0; j < k; ++j) z += exp((double)lg[ids[(size_t)t * k + j]] - m);
    for (int j = 0; j < k; ++j) w[(size_t)t * k + j] = (float)(exp((double)lg[ids[(size_t)t * k + j]] - m) / z);
  }
  return 0;
}
