/* Drives the CPU oracle under AddressSanitizer and UndefinedBehaviorSanitizer
 * (built by tests/test_oracle_sanitizers.py with -fsanitize=address,undefined
 * -fno-sanitize-recover=all, single-threaded).  Every entry point runs on
 * small seeded inputs that include ragged shapes, the shared expert, dropped
 * ids, all five weight formats and the router; any out-of-bounds access, leak or
 * undefined operation aborts with a non-zero exit status. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "moe_oracle.h"

static uint32_t rng_state = 12345u;
static uint32_t rnd(void) {
  rng_state = rng_state * 1664525u + 1013904223u;
  return rng_state >> 8;
}
static float unit(void) { return (float)rnd() / 16777216.0f - 0.5f; }

static int check_finite(const float* v, size_t n) {
  for (size_t i = 0; i < n; ++i)
    if (!isfinite(v[i])) return 0;
  return 1;
}

static int run_layer(int T, int H, int I, int E, int k, int wfmt, int n_shared, int bad_ids) {
  const int NE = E + n_shared;
  const size_t S = (size_t)T * k;
  uint16_t* x = malloc(sizeof(uint16_t) * T * H);
  int32_t* ids = malloc(sizeof(int32_t) * S);
  float* w = malloc(sizeof(float) * S);
  for (size_t i = 0; i < (size_t)T * H; ++i) x[i] = orc_bf16_encode(4.0f * unit());
  for (size_t i = 0; i < S; ++i) {
    ids[i] = (int32_t)(rnd() % (uint32_t)E);
    w[i] = 0.1f + 0.5f * (unit() + 0.5f);
  }
  if (bad_ids && S > 2) {
    ids[0] = -1;
    ids[S - 1] = E + 3;
  }
  size_t w13_bytes, s13_bytes, w2_bytes, s2_bytes;
  if (wfmt == ORC_WFMT_FP8) {
    w13_bytes = (size_t)NE * 2 * I * H;
    s13_bytes = sizeof(float) * NE * (2 * I / 128) * (H / 128);
    w2_bytes = (size_t)NE * H * I;
    s2_bytes = sizeof(float) * NE * (H / 128) * (I / 128);
  } else if (wfmt == ORC_WFMT_MXFP8) {
    w13_bytes = (size_t)NE * 2 * I * H;
    s13_bytes = (size_t)NE * 2 * I * (H / 32);
    w2_bytes = (size_t)NE * H * I;
    s2_bytes = (size_t)NE * H * (I / 32);
  } else if (wfmt == ORC_WFMT_NVFP4) {
    w13_bytes = (size_t)NE * 2 * I * H / 2;
    s13_bytes = (size_t)NE * 2 * I * (H / 16);
    w2_bytes = (size_t)NE * H * I / 2;
    s2_bytes = (size_t)NE * H * (I / 16);
  } else {
    w13_bytes = (size_t)NE * 2 * I * H / 2;
    s13_bytes = (size_t)NE * 2 * I * (H / 32);
    w2_bytes = (size_t)NE * H * I / 2;
    s2_bytes = (size_t)NE * H * (I / 32);
  }
  uint8_t* w13 = malloc(w13_bytes);
  uint8_t* w2 = malloc(w2_bytes);
  uint8_t* s13 = malloc(s13_bytes);
  uint8_t* s2 = malloc(s2_bytes);
  for (size_t i = 0; i < w13_bytes; ++i) w13[i] = (uint8_t)(rnd() & 0x77);
  for (size_t i = 0; i < w2_bytes; ++i) w2[i] = (uint8_t)(rnd() & 0x77);
  if (wfmt == ORC_WFMT_FP8) {
    float* f13 = (float*)s13;
    float* f2 = (float*)s2;
    for (size_t i = 0; i < s13_bytes / sizeof(float); ++i) f13[i] = 0.001f + 0.01f * (unit() + 0.5f);
    for (size_t i = 0; i < s2_bytes / sizeof(float); ++i) f2[i] = 0.001f + 0.01f * (unit() + 0.5f);
  } else if (wfmt == ORC_WFMT_NVFP4) {
    for (size_t i = 0; i < s13_bytes; ++i) s13[i] = (uint8_t)(0x30 + rnd() % 0x40); /* E4M3 0.25 .. 240 */
    for (size_t i = 0; i < s2_bytes; ++i) s2[i] = (uint8_t)(0x30 + rnd() % 0x40);
  } else {
    for (size_t i = 0; i < s13_bytes; ++i) s13[i] = (uint8_t)(118 + rnd() % 8);
    for (size_t i = 0; i < s2_bytes; ++i) s2[i] = (uint8_t)(118 + rnd() % 8);
  }
  float* g13 = malloc(sizeof(float) * NE);
  float* g2 = malloc(sizeof(float) * NE);
  for (int e = 0; e < NE; ++e) {
    g13[e] = 1e-4f * (1.0f + unit());
    g2[e] = 1e-4f * (1.0f + unit());
  }
  const size_t P = S + (size_t)n_shared * T;
  float* out = malloc(sizeof(float) * T * H);
  uint16_t* outb = malloc(sizeof(uint16_t) * T * H);
  uint8_t* xq = malloc((size_t)T * H);
  uint8_t* xsc = malloc((size_t)T * (H / 16));  /* the largest block-code count (16 per code) */
  float* xs = malloc(sizeof(float) * T * (H / 128));
  uint8_t* hq = malloc(P * I + 1);
  uint8_t* hsc = malloc(P * (I / 16) + 1);
  float* hs = malloc(sizeof(float) * (P * (I / 128) + 1));
  orc_dims d = {T, H, I, E, k, wfmt, n_shared};
  const int dropped = (wfmt == ORC_WFMT_NVFP4 || wfmt == ORC_WFMT_MXFP4_A4 || wfmt == ORC_WFMT_MXFP8)
      ? orc_forward_ex(&d, x, ids, w, w13, s13, g13, w2, s2, g2, NULL, out, outb, xq, xsc, xs, hq, hsc, hs)
      : orc_forward(&d, x, ids, w, w13, s13, w2, s2, NULL, out, outb, xq, xs, hq, hs);
  int ok = dropped == (bad_ids && S > 2 ? 2 : 0) && check_finite(out, (size_t)T * H);
  int32_t* counts = malloc(sizeof(int32_t) * (NE + 1));
  int32_t* offsets = malloc(sizeof(int32_t) * (NE + 2));
  int32_t* perm = malloc(sizeof(int32_t) * (P + 1));
  int32_t* inv = malloc(sizeof(int32_t) * (P + 1));
  ok = ok && orc_route(T, k, E, n_shared, ids, counts, offsets, perm, inv) == dropped;
  free(x); free(ids); free(w); free(w13); free(w2); free(s13); free(s2); free(out); free(outb);
  free(xq); free(xs); free(hq); free(hs); free(counts); free(offsets); free(perm); free(inv);
  free(g13); free(g2); free(xsc); free(hsc);
  return ok;
}

static int run_router(int T, int H, int E, int k) {
  uint16_t* x = malloc(sizeof(uint16_t) * T * H);
  uint16_t* wr = malloc(sizeof(uint16_t) * E * H);
  for (size_t i = 0; i < (size_t)T * H; ++i) x[i] = orc_bf16_encode(2.0f * unit());
  for (size_t i = 0; i < (size_t)E * H; ++i) wr[i] = orc_bf16_encode(0.1f * unit());
  float* lg = malloc(sizeof(float) * T * E);
  int32_t* ids = malloc(sizeof(int32_t) * T * k);
  float* w = malloc(sizeof(float) * T * k);
  int ok = orc_router(T, H, E, k, x, wr, lg, ids, w) == 0 && check_finite(w, (size_t)T * k);
  ok = ok && orc_router(T, H, E, E + 1, x, wr, NULL, ids, w) == -1;  /* k > E is rejected */
  free(x); free(wr); free(lg); free(ids); free(w);
  return ok;
}

int main(void) {
  int ok = 1;
  ok &= run_layer(5, 256, 128, 6, 2, ORC_WFMT_FP8, 0, 0);
  ok &= run_layer(7, 384, 256, 5, 3, ORC_WFMT_FP8, 1, 1);
  ok &= run_layer(3, 256, 128, 4, 2, ORC_WFMT_MXFP4, 1, 0);
  ok &= run_layer(1, 128, 128, 1, 1, ORC_WFMT_MXFP4, 0, 0);
  ok &= run_layer(5, 256, 128, 6, 2, ORC_WFMT_NVFP4, 1, 1);
  ok &= run_layer(2, 384, 256, 3, 3, ORC_WFMT_NVFP4, 0, 0);
  ok &= run_layer(4, 256, 128, 5, 2, ORC_WFMT_MXFP4_A4, 1, 1);
  ok &= run_layer(5, 256, 128, 6, 2, ORC_WFMT_MXFP8, 1, 1);
  ok &= run_layer(2, 384, 256, 3, 3, ORC_WFMT_MXFP8, 0, 0);
  ok &= run_router(9, 256, 16, 4);
  ok &= run_router(2, 128, 8, 8);
  uint8_t codes[256];
  float vals[256];
  for (int i = 0; i < 256; ++i) codes[i] = (uint8_t)i;
  orc_e4m3_decode_n(codes, vals, 256);
  uint8_t back[256];
  for (int i = 0; i < 256; ++i) vals[i] = isfinite(vals[i]) ? vals[i] : 0.0f;
  orc_e4m3_encode_n(vals, back, 256);
  {
    float v16[16];
    uint8_t c16[16];
    for (int i = 0; i < 16; ++i) v16[i] = 8.0f * unit();
    orc_e2m1_encode_n(v16, c16, 16);
  }
  printf(ok ? "sanitized oracle run ok\n" : "sanitized oracle run FAILED\n");
  return ok ? 0 : 1;
}
