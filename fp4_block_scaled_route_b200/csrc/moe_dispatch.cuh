// moe_dispatch.cuh -- the dispatch phase of GEMM1 launched with dispatch
// overlap: step 2 (per-token, per-128-column FP8 quantisation of the
// activations) run by the epilogue warps of the last GemmParams::disp CTAs of
// the GEMM1 grid, concurrently with the other CTAs' weight streaming, and
// published per expert through ready counters (GC-MoE abstract: a small
// dispatch partition of the SMs runs the token dispatch concurrently with the
// grouped GEMM of the large one; single-GPU form, the partition being CTAs of
// one cooperative launch).
#pragma once

#include "moe_internal.h"
#include "moe_ptx.cuh"

namespace moe {

// Quantises routing positions pos = gw, gw + nw, ... (one warp per position,
// in routing order, so the groups become ready in the order their tiles are
// listed), then clears the fp32 combine buffer.  gw / nw: this warp's index
// among the dispatch warps of the grid and their number.  Within a position
// each lane takes whole 128-column groups (gi = lane, lane + 32, ...), whose
// 16 loads of 16 bytes are all in flight before any is used.  Each
// position's codes and scales are those of quant_kernel for its token, bit
// for bit (the same per-element operations; a maximum does not depend on
// the order it is taken in).
__device__ __forceinline__ void dispatch_quant_fp8(const GemmParams& p, int gw, int nw) {
  const int lane = threadIdx.x & 31;
  const int H = p.H, HB = p.H / 128, S = p.S;
  const int P = p.offsets[p.NG];  // valid positions (dropped slots hold none)
  int g = 0;                      // group of pos: positions only grow, so a forward walk suffices
  int g_end = p.offsets[1];
  for (int pos = gw; pos < P; pos += nw) {
    while (pos >= g_end) g_end = p.offsets[++g + 1];
    const int slot = p.perm[pos];
    const int t = slot < S ? slot / p.k : slot - S;
    const uint16_t* xr = p.x + (size_t)t * H;
    uint8_t* dst = p.xq + (size_t)pos * H;
    for (int gi = lane; gi < HB; gi += 32) {
      const uint4* src = reinterpret_cast<const uint4*>(xr + gi * 128);
      uint4 v[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) v[i] = src[i];
      float amax = 0.0f;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
        for (int j = 0; j < 4; ++j)
          amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(w[j] << 16)), fabsf(__uint_as_float(w[j] & 0xFFFF0000u))));
      }
      const float sc = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 448.0f);
      uint4* out = reinterpret_cast<uint4*>(dst + gi * 128);
#pragma unroll
      for (int i = 0; i < 8; ++i) {  // 16 values -> one 16-byte store of codes
        const uint32_t w[8] = {v[2 * i].x, v[2 * i].y, v[2 * i].z, v[2 * i].w,
                               v[2 * i + 1].x, v[2 * i + 1].y, v[2 * i + 1].z, v[2 * i + 1].w};
        uint32_t c[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint32_t a = w[2 * j], b = w[2 * j + 1];
          c[j] = f32x2_to_e4m3x2(__fdiv_rn(__uint_as_float(a << 16), sc), __fdiv_rn(__uint_as_float(a & 0xFFFF0000u), sc)) |
                 (f32x2_to_e4m3x2(__fdiv_rn(__uint_as_float(b << 16), sc), __fdiv_rn(__uint_as_float(b & 0xFFFF0000u), sc))
                  << 16);
        }
        out[i] = make_uint4(c[0], c[1], c[2], c[3]);
      }
      p.xs[(size_t)gi * p.scale_ld + pos] = sc;
    }
    // the codes go to the consumer's TMA (async proxy), the scales to its
    // plain loads: fence, then publish the position with a release add
    fence_proxy_async_global();
    __threadfence();
    __syncwarp();
    // failure-injection hook (moe_set_fault_injection mode 2): position 0
    // is never published, so its group's consumers run out of time
    if (lane == 0 && !(p.inject == 2 && pos == 0)) red_release_add_gpu(&p.ready[g], 1);
  }
  if (p.zero_acc) {
    float4* acc = reinterpret_cast<float4*>(p.zero_acc);
    const long long n4 = (long long)p.T * H / 4;
    for (long long i = (long long)gw * 32 + lane; i < n4; i += (long long)nw * 32)
      acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

// Consumer side: group g's positions are all quantised (bounded wait; on
// running out the CTA's abort word is set and false returned), with the
// proxy fence that orders the following TMA reads after the acquire.
__device__ __forceinline__ bool dispatch_ready(const GemmParams& p, int g, volatile int* abort) {
  const bool ok = ready_wait(p.ready + g, p.counts[g], abort);
  fence_proxy_async_global();
  return ok;
}

}  // namespace moe
