// moe_api.cu -- the C ABI (include/moe.h): context, workspace, tensor maps
// and the launch sequence of one MoE layer.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <iterator>
#include <map>
#include <mutex>
#include <new>

#include "moe.h"
#include "moe_internal.h"
#include "moe_ptx.cuh"

using moe::GemmParams;
using moe::QuantParams;
using moe::RouteParams;

struct moe_ctx {
  int H, I, E, k, wfmt, max_T, n_shared, NG;
  int dev, num_sms;
  int S_max, P_max, S_pad, max_tiles;
  void* ws_base;
  int32_t *counts, *offsets, *perm, *inv, *num_tiles, *status;
  int4* tiles;
  uint8_t *xq, *hq;
  float *xs, *hs, *out_acc;
  // 4-bit activations: block codes, 16-byte entries of four codes then zeros
  // (NVFP4: E4M3, [K/64][S_pad][16], one entry per 64-column MMA step;
  // MXFP4 x MXFP4: E8M0, [K/128][S_pad][16], one entry per K block), and
  // their TMA maps (boxes of 16 bytes x 32 rows = one block-scale atom)
  uint8_t *xsc, *hsc;
  CUtensorMap tm_xsc, tm_hsc;
  // tensor-map cache
  const void* c_w13;
  const void* c_w2;
  int c_bn;
  CUtensorMap tm_w13, tm_w2, tm_xq, tm_hq;
  // MOE_PAIR_MMA=1 (MXFP4 weights, FP8 activations): GEMM1 of 16-token
  // tiles on CTA pairs; its activation map (8-row boxes) and scale map
  int pair_mma;
  CUtensorMap tm_xq8, tm_s13;
  const void* c_s13;
  // last call
  int last_T, last_bn, last_grid;
  // profiling: events[call][stage boundary]
  int prof_on, prof_calls;
  cudaEvent_t* prof_ev;
  int tile_n_override;  // MOE_TILE_N environment variable (16/32/64/128), 0 = automatic
  float* y_rows;        // [S_pad, H] fp32 per-position expert outputs (MOE_COMBINE=rows only)
  int combine_mode;     // MOE_COMBINE: 0/1 fused fp32 reductions (default), 2 stored rows
  int inject;           // moe_set_fault_injection mode
  // Green-Context partition (moe_set_green_ctx): dispatch kernels on gc_sms
  // SMs, the grouped GEMMs on the remaining gc_gemm_sms.
  int gc_sms, gc_gemm_sms;
  CUgreenCtx gc_small, gc_large;
  CUstream gs_small, gs_large;
  cudaEvent_t gev_in, gev_disp, gev_done;
  // fused router (moe_router_topk): fp32 logit accumulators
  float* rt_logits;
  const void* c_wr;
  CUtensorMap tm_wr;
  // dispatch overlap (moe_set_dispatch_overlap): CTAs of the GEMM1 launch
  // that quantise the activations first, and the per-group ready counters
  int disp_ctas;
  int32_t* ready;
  // MXFP8: the first tile of each group, and the A-operand scale atoms of
  // GEMM1 (xsf, [tiles][H/128][512]) and GEMM2 (hsf, [tiles][I/128][512])
  int32_t* tile_off;
  uint8_t *xsf, *hsf;
  int max_tiles128;
  int32_t* route_part;  // per-chunk expert counts of the multi-CTA route [kMaxRouteParts][E]
};



namespace {
constexpr int kProfMaxCalls = 4096;
constexpr int kProfEvents = MOE_NUM_STAGES + 1;
}

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// Green-Context driver entry points (CUDA 12.4+ drivers), fetched at run time
// like cuTensorMapEncodeTiled so the library still loads without them.
struct GreenFns {
  CUresult (*device_get)(CUdevice*, int);
  CUresult (*get_dev_resource)(CUdevice, CUdevResource*, CUdevResourceType);
  CUresult (*split_by_count)(CUdevResource*, unsigned int*, const CUdevResource*, CUdevResource*, unsigned int,
                             unsigned int);
  CUresult (*generate_desc)(CUdevResourceDesc*, CUdevResource*, unsigned int);
  CUresult (*create)(CUgreenCtx*, CUdevResourceDesc, CUdevice, unsigned int);
  CUresult (*destroy)(CUgreenCtx);
  CUresult (*stream_create)(CUstream*, CUgreenCtx, unsigned int, int);
  CUresult (*stream_destroy)(CUstream);
  bool ok;
};

template <typename F>
bool driver_fn(const char* name, F* out) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess)
    return false;
  *out = reinterpret_cast<F>(p);
  return true;
}

const GreenFns& green_fns() {
  static GreenFns g = [] {
    GreenFns f = {};
    f.ok = driver_fn("cuDeviceGet", &f.device_get) && driver_fn("cuDeviceGetDevResource", &f.get_dev_resource) &&
           driver_fn("cuDevSmResourceSplitByCount", &f.split_by_count) &&
           driver_fn("cuDevResourceGenerateDesc", &f.generate_desc) && driver_fn("cuGreenCtxCreate", &f.create) &&
           driver_fn("cuGreenCtxDestroy", &f.destroy) && driver_fn("cuGreenCtxStreamCreate", &f.stream_create) &&
           driver_fn("cuStreamDestroy", &f.stream_destroy);
    return f;
  }();
  return g;
}

// 2-D map over a row-major matrix [rows, inner] (inner contiguous), box
// {box_inner elements, box_rows}, 128-byte swizzle unless given.
bool make_map(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t rows,
              uint64_t row_bytes, uint32_t box_rows, CUtensorMapL2promotion l2, uint32_t box_inner = 128,
              CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t gdim[2] = {inner, rows};
  cuuint64_t gstride[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, dt, 2, const_cast<void*>(base), gdim, gstride, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swz, l2, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Device ranges holding packed block scales: start -> (end, format).  A new
// range replaces every range it overlaps (their contents were overwritten).
std::mutex g_packed_mu;
std::map<uintptr_t, std::pair<uintptr_t, int>> g_packed;

void register_packed(const void* p, size_t bytes, int fmt) {
  const uintptr_t lo = reinterpret_cast<uintptr_t>(p), hi = lo + bytes;
  std::lock_guard<std::mutex> lock(g_packed_mu);
  auto it = g_packed.lower_bound(lo);
  if (it != g_packed.begin() && std::prev(it)->second.first > lo) --it;
  while (it != g_packed.end() && it->first < hi) it = g_packed.erase(it);
  g_packed[lo] = {hi, fmt};
}

// Bytes of packed s13 and s2 of a layer (same count as the plain layout).
size_t packed_bytes(int fmt, int NE, int rows, int K) {
  return (size_t)NE * rows * (K / (fmt == MOE_WFMT_NVFP4_E2M1_E4M3_K16 ? 16 : 32));
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int pick_tile_n(const moe_ctx* c, int T) {
  if (c->wfmt == MOE_WFMT_MXFP8_E4M3_E8M0_K32) return 128;  // token-major kernels only
  const double avg = (double)T * c->k / c->E;  // expected tokens per routed expert
  int bn = avg <= 8 ? 16 : avg <= 20 ? 32 : avg <= 48 ? 64 : 128;
  if (c->tile_n_override) bn = c->tile_n_override;
  if (c->wfmt == MOE_WFMT_MXFP4_E2M1_E8M0_K32 && bn > 64) bn = 64;
  if ((c->wfmt == MOE_WFMT_NVFP4_E2M1_E4M3_K16 || c->wfmt == MOE_WFMT_MXFP4_W4A4) && bn > 32)
    bn = 32;  // token scale atom: 32 tokens
  return bn;
}

}  // namespace

extern "C" {

const char* moe_status_string(int s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported shape, format or device";
    case MOE_ERR_CUDA: return "CUDA call failed";
    case MOE_ERR_NO_MEMORY: return "out of device memory";
    case MOE_ERR_TIMEOUT: return "device pipeline wait timed out";
    case MOE_ERR_BAD_ROUTING: return "expert id out of range (slot dropped)";
  }
  return "unknown status";
}

moe_status moe_create(int H, int I, int E, int k, int wfmt, moe_ctx** out) {
  return moe_create_ex(H, I, E, k, wfmt, 4096, 0, out);
}

moe_status moe_create_ex(int H, int I, int E, int k, int wfmt, int max_T, int n_shared, moe_ctx** out) {
  if (!out) return MOE_ERR_INVALID_ARG;
  *out = nullptr;
  if (H <= 0 || I <= 0 || E <= 0 || k <= 0 || max_T <= 0 || n_shared < 0) return MOE_ERR_INVALID_ARG;
  if (H % 128 || I % 128 || H > 8192 || I > 8192 || E > 1024 || k > moe::kMaxK || n_shared > 1)
    return MOE_ERR_UNSUPPORTED;
  if (wfmt != MOE_WFMT_FP8_E4M3_B128 && wfmt != MOE_WFMT_MXFP4_E2M1_E8M0_K32 && wfmt != MOE_WFMT_NVFP4_E2M1_E4M3_K16 &&
      wfmt != MOE_WFMT_MXFP4_W4A4 && wfmt != MOE_WFMT_MXFP8_E4M3_E8M0_K32)
    return MOE_ERR_UNSUPPORTED;
  if ((long long)max_T * (k + n_shared) > (1LL << 26)) return MOE_ERR_UNSUPPORTED;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  int major = 0, sms = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (major != 10) return MOE_ERR_UNSUPPORTED;
  if (!encode_fn()) return MOE_ERR_CUDA;
  // MXFP8 runs on the token-major block-scaled kernels only
  if ((wfmt == MOE_WFMT_MXFP8_E4M3_E8M0_K32 ? moe::gemm_tmx_setup() : moe::gemm_setup(wfmt)) != cudaSuccess)
    return MOE_ERR_CUDA;

  moe_ctx* c = new (std::nothrow) moe_ctx();
  if (!c) return MOE_ERR_NO_MEMORY;
  c->H = H; c->I = I; c->E = E; c->k = k; c->wfmt = wfmt; c->max_T = max_T; c->n_shared = n_shared;
  c->NG = E + n_shared;
  c->dev = dev;
  c->num_sms = sms;
  c->S_max = max_T * k;
  c->P_max = c->S_max + n_shared * max_T;
  c->S_pad = c->P_max + 128;
  c->max_tiles = c->P_max / 16 + c->NG + 1;
  if (const char* env = getenv("MOE_COMBINE")) {
    if (!strcmp(env, "atomic")) c->combine_mode = 1;
    if (!strcmp(env, "rows")) c->combine_mode = 2;
  }
  if (const char* env = getenv("MOE_GREEN_CTX")) c->gc_sms = atoi(env);  // applied below, once created
  if (const char* env = getenv("MOE_PAIR_MMA"))
    c->pair_mma = (wfmt == MOE_WFMT_MXFP4_E2M1_E8M0_K32 && !strcmp(env, "1") && moe::gemm_pair_setup() == cudaSuccess);
  int want_disp = 0;
  if (const char* env = getenv("MOE_DISPATCH_CTAS")) want_disp = atoi(env);  // applied below, once created
  if (const char* env = getenv("MOE_TILE_N")) {
    const int v = atoi(env);
    if (v == 16 || v == 32 ||
        (v == 64 && wfmt != MOE_WFMT_NVFP4_E2M1_E4M3_K16 && wfmt != MOE_WFMT_MXFP4_W4A4) ||
        (v == 128 && wfmt == MOE_WFMT_FP8_E4M3_B128))
      c->tile_n_override = v;
    if (wfmt == MOE_WFMT_MXFP8_E4M3_E8M0_K32) c->tile_n_override = 0;  // 128-token tiles only
  }

  const size_t HB = H / 128, IB = I / 128;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  const size_t o_counts = take(sizeof(int32_t) * c->NG);
  const size_t o_offsets = take(sizeof(int32_t) * (c->NG + 1));
  const size_t o_perm = take(sizeof(int32_t) * c->P_max);
  const size_t o_inv = take(sizeof(int32_t) * c->P_max);
  const size_t o_ntiles = take(sizeof(int32_t) * 4);
  const size_t o_status = take(sizeof(int32_t) * 4);
  const size_t o_ready = take(sizeof(int32_t) * c->NG);
  const size_t o_tileoff = take(sizeof(int32_t) * (c->NG + 1));
  const size_t o_rpart = take(sizeof(int32_t) * moe::kMaxRouteParts * E);
  const bool mx8 = wfmt == MOE_WFMT_MXFP8_E4M3_E8M0_K32;
  c->max_tiles128 = c->P_max / 128 + c->NG + 1;
  const size_t o_xsf = mx8 ? take((size_t)c->max_tiles128 * HB * 512) : 0;
  const size_t o_hsf = mx8 ? take((size_t)c->max_tiles128 * IB * 512) : 0;
  const size_t o_tiles = take(sizeof(int4) * c->max_tiles);
  const size_t o_xq = take((size_t)c->S_pad * H);
  const size_t o_hq = take((size_t)c->S_pad * I);
  const size_t o_xs = take(sizeof(float) * (size_t)c->S_pad * HB);
  const size_t o_hs = take(sizeof(float) * (size_t)c->S_pad * IB);
  const size_t o_acc = take(sizeof(float) * (size_t)max_T * H);
  const bool a4 = wfmt == MOE_WFMT_NVFP4_E2M1_E4M3_K16 || wfmt == MOE_WFMT_MXFP4_W4A4;  // 4-bit activations
  const int code_step = (wfmt == MOE_WFMT_NVFP4_E2M1_E4M3_K16) ? 64 : 128;  // K columns per code entry
  const size_t o_xsc = a4 ? take((size_t)(H / code_step) * c->S_pad * 16) : 0;
  const size_t o_hsc = a4 ? take((size_t)(I / code_step) * c->S_pad * 16) : 0;
  const bool want_rows = c->combine_mode == 2;
  const size_t o_rows = want_rows ? take(sizeof(float) * (size_t)c->S_pad * H) : 0;
  // fused router workspace (E <= 256, E % 4 == 0): logits of every token tile
  const bool want_router = E <= 256 && E % 4 == 0;
  const size_t rt_tiles = ((size_t)max_T + 127) / 128;
  const size_t o_rt_logits = want_router ? take(sizeof(float) * rt_tiles * 128 * E) : 0;
  void* base = nullptr;
  if (cudaMalloc(&base, off) != cudaSuccess) {
    delete c;
    cudaGetLastError();
    return MOE_ERR_NO_MEMORY;
  }
  if (cudaMemset(base, 0, off) != cudaSuccess) {
    cudaFree(base);
    delete c;
    return MOE_ERR_CUDA;
  }
  char* b = static_cast<char*>(base);
  c->ws_base = base;
  c->counts = reinterpret_cast<int32_t*>(b + o_counts);
  c->offsets = reinterpret_cast<int32_t*>(b + o_offsets);
  c->perm = reinterpret_cast<int32_t*>(b + o_perm);
  c->inv = reinterpret_cast<int32_t*>(b + o_inv);
  c->num_tiles = reinterpret_cast<int32_t*>(b + o_ntiles);
  c->status = reinterpret_cast<int32_t*>(b + o_status);
  c->ready = reinterpret_cast<int32_t*>(b + o_ready);
  c->tile_off = reinterpret_cast<int32_t*>(b + o_tileoff);
  c->route_part = reinterpret_cast<int32_t*>(b + o_rpart);
  c->xsf = mx8 ? reinterpret_cast<uint8_t*>(b + o_xsf) : nullptr;
  c->hsf = mx8 ? reinterpret_cast<uint8_t*>(b + o_hsf) : nullptr;
  c->tiles = reinterpret_cast<int4*>(b + o_tiles);
  c->xq = reinterpret_cast<uint8_t*>(b + o_xq);
  c->hq = reinterpret_cast<uint8_t*>(b + o_hq);
  c->xs = reinterpret_cast<float*>(b + o_xs);
  c->hs = reinterpret_cast<float*>(b + o_hs);
  c->out_acc = reinterpret_cast<float*>(b + o_acc);
  c->xsc = a4 ? reinterpret_cast<uint8_t*>(b + o_xsc) : nullptr;
  c->hsc = a4 ? reinterpret_cast<uint8_t*>(b + o_hsc) : nullptr;
  if (a4 && (!make_map(&c->tm_xsc, CU_TENSOR_MAP_DATA_TYPE_UINT8, c->xsc, 16,
                       (uint64_t)(H / code_step) * c->S_pad, 16, 32, CU_TENSOR_MAP_L2_PROMOTION_L2_128B, 16,
                       CU_TENSOR_MAP_SWIZZLE_NONE) ||
             !make_map(&c->tm_hsc, CU_TENSOR_MAP_DATA_TYPE_UINT8, c->hsc, 16,
                       (uint64_t)(I / code_step) * c->S_pad, 16, 32, CU_TENSOR_MAP_L2_PROMOTION_L2_128B, 16,
                       CU_TENSOR_MAP_SWIZZLE_NONE))) {
    cudaFree(base);
    delete c;
    return MOE_ERR_CUDA;
  }
  if (c->pair_mma && !make_map(&c->tm_xq8, CU_TENSOR_MAP_DATA_TYPE_UINT8, c->xq, H, c->S_pad, H, 8,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_128B))
    c->pair_mma = 0;
  c->y_rows = want_rows ? reinterpret_cast<float*>(b + o_rows) : nullptr;
  c->rt_logits = want_router ? reinterpret_cast<float*>(b + o_rt_logits) : nullptr;
  if (want_router && moe::router_setup(E) != cudaSuccess) {
    cudaFree(base);
    delete c;
    return MOE_ERR_CUDA;
  }
  const int want_green = c->gc_sms;
  c->gc_sms = 0;
  if (want_green > 0) {
    const moe_status gs = moe_set_green_ctx(c, want_green);
    if (gs != MOE_OK) {
      moe_destroy(c);
      return gs;
    }
  }
  if (want_disp > 0) {
    const moe_status ds = moe_set_dispatch_overlap(c, want_disp);
    if (ds != MOE_OK) {
      moe_destroy(c);
      return ds;
    }
  }
  *out = c;
  return MOE_OK;
}

static void prof_free(moe_ctx* c) {
  if (!c->prof_ev) return;
  for (int i = 0; i < kProfMaxCalls * kProfEvents; ++i) cudaEventDestroy(c->prof_ev[i]);
  delete[] c->prof_ev;
  c->prof_ev = nullptr;
}

static void green_free(moe_ctx* c) {
  const GreenFns& g = green_fns();
  if (c->gs_small) g.stream_destroy(c->gs_small);
  if (c->gs_large) g.stream_destroy(c->gs_large);
  if (c->gc_small) g.destroy(c->gc_small);
  if (c->gc_large) g.destroy(c->gc_large);
  if (c->gev_in) cudaEventDestroy(c->gev_in);
  if (c->gev_disp) cudaEventDestroy(c->gev_disp);
  if (c->gev_done) cudaEventDestroy(c->gev_done);
  c->gs_small = c->gs_large = nullptr;
  c->gc_small = c->gc_large = nullptr;
  c->gev_in = c->gev_disp = c->gev_done = nullptr;
  c->gc_sms = c->gc_gemm_sms = 0;
}

moe_status moe_set_green_ctx(moe_ctx* c, int dispatch_sms) {
  if (!c || dispatch_sms < 0) return MOE_ERR_INVALID_ARG;
  if (dispatch_sms > 0 && c->disp_ctas) return MOE_ERR_UNSUPPORTED;  // dispatch overlap is the other form
  if (cudaDeviceSynchronize() != cudaSuccess) return MOE_ERR_CUDA;
  green_free(c);
  if (dispatch_sms == 0) return MOE_OK;
  const GreenFns& g = green_fns();
  if (!g.ok) return MOE_ERR_UNSUPPORTED;
  CUdevice dev;
  CUdevResource all = {}, small = {}, rest = {};
  unsigned int groups = 1;
  if (g.device_get(&dev, c->dev) != CUDA_SUCCESS ||
      g.get_dev_resource(dev, &all, CU_DEV_RESOURCE_TYPE_SM) != CUDA_SUCCESS ||
      g.split_by_count(&small, &groups, &all, &rest, 0, (unsigned int)dispatch_sms) != CUDA_SUCCESS || groups != 1)
    return MOE_ERR_UNSUPPORTED;
  if (small.sm.smCount == 0 || rest.sm.smCount < 8) return MOE_ERR_UNSUPPORTED;
  CUdevResourceDesc dsmall = nullptr, drest = nullptr;
  moe_status st = MOE_OK;
  if (g.generate_desc(&dsmall, &small, 1) != CUDA_SUCCESS || g.generate_desc(&drest, &rest, 1) != CUDA_SUCCESS ||
      g.create(&c->gc_small, dsmall, dev, CU_GREEN_CTX_DEFAULT_STREAM) != CUDA_SUCCESS ||
      g.create(&c->gc_large, drest, dev, CU_GREEN_CTX_DEFAULT_STREAM) != CUDA_SUCCESS ||
      g.stream_create(&c->gs_small, c->gc_small, CU_STREAM_NON_BLOCKING, 0) != CUDA_SUCCESS ||
      g.stream_create(&c->gs_large, c->gc_large, CU_STREAM_NON_BLOCKING, 0) != CUDA_SUCCESS)
    st = MOE_ERR_UNSUPPORTED;
  if (st == MOE_OK && (cudaEventCreateWithFlags(&c->gev_in, cudaEventDisableTiming) != cudaSuccess ||
                       cudaEventCreateWithFlags(&c->gev_disp, cudaEventDisableTiming) != cudaSuccess ||
                       cudaEventCreateWithFlags(&c->gev_done, cudaEventDisableTiming) != cudaSuccess))
    st = MOE_ERR_CUDA;
  if (st != MOE_OK) {
    green_free(c);
    return st;
  }
  c->gc_sms = (int)small.sm.smCount;
  c->gc_gemm_sms = (int)rest.sm.smCount;
  return MOE_OK;
}

moe_status moe_green_ctx_sms(moe_ctx* c, int* dispatch_sms, int* gemm_sms) {
  if (!c) return MOE_ERR_INVALID_ARG;
  if (dispatch_sms) *dispatch_sms = c->gc_sms;
  if (gemm_sms) *gemm_sms = c->gc_gemm_sms;
  return MOE_OK;
}

void moe_destroy(moe_ctx* c) {
  if (!c) return;
  cudaDeviceSynchronize();
  green_free(c);
  prof_free(c);
  cudaFree(c->ws_base);
  delete c;
}

// The launch sequence of one layer for every weight format; g13 / g2 are the
// NVFP4 global scales (null for the other formats).  With partial_out the
// fp32 combine result goes to that caller buffer (GEMM2 reduces into it) and
// no bf16 output is written (out is ignored).
static moe_status forward_impl(moe_ctx* c, int T, const void* x, const int32_t* ids, const float* topk_w,
                               const void* w13, const void* s13, const float* g13, const void* w2, const void* s2,
                               const float* g2, void* out, void* stream, float* partial_out = nullptr) {
  if (!c || T < 0 || T > c->max_T) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  const bool partial = partial_out != nullptr;
  if (!x || !ids || !topk_w || !w13 || !s13 || !w2 || !s2 || (!out && !partial)) return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || (!partial && !aligned(out, 16)) || (partial && !aligned(partial_out, 16)) ||
      !aligned(w13, 128) || !aligned(w2, 128) || !aligned(s13, 16) || !aligned(s2, 16) || !aligned(ids, 4) ||
      !aligned(topk_w, 4))
    return MOE_ERR_INVALID_ARG;
  const bool nvfp4 = (c->wfmt == MOE_WFMT_NVFP4_E2M1_E4M3_K16);
  const bool a4 = nvfp4 || c->wfmt == MOE_WFMT_MXFP4_W4A4;  // 4-bit activations, packed operands
  if (nvfp4 && (!g13 || !g2 || !aligned(g13, 4) || !aligned(g2, 4))) return MOE_ERR_INVALID_ARG;
  if (c->wfmt != MOE_WFMT_FP8_E4M3_B128) {
    // 4-bit weights read their block scales in the packed layout only; plain
    // scales would give wrong results without any error, so refuse scale
    // buffers that no pack call wrote (or moe_declare_packed_scales declared)
    const int sf = nvfp4 ? MOE_WFMT_NVFP4_E2M1_E4M3_K16 : MOE_WFMT_MXFP4_E2M1_E8M0_K32;
    if (!moe::packed_scales_known(s13, packed_bytes(sf, c->NG, 2 * c->I, c->H), sf) ||
        !moe::packed_scales_known(s2, packed_bytes(sf, c->NG, c->H, c->I), sf))
      return MOE_ERR_INVALID_ARG;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int H = c->H, I = c->I, NE = c->NG;
  const int S = T * c->k;
  const int BN = pick_tile_n(c, T);
  // Green-Context partition: route + quant on the small partition's stream,
  // GEMMs + output on the large one, ordered by events after the caller's
  // stream and before its next work.  Otherwise everything runs on `s`.
  const bool green = c->gc_small != nullptr;
  cudaStream_t s_disp = green ? reinterpret_cast<cudaStream_t>(c->gs_small) : s;
  cudaStream_t s_gemm = green ? reinterpret_cast<cudaStream_t>(c->gs_large) : s;
  const int grid = green ? c->gc_gemm_sms : c->num_sms;
  const bool mx8 = (c->wfmt == MOE_WFMT_MXFP8_E4M3_E8M0_K32);
  const bool fp8 = (c->wfmt == MOE_WFMT_FP8_E4M3_B128) || mx8;  // one byte per weight

  // weight maps (re-encoded only when the caller's pointers change)
  const CUtensorMapL2promotion wpromo = CU_TENSOR_MAP_L2_PROMOTION_L2_256B;
  // NVFP4: packed bytes [rows, K/2], boxes of 64 bytes (one 128-wide K
  // block) x 128 rows with 64-byte swizzle
  constexpr CUtensorMapSwizzle sw64 = CU_TENSOR_MAP_SWIZZLE_64B;
  if (w13 != c->c_w13) {
    const bool ok = fp8 ? make_map(&c->tm_w13, CU_TENSOR_MAP_DATA_TYPE_UINT8, w13, H, (uint64_t)NE * 2 * I, H, 128,
                                   wpromo)
                    : a4 ? make_map(&c->tm_w13, CU_TENSOR_MAP_DATA_TYPE_UINT8, w13, H / 2, (uint64_t)NE * 2 * I,
                                       H / 2, 128, wpromo, 64, sw64)
                        : make_map(&c->tm_w13, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, w13, H, (uint64_t)NE * 2 * I,
                                   H / 2, 128, wpromo);
    if (!ok) {
      c->c_w13 = nullptr;
      return MOE_ERR_CUDA;
    }
    c->c_w13 = w13;
  }
  if (w2 != c->c_w2) {
    const bool ok = fp8 ? make_map(&c->tm_w2, CU_TENSOR_MAP_DATA_TYPE_UINT8, w2, I, (uint64_t)NE * H, I, 128,
                                   wpromo)
                    : a4 ? make_map(&c->tm_w2, CU_TENSOR_MAP_DATA_TYPE_UINT8, w2, I / 2, (uint64_t)NE * H, I / 2,
                                       128, wpromo, 64, sw64)
                        : make_map(&c->tm_w2, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, w2, I, (uint64_t)NE * H, I / 2,
                                   128, wpromo);
    if (!ok) {
      c->c_w2 = nullptr;
      return MOE_ERR_CUDA;
    }
    c->c_w2 = w2;
  }
  if (BN != c->c_bn) {
    const bool ok = a4
        ? make_map(&c->tm_xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, c->xq, H / 2, c->S_pad, H / 2, BN,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_128B, 64, sw64) &&
              make_map(&c->tm_hq, CU_TENSOR_MAP_DATA_TYPE_UINT8, c->hq, I / 2, c->S_pad, I / 2, BN,
                       CU_TENSOR_MAP_L2_PROMOTION_L2_128B, 64, sw64)
        : make_map(&c->tm_xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, c->xq, H, c->S_pad, H, BN,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_128B) &&
              make_map(&c->tm_hq, CU_TENSOR_MAP_DATA_TYPE_UINT8, c->hq, I, c->S_pad, I, BN,
                       CU_TENSOR_MAP_L2_PROMOTION_L2_128B);
    if (!ok) {
      c->c_bn = 0;
      return MOE_ERR_CUDA;
    }
    c->c_bn = BN;
  }

  cudaEvent_t* ev = nullptr;
  if (c->prof_on && c->prof_calls < kProfMaxCalls) ev = c->prof_ev + (size_t)c->prof_calls++ * kProfEvents;
  auto mark = [&](int i) {
    if (ev) cudaEventRecord(ev[i], i <= MOE_STAGE_QUANT ? s_disp : s_gemm);
  };
  if (green) {
    if (cudaEventRecord(c->gev_in, s) != cudaSuccess || cudaStreamWaitEvent(s_disp, c->gev_in, 0) != cudaSuccess)
      return MOE_ERR_CUDA;
  }

  // Dispatch overlap: no quantisation kernel; the GEMM1 launch quantises in
  // its last disp_ctas CTAs and publishes per-group ready counters.
  const bool overlap = c->disp_ctas > 0 && !green && !a4;
  RouteParams rp{};
  rp.T = T; rp.k = c->k; rp.E = c->E; rp.n_shared = c->n_shared; rp.BN = BN;
  rp.ids = ids; rp.counts = c->counts; rp.offsets = c->offsets; rp.perm = c->perm; rp.inv = c->inv;
  rp.tiles = c->tiles; rp.num_tiles = c->num_tiles; rp.status = c->status;
  rp.ready = overlap ? c->ready : nullptr;
  rp.tile_off = mx8 ? c->tile_off : nullptr;
  rp.part = c->route_part;
  mark(MOE_STAGE_ROUTE);
  if (moe::launch_route(rp, s_disp) != cudaSuccess) return MOE_ERR_CUDA;

  const bool rows = c->y_rows != nullptr && !partial;  // a partial sum always uses the fused combine
  float* acc = partial ? partial_out : c->out_acc;

  QuantParams qp{};
  qp.T = T; qp.H = H; qp.k = c->k; qp.n_shared = c->n_shared;
  qp.x = static_cast<const uint16_t*>(x); qp.inv = c->inv; qp.xq = c->xq; qp.xs = c->xs;
  qp.xs_ld = c->S_pad;
  qp.out_acc = rows ? nullptr : acc;
  qp.xsc = c->xsc;
  qp.sf_atoms = c->xsf; qp.ids = ids; qp.offsets = c->offsets; qp.tile_off = c->tile_off; qp.E = c->E;
  qp.pdl = moe::quant_pdl(T, c->k, c->E, c->n_shared, H, I);
  mark(MOE_STAGE_QUANT);
  if (!overlap) {
    const cudaError_t qe = nvfp4 ? moe::launch_quant_nvfp4(qp, s_disp)
                           : a4  ? moe::launch_quant_mxfp4(qp, s_disp)
                           : mx8 ? moe::launch_quant_mxfp8(qp, s_disp)
                                 : moe::launch_quant(qp, s_disp);
    if (qe != cudaSuccess) return MOE_ERR_CUDA;
  }
  if (green) {
    if (cudaEventRecord(c->gev_disp, s_disp) != cudaSuccess || cudaStreamWaitEvent(s_gemm, c->gev_disp, 0) != cudaSuccess)
      return MOE_ERR_CUDA;
  }

  GemmParams g{};
  g.H = H; g.I = I; g.k = c->k; g.S = S;
  g.kblocks = H / 128;
  g.wscale = static_cast<const float*>(s13);
  g.ascale = c->xs;
  g.scale_ld = c->S_pad;
  g.hq = c->hq; g.hs = c->hs;
  g.perm = c->perm; g.topk_w = topk_w; g.out_acc = acc;
  g.tiles = c->tiles; g.num_tiles = c->num_tiles; g.status = c->status;
  g.y_rows = nullptr;
  g.inject = c->inject;
  g.wglobal = g13;
  g.hsc = c->hsc;
  // the token block-code maps exist for 4-bit activations only; the other formats ignore the argument
  const CUtensorMap& tsx = a4 ? c->tm_xsc : c->tm_xq;
  const CUtensorMap& tsh = a4 ? c->tm_hsc : c->tm_hq;
  if (overlap) {
    g.disp = c->disp_ctas;
    g.ready = c->ready; g.counts = c->counts; g.offsets = c->offsets;
    g.x = static_cast<const uint16_t*>(x); g.xq = c->xq; g.xs = c->xs;
    g.zero_acc = rows ? nullptr : acc;
    g.T = T; g.NG = c->NG;
  }
  mark(MOE_STAGE_GEMM1);
  const bool pair = c->pair_mma && BN == 16 && !overlap && !green;
  if (pair && s13 != c->c_s13) {
    // the packed scales as rows of 256 bytes: atom (row / 128, K block) = rows 2a, 2a + 1
    const uint64_t atoms = (uint64_t)(c->E + c->n_shared) * (2 * I / 128) * (H / 128);
    if (!make_map(&c->tm_s13, CU_TENSOR_MAP_DATA_TYPE_UINT8, s13, 256, 2 * atoms, 256, 2,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, 256, CU_TENSOR_MAP_SWIZZLE_NONE)) {
      c->c_s13 = nullptr;
      return MOE_ERR_CUDA;
    }
    c->c_s13 = s13;
  }
  if (mx8) {
    g.act_sf = c->xsf;
    g.hsc = c->hsf;
    if (moe::launch_gemm1_tmx(grid, c->tm_w13, c->tm_xq, g, s_gemm) != cudaSuccess) return MOE_ERR_CUDA;
  } else if (pair) {
    if (moe::launch_gemm1_pair(c->tm_w13, c->tm_xq8, c->tm_s13, g, s_gemm) != cudaSuccess) return MOE_ERR_CUDA;
  } else if (moe::launch_gemm1(c->wfmt, BN, grid, c->tm_w13, c->tm_xq, tsx, g, s_gemm) != cudaSuccess) {
    return MOE_ERR_CUDA;
  }

  g.disp = 0;  // GEMM2 reads GEMM1's outputs after the kernel boundary
  g.zero_acc = nullptr;
  g.kblocks = I / 128;
  g.wscale = static_cast<const float*>(s2);
  g.wglobal = g2;
  g.ascale = c->hs;
  mark(MOE_STAGE_GEMM2);
  g.y_rows = rows ? c->y_rows : nullptr;
  if (mx8) {
    g.act_sf = c->hsf;
    if (moe::launch_gemm2_tmx(grid, c->tm_w2, c->tm_hq, g, s_gemm) != cudaSuccess) return MOE_ERR_CUDA;
  } else if (moe::launch_gemm2(c->wfmt, BN, grid, c->tm_w2, c->tm_hq, tsh, g, s_gemm) != cudaSuccess) {
    return MOE_ERR_CUDA;
  }

  mark(MOE_STAGE_FINALIZE);
  if (partial) {
    // the caller sums the partials (e.g. across tensor-parallel ranks) and
    // converts them with moe_finalize_bf16
  } else if (rows) {
    moe::CombineParams cp;
    cp.T = T; cp.H = H; cp.k = c->k; cp.n_shared = c->n_shared;
    cp.y_rows = c->y_rows; cp.inv = c->inv; cp.topk_w = topk_w; cp.out = static_cast<uint16_t*>(out);
    if (moe::launch_combine(cp, s_gemm) != cudaSuccess) return MOE_ERR_CUDA;
  } else if (moe::launch_finalize(c->out_acc, static_cast<uint16_t*>(out), (long long)T * H, s_gemm) != cudaSuccess) {
    return MOE_ERR_CUDA;
  }
  mark(MOE_NUM_STAGES);
  if (green) {
    if (cudaEventRecord(c->gev_done, s_gemm) != cudaSuccess || cudaStreamWaitEvent(s, c->gev_done, 0) != cudaSuccess)
      return MOE_ERR_CUDA;
  }
  c->last_T = T;
  c->last_bn = BN;
  c->last_grid = grid;
  return MOE_OK;
}

moe_status moe_forward(moe_ctx* c, int T, const void* x, const int32_t* ids, const float* topk_w, const void* w13,
                       const void* s13, const void* w2, const void* s2, void* out, void* stream) {
  if (c && c->wfmt == MOE_WFMT_NVFP4_E2M1_E4M3_K16) return MOE_ERR_INVALID_ARG;  // needs moe_forward_nvfp4
  return forward_impl(c, T, x, ids, topk_w, w13, s13, nullptr, w2, s2, nullptr, out, stream);
}

moe_status moe_forward_partial(moe_ctx* c, int T, const void* x, const int32_t* ids, const float* topk_w,
                               const void* w13, const void* s13, const float* g13, const void* w2, const void* s2,
                               const float* g2, float* out_f32, void* stream) {
  if (!out_f32) return MOE_ERR_INVALID_ARG;
  return forward_impl(c, T, x, ids, topk_w, w13, s13, g13, w2, s2, g2, nullptr, stream, out_f32);
}

moe_status moe_finalize_bf16(const float* in, void* out, long long n, void* stream) {
  if (n < 0 || n % 4) return MOE_ERR_INVALID_ARG;
  if (n == 0) return MOE_OK;
  if (!in || !out || !aligned(in, 16) || !aligned(out, 8)) return MOE_ERR_INVALID_ARG;
  if (moe::launch_finalize(in, static_cast<uint16_t*>(out), n, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

}  // extern "C"

namespace moe {
bool packed_scales_known(const void* p, size_t bytes, int fmt) {
  const uintptr_t lo = reinterpret_cast<uintptr_t>(p);
  std::lock_guard<std::mutex> lock(g_packed_mu);
  auto it = g_packed.upper_bound(lo);
  if (it == g_packed.begin()) return false;
  --it;
  return it->second.second == fmt && lo + bytes <= it->second.first;
}
}  // namespace moe

extern "C" {

moe_status moe_forward_nvfp4(moe_ctx* c, int T, const void* x, const int32_t* ids, const float* topk_w,
                             const void* w13, const void* s13, const float* g13, const void* w2, const void* s2,
                             const float* g2, void* out, void* stream) {
  if (!c || c->wfmt != MOE_WFMT_NVFP4_E2M1_E4M3_K16) return MOE_ERR_INVALID_ARG;
  return forward_impl(c, T, x, ids, topk_w, w13, s13, g13, w2, s2, g2, out, stream);
}

moe_status moe_router_topk(moe_ctx* c, int T, const void* x, const void* wr, int32_t* topk_ids, float* topk_w,
                           void* stream) {
  if (!c || T < 0 || T > c->max_T) return MOE_ERR_INVALID_ARG;
  if (!c->rt_logits) return MOE_ERR_UNSUPPORTED;  // E > 256 or E % 4 != 0
  if (T == 0) return MOE_OK;
  if (!x || !wr || !topk_ids || !topk_w || !aligned(x, 16) || !aligned(wr, 16) || !aligned(topk_ids, 4) ||
      !aligned(topk_w, 4))
    return MOE_ERR_INVALID_ARG;
  const int H = c->H, E = c->E;
  const int NP = (E + 15) / 16 * 16;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  CUtensorMap tx;
  if (!make_map(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, H, (uint64_t)T, (uint64_t)H * 2, 128,
                CU_TENSOR_MAP_L2_PROMOTION_L2_128B, 64))
    return MOE_ERR_CUDA;
  if (wr != c->c_wr) {
    if (!make_map(&c->tm_wr, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, wr, H, (uint64_t)E, (uint64_t)H * 2, NP,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_128B, 64)) {
      c->c_wr = nullptr;
      return MOE_ERR_CUDA;
    }
    c->c_wr = wr;
  }
  moe::RouterParams rp;
  rp.T = T; rp.H = H; rp.E = E; rp.k = c->k; rp.N = NP;
  rp.kblocks = H / 64;
  const int tiles = (T + 127) / 128;
  // K splits fill the GPU, but keep at least 8 K blocks per split: every
  // split adds its partial logits into the same rows with fp32 reductions.
  int splits = c->num_sms / tiles;
  if (splits > rp.kblocks / 8) splits = rp.kblocks / 8;
  if (splits < 1) splits = 1;
  rp.splits = splits;
  rp.wbox_rows = NP;
  rp.tmem_cols = NP <= 32 ? 32 : NP <= 64 ? 64 : NP <= 128 ? 128 : 256;
  rp.logits = c->rt_logits;
  rp.ids = topk_ids; rp.w = topk_w; rp.status = c->status;
  if (moe::launch_router(tx, c->tm_wr, rp, s) != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}

moe_status moe_pack_mxfp4_scales(const uint8_t* src, uint8_t* dst, int rows, int K, void* stream) {
  if (!src || !dst || src == dst || rows <= 0 || K <= 0 || rows % 128 || K % 128) return MOE_ERR_INVALID_ARG;
  if (moe::launch_pack_e8m0(src, dst, rows, K / 32, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return MOE_ERR_CUDA;
  register_packed(dst, (size_t)rows * (K / 32), MOE_WFMT_MXFP4_E2M1_E8M0_K32);
  return MOE_OK;
}

moe_status moe_pack_nvfp4_scales(const uint8_t* src, uint8_t* dst, int rows, int K, void* stream) {
  if (!src || !dst || src == dst || rows <= 0 || K <= 0 || rows % 128 || K % 128) return MOE_ERR_INVALID_ARG;
  if (moe::launch_pack_e8m0(src, dst, rows, K / 16, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return MOE_ERR_CUDA;
  register_packed(dst, (size_t)rows * (K / 16), MOE_WFMT_NVFP4_E2M1_E4M3_K16);
  return MOE_OK;
}

moe_status moe_declare_packed_scales(const void* p, long long bytes, int wfmt) {
  if (!p || bytes <= 0) return MOE_ERR_INVALID_ARG;
  if (wfmt == MOE_WFMT_MXFP4_W4A4 || wfmt == MOE_WFMT_MXFP8_E4M3_E8M0_K32)
    wfmt = MOE_WFMT_MXFP4_E2M1_E8M0_K32;  // the same E8M0 atoms
  if (wfmt != MOE_WFMT_MXFP4_E2M1_E8M0_K32 && wfmt != MOE_WFMT_NVFP4_E2M1_E4M3_K16) return MOE_ERR_INVALID_ARG;
  register_packed(p, (size_t)bytes, wfmt);
  return MOE_OK;
}

moe_status moe_get_routing(moe_ctx* c, int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* inv,
                           void* stream) {
  if (!c) return MOE_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return MOE_ERR_CUDA;
  const size_t P = (size_t)c->last_T * c->k + (size_t)c->n_shared * c->last_T;
  cudaError_t e = cudaSuccess;
  if (counts && e == cudaSuccess) e = cudaMemcpy(counts, c->counts, sizeof(int32_t) * c->NG, cudaMemcpyDefault);
  if (offsets && e == cudaSuccess)
    e = cudaMemcpy(offsets, c->offsets, sizeof(int32_t) * (c->NG + 1), cudaMemcpyDefault);
  if (perm && P && e == cudaSuccess) e = cudaMemcpy(perm, c->perm, sizeof(int32_t) * P, cudaMemcpyDefault);
  if (inv && P && e == cudaSuccess) e = cudaMemcpy(inv, c->inv, sizeof(int32_t) * P, cudaMemcpyDefault);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status moe_get_activations(moe_ctx* c, uint8_t* xq, float* xs, uint8_t* hq, float* hs, void* stream) {
  if (!c) return MOE_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return MOE_ERR_CUDA;
  const size_t P = (size_t)c->last_T * c->k + (size_t)c->n_shared * c->last_T;
  cudaError_t e = cudaSuccess;
  const size_t cw = (c->wfmt == MOE_WFMT_NVFP4_E2M1_E4M3_K16 || c->wfmt == MOE_WFMT_MXFP4_W4A4) ? 2 : 1;  // codes per byte
  if (xq && P && e == cudaSuccess) e = cudaMemcpy(xq, c->xq, P * c->H / cw, cudaMemcpyDefault);
  if (hq && P && e == cudaSuccess) e = cudaMemcpy(hq, c->hq, P * c->I / cw, cudaMemcpyDefault);
  // The scales are stored K-block major on the device ([K/128][S_pad]); the
  // caller gets them position major ([P][K/128]).
  auto scales = [&](float* dst, const float* src, int kb) {
    if (!dst || !P || e != cudaSuccess) return;
    float* tmp = new (std::nothrow) float[(size_t)kb * P];
    if (!tmp) {
      e = cudaErrorMemoryAllocation;
      return;
    }
    e = cudaMemcpy2D(tmp, P * sizeof(float), src, (size_t)c->S_pad * sizeof(float), P * sizeof(float), kb,
                     cudaMemcpyDeviceToHost);
    if (e == cudaSuccess) {
      float* stage = new (std::nothrow) float[(size_t)kb * P];
      if (!stage) {
        e = cudaErrorMemoryAllocation;
      } else {
        for (size_t i = 0; i < P; ++i)
          for (int b = 0; b < kb; ++b) stage[i * kb + b] = tmp[(size_t)b * P + i];
        e = cudaMemcpy(dst, stage, sizeof(float) * kb * P, cudaMemcpyDefault);
        delete[] stage;
      }
    }
    delete[] tmp;
  };
  scales(xs, c->xs, c->H / 128);
  scales(hs, c->hs, c->I / 128);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// MXFP8: the E8M0 codes of the last call's activations, gathered from the
// per-tile scale atoms into [P][K/32] rows in routing-position order.
static moe_status get_block_scales_mxfp8(moe_ctx* c, uint8_t* xsc, uint8_t* hsc, void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return MOE_ERR_CUDA;
  const int NG = c->NG;
  const size_t P = (size_t)c->last_T * c->k + (size_t)c->n_shared * c->last_T;
  if (!P) return MOE_OK;
  int32_t* off = new (std::nothrow) int32_t[NG + 1];
  int32_t* toff = new (std::nothrow) int32_t[NG + 1];
  moe_status st = (off && toff) ? MOE_OK : MOE_ERR_NO_MEMORY;
  if (st == MOE_OK && (cudaMemcpy(off, c->offsets, sizeof(int32_t) * (NG + 1), cudaMemcpyDeviceToHost) != cudaSuccess ||
                       cudaMemcpy(toff, c->tile_off, sizeof(int32_t) * (NG + 1), cudaMemcpyDeviceToHost) != cudaSuccess))
    st = MOE_ERR_CUDA;
  auto gather = [&](uint8_t* dst, const uint8_t* atoms, int K) {
    if (!dst || st != MOE_OK) return;
    const int KB = K / 128;
    const size_t nt = (size_t)toff[NG];
    uint8_t* a = new (std::nothrow) uint8_t[nt * KB * 512 + 1];
    uint8_t* out = new (std::nothrow) uint8_t[P * (K / 32)];
    if (!a || !out) {
      st = MOE_ERR_NO_MEMORY;
    } else if (cudaMemcpy(a, atoms, nt * KB * 512, cudaMemcpyDeviceToHost) != cudaSuccess) {
      st = MOE_ERR_CUDA;
    } else {
      memset(out, 0, P * (K / 32));
      int g = 0;
      for (size_t pos = 0; pos < (size_t)off[NG]; ++pos) {
        while ((int)pos >= off[g + 1]) ++g;
        const int within = (int)pos - off[g];
        const int ti = toff[g] + within / 128, r = within % 128;
        for (int kb = 0; kb < KB; ++kb)
          for (int j = 0; j < 4; ++j)
            out[pos * (K / 32) + kb * 4 + j] = a[((size_t)ti * KB + kb) * 512 + (r % 32) * 16 + (r / 32) * 4 + j];
      }
      if (cudaMemcpy(dst, out, P * (K / 32), cudaMemcpyDefault) != cudaSuccess) st = MOE_ERR_CUDA;
    }
    delete[] a;
    delete[] out;
  };
  gather(xsc, c->xsf, c->H);
  gather(hsc, c->hsf, c->I);
  delete[] off;
  delete[] toff;
  return st;
}

moe_status moe_get_block_scales(moe_ctx* c, uint8_t* xsc, uint8_t* hsc, void* stream) {
  if (!c) return MOE_ERR_INVALID_ARG;
  if (c->wfmt == MOE_WFMT_MXFP8_E4M3_E8M0_K32) return get_block_scales_mxfp8(c, xsc, hsc, stream);
  if (c->wfmt != MOE_WFMT_NVFP4_E2M1_E4M3_K16 && c->wfmt != MOE_WFMT_MXFP4_W4A4) return MOE_ERR_UNSUPPORTED;
  const int code_step = (c->wfmt == MOE_WFMT_NVFP4_E2M1_E4M3_K16) ? 64 : 128;  // K columns per 4-code entry
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return MOE_ERR_CUDA;
  const size_t P = (size_t)c->last_T * c->k + (size_t)c->n_shared * c->last_T;
  cudaError_t e = cudaSuccess;
  // device [K/code_step][S_pad][16] (four codes per entry and position) ->
  // caller [P][4 K/code_step] (NVFP4 [P][K/16], MXFP4 [P][K/32])
  auto gather = [&](uint8_t* dst, const uint8_t* src, int K) {
    if (!dst || !P || e != cudaSuccess) return;
    const size_t steps = (size_t)K / code_step;
    uint8_t* tmp = new (std::nothrow) uint8_t[steps * P * 4];
    uint8_t* out = new (std::nothrow) uint8_t[steps * P * 4];
    if (!tmp || !out) {
      e = cudaErrorMemoryAllocation;
    } else {
      for (size_t st = 0; st < steps && e == cudaSuccess; ++st)
        e = cudaMemcpy2D(tmp + st * P * 4, 4, src + st * c->S_pad * 16, 16, 4, P, cudaMemcpyDeviceToHost);
      if (e == cudaSuccess) {
        for (size_t i = 0; i < P; ++i)
          for (size_t st = 0; st < steps; ++st) memcpy(out + (i * steps + st) * 4, tmp + (st * P + i) * 4, 4);
        e = cudaMemcpy(dst, out, steps * P * 4, cudaMemcpyDefault);
      }
    }
    delete[] tmp;
    delete[] out;
  };
  gather(xsc, c->xsc, c->H);
  gather(hsc, c->hsc, c->I);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status moe_get_device_status(moe_ctx* c, void* stream) {
  if (!c) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  int32_t v = 0;
  if (cudaMemcpy(&v, c->status, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaMemset(c->status, 0, sizeof(int32_t)) != cudaSuccess) return MOE_ERR_CUDA;
  if (v & moe::DEV_TIMEOUT) return MOE_ERR_TIMEOUT;
  if (v & moe::DEV_BAD_ROUTING) return MOE_ERR_BAD_ROUTING;
  return MOE_OK;
}

moe_status moe_profile_enable(moe_ctx* c, int on) {
  if (!c) return MOE_ERR_INVALID_ARG;
  if (on && !c->prof_ev) {
    c->prof_ev = new (std::nothrow) cudaEvent_t[kProfMaxCalls * kProfEvents];
    if (!c->prof_ev) return MOE_ERR_NO_MEMORY;
    for (int i = 0; i < kProfMaxCalls * kProfEvents; ++i) {
      if (cudaEventCreate(&c->prof_ev[i]) != cudaSuccess) {
        for (int j = 0; j < i; ++j) cudaEventDestroy(c->prof_ev[j]);
        delete[] c->prof_ev;
        c->prof_ev = nullptr;
        return MOE_ERR_CUDA;
      }
    }
  }
  if (!on) prof_free(c);
  c->prof_on = on ? 1 : 0;
  c->prof_calls = 0;
  return MOE_OK;
}

moe_status moe_profile_read(moe_ctx* c, float* avg_ms, int* calls) {
  if (!c || !avg_ms) return MOE_ERR_INVALID_ARG;
  double sum[MOE_NUM_STAGES] = {0};
  const int n = c->prof_calls;
  for (int i = 0; i < n; ++i) {
    cudaEvent_t* ev = c->prof_ev + (size_t)i * kProfEvents;
    if (cudaEventSynchronize(ev[MOE_NUM_STAGES]) != cudaSuccess) return MOE_ERR_CUDA;
    for (int st = 0; st < MOE_NUM_STAGES; ++st) {
      float ms = 0.0f;
      if (cudaEventElapsedTime(&ms, ev[st], ev[st + 1]) != cudaSuccess) return MOE_ERR_CUDA;
      sum[st] += ms;
    }
  }
  for (int st = 0; st < MOE_NUM_STAGES; ++st) avg_ms[st] = n ? (float)(sum[st] / n) : 0.0f;
  if (calls) *calls = n;
  c->prof_calls = 0;
  return MOE_OK;
}

moe_status moe_set_dispatch_overlap(moe_ctx* c, int dispatch_ctas) {
  if (!c || dispatch_ctas < 0 || dispatch_ctas > c->num_sms) return MOE_ERR_INVALID_ARG;
  if (dispatch_ctas == 0) {
    c->disp_ctas = 0;
    return MOE_OK;
  }
  // FP8 activations only (the two formats whose step 2 is the FP8 quantiser)
  if (c->wfmt != MOE_WFMT_FP8_E4M3_B128 && c->wfmt != MOE_WFMT_MXFP4_E2M1_E8M0_K32) return MOE_ERR_UNSUPPORTED;
  if (c->gc_small) return MOE_ERR_UNSUPPORTED;  // the Green-Context partition is the other form of the split
  int coop = 0;
  if (cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, c->dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (!coop) return MOE_ERR_UNSUPPORTED;
  c->disp_ctas = dispatch_ctas;
  return MOE_OK;
}

moe_status moe_dispatch_overlap_ctas(moe_ctx* c, int* dispatch_ctas) {
  if (!c || !dispatch_ctas) return MOE_ERR_INVALID_ARG;
  *dispatch_ctas = c->disp_ctas;
  return MOE_OK;
}

moe_status moe_set_fault_injection(moe_ctx* c, int mode) {
  if (!c || mode < 0 || mode > 2) return MOE_ERR_INVALID_ARG;
  c->inject = mode;
  return MOE_OK;
}

moe_status moe_last_config(moe_ctx* c, int* tile_n, int* grid) {
  if (!c) return MOE_ERR_INVALID_ARG;
  if (tile_n) *tile_n = c->last_bn;
  if (grid) *grid = c->last_grid;
  return MOE_OK;
}

}  // extern "C"
