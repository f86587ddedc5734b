// moe_noalloc.cu -- moe_forward_noalloc(): the MoE layer without any device
// allocation, for callers that cannot call cudaMalloc (for example code that
// runs inside a host framework which owns every device allocation, or while
// a memory pool is locked).  The layer's scratch (routing arrays, tile list, quantised
// activations, fp32 combine buffer, status word) lives in one file-scope
// device array of fixed size instead of a context's workspace.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <mutex>

#include "moe.h"
#include "moe_internal.h"
#include "moe_ptx.cuh"

namespace {

// The array every GPU that loads the library holds until process exit.
static __device__ __align__(256) unsigned char g_noalloc_scratch[MOE_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
// Device address of g_noalloc_scratch and SM count per device, written once
// by the first call on that device under g_setup_mu and published by the
// release store of g_setup_done[dev]; later calls read them after an acquire
// load of that flag, so concurrent first calls from several host threads are
// safe.
void* g_scratch_addr[kMaxDevices] = {nullptr};
int g_num_sms[kMaxDevices] = {0};
std::atomic<bool> g_setup_done[kMaxDevices];
std::mutex g_setup_mu;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn lookup_encoder() {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    return reinterpret_cast<EncodeTiledFn>(p);
  return nullptr;
}

EncodeTiledFn encoder() {
  static const EncodeTiledFn fn = lookup_encoder();  // initialised once, thread-safe
  return fn;
}

// One-time set-up on device `dev`, which is current: the array's device
// address, the SM count and the kernels' shared-memory limits.  Returns
// MOE_OK once done; on failure nothing is published and the next call
// tries again.
moe_status setup_device(int dev) {
  if (g_setup_done[dev].load(std::memory_order_acquire)) return MOE_OK;
  std::lock_guard<std::mutex> lock(g_setup_mu);
  if (g_setup_done[dev].load(std::memory_order_relaxed)) return MOE_OK;
  int major = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (major != 10) return MOE_ERR_UNSUPPORTED;
  void* addr = nullptr;
  if (cudaGetSymbolAddress(&addr, g_noalloc_scratch) != cudaSuccess || !addr) return MOE_ERR_CUDA;
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (moe::gemm_setup(MOE_WFMT_FP8_E4M3_B128) != cudaSuccess ||
      moe::gemm_setup(MOE_WFMT_MXFP4_E2M1_E8M0_K32) != cudaSuccess)
    return MOE_ERR_CUDA;
  g_scratch_addr[dev] = addr;
  g_num_sms[dev] = sms;
  g_setup_done[dev].store(true, std::memory_order_release);
  return MOE_OK;
}

bool map2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t rows,
           uint64_t row_bytes, uint32_t box_rows, CUtensorMapL2promotion l2) {
  EncodeTiledFn fn = encoder();
  if (!fn) return false;
  cuuint64_t gdim[2] = {inner, rows};
  cuuint64_t gstride[1] = {row_bytes};
  cuuint32_t box[2] = {128, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void*>(base), gdim, gstride, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, l2, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t up256(size_t v) { return (v + 255) / 256 * 256; }

struct Carve {
  size_t counts, offsets, perm, inv, ntiles, status, tiles, xq, hq, xs, hs, acc, total;
};

Carve carve(int H, int I, int E, int k, int n_shared, int T) {
  const size_t NG = (size_t)E + n_shared;
  const size_t P = (size_t)T * k + (size_t)n_shared * T;
  const size_t S_pad = P + 128;
  const size_t tiles = P / 16 + NG + 1;
  Carve c;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = up256(off + bytes);
    return o;
  };
  c.counts = take(4 * NG);
  c.offsets = take(4 * (NG + 1));
  c.perm = take(4 * P);
  c.inv = take(4 * P);
  c.ntiles = take(16);
  c.status = take(16);
  c.tiles = take(sizeof(int4) * tiles);
  c.xq = take(S_pad * H);
  c.hq = take(S_pad * I);
  c.xs = take(4 * S_pad * (H / 128));
  c.hs = take(4 * S_pad * (I / 128));
  c.acc = take(4 * (size_t)T * H);
  c.total = off;
  return c;
}

}  // namespace

extern "C" moe_status moe_forward_noalloc(int H, int I, int E, int k, int wfmt, int n_shared, int T, const void* x,
                                          const int32_t* topk_ids, const float* topk_w, const void* w13,
                                          const void* s13, const void* w2, const void* s2, void* out,
                                          int32_t* d_status, void* stream) {
  if (H <= 0 || I <= 0 || E <= 0 || k <= 0 || T < 0 || n_shared < 0) return MOE_ERR_INVALID_ARG;
  if (H % 128 || I % 128 || H > 8192 || I > 8192 || E > 1024 || k > moe::kMaxK || n_shared > 1)
    return MOE_ERR_UNSUPPORTED;
  if (wfmt != MOE_WFMT_FP8_E4M3_B128 && wfmt != MOE_WFMT_MXFP4_E2M1_E8M0_K32) return MOE_ERR_UNSUPPORTED;
  if ((long long)T * (k + n_shared) > (1LL << 26)) return MOE_ERR_UNSUPPORTED;
  const Carve cv = carve(H, I, E, k, n_shared, T);
  if (cv.total > (size_t)MOE_NOALLOC_SCRATCH_BYTES) return MOE_ERR_UNSUPPORTED;  // beyond the fixed scratch
  if (T == 0) return MOE_OK;
  if (!x || !topk_ids || !topk_w || !w13 || !s13 || !w2 || !s2 || !out) return MOE_ERR_INVALID_ARG;
  auto al = [](const void* p, uintptr_t a) { return reinterpret_cast<uintptr_t>(p) % a == 0; };
  if (!al(x, 16) || !al(out, 16) || !al(w13, 128) || !al(w2, 128) || !al(s13, 16) || !al(s2, 16) ||
      !al(topk_ids, 4) || !al(topk_w, 4) || !al(d_status, 4))
    return MOE_ERR_INVALID_ARG;
  if (wfmt == MOE_WFMT_MXFP4_E2M1_E8M0_K32 &&
      (!moe::packed_scales_known(s13, (size_t)(E + n_shared) * 2 * I * (H / 32), wfmt) ||
       !moe::packed_scales_known(s2, (size_t)(E + n_shared) * H * (I / 32), wfmt)))
    return MOE_ERR_INVALID_ARG;  // scales not in the packed layout (see moe_declare_packed_scales)

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return MOE_ERR_CUDA;
  if (dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;  // more GPUs than the per-device tables hold
  const moe_status st = setup_device(dev);
  if (st != MOE_OK) return st;
  char* b = static_cast<char*>(g_scratch_addr[dev]);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const bool fp8 = (wfmt == MOE_WFMT_FP8_E4M3_B128);
  const int NE = E + n_shared;
  const size_t P = (size_t)T * k + (size_t)n_shared * T;
  const size_t S_pad = P + 128;
  const double avg = (double)T * k / E;
  int BN = avg <= 8 ? 16 : avg <= 20 ? 32 : avg <= 48 ? 64 : 128;
  if (!fp8 && BN > 64) BN = 64;

  int32_t* status = d_status ? d_status : reinterpret_cast<int32_t*>(b + cv.status);
  uint8_t* xq = reinterpret_cast<uint8_t*>(b + cv.xq);
  uint8_t* hq = reinterpret_cast<uint8_t*>(b + cv.hq);
  CUtensorMap tw13, tw2, txq, thq;
  const bool ok =
      (fp8 ? map2d(&tw13, CU_TENSOR_MAP_DATA_TYPE_UINT8, w13, H, (uint64_t)NE * 2 * I, H, 128,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B) &&
                 map2d(&tw2, CU_TENSOR_MAP_DATA_TYPE_UINT8, w2, I, (uint64_t)NE * H, I, 128,
                       CU_TENSOR_MAP_L2_PROMOTION_L2_256B)
           : map2d(&tw13, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, w13, H, (uint64_t)NE * 2 * I, H / 2, 128,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B) &&
                 map2d(&tw2, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, w2, I, (uint64_t)NE * H, I / 2, 128,
                       CU_TENSOR_MAP_L2_PROMOTION_L2_256B)) &&
      map2d(&txq, CU_TENSOR_MAP_DATA_TYPE_UINT8, xq, H, S_pad, H, BN, CU_TENSOR_MAP_L2_PROMOTION_L2_128B) &&
      map2d(&thq, CU_TENSOR_MAP_DATA_TYPE_UINT8, hq, I, S_pad, I, BN, CU_TENSOR_MAP_L2_PROMOTION_L2_128B);
  if (!ok) return MOE_ERR_CUDA;

  // The only word that must start at zero each call; the combine buffer is
  // cleared by the quantisation kernel as in moe_forward().
  if (cudaMemsetAsync(status, 0, sizeof(int32_t), s) != cudaSuccess) return MOE_ERR_CUDA;

  moe::RouteParams rp{};
  rp.T = T; rp.k = k; rp.E = E; rp.n_shared = n_shared; rp.BN = BN;
  rp.ids = topk_ids;
  rp.counts = reinterpret_cast<int32_t*>(b + cv.counts);
  rp.offsets = reinterpret_cast<int32_t*>(b + cv.offsets);
  rp.perm = reinterpret_cast<int32_t*>(b + cv.perm);
  rp.inv = reinterpret_cast<int32_t*>(b + cv.inv);
  rp.tiles = reinterpret_cast<int4*>(b + cv.tiles);
  rp.num_tiles = reinterpret_cast<int32_t*>(b + cv.ntiles);
  rp.status = status;
  if (moe::launch_route(rp, s) != cudaSuccess) return MOE_ERR_CUDA;

  float* acc = reinterpret_cast<float*>(b + cv.acc);
  float* xs = reinterpret_cast<float*>(b + cv.xs);
  float* hs = reinterpret_cast<float*>(b + cv.hs);
  moe::QuantParams qp{};
  qp.T = T; qp.H = H; qp.k = k; qp.n_shared = n_shared;
  qp.x = static_cast<const uint16_t*>(x); qp.inv = rp.inv; qp.xq = xq; qp.xs = xs; qp.out_acc = acc;
  qp.xs_ld = (int)S_pad;
  qp.pdl = moe::quant_pdl(T, k, E, n_shared, H, I);
  if (moe::launch_quant(qp, s) != cudaSuccess) return MOE_ERR_CUDA;

  moe::GemmParams g{};
  g.H = H; g.I = I; g.k = k; g.S = T * k;
  g.kblocks = H / 128;
  g.wscale = static_cast<const float*>(s13);
  g.ascale = xs;
  g.scale_ld = (int)S_pad;
  g.hq = hq; g.hs = hs;
  g.perm = rp.perm; g.topk_w = topk_w; g.out_acc = acc;
  g.tiles = rp.tiles; g.num_tiles = rp.num_tiles; g.status = status;
  g.y_rows = nullptr;  // fused combine into the fp32 accumulator
  g.inject = 0;
  g.wglobal = nullptr; g.hsc = nullptr;
  if (moe::launch_gemm1(wfmt, BN, g_num_sms[dev], tw13, txq, txq, g, s) != cudaSuccess) return MOE_ERR_CUDA;
  g.kblocks = I / 128;
  g.wscale = static_cast<const float*>(s2);
  g.ascale = hs;
  if (moe::launch_gemm2(wfmt, BN, g_num_sms[dev], tw2, thq, thq, g, s) != cudaSuccess) return MOE_ERR_CUDA;
  if (moe::launch_finalize(acc, static_cast<uint16_t*>(out), (long long)T * H, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}
