// Host side of libattn.so: argument validation, TMA tensor-map encoding and kernel launches behind the
// C ABI declared in include/attn.h. No allocation, no synchronisation on the attention path.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "attn.h"
#include "attn_bwd.cuh"
#include "attn_errors.h"
#include "attn_decode.cuh"
#include "attn_fwd.cuh"

namespace attn {
thread_local char g_cuda_error[kErrorTextBytes] = "";
}  // namespace attn

namespace {

using attn::g_cuda_error;
uint64_t g_wait_limit_ns = 1000ull * 1000 * 1000;  // 1 s

attn_status cuda_fail(cudaError_t e, const char* what) {
  std::snprintf(g_cuda_error, sizeof(g_cuda_error), "%s: %s", what, cudaGetErrorString(e));
  return ATTN_ERR_CUDA;
}

// ---------------------------------------------------------------------------------------------- tensor maps

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn(cudaError_t* err) {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  static cudaError_t e0 = cudaSuccess;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    e0 = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
    if (e0 == cudaSuccess && q == cudaDriverEntryPointSuccess) fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  *err = e0;
  return fn;
}

// A [B, T, H, 128] bf16 tensor seen by TMA as dims {D, H, T, B} (strides increase outward), with a box of
// 64 head-dim columns (128 bytes, the 128-byte swizzle span) x one head x `rows` time steps.
attn_status make_map(CUtensorMap* m, const void* ptr, int B, int H, int T, int rows) {
  cudaError_t e;
  EncodeTiledFn fn = encode_fn(&e);
  if (!fn) return cuda_fail(e == cudaSuccess ? cudaErrorNotSupported : e, "cuTensorMapEncodeTiled lookup");
  const cuuint64_t dims[4] = {128, static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(T), static_cast<cuuint64_t>(B)};
  const cuuint64_t strides[3] = {256, static_cast<cuuint64_t>(H) * 256, static_cast<cuuint64_t>(T) * H * 256};
  const cuuint32_t box[4] = {64, 1, static_cast<cuuint32_t>(rows), 1};
  const cuuint32_t elem[4] = {1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box, elem,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    std::snprintf(g_cuda_error, sizeof(g_cuda_error), "cuTensorMapEncodeTiled failed (CUresult %d)", (int)r);
    return ATTN_ERR_CUDA;
  }
  return ATTN_OK;
}

// ---------------------------------------------------------------------------------------------- checks

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Range {
  uintptr_t lo, hi;
};
Range span(const void* p, size_t bytes) {
  const uintptr_t a = reinterpret_cast<uintptr_t>(p);
  return {a, a + bytes};
}
bool overlap(Range a, Range b) { return a.lo < b.hi && b.lo < a.hi; }

attn_status check_sizes(int B, int H, int T, int D, float scale) {
  if (B < 1 || H < 1 || T < 1) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !(scale > 0.f)) return ATTN_ERR_INVALID_ARG;
  if (D != 128) return ATTN_ERR_UNSUPPORTED;
  // Kernel indexing: CTA counts and (b*H + h) fit in 31 bits; element offsets use 64-bit arithmetic.
  const long long bh = static_cast<long long>(B) * H;
  const long long qtiles = (static_cast<long long>(T) + 127) / 128;
  if (bh * qtiles * 2 > 0x7fffffffLL) return ATTN_ERR_UNSUPPORTED;
  if (T > (1 << 30)) return ATTN_ERR_UNSUPPORTED;
  return ATTN_OK;
}

// Grouped-query attention: H_kv key/value heads, dividing the H query heads.
attn_status check_kv_heads(int H, int Hkv) {
  if (Hkv < 1 || Hkv > H || H % Hkv != 0) return ATTN_ERR_INVALID_ARG;
  return ATTN_OK;
}

// Set the dynamic shared-memory opt-in of both big kernels once per device.
int g_sm_count[64] = {};       // multiprocessors per device, set by prepare_device
int g_fwd_clusters[64] = {};   // CTA pairs of the forward kernel that fit on the device at once

attn_status prepare_device(int* dev_out) {
  static std::mutex mu;
  static bool done[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  // Make the device's primary context current on this thread (a thread that has only queued work through
  // another runtime, such as an autograd worker, may have none); the tensor-map encoder needs one.
  if ((e = cudaSetDevice(dev)) != cudaSuccess) return cuda_fail(e, "cudaSetDevice");
  *dev_out = dev;
  std::lock_guard<std::mutex> lock(mu);
  if (dev >= 0 && dev < 64 && done[dev]) return ATTN_OK;
  int major = 0, minor = 0;
  if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
      (e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess)
    return cuda_fail(e, "cudaDeviceGetAttribute");
  int sms = 0;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return cuda_fail(e, "cudaDeviceGetAttribute");
  if (dev >= 0 && dev < 64) g_sm_count[dev] = sms;
  if (major != 10 || minor != 0) {
    std::snprintf(g_cuda_error, sizeof(g_cuda_error), "device %d is sm_%d%d; this library is built for sm_100a",
                  dev, major, minor);
    return ATTN_ERR_CUDA;
  }
  if ((e = cudaFuncSetAttribute(attn::attn_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                attn::kFwdSmemAlloc)) != cudaSuccess)
    return cuda_fail(e, "cudaFuncSetAttribute(attn_fwd_kernel)");
  if ((e = cudaFuncSetAttribute(attn::attn_bwd_dkdv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                attn::kBwdSmemAlloc)) != cudaSuccess)
    return cuda_fail(e, "cudaFuncSetAttribute(attn_bwd_dkdv_kernel)");
  {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * 74);
    cfg.blockDim = dim3(attn::kFwdThreads);
    cfg.dynamicSmemBytes = attn::kFwdSmemAlloc;
    int n = 0;
    if ((e = cudaOccupancyMaxActiveClusters(&n, attn::attn_fwd_kernel, &cfg)) != cudaSuccess)
      return cuda_fail(e, "cudaOccupancyMaxActiveClusters(attn_fwd_kernel)");
    if (n < 1) {
      std::snprintf(g_cuda_error, sizeof(g_cuda_error), "device %d cannot co-schedule a pair of forward CTAs", dev);
      return ATTN_ERR_CUDA;
    }
    if (dev >= 0 && dev < 64) g_fwd_clusters[dev] = n;
  }
  if (dev >= 0 && dev < 64) done[dev] = true;
  return ATTN_OK;
}

struct WorkspaceLayout {
  size_t lse2, delta, acc, total;
};
WorkspaceLayout workspace_layout(int B, int H, int T) {
  const size_t rows = static_cast<size_t>(B) * H * attn::padded_T(T);
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  WorkspaceLayout w;
  w.lse2 = 0;
  w.delta = up(rows * 4);
  w.acc = w.delta + up(rows * 4);
  w.total = w.acc + up(rows * 128 * 4);
  return w;
}

int grid_for(size_t work_items, int per_block) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const size_t blocks = (work_items + per_block - 1) / per_block;
  const size_t cap = static_cast<size_t>(sms) * 8;
  return static_cast<int>(blocks < cap ? (blocks > 0 ? blocks : 1) : cap);
}

// Self-test kernel for the bounded-wait path (see attn_selftest_wait_timeout).
__global__ void wait_timeout_selftest_kernel(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    sm100::mbar_init(&bar, 1);
    abort_flag = 0;
    sm100::fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) sm100::mbar_wait(&bar, 0, &abort_flag, limit_ns, &attn::g_device_error, 0x7f);
}

#ifdef ATTN_DEBUG
// Self-test of the debug build's address checks (see attn_selftest_bounds_check): one checked store whose
// index (1) lies past the declared one-element extent of its array. The check records the site and skips the
// store, so nothing is written; the array has a second element all the same, so the index is inside the memory.
__device__ int g_bounds_selftest_cell[2];
__global__ void bounds_selftest_kernel(int index) {
  if (ATTN_IN_RANGE(index, 1, 1, attn::kSiteChkSelftest, &attn::g_device_error)) g_bounds_selftest_cell[index] = 1;
}
#endif

}  // namespace

extern "C" {

int attn_abi_version(void) { return 2; }

const char* attn_status_string(attn_status s) {
  switch (s) {
    case ATTN_OK: return "ATTN_OK";
    case ATTN_ERR_INVALID_ARG: return "ATTN_ERR_INVALID_ARG";
    case ATTN_ERR_UNSUPPORTED: return "ATTN_ERR_UNSUPPORTED";
    case ATTN_ERR_MISALIGNED: return "ATTN_ERR_MISALIGNED";
    case ATTN_ERR_CUDA: return "ATTN_ERR_CUDA";
    case ATTN_ERR_TIMEOUT: return "ATTN_ERR_TIMEOUT";
    case ATTN_ERR_WORKSPACE: return "ATTN_ERR_WORKSPACE";
    case ATTN_ERR_BOUNDS: return "ATTN_ERR_BOUNDS";
  }
  return "ATTN_ERR_UNKNOWN";
}

const char* attn_last_cuda_error(void) { return g_cuda_error; }

attn_status attn_set_wait_limit_ns(uint64_t limit_ns) {
  if (limit_ns < 1000) return ATTN_ERR_INVALID_ARG;
  g_wait_limit_ns = limit_ns;
  return ATTN_OK;
}

}  // extern "C"

namespace {

attn_status fwd_launch(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Hkv,
                       int T, int D, float scale, int window, void* stream) {
  if (!q || !k || !v || !o || !lse) return ATTN_ERR_INVALID_ARG;
  attn_status st = check_sizes(B, H, T, D, scale);
  if (st != ATTN_OK) return st;
  if ((st = check_kv_heads(H, Hkv)) != ATTN_OK) return st;
  if (window < -1) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return ATTN_ERR_MISALIGNED;
  const size_t nbytes = static_cast<size_t>(B) * T * H * D * 2;
  const size_t kvbytes = static_cast<size_t>(B) * T * Hkv * D * 2;
  const size_t lbytes = static_cast<size_t>(B) * H * T * 4;
  const Range rq = span(q, nbytes), rk = span(k, kvbytes), rv = span(v, kvbytes), ro = span(o, nbytes),
              rl = span(lse, lbytes);
  for (Range in : {rq, rk, rv})
    if (overlap(ro, in) || overlap(rl, in)) return ATTN_ERR_INVALID_ARG;
  if (overlap(ro, rl)) return ATTN_ERR_INVALID_ARG;

  int dev = 0;
  if ((st = prepare_device(&dev)) != ATTN_OK) return st;
  CUtensorMap mq, mk, mv, mo;
  if ((st = make_map(&mq, q, B, H, T, attn::kTile)) != ATTN_OK) return st;
  if ((st = make_map(&mk, k, B, Hkv, T, attn::kFwdKRows)) != ATTN_OK) return st;
  if ((st = make_map(&mv, v, B, Hkv, T, attn::kTile)) != ATTN_OK) return st;
  if ((st = make_map(&mo, o, B, H, T, attn::kTile)) != ATTN_OK) return st;

  attn::FwdParams p;
  p.lse = lse;
  p.B = B;
  p.H = H;
  p.Hkv = Hkv;
  p.window = window;
  p.T = T;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.timeout_ns = g_wait_limit_ns;
  // Persistent grid of CTA pairs: as many pairs as fit at once (one per TPC), fewer when there are fewer work
  // items (pairs of query tiles).
  const long long n_items = static_cast<long long>((T + 2 * attn::kTile - 1) / (2 * attn::kTile)) * B * H;
  const int pairs = (dev >= 0 && dev < 64 && g_fwd_clusters[dev] > 0) ? g_fwd_clusters[dev] : 74;
  const dim3 grid(2u * static_cast<unsigned>(n_items < pairs ? n_items : pairs));
  attn::attn_fwd_kernel<<<grid, attn::kFwdThreads, attn::kFwdSmemAlloc, static_cast<cudaStream_t>(stream)>>>(
      mq, mk, mv, mo, p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "attn_fwd_kernel launch");
  return ATTN_OK;
}

}  // namespace

extern "C" {

attn_status attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int T, int D,
                     float scale, void* stream) {
  return fwd_launch(q, k, v, o, lse, B, H, H, T, D, scale, -1, stream);
}

attn_status attn_fwd_gqa(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int H_kv,
                         int T, int D, float scale, void* stream) {
  return fwd_launch(q, k, v, o, lse, B, H, H_kv, T, D, scale, -1, stream);
}

attn_status attn_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int H_kv,
                        int T, int D, float scale, int window, void* stream) {
  return fwd_launch(q, k, v, o, lse, B, H, H_kv, T, D, scale, window, stream);
}

size_t attn_bwd_workspace_bytes(int B, int H, int T, int D) {
  if (check_sizes(B, H, T, D, 1.0f) != ATTN_OK) return 0;
  return workspace_layout(B, H, T).total;
}

}  // extern "C"

namespace {

// Validates the backward arguments and launches the stages selected by `stages` (bit 0: preprocess,
// bit 1: dK/dV with dQ accumulation, bit 2: dQ conversion) in that order on `stream`.
attn_status bwd_launch(unsigned stages, const void* q, const void* k, const void* v, const void* o, const float* lse,
                       const void* dO, void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes, int B,
                       int H, int Hkv, int T, int D, float scale, int window, void* stream) {
  if (!q || !k || !v || !o || !lse || !dO || !dq || !dk || !dv) return ATTN_ERR_INVALID_ARG;
  attn_status st = check_sizes(B, H, T, D, scale);
  if (st != ATTN_OK) return st;
  if ((st = check_kv_heads(H, Hkv)) != ATTN_OK) return st;
  if (window < -1) return ATTN_ERR_INVALID_ARG;
  const WorkspaceLayout wl = workspace_layout(B, H, T);
  if (!workspace || workspace_bytes < wl.total) return ATTN_ERR_WORKSPACE;
  for (const void* ptr : {q, k, v, o, dO, static_cast<const void*>(lse), static_cast<const void*>(dq),
                          static_cast<const void*>(dk), static_cast<const void*>(dv)})
    if (!aligned16(ptr)) return ATTN_ERR_MISALIGNED;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return ATTN_ERR_MISALIGNED;
  const size_t nbytes = static_cast<size_t>(B) * T * H * D * 2;
  const size_t kvbytes = static_cast<size_t>(B) * T * Hkv * D * 2;
  const size_t lbytes = static_cast<size_t>(B) * H * T * 4;
  const Range ins[6] = {span(q, nbytes), span(k, kvbytes), span(v, kvbytes), span(o, nbytes), span(dO, nbytes),
                        span(lse, lbytes)};
  const Range outs[4] = {span(dq, nbytes), span(dk, kvbytes), span(dv, kvbytes), span(workspace, wl.total)};
  for (int i = 0; i < 4; ++i) {
    for (int j = 0; j < 6; ++j)
      if (overlap(outs[i], ins[j])) return ATTN_ERR_INVALID_ARG;
    for (int j = i + 1; j < 4; ++j)
      if (overlap(outs[i], outs[j])) return ATTN_ERR_INVALID_ARG;
  }

  int dev = 0;
  if ((st = prepare_device(&dev)) != ATTN_OK) return st;
  CUtensorMap mq, mk, mv, mdo, mdk, mdv;
  if ((st = make_map(&mq, q, B, H, T, attn::kBwdQTile)) != ATTN_OK) return st;
  if ((st = make_map(&mdo, dO, B, H, T, attn::kBwdQTile)) != ATTN_OK) return st;
  if ((st = make_map(&mk, k, B, Hkv, T, attn::kBwdKTile)) != ATTN_OK) return st;
  if ((st = make_map(&mv, v, B, Hkv, T, attn::kBwdKTile)) != ATTN_OK) return st;
  if ((st = make_map(&mdk, dk, B, Hkv, T, attn::kBwdKTile)) != ATTN_OK) return st;
  if ((st = make_map(&mdv, dv, B, Hkv, T, attn::kBwdKTile)) != ATTN_OK) return st;

  uint8_t* ws = static_cast<uint8_t*>(workspace);
  attn::BwdParams p;
  p.o = static_cast<const __nv_bfloat16*>(o);
  p.dO = static_cast<const __nv_bfloat16*>(dO);
  p.lse = lse;
  p.lse2 = reinterpret_cast<float*>(ws + wl.lse2);
  p.delta = reinterpret_cast<float*>(ws + wl.delta);
  p.dq_acc = reinterpret_cast<float*>(ws + wl.acc);
  p.dq = static_cast<__nv_bfloat16*>(dq);
  p.B = B;
  p.H = H;
  p.Hkv = Hkv;
  p.window = window;
  p.T = T;
  p.Tp = attn::padded_T(T);
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.timeout_ns = g_wait_limit_ns;
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  cudaError_t e;
  if (stages & 1u) {
    const size_t quads = static_cast<size_t>(B) * H * p.Tp / 4;  // a 16-thread group per four padded rows
    attn::attn_bwd_prep_kernel<<<grid_for(quads * 16, 256), 256, 0, s>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "attn_bwd_prep_kernel launch");
  }
  if (stages & 2u) {
    // Persistent grid: one CTA per SM (fewer when there are fewer work items, key tiles x key/value heads).
    const long long n_items = static_cast<long long>((T + attn::kBwdKTile - 1) / attn::kBwdKTile) * B * Hkv;
    const int sms = (dev >= 0 && dev < 64 && g_sm_count[dev] > 0) ? g_sm_count[dev] : 148;
    attn::attn_bwd_dkdv_kernel<<<dim3(static_cast<unsigned>(n_items < sms ? n_items : sms)), attn::kBwdThreads,
                                 attn::kBwdSmemAlloc, s>>>(mq, mk, mv, mdo, mdk, mdv, p);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "attn_bwd_dkdv_kernel launch");
  }
  if (stages & 4u) {
    const size_t items = static_cast<size_t>(B) * H * ((T + 3) / 4) * 32;
    attn::attn_bwd_dq_kernel<<<grid_for(items, 256), 256, 0, s>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "attn_bwd_dq_kernel launch");
  }
  return ATTN_OK;
}

}  // namespace

extern "C" {

#define ATTN_BWD_ARGS                                                                                          \
  const void *q, const void *k, const void *v, const void *o, const float *lse, const void *dO, void *dq,     \
      void *dk, void *dv, void *workspace, size_t workspace_bytes, int B, int H, int T, int D, float scale,     \
      void *stream
#define ATTN_BWD_PASS q, k, v, o, lse, dO, dq, dk, dv, workspace, workspace_bytes, B, H, H, T, D, scale, -1, stream

attn_status attn_bwd(ATTN_BWD_ARGS) { return bwd_launch(7u, ATTN_BWD_PASS); }
attn_status attn_bwd_preprocess(ATTN_BWD_ARGS) { return bwd_launch(1u, ATTN_BWD_PASS); }
attn_status attn_bwd_dkdv(ATTN_BWD_ARGS) { return bwd_launch(2u, ATTN_BWD_PASS); }
attn_status attn_bwd_dq_convert(ATTN_BWD_ARGS) { return bwd_launch(4u, ATTN_BWD_PASS); }

attn_status attn_bwd_gqa(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
                         void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes, int B, int H, int H_kv,
                         int T, int D, float scale, void* stream) {
  return bwd_launch(7u, q, k, v, o, lse, dO, dq, dk, dv, workspace, workspace_bytes, B, H, H_kv, T, D, scale, -1,
                    stream);
}

attn_status attn_bwd_ex(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
                        void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes, int B, int H, int H_kv,
                        int T, int D, float scale, int window, void* stream) {
  return bwd_launch(7u, q, k, v, o, lse, dO, dq, dk, dv, workspace, workspace_bytes, B, H, H_kv, T, D, scale, window,
                    stream);
}

attn_status attn_get_device_error(uint32_t* word) {
  if (!word) return ATTN_ERR_INVALID_ARG;
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
  e = cudaMemcpyFromSymbol(word, attn::g_device_error, sizeof(uint32_t));
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyFromSymbol(g_device_error)");
  uint32_t rope_word = 0;
  e = static_cast<cudaError_t>(attn::rope_error_word(&rope_word));
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyFromSymbol(g_rope_error)");
  *word |= rope_word;
  if (*word & sm100::DEV_ERR_TIMEOUT) return ATTN_ERR_TIMEOUT;
  return *word ? ATTN_ERR_BOUNDS : ATTN_OK;
}

attn_status attn_clear_device_error(void) {
  const uint32_t zero = 0;
  cudaError_t e = cudaMemcpyToSymbol(attn::g_device_error, &zero, sizeof(uint32_t));
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyToSymbol(g_device_error)");
  e = static_cast<cudaError_t>(attn::rope_error_clear());
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyToSymbol(g_rope_error)");
  e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
  return ATTN_OK;
}

#ifdef ATTN_TRACE
// Profiling builds only (-DATTN_TRACE): copy the pipeline trace of the last launch to host memory.
int attn_trace_dump(void* dst, size_t bytes) {
  if (bytes < attn::kTraceBytes) return -1;
  cudaError_t e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpyFromSymbol(dst, attn::g_trace, attn::kTraceBytes);
  if (e == cudaSuccess) {
    static unsigned long long zeros[attn::kTraceBytes / 8];
    e = cudaMemcpyToSymbol(attn::g_trace, zeros, attn::kTraceBytes);
  }
  return e == cudaSuccess ? 0 : -1;
}
#endif

int attn_is_debug_build(void) {
#ifdef ATTN_DEBUG
  return 1;
#else
  return 0;
#endif
}

attn_status attn_selftest_bounds_check(void* stream) {
#ifdef ATTN_DEBUG
  bounds_selftest_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(1);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "bounds_selftest_kernel launch");
  return ATTN_OK;
#else
  (void)stream;
  return ATTN_ERR_UNSUPPORTED;  // the release build has no address checks to test
#endif
}

attn_status attn_selftest_wait_timeout(uint64_t limit_ns, void* stream) {
  if (limit_ns < 1000 || limit_ns > 10ull * 1000 * 1000 * 1000) return ATTN_ERR_INVALID_ARG;
  wait_timeout_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "wait_timeout_selftest_kernel launch");
  return ATTN_OK;
}

// ---------------------------------------------------------------------------------------------- no-alloc bwd
//
// Backward for callers that cannot allocate device memory: code running inside a framework's custom-op or
// plugin interface that hands over tensors but offers no allocator and no workspace, and code working under
// a fixed memory plan that forbids allocation (and the device-wide synchronisation cudaMalloc/cudaFree can
// bring) during a step. The scratch space attn_bwd takes from its caller lives instead in the file-scope
// device array below, which every GPU that loads this library holds until the process exits.

}  // extern "C"

namespace {

constexpr size_t kNoAllocScratchBytes = 32ull << 20;  // 32 MiB: B * H * roundup(T, 128) <= 64512 rows
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch, looked up once per device with that device current. In host code the
// array's name is only a host-side stand-in, never a device address, so kernels get this pointer instead.
attn_status noalloc_scratch_ptr(void** out) {
  static std::mutex mu;
  static void* addr[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return ATTN_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    if ((e = cudaSetDevice(dev)) != cudaSuccess) return cuda_fail(e, "cudaSetDevice");
    void* p = nullptr;
    if ((e = cudaGetSymbolAddress(&p, g_noalloc_scratch)) != cudaSuccess)
      return cuda_fail(e, "cudaGetSymbolAddress(g_noalloc_scratch)");
    addr[dev] = p;
  }
  *out = addr[dev];
  return ATTN_OK;
}

}  // namespace

extern "C" {

attn_status attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                             const void* dO, void* dq, void* dk, void* dv, int B, int H, int T, int D, float scale,
                             void* stream) {
  attn_status st = check_sizes(B, H, T, D, scale);
  if (st != ATTN_OK) return st;
  const size_t need = workspace_layout(B, H, T).total;
  if (need > kNoAllocScratchBytes) {
    std::snprintf(g_cuda_error, sizeof(g_cuda_error),
                  "attn_bwd_noalloc: these sizes need %zu bytes of scratch, the built-in array holds %zu", need,
                  kNoAllocScratchBytes);
    return ATTN_ERR_WORKSPACE;
  }
  void* scratch = nullptr;
  if ((st = noalloc_scratch_ptr(&scratch)) != ATTN_OK) return st;
  // Same three kernels as attn_bwd; the preprocess kernel rewrites every scratch byte the later kernels read
  // (including zeroing the dQ accumulator), so whatever an earlier call left there does not matter.
  return bwd_launch(7u, q, k, v, o, lse, dO, dq, dk, dv, scratch, kNoAllocScratchBytes, B, H, H, T, D, scale, -1,
                    stream);
}

}  // extern "C"

namespace {

// Splits of the cache per (sequence, key/value head): about 4 units per SM of a 148-SM part in all, each split at
// least kDecChunkKeys keys (a multiple of the 128-key block). The persistent split kernel deals the units out
// longest first; a few units per SM let the short ones even out the SMs' totals, while more would add merge work
// (with one CTA per unit, 4 per SM ran 1-6 % faster than 8 and 10-25 % faster than 16, and 2 or 1 lost 10 % with
// grouped heads).
void decode_split(int B, int Hkv, int Tk, int* n_split, int* chunk) {
  const long long pairs = static_cast<long long>(B) * Hkv;
  long long want = (4 * 148 + pairs - 1) / pairs;
  const long long max_split = (Tk + attn::kDecChunkKeys - 1) / attn::kDecChunkKeys;
  if (want > max_split) want = max_split;
  if (want < 1) want = 1;
  long long c = (Tk + want - 1) / want;
  c = (c + attn::kDecKeys - 1) / attn::kDecKeys * attn::kDecKeys;
  *chunk = static_cast<int>(c);
  *n_split = static_cast<int>((Tk + c - 1) / c);
}

attn_status check_decode(int B, int H, int Hkv, int Tq, int Tk, int D, float scale) {
  if (B < 1 || H < 1 || Tq < 1 || Tk < 1) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !(scale > 0.f)) return ATTN_ERR_INVALID_ARG;
  attn_status st = check_kv_heads(H, Hkv);
  if (st != ATTN_OK) return st;
  if (D != 128) return ATTN_ERR_UNSUPPORTED;
  if ((H / Hkv) * static_cast<long long>(Tq) > attn::kDecMaxRows) return ATTN_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * Hkv * ((Tk + attn::kDecChunkKeys - 1) / attn::kDecChunkKeys) > 0x7fffffffLL ||
      static_cast<long long>(B) * H * Tq > 0x7fffffffLL / 8)
    return ATTN_ERR_UNSUPPORTED;
  return ATTN_OK;
}

// Keys a sequence's rows can see: the whole cache, or with a sliding window the Tq + window before its end.
int decode_span(int Tq, int Tk, int window) {
  return window < 0 ? Tk : static_cast<int>(std::min<long long>(Tk, static_cast<long long>(Tq) + window));
}

size_t decode_workspace(int B, int H, int Hkv, int Tq, int Tk) {
  int n_split = 1, chunk = 0;
  decode_split(B, Hkv, Tk, &n_split, &chunk);  // no window: the most chunks, enough for any window
  const size_t rows = static_cast<size_t>(B) * Hkv * n_split * ((H / Hkv) * Tq);
  return rows * 128 * 4 + rows * 2 * 4;
}

}  // namespace

extern "C" {

size_t attn_decode_workspace_bytes(int B, int H, int H_kv, int Tq, int Tk, int D) {
  if (check_decode(B, H, H_kv, Tq, Tk, D, 1.0f) != ATTN_OK) return 0;
  return decode_workspace(B, H, H_kv, Tq, Tk);
}

int attn_decode_kernels(int B, int H, int H_kv, int Tq, int Tk, int D, int window) {
  if (check_decode(B, H, H_kv, Tq, Tk, D, 1.0f) != ATTN_OK || window < -1) return 0;
  int n_split = 1, chunk = 0;
  decode_split(B, H_kv, decode_span(Tq, Tk, window), &n_split, &chunk);
  return n_split > 1 ? 2 : 1;
}

attn_status attn_decode_ex(const void* q, const void* k_cache, const void* v_cache, const int* cache_seqlens,
                           void* o, float* lse, void* workspace, size_t workspace_bytes, int B, int H, int H_kv,
                           int Tq, int Tk, int D, float scale, int window, void* stream) {
  if (!q || !k_cache || !v_cache || !cache_seqlens || !o || !lse) return ATTN_ERR_INVALID_ARG;
  attn_status st = check_decode(B, H, H_kv, Tq, Tk, D, scale);
  if (st != ATTN_OK) return st;
  if (window < -1) return ATTN_ERR_INVALID_ARG;
  const size_t need = decode_workspace(B, H, H_kv, Tq, Tk);
  if (!workspace || workspace_bytes < need) return ATTN_ERR_WORKSPACE;
  for (const void* ptr : {q, k_cache, v_cache, static_cast<const void*>(o), static_cast<const void*>(workspace)})
    if (!aligned16(ptr)) return ATTN_ERR_MISALIGNED;
  if ((reinterpret_cast<uintptr_t>(lse) & 3u) || (reinterpret_cast<uintptr_t>(cache_seqlens) & 3u))
    return ATTN_ERR_MISALIGNED;
  const size_t qbytes = static_cast<size_t>(B) * Tq * H * D * 2;
  const size_t cbytes = static_cast<size_t>(B) * Tk * H_kv * D * 2;
  const Range ins[4] = {span(q, qbytes), span(k_cache, cbytes), span(v_cache, cbytes),
                        span(cache_seqlens, static_cast<size_t>(B) * 4)};
  const Range outs[3] = {span(o, qbytes), span(lse, static_cast<size_t>(B) * H * Tq * 4), span(workspace, need)};
  for (int i = 0; i < 3; ++i) {
    for (int j = 0; j < 4; ++j)
      if (overlap(outs[i], ins[j])) return ATTN_ERR_INVALID_ARG;
    for (int j = i + 1; j < 3; ++j)
      if (overlap(outs[i], outs[j])) return ATTN_ERR_INVALID_ARG;
  }
  int dev = 0;
  if ((st = prepare_device(&dev)) != ATTN_OK) return st;
  attn::DecodeParams p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k = static_cast<const __nv_bfloat16*>(k_cache);
  p.v = static_cast<const __nv_bfloat16*>(v_cache);
  p.seqlens = cache_seqlens;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.B = B;
  p.H = H;
  p.Hkv = H_kv;
  p.Tq = Tq;
  p.Tk = Tk;
  p.R = (H / H_kv) * Tq;
  p.window = window;
  decode_split(B, H_kv, decode_span(Tq, Tk, window), &p.n_split, &p.chunk);
  // Longest chunks first whenever the sort's scratch (a count per block count, 16 bits per (sequence, chunk)
  // pair) fits the ring's first stage: up to about 32k pairs.
  const long long order_nb = p.chunk / attn::kDecKeys;
  const long long order_bytes = (order_nb + 1) * 4 + static_cast<long long>(B) * p.n_split * 2;
  p.order_nb = order_bytes <= attn::kDecOrderScratch ? static_cast<int>(order_nb) : 0;
  const size_t rows = static_cast<size_t>(B) * H_kv * p.n_split * p.R;
  p.part_o = static_cast<float*>(workspace);
  p.part_ml = static_cast<float*>(workspace) + rows * 128;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.timeout_ns = g_wait_limit_ns;
  CUtensorMap mk, mv;  // the caches as [B, Tk, H_kv, 128]: 128-key x 64-dim boxes
  if ((st = make_map(&mk, k_cache, B, H_kv, Tk, attn::kDecKeys)) != ATTN_OK) return st;
  if ((st = make_map(&mv, v_cache, B, H_kv, Tk, attn::kDecKeys)) != ATTN_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // One CTA per SM (a CTA's ring takes most of an SM's shared memory) walks its share of the units, its ring
  // running on from one unit into the next, while each share fits a CTA's unit list; else one CTA per unit.
  const long long n_units = static_cast<long long>(B) * H_kv * p.n_split;
  const long long sms = (dev >= 0 && dev < 64 && g_sm_count[dev] > 0) ? g_sm_count[dev] : 148;
  const unsigned grid = static_cast<unsigned>(n_units <= attn::kDecMaxUnits * sms ? std::min(n_units, sms) : n_units);
  cudaError_t e = cudaSuccess;
  auto launch = [&](auto kernel, size_t smem_bytes, int threads) {
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem_bytes));
    if (e == cudaSuccess) kernel<<<grid, threads, smem_bytes, s>>>(mk, mv, p);
  };
#define ATTN_DEC_LAUNCH(R) \
  launch(attn::attn_decode_split_kernel<R>, attn::dec_smem_bytes<R>(), attn::dec_threads<R>())
  if (p.R <= 1) ATTN_DEC_LAUNCH(1);
  else if (p.R <= 2) ATTN_DEC_LAUNCH(2);
  else if (p.R <= 4) ATTN_DEC_LAUNCH(4);
  else if (p.R <= 8) ATTN_DEC_LAUNCH(8);
  else if (p.R <= 16) ATTN_DEC_LAUNCH(16);
  else ATTN_DEC_LAUNCH(32);
#undef ATTN_DEC_LAUNCH
  if (e != cudaSuccess) return cuda_fail(e, "attn_decode_split_kernel attribute");
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "attn_decode_split_kernel launch");
  if (p.n_split > 1) {  // (with one chunk per (sequence, head) the split kernel wrote o and lse itself)
    const long long out_rows = static_cast<long long>(B) * H * Tq;
    attn::attn_decode_combine_kernel<<<static_cast<unsigned>((out_rows + 7) / 8), 256, 0, s>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "attn_decode_combine_kernel launch");
  }
  return ATTN_OK;
}

attn_status attn_decode(const void* q, const void* k_cache, const void* v_cache, const int* cache_seqlens, void* o,
                        float* lse, void* workspace, size_t workspace_bytes, int B, int H, int H_kv, int Tq, int Tk,
                        int D, float scale, void* stream) {
  return attn_decode_ex(q, k_cache, v_cache, cache_seqlens, o, lse, workspace, workspace_bytes, B, H, H_kv, Tq, Tk, D,
                        scale, -1, stream);
}

}  // extern "C"

