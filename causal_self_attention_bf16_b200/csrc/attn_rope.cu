// QK normalisation + rotary embedding: the prologue the model applies to q and k before attention, and its
// backward (apidog "Train your own ChatGPT", section 1 "GPT model", architecture features: rotary embeddings
// for relative positions without learned position embeddings, QK normalisation for stability at scale).
//
// The pages give no formula; this file implements
//   y = x / sqrt(mean_d(x^2) + eps)                           RMS normalisation of each head vector, no weight
//   (a, b) -> (a cos w - b sin w, a sin w + b cos w)          RoFormer rotation of each pair (Su et al. 2021)
//   w = p * base^(-2i/D),  p = pos_offsets[b] + t             pair i of the row at time t of sequence b
// with pair i = (2i, 2i+1) (interleaved) or (i, i + D/2) (half). Backward, by the chain rule:
//   g = rotation by -w of dy,   dx = r (g - y mean_d(g y)),   r = (mean_d(x^2) + eps)^(-1/2).
//
// HBM-bound elementwise work, one launch for the rows of q and k together. A thread owns one 16-byte chunk
// (8 of the 128 dims) of a row: 16 threads cover a row, so a half-warp reads 256 contiguous bytes, and a
// 256-thread block covers 16 positions. Every row of a position shares its angles, so a thread computes the
// cos/sin of its pairs once per position (a double product reduced exactly to [-1, 1] half-turns, then
// sincospif) and reuses them over all H + H_kv rows. The RMS and the backward's dot product are 16-lane
// shuffle reductions; for the half pairing the partner chunk comes from lane c ^ 8 by one shuffle.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstdio>

#include "attn.h"
#include "attn_errors.h"

namespace attn {
// This unit's device error word (kind 2 = an address check of the debug build failed, site in the higher bits).
__device__ uint32_t g_rope_error;
}  // namespace attn
using attn::g_rope_error;

namespace {

constexpr int kRopeThreads = 256;
constexpr int kRopeChunks = 16;                            // 16-byte chunks in a 128-dim bf16 row
constexpr int kRopePositions = kRopeThreads / kRopeChunks;  // positions per block iteration
constexpr int kRopeUnroll = 4;                             // rows in flight per thread

struct RopeParams {
  const __nv_bfloat16* x[2];  // q, k as given (the input of the prologue)
  const __nv_bfloat16* g[2];  // gradients of the prologue's outputs (backward only)
  __nv_bfloat16* out[2];      // forward: normalised, rotated q, k; backward: gradients of q, k
  const int* pos_offsets;     // [B] or null
  long long n_pos;            // B * T
  int T;
  int heads[2];               // H, H_kv
  float eps;
  double base;
};

__device__ __forceinline__ void unpack8(const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162*>(&w[i]);
    const float2 v = __bfloat1622float2(h);
    f[2 * i] = v.x;
    f[2 * i + 1] = v.y;
  }
}

__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
    w[i] = *reinterpret_cast<const uint32_t*>(&h);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

__device__ __forceinline__ float sum16(float v) {
#pragma unroll
  for (int m = 1; m < 16; m <<= 1) v += __shfl_xor_sync(0xffffffffu, v, m);
  return v;
}

__device__ __forceinline__ uint4 shfl_xor8(const uint4& u) {
  return make_uint4(__shfl_xor_sync(0xffffffffu, u.x, 8), __shfl_xor_sync(0xffffffffu, u.y, 8),
                    __shfl_xor_sync(0xffffffffu, u.z, 8), __shfl_xor_sync(0xffffffffu, u.w, 8));
}

// Chunk c of row h (q heads first, then k heads) at flat position P = b * T + t, in buffer pair {b0, b1}.
template <typename Ptr>
__device__ __forceinline__ Ptr row_ptr(const RopeParams& p, Ptr b0, Ptr b1, int h, long long P, int c) {
  return h < p.heads[0] ? b0 + (P * p.heads[0] + h) * 128 + 8 * c
                        : b1 + (P * p.heads[1] + (h - p.heads[0])) * 128 + 8 * c;
}

// The 64 pair frequencies in half-turns, base^(-2i/128) / pi, once per block in shared memory.
__device__ __forceinline__ void frequency_table(const RopeParams& p, double* s_fop) {
  if (threadIdx.x < 64)
    s_fop[threadIdx.x] = pow(p.base, -static_cast<double>(threadIdx.x) / 64.0) * 0.31830988618379067154;  // 1/pi
  __syncthreads();
}

// Pair of dim 8c + j: (2i, 2i+1) interleaved, (i, i + 64) half. Sign of the partner term: out = self cos +
// sign * partner sin, -1 for a pair's first member and +1 for its second.
template <bool kHalf>
__device__ __forceinline__ int pair_of(int c, int j) { return kHalf ? ((8 * c + j) & 63) : (4 * c + (j >> 1)); }

template <bool kHalf>
__device__ __forceinline__ float sign_of(int c, int j) { return kHalf ? (c < 8 ? -1.f : 1.f) : ((j & 1) ? 1.f : -1.f); }

template <bool kHalf>
__device__ __forceinline__ void angles(const double* s_fop, int c, double pos, float (&cs)[8], float (&sn)[8]) {
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    if (!kHalf && (j & 1)) {  // interleaved: both members of a pair share the angle
      cs[j] = cs[j - 1];
      sn[j] = sn[j - 1];
      continue;
    }
    double u = pos * s_fop[pair_of<kHalf>(c, j)];  // half-turns
    u -= 2.0 * rint(0.5 * u);                       // exact reduction to [-1, 1]
    sincospif(static_cast<float>(u), &sn[j], &cs[j]);
  }
}

template <bool kHalf>
__device__ __forceinline__ void partner(const uint4& raw, const float (&v)[8], float (&pv)[8]) {
  if (kHalf) {
    unpack8(shfl_xor8(raw), pv);
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) pv[j] = v[j ^ 1];
  }
}

// Debug builds (-DATTN_DEBUG) check each row chunk's address against the rows the host passed before the access;
// a failed check records kind 2 (out of range) with its site in this unit's own device error word (the
// attention kernels' word lives in another translation unit; attn_get_device_error ORs the two) and the access
// is skipped. In the release build the check is the constant true.
constexpr uint32_t kRopeSiteLoad = 0x91, kRopeSiteStore = 0x92;
__device__ __forceinline__ bool row_ok(const RopeParams& p, int h, long long P, int c, uint32_t site) {
#ifdef ATTN_DEBUG
  const bool is_q = h < p.heads[0];
  const long long nh = is_q ? p.heads[0] : p.heads[1];
  const long long off = (P * nh + (is_q ? h : h - p.heads[0])) * 128 + 8 * c;
  if (P >= 0 && h >= 0 && off >= 0 && off + 8 <= p.n_pos * nh * 128) return true;
  atomicOr(&g_rope_error, 2u | (site << 8));
  return false;
#else
  (void)p, (void)h, (void)P, (void)c, (void)site;
  return true;
#endif
}

__device__ __forceinline__ double position(const RopeParams& p, long long P) {
  const int b = static_cast<int>(P / p.T);
  const long long t = P - static_cast<long long>(b) * p.T;
  return static_cast<double>(t) + (p.pos_offsets ? static_cast<double>(p.pos_offsets[b]) : 0.0);
}

constexpr uint4 kZero4 = {0u, 0u, 0u, 0u};

template <bool kHalf>
__global__ void __launch_bounds__(kRopeThreads, 4) qk_norm_rope_kernel(RopeParams p) {
  __shared__ double s_fop[64];
  frequency_table(p, s_fop);
  const int c = threadIdx.x & (kRopeChunks - 1);
  const int slot = threadIdx.x / kRopeChunks;
  const int rows = p.heads[0] + p.heads[1];
  // Every lane stays in the loop (the shuffles involve the whole warp); rows past the end are computed on
  // zeros and not stored. The loop bounds are uniform over the block.
  for (long long P0 = static_cast<long long>(blockIdx.x) * kRopePositions; P0 < p.n_pos;
       P0 += static_cast<long long>(gridDim.x) * kRopePositions) {
    const long long P = P0 + slot;
    const bool valid = P < p.n_pos;
    float cs[8], sn[8];
    angles<kHalf>(s_fop, c, position(p, valid ? P : p.n_pos - 1), cs, sn);
    for (int h0 = 0; h0 < rows; h0 += kRopeUnroll) {
      uint4 raw[kRopeUnroll];
#pragma unroll
      for (int u = 0; u < kRopeUnroll; ++u) {
        const bool live = valid && h0 + u < rows;
        raw[u] = live && row_ok(p, h0 + u, P, c, kRopeSiteLoad)
                     ? *reinterpret_cast<const uint4*>(row_ptr(p, p.x[0], p.x[1], h0 + u, P, c))
                     : kZero4;
      }
#pragma unroll
      for (int u = 0; u < kRopeUnroll; ++u) {
        float x[8], px[8], y[8];
        unpack8(raw[u], x);
        float ss = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) ss = fmaf(x[j], x[j], ss);
        const float r = rsqrtf(sum16(ss) * (1.f / 128.f) + p.eps);
        partner<kHalf>(raw[u], x, px);
#pragma unroll
        for (int j = 0; j < 8; ++j) y[j] = (x[j] * r) * cs[j] + sign_of<kHalf>(c, j) * (px[j] * r) * sn[j];
        if (valid && h0 + u < rows && row_ok(p, h0 + u, P, c, kRopeSiteStore))
          *reinterpret_cast<uint4*>(row_ptr(p, p.out[0], p.out[1], h0 + u, P, c)) = pack8(y);
      }
    }
  }
}

template <bool kHalf>
__global__ void __launch_bounds__(kRopeThreads) qk_norm_rope_bwd_kernel(RopeParams p) {
  __shared__ double s_fop[64];
  frequency_table(p, s_fop);
  const int c = threadIdx.x & (kRopeChunks - 1);
  const int slot = threadIdx.x / kRopeChunks;
  const int rows = p.heads[0] + p.heads[1];
  for (long long P0 = static_cast<long long>(blockIdx.x) * kRopePositions; P0 < p.n_pos;
       P0 += static_cast<long long>(gridDim.x) * kRopePositions) {
    const long long P = P0 + slot;
    const bool valid = P < p.n_pos;
    float cs[8], sn[8];
    angles<kHalf>(s_fop, c, position(p, valid ? P : p.n_pos - 1), cs, sn);
    for (int h0 = 0; h0 < rows; h0 += kRopeUnroll) {
      uint4 xr[kRopeUnroll], gr[kRopeUnroll];
#pragma unroll
      for (int u = 0; u < kRopeUnroll; ++u) {
        const bool live = valid && h0 + u < rows;
        const bool in = live && row_ok(p, h0 + u, P, c, kRopeSiteLoad);
        xr[u] = in ? *reinterpret_cast<const uint4*>(row_ptr(p, p.x[0], p.x[1], h0 + u, P, c)) : kZero4;
        gr[u] = in ? *reinterpret_cast<const uint4*>(row_ptr(p, p.g[0], p.g[1], h0 + u, P, c)) : kZero4;
      }
#pragma unroll
      for (int u = 0; u < kRopeUnroll; ++u) {
        float x[8], dy[8], pdy[8], g[8];
        unpack8(xr[u], x);
        unpack8(gr[u], dy);
        float ss = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) ss = fmaf(x[j], x[j], ss);
        const float r = rsqrtf(sum16(ss) * (1.f / 128.f) + p.eps);
        partner<kHalf>(gr[u], dy, pdy);
        float dot = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          g[j] = dy[j] * cs[j] - sign_of<kHalf>(c, j) * pdy[j] * sn[j];  // rotation by -w
          dot = fmaf(g[j], x[j] * r, dot);
        }
        dot = sum16(dot) * (1.f / 128.f);
#pragma unroll
        for (int j = 0; j < 8; ++j) g[j] = r * (g[j] - (x[j] * r) * dot);
        if (valid && h0 + u < rows && row_ok(p, h0 + u, P, c, kRopeSiteStore))
          *reinterpret_cast<uint4*>(row_ptr(p, p.out[0], p.out[1], h0 + u, P, c)) = pack8(g);
      }
    }
  }
}

// ---------------------------------------------------------------------------------------------- host side

struct Span {
  uintptr_t lo, hi;
};

Span span_of(const void* p, size_t bytes) {
  const uintptr_t a = reinterpret_cast<uintptr_t>(p);
  return {a, a + bytes};
}

bool overlaps(const Span& a, const Span& b) { return a.lo < b.hi && b.lo < a.hi; }
bool same(const Span& a, const Span& b) { return a.lo == b.lo && a.hi == b.hi; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

attn_status check_shape(int B, int T, int H, int H_kv, int D, float rope_base, float eps, int pairing) {
  if (B < 1 || T < 1 || H < 1 || H_kv < 1) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(rope_base) || !(rope_base > 0.f)) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(eps) || eps < 0.f) return ATTN_ERR_INVALID_ARG;
  if (pairing != ATTN_ROPE_INTERLEAVED && pairing != ATTN_ROPE_HALF) return ATTN_ERR_INVALID_ARG;
  if (D != 128) return ATTN_ERR_UNSUPPORTED;
  return ATTN_OK;
}

attn_status launch(bool backward, const RopeParams& p, int pairing, void* stream) {
  const long long blocks = (p.n_pos + kRopePositions - 1) / kRopePositions;
  const unsigned grid = static_cast<unsigned>(blocks < (1LL << 20) ? blocks : (1LL << 20));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (backward) {
    if (pairing == ATTN_ROPE_HALF) qk_norm_rope_bwd_kernel<true><<<grid, kRopeThreads, 0, s>>>(p);
    else qk_norm_rope_bwd_kernel<false><<<grid, kRopeThreads, 0, s>>>(p);
  } else {
    if (pairing == ATTN_ROPE_HALF) qk_norm_rope_kernel<true><<<grid, kRopeThreads, 0, s>>>(p);
    else qk_norm_rope_kernel<false><<<grid, kRopeThreads, 0, s>>>(p);
  }
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    std::snprintf(attn::g_cuda_error, attn::kErrorTextBytes, "%s launch: %s",
                  backward ? "qk_norm_rope_bwd_kernel" : "qk_norm_rope_kernel", cudaGetErrorString(e));
    return ATTN_ERR_CUDA;
  }
  return ATTN_OK;
}

}  // namespace

extern "C" {

attn_status attn_qk_norm_rope(const void* q, const void* k, void* q_out, void* k_out, const int* pos_offsets, int B,
                              int T, int H, int H_kv, int D, float rope_base, float eps, int pairing, void* stream) {
  if (!q || !k || !q_out || !k_out) return ATTN_ERR_INVALID_ARG;
  attn_status st = check_shape(B, T, H, H_kv, D, rope_base, eps, pairing);
  if (st != ATTN_OK) return st;
  for (const void* ptr : {q, k, static_cast<const void*>(q_out), static_cast<const void*>(k_out)})
    if (!aligned16(ptr)) return ATTN_ERR_MISALIGNED;
  if (reinterpret_cast<uintptr_t>(pos_offsets) & 3u) return ATTN_ERR_MISALIGNED;
  const size_t n_pos = static_cast<size_t>(B) * T;
  const Span sq = span_of(q, n_pos * H * 256), sk = span_of(k, n_pos * H_kv * 256);
  const Span oq = span_of(q_out, n_pos * H * 256), ok = span_of(k_out, n_pos * H_kv * 256);
  // in place (an output equal to its own input) is allowed; any other overlap is not
  if ((overlaps(oq, sq) && !same(oq, sq)) || (overlaps(ok, sk) && !same(ok, sk))) return ATTN_ERR_INVALID_ARG;
  if (overlaps(oq, sk) || overlaps(ok, sq) || overlaps(oq, ok)) return ATTN_ERR_INVALID_ARG;
  if (pos_offsets) {
    const Span so = span_of(pos_offsets, static_cast<size_t>(B) * 4);
    if (overlaps(so, oq) || overlaps(so, ok)) return ATTN_ERR_INVALID_ARG;
  }
  RopeParams p{};
  p.x[0] = static_cast<const __nv_bfloat16*>(q);
  p.x[1] = static_cast<const __nv_bfloat16*>(k);
  p.out[0] = static_cast<__nv_bfloat16*>(q_out);
  p.out[1] = static_cast<__nv_bfloat16*>(k_out);
  p.pos_offsets = pos_offsets;
  p.n_pos = static_cast<long long>(n_pos);
  p.T = T;
  p.heads[0] = H;
  p.heads[1] = H_kv;
  p.eps = eps;
  p.base = rope_base;
  return launch(false, p, pairing, stream);
}

attn_status attn_qk_norm_rope_bwd(const void* q, const void* k, const void* dq_out, const void* dk_out, void* dq,
                                  void* dk, const int* pos_offsets, int B, int T, int H, int H_kv, int D,
                                  float rope_base, float eps, int pairing, void* stream) {
  if (!q || !k || !dq_out || !dk_out || !dq || !dk) return ATTN_ERR_INVALID_ARG;
  attn_status st = check_shape(B, T, H, H_kv, D, rope_base, eps, pairing);
  if (st != ATTN_OK) return st;
  for (const void* ptr : {q, k, dq_out, dk_out, static_cast<const void*>(dq), static_cast<const void*>(dk)})
    if (!aligned16(ptr)) return ATTN_ERR_MISALIGNED;
  if (reinterpret_cast<uintptr_t>(pos_offsets) & 3u) return ATTN_ERR_MISALIGNED;
  const size_t n_pos = static_cast<size_t>(B) * T;
  const size_t qb = n_pos * H * 256, kb = n_pos * H_kv * 256;
  const Span sq = span_of(q, qb), sk = span_of(k, kb), gq = span_of(dq_out, qb), gk = span_of(dk_out, kb);
  const Span oq = span_of(dq, qb), ok = span_of(dk, kb);
  // dq may be dq_out itself and dk may be dk_out itself; no other overlap of an output
  if ((overlaps(oq, gq) && !same(oq, gq)) || (overlaps(ok, gk) && !same(ok, gk))) return ATTN_ERR_INVALID_ARG;
  for (const Span& in : {sq, sk}) {
    if (overlaps(oq, in) || overlaps(ok, in)) return ATTN_ERR_INVALID_ARG;
  }
  if (overlaps(oq, gk) || overlaps(ok, gq) || overlaps(oq, ok)) return ATTN_ERR_INVALID_ARG;
  if (pos_offsets) {
    const Span so = span_of(pos_offsets, static_cast<size_t>(B) * 4);
    if (overlaps(so, oq) || overlaps(so, ok)) return ATTN_ERR_INVALID_ARG;
  }
  RopeParams p{};
  p.x[0] = static_cast<const __nv_bfloat16*>(q);
  p.x[1] = static_cast<const __nv_bfloat16*>(k);
  p.g[0] = static_cast<const __nv_bfloat16*>(dq_out);
  p.g[1] = static_cast<const __nv_bfloat16*>(dk_out);
  p.out[0] = static_cast<__nv_bfloat16*>(dq);
  p.out[1] = static_cast<__nv_bfloat16*>(dk);
  p.pos_offsets = pos_offsets;
  p.n_pos = static_cast<long long>(n_pos);
  p.T = T;
  p.heads[0] = H;
  p.heads[1] = H_kv;
  p.eps = eps;
  p.base = rope_base;
  return launch(true, p, pairing, stream);
}

}  // extern "C"

namespace attn {
// Read and clear this unit's device error word (synchronous; the caller has synchronised the device).
int rope_error_word(uint32_t* word) {
  return static_cast<int>(cudaMemcpyFromSymbol(word, g_rope_error, sizeof(uint32_t)));
}
int rope_error_clear() {
  const uint32_t zero = 0;
  return static_cast<int>(cudaMemcpyToSymbol(g_rope_error, &zero, sizeof(uint32_t)));
}
}  // namespace attn
