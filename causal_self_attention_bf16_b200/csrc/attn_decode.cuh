// Attention of a few new queries against a key/value cache, for the inference engine's cached decode
// (apidog "Train your own ChatGPT", section 6 "Inference engine": flash_attn_with_kvcache over a prefilled
// prompt cache).
//
//   q [B, Tq, H, D] bf16; k_cache, v_cache [B, Tk, H_kv, D] bf16; cache_seqlens [B] int32 (valid keys per
//   sequence, the new tokens' keys included). Query i of sequence b sits at position p = L_b - Tq + i and sees
//   keys 0 .. p, or with a sliding window keys p - window .. p. Out: o [B, Tq, H, D] bf16, lse [B, H, Tq] fp32
//   (natural log; -inf and o = 0 for a query that sees no key).
//
// The work is a stream over the cache, HBM-bound (a few FLOPs per byte of K/V), so it runs on CUDA cores:
//   1. attn_decode_split_kernel: one CTA per (sequence, key/value head, chunk of the cache). The G = H / H_kv
//      query heads of the group and their Tq new tokens (R = G * Tq rows) share every K and V row the CTA
//      reads, so the cache is read once. Per block of 128 keys: each thread scores one key against all rows
//      (its K row in registers, the rows in shared memory) while the V block streams into shared memory with
//      16-byte coalesced loads, a warp per row updates the running max and sum (online softmax in base 2), and
//      each thread accumulates one of the 128 output dimensions of every row from the V block. The chunk's
//      unnormalised O, running max and sum go to a workspace. The kernel is instantiated for 1, 2, 4, 8, 16 and
//      32 rows so that the row accumulators of small groups take few registers.
//   2. attn_decode_combine_kernel: one warp per (sequence, query head, new token) merges the chunks by their
//      log-sum-exp and writes o and lse.
#pragma once
#include "attn_common.cuh"
#include "sm100.cuh"

namespace attn {

constexpr int kDecThreads = 128;   // one thread per key of a block and per output dimension
constexpr int kDecKeys = 128;      // keys per block
constexpr int kDecMaxRows = 32;    // R = (H / H_kv) * Tq query rows per CTA, at most
constexpr int kDecChunkKeys = 256; // keys per split of the cache, at least

struct DecodeParams {
  const __nv_bfloat16* q;      // [B, Tq, H, D]
  const __nv_bfloat16* k;      // [B, Tk, H_kv, D]
  const __nv_bfloat16* v;      // [B, Tk, H_kv, D]
  const int* seqlens;          // [B]
  __nv_bfloat16* o;            // [B, Tq, H, D]
  float* lse;                  // [B, H, Tq]
  float* part_o;               // [B * H_kv, n_split, R, D] fp32, unnormalised
  float* part_ml;              // [B * H_kv, n_split, R, 2]: running max (log2 units) and sum
  int B, H, Hkv, Tq, Tk, R, n_split, chunk;
  int window;                  // sliding window: query at position p sees keys p - window .. p; -1: none
  float scale_log2;            // scale * log2(e)
};

// Dynamic shared memory of the split kernel for up to kRows query rows: the rows (fp32, pre-scaled), the
// block's scores, and the block's V rows (bf16).
template <int kRows>
constexpr size_t dec_smem_bytes() {
  return kRows * 128 * 4 + kRows * kDecKeys * 4 + kDecKeys * 128 * 2;
}

template <int kRows>
__global__ void __launch_bounds__(kDecThreads) attn_decode_split_kernel(const DecodeParams p) {
  extern __shared__ float4 dec_smem[];
  float (*qs)[128] = reinterpret_cast<float (*)[128]>(dec_smem);                  // query rows * scale*log2(e)
  float (*sc)[kDecKeys] = reinterpret_cast<float (*)[kDecKeys]>(qs + kRows);      // scores, then P
  __nv_bfloat16 (*vs)[128] = reinterpret_cast<__nv_bfloat16 (*)[128]>(sc + kRows); // the block's V rows
  __shared__ float row_m[kRows], row_l[kRows], row_a[kRows];

  const int t = threadIdx.x, warp = t / 32, lane = t % 32;
  const int bhk = blockIdx.x / p.n_split, sp = blockIdx.x % p.n_split;
  const int b = bhk / p.Hkv, hk = bhk % p.Hkv;
  const int G = p.H / p.Hkv, R = p.R;
  const int L = min(max(p.seqlens[b], 0), p.Tk);   // lengths outside [0, Tk] are clamped
  // The chunks split the keys any row of this sequence sees: from the first row's window start (0 without a
  // window) to the end of the cache.
  const int start = p.window < 0 ? 0 : max(0, L - p.Tq - p.window);
  const int key_lo = start + sp * p.chunk, key_hi = min(L, key_lo + p.chunk);
  const size_t row_stride = static_cast<size_t>(p.Hkv) * 128;   // elements between consecutive keys
  const size_t n_q = static_cast<size_t>(p.B) * p.Tq * p.H * 128, n_kv = static_cast<size_t>(p.B) * p.Tk * row_stride;

  // Row r = g * Tq + i: query head hk * G + g, new token i, which sees keys up to L - Tq + i.
  for (int r = 0; r < R; ++r) {
    const int g = r / p.Tq, i = r % p.Tq;
    const size_t qi = ((static_cast<size_t>(b) * p.Tq + i) * p.H + hk * G + g) * 128 + t;
    qs[r][t] = ATTN_IN_RANGE(qi, 1, n_q, kSiteChkDecQ, &g_device_error) ? __bfloat162float(p.q[qi]) * p.scale_log2
                                                                         : 0.f;
  }
  if (t < R) {
    row_m[t] = -INFINITY;
    row_l[t] = 0.f;
  }
  float acc[kRows];
#pragma unroll
  for (int r = 0; r < kRows; ++r) acc[r] = 0.f;
  __syncthreads();

  for (int kb = key_lo; kb < key_hi; kb += kDecKeys) {
    const int nk = min(kDecKeys, key_hi - kb);
    const size_t kv_off = ((static_cast<size_t>(b) * p.Tk + kb) * p.Hkv + hk) * 128;  // key kb's row
    const __nv_bfloat16* kbase = p.k + kv_off;
    const __nv_bfloat16* vbase = p.v + kv_off;
    // Issue this block's loads first: the thread's K row (16 x 16 bytes) and 16 of the V block's 16-byte
    // chunks (coalesced: consecutive threads, consecutive chunks of a row), so ~64 KB per CTA are in flight.
    uint4 kw[16], vw[16];
#pragma unroll
    for (int c = 0; c < 16; ++c)
      kw[c] = t < nk && ATTN_IN_RANGE(kv_off + t * row_stride + c * 8, 8, n_kv, kSiteChkDecK, &g_device_error)
                  ? reinterpret_cast<const uint4*>(kbase + t * row_stride)[c]
                  : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int idx = u * kDecThreads + t, row = idx / 16, c = idx % 16;
      vw[u] = row < nk && ATTN_IN_RANGE(kv_off + row * row_stride + c * 8, 8, n_kv, kSiteChkDecV, &g_device_error)
                  ? reinterpret_cast<const uint4*>(vbase + row * row_stride)[c]
                  : make_uint4(0, 0, 0, 0);
    }
    // Scores of key kb + t against every row (keys past the block, or past a row's last key, are -inf).
    for (int r = 0; r < R; ++r) {
      const float4* q4 = reinterpret_cast<const float4*>(qs[r]);
      float s0 = 0.f, s1 = 0.f;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const float4 qa = q4[2 * c], qb = q4[2 * c + 1];
        const uint32_t w[4] = {kw[c].x, kw[c].y, kw[c].z, kw[c].w};
        s0 = fmaf(qa.x, __uint_as_float(w[0] << 16), s0);
        s1 = fmaf(qa.y, __uint_as_float(w[0] & 0xffff0000u), s1);
        s0 = fmaf(qa.z, __uint_as_float(w[1] << 16), s0);
        s1 = fmaf(qa.w, __uint_as_float(w[1] & 0xffff0000u), s1);
        s0 = fmaf(qb.x, __uint_as_float(w[2] << 16), s0);
        s1 = fmaf(qb.y, __uint_as_float(w[2] & 0xffff0000u), s1);
        s0 = fmaf(qb.z, __uint_as_float(w[3] << 16), s0);
        s1 = fmaf(qb.w, __uint_as_float(w[3] & 0xffff0000u), s1);
      }
      const int last = L - p.Tq + r % p.Tq;  // last key this row sees (its own position)
      const bool seen = t < nk && kb + t <= last && (p.window < 0 || kb + t >= last - p.window);
      sc[r][t] = seen ? s0 + s1 : -INFINITY;
    }
    // The V block to shared memory (rows past the block are zeros, so P = 0 times them stays 0).
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int idx = u * kDecThreads + t;
      reinterpret_cast<uint4*>(vs)[idx] = vw[u];
    }
    __syncthreads();
    // Online softmax, a warp per row: block max, running max, exp2 in place, running sum, O's rescale factor.
    for (int r = warp; r < R; r += kDecThreads / 32) {
      float x[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) x[e] = sc[r][lane * 4 + e];
      float mb = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, o));
      const float m_old = row_m[r];
      const float m_new = fmaxf(m_old, mb);
      float sum = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float pe = m_new == -INFINITY ? 0.f : exp2f(x[e] - m_new);
        sc[r][lane * 4 + e] = pe;
        sum += pe;
      }
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      __syncwarp();
      if (lane == 0) {
        const float a = m_old == m_new ? 1.f : exp2f(m_old - m_new);  // 0 when nothing was seen before
        row_a[r] = a;
        row_l[r] = row_l[r] * a + sum;
        row_m[r] = m_new;
      }
    }
    __syncthreads();
    // O[r][t] = O[r][t] * a_r + sum_j P[r][j] V[j][t]: thread t is output dimension t.
#pragma unroll
    for (int r = 0; r < kRows; ++r)
      if (r < R) acc[r] *= row_a[r];
    for (int j0 = 0; j0 < nk; j0 += 8) {
      float vv[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) vv[e] = __bfloat162float(vs[j0 + e][t]);
#pragma unroll
      for (int r = 0; r < kRows; ++r) {
        if (r < R) {
          float a = acc[r];
#pragma unroll
          for (int e = 0; e < 8; ++e) a = fmaf(sc[r][j0 + e], vv[e], a);  // P and V are 0 past the block
          acc[r] = a;
        }
      }
    }
    __syncthreads();  // the next block overwrites sc and vs
  }

  // The chunk's partial result (an empty chunk leaves max -inf, sum 0, O 0).
  const size_t n_part = static_cast<size_t>(p.B) * p.Hkv * p.n_split * R;  // partial rows
  const size_t part = (static_cast<size_t>(bhk) * p.n_split + sp) * R;      // this chunk's first one
  float* po = p.part_o + part * 128;
  if (ATTN_IN_RANGE(part, R, n_part, kSiteChkDecPart, &g_device_error)) {
#pragma unroll
    for (int r = 0; r < kRows; ++r)
      if (r < R) po[r * 128 + t] = acc[r];
    if (t < R) {
      float* pml = p.part_ml + (part + t) * 2;
      pml[0] = row_m[t];
      pml[1] = row_l[t];
    }
  }
}

// One warp per output row (b, h, i): O = sum_s O_s 2^(m_s - m) / sum_s l_s 2^(m_s - m), m = max_s m_s.
__global__ void __launch_bounds__(256) attn_decode_combine_kernel(const DecodeParams p) {
  const int row = blockIdx.x * 8 + threadIdx.x / 32, lane = threadIdx.x % 32;
  if (row >= p.B * p.H * p.Tq) return;
  const int i = row % p.Tq, h = (row / p.Tq) % p.H, b = row / (p.Tq * p.H);
  const int G = p.H / p.Hkv, hk = h / G, r = (h % G) * p.Tq + i;
  const size_t base = static_cast<size_t>(b) * p.Hkv + hk;
  const size_t n_part = static_cast<size_t>(p.B) * p.Hkv * p.n_split * p.R;  // partial rows
  if (!ATTN_IN_RANGE((base * p.n_split) * p.R + r, static_cast<size_t>(p.n_split - 1) * p.R + 1, n_part,
                     kSiteChkDecComb, &g_device_error))
    return;  // every partial row of this output (s = 0 .. n_split - 1) must lie in the workspace
  float m = -INFINITY;
  for (int s = 0; s < p.n_split; ++s) m = fmaxf(m, p.part_ml[((base * p.n_split + s) * p.R + r) * 2]);
  float l = 0.f;
  float4 o4 = make_float4(0.f, 0.f, 0.f, 0.f);
  if (m != -INFINITY) {
    for (int s = 0; s < p.n_split; ++s) {
      const float* pml = p.part_ml + ((base * p.n_split + s) * p.R + r) * 2;
      const float ms = pml[0];
      if (ms == -INFINITY) continue;
      const float w = exp2f(ms - m);
      l += pml[1] * w;
      const float4 x = reinterpret_cast<const float4*>(p.part_o + ((base * p.n_split + s) * p.R + r) * 128)[lane];
      o4.x += x.x * w;
      o4.y += x.y * w;
      o4.z += x.z * w;
      o4.w += x.w * w;
    }
  }
  const float inv = l > 0.f ? 1.f / l : 0.f;
  uint2 out;
  out.x = sm100::pack_bf16x2(o4.x * inv, o4.y * inv);
  out.y = sm100::pack_bf16x2(o4.z * inv, o4.w * inv);
  const size_t o_off = ((static_cast<size_t>(b) * p.Tq + i) * p.H + h) * 128;
  if (ATTN_IN_RANGE(o_off + lane * 4, 4, static_cast<size_t>(p.B) * p.Tq * p.H * 128, kSiteChkDecO, &g_device_error))
    reinterpret_cast<uint2*>(p.o + o_off)[lane] = out;
  const size_t lse_i = (static_cast<size_t>(b) * p.H + h) * p.Tq + i;
  if (lane == 0 && ATTN_IN_RANGE(lse_i, 1, static_cast<size_t>(p.B) * p.H * p.Tq, kSiteChkDecLse, &g_device_error))
    p.lse[lse_i] = l > 0.f ? (m + __log2f(l)) * 0.69314718055994531f : -INFINITY;
}

}  // namespace attn
