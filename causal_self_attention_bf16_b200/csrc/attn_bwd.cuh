// Backward kernels of causal multi-head self-attention for sm_100a: dQ, dK, dV from Q, K, V, O, LSE, dO.
//
// Definition (textbook backward of softmax attention; the pages train through flash_attn_func but print no
// formula: apidog "Train your own ChatGPT", section 5 "Flash Attention integration"):
//   P = exp(scale*Q K^T - LSE) (causal), dV = P^T dO, dP = dO V^T, Delta = rowsum(dO * O),
//   dS = P * (dP - Delta), dQ = scale * dS K, dK = scale * dS^T Q.
//
// Three launches on the caller's stream:
//   1. attn_bwd_prep_kernel: Delta (fp32, from the stored bf16 O), LSE * log2(e), and zeroing of the fp32 dQ
//      accumulator. Rows past T are padded with LSE = +inf and Delta = 0 so they contribute nothing.
//   2. attn_bwd_dkdv_kernel: one CTA per (128-key tile, batch, head) walks the 64-query tiles at or after
//      its keys. Per query tile, five tcgen05 MMAs:
//        S^T = K Q^T, dP^T = V dO^T            (K-major operands in shared memory)
//        dV += P^T dO, dK += dS^T Q             (P^T, dS^T from tensor memory; dO, Q MN-major)
//        dQ^T = K^T dS^T                        (both operands MN-major in shared memory)
//      One thread per key row turns S^T, dP^T into P^T, dS^T (exp2 against the stored LSE); a second warp
//      group reads dQ^T out of tensor memory and adds it into the fp32 accumulator with 16-byte vector
//      reductions laid out so that each warp instruction covers 512 contiguous bytes. dK, dV stay in tensor
//      memory for the whole walk and leave through a TMA store.
//   3. attn_bwd_dq_kernel: dQ = bf16(scale * accumulator) back in [B, T, H, D].
//
// Tensor memory of the dK/dV kernel (512 columns): dV [0,128), dK [128,256), and two 128-column tile
// buffers R0 = [256,384), R1 = [384,512). A buffer holds S^T in its first 64 columns and dP^T in the last
// 64; after the softmax step its first 32 columns hold P^T and the next 32 dS^T (bf16 pairs), and the dQ^T
// MMA writes its last 64 columns.
#pragma once
#include "attn_common.cuh"
#include "sm100.cuh"

namespace attn {

constexpr int kBwdQTile = 64;       // queries per inner tile
constexpr int kBwdKTile = 128;      // keys per CTA
constexpr int kBwdStages = 3;       // Q/dO/LSE/Delta ring depth
constexpr int kBwdThreads = 320;    // warp 0 TMA, warp 1 MMA, warps 2..5 softmax, warps 6..9 dQ

constexpr uint32_t kBwdSmemK = 0;                                 // 32 KB
constexpr uint32_t kBwdSmemV = 32768;                             // 32 KB
constexpr uint32_t kBwdSmemQ = 65536;                             // 3 x 16 KB (two 8 KB boxes each)
constexpr uint32_t kBwdSmemDO = kBwdSmemQ + kBwdStages * 16384;   // 3 x 16 KB
constexpr uint32_t kBwdSmemDS = kBwdSmemDO + kBwdStages * 16384;  // 2 x 16 KB: dS^T [128 keys][64 q]
constexpr uint32_t kBwdSmemLse = kBwdSmemDS + 2 * 16384;          // 3 x 256 B
constexpr uint32_t kBwdSmemDelta = kBwdSmemLse + kBwdStages * 256;  // 3 x 256 B
constexpr uint32_t kBwdSmemBytes = kBwdSmemDelta + kBwdStages * 256;
constexpr uint32_t kBwdSmemAlloc = kBwdSmemBytes + 1024;

constexpr uint32_t kTmemDV = 0, kTmemDK = 128, kTmemR = 256;

// Round T up to a multiple of 128: the padded length of the per-row workspace arrays.
__host__ __device__ constexpr int padded_T(int T) { return (T + 127) / 128 * 128; }

struct BwdParams {
  const __nv_bfloat16* o;    // [B, T, H, D]
  const __nv_bfloat16* dO;   // [B, T, H, D]
  const float* lse;          // [B, H, T]
  float* lse2;               // [B*H, Tp]  LSE * log2(e), +inf past T
  float* delta;              // [B*H, Tp]  rowsum(dO * O), 0 past T
  float* dq_acc;             // [B*H, Tp/4, D, 4] fp32
  __nv_bfloat16* dq;         // [B, T, H, D]
  int B, H, T, Tp;
  float scale, scale_log2;
  uint64_t timeout_ns;
};

// ------------------------------------------------------------------------------------------------ prep

// One 16-thread group per (b, t, h) row: Delta = sum_d dO * O in fp32; LSE * log2(e); zero the accumulator.
__global__ void __launch_bounds__(256) attn_bwd_prep_kernel(const BwdParams p) {
  const int64_t rows = static_cast<int64_t>(p.B) * p.H * p.Tp;  // padded rows, ordered (bh, t)
  const int sub = threadIdx.x & 15;
  const int64_t group = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 4;
  const int64_t ngroups = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 4;
  for (int64_t r = group; r < rows; r += ngroups) {
    const int bh = static_cast<int>(r / p.Tp), t = static_cast<int>(r % p.Tp);
    const int b = bh / p.H, h = bh % p.H;
    float acc = 0.f;
    if (t < p.T) {
      const size_t off = ((static_cast<size_t>(b) * p.T + t) * p.H + h) * 128 + sub * 8;
      const uint4 ov = *reinterpret_cast<const uint4*>(p.o + off);
      const uint4 gv = *reinterpret_cast<const uint4*>(p.dO + off);
      const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&ov);
      const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&gv);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 of = __bfloat1622float2(o2[i]);
        const float2 gf = __bfloat1622float2(g2[i]);
        acc = fmaf(of.x, gf.x, acc);
        acc = fmaf(of.y, gf.y, acc);
      }
    }
#pragma unroll
    for (int w = 8; w >= 1; w >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, w, 16);
    if (sub == 0) {
      p.delta[r] = acc;
      p.lse2[r] = t < p.T ? p.lse[static_cast<size_t>(bh) * p.T + t] * 1.4426950408889634f : INFINITY;
    }
  }
  // Zero the dQ accumulator with 16-byte stores.
  const int64_t n4 = static_cast<int64_t>(p.B) * p.H * p.Tp * 128 / 4;
  float4* acc4 = reinterpret_cast<float4*>(p.dq_acc);
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    acc4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// ------------------------------------------------------------------------------------------------ dQ out

// dq[b, t, h, d] = bf16(scale * acc[bh, t/4, d, t%4]). One thread per (bh, t/4, 4 consecutive d).
__global__ void __launch_bounds__(256) attn_bwd_dq_kernel(const BwdParams p) {
  const int64_t t4n = (p.T + 3) / 4;
  const int64_t items = static_cast<int64_t>(p.B) * p.H * t4n * 32;
  for (int64_t it = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; it < items;
       it += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int dc = static_cast<int>(it & 31);         // d chunk: d = 4*dc .. 4*dc+3
    const int64_t rest = it >> 5;
    const int t4 = static_cast<int>(rest % t4n);
    const int bh = static_cast<int>(rest / t4n);
    const int b = bh / p.H, h = bh % p.H;
    const float4* src = reinterpret_cast<const float4*>(p.dq_acc + static_cast<size_t>(bh) * p.Tp * 128 +
                                                        static_cast<size_t>(t4) * 512 + dc * 16);
    const float4 a0 = src[0], a1 = src[1], a2 = src[2], a3 = src[3];  // d = 4dc+0..3, each holding t%4 = 0..3
    const float s = p.scale;
    const float v[4][4] = {{a0.x, a1.x, a2.x, a3.x}, {a0.y, a1.y, a2.y, a3.y}, {a0.z, a1.z, a2.z, a3.z},
                           {a0.w, a1.w, a2.w, a3.w}};
#pragma unroll
    for (int tt = 0; tt < 4; ++tt) {
      const int t = t4 * 4 + tt;
      if (t < p.T) {
        uint2 w;
        w.x = sm100::pack_bf16x2(v[tt][0] * s, v[tt][1] * s);
        w.y = sm100::pack_bf16x2(v[tt][2] * s, v[tt][3] * s);
        *reinterpret_cast<uint2*>(p.dq + ((static_cast<size_t>(b) * p.T + t) * p.H + h) * 128 + dc * 4) = w;
      }
    }
  }
}

// ------------------------------------------------------------------------------------------------ dK/dV

struct BwdBarriers {
  uint64_t kv_full;
  uint64_t q_full[kBwdStages], q_empty[kBwdStages];
  uint64_t s_full[2];    // S^T, dP^T of buffer b ready
  uint64_t p_full[2];    // P^T, dS^T written (TMEM + smem)
  uint64_t dq_full[2];   // dQ^T of buffer b ready (also: dV, dK MMAs of that tile done)
  uint64_t dq_empty[2];  // dQ^T read out: buffer b free
  uint64_t acc_done;     // all MMAs done (epilogue)
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

enum : uint32_t {
  kSiteBwdProdQEmpty = 0x41, kSiteBwdMmaKV = 0x51, kSiteBwdMmaQ = 0x52, kSiteBwdMmaDqEmpty = 0x53,
  kSiteBwdMmaP = 0x54, kSiteBwdSmS = 0x61, kSiteBwdSmQ = 0x62, kSiteBwdSmEpi = 0x63, kSiteBwdDq = 0x71,
  kSiteBwdDrain = 0x72
};

__device__ __forceinline__ void red_add_v4(float* addr, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}

__global__ void __launch_bounds__(kBwdThreads, 1)
attn_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                     const __grid_constant__ CUtensorMap tm_dk, const __grid_constant__ CUtensorMap tm_dv,
                     const BwdParams p) {
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ BwdBarriers bars;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int BH = p.B * p.H;
  const int kt = static_cast<int>(blockIdx.x / BH);  // key tile; low tiles (most query tiles) first
  const int bh = static_cast<int>(blockIdx.x % BH);
  const int b = bh / p.H, h = bh % p.H;
  const int k0 = kt * kBwdKTile;
  const int n_q64 = (p.T + kBwdQTile - 1) / kBwdQTile;
  const int i0 = k0 / kBwdQTile;           // first query tile that sees these keys
  const int n = n_q64 - i0;                // query tiles this CTA walks (>= 1)
  volatile int* abort = &bars.abort;

  if (threadIdx.x == 0) {
    mbar_init(&bars.kv_full, 1);
    for (int s = 0; s < kBwdStages; ++s) {
      mbar_init(&bars.q_full[s], 1);
      mbar_init(&bars.q_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars.s_full[s], 1);
      mbar_init(&bars.p_full[s], 128);
      mbar_init(&bars.dq_full[s], 1);
      mbar_init(&bars.dq_empty[s], 128);
    }
    mbar_init(&bars.acc_done, 1);
    mbar_init(&bars.drain, 1);
    bars.abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_do);
      mbar_arrive_expect_tx(&bars.kv_full, 4 * 16384);
      for (int c = 0; c < 2; ++c) {
        tma_load_4d(smem + kBwdSmemK + c * 16384, &tm_k, &bars.kv_full, c * 64, h, k0, b);
        tma_load_4d(smem + kBwdSmemV + c * 16384, &tm_v, &bars.kv_full, c * 64, h, k0, b);
      }
      int last_issued[kBwdStages] = {-1, -1, -1};
      for (int i = 0; i < n; ++i) {
        const int s = i % kBwdStages;
        if (i >= kBwdStages && !mbar_wait(&bars.q_empty[s], ((i - kBwdStages) / kBwdStages) & 1, abort,
                                          p.timeout_ns, &g_device_error, kSiteBwdProdQEmpty))
          break;
        const int q0 = (i0 + i) * kBwdQTile;
        mbar_arrive_expect_tx(&bars.q_full[s], 2 * 16384 + 2 * 256);
        for (int c = 0; c < 2; ++c) {
          tma_load_4d(smem + kBwdSmemQ + s * 16384 + c * 8192, &tm_q, &bars.q_full[s], c * 64, h, q0, b);
          tma_load_4d(smem + kBwdSmemDO + s * 16384 + c * 8192, &tm_do, &bars.q_full[s], c * 64, h, q0, b);
        }
        bulk_load(smem + kBwdSmemLse + s * 256, p.lse2 + static_cast<size_t>(bh) * p.Tp + q0, 256, &bars.q_full[s]);
        bulk_load(smem + kBwdSmemDelta + s * 256, p.delta + static_cast<size_t>(bh) * p.Tp + q0, 256, &bars.q_full[s]);
        last_issued[s] = i;
      }
      if (*abort) {
        volatile int no_abort = 0;
        mbar_wait(&bars.kv_full, 0, &no_abort, p.timeout_ns, &g_device_error, kSiteBwdDrain);
        for (int s = 0; s < kBwdStages; ++s)
          if (last_issued[s] >= 0)
            mbar_wait(&bars.q_full[s], (last_issued[s] / kBwdStages) & 1, &no_abort, p.timeout_ns, &g_device_error,
                      kSiteBwdDrain);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t id_s = idesc_bf16_f32(128, 64, false, false);   // K x Q^T, V x dO^T
      const uint32_t id_acc = idesc_bf16_f32(128, 128, false, true); // P^T (TMEM) x dO, dS^T (TMEM) x Q
      const uint32_t id_dq = idesc_bf16_f32(128, 64, true, true);    // K^T (MN-major) x dS^T (MN-major)
      const uint32_t sk = smem_u32(smem + kBwdSmemK), sv = smem_u32(smem + kBwdSmemV);
      bool ok = mbar_wait(&bars.kv_full, 0, abort, p.timeout_ns, &g_device_error, kSiteBwdMmaKV);
      tc_fence_after();
      // A(i): S^T and dP^T of query tile i into buffer i%2.
      auto issue_a = [&](int i) -> bool {
        const int s = i % kBwdStages, rb = i & 1;
        if (!mbar_wait(&bars.q_full[s], (i / kBwdStages) & 1, abort, p.timeout_ns, &g_device_error, kSiteBwdMmaQ))
          return false;
        if (i >= 2 && !mbar_wait(&bars.dq_empty[rb], ((i - 2) >> 1) & 1, abort, p.timeout_ns, &g_device_error,
                                 kSiteBwdMmaDqEmpty))
          return false;
        tc_fence_after();
        const uint32_t sq = smem_u32(smem + kBwdSmemQ + s * 16384), sdo = smem_u32(smem + kBwdSmemDO + s * 16384);
        const uint32_t r = tmem + kTmemR + rb * 128;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t ka = (kk >> 2) * 16384 + (kk & 3) * 32;  // 128-row boxes
          const uint32_t kb = (kk >> 2) * 8192 + (kk & 3) * 32;   // 64-row boxes
          mma_ss(r, sdesc_sw128(sk + ka, 16, 1024), sdesc_sw128(sq + kb, 16, 1024), id_s, kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t ka = (kk >> 2) * 16384 + (kk & 3) * 32;
          const uint32_t kb = (kk >> 2) * 8192 + (kk & 3) * 32;
          mma_ss(r + 64, sdesc_sw128(sv + ka, 16, 1024), sdesc_sw128(sdo + kb, 16, 1024), id_s, kk > 0);
        }
        mma_commit(&bars.s_full[rb]);
        return true;
      };
      // B(i): dV += P^T dO, dK += dS^T Q, dQ^T = K^T dS^T.
      auto issue_b = [&](int i) -> bool {
        const int s = i % kBwdStages, rb = i & 1;
        if (!mbar_wait(&bars.p_full[rb], (i >> 1) & 1, abort, p.timeout_ns, &g_device_error, kSiteBwdMmaP))
          return false;
        tc_fence_after();
        const uint32_t sq = smem_u32(smem + kBwdSmemQ + s * 16384), sdo = smem_u32(smem + kBwdSmemDO + s * 16384);
        const uint32_t sds = smem_u32(smem + kBwdSmemDS + rb * 16384);
        const uint32_t r = tmem + kTmemR + rb * 128;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ts(tmem + kTmemDV, r + kk * 8, sdesc_sw128(sdo + kk * 2048, 8192, 1024), id_acc, (i > 0 || kk > 0));
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ts(tmem + kTmemDK, r + 32 + kk * 8, sdesc_sw128(sq + kk * 2048, 8192, 1024), id_acc, (i > 0 || kk > 0));
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss(r + 64, sdesc_sw128(sk + kk * 2048, 16384, 1024), sdesc_sw128(sds + kk * 2048, 8192, 1024), id_dq,
                 kk > 0);
        mma_commit(&bars.dq_full[rb]);
        mma_commit(&bars.q_empty[s]);
        return true;
      };
      // Pairs: A(i), A(i+1), B(i), B(i+1): the dQ read-out of one tile overlaps the MMAs of the next.
      for (int i = 0; ok && i < n; i += 2) {
        ok = issue_a(i) && (i + 1 >= n || issue_a(i + 1));
        ok = ok && issue_b(i) && (i + 1 >= n || issue_b(i + 1));
      }
      mma_commit(&bars.acc_done);
      mma_commit(&bars.drain);
      volatile int no_abort = 0;
      mbar_wait(&bars.drain, 0, &no_abort, p.timeout_ns, &g_device_error, kSiteBwdDrain);
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------------ softmax: one thread per key row
    const int quarter = warp & 3;
    const int krow = quarter * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const int kg = k0 + krow;
    const float c = p.scale_log2;
    bool ok = true;
    for (int i = 0; i < n; ++i) {
      const int s = i % kBwdStages, rb = i & 1;
      const int q0 = (i0 + i) * kBwdQTile;
      if (!mbar_wait_warp(&bars.q_full[s], (i / kBwdStages) & 1, abort, p.timeout_ns, &g_device_error, kSiteBwdSmQ) ||
          !mbar_wait_warp(&bars.s_full[rb], (i >> 1) & 1, abort, p.timeout_ns, &g_device_error, kSiteBwdSmS)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t r = tmem + lane_base + kTmemR + rb * 128;
      const float* lse2 = reinterpret_cast<const float*>(smem + kBwdSmemLse + s * 256);
      const float* dlt = reinterpret_cast<const float*>(smem + kBwdSmemDelta + s * 256);
      float pr[64];
      {
        uint32_t a[32], bb[32];
        tmem_ld32(r + 0, a);
        tmem_ld32(r + 32, bb);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 32; ++q) {
          pr[q] = ex2(fmaf(__uint_as_float(a[q]), c, -lse2[q]));
          pr[32 + q] = ex2(fmaf(__uint_as_float(bb[q]), c, -lse2[32 + q]));
        }
      }
      if (q0 < k0 + kBwdKTile) {  // query tile overlaps the key tile: queries before a key see nothing
#pragma unroll
        for (int q = 0; q < 64; ++q)
          if (q0 + q < kg) pr[q] = 0.f;
      }
      uint8_t* dsrow = smem + kBwdSmemDS + rb * 16384;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t dp[32];
        tmem_ld32(r + 64 + hh * 32, dp);
        tmem_wait_ld();
        uint32_t ppk[16], dpk[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          const int qa = hh * 32 + 2 * q, qb = qa + 1;
          const float ds0 = pr[qa] * (__uint_as_float(dp[2 * q]) - dlt[qa]);
          const float ds1 = pr[qb] * (__uint_as_float(dp[2 * q + 1]) - dlt[qb]);
          ppk[q] = pack_bf16x2(pr[qa], pr[qb]);
          dpk[q] = pack_bf16x2(ds0, ds1);
        }
        tmem_st16(r + hh * 16, ppk);
        tmem_st16(r + 32 + hh * 16, dpk);
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          uint4 v = make_uint4(dpk[ch * 4 + 0], dpk[ch * 4 + 1], dpk[ch * 4 + 2], dpk[ch * 4 + 3]);
          *reinterpret_cast<uint4*>(dsrow + sw128_offset(krow, hh * 4 + ch)) = v;
        }
      }
      tmem_wait_st();
      fence_async_shared();
      tc_fence_before();
      mbar_arrive(&bars.p_full[rb]);
    }
    // Epilogue: dV and scale*dK from TMEM -> bf16 -> swizzled staging -> TMA store (rows past T are clipped).
    // Every thread of the group reaches the named barrier, failed or not; the stores are skipped on abort.
    const bool epi_ok = __all_sync(0xffffffffu, ok) &&
                        mbar_wait_warp(&bars.acc_done, 0, abort, p.timeout_ns, &g_device_error, kSiteBwdSmEpi);
    if (epi_ok) {
      tc_fence_after();
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        uint8_t* stage = smem + (which == 0 ? kBwdSmemQ : kBwdSmemDO);  // 32 KB each (first two stages)
        const float mul = which == 0 ? 1.0f : p.scale;
        const uint32_t col = which == 0 ? kTmemDV : kTmemDK;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t o[32];
          tmem_ld32(tmem + lane_base + col + cc * 32, o);
          tmem_wait_ld();
          uint8_t* box = stage + (cc >> 1) * 16384;
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) {
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(o[ch * 8 + 0]) * mul, __uint_as_float(o[ch * 8 + 1]) * mul);
            v.y = pack_bf16x2(__uint_as_float(o[ch * 8 + 2]) * mul, __uint_as_float(o[ch * 8 + 3]) * mul);
            v.z = pack_bf16x2(__uint_as_float(o[ch * 8 + 4]) * mul, __uint_as_float(o[ch * 8 + 5]) * mul);
            v.w = pack_bf16x2(__uint_as_float(o[ch * 8 + 6]) * mul, __uint_as_float(o[ch * 8 + 7]) * mul);
            *reinterpret_cast<uint4*>(box + sw128_offset(krow, (cc & 1) * 4 + ch)) = v;
          }
        }
      }
    }
    fence_async_shared();
    named_barrier(1, 128);
    if (warp == 2 && lane == 0 && !*abort) {
      for (int cc = 0; cc < 2; ++cc) {
        tma_store_4d(&tm_dv, smem + kBwdSmemQ + cc * 16384, cc * 64, h, k0, b);
        tma_store_4d(&tm_dk, smem + kBwdSmemDO + cc * 16384, cc * 64, h, k0, b);
      }
      tma_store_commit();
      tma_store_wait_read_all();
    }
  } else {
    // ------------------------------------------------------------------ dQ^T read-out: one thread per d
    const int quarter = warp & 3;
    const int d = quarter * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    float* acc_bh = p.dq_acc + static_cast<size_t>(bh) * p.Tp * 128;
    for (int i = 0; i < n; ++i) {
      const int rb = i & 1;
      const int q0 = (i0 + i) * kBwdQTile;
      if (!mbar_wait_warp(&bars.dq_full[rb], (i >> 1) & 1, abort, p.timeout_ns, &g_device_error, kSiteBwdDq)) break;
      tc_fence_after();
      uint32_t a[32], bb[32];
      tmem_ld32(tmem + lane_base + kTmemR + rb * 128 + 64, a);
      tmem_ld32(tmem + lane_base + kTmemR + rb * 128 + 96, bb);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&bars.dq_empty[rb]);
      float* dst = acc_bh + static_cast<size_t>(q0 >> 2) * 512 + d * 4;
#pragma unroll
      for (int q4 = 0; q4 < 8; ++q4)
        red_add_v4(dst + q4 * 512, __uint_as_float(a[4 * q4]), __uint_as_float(a[4 * q4 + 1]),
                   __uint_as_float(a[4 * q4 + 2]), __uint_as_float(a[4 * q4 + 3]));
#pragma unroll
      for (int q4 = 0; q4 < 8; ++q4)
        red_add_v4(dst + (8 + q4) * 512, __uint_as_float(bb[4 * q4]), __uint_as_float(bb[4 * q4 + 1]),
                   __uint_as_float(bb[4 * q4 + 2]), __uint_as_float(bb[4 * q4 + 3]));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace attn
