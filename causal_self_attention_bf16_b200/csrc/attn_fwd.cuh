// Forward kernel of causal multi-head self-attention for sm_100a:
//   O = softmax(scale * Q K^T + causal mask) V, and LSE = natural log-sum-exp of each row's scaled logits.
//
// The pages only call flash_attn_func(q, k, v, causal=True) on [B, T, H, D] bf16 tensors (apidog "Train your
// own ChatGPT", section 5 "Flash Attention integration"; layout from section 1 "GPT model") and name the
// Hopper Flash-Attention-3 kernel as the implementation. This kernel is a new design for Blackwell:
//
//   * one CTA per (128-query tile, batch, head), head-major so a head's K/V stay in L2 while its tiles run,
//     heaviest (latest) query tile of each head first;
//   * warp 0 stages Q once and K/V tiles (three-deep rings) with TMA into 128-byte-swizzled shared memory;
//   * warp 1 issues tcgen05.mma: S = Q K^T (both operands K-major in shared memory) and O += P V (P from
//     tensor memory, V MN-major in shared memory), accumulating in fp32 tensor memory;
//   * warps 2..5 (one thread per query row) run the online softmax straight out of tensor memory: each
//     thread owns a whole row of S, so row max and row sum need no shuffles; masking happens only on the
//     diagonal tile (tiles above it are skipped); O is rescaled lazily, only when the running max grows by
//     more than 2^8; the epilogue normalises O, stages it in shared memory and writes it with a TMA store.
//
// Tensor memory (512 columns): S double buffer [0,256), O [256,384), P double buffer (bf16 pairs) [384,512).
// Issue order of the MMA warp: S(0), S(1), PV(0), S(2), PV(1), ... so that a commit after S(j) also covers
// PV(j-2); that is what frees S buffer j%2 and P buffer j%2 for reuse without further handshakes.
#pragma once
#include "attn_common.cuh"
#include "sm100.cuh"

namespace attn {

constexpr int kTile = 128;        // query rows per CTA and keys per KV tile
constexpr int kHeadDim = 128;     // D
constexpr int kFwdThreads = 192;  // warp 0 TMA, warp 1 MMA, warps 2..5 softmax

// Shared-memory layout of the forward kernel (offsets from a 1024-byte aligned base).
constexpr uint32_t kFwdSmemQ = 0;                       // 32 KB: Q tile, two 64-column boxes of 16 KB
constexpr int kFwdStages = 3;                           // depth of the K and V rings
constexpr uint32_t kFwdSmemK = 32768;                   // 3 x 32 KB: K ring
constexpr uint32_t kFwdSmemV = kFwdSmemK + kFwdStages * 32768;   // 3 x 32 KB: V ring
constexpr uint32_t kFwdSmemBytes = kFwdSmemV + kFwdStages * 32768;  // 224 KB
constexpr uint32_t kFwdSmemAlloc = kFwdSmemBytes + 1024;   // + alignment slack

constexpr uint32_t kTmemS = 0, kTmemO = 256, kTmemP = 384;

// Lazy rescaling threshold on the running max, in log2 units (values of P stay below 2^8).
constexpr float kRescaleThreshold = 8.0f;

struct FwdParams {
  float* lse;        // [B, H, T] fp32
  int B, H, T;
  float scale_log2;  // scale * log2(e)
  uint64_t timeout_ns;
};

struct FwdBarriers {
  uint64_t q_full;
  uint64_t k_full[kFwdStages], k_empty[kFwdStages];
  uint64_t v_full[kFwdStages], v_empty[kFwdStages];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t pv_done;
  uint64_t o_final;  // committed once after the last PV: the epilogue's wait (pv_done may be 2 phases behind)
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

// Error sites (recorded with a timeout in the device error word): 0x10 + barrier id, per role.
enum : uint32_t {
  kSiteFwdProdKEmpty = 0x11, kSiteFwdProdVEmpty = 0x12, kSiteFwdMmaQ = 0x21, kSiteFwdMmaK = 0x22,
  kSiteFwdMmaP = 0x23, kSiteFwdMmaV = 0x24, kSiteFwdSmS = 0x31, kSiteFwdSmPV = 0x32, kSiteFwdEpi = 0x33,
  kSiteFwdDrain = 0x34
};

__global__ void __launch_bounds__(kFwdThreads, 1)
attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                const FwdParams p) {
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base for the 128-byte-swizzle tiles. Offsetting the array itself (not a round trip
  // through an integer) keeps the pointer in the shared address space, so accesses compile to LDS/STS.
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  __shared__ FwdBarriers bars;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int n_qt = (p.T + kTile - 1) / kTile;
  // Head-major order, heaviest (latest) query tile first within a head: the CTAs in flight at any time
  // cover only ~10 heads, so their K/V stay in L2 while every query tile of the head reads them.
  const int bh = static_cast<int>(blockIdx.x / n_qt);
  const int qt = n_qt - 1 - static_cast<int>(blockIdx.x % n_qt);
  const int b = bh / p.H, h = bh % p.H;
  const int q0 = qt * kTile;
  const int n_kv = qt + 1;  // causal: KV tiles 0..qt
  volatile int* abort = &bars.abort;

  if (threadIdx.x == 0) {
    mbar_init(&bars.q_full, 1);
    for (int s = 0; s < kFwdStages; ++s) {
      mbar_init(&bars.k_full[s], 1);
      mbar_init(&bars.k_empty[s], 1);
      mbar_init(&bars.v_full[s], 1);
      mbar_init(&bars.v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars.s_full[s], 1);
      mbar_init(&bars.p_full[s], 128);
    }
    mbar_init(&bars.pv_done, 1);
    mbar_init(&bars.o_final, 1);
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
  if (threadIdx.x == 0) ATTN_TRACE_EVENT(0, 0);

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    // The whole warp walks the loop (warp-uniform control flow, so addresses and coordinates stay in uniform
    // registers); one lane, elected once, issues every copy.
    const bool leader = elect_one();
    if (leader) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      mbar_arrive_expect_tx(&bars.q_full, 2 * 16384);
      for (int c = 0; c < 2; ++c) tma_load_4d(smem + kFwdSmemQ + c * 16384, &tm_q, &bars.q_full, c * 64, h, q0, b);
    }
    int issued_k[kFwdStages], issued_v[kFwdStages];
    for (int s = 0; s < kFwdStages; ++s) issued_k[s] = issued_v[s] = -1;
    for (int j = 0; j < n_kv; ++j) {
      const int s = j % kFwdStages;
      const uint32_t prev = ((j - kFwdStages) / kFwdStages) & 1;  // phase of this slot's previous use
      if (j >= kFwdStages &&
          !mbar_wait_warp(&bars.k_empty[s], prev, abort, p.timeout_ns, &g_device_error, kSiteFwdProdKEmpty))
        break;
      if (leader) {
        mbar_arrive_expect_tx(&bars.k_full[s], 2 * 16384);
        for (int c = 0; c < 2; ++c)
          tma_load_4d(smem + kFwdSmemK + s * 32768 + c * 16384, &tm_k, &bars.k_full[s], c * 64, h, j * kTile, b);
        ATTN_TRACE_EVENT(1, j);
      }
      issued_k[s] = j;
      if (j >= kFwdStages &&
          !mbar_wait_warp(&bars.v_empty[s], prev, abort, p.timeout_ns, &g_device_error, kSiteFwdProdVEmpty))
        break;
      if (leader) {
        mbar_arrive_expect_tx(&bars.v_full[s], 2 * 16384);
        for (int c = 0; c < 2; ++c)
          tma_load_4d(smem + kFwdSmemV + s * 32768 + c * 16384, &tm_v, &bars.v_full[s], c * 64, h, j * kTile, b);
      }
      issued_v[s] = j;
    }
    if (*abort) {
      // Let every copy this warp started land before the CTA's shared memory is released.
      volatile int no_abort = 0;
      const uint64_t lim = p.timeout_ns;
      mbar_wait(&bars.q_full, 0, &no_abort, lim, &g_device_error, kSiteFwdDrain);
      for (int s = 0; s < kFwdStages; ++s) {
        if (issued_k[s] >= 0)
          mbar_wait(&bars.k_full[s], (issued_k[s] / kFwdStages) & 1, &no_abort, lim, &g_device_error, kSiteFwdDrain);
        if (issued_v[s] >= 0)
          mbar_wait(&bars.v_full[s], (issued_v[s] / kFwdStages) & 1, &no_abort, lim, &g_device_error, kSiteFwdDrain);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    // The whole warp walks the schedule and computes the descriptors (warp-uniform, so they live in uniform
    // registers); the lane elected once issues every tcgen05.mma and tcgen05.commit (a commit tracks the
    // MMAs of the thread that issues it, so it must be the same lane throughout).
    const bool leader = elect_one();
    const uint32_t idesc_s = idesc_bf16_f32(128, 128, false, false);  // Q (K-major) x K (K-major)
    const uint32_t idesc_pv = idesc_bf16_f32(128, 128, false, true);  // P (TMEM) x V (MN-major)
    // Descriptors are built once per operand and advanced by adding byte offsets in 16-byte units to the
    // start-address field (one 64-bit add per K step; the tiles stay below 256 KB).
    const uint64_t dq = sdesc_sw128(smem_u32(smem + kFwdSmemQ), 16, 1024);  // Q, K-major
    bool ok = mbar_wait_warp(&bars.q_full, 0, abort, p.timeout_ns, &g_device_error, kSiteFwdMmaQ);
    // PV(jp): O += P(jp) V(jp); P from TMEM buffer jp % 2, V from ring slot jp % kFwdStages.
    auto issue_pv = [&](int jp) -> bool {
      const int pb = jp & 1, vs = jp % kFwdStages;
      if (!mbar_wait_warp(&bars.p_full[pb], (jp >> 1) & 1, abort, p.timeout_ns, &g_device_error, kSiteFwdMmaP))
        return false;
      if (!mbar_wait_warp(&bars.v_full[vs], (jp / kFwdStages) & 1, abort, p.timeout_ns, &g_device_error, kSiteFwdMmaV))
        return false;
      tc_fence_after();
      const uint64_t dv = sdesc_sw128(smem_u32(smem + kFwdSmemV + vs * 32768), 16384, 1024);  // V, MN-major
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)  // K step kk: 16 keys = 2048 bytes further (128 in 16-byte units)
        if (leader) mma_ts(tmem + kTmemO, tmem + kTmemP + pb * 64 + kk * 8, dv + kk * 128, idesc_pv, (jp > 0 || kk > 0) ? 1u : 0u);
      if (leader) {
        mma_commit(&bars.pv_done);
        ATTN_TRACE_EVENT(3, jp);
        mma_commit(&bars.v_empty[vs]);
      }
      return true;
    };
    for (int j = 0; ok && j < n_kv; ++j) {
      const int ks = j % kFwdStages, sb = j & 1;
      if (!mbar_wait_warp(&bars.k_full[ks], (j / kFwdStages) & 1, abort, p.timeout_ns, &g_device_error, kSiteFwdMmaK)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint64_t dk = sdesc_sw128(smem_u32(smem + kFwdSmemK + ks * 32768), 16, 1024);  // K, K-major
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {  // K step kk: second 64-column box from kk = 4, 32 bytes per step within
        const uint32_t koff = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
        if (leader) mma_ss(tmem + kTmemS + sb * 128, dq + koff, dk + koff, idesc_s, kk > 0 ? 1u : 0u);
      }
      if (leader) {
        mma_commit(&bars.s_full[sb]);
        ATTN_TRACE_EVENT(2, j);
        mma_commit(&bars.k_empty[ks]);
      }
      if (j >= 1 && !issue_pv(j - 1)) { ok = false; break; }
    }
    if (ok && issue_pv(n_kv - 1) && leader) mma_commit(&bars.o_final);
    // Drain: wait until every MMA the leader issued has completed before tensor memory is released.
    if (leader) mma_commit(&bars.drain);
    volatile int no_abort = 0;
    mbar_wait(&bars.drain, 0, &no_abort, p.timeout_ns, &g_device_error, kSiteFwdDrain);
  } else {
    // ------------------------------------------------------------------ softmax / correction / epilogue
    const int quarter = warp & 3;           // TMEM lane quarter this warp may access
    const int row = quarter * 32 + lane;    // query row within the tile
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const float c = p.scale_log2;
    float m = -INFINITY;  // running max of scale*log2(e)*S (possibly stale by < 2^8)
    float l = 0.f;        // running row sum of exp2(...)
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      const int sb = j & 1;
      if (!mbar_wait_warp(&bars.s_full[sb], (j >> 1) & 1, abort, p.timeout_ns, &g_device_error, kSiteFwdSmS)) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (threadIdx.x == 64) ATTN_TRACE_EVENT(4, j);
      float s[128];
      {
        uint32_t r0[32], r1[32], r2[32], r3[32];
        tmem_ld32(tmem + lane_base + kTmemS + sb * 128 + 0, r0);
        tmem_ld32(tmem + lane_base + kTmemS + sb * 128 + 32, r1);
        tmem_ld32(tmem + lane_base + kTmemS + sb * 128 + 64, r2);
        tmem_ld32(tmem + lane_base + kTmemS + sb * 128 + 96, r3);
        tmem_wait_ld();
        if (threadIdx.x == 64) ATTN_TRACE_EVENT(8, j);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          s[i] = __uint_as_float(r0[i]);
          s[32 + i] = __uint_as_float(r1[i]);
          s[64 + i] = __uint_as_float(r2[i]);
          s[96 + i] = __uint_as_float(r3[i]);
        }
      }
      if (j == qt) {  // diagonal tile: key column > query row is masked
#pragma unroll
        for (int i = 0; i < 128; ++i)
          if (i > row) s[i] = -INFINITY;
      }
      // Row max as a tree over 16 independent partial maxima (a single 128-long dependent chain would leave
      // ~500 cycles of latency exposed: there is one softmax warp per SM sub-partition).
      float pm[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) pm[i] = s[i];
#pragma unroll
      for (int i = 16; i < 128; ++i) pm[i & 15] = fmaxf(pm[i & 15], s[i]);
#pragma unroll
      for (int w = 8; w >= 1; w >>= 1)
#pragma unroll
        for (int i = 0; i < w; ++i) pm[i] = fmaxf(pm[i], pm[i + w]);
      const float m_tile = pm[0] * c;
      if (threadIdx.x == 64) ATTN_TRACE_EVENT(11, j);
      if (j == 0) {
        m = m_tile;
      } else if (const bool need = m_tile > m + kRescaleThreshold; __any_sync(0xffffffffu, need)) {
        // Some row of this warp saw its running max grow by more than 2^8. TMEM access is warp-collective,
        // so the whole warp walks its rows of O, but only the rows that crossed the threshold change: the
        // others keep their max and get alpha = 1 exactly, so every row's arithmetic is independent of its
        // neighbours (outputs before a position do not depend on inputs after it, bit for bit).
        // O may be touched only after PV(j-1) has landed: S(j) completing implies PV(j-2) completed, and
        // PV(j) is not issued yet, so pv_done is within one phase of j-1 and the parity wait is unambiguous.
        const float m_new = need ? m_tile : m;
        const float alpha = need ? ex2(m - m_new) : 1.0f;
        if (!mbar_wait_warp(&bars.pv_done, (j - 1) & 1, abort, p.timeout_ns, &g_device_error, kSiteFwdSmPV)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t o[32];
          tmem_ld32(tmem + lane_base + kTmemO + cc * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32(tmem + lane_base + kTmemO + cc * 32, o);
        }
        l *= alpha;
        m = m_new;
      }
      // P = exp2(c*S - m), row sum, pack to bf16 pairs into the P buffer of this tile.
      const float neg_m = -m;
      float ps[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};  // 8 independent partial row sums
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float p0 = ex2(fmaf(s[cc * 32 + 2 * i], c, neg_m));
          const float p1 = ex2(fmaf(s[cc * 32 + 2 * i + 1], c, neg_m));
          ps[(2 * i) & 7] += p0;
          ps[(2 * i + 1) & 7] += p1;
          pk[i] = pack_bf16x2(p0, p1);
        }
        tmem_st16(tmem + lane_base + kTmemP + sb * 64 + cc * 16, pk);
      }
      l += ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
      if (threadIdx.x == 64) ATTN_TRACE_EVENT(9, j);
      tmem_wait_st();
      if (threadIdx.x == 64) ATTN_TRACE_EVENT(10, j);
      tc_fence_before();
      mbar_arrive(&bars.p_full[sb]);
      if (threadIdx.x == 64) ATTN_TRACE_EVENT(5, j);
    }
    // Epilogue: O / l -> bf16 -> swizzled staging (reusing the Q buffer) -> TMA store; LSE in natural log.
    // Every thread of the group reaches the named barrier, failed or not; the store is skipped on abort.
    if (threadIdx.x == 64) ATTN_TRACE_EVENT(6, 0);
    const bool epi_ok =
        __all_sync(0xffffffffu, ok) && mbar_wait_warp(&bars.o_final, 0, abort, p.timeout_ns, &g_device_error, kSiteFwdEpi);
    if (epi_ok) {
      if (threadIdx.x == 64) ATTN_TRACE_EVENT(7, 0);
      tc_fence_after();
      const float inv_l = 1.0f / l;
      uint8_t* stage = smem + kFwdSmemQ;
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_base + kTmemO + cc * 32, o);
        tmem_wait_ld();
        uint8_t* box = stage + (cc >> 1) * 16384;
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          uint4 v;
          v.x = pack_bf16x2(__uint_as_float(o[ch * 8 + 0]) * inv_l, __uint_as_float(o[ch * 8 + 1]) * inv_l);
          v.y = pack_bf16x2(__uint_as_float(o[ch * 8 + 2]) * inv_l, __uint_as_float(o[ch * 8 + 3]) * inv_l);
          v.z = pack_bf16x2(__uint_as_float(o[ch * 8 + 4]) * inv_l, __uint_as_float(o[ch * 8 + 5]) * inv_l);
          v.w = pack_bf16x2(__uint_as_float(o[ch * 8 + 6]) * inv_l, __uint_as_float(o[ch * 8 + 7]) * inv_l);
          *reinterpret_cast<uint4*>(box + sw128_offset(row, (cc & 1) * 4 + ch)) = v;
        }
      }
      const int t = q0 + row;
      if (t < p.T) p.lse[static_cast<size_t>(bh) * p.T + t] = (m + __log2f(l)) * 0.69314718055994531f;
    }
    fence_async_shared();
    named_barrier(1, 128);
    if (warp == 2 && lane == 0 && !*abort) {
      for (int cc = 0; cc < 2; ++cc) tma_store_4d(&tm_o, smem + kFwdSmemQ + cc * 16384, cc * 64, h, q0, b);
      tma_store_commit();
      tma_store_wait_read_all();
      ATTN_TRACE_EVENT(6, 1);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) ATTN_TRACE_EVENT(0, 1);
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace attn
