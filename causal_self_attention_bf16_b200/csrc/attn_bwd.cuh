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
//   2. attn_bwd_dkdv_kernel: one CTA per (128-key tile, batch, key/value head) walks the 64-query tiles at
//      or after its keys, of every query head that reads this key/value head (one, or a group of them with
//      grouped-query attention). Per query tile, five tcgen05 MMAs:
//        S^T = K Q^T, dP^T = V dO^T            (K-major operands in shared memory)
//        dV += P^T dO, dK += dS^T Q             (P^T, dS^T from tensor memory; dO, Q MN-major)
//        dQ^T = K^T dS^T                        (both operands MN-major in shared memory)
//      Two warp groups taking alternate query tiles (one thread per key row) turn S^T, dP^T into P^T, dS^T
//      (exp2 against the stored LSE), then read their tile's dQ^T out of tensor memory and stage it in shared
//      memory in the accumulator's layout; a reduction warp adds it into the fp32 accumulator with one bulk
//      reduction (cp.reduce.async.bulk .add.f32, 32 contiguous KB) on the async engine. dK, dV stay in tensor memory
//      for the whole walk; the groups stage them in shared memory and the K/V warp stores them by TMA while
//      the groups go on with the next key tile.
//   3. attn_bwd_dq_kernel: dQ = bf16(scale * accumulator) back in [B, T, H, D].
//
// Tensor memory of the dK/dV kernel (512 columns): dV [0,128), dK [128,256), and two 128-column tile
// buffers R0 = [256,384), R1 = [384,512). A buffer holds S^T in its first 64 columns and dP^T in the last
// 64; after the softmax step, for each half h of the 64 queries, columns [32h, 32h+16) hold P^T and
// [32h+16, 32h+32) hold dS^T (bf16 pairs) of those 32 queries, and the dQ^T MMA writes the last 64 columns.
#pragma once
#include <type_traits>

#include "attn_common.cuh"
#include "sm100.cuh"

namespace attn {

constexpr int kBwdQTile = 64;       // queries per inner tile
constexpr int kBwdKTile = 128;      // keys per CTA
constexpr int kBwdStages = 3;       // Q/dO/LSE/Delta ring depth
constexpr int kBwdThreads = 384;    // warp 0 TMA (query tiles), warp 1 MMA, warps 2..9 two softmax/dQ
                                    // groups, warp 10 TMA (K, V in; dV, dK out), warp 11 dQ reductions
constexpr int kBwdWarpKV = 10, kBwdWarpReduce = 11;

constexpr uint32_t kBwdSmemK = 0;                                 // 32 KB
constexpr uint32_t kBwdSmemV = 32768;                             // 32 KB
constexpr uint32_t kBwdSmemQ = 65536;                             // 3 x 16 KB (two 8 KB boxes each)
constexpr uint32_t kBwdSmemDO = kBwdSmemQ + kBwdStages * 16384;   // 3 x 16 KB
constexpr uint32_t kBwdSmemDS = kBwdSmemDO + kBwdStages * 16384;  // 2 x 16 KB: dS^T [128 keys][64 q]
constexpr uint32_t kBwdSmemDQ = kBwdSmemDS + 2 * 16384;           // 32 KB: a dQ^T tile staged for its bulk reduce
constexpr uint32_t kBwdSmemLse = kBwdSmemDQ + 32768;              // 3 x 256 B
constexpr uint32_t kBwdSmemDelta = kBwdSmemLse + kBwdStages * 256;  // 3 x 256 B
constexpr uint32_t kBwdSmemBytes = kBwdSmemDelta + kBwdStages * 256;  // barriers follow (see BwdBarriers)

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
  int Hkv;                   // key/value heads (divides H): the dK/dV kernel's CTA covers one of them
  int window;                // sliding window: query i sees keys i - window .. i; -1: no window
  float scale, scale_log2;
  uint64_t timeout_ns;
};

// ------------------------------------------------------------------------------------------------ prep

// One 16-thread group per (bh, four consecutive padded rows): Delta = sum_d dO * O in fp32 and LSE * log2(e)
// for the four rows, and zeroing of the accumulator block that holds them (2 KB, contiguous in the [t/4][d][4]
// layout). Each thread has its eight 16-byte loads (four rows of o and dO) in flight at once, and every group
// writes as many bytes as it reads, so the read and write streams interleave over the whole grid.
__global__ void __launch_bounds__(256) attn_bwd_prep_kernel(const BwdParams p) {
  const int64_t quads = static_cast<int64_t>(p.B) * p.H * (p.Tp / 4);  // ordered (bh, t/4)
  const size_t n_lse = static_cast<size_t>(p.B) * p.H * p.T, n_in = n_lse * 128;  // lse; o and dO
  const size_t n_rows = static_cast<size_t>(p.B) * p.H * p.Tp;                       // padded rows
  const int sub = threadIdx.x & 15;
  const int64_t group = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 4;
  const int64_t ngroups = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 4;
  for (int64_t qd = group; qd < quads; qd += ngroups) {
    const int bh = static_cast<int>(qd / (p.Tp / 4)), t0 = static_cast<int>(qd % (p.Tp / 4)) * 4;
    const int b = bh / p.H, h = bh % p.H;
    uint4 ov[4], gv[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      ov[j] = make_uint4(0u, 0u, 0u, 0u);
      gv[j] = make_uint4(0u, 0u, 0u, 0u);
      const size_t off = ((static_cast<size_t>(b) * p.T + t0 + j) * p.H + h) * 128 + sub * 8;
      if (t0 + j < p.T && ATTN_IN_RANGE(off, 8, n_in, kSiteChkPrepIn, &g_device_error)) {
        ov[j] = *reinterpret_cast<const uint4*>(p.o + off);
        gv[j] = *reinterpret_cast<const uint4*>(p.dO + off);
      }
    }
    // zero the block of these four rows: 512 floats, 8 float4 per thread
    const size_t blk_off = static_cast<size_t>(bh) * p.Tp * 128 + static_cast<size_t>(t0) * 128;
    float4* blk = reinterpret_cast<float4*>(p.dq_acc + blk_off);
    if (ATTN_IN_RANGE(blk_off, 512, n_rows * 128, kSiteChkPrepAcc, &g_device_error)) {
#pragma unroll
      for (int j = 0; j < 8; ++j) blk[j * 16 + sub] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float acc[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&ov[j]);
      const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&gv[j]);
      acc[j] = 0.f;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 of = __bfloat1622float2(o2[i]);
        const float2 gf = __bfloat1622float2(g2[i]);
        acc[j] = fmaf(of.x, gf.x, acc[j]);
        acc[j] = fmaf(of.y, gf.y, acc[j]);
      }
    }
#pragma unroll
    for (int w = 8; w >= 1; w >>= 1)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], w, 16);
    if (sub < 4) {  // thread j of the group writes row t0 + j
      const int t = t0 + sub;
      const float a = sub == 0 ? acc[0] : sub == 1 ? acc[1] : sub == 2 ? acc[2] : acc[3];
      const int64_t r = static_cast<int64_t>(bh) * p.Tp + t;
      const size_t li = static_cast<size_t>(bh) * p.T + t;
      const bool lse_ok = t < p.T && ATTN_IN_RANGE(li, 1, n_lse, kSiteChkPrepLse, &g_device_error);
      if (ATTN_IN_RANGE(r, 1, n_rows, kSiteChkPrepRow, &g_device_error)) {
        p.delta[r] = a;
        p.lse2[r] = lse_ok ? p.lse[li] * 1.4426950408889634f : INFINITY;
      }
    }
  }
}

// ------------------------------------------------------------------------------------------------ dQ out

// dq[b, t, h, d] = bf16(scale * acc[bh, t/4, d, t%4]). One thread per (bh, t/4, 4 consecutive d): 64
// contiguous accumulator bytes in, 8 bytes of four rows out (a warp writes whole 256-byte rows). Each thread
// takes two items per pass of the grid-stride loop and issues both items' loads before either's stores.
__global__ void __launch_bounds__(256) attn_bwd_dq_kernel(const BwdParams p) {
  const int64_t t4n = (p.T + 3) / 4;
  const int64_t items = static_cast<int64_t>(p.B) * p.H * t4n * 32;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const size_t n_acc = static_cast<size_t>(p.B) * p.H * p.Tp * 128, n_dq = static_cast<size_t>(p.B) * p.T * p.H * 128;
  for (int64_t it0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; it0 < items; it0 += 2 * stride) {
    float4 a[2][4] = {};
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int64_t it = it0 + u * stride;
      if (it < items) {
        const int dc = static_cast<int>(it & 31);  // d chunk: d = 4*dc .. 4*dc+3
        const int64_t rest = it >> 5;
        const int t4 = static_cast<int>(rest % t4n);
        const int bh = static_cast<int>(rest / t4n);
        const size_t off = static_cast<size_t>(bh) * p.Tp * 128 + static_cast<size_t>(t4) * 512 + dc * 16;
        const float4* src = reinterpret_cast<const float4*>(p.dq_acc + off);
        if (ATTN_IN_RANGE(off, 16, n_acc, kSiteChkDqIn, &g_device_error)) {
#pragma unroll
          for (int c = 0; c < 4; ++c) a[u][c] = src[c];  // d = 4dc + c, holding t%4 = 0..3
        }
      }
    }
    const float s = p.scale;
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int64_t it = it0 + u * stride;
      if (it >= items) break;
      const int dc = static_cast<int>(it & 31);
      const int64_t rest = it >> 5;
      const int t4 = static_cast<int>(rest % t4n);
      const int bh = static_cast<int>(rest / t4n);
      const int b = bh / p.H, h = bh % p.H;
      const float4* x = a[u];
      const float v[4][4] = {{x[0].x, x[1].x, x[2].x, x[3].x}, {x[0].y, x[1].y, x[2].y, x[3].y},
                             {x[0].z, x[1].z, x[2].z, x[3].z}, {x[0].w, x[1].w, x[2].w, x[3].w}};
#pragma unroll
      for (int tt = 0; tt < 4; ++tt) {
        const int t = t4 * 4 + tt;
        const size_t off = ((static_cast<size_t>(b) * p.T + t) * p.H + h) * 128 + dc * 4;
        if (t < p.T && ATTN_IN_RANGE(off, 4, n_dq, kSiteChkDqOut, &g_device_error)) {
          uint2 w;
          w.x = sm100::pack_bf16x2(v[tt][0] * s, v[tt][1] * s);
          w.y = sm100::pack_bf16x2(v[tt][2] * s, v[tt][3] * s);
          *reinterpret_cast<uint2*>(p.dq + off) = w;
        }
      }
    }
  }
}

// ------------------------------------------------------------------------------------------------ dK/dV

struct BwdBarriers {
  uint64_t k_full, v_full;  // K / V of the current work item landed (one phase per item)
  uint64_t k_free, v_free;  // the MMAs that read an item's K / V are done: the next item's may load
  uint64_t kv_issued;       // an item's K and V loads are issued: its query tiles may queue behind them
  uint64_t q_full[kBwdStages], q_empty[kBwdStages];
  uint64_t s_full[2];    // S^T, dP^T of buffer b ready
  uint64_t p_full[2];    // P^T, dS^T written (TMEM + smem)
  uint64_t dq_full[2];   // dQ^T of buffer b ready
  uint64_t dq_empty[2];  // dQ^T read out: buffer b's last 64 columns free
  uint64_t b_done[2];    // dV, dK MMAs of the step in buffer b done (buffer's P^T, dS^T consumed)
  uint64_t dq_staged[2];   // a step's dQ^T tile is staged for its reduction: [gs % 2], arrived by that step's
                          // group leader after the group's staging barrier (one phase per step of that group)
  uint64_t stage_free[2];  // the dQ staging buffer has been read by the bulk reduction of a step: [gs % 2],
                          // arrived by the reduction warp (one phase per step of that group)
  uint64_t acc_done;     // every MMA of an item done: its dV, dK are final (one phase per item)
  uint64_t acc_free;     // dV, dK read out of tensor memory by the epilogue (8 warps, one phase per item)
  uint64_t dk_staged;    // an item's dK staged in the dS^T buffers for its store (4 warps, one phase per item)
  uint64_t dv_staged;    // an item's dV staged in the dQ staging buffer for its store (4 warps, one phase per item)
  uint64_t ds_read;      // an item's dK stores have read the dS^T buffers (one phase per item)
  uint64_t dq_read;      // an item's dV stores have read the dQ staging buffer (one phase per item)
  uint64_t drain;
  float* red_dst[2];     // accumulator address of the tile staged for dq_staged[g], written before that arrival
  uint32_t tmem_base;
  int abort;
};
// The kernel uses no static shared memory, so the dynamic block starts 1024-byte aligned and needs no slack
// (the kernel checks this and refuses to run otherwise): tiles, then the barriers. 226 KB in all.
constexpr uint32_t kBwdSmemAlloc = kBwdSmemBytes + sizeof(BwdBarriers);
static_assert(kBwdSmemAlloc <= 232448, "dK/dV kernel exceeds the 227 KB shared-memory opt-in");

enum : uint32_t {
  kSiteBwdLayout = 0x40, kSiteBwdProdQEmpty = 0x41, kSiteBwdProdKV = 0x42, kSiteBwdMmaKV = 0x51, kSiteBwdMmaQ = 0x52,
  kSiteBwdMmaDqEmpty = 0x53, kSiteBwdMmaP = 0x54, kSiteBwdMmaAcc = 0x55, kSiteBwdSmS = 0x61, kSiteBwdSmQ = 0x62,
  kSiteBwdSmEpi = 0x63, kSiteBwdSmEpiRead = 0x64, kSiteBwdKvEpi = 0x43, kSiteBwdDq = 0x71, kSiteBwdDrain = 0x72,
  kSiteBwdReduce = 0x73
};

// Work item k of this CTA: one 128-key tile of one key/value head. Items are ordered head-major with the
// heaviest key tile (the first, seen by every query tile) first within a head, and dealt to the CTAs in rounds
// that alternate direction, as the forward does: the CTAs in flight cover only ~10 heads, so their Q, dO and
// the heads' fp32 dQ accumulators stay in L2, and the causal work per CTA evens out.
struct BwdItem {
  int b, hk, kt;
  int i0, n;  // query tiles i0 .. i0+n-1 of every query head of the group see these keys
};
// The host caps B * H * ceil(T / 128) at 2^30, so item indices (fewer than that plus one round of CTAs) fit in
// 32 bits and decode with 32-bit divisions.
__device__ __forceinline__ bool bwd_item(int k, const BwdParams& p, BwdItem& it) {
  const unsigned n_kt = static_cast<unsigned>(p.T + kBwdKTile - 1) / kBwdKTile;
  const unsigned n_items = static_cast<unsigned>(p.B) * static_cast<unsigned>(p.Hkv) * n_kt;
  const unsigned G = gridDim.x, c = blockIdx.x;
  const unsigned idx = static_cast<unsigned>(k) * G + ((k & 1) ? G - 1 - c : c);
  if (idx >= n_items) return false;
  const int bhk = static_cast<int>(idx / n_kt);
  it.kt = static_cast<int>(idx % n_kt);
  it.b = bhk / p.Hkv;
  it.hk = bhk % p.Hkv;
  const int n_q64 = (p.T + kBwdQTile - 1) / kBwdQTile;
  const int k0 = it.kt * kBwdKTile;
  it.i0 = k0 / kBwdQTile;  // first query tile that sees these keys
  // last query tile + 1: all of them, or with a sliding window those holding queries <= k0 + 127 + window
  const int i_end = p.window < 0 ? n_q64 : min(n_q64, (k0 + kBwdKTile - 1 + p.window) / kBwdQTile + 1);
  it.n = i_end - it.i0;
  return true;
}

// Persistent: one CTA per SM walks its work items. Every ring slot, tensor-memory buffer and per-step barrier
// phase follows a running step count over all of the CTA's items (gs), every per-item barrier phase the item
// count (k), so the query tiles of the next item stream in during the current one, and the next item's V and K
// load as soon as the last MMA that reads this item's has completed.
__global__ void __launch_bounds__(kBwdThreads, 1)
attn_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                     const __grid_constant__ CUtensorMap tm_dk, const __grid_constant__ CUtensorMap tm_dv,
                     const BwdParams p) {
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base for the 128-byte-swizzle tiles. Offsetting the array itself (not a round trip
  // through an integer) keeps the pointer in the shared address space, so accesses compile to LDS/STS.
  uint8_t* smem = smem_raw;
  if (smem_u32(smem_raw) & 1023u) {  // the layout below needs a 1024-byte aligned dynamic block
    if (threadIdx.x == 0) atomicOr(&g_device_error, sm100::DEV_ERR_TIMEOUT | (kSiteBwdLayout << 8));
    return;
  }
  BwdBarriers& bars = *reinterpret_cast<BwdBarriers*>(smem + kBwdSmemBytes);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int G = p.H / p.Hkv;  // query heads per key/value head: a step is (query head, 64-query tile)
  volatile int* abort = &bars.abort;
  const uint64_t lim = p.timeout_ns;

  if (threadIdx.x == 0) {
    mbar_init(&bars.k_full, 1);
    mbar_init(&bars.v_full, 1);
    mbar_init(&bars.k_free, 1);
    mbar_init(&bars.v_free, 1);
    mbar_init(&bars.kv_issued, 1);
    for (int s = 0; s < kBwdStages; ++s) {
      mbar_init(&bars.q_full[s], 1);
      mbar_init(&bars.q_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars.s_full[s], 1);
      mbar_init(&bars.p_full[s], 4);    // counts the warps of one softmax group
      mbar_init(&bars.dq_full[s], 1);
      mbar_init(&bars.dq_empty[s], 4);  // likewise
      mbar_init(&bars.b_done[s], 1);
    }
    mbar_init(&bars.dq_staged[0], 1);
    mbar_init(&bars.dq_staged[1], 1);
    mbar_init(&bars.stage_free[0], 1);
    mbar_init(&bars.stage_free[1], 1);
    mbar_init(&bars.acc_done, 1);
    mbar_init(&bars.acc_free, 8);  // the warps of both groups
    mbar_init(&bars.dk_staged, 4);
    mbar_init(&bars.dv_staged, 4);
    mbar_init(&bars.ds_read, 1);
    mbar_init(&bars.dq_read, 1);
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
    // ------------------------------------------------------------------ TMA producer: query tiles
    // Q, dO, LSE*log2(e) and Delta of every step through the ring. The whole warp walks the loop (warp-uniform
    // control flow, so addresses and coordinates stay in uniform registers); one lane, elected once, issues.
    const bool leader = elect_one();
    if (leader) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_do);
    }
    int last_issued[kBwdStages];
    for (int s = 0; s < kBwdStages; ++s) last_issued[s] = -1;
    int gs = 0;
    bool ok = true;
    BwdItem it;
    for (int k = 0; ok && bwd_item(k, p, it); ++k) {
      // An item's K loads only once the previous item's last MMAs have read that item's K, and its first S^T
      // MMA waits for it; its first dP^T MMA needs only V, loaded earlier, and the first dO tile. So the item's
      // first two query tiles go out as soon as their ring slots are free, ahead of K, and the later ones
      // queue behind K on the copy engine (with nothing else in flight, the CTA's first item loads K and V
      // first). The wait on kv_issued comes exactly once per item, so its parity never skips a phase.
      const int ns = G * it.n;
      const int kv_gate = k == 0 ? 0 : min(2, ns - 1);
      for (int i = 0; i < ns; ++i, ++gs) {
        const int s = gs % kBwdStages;
        if (i == kv_gate && !mbar_wait_warp(&bars.kv_issued, k & 1, abort, lim, &g_device_error, kSiteBwdProdQEmpty)) {
          ok = false;
          break;
        }
        if (gs >= kBwdStages && !mbar_wait_warp(&bars.q_empty[s], ((gs - kBwdStages) / kBwdStages) & 1, abort, lim,
                                                &g_device_error, kSiteBwdProdQEmpty)) {
          ok = false;
          break;
        }
        const int h = it.hk * G + i / it.n, bh = it.b * p.H + h;  // the step's query head
        const int q0 = (it.i0 + i % it.n) * kBwdQTile;
        if (leader) {
          // the step's 64 rows of LSE*log2(e) and Delta (plain addresses: checked in the debug build, where a
          // failed check skips the two loads and the barrier expects only the tiles)
          const size_t roff = static_cast<size_t>(bh) * p.Tp + q0;
          const bool rows_ok =
              ATTN_IN_RANGE(roff, 64, static_cast<size_t>(p.B) * p.H * p.Tp, kSiteChkBwdRows, &g_device_error);
          mbar_arrive_expect_tx(&bars.q_full[s], 2 * 16384 + (rows_ok ? 2 * 256 : 0));
          for (int c = 0; c < 2; ++c) {
            tma_load_4d(smem + kBwdSmemQ + s * 16384 + c * 8192, &tm_q, &bars.q_full[s], c * 64, h, q0, it.b);
            tma_load_4d(smem + kBwdSmemDO + s * 16384 + c * 8192, &tm_do, &bars.q_full[s], c * 64, h, q0, it.b);
          }
          if (rows_ok) {
            bulk_load(smem + kBwdSmemLse + s * 256, p.lse2 + roff, 256, &bars.q_full[s]);
            bulk_load(smem + kBwdSmemDelta + s * 256, p.delta + roff, 256, &bars.q_full[s]);
          }
          ATTN_TRACE_EVENT(1, gs);
        }
        last_issued[s] = gs;
      }
    }
    if (*abort) {
      volatile int no_abort = 0;
      for (int s = 0; s < kBwdStages; ++s)
        if (last_issued[s] >= 0)
          mbar_wait(&bars.q_full[s], (last_issued[s] / kBwdStages) & 1, &no_abort, lim, &g_device_error,
                    kSiteBwdDrain);
    }
  } else if (warp == kBwdWarpKV) {
    // ------------------------------------------------------------------ TMA: K and V in, dV and dK out
    // V is read only by the dP^T MMAs, K also by the dQ^T MMAs of the last step: each loads for the next item
    // as soon as the MMAs that read the current one have completed. Both come from DRAM (a key tile is read by
    // one CTA only), so the next item's are first prefetched into L2 while the current item is computed.
    // This warp also stores each item's dK as soon as it is staged in the two dS^T buffers and reports when the
    // store has read them (ds_read: the next item's first step writes a dS^T buffer early), then dV, staged in
    // the dQ staging buffer (dq_read: the dQ staging comes at a step's end). The softmax groups go on with the
    // next item meanwhile and wait for a report only before they write to that buffer again. In time, item
    // k-1's stores come after item k's K load.
    const bool leader = elect_one();
    int k_issued = -1, v_issued = -1;
    BwdItem it, nx, prev;
    auto store_epilogue = [&](int k, const BwdItem& e) -> bool {  // item k = e: dK, then dV, to global
      const int r0 = e.kt * kBwdKTile;
      if (!mbar_wait_warp(&bars.dk_staged, k & 1, abort, lim, &g_device_error, kSiteBwdKvEpi)) return false;
      if (leader && !*abort) {
        for (int c = 0; c < 2; ++c) tma_store_4d(&tm_dk, smem + kBwdSmemDS + c * 16384, c * 64, e.hk, r0, e.b);
        tma_store_commit();
        tma_store_wait_read<0>();
        mbar_arrive(&bars.ds_read);
      }
      __syncwarp();
      if (!mbar_wait_warp(&bars.dv_staged, k & 1, abort, lim, &g_device_error, kSiteBwdKvEpi)) return false;
      if (leader && !*abort) {
        for (int c = 0; c < 2; ++c) tma_store_4d(&tm_dv, smem + kBwdSmemDQ + c * 16384, c * 64, e.hk, r0, e.b);
        tma_store_commit();
        tma_store_wait_read<0>();
        mbar_arrive(&bars.dq_read);
      }
      __syncwarp();
      return true;
    };
    int k = 0;
    bool ok = true;
    for (; bwd_item(k, p, it); ++k) {
      const int k0 = it.kt * kBwdKTile;
      if (leader && bwd_item(k + 1, p, nx))
        for (int c = 0; c < 2; ++c) {
          tma_prefetch_l2_4d(&tm_k, c * 64, nx.hk, nx.kt * kBwdKTile, nx.b);
          tma_prefetch_l2_4d(&tm_v, c * 64, nx.hk, nx.kt * kBwdKTile, nx.b);
        }
      if (k >= 1 && !mbar_wait_warp(&bars.v_free, (k - 1) & 1, abort, lim, &g_device_error, kSiteBwdProdKV)) {
        ok = false;
        break;
      }
      if (leader) {
        mbar_arrive_expect_tx(&bars.v_full, 2 * 16384);
        for (int c = 0; c < 2; ++c)
          tma_load_4d(smem + kBwdSmemV + c * 16384, &tm_v, &bars.v_full, c * 64, it.hk, k0, it.b);
      }
      v_issued = k;
      if (k >= 1 && !mbar_wait_warp(&bars.k_free, (k - 1) & 1, abort, lim, &g_device_error, kSiteBwdProdKV)) {
        ok = false;
        break;
      }
      if (leader) {
        mbar_arrive_expect_tx(&bars.k_full, 2 * 16384);
        for (int c = 0; c < 2; ++c)
          tma_load_4d(smem + kBwdSmemK + c * 16384, &tm_k, &bars.k_full, c * 64, it.hk, k0, it.b);
      }
      k_issued = k;
      mbar_arrive_warp(&bars.kv_issued);
      if (k >= 1 && !store_epilogue(k - 1, prev)) {
        ok = false;
        break;
      }
      prev = it;
    }
    if (ok && k >= 1) store_epilogue(k - 1, prev);  // the last item's
    if (leader) tma_store_wait_all();  // the stores are complete before the CTA exits
    if (*abort) {
      volatile int no_abort = 0;
      if (v_issued >= 0) mbar_wait(&bars.v_full, v_issued & 1, &no_abort, lim, &g_device_error, kSiteBwdDrain);
      if (k_issued >= 0) mbar_wait(&bars.k_full, k_issued & 1, &no_abort, lim, &g_device_error, kSiteBwdDrain);
    }
  } else if (warp == kBwdWarpReduce) {
    // ------------------------------------------------------------------ dQ reductions
    // Each step's dQ^T tile, staged by its softmax group in the accumulator's layout, is one contiguous 32 KB
    // block of the fp32 accumulator: one bulk reduce-add on the async engine adds it in. This warp issues them
    // in step order and waits for each to have read the staging buffer before handing the buffer on
    // (stage_free), so no softmax warp ever stalls on that read.
    const bool leader = elect_one();
    const size_t acc_floats = static_cast<size_t>(p.B) * p.H * p.Tp * 128;
    int gs = 0;
    bool ok = true;
    BwdItem it;
    for (int k = 0; ok && bwd_item(k, p, it); ++k) {
      const int ns = G * it.n;
      for (int i = 0; i < ns; ++i, ++gs) {
        const int g = gs & 1;
        if (!mbar_wait_warp(&bars.dq_staged[g], (gs >> 1) & 1, abort, lim, &g_device_error, kSiteBwdReduce)) {
          ok = false;
          break;
        }
        if (leader) {
          // the tile's 8192 accumulator floats (checked in the debug build; a failed check skips the reduction)
          float* dst = bars.red_dst[g];
          if (ATTN_IN_RANGE(static_cast<size_t>(dst - p.dq_acc), 8192, acc_floats, kSiteChkBwdReduce, &g_device_error))
            bulk_reduce_add_f32(dst, smem + kBwdSmemDQ, 32768);
          tma_store_commit();
          tma_store_wait_read_all();  // the staging buffer has been read: hand it to the next step
          mbar_arrive(&bars.stage_free[g]);
          ATTN_TRACE_EVENT(7, gs);
        }
        __syncwarp();
      }
    }
    if (leader) tma_store_wait_all();  // the reductions are complete before the CTA exits
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    // The whole warp walks the schedule and computes the descriptors (warp-uniform, so they live in uniform
    // registers); the lane elected once issues every tcgen05.mma and tcgen05.commit (a commit tracks the
    // MMAs of the thread that issues it, so it must be the same lane throughout).
    const bool leader = elect_one();
    const uint32_t id_s = idesc_bf16_f32(128, 64, false, false);   // K x Q^T, V x dO^T
    const uint32_t id_acc = idesc_bf16_f32(128, 128, false, true); // P^T (TMEM) x dO, dS^T (TMEM) x Q
    const uint32_t id_dq = idesc_bf16_f32(128, 64, true, true);    // K^T (MN-major) x dS^T (MN-major)
    // Shared-memory descriptors are built once per operand and advanced by adding the byte offset in
    // 16-byte units to the start-address field (a K step is one 64-bit add; tiles stay below 256 KB).
    const uint64_t dk_kmaj = sdesc_sw128(smem_u32(smem + kBwdSmemK), 16, 1024);      // K as K-major A
    const uint64_t dv_kmaj = sdesc_sw128(smem_u32(smem + kBwdSmemV), 16, 1024);      // V as K-major A
    const uint64_t dk_mnmaj = sdesc_sw128(smem_u32(smem + kBwdSmemK), 16384, 1024);  // K^T as MN-major A
    // A(gs): dP^T and S^T of step gs into buffer gs%2, once its Q/dO tile has landed. dP^T goes first: it
    // overwrites the buffer's last 64 columns, free once the softmax group has read dQ^T of step gs-2 out of
    // them; S^T overwrites the first 64, where P^T and dS^T of step gs-2 stay until the dV and dK MMAs of
    // B(gs-2) have read them, so that wait comes second and overlaps dP^T's execution. An item's first step
    // also waits for the item's V (before dP^T) and K (before S^T).
    auto issue_a = [&](int gs, bool first, int k) -> bool {
      const int s = gs % kBwdStages, rb = gs & 1;
      if (!mbar_wait_warp(&bars.q_full[s], (gs / kBwdStages) & 1, abort, lim, &g_device_error, kSiteBwdMmaQ))
        return false;
      if (gs >= 2 && !mbar_wait_warp(&bars.dq_empty[rb], ((gs - 2) >> 1) & 1, abort, lim, &g_device_error,
                                     kSiteBwdMmaDqEmpty))
        return false;
      if (first && !mbar_wait_warp(&bars.v_full, k & 1, abort, lim, &g_device_error, kSiteBwdMmaKV)) return false;
      if (leader) ATTN_TRACE_EVENT(12, gs);
      tc_fence_after();
      const uint64_t dq0 = sdesc_sw128(smem_u32(smem + kBwdSmemQ + s * 16384), 16, 1024);
      const uint64_t ddo0 = sdesc_sw128(smem_u32(smem + kBwdSmemDO + s * 16384), 16, 1024);
      const uint32_t r = tmem + kTmemR + rb * 128;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t ka = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;  // 128-row boxes, in 16-byte units
        const uint32_t kb = ((kk >> 2) * 8192 + (kk & 3) * 32) >> 4;   // 64-row boxes
        if (leader) mma_ss(r + 64, dv_kmaj + ka, ddo0 + kb, id_s, kk > 0);
      }
      if (gs >= 2 && !mbar_wait_warp(&bars.b_done[rb], ((gs - 2) >> 1) & 1, abort, lim, &g_device_error,
                                     kSiteBwdMmaDqEmpty))
        return false;
      if (first && !mbar_wait_warp(&bars.k_full, k & 1, abort, lim, &g_device_error, kSiteBwdMmaKV)) return false;
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t ka = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
        const uint32_t kb = ((kk >> 2) * 8192 + (kk & 3) * 32) >> 4;
        if (leader) mma_ss(r, dk_kmaj + ka, dq0 + kb, id_s, kk > 0);
      }
      if (leader) {
        mma_commit(&bars.s_full[rb]);
        ATTN_TRACE_EVENT(2, gs);
      }
      return true;
    };
    // B(gs): dQ^T = K^T dS^T first (its own commit, so the read-out of dQ^T overlaps the rest), then
    // dV += P^T dO and dK += dS^T Q (commit: the step's buffer and its Q/dO ring slot are free). An item's
    // last dQ^T is the last MMA to read its K; its first dV, dK MMAs overwrite the accumulators, which the
    // previous item's epilogue must have read out.
    auto issue_b = [&](int gs, bool first, bool last, int k) -> bool {
      const int s = gs % kBwdStages, rb = gs & 1;
      if (!mbar_wait_warp(&bars.p_full[rb], (gs >> 1) & 1, abort, lim, &g_device_error, kSiteBwdMmaP))
        return false;
      tc_fence_after();
      const uint64_t dq_mn = sdesc_sw128(smem_u32(smem + kBwdSmemQ + s * 16384), 8192, 1024);
      const uint64_t ddo_mn = sdesc_sw128(smem_u32(smem + kBwdSmemDO + s * 16384), 8192, 1024);
      const uint64_t dds_mn = sdesc_sw128(smem_u32(smem + kBwdSmemDS + rb * 16384), 8192, 1024);
      const uint32_t r = tmem + kTmemR + rb * 128;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        if (leader) mma_ss(r + 64, dk_mnmaj + kk * 128, dds_mn + kk * 128, id_dq, kk > 0);
      if (leader) {
        mma_commit(&bars.dq_full[rb]);
        if (last) mma_commit(&bars.k_free);
      }
      if (first && k >= 1 &&
          !mbar_wait_warp(&bars.acc_free, (k - 1) & 1, abort, lim, &g_device_error, kSiteBwdMmaAcc))
        return false;
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        if (leader)
          mma_ts(tmem + kTmemDV, r + (kk >> 1) * 32 + (kk & 1) * 8, ddo_mn + kk * 128, id_acc, (!first || kk > 0));
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        if (leader)
          mma_ts(tmem + kTmemDK, r + (kk >> 1) * 32 + 16 + (kk & 1) * 8, dq_mn + kk * 128, id_acc, (!first || kk > 0));
      if (leader) {
        mma_commit(&bars.b_done[rb]);
        mma_commit(&bars.q_empty[s]);
        ATTN_TRACE_EVENT(3, gs);
      }
      return true;
    };
    // Per item: A(0), A(1), B(0), A(2), B(1), ..., A(n-1), B(n-2), B(n-1). While the softmax group of step i
    // works (from the end of A(i) until B(i) can start), the tensor core has B(i-1) and A(i+1) to do, a whole
    // step of MMAs; the groups' steps alternate, so their softmax phases hardly overlap.
    bool ok = true;
    int gs = 0;
    BwdItem it;
    for (int k = 0; ok && bwd_item(k, p, it); ++k) {
      const int ns = G * it.n;
      ok = issue_a(gs, true, k);
      for (int i = 1; ok && i < ns; ++i) ok = issue_a(gs + i, false, k) && issue_b(gs + i - 1, i == 1, false, k);
      if (ok && leader) mma_commit(&bars.v_free);  // every dP^T of the item (the last in A(n-1)) issued
      ok = ok && issue_b(gs + ns - 1, ns == 1, true, k);
      if (ok && leader) mma_commit(&bars.acc_done);
      gs += ns;
    }
    if (leader) mma_commit(&bars.drain);
    volatile int no_abort = 0;
    mbar_wait(&bars.drain, 0, &no_abort, lim, &g_device_error, kSiteBwdDrain);
  } else {
    // ------------------------------------------------------------------ softmax: one thread per (key row, half)
    // Two warp groups alternate steps (ping-pong): group g (warps 2..5 or 6..9) handles the steps with
    // gs % 2 == g, which are exactly the steps of tensor-memory buffer g, so each group has a whole step of
    // tensor-core work to hide its softmax behind. A thread handles one key row, in two halves of 32 query
    // columns; each half's packed P^T and dS^T (16 + 16 columns) go over that half's own 32 columns of S^T.
    // After an item's steps both groups write its dV (group 0) and dK (group 1).
    const int g = (warp - 2) >> 2;
    const int quarter = warp & 3;
    const int krow = quarter * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const float c = p.scale_log2;
    const bool group_leader = lane == 0 && quarter == 2;  // first warp of the group
    float* dq_stage = reinterpret_cast<float*>(smem + kBwdSmemDQ);
    // The staging buffer passes between the groups in step order. Step gs's reduction reports on
    // stage_free[gs % 2], so a group waits only on the other group's barrier, whose phase can be neither behind
    // nor ahead of the wait by more than one: the other group's next arrival needs this group's next staging.
    // (With one barrier for both groups a warp could wait two phases ahead of it -- its own leader's arrival
    // for the previous step still pending -- and a parity wait would then pass at once.)
    auto wait_staged = [&](int step) -> bool {  // the reduction of `step` has read the staging buffer
      return mbar_wait_warp(&bars.stage_free[step & 1], (step >> 1) & 1, abort, lim, &g_device_error, kSiteBwdDq);
    };
    bool ok = true;
    int gs0 = 0;  // running step count at the start of the item
    BwdItem it, nxt;
    bool have = bwd_item(0, p, it);
    for (int k = 0; have; ++k) {
      const int ns = G * it.n;
      const int k0 = it.kt * kBwdKTile;
      const int kg = k0 + krow;
      // Step i of the item is query tile qi = i mod n of query head hq = i / n of the group; the group takes
      // every second step, so both advance by counting (no division per step).
      int qi = (g - gs0) & 1, hq = 0;
      while (qi >= it.n) qi -= it.n, ++hq;
      for (int gs = gs0 + ((g - gs0) & 1); ok && gs < gs0 + ns; gs += 2) {
        const int s = gs % kBwdStages, rb = g;
        const int q0 = (it.i0 + qi) * kBwdQTile;
        // the step's query head's accumulator
        float* acc_bh = p.dq_acc + static_cast<size_t>(it.b * p.H + it.hk * G + hq) * p.Tp * 128;
        // The group's first step of an item writes its dS^T buffer and then the dQ staging buffer, which the
        // previous item's dK and dV stores read from: it waits for each report just before the first write.
        const bool first_of_item = k > 0 && gs < gs0 + 2;
        bool step_ok =
            mbar_wait_warp(&bars.q_full[s], (gs / kBwdStages) & 1, abort, lim, &g_device_error, kSiteBwdSmQ) &&
            mbar_wait_warp(&bars.s_full[rb], (gs >> 1) & 1, abort, lim, &g_device_error, kSiteBwdSmS);
        if (step_ok) {
          tc_fence_after();
          if (threadIdx.x == 64 || threadIdx.x == 192) ATTN_TRACE_EVENT(4, gs);
          const bool diag = q0 < k0 + kBwdKTile;  // tile overlaps the key tile: queries before a key see nothing
          // sliding window: queries after key + window see nothing (only tiles reaching past k0 + window have any)
          const bool band = p.window >= 0 && q0 + kBwdQTile - 1 > k0 + p.window;
          uint8_t* dsrow = smem + kBwdSmemDS + rb * 16384;
          // The half-tile body is instantiated twice: with the sliding-window mask (tiles that reach past a key's
          // window) and without it, so unwindowed tiles carry no per-element window test.
          bool ds_ok = true;  // the dS^T buffer may be written (the previous item's dK stores have read it)
          auto halves = [&](auto band_flag) {
            constexpr bool kBand = decltype(band_flag)::value;
#pragma unroll 1
            for (int hh = 0; hh < 2; ++hh) {  // one half at a time keeps the live registers to one half's worth
              const uint32_t r = tmem + lane_base + kTmemR + rb * 128 + 32 * hh;
              const float4* lse4 = reinterpret_cast<const float4*>(smem + kBwdSmemLse + s * 256) + 8 * hh;
              const float4* dlt4 = reinterpret_cast<const float4*>(smem + kBwdSmemDelta + s * 256) + 8 * hh;
              uint32_t sv[32], dp[32];
              tmem_ld32(r, sv);        // S^T of queries [32hh, 32hh+32)
              tmem_ld32(r + 64, dp);   // dP^T of the same queries
              tmem_wait_ld();
              uint32_t ppk[16], dpk[16];
#pragma unroll
              for (int q4 = 0; q4 < 8; ++q4) {
                const float4 l4 = lse4[q4], d4 = dlt4[q4];
                const float lv[4] = {l4.x, l4.y, l4.z, l4.w}, dv4[4] = {d4.x, d4.y, d4.z, d4.w};
                float pv[4], dsv[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const int q = q4 * 4 + e;
                  float pe = ex2(fmaf(__uint_as_float(sv[q]), c, -lv[e]));
                  if (diag && q0 + 32 * hh + q < kg) pe = 0.f;
                  if (kBand && q0 + 32 * hh + q > kg + p.window) pe = 0.f;
                  pv[e] = pe;
                  dsv[e] = pe * (__uint_as_float(dp[q]) - dv4[e]);
                }
                ppk[q4 * 2] = pack_bf16x2(pv[0], pv[1]);
                ppk[q4 * 2 + 1] = pack_bf16x2(pv[2], pv[3]);
                dpk[q4 * 2] = pack_bf16x2(dsv[0], dsv[1]);
                dpk[q4 * 2 + 1] = pack_bf16x2(dsv[2], dsv[3]);
              }
              tmem_st16(r, ppk);        // P^T  of these 32 queries: columns [32hh, 32hh+16)
              tmem_st16(r + 16, dpk);   // dS^T of these 32 queries: columns [32hh+16, 32hh+32)
              if (hh == 0 && first_of_item)
                ds_ok = mbar_wait_warp(&bars.ds_read, (k - 1) & 1, abort, lim, &g_device_error, kSiteBwdSmEpiRead);
              if (ds_ok) {
#pragma unroll
                for (int ch = 0; ch < 4; ++ch) {
                  uint4 v = make_uint4(dpk[ch * 4 + 0], dpk[ch * 4 + 1], dpk[ch * 4 + 2], dpk[ch * 4 + 3]);
                  *reinterpret_cast<uint4*>(dsrow + sw128_offset(krow, 4 * hh + ch)) = v;
                }
              }
            }
          };
          if (band) halves(std::true_type{});
          else halves(std::false_type{});
          tmem_wait_st();
          step_ok = ds_ok;
          if (step_ok) {
            fence_async_shared();
            tc_fence_before();
            mbar_arrive_warp(&bars.p_full[rb]);
          }
          if (threadIdx.x == 64 || threadIdx.x == 192) ATTN_TRACE_EVENT(5, gs);
        }

        // dQ^T of this step (thread = d, 64 query columns) -> staging buffer in the accumulator's [q/4][d][4]
        // layout, where the tile is one contiguous 32 KB block -> one bulk reduce-add on the async engine. The
        // staging buffer passes between the two groups in step order through stage_free.
        step_ok = step_ok && mbar_wait_warp(&bars.dq_full[rb], (gs >> 1) & 1, abort, lim, &g_device_error, kSiteBwdDq);
        uint32_t a[2][32];
        if (step_ok) {
          tc_fence_after();
          if (threadIdx.x == 64) ATTN_TRACE_EVENT(6, gs);
          tmem_ld32(tmem + lane_base + kTmemR + rb * 128 + 64, a[0]);
          tmem_ld32(tmem + lane_base + kTmemR + rb * 128 + 96, a[1]);
          tmem_wait_ld();
          tc_fence_before();
          mbar_arrive_warp(&bars.dq_empty[rb]);  // dQ^T is in registers: the tensor-memory columns are free
        }
        step_ok = step_ok && (gs == 0 || wait_staged(gs - 1)) &&
                  (!first_of_item ||  // the previous item's dV stores have read the staging buffer
                   mbar_wait_warp(&bars.dq_read, (k - 1) & 1, abort, lim, &g_device_error, kSiteBwdSmEpiRead));
        if (step_ok) {
#pragma unroll
          for (int hh = 0; hh < 2; ++hh)
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4)
              *reinterpret_cast<float4*>(dq_stage + ((8 * hh + q4) * 128 + krow) * 4) =
                  make_float4(__uint_as_float(a[hh][4 * q4]), __uint_as_float(a[hh][4 * q4 + 1]),
                              __uint_as_float(a[hh][4 * q4 + 2]), __uint_as_float(a[hh][4 * q4 + 3]));
          fence_async_shared();
        }
        // Every warp of the group reaches this barrier, failed or not, and the group leaves the walk together
        // on the AND of the warps' states (a warp leaving alone would meet its siblings at a later barrier of
        // the same id and desynchronise the group).
        if (!named_barrier_and(2 + g, 128, step_ok)) {
          ok = false;
          break;
        }
        if (group_leader) {  // the reduction warp adds the staged tile into the accumulator
          bars.red_dst[g] = acc_bh + static_cast<size_t>(q0 >> 2) * 512;
          mbar_arrive(&bars.dq_staged[g]);
        }
        qi += 2;
        while (qi >= it.n) qi -= it.n, ++hq;
      }
      // Epilogue of the item: TMEM -> bf16 -> swizzled shared memory, and the K/V warp stores (rows past T are
      // clipped). The group of the item's last step is the late one: its last bulk reduction still reads the dQ
      // staging buffer, so it stages dV there once that (and the other group's last reduction) has read it. The
      // other group stages scale*dK in the two dS^T buffers, free once the item's MMAs are done, and its store
      // goes out at once; that group also runs the next item's first step. Each group first waits until the
      // previous item's store has read its buffer (a group without a step in this item has not waited for that
      // yet). The group leaves the item together, failed or not.
      const int gs_last = gs0 + ns - 1;
      const bool dv_group = (gs_last & 1) == g;
      const bool have_next = bwd_item(k + 1, p, nxt);  // decoded while the item's last MMAs finish
      bool epi_ok = __all_sync(0xffffffffu, ok) &&
                    mbar_wait_warp(&bars.acc_done, k & 1, abort, lim, &g_device_error, kSiteBwdSmEpi) &&
                    (k == 0 || mbar_wait_warp(dv_group ? &bars.dq_read : &bars.ds_read, (k - 1) & 1, abort, lim,
                                              &g_device_error, kSiteBwdSmEpiRead));
      // the dV group: the last reductions of both groups (steps gs_last and gs_last - 1) have read the buffer
      if (epi_ok && dv_group) epi_ok = wait_staged(gs_last) && (gs_last == 0 || wait_staged(gs_last - 1));
      uint8_t* stage = smem + (dv_group ? kBwdSmemDQ : kBwdSmemDS);  // 32 KB each: two 16 KB boxes
      if (epi_ok) {
        tc_fence_after();
        const float mul = dv_group ? 1.0f : p.scale;
        const uint32_t col = dv_group ? kTmemDV : kTmemDK;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t o[32];
          tmem_ld32(tmem + lane_base + col + cc * 32, o);
          tmem_wait_ld();
          if (cc == 3) {  // the accumulator has been read: the next item's first dV, dK MMAs may overwrite it
            tc_fence_before();
            mbar_arrive_warp(&bars.acc_free);
          }
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
        fence_async_shared();
        mbar_arrive_warp(dv_group ? &bars.dv_staged : &bars.dk_staged);  // the K/V warp stores it
      }
      if (!named_barrier_and(2 + g, 128, epi_ok && !*abort)) break;
      gs0 += ns;
      it = nxt;
      have = have_next;
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
