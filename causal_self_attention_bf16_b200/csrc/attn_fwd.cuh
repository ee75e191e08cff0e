// Forward kernel of causal multi-head self-attention for sm_100a:
//   O = softmax(scale * Q K^T + causal mask) V, and LSE = natural log-sum-exp of each row's scaled logits.
//
// The pages only call flash_attn_func(q, k, v, causal=True) on [B, T, H, D] bf16 tensors (apidog "Train your
// own ChatGPT", section 5 "Flash Attention integration"; layout from section 1 "GPT model") and name the
// Hopper Flash-Attention-3 kernel as the implementation. This kernel is a new design for Blackwell:
//
//   * CTA pairs: a cluster of two CTAs (the two SMs of a TPC) computes two query tiles of one head at once,
//     CTA r the 128 rows of tile 2p + r. One thread of the even CTA issues tcgen05.mma with cta_group::2 and
//     M = 256: the A operand (Q, then P) and the accumulators (S, O) are split by rows between the two CTAs'
//     tensor memories, the B operand (K, then V) by columns between their shared memories. So each SM stages
//     and reads half of every K and V tile: CTA r loads keys [64r, 64r+64) of a K tile and head dimensions
//     [64r, 64r+64) of a V tile, 32 KB per 128x128 tile instead of 64. (One SM loading whole K and V tiles
//     for one query tile cannot keep its tensor core busy: the tiles arrive too slowly.) All loads are plain
//     per-CTA TMA copies (no multicast) whose completion is counted on the even CTA's barriers.
//   * persistent: the pairs walk work items (pair of query tiles, batch, head) in head-major order, so the
//     K/V of the few heads in flight stay in L2; the rings run on across items.
//   * in each CTA: warp 0 stages Q once per item and the K ring, warp 2 the V ring (four-deep), warp 1 (of
//     the even CTA) issues the MMAs, warps 4..11, two groups of four, run the online softmax straight out of
//     tensor memory, one thread per query row: group g takes KV tiles j = g, g+2, ..., and only the running
//     row max passes between the groups (through shared memory), so one tile's exponentials overlap the next
//     tile's load and max. A thread owns a whole row of S, so row max and row sum need no shuffles; O is
//     rescaled lazily, only when the running max grows by more than 2^8; warp 3 writes the normalised O.
//     The first warpgroup (warps 0..3) hands most of its registers to the two softmax warpgroups, whose
//     threads hold a row of scores and its packed probabilities at once (setmaxnreg: 40 and 232 registers
//     per thread against 168 at launch; 4 x 32 x 40 + 8 x 32 x 232 = 384 x 168, the launch's whole file).
//   * the pair's last KV tile is the odd CTA's diagonal tile and lies wholly above the even CTA's diagonal:
//     the even CTA masks all of it (P = 0) without computing exponentials.
//
// Tensor memory (512 columns per CTA, allocated for the pair): S double buffer [0,256) (buffer j%2 belongs to
// the group of tile j), O [256,384), Q (bf16 pairs) [384,448), P (bf16 pairs) [448,512). The MMA thread issues
// whichever MMA is ready, PV first: PV(j) in tile order once P(j) is stored, S(j+2) as soon as S(j) has been
// read out in both CTAs and K(j+2) has landed; the group of tile j stores P(j) once PV(j-1) has landed.
#pragma once
#include "attn_common.cuh"
#include "sm100.cuh"

namespace attn {

constexpr int kTile = 128;        // query rows per CTA and keys per KV tile
constexpr int kHeadDim = 128;     // D
constexpr int kFwdThreads = 384;  // warp 0 TMA (Q, K), warp 1 MMA, warp 2 TMA (V), warp 3 TMA store of O,
                                  // warps 4..11 two softmax groups
constexpr int kFwdWarpV = 2, kFwdWarpStore = 3;
// Registers per thread after the split (setmaxnreg): the launch gives each of the 384 threads 168 (the
// launch bounds' limit); the producer warpgroup keeps 40 and the two softmax warpgroups take the rest.
constexpr int kFwdRegsLaunch = 168, kFwdRegsProducer = 40, kFwdRegsSoftmax = 232;
static_assert(4 * 32 * kFwdRegsProducer + 8 * 32 * kFwdRegsSoftmax == kFwdThreads * kFwdRegsLaunch,
              "the register split must hand over exactly the launch's registers");
static_assert(kFwdRegsLaunch * kFwdThreads <= 65536 && kFwdRegsLaunch % 8 == 0 && kFwdRegsLaunch <= 65536 / kFwdThreads,
              "launch register count");
constexpr int kFwdKRows = kTile / 2;  // keys of a KV tile staged by each CTA of the pair

// Shared-memory layout of the forward kernel (offsets from a 1024-byte aligned base; the same in both CTAs).
constexpr uint32_t kFwdSmemQ = 0;                                  // 32 KB: Q tile, two 64-column boxes of 16 KB
constexpr int kFwdStages = 4;                                      // depth of the K and V rings
constexpr uint32_t kFwdSlot = 16384;                               // one ring slot: half a K or V tile
constexpr uint32_t kFwdSmemK = 32768;                              // 4 x 16 KB: 64 keys x 128 dims (two boxes)
constexpr uint32_t kFwdSmemV = kFwdSmemK + kFwdStages * kFwdSlot;  // 4 x 16 KB: 128 keys x 64 dims
constexpr uint32_t kFwdSmemXchg = kFwdSmemV + kFwdStages * kFwdSlot;  // 2 KB: row-max / row-sum exchange
constexpr uint32_t kFwdSmemBytes = kFwdSmemXchg + 2 * 2 * 128 * 4;    // barriers follow (see FwdBarriers)

constexpr uint32_t kTmemS = 0, kTmemO = 256, kTmemQ = 384, kTmemP = 448;

// Lazy rescaling threshold on the running max, in log2 units (values of P stay below 2^8).
constexpr float kRescaleThreshold = 8.0f;

struct FwdParams {
  float* lse;        // [B, H, T] fp32
  int B, H, T;
  int Hkv;           // key/value heads (divides H); query head h reads key/value head h / (H / Hkv)
  int window;        // sliding window: query i sees keys i - window .. i; -1: no window
  float scale_log2;  // scale * log2(e)
  uint64_t timeout_ns;
};

// Barriers, at the same offsets in both CTAs. "pair" barriers live in the even CTA and count arrivals from
// both; "mc" barriers exist in both CTAs and are completed by the even CTA's multicast tcgen05.commit.
struct FwdBarriers {
  uint64_t q_full;      // local: this CTA's Q tile landed
  uint64_t q_tmem;      // local: this CTA's Q copied into its tensor memory (the 4 warps of one group)
  uint64_t q_ready;     // pair: both CTAs' Q in tensor memory (8 warps)
  uint64_t o_staged;    // local: both softmax groups have staged the item's output in the Q buffer (8 warps)
  uint64_t q_free;      // local: the Q buffer's other use, staging an item's output for its TMA store, is over
  uint64_t k_full[kFwdStages], v_full[kFwdStages];    // pair: both halves of a K / V tile landed
  uint64_t k_empty[kFwdStages], v_empty[kFwdStages];  // mc: the MMAs that read a ring slot are done
  uint64_t s_full[2];   // mc: S(j) landed in buffer j%2
  uint64_t s_free[2];   // pair: S(j) read out of buffer j%2 in both CTAs (8 warps)
  uint64_t p_full[2];   // pair: P(j) stored (and O rescaled if needed) in both CTAs (8 warps)
  uint64_t xchg[2];     // local: running max after tile j published in slot j%2 (4 warps)
  uint64_t pv_done[2];  // mc: PV(j) completed (barrier j%2): P is free, O holds tiles 0..j
  uint64_t o_final;     // mc: committed once after an item's last PV: the epilogue's wait
  uint64_t s_done;      // mc: committed once after an item's last S: its Q in tensor memory is no longer read
  uint64_t drain;       // local (even CTA): every MMA done
  uint32_t tmem_base;
  int abort;
};
// No static shared memory: the dynamic block starts 1024-byte aligned and needs no slack (the kernel checks
// this and refuses to run otherwise): tiles, the exchange area, then the barriers. 164 KB in all.
constexpr uint32_t kFwdSmemAlloc = kFwdSmemBytes + sizeof(FwdBarriers);
static_assert(kFwdSmemAlloc <= 232448, "forward kernel exceeds the 227 KB shared-memory opt-in");

// Error sites (recorded with a timeout in the device error word): 0x10 + barrier id, per role.
enum : uint32_t {
  kSiteFwdLayout = 0x10, kSiteFwdProdKEmpty = 0x11, kSiteFwdProdVEmpty = 0x12, kSiteFwdProdQ = 0x13,
  kSiteFwdStore = 0x14, kSiteFwdMmaQ = 0x21, kSiteFwdMmaK = 0x22, kSiteFwdMmaP = 0x23, kSiteFwdMmaV = 0x24,
  kSiteFwdMmaS = 0x25, kSiteFwdSmS = 0x31, kSiteFwdSmPV = 0x32, kSiteFwdEpi = 0x33, kSiteFwdDrain = 0x34,
  kSiteFwdSmX = 0x35, kSiteFwdSmQ = 0x36
};

// Work item k of this pair: (batch*head, pair of query tiles), head-major, the heaviest pair of each head
// first. Items are dealt to the G pairs in rounds of G that alternate direction (item k*G + c on even rounds,
// k*G + G-1-c on odd ones), which balances the causal work per pair, and the items in flight at any time
// cover only a few heads, whose K/V stay in L2.
struct FwdItem {
  int bh, qp;
};
// First KV tile a query tile needs: 0, or with a sliding window the tile holding key q0 - window.
__device__ __forceinline__ int fwd_first_kv_tile(int qt, int window) {
  return window < 0 ? 0 : max(0, qt * kTile - window) / kTile;
}

// The host caps B * H * (query tiles) well below 2^31, so item indices (fewer than n_items plus one round of
// pairs) fit in 32 bits and decode with 32-bit divisions.
__device__ __forceinline__ bool fwd_item(int k, int n_items, int n_qp, FwdItem& it) {
  const unsigned G = gridDim.x / 2, c = blockIdx.x / 2;
  const unsigned idx = static_cast<unsigned>(k) * G + ((k & 1) ? G - 1 - c : c);
  if (idx >= static_cast<unsigned>(n_items)) return false;
  it.bh = static_cast<int>(idx / static_cast<unsigned>(n_qp));
  it.qp = n_qp - 1 - static_cast<int>(idx % static_cast<unsigned>(n_qp));
  return true;
}

// KV tiles of a pair item: from the even tile's first one to the odd tile's diagonal (or the last tile).
__device__ __forceinline__ void fwd_item_tiles(int qp, int n_qt, int window, int& kt0, int& n_kv) {
  kt0 = fwd_first_kv_tile(2 * qp, window);
  n_kv = min(2 * qp + 2, n_qt) - kt0;
}

// Persistent pairs: every ring and buffer index is a running count over the pair's KV tiles (t) or items (k),
// so the producers stream the next item's Q, K and V while the current item is computed, and the next item's
// first S tiles run while the current item's output is written.
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kFwdThreads, 1)
attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                const FwdParams p) {
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base for the 128-byte-swizzle tiles. Offsetting the array itself (not a round trip
  // through an integer) keeps the pointer in the shared address space, so accesses compile to LDS/STS.
  uint8_t* smem = smem_raw;
  const bool misaligned = (smem_u32(smem_raw) & 1023u) != 0;
  FwdBarriers& bars = *reinterpret_cast<FwdBarriers*>(smem + kFwdSmemBytes);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = cluster_ctarank();  // 0: the even CTA, which issues the MMAs
  const bool is_lead = rank == 0;
  const int n_qt = (p.T + kTile - 1) / kTile;
  const int n_qp = (n_qt + 1) / 2;
  const int n_items = p.B * p.H * n_qp;
  volatile int* abort = &bars.abort;

  if (threadIdx.x == 0) {
    mbar_init(&bars.q_full, 1);
    mbar_init(&bars.q_tmem, 4);    // counts warps (one softmax group copies both head-dim halves of its rows)
    mbar_init(&bars.q_ready, 8);   // the same arrivals from both CTAs
    mbar_init(&bars.o_staged, 8);  // counts warps
    mbar_init(&bars.q_free, 1);
    for (int s = 0; s < kFwdStages; ++s) {
      mbar_init(&bars.k_full[s], 1);
      mbar_init(&bars.k_empty[s], 1);
      mbar_init(&bars.v_full[s], 1);
      mbar_init(&bars.v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars.s_full[s], 1);
      mbar_init(&bars.s_free[s], 8);  // the warps of one softmax group in both CTAs
      mbar_init(&bars.p_full[s], 8);
      mbar_init(&bars.xchg[s], 4);    // the warps of one softmax group of this CTA
      mbar_init(&bars.pv_done[s], 1);
    }
    mbar_init(&bars.o_final, 1);
    mbar_init(&bars.s_done, 1);
    mbar_init(&bars.drain, 1);
    bars.abort = misaligned ? 1 : 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(&bars.tmem_base, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers exist before any remote arrival or copy completion
  tc_fence_after();
  const uint32_t tmem = bars.tmem_base;
  const uint32_t peer_abort = mapa_shared(&bars.abort, rank ^ 1u);
  if (misaligned) {  // the layout needs a 1024-byte aligned dynamic block: both CTAs give up
    if (threadIdx.x == 0) {
      atomicOr(&g_device_error, sm100::DEV_ERR_TIMEOUT | (kSiteFwdLayout << 8));
      asm volatile("st.relaxed.cluster.shared::cluster.u32 [%0], %1;" ::"r"(peer_abort), "r"(1) : "memory");
    }
  }
  cluster_sync_all();
  if (threadIdx.x == 0) ATTN_TRACE_EVENT(0, 0);
  const uint64_t lim = p.timeout_ns;

  if (*abort) {
    // nothing was issued
  } else if (warp < 4) {
    // The producer warpgroup gives registers back before the softmax warpgroups claim them (every warp of a
    // warpgroup executes the same setmaxnreg).
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(kFwdRegsProducer) : "memory");
    if (warp == 0 || warp == kFwdWarpV) {
      // ------------------------------------------------------------------ TMA producers (both CTAs)
      // Warp 0 stages Q and this CTA's half of every K tile, warp 2 its half of every V tile. Each walks its
      // loop warp-uniformly (addresses and coordinates stay in uniform registers); one elected lane issues. The
      // even CTA's lane also arms the pair's full barrier with the bytes of both halves.
      const bool is_k = warp == 0;
      const bool leader = elect_one();
      const CUtensorMap* tm = is_k ? &tm_k : &tm_v;
      uint64_t* full = is_k ? bars.k_full : bars.v_full;
      uint64_t* empty = is_k ? bars.k_empty : bars.v_empty;
      uint8_t* ring = smem + (is_k ? kFwdSmemK : kFwdSmemV);
      if (leader) {
        tma_prefetch_desc(tm);
        if (is_k) tma_prefetch_desc(&tm_q);
      }
      int issued[kFwdStages];
      for (int s = 0; s < kFwdStages; ++s) issued[s] = -1;
      int q_issued = -1;
      int t0 = 0;  // running KV tile count: ring slot t % kFwdStages, phase (t / kFwdStages) & 1
      FwdItem it;
      for (int k = 0; fwd_item(k, n_items, n_qp, it); ++k) {
        const int b = it.bh / p.H, h = it.bh % p.H;
        int kt0, n_kv;
        fwd_item_tiles(it.qp, n_qt, p.window, kt0, n_kv);
        const int hk = h / (p.H / p.Hkv);  // grouped-query attention: the group's key/value head
        if (is_k) {
          // One Q buffer, which also stages each item's output for its TMA store. Q(1) may go in once Q(0) is in
          // tensor memory; Q(k), k >= 2, once item k-2's output has been read out of the buffer by its store
          // (which follows the copy of Q(k-1) into tensor memory in the same epilogue).
          if (k == 1 && !mbar_wait_pair_warp(&bars.q_tmem, 0, abort, peer_abort, lim, &g_device_error, kSiteFwdProdQ))
            break;
          if (k >= 2 &&
              !mbar_wait_pair_warp(&bars.q_free, (k - 2) & 1, abort, peer_abort, lim, &g_device_error, kSiteFwdProdQ))
            break;
          if (leader) {
            mbar_arrive_expect_tx(&bars.q_full, 2 * 16384);
            for (int c = 0; c < 2; ++c)
              tma_load_4d(smem + kFwdSmemQ + c * 16384, &tm_q, &bars.q_full, c * 64, h,
                          (2 * it.qp + static_cast<int>(rank)) * kTile, b);
          }
          q_issued = k;
        }
        bool ok = true;
        for (int j = 0; j < n_kv; ++j) {
          const int t = t0 + j, s = t % kFwdStages;
          if (t >= kFwdStages &&
              !mbar_wait_pair_warp(&empty[s], ((t - kFwdStages) / kFwdStages) & 1, abort, peer_abort, lim,
                                   &g_device_error, is_k ? kSiteFwdProdKEmpty : kSiteFwdProdVEmpty)) {
            ok = false;
            break;
          }
          if (leader) {
            if (is_lead) mbar_arrive_expect_tx(&full[s], 2 * kFwdSlot);
            const uint32_t bar = mapa_shared(&full[s], 0);
            const int kt = kt0 + j;
            if (is_k) {  // keys [kt*128 + 64r, +64), both head-dim boxes
              for (int c = 0; c < 2; ++c)
                tma_load_4d_pair(ring + s * kFwdSlot + c * 8192, tm, bar, c * 64, hk,
                                 kt * kTile + kFwdKRows * static_cast<int>(rank), b);
              ATTN_TRACE_EVENT(1, t);
            } else {     // all 128 keys, head dimensions [64r, 64r+64)
              tma_load_4d_pair(ring + s * kFwdSlot, tm, bar, 64 * static_cast<int>(rank), hk, kt * kTile, b);
            }
          }
          issued[s] = t;
        }
        if (!ok) break;
        t0 += n_kv;
      }
      if (*abort) {
        // Let every copy this CTA started land before its shared memory is released. The K/V halves count on
        // the even CTA's barriers, which the even CTA drains; this CTA's own Q copy counts here.
        volatile int no_abort = 0;
        if (q_issued >= 0) mbar_wait(&bars.q_full, q_issued & 1, &no_abort, lim, &g_device_error, kSiteFwdDrain);
        if (is_lead) {
          for (int s = 0; s < kFwdStages; ++s)
            if (issued[s] >= 0)
              mbar_wait(&full[s], (issued[s] / kFwdStages) & 1, &no_abort, lim, &g_device_error, kSiteFwdDrain);
        } else {
          const uint64_t t_end = global_timer_ns() + 50000;  // the odd CTA cannot see its halves land: 50 us
          while (global_timer_ns() < t_end) {
          }
        }
      }
    } else if (warp == kFwdWarpStore) {
      // ------------------------------------------------------------------ output store (both CTAs)
      // Once both softmax groups have staged an item's output in the Q buffer, one elected lane writes it with
      // two TMA stores (rows past T are clipped; a tile wholly past T is not stored) and frees the buffer for
      // the next Q as soon as the stores have read it.
      const bool leader = elect_one();
      if (leader) tma_prefetch_desc(&tm_o);
      FwdItem it;
      for (int k = 0; fwd_item(k, n_items, n_qp, it); ++k) {
        if (!mbar_wait_pair_warp(&bars.o_staged, k & 1, abort, peer_abort, lim, &g_device_error, kSiteFwdStore)) break;
        if (__any_sync(0xffffffffu, *abort != 0)) break;  // warp-uniform: the loop ends in a __syncwarp
        const int qt = 2 * it.qp + static_cast<int>(rank);
        if (leader) {
          if (qt < n_qt) {
            for (int c = 0; c < 2; ++c)
              tma_store_4d(&tm_o, smem + kFwdSmemQ + c * 16384, c * 64, it.bh % p.H, qt * kTile, it.bh / p.H);
            tma_store_commit();
            tma_store_wait_read_all();
          }
          mbar_arrive(&bars.q_free);
        }
        __syncwarp();
      }
      if (leader) tma_store_wait_all();
    } else if (warp == 1) {
      // ------------------------------------------------------------------ MMA issuer (even CTA only)
      // The whole warp walks the schedule and computes the descriptors (warp-uniform, so they live in uniform
      // registers); the lane elected once issues every tcgen05.mma and tcgen05.commit (a commit tracks the
      // MMAs of the thread that issues it, so it must be the same lane throughout).
      if (is_lead) {
        const bool leader = elect_one();
        const uint32_t idesc_s = idesc_bf16_f32(256, 128, false, false);  // Q (TMEM) x K (K-major), M = 256
        const uint32_t idesc_pv = idesc_bf16_f32(256, 128, false, true);  // P (TMEM) x V (MN-major), M = 256
        // PV(t): O += P(t) V(t) (the first tile of an item overwrites O); P from tensor memory, V from ring slot
        // t % kFwdStages: each CTA holds all 128 keys of its 64 output dimensions, one 16 KB box.
        auto issue_pv = [&](int t, bool first) {
          const int pb = t & 1, vs = t % kFwdStages;
          if (leader) ATTN_TRACE_EVENT(15, t);
          tc_fence_after();
          const uint64_t dv = sdesc_sw128(smem_u32(smem + kFwdSmemV + vs * kFwdSlot), kFwdSlot, 1024);  // MN-major
  #pragma unroll
          for (int kk = 0; kk < 8; ++kk)  // K step kk: 16 keys = 2048 bytes further (128 in 16-byte units)
            if (leader)
              mma_ts_pair(tmem + kTmemO, tmem + kTmemP + kk * 8, dv + kk * 128, idesc_pv, (!first || kk > 0) ? 1u : 0u);
          if (leader) {
            mma_commit_pair(&bars.pv_done[pb], 3);
            ATTN_TRACE_EVENT(3, t);
            mma_commit_pair(&bars.v_empty[vs], 3);
          }
        };
        // S(t) = Q K(t)^T into S buffer t%2. Each CTA holds 64 keys of the tile as two 8 KB boxes of 64 head
        // dimensions.
        auto issue_s = [&](int t) {
          const int ks = t % kFwdStages, sb = t & 1;
          if (leader) ATTN_TRACE_EVENT(14, t);
          tc_fence_after();
          const uint64_t dk = sdesc_sw128(smem_u32(smem + kFwdSmemK + ks * kFwdSlot), 16, 1024);  // K, K-major
  #pragma unroll
          for (int kk = 0; kk < 8; ++kk) {  // K step kk: 16 head-dim columns = 8 TMEM columns of Q; for K the
            // second 64-column box from kk = 4, 32 bytes per step within a box
            const uint32_t koff = ((kk >> 2) * 8192 + (kk & 3) * 32) >> 4;
            if (leader)
              mma_ts_pair(tmem + kTmemS + sb * 128, tmem + kTmemQ + kk * 8, dk + koff, idesc_s, kk > 0 ? 1u : 0u);
          }
          if (leader) {
            mma_commit_pair(&bars.s_full[sb], 3);
            ATTN_TRACE_EVENT(2, t);
            mma_commit_pair(&bars.k_empty[ks], 3);
          }
        };
        // Readiness tests (warp-uniform, non-blocking). S(t) needs its K tile and S buffer t%2 read out of S(t-2)
        // in both CTAs; PV(t) needs P(t) from both CTAs and its V tile.
        auto s_ready = [&](int t) {
          const bool ok_s = t < 2 || mbar_test(&bars.s_free[t & 1], ((t - 2) >> 1) & 1);
          return __all_sync(0xffffffffu, ok_s && mbar_test(&bars.k_full[t % kFwdStages], (t / kFwdStages) & 1));
        };
        auto pv_ready = [&](int t) {
          return __all_sync(0xffffffffu, mbar_test(&bars.p_full[t & 1], (t >> 1) & 1) &&
                                             mbar_test(&bars.v_full[t % kFwdStages], (t / kFwdStages) & 1));
        };
        bool ok = true;
        int t0 = 0;
        FwdItem it;
        for (int k = 0; ok && fwd_item(k, n_items, n_qp, it); ++k) {
          int kt0, n_kv;
          fwd_item_tiles(it.qp, n_qt, p.window, kt0, n_kv);
          // This item's Q is in both CTAs' tensor memory (copied once the previous item's MMAs had completed).
          if (!mbar_wait_pair_warp(&bars.q_ready, k & 1, abort, peer_abort, lim, &g_device_error, kSiteFwdMmaQ)) break;
          // Issue whichever MMA is ready, PV first. The PVs go in tile order as their P arrives, and P(j+1) can
          // only be stored once PV(j) has read P(j), so a PV that queued behind an S would hold up the next
          // tile's P; the S tiles run ahead as far as the two S buffers allow and have time to spare. The
          // tensor cores execute in issue order.
          int js = 0, jp = 0;  // next S and next PV of the item
          uint64_t t_idle = 0;
          while (jp < n_kv) {
            if (jp < js && pv_ready(t0 + jp)) {
              issue_pv(t0 + jp, jp == 0);
              ++jp;
              t_idle = 0;
            } else if (js < n_kv && s_ready(t0 + js)) {
              issue_s(t0 + js++);
              if (js == n_kv && leader) mma_commit_pair(&bars.s_done, 3);  // the item's Q may be replaced
              t_idle = 0;
            } else {
              // Nothing ready: bounded like every wait of the kernel.
              const uint64_t now = global_timer_ns();
              if (t_idle == 0) t_idle = now;
              const bool give_up = __any_sync(0xffffffffu, *abort != 0 || now - t_idle > lim);
              if (give_up) {
                if (lane == 0 && !*abort) {
                  *abort = 1;
                  asm volatile("st.relaxed.cluster.shared::cluster.u32 [%0], %1;" ::"r"(peer_abort), "r"(1) : "memory");
                  atomicOr(&g_device_error, DEV_ERR_TIMEOUT | (kSiteFwdMmaS << 8));
                }
                ok = false;
                break;
              }
            }
          }
          if (ok && leader) mma_commit_pair(&bars.o_final, 3);
          t0 += n_kv;
        }
        // Drain: wait until every MMA the leader issued has completed before tensor memory is released.
        if (leader) mma_commit_pair(&bars.drain, 1);
        volatile int no_abort = 0;
        mbar_wait(&bars.drain, 0, &no_abort, lim, &g_device_error, kSiteFwdDrain);
      }
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(kFwdRegsSoftmax) : "memory");
    // ------------------------------------------------------------------ softmax / correction / epilogue
    // Two warp groups take the KV tiles in turn: group g (warps 4..7 or 8..11) owns the tiles whose running
    // index t is g modulo 2, and S buffer g. A thread holds one query row of its tile (128 keys) in registers.
    // The online softmax is sequential only through the running max: the group publishes the max after its
    // tile in shared memory and the other group, which has already loaded and reduced the next tile, takes
    // it from there. So the exponentials of one tile overlap the load, max and exchange of the next, and two
    // softmax warps per SM sub-partition keep the MUFU and FMA pipes busy.
    const int g = (warp - 4) >> 2;
    const int quarter = warp & 3;           // TMEM lane quarter this warp may access
    const int row = quarter * 32 + lane;    // query row within the tile
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const float c = p.scale_log2;
    float* xm = reinterpret_cast<float*>(smem + kFwdSmemXchg);  // [2 slots, by tile parity][128 rows]: running max
    float* xl = xm + 2 * 128;                                    // [2 groups][128 rows]: partial sums, at the end
    const bool tracer = (threadIdx.x & 127) == 0;                // one thread per group records trace events
    // Q of item k goes to tensor memory, so S = Q K^T reads only K from shared memory. One group copies both
    // head-dim boxes of its rows: word w of a row (head dims 2w, 2w+1) becomes TMEM column w, the A-operand
    // layout. Each of its warps then arrives on this CTA's q_tmem and on the pair's q_ready.
    auto copy_q = [&](int k) -> bool {
      if (!mbar_wait_pair_warp(&bars.q_full, k & 1, abort, peer_abort, lim, &g_device_error, kSiteFwdSmQ)) return false;
#pragma unroll 1
      for (int box = 0; box < 2; ++box) {
        uint32_t qw[32];
        const uint8_t* src = smem + kFwdSmemQ + box * 16384;
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          const uint4 v = *reinterpret_cast<const uint4*>(src + sw128_offset(row, ch));
          qw[ch * 4 + 0] = v.x;
          qw[ch * 4 + 1] = v.y;
          qw[ch * 4 + 2] = v.z;
          qw[ch * 4 + 3] = v.w;
        }
        tmem_st32(tmem + lane_base + kTmemQ + 32 * box, qw);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive_warp(&bars.q_tmem);
      mbar_arrive_warp_cluster(&bars.q_ready, 0);
      return true;
    };
    FwdItem it;
    bool have = fwd_item(0, n_items, n_qp, it);
    bool ok = have && g == 0 ? copy_q(0) : true;  // group 0 copies the first item's Q
    int t0 = 0;
    for (int k = 0; have; ++k) {
      int kt0, n_kv;
      fwd_item_tiles(it.qp, n_qt, p.window, kt0, n_kv);
      const int qt = 2 * it.qp + static_cast<int>(rank);  // this CTA's query tile
      const int qrow = qt * kTile + row;                   // this thread's query position
      float m = -INFINITY;  // running max (scale*log2(e) units, stale by < 2^8) after this group's last tile
      float l = 0.f;        // this group's partial row sum of exp2(c*S - m)
      for (int t = t0 + ((g - t0) & 1); ok && t < t0 + n_kv; t += 2) {
        const int kt = kt0 + (t - t0);  // KV tile
        const int sb = g;               // = t % 2
        if (!mbar_wait_pair_warp(&bars.s_full[sb], (t >> 1) & 1, abort, peer_abort, lim, &g_device_error,
                                 kSiteFwdSmS)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (tracer) ATTN_TRACE_EVENT(4, t);
        // The whole tile lies above this CTA's diagonal (the pair's last tile, seen only by the odd CTA): all
        // of it is masked. The row keeps its max and sum, P is 0, and no score is read.
        if (kt > qt) {
          tc_fence_before();
          mbar_arrive_warp_cluster(&bars.s_free[sb], 0);
          float m_prev = -INFINITY;
          if (t > t0) {
            if (!mbar_wait_pair_warp(&bars.xchg[sb ^ 1], ((t - 1) >> 1) & 1, abort, peer_abort, lim,
                                     &g_device_error, kSiteFwdSmX)) {
              ok = false;
              break;
            }
            m_prev = xm[(sb ^ 1) * 128 + row];
          }
          xm[sb * 128 + row] = m_prev;
          mbar_arrive_warp(&bars.xchg[sb]);
          if (t > 0) {
            if (!mbar_wait_pair_warp(&bars.pv_done[sb ^ 1], ((t - 1) >> 1) & 1, abort, peer_abort, lim,
                                     &g_device_error, kSiteFwdSmPV)) {
              ok = false;
              break;
            }
            tc_fence_after();
          }
          uint32_t zero[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) zero[i] = 0u;
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) tmem_st16(tmem + lane_base + kTmemP + cc * 16, zero);
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive_warp_cluster(&bars.p_full[sb], 0);
          continue;
        }
        float s[128];
        {
          uint32_t r[4][32];
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) tmem_ld32(tmem + lane_base + kTmemS + sb * 128 + cc * 32, r[cc]);
          tmem_wait_ld();
#pragma unroll
          for (int cc = 0; cc < 4; ++cc)
#pragma unroll
            for (int i = 0; i < 32; ++i) s[cc * 32 + i] = __uint_as_float(r[cc][i]);
        }
        tc_fence_before();
        mbar_arrive_warp_cluster(&bars.s_free[sb], 0);  // S(t+2) may now be written over this buffer
        if (tracer) ATTN_TRACE_EVENT(8, t);
        if (kt == qt) {  // diagonal tile: key column > query row is masked
#pragma unroll
          for (int i = 0; i < 128; ++i)
            if (i > row) s[i] = -INFINITY;
        }
        if (p.window >= 0) {  // sliding window: key kt*128 + i < query - window is masked
          const int lo = qrow - p.window - kt * kTile;  // first visible column of this row
          if (lo > 0) {
#pragma unroll
            for (int i = 0; i < 128; ++i)
              if (i < lo) s[i] = -INFINITY;
          }
        }
        // Row max of the tile as a tree over 16 independent partial maxima.
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
        // Running max after tile t-1, from the other group (none before an item's first tile). A slot is
        // rewritten two tiles later only after its reader has published the tile in between (or, across
        // items, after both groups have passed the epilogue), so one phase of xchg per tile suffices.
        float m_prev = -INFINITY;
        if (t > t0) {
          if (!mbar_wait_pair_warp(&bars.xchg[sb ^ 1], ((t - 1) >> 1) & 1, abort, peer_abort, lim, &g_device_error,
                                   kSiteFwdSmX)) {
            ok = false;
            break;
          }
          m_prev = xm[(sb ^ 1) * 128 + row];
        }
        // Lazy rescaling: the running max moves only when the tile's max exceeds it by more than 2^8 (always
        // on an item's first tile with a visible key). Each row decides for itself, so a row's arithmetic never
        // depends on another row's inputs (outputs before a position do not depend on inputs after it).
        const bool need = m_tile > m_prev + kRescaleThreshold;
        const float m_j = need ? m_tile : m_prev;
        xm[sb * 128 + row] = m_j;
        mbar_arrive_warp(&bars.xchg[sb]);
        if (tracer) ATTN_TRACE_EVENT(11, t);
        // P = exp2(c*S - m_j) for the 128 keys (MUFU ex2) and the row sum, packed to bf16 pairs in registers.
        // A row that has seen no key yet (only possible left of a sliding window) keeps m_j = -inf and all its
        // scores are -inf: the reference 0 gives P = 0 there instead of NaN.
        const float neg_m = m_j == -INFINITY ? 0.f : -m_j;
        float ps[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};  // 8 independent partial row sums
        uint32_t pk[4][16];
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float x0 = fmaf(s[cc * 32 + 2 * i], c, neg_m), x1 = fmaf(s[cc * 32 + 2 * i + 1], c, neg_m);
            const float p0 = ex2(x0), p1 = ex2(x1);
            ps[(2 * i) & 7] += p0;
            ps[(2 * i + 1) & 7] += p1;
            pk[cc][i] = pack_bf16x2(p0, p1);
          }
        }
        const float rs = ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
        l = (m == m_j ? l : l * ex2(m - m_j)) + rs;  // this group's sum was relative to its previous max
        m = m_j;
        if (tracer) ATTN_TRACE_EVENT(9, t);
        // P and O are free once PV(t-1) has landed (for an item's first tile, the previous item's last PV).
        // PV(t-3) landed before S(t) (issue order) and PV(t+1) waits for PV(t), which waits for this group,
        // so pv_done[sb^1] is within one phase of t-1.
        if (t > 0) {
          if (!mbar_wait_pair_warp(&bars.pv_done[sb ^ 1], ((t - 1) >> 1) & 1, abort, peer_abort, lim,
                                   &g_device_error, kSiteFwdSmPV)) {
            ok = false;
            break;
          }
          tc_fence_after();
        }
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) tmem_st16(tmem + lane_base + kTmemP + cc * 16, pk[cc]);
        if (t > t0 && __any_sync(0xffffffffu, need)) {
          // Some row of this warp moved its max: O (tiles before t, relative to m_prev) is scaled by
          // 2^(m_prev - m_j) before PV(t) is issued. TMEM access is warp-collective, so the whole warp walks
          // its rows; rows that kept their max get alpha = 1 exactly.
          const float alpha = need ? ex2(m_prev - m_j) : 1.0f;
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            uint32_t o[32];
            tmem_ld32(tmem + lane_base + kTmemO + cc * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(tmem + lane_base + kTmemO + cc * 32, o);
          }
        }
        tmem_wait_st();
        if (tracer) ATTN_TRACE_EVENT(10, t);
        tc_fence_before();
        mbar_arrive_warp_cluster(&bars.p_full[sb], 0);
        if (tracer) ATTN_TRACE_EVENT(5, t);
      }
      // The next item, decoded here, where the wait for this item's last PV hides the arithmetic.
      FwdItem next;
      const bool have_next = fwd_item(k + 1, n_items, n_qp, next);
      // The group without the item's last tile (it has finished its own tiles) copies the next item's Q into
      // tensor memory once the item's last S MMA has completed, so the next item's first S tiles queue right
      // behind this item's last PV instead of waiting for this epilogue. The copy reads the Q buffer before the
      // epilogue's first barrier, after which both groups stage the output there.
      if (ok && have_next && g == (((t0 + n_kv - 1) & 1) ^ 1))
        ok = mbar_wait_pair_warp(&bars.s_done, k & 1, abort, peer_abort, lim, &g_device_error, kSiteFwdSmQ) &&
             copy_q(k + 1);
      // Epilogue of item k. The final running max is the one published for the item's last tile; each group
      // brings its partial sum to it and the two are added. Every thread of both groups reaches the named
      // barriers, failed or not, and both leave the item loop on the same decision (a barrier reduction).
      if (tracer && k < 64) ATTN_TRACE_EVENT(6, k);
      named_barrier(1, 256);
      const float m_f = xm[((t0 + n_kv - 1) & 1) * 128 + row];
      xl[g * 128 + row] = m == m_f ? l : l * ex2(m - m_f);  // a group without tiles has l = 0, m = -inf
      named_barrier(1, 256);
      const float l_row = xl[row] + xl[128 + row];
      bool o_ready = __all_sync(0xffffffffu, ok) &&
                     mbar_wait_pair_warp(&bars.o_final, k & 1, abort, peer_abort, lim, &g_device_error, kSiteFwdEpi);
      if (!o_ready) ok = false;
      // The Q buffer takes this item's output once the store of the previous item's output has read it (the
      // next Q, loaded in between, implies that, but the last item has none); the next Q was copied out of it
      // before the barriers above.
      if (o_ready && k > 0 &&
          !mbar_wait_pair_warp(&bars.q_free, (k - 1) & 1, abort, peer_abort, lim, &g_device_error, kSiteFwdEpi)) {
        o_ready = false;
        ok = false;
      }
      if (o_ready) {
        if (tracer && k < 64) ATTN_TRACE_EVENT(7, k);
        tc_fence_after();
        const float inv_l = 1.0f / l_row;
        // O / l -> bf16 -> this group's 64-column box of the Q buffer, in the 128-byte-swizzled layout of the
        // TMA store.
        uint8_t* box = smem + kFwdSmemQ + g * 16384;
        uint32_t o[2][32];  // both 32-column chunks of this group's half of O, loaded before one wait
        tmem_ld32(tmem + lane_base + kTmemO + 64 * g, o[0]);
        tmem_ld32(tmem + lane_base + kTmemO + 64 * g + 32, o[1]);
        tmem_wait_ld();
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) {
            const uint32_t* w = o[cc] + ch * 8;
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(w[0]) * inv_l, __uint_as_float(w[1]) * inv_l);
            v.y = pack_bf16x2(__uint_as_float(w[2]) * inv_l, __uint_as_float(w[3]) * inv_l);
            v.z = pack_bf16x2(__uint_as_float(w[4]) * inv_l, __uint_as_float(w[5]) * inv_l);
            v.w = pack_bf16x2(__uint_as_float(w[6]) * inv_l, __uint_as_float(w[7]) * inv_l);
            *reinterpret_cast<uint4*>(box + sw128_offset(row, cc * 4 + ch)) = v;
          }
        }
        const size_t lse_i = static_cast<size_t>(it.bh) * p.T + qrow;
        if (g == 0 && qrow < p.T &&
            ATTN_IN_RANGE(lse_i, 1, static_cast<size_t>(p.B) * p.H * p.T, kSiteChkFwdLse, &g_device_error))
          p.lse[lse_i] = (m_f + __log2f(l_row)) * 0.69314718055994531f;
      }
      // The staged rows go to the store warp; both groups have read O (the next item's first PV overwrites
      // it) and agree on whether to go on.
      fence_async_shared();
      tc_fence_before();
      mbar_arrive_warp(&bars.o_staged);
      if (!named_barrier_and(1, 256, ok && have_next && !*abort)) break;
      it = next;
      t0 += n_kv;
    }
  }

  // Both CTAs end together: the even CTA's MMAs read the odd CTA's shared and tensor memory, and threads of the
  // odd CTA arrive on the even CTA's barriers.
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  if (threadIdx.x == 0) ATTN_TRACE_EVENT(0, 1);
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc_pair(tmem, 512);
  }
}

}  // namespace attn
