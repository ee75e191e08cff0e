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
//   1. attn_decode_split_kernel: the units are (sequence, key/value head, chunk of the cache), the chunks with
//      the most blocks first (each CTA counting-sorts the lengths). A persistent grid, one CTA per SM, deals
//      them out in rounds, back and forth; the G = H / H_kv query heads of a unit's group and their Tq new
//      tokens (R = G * Tq rows) share every K and V row the CTA reads, so the cache is read once. The CTA's
//      units stream through a shared-memory ring of 128-key K and V blocks loaded by TMA (three stages, two
//      for 32 rows; one thread issues four 16 KB boxes per block onto the stage's mbarrier), all but one block
//      in flight while one is used, on from one unit into the next; rows past a sequence's length are masked,
//      never used. Per block, in four independent groups of two warps that each take 32 of the block's keys
//      (one CTA barrier per block, for the ring): two threads score each key against all rows (half the dims
//      each, a shuffle to add), the group updates its own running max and its warps' running sums (online
//      softmax in base 2), and a thread per pair of output dimensions accumulates O over the group's keys. The
//      groups' results are merged once per unit by their maxima.
//      The chunk's unnormalised O, running max and sum go to a workspace; when the cache is not split (one
//      chunk per (sequence, head)) the kernel normalises and writes o and lse itself. The kernel is
//      instantiated for 1, 2, 4, 8, 16 and 32 rows.
//   2. attn_decode_combine_kernel (only when the cache is split): one warp per (sequence, query head, new
//      token) merges the chunks by their log-sum-exp and writes o and lse.
#pragma once
#include "attn_common.cuh"
#include "sm100.cuh"

namespace attn {

// Threads of the split kernel. Scoring takes kThreads / 128 threads per key, each over 128 / that dims; the
// threads form kThreads / 64 groups of two warps, each taking kThreads / 64-th of a block's keys (scoring,
// softmax and P V) with a thread per pair of output dimensions. 256 for every group size: 512 (four threads per
// key, eight groups) measured 29-36 % slower on the decode workloads, the extra warps only lengthening each
// block's chains of shared-memory loads and shuffles.
template <int kRows>
__host__ __device__ constexpr int dec_threads() { return 256; }
constexpr int kDecKeys = 128;       // keys per block
constexpr int kDecMaxRows = 32;     // R = (H / H_kv) * Tq query rows per CTA, at most
constexpr int kDecChunkKeys = 256;  // keys per split of the cache, at least
constexpr int kDecMaxUnits = 64;    // (sequence, key/value head, chunk) units one CTA walks, at most
constexpr uint32_t kDecBlockBytes = kDecKeys * 256;  // one K or V block: 128 keys x 128 dims, bf16

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
  int order_nb;                // > 0: the CTAs take the (sequence, chunk) pairs longest first, and no chunk
                               // holds more than order_nb 128-key blocks; 0: in index order
  float scale_log2;            // scale * log2(e)
  uint64_t timeout_ns;         // limit of any single wait
};

// K/V blocks in the shared-memory ring: three (two in flight while one is used), two for 32 rows, whose q rows
// and scores (32 KB) leave no room for a third beside the groups' softmax state.
template <int kRows>
__host__ __device__ constexpr int dec_stages() { return kRows >= 32 ? 2 : 3; }

// A unit of the split kernel's walk: chunk sp of sequence b for key/value head hk, and the chunk's keys
// [key_lo, key_hi) of the sequence's L, in nblk 128-key blocks.
struct DecUnit {
  int b, sp, hk, L, key_lo, key_hi, nblk;
};

// Dynamic shared memory of the split kernel for up to kRows query rows (no static shared memory, so the block
// starts 1024-byte aligned, as the 128-byte-swizzled TMA boxes need): the ring of (K block, V block) pairs, the
// rows (fp32, pre-scaled), the block's scores, then P, each warp's block max and running sum per row, each
// group's running max per row (two slots), one mbarrier per ring stage, the abort flag (8 bytes) and the CTA's
// units (DecUnit each): 195 KB for one row, 211 KB for 16, 165 KB for 32 (two ring stages).
template <int kRows>
__host__ __device__ constexpr size_t dec_bar_offset() {  // the stage barriers, 8-byte aligned
  constexpr int kWarps = dec_threads<kRows>() / 32, kGroups = kWarps / 2;
  return (dec_stages<kRows>() * 2 * kDecBlockBytes + 2 * kRows * 128 * 4 + (2 * kWarps + 2 * kGroups) * kRows * 4 + 7) /
         8 * 8;
}
template <int kRows>
__host__ __device__ constexpr size_t dec_smem_bytes() {
  return dec_bar_offset<kRows>() + dec_stages<kRows>() * 8 + 8 + kDecMaxUnits * sizeof(DecUnit);
}
static_assert(dec_smem_bytes<kDecMaxRows>() <= 232448, "decode split kernel exceeds the 227 KB shared-memory opt-in");

// A K or V block is two TMA boxes of 64 dims x 128 keys (16 KB each, dims 0-63 then 64-127) in the 128-byte
// swizzle: 16-byte chunk c of key j's 128-byte row of a box sits at chunk c ^ (j & 7). The scoring reads (a lane
// pair per key, eight chunks each) and the P V reads (a warp over one 128-byte row) hit every bank evenly.
__device__ __forceinline__ uint32_t dec_box_off(int j, int c) { return j * 128 + ((c ^ (j & 7)) << 4); }

enum : uint32_t { kSiteDecFull = 0x31, kSiteDecDrain = 0x32 };

// The keys [key_lo, key_hi) that chunk sp of sequence b covers, in nblk 128-key blocks: from the first row's
// window start (0 without a window) on, chunk keys per split, up to the sequence's length L.
struct DecChunk {
  int L, key_lo, key_hi, nblk;
};
__device__ __forceinline__ DecChunk dec_chunk(const DecodeParams& p, int b, int sp) {
  DecChunk c;
  c.L = min(max(p.seqlens[b], 0), p.Tk);  // lengths outside [0, Tk] are clamped
  const int start = p.window < 0 ? 0 : max(0, c.L - p.Tq - p.window);
  c.key_lo = start + sp * p.chunk;
  c.key_hi = min(c.L, c.key_lo + p.chunk);
  c.nblk = c.key_hi > c.key_lo ? (c.key_hi - c.key_lo + kDecKeys - 1) / kDecKeys : 0;
  return c;
}

// Bytes of the ring's first stage that the longest-first order may use as scratch: a histogram of order_nb + 1
// ints and a block count (16 bits) per (sequence, chunk) pair.
constexpr int kDecOrderScratch = 2 * kDecBlockBytes;

// The longest-first order of the (sequence, chunk) pairs b * n_split + sp: a counting sort by block count, most
// blocks first, equal counts in index order. The CTAs deal the units out in this order, so that the short chunks
// fill in at the end (the list-scheduling rule); in index order each SM's last units hold long and short chunks
// alike and SMs idle while the long ones finish. Every CTA sorts the same lengths the same way, so the order is
// one permutation. dec_order_build (all threads) counts the pairs per block count into scratch: a histogram of
// order_nb + 1 ints, then each pair's count in 16 bits.
template <int kThreads>
__device__ void dec_order_build(const DecodeParams& p, uint8_t* scratch) {
  int* hist = reinterpret_cast<int*>(scratch);                        // [order_nb + 1]
  uint16_t* nb = reinterpret_cast<uint16_t*>(hist + p.order_nb + 1);  // [B * n_split]
  const int t = threadIdx.x, n_pairs = p.B * p.n_split;
  for (int i = t; i <= p.order_nb; i += kThreads) hist[i] = 0;
  __syncthreads();
  for (int i = t; i < n_pairs; i += kThreads) {
    const int n = min(dec_chunk(p, i / p.n_split, i % p.n_split).nblk, p.order_nb);
    nb[i] = static_cast<uint16_t>(n);
    atomicAdd(&hist[n], 1);
  }
  __syncthreads();
}

// The pair at position q of the order (called by a whole warp; the same value in every lane), or -1 if q is not a
// position (it always is for q in 0 .. B * n_split - 1: the counts' position ranges partition them).
__device__ __forceinline__ int dec_order_find(const DecodeParams& p, int q, const uint8_t* scratch) {
  const int* hist = reinterpret_cast<const int*>(scratch);
  const uint16_t* nb = reinterpret_cast<const uint16_t*>(hist + p.order_nb + 1);
  const int lane = threadIdx.x & 31, n_pairs = p.B * p.n_split;
  // The count x whose pairs hold position q, walking the counts from order_nb down 32 at a time (lane l takes
  // count top - l), and q's rank r among them.
  int x = -1, r = 0, above = 0;  // above: pairs with more blocks than this window's counts
  for (int top = p.order_nb; top >= 0 && x < 0; top -= 32) {
    const int c = top - lane >= 0 ? hist[top - lane] : 0;
    int s = c;  // pairs in this window's counts top .. top - lane
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, d);
      if (lane >= d) s += y;
    }
    const int first = above + s - c;  // position of this count's first pair
    const unsigned hit = __ballot_sync(0xffffffffu, c > 0 && q >= first && q < first + c);
    if (hit) {
      const int l = __ffs(hit) - 1;
      x = top - l;
      r = q - __shfl_sync(0xffffffffu, first, l);
    }
    above += __shfl_sync(0xffffffffu, s, 31);
  }
  // The r-th pair with x blocks, in index order, 32 pairs at a time.
  for (int base = 0; x >= 0 && base < n_pairs; base += 32) {
    unsigned m = __ballot_sync(0xffffffffu, base + lane < n_pairs && nb[base + lane] == x);
    const int c = __popc(m);
    if (r < c) {
      for (int k = 0; k < r; ++k) m &= m - 1;
      return base + __ffs(m) - 1;
    }
    r -= c;
  }
  return -1;
}

// Position of a CTA's k-th unit: the units are dealt to the G CTAs in rounds, back and forth (CTA c takes
// positions c, 2G - 1 - c, 2G + c, ...), so that with the units longest first every CTA's total is about even.
__device__ __forceinline__ long long dec_unit_pos(int c, int k, int G) {
  return static_cast<long long>(k) * G + ((k & 1) ? G - 1 - c : c);
}

// (One CTA fits an SM by shared memory. The one-row kernel is held to 128 registers, at which it ran 2 % faster
// than at 125 with the bound at one CTA; the others take what they need, unspilled.)
template <int kRows>
__global__ void __launch_bounds__(dec_threads<kRows>(), kRows == 1 ? 2 : 1) attn_decode_split_kernel(
    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v, const DecodeParams p) {
  using namespace sm100;
  constexpr int kThreads = dec_threads<kRows>();
  constexpr int kStages = dec_stages<kRows>();
  constexpr int kWarps = kThreads / 32, kGroups = kWarps / 2;  // a group: two warps, one key slice
  constexpr bool kPvSplit = kRows == 2;  // P V keeps two partial sums per output for two rows
  constexpr int kPart = kThreads / kDecKeys;   // scoring threads per key (2 or 4), kDims = 128 / kPart dims each
  constexpr int kDims = 128 / kPart;
  constexpr int kSlices = kThreads / 64;       // P V: key slices of kSliceKeys keys (4 x 32 or 8 x 16)
  constexpr int kSliceKeys = kDecKeys / kSlices;
  extern __shared__ __align__(1024) uint8_t dec_smem[];
  if (smem_u32(dec_smem) & 1023u) {  // the swizzled boxes need a 1024-byte aligned block
    if (threadIdx.x == 0) atomicOr(&g_device_error, DEV_ERR_TIMEOUT | (kSiteDecFull << 8));
    return;
  }
  float (*qs)[128] = reinterpret_cast<float (*)[128]>(dec_smem + kStages * 2 * kDecBlockBytes);
  float (*sc)[kDecKeys] = reinterpret_cast<float (*)[kDecKeys]>(qs + kRows);  // scores, then P
  float* wmax = reinterpret_cast<float*>(sc + kRows);  // [kWarps][kRows]: each warp's block max per row
  float* gl = wmax + kWarps * kRows;                   // [kWarps][kRows]: each warp's running sum per row
  float* gm = gl + kWarps * kRows;                     // [2][kGroups][kRows]: each group's running max, by parity
  uint64_t* full = reinterpret_cast<uint64_t*>(dec_smem + dec_bar_offset<kRows>());
  volatile int* abort = reinterpret_cast<volatile int*>(full + kStages);
  DecUnit* units = reinterpret_cast<DecUnit*>(full + kStages + 1);  // this CTA's units, in walk order

  const int t = threadIdx.x, warp = t / 32, lane = t % 32;
  const int G = p.H / p.Hkv, R = p.R;
  const size_t n_q = static_cast<size_t>(p.B) * p.Tq * p.H * 128;
  const uint64_t lim = p.timeout_ns;
  // The units (sequence, key/value head, chunk) in order: position i is head i % H_kv of the (sequence, chunk)
  // pair at position i / H_kv of the pairs, longest first or in index order. This CTA takes positions
  // dec_unit_pos(blockIdx.x, k, gridDim.x), k = 0, 1, ...: one unit per CTA when the grid has one CTA per unit,
  // else a persistent walk whose K/V ring runs on from one unit into the next.
  const long long n_units = static_cast<long long>(p.B) * p.Hkv * p.n_split;
  int n_mine = 0;
  while (n_mine < kDecMaxUnits && dec_unit_pos(blockIdx.x, n_mine, gridDim.x) < n_units) ++n_mine;
  if (p.order_nb > 0) dec_order_build<kThreads>(p, dec_smem);
  for (int k = warp; k < n_mine; k += kThreads / 32) {
    const long long pos = dec_unit_pos(blockIdx.x, k, gridDim.x);
    const int pp = static_cast<int>(pos / p.Hkv), hk = static_cast<int>(pos % p.Hkv);
    int pair = p.order_nb > 0 ? dec_order_find(p, pp, dec_smem) : pp;
    if (pair < 0) pair = pp;
    if (lane == 0) {
      const DecChunk c = dec_chunk(p, pair / p.n_split, pair % p.n_split);
      units[k] = DecUnit{pair / p.n_split, pair % p.n_split, hk, c.L, c.key_lo, c.key_hi, c.nblk};
    }
  }
  if (t == 0) {
    for (int st = 0; st < kStages; ++st) mbar_init(&full[st], 1);
    *abort = 0;
    fence_barrier_init();
  }
  fence_async_shared();  // the order's generic accesses to the ring come before the TMA copies into it
  __syncthreads();

  // The issue cursor (thread 0 only): block ib of unit ik's inb blocks, keys from ikey, sequence ibq, head ihk.
  // Blocks go out in one stream over the CTA's units: the n-th into ring stage n % kStages.
  const bool issuer = t == 0;
  int issued = 0, ik = 0, ib = 0, inb = -1, ikey = 0, ibq = 0, ihk = 0;
  auto issue_next = [&]() {
    if (!issuer) return;
    while (ik < n_mine) {
      if (inb < 0) {
        const DecUnit& un = units[ik];
        inb = un.nblk, ikey = un.key_lo, ibq = un.b, ihk = un.hk, ib = 0;
      }
      if (ib < inb) break;
      ++ik, inb = -1;
    }
    if (ik >= n_mine) return;
    // Four TMA boxes, 64 KB on the stage's barrier. The tensor maps bound the copies (rows past the cache come
    // as zeros); rows past a sequence's length are masked below.
    const int kb = ikey + ib * kDecKeys, st = issued % kStages;
    uint8_t* ks = dec_smem + st * 2 * kDecBlockBytes;
    mbar_arrive_expect_tx(&full[st], 2 * kDecBlockBytes);
    for (int c = 0; c < 2; ++c) {
      tma_load_4d(ks + c * 16384, &tm_k, &full[st], c * 64, ihk, kb, ibq);
      tma_load_4d(ks + kDecBlockBytes + c * 16384, &tm_v, &full[st], c * 64, ihk, kb, ibq);
    }
    ++ib, ++issued;
  };
  if (issuer) {
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
#pragma unroll
  for (int n = 0; n < kStages - 1; ++n) issue_next();

  // Unit k's rows, R x 128 bf16 of q, in registers (elements t, t + kThreads, ...): read a unit ahead, so that
  // the loads' latency hides behind the previous unit's blocks. Row r = g * Tq + i is query head hk * G + g,
  // new token i, which sees keys up to L - Tq + i.
  constexpr int kQPer = (kRows * 128 + kThreads - 1) / kThreads;
  __nv_bfloat16 qv[kQPer];
  auto fetch_q = [&](int k) {
    const int qb = units[k].b, qh = units[k].hk;
#pragma unroll
    for (int x = 0; x < kQPer; ++x) {
      const int e = t + x * kThreads;
      qv[x] = __float2bfloat16_rn(0.f);
      if (e < R * 128) {
        const int r = e / 128, d = e % 128, g = r / p.Tq, i = r % p.Tq;
        const size_t qi = ((static_cast<size_t>(qb) * p.Tq + i) * p.H + qh * G + g) * 128 + d;
        if (ATTN_IN_RANGE(qi, 1, n_q, kSiteChkDecQ, &g_device_error)) qv[x] = p.q[qi];
      }
    }
  };
  fetch_q(0);  // (every CTA has a unit: position blockIdx.x < the grid <= the units)

  // P V: output dimensions 2 dp, 2 dp + 1 over keys [kSliceKeys kq, kSliceKeys (kq + 1)) of each block
  const int dp = t & 63, kq = t >> 6;
  int consumed = 0;  // blocks of the stream whose barrier phase this CTA has waited for
  bool ok = true;
  for (int k = 0; k < n_mine && ok; ++k) {
    const DecUnit un = units[k];
    const int b = un.b, sp = un.sp, hk = un.hk, bhk = b * p.Hkv + hk;
    const int L = un.L, key_lo = un.key_lo, key_hi = un.key_hi, nblk = un.nblk;
#pragma unroll
    for (int x = 0; x < kQPer; ++x) {
      const int e = t + x * kThreads;
      if (e < R * 128) qs[e / 128][e % 128] = __bfloat162float(qv[x]) * p.scale_log2;
    }
    if (k + 1 < n_mine) fetch_q(k + 1);
    for (int i = t; i < kWarps * kRows; i += kThreads) gl[i] = 0.f;
    for (int i = t; i < kGroups * kRows; i += kThreads) gm[i] = -INFINITY;  // parity 0, which the first block reads
    float acc[kRows][2], acc2[kRows][2];
#pragma unroll
    for (int r = 0; r < kRows; ++r) acc[r][0] = acc[r][1] = acc2[r][0] = acc2[r][1] = 0.f;

    for (int n = 0; n < nblk; ++n) {
      // The previous block's stage and P are no longer read (the stage takes the stream's block after next), and
      // every warp's waits so far succeeded. A warp whose wait for this block runs out computes on regardless;
      // the CTA leaves at the next block's barrier (or the unit's) without writing the unit.
      if (!__syncthreads_and(ok)) {
        ok = false;
        break;
      }
      issue_next();
      const int g = consumed;
      if (mbar_wait_warp(&full[g % kStages], (g / kStages) & 1, abort, lim, &g_device_error, kSiteDecFull))
        consumed = g + 1;
      else
        ok = false;
      const uint8_t* ks = dec_smem + (g % kStages) * 2 * kDecBlockBytes;
      const uint8_t* vs = ks + kDecBlockBytes;
      const int kb = key_lo + n * kDecKeys, nk = min(kDecKeys, key_hi - kb);
      {
        // Scores of key j = t / kPart against every row: this thread takes dims [kDims h, kDims (h + 1)),
        // h = t % kPart, and the key's threads (adjacent lanes) add their parts. Keys past the block, past the
        // sequence or past a row's last key are -inf (selected, so whatever those rows of the cache hold never
        // enters a score).
        const int j = t / kPart, h = t % kPart;
        const int box = (h * kDims) / 64, c0 = ((h * kDims) % 64) / 8;  // the part's first 16-byte chunk
        uint4 kw[kDims / 8];
#pragma unroll
        for (int c = 0; c < kDims / 8; ++c)
          kw[c] = *reinterpret_cast<const uint4*>(ks + box * 16384 + dec_box_off(j, c0 + c));
        // Rows in turn; up to four rows unrolled so that their chains overlap (two rows: 7.7 % less time on
        // decode_d20_gqa).
#pragma unroll
        for (int r = 0; r < (kRows <= 4 ? kRows : R); ++r) {
          if (r >= R) break;
          const float4* q4 = reinterpret_cast<const float4*>(qs[r] + kDims * h);
          float s0 = 0.f, s1 = 0.f;
#pragma unroll
          for (int c = 0; c < kDims / 8; ++c) {
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
          float sj = s0 + s1;
#pragma unroll
          for (int o = 1; o < kPart; o <<= 1) sj += __shfl_xor_sync(0xffffffffu, sj, o);
          const int last = L - p.Tq + r % p.Tq;  // last key this row sees (its own position)
          const bool seen = j < nk && kb + j <= last && (p.window < 0 || kb + j >= last - p.window);
          const float v = seen ? sj : -INFINITY;
          if (h == 0) sc[r][j] = v;
          float mx = v;  // the warp's block max (its 32 / kPart keys)
#pragma unroll
          for (int o = kPart; o < 32; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
          if (lane == 0) wmax[warp * kRows + r] = mx;
        }
      }
      // The group's online softmax (its two warps; keys [32 kq, 32 kq + 32) of the block): the running max of
      // each row takes the two warps' block maxima, P = exp2(s - max) replaces the scores in place, each warp
      // adds its P to its own running sum, and O is rescaled. The running max alternates between two slots by
      // block parity, so this block's reads never meet the write for the next.
      named_barrier(1 + kq, 64);
      {
        const int j = t / kPart, h = t % kPart;
        const float* gm_old = gm + ((n & 1) * kGroups + kq) * kRows;
        float* gm_new = gm + (((n + 1) & 1) * kGroups + kq) * kRows;
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
          if (r < R) {
            const float m_old = gm_old[r];
            const float m_new = fmaxf(m_old, fmaxf(wmax[2 * kq * kRows + r], wmax[(2 * kq + 1) * kRows + r]));
            const float a = m_old == m_new ? 1.f : exp2f(m_old - m_new);  // 0 when nothing was seen before
            float pe = 0.f;
            if (h == 0) {
              pe = m_new == -INFINITY ? 0.f : exp2f(sc[r][j] - m_new);
              sc[r][j] = pe;
            }
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) pe += __shfl_xor_sync(0xffffffffu, pe, o);
            if (lane == 0) gl[warp * kRows + r] = gl[warp * kRows + r] * a + pe;
            if ((t & 63) == 0) gm_new[r] = m_new;
            acc[r][0] *= a, acc[r][1] *= a;
            if constexpr (kPvSplit) acc2[r][0] *= a, acc2[r][1] *= a;
          }
        }
      }
      named_barrier(1 + kq, 64);  // the group's P is written
      // O[r][d] = O[r][d] * a_r + sum_j P[r][j] V[j][d] for this thread's two dims over its slice of the keys:
      // one 4-byte load per key for V (a warp reads one 128-byte box row), P four keys at a time. V rows past
      // the sequence's keys are taken as 0 (selected, not multiplied, so the cache's contents there do not
      // matter), and their P is 0.
      const uint8_t* vbox = vs + (dp >> 5) * 16384;
#pragma unroll 2
      for (int j0 = kSliceKeys * kq; j0 < kSliceKeys * (kq + 1); j0 += 4) {
        float v0[4], v1[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(
              *reinterpret_cast<const __nv_bfloat162*>(vbox + dec_box_off(j0 + e, (dp & 31) >> 2) + (dp & 3) * 4));
          const bool in = j0 + e < nk;
          v0[e] = in ? f.x : 0.f;
          v1[e] = in ? f.y : 0.f;
        }
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
          if (r < R) {
            const float4 pr = *reinterpret_cast<const float4*>(&sc[r][j0]);
            const float pe[4] = {pr.x, pr.y, pr.z, pr.w};
            float a0 = acc[r][0], a1 = acc[r][1];
            if constexpr (kPvSplit) {  // even keys into acc, odd keys into acc2: two chains of half the length
              float b0 = acc2[r][0], b1 = acc2[r][1];
#pragma unroll
              for (int e = 0; e < 4; e += 2) {
                a0 = fmaf(pe[e], v0[e], a0), a1 = fmaf(pe[e], v1[e], a1);
                b0 = fmaf(pe[e + 1], v0[e + 1], b0), b1 = fmaf(pe[e + 1], v1[e + 1], b1);
              }
              acc2[r][0] = b0;
              acc2[r][1] = b1;
            } else {
#pragma unroll
              for (int e = 0; e < 4; ++e) a0 = fmaf(pe[e], v0[e], a0), a1 = fmaf(pe[e], v1[e], a1);
            }
            acc[r][0] = a0;
            acc[r][1] = a1;
          }
        }
      }
    }
    if (!ok) break;
    __syncthreads();  // the groups' states are final; the q rows and scores become the reduction's buffers
    // The unit's result (an empty chunk leaves max -inf, sum 0, O 0). Per row the largest group max M; group g's
    // O and sums count with the factor 2^(m_g - M) (0 for a group that saw no key). The key slices' scaled O of
    // each pair of dims are added in slice order by slice 0's threads, handed over through two buffers in turn
    // (the q rows and the scores, R x 128 floats each); thread r < R puts row r's M and sum in wmax.
    const float* gm_fin = gm + (nblk & 1) * kGroups * kRows;  // the parity the unit's last block wrote
    float* xb[2] = {&qs[0][0], &sc[0][0]};
    float sum[kRows][2];
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      if (r < R) {
        float M = -INFINITY;
#pragma unroll
        for (int q = 0; q < kGroups; ++q) M = fmaxf(M, gm_fin[q * kRows + r]);
        if constexpr (kPvSplit) acc[r][0] += acc2[r][0], acc[r][1] += acc2[r][1];
        const float mg = gm_fin[kq * kRows + r];
        const float f = mg == -INFINITY ? 0.f : exp2f(mg - M);
        acc[r][0] *= f, acc[r][1] *= f;
        sum[r][0] = 0.f + acc[r][0], sum[r][1] = 0.f + acc[r][1];
        if (t == r) {
          float l = 0.f;
#pragma unroll
          for (int q = 0; q < kGroups; ++q) {
            const float mq = gm_fin[q * kRows + r];
            l += (mq == -INFINITY ? 0.f : exp2f(mq - M)) * (gl[2 * q * kRows + r] + gl[(2 * q + 1) * kRows + r]);
          }
          wmax[r] = M;
          wmax[kRows + r] = l;
        }
      }
    }
#pragma unroll
    for (int j = 1; j <= kSlices; ++j) {
      if (j < kSlices && kq == j) {
#pragma unroll
        for (int r = 0; r < kRows; ++r)
          if (r < R)
            *reinterpret_cast<float2*>(xb[(j - 1) & 1] + r * 128 + 2 * dp) = make_float2(acc[r][0], acc[r][1]);
      }
      if (j >= 2 && kq == 0) {
#pragma unroll
        for (int r = 0; r < kRows; ++r)
          if (r < R) {
            const float2 x = *reinterpret_cast<const float2*>(xb[j & 1] + r * 128 + 2 * dp);
            sum[r][0] += x.x, sum[r][1] += x.y;
          }
      }
      if (j < kSlices) __syncthreads();
    }
    if (p.n_split == 1) {
      // The only chunk of its (sequence, head): the result is final, so it is normalised and written here as the
      // combine kernel would (that kernel is not launched): o = O / l, lse = M + log2(l) in natural-log units.
      if (kq == 0) {
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
          if (r < R) {
            const int i = r % p.Tq, h = hk * G + r / p.Tq;
            const float l = wmax[kRows + r];
            const float inv = l > 0.f ? 1.f / l : 0.f;
            const size_t o_off = ((static_cast<size_t>(b) * p.Tq + i) * p.H + h) * 128 + 2 * dp;
            if (ATTN_IN_RANGE(o_off, 2, static_cast<size_t>(p.B) * p.Tq * p.H * 128, kSiteChkDecO, &g_device_error))
              *reinterpret_cast<__nv_bfloat162*>(p.o + o_off) =
                  __halves2bfloat162(__float2bfloat16_rn(sum[r][0] * inv), __float2bfloat16_rn(sum[r][1] * inv));
          }
        }
      }
      if (t < R) {
        const int i = t % p.Tq, h = hk * G + t / p.Tq;
        const float l = wmax[kRows + t];
        const size_t lse_i = (static_cast<size_t>(b) * p.H + h) * p.Tq + i;
        if (ATTN_IN_RANGE(lse_i, 1, static_cast<size_t>(p.B) * p.H * p.Tq, kSiteChkDecLse, &g_device_error))
          p.lse[lse_i] = l > 0.f ? (wmax[t] + __log2f(l)) * 0.69314718055994531f : -INFINITY;
      }
    } else {
      const size_t n_part = static_cast<size_t>(p.B) * p.Hkv * p.n_split * R;  // partial rows
      const size_t part = (static_cast<size_t>(bhk) * p.n_split + sp) * R;      // this chunk's first one
      if (ATTN_IN_RANGE(part, R, n_part, kSiteChkDecPart, &g_device_error)) {
        if (kq == 0) {
#pragma unroll
          for (int r = 0; r < kRows; ++r)
            if (r < R)
              *reinterpret_cast<float2*>(p.part_o + (part + r) * 128 + 2 * dp) = make_float2(sum[r][0], sum[r][1]);
        }
        if (t < R) {
          float* pml = p.part_ml + (part + t) * 2;
          pml[0] = wmax[t];
          pml[1] = wmax[kRows + t];
        }
      }
    }
    __syncthreads();  // the q rows, scores and the groups' states are free for the next unit
  }
  // Blocks issued but not consumed (only after a failure: at most the failed block and the two after it) land
  // before the CTA leaves.
  if (t == 0) {
    volatile int no_abort = 0;
    for (int g = consumed; g < issued; ++g)
      mbar_wait(&full[g % kStages], (g / kStages) & 1, &no_abort, lim, &g_device_error, kSiteDecDrain);
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
