// sm_100a building blocks written from the PTX ISA: mbarriers with bounded waits, TMA tensor copies,
// tcgen05 tensor-memory allocation, MMA issue, commit, and TMEM <-> register moves.
//
// Every wait in this file is bounded: after `limit_ns` of global time it records an error code in the
// module's device error word and returns false, so a kernel that loses a handshake ends instead of hanging
// the GPU. Callers propagate the failure by raising the CTA's shared abort flag.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

#ifndef ATTN_DEVICE_INLINE
#define ATTN_DEVICE_INLINE __device__ __forceinline__
#endif

namespace sm100 {

// ---------------------------------------------------------------------------------------------------------
// Error reporting shared with the host (see attn_get_device_error in include/attn.h).
// Bits: low 8 bits = error kind, next bits = where (kernel-specific site id).
enum : uint32_t { DEV_ERR_TIMEOUT = 1u, DEV_ERR_BOUNDS = 2u };

// Debug builds (-DATTN_DEBUG, libattn_debug.so) check every plain-address access -- the ones no tensor map
// bounds -- before it is made: `off` .. `off + len` (in elements) must lie inside the `n` elements the host
// passed for that array. A failed check records DEV_ERR_BOUNDS | (site << 8) in *err and the caller skips the
// access. In the release build the check is the constant true and costs nothing.
ATTN_DEVICE_INLINE bool range_ok(uint64_t off, uint64_t len, uint64_t n, uint32_t site, uint32_t* err) {
  if (off <= n && len <= n - off) return true;
  atomicOr(err, DEV_ERR_BOUNDS | (site << 8));
  return false;
}
#ifdef ATTN_DEBUG
#define ATTN_IN_RANGE(off, len, n, site, err) \
  (::sm100::range_ok(static_cast<uint64_t>(off), static_cast<uint64_t>(len), static_cast<uint64_t>(n), (site), (err)))
#else  // the arguments are referenced (not evaluated), so extents computed only for the checks stay "used"
#define ATTN_IN_RANGE(off, len, n, site, err) (static_cast<void>(sizeof((off) + (len) + (n))), true)
#endif

ATTN_DEVICE_INLINE uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

ATTN_DEVICE_INLINE uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

ATTN_DEVICE_INLINE bool elect_one() {
  uint32_t pred = 0;
  asm volatile(
      "{\n\t.reg .pred P;\n\t"
      "elect.sync _|P, 0xffffffff;\n\t"
      "selp.b32 %0, 1, 0, P;\n\t}"
      : "=r"(pred));
  return pred != 0;
}

// Named barrier among `count` threads (a multiple of 32) of the CTA; id 0 is __syncthreads.
ATTN_DEVICE_INLINE void named_barrier(uint32_t id, uint32_t count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Named barrier that also ANDs `pred` over the participating threads; every participant gets the result,
// so a decision taken on it (leave a loop, say) is the same in all of them.
ATTN_DEVICE_INLINE bool named_barrier_and(uint32_t id, uint32_t count, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred P, Q;\n\t"
      "setp.ne.u32 P, %1, 0;\n\t"
      "bar.red.and.pred Q, %2, %3, P;\n\t"
      "selp.u32 %0, 1, 0, Q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred)), "r"(id), "r"(count)
      : "memory");
  return r != 0;
}

// ---------------------------------------------------------------------------------------------------------
// mbarrier

ATTN_DEVICE_INLINE void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

ATTN_DEVICE_INLINE void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

ATTN_DEVICE_INLINE void mbar_arrive(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\t"
      "mbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
      : "memory");
}

ATTN_DEVICE_INLINE void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

ATTN_DEVICE_INLINE bool mbar_try_wait(uint32_t bar_addr, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred P;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 P, [%1], %2;\n\t"
      "selp.b32 %0, 1, 0, P;\n\t}"
      : "=r"(ok)
      : "r"(bar_addr), "r"(parity)
      : "memory");
  return ok != 0;
}

// Non-blocking test: has the phase with the given parity of `bar` completed? (Unlike try_wait, never suspends.)
ATTN_DEVICE_INLINE bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred P;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 P, [%1], %2;\n\t"
      "selp.b32 %0, 1, 0, P;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait until the phase with the given parity of `bar` has completed. Gives up when `*abort` becomes
// non-zero (another role of the CTA failed) or after `limit_ns`; on a timeout it raises `*abort`, records
// `site` in `err_word` and returns false.
ATTN_DEVICE_INLINE bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort, uint64_t limit_ns,
                                  uint32_t* err_word, uint32_t site) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try_wait(a, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(a, parity)) return true;
    if ((i & 63u) == 0) {
      if (*abort) return false;
      if (global_timer_ns() - t0 > limit_ns) {
        *abort = 1;
        atomicOr(err_word, DEV_ERR_TIMEOUT | (site << 8));
        return false;
      }
    }
  }
}

// One arrival for the whole warp: the lanes synchronise, which orders their earlier writes (and, after a
// tcgen05.fence::before_thread_sync, their tensor-memory accesses) before lane 0's release-arrive, so the
// barrier counts warps. All 32 lanes must call it together. (Arrivals are atomics on one shared-memory word:
// 128 per phase, one per thread, serialise into hundreds of cycles on a critical path.)
ATTN_DEVICE_INLINE void mbar_arrive_warp(uint64_t* bar) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

// Warp-uniform form of mbar_wait for roles in which the whole warp then issues warp-collective tcgen05.ld/st
// (.sync.aligned): every lane waits, and the warp proceeds only if every lane succeeded, so a failure can
// never leave part of a warp inside a collective. All 32 lanes must call it together.
ATTN_DEVICE_INLINE bool mbar_wait_warp(uint64_t* bar, uint32_t parity, volatile int* abort, uint64_t limit_ns,
                                       uint32_t* err_word, uint32_t site) {
  const bool ok = mbar_wait(bar, parity, abort, limit_ns, err_word, site);
  return __all_sync(0xffffffffu, ok);
}

// ---------------------------------------------------------------------------------------------------------
// Proxy fences

// Make generic-proxy writes to shared memory visible to the async proxy (TMA store, tcgen05.mma reads).
ATTN_DEVICE_INLINE void fence_async_shared() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------------------------------------------------
// TMA (cp.async.bulk.tensor) with a CUtensorMap passed as a __grid_constant__ kernel parameter.

ATTN_DEVICE_INLINE void tma_prefetch_desc(const void* tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}

ATTN_DEVICE_INLINE void tma_load_4d(void* dst, const void* tmap, uint64_t* bar, int c0, int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

// Prefetch a TMA tile into L2 (no shared memory, no completion to wait for).
ATTN_DEVICE_INLINE void tma_prefetch_l2_4d(const void* tmap, int c0, int c1, int c2, int c3) {
  asm volatile("cp.async.bulk.prefetch.tensor.4d.L2.global.tile [%0, {%1, %2, %3, %4}];" ::"l"(
                   reinterpret_cast<uint64_t>(tmap)),
               "r"(c0), "r"(c1), "r"(c2), "r"(c3)
               : "memory");
}

ATTN_DEVICE_INLINE void tma_store_4d(const void* tmap, const void* src, int c0, int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(tmap)),
      "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

ATTN_DEVICE_INLINE void tma_store_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

ATTN_DEVICE_INLINE void tma_store_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

ATTN_DEVICE_INLINE void tma_store_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Wait until at most N of this thread's most recent bulk groups still read their shared-memory source.
template <int N>
ATTN_DEVICE_INLINE void tma_store_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

// 16-byte asynchronous copy global -> shared through L2 only (cp.async.cg), tracked by this thread's cp.async
// groups; with fill = false nothing is read and the 16 bytes are zeroed. Both addresses 16-byte aligned.
ATTN_DEVICE_INLINE void cp_async_16(void* smem_dst, const void* gmem_src, bool fill) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem_dst)), "l"(gmem_src),
               "r"(fill ? 16 : 0)
               : "memory");
}
ATTN_DEVICE_INLINE void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// Wait until at most N of this thread's most recent cp.async groups are still in flight.
template <int N>
ATTN_DEVICE_INLINE void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Untiled bulk copy global -> shared; both addresses 16-byte aligned, bytes a multiple of 16.
ATTN_DEVICE_INLINE void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Untiled bulk reduction shared -> global: dst[i] += src[i] for `bytes / 4` fp32 values, done by the async
// engine (not the load/store unit). Both addresses 16-byte aligned, bytes a multiple of 16; completes through
// the issuing thread's bulk group (tma_store_commit / tma_store_wait_*).
ATTN_DEVICE_INLINE void bulk_reduce_add_f32(float* dst, const void* src, uint32_t bytes) {
  asm volatile("cp.reduce.async.bulk.global.shared::cta.bulk_group.add.f32 [%0], [%1], %2;" ::"l"(
                   reinterpret_cast<uint64_t>(dst)),
               "r"(smem_u32(src)), "r"(bytes)
               : "memory");
}

// ---------------------------------------------------------------------------------------------------------
// tcgen05: tensor memory

ATTN_DEVICE_INLINE void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {  // whole warp
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}

ATTN_DEVICE_INLINE void tmem_relinquish() {  // whole warp
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

ATTN_DEVICE_INLINE void tmem_dealloc(uint32_t taddr, uint32_t ncols) {  // whole warp
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

ATTN_DEVICE_INLINE void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
ATTN_DEVICE_INLINE void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// TMEM address: lane in bits [31:16], column in bits [15:0].
ATTN_DEVICE_INLINE uint32_t tmem_addr(uint32_t base, uint32_t lane, uint32_t col) {
  return base + (lane << 16) + col;
}

// ---------------------------------------------------------------------------------------------------------
// tcgen05: descriptors

// Instruction descriptor, kind::f16 with bf16 A and B, fp32 accumulator, dense.
//   [4,6) D format (1 = f32); [7,10) A format (1 = bf16); [10,13) B format (1 = bf16);
//   [15] A major (0 = K-major, 1 = MN-major); [16] B major; [17,23) N >> 3; [24,29) M >> 4.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(uint32_t M, uint32_t N, bool a_mn_major, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) |
         ((N >> 3) << 17) | ((M >> 4) << 24);
}

// Shared-memory matrix descriptor for the 128-byte swizzle layout that TMA writes with
// CU_TENSOR_MAP_SWIZZLE_128B (rows of 128 bytes, 8-row / 1024-byte swizzle atoms, atoms 1024-byte aligned).
//   [0,14) start address >> 4; [16,30) leading byte offset >> 4; [32,46) stride byte offset >> 4;
//   [46,48) version = 1; [49,52) base offset = 0; [52] LBO mode = 0; [61,64) layout = 2 (128B swizzle).
// K-major operand: rows = M or N, 64 K-elements per 128-byte row; LBO unused, SBO = 1024 (next 8 rows).
// MN-major operand: 128-byte rows hold 64 M/N-elements, consecutive rows are consecutive K;
//   LBO = byte distance between 64-element M/N chunks, SBO = 1024 (next 8 K rows).
ATTN_DEVICE_INLINE uint64_t sdesc_sw128(uint32_t smem_addr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= 1ull << 46;
  d |= 2ull << 61;
  return d;
}

// ---------------------------------------------------------------------------------------------------------
// tcgen05: MMA issue (one thread) and commit

// D[tmem] (+)= A[smem] * B[smem]^T-by-descriptor, cta_group::1, kind::f16.
ATTN_DEVICE_INLINE void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc, uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accum)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem], cta_group::1, kind::f16 (A: lane = row, two bf16 per 32-bit column).
ATTN_DEVICE_INLINE void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc, uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accum)
      : "memory");
}

// Arrive once on `bar` when every tcgen05 operation issued so far by this thread has completed.
ATTN_DEVICE_INLINE void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// ---------------------------------------------------------------------------------------------------------
// tcgen05: TMEM <-> registers, shape 32x32b (thread i of the warp <-> lane (warp's lane base + i)).

ATTN_DEVICE_INLINE void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
ATTN_DEVICE_INLINE void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

ATTN_DEVICE_INLINE void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]),
        "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
        "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

ATTN_DEVICE_INLINE void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

ATTN_DEVICE_INLINE void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

ATTN_DEVICE_INLINE void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// ---------------------------------------------------------------------------------------------------------
// CTA pairs (a cluster of two CTAs on the two SMs of a TPC): tcgen05 with cta_group::2 lets one thread of the
// even CTA issue MMAs of M = 256 whose A operand and accumulator are split by rows between the two CTAs'
// tensor memories and whose B operand is split by columns between the two CTAs' shared memories, so each SM
// stages and reads only half of B.

ATTN_DEVICE_INLINE uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Every thread of both CTAs; orders earlier shared-memory writes and barrier inits cluster-wide.
ATTN_DEVICE_INLINE void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Shared::cluster address of the variable at the same offset in the shared memory of CTA `rank` of the cluster.
ATTN_DEVICE_INLINE uint32_t mapa_shared(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}

// Arrive on an mbarrier of either CTA of the cluster. The default (CTA-scope release) semantics, as for a local
// arrival: what the pair hands over this way is tensor memory, ordered by tcgen05.wait and the tcgen05 fences
// around the barrier, and shared memory that only the tensor cores read. (A cluster-scope release waits for
// all of the thread's earlier writes to become visible cluster-wide: ~1-2k cycles on a hot path.)
ATTN_DEVICE_INLINE void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// One arrival for the whole warp on a barrier of CTA `rank` (see mbar_arrive_warp).
ATTN_DEVICE_INLINE void mbar_arrive_warp_cluster(uint64_t* bar, uint32_t rank) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive_cluster(mapa_shared(bar, rank));
}

// mbar_wait for a barrier of a CTA pair. On a timeout it also raises the other CTA's abort flag (`peer_abort`,
// a shared::cluster address), so the pair stops together.
ATTN_DEVICE_INLINE bool mbar_wait_pair(uint64_t* bar, uint32_t parity, volatile int* abort, uint32_t peer_abort,
                                       uint64_t limit_ns, uint32_t* err_word, uint32_t site) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try_wait(a, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(a, parity)) return true;
    if ((i & 63u) == 0) {
      if (*abort) return false;
      if (global_timer_ns() - t0 > limit_ns) {
        *abort = 1;
        asm volatile("st.relaxed.cluster.shared::cluster.u32 [%0], %1;" ::"r"(peer_abort), "r"(1) : "memory");
        atomicOr(err_word, DEV_ERR_TIMEOUT | (site << 8));
        return false;
      }
    }
  }
}

ATTN_DEVICE_INLINE bool mbar_wait_pair_warp(uint64_t* bar, uint32_t parity, volatile int* abort, uint32_t peer_abort,
                                            uint64_t limit_ns, uint32_t* err_word, uint32_t site) {
  const bool ok = mbar_wait_pair(bar, parity, abort, peer_abort, limit_ns, err_word, site);
  return __all_sync(0xffffffffu, ok);
}

// TMA tile load into this CTA's shared memory whose completion (complete_tx) is counted on an mbarrier of
// either CTA of the pair (`bar_cluster`, a shared::cluster address). No multicast.
ATTN_DEVICE_INLINE void tma_load_4d_pair(void* dst, const void* tmap, uint32_t bar_cluster, int c0, int c1, int c2,
                                         int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(bar_cluster), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

// Tensor memory of a pair: executed by the same warp of both CTAs; both get the same column base.
ATTN_DEVICE_INLINE void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
ATTN_DEVICE_INLINE void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
ATTN_DEVICE_INLINE void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem], M = 256 over the pair (issued by one thread of the even CTA).
ATTN_DEVICE_INLINE void mma_ts_pair(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                    uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accum)
      : "memory");
}

// Arrive once on the barrier at `bar`'s offset in each CTA of `cta_mask` when every tcgen05 operation issued so
// far by this thread has completed.
ATTN_DEVICE_INLINE void mma_commit_pair(uint64_t* bar, uint16_t cta_mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(cta_mask)
      : "memory");
}

// ---------------------------------------------------------------------------------------------------------
// Small numeric helpers

ATTN_DEVICE_INLINE float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Pack two floats into bf16x2 (round to nearest even); `lo` goes to the low 16 bits.
ATTN_DEVICE_INLINE uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// 128-byte-swizzle position of the 16-byte chunk `chunk` (0..7) in row `row` of a tile written by TMA with
// CU_TENSOR_MAP_SWIZZLE_128B: the chunk index is XOR-ed with the row index modulo 8.
ATTN_DEVICE_INLINE uint32_t sw128_offset(uint32_t row, uint32_t chunk) {
  return row * 128u + ((chunk ^ (row & 7u)) << 4);
}

}  // namespace sm100
