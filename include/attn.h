/*
 * attn.h - C ABI of the B200 (sm_100a) bf16 causal multi-head self-attention library (libattn.so).
 *
 * What it computes. nanochat calls flash_attn_func(q, k, v, causal=True, window_size=...) on [B, T, H, D]
 * tensors and trains through it (apidog "Train your own ChatGPT", section 5 "Flash Attention integration";
 * the [B, T, n_head, head_dim] view is in section 1 "GPT model"). The pages print no formula, so this
 * library implements the textbook definition, per batch b and head h, with s = `scale`:
 *
 *   forward   S = s * Q K^T with S[i][j] = -inf for j > i (top-left causal mask, T_q = T_k)
 *             O = softmax_rows(S) V,   LSE[i] = ln sum_j exp(S[i][j])          (natural log)
 *   backward  P = exp(S - LSE),  dV = P^T dO,  dP = dO V^T,  Delta = rowsum(dO * O),
 *             dS = P * (dP - Delta),  dQ = s * dS K,  dK = s * dS^T Q
 *
 * Shapes come from nanochat's depth dial: width 64 * depth, 128 dims per head (aisight.pl nanochat review,
 * "Model and scaling assumptions": d20 = 1280 channels, 10 heads of 128), so D = 128 is the only head size.
 *
 * Conventions for every entry point
 *   - Tensors are device pointers. q, k, v, o, dO, dq, dk, dv: bf16, [B, T, H, D] contiguous (D fastest).
 *     lse: fp32 [B, H, T] contiguous. Every pointer must be 16-byte aligned (TMA requirement), except the
 *     int32 / fp32 vectors of attn_decode (lse, cache_seqlens) and attn_qk_norm_rope[_bwd] (pos_offsets),
 *     which need 4 bytes.
 *   - The caller owns and allocates every buffer, including the backward workspace. The library never
 *     allocates, frees or synchronises; all work is enqueued asynchronously on `stream` (a cudaStream_t;
 *     NULL = legacy default stream) on the current CUDA device.
 *   - Outputs must not overlap inputs or each other (the QK-norm + RoPE prologue calls alone also accept an
 *     output that is exactly its own input, for in-place use).
 *   - Argument errors are detected on the host before anything is launched and leave outputs untouched.
 *   - There is no CPU fallback: on a machine without an sm_100 device the calls return ATTN_ERR_CUDA.
 */
#ifndef ATTN_H_
#define ATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ATTN_OK = 0,
  ATTN_ERR_INVALID_ARG = 1,  /* null pointer, non-positive size, non-finite or non-positive scale, overlap */
  ATTN_ERR_UNSUPPORTED = 2,  /* D != 128, or sizes beyond the kernels' index range */
  ATTN_ERR_MISALIGNED = 3,   /* a pointer is not 16-byte aligned */
  ATTN_ERR_CUDA = 4,         /* a CUDA runtime/driver call or a launch failed; see attn_last_cuda_error() */
  ATTN_ERR_TIMEOUT = 5,      /* a kernel gave up on a bounded wait (reported by attn_get_device_error) */
  ATTN_ERR_WORKSPACE = 6,    /* backward workspace missing or smaller than attn_bwd_workspace_bytes() */
  ATTN_ERR_BOUNDS = 7        /* debug build: a kernel's address check failed (reported by attn_get_device_error) */
} attn_status;

/* Version of this ABI; bumped on any incompatible change of a signature or of a buffer layout
 * (2: the prologue calls report CUDA errors through attn_last_cuda_error like every other call). */
int attn_abi_version(void);

/* Human-readable name of a status code (static storage; never NULL). */
const char* attn_status_string(attn_status s);

/* Text of the last CUDA error seen by this library on the calling thread ("" if none). */
const char* attn_last_cuda_error(void);

/*
 * Forward: o = softmax(scale * q k^T + causal mask) v and lse = per-row natural log-sum-exp of the scaled,
 * masked logits (the saved statistic the backward needs).
 *   q, k, v  in : bf16 [B, T, H, D]
 *   o       out : bf16 [B, T, H, D]
 *   lse     out : fp32 [B, H, T]
 *   B, H, T >= 1; D must be 128; scale finite and > 0 (usually 1/sqrt(D)).
 * Launches one kernel. Returns ATTN_OK once the launch is enqueued.
 */
attn_status attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int T,
                     int D, float scale, void* stream);

/*
 * Size in bytes of the scratch buffer attn_bwd needs for these sizes (0 if the sizes are invalid):
 * per (b, h) row, LSE * log2(e) and Delta (fp32, T rounded up to 128) and an fp32 dQ accumulator.
 */
size_t attn_bwd_workspace_bytes(int B, int H, int T, int D);

/*
 * Backward: dq, dk, dv of L = sum(dO * o), for o and lse returned by attn_fwd on the same q, k, v, scale.
 *   q, k, v, o, dO    in : bf16 [B, T, H, D];   lse in : fp32 [B, H, T]
 *   dq, dk, dv       out : bf16 [B, T, H, D]
 *   workspace  scratch   : device buffer of at least attn_bwd_workspace_bytes(B, H, T, D) bytes,
 *                          256-byte aligned; its contents on entry do not matter and are overwritten.
 * Launches three kernels (Delta/LSE preprocessing with accumulator zeroing; dK/dV with dQ accumulation;
 * dQ conversion). Calls that share one workspace must not overlap in time on the GPU.
 */
attn_status attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                     const void* dO, void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes,
                     int B, int H, int T, int D, float scale, void* stream);

/*
 * The three stages of attn_bwd, callable one at a time with exactly attn_bwd's arguments (the same checks
 * apply). Calling attn_bwd_preprocess, attn_bwd_dkdv, attn_bwd_dq_convert in this order on one stream is
 * the same work as one attn_bwd call; profilers and benchmarks use them to time each kernel on its own.
 *   attn_bwd_preprocess : Delta = rowsum(dO * o), LSE * log2(e) into the workspace; zero the dQ accumulator.
 *   attn_bwd_dkdv       : dk, dv, and dQ partial sums added into the workspace accumulator.
 *   attn_bwd_dq_convert : dq = bf16(scale * accumulator).
 */
attn_status attn_bwd_preprocess(const void* q, const void* k, const void* v, const void* o, const float* lse,
                                const void* dO, void* dq, void* dk, void* dv, void* workspace,
                                size_t workspace_bytes, int B, int H, int T, int D, float scale, void* stream);
attn_status attn_bwd_dkdv(const void* q, const void* k, const void* v, const void* o, const float* lse,
                          const void* dO, void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes,
                          int B, int H, int T, int D, float scale, void* stream);
attn_status attn_bwd_dq_convert(const void* q, const void* k, const void* v, const void* o, const float* lse,
                                const void* dO, void* dq, void* dk, void* dv, void* workspace,
                                size_t workspace_bytes, int B, int H, int T, int D, float scale, void* stream);

/*
 * Grouped-query attention (apidog "Train your own ChatGPT", section 1 "GPT model": fewer key/value heads than
 * query heads). H_kv key/value heads, H_kv >= 1 dividing H; query head h reads key/value head h / (H / H_kv),
 * so consecutive query heads share one (the pages do not print the mapping; this is the plainest reading).
 * H_kv = H is exactly attn_fwd / attn_bwd. Otherwise the same contract, with these shapes:
 *   q, o, dO, dq : bf16 [B, T, H, D];   k, v, dk, dv : bf16 [B, T, H_kv, D];   lse : fp32 [B, H, T]
 * dk, dv are the gradients of the shared heads: the sum over each group's query heads. The workspace is
 * attn_bwd_workspace_bytes(B, H, T, D) bytes (per query head). H_kv out of range: ATTN_ERR_INVALID_ARG.
 */
attn_status attn_fwd_gqa(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int H_kv,
                         int T, int D, float scale, void* stream);
attn_status attn_bwd_gqa(const void* q, const void* k, const void* v, const void* o, const float* lse,
                         const void* dO, void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes,
                         int B, int H, int H_kv, int T, int D, float scale, void* stream);

/*
 * General form: grouped-query attention (H_kv as for attn_fwd_gqa) and a sliding window. With window >= 0,
 * query i sees keys i - window .. i only: itself and the `window` keys before it, flash_attn's
 * window_size = (window, 0) next to causal (apidog "Train your own ChatGPT", section 5 "Flash Attention
 * integration": flash_attn_func takes window_size; section 1 "GPT model": layers alternate short and long
 * windows, "SSSL"; the pages give no length). window = -1: no window (plain causal). KV tiles wholly left
 * of a query tile's window, and query tiles wholly past a key tile's window, are skipped. The forward's lse
 * is the log-sum-exp over the window. window < -1: ATTN_ERR_INVALID_ARG. Same shapes and contract otherwise.
 */
attn_status attn_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int H_kv,
                        int T, int D, float scale, int window, void* stream);
attn_status attn_bwd_ex(const void* q, const void* k, const void* v, const void* o, const float* lse,
                        const void* dO, void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes,
                        int B, int H, int H_kv, int T, int D, float scale, int window, void* stream);

/*
 * Attention of Tq new queries against a key/value cache: the inference engine's cached decode
 * (apidog "Train your own ChatGPT", section 6 "Inference engine": flash_attn_with_kvcache over a prefilled
 * prompt cache). Forward only.
 *   q            in : bf16 [B, Tq, H, D]
 *   k_cache      in : bf16 [B, Tk, H_kv, D];  v_cache in : bf16 [B, Tk, H_kv, D]  (H_kv divides H, grouped as
 *                     in attn_fwd_gqa)
 *   cache_seqlens in: device int32 [B], valid keys of each sequence, the new tokens' keys included (the
 *                     caller writes them into the cache first); values outside [0, Tk] are clamped
 *   o           out : bf16 [B, Tq, H, D];  lse out : fp32 [B, H, Tq] (natural log)
 *   workspace scratch: attn_decode_workspace_bytes(B, H, H_kv, Tq, Tk, D) bytes, 16-byte aligned
 * Query i of sequence b sits at position L_b - Tq + i and sees keys 0 .. L_b - Tq + i; a query that sees no
 * key gets o = 0, lse = -inf. (H / H_kv) * Tq must be <= 32 and D = 128 (else ATTN_ERR_UNSUPPORTED).
 * Launches one or two kernels (per cache chunk, then, when the cache is split into several chunks per (sequence,
 * head), the merge of the chunks; attn_decode_kernels tells which). Calls sharing a workspace must not overlap
 * in time on the GPU.
 */
size_t attn_decode_workspace_bytes(int B, int H, int H_kv, int Tq, int Tk, int D);
/*
 * Kernels one attn_decode_ex call with these sizes and window launches: 1 when each (sequence, key/value head)
 * is one chunk of the cache, 2 when the chunks are merged by a second kernel. 0 for arguments attn_decode_ex
 * rejects (sizes, D, the row limit, window < -1). Host-only; no CUDA call.
 */
int attn_decode_kernels(int B, int H, int H_kv, int Tq, int Tk, int D, int window);
attn_status attn_decode(const void* q, const void* k_cache, const void* v_cache, const int* cache_seqlens, void* o,
                        float* lse, void* workspace, size_t workspace_bytes, int B, int H, int H_kv, int Tq, int Tk,
                        int D, float scale, void* stream);

/*
 * attn_decode with a sliding window, for the model's short-window layers (apidog "Train your own ChatGPT",
 * section 1 "GPT model": layers alternate short and long windows, "SSSL"; section 6 "Inference engine": the
 * engine decodes every layer through the same cached call). With window >= 0 the query at position
 * p = L_b - Tq + i sees keys p - window .. p only, the band of attn_fwd_ex aligned to the end of the cache;
 * window = -1 is attn_decode. Chunks of the cache wholly outside every row's band are not read. The
 * workspace is attn_decode_workspace_bytes(B, H, H_kv, Tq, Tk, D) bytes, enough for any window.
 * window < -1: ATTN_ERR_INVALID_ARG. Otherwise the contract of attn_decode.
 */
attn_status attn_decode_ex(const void* q, const void* k_cache, const void* v_cache, const int* cache_seqlens,
                           void* o, float* lse, void* workspace, size_t workspace_bytes, int B, int H, int H_kv,
                           int Tq, int Tk, int D, float scale, int window, void* stream);

/*
 * Backward without caller-provided workspace, for callers that cannot allocate device memory (a custom-op or
 * plugin interface that passes tensors but no allocator or workspace; a fixed memory plan that forbids
 * cudaMalloc/cudaFree, and the synchronisation they can cause, during a step). The pages have no counterpart:
 * this is an addition of this library. Arguments and results are those of attn_bwd minus the workspace.
 *   - Scratch: a 32 MiB array inside the library (held by every GPU that loads it, until the process exits),
 *     enough for B * H * roundup(T, 128) <= 64512; larger sizes return ATTN_ERR_WORKSPACE and launch nothing.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 *   - The first call on each device looks the array's device address up (cudaGetSymbolAddress, with that
 *     device current); make that first call before any stream capture. The address is kept for the life of
 *     the process: after cudaDeviceReset on that device it is stale, so do not call this entry point there
 *     again in the same process.
 *   - All calls share the one array, which keeps the last call's contents; each call rewrites everything it
 *     reads from it (the dQ accumulator is zeroed first). Calls that overlap in time on the GPU (different
 *     streams, or different host threads on one device) race on the array and give wrong results.
 */
attn_status attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                             const void* dO, void* dq, void* dk, void* dv, int B, int H, int T, int D,
                             float scale, void* stream);

/*
 * QK normalisation + rotary embedding: the prologue the model applies to q and k before attention
 * (apidog "Train your own ChatGPT", section 1 "GPT model", architecture features: rotary embeddings for
 * relative positions without learned position embeddings, QK normalisation for stability). The pages give no
 * formula; this library's reading, per head vector x of D = 128 dims at time t of sequence b:
 *   y = x / sqrt(mean(x^2) + eps)                       RMS normalisation, no learnable weight
 *   (a, b) -> (a cos w - b sin w, a sin w + b cos w)    rotation of each pair (RoFormer, Su et al. 2021)
 *   w = p * rope_base^(-2i/D),  p = pos_offsets[b] + t  (p = t when pos_offsets is NULL)
 * Pair i is (2i, 2i+1) for ATTN_ROPE_INTERLEAVED (the paper's form) or (i, i + D/2) for ATTN_ROPE_HALF.
 *   q      in : bf16 [B, T, H, D];     k     in : bf16 [B, T, H_kv, D]
 *   q_out out : bf16 [B, T, H, D];     k_out out : bf16 [B, T, H_kv, D]
 *               q_out may be q itself and k_out may be k itself (in place); no other overlap
 *   pos_offsets in : device int32 [B] or NULL (decode: the cache length before the new tokens)
 *   rope_base finite and > 0 (usually 10000); eps finite and >= 0; D = 128 (else ATTN_ERR_UNSUPPORTED).
 *   With eps = 0 an all-zero row has no direction and its output is NaN (the formula's 0/0); eps > 0 maps it to 0.
 * One kernel launch over the rows of both tensors. On ATTN_ERR_CUDA, attn_last_cuda_error() describes the
 * failure.
 */
typedef enum { ATTN_ROPE_INTERLEAVED = 0, ATTN_ROPE_HALF = 1 } attn_rope_pairing;

attn_status attn_qk_norm_rope(const void* q, const void* k, void* q_out, void* k_out, const int* pos_offsets, int B,
                              int T, int H, int H_kv, int D, float rope_base, float eps, int pairing, void* stream);

/*
 * Backward of attn_qk_norm_rope: from q, k (its inputs) and dq_out, dk_out (the gradients of its outputs,
 * e.g. attn_bwd's dq, dk), the gradients dq, dk of its inputs. Chain rule, per row, with r = (mean(x^2) +
 * eps)^(-1/2) and y = x r: g = dy turned back by -w, dx = r (g - y mean(g y)).
 *   dq may be dq_out itself and dk may be dk_out itself (in place); no other overlap of an output.
 * Same arguments, layouts and errors as attn_qk_norm_rope otherwise. One kernel launch.
 */
attn_status attn_qk_norm_rope_bwd(const void* q, const void* k, const void* dq_out, const void* dk_out, void* dq,
                                  void* dk, const int* pos_offsets, int B, int T, int H, int H_kv, int D,
                                  float rope_base, float eps, int pairing, void* stream);

/*
 * Device-side error word of the kernels of this library on the current device since the last clear: 0, or the
 * OR of (site << 8) | kind over what went wrong, kind 1 = a kernel gave up on a bounded wait, kind 2 = (debug
 * build only) a kernel's address check failed and the access was skipped; the site bits name the wait or the
 * check (diagnostic only). Synchronises the device. Returns ATTN_ERR_TIMEOUT if kind 1 is set, else
 * ATTN_ERR_BOUNDS if the word is non-zero, ATTN_OK if it is zero, ATTN_ERR_CUDA on a CUDA error.
 */
attn_status attn_get_device_error(uint32_t* word);

/* Clear the device-side error word of the current device (synchronous). */
attn_status attn_clear_device_error(void);

/*
 * Upper bound, in nanoseconds of GPU global time, on any single wait inside the kernels (default 1e9).
 * A wait that runs out ends its kernel early with the error word set, instead of hanging the GPU.
 * Values below 1000 are rejected with ATTN_ERR_INVALID_ARG.
 */
attn_status attn_set_wait_limit_ns(uint64_t limit_ns);

/*
 * Self-test of the bounded-wait path: launches one CTA that waits on a barrier nothing ever completes,
 * with a limit of `limit_ns`; the kernel gives up, records its site (0x7f) in the error word and returns.
 * Used by the failure-detection test; never part of the attention path.
 */
attn_status attn_selftest_wait_timeout(uint64_t limit_ns, void* stream);

/*
 * Debug build. libattn_debug.so is this library compiled with -DATTN_DEBUG: every kernel access through a plain
 * address (the ones no TMA tensor map bounds: LSE/Delta rows, dQ accumulator reductions and conversion, the
 * forward's LSE, the decode kernels' cache, partial and output rows, the prologue's rows) is first checked
 * against the extent of its array; a failed check sets kind 2 in the device error word and skips the access.
 * Same symbols, same results, slower. attn_is_debug_build() returns 1 in it, 0 in libattn.so.
 * attn_selftest_bounds_check() launches one checked store past its array's declared extent (debug build: the
 * check records site 0x7e and skips the store); in the release build it returns ATTN_ERR_UNSUPPORTED.
 */
int attn_is_debug_build(void);
attn_status attn_selftest_bounds_check(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_H_ */
