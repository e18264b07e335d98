/*
 * fa.h -- C ABI of the exact, fused attention library (libfa.so): the forward
 * (square, grouped heads, split-KV decoding, e4m3 inputs) and its backward.
 *
 * The operation is the attention of "FlashAttention (UR)", section "Problem
 * of standard attention":
 *
 *     O = softmax(scale * Q K^T + mask) V,      lse_i = ln sum_j exp(s_ij)
 *
 * with s_ij = scale * <q_i, k_j> + mask_ij and mask_ij = -inf for hidden keys
 * (masking sits between Q K^T and the softmax in the fused chain of section
 * "Fusing operations into one CUDA kernel"). It is evaluated tile by tile
 * with an online softmax (section "Online softmax") so the N x N score matrix
 * never reaches device memory, and the per-row log-sum-exp is emitted as the
 * O(N) statistic (section "Complexity and optimality").
 *
 * Conventions shared by every entry point:
 *   - Pointers are DEVICE pointers owned by the caller. The library allocates
 *     no device memory per call and keeps no reference after it returns.
 *   - Layout: q, k, v, o are bf16 [B, H, N, d], contiguous, d innermost
 *     (row (b,h,i) starts at element ((b*H + h)*N + i)*d). lse is fp32
 *     [B, H, N], natural log, scale included.
 *   - q, k, v, o must be 16-byte aligned (the tensor-memory-access engine
 *     requires it); lse 4-byte aligned. o and lse must not overlap each other
 *     or the inputs.
 *   - d must be 64, 128 or 256; anything else returns FA_ERR_UNSUPPORTED.
 *   - B, H, N >= 0. If any is 0 there is nothing to compute: the call returns
 *     FA_OK without launching (pointers may then be NULL).
 *   - scale must be finite and > 0; causal must be 0 or 1.
 *   - Causal masking is square: query row i sees key j iff j <= i.
 *   - A row with no visible key gets O = 0 and lse = -inf.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream). Calls are
 *     asynchronous: they return once the kernel is enqueued. q, k, v are only
 *     read; every element of o and lse is written.
 *   - Argument errors are reported synchronously and launch nothing.
 *   - Results are deterministic: identical inputs give bitwise identical
 *     outputs on the same GPU (the method is exact and deterministic,
 *     "FlashAttention-2 (HI)", section "Performance and efficiency").
 *   - Requires a B200-class GPU (compute capability 10.0, sm_100a); other
 *     devices get FA_ERR_UNSUPPORTED. There is no CPU fallback.
 */
#ifndef FA_H_
#define FA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FA_OK = 0,
    FA_ERR_INVALID_ARG = 1,  /* null/misaligned/overlapping pointer, bad size, scale, causal */
    FA_ERR_UNSUPPORTED = 2,  /* head dim other than 64/128/256, or not an sm_100 device */
    FA_ERR_LAUNCH = 3,       /* the CUDA runtime refused the launch or a sync failed */
    FA_ERR_TIMEOUT = 4       /* a kernel's bounded wait ran out (see fa_last_device_error) */
} fa_status_t;

/*
 * Exact attention forward, optional causal mask.
 * q, k, v: bf16 [B,H,N,d] in; o: bf16 [B,H,N,d] out; lse: fp32 [B,H,N] out.
 * Returns an fa_status_t value.
 */
int fa_fwd(const void *q, const void *k, const void *v, void *o, float *lse,
           int B, int H, int N, int d, float scale, int causal, void *stream);

/*
 * Same, plus a per-sequence key-padding mask: keys j >= kv_len[b] are hidden
 * from every query row of batch b (query rows past kv_len[b] are still
 * computed against the visible keys). kv_len: device int32 [B], or NULL for
 * "all N keys visible". Values are clamped to [0, N]; 0 hides every key.
 * The pages name masking inside the fused kernel but no mask interface; a
 * valid length per sequence is the plainest form that keeps an N x N mask
 * out of device memory.
 */
int fa_fwd_kvlen(const void *q, const void *k, const void *v, void *o, float *lse,
                 int B, int H, int N, int d, float scale, int causal,
                 const int32_t *kv_len, void *stream);

/*
 * Grouped- and multi-query attention (the FlashAttention-2 extension to
 * multi-query attention, "FlashAttention (UR)", section "FlashAttention-2
 * (2023)"): q, o are bf16 [B, H, N, d] and lse fp32 [B, H, N] as above, but
 * k, v are bf16 [B, H_kv, N, d] with H a multiple of H_kv; query head h
 * attends with K/V head h / (H / H_kv). H_kv == H is fa_fwd_kvlen; H_kv == 1
 * is multi-query attention. kv_len as in fa_fwd_kvlen (nullable). H_kv < 1,
 * H_kv > H or H % H_kv != 0 returns FA_ERR_INVALID_ARG.
 */
int fa_fwd_gqa(const void *q, const void *k, const void *v, void *o, float *lse,
               int B, int H, int H_kv, int N, int d, float scale, int causal,
               const int32_t *kv_len, void *stream);

/* Largest num_splits fa_fwd_splitkv accepts. */
#define FA_MAX_SPLITS 128

/*
 * Split-KV forward for few queries against many keys (decoding with a key-value
 * cache; the specialised inference kernels of "FlashAttention (UR)", section
 * "Specialised solutions"). The result is the same attention as above:
 *   q, o: bf16 [B, H, Nq, d]; lse: fp32 [B, H, Nq];
 *   k, v: bf16 [B, H_kv, Nk, d], H a multiple of H_kv (grouped heads as in
 *   fa_fwd_gqa); 0 <= Nq <= Nk.
 * Query row i stands at key position i + Nk - Nq: with causal = 1 it sees keys
 * j <= i + Nk - Nq (Nq == Nk is the square mask of fa_fwd). kv_len (nullable)
 * hides keys j >= kv_len[b] as in fa_fwd_kvlen; the causal offset stays
 * Nk - Nq.
 * Each row's keys are cut into num_splits contiguous ranges of whole 128-key
 * tiles, handled by different CTAs; each range's normalised output and
 * log-sum-exp go to `workspace`, and a second kernel merges them by
 * lse-weighted rescaling (the online-softmax update of section "Online
 * softmax", applied once per range). The query heads that share a K/V head
 * are processed together, so each K/V tile is read once per group.
 *   num_splits: 1..FA_MAX_SPLITS (1: no workspace, one kernel; more splits
 *     than key tiles leave some ranges empty, which is allowed).
 *   workspace: device memory owned by the caller, 16-byte aligned, at least
 *     fa_splitkv_workspace_bytes(B, H, Nq, d, num_splits) bytes, not
 *     overlapping any other argument; may be NULL when num_splits == 1. Its
 *     contents need no initialisation and are scratch after the call returns;
 *     two calls in flight at once must not share it.
 * Errors as in fa_fwd; additionally Nq > Nk, num_splits out of range or a
 * missing/short/misaligned workspace return FA_ERR_INVALID_ARG.
 */
int fa_fwd_splitkv(const void *q, const void *k, const void *v, void *o, float *lse,
                   int B, int H, int H_kv, int Nq, int Nk, int d, float scale,
                   int causal, const int32_t *kv_len, int num_splits,
                   void *workspace, size_t workspace_bytes, void *stream);

/*
 * Bytes of workspace fa_fwd_splitkv needs: 0 for num_splits == 1, else
 * num_splits * B * H * Nq * (d + 1) * 4 rounded up to 256 bytes in the middle.
 * Returns 0 for invalid arguments. Host-only, no device call.
 */
size_t fa_splitkv_workspace_bytes(int B, int H, int Nq, int d, int num_splits);

/*
 * A num_splits for fa_fwd_splitkv on the current device: the most key ranges
 * that keep the work units (one per head group, row block and range) within
 * one wave, units <= the device's SM count, or <= 128 for the decoding tile
 * (bf16, d = 128, at most 8 query heads x rows per K/V head), which measured
 * fastest there; each range at least four 128-key tiles long and at most
 * FA_MAX_SPLITS; 1 when there are at least that many units without splitting
 * (every unit pays a fixed cost, and a second wave leaves most SMs idle for its
 * last part). Returns 1 for invalid arguments. Reads only device attributes.
 */
int fa_splitkv_default_splits(int B, int H, int H_kv, int Nq, int Nk, int d);

/*
 * FP8 forward: q, k, v hold e4m3 codes (OCP 8-bit float: 1 sign, 4 exponent
 * bits with bias 7, 3 mantissa bits, largest finite 448), one byte each, laid
 * out like the bf16 tensors of fa_fwd_gqa ([B, H, N, d] and [B, H_kv, N, d]);
 * q_descale, k_descale, v_descale (finite, > 0) give the tensors' values as
 * descale * code. The result is the attention of those dequantized tensors,
 * O bf16 [B, H, N, d] and lse fp32 [B, H, N] as in fa_fwd. This is the
 * lower-precision-input direction of FlashAttention-3 ("FlashAttention (UR)",
 * section "FlashAttention-3"): both tile products run on the tensor cores in
 * e4m3 with fp32 accumulation, and the probabilities P are rounded to e4m3
 * (relative error up to 2^-4) before the P.V product, so O carries that
 * error; lse does not (scores are exact products of e4m3 values). d is 64,
 * 128 or 256; causal, kv_len, H_kv, errors as in fa_fwd_gqa.
 */
int fa_fwd_fp8(const void *q, const void *k, const void *v, float q_descale, float k_descale,
               float v_descale, void *o, float *lse, int B, int H, int H_kv, int N, int d,
               float scale, int causal, const int32_t *kv_len, void *stream);

/*
 * FP8 split-KV forward: fa_fwd_splitkv with e4m3 q [B, H, Nq, d] and k, v
 * [B, H_kv, Nk, d] and their descales as in fa_fwd_fp8 (same precision
 * statement). O bf16 [B, H, Nq, d], lse fp32 [B, H, Nq]; the partials in
 * `workspace` are fp32, sized by fa_splitkv_workspace_bytes as for bf16
 * inputs. d is 64, 128 or 256; every other argument and error as in
 * fa_fwd_splitkv.
 */
int fa_fwd_splitkv_fp8(const void *q, const void *k, const void *v, float q_descale,
                       float k_descale, float v_descale, void *o, float *lse, int B, int H,
                       int H_kv, int Nq, int Nk, int d, float scale, int causal,
                       const int32_t *kv_len, int num_splits, void *workspace,
                       size_t workspace_bytes, void *stream);

/*
 * Backward pass: gradients of the attention of fa_fwd / fa_fwd_gqa for a
 * scalar loss, given dO = dL/dO. The pages report the training speed-ups of
 * the method ("FlashAttention (UR)", section "Experimental results") but state
 * no backward algorithm; this is the exact gradient of the forward definition
 * (chain rule through the row softmax), with P recomputed tile by tile from Q,
 * K and the forward's lse (the O(N) statistic of section "Complexity and
 * optimality"), never stored:
 *   dV = P^T dO,  dS = P * (dO V^T - D),  D_i = dO_i . O_i,
 *   dQ = scale dS K,  dK = scale dS^T Q.
 *   q, o, d_o: bf16 [B, H, N, d]; k, v: bf16 [B, H_kv, N, d] (as fa_fwd_gqa);
 *   lse: fp32 [B, H, N], the forward's (natural log, scale included);
 *   dq: bf16 [B, H, N, d] out; dk, dv: bf16 [B, H_kv, N, d] out (a shared K/V
 *   head gets the sum over its group of query heads);
 *   causal, kv_len, scale: as in the forward call that produced o and lse.
 *   d must be 64 or 128 (FA_ERR_UNSUPPORTED otherwise).
 *   workspace: device memory owned by the caller, 16-byte aligned, at least
 *   fa_bwd_workspace_bytes(B, H, N) bytes, overlapping no other argument; no
 *   initialisation needed; scratch after the call.
 * All outputs are fully written; they must not overlap each other, the inputs
 * or the workspace. Deterministic (no atomics). Errors as in fa_fwd.
 */
int fa_bwd(const void *q, const void *k, const void *v, const void *o, const float *lse,
           const void *d_o, void *dq, void *dk, void *dv, int B, int H, int H_kv, int N,
           int d, float scale, int causal, const int32_t *kv_len, void *workspace,
           size_t workspace_bytes, void *stream);

/* Workspace bytes of fa_bwd: 2 * B * H * ceil(N / 128) * 128 * 4 (0 if invalid). */
size_t fa_bwd_workspace_bytes(int B, int H, int N);

/* Bytes of split-KV scratch the library itself holds on each device. */
#define FA_STATIC_SCRATCH_BYTES (16u << 20)

/*
 * fa_fwd_splitkv without a workspace argument, for callers that cannot
 * allocate device memory at call time: for instance a serving loop that hands
 * all free device memory to a key/value cache pool up front, or a C caller
 * with no device allocator of its own. The partial results go to a scratch
 * array of FA_STATIC_SCRATCH_BYTES (16 MiB) that the library's CUDA module
 * reserves on each device when it is loaded; the call itself allocates
 * nothing. The pages have no counterpart: this is an interface variant of the
 * split-KV forward above, with the same arguments, results and errors apart
 * from the workspace.
 *   - The first call on a device (with that device current) looks up the
 *     scratch's address and prepares the kernels; make it once before any
 *     stream capture or latency-critical section.
 *   - If fa_splitkv_workspace_bytes(B, H, Nq, d, num_splits) exceeds
 *     FA_STATIC_SCRATCH_BYTES the call returns FA_ERR_INVALID_ARG before any
 *     CUDA call; use fewer splits or fa_fwd_splitkv with your own workspace.
 *   - One scratch per device: calls that overlap on the GPU (on different
 *     streams, or from several host threads without ordering) race on it and
 *     give wrong results. Calls on one stream are ordered and safe.
 *   - Nothing in the scratch has to start at zero: every partial is written
 *     before the merge reads it.
 */
int fa_fwd_splitkv_static(const void *q, const void *k, const void *v, void *o, float *lse,
                          int B, int H, int H_kv, int Nq, int Nk, int d, float scale,
                          int causal, const int32_t *kv_len, int num_splits, void *stream);

/* Static, human-readable name of a status code (never NULL). */
const char *fa_status_string(int status);

/*
 * Synchronises `stream`, then reads and clears the current device's status
 * word, which kernels set when a bounded wait runs out (FA_ERR_TIMEOUT). The
 * word is sticky: while it is set, later launches on that device skip their
 * work, so call this after any call whose results matter. Returns FA_OK,
 * FA_ERR_TIMEOUT, or FA_ERR_LAUNCH if the synchronisation itself failed.
 */
int fa_last_device_error(void *stream);

/*
 * Diagnostic for the kernels' failure detection (the pages have no
 * counterpart: it checks this library's bounded waits). Launches one CTA on
 * `stream` whose thread waits, with the same bounded-wait routine the
 * attention kernel uses, on a shared-memory barrier that nothing completes.
 * After limit_ns nanoseconds the wait gives up, the kernel sets the timeout
 * bit of the device status word and returns; fa_last_device_error(stream)
 * then reports FA_ERR_TIMEOUT (and clears the word). limit_ns must be in
 * [1000, 5e9], else FA_ERR_INVALID_ARG. While the word is set, attention
 * launches on the device skip their work, so read it before the next call.
 */
int fa_watchdog_selftest(uint64_t limit_ns, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* FA_H_ */
