/*
 * lrkv.h -- C ABI of liblrkv.so: low-rank compressed-KV decode attention
 * on NVIDIA B200 (sm_100a).
 *
 * What the library computes (one transformer layer per call):
 *
 *   Write path -- OjaKV repository README, "Method Summary > StaticPCA"
 *   (a fixed offline per-head basis) and "Method Summary > OjaKV" (hybrid
 *   storage: tokens with a high reconstruction error stay in full rank, the
 *   rest are compressed).  For every new token t of kv head h:
 *       c_k = U_k[h]^T k_t,  c_v = U_v[h]^T v_t             (fp32 accumulate)
 *       e_k = ||k_t - U_k c_k|| / ||k_t||,  e_v likewise,  e_t = max(e_k, e_v)
 *       the coefficients are stored as bf16 (round to nearest even) at the
 *       token's position; if e_t > tau the token is also appended, in
 *       ascending position order, to the full-rank list (its k and v rows
 *       copied) and its route-mask bit is set.
 *
 *   Read path -- decode attention directly over the compressed cache, the
 *   coefficient-space form of "reconstruct on the fly, then attend":
 *       q~_h = U_k^T q_h
 *       s_t  = q~_h . c_k,t / sqrt(d)   (t compressed)
 *       s_t  = q_h  . k_t   / sqrt(d)   (t full rank)
 *       p    = softmax over all tokens of the sequence, both sets together
 *       o_h  = U_v sum_{t compressed} p_t c_v,t + sum_{t full} p_t v_t
 *   Query head h reads kv head floor(h / g), g = Hq / Hkv (grouped-query).
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers, caller-allocated and
 *     caller-owned; the library never allocates, frees or synchronises.
 *     All work is enqueued on the given stream (a cudaStream_t passed as
 *     void*; NULL is the legacy default stream).
 *   - bf16 values are raw bfloat16 bit patterns (uint16_t), row-major,
 *     densely packed in the shapes given below.
 *   - Every pointer must be 16-byte aligned.
 *   - Synchronous errors (returned, nothing launched): null pointers, d != 128,
 *     r_k or r_v not a multiple of 16 or outside [16, d], Hq % Hkv != 0,
 *     T_cap not a positive multiple of 32, F_cap < 0, workspace too small,
 *     misaligned pointers, a launch failure (LRKV_ERR_CUDA).
 *   - Asynchronous conditions are OR-ed into *dev_status (device word),
 *     read by the caller after synchronising; kernels never trap.
 *   - A sequence with no tokens attends to nothing: its output rows are 0.
 *   - Non-finite inputs give undefined (but memory-safe) results.
 *   - Two calls that share a cache or a workspace must not overlap in time
 *     (issue them on one stream, or order them with events).
 */
#ifndef LRKV_H
#define LRKV_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LRKV_API __attribute__((visibility("default")))
#else
#define LRKV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t lrkv_bf16; /* raw bfloat16 bits */

typedef enum {
  LRKV_OK = 0,
  LRKV_ERR_INVALID_ARG = 1, /* null pointer, bad size, workspace too small */
  LRKV_ERR_UNSUPPORTED = 2, /* a shape this build does not handle (d != 128, ...) */
  LRKV_ERR_ALIGNMENT = 3,   /* a pointer not 16-byte aligned */
  LRKV_ERR_CUDA = 4         /* a CUDA launch failed; cudaGetLastError() was cleared */
} lrkv_status;

/* Bits OR-ed into *dev_status by the kernels. */
#define LRKV_DEV_FULL_OVERFLOW 0x1u /* a routed token found the full-rank list full: it was
                                       kept compressed (mask bit clear) instead */
#define LRKV_DEV_SEQ_OVERFLOW 0x2u  /* seq_len + new tokens exceeded T_cap: the tokens past
                                       T_cap were dropped */
#define LRKV_DEV_BAD_COUNT 0x4u     /* a t_new_b entry outside [0, t_new]: clamped into it */
#define LRKV_DEV_WAIT_TIMEOUT 0x8u  /* a kernel gave up waiting for its own copies (bounded
                                       wait): its outputs for that call are not valid.
                                       The environment variable LRKV_MAIN_WAIT_ITERS
                                       (a positive integer, read by each prefill-sized
                                       lrkv_compress) lowers the limit of the prefill
                                       projection's wait for each input tile, so a test
                                       can make it run out; the waits that drain copies
                                       and MMAs in flight keep their full limit. */

/* Problem sizes of one layer. */
typedef struct {
  int32_t B;     /* batch rows (sequences) */
  int32_t Hq;    /* query heads */
  int32_t Hkv;   /* kv heads; Hq % Hkv == 0 */
  int32_t d;     /* head dimension; 128 in this build */
  int32_t r_k;   /* key rank, multiple of 16 in [16, d] */
  int32_t r_v;   /* value rank, multiple of 16 in [16, d] */
  int32_t T_cap; /* positions per sequence the cache can hold, multiple of 32 */
  int32_t F_cap; /* full-rank rows per (sequence, kv head) the list can hold, >= 0 */
  int32_t coef_bits; /* stored coefficient format: 0 or 16 = bf16; 8 = int8 codes;
                        4 = int4 codes (see "Quantised coefficients" below) */
} lrkv_dims;

/* Quantised coefficients (coef_bits 8 or 4).  KVQuant record ("Quant method":
 * sub-8-bit codes with a per-vector scale) and NOVA-KV summary (fixed-width
 * codes read inside attention), applied to this cache's coefficient rows: each
 * stored row (c_k or c_v of one token and kv head) is quantised on its own,
 * symmetric and absmax-scaled, from its bf16 value c (round to nearest even):
 *     Q = 127 (8 bits) or 7 (4 bits)
 *     s = max_j |c_j| / Q                     (fp32 division, correctly rounded)
 *     q_j = round_half_even(c_j / s)          (fp32 division), clamped to [-Q, Q]
 *     s = 0 (an all-zero row) gives q = 0;    c_hat_j = s q_j
 * with no flush of subnormals, so any implementation of these IEEE steps takes
 * the same decisions.  Codes are two's complement; 4-bit codes are packed two
 * per byte, element 2i in the low nibble.  The decode reads c_hat: compressed
 * logits s_k,t (q~ . q_k,t) / sqrt(d), value weights p_t s_v,t.  The routing
 * error is still that of the unrounded projection. */

/* One layer of compressed cache.  Every pointer is a device pointer. */
typedef struct {
  const lrkv_bf16* U_k; /* [Hkv][d][r_k] key basis (orthonormal columns, rounded to bf16) */
  const lrkv_bf16* U_v; /* [Hkv][d][r_v] value basis */
  void* coef_k;         /* [B][Hkv][T_cap][r_k] key coefficients, indexed by position: bf16,
                           or [B][Hkv][T_cap][r_k * coef_bits / 8] bytes of codes */
  void* coef_v;         /* [B][Hkv][T_cap][r_v] value coefficients, likewise */
  uint32_t* route_mask; /* [B][Hkv][T_cap/32]; bit p%32 of word p/32 = position p is full rank */
  int32_t* full_idx;    /* [B][Hkv][F_cap] positions of the full-rank rows, ascending */
  lrkv_bf16* full_k;    /* [B][Hkv][F_cap][d] key rows of full-rank tokens */
  lrkv_bf16* full_v;    /* [B][Hkv][F_cap][d] value rows of full-rank tokens */
  int32_t* full_cnt;    /* [B][Hkv] rows in use in the full-rank list */
  int32_t* seq_len;     /* [B] tokens already in the cache (positions 0..seq_len-1) */
  uint32_t* dev_status; /* 1 word, LRKV_DEV_* bits */
  /* Attention-aware key basis (NOVA-KV summary, "Methodology > Key Transform
     Derivation", Theorem 1: the optimal rank-p key transform R = M_q^{1/2} E_p,
     non-orthogonal, with the query side projected by M_q^{-1/2} E_p).  Both
     null: the plain StaticPCA cache described above.  When given:
       c_k   = U_k^T (k - mu_k)                 U_k: the key-side basis R
       k_hat = mu_k + U_kq c_k                  U_kq: the query-side basis
       e_k   = ||k - k_hat|| / ||k||
       q~    = U_kq^T q,  compressed logit (q . mu_k + q~ . c_k) / sqrt(d).
     Either may be null on its own (U_kq = U_k, or mu_k = 0).  Values are not
     transformed.  A cache must keep the same choice for all its calls. */
  const lrkv_bf16* U_kq; /* nullable [Hkv][d][r_k] query-side / key reconstruction basis */
  const float* mu_k;     /* nullable [Hkv][d] fp32 key mean */
  float* scale_k;        /* [B][Hkv][T_cap] fp32 per-row scales of quantised key codes
                            (coef_bits 8 or 4; unused, may be null, for bf16) */
  float* scale_v;        /* [B][Hkv][T_cap] likewise for the value codes */
} lrkv_cache;
/* A new cache is all zeros (seq_len = full_cnt = 0).  The library writes every
   mask bit, coefficient row and list entry it covers, so stale contents past
   seq_len / full_cnt are harmless. */

/* Stream ordering.  lrkv_compress's decode-time append and lrkv_decode_attn
   launch with programmatic dependent launch: their kernels may begin on the
   GPU while the preceding kernel of the stream is finishing.  Before waiting
   for it they read only the bases (U_k, U_v, U_kq) and mu_k, so the kernel
   issued just before a call must not write them.  Every other input (q, k_new,
   v_new and all cache state) is read after the preceding kernel completed. */

/* Bytes of device workspace that lrkv_compress and lrkv_decode_attn need for
   these sizes (0 for invalid sizes).  The decode part depends on the current
   device's number of SMs (the split-K grid is sized for it; 148 is assumed
   when no device is visible): query it with the device current on which the
   calls will run.  The workspace must be zero-filled once after allocation;
   the kernels leave it zeroed where it needs to be, so it can be reused by any
   later call with the same dims.  One workspace serves one stream of calls:
   concurrent calls need their own. */
LRKV_API size_t lrkv_workspace_size(const lrkv_dims* dims);

/* Append new tokens to every sequence of the cache (prefill or a decode step).
 *
 * k_new, v_new: [B][t_new][Hkv][d] bf16, the new key and value rows.  Row b
 *   contributes its first n_b tokens: n_b = t_new_b[b] when t_new_b (device
 *   [B] int32, nullable) is given, else t_new (ragged prefill passes padded
 *   rows plus t_new_b).  They go to positions seq_len[b] .. seq_len[b]+n_b-1;
 *   seq_len[b] is advanced on the device.  Positions at or past T_cap are
 *   dropped (LRKV_DEV_SEQ_OVERFLOW).
 * tau: routing threshold on the relative reconstruction error (strict >).
 * err_out: nullable device [B][Hkv][t_new] fp32; receives e_t for every token
 *   written (entries of dropped or padding tokens are left untouched).
 * ws: workspace of at least lrkv_workspace_size(dims) bytes (ws_bytes).
 * Returns LRKV_OK when the work was enqueued.
 */
LRKV_API lrkv_status lrkv_compress(const lrkv_dims* dims, const lrkv_cache* cache,
                                   const lrkv_bf16* k_new, const lrkv_bf16* v_new,
                                   int32_t t_new, const int32_t* t_new_b, float tau,
                                   float* err_out, void* ws, size_t ws_bytes, void* stream);

/* Single-token decode attention for every query head of every sequence.
 *
 * q:   [B][Hq][d] bf16, one query per head.
 * out: [B][Hq][d] fp32, the attention output (0 for an empty sequence).
 * Attends to positions 0..seq_len[b]-1 as the cache holds them on the
 * device when the kernel runs (so an append issued earlier on the same
 * stream is included).  The split-K grid is sized for a full cache (T_cap
 * positions); each sequence's splits are cut from its live length on the
 * device, so a cache allocated far larger than it holds costs no more than a
 * snug one.
 * ws: workspace of at least lrkv_workspace_size(dims) bytes (ws_bytes).
 */
LRKV_API lrkv_status lrkv_decode_attn(const lrkv_dims* dims, const lrkv_cache* cache,
                                      const lrkv_bf16* q, float* out, void* ws,
                                      size_t ws_bytes, void* stream);

/* One decode step with its append, in one launch: the same result as
 *   lrkv_compress(dims, cache, k_new, v_new, 1, t_new_b, tau, err_out, ...)
 *   lrkv_decode_attn(dims, cache, q, out, ...)
 * issued back to back on `stream` (append-then-attend: the new token is
 * attended).  k_new, v_new: [B][1][Hkv][d] bf16; t_new_b: nullable device [B]
 * int32, each 0 or 1 (a row with 0 only attends); err_out: nullable device
 * [B][Hkv][1] fp32.  The append is done inside the decode kernel by one extra
 * CTA per (batch row, kv head); the list length and seq_len are advanced on
 * the device once every CTA has read them.  With more than 4 query heads per
 * kv head (or 3) the streaming kernel runs in launches of 4 heads, the first
 * of which appends.  Rank pairs the streaming kernel has no instantiation for
 * run the two calls above instead (two launches).
 * Arguments, layouts and errors otherwise as lrkv_compress / lrkv_decode_attn.
 */
LRKV_API lrkv_status lrkv_append_decode_attn(const lrkv_dims* dims, const lrkv_cache* cache,
                                             const lrkv_bf16* k_new, const lrkv_bf16* v_new,
                                             const int32_t* t_new_b, float tau, float* err_out,
                                             const lrkv_bf16* q, float* out, void* ws,
                                             size_t ws_bytes, void* stream);

/* StaticPCA's offline basis (OjaKV repository README, "Method Summary >
 * StaticPCA": a fixed basis computed offline from calibration rows; KV-CoRE
 * page, abstract: the Frobenius-optimal low-rank approximation).  For every
 * kv head h, the top-r eigenvectors of the uncentred scatter matrix
 * G_h = sum over rows n of x_{n,h} x_{n,h}^T, computed on the GPU: G in fp32 on
 * the tensor cores (exact bf16 products), summed in fp64, cyclic Jacobi in
 * fp64 (eigenvectors in fp32).
 *
 * X:        [n_rows][Hkv][d] bf16 calibration rows (keys or values; the layout
 *           of lrkv_compress's k_new with B * t_new rows).  Only dims->Hkv and
 *           dims->d (128) are used.
 * r:        1..d columns to keep.
 * U_out:    [Hkv][d][r] bf16, unit eigenvectors by decreasing eigenvalue, each
 *           signed so that its largest-magnitude entry is positive (the lowest
 *           index on a tie), rounded to nearest even: a basis for lrkv_cache.
 * eigvals_out: nullable [Hkv][d] fp32, every eigenvalue of G_h, descending (the
 *           discarded mass of a rank-r basis is the sum past index r).
 * ws:       lrkv_fit_workspace_size(dims, n_rows) bytes (any contents).
 * Returns LRKV_OK when the work was enqueued (two kernels on `stream`, then an
 * empty one, so that a decode issued next finds the bases written).
 */
LRKV_API size_t lrkv_fit_workspace_size(const lrkv_dims* dims, int32_t n_rows);
LRKV_API lrkv_status lrkv_fit_basis(const lrkv_dims* dims, const lrkv_bf16* X, int32_t n_rows,
                                    int32_t r, lrkv_bf16* U_out, float* eigvals_out, void* ws,
                                    size_t ws_bytes, void* stream);

/* Rank by error budget for a StaticPCA basis (OjaKV repository README, the
 * calibration command's `--error_budget`; KV-CoRE page, abstract: the
 * Frobenius-optimal rank-r approximation).  By Eckart-Young the relative
 * squared Frobenius error of the best rank-r approximation of the calibration
 * rows is the discarded eigenvalue mass over the total; for each head the
 * call returns the smallest r in 1..d with
 *     sum_{j >= r} max(lambda_j, 0) <= budget * sum_j max(lambda_j, 0),
 * sums in fp64 taken from the smallest eigenvalue up (j = d-1 first).
 * Negative eigenvalues (rounding of a positive semi-definite matrix) count as
 * zero; a head whose eigenvalues are all zero gets r = 1.
 *
 * Host call: no GPU work, nothing is enqueued.
 * eigvals: HOST [n_heads][d] fp32, each row descending (lrkv_fit_basis's
 *          eigvals_out, copied to the host).
 * d:       eigenvalues per head, 1..4096.
 * budget:  0 <= budget <= 1 (not NaN); 0 keeps every direction with mass.
 * r_out:   HOST [n_heads] int32.
 * Returns LRKV_ERR_INVALID_ARG for null pointers, n_heads < 1, d out of range
 * or a budget outside [0, 1]; r_out is then untouched.
 */
LRKV_API lrkv_status lrkv_rank_for_budget(const float* eigvals, int32_t n_heads, int32_t d,
                                          double budget, int32_t* r_out);

/* Online basis update (OjaKV repository README, "Method Summary > OjaKV": the
 * low-rank subspace is updated online with Oja's algorithm during prefill and
 * decoding).  The page gives no rule, step size or normalisation; this is
 * Oja's subspace rule for every kv head h, over a batch of N = n_rows rows x_n
 * (a prefill chunk; N = 1 per decode step):
 *     y_n = U^T x_n,   V = U + eta (1/N) sum_n (x_n - U y_n) y_n^T,
 *     U <- Q of V = Q R with R's diagonal positive (columns kept orthonormal).
 * The sums are taken in fp32, the step and the orthonormalisation (Gram-
 * Schmidt with a second pass) in fp64.
 *
 * X:     [n_rows][Hkv][d] bf16 rows (keys or values: lrkv_compress's k_new
 *        layout with B * t_new rows).  Only dims->Hkv and dims->d (128) are used.
 * r:     columns of the basis, a multiple of 16 in [16, d].
 * eta:   step size, >= 0 and finite.
 * U:     [Hkv][d][r] fp32, the basis, updated in place.  Kept in fp32 so that
 *        small steps accumulate (a bf16 basis would round most of them away).
 * U_out: nullable [Hkv][d][r] bf16, the updated basis rounded to nearest even:
 *        what lrkv_cache takes as U_k or U_v.
 * ws:    lrkv_oja_workspace_size(dims, n_rows, r) bytes (any contents).
 * A cache keeps one basis per kv head: after an update, compressed rows stored
 * earlier are read with the new basis (the library does not rewrite them).
 * Returns LRKV_OK when the work was enqueued (two kernels on `stream`, then an
 * empty one, so that a decode issued next, which reads the bases before
 * waiting on the preceding kernel, finds them written). */
LRKV_API size_t lrkv_oja_workspace_size(const lrkv_dims* dims, int32_t n_rows, int32_t r);
LRKV_API lrkv_status lrkv_oja_update(const lrkv_dims* dims, const lrkv_bf16* X, int32_t n_rows,
                                     int32_t r, float eta, float* U, lrkv_bf16* U_out, void* ws,
                                     size_t ws_bytes, void* stream);

/* Device scratch built into the library for lrkv_decode_attn_noalloc, bytes. */
#define LRKV_NOALLOC_SCRATCH_BYTES (4u << 20)

/* lrkv_decode_attn without a workspace: the same computation and result, with
 * the split-K scratch taken from memory the library itself holds.  The paper
 * has no counterpart; this is an interface addition.
 *
 * Who it is for: callers that may not allocate device memory at decode time --
 * a plugin's enqueue hook in an inference engine that may only touch memory
 * the engine handed it when it was built, a latency-critical decode loop that
 * cannot afford cudaMalloc/cudaFree (they cost host time and can synchronise
 * the whole device), or a plain C caller with no device allocator of its own.
 *
 * The scratch is one file-scope device array of LRKV_NOALLOC_SCRATCH_BYTES.
 * It exists on every GPU that loads the library, from load until the process
 * exits.  A call needs 256-byte-rounded B*Hkv*4 bytes of tickets plus the split
 * partials (the decode part of lrkv_workspace_size for the same dims); when
 * that exceeds the maximum the call returns LRKV_ERR_UNSUPPORTED and launches
 * nothing.  The function calls no cudaMalloc, cudaFree or other allocating
 * routine; it clears the tickets with cudaMemsetAsync on `stream`, then
 * launches the decode kernel there.
 *
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress), with that device current: make that first call
 * before any stream capture starts.  The address is kept once the lookup has
 * succeeded; a failed lookup returns LRKV_ERR_CUDA and is tried again by the
 * next call.
 * All calls on one device share the array.  Calls whose executions overlap on
 * the GPU (different streams, or host threads without ordering) race on it
 * and give wrong results: order them, e.g. issue them on one stream.
 * Arguments and layouts are those of lrkv_decode_attn.  Checks, in order: the
 * sizes (as lrkv_decode_attn checks them), then the scratch limit
 * (LRKV_ERR_UNSUPPORTED, nothing else looked at), then the cache, q and out
 * pointers (as lrkv_decode_attn checks them).
 */
LRKV_API lrkv_status lrkv_decode_attn_noalloc(const lrkv_dims* dims, const lrkv_cache* cache,
                                              const lrkv_bf16* q, float* out, void* stream);

/* Static text for a status code. */
LRKV_API const char* lrkv_status_str(lrkv_status status);

#ifdef __cplusplus
}
#endif

#endif /* LRKV_H */
