/*
 * tq.h -- TurboQuant KV-cache vector quantisation on NVIDIA B200 (sm_100a): the C ABI of libtq.
 *
 * The method (web write-ups of TurboQuant, arXiv 2504.19874):
 *   Algorithm 1 (MSE): rotate a vector by a random orthogonal Pi, quantise every coordinate with a
 *     Lloyd-Max scalar codebook precomputed for the coordinate law of a rotated unit vector, and
 *     invert the rotation on decode (ai-navigate-news page, "how it works (technical)"; aiboss88
 *     page, "TurboQuant technical principles"; techblog-plum page, "step 1: PolarQuant").
 *   Algorithm 2 (inner product): Algorithm 1 at b-1 bits, then one sign bit per coordinate of
 *     S r for the residual r, with |r|; inner products estimated from the codes are unbiased
 *     (ai-navigate-news page, "how it works"; aiboss88 page, "two-stage residual correction";
 *     techblog-plum page, "step 2: QJL").
 *   Packing: indices and signs bit-packed, norms and residual norms in float16 (ai-navigate-news
 *     page, bit-packing paragraph).
 *   Attention on the compressed cache and vector search from the codes (aiboss88 page, features
 *     and applications).
 *
 * Conventions shared by every call
 *   - d (vector length) is a multiple of 32, 32 <= d <= 4096 (UNSUPPORTED otherwise; some calls
 *     have narrower limits, stated below). bits of a codebook: 1..4.
 *   - All array arguments are DEVICE pointers owned by the caller, 16-byte aligned, row-major,
 *     unless a comment says "host". The library keeps no pointer after a call returns.
 *   - fp16 values (norms, residual norms) are passed as raw IEEE binary16 bit patterns (uint16_t).
 *   - Calls enqueue work on `stream` (a cudaStream_t; NULL = the legacy default stream) and return
 *     without synchronising. Argument errors are detected on the host before anything is
 *     enqueued; the call then returns a non-zero status and enqueues nothing.
 *   - Kernels never trap. A device-side wait that exceeds its bound records an error that
 *     tq_sync_check() reports as TQ_ERR_DEVICE_TIMEOUT.
 *   - tq_last_error() returns a message for the last failing call on the calling thread.
 *
 * Packed layout (one vector; G = d/32 groups of 32 coordinates; L = 2^b levels)
 *   codes  uint32 [G][b]  bit l of codes[g][p] = bit p of idx[32 g + l]      (bit planes)
 *   signs  uint32 [G]     bit l of signs[g]    = [ (S r)_{32 g + l} >= 0 ]    (Algorithm 2)
 *   norms  fp16           n = ||x||, round to nearest even
 *   gammas fp16           gamma = ||r||, r = x/n - Pi^T c[idx]            (Algorithm 2)
 *   idx_j = #{k : t_k < y_j} for y = Pi x / n (ties to the lower index); the zero vector stores
 *   n = 0, idx_j = L/2 - 1, and for Algorithm 2 gamma = 0 with all sign bits 1.
 *   Non-finite input (a policy of this library; the method is stated for finite vectors): a row
 *   with a NaN entry stores n = NaN, a row with an infinite entry and no NaN stores n = +Inf, and
 *   either row is otherwise stored as the zero vector (idx_j = L/2 - 1; gamma = 0, all sign bits
 *   1); other rows of the call are unaffected. Decoding such a record gives non-finite values;
 *   attention and scores over it are not specified. A finite row whose norm exceeds the fp16 range
 *   (65504) stores n = +Inf with its ordinary codes.
 *   Bytes per vector: b d/8 + 2 (Algorithm 1); (b-1) d/8 + d/8 + 4 (Algorithm 2 at b bits).
 *   Arrays of vectors are the per-vector records above, back to back: codes [n][G][b],
 *   signs [n][G], norms [n], gammas [n].
 *
 * Decode: x_hat = n (Pi^T c[idx] + alpha gamma S^T (2 z - 1)), alpha = sqrt(pi/2) / d; the last
 * term for Algorithm 2 only. alpha makes E_S[<q, x_hat>] = <q, x> (the residual-sign estimator's
 * scale, derived from E[s sign(<s, r>)] = sqrt(2/pi) r/|r| for a Gaussian row s).
 */
#ifndef TQ_H_
#define TQ_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define TQ_API __attribute__((visibility("default")))
#else
#define TQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t tq_status;
#define TQ_OK 0
#define TQ_ERR_INVALID_ARG 1     /* NULL / misaligned pointer, negative size, inconsistent shapes */
#define TQ_ERR_UNSUPPORTED 2     /* d or bits outside the supported range */
#define TQ_ERR_CUDA 3            /* a CUDA runtime call failed (message has the CUDA error) */
#define TQ_ERR_NOT_CONVERGED 4   /* the codebook iteration did not converge */
#define TQ_ERR_DEVICE_TIMEOUT 5  /* a bounded device-side wait gave up (see tq_sync_check) */
#define TQ_ERR_WORKSPACE 6       /* workspace missing or smaller than the *_workspace_bytes value */

/* element types of dense inputs / outputs */
#define TQ_F32 0
#define TQ_BF16 1
#define TQ_F16 2

/* Codebook of the Lloyd-Max quantiser for one coordinate of a rotated unit vector in R^d.
 * Host plain-old-data; pass it by pointer to the device calls (it is copied into the launch).
 * c: ascending centroids (first `levels` = 2^bits used); t: boundaries, t[k] between c[k] and
 * c[k+1] (first levels-1 used). c, t are the fp32 values that define the packed format; c64,
 * t64 the fp64 values they were rounded from. distortion = E|u - Q(u)|^2 for a unit u. */
typedef struct tq_codebook {
  int32_t d;
  int32_t bits;
  int32_t levels;
  int32_t iterations;
  float c[16];
  float t[16];
  double c64[16];
  double t64[16];
  double distortion;
} tq_codebook;

/* Message of the last failing call on this thread ("" if none). Never NULL. */
TQ_API const char* tq_last_error(void);

/* Library version string. */
TQ_API const char* tq_version(void);

/* Lloyd-Max codebook for the density f_d(x) ~ (1 - x^2)^((d-3)/2) on [-1, 1], the law of one
 * coordinate of a uniformly random unit vector in R^d (aiboss88 page, technical principles:
 * Beta-distributed coordinates, Lloyd-Max / continuous 1-D k-means; techblog-plum page: the
 * buckets are computed once, no inference-time cost). HOST ONLY, fp64, deterministic.
 * d >= 3 (any d, not only multiples of 32), bits in 1..4; `out` is a host pointer.
 * Errors: INVALID_ARG (out NULL), UNSUPPORTED (d, bits), NOT_CONVERGED. */
TQ_API tq_status tq_codebook_init(int32_t d, int32_t bits, tq_codebook* out);

/* Size in bytes of the prepared-rotation buffer for dimension d. */
TQ_API size_t tq_rotation_bytes(int32_t d);

/* Prepares the rotation operands every device call reads: copies Pi and S (fp32 d x d,
 * row-major, y = Pi x, s = S r) and derives T = S Pi^T, the transposes and the split-fp16 forms
 * the tensor-core kernels consume. Pi must be orthogonal (the method's random rotation, drawn
 * by the caller); S has i.i.d. N(0,1) entries (the JL matrix of the residual sign). Both are
 * device pointers; `rot` is a caller-owned device buffer of tq_rotation_bytes(d) bytes, valid
 * until the caller frees it or prepares it again. Asynchronous on `stream`.
 * Errors: INVALID_ARG, UNSUPPORTED (d), WORKSPACE (rot_bytes too small), CUDA. */
TQ_API tq_status tq_rotation_prepare(int32_t d, const float* Pi, const float* S, void* rot, size_t rot_bytes,
                              void* stream);

/* Algorithm 1 encode of n vectors x [n][d] (x_dtype TQ_F32 or TQ_BF16) with a b-bit codebook
 * (cb->d must equal d): writes codes [n][d/32][b] and norms [n] (fp16 bits).
 * (ai-navigate-news page: Algorithm 1 = rotation, Lloyd-Max scalar quantisation, MSE-optimal;
 * keys use it.) d <= 128 (any multiple of 32) runs the fused kernel; d > 128 must be a multiple of
 * 128 (up to 4096) and runs the tiled kernel. n may be 0 (no work). */
TQ_API tq_status tq_encode_mse(const tq_codebook* cb, int64_t n, int32_t d, const void* x, int32_t x_dtype,
                        const void* rot, uint32_t* codes, uint16_t* norms, void* stream);

/* Algorithm 2 encode at b bits: Algorithm 1 with the (b-1)-bit codebook `cb_bm1`, then the
 * residual sign bits and the residual norm (ai-navigate-news page: Algorithm 2 = Algorithm 1 at
 * b-1 bits plus sign(S r), unbiased inner products; values use it). Writes codes
 * [n][d/32][b-1], signs [n][d/32], norms [n], gammas [n]. Limits as tq_encode_mse.
 * ws: caller device workspace of tq_encode_workspace_bytes(n, d, 2) bytes (16-byte aligned); that
 * is 0 for d <= 128 (ws may then be NULL). For d > 128 it holds the residuals of the tiles in
 * flight (one slot per SM). */
TQ_API tq_status tq_encode_prod(const tq_codebook* cb_bm1, int64_t n, int32_t d, const void* x, int32_t x_dtype,
                         const void* rot, uint32_t* codes, uint32_t* signs, uint16_t* norms, uint16_t* gammas,
                         void* ws, size_t ws_bytes, void* stream);

/* Workspace bytes an encode of n vectors of length d needs (alg 1: tq_encode_mse, which needs
 * none; alg 2: tq_encode_prod). Depends on the SM count of the current device. */
TQ_API size_t tq_encode_workspace_bytes(int64_t n, int32_t d, int32_t alg);

/* Dequantise n packed vectors: x_hat = n (Pi^T c[idx] (+ alpha gamma S^T (2z-1))) into
 * out [n][d] of out_dtype (TQ_F32 or TQ_BF16). signs and gammas both NULL for Algorithm 1
 * codes, both non-NULL for Algorithm 2 (then cb is the (b-1)-bit codebook the codes use).
 * (ai-navigate-news page: inverse rotation after the scalar codebook.) */
TQ_API tq_status tq_decode(const tq_codebook* cb, int64_t n, int32_t d, const void* rot, const uint32_t* codes,
                    const uint32_t* signs, const uint16_t* norms, const uint16_t* gammas, void* out,
                    int32_t out_dtype, void* stream);

/* Mixed widths per channel group (Algorithm 1). The d rotated coordinates form d/32 groups of 32
 * (the packing groups of the layout); group g is quantised with its own width b_g = group_bits[g]
 * (1..4) and the b_g-bit Lloyd-Max codebook of the same coordinate law (after the rotation every
 * coordinate has that law), so fractional average rates such as 2.5 bits per coordinate, or more
 * bits where a caller wants them, keep the per-coordinate optimality of each group. (The scope of
 * this library's "mixed / fractional bit widths"; the techblog-plum page's compression table quotes
 * an average of 2.5 bits, which is keys at 3 bits with values at 2, and the aigentlab page advises
 * choosing the width per task.)
 *   cbs         HOST array of 4 codebooks for d: cbs[b - 1] has b bits (entries for widths that
 *               group_bits does not use are not read)
 *   group_bits  HOST array of d/32 widths
 *   codes       [n][W] words, W = sum_g b_g: group g's b_g bit-plane words (bit l of word p = bit p
 *               of idx[32 g + l]) at word sum_{g' < g} b_g' of the record; norms [n] as tq_encode_mse
 * d <= 128 (one fused kernel; 32, 64, 96 or 128). Errors: INVALID_ARG, UNSUPPORTED, CUDA. */
TQ_API tq_status tq_encode_mse_mixed(const tq_codebook* cbs, const int32_t* group_bits, int64_t n, int32_t d,
                                     const void* x, int32_t x_dtype, const void* rot, uint32_t* codes,
                                     uint16_t* norms, void* stream);

/* Dequantise the mixed-width format of tq_encode_mse_mixed: x_hat = n Pi^T c_g[idx] with each group's
 * codebook, into out [n][d] of out_dtype (TQ_F32 or TQ_BF16). Arguments as tq_encode_mse_mixed. */
TQ_API tq_status tq_decode_mixed(const tq_codebook* cbs, const int32_t* group_bits, int64_t n, int32_t d,
                                 const void* rot, const uint32_t* codes, const uint16_t* norms, void* out,
                                 int32_t out_dtype, void* stream);

/* Workspace bytes tq_scores needs for these sizes. */
TQ_API size_t tq_scores_workspace_bytes(int64_t nq, int64_t n, int32_t d, int32_t k);

/* Inner-product estimates <q, x_hat_v> of nq queries q [nq][d] (TQ_F32 / TQ_BF16) against n
 * packed database vectors (layout as tq_decode; signs/gammas NULL for Algorithm 1 codes),
 * computed from the codes: the query is rotated (q' = Pi q) and projected (q'' = S q) once and
 * <q, x_hat> = n (<q', c[idx]> + alpha gamma <q'', 2z-1>) (aiboss88 page: inner-product mode,
 * unbiased estimates; vector-database nearest-neighbour search).
 * scores: optional [nq][n] fp32 output (NULL: not written).
 * k: 0, or 1..16 -- then topk_ids [nq][k] (int32) and topk_scores [nq][k] receive, per query,
 * the k largest scores in descending order, ties to the lower id (ids < 2^31); when n < k the
 * missing entries are id -1 with score -inf. k = 0 needs scores.
 * cb: the codebook the codes use (1..4 bits; b-1 bits for Algorithm 2 codes). d: a multiple of
 * 64 up to 4096. n may be 0 (codes / norms may then be NULL).
 * Arithmetic: one tensor-core GEMM over the Walsh bit planes of the codes (exact 0/1 operands) and
 * the sign plane, against the rotated / projected query in two fp16 parts (about 22 bits);
 * fp32 accumulation. Without `scores` the database is scanned in chunks and only the top-k kept.
 * ws: caller device workspace of at least tq_scores_workspace_bytes(nq, n, d, k) bytes. */
TQ_API tq_status tq_scores(const tq_codebook* cb, int64_t nq, int64_t n, int32_t d, const void* q, int32_t q_dtype,
                    const void* rot, const uint32_t* codes, const uint32_t* signs, const uint16_t* norms,
                    const uint16_t* gammas, float* scores, int32_t k, int32_t* topk_ids, float* topk_scores,
                    void* ws, size_t ws_bytes, void* stream);

/* Workspace bytes tq_attend_decode needs for these sizes. */
TQ_API size_t tq_attend_workspace_bytes(int32_t B, int32_t Hq, int32_t Hkv, int64_t T, int32_t d);

/* One decode step of attention over a packed KV cache (aiboss88 page: attention computed on the
 * quantised cache; ai-navigate-news page: keys by Algorithm 1, values by Algorithm 2):
 *   out[b][h] = sum_t softmax_t(scale <q[b][h], k_hat[b][g][t]>) v_hat[b][g][t],  g = h / (Hq/Hkv)
 * with k_hat, v_hat the decoded cache, evaluated from the codes: the query is rotated once,
 * scores come from the key codes, and values are accumulated in the rotated / sign domain with
 * Pi^T and S^T applied once per query head. No mask: every one of the T tokens is attended.
 *   q       [B][Hq][d]  TQ_BF16 or TQ_F32
 *   keys    Algorithm 1 with cb_k (b_k bits): k_codes [B][Hkv][T][d/32][b_k], k_norms [B][Hkv][T],
 *           k_signs and k_gammas NULL; or Algorithm 2 with cb_k the (b_k-1)-bit codebook (1..2 bits):
 *           k_codes [B][Hkv][T][d/32][b_k-1], k_signs [B][Hkv][T][d/32], k_norms, k_gammas
 *           [B][Hkv][T]. Algorithm 2 keys give the unbiased inner-product estimate
 *           <q, k_hat> = n (<Pi q, c[idx]> + alpha gamma <S q, 2z - 1>) (aiboss88 page, QJL stage).
 *   values  Algorithm 2 with cb_v the (b_v-1)-bit codebook: v_codes [B][Hkv][T][d/32][b_v-1],
 *           v_signs [B][Hkv][T][d/32], v_norms, v_gammas [B][Hkv][T];
 *           or Algorithm 1 (v_signs and v_gammas NULL, cb_v the b_v-bit codebook)
 *   scale   the softmax scale; 0 (or any value that is not > 0) selects 1/sqrt(d)
 *   out     [B][Hq][d] fp32
 * Supported: d = 128, Hq a multiple of Hkv with Hq/Hkv <= 8, T >= 1, key codebooks of 1..3 bits,
 * value codebooks of 1..2 bits (Algorithm 2 values at 2..3 bits, Algorithm 1 values at 1..2 bits).
 * ws: caller device workspace of at least tq_attend_workspace_bytes(...) bytes. */
TQ_API tq_status tq_attend_decode(const tq_codebook* cb_k, const tq_codebook* cb_v, int32_t B, int32_t Hq, int32_t Hkv,
                           int64_t T, int32_t d, const void* q, int32_t q_dtype, const void* rot,
                           const uint32_t* k_codes, const uint16_t* k_norms, const uint32_t* k_signs,
                           const uint16_t* k_gammas, const uint32_t* v_codes,
                           const uint32_t* v_signs, const uint16_t* v_norms, const uint16_t* v_gammas, float scale,
                           float* out, void* ws, size_t ws_bytes, void* stream);

/* Workspace bytes tq_attend_prefill needs for these sizes (0 for invalid sizes). */
TQ_API size_t tq_attend_prefill_workspace_bytes(int32_t B, int32_t Hq, int32_t Hkv, int32_t Qn, int64_t T, int32_t d);

/* Multi-query (prefill) attention over a packed KV cache with a causal mask (techblog-plum page,
 * notes: the rotation / QJL overhead shows once many queries share the cache; aiboss88 page:
 * attention on the quantised cache). The last Qn of the T cached tokens of every slice are the new
 * tokens themselves; query token j (0 <= j < Qn) sits at cache position T - Qn + j and attends the
 * tokens t <= T - Qn + j:
 *   out[b][j][h] = sum_{t <= T-Qn+j} softmax_t(scale <q[b][j][h], k_hat[b][g][t]>) v_hat[b][g][t],
 *   g = h / (Hq/Hkv).
 *   q    [B][Qn][Hq][d]  TQ_BF16 or TQ_F32;  out [B][Qn][Hq][d] fp32
 *   cache, codebooks, rot, scale: as tq_attend_decode (keys Algorithm 1 or 2, values Algorithm 1
 *   or 2), with the same limits; 1 <= Qn <= T. Qn = 1 is tq_attend_decode.
 * The kernels evaluate up to 8 (query token, query head) pairs per KV head in one pass over the
 * cache (8 / (Hq/Hkv) query tokens per pass); longer prefills take several passes, each over the
 * tokens its queries can see. ws: caller device workspace of at least
 * tq_attend_prefill_workspace_bytes(B, Hq, Hkv, Qn, T, d) bytes. */
TQ_API tq_status tq_attend_prefill(const tq_codebook* cb_k, const tq_codebook* cb_v, int32_t B, int32_t Hq,
                                   int32_t Hkv, int32_t Qn, int64_t T, int32_t d, const void* q, int32_t q_dtype,
                                   const void* rot, const uint32_t* k_codes, const uint16_t* k_norms,
                                   const uint32_t* k_signs, const uint16_t* k_gammas, const uint32_t* v_codes,
                                   const uint32_t* v_signs, const uint16_t* v_norms, const uint16_t* v_gammas,
                                   float scale, float* out, void* ws, size_t ws_bytes, void* stream);

/* Workspace bytes of tq_attend_append for these sizes (k_bits: the key codebook's bits;
 * v_codebook_bits: the value codebook's bits, b_v - 1); 0 for invalid sizes. */
TQ_API size_t tq_attend_append_workspace_bytes(int32_t B, int32_t Hq, int32_t Hkv, int64_t T_cur, int32_t d,
                                               int32_t k_bits, int32_t v_codebook_bits);

/* One decode step on a packed KV cache with room to grow: the new token's key and value of every
 * (batch, KV head) slice are encoded into the next free slot, then the query attends over all
 * filled slots. This is the cache-integration step around the attention (ai-navigate-news page:
 * keys by Algorithm 1, values by Algorithm 2, appended as tokens are generated; aiboss88 page:
 * attention on the quantised cache). The result equals tq_encode_mse / tq_encode_prod of the new
 * vectors written to slot T_cur, followed by tq_attend_decode over T_cur + 1 tokens.
 *   cache   the arrays of tq_attend_decode with T_max slots per slice: k_codes [B][Hkv][T_max][d/32][b_k],
 *           k_norms [B][Hkv][T_max], v_codes [B][Hkv][T_max][d/32][b_v-1], v_signs
 *           [B][Hkv][T_max][d/32], v_norms, v_gammas [B][Hkv][T_max]; slots [0, T_cur) hold
 *           earlier tokens, slot T_cur is written, slots beyond it are neither read nor written
 *   k_new, v_new  [B][Hkv][d] in x_dtype (TQ_F32 or TQ_BF16)
 *   q, out, scale, cb_k, cb_v (the (b_v-1)-bit codebook), rot  as in tq_attend_decode
 * Requires 0 <= T_cur < T_max and the limits of tq_attend_decode (d = 128, ...); values are
 * Algorithm 2 (v_signs, v_gammas required). ws: caller device workspace of at least
 * tq_attend_append_workspace_bytes(B, Hq, Hkv, T_cur, d, b_k, b_v - 1) bytes. Errors: those of
 * the encoders and of tq_attend_decode; on an error nothing after the failing stage is enqueued.
 * Launches, in stream order: the two encoders, one record-scatter kernel, the attention kernels. */
TQ_API tq_status tq_attend_append(const tq_codebook* cb_k, const tq_codebook* cb_v, int32_t B, int32_t Hq,
                                  int32_t Hkv, int64_t T_cur, int64_t T_max, int32_t d, const void* q,
                                  int32_t q_dtype, const void* k_new, const void* v_new, int32_t x_dtype,
                                  const void* rot, uint32_t* k_codes, uint16_t* k_norms, uint32_t* v_codes,
                                  uint32_t* v_signs, uint16_t* v_norms, uint16_t* v_gammas, float scale,
                                  float* out, void* ws, size_t ws_bytes, void* stream);

/* Size of the fixed scratch array behind tq_attend_decode_noalloc (8 MiB per device). It covers,
 * for example, B = 16, Hkv = 8, Hq = 32, T = 131072 (about 3.4 MB). */
#define TQ_ATTEND_NOALLOC_MAX_BYTES (8u << 20)

/* tq_attend_decode without a caller workspace: the same computation, arguments, layouts and
 * limits, but the scratch is a fixed array of TQ_ATTEND_NOALLOC_MAX_BYTES bytes that the library
 * holds in device memory (one per device). No counterpart in the TurboQuant write-ups: it exists
 * for callers that cannot allocate device memory -- a plain C host holding only the cache
 * pointers, a runtime whose memory pool already owns all of HBM, a latency-critical stream that
 * must not meet cudaFree's device-wide wait. The call allocates and frees nothing.
 * Errors: TQ_ERR_WORKSPACE when tq_attend_workspace_bytes(B, Hq, Hkv, T, d) exceeds the array
 * (nothing is enqueued); otherwise those of tq_attend_decode. Every call on a device shares that
 * device's array: calls whose GPU work overlaps (different streams, different host threads) race
 * and give wrong results, so order them (one stream, or events). Nothing in the array needs to be
 * zero beforehand; no state carries from one call to the next. */
TQ_API tq_status tq_attend_decode_noalloc(const tq_codebook* cb_k, const tq_codebook* cb_v, int32_t B, int32_t Hq,
                                   int32_t Hkv, int64_t T, int32_t d, const void* q, int32_t q_dtype,
                                   const void* rot, const uint32_t* k_codes, const uint16_t* k_norms,
                                   const uint32_t* k_signs, const uint16_t* k_gammas, const uint32_t* v_codes,
                                   const uint32_t* v_signs, const uint16_t* v_norms, const uint16_t* v_gammas,
                                   float scale, float* out, void* stream);

/* Self-test of the failure-detection path; no counterpart in the TurboQuant write-ups. Every
 * hand-off between the warps of a libtq kernel is a wait bounded in time: one that runs out records
 * an error and lets the kernel return, so a lost arrival is reported instead of hanging the GPU.
 * This call enqueues one small kernel that makes such a wait run out on purpose (an mbarrier that
 * nothing arrives on, limit `limit_ns` nanoseconds, 1000 <= limit_ns <= 1e9); the next
 * tq_sync_check then returns TQ_ERR_DEVICE_TIMEOUT once and clears it, and later calls work as
 * before. Nothing faults and nothing hangs. Errors: INVALID_ARG (limit), CUDA. */
TQ_API tq_status tq_selftest_wait(uint64_t limit_ns, void* stream);

/* Synchronises `stream`, then reports a pending CUDA error (TQ_ERR_CUDA) or a device-side
 * timeout recorded by any libtq kernel since the last check (TQ_ERR_DEVICE_TIMEOUT, which this
 * call clears). TQ_OK otherwise. */
TQ_API tq_status tq_sync_check(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* TQ_H_ */
