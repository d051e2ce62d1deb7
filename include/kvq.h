/*
 * kvq.h -- C ABI of the B200 quantized-KV decode-attention library (libkvq.so).
 *
 * The operations follow the tiered, runtime-certified quantized attention of
 * "Runtime-Certified Bounded-Error Quantized Attention":
 *   - Methodology 1 (Tiered storage): Tier 1 in GPU memory holds INT8 (or
 *     INT4) key codes and per-group INT4 value codes with scale/offset
 *     metadata and a per-block error annotation eta_b; Tier 2 in pinned host
 *     memory holds the unquantized originals.
 *   - Methodology 2 (Two-term error decomposition): per query, a bound
 *     E_key + E_val on the error of the quantized attention output, computed
 *     online from the quantization scales, the query norms and the value
 *     range, without touching the originals.
 *   - Methodology 1 (Fallback) / 3 (ladder, per-head rung): a query whose
 *     bound exceeds tau is recomputed as exact dense attention from Tier 2.
 * and the rotated-key codec of "Statistical Inference and Quality Measures of
 * KV Cache Quantisations Inspired by TurboQuant" (Quantisation schemes, KQV:
 * Walsh-Hadamard transform before scalar quantization of K), and two codecs of
 * their own: that page's KQV codec and the quaternion codec of "Hurwitz
 * Quaternion Multiplicative Quantization for KV Cache Compression" (HQMQ).
 *
 * Conventions
 *   - Every pointer is caller-owned; the library never allocates or frees
 *     memory on the decode path and keeps no state between calls except a
 *     cache of device properties (and the static scratch of
 *     kvq_decode_attention_noalloc).  "device" = CUDA device memory
 *     (or managed), "host" = host memory, "pinned" = page-locked host memory.
 *   - Every call validates its arguments before launching anything and
 *     returns a kvq_status (0 = KVQ_OK); no exception crosses the ABI.
 *     kvq_last_error() gives a message for the last failure on this thread.
 *   - All calls are asynchronous on the given stream except
 *     kvq_fallback_exact and kvq_device_error, which wait (with a deadline).
 *   - Calls on distinct streams with distinct output/workspace buffers are
 *     independent.  Only devices of compute capability 10.0 (sm_100a) run
 *     the kernels.
 *   - The decode entry points launch with programmatic stream serialization:
 *     their CTAs may start while the previous kernel in the stream is
 *     finishing, but before griddepcontrol.wait they only set up shared
 *     memory and prefetch cache pages into L2 (which changes no memory), so
 *     every result is the same as after a plain stream-ordered launch,
 *     whatever that kernel writes.
 *
 * Quantized cache layout (one block per physical page and kv head, 16 tokens;
 * nb = head_dim/32):
 *   [K codes 16*head_dim*k_bits/8 B][V codes 16*head_dim/2 B]
 *   [K scales fp16 [16][head_dim/k_group]][V (scale, zero) fp16 [16][nb][2]]
 *   K code of channel c (b = c/32, w = c%32, s = w/8, i = w%8) in a token row:
 *     8 bit: byte s*8*nb + 8*b + i (int8); for head_dim 128 (128-byte rows)
 *            that byte's 16-byte chunk index is XORed with slot % 8, slot =
 *            the token's row in the page;
 *     4 bit: byte s*4*nb + 4*b + i/2, low nibble for even c (4-bit two's complement).
 *   V code of channel c (g = c/32, w = c%32): byte (w/4)*2*nb + 2*g + (w%4)/2,
 *     low nibble for even c (unsigned).
 *   Key codec per token and k_group channels: s = fp16 rounded up of
 *   max|x|/Q (Q = 127 or 7), code = rint(x/s) in [-Q, Q].  Value codec per
 *   token and 32 channels: z = fp16 rounded down of min x, s = fp16 rounded up
 *   of (max x - z)/15, code = rint((x - z)/s) in [0, 15].
 *   eta[page][kv_head] = max over the block's tokens of |v - fmaf(code, s, z)|,
 *   rounded up by one fp32 ulp.
 *
 * Outlier extraction (outliers = 1; the median-multiplier rule of "Hurwitz
 * Quaternion Multiplicative Quantization for KV Cache Compression", Method 3):
 *   a token's vector (K after the rotation, if any, and V) is cut into
 *   4-channel chunks; the chunk with the largest norm
 *   sqrt((x0*x0 + x1*x1) + (x2*x2 + x3*x3)) (fp32, each operation rounded)
 *   above 3 * median of the vector's chunk norms (the median of the even
 *   count is 0.5 * (a + b) of the two middle norms) is kept in fp16 (round to
 *   nearest; ties: the lower chunk index; no extraction if a norm is NaN).
 *   Its channels get code 0 and take no part in their group's scale, zero or
 *   error; eta also covers the fp16 rounding of the extracted values.  The
 *   block then ends in a 288-byte outlier section:
 *     [K chunk index u8 [16]][V chunk index u8 [16]]
 *     [K chunk values fp16 [16][4]][V chunk values fp16 [16][4]]
 *   index 0xFF = no extraction in that token (its values are then 0).
 *   An extracted value that is not finite or above 65504 in magnitude is
 *   stored as 0 and sets KVQ_ERR_RANGE.
 */
#ifndef KVQ_H_
#define KVQ_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KVQ_API __attribute__((visibility("default")))
#else
#define KVQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st* kvq_stream_t;

typedef enum {
  KVQ_OK = 0,
  KVQ_ERR_INVALID_ARG = -1, /* null pointer, bad size, layout or stride */
  KVQ_ERR_UNSUPPORTED = -2, /* valid but unsupported shape (head_dim, group, rows) */
  KVQ_ERR_RANGE = -3,       /* non-finite input or fp16-overflowing scale/zero */
  KVQ_ERR_CUDA = -4,        /* a CUDA runtime call failed */
  KVQ_ERR_TIMEOUT = -5,     /* a bounded host wait gave up */
  KVQ_ERR_DEVICE = -6       /* reserved; no call returns it.  Kernels report their errors
                               (KVQ_ERR_INVALID_ARG, KVQ_ERR_RANGE, KVQ_ERR_TIMEOUT) in
                               the cache's error word, read by kvq_device_error */
} kvq_status;

typedef enum { KVQ_F32 = 0, KVQ_BF16 = 1 } kvq_dtype;

#define KVQ_PAGE_SIZE 16

typedef struct kvq_cache {
  int32_t num_kv_heads;    /* Hkv >= 1 */
  int32_t head_dim;        /* d: 64 or 128 */
  int32_t page_size;       /* tokens per page: must be 16 */
  int32_t num_pages;       /* physical pages in the pool */
  int32_t k_bits;          /* 8 or 4 */
  int32_t k_group;         /* 32, 64 or 128, divides head_dim */
  int32_t k_rotate;        /* 1: keys (and queries) get the randomized Hadamard rotation */
  int32_t v_bits;          /* must be 4 */
  int32_t v_group;         /* must be 32 */
  void* pool;              /* device, kvq_pool_bytes() bytes, 16-byte aligned */
  float* v_eta;            /* device, [num_pages][num_kv_heads]; zero before a page's first append */
  const int8_t* rot_signs; /* device, head_dim entries of +1/-1; required iff k_rotate */
  int32_t* error_word;     /* device, one int32 kernels set to a kvq_status on error; may be NULL */
  int32_t outliers;        /* 1: outlier extraction (see the layout above); 0: none */
  int32_t codec;           /* KVQ_CODEC_INT (0: the layout above), KVQ_CODEC_KQV (1) or
                              KVQ_CODEC_HQMQ (2) */
  const float* qjl;        /* device, KVQ_CODEC_KQV: the QJL projections S, fp32
                              [head_dim][head_dim] row-major (row i = projection i) */
  const float* hq_sec;     /* device, KVQ_CODEC_HQMQ: the secondary unit quaternions,
                              fp32 [num_kv_heads][2 (K, V)][hq_s][4] */
  int32_t hq_s;            /* KVQ_CODEC_HQMQ: secondary units per (kv head, role) S,
                              1..64 */
} kvq_cache;

#define KVQ_CODEC_INT 0
#define KVQ_CODEC_KQV 1
#define KVQ_CODEC_HQMQ 2
#define KVQ_HQMQ_MAX_S 64

/* The KQV codec ("Statistical Inference and Quality Measures of KV Cache
 * Quantisations Inspired by TurboQuant", Quantisation schemes: KQV), codec =
 * KVQ_CODEC_KQV: K and V rotated by the randomized Walsh-Hadamard transform
 * (rot_signs, required; k_rotate must be 1), K coded by the 4-bit Lloyd-Max
 * quantizer of the rotated unit vector's coordinates, V by the 3-bit one
 * plus the 1-bit QJL sketch of its residual (k_bits 4, v_bits 3, k_group =
 * v_group = head_dim, outliers 0):
 *   x' = rotation of x; n = |x'|_2 (fp32, a sequential fmaf chain over the
 *   channels); u = x' / n (0 when n = 0); code = the number of thresholds
 *   below u (kvq_kqv_codebook); k^' = n * centroid[code];
 *   V: r = u - centroid3[code]; bit i = [sum_c S_ic r_c >= 0] (sequential
 *   fmaf chain); v^' = n_v (centroid3[code] + sqrt(pi/2)/d |r| S^T b);
 *   v^ = sigma o (H v^') / sqrt(d).
 * Block of one (page, kv head), 16 tokens (d = head_dim):
 *   [K codes 4-bit [16][d/2]][V codes 3-bit in nibbles [16][d/2]]
 *   [V sketch bits [16][d/8]][|k'| f32 [16]][eps f32 [16]][|v'| f32 [16]]
 *   [|r| f32 [16]][v^ max, min f32 [d/32][2]]
 * nibble of channel c in byte c/2 (low nibble for even c); sketch bit i in
 * byte i/8, bit i%8.  eps = max_c |k'_c - k^'_c| one ulp up; eta[page][h] =
 * max over the block of (max_c |v_c - v^_c| + 2^-16 n_v) one ulp up; the
 * range of each 32-channel group starts at [0, 0] in a zeroed block and
 * widens to every v^ appended.  The decode's bound uses Delta_j =
 * kappa*s*(|q'|_1 eps_j + 2^-16 |q'|_2 n_kj) and E_key = TV (max_g range_g +
 * 2 max eta).  kvq_decode_attention_append and kvq_adaptive_precision return
 * KVQ_ERR_UNSUPPORTED for this codec. */

/* The HQMQ codec ("Hurwitz Quaternion Multiplicative Quantization for KV
 * Cache Compression", Method 1-2), codec = KVQ_CODEC_HQMQ: every 4-channel
 * chunk x of K and of V is a quaternion split into its radius r = |x| and
 * its direction, coded by the product codebook {q_p q_s}: q_p one of the 24
 * Hurwitz units (the binary tetrahedral group 2T: p = 0..7 the units +-1,
 * +-i, +-j, +-k as p = 2 n + [negative]; p = 8..23 (+-1 +-i +-j +-k)/2 with
 * component n negative when bit n of p - 8 is set), q_s one of the hq_s
 * secondary units of the kv head and role (k_bits = v_bits = 6, k_group =
 * v_group = 4, k_rotate 0; outliers 0, or 1 for Med3x over this codec):
 *   code i = 24 s + p maximizing <x, q_p q_s>, evaluated as <x conj(q_s),
 *   q_p>: y = x conj(q_s) with each component a sequential fmaf chain over
 *   x0..x3; the best axis unit is max_n |y_n| (first n on ties), the best
 *   half unit 0.5 (((|y0| + |y1|) + |y2|) + |y3|) with y's signs (-0 as +),
 *   taken only when strictly larger; a later s only when strictly larger;
 *   r = sqrt((x0^2 + x1^2) + (x2^2 + x3^2)) (fp32), stored as fp8 E4M3
 *   (round to nearest even, saturating at 448); codeword c = q_p q_s in fp32
 *   (exact term products summed left to right); x^ = r^ * c16 with c16 the
 *   codeword rounded to fp16 per component (nearest even; the product is
 *   exact in fp32).
 *   A chunk with a non-finite r gets code 0, radius 0; a token with a
 *   non-finite value sets KVQ_ERR_RANGE and eps (K) and eta to +inf.
 *   With outliers = 1 the Med3x chunk of K and of V (chosen as for the INT
 *   codec) takes code 0 and radius 0, is stored in fp16 in the outlier
 *   section appended to the block (the layout above) and reconstructs to its
 *   fp16 values.
 * Block of one (page, kv head), 16 tokens, n = head_dim / 4 chunks,
 * chunk-major (token t of chunk ch at [ch][t]):
 *   [K codes u16 [n][16]][V codes u16 [n][16]][K radii e4m3 [n][16]]
 *   [V radii e4m3 [n][16]][|k|_2 f32 [16]][eps f32 [16]]
 *   [v^ max, min f32 [head_dim/32][2]]
 * eps = |k - k^|_2 (sequential fmaf chain) raised by 2^-16 of itself, one
 * ulp up; eta[page][h] = max over the block of (max_c |v_c - v^_c| + 2^-16
 * |v|_2) one ulp up; the range of each 32-channel group starts at [0, 0] in a
 * zeroed block.  The decode's bound uses Delta_j = kappa*s*|q|_2 (eps_j +
 * 2^-16 |k_j|_2) and E_key = TV (max_g range_g + 2 max eta), E_val as for
 * the other codecs.  kvq_decode_attention_append and kvq_adaptive_precision
 * return KVQ_ERR_UNSUPPORTED for this codec. */

/* Centroids (2^bits) and decision thresholds (2^bits - 1) of the KQV codec's
 * scalar quantizer for unit vectors in dimension head_dim: the Lloyd-Max
 * quantizer of N(0, 1) (the Gaussian limit of the Beta((d-1)/2, (d-1)/2)
 * coordinate marginal) divided by sqrt(head_dim), computed in fp64 and
 * rounded to fp32.  bits 1..6; host memory; returns a kvq_status. */
KVQ_API int kvq_kqv_codebook(int32_t bits, int32_t head_dim, float* centroids,
                             float* thresholds);

/* Bytes of one (page, kv head) block, and of the whole pool; 0 if the cache
 * description is invalid or unsupported. */
KVQ_API size_t kvq_block_bytes(const kvq_cache* cache);
KVQ_API size_t kvq_pool_bytes(const kvq_cache* cache);

/* Quantize-on-append (Methodology 1, Tier 1).
 * Token t < valid_tokens[s] (or < num_tokens when valid_tokens is NULL) of
 * sequence s is written at logical position start_pos[s] + t, i.e. into
 * physical page page_table[s*max_pages_per_seq + pos/16], slot pos%16, of
 * every kv head.  k, v (device, in_dtype) element (s, h, t, c) is at
 * s*seq_stride + h*head_stride + t*token_stride + c (strides in elements;
 * channels contiguous); every element with t < num_tokens must be readable,
 * also for tokens at or past valid_tokens[s] (they are loaded before the
 * valid count is known, and ignored).  page_table, start_pos, valid_tokens:
 * device int32.  eta of the touched blocks is raised with an atomic max, so eta of a reused
 * page must be zeroed by the caller first.  A non-finite input or an
 * fp16-overflowing scale writes zero codes and scale for that group and sets
 * *error_word = KVQ_ERR_RANGE; a page index outside [0, num_pages) skips the
 * token and sets KVQ_ERR_INVALID_ARG.  Asynchronous on `stream`. */
KVQ_API int kvq_quantize_append(const kvq_cache* cache, const void* k, const void* v, int in_dtype,
                        int64_t seq_stride, int64_t head_stride, int64_t token_stride,
                        int32_t num_seqs, int32_t num_tokens, const int32_t* valid_tokens,
                        const int32_t* start_pos, const int32_t* page_table,
                        int32_t max_pages_per_seq, kvq_stream_t stream);

/* Workspace bytes kvq_decode_attention / kvq_error_bound need for this shape
 * on the current device (split-K partials and per-(sequence, kv head)
 * counters).  The workspace must be zero-filled once before its first use;
 * every call leaves its counters at zero again.  Returns 0 on invalid input. */
KVQ_API size_t kvq_workspace_size(const kvq_cache* cache, int32_t num_seqs, int32_t num_queries,
                          int32_t num_q_heads, int32_t max_pages_per_seq);

/* Quantized decode attention with the certified bound (Methodology 2).
 * q (device, q_dtype) [num_seqs][num_queries][num_q_heads][head_dim]; q head h
 * attends kv head h / (num_q_heads/num_kv_heads) over tokens [0, seq_lens[s])
 * of its sequence (no mask inside the context).  num_queries *
 * (num_q_heads/num_kv_heads) must be <= 4.  softmax_scale <= 0 selects
 * 1/sqrt(head_dim).  Writes (device) out fp32 [..][head_dim] (quantized-path
 * attention), bound fp32 [num_seqs][num_queries][num_q_heads] (a certified
 * upper bound on max_c |o_exact - out| against exact attention over the
 * originals) and flags uint8 (bound > tau; tau = INFINITY never flags).
 * An empty context gives out = 0, bound = 0, flag = 0.  page_table and
 * seq_lens: device int32.  A page that cannot be read leaves its (sequence,
 * kv head) without a certified bound: a page index outside the pool (never
 * copied; *error_word = KVQ_ERR_INVALID_ARG), a bounded wait for a page copy
 * that ran out (KVQ_ERR_TIMEOUT) or seq_lens[s] > 16*max_pages_per_seq (the
 * context is cut to the page table; KVQ_ERR_INVALID_ARG).  Every query row of
 * that (sequence, kv head) then gets bound = +INFINITY and flag = 1 whatever
 * tau is, so kvq_fallback_exact recomputes it; out holds attention over the
 * pages that were read.  With outlier extraction (cache->outliers = 1) the
 * scores use the extracted key chunks' fp16 values (against q' in fp32) and
 * Delta_j adds, per extracted channel, |q'_c| (2^-11 |k16_c| + 2^-25) (half
 * an fp16 ulp; for rotated keys also s*2^-16*|q'|_2 times the chunk's norm,
 * all times kappa * softmax scale); the outputs use the extracted value
 * chunks' fp16 values, and the value range of each group widens to them.
 * workspace: device, >= kvq_workspace_size() bytes, 16-byte aligned.
 * Asynchronous. */
KVQ_API int kvq_decode_attention(const kvq_cache* cache, const void* q, int q_dtype, int32_t num_seqs,
                         int32_t num_queries, int32_t num_q_heads, const int32_t* page_table,
                         int32_t max_pages_per_seq, const int32_t* seq_lens,
                         float softmax_scale, float tau, float* out, float* bound,
                         uint8_t* flags, void* workspace, size_t workspace_bytes,
                         kvq_stream_t stream);

/* The certified bound and flags alone: the same pass as
 * kvq_decode_attention without writing attention outputs. */
KVQ_API int kvq_error_bound(const kvq_cache* cache, const void* q, int q_dtype, int32_t num_seqs,
                    int32_t num_queries, int32_t num_q_heads, const int32_t* page_table,
                    int32_t max_pages_per_seq, const int32_t* seq_lens, float softmax_scale,
                    float tau, float* bound, uint8_t* flags, void* workspace,
                    size_t workspace_bytes, kvq_stream_t stream);

/* One decode step in one launch: kvq_quantize_append of the step's new token
 * fused into kvq_decode_attention.  For every sequence s with seq_lens[s] >= 1
 * the new token -- k_new / v_new (device, in_dtype) element (s, h, c) at
 * s*new_seq_stride + h*new_head_stride + c -- is quantized exactly as
 * kvq_quantize_append would (same codes, scales and eta) into logical
 * position seq_lens[s] - 1, i.e. physical page
 * page_table[s*max_pages_per_seq + (seq_lens[s]-1)/16], and the attention over
 * seq_lens[s] tokens includes it.  Equivalent to kvq_quantize_append
 * (num_tokens = 1, start_pos = seq_lens - 1) followed by kvq_decode_attention,
 * with the same results, minus one launch and its dependent round trips; the
 * warp of the decode that reads the sequence's last page writes the token
 * into it first.  Sequences with seq_lens[s] == 0 append nothing.  Errors as
 * for the two calls.  Not the "Runtime-Certified..." pages' own interface: a
 * fusion of two of its calls. */
KVQ_API int kvq_decode_attention_append(const kvq_cache* cache, const void* k_new,
                                        const void* v_new, int in_dtype,
                                        int64_t new_seq_stride, int64_t new_head_stride,
                                        const void* q, int q_dtype, int32_t num_seqs,
                                        int32_t num_queries, int32_t num_q_heads,
                                        const int32_t* page_table, int32_t max_pages_per_seq,
                                        const int32_t* seq_lens, float softmax_scale, float tau,
                                        float* out, float* bound, uint8_t* flags,
                                        void* workspace, size_t workspace_bytes,
                                        kvq_stream_t stream);

/* Staging bytes kvq_fallback_exact needs to recompute one (sequence, kv head)
 * of up to max_ctx tokens: a merge scratch (48 items x 8 rows x (head_dim
 * + 2) floats, rounded up to 256 B) plus K and V of max_ctx tokens (each
 * rounded up to 256 B).  This is the minimum; with room for two such K/V
 * pairs beyond the scratch, the call splits the buffer in two halves and the
 * copies into one overlap the recomputation from the other.  0 for an
 * unsupported head_dim or dtype. */
KVQ_API size_t kvq_fallback_staging_size(const kvq_cache* cache, int orig_dtype, int32_t max_ctx);

/* Exact recomputation from Tier 2 (Methodology 1, Fallback; per-head rung of
 * the ladder, applied per query).  Waits on `main` for the decode that wrote
 * `flags` (device uint8, same shape as bound), copies them to flags_host
 * (pinned, num_seqs*num_queries*num_q_heads bytes) on `side`, and polls with
 * a deadline of timeout_ms (KVQ_ERR_TIMEOUT when it passes; 0 times out at
 * once).  For every (sequence, kv head) with a flagged query it copies the
 * originals k_orig_host, v_orig_host (pinned, orig_dtype, element (s, h, t, c)
 * at s*orig_seq_stride + h*orig_head_stride + t*head_dim + c) for tokens
 * [0, seq_lens_host[s]) into `staging` (device, 16-byte aligned, at least
 * kvq_fallback_staging_size bytes) with cudaMemcpyAsync on `side`, and
 * overwrites out rows of the flagged queries with exact fp32 softmax
 * attention (softmax_scale as in decode).  q as in decode.  The recompute
 * kernels run on `main`, each after the copies it reads (events), so `main`
 * is ordered after all of this call's work when it returns; the copies into
 * a staging half that is being reused wait (on `side`) for the recompute
 * that read it before.  *num_fallback (host) = number of recomputed
 * queries.  On any error out is left unmodified for the rows not yet
 * recomputed.  Blocks the calling thread until the flags are on the host.
 * After an error return (KVQ_ERR_TIMEOUT included) copies and kernels this
 * call queued may still be pending on main_stream and side_stream: the flag
 * read-back into flags_host, page-ins into staging and recomputes into out.
 * Synchronize both streams (or order later work after them) before reusing
 * flags_host, staging or out. */
KVQ_API int kvq_fallback_exact(const kvq_cache* cache, const void* k_orig_host, const void* v_orig_host,
                       int orig_dtype, int64_t orig_seq_stride, int64_t orig_head_stride,
                       const void* q, int q_dtype, int32_t num_seqs, int32_t num_queries,
                       int32_t num_q_heads, const int32_t* seq_lens_host, float softmax_scale,
                       const uint8_t* flags, uint8_t* flags_host, float* out, void* staging,
                       size_t staging_bytes, kvq_stream_t main_stream,
                       kvq_stream_t side_stream, int32_t timeout_ms, int32_t* num_fallback);

/* Adaptive precision and the first rungs of the fallback ladder ("Runtime-
 * Certified Bounded-Error Quantized Attention", Methodology 3: adaptive top-K*
 * selection from a light scoring pass with the quantized keys, the
 * ranking-consistency check, rung 2 value promotion), for the rows a decode
 * flagged.  A block is one 16-token page of one kv head.  Per flagged query
 * row (sequence, query, q head; kv head h / (num_q_heads/num_kv_heads)):
 *   M^_b  = the block's mass under the softmax of the quantized scores
 *   keys  : the blocks in order of M^_b (descending; ties by lower page) up
 *           to the fewest whose mass reaches tau_cov (none if tau_cov <= 0)
 *           take the original keys: exact scores s*q.k (q unrotated) with
 *           Delta_j = kappa*s*2^-16*|q|_2*|k_j|_2 (an allowance for the fp32
 *           dot product) instead of the quantized Delta_j
 *   values: blocks with M^_b * eta_b > v_tol take the original values and
 *           leave E_val
 *   out, bound: attention and the certified bound of kvq_decode_attention
 *           recomputed with these scores, Delta and values
 *   ranking check: along the key-promoted blocks in order of M^_b, a block
 *           whose exact log-mass log sum_{j in b} e^{z_j} exceeds an earlier
 *           block's by more than rank_tol makes the ranking inconsistent
 *   flag  = inconsistent || bound > tau (|| a page could not be read)
 * Waits on `main_stream` for the decode that wrote `flags`, reads them into
 * flags_host (pinned, num_seqs*num_queries*num_q_heads bytes) on
 * `side_stream` with a deadline of timeout_ms for the whole call
 * (KVQ_ERR_TIMEOUT when it passes), scores and selects on `main_stream`,
 * reads back the union of promoted blocks per (sequence, kv head), copies
 * only those blocks' originals (k_orig_host, v_orig_host: pinned, layout as
 * for kvq_fallback_exact) into `staging` with cudaMemcpyAsync on
 * `side_stream`, and recomputes the flagged rows on `main_stream`,
 * overwriting their out, bound and flags (device, as written by the decode);
 * rows not flagged are left as they are.  promoted_keys / promoted_values
 * (device, [rows][max_pages_per_seq] uint8, or NULL) get the flagged rows'
 * promotion maps.  work: device, >= kvq_adaptive_work_size() bytes; host_work:
 * pinned, >= kvq_adaptive_host_size() bytes; staging: device, at least
 * kvq_adaptive_staging_size() bytes (the promoted blocks of one (sequence, kv
 * head)); all 16-byte aligned.  max_pages_per_seq <= 8192.  On return
 * *num_rows = the rows that ran through the ladder and *num_flagged = the
 * rows flagged afterwards (flags_host holds the new flags); `main_stream` is
 * ordered after all of this call's work.  After an error return, queued work
 * may still be pending on both streams (synchronize them before reusing the
 * buffers).  KVQ_FAULT=memcpy makes the page-in fail (KVQ_ERR_CUDA) for
 * tests.  Blocks the calling thread on the bounded waits.  With outlier
 * extraction the quantized scores, values, Delta and value range include the
 * extracted chunks exactly as kvq_decode_attention does.  A KQV or HQMQ cache
 * returns KVQ_ERR_UNSUPPORTED (and kvq_adaptive_work_size 0). */
KVQ_API size_t kvq_adaptive_work_size(const kvq_cache* cache, int32_t num_seqs,
                                      int32_t num_queries, int32_t num_q_heads,
                                      int32_t max_pages_per_seq);
KVQ_API size_t kvq_adaptive_host_size(const kvq_cache* cache, int32_t num_seqs,
                                      int32_t max_pages_per_seq);
KVQ_API size_t kvq_adaptive_staging_size(const kvq_cache* cache, int orig_dtype,
                                         int32_t max_pages_per_seq);
KVQ_API int kvq_adaptive_precision(const kvq_cache* cache, const void* k_orig_host,
                                   const void* v_orig_host, int orig_dtype,
                                   int64_t orig_seq_stride, int64_t orig_head_stride,
                                   const void* q, int q_dtype, int32_t num_seqs,
                                   int32_t num_queries, int32_t num_q_heads,
                                   const int32_t* page_table, int32_t max_pages_per_seq,
                                   const int32_t* seq_lens, const int32_t* seq_lens_host,
                                   float softmax_scale, float tau, float tau_cov, float v_tol,
                                   float rank_tol, uint8_t* flags, uint8_t* flags_host,
                                   float* out, float* bound, uint8_t* promoted_keys,
                                   uint8_t* promoted_values, void* work, size_t work_bytes,
                                   void* host_work, size_t host_work_bytes, void* staging,
                                   size_t staging_bytes, kvq_stream_t main_stream,
                                   kvq_stream_t side_stream, int32_t timeout_ms,
                                   int32_t* num_rows, int32_t* num_flagged);

/* Size of the static device scratch of kvq_decode_attention_noalloc. */
#define KVQ_NOALLOC_SCRATCH_BYTES (16 * 1024 * 1024)

/* kvq_decode_attention for callers that cannot allocate device memory where
 * they call it (an allocator-free runtime, fixed buffers handed over by a
 * host framework, code where cudaMalloc is forbidden or would synchronize).
 * The pages have no counterpart of this entry point: it exists for such
 * callers only.  Same arguments and results as kvq_decode_attention, without
 * the workspace: the split-K scratch is a static device array of
 * KVQ_NOALLOC_SCRATCH_BYTES that every GPU loading the library holds until
 * the process exits.  Shapes whose scratch (kvq_workspace_size) exceeds it
 * return KVQ_ERR_UNSUPPORTED.  The call allocates no device memory (no
 * cudaMalloc, cudaFree or any allocating CUDA or framework routine); it clears
 * the scratch's counters with cudaMemsetAsync on `stream` before the decode.
 * Each call made outside a stream capture looks up the array's device address
 * on the current device (so a device reset, which may move it, is followed);
 * a call while `stream` is capturing uses the address the last uncaptured call
 * on that device found, so make one call on the device before any capture
 * (without one, the captured call returns KVQ_ERR_INVALID_ARG).  Every
 * call shares the one array: calls that may overlap on the GPU (on different
 * streams, or from several threads) race on it and must be serialized by the
 * caller.  Asynchronous on `stream`. */
KVQ_API int kvq_decode_attention_noalloc(const kvq_cache* cache, const void* q, int q_dtype,
                                         int32_t num_seqs, int32_t num_queries,
                                         int32_t num_q_heads, const int32_t* page_table,
                                         int32_t max_pages_per_seq, const int32_t* seq_lens,
                                         float softmax_scale, float tau, float* out,
                                         float* bound, uint8_t* flags, kvq_stream_t stream);

/* Waits for `stream`, reads *cache->error_word into *code (KVQ_OK when no
 * kernel reported an error) and resets it to KVQ_OK. */
KVQ_API int kvq_device_error(const kvq_cache* cache, kvq_stream_t stream, int32_t* code);

KVQ_API const char* kvq_status_string(int status);
KVQ_API const char* kvq_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H_ */
