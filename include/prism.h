/*
 * prism.h -- C ABI of libprism.so: the decode hot path of Prism Attention
 * ("Prism Attention: Proposal-Refined Index Sharing Mechanism for Efficient
 * LLMs Inference") on NVIDIA B200 (sm_100a).
 *
 * One decode step, per layer l (sec. 4 Overview, sec. 5.3 "Accuracy-efficiency
 * trade-off": in the "g x" setting one layer in every x is a proposal layer):
 *
 *   proposal layer:  prism_propose_append (the scorer quantizes the token's
 *                    key rows itself), or prism_quantize_k (new token rows)
 *                    -> prism_propose
 *   every layer:     prism_refine_decode on the latest pool (rescoring, top
 *                    kappa, sparse decode and merge in one launch, appending
 *                    the token's K/V rows), or prism_refine ->
 *                    prism_sparse_decode
 *
 * prism_dense_decode is the dense flash-decode over the same cache, the
 * comparison path (the pages compare against FlashAttention, sec. 5.3).
 *
 * Notation: B sequences, Hq query heads, Hkv KV heads, G = Hq / Hkv, head
 * dimension d, sequence b has L_b = cu[b+1] - cu[b] tokens, T = total_tokens
 * (>= cu[B]: rows past cu[B] are spare capacity).
 * Query head hq reads KV head hq / G.
 *
 * Layouts (row-major, all device memory unless stated):
 *   q        [B][Hq][d]          dtype of the shape (bf16 or fp32)
 *   K, V     [Hkv][T][d]         packed over sequences: sequence b occupies
 *                                 rows cu[b] .. cu[b+1]-1 of every head
 *   kq       [Hkv][T][d]  int8    k_scale [Hkv][T] fp32
 *   pool     [B][Hkv][kappa_p] int32, pool_cnt [B][Hkv] int32
 *   idx      [B][Hkv][kappa]   int32, cnt      [B][Hkv] int32
 *   out      [B][Hq][d] fp32,   lse [B][Hq] fp32 (natural log)
 * Index values are positions inside their sequence (0 <= t < L_b).  Every
 * index set is written in strictly ascending order and padded with -1 past
 * its count.
 *
 * Ownership: the caller allocates and owns every buffer.  The library never
 * allocates, frees or synchronises (prism_get_device_status excepted), keeps
 * no mutable global state, and may be called from several streams at once
 * with disjoint outputs and workspaces.  The one exception is
 * prism_sparse_decode_noalloc (end of this file), which works in a fixed
 * scratch array that the library itself holds on every device.  All work is
 * enqueued on `stream` (a cudaStream_t; NULL is the legacy default stream).
 *
 * Errors: every argument that can be checked on the host (null pointers,
 * sizes, head_dim, kappa <= kappa_p, monotone cu_seqlens_host, workspace
 * size, supported lengths) is checked before anything is enqueued; a failed
 * check returns PRISM_ERR_INVALID_ARG / _UNSUPPORTED / _WORKSPACE and
 * enqueues nothing.  A launch failure returns PRISM_ERR_CUDA.  Values that
 * live in device memory (indices, counts, token rows) are checked by the
 * kernels: an out-of-range value is skipped and recorded in the workspace
 * status word (read it with prism_get_device_status).  Inputs must be finite.
 */
#ifndef PRISM_H_
#define PRISM_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PRISM_API __attribute__((visibility("default")))
#else
#define PRISM_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum prism_dtype { PRISM_F32 = 0, PRISM_BF16 = 1 } prism_dtype;

typedef enum prism_status {
  PRISM_OK = 0,
  PRISM_ERR_INVALID_ARG = 1,
  PRISM_ERR_UNSUPPORTED = 2,
  PRISM_ERR_WORKSPACE = 3,
  PRISM_ERR_CUDA = 4,
  PRISM_ERR_TIMEOUT = 5,
  PRISM_ERR_SCRATCH_LIMIT = 6
} prism_status;

typedef enum prism_op {
  PRISM_OP_QUANTIZE = 0,
  PRISM_OP_PROPOSE = 1,
  PRISM_OP_REFINE = 2,
  PRISM_OP_SPARSE_DECODE = 3,
  PRISM_OP_DENSE_DECODE = 4,
  PRISM_OP_REFINE_DECODE = 5
} prism_op;

/* Bits of the device status word kept in every workspace. */
#define PRISM_DEV_BAD_INDEX 0x1   /* an index / token row outside its sequence */
#define PRISM_DEV_TOO_LONG  0x2   /* a row longer than the selection capacity  */
#define PRISM_DEV_TIMEOUT   0x4   /* a bounded device-side wait gave up        */

/* Shape of one layer's decode problem.  cu_seqlens_host mirrors
 * cu_seqlens_dev (B+1 entries, cu[0] = 0, non-decreasing, cu[B] <=
 * total_tokens); the host copy sizes grids and is validated, the device copy
 * is what kernels read.  total_tokens is the number of rows of every
 * per-token array ([Hkv][total_tokens][...]: K, V, kq, k_scale, INT2 codes
 * and params); rows past cu[B] are spare capacity, which a decode loop fills
 * by growing the last sequence (cu[B] += 1 per step, device copy included).
 * Kernels read the lengths from the device copy when they run, so a captured
 * CUDA graph of the decode path (prism_append_kv, prism_quantize_k,
 * prism_propose, prism_propose_append, prism_refine_decode, prism_refine,
 * prism_sparse_decode) stays valid while the last sequence grows, as long as
 * it stays within 131072 positions when the graph was captured at or below
 * that (the proposal selection then takes the same path; its cluster size is
 * planned from the longest length a row can reach, the last row counted up
 * to total_tokens).
 * prism_dense_decode sizes its split grid from the host copy,
 * which must be current for it.  head_dim is 64 or 128; num_q_heads is a
 * multiple of num_kv_heads with G <= 16; batch <= 4096. */
typedef struct prism_shape {
  int32_t batch;
  int32_t num_q_heads;
  int32_t num_kv_heads;
  int32_t head_dim;
  int32_t dtype; /* prism_dtype of q, K and V */
  const int32_t* cu_seqlens_dev;
  const int32_t* cu_seqlens_host;
  int64_t total_tokens;
} prism_shape;

/* Longest sequence (propose) and largest pool (refine) one selection row can
 * hold: 8 cooperating thread blocks x 49152 keys. */
#define PRISM_MAX_SELECT_ROW 393216

/* Bytes of workspace an operation needs for this shape and budget
 * (kappa_p / kappa are ignored where they do not apply).  Every workspace
 * starts with a 256-byte header holding the device status word; zero it once
 * (prism_clear_device_status) before first use. */
PRISM_API prism_status prism_workspace_size(const prism_shape* shape, int32_t op, int32_t kappa_p,
                                  int32_t kappa, size_t* bytes);

/*
 * Quantized key cache for proposal scoring (sec. 4.2 "Quantized Proposal
 * Construction": the key cache that proposal layers read is compressed to
 * low-bit codes; the pages' INT2 scheme is not stated, this library uses
 * symmetric per-token int8):
 *   scale[h][t] = max_j |K[h][t][j]| / 127            (IEEE fp32 division)
 *   kq[h][t][j] = clamp(round_half_even(K[h][t][j] / scale), -127, 127)
 * and scale = 0, kq = 0 for an all-zero row.
 * tok_rows: NULL quantizes all T rows of every KV head (prefill); otherwise
 * a device array of n_rows packed token indices in [0, T) (e.g. the newly
 * appended token of each sequence), quantized for every KV head.
 * ws may be NULL (no status reporting); out-of-range token rows are skipped.
 */
PRISM_API prism_status prism_quantize_k(const prism_shape* shape, const void* k, int8_t* kq,
                              float* k_scale, const int32_t* tok_rows, int32_t n_rows,
                              void* ws, size_t ws_bytes, void* stream);

/*
 * Decode-time cache update (the step either side of the method: the new
 * token's key and value join the cache before attention; the decode query
 * sits at position L_b - 1).  k_new, v_new are [B][Hkv][d] in the shape's
 * dtype; row b is written to position L_b - 1 of sequence b (packed row
 * cu[b+1] - 1) of every KV head in k_cache / v_cache.  Sequences with
 * L_b = 0 are skipped.
 */
PRISM_API prism_status prism_append_kv(const prism_shape* shape, const void* k_new,
                                       const void* v_new, void* k_cache, void* v_cache,
                                       void* stream);

/*
 * Proposal layer (sec. 4.1 "Proposal-Refined Index Sharing", sec. 4.2): for
 * every sequence b and KV head h, score every position t < L_b with the
 * quantized keys,
 *   s_t = k_scale[h][t] * max_{g<G} sum_j q[b][h*G+g][j] * kq[h][t][j],
 * and keep the top min(kappa_p, L_b) positions (higher score first, lower
 * position on ties) as the candidate pool, written ascending.
 * kappa_p is the pool size n = rho * kappa of sec. 5.1 "Implementation
 * Details".  L_b <= PRISM_MAX_SELECT_ROW.
 */
PRISM_API prism_status prism_propose(const prism_shape* shape, const void* q, const int8_t* kq,
                           const float* k_scale, int32_t kappa_p, int32_t* pool_idx,
                           int32_t* pool_cnt, void* ws, size_t ws_bytes, void* stream);

/*
 * prism_propose for a decode step whose new key rows are not in the codes
 * yet: k_new [B][Hkv][d] (the token's key rows, cache dtype) are quantized as
 * prism_quantize_k does and written to kq / k_scale at position L_b - 1 of
 * every non-empty sequence by the scorer itself, which then scores them with
 * the rest -- one launch fewer than prism_quantize_k + prism_propose, and the
 * K cache itself is not read (the new row may be appended to it later, e.g.
 * by prism_refine_decode).  Same outputs, workspace and rules as
 * prism_propose.  bf16, d = 128, G <= 8 and L_b <= 131072 only (else
 * PRISM_ERR_UNSUPPORTED); q, k_new and kq 16-byte aligned.
 * flags: PRISM_PROPOSE_SUM_GROUP selects the group-sum variant,
 *   s_t = k_scale[h][t] * sum_{g<G} sum_j q[b][h*G+g][j] * kq[h][t][j];
 * other bits are rejected (PRISM_ERR_INVALID_ARG).
 */
#define PRISM_PROPOSE_SUM_GROUP 0x1u
PRISM_API prism_status prism_propose_append(const prism_shape* shape, const void* q,
                                            const void* k_new, int8_t* kq, float* k_scale,
                                            int32_t kappa_p, int32_t* pool_idx, int32_t* pool_cnt,
                                            uint32_t flags, void* ws, size_t ws_bytes,
                                            void* stream);

/*
 * INT2 proposal keys (sec. 4.2: the pages compress the proposal layers' key
 * cache to INT2 without stating the scheme; this is the library's scheme).
 * Per KV head h, token t and group of 32 consecutive features (d = 128: four
 * groups), with lo / hi the group's min / max (-0 taken as +0):
 *   L = fp16(lo),  S = fp16((hi - L) / 3)          (round to nearest even)
 *   c_j = clamp(round_half_even((K_j - L) / S), 0, 3)   (all 0 when S = 0)
 * in IEEE fp32 arithmetic, so the dequantized key is L + S * c.
 * Layouts: codes [Hkv][T][d/4] uint8, feature f at bits 2 (f mod 4) of byte
 * f / 4; params [Hkv][T][d/32][2] uint16 holding the fp16 bits of (S, L).
 * 48 bytes per key row at d = 128 (int8: 132).  tok_rows, n_rows, ws as for
 * prism_quantize_k.  bf16 or fp32 keys, d = 64 or 128; |K| < 65504.
 */
PRISM_API prism_status prism_quantize_k_int2(const prism_shape* shape, const void* k,
                                             uint8_t* codes, uint16_t* params,
                                             const int32_t* tok_rows, int32_t n_rows, void* ws,
                                             size_t ws_bytes, void* stream);

/*
 * prism_propose on INT2 keys: per position t < L_b and query head g,
 *   score_g = sum over groups of (S * D + L * Q),
 *   D = sum_{j in group} q[g][j] * c_j,   Q = sum_{j in group} q[g][j],
 * i.e. q . (L + S c), and s_t = max_g score_g; the pool is the top
 * min(kappa_p, L_b) positions as in prism_propose.  The workspace is
 * PRISM_OP_PROPOSE's.  bf16 queries and d = 128 only (else
 * PRISM_ERR_UNSUPPORTED); L_b <= PRISM_MAX_SELECT_ROW.
 */
PRISM_API prism_status prism_propose_int2(const prism_shape* shape, const void* q,
                                          const uint8_t* codes, const uint16_t* params,
                                          int32_t kappa_p, int32_t* pool_idx, int32_t* pool_cnt,
                                          void* ws, size_t ws_bytes, void* stream);

/*
 * Refined layer (sec. 4.1; sec. 6: refined layers re-select their own top
 * kappa inside the proposed region, at a cost independent of context
 * length, sec. 5.3 "End-to-end latency"): exact scores of the pool members
 *   r_i = max_g sum_j q[b][h*G+g][j] * K[h][cu[b] + pool_i][j]   (fp32)
 * and the top min(kappa, pool_cnt) members (ties to the lower position),
 * written as ascending positions.  kappa <= kappa_p; kappa_p is the row
 * stride of pool_idx.  logits_opt, if not NULL, receives [B][Hq][kappa] the
 * unscaled dot product q_hq . K[idx] of every selected position (slot order
 * of idx); slots past cnt are left untouched.
 */
PRISM_API prism_status prism_refine(const prism_shape* shape, const void* q, const void* k,
                          const int32_t* pool_idx, const int32_t* pool_cnt, int32_t kappa_p,
                          int32_t kappa, int32_t* idx, int32_t* cnt, float* logits_opt,
                          void* ws, size_t ws_bytes, void* stream);

/*
 * Refined selection by softmax mass (sec. 4.1 and sec. 6 leave open how the
 * G query heads of a KV head share one set; this is the third reading next
 * to the maximum and the sum): for each (sequence, KV head) row and each
 * pool member i, with l_g,i = softmax_scale * q_g . K[pool_i] (the exact fp32
 * per-head score),
 *   r_i = sum_g exp(l_g,i - max_i' l_g,i') / sum_i' exp(l_g,i' - max_i' l_g,i'),
 * the attention mass the group puts on the member, each head's softmax over
 * the pool.  idx / cnt as prism_refine: the top min(kappa, n) members by r_i,
 * ties to the lower pool slot, positions ascending, -1 padded.  The masses
 * are fp32 (the oracle's fp64), so sets agree with it up to near-ties.
 * Workspace: PRISM_OP_REFINE with the same kappa_p, kappa.  softmax_scale
 * finite and > 0 (else PRISM_ERR_INVALID_ARG); other errors as prism_refine.
 */
PRISM_API prism_status prism_refine_mass(const prism_shape* shape, const void* q, const void* k,
                                         const int32_t* pool_idx, const int32_t* pool_cnt,
                                         int32_t kappa_p, int32_t kappa, float softmax_scale,
                                         int32_t* idx, int32_t* cnt, void* ws, size_t ws_bytes,
                                         void* stream);

/*
 * Selection granularity (sec. 4.1 shares index sets under GQA without saying
 * at which granularity; sec. 3 analyses attention per head; sec. 2 "Related
 * Work" names a set shared by all heads).  The plain calls use one pool and
 * one set per (sequence, KV head), the scores of its G query heads combined
 * by their maximum.  The _ex calls take `sets`:
 *   PRISM_SETS_KV_HEAD   that default (the _ex calls forward to the plain ones);
 *   PRISM_SETS_Q_HEAD    the pool stays per (sequence, KV head); each query
 *                        head keeps its own top kappa of that pool by its own
 *                        exact score q_hq . K and attends over it: idx / cnt
 *                        are [B][Hq][kappa] / [B][Hq];
 *   PRISM_SETS_SEQUENCE  one pool and one set per sequence, shared by every
 *                        head: a position's score is the maximum over all KV
 *                        heads of the per-KV-head score; pool / pool_cnt are
 *                        [B][kappa_p] / [B], idx / cnt [B][kappa] / [B], and
 *                        every query head attends over the sequence's set
 *                        with its own KV head's rows.
 * Workspaces are those of the plain calls (prism_workspace_size covers every
 * granularity).  Other `sets` values: PRISM_ERR_INVALID_ARG.
 */
#define PRISM_SETS_KV_HEAD 0u
#define PRISM_SETS_Q_HEAD 1u
#define PRISM_SETS_SEQUENCE 2u
PRISM_API prism_status prism_propose_ex(const prism_shape* shape, const void* q, const int8_t* kq,
                                        const float* k_scale, int32_t kappa_p, int32_t* pool_idx,
                                        int32_t* pool_cnt, uint32_t sets, void* ws,
                                        size_t ws_bytes, void* stream);
PRISM_API prism_status prism_refine_ex(const prism_shape* shape, const void* q, const void* k,
                                       const int32_t* pool_idx, const int32_t* pool_cnt,
                                       int32_t kappa_p, int32_t kappa, int32_t* idx, int32_t* cnt,
                                       uint32_t sets, void* ws, size_t ws_bytes, void* stream);
PRISM_API prism_status prism_sparse_decode_ex(const prism_shape* shape, const void* q,
                                              const void* k, const void* v, const int32_t* idx,
                                              const int32_t* cnt, int32_t kappa,
                                              float softmax_scale, uint32_t sets, float* out,
                                              float* lse_opt, void* ws, size_t ws_bytes,
                                              void* stream);

/*
 * The proposal layer's own index set under the other reading of sec. 4.1
 * (refined layers re-select inside the pool; what the proposal layer itself
 * attends over is not stated): the top min(kappa, pool_cnt) members of the
 * pool by the proposal scores the proposal call just computed -- no exact
 * rescoring -- written as ascending positions to idx [B][Hkv][kappa] and cnt
 * [B][Hkv] (ties to the lower position).  The default reading is
 * prism_refine / prism_refine_decode on the proposal layer's own pool.
 * propose_ws is the workspace of the prism_propose, prism_propose_append or
 * prism_propose_int2 call that produced pool_idx / pool_cnt, on the same
 * stream and shape, with no call on that workspace in between (its scores
 * are read); ws is sized by PRISM_OP_REFINE for (kappa_p, kappa).  Follow
 * with prism_sparse_decode on idx for the layer's attention.
 */
PRISM_API prism_status prism_propose_topk(const prism_shape* shape, const void* propose_ws,
                                          size_t propose_ws_bytes, const int32_t* pool_idx,
                                          const int32_t* pool_cnt, int32_t kappa_p, int32_t kappa,
                                          int32_t* idx, int32_t* cnt, void* ws, size_t ws_bytes,
                                          void* stream);

/*
 * Token-level sparse attention over the selected rows (sec. 1, sec. 2.1):
 * for every query head hq of sequence b, with h = hq / G and the rows
 * t in idx[b][h][0 .. cnt[b][h]),
 *   l_t = softmax_scale * q[b][hq] . K[h][cu[b]+t],
 *   out[b][hq] = sum_t softmax(l)_t V[h][cu[b]+t],   lse = log sum_t exp(l_t).
 * Split-K over the index list with a log-sum-exp merge.  An empty set gives
 * out = 0 and lse = -inf.  kappa is the row stride of idx.
 */
PRISM_API prism_status prism_sparse_decode(const prism_shape* shape, const void* q, const void* k,
                                 const void* v, const int32_t* idx, const int32_t* cnt,
                                 int32_t kappa, float softmax_scale, float* out, float* lse_opt,
                                 void* ws, size_t ws_bytes, void* stream);

/*
 * A refined layer in one call: prism_refine followed by prism_sparse_decode
 * on its result, with the same outputs (idx, cnt, out, lse_opt) and the same
 * definitions.  The exact scores, the selection and the attention partials
 * stay on chip (one thread-block cluster of up to 16 CTAs per sequence and
 * KV head), so the workspace is only the 256-byte status header
 * (PRISM_OP_REFINE_DECODE), and the key rows of the pool are read once.
 * Returns PRISM_ERR_UNSUPPORTED when a pool of kappa_p members does not fit
 * on chip (kappa_p > 65535, or more than 16 x 3328 members at G <= 4,
 * d = 128); use the two calls then.
 *
 * k_new_opt / v_new_opt, if not NULL, are this token's key and value rows,
 * [B][Hkv][d] in the cache dtype: the call first appends them at position
 * L_b - 1 of every sequence (as prism_append_kv would; k and v are written
 * there) and every read of that position uses them.  NULL: the caches
 * already hold the rows, and k and v are only read.
 *
 * k_prefetch, if not NULL, is the key cache ([Hkv][T][d], same shape) of the
 * next layer that will be refined on the same pool: once this layer's key
 * rows are consumed, the same pool rows of k_prefetch are prefetched into L2
 * (a hint; results do not depend on it).
 *
 * flags: PRISM_RD_OVERLAP lets the launch begin while the previous kernel on
 * `stream` is still running (programmatic dependent launch).  Until that
 * kernel ends the call reads only cu_seqlens_dev, pool_idx, pool_cnt and the
 * key rows at pool positions other than L_b - 1, and writes nothing but the
 * status word; it touches q, v, k_new_opt, v_new_opt and its outputs only
 * afterwards.  Set it only when the previous kernel writes none of the
 * former (e.g. the refined layer before this one, on the same pool).
 * PRISM_RD_SUM_GROUP selects the group-sum variant of the exact score:
 * r_i = sum_g sum_j q[g][j] * K[pool_i][j] in place of the maximum over g
 * (the selection and the attention are unchanged).  PRISM_RD_MASS selects
 * by the group's softmax mass over the pool, as prism_refine_mass at
 * softmax_scale (not with PRISM_RD_SUM_GROUP: PRISM_ERR_INVALID_ARG).
 */
#define PRISM_RD_OVERLAP 0x1u
#define PRISM_RD_SUM_GROUP 0x2u
#define PRISM_RD_MASS 0x4u
PRISM_API prism_status prism_refine_decode(const prism_shape* shape, const void* q, void* k,
                                           void* v, const int32_t* pool_idx,
                                           const int32_t* pool_cnt, int32_t kappa_p,
                                           int32_t kappa, float softmax_scale, int32_t* idx,
                                           int32_t* cnt, float* out, float* lse_opt,
                                           const void* k_new_opt, const void* v_new_opt,
                                           const void* k_prefetch, uint32_t flags, void* ws,
                                           size_t ws_bytes, void* stream);

/*
 * Dense decode attention over every position t < L_b (the comparison path):
 * the same definition as prism_sparse_decode with idx = 0 .. L_b - 1.  A
 * bf16 cache with up to 8 query heads per KV head runs on tensor cores,
 * split along t by a plan made from every sequence's length (host copy of
 * cu_seqlens): the workspace (prism_workspace_size, PRISM_OP_DENSE_DECODE)
 * must be sized with the lengths of the call.  q, k and v 16-byte aligned.
 */
PRISM_API prism_status prism_dense_decode(const prism_shape* shape, const void* q, const void* k,
                                const void* v, float softmax_scale, float* out, float* lse_opt,
                                void* ws, size_t ws_bytes, void* stream);

/*
 * Index overlap of two selections, per row (sec. 3 "Observations", Figure 1:
 * the overlap ratio between a reference layer's index set and the set of a
 * layer at some offset; Figure 12: the share of one layer's top-kappa that an
 * expanded top-rho*kappa set of another layer covers).  A diagnostic outside
 * the decode step.  a [rows][stride_a] and b [rows][stride_b] are device
 * index sets, row r holding cnt_a[r] / cnt_b[r] members (clamped to
 * [0, stride]) in strictly ascending order, as every selection of this
 * library is written; out[r] = |a_r intersect b_r| (device int32 [rows]).
 * Rows whose lists are not ascending give an unspecified count (no memory
 * outside the rows is read).  rows = 0 enqueues nothing.
 */
PRISM_API prism_status prism_index_overlap(int32_t rows, const int32_t* a, const int32_t* cnt_a,
                                           int32_t stride_a, const int32_t* b,
                                           const int32_t* cnt_b, int32_t stride_b, int32_t* out,
                                           void* stream);

/* Zero the workspace header (status word) on `stream`. */
PRISM_API prism_status prism_clear_device_status(void* ws, size_t ws_bytes, void* stream);

/* Read the status word (PRISM_DEV_* bits) after the work on `stream` ends.
 * This call synchronises `stream`. */
PRISM_API prism_status prism_get_device_status(const void* ws, size_t ws_bytes, void* stream,
                                     int32_t* code);

/* Static description of a status code. */
PRISM_API const char* prism_status_str(prism_status s);

/*
 * No-allocation variant of prism_sparse_decode.  The paper has no
 * counterpart to this entry point: it exists for callers that cannot hand
 * the library a workspace, because they may not allocate device memory at
 * the point of the call -- code that runs inside a memory pool it does not
 * own, an allocator callback, or an engine whose device memory is fixed
 * once at start-up.  It computes exactly what prism_sparse_decode computes
 * (same kernels, same split plan, same summation order), but keeps the
 * split-K partial results in a scratch array that the library declares at
 * file scope: PRISM_NOALLOC_SCRATCH_BYTES (4 MiB) of device memory, held by
 * every GPU that loads the library until the process exits.
 *
 * Arguments are those of prism_sparse_decode, except that the workspace is
 * replaced by status_dev: a caller-owned device int32 into which the
 * kernels OR the PRISM_DEV_* bits of any bad index or count they meet (the
 * caller zeroes it and reads it back).  It must not be NULL.
 *
 * The call allocates nothing: no cudaMalloc, no cudaFree, no allocating
 * library routine.  Its first call on a device, with that device current,
 * looks up the device address of the scratch array (cudaGetSymbolAddress),
 * which may load the library's device code onto that device; make that
 * first call before any stream capture begins.
 *
 * A request whose partial results need more than the scratch holds
 * (B * Hq * splits * (d + 2) * 4 bytes, rounded up) returns
 * PRISM_ERR_SCRATCH_LIMIT and enqueues nothing.  Every call on a device
 * shares the one array, and the array keeps the last call's contents (every
 * partial a call reads is first written by that call).  Calls whose work
 * overlaps on the GPU -- on different streams, or from different host
 * threads -- race on the array and give wrong results: serialise them.
 */
#define PRISM_NOALLOC_SCRATCH_BYTES (4u << 20)
PRISM_API prism_status prism_sparse_decode_noalloc(const prism_shape* shape, const void* q,
                                                   const void* k, const void* v,
                                                   const int32_t* idx, const int32_t* cnt,
                                                   int32_t kappa, float softmax_scale, float* out,
                                                   float* lse_opt, int32_t* status_dev,
                                                   void* stream);

#ifdef __cplusplus
}
#endif

#endif /* PRISM_H_ */
