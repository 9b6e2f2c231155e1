// Internal launchers of libprism (host side).  Arguments are validated by
// the C ABI layer (prism_api.cu) before any of these is called.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace prism {

// Workspace header: the first 256 bytes of every workspace (status word).
constexpr size_t kWsHeader = 256;

struct Dims {
  int B, Hq, Hkv, G, D;
  int64_t T;
  bool bf16;
  const int32_t* cu_dev;
  const int32_t* cu_host;
  int max_len;  // max_b L_b (from the host mirror)
  int num_sms;
};

// Query-group sizes a kernel is instantiated for; a group of G query heads
// runs on the smallest instantiation >= G with the extra heads masked.
inline int padded_group(int G) { return G <= 1 ? 1 : G <= 2 ? 2 : G <= 4 ? 4 : G <= 8 ? 8 : 16; }

// cuTensorMapEncodeTiled from the driver, looked up once (null if missing)
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

cudaError_t launch_append(const Dims& d, const void* k_new, const void* v_new, void* k_cache,
                          void* v_cache, cudaStream_t st);

cudaError_t launch_quantize(const Dims& d, const void* k, int8_t* kq, float* scale,
                            const int32_t* tok_rows, int64_t n_rows, int32_t* status,
                            cudaStream_t st);
// INT2 codes [Hkv][T][d/4] (four per byte) and (step, zero point) fp16 bits
// [Hkv][T][d/32][2] of the listed token rows (quantize.cu).
cudaError_t launch_quantize_int2(const Dims& d, const void* k, uint8_t* codes, uint16_t* params,
                                 const int32_t* tok_rows, int64_t n_rows, int32_t* status,
                                 cudaStream_t st);

// Proposal scores s[h][t] (fp32, [Hkv][T]).  use_mma selects the tensor-core
// (mma.sync, fp16 operands) scorer, valid for bf16 queries only.
// hist (optional, mma scorer only): [B*Hkv][4096] first-digit histogram of
// ord(score), added to (the caller clears it).
cudaError_t launch_propose_scores(const Dims& d, const void* q, const int8_t* kq,
                                  const float* scale, float* scores, uint32_t* hist, bool use_mma,
                                  int32_t* status, cudaStream_t st);
// INT2 proposal scores from packed codes and (step, zero point) pairs, with
// the first-digit histogram (bf16 queries, d = 128; score.cu).
// The integer scorer with this token's key rows k_new [B][Hkv][d] (bf16),
// quantized by the scorer into kq / scale at position L_b - 1 of every
// non-empty sequence before that position is scored; sum_group: the
// selection score sums the group's query heads instead of taking their
// maximum.  bf16, d = 128, G <= 8 only (cudaErrorInvalidValue otherwise).
cudaError_t launch_propose_scores_new_rows(const Dims& d, const void* q, int8_t* kq, float* scale,
                                           const void* k_new, float* scores, uint32_t* hist,
                                           bool sum_group, int32_t* status, cudaStream_t st);
cudaError_t launch_propose_scores_int2(const Dims& d, const void* q, const uint8_t* codes,
                                       const uint16_t* params, float* scores, uint32_t* hist,
                                       int32_t* status, cudaStream_t st);

// Cluster radix top-k.  mode 0 (propose): keys scores[h][cu[b] + i], row
// length L_b, output position i.  mode 1 (refine): keys r[row][i], row length
// pool_cnt[row], output position pool[row][i]; dots/logits optional.
struct SelectArgs {
  int mode;
  int Hkv, G, Hq;
  int64_t T;
  const int32_t* cu;
  const float* keys;
  const int32_t* pool;
  const int32_t* pool_cnt;
  int pool_stride;
  int k_req;
  int32_t* out;
  int32_t* out_cnt;
  const float* dots;
  float* logits;
  int32_t* status;
  int pool_div;  // mode 1: pool row = row / pool_div (0 or 1: the row itself)
};
int select_capacity_per_row();  // longest row one cluster can select from

// Proposal-layer selection from the scorer's first-digit histogram (see
// propose_select.cu); rows up to propose_select_max_row() positions.
int propose_select_cluster(const Dims& d);
int propose_select_max_row();
cudaError_t launch_propose_select(const Dims& d, const float* scores, const uint32_t* hist,
                                  int kappa_p, int32_t* pool, int32_t* pool_cnt, int32_t* status,
                                  cudaStream_t st);
cudaError_t launch_select(const Dims& d, const SelectArgs& a, int max_row_len, cudaStream_t st);

// Exact pool scores r[row][i] = max_g q_g . K[pool_i] (+ per-head dots);
// row (b, h) reads pool row (b * Hkv + h) / pool_div (pool_div = Hkv: one
// pool per sequence shared by its KV heads).
// Softmax mass of every pool member over the G query heads of its row, in
// place of r (refine.cu); dots [rows][G][pool_stride] from launch_refine_scores.
cudaError_t launch_refine_mass(const Dims& d, float* r, const float* dots, const int32_t* pool_cnt,
                               int pool_stride, float softmax_scale, cudaStream_t st);
cudaError_t launch_refine_scores(const Dims& d, const void* q, const void* k, const int32_t* pool,
                                 const int32_t* pool_cnt, int pool_stride, float* r, float* dots,
                                 int32_t* status, cudaStream_t st, int pool_div = 1);
// out[o][i] = max_h in[(o * H + h) * inner + i] over h < H, for o < outer,
// i < inner (the maximum of per-head scores over the heads; sets.cu).
cudaError_t launch_head_max(const float* in, int H, int64_t outer, int64_t inner, float* out,
                            cudaStream_t st);

// Proposal scores of the pool members: r[row][i] = scores[h][cu[b] + pool[row][i]].
cudaError_t launch_pool_gather(const Dims& d, const float* scores, const int32_t* pool,
                               const int32_t* pool_cnt, int pool_stride, float* r, int32_t* status,
                               cudaStream_t st);

// Fused refine -> top-kappa -> sparse decode, one cluster of `cluster` CTAs
// per (sequence, KV head); mc = pool members per CTA.  ok = false when the
// pool does not fit on chip.
struct RefineDecodePlan {
  int cluster;
  int mc;
  bool ok;
  bool inplace;  // the softmax weights replace the logits (no separate weight array)
};
RefineDecodePlan plan_refine_decode(const Dims& d, int kappa_p);
cudaError_t launch_refine_decode(const Dims& d, const RefineDecodePlan& p, const void* q,
                                 const void* k, const void* v, const void* k_new,
                                 const void* v_new, const void* k_next, const int32_t* pool,
                                 const int32_t* pool_cnt, int kappa_p, int kappa,
                                 float softmax_scale, int32_t* idx, int32_t* cnt, float* out,
                                 float* lse, int32_t* status, bool overlap, int agg,
                                 cudaStream_t st);

// Split-K attention partials over idx rows (idx == nullptr: every position).
struct AttendPlan {
  int splits;
  int per_split;
};
AttendPlan plan_attend(const Dims& d, int64_t max_rows_per_seq, bool dense);
// kv_div: row (b, h) of d reads K/V head h / kv_div (d.Hkv = Hq, G = 1 for
// one set per query head); idx_div: it reads idx / cnt row (b Hkv + h) /
// idx_div (idx_div = Hkv for one set per sequence).
cudaError_t launch_attend(const Dims& d, const AttendPlan& p, const void* q, const void* k,
                          const void* v, const int32_t* idx, const int32_t* cnt, int idx_stride,
                          float softmax_scale, float* part_o, float* part_ml, float* out,
                          float* lse, int32_t* status, cudaStream_t st, int kv_div = 1,
                          int idx_div = 1);

// |a_row intersect b_row| per row of two ascending index-set arrays
// (overlap.cu); counts are clamped to [0, stride].
cudaError_t launch_overlap(int rows, const int32_t* a, const int32_t* cnt_a, int stride_a,
                           const int32_t* b, const int32_t* cnt_b, int stride_b, int32_t* out,
                           cudaStream_t st);

}  // namespace prism
