// C ABI of libprism.so (declared in include/prism.h): argument validation,
// workspace layout and kernel dispatch.  Nothing here allocates device
// memory or synchronises (prism_get_device_status excepted).
#include <cuda_runtime.h>

#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "../../include/prism.h"
#include "kernels.h"

namespace prism {
namespace {

// Split plans are sized for B200's 148 SMs on every device, so workspace
// sizes (and the summation order of split-K) do not depend on the GPU.
constexpr int kPlanSms = 148;
constexpr int kMaxBatch = 4096;
constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

prism_status check_shape(const prism_shape* s, Dims* d) {
  if (!s || !s->cu_seqlens_dev || !s->cu_seqlens_host) return PRISM_ERR_INVALID_ARG;
  if (s->batch < 1 || s->batch > kMaxBatch) return PRISM_ERR_INVALID_ARG;
  if (s->num_kv_heads < 1 || s->num_q_heads < s->num_kv_heads) return PRISM_ERR_INVALID_ARG;
  if (s->num_q_heads % s->num_kv_heads != 0) return PRISM_ERR_INVALID_ARG;
  if (s->num_q_heads / s->num_kv_heads > 16) return PRISM_ERR_UNSUPPORTED;
  if (s->head_dim != 64 && s->head_dim != 128) return PRISM_ERR_UNSUPPORTED;
  if (s->dtype != PRISM_F32 && s->dtype != PRISM_BF16) return PRISM_ERR_INVALID_ARG;
  if (s->total_tokens < 0) return PRISM_ERR_INVALID_ARG;
  const int32_t* cu = s->cu_seqlens_host;
  if (cu[0] != 0) return PRISM_ERR_INVALID_ARG;
  int max_len = 0;
  for (int b = 0; b < s->batch; ++b) {
    if (cu[b + 1] < cu[b]) return PRISM_ERR_INVALID_ARG;
    const int L = cu[b + 1] - cu[b];
    if (L > max_len) max_len = L;
  }
  if ((int64_t)cu[s->batch] > s->total_tokens) return PRISM_ERR_INVALID_ARG;  // spare rows allowed
  d->B = s->batch;
  d->Hq = s->num_q_heads;
  d->Hkv = s->num_kv_heads;
  d->G = s->num_q_heads / s->num_kv_heads;
  d->D = s->head_dim;
  d->T = s->total_tokens;
  d->bf16 = s->dtype == PRISM_BF16;
  d->cu_dev = s->cu_seqlens_dev;
  d->cu_host = s->cu_seqlens_host;
  d->max_len = max_len;
  d->num_sms = kPlanSms;
  return PRISM_OK;
}

prism_status set_live_sms(Dims* d) {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PRISM_ERR_CUDA;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return PRISM_ERR_CUDA;
  d->num_sms = n > 0 ? n : kPlanSms;
  return PRISM_OK;
}

prism_status cuda_status(cudaError_t e) { return e == cudaSuccess ? PRISM_OK : PRISM_ERR_CUDA; }

// Workspace layout per operation (offsets after the 256-byte header).
struct Layout {
  size_t a = 0, b = 0, c = 0, d = 0, e = 0, total = 0;  // array offsets
};

Layout layout(const Dims& d, int op, int kappa_p, int kappa) {
  Layout L;
  size_t off = kWsHeader;
  const size_t rows = (size_t)d.B * d.Hkv;
  switch (op) {
    case PRISM_OP_QUANTIZE:
      break;
    case PRISM_OP_PROPOSE:  // scores [Hkv][T] fp32, first-digit histogram [rows][4096] u32,
                            // per-sequence head maxima [T] fp32
      L.a = off;
      off = align_up(off + (size_t)d.Hkv * (size_t)d.T * sizeof(float));
      L.b = off;
      off = align_up(off + rows * 4096 * 4);
      L.c = off;
      off = align_up(off + (size_t)d.T * sizeof(float));
      break;
    case PRISM_OP_REFINE:  // r [rows][kappa_p], dots [rows][G][kappa_p], head maxima [B][kappa_p]
      L.a = off;
      off = align_up(off + rows * (size_t)kappa_p * sizeof(float));
      L.b = off;
      off = align_up(off + rows * (size_t)d.G * (size_t)kappa_p * sizeof(float));
      L.c = off;
      off = align_up(off + (size_t)d.B * (size_t)kappa_p * sizeof(float));
      break;
    case PRISM_OP_SPARSE_DECODE:
    case PRISM_OP_DENSE_DECODE: {
      const AttendPlan p = plan_attend(d, op == PRISM_OP_SPARSE_DECODE ? kappa : d.max_len,
                                      op == PRISM_OP_DENSE_DECODE);
      const size_t parts = (size_t)d.B * d.Hq * (size_t)p.splits;
      L.a = off;  // partial o [B][Hq][splits][D]
      off = align_up(off + parts * (size_t)d.D * sizeof(float));
      L.b = off;  // partial (m, l) [B][Hq][splits][2]
      off = align_up(off + parts * 2 * sizeof(float));
      break;
    }
    default:
      break;
  }
  L.total = off;
  (void)kappa;
  return L;
}

bool ws_ok(const void* ws, size_t ws_bytes, const Layout& L) {
  return ws && ws_bytes >= L.total && ((uintptr_t)ws % kAlign) == 0;
}

bool use_mma_scorer() {
  const char* e = std::getenv("PRISM_PROPOSE_SCORER");
  return !(e && std::strcmp(e, "simt") == 0);
}

}  // namespace
}  // namespace prism

using namespace prism;

extern "C" {

prism_status prism_workspace_size(const prism_shape* shape, int32_t op, int32_t kappa_p,
                                  int32_t kappa, size_t* bytes) {
  Dims d;
  prism_status s = check_shape(shape, &d);
  if (s != PRISM_OK) return s;
  if (!bytes || op < PRISM_OP_QUANTIZE || op > PRISM_OP_REFINE_DECODE) return PRISM_ERR_INVALID_ARG;
  if (op == PRISM_OP_PROPOSE && kappa_p < 1) return PRISM_ERR_INVALID_ARG;
  if ((op == PRISM_OP_REFINE || op == PRISM_OP_REFINE_DECODE) &&
      (kappa_p < 1 || kappa < 1 || kappa > kappa_p))
    return PRISM_ERR_INVALID_ARG;
  if (op == PRISM_OP_SPARSE_DECODE && kappa < 1) return PRISM_ERR_INVALID_ARG;
  *bytes = layout(d, op, kappa_p, kappa).total;
  return PRISM_OK;
}

prism_status prism_append_kv(const prism_shape* shape, const void* k_new, const void* v_new,
                             void* k_cache, void* v_cache, void* stream) {
  Dims d;
  prism_status s = check_shape(shape, &d);
  if (s != PRISM_OK) return s;
  if (!k_new || !v_new || !k_cache || !v_cache) return PRISM_ERR_INVALID_ARG;
  const uintptr_t all = (uintptr_t)k_new | (uintptr_t)v_new | (uintptr_t)k_cache | (uintptr_t)v_cache;
  if (all % 16 != 0) return PRISM_ERR_INVALID_ARG;
  return cuda_status(launch_append(d, k_new, v_new, k_cache, v_cache, static_cast<cudaStream_t>(stream)));
}

prism_status prism_quantize_k(const prism_shape* shape, const void* k, int8_t* kq, float* k_scale,
                              const int32_t* tok_rows, int32_t n_rows, void* ws, size_t ws_bytes,
                              void* stream) {
  Dims d;
  prism_status s = check_shape(shape, &d);
  if (s != PRISM_OK) return s;
  if (!k || !kq || !k_scale) return PRISM_ERR_INVALID_ARG;
  if (tok_rows && n_rows < 0) return PRISM_ERR_INVALID_ARG;
  if (ws && (ws_bytes < kWsHeader || ((uintptr_t)ws % kAlign) != 0)) return PRISM_ERR_WORKSPACE;
  if ((s = set_live_sms(&d)) != PRISM_OK) return s;
  const int64_t rows = tok_rows ? (int64_t)n_rows : d.T;
  return cuda_status(launch_quantize(d, k, kq, k_scale, tok_rows, rows, static_cast<int32_t*>(ws),
                                     static_cast<cudaStream_t>(stream)));
}

prism_status prism_propose(const prism_shape* shape, const void* q, const int8_t* kq,
                           const float* k_scale, int32_t kappa_p, int32_t* pool_idx,
                           int32_t* pool_cnt, void* ws, size_t ws_bytes, void* stream) {
  Dims d;
  prism_status s = check_shape(shape, &d);
  if (s != PRISM_OK) return s;
  if (!q || !kq || !k_scale || !pool_idx || !pool_cnt || kappa_p < 1) return PRISM_ERR_INVALID_ARG;
  if (d.max_len > select_capacity_per_row()) return PRISM_ERR_UNSUPPORTED;
  const Layout L = layout(d, PRISM_OP_PROPOSE, kappa_p, 0);
  if (!ws_ok(ws, ws_bytes, L)) return PRISM_ERR_WORKSPACE;
  if ((s = set_live_sms(&d)) != PRISM_OK) return s;
  char* w = static_cast<char*>(ws);
  int32_t* status = reinterpret_cast<int32_t*>(w);
  float* scores = reinterpret_cast<float*>(w + L.a);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const bool mma = use_mma_scorer() && d.bf16;
  if (mma && d.max_len <= propose_select_max_row()) {
    // scorer builds the first-digit histogram; selection resolves from it
    uint32_t* hist = reinterpret_cast<uint32_t*>(w + L.b);
    const size_t rows = (size_t)d.B * d.Hkv;
    if (cudaMemsetAsync(hist, 0, rows * 4096 * 4, st) != cudaSuccess) return PRISM_ERR_CUDA;
    cudaError_t e = launch_propose_scores(d, q, kq, k_scale, scores, hist, true, status, st);
    if (e != cudaSuccess) return PRISM_ERR_CUDA;
    return cuda_status(launch_propose_select(d, scores, hist, kappa_p, pool_idx, pool_cnt, status, st));
  }
  cudaError_t e = launch_propose_scores(d, q, kq, k_scale, scores, nullptr, mma, status, st);
  if (e != cudaSuccess) return PRISM_ERR_CUDA;
  SelectArgs a{};
  a.mode = 0;
  a.Hkv = d.Hkv;
  a.G = d.G;
  a.Hq = d.Hq;
  a.T = d.T;
  a.cu = d.cu_dev;
  a.keys = scores;
  a.k_req = kappa_p;
  a.out = pool_idx;
  a.out_cnt = pool_cnt;
  a.status = status;
  return cuda_status(launch_select(d, a, d.max_len, st));
}

prism_status prism_propose_append(const prism_shape* shape, const void* q, const void* k_new,
                                  int8_t* kq, float* k_scale, int32_t kappa_p, int32_t* pool_idx,
                                  int32_t* pool_cnt, uint32_t flags, void* ws, size_t ws_bytes,
                                  void* stream) {
  Dims d;
  prism_status s = check_shape(shape, &d);
  if (s != PRISM_OK) return s;
  if (!q || !k_new || !kq || !k_scale || !pool_idx || !pool_cnt || kappa_p < 1)
    return PRISM_ERR_INVALID_ARG;
  if (flags & ~PRISM_PROPOSE_SUM_GROUP) return PRISM_ERR_INVALID_ARG;
  if (!d.bf16 || d.D != 128 || d.G > 8 || d.max_len > propose_select_max_row())
    return PRISM_ERR_UNSUPPORTED;
  if (((uintptr_t)q | (uintptr_t)k_new | (uintptr_t)kq) % 16) return PRISM_ERR_INVALID_ARG;
  const Layout L = layout(d, PRISM_OP_PROPOSE, kappa_p, 0);
  if (!ws_ok(ws, ws_bytes, L)) return PRISM_ERR_WORKSPACE;
  if ((s = set_live_sms(&d)) != PRISM_OK) return s;
  char* w = static_cast<char*>(ws);
  int32_t* status = reinterpret_cast<int32_t*>(w);
  float* scores = reinterpret_cast<float*>(w + L.a);
  uint32_t* hist = reinterpret_cast<uint32_t*>(w + L.b);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t rows = (size_t)d.B * d.Hkv;
  if (cudaMemsetAsync(hist, 0, rows * 4096 * 4, st) != cudaSuccess) return PRISM_ERR_CUDA;
  cudaError_t e = launch_propose_scores_new_rows(d, q, kq, k_scale, k_new, scores, hist,
                                                 (flags & PRISM_PROPOSE_SUM_GROUP) != 0, status, st);
  if (e == cudaErrorInvalidValue) return PRISM_ERR_UNSUPPORTED;
  if (e != cudaSuccess) return PRISM_ERR_CUDA;
  return cuda_status(launch_propose_select(d, scores, hist, kappa_p, pool_idx, pool_cnt, status, st));
}

prism_status prism_quantize_k_int2(const prism_shape* shape, const void* k, uint8_t* codes,
                                   uint16_t* params, const int32_t* tok_rows, int32_t n_rows,
                                   void* ws, size_t ws_bytes, void* stream) {
  Dims d;
  prism_status s = check_shape(shape, &d);
  if (s != PRISM_OK) return s;
  if (!k || !codes || !params) return PRISM_ERR_INVALID_ARG;
  if (tok_rows && n_rows < 0) return PRISM_ERR_INVALID_ARG;
  if (ws && (ws_bytes < kWsHeader || ((uintptr_t)ws % kAlign) != 0)) return PRISM_ERR_WORKSPACE;
  if ((s = set_live_sms(&d)) != PRISM_OK) return s;
  const int64_t rows = tok_rows ? (int64_t)n_rows : d.T;
  return cuda_status(launch_quantize_int2(d, k, codes, params, tok_rows, rows,
                                          static_cast<int32_t*>(ws), static_cast<cudaStream_t>(stream)));
}

prism_status prism_propose_int2(const prism_shape* shape, const void* q, const uint8_t* codes,
                                const uint16_t* params, int32_t kappa_p, int32_t* pool_idx,
                                int32_t* pool_cnt, void* ws, size_t ws_bytes, void* stream) {
  Dims d;
  prism_status s = check_shape(shape, &d);
  if (s != PRISM_OK) return s;
  if (!q || !codes || !params || !pool_idx || !pool_cnt || kappa_p < 1) return PRISM_ERR_INVALID_ARG;
  if (!d.bf16 || d.D != 128) return PRISM_ERR_UNSUPPORTED;
  if (((uintptr_t)codes | (uintptr_t)params) % 16) return PRISM_ERR_INVALID_ARG;
  if (d.max_len > select_capacity_per_row()) return PRISM_ERR_UNSUPPORTED;
  const Layout L = layout(d, PRISM_OP_PROPOSE, kappa_p, 0);
  if (!ws_ok(ws, ws_bytes, L)) return PRISM_ERR_WORKSPACE;
  if ((s = set_live_sms(&d)) != PRISM_OK) return s;
  char* w = static_cast<char*>(ws);
  int32_t* status = reinterpret_cast<int32_t*>(w);
  float* scores = reinterpret_cast<float*>(w + L.a);
  uint32_t* hist = reinterpret_cast<uint32_t*>(w + L.b);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t rows = (size_t)d.B * d.Hkv;
  if (cudaMemsetAsync(hist, 0, rows * 4096 * 4, st) != cudaSuccess) return PRISM_ERR_CUDA;
  cudaError_t e = launch_propose_scores_int2(d, q, codes, params, scores, hist, status, st);
  if (e != cudaSuccess) return PRISM_ERR_CUDA;
  if (d.max_len <= propose_select_max_row())
    return cuda_status(launch_propose_select(d, scores, hist, kappa_p, pool_idx, pool_cnt, status, st));
  SelectArgs a{};
  a.mode = 0;
  a.Hkv = d.Hkv;
  a.G = d.G;
  a.Hq = d.Hq;
  a.T = d.T;
  a.cu = d.cu_dev;
  a.keys = scores;
  a.k_req = kappa_p;
  a.out = pool_idx;
  a.out_cnt = pool_cnt;
  a.status = status;
  return cuda_status(launch_select(d, a, d.max_len, st));
}

prism_status prism_refine(const prism_shape* shape, const void* q, const void* k,
                          const int32_t* pool_idx, const int32_t* pool_cnt, int32_t kappa_p,
                          int32_t kappa, int32_t* idx, int32_t* cnt, float* logits_opt, void* ws,
                          size_t ws_bytes, void* stream) {
  Dims d;
  prism_status s = check_shape(shape, &d);
  if (s != PRISM_OK) return s;
  if (!q || !k || !pool_idx || !pool_cnt || !idx || !cnt) return PRISM_ERR_INVALID_ARG;
  if (kappa_p < 1 || kappa < 1 || kappa > kappa_p) return PRISM_ERR_INVALID_ARG;
  if (kappa_p > select_capacity_per_row()) return PRISM_ERR_UNSUPPORTED;
  const Layout L = layout(d, PRISM_OP_REFINE, kappa_p, kappa);
  if (!ws_ok(ws, ws_bytes, L)) return PRISM_ERR_WORKSPACE;
  if ((s = set_live_sms(&d)) != PRISM_OK) return s;
  char* w = static_cast<char*>(ws);
  int32_t* status = reinterpret_cast<int32_t*>(w);
  float* r = reinterpret_cast<float*>(w + L.a);
  float* dots = logits_opt ? reinterpret_cast<float*>(w + L.b) : nullptr;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_refine_scores(d, q, k, pool_idx, pool_cnt, kappa_p, r, dots, status, st);
  if (e != cudaSuccess) return PRISM_ERR_CUDA;
  SelectArgs a{};
  a.mode = 1;
  a.Hkv = d.Hkv;
  a.G = d.G;
  a.Hq = d.Hq;
  a.T = d.T;
  a.cu = d.cu_dev;
  a.keys = r;
  a.pool = pool_idx;
  a.pool_cnt = pool_cnt;
  a.pool_stride = kappa_p;
  a.k_req = kappa;
  a.out = idx;
  a.out_cnt = cnt;
  a.dots = dots;
  a.logits = logits_opt;
  a.status = status;
  return cuda_status(launch_select(d, a, kappa_p, st));
}

prism_status prism_propose_topk(const prism_shape* shape, const void* propose_ws,
                                size_t propose_ws_bytes, const int32_t* pool_idx,
                                const int32_t* pool_cnt, int32_t kappa_p, int32_t kappa,
                                int32_t* idx, int32_t* cnt, void* ws, size_t ws_bytes,
                                void* stream) {
  Dims d;
  prism_status s = check_shape(shape, &d);
  if (s != PRISM_OK) return s;
  if (!pool_idx || !pool_cnt || !idx || !cnt) return PRISM_ERR_INVALID_ARG;
  if (kappa_p < 1 || kappa < 1 || kappa > kappa_p) return PRISM_ERR_INVALID_ARG;
  if (kappa_p > select_capacity_per_row()) return PRISM_ERR_UNSUPPORTED;
  const Layout P = layout(d, PRISM_OP_PROPOSE, kappa_p, 0);
  if (!ws_ok(propose_ws, propose_ws_bytes, P)) return PRISM_ERR_WORKSPACE;
  const Layout L = layout(d, PRISM_OP_REFINE, kappa_p, kappa);
  if (!ws_ok(ws, ws_bytes, L)) return PRISM_ERR_WORKSPACE;
  if ((s = set_live_sms(&d)) != PRISM_OK) return s;
  char* w = static_cast<char*>(ws);
  int32_t* status = reinterpret_cast<int32_t*>(w);
  float* r = reinterpret_cast<float*>(w + L.a);
  const float* scores = reinterpret_cast<const float*>(static_cast<const char*>(propose_ws) + P.a);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_pool_gather(d, scores, pool_idx, pool_cnt, kappa_p, r, status, st);
  if (e != cudaSuccess) return PRISM_ERR_CUDA;
  SelectArgs a{};
  a.mode = 1;
  a.Hkv = d.Hkv;
  a.G = d.G;
  a.Hq = d.Hq;
  a.T = d.T;
  a.cu = d.cu_dev;
  a.keys = r;
  a.pool = pool_idx;
  a.pool_cnt = pool_cnt;
  a.pool_stride = kappa_p;
  a.k_req = kappa;
  a.out = idx;
  a.out_cnt = cnt;
  a.status = status;
  return cuda_status(launch_select(d, a, kappa_p, st));
}

prism_status prism_propose_ex(const prism_shape* shape, const void* q, const int8_t* kq,
                              const float* k_scale, int32_t kappa_p, int32_t* pool_idx,
                              int32_t* pool_cnt, uint32_t sets, void* ws, size_t ws_bytes,
                              void* stream) {
  if (sets == PRISM_SETS_KV_HEAD || sets == PRISM_SETS_Q_HEAD)
    return prism_propose(shape, q, kq, k_scale, kappa_p, pool_idx, pool_cnt, ws, ws_bytes, stream);
  if (sets != PRISM_SETS_SEQUENCE) return PRISM_ERR_INVALID_ARG;
  Dims d;
  prism_status s = check_shape(shape, &d);
  if (s != PRISM_OK) return s;
  if (!q || !kq || !k_scale || !pool_idx || !pool_cnt || kappa_p < 1) return PRISM_ERR_INVALID_ARG;
  if (d.max_len > select_capacity_per_row()) return PRISM_ERR_UNSUPPORTED;
  const Layout L = layout(d, PRISM_OP_PROPOSE, kappa_p, 0);
  if (!ws_ok(ws, ws_bytes, L)) return PRISM_ERR_WORKSPACE;
  if ((s = set_live_sms(&d)) != PRISM_OK) return s;
  char* w = static_cast<char*>(ws);
  int32_t* status = reinterpret_cast<int32_t*>(w);
  float* scores = reinterpret_cast<float*>(w + L.a);
  float* smax = reinterpret_cast<float*>(w + L.c);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_propose_scores(d, q, kq, k_scale, scores, nullptr, use_mma_scorer() && d.bf16,
                                        status, st);
  if (e != cudaSuccess) return PRISM_ERR_CUDA;
  if ((e = launch_head_max(scores, d.Hkv, 1, d.T, smax, st)) != cudaSuccess) return PRISM_ERR_CUDA;
  Dims d1 = d;  // one selection row per sequence over the head maxima
  d1.Hkv = 1;
  d1.G = d.Hq;
  SelectArgs a{};
  a.mode = 0;
  a.Hkv = 1;
  a.G = d.Hq;
  a.Hq = d.Hq;
  a.T = d.T;
  a.cu = d.cu_dev;
  a.keys = smax;
  a.k_req = kappa_p;
  a.out = pool_idx;
  a.out_cnt = pool_cnt;
  a.status = status;
  return cuda_status(launch_select(d1, a, d.max_len, st));
}

prism_status prism_refine_mass(const prism_shape* shape, const void* q, const void* k,
                               const int32_t* pool_idx, const int32_t* pool_cnt, int32_t kappa_p,
                               int32_t kappa, float softmax_scale, int32_t* idx, int32_t* cnt, void* ws,
                               size_t ws_bytes, void* stream) {
  Dims d;
  prism_status s = check_shape(shape, &d);
  if (s != PRISM_OK) return s;
  if (!q || !k || !pool_idx || !pool_cnt || !idx || !cnt) return PRISM_ERR_INVALID_ARG;
  if (kappa_p < 1 || kappa < 1 || kappa > kappa_p) return PRISM_ERR_INVALID_ARG;
  if (!std::isfinite(softmax_scale) || softmax_scale <= 0.0f) return PRISM_ERR_INVALID_ARG;
  if (kappa_p > select_capacity_per_row()) return PRISM_ERR_UNSUPPORTED;
  const Layout L = layout(d, PRISM_OP_REFINE, kappa_p, kappa);
  if (!ws_ok(ws, ws_bytes, L)) return PRISM_ERR_WORKSPACE;
  if ((s = set_live_sms(&d)) != PRISM_OK) return s;
  char* w = static_cast<char*>(ws);
  int32_t* status = reinterpret_cast<int32_t*>(w);
  float* r = reinterpret_cast<float*>(w + L.a);
  float* dots = reinterpret_cast<float*>(w + L.b);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_refine_scores(d, q, k, pool_idx, pool_cnt, kappa_p, r, dots, status, st);
  if (e != cudaSuccess) return PRISM_ERR_CUDA;
  if ((e = launch_refine_mass(d, r, dots, pool_cnt, kappa_p, softmax_scale, st)) != cudaSuccess)
    return PRISM_ERR_CUDA;
  SelectArgs a{};
  a.mode = 1;
  a.Hkv = d.Hkv;
  a.G = d.G;
  a.Hq = d.Hq;
  a.T = d.T;
  a.cu = d.cu_dev;
  a.keys = r;
  a.pool = pool_idx;
  a.pool_cnt = pool_cnt;
  a.pool_stride = kappa_p;
  a.k_req = kappa;
  a.out = idx;
  a.out_cnt = cnt;
  a.status = status;
  return cuda_status(launch_select(d, a, kappa_p, st));
}

prism_status prism_refine_ex(const prism_shape* shape, const void* q, const void* k,
                             const int32_t* pool_idx, const int32_t* pool_cnt, int32_t kappa_p,
                             int32_t kappa, int32_t* idx, int32_t* cnt, uint32_t sets, void* ws,
                             size_t ws_bytes, void* stream) {
  if (sets == PRISM_SETS_KV_HEAD)
    return prism_refine(shape, q, k, pool_idx, pool_cnt, kappa_p, kappa, idx, cnt, nullptr, ws,
                        ws_bytes, stream);
  if (sets != PRISM_SETS_Q_HEAD && sets != PRISM_SETS_SEQUENCE) return PRISM_ERR_INVALID_ARG;
  Dims d;
  prism_status s = check_shape(shape, &d);
  if (s != PRISM_OK) return s;
  if (!q || !k || !pool_idx || !pool_cnt || !idx || !cnt) return PRISM_ERR_INVALID_ARG;
  if (kappa_p < 1 || kappa < 1 || kappa > kappa_p) return PRISM_ERR_INVALID_ARG;
  if (kappa_p > select_capacity_per_row()) return PRISM_ERR_UNSUPPORTED;
  const Layout L = layout(d, PRISM_OP_REFINE, kappa_p, kappa);
  if (!ws_ok(ws, ws_bytes, L)) return PRISM_ERR_WORKSPACE;
  if ((s = set_live_sms(&d)) != PRISM_OK) return s;
  char* w = static_cast<char*>(ws);
  int32_t* status = reinterpret_cast<int32_t*>(w);
  float* r = reinterpret_cast<float*>(w + L.a);
  float* dots = reinterpret_cast<float*>(w + L.b);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  SelectArgs a{};
  a.mode = 1;
  a.T = d.T;
  a.cu = d.cu_dev;
  a.pool = pool_idx;
  a.pool_cnt = pool_cnt;
  a.pool_stride = kappa_p;
  a.k_req = kappa;
  a.out = idx;
  a.out_cnt = cnt;
  a.status = status;
  Dims d1 = d;
  if (sets == PRISM_SETS_Q_HEAD) {
    // per-head exact scores dots [B][Hkv][G][kappa_p] = [B Hq][kappa_p]: one
    // selection row per query head over its group's pool
    cudaError_t e = launch_refine_scores(d, q, k, pool_idx, pool_cnt, kappa_p, r, dots, status, st);
    if (e != cudaSuccess) return PRISM_ERR_CUDA;
    d1.Hkv = d.Hq;
    d1.G = 1;
    a.keys = dots;
    a.pool_div = d.G;
  } else {
    // every KV head scores the sequence's pool; the head maxima select
    float* rmax = reinterpret_cast<float*>(w + L.c);
    cudaError_t e = launch_refine_scores(d, q, k, pool_idx, pool_cnt, kappa_p, r, nullptr, status, st,
                                         d.Hkv);
    if (e != cudaSuccess) return PRISM_ERR_CUDA;
    if ((e = launch_head_max(r, d.Hkv, d.B, kappa_p, rmax, st)) != cudaSuccess) return PRISM_ERR_CUDA;
    d1.Hkv = 1;
    d1.G = d.Hq;
    a.keys = rmax;
  }
  a.Hkv = d1.Hkv;
  a.G = d1.G;
  a.Hq = d.Hq;
  return cuda_status(launch_select(d1, a, kappa_p, st));
}

prism_status prism_sparse_decode_ex(const prism_shape* shape, const void* q, const void* k,
                                    const void* v, const int32_t* idx, const int32_t* cnt,
                                    int32_t kappa, float softmax_scale, uint32_t sets, float* out,
                                    float* lse_opt, void* ws, size_t ws_bytes, void* stream) {
  if (sets == PRISM_SETS_KV_HEAD)
    return prism_sparse_decode(shape, q, k, v, idx, cnt, kappa, softmax_scale, out, lse_opt, ws,
                               ws_bytes, stream);
  if (sets != PRISM_SETS_Q_HEAD && sets != PRISM_SETS_SEQUENCE) return PRISM_ERR_INVALID_ARG;
  Dims d;
  prism_status s = check_shape(shape, &d);
  if (s != PRISM_OK) return s;
  if (!q || !k || !v || !idx || !cnt || !out || kappa < 1) return PRISM_ERR_INVALID_ARG;
  if (!std::isfinite(softmax_scale)) return PRISM_ERR_INVALID_ARG;
  const Layout L = layout(d, PRISM_OP_SPARSE_DECODE, 0, kappa);
  if (!ws_ok(ws, ws_bytes, L)) return PRISM_ERR_WORKSPACE;
  Dims d1 = d;
  int kv_div = 1, idx_div = 1;
  if (sets == PRISM_SETS_Q_HEAD) {  // a row per query head, reading its group's K/V head
    d1.Hkv = d.Hq;
    d1.G = 1;
    kv_div = d.G;
  } else {  // every KV head reads the sequence's one set
    idx_div = d.Hkv;
  }
  // the per-query-head rows split no finer than the per-KV-head plan the
  // workspace is sized for: B Hq splits' <= B Hq splits
  const AttendPlan p = plan_attend(d1, kappa, false);
  if ((s = set_live_sms(&d)) != PRISM_OK) return s;
  char* w = static_cast<char*>(ws);
  return cuda_status(launch_attend(d1, p, q, k, v, idx, cnt, kappa, softmax_scale,
                                   reinterpret_cast<float*>(w + L.a),
                                   reinterpret_cast<float*>(w + L.b), out, lse_opt,
                                   reinterpret_cast<int32_t*>(w), static_cast<cudaStream_t>(stream),
                                   kv_div, idx_div));
}

prism_status prism_sparse_decode(const prism_shape* shape, const void* q, const void* k,
                                 const void* v, const int32_t* idx, const int32_t* cnt,
                                 int32_t kappa, float softmax_scale, float* out, float* lse_opt,
                                 void* ws, size_t ws_bytes, void* stream) {
  Dims d;
  prism_status s = check_shape(shape, &d);
  if (s != PRISM_OK) return s;
  if (!q || !k || !v || !idx || !cnt || !out || kappa < 1) return PRISM_ERR_INVALID_ARG;
  if (!std::isfinite(softmax_scale)) return PRISM_ERR_INVALID_ARG;
  const Layout L = layout(d, PRISM_OP_SPARSE_DECODE, 0, kappa);
  if (!ws_ok(ws, ws_bytes, L)) return PRISM_ERR_WORKSPACE;
  const AttendPlan p = plan_attend(d, kappa, false);
  if ((s = set_live_sms(&d)) != PRISM_OK) return s;
  char* w = static_cast<char*>(ws);
  return cuda_status(launch_attend(d, p, q, k, v, idx, cnt, kappa, softmax_scale,
                                   reinterpret_cast<float*>(w + L.a),
                                   reinterpret_cast<float*>(w + L.b), out, lse_opt,
                                   reinterpret_cast<int32_t*>(w), static_cast<cudaStream_t>(stream)));
}

prism_status prism_refine_decode(const prism_shape* shape, const void* q, void* k, void* v,
                                 const int32_t* pool_idx, const int32_t* pool_cnt,
                                 int32_t kappa_p, int32_t kappa, float softmax_scale, int32_t* idx,
                                 int32_t* cnt, float* out, float* lse_opt, const void* k_new_opt,
                                 const void* v_new_opt, const void* k_prefetch, uint32_t flags,
                                 void* ws, size_t ws_bytes, void* stream) {
  Dims d;
  prism_status s = check_shape(shape, &d);
  if (s != PRISM_OK) return s;
  if (!q || !k || !v || !pool_idx || !pool_cnt || !idx || !cnt || !out) return PRISM_ERR_INVALID_ARG;
  if (kappa_p < 1 || kappa < 1 || kappa > kappa_p) return PRISM_ERR_INVALID_ARG;
  if (!std::isfinite(softmax_scale)) return PRISM_ERR_INVALID_ARG;
  if (flags & ~(PRISM_RD_OVERLAP | PRISM_RD_SUM_GROUP | PRISM_RD_MASS)) return PRISM_ERR_INVALID_ARG;
  if ((flags & PRISM_RD_SUM_GROUP) && (flags & PRISM_RD_MASS)) return PRISM_ERR_INVALID_ARG;
  if ((flags & PRISM_RD_MASS) && !(softmax_scale > 0.0f)) return PRISM_ERR_INVALID_ARG;
  if ((k_new_opt == nullptr) != (v_new_opt == nullptr)) return PRISM_ERR_INVALID_ARG;
  if (((uintptr_t)q | (uintptr_t)k | (uintptr_t)v) % 16) return PRISM_ERR_INVALID_ARG;
  if (k_new_opt && (((uintptr_t)k_new_opt | (uintptr_t)v_new_opt | (uintptr_t)k | (uintptr_t)v) % 16))
    return PRISM_ERR_INVALID_ARG;
  const Layout L = layout(d, PRISM_OP_REFINE_DECODE, kappa_p, kappa);
  if (!ws_ok(ws, ws_bytes, L)) return PRISM_ERR_WORKSPACE;
  const RefineDecodePlan p = plan_refine_decode(d, kappa_p);
  if (!p.ok) return PRISM_ERR_UNSUPPORTED;
  return cuda_status(launch_refine_decode(d, p, q, k, v, k_new_opt, v_new_opt, k_prefetch, pool_idx,
                                          pool_cnt, kappa_p, kappa, softmax_scale, idx, cnt, out,
                                          lse_opt, static_cast<int32_t*>(ws),
                                          (flags & PRISM_RD_OVERLAP) != 0,
                                          (flags & PRISM_RD_SUM_GROUP) ? 1 : (flags & PRISM_RD_MASS) ? 2 : 0,
                                          static_cast<cudaStream_t>(stream)));
}

prism_status prism_dense_decode(const prism_shape* shape, const void* q, const void* k,
                                const void* v, float softmax_scale, float* out, float* lse_opt,
                                void* ws, size_t ws_bytes, void* stream) {
  Dims d;
  prism_status s = check_shape(shape, &d);
  if (s != PRISM_OK) return s;
  if (!q || !k || !v || !out) return PRISM_ERR_INVALID_ARG;
  if (((uintptr_t)q | (uintptr_t)k | (uintptr_t)v) % 16) return PRISM_ERR_INVALID_ARG;
  if (!std::isfinite(softmax_scale)) return PRISM_ERR_INVALID_ARG;
  const Layout L = layout(d, PRISM_OP_DENSE_DECODE, 0, 0);
  if (!ws_ok(ws, ws_bytes, L)) return PRISM_ERR_WORKSPACE;
  const AttendPlan p = plan_attend(d, d.max_len, true);
  if ((s = set_live_sms(&d)) != PRISM_OK) return s;
  char* w = static_cast<char*>(ws);
  return cuda_status(launch_attend(d, p, q, k, v, nullptr, nullptr, 0, softmax_scale,
                                   reinterpret_cast<float*>(w + L.a),
                                   reinterpret_cast<float*>(w + L.b), out, lse_opt,
                                   reinterpret_cast<int32_t*>(w), static_cast<cudaStream_t>(stream)));
}

prism_status prism_index_overlap(int32_t rows, const int32_t* a, const int32_t* cnt_a,
                                 int32_t stride_a, const int32_t* b, const int32_t* cnt_b,
                                 int32_t stride_b, int32_t* out, void* stream) {
  if (rows < 0 || stride_a < 1 || stride_b < 1) return PRISM_ERR_INVALID_ARG;
  if (rows == 0) return PRISM_OK;
  if (!a || !cnt_a || !b || !cnt_b || !out) return PRISM_ERR_INVALID_ARG;
  return cuda_status(launch_overlap(rows, a, cnt_a, stride_a, b, cnt_b, stride_b, out,
                                    static_cast<cudaStream_t>(stream)));
}

prism_status prism_clear_device_status(void* ws, size_t ws_bytes, void* stream) {
  if (!ws || ws_bytes < kWsHeader) return PRISM_ERR_WORKSPACE;
  return cuda_status(cudaMemsetAsync(ws, 0, kWsHeader, static_cast<cudaStream_t>(stream)));
}

prism_status prism_get_device_status(const void* ws, size_t ws_bytes, void* stream,
                                     int32_t* code) {
  if (!ws || ws_bytes < kWsHeader) return PRISM_ERR_WORKSPACE;
  if (!code) return PRISM_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t v = 0;
  if (cudaMemcpyAsync(&v, ws, sizeof(v), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return PRISM_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return PRISM_ERR_CUDA;
  *code = v;
  return PRISM_OK;
}

const char* prism_status_str(prism_status s) {
  switch (s) {
    case PRISM_OK: return "ok";
    case PRISM_ERR_INVALID_ARG: return "invalid argument";
    case PRISM_ERR_UNSUPPORTED: return "unsupported shape or size";
    case PRISM_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case PRISM_ERR_CUDA: return "CUDA launch or runtime error";
    case PRISM_ERR_TIMEOUT: return "device-side wait timed out";
    case PRISM_ERR_SCRATCH_LIMIT:
      return "request needs more than the fixed scratch of the no-allocation entry point";
  }
  return "unknown status";
}

}  // extern "C"

// ---------------------------------------------------------------------------
// No-allocation sparse decode.  Callers that may not allocate device memory
// when they call (a memory pool they do not own, an allocator callback, an
// engine whose memory is fixed at start-up) get the split-K partials kept in
// this file-scope array instead of a caller workspace.  In host code the name
// is only a stand-in for the device symbol; its device address is looked up
// once per device with that device current, and the lookup's result is
// checked before any kernel sees it.
namespace prism {
namespace {

static __device__ __align__(256) unsigned char noalloc_scratch[PRISM_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex noalloc_mu;
void* noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch on the current device (looked up on the
// first call on that device).
prism_status noalloc_scratch_ptr(char** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PRISM_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return PRISM_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(noalloc_mu);
  if (!noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, noalloc_scratch) != cudaSuccess || !p) return PRISM_ERR_CUDA;
    noalloc_ptr[dev] = p;
  }
  *out = static_cast<char*>(noalloc_ptr[dev]);
  return PRISM_OK;
}

}  // namespace
}  // namespace prism

extern "C" prism_status prism_sparse_decode_noalloc(const prism_shape* shape, const void* q,
                                                    const void* k, const void* v,
                                                    const int32_t* idx, const int32_t* cnt,
                                                    int32_t kappa, float softmax_scale, float* out,
                                                    float* lse_opt, int32_t* status_dev,
                                                    void* stream) {
  Dims d;
  prism_status s = check_shape(shape, &d);
  if (s != PRISM_OK) return s;
  if (!q || !k || !v || !idx || !cnt || !out || !status_dev || kappa < 1) return PRISM_ERR_INVALID_ARG;
  if (!std::isfinite(softmax_scale)) return PRISM_ERR_INVALID_ARG;
  // The same partial layout as the workspace of prism_sparse_decode; the
  // header bytes at its start stay unused (the status goes to status_dev).
  const Layout L = layout(d, PRISM_OP_SPARSE_DECODE, 0, kappa);
  if (L.total > (size_t)PRISM_NOALLOC_SCRATCH_BYTES) return PRISM_ERR_SCRATCH_LIMIT;
  const AttendPlan p = plan_attend(d, kappa, false);
  if ((s = set_live_sms(&d)) != PRISM_OK) return s;
  char* w = nullptr;
  if ((s = noalloc_scratch_ptr(&w)) != PRISM_OK) return s;
  return cuda_status(launch_attend(d, p, q, k, v, idx, cnt, kappa, softmax_scale,
                                   reinterpret_cast<float*>(w + L.a),
                                   reinterpret_cast<float*>(w + L.b), out, lse_opt, status_dev,
                                   static_cast<cudaStream_t>(stream)));
}
