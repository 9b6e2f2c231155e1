// Exact rescoring of the candidate pool at every layer (Prism Attention,
// sec. 4.1 "Proposal-Refined Index Sharing"; sec. 6: refined layers re-select
// their own top-kappa inside the proposed region at a cost independent of
// context length):
//   r[row][i] = max_g sum_j q[b][h*G+g][j] * K[h][cu[b] + pool[row][i]][j]
// with fp32 accumulation (bf16 x bf16 products are exact in fp32).  The
// per-head dot products are kept as well when the caller wants logits.
//
// A gather of kappa_p key rows per (sequence, KV head): d*sizeof(T) bytes per
// pool member, 256 B at bf16 d = 128.  A row is spread over d*sizeof(T)/16
// lanes with one 16-byte load each; four rows per lane group are in flight.
#include "common.cuh"
#include "kernels.h"

namespace prism {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kUnroll = 4;

struct RefineArgs {
  const void* q;
  const void* k;
  const int32_t* cu;
  const int32_t* pool;
  const int32_t* pool_cnt;
  int pool_stride;
  int Hkv, G;
  int64_t T;
  int per_cta;
  float* r;
  float* dots;
  int32_t* status;
  int pool_div;  // row (b, h) reads pool row (b Hkv + h) / pool_div
};

template <typename T, int D, int GP>
__global__ void __launch_bounds__(kThreads) refine_score_kernel(const RefineArgs a) {
  constexpr int E = Vec16<T>::E;
  constexpr int LPR = D / E;
  constexpr int RPW = 32 / LPR;
  const int row = blockIdx.y;
  const int b = row / a.Hkv, h = row - b * a.Hkv;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int sub = lane / LPR, li = lane % LPR;
  const int prow = row / a.pool_div;
  int n = a.pool_cnt[prow];
  n = n < 0 ? 0 : (n > a.pool_stride ? a.pool_stride : n);
  const int e0 = blockIdx.x * a.per_cta;
  const int e1 = min(n, e0 + a.per_cta);
  if (e0 >= e1) return;
  const int t0 = a.cu[b];
  const int L = a.cu[b + 1] - t0;
  const T* kbase = static_cast<const T*>(a.k) + ((int64_t)h * a.T + t0) * D + li * E;
  const T* q = static_cast<const T*>(a.q) + ((int64_t)b * a.Hkv * a.G + (int64_t)h * a.G) * D;
  const int32_t* pool = a.pool + (int64_t)prow * a.pool_stride;

  float qf[GP][E];
#pragma unroll
  for (int g = 0; g < GP; ++g) {
    if (g < a.G) {
      Vec16<T>::unpack(ld16(q + (int64_t)g * D + li * E), qf[g]);
    } else {
#pragma unroll
      for (int e = 0; e < E; ++e) qf[g][e] = 0.0f;
    }
  }

  for (int base = e0 + warp * RPW * kUnroll; base < e1; base += kWarps * RPW * kUnroll) {
    uint4 raw[kUnroll];
    bool ok[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int e = base + u * RPW + sub;
      ok[u] = e < e1;
      int pos = ok[u] ? pool[e] : 0;
      if (ok[u] && (pos < 0 || pos >= L)) {
        if (li == 0) flag_status(a.status, PRISM_DEV_BAD_INDEX);
        ok[u] = false;
        pos = 0;
      }
      raw[u] = ok[u] ? ld16(kbase + (int64_t)pos * D) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      float f[E];
      Vec16<T>::unpack(raw[u], f);
      float acc[GP];
#pragma unroll
      for (int g = 0; g < GP; ++g) {
        float s = 0.0f;
#pragma unroll
        for (int e = 0; e < E; ++e) s = fmaf(qf[g][e], f[e], s);
        acc[g] = group_sum<LPR>(s);
      }
      float best = acc[0];
#pragma unroll
      for (int g = 1; g < GP; ++g)
        if (g < a.G) best = fmaxf(best, acc[g]);
      const int e = base + u * RPW + sub;
      if (e < e1 && li == 0) {
        a.r[(int64_t)row * a.pool_stride + e] = ok[u] ? best : -INFINITY;
        if (a.dots) {
#pragma unroll
          for (int g = 0; g < GP; ++g)
            if (g < a.G) a.dots[((int64_t)row * a.G + g) * a.pool_stride + e] = acc[g];
        }
      }
    }
  }
}

template <typename T, int D, int GP>
cudaError_t run(const Dims& d, const RefineArgs& a0, cudaStream_t st) {
  constexpr int RPW = 32 / (D / Vec16<T>::E);
  constexpr int step = kWarps * RPW * kUnroll;
  RefineArgs a = a0;
  const int rows = d.B * d.Hkv;
  const int64_t target = 2LL * d.num_sms;
  int64_t per = cdiv((int64_t)a.pool_stride * rows, target);
  per = cdiv(per, step) * step;
  if (per < step) per = step;
  a.per_cta = (int)per;
  const int splits = (int)cdiv(a.pool_stride, per);
  refine_score_kernel<T, D, GP><<<dim3(splits, rows), kThreads, 0, st>>>(a);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t by_group(const Dims& d, const RefineArgs& a, cudaStream_t st) {
  switch (padded_group(d.G)) {
    case 1: return run<T, D, 1>(d, a, st);
    case 2: return run<T, D, 2>(d, a, st);
    case 4: return run<T, D, 4>(d, a, st);
    case 8: return run<T, D, 8>(d, a, st);
    default: return run<T, D, 16>(d, a, st);
  }
}

// The proposal scores of the pool members, r[row][i] = scores[h][cu[b] +
// pool[row][i]] (the selection keys of a proposal layer that takes its own
// set from its quantized scores); a position outside its sequence is flagged
// and ranks last.  4 B gathered per member (the scores are L2-resident after
// the proposal).
__global__ void __launch_bounds__(kThreads) pool_gather_kernel(const float* __restrict__ scores,
                                                               const int32_t* __restrict__ cu,
                                                               const int32_t* __restrict__ pool,
                                                               const int32_t* __restrict__ pool_cnt,
                                                               int pool_stride, int Hkv, int64_t T,
                                                               float* __restrict__ r,
                                                               int32_t* status) {
  const int row = blockIdx.y;
  const int b = row / Hkv, h = row - b * Hkv;
  int n = pool_cnt[row];
  n = n < 0 ? 0 : (n > pool_stride ? pool_stride : n);
  const int t0 = cu[b], L = cu[b + 1] - t0;
  const float* sb = scores + (int64_t)h * T + t0;
  const int32_t* pr = pool + (int64_t)row * pool_stride;
  float* rr = r + (int64_t)row * pool_stride;
  for (int i = blockIdx.x * kThreads + threadIdx.x; i < n; i += gridDim.x * kThreads) {
    const int p = pr[i];
    const bool ok = p >= 0 && p < L;
    if (!ok) flag_status(status, PRISM_DEV_BAD_INDEX);
    rr[i] = ok ? sb[p] : -INFINITY;
  }
}

// Softmax-mass aggregation of a row's pool members (the group's G query
// heads share one set; each member's score is the attention mass the heads
// put on it, each head's softmax over the pool):
//   r_i <- sum_g 2^((d_g,i - M_g) c) / sum_i' 2^((d_g,i' - M_g) c),
// c = softmax_scale * log2 e, M_g the largest d_g over the row's members.
// Members flagged by the scoring pass (r_i = -inf) take no part and stay
// -inf.  One CTA per row; dots [row][G][stride] from the scoring pass.
template <int GP>
__global__ void __launch_bounds__(kThreads) mass_kernel(float* __restrict__ r, const float* __restrict__ dots,
                                                        const int32_t* __restrict__ pool_cnt, int stride,
                                                        int G, float c) {
  __shared__ float s_a[kWarps][GP];
  const int row = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int n = pool_cnt[row];
  n = n < 0 ? 0 : (n > stride ? stride : n);
  float* rr = r + (int64_t)row * stride;
  const float* dr = dots + (int64_t)row * G * stride;
  // the whole CTA's value of v per head, through the warps
  auto reduce = [&](float (&v)[GP], bool is_max) {
#pragma unroll
    for (int g = 0; g < GP; ++g) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float x = __shfl_xor_sync(0xffffffffu, v[g], o);
        v[g] = is_max ? fmaxf(v[g], x) : v[g] + x;
      }
      if (lane == 0) s_a[warp][g] = v[g];
    }
    __syncthreads();
#pragma unroll
    for (int g = 0; g < GP; ++g) {
      float t = s_a[0][g];
#pragma unroll
      for (int w = 1; w < kWarps; ++w) t = is_max ? fmaxf(t, s_a[w][g]) : t + s_a[w][g];
      v[g] = t;
    }
    __syncthreads();
  };
  float m[GP], z[GP];
#pragma unroll
  for (int g = 0; g < GP; ++g) {
    m[g] = -INFINITY;
    z[g] = 0.0f;
  }
  for (int i = tid; i < n; i += kThreads)
    if (rr[i] != -INFINITY)
#pragma unroll
      for (int g = 0; g < GP; ++g)
        if (g < G) m[g] = fmaxf(m[g], dr[(int64_t)g * stride + i]);
  reduce(m, true);
  for (int i = tid; i < n; i += kThreads)
    if (rr[i] != -INFINITY)
#pragma unroll
      for (int g = 0; g < GP; ++g)
        if (g < G) z[g] += exp2f((dr[(int64_t)g * stride + i] - m[g]) * c);
  reduce(z, false);
  for (int i = tid; i < n; i += kThreads) {
    if (rr[i] == -INFINITY) continue;
    float mass = 0.0f;
#pragma unroll
    for (int g = 0; g < GP; ++g)
      if (g < G) mass += exp2f((dr[(int64_t)g * stride + i] - m[g]) * c) / z[g];
    rr[i] = mass;
  }
}

}  // namespace

cudaError_t launch_pool_gather(const Dims& d, const float* scores, const int32_t* pool,
                               const int32_t* pool_cnt, int pool_stride, float* r, int32_t* status,
                               cudaStream_t st) {
  const int rows = d.B * d.Hkv;
  if (rows == 0 || pool_stride == 0) return cudaSuccess;
  const int bx = (int)cdiv(pool_stride, kThreads) < 8 ? (int)cdiv(pool_stride, kThreads) : 8;
  pool_gather_kernel<<<dim3(bx, rows), kThreads, 0, st>>>(scores, d.cu_dev, pool, pool_cnt, pool_stride,
                                                          d.Hkv, d.T, r, status);
  return cudaGetLastError();
}

cudaError_t launch_refine_scores(const Dims& d, const void* q, const void* k, const int32_t* pool,
                                 const int32_t* pool_cnt, int pool_stride, float* r, float* dots,
                                 int32_t* status, cudaStream_t st, int pool_div) {
  if (d.B * d.Hkv == 0 || pool_stride == 0) return cudaSuccess;
  RefineArgs a{q, k, d.cu_dev, pool, pool_cnt, pool_stride, d.Hkv, d.G, d.T, 0, r, dots, status,
               pool_div > 1 ? pool_div : 1};
  if (d.bf16)
    return d.D == 128 ? by_group<__nv_bfloat16, 128>(d, a, st) : by_group<__nv_bfloat16, 64>(d, a, st);
  return d.D == 128 ? by_group<float, 128>(d, a, st) : by_group<float, 64>(d, a, st);
}

}  // namespace prism

namespace prism {

cudaError_t launch_refine_mass(const Dims& d, float* r, const float* dots, const int32_t* pool_cnt,
                               int pool_stride, float softmax_scale, cudaStream_t st) {
  const int rows = d.B * d.Hkv;
  if (rows == 0 || pool_stride == 0) return cudaSuccess;
  const float c = softmax_scale * 1.4426950408889634f;
  switch (padded_group(d.G)) {
    case 1: mass_kernel<1><<<rows, kThreads, 0, st>>>(r, dots, pool_cnt, pool_stride, d.G, c); break;
    case 2: mass_kernel<2><<<rows, kThreads, 0, st>>>(r, dots, pool_cnt, pool_stride, d.G, c); break;
    case 4: mass_kernel<4><<<rows, kThreads, 0, st>>>(r, dots, pool_cnt, pool_stride, d.G, c); break;
    case 8: mass_kernel<8><<<rows, kThreads, 0, st>>>(r, dots, pool_cnt, pool_stride, d.G, c); break;
    default: mass_kernel<16><<<rows, kThreads, 0, st>>>(r, dots, pool_cnt, pool_stride, d.G, c); break;
  }
  return cudaGetLastError();
}

}  // namespace prism
