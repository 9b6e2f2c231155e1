// Split-K flash-decode over a list of cache rows, with a log-sum-exp merge:
// the token-level sparse attention over the refined set (Prism Attention,
// sec. 1 and sec. 2.1) and, with the list "every position", the dense decode
// the pages compare against (sec. 5.3 "End-to-end latency").
//
// Split s of row (b, h) covers list entries [s*per, (s+1)*per).  Every lane
// group of d*sizeof(T)/16 lanes walks rows of K and V with 16-byte loads and
// keeps an online softmax state per query head of the group in the log2
// domain (logit * softmax_scale * log2 e):
//   m = max logit so far, l = sum 2^(logit - m), o = sum 2^(logit - m) v.
// The CTA combines its lane groups in a fixed order and writes one partial
// (o, m, l) per query head and split; merge_kernel combines the splits:
//   M = max_s m_s,  out = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s,
//   lse = (M + log2 sum_s 2^(m_s - M) l_s) * ln 2.
// HBM bound: 2 * d * sizeof(T) bytes per listed row.
#include <algorithm>
#include <queue>
#include <type_traits>
#include <vector>

#include "common.cuh"
#include "kernels.h"

namespace prism {

namespace {

constexpr int kThreads = 128;
constexpr int kWarps = kThreads / 32;
// rows a lane group loads before it computes (a deeper unroll costs
// registers, hence resident warps, and moved no more bytes per SM)
constexpr int kUnroll = 2;

struct AttendArgs {
  const void* q;
  const void* k;
  const void* v;
  const int32_t* cu;
  const int32_t* idx;
  const int32_t* cnt;
  int idx_stride;
  int Hkv, G, Hq;
  int64_t T;
  int per_split, splits;
  float scale_log2;
  float* part_o;
  float* part_ml;
  int32_t* status;
  int kv_div;   // row (b, h) reads K/V head h / kv_div
  int idx_div;  // and idx / cnt row (b Hkv + h) / idx_div
};

template <typename T, int D, int GP>
__global__ void __launch_bounds__(kThreads) attend_kernel(const AttendArgs a) {
  constexpr int E = Vec16<T>::E;
  constexpr int LPR = D / E;
  constexpr int RPW = 32 / LPR;
  constexpr int SLOTS = kWarps * RPW;
  extern __shared__ __align__(16) float sm[];
  float* s_o = sm;                       // [SLOTS][GP][D]
  float* s_m = sm + SLOTS * GP * D;      // [SLOTS][GP]
  float* s_l = s_m + SLOTS * GP;         // [SLOTS][GP]

  const int row = blockIdx.x, split = blockIdx.y;  // rows on x: B * Hkv may exceed 65535
  const int b = row / a.Hkv, h = row - b * a.Hkv;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int sub = lane / LPR, li = lane % LPR;
  const int slot = warp * RPW + sub;
  const int t0 = a.cu[b];
  const int L = a.cu[b + 1] - t0;
  int n = L;
  const int irow = row / a.idx_div;
  if (a.idx) {
    n = a.cnt[irow];
    if (n < 0 || n > a.idx_stride) {
      if (threadIdx.x == 0 && split == 0) flag_status(a.status, PRISM_DEV_BAD_INDEX);
      n = n < 0 ? 0 : a.idx_stride;
    }
  }
  const int e0 = split * a.per_split;
  const int e1 = min(n, e0 + a.per_split);
  const int64_t off = ((int64_t)(h / a.kv_div) * a.T + t0) * D + li * E;
  const T* kbase = static_cast<const T*>(a.k) + off;
  const T* vbase = static_cast<const T*>(a.v) + off;
  const int32_t* idx = a.idx ? a.idx + (int64_t)irow * a.idx_stride : nullptr;

  float qf[GP][E];
  {
    const T* q = static_cast<const T*>(a.q) + ((int64_t)b * a.Hq + (int64_t)h * a.G) * D + li * E;
#pragma unroll
    for (int g = 0; g < GP; ++g) {
      if (g < a.G) {
        Vec16<T>::unpack(ld16(q + (int64_t)g * D), qf[g]);
      } else {
#pragma unroll
        for (int e = 0; e < E; ++e) qf[g][e] = 0.0f;
      }
    }
  }
  float m[GP], l[GP], o[GP][E];
#pragma unroll
  for (int g = 0; g < GP; ++g) {
    m[g] = -INFINITY;
    l[g] = 0.0f;
#pragma unroll
    for (int e = 0; e < E; ++e) o[g][e] = 0.0f;
  }

  for (int base = e0 + warp * RPW * kUnroll; base < e1; base += kWarps * RPW * kUnroll) {
    uint4 kr[kUnroll], vr[kUnroll];
    bool ok[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int e = base + u * RPW + sub;
      ok[u] = e < e1;
      int pos = e;
      if (idx && ok[u]) pos = idx[e];
      if (ok[u] && (pos < 0 || pos >= L)) {
        if (li == 0) flag_status(a.status, PRISM_DEV_BAD_INDEX);
        ok[u] = false;
      }
      if (!ok[u]) pos = 0;
      if (idx) {
        kr[u] = ok[u] ? ld16(kbase + (int64_t)pos * D) : make_uint4(0, 0, 0, 0);
        vr[u] = ok[u] ? ld16(vbase + (int64_t)pos * D) : make_uint4(0, 0, 0, 0);
      } else {
        kr[u] = ok[u] ? ld16_stream(kbase + (int64_t)pos * D) : make_uint4(0, 0, 0, 0);
        vr[u] = ok[u] ? ld16_stream(vbase + (int64_t)pos * D) : make_uint4(0, 0, 0, 0);
      }
    }
    float lg[kUnroll][GP];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      float f[E];
      Vec16<T>::unpack(kr[u], f);
#pragma unroll
      for (int g = 0; g < GP; ++g) {
        float s = 0.0f;
#pragma unroll
        for (int e = 0; e < E; ++e) s = fmaf(qf[g][e], f[e], s);
        s = group_sum<LPR>(s);
        lg[u][g] = ok[u] ? s * a.scale_log2 : -INFINITY;
      }
    }
    float vf[kUnroll][E];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) Vec16<T>::unpack(vr[u], vf[u]);
#pragma unroll
    for (int g = 0; g < GP; ++g) {
      float mx = m[g];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) mx = fmaxf(mx, lg[u][g]);
      if (mx == -INFINITY) continue;
      const float alpha = exp2f(m[g] - mx);
      float p[kUnroll];
      float ps = 0.0f;
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        p[u] = exp2f(lg[u][g] - mx);
        ps += p[u];
      }
      l[g] = l[g] * alpha + ps;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        float acc = o[g][e] * alpha;
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) acc = fmaf(p[u], vf[u][e], acc);
        o[g][e] = acc;
      }
      m[g] = mx;
    }
  }

  // Combine the CTA's lane groups in slot order (deterministic).
#pragma unroll
  for (int g = 0; g < GP; ++g) {
#pragma unroll
    for (int e = 0; e < E; ++e) s_o[(slot * GP + g) * D + li * E + e] = o[g][e];
    if (li == 0) {
      s_m[slot * GP + g] = m[g];
      s_l[slot * GP + g] = l[g];
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < a.G * D; i += kThreads) {
    const int g = i / D, j = i - g * D;
    float M = -INFINITY;
#pragma unroll
    for (int s = 0; s < SLOTS; ++s) M = fmaxf(M, s_m[s * GP + g]);
    float Ls = 0.0f, O = 0.0f;
    if (M != -INFINITY) {
#pragma unroll
      for (int s = 0; s < SLOTS; ++s) {
        const float ms = s_m[s * GP + g];
        const float w = ms == -INFINITY ? 0.0f : exp2f(ms - M);
        Ls = fmaf(w, s_l[s * GP + g], Ls);
        O = fmaf(w, s_o[(s * GP + g) * D + j], O);
      }
    }
    const int64_t pr = ((int64_t)b * a.Hq + (int64_t)h * a.G + g) * a.splits + split;
    a.part_o[pr * D + j] = O;
    if (j == 0) {
      a.part_ml[pr * 2] = M;
      a.part_ml[pr * 2 + 1] = Ls;
    }
  }
}

// ---- dense pass (the comparison path): contiguous rows staged by bulk copies
//
// Split s of row (b, h) covers positions [s*per, (s+1)*per) of sequence b.
// Thread 0 keeps kDStages stages in flight, each one 1D bulk copy of kDRows
// K rows and one of kDRows V rows (8 KB each, contiguous in the cache) into
// shared memory, completing on the stage's mbarrier; the CTA computes on the
// oldest stage with the same lane-group math as attend_kernel (two rows per
// lane group per stage pass) and hands the stage back.  Bytes in flight per
// SM come from the stage ring, not from registers.  A stage wait is bounded:
// past kDWaitLimit polls the CTA flags PRISM_DEV_TIMEOUT, waits (bounded) for
// its copies in flight and returns.
constexpr int kDThreads = 256;
constexpr int kDWarps = kDThreads / 32;
constexpr int kDStages = 6;
constexpr int kDPartBytes = 8192;  // K (or V) bytes of one stage
constexpr uint32_t kDWaitLimit = 1u << 24;

__device__ __forceinline__ void d_mbar_init(uint64_t* bar) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;\n" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool d_mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ void d_bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

template <typename T, int D, int GP>
__global__ void __launch_bounds__(kDThreads, GP <= 4 ? 2 : 1) dense_kernel(const AttendArgs a) {
  constexpr int E = Vec16<T>::E;
  constexpr int LPR = D / E;            // lanes per row
  constexpr int RPW = 32 / LPR;         // rows per warp per pass
  constexpr int RB = D * (int)sizeof(T);
  constexpr int R = kDPartBytes / RB;   // rows per stage
  constexpr int PASS = kDWarps * RPW;   // rows per CTA pass
  static_assert(R == 2 * PASS, "two passes per stage");
  constexpr int SLOTS = kDWarps * RPW;
  extern __shared__ __align__(128) unsigned char dsm[];
  __shared__ __align__(8) uint64_t full[kDStages];

  const int row = blockIdx.x, split = blockIdx.y;
  const int b = row / a.Hkv, h = row - b * a.Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int sub = lane / LPR, li = lane % LPR;
  const int slot = warp * RPW + sub;
  const int t0 = a.cu[b];
  const int L = a.cu[b + 1] - t0;
  const int e0 = split * a.per_split;
  const int e1 = min(L, e0 + a.per_split);
  const int nst = e1 > e0 ? (e1 - e0 + R - 1) / R : 0;
  const unsigned char* kg = reinterpret_cast<const unsigned char*>(static_cast<const T*>(a.k) +
                                                                   ((int64_t)h * a.T + t0) * D);
  const unsigned char* vg = reinterpret_cast<const unsigned char*>(static_cast<const T*>(a.v) +
                                                                   ((int64_t)h * a.T + t0) * D);
  auto stage_k = [&](int i) { return dsm + (i % kDStages) * 2 * kDPartBytes; };
  auto issue = [&](int i) {  // thread 0
    if (i < nst) {
      const int r0 = e0 + i * R, n = min(R, e1 - r0);
      uint64_t* bar = &full[i % kDStages];
      asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_u32(bar)),
                   "r"(2 * n * RB)
                   : "memory");
      d_bulk_load(stage_k(i), kg + (int64_t)r0 * RB, n * RB, bar);
      d_bulk_load(stage_k(i) + kDPartBytes, vg + (int64_t)r0 * RB, n * RB, bar);
    }
  };
  if (tid == 0) {
    for (int i = 0; i < kDStages; ++i) d_mbar_init(&full[i]);
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    for (int i = 0; i < kDStages; ++i) issue(i);
  }
  __syncthreads();

  float qf[GP][E];
  {
    const T* q = static_cast<const T*>(a.q) + ((int64_t)b * a.Hq + (int64_t)h * a.G) * D + li * E;
#pragma unroll
    for (int g = 0; g < GP; ++g) {
      if (g < a.G) {
        Vec16<T>::unpack(ld16(q + (int64_t)g * D), qf[g]);
      } else {
#pragma unroll
        for (int e = 0; e < E; ++e) qf[g][e] = 0.0f;
      }
    }
  }
  float m[GP], l[GP], o[GP][E];
#pragma unroll
  for (int g = 0; g < GP; ++g) {
    m[g] = -INFINITY;
    l[g] = 0.0f;
#pragma unroll
    for (int e = 0; e < E; ++e) o[g][e] = 0.0f;
  }

  for (int i = 0; i < nst; ++i) {
    bool late = false;
    {
      uint32_t it = 0;
      while (!d_mbar_try_wait(&full[i % kDStages], (uint32_t)(i / kDStages) & 1u)) {
        if (++it == kDWaitLimit) {
          late = true;
          break;
        }
      }
    }
    if (__syncthreads_or(late)) {  // a stage never arrived: report, drain, stop
      if (tid == 0) {
        flag_status(a.status, PRISM_DEV_TIMEOUT);
        for (int j = i; j < nst && j < i + kDStages; ++j) {
          uint32_t it = 0;
          while (!d_mbar_try_wait(&full[j % kDStages], (uint32_t)(j / kDStages) & 1u) && ++it < kDWaitLimit) {
          }
        }
      }
      return;
    }
    const unsigned char* ks = stage_k(i);
    const unsigned char* vs = ks + kDPartBytes;
    const int r0 = e0 + i * R, n = min(R, e1 - r0);
    uint4 kr[2], vr[2];
    bool ok[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int r = u * PASS + slot;
      ok[u] = r < n;
      kr[u] = ok[u] ? *reinterpret_cast<const uint4*>(ks + r * RB + li * 16) : make_uint4(0, 0, 0, 0);
      vr[u] = ok[u] ? *reinterpret_cast<const uint4*>(vs + r * RB + li * 16) : make_uint4(0, 0, 0, 0);
    }
    __syncthreads();  // the stage is in registers: hand it back
    if (tid == 0) issue(i + kDStages);
    float lg[2][GP];
    if constexpr (LPR == 16 && GP == 4) {
      // both rows' four head dot products reduced over the 16 lanes of the
      // group at once, transposed (each exchange halves the values a lane
      // keeps), then every value broadcast from the lane that holds it
      float v[8];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        float f[E];
        Vec16<T>::unpack(kr[u], f);
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          float sdot = 0.0f;
#pragma unroll
          for (int e = 0; e < E; ++e) sdot = fmaf(qf[g][e], f[e], sdot);
          v[u * 4 + g] = sdot;
        }
      }
      const bool b8 = li & 8, b4 = li & 4, b2 = li & 2;
      float w[4];
#pragma unroll
      for (int j = 0; j < 4; ++j)
        w[j] = (b8 ? v[4 + j] : v[j]) + __shfl_xor_sync(0xffffffffu, b8 ? v[j] : v[4 + j], 8);
      float x[2];
#pragma unroll
      for (int j = 0; j < 2; ++j)
        x[j] = (b4 ? w[2 + j] : w[j]) + __shfl_xor_sync(0xffffffffu, b4 ? w[j] : w[2 + j], 4);
      float y = (b2 ? x[1] : x[0]) + __shfl_xor_sync(0xffffffffu, b2 ? x[0] : x[1], 2);
      y += __shfl_xor_sync(0xffffffffu, y, 1);  // value (li >> 1) & 7: row u = bit 2, head = bits 0-1
#pragma unroll
      for (int vi = 0; vi < 8; ++vi) {
        const float sdot = __shfl_sync(0xffffffffu, y, (lane & 16) + 2 * vi);
        lg[vi >> 2][vi & 3] = ok[vi >> 2] ? sdot * a.scale_log2 : -INFINITY;
      }
    } else {
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        float f[E];
        Vec16<T>::unpack(kr[u], f);
#pragma unroll
        for (int g = 0; g < GP; ++g) {
          float sdot = 0.0f;
#pragma unroll
          for (int e = 0; e < E; ++e) sdot = fmaf(qf[g][e], f[e], sdot);
          sdot = group_sum<LPR>(sdot);
          lg[u][g] = ok[u] ? sdot * a.scale_log2 : -INFINITY;
        }
      }
    }
    float vf[2][E];
#pragma unroll
    for (int u = 0; u < 2; ++u) Vec16<T>::unpack(vr[u], vf[u]);
#pragma unroll
    for (int g = 0; g < GP; ++g) {
      // the accumulators are rescaled only when the running maximum grows
      // (the same value per lane group, so the branch is uniform there)
      const float mx = fmaxf(lg[0][g], lg[1][g]);
      if (mx > m[g]) {
        const float alpha = exp2f(m[g] - mx);  // 0 while nothing was seen
        l[g] *= alpha;
#pragma unroll
        for (int e = 0; e < E; ++e) o[g][e] *= alpha;
        m[g] = mx;
      }
      if (m[g] == -INFINITY) continue;
      const float p0 = exp2f(lg[0][g] - m[g]), p1 = exp2f(lg[1][g] - m[g]);
      l[g] += p0 + p1;
#pragma unroll
      for (int e = 0; e < E; ++e) o[g][e] = fmaf(p1, vf[1][e], fmaf(p0, vf[0][e], o[g][e]));
    }
  }

  // combine the CTA's lane groups in slot order (the ring is free now)
  float* s_o = reinterpret_cast<float*>(dsm);  // [SLOTS][GP][D]
  float* s_m = s_o + SLOTS * GP * D;           // [SLOTS][GP]
  float* s_l = s_m + SLOTS * GP;               // [SLOTS][GP]
#pragma unroll
  for (int g = 0; g < GP; ++g) {
#pragma unroll
    for (int e = 0; e < E; ++e) s_o[(slot * GP + g) * D + li * E + e] = o[g][e];
    if (li == 0) {
      s_m[slot * GP + g] = m[g];
      s_l[slot * GP + g] = l[g];
    }
  }
  __syncthreads();
  for (int x = tid; x < a.G * D; x += kDThreads) {
    const int g = x / D, j = x - g * D;
    float M = -INFINITY;
#pragma unroll
    for (int sl = 0; sl < SLOTS; ++sl) M = fmaxf(M, s_m[sl * GP + g]);
    float Ls = 0.0f, O = 0.0f;
    if (M != -INFINITY) {
#pragma unroll
      for (int sl = 0; sl < SLOTS; ++sl) {
        const float ms = s_m[sl * GP + g];
        const float w = ms == -INFINITY ? 0.0f : exp2f(ms - M);
        Ls = fmaf(w, s_l[sl * GP + g], Ls);
        O = fmaf(w, s_o[(sl * GP + g) * D + j], O);
      }
    }
    const int64_t pr = ((int64_t)b * a.Hq + (int64_t)h * a.G + g) * a.splits + split;
    a.part_o[pr * D + j] = O;
    if (j == 0) {
      a.part_ml[pr * 2] = M;
      a.part_ml[pr * 2 + 1] = Ls;
    }
  }
}

// dense shared memory: the stage ring, which also holds the lane groups'
// partials at the end
template <typename T, int D, int GP>
constexpr int dense_smem() {
  constexpr int ring = kDStages * 2 * kDPartBytes;
  constexpr int slots = kDWarps * (32 / (D / Vec16<T>::E));
  constexpr int comb = (slots * GP * D + 2 * slots * GP) * 4;
  return ring > comb ? ring : comb;
}

// ---- dense pass on tensor cores (bf16 cache, up to 8 query heads per KV head)
//
// Stages of kTRows = 128 contiguous K rows and the same V rows arrive by 2D
// tensor copies with the 128-byte swizzle (16-byte chunk c of row r of a
// 64-feature box at r * 128 + ((c ^ (r & 7)) << 4)), so eight rows read at
// one chunk by ldmatrix hit eight bank groups.  Warp w takes rows
// [16 w, 16 w + 16) of every stage:
//   S = K_w Q^T      mma m16n8k16: 16 rows x 8 heads, k over d (Q in registers)
//   per head: online softmax over the 16 rows (log2 domain, the accumulators
//   rescaled only when the running maximum grows)
//   O^T += V_w^T P^T mma m16n8k16: 16 features x 8 heads, k over the rows;
//   V^T by transposing ldmatrix, P^T by movmatrix from S's accumulator
//   layout, as three bf16 parts whose sum is p to 2^-24 relative
// bf16 operands make every product exact in fp32; the sums are fp32.  One CTA
// per SM keeps 192 KB of stages in flight.
constexpr int kTRows = 128;
constexpr int kTBox = kTRows * 128;  // one tensor copy: 128 rows x 64 features

template <int D>
__host__ __device__ constexpr int tc_part() { return kTRows * D * 2; }  // one stage's K (or V) bytes
template <int D>
__host__ __device__ constexpr int tc_stages() { return D == 128 ? 3 : 6; }
template <int D>
__host__ __device__ constexpr int tc_smem() { return tc_stages<D>() * 2 * tc_part<D>() + 1024; }  // + alignment

__device__ __forceinline__ void t_ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void t_ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ uint32_t t_movtrans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(y) : "r"(x));
  return y;
}
__device__ __forceinline__ void t_mma(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t t_bits(__nv_bfloat162 x) { return *reinterpret_cast<uint32_t*>(&x); }
// rows [y, y + 128) x features [x, x + 64) into a swizzled box; completes on bar
__device__ __forceinline__ void t_box(unsigned char* dst, const CUtensorMap* tm, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];\n" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

template <int D, int GP>
__global__ void __launch_bounds__(kDThreads, 1)
    dense_tc_kernel(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                    const AttendArgs a) {
  static_assert(GP <= 8, "eight heads per tile");
  constexpr int S = tc_stages<D>();
  constexpr int PB = tc_part<D>();
  constexpr int BOX = D / 64;  // tensor copies per part
  constexpr int KS = D / 16;   // k-steps of S = K Q^T, and 16-feature tiles of O^T
  constexpr int SLOTS = kDWarps;
  extern __shared__ unsigned char dsm_raw[];
  __shared__ __align__(8) uint64_t full[S];
  unsigned char* dsm = dsm_raw + ((1024u - (smem_u32(dsm_raw) & 1023u)) & 1023u);

  const int row = blockIdx.x, split = blockIdx.y;
  const int b = row / a.Hkv, h = row - b * a.Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int t0 = a.cu[b];
  const int L = a.cu[b + 1] - t0;
  const int e0 = split * a.per_split;
  const int e1 = min(L, e0 + a.per_split);
  const int nst = e1 > e0 ? (e1 - e0 + kTRows - 1) / kTRows : 0;
  const int64_t y0 = (int64_t)h * a.T + t0 + e0;  // tensor row of the split's first position
  auto stage = [&](int i) { return dsm + (i % S) * 2 * PB; };
  auto issue = [&](int i) {  // thread 0
    if (i < nst) {
      uint64_t* bar = &full[i % S];
      asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_u32(bar)),
                   "r"(2 * PB)
                   : "memory");
      const int y = (int)(y0 + (int64_t)i * kTRows);
#pragma unroll
      for (int x = 0; x < BOX; ++x) {
        t_box(stage(i) + x * kTBox, &tk, x * 64, y, bar);
        t_box(stage(i) + PB + x * kTBox, &tv, x * 64, y, bar);
      }
    }
  };
  if (tid == 0) {
    asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(&tk)) : "memory");
    asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(&tv)) : "memory");
    for (int i = 0; i < S; ++i) d_mbar_init(&full[i]);
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    for (int i = 0; i < S; ++i) issue(i);
  }
  // B operand of S = K Q^T: b0 = q_g[16 j + 2 t, + 1], b1 = q_g[16 j + 2 t + 8, + 9]
  uint32_t qb[KS][2];
  {
    const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(a.q) +
                             ((int64_t)b * a.Hq + (int64_t)h * a.G + (g < a.G ? g : 0)) * D + 2 * t;
#pragma unroll
    for (int j = 0; j < KS; ++j) {
      qb[j][0] = g < a.G ? *reinterpret_cast<const uint32_t*>(q + 16 * j) : 0u;
      qb[j][1] = g < a.G ? *reinterpret_cast<const uint32_t*>(q + 16 * j + 8) : 0u;
    }
  }
  __syncthreads();

  // O^T tile mt: (feature 16 mt + g, heads 2t, 2t+1) and (feature 16 mt + g + 8, same)
  float acc[KS][4];
#pragma unroll
  for (int mt = 0; mt < KS; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.0f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.0f, l1 = 0.0f;  // heads 2t, 2t + 1
  const int mi = lane >> 3, rr = lane & 7;
  const int kr = 16 * warp + (mi & 1) * 8 + rr;   // K: matrix mi = (row half mi & 1, chunk half mi >> 1)
  const int vr = 16 * warp + (mi >> 1) * 8 + rr;  // V: matrix mi = (row half mi >> 1, chunk half mi & 1)

  for (int i = 0; i < nst; ++i) {
    bool late = false;
    {
      uint32_t it = 0;
      while (!d_mbar_try_wait(&full[i % S], (uint32_t)(i / S) & 1u)) {
        if (++it == kDWaitLimit) {
          late = true;
          break;
        }
      }
    }
    if (__syncthreads_or(late)) {  // a stage never arrived: report, drain, stop
      if (tid == 0) {
        flag_status(a.status, PRISM_DEV_TIMEOUT);
        for (int j = i; j < nst && j < i + S; ++j) {
          uint32_t it = 0;
          while (!d_mbar_try_wait(&full[j % S], (uint32_t)(j / S) & 1u) && ++it < kDWaitLimit) {
          }
        }
      }
      return;
    }
    const uint32_t kb = smem_u32(stage(i)), vb = kb + PB;
    uint32_t kf[KS][4], vf[KS][4];
#pragma unroll
    for (int j = 0; j < KS; ++j) {
      const int ck = 2 * j + (mi >> 1), cv = 2 * j + (mi & 1);
      t_ldsm_x4(kb + (ck >> 3) * kTBox + kr * 128 + (((ck & 7) ^ (kr & 7)) << 4), kf[j]);
      t_ldsm_x4_trans(vb + (cv >> 3) * kTBox + vr * 128 + (((cv & 7) ^ (vr & 7)) << 4), vf[j]);
    }
    __syncthreads();  // the stage is in registers: hand it back
    if (tid == 0) issue(i + S);
    const int nv = min(kTRows, e1 - (e0 + i * kTRows)) - 16 * warp;  // valid rows of the warp's tile
    if (nv <= 0) continue;
    float sv[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
    for (int j = 0; j < KS; ++j) t_mma(sv, kf[j], qb[j][0], qb[j][1]);
    const bool ok0 = g < nv, ok1 = g + 8 < nv;
    const float x0 = ok0 ? sv[0] * a.scale_log2 : -INFINITY;  // row g, head 2t
    const float x1 = ok0 ? sv[1] * a.scale_log2 : -INFINITY;  // row g, head 2t + 1
    const float x2 = ok1 ? sv[2] * a.scale_log2 : -INFINITY;  // row g + 8, head 2t
    const float x3 = ok1 ? sv[3] * a.scale_log2 : -INFINITY;  // row g + 8, head 2t + 1
    float mx0 = fmaxf(x0, x2), mx1 = fmaxf(x1, x3);
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
    }
    if (mx0 > m0) {  // row 0 of the tile is valid, so mx0 is finite
      const float al = exp2f(m0 - mx0);
      l0 *= al;
#pragma unroll
      for (int mt = 0; mt < KS; ++mt) {
        acc[mt][0] *= al;
        acc[mt][2] *= al;
      }
      m0 = mx0;
    }
    if (mx1 > m1) {
      const float al = exp2f(m1 - mx1);
      l1 *= al;
#pragma unroll
      for (int mt = 0; mt < KS; ++mt) {
        acc[mt][1] *= al;
        acc[mt][3] *= al;
      }
      m1 = mx1;
    }
    const float p0 = exp2f(x0 - m0), p1 = exp2f(x1 - m1), p2 = exp2f(x2 - m0), p3 = exp2f(x3 - m1);
    l0 += p0 + p2;
    l1 += p1 + p3;
    // P (rows x heads) packed by rows, each 8 x 8 block transposed into the
    // B operand (k = rows, n = heads): b0 rows 0-7, b1 rows 8-15
    uint32_t bp[3][2];  // p = part 0 + part 1 + part 2, each bf16: exact to 2^-24 p
    {
      float r0 = p0, r1 = p1, r2 = p2, r3 = p3;
#pragma unroll
      for (int u = 0; u < 3; ++u) {
        const __nv_bfloat162 c01 = __floats2bfloat162_rn(r0, r1), c23 = __floats2bfloat162_rn(r2, r3);
        bp[u][0] = t_movtrans(t_bits(c01));
        bp[u][1] = t_movtrans(t_bits(c23));
        const float2 f01 = __bfloat1622float2(c01), f23 = __bfloat1622float2(c23);
        r0 -= f01.x;  // exact: r and its bf16 rounding share the leading bits
        r1 -= f01.y;
        r2 -= f23.x;
        r3 -= f23.y;
      }
    }
    if (nv < 16) {  // rows past the split carry no weight, and their bytes may be anything
      const uint32_t k0 = (2 * t < nv ? 0x0000FFFFu : 0u) | (2 * t + 1 < nv ? 0xFFFF0000u : 0u);
      const uint32_t k1 = (2 * t + 8 < nv ? 0x0000FFFFu : 0u) | (2 * t + 9 < nv ? 0xFFFF0000u : 0u);
#pragma unroll
      for (int mt = 0; mt < KS; ++mt) {
        vf[mt][0] &= k0;
        vf[mt][1] &= k0;
        vf[mt][2] &= k1;
        vf[mt][3] &= k1;
      }
    }
#pragma unroll
    for (int mt = 0; mt < KS; ++mt)
#pragma unroll
      for (int u = 0; u < 3; ++u) t_mma(acc[mt], vf[mt], bp[u][0], bp[u][1]);
  }
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, o);
    l1 += __shfl_xor_sync(0xffffffffu, l1, o);
  }

  // combine the warps in warp order (the ring is free now)
  float* s_o = reinterpret_cast<float*>(dsm);  // [SLOTS][GP][D]
  float* s_m = s_o + SLOTS * GP * D;           // [SLOTS][GP]
  float* s_l = s_m + SLOTS * GP;               // [SLOTS][GP]
  const int ha = 2 * t, hb = 2 * t + 1;
#pragma unroll
  for (int mt = 0; mt < KS; ++mt) {
    if (ha < GP) {
      s_o[(warp * GP + ha) * D + 16 * mt + g] = acc[mt][0];
      s_o[(warp * GP + ha) * D + 16 * mt + g + 8] = acc[mt][2];
    }
    if (hb < GP) {
      s_o[(warp * GP + hb) * D + 16 * mt + g] = acc[mt][1];
      s_o[(warp * GP + hb) * D + 16 * mt + g + 8] = acc[mt][3];
    }
  }
  if (g == 0) {
    if (ha < GP) {
      s_m[warp * GP + ha] = m0;
      s_l[warp * GP + ha] = l0;
    }
    if (hb < GP) {
      s_m[warp * GP + hb] = m1;
      s_l[warp * GP + hb] = l1;
    }
  }
  __syncthreads();
  for (int x = tid; x < a.G * D; x += kDThreads) {
    const int gg = x / D, j = x - gg * D;
    float M = -INFINITY;
#pragma unroll
    for (int sl = 0; sl < SLOTS; ++sl) M = fmaxf(M, s_m[sl * GP + gg]);
    float Ls = 0.0f, O = 0.0f;
    if (M != -INFINITY) {
#pragma unroll
      for (int sl = 0; sl < SLOTS; ++sl) {
        const float ms = s_m[sl * GP + gg];
        const float w = ms == -INFINITY ? 0.0f : exp2f(ms - M);
        Ls = fmaf(w, s_l[sl * GP + gg], Ls);
        O = fmaf(w, s_o[(sl * GP + gg) * D + j], O);
      }
    }
    const int64_t pr = ((int64_t)b * a.Hq + (int64_t)h * a.G + gg) * a.splits + split;
    a.part_o[pr * D + j] = O;
    if (j == 0) {
      a.part_ml[pr * 2] = M;
      a.part_ml[pr * 2 + 1] = Ls;
    }
  }
}

// The tensor-core dense kernel, when the cache can be described by tensor
// maps (bf16, 16-byte aligned bases, fewer than 2^31 rows); false otherwise.
template <int D, int GP>
bool run_dense_tc(const Dims& d, const AttendPlan& p, const AttendArgs& a, cudaStream_t st, cudaError_t* err) {
  const PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
  if (!encode || (reinterpret_cast<uintptr_t>(a.k) & 15) || (reinterpret_cast<uintptr_t>(a.v) & 15))
    return false;
  const uint64_t nrows = (uint64_t)d.Hkv * (uint64_t)d.T;
  if (nrows == 0 || nrows > 0x7fffff00ull) return false;  // row coordinates + 128 fit an int
  CUtensorMap tk, tv;
  const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)nrows};
  const cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)kTRows};
  const cuuint32_t estr[2] = {1, 1};
  for (int x = 0; x < 2; ++x) {
    if (encode(x ? &tv : &tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x ? a.v : a.k), dims,
               strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return false;
  }
  constexpr int smem = tc_smem<D>();
  auto kd = dense_tc_kernel<D, GP>;
  cudaError_t e = cudaFuncSetAttribute(kd, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess) {
    kd<<<dim3(d.B * d.Hkv, p.splits), kDThreads, smem, st>>>(tk, tv, a);
    e = cudaGetLastError();
  }
  *err = e;
  return true;
}

// One CTA of D threads per (sequence, query head): the split weights
// 2^(m_s - M) are computed in parallel into shared memory, then thread j sums
// its feature over the splits with independent (pipelined) loads.
template <int D>
__global__ void __launch_bounds__(D) merge_kernel(int splits, const float* __restrict__ part_o,
                                                 const float* __restrict__ part_ml,
                                                 float* __restrict__ out, float* __restrict__ lse) {
  extern __shared__ float s_w[];  // [splits]
  __shared__ float s_red[D / 32];
  __shared__ float s_M, s_L;
  const int w = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float* ml = part_ml + (int64_t)w * splits * 2;
  const float* po = part_o + (int64_t)w * splits * D;
  float M = -INFINITY;
  for (int s = tid; s < splits; s += D) M = fmaxf(M, ml[s * 2]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  if (lane == 0) s_red[warp] = M;
  __syncthreads();
  if (tid == 0) {
    float v = s_red[0];
    for (int i = 1; i < D / 32; ++i) v = fmaxf(v, s_red[i]);
    s_M = v;
  }
  __syncthreads();
  M = s_M;
  float Ls = 0.0f;
  for (int s = tid; s < splits; s += D) {
    const float ms = ml[s * 2];
    const float wt = (M == -INFINITY || ms == -INFINITY) ? 0.0f : exp2f(ms - M);
    s_w[s] = wt;
    Ls = fmaf(wt, ml[s * 2 + 1], Ls);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) Ls += __shfl_xor_sync(0xffffffffu, Ls, o);
  __syncthreads();
  if (lane == 0) s_red[warp] = Ls;
  __syncthreads();
  if (tid == 0) {
    float v = 0.0f;
    for (int i = 0; i < D / 32; ++i) v += s_red[i];
    s_L = v;
  }
  __syncthreads();
  Ls = s_L;
  float acc = 0.0f;
#pragma unroll 8
  for (int s = 0; s < splits; ++s) acc = fmaf(s_w[s], po[(int64_t)s * D + tid], acc);
  const bool any = Ls > 0.0f;
  out[(int64_t)w * D + tid] = any ? acc / Ls : 0.0f;
  if (lse && tid == 0) lse[w] = any ? (M + log2f(Ls)) * 0.69314718055994530942f : -INFINITY;
}

template <typename T, int D, int GP>
cudaError_t run(const Dims& d, const AttendPlan& p, const AttendArgs& a, cudaStream_t st) {
  if (!a.idx) {  // dense: the tensor-core kernel, else the staged one
    if constexpr (std::is_same<T, __nv_bfloat16>::value && GP <= 8) {
      cudaError_t e;
      if (run_dense_tc<D, GP>(d, p, a, st, &e)) return e;
    }
    constexpr int smem = dense_smem<T, D, GP>();
    auto kd = dense_kernel<T, D, GP>;
    cudaError_t e = cudaFuncSetAttribute(kd, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    kd<<<dim3(d.B * d.Hkv, p.splits), kDThreads, smem, st>>>(a);
    return cudaGetLastError();
  }
  constexpr int RPW = 32 / (D / Vec16<T>::E);
  constexpr int SLOTS = kWarps * RPW;
  const int smem = (SLOTS * GP * D + 2 * SLOTS * GP) * (int)sizeof(float);
  auto k = attend_kernel<T, D, GP>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
  }
  k<<<dim3(d.B * d.Hkv, p.splits), kThreads, smem, st>>>(a);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t by_group(const Dims& d, const AttendPlan& p, const AttendArgs& a, cudaStream_t st) {
  switch (padded_group(d.G)) {
    case 1: return run<T, D, 1>(d, p, a, st);
    case 2: return run<T, D, 2>(d, p, a, st);
    case 4: return run<T, D, 4>(d, p, a, st);
    case 8: return run<T, D, 8>(d, p, a, st);
    default: return run<T, D, 16>(d, p, a, st);
  }
}

}  // namespace

namespace {

// Makespan, in row units, of the tensor-core dense grid (splits of `per`
// rows, launched split-major and row-minor, one CTA per SM at a time) under
// greedy placement: a CTA costs its rows plus a fixed start, an empty one
// only the start of a CTA that exits.
int64_t tc_makespan(const Dims& d, int64_t per, int64_t splits) {
  constexpr int64_t kStart = 256, kEmpty = 32;
  std::priority_queue<int64_t, std::vector<int64_t>, std::greater<int64_t>> free_at;
  for (int i = 0; i < d.num_sms; ++i) free_at.push(0);
  int64_t end = 0;
  for (int64_t s = 0; s < splits; ++s)
    for (int b = 0; b < d.B; ++b) {
      const int64_t L = d.cu_host ? (int64_t)d.cu_host[b + 1] - d.cu_host[b] : d.max_len;
      const int64_t w = std::min(L, (s + 1) * per) - s * per;
      const int64_t c = w > 0 ? w + kStart : kEmpty;
      for (int h = 0; h < d.Hkv; ++h) {
        const int64_t t = free_at.top() + c;
        free_at.pop();
        free_at.push(t);
        end = std::max(end, t);
      }
    }
  return end;
}

}  // namespace

AttendPlan plan_attend(const Dims& d, int64_t max_rows_per_seq, bool dense) {
  const int64_t maxl = max_rows_per_seq > 0 ? max_rows_per_seq : 1;
  if (dense && d.bf16 && padded_group(d.G) <= 8 && d.num_sms > 0) {
    // tensor-core dense: 128-row stages, one CTA per SM.  Split lengths for
    // 1, 2, 3, 4, 6 or 8 waves of the rows' CTAs; the shortest simulated
    // makespan wins (equal lengths fill one wave exactly, ragged ones need
    // shorter splits to spread the long rows)
    const int64_t rows = std::max<int64_t>(1, (int64_t)d.B * d.Hkv);
    AttendPlan best{1, (int)(cdiv(maxl, 128) * 128)};
    if (rows >= 8LL * d.num_sms) return best;  // one CTA per row: many waves already
    int64_t best_t = -1;
    for (int w : {1, 2, 3, 4, 6, 8}) {
      const int64_t s0 = std::max<int64_t>(1, (int64_t)w * d.num_sms / rows);
      int64_t per = cdiv(cdiv(maxl, s0), 128) * 128;
      const int64_t splits = cdiv(maxl, per);
      const int64_t t = tc_makespan(d, per, splits);
      if (best_t < 0 || t < best_t) {
        best_t = t;
        best = AttendPlan{(int)splits, (int)per};
      }
    }
    return best;
  }
  // rows one CTA covers per iteration: a sparse pass step (bf16, d = 128), or
  // a dense stage (the largest, fp32 d = 64: 64 rows, so every dtype's
  // stage divides it)
  const int step = dense ? 64 : 16;
  const int64_t rows = (int64_t)d.B * d.Hkv;
  // dense: one wave of two CTAs per SM; sparse: four CTAs per SM
  const int64_t target = (dense ? 2LL : 4LL) * d.num_sms;
  int64_t splits = rows > 0 ? cdiv(target, rows) : 1;
  const int64_t max_splits = cdiv(max_rows_per_seq > 0 ? max_rows_per_seq : 1, step);
  if (splits > max_splits) splits = max_splits;
  if (splits < 1) splits = 1;
  int64_t per = cdiv(max_rows_per_seq > 0 ? max_rows_per_seq : 1, splits);
  per = cdiv(per, step) * step;
  splits = cdiv(max_rows_per_seq > 0 ? max_rows_per_seq : 1, per);
  return AttendPlan{(int)splits, (int)per};
}

cudaError_t launch_attend(const Dims& d, const AttendPlan& p, const void* q, const void* k,
                          const void* v, const int32_t* idx, const int32_t* cnt, int idx_stride,
                          float softmax_scale, float* part_o, float* part_ml, float* out,
                          float* lse, int32_t* status, cudaStream_t st, int kv_div, int idx_div) {
  if (d.B * d.Hq == 0) return cudaSuccess;
  AttendArgs a{q, k, v, d.cu_dev, idx, cnt, idx_stride, d.Hkv, d.G, d.Hq, d.T,
               p.per_split, p.splits, softmax_scale * 1.4426950408889634f, part_o, part_ml, status,
               kv_div > 1 ? kv_div : 1, idx_div > 1 ? idx_div : 1};
  cudaError_t e;
  if (d.bf16)
    e = d.D == 128 ? by_group<__nv_bfloat16, 128>(d, p, a, st) : by_group<__nv_bfloat16, 64>(d, p, a, st);
  else
    e = d.D == 128 ? by_group<float, 128>(d, p, a, st) : by_group<float, 64>(d, p, a, st);
  if (e != cudaSuccess) return e;
  const int BHq = d.B * d.Hq;
  const size_t smem = (size_t)p.splits * sizeof(float);
  if (d.D == 128)
    merge_kernel<128><<<BHq, 128, smem, st>>>(p.splits, part_o, part_ml, out, lse);
  else
    merge_kernel<64><<<BHq, 64, smem, st>>>(p.splits, part_o, part_ml, out, lse);
  return cudaGetLastError();
}

}  // namespace prism
