// Proposal scoring over the quantized key cache (Prism Attention, sec. 4.1
// "Proposal-Refined Index Sharing" and sec. 4.2 "Quantized Proposal
// Construction"):
//   s[h][t] = k_scale[h][t] * max_{g<G} sum_j q[b][h*G+g][j] * kq[h][t][j]
// for every position of every sequence, written as fp32 [Hkv][T].
//
// This is the bandwidth-dominant step of a decode step: d + 4 bytes per key
// row and per KV head (132 B at d = 128).  Per row it also does G*d
// multiply-adds plus d int8 -> float conversions, which at G = 4 is close to
// the fp32 pipe's limit at full HBM rate, so two kernels exist:
//
//  * score_mma_kernel (bf16 queries): tensor cores.  Key rows are the M
//    dimension of mma.sync.m16n8k16 (f16 x f16 -> f32), the G query heads the
//    N dimension.  int8 codes convert exactly to fp16 with one byte-permute
//    and one packed subtraction per pair; the bf16 query is scaled by a power
//    of two so that its largest element lands in [2^14, 2^15) and converted
//    to fp16, exact for every element down to 2^-31 of the largest; products
//    are exact and accumulate in fp32.  The feature axis is permuted so that
//    each thread's A-fragment elements are two contiguous 16-byte pieces of
//    its rows (the same permutation is applied to the query), so rows load
//    straight from global memory with fully used 32-byte sectors, double
//    buffered in registers.
//  * score_simt_kernel: plain fp32 FMAs on CUDA cores (fp32 queries, and the
//    comparison kernel for bf16).
#include "common.cuh"
#include "kernels.h"

namespace prism {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kChunkRows = 1024;  // key rows of one (sequence, KV head) per work item

struct ScoreArgs {
  const void* q;
  const int8_t* kq;
  const float* scale;
  float* scores;
  const int32_t* cu;
  int64_t T;
  int B, Hkv, G;
};

// s_pref[b] = number of work items of sequences before b (per KV head).
__device__ void chunk_prefix(const int32_t* __restrict__ cu, int B, int* s_pref) {
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    int carry = 0;
    for (int b0 = 0; b0 < B; b0 += 32) {
      const int b = b0 + lane;
      int n = 0;
      if (b < B) n = (cu[b + 1] - cu[b] + kChunkRows - 1) / kChunkRows;
      const int inc = warp_incl_scan(n);
      if (b < B) s_pref[b + 1] = carry + inc;
      carry += __shfl_sync(0xffffffffu, inc, 31);
    }
    if (lane == 0) s_pref[0] = 0;
  }
  __syncthreads();
}

// The sequence owning work item c: s_pref[b] <= c < s_pref[b + 1].
__device__ __forceinline__ int find_seq(const int* s_pref, int B, int c) {
  int lo = 0, hi = B;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (s_pref[mid] <= c) lo = mid; else hi = mid;
  }
  return lo;
}

// Four int8 codes -> two fp16 pairs, exactly: bytes biased by 128 become the
// low mantissa byte of fp16 1024 + u, then 1152 = 1024 + 128 is subtracted.
__device__ __forceinline__ void i8x4_to_f16(uint32_t w, uint32_t& lo, uint32_t& hi) {
  const uint32_t x = w ^ 0x80808080u;
  lo = __byte_perm(x, 0x64646464u, 0x4140);
  hi = __byte_perm(x, 0x64646464u, 0x4342);
  asm("sub.rn.f16x2 %0, %0, %1;" : "+r"(lo) : "r"(0x64806480u));
  asm("sub.rn.f16x2 %0, %0, %1;" : "+r"(hi) : "r"(0x64806480u));
}

__device__ __forceinline__ uint32_t pack_f16(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t word_of(const uint4& v, int i) {
  return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

// Tensor-core scorer.  NT = number of 8-wide query-head tiles (G <= 8*NT).
template <int D, int NT>
__global__ void __launch_bounds__(kThreads) score_mma_kernel(ScoreArgs a) {
  constexpr int KS = D / 16;   // k-steps of 16 features
  constexpr int NCH = D / 64;  // 16-byte pieces per thread per row
  extern __shared__ int s_pref[];
  chunk_prefix(a.cu, a.B, s_pref);
  const int per_head = s_pref[a.B];
  const int64_t total = (int64_t)a.Hkv * per_head;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, tig = lane & 3;
  const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(a.q);

  for (int64_t c = blockIdx.x; c < total; c += gridDim.x) {
    const int h = (int)(c / per_head);
    const int cc = (int)(c - (int64_t)h * per_head);
    const int b = find_seq(s_pref, a.B, cc);
    const int t0 = a.cu[b];
    const int r0 = (cc - s_pref[b]) * kChunkRows;
    const int rows = min(kChunkRows, a.cu[b + 1] - t0 - r0);
    const int64_t rowbase = (int64_t)h * a.T + t0 + r0;

    // Query fragments (B operand, "col" layout): thread (g, tig) holds
    // column n = g of each head tile; k-step s covers features
    // base(s) .. base(s)+3 with base(s) = 64*(s/4) + 16*tig + 4*(s%4).
    uint32_t bq[NT][KS][2];
    int qexp;
    {
      float qv[NT][KS][4];
      float mx = 0.0f;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int n = nt * 8 + g;
#pragma unroll
        for (int s = 0; s < KS; ++s) {
          const int base = 64 * (s / 4) + 16 * tig + 4 * (s % 4);
          if (n < a.G) {
            const uint2 w = *reinterpret_cast<const uint2*>(
                q + ((int64_t)b * a.Hkv * a.G + (int64_t)h * a.G + n) * D + base);
            qv[nt][s][0] = bf16lo(w.x); qv[nt][s][1] = bf16hi(w.x);
            qv[nt][s][2] = bf16lo(w.y); qv[nt][s][3] = bf16hi(w.y);
          } else {
            qv[nt][s][0] = qv[nt][s][1] = qv[nt][s][2] = qv[nt][s][3] = 0.0f;
          }
#pragma unroll
          for (int e = 0; e < 4; ++e) mx = fmaxf(mx, fabsf(qv[nt][s][e]));
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      int e2 = 0;
      frexpf(mx, &e2);  // mx < 2^e2
      qexp = (mx > 0.0f) ? 15 - e2 : 0;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int s = 0; s < KS; ++s) {
          bq[nt][s][0] = pack_f16(ldexpf(qv[nt][s][0], qexp), ldexpf(qv[nt][s][1], qexp));
          bq[nt][s][1] = pack_f16(ldexpf(qv[nt][s][2], qexp), ldexpf(qv[nt][s][3], qexp));
        }
    }

    const int ntiles = (rows + 15) / 16;
    uint4 cur[2][NCH], nxt[2][NCH];
    float csc = 0.0f, nsc = 0.0f;
    auto load = [&](int t, uint4 (&buf)[2][NCH], float& sc) {
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int r = t * 16 + g + 8 * half;
#pragma unroll
        for (int ch = 0; ch < NCH; ++ch)
          buf[half][ch] = (r < rows) ? ld16_stream(a.kq + (rowbase + r) * D + ch * 64 + tig * 16)
                                     : make_uint4(0, 0, 0, 0);
      }
      const int rs = t * 16 + g + 8 * tig;  // tig 0: row g, tig 1: row g + 8
      sc = (tig < 2 && rs < rows) ? __ldg(a.scale + rowbase + rs) : 0.0f;
    };
    int t = warp;
    if (t < ntiles) load(t, cur, csc);
    for (; t < ntiles; t += kWarps) {
      const int tn = t + kWarps;
      if (tn < ntiles) load(tn, nxt, nsc);
      float acc[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.0f;
#pragma unroll
      for (int s = 0; s < KS; ++s) {
        uint32_t a0, a1, a2, a3;
        i8x4_to_f16(word_of(cur[0][s / 4], s % 4), a0, a2);  // row g
        i8x4_to_f16(word_of(cur[1][s / 4], s % 4), a1, a3);  // row g + 8
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma16816(acc[nt], a0, a1, a2, a3, bq[nt][s][0], bq[nt][s][1]);
      }
      float mA = -INFINITY, mB = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int col = nt * 8 + 2 * tig;
        if (col < a.G) { mA = fmaxf(mA, acc[nt][0]); mB = fmaxf(mB, acc[nt][2]); }
        if (col + 1 < a.G) { mA = fmaxf(mA, acc[nt][1]); mB = fmaxf(mB, acc[nt][3]); }
      }
      mA = fmaxf(mA, __shfl_xor_sync(0xffffffffu, mA, 1));
      mA = fmaxf(mA, __shfl_xor_sync(0xffffffffu, mA, 2));
      mB = fmaxf(mB, __shfl_xor_sync(0xffffffffu, mB, 1));
      mB = fmaxf(mB, __shfl_xor_sync(0xffffffffu, mB, 2));
      const int rs = t * 16 + g + 8 * tig;
      if (tig < 2 && rs < rows) a.scores[rowbase + rs] = csc * ldexpf(tig == 0 ? mA : mB, -qexp);
#pragma unroll
      for (int half = 0; half < 2; ++half)
#pragma unroll
        for (int ch = 0; ch < NCH; ++ch) cur[half][ch] = nxt[half][ch];
      csc = nsc;
    }
  }
}

// CUDA-core scorer: one thread per key row, query in shared memory (fp32).
template <typename T, int D, int GP>
__global__ void __launch_bounds__(kThreads) score_simt_kernel(ScoreArgs a) {
  extern __shared__ int smem[];
  int* s_pref = smem;
  float* sq = reinterpret_cast<float*>(smem + ((a.B + 1 + 3) & ~3));
  chunk_prefix(a.cu, a.B, s_pref);
  const int per_head = s_pref[a.B];
  const int64_t total = (int64_t)a.Hkv * per_head;
  const T* q = static_cast<const T*>(a.q);
  for (int64_t c = blockIdx.x; c < total; c += gridDim.x) {
    const int h = (int)(c / per_head);
    const int cc = (int)(c - (int64_t)h * per_head);
    const int b = find_seq(s_pref, a.B, cc);
    const int t0 = a.cu[b];
    const int r0 = (cc - s_pref[b]) * kChunkRows;
    const int rows = min(kChunkRows, a.cu[b + 1] - t0 - r0);
    const int64_t rowbase = (int64_t)h * a.T + t0 + r0;
    __syncthreads();
    for (int i = threadIdx.x; i < GP * D; i += blockDim.x) {
      const int gg = i / D, j = i % D;
      sq[i] = gg < a.G ? to_f32(q[((int64_t)b * a.Hkv * a.G + (int64_t)h * a.G + gg) * D + j]) : 0.0f;
    }
    __syncthreads();
    for (int r = threadIdx.x; r < rows; r += blockDim.x) {
      const int8_t* kr = a.kq + (rowbase + r) * D;
      float acc[GP];
#pragma unroll
      for (int gg = 0; gg < GP; ++gg) acc[gg] = 0.0f;
#pragma unroll 2
      for (int c16 = 0; c16 < D / 16; ++c16) {
        const uint4 raw = ld16(kr + c16 * 16);
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const uint32_t word = word_of(raw, w);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float v = (float)(int8_t)(word >> (8 * e));
            const int j = c16 * 16 + w * 4 + e;
#pragma unroll
            for (int gg = 0; gg < GP; ++gg) acc[gg] = fmaf(sq[gg * D + j], v, acc[gg]);
          }
        }
      }
      float best = acc[0];
#pragma unroll
      for (int gg = 1; gg < GP; ++gg)
        if (gg < a.G) best = fmaxf(best, acc[gg]);
      a.scores[rowbase + r] = a.scale[rowbase + r] * best;
    }
  }
}

template <typename K>
int grid_for(K kernel, int smem, int num_sms, int64_t total) {
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kThreads, smem) != cudaSuccess ||
      per_sm < 1)
    per_sm = 1;
  int64_t grid = (int64_t)per_sm * num_sms;
  if (grid > total) grid = total;
  return (int)(grid < 1 ? 1 : grid);
}

template <int D, int NT>
cudaError_t run_mma(const Dims& d, const ScoreArgs& a, int64_t total, cudaStream_t st) {
  const int smem = (d.B + 1) * (int)sizeof(int);
  auto k = score_mma_kernel<D, NT>;
  const int grid = grid_for(k, smem, d.num_sms, total);
  k<<<grid, kThreads, smem, st>>>(a);
  return cudaGetLastError();
}

template <typename T, int D, int GP>
cudaError_t run_simt(const Dims& d, const ScoreArgs& a, int64_t total, cudaStream_t st) {
  const int smem = (((d.B + 1 + 3) & ~3) + GP * D) * (int)sizeof(int);
  auto k = score_simt_kernel<T, D, GP>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
  }
  const int grid = grid_for(k, smem, d.num_sms, total);
  k<<<grid, kThreads, smem, st>>>(a);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t simt_by_group(const Dims& d, const ScoreArgs& a, int64_t total, cudaStream_t st) {
  switch (padded_group(d.G)) {
    case 1: return run_simt<T, D, 1>(d, a, total, st);
    case 2: return run_simt<T, D, 2>(d, a, total, st);
    case 4: return run_simt<T, D, 4>(d, a, total, st);
    case 8: return run_simt<T, D, 8>(d, a, total, st);
    default: return run_simt<T, D, 16>(d, a, total, st);
  }
}

}  // namespace

cudaError_t launch_propose_scores(const Dims& d, const void* q, const int8_t* kq,
                                  const float* scale, float* scores, bool use_mma,
                                  cudaStream_t st) {
  int64_t per_head = 0;
  for (int b = 0; b < d.B; ++b) per_head += cdiv(d.cu_host[b + 1] - d.cu_host[b], kChunkRows);
  const int64_t total = per_head * d.Hkv;
  if (total == 0) return cudaSuccess;
  ScoreArgs a{q, kq, scale, scores, d.cu_dev, d.T, d.B, d.Hkv, d.G};
  if (use_mma && d.bf16) {
    if (d.D == 128) return d.G <= 8 ? run_mma<128, 1>(d, a, total, st) : run_mma<128, 2>(d, a, total, st);
    return d.G <= 8 ? run_mma<64, 1>(d, a, total, st) : run_mma<64, 2>(d, a, total, st);
  }
  if (d.bf16) {
    return d.D == 128 ? simt_by_group<__nv_bfloat16, 128>(d, a, total, st)
                      : simt_by_group<__nv_bfloat16, 64>(d, a, total, st);
  }
  return d.D == 128 ? simt_by_group<float, 128>(d, a, total, st)
                    : simt_by_group<float, 64>(d, a, total, st);
}

}  // namespace prism
