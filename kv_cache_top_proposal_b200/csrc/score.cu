// Proposal scoring over the quantized key cache (Prism Attention, sec. 4.1
// "Proposal-Refined Index Sharing" and sec. 4.2 "Quantized Proposal
// Construction"):
//   s[h][t] = k_scale[h][t] * max_{g<G} sum_j q[b][h*G+g][j] * kq[h][t][j]
// for every position of every sequence, written as fp32 [Hkv][T].
//
// This is the bandwidth-dominant step of a decode step: d + 4 bytes per key
// row and per KV head (132 B at d = 128).  The kernels:
//
//  * score_i8_kernel (default; bf16 queries, d = 128, G <= 8): tensor copies
//    (cp.async.bulk.tensor, 128-row stages, evict-first in L2) feed integer
//    tensor cores (mma.sync.m16n8k32, s8): the stored codes are the A
//    operand as they are, each query head enters as four int8 limbs of a
//    31-bit fixed-point value, and the int32 sums are exact.  It can also
//    quantize this token's key rows into the codes (prism_propose_append)
//    and sum the group's heads instead of taking their maximum.
//  * score_tma_kernel and score_mma_kernel (bf16 queries): fp16 tensor
//    cores.  Key rows are the M dimension of mma.sync.m16n8k16, the G query
//    heads the N dimension; int8 codes convert exactly to fp16 with one
//    byte-permute and one packed subtraction per pair; the bf16 query is
//    scaled by a power of two so that its largest element lands in
//    [2^14, 2^15) and converted to fp16; products are exact and accumulate in
//    fp32.  The first moves stages by tensor copies, the second by cp.async
//    (PRISM_PROPOSE_SCORER=tma / =mma select them).
//  * score_int2_kernel: INT2 keys on fp16 tensor cores (codes as fp16
//    subnormals), cp.async stages.
//  * score_simt_kernel: plain fp32 FMAs on CUDA cores (fp32 queries, and the
//    comparison kernel for bf16).
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstdlib>
#include <cstring>

#include "common.cuh"
#include "kernels.h"

namespace prism {

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult res;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &res) != cudaSuccess ||
        res != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }();
  return fn;
}

namespace {

constexpr int kThreads = 256;
constexpr int kChunkRows = 1024;  // key rows of one (sequence, KV head) per work item

struct ScoreArgs {
  const void* q;
  const int8_t* kq;
  const float* scale;
  float* scores;
  uint32_t* hist;  // [B*Hkv][kHist] first-digit histogram of ord(score), or null
  const int32_t* cu;
  int64_t T;
  int B, Hkv, G;
  int32_t* status;
  const uint8_t* codes;    // INT2 keys: [Hkv][T][d/4], four codes per byte
  const uint16_t* params;  // INT2 keys: [Hkv][T][d/32][2] fp16 bits of (step, zero point)
  const void* k_new;       // integer scorer: [B][Hkv][d] new key rows to quantize at L_b - 1, or null
  int8_t* kq_w;            // with k_new: where its codes go (the same codes as kq)
  float* scale_w;          // with k_new: where its scales go
  int sum_group;           // integer scorer: sum over the group's query heads, not the maximum
};

// s_pref[b] = number of work items of sequences before b (per KV head).
__device__ void chunk_prefix(const int32_t* __restrict__ cu, int B, int rows_per_item, int* s_pref) {
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    int carry = 0;
    for (int b0 = 0; b0 < B; b0 += 32) {
      const int b = b0 + lane;
      int n = 0;
      if (b < B) n = (cu[b + 1] - cu[b] + rows_per_item - 1) / rows_per_item;
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

// Shared first-digit histogram with two 16-bit counts per word (bin b in
// word b / 2, high half when b is odd); lanes sharing a bin issue one atomic.
__device__ __forceinline__ void warp_hist_add_packed(uint32_t* hw, uint32_t bin, bool valid) {
  const unsigned act = __ballot_sync(0xffffffffu, valid);
  if (!act) return;
  const unsigned peers = __match_any_sync(0xffffffffu, valid ? bin : 0xffffffffu) & act;
  const int lane = threadIdx.x & 31;
  if (valid && (peers & ((1u << lane) - 1u)) == 0)
    atomicAdd(&hw[bin >> 1], (uint32_t)__popc(peers) << ((bin & 1u) * 16));
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
// Persistent CTAs walk a flat list of 128-row stages (stage s of KV head h,
// sequence b), kScoreStages of them in flight per CTA through a cp.async ring
// (codes + scales); warp w takes 16-row tile w of each stage.
constexpr int kStageRows = 128;
constexpr int kScoreStages = 5;
constexpr int kHist = 4096;  // first radix digit of the selection keys (12 bits)

template <int D>
struct StageLayout {
  static constexpr int ROWB = D;                         // int8 codes per row
  static constexpr int CODES = kStageRows * ROWB;        // code bytes per stage
  static constexpr int BYTES = CODES + kStageRows * 4;   // + fp32 scales
  // 16-byte chunk c of row r: rows g and g+1 of a quarter-warp read chunks
  // tig (and 4 + tig); flipping bit 2 on odd rows puts them in different
  // bank halves at d = 128
  __device__ __forceinline__ static int off(int r, int c) {
    return r * ROWB + ((D == 128 ? (c ^ ((r & 1) << 2)) : c) << 4);
  }
};

// 2^e as an exact float for e in [-126, 127]
__device__ __forceinline__ float pow2f(int e) { return __int_as_float((127 + e) << 23); }

// Walks stages (KV head h, sequence b, first row r0) in order, skipping empty
// sequences; cu is the shared-memory copy of cu_seqlens.  No divisions.
struct StageIter {
  int h, b, r0;
  __device__ __forceinline__ void advance(const int* cu, int B) {
    r0 += kStageRows;
    while (h >= 0 && r0 >= cu[b + 1] - cu[b]) {
      r0 = 0;
      if (++b == B) {
        b = 0;
        ++h;
      }
    }
  }
};

__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(dst), "l"(src) : "memory");
}

template <int D, int NT>
__global__ void __launch_bounds__(kThreads, 2) score_mma_kernel(ScoreArgs a) {
  constexpr int KS = D / 16;   // k-steps of 16 features
  constexpr int NCH = D / 64;  // 16-byte pieces per thread per row
  constexpr int VPR = D / 16;  // 16-byte chunks per row
  using SL = StageLayout<D>;
  extern __shared__ __align__(16) unsigned char ring[];  // stages, hist, s_pref[B+1], cu[B+1]
  uint32_t* s_hist = reinterpret_cast<uint32_t*>(ring + kScoreStages * SL::BYTES);
  int* s_pref = reinterpret_cast<int*>(s_hist + kHist);
  int* s_cu = s_pref + a.B + 1;
  for (int i = threadIdx.x; i <= a.B; i += kThreads) s_cu[i] = a.cu[i];
  for (int i = threadIdx.x; i < kHist; i += kThreads) s_hist[i] = 0u;
  chunk_prefix(a.cu, a.B, kStageRows, s_pref);
  const int per_head = s_pref[a.B];
  const int64_t total = (int64_t)a.Hkv * per_head;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, tig = lane & 3;
  const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(a.q);
  // this CTA's contiguous range of stages
  const int64_t s_begin = total * blockIdx.x / gridDim.x;
  const int64_t s_end = total * (blockIdx.x + 1) / gridDim.x;
  const int nk = (int)(s_end - s_begin);
  StageIter it_issue, it_comp;
  {
    const int h = (int)(s_begin / per_head);
    const int cc = (int)(s_begin - (int64_t)h * per_head);
    const int b = find_seq(s_pref, a.B, cc);
    it_issue = StageIter{h, b, (cc - s_pref[b]) * kStageRows};
    it_comp = it_issue;
  }

  auto issue = [&](int kk) {
    if (kk < nk) {
      const int L = s_cu[it_issue.b + 1] - s_cu[it_issue.b];
      const int rows = min(kStageRows, L - it_issue.r0);
      const int64_t rowbase = (int64_t)it_issue.h * a.T + s_cu[it_issue.b] + it_issue.r0;
      unsigned char* buf = ring + (kk % kScoreStages) * SL::BYTES;
      const int8_t* src = a.kq + rowbase * D;
      for (int x = tid; x < rows * VPR; x += kThreads) {
        const int r = x / VPR, c = x - r * VPR;
        cp_async16(smem_u32(buf + SL::off(r, c)), src + r * D + c * 16, true);
      }
      if (tid < rows) cp_async4(smem_u32(buf + SL::CODES + tid * 4), a.scale + rowbase + tid);
      it_issue.advance(s_cu, a.B);
    }
    cp_async_commit();
  };

  uint32_t bq[NT][KS][2];
  float unscale = 1.0f;
  int cur_b = -1, cur_h = -1;
  int hist_row = -1;  // (sequence, KV head) row the shared histogram holds
  auto flush = [&]() {  // shared histogram -> global (non-zero bins), then clear
    if (a.hist && hist_row >= 0) {
      uint32_t* gh = a.hist + (int64_t)hist_row * kHist;
      for (int i = tid; i < kHist; i += kThreads) {
        const uint32_t c = s_hist[i];
        if (c) {
          atomicAdd(gh + i, c);
          s_hist[i] = 0u;
        }
      }
    }
    __syncthreads();
  };
#pragma unroll 1
  for (int kk = 0; kk < kScoreStages; ++kk) issue(kk);
#pragma unroll 1
  for (int kk = 0; kk < nk; ++kk) {
    const int L = s_cu[it_comp.b + 1] - s_cu[it_comp.b];
    const int rows = min(kStageRows, L - it_comp.r0);
    const int64_t rowbase = (int64_t)it_comp.h * a.T + s_cu[it_comp.b] + it_comp.r0;
    if (it_comp.b != cur_b || it_comp.h != cur_h) {
      // query fragments of (b, h), scaled by a power of two into fp16 range;
      // thread (g, tig) holds column n = g; k-step s covers features
      // base(s) .. base(s)+3, base(s) = 64*(s/4) + 16*tig + 4*(s%4)
      cur_b = it_comp.b;
      cur_h = it_comp.h;
      float qv[NT][KS][4];
      float mx = 0.0f;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int n = nt * 8 + g;
#pragma unroll
        for (int s2 = 0; s2 < KS; ++s2) {
          const int base = 64 * (s2 / 4) + 16 * tig + 4 * (s2 % 4);
          if (n < a.G) {
            const uint2 w = *reinterpret_cast<const uint2*>(
                q + ((int64_t)cur_b * a.Hkv * a.G + (int64_t)cur_h * a.G + n) * D + base);
            qv[nt][s2][0] = bf16lo(w.x); qv[nt][s2][1] = bf16hi(w.x);
            qv[nt][s2][2] = bf16lo(w.y); qv[nt][s2][3] = bf16hi(w.y);
          } else {
            qv[nt][s2][0] = qv[nt][s2][1] = qv[nt][s2][2] = qv[nt][s2][3] = 0.0f;
          }
#pragma unroll
          for (int e = 0; e < 4; ++e) mx = fmaxf(mx, fabsf(qv[nt][s2][e]));
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      // largest |q| scaled into [2^14, 2^15): exponent of mx from its bits
      // (mx is a normal fp32 or 0); kept inside the normal range of 2^e
      int qexp = 0;
      if (mx > 0.0f) {
        const int e2 = ((__float_as_int(mx) >> 23) & 0xFF) - 126;  // mx < 2^e2
        qexp = min(126, max(-126, 15 - e2));
      }
      const float up = pow2f(qexp);
      unscale = pow2f(-qexp);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int s2 = 0; s2 < KS; ++s2) {
          bq[nt][s2][0] = pack_f16(qv[nt][s2][0] * up, qv[nt][s2][1] * up);
          bq[nt][s2][1] = pack_f16(qv[nt][s2][2] * up, qv[nt][s2][3] * up);
        }
    }
    const int row_id = it_comp.b * a.Hkv + it_comp.h;  // CTA-uniform
    if (row_id != hist_row) {
      flush();
      hist_row = row_id;
    }
    it_comp.advance(s_cu, a.B);
    cp_async_wait<kScoreStages - 1>();
    __syncthreads();
    const unsigned char* buf = ring + (kk % kScoreStages) * SL::BYTES;
    const int t = warp;  // one 16-row tile per warp
    if (t * 16 < rows) {
      uint4 cur[2][NCH];
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int r = t * 16 + g + 8 * half;
#pragma unroll
        for (int ch = 0; ch < NCH; ++ch)
          cur[half][ch] = *reinterpret_cast<const uint4*>(buf + SL::off(r, ch * 4 + tig));
      }
      float acc[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.0f;
#pragma unroll
      for (int s2 = 0; s2 < KS; ++s2) {
        uint32_t a0, a1, a2, a3;
        i8x4_to_f16(word_of(cur[0][s2 / 4], s2 % 4), a0, a2);  // row g
        i8x4_to_f16(word_of(cur[1][s2 / 4], s2 % 4), a1, a3);  // row g + 8
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma16816(acc[nt], a0, a1, a2, a3, bq[nt][s2][0], bq[nt][s2][1]);
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
      const int rs = t * 16 + g + 8 * tig;  // tig 0: row g, tig 1: row g + 8
      const bool mine = tig < 2 && rs < rows;
      float score = 0.0f;
      if (mine) {
        const float sc = reinterpret_cast<const float*>(buf + SL::CODES)[rs];
        score = sc * ((tig == 0 ? mA : mB) * unscale);
        a.scores[rowbase + rs] = score;
      }
      if (a.hist) warp_hist_add(s_hist, ord_key(score) >> 20, mine);
    }
    __syncthreads();
    issue(kk + kScoreStages);
  }
  cp_async_wait<0>();
  flush();
}

// TMA scorer (d = 128).  The same arithmetic as score_mma_kernel, with each
// 128-row stage of codes moved by one 2D tensor copy (cp.async.bulk.tensor,
// 128-byte swizzle: 16-byte chunk c of row r lands at chunk c ^ (r & 7))
// that completes on the stage's mbarrier, so one thread issues a whole stage.
// Thread (g, tig) reads chunks 2 tig and 2 tig + 1 of its two rows -- under
// the swizzle, the 8 lanes of each quarter-warp hit 8 different chunks -- so
// k-step s covers features 32 tig + 4 s .. + 3 of the permuted feature axis.
// Scales come straight from global memory, one per row.  The first-digit
// histogram keeps two 16-bit counts per word (flushed before they could
// overflow), so three CTAs fit on an SM.
constexpr int kTmaStages = 4;
constexpr int kTmaStageBytes = kStageRows * 128;
constexpr int kTmaFlushStages = 256;  // stages between histogram flushes (< 65536 keys)
constexpr uint32_t kWaitLimit = 1u << 24;  // polls of a stage barrier before giving up

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// rows [y, y + 128) of the code tensor into a swizzled stage; completes on bar
__device__ __forceinline__ void tma_rows(void* dst, const CUtensorMap* tm, int y, uint64_t* bar) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_u32(bar)),
               "r"(kTmaStageBytes)
               : "memory");
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];\n" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(0), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// The same copy marked evict-first in L2: the code stream is read once, and
// should not push out of L2 the scores and histograms the selection reads
// right after the scorer.
__device__ __forceinline__ void tma_rows_stream(void* dst, const CUtensorMap* tm, int y, uint64_t* bar,
                                                uint64_t policy) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_u32(bar)),
               "r"(kTmaStageBytes)
               : "memory");
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;\n" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(0), "r"(y), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

template <int NT>
__global__ void __launch_bounds__(kThreads, 3) score_tma_kernel(const __grid_constant__ CUtensorMap tm,
                                                                ScoreArgs a) {
  constexpr int D = 128;
  constexpr int KS = D / 16;
  extern __shared__ unsigned char dsm_raw[];
  // the swizzle pattern repeats every 1024 bytes: stages start on that boundary
  unsigned char* ring =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
  uint32_t* s_hist = reinterpret_cast<uint32_t*>(ring + kTmaStages * kTmaStageBytes);  // [kHist / 2]
  int* s_pref = reinterpret_cast<int*>(s_hist + kHist / 2);
  int* s_cu = s_pref + a.B + 1;
  __shared__ __align__(8) uint64_t full[kTmaStages];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, tig = lane & 3;
  for (int i = tid; i <= a.B; i += kThreads) s_cu[i] = a.cu[i];
  for (int i = tid; i < kHist / 2; i += kThreads) s_hist[i] = 0u;
  if (tid == 0) {
    for (int i = 0; i < kTmaStages; ++i) mbar_init(&full[i], 1);
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  chunk_prefix(a.cu, a.B, kStageRows, s_pref);  // ends with __syncthreads
  const int per_head = s_pref[a.B];
  const int64_t total = (int64_t)a.Hkv * per_head;
  const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(a.q);
  const int64_t s_begin = total * blockIdx.x / gridDim.x;
  const int64_t s_end = total * (blockIdx.x + 1) / gridDim.x;
  const int nk = (int)(s_end - s_begin);
  StageIter it_issue, it_comp;
  {
    const int h = (int)(s_begin / per_head);
    const int cc = (int)(s_begin - (int64_t)h * per_head);
    const int b = find_seq(s_pref, a.B, cc);
    it_issue = StageIter{h, b, (cc - s_pref[b]) * kStageRows};
    it_comp = it_issue;
  }
  auto issue = [&](int kk) {  // thread 0
    if (kk < nk) {
      const int64_t y = (int64_t)it_issue.h * a.T + s_cu[it_issue.b] + it_issue.r0;
      tma_rows(ring + (kk % kTmaStages) * kTmaStageBytes, &tm, (int)y, &full[kk % kTmaStages]);
      it_issue.advance(s_cu, a.B);
    }
  };
  // A stage that never arrived: report it, wait (bounded) for the copies
  // still in flight into this CTA's ring, issue nothing more.
  auto abandon = [&](int kk) {
    if (tid == 0) flag_status(a.status, PRISM_DEV_TIMEOUT);
    for (int j = kk; j < nk && j < kk + kTmaStages; ++j) {
      uint32_t it = 0;
      while (!mbar_try_wait(&full[j % kTmaStages], (uint32_t)(j / kTmaStages) & 1u) && ++it < kWaitLimit) {
      }
    }
  };
  if (tid == 0) {
    asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(&tm)) : "memory");
    for (int kk = 0; kk < kTmaStages; ++kk) issue(kk);
  }

  uint32_t bq[NT][KS][2];
  float unscale = 1.0f;
  int cur_b = -1, cur_h = -1;
  int hist_row = -1, since_flush = 0;
  // this thread's key-row scale, loaded one stage ahead (row g of tile warp
  // for tig 0, row g + 8 for tig 1)
  const int rs = warp * 16 + g + 8 * tig;
  auto load_scale = [&](const StageIter& it) {
    if (tig >= 2 || it.h >= a.Hkv) return 0.0f;
    const int L = s_cu[it.b + 1] - s_cu[it.b];
    if (rs >= min(kStageRows, L - it.r0)) return 0.0f;
    return __ldg(a.scale + (int64_t)it.h * a.T + s_cu[it.b] + it.r0 + rs);
  };
  float sc_next = nk > 0 ? load_scale(it_comp) : 0.0f;
  auto flush = [&]() {  // packed shared histogram -> global (non-zero bins), then clear
    if (a.hist && hist_row >= 0) {
      uint32_t* gh = a.hist + (int64_t)hist_row * kHist;
      for (int i = tid; i < kHist / 2; i += kThreads) {
        const uint32_t c = s_hist[i];
        if (c) {
          if (c & 0xFFFFu) atomicAdd(gh + 2 * i, c & 0xFFFFu);
          if (c >> 16) atomicAdd(gh + 2 * i + 1, c >> 16);
          s_hist[i] = 0u;
        }
      }
    }
    since_flush = 0;
    __syncthreads();
  };
#pragma unroll 1
  for (int kk = 0; kk < nk; ++kk) {
    const int L = s_cu[it_comp.b + 1] - s_cu[it_comp.b];
    const int rows = min(kStageRows, L - it_comp.r0);
    const int64_t rowbase = (int64_t)it_comp.h * a.T + s_cu[it_comp.b] + it_comp.r0;
    if (it_comp.b != cur_b || it_comp.h != cur_h) {
      // query fragments of (b, h), scaled by a power of two into fp16 range;
      // thread (g, tig) holds column n = g; k-step s covers features
      // 32 tig + 4 s .. + 3
      cur_b = it_comp.b;
      cur_h = it_comp.h;
      float qv[NT][KS][4];
      float mx = 0.0f;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int n = nt * 8 + g;
#pragma unroll
        for (int s2 = 0; s2 < KS; ++s2) {
          const int base = 32 * tig + 4 * s2;
          if (n < a.G) {
            const uint2 w = *reinterpret_cast<const uint2*>(
                q + ((int64_t)cur_b * a.Hkv * a.G + (int64_t)cur_h * a.G + n) * D + base);
            qv[nt][s2][0] = bf16lo(w.x); qv[nt][s2][1] = bf16hi(w.x);
            qv[nt][s2][2] = bf16lo(w.y); qv[nt][s2][3] = bf16hi(w.y);
          } else {
            qv[nt][s2][0] = qv[nt][s2][1] = qv[nt][s2][2] = qv[nt][s2][3] = 0.0f;
          }
#pragma unroll
          for (int e = 0; e < 4; ++e) mx = fmaxf(mx, fabsf(qv[nt][s2][e]));
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      int qexp = 0;
      if (mx > 0.0f) {
        const int e2 = ((__float_as_int(mx) >> 23) & 0xFF) - 126;  // mx < 2^e2
        qexp = min(126, max(-126, 15 - e2));
      }
      const float up = pow2f(qexp);
      unscale = pow2f(-qexp);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int s2 = 0; s2 < KS; ++s2) {
          bq[nt][s2][0] = pack_f16(qv[nt][s2][0] * up, qv[nt][s2][1] * up);
          bq[nt][s2][1] = pack_f16(qv[nt][s2][2] * up, qv[nt][s2][3] * up);
        }
    }
    const int row_id = it_comp.b * a.Hkv + it_comp.h;  // CTA-uniform
    if (row_id != hist_row || since_flush == kTmaFlushStages) {
      flush();
      hist_row = row_id;
    }
    ++since_flush;
    it_comp.advance(s_cu, a.B);
    const float sc = sc_next;
    if (kk + 1 < nk) sc_next = load_scale(it_comp);
    const int slot = kk % kTmaStages;
    bool late = false;  // this thread gave up waiting for the stage
    {
      uint32_t it = 0;
      while (!mbar_try_wait(&full[slot], (uint32_t)(kk / kTmaStages) & 1u)) {
        if (++it == kWaitLimit) {
          late = true;
          break;
        }
      }
    }
    const unsigned char* buf = ring + slot * kTmaStageBytes;
    const int t = warp;  // one 16-row tile per warp
    if (t * 16 < rows) {
      const bool mine = tig < 2 && rs < rows;  // tig 0: row g, tig 1: row g + 8
      uint4 cur[2][2];
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int r = t * 16 + g + 8 * half;  // r & 7 == g
#pragma unroll
        for (int ch = 0; ch < 2; ++ch)
          cur[half][ch] = *reinterpret_cast<const uint4*>(buf + r * 128 + (((2 * tig + ch) ^ g) << 4));
      }
      float acc[2][NT][4];
#pragma unroll
      for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) acc[u][nt][0] = acc[u][nt][1] = acc[u][nt][2] = acc[u][nt][3] = 0.0f;
#pragma unroll
      for (int s2 = 0; s2 < KS; ++s2) {
        uint32_t a0, a1, a2, a3;
        i8x4_to_f16(word_of(cur[0][s2 / 4], s2 % 4), a0, a2);  // row g
        i8x4_to_f16(word_of(cur[1][s2 / 4], s2 % 4), a1, a3);  // row g + 8
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
          mma16816(acc[s2 & 1][nt], a0, a1, a2, a3, bq[nt][s2][0], bq[nt][s2][1]);
      }
      float mA = -INFINITY, mB = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int col = nt * 8 + 2 * tig;
        const float c0 = acc[0][nt][0] + acc[1][nt][0], c1 = acc[0][nt][1] + acc[1][nt][1];
        const float c2 = acc[0][nt][2] + acc[1][nt][2], c3 = acc[0][nt][3] + acc[1][nt][3];
        if (col < a.G) { mA = fmaxf(mA, c0); mB = fmaxf(mB, c2); }
        if (col + 1 < a.G) { mA = fmaxf(mA, c1); mB = fmaxf(mB, c3); }
      }
      mA = fmaxf(mA, __shfl_xor_sync(0xffffffffu, mA, 1));
      mA = fmaxf(mA, __shfl_xor_sync(0xffffffffu, mA, 2));
      mB = fmaxf(mB, __shfl_xor_sync(0xffffffffu, mB, 1));
      mB = fmaxf(mB, __shfl_xor_sync(0xffffffffu, mB, 2));
      float score = 0.0f;
      if (mine && !late) {
        score = sc * ((tig == 0 ? mA : mB) * unscale);
        a.scores[rowbase + rs] = score;
      }
      if (a.hist) warp_hist_add_packed(s_hist, ord_key(score) >> 20, mine && !late);
    }
    // every warp is done with the stage; a stage that never arrived ends the CTA
    if (__syncthreads_or(late)) {
      abandon(kk);
      return;
    }
    if (tid == 0) issue(kk + kTmaStages);
  }
  flush();
}

// Integer tensor-core scorer (bf16 queries, d = 128), on the tensor-copy
// pipeline above.  The int8 codes enter mma.sync.m16n8k32 (s8 x s8 -> s32)
// as stored: no conversion.  Each query head is held in fixed point,
// Q = rint(q * 2^sh) with sh per head such that its largest |q| lands in
// [2^29, 2^30), written as four signed base-256 digits (limbs)
// Q = l0 2^24 + l1 2^16 + l2 2^8 + l3, each an int8.  A bf16 element within
// 2^-22 of its head's largest lies on that grid exactly; a smaller one rounds
// to it (by less than 2^-30 of the largest).  Code x limb products and their
// sums over a row are exact in int32 (at most 128 * 128 * 127 < 2^21 in
// magnitude); the four limb sums combine exactly in 64-bit integers and are
// rounded to fp32 once, then taken back by 2^-sh and multiplied by the row's
// scale.  Head quad j uses two n8 tiles: column 2 t + i of tile u holds limb
// 2 u + i of head 4 j + t, so thread (g, t) ends with all four limb sums of
// head 4 j + t for its rows g and g + 8.  At k-step s thread (g, t) covers
// features 32 t + 8 s .. + 7: words 2 (s & 1) and 2 (s & 1) + 1 of its chunk
// s / 2 (the tensor-copy scorer's chunk assignment).
__device__ __forceinline__ void mma_s8(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                       uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// low byte of x as a signed value in [-128, 127]
__device__ __forceinline__ int sbyte(int x) { return ((x & 0xFF) ^ 0x80) - 0x80; }

template <int NH>
__global__ void __launch_bounds__(kThreads, 3) score_i8_kernel(const __grid_constant__ CUtensorMap tm,
                                                              ScoreArgs a) {
  constexpr int D = 128;
  extern __shared__ unsigned char dsm_raw[];
  unsigned char* ring =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
  uint32_t* s_hist = reinterpret_cast<uint32_t*>(ring + kTmaStages * kTmaStageBytes);  // [kHist / 2]
  int* s_pref = reinterpret_cast<int*>(s_hist + kHist / 2);
  int* s_cu = s_pref + a.B + 1;
  __shared__ __align__(8) uint64_t full[kTmaStages];
  __shared__ float s_newscale;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, tig = lane & 3;
  // the descriptor's fetch overlaps the loads of the sequence offsets
  if (tid == 0) asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(&tm)) : "memory");
  for (int i = tid; i <= a.B; i += kThreads) s_cu[i] = a.cu[i];
  for (int i = tid; i < kHist / 2; i += kThreads) s_hist[i] = 0u;
  if (tid == 0) {
    for (int i = 0; i < kTmaStages; ++i) mbar_init(&full[i], 1);
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  chunk_prefix(a.cu, a.B, kStageRows, s_pref);  // ends with __syncthreads
  const int per_head = s_pref[a.B];
  const int64_t total = (int64_t)a.Hkv * per_head;
  const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(a.q);
  const int64_t s_begin = total * blockIdx.x / gridDim.x;
  const int64_t s_end = total * (blockIdx.x + 1) / gridDim.x;
  const int nk = (int)(s_end - s_begin);
  StageIter it_issue, it_comp;
  {
    const int h = (int)(s_begin / per_head);
    const int cc = (int)(s_begin - (int64_t)h * per_head);
    const int b = find_seq(s_pref, a.B, cc);
    it_issue = StageIter{h, b, (cc - s_pref[b]) * kStageRows};
    it_comp = it_issue;
  }
  auto issue = [&](int kk) {  // thread 0
    if (kk < nk) {
      const int64_t y = (int64_t)it_issue.h * a.T + s_cu[it_issue.b] + it_issue.r0;
      uint64_t evict_first;
      asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;\n" : "=l"(evict_first));
      tma_rows_stream(ring + (kk % kTmaStages) * kTmaStageBytes, &tm, (int)y, &full[kk % kTmaStages],
                      evict_first);
      it_issue.advance(s_cu, a.B);
    }
  };
  // A stage that never arrived: report it, wait (bounded) for the copies
  // still in flight into this CTA's ring, issue nothing more.
  auto abandon = [&](int kk) {
    if (tid == 0) flag_status(a.status, PRISM_DEV_TIMEOUT);
    for (int j = kk; j < nk && j < kk + kTmaStages; ++j) {
      uint32_t it = 0;
      while (!mbar_try_wait(&full[j % kTmaStages], (uint32_t)(j / kTmaStages) & 1u) && ++it < kWaitLimit) {
      }
    }
  };
  if (tid == 0)
    for (int kk = 0; kk < kTmaStages; ++kk) issue(kk);

  uint32_t bq[NH][2][4][2];  // [quad][tile][k-step][b0, b1]
  float us1[NH], us2[NH];    // 2^-sh of head 4 j + tig, as two exact factors
  int cur_b = -1, cur_h = -1;
  int hist_row = -1, since_flush = 0;
  const int rs = warp * 16 + g + 8 * tig;
  auto load_scale = [&](const StageIter& it) {
    if (tig >= 2 || it.h >= a.Hkv) return 0.0f;
    const int L = s_cu[it.b + 1] - s_cu[it.b];
    if (rs >= min(kStageRows, L - it.r0)) return 0.0f;
    return __ldg(a.scale + (int64_t)it.h * a.T + s_cu[it.b] + it.r0 + rs);
  };
  float sc_next = nk > 0 ? load_scale(it_comp) : 0.0f;
  auto flush = [&]() {
    if (a.hist && hist_row >= 0) {
      uint32_t* gh = a.hist + (int64_t)hist_row * kHist;
      for (int i = tid; i < kHist / 2; i += kThreads) {
        const uint32_t c = s_hist[i];
        if (c) {
          if (c & 0xFFFFu) atomicAdd(gh + 2 * i, c & 0xFFFFu);
          if (c >> 16) atomicAdd(gh + 2 * i + 1, c >> 16);
          s_hist[i] = 0u;
        }
      }
    }
    since_flush = 0;
    __syncthreads();
  };
#pragma unroll 1
  for (int kk = 0; kk < nk; ++kk) {
    const int L = s_cu[it_comp.b + 1] - s_cu[it_comp.b];
    const int rows = min(kStageRows, L - it_comp.r0);
    const int nr = L - 1 - it_comp.r0;  // the stage row of position L - 1 when nr < rows
    const int64_t rowbase = (int64_t)it_comp.h * a.T + s_cu[it_comp.b] + it_comp.r0;
    if (it_comp.b != cur_b || it_comp.h != cur_h) {
      // limbs of the query heads of (b, h): thread (g, tig) supplies column g
      // of both tiles of each quad -- head 4 j + g / 2, limbs g % 2 and
      // 2 + g % 2 -- at its features 32 tig .. + 31
      cur_b = it_comp.b;
      cur_h = it_comp.h;
#pragma unroll
      for (int j = 0; j < NH; ++j) {
        const int hd = 4 * j + (g >> 1);
        float qv[32];
        if (hd < a.G) {
          const uint4* src = reinterpret_cast<const uint4*>(
              q + ((int64_t)cur_b * a.Hkv * a.G + (int64_t)cur_h * a.G + hd) * D + 32 * tig);
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint4 w = src[c];
            qv[8 * c + 0] = bf16lo(w.x); qv[8 * c + 1] = bf16hi(w.x);
            qv[8 * c + 2] = bf16lo(w.y); qv[8 * c + 3] = bf16hi(w.y);
            qv[8 * c + 4] = bf16lo(w.z); qv[8 * c + 5] = bf16hi(w.z);
            qv[8 * c + 6] = bf16lo(w.w); qv[8 * c + 7] = bf16hi(w.w);
          }
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) qv[e] = 0.0f;
        }
        float mx = 0.0f;
#pragma unroll
        for (int e = 0; e < 32; ++e) mx = fmaxf(mx, fabsf(qv[e]));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));  // the head's four feature quarters
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        int sh = 0;
        if (mx > 0.0f) sh = 30 - (((__float_as_int(mx) >> 23) & 0xFF) - 126);  // mx * 2^sh < 2^30
        // sh lies in [-98, 156]: each factor is an exact power of two
        const float up1 = pow2f(min(sh, 126)), up2 = pow2f(max(sh - 126, 0));
        const float dn1 = pow2f(-min(sh, 126)), dn2 = pow2f(-max(sh - 126, 0));
        const int li = g & 1;
#pragma unroll
        for (int st = 0; st < 4; ++st)
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            uint32_t w0 = 0u, w1 = 0u;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int Q = __float2int_rn(qv[8 * st + 4 * hf + e] * up1 * up2);
              const int d3 = sbyte(Q);
              const int q1 = (Q - d3) >> 8;
              const int d2 = sbyte(q1);
              const int q2 = (q1 - d2) >> 8;
              const int d1 = sbyte(q2);
              const int d0 = (q2 - d1) >> 8;
              const int t0 = li ? d1 : d0, t1 = li ? d3 : d2;  // tile 0: limb li, tile 1: limb 2 + li
              w0 |= (uint32_t)(t0 & 0xFF) << (8 * e);
              w1 |= (uint32_t)(t1 & 0xFF) << (8 * e);
            }
            bq[j][0][st][hf] = w0;
            bq[j][1][st][hf] = w1;
          }
        // head 4 j + tig was prepared by the lanes with g = 2 tig
        us1[j] = __shfl_sync(0xffffffffu, dn1, 8 * tig);
        us2[j] = __shfl_sync(0xffffffffu, dn2, 8 * tig);
      }
    }
    const int row_id = it_comp.b * a.Hkv + it_comp.h;  // CTA-uniform
    if (row_id != hist_row || since_flush == kTmaFlushStages) {
      flush();
      hist_row = row_id;
    }
    ++since_flush;
    it_comp.advance(s_cu, a.B);
    float sc = sc_next;
    if (kk + 1 < nk) sc_next = load_scale(it_comp);
    const int slot = kk % kTmaStages;
    bool late = false;  // this thread gave up waiting for the stage
    {
      uint32_t it = 0;
      while (!mbar_try_wait(&full[slot], (uint32_t)(kk / kTmaStages) & 1u)) {
        if (++it == kWaitLimit) {
          late = true;
          break;
        }
      }
    }
    unsigned char* buf = ring + slot * kTmaStageBytes;
    if (a.k_new && nr < rows) {  // CTA-uniform
      // this token's key row, not in the codes yet: warp 0 quantizes it as
      // the quantizer does (amax / 127, round half to even, clamp to 127)
      // into the stage and into the cache's codes and scales
      if (warp == 0) {
        const __nv_bfloat16* kn =
            static_cast<const __nv_bfloat16*>(a.k_new) + ((int64_t)cur_b * a.Hkv + cur_h) * D;
        const uint2 w = *reinterpret_cast<const uint2*>(kn + 4 * lane);
        const float f[4] = {bf16lo(w.x), bf16hi(w.x), bf16lo(w.y), bf16hi(w.y)};
        float amax = fmaxf(fmaxf(fabsf(f[0]), fabsf(f[1])), fmaxf(fabsf(f[2]), fabsf(f[3])));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const float sq = __fdiv_rn(amax, 127.0f);
        uint32_t packed = 0u;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          int c = 0;
          if (amax != 0.0f) c = (int)fminf(fmaxf(rintf(__fdiv_rn(f[e], sq)), -127.0f), 127.0f);
          packed |= ((uint32_t)(c & 0xFF)) << (8 * e);
        }
        // features 4 lane .. + 3: chunk lane / 4 of the row, swizzled as the copy lays it out
        *reinterpret_cast<uint32_t*>(buf + nr * 128 + ((((lane >> 2) ^ (nr & 7)) << 4) | ((lane & 3) << 2))) =
            packed;
        asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");  // before the slot's next copy
        *reinterpret_cast<uint32_t*>(a.kq_w + (rowbase + nr) * D + 4 * lane) = packed;
        if (lane == 0) {
          s_newscale = amax != 0.0f ? sq : 0.0f;
          a.scale_w[rowbase + nr] = s_newscale;
        }
      }
      __syncthreads();
      if (rs == nr) sc = s_newscale;
    }
    const int t = warp;  // one 16-row tile per warp
    if (t * 16 < rows) {
      const bool mine = tig < 2 && rs < rows;  // tig 0: row g, tig 1: row g + 8
      uint4 cur[2][2];
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int r = t * 16 + g + 8 * half;  // r & 7 == g
#pragma unroll
        for (int ch = 0; ch < 2; ++ch)
          cur[half][ch] = *reinterpret_cast<const uint4*>(buf + r * 128 + (((2 * tig + ch) ^ g) << 4));
      }
      int acc[NH][2][4];
#pragma unroll
      for (int j = 0; j < NH; ++j)
#pragma unroll
        for (int u = 0; u < 2; ++u) acc[j][u][0] = acc[j][u][1] = acc[j][u][2] = acc[j][u][3] = 0;
#pragma unroll
      for (int st = 0; st < 4; ++st) {
        const uint32_t a0 = word_of(cur[0][st >> 1], 2 * (st & 1));      // row g
        const uint32_t a2 = word_of(cur[0][st >> 1], 2 * (st & 1) + 1);
        const uint32_t a1 = word_of(cur[1][st >> 1], 2 * (st & 1));      // row g + 8
        const uint32_t a3 = word_of(cur[1][st >> 1], 2 * (st & 1) + 1);
#pragma unroll
        for (int j = 0; j < NH; ++j)
#pragma unroll
          for (int u = 0; u < 2; ++u) mma_s8(acc[j][u], a0, a1, a2, a3, bq[j][u][st][0], bq[j][u][st][1]);
      }
      const bool sum = a.sum_group != 0;  // CTA-uniform
      float mA = sum ? 0.0f : -INFINITY, mB = mA;
#pragma unroll
      for (int j = 0; j < NH; ++j) {
        if (4 * j + tig < a.G) {
          const long long sA = ((long long)(acc[j][0][0] * 256 + acc[j][0][1]) << 16) +
                               (long long)(acc[j][1][0] * 256 + acc[j][1][1]);
          const long long sB = ((long long)(acc[j][0][2] * 256 + acc[j][0][3]) << 16) +
                               (long long)(acc[j][1][2] * 256 + acc[j][1][3]);
          const float vA = __ll2float_rn(sA) * us1[j] * us2[j], vB = __ll2float_rn(sB) * us1[j] * us2[j];
          mA = sum ? mA + vA : fmaxf(mA, vA);
          mB = sum ? mB + vB : fmaxf(mB, vB);
        }
      }
      // over the heads held by the four lanes of a row (head 4 j + tig)
#pragma unroll
      for (int o = 1; o <= 2; o <<= 1) {
        const float xA = __shfl_xor_sync(0xffffffffu, mA, o), xB = __shfl_xor_sync(0xffffffffu, mB, o);
        mA = sum ? mA + xA : fmaxf(mA, xA);
        mB = sum ? mB + xB : fmaxf(mB, xB);
      }
      float score = 0.0f;
      if (mine && !late) {
        score = sc * (tig == 0 ? mA : mB);
        a.scores[rowbase + rs] = score;
      }
      if (a.hist) warp_hist_add_packed(s_hist, ord_key(score) >> 20, mine && !late);
    }
    // every warp is done with the stage; a stage that never arrived ends the CTA
    if (__syncthreads_or(late)) {
      abandon(kk);
      return;
    }
    if (tid == 0) issue(kk + kTmaStages);
  }
  flush();
}

// INT2 scorer (bf16 queries, d = 128).  Per key row and query head the
// score is sum over 32-feature groups of (S * D + L * Q), with D = q . c over
// the group's 2-bit codes and Q = sum of q over the group (the dot product
// with the dequantized key L + S c).  Rows stream through a cp.async ring
// of 128-row stages (codes, then (S, L) pairs); warp w takes 16-row tile w.
// The contraction D runs on tensor cores: a code c enters as the fp16
// subnormal c * 2^-24 (its bits are c), the query is scaled by a power of
// two into fp16 range as in the int8 scorer, so every product and sum is
// exact up to fp32 rounding and one power of two undoes both scalings; each
// k-step of 16 stays inside one group (two k-steps per group, one
// accumulator per group).  Thread (g, tig)
// takes, at k-step s, word s of its rows' codes (features 16 s .. 16 s + 15,
// feature f at bits 2 (f mod 16)) and from it features 16 s + 2 tig + {0, 8}
// and 16 s + 2 tig + {1, 9}: the query fragments follow the same features.
// The query rows of a (sequence, KV head) go to shared memory once; Q is
// summed there in feature order, and the group terms combine in the
// definition's order, without fused multiply-adds.
constexpr int kInt2Stages = 6;

template <int D>
struct Int2Layout {
  static constexpr int CB = D / 4;                   // code bytes per row
  static constexpr int NG = D / 32;                  // groups per row
  static constexpr int PB = NG * 4;                  // (S, L) bytes per row
  static constexpr int CODES = kStageRows * CB;
  static constexpr int BYTES = CODES + kStageRows * PB;
};

// two codes (bits 0-1 and 16-17 of w) as fp16 subnormals c * 2^-24
__device__ __forceinline__ uint32_t int2_pair(uint32_t w) { return w & 0x00030003u; }

template <int NT>
__global__ void __launch_bounds__(kThreads, 3) score_int2_kernel(ScoreArgs a) {
  constexpr int D = 128;
  constexpr int KS = D / 16;
  using IL = Int2Layout<D>;
  constexpr int NG = IL::NG;
  extern __shared__ __align__(16) unsigned char ring[];  // stages, hist, s_pref[B+1], cu[B+1]
  uint32_t* s_hist = reinterpret_cast<uint32_t*>(ring + kInt2Stages * IL::BYTES);  // [kHist / 2]
  int* s_pref = reinterpret_cast<int*>(s_hist + kHist / 2);
  int* s_cu = s_pref + a.B + 1;
  __shared__ float sq[NT * 8 * D];   // the (b, h) group's query rows, fp32
  __shared__ float sQ[NT * 8 * NG];  // per head and group: sum of q (features in order)
  __shared__ float s_mx[kThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, tig = lane & 3;
  for (int i = tid; i <= a.B; i += kThreads) s_cu[i] = a.cu[i];
  for (int i = tid; i < kHist / 2; i += kThreads) s_hist[i] = 0u;
  chunk_prefix(a.cu, a.B, kStageRows, s_pref);
  const int per_head = s_pref[a.B];
  const int64_t total = (int64_t)a.Hkv * per_head;
  const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(a.q);
  const int64_t s_begin = total * blockIdx.x / gridDim.x;
  const int64_t s_end = total * (blockIdx.x + 1) / gridDim.x;
  const int nk = (int)(s_end - s_begin);
  StageIter it_issue, it_comp;
  {
    const int h = (int)(s_begin / per_head);
    const int cc = (int)(s_begin - (int64_t)h * per_head);
    const int b = find_seq(s_pref, a.B, cc);
    it_issue = StageIter{h, b, (cc - s_pref[b]) * kStageRows};
    it_comp = it_issue;
  }
  auto issue = [&](int kk) {
    if (kk < nk) {
      const int L = s_cu[it_issue.b + 1] - s_cu[it_issue.b];
      const int rows = min(kStageRows, L - it_issue.r0);
      const int64_t rowbase = (int64_t)it_issue.h * a.T + s_cu[it_issue.b] + it_issue.r0;
      unsigned char* buf = ring + (kk % kInt2Stages) * IL::BYTES;
      const unsigned char* cs = a.codes + rowbase * IL::CB;
      const unsigned char* ps = reinterpret_cast<const unsigned char*>(a.params) + rowbase * IL::PB;
      for (int x = tid; x < rows * (IL::CB / 16); x += kThreads)
        cp_async16(smem_u32(buf + x * 16), cs + x * 16, true);
      for (int x = tid; x < rows * (IL::PB / 16); x += kThreads)
        cp_async16(smem_u32(buf + IL::CODES + x * 16), ps + x * 16, true);
      it_issue.advance(s_cu, a.B);
    }
    cp_async_commit();
  };

  uint32_t bq[NT][KS][2];
  float Qv[NT][NG][2];  // sum of q over each group, heads nt*8 + 2 tig, + 1
  float unscale = 1.0f;
  int cur_b = -1, cur_h = -1;
  int hist_row = -1, since_flush = 0;
  auto flush = [&]() {  // packed shared histogram -> global (non-zero bins), then clear
    if (a.hist && hist_row >= 0) {
      uint32_t* gh = a.hist + (int64_t)hist_row * kHist;
      for (int i = tid; i < kHist / 2; i += kThreads) {
        const uint32_t c = s_hist[i];
        if (c) {
          if (c & 0xFFFFu) atomicAdd(gh + 2 * i, c & 0xFFFFu);
          if (c >> 16) atomicAdd(gh + 2 * i + 1, c >> 16);
          s_hist[i] = 0u;
        }
      }
    }
    since_flush = 0;
    __syncthreads();
  };
#pragma unroll 1
  for (int kk = 0; kk < kInt2Stages; ++kk) issue(kk);
#pragma unroll 1
  for (int kk = 0; kk < nk; ++kk) {
    const int L = s_cu[it_comp.b + 1] - s_cu[it_comp.b];
    const int rows = min(kStageRows, L - it_comp.r0);
    const int64_t rowbase = (int64_t)it_comp.h * a.T + s_cu[it_comp.b] + it_comp.r0;
    if (it_comp.b != cur_b || it_comp.h != cur_h) {  // CTA-uniform
      cur_b = it_comp.b;
      cur_h = it_comp.h;
      // the group's query rows into shared memory (fp32), then the fragments,
      // the power-of-two scale and the per-group sums Q from there
      const __nv_bfloat16* qb = q + ((int64_t)cur_b * a.Hkv * a.G + (int64_t)cur_h * a.G) * D;
      __syncthreads();  // the previous (b, h)'s sq / sQ are no longer read
      float mxl = 0.0f;
      for (int i = tid; i < a.G * D; i += kThreads) {
        const float v = __bfloat162float(qb[i]);
        sq[i] = v;
        mxl = fmaxf(mxl, fabsf(v));
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mxl = fmaxf(mxl, __shfl_xor_sync(0xffffffffu, mxl, o));
      if (lane == 0) s_mx[warp] = mxl;
      __syncthreads();
      float mx = 0.0f;
#pragma unroll
      for (int w = 0; w < kThreads / 32; ++w) mx = fmaxf(mx, s_mx[w]);
      if (tid < a.G * NG) {  // Q of head tid / NG, group tid % NG, features in order
        const float* qr = sq + (tid / NG) * D + (tid % NG) * 32;
        float acc = 0.0f;
        for (int j = 0; j < 32; ++j) acc = __fadd_rn(acc, qr[j]);
        sQ[tid] = acc;
      }
      int qexp = 0;
      if (mx > 0.0f) {
        const int e2 = ((__float_as_int(mx) >> 23) & 0xFF) - 126;  // mx < 2^e2
        qexp = min(103, max(-103, 15 - e2));  // 2^qexp and 2^(24 - qexp) stay normal
      }
      const float up = pow2f(qexp);
      // codes enter the tensor cores as fp16 subnormals c * 2^-24: undo both
      unscale = pow2f(24 - qexp);
      __syncthreads();
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int n = nt * 8 + g;
#pragma unroll
        for (int s2 = 0; s2 < KS; ++s2) {
          const int f = 16 * s2 + 2 * tig;
          float v0 = 0.0f, v1 = 0.0f, v2 = 0.0f, v3 = 0.0f;
          if (n < a.G) {
            const float* qr = sq + n * D;
            v0 = qr[f];
            v1 = qr[f + 8];
            v2 = qr[f + 1];
            v3 = qr[f + 9];
          }
          bq[nt][s2][0] = pack_f16(v0 * up, v1 * up);
          bq[nt][s2][1] = pack_f16(v2 * up, v3 * up);
        }
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int head = nt * 8 + 2 * tig + c;
#pragma unroll
          for (int gr = 0; gr < NG; ++gr) Qv[nt][gr][c] = head < a.G ? sQ[head * NG + gr] : 0.0f;
        }
      }
    }
    const int row_id = it_comp.b * a.Hkv + it_comp.h;  // CTA-uniform
    if (row_id != hist_row || since_flush == kTmaFlushStages) {
      flush();
      hist_row = row_id;
    }
    ++since_flush;
    it_comp.advance(s_cu, a.B);
    cp_async_wait<kInt2Stages - 1>();
    __syncthreads();
    const unsigned char* buf = ring + (kk % kInt2Stages) * IL::BYTES;
    const int t = warp;  // one 16-row tile per warp
    if (t * 16 < rows) {
      const int rA = t * 16 + g, rB = rA + 8;
      uint32_t wa[KS], wb[KS];
      {
        const uint4* ca = reinterpret_cast<const uint4*>(buf + rA * IL::CB);
        const uint4* cb = reinterpret_cast<const uint4*>(buf + rB * IL::CB);
        const uint4 a0 = ca[0], a1 = ca[1], b0 = cb[0], b1 = cb[1];
        wa[0] = a0.x; wa[1] = a0.y; wa[2] = a0.z; wa[3] = a0.w;
        wa[4] = a1.x; wa[5] = a1.y; wa[6] = a1.z; wa[7] = a1.w;
        wb[0] = b0.x; wb[1] = b0.y; wb[2] = b0.z; wb[3] = b0.w;
        wb[4] = b1.x; wb[5] = b1.y; wb[6] = b1.z; wb[7] = b1.w;
      }
      float acc[NG][NT][4];
#pragma unroll
      for (int gr = 0; gr < NG; ++gr)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) acc[gr][nt][0] = acc[gr][nt][1] = acc[gr][nt][2] = acc[gr][nt][3] = 0.0f;
      const int sh = 4 * tig;
#pragma unroll
      for (int s2 = 0; s2 < KS; ++s2) {
        const uint32_t xa = wa[s2] >> sh, xb = wb[s2] >> sh;
        const uint32_t a0 = int2_pair(xa), a2 = int2_pair(xa >> 2);
        const uint32_t a1 = int2_pair(xb), a3 = int2_pair(xb >> 2);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
          mma16816(acc[s2 / 2][nt], a0, a1, a2, a3, bq[nt][s2][0], bq[nt][s2][1]);
      }
      // (S, L) of the two rows, group by group
      const uint4 pA4 = *reinterpret_cast<const uint4*>(buf + IL::CODES + rA * IL::PB);
      const uint4 pB4 = *reinterpret_cast<const uint4*>(buf + IL::CODES + rB * IL::PB);
      const uint32_t pA[4] = {pA4.x, pA4.y, pA4.z, pA4.w}, pB[4] = {pB4.x, pB4.y, pB4.z, pB4.w};
      float mA = -INFINITY, mB = -INFINITY;
      // S' = S * unscale is exact (a power of two), and S' * D_mma = S * D
      float SA[NG], LA[NG], SB[NG], LB[NG];
#pragma unroll
      for (int gr = 0; gr < NG; ++gr) {
        const float2 fa = __half22float2(*reinterpret_cast<const __half2*>(&pA[gr]));
        const float2 fb = __half22float2(*reinterpret_cast<const __half2*>(&pB[gr]));
        SA[gr] = fa.x * unscale;
        LA[gr] = fa.y;
        SB[gr] = fb.x * unscale;
        LB[gr] = fb.y;
      }
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        float sc[4] = {0.0f, 0.0f, 0.0f, 0.0f};  // c0..c3
#pragma unroll
        for (int gr = 0; gr < NG; ++gr) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float S = e < 2 ? SA[gr] : SB[gr], Lz = e < 2 ? LA[gr] : LB[gr];
            const float term = __fadd_rn(__fmul_rn(S, acc[gr][nt][e]), __fmul_rn(Lz, Qv[nt][gr][e & 1]));
            sc[e] = __fadd_rn(sc[e], term);
          }
        }
        const int col = nt * 8 + 2 * tig;
        if (col < a.G) { mA = fmaxf(mA, sc[0]); mB = fmaxf(mB, sc[2]); }
        if (col + 1 < a.G) { mA = fmaxf(mA, sc[1]); mB = fmaxf(mB, sc[3]); }
      }
      mA = fmaxf(mA, __shfl_xor_sync(0xffffffffu, mA, 1));
      mA = fmaxf(mA, __shfl_xor_sync(0xffffffffu, mA, 2));
      mB = fmaxf(mB, __shfl_xor_sync(0xffffffffu, mB, 1));
      mB = fmaxf(mB, __shfl_xor_sync(0xffffffffu, mB, 2));
      const int rs = t * 16 + g + 8 * tig;  // tig 0: row g, tig 1: row g + 8
      const bool mine = tig < 2 && rs < rows;
      float score = 0.0f;
      if (mine) {
        score = tig == 0 ? mA : mB;
        a.scores[rowbase + rs] = score;
      }
      if (a.hist) warp_hist_add_packed(s_hist, ord_key(score) >> 20, mine);
    }
    __syncthreads();
    issue(kk + kInt2Stages);
  }
  cp_async_wait<0>();
  flush();
}

// CUDA-core scorer: one thread per key row, query in shared memory (fp32).
template <typename T, int D, int GP>
__global__ void __launch_bounds__(kThreads) score_simt_kernel(ScoreArgs a) {
  extern __shared__ int smem[];
  int* s_pref = smem;
  float* sq = reinterpret_cast<float*>(smem + ((a.B + 1 + 3) & ~3));
  chunk_prefix(a.cu, a.B, kChunkRows, s_pref);
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
cudaError_t run_mma(const Dims& d, const ScoreArgs& a, cudaStream_t st) {
  int64_t per_head = 0;
  for (int b = 0; b < d.B; ++b) per_head += cdiv(d.cu_host[b + 1] - d.cu_host[b], kStageRows);
  const int64_t total = per_head * d.Hkv;
  if (total == 0) return cudaSuccess;
  const int smem = kScoreStages * StageLayout<D>::BYTES + kHist * 4 + 2 * (d.B + 1) * (int)sizeof(int);
  auto k = score_mma_kernel<D, NT>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int grid = grid_for(k, smem, d.num_sms, total);
  k<<<grid, kThreads, smem, st>>>(a);
  return cudaGetLastError();
}

// PRISM_PROPOSE_SCORER=mma selects the cp.async fp16 tensor-core scorer,
// =tma the tensor-copy fp16 one; by default the integer one runs (G <= 8)
int scorer_choice() {
  const char* e = std::getenv("PRISM_PROPOSE_SCORER");
  if (e && std::strcmp(e, "mma") == 0) return 0;
  if (e && std::strcmp(e, "tma") == 0) return 1;
  return 2;
}

using TmaScoreKernel = void (*)(const CUtensorMap, ScoreArgs);

// Launches a tensor-copy scorer when the code tensor can be described by a
// tensor map (d = 128, 16-byte aligned base); returns false to fall back.
bool run_tma(TmaScoreKernel k, const Dims& d, const ScoreArgs& a, int64_t total, cudaError_t* err,
             cudaStream_t st) {
  const PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
  if (!encode || d.D != 128 || (reinterpret_cast<uintptr_t>(a.kq) & 15) != 0) return false;
  const uint64_t nrows = (uint64_t)d.Hkv * (uint64_t)d.T;
  if (nrows == 0 || nrows > 0x7fffffffull) return false;
  CUtensorMap tm;
  const cuuint64_t dims[2] = {128, (cuuint64_t)nrows};
  const cuuint64_t strides[1] = {128};
  const cuuint32_t box[2] = {128, (cuuint32_t)kStageRows};
  const cuuint32_t estr[2] = {1, 1};
  if (encode(&tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t*>(a.kq), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  const int smem = 1024 + kTmaStages * kTmaStageBytes + kHist / 2 * 4 + 2 * (d.B + 1) * (int)sizeof(int);
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess) {
    const int grid = grid_for(k, smem, d.num_sms, total);
    k<<<grid, kThreads, smem, st>>>(tm, a);
    e = cudaGetLastError();
  }
  *err = e;
  return true;
}

template <int NT>
cudaError_t run_int2(const Dims& d, const ScoreArgs& a, int64_t total, cudaStream_t st) {
  const int smem = kInt2Stages * Int2Layout<128>::BYTES + kHist / 2 * 4 + 2 * (d.B + 1) * (int)sizeof(int);
  auto k = score_int2_kernel<NT>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
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
                                  const float* scale, float* scores, uint32_t* hist, bool use_mma,
                                  int32_t* status, cudaStream_t st) {
  int64_t per_head = 0;
  for (int b = 0; b < d.B; ++b) per_head += cdiv(d.cu_host[b + 1] - d.cu_host[b], kChunkRows);
  const int64_t total = per_head * d.Hkv;
  if (total == 0) return cudaSuccess;
  ScoreArgs a{q, kq, scale, scores, hist, d.cu_dev, d.T, d.B, d.Hkv, d.G, status, nullptr, nullptr,
              nullptr, nullptr, nullptr, 0};
  const int choice = scorer_choice();
  if (use_mma && d.bf16 && d.D == 128 && choice > 0) {
    int64_t stages = 0;
    for (int b = 0; b < d.B; ++b) stages += cdiv(d.cu_host[b + 1] - d.cu_host[b], kStageRows);
    TmaScoreKernel k = d.G <= 8 ? score_tma_kernel<1> : score_tma_kernel<2>;
    // the integer scorer reads query rows in 16-byte pieces
    if (choice == 2 && d.G <= 8 && (reinterpret_cast<uintptr_t>(q) & 15) == 0)
      k = d.G <= 4 ? score_i8_kernel<1> : score_i8_kernel<2>;
    cudaError_t e = cudaSuccess;
    if (run_tma(k, d, a, stages * d.Hkv, &e, st)) return e;
  }
  if (use_mma && d.bf16) {
    if (d.D == 128) return d.G <= 8 ? run_mma<128, 1>(d, a, st) : run_mma<128, 2>(d, a, st);
    return d.G <= 8 ? run_mma<64, 1>(d, a, st) : run_mma<64, 2>(d, a, st);
  }
  if (d.bf16) {
    return d.D == 128 ? simt_by_group<__nv_bfloat16, 128>(d, a, total, st)
                      : simt_by_group<__nv_bfloat16, 64>(d, a, total, st);
  }
  return d.D == 128 ? simt_by_group<float, 128>(d, a, total, st)
                    : simt_by_group<float, 64>(d, a, total, st);
}

cudaError_t launch_propose_scores_new_rows(const Dims& d, const void* q, int8_t* kq, float* scale,
                                           const void* k_new, float* scores, uint32_t* hist,
                                           bool sum_group, int32_t* status, cudaStream_t st) {
  if (!d.bf16 || d.D != 128 || d.G > 8 || (reinterpret_cast<uintptr_t>(q) & 15) != 0 ||
      (reinterpret_cast<uintptr_t>(k_new) & 7) != 0)
    return cudaErrorInvalidValue;
  int64_t stages = 0;
  for (int b = 0; b < d.B; ++b) stages += cdiv(d.cu_host[b + 1] - d.cu_host[b], kStageRows);
  if (stages == 0) return cudaSuccess;
  ScoreArgs a{q, kq, scale, scores, hist, d.cu_dev, d.T, d.B, d.Hkv, d.G, status, nullptr, nullptr,
              k_new, kq, scale, sum_group ? 1 : 0};
  cudaError_t e = cudaSuccess;
  if (!run_tma(d.G <= 4 ? score_i8_kernel<1> : score_i8_kernel<2>, d, a, stages * d.Hkv, &e, st))
    return cudaErrorInvalidValue;
  return e;
}

cudaError_t launch_propose_scores_int2(const Dims& d, const void* q, const uint8_t* codes,
                                       const uint16_t* params, float* scores, uint32_t* hist,
                                       int32_t* status, cudaStream_t st) {
  if (!d.bf16 || d.D != 128) return cudaErrorInvalidValue;
  int64_t stages = 0;
  for (int b = 0; b < d.B; ++b) stages += cdiv(d.cu_host[b + 1] - d.cu_host[b], kStageRows);
  if (stages == 0) return cudaSuccess;
  ScoreArgs a{q, nullptr, nullptr, scores, hist, d.cu_dev, d.T, d.B, d.Hkv, d.G, status, codes, params,
              nullptr, nullptr, nullptr, 0};
  return d.G <= 8 ? run_int2<1>(d, a, stages * d.Hkv, st) : run_int2<2>(d, a, stages * d.Hkv, st);
}

}  // namespace prism
