// Refined layer, fused: exact rescoring of the candidate pool, top-kappa
// selection inside it, and sparse flash-decode over the selected rows, in one
// launch per layer (Prism Attention, sec. 4.1 "Proposal-Refined Index
// Sharing": each refined layer re-selects its own top-kappa inside the pool;
// sec. 1 / 2.1: token-level sparse attention over the selected tokens).
//
// One thread-block cluster of CL CTAs owns one (sequence, KV head) row; two
// CTAs fit on an SM.  With CL > 1, rank 0 coordinates and ranks 1..CL-1 are
// workers, each owning a contiguous slice of the row's pool (CL = 1: one CTA
// does both jobs):
//   1. a worker streams its slice's key rows through a ring of shared-memory
//      stages with cp.async (16-byte chunks XOR-swizzled by row); the dot
//      products with the G query heads are a [rows x d] x [d x G] contraction
//      done by mma.sync (bf16 operands, fp32 accumulation, exact bf16
//      products) from ldmatrix fragments -- an fp32 cache takes a CUDA-core
//      path; logits stay in the worker, and the selection key
//      ord(max_g q_g . k) is also stored into rank 0's shared memory;
//   2. rank 0 finds the kappa-th largest key: a 12-bit histogram of all keys
//      locates the bin holding it, the (few) keys in that bin are ranked
//      exactly by (key desc, pool slot asc), giving the threshold key T and
//      the last taken slot I*; rank 0 also counts every slice's selected
//      members into output offsets (a 3-pass radix select is the fallback
//      when the bin holds too many keys);
//   3. every worker keeps the members with key > T or (key == T and slot <=
//      I*), and writes their positions to idx in ascending order;
//   4. softmax partial over the selected members: logits are on chip, so
//      the CTA maximum and the weights 2^(l - m) come first and only the
//      value rows are streamed (same ring);
//   5. workers store their partials (m, l, o) into rank 0, which merges them
//      and writes out and lse.
// Three cluster barriers per launch; nothing goes to global scratch.  Bytes
// per row: kappa_p key rows and kappa value rows, d * sizeof(T) each.
#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.h"

namespace cg = cooperative_groups;

namespace prism {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kStages = 4;
constexpr int kStageBytes = 16384;
constexpr int kRingMin = kStages * kStageBytes;
constexpr int kHistBins = 4096;                      // first radix digit: 12 bits
constexpr int kHistWords = kHistBins + kHistBins / 32;  // one pad word per 32 bins
constexpr int kCandCap = 2048;                       // keys ranked directly by rank 0
constexpr int kMaxCluster = 16;

struct RDArgs {
  const void* q;
  const void* k;
  const void* v;
  const void* k_next;  // next layer's keys: pool rows prefetched into L2, or null
  const int32_t* cu;
  const int32_t* pool;
  const int32_t* pool_cnt;
  int kp;     // pool row stride (kappa_p)
  int kappa;  // selection budget and idx row stride
  int Hkv, G, Hq;
  int64_t T;
  int mc;     // slice capacity (members per worker)
  int ring;   // bytes of the stage ring (rank 0: selection and merge scratch)
  float scale_log2;
  int32_t* idx;
  int32_t* cnt;
  float* out;
  float* lse;
  int32_t* status;
};

// padded histogram index: 16 (or 4) consecutive bins per thread are read
// without bank conflicts
__device__ __forceinline__ int hpad(int b) { return b + (b >> 5); }

// Byte offset of 16-byte chunk `c` of row `r` in a stage: chunks are XOR
// swizzled by the row's low 3 bits, so 8 consecutive rows read at one chunk
// index (ldmatrix, or lane groups) hit 8 different bank groups.
template <int RB>
__device__ __forceinline__ int swz(int r, int c) {
  return r * RB + ((c ^ (r & 7)) << 4);
}

// Streams `rows` cache rows (row j at position spos[list ? list[j] : j] of
// base; negative positions are zero-filled without reading) through the
// stage ring and calls body(first_row, stage, rows_in_chunk) once per chunk
// of SR rows, with kStages chunks in flight.
template <typename T, int D, typename Body, typename Hook>
__device__ __forceinline__ void stream_rows(const T* base, const int* spos, const int* list,
                                            int rows, unsigned char* ring, Body body, Hook hook) {
  constexpr int RB = D * (int)sizeof(T);  // row bytes
  constexpr int VPR = RB / 16;            // 16-byte chunks per row
  constexpr int SR = kStageBytes / RB;
  const int tid = threadIdx.x;
  const int nchunk = (rows + SR - 1) / SR;
  auto issue = [&](int c) {
    if (c < nchunk) {
      const int r0 = c * SR, n = min(SR, rows - r0);
      unsigned char* buf = ring + (c % kStages) * kStageBytes;
      for (int x = tid; x < n * VPR; x += kThreads) {
        const int r = x / VPR, vv = x - r * VPR;
        const int pos = spos[list ? list[r0 + r] : r0 + r];
        const T* src = base + (int64_t)(pos >= 0 ? pos : 0) * D + vv * (16 / (int)sizeof(T));
        cp_async16(smem_u32(buf + swz<RB>(r, vv)), src, pos >= 0);
      }
    }
    cp_async_commit();  // one group per call (possibly empty): constant wait depth
  };
#pragma unroll
  for (int c = 0; c < kStages; ++c) issue(c);
  hook();  // runs while the first stages are in flight
  for (int c = 0; c < nchunk; ++c) {
    cp_async_wait<kStages - 1>();
    __syncthreads();
    body(c * SR, ring + (c % kStages) * kStageBytes, min(SR, rows - c * SR));
    __syncthreads();
    issue(c + kStages);
  }
  cp_async_wait<0>();
}

// split cluster barrier: arrive early, wait late
__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;\n" ::: "memory");
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t& a0, uint32_t& a1,
                                            uint32_t& a2, uint32_t& a3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(a0), "=r"(a1), "=r"(a2), "=r"(a3)
               : "r"(addr));
}

__device__ __forceinline__ void mma_bf16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Local first-digit histogram, two 16-bit counts per word (bin b in word
// b / 2, high half when b is odd); lanes sharing a bin issue one atomic.
__device__ __forceinline__ void warp_hist_add_packed(uint32_t* lh, uint32_t bin, bool valid) {
  const unsigned act = __ballot_sync(0xffffffffu, valid);
  if (!act) return;
  const unsigned peers = __match_any_sync(0xffffffffu, valid ? bin : 0xffffffffu) & act;
  const int lane = threadIdx.x & 31;
  if (valid && (peers & ((1u << lane) - 1u)) == 0)
    atomicAdd(&lh[bin >> 1], (uint32_t)__popc(peers) << ((bin & 1u) * 16));
}

// ---- phase 1: logits of one chunk of key rows ------------------------------
// The key of slice member i goes to keys[i] and to gkeys[lo + i] (rank 0).

// Tensor cores (bf16 cache): warp w takes 16-row tiles w, w + 8, ...; rows
// are the M dimension, query heads the N dimension (8 per n-tile).
template <int D, int GP>
struct ScoreMma {
  static constexpr int KS = D / 16;
  static constexpr int NT = (GP + 7) / 8;
  uint32_t bq[NT][KS][2];

  __device__ __forceinline__ void init(const __nv_bfloat16* q, int G) {
    const int lane = threadIdx.x & 31, g = lane >> 2, tig = lane & 3;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int n = nt * 8 + g;
#pragma unroll
      for (int s = 0; s < KS; ++s) {
        if (n < G) {
          const uint32_t* qr = reinterpret_cast<const uint32_t*>(q + (int64_t)n * D + s * 16);
          bq[nt][s][0] = qr[tig];
          bq[nt][s][1] = qr[4 + tig];
        } else {
          bq[nt][s][0] = bq[nt][s][1] = 0u;
        }
      }
    }
  }

  __device__ __forceinline__ void run(const unsigned char* buf, int r0, int nrows, const int* spos,
                                      int G, int mc, float* dots, uint32_t* keys,
                                      uint32_t* gkeys, uint32_t* lhist) const {
    constexpr int RB = D * 2;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, tig = lane & 3;
    const int ntile = (nrows + 15) >> 4;
    for (int t = warp; t < ntile; t += kWarps) {
      float acc[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.0f;
      const int lrow = t * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
      for (int s = 0; s < KS; ++s) {
        uint32_t a0, a1, a2, a3;
        ldmatrix_x4(smem_u32(buf + swz<RB>(lrow, 2 * s + (lane >> 4))), a0, a1, a2, a3);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma_bf16(acc[nt], a0, a1, a2, a3, bq[nt][s][0], bq[nt][s][1]);
      }
      // c0,c1: row t*16+g, heads col, col+1; c2,c3: row t*16+g+8
      float mA = -INFINITY, mB = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int col = nt * 8 + 2 * tig;
        if (col < G) { mA = fmaxf(mA, acc[nt][0]); mB = fmaxf(mB, acc[nt][2]); }
        if (col + 1 < G) { mA = fmaxf(mA, acc[nt][1]); mB = fmaxf(mB, acc[nt][3]); }
      }
      mA = fmaxf(mA, __shfl_xor_sync(0xffffffffu, mA, 1));
      mA = fmaxf(mA, __shfl_xor_sync(0xffffffffu, mA, 2));
      mB = fmaxf(mB, __shfl_xor_sync(0xffffffffu, mB, 1));
      mB = fmaxf(mB, __shfl_xor_sync(0xffffffffu, mB, 2));
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int r = t * 16 + g + 8 * half;
        if (r < nrows) {
          const int i = r0 + r;
          const bool ok = spos[i] >= 0;  // an out-of-range position ranks last, weighs 0
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            const int col = nt * 8 + 2 * tig;
            if (col < G) dots[col * mc + i] = ok ? acc[nt][2 * half] : -INFINITY;
            if (col + 1 < G) dots[(col + 1) * mc + i] = ok ? acc[nt][2 * half + 1] : -INFINITY;
          }
          if (tig == half) {
            const uint32_t key = ord_key(ok ? (half ? mB : mA) : -INFINITY);
            keys[i] = key;
            gkeys[i] = key;
          }
        }
      }
      // first radix digit of this tile's keys into the local histogram
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int r = t * 16 + g + 8 * half;
        const bool mine = r < nrows && tig == half;
        const uint32_t key = mine ? keys[r0 + r] : 0u;
        if (lhist) warp_hist_add_packed(lhist, key >> 20, mine);
      }
    }
  }
};

// CUDA cores (fp32 cache): lane groups of LPR lanes per row, transposed
// butterfly over the query heads.
template <typename T, int D, int GP>
struct ScoreSimt {
  static constexpr int E = Vec16<T>::E;
  static constexpr int LPR = D / E;
  static constexpr int RPW = 32 / LPR;
  static constexpr int NG = kThreads / LPR;
  using GS = GroupSumT<GP, LPR>;
  float qf[GP][E];

  __device__ __forceinline__ void init(const T* q, int G) {
    const int li = (threadIdx.x & 31) % LPR;
#pragma unroll
    for (int g = 0; g < GP; ++g) {
      if (g < G) {
        Vec16<T>::unpack(ld16(q + (int64_t)g * D + li * E), qf[g]);
      } else {
#pragma unroll
        for (int e = 0; e < E; ++e) qf[g][e] = 0.0f;
      }
    }
  }

  __device__ __forceinline__ void run(const unsigned char* buf, int r0, int nrows, const int* spos,
                                      int G, int mc, float* dots, uint32_t* keys,
                                      uint32_t* gkeys, uint32_t* lhist) const {
    constexpr int RB = D * (int)sizeof(T);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int sub = lane / LPR, li = lane % LPR;
    const int h0 = GS::head0(li);
    for (int wb = warp * RPW; wb < nrows; wb += NG) {  // warp-uniform trip count
      const int r = wb + sub;
      const bool in = r < nrows;
      float f[E];
      Vec16<T>::unpack(in ? *reinterpret_cast<const uint4*>(buf + swz<RB>(r, li))
                          : make_uint4(0, 0, 0, 0), f);
      float acc[GP];
#pragma unroll
      for (int g = 0; g < GP; ++g) {
        float s = 0.0f;
#pragma unroll
        for (int e = 0; e < E; ++e) s = fmaf(qf[g][e], f[e], s);
        acc[g] = s;
      }
      GS::run(acc, li);
      float best = -INFINITY;
#pragma unroll
      for (int j = 0; j < GS::NH; ++j)
        if (h0 + j < G) best = fmaxf(best, acc[j]);
#pragma unroll
      for (int o = LPR / 2; o >= LPR / GS::SPLIT && o > 0; o >>= 1)
        best = fmaxf(best, __shfl_xor_sync(0xffffffffu, best, o));
      if (in) {
        const int i = r0 + r;
        const bool ok = spos[i] >= 0;
        if (GS::writer(li)) {
#pragma unroll
          for (int j = 0; j < GS::NH; ++j)
            if (h0 + j < G) dots[(h0 + j) * mc + i] = ok ? acc[j] : -INFINITY;
        }
        if (li == 0) {
          const uint32_t key = ord_key(ok ? best : -INFINITY);
          keys[i] = key;
          gkeys[i] = key;
        }
      }
      const bool mine = in && li == 0;
      const uint32_t key = mine ? ord_key(spos[r0 + r] >= 0 ? best : -INFINITY) : 0u;
      if (lhist) warp_hist_add_packed(lhist, key >> 20, mine);
    }
  }
};

template <typename T, int D, int GP>
struct ScorePick {
  using type = ScoreSimt<T, D, GP>;
};
template <int D, int GP>
struct ScorePick<__nv_bfloat16, D, GP> {
  using type = ScoreMma<D, GP>;
};

// ---- phase 2 (rank 0): exact threshold over the gathered keys -------------

// Locates the bin of `digit` (bits [shift, shift + log2 nb) of keys matching
// prefix under pmask) that holds the r-th largest such key; returns
// (bin, count above the bin, count in the bin) in s_res[0..2].  hist is
// padded (hpad).  Whole CTA.
__device__ void find_bin(const uint32_t* gk, int n, uint32_t prefix, uint32_t pmask, int shift,
                         int nb, int r, uint32_t* hist, int* scratch, int* s_res) {
  const int tid = threadIdx.x;
  for (int i = tid; i < nb + nb / 32; i += kThreads) hist[i] = 0;
  __syncthreads();
  for (int i0 = tid & ~31; i0 < n; i0 += kThreads) {  // warp-uniform trip count
    const int i = i0 + (tid & 31);
    const uint32_t key = i < n ? gk[i] : 0u;
    const uint32_t bin = (key >> shift) & (uint32_t)(nb - 1);
    warp_hist_add(hist, (uint32_t)hpad((int)bin), i < n && (key & pmask) == prefix);
  }
  __syncthreads();
  const int per = nb / kThreads;  // consecutive bins of this thread (16 or 4)
  int v = 0;
  for (int j = 0; j < per; ++j) v += (int)hist[hpad(tid * per + j)];
  int total;
  const int excl = block_excl_scan(v, scratch, &total);
  int above = total - excl - v;
  for (int j = per - 1; j >= 0; --j) {
    const int c = (int)hist[hpad(tid * per + j)];
    if (above < r && r <= above + c) {
      s_res[0] = tid * per + j;
      s_res[1] = above;
      s_res[2] = c;
    }
    above += c;
  }
  __syncthreads();
}

// Exact threshold (key T, last taken slot I*) of the k-th largest of gk[0..n)
// under (key desc, slot asc): the selected slots are those with key > T, or
// key == T and slot <= I*.  hist holds the 12-bit histogram of the first
// digit (padded).  The keys of the bin holding the threshold are listed in
// slot order (they are few) and the two remaining digits (10 + 10 bits) are
// resolved on the list; keys equal to T are taken in slot order.  When the
// bin holds more than kCandCap keys the digits run over all keys instead.
// Whole CTA; `ws` holds 2*kCandCap words plus a count table.
__device__ void select_row(const uint32_t* gk, int n, int k, uint32_t* hist, uint32_t* ws,
                           int* scratch, int* s_res, uint32_t* T_out, int* istar_out) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t* ckey = ws;
  int* cslot = reinterpret_cast<int*>(ws + kCandCap);
  int* tab = cslot + kCandCap;  // per (256-slot block, warp): listed keys before it
  __shared__ int s_I;

  // first digit from the histogram
  {
    constexpr int per = kHistBins / kThreads;
    int v = 0;
    for (int j = 0; j < per; ++j) v += (int)hist[hpad(tid * per + j)];
    int total;
    const int excl = block_excl_scan(v, scratch, &total);
    int above = total - excl - v;
    for (int j = per - 1; j >= 0; --j) {
      const int c = (int)hist[hpad(tid * per + j)];
      if (above < k && k <= above + c) {
        s_res[0] = tid * per + j;
        s_res[1] = above;
        s_res[2] = c;
      }
      above += c;
    }
    __syncthreads();
  }
  const uint32_t b1 = (uint32_t)s_res[0];
  int r = k - s_res[1];
  const int nb1 = s_res[2];
  const bool listed = nb1 <= kCandCap;
  if (listed) {
    // the bin's keys, in slot order: count per (block, warp), scan, place
    const int nblk = (n + kThreads - 1) / kThreads;
#pragma unroll 4
    for (int u = 0; u < nblk; ++u) {
      const int i = u * kThreads + tid;
      const bool c = i < n && (gk[i] >> 20) == b1;
      const unsigned bal = __ballot_sync(0xffffffffu, c);
      if (lane == 0) tab[u * kWarps + warp] = __popc(bal);
    }
    __syncthreads();
    {
      const int ne = nblk * kWarps;
      const int per = (ne + kThreads - 1) / kThreads;
      int v = 0;
      for (int j = 0; j < per; ++j) {
        const int e = tid * per + j;
        if (e < ne) v += tab[e];
      }
      int total;
      int acc = block_excl_scan(v, scratch, &total);
      for (int j = 0; j < per; ++j) {
        const int e = tid * per + j;
        if (e < ne) {
          const int c = tab[e];
          tab[e] = acc;
          acc += c;
        }
      }
      __syncthreads();
    }
#pragma unroll 4
    for (int u = 0; u < nblk; ++u) {
      const int i = u * kThreads + tid;
      const uint32_t key = i < n ? gk[i] : 0u;
      const bool c = i < n && (key >> 20) == b1;
      const unsigned bal = __ballot_sync(0xffffffffu, c);
      if (c) {
        const int at = tab[u * kWarps + warp] + __popc(bal & ((1u << lane) - 1u));
        ckey[at] = key;
        cslot[at] = i;
      }
    }
    __syncthreads();
  }
  const uint32_t* sk = listed ? ckey : gk;  // keys the last two digits run over
  const int ns = listed ? nb1 : n;
  uint32_t prefix = b1 << 20, pmask = 0xFFF00000u;
  find_bin(sk, ns, prefix, pmask, 10, 1024, r, hist, scratch, s_res);
  prefix |= (uint32_t)s_res[0] << 10;
  pmask |= 0x000FFC00u;
  r -= s_res[1];
  find_bin(sk, ns, prefix, pmask, 0, 1024, r, hist, scratch, s_res);
  prefix |= (uint32_t)s_res[0];
  r -= s_res[1];
  const uint32_t T = prefix;
  // the r-th key equal to T in slot order (the list is in slot order too):
  // 32-key warp blocks in order, counted with ballots
  {
    __shared__ int s_wc[kWarps];
    const uint32_t* ek = listed ? ckey : gk;
    int before = 0;
    for (int blk0 = 0; blk0 * 32 < ns && before < r; blk0 += kWarps) {  // CTA-uniform
      const int j = (blk0 + warp) * 32 + lane;
      const unsigned eqm = __ballot_sync(0xffffffffu, j < ns && ek[j] == T);
      if (lane == 0) s_wc[warp] = __popc(eqm);
      __syncthreads();
      int mine = before, tot = before;
      for (int w = 0; w < kWarps; ++w) {
        if (w < warp) mine += s_wc[w];
        tot += s_wc[w];
      }
      if (lane == 0 && mine < r && r <= mine + __popc(eqm)) {
        unsigned m = eqm;
        for (int t = 1; t < r - mine; ++t) m &= m - 1;
        const int jj = j - lane + __ffs(m) - 1;
        s_I = listed ? cslot[jj] : jj;
      }
      before = tot;
      __syncthreads();
    }
  }
  *T_out = T;
  *istar_out = s_I;
  __syncthreads();
}

template <typename T, int D, int GP>
__global__ void __launch_bounds__(kThreads, 2) refine_decode_kernel(const RDArgs a) {
  constexpr int E = Vec16<T>::E;
  constexpr int LPR = D / E;     // lanes per cache row (value pass)
  constexpr int RPW = 32 / LPR;
  constexpr int NG = kThreads / LPR;
  constexpr int RB = D * (int)sizeof(T);
  constexpr int PART = GP * D + 2 * GP;  // one partial: o[GP][D], m[GP], l[GP]

  extern __shared__ __align__(16) unsigned char dsm[];
  unsigned char* ring = dsm;                                         // a.ring bytes
  int* spos = reinterpret_cast<int*>(dsm + a.ring);                  // [mc]
  uint32_t* keys = reinterpret_cast<uint32_t*>(spos + a.mc);         // [mc]
  float* dots = reinterpret_cast<float*>(keys + a.mc);               // [GP][mc]
  float* pw = dots + GP * a.mc;                                      // [mc][GP] weights
  int* sel = reinterpret_cast<int*>(pw + GP * a.mc);                 // [mc]
  uint32_t* lhist = reinterpret_cast<uint32_t*>(sel + a.mc);         // [kHistBins / 2]

  __shared__ int scratch[33];
  __shared__ int s_res[3];
  __shared__ uint32_t s_thr;       // rank 0: threshold key T
  __shared__ int s_istar;          // rank 0: last taken pool slot among keys == T
  __shared__ int s_nsel;           // this worker's selected count (published)
  __shared__ int s_mine[3];        // this CTA's copy of (T, I*, offset)
  __shared__ float s_red[kWarps][GP];
  __shared__ float part_o[GP * D];  // this CTA's partial

  cg::cluster_group cluster = cg::this_cluster();
  const int CL = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const int row = blockIdx.x / CL;
  const int b = row / a.Hkv, h = row - b * a.Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  const int t0 = a.cu[b];
  const int L = a.cu[b + 1] - t0;
  int n = a.pool_cnt[row];
  if (n < 0 || n > a.kp) {
    if (rank == 0 && tid == 0) flag_status(a.status, PRISM_DEV_BAD_INDEX);
    n = n < 0 ? 0 : a.kp;
  }
  const int k = min(a.kappa, n);
  const int nworkers = CL > 1 ? CL - 1 : 1;
  const int wid = CL > 1 ? rank - 1 : 0;  // worker index (-1: coordinator)
  const int chunk = max(1, (n + nworkers - 1) / nworkers);
  const int lo = wid < 0 ? 0 : min(n, wid * chunk);
  const int hi = wid < 0 ? 0 : min(n, lo + chunk);
  const int m = hi - lo;
  const int32_t* pool = a.pool + (int64_t)row * a.kp + lo;
  const int64_t rowbase = ((int64_t)h * a.T + t0) * D;
  const T* kb = static_cast<const T*>(a.k) + rowbase;
  const T* vb = static_cast<const T*>(a.v) + rowbase;
  const T* qrow = static_cast<const T*>(a.q) + ((int64_t)b * a.Hq + (int64_t)h * a.G) * D;
  // rank 0's ring: the gathered keys, the first-digit histogram, the
  // candidate list (a lone CTA keeps its keys in `keys` and builds the
  // histogram after streaming, when the ring is free)
  const int gkw = CL > 1 ? ((n + 31) & ~31) : 0;
  uint32_t* ring0 = CL > 1 ? reinterpret_cast<uint32_t*>(cluster.map_shared_rank(ring, 0))
                           : reinterpret_cast<uint32_t*>(ring);
  uint32_t* gk0 = CL > 1 ? ring0 : keys;
  uint32_t* ghist0 = ring0 + gkw;

  // ---- 0. the slice's positions (an out-of-range one is flagged, skipped)
  for (int i = tid; i < m; i += kThreads) {
    const int p = pool[i];
    const bool ok = p >= 0 && p < L;
    if (!ok) flag_status(a.status, PRISM_DEV_BAD_INDEX);
    spos[i] = ok ? p : -1;
  }
  for (int i = tid; i < kHistBins / 2; i += kThreads) lhist[i] = 0u;
  if (rank == 0 && CL > 1)
    for (int i = tid; i < kHistWords; i += kThreads) ghist0[i] = 0u;
  __syncthreads();
  cluster_arrive();  // rank 0's histogram is cleared once every CTA has arrived

  // ---- 1. exact logits and keys of the slice (workers)
  if (wid >= 0) {
    typename ScorePick<T, D, GP>::type sc;
    sc.init(qrow, a.G);
    uint32_t* gkeys = gk0 + lo;
    stream_rows<T, D>(kb, spos, nullptr, m, ring,
                      [&](int r0, const unsigned char* buf, int nrows) {
                        sc.run(buf, r0, nrows, spos, a.G, a.mc, dots, keys, gkeys, lhist);
                      },
                      [] {});
  }
  // the next layer's key rows at the same pool positions into L2, while
  // this layer selects and attends (the DRAM is otherwise idle meanwhile)
  if (a.k_next && wid >= 0) {
    const T* kn = static_cast<const T*>(a.k_next) + rowbase;
    for (int i = tid; i < m; i += kThreads) {
      const int pos = spos[i];
      if (pos >= 0)
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;\n" ::"l"(kn + (int64_t)pos * D),
                     "r"(RB)
                     : "memory");
    }
  }
  cluster_wait();
  __syncthreads();
  // the local first-digit histogram into rank 0's (a lone CTA: into its ring)
  if (wid >= 0) {
    uint32_t* gh = ghist0;
    if (CL == 1) {
      for (int i = tid; i < kHistWords; i += kThreads) gh[i] = 0u;
      __syncthreads();
    }
    for (int w = tid; w < kHistBins / 2; w += kThreads) {
      const uint32_t v = lhist[w];
      if (v & 0xFFFFu) atomicAdd(gh + hpad(2 * w), v & 0xFFFFu);
      if (v >> 16) atomicAdd(gh + hpad(2 * w + 1), v >> 16);
    }
  }
  cluster.sync();  // S1: every key and the histogram are in rank 0

  // ---- 2. rank 0: the threshold (T, I*)
  if (rank == 0) {
    uint32_t* hist = reinterpret_cast<uint32_t*>(ring) + gkw;
    uint32_t* cands = hist + kHistWords;
    uint32_t thr = 0u;
    int istar = 0x7fffffff;  // n <= kappa: every key is >= 0 and every slot <= I*
    if (n > a.kappa)
      select_row(CL > 1 ? reinterpret_cast<uint32_t*>(ring) : keys, n, k, hist, cands, scratch,
                 s_res, &thr, &istar);
    if (tid == 0) {
      s_thr = thr;
      s_istar = istar;
    }
  }
  cluster.sync();  // S2: rank 0's answer is ready
  if (tid == 0) {
    s_mine[0] = (int)*cluster.map_shared_rank(&s_thr, 0);
    s_mine[1] = *cluster.map_shared_rank(&s_istar, 0);
  }
  __syncthreads();
  const uint32_t thr = (uint32_t)s_mine[0];
  const int istar = s_mine[1];

  // ---- 3. selected members of the slice, positions to idx (ascending)
  auto taken = [&](int i) {
    const uint32_t key = keys[i];
    return key > thr || (key == thr && lo + i <= istar);
  };
  {
    int c = 0;
    for (int i = tid; i < m; i += kThreads) c += taken(i);
    int tot;
    block_excl_scan(c, scratch, &tot);
    if (tid == 0) s_nsel = tot;
  }
  cluster.sync();  // S2b: every worker's selected count is published
  if (warp == 0) {
    int c = 0;
    if (lane < wid) c = *cluster.map_shared_rank(&s_nsel, lane + 1);  // workers before this one
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
    if (lane == 0) s_mine[2] = c;
  }
  __syncthreads();
  int nsel = 0;
  {
    // blocks of 256 consecutive members, in order: ballot + prefix
    int32_t* idx = a.idx + (int64_t)row * a.kappa;
    __shared__ int s_wsel[kWarps];
    int base = 0;
    for (int i0 = 0; i0 < m; i0 += kThreads) {
      const int i = i0 + tid;
      const bool s = i < m && taken(i);
      const unsigned bal = __ballot_sync(0xffffffffu, s);
      if (lane == 0) s_wsel[warp] = __popc(bal);
      __syncthreads();
      int before = base;
      for (int w = 0; w < warp; ++w) before += s_wsel[w];
      int tot = base;
      for (int w = 0; w < kWarps; ++w) tot += s_wsel[w];
      if (s) {
        const int o = before + __popc(bal & ((1u << lane) - 1u));
        const int slot = s_mine[2] + o;
        if (slot < k) idx[slot] = pool[i];
        else flag_status(a.status, PRISM_DEV_TOO_LONG);  // unreachable if counts are right
        sel[o] = i;
      }
      base = tot;
      __syncthreads();
    }
    nsel = base;
    for (int s = k + rank * kThreads + tid; s < a.kappa; s += CL * kThreads) idx[s] = -1;
    if (rank == 0 && tid == 0) a.cnt[row] = k;
  }

  // ---- 4. softmax partial over the selected members of the slice
  float mx[GP];
#pragma unroll
  for (int g = 0; g < GP; ++g) mx[g] = -INFINITY;
  for (int j = tid; j < nsel; j += kThreads) {
    const int i = sel[j];
#pragma unroll
    for (int g = 0; g < GP; ++g)
      if (g < a.G) mx[g] = fmaxf(mx[g], dots[g * a.mc + i]);
  }
#pragma unroll
  for (int g = 0; g < GP; ++g) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx[g] = fmaxf(mx[g], __shfl_xor_sync(0xffffffffu, mx[g], o));
    if (lane == 0) s_red[warp][g] = mx[g];
  }
  __syncthreads();
#pragma unroll
  for (int g = 0; g < GP; ++g) {
    float v = s_red[0][g];
#pragma unroll
    for (int w = 1; w < kWarps; ++w) v = fmaxf(v, s_red[w][g]);
    mx[g] = v * a.scale_log2;  // CTA maximum logit (log2 domain); -inf if nothing selected
  }
  __syncthreads();
  float lsum[GP];
#pragma unroll
  for (int g = 0; g < GP; ++g) lsum[g] = 0.0f;
  for (int j = tid; j < nsel; j += kThreads) {
    const int i = sel[j];
#pragma unroll
    for (int g = 0; g < GP; ++g) {
      const float l = g < a.G ? dots[g * a.mc + i] : -INFINITY;
      const float p = l == -INFINITY ? 0.0f : exp2f(l * a.scale_log2 - mx[g]);
      pw[j * GP + g] = p;
      lsum[g] += p;
    }
  }
#pragma unroll
  for (int g = 0; g < GP; ++g) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) lsum[g] += __shfl_xor_sync(0xffffffffu, lsum[g], o);
    if (lane == 0) s_red[warp][g] = lsum[g];
  }
  const int sub = lane / LPR, li = lane % LPR;
  float o[GP][E];
#pragma unroll
  for (int g = 0; g < GP; ++g)
#pragma unroll
    for (int e = 0; e < E; ++e) o[g][e] = 0.0f;
  if (wid >= 0) {
    // stream the selected value rows (the weights are read after the first
    // stage barrier inside stream_rows)
    stream_rows<T, D>(
        vb, spos, sel, nsel, ring,
        [&](int j0, const unsigned char* buf, int nrows) {
          for (int r = warp * RPW + sub; r < nrows; r += NG) {
            float f[E];
            Vec16<T>::unpack(*reinterpret_cast<const uint4*>(buf + swz<RB>(r, li)), f);
            const float* p = pw + (j0 + r) * GP;
#pragma unroll
            for (int g = 0; g < GP; ++g) {
              const float pg = p[g];
#pragma unroll
              for (int e = 0; e < E; ++e) o[g][e] = fmaf(pg, f[e], o[g][e]);
            }
          }
        },
        [] {});
  }
  // lane groups of a warp hold the same feature slice: add them, then warps
#pragma unroll
  for (int g = 0; g < GP; ++g)
#pragma unroll
    for (int s = LPR; s < 32; s <<= 1)
#pragma unroll
      for (int e = 0; e < E; ++e) o[g][e] += __shfl_xor_sync(0xffffffffu, o[g][e], s);
  if (wid >= 0) {  // (a coordinating rank 0 has no partial; workers fill its ring)
    __syncthreads();  // the ring is free (value rows consumed): warp partials go there
    float* comb = reinterpret_cast<float*>(ring);  // [kWarps][GP][D]
    if (sub == 0) {
#pragma unroll
      for (int g = 0; g < GP; ++g)
#pragma unroll
        for (int e = 0; e < E; ++e) comb[(warp * GP + g) * D + li * E + e] = o[g][e];
    }
    __syncthreads();
    for (int i = tid; i < GP * D; i += kThreads) {
      float acc = 0.0f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) acc += comb[w * GP * D + i];
      part_o[i] = acc;
    }
    __syncthreads();
  }
  // publish this worker's partial into rank 0's ring (rank 0 keeps its own)
  {
    float* dst = reinterpret_cast<float*>(CL > 1 ? cluster.map_shared_rank(ring, 0) : ring) +
                 (size_t)(CL > 1 ? wid : 0) * PART;
    if (wid >= 0) {
      for (int i = tid; i < GP * D; i += kThreads) dst[i] = part_o[i];
      if (tid < GP) {
        float s = 0.0f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) s += s_red[w][tid];
        dst[GP * D + tid] = mx[tid];
        dst[GP * D + GP + tid] = s;
      }
    }
  }
  cluster.sync();  // S3: every partial is in rank 0

  // ---- 5. rank 0 merges the partials
  if (rank == 0) {
    const float* parts = reinterpret_cast<const float*>(ring);
    for (int i = tid; i < a.G * D; i += kThreads) {
      const int g = i / D, j = i - g * D;
      float M = -INFINITY;
      for (int w = 0; w < nworkers; ++w) M = fmaxf(M, parts[w * PART + GP * D + g]);
      float Ls = 0.0f, O = 0.0f;
      if (M != -INFINITY) {
        for (int w = 0; w < nworkers; ++w) {
          const float mw = parts[w * PART + GP * D + g];
          if (mw == -INFINITY) continue;
          const float wt = exp2f(mw - M);
          Ls = fmaf(wt, parts[w * PART + GP * D + GP + g], Ls);
          O = fmaf(wt, parts[w * PART + i], O);
        }
      }
      const int64_t hq = (int64_t)b * a.Hq + (int64_t)h * a.G + g;
      a.out[hq * D + j] = Ls > 0.0f ? O / Ls : 0.0f;
      if (j == 0 && a.lse)
        a.lse[hq] = Ls > 0.0f ? (M + log2f(Ls)) * 0.69314718055994530942f : -INFINITY;
    }
  }
}

template <int GP>
constexpr int per_member_bytes() {
  return (int)(2 * sizeof(int) + sizeof(uint32_t) + 2 * GP * sizeof(float));
}
constexpr int kLocalHistBytes = kHistBins / 2 * 4;

// Stage ring size: rank 0 also keeps there the gathered keys with the
// selection scratch, and later the workers' partials.
int ring_bytes(int kappa_p, int GP, int D, int cl) {
  const int sel = (((kappa_p + 31) & ~31) + kHistWords + 2 * kCandCap +
                   ((kappa_p + kThreads - 1) / kThreads) * kWarps) * 4;
  const int parts = cl * (GP * D + 2 * GP) * 4;
  const int comb = kWarps * GP * D * 4;
  int need = sel > parts ? sel : parts;
  need = need > comb ? need : comb;
  need = (need + 15) & ~15;
  return need > kRingMin ? need : kRingMin;
}

// dynamic shared memory one CTA may use (two CTAs per SM when it is small)
constexpr int kDynBudget = 227 * 1024 - 8 * 1024;

template <typename T, int D, int GP>
cudaError_t run(const Dims& d, RDArgs a, int cl, cudaStream_t st) {
  auto kern = refine_decode_kernel<T, D, GP>;
  const int smem = a.ring + a.mc * per_member_bytes<GP>() + kLocalHistBytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  if (cl > 8) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(d.B * d.Hkv * cl));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)cl;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

template <typename T, int D>
cudaError_t by_group(const Dims& d, const RDArgs& a, int cl, cudaStream_t st) {
  switch (padded_group(d.G)) {
    case 1: return run<T, D, 1>(d, a, cl, st);
    case 2: return run<T, D, 2>(d, a, cl, st);
    case 4: return run<T, D, 4>(d, a, cl, st);
    case 8: return run<T, D, 8>(d, a, cl, st);
    default: return run<T, D, 16>(d, a, cl, st);
  }
}

}  // namespace

RefineDecodePlan plan_refine_decode(const Dims& d, int kappa_p) {
  const int rows = d.B * d.Hkv;
  const int GP = padded_group(d.G);
  const int per = (int)(2 * sizeof(int) + sizeof(uint32_t) + 2 * GP * sizeof(float));
  int cl = 1;
  while (cl < kMaxCluster && (int64_t)rows * cl < 2LL * d.num_sms) cl *= 2;
  auto need = [&](int c) {
    const int w = c > 1 ? c - 1 : 1;
    return ring_bytes(kappa_p, GP, d.D, c) + ((kappa_p + w - 1) / w + 3) / 4 * 4 * per +
           kLocalHistBytes;
  };
  while (cl < kMaxCluster && need(cl) > kDynBudget) cl *= 2;
  const int w = cl > 1 ? cl - 1 : 1;
  const int mc = ((kappa_p + w - 1) / w + 3) & ~3;
  const bool ok = need(cl) <= kDynBudget;
  return RefineDecodePlan{cl, mc, ok};
}

cudaError_t launch_refine_decode(const Dims& d, const RefineDecodePlan& p, const void* q,
                                 const void* k, const void* v, const void* k_next,
                                 const int32_t* pool,
                                 const int32_t* pool_cnt, int kappa_p, int kappa,
                                 float softmax_scale, int32_t* idx, int32_t* cnt, float* out,
                                 float* lse, int32_t* status, cudaStream_t st) {
  if (d.B * d.Hkv == 0) return cudaSuccess;
  RDArgs a{q, k, v, k_next, d.cu_dev, pool, pool_cnt, kappa_p, kappa, d.Hkv, d.G, d.Hq, d.T, p.mc,
           ring_bytes(kappa_p, padded_group(d.G), d.D, p.cluster),
           softmax_scale * 1.4426950408889634f, idx, cnt, out, lse, status};
  if (d.bf16)
    return d.D == 128 ? by_group<__nv_bfloat16, 128>(d, a, p.cluster, st)
                      : by_group<__nv_bfloat16, 64>(d, a, p.cluster, st);
  return d.D == 128 ? by_group<float, 128>(d, a, p.cluster, st)
                    : by_group<float, 64>(d, a, p.cluster, st);
}

}  // namespace prism
