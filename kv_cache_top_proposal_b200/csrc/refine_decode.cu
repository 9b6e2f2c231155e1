// Refined layer, fused: exact rescoring of the candidate pool, top-kappa
// selection inside it, and sparse flash-decode over the selected rows, in one
// launch per layer (Prism Attention, sec. 4.1 "Proposal-Refined Index
// Sharing": each refined layer re-selects its own top-kappa inside the pool;
// sec. 1 / 2.1: token-level sparse attention over the selected tokens).
//
// One thread-block cluster of CL CTAs owns one (sequence, KV head) row; two
// CTAs fit on an SM.  CTA r owns the contiguous slice r of the row's pool
// (pool slots are in ascending position order, so lower ranks hold lower
// positions):
//   1. the slice's key rows stream through a ring of shared-memory stages
//      with cp.async (16-byte chunks XOR-swizzled by row); the dot products
//      with the G query heads are a [rows x d] x [d x G] contraction done by
//      mma.sync (bf16 operands, fp32 accumulation, exact bf16 products) from
//      ldmatrix fragments -- an fp32 cache takes a CUDA-core path; the logits
//      stay in shared memory;
//   2. the selection key of a member is ord(max_g q_g . k) (or of the sum
//      over g, the group-sum variant; or, in the MASS instance, of the
//      group's softmax mass over the pool, after two cluster exchanges of
//      each head's maximum and normalizer); its first 12 bits go into the
//      CTA's own histogram (two 16-bit counts per word);
//   3. CTA c sums slice c of every CTA's histogram (distributed shared
//      memory reads, no remote atomics), and every CTA finds, from the
//      slice totals and then the right slice, the bin holding the kappa-th
//      largest key.  Unless the whole bin is taken,
//      the keys in it build a histogram of the next 10 bits in rank 0, and
//      then of the last 10: this gives the threshold prefix P (12, 22 or 32
//      bits) and how many keys at P are taken.  Keys at P are taken in
//      pool-slot order ("lower index wins");
//   4. the CTAs exchange their counts above and at P, which gives each one
//      its share of the keys at P and its output offset; it writes its
//      selected positions to idx in ascending order;
//   5. softmax partial over the selected members: the logits are on chip, so
//      the CTA maximum and the weights 2^(l - m) come first and only the
//      value rows are streamed (same ring);
//   6. every CTA owns one slice of the G x d outputs: the others store the
//      matching slices of their partials (o, m, l) into it, and it merges
//      them (every source's partial loaded at once) and writes out and lse.
// The same launch can append this token's K and V rows (rank 0 writes them
// into the cache; reads of that position take them directly), and may start
// while the previous refined layer still runs (programmatic dependent
// launch): until that layer ends it reads only the pool and the key rows.
// Nothing goes to global scratch.  Bytes per row: kappa_p key rows and kappa
// value rows, d * sizeof(T) each.
#include <cooperative_groups.h>

#include <type_traits>

#include "common.cuh"
#include "kernels.h"

namespace cg = cooperative_groups;

namespace prism {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kStages = 4;
constexpr int kStageBytes = 16384;
constexpr int kRing = kStages * kStageBytes;
constexpr int kBins1 = 4096;  // first radix digit: key bits 31..20
constexpr int kBins2 = 1024;  // second and third digits: bits 19..10, 9..0
// rank 0's packed histograms (two 16-bit counts per word): digits 1, 2, 3
constexpr int kH1 = 0;
constexpr int kH2 = kH1 + kBins1 / 2;
constexpr int kH3 = kH2 + kBins2 / 2;
constexpr int kHistWords = kH3 + kBins2 / 2;
constexpr int kMaxCount = 65535;  // largest pool a 16-bit bin count can hold
constexpr int kMaxCluster = 16;

struct RDArgs {
  const void* q;
  const void* k;
  const void* v;
  const void* k_next;  // next layer's keys: pool rows prefetched into L2, or null
  const void* k_new;   // [B][Hkv][d] this token's key row, appended first, or null
  const void* v_new;   // [B][Hkv][d] this token's value row, or null
  const int32_t* cu;
  const int32_t* pool;
  const int32_t* pool_cnt;
  int kp;     // pool row stride (kappa_p)
  int kappa;  // selection budget and idx row stride
  int Hkv, G, Hq;
  int64_t T;
  int mc;     // slice capacity (members per CTA)
  float scale_log2;
  int32_t* idx;
  int32_t* cnt;
  float* out;
  float* lse;
  int32_t* status;
  int agg;  // selection score over the group's query heads: 0 maximum, 1 sum, 2 softmax mass
};

// Byte offset of 16-byte chunk `c` of row `r` in a stage: chunks are XOR
// swizzled by the row's low 3 bits, so 8 consecutive rows read at one chunk
// index (ldmatrix, or lane groups) hit 8 different bank groups.
template <int RB>
__device__ __forceinline__ int swz(int r, int c) {
  return r * RB + ((c ^ (r & 7)) << 4);
}

// Streams `rows` cache rows (row j at position spos[list ? list[j] : j] of
// base; negative positions are zero-filled without reading; position npos is
// read from nrow instead when nrow is set) through the stage ring with
// cp.async, kStages chunks of SR rows in flight.  prime() issues the first
// kStages chunks; with defer_new it leaves the row at npos unwritten, and
// fill_new() later copies it from nrow (so prime() reads the cache only);
// run() calls body(first_row, stage, rows_in_chunk) once per chunk.
template <typename T, int D>
struct RowStream {
  static constexpr int RB = D * (int)sizeof(T);  // row bytes
  static constexpr int VPR = RB / 16;            // 16-byte chunks per row
  static constexpr int SR = kStageBytes / RB;    // rows per stage
  const T* base;
  const T* nrow;
  int npos;
  const int* spos;
  const int* list;
  int rows, nchunk;
  unsigned char* ring;

  __device__ __forceinline__ RowStream(const T* base_, const T* nrow_, int npos_, const int* spos_,
                                       const int* list_, int rows_, unsigned char* ring_)
      : base(base_), nrow(nrow_), npos(npos_), spos(spos_), list(list_), rows(rows_),
        nchunk((rows_ + SR - 1) / SR), ring(ring_) {}

  // thread t always copies 16-byte chunk t % VPR of rows t / VPR, t / VPR +
  // kThreads / VPR, ... (the row step is a multiple of 8, so the chunk's
  // swizzled position within a row is fixed too)
  __device__ __forceinline__ void issue(int c, bool defer_new) {
    static_assert(kThreads % VPR == 0 && (kThreads / VPR) % 8 == 0, "row step");
    if (c < nchunk) {
      const int r0 = c * SR, n = min(SR, rows - r0);
      unsigned char* buf = ring + (c % kStages) * kStageBytes;
      const int vv = threadIdx.x % VPR;
      const T* col = base + vv * (16 / (int)sizeof(T));
      for (int r = threadIdx.x / VPR; r < n; r += kThreads / VPR) {
        const int pos = spos[list ? list[r0 + r] : r0 + r];
        const bool fresh = nrow && pos == npos;
        if (fresh && defer_new) continue;
        const T* src = fresh ? nrow + vv * (16 / (int)sizeof(T)) : col + (int64_t)(pos >= 0 ? pos : 0) * D;
        cp_async16(smem_u32(buf + swz<RB>(r, vv)), src, pos >= 0);
      }
    }
    cp_async_commit();  // one group per call (possibly empty): constant wait depth
  }
  __device__ __forceinline__ void prime(bool defer_new) {
#pragma unroll
    for (int c = 0; c < kStages; ++c) issue(c, defer_new);
  }
  __device__ __forceinline__ void fill_new() {
    if (!nrow) return;
    const int lim = min(rows, kStages * SR);
    for (int i = threadIdx.x; i < lim; i += kThreads) {
      if (spos[list ? list[i] : i] != npos) continue;
      unsigned char* buf = ring + (i / SR) * kStageBytes;
      for (int vv = 0; vv < VPR; ++vv)
        *reinterpret_cast<uint4*>(buf + swz<RB>(i % SR, vv)) = ld16(nrow + vv * (16 / (int)sizeof(T)));
    }
  }
  template <typename Body>
  __device__ __forceinline__ void run(Body body) {
    for (int c = 0; c < nchunk; ++c) {
      cp_async_wait<kStages - 1>();
      __syncthreads();
      body(c * SR, ring + (c % kStages) * kStageBytes, min(SR, rows - c * SR));
      __syncthreads();
      issue(c + kStages, false);
    }
    cp_async_wait<0>();
  }
};

// programmatic dependent launch: wait for the previous kernel on the stream
// (a no-op when the launch did not overlap it), let the next one start
__device__ __forceinline__ void wait_previous_grid() {
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
}
__device__ __forceinline__ void allow_next_grid() {
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
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


// ---- phase 1: logits of one chunk of key rows ------------------------------
// dots[g * mc + i] = q_g . k_i for slice member i (-inf for a member whose
// position is out of range: it ranks last and weighs 0).

// Key rows of a bf16 cache, per warp: warp w streams its own 16-row tiles
// (w, w + kWarps, ...) through its own kWS slots of the ring with cp.async and
// scores each tile with mma.sync as soon as it lands, so the key phase has no
// block-wide barrier.  Slots are laid out as the shared ring's stages (16-byte
// chunks XOR-swizzled by row: conflict-free ldmatrix).  prime() issues the
// first kWS tiles and leaves the row at npos unwritten; fill_new() copies it
// from nrow (so prime() reads the cache only).
template <int D, int GP>
struct WarpKeys {
  static constexpr int RB = D * 2;
  static constexpr int VPR = RB / 16;                // 16-byte chunks per row
  static constexpr int TB = 16 * RB;                 // tile bytes
  static constexpr int kWS = kRing / (kWarps * TB);  // slots per warp: 2 (d = 128), 4 (d = 64)
  static constexpr int CPL = 16 * VPR / 32;          // chunks one lane copies per tile
  static constexpr int KS = D / 16;
  static constexpr int NT = (GP + 7) / 8;
  static_assert(kWS >= 2 && CPL >= 1, "per-warp slots");
  const __nv_bfloat16* kb;
  const __nv_bfloat16* nrow;
  int npos;
  const int* spos;
  int m, nt;
  unsigned char* slots;
  uint32_t bq[NT][KS][2];

  __device__ __forceinline__ WarpKeys(const __nv_bfloat16* kb_, const __nv_bfloat16* nrow_, int npos_,
                                      const int* spos_, int m_, unsigned char* ring)
      : kb(kb_), nrow(nrow_), npos(npos_), spos(spos_), m(m_) {
    const int warp = threadIdx.x >> 5;
    const int tiles = (m_ + 15) >> 4;
    nt = tiles > warp ? (tiles - warp + kWarps - 1) / kWarps : 0;
    slots = ring + warp * kWS * TB;
  }
  // this warp's tile tl (slice tile warp + tl kWarps) into slot tl % kWS
  __device__ __forceinline__ void issue(int tl, bool defer_new) {
    const int lane = threadIdx.x & 31;
    if (tl < nt) {
      const int r0 = ((threadIdx.x >> 5) + tl * kWarps) * 16;
      unsigned char* buf = slots + (tl % kWS) * TB;
#pragma unroll
      for (int j = 0; j < CPL; ++j) {
        const int x = lane + 32 * j, rr = x / VPR, c = x % VPR;
        const int i = r0 + rr;
        const int pos = i < m ? spos[i] : -1;
        const bool fresh = nrow && pos == npos;
        if (fresh && defer_new) continue;
        const __nv_bfloat16* src = fresh ? nrow + c * 8 : kb + (int64_t)(pos >= 0 ? pos : 0) * D + c * 8;
        cp_async16(smem_u32(buf + swz<RB>(rr, c)), src, pos >= 0);
      }
    }
    cp_async_commit();  // one group per call (possibly empty): constant wait depth
  }
  __device__ __forceinline__ void prime() {
#pragma unroll
    for (int tl = 0; tl < kWS; ++tl) issue(tl, true);
  }
  __device__ __forceinline__ void fill_new() {
    if (!nrow) return;
    const int lane = threadIdx.x & 31;
    for (int tl = 0; tl < kWS && tl < nt; ++tl) {
      const int r0 = ((threadIdx.x >> 5) + tl * kWarps) * 16;
      unsigned char* buf = slots + tl * TB;
#pragma unroll
      for (int j = 0; j < CPL; ++j) {
        const int x = lane + 32 * j, rr = x / VPR, c = x % VPR;
        const int i = r0 + rr;
        if (i < m && spos[i] == npos) *reinterpret_cast<uint4*>(buf + swz<RB>(rr, c)) = ld16(nrow + c * 8);
      }
    }
  }
  __device__ __forceinline__ void load_q(const __nv_bfloat16* q, int G) {
    const int lane = threadIdx.x & 31, g = lane >> 2, tig = lane & 3;
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      const int n = t * 8 + g;
#pragma unroll
      for (int s = 0; s < KS; ++s) {
        if (n < G) {
          const uint32_t* qr = reinterpret_cast<const uint32_t*>(q + (int64_t)n * D + s * 16);
          bq[t][s][0] = qr[tig];
          bq[t][s][1] = qr[4 + tig];
        } else {
          bq[t][s][0] = bq[t][s][1] = 0u;
        }
      }
    }
  }
  // dots[g * mc + i] = q_g . k_i for the warp's tiles (-inf at a bad position)
  __device__ __forceinline__ void run(int G, int mc, float* dots) {
    const int lane = threadIdx.x & 31, g = lane >> 2, tig = lane & 3;
    const int lrow = (lane & 7) + ((lane >> 3) & 1) * 8;
    for (int tl = 0; tl < nt; ++tl) {
      cp_async_wait<kWS - 1>();
      __syncwarp();
      const unsigned char* buf = slots + (tl % kWS) * TB;
      float acc[2][NT][4];
#pragma unroll
      for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int t = 0; t < NT; ++t) acc[u][t][0] = acc[u][t][1] = acc[u][t][2] = acc[u][t][3] = 0.0f;
#pragma unroll
      for (int s = 0; s < KS; ++s) {
        uint32_t a0, a1, a2, a3;
        ldmatrix_x4(smem_u32(buf + swz<RB>(lrow, 2 * s + (lane >> 4))), a0, a1, a2, a3);
#pragma unroll
        for (int t = 0; t < NT; ++t) mma_bf16(acc[s & 1][t], a0, a1, a2, a3, bq[t][s][0], bq[t][s][1]);
      }
      __syncwarp();  // the slot is read: refill it
      issue(tl + kWS, false);
      const int r0 = ((threadIdx.x >> 5) + tl * kWarps) * 16;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int i = r0 + g + 8 * half;
        if (i < m) {
          const bool ok = spos[i] >= 0;
#pragma unroll
          for (int t = 0; t < NT; ++t) {
            const int col = t * 8 + 2 * tig;
            const float v0 = acc[0][t][2 * half] + acc[1][t][2 * half];
            const float v1 = acc[0][t][2 * half + 1] + acc[1][t][2 * half + 1];
            if (col < G) dots[col * mc + i] = ok ? v0 : -INFINITY;
            if (col + 1 < G) dots[(col + 1) * mc + i] = ok ? v1 : -INFINITY;
          }
        }
      }
    }
    cp_async_wait<0>();
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
                                      int G, int mc, float* dots, float*) const {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int sub = lane / LPR, li = lane % LPR;
    const int h0 = GS::head0(li);
    for (int wb = warp * RPW; wb < nrows; wb += NG) {  // warp-uniform trip count
      const int r = wb + sub;
      const bool in = r < nrows;
      float f[E];
      Vec16<T>::unpack(in ? *reinterpret_cast<const uint4*>(buf + swz<D * (int)sizeof(T)>(r, li))
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
      if (in && GS::writer(li)) {
        const int i = r0 + r;
        const bool ok = spos[i] >= 0;
#pragma unroll
        for (int j = 0; j < GS::NH; ++j)
          if (h0 + j < G) dots[(h0 + j) * mc + i] = ok ? acc[j] : -INFINITY;
      }
    }
  }
};

// ---- phase 3: one radix digit from rank 0's histogram ----------------------

// hw: NB bins packed two per word (bin b: word b / 2, high half when b is
// odd).  Finds the bin holding the r-th largest counted key (bins rank in
// descending order) and returns (bin, keys above the bin, keys in the bin) in
// res[0..2].  Whole CTA.
template <int NB>
__device__ void find_digit(const uint32_t* hw, int r, int* scratch, int* res) {
  constexpr int PER = NB / kThreads;  // consecutive bins of this thread: 16 or 4
  constexpr int WPT = PER / 2;        // words: 8 or 2
  const int tid = threadIdx.x;
  uint32_t w[WPT];
  if constexpr (WPT == 8) {
    const uint4* p = reinterpret_cast<const uint4*>(hw) + tid * 2;
    const uint4 x = p[0], y = p[1];
    w[0] = x.x; w[1] = x.y; w[2] = x.z; w[3] = x.w;
    w[4] = y.x; w[5] = y.y; w[6] = y.z; w[7] = y.w;
  } else {
    const uint2 x = reinterpret_cast<const uint2*>(hw)[tid];
    w[0] = x.x; w[1] = x.y;
  }
  int v = 0;
#pragma unroll
  for (int j = 0; j < WPT; ++j) v += (int)(w[j] & 0xFFFFu) + (int)(w[j] >> 16);
  if (tid == 0) res[0] = res[1] = res[2] = 0;
  int total;
  const int excl = block_excl_scan(v, scratch, &total);
  int above = total - excl - v;
#pragma unroll
  for (int j = PER - 1; j >= 0; --j) {
    const int c = (int)((w[j >> 1] >> ((j & 1) * 16)) & 0xFFFFu);
    if (above < r && r <= above + c) {
      res[0] = tid * PER + j;
      res[1] = above;
      res[2] = c;
    }
    above += c;
  }
  __syncthreads();
}

// count one key into a packed histogram word of rank 0
__device__ __forceinline__ void hist_push(uint32_t* hw, uint32_t bin) {
  atomicAdd(hw + (bin >> 1), 1u << ((bin & 1u) << 4));
}


// Softmax mass: the cluster's per-head maximum (is_max) or sum of the CTAs'
// values v[GP]: the CTA reduces its threads' values, stores them into slot
// `rank` of every CTA's buf, and after one cluster barrier every thread
// combines the CL slots in rank order into v.  Whole cluster.
template <int GP>
__device__ __forceinline__ void mass_exchange(float (&v)[GP], bool is_max, float (&red)[kWarps][GP],
                                              float (&buf)[kMaxCluster][GP], cg::cluster_group& cluster,
                                              int CL, int rank) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int g = 0; g < GP; ++g) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float x = __shfl_xor_sync(0xffffffffu, v[g], o);
      v[g] = is_max ? fmaxf(v[g], x) : v[g] + x;
    }
    if (lane == 0) red[warp][g] = v[g];
  }
  __syncthreads();
  if (threadIdx.x < GP * CL) {
    const int g = threadIdx.x % GP, dst = threadIdx.x / GP;
    float t = red[0][g];
#pragma unroll
    for (int w = 1; w < kWarps; ++w) t = is_max ? fmaxf(t, red[w][g]) : t + red[w][g];
    cluster.map_shared_rank(&buf[0][0], dst)[rank * GP + g] = t;
  }
  cluster.sync();
#pragma unroll
  for (int g = 0; g < GP; ++g) {
    float t = buf[0][g];
    for (int c = 1; c < CL; ++c) t = is_max ? fmaxf(t, buf[c][g]) : t + buf[c][g];
    v[g] = t;
  }
  __syncthreads();  // red is free again
}

// the stage ring, which also holds the warps' value partials at the end
template <typename T, int D, int GP>
__host__ __device__ constexpr int ring_bytes() {
  return kRing > kWarps * GP * D * 4 ? kRing : kWarps * GP * D * 4;
}

// MASS: the softmax-mass selection (a separate instance, so that the other
// selections run none of its code).  INPL: the selected members' softmax
// weights replace their logits, with no weight array (fewer shared-memory
// bytes per member, for clusters with more members per CTA)
template <typename T, int D, int GP, bool MASS, bool INPL>
__global__ void __launch_bounds__(kThreads, 2) refine_decode_kernel(const RDArgs a) {
  constexpr int E = Vec16<T>::E;
  constexpr int LPR = D / E;     // lanes per cache row (value pass)
  constexpr int RPW = 32 / LPR;
  constexpr int NG = kThreads / LPR;
  constexpr int RB = D * (int)sizeof(T);
  constexpr int PART = GP * D + 2 * GP;  // one partial: o[GP][D], m[GP], l[GP]

  constexpr int RING = ring_bytes<T, D, GP>();
  extern __shared__ __align__(16) unsigned char dsm[];
  unsigned char* ring = dsm;                                          // RING bytes
  uint32_t* hist = reinterpret_cast<uint32_t*>(dsm + RING);           // [kHistWords] (rank 0)
  int* spos = reinterpret_cast<int*>(hist + kHistWords);              // [mc]
  uint32_t* keys = reinterpret_cast<uint32_t*>(spos + a.mc);          // [mc]
  float* dots = reinterpret_cast<float*>(keys + a.mc);                // [GP][mc]
  float* pw = INPL ? dots : dots + GP * a.mc;  // [mc][GP] softmax weights (unless INPL)
  int* sel = reinterpret_cast<int*>(dots + (INPL ? 1 : 2) * GP * a.mc);  // [mc]
  // partials of this CTA's outputs from every CTA: o [CL][per], (m, l) [CL][2 GP]
  float* recv = reinterpret_cast<float*>(sel + a.mc);

  __shared__ int scratch[33];
  __shared__ int s_dig[3];
  __shared__ int s_cnt[2];        // this CTA's keys above / at the threshold prefix
  __shared__ int s_mine[2];       // output offset, keys at the prefix taken
  __shared__ int s_slice;         // keys in this CTA's slice of the first-digit bins
  __shared__ int s_wa[kWarps], s_wb[kWarps];
  __shared__ float s_red[kWarps][GP];
  __shared__ float s_mm[kMaxCluster][GP];  // softmax mass: every CTA's per-head maxima
  __shared__ float s_zz[kMaxCluster][GP];  // and normalizer partials
  __shared__ __align__(16) float part[PART];  // this CTA's partial o, m, l

  cg::cluster_group cluster = cg::this_cluster();
  const int CL = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const int row = blockIdx.x / CL;
  const int b = row / a.Hkv, h = row - b * a.Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const unsigned lt = (1u << lane) - 1u;

  const int t0 = a.cu[b];
  const int L = a.cu[b + 1] - t0;
  int n = a.pool_cnt[row];
  if (n < 0 || n > a.kp) {
    if (rank == 0 && tid == 0) flag_status(a.status, PRISM_DEV_BAD_INDEX);
    n = n < 0 ? 0 : a.kp;
  }
  const int k = min(a.kappa, n);
  const bool all = n <= a.kappa;  // every member is taken: no selection
  const int chunk = ((n + CL - 1) / CL + 3) & ~3;  // slices start at multiples of 4 slots
  const int lo = min(n, rank * chunk);
  const int hi = min(n, lo + chunk);
  const int m = hi - lo;
  const int32_t* pool = a.pool + (int64_t)row * a.kp + lo;
  const int64_t rowbase = ((int64_t)h * a.T + t0) * D;
  const T* kb = static_cast<const T*>(a.k) + rowbase;
  const T* vb = static_cast<const T*>(a.v) + rowbase;
  const T* qrow = static_cast<const T*>(a.q) + ((int64_t)b * a.Hq + (int64_t)h * a.G) * D;
  uint32_t* h0 = cluster.map_shared_rank(hist, 0);  // the cluster's histograms
  // this token's rows: every read of position L - 1 takes them from k_new /
  // v_new, and rank 0 also writes them into the cache (for later calls)
  const T* knew = a.k_new && L > 0 ? static_cast<const T*>(a.k_new) + ((int64_t)b * a.Hkv + h) * D : nullptr;
  const T* vnew = a.v_new && L > 0 ? static_cast<const T*>(a.v_new) + ((int64_t)b * a.Hkv + h) * D : nullptr;

  // ---- 0. the slice's positions (an out-of-range one is flagged, skipped)
  for (int i = tid; i < m; i += kThreads) {
    const int p = pool[i];
    const bool ok = p >= 0 && p < L;
    if (!ok) flag_status(a.status, PRISM_DEV_BAD_INDEX);
    spos[i] = ok ? p : -1;
  }
  if (!all)  // this CTA's first-digit histogram; rank 0 also the cluster's later digits
    for (int i = tid; i < (rank == 0 ? kHistWords : kH2); i += kThreads) hist[i] = 0u;
  __syncthreads();
  cluster_arrive();  // rank 0's histograms are cleared once every CTA has arrived
  // bf16: every warp streams its own key tiles; fp32: the shared stage ring
  constexpr bool kWarpKeys = std::is_same<T, __nv_bfloat16>::value;
  RowStream<T, D> kst(kb, knew, L - 1, spos, nullptr, m, ring);
  WarpKeys<D, GP> wk(reinterpret_cast<const __nv_bfloat16*>(kb),
                     reinterpret_cast<const __nv_bfloat16*>(knew), L - 1, spos, m, ring);
  if constexpr (kWarpKeys) wk.prime();  // cache rows at pool positions only
  else kst.prime(true);

  // Up to here the kernel has read the pool and the key cache only, which
  // the previous kernel on the stream does not write when the launch
  // overlaps it; everything below may depend on that kernel.
  wait_previous_grid();
  allow_next_grid();
  if (rank == 0 && knew) {
    constexpr int VPR = RB / 16;
    if (tid < VPR) {
      reinterpret_cast<uint4*>(const_cast<T*>(kb) + (int64_t)(L - 1) * D)[tid] = ld16(knew + tid * (16 / (int)sizeof(T)));
    } else if (tid < 2 * VPR) {
      const int c = tid - VPR;
      reinterpret_cast<uint4*>(const_cast<T*>(vb) + (int64_t)(L - 1) * D)[c] = ld16(vnew + c * (16 / (int)sizeof(T)));
    }
  }
  if constexpr (kWarpKeys) wk.fill_new();
  else kst.fill_new();

  // ---- 1. exact logits of the slice
  if constexpr (kWarpKeys) {
    wk.load_q(reinterpret_cast<const __nv_bfloat16*>(qrow), a.G);
    wk.run(a.G, a.mc, dots);
  } else {
    ScoreSimt<T, D, GP> sc;
    sc.init(qrow, a.G);
    kst.run([&](int r0, const unsigned char* buf, int nrows) {
      sc.run(buf, r0, nrows, spos, a.G, a.mc, dots, pw);
    });
  }
  // the next layer's key rows at the same pool positions into L2, while
  // this layer selects and attends (the DRAM is otherwise idle meanwhile)
  if (a.k_next) {
    const T* kn = static_cast<const T*>(a.k_next) + rowbase;
    for (int i = tid; i < m; i += kThreads) {
      const int pos = spos[i];
      if (pos >= 0)
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;\n" ::"l"(kn + (int64_t)pos * D),
                     "r"(RB)
                     : "memory");
    }
  }
  __syncthreads();
  cluster_wait();

  // ---- 2. selection keys; their first digit into the cluster histogram
  const bool sum_group = a.agg == 1;  // the group's heads summed, not maxed
  if (MASS && !all) {
    // softmax mass: each head's maximum and normalizer over the row's pool,
    // through the cluster (every CTA's partials into every CTA), then the
    // key of a member is ord(sum_g 2^((l_g - M_g) c) / Z_g)
    float v[GP];
#pragma unroll
    for (int g = 0; g < GP; ++g) v[g] = -INFINITY;
    for (int i = tid; i < m; i += kThreads)
#pragma unroll
      for (int g = 0; g < GP; ++g)
        if (g < a.G) v[g] = fmaxf(v[g], dots[g * a.mc + i]);
    mass_exchange<GP>(v, true, s_red, s_mm, cluster, CL, rank);
    float z[GP];
#pragma unroll
    for (int g = 0; g < GP; ++g) z[g] = 0.0f;
    for (int i = tid; i < m; i += kThreads)
#pragma unroll
      for (int g = 0; g < GP; ++g)
        if (g < a.G && v[g] != -INFINITY) {
          const float l = dots[g * a.mc + i];
          if (l != -INFINITY) z[g] += exp2f((l - v[g]) * a.scale_log2);
        }
    mass_exchange<GP>(z, false, s_red, s_zz, cluster, CL, rank);
    for (int i = tid; i < m; i += kThreads) {
      float mass = 0.0f;
      bool any = false;
#pragma unroll
      for (int g = 0; g < GP; ++g) {
        if (g < a.G) {
          const float l = dots[g * a.mc + i];
          if (l != -INFINITY && z[g] > 0.0f) {
            mass += exp2f((l - v[g]) * a.scale_log2) / z[g];
            any = true;
          }
        }
      }
      keys[i] = ord_key(any ? mass : -INFINITY);
    }
    __syncthreads();
  }
  for (int i = tid; i < m; i += kThreads) {
    if (MASS && !all) {  // the key is the mass above
      hist_push(hist + kH1, keys[i] >> 20);
      continue;
    }
    float best = sum_group ? 0.0f : -INFINITY;
#pragma unroll
    for (int g = 0; g < GP; ++g) {
      if (g < a.G) {
        float v = dots[g * a.mc + i];
        best = sum_group ? best + v : fmaxf(best, v);
      }
    }
    const uint32_t key = ord_key(best);
    keys[i] = key;
    if (!all) hist_push(hist + kH1, key >> 20);  // this CTA's own histogram
  }

  // ---- 3. threshold prefix P: keys with (key >> shift) > P are taken, and
  // the first rtie keys with (key >> shift) == P in pool-slot order.  Rank 0
  // resolves each digit from its own histograms; the others read the answer.
  uint32_t P = 0u;
  int shift = 0, rtie = 0;
  if (!all) {
    int* dig0 = cluster.map_shared_rank(s_dig, 0);
    auto resolve = [&](const uint32_t* hw, int nb, int r) {
      cluster.sync();  // the level's histogram is complete
      if (rank == 0) {
        if (nb == kBins1) find_digit<kBins1>(hw, r, scratch, s_dig);
        else find_digit<kBins2>(hw, r, scratch, s_dig);
      }
      cluster.sync();  // rank 0's answer is ready
      if (rank != 0 && tid < 3) s_dig[tid] = dig0[tid];
      __syncthreads();
    };
    // Without remote atomics: every CTA holds a packed histogram hl of nb
    // bins; CTA c sums slice c of all of them into its ring, with the slice
    // total; then every CTA finds, from the slice totals and the right
    // slice, the bin holding the r-th largest key (s_dig = bin, keys above
    // it, keys in it).  Two cluster barriers; the first orders the hl writes.
    auto cluster_digit = [&](const uint32_t* hl, int nb, int r, uint32_t* sw) {
      const int WS = (nb / 2) / CL;  // packed words per slice
      __syncthreads();
      cluster.sync();  // every CTA's histogram is complete
      int part = 0;
      for (int x = tid; x < WS; x += kThreads) {
        uint32_t v[kMaxCluster];  // every CTA's word, all loads in flight at once
#pragma unroll
        for (int c = 0; c < kMaxCluster; ++c)
          v[c] = c < CL ? cluster.map_shared_rank(hl, c)[rank * WS + x] : 0u;
        uint32_t acc = 0u;  // 16-bit halves: a bin never holds more than kappa_p keys
#pragma unroll
        for (int c = 0; c < kMaxCluster; ++c) acc += v[c];
        sw[x] = acc;
        part += (int)(acc & 0xFFFFu) + (int)(acc >> 16);
      }
      int tot;
      block_excl_scan(part, scratch, &tot);
      if (tid == 0) s_slice = tot;
      cluster.sync();  // every slice and its total are ready
      if (warp == 0) {
        const int t = lane < CL ? *cluster.map_shared_rank(&s_slice, lane) : 0;
        // slices rank in descending bin order: count above slice `lane`
        const int incl = warp_incl_scan(t);
        const int total = __shfl_sync(0xffffffffu, incl, 31);
        const int above = total - incl;
        const unsigned hit = __ballot_sync(0xffffffffu, lane < CL && above < r && r <= above + t);
        const int src = hit ? __ffs(hit) - 1 : 0;  // always exactly one lane when counts are right
        const int above_src = __shfl_sync(0xffffffffu, above, src);
        if (lane == 0) {
          s_dig[0] = src;
          s_dig[1] = above_src;
        }
      }
      __syncthreads();
      const int src = s_dig[0], above_s = s_dig[1];
      const uint32_t* swr = cluster.map_shared_rank(sw, src);
      const int sb = 2 * WS;  // bins in the slice
      const int per = (sb + kThreads - 1) / kThreads;
      uint32_t cnt[8];
      int v = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int bin = tid * per + j;
        cnt[j] = 0u;
        if (j < per && bin < sb) cnt[j] = (swr[bin >> 1] >> ((bin & 1) * 16)) & 0xFFFFu;
        v += (int)cnt[j];
      }
      int total2;
      const int excl = block_excl_scan(v, scratch, &total2);
      int above = above_s + total2 - excl - v;
      __syncthreads();
#pragma unroll
      for (int j = 7; j >= 0; --j) {
        const int c = (int)cnt[j];
        if (j < per && above < r && r <= above + c) {
          s_dig[0] = src * sb + tid * per + j;
          s_dig[1] = above;
          s_dig[2] = c;
        }
        above += c;
      }
      __syncthreads();
    };
    int r = k;
    // the summed slices go to the ring: the later cluster barriers keep it
    // intact while the peers read it
    if (CL == 1) resolve(hist + kH1, kBins1, r);
    else cluster_digit(hist + kH1, kBins1, r, reinterpret_cast<uint32_t*>(ring));
    P = (uint32_t)s_dig[0];
    shift = 20;
    r -= s_dig[1];
    if (r < s_dig[2]) {  // part of the bin: the second digit of its (few) keys, in rank 0
      for (int i = tid; i < m; i += kThreads) {
        const uint32_t key = keys[i];
        if ((key >> 20) == P) hist_push(h0 + kH2, (key >> 10) & 1023u);
      }
      resolve(hist + kH2, kBins2, r);
      P = (P << 10) | (uint32_t)s_dig[0];
      shift = 10;
      r -= s_dig[1];
      if (r < s_dig[2]) {  // the last digit
        for (int i = tid; i < m; i += kThreads) {
          const uint32_t key = keys[i];
          if ((key >> 10) == P) hist_push(h0 + kH3, key & 1023u);
        }
        resolve(hist + kH3, kBins2, r);
        P = (P << 10) | (uint32_t)s_dig[0];
        shift = 0;
        r -= s_dig[1];
      }
    }
    rtie = r;
    // this CTA's counts above and at P, then every CTA's, in rank order
    int gt = 0, eq = 0;
    for (int i = tid; i < m; i += kThreads) {
      const uint32_t pre = keys[i] >> shift;
      gt += pre > P;
      eq += pre == P;
    }
    int tot;
    block_excl_scan((gt << 16) | eq, scratch, &tot);  // both counts <= 65535
    if (tid == 0) {
      s_cnt[0] = tot >> 16;
      s_cnt[1] = tot & 0xFFFF;
    }
    cluster.sync();  // S4: every CTA's counts are published
    if (warp == 0) {
      int g_s = 0, e_s = 0;
      if (lane < CL) {
        const int* rc = cluster.map_shared_rank(s_cnt, lane);
        g_s = rc[0];
        e_s = rc[1];
      }
      const int ebefore = warp_incl_scan(e_s) - e_s;
      const int take = min(max(rtie - ebefore, 0), e_s);
      const int nsel_s = g_s + take;
      const int before = warp_incl_scan(nsel_s) - nsel_s;
      if (lane == rank) {
        s_mine[0] = before;
        s_mine[1] = take;
      }
    }
    __syncthreads();
  }

  // ---- 4. selected members of the slice, positions to idx (ascending).
  // Warp w owns members [w pw, (w + 1) pw) in slot order; three ballot passes
  // (keys at P per warp, selected per warp, placement) with two block barriers.
  int nsel = 0;
  {
    const int off = all ? lo : s_mine[0];
    const int take = all ? 0 : s_mine[1];
    int32_t* idx = a.idx + (int64_t)row * a.kappa;
    const int pw = ((m + kWarps - 1) / kWarps + 31) & ~31;
    const int w0 = warp * pw;
    auto flags = [&](int i, bool& gt, bool& eq) {
      gt = eq = false;
      if (i < m) {
        if (all) {
          gt = true;
        } else {
          const uint32_t pre = keys[i] >> shift;
          gt = pre > P;
          eq = pre == P;
        }
      }
    };
    int ecount = 0;
    for (int c = 0; c < pw; c += 32) {
      bool gt, eq;
      flags(w0 + c + lane, gt, eq);
      ecount += __popc(__ballot_sync(0xffffffffu, eq));
    }
    if (lane == 0) s_wa[warp] = ecount;
    __syncthreads();
    int ebase = 0;
    for (int w = 0; w < warp; ++w) ebase += s_wa[w];
    int scount = 0;  // a key at P is taken while its rank among the keys at P is below take
    for (int c = 0, er = ebase; c < pw; c += 32) {
      bool gt, eq;
      flags(w0 + c + lane, gt, eq);
      const unsigned eb = __ballot_sync(0xffffffffu, eq);
      scount += __popc(__ballot_sync(0xffffffffu, gt || (eq && er + __popc(eb & lt) < take)));
      er += __popc(eb);
    }
    if (lane == 0) s_wb[warp] = scount;
    __syncthreads();
    int base = 0, o = 0;
    for (int w = 0; w < kWarps; ++w) {
      if (w < warp) o += s_wb[w];
      base += s_wb[w];
    }
    for (int c = 0, er = ebase; c < pw; c += 32) {
      const int i = w0 + c + lane;
      bool gt, eq;
      flags(i, gt, eq);
      const unsigned eb = __ballot_sync(0xffffffffu, eq);
      const bool sl = gt || (eq && er + __popc(eb & lt) < take);
      const unsigned bal = __ballot_sync(0xffffffffu, sl);
      if (sl) {
        const int oo = o + __popc(bal & lt);
        const int slot = off + oo;
        if (slot < k) idx[slot] = spos[i];
        else flag_status(a.status, PRISM_DEV_TOO_LONG);  // unreachable if counts are right
        sel[oo] = i;
      }
      o += __popc(bal);
      er += __popc(eb);
    }
    nsel = min(base, m);
    for (int s = k + rank * kThreads + tid; s < a.kappa; s += CL * kThreads) idx[s] = -1;
    if (rank == 0 && tid == 0) a.cnt[row] = k;
    __syncthreads();  // sel is complete
  }

  // ---- 5. softmax partial over the selected members of the slice.  The
  // value rows are requested first (the ring is free: no peer reads it after
  // the selection's last cluster barrier), so their latency overlaps the
  // softmax statistics
  RowStream<T, D> vst(vb, vnew, L - 1, spos, sel, nsel, ring);
  vst.prime(false);
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
      if constexpr (INPL) {
        if (g < a.G) dots[g * a.mc + i] = p;  // the member's weight, in place of its logit
      } else {
        pw[j * GP + g] = p;
      }
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
  // stream the selected value rows (the weights are read after the first
  // stage barrier of the stream)
  vst.run([&](int j0, const unsigned char* buf, int nrows) {
        for (int r = warp * RPW + sub; r < nrows; r += NG) {
          float f[E];
          Vec16<T>::unpack(*reinterpret_cast<const uint4*>(buf + swz<RB>(r, li)), f);
          const float* p = INPL ? dots + sel[j0 + r] : pw + (j0 + r) * GP;
#pragma unroll
          for (int g = 0; g < GP; ++g) {
            const float pg = INPL ? (g < a.G ? p[g * a.mc] : 0.0f) : p[g];
#pragma unroll
            for (int e = 0; e < E; ++e) o[g][e] = fmaf(pg, f[e], o[g][e]);
          }
        }
      });
  // lane groups of a warp hold the same feature slice: add them, then warps
#pragma unroll
  for (int g = 0; g < GP; ++g)
#pragma unroll
    for (int s = LPR; s < 32; s <<= 1)
#pragma unroll
      for (int e = 0; e < E; ++e) o[g][e] += __shfl_xor_sync(0xffffffffu, o[g][e], s);
  __syncthreads();  // the ring is free (value rows consumed): warp partials go there
  {
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
      part[i] = acc;
    }
    if (tid < GP) {
      float s = 0.0f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) s += s_red[w][tid];
      float mv = -INFINITY;
#pragma unroll
      for (int g = 0; g < GP; ++g)
        if (g == tid) mv = mx[g];
      part[GP * D + tid] = mv;
      part[GP * D + GP + tid] = s;
    }
    __syncthreads();
  }
  // ---- 6. CTA r owns outputs [r * per, (r + 1) * per) of the G x d: every
  // CTA stores the matching slice of its partial, and its (m, l), into the
  // owner (remote stores), then the owners combine them by log-sum-exp
  const int nout = a.G * D;
  const int per = (nout + CL - 1) / CL;
  float* recv_ml = recv + CL * per;
  for (int i = tid; i < nout; i += kThreads) {
    const int dst = i / per;
    float* r = cluster.map_shared_rank(recv, dst);
    r[rank * per + (i - dst * per)] = part[i];
  }
  for (int i = tid; i < CL * 2 * GP; i += kThreads) {
    const int dst = i / (2 * GP), j = i - dst * 2 * GP;
    float* r = cluster.map_shared_rank(recv_ml, dst);
    r[rank * 2 * GP + j] = part[GP * D + j];
  }
  cluster.sync();  // S5: every partial slice is with its owner
  {
    const int o_lo = rank * per, o_hi = min(nout, o_lo + per);
    for (int oi = o_lo + tid; oi < o_hi; oi += kThreads) {
      const int g = oi / D, j = oi - g * D;
      // every source's (m, l, o) loaded at once (sources past CL count as empty)
      float mv[kMaxCluster], lv[kMaxCluster], ov[kMaxCluster];
#pragma unroll
      for (int src = 0; src < kMaxCluster; ++src) {
        const bool in = src < CL;
        mv[src] = in ? recv_ml[src * 2 * GP + g] : -INFINITY;
        lv[src] = in ? recv_ml[src * 2 * GP + GP + g] : 0.0f;
        ov[src] = in ? recv[src * per + (oi - o_lo)] : 0.0f;
      }
      float M = -INFINITY;
#pragma unroll
      for (int src = 0; src < kMaxCluster; ++src) M = fmaxf(M, mv[src]);
      float Ls = 0.0f, O = 0.0f;
      if (M != -INFINITY) {
#pragma unroll
        for (int src = 0; src < kMaxCluster; ++src) {
          if (mv[src] == -INFINITY) continue;
          const float wt = exp2f(mv[src] - M);
          Ls = fmaf(wt, lv[src], Ls);
          O = fmaf(wt, ov[src], O);
        }
      }
      const int64_t hq = (int64_t)b * a.Hq + (int64_t)h * a.G + g;
      a.out[hq * D + j] = Ls > 0.0f ? O / Ls : 0.0f;
      if (j == 0 && a.lse)
        a.lse[hq] = Ls > 0.0f ? (M + log2f(Ls)) * 0.69314718055994530942f : -INFINITY;
    }
  }
  // every access to this CTA's shared memory by another CTA came before S5
}

// spos, sel, keys, dots and (unless in place) the weights
inline int per_member_bytes(int GP, bool inplace) {
  return (int)(2 * sizeof(int) + sizeof(uint32_t) + (inplace ? 1 : 2) * GP * sizeof(float));
}
// stage ring (at least the warps' value partials) and rank 0's histograms
int fixed_bytes(int D, int GP) {
  const int comb = kWarps * GP * D * 4;
  return (kRing > comb ? kRing : comb) + kHistWords * 4;
}
// the owners' receive buffers: CL * ceil(G d / CL) + CL * 2 GP floats
constexpr int recv_bytes(int GP, int D) { return (GP * D + kMaxCluster + 2 * GP * kMaxCluster) * 4; }

// dynamic shared memory one CTA may use; two CTAs share an SM when each
// stays under kPairBudget
constexpr int kDynBudget = 227 * 1024 - 8 * 1024;
constexpr int kPairBudget = 110 * 1024;

template <typename T, int D, int GP>
cudaError_t run(const Dims& d, RDArgs a, int cl, bool inplace, bool overlap, cudaStream_t st) {
  auto kern = a.agg == 2 ? (inplace ? refine_decode_kernel<T, D, GP, true, true>
                                    : refine_decode_kernel<T, D, GP, true, false>)
                         : (inplace ? refine_decode_kernel<T, D, GP, false, true>
                                    : refine_decode_kernel<T, D, GP, false, false>);
  const int smem = ring_bytes<T, D, GP>() + kHistWords * 4 + a.mc * per_member_bytes(GP, inplace) +
                   recv_bytes(GP, D);
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
  cudaLaunchAttribute attr[3];
  int na = 0;
  attr[na].id = cudaLaunchAttributeClusterDimension;
  attr[na].val.clusterDim.x = (unsigned)cl;
  attr[na].val.clusterDim.y = 1;
  attr[na].val.clusterDim.z = 1;
  ++na;
  // a grid of at most one CTA per SM: let the hardware balance each
  // cluster's CTAs over the SMs (measured at c128k: 21.4 against 21.7 us per
  // chained layer; grids of several waves do not gain)
  if ((int64_t)d.B * d.Hkv * cl <= d.num_sms) {
    attr[na].id = cudaLaunchAttributeClusterSchedulingPolicyPreference;
    attr[na].val.clusterSchedulingPolicyPreference = cudaClusterSchedulingPolicyLoadBalancing;
    ++na;
  }
  if (overlap) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

template <typename T, int D>
cudaError_t by_group(const Dims& d, const RDArgs& a, int cl, bool inpl, bool ov, cudaStream_t st) {
  switch (padded_group(d.G)) {
    case 1: return run<T, D, 1>(d, a, cl, inpl, ov, st);
    case 2: return run<T, D, 2>(d, a, cl, inpl, ov, st);
    case 4: return run<T, D, 4>(d, a, cl, inpl, ov, st);
    case 8: return run<T, D, 8>(d, a, cl, inpl, ov, st);
    default: return run<T, D, 16>(d, a, cl, inpl, ov, st);
  }
}

}  // namespace

RefineDecodePlan plan_refine_decode(const Dims& d, int kappa_p) {
  const int rows = d.B * d.Hkv;
  const int GP = padded_group(d.G);
  auto mc_of = [&](int c) { return ((kappa_p + c - 1) / c + 3) & ~3; };
  auto need = [&](int c, bool inpl) {
    return fixed_bytes(d.D, GP) + mc_of(c) * per_member_bytes(GP, inpl) + recv_bytes(GP, d.D);
  };
  // The largest cluster whose grid still fits one wave of two CTAs per SM:
  // with more rows, smaller clusters and more pool members per CTA (16-CTA
  // clusters need their SMs in one GPC, and few are resident at once).  Then
  // small enough for two CTAs per SM: with a separate weight array if that
  // fits, else with the weights in place of the logits, else a larger cluster.
  int cl = 1;
  while (cl < kMaxCluster && (int64_t)rows * cl * 2 <= 2LL * d.num_sms) cl *= 2;
  bool inpl = false;
  for (;;) {
    if (need(cl, false) <= kPairBudget) {
      inpl = false;
      break;
    }
    if (need(cl, true) <= kPairBudget) {
      inpl = true;
      break;
    }
    if (cl >= kMaxCluster) {
      inpl = need(cl, false) > kDynBudget;
      break;
    }
    cl *= 2;
  }
  const bool ok = kappa_p <= kMaxCount && need(cl, inpl) <= kDynBudget;
  return RefineDecodePlan{cl, mc_of(cl), ok, inpl};
}

cudaError_t launch_refine_decode(const Dims& d, const RefineDecodePlan& p, const void* q,
                                 const void* k, const void* v, const void* k_new,
                                 const void* v_new, const void* k_next, const int32_t* pool,
                                 const int32_t* pool_cnt, int kappa_p, int kappa,
                                 float softmax_scale, int32_t* idx, int32_t* cnt, float* out,
                                 float* lse, int32_t* status, bool overlap, int agg,
                                 cudaStream_t st) {
  if (d.B * d.Hkv == 0) return cudaSuccess;
  RDArgs a{q, k, v, k_next, k_new, v_new, d.cu_dev, pool, pool_cnt, kappa_p, kappa, d.Hkv, d.G, d.Hq, d.T, p.mc,
           softmax_scale * 1.4426950408889634f, idx, cnt, out, lse, status, agg};
  if (d.bf16)
    return d.D == 128 ? by_group<__nv_bfloat16, 128>(d, a, p.cluster, p.inplace, overlap, st)
                      : by_group<__nv_bfloat16, 64>(d, a, p.cluster, p.inplace, overlap, st);
  return d.D == 128 ? by_group<float, 128>(d, a, p.cluster, p.inplace, overlap, st)
                    : by_group<float, 64>(d, a, p.cluster, p.inplace, overlap, st);
}

}  // namespace prism
