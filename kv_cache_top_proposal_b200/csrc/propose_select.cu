// Candidate pool of a proposal layer: the top kappa_p positions of every
// (sequence, KV head) row by proposal score, "lower index wins" on ties,
// written in ascending position order (Prism Attention, sec. 4.1
// "Proposal-Refined Index Sharing"; pool size n = rho * kappa, sec. 5.1
// "Implementation Details").
//
// The scorer has already built, per row, the histogram of the first 12 bits
// of ord(score).  One cluster of kCL CTAs per row; CTA r owns the contiguous
// slice r of positions and keeps its keys in registers (KPT per thread,
// coalesced: key u of thread t is slice position u * kThreads + t):
//   1. every CTA reads the row's histogram and locates the bin holding the
//      kappa_p-th largest key (same answer in every CTA).  Each CTA hands
//      rank 0 its keys in that bin, in position order, with its count above
//      the bin; rank 0 ranks these candidates exactly (two more 10-bit
//      digits over its own histograms) and returns the threshold key T,
//      each CTA's output offset and its share of the keys equal to T ("lower
//      index wins").  If a CTA has more candidates than rank 0 holds, the
//      digits are resolved over the cluster instead, one barrier per digit;
//   2. every CTA writes its kept positions in ascending order (ballot counts
//      per (key block, warp), one block scan, placement).
#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.h"

namespace cg = cooperative_groups;

namespace prism {

namespace {

constexpr int kCL = 16;                       // CTAs per row (a non-portable cluster size)
constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kKPT = 16;                      // keys per thread
constexpr int kMaxSlice = kKPT * kThreads;    // keys per CTA
constexpr int kHist = 4096;                   // first digit (from the scorer)
constexpr int kBins = 1024;                   // second and third digits
constexpr int kCandCap = 512;                 // first-digit candidates per CTA ranked by rank 0

struct PSArgs {
  const float* scores;   // [Hkv][T]
  const uint32_t* hist;  // [rows][kHist]
  const int32_t* cu;
  int Hkv;
  int64_t T;
  int kp;
  int32_t* out;          // [rows][kp]
  int32_t* out_cnt;      // [rows]
  int32_t* status;
};

__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;\n" ::: "memory");
}

// Bin of an NB-bin histogram (PER consecutive bins per thread, read through
// load(bin)) holding the r-th largest counted key, bins ranked in descending
// order: res = (bin, keys above it, keys in it).  Whole CTA.
template <int PER, typename Load>
__device__ void find_digit(Load load, int r, int* scratch, int* res) {
  const int tid = threadIdx.x;
  uint32_t c[PER];
  int v = 0;
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    c[j] = load(tid * PER + j);
    v += (int)c[j];
  }
  if (tid == 0) res[0] = res[1] = res[2] = 0;
  int total;
  const int excl = block_excl_scan(v, scratch, &total);
  int above = total - excl - v;
#pragma unroll
  for (int j = PER - 1; j >= 0; --j) {
    if (above < r && r <= above + (int)c[j]) {
      res[0] = tid * PER + j;
      res[1] = above;
      res[2] = (int)c[j];
    }
    above += (int)c[j];
  }
  __syncthreads();
}

// Exclusive scan, in place, of the kKPT * kWarps per-(block, warp) counts
// (one entry per thread for the first kKPT * kWarps threads), plus `base`.
__device__ __forceinline__ void scan_table(int* tab, int base, int* scratch) {
  const int tid = threadIdx.x;
  const int v = tid < kKPT * kWarps ? tab[tid] : 0;
  int total;
  const int excl = block_excl_scan(v, scratch, &total);
  if (tid < kKPT * kWarps) tab[tid] = excl + base;
  __syncthreads();
}

// Rank 0: the candidates are every CTA's keys of first-digit bin b1, CTA w's
// in cand[w * kCandCap ..] in position order, cnt[3w] of them, with
// cnt[3w + 1] of its keys above the bin.  Finds the r-th largest candidate T
// (two 10-bit digits over local histograms) and writes fin = {0, T, then per
// CTA (output offset, keys equal to T it takes, keys equal to T it holds)}:
// keys equal to T are taken in CTA order, then position order.  fin[0] = 1
// (nothing else written) when a CTA had more than kCandCap candidates.
// Whole CTA.
__device__ void rank_candidates(const uint2* cand, uint32_t b1, int r, uint32_t* h2, uint32_t* h3,
                                int* scratch, int* dig, const int* cnt, int* fin) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  __shared__ int s_over;
  __shared__ int s_ge[kCL][2];
  if (tid == 0) s_over = 0;
  __syncthreads();
  if (tid < kCL && cnt[3 * tid] > kCandCap) s_over = 1;
  __syncthreads();
  if (s_over) {
    if (tid == 0) fin[0] = 1;
    __syncthreads();
    return;
  }
  constexpr int WPR = kWarps / kCL;  // warps per CTA region
  const int w = warp / WPR, sub = warp % WPR;
  const int nw = cnt[3 * w];
  const uint2* cw = cand + w * kCandCap;
  for (int j = sub * 32 + lane; j < nw; j += WPR * 32) atomicAdd(h2 + ((cw[j].x >> 10) & (kBins - 1)), 1u);
  __syncthreads();
  find_digit<kBins / kThreads>([&](int bin) { return h2[bin]; }, r, scratch, dig);
  const uint32_t p2 = (b1 << 10) | (uint32_t)dig[0];
  r -= dig[1];
  for (int j = sub * 32 + lane; j < nw; j += WPR * 32) {
    const uint32_t key = cw[j].x;
    if ((key >> 10) == p2) atomicAdd(h3 + (key & (kBins - 1)), 1u);
  }
  __syncthreads();
  find_digit<kBins / kThreads>([&](int bin) { return h3[bin]; }, r, scratch, dig);
  const uint32_t T = (p2 << 10) | (uint32_t)dig[0];
  r -= dig[1];  // keys equal to T to take, in order
  if (tid < kCL * 2) (&s_ge[0][0])[tid] = 0;
  __syncthreads();
  {
    int gt = 0, eq = 0;
    for (int j = sub * 32 + lane; j < nw; j += WPR * 32) {
      const uint32_t key = cw[j].x;
      gt += key > T;
      eq += key == T;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      gt += __shfl_xor_sync(0xffffffffu, gt, o);
      eq += __shfl_xor_sync(0xffffffffu, eq, o);
    }
    if (lane == 0) {
      atomicAdd(&s_ge[w][0], gt);
      atomicAdd(&s_ge[w][1], eq);
    }
  }
  __syncthreads();
  if (warp == 0) {
    const int gt = lane < kCL ? cnt[3 * lane + 1] + s_ge[lane][0] : 0;
    const int eq = lane < kCL ? s_ge[lane][1] : 0;
    const int ebefore = warp_incl_scan(eq) - eq;
    const int take = min(max(r - ebefore, 0), eq);
    const int nsel = gt + take;
    const int before = warp_incl_scan(nsel) - nsel;
    if (lane < kCL) {
      fin[2 + 3 * lane] = before;
      fin[3 + 3 * lane] = take;
      fin[4 + 3 * lane] = eq;
    }
    if (lane == 0) {
      fin[0] = 0;
      fin[1] = (int)T;
    }
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kThreads, 2) propose_select_kernel(const PSArgs a) {
  extern __shared__ __align__(16) uint2 cand[];      // rank 0: [kCL][kCandCap] (key, position)
  __shared__ __align__(16) uint32_t hist2[kBins];  // rank 0: digit-2 counts
  __shared__ __align__(16) uint32_t hist3[kBins];  // rank 0: digit-3 counts
  __shared__ int tabE[kKPT * kWarps];  // per (key block, warp): keys at P, then their prefix
  __shared__ int tabK[kKPT * kWarps];  // per (key block, warp): kept keys, then output slots
  __shared__ int scratch[33];
  __shared__ int s_dig[3];
  __shared__ int s_cnt[3 * kCL];    // rank 0: per CTA, candidates, keys above, (spare)
  __shared__ int s_fin[2 + 3 * kCL];  // rank 0: mode, T, per CTA (offset, share, at T)
  __shared__ int s_mine[3];  // output offset, keys at the prefix taken, keys at the prefix

  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int row = blockIdx.x / kCL;
  const int b = row / a.Hkv, h = row - b * a.Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const unsigned lt = (1u << lane) - 1u;
  const int t0 = a.cu[b];
  const int n = a.cu[b + 1] - t0;
  const int chunk = (n + kCL - 1) / kCL;
  const int lo = min(n, rank * chunk), hi = min(n, lo + chunk);
  const int m = hi - lo;
  int32_t* out = a.out + (int64_t)row * a.kp;

  // every branch depends on cluster-wide values only
  if (n <= a.kp || chunk > kMaxSlice) {
    const bool all = n <= a.kp;
    if (all) {
      for (int i = lo + tid; i < hi; i += kThreads) out[i] = i;
    } else if (rank == 0 && tid == 0) {
      flag_status(a.status, PRISM_DEV_TOO_LONG);
    }
    const int filled = all ? n : 0;
    for (int i = filled + rank * kThreads + tid; i < a.kp; i += kCL * kThreads) out[i] = -1;
    if (rank == 0 && tid == 0) a.out_cnt[row] = filled;
    return;
  }
  const int k = a.kp;
  uint32_t* h2 = cluster.map_shared_rank(hist2, 0);
  uint32_t* h3 = cluster.map_shared_rank(hist3, 0);
  if (rank == 0) {
    for (int i = tid; i < kBins; i += kThreads) {
      hist2[i] = 0u;
      hist3[i] = 0u;
    }
  }
  __syncthreads();
  cluster_arrive();  // rank 0's histograms are cleared once every CTA has arrived

  // ---- the slice's keys, kKPT loads in flight per thread
  uint32_t key[kKPT];
  {
    const float* kb = a.scores + (int64_t)h * a.T + t0 + lo;
    float v[kKPT];
#pragma unroll
    for (int u = 0; u < kKPT; ++u) {
      const int i = u * kThreads + tid;
      v[u] = i < m ? __ldcg(kb + i) : 0.0f;
    }
#pragma unroll
    for (int u = 0; u < kKPT; ++u) key[u] = ord_key(v[u]);
  }
  auto in = [&](int u) { return u * kThreads + tid < m; };

  // ---- 1. threshold: keys with (key >> shift) > P are taken, and the first
  // rtie keys with (key >> shift) == P in position order.  Every CTA finds
  // the first digit's bin b1 from the row's histogram.  Each CTA hands rank 0
  // its keys in b1 (in position order) and its count above b1; rank 0 ranks
  // the candidates exactly and returns the threshold T with every CTA's
  // offset and share of the keys equal to T (then P = T, shift = 0).  When a
  // CTA has more than kCandCap candidates, the last two digits are resolved
  // over the whole cluster instead (remote histograms, one digit per round).
  const uint32_t* gh = a.hist + (int64_t)row * kHist;
  find_digit<kHist / kThreads>([&](int bin) { return __ldcg(gh + bin); }, k, scratch, s_dig);
  const uint32_t b1 = (uint32_t)s_dig[0];
  const int c1 = s_dig[2];
  int r = k - s_dig[1];
  cluster_wait();
  {
    // candidates in position order: counts per (key block, warp), one scan
    int gt1 = 0;
#pragma unroll
    for (int u = 0; u < kKPT; ++u) {
      const bool c = in(u) && (key[u] >> 20) == b1;
      gt1 += in(u) && (key[u] >> 20) > b1;
      const unsigned bal = __ballot_sync(0xffffffffu, c);
      if (lane == 0) tabE[u * kWarps + warp] = __popc(bal);
    }
    __syncthreads();
    const int v = tid < kKPT * kWarps ? tabE[tid] : 0;
    int ncand;
    const int excl = block_excl_scan(v, scratch, &ncand);
    if (tid < kKPT * kWarps) tabE[tid] = excl;
    int gtot;
    block_excl_scan(gt1, scratch, &gtot);  // (also orders the table writes)
    uint2* region = cluster.map_shared_rank(cand, 0) + rank * kCandCap;
#pragma unroll
    for (int u = 0; u < kKPT; ++u) {
      const bool c = in(u) && (key[u] >> 20) == b1;
      const unsigned bal = __ballot_sync(0xffffffffu, c);
      if (c) {
        const int o = tabE[u * kWarps + warp] + __popc(bal & lt);
        if (o < kCandCap) region[o] = make_uint2(key[u], (uint32_t)(lo + u * kThreads + tid));
      }
    }
    if (tid == 0) {
      int* cm = cluster.map_shared_rank(s_cnt, 0);
      cm[3 * rank] = ncand;
      cm[3 * rank + 1] = gtot;
    }
  }
  cluster.sync();  // S1: every slice's candidates and count are with rank 0
  if (rank == 0) rank_candidates(cand, b1, r, hist2, hist3, scratch, s_dig, s_cnt, s_fin);
  cluster.sync();  // S2: rank 0's answer is ready
  uint32_t P;
  int shift;
  {
    if (tid < 5) {
      const int* f = cluster.map_shared_rank(s_fin, 0);
      const int v = tid == 0 ? f[0] : tid == 1 ? f[1] : f[tid + 3 * rank];
      if (tid < 2) s_dig[tid] = v;
      else s_mine[tid - 2] = v;
    }
    __syncthreads();
  }
  const bool ranked = s_dig[0] == 0;
  if (ranked) {
    P = (uint32_t)s_dig[1];
    shift = 0;
  } else {
    P = b1;
    shift = 20;
    __syncthreads();  // s_dig is rewritten below
    if (r < c1) {  // part of the bin: the second digit of its keys
#pragma unroll
      for (int u = 0; u < kKPT; ++u)
        if (in(u) && (key[u] >> 20) == P) atomicAdd(h2 + ((key[u] >> 10) & (kBins - 1)), 1u);
      cluster.sync();
      find_digit<kBins / kThreads>([&](int bin) { return h2[bin]; }, r, scratch, s_dig);
      P = (P << 10) | (uint32_t)s_dig[0];
      shift = 10;
      r -= s_dig[1];
      if (r < s_dig[2]) {  // the last digit
#pragma unroll
        for (int u = 0; u < kKPT; ++u)
          if (in(u) && (key[u] >> 10) == P) atomicAdd(h3 + (key[u] & (kBins - 1)), 1u);
        cluster.sync();
        find_digit<kBins / kThreads>([&](int bin) { return h3[bin]; }, r, scratch, s_dig);
        P = (P << 10) | (uint32_t)s_dig[0];
        shift = 0;
        r -= s_dig[1];
      }
    }
    const int rtie = r;
    // counts above / at P, then every CTA's, in rank order
    int gt = 0, eq = 0;
#pragma unroll
    for (int u = 0; u < kKPT; ++u) {
      if (in(u)) {
        const uint32_t pre = key[u] >> shift;
        gt += pre > P;
        eq += pre == P;
      }
    }
    int tot;
    block_excl_scan((gt << 16) | eq, scratch, &tot);  // both counts <= kMaxSlice < 65536
    if (tid == 0) {
      s_cnt[0] = tot >> 16;
      s_cnt[1] = tot & 0xFFFF;
    }
    cluster.sync();  // every CTA's counts are published
    if (warp == 0) {
      int g_s = 0, e_s = 0;
      if (lane < kCL) {
        const int* rc = cluster.map_shared_rank(s_cnt, lane);
        g_s = rc[0];
        e_s = rc[1];
      }
      const int ebefore = warp_incl_scan(e_s) - e_s;
      const int take = min(max(rtie - ebefore, 0), e_s);
      const int nsel = g_s + take;
      const int before = warp_incl_scan(nsel) - nsel;
      if (lane == rank) {
        s_mine[0] = before;
        s_mine[1] = take;
        s_mine[2] = e_s;
      }
    }
    __syncthreads();
  }
  const int off = s_mine[0], take = s_mine[1];
  const bool part = take < s_mine[2];  // the slice keeps only some of its keys at P

  // ---- 2. kept positions of the slice, ascending, from the offset
  if (part) {  // rank of each key at P among the slice's keys at P
#pragma unroll
    for (int u = 0; u < kKPT; ++u) {
      const unsigned bal = __ballot_sync(0xffffffffu, in(u) && (key[u] >> shift) == P);
      if (lane == 0) tabE[u * kWarps + warp] = __popc(bal);
    }
    __syncthreads();
    scan_table(tabE, 0, scratch);
  }
#pragma unroll
  for (int u = 0; u < kKPT; ++u) {
    const uint32_t pre = key[u] >> shift;
    const bool at = in(u) && pre == P;
    bool keep = in(u) && pre > P;
    if (part) {
      const unsigned eb = __ballot_sync(0xffffffffu, at);
      keep = keep || (at && tabE[u * kWarps + warp] + __popc(eb & lt) < take);
    } else {
      keep = keep || at;
    }
    const unsigned bal = __ballot_sync(0xffffffffu, keep);
    if (lane == 0) tabK[u * kWarps + warp] = __popc(bal);
  }
  __syncthreads();
  scan_table(tabK, off, scratch);
#pragma unroll
  for (int u = 0; u < kKPT; ++u) {
    const uint32_t pre = key[u] >> shift;
    const bool at = in(u) && pre == P;
    bool keep = in(u) && pre > P;
    if (part) {
      const unsigned eb = __ballot_sync(0xffffffffu, at);
      keep = keep || (at && tabE[u * kWarps + warp] + __popc(eb & lt) < take);
    } else {
      keep = keep || at;
    }
    const unsigned bal = __ballot_sync(0xffffffffu, keep);
    if (keep) {
      const int slot = tabK[u * kWarps + warp] + __popc(bal & lt);
      if (slot < k) out[slot] = lo + u * kThreads + tid;
      else flag_status(a.status, PRISM_DEV_TOO_LONG);  // unreachable if counts are right
    }
  }
  if (rank == 0 && tid == 0) a.out_cnt[row] = k;
  // no CTA exits while rank 0's shared memory or its counts may still be read
  cluster_arrive();
  cluster_wait();
}

}  // namespace

int propose_select_cluster() { return kCL; }
int propose_select_max_row() { return kCL * kMaxSlice; }

cudaError_t launch_propose_select(const Dims& d, const float* scores, const uint32_t* hist,
                                  int kappa_p, int32_t* pool, int32_t* pool_cnt, int32_t* status,
                                  cudaStream_t st) {
  const int rows = d.B * d.Hkv;
  if (rows == 0) return cudaSuccess;
  PSArgs a{scores, hist, d.cu_dev, d.Hkv, d.T, kappa_p, pool, pool_cnt, status};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(rows * kCL));
  cfg.blockDim = dim3(kThreads);
  const int smem = kCL * kCandCap * (int)sizeof(uint2);
  cudaError_t e = cudaFuncSetAttribute(propose_select_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(propose_select_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e != cudaSuccess) return e;
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kCL;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, propose_select_kernel, a);
}

}  // namespace prism
