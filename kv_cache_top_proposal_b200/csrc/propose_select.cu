// Candidate pool of a proposal layer: the top kappa_p positions of every
// (sequence, KV head) row by proposal score, "lower index wins" on ties,
// written in ascending position order (Prism Attention, sec. 4.1
// "Proposal-Refined Index Sharing"; pool size n = rho * kappa, sec. 5.1
// "Implementation Details").
//
// The scorer has already built, per row, the histogram of the first 12 bits
// of ord(score).  One cluster of CL CTAs per row (CL = 4, 8 or 16: see
// propose_select_cluster); CTA r owns the contiguous
// slice r of positions and keeps its keys in registers (KPT per thread,
// coalesced: key u of thread t is slice position u * kThreads + t):
//   1. every CTA reads the row's histogram and locates the bin holding the
//      kappa_p-th largest key (same answer in every CTA).  Unless the whole
//      bin is taken, the CTAs histogram the next 10 bits of their keys in
//      it, each into its own shared memory; CTA c sums slice c of those
//      histograms over distributed shared memory and every CTA finds the
//      next bin from the slice totals and the right slice; then the last 10
//      bits.  This gives the threshold prefix P and how many keys at P are
//      taken, in position order ("lower index wins");
//   2. the CTAs exchange their counts above and at P, which gives each one
//      its share of the keys at P and its output offset;
//   3. every CTA writes its kept positions in ascending order (ballot counts
//      per (key block, warp), one block scan, placement).
#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.h"

namespace cg = cooperative_groups;

namespace prism {

namespace {

constexpr int kMaxCL = 16;                    // largest cluster (non-portable size)
constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kKPT = 16;                      // keys per thread
constexpr int kMaxSlice = kKPT * kThreads;    // keys per CTA
constexpr int kHist = 4096;                   // first digit (from the scorer)
constexpr int kBins = 1024;                   // second and third digits

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

template <int CL>
__global__ void __launch_bounds__(kThreads, 2) propose_select_kernel(const PSArgs a) {
  static_assert(kBins / CL <= kThreads && CL <= 32, "one slice bin per thread, one rank per lane");
  __shared__ __align__(16) uint32_t hist2[kBins];  // this CTA's digit-2 counts
  __shared__ __align__(16) uint32_t hist3[kBins];  // this CTA's digit-3 counts
  __shared__ int tabE[kKPT * kWarps];  // per (key block, warp): keys at P, then their prefix
  __shared__ int tabK[kKPT * kWarps];  // per (key block, warp): kept keys, then output slots
  __shared__ uint32_t s_sw[kBins / CL];  // this CTA's slice of the cluster's digit counts
  __shared__ int s_slice;
  __shared__ int scratch[33];
  __shared__ int s_dig[3];
  __shared__ int s_cnt[2];   // this CTA's keys above / at the prefix
  __shared__ int s_mine[3];  // output offset, keys at the prefix taken, keys at the prefix

  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int row = blockIdx.x / CL;
  const int b = row / a.Hkv, h = row - b * a.Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const unsigned lt = (1u << lane) - 1u;
  // this thread's bins of the row's first-digit histogram, loaded beside the
  // lengths: they do not depend on them
  constexpr int kHPer = kHist / kThreads;
  uint32_t hc[kHPer];
  {
    const uint32_t* gh = a.hist + (int64_t)row * kHist + tid * kHPer;
#pragma unroll
    for (int j = 0; j < kHPer; ++j) hc[j] = __ldcg(gh + j);
  }
  const int t0 = a.cu[b];
  const int n = a.cu[b + 1] - t0;
  const int chunk = (n + CL - 1) / CL;
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
    for (int i = filled + rank * kThreads + tid; i < a.kp; i += CL * kThreads) out[i] = -1;
    if (rank == 0 && tid == 0) a.out_cnt[row] = filled;
    return;
  }
  const int k = a.kp;
  for (int i = tid; i < kBins; i += kThreads) {
    hist2[i] = 0u;
    hist3[i] = 0u;
  }
  __syncthreads();
  cluster_arrive();  // pairs with the wait below (every CTA is running)

  // ---- the slice's keys, kKPT loads in flight per thread while the first
  // digit's bin is found (step 1 below)
  uint32_t key[kKPT];
  {
    const float* kb = a.scores + (int64_t)h * a.T + t0 + lo;
    float v[kKPT];
#pragma unroll
    for (int u = 0; u < kKPT; ++u) {
      const int i = u * kThreads + tid;
      v[u] = i < m ? __ldcg(kb + i) : 0.0f;
    }
    find_digit<kHPer>([&](int bin) { return hc[bin - tid * kHPer]; }, k, scratch, s_dig);
#pragma unroll
    for (int u = 0; u < kKPT; ++u) key[u] = ord_key(v[u]);
  }
  auto in = [&](int u) { return u * kThreads + tid < m; };

  // ---- 1. threshold: keys with (key >> shift) > P are taken, and the first
  // rtie keys with (key >> shift) == P in position order.  Every CTA finds
  // the first digit's bin b1 from the row's histogram.  Unless the whole
  // bin is taken, each CTA counts the next 10 bits of its keys in b1 into its
  // own histogram; CTA c sums slice c of all of them (distributed shared
  // memory reads, no remote atomics) and every CTA finds the next bin from
  // the slice totals and the right slice; then the same for the last 10
  // bits.  Finally the CTAs exchange their counts above and at P.
  uint32_t P = (uint32_t)s_dig[0];
  int shift = 20;
  const int c1 = s_dig[2];
  int r = k - s_dig[1];
  cluster_wait();
  auto cluster_digit = [&](const uint32_t* hl, int rr) {
    constexpr int WS = kBins / CL;  // bins per slice
    __syncthreads();
    cluster.sync();  // every CTA's histogram is complete
    int part = 0;
    for (int x = tid; x < WS; x += kThreads) {
      uint32_t v[CL];  // every CTA's count, all loads in flight at once
#pragma unroll
      for (int c = 0; c < CL; ++c) v[c] = cluster.map_shared_rank(hl, c)[rank * WS + x];
      uint32_t acc = 0u;
#pragma unroll
      for (int c = 0; c < CL; ++c) acc += v[c];
      s_sw[x] = acc;
      part += (int)acc;
    }
    int tot;
    block_excl_scan(part, scratch, &tot);
    if (tid == 0) s_slice = tot;
    cluster.sync();  // every slice and its total are ready
    if (warp == 0) {
      const int t = lane < CL ? *cluster.map_shared_rank(&s_slice, lane) : 0;
      const int incl = warp_incl_scan(t);  // slices rank in descending bin order
      const int above = __shfl_sync(0xffffffffu, incl, 31) - incl;
      const unsigned hit = __ballot_sync(0xffffffffu, lane < CL && above < rr && rr <= above + t);
      const int src = hit ? __ffs(hit) - 1 : 0;  // exactly one lane when counts are right
      const int above_src = __shfl_sync(0xffffffffu, above, src);
      if (lane == 0) {
        s_dig[0] = src;
        s_dig[1] = above_src;
      }
    }
    __syncthreads();
    const int src = s_dig[0], above_s = s_dig[1];
    const uint32_t* swr = cluster.map_shared_rank(s_sw, src);
    const int v = tid < WS ? (int)swr[tid] : 0;  // one bin per thread (WS <= kThreads)
    int total2;
    const int excl = block_excl_scan(v, scratch, &total2);
    const int above = above_s + total2 - excl - v;
    if (tid < WS && above < rr && rr <= above + v) {
      s_dig[0] = src * WS + tid;
      s_dig[1] = above;
      s_dig[2] = v;
    }
    __syncthreads();
  };
  if (r < c1) {  // part of the bin: the second digit of its keys
#pragma unroll
    for (int u = 0; u < kKPT; ++u)
      if (in(u) && (key[u] >> 20) == P) atomicAdd(hist2 + ((key[u] >> 10) & (kBins - 1)), 1u);
    cluster_digit(hist2, r);
    P = (P << 10) | (uint32_t)s_dig[0];
    shift = 10;
    r -= s_dig[1];
    if (r < s_dig[2]) {  // the last digit
#pragma unroll
      for (int u = 0; u < kKPT; ++u)
        if (in(u) && (key[u] >> 10) == P) atomicAdd(hist3 + (key[u] & (kBins - 1)), 1u);
      cluster_digit(hist3, r);
      P = (P << 10) | (uint32_t)s_dig[0];
      shift = 0;
      r -= s_dig[1];
    }
  }
  const int rtie = r;
  // counts above / at P, then every CTA's, in rank order
  {
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
  }
  cluster.sync();  // every CTA's counts are published
  if (warp == 0) {
    int g_s = 0, e_s = 0;
    if (lane < CL) {
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
  // this CTA's last read of another CTA's shared memory is done; the wait
  // at the end keeps every CTA's shared memory alive until all have arrived
  cluster_arrive();
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
  cluster_wait();  // no CTA exits while its counts may still be read
}

}  // namespace

// Smallest cluster whose CTAs hold the longest row the captured call can
// meet: the other rows keep their lengths and the last one may grow into the
// spare rows up to total_tokens.  A shorter row leaves most key registers of
// its CTAs empty, and every CTA costs about the same whatever its fill, so a
// cluster sized to the rows cuts the CTAs (and the waves) of a batch of
// shorter rows.  Past the largest cluster's capacity the largest is used
// (rows longer than that flag PRISM_DEV_TOO_LONG, as before).
int propose_select_cluster(const Dims& d) {
  int64_t bound = 0;
  for (int b = 0; b < d.B; ++b) {
    const int64_t L = b + 1 < d.B ? (int64_t)(d.cu_host[b + 1] - d.cu_host[b])
                                  : d.T - d.cu_host[b];
    bound = L > bound ? L : bound;
  }
  int cl = 4;
  while (cl < kMaxCL && (int64_t)cl * kMaxSlice < bound) cl *= 2;
  return cl;
}
int propose_select_max_row() { return kMaxCL * kMaxSlice; }

namespace {
template <int CL>
cudaError_t launch_ps(const PSArgs& a, int rows, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(rows * CL));
  cfg.blockDim = dim3(kThreads);
  if (CL > 8) {
    cudaError_t e = cudaFuncSetAttribute(propose_select_kernel<CL>,
                                         cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CL;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, propose_select_kernel<CL>, a);
}
}  // namespace

cudaError_t launch_propose_select(const Dims& d, const float* scores, const uint32_t* hist,
                                  int kappa_p, int32_t* pool, int32_t* pool_cnt, int32_t* status,
                                  cudaStream_t st) {
  const int rows = d.B * d.Hkv;
  if (rows == 0) return cudaSuccess;
  PSArgs a{scores, hist, d.cu_dev, d.Hkv, d.T, kappa_p, pool, pool_cnt, status};
  switch (propose_select_cluster(d)) {
    case 4: return launch_ps<4>(a, rows, st);
    case 8: return launch_ps<8>(a, rows, st);
    default: return launch_ps<16>(a, rows, st);
  }
}

}  // namespace prism
