// Exact top-k selection with the "lower index wins" tie rule, output in
// ascending position order -- the pool of a proposal layer and the refined
// set of every layer (Prism Attention, sec. 4.1 "Proposal-Refined Index
// Sharing"; pool size n = rho * kappa, sec. 5.1 "Implementation Details").
//
// One thread-block cluster of kCluster CTAs owns one selection row (a
// (sequence, KV head) pair).  Each CTA keeps its contiguous slice of the row's
// keys -- ord(score), an order-preserving uint32 -- in shared memory, and the
// cluster runs an MSD radix select over the 32 key bits in three digit passes
// (11, 11, 10 bits): every CTA histograms the keys that still match the
// digit prefix, the histograms are summed through distributed shared memory
// (DSMEM), and every CTA locates the digit that holds the k-th largest key.
// After the last pass the exact threshold key T is known together with how
// many keys equal to T are still needed; those are taken in position order
// (lower position wins).  A final ordered compaction -- block scans inside a
// CTA, per-CTA counts exchanged over DSMEM -- writes the chosen positions in
// ascending order with no sort.  The cluster barriers are hardware
// barriers; no thread ever spins on memory.
//
// Because selection needs no output order beyond "ascending position", and
// the position order is the slice order, the k-th-largest threshold is the
// only global fact the row needs; the scores are read once from L2.
#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.h"

namespace cg = cooperative_groups;

namespace prism {

namespace {

constexpr int kCluster = 8;
constexpr int kThreads = 1024;
constexpr int kMaxChunk = 49152;  // keys per CTA (192 KB of shared memory)

// mode 1: selection row `row` draws from pool row row / pool_div (several
// selection rows -- the query heads of a group -- may share one pool)
__device__ __forceinline__ int pool_row(const SelectArgs& a, int row) {
  return a.pool_div > 1 ? row / a.pool_div : row;
}

__device__ __forceinline__ int32_t position_of(const SelectArgs& a, int row, int i) {
  return a.mode == 0 ? i : a.pool[(int64_t)pool_row(a, row) * a.pool_stride + i];
}

__device__ __forceinline__ void emit(const SelectArgs& a, int row, int b, int h, int i, int slot,
                                     int32_t* out) {
  out[slot] = position_of(a, row, i);
  if (a.logits) {
    for (int g = 0; g < a.G; ++g)
      a.logits[((int64_t)b * a.Hq + (int64_t)h * a.G + g) * a.k_req + slot] =
          a.dots[((int64_t)row * a.G + g) * a.pool_stride + i];
  }
}

__global__ void __launch_bounds__(kThreads, 1) select_kernel(const SelectArgs a) {
  extern __shared__ __align__(16) uint32_t skeys[];
  __shared__ uint32_t hist[2][2048];
  __shared__ uint32_t ghist[2048];
  __shared__ int scratch[33];
  __shared__ int s_digit, s_above;
  __shared__ int s_counts[2];  // published to the cluster: #equal, #greater
  __shared__ int s_before[2];  // #equal and #selected in lower-ranked CTAs

  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int row = blockIdx.x / kCluster;
  const int b = row / a.Hkv, h = row - b * a.Hkv;
  const int tid = threadIdx.x;

  int n;
  const float* kbase;
  if (a.mode == 0) {
    const int t0 = a.cu[b];
    n = a.cu[b + 1] - t0;
    kbase = a.keys + (int64_t)h * a.T + t0;
  } else {
    n = a.pool_cnt[pool_row(a, row)];
    if (n < 0 || n > a.pool_stride) {
      if (rank == 0 && tid == 0) flag_status(a.status, PRISM_DEV_BAD_INDEX);
      n = n < 0 ? 0 : a.pool_stride;
    }
    kbase = a.keys + (int64_t)row * a.pool_stride;
  }
  int32_t* out = a.out + (int64_t)row * a.k_req;
  const int chunk = (n + kCluster - 1) / kCluster;
  const int lo = min(n, rank * chunk), hi = min(n, lo + chunk);
  const int m = hi - lo;

  // Every branch below depends only on values shared by the whole cluster,
  // so all of its CTAs take the same one.
  if (n <= a.k_req || chunk > kMaxChunk) {
    const bool all = n <= a.k_req;
    if (all) {
      for (int i = lo + tid; i < hi; i += kThreads) emit(a, row, b, h, i, i, out);
    } else if (rank == 0 && tid == 0) {
      flag_status(a.status, PRISM_DEV_TOO_LONG);
    }
    const int filled = all ? n : 0;
    for (int i = filled + rank * kThreads + tid; i < a.k_req; i += kCluster * kThreads) out[i] = -1;
    if (rank == 0 && tid == 0) a.out_cnt[row] = filled;
    return;
  }
  const int k = a.k_req;  // n > k_req here

  for (int i = tid; i < m; i += kThreads) skeys[i] = ord_key(kbase[lo + i]);
  for (int i = tid; i < 2048; i += kThreads) hist[0][i] = 0;
  __syncthreads();

  uint32_t prefix = 0, pmask = 0;
  int krem = k;  // rank (1-based, from the top) of the threshold among prefix matches
#pragma unroll 1
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
    const int nb = pass == 2 ? 1024 : 2048;
    uint32_t* hh = hist[pass & 1];
    for (int i0 = tid & ~31; i0 < m; i0 += kThreads) {  // warp-uniform trip count
      const int i = i0 + (tid & 31);
      const uint32_t key = i < m ? skeys[i] : 0u;
      warp_hist_add(hh, (key >> shift) & (nb - 1), i < m && (key & pmask) == prefix);
    }
    cluster.sync();  // every CTA's histogram of this pass is complete
    // All CTAs have finished reading the other buffer (previous pass) before
    // arriving here, so it can be cleared for the next pass.
    if (pass < 2)
      for (int i = tid; i < 2048; i += kThreads) hist[(pass + 1) & 1][i] = 0;
    for (int bin = tid; bin < nb; bin += kThreads) {
      uint32_t s = 0;
#pragma unroll
      for (int r = 0; r < kCluster; ++r) s += cluster.map_shared_rank(hh, r)[bin];
      ghist[bin] = s;
    }
    __syncthreads();
    // Thread t owns bins [t*per, t*per + per); count keys above its bins.
    const int per = nb / kThreads;
    int v = 0;
    for (int j = 0; j < per; ++j) v += (int)ghist[tid * per + j];
    int total;
    const int excl = block_excl_scan(v, scratch, &total);
    int above = total - excl - v;
    for (int j = per - 1; j >= 0; --j) {
      const int c = (int)ghist[tid * per + j];
      if (above < krem && krem <= above + c) {
        s_digit = tid * per + j;
        s_above = above;
      }
      above += c;
    }
    __syncthreads();
    prefix |= (uint32_t)s_digit << shift;
    pmask |= (uint32_t)(nb - 1) << shift;
    krem -= s_above;
    __syncthreads();
  }
  const uint32_t T = prefix;  // the k-th largest key; krem keys equal to T are taken

  // Ordered compaction: thread tid owns the contiguous slice [i0, i1).
  const int per = (m + kThreads - 1) / kThreads;
  const int i0 = min(m, tid * per), i1 = min(m, i0 + per);
  int gt = 0, eq = 0;
  for (int i = i0; i < i1; ++i) {
    const uint32_t key = skeys[i];
    gt += key > T;
    eq += key == T;
  }
  int eq_tot, gt_tot;
  const int eq_pre = block_excl_scan(eq, scratch, &eq_tot);
  block_excl_scan(gt, scratch, &gt_tot);
  if (tid == 0) {
    s_counts[0] = eq_tot;
    s_counts[1] = gt_tot;
  }
  cluster.sync();
  if (tid == 0) {
    int eb = 0, sb = 0;
    for (int r = 0; r < rank; ++r) {
      const int* cnt = cluster.map_shared_rank(s_counts, r);
      const int e = cnt[0], g = cnt[1];
      sb += g + max(0, min(krem - eb, e));
      eb += e;
    }
    s_before[0] = eb;
    s_before[1] = sb;
  }
  __syncthreads();
  const int take = max(0, min(krem - (s_before[0] + eq_pre), eq));
  int sel_tot;
  const int sel_pre = block_excl_scan(gt + take, scratch, &sel_tot);
  int o = s_before[1] + sel_pre;
  int taken = 0;
  for (int i = i0; i < i1; ++i) {
    const uint32_t key = skeys[i];
    bool s = key > T;
    if (key == T) s = taken++ < take;
    if (s) {
      if (o < k) emit(a, row, b, h, lo + i, o, out);
      else flag_status(a.status, PRISM_DEV_TOO_LONG);  // unreachable if the count is right
      ++o;
    }
  }
  if (rank == 0 && tid == 0) a.out_cnt[row] = k;
  cluster.sync();  // keep s_counts alive until every remote read is done
}

}  // namespace

int select_capacity_per_row() { return kCluster * kMaxChunk; }

cudaError_t launch_select(const Dims& d, const SelectArgs& a, int max_row_len, cudaStream_t st) {
  const int rows = d.B * d.Hkv;
  if (rows == 0) return cudaSuccess;
  int chunk = (max_row_len + kCluster - 1) / kCluster;
  if (chunk > kMaxChunk) chunk = kMaxChunk;
  if (chunk < 1) chunk = 1;
  const size_t smem = (size_t)chunk * sizeof(uint32_t);
  cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)(kMaxChunk * sizeof(uint32_t)));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(rows * kCluster));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kCluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, select_kernel, a);
}

}  // namespace prism
