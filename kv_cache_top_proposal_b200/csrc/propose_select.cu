// Candidate pool of a proposal layer: the top kappa_p positions of every
// (sequence, KV head) row by proposal score, "lower index wins" on ties,
// written in ascending position order (Prism Attention, sec. 4.1
// "Proposal-Refined Index Sharing"; pool size n = rho * kappa, sec. 5.1
// "Implementation Details").
//
// The scorer has already built, per row, the histogram of the first 12 bits
// of ord(score).  One cluster of kCL CTAs per row, each owning a contiguous
// slice of positions:
//   1. every CTA reads the row's histogram and locates the bin b1 that holds
//      the kappa_p-th largest key (same answer in every CTA), loads its slice
//      of keys into shared memory, counts its keys above b1 and lists its
//      keys in b1 -- in position order -- into a global candidate region;
//   2. rank 0 resolves the exact threshold T (the two remaining digits) and
//      the last taken position I* among keys equal to T (lower positions
//      first) over the concatenated candidate lists, and every slice's
//      output offset;
//   3. every CTA writes its kept positions (key > T, or key == T and position
//      <= I*) in ascending order from its offset.
// Hand-offs go through global memory (L2) ordered by the cluster barrier;
// two barriers in all, no distributed shared memory.
#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.h"

namespace cg = cooperative_groups;

namespace prism {

namespace {

constexpr int kCL = 8;
constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kHist = 4096;
constexpr int kMaxSlice = 16384;  // keys per CTA (+ the candidate copy: 192 KB of shared memory)

struct PSArgs {
  const float* scores;  // [Hkv][T]
  const uint32_t* hist;  // [rows][kHist]
  const int32_t* cu;
  int Hkv;
  int64_t T;
  int kp;
  int cap;               // candidate capacity per CTA (slice length bound)
  uint32_t* ckey;        // [rows][kCL][cap]
  int32_t* cpos;         // [rows][kCL][cap]
  int32_t* cmeta;        // [rows][kCL][2]: listed count, count above b1
  int32_t* res;          // [rows][2 + kCL]: T, I*, offsets
  int32_t* out;          // [rows][kp]
  int32_t* out_cnt;      // [rows]
  int32_t* status;
};

// bin of `nb` (padded-free) holding the r-th largest among keys matching
// prefix/pmask, over n keys read by get(j); whole CTA; returns in s3[0..2]
// (bin, count above, count in bin).
template <typename Get>
__device__ void find_bin_any(Get get, int n, uint32_t prefix, uint32_t pmask, int shift, int nb,
                             int r, uint32_t* hist, int* scratch, int* s3) {
  const int tid = threadIdx.x;
  for (int i = tid; i < nb; i += kThreads) hist[i] = 0u;
  __syncthreads();
  for (int j0 = tid & ~31; j0 < n; j0 += kThreads) {  // warp-uniform trip count
    const int j = j0 + (tid & 31);
    const uint32_t key = j < n ? get(j) : 0u;
    warp_hist_add(hist, (key >> shift) & (uint32_t)(nb - 1), j < n && (key & pmask) == prefix);
  }
  __syncthreads();
  const int v = tid < nb ? (int)hist[tid] : 0;  // nb <= kThreads
  int total;
  const int excl = block_excl_scan(v, scratch, &total);
  const int above = total - excl - v;
  if (tid < nb && above < r && r <= above + v) {
    s3[0] = tid;
    s3[1] = above;
    s3[2] = v;
  }
  __syncthreads();
}


// Ordered compaction of the CTA's m items: pred(i) selects, emit(i, slot)
// receives slot = base + rank of i among the selected, in index order.
// Two passes over blocks of kThreads items: ballot counts per (block, warp)
// into tab, one block-wide scan, then placement.  tab holds >= ceil(m /
// kThreads) * kWarps ints.  Returns the selected count.  Whole CTA.
template <typename Pred, typename Emit>
__device__ int ordered_compact(int m, int base, Pred pred, Emit emit, int* tab, int* scratch) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nblk = (m + kThreads - 1) / kThreads;
#pragma unroll 4
  for (int u = 0; u < nblk; ++u) {
    const int i = u * kThreads + tid;
    const unsigned bal = __ballot_sync(0xffffffffu, i < m && pred(i));
    if (lane == 0) tab[u * kWarps + warp] = __popc(bal);
  }
  __syncthreads();
  const int ne = nblk * kWarps;
  const int per = (ne + kThreads - 1) / kThreads;
  int v = 0;
  for (int j = 0; j < per; ++j) {
    const int e = tid * per + j;
    if (e < ne) v += tab[e];
  }
  int total;
  int acc = block_excl_scan(v, scratch, &total) + base;
  for (int j = 0; j < per; ++j) {
    const int e = tid * per + j;
    if (e < ne) {
      const int c = tab[e];
      tab[e] = acc;
      acc += c;
    }
  }
  __syncthreads();
#pragma unroll 4
  for (int u = 0; u < nblk; ++u) {
    const int i = u * kThreads + tid;
    const bool s = i < m && pred(i);
    const unsigned bal = __ballot_sync(0xffffffffu, s);
    if (s) emit(i, tab[u * kWarps + warp] + __popc(bal & ((1u << lane) - 1u)));
  }
  __syncthreads();
  return total;
}

__global__ void __launch_bounds__(kThreads, 1) propose_select_kernel(const PSArgs a) {
  extern __shared__ __align__(16) uint32_t skeys[];  // [slice], then the candidate copy
  __shared__ uint32_t hist[kThreads];
  __shared__ int tab[(kMaxSlice / kThreads) * kWarps];
  __shared__ int scratch[33];
  __shared__ int s3[3];
  __shared__ int s_wc[kWarps];
  __shared__ int s_meta[kCL][2];
  __shared__ int s_res[2 + kCL];

  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int row = blockIdx.x / kCL;
  const int b = row / a.Hkv, h = row - b * a.Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int t0 = a.cu[b];
  const int n = a.cu[b + 1] - t0;
  const int chunk = (n + kCL - 1) / kCL;
  const int lo = min(n, rank * chunk), hi = min(n, lo + chunk);
  const int m = hi - lo;
  int32_t* out = a.out + (int64_t)row * a.kp;

  // every branch depends on cluster-wide values only
  if (n <= a.kp || chunk > a.cap) {
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

  // ---- 1. first digit from the histogram; the slice's keys
  const uint32_t* gh = a.hist + (int64_t)row * kHist;
  {
    // 4 bins per thread, consecutive: bins 4t .. 4t+3
    const uint4 v4 = reinterpret_cast<const uint4*>(gh)[tid];
    const int v = (int)(v4.x + v4.y + v4.z + v4.w);
    int total;
    const int excl = block_excl_scan(v, scratch, &total);
    int above = total - excl - v;
    const uint32_t c4[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
    for (int j = 3; j >= 0; --j) {
      const int c = (int)c4[j];
      if (above < k && k <= above + c) {
        s3[0] = 4 * tid + j;
        s3[1] = above;
        s3[2] = c;
      }
      above += c;
    }
  }
  const float* kbase = a.scores + (int64_t)h * a.T + t0 + lo;
  for (int i0 = 0; i0 < m; i0 += 8 * kThreads) {  // eight independent loads in flight
    float v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = i0 + u * kThreads + tid;
      v[u] = i < m ? __ldcg(kbase + i) : 0.0f;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = i0 + u * kThreads + tid;
      if (i < m) skeys[i] = ord_key(v[u]);
    }
  }
  __syncthreads();
  const uint32_t b1 = (uint32_t)s3[0];
  const int r1 = k - s3[1];
  // keys above b1 (count) and in b1 (listed in position order)
  {
    uint32_t* ck = a.ckey + ((int64_t)row * kCL + rank) * a.cap;
    int32_t* cp = a.cpos + ((int64_t)row * kCL + rank) * a.cap;
    int gt = 0;
    for (int i = tid; i < m; i += kThreads) gt += (skeys[i] >> 20) > b1;
    const int nc = ordered_compact(
        m, 0, [&](int i) { return (skeys[i] >> 20) == b1; },
        [&](int i, int at) {
          ck[at] = skeys[i];
          cp[at] = lo + i;
        },
        tab, scratch);
    int gtot;
    block_excl_scan(gt, scratch, &gtot);
    if (tid == 0) {
      a.cmeta[((int64_t)row * kCL + rank) * 2] = nc;
      a.cmeta[((int64_t)row * kCL + rank) * 2 + 1] = gtot;
    }
  }
  cluster.sync();  // S1: every candidate list is in global memory

  // ---- 2. rank 0: exact threshold over the concatenated lists, offsets
  if (rank == 0) {
    if (tid < kCL * 2) s_meta[tid / 2][tid % 2] = __ldcg(a.cmeta + (int64_t)row * kCL * 2 + tid);
    __syncthreads();
    int pre[kCL + 1];
    pre[0] = 0;
#pragma unroll
    for (int c = 0; c < kCL; ++c) pre[c + 1] = pre[c] + s_meta[c][0];
    const int nc = pre[kCL];
    const uint32_t* ckr = a.ckey + (int64_t)row * kCL * a.cap;
    const int32_t* cpr = a.cpos + (int64_t)row * kCL * a.cap;
    // list index j -> (CTA c, entry) by the prefix of the counts
    auto where = [&](int j) {
      int c = 0;
#pragma unroll
      for (int x = 1; x < kCL; ++x) c += j >= pre[x];
      return (int64_t)c * a.cap + (j - pre[c]);
    };
    // the concatenated list into shared memory when it fits (else read from L2)
    uint32_t* lk = skeys + ((a.cap + 3) & ~3);
    int32_t* lp = reinterpret_cast<int32_t*>(lk + a.cap);
    const bool local = nc <= a.cap;
    if (local) {
      for (int c = 0; c < kCL; ++c) {
        const int cnt = s_meta[c][0];
        for (int j = tid; j < cnt; j += kThreads) {
          lk[pre[c] + j] = __ldcg(ckr + (int64_t)c * a.cap + j);
          lp[pre[c] + j] = __ldcg(cpr + (int64_t)c * a.cap + j);
        }
      }
      __syncthreads();
    }
    auto getk = [&](int j) { return local ? lk[j] : __ldcg(ckr + where(j)); };
    auto getp = [&](int j) { return local ? lp[j] : __ldcg(cpr + where(j)); };
    uint32_t prefix = b1 << 20, pmask = 0xFFF00000u;
    int r = r1;
    find_bin_any(getk, nc, prefix, pmask, 10, 1024, r, hist, scratch, s3);
    prefix |= (uint32_t)s3[0] << 10;
    pmask |= 0x000FFC00u;
    r -= s3[1];
    find_bin_any(getk, nc, prefix, pmask, 0, 1024, r, hist, scratch, s3);
    prefix |= (uint32_t)s3[0];
    r -= s3[1];
    const uint32_t T = prefix;
    // the r-th listed key equal to T, in list (= position) order
    __shared__ int s_I;
    int before = 0;
    for (int j0 = 0; j0 < nc && before < r; j0 += kThreads) {  // CTA-uniform
      const int j = j0 + tid;
      const unsigned eqm = __ballot_sync(0xffffffffu, j < nc && getk(j) == T);
      if (lane == 0) s_wc[warp] = __popc(eqm);
      __syncthreads();
      int mine = before, tot = before;
      for (int w = 0; w < kWarps; ++w) {
        if (w < warp) mine += s_wc[w];
        tot += s_wc[w];
      }
      if (lane == 0 && mine < r && r <= mine + __popc(eqm)) {
        unsigned msk = eqm;
        for (int t = 1; t < r - mine; ++t) msk &= msk - 1;
        s_I = getp(j - lane + __ffs(msk) - 1);
      }
      before = tot;
      __syncthreads();
    }
    const int I = s_I;
    // selected listed keys per CTA region -> offsets
    __shared__ int s_sel[kCL];
    if (tid < kCL) s_sel[tid] = 0;
    __syncthreads();
    for (int j0 = warp * 32; j0 < nc; j0 += kThreads) {  // warp-uniform trip count
      const int j = j0 + lane;
      bool sel = false;
      int c = 0;
      if (j < nc) {
        const uint32_t key = getk(j);
        sel = key > T || (key == T && getp(j) <= I);
#pragma unroll
        for (int x = 1; x < kCL; ++x) c += j >= pre[x];
      }
      const int cf = __shfl_sync(0xffffffffu, c, 0);
      const int cl = __shfl_sync(0xffffffffu, c, min(31, nc - 1 - j0));
      for (int cc = cf; cc <= cl; ++cc) {  // the regions this block of 32 spans
        const unsigned m2 = __ballot_sync(0xffffffffu, sel && c == cc);
        if (lane == 0 && m2) atomicAdd(&s_sel[cc], __popc(m2));
      }
    }
    __syncthreads();
    if (tid == 0) {
      int32_t* rr = a.res + (int64_t)row * (2 + kCL);
      rr[0] = (int32_t)T;
      rr[1] = I;
      int acc = 0;
      for (int c = 0; c < kCL; ++c) {
        rr[2 + c] = acc;
        acc += s_meta[c][1] + s_sel[c];
      }
      a.out_cnt[row] = k;
    }
  }
  cluster.sync();  // S2: threshold and offsets are in global memory

  // ---- 3. kept positions of the slice, ascending, from the offset
  if (tid < 3) s_res[tid] = __ldcg(a.res + (int64_t)row * (2 + kCL) + (tid < 2 ? tid : 2 + rank));
  __syncthreads();
  const uint32_t T = (uint32_t)s_res[0];
  const int I = s_res[1];
  ordered_compact(
      m, s_res[2], [&](int i) { return skeys[i] > T || (skeys[i] == T && lo + i <= I); },
      [&](int i, int slot) {
        if (slot < k) out[slot] = lo + i;
        else flag_status(a.status, PRISM_DEV_TOO_LONG);  // unreachable if counts are right
      },
      tab, scratch);
}

}  // namespace

int propose_select_cap(int max_len) { return (max_len + kCL - 1) / kCL; }
int propose_select_cluster() { return kCL; }
int propose_select_max_row() { return kCL * kMaxSlice; }

cudaError_t launch_propose_select(const Dims& d, const float* scores, const uint32_t* hist,
                                  int kappa_p, int cap, uint32_t* ckey, int32_t* cpos,
                                  int32_t* cmeta, int32_t* res, int32_t* pool, int32_t* pool_cnt,
                                  int32_t* status, cudaStream_t st) {
  const int rows = d.B * d.Hkv;
  if (rows == 0) return cudaSuccess;
  PSArgs a{scores, hist, d.cu_dev, d.Hkv, d.T, kappa_p, cap, ckey, cpos, cmeta, res, pool, pool_cnt,
           status};
  const int slice = cap > 0 ? cap : 1;
  const size_t smem = (size_t)(((slice + 3) & ~3) + 2 * slice) * sizeof(uint32_t);
  cudaError_t e = cudaFuncSetAttribute(propose_select_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(rows * kCL));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
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
