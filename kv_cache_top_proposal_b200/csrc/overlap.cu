// Index overlap of two selections per row (Prism Attention, sec. 3
// "Observations", Figure 1: the overlap ratio between a reference layer's
// index set and the set of a layer at some offset; Figure 12: how much of a
// layer's top-kappa an expanded top-rho*kappa set covers).  One CTA per row:
// each thread takes members of a and looks them up in b by binary search
// (both lists ascending), and the CTA adds up the hits.  A diagnostic, not
// a step of the decode path: it reads 4 (|a| log |b|) bytes per row.
#include "common.cuh"
#include "kernels.h"

namespace prism {
namespace {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads) overlap_kernel(const int32_t* __restrict__ a,
                                                           const int32_t* __restrict__ cnt_a,
                                                           int stride_a,
                                                           const int32_t* __restrict__ b,
                                                           const int32_t* __restrict__ cnt_b,
                                                           int stride_b, int32_t* __restrict__ out) {
  __shared__ int scratch[33];
  const int row = blockIdx.x;
  const int na = min(max(cnt_a[row], 0), stride_a);
  const int nb = min(max(cnt_b[row], 0), stride_b);
  const int32_t* ar = a + (int64_t)row * stride_a;
  const int32_t* br = b + (int64_t)row * stride_b;
  int hits = 0;
  for (int i = threadIdx.x; i < na; i += kThreads) {
    const int32_t x = ar[i];
    int lo = 0, hi = nb;  // first member of b that is >= x
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (br[mid] < x) lo = mid + 1;
      else hi = mid;
    }
    hits += lo < nb && br[lo] == x;
  }
  int total;
  block_excl_scan(hits, scratch, &total);
  if (threadIdx.x == 0) out[row] = total;
}

}  // namespace

cudaError_t launch_overlap(int rows, const int32_t* a, const int32_t* cnt_a, int stride_a,
                           const int32_t* b, const int32_t* cnt_b, int stride_b, int32_t* out,
                           cudaStream_t st) {
  if (rows == 0) return cudaSuccess;
  overlap_kernel<<<rows, kThreads, 0, st>>>(a, cnt_a, stride_a, b, cnt_b, stride_b, out);
  return cudaGetLastError();
}

}  // namespace prism
