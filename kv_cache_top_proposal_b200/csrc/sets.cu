// Selection granularity: the maximum of per-head scores over the heads, for
// one pool and one index set per sequence shared by every head (Prism
// Attention, sec. 4.1 leaves the granularity of the shared sets open; sec. 2
// "Related Work" names a set shared by all heads).  The proposal scores
// [Hkv][T] become one score per position, the exact pool scores
// [B][Hkv][kappa_p] one per pool member; the selections then run on them
// as on a single KV head.  HBM bound: H + 1 floats per output (L2-resident
// after the scorer).
#include "common.cuh"
#include "kernels.h"

namespace prism {
namespace {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads) head_max_kernel(const float* __restrict__ in, int H,
                                                            int64_t outer, int64_t inner,
                                                            float* __restrict__ out) {
  const int64_t total = outer * inner;
  for (int64_t x = (int64_t)blockIdx.x * kThreads + threadIdx.x; x < total;
       x += (int64_t)gridDim.x * kThreads) {
    const int64_t o = x / inner, i = x - o * inner;
    const float* src = in + o * H * inner + i;
    float m = src[0];
    for (int h = 1; h < H; ++h) m = fmaxf(m, src[(int64_t)h * inner]);
    out[x] = m;
  }
}

}  // namespace

cudaError_t launch_head_max(const float* in, int H, int64_t outer, int64_t inner, float* out,
                            cudaStream_t st) {
  const int64_t total = outer * inner;
  if (total == 0 || H < 1) return cudaSuccess;
  int64_t blocks = cdiv(total, kThreads);
  if (blocks > 148 * 8) blocks = 148 * 8;
  head_max_kernel<<<(unsigned)blocks, kThreads, 0, st>>>(in, H, outer, inner, out);
  return cudaGetLastError();
}

}  // namespace prism
