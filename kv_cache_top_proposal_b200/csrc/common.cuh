// Device helpers shared by the libprism kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/prism.h"

namespace prism {

__device__ __forceinline__ void flag_status(int32_t* status, int32_t bits) {
  if (status) atomicOr(status, bits);
}

// Order-preserving map of an fp32 score to uint32 (after -0.0 -> +0.0):
// a > b as floats  <=>  ord(a) > ord(b) as unsigned.  Selection keys compare
// (ord(score) desc, position asc), the "lower index wins" total order.
__device__ __forceinline__ uint32_t ord_key(float x) {
  uint32_t u = __float_as_uint(__fadd_rn(x, 0.0f));
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// bf16 pair in one 32-bit word -> two exact fp32 values.
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// 16 bytes of a row as E fp32 values (E = 8 for bf16, 4 for fp32).
template <typename T>
struct Vec16;

template <>
struct Vec16<__nv_bfloat16> {
  static constexpr int E = 8;
  __device__ __forceinline__ static void unpack(const uint4& r, float* f) {
    f[0] = bf16lo(r.x); f[1] = bf16hi(r.x);
    f[2] = bf16lo(r.y); f[3] = bf16hi(r.y);
    f[4] = bf16lo(r.z); f[5] = bf16hi(r.z);
    f[6] = bf16lo(r.w); f[7] = bf16hi(r.w);
  }
};

template <>
struct Vec16<float> {
  static constexpr int E = 4;
  __device__ __forceinline__ static void unpack(const uint4& r, float* f) {
    f[0] = __uint_as_float(r.x); f[1] = __uint_as_float(r.y);
    f[2] = __uint_as_float(r.z); f[3] = __uint_as_float(r.w);
  }
};

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

// Read-only 16-byte loads: streaming (touched once) and default-cached.
__device__ __forceinline__ uint4 ld16_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}
__device__ __forceinline__ uint4 ld16(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

// Sum over the W lanes of an aligned lane group; every lane of the group
// ends with the bit-identical total (each xor step adds the two partners'
// values in both lanes, and fp32 addition is commutative).
template <int W>
__device__ __forceinline__ float group_sum(float v) {
#pragma unroll
  for (int o = W / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ int warp_incl_scan(int v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  return v;
}

// Block-wide exclusive scan of one int per thread; returns the exclusive
// prefix and writes the block total to *total.  scratch holds >= 33 ints.
// Contains __syncthreads(): call from every thread.
__device__ __forceinline__ int block_excl_scan(int v, int* scratch, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = (blockDim.x + 31) >> 5;
  int inc = warp_incl_scan(v);
  if (lane == 31) scratch[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    int w = lane < nwarps ? scratch[lane] : 0;
    int wi = warp_incl_scan(w);
    if (lane < nwarps) scratch[lane] = wi - w;
    if (lane == 31) scratch[32] = wi;
  }
  __syncthreads();
  int res = scratch[warp] + inc - v;
  *total = scratch[32];
  __syncthreads();
  return res;
}


// ---- cp.async (16-byte global -> shared copies, L2 only), no mbarrier waits
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
// Copies 16 bytes, or writes 16 zero bytes without reading when !valid.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;\n" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// Sums each of the GP values v[] over the LPR lanes of an aligned lane group
// with a transposed butterfly: at each of the first log2(min(GP, LPR)) levels
// a lane keeps half of the values it carries (the lower half if its level bit
// is clear) and adds the partner's copy of that half, so GP totals cost about
// GP + log2(LPR) shuffles instead of GP * log2(LPR).  On return v[0..NH) hold
// the totals of heads head0(li) .. head0(li) + NH - 1, NH = GP / min(GP, LPR);
// lanes that differ only in the remaining bits hold identical values.
template <int GP, int LPR>
struct GroupSumT {
  static constexpr int SPLIT = GP < LPR ? GP : LPR;
  static constexpr int NH = GP / SPLIT;

  __device__ __forceinline__ static void run(float (&v)[GP], int li) {
    int nh = GP;
#pragma unroll
    for (int o = LPR / 2; o > 0; o >>= 1) {
      if (nh > NH) {
        const bool up = (li & o) != 0;
        const int half = nh / 2;
#pragma unroll
        for (int j = 0; j < GP / 2; ++j) {
          if (j < half) {
            const float mine = up ? v[half + j] : v[j];
            const float other = up ? v[j] : v[half + j];
            v[j] = mine + __shfl_xor_sync(0xffffffffu, other, o);
          }
        }
        nh = half;
      } else {
#pragma unroll
        for (int j = 0; j < NH; ++j) v[j] += __shfl_xor_sync(0xffffffffu, v[j], o);
      }
    }
  }

  __device__ __forceinline__ static int head0(int li) {
    int nh = GP, h = 0;
#pragma unroll
    for (int o = LPR / 2; o > 0; o >>= 1) {
      if (nh > NH) {
        nh /= 2;
        if (li & o) h += nh;
      }
    }
    return h;
  }

  // true on one lane per distinct head set (the lowest such lane)
  __device__ __forceinline__ static bool writer(int li) { return (li % (LPR / SPLIT)) == 0; }
};

// Histogram increment aggregated over the warp: lanes with valid = true add
// one to hist[bin]; lanes that share a bin issue a single atomic (scores
// concentrate in few bins, where per-lane atomics would serialise).  Call
// with the whole warp (warp-uniform control flow).
__device__ __forceinline__ void warp_hist_add(uint32_t* hist, uint32_t bin, bool valid) {
  const unsigned act = __ballot_sync(0xffffffffu, valid);
  if (!act) return;
  const unsigned peers = __match_any_sync(0xffffffffu, valid ? bin : 0xffffffffu) & act;
  const int lane = threadIdx.x & 31;
  if (valid && (peers & ((1u << lane) - 1u)) == 0) atomicAdd(&hist[bin], (uint32_t)__popc(peers));
}

__host__ __device__ __forceinline__ int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

}  // namespace prism
