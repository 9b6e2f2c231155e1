// Cache update and per-token symmetric int8 quantization of the key cache (Prism Attention,
// sec. 4.2 "Quantized Proposal Construction"; int8 per-token scheme because
// the pages do not state their INT2 one).
//
// One row of d elements is spread over d*sizeof(T)/16 lanes, each holding one
// 16-byte vector: a coalesced read of the row, a shuffle max for amax, IEEE
// divisions and round-half-even, one 8- or 4-byte store of codes per lane.
// HBM bound: reads d*sizeof(T) and writes d + 4 bytes per row.
#include <cuda_fp16.h>

#include "common.cuh"
#include "kernels.h"

namespace prism {

template <typename T, int D>
__global__ void __launch_bounds__(256) quantize_kernel(const T* __restrict__ k,
                                                       int8_t* __restrict__ kq,
                                                       float* __restrict__ scale, int64_t T_tok,
                                                       int Hkv, const int32_t* __restrict__ tok_rows,
                                                       int64_t n_rows, int32_t* status) {
  constexpr int E = Vec16<T>::E;
  constexpr int LPR = D / E;  // lanes per row
  constexpr int RPW = 32 / LPR;
  const int lane = threadIdx.x & 31;
  const int sub = lane / LPR, li = lane % LPR;
  const int64_t rows_total = (int64_t)Hkv * n_rows;
  const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t base = warp0 * RPW; base < rows_total; base += nwarps * RPW) {
    const int64_t r = base + sub;
    bool valid = r < rows_total;
    int64_t row = 0;
    if (valid) {
      const int64_t h = r / n_rows, i = r - h * n_rows;
      const int64_t t = tok_rows ? (int64_t)tok_rows[i] : i;
      if (t < 0 || t >= T_tok) {
        if (li == 0) flag_status(status, PRISM_DEV_BAD_INDEX);
        valid = false;
      }
      row = h * T_tok + t;
    }
    float f[E];
    if (valid) {
      Vec16<T>::unpack(ld16_stream(k + row * D + li * E), f);
    } else {
#pragma unroll
      for (int e = 0; e < E; ++e) f[e] = 0.0f;
    }
    float amax = 0.0f;
#pragma unroll
    for (int e = 0; e < E; ++e) amax = fmaxf(amax, fabsf(f[e]));
#pragma unroll
    for (int o = LPR / 2; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float s = __fdiv_rn(amax, 127.0f);
    uint32_t packed[E / 4];
#pragma unroll
    for (int w = 0; w < E / 4; ++w) {
      uint32_t acc = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        int c = 0;
        if (amax != 0.0f) {
          float y = rintf(__fdiv_rn(f[w * 4 + e], s));
          y = fminf(fmaxf(y, -127.0f), 127.0f);
          c = (int)y;
        }
        acc |= ((uint32_t)(c & 0xFF)) << (8 * e);
      }
      packed[w] = acc;
    }
    if (valid) {
      int8_t* dst = kq + row * D + li * E;
      if constexpr (E == 8) {
        *reinterpret_cast<uint2*>(dst) = make_uint2(packed[0], packed[1]);
      } else {
        *reinterpret_cast<uint32_t*>(dst) = packed[0];
      }
      if (li == 0) scale[row] = (amax != 0.0f) ? s : 0.0f;
    }
  }
}

// Write the new token row of every (sequence, KV head): one 16-byte vector
// per thread, rows of k_new / v_new to packed row cu[b+1] - 1.
template <int VEC_PER_ROW>
__global__ void __launch_bounds__(256) append_kernel(const uint4* __restrict__ k_new,
                                                     const uint4* __restrict__ v_new,
                                                     uint4* __restrict__ k_cache,
                                                     uint4* __restrict__ v_cache,
                                                     const int32_t* __restrict__ cu, int B, int Hkv,
                                                     int64_t T_tok) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t per_seq = (int64_t)Hkv * VEC_PER_ROW;
  if (i >= (int64_t)B * per_seq) return;
  const int b = (int)(i / per_seq);
  const int64_t r = i - (int64_t)b * per_seq;
  const int h = (int)(r / VEC_PER_ROW), c = (int)(r % VEC_PER_ROW);
  const int end = cu[b + 1];
  if (end <= cu[b]) return;
  const int64_t dst = ((int64_t)h * T_tok + end - 1) * VEC_PER_ROW + c;
  k_cache[dst] = k_new[i];
  v_cache[dst] = v_new[i];
}

cudaError_t launch_append(const Dims& d, const void* k_new, const void* v_new, void* k_cache,
                          void* v_cache, cudaStream_t st) {
  const int vec = d.D * (d.bf16 ? 2 : 4) / 16;
  const int64_t n = (int64_t)d.B * d.Hkv * vec;
  if (n == 0) return cudaSuccess;
  const unsigned blocks = (unsigned)cdiv(n, 256);
  auto* kn = static_cast<const uint4*>(k_new);
  auto* vn = static_cast<const uint4*>(v_new);
  auto* kc = static_cast<uint4*>(k_cache);
  auto* vc = static_cast<uint4*>(v_cache);
  switch (vec) {
    case 8: append_kernel<8><<<blocks, 256, 0, st>>>(kn, vn, kc, vc, d.cu_dev, d.B, d.Hkv, d.T); break;
    case 16: append_kernel<16><<<blocks, 256, 0, st>>>(kn, vn, kc, vc, d.cu_dev, d.B, d.Hkv, d.T); break;
    default: append_kernel<32><<<blocks, 256, 0, st>>>(kn, vn, kc, vc, d.cu_dev, d.B, d.Hkv, d.T); break;
  }
  return cudaGetLastError();
}

template <typename T, int D>
static cudaError_t run(const Dims& d, const void* k, int8_t* kq, float* scale, const int32_t* tok,
                       int64_t n_rows, int32_t* status, cudaStream_t st) {
  constexpr int LPR = D / Vec16<T>::E;
  const int64_t rows = (int64_t)d.Hkv * n_rows;
  const int64_t warps = cdiv(rows, 32 / LPR);
  int64_t blocks = cdiv(warps, 8);
  const int64_t cap = (int64_t)d.num_sms * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  quantize_kernel<T, D><<<(unsigned)blocks, 256, 0, st>>>(
      static_cast<const T*>(k), kq, scale, d.T, d.Hkv, tok, n_rows, status);
  return cudaGetLastError();
}

cudaError_t launch_quantize(const Dims& d, const void* k, int8_t* kq, float* scale,
                            const int32_t* tok_rows, int64_t n_rows, int32_t* status,
                            cudaStream_t st) {
  if (n_rows == 0 || d.Hkv == 0) return cudaSuccess;
  if (d.bf16) {
    return d.D == 128 ? run<__nv_bfloat16, 128>(d, k, kq, scale, tok_rows, n_rows, status, st)
                      : run<__nv_bfloat16, 64>(d, k, kq, scale, tok_rows, n_rows, status, st);
  }
  return d.D == 128 ? run<float, 128>(d, k, kq, scale, tok_rows, n_rows, status, st)
                    : run<float, 64>(d, k, kq, scale, tok_rows, n_rows, status, st);
}

// ---- INT2 proposal keys ------------------------------------------------------
// Per (KV head, token) and per group of 32 consecutive features (sec. 4.2
// names INT2 for the proposal key cache; this is the scheme the library
// defines for it): L = fp16(min), S = fp16((max - L) / 3) and
// c = clamp(rne((k - L) / S), 0, 3) (all codes 0 when S is 0), with the
// same IEEE operations in the same order as the definition, so codes and
// (S, L) are bit-exact.  One warp per group: lane j holds feature j, a
// shuffle min/max, four lanes' codes packed per byte (feature f at bits
// 2 (f mod 4) of byte f / 4), (S, L) as fp16 bits.
template <typename T, int D>
__global__ void __launch_bounds__(256) quantize_int2_kernel(const T* __restrict__ k,
                                                            uint8_t* __restrict__ codes,
                                                            uint16_t* __restrict__ params,
                                                            int64_t T_tok, int Hkv,
                                                            const int32_t* __restrict__ tok_rows,
                                                            int64_t n_rows, int32_t* status) {
  constexpr int NG = D / 32;
  const int lane = threadIdx.x & 31;
  const int64_t groups = (int64_t)Hkv * n_rows * NG;
  const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t gi = warp0; gi < groups; gi += nwarps) {  // warp-uniform
    const int64_t r = gi / NG;
    const int grp = (int)(gi - r * NG);
    const int64_t h = r / n_rows, i = r - h * n_rows;
    const int64_t t = tok_rows ? (int64_t)tok_rows[i] : i;
    if (t < 0 || t >= T_tok) {
      if (lane == 0 && grp == 0) flag_status(status, PRISM_DEV_BAD_INDEX);
      continue;
    }
    const int64_t row = h * T_tok + t;
    float x;
    if constexpr (sizeof(T) == 2) {
      x = __bfloat162float(k[row * D + grp * 32 + lane]);
    } else {
      x = k[row * D + grp * 32 + lane];
    }
    float lo = x, hi = x;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
      hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    lo = __fadd_rn(lo, 0.0f);  // -0 is taken as +0 (unique fp16 bits)
    hi = __fadd_rn(hi, 0.0f);
    const __half lo_h = __float2half_rn(lo);
    const float L = __half2float(lo_h);
    const __half s_h = __float2half_rn(__fdiv_rn(__fsub_rn(hi, L), 3.0f));
    const float S = __half2float(s_h);
    int c = 0;
    if (S > 0.0f) c = (int)fminf(fmaxf(rintf(__fdiv_rn(__fsub_rn(x, L), S)), 0.0f), 3.0f);
    uint32_t b = (uint32_t)c;
    b |= (uint32_t)__shfl_down_sync(0xffffffffu, c, 1) << 2;
    b |= (uint32_t)__shfl_down_sync(0xffffffffu, c, 2) << 4;
    b |= (uint32_t)__shfl_down_sync(0xffffffffu, c, 3) << 6;
    if ((lane & 3) == 0) codes[row * (D / 4) + grp * 8 + (lane >> 2)] = (uint8_t)b;
    if (lane == 0) {
      params[(row * NG + grp) * 2] = __half_as_ushort(s_h);
      params[(row * NG + grp) * 2 + 1] = __half_as_ushort(lo_h);
    }
  }
}

template <typename T, int D>
static cudaError_t run_int2(const Dims& d, const void* k, uint8_t* codes, uint16_t* params,
                            const int32_t* tok, int64_t n_rows, int32_t* status, cudaStream_t st) {
  const int64_t groups = (int64_t)d.Hkv * n_rows * (D / 32);
  int64_t blocks = cdiv(groups, 8);
  const int64_t cap = (int64_t)d.num_sms * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  quantize_int2_kernel<T, D><<<(unsigned)blocks, 256, 0, st>>>(
      static_cast<const T*>(k), codes, params, d.T, d.Hkv, tok, n_rows, status);
  return cudaGetLastError();
}

cudaError_t launch_quantize_int2(const Dims& d, const void* k, uint8_t* codes, uint16_t* params,
                                 const int32_t* tok_rows, int64_t n_rows, int32_t* status,
                                 cudaStream_t st) {
  if (n_rows == 0 || d.Hkv == 0) return cudaSuccess;
  if (d.bf16) {
    return d.D == 128 ? run_int2<__nv_bfloat16, 128>(d, k, codes, params, tok_rows, n_rows, status, st)
                      : run_int2<__nv_bfloat16, 64>(d, k, codes, params, tok_rows, n_rows, status, st);
  }
  return d.D == 128 ? run_int2<float, 128>(d, k, codes, params, tok_rows, n_rows, status, st)
                    : run_int2<float, 64>(d, k, codes, params, tok_rows, n_rows, status, st);
}

}  // namespace prism
