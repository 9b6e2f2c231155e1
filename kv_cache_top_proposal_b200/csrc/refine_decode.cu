// Refined layer, fused: exact rescoring of the candidate pool, top-kappa
// selection inside it, and sparse flash-decode over the selected rows, in one
// launch per layer (Prism Attention, sec. 4.1 "Proposal-Refined Index
// Sharing": each refined layer re-selects its own top-kappa inside the pool;
// sec. 1 / 2.1: token-level sparse attention over the selected tokens).
//
// One thread-block cluster of CL CTAs owns one (sequence, KV head) row.  CTA
// c takes a contiguous slice of the row's pool (mc members at most):
//   1. the slice's key rows stream into a ring of shared-memory stages with
//      cp.async (all stages in flight at once); lane groups compute the exact
//      dot product with every query head of the group (a transposed butterfly
//      reduction), keeping the logits and the selection key
//      ord(max_g q_g . k) in shared memory;
//   2. the cluster finds the exact kappa-th largest key by an MSD radix
//      select (11/11/10-bit digits): CTAs push their non-zero histogram bins
//      into rank 0's shared memory (distributed shared memory atomics), rank 0
//      locates the digit, every CTA reads it back;
//   3. every CTA marks its selected members (keys above the threshold, plus
//      the lowest-position members equal to it) and writes their positions to
//      idx in ascending order (per-CTA counts exchanged over DSMEM);
//   4. softmax partial over the selected members: the logits are already on
//      chip, so the CTA maximum and the weights 2^(l - m) are computed first
//      and only the value rows are streamed (same cp.async ring);
//   5. the CL partials (m, l, o) are merged through DSMEM, each CTA merging a
//      slice of the G*d outputs, and out / lse are written directly.
// Nothing goes to global scratch.  Bytes per row: kappa_p key rows and kappa
// value rows, d * sizeof(T) each.
#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.h"

namespace cg = cooperative_groups;

namespace prism {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kStages = 4;

// bytes of one pipeline stage (kStages are in flight)
template <int GP>
struct Stage {
  static constexpr int BYTES = GP <= 4 ? 32768 : 16384;
};

struct RDArgs {
  const void* q;
  const void* k;
  const void* v;
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
};

// Streams `rows` cache rows (row j at position spos[list ? list[j] : j] of
// base; negative positions are zero-filled without reading) through the
// stage ring and calls body(first_row, stage, rows_in_chunk) once per chunk
// of SR rows, with kStages chunks in flight.
template <typename T, int D, int GP, typename Body>
__device__ __forceinline__ void stream_rows(const T* base, const int* spos, const int* list,
                                            int rows, unsigned char* stage, Body body) {
  constexpr int RB = D * (int)sizeof(T);  // row bytes
  constexpr int VPR = RB / 16;            // 16-byte vectors per row
  constexpr int SR = Stage<GP>::BYTES / RB;
  const int tid = threadIdx.x;
  const int nchunk = (rows + SR - 1) / SR;
  auto issue = [&](int c) {
    if (c < nchunk) {
      const int r0 = c * SR, n = min(SR, rows - r0);
      unsigned char* buf = stage + (c % kStages) * Stage<GP>::BYTES;
      for (int x = tid; x < n * VPR; x += kThreads) {
        const int r = x / VPR, vv = x - r * VPR;
        const int pos = spos[list ? list[r0 + r] : r0 + r];
        const T* src = base + (int64_t)(pos >= 0 ? pos : 0) * D + vv * (16 / (int)sizeof(T));
        cp_async16(smem_u32(buf + r * RB + vv * 16), src, pos >= 0);
      }
    }
    cp_async_commit();  // one group per call (possibly empty): constant wait depth
  };
#pragma unroll
  for (int c = 0; c < kStages; ++c) issue(c);
  for (int c = 0; c < nchunk; ++c) {
    cp_async_wait<kStages - 1>();
    __syncthreads();
    body(c * SR, stage + (c % kStages) * Stage<GP>::BYTES, min(SR, rows - c * SR));
    __syncthreads();
    issue(c + kStages);
  }
  cp_async_wait<0>();
}

template <typename T, int D, int GP>
__global__ void __launch_bounds__(kThreads, 1) refine_decode_kernel(const RDArgs a) {
  constexpr int E = Vec16<T>::E;
  constexpr int LPR = D / E;     // lanes per cache row
  constexpr int RPW = 32 / LPR;  // rows per warp
  constexpr int NG = kThreads / LPR;  // lane groups per CTA
  constexpr int RB = D * (int)sizeof(T);
  using GS = GroupSumT<GP, LPR>;

  extern __shared__ __align__(16) unsigned char dsm[];
  unsigned char* stage = dsm;                                              // kStages stages
  int* spos = reinterpret_cast<int*>(dsm + kStages * Stage<GP>::BYTES);    // [mc]
  uint32_t* keys = reinterpret_cast<uint32_t*>(spos + a.mc);               // [mc]
  float* dots = reinterpret_cast<float*>(keys + a.mc);                     // [GP][mc]
  float* pw = dots + GP * a.mc;                                            // [mc][GP] weights
  int* sel = reinterpret_cast<int*>(pw + GP * a.mc);                       // [mc]
  float* comb = reinterpret_cast<float*>(stage);  // [kWarps][GP][D], after the value pass

  __shared__ uint32_t ghist[2][2048];  // cluster histogram (used in rank 0)
  __shared__ uint32_t lh[2048];        // this CTA's histogram
  __shared__ int scratch[33];
  __shared__ int s_res[2];             // rank 0: digit, count above it
  __shared__ int s_cnt[2];             // published: #equal, #greater
  __shared__ int s_before[2];
  __shared__ float s_red[kWarps][GP];
  __shared__ float part_o[GP * D];     // published partial
  __shared__ float part_m[GP], part_l[GP];

  cg::cluster_group cluster = cg::this_cluster();
  const int CL = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const int row = blockIdx.x / CL;
  const int b = row / a.Hkv, h = row - b * a.Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int sub = lane / LPR, li = lane % LPR;

  const int t0 = a.cu[b];
  const int L = a.cu[b + 1] - t0;
  int n = a.pool_cnt[row];
  if (n < 0 || n > a.kp) {
    if (rank == 0 && tid == 0) flag_status(a.status, PRISM_DEV_BAD_INDEX);
    n = n < 0 ? 0 : a.kp;
  }
  const int k = min(a.kappa, n);
  const int chunk = (n + CL - 1) / CL;
  const int lo = min(n, rank * chunk), hi = min(n, lo + chunk);
  const int m = hi - lo;
  const int32_t* pool = a.pool + (int64_t)row * a.kp + lo;
  const int64_t rowbase = ((int64_t)h * a.T + t0) * D;
  const T* kb = static_cast<const T*>(a.k) + rowbase;
  const T* vb = static_cast<const T*>(a.v) + rowbase;

  // ---- 0. the slice's positions (an out-of-range one is flagged, skipped)
  for (int i = tid; i < m; i += kThreads) {
    const int p = pool[i];
    const bool ok = p >= 0 && p < L;
    if (!ok) flag_status(a.status, PRISM_DEV_BAD_INDEX);
    spos[i] = ok ? p : -1;
  }
  if (rank == 0)
    for (int i = tid; i < 2048; i += kThreads) ghist[0][i] = 0;
  __syncthreads();

  // ---- 1. exact scores of the slice
  {
    float qf[GP][E];
    const T* q = static_cast<const T*>(a.q) + ((int64_t)b * a.Hq + (int64_t)h * a.G) * D + li * E;
#pragma unroll
    for (int g = 0; g < GP; ++g) {
      if (g < a.G) {
        Vec16<T>::unpack(ld16(q + (int64_t)g * D), qf[g]);
      } else {
#pragma unroll
        for (int e = 0; e < E; ++e) qf[g][e] = 0.0f;
      }
    }
    const int h0 = GS::head0(li);
    stream_rows<T, D, GP>(kb, spos, nullptr, m, stage,
                          [&](int r0, const unsigned char* buf, int nrows) {
      // warp-uniform trip count: the reduction shuffles over the whole warp
      for (int wb = warp * RPW; wb < nrows; wb += NG) {
        const int r = wb + sub;
        const bool in = r < nrows;
        float f[E];
        Vec16<T>::unpack(in ? *reinterpret_cast<const uint4*>(buf + r * RB + li * 16)
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
          if (h0 + j < a.G) best = fmaxf(best, acc[j]);
#pragma unroll
        for (int o = LPR / 2; o >= LPR / GS::SPLIT && o > 0; o >>= 1)
          best = fmaxf(best, __shfl_xor_sync(0xffffffffu, best, o));
        if (in) {
          const int i = r0 + r;
          const bool ok = spos[i] >= 0;  // an out-of-range position ranks last, weighs 0
          if (GS::writer(li)) {
#pragma unroll
            for (int j = 0; j < GS::NH; ++j) dots[(h0 + j) * a.mc + i] = ok ? acc[j] : -INFINITY;
          }
          if (li == 0) keys[i] = ord_key(ok ? best : -INFINITY);
        }
      }
    });
  }
  cluster.sync();  // scores of every slice ready; rank 0's histogram cleared

  // ---- 2. cluster radix select of the kappa-th largest key
  const bool radix = n > a.kappa;
  uint32_t thr = 0;
  int krem = 0;
  if (radix) {
    uint32_t prefix = 0, pmask = 0;
    krem = k;
#pragma unroll 1
    for (int pass = 0; pass < 3; ++pass) {
      const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
      const int nb = pass == 2 ? 1024 : 2048;
      for (int i = tid; i < nb; i += kThreads) lh[i] = 0;
      __syncthreads();
      for (int i = tid; i < m; i += kThreads) {
        const uint32_t key = keys[i];
        if ((key & pmask) == prefix) atomicAdd(&lh[(key >> shift) & (nb - 1)], 1u);
      }
      __syncthreads();
      uint32_t* g0 = cluster.map_shared_rank(&ghist[pass & 1][0], 0);
      for (int i = tid; i < nb; i += kThreads) {
        const uint32_t c = lh[i];
        if (c) atomicAdd(g0 + i, c);
      }
      cluster.sync();  // every push of this pass has landed in rank 0
      if (rank == 0) {
        const uint32_t* gh = ghist[pass & 1];
        const int per = nb / kThreads;
        int v = 0;
        for (int j = 0; j < per; ++j) v += (int)gh[tid * per + j];
        int total;
        const int excl = block_excl_scan(v, scratch, &total);
        int above = total - excl - v;
        for (int j = per - 1; j >= 0; --j) {
          const int c = (int)gh[tid * per + j];
          if (above < krem && krem <= above + c) {
            s_res[0] = tid * per + j;
            s_res[1] = above;
          }
          above += c;
        }
        if (pass < 2)
          for (int i = tid; i < 2048; i += kThreads) ghist[(pass + 1) & 1][i] = 0;
      }
      cluster.sync();  // rank 0's answer is ready
      if (tid == 0) {
        const int* r0 = cluster.map_shared_rank(s_res, 0);
        s_before[0] = r0[0];
        s_before[1] = r0[1];
      }
      __syncthreads();
      prefix |= (uint32_t)s_before[0] << shift;
      pmask |= (uint32_t)(nb - 1) << shift;
      krem -= s_before[1];
      __syncthreads();
    }
    thr = prefix;
  }

  // ---- 3. selected members of the slice, positions to idx (ascending)
  const int per = (m + kThreads - 1) / kThreads;
  const int i0 = min(m, tid * per), i1 = min(m, i0 + per);
  int gt = 0, eq = 0;
  for (int i = i0; i < i1; ++i) {
    const uint32_t key = keys[i];
    if (!radix || key > thr) ++gt;
    else if (key == thr) ++eq;
  }
  int eq_tot, gt_tot;
  const int eq_pre = block_excl_scan(eq, scratch, &eq_tot);
  block_excl_scan(gt, scratch, &gt_tot);
  if (tid == 0) {
    s_cnt[0] = eq_tot;
    s_cnt[1] = gt_tot;
  }
  cluster.sync();
  if (warp == 0) {
    // lane r < rank reads rank r's counts; members equal to the threshold go
    // to the lowest ranks first (lower positions win)
    int e = 0, g = 0;
    if (lane < rank) {
      const int* c = cluster.map_shared_rank(s_cnt, lane);
      e = c[0];
      g = c[1];
    }
    const int einc = warp_incl_scan(e);
    const int take_r = max(0, min(krem - (einc - e), e));
    int sb = g + take_r, eb = e;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      sb += __shfl_xor_sync(0xffffffffu, sb, o);
      eb += __shfl_xor_sync(0xffffffffu, eb, o);
    }
    if (lane == 0) {
      s_before[0] = eb;
      s_before[1] = sb;
    }
  }
  __syncthreads();
  const int take = radix ? max(0, min(krem - (s_before[0] + eq_pre), eq)) : 0;
  int nsel;
  const int sel_pre = block_excl_scan(gt + take, scratch, &nsel);
  {
    int o = sel_pre, taken = 0;
    int32_t* idx = a.idx + (int64_t)row * a.kappa;
    for (int i = i0; i < i1; ++i) {
      const uint32_t key = keys[i];
      bool s = !radix || key > thr;
      if (radix && key == thr) s = taken++ < take;
      if (s) {
        const int slot = s_before[1] + o;
        if (slot < k) idx[slot] = pool[i];
        else flag_status(a.status, PRISM_DEV_TOO_LONG);  // unreachable if counts are right
        sel[o++] = i;
      }
    }
    for (int s = k + rank * kThreads + tid; s < a.kappa; s += CL * kThreads) idx[s] = -1;
    if (rank == 0 && tid == 0) a.cnt[row] = k;
  }
  __syncthreads();

  // ---- 4. softmax partial over the selected members of the slice
  float mx[GP];
#pragma unroll
  for (int g = 0; g < GP; ++g) mx[g] = -INFINITY;
  for (int j = tid; j < nsel; j += kThreads) {
    const int i = sel[j];
#pragma unroll
    for (int g = 0; g < GP; ++g) mx[g] = fmaxf(mx[g], dots[g * a.mc + i]);
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
      const float l = dots[g * a.mc + i];
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
  float o[GP][E];
#pragma unroll
  for (int g = 0; g < GP; ++g)
#pragma unroll
    for (int e = 0; e < E; ++e) o[g][e] = 0.0f;
  // stream the selected value rows (the weights are read after the first
  // stage barrier inside stream_rows)
  stream_rows<T, D, GP>(vb, spos, sel, nsel, stage,
                        [&](int j0, const unsigned char* buf, int nrows) {
    for (int r = warp * RPW + sub; r < nrows; r += NG) {
      float f[E];
      Vec16<T>::unpack(*reinterpret_cast<const uint4*>(buf + r * RB + li * 16), f);
      const float* p = pw + (j0 + r) * GP;
#pragma unroll
      for (int g = 0; g < GP; ++g) {
        const float pg = p[g];
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
  __syncthreads();  // the stage ring is free: reuse it for the warp partials
  if (sub == 0) {
#pragma unroll
    for (int g = 0; g < GP; ++g)
#pragma unroll
      for (int e = 0; e < E; ++e) comb[(warp * GP + g) * D + li * E + e] = o[g][e];
  }
  __syncthreads();
  for (int i = tid; i < GP * D; i += kThreads) {
    float s = 0.0f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) s += comb[w * GP * D + i];
    part_o[i] = s;
  }
  if (tid < GP) {
    float s = 0.0f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) s += s_red[w][tid];
    part_l[tid] = s;
    part_m[tid] = mx[tid];
  }
  cluster.sync();  // every CTA's partial is published

  // ---- 5. merge the CL partials; CTA c merges outputs [c*per_c, ...).
  // CL consecutive lanes handle one output, lane r reading rank r's partial,
  // so every remote load of an iteration is in flight at once.
  {
    const int nout = a.G * D;
    const int per_c = (nout + CL - 1) / CL;
    const int r = tid % CL;
    const int first = rank * per_c, last = min(nout, first + per_c);
    for (int base = 0; base < per_c; base += kThreads / CL) {  // uniform trip count
      const int i = first + base + tid / CL;
      const bool live = base + tid / CL < per_c && i < last;
      const int ii = live ? i : first;
      const int g = ii / D, j = ii - g * D;
      const float mr = cluster.map_shared_rank(part_m, r)[g];
      const float lr = cluster.map_shared_rank(part_l, r)[g];
      const float orr = cluster.map_shared_rank(part_o, r)[ii];
      float M = mr;
      for (int s = 1; s < CL; s <<= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, s));
      const float w = (mr == -INFINITY) ? 0.0f : exp2f(mr - M);
      float Ls = w * lr, O = w * orr;
      for (int s = 1; s < CL; s <<= 1) {
        Ls += __shfl_xor_sync(0xffffffffu, Ls, s);
        O += __shfl_xor_sync(0xffffffffu, O, s);
      }
      if (live && r == 0) {
        const int64_t hq = (int64_t)b * a.Hq + (int64_t)h * a.G + g;
        a.out[hq * D + j] = Ls > 0.0f ? O / Ls : 0.0f;
        if (j == 0 && a.lse)
          a.lse[hq] = Ls > 0.0f ? (M + log2f(Ls)) * 0.69314718055994530942f : -INFINITY;
      }
    }
  }
  cluster.sync();  // keep shared memory alive until every remote read is done
}

template <int GP>
constexpr int per_member_bytes() {
  return (int)(2 * sizeof(int) + sizeof(uint32_t) + 2 * GP * sizeof(float));
}

template <int GP>
int smem_bytes(int mc) {
  return kStages * Stage<GP>::BYTES + mc * per_member_bytes<GP>();
}

// dynamic shared memory available next to the kernel's static arrays
constexpr int kDynBudget = 227 * 1024 - 40 * 1024;

template <typename T, int D, int GP>
cudaError_t run(const Dims& d, RDArgs a, int cl, cudaStream_t st) {
  auto kern = refine_decode_kernel<T, D, GP>;
  const int smem = smem_bytes<GP>(a.mc);
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

int slice_capacity(int GP) {
  const int stages = kStages * (GP <= 4 ? 32768 : 16384);
  const int per = (int)(2 * sizeof(int) + sizeof(uint32_t) + 2 * GP * sizeof(float));
  return (kDynBudget - stages) / per;
}

}  // namespace

RefineDecodePlan plan_refine_decode(const Dims& d, int kappa_p) {
  const int rows = d.B * d.Hkv;
  const int GP = padded_group(d.G);
  int cl = 1;
  while (cl < 16 && (int64_t)rows * cl < d.num_sms) cl *= 2;
  const int cap = slice_capacity(GP);
  while (cl < 16 && (kappa_p + cl - 1) / cl > cap) cl *= 2;
  const int mc = (kappa_p + cl - 1) / cl;
  return RefineDecodePlan{cl, mc, mc <= cap};
}

cudaError_t launch_refine_decode(const Dims& d, const RefineDecodePlan& p, const void* q,
                                 const void* k, const void* v, const int32_t* pool,
                                 const int32_t* pool_cnt, int kappa_p, int kappa,
                                 float softmax_scale, int32_t* idx, int32_t* cnt, float* out,
                                 float* lse, int32_t* status, cudaStream_t st) {
  if (d.B * d.Hkv == 0) return cudaSuccess;
  RDArgs a{q, k, v, d.cu_dev, pool, pool_cnt, kappa_p, kappa, d.Hkv, d.G, d.Hq, d.T, p.mc,
           softmax_scale * 1.4426950408889634f, idx, cnt, out, lse, status};
  if (d.bf16)
    return d.D == 128 ? by_group<__nv_bfloat16, 128>(d, a, p.cluster, st)
                      : by_group<__nv_bfloat16, 64>(d, a, p.cluster, st);
  return d.D == 128 ? by_group<float, 128>(d, a, p.cluster, st)
                    : by_group<float, 64>(d, a, p.cluster, st);
}

}  // namespace prism
