// Router of the RoM block: logits x_t W_r (+ bias), softmax, top-k selection
// and the per-chunk expert histogram, fused in one kernel.
// ("Routing Mamba ..." chapterpal summary page, Knowl 1: p_t = Softmax(x_t W_r),
// S_t = the K largest probabilities, r_{t,i} = p_{t,i} 1[i in S_t].)
//
// Work split: a CTA of 8 warps owns a chunk of 128 tokens; a warp handles
// TPW tokens at a time, its 32 lanes splitting d_model into 16-byte slices.
// Each lane accumulates its slice sequentially in float32 FMA, then a 5-level
// xor butterfly sums the lanes (every lane ends with the identical sum).
// The same pass accumulates |x|^2, which with the per-expert |w_e| gives the
// Cauchy-Schwarz bound sum_i |x_i w_ie| <= |x| |w_e| and hence a rigorous
// bound gamma_n |x| |w_e| on the rounding error of each float32 logit
// (n = the longest accumulation chain, gamma_n = n u / (1 - n u)).
// If a gap that decides S_t or its slot order is not larger than the two
// bounds, the warp recomputes that token's logits in float64 before deciding.
// The routing decision is therefore the one exact arithmetic would take,
// except for gaps below the float64 rounding level.
#include <cuda_bf16.h>
#include <math.h>

#include <algorithm>

#include "rom_internal.cuh"

namespace rom {
namespace {

constexpr int kRouterThreads = 256;
constexpr int kRouterWarps = kRouterThreads / 32;

template <typename InT>
struct Vec;
template <>
struct Vec<__nv_bfloat16> {
  static constexpr int V = 8;
};
template <>
struct Vec<float> {
  static constexpr int V = 4;
};

// 16 bytes of x (8 bf16 or 4 float) -> float.
__device__ __forceinline__ void load16(const __nv_bfloat16* p, float (&f)[8]) {
  const uint4 v = __ldg(reinterpret_cast<const uint4*>(p));
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}
__device__ __forceinline__ void load16(const float* p, float (&f)[4]) {
  const float4 v = __ldg(reinterpret_cast<const float4*>(p));
  f[0] = v.x;
  f[1] = v.y;
  f[2] = v.z;
  f[3] = v.w;
}

// W_r value of expert e at feature d: from the transposed shared copy
// [EB][Dm] or from the global [Dm][E] array.
template <bool SMEM_W>
__device__ __forceinline__ float wval(const float* sW, const float* w_r, int Dm, int E, int e,
                                      int d) {
  return SMEM_W ? sW[e * Dm + d] : __ldg(w_r + static_cast<int64_t>(d) * E + e);
}

// Top-(k+1) scan over EB values: slot j gets the j-th largest (equal values:
// lower index first); idx[k] is the best unselected expert (or -1).
template <int EB, typename VT>
__device__ __forceinline__ void select_topk(const VT (&l)[EB], int E, int k,
                                            int (&idx)[kMaxTopK + 1]) {
  uint64_t used = 0;
#pragma unroll
  for (int j = 0; j <= kMaxTopK; ++j) {
    idx[j] = -1;
    if (j <= k) {
      int bi = -1;
      VT bv = 0;
#pragma unroll
      for (int e = 0; e < EB; ++e) {
        if (e < E && !((used >> e) & 1ull) && (bi < 0 || l[e] > bv)) {
          bi = e;
          bv = l[e];
        }
      }
      idx[j] = bi;
      if (bi >= 0) used |= 1ull << bi;
    }
  }
}

template <int EB>
__device__ __forceinline__ float pick(const float (&a)[EB], int e) {
  float r = 0.f;
#pragma unroll
  for (int i = 0; i < EB; ++i) r = (i == e) ? a[i] : r;
  return r;
}

// float64 logits of one token, computed by the whole warp; written to out[0..E).
template <typename InT, int EB, bool SMEM_W>
__device__ __noinline__ void refine_logits_f64(const InT* __restrict__ xrow, int Dm,
                                               const float* sW, const float* w_r,
                                               const float* bias, int E, double* out,
                                               int lane) {
  constexpr int V = Vec<InT>::V;
  constexpr int G = EB < 16 ? EB : 16;
  for (int e0 = 0; e0 < EB; e0 += G) {
    double a[G];
#pragma unroll
    for (int g = 0; g < G; ++g) a[g] = 0.0;
    for (int d0 = lane * V; d0 < Dm; d0 += 32 * V) {
      float xv[V];
      load16(xrow + d0, xv);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const int e = e0 + g;
        if (e < E) {
#pragma unroll
          for (int v = 0; v < V; ++v)
            a[g] = fma(static_cast<double>(xv[v]),
                       static_cast<double>(wval<SMEM_W>(sW, w_r, Dm, E, e, d0 + v)), a[g]);
        }
      }
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) a[g] += __shfl_xor_sync(0xffffffffu, a[g], off);
    }
    if (lane == 0) {
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const int e = e0 + g;
        if (e < E) out[e] = a[g] + (bias ? static_cast<double>(bias[e]) : 0.0);
      }
    }
  }
  __syncwarp();
}

template <typename InT, int EB, int TPW, bool SMEM_W>
__global__ void __launch_bounds__(kRouterThreads)
    router_kernel(const InT* __restrict__ x, int64_t T, int Dm, const float* __restrict__ w_r,
                  const float* __restrict__ bias, int E, int k, int renorm,
                  int32_t* __restrict__ topk_idx, float* __restrict__ topk_w,
                  int32_t* __restrict__ counts, int32_t* __restrict__ chunk_hist,
                  int64_t nchunks, float gamma) {
  constexpr int V = Vec<InT>::V;
  constexpr int kPasses = kChunkTokens / (kRouterWarps * TPW);
  static_assert(kPasses * kRouterWarps * TPW == kChunkTokens, "chunk geometry");
  extern __shared__ float4 router_smem[];
  float* sW = reinterpret_cast<float*>(router_smem);  // [EB][Dm] when SMEM_W
  __shared__ float s_wnorm[EB];
  __shared__ int s_hist[EB];
  __shared__ double s_l64[kRouterWarps][EB];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  if (SMEM_W) {
    for (int i = tid; i < Dm * E; i += kRouterThreads) sW[(i % E) * Dm + i / E] = w_r[i];
    for (int i = tid; i < Dm * (EB - E); i += kRouterThreads) sW[E * Dm + i] = 0.f;
    __syncthreads();
  }
  for (int e = warp; e < EB; e += kRouterWarps) {
    float s = 0.f;
    if (e < E)
      for (int d = lane; d < Dm; d += 32) {
        const float w = wval<SMEM_W>(sW, w_r, Dm, E, e, d);
        s = fmaf(w, w, s);
      }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (lane == 0) s_wnorm[e] = sqrtf(s);
  }

  for (int64_t c = blockIdx.x; c < nchunks; c += gridDim.x) {
    for (int e = tid; e < EB; e += kRouterThreads) s_hist[e] = 0;
    __syncthreads();
    for (int pass = 0; pass < kPasses; ++pass) {
      const int64_t t0 = c * kChunkTokens + static_cast<int64_t>(pass * kRouterWarps + warp) * TPW;
      float acc[TPW][EB];
      float sq[TPW];
#pragma unroll
      for (int t = 0; t < TPW; ++t) {
        sq[t] = 0.f;
#pragma unroll
        for (int e = 0; e < EB; ++e) acc[t][e] = 0.f;
      }
      for (int d0 = lane * V; d0 < Dm; d0 += 32 * V) {
        float xv[TPW][V];
#pragma unroll
        for (int t = 0; t < TPW; ++t) {
          if (t0 + t < T) {
            load16(x + (t0 + t) * static_cast<int64_t>(Dm) + d0, xv[t]);
          } else {
#pragma unroll
            for (int v = 0; v < V; ++v) xv[t][v] = 0.f;
          }
#pragma unroll
          for (int v = 0; v < V; ++v) sq[t] = fmaf(xv[t][v], xv[t][v], sq[t]);
        }
#pragma unroll
        for (int e = 0; e < EB; ++e) {
          float wv[V];
          if (SMEM_W) {
#pragma unroll
            for (int v4 = 0; v4 < V / 4; ++v4) {
              const float4 q = *reinterpret_cast<const float4*>(sW + e * Dm + d0 + 4 * v4);
              wv[4 * v4] = q.x;
              wv[4 * v4 + 1] = q.y;
              wv[4 * v4 + 2] = q.z;
              wv[4 * v4 + 3] = q.w;
            }
          } else {
#pragma unroll
            for (int v = 0; v < V; ++v) wv[v] = (e < E) ? wval<false>(sW, w_r, Dm, E, e, d0 + v) : 0.f;
          }
#pragma unroll
          for (int t = 0; t < TPW; ++t) {
#pragma unroll
            for (int v = 0; v < V; ++v) acc[t][e] = fmaf(xv[t][v], wv[v], acc[t][e]);
          }
        }
      }
#pragma unroll
      for (int t = 0; t < TPW; ++t) {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
          sq[t] += __shfl_xor_sync(0xffffffffu, sq[t], off);
#pragma unroll
          for (int e = 0; e < EB; ++e) acc[t][e] += __shfl_xor_sync(0xffffffffu, acc[t][e], off);
        }
      }

      // Decisions: warp-uniform, one token at a time.
#pragma unroll
      for (int t = 0; t < TPW; ++t) {
        const int64_t tok = t0 + t;
        if (tok >= T) continue;
        float l[EB], err[EB];
        const float xn = sqrtf(sq[t]);
#pragma unroll
        for (int e = 0; e < EB; ++e) {
          if (e < E) {
            l[e] = acc[t][e] + (bias ? __ldg(bias + e) : 0.f);
            err[e] = gamma * xn * s_wnorm[e] + 1.2e-7f * fabsf(l[e]);
          } else {
            l[e] = -INFINITY;
            err[e] = 0.f;
          }
        }
        int sel[kMaxTopK + 1];
        select_topk<EB, float>(l, E, k, sel);
        bool certain = true;
#pragma unroll
        for (int j = 0; j < kMaxTopK; ++j) {
          if (j < k && sel[j + 1] >= 0) {
            const int a = sel[j], b = sel[j + 1];
            if (!(pick<EB>(l, a) - pick<EB>(l, b) > pick<EB>(err, a) + pick<EB>(err, b)))
              certain = false;
          }
        }
        if (!certain) {
          refine_logits_f64<InT, EB, SMEM_W>(x + tok * static_cast<int64_t>(Dm), Dm, sW, w_r,
                                             bias, E, s_l64[warp], lane);
          double l64[EB];
#pragma unroll
          for (int e = 0; e < EB; ++e) l64[e] = (e < E) ? s_l64[warp][e] : -INFINITY;
          select_topk<EB, double>(l64, E, k, sel);
#pragma unroll
          for (int e = 0; e < EB; ++e) l[e] = (e < E) ? static_cast<float>(l64[e]) : -INFINITY;
          __syncwarp();
        }
        // Softmax in float32 (exp of the shifted logits).
        const float m = pick<EB>(l, sel[0]);
        float den = 0.f;
        if (renorm) {
#pragma unroll
          for (int j = 0; j < kMaxTopK; ++j)
            if (j < k) den += expf(pick<EB>(l, sel[j]) - m);
        } else {
#pragma unroll
          for (int e = 0; e < EB; ++e)
            if (e < E) den += expf(l[e] - m);
        }
        if (lane == 0) {
#pragma unroll
          for (int j = 0; j < kMaxTopK; ++j) {
            if (j < k) {
              topk_idx[tok * k + j] = sel[j];
              topk_w[tok * k + j] = expf(pick<EB>(l, sel[j]) - m) / den;
              atomicAdd(&s_hist[sel[j]], 1);
            }
          }
        }
      }
    }
    __syncthreads();
    for (int e = tid; e < E; e += kRouterThreads) {
      chunk_hist[c * E + e] = s_hist[e];
      if (counts && s_hist[e]) atomicAdd(counts + e, s_hist[e]);
    }
    __syncthreads();
  }
}

template <typename InT, int EB, int TPW>
cudaError_t launch_eb(const InT* x, int64_t T, int Dm, const float* w_r, const float* bias,
                      int E, int k, int renorm, int32_t* topk_idx, float* topk_w,
                      int32_t* counts, int32_t* chunk_hist, cudaStream_t stream) {
  constexpr int V = Vec<InT>::V;
  const int64_t nchunks = num_chunks(T);
  if (nchunks == 0) return cudaSuccess;
  // Longest float32 accumulation chain: the lane's sequential slice, the
  // 5-level butterfly and the bias add (+1 spare); 1 % slack for the norms.
  const double n = static_cast<double>(((Dm + 32 * V - 1) / (32 * V)) * V + 5 + 2);
  const double u = 1.0 / 16777216.0;
  const float gamma = static_cast<float>(1.01 * n * u / (1.0 - n * u));
  const size_t smem_w = static_cast<size_t>(EB) * Dm * sizeof(float);
  const int sms = device_sm_count();
  if (smem_w <= 160 * 1024) {
    auto kern = router_kernel<InT, EB, TPW, true>;
    cudaError_t err =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_w);
    if (err != cudaSuccess) return err;
    int per_sm = 1;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kRouterThreads, smem_w);
    if (per_sm < 1) per_sm = 1;
    const int64_t grid = std::min<int64_t>(nchunks, static_cast<int64_t>(sms) * per_sm);
    kern<<<static_cast<unsigned>(grid), kRouterThreads, smem_w, stream>>>(
        x, T, Dm, w_r, bias, E, k, renorm, topk_idx, topk_w, counts, chunk_hist, nchunks, gamma);
  } else {
    auto kern = router_kernel<InT, EB, TPW, false>;
    const int64_t grid = std::min<int64_t>(nchunks, static_cast<int64_t>(sms) * 4);
    kern<<<static_cast<unsigned>(grid), kRouterThreads, 0, stream>>>(
        x, T, Dm, w_r, bias, E, k, renorm, topk_idx, topk_w, counts, chunk_hist, nchunks, gamma);
  }
  return cudaGetLastError();
}

template <typename InT>
cudaError_t launch_typed(const InT* x, int64_t T, int Dm, const float* w_r, const float* bias,
                         int E, int k, int renorm, int32_t* topk_idx, float* topk_w,
                         int32_t* counts, int32_t* chunk_hist, cudaStream_t stream) {
  if (E <= 4)
    return launch_eb<InT, 4, 4>(x, T, Dm, w_r, bias, E, k, renorm, topk_idx, topk_w, counts,
                                chunk_hist, stream);
  if (E <= 8)
    return launch_eb<InT, 8, 4>(x, T, Dm, w_r, bias, E, k, renorm, topk_idx, topk_w, counts,
                                chunk_hist, stream);
  if (E <= 16)
    return launch_eb<InT, 16, 4>(x, T, Dm, w_r, bias, E, k, renorm, topk_idx, topk_w, counts,
                                 chunk_hist, stream);
  if (E <= 32)
    return launch_eb<InT, 32, 2>(x, T, Dm, w_r, bias, E, k, renorm, topk_idx, topk_w, counts,
                                 chunk_hist, stream);
  return launch_eb<InT, 64, 1>(x, T, Dm, w_r, bias, E, k, renorm, topk_idx, topk_w, counts,
                               chunk_hist, stream);
}

}  // namespace

cudaError_t launch_router(const void* x, bool bf16, int64_t T, int Dm, const float* w_r,
                          const float* bias, int E, int k, int renorm, int32_t* topk_idx,
                          float* topk_w, int32_t* counts, int32_t* chunk_hist, int* /*status*/,
                          cudaStream_t stream) {
  if (bf16)
    return launch_typed(static_cast<const __nv_bfloat16*>(x), T, Dm, w_r, bias, E, k, renorm,
                        topk_idx, topk_w, counts, chunk_hist, stream);
  return launch_typed(static_cast<const float*>(x), T, Dm, w_r, bias, E, k, renorm, topk_idx,
                      topk_w, counts, chunk_hist, stream);
}

}  // namespace rom
