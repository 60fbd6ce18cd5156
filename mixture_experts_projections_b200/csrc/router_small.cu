// Router for small batches (decode-sized T), one CTA per token
// ("Routing Mamba ..." chapterpal summary page, Knowl 1: p_t = Softmax(x_t W_r),
// S_t = the K largest probabilities, r_{t,i} = p_{t,i} 1[i in S_t]).
//
// With few tokens the chunk-per-CTA routers leave almost every SM idle and
// run d_model sequentially on one SM. Here each token gets a CTA of 8 warps
// that split d_model into 16-byte pieces of the token's row (piece q goes to
// thread q mod 256); the thread reads the matching rows of W_r (E floats per
// feature, contiguous across the warp) straight from L2 and accumulates, in
// float32 FMA and in feature order, the token's partial logits, |x|^2 and
// |w_e|^2. A butterfly over the warp (5 levels) and an ordered sum over the 8
// warps give the logits; every logit has passed through at most
// m + 5 + 8 + 1 roundings (m = the features of one thread), which with |x| and
// |w_e| bounds its error by gamma_n |x| |w_e| (Cauchy-Schwarz). A token whose
// selected logits' lower bounds do not all clear the upper bound of every
// expert ranked after them is re-decided on float64 logits computed by the
// same CTA. Equal logits go to the lower expert index.
// The chunk histograms the dispatch reads are accumulated with integer
// atomics (the launcher zeroes them), so the result is deterministic.
#include <cuda_bf16.h>
#include <math.h>

#include <algorithm>

#include "rom_internal.cuh"

namespace rom {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

template <typename InT>
__device__ __forceinline__ void unpack16(const uint4& v, float (&f)[16 / sizeof(InT)]);

template <>
__device__ __forceinline__ void unpack16<__nv_bfloat16>(const uint4& v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

template <>
__device__ __forceinline__ void unpack16<float>(const uint4& v, float (&f)[4]) {
  f[0] = __uint_as_float(v.x);
  f[1] = __uint_as_float(v.y);
  f[2] = __uint_as_float(v.z);
  f[3] = __uint_as_float(v.w);
}

template <typename InT, int EB>
__global__ void __launch_bounds__(kThreads)
    router_small_kernel(const InT* __restrict__ x, int Dm, const float* __restrict__ w_r,
                        const float* __restrict__ bias, int k, int renorm,
                        int32_t* __restrict__ topk_idx, float* __restrict__ topk_w,
                        int32_t* __restrict__ counts, int32_t* __restrict__ chunk_hist,
                        float gamma) {
  constexpr int kPiece = 16 / static_cast<int>(sizeof(InT));  // features per piece
  constexpr int NV = 2 * EB + 1;  // logits, |w_e|^2, |x|^2
  __shared__ float s_part[kWarps][NV];
  __shared__ double s_part64[kWarps][EB];
  __shared__ float s_l[EB];
  __shared__ int s_refine;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t t = blockIdx.x;
  const uint4* xr = reinterpret_cast<const uint4*>(x + t * Dm);
  // The dispatch that follows may be launched now: its CTAs wait for this
  // grid to complete before they read anything it writes.
  pdl_launch_dependents();
  const int npc = Dm / kPiece;

  float v[NV];
#pragma unroll
  for (int i = 0; i < NV; ++i) v[i] = 0.f;
  for (int q = tid; q < npc; q += kThreads) {
    float f[kPiece];
    unpack16<InT>(__ldg(xr + q), f);
    const float4* wp = reinterpret_cast<const float4*>(w_r + static_cast<int64_t>(q) * kPiece * EB);
#pragma unroll
    for (int j = 0; j < kPiece; ++j) {
      v[2 * EB] = fmaf(f[j], f[j], v[2 * EB]);
#pragma unroll
      for (int e4 = 0; e4 < EB / 4; ++e4) {
        const float4 w = __ldg(wp + j * (EB / 4) + e4);
        const float ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          v[4 * e4 + i] = fmaf(f[j], ws[i], v[4 * e4 + i]);
          v[EB + 4 * e4 + i] = fmaf(ws[i], ws[i], v[EB + 4 * e4 + i]);
        }
      }
    }
  }
#pragma unroll
  for (int i = 0; i < NV; ++i) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v[i] += __shfl_xor_sync(0xffffffffu, v[i], o);
  }
  if (lane == 0)
#pragma unroll
    for (int i = 0; i < NV; ++i) s_part[warp][i] = v[i];
  __syncthreads();

  int sel[kMaxTopK + 1];
  if (tid == 0) {
    float tot[NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      tot[i] = s_part[0][i];
      for (int w = 1; w < kWarps; ++w) tot[i] += s_part[w][i];
    }
    const float xn = sqrtf(tot[2 * EB]);
    float l[EB], err[EB];
#pragma unroll
    for (int e = 0; e < EB; ++e) {
      l[e] = tot[e] + (bias ? __ldg(bias + e) : 0.f);
      err[e] = gamma * xn * sqrtf(tot[EB + e]) + 1.2e-7f * fabsf(l[e]);
      s_l[e] = l[e];
    }
    uint64_t used = 0;
    for (int j = 0; j <= kMaxTopK; ++j) {
      sel[j] = -1;
      if (j <= k) {
        int bi = -1;
        float bv = 0.f;
        for (int e = 0; e < EB; ++e)
          if (!((used >> e) & 1ull) && (bi < 0 || l[e] > bv)) {
            bi = e;
            bv = l[e];
          }
        sel[j] = bi;
        if (bi >= 0) used |= 1ull << bi;
      }
    }
    // The decision is certain when, for every slot j < k, the lower bound of
    // the j-th selected logit lies above the upper bound of EVERY expert
    // ranked after it (not only the next one: the bounds differ per expert
    // through |w_e|, so a lower-ranked expert with a wide bound can reach
    // higher than the one just below).
    bool certain = true;
    uint64_t above = 0;
    for (int j = 0; j < k; ++j) {
      const int a = sel[j];
      above |= 1ull << a;
      const float lb = l[a] - err[a];
#pragma unroll
      for (int e = 0; e < EB; ++e)
        if (!((above >> e) & 1ull) && !(lb > l[e] + err[e])) certain = false;
    }
    s_refine = certain ? 0 : 1;
  }
  __syncthreads();

  if (s_refine) {
    // float64 logits, same split of the row
    double a[EB];
#pragma unroll
    for (int e = 0; e < EB; ++e) a[e] = 0.0;
    for (int q = tid; q < npc; q += kThreads) {
      float f[kPiece];
      unpack16<InT>(__ldg(xr + q), f);
      const float* wp = w_r + static_cast<int64_t>(q) * kPiece * EB;
#pragma unroll
      for (int j = 0; j < kPiece; ++j)
#pragma unroll
        for (int e = 0; e < EB; ++e)
          a[e] = fma(static_cast<double>(f[j]), static_cast<double>(__ldg(wp + j * EB + e)), a[e]);
    }
#pragma unroll
    for (int e = 0; e < EB; ++e) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) a[e] += __shfl_xor_sync(0xffffffffu, a[e], o);
    }
    if (lane == 0)
#pragma unroll
      for (int e = 0; e < EB; ++e) s_part64[warp][e] = a[e];
    __syncthreads();
    if (tid == 0) {
      double l64[EB];
      for (int e = 0; e < EB; ++e) {
        l64[e] = s_part64[0][e];
        for (int w = 1; w < kWarps; ++w) l64[e] += s_part64[w][e];
        l64[e] += bias ? static_cast<double>(bias[e]) : 0.0;
        s_l[e] = static_cast<float>(l64[e]);
      }
      uint64_t used = 0;
      for (int j = 0; j <= kMaxTopK; ++j) {
        sel[j] = -1;
        if (j <= k) {
          int bi = -1;
          double bv = 0.0;
          for (int e = 0; e < EB; ++e)
            if (!((used >> e) & 1ull) && (bi < 0 || l64[e] > bv)) {
              bi = e;
              bv = l64[e];
            }
          sel[j] = bi;
          if (bi >= 0) used |= 1ull << bi;
        }
      }
    }
  }

  if (tid == 0) {
    const float m = s_l[sel[0]];
    float den = 0.f;
    if (renorm) {
      for (int j = 0; j < k; ++j) den += expf(s_l[sel[j]] - m);
    } else {
      for (int e = 0; e < EB; ++e) den += expf(s_l[e] - m);
    }
    const int64_t chunk = t / kChunkTokens;
    for (int j = 0; j < k; ++j) {
      topk_idx[t * k + j] = sel[j];
      topk_w[t * k + j] = expf(s_l[sel[j]] - m) / den;
      if (chunk_hist) atomicAdd(chunk_hist + chunk * EB + sel[j], 1);
      if (counts) atomicAdd(counts + sel[j], 1);
    }
  }
}

template <typename InT, int EB>
cudaError_t launch_eb(const void* x, int64_t T, int Dm, const float* w_r, const float* bias,
                      int k, int renorm, int32_t* topk_idx, float* topk_w, int32_t* counts,
                      int32_t* chunk_hist, cudaStream_t stream) {
  constexpr int kPiece = 16 / static_cast<int>(sizeof(InT));
  cudaError_t err = cudaSuccess;
  if (chunk_hist) {
    err = cudaMemsetAsync(chunk_hist, 0, sizeof(int32_t) * num_chunks(T) * EB, stream);
    if (err != cudaSuccess) return err;
  }
  // Longest rounding chain of a logit: the features of one thread, the warp
  // butterfly, the sum over the warps, the bias (+1 spare); 1 % slack covers
  // the norms.
  const int npc = Dm / kPiece;
  const double m = static_cast<double>((npc + kThreads - 1) / kThreads) * kPiece;
  const double n = m + 5.0 + kWarps + 2.0;
  const double u = 1.0 / 16777216.0;
  const float gamma = static_cast<float>(1.01 * n * u / (1.0 - n * u));
  // The kernel after this one (the projection, or the dispatch) starts as a
  // programmatic dependent while these CTAs run, and it needs most of an SM's
  // shared memory: an SM whose shared-memory carve-out was set small for
  // this kernel could take none of its CTAs until this one left. So these
  // CTAs ask for the largest carve-out.
  err = cudaFuncSetAttribute(router_small_kernel<InT, EB>,
                             cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
  if (err != cudaSuccess) return err;
  router_small_kernel<InT, EB><<<static_cast<unsigned>(T), kThreads, 0, stream>>>(
      static_cast<const InT*>(x), Dm, w_r, bias, k, renorm, topk_idx, topk_w, counts, chunk_hist,
      gamma);
  return cudaGetLastError();
}

template <typename InT>
cudaError_t launch_typed(const void* x, int64_t T, int Dm, const float* w_r, const float* bias,
                         int E, int k, int renorm, int32_t* topk_idx, float* topk_w,
                         int32_t* counts, int32_t* chunk_hist, cudaStream_t stream) {
  switch (E) {
    case 4:
      return launch_eb<InT, 4>(x, T, Dm, w_r, bias, k, renorm, topk_idx, topk_w, counts,
                               chunk_hist, stream);
    case 8:
      return launch_eb<InT, 8>(x, T, Dm, w_r, bias, k, renorm, topk_idx, topk_w, counts,
                               chunk_hist, stream);
    case 16:
      return launch_eb<InT, 16>(x, T, Dm, w_r, bias, k, renorm, topk_idx, topk_w, counts,
                                chunk_hist, stream);
    default:
      return cudaErrorNotSupported;
  }
}

}  // namespace

cudaError_t launch_router_small(const void* x, bool bf16, int64_t T, int Dm, const float* w_r,
                                const float* bias, int E, int k, int renorm, int32_t* topk_idx,
                                float* topk_w, int32_t* counts, int32_t* chunk_hist,
                                cudaStream_t stream) {
  // 16-byte pieces of x and of W_r rows: E in {4, 8, 16}, aligned data.
  const int piece = bf16 ? 8 : 4;
  if (T <= 0 || T > kSmallRouterMaxTokens || Dm % piece != 0 ||
      (reinterpret_cast<uintptr_t>(x) & 15u) || (reinterpret_cast<uintptr_t>(w_r) & 15u))
    return cudaErrorNotSupported;
  if (bf16)
    return launch_typed<__nv_bfloat16>(x, T, Dm, w_r, bias, E, k, renorm, topk_idx, topk_w,
                                       counts, chunk_hist, stream);
  return launch_typed<float>(x, T, Dm, w_r, bias, E, k, renorm, topk_idx, topk_w, counts,
                             chunk_hist, stream);
}

}  // namespace rom
