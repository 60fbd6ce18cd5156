// Router of the RoM block: logits x_t W_r (+ bias), softmax, top-k selection
// and the per-chunk expert histogram, fused in one kernel.
// ("Routing Mamba ..." chapterpal summary page, Knowl 1: p_t = Softmax(x_t W_r),
// S_t = the K largest probabilities, r_{t,i} = p_{t,i} 1[i in S_t].)
//
// Work split. A CTA of 16 warps owns a chunk of 128 tokens. A warp takes TPW
// tokens per pass and holds NV = TPW * EB partial logits per lane (EB = the
// expert count rounded up to a power of two); its 32 lanes split d_model so
// that every shared-memory read of the router weight is conflict-free.
// Each lane accumulates its slice sequentially in float32 FMA; a
// transpose-reduce (31 shuffles per 32 values) then leaves lane L holding the
// complete logit of (token, expert) = divmod(i * 32 + L, EB) for each of its
// NV / 32 values. Top-k selection, softmax and the outputs are computed
// lane-parallel over segments of EB lanes with shuffles.
//
// Exactness of the decision. The same pass accumulates |x|^2; with the
// per-expert |w_e| this bounds sum_i |x_i w_ie| <= |x| |w_e| (Cauchy-Schwarz),
// hence the float32 rounding error of each logit by gamma_n |x| |w_e| (+ the
// bias add), n being the longest accumulation chain and
// gamma_n = n u / (1 - n u). If the lower bound of some selected logit does
// not clear the upper bound of every expert ranked after it, the warp
// recomputes that token's logits in float64 and decides on those. The selection is then the one exact
// arithmetic would make, except for gaps below the float64 rounding level.
// Equal logits go to the lower expert index.
#include <cuda_bf16.h>
#include <math.h>

#include <algorithm>

#include "rom_internal.cuh"

namespace rom {
namespace {

constexpr int kRouterThreads = 512;
constexpr int kRouterWarps = kRouterThreads / 32;

template <typename InT>
struct Elem;
template <>
struct Elem<__nv_bfloat16> {
  static constexpr int V = 8;        // elements per lane per step (two groups of 4)
  static constexpr int STEP = 256;   // elements per warp per step
};
template <>
struct Elem<float> {
  static constexpr int V = 4;        // one group of 4
  static constexpr int STEP = 128;
};

template <int EB>
struct Geo {
  static constexpr int NV = EB <= 8 ? 32 : 64;     // partial logits per lane
  static constexpr int TPW = NV / EB;              // tokens per warp per pass
  static constexpr int VPL = NV / 32;              // complete logits per lane
  static constexpr int W = EB < 32 ? EB : 32;      // lanes per token segment
  static constexpr int VPT = EB > 32 ? EB / 32 : 1;  // logits per lane per token
};

// 4 consecutive elements of x -> float.
__device__ __forceinline__ void load4(const __nv_bfloat16* p, float* f) {
  const uint2 v = __ldg(reinterpret_cast<const uint2*>(p));
  f[0] = __uint_as_float(v.x << 16);
  f[1] = __uint_as_float(v.x & 0xFFFF0000u);
  f[2] = __uint_as_float(v.y << 16);
  f[3] = __uint_as_float(v.y & 0xFFFF0000u);
}
__device__ __forceinline__ void load4(const float* p, float* f) {
  const float4 v = __ldg(reinterpret_cast<const float4*>(p));
  f[0] = v.x;
  f[1] = v.y;
  f[2] = v.z;
  f[3] = v.w;
}

// Element offset (within a step) of the lane's group g of 4 elements.
template <typename InT>
__device__ __forceinline__ int group_off(int g, int lane) {
  return g * 128 + 4 * lane;
}

// Argmax over the W lanes of each aligned segment: larger value wins, equal
// values go to the lower expert index. Every lane of the segment receives
// the winner.
template <int W, typename VT>
__device__ __forceinline__ void seg_argmax(VT& v, int& e) {
#pragma unroll
  for (int o = W / 2; o > 0; o >>= 1) {
    const VT ov = __shfl_xor_sync(0xffffffffu, v, o);
    const int oe = __shfl_xor_sync(0xffffffffu, e, o);
    if (ov > v || (ov == v && oe < e)) {
      v = ov;
      e = oe;
    }
  }
}

template <int W>
__device__ __forceinline__ float seg_sum(float v) {
#pragma unroll
  for (int o = W / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <int W>
__device__ __forceinline__ float seg_max(float v) {
#pragma unroll
  for (int o = W / 2; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Selection for one token segment. Each lane holds VPT candidate logits
// `lv` of experts `le` (le >= E: padding, value -inf). Produces, uniform
// over the segment, the experts sel[0..k] (sel[k] = the best unselected one,
// or -1) and their logits selv[]; `slot[v]` = slot of the lane's own
// candidate v (or -1).
template <int W, int VPT, typename VT>
__device__ __forceinline__ void seg_select(const VT (&lv)[VPT], const int (&le)[VPT], int E, int k,
                                           int (&sel)[kMaxTopK + 1], VT (&selv)[kMaxTopK + 1],
                                           int (&slot)[VPT]) {
  bool used[VPT];
#pragma unroll
  for (int v = 0; v < VPT; ++v) {
    used[v] = false;
    slot[v] = -1;
  }
#pragma unroll
  for (int j = 0; j <= kMaxTopK; ++j) {
    sel[j] = -1;
    selv[j] = -INFINITY;
    if (j <= k) {
      VT cv = -INFINITY;
      int ce = 1 << 20;
#pragma unroll
      for (int v = 0; v < VPT; ++v) {
        if (!used[v] && le[v] < E && (lv[v] > cv || (lv[v] == cv && le[v] < ce))) {
          cv = lv[v];
          ce = le[v];
        }
      }
      seg_argmax<W, VT>(cv, ce);
      if (ce < E) {
        sel[j] = ce;
        selv[j] = cv;
#pragma unroll
        for (int v = 0; v < VPT; ++v)
          if (le[v] == ce) {
            used[v] = true;
            if (j < k) slot[v] = j;
          }
      }
    }
  }
}

// float64 logits of one token, computed by the whole warp; lane 0 writes
// out[0..E).
template <typename InT, int EB>
__device__ __noinline__ void refine_logits_f64(const InT* __restrict__ xrow, int Dm, int DS,
                                               const float* sW, const float* w_r,
                                               const float* bias, int E, bool smem_w,
                                               double* out, int lane) {
  constexpr int G = EB < 16 ? EB : 16;
  for (int e0 = 0; e0 < EB; e0 += G) {
    double a[G];
#pragma unroll
    for (int g = 0; g < G; ++g) a[g] = 0.0;
    for (int d = 4 * lane; d < Dm; d += 128) {
      float xv[4];
      load4(xrow + d, xv);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const int e = e0 + g;
        if (e < E) {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float w = smem_w ? sW[e * DS + d + j] : __ldg(w_r + static_cast<int64_t>(d + j) * E + e);
            a[g] = fma(static_cast<double>(xv[j]), static_cast<double>(w), a[g]);
          }
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

template <int N>
__device__ __forceinline__ float pickf(const float (&a)[N], int i) {
  float r = a[0];
#pragma unroll
  for (int q = 1; q < N; ++q) r = (q == i) ? a[q] : r;
  return r;
}

// Loads W_r^T[e][D0 .. D0+DS) into sW[e][0 .. DS) (zero beyond Dm and for
// padding experts e >= E). The global reads walk w_r in memory order.
__device__ __forceinline__ void load_w_slice(float* sW, const float* __restrict__ w_r, int Dm,
                                             int E, int EB, int D0, int DS, int tid) {
  const int dn = min(DS, Dm - D0);  // features of this slice that exist
  const float* src = w_r + static_cast<int64_t>(D0) * E;
  for (int i = tid; i < dn * E; i += kRouterThreads) {
    const int d = i / E, e = i - d * E;
    sW[e * DS + d] = __ldg(src + i);
  }
  for (int i = tid; i < DS * EB; i += kRouterThreads) {
    const int e = i / DS, d = i - e * DS;
    if (e >= E || d >= dn) sW[i] = 0.f;
  }
}

template <typename InT, int EB>
__global__ void __launch_bounds__(kRouterThreads)
    router_kernel(const InT* __restrict__ x, int64_t T, int Dm, const float* __restrict__ w_r,
                  const float* __restrict__ bias, int E, int k, int renorm,
                  int32_t* __restrict__ topk_idx, float* __restrict__ topk_w,
                  int32_t* __restrict__ counts, int32_t* __restrict__ chunk_hist,
                  int64_t nchunks, float gamma, int DS) {
  using G = Geo<EB>;
  constexpr int NV = G::NV, TPW = G::TPW, VPL = G::VPL, W = G::W, VPT = G::VPT;
  constexpr int V = Elem<InT>::V, STEP = Elem<InT>::STEP;
  constexpr int kPasses = kChunkTokens / (kRouterWarps * TPW);
  static_assert(kPasses * kRouterWarps * TPW == kChunkTokens, "chunk geometry");
  extern __shared__ float4 router_smem[];
  // W_r^T slice [EB][DS] (+ STEP zero pad): the whole of d_model when it fits
  // (loaded once per CTA), otherwise d_model slices reloaded per pass.
  float* sW = reinterpret_cast<float*>(router_smem);
  __shared__ float s_wsq[EB];
  __shared__ float s_wnorm[EB];
  __shared__ int s_hist[EB];
  __shared__ double s_l64[kRouterWarps][EB];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nslices = (Dm + DS - 1) / DS;
  const bool resident = nslices == 1;

  for (int i = tid; i < EB * DS + STEP; i += kRouterThreads)
    if (i >= EB * DS) sW[i] = 0.f;  // pad read by the last lanes of a step
  for (int e = tid; e < EB; e += kRouterThreads) s_wsq[e] = 0.f;
  bool norms_ready = false;
  if (resident) {
    load_w_slice(sW, w_r, Dm, E, EB, 0, DS, tid);
    __syncthreads();
  }

  for (int64_t c = blockIdx.x; c < nchunks; c += gridDim.x) {
    for (int e = tid; e < EB; e += kRouterThreads) s_hist[e] = 0;
    __syncthreads();
    for (int pass = 0; pass < kPasses; ++pass) {
      const int64_t t0 =
          c * kChunkTokens + static_cast<int64_t>(pass * kRouterWarps + warp) * TPW;
      float acc[NV];
      float sq[TPW];
#pragma unroll
      for (int i = 0; i < NV; ++i) acc[i] = 0.f;
#pragma unroll
      for (int t = 0; t < TPW; ++t) sq[t] = 0.f;

      for (int s = 0; s < nslices; ++s) {
        const int D0 = s * DS;
        if (!resident) {
          __syncthreads();  // every warp is done with the previous slice
          load_w_slice(sW, w_r, Dm, E, EB, D0, DS, tid);
          __syncthreads();
        }
        if (!norms_ready) {
          // |w_e|^2 over this slice, accumulated per expert in slice order.
          for (int e = warp; e < EB; e += kRouterWarps) {
            float q = 0.f;
            for (int d = lane; d < DS; d += 32) q = fmaf(sW[e * DS + d], sW[e * DS + d], q);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) q += __shfl_xor_sync(0xffffffffu, q, off);
            if (lane == 0) s_wsq[e] += q;
          }
        }
        const int dend = min(Dm, D0 + DS);
        for (int d0 = D0; d0 < dend; d0 += STEP) {
          float xv[TPW][V];
#pragma unroll
          for (int t = 0; t < TPW; ++t) {
#pragma unroll
            for (int g = 0; g < V / 4; ++g) {
              const int d = d0 + group_off<InT>(g, lane);
              if (t0 + t < T && d < Dm) {
                load4(x + (t0 + t) * static_cast<int64_t>(Dm) + d, &xv[t][4 * g]);
              } else {
#pragma unroll
                for (int j = 0; j < 4; ++j) xv[t][4 * g + j] = 0.f;
              }
            }
#pragma unroll
            for (int v = 0; v < V; ++v) sq[t] = fmaf(xv[t][v], xv[t][v], sq[t]);
          }
#pragma unroll
          for (int e = 0; e < EB; ++e) {
            float wv[V];
#pragma unroll
            for (int g = 0; g < V / 4; ++g) {
              const float4 q = *reinterpret_cast<const float4*>(
                  sW + e * DS + (d0 - D0) + group_off<InT>(g, lane));
              wv[4 * g] = q.x;
              wv[4 * g + 1] = q.y;
              wv[4 * g + 2] = q.z;
              wv[4 * g + 3] = q.w;
            }
#pragma unroll
            for (int t = 0; t < TPW; ++t) {
#pragma unroll
              for (int v = 0; v < V; ++v)
                acc[t * EB + e] = fmaf(xv[t][v], wv[v], acc[t * EB + e]);
            }
          }
        }
      }
      if (!norms_ready) {
        __syncthreads();
        for (int e = tid; e < EB; e += kRouterThreads) s_wnorm[e] = sqrtf(s_wsq[e]);
        __syncthreads();
        norms_ready = true;
      }

      // |x|^2 of every token of the pass, on every lane.
#pragma unroll
      for (int t = 0; t < TPW; ++t) {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) sq[t] += __shfl_xor_sync(0xffffffffu, sq[t], off);
      }
      // Transpose-reduce: lane L ends with the sum of flat index i*32 + L.
#pragma unroll
      for (int blk = 0; blk < VPL; ++blk) {
        float* a = acc + blk * 32;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          const bool up = (lane & o) != 0;
#pragma unroll
          for (int j = 0; j < o; ++j) {
            const float send = up ? a[j] : a[j + o];
            const float keep = up ? a[j + o] : a[j];
            a[j] = keep + __shfl_xor_sync(0xffffffffu, send, o);
          }
        }
      }

      // Lane-parallel decisions: a token occupies W lanes x VPT values.
      constexpr int NSEG = VPL / VPT;  // token groups per lane
#pragma unroll
      for (int sg = 0; sg < NSEG; ++sg) {
        float lv[VPT];
        int le[VPT];
        int tl = 0;
#pragma unroll
        for (int v = 0; v < VPT; ++v) {
          const int f = (sg * VPT + v) * 32 + lane;  // flat index of acc[sg*VPT+v]'s block
          tl = f / EB;
          le[v] = f % EB;
          const float b = (bias && le[v] < E) ? __ldg(bias + le[v]) : 0.f;
          lv[v] = (le[v] < E) ? acc[(sg * VPT + v) * 32] + b : -INFINITY;
        }
        const int64_t tok = t0 + tl;
        const bool tok_ok = tok < T;
        const float xn = sqrtf(pickf<TPW>(sq, tl));
        int sel[kMaxTopK + 1];
        float selv[kMaxTopK + 1];
        int slot[VPT];
        seg_select<W, VPT, float>(lv, le, E, k, sel, selv, slot);
        // Certain when, for every slot j < k, the lower bound of the j-th
        // selected logit clears the upper bound of every expert ranked after
        // it: the unselected experts (their largest upper bound, over the
        // segment) and the selected slots j+1 .. k-1 (a running maximum,
        // walking the slots from the last). The bounds differ per expert
        // through |w_e|, so the next-ranked expert alone does not decide.
        float ub_rest = -INFINITY;
#pragma unroll
        for (int v = 0; v < VPT; ++v)
          if (le[v] < E && slot[v] < 0)
            ub_rest = fmaxf(ub_rest, lv[v] + gamma * xn * s_wnorm[le[v]] + 1.2e-7f * fabsf(lv[v]));
        ub_rest = seg_max<W>(ub_rest);
        bool certain = true;
#pragma unroll
        for (int j = kMaxTopK - 1; j >= 0; --j) {
          if (j < k) {
            const float ea = gamma * xn * s_wnorm[sel[j]] + 1.2e-7f * fabsf(selv[j]);
            if (!(selv[j] - ea > ub_rest)) certain = false;
            ub_rest = fmaxf(ub_rest, selv[j] + ea);
          }
        }
        // Tokens whose float32 decision is not certain: float64 logits.
        unsigned todo = __ballot_sync(0xffffffffu, tok_ok && !certain);
        while (todo) {
          const int src = __ffs(todo) - 1;
          const int tl_r = __shfl_sync(0xffffffffu, tl, src);
          todo &= ~(((W == 32) ? 0xffffffffu : ((1u << W) - 1u)) << (src & ~(W - 1)));
          refine_logits_f64<InT, EB>(x + (t0 + tl_r) * static_cast<int64_t>(Dm), Dm, DS, sW, w_r,
                                     bias, E, resident, s_l64[warp], lane);
          double lv64[VPT];
#pragma unroll
          for (int v = 0; v < VPT; ++v)
            lv64[v] = (le[v] < E) ? s_l64[warp][le[v] < E ? le[v] : 0] : -INFINITY;
          int sel2[kMaxTopK + 1];
          double selv2[kMaxTopK + 1];
          int slot2[VPT];
          seg_select<W, VPT, double>(lv64, le, E, k, sel2, selv2, slot2);
          if (tl == tl_r) {
#pragma unroll
            for (int j = 0; j <= kMaxTopK; ++j) {
              sel[j] = sel2[j];
              selv[j] = static_cast<float>(selv2[j]);
            }
#pragma unroll
            for (int v = 0; v < VPT; ++v) {
              slot[v] = slot2[v];
              lv[v] = static_cast<float>(lv64[v]);
            }
          }
          __syncwarp();
        }
        // Softmax (float32) and outputs.
        const float m = selv[0];
        float den = 0.f;
        if (renorm) {
#pragma unroll
          for (int j = 0; j < kMaxTopK; ++j)
            if (j < k) den += expf(selv[j] - m);
        } else {
          float part = 0.f;
#pragma unroll
          for (int v = 0; v < VPT; ++v)
            if (le[v] < E) part += expf(lv[v] - m);
          den = seg_sum<W>(part);
        }
#pragma unroll
        for (int v = 0; v < VPT; ++v) {
          if (tok_ok && slot[v] >= 0) {
            topk_idx[tok * k + slot[v]] = le[v];
            topk_w[tok * k + slot[v]] = expf(lv[v] - m) / den;
            atomicAdd(&s_hist[le[v]], 1);
          }
        }
      }
    }
    __syncthreads();
    for (int e = tid; e < E; e += kRouterThreads) {
      if (chunk_hist) chunk_hist[c * E + e] = s_hist[e];
      if (counts && s_hist[e]) atomicAdd(counts + e, s_hist[e]);
    }
    __syncthreads();
  }
}

template <typename InT, int EB>
cudaError_t launch_eb(const InT* x, int64_t T, int Dm, const float* w_r, const float* bias,
                      int E, int k, int renorm, int32_t* topk_idx, float* topk_w,
                      int32_t* counts, int32_t* chunk_hist, cudaStream_t stream) {
  constexpr int V = Elem<InT>::V, STEP = Elem<InT>::STEP;
  const int64_t nchunks = num_chunks(T);
  if (nchunks == 0) return cudaSuccess;
  // Longest float32 accumulation chain: the lane's sequential slice, the
  // 5-level reduction tree and the bias add (+1 spare); 1 % slack covers the
  // rounding of the two norms.
  const double n = static_cast<double>(((Dm + STEP - 1) / STEP) * V + 5 + 2);
  const double u = 1.0 / 16777216.0;
  const float gamma = static_cast<float>(1.01 * n * u / (1.0 - n * u));
  // d_model slice held in shared memory: all of it when it fits in 160 KB.
  const int dm_pad = (Dm + STEP - 1) / STEP * STEP;
  const int ds_max = ((160 * 1024 / 4 - STEP) / EB) / STEP * STEP;
  const int DS = std::min(dm_pad, ds_max);
  const size_t smem_w = (static_cast<size_t>(EB) * DS + STEP) * sizeof(float);
  const int sms = device_sm_count();
  auto kern = router_kernel<InT, EB>;
  cudaError_t err =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_w);
  if (err != cudaSuccess) return err;
  int per_sm = 1;
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kRouterThreads, smem_w);
  if (per_sm < 1) per_sm = 1;
  const int64_t grid = std::min<int64_t>(nchunks, static_cast<int64_t>(sms) * per_sm);
  kern<<<static_cast<unsigned>(grid), kRouterThreads, smem_w, stream>>>(
      x, T, Dm, w_r, bias, E, k, renorm, topk_idx, topk_w, counts, chunk_hist, nchunks, gamma,
      DS);
  return cudaGetLastError();
}

template <typename InT>
cudaError_t launch_typed(const InT* x, int64_t T, int Dm, const float* w_r, const float* bias,
                         int E, int k, int renorm, int32_t* topk_idx, float* topk_w,
                         int32_t* counts, int32_t* chunk_hist, cudaStream_t stream) {
#define ROM_ROUTER_CASE(EBV)                                                                 \
  if (E <= EBV)                                                                              \
    return launch_eb<InT, EBV>(x, T, Dm, w_r, bias, E, k, renorm, topk_idx, topk_w, counts, \
                               chunk_hist, stream);
  ROM_ROUTER_CASE(4)
  ROM_ROUTER_CASE(8)
  ROM_ROUTER_CASE(16)
  ROM_ROUTER_CASE(32)
  ROM_ROUTER_CASE(64)
#undef ROM_ROUTER_CASE
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_router(const void* x, bool bf16, int64_t T, int Dm, const float* w_r,
                          const float* bias, int E, int k, int renorm, int32_t* topk_idx,
                          float* topk_w, int32_t* counts, int32_t* chunk_hist, int* status,
                          cudaStream_t stream) {
  // Small batches: one CTA per token (router_small.cu).
  {
    const cudaError_t e = launch_router_small(x, bf16, T, Dm, w_r, bias, E, k, renorm, topk_idx,
                                              topk_w, counts, chunk_hist, stream);
    if (e != cudaErrorNotSupported) return e;
  }
  if (bf16) {
    // The streaming router (router_stream.cu) when W_r stays resident in
    // shared memory; the register-tiled kernel below otherwise.
    const cudaError_t e = launch_router_stream(x, T, Dm, w_r, bias, E, k, renorm, topk_idx,
                                               topk_w, counts, chunk_hist, status, stream);
    if (e != cudaErrorNotSupported) return e;
    return launch_typed(static_cast<const __nv_bfloat16*>(x), T, Dm, w_r, bias, E, k, renorm,
                        topk_idx, topk_w, counts, chunk_hist, stream);
  }
  return launch_typed(static_cast<const float*>(x), T, Dm, w_r, bias, E, k, renorm, topk_idx,
                      topk_w, counts, chunk_hist, stream);
}

}  // namespace rom
