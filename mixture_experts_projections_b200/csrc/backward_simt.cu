// Bandwidth-bound pieces of the RoM block backward ("Routing Mamba ..."
// chapterpal summary page, Knowl 1, differentiated with S_t held fixed):
//
//  scale_gather  rdO_sorted[p] = r_s * dO[s / k]   (s = sorted_slot[p]); the A
//                operand of the Out dgrad (giving g'_s = r_s g_s) and of dW_out.
//  gate_bwd      per token t and column c, with H = sum_j u_{t,j},
//                Z = sum_j z_{t,j} (the forward's float32 slot partials) and
//                dYG = sum_j g'_{t,j} = sum_j r_j g_j:
//                  dH = dYG * SiLU(Z),  dZ = dYG * H * SiLU'(Z),
//                  SiLU'(Z) = s (1 + Z (1 - s)), s = sigmoid(Z);
//                written as [dH | dZ] rows in expert-sorted order for every
//                slot of the token (A operand of dX and of dW_in / dW_g).
//  route_bwd     per token: dr_j = <Y(.)G, g_j> = (sum of the Out dgrad's
//                partial dots) / r_j; with s = sum_i r_i dr_i,
//                  dlogit_j = r_j (dr_j - s) on S_t, and off S_t 0 for
//                  renormalised weights (r = softmax over the selected
//                  logits) or -p_m s for r = p (the softmax over all E);
//                dX_t = sum_j dX_{t,j} + sum_m dlogit_m W_r[:, m].
//  route_probs   p = softmax over all E experts (float32), for the r = p case.
//  route_wgrad   dW_r = X^T dlogits and dbias = the column sums of dlogits.
#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <math.h>

#include <algorithm>
#include <type_traits>

#include "rom_internal.cuh"

namespace cg = cooperative_groups;

namespace rom {
namespace {

constexpr int kThreads = 256;
constexpr int kRouteBwdThreads = 1024;  // one warp per token, many tokens in flight

__device__ __forceinline__ uint32_t pack2(float a, float b) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// One warp per sorted row; 8 bf16 (16 bytes) per lane per step.
__global__ void __launch_bounds__(kThreads)
    scale_gather_kernel(const __nv_bfloat16* __restrict__ dout, int64_t R, int k, int N,
                        const int32_t* __restrict__ sorted_slot,
                        const float* __restrict__ topk_w, __nv_bfloat16* __restrict__ dst) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (blockIdx.x * static_cast<int64_t>(kThreads) + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * kThreads) >> 5;
  const int nv = N / 8;
  for (int64_t p = warp; p < R; p += nwarps) {
    const int64_t s = sorted_slot[p];
    const float r = topk_w[s];
    const uint4* src = reinterpret_cast<const uint4*>(dout + (s / k) * N);
    uint4* d = reinterpret_cast<uint4*>(dst + p * N);
    for (int i = lane; i < nv; i += 32) {
      const uint4 v = __ldg(src + i);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
      uint32_t o[4];
#pragma unroll
      for (int q = 0; q < 4; ++q)
        o[q] = pack2(r * __uint_as_float(w[q] << 16), r * __uint_as_float(w[q] & 0xFFFF0000u));
      d[i] = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

// One thread per (token, 4 columns).
__global__ void __launch_bounds__(kThreads)
    gate_bwd_kernel(const float* __restrict__ uz, const float* __restrict__ gp, int64_t T, int k,
                    int De, const int32_t* __restrict__ slot_pos, __nv_bfloat16* __restrict__ dhz) {
  const int nq = De / 4;
  const int64_t total = T * nq;
  const int64_t R = T * k;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(kThreads) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * kThreads) {
    const int64_t t = i / nq;
    const int c = static_cast<int>(i - t * nq) * 4;
    float h[4] = {0.f, 0.f, 0.f, 0.f}, z[4] = {0.f, 0.f, 0.f, 0.f}, g[4] = {0.f, 0.f, 0.f, 0.f};
    for (int j = 0; j < k; ++j) {
      const int64_t s = t * k + j;
      const float4 a = __ldg(reinterpret_cast<const float4*>(uz + s * De + c));
      const float4 b = __ldg(reinterpret_cast<const float4*>(uz + (R + s) * De + c));
      const float4 d = __ldg(reinterpret_cast<const float4*>(gp + s * De + c));
      h[0] += a.x; h[1] += a.y; h[2] += a.z; h[3] += a.w;
      z[0] += b.x; z[1] += b.y; z[2] += b.z; z[3] += b.w;
      g[0] += d.x; g[1] += d.y; g[2] += d.z; g[3] += d.w;
    }
    float dh[4], dz[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float s = 1.0f / (1.0f + expf(-z[q]));
      dh[q] = g[q] * (z[q] * s);
      dz[q] = g[q] * h[q] * (s * (1.0f + z[q] * (1.0f - s)));
    }
    const uint2 wh = make_uint2(pack2(dh[0], dh[1]), pack2(dh[2], dh[3]));
    const uint2 wz = make_uint2(pack2(dz[0], dz[1]), pack2(dz[2], dz[3]));
    for (int j = 0; j < k; ++j) {
      const int64_t row = slot_pos[t * k + j];
      *reinterpret_cast<uint2*>(dhz + row * (2 * De) + c) = wh;
      *reinterpret_cast<uint2*>(dhz + row * (2 * De) + De + c) = wz;
    }
  }
}

// One warp per token; W_r^T slice [E][DS] staged in shared memory.
// probs == nullptr: renormalised weights (dlogit zero off S_t). Otherwise
// r = p (the softmax over all E experts, probs [T][E]) and every expert m
// off S_t gets dlogit_m = -p_m sum_i r_i dr_i, which also enters dX.
__global__ void __launch_bounds__(kRouteBwdThreads)
    route_bwd_kernel(int64_t T, int k, int E, int Dm, const int32_t* __restrict__ topk_idx,
                     const float* __restrict__ topk_w, const float* __restrict__ probs,
                     const float* __restrict__ dr_part, int n_parts,
                     const float* __restrict__ dx_slots, const float* __restrict__ w_r,
                     float* __restrict__ dlogits, __nv_bfloat16* __restrict__ dx, int DS) {
  extern __shared__ float sWt[];  // [E][DS]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nw = kRouteBwdThreads / 32;
  __shared__ float s_coef[kRouteBwdThreads / 32][kMaxExperts];  // off-S dlogits (probs given)
  for (int D0 = 0; D0 < Dm; D0 += DS) {
    const int dn = min(DS, Dm - D0);
    __syncthreads();
    for (int i = threadIdx.x; i < dn * E; i += kRouteBwdThreads) {
      const int d = i / E, e = i - d * E;
      sWt[e * DS + d] = __ldg(w_r + static_cast<int64_t>(D0) * E + i);
    }
    __syncthreads();
    for (int64_t t = blockIdx.x * static_cast<int64_t>(nw) + warp; t < T;
         t += static_cast<int64_t>(gridDim.x) * nw) {
      // dr_j and dlogit_j (recomputed per slice; a few dozen flops)
      float dl[kMaxTopK];
      int sel[kMaxTopK];
      float s = 0.f;
      float dr[kMaxTopK], rw[kMaxTopK];
#pragma unroll
      for (int j = 0; j < kMaxTopK; ++j) {
        dl[j] = 0.f;
        sel[j] = 0;
        dr[j] = 0.f;
        rw[j] = 0.f;
        if (j < k) {
          const int64_t slot = t * k + j;
          float acc = 0.f;
          for (int q = lane; q < n_parts; q += 32) acc += dr_part[slot * n_parts + q];
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
          rw[j] = topk_w[slot];
          sel[j] = topk_idx[slot];
          dr[j] = acc / rw[j];
          s += rw[j] * dr[j];
        }
      }
#pragma unroll
      for (int j = 0; j < kMaxTopK; ++j)
        if (j < k) dl[j] = rw[j] * (dr[j] - s);
      if (probs) {
        // experts off S_t: dlogit_m = -p_m s (0 for the selected ones here;
        // theirs are dl[j])
        for (int e = lane; e < E; e += 32) {
          bool on = false;
#pragma unroll
          for (int j = 0; j < kMaxTopK; ++j)
            if (j < k && sel[j] == e) on = true;
          s_coef[warp][e] = on ? 0.f : -probs[t * E + e] * s;
        }
        __syncwarp();
      }
      if (D0 == 0 && dlogits) {
        for (int e = lane; e < E; e += 32) {
          float v = probs ? s_coef[warp][e] : 0.f;
#pragma unroll
          for (int j = 0; j < kMaxTopK; ++j)
            if (j < k && sel[j] == e) v = dl[j];
          dlogits[t * E + e] = v;
        }
      }
      for (int d = lane * 4; d < dn; d += 128) {
        float4 acc = __ldg(reinterpret_cast<const float4*>(dx_slots + (t * k) * Dm + D0 + d));
        for (int j = 1; j < k; ++j) {
          const float4 v =
              __ldg(reinterpret_cast<const float4*>(dx_slots + (t * k + j) * Dm + D0 + d));
          acc.x += v.x;
          acc.y += v.y;
          acc.z += v.z;
          acc.w += v.w;
        }
#pragma unroll
        for (int j = 0; j < kMaxTopK; ++j) {
          if (j < k) {
            const float4 w = *reinterpret_cast<const float4*>(sWt + sel[j] * DS + d);
            acc.x = fmaf(dl[j], w.x, acc.x);
            acc.y = fmaf(dl[j], w.y, acc.y);
            acc.z = fmaf(dl[j], w.z, acc.z);
            acc.w = fmaf(dl[j], w.w, acc.w);
          }
        }
        if (probs) {
          for (int e = 0; e < E; ++e) {
            const float c = s_coef[warp][e];
            const float4 w = *reinterpret_cast<const float4*>(sWt + e * DS + d);
            acc.x = fmaf(c, w.x, acc.x);
            acc.y = fmaf(c, w.y, acc.y);
            acc.z = fmaf(c, w.z, acc.z);
            acc.w = fmaf(c, w.w, acc.w);
          }
        }
        *reinterpret_cast<uint2*>(dx + t * Dm + D0 + d) =
            make_uint2(pack2(acc.x, acc.y), pack2(acc.z, acc.w));
      }
      __syncwarp();  // s_coef is rewritten for the warp's next token
    }
  }
}

template <typename InT>
__device__ __forceinline__ float to_f(InT v);
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}
template <>
__device__ __forceinline__ float to_f<float>(float v) {
  return v;
}

// Softmax over all E experts of every token, float32 (the routing weights'
// full distribution, which the backward needs when r = p is not
// renormalised). One warp per token: lanes split d_model and accumulate 16
// experts at a time in feature order, then a butterfly sum.
template <typename InT>
__global__ void __launch_bounds__(256)
    route_probs_kernel(const InT* __restrict__ x, int64_t T, int Dm, const float* __restrict__ w_r,
                       const float* __restrict__ bias, int E, float* __restrict__ probs) {
  __shared__ float s_l[8][kMaxExperts];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int64_t t = blockIdx.x * 8ll + warp; t < T; t += static_cast<int64_t>(gridDim.x) * 8) {
    for (int e0 = 0; e0 < E; e0 += 16) {
      float acc[16];
#pragma unroll
      for (int q = 0; q < 16; ++q) acc[q] = 0.f;
      for (int d = lane; d < Dm; d += 32) {
        const float xv = to_f<InT>(x[t * Dm + d]);
#pragma unroll
        for (int q = 0; q < 16; ++q)
          if (e0 + q < E) acc[q] = fmaf(xv, __ldg(w_r + static_cast<int64_t>(d) * E + e0 + q), acc[q]);
      }
#pragma unroll
      for (int q = 0; q < 16; ++q) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc[q] += __shfl_xor_sync(0xffffffffu, acc[q], o);
      }
      if (lane == 0)
#pragma unroll
        for (int q = 0; q < 16; ++q)
          if (e0 + q < E) s_l[warp][e0 + q] = acc[q] + (bias ? __ldg(bias + e0 + q) : 0.f);
    }
    __syncwarp();
    float m = -INFINITY;
    for (int e = 0; e < E; ++e) m = fmaxf(m, s_l[warp][e]);
    float den = 0.f;
    for (int e = 0; e < E; ++e) den += expf(s_l[warp][e] - m);
    for (int e = lane; e < E; e += 32) probs[t * E + e] = expf(s_l[warp][e] - m) / den;
    __syncwarp();
  }
}

// Router weight gradients: dW_r[d][e] = sum_t x[t][d] dlogit[t][e] and
// dbias[e] = sum_t dlogit[t][e], in float32. A cluster of `split` CTAs (sized
// at launch so that the grid fits the SMs in one wave) owns 64 features of
// d_model; CTA r of the cluster sums the tokens of its slice r of T. Warp w
// of a CTA takes the 16-token groups w, w + 8, ... of the slice on its own
// (no block-wide barrier in the loop): each lane holds two features for all
// experts, the group's logit gradients go through the warp's own shared
// buffer and are read back as broadcast float4s, one packed FMA per token and
// expert updates the lane's two sums, and the next group's x and gradient
// loads are in flight while the current group is computed. The 8 warps' sums
// are added in warp order, then CTA 0 of the cluster adds the `split` partial
// sums in rank order through distributed shared memory. The order of every
// sum is fixed for a given launch shape, so the result is deterministic.
constexpr int kRwFeat = 64, kRwMaxSplit = 8, kRwGroup = 16;

// x[da], x[da + 1] of one row (zero past d_model or for a token past the
// slice), kept packed until use: bf16 as one 32-bit word, float32 as a pair.
// `pair` (uniform): the two values are one aligned 4- or 8-byte load.
__device__ __forceinline__ uint32_t load_pair(const __nv_bfloat16* row, int da, int Dm, bool ok,
                                              bool pair) {
  if (!ok) return 0u;
  if (pair && da + 1 < Dm) return __ldg(reinterpret_cast<const unsigned int*>(row + da));
  const uint32_t lo = da < Dm ? __bfloat16_as_ushort(row[da]) : 0u;
  const uint32_t hi = da + 1 < Dm ? __bfloat16_as_ushort(row[da + 1]) : 0u;
  return lo | (hi << 16);
}
__device__ __forceinline__ float2 load_pair(const float* row, int da, int Dm, bool ok, bool pair) {
  if (!ok) return make_float2(0.f, 0.f);
  if (pair && da + 1 < Dm) return __ldg(reinterpret_cast<const float2*>(row + da));
  return make_float2(da < Dm ? row[da] : 0.f, da + 1 < Dm ? row[da + 1] : 0.f);
}
__device__ __forceinline__ float2 unpack_pair(uint32_t v) {
  return make_float2(__uint_as_float(v << 16), __uint_as_float(v & 0xFFFF0000u));
}
__device__ __forceinline__ float2 unpack_pair(float2 v) { return v; }

template <int EB, typename InT>
__global__ void __launch_bounds__(256)
    route_wgrad_kernel(const InT* __restrict__ x, int64_t T, int Dm, int E,
                       const float* __restrict__ dl, float* __restrict__ dw_r,
                       float* __restrict__ dbias, bool pair) {
  using Packed = typename std::conditional<std::is_same<InT, float>::value, float2, uint32_t>::type;
  constexpr int kPer = kRwGroup * EB / 32;  // gradient values a lane stages per group
  static_assert(kPer >= 1 && 8 * kRwGroup >= kRwFeat, "layout");
  __shared__ __align__(16) float s_dl[8][kRwGroup][EB];  // after the loop: s_part
  __shared__ float s_bsum[8][EB];
  __shared__ float s_bias[EB];
  float(*s_part)[kRwFeat + 1] = reinterpret_cast<float(*)[kRwFeat + 1]>(&s_dl[0][0][0]);  // [EB][65]
  static_assert(EB * (kRwFeat + 1) <= 8 * kRwGroup * EB, "partials fit the staging buffer");
  cg::cluster_group cluster = cg::this_cluster();
  const int split = static_cast<int>(cluster.num_blocks());
  const int rank = static_cast<int>(cluster.block_rank());
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int d0 = (blockIdx.x / split) * kRwFeat;
  const int da = d0 + 2 * lane;  // this lane's features da, da + 1
  const bool bias_cluster = blockIdx.x / split == 0 && dbias != nullptr;
  const int64_t per = (T + split - 1) / split;
  const int64_t ta = rank * per, tb = ta + per < T ? ta + per : T;
  float2 acc[EB];
#pragma unroll
  for (int e = 0; e < EB; ++e) acc[e] = make_float2(0.f, 0.f);
  float bacc = 0.f;  // bias (lane < EB): expert `lane` over this warp's tokens
  float(*buf)[EB] = s_dl[warp];

  // loads of one group (tokens g0 .. g0+15 of the slice) into registers
  Packed xn[kRwGroup];
  float dn[kPer];
  auto fetch = [&](int64_t g0) {
    const InT* row = x + g0 * Dm;
#pragma unroll
    for (int u = 0; u < kRwGroup; ++u, row += Dm) xn[u] = load_pair(row, da, Dm, g0 + u < tb, pair);
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int i = lane + 32 * j, u = i / EB, e = i - u * EB;
      const int64_t t = g0 + u;
      dn[j] = (t < tb && e < E) ? __ldg(dl + t * E + e) : 0.f;
    }
  };
  int64_t g0 = ta + static_cast<int64_t>(warp) * kRwGroup;
  if (g0 < tb) fetch(g0);
  for (; g0 < tb; g0 += 8 * kRwGroup) {
    Packed xc[kRwGroup];
#pragma unroll
    for (int u = 0; u < kRwGroup; ++u) xc[u] = xn[u];
    __syncwarp();  // the previous group's reads of buf are done
#pragma unroll
    for (int j = 0; j < kPer; ++j) (&buf[0][0])[lane + 32 * j] = dn[j];
    __syncwarp();
    if (g0 + 8 * kRwGroup < tb) fetch(g0 + 8 * kRwGroup);  // in flight during the FMAs
#pragma unroll
    for (int u = 0; u < kRwGroup; ++u) {
      const float2 xv = unpack_pair(xc[u]);
      const float4* g4 = reinterpret_cast<const float4*>(&buf[u][0]);
#pragma unroll
      for (int e4 = 0; e4 < EB / 4; ++e4) {
        const float4 g = g4[e4];
        acc[4 * e4] = __ffma2_rn(xv, make_float2(g.x, g.x), acc[4 * e4]);
        acc[4 * e4 + 1] = __ffma2_rn(xv, make_float2(g.y, g.y), acc[4 * e4 + 1]);
        acc[4 * e4 + 2] = __ffma2_rn(xv, make_float2(g.z, g.z), acc[4 * e4 + 2]);
        acc[4 * e4 + 3] = __ffma2_rn(xv, make_float2(g.w, g.w), acc[4 * e4 + 3]);
      }
    }
    if (bias_cluster)
      for (int e = lane; e < EB; e += 32)
#pragma unroll
        for (int u = 0; u < kRwGroup; ++u) bacc += buf[u][e];
  }
  __syncthreads();  // every warp is done with its staging buffer
  // the warps' sums, added in warp order (s_part[e][f]: lanes 2 floats apart)
#pragma unroll 1
  for (int w = 0; w < 8; ++w) {
    if (warp == w) {
#pragma unroll
      for (int e = 0; e < EB; ++e) {
        s_part[e][2 * lane] = (w == 0) ? acc[e].x : s_part[e][2 * lane] + acc[e].x;
        s_part[e][2 * lane + 1] = (w == 0) ? acc[e].y : s_part[e][2 * lane + 1] + acc[e].y;
      }
    }
    __syncthreads();
  }
  if (bias_cluster) {
    if (lane < EB) s_bsum[warp][lane] = bacc;
    __syncthreads();
    if (tid < EB) {
      float v = s_bsum[0][tid];
      for (int w = 1; w < 8; ++w) v += s_bsum[w][tid];
      s_bias[tid] = v;
    }
  }
  cluster.sync();  // every CTA's partial sums are in its shared memory
  if (rank == 0) {
    for (int i = tid; i < kRwFeat * E; i += 256) {
      const int ff = i / E, e = i - ff * E;
      float v = 0.f;
      for (int rr = 0; rr < split; ++rr) v += cluster.map_shared_rank(&s_part[e][ff], rr)[0];
      if (d0 + ff < Dm) dw_r[static_cast<int64_t>(d0 + ff) * E + e] = v;
    }
    if (bias_cluster)
      for (int e = tid; e < E; e += 256) {
        float v = 0.f;
        for (int rr = 0; rr < split; ++rr) v += cluster.map_shared_rank(&s_bias[e], rr)[0];
        dbias[e] = v;
      }
  }
  cluster.sync();  // no CTA exits while CTA 0 still reads its shared memory
}

unsigned grid_for(int64_t work_items, int per_block) {
  const int64_t g = (work_items + per_block - 1) / per_block;
  return static_cast<unsigned>(std::max<int64_t>(1, std::min<int64_t>(g, device_sm_count() * 16)));
}

}  // namespace

cudaError_t launch_scale_gather(const void* dout, int64_t R, int k, int N,
                                const int32_t* sorted_slot, const float* topk_w, void* dst,
                                cudaStream_t stream) {
  if (R == 0) return cudaSuccess;
  scale_gather_kernel<<<grid_for(R, kThreads / 32), kThreads, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(dout), R, k, N, sorted_slot, topk_w,
      static_cast<__nv_bfloat16*>(dst));
  return cudaGetLastError();
}

cudaError_t launch_gate_bwd(const float* uz, const float* gp, int64_t T, int k, int De,
                            const int32_t* slot_pos, void* dhz, cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  gate_bwd_kernel<<<grid_for(T * (De / 4), kThreads), kThreads, 0, stream>>>(
      uz, gp, T, k, De, slot_pos, static_cast<__nv_bfloat16*>(dhz));
  return cudaGetLastError();
}

cudaError_t launch_route_wgrad(const void* x, bool bf16, int64_t T, int Dm, int E,
                               const float* dlogits, float* dw_r, float* dbias,
                               cudaStream_t stream) {
  // experts rounded up to 4, 8, 16, 32 or 64 (the padded columns are zero)
  const int eb = E <= 4 ? 4 : E <= 8 ? 8 : E <= 16 ? 16 : E <= 32 ? 32 : 64;
  // Token split (the cluster size): as many CTAs as are resident on the SMs
  // at once (one wave), at most kRwMaxSplit per 64-feature block.
  const int blocks = (Dm + kRwFeat - 1) / kRwFeat;
  // x[da], x[da + 1] as one aligned load: even d_model and an aligned base
  const size_t esz = bf16 ? 2 : 4;
  const bool pair = Dm % 2 == 0 && (reinterpret_cast<uintptr_t>(x) % (2 * esz)) == 0;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(256, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  auto go = [&](auto kern, auto xp) -> cudaError_t {
    // the largest split whose clusters (one per feature block) are all
    // resident at once
    int split = 1;
    for (int sp = kRwMaxSplit; sp > 1; --sp) {
      attr[0].val.clusterDim.x = static_cast<unsigned>(sp);
      cfg.gridDim = dim3(static_cast<unsigned>(blocks * sp), 1, 1);
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) == cudaSuccess && n >= blocks) {
        split = sp;
        break;
      }
    }
    (void)cudaGetLastError();  // a refused query leaves no error behind
    attr[0].val.clusterDim.x = static_cast<unsigned>(split);
    cfg.gridDim = dim3(static_cast<unsigned>(blocks * split), 1, 1);
    return cudaLaunchKernelEx(&cfg, kern, xp, T, Dm, E, dlogits, dw_r, dbias, pair);
  };
#define ROM_RWG_CASE(EBV)                                                              \
  if (eb == EBV)                                                                       \
    return bf16 ? go(route_wgrad_kernel<EBV, __nv_bfloat16>,                           \
                     static_cast<const __nv_bfloat16*>(x))                             \
                : go(route_wgrad_kernel<EBV, float>, static_cast<const float*>(x));
  ROM_RWG_CASE(4)
  ROM_RWG_CASE(8)
  ROM_RWG_CASE(16)
  ROM_RWG_CASE(32)
  ROM_RWG_CASE(64)
#undef ROM_RWG_CASE
  return cudaErrorInvalidValue;
}

cudaError_t launch_route_probs(const void* x, bool bf16, int64_t T, int Dm, const float* w_r,
                               const float* bias, int E, float* probs, cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  const unsigned grid = grid_for(T, 8);
  if (bf16)
    route_probs_kernel<__nv_bfloat16><<<grid, 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(x), T, Dm, w_r, bias, E, probs);
  else
    route_probs_kernel<float><<<grid, 256, 0, stream>>>(static_cast<const float*>(x), T, Dm, w_r,
                                                         bias, E, probs);
  return cudaGetLastError();
}

cudaError_t launch_route_bwd(int64_t T, int k, int E, int Dm, const int32_t* topk_idx,
                             const float* topk_w, const float* probs, const float* dr_part,
                             int n_parts, const float* dx_slots, const float* w_r, float* dlogits,
                             void* dx, cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  // W_r^T slice: all of d_model when E * Dm floats fit in 160 KB.
  const int ds_max = (160 * 1024 / 4 / E) / 128 * 128;
  const int DS = std::min((Dm + 127) / 128 * 128, std::max(128, ds_max));
  const size_t smem = static_cast<size_t>(E) * DS * sizeof(float);
  cudaError_t err = cudaFuncSetAttribute(route_bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  const unsigned grid =
      static_cast<unsigned>(std::min<int64_t>((T + 31) / 32, device_sm_count()));
  route_bwd_kernel<<<grid, kRouteBwdThreads, smem, stream>>>(
      T, k, E, Dm, topk_idx, topk_w, probs, dr_part, n_parts, dx_slots, w_r, dlogits,
      static_cast<__nv_bfloat16*>(dx), DS);
  return cudaGetLastError();
}

}  // namespace rom
