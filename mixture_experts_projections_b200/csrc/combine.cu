// Slot reduction for top-k > 1 ("Routing Mamba ..." chapterpal summary page,
// Knowl 1):
//  - SUM:  O_t = sum_j (slot j's r-weighted Out projection), summed in slot
//          order 0..k-1 in float32;
//  - GATE: H_t = sum_j u_{t,j}, the pre-activation Z_t = sum_j z_{t,j}, and
//          h_t = H_t * SiLU(Z_t) (SiLU after the sum over the selected
//          experts; the identity stands in for the conv + SSM core), written
//          in expert-sorted order for every slot of the token so that the Out
//          projection can read it as its A operand. u and z may come from
//          two different routings (independently routed MoE-Mamba, Knowl 4);
//  - GATE_DENSE: as GATE, but H_t = u_t is one dense Conv projection per token
//          (the "RoM (Gate, Out)" variant of Knowl 3).
// Both are bandwidth-bound: one thread handles 4 consecutive columns (16-byte
// loads), the grid strides over tokens x column groups.
#include <cuda_bf16.h>
#include <math.h>

#include <algorithm>

#include "rom_internal.cuh"

namespace rom {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ void store4(float* out, int64_t idx, float4 v) {
  *reinterpret_cast<float4*>(out + idx) = v;
}
__device__ __forceinline__ void store4(__nv_bfloat16* out, int64_t idx, float4 v) {
  const __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y);
  const __nv_bfloat162 b = __floats2bfloat162_rn(v.z, v.w);
  uint2 w;
  w.x = *reinterpret_cast<const uint32_t*>(&a);
  w.y = *reinterpret_cast<const uint32_t*>(&b);
  *reinterpret_cast<uint2*>(out + idx) = w;
}

template <typename OutT>
__global__ void __launch_bounds__(kThreads)
    combine_sum_kernel(const float* __restrict__ in, int64_t T, int k, int N,
                       OutT* __restrict__ out) {
  const int nq = N / 4;
  const int64_t total = T * nq;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(kThreads) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * kThreads) {
    const int64_t t = i / nq;
    const int c = static_cast<int>(i - t * nq) * 4;
    float4 s = __ldg(reinterpret_cast<const float4*>(in + (t * k) * N + c));
    for (int j = 1; j < k; ++j) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(in + (t * k + j) * N + c));
      s.x += v.x;
      s.y += v.y;
      s.z += v.z;
      s.w += v.w;
    }
    store4(out, t * N + c, s);
  }
}

__device__ __forceinline__ float silu_mul(float h, float z) { return h * (z / (1.0f + expf(-z))); }

template <typename OutT>
__global__ void __launch_bounds__(kThreads)
    combine_gate_kernel(const float* __restrict__ in, int64_t T, int k, int N,
                        const int32_t* __restrict__ slot_pos, OutT* __restrict__ out) {
  const int nq = N / 4;
  const int64_t total = T * nq;
  const int64_t R = T * k;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(kThreads) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * kThreads) {
    const int64_t t = i / nq;
    const int c = static_cast<int>(i - t * nq) * 4;
    float4 u = __ldg(reinterpret_cast<const float4*>(in + (t * k) * N + c));
    float4 z = __ldg(reinterpret_cast<const float4*>(in + (R + t * k) * N + c));
    for (int j = 1; j < k; ++j) {
      const float4 a = __ldg(reinterpret_cast<const float4*>(in + (t * k + j) * N + c));
      const float4 b = __ldg(reinterpret_cast<const float4*>(in + (R + t * k + j) * N + c));
      u.x += a.x;
      u.y += a.y;
      u.z += a.z;
      u.w += a.w;
      z.x += b.x;
      z.y += b.y;
      z.z += b.z;
      z.w += b.w;
    }
    const float4 h = make_float4(silu_mul(u.x, z.x), silu_mul(u.y, z.y), silu_mul(u.z, z.z),
                                 silu_mul(u.w, z.w));
    if (!slot_pos) {
      store4(out, t * N + c, h);  // token order (a dense Out projection)
    } else {
      for (int j = 0; j < k; ++j)
        store4(out, static_cast<int64_t>(slot_pos[t * k + j]) * N + c, h);
    }
  }
}

// in = [T + T*k][N]: the dense u per token, then the gate partials per slot.
template <typename OutT>
__global__ void __launch_bounds__(kThreads)
    combine_gate_dense_kernel(const float* __restrict__ in, int64_t T, int k, int N,
                              const int32_t* __restrict__ slot_pos, OutT* __restrict__ out) {
  const int nq = N / 4;
  const int64_t total = T * nq;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(kThreads) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * kThreads) {
    const int64_t t = i / nq;
    const int c = static_cast<int>(i - t * nq) * 4;
    const float4 u = __ldg(reinterpret_cast<const float4*>(in + t * N + c));
    float4 z = __ldg(reinterpret_cast<const float4*>(in + (T + t * k) * N + c));
    for (int j = 1; j < k; ++j) {
      const float4 b = __ldg(reinterpret_cast<const float4*>(in + (T + t * k + j) * N + c));
      z.x += b.x;
      z.y += b.y;
      z.z += b.z;
      z.w += b.w;
    }
    const float4 h = make_float4(silu_mul(u.x, z.x), silu_mul(u.y, z.y), silu_mul(u.z, z.z),
                                 silu_mul(u.w, z.w));
    if (!slot_pos) {
      store4(out, t * N + c, h);  // token order (a dense Out projection)
    } else {
      for (int j = 0; j < k; ++j)
        store4(out, static_cast<int64_t>(slot_pos[t * k + j]) * N + c, h);
    }
  }
}

}  // namespace

cudaError_t launch_combine(int mode, bool bf16, const float* in, int64_t T, int k, int N,
                           const int32_t* slot_pos, void* out, cudaStream_t stream) {
  const int64_t total = T * (N / 4);
  if (total == 0) return cudaSuccess;
  const int64_t grid =
      std::min<int64_t>((total + kThreads - 1) / kThreads, static_cast<int64_t>(device_sm_count()) * 16);
  if (mode == 0) {
    if (bf16)
      combine_sum_kernel<<<static_cast<unsigned>(grid), kThreads, 0, stream>>>(
          in, T, k, N, static_cast<__nv_bfloat16*>(out));
    else
      combine_sum_kernel<<<static_cast<unsigned>(grid), kThreads, 0, stream>>>(
          in, T, k, N, static_cast<float*>(out));
  } else if (mode == 1) {
    if (bf16)
      combine_gate_kernel<<<static_cast<unsigned>(grid), kThreads, 0, stream>>>(
          in, T, k, N, slot_pos, static_cast<__nv_bfloat16*>(out));
    else
      combine_gate_kernel<<<static_cast<unsigned>(grid), kThreads, 0, stream>>>(
          in, T, k, N, slot_pos, static_cast<float*>(out));
  } else {
    if (bf16)
      combine_gate_dense_kernel<<<static_cast<unsigned>(grid), kThreads, 0, stream>>>(
          in, T, k, N, slot_pos, static_cast<__nv_bfloat16*>(out));
    else
      combine_gate_dense_kernel<<<static_cast<unsigned>(grid), kThreads, 0, stream>>>(
          in, T, k, N, slot_pos, static_cast<float*>(out));
  }
  return cudaGetLastError();
}

}  // namespace rom
