// float32 grouped GEMM of the RoM expert projections on the CUDA cores (FFMA).
// Same semantics and epilogues as the tensor-core kernel; used for float32
// data, where tensor-core tf32 would not meet a 1e-5 relative tolerance.
// ("Routing Mamba ..." chapterpal summary page, Knowl 1.)
//
// One CTA per 64 x 64 output tile (x2 for Conv+Gate: u and z), 256 threads,
// each owning a 4 x 4 block; K advances 16 at a time through shared memory.
// The tile list is rebuilt on the device from `offsets`; CTAs past its end
// exit at once.
#include <math.h>

#include "rom_internal.cuh"

namespace rom {
namespace {

constexpr int TM = 64, TN = 64, TK = 16;
constexpr int kThreads = 256;

template <int MODE>
__global__ void __launch_bounds__(kThreads)
    simt_grouped_gemm_kernel(const float* __restrict__ A, int64_t R, int K,
                             const float* __restrict__ W0, const float* __restrict__ W1, int N,
                             int E, int k, const int32_t* __restrict__ offsets,
                             const int32_t* __restrict__ sorted_slot,
                             const float* __restrict__ topk_w, float* __restrict__ out) {
  constexpr bool kGate = (MODE == kEpiGateH || MODE == kEpiGateSlots);
  __shared__ int s_off[kMaxExperts + 1];
  __shared__ int s_start[kMaxExperts + 1];
  __shared__ int s_mt[kMaxExperts];
  __shared__ float sA[TK][TM + 4];
  __shared__ float sB0[TK][TN + 4];
  __shared__ float sB1[kGate ? TK : 1][TN + 4];
  const int tid = threadIdx.x;
  const int n_tiles_n = (N + TN - 1) / TN;
  // No offsets: one expert owns all R rows (a dense projection).
  for (int i = tid; i <= E; i += kThreads)
    s_off[i] = offsets ? offsets[i] : (i == 0 ? 0 : static_cast<int>(R));
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    for (int e = 0; e < E; ++e) {
      s_mt[e] = (s_off[e + 1] - s_off[e] + TM - 1) / TM;
      s_start[e] = run;
      run += s_mt[e] * n_tiles_n;
    }
    s_start[E] = run;
  }
  __syncthreads();
  const int tile = blockIdx.x;
  if (tile >= s_start[E]) return;
  int e = 0;
  while (tile >= s_start[e + 1]) ++e;
  const int local = tile - s_start[e];
  const int n_blk = local / s_mt[e];
  const int m_blk = local - n_blk * s_mt[e];
  const int n_e = s_off[e + 1] - s_off[e];
  const int64_t row_base = static_cast<int64_t>(s_off[e]) + m_blk * TM;
  const int rows_here = min(TM, n_e - m_blk * TM);
  const int n_base = n_blk * TN;
  const float* We0 = W0 + static_cast<int64_t>(e) * N * K;
  const float* We1 = kGate ? W1 + static_cast<int64_t>(e) * N * K : nullptr;

  const int tr = tid / 16, tc = tid % 16;  // 16 x 16 threads, 4 x 4 outputs each
  float acc0[4][4] = {}, acc1[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += TK) {
    for (int i = tid; i < TM * TK; i += kThreads) {
      const int r = i / TK, kk = i % TK;
      sA[kk][r] = (r < rows_here && k0 + kk < K) ? A[(row_base + r) * K + k0 + kk] : 0.f;
    }
    for (int i = tid; i < TN * TK; i += kThreads) {
      const int n = i / TK, kk = i % TK;
      const bool ok = (n_base + n < N && k0 + kk < K);
      sB0[kk][n] = ok ? We0[static_cast<int64_t>(n_base + n) * K + k0 + kk] : 0.f;
      if (kGate) sB1[kk][n] = ok ? We1[static_cast<int64_t>(n_base + n) * K + k0 + kk] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < TK; ++kk) {
      float a[4], b0[4], b1[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = sA[kk][tr * 4 + i];
        b0[i] = sB0[kk][tc * 4 + i];
        if (kGate) b1[i] = sB1[kk][tc * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc0[i][j] = fmaf(a[i], b0[j], acc0[i][j]);
          if (kGate) acc1[i][j] = fmaf(a[i], b1[j], acc1[i][j]);
        }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = tr * 4 + i;
    if (r >= rows_here) continue;
    const int64_t prow = row_base + r;
    const int64_t slot = (MODE == kEpiGateH) ? 0 : (sorted_slot ? sorted_slot[prow] : prow);
    const float rw = (MODE == kEpiScaleToken || MODE == kEpiScaleSlots)
                         ? (topk_w ? topk_w[slot] : 1.f)  // no weights passed: r = 1
                         : 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n_base + tc * 4 + j;
      if (n >= N) continue;
      if (MODE == kEpiGateH) {
        const float z = acc1[i][j];
        out[prow * N + n] = acc0[i][j] * (z / (1.0f + expf(-z)));
      } else if (MODE == kEpiGateSlots) {
        out[slot * N + n] = acc0[i][j];
        out[(R + slot) * N + n] = acc1[i][j];
      } else if (MODE == kEpiScaleToken) {
        out[(slot / k) * N + n] = rw * acc0[i][j];
      } else {
        out[slot * N + n] = rw * acc0[i][j];
      }
    }
  }
}

}  // namespace

cudaError_t launch_simt_grouped_gemm(int mode, const float* a_sorted, int64_t R, int K,
                                     const float* w0, const float* w1, int N, int E, int k,
                                     const int32_t* offsets, const int32_t* sorted_slot,
                                     const float* topk_w, float* out, cudaStream_t stream) {
  if (R == 0) return cudaSuccess;
  const int64_t n_tiles_n = (N + TN - 1) / TN;
  const int64_t max_tiles = ((R + TM - 1) / TM + E) * n_tiles_n;
  if (max_tiles >= (int64_t(1) << 31)) return cudaErrorInvalidValue;
  const unsigned grid = static_cast<unsigned>(max_tiles);
  switch (mode) {
    case kEpiGateH:
      simt_grouped_gemm_kernel<kEpiGateH><<<grid, kThreads, 0, stream>>>(
          a_sorted, R, K, w0, w1, N, E, k, offsets, sorted_slot, topk_w, out);
      break;
    case kEpiGateSlots:
      simt_grouped_gemm_kernel<kEpiGateSlots><<<grid, kThreads, 0, stream>>>(
          a_sorted, R, K, w0, w1, N, E, k, offsets, sorted_slot, topk_w, out);
      break;
    case kEpiScaleToken:
      simt_grouped_gemm_kernel<kEpiScaleToken><<<grid, kThreads, 0, stream>>>(
          a_sorted, R, K, w0, w1, N, E, k, offsets, sorted_slot, topk_w, out);
      break;
    case kEpiScaleSlots:
      simt_grouped_gemm_kernel<kEpiScaleSlots><<<grid, kThreads, 0, stream>>>(
          a_sorted, R, K, w0, w1, N, E, k, offsets, sorted_slot, topk_w, out);
      break;
    default:
      return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace rom
