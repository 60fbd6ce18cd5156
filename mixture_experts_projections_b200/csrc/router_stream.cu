// Streaming router for bf16 activations ("Routing Mamba ..." chapterpal
// summary page, Knowl 1: p_t = Softmax(x_t W_r), S_t = the K largest
// probabilities, r_{t,i} = p_{t,i} 1[i in S_t]).
//
// One CTA owns a 128-token tile (= one histogram chunk of the dispatch) at a
// time. A producer warp streams the tile's X in 64-feature blocks through a
// TMA ring (128 x 64 bf16, 128-byte swizzle); the router weight W_r^T stays
// resident in shared memory as float32 [E][d_model].
// 4 Q compute warps (Q = 4 feature quarters for E <= 8, Q = 2 halves for
// E = 16, whose larger W_r leaves less shared memory): warp w owns tokens
// 32 (w % 4) .. +31 (one token per lane) and feature part h = w / 4 (64 / Q
// features) of every block. A lane reads its token's features of the block
// from shared memory and the weights as broadcast float4 reads, accumulates
// a block partial per expert sequentially in float32 FMA and adds it to its
// running sum. The h > 0 warps hand their sums (and |x|^2) to the h = 0 warp
// of the same tokens, which adds them in order h = 1 .. Q-1. Each logit
// therefore goes through at most 64 / Q + ceil(d_model / 64) + (Q - 1) + 1
// roundings in a fixed order; with |x| and |w_e| this bounds its error by
// gamma_n |x| |w_e| (Cauchy-Schwarz). A token whose selected logits' lower
// bounds do not all clear the upper bound of every expert ranked after them
// is re-decided on float64 logits (warp-cooperative, weights from shared
// memory). Equal logits go to the lower expert index.
// Every wait is bounded; no block-wide barrier follows the set-up.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>
#include <math.h>

#include <algorithm>
#include <mutex>

#include "rom_internal.cuh"
#include "sm100_ptx.cuh"

namespace rom {
namespace {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int A_BYTES = BM * BK * 2;  // 16 KB per stage
constexpr int kMaxStages = 8;

template <int Q>
struct Geo {
  static constexpr int kCompute = 4 * Q;               // compute warps
  static constexpr int kThreads = 32 * (1 + kCompute);  // + the producer warp
  static constexpr int kFeat = BK / Q;                  // features per warp per block
};

template <int EB, int Q>
struct SCtl {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  uint64_t part_ready[4][2];
  uint64_t part_free[4][2];
  uint64_t wload;
  int abort;
  int done[2];
  int hist[2][EB];
  float wnorm[EB];
  float part[2][Q - 1][BM][EB + 1];  // h > 0 sums (+ |x|^2 in the last column)
  double l64[4][EB];
};

__device__ __forceinline__ uint32_t sw128_off(int n, int k) {
  const uint32_t o = static_cast<uint32_t>(n) * 128u + static_cast<uint32_t>(k) * 2u;
  return o ^ (((o >> 7) & 7u) << 4);
}

template <int EB, int Q>
__global__ void __launch_bounds__(Geo<Q>::kThreads, 1)
    router_stream_kernel(const __grid_constant__ CUtensorMap tmX,
                         const __nv_bfloat16* __restrict__ x, int64_t T, int Dm,
                         const float* __restrict__ w_r, const float* __restrict__ bias, int E,
                         int k, int renorm, int32_t* __restrict__ topk_idx,
                         float* __restrict__ topk_w, int32_t* __restrict__ counts,
                         int32_t* __restrict__ chunk_hist, int64_t ntiles, int stages,
                         int DW, float gamma, int* status) {
  using Ctl = SCtl<EB, Q>;
  constexpr int kThreads = Geo<Q>::kThreads;
  constexpr int kCompute = Geo<Q>::kCompute;
  constexpr int FQ = Geo<Q>::kFeat;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base, kept as a shared-memory pointer (an offset into
  // the shared array, not an integer round-trip) so accesses stay LDS/STS.
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  Ctl& ctl = *reinterpret_cast<Ctl*>(smem + stages * A_BYTES);
  float* sW = reinterpret_cast<float*>(smem + stages * A_BYTES +
                                       ((sizeof(Ctl) + 15) / 16) * 16);  // [DW][EB]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int KB = (Dm + BK - 1) / BK;

  // W_r as stored, [d_model][E] float32 (E == EB here), copied by the bulk
  // copy engine; rows d_model .. DW-1 are zero.
  for (int i = tid; i < (DW - Dm) * EB; i += kThreads) sW[Dm * EB + i] = 0.f;
  for (int i = tid; i < 2 * EB; i += kThreads) (&ctl.hist[0][0])[i] = 0;
  if (tid == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&ctl.full[s], 1);
      mbar_init(&ctl.empty[s], kCompute);
    }
    for (int g = 0; g < 4; ++g)
      for (int p = 0; p < 2; ++p) {
        mbar_init(&ctl.part_ready[g][p], Q - 1);
        mbar_init(&ctl.part_free[g][p], 1);
      }
    mbar_init(&ctl.wload, 1);
    ctl.abort = 0;
    ctl.done[0] = ctl.done[1] = 0;
    fence_barrier_init();
  }
  __syncthreads();
  volatile int* abort_flag = &ctl.abort;
  if (tid == 0) {
    const uint32_t bytes = static_cast<uint32_t>(Dm) * EB * 4u;
    mbar_arrive_expect_tx(&ctl.wload, bytes);
    for (uint32_t off = 0; off < bytes; off += 32768u) {
      const uint32_t n = (bytes - off < 32768u) ? bytes - off : 32768u;
      bulk_load(reinterpret_cast<uint8_t*>(sW) + off,
                reinterpret_cast<const uint8_t*>(w_r) + off, n, &ctl.wload);
    }
  }

  if (warp == 0) {
    // -------------------------------------------------- TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmX);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, last_par = 0;
      bool ok = true;
      for (int64_t tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&ctl.empty[stage], phase ^ 1u, abort_flag, status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&ctl.full[stage], A_BYTES);
          tma_load_2d(smem + stage * A_BYTES, &tmX, &ctl.full[stage], kb * BK,
                      static_cast<int>(tile * BM));
          issued |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
          if (++stage == stages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      int never = 0;
      for (int s = 0; s < stages; ++s)
        if ((issued >> s) & 1u) mbar_wait(&ctl.full[s], (last_par >> s) & 1u, &never, status);
    }
    return;
  }

  // ---------------------------------------------------- compute warps
  // (the producer streams X meanwhile)
  const int cw = warp - 1;  // 0 .. kCompute-1
  const int g = cw & 3, h = cw >> 2;
  const int row = 32 * g + lane;
  {
    int never = 0;
    mbar_wait(&ctl.wload, 0, &never, status);
  }
  for (int e = cw; e < EB; e += kCompute) {
    float q = 0.f;
    for (int d = lane; d < Dm; d += 32) q = fmaf(sW[d * EB + e], sW[d * EB + e], q);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
    if (lane == 0) ctl.wnorm[e] = sqrtf(q);
  }
  // The norms are read by the deciding warps: a barrier over the compute
  // warps only (every compute warp reaches it; the producer does not take part).
  named_barrier_sync(1, 32 * kCompute);
  int stage = 0;
  uint32_t phase = 0;
  int tpar = 0;
  uint32_t tphase = 0;
  for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
    float acc[EB];
#pragma unroll
    for (int e = 0; e < EB; ++e) acc[e] = 0.f;
    float sq = 0.f;
    bool ok = true;
    for (int kb = 0; kb < KB; ++kb) {
      if (!__all_sync(0xffffffffu, mbar_wait(&ctl.full[stage], phase, abort_flag, status))) {
        ok = false;
        break;
      }
      const uint8_t* sa = smem + stage * A_BYTES;
      float xs[FQ];
#pragma unroll
      for (int j = 0; j < FQ / 8; ++j) {
        const uint4 v = *reinterpret_cast<const uint4*>(sa + sw128_off(row, FQ * h + 8 * j));
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          xs[8 * j + 2 * i] = __uint_as_float(w[i] << 16);
          xs[8 * j + 2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl.empty[stage]);  // x is in registers
      if (++stage == stages) {
        stage = 0;
        phase ^= 1u;
      }
      const float* wrow = sW + static_cast<int64_t>(kb * BK + FQ * h) * EB;
#pragma unroll
      for (int i = 0; i < FQ; ++i) sq = fmaf(xs[i], xs[i], sq);
      // block partials, two experts per packed FMA; per expert the FQ
      // features are accumulated in order
      float2 p2[EB / 2];
#pragma unroll
      for (int e2 = 0; e2 < EB / 2; ++e2) p2[e2] = make_float2(0.f, 0.f);
#pragma unroll
      for (int i = 0; i < FQ; ++i) {
        const float2 xx = make_float2(xs[i], xs[i]);
        const float4* wv = reinterpret_cast<const float4*>(wrow + i * EB);
#pragma unroll
        for (int e4 = 0; e4 < EB / 4; ++e4) {
          const float4 w4 = wv[e4];
          p2[2 * e4] = __ffma2_rn(xx, make_float2(w4.x, w4.y), p2[2 * e4]);
          p2[2 * e4 + 1] = __ffma2_rn(xx, make_float2(w4.z, w4.w), p2[2 * e4 + 1]);
        }
      }
#pragma unroll
      for (int e2 = 0; e2 < EB / 2; ++e2) {
        const float2 a2 = __fadd2_rn(make_float2(acc[2 * e2], acc[2 * e2 + 1]), p2[e2]);
        acc[2 * e2] = a2.x;
        acc[2 * e2 + 1] = a2.y;
      }
    }
    if (!ok) break;
    if (h > 0) {
      // hand the part sums to the h = 0 warp of the same tokens
      if (!__all_sync(0xffffffffu,
                      mbar_wait(&ctl.part_free[g][tpar], tphase ^ 1u, abort_flag, status)))
        break;
#pragma unroll
      for (int e = 0; e < EB; ++e) ctl.part[tpar][h - 1][row][e] = acc[e];
      ctl.part[tpar][h - 1][row][EB] = sq;
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl.part_ready[g][tpar]);
    } else {
      if (!__all_sync(0xffffffffu,
                      mbar_wait(&ctl.part_ready[g][tpar], tphase, abort_flag, status)))
        break;
#pragma unroll
      for (int hh = 0; hh < Q - 1; ++hh) {
#pragma unroll
        for (int e = 0; e < EB; ++e) acc[e] += ctl.part[tpar][hh][row][e];
        sq += ctl.part[tpar][hh][row][EB];
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl.part_free[g][tpar]);

      // ------------------------------------------------ decisions
      const int64_t tok = tile * BM + row;
      const bool valid = tok < T;
      const float xn = sqrtf(sq);
      float l[EB], err[EB];
#pragma unroll
      for (int e = 0; e < EB; ++e) {
        if (e < E) {
          l[e] = acc[e] + (bias ? __ldg(bias + e) : 0.f);
          err[e] = gamma * xn * ctl.wnorm[e] + 1.2e-7f * fabsf(l[e]);
        } else {
          l[e] = -INFINITY;
          err[e] = 0.f;
        }
      }
      int sel[kMaxTopK + 1];
      uint64_t used = 0;
#pragma unroll
      for (int j = 0; j <= kMaxTopK; ++j) {
        sel[j] = -1;
        if (j <= k) {
          int bi = -1;
          float bv = 0.f;
#pragma unroll
          for (int e = 0; e < EB; ++e)
            if (e < E && !((used >> e) & 1ull) && (bi < 0 || l[e] > bv)) {
              bi = e;
              bv = l[e];
            }
          sel[j] = bi;
          if (bi >= 0) used |= 1ull << bi;
        }
      }
      auto pick = [&](const float (&a)[EB], int i) {
        float r = 0.f;
#pragma unroll
        for (int e = 0; e < EB; ++e) r = (e == i) ? a[e] : r;
        return r;
      };
      // Certain when, for every slot j < k, the lower bound of the j-th
      // selected logit clears the upper bound of every expert ranked after
      // it (the bounds differ per expert through |w_e|).
      bool certain = true;
      uint64_t above = 0;
#pragma unroll
      for (int j = 0; j < kMaxTopK; ++j)
        if (j < k) {
          const int a = sel[j];
          above |= 1ull << a;
          const float lb = pick(l, a) - pick(err, a);
#pragma unroll
          for (int e = 0; e < EB; ++e)
            if (e < E && !((above >> e) & 1ull) && !(lb > l[e] + err[e])) certain = false;
        }
      unsigned todo = __ballot_sync(0xffffffffu, valid && !certain);
      while (todo) {
        const int src = __ffs(todo) - 1;
        todo &= todo - 1;
        const int64_t tr = __shfl_sync(0xffffffffu, tok, src);
        // float64 logits of token tr: lane i takes the 16-byte pieces
        // i, i + 32, ... of the row (8 features each), four loads in flight.
        const uint4* xr = reinterpret_cast<const uint4*>(x + tr * Dm);
        const int npc = Dm / 8;
        double a[EB];
#pragma unroll
        for (int e = 0; e < EB; ++e) a[e] = 0.0;
        for (int pc0 = lane; pc0 < npc; pc0 += 4 * 32) {
          uint4 v[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int pc = pc0 + 32 * u;
            v[u] = (pc < npc) ? __ldg(xr + pc) : make_uint4(0u, 0u, 0u, 0u);
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int pc = pc0 + 32 * u;
            if (pc >= npc) break;
            const uint32_t w4[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const uint32_t bits = (j & 1) ? (w4[j >> 1] & 0xFFFF0000u) : (w4[j >> 1] << 16);
              const double xv = static_cast<double>(__uint_as_float(bits));
              const float* wr = sW + static_cast<int64_t>(pc * 8 + j) * EB;
#pragma unroll
              for (int e = 0; e < EB; ++e) a[e] = fma(xv, static_cast<double>(wr[e]), a[e]);
            }
          }
        }
#pragma unroll
        for (int e = 0; e < EB; ++e) {
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) a[e] += __shfl_xor_sync(0xffffffffu, a[e], o);
        }
        if (lane == src)
#pragma unroll
          for (int e = 0; e < EB; ++e)
            if (e < E) ctl.l64[g][e] = a[e] + (bias ? static_cast<double>(bias[e]) : 0.0);
        __syncwarp();
        if (lane == src) {
          uint64_t u2 = 0;
          for (int j = 0; j <= kMaxTopK; ++j) {
            sel[j] = -1;
            if (j <= k) {
              int bi = -1;
              double bv = 0.0;
              for (int e = 0; e < E; ++e)
                if (!((u2 >> e) & 1ull) && (bi < 0 || ctl.l64[g][e] > bv)) {
                  bi = e;
                  bv = ctl.l64[g][e];
                }
              sel[j] = bi;
              if (bi >= 0) u2 |= 1ull << bi;
            }
          }
#pragma unroll
          for (int e = 0; e < EB; ++e) l[e] = (e < E) ? static_cast<float>(ctl.l64[g][e]) : -INFINITY;
        }
        __syncwarp();
      }
      if (valid) {
        const float m = pick(l, sel[0]);
        float den = 0.f;
        if (renorm) {
#pragma unroll
          for (int j = 0; j < kMaxTopK; ++j)
            if (j < k) den += expf(pick(l, sel[j]) - m);
        } else {
#pragma unroll
          for (int e = 0; e < EB; ++e)
            if (e < E) den += expf(l[e] - m);
        }
#pragma unroll
        for (int j = 0; j < kMaxTopK; ++j)
          if (j < k) {
            topk_idx[tok * k + j] = sel[j];
            topk_w[tok * k + j] = expf(pick(l, sel[j]) - m) / den;
            atomicAdd(&ctl.hist[tpar][sel[j]], 1);
          }
      }
      // The last of the four deciding warps publishes the tile's histogram.
      __threadfence_block();
      __syncwarp();
      int last = 0;
      if (lane == 0) last = (atomicAdd(&ctl.done[tpar], 1) == 3);
      last = __shfl_sync(0xffffffffu, last, 0);
      if (last) {
        __threadfence_block();
        for (int e = lane; e < E; e += 32) {
          const int v = atomicExch(&ctl.hist[tpar][e], 0);
          chunk_hist[tile * E + e] = v;
          if (counts && v) atomicAdd(counts + e, v);
        }
        if (lane == 0) ctl.done[tpar] = 0;
        __threadfence_block();
      }
    }
    tpar ^= 1;
    if (tpar == 0) tphase ^= 1u;
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

template <int EB, int Q>
cudaError_t launch_eb(const void* x, int64_t T, int Dm, const float* w_r, const float* bias, int E,
                      int k, int renorm, int32_t* topk_idx, float* topk_w, int32_t* counts,
                      int32_t* chunk_hist, int* status, cudaStream_t stream) {
  const int64_t ntiles = num_chunks(T);
  const int DW = (Dm + BK - 1) / BK * BK;
  const size_t ctl = (sizeof(SCtl<EB, Q>) + 15) / 16 * 16;
  const size_t wbytes = static_cast<size_t>(EB) * DW * sizeof(float);
  const size_t budget = 224 * 1024;
  int stages = kMaxStages;
  while (stages >= 2 && stages * A_BYTES + ctl + wbytes + 1024 > budget) --stages;
  if (stages < 2) return cudaErrorNotSupported;  // the weight does not stay resident
  if (ntiles == 0) return cudaSuccess;
  auto fn = encode_fn();
  if (!fn) return cudaErrorInvalidValue;
  CUtensorMap tm;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(Dm), static_cast<cuuint64_t>(T)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(Dm) * 2};
  cuuint32_t box[2] = {BK, BM};
  cuuint32_t estr[2] = {1, 1};
  if (fn(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), dims, strides, box, estr,
         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  // Longest rounding chain of a logit: 64 / Q block FMAs, one add per
  // block, Q - 1 adds of the parts, the bias (+1 spare); 1 % slack covers
  // the norms.
  const double n = static_cast<double>(Geo<Q>::kFeat) +
                   static_cast<double>((Dm + BK - 1) / BK) + static_cast<double>(Q - 1) + 2.0;
  const double u = 1.0 / 16777216.0;
  const float gamma = static_cast<float>(1.01 * n * u / (1.0 - n * u));
  const size_t smem = stages * A_BYTES + ctl + wbytes + 1024;
  auto kern = router_stream_kernel<EB, Q>;
  cudaError_t err =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  const int grid = static_cast<int>(std::min<int64_t>(ntiles, device_sm_count()));
  kern<<<grid, Geo<Q>::kThreads, smem, stream>>>(tm, static_cast<const __nv_bfloat16*>(x), T, Dm, w_r,
                                         bias, E, k, renorm, topk_idx, topk_w, counts, chunk_hist,
                                         ntiles, stages, DW, gamma, status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_router_stream(const void* x, int64_t T, int Dm, const float* w_r,
                                 const float* bias, int E, int k, int renorm, int32_t* topk_idx,
                                 float* topk_w, int32_t* counts, int32_t* chunk_hist, int* status,
                                 cudaStream_t stream) {
  // W_r is staged as stored ([d_model][E], 16-byte rows): E in {4, 8, 16}.
  if (reinterpret_cast<uintptr_t>(w_r) & 15u) return cudaErrorNotSupported;
  if (E == 4)
    return launch_eb<4, 4>(x, T, Dm, w_r, bias, E, k, renorm, topk_idx, topk_w, counts, chunk_hist,
                        status, stream);
  if (E == 8)
    return launch_eb<8, 4>(x, T, Dm, w_r, bias, E, k, renorm, topk_idx, topk_w, counts, chunk_hist,
                        status, stream);
  if (E == 16)
    return launch_eb<16, 2>(x, T, Dm, w_r, bias, E, k, renorm, topk_idx, topk_w, counts, chunk_hist,
                         status, stream);
  return cudaErrorNotSupported;  // other expert counts use the register-tiled kernel
}

}  // namespace rom
