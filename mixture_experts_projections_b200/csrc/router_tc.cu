// Router of the RoM block for bf16 activations, on the tensor cores
// ("Routing Mamba ..." chapterpal summary page, Knowl 1: p_t =
// Softmax(x_t W_r), S_t = the K largest probabilities, r_{t,i} = p_{t,i}
// 1[i in S_t]).
//
// The logits x_t W_r are a skinny GEMM (E columns) that streams X once, so
// the kernel is a TMA-fed tcgen05 GEMM over 128-token tiles (one tile = one
// histogram chunk of the dispatch):
//  * W_r (float32) is split on the fly into three bf16 parts
//    w = hi + lo + lo2 (hi = bf16(w), lo = bf16(w - hi), lo2 = bf16(w - hi - lo)),
//    so every product x_i * part_i is exact in float32; the producer warp
//    writes the three parts as the B tile (rows part * EP + e) directly in
//    the 128-byte-swizzled K-major layout, next to the TMA-loaded X tile.
//  * two "norm" warps accumulate |x_t|^2 from the same shared-memory X tiles,
//    sequentially per token.
//  * the epilogue (one thread per token) forms l_e = (hi_e + lo_e) + lo2_e
//    (+ bias), bounds its rounding error by g |x_t| |w_e| + 2u|l_e| with
//    g = gamma_{2(n+8)} (every addition inside the tensor core counted as
//    an error of up to 2 ulp, n = d_model) and |hi|+|lo|+|lo2| <= (1+2^-7)|w|,
//    selects the top k (+1) by value (equal values: lower expert index),
//    and when a deciding gap is not larger than the two bounds recomputes
//    that token's logits in float64 (warp-cooperative) before deciding.
//    Softmax in float32; outputs and a per-tile expert histogram.
// Warps: 0 producer (lane 0 issues TMA, all lanes build B), 1 MMA issuer and
// TMEM owner, 2-5 epilogue, 6-7 norms. Every wait is bounded.
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
constexpr int kThreads = 256;
constexpr int A_BYTES = BM * BK * 2;

template <int EP>
struct RCfg {
  static constexpr int NP = 3 * EP;                       // MMA N: hi | lo | lo2
  static constexpr int B_BYTES = NP * BK * 2;
  static constexpr int STAGE_BYTES = ((A_BYTES + B_BYTES) + 1023) / 1024 * 1024;
  static constexpr int STAGES = (200 * 1024 / STAGE_BYTES) < 6 ? (200 * 1024 / STAGE_BYTES) : 6;
  // accumulator column stride: a power of two >= NP; two accumulators
  static constexpr uint32_t ACC_STRIDE = NP <= 16 ? 16 : NP <= 32 ? 32 : NP <= 64 ? 64 : NP <= 128 ? 128 : 256;
  static constexpr uint32_t TMEM_COLS = 2 * ACC_STRIDE < 32 ? 32 : 2 * ACC_STRIDE;
};

struct RCtl {
  uint64_t full[8];
  uint64_t empty[8];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  float sq[2][BM];
  int hist[2][kMaxExperts];
  int done[2];
  float wnorm[kMaxExperts];
  double l64[4][kMaxExperts];
};

__device__ __forceinline__ uint16_t bf16_bits_rn(float v) {
  const __nv_bfloat16 b = __float2bfloat16_rn(v);
  return *reinterpret_cast<const uint16_t*>(&b);
}
__device__ __forceinline__ float bf16_to_f(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// Byte offset of element (row n, k) in a K-major 128-byte-swizzled tile.
__device__ __forceinline__ uint32_t sw128_off(int n, int k) {
  const uint32_t o = static_cast<uint32_t>(n) * 128u + static_cast<uint32_t>(k) * 2u;
  return o ^ (((o >> 7) & 7u) << 4);
}

template <int EP>
__global__ void __launch_bounds__(kThreads, 1)
    router_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __nv_bfloat16* __restrict__ x,
                     int64_t T, int Dm, const float* __restrict__ w_r,
                     const float* __restrict__ bias, int E, int k, int renorm,
                     int32_t* __restrict__ topk_idx, float* __restrict__ topk_w,
                     int32_t* __restrict__ counts, int32_t* __restrict__ chunk_hist,
                     int64_t ntiles, float gbound, int* status) {
  using C = RCfg<EP>;
  constexpr int NP = C::NP, STAGES = C::STAGES, STAGE_BYTES = C::STAGE_BYTES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  RCtl& ctl = *reinterpret_cast<RCtl*>(smem + STAGES * STAGE_BYTES);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int KB = (Dm + BK - 1) / BK;

  // Zero every B region once (the padding rows e >= E stay zero), |w_e|.
  for (int s = 0; s < STAGES; ++s) {
    uint4* b = reinterpret_cast<uint4*>(smem + s * STAGE_BYTES + A_BYTES);
    for (int i = tid; i < C::B_BYTES / 16; i += kThreads) b[i] = make_uint4(0u, 0u, 0u, 0u);
  }
  for (int e = warp; e < E; e += kThreads / 32) {
    float q = 0.f;
    for (int d = lane; d < Dm; d += 32) {
      const float w = __ldg(w_r + static_cast<int64_t>(d) * E + e);
      q = fmaf(w, w, q);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
    if (lane == 0) ctl.wnorm[e] = sqrtf(q);
  }
  for (int e = tid; e < 2 * kMaxExperts; e += kThreads) (&ctl.hist[0][0])[e] = 0;
  if (tid < 2) ctl.done[tid] = 0;
  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&ctl.full[s], 2);
      mbar_init(&ctl.empty[s], 3);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&ctl.tfull[a], 3);
      mbar_init(&ctl.tempty[a], 4);
    }
    mbar_init(&ctl.drain, 1);
    ctl.abort = 0;
    fence_barrier_init();
  }
  fence_async_shared();  // the zeroed B regions are read by the tensor cores
  if (warp == 0 && lane == 0) tma_prefetch_desc(&tmX);
  if (warp == 1) {
    tmem_alloc(&ctl.tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = ctl.tmem_base;
  volatile int* abort_flag = &ctl.abort;

  if (warp == 0) {
    // -------------------------------------------------- producer warp
    // Lane L owns features d0 + L and d0 + L + 32 of each K block: it loads
    // their E router weights (contiguous in w_r) and writes the three bf16
    // parts into the B tile. For E <= 16 the next block's weights are loaded
    // while the current block is converted.
    constexpr bool kPrefetch = EP <= 16;
    float wcur[2][EP], wnext[2][EP];
    const bool vec4 = (E % 4) == 0;
    auto load_w = [&](int kb, float (&dst)[2][EP]) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int d = kb * BK + lane + 32 * h;
        const float* src = w_r + static_cast<int64_t>(d) * E;
        if (d < Dm && vec4) {
#pragma unroll
          for (int e4 = 0; e4 < EP / 4; ++e4) {
            if (4 * e4 < E) {
              const float4 v = __ldg(reinterpret_cast<const float4*>(src) + e4);
              dst[h][4 * e4] = v.x;
              dst[h][4 * e4 + 1] = v.y;
              dst[h][4 * e4 + 2] = v.z;
              dst[h][4 * e4 + 3] = v.w;
            } else {
              dst[h][4 * e4] = dst[h][4 * e4 + 1] = dst[h][4 * e4 + 2] = dst[h][4 * e4 + 3] = 0.f;
            }
          }
        } else {
#pragma unroll
          for (int e = 0; e < EP; ++e) dst[h][e] = (d < Dm && e < E) ? __ldg(src + e) : 0.f;
        }
      }
    };
    int stage = 0;
    uint32_t phase = 0;
    uint32_t issued = 0, last_par = 0;
    bool ok = true;
    bool have_next = false;
    for (int64_t tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
      for (int kb = 0; kb < KB; ++kb) {
        if constexpr (kPrefetch) {
          if (have_next) {
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
              for (int e = 0; e < EP; ++e) wcur[h][e] = wnext[h][e];
          } else {
            load_w(kb, wcur);
          }
          const int nkb = (kb + 1 < KB) ? kb + 1 : 0;  // the next tile restarts at block 0
          load_w(nkb, wnext);
          have_next = true;
        } else {
          load_w(kb, wcur);
        }
        // every lane waits (and acquires); the outcome is made warp-uniform
        const bool got = mbar_wait(&ctl.empty[stage], phase ^ 1u, abort_flag, status);
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
        uint8_t* sa = smem + stage * STAGE_BYTES;
        uint8_t* sb = sa + A_BYTES;
        if (lane == 0) {
          mbar_arrive_expect_tx(&ctl.full[stage], A_BYTES);
          tma_load_2d(sa, &tmX, &ctl.full[stage], kb * BK, static_cast<int>(tile * BM));
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int d = lane + 32 * h;
#pragma unroll
          for (int e = 0; e < EP; ++e) {
            if (e < E) {
              const float w = wcur[h][e];
              const uint16_t hi = bf16_bits_rn(w);
              const float r1 = w - bf16_to_f(hi);
              const uint16_t lo = bf16_bits_rn(r1);
              const uint16_t lo2 = bf16_bits_rn(r1 - bf16_to_f(lo));
              *reinterpret_cast<uint16_t*>(sb + sw128_off(e, d)) = hi;
              *reinterpret_cast<uint16_t*>(sb + sw128_off(EP + e, d)) = lo;
              *reinterpret_cast<uint16_t*>(sb + sw128_off(2 * EP + e, d)) = lo2;
            }
          }
        }
        fence_async_shared();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&ctl.full[stage]);
          issued |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
        }
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (lane == 0) {
      int never = 0;
      for (int s = 0; s < STAGES; ++s)
        if ((issued >> s) & 1u) mbar_wait(&ctl.full[s], (last_par >> s) & 1u, &never, status);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer
      const uint32_t idesc = idesc_bf16_f32(BM, NP);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int64_t tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
        if (!mbar_wait(&ctl.tempty[acc], acc_phase ^ 1u, abort_flag, status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc) * C::ACC_STRIDE;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&ctl.full[stage], phase, abort_flag, status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + stage * STAGE_BYTES);
          const uint32_t b_addr = a_addr + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            mma_bf16_ss(d_tmem, sw128_kmajor_desc(a_addr + kk * 32),
                        sw128_kmajor_desc(b_addr + kk * 32), idesc, (kb | kk) != 0);
          mma_commit(&ctl.empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit(&ctl.tfull[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      mma_commit(&ctl.drain);
      int never = 0;
      mbar_wait(&ctl.drain, 0, &never, status);
    }
  } else if (warp >= 6) {
    // -------------------------------------------------- norm warps: |x|^2
    const int r0 = (warp - 6) * 64 + lane, r1 = r0 + 32;
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    for (int64_t tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
      if (!__all_sync(0xffffffffu, mbar_wait(&ctl.tempty[acc], acc_phase ^ 1u, abort_flag, status)))
        break;
      float q0 = 0.f, q1 = 0.f;
      for (int kb = 0; kb < KB; ++kb) {
        if (!__all_sync(0xffffffffu, mbar_wait(&ctl.full[stage], phase, abort_flag, status))) {
          ok = false;
          break;
        }
        const uint8_t* sa = smem + stage * STAGE_BYTES;
#pragma unroll
        for (int j = 0; j < 8; ++j) {  // logical 16-byte chunk j of the row
          const uint4 v0 = *reinterpret_cast<const uint4*>(sa + sw128_off(r0, 8 * j));
          const uint4 v1 = *reinterpret_cast<const uint4*>(sa + sw128_off(r1, 8 * j));
          const uint32_t a[4] = {v0.x, v0.y, v0.z, v0.w};
          const uint32_t b[4] = {v1.x, v1.y, v1.z, v1.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float a0 = __uint_as_float(a[i] << 16), a1 = __uint_as_float(a[i] & 0xFFFF0000u);
            const float b0 = __uint_as_float(b[i] << 16), b1 = __uint_as_float(b[i] & 0xFFFF0000u);
            q0 = fmaf(a0, a0, q0);
            q0 = fmaf(a1, a1, q0);
            q1 = fmaf(b0, b0, q1);
            q1 = fmaf(b1, b1, q1);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl.empty[stage]);
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
      ctl.sq[acc][r0] = q0;
      ctl.sq[acc][r1] = q1;
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl.tfull[acc]);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
  } else {
    // -------------------------------------------------- epilogue (warps 2..5)
    const int q = warp & 3;
    const int ew = warp - 2;  // 0..3
    const int row = q * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
      if (!__all_sync(0xffffffffu, mbar_wait(&ctl.tfull[acc], acc_phase, abort_flag, status))) break;
      tc_fence_after();
      const uint32_t t_row =
          tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc) * C::ACC_STRIDE;
      float l[EP];
#pragma unroll
      for (int c = 0; c < EP / 16; ++c) {
        uint32_t h[16], a[16], b[16];
        tmem_ld16(t_row + c * 16, h);
        tmem_ld16(t_row + EP + c * 16, a);
        tmem_ld16(t_row + 2 * EP + c * 16, b);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i)
          l[c * 16 + i] = (__uint_as_float(h[i]) + __uint_as_float(a[i])) + __uint_as_float(b[i]);
      }
      const float sqv = ctl.sq[acc][row];
      tc_fence_before();

      const int64_t tok = tile * BM + row;
      const bool valid = tok < T;
      const float xn = sqrtf(sqv);
      float err[EP];
#pragma unroll
      for (int e = 0; e < EP; ++e) {
        if (e < E) {
          l[e] += bias ? __ldg(bias + e) : 0.f;
          err[e] = gbound * xn * ctl.wnorm[e] + 2.4e-7f * fabsf(l[e]);
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
          for (int e = 0; e < EP; ++e)
            if (e < E && !((used >> e) & 1ull) && (bi < 0 || l[e] > bv)) {
              bi = e;
              bv = l[e];
            }
          sel[j] = bi;
          if (bi >= 0) used |= 1ull << bi;
        }
      }
      auto pick = [&](const float (&a)[EP], int i) {
        float r = 0.f;
#pragma unroll
        for (int e = 0; e < EP; ++e) r = (e == i) ? a[e] : r;
        return r;
      };
      bool certain = true;
#pragma unroll
      for (int j = 0; j < kMaxTopK; ++j)
        if (j < k && sel[j + 1] >= 0) {
          const int a = sel[j], b = sel[j + 1];
          if (!(pick(l, a) - pick(l, b) > pick(err, a) + pick(err, b))) certain = false;
        }
      unsigned todo = __ballot_sync(0xffffffffu, valid && !certain);
      while (todo) {
        const int src = __ffs(todo) - 1;
        todo &= todo - 1;
        const int64_t tr = __shfl_sync(0xffffffffu, tok, src);
        const __nv_bfloat16* xr = x + tr * Dm;
        for (int e0 = 0; e0 < E; e0 += 16) {
          double a[16];
#pragma unroll
          for (int g = 0; g < 16; ++g) a[g] = 0.0;
          for (int d = lane; d < Dm; d += 32) {
            const double xv = static_cast<double>(__bfloat162float(xr[d]));
#pragma unroll
            for (int g = 0; g < 16; ++g)
              if (e0 + g < E) a[g] = fma(xv, static_cast<double>(__ldg(w_r + static_cast<int64_t>(d) * E + e0 + g)), a[g]);
          }
#pragma unroll
          for (int g = 0; g < 16; ++g) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) a[g] += __shfl_xor_sync(0xffffffffu, a[g], o);
          }
          if (lane == src)
#pragma unroll
            for (int g = 0; g < 16; ++g)
              if (e0 + g < E) ctl.l64[ew][e0 + g] = a[g] + (bias ? static_cast<double>(bias[e0 + g]) : 0.0);
        }
        __syncwarp();
        if (lane == src) {
          uint64_t u2 = 0;
#pragma unroll
          for (int j = 0; j <= kMaxTopK; ++j) {
            sel[j] = -1;
            if (j <= k) {
              int bi = -1;
              double bv = 0.0;
              for (int e = 0; e < E; ++e)
                if (!((u2 >> e) & 1ull) && (bi < 0 || ctl.l64[ew][e] > bv)) {
                  bi = e;
                  bv = ctl.l64[ew][e];
                }
              sel[j] = bi;
              if (bi >= 0) u2 |= 1ull << bi;
            }
          }
#pragma unroll
          for (int e = 0; e < EP; ++e) l[e] = (e < E) ? static_cast<float>(ctl.l64[ew][e]) : -INFINITY;
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
          for (int e = 0; e < EP; ++e)
            if (e < E) den += expf(l[e] - m);
        }
#pragma unroll
        for (int j = 0; j < kMaxTopK; ++j)
          if (j < k) {
            topk_idx[tok * k + j] = sel[j];
            topk_w[tok * k + j] = expf(pick(l, sel[j]) - m) / den;
            atomicAdd(&ctl.hist[acc][sel[j]], 1);
          }
      }
      // The last of the four epilogue warps to finish this tile publishes
      // its histogram (no block-wide barrier: every wait stays bounded).
      __threadfence_block();
      __syncwarp();
      int last = 0;
      if (lane == 0) last = (atomicAdd(&ctl.done[acc], 1) == 3);
      last = __shfl_sync(0xffffffffu, last, 0);
      if (last) {
        __threadfence_block();
        for (int e = lane; e < E; e += 32) {
          const int v = atomicExch(&ctl.hist[acc][e], 0);
          chunk_hist[tile * E + e] = v;
          if (counts && v) atomicAdd(counts + e, v);
        }
        if (lane == 0) ctl.done[acc] = 0;
        __threadfence_block();
      }
      // The accumulator and this histogram buffer are free again.
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl.tempty[acc]);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
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

template <int EP>
cudaError_t launch_ep(const void* x, int64_t T, int Dm, const float* w_r, const float* bias, int E,
                      int k, int renorm, int32_t* topk_idx, float* topk_w, int32_t* counts,
                      int32_t* chunk_hist, int* status, cudaStream_t stream) {
  using C = RCfg<EP>;
  const int64_t ntiles = num_chunks(T);
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
  // Rounding bound of the tensor-core logits (see the header comment).
  const double n = 2.0 * (Dm + 8);
  const double u = 1.0 / 16777216.0;
  const float gbound = static_cast<float>(1.02 * (1.0 + 1.0 / 128) * n * u / (1.0 - n * u));
  const size_t smem = static_cast<size_t>(C::STAGES) * C::STAGE_BYTES + sizeof(RCtl) + 1024;
  auto kern = router_tc_kernel<EP>;
  cudaError_t err =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  const int grid = static_cast<int>(std::min<int64_t>(ntiles, device_sm_count()));
  kern<<<grid, kThreads, smem, stream>>>(tm, static_cast<const __nv_bfloat16*>(x), T, Dm, w_r, bias,
                                         E, k, renorm, topk_idx, topk_w, counts, chunk_hist,
                                         ntiles, gbound, status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_router_tc(const void* x, int64_t T, int Dm, const float* w_r, const float* bias,
                             int E, int k, int renorm, int32_t* topk_idx, float* topk_w,
                             int32_t* counts, int32_t* chunk_hist, int* status,
                             cudaStream_t stream) {
#define ROM_RTC_CASE(EPV)                                                                     \
  if (E <= EPV)                                                                               \
    return launch_ep<EPV>(x, T, Dm, w_r, bias, E, k, renorm, topk_idx, topk_w, counts,        \
                          chunk_hist, status, stream);
  ROM_RTC_CASE(16)
  ROM_RTC_CASE(32)
  ROM_RTC_CASE(48)
  ROM_RTC_CASE(64)
#undef ROM_RTC_CASE
  return cudaErrorInvalidValue;
}

}  // namespace rom
