// Grouped bf16 GEMM of the RoM expert projections on the 5th-generation tensor
// cores (tcgen05.mma, fp32 accumulators in TMEM, operands staged by TMA).
// ("Routing Mamba ..." chapterpal summary page, Knowl 1: H_t, G_t and O_t are
// linear projections by the selected experts; Swimba project page, Extended
// abstract: routed in-projection experts.)
//
// For expert e the rows offsets[e] .. offsets[e+1]-1 of A ([R][K] bf16,
// expert-contiguous) are multiplied by B_e^T, B_e = W[e] stored [N][K]. The
// expert row counts are read on the device: each CTA rebuilds the tile list
// from `offsets` (no host synchronisation). Tiles never straddle experts;
// rows past an expert's end are computed and discarded at the store.
//
// Tile: 128 rows x 256 accumulator columns x 64-element K steps.
//   Conv+Gate: the 256 columns are 128 columns of W_in next to the same 128
//   columns of W_g, so one MMA of N = 256 yields u and z side by side, and the
//   epilogue forms h = u * SiLU(z) (top-1) or stores u and z per slot (top-k).
//   Out / in-projection: 256 output columns, scaled by r in the epilogue (a
//   last tile of 128 columns when N % 256 == 128: the weight rows past N are
//   zero-filled by TMA and those columns are not stored).
// CTA: persistent (one per SM), 6 warps:
//   warp 0  TMA producer (one thread), 4-stage shared-memory ring (48 KB/stage)
//   warp 1  TMEM allocator and MMA issuer (one thread)
//   warps 2-5  epilogue; warp w reads TMEM lanes 32*(w%4) .. +31
// Two TMEM accumulators (2 x 256 columns) let the epilogue of one tile run
// while the MMAs of the next tile proceed. Every wait is bounded.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "rom_internal.cuh"
#include "sm100_ptx.cuh"

namespace rom {
namespace {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int UMMA_N = 256;
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;      // 16 KB
constexpr int B_BYTES = UMMA_N * BK * 2;  // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr uint32_t TMEM_COLS = 2 * UMMA_N;
constexpr int kThreads = 192;
// Out / in-projection calls with at most this many routed rows use the
// swap-AB kernel (weights on the MMA's M side).
constexpr int64_t kSwapMaxRows = 1024;

struct Params {
  const int32_t* offsets;
  const int32_t* sorted_slot;
  const float* topk_w;
  void* out;
  int64_t R;
  int K;
  int N;
  int E;
  int k;
  int n_tiles_n;
  int* status;
};

struct SmemCtl {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int tile_start[kMaxExperts + 1];
  int off[kMaxExperts + 1];
  int mt[kMaxExperts];
};

constexpr size_t kSmemBytes = STAGES * STAGE_BYTES + sizeof(SmemCtl) + 1024;

__device__ __forceinline__ void tile_coords(const SmemCtl& c, int tile, int& e, int& m_blk,
                                            int& n_blk) {
  e = 0;
  while (tile >= c.tile_start[e + 1]) ++e;
  const int local = tile - c.tile_start[e];
  n_blk = local / c.mt[e];
  m_blk = local - n_blk * c.mt[e];
}

__device__ __forceinline__ float silu_gate(float u, float z) {
  return u * (z / (1.0f + expf(-z)));
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&v);
}

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    tc_grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                           const __grid_constant__ CUtensorMap tmB0,
                           const __grid_constant__ CUtensorMap tmB1, const Params p) {
  constexpr bool kGate = (MODE == kEpiGateH || MODE == kEpiGateSlots);
  constexpr int kTileN = kGate ? 128 : 256;  // output columns per tile
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base, kept as a shared-memory pointer (an offset into
  // the shared array, not an integer round-trip) so accesses stay LDS/STS.
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  SmemCtl& ctl = *reinterpret_cast<SmemCtl*>(smem + STAGES * STAGE_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = p.E;

  for (int i = threadIdx.x; i <= E; i += kThreads) ctl.off[i] = p.offsets[i];
  __syncthreads();
  if (threadIdx.x == 0) {
    int run = 0;
    for (int e = 0; e < E; ++e) {
      const int mt = (ctl.off[e + 1] - ctl.off[e] + BM - 1) / BM;
      ctl.mt[e] = mt;
      ctl.tile_start[e] = run;
      run += mt * p.n_tiles_n;
    }
    ctl.tile_start[E] = run;
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&ctl.full[s], 1);
      mbar_init(&ctl.empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&ctl.tfull[a], 1);
      mbar_init(&ctl.tempty[a], 4);
    }
    mbar_init(&ctl.drain, 1);
    ctl.abort = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB0);
    if (kGate) tma_prefetch_desc(&tmB1);
  }
  if (warp == 1) {
    tmem_alloc(&ctl.tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = ctl.tmem_base;
  const int total = ctl.tile_start[E];
  const int KB = (p.K + BK - 1) / BK;
  volatile int* abort_flag = &ctl.abort;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, last_par = 0;  // per-stage: ever armed, parity of last arming
      for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
        int e, m_blk, n_blk;
        tile_coords(ctl, tile, e, m_blk, n_blk);
        const int row0 = ctl.off[e] + m_blk * BM;
        const int n0 = n_blk * kTileN;
        bool ok = true;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&ctl.empty[stage], phase ^ 1u, abort_flag, p.status)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + stage * STAGE_BYTES;
          uint8_t* sb = sa + A_BYTES;
          mbar_arrive_expect_tx(&ctl.full[stage], STAGE_BYTES);
          tma_load_2d(sa, &tmA, &ctl.full[stage], kb * BK, row0);
          if (kGate) {
            tma_load_3d(sb, &tmB0, &ctl.full[stage], kb * BK, n0, e);
            tma_load_3d(sb + B_BYTES / 2, &tmB1, &ctl.full[stage], kb * BK, n0, e);
          } else {
            tma_load_3d(sb, &tmB0, &ctl.full[stage], kb * BK, n0, e);
          }
          issued |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
      }
      // No TMA write may still be landing when the CTA exits.
      int never = 0;
      for (int s = 0; s < STAGES; ++s)
        if ((issued >> s) & 1u) mbar_wait(&ctl.full[s], (last_par >> s) & 1u, &never, p.status);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer
      const uint32_t idesc = idesc_bf16_f32(BM, UMMA_N);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        if (!mbar_wait(&ctl.tempty[acc], acc_phase ^ 1u, abort_flag, p.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * UMMA_N);
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&ctl.full[stage], phase, abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + stage * STAGE_BYTES);
          const uint32_t b_addr = a_addr + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            mma_bf16_ss(d_tmem, sw128_kmajor_desc(a_addr + kk * 32),
                        sw128_kmajor_desc(b_addr + kk * 32), idesc, (kb | kk) != 0);
          }
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
      // Every issued MMA has completed before TMEM is released.
      mma_commit(&ctl.drain);
      int never = 0;
      mbar_wait(&ctl.drain, 0, &never, p.status);
    }
  } else {
    // -------------------------------------------------- epilogue (warps 2..5)
    const int q = warp & 3;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
      int e, m_blk, n_blk;
      tile_coords(ctl, tile, e, m_blk, n_blk);
      if (!mbar_wait(&ctl.tfull[acc], acc_phase, abort_flag, p.status)) break;
      tc_fence_after();
      const int row_local = m_blk * BM + q * 32 + lane;
      const bool valid = row_local < ctl.off[e + 1] - ctl.off[e];
      const int64_t prow = static_cast<int64_t>(ctl.off[e]) + row_local;
      const uint32_t t_row =
          tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * UMMA_N);
      const int n0 = n_blk * kTileN;
      if (MODE == kEpiGateH) {
        __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out);
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t u[32], z[32];
          tmem_ld32(t_row + c * 32, u);
          tmem_ld32(t_row + 128 + c * 32, z);
          tmem_ld_wait();
          if (valid) {
            uint4* dst = reinterpret_cast<uint4*>(out + prow * p.N + n0 + c * 32);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              uint4 w;
              w.x = pack_bf16(silu_gate(__uint_as_float(u[8 * v + 0]), __uint_as_float(z[8 * v + 0])),
                              silu_gate(__uint_as_float(u[8 * v + 1]), __uint_as_float(z[8 * v + 1])));
              w.y = pack_bf16(silu_gate(__uint_as_float(u[8 * v + 2]), __uint_as_float(z[8 * v + 2])),
                              silu_gate(__uint_as_float(u[8 * v + 3]), __uint_as_float(z[8 * v + 3])));
              w.z = pack_bf16(silu_gate(__uint_as_float(u[8 * v + 4]), __uint_as_float(z[8 * v + 4])),
                              silu_gate(__uint_as_float(u[8 * v + 5]), __uint_as_float(z[8 * v + 5])));
              w.w = pack_bf16(silu_gate(__uint_as_float(u[8 * v + 6]), __uint_as_float(z[8 * v + 6])),
                              silu_gate(__uint_as_float(u[8 * v + 7]), __uint_as_float(z[8 * v + 7])));
              dst[v] = w;
            }
          }
        }
      } else if (MODE == kEpiGateSlots) {
        float* out = static_cast<float*>(p.out);
        const int64_t slot = valid ? p.sorted_slot[prow] : 0;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t u[32], z[32];
          tmem_ld32(t_row + c * 32, u);
          tmem_ld32(t_row + 128 + c * 32, z);
          tmem_ld_wait();
          if (valid) {
            uint4* du = reinterpret_cast<uint4*>(out + slot * p.N + n0 + c * 32);
            uint4* dz = reinterpret_cast<uint4*>(out + (p.R + slot) * p.N + n0 + c * 32);
#pragma unroll
            for (int v = 0; v < 8; ++v) {
              du[v] = make_uint4(u[4 * v], u[4 * v + 1], u[4 * v + 2], u[4 * v + 3]);
              dz[v] = make_uint4(z[4 * v], z[4 * v + 1], z[4 * v + 2], z[4 * v + 3]);
            }
          }
        }
      } else {
        const int64_t slot = valid ? p.sorted_slot[prow] : 0;
        const float r = valid ? p.topk_w[slot] : 0.f;
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
          if (n0 + c * 32 >= p.N) break;  // partial last tile (N % 256 == 128)
          uint32_t a[32];
          tmem_ld32(t_row + c * 32, a);
          tmem_ld_wait();
          if (valid) {
            if (MODE == kEpiScaleToken) {
              __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out);
              uint4* dst = reinterpret_cast<uint4*>(out + (slot / p.k) * p.N + n0 + c * 32);
#pragma unroll
              for (int v = 0; v < 4; ++v) {
                uint4 w;
                w.x = pack_bf16(r * __uint_as_float(a[8 * v + 0]), r * __uint_as_float(a[8 * v + 1]));
                w.y = pack_bf16(r * __uint_as_float(a[8 * v + 2]), r * __uint_as_float(a[8 * v + 3]));
                w.z = pack_bf16(r * __uint_as_float(a[8 * v + 4]), r * __uint_as_float(a[8 * v + 5]));
                w.w = pack_bf16(r * __uint_as_float(a[8 * v + 6]), r * __uint_as_float(a[8 * v + 7]));
                dst[v] = w;
              }
            } else {
              float* out = static_cast<float*>(p.out);
              float4* dst = reinterpret_cast<float4*>(out + slot * p.N + n0 + c * 32);
#pragma unroll
              for (int v = 0; v < 8; ++v)
                dst[v] = make_float4(r * __uint_as_float(a[4 * v]), r * __uint_as_float(a[4 * v + 1]),
                                     r * __uint_as_float(a[4 * v + 2]), r * __uint_as_float(a[4 * v + 3]));
            }
          }
        }
      }
      tc_fence_before();
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
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// Swap-AB variant for few tokens per expert (decode): the weight rows are the
// MMA's M side (128 per tile) and the expert's tokens its N side (64 per
// tile), so a tile streams 128 x K of weights once and the tile count is
// E x N/128 x ceil(n_e / 64) -- enough tiles to cover the SMs even when every
// expert has only a handful of tokens. Same output as the Out / in-projection
// epilogue: out[token][n] = r * acc (bf16, k == 1) or per slot in float32.
constexpr int SW_BN = 64;                      // tokens per tile (MMA N)
constexpr int SW_STAGES = 8;
constexpr int SW_A_BYTES = BM * BK * 2;        // 16 KB of weights
constexpr int SW_B_BYTES = SW_BN * BK * 2;     // 8 KB of tokens
constexpr int SW_STAGE_BYTES = SW_A_BYTES + SW_B_BYTES;
constexpr uint32_t SW_TMEM_COLS = 2 * SW_BN;

struct SwapCtl {
  uint64_t full[SW_STAGES];
  uint64_t empty[SW_STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int tile_start[kMaxExperts + 1];
  int off[kMaxExperts + 1];
  int tt[kMaxExperts];  // token tiles per expert
};

constexpr size_t kSwapSmemBytes = SW_STAGES * SW_STAGE_BYTES + sizeof(SwapCtl) + 1024;

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    tc_swap_gemm_kernel(const __grid_constant__ CUtensorMap tmW,
                        const __grid_constant__ CUtensorMap tmX, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base, kept as a shared-memory pointer (an offset into
  // the shared array, not an integer round-trip) so accesses stay LDS/STS.
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  SwapCtl& ctl = *reinterpret_cast<SwapCtl*>(smem + SW_STAGES * SW_STAGE_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = p.E;
  const int n_wt = p.N / BM;  // weight-row tiles per expert

  for (int i = threadIdx.x; i <= E; i += kThreads) ctl.off[i] = p.offsets[i];
  __syncthreads();
  if (threadIdx.x == 0) {
    int run = 0;
    for (int e = 0; e < E; ++e) {
      const int tt = (ctl.off[e + 1] - ctl.off[e] + SW_BN - 1) / SW_BN;
      ctl.tt[e] = tt;
      ctl.tile_start[e] = run;
      run += tt * n_wt;
    }
    ctl.tile_start[E] = run;
    for (int s = 0; s < SW_STAGES; ++s) {
      mbar_init(&ctl.full[s], 1);
      mbar_init(&ctl.empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&ctl.tfull[a], 1);
      mbar_init(&ctl.tempty[a], 4);
    }
    mbar_init(&ctl.drain, 1);
    ctl.abort = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmX);
  }
  if (warp == 1) {
    tmem_alloc(&ctl.tmem_base, SW_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = ctl.tmem_base;
  const int total = ctl.tile_start[E];
  const int KB = (p.K + BK - 1) / BK;
  volatile int* abort_flag = &ctl.abort;
  // tile -> (expert, weight-row block, token block); weight-row blocks vary
  // fastest so that CTAs running together share the expert's token rows.
  auto coords = [&](int tile, int& e, int& w_blk, int& t_blk) {
    e = 0;
    while (tile >= ctl.tile_start[e + 1]) ++e;
    const int local = tile - ctl.tile_start[e];
    t_blk = local / n_wt;
    w_blk = local - t_blk * n_wt;
  };

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, last_par = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        int e, w_blk, t_blk;
        coords(tile, e, w_blk, t_blk);
        const int n0 = w_blk * BM;
        const int r0 = ctl.off[e] + t_blk * SW_BN;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&ctl.empty[stage], phase ^ 1u, abort_flag, p.status)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + stage * SW_STAGE_BYTES;
          mbar_arrive_expect_tx(&ctl.full[stage], SW_STAGE_BYTES);
          tma_load_3d(sa, &tmW, &ctl.full[stage], kb * BK, n0, e);
          tma_load_2d(sa + SW_A_BYTES, &tmX, &ctl.full[stage], kb * BK, r0);
          issued |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
          if (++stage == SW_STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      int never = 0;
      for (int s = 0; s < SW_STAGES; ++s)
        if ((issued >> s) & 1u) mbar_wait(&ctl.full[s], (last_par >> s) & 1u, &never, p.status);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(BM, SW_BN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        if (!mbar_wait(&ctl.tempty[acc], acc_phase ^ 1u, abort_flag, p.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * SW_BN);
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&ctl.full[stage], phase, abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + stage * SW_STAGE_BYTES);
          const uint32_t b_addr = a_addr + SW_A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            mma_bf16_ss(d_tmem, sw128_kmajor_desc(a_addr + kk * 32),
                        sw128_kmajor_desc(b_addr + kk * 32), idesc, (kb | kk) != 0);
          mma_commit(&ctl.empty[stage]);
          if (++stage == SW_STAGES) {
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
      mbar_wait(&ctl.drain, 0, &never, p.status);
    }
  } else {
    const int q = warp & 3;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
      int e, w_blk, t_blk;
      coords(tile, e, w_blk, t_blk);
      if (!mbar_wait(&ctl.tfull[acc], acc_phase, abort_flag, p.status)) break;
      tc_fence_after();
      const uint32_t t_row =
          tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * SW_BN);
      const int n = w_blk * BM + q * 32 + lane;  // this thread's output column
      const int n_e = ctl.off[e + 1] - ctl.off[e];
#pragma unroll 1
      for (int c = 0; c < SW_BN / 32; ++c) {
        const int j0 = t_blk * SW_BN + c * 32;  // first token of this column chunk
        if (j0 >= n_e) break;
        uint32_t a[32];
        tmem_ld32(t_row + c * 32, a);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          if (j0 + j >= n_e) continue;
          const int64_t prow = ctl.off[e] + j0 + j;
          const int64_t slot = p.sorted_slot[prow];
          const float v = p.topk_w[slot] * __uint_as_float(a[j]);
          if (MODE == kEpiScaleToken)
            static_cast<__nv_bfloat16*>(p.out)[(slot / p.k) * p.N + n] = __float2bfloat16_rn(v);
          else
            static_cast<float*>(p.out)[slot * p.N + n] = v;
        }
      }
      tc_fence_before();
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
    tmem_dealloc(tmem_base, SW_TMEM_COLS);
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

// bf16 tensor map over a row-major [rows][K] matrix (or [E][rows][K] when
// experts > 0), box of box_rows x 64 elements, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, int64_t K, int64_t rows, int experts,
              int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(experts > 0 ? experts : 1)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(K * 2), static_cast<cuuint64_t>(K * 2 * rows)};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(BK), static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  const cuuint32_t rank = experts > 0 ? 3 : 2;
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims,
                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int MODE>
cudaError_t launch_mode(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                        const Params& p, int grid, cudaStream_t stream) {
  auto kern = tc_grouped_gemm_kernel<MODE>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kSmemBytes));
  if (err != cudaSuccess) return err;
  kern<<<grid, kThreads, kSmemBytes, stream>>>(a, b0, b1, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_tc_grouped_gemm(int mode, const void* a_sorted, int64_t R, int K,
                                   const void* w0, const void* w1, int N, int E, int k,
                                   const int32_t* offsets, const int32_t* sorted_slot,
                                   const float* topk_w, void* out, int* status,
                                   cudaStream_t stream) {
  const bool gate = (mode == kEpiGateH || mode == kEpiGateSlots);
  const int tile_n = gate ? 128 : 256;
  // Few tokens (decode): the swap-AB kernel streams every weight tile once.
  if (!gate && R <= kSwapMaxRows && N % BM == 0 && K % 8 == 0 && E <= kMaxExperts) {
    if (R == 0) return cudaSuccess;
    CUtensorMap tw, tx;
    if (!make_map(&tw, w0, K, N, E, BM)) return cudaErrorInvalidValue;
    if (!make_map(&tx, a_sorted, K, R, 0, SW_BN)) return cudaErrorInvalidValue;
    Params p{};
    p.offsets = offsets;
    p.sorted_slot = sorted_slot;
    p.topk_w = topk_w;
    p.out = out;
    p.R = R;
    p.K = K;
    p.N = N;
    p.E = E;
    p.k = k;
    p.status = status;
    const int64_t max_tiles = ((R + SW_BN - 1) / SW_BN + E) * static_cast<int64_t>(N / BM);
    const int grid = static_cast<int>(std::min<int64_t>(device_sm_count(), max_tiles));
    auto kern = (mode == kEpiScaleToken) ? tc_swap_gemm_kernel<kEpiScaleToken>
                                         : tc_swap_gemm_kernel<kEpiScaleSlots>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(kSwapSmemBytes));
    if (err != cudaSuccess) return err;
    kern<<<grid, kThreads, kSwapSmemBytes, stream>>>(tw, tx, p);
    return cudaGetLastError();
  }
  if (K % 8 != 0 || N % 128 != 0 || E > kMaxExperts || R >= (int64_t(1) << 31))
    return cudaErrorInvalidValue;
  if (R == 0) return cudaSuccess;
  CUtensorMap ta, tb0, tb1;
  if (!make_map(&ta, a_sorted, K, R, 0, BM)) return cudaErrorInvalidValue;
  if (!make_map(&tb0, w0, K, N, E, gate ? 128 : 256)) return cudaErrorInvalidValue;
  if (gate) {
    if (!make_map(&tb1, w1, K, N, E, 128)) return cudaErrorInvalidValue;
  } else {
    tb1 = tb0;
  }
  Params p;
  p.offsets = offsets;
  p.sorted_slot = sorted_slot;
  p.topk_w = topk_w;
  p.out = out;
  p.R = R;
  p.K = K;
  p.N = N;
  p.E = E;
  p.k = k;
  p.n_tiles_n = (N + tile_n - 1) / tile_n;
  p.status = status;
  const int64_t max_tiles = ((R + BM - 1) / BM + E) * static_cast<int64_t>(p.n_tiles_n);
  const int grid = static_cast<int>(std::min<int64_t>(device_sm_count(), max_tiles));
  switch (mode) {
    case kEpiGateH:
      return launch_mode<kEpiGateH>(ta, tb0, tb1, p, grid, stream);
    case kEpiGateSlots:
      return launch_mode<kEpiGateSlots>(ta, tb0, tb1, p, grid, stream);
    case kEpiScaleToken:
      return launch_mode<kEpiScaleToken>(ta, tb0, tb1, p, grid, stream);
    case kEpiScaleSlots:
      return launch_mode<kEpiScaleSlots>(ta, tb0, tb1, p, grid, stream);
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace rom
