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
// Tile: 256 rows x 256 accumulator columns x 64-element K steps, computed
// by a pair of CTAs on two SMs (a 2-CTA cluster, tcgen05.mma.cta_group::2):
// each CTA holds 128 of the rows and half of the 256 B columns in its shared
// memory and receives its rows' 128 x 256 fp32 accumulator in its own TMEM.
//   Conv+Gate: the 256 columns are 128 columns of W_in (held by CTA 0) next
//   to the same 128 columns of W_g (CTA 1), so one MMA of N = 256 yields u
//   and z side by side, and the epilogue forms h = u * SiLU(z) (top-1) or
//   stores u and z per slot (top-k).
//   Out / in-projection: 256 output columns, scaled by r in the epilogue (a
//   last tile of 128 columns when N % 256 == 128: the weight rows past N are
//   zero-filled by TMA and those columns are not stored).
// CTA: persistent (one pair of CTAs per pair of SMs), 6 warps:
//   warp 0  TMA producer (one thread), 6- or 7-stage ring (32 KB/stage/CTA)
//   warp 1  TMEM allocator; in CTA 0 also the MMA issuer (one thread)
//   warps 2-5  epilogue; warp w reads TMEM lanes 32*(w%4) .. +31
// Two TMEM accumulators (2 x 256 columns) let the epilogue of one tile run
// while the MMAs of the next tile proceed. Every wait is bounded.
// Few routed rows (decode) take a swap-AB kernel instead (below).
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
  // the dense small-batch in-projection: every token's experts (else null)
  const int32_t* topk_idx;
  // dense small-batch kernel: weights in the tile-major layout
  // [E][N/128][K/64][128][64] (one 16 KB block per weight tile)
  int w_tiled;
};

// u * SiLU(z) = u * z / (1 + e^-z), with the fast exp and divide intrinsics:
// their relative error (~1e-6) is far below the bf16 rounding of h (2^-9),
// and for z < -88 (e^-z = inf) the quotient is 0 as SiLU's limit.
__device__ __forceinline__ float silu_gate(float u, float z) {
  return u * __fdividef(z, 1.0f + __expf(-z));
}

// Slot of sorted row `prow` (row order itself for a dense projection, which
// passes no sorted_slot) and the expert row bounds (one expert owning all R
// rows when no offsets are passed).
__device__ __forceinline__ int64_t slot_of(const Params& p, int64_t prow) {
  return p.sorted_slot ? static_cast<int64_t>(p.sorted_slot[prow]) : prow;
}
__device__ __forceinline__ int offset_of(const Params& p, int i) {
  return p.offsets ? p.offsets[i] : (i == 0 ? 0 : static_cast<int>(p.R));
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// Epilogue of one accumulator tile for one warp: thread i reads TMEM lane
// t_row.lane + i, i.e. sorted row `prow` (stored only when `valid`), output
// columns n0 .. n0 + w - 1 (w = 128 for the gate modes, whose z columns
// follow the w u columns in TMEM, 256 otherwise; half of that for the half
// tiles of a last wave). The
// float32 outputs (per-slot partials) go row by row through the warp's
// staging tile `stg` (row-coalesced stores); the bf16 rows, half as wide,
// are stored directly in 16-byte pieces, which measured faster for them.
template <int MODE>
__device__ __forceinline__ void epilogue_rows(const Params& p, uint32_t t_row, bool valid,
                                              int64_t prow, int n0, int w, float* stg) {
  if (MODE == kEpiGateH) {
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out);
#pragma unroll 1
    for (int c = 0; c < w / 32; ++c) {
      uint32_t u[32], z[32];
      tmem_ld32(t_row + c * 32, u);
      tmem_ld32(t_row + w + c * 32, z);
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
    const int64_t slot = valid ? slot_of(p, prow) : 0;
#pragma unroll 1
    for (int c = 0; c < w / 32; ++c) {
      uint32_t u[32], z[32];
      tmem_ld32(t_row + c * 32, u);
      tmem_ld32(t_row + w + c * 32, z);
      tmem_ld_wait();
      float f[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) f[j] = __uint_as_float(u[j]);
      store_rows_f32(stg, f, valid ? out + slot * p.N + n0 + c * 32 : nullptr);
#pragma unroll
      for (int j = 0; j < 32; ++j) f[j] = __uint_as_float(z[j]);
      store_rows_f32(stg, f, valid ? out + (p.R + slot) * p.N + n0 + c * 32 : nullptr);
    }
  } else {
    const int64_t slot = valid ? slot_of(p, prow) : 0;
    // no routing weights passed: r = 1
    const float r = valid ? (p.topk_w ? p.topk_w[slot] : 1.f) : 0.f;
#pragma unroll 1
    for (int c = 0; c < w / 32; ++c) {
      if (n0 + c * 32 >= p.N) break;  // partial last tile (N % 256 == 128)
      uint32_t a[32];
      tmem_ld32(t_row + c * 32, a);
      tmem_ld_wait();
      if (MODE == kEpiScaleToken) {
        if (valid) {
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
        }
      } else {
        float f[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) f[j] = r * __uint_as_float(a[j]);
        float* out = static_cast<float*>(p.out);
        store_rows_f32(stg, f, valid ? out + slot * p.N + n0 + c * 32 : nullptr);
      }
    }
  }
}

// ---------------------------------------------------------------------------
// SM-pair variant (cluster of two CTAs, tcgen05.mma.cta_group::2): a pair
// tile is 256 rows x 256 accumulator columns. CTA v of the pair loads rows
// 128v .. 128v+127 of the tile's A rows and half of the B rows (Conv+Gate:
// CTA 0 the 128 W_in columns, CTA 1 the same 128 W_g columns; Out: CTA v
// the output columns 128v .. 128v+127), so each SM streams 32 KB per K step
// instead of 48 KB, and the 128 x 256 accumulator of its own rows lands in
// its own TMEM, where its own epilogue warps read it, one row per
// thread. Protocol:
//   full[s]   lives in CTA 0: CTA 0's producer arms it with both CTAs'
//             bytes; both producers' TMA loads complete on it.
//   empty[s]  one per CTA: the MMA commit arrives on both (multicast).
//   tfull[a]  one per CTA: the commit after a tile's last MMA, multicast.
//   tempty[a] lives in CTA 0: the 4 epilogue warps of each CTA arrive
//             (CTA 1's through the cluster window).
// A CTA never exits while the other may still touch its shared memory or
// TMEM: both end at a cluster barrier that every path reaches after bounded
// waits.
constexpr int PM = 256;                      // rows per pair tile
// Ring depth: 7 stages for the bf16-output modes, 6 (plus the epilogue
// warps' staging tiles) for the float32-output modes.
constexpr int P_MAX_STAGES = 7;
template <int MODE>
struct PairGeo {
  static constexpr bool kStaged = (MODE == kEpiGateSlots || MODE == kEpiScaleSlots);
  static constexpr int kStages = kStaged ? 6 : 7;
};
constexpr int P_A_BYTES = BM * BK * 2;       // 16 KB: this CTA's 128 rows
constexpr int P_B_BYTES = 128 * BK * 2;      // 16 KB: this CTA's half of B
constexpr int P_STAGE_BYTES = P_A_BYTES + P_B_BYTES;

struct PairCtl {
  uint64_t full[P_MAX_STAGES];
  uint64_t empty[P_MAX_STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int tile_start[kMaxExperts + 1];
  int off[kMaxExperts + 1];
  int mt[kMaxExperts];
};

constexpr size_t kPairCtlBytes = (sizeof(PairCtl) + 15) / 16 * 16;
// ring, control block, the 4 epilogue warps' staging tiles, alignment slack
template <int MODE>
constexpr size_t pair_smem_bytes() {
  return PairGeo<MODE>::kStages * P_STAGE_BYTES + kPairCtlBytes +
         (PairGeo<MODE>::kStaged ? 4 * kStageFloats * sizeof(float) : 0) + 1024;
}

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    tc_pair_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB0,
                        const __grid_constant__ CUtensorMap tmB1,
                        const __grid_constant__ CUtensorMap tmB0h,
                        const __grid_constant__ CUtensorMap tmB1h, const Params p) {
  constexpr bool kGate = (MODE == kEpiGateH || MODE == kEpiGateSlots);
  constexpr int kTileN = kGate ? 128 : 256;  // output columns per tile
  constexpr int P_STAGES = PairGeo<MODE>::kStages;
  extern __shared__ uint8_t smem_raw[];
  // Same 1024-byte aligned offset in both CTAs (same kernel, same static
  // layout), as the pair MMA reads the peer's operands at the leader's offsets.
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  PairCtl& ctl = *reinterpret_cast<PairCtl*>(smem + P_STAGES * P_STAGE_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = p.E;
  const uint32_t rank = cluster_ctarank();
  const bool leader = (rank == 0);
  const int pair = static_cast<int>(blockIdx.x >> 1);
  const int npairs = static_cast<int>(gridDim.x >> 1);

  for (int i = threadIdx.x; i <= E; i += kThreads) ctl.off[i] = offset_of(p, i);
  __syncthreads();
  if (threadIdx.x == 0) {
    int run = 0;
    for (int e = 0; e < E; ++e) {
      const int mt = (ctl.off[e + 1] - ctl.off[e] + PM - 1) / PM;
      ctl.mt[e] = mt;
      ctl.tile_start[e] = run;
      run += mt * p.n_tiles_n;
    }
    ctl.tile_start[E] = run;
    for (int s = 0; s < P_STAGES; ++s) {
      mbar_init(&ctl.full[s], 1);
      mbar_init(&ctl.empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&ctl.tfull[a], 1);
      mbar_init(&ctl.tempty[a], 8);
    }
    mbar_init(&ctl.drain, 1);
    ctl.abort = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(kGate && !leader ? &tmB1 : &tmB0);
  }
  if (warp == 1) {
    tmem_alloc_pair(&ctl.tmem_base, TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // barriers initialised in both CTAs before any remote use
  tc_fence_after();
  const uint32_t tmem_base = ctl.tmem_base;
  const int total = ctl.tile_start[E];
  const int KB = (p.K + BK - 1) / BK;
  volatile int* abort_flag = &ctl.abort;

  auto coords = [&](int tile, int& e, int& m_blk, int& n_blk) {
    e = 0;
    while (tile >= ctl.tile_start[e + 1]) ++e;
    const int local = tile - ctl.tile_start[e];
    n_blk = local / ctl.mt[e];
    m_blk = local - n_blk * ctl.mt[e];
  };
  // Work items of this pair: its whole tiles pair, pair + npairs, ... of the
  // full waves, then its item of the last wave. When the last wave holds at
  // most npairs / 2 tiles, each of them is cut into two halves of N / 2
  // columns (pair 2i and 2i + 1 take tile i's halves), so that wave keeps
  // every pair busy for half a tile's time instead of some pairs for a
  // whole one. half: -1 for a whole tile, else 0 or 1.
  const int full_waves = total / npairs;
  const int rem = total - full_waves * npairs;
  const bool halve = rem > 0 && 2 * rem <= npairs;
  auto item = [&](int j, int& tile, int& half) -> bool {
    if (j < full_waves) {
      tile = pair + j * npairs;
      half = -1;
      return true;
    }
    if (j > full_waves) return false;
    if (halve) {
      if (pair >= 2 * rem) return false;
      tile = full_waves * npairs + pair / 2;
      half = pair & 1;
      return true;
    }
    if (pair >= rem) return false;
    tile = full_waves * npairs + pair;
    half = -1;
    return true;
  };

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer (both CTAs)
      const CUtensorMap* tmB = (kGate && !leader) ? &tmB1 : &tmB0;
      const CUtensorMap* tmBh = (kGate && !leader) ? &tmB1h : &tmB0h;
      const uint32_t full0 = mapa_shared(smem_u32(&ctl.full[0]), 0);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, last_par = 0;
      bool ok = true;
      int tile, half;
      for (int j = 0; ok && item(j, tile, half); ++j) {
        int e, m_blk, n_blk;
        coords(tile, e, m_blk, n_blk);
        const int row0 = ctl.off[e] + m_blk * PM + static_cast<int>(rank) * BM;
        // B rows of this CTA: whole tile 128 (Conv+Gate: the tile's 128 W_in
        // or W_g rows; Out: its half of the 256 columns), half tile 64
        const int r = static_cast<int>(rank);
        const int brow0 = half < 0 ? (kGate ? n_blk * 128 : n_blk * 256 + r * 128)
                                   : (kGate ? n_blk * 128 + half * 64
                                            : n_blk * 256 + half * 128 + r * 64);
        const CUtensorMap* mb = half < 0 ? tmB : tmBh;
        const uint32_t bytes =
            half < 0 ? 2u * P_STAGE_BYTES : 2u * (P_A_BYTES + P_B_BYTES / 2);
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&ctl.empty[stage], phase ^ 1u, abort_flag, p.status)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + stage * P_STAGE_BYTES;
          const uint32_t fb = full0 + static_cast<uint32_t>(stage * sizeof(uint64_t));
          if (leader) mbar_arrive_expect_tx(&ctl.full[stage], bytes);
          tma_load_2d_pair(sa, &tmA, fb, kb * BK, row0);
          tma_load_3d_pair(sa + P_A_BYTES, mb, fb, kb * BK, brow0, e);
          issued |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
          if (++stage == P_STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (leader) {
        // Every load of both CTAs has landed before the pair can exit.
        int never = 0;
        for (int s = 0; s < P_STAGES; ++s)
          if ((issued >> s) & 1u) mbar_wait(&ctl.full[s], (last_par >> s) & 1u, &never, p.status);
      } else if (!ok) {
        // Aborted: this CTA's loads complete on the leader's barriers, which
        // it cannot wait on; give copies in flight a fixed time to land.
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 200000ull) {
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ------------------------------------------------ MMA issuer (CTA 0)
      const uint32_t idesc_whole = idesc_bf16_f32(PM, UMMA_N);
      const uint32_t idesc_half = idesc_bf16_f32(PM, UMMA_N / 2);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      int tile, half;
      for (int j = 0; ok && item(j, tile, half); ++j) {
        const uint32_t idesc = half < 0 ? idesc_whole : idesc_half;
        if (!mbar_wait(&ctl.tempty[acc], acc_phase ^ 1u, abort_flag, p.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * UMMA_N);
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&ctl.full[stage], phase, abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + stage * P_STAGE_BYTES);
          const uint32_t b_addr = a_addr + P_A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            mma_bf16_ss_pair(d_tmem, sw128_kmajor_desc(a_addr + kk * 32),
                             sw128_kmajor_desc(b_addr + kk * 32), idesc, (kb | kk) != 0);
          }
          mma_commit_pair_mc(&ctl.empty[stage], 0x3);
          if (++stage == P_STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit_pair_mc(&ctl.tfull[acc], 0x3);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      // Every issued MMA has completed before TMEM is released.
      mma_commit_pair(&ctl.drain);
      int never = 0;
      mbar_wait(&ctl.drain, 0, &never, p.status);
    }
  } else {
    // -------------------------------------------------- epilogue (warps 2..5)
    const int q = warp & 3;
    const uint32_t tempty0 = mapa_shared(smem_u32(&ctl.tempty[0]), 0);
    float* stg = reinterpret_cast<float*>(smem + P_STAGES * P_STAGE_BYTES + kPairCtlBytes) +
                 (warp - 2) * kStageFloats;
    int acc = 0;
    uint32_t acc_phase = 0;
    int tile, half;
    for (int j = 0; item(j, tile, half); ++j) {
      int e, m_blk, n_blk;
      coords(tile, e, m_blk, n_blk);
      if (!mbar_wait(&ctl.tfull[acc], acc_phase, abort_flag, p.status)) break;
      tc_fence_after();
      const int row_local = m_blk * PM + static_cast<int>(rank) * BM + q * 32 + lane;
      const bool valid = row_local < ctl.off[e + 1] - ctl.off[e];
      const int64_t prow = static_cast<int64_t>(ctl.off[e]) + row_local;
      const uint32_t t_row =
          tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * UMMA_N);
      const int w = half < 0 ? kTileN : kTileN / 2;
      epilogue_rows<MODE>(p, t_row, valid, prow, n_blk * kTileN + (half < 0 ? 0 : half * w), w,
                          stg);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (leader)
          mbar_arrive(&ctl.tempty[acc]);
        else
          mbar_arrive_remote(tempty0 + static_cast<uint32_t>(acc * sizeof(uint64_t)));
      }
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // neither CTA releases TMEM or exits while the other works
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// Swap-AB variant for few tokens per expert (decode): the weight rows are the
// MMA's M side (128 per tile) and the expert's tokens its N side (64 per
// tile), so a tile streams 128 x K of weights once and the tile count is
// E x N/128 x ceil(n_e / 64) -- enough tiles to cover the SMs even when every
// expert has only a handful of tokens. The kernel is bound by HBM, not by
// the SM count, so the grid is sized to give every CTA the same number of
// tiles (320 tiles: 107 CTAs of 3 tiles, not 148 CTAs and a partial wave). Same output as the Out / in-projection
// epilogue: out[token][n] = r * acc (bf16, k == 1) or per slot in float32.
constexpr int SW_BM = 128;                     // weight rows per tile (MMA M)
constexpr int SW_BN = 64;                      // tokens per tile (MMA N)
constexpr int SW_STAGES = 8;
constexpr int SW_A_BYTES = SW_BM * BK * 2;     // 16 KB of weights
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

// Output row and router weight of one token of the tile, for the lane that
// holds it (one token per lane, so the slot and weight loads of a chunk of
// 32 tokens are issued together rather than one dependent pair per store).
template <int MODE>
__device__ __forceinline__ void swap_token(const Params& p, int64_t prow, bool valid, int& orow,
                                           float& r) {
  orow = 0;
  r = 0.f;
  if (valid) {
    const int slot = static_cast<int>(slot_of(p, prow));
    r = p.topk_w ? p.topk_w[slot] : 1.f;  // no routing weights: r = 1
    orow = MODE == kEpiScaleToken ? slot / p.k : slot;
  }
}

// kDense: the small-batch form without a dispatch (T <= 64 tokens, one token
// block). Every expert's weight tiles meet all T tokens, which the producer
// loads in token order; the routing decides only which results are kept: for
// token t and expert e, the epilogue stores r * acc where e is one of t's
// selected experts and nothing otherwise. The weights stream once either
// way (each expert's tiles for its single token block), and since nothing
// before the epilogue depends on the routing, the kernel is launched as a
// programmatic dependent of the router and only its epilogue waits for it.
template <int MODE, bool kDense>
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
  const int n_wt = p.N / SW_BM;  // weight-row tiles per expert

  // Set-up that needs no routing: barriers, TMEM, tensor maps. The kernel is
  // launched as a programmatic dependent of the dispatch, so this overlaps
  // the router and the dispatch. (An L2 prefetch of each CTA's first weight
  // tile here measured no gain on the decode step: 79.9 us either way.)
  if (threadIdx.x == 0) {
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
  if (!kDense) {
    pdl_wait();  // the routing (offsets, sorted rows, weights) is complete from here
    for (int i = threadIdx.x; i <= E; i += kThreads) ctl.off[i] = offset_of(p, i);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int run = 0;
    for (int e = 0; e < E; ++e) {
      // dense: one block of all (<= 64) tokens per expert, in token order
      const int tt = kDense ? 1 : (ctl.off[e + 1] - ctl.off[e] + SW_BN - 1) / SW_BN;
      ctl.tt[e] = tt;
      ctl.tile_start[e] = run;
      run += tt * n_wt;
    }
    ctl.tile_start[E] = run;
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
        const int n0 = w_blk * SW_BM;
        const int r0 = kDense ? 0 : ctl.off[e] + t_blk * SW_BN;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&ctl.empty[stage], phase ^ 1u, abort_flag, p.status)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + stage * SW_STAGE_BYTES;
          mbar_arrive_expect_tx(&ctl.full[stage], SW_STAGE_BYTES);
          if (kDense && p.w_tiled)
            tma_load_5d(sa, &tmW, &ctl.full[stage], 0, 0, kb, w_blk, e);
          else
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
      const uint32_t idesc = idesc_bf16_f32(SW_BM, SW_BN);
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
    if (kDense) pdl_wait();  // the router's topk_idx / topk_w are complete from here
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
      int e, w_blk, t_blk;
      coords(tile, e, w_blk, t_blk);
      int nv;  // token columns of the tile that may be stored
      int orow[2];
      float rw[2];
      bool keep[2] = {true, true};
      if (kDense) {
        nv = static_cast<int>(p.R < SW_BN ? p.R : SW_BN);  // all T tokens, one block
        // column c*32 + lane is token t; kept where e is one of its experts
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int t = 32 * c + lane;
          keep[c] = false;
          orow[c] = 0;
          rw[c] = 0.f;
          if (t < nv)
            for (int j = 0; j < p.k; ++j) {
              const int64_t slot = static_cast<int64_t>(t) * p.k + j;
              if (p.topk_idx[slot] == e) {
                keep[c] = true;
                rw[c] = p.topk_w[slot];
                orow[c] = MODE == kEpiScaleToken ? t : static_cast<int>(slot);
              }
            }
        }
      } else {
        const int n_e = ctl.off[e + 1] - ctl.off[e];
        nv = min(SW_BN, n_e - t_blk * SW_BN);  // valid token columns, >= 1
        // token info first: its loads overlap the wait for the accumulator
        const int64_t prow0 = static_cast<int64_t>(ctl.off[e]) + t_blk * SW_BN;
        swap_token<MODE>(p, prow0 + lane, lane < nv, orow[0], rw[0]);
        swap_token<MODE>(p, prow0 + 32 + lane, 32 + lane < nv, orow[1], rw[1]);
      }
      if (!mbar_wait(&ctl.tfull[acc], acc_phase, abort_flag, p.status)) break;
      tc_fence_after();
      const uint32_t t_row =
          tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * SW_BN);
      const int n = w_blk * SW_BM + q * 32 + lane;  // this thread's output column
#pragma unroll
      for (int c = 0; c < SW_BN / 32; ++c) {
        if (32 * c < nv) {  // warp-uniform
          uint32_t a[32];
          tmem_ld32(t_row + c * 32, a);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            if (32 * c + j < nv) {  // warp-uniform
              const int o = __shfl_sync(0xffffffffu, orow[c], j);
              const float v = __shfl_sync(0xffffffffu, rw[c], j) * __uint_as_float(a[j]);
              const bool kept = __shfl_sync(0xffffffffu, keep[c] ? 1 : 0, j) != 0;
              const int64_t i = static_cast<int64_t>(o) * p.N + n;
              if (kept) {
                if (MODE == kEpiScaleToken)
                  static_cast<__nv_bfloat16*>(p.out)[i] = __float2bfloat16_rn(v);
                else
                  static_cast<float*>(p.out)[i] = v;
              }
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
cudaError_t launch_pair_mode(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                             const CUtensorMap& b0h, const CUtensorMap& b1h, const Params& p,
                             int64_t max_tiles, cudaStream_t stream) {
  auto kern = tc_pair_gemm_kernel<MODE>;
  constexpr size_t kPairSmemBytes = pair_smem_bytes<MODE>();
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kPairSmemBytes));
  if (err != cudaSuccess) return err;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kPairSmemBytes;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // Co-resident pairs on this device (one CTA per SM), cached per device.
  static int pairs_cache[64] = {0};
  int dev = 0;
  err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  int pairs = (dev < 64) ? pairs_cache[dev] : 0;
  if (pairs == 0) {
    cfg.gridDim = dim3(2 * 64, 1, 1);
    err = cudaOccupancyMaxActiveClusters(&pairs, kern, &cfg);
    if (err != cudaSuccess) return err;
    if (pairs <= 0) return cudaErrorNotSupported;
    if (dev < 64) pairs_cache[dev] = pairs;
  }
  const int64_t n = std::min<int64_t>(pairs, max_tiles);
  cfg.gridDim = dim3(static_cast<unsigned>(2 * n), 1, 1);
  return cudaLaunchKernelEx(&cfg, kern, a, b0, b1, b0h, b1h, p);
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
  if (!gate && R <= kSwapMaxRows && N % SW_BM == 0 && K % 8 == 0 && E <= kMaxExperts) {
    if (R == 0) return cudaSuccess;
    CUtensorMap tw, tx;
    if (!make_map(&tw, w0, K, N, E, SW_BM)) return cudaErrorInvalidValue;
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
    // Upper bound of the tile count (the exact count depends on the routing,
    // read on the device); every CTA gets ceil(tiles / SMs) tiles.
    const int64_t max_tiles = ((R + SW_BN - 1) / SW_BN + E) * static_cast<int64_t>(N / SW_BM);
    const int64_t tiles_ub = std::min<int64_t>(
        max_tiles, static_cast<int64_t>(E) * (N / SW_BM) * ((R + SW_BN - 1) / SW_BN));
    const int64_t sms = device_sm_count();
    const int64_t per_cta = (tiles_ub + sms - 1) / sms;
    const int grid = static_cast<int>(std::min<int64_t>(sms, (tiles_ub + per_cta - 1) / per_cta));
    auto kern = (mode == kEpiScaleToken) ? tc_swap_gemm_kernel<kEpiScaleToken, false>
                                         : tc_swap_gemm_kernel<kEpiScaleSlots, false>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(kSwapSmemBytes));
    if (err != cudaSuccess) return err;
    // Programmatic dependent launch: the set-up runs
    // while the kernel before (the dispatch) finishes.
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = kSwapSmemBytes;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, tw, tx, p);
  }
  if (K % 8 != 0 || N % 128 != 0 || E > kMaxExperts || R >= (int64_t(1) << 31))
    return cudaErrorInvalidValue;
  if (R == 0) return cudaSuccess;
  CUtensorMap ta, tb0, tb1, tb0h, tb1h;
  {
    // B maps: boxes of 128 rows (whole tiles) and 64 rows (half tiles)
    if (!make_map(&ta, a_sorted, K, R, 0, BM)) return cudaErrorInvalidValue;
    if (!make_map(&tb0, w0, K, N, E, 128)) return cudaErrorInvalidValue;
    if (!make_map(&tb0h, w0, K, N, E, 64)) return cudaErrorInvalidValue;
    if (gate) {
      if (!make_map(&tb1, w1, K, N, E, 128)) return cudaErrorInvalidValue;
      if (!make_map(&tb1h, w1, K, N, E, 64)) return cudaErrorInvalidValue;
    } else {
      tb1 = tb0;
      tb1h = tb0h;
    }
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
    p.n_tiles_n = (N + tile_n - 1) / tile_n;
    p.status = status;
    const int64_t max_tiles = ((R + PM - 1) / PM + E) * static_cast<int64_t>(p.n_tiles_n);
    switch (mode) {
      case kEpiGateH:
        return launch_pair_mode<kEpiGateH>(ta, tb0, tb1, tb0h, tb1h, p, max_tiles, stream);
      case kEpiGateSlots:
        return launch_pair_mode<kEpiGateSlots>(ta, tb0, tb1, tb0h, tb1h, p, max_tiles, stream);
      case kEpiScaleToken:
        return launch_pair_mode<kEpiScaleToken>(ta, tb0, tb1, tb0h, tb1h, p, max_tiles, stream);
      case kEpiScaleSlots:
        return launch_pair_mode<kEpiScaleSlots>(ta, tb0, tb1, tb0h, tb1h, p, max_tiles, stream);
      default:
        return cudaErrorInvalidValue;
    }
  }
}

cudaError_t launch_tc_dense_small(int mode, const void* x, int64_t T, int K, const void* w, int N,
                                  int E, int k, const int32_t* topk_idx, const float* topk_w,
                                  void* out, bool w_tiled, int* status, cudaStream_t stream) {
  if (T <= 0) return cudaSuccess;
  if (T > SW_BN || N % SW_BM != 0 || K % 8 != 0 || E > kMaxExperts) return cudaErrorInvalidValue;
  if (w_tiled && K % BK != 0) return cudaErrorInvalidValue;
  CUtensorMap tw, tx;
  if (w_tiled) {
    // [E][N/128][K/64][128][64]: a box of one whole 128 x 64 tile (16 KB)
    auto fn = encode_fn();
    if (!fn) return cudaErrorInvalidValue;
    const cuuint64_t kb = static_cast<cuuint64_t>(K / BK), nt = static_cast<cuuint64_t>(N / SW_BM);
    const cuuint64_t tile_bytes = static_cast<cuuint64_t>(SW_BM) * BK * 2;
    cuuint64_t dims[5] = {static_cast<cuuint64_t>(BK), static_cast<cuuint64_t>(SW_BM), kb, nt,
                          static_cast<cuuint64_t>(E)};
    cuuint64_t strides[4] = {static_cast<cuuint64_t>(BK) * 2, tile_bytes, tile_bytes * kb,
                             tile_bytes * kb * nt};
    cuuint32_t box[5] = {static_cast<cuuint32_t>(BK), static_cast<cuuint32_t>(SW_BM), 1, 1, 1};
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    if (fn(&tw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(w), dims, strides, box,
           estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  } else if (!make_map(&tw, w, K, N, E, SW_BM)) {
    return cudaErrorInvalidValue;
  }
  if (!make_map(&tx, x, K, T, 0, SW_BN)) return cudaErrorInvalidValue;
  Params p{};
  p.topk_idx = topk_idx;
  p.w_tiled = w_tiled ? 1 : 0;
  p.topk_w = topk_w;
  p.out = out;
  p.R = T;  // token rows (in token order)
  p.K = K;
  p.N = N;
  p.E = E;
  p.k = k;
  p.status = status;
  // every CTA gets the same number of tiles (E x N/128 tiles in all)
  const int64_t tiles = static_cast<int64_t>(E) * (N / SW_BM);
  const int64_t sms = device_sm_count();
  const int64_t per_cta = (tiles + sms - 1) / sms;
  const int grid = static_cast<int>(std::min<int64_t>(sms, (tiles + per_cta - 1) / per_cta));
  auto kern = (mode == kEpiScaleToken) ? tc_swap_gemm_kernel<kEpiScaleToken, true>
                                       : tc_swap_gemm_kernel<kEpiScaleSlots, true>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kSwapSmemBytes));
  if (err != cudaSuccess) return err;
  // a programmatic dependent of the router: the weight streaming and the
  // MMAs run while the router finishes; the epilogue waits for it
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSwapSmemBytes;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, tw, tx, p);
}

}  // namespace rom
