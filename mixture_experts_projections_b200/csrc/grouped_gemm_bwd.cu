// Backward grouped GEMMs of the RoM block on the tcgen05 tensor cores
// ("Routing Mamba ..." chapterpal summary page, Knowl 1, differentiated with
// the selection S_t held fixed). Three modes share one persistent,
// warp-specialised kernel run by pairs of CTAs on two SMs (2-CTA clusters,
// tcgen05.mma.cta_group::2, 256 x 256 pair tiles; per CTA a TMA producer,
// 4 epilogue warps and, in CTA 0, the single-thread MMA issuer; each CTA's
// 128 x 256 fp32 accumulators double-buffered in its own TMEM):
//
//  kBwdDgradOut  g'_s = (r dO)_s W_out,e^T for the rows s of expert e
//                (rows in expert-sorted order; A = r-scaled dO rows, K-major;
//                B = W_out,e stored [d_model][d_inner], read MN-major).
//                Epilogue: g' in float32 per slot, and the partial row dots
//                <h_s, g'_s> of the tile's columns (for dr = <Y(.)G, g>).
//  kBwdDgradIn   dX_s = [dH | dZ]_s [W_in,e ; W_g,e]^T (K = 2 d_inner; the
//                first half of K reads W_in, the second W_g, both MN-major).
//                Epilogue: float32 per slot.
//  kBwdWgrad     dW_e = A_e^T B_e with A_e, B_e the rows of expert e of two
//                expert-sorted arrays (both read MN-major, K = the expert's
//                row count). The last K block of an expert is partial: a
//                fix-up warp zeroes its rows past the expert's end in shared
//                memory (whole 128-byte lines, so the swizzle does not matter)
//                before the MMA reads them. Output rows m < m_split go to
//                out0[e], the others to out1[e] (dW_in and dW_g from one pass).
//
// Shared-memory operand layouts (bf16, 128-byte swizzle):
//  K-major  tile [rows][64]: 128-byte lines = rows, 8-line groups 1024 B
//           apart; a 16-element K step moves the start address by 32 B.
//  MN-major tile = chunks of 64 MN elements; chunk c holds 64 K rows of
//           128-byte lines (8-line groups 1024 B apart), chunks LBO = 8 KB
//           apart; a 16-row K step moves the start address by 2 KB.
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
constexpr int BN = 256;
constexpr int BK = 64;
constexpr int CHUNK_BYTES = 64 * BK * 2;  // one 64 x 64 MN-major box, 8 KB
constexpr uint32_t TMEM_COLS = 2 * BN;

struct BwdParams {
  const int32_t* offsets;
  const int32_t* sorted_slot;
  const __nv_bfloat16* h_sorted;  // kBwdDgradOut: Y (.) G rows, sorted order, [R][N]
  float* out0;
  float* out1;
  float* dr_part;  // kBwdDgradOut: [R][n_tiles_n]
  int64_t R;
  int K;        // dgrad: contraction length
  int N;        // output columns
  int M;        // wgrad: output rows (A's width)
  int E;
  int k;
  int n_tiles_n;
  int m_tiles;   // wgrad: M / 128
  int kb_split;  // dgrad-in: K blocks read from w0 before switching to w1
  int m_split;   // wgrad: rows of out0
  int* status;
};

__device__ __forceinline__ uint64_t sw128_mn_desc(uint32_t smem_addr, uint32_t lbo_bytes) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;  // MN chunk stride
  d |= static_cast<uint64_t>(1024u >> 4) << 32;                   // 8-row K group stride
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(2u) << 61;
  return d;
}

__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn, bool b_mn) {
  return idesc_bf16_f32(M, N) | (a_mn ? (1u << 15) : 0u) | (b_mn ? (1u << 16) : 0u);
}

template <int MODE>
struct Mode {
  static constexpr bool kWgrad = MODE == kBwdWgrad;
  static constexpr int kThreads = kWgrad ? 224 : 192;  // + the fix-up warp
};

// Epilogue of one accumulator tile for one warp: thread i reads TMEM lane
// t_row.lane + i, which holds output row `row` (wgrad: row m of dW_e; dgrad:
// row `row` of expert e's rows e_begin .. e_end - 1), columns
// n_blk * 256 .. + 255. Each 32-column chunk is stored row by row through the
// warp's staging tile `stg` (row-coalesced stores).
template <int MODE>
__device__ __forceinline__ void bwd_epilogue_rows(const BwdParams& p, uint32_t t_row, int e,
                                                  int e_begin, int e_end, int row, int n_blk,
                                                  float* stg) {
  const int n0 = n_blk * BN;
  if (MODE == kBwdWgrad) {
    const bool has_k = e_end > e_begin;
    const int m = row;
    float* dst_row = (m < p.m_split)
                         ? p.out0 + (static_cast<int64_t>(e) * p.m_split + m) * p.N
                         : p.out1 + (static_cast<int64_t>(e) * (p.M - p.m_split) + (m - p.m_split)) * p.N;
    const bool valid = m < p.M;
#pragma unroll 1
    for (int c = 0; c < 8; ++c) {
      if (n0 + c * 32 >= p.N) break;
      uint32_t a[32];
      tmem_ld32(t_row + c * 32, a);
      tmem_ld_wait();
      float f[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) f[j] = has_k ? __uint_as_float(a[j]) : 0.f;
      store_rows_f32(stg, f, valid ? dst_row + n0 + c * 32 : nullptr);
    }
  } else {
    const int row_local = row;
    const bool valid = row_local < e_end - e_begin;
    const int64_t prow = static_cast<int64_t>(e_begin) + row_local;
    const int64_t slot = valid ? p.sorted_slot[prow] : 0;
    float dot = 0.f;
#pragma unroll 1
    for (int c = 0; c < 8; ++c) {
      if (n0 + c * 32 >= p.N) break;
      uint32_t a[32];
      tmem_ld32(t_row + c * 32, a);
      tmem_ld_wait();
      if (MODE == kBwdDgradOut && valid) {
        const uint4* hp = reinterpret_cast<const uint4*>(p.h_sorted + prow * p.N + n0 + c * 32);
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const uint4 hv = __ldg(hp + v);
          const uint32_t w[4] = {hv.x, hv.y, hv.z, hv.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            dot = fmaf(__uint_as_float(w[i] << 16), __uint_as_float(a[8 * v + 2 * i]), dot);
            dot = fmaf(__uint_as_float(w[i] & 0xFFFF0000u), __uint_as_float(a[8 * v + 2 * i + 1]), dot);
          }
        }
      }
      float f[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) f[j] = __uint_as_float(a[j]);
      store_rows_f32(stg, f, valid ? p.out0 + slot * p.N + n0 + c * 32 : nullptr);
    }
    if (MODE == kBwdDgradOut && valid) p.dr_part[slot * p.n_tiles_n + n_blk] = dot;
  }
}

// ---------------------------------------------------------------------------
// SM-pair variant (cluster of two CTAs, tcgen05.mma.cta_group::2, M = 256):
// CTA v of the pair loads rows 128v .. 128v+127 of the pair tile's A rows
// (dgrad: 128 sorted rows; wgrad: 128 output rows m, as two 64-wide MN
// chunks) and B columns n0 + 128v .. + 127 (two 64-wide MN chunks), 32 KB
// per K step instead of 48 KB, and receives the 128 x 256 accumulator of its
// own rows in its own TMEM.
//  Full K blocks: both CTAs' TMA loads complete on CTA 0's full[s], which
//         CTA 0's producer arms with the bytes of both.
//  The ragged last K block of an expert (wgrad): each CTA's loads complete
//         on its own own[s]; its fix-up warp zeroes the K rows past the
//         expert's end in its own shared memory and then arrives on CTA 0's
//         ready[s] (two arrivals per phase), on which the MMA issuer waits
//         with cluster-scope acquire.
//  full[s], own[s] and ready[s] each advance only on the uses that arm them,
//  and every waiter tracks a per-stage parity of exactly those uses: a wait
//  can then never see a barrier one phase behind (which a parity wait would
//  take for complete).
// empty[s] and tfull[a] are armed in both CTAs by multicast commits; CTA 0's
// tempty[a] takes the arrivals of all 8 epilogue warps. Both CTAs end at a
// cluster barrier that every path reaches after bounded waits.
constexpr int PM = 256;
constexpr int P_STAGES = 6;
constexpr int P_A_BYTES = BM * BK * 2;   // 16 KB
constexpr int P_B_BYTES = 128 * BK * 2;  // 16 KB: two 64-wide MN chunks
constexpr int P_STAGE_BYTES = P_A_BYTES + P_B_BYTES;

struct PairCtl {
  uint64_t full[P_STAGES];
  uint64_t own[P_STAGES];
  uint64_t ready[P_STAGES];
  uint64_t empty[P_STAGES];
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
constexpr size_t kPairSmemBytes =
    P_STAGES * P_STAGE_BYTES + kPairCtlBytes + 4 * kStageFloats * sizeof(float) + 1024;

template <int MODE>
__global__ void __launch_bounds__(Mode<MODE>::kThreads, 1)
    tc_bwd_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                       const __grid_constant__ CUtensorMap tmB0,
                       const __grid_constant__ CUtensorMap tmB1, const BwdParams p) {
  constexpr bool kW = Mode<MODE>::kWgrad;
  extern __shared__ uint8_t smem_raw[];
  // Same 1024-byte aligned offset in both CTAs: the pair MMA reads the peer's
  // operands at the leader's offsets.
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  PairCtl& ctl = *reinterpret_cast<PairCtl*>(smem + P_STAGES * P_STAGE_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = p.E;
  const uint32_t rank = cluster_ctarank();
  const bool leader = (rank == 0);
  const int pair = static_cast<int>(blockIdx.x >> 1);
  const int npairs = static_cast<int>(gridDim.x >> 1);

  for (int i = threadIdx.x; i <= E; i += Mode<MODE>::kThreads) ctl.off[i] = p.offsets[i];
  __syncthreads();
  if (threadIdx.x == 0) {
    int run = 0;
    for (int e = 0; e < E; ++e) {
      const int mt = (ctl.off[e + 1] - ctl.off[e] + PM - 1) / PM;
      ctl.mt[e] = mt;
      ctl.tile_start[e] = run;
      run += kW ? p.m_tiles * p.n_tiles_n : mt * p.n_tiles_n;
    }
    ctl.tile_start[E] = run;
    for (int s = 0; s < P_STAGES; ++s) {
      mbar_init(&ctl.full[s], 1);
      mbar_init(&ctl.own[s], 1);
      mbar_init(&ctl.ready[s], 2);
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
    tma_prefetch_desc(&tmB0);
    tma_prefetch_desc(&tmB1);
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
  volatile int* abort_flag = &ctl.abort;

  auto tile_of = [&](int tile, int& e, int& m_blk, int& n_blk) {
    if (kW) {
      const int per_e = p.m_tiles * p.n_tiles_n;
      e = tile / per_e;
      const int rem = tile - e * per_e;
      n_blk = rem / p.m_tiles;
      m_blk = rem - n_blk * p.m_tiles;
    } else {
      e = 0;
      while (tile >= ctl.tile_start[e + 1]) ++e;
      const int local = tile - ctl.tile_start[e];
      n_blk = local / ctl.mt[e];
      m_blk = local - n_blk * ctl.mt[e];
    }
  };
  auto tile_kb = [&](int e) -> int {
    if (kW) return (ctl.off[e + 1] - ctl.off[e] + BK - 1) / BK;
    return (p.K + BK - 1) / BK;
  };
  const int half = static_cast<int>(rank) * 128;

  // wgrad: is K block kb of expert e the expert's ragged last block?
  auto ragged = [&](int e, int kb) -> bool {
    return kW && (ctl.off[e + 1] - ctl.off[e] - kb * BK) < BK;
  };

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer (both CTAs)
      const uint32_t full0 = mapa_shared(smem_u32(&ctl.full[0]), 0);
      int stage = 0;
      uint32_t phase = 0;
      // Per-stage parities: full[s] advances on full-block uses only, own[s]
      // on ragged-block uses only (so no waiter can be a phase behind).
      uint32_t full_par = 0, own_par = 0;
      uint32_t full_used = 0, own_used = 0;
      bool ok = true;
      for (int tile = pair; tile < total && ok; tile += npairs) {
        int e, m_blk, n_blk;
        tile_of(tile, e, m_blk, n_blk);
        const int KB = tile_kb(e);
        const int nb = n_blk * BN + half;  // this CTA's first B column
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&ctl.empty[stage], phase ^ 1u, abort_flag, p.status)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + stage * P_STAGE_BYTES;
          uint8_t* sb = sa + P_A_BYTES;
          const uint32_t fb = full0 + static_cast<uint32_t>(stage * sizeof(uint64_t));
          const bool own = ragged(e, kb);  // loads complete on this CTA's own[s]
          if (own) {
            mbar_arrive_expect_tx(&ctl.own[stage], P_STAGE_BYTES);
          } else if (leader) {
            mbar_arrive_expect_tx(&ctl.full[stage], 2 * P_STAGE_BYTES);
          }
          if (kW) {
            const int r0 = ctl.off[e] + kb * BK;
            const int m0 = m_blk * PM + half;
            if (own) {
              uint64_t* bar = &ctl.own[stage];
              tma_load_2d(sa, &tmA, bar, m0, r0);
              tma_load_2d(sa + CHUNK_BYTES, &tmA, bar, m0 + 64, r0);
              tma_load_2d(sb, &tmB0, bar, nb, r0);
              tma_load_2d(sb + CHUNK_BYTES, &tmB0, bar, nb + 64, r0);
            } else {
              tma_load_2d_pair(sa, &tmA, fb, m0, r0);
              tma_load_2d_pair(sa + CHUNK_BYTES, &tmA, fb, m0 + 64, r0);
              tma_load_2d_pair(sb, &tmB0, fb, nb, r0);
              tma_load_2d_pair(sb + CHUNK_BYTES, &tmB0, fb, nb + 64, r0);
            }
          } else {
            const int row0 = ctl.off[e] + m_blk * PM + half;
            tma_load_2d_pair(sa, &tmA, fb, kb * BK, row0);
            const bool second = (MODE == kBwdDgradIn) && kb >= p.kb_split;
            const CUtensorMap* mb = second ? &tmB1 : &tmB0;
            const int kk = second ? kb - p.kb_split : kb;
            tma_load_3d_pair(sb, mb, fb, nb, kk * BK, e);
            tma_load_3d_pair(sb + CHUNK_BYTES, mb, fb, nb + 64, kk * BK, e);
          }
          if (own) {
            own_used |= 1u << stage;
            own_par ^= 1u << stage;
          } else if (leader) {
            full_used |= 1u << stage;
            full_par ^= 1u << stage;
          }
          if (++stage == P_STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Loads that complete on this CTA's barriers have all landed (the last
      // armed phase of a barrier has the parity before its last toggle).
      int never = 0;
      for (int s = 0; s < P_STAGES; ++s) {
        if ((full_used >> s) & 1u)
          mbar_wait(&ctl.full[s], ((full_par >> s) & 1u) ^ 1u, &never, p.status);
        if ((own_used >> s) & 1u)
          mbar_wait(&ctl.own[s], ((own_par >> s) & 1u) ^ 1u, &never, p.status);
      }
      if (!leader && !ok) {
        // Aborted: this CTA's other loads complete on the leader's barriers,
        // which it cannot wait on; give copies in flight a fixed time to land.
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 200000ull) {
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ------------------------------------------------ MMA issuer (CTA 0)
      const uint32_t idesc = idesc_bf16(PM, BN, kW, true);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t ready_par = 0;  // per-stage parity of ready[s] (ragged uses only)
      uint32_t full_par = 0;   // per-stage parity of full[s] (full-block uses only)
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int tile = pair; tile < total && ok; tile += npairs) {
        int e, m_blk, n_blk;
        tile_of(tile, e, m_blk, n_blk);
        const int KB = tile_kb(e);
        if (!mbar_wait(&ctl.tempty[acc], acc_phase ^ 1u, abort_flag, p.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = 0; kb < KB; ++kb) {
          bool got;
          if (ragged(e, kb)) {
            // both CTAs' fix-up warps have zeroed the rows past the expert
            got = mbar_wait_cluster(&ctl.ready[stage], (ready_par >> stage) & 1u, abort_flag,
                                    p.status);
            ready_par ^= 1u << stage;
          } else {
            got = mbar_wait(&ctl.full[stage], (full_par >> stage) & 1u, abort_flag, p.status);
            full_par ^= 1u << stage;
          }
          if (!got) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + stage * P_STAGE_BYTES);
          const uint32_t b_addr = a_addr + P_A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t ad = kW ? sw128_mn_desc(a_addr + kk * 2048, CHUNK_BYTES)
                                   : sw128_kmajor_desc(a_addr + kk * 32);
            const uint64_t bd = sw128_mn_desc(b_addr + kk * 2048, CHUNK_BYTES);
            mma_bf16_ss_pair(d_tmem, ad, bd, idesc, (kb | kk) != 0);
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
      mma_commit_pair(&ctl.drain);
      int never = 0;
      mbar_wait(&ctl.drain, 0, &never, p.status);
    }
  } else if (warp == 6) {
    // -------------------------------------------------- fix-up warp (wgrad, both CTAs)
    // Only the ragged last K block of an expert passes through here: after
    // this CTA's own loads land, zero its rows past the expert's end, then
    // report to CTA 0's ready[s].
    const uint32_t ready0 = mapa_shared(smem_u32(&ctl.ready[0]), 0);
    int stage = 0;
    uint32_t own_par = 0;  // per-stage parity of own[s]
    bool ok = true;
    for (int tile = pair; tile < total && ok; tile += npairs) {
      int e, m_blk, n_blk;
      tile_of(tile, e, m_blk, n_blk);
      const int n_e = ctl.off[e + 1] - ctl.off[e];
      const int KB = tile_kb(e);
      for (int kb = 0; kb < KB; ++kb) {
        if (ragged(e, kb)) {
          const uint32_t par = (own_par >> stage) & 1u;
          own_par ^= 1u << stage;
          if (!mbar_wait(&ctl.own[stage], par, abort_flag, p.status)) {
            ok = false;
            break;
          }
          // zero lines valid..63 of the 4 chunks (2 of A, 2 of B)
          const int valid = n_e - kb * BK;
          uint8_t* base = smem + stage * P_STAGE_BYTES;
          const int per_chunk = (BK - valid) * 8;  // 16-byte pieces
          for (int i = lane; i < 4 * per_chunk; i += 32) {
            const int c = i / per_chunk, q = i - c * per_chunk;
            uint4* dst = reinterpret_cast<uint4*>(base + c * CHUNK_BYTES + valid * 128) + q;
            *dst = make_uint4(0u, 0u, 0u, 0u);
          }
          fence_async_shared();
          __syncwarp();
          if (lane == 0) {
            if (leader)
              mbar_arrive(&ctl.ready[stage]);
            else
              mbar_arrive_remote(ready0 + static_cast<uint32_t>(stage * sizeof(uint64_t)));
          }
        }
        if (++stage == P_STAGES) stage = 0;
      }
    }
  } else {
    // -------------------------------------------------- epilogue (warps 2..5, both CTAs)
    const int q = warp & 3;
    const uint32_t tempty0 = mapa_shared(smem_u32(&ctl.tempty[0]), 0);
    float* stg = reinterpret_cast<float*>(smem + P_STAGES * P_STAGE_BYTES + kPairCtlBytes) +
                 (warp - 2) * kStageFloats;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = pair; tile < total; tile += npairs) {
      int e, m_blk, n_blk;
      tile_of(tile, e, m_blk, n_blk);
      if (!mbar_wait(&ctl.tfull[acc], acc_phase, abort_flag, p.status)) break;
      tc_fence_after();
      const uint32_t t_row =
          tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * BN);
      const int row = m_blk * PM + half + q * 32 + lane;
      bwd_epilogue_rows<MODE>(p, t_row, e, ctl.off[e], ctl.off[e + 1], row, n_blk, stg);
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

// bf16 tensor map over [outer][rows][inner] (outer == 0: 2-D [rows][inner]),
// box 64 (inner) x box_rows, 128-byte swizzle.
bool map_bf16(CUtensorMap* m, const void* base, int64_t inner, int64_t rows, int outer,
              int box_inner, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(outer > 0 ? outer : 1)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(inner * 2),
                           static_cast<cuuint64_t>(inner * 2 * rows)};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(box_inner), static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, outer > 0 ? 3 : 2, const_cast<void*>(base),
                  dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int MODE>
cudaError_t launch_pair_mode(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                             const BwdParams& p, int64_t max_tiles, cudaStream_t stream) {
  auto kern = tc_bwd_pair_kernel<MODE>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kPairSmemBytes));
  if (err != cudaSuccess) return err;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(Mode<MODE>::kThreads, 1, 1);
  cfg.dynamicSmemBytes = kPairSmemBytes;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // Co-resident pairs on this device (one CTA per SM), cached per device and mode.
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
  return cudaLaunchKernelEx(&cfg, kern, a, b0, b1, p);
}

BwdParams base_params(const int32_t* offsets, int64_t R, int E, int k, int* status) {
  BwdParams p{};
  p.offsets = offsets;
  p.R = R;
  p.E = E;
  p.k = k;
  p.status = status;
  return p;
}

}  // namespace

cudaError_t launch_bwd_dgrad_out(const void* rdo_sorted, int64_t R, int Dm, const void* w_out,
                                 int De, int E, int k, const int32_t* offsets,
                                 const int32_t* sorted_slot, const void* h_sorted, float* g_slots,
                                 float* dr_part, int* status, cudaStream_t stream) {
  if (Dm % 64 || De % 256 || E > kMaxExperts) return cudaErrorInvalidValue;
  if (R == 0) return cudaSuccess;
  CUtensorMap ta, tb;
  if (!map_bf16(&ta, rdo_sorted, Dm, R, 0, BK, BM)) return cudaErrorInvalidValue;
  // W_out stored [E][Dm][De]: inner De (= N), rows Dm (= K).
  if (!map_bf16(&tb, w_out, De, Dm, E, 64, BK)) return cudaErrorInvalidValue;
  BwdParams p = base_params(offsets, R, E, k, status);
  p.sorted_slot = sorted_slot;
  p.h_sorted = static_cast<const __nv_bfloat16*>(h_sorted);
  p.out0 = g_slots;
  p.dr_part = dr_part;
  p.K = Dm;
  p.N = De;
  p.n_tiles_n = De / BN;
  return launch_pair_mode<kBwdDgradOut>(
      ta, tb, tb, p, ((R + PM - 1) / PM + E) * static_cast<int64_t>(p.n_tiles_n), stream);
}

cudaError_t launch_bwd_dgrad_in(const void* dhz_sorted, int64_t R, int De, const void* w_in,
                                const void* w_g, int Dm, int E, int k, const int32_t* offsets,
                                const int32_t* sorted_slot, float* dx_slots, int* status,
                                cudaStream_t stream) {
  if (De % 64 || Dm % 256 || E > kMaxExperts) return cudaErrorInvalidValue;
  if (R == 0) return cudaSuccess;
  CUtensorMap ta, tb0, tb1;
  if (!map_bf16(&ta, dhz_sorted, 2 * static_cast<int64_t>(De), R, 0, BK, BM))
    return cudaErrorInvalidValue;
  // W_in, W_g stored [E][De][Dm]: inner Dm (= N), rows De (= K).
  if (!map_bf16(&tb0, w_in, Dm, De, E, 64, BK)) return cudaErrorInvalidValue;
  if (!map_bf16(&tb1, w_g, Dm, De, E, 64, BK)) return cudaErrorInvalidValue;
  BwdParams p = base_params(offsets, R, E, k, status);
  p.sorted_slot = sorted_slot;
  p.out0 = dx_slots;
  p.K = 2 * De;
  p.N = Dm;
  p.kb_split = De / BK;
  p.n_tiles_n = Dm / BN;
  return launch_pair_mode<kBwdDgradIn>(
      ta, tb0, tb1, p, ((R + PM - 1) / PM + E) * static_cast<int64_t>(p.n_tiles_n), stream);
}

cudaError_t launch_bwd_wgrad(const void* a_sorted, int M, const void* b_sorted, int N, int64_t R,
                             int E, const int32_t* offsets, int m_split, float* out0, float* out1,
                             int* status, cudaStream_t stream) {
  if (M % BM || N % BN || m_split % BM || m_split > M || E > kMaxExperts)
    return cudaErrorInvalidValue;
  CUtensorMap ta, tb;
  if (!map_bf16(&ta, a_sorted, M, std::max<int64_t>(R, 1), 0, 64, BK)) return cudaErrorInvalidValue;
  if (!map_bf16(&tb, b_sorted, N, std::max<int64_t>(R, 1), 0, 64, BK)) return cudaErrorInvalidValue;
  BwdParams p = base_params(offsets, R, E, 1, status);
  p.out0 = out0;
  p.out1 = out1 ? out1 : out0;
  p.M = M;
  p.N = N;
  p.m_split = m_split;
  p.n_tiles_n = N / BN;
  p.m_tiles = (M + PM - 1) / PM;
  return launch_pair_mode<kBwdWgrad>(ta, tb, tb, p,
                                     static_cast<int64_t>(E) * p.m_tiles * p.n_tiles_n, stream);
}

}  // namespace rom
