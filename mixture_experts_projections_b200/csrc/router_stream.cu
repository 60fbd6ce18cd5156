// Streaming router for bf16 activations ("Routing Mamba ..." chapterpal
// summary page, Knowl 1: p_t = Softmax(x_t W_r), S_t = the K largest
// probabilities, r_{t,i} = p_{t,i} 1[i in S_t]).
//
// One CTA owns a 128-token tile (= one histogram chunk of the dispatch) at a
// time. A producer warp streams the tile through a ring of stages, one
// 64-feature block per stage: the X block by TMA (128 x 64 bf16, 128-byte
// swizzle; its lines kept in L2 ahead of other data, since the dispatch reads
// the rows again right after) and the matching 64 rows of W_r ([d_model][E]
// float32, contiguous) by a bulk copy. W_r is not kept resident: each CTA re-reads it (from L2)
// once per tile, which leaves the shared memory to a deep ring.
//
// 8 compute warps: warp h owns features 8h .. 8h+7 of every block and all 128
// tokens, 4 per lane (tokens lane + 32 j). Per block a lane reads its tokens'
// 8 features (one 16-byte piece each, conflict-free under the swizzle) and
// the 8 x E weights as broadcast float4 reads, each of which feeds 4 tokens.
// Per pair of blocks (per block when E = 16) and expert it forms a partial
// over its 16 (8) features (sequential float32 FMA, two experts per packed
// FMA) and adds it to its running sum. At the end of the tile the 8 warps'
// sums and |x|^2 meet in shared memory and warp h decides tokens
// 16h .. 16h+15, adding the parts in order h = 0 .. 7. Each logit therefore
// goes through at most 16 + d_model/128 + 7 + 1 roundings (E = 16:
// 8 + d_model/64 + 7 + 1);
// with |x| and |w_e| this bounds its error by gamma_n |x| |w_e|
// (Cauchy-Schwarz). |w_e| is formed from the streamed weight blocks during a
// CTA's first tile. A token whose selected logits' lower bounds do not all
// clear the upper bound of every expert ranked after them is re-decided on
// float64 logits, which all 8 compute warps form together (each over an
// eighth of the features). Equal logits go to the lower expert index.
// Every wait is bounded; after the set-up the roles meet only on mbarriers.
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

constexpr int BM = 128;                 // tokens per tile
constexpr int BK = 64;                  // features per block
constexpr int X_BYTES = BM * BK * 2;    // 16 KB
constexpr int kCompute = 8;             // compute warps
constexpr int kThreads = 32 * (1 + kCompute);
constexpr int kFeat = BK / kCompute;    // features per warp per block
constexpr int TPL = BM / 32;            // tokens per lane
constexpr int kDecide = BM / kCompute;  // tokens decided per warp
constexpr int kMaxStages = 8;
constexpr int kUB = 4;                  // uncertain tokens per float64 batch

template <int EB>
struct Geo {
  static constexpr int kWBytes = BK * EB * 4;
  static constexpr int kStage = X_BYTES + kWBytes;  // a multiple of 1024
  static constexpr int kEG = EB < 8 ? EB : 8;        // experts per register group
  // blocks per partial sum: two (16 features) when one register group holds
  // every expert, else one (the partials of both groups would not fit)
  static constexpr int kPB = EB / kEG == 1 ? 2 : 1;
  static constexpr int kPCols = EB + 4;              // part row: sums, |x|^2, pad
  static constexpr int kNormPerLane = kFeat * EB / 32;
};

template <int EB>
struct SCtl {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  uint64_t part_ready;
  uint64_t part_free;
  int abort;
  int done;
  int hist[EB];
  float wsq[kCompute][EB];
  // float64 re-decision of uncertain tokens: their tile rows, and the 8
  // warps' partial logits of a batch of kUB of them
  int nunc;
  int unc_row[BM];
  uint64_t unc_ready;
  uint64_t p64_ready;
  uint64_t p64_free;
  double p64[kUB][kCompute][EB];
};

__device__ __forceinline__ uint32_t sw128_off(int n, int k) {
  const uint32_t o = static_cast<uint32_t>(n) * 128u + static_cast<uint32_t>(k) * 2u;
  return o ^ (((o >> 7) & 7u) << 4);
}

template <int EB>
__global__ void __launch_bounds__(kThreads, 1)
    router_stream_kernel(const __grid_constant__ CUtensorMap tmX,
                         const __nv_bfloat16* __restrict__ x, int64_t T, int Dm,
                         const float* __restrict__ w_r, const float* __restrict__ bias, int E,
                         int k, int renorm, int32_t* __restrict__ topk_idx,
                         float* __restrict__ topk_w, int32_t* __restrict__ counts,
                         int32_t* __restrict__ chunk_hist, int64_t ntiles, int stages,
                         float gamma, int* status) {
  using G = Geo<EB>;
  using Ctl = SCtl<EB>;
  constexpr int EG = G::kEG;
  constexpr int PC = G::kPCols;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base, kept as a shared-memory pointer (an offset into
  // the shared array, not an integer round-trip) so accesses stay LDS/STS.
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  Ctl& ctl = *reinterpret_cast<Ctl*>(smem + stages * G::kStage);
  float* part = reinterpret_cast<float*>(smem + stages * G::kStage +
                                         ((sizeof(Ctl) + 15) / 16) * 16);  // [8][BM][PC]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int KB = Dm / BK;
  // The dispatch is launched as a programmatic dependent and waits for this
  // grid's completion before it reads the outputs.
  pdl_launch_dependents();

  if (tid == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&ctl.full[s], 1);
      mbar_init(&ctl.empty[s], kCompute);
    }
    mbar_init(&ctl.part_ready, kCompute);
    mbar_init(&ctl.part_free, kCompute);
    mbar_init(&ctl.unc_ready, kCompute);
    mbar_init(&ctl.p64_ready, kCompute);
    mbar_init(&ctl.p64_free, kCompute);
    ctl.abort = 0;
    ctl.done = 0;
    ctl.nunc = 0;
    for (int e = 0; e < EB; ++e) ctl.hist[e] = 0;
    fence_barrier_init();
  }
  __syncthreads();
  volatile int* abort_flag = &ctl.abort;

  if (warp == 0) {
    // -------------------------------------------------- producer
    if (lane == 0) {
      tma_prefetch_desc(&tmX);
      // X is read again right after this kernel by the dispatch's row copy:
      // its lines are kept in L2 ahead of other data
      const uint64_t pol_x = l2_policy_evict_last();
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
          uint8_t* st = smem + stage * G::kStage;
          mbar_arrive_expect_tx(&ctl.full[stage], G::kStage);
          tma_load_2d_hint(st, &tmX, &ctl.full[stage], kb * BK, static_cast<int>(tile * BM),
                           pol_x);
          bulk_load(st + X_BYTES, w_r + static_cast<int64_t>(kb) * BK * EB, G::kWBytes,
                    &ctl.full[stage]);
          issued |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
          if (++stage == stages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Every copy this CTA started has landed before it exits.
      int never = 0;
      for (int s = 0; s < stages; ++s)
        if ((issued >> s) & 1u) mbar_wait(&ctl.full[s], (last_par >> s) & 1u, &never, status);
    }
    return;
  }

  // ---------------------------------------------------- compute warps
  const int h = warp - 1;  // feature slice of every block; decided tokens 16h ..
  constexpr int PB = G::kPB;
  float wn[EB];            // |w_e|, formed in the first tile
  float nq = 0.f;          // this lane's share of |w_{lane % EB}|^2 over the warp's features
  int stage = 0;
  uint32_t phase = 0;
  uint32_t p64_phase = 0, p64_free_phase = 0;
  int it = 0;
  for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++it) {
    float acc[TPL][EB];
    float2 p[EB / EG][TPL][EG / 2];  // the current partial sums (PB blocks each)
    float sq[TPL];
#pragma unroll
    for (int t = 0; t < TPL; ++t) {
      sq[t] = 0.f;
#pragma unroll
      for (int e = 0; e < EB; ++e) acc[t][e] = 0.f;
    }
    bool ok = true;
    for (int kb = 0; kb < KB; ++kb) {
      if (!__all_sync(0xffffffffu, mbar_wait(&ctl.full[stage], phase, abort_flag, status))) {
        ok = false;
        break;
      }
      const uint8_t* st = smem + stage * G::kStage;
      const float* sw = reinterpret_cast<const float*>(st + X_BYTES) + kFeat * h * EB;
      // the lane's tokens' 8 features of the block, as bf16 pairs (unpacked
      // where the FMAs use them, which keeps fewer registers live)
      uint4 xc[TPL];
#pragma unroll
      for (int t = 0; t < TPL; ++t)
        xc[t] = *reinterpret_cast<const uint4*>(st + sw128_off(lane + 32 * t, kFeat * h));
      if (it == 0) {
        // the warp's 8 x EB weights of the block, lane l taking l, l + 32, ...
        // (all of expert l % EB)
#pragma unroll
        for (int j = 0; j < G::kNormPerLane; ++j) {
          const float w = sw[lane + 32 * j];
          nq = fmaf(w, w, nq);
        }
      }
      const bool p_first = kb % PB == 0;
      const bool p_last = kb % PB == PB - 1 || kb == KB - 1;
#pragma unroll
      for (int g = 0; g < EB / EG; ++g) {
        if (p_first) {
#pragma unroll
          for (int t = 0; t < TPL; ++t)
#pragma unroll
            for (int e2 = 0; e2 < EG / 2; ++e2) p[g][t][e2] = make_float2(0.f, 0.f);
        }
#pragma unroll
        for (int i = 0; i < kFeat; ++i) {
          // feature i of the lane's tokens, unpacked from the bf16 pieces
          // where it is used (and |x|^2 formed on the first group's pass)
          float xi[TPL];
#pragma unroll
          for (int t = 0; t < TPL; ++t) {
            const uint32_t wd = (i >> 1) == 0   ? xc[t].x
                                : (i >> 1) == 1 ? xc[t].y
                                : (i >> 1) == 2 ? xc[t].z
                                                : xc[t].w;
            xi[t] = __uint_as_float((i & 1) ? (wd & 0xFFFF0000u) : (wd << 16));
            if (g == 0) sq[t] = fmaf(xi[t], xi[t], sq[t]);
          }
          const float4* wv = reinterpret_cast<const float4*>(sw + i * EB + g * EG);
#pragma unroll
          for (int q4 = 0; q4 < EG / 4; ++q4) {
            const float4 w4 = wv[q4];
            const float2 wa = make_float2(w4.x, w4.y), wb = make_float2(w4.z, w4.w);
#pragma unroll
            for (int t = 0; t < TPL; ++t) {
              const float2 xx = make_float2(xi[t], xi[t]);
              p[g][t][2 * q4] = __ffma2_rn(xx, wa, p[g][t][2 * q4]);
              p[g][t][2 * q4 + 1] = __ffma2_rn(xx, wb, p[g][t][2 * q4 + 1]);
            }
          }
        }
        if (p_last) {
#pragma unroll
          for (int t = 0; t < TPL; ++t)
#pragma unroll
            for (int e2 = 0; e2 < EG / 2; ++e2) {
              const int e = g * EG + 2 * e2;
              const float2 a2 = __fadd2_rn(make_float2(acc[t][e], acc[t][e + 1]), p[g][t][e2]);
              acc[t][e] = a2.x;
              acc[t][e + 1] = a2.y;
            }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl.empty[stage]);  // done with the stage
      if (++stage == stages) {
        stage = 0;
        phase ^= 1u;
      }
    }
    if (!ok) break;

    // ------------------------------------------------ parts to shared memory
    if (it > 0 &&
        !__all_sync(0xffffffffu,
                    mbar_wait(&ctl.part_free, static_cast<uint32_t>(it - 1) & 1u, abort_flag,
                              status)))
      break;
#pragma unroll
    for (int t = 0; t < TPL; ++t) {
      float* row = part + (h * BM + lane + 32 * t) * PC;
#pragma unroll
      for (int e4 = 0; e4 < EB / 4; ++e4)
        *reinterpret_cast<float4*>(row + 4 * e4) =
            make_float4(acc[t][4 * e4], acc[t][4 * e4 + 1], acc[t][4 * e4 + 2], acc[t][4 * e4 + 3]);
      *reinterpret_cast<float4*>(row + EB) = make_float4(sq[t], 0.f, 0.f, 0.f);
    }
    if (it == 0) {
#pragma unroll
      for (int o = 16; o >= EB; o >>= 1) nq += __shfl_xor_sync(0xffffffffu, nq, o);
      if (lane < EB) ctl.wsq[h][lane] = nq;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&ctl.part_ready);
    if (!__all_sync(0xffffffffu, mbar_wait(&ctl.part_ready, static_cast<uint32_t>(it) & 1u,
                                           abort_flag, status)))
      break;
    if (it == 0) {
#pragma unroll
      for (int e = 0; e < EB; ++e) {
        float s = ctl.wsq[0][e];
#pragma unroll
        for (int hh = 1; hh < kCompute; ++hh) s += ctl.wsq[hh][e];
        wn[e] = sqrtf(s);
      }
    }

    // ------------------------------------------------ decisions
    const int r = kDecide * h + (lane & (kDecide - 1));
    const int64_t tok = tile * BM + r;
    const bool valid = lane < kDecide && tok < T;
    float l[EB], err[EB];
    float sqt;
    {
      const float* row0 = part + r * PC;
#pragma unroll
      for (int e4 = 0; e4 < EB / 4; ++e4) {
        const float4 v = *reinterpret_cast<const float4*>(row0 + 4 * e4);
        l[4 * e4] = v.x;
        l[4 * e4 + 1] = v.y;
        l[4 * e4 + 2] = v.z;
        l[4 * e4 + 3] = v.w;
      }
      sqt = row0[EB];
#pragma unroll
      for (int hh = 1; hh < kCompute; ++hh) {
        const float* rowh = part + (hh * BM + r) * PC;
#pragma unroll
        for (int e4 = 0; e4 < EB / 4; ++e4) {
          const float4 v = *reinterpret_cast<const float4*>(rowh + 4 * e4);
          l[4 * e4] += v.x;
          l[4 * e4 + 1] += v.y;
          l[4 * e4 + 2] += v.z;
          l[4 * e4 + 3] += v.w;
        }
        sqt += rowh[EB];
      }
    }
    const float xn = sqrtf(sqt);
#pragma unroll
    for (int e = 0; e < EB; ++e) {
      if (e < E) {
        l[e] = l[e] + (bias ? __ldg(bias + e) : 0.f);
        err[e] = gamma * xn * wn[e] + 1.2e-7f * fabsf(l[e]);
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
      float v = 0.f;
#pragma unroll
      for (int e = 0; e < EB; ++e) v = (e == i) ? a[e] : v;
      return v;
    };
    // Certain when, for every slot j < k, the lower bound of the j-th selected
    // logit clears the upper bound of every expert ranked after it (the bounds
    // differ per expert through |w_e|).
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
    // Tokens whose float32 decision is not certain get float64 logits from
    // all 8 compute warps together, kUB tokens at a time: warp h sums its
    // feature slice h*Dm/8 .. (h+1)*Dm/8 - 1 (lane l: the 8-feature pieces
    // l, l + 32, ... of the slice), the slices meet in shared memory and the
    // deciding lane adds them in the order h = 0 .. 7 and decides again.
    const bool unsure = valid && !certain;
    const unsigned mine = __ballot_sync(0xffffffffu, unsure);
    int my_idx = 0;
    {
      int base = 0;
      if (lane == 0 && mine) base = atomicAdd(&ctl.nunc, __popc(mine));
      base = __shfl_sync(0xffffffffu, base, 0);
      my_idx = base + __popc(mine & ((1u << lane) - 1u));
      if (unsure) ctl.unc_row[my_idx] = r;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&ctl.unc_ready);
    if (!__all_sync(0xffffffffu, mbar_wait(&ctl.unc_ready, static_cast<uint32_t>(it) & 1u,
                                           abort_flag, status)))
      break;
    const int nunc = *reinterpret_cast<volatile int*>(&ctl.nunc);
    bool batch_ok = true;
    for (int b0 = 0; b0 < nunc && batch_ok; b0 += kUB) {
      const int nb = min(kUB, nunc - b0);
      for (int u = 0; u < nb; ++u) {
        const int64_t tr = tile * BM + ctl.unc_row[b0 + u];
        const uint4* xr = reinterpret_cast<const uint4*>(x + tr * Dm + h * (Dm / kCompute));
        double a[EB];
#pragma unroll
        for (int e = 0; e < EB; ++e) a[e] = 0.0;
        for (int pc = lane; pc < Dm / (kCompute * 8); pc += 32) {
          const uint4 v = __ldg(xr + pc);
          const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
          const float* wrow = w_r + (static_cast<int64_t>(h) * (Dm / kCompute) + 8 * pc) * EB;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const uint32_t bits = (j & 1) ? (w4[j >> 1] & 0xFFFF0000u) : (w4[j >> 1] << 16);
            const double xd = static_cast<double>(__uint_as_float(bits));
            const float4* wq = reinterpret_cast<const float4*>(wrow + j * EB);
#pragma unroll
            for (int e4 = 0; e4 < EB / 4; ++e4) {
              const float4 w = __ldg(wq + e4);
              a[4 * e4] = fma(xd, static_cast<double>(w.x), a[4 * e4]);
              a[4 * e4 + 1] = fma(xd, static_cast<double>(w.y), a[4 * e4 + 1]);
              a[4 * e4 + 2] = fma(xd, static_cast<double>(w.z), a[4 * e4 + 2]);
              a[4 * e4 + 3] = fma(xd, static_cast<double>(w.w), a[4 * e4 + 3]);
            }
          }
        }
#pragma unroll
        for (int e = 0; e < EB; ++e)
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) a[e] += __shfl_xor_sync(0xffffffffu, a[e], o);
        if (lane == 0)
#pragma unroll
          for (int e = 0; e < EB; ++e) ctl.p64[u][h][e] = a[e];
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl.p64_ready);
      if (!__all_sync(0xffffffffu,
                      mbar_wait(&ctl.p64_ready, p64_phase, abort_flag, status))) {
        batch_ok = false;
        break;
      }
      p64_phase ^= 1u;
      if (unsure && my_idx >= b0 && my_idx < b0 + nb) {
        const int u = my_idx - b0;
        double l64[EB];
#pragma unroll
        for (int e = 0; e < EB; ++e) {
          double v = ctl.p64[u][0][e];
#pragma unroll
          for (int hh = 1; hh < kCompute; ++hh) v += ctl.p64[u][hh][e];
          l64[e] = v + (bias && e < E ? static_cast<double>(bias[e]) : 0.0);
        }
        uint64_t u2 = 0;
#pragma unroll
        for (int j = 0; j <= kMaxTopK; ++j) {
          sel[j] = -1;
          if (j <= k) {
            int bi = -1;
            double bv = 0.0;
#pragma unroll
            for (int e = 0; e < EB; ++e)
              if (e < E && !((u2 >> e) & 1ull) && (bi < 0 || l64[e] > bv)) {
                bi = e;
                bv = l64[e];
              }
            sel[j] = bi;
            if (bi >= 0) u2 |= 1ull << bi;
          }
        }
#pragma unroll
        for (int e = 0; e < EB; ++e) l[e] = (e < E) ? static_cast<float>(l64[e]) : -INFINITY;
      }
      if (b0 + kUB < nunc) {
        // the partials are read before the next batch overwrites them
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl.p64_free);
        if (!__all_sync(0xffffffffu,
                        mbar_wait(&ctl.p64_free, p64_free_phase, abort_flag, status))) {
          batch_ok = false;
          break;
        }
        p64_free_phase ^= 1u;
      }
    }
    if (!batch_ok) break;
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
          atomicAdd(&ctl.hist[sel[j]], 1);
        }
    }
    // The last of the deciding warps publishes the tile's histogram (before
    // it frees the parts, so the next tile's counts start from zero).
    __threadfence_block();
    __syncwarp();
    int last = 0;
    if (lane == 0) last = (atomicAdd(&ctl.done, 1) == kCompute - 1);
    last = __shfl_sync(0xffffffffu, last, 0);
    if (last) {
      __threadfence_block();
      for (int e = lane; e < E; e += 32) {
        const int v = atomicExch(&ctl.hist[e], 0);
        if (chunk_hist) chunk_hist[tile * E + e] = v;
        if (counts && v) atomicAdd(counts + e, v);
      }
      if (lane == 0) {
        ctl.done = 0;
        ctl.nunc = 0;  // every warp read it after unc_ready, before its decisions
      }
      __threadfence_block();
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&ctl.part_free);
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

template <int EB>
cudaError_t launch_eb(const void* x, int64_t T, int Dm, const float* w_r, const float* bias, int E,
                      int k, int renorm, int32_t* topk_idx, float* topk_w, int32_t* counts,
                      int32_t* chunk_hist, int* status, cudaStream_t stream) {
  using G = Geo<EB>;
  const int64_t ntiles = num_chunks(T);
  const size_t ctl = (sizeof(SCtl<EB>) + 15) / 16 * 16;
  const size_t part = static_cast<size_t>(kCompute) * BM * G::kPCols * sizeof(float);
  const size_t budget = 224 * 1024;
  int stages = kMaxStages;
  while (stages > 2 && stages * G::kStage + ctl + part + 1024 > budget) --stages;
  if (stages * G::kStage + ctl + part + 1024 > budget) return cudaErrorNotSupported;
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
  // Longest rounding chain of a logit: the FMAs of one partial sum (8
  // features per block, G::kPB blocks), one add per partial, 7 adds of the
  // warps' parts, the bias (+1 spare); 1 % slack covers the norms.
  const int kb_total = Dm / BK;
  const double n = static_cast<double>(kFeat * std::min(G::kPB, kb_total)) +
                   static_cast<double>((kb_total + G::kPB - 1) / G::kPB) +
                   static_cast<double>(kCompute - 1) + 2.0;
  const double u = 1.0 / 16777216.0;
  const float gamma = static_cast<float>(1.01 * n * u / (1.0 - n * u));
  const size_t smem = stages * G::kStage + ctl + part + 1024;
  auto kern = router_stream_kernel<EB>;
  cudaError_t err =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  const int grid = static_cast<int>(std::min<int64_t>(ntiles, device_sm_count()));
  kern<<<grid, kThreads, smem, stream>>>(tm, static_cast<const __nv_bfloat16*>(x), T, Dm, w_r, bias,
                                         E, k, renorm, topk_idx, topk_w, counts, chunk_hist,
                                         ntiles, stages, gamma, status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_router_stream(const void* x, int64_t T, int Dm, const float* w_r,
                                 const float* bias, int E, int k, int renorm, int32_t* topk_idx,
                                 float* topk_w, int32_t* counts, int32_t* chunk_hist, int* status,
                                 cudaStream_t stream) {
  // W_r is streamed as stored ([d_model][E], 16-byte rows) in whole 64-row
  // blocks: E in {4, 8, 16} and d_model a multiple of 64.
  if ((reinterpret_cast<uintptr_t>(w_r) & 15u) || Dm % BK != 0 || Dm <= 0)
    return cudaErrorNotSupported;
  if (E == 4)
    return launch_eb<4>(x, T, Dm, w_r, bias, E, k, renorm, topk_idx, topk_w, counts, chunk_hist,
                        status, stream);
  if (E == 8)
    return launch_eb<8>(x, T, Dm, w_r, bias, E, k, renorm, topk_idx, topk_w, counts, chunk_hist,
                        status, stream);
  if (E == 16)
    return launch_eb<16>(x, T, Dm, w_r, bias, E, k, renorm, topk_idx, topk_w, counts, chunk_hist,
                         status, stream);
  return cudaErrorNotSupported;  // other expert counts use the register-tiled kernel
}

}  // namespace rom
