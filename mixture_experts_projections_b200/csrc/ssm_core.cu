// The dense core between the projections of the RoM block ("Routing Mamba
// ..." chapterpal summary page, Knowl 1: the short convolution and the
// selective state-space computation applied to H_t produce Y_t; Knowl 9: the
// 1D convolution, the x projection and the dt projection are shared by all
// experts), in the original Mamba form (Gu and Dao 2023, Section 3: zero-order
// hold for A, Euler step for the input):
//
//   X = SiLU(conv1d(H));  [dt | B | C] = X W_x;  delta = softplus(dt W_dt + b_dt)
//   h_t = exp(delta_t A) (.) h_{t-1} + (delta_t x_t) B_t,   y_t = h_t C_t + D (.) x_t
//   with A = -exp(A_log), per channel d and state n.
//
// Kernels, in order (all on the caller's stream, no host synchronisation):
//  1. conv_silu_kernel: causal depthwise convolution (K taps, restart at
//     every sequence) + bias + SiLU; one thread per channel walks a chunk of
//     time steps. X is kept as two bf16 parts, hi and lo = bf16(X - hi).
//  2. the x projection, [hi | lo] x [W_x ; W_x] -> float32 [T][Np] (the
//     tensor-core grouped GEMM with one expert and K = 2 De, so the product
//     is accurate to ~2^-16 although the tensor cores take bf16; W_x stored
//     [Np][De], rows past R + 2N zero, doubled along K by dup_k_kernel).
//  3. dt_split_kernel: the dt columns as two bf16 parts.
//  4. the dt projection, the same way, K = 2R -> float32 [T][De].
//  5. the scan in chunks of kChunk steps, parallel over channels and chunks:
//     scan_kernel<false> turns dt W_dt into delta = softplus(. + b_dt) in
//     place and runs each chunk from a zero state, keeping its final state
//     and sum of delta; scan_carry_kernel chains the chunks of each
//     sequence (the state entering chunk c+1 is exp(A sum_c delta) times the
//     state entering chunk c plus chunk c's own final state); scan_kernel<true>
//     runs every chunk again from its entering state and writes y.
// With the x and dt projections expertized (RoM page, Knowl 3 and Knowl 9:
// "RoM (Conv, Gate, dt, x, Out)"), steps 2 and 4 gather the rows into the
// block's expert order, run the grouped GEMM with each slot's expert and sum
// a token's k slots in slot order.
// One thread owns one channel and all N <= 16 states of it in registers; the
// 32 lanes of a warp are 32 consecutive channels, so every per-step load of
// delta and x is one row segment, issued kBatch steps at a time (enough
// loads in flight to stream from HBM), and B_t, C_t (the same for every
// channel) are staged in shared memory per chunk.
#include <cuda_bf16.h>
#include <math.h>

#include <algorithm>

#include "../../include/rom.h"
#include "rom_internal.cuh"

namespace rom {
namespace {

constexpr int kMaxState = 16;
constexpr int kMaxTaps = 8;
constexpr int kChunk = 128;        // time steps per scan chunk
constexpr int kScanThreads = 128;  // channels per scan CTA
constexpr float kLog2e = 1.4426950408889634f;

// One thread per 4 adjacent channels and a chunk of kConvSteps time steps (a
// CTA holds 512 consecutive channels, so every load and store of a step is
// one row segment: 16-byte loads, 8-byte stores); the K - 1 previous inputs
// stay in registers, so each input is read once (plus K - 1 at the chunk's
// start), and the loads of kBatch steps are issued together. The tap count is
// a template parameter, which keeps taps and windows in few registers: many
// resident warps and wide loads keep enough bytes in flight (the kernel is
// bound by HBM latency otherwise). X is written as two bf16 parts per value,
// hi = bf16(v) in row t, columns [0, De) and lo = bf16(v - hi) in columns
// [De, 2 De): the x projection multiplies both by W_x (a product accurate to
// ~2^-16 on the bf16 tensor cores) and the scan reads hi + lo.
constexpr int kConvSteps = 64;
constexpr int kBatch = 8;  // time steps whose loads are issued together

__device__ __forceinline__ void split_bf16(float v, __nv_bfloat16& hi, __nv_bfloat16& lo) {
  hi = __float2bfloat16_rn(v);
  lo = __float2bfloat16_rn(v - __bfloat162float(hi));
}

__device__ __forceinline__ uint32_t bf16x2_bits(__nv_bfloat16 a, __nv_bfloat16 b) {
  return static_cast<uint32_t>(__bfloat16_as_ushort(a)) |
         (static_cast<uint32_t>(__bfloat16_as_ushort(b)) << 16);
}

template <int K>
__global__ void __launch_bounds__(128)
    conv_silu_kernel(const float* __restrict__ h, int64_t T, int De, int L,
                     const float* __restrict__ w, const float* __restrict__ b,
                     __nv_bfloat16* __restrict__ x2) {
  const int d0 = (blockIdx.x * 128 + threadIdx.x) * 4;  // channels d0 .. d0 + 3
  const int64_t t0 = static_cast<int64_t>(blockIdx.y) * kConvSteps;
  if (d0 >= De) return;
  float tap[4][K], win[4][K];  // win[c][j] = h_{t-1-j} of channel d0 + c (0 before the sequence)
  float bias[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
#pragma unroll
    for (int j = 0; j < K; ++j) {
      tap[c][j] = __ldg(w + static_cast<int64_t>(d0 + c) * K + j);
      win[c][j] = 0.f;
    }
    bias[c] = __ldg(b + d0 + c);
  }
  int64_t seq0 = (t0 / L) * L;
#pragma unroll
  for (int j = 0; j < K - 1; ++j)
    if (t0 - 1 - j >= seq0) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(h + (t0 - 1 - j) * De + d0));
      win[0][j] = v.x;
      win[1][j] = v.y;
      win[2][j] = v.z;
      win[3][j] = v.w;
    }
  const int n = static_cast<int>(T - t0 < kConvSteps ? T - t0 : kConvSteps);
  int64_t next_seq = seq0 + L;  // the windows restart where the next sequence begins
  const float* hp = h + t0 * De + d0;
  uint2* xp = reinterpret_cast<uint2*>(x2 + t0 * (2 * static_cast<int64_t>(De)) + d0);
  const int64_t row2 = (2 * static_cast<int64_t>(De)) / 4;  // one X row in uint2 (4 bf16)
  const int64_t lo_off = De / 4;
  for (int s0 = 0; s0 < n; s0 += kBatch) {
    float4 cur[kBatch];
#pragma unroll
    for (int q = 0; q < kBatch; ++q)
      cur[q] = s0 + q < n ? __ldg(reinterpret_cast<const float4*>(hp + static_cast<int64_t>(s0 + q) * De))
                          : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int q = 0; q < kBatch; ++q) {
      const int s = s0 + q;
      if (s >= n) break;
      if (t0 + s == next_seq) {
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int j = 0; j < K; ++j) win[c][j] = 0.f;
        next_seq += L;
      }
      const float cv[4] = {cur[q].x, cur[q].y, cur[q].z, cur[q].w};
      __nv_bfloat16 hi[4], lo[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        // tap K-1 multiplies the current step, tap K-1-j the step j back
        float acc = fmaf(tap[c][K - 1], cv[c], bias[c]);
#pragma unroll
        for (int j = 1; j < K; ++j) acc = fmaf(tap[c][K - 1 - j], win[c][j - 1], acc);
#pragma unroll
        for (int j = K - 1; j > 0; --j) win[c][j] = win[c][j - 1];
        win[c][0] = cv[c];
        // SiLU with the fast exp and divide (relative error ~1e-6; for
        // acc < -88 the quotient is SiLU's limit 0)
        split_bf16(__fdividef(acc, 1.0f + __expf(-acc)), hi[c], lo[c]);
      }
      uint2* dst = xp + static_cast<int64_t>(s) * row2;
      dst[0] = make_uint2(bf16x2_bits(hi[0], hi[1]), bf16x2_bits(hi[2], hi[3]));
      dst[lo_off] = make_uint2(bf16x2_bits(lo[0], lo[1]), bf16x2_bits(lo[2], lo[3]));
    }
  }
}

// The dt columns of [dt | B | C] as two bf16 parts: dt2[t] = [hi | lo]
// (the dt projection multiplies both by W_dt).
__global__ void __launch_bounds__(256)
    dt_split_kernel(const float* __restrict__ dbc, int64_t T, int Np, int R,
                    __nv_bfloat16* __restrict__ dt2) {
  const int64_t total = T * R;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = i / R;
    const int r = static_cast<int>(i - t * R);
    __nv_bfloat16 hi, lo;
    split_bf16(dbc[t * Np + r], hi, lo);
    dt2[t * 2 * R + r] = hi;
    dt2[t * 2 * R + R + r] = lo;
  }
}

// w2[row] = [w[row] | w[row]] (rows of K bf16, K % 8 == 0): the weight twice
// along K, so that one GEMM over [hi | lo] rows adds hi W + lo W.
__global__ void __launch_bounds__(256)
    dup_k_kernel(const uint4* __restrict__ w, int64_t rows, int kv, uint4* __restrict__ w2) {
  const int64_t total = rows * kv;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t row = i / kv;
    const int v = static_cast<int>(i - row * kv);
    const uint4 val = __ldg(w + i);
    w2[row * 2 * kv + v] = val;
    w2[row * 2 * kv + kv + v] = val;
  }
}

// dst[p] = src[sorted_slot[p] / k] (rows of row_vec16 16-byte vectors): the
// core's X or dt rows in the block's expert order, for expertized x and dt
// projections.
__global__ void __launch_bounds__(256)
    gather_rows_kernel(const uint4* __restrict__ src, int row_vec16,
                       const int32_t* __restrict__ sorted_slot, int k, int64_t R,
                       uint4* __restrict__ dst) {
  const int64_t total = R * row_vec16;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t p = i / row_vec16;
    const int v = static_cast<int>(i - p * row_vec16);
    dst[i] = __ldg(src + static_cast<int64_t>(sorted_slot[p] / k) * row_vec16 + v);
  }
}

// softplus(v) = ln(1 + e^v), accurate for small results (delta is often
// ~1e-3); for v > 20 it equals v in float32.
__device__ __forceinline__ float softplus_f(float v) {
  return v > 20.f ? v : log1pf(__expf(v));
}

// 2^v on the special-function unit (relative error ~2^-22; inputs here are
// <= 0, results underflow to 0 for v < -126).
__device__ __forceinline__ float ex2_approx(float v) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(v));
  return r;
}

struct ScanArgs {
  const __nv_bfloat16* x2;  // [T][2 De]: hi | lo parts of X
  float* delta;            // [T][De]: dt W_dt on entry; delta = softplus(. + b_dt) after pass 1
  const float* b_dt;       // [De]
  const float* dbc;        // [T][Np]: dt | B | C | zero padding
  const float* a_log;      // [De][N]
  const float* d;          // [De]
  float* S;                // [chunks][De]: sum of delta over a chunk
  float* hend;             // [chunks][N][De]: final state of a chunk from zero
  float* carry;            // [chunks][N][De]: state entering a chunk
  float* y;                // [T][De]
  int64_t T;
  int De, L, nc, Np, R, N;
};

// One chunk of one sequence for 128 channels.
// kOut = false: delta = softplus(dt W_dt + b_dt) written over its input, then
//   (except for a sequence's last chunk, which feeds nothing) the chunk's
//   own recurrence from a zero state: its final state and sum of delta.
// kOut = true: the recurrence again from the chunk's entering state, y out.
// NP: the state count rounded up to 4, 8 or 16 (the padded states have
// A = 0, B = C = 0 and stay 0). The states are updated in pairs with packed
// float32 arithmetic (one multiply for both exponents' arguments, one for
// both inputs, one fused multiply-add for both states, one for y's two
// partial sums), B and C are read from shared memory as float4 rows, and the
// loads of kBatch steps' delta and x are issued together.
template <bool kOut, int NP>
__global__ void __launch_bounds__(kScanThreads) scan_kernel(const ScanArgs a) {
  __shared__ __align__(16) float sB[kChunk][NP];
  __shared__ __align__(16) float sC[kOut ? kChunk : 1][NP];
  const int cg = blockIdx.y;  // chunk over all sequences
  const int seq = cg / a.nc, c = cg - (cg / a.nc) * a.nc;
  const bool last = c == a.nc - 1;
  const int d = blockIdx.x * kScanThreads + threadIdx.x;
  const int64_t t0 = static_cast<int64_t>(seq) * a.L + static_cast<int64_t>(c) * kChunk;
  const int len = min(kChunk, a.L - c * kChunk);
  const int N = a.N;
  float* dp = a.delta + t0 * a.De + d;
  if (!kOut && last) {
    const float bd = __ldg(a.b_dt + d);
    for (int s = 0; s < len; ++s) dp[s * a.De] = softplus_f(dp[s * a.De] + bd);
    return;
  }
  for (int i = threadIdx.x; i < len * NP; i += kScanThreads) {
    const int s = i / NP, n = i - (i / NP) * NP;
    const float* row = a.dbc + (t0 + s) * a.Np + a.R;
    sB[s][n] = n < N ? row[n] : 0.f;
    if (kOut) sC[s][n] = n < N ? row[N + n] : 0.f;
  }
  __syncthreads();
  float2 A2[NP / 2], h[NP / 2];
#pragma unroll
  for (int q = 0; q < NP / 2; ++q) {
    float av[2], hv[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int n = 2 * q + u;
      av[u] = n < N ? -expf(__ldg(a.a_log + static_cast<int64_t>(d) * N + n)) * kLog2e : 0.f;
      hv[u] = (kOut && n < N) ? a.carry[(static_cast<int64_t>(cg) * N + n) * a.De + d] : 0.f;
    }
    A2[q] = make_float2(av[0], av[1]);
    h[q] = make_float2(hv[0], hv[1]);
  }
  const float bd = kOut ? 0.f : __ldg(a.b_dt + d);
  const float Dd = kOut ? __ldg(a.d + d) : 0.f;
  // x = hi + lo of the two bf16 parts written by the convolution
  const __nv_bfloat16* xp = a.x2 + t0 * (2 * static_cast<int64_t>(a.De)) + d;
  float* yp = kOut ? a.y + t0 * a.De + d : nullptr;
  float ssum = 0.f;
  for (int s0 = 0; s0 < len; s0 += kBatch) {
    float pre[kBatch], xv[kBatch];
#pragma unroll
    for (int q = 0; q < kBatch; ++q) {
      const int s = s0 + q < len ? s0 + q : len - 1;
      pre[q] = dp[s * a.De];
      xv[q] = __bfloat162float(xp[static_cast<int64_t>(s) * 2 * a.De]) +
              __bfloat162float(xp[static_cast<int64_t>(s) * 2 * a.De + a.De]);
    }
#pragma unroll
    for (int q = 0; q < kBatch; ++q) {
      const int s = s0 + q;
      if (s >= len) break;
      float delta = pre[q];
      if (!kOut) {
        delta = softplus_f(pre[q] + bd);
        dp[s * a.De] = delta;
      }
      const float dx = delta * xv[q];
      ssum += delta;
      const float2 dd = make_float2(delta, delta), dx2 = make_float2(dx, dx);
      float2 y2 = make_float2(0.f, 0.f);
      const float4* b4 = reinterpret_cast<const float4*>(&sB[s][0]);
      const float4* c4 = reinterpret_cast<const float4*>(&sC[kOut ? s : 0][0]);
#pragma unroll
      for (int g = 0; g < NP / 4; ++g) {
        const float4 bq = b4[g];
        float4 cq;
        if (kOut) cq = c4[g];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int q2 = 2 * g + u;
          const float2 arg = __fmul2_rn(dd, A2[q2]);
          const float2 e = make_float2(ex2_approx(arg.x), ex2_approx(arg.y));
          const float2 bv = u == 0 ? make_float2(bq.x, bq.y) : make_float2(bq.z, bq.w);
          h[q2] = __ffma2_rn(e, h[q2], __fmul2_rn(dx2, bv));
          if (kOut) {
            const float2 cv = u == 0 ? make_float2(cq.x, cq.y) : make_float2(cq.z, cq.w);
            y2 = __ffma2_rn(h[q2], cv, y2);
          }
        }
      }
      if (kOut) yp[s * a.De] = fmaf(Dd, xv[q], y2.x + y2.y);
    }
  }
  if (!kOut) {
    a.S[static_cast<int64_t>(cg) * a.De + d] = ssum;
#pragma unroll
    for (int q = 0; q < NP / 2; ++q) {
      if (2 * q < N) a.hend[(static_cast<int64_t>(cg) * N + 2 * q) * a.De + d] = h[q].x;
      if (2 * q + 1 < N) a.hend[(static_cast<int64_t>(cg) * N + 2 * q + 1) * a.De + d] = h[q].y;
    }
  }
}

// State entering every chunk: one thread per (sequence, state, channel),
// sequential over the sequence's chunks.
__global__ void __launch_bounds__(256) scan_carry_kernel(const ScanArgs a, int nseq) {
  const int64_t total = static_cast<int64_t>(nseq) * a.N * a.De;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int d = static_cast<int>(i % a.De);
    const int n = static_cast<int>((i / a.De) % a.N);
    const int seq = static_cast<int>(i / (static_cast<int64_t>(a.De) * a.N));
    const float A2 = -expf(__ldg(a.a_log + static_cast<int64_t>(d) * a.N + n)) * kLog2e;
    float cin = 0.f;
    for (int c = 0; c < a.nc; ++c) {
      const int64_t cg = static_cast<int64_t>(seq) * a.nc + c;
      a.carry[(cg * a.N + n) * a.De + d] = cin;
      if (c + 1 < a.nc)
        cin = fmaf(ex2_approx(a.S[cg * a.De + d] * A2), cin, a.hend[(cg * a.N + n) * a.De + d]);
    }
  }
}

size_t align256(size_t v) { return (v + 255) / 256 * 256; }

struct CoreWs {
  __nv_bfloat16* x2;   // [T][2 De]: X as hi | lo bf16 parts
  float* dbc;          // [T][Np]: dt | B | C | 0
  __nv_bfloat16* dt2;  // [T][2 R]: dt as hi | lo bf16 parts
  float* dpre;         // [T][De]: dt W_dt, then delta
  float* S;
  float* hend;
  float* carry;
  __nv_bfloat16* wx2;   // [E][Np][2 De]: W_x twice along K
  __nv_bfloat16* wdt2;  // [E][De][2 R]: W_dt twice along K
  // expertized x and dt projections (k slots per token)
  __nv_bfloat16* xs;   // [T*k][2 De]: X rows in expert order
  __nv_bfloat16* dts;  // [T*k][2 R]: dt rows in expert order
  float* dbc_slots;    // [T*k][Np] (k > 1; else the token-order buffer)
  float* dpre_slots;   // [T*k][De] (k > 1; else the token-order buffer)
  size_t bytes;
};

// k == 0: the shared core (E == 1); k >= 1: expertized x and dt projections.
CoreWs core_ws_layout(void* base, int64_t T, int De, int seq_len, int R, int N, int Np, int E,
                      int k) {
  const int64_t nchunks = (T / seq_len) * ((seq_len + kChunk - 1) / kChunk);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align256(bytes);
    return static_cast<uint8_t*>(base) + o;
  };
  CoreWs w;
  w.x2 = reinterpret_cast<__nv_bfloat16*>(take(static_cast<size_t>(T) * De * 4));
  w.dbc = reinterpret_cast<float*>(take(static_cast<size_t>(T) * Np * 4));
  w.dt2 = reinterpret_cast<__nv_bfloat16*>(take(static_cast<size_t>(T) * R * 4));
  w.dpre = reinterpret_cast<float*>(take(static_cast<size_t>(T) * De * 4));
  w.S = reinterpret_cast<float*>(take(static_cast<size_t>(nchunks) * De * 4));
  w.hend = reinterpret_cast<float*>(take(static_cast<size_t>(nchunks) * N * De * 4));
  w.carry = reinterpret_cast<float*>(take(static_cast<size_t>(nchunks) * N * De * 4));
  w.wx2 = reinterpret_cast<__nv_bfloat16*>(take(static_cast<size_t>(E) * Np * De * 4));
  w.wdt2 = reinterpret_cast<__nv_bfloat16*>(take(static_cast<size_t>(E) * De * R * 4));
  w.xs = w.dts = nullptr;
  w.dbc_slots = w.dbc;
  w.dpre_slots = w.dpre;
  if (k >= 1) {
    const size_t Rs = static_cast<size_t>(T) * k;
    w.xs = reinterpret_cast<__nv_bfloat16*>(take(Rs * De * 4));
    w.dts = reinterpret_cast<__nv_bfloat16*>(take(Rs * R * 4));
    if (k > 1) {
      w.dbc_slots = reinterpret_cast<float*>(take(Rs * Np * 4));
      w.dpre_slots = reinterpret_cast<float*>(take(Rs * De * 4));
    }
  }
  w.bytes = off;
  return w;
}

unsigned grid_for(int64_t total, int threads) {
  const int64_t want = (total + threads - 1) / threads;
  return static_cast<unsigned>(std::max<int64_t>(
      1, std::min<int64_t>(want, static_cast<int64_t>(device_sm_count()) * 16)));
}

}  // namespace

size_t ssm_core_workspace_bytes(int64_t T, int De, int seq_len, int R, int N, int Np, int E,
                                int k) {
  return core_ws_layout(nullptr, T, De, seq_len, R, N, Np, E, k).bytes;
}

// One projection of the core, to float32 rows in token order: shared (one
// matrix over the T rows in order) or expertized (the rows gathered into the
// block's expert order, the grouped GEMM with each slot's expert, the k
// slots of a token summed in slot order).
cudaError_t core_projection(const __nv_bfloat16* a, int64_t T, int Kdim, const void* w, int Nout,
                            int E, int k, const int32_t* offsets, const int32_t* sorted_slot,
                            __nv_bfloat16* a_sorted, float* out_slots, float* out, int* status,
                            cudaStream_t stream) {
  if (k == 0)
    return launch_tc_grouped_gemm(kEpiScaleSlots, a, T, Kdim, w, nullptr, Nout, 1, 1, nullptr,
                                  nullptr, nullptr, out, status, stream);
  const int64_t R = T * k;
  gather_rows_kernel<<<grid_for(R * (Kdim / 8), 256), 256, 0, stream>>>(
      reinterpret_cast<const uint4*>(a), Kdim / 8, sorted_slot, k, R,
      reinterpret_cast<uint4*>(a_sorted));
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = launch_tc_grouped_gemm(kEpiScaleSlots, a_sorted, R, Kdim, w, nullptr, Nout, E, k, offsets,
                             sorted_slot, nullptr, out_slots, status, stream);
  if (e != cudaSuccess || k == 1) return e;
  return launch_combine(0, false, out_slots, T, k, Nout, nullptr, out, stream);
}

cudaError_t launch_ssm_core(const float* h, int64_t T, int De, int seq_len, const float* conv_w,
                            const float* conv_b, int K, const void* w_x, int R, int N, int Np,
                            const void* w_dt, const float* b_dt, const float* a_log,
                            const float* d, int E, int k, const int32_t* offsets,
                            const int32_t* sorted_slot, float* y, void* ws, int* status,
                            cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  const CoreWs w = core_ws_layout(ws, T, De, seq_len, R, N, Np, E, k);
  // the projections' weights twice along K (one GEMM then adds hi W + lo W)
  const int64_t ex = static_cast<int64_t>(E);
  dup_k_kernel<<<grid_for(ex * Np * (De / 8), 256), 256, 0, stream>>>(
      static_cast<const uint4*>(w_x), ex * Np, De / 8, reinterpret_cast<uint4*>(w.wx2));
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dup_k_kernel<<<grid_for(ex * De * (R / 8), 256), 256, 0, stream>>>(
      static_cast<const uint4*>(w_dt), ex * De, R / 8, reinterpret_cast<uint4*>(w.wdt2));
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  {
    const dim3 grid(static_cast<unsigned>((De + 511) / 512),
                    static_cast<unsigned>((T + kConvSteps - 1) / kConvSteps));
    switch (K) {
#define ROM_CONV_CASE(KV)                                                                    \
  case KV:                                                                                   \
    conv_silu_kernel<KV><<<grid, 128, 0, stream>>>(h, T, De, seq_len, conv_w, conv_b, w.x2); \
    break;
      ROM_CONV_CASE(1)
      ROM_CONV_CASE(2)
      ROM_CONV_CASE(3)
      ROM_CONV_CASE(4)
      ROM_CONV_CASE(5)
      ROM_CONV_CASE(6)
      ROM_CONV_CASE(7)
      ROM_CONV_CASE(8)
#undef ROM_CONV_CASE
      default:
        return cudaErrorInvalidValue;
    }
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // x projection to [dt | B | C | 0] float32 rows, token order
  e = core_projection(w.x2, T, 2 * De, w.wx2, Np, E, k, offsets, sorted_slot, w.xs, w.dbc_slots,
                      w.dbc, status, stream);
  if (e != cudaSuccess) return e;
  dt_split_kernel<<<grid_for(T * R, 256), 256, 0, stream>>>(w.dbc, T, Np, R, w.dt2);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = core_projection(w.dt2, T, 2 * R, w.wdt2, De, E, k, offsets, sorted_slot, w.dts,
                      w.dpre_slots, w.dpre, status, stream);
  if (e != cudaSuccess) return e;
  ScanArgs a;
  a.x2 = w.x2;
  a.delta = w.dpre;
  a.b_dt = b_dt;
  a.dbc = w.dbc;
  a.a_log = a_log;
  a.d = d;
  a.S = w.S;
  a.hend = w.hend;
  a.carry = w.carry;
  a.y = y;
  a.T = T;
  a.De = De;
  a.L = seq_len;
  a.nc = (seq_len + kChunk - 1) / kChunk;
  a.Np = Np;
  a.R = R;
  a.N = N;
  const int nseq = static_cast<int>(T / seq_len);
  const dim3 grid(static_cast<unsigned>(De / kScanThreads),
                  static_cast<unsigned>(static_cast<int64_t>(nseq) * a.nc));
  // states padded to 4, 8 or 16
  const int np = N <= 4 ? 4 : N <= 8 ? 8 : 16;
  if (np == 4) scan_kernel<false, 4><<<grid, kScanThreads, 0, stream>>>(a);
  else if (np == 8) scan_kernel<false, 8><<<grid, kScanThreads, 0, stream>>>(a);
  else scan_kernel<false, 16><<<grid, kScanThreads, 0, stream>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  scan_carry_kernel<<<grid_for(static_cast<int64_t>(nseq) * N * De, 256), 256, 0, stream>>>(
      a, nseq);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (np == 4) scan_kernel<true, 4><<<grid, kScanThreads, 0, stream>>>(a);
  else if (np == 8) scan_kernel<true, 8><<<grid, kScanThreads, 0, stream>>>(a);
  else scan_kernel<true, 16><<<grid, kScanThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace rom

namespace {

int ssm_core_entry(const float* h, int64_t T, int De, int seq_len, const float* conv_w,
                   const float* conv_b, int K, const void* w_x, int R, int N, int Np,
                   const void* w_dt, const float* b_dt, const float* a_log, const float* d, int E,
                   int k, const int32_t* offsets, const int32_t* sorted_slot, float* y, void* ws,
                   size_t ws_bytes, void* stream) {
  if (T < 0 || De <= 0 || seq_len <= 0 || K < 1 || R < 1 || N < 1) return ROM_ERR_INVALID_ARG;
  if (k > 0 && (E < 1 || E > rom::kMaxExperts || k > E || k > rom::kMaxTopK))
    return ROM_ERR_INVALID_ARG;
  if (k > 0 && T > 0 && (!offsets || !sorted_slot)) return ROM_ERR_INVALID_ARG;
  if (T * (k > 0 ? k : 1) >= (int64_t(1) << 31)) return ROM_ERR_UNSUPPORTED;
  if (T > 0 && T % seq_len != 0) return ROM_ERR_INVALID_ARG;
  if (K > rom::kMaxTaps || N > rom::kMaxState || De % 128 != 0 || R % 8 != 0 ||
      Np % 128 != 0 || Np < R + 2 * N || T >= (int64_t(1) << 31))
    return ROM_ERR_UNSUPPORTED;
  if (T == 0) return ROM_OK;
  if (!h || !conv_w || !conv_b || !w_x || !w_dt || !b_dt || !a_log || !d || !y)
    return ROM_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(h) & 15u) || (reinterpret_cast<uintptr_t>(w_x) & 15u) ||
      (reinterpret_cast<uintptr_t>(w_dt) & 15u))
    return ROM_ERR_UNSUPPORTED;
  if (!ws || ws_bytes < rom::ssm_core_workspace_bytes(T, De, seq_len, R, N, Np, k > 0 ? E : 1, k) ||
      (reinterpret_cast<uintptr_t>(ws) & 255u))
    return ROM_ERR_WORKSPACE;
  int* st = rom::status_ptr();
  if (!st) return ROM_ERR_CUDA;
  const cudaError_t e = rom::launch_ssm_core(h, T, De, seq_len, conv_w, conv_b, K, w_x, R, N, Np,
                                             w_dt, b_dt, a_log, d, E, k, offsets, sorted_slot, y,
                                             ws, st, static_cast<cudaStream_t>(stream));
  if (e == cudaSuccess) return ROM_OK;
  return e == cudaErrorInvalidValue ? ROM_ERR_UNSUPPORTED : ROM_ERR_CUDA;
}

bool core_sizes_ok(int64_t T, int De, int seq_len, int R, int N, int Np) {
  return T > 0 && De > 0 && seq_len > 0 && T % seq_len == 0 && R > 0 && N > 0 && Np > 0;
}

}  // namespace

extern "C" size_t rom_ssm_core_workspace_size(int64_t T, int De, int seq_len, int R, int N,
                                              int Np) {
  if (!core_sizes_ok(T, De, seq_len, R, N, Np)) return 0;
  return rom::ssm_core_workspace_bytes(T, De, seq_len, R, N, Np, 1, 0);
}

extern "C" size_t rom_ssm_core_routed_workspace_size(int64_t T, int De, int seq_len, int R, int N,
                                                     int Np, int E, int k) {
  if (!core_sizes_ok(T, De, seq_len, R, N, Np) || k < 1 || E < 1) return 0;
  return rom::ssm_core_workspace_bytes(T, De, seq_len, R, N, Np, E, k);
}

extern "C" int rom_ssm_core(const float* h, int64_t T, int De, int seq_len, const float* conv_w,
                            const float* conv_b, int K, const void* w_x, int R, int N, int Np,
                            const void* w_dt, const float* b_dt, const float* a_log,
                            const float* d, float* y, void* ws, size_t ws_bytes, void* stream) {
  return ssm_core_entry(h, T, De, seq_len, conv_w, conv_b, K, w_x, R, N, Np, w_dt, b_dt, a_log, d,
                        1, 0, nullptr, nullptr, y, ws, ws_bytes, stream);
}

extern "C" int rom_ssm_core_routed(const float* h, int64_t T, int De, int seq_len,
                                   const float* conv_w, const float* conv_b, int K,
                                   const void* w_x, int R, int N, int Np, const void* w_dt,
                                   const float* b_dt, const float* a_log, const float* d, int E,
                                   int k, const int32_t* offsets, const int32_t* sorted_slot,
                                   float* y, void* ws, size_t ws_bytes, void* stream) {
  if (k < 1) return ROM_ERR_INVALID_ARG;
  return ssm_core_entry(h, T, De, seq_len, conv_w, conv_b, K, w_x, R, N, Np, w_dt, b_dt, a_log, d,
                        E, k, offsets, sorted_slot, y, ws, ws_bytes, stream);
}
