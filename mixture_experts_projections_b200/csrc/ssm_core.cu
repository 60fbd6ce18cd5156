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
//     every sequence) + bias + SiLU, bf16 X (the A operand of the next GEMM);
//     one thread per channel walks a chunk of time steps.
//  2. the x projection, X [T][De] x W_x -> float32 [T][Np] (the tensor-core
//     grouped GEMM with one expert; W_x stored [Np][De], rows past R + 2N
//     zero).
//  3. dt_cast_kernel: the dt columns to bf16 [T][R].
//  4. the dt projection, dt [T][R] x W_dt -> float32 [T][De] (same GEMM).
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
// delta and x is one 128-byte row segment, and B_t, C_t (the same for every
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

// One thread per channel and a chunk of kConvSteps time steps (a CTA holds
// 128 consecutive channels, so every load and store of a step is one row
// segment); the K - 1 previous inputs stay in registers, so each input is
// read once (plus K - 1 at the chunk's start).
constexpr int kConvSteps = 64;

__global__ void __launch_bounds__(128)
    conv_silu_kernel(const float* __restrict__ h, int64_t T, int De, int L,
                     const float* __restrict__ w, const float* __restrict__ b, int K,
                     __nv_bfloat16* __restrict__ x) {
  const int d = blockIdx.x * 128 + threadIdx.x;
  const int64_t t0 = static_cast<int64_t>(blockIdx.y) * kConvSteps;
  if (d >= De) return;
  float tap[kMaxTaps], win[kMaxTaps];  // win[j] = h_{t-1-j} (0 before the sequence)
#pragma unroll
  for (int j = 0; j < kMaxTaps; ++j) {
    tap[j] = j < K ? __ldg(w + static_cast<int64_t>(d) * K + j) : 0.f;
    win[j] = 0.f;
  }
  const float bias = __ldg(b + d);
  int64_t seq0 = (t0 / L) * L;
#pragma unroll
  for (int j = 0; j < kMaxTaps - 1; ++j)
    if (j < K - 1 && t0 - 1 - j >= seq0) win[j] = __ldg(h + (t0 - 1 - j) * De + d);
  const int n = static_cast<int>(T - t0 < kConvSteps ? T - t0 : kConvSteps);
  int64_t next_seq = seq0 + L;  // the window restarts where the next sequence begins
  const float* hp = h + t0 * De + d;
  __nv_bfloat16* xp = x + t0 * De + d;
  for (int s = 0; s < n; ++s) {
    if (t0 + s == next_seq) {
#pragma unroll
      for (int j = 0; j < kMaxTaps; ++j) win[j] = 0.f;
      next_seq += L;
    }
    const float cur = __ldg(hp + static_cast<int64_t>(s) * De);
    // tap K-1 multiplies the current step, tap K-1-j the step j back
    float acc = fmaf(tap[K - 1], cur, bias);
#pragma unroll
    for (int j = 1; j < kMaxTaps; ++j)
      if (j < K) acc = fmaf(tap[K - 1 - j], win[j - 1], acc);
#pragma unroll
    for (int j = kMaxTaps - 1; j > 0; --j) win[j] = win[j - 1];
    win[0] = cur;
    // SiLU with the fast exp and divide (their error is far below the bf16
    // rounding of X; for acc < -88 the quotient is SiLU's limit 0)
    xp[static_cast<int64_t>(s) * De] = __float2bfloat16_rn(__fdividef(acc, 1.0f + __expf(-acc)));
  }
}

__global__ void __launch_bounds__(256)
    dt_cast_kernel(const float* __restrict__ dbc, int64_t T, int Np, int R,
                   __nv_bfloat16* __restrict__ dt) {
  const int64_t total = T * R;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = i / R;
    const int r = static_cast<int>(i - t * R);
    dt[i] = __float2bfloat16_rn(dbc[t * Np + r]);
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
  const __nv_bfloat16* x;  // [T][De]
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
// Each step's delta and x are loaded one step ahead of their use.
template <bool kOut>
__global__ void __launch_bounds__(kScanThreads) scan_kernel(const ScanArgs a) {
  __shared__ float sB[kChunk][kMaxState];
  __shared__ float sC[kOut ? kChunk : 1][kMaxState];
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
  for (int i = threadIdx.x; i < len * N; i += kScanThreads) {
    const int s = i / N, n = i - (i / N) * N;
    const float* row = a.dbc + (t0 + s) * a.Np + a.R;
    sB[s][n] = row[n];
    if (kOut) sC[s][n] = row[N + n];
  }
  __syncthreads();
  float A2[kMaxState], h[kMaxState];
#pragma unroll
  for (int n = 0; n < kMaxState; ++n) {
    A2[n] = n < N ? -expf(__ldg(a.a_log + static_cast<int64_t>(d) * N + n)) * kLog2e : 0.f;
    h[n] = (kOut && n < N) ? a.carry[(static_cast<int64_t>(cg) * N + n) * a.De + d] : 0.f;
  }
  const float bd = kOut ? 0.f : __ldg(a.b_dt + d);
  const float Dd = kOut ? __ldg(a.d + d) : 0.f;
  const __nv_bfloat16* xp = a.x + t0 * a.De + d;
  float* yp = kOut ? a.y + t0 * a.De + d : nullptr;
  float ssum = 0.f;
  float pre_next = dp[0];
  float x_next = __bfloat162float(xp[0]);
  for (int s = 0; s < len; ++s) {
    const float pre = pre_next, xv = x_next;
    if (s + 1 < len) {
      pre_next = dp[(s + 1) * a.De];
      x_next = __bfloat162float(xp[(s + 1) * a.De]);
    }
    float delta = pre;
    if (!kOut) {
      delta = softplus_f(pre + bd);
      dp[s * a.De] = delta;
    }
    const float dx = delta * xv;
    ssum += delta;
    float yv = 0.f;
#pragma unroll
    for (int n = 0; n < kMaxState; ++n) {
      if (n < N) {
        h[n] = fmaf(ex2_approx(delta * A2[n]), h[n], dx * sB[s][n]);
        if (kOut) yv = fmaf(h[n], sC[s][n], yv);
      }
    }
    if (kOut) yp[s * a.De] = fmaf(Dd, xv, yv);
  }
  if (!kOut) {
    a.S[static_cast<int64_t>(cg) * a.De + d] = ssum;
#pragma unroll
    for (int n = 0; n < kMaxState; ++n)
      if (n < N) a.hend[(static_cast<int64_t>(cg) * N + n) * a.De + d] = h[n];
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
  __nv_bfloat16* x;
  float* dbc;
  __nv_bfloat16* dt;
  float* dpre;
  float* S;
  float* hend;
  float* carry;
  // expertized x and dt projections (k slots per token)
  __nv_bfloat16* xs;   // [T*k][De]: X rows in expert order
  __nv_bfloat16* dts;  // [T*k][R]: dt rows in expert order
  float* dbc_slots;    // [T*k][Np] (k > 1; else the token-order buffer)
  float* dpre_slots;   // [T*k][De] (k > 1; else the token-order buffer)
  size_t bytes;
};

// k == 0: the shared core; k >= 1: expertized x and dt projections.
CoreWs core_ws_layout(void* base, int64_t T, int De, int seq_len, int R, int N, int Np,
                      int k = 0) {
  const int64_t nchunks = (T / seq_len) * ((seq_len + kChunk - 1) / kChunk);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align256(bytes);
    return static_cast<uint8_t*>(base) + o;
  };
  CoreWs w;
  w.x = reinterpret_cast<__nv_bfloat16*>(take(static_cast<size_t>(T) * De * 2));
  w.dbc = reinterpret_cast<float*>(take(static_cast<size_t>(T) * Np * 4));
  w.dt = reinterpret_cast<__nv_bfloat16*>(take(static_cast<size_t>(T) * R * 2));
  w.dpre = reinterpret_cast<float*>(take(static_cast<size_t>(T) * De * 4));
  w.S = reinterpret_cast<float*>(take(static_cast<size_t>(nchunks) * De * 4));
  w.hend = reinterpret_cast<float*>(take(static_cast<size_t>(nchunks) * N * De * 4));
  w.carry = reinterpret_cast<float*>(take(static_cast<size_t>(nchunks) * N * De * 4));
  w.xs = w.dts = nullptr;
  w.dbc_slots = w.dbc;
  w.dpre_slots = w.dpre;
  if (k >= 1) {
    const size_t Rs = static_cast<size_t>(T) * k;
    w.xs = reinterpret_cast<__nv_bfloat16*>(take(Rs * De * 2));
    w.dts = reinterpret_cast<__nv_bfloat16*>(take(Rs * R * 2));
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

size_t ssm_core_workspace_bytes(int64_t T, int De, int seq_len, int R, int N, int Np, int k) {
  return core_ws_layout(nullptr, T, De, seq_len, R, N, Np, k).bytes;
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
  const CoreWs w = core_ws_layout(ws, T, De, seq_len, R, N, Np, k);
  conv_silu_kernel<<<dim3(static_cast<unsigned>(De / 128),
                         static_cast<unsigned>((T + kConvSteps - 1) / kConvSteps)),
                    128, 0, stream>>>(h, T, De, seq_len, conv_w, conv_b, K, w.x);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // x projection to [dt | B | C | 0] float32 rows, token order
  e = core_projection(w.x, T, De, w_x, Np, E, k, offsets, sorted_slot, w.xs, w.dbc_slots, w.dbc,
                      status, stream);
  if (e != cudaSuccess) return e;
  dt_cast_kernel<<<grid_for(T * R, 256), 256, 0, stream>>>(w.dbc, T, Np, R, w.dt);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = core_projection(w.dt, T, R, w_dt, De, E, k, offsets, sorted_slot, w.dts, w.dpre_slots,
                      w.dpre, status, stream);
  if (e != cudaSuccess) return e;
  ScanArgs a;
  a.x = w.x;
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
  scan_kernel<false><<<grid, kScanThreads, 0, stream>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  scan_carry_kernel<<<grid_for(static_cast<int64_t>(nseq) * N * De, 256), 256, 0, stream>>>(
      a, nseq);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  scan_kernel<true><<<grid, kScanThreads, 0, stream>>>(a);
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
  if (!ws || ws_bytes < rom::ssm_core_workspace_bytes(T, De, seq_len, R, N, Np, k) ||
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
  return rom::ssm_core_workspace_bytes(T, De, seq_len, R, N, Np, 0);
}

extern "C" size_t rom_ssm_core_routed_workspace_size(int64_t T, int De, int seq_len, int R, int N,
                                                     int Np, int k) {
  if (!core_sizes_ok(T, De, seq_len, R, N, Np) || k < 1) return 0;
  return rom::ssm_core_workspace_bytes(T, De, seq_len, R, N, Np, k);
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
