// C ABI of librom.so: argument validation, mode selection and launches.
// The declarations and their contracts are in include/rom.h.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/rom.h"
#include "rom_internal.cuh"
#include "sm100_ptx.cuh"

namespace rom {

// One device status word per device (set by bounded waits that ran out).
__device__ int g_status_word;

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
int g_sm_count[kMaxDevices];
int* g_status_ptr[kMaxDevices];

int current_device() {
  int d = 0;
  if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= kMaxDevices) return -1;
  return d;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int to_status(cudaError_t e) {
  if (e == cudaSuccess) return ROM_OK;
  if (e == cudaErrorInvalidValue) return ROM_ERR_UNSUPPORTED;
  return ROM_ERR_CUDA;
}

__global__ void debug_wait_kernel(uint64_t limit_ns, int* status) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  // Nothing ever arrives on `bar`: the wait must run out and report.
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, status, limit_ns);
}

}  // namespace

int* status_ptr() {
  const int d = current_device();
  if (d < 0) return nullptr;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_status_ptr[d]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return nullptr;
    g_status_ptr[d] = static_cast<int*>(p);
  }
  return g_status_ptr[d];
}

int device_sm_count() {
  const int d = current_device();
  if (d < 0) return 1;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_sm_count[d] <= 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, d) != cudaSuccess || n <= 0)
      n = 1;
    g_sm_count[d] = n;
  }
  return g_sm_count[d];
}

}  // namespace rom

using rom::aligned16;

extern "C" {

const char* rom_status_string(int status) {
  switch (status) {
    case ROM_OK:
      return "ROM_OK";
    case ROM_ERR_INVALID_ARG:
      return "ROM_ERR_INVALID_ARG";
    case ROM_ERR_UNSUPPORTED:
      return "ROM_ERR_UNSUPPORTED";
    case ROM_ERR_WORKSPACE:
      return "ROM_ERR_WORKSPACE";
    case ROM_ERR_CUDA:
      return "ROM_ERR_CUDA";
    case ROM_ERR_TIMEOUT:
      return "ROM_ERR_TIMEOUT";
    case ROM_ERR_ROUTING:
      return "ROM_ERR_ROUTING";
    default:
      return "ROM_ERR_UNKNOWN";
  }
}

int rom_version(void) { return 2; }

size_t rom_workspace_size(int64_t T, int E) {
  if (T <= 0 || E <= 0) return 0;
  return static_cast<size_t>(rom::num_chunks(T)) * static_cast<size_t>(E) * sizeof(int32_t);
}

int rom_route(const void* x, int dtype, int64_t T, int Dm, const float* w_r, const float* bias,
              int E, int k, int renorm, int32_t* topk_idx, float* topk_w, int32_t* counts,
              void* ws, size_t ws_bytes, void* stream) {
  if (dtype != ROM_F32 && dtype != ROM_BF16) return ROM_ERR_INVALID_ARG;
  if (T < 0 || Dm <= 0 || E < 1 || E > rom::kMaxExperts || k < 1 || k > E ||
      k > rom::kMaxTopK || (renorm != 0 && renorm != 1))
    return ROM_ERR_INVALID_ARG;
  if (T * k >= (int64_t(1) << 31)) return ROM_ERR_UNSUPPORTED;
  const bool bf16 = dtype == ROM_BF16;
  if (Dm % (bf16 ? 8 : 4) != 0) return ROM_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (T > 0) {
    if (!x || !w_r || !topk_idx || !topk_w) return ROM_ERR_INVALID_ARG;
    if (!aligned16(x)) return ROM_ERR_UNSUPPORTED;
    if (ws && ws_bytes < rom_workspace_size(T, E)) return ROM_ERR_WORKSPACE;
  }
  if (counts) {
    const cudaError_t e = cudaMemsetAsync(counts, 0, sizeof(int32_t) * E, s);
    if (e != cudaSuccess) return ROM_ERR_CUDA;
  }
  if (T == 0) return ROM_OK;
  int* st = rom::status_ptr();
  if (!st) return ROM_ERR_CUDA;
  return rom::to_status(rom::launch_router(x, bf16, T, Dm, w_r, bias, E, k, renorm, topk_idx,
                                           topk_w, counts, static_cast<int32_t*>(ws), st, s));
}

int rom_dispatch(const void* x, int dtype, int64_t T, int Dm, int E, int k,
                 const int32_t* topk_idx, const void* ws, size_t ws_bytes, int32_t* offsets,
                 int32_t* sorted_slot, int32_t* slot_pos, void* x_sorted, void* stream) {
  if (dtype != ROM_F32 && dtype != ROM_BF16) return ROM_ERR_INVALID_ARG;
  if (T < 0 || Dm <= 0 || E < 1 || E > rom::kMaxExperts || k < 1 || k > E || k > rom::kMaxTopK)
    return ROM_ERR_INVALID_ARG;
  if (T * k >= (int64_t(1) << 31)) return ROM_ERR_UNSUPPORTED;
  const bool bf16 = dtype == ROM_BF16;
  if (Dm % (bf16 ? 8 : 4) != 0) return ROM_ERR_UNSUPPORTED;
  if (!offsets) return ROM_ERR_INVALID_ARG;
  if (T > 0) {
    if (!x || !topk_idx || !sorted_slot || !slot_pos || !x_sorted) return ROM_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(x_sorted)) return ROM_ERR_UNSUPPORTED;
    if (!ws || ws_bytes < rom_workspace_size(T, E)) return ROM_ERR_WORKSPACE;
  }
  int* st = rom::status_ptr();
  if (!st) return ROM_ERR_CUDA;
  return rom::to_status(rom::launch_dispatch(x, bf16, T, Dm, E, k, topk_idx,
                                             static_cast<const int32_t*>(ws), offsets,
                                             sorted_slot, slot_pos, x_sorted, st,
                                             static_cast<cudaStream_t>(stream)));
}

int rom_expert_proj(int proj, int dtype, const void* a_sorted, int64_t R, int K, const void* w0,
                    const void* w1, int N, int E, int k, const int32_t* offsets,
                    const int32_t* sorted_slot, const float* topk_w, void* out, void* stream) {
  if (proj != ROM_PROJ_CONV_GATE && proj != ROM_PROJ_OUT && proj != ROM_PROJ_INPROJ &&
      proj != ROM_PROJ_SLOTS && proj != ROM_PROJ_CONV_GATE_SLOTS)
    return ROM_ERR_INVALID_ARG;
  if (dtype != ROM_F32 && dtype != ROM_BF16) return ROM_ERR_INVALID_ARG;
  if (R < 0 || K <= 0 || N <= 0 || E < 1 || E > rom::kMaxExperts || k < 1 || k > E ||
      k > rom::kMaxTopK || R % k != 0)
    return ROM_ERR_INVALID_ARG;
  if (R >= (int64_t(1) << 31)) return ROM_ERR_UNSUPPORTED;
  const bool gate = proj == ROM_PROJ_CONV_GATE || proj == ROM_PROJ_CONV_GATE_SLOTS;
  const bool gate_slots = proj == ROM_PROJ_CONV_GATE_SLOTS || (gate && k > 1);
  const bool slots = proj == ROM_PROJ_SLOTS;
  // A dense projection (ROM_PROJ_SLOTS only): no routing arrays, one matrix.
  const bool dense = slots && !offsets && !sorted_slot;
  if (dense && E != 1) return ROM_ERR_INVALID_ARG;
  if ((!offsets && !dense) || !w0 || !out || (gate && !w1)) return ROM_ERR_INVALID_ARG;
  if (!gate && !dense && (!sorted_slot || (!slots && !topk_w))) return ROM_ERR_INVALID_ARG;
  if (gate_slots && !sorted_slot) return ROM_ERR_INVALID_ARG;
  if (R > 0 && !a_sorted) return ROM_ERR_INVALID_ARG;
  if (slots) w1 = nullptr;
  // ROM_PROJ_SLOTS is the slot-order float32 epilogue; r = 1 when topk_w is
  // NULL, and row p is slot p when sorted_slot is NULL.
  const int mode = gate    ? (gate_slots ? rom::kEpiGateSlots : rom::kEpiGateH)
                   : slots ? rom::kEpiScaleSlots
                           : (k == 1 ? rom::kEpiScaleToken : rom::kEpiScaleSlots);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dtype == ROM_F32) {
    return rom::to_status(rom::launch_simt_grouped_gemm(
        mode, static_cast<const float*>(a_sorted), R, K, static_cast<const float*>(w0),
        static_cast<const float*>(w1), N, E, k, offsets, sorted_slot, topk_w,
        static_cast<float*>(out), s));
  }
  if (K % 8 != 0 || N % 128 != 0) return ROM_ERR_UNSUPPORTED;
  if (!aligned16(a_sorted) || !aligned16(w0) || (gate && !aligned16(w1)) || !aligned16(out))
    return ROM_ERR_UNSUPPORTED;
  int* st = rom::status_ptr();
  if (!st) return ROM_ERR_CUDA;
  return rom::to_status(rom::launch_tc_grouped_gemm(mode, a_sorted, R, K, w0, w1, N, E, k,
                                                    offsets, sorted_slot, topk_w, out, st, s));
}

int rom_expert_proj_dense(int proj, int dtype, const void* x, int64_t T, int K, const void* w,
                          int N, int E, int k, const int32_t* topk_idx, const float* topk_w,
                          void* out, void* stream) {
  const bool w_tiled = (proj & ROM_W_TILED) != 0;
  proj &= ~ROM_W_TILED;
  if (proj != ROM_PROJ_OUT && proj != ROM_PROJ_INPROJ) return ROM_ERR_INVALID_ARG;
  if (dtype != ROM_F32 && dtype != ROM_BF16) return ROM_ERR_INVALID_ARG;
  if (T < 0 || K <= 0 || N <= 0 || E < 1 || E > rom::kMaxExperts || k < 1 || k > E ||
      k > rom::kMaxTopK)
    return ROM_ERR_INVALID_ARG;
  if (dtype != ROM_BF16 || T > 64 || K % 8 != 0 || N % 128 != 0) return ROM_ERR_UNSUPPORTED;
  if (w_tiled && K % 64 != 0) return ROM_ERR_UNSUPPORTED;
  if (T == 0) return ROM_OK;
  if (!x || !w || !topk_idx || !topk_w || !out) return ROM_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w) || !aligned16(out)) return ROM_ERR_UNSUPPORTED;
  int* st = rom::status_ptr();
  if (!st) return ROM_ERR_CUDA;
  return rom::to_status(rom::launch_tc_dense_small(
      k == 1 ? rom::kEpiScaleToken : rom::kEpiScaleSlots, x, T, K, w, N, E, k, topk_idx, topk_w,
      out, w_tiled, st, static_cast<cudaStream_t>(stream)));
}

int rom_pack_expert_weights(int dtype, const void* w, int E, int N, int K, void* w_tiled,
                            void* stream) {
  if (dtype != ROM_F32 && dtype != ROM_BF16) return ROM_ERR_INVALID_ARG;
  if (E < 1 || N <= 0 || K <= 0) return ROM_ERR_INVALID_ARG;
  if (dtype != ROM_BF16 || N % 128 != 0 || K % 64 != 0) return ROM_ERR_UNSUPPORTED;
  if (!w || !w_tiled) return ROM_ERR_INVALID_ARG;
  if (!aligned16(w) || !aligned16(w_tiled)) return ROM_ERR_UNSUPPORTED;
  const uintptr_t a = reinterpret_cast<uintptr_t>(w), b = reinterpret_cast<uintptr_t>(w_tiled);
  const uintptr_t bytes = static_cast<uintptr_t>(E) * N * K * 2;
  if (a < b + bytes && b < a + bytes) return ROM_ERR_INVALID_ARG;  // overlapping
  return rom::to_status(rom::launch_pack_expert_weights(w, E, N, K, w_tiled,
                                                        static_cast<cudaStream_t>(stream)));
}

int rom_combine(int mode, int dtype, const void* in, int64_t T, int k, int N,
                const int32_t* slot_pos, void* out, void* stream) {
  if (mode != ROM_COMBINE_SUM && mode != ROM_COMBINE_GATE && mode != ROM_COMBINE_GATE_DENSE)
    return ROM_ERR_INVALID_ARG;
  if (dtype != ROM_F32 && dtype != ROM_BF16) return ROM_ERR_INVALID_ARG;
  if (T < 0 || k < 1 || k > rom::kMaxTopK || N <= 0) return ROM_ERR_INVALID_ARG;
  if (N % 4 != 0) return ROM_ERR_UNSUPPORTED;
  if (T == 0) return ROM_OK;
  if (!in || !out) return ROM_ERR_INVALID_ARG;
  if (!aligned16(in) || !aligned16(out)) return ROM_ERR_UNSUPPORTED;
  return rom::to_status(rom::launch_combine(mode, dtype == ROM_BF16,
                                            static_cast<const float*>(in), T, k, N, slot_pos,
                                            out, static_cast<cudaStream_t>(stream)));
}

int rom_get_status(void* stream, int32_t* host_status) {
  if (!host_status) return ROM_ERR_INVALID_ARG;
  int* st = rom::status_ptr();
  if (!st) return ROM_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return ROM_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, st, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return ROM_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpy(st, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
    return ROM_ERR_CUDA;
  *host_status = v;
  return ROM_OK;
}

int rom_bwd_gather(const void* dout, int64_t T, int k, int N, const int32_t* sorted_slot,
                   const float* topk_w, void* rdo_sorted, void* stream) {
  if (T < 0 || k < 1 || k > rom::kMaxTopK || N <= 0) return ROM_ERR_INVALID_ARG;
  if (N % 8 != 0 || T * k >= (int64_t(1) << 31)) return ROM_ERR_UNSUPPORTED;
  if (T == 0) return ROM_OK;
  if (!dout || !sorted_slot || !topk_w || !rdo_sorted) return ROM_ERR_INVALID_ARG;
  if (!aligned16(dout) || !aligned16(rdo_sorted)) return ROM_ERR_UNSUPPORTED;
  return rom::to_status(rom::launch_scale_gather(dout, T * k, k, N, sorted_slot, topk_w,
                                                 rdo_sorted, static_cast<cudaStream_t>(stream)));
}

int rom_bwd_dgrad_out(const void* rdo_sorted, int64_t R, int Dm, const void* w_out, int De, int E,
                      int k, const int32_t* offsets, const int32_t* sorted_slot,
                      const void* h_sorted, float* g_slots, float* dr_part, void* stream) {
  if (R < 0 || Dm <= 0 || De <= 0 || E < 1 || E > rom::kMaxExperts || k < 1 || k > E ||
      k > rom::kMaxTopK || R % k != 0)
    return ROM_ERR_INVALID_ARG;
  if (Dm % 64 != 0 || De % 256 != 0 || R >= (int64_t(1) << 31)) return ROM_ERR_UNSUPPORTED;
  if (!offsets || !w_out || !sorted_slot || !h_sorted || !g_slots || !dr_part ||
      (R > 0 && !rdo_sorted))
    return ROM_ERR_INVALID_ARG;
  if (!aligned16(rdo_sorted) || !aligned16(w_out) || !aligned16(h_sorted) || !aligned16(g_slots))
    return ROM_ERR_UNSUPPORTED;
  int* st = rom::status_ptr();
  if (!st) return ROM_ERR_CUDA;
  return rom::to_status(rom::launch_bwd_dgrad_out(rdo_sorted, R, Dm, w_out, De, E, k, offsets,
                                                  sorted_slot, h_sorted, g_slots, dr_part, st,
                                                  static_cast<cudaStream_t>(stream)));
}

int rom_bwd_gate(const float* uz, const float* g_slots, int64_t T, int k, int De,
                 const int32_t* slot_pos, void* dhz_sorted, void* stream) {
  if (T < 0 || k < 1 || k > rom::kMaxTopK || De <= 0) return ROM_ERR_INVALID_ARG;
  if (De % 4 != 0) return ROM_ERR_UNSUPPORTED;
  if (T == 0) return ROM_OK;
  if (!uz || !g_slots || !slot_pos || !dhz_sorted) return ROM_ERR_INVALID_ARG;
  if (!aligned16(uz) || !aligned16(g_slots) || !aligned16(dhz_sorted)) return ROM_ERR_UNSUPPORTED;
  return rom::to_status(rom::launch_gate_bwd(uz, g_slots, T, k, De, slot_pos, dhz_sorted,
                                             static_cast<cudaStream_t>(stream)));
}

int rom_bwd_dgrad_in(const void* dhz_sorted, int64_t R, int De, const void* w_in,
                     const void* w_g, int Dm, int E, int k, const int32_t* offsets,
                     const int32_t* sorted_slot, float* dx_slots, void* stream) {
  if (R < 0 || Dm <= 0 || De <= 0 || E < 1 || E > rom::kMaxExperts || k < 1 || k > E ||
      k > rom::kMaxTopK || R % k != 0)
    return ROM_ERR_INVALID_ARG;
  if (De % 64 != 0 || Dm % 256 != 0 || R >= (int64_t(1) << 31)) return ROM_ERR_UNSUPPORTED;
  if (!offsets || !w_in || !w_g || !sorted_slot || !dx_slots || (R > 0 && !dhz_sorted))
    return ROM_ERR_INVALID_ARG;
  if (!aligned16(dhz_sorted) || !aligned16(w_in) || !aligned16(w_g) || !aligned16(dx_slots))
    return ROM_ERR_UNSUPPORTED;
  int* st = rom::status_ptr();
  if (!st) return ROM_ERR_CUDA;
  return rom::to_status(rom::launch_bwd_dgrad_in(dhz_sorted, R, De, w_in, w_g, Dm, E, k, offsets,
                                                 sorted_slot, dx_slots, st,
                                                 static_cast<cudaStream_t>(stream)));
}

int rom_route_bwd(int64_t T, int k, int E, int Dm, int renorm, const int32_t* topk_idx,
                  const float* topk_w, const float* probs, const float* dr_part, int n_parts,
                  const float* dx_slots, const float* w_r, float* dlogits, void* dx,
                  void* stream) {
  if (T < 0 || E < 1 || E > rom::kMaxExperts || k < 1 || k > E || k > rom::kMaxTopK || Dm <= 0 ||
      n_parts < 1 || (renorm != 0 && renorm != 1))
    return ROM_ERR_INVALID_ARG;
  if (Dm % 4 != 0) return ROM_ERR_UNSUPPORTED;
  if (T == 0) return ROM_OK;
  if (!topk_idx || !topk_w || !dr_part || !dx_slots || !w_r || !dx || (renorm == 0 && !probs))
    return ROM_ERR_INVALID_ARG;
  if (!aligned16(dx_slots) || !aligned16(w_r) || (reinterpret_cast<uintptr_t>(dx) & 7u))
    return ROM_ERR_UNSUPPORTED;
  return rom::to_status(rom::launch_route_bwd(T, k, E, Dm, topk_idx, topk_w,
                                              renorm ? nullptr : probs, dr_part, n_parts,
                                              dx_slots, w_r, dlogits, dx,
                                              static_cast<cudaStream_t>(stream)));
}

int rom_route_probs(const void* x, int dtype, int64_t T, int Dm, const float* w_r,
                    const float* bias, int E, float* probs, void* stream) {
  if (dtype != ROM_F32 && dtype != ROM_BF16) return ROM_ERR_INVALID_ARG;
  if (T < 0 || Dm <= 0 || E < 1 || E > rom::kMaxExperts) return ROM_ERR_INVALID_ARG;
  if (T > 0 && (!x || !w_r || !probs)) return ROM_ERR_INVALID_ARG;
  return rom::to_status(rom::launch_route_probs(x, dtype == ROM_BF16, T, Dm, w_r, bias, E, probs,
                                                static_cast<cudaStream_t>(stream)));
}

int rom_bwd_wgrad(const void* a_sorted, int M, const void* b_sorted, int N, int64_t R, int E,
                  const int32_t* offsets, int m_split, float* out0, float* out1, void* stream) {
  if (M <= 0 || N <= 0 || R < 0 || E < 1 || E > rom::kMaxExperts || m_split < 0 || m_split > M)
    return ROM_ERR_INVALID_ARG;
  if (M % 128 != 0 || N % 256 != 0 || m_split % 128 != 0 || R >= (int64_t(1) << 31))
    return ROM_ERR_UNSUPPORTED;
  if (!a_sorted || !b_sorted || !offsets || !out0 || (m_split < M && !out1))
    return ROM_ERR_INVALID_ARG;
  if (!aligned16(a_sorted) || !aligned16(b_sorted) || !aligned16(out0) ||
      (out1 && !aligned16(out1)))
    return ROM_ERR_UNSUPPORTED;
  int* st = rom::status_ptr();
  if (!st) return ROM_ERR_CUDA;
  return rom::to_status(rom::launch_bwd_wgrad(a_sorted, M, b_sorted, N, R, E, offsets, m_split,
                                              out0, out1, st, static_cast<cudaStream_t>(stream)));
}

int rom_route_wgrad(const void* x, int dtype, int64_t T, int Dm, int E, const float* dlogits,
                    float* dw_r, float* dbias, void* stream) {
  if (dtype != ROM_F32 && dtype != ROM_BF16) return ROM_ERR_INVALID_ARG;
  if (T < 0 || Dm <= 0 || E < 1 || E > rom::kMaxExperts) return ROM_ERR_INVALID_ARG;
  if (!dw_r || (T > 0 && (!x || !dlogits))) return ROM_ERR_INVALID_ARG;
  return rom::to_status(rom::launch_route_wgrad(x, dtype == ROM_BF16, T, Dm, E, dlogits, dw_r,
                                                dbias, static_cast<cudaStream_t>(stream)));
}

int rom_debug_wait_timeout(uint64_t limit_ns, void* stream) {
  if (limit_ns < 1000ull || limit_ns > 10000000000ull) return ROM_ERR_INVALID_ARG;
  int* st = rom::status_ptr();
  if (!st) return ROM_ERR_CUDA;
  rom::debug_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns, st);
  return rom::to_status(cudaGetLastError());
}

}  // extern "C"
