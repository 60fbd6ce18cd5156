// Internal declarations shared by the translation units of librom.so.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace rom {

// Router / dispatch geometry: tokens are processed in chunks of this many
// tokens; the router writes one expert histogram per chunk into the
// workspace and the dispatch kernel runs one CTA per chunk.
constexpr int kChunkTokens = 128;
constexpr int kMaxExperts = 64;
constexpr int kMaxTopK = 8;

inline int64_t num_chunks(int64_t T) { return (T + kChunkTokens - 1) / kChunkTokens; }

// Device status codes written by kernels (the same values as rom_status).
constexpr int kStatusRouting = 6;  // == ROM_ERR_ROUTING

// Programmatic dependent launch. A kernel launched with
// cudaLaunchAttributeProgrammaticStreamSerialization may start while the
// kernel before it on the stream still runs, once every CTA of that kernel
// has called pdl_launch_dependents() (or exited). It must call pdl_wait()
// -- which returns when the kernels before it have completed and their
// writes are visible -- before it reads anything they wrote, and every CTA
// calls it before exiting, so that its own completion still implies theirs.
// Without the launch attribute both are no-ops.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

int device_sm_count();  // cached per device

// Device address of this device's status word (nullptr on failure), looked
// up once per device with that device current.
int* status_ptr();

cudaError_t launch_router(const void* x, bool bf16, int64_t T, int Dm, const float* w_r,
                          const float* bias, int E, int k, int renorm, int32_t* topk_idx,
                          float* topk_w, int32_t* counts, int32_t* chunk_hist, int* status,
                          cudaStream_t stream);

// One CTA per token (small batches); cudaErrorNotSupported when T exceeds
// kSmallRouterMaxTokens, E is not 4, 8 or 16, or the data is not 16-byte
// aligned.
constexpr int64_t kSmallRouterMaxTokens = 1024;
cudaError_t launch_router_small(const void* x, bool bf16, int64_t T, int Dm, const float* w_r,
                                const float* bias, int E, int k, int renorm, int32_t* topk_idx,
                                float* topk_w, int32_t* counts, int32_t* chunk_hist,
                                cudaStream_t stream);

// Returns cudaErrorNotSupported when W_r does not fit in shared memory.
cudaError_t launch_router_stream(const void* x, int64_t T, int Dm, const float* w_r,
                                 const float* bias, int E, int k, int renorm, int32_t* topk_idx,
                                 float* topk_w, int32_t* counts, int32_t* chunk_hist, int* status,
                                 cudaStream_t stream);

// Records kStatusRouting in *status (when not null) if topk_idx or
// chunk_hist are out of range or inconsistent; the outputs then stay in
// range (offsets monotone in [0, T*k], sorted_slot and slot_pos in [0, T*k)).
cudaError_t launch_dispatch(const void* x, bool bf16, int64_t T, int Dm, int E, int k,
                            const int32_t* topk_idx, const int32_t* chunk_hist,
                            int32_t* offsets, int32_t* sorted_slot, int32_t* slot_pos,
                            void* x_sorted, int* status, cudaStream_t stream);

// Epilogue variants of the grouped GEMMs.
enum EpiMode : int {
  kEpiGateH = 0,      // h = u * SiLU(z) -> dtype rows in sorted order
  kEpiGateSlots = 1,  // u, z -> float32 [2][R][N] in slot order
  kEpiScaleToken = 2, // r * acc -> dtype [T][N] in token order (k == 1)
  kEpiScaleSlots = 3  // r * acc -> float32 [R][N] in slot order
};

// bf16 tensor-core grouped GEMM (tcgen05 + TMA). Returns cudaErrorInvalidValue
// when the shape is outside what the kernel supports.
cudaError_t launch_tc_grouped_gemm(int mode, const void* a_sorted, int64_t R, int K,
                                   const void* w0, const void* w1, int N, int E, int k,
                                   const int32_t* offsets, const int32_t* sorted_slot,
                                   const float* topk_w, void* out, int* status,
                                   cudaStream_t stream);

// Small-batch (T <= 64) routed projection without a dispatch: x in token
// order, the router's topk_idx / topk_w read only by the epilogue.
cudaError_t launch_tc_dense_small(int mode, const void* x, int64_t T, int K, const void* w, int N,
                                  int E, int k, const int32_t* topk_idx, const float* topk_w,
                                  void* out, bool w_tiled, int* status, cudaStream_t stream);
// [E][N][K] bf16 -> the tile-major [E][N/128][K/64][128][64] (pack.cu)
cudaError_t launch_pack_expert_weights(const void* w, int E, int N, int K, void* w_tiled,
                                       cudaStream_t stream);

// float32 SIMT grouped GEMM (same semantics as the tensor-core one).
cudaError_t launch_simt_grouped_gemm(int mode, const float* a_sorted, int64_t R, int K,
                                     const float* w0, const float* w1, int N, int E, int k,
                                     const int32_t* offsets, const int32_t* sorted_slot,
                                     const float* topk_w, float* out, cudaStream_t stream);

cudaError_t launch_combine(int mode, bool bf16, const float* in, int64_t T, int k, int N,
                           const int32_t* slot_pos, void* out, cudaStream_t stream);

cudaError_t launch_debug_wait(uint64_t limit_ns, int* status, cudaStream_t stream);

// ---- backward (grouped_gemm_bwd.cu, backward_simt.cu)
enum BwdMode : int { kBwdDgradOut = 0, kBwdDgradIn = 1, kBwdWgrad = 2 };

cudaError_t launch_bwd_dgrad_out(const void* rdo_sorted, int64_t R, int Dm, const void* w_out,
                                 int De, int E, int k, const int32_t* offsets,
                                 const int32_t* sorted_slot, const void* h_sorted, float* g_slots,
                                 float* dr_part, int* status, cudaStream_t stream);
cudaError_t launch_bwd_dgrad_in(const void* dhz_sorted, int64_t R, int De, const void* w_in,
                                const void* w_g, int Dm, int E, int k, const int32_t* offsets,
                                const int32_t* sorted_slot, float* dx_slots, int* status,
                                cudaStream_t stream);
cudaError_t launch_bwd_wgrad(const void* a_sorted, int M, const void* b_sorted, int N, int64_t R,
                             int E, const int32_t* offsets, int m_split, float* out0, float* out1,
                             int* status, cudaStream_t stream);
cudaError_t launch_scale_gather(const void* dout, int64_t R, int k, int N,
                                const int32_t* sorted_slot, const float* topk_w, void* dst,
                                cudaStream_t stream);
cudaError_t launch_gate_bwd(const float* uz, const float* gp, int64_t T, int k, int De,
                            const int32_t* slot_pos, void* dhz, cudaStream_t stream);
cudaError_t launch_route_wgrad(const void* x, bool bf16, int64_t T, int Dm, int E,
                               const float* dlogits, float* dw_r, float* dbias,
                               cudaStream_t stream);
cudaError_t launch_route_probs(const void* x, bool bf16, int64_t T, int Dm, const float* w_r,
                               const float* bias, int E, float* probs, cudaStream_t stream);
cudaError_t launch_route_bwd(int64_t T, int k, int E, int Dm, const int32_t* topk_idx,
                             const float* topk_w, const float* probs, const float* dr_part,
                             int n_parts, const float* dx_slots, const float* w_r, float* dlogits,
                             void* dx, cudaStream_t stream);

}  // namespace rom
