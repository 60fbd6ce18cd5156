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

int device_sm_count();  // cached per device

cudaError_t launch_router(const void* x, bool bf16, int64_t T, int Dm, const float* w_r,
                          const float* bias, int E, int k, int renorm, int32_t* topk_idx,
                          float* topk_w, int32_t* counts, int32_t* chunk_hist, int* status,
                          cudaStream_t stream);

cudaError_t launch_dispatch(const void* x, bool bf16, int64_t T, int Dm, int E, int k,
                            const int32_t* topk_idx, const int32_t* chunk_hist,
                            int32_t* offsets, int32_t* sorted_slot, int32_t* slot_pos,
                            void* x_sorted, cudaStream_t stream);

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

// float32 SIMT grouped GEMM (same semantics as the tensor-core one).
cudaError_t launch_simt_grouped_gemm(int mode, const float* a_sorted, int64_t R, int K,
                                     const float* w0, const float* w1, int N, int E, int k,
                                     const int32_t* offsets, const int32_t* sorted_slot,
                                     const float* topk_w, float* out, cudaStream_t stream);

cudaError_t launch_combine(int mode, bool bf16, const float* in, int64_t T, int k, int N,
                           const int32_t* slot_pos, void* out, cudaStream_t stream);

cudaError_t launch_debug_wait(uint64_t limit_ns, int* status, cudaStream_t stream);

}  // namespace rom
