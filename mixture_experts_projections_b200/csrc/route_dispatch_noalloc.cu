// rom_route_dispatch_noalloc: routing + dispatch for callers that cannot
// allocate device memory.
//
// rom_route() and rom_dispatch() pass the router's per-chunk expert
// histograms through a caller-allocated workspace. Some callers cannot
// allocate at all: code running inside a memory pool that is already
// carved up, a plugin of a host framework that hands over only its own
// buffers, or a process whose allocator must not be touched. For them this
// entry point keeps that scratch in a fixed array in the library's own device
// memory (a file-scope __device__ array, present on every GPU that loads the
// library until the process exits), and runs the same two kernels.
//
// Limits and sharing: the array holds kNoAllocScratchWords int32 entries;
// a call needs ceil(T / 128) * E of them and is refused with
// ROM_ERR_WORKSPACE when that is more. Every call on a device uses the same
// array, so calls that may overlap on the GPU (different streams without
// ordering) race on it; calls on one stream are ordered and safe. The router
// overwrites every entry that the dispatch then reads, so nothing has to be
// cleared between calls even though the array keeps the previous contents;
// should the router give up on a bounded wait, the dispatch checks the
// entries against the expert indices and reports ROM_ERR_ROUTING instead of
// using stale ones.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/rom.h"
#include "rom_internal.cuh"

namespace rom {
namespace {

constexpr int64_t kNoAllocScratchWords = ROM_NOALLOC_SCRATCH_WORDS;

static __device__ __align__(256) int32_t g_noalloc_scratch[kNoAllocScratchWords];

// Device address of g_noalloc_scratch on the current device. In host code
// the array's name is only a host-side stand-in, so the address is looked up
// once per device (with that device current) and cached.
int32_t* noalloc_scratch() {
  static std::mutex mu;
  static int32_t* addr[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
    addr[dev] = static_cast<int32_t*>(p);
  }
  return addr[dev];
}

}  // namespace
}  // namespace rom

extern "C" int rom_route_dispatch_noalloc(const void* x, int dtype, int64_t T, int Dm,
                                          const float* w_r, const float* bias, int E, int k,
                                          int renorm, int32_t* topk_idx, float* topk_w,
                                          int32_t* counts, int32_t* offsets,
                                          int32_t* sorted_slot, int32_t* slot_pos,
                                          void* x_sorted, void* stream) {
  if (dtype != ROM_F32 && dtype != ROM_BF16) return ROM_ERR_INVALID_ARG;
  if (T < 0 || Dm <= 0 || E < 1 || E > rom::kMaxExperts || k < 1 || k > E ||
      k > rom::kMaxTopK || (renorm != 0 && renorm != 1))
    return ROM_ERR_INVALID_ARG;
  if (T * k >= (int64_t(1) << 31)) return ROM_ERR_UNSUPPORTED;
  const bool bf16 = dtype == ROM_BF16;
  if (Dm % (bf16 ? 8 : 4) != 0) return ROM_ERR_UNSUPPORTED;
  if (!offsets) return ROM_ERR_INVALID_ARG;
  if (T > 0) {
    if (!x || !w_r || !topk_idx || !topk_w || !sorted_slot || !slot_pos || !x_sorted)
      return ROM_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(x) & 15u) || (reinterpret_cast<uintptr_t>(x_sorted) & 15u))
      return ROM_ERR_UNSUPPORTED;
  }
  if (rom::num_chunks(T) * E > rom::kNoAllocScratchWords) return ROM_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t* scratch = rom::noalloc_scratch();
  if (!scratch) return ROM_ERR_CUDA;
  // The device status word: a bounded wait of the router that runs out, or
  // routing the dispatch finds inconsistent, is recorded there for
  // rom_get_status(), as for rom_route() and rom_dispatch().
  int* st = rom::status_ptr();
  if (!st) return ROM_ERR_CUDA;
  if (counts && cudaMemsetAsync(counts, 0, sizeof(int32_t) * E, s) != cudaSuccess)
    return ROM_ERR_CUDA;
  if (T > 0) {
    const cudaError_t e = rom::launch_router(x, bf16, T, Dm, w_r, bias, E, k, renorm, topk_idx,
                                             topk_w, counts, scratch, st, s);
    if (e != cudaSuccess) return e == cudaErrorInvalidValue ? ROM_ERR_UNSUPPORTED : ROM_ERR_CUDA;
  }
  const cudaError_t e = rom::launch_dispatch(x, bf16, T, Dm, E, k, topk_idx, scratch, offsets,
                                             sorted_slot, slot_pos, x_sorted, st, s);
  if (e != cudaSuccess) return e == cudaErrorInvalidValue ? ROM_ERR_UNSUPPORTED : ROM_ERR_CUDA;
  return ROM_OK;
}
