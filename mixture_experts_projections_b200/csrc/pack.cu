// One-time copy of expert weights [E][N][K] (bf16) into the tile-major
// layout [E][N/128][K/64][128][64] read by the dense small-batch projection:
// each 128 x 64 weight tile (128 output rows, 64 contraction elements) becomes
// one contiguous 16 KB block. A storage layout of the same weights, not a
// step of the method. One thread per 16-byte piece of the output (coalesced
// stores; each 128-byte input row segment is read by 8 consecutive threads).
#include <cuda_bf16.h>

#include <algorithm>

#include "rom_internal.cuh"

namespace rom {
namespace {

__global__ void __launch_bounds__(256)
    pack_expert_weights_kernel(const uint4* __restrict__ w, int64_t pieces, int N, int K,
                               uint4* __restrict__ out) {
  const int kb_n = K / 64, nt_n = N / 128;
  for (int64_t q = blockIdx.x * 256ll + threadIdx.x; q < pieces;
       q += static_cast<int64_t>(gridDim.x) * 256) {
    // output piece q: 8 elements at (e, nt, kb, r, c) with c a multiple of 8
    const int c8 = static_cast<int>(q & 7);
    const int r = static_cast<int>((q >> 3) & 127);
    const int64_t blk = q >> 10;  // (e, nt, kb) block of 1024 pieces
    const int kb = static_cast<int>(blk % kb_n);
    const int64_t et = blk / kb_n;
    const int nt = static_cast<int>(et % nt_n);
    const int64_t e = et / nt_n;
    const int64_t src = ((e * N + static_cast<int64_t>(nt) * 128 + r) * K + kb * 64) / 8 + c8;
    out[q] = __ldg(w + src);
  }
}

}  // namespace

cudaError_t launch_pack_expert_weights(const void* w, int E, int N, int K, void* w_tiled,
                                       cudaStream_t stream) {
  const int64_t pieces = static_cast<int64_t>(E) * N * K / 8;
  if (pieces == 0) return cudaSuccess;
  const int64_t blocks = std::min<int64_t>((pieces + 255) / 256, int64_t(device_sm_count()) * 32);
  pack_expert_weights_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
      static_cast<const uint4*>(w), pieces, N, K, static_cast<uint4*>(w_tiled));
  return cudaGetLastError();
}

}  // namespace rom
