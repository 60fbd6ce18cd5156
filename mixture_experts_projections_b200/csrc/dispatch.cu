// Dropless dispatch of the RoM block: a stable counting sort of the routed
// slots by expert, and the gather of the token rows into expert-contiguous
// order. ("Routing Mamba ..." chapterpal summary page, Knowl 12: no expert
// parallelism, no capacity factor, no token dropping.)
//
// One CTA per 128-token chunk (the router's chunk). From the per-chunk expert
// histograms the router left in the workspace, the CTA forms the global
// offsets (exclusive prefix of the totals) and its own base per expert (sum
// of the earlier chunks). Inside the chunk, slots are ranked per expert in
// ascending slot order: warps rank 32 consecutive slots with __match_any_sync,
// and a per-expert prefix over the 32-slot groups orders the groups. The
// result needs no atomics on the global order and is deterministic.
//
// Few chunks (small batches, decode): gridDim.y CTAs share a chunk. Each
// repeats the (cheap) ranking and copies one slice of the row's 16-byte
// columns; slice 0 writes the index outputs.
//
// The inputs are checked before they are used as indices: every histogram
// entry must lie in [0, slots of its chunk] and the entries must add up to
// R = T*k; every expert index of the chunk must lie in [0, E) and the chunk's
// own count of each expert must equal its histogram entry. When a check
// fails (a router that gave up on a bounded wait, or a workspace that does
// not belong to these indices) the kernel records ROM_ERR_ROUTING in the
// device status word and still leaves outputs that every later kernel can
// read without leaving its buffers: offsets monotone in [0, R], and
// sorted_slot and slot_pos in [0, R).
#include <cuda_bf16.h>

#include <algorithm>

#include "rom_internal.cuh"
#include "sm100_ptx.cuh"

namespace rom {
namespace {

constexpr int kDispatchThreads = 512;
constexpr int kDispatchWarps = kDispatchThreads / 32;
constexpr int kMaxGroups = kChunkTokens * kMaxTopK / 32;  // 32-slot groups per chunk

__global__ void __launch_bounds__(kDispatchThreads)
    dispatch_kernel(const uint4* __restrict__ x, int64_t T, int row_vec16, int E, int k,
                    const int32_t* __restrict__ topk_idx, const int32_t* __restrict__ chunk_hist,
                    int64_t nchunks, int32_t* __restrict__ offsets,
                    int32_t* __restrict__ sorted_slot, int32_t* __restrict__ slot_pos,
                    uint4* __restrict__ x_sorted, int* status) {
  const int slice = blockIdx.y, nslices = gridDim.y;
  __shared__ int s_tot[kMaxExperts];
  __shared__ int s_base[kMaxExperts];
  __shared__ int s_own[kMaxExperts];
  __shared__ int s_off[kMaxExperts + 1];
  __shared__ int s_gcount[kMaxGroups][kMaxExperts];
  __shared__ int s_pos[kChunkTokens * kMaxTopK];
  __shared__ int s_bad_hist, s_bad_chunk;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t c = blockIdx.x;
  const int64_t R = T * k;
  const int64_t chunk_slots = static_cast<int64_t>(kChunkTokens) * k;
  const int64_t s0 = c * chunk_slots;
  const int ns = static_cast<int>(std::min<int64_t>(chunk_slots, R - s0));
  const int ngroups = (ns + 31) / 32;
  // Launched as a programmatic dependent of the router: the kernel after
  // this one may start now; the router's outputs are read only after
  // pdl_wait().
  pdl_launch_dependents();

  for (int e = tid; e < E; e += kDispatchThreads) {
    s_tot[e] = 0;
    s_base[e] = 0;
    s_own[e] = 0;
  }
  for (int i = tid; i < ngroups * kMaxExperts; i += kDispatchThreads)
    s_gcount[i / kMaxExperts][i % kMaxExperts] = 0;
  if (tid == 0) {
    s_bad_hist = 0;
    s_bad_chunk = 0;
  }
  pdl_wait();
  __syncthreads();
  // Histogram entries outside [0, slots of their chunk] are refused; with
  // that bound no per-expert total can exceed R.
  for (int64_t i = tid; i < nchunks * E; i += kDispatchThreads) {
    const int v = chunk_hist[i];
    const int e = static_cast<int>(i % E);
    const int64_t ci = i / E;
    if (v < 0 || v > std::min<int64_t>(chunk_slots, R - ci * chunk_slots)) {
      s_bad_hist = 1;
    } else if (v) {
      atomicAdd(&s_tot[e], v);
      if (ci < c) atomicAdd(&s_base[e], v);
      if (ci == c) s_own[e] = v;
    }
  }
  __syncthreads();
  if (tid == 0) {
    int64_t run = 0;
    for (int e = 0; e < E; ++e) {
      s_off[e] = static_cast<int>(std::min<int64_t>(run, R));
      run += s_tot[e];
    }
    s_off[E] = static_cast<int>(std::min<int64_t>(run, R));
    if (run != R) s_bad_hist = 1;
  }
  __syncthreads();
  if (s_bad_hist) {
    // The histograms do not describe R slots (every CTA reads the same ones
    // and reaches this branch together): no expert gets rows, and the
    // permutation is the identity, so whatever reads it stays in bounds.
    if (c == 0 && slice == 0) {
      for (int e = tid; e <= E; e += kDispatchThreads) offsets[e] = 0;
      if (tid == 0 && status) atomicExch(status, kStatusRouting);
    }
    if (slice == 0)
      for (int ls = tid; ls < ns; ls += kDispatchThreads) {
        sorted_slot[s0 + ls] = static_cast<int32_t>(s0 + ls);
        slot_pos[s0 + ls] = static_cast<int32_t>(s0 + ls);
      }
    return;
  }
  if (c == 0 && slice == 0)
    for (int e = tid; e <= E; e += kDispatchThreads) offsets[e] = s_off[e];

  // Per-group, per-expert counts and the rank of each slot inside its group.
  // An index outside [0, E) marks the chunk as inconsistent and takes a key
  // of its own (as idle lanes do), so it never joins a valid expert's group.
  int my_rank[kMaxGroups / kDispatchWarps];
  int my_e[kMaxGroups / kDispatchWarps];
#pragma unroll
  for (int q = 0; q < kMaxGroups / kDispatchWarps; ++q) {
    const int g = warp + q * kDispatchWarps;
    my_e[q] = -1;
    my_rank[q] = 0;
    if (g < ngroups) {
      const int ls = g * 32 + lane;
      const int e = (ls < ns) ? topk_idx[s0 + ls] : -1;
      const bool ok = ls < ns && e >= 0 && e < E;
      if (ls < ns && !ok) s_bad_chunk = 1;
      const int key = ok ? e : -1 - lane;
      const unsigned same = __match_any_sync(0xffffffffu, key);
      my_rank[q] = __popc(same & ((1u << lane) - 1u));
      my_e[q] = ok ? e : -1;
      if (ok && my_rank[q] == 0) s_gcount[g][e] = __popc(same);
    }
  }
  __syncthreads();
  // Exclusive prefix over groups, per expert (in place); the chunk's count
  // of each expert must equal its histogram entry.
  for (int e = tid; e < E; e += kDispatchThreads) {
    int run = 0;
    for (int g = 0; g < ngroups; ++g) {
      const int v = s_gcount[g][e];
      s_gcount[g][e] = run;
      run += v;
    }
    if (run != s_own[e]) s_bad_chunk = 1;
  }
  __syncthreads();
  if (s_bad_chunk) {
    // This chunk's indices disagree with its histogram row. The positions the
    // row assigns to the chunk (its share of each expert's range) are filled
    // with the chunk's first slot and zero rows, and its slots point at the
    // identity position: every value stays in [0, R).
    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
    const int v0 = static_cast<int>(static_cast<int64_t>(row_vec16) * slice / nslices);
    const int v1 = static_cast<int>(static_cast<int64_t>(row_vec16) * (slice + 1) / nslices);
    if (tid == 0 && status) atomicExch(status, kStatusRouting);
    for (int e = 0; e < E; ++e) {
      const int p0 = s_off[e] + s_base[e];
      for (int i = warp; i < s_own[e]; i += kDispatchWarps) {
        if (slice == 0 && lane == 0) sorted_slot[p0 + i] = static_cast<int32_t>(s0);
        uint4* drow = x_sorted + static_cast<int64_t>(p0 + i) * row_vec16;
        for (int v = v0 + lane; v < v1; v += 32) drow[v] = zero;
      }
    }
    if (slice == 0)
      for (int ls = tid; ls < ns; ls += kDispatchThreads)
        slot_pos[s0 + ls] = static_cast<int32_t>(s0 + ls);
    return;
  }
#pragma unroll
  for (int q = 0; q < kMaxGroups / kDispatchWarps; ++q) {
    const int g = warp + q * kDispatchWarps;
    if (g < ngroups && my_e[q] >= 0) {
      const int ls = g * 32 + lane;
      const int e = my_e[q];
      // in [s_off[e] + s_base[e], + s_own[e]): this chunk's share of expert e
      const int pos = s_off[e] + s_base[e] + s_gcount[g][e] + my_rank[q];
      if (slice == 0) {
        sorted_slot[pos] = static_cast<int32_t>(s0 + ls);
        slot_pos[s0 + ls] = pos;
      }
      s_pos[ls] = pos;
    }
  }
  __syncthreads();
  // Gather this CTA's column slice [v0, v1) of every slot row: one warp per
  // row, 16-byte vectors, 4 in flight per lane. The rows are read for the
  // last time here (the router kept them in L2): their lines go first.
  const uint64_t pol = l2_policy_evict_first();
  const int v0 = static_cast<int>(static_cast<int64_t>(row_vec16) * slice / nslices);
  const int v1 = static_cast<int>(static_cast<int64_t>(row_vec16) * (slice + 1) / nslices);
  for (int ls = warp; ls < ns; ls += kDispatchWarps) {
    const int64_t src = (s0 + ls) / k;
    const uint4* srow = x + src * row_vec16;
    uint4* drow = x_sorted + static_cast<int64_t>(s_pos[ls]) * row_vec16;
    int i = v0 + lane;
    for (; i + 96 < v1; i += 128) {
      const uint4 a = ld_nc_hint(srow + i, pol), b = ld_nc_hint(srow + i + 32, pol),
                  cc = ld_nc_hint(srow + i + 64, pol), d = ld_nc_hint(srow + i + 96, pol);
      drow[i] = a;
      drow[i + 32] = b;
      drow[i + 64] = cc;
      drow[i + 96] = d;
    }
    for (; i < v1; i += 32) drow[i] = ld_nc_hint(srow + i, pol);
  }
}

}  // namespace

cudaError_t launch_dispatch(const void* x, bool bf16, int64_t T, int Dm, int E, int k,
                            const int32_t* topk_idx, const int32_t* chunk_hist,
                            int32_t* offsets, int32_t* sorted_slot, int32_t* slot_pos,
                            void* x_sorted, int* status, cudaStream_t stream) {
  const int64_t nchunks = num_chunks(T);
  if (nchunks == 0) {
    // No tokens: offsets are all zero.
    return cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (E + 1), stream);
  }
  const int row_bytes = Dm * (bf16 ? 2 : 4);
  // Slices per chunk: enough CTAs to cover the SMs twice, at most 16, and
  // at least 32 vectors (512 bytes) of each row per slice.
  const int64_t want = (2 * static_cast<int64_t>(device_sm_count())) / nchunks;
  const int nslices = static_cast<int>(
      std::max<int64_t>(1, std::min<int64_t>({want, 16, (row_bytes / 16) / 32})));
  // Programmatic dependent launch: the CTAs may start (and be resident)
  // while the router finishes; they wait for it before reading its outputs.
  // The projection after it is a programmatic dependent too and needs most
  // of an SM's shared memory; an SM whose shared-memory carve-out was set
  // small for this kernel would take none of its CTAs until this kernel's
  // CTAs left, so these CTAs ask for the largest carve-out.
  const cudaError_t ce = cudaFuncSetAttribute(
      dispatch_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
  if (ce != cudaSuccess) return ce;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(nchunks), static_cast<unsigned>(nslices), 1);
  cfg.blockDim = dim3(kDispatchThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, dispatch_kernel, static_cast<const uint4*>(x), T,
                            row_bytes / 16, E, k, topk_idx, chunk_hist, nchunks, offsets,
                            sorted_slot, slot_pos, static_cast<uint4*>(x_sorted), status);
}

}  // namespace rom
