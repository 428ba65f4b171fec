// k_cache.cu -- expert cache in HBM in front of experts resident in host memory.
//
// "What is Flash-MoE" (a2a-mcp.org), section 1, and the "Flash-MoE" wiki summary
// (jeongsk), key technique 1: only the K selected experts of a layer are read from the
// slow store, after routing.  Here the store is pinned host memory read by the GPU over
// the host link, and the cache is managed on the GPU:
//   cache_plan_kernel  (one warp; cache_lookup_warp) marks the selected experts used, picks
//                      a victim slot for each missing one (least recently used among slots
//                      this lookup has not used; empty slots first), updates the tables and
//                      writes the copy list and the slot of every selected expert (inside a
//                      layer call the router's selecting warp does this lookup itself);
//   cache_copy_kernel  (every SM) copies the listed records, host -> slot, with 16-byte
//                      loads from host memory (four in flight per thread) and stores to HBM.
// Both run under dependent launch after the router, and the expert kernels after them.
#include <cstdint>

#include "fmoe_internal.h"

namespace fmoe {
namespace {

constexpr int kCopyThreads = 256;
constexpr int kCopyUnroll = 4;

__global__ void cache_reset_kernel(const CacheParams c) {
  CacheHeader* hd = reinterpret_cast<CacheHeader*>(c.state);
  int* slot_of = cache_slot_of(c);
  int* expert_of = cache_expert_of(c);
  unsigned int* last_use = cache_last_use(c);
  const int i0 = blockIdx.x * blockDim.x + threadIdx.x, n = gridDim.x * blockDim.x;
  for (int e = i0; e < c.E; e += n) slot_of[e] = -1;
  for (int s = i0; s < c.C; s += n) {
    expert_of[s] = -1;
    last_use[s] = 0u;
  }
  if (i0 == 0) {
    hd->clock = 0u;
    hd->err = 0;
    hd->n_copy = 0;
    hd->hits = 0ull;
    hd->misses = 0ull;
    hd->bytes = 0ull;
  }
}

// One warp.  idx: [K] selected experts; slot_out: [K] or NULL.
__global__ void __launch_bounds__(32) cache_plan_kernel(const CacheParams c, const int32_t* idx, int K,
                                                        int32_t* slot_out, int* err) {
  pdl_wait();  // the routing is complete
  pdl_trigger();
  const int lane = threadIdx.x;
  const int mine = lane < K ? __ldcg(idx + lane) : 0;
  cache_lookup_warp(c, mine, K, slot_out, err);
}

// Copies the plan's records: CTA b takes the same contiguous share of every record.
__global__ void __launch_bounds__(kCopyThreads) cache_copy_kernel(const CacheParams c) {
  pdl_wait();  // the plan is complete
  pdl_trigger();
  const CacheHeader* hd = reinterpret_cast<const CacheHeader*>(c.state);
  const int n = min(hd->n_copy, kCacheMaxK);
  const long long r16 = c.rec / 16;
  const long long per = (r16 + gridDim.x - 1) / gridDim.x;
  const long long b0 = (long long)blockIdx.x * per;
  const long long b1 = b0 + per < r16 ? b0 + per : r16;
  for (int j = 0; j < n; ++j) {
    if (!FMOE_IN_BOUNDS(n <= kCacheMaxK && cache_copy_expert(c)[j] >= 0 && cache_copy_expert(c)[j] < c.E &&
                            cache_copy_slot(c)[j] >= 0 && cache_copy_slot(c)[j] < c.C,
                        &reinterpret_cast<CacheHeader*>(c.state)->err))
      continue;
    const uint4* src = reinterpret_cast<const uint4*>(c.host + (long long)cache_copy_expert(c)[j] * c.host_stride);
    uint4* dst = reinterpret_cast<uint4*>(c.slots + (long long)cache_copy_slot(c)[j] * c.slot_stride);
    for (long long i = b0 + threadIdx.x; i < b1; i += kCopyThreads * kCopyUnroll) {
      uint4 v[kCopyUnroll];
#pragma unroll
      for (int u = 0; u < kCopyUnroll; ++u)
        if (i + u * kCopyThreads < b1) v[u] = __ldg(src + i + u * kCopyThreads);
#pragma unroll
      for (int u = 0; u < kCopyUnroll; ++u)
        if (i + u * kCopyThreads < b1) __stcg(dst + i + u * kCopyThreads, v[u]);
    }
  }
}

}  // namespace

size_t cache_state_bytes(int E, int C) {
  auto up16 = [](size_t v) { return (v + 15) / 16 * 16; };
  return sizeof(CacheHeader) + 3 * kCacheMaxK * sizeof(int) + up16((size_t)E * 4) + 2 * up16((size_t)C * 4);
}

cudaError_t launch_cache_reset(const CacheParams& c, cudaStream_t s) {
  const int n = c.E > c.C ? c.E : c.C;
  cache_reset_kernel<<<(n + 255) / 256, 256, 0, s>>>(c);
  return cudaGetLastError();
}

cudaError_t launch_cache_lookup(const CacheParams& c, const int32_t* idx, int K, int32_t* slot_out, int* err, bool pdl,
                                cudaStream_t s) {
  cudaError_t e = launch_pdl(cache_plan_kernel, dim3(1), dim3(32), 0, s, pdl, c, idx, K, slot_out, err);
  if (e != cudaSuccess) return e;
  return launch_cache_copy(c, pdl, s);
}

cudaError_t launch_cache_copy(const CacheParams& c, bool pdl, cudaStream_t s) {
  return launch_pdl(cache_copy_kernel, dim3(4 * num_sms()), dim3(kCopyThreads), 0, s, pdl, c);
}

}  // namespace fmoe
