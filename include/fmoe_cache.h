/*
 * fmoe_cache.h -- C ABI of libfmoe.so, part 3: experts resident in host memory, streamed
 * on demand into an expert cache in HBM.
 *
 * "What is Flash-MoE" (a2a-mcp.org), section 1 (SSD expert streaming, "trust the OS"), and
 * the "Flash-MoE" wiki summary (jeongsk), key technique 1 and the per-layer pipeline: the
 * 209 GB of experts stay on SSD; per layer only the K = 4 selected experts (about 6.75 MB
 * each) are read, with parallel pread, after the router has chosen them, and the OS page
 * cache serves most of them (71 % hit rate).  Here the backing store is pinned host memory
 * and the cache is a set of record slots in HBM that the GPU manages itself, with no host
 * round trip: a lookup marks the selected experts used, copies each missing one from host
 * memory into the least recently used slot, and gives back slot indices; the expert kernels
 * then read the slots.
 *
 * Conventions as in fmoe.h: stream-ordered, arguments checked on the host before anything
 * is enqueued, the library allocates nothing.
 */
#ifndef FMOE_CACHE_H
#define FMOE_CACHE_H

#include "fmoe.h"

#ifdef __cplusplus
extern "C" {
#endif

/* An expert cache.
 * host_base:   E records at host_stride in pinned host memory (cudaHostAlloc, or
 *              cudaHostRegister with the mapped flag) that the device reads directly under
 *              unified addressing; 16-byte aligned, host_stride a multiple of 16.
 * slots:       num_slots records at slot_stride in device memory (16-byte aligned).
 * record_bytes: bytes copied per miss (a multiple of 16, <= both strides): the record size
 *              of fmoe_bank_layout.
 * num_experts: E; num_slots: C >= the K of every lookup.
 * state:       device memory of fmoe_expert_cache_state_size(E, C) bytes, 16-byte aligned,
 *              set up by fmoe_expert_cache_reset before first use: which expert each slot
 *              holds, its last use, the hit and miss counts and an error word.
 * Replacement: least recently used slot among those the current lookup has not used; an
 * empty slot first (lowest index among equals).  Every lookup is one time step. */
typedef struct {
  const void* host_base;
  int64_t host_stride;
  void* slots;
  int64_t slot_stride;
  int64_t record_bytes;
  int32_t num_experts;
  int32_t num_slots;
  void* state;
} fmoe_expert_cache;

size_t fmoe_expert_cache_state_size(int num_experts, int num_slots);

/* Empties the cache and clears its counters (enqueued on `stream`). */
fmoe_status fmoe_expert_cache_reset(const fmoe_expert_cache* cache, fmoe_stream_t stream);

/* One lookup of K experts: idx: device int32 [K] (each in [0, E); repeats allowed);
 * slot: device int32 [K], the slot that holds idx[k] once the call's work is done (NULL:
 * not written).  Missing experts are copied from host memory by the GPU (one kernel reads
 * the host records and writes the slots).  An index outside [0, E) is replaced by 0 and
 * recorded; fmoe_expert_cache_stats then returns FMOE_ERR_INVALID_ARG.
 * Requirements: 1 <= K <= min(C, 32). */
fmoe_status fmoe_expert_cache_fetch(const fmoe_expert_cache* cache, const int32_t* idx, int K, int32_t* slot,
                                    fmoe_stream_t stream);

/* Synchronises `stream`, then reads the counters since the last reset: lookups that found
 * the expert resident (hits), that copied it (misses), and bytes copied from host memory
 * (any of the three outputs may be NULL).  Returns FMOE_ERR_INVALID_ARG (and clears the
 * record) if a lookup met an index outside the bank. */
fmoe_status fmoe_expert_cache_stats(const fmoe_expert_cache* cache, int64_t* hits, int64_t* misses,
                                    int64_t* bytes, fmoe_stream_t stream);

/* The MoE block of fmoe_moe_layer with the routed experts behind an expert cache, token by
 * token: RMSNorm, router and top-K (the router's last CTA selects), one lookup of the K
 * selected experts, then gate/up + SwiGLU and down + combine reading the cache's slots.
 * layer->routed gives the record format (bits, group, hidden, inter, offsets) and E; its
 * base and stride are not used (the experts are in cache->host_base).  The shared expert,
 * router and gate stay in device memory as in fmoe_moe_layer.
 * topk_idx, topk_w: optional device outputs [T][K] (expert ids and weights).
 * ws: fmoe_moe_layer_workspace_size(layer, 1) bytes, initialised by fmoe_workspace_init.
 * Requirements: those of fmoe_moe_layer for one token, E == cache->num_experts,
 * K <= cache->num_slots, record_bytes covering the record of fmoe_bank_layout. */
fmoe_status fmoe_moe_layer_cached(const fmoe_layer* layer, const fmoe_expert_cache* cache, const float* h, int T,
                                  float* out, int32_t* topk_idx, float* topk_w, void* ws, size_t ws_bytes,
                                  fmoe_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* FMOE_CACHE_H */
