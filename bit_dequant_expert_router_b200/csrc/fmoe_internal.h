// fmoe_internal.h -- host-side declarations shared by the C-ABI layer and the kernel files.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "fmoe_device.cuh"

namespace fmoe {

// Expert cache (k_cache.cu): host-resident records, HBM slots, tables in `state`.
constexpr int kCacheMaxK = 32;
struct CacheHeader {          // first 64 bytes of the state
  unsigned int clock;         // lookups so far (a slot's last use is the lookup that used it)
  int err;                    // kDevBadIndex after an index outside the bank (fetch entry point)
  int n_copy;                 // records the current lookup copies
  int pad0;
  unsigned long long hits, misses, bytes;
  unsigned long long pad1[3];
};
struct CacheParams {
  const uint8_t* host;        // E records at host_stride (pinned host memory, mapped)
  long long host_stride;
  uint8_t* slots;             // C records at slot_stride (device)
  long long slot_stride;
  long long rec;              // bytes per copied record (multiple of 16)
  int E, C;
  uint8_t* state;             // header, copy list [2][kCacheMaxK], slots of the last lookup [kCacheMaxK],
                              // slot_of [E], expert_of [C], last_use [C]
};
__host__ __device__ inline size_t cache_up16(size_t v) { return (v + 15) / 16 * 16; }
__host__ __device__ inline int* cache_copy_expert(const CacheParams& c) {
  return reinterpret_cast<int*>(c.state + sizeof(CacheHeader));
}
__host__ __device__ inline int* cache_copy_slot(const CacheParams& c) { return cache_copy_expert(c) + kCacheMaxK; }
__host__ __device__ inline int* cache_slot_out(const CacheParams& c) { return cache_copy_slot(c) + kCacheMaxK; }
__host__ __device__ inline int* cache_slot_of(const CacheParams& c) { return cache_slot_out(c) + kCacheMaxK; }
__host__ __device__ inline int* cache_expert_of(const CacheParams& c) {
  return reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(cache_slot_of(c)) + cache_up16((size_t)c.E * 4));
}
__host__ __device__ inline unsigned int* cache_last_use(const CacheParams& c) {
  return reinterpret_cast<unsigned int*>(reinterpret_cast<uint8_t*>(cache_expert_of(c)) + cache_up16((size_t)c.C * 4));
}

// One lookup of K experts by one warp (every lane calls it; expert k is lane k's `mine`).
// Marks them used, picks a victim slot for each missing one (least recently used among the
// slots this lookup has not used; empty slots first, lowest index among equals), updates
// the tables, writes the copy list and slot_out[k] (if not NULL).  An id outside [0, E)
// is replaced by 0 and recorded in *err.  Lane 0 writes the tables; __syncwarp orders them.
__device__ inline void cache_lookup_warp(const CacheParams& c, int mine, int K, int32_t* slot_out, int* err) {
  const int lane = threadIdx.x & 31;
  CacheHeader* hd = reinterpret_cast<CacheHeader*>(c.state);
  int* slot_of = cache_slot_of(c);
  int* expert_of = cache_expert_of(c);
  unsigned int* last_use = cache_last_use(c);
  const unsigned int now = hd->clock + 1u;
  int n = 0;
  unsigned long long hits = 0, misses = 0;
  for (int k = 0; k < K; ++k) {  // uniform over the warp
    int e = __shfl_sync(0xffffffffu, mine, k);
    if (e < 0 || e >= c.E) {
      if (lane == 0) atomicExch(err, 7);  // kDevBadIndex
      e = 0;
    }
    int s = __ldcg(slot_of + e);
    if (s < 0) {
      unsigned long long best = ~0ull;
      for (int q = lane; q < c.C; q += 32) {
        const unsigned int t = __ldcg(last_use + q);
        if (t != now) best = min(best, ((unsigned long long)t << 32) | (unsigned int)q);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) best = min(best, __shfl_xor_sync(0xffffffffu, best, o));
      s = (int)(best & 0xffffffffull);  // exists: at most K - 1 < C slots carry `now` so far
      if (lane == 0) {
        const int old = expert_of[s];
        if (old >= 0) slot_of[old] = -1;
        expert_of[s] = e;
        slot_of[e] = s;
        cache_copy_expert(c)[n] = e;
        cache_copy_slot(c)[n] = s;
      }
      ++n;
      ++misses;
    } else {
      ++hits;
    }
    if (lane == 0) {
      last_use[s] = now;
      if (slot_out) slot_out[k] = s;
    }
    __syncwarp();
  }
  if (lane == 0) {
    hd->clock = now;
    hd->n_copy = n;
    hd->hits += hits;
    hd->misses += misses;
    hd->bytes += misses * (unsigned long long)c.rec;
  }
}

// Router GEMV: logits[t][0..E) = Wr x_t (+ bias), logits[t][E] = wsg . x_t; one grid row per token.
struct RouterParams {
  const float* h;             // [T][H] input (normalised in-kernel when norm != 0)
  const float* gamma;         // [H] or NULL (unit)
  float eps;
  int norm;                   // 1: x = RMSNorm(h); 0: x = h
  const uint16_t* w_router;   // bf16 [E][H]
  const float* bias;          // [E] or NULL
  const uint16_t* w_sgate;    // bf16 [H] or NULL (no shared-gate row)
  int T, H, E;
  int rows_per_cta;
  uint8_t* xq_limbs;          // per-token activation digits, or NULL
  float2* xq_cs;
  long long xq_limb_stride;   // bytes per token
  long long xq_cs_stride;     // float2 per token
  float* logits;              // [T][E+1]
  int top_k;                  // > 0: the last CTA of each token selects the top-K (route_* outputs)
  int32_t* route_idx;         // [T][K] selected experts
  float* route_w;             // [T][K+1]: renormalised weights, slot K = shared-gate sigma
  int32_t* idx_out;           // optional user copies [T][K]
  float* w_out;
  unsigned int* tickets;      // [T], zero between calls
  unsigned int* route_ready;  // or NULL: cleared once the predecessor is complete (see ExpertParams)
  unsigned int* clear;        // or NULL: nclear counters that CTA 0 zeroes once the predecessor is
  int nclear;                 // complete (the gate/up kernel's group counters, so that a call never
                              // depends on the previous one having finished cleanly)
  CacheParams cache;           // cache.state != NULL: the selecting CTA also runs the expert-cache
                              // lookup of the selected experts (slots to cache_slot_out(cache))
  int* err;
};

// Standalone selection from logits (the router_topk entry point).
struct TopkParams {
  const float* logits;        // [T][E+1]
  int T, E, K;
  int32_t* idx;               // [T][K]
  float* w;                   // [T][K]
  float* probs;               // [T][E] or NULL
};

struct ExpertParams {
  BankRef routed;
  BankRef shared;
  const float* logits;        // [E+1] router logits (+ shared-gate logit): each kernel selects the
                              // experts itself; NULL: the routing below
  const int32_t* route_idx;   // [K] selected experts or NULL (fixed_expert)
  const float* route_w;       // [K+1] weights, slot K = shared-gate sigma; NULL: weight 1
  const float* sigma_logit;   // or NULL; when set, the down kernel takes the routed weights from route_w
                              // [K] and sigma = sigmoid(*sigma_logit) (the routing given by the caller)
  int32_t* idx_out;           // with logits: the caller's copy of the routing [K], [K] (gate/up CTA 0), or NULL
  float* w_out;
  int32_t* rt_idx;            // with logits: gate/up CTA 0 writes the routing here for the down kernel
  float* rt_w;                // [K+1], slot K = shared-gate sigma
  int E;
  int fixed_expert;
  int gsh;                    // weight groups of 64 << gsh columns (0: 64, 1: 128); x digits stay per 64
  int gu_sw;                  // gate/up split: a shared-expert unit weighs gu_sw eighths of a routed one
  int K;                      // routed slots
  int has_shared;             // slot K is the shared expert
  int H, I;
  const uint32_t* xq_limbs;   // gate/up: digits of x (chunk-major)
  const float2* xq_cs;
  float* act;                 // [K+has_shared][I]: gate/up output (SwiGLU activations)
  uint8_t* act_limbs;         // digits of act, per slot [I*bits/128 chunks][limb words] (down input)
  float2* act_cs;             // per slot [I*bits/128] chunk scalars
  unsigned int* grp_cnt;      // [K+has_shared][I/64] rows finished per group of 64 (zero between calls)
  const float* resid;         // down: residual [H] or NULL
  float* out;                 // down: [H]
  int prefetch_down;          // gate/up asks L2 for the routed experts' down matrices: 1 after the
                              // routing, 2 after the CTA's last chunk has landed, 0 never
  unsigned int* route_ready;  // or NULL.  Gate/up CTA 0 sets it (release) after writing rt_idx / rt_w;
                              // the down kernel, seeing it set (acquire), reads the routing and requests
                              // the routed rows before its dependency wait; the next router clears it
  int* err;
};

// ---- expert-grouped path for batched decode (k_grouped.cu): T tokens, each active
// expert's weights read once for all the tokens routed to it

// A work unit of the grouped expert kernels: up to kUnitToks members of one
// expert's group, whose rows in act / act_limbs / y are row0 .. row0 + n - 1.
constexpr int kUnitToks = 2;
struct alignas(16) UnitDesc {
  int e;       // routed expert, -1 = the shared expert
  int row0;    // first member row
  int n;       // members
  int pad;
  int tok[4];  // token of each member (the first kUnitToks used)
};
static_assert(kUnitToks <= 4, "UnitDesc holds at most four members");

struct GroupedParams {
  BankRef routed, shared;
  int T, E, K, H, I;
  const float* logits;        // [T][E+1] router logits (+ shared-gate logit)
  const uint8_t* xq_limbs;    // [T][3H] digits of x per token, tensor-core layout
  const float2* xq_cs;        // [T][H/64] per group {digit scale, sum of x}
  int32_t* route_idx;         // [T][K]
  float* route_w;             // [T][K+1], slot K = sigma
  int32_t* idx_out;           // caller's copies [T][K] or NULL
  float* w_out;
  int32_t* n_active;          // [2] U: active experts, W: work units
  UnitDesc* units;            // [T*K + T] work units of the expert kernels, the shared expert's first
  float* rt_part;             // [rt_split][T][E+1] the router's slice sums
  int rt_split;
  const float* rt_bias;       // [E] or NULL
  int32_t* act_expert;        // [T*K] active experts, increasing
  int32_t* act_off;           // [T*K+1] first pair of each active expert in the sorted pair list
  int32_t* pair_tok;          // [T*K] sorted pairs (expert, token, k): value t*K + k
  int32_t* pair_pos;          // [T*K] position of pair t*K + k in the sorted list
  float* act;                 // [(T*K + T)][I] SwiGLU outputs: sorted pairs, then the shared expert per token
  uint8_t* act_limbs;         // [(T*K + T)][3I], tensor-core layout
  float2* act_cs;             // [(T*K + T)][I/64]
  float* y;                   // [(T*K + T)][H] down outputs (unweighted)
  const float* h;             // [T][H] residual
  float* out;                 // [T][H]
  int* err;
};

// The batched router: x = RMSNorm(h) and its digits per token, then the router GEMM.
struct RouterBatch {
  const float* gamma;         // [H] or NULL (no norm)
  float eps;
  const uint16_t* w_router;   // bf16 [E][H]
  const uint16_t* w_sgate;    // bf16 [H]
  const float* bias;          // [E] or NULL
  float* x;                   // workspace [T][H]: x in fp32
};

// The batched router's split-K factor: the workspace holds split * T * (E+1) partial logits.
int grouped_router_split(int H, int E, int T);
// pdl: chain each launch to its predecessor by dependent launch (every grouped kernel
// waits for its predecessor at entry, then lets its successor launch).
cudaError_t launch_grouped_router(const GroupedParams& p, const RouterBatch& rb, int bits, bool pdl, cudaStream_t s);
cudaError_t launch_grouped_select(const GroupedParams& p, bool pdl, cudaStream_t s);
cudaError_t launch_grouped_gateup(const GroupedParams& p, int bits, bool pdl, cudaStream_t s);
cudaError_t launch_grouped_actq(const GroupedParams& p, int bits, bool pdl, cudaStream_t s);
cudaError_t launch_grouped_down(const GroupedParams& p, int bits, bool pdl, cudaStream_t s);
cudaError_t launch_grouped_combine(const GroupedParams& p, bool pdl, cudaStream_t s);
bool grouped_shapes_supported(int bits, int H, int I, int E, int K, int T);

// ---- single-kernel path (k_fused.cu): a sequence of T tokens x L layers, one CTA per SM

constexpr int kFusedWarps = 8;
constexpr int kFusedMaxRing = 16;        // chunk buffers
constexpr int kFusedMaxItems = 64;       // staged items per CTA and step
constexpr int kFusedMaxKS = 8;           // warps sharing one row
constexpr int kFusedMaxChunkRows = 32;   // gate/up row pairs per chunk
constexpr int kFusedMaxDnRows = 64;      // down rows per CTA
constexpr int kFusedMaxGuRows = 64;      // gate/up row pairs per CTA
constexpr int kFusedMaxRtRows = 4;       // router rows per staged item
constexpr int kFusedMaxLayers = 32;      // layers per launch
constexpr long long kFusedSmemBudget = 223232;  // dynamic shared memory, bytes (static use is about 8.5 KiB)

struct FusedLayer {                      // 64 bytes
  const uint8_t* routed;                 // routed bank: record 0
  long long stride;                      // bytes between records
  const uint8_t* shared;                 // the shared expert's record
  const uint16_t* w_router;              // bf16 [E][H]
  const float* bias;                     // [E] or NULL
  const uint16_t* w_sgate;               // bf16 [H]
  const float* gamma;                    // [H] or NULL (no RMSNorm)
  float eps;
  int pad;
};

struct FusedParams {
  FusedLayer layers[kFusedMaxLayers];
  long long off[9];                      // record offsets, common to both banks of every layer
  int L, T, H, I, E, K;
  const float* h;                        // [T][H] input of layer 0
  float* out;                            // [T][H] output of the last layer (also the stack's running state)
  int32_t* idx_out;                      // [T][K] or NULL (single-layer calls)
  float* w_out;
  // workspace: epoch-tagged exchange words {value (low 32 bits), epoch (high 32 bits)},
  // two copies each (step parity), zero before first use
  unsigned long long* xlog;              // [2][E+1] router logits (+ the shared-gate logit)
  unsigned long long* xact;              // [2][(K+1)*I] SwiGLU activations, slot-major
  unsigned long long* xh;                // [2][H] a stacked layer's output, the next layer's input
  unsigned* epoch;                       // steps run on this workspace so far
  int* err;
  int nbuf, chb, cu, rt_rows, ru, rd, dn_rows_max, dn_slot_bytes, dn_off, ring_off;
};

struct FusedPlan {
  bool ok;
  int P, nbuf, chb, cu, rt_rows, ru, rd, dn_rows_max, dn_slot_bytes, dn_off, ring_off;
  size_t smem;
};

FusedPlan plan_fused(int bits, int H, int I, int E, int K);
cudaError_t launch_fused(const FusedParams& p, const FusedPlan& pl, int bits, bool pdl, cudaStream_t s);

// ---- per-token path (k_token.cu): a router kernel and one expert kernel per token

struct TokRouterParams {
  const float* h;             // [H] the block's input
  const float* gamma;         // [H] RMSNorm weight, or NULL
  float eps;
  int norm;                   // 1: x = RMSNorm(h); 0: x = h
  const uint16_t* w_router;   // bf16 [E][H]
  const float* bias;          // [E] or NULL
  const uint16_t* w_sgate;    // bf16 [H]: row E of the router's output
  int H, E;
  int row0;                   // first output row: 0, or E (the shared-gate row alone)
  int rpc;                    // rows per CTA (set by the launcher)
  uint8_t* xq_limbs;          // digits of x for the expert kernel
  float2* xq_cs;
  float* logits;              // [E + 1]
  unsigned int* count;        // the expert kernel's arrival counter, cleared once per token
  int* err;
};

struct TokExpertParams {
  BankRef routed, shared;
  const float* logits;        // [E + 1]: the routing is the top-K of logits[0, E) unless route_idx is
                              // given; sigma = sigmoid(logits[E])
  const int32_t* route_idx;   // [K] given routing, or NULL
  const float* route_w;       // [K] given weights, or NULL (weight 1)
  int fixed_expert;           // the routing when logits and route_idx are both NULL (K = 1)
  int32_t* idx_out;           // the caller's copy of the routing [K] (CTA 0), or NULL
  float* w_out;
  int E, K, has_shared, H, I;
  const uint8_t* xq_limbs;    // digits of x
  const float2* xq_cs;
  float* act;                 // [K + has_shared][I] SwiGLU activations, exchanged between CTAs
  unsigned int* count;        // CTAs whose activations are written (cleared by the kernel before this one)
  const float* resid;         // [H] residual, or NULL
  float* out;                 // [H]
  int* err;
  // set by the launcher
  int gmax_s, gmax_r, dmax;   // units per shared / routed gate/up chunk, per down range
  int xd_bytes, sc_bytes, ring_bytes;  // shared-memory regions: digits, scales, staged codes
  int sbox_s, sbox_r, drows;  // staged scale rows: shared and routed gate/up, down (per CTA, at most)
};

struct TokPlan {
  bool ok;
  int grid, gmax_s, gmax_r, dmax, xd_bytes, sc_bytes, sbox_s, sbox_r, drows, ring_bytes, dppl;
  size_t smem;
};

TokPlan plan_token(int bits, int H, int I, int K, int has_shared);
cudaError_t launch_tok_router(TokRouterParams p, int bits, bool pdl, cudaStream_t s);
cudaError_t launch_tok_xq(const float* x, int H, int bits, uint8_t* limbs, float2* cs, unsigned int* count, bool pdl,
                          cudaStream_t s);
cudaError_t launch_tok_expert(TokExpertParams p, int bits, bool pdl, cudaStream_t s);
// Whether the two-kernel path takes these shapes and record layouts.
bool token_path_supported(int bits, int H, int I, int K, int has_shared, const BankRef& routed, const BankRef& shared);

cudaError_t launch_rmsnorm(const float* h, const float* gamma, float eps, int T, int H, float* y, cudaStream_t s);
cudaError_t launch_xq(const float* x, int H, int bits, uint8_t* limbs, float2* cs, cudaStream_t s);
cudaError_t launch_router(RouterParams p, int xq_bits, bool pdl, cudaStream_t s);
cudaError_t launch_topk(const TopkParams& p, cudaStream_t s);
cudaError_t launch_gateup(const ExpertParams& p, int bits, bool pdl, cudaStream_t s);
cudaError_t launch_down(const ExpertParams& p, int bits, bool pdl, cudaStream_t s);

int num_sms();
bool expert_shapes_supported(int bits, int H, int I, int num_slots);

// Gated DeltaNet state update, one decode step of `rows / dv` heads (k_gdn.cu).
struct GdnParams {
  float* state;               // [n][dv][dk], updated in place
  const float* q;             // [n][dk]
  const float* k;             // [n][dk]
  const float* v;             // [n][dv]
  const float* alpha;         // [n]
  const float* beta;          // [n]
  float* o;                   // [n][dv]
  int rows;                   // n * dv
  int dk, dv;
  int early;                  // 1: read the state before the dependency wait
};
// Tensor-map encoding (cuTensorMapEncodeTiled through the runtime's driver entry point).
// encode_map: one map over 8-byte elements, dims[0] elements per row, then the outer dims
// with their byte strides (rank - 1 of them), and the box; false if it cannot be encoded.
bool encode_map(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims, const cuuint64_t* strides,
                const cuuint32_t* box);

bool gdn_shape_supported(int dk);

size_t cache_state_bytes(int E, int C);
cudaError_t launch_cache_reset(const CacheParams& c, cudaStream_t s);
// One lookup: the plan kernel (tables, copy list, slot_out [K]) then the copy kernel.
cudaError_t launch_cache_lookup(const CacheParams& c, const int32_t* idx, int K, int32_t* slot_out, int* err, bool pdl,
                                cudaStream_t s);
// The copy kernel alone (after a lookup made elsewhere, e.g. by the router's selecting CTA).
cudaError_t launch_cache_copy(const CacheParams& c, bool pdl, cudaStream_t s);
cudaError_t launch_gdn_step(const GdnParams& p, bool pdl, cudaStream_t s);
bool pdl_enabled();
cudaError_t launch_wait_flag(const unsigned int* flag, unsigned int value, unsigned long long limit_ns, int* err,
                             cudaStream_t s);
cudaError_t set_smem(const void* kernel, size_t bytes);
cudaError_t set_carveout_max(const void* kernel);

// Launch with optional programmatic stream serialisation (dependent launch).
template <typename... Exp, typename... Act>
cudaError_t launch_pdl(void (*kern)(Exp...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, bool pdl,
                       Act&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = pdl ? attr : nullptr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<Act&&>(args)...);
}

}  // namespace fmoe
