// fmoe_device.cuh -- device-side building blocks shared by the sm_100a kernels:
// mbarrier + bulk-copy (TMA engine) staging, the packed-code dot product and
// the fixed-point activation format it consumes.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace fmoe {

constexpr int kGroup = 64;        // codes per scale/bias group
constexpr int kChunkBytes = 16;   // one 128-bit load of codes
constexpr int kDevTimeout = 6;    // workspace error word: a bounded wait gave up (FMOE_ERR_DEVICE_TIMEOUT)
constexpr int kDevBadIndex = 7;   // workspace error word: an expert index outside the bank
constexpr int kDevBounds = 8;     // workspace error word: a bounds check of a debug build failed

// Device-side bounds checks of the debug build (compiled with FMOE_DEBUG_BOUNDS): where
// an index, a row range or a copy would leave its buffer, FMOE_IN_BOUNDS records
// kDevBounds in the error word and yields false, and the caller skips the access (a
// skipped copy then also ends its barrier wait by the time limit).  In the normal build
// it is the constant true and costs nothing.
#ifdef FMOE_DEBUG_BOUNDS
#define FMOE_IN_BOUNDS(cond, err) ((cond) ? true : (atomicExch((err), kDevBounds), false))
#else
#define FMOE_IN_BOUNDS(cond, err) true
#endif
constexpr unsigned long long kWaitNs = 2000000000ull;  // bound on any device-side wait (2 s)

// Control words at the start of every workspace.
struct WsControl {
  unsigned int tickets[992];   // last-CTA tickets, one per token
  unsigned int epoch;          // single-kernel path: steps run on this workspace (its own 128-byte line)
  unsigned int route_ready;    // three-kernel path: 1 once the gate/up kernel has published this token's routing
  unsigned int pad0[30];
  int err;                     // nonzero once a bounded wait gave up
  int pad[31];
  unsigned int tok_count;      // per-token path: expert-kernel CTAs whose activations are written
  unsigned int pad1[31];       // (its own 128-byte line; cleared by the first kernel of each token)
};
constexpr int kMaxTokenCtas = 256;

// ------------------------------------------------------------------------------------------ small helpers

__device__ __forceinline__ uint32_t smem_addr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ unsigned int ld_acquire_gpu(const unsigned int* p) {
  unsigned int v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ unsigned int ld_relaxed_gpu(const unsigned int* p) {
  unsigned int v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void fence_acq_rel_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }

__device__ __forceinline__ void st_release_gpu(unsigned int* p, unsigned int v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ float bf16_to_f32(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

// Barrier `id` (1..15) over the first `n` threads of the block (n a multiple of 32).
__device__ __forceinline__ void named_bar_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// ------------------------------------------------------------------------------------------ dependent launch
//
// Kernels are launched with programmatic stream serialisation: a kernel may
// start while its predecessor is still running, do work that reads only
// constant data (weights), then pdl_wait() for the predecessor's results.
// pdl_trigger() lets the successor start its own constant-data prologue.
// Without the launch attribute both are no-ops.

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ------------------------------------------------------------------------------------------ mbarrier + bulk copy

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_fence_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

// Plain arrival (no transaction bytes).
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits for phase `parity` of the barrier, at most kWaitNs; on timeout records
// the error in the workspace and returns false.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity, int* err) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  for (;;) {
#pragma unroll 1
    for (int i = 0; i < 64; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (global_ns() - t0 > kWaitNs) {
      atomicExch(err, kDevTimeout);
      return false;
    }
  }
}

// Waits until *flag == value (acquire, gpu scope), at most limit_ns; on timeout
// records the error and returns false.
__device__ __forceinline__ bool flag_wait_bounded(const unsigned int* flag, unsigned int value, unsigned long long limit_ns,
                                                  int* err) {
  if (ld_acquire_gpu(flag) == value) return true;
  const unsigned long long t0 = global_ns();
  for (;;) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (ld_acquire_gpu(flag) == value) return true;
    if (global_ns() - t0 > limit_ns) {
      atomicExch(err, kDevTimeout);
      return false;
    }
  }
}

// One thread waits until *count >= target (relaxed reads with a short sleep between
// them, then one acquire fence), at most kWaitNs; on timeout records the error and
// returns false.  One thread per CTA polls one word, so waiting CTAs do not flood L2.
__device__ __forceinline__ bool count_wait_bounded(const unsigned int* count, unsigned int target, int* err) {
  unsigned long long t0 = 0;
  for (int round = 0;; ++round) {
    if (ld_relaxed_gpu(count) >= target) {
      fence_acq_rel_gpu();
      return true;
    }
    if (round == 0) t0 = global_ns();
    else if (global_ns() - t0 > kWaitNs) {
      atomicExch(err, kDevTimeout);
      return false;
    }
    __nanosleep(32);
  }
}

// Asks L1 for the 128-byte line holding p.
__device__ __forceinline__ void prefetch_l1(const void* p) { asm volatile("prefetch.global.L1 [%0];" ::"l"(p)); }

__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// Orders this thread's earlier generic-proxy accesses to shared memory before
// later async-proxy (bulk copy) writes to the same bytes.
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// Asks L2 to fetch [src, src + bytes) ahead of use (16-byte aligned, bytes % 16 == 0).
__device__ __forceinline__ void prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// Bulk copy global -> this CTA's shared memory, completing `bytes` of
// transaction count on barrier `bar`.  dst, src 16-byte aligned; bytes % 16 == 0.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar, uint64_t pol) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
          dst),
      "l"(src), "r"(bytes), "r"(bar), "l"(pol)
      : "memory");
}

// 16-byte asynchronous copy global -> shared on the load path (not the TMA engine,
// whose fixed cost per copy makes small copies slow); dst, src 16-byte aligned.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

// The barrier receives one arrival once every cp.async this thread issued so far has
// landed (the arrival is counted in the barrier's expected count).
__device__ __forceinline__ void cp_async_arrive(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

// Copies `bytes` (a multiple of 16) from src to shared dst with cp_async16, the pieces
// spread over the 32 lanes of the calling warp.
__device__ __forceinline__ void cp_async_warp(uint32_t dst, const uint8_t* src, uint32_t bytes, int lane) {
  for (uint32_t o = 16u * lane; o < bytes; o += 512u) cp_async16(dst + o, src + o);
}

// ------------------------------------------------------------------------------------------ activation format
//
// The dot product sum_c code_c * x_c over a group of 64 codes runs on integer
// dp4a units.  x is held per group of 64 as a fixed-point value:
//   x_c ~= cscale * X_c,  X_c = rint(x_c * 2^(22-e)),  2^(e-1) <= max|x| < 2^e,
// X_c = d0 * 2^16 + d1 * 2^8 + d2 with signed byte digits (|d0| <= 64).
// The digits are stored as 32-bit packs lined up with the way a code word is
// split into bytes:
//   8-bit: word w is one pack itself (codes 0,1,2,3)
//   4-bit: word w -> lo = w & 0x0F0F0F0F (codes 0,2,4,6), hi = (w >> 4) & ... (1,3,5,7)
//   2-bit: word w -> pack m = (w >> 2m) & 0x03030303 (codes m, m+4, m+8, m+12)
// One group is 48 words: chunk by chunk (a chunk is 16 bytes of codes: four per
// group at 8-bit, two at 4-bit, one at 2-bit), and within a chunk [limb 0..2][word
// 0..3][pack].  Across a vector of NG groups the 16-byte pieces are interleaved, piece
// i of group g at uint4 index i*NG + g, so that lanes reading consecutive groups hit
// distinct shared-memory banks.  Per 32 elements (4- and 8-bit; per group at 2-bit)
// there is a float2 {cscale, sum of x over the 32}, in element order.

template <int BITS>
struct Fmt {
  static constexpr int kCodesPerWord = 32 / BITS;          // 4, 8 or 16
  static constexpr int kCodesPerChunk = 4 * kCodesPerWord;  // 16, 32 or 64
  static constexpr int kPacksPerWord = 8 / BITS;           // 1, 2 or 4
  static constexpr int kLimbWords = 3 * 4 * kPacksPerWord; // 12, 24 or 48 uint32 per chunk
  static constexpr int kCsPerGroup = BITS == 2 ? 1 : 2;    // {cscale, sum x} pairs per group of 64
};

constexpr int kGroupWords = 48;  // digit words of one group of 64

// Quantises one group of 64 values held two per lane (lane l: elements 2l, 2l+1)
// into the format above.  `limb_bytes` addresses the vector's digits (NG
// groups), `cs` its per-chunk scalars; g is the group index.  Whole warp participates.
template <int BITS>
__device__ __forceinline__ void xq_quantize_group(float v0, float v1, int g, int NG, uint8_t* limb_bytes,
                                                  float2* cs) {
  const int lane = threadIdx.x & 31;
  const float m = warp_max(fmaxf(fabsf(v0), fabsf(v1)));
  int e = 0;
  if (m > 0.0f) {
    const int ef = (int)((__float_as_uint(m) >> 23) & 0xFFu);
    e = ef == 0 ? -125 : ef - 126;  // m < 2^e
  }
  e = e < -100 ? -100 : (e > 100 ? 100 : e);
  const float inv = __uint_as_float((uint32_t)(127 + 22 - e) << 23);  // 2^(22-e)
  const float csc = __uint_as_float((uint32_t)(127 + e - 22) << 23);  // 2^(e-22)
  constexpr int CPC = Fmt<BITS>::kCodesPerChunk;
  constexpr int CPW = Fmt<BITS>::kCodesPerWord;
  constexpr int PPW = Fmt<BITS>::kPacksPerWord;
  constexpr int LW = Fmt<BITS>::kLimbWords;
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const float v = k ? v1 : v0;
    const int i = 2 * lane + k;  // element within the group
    const int X = __float2int_rn(v * inv);
    const int d2 = ((X + 128) & 255) - 128;
    const int X1 = (X - d2) >> 8;
    const int d1 = ((X1 + 128) & 255) - 128;
    const int d0 = (X1 - d1) >> 8;
    const int ch = i / CPC, ii = i % CPC;
    const int wi = ii / CPW, j = ii % CPW;
    const int pack = j % PPW, byte = j / PPW;
    const int d[3] = {d0, d1, d2};
#pragma unroll
    for (int L = 0; L < 3; ++L) {
      const int w = ch * LW + (L * 4 + wi) * PPW + pack;  // word within the group
      limb_bytes[(((w >> 2) * NG + g) * 4 + (w & 3)) * 4 + byte] = (uint8_t)(int8_t)d[L];
    }
  }
  float s = v0 + v1;
  if (BITS != 2) {  // two halves of 32 per group: half-warp sums
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if ((lane & 15) == 0) cs[2 * g + (lane >> 4)] = make_float2(csc, s);
  } else {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) cs[g] = make_float2(csc, s);
  }
}

// Same format, one block of 16 consecutive elements per lane: block `part`
// (0..3) of group g, the four blocks of a group on lanes 4k..4k+3 of the warp.
// Every lane of the warp calls it (shuffles); lanes with active == false take
// part in the reductions with zeros and store nothing.  Bytes written are those
// of xq_quantize_group; the chunk sums may differ in rounding order.
template <int BITS>
__device__ __forceinline__ void xq_quantize_block16(const float (&v)[16], int g, int part, int NG, uint8_t* limb_bytes,
                                                   float2* cs, bool active) {
  float m = 0.0f;
#pragma unroll
  for (int e = 0; e < 16; ++e) m = fmaxf(m, fabsf(v[e]));
  m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
  m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
  int ex = 0;
  if (m > 0.0f) {
    const int ef = (int)((__float_as_uint(m) >> 23) & 0xFFu);
    ex = ef == 0 ? -125 : ef - 126;  // m < 2^ex
  }
  ex = ex < -100 ? -100 : (ex > 100 ? 100 : ex);
  const float inv = __uint_as_float((uint32_t)(127 + 22 - ex) << 23);
  const float csc = __uint_as_float((uint32_t)(127 + ex - 22) << 23);
  uint32_t d[3][16];
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const int X = __float2int_rn(v[e] * inv);
    const int d2 = ((X + 128) & 255) - 128;
    const int X1 = (X - d2) >> 8;
    const int d1 = ((X1 + 128) & 255) - 128;
    const int d0 = (X1 - d1) >> 8;
    d[0][e] = (uint32_t)d0 & 0xFFu;
    d[1][e] = (uint32_t)d1 & 0xFFu;
    d[2][e] = (uint32_t)d2 & 0xFFu;
  }
  if (active) {
    uint4* dst = reinterpret_cast<uint4*>(limb_bytes);
#pragma unroll
    for (int L = 0; L < 3; ++L) {
      uint32_t w[4];
#pragma unroll
      for (int wd = 0; wd < 4; ++wd) {
        // element of byte k of word wd (see the word/byte formula of xq_quantize_group)
        uint32_t acc = 0;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int e = BITS == 8 ? 4 * wd + k : BITS == 4 ? 8 * (wd >> 1) + (wd & 1) + 2 * k : 4 * k + wd;
          acc |= d[L][e] << (8 * k);
        }
        w[wd] = acc;
      }
      const int piece = BITS == 8 ? 3 * part + L : BITS == 4 ? 6 * (part >> 1) + 2 * L + (part & 1) : 4 * L + part;
      dst[piece * NG + g] = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
  float sx = 0.0f;
#pragma unroll
  for (int e = 0; e < 16; ++e) sx += v[e];
  sx += __shfl_xor_sync(0xffffffffu, sx, 1);
  if (BITS != 2) {
    if (active && (part & 1) == 0) cs[2 * g + (part >> 1)] = make_float2(csc, sx);
  } else {
    sx += __shfl_xor_sync(0xffffffffu, sx, 2);
    if (active && part == 0) cs[g] = make_float2(csc, sx);
  }
}

// Integer dot product of one group of 64 codes (4-bit: two chunks q0, q1;
// 2-bit: q0 only) with the group's digits L (chunk-major, as stored), returned
// as a float S with sum_c code_c * X_c == S up to one rounding.
template <int BITS>
__device__ __forceinline__ float group_dot(const uint4 q0, const uint4 q1, const uint32_t (&L)[48]) {
  int a0 = 0, a1 = 0, a2 = 0;
  constexpr int PPW = Fmt<BITS>::kPacksPerWord;
  constexpr int NCH = BITS == 4 ? 2 : 1;
  constexpr int LWC = Fmt<BITS>::kLimbWords;  // words of one chunk
#pragma unroll
  for (int ch = 0; ch < NCH; ++ch) {
    const uint4 q = ch ? q1 : q0;
    const uint32_t w4[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int wi = 0; wi < 4; ++wi) {
      const uint32_t w = w4[wi];
#pragma unroll
      for (int pk = 0; pk < PPW; ++pk) {
        const uint32_t c = BITS == 4 ? ((w >> (4 * pk)) & 0x0F0F0F0Fu) : ((w >> (2 * pk)) & 0x03030303u);
        a0 = __dp4a((int)c, (int)L[ch * LWC + (0 * 4 + wi) * PPW + pk], a0);
        a1 = __dp4a((int)c, (int)L[ch * LWC + (1 * 4 + wi) * PPW + pk], a1);
        a2 = __dp4a((int)c, (int)L[ch * LWC + (2 * 4 + wi) * PPW + pk], a2);
      }
    }
  }
  const int A = a0 * 256 + a1;  // |A| < 2^24: exact in fp32
  return fmaf((float)A, 256.0f, (float)a2);
}

// dp4a with unsigned bytes in a (codes up to 255) and signed bytes in b (digits).
__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// group_dot for 8-bit codes: four chunks q[0..3] (64 bytes, one code per byte).  The
// limb sums reach 2^21, so they are combined in 64-bit integers and rounded once.
__device__ __forceinline__ float group_dot8(const uint4 (&q)[4], const uint32_t (&L)[48]) {
  int a0 = 0, a1 = 0, a2 = 0;
#pragma unroll
  for (int ch = 0; ch < 4; ++ch) {
    const uint32_t w4[4] = {q[ch].x, q[ch].y, q[ch].z, q[ch].w};
#pragma unroll
    for (int wi = 0; wi < 4; ++wi) {
      a0 = dp4a_us(w4[wi], L[ch * 12 + wi], a0);
      a1 = dp4a_us(w4[wi], L[ch * 12 + 4 + wi], a1);
      a2 = dp4a_us(w4[wi], L[ch * 12 + 8 + wi], a2);
    }
  }
  const long long A = (long long)a0 * 65536 + (long long)a1 * 256 + a2;
  return (float)A;
}

__device__ __forceinline__ void load_group_codes8(const uint8_t* row, int g, uint4 (&q)[4]) {
#pragma unroll
  for (int c = 0; c < 4; ++c) q[c] = *reinterpret_cast<const uint4*>(row + g * 64 + 16 * c);
}

// Loads group g's 48 digit words from a vector of NG groups (interleaved pieces).
__device__ __forceinline__ void load_group_limbs(const uint32_t* src, int g, int NG, uint32_t (&L)[48]) {
#pragma unroll
  for (int i = 0; i < 12; ++i) {
    const uint4 v = reinterpret_cast<const uint4*>(src)[i * NG + g];
    L[4 * i] = v.x;
    L[4 * i + 1] = v.y;
    L[4 * i + 2] = v.z;
    L[4 * i + 3] = v.w;
  }
}

// load_group_limbs from global memory (through L2: the digits are written by the previous kernel).
__device__ __forceinline__ void load_group_limbs_global(const uint32_t* src, int g, int NG, uint32_t (&L)[48]) {
#pragma unroll
  for (int i = 0; i < 12; ++i) {
    const uint4 v = __ldcg(reinterpret_cast<const uint4*>(src) + i * NG + g);
    L[4 * i] = v.x;
    L[4 * i + 1] = v.y;
    L[4 * i + 2] = v.z;
    L[4 * i + 3] = v.w;
  }
}

// Order-preserving key of (logit, index): larger value first, then lower index.
__device__ __forceinline__ unsigned long long topk_key(float v, int e) {
  uint32_t u = __float_as_uint(v);
  u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return ((unsigned long long)u << 32) | (uint32_t)(0xFFFFFFFFu - (uint32_t)e);
}

__device__ __forceinline__ float topk_key_value(unsigned long long k) {
  uint32_t u = (uint32_t)(k >> 32);
  u = (u & 0x80000000u) ? (u & 0x7FFFFFFFu) : ~u;
  return __uint_as_float(u);
}

__device__ __forceinline__ int topk_key_index(unsigned long long k) { return (int)(0xFFFFFFFFu - (uint32_t)k); }

// Largest key over the warp (every lane gets it).
__device__ __forceinline__ unsigned long long warp_max_key(unsigned long long k) {
  const uint32_t hi = __reduce_max_sync(0xffffffffu, (uint32_t)(k >> 32));
  const uint32_t lo = __reduce_max_sync(0xffffffffu, (uint32_t)(k >> 32) == hi ? (uint32_t)k : 0u);
  return ((unsigned long long)hi << 32) | lo;
}

// One warp: the K largest logits[0..E) in descending order (ties to the lower
// index), their renormalised softmax weights w_k = exp(l_k - l_0) / sum_j exp(l_j - l_0),
// and, when has_gate, sigma = sigmoid(logits[E]).  Each lane keeps its logits
// e = lane + 32 i (NV of them, E <= 32 * NV) in registers with its best
// remaining key; each round takes the warp maximum and only the winning lane
// rescans.  Lane k < K returns pick k in (idx_k, w_k); every lane gets sigma.
template <int NV>
__device__ __forceinline__ void warp_topk_impl(const float* logits, int E, int K, int has_gate, int& idx_k,
                                               float& w_k, float& sigma) {
  const int lane = threadIdx.x & 31;
  unsigned long long key[NV];
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int e = lane + 32 * i;
    key[i] = e < E ? topk_key(__ldcg(logits + e), e) : 0ull;
  }
  const float zg = has_gate ? __ldcg(logits + E) : 0.0f;
  unsigned long long best = 0ull;
#pragma unroll
  for (int i = 0; i < NV; ++i) best = key[i] > best ? key[i] : best;
  float top = 0.0f, mine_v = 0.0f;
  idx_k = 0;
  for (int k = 0; k < K; ++k) {
    const unsigned long long w = warp_max_key(best);
    int e = topk_key_index(w);
    const float v = topk_key_value(w);
    if (e < 0 || e >= E) e = 0;  // only with non-finite logits
    if (k == 0) top = v;
    if (lane == k) {
      idx_k = e;
      mine_v = v;
    }
    if (best == w) {  // the winning lane drops the pick and rescans its own logits
      best = 0ull;
#pragma unroll
      for (int i = 0; i < NV; ++i) {
        key[i] = key[i] == w ? 0ull : key[i];
        best = key[i] > best ? key[i] : best;
      }
    }
  }
  const float ek = lane < K ? expf(mine_v - top) : 0.0f;
  w_k = ek / warp_sum(ek);
  sigma = has_gate ? 1.0f / (1.0f + expf(-zg)) : 0.0f;
}

// Any E: the logits stay in memory and every round rescans them.
__device__ __forceinline__ void warp_topk_mem(const float* logits, int E, int K, int has_gate, int& idx_k, float& w_k,
                                              float& sigma) {
  const int lane = threadIdx.x & 31;
  unsigned long long prev = ~0ull;
  float top = 0.0f, mine_v = 0.0f;
  idx_k = 0;
  for (int k = 0; k < K; ++k) {
    unsigned long long best = 0ull;
    for (int e = lane; e < E; e += 32) {
      const unsigned long long x = topk_key(__ldcg(logits + e), e);
      best = (x < prev && x > best) ? x : best;
    }
    const unsigned long long w = warp_max_key(best);
    int e = topk_key_index(w);
    const float v = topk_key_value(w);
    if (e < 0 || e >= E) e = 0;
    if (k == 0) top = v;
    if (lane == k) {
      idx_k = e;
      mine_v = v;
    }
    prev = w;
  }
  const float ek = lane < K ? expf(mine_v - top) : 0.0f;
  w_k = ek / warp_sum(ek);
  sigma = has_gate ? 1.0f / (1.0f + expf(-__ldcg(logits + E))) : 0.0f;
}

__device__ __forceinline__ void warp_topk(const float* logits, int E, int K, int has_gate, int& idx_k, float& w_k,
                                          float& sigma) {
  if (E <= 256)
    warp_topk_impl<8>(logits, E, K, has_gate, idx_k, w_k, sigma);
  else if (E <= 512)
    warp_topk_impl<16>(logits, E, K, has_gate, idx_k, w_k, sigma);
  else if (E <= 1024)
    warp_topk_impl<32>(logits, E, K, has_gate, idx_k, w_k, sigma);
  else
    warp_topk_mem(logits, E, K, has_gate, idx_k, w_k, sigma);
}

// Lane geometry over rows of NG groups of 64 codes: LPR lanes per row, RPP rows
// side by side in a warp, GPL groups per lane.
template <int NG>
struct Geo {
  static constexpr int kLanesPerRow = NG < 32 ? NG : 32;
  static constexpr int kRowsPerPass = 32 / kLanesPerRow;
  static constexpr int kGroupsPerLane = NG / kLanesPerRow;
};

// One group's code words from a staged row (4-bit: 32 bytes, 2-bit: 16 bytes).
template <int BITS>
__device__ __forceinline__ void load_group_codes(const uint8_t* row, int g, uint4& q0, uint4& q1) {
  constexpr int GB = kGroup * BITS / 8;
  q0 = *reinterpret_cast<const uint4*>(row + g * GB);
  q1 = BITS == 4 ? *reinterpret_cast<const uint4*>(row + g * GB + 16) : q0;
}

// Chunk scalars of group g: {power-of-two scale of the digits, sum of x over the group}.
template <int BITS>
__device__ __forceinline__ float2 group_scalars(const float2* cs, int g) {
  if (BITS != 2) {
    const float2 a = cs[2 * g], b = cs[2 * g + 1];
    return make_float2(a.x, a.y + b.y);
  }
  return cs[g];
}

template <int BITS>
__device__ __forceinline__ float2 group_scalars_global(const float2* cs, int g) {
  if (BITS != 2) {
    const float2 a = __ldcg(cs + 2 * g), b = __ldcg(cs + 2 * g + 1);
    return make_float2(a.x, a.y + b.y);
  }
  return __ldcg(cs + g);
}

// Block-wide top-K of logits [E] (E <= 8 * 64) with 256 threads, in two stages.
// Stage 1 (every warp w): the K largest keys of slice w of ceil(E/8) logits into
// cand[w*K + k].  Stage 2 (warp 0, after a block barrier): the K largest of the
// 8K candidates, the renormalised weights w_k = exp(l_k - l_0) / sum_j exp(l_j - l_0)
// into idx[0..K), w[0..K), and w[K] = sigmoid(logits[E]) when has_gate.  Keys
// order by value, then by lower index (topk_key): the result is that of one sort.
__device__ __forceinline__ void block_topk_stage1(const float* logits, int E, int K, unsigned long long* cand) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int ES = (E + 7) / 8;
  const int e0 = warp * ES + lane, e1 = e0 + 32;
  unsigned long long k0 = (lane < ES && e0 < E) ? topk_key(__ldcg(logits + e0), e0) : 0ull;
  unsigned long long k1 = (lane + 32 < ES && e1 < E) ? topk_key(__ldcg(logits + e1), e1) : 0ull;
#pragma unroll 1
  for (int k = 0; k < K; ++k) {
    const unsigned long long m = warp_max_key(k0 > k1 ? k0 : k1);
    if (lane == 0) cand[warp * K + k] = m;
    k0 = k0 == m ? 0ull : k0;
    k1 = k1 == m ? 0ull : k1;
  }
}

__device__ __forceinline__ void block_topk_stage2(float zg, int E, int K, int has_gate,
                                                  const unsigned long long* cand, int* idx, float* w) {
  const int lane = threadIdx.x & 31;
  float top = 0.0f, mine = 0.0f;
  int mi = 0;
  auto take = [&](int k, unsigned long long m) {
    int e = m ? topk_key_index(m) : 0;
    const float v = topk_key_value(m);
    if (e < 0 || e >= E) e = 0;  // only with non-finite logits
    if (k == 0) top = v;
    if (lane == k) {
      mi = e;
      mine = v;
    }
  };
  if (8 * K <= 32) {  // at most one candidate per lane
    unsigned long long key = lane < 8 * K ? cand[lane] : 0ull;
#pragma unroll 1
    for (int k = 0; k < K; ++k) {
      const unsigned long long m = warp_max_key(key);
      key = key == m ? 0ull : key;
      take(k, m);
    }
  } else {
    unsigned long long key[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) key[i] = lane + 32 * i < 8 * K ? cand[lane + 32 * i] : 0ull;
#pragma unroll 1
    for (int k = 0; k < K; ++k) {
      unsigned long long best = 0ull;
#pragma unroll
      for (int i = 0; i < 8; ++i) best = key[i] > best ? key[i] : best;
      const unsigned long long m = warp_max_key(best);
#pragma unroll
      for (int i = 0; i < 8; ++i) key[i] = key[i] == m ? 0ull : key[i];
      take(k, m);
    }
  }
  const float ek = lane < K ? expf(mine - top) : 0.0f;
  const float wk = ek / warp_sum(ek);
  if (lane < K) {
    idx[lane] = mi;
    w[lane] = wk;
  }
  if (lane == 0) w[K] = has_gate ? 1.0f / (1.0f + expf(-zg)) : 0.0f;
}

// The routing of one token by the whole block (256 threads; contains block
// barriers): the two-stage top-K for E <= 512, a single-warp rescan otherwise.
__device__ __forceinline__ void block_topk(const float* logits, int E, int K, int has_gate, unsigned long long* cand,
                                           int* idx, float* w) {
  if (E <= 512) {
    // thread 0 reads the shared-gate logit now, so that its latency overlaps stage 1
    const float zg = (has_gate && threadIdx.x == 0) ? __ldcg(logits + E) : 0.0f;
    block_topk_stage1(logits, E, K, cand);
    __syncthreads();
    if ((threadIdx.x >> 5) == 0) block_topk_stage2(zg, E, K, has_gate, cand, idx, w);
  } else if ((threadIdx.x >> 5) == 0) {
    int ik;
    float wk, sig;
    warp_topk(logits, E, K, has_gate, ik, wk, sig);
    const int lane = threadIdx.x & 31;
    if (lane < K) {
      idx[lane] = ik;
      w[lane] = wk;
    }
    if (lane == 0) w[K] = sig;
  }
  __syncthreads();
}

// Record base pointer for one expert slot.
struct BankRef {
  const uint8_t* base;
  long long stride;
  long long off[9];
  int num_experts;
};

// Tensor copies global -> shared of one box (coordinates: the innermost is 0), completing
// on the mbarrier `bar`, with an L2 cache policy.
__device__ __forceinline__ void tma_3d(uint32_t dst, const CUtensorMap* m, int c1, int c2, uint32_t bar, uint64_t pol) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(dst),
      "l"(m), "r"(0), "r"(c1), "r"(c2), "r"(bar), "l"(pol)
      : "memory");
}

__device__ __forceinline__ void tma_4d(uint32_t dst, const CUtensorMap* m, int c1, int c2, int c3, uint32_t bar,
                                       uint64_t pol) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4, %5}], [%6], %7;" ::"r"(dst),
      "l"(m), "r"(0), "r"(c1), "r"(c2), "r"(c3), "r"(bar), "l"(pol)
      : "memory");
}

__device__ __forceinline__ void tma_5d(uint32_t dst, const CUtensorMap* m, int c1, int c2, int c3, int c4, uint32_t bar,
                                       uint64_t pol) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4, %5, %6}], [%7], %8;" ::"r"(dst),
      "l"(m), "r"(0), "r"(c1), "r"(c2), "r"(c3), "r"(c4), "r"(bar), "l"(pol)
      : "memory");
}

}  // namespace fmoe
