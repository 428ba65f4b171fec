// fmoe_device.cuh -- device-side building blocks shared by the sm_100a kernels:
// mbarrier + bulk-copy (TMA engine) staging, the packed-code dot product and
// the fixed-point activation format it consumes.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace fmoe {

constexpr int kGroup = 64;        // codes per scale/bias group
constexpr int kChunkBytes = 16;   // one 128-bit load of codes
constexpr int kDevTimeout = 6;    // workspace error word: a bounded wait gave up (FMOE_ERR_DEVICE_TIMEOUT)
constexpr int kDevBadIndex = 7;   // workspace error word: an expert index outside the bank
constexpr unsigned long long kWaitNs = 2000000000ull;  // bound on any device-side wait (2 s)

// Control words at the start of every workspace.
struct WsControl {
  unsigned int tickets[1024];  // last-CTA tickets, one per token
  int err;                     // nonzero once a bounded wait gave up
  int pad[63];
};

// ------------------------------------------------------------------------------------------ small helpers

__device__ __forceinline__ uint32_t smem_addr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ float bf16_to_f32(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

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

// ------------------------------------------------------------------------------------------ mbarrier + bulk copy

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_fence_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
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
    for (int i = 0; i < 64; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (global_ns() - t0 > kWaitNs) {
      atomicExch(err, kDevTimeout);
      return false;
    }
  }
}

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

// Bulk copy global -> this CTA's shared memory, completing `bytes` of
// transaction count on barrier `bar`.  dst, src 16-byte aligned; bytes % 16 == 0.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar, uint64_t pol) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
          dst),
      "l"(src), "r"(bytes), "r"(bar), "l"(pol)
      : "memory");
}

// ------------------------------------------------------------------------------------------ activation format
//
// The dot product sum_c code_c * x_c over one 16-byte chunk of codes runs on
// integer dp4a units.  x is held per group of 64 as a fixed-point value:
//   x_c ~= cscale * X_c,  X_c = rint(x_c * 2^(22-e)),  2^(e-1) <= max|x| < 2^e,
// X_c = d0 * 2^16 + d1 * 2^8 + d2 with signed byte digits (|d0| <= 64).
// The digits of one chunk are stored as 32-bit packs lined up with the way a
// code word is split into bytes:
//   4-bit: word w -> lo = w & 0x0F0F0F0F (codes 0,2,4,6), hi = (w >> 4) & ... (1,3,5,7)
//   2-bit: word w -> pack m = (w >> 2m) & 0x03030303 (codes m, m+4, m+8, m+12)
// Chunk layout: uint32 limbs[limb 0..2][word 0..3][pack 0..PPW-1], then per
// chunk a float2 {cscale, sum of x over the chunk}.

template <int BITS>
struct Fmt {
  static constexpr int kCodesPerWord = 32 / BITS;          // 8 or 16
  static constexpr int kCodesPerChunk = 4 * kCodesPerWord;  // 32 or 64
  static constexpr int kPacksPerWord = 8 / BITS;           // 2 or 4
  static constexpr int kLimbWords = 3 * 4 * kPacksPerWord; // 24 or 48 uint32 per chunk
};

// Quantises one group of 64 values held two per lane (lane l: elements 2l, 2l+1)
// into the format above.  `limb_bytes` addresses chunk 0 of the vector, `cs` its
// per-chunk scalars; g is the group index.  Whole warp participates.
template <int BITS>
__device__ __forceinline__ void xq_quantize_group(float v0, float v1, int g, uint8_t* limb_bytes, float2* cs) {
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
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const float v = k ? v1 : v0;
    const int i = 2 * lane + k;  // element within the group
    const int X = __float2int_rn(v * inv);
    const int d2 = ((X + 128) & 255) - 128;
    const int X1 = (X - d2) >> 8;
    const int d1 = ((X1 + 128) & 255) - 128;
    const int d0 = (X1 - d1) >> 8;
    const int p = g * (kGroup / CPC) + i / CPC;  // chunk
    const int ii = i % CPC;
    const int wi = ii / CPW, j = ii % CPW;
    const int pack = j % PPW, byte = j / PPW;
    const int base = ((p * 3 * 4 + wi) * PPW + pack) * 4 + byte;  // limb 0
    limb_bytes[base] = (uint8_t)(int8_t)d0;
    limb_bytes[base + 4 * PPW * 4] = (uint8_t)(int8_t)d1;
    limb_bytes[base + 2 * 4 * PPW * 4] = (uint8_t)(int8_t)d2;
  }
  float s = v0 + v1;
  if (BITS == 4) {  // two chunks of 32 per group: half-warp sums
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if ((lane & 15) == 0) cs[2 * g + (lane >> 4)] = make_float2(csc, s);
  } else {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) cs[g] = make_float2(csc, s);
  }
}

// Integer dot product of one 16-byte chunk of codes with the chunk's digits L,
// recombined into a float S with sum_c code_c * X_c == S (up to one rounding).
template <int BITS>
__device__ __forceinline__ float chunk_dot(const uint4 q, const uint32_t (&L)[Fmt<BITS>::kLimbWords]) {
  constexpr int PPW = Fmt<BITS>::kPacksPerWord;
  int a0 = 0, a1 = 0, a2 = 0;
  const uint32_t w4[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int wi = 0; wi < 4; ++wi) {
    const uint32_t w = w4[wi];
#pragma unroll
    for (int pk = 0; pk < PPW; ++pk) {
      const uint32_t c = BITS == 4 ? ((w >> (4 * pk)) & 0x0F0F0F0Fu) : ((w >> (2 * pk)) & 0x03030303u);
      a0 = __dp4a((int)c, (int)L[(0 * 4 + wi) * PPW + pk], a0);
      a1 = __dp4a((int)c, (int)L[(1 * 4 + wi) * PPW + pk], a1);
      a2 = __dp4a((int)c, (int)L[(2 * 4 + wi) * PPW + pk], a2);
    }
  }
  const int A = a0 * 256 + a1;  // |A| < 2^23: exact in fp32
  return fmaf((float)A, 256.0f, (float)a2);
}

// Loads one chunk's digits (uint4 granularity) from global or shared memory.
template <int BITS>
__device__ __forceinline__ void load_limbs(const uint32_t* src, uint32_t (&L)[Fmt<BITS>::kLimbWords]) {
#pragma unroll
  for (int i = 0; i < Fmt<BITS>::kLimbWords / 4; ++i) {
    const uint4 v = reinterpret_cast<const uint4*>(src)[i];
    L[4 * i] = v.x;
    L[4 * i + 1] = v.y;
    L[4 * i + 2] = v.z;
    L[4 * i + 3] = v.w;
  }
}

// Record base pointer for one expert slot.
struct BankRef {
  const uint8_t* base;
  long long stride;
  long long off[9];
  int num_experts;
};

}  // namespace fmoe
