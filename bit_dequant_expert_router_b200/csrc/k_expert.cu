// k_expert.cu -- packed-code dequant GEMVs of the selected experts.
//
// gate/up + SwiGLU and down + combine, after "What is Flash-MoE" (a2a-mcp.org),
// sections 2-3: 4-bit / 2-bit tiled dequant matvec, fused SwiGLU, and one
// combine pass of the weighted experts, the sigmoid-gated shared expert and the
// residual.  Weight = code * scale + bias per group of 64; the pages fold the
// affine into fma(code, scale*x, bias*x) per element.  Here the fold is taken
// one level up, per 16-byte chunk of codes:
//     sum_c (q_c s + b) x_c = s * sum_c q_c x_c + b * sum_c x_c,
// with sum_c x_c precomputed once per token and sum_c q_c x_c an exact integer
// dp4a dot product against a 3-digit fixed-point x (see fmoe_device.cuh).
//
// Both kernels are persistent (one 512-thread CTA per SM, static contiguous
// share of the tiles) and stream their weight tiles through a ring of shared-
// memory stages filled by bulk copies (TMA engine) that complete on mbarriers;
// one thread refills a stage as soon as the CTA has consumed it.
#include "fmoe_internal.h"

namespace fmoe {
namespace {

constexpr int kThreads = 512;
constexpr int kRT = 4;   // gate/up tile: 4 rows of gate and the same 4 rows of up
constexpr int kRD = 4;   // down tile: 4 output rows of every selected expert
constexpr int kMaxNP = 16;

__device__ __forceinline__ const uint8_t* slot_record(const ExpertParams& p, int slot, int* err) {
  if (slot < p.K) {
    int e = p.idx ? p.idx[slot] : p.fixed_expert;
    if (e < 0 || e >= p.routed.num_experts) {
      atomicExch(err, kDevBadIndex);
      e = 0;
    }
    return p.routed.base + (long long)e * p.routed.stride;
  }
  return p.shared.base;
}

template <int BITS>
__global__ void __launch_bounds__(kThreads, 1) gateup_kernel(const ExpertParams p, int stages, int stage_bytes) {
  extern __shared__ __align__(128) uint8_t sm[];
  using F = Fmt<BITS>;
  const int tid = threadIdx.x;
  const int H = p.H, I = p.I;
  const int RB = H * BITS / 8;  // code bytes per row
  const int SB = H / kGroup * 2;  // scale (or bias) bytes per row
  const int NC = H * BITS / 128;  // 16-byte chunks per row
  const int NP = NC >= 32 ? NC / 32 : 1;
  const int NE = p.K + p.has_shared;
  const int tps = I / kRT;
  const int ntiles = NE * tps;
  const int t0 = (int)((long long)blockIdx.x * ntiles / gridDim.x);
  const int mine = (int)((long long)(blockIdx.x + 1) * ntiles / gridDim.x) - t0;
  const uint32_t cb = kRT * RB, sb = kRT * SB;

  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + (size_t)stages * stage_bytes);
  float* red = reinterpret_cast<float*>(bars + stages);  // [2][2*kRT][kMaxNP]
  const uint8_t** rec = reinterpret_cast<const uint8_t**>(red + 2 * 2 * kRT * kMaxNP);
  __shared__ int s_abort;

  if (tid < NE) rec[tid] = slot_record(p, tid, p.err);
  if (tid == 0) {
    for (int s = 0; s < stages; ++s) mbar_init(smem_addr(&bars[s]), 1);
    mbar_fence_init();
    s_abort = 0;
  }
  __syncthreads();

  const uint64_t pol_r = l2_policy_evict_first(), pol_s = l2_policy_evict_last();
  auto issue = [&](int j) {
    const int tile = t0 + j, slot = tile / tps, r0 = (tile % tps) * kRT;
    const uint8_t* r = rec[slot];
    const uint64_t pol = slot < p.K ? pol_r : pol_s;
    const long long* off = slot < p.K ? p.routed.off : p.shared.off;
    const int st = j % stages;
    const uint32_t dst = smem_addr(sm + (size_t)st * stage_bytes), bar = smem_addr(&bars[st]);
    mbar_expect_tx(bar, 2 * cb + 4 * sb);
    bulk_g2s(dst, r + off[0] + (long long)r0 * RB, cb, bar, pol);
    bulk_g2s(dst + cb, r + off[3] + (long long)r0 * RB, cb, bar, pol);
    bulk_g2s(dst + 2 * cb, r + off[1] + (long long)r0 * SB, sb, bar, pol);
    bulk_g2s(dst + 2 * cb + sb, r + off[2] + (long long)r0 * SB, sb, bar, pol);
    bulk_g2s(dst + 2 * cb + 2 * sb, r + off[4] + (long long)r0 * SB, sb, bar, pol);
    bulk_g2s(dst + 2 * cb + 3 * sb, r + off[5] + (long long)r0 * SB, sb, bar, pol);
  };
  if (tid == 0)
    for (int j = 0; j < stages && j < mine; ++j) issue(j);

  // This thread's chunk of every row and its digits of x.
  const int pc = tid % NC, rs = tid / NC, RS = kThreads / NC;
  uint32_t L[F::kLimbWords];
  load_limbs<BITS>(p.xq_limbs + (size_t)pc * F::kLimbWords, L);
  const float2 cs = p.xq_cs[pc];
  const int grp = pc * F::kCodesPerChunk / kGroup;
  const int nsub = (2 * kRT + RS - 1) / RS;  // streams per thread (uniform)

  int j = 0;
  for (; j < mine; ++j) {
    const int st = j % stages;
    if (!mbar_wait_bounded(smem_addr(&bars[st]), (uint32_t)((j / stages) & 1), p.err)) s_abort = 1;
    const uint8_t* sbuf = sm + (size_t)st * stage_bytes;
    float* rb = red + (j & 1) * (2 * kRT * kMaxNP);
    for (int k = 0; k < nsub; ++k) {
      const int s = rs + k * RS;
      const bool valid = s < 2 * kRT;
      float part = 0.0f;
      if (valid) {
        const int m = s & 1, r = s >> 1;
        const uint4 q = *reinterpret_cast<const uint4*>(sbuf + m * cb + r * RB + 16 * pc);
        const float S = chunk_dot<BITS>(q, L);
        const uint8_t* sc = sbuf + 2 * cb + 2 * m * sb + r * SB;
        const float sf = bf16_to_f32(reinterpret_cast<const uint16_t*>(sc)[grp]);
        const float bf = bf16_to_f32(reinterpret_cast<const uint16_t*>(sc + sb)[grp]);
        part = fmaf(sf, cs.x * S, bf * cs.y);
      }
      for (int o = (NC >= 32 ? 16 : NC / 2); o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
      if (valid && (pc & 31) == 0) rb[s * kMaxNP + (pc >> 5)] = part;
    }
    __syncthreads();
    if (s_abort) break;
    if (tid == 0 && j + stages < mine) issue(j + stages);
    if (tid < kRT) {
      const int tile = t0 + j, slot = tile / tps, row = (tile % tps) * kRT + tid;
      float g = 0.0f, u = 0.0f;
      for (int n = 0; n < NP; ++n) {
        g += rb[(2 * tid) * kMaxNP + n];
        u += rb[(2 * tid + 1) * kMaxNP + n];
      }
      p.act[(size_t)slot * I + row] = g / (1.0f + expf(-g)) * u;
    }
  }
  if (s_abort && tid == 0) {  // let copies already in flight land before the CTA exits
    for (int k = j; k < mine && k < j + stages; ++k)
      mbar_wait_bounded(smem_addr(&bars[k % stages]), (uint32_t)((k / stages) & 1), p.err);
  }
}

template <int BITS>
__global__ void __launch_bounds__(kThreads, 1) down_kernel(const ExpertParams p, int stages, int stage_bytes) {
  extern __shared__ __align__(128) uint8_t sm[];
  using F = Fmt<BITS>;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int H = p.H, I = p.I;
  const int RB = I * BITS / 8, SB = I / kGroup * 2, NC = I * BITS / 128;
  const int NP = NC >= 32 ? NC / 32 : 1;
  const int NE = p.K + p.has_shared;
  const int sub = kRD * (RB + 2 * SB);  // bytes of one slot inside a stage
  const int ntiles = H / kRD;
  const int t0 = (int)((long long)blockIdx.x * ntiles / gridDim.x);
  const int mine = (int)((long long)(blockIdx.x + 1) * ntiles / gridDim.x) - t0;

  // [stages][digits NE*NC*LW u32][scalars NE*NC float2][red 2*kRD*NE*NP f32][bars][record pointers]
  uint8_t* xl = sm + (size_t)stages * stage_bytes;
  float2* xc = reinterpret_cast<float2*>(xl + (size_t)NE * NC * F::kLimbWords * 4);
  float* red = reinterpret_cast<float*>(xc + NE * NC);
  uint64_t* bars = reinterpret_cast<uint64_t*>(red + 2 * kRD * NE * NP);
  const uint8_t** rec = reinterpret_cast<const uint8_t**>(bars + stages);
  __shared__ int s_abort;

  if (tid < NE) rec[tid] = slot_record(p, tid, p.err);
  if (tid == 0) {
    for (int s = 0; s < stages; ++s) mbar_init(smem_addr(&bars[s]), 1);
    mbar_fence_init();
    s_abort = 0;
  }
  __syncthreads();

  const uint64_t pol_r = l2_policy_evict_first(), pol_s = l2_policy_evict_last();
  auto issue = [&](int j) {
    const int r0 = (t0 + j) * kRD;
    const int st = j % stages;
    const uint32_t dst = smem_addr(sm + (size_t)st * stage_bytes), bar = smem_addr(&bars[st]);
    mbar_expect_tx(bar, (uint32_t)(NE * sub));
    for (int s = 0; s < NE; ++s) {
      const uint8_t* r = rec[s];
      const long long* off = s < p.K ? p.routed.off : p.shared.off;
      const uint64_t pol = s < p.K ? pol_r : pol_s;
      const uint32_t d = dst + s * sub;
      bulk_g2s(d, r + off[6] + (long long)r0 * RB, kRD * RB, bar, pol);
      bulk_g2s(d + kRD * RB, r + off[7] + (long long)r0 * SB, kRD * SB, bar, pol);
      bulk_g2s(d + kRD * RB + kRD * SB, r + off[8] + (long long)r0 * SB, kRD * SB, bar, pol);
    }
  };
  if (tid == 0)
    for (int j = 0; j < stages && j < mine; ++j) issue(j);

  // Digits of every slot's activation vector (all CTAs, while the first stages land).
  for (int g = warp; g < NE * (I / kGroup); g += kThreads / 32) {
    const int slot = g / (I / kGroup), gg = g % (I / kGroup);
    const float2 v = reinterpret_cast<const float2*>(p.act + (size_t)slot * I + gg * kGroup)[lane];
    xq_quantize_group<BITS>(v.x, v.y, gg, xl + (size_t)slot * NC * F::kLimbWords * 4, xc + slot * NC);
  }
  __syncthreads();

  const int pc = tid % NC, q = tid / NC, s = q % NE, rg = q / NE;
  const int RGN = (kThreads / NC) / NE;
  const bool active = rg < RGN;
  uint32_t L[F::kLimbWords];
  float2 cs = make_float2(0.0f, 0.0f);
  float wsl = 0.0f;
  if (active) {
    load_limbs<BITS>(reinterpret_cast<const uint32_t*>(xl) + ((size_t)s * NC + pc) * F::kLimbWords, L);
    cs = xc[s * NC + pc];
    wsl = p.wts ? p.wts[s] : 1.0f;
  } else {
#pragma unroll
    for (int i = 0; i < F::kLimbWords; ++i) L[i] = 0u;
  }
  const int grp = pc * F::kCodesPerChunk / kGroup;
  const int nsub = (kRD + RGN - 1) / RGN;

  int j = 0;
  for (; j < mine; ++j) {
    const int st = j % stages;
    if (!mbar_wait_bounded(smem_addr(&bars[st]), (uint32_t)((j / stages) & 1), p.err)) s_abort = 1;
    const uint8_t* sbuf = sm + (size_t)st * stage_bytes + s * sub;
    float* rb = red + (j & 1) * (kRD * NE * NP);
    for (int k = 0; k < nsub; ++k) {
      const int r = rg + k * RGN;
      const bool valid = active && r < kRD;
      float part = 0.0f;
      if (valid) {
        const uint4 qv = *reinterpret_cast<const uint4*>(sbuf + r * RB + 16 * pc);
        const float S = chunk_dot<BITS>(qv, L);
        const float sf = bf16_to_f32(reinterpret_cast<const uint16_t*>(sbuf + kRD * RB + r * SB)[grp]);
        const float bf = bf16_to_f32(reinterpret_cast<const uint16_t*>(sbuf + kRD * RB + kRD * SB + r * SB)[grp]);
        part = wsl * fmaf(sf, cs.x * S, bf * cs.y);
      }
      for (int o = (NC >= 32 ? 16 : NC / 2); o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
      if (valid && (pc & 31) == 0) rb[r * NE * NP + s * NP + (pc >> 5)] = part;
    }
    __syncthreads();
    if (s_abort) break;
    if (tid == 0 && j + stages < mine) issue(j + stages);
    if (tid < kRD) {
      const int row = (t0 + j) * kRD + tid;
      float acc = p.resid ? p.resid[row] : 0.0f;
      for (int n = 0; n < NE * NP; ++n) acc += rb[tid * NE * NP + n];
      p.out[row] = acc;
    }
  }
  if (s_abort && tid == 0) {
    for (int k = j; k < mine && k < j + stages; ++k)
      mbar_wait_bounded(smem_addr(&bars[k % stages]), (uint32_t)((k / stages) & 1), p.err);
  }
}

constexpr size_t kSmemBudget = 200 * 1024;

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Raises a kernel's dynamic shared-memory limit once per device (and again only
// if a larger size is asked for), so that captured launches make no attribute call.
template <typename Kern>
cudaError_t set_smem(Kern k, size_t bytes) {
  static size_t done[64] = {0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < 64 && done[dev] >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess && dev >= 0 && dev < 64) done[dev] = bytes;
  return e;
}

}  // namespace

cudaError_t launch_gateup(const ExpertParams& p, int bits, cudaStream_t s) {
  const int NE = p.K + p.has_shared;
  const size_t stage = round_up((size_t)2 * kRT * (p.H * bits / 8) + (size_t)4 * kRT * (p.H / kGroup * 2), 128);
  const size_t extra = 8 * 8 + sizeof(float) * 2 * 2 * kRT * kMaxNP + sizeof(void*) * (NE + 1) + 128;
  int stages = (int)((kSmemBudget - extra) / stage);
  stages = stages > 8 ? 8 : stages;
  if (stages < 2) return cudaErrorInvalidValue;
  const size_t bytes = stages * stage + extra;
  const int ntiles = NE * (p.I / kRT);
  int grid = num_sms();
  grid = grid > ntiles ? ntiles : grid;
  cudaError_t e;
  if (bits == 4) {
    if ((e = set_smem(gateup_kernel<4>, bytes)) != cudaSuccess) return e;
    gateup_kernel<4><<<grid, kThreads, bytes, s>>>(p, stages, (int)stage);
  } else {
    if ((e = set_smem(gateup_kernel<2>, bytes)) != cudaSuccess) return e;
    gateup_kernel<2><<<grid, kThreads, bytes, s>>>(p, stages, (int)stage);
  }
  return cudaGetLastError();
}

cudaError_t launch_down(const ExpertParams& p, int bits, cudaStream_t s) {
  const int NE = p.K + p.has_shared;
  const int NC = p.I * bits / 128, NP = NC >= 32 ? NC / 32 : 1;
  const size_t sub = (size_t)kRD * (p.I * bits / 8 + 2 * (p.I / kGroup * 2));
  const size_t stage = round_up(NE * sub, 128);
  const size_t extra = 8 * 8 + (size_t)NE * NC * (3 * 4 * (8 / bits)) * 4 + (size_t)NE * NC * 8 +
                       sizeof(float) * (2 * kRD * NE * NP + 2) + sizeof(void*) * (NE + 1) + 128;
  int stages = (int)((kSmemBudget - extra) / stage);
  stages = stages > 8 ? 8 : stages;
  if (stages < 2) return cudaErrorInvalidValue;
  const size_t bytes = stages * stage + extra;
  const int ntiles = p.H / kRD;
  int grid = num_sms();
  grid = grid > ntiles ? ntiles : grid;
  cudaError_t e;
  if (bits == 4) {
    if ((e = set_smem(down_kernel<4>, bytes)) != cudaSuccess) return e;
    down_kernel<4><<<grid, kThreads, bytes, s>>>(p, stages, (int)stage);
  } else {
    if ((e = set_smem(down_kernel<2>, bytes)) != cudaSuccess) return e;
    down_kernel<2><<<grid, kThreads, bytes, s>>>(p, stages, (int)stage);
  }
  return cudaGetLastError();
}

}  // namespace fmoe
