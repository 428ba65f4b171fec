// k_expert.cu -- packed-code dequant GEMVs of the selected experts.
//
// gate/up + SwiGLU and down + combine, after "What is Flash-MoE" (a2a-mcp.org),
// sections 2-3: 4-bit / 2-bit tiled dequant matvec (and 8-bit, which one page lists
// among the formats the engine has tried), fused SwiGLU, and one
// combine pass of the weighted experts, the sigmoid-gated shared expert and the
// residual.  Weight = code * scale + bias per group of 64; the pages fold the
// affine into fma(code, scale*x, bias*x) per element.  Here the fold is taken
// one level up, per 16-byte chunk of codes:
//     sum_c (q_c s + b) x_c = s * sum_c q_c x_c + b * sum_c x_c,
// with sum_c x_c precomputed once per token and sum_c q_c x_c an exact integer
// dp4a dot product against a 3-digit fixed-point x (fmoe_device.cuh).
//
// Both kernels run in one wave, one CTA per SM.  Each CTA owns a contiguous
// range of work units (gate/up: a row pair of gate and up of one expert slot;
// down: a few output rows of every selected expert) and stages them with bulk
// copies on the TMA engine in a few large chunks, each completing on its own
// mbarrier: a copy costs issue time on the SM's copy engine, so there are few
// of them, and as much of the CTA's share as fits is requested at once.  Lanes
// keep their groups' digits in registers; warps reduce across their lanes.
// Weight copies that do not depend on the previous kernel (the shared expert's
// rows; the routed down rows once the routing is published) are issued before
// griddepcontrol.wait, so they overlap the previous kernel under programmatic
// dependent launch.
#include <cstdlib>
#include <mutex>

#include "fmoe_internal.h"

namespace fmoe {
namespace {

// ------------------------------------------------------------------------------------------ gate/up

constexpr int kGuWarps = 8;
constexpr int kMaxChunkUnits = 20;  // units per staged chunk, at most (few, large copies: each costs issue time)
constexpr size_t kGuSmemBudget = 220 * 1024;  // shared memory of the gate/up kernel

// GSH: log2 of the weight group size over 64 (0: groups of 64, 1: groups of 128; the
// digits of x stay per 64 columns, and group g of 64 takes scale and bias g >> GSH).
template <int BITS, int NG, int GSH = 0>
struct GuCfg {
  using G = Geo<NG>;
  static constexpr int kPasses = NG >= 32 && BITS == 2 ? 2 : 1;
  static constexpr int kRowPairs = G::kRowsPerPass * kPasses;  // rows of gate (and of up) per unit
  static constexpr int kRowBytes = NG * kGroup * BITS / 8;
  static constexpr int kScaleBytes = (NG >> GSH) * 2;
  static constexpr int kChunks = NG * Fmt<BITS>::kCsPerGroup;             // {cscale, sum x} pairs of x
  static constexpr int kDigitBytes = NG * kGroupWords * 4 + kChunks * 8;  // x digits + their scalars
  static constexpr int kHead = (kDigitBytes + 127) / 128 * 128;
  // units per chunk: kMaxChunkUnits, or fewer where two chunk buffers would not fit
  static constexpr int kUnitBytes = 2 * kRowPairs * (kRowBytes + 2 * kScaleBytes);
  static constexpr int kFit = (int)((kGuSmemBudget - kHead - 256) / (2 * (size_t)kUnitBytes));
  static constexpr int kChunkUnits = kFit < 1 ? 1 : kFit < kMaxChunkUnits ? kFit : kMaxChunkUnits;
  static constexpr int kChunkRows = kChunkUnits * kRowPairs;
  // chunk buffer: gate codes | up codes | gate scales | gate biases | up scales | up biases
  static constexpr int kChunkBytes = (2 * kChunkRows * (kRowBytes + 2 * kScaleBytes) + 127) / 128 * 128;
  static_assert(kRowPairs * kScaleBytes % 16 == 0 && kRowBytes % 16 == 0, "bulk copies move 16-byte multiples");
};

// CTA b's units [u0, u1) under a weighted split of the unit line: a routed unit weighs 8,
// a shared-expert unit sw (1..8).  The shared expert's rows are requested before the
// dependency wait, so with sw < 8 its CTAs take more of them and the routed CTAs less.
// sw = 8 is the even split.  The shared slot's units come last.
__host__ __device__ inline void gu_range(int b, int G, int K, int ups, int has_shared, int sw, int& u0, int& u1) {
  const long long R8 = 8LL * K * ups, Wt = R8 + (has_shared ? (long long)ups * sw : 0);
  const long long w0 = (long long)b * Wt / G, w1 = (long long)(b + 1) * Wt / G;
  u0 = w0 <= R8 ? (int)(w0 / 8) : K * ups + (int)((w0 - R8) / sw);
  u1 = w1 <= R8 ? (int)(w1 / 8) : K * ups + (int)((w1 - R8) / sw);
}

// The four scale arrays of a chunk (gate scales, gate biases, up scales, up biases) as
// one tensor copy: a map over (row bytes / 8, {scale, bias}, {gate, up}, rows, experts)
// lands a box as rows of [gate s | gate b | up s | up b].  sb[0]: routed bank, sb[1]: shared.
struct GuMaps {
  CUtensorMap sb[2];
};

// Persistent: CTA b owns units [b*U/G, (b+1)*U/G) (a unit = kRowPairs rows of
// gate and up of one expert slot), cut into chunks of up to C::kChunkUnits units
// of one slot, each staged into a ring of nbuf chunk buffers with three copies (gate
// codes, up codes, and the four scale arrays as one tensor copy of a whole box: as many
// rows as the largest chunk of the launch) or, where the record layout has no such map,
// six bulk copies;
// warp w computes units w, w+8, .. of the chunk.  A lane always works on the same
// groups of 64 columns, so it keeps their digits of x in registers for the whole kernel.
template <int BITS, int NG, int GSH>
__global__ void __launch_bounds__(kGuWarps * 32, 1) gateup_kernel(const ExpertParams p, int nbuf, int use_maps,
                                                                  int box_rows, const __grid_constant__ GuMaps maps) {
  using G = Geo<NG>;
  using C = GuCfg<BITS, NG, GSH>;
  constexpr int RP = C::kRowPairs, PASSES = C::kPasses;
  constexpr int LPR = G::kLanesPerRow, RPP = G::kRowsPerPass, GPL = G::kGroupsPerLane;
  constexpr int RB = C::kRowBytes, SB = C::kScaleBytes, CR = C::kChunkRows, CHB = C::kChunkBytes;
  extern __shared__ __align__(128) uint8_t sm[];
  __shared__ __align__(8) uint64_t s_bar[8];
  __shared__ __align__(8) uint64_t s_bar_x;
  __shared__ int s_idx[32];
  __shared__ float s_wt[33];
  __shared__ unsigned long long s_cand[8 * 32];
  __shared__ int s_done[kGuWarps * 32];
  __shared__ int s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int I = p.I;
  [[maybe_unused]] const int NE = p.K + p.has_shared;  // read only by the debug build's bounds checks
  const int ups = I / RP;
  int u0, u1;
  gu_range(blockIdx.x, gridDim.x, p.K, ups, p.has_shared, p.gu_sw, u0, u1);
  const uint32_t* xs = reinterpret_cast<const uint32_t*>(sm);
  const float2* xcs = reinterpret_cast<const float2*>(sm + NG * kGroupWords * 4);

  if (tid == 0) {
    for (int b = 0; b < nbuf; ++b) mbar_init(smem_addr(&s_bar[b]), 1);
    mbar_init(smem_addr(&s_bar_x), 1);
    mbar_fence_init();
    s_abort = 0;
  }
  __syncthreads();

  // Chunk c covers units [cu, ce): up to C::kChunkUnits units, never across a slot boundary.
  auto chunk_end = [&](int cu) { return min(min(cu + C::kChunkUnits, u1), (cu / ups + 1) * ups); };
  auto issue = [&](int c, int cu, int ce) {  // thread 0
    const int sl = cu / ups, r0 = (cu % ups) * RP, rows = (ce - cu) * RP;
    const bool routed = sl < p.K;
    const uint8_t* rec = routed ? p.routed.base + (long long)s_idx[sl] * p.routed.stride : p.shared.base;
    const long long* off = routed ? p.routed.off : p.shared.off;
    const uint64_t pol = l2_policy_evict_first();  // weights come back only after a whole model pass
    uint8_t* buf = sm + C::kHead + (size_t)(c % nbuf) * CHB;
    const uint32_t dst = smem_addr(buf), bar = smem_addr(&s_bar[c % nbuf]);
    const uint32_t cb = rows * RB, sb = rows * SB;
    // the rows stay inside the matrix and the chunk buffer; the record inside its bank
    if (!FMOE_IN_BOUNDS(r0 >= 0 && rows > 0 && rows <= CR && r0 + rows <= p.I && c >= 0 &&
                            (!routed || (s_idx[sl] >= 0 && s_idx[sl] < p.routed.num_experts)),
                        p.err))
      return;
    if (use_maps) {  // the scale box always moves box_rows rows (past the last row: zeros)
      mbar_expect_tx(bar, 2 * cb + 4 * box_rows * SB);
      bulk_g2s(dst, rec + off[0] + (long long)r0 * RB, cb, bar, pol);
      bulk_g2s(dst + CR * RB, rec + off[3] + (long long)r0 * RB, cb, bar, pol);
      tma_5d(dst + 2 * CR * RB, &maps.sb[routed ? 0 : 1], 0, 0, r0, routed ? s_idx[sl] : 0, bar, pol);
    } else {
      mbar_expect_tx(bar, 2 * cb + 4 * sb);
      bulk_g2s(dst, rec + off[0] + (long long)r0 * RB, cb, bar, pol);
      bulk_g2s(dst + CR * RB, rec + off[3] + (long long)r0 * RB, cb, bar, pol);
      bulk_g2s(dst + 2 * CR * RB, rec + off[1] + (long long)r0 * SB, sb, bar, pol);
      bulk_g2s(dst + 2 * CR * RB + CR * SB, rec + off[2] + (long long)r0 * SB, sb, bar, pol);
      bulk_g2s(dst + 2 * CR * RB + 2 * CR * SB, rec + off[4] + (long long)r0 * SB, sb, bar, pol);
      bulk_g2s(dst + 2 * CR * RB + 3 * CR * SB, rec + off[5] + (long long)r0 * SB, sb, bar, pol);
    }
  };
  // where a row's four scale arrays sit in a chunk buffer: row r, array a at (r * srow + a * sarr) bf16
  const int srow = use_maps ? 2 * SB : SB / 2, sarr = use_maps ? SB / 2 : CR * SB / 2;

  // Shared-expert chunks need nothing from the router: request them first.
  if (tid == 0) {
    int cu = u0;
    for (int c = 0; c < nbuf && cu < u1; ++c) {
      const int ce = chunk_end(cu);
      if (cu / ups >= p.K) issue(c, cu, ce);
      cu = ce;
    }
  }

  pdl_wait();  // the router's logits and x digits are complete
  pdl_trigger();

  // The routing: from the logits, by the whole block (every CTA the same), or given.
  if (p.logits) {
    block_topk(p.logits, p.E, p.K, 1, s_cand, s_idx, s_wt);
  } else if (warp == 0 && lane < p.K) {
    s_idx[lane] = p.route_idx ? p.route_idx[lane] : p.fixed_expert;
  }
  __syncthreads();
  if (tid < p.K) {
    const int e = s_idx[tid];
    if (e < 0 || e >= p.routed.num_experts) {
      atomicExch(p.err, kDevBadIndex);
      s_idx[tid] = 0;
    }
  }
  __syncthreads();
  if (p.logits && blockIdx.x == 0 && tid <= p.K) {  // the routing for the down kernel and the caller
    if (tid < p.K) {
      if (p.rt_idx) p.rt_idx[tid] = s_idx[tid];
      if (p.idx_out) p.idx_out[tid] = s_idx[tid];
      if (p.w_out) p.w_out[tid] = s_wt[tid];
    }
    if (p.rt_w) p.rt_w[tid] = s_wt[tid];
  }
  if (p.logits && p.route_ready && blockIdx.x == 0) {
    // publish it: lane 1 of warp 1 has no copies in flight, so its release does not
    // wait for any (a gpu-scope release waits for the issuing thread's own bulk copies)
    __syncthreads();
    if (tid == 33) {
      __threadfence();
      st_release_gpu(p.route_ready, 1u);
    }
  }
  // Warm L2 with this CTA's slice of each routed expert's down matrix (lane 0 of the
  // last warp; CTAs whose range starts in a routed slot).
  auto prefetch_down_rows = [&]() {
    if (u0 / ups >= p.K) return;
    const long long len[3] = {(long long)p.H * (I * BITS / 8), (long long)p.H * (I / (kGroup << GSH)) * 2,
                              (long long)p.H * (I / (kGroup << GSH)) * 2};
    for (int k = 0; k < p.K; ++k) {
      const uint8_t* rec = p.routed.base + (long long)s_idx[k] * p.routed.stride;
      for (int m = 0; m < 3; ++m) {
        const long long a0 = (len[m] * blockIdx.x / gridDim.x) & ~15LL;
        const long long a1 = (len[m] * (blockIdx.x + 1) / gridDim.x) & ~15LL;
        if (a1 > a0) prefetch_l2(rec + p.routed.off[6 + m] + a0, (uint32_t)(a1 - a0));
      }
    }
  };
  if (lane == 0) {
    // x digits by warp 0; the first routed chunks one per warp (lane 0), so that
    // their copies go out from several warps at once; the L2 warm-up by warp 7
    if (warp == 0) {
      const uint32_t bx = smem_addr(&s_bar_x);
      mbar_expect_tx(bx, C::kDigitBytes);
      bulk_g2s(smem_addr(sm), p.xq_limbs, NG * kGroupWords * 4, bx, l2_policy_evict_last());
      bulk_g2s(smem_addr(sm + NG * kGroupWords * 4), p.xq_cs, C::kChunks * 8, bx, l2_policy_evict_last());
    }
    int cu = u0;
    for (int c = 0; c < nbuf && cu < u1; ++c) {
      const int ce = chunk_end(cu);
      if (cu / ups < p.K && c % kGuWarps == warp) issue(c, cu, ce);
      cu = ce;
    }
    if (warp == kGuWarps - 1 && p.prefetch_down == 1) prefetch_down_rows();
  }
  __syncwarp();

  // This lane's groups and their digits of x, for the whole kernel.
  const int sub = lane / LPR, gl = lane % LPR;
  uint32_t L[GPL][48];
  float2 cs[GPL];
  bool ok = mbar_wait_bounded(smem_addr(&s_bar_x), 0, p.err);
#pragma unroll
  for (int j = 0; j < GPL; ++j) {
    const int g = gl + LPR * j;
    load_group_limbs(xs, g, NG, L[j]);
    cs[j] = group_scalars<BITS>(xcs, g);
  }

  int cu = u0;
  for (int c = 0; cu < u1; ++c) {
    const int ce = chunk_end(cu);
    const int sl = cu / ups, rbase = (cu % ups) * RP;
    if (!mbar_wait_bounded(smem_addr(&s_bar[c % nbuf]), (uint32_t)((c / nbuf) & 1), p.err)) ok = false;
    // the late down prefetch: once the CTA's last chunk is in, its DRAM traffic no longer
    // competes with this CTA's gate/up stream
    if (ok && ce == u1 && p.prefetch_down == 2 && warp == kGuWarps - 1 && lane == 0) prefetch_down_rows();
    const uint8_t* buf = sm + C::kHead + (size_t)(c % nbuf) * CHB;
    for (int k = warp; ok && k < ce - cu; k += kGuWarps) {
      float accg[PASSES], accu[PASSES];
#pragma unroll
      for (int i = 0; i < PASSES; ++i) accg[i] = accu[i] = 0.0f;
#pragma unroll
      for (int j = 0; j < GPL; ++j) {
        const int g = gl + LPR * j;
#pragma unroll
        for (int i = 0; i < PASSES; ++i) {
          const int r = k * RP + sub + RPP * i;  // row within the chunk
          float Sg, Su;
          if constexpr (BITS == 8) {
            uint4 q[4], v[4];
            load_group_codes8(buf + r * RB, g, q);
            load_group_codes8(buf + CR * RB + r * RB, g, v);
            Sg = group_dot8(q, L[j]);
            Su = group_dot8(v, L[j]);
          } else {
            uint4 q0, q1, v0, v1;
            load_group_codes<BITS>(buf + r * RB, g, q0, q1);
            load_group_codes<BITS>(buf + CR * RB + r * RB, g, v0, v1);
            Sg = group_dot<BITS>(q0, q1, L[j]);
            Su = group_dot<BITS>(v0, v1, L[j]);
          }
          const uint16_t* sc = reinterpret_cast<const uint16_t*>(buf + 2 * CR * RB) + r * srow + (g >> GSH);
          const float gs = bf16_to_f32(sc[0]);
          const float gb = bf16_to_f32(sc[sarr]);
          const float us = bf16_to_f32(sc[2 * sarr]);
          const float ub = bf16_to_f32(sc[3 * sarr]);
          accg[i] = fmaf(gs, cs[j].x * Sg, fmaf(gb, cs[j].y, accg[i]));
          accu[i] = fmaf(us, cs[j].x * Su, fmaf(ub, cs[j].y, accu[i]));
        }
      }
#pragma unroll
      for (int i = 0; i < PASSES; ++i) {
#pragma unroll
        for (int o = LPR / 2; o > 0; o >>= 1) {
          accg[i] += __shfl_xor_sync(0xffffffffu, accg[i], o);
          accu[i] += __shfl_xor_sync(0xffffffffu, accu[i], o);
        }
      }
      if (gl == 0) {
#pragma unroll
        for (int i = 0; i < PASSES; ++i) {
          const float g = accg[i], uu = accu[i];
          const int row = rbase + k * RP + sub + RPP * i;
          if (FMOE_IN_BOUNDS(row < I && sl < NE, p.err)) p.act[(size_t)sl * I + row] = g / (1.0f + expf(-g)) * uu;
        }
      }
    }
    __syncthreads();  // every warp is done with this chunk buffer
    if (!ok) s_abort = 1;
    if (tid == 0) {  // refill the buffer with chunk c + nbuf
      int nu = ce, nc = c + 1;
      while (nc < c + nbuf && nu < u1) {
        nu = chunk_end(nu);
        ++nc;
      }
      if (nu < u1 && !s_abort) {
        fence_proxy_async();
        issue(c + nbuf, nu, chunk_end(nu));
      }
    }
    cu = ce;
  }

  // Groups of 64 activations: the CTA that completes a group writes its digits
  // for the down kernel.  The counting threads (warps 1..) fence after the block
  // barrier (release of every act write of the CTA), the writing warps before
  // reading (acquire).  Warp 7 lane 0 issued L2 prefetches and warp 0 nothing
  // that matters here, but a gpu-scope fence waits for its own thread's copies,
  // so neither takes part.
  __syncthreads();
  if (s_abort) {  // let copies still in flight land before the CTA exits
    if (tid == 0)
      for (int b = 0; b < nbuf; ++b) mbar_wait_bounded(smem_addr(&s_bar[b]), 0, p.err);
    return;
  }
  const int g0 = u0 * RP / kGroup, ng = (u1 * RP - 1) / kGroup - g0 + 1;  // groups over concatenated slot rows
  const int ct = tid - 32;
  if (ct >= 0 && ct < ng) {
    const int g = g0 + ct;
    const int lo = max(u0 * RP, g * kGroup), hi = min(u1 * RP, (g + 1) * kGroup);
    __threadfence();
    const unsigned prev = atomicAdd(&p.grp_cnt[g], (unsigned)(hi - lo));
    s_done[ct] = prev + (unsigned)(hi - lo) == (unsigned)kGroup;
  }
  __syncthreads();
  for (int t = warp - 1; warp >= 1 && warp < kGuWarps - 1 && t < ng; t += kGuWarps - 2) {
    if (!s_done[t]) continue;
    __threadfence();
    const int g = g0 + t, slot = g * kGroup / I, gg = (g * kGroup % I) / kGroup;
    const float2 v = __ldcg(reinterpret_cast<const float2*>(p.act + (size_t)g * kGroup) + lane);
    xq_quantize_group<BITS>(v.x, v.y, gg, I / kGroup, p.act_limbs + (size_t)slot * I * 3,
                            p.act_cs + (size_t)slot * (I / kGroup) * Fmt<BITS>::kCsPerGroup);
    if (lane == 0) p.grp_cnt[g] = 0u;
  }
}

// ------------------------------------------------------------------------------------------ down + combine

constexpr int kDnWarps = 8;

template <int BITS, int NG, int GSH = 0>
struct DnCfg {
  static constexpr int kRowBytes = NG * kGroup * BITS / 8;
  static constexpr int kScaleBytes = (NG >> GSH) * 2;
  // output rows per unit: 2, or more when a row's scales are too short for a 16-byte copy
  static constexpr int kRows = kScaleBytes >= 8 ? 2 : 16 / kScaleBytes;
  static constexpr int kChunks = NG * Fmt<BITS>::kCsPerGroup;  // {cscale, sum a} pairs of a slot's activations
  static_assert(kRows * kScaleBytes % 16 == 0 && kRowBytes % 16 == 0, "bulk copies move 16-byte multiples");
};

// Persistent: CTA b owns units [b*U/G, (b+1)*U/G) of kRows output rows,
// staged in chunks of up to `chunk_units` units: for every selected expert the
// chunk's rows of its down matrix (codes, scales, biases: three bulk copies).
// The experts are known once the gate/up kernel (CTA 0) has written the
// routing, i.e. after the wait; the gate/up kernel has warmed L2 with this
// CTA's rows by then, so the copies come mostly from L2.  Lane l owns the (slot, group) pairs
// q = l, l+32, .. (PPL of them) of every row and keeps their digits in
// registers; the warp sums a row's pairs by shuffles.
template <int BITS, int NG, int PPL, int GSH>
__global__ void __launch_bounds__(kDnWarps * 32, 1) down_kernel(const ExpertParams p, int chunk_units, int nbuf) {
  using C = DnCfg<BITS, NG, GSH>;
  constexpr int RD = C::kRows;
  constexpr int RB = C::kRowBytes, SB = C::kScaleBytes;
  constexpr int NCH = C::kChunks;
  extern __shared__ __align__(128) uint8_t sm[];
  __shared__ __align__(8) uint64_t s_bar[8];
  __shared__ __align__(8) uint64_t s_bar_x;
  __shared__ const uint8_t* s_src[33][3];
  __shared__ float s_w[33];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int NE = p.K + p.has_shared, NP = NE * NG;
  const int U = p.H / RD;
  const int u0 = (int)((long long)blockIdx.x * U / gridDim.x);
  const int u1 = (int)((long long)(blockIdx.x + 1) * U / gridDim.x);
  const int dwords = NE * NG * kGroupWords;  // digits of every slot's activations
  const uint32_t* xs = reinterpret_cast<const uint32_t*>(sm);
  const float2* xcs = reinterpret_cast<const float2*>(sm + (size_t)dwords * 4);
  const int head = (dwords * 4 + NE * NCH * 8 + 127) / 128 * 128;
  const int crows = chunk_units * RD;
  const int slot_bytes = crows * (RB + 2 * SB);  // one expert's rows of a chunk
  const int chb = (NE * slot_bytes + 127) / 128 * 128;

  // The shared expert's rows are weights: thread 0 requests them for the first
  // chunks before the wait.  The routing is written by CTA 0 of the gate/up
  // kernel: if it is published already (route_ready), it is read and the routed
  // rows requested before the wait, otherwise after it.
  if (tid == 0 && p.has_shared) {
    s_src[p.K][0] = p.shared.base + p.shared.off[6];
    s_src[p.K][1] = p.shared.base + p.shared.off[7];
    s_src[p.K][2] = p.shared.base + p.shared.off[8];
  }
  // chunk c, slots [s0, s1): units [u0 + c*chunk_units, ..) of each slot (thread 0);
  // `expect` arms the chunk's barrier for all NE slots
  auto issue = [&](int c, int s0, int s1, bool expect) {
    const int cu = u0 + c * chunk_units, ce = min(cu + chunk_units, u1);
    const long long j0 = (long long)cu * RD;
    const uint32_t rows = (uint32_t)(ce - cu) * RD;
    uint8_t* buf = sm + head + (size_t)(c % nbuf) * chb;
    const uint32_t bar = smem_addr(&s_bar[c % nbuf]);
    const uint64_t pol_r = l2_policy_evict_first(), pol_s = l2_policy_evict_last();
    if (expect) mbar_expect_tx(bar, (uint32_t)NE * rows * (RB + 2 * SB));
    for (int s = s0; s < s1; ++s) {
      // the chunk's rows stay inside the matrix and the slot's part of the buffer
      if (!FMOE_IN_BOUNDS(j0 + rows <= p.H && rows <= (uint32_t)crows && s < NE, p.err)) continue;
      const uint64_t pol = s < p.K ? pol_r : pol_s;
      const uint32_t d = smem_addr(buf + (size_t)s * slot_bytes);
      bulk_g2s(d, s_src[s][0] + j0 * RB, rows * RB, bar, pol);
      bulk_g2s(d + crows * RB, s_src[s][1] + j0 * SB, rows * SB, bar, pol);
      bulk_g2s(d + crows * RB + crows * SB, s_src[s][2] + j0 * SB, rows * SB, bar, pol);
    }
  };
  const int nchunk = (u1 - u0 + chunk_units - 1) / chunk_units;
  __shared__ int s_early;
  if (tid == 0) {
    for (int b = 0; b < nbuf; ++b) mbar_init(smem_addr(&s_bar[b]), 1);
    mbar_init(smem_addr(&s_bar_x), 1);
    mbar_fence_init();
    for (int c = 0; c < nbuf && c < nchunk; ++c) issue(c, p.K, NE, true);  // the shared slot (if any)
  }
  // the routing, from the slots the gate/up kernel wrote (or given)
  auto read_routing = [&]() {  // warp 1
    if (lane < p.K) {
      int ik = p.route_idx ? __ldcg(p.route_idx + lane) : p.fixed_expert;
      if (ik < 0 || ik >= p.routed.num_experts) {
        atomicExch(p.err, kDevBadIndex);
        ik = 0;
      }
      const uint8_t* rec = p.routed.base + (long long)ik * p.routed.stride;
      s_src[lane][0] = rec + p.routed.off[6];
      s_src[lane][1] = rec + p.routed.off[7];
      s_src[lane][2] = rec + p.routed.off[8];
      s_w[lane] = p.route_w ? __ldcg(p.route_w + lane) : 1.0f;
    }
    if (lane == 0 && p.has_shared)
      s_w[p.K] = p.sigma_logit ? 1.0f / (1.0f + expf(-__ldcg(p.sigma_logit)))
                               : (p.route_w ? __ldcg(p.route_w + p.K) : 1.0f);
  };
  // Published already (gate/up CTA 0 finished its selection long before this grid
  // starts, in practice)?  Warp 1 has no copies in flight, so its acquire does not wait.
  if (warp == 1) {  // every lane acquires, so that its own reads of the routing follow
    const bool seen = p.route_ready && ld_acquire_gpu(p.route_ready) == 1u;
    const bool early = __all_sync(0xffffffffu, seen);
    if (early) read_routing();
    if (lane == 0) s_early = early ? 1 : 0;
  }
  __syncthreads();
  const bool early = s_early != 0;
  // the routed rows of the first chunks (mostly from L2; their barriers are armed): one
  // (chunk, slot) per issuing lane, lane 0 of warps 1.., so that the requests go out side by side
  auto issue_routed = [&]() {
    if (lane == 0 && warp > 0)
      for (int cs = warp - 1; cs < min(nbuf, nchunk) * p.K; cs += kDnWarps - 1) issue(cs / p.K, cs % p.K, cs % p.K + 1, false);
  };
  if (early) issue_routed();
  pdl_wait();  // the activations' digits (and the routing) are complete
  pdl_trigger();
  if (!early) {
    if (warp == 1) read_routing();
    __syncthreads();
  }

  if (tid == 0) {  // every slot's digits, once per CTA
    const uint32_t bx = smem_addr(&s_bar_x);
    mbar_expect_tx(bx, (uint32_t)(dwords * 4 + NE * NCH * 8));
    bulk_g2s(smem_addr(sm), p.act_limbs, (uint32_t)dwords * 4, bx, l2_policy_evict_first());
    bulk_g2s(smem_addr(sm + (size_t)dwords * 4), p.act_cs, (uint32_t)(NE * NCH * 8), bx, l2_policy_evict_first());
  }
  if (!early) issue_routed();
  __syncwarp();  // lanes 1..31 of warp 0 wait for the issue instead of spinning beside it

  // This lane's (slot, group) pairs and their digits.
  uint32_t L[PPL][48];
  float2 cs[PPL];
  float wq[PPL];
  int qoff[PPL], qg[PPL];
  bool ok = mbar_wait_bounded(smem_addr(&s_bar_x), 0, p.err);
#pragma unroll
  for (int m = 0; m < PPL; ++m) {
    const int q = lane + 32 * m;
    const bool has = q < NP;
    const int s = has ? q / NG : 0, g = has ? q % NG : 0;
    load_group_limbs(xs + (size_t)s * NG * kGroupWords, g, NG, L[m]);
    cs[m] = group_scalars<BITS>(xcs + s * NCH, g);
    wq[m] = has ? s_w[s] : 0.0f;
    qoff[m] = s * slot_bytes;
    qg[m] = g;
  }

  for (int c = 0; c < nchunk; ++c) {
    const int cu = u0 + c * chunk_units, ce = min(cu + chunk_units, u1);
    if (!mbar_wait_bounded(smem_addr(&s_bar[c % nbuf]), (uint32_t)((c / nbuf) & 1), p.err)) ok = false;
    const uint8_t* buf = sm + head + (size_t)(c % nbuf) * chb;
    for (int k = warp; ok && k < ce - cu; k += kDnWarps) {
      float acc[RD];
#pragma unroll
      for (int r = 0; r < RD; ++r) acc[r] = 0.0f;
#pragma unroll
      for (int m = 0; m < PPL; ++m) {
        const uint8_t* sb = buf + qoff[m];
#pragma unroll
        for (int r = 0; r < RD; ++r) {
          const int row = k * RD + r;  // row within the chunk
          float S;
          if constexpr (BITS == 8) {
            uint4 q[4];
            load_group_codes8(sb + row * RB, qg[m], q);
            S = group_dot8(q, L[m]);
          } else {
            uint4 q0, q1;
            load_group_codes<BITS>(sb + row * RB, qg[m], q0, q1);
            S = group_dot<BITS>(q0, q1, L[m]);
          }
          const float sc =
              bf16_to_f32(reinterpret_cast<const uint16_t*>(sb + crows * RB + row * SB)[qg[m] >> GSH]);
          const float bi =
              bf16_to_f32(reinterpret_cast<const uint16_t*>(sb + crows * RB + crows * SB + row * SB)[qg[m] >> GSH]);
          acc[r] = fmaf(wq[m], fmaf(sc, cs[m].x * S, bi * cs[m].y), acc[r]);
        }
      }
#pragma unroll
      for (int r = 0; r < RD; ++r) acc[r] = warp_sum(acc[r]);
#pragma unroll
      for (int r = 0; r < RD; ++r)
        if (lane == r) {
          const int row = (cu + k) * RD + r;
          if (FMOE_IN_BOUNDS(row < p.H, p.err)) p.out[row] = (p.resid ? p.resid[row] : 0.0f) + acc[r];
        }
    }
    __syncthreads();  // every warp is done with this chunk buffer
    if (tid == 0 && c + nbuf < nchunk && ok) {
      fence_proxy_async();
      issue(c + nbuf, 0, NE, true);
    }
  }
  if (!ok && tid == 0)
    for (int b = 0; b < nbuf; ++b) mbar_wait_bounded(smem_addr(&s_bar[b]), 0, p.err);
}

// One thread waits until *flag == value, at most limit_ns; on timeout it records
// FMOE_ERR_DEVICE_TIMEOUT in *err and returns.
__global__ void wait_flag_kernel(const unsigned int* flag, unsigned int value, unsigned long long limit_ns, int* err) {
  flag_wait_bounded(flag, value, limit_ns, err);
}

size_t round128(size_t v) { return (v + 127) / 128 * 128; }

constexpr size_t kSmemBudget = 220 * 1024;

// The gate/up scale maps of the routed and the shared bank, if the record layout allows
// them: scale rows of a multiple of 16 bytes, and one distance from each scale array to
// its bias array and from gate's arrays to up's.  The bank records are only read.
bool encode_gu_scale_maps(GuMaps& m, const ExpertParams& p, int SB, int box_rows) {
  if (SB % 16 != 0 || box_rows > 256 || SB / 8 > 256 || p.I > (1 << 24)) return false;
  for (int bk = 0; bk < 2; ++bk) {
    const BankRef& r = bk == 0 ? p.routed : p.shared;
    if (bk == 1 && !p.has_shared) {
      m.sb[1] = m.sb[0];
      continue;
    }
    const long long* o = r.off;
    const long long sb = o[2] - o[1], gu = o[4] - o[1];
    if (sb <= 0 || gu <= 0 || o[5] - o[4] != sb || (sb & 15) || (gu & 15)) return false;
    const long long ne = bk == 0 ? r.num_experts : 1;
    if (ne < 1 || (bk == 0 && (r.stride <= 0 || (r.stride & 15)))) return false;
    const cuuint64_t dims[5] = {(cuuint64_t)(SB / 8), 2, 2, (cuuint64_t)p.I, (cuuint64_t)ne};
    const cuuint64_t st[4] = {(cuuint64_t)sb, (cuuint64_t)gu, (cuuint64_t)SB, (cuuint64_t)(bk == 0 ? r.stride : 16)};
    const cuuint32_t box[5] = {(cuuint32_t)(SB / 8), 2, 2, (cuuint32_t)box_rows, 1};
    if (!encode_map(&m.sb[bk], r.base + o[1], 5, dims, st, box)) return false;
  }
  return true;
}

template <int BITS, int NG, int GSH>
cudaError_t gateup_dispatch(const ExpertParams& p, bool pdl, cudaStream_t s) {
  using C = GuCfg<BITS, NG, GSH>;
  const int NE = p.K + p.has_shared;
  const int units = NE * (p.I / C::kRowPairs);
  int grid = num_sms();
  grid = grid > units ? units : grid;
  int per_cta = 0;  // the largest CTA range of the weighted split
  for (int b = 0; b < grid; ++b) {
    int a0, a1;
    gu_range(b, grid, p.K, p.I / C::kRowPairs, p.has_shared, p.gu_sw, a0, a1);
    per_cta = a1 - a0 > per_cta ? a1 - a0 : per_cta;
  }
  // each CTA counts at most one block of threads' worth of activation groups
  if ((long long)per_cta * C::kRowPairs / kGroup + 2 > kGuWarps * 32 - 32) return cudaErrorInvalidValue;
  int nbuf = (int)((kGuSmemBudget - C::kHead) / C::kChunkBytes);
  const int need = (per_cta + C::kChunkUnits - 1) / C::kChunkUnits + 1;  // +1: a chunk may stop at a slot boundary
  nbuf = nbuf > need ? need : nbuf;
  nbuf = nbuf > 8 ? 8 : nbuf;
  if (nbuf < 1) return cudaErrorInvalidValue;
  const size_t smem = C::kHead + (size_t)nbuf * C::kChunkBytes;
  void (*k)(const ExpertParams, int, int, int, const GuMaps) = gateup_kernel<BITS, NG, GSH>;
  cudaError_t e = set_smem((const void*)k, smem);
  if (e != cudaSuccess) return e;
  GuMaps maps;
  // a chunk never holds more units than a CTA's range: the scale box need not either
  const int box_rows = C::kRowPairs * (per_cta < C::kChunkUnits ? per_cta : C::kChunkUnits);
  const int use_maps = encode_gu_scale_maps(maps, p, C::kScaleBytes, box_rows) ? 1 : 0;
  return launch_pdl(k, dim3(grid), dim3(kGuWarps * 32), smem, s, pdl, p, nbuf, use_maps, box_rows, maps);
}

// Down-kernel staging: (chunk units, buffers, shared bytes) for NE slots, or false.
template <int BITS, int NG, int GSH = 0>
bool down_plan(int H, int NE, int& chunk_units, int& nbuf, size_t& smem) {
  using C = DnCfg<BITS, NG, GSH>;
  const int units = H / C::kRows;
  int grid = num_sms();
  grid = grid > units ? units : grid;
  const int per_cta = (units + grid - 1) / grid;
  const size_t head = round128((size_t)NE * NG * kGroupWords * 4 + (size_t)NE * C::kChunks * 8);
  const size_t unit_bytes = (size_t)NE * C::kRows * (C::kRowBytes + 2 * C::kScaleBytes);
  if (head + 2 * round128(unit_bytes) > kSmemBudget) return false;
  // the whole share in one buffer when it fits, otherwise a ring of two
  if (head + round128(per_cta * unit_bytes) <= kSmemBudget) {
    chunk_units = per_cta;
    nbuf = 1;
  } else {
    chunk_units = (int)((kSmemBudget - head) / 2 / unit_bytes);
    nbuf = 2;
  }
  smem = head + (size_t)nbuf * round128((size_t)chunk_units * unit_bytes);
  return true;
}

template <int BITS, int NG, int GSH>
cudaError_t down_dispatch(const ExpertParams& p, bool pdl, cudaStream_t s) {
  using C = DnCfg<BITS, NG, GSH>;
  const int NE = p.K + p.has_shared;
  int cu = 0, nbuf = 0;
  size_t smem = 0;
  const int ppl = (NE * NG + 31) / 32;
  if (!down_plan<BITS, NG, GSH>(p.H, NE, cu, nbuf, smem) || ppl > 4) return cudaErrorInvalidValue;
  const int units = p.H / C::kRows;
  int grid = num_sms();
  grid = grid > units ? units : grid;
  void (*k)(const ExpertParams, int, int) = ppl == 1 ? down_kernel<BITS, NG, 1, GSH>
                                          : ppl == 2 ? down_kernel<BITS, NG, 2, GSH>
                                          : ppl == 3 ? down_kernel<BITS, NG, 3, GSH>
                                                     : down_kernel<BITS, NG, 4, GSH>;
  cudaError_t e = set_smem((const void*)k, smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(k, dim3(grid), dim3(kDnWarps * 32), smem, s, pdl, p, cu, nbuf);
}

template <int BITS>
cudaError_t gateup_bits(const ExpertParams& p, bool pdl, cudaStream_t s) {
  if (p.gsh == 1) {  // groups of 128: rows of at least 16 groups of 64
    switch (p.H / kGroup) {
      case 16: return gateup_dispatch<BITS, 16, 1>(p, pdl, s);
      case 32: return gateup_dispatch<BITS, 32, 1>(p, pdl, s);
      case 64: return gateup_dispatch<BITS, 64, 1>(p, pdl, s);
      case 128: return gateup_dispatch<BITS, 128, 1>(p, pdl, s);
    }
    return cudaErrorInvalidValue;
  }
  switch (p.H / kGroup) {
    case 2: return gateup_dispatch<BITS, 2, 0>(p, pdl, s);
    case 4: return gateup_dispatch<BITS, 4, 0>(p, pdl, s);
    case 8: return gateup_dispatch<BITS, 8, 0>(p, pdl, s);
    case 16: return gateup_dispatch<BITS, 16, 0>(p, pdl, s);
    case 32: return gateup_dispatch<BITS, 32, 0>(p, pdl, s);
    case 64: return gateup_dispatch<BITS, 64, 0>(p, pdl, s);
    case 128: return gateup_dispatch<BITS, 128, 0>(p, pdl, s);
  }
  return cudaErrorInvalidValue;
}

template <int BITS>
cudaError_t down_bits(const ExpertParams& p, bool pdl, cudaStream_t s) {
  if (p.gsh == 1) {
    switch (p.I / kGroup) {
      case 16: return down_dispatch<BITS, 16, 1>(p, pdl, s);
      case 32: return down_dispatch<BITS, 32, 1>(p, pdl, s);
      case 64: return down_dispatch<BITS, 64, 1>(p, pdl, s);
      case 128: return down_dispatch<BITS, 128, 1>(p, pdl, s);
    }
    return cudaErrorInvalidValue;
  }
  switch (p.I / kGroup) {
    case 2: return down_dispatch<BITS, 2, 0>(p, pdl, s);
    case 4: return down_dispatch<BITS, 4, 0>(p, pdl, s);
    case 8: return down_dispatch<BITS, 8, 0>(p, pdl, s);
    case 16: return down_dispatch<BITS, 16, 0>(p, pdl, s);
    case 32: return down_dispatch<BITS, 32, 0>(p, pdl, s);
    case 64: return down_dispatch<BITS, 64, 0>(p, pdl, s);
    case 128: return down_dispatch<BITS, 128, 0>(p, pdl, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

// Asks for the largest shared-memory carveout for a kernel, once per (kernel, device):
// kernels that sit on an SM together under dependent launch must run with the same
// carveout, else the later one waits for the SM to drain before it can start there.
cudaError_t set_carveout_max(const void* kernel) {
  static const void* done[64][32] = {};
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  if (dev < 0 || dev >= 64) return cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  for (const void*& k : done[dev]) {
    if (k == kernel) return cudaSuccess;
    if (k == nullptr) {
      e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
      if (e == cudaSuccess) k = kernel;
      return e;
    }
  }
  return cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
}

// Raises a kernel's dynamic shared-memory limit once per (kernel, device), and
// again only if a larger size is asked for, so that launches captured into a
// CUDA graph make no attribute call.
cudaError_t set_smem(const void* kernel, size_t bytes) {
  struct Entry {
    const void* fn;
    size_t bytes[64];
  };
  static Entry table[96] = {};
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (bytes <= 32 * 1024) return cudaSuccess;  // below the default limit even with static shared memory
  std::lock_guard<std::mutex> lock(mu);
  Entry* slot = nullptr;
  for (Entry& t : table) {
    if (t.fn == kernel || t.fn == nullptr) {
      slot = &t;
      break;
    }
  }
  if (slot && slot->fn == kernel && dev >= 0 && dev < 64 && slot->bytes[dev] >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess && slot && dev >= 0 && dev < 64) {
    slot->fn = kernel;
    slot->bytes[dev] = bytes;
  }
  return e;
}

namespace {
template <int BITS, int NGU, int NGD>
bool fits(int ne) {
  int cu, nb;
  size_t sm;
  return GuCfg<BITS, NGU>::kHead + GuCfg<BITS, NGU>::kChunkBytes <= kGuSmemBudget &&
         down_plan<BITS, NGD>(1 << 20, ne, cu, nb, sm) && ne * NGD <= 4 * 32;
}
template <int BITS, int NGU>
bool fits_d(int ngd, int ne) {
  switch (ngd) {
    case 2: return fits<BITS, NGU, 2>(ne);
    case 4: return fits<BITS, NGU, 4>(ne);
    case 8: return fits<BITS, NGU, 8>(ne);
    case 16: return fits<BITS, NGU, 16>(ne);
    case 32: return fits<BITS, NGU, 32>(ne);
    case 64: return fits<BITS, NGU, 64>(ne);
    case 128: return fits<BITS, NGU, 128>(ne);
  }
  return false;
}
template <int BITS>
bool fits_u(int ngu, int ngd, int ne) {
  switch (ngu) {
    case 2: return fits_d<BITS, 2>(ngd, ne);
    case 4: return fits_d<BITS, 4>(ngd, ne);
    case 8: return fits_d<BITS, 8>(ngd, ne);
    case 16: return fits_d<BITS, 16>(ngd, ne);
    case 32: return fits_d<BITS, 32>(ngd, ne);
    case 64: return fits_d<BITS, 64>(ngd, ne);
    case 128: return fits_d<BITS, 128>(ngd, ne);
  }
  return false;
}
}  // namespace

bool expert_shapes_supported(int bits, int H, int I, int ne) {
  if (H % kGroup || I % kGroup) return false;
  return bits == 8   ? fits_u<8>(H / kGroup, I / kGroup, ne)
         : bits == 4 ? fits_u<4>(H / kGroup, I / kGroup, ne)
                     : fits_u<2>(H / kGroup, I / kGroup, ne);
}

cudaError_t launch_wait_flag(const unsigned int* flag, unsigned int value, unsigned long long limit_ns, int* err,
                             cudaStream_t s) {
  wait_flag_kernel<<<1, 1, 0, s>>>(flag, value, limit_ns, err);
  return cudaGetLastError();
}

// Weight of a shared-expert unit in the gate/up split, in eighths of a routed unit
// (FMOE_GU_SHARED_WEIGHT, 1..8; 8, the even split, unless set).
static int gu_shared_weight() {
  static const int w = [] {  // read once (thread-safe static initialisation)
    const char* v = getenv("FMOE_GU_SHARED_WEIGHT");
    const int x = v ? atoi(v) : 8;
    return x >= 1 && x <= 8 ? x : 8;
  }();
  return w;
}

cudaError_t launch_gateup(const ExpertParams& p, int bits, bool pdl, cudaStream_t s) {
  ExpertParams q = p;
  q.gu_sw = gu_shared_weight();
  return bits == 8 ? gateup_bits<8>(q, pdl, s) : bits == 4 ? gateup_bits<4>(q, pdl, s) : gateup_bits<2>(q, pdl, s);
}

cudaError_t launch_down(const ExpertParams& p, int bits, bool pdl, cudaStream_t s) {
  return bits == 8 ? down_bits<8>(p, pdl, s) : bits == 4 ? down_bits<4>(p, pdl, s) : down_bits<2>(p, pdl, s);
}

}  // namespace fmoe
