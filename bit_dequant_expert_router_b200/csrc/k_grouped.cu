// k_grouped.cu -- the MoE block for a batch of T decode tokens, grouped by expert.
//
// Per step the batch selects up to T*K (expert, token) pairs over at most
// min(E, T*K) distinct experts.  Running the tokens one after another would
// read an expert's weights once per token that picked it; here the pairs are
// sorted by expert (counting sort, ties in (token, k) order) and every active
// expert's gate/up and down rows are read once for its whole token group.
// The shared expert is an active expert whose group is the whole batch.
// Results are scattered back with the renormalised top-K weights in fixed k
// order, so the output does not depend on the grouping.
//
// Kernels, in stream order after the router (which already writes the logits
// and the digits of x of every token):
//   select  : top-K per token, the sorted pair list and the active experts
//   gate/up : one CTA per (active expert, block of rows): stage the rows once,
//             then gate/up + SwiGLU for each token of the group
//   actq    : digits of every pair's activations (fmoe_device.cuh format)
//   down    : one CTA per (active expert, block of output rows), same scheme
//   combine : out[t] = h[t] + sum_k w_tk y[pair(t,k)] + sigma_t y_shared[t]
// Dequant dot products use the per-group fold sum_c (q s + b) x = s*sum q x + b*sum x
// with exact dp4a sums ("What is Flash-MoE", sections 2-3, for the block itself).
#include "fmoe_internal.h"

namespace fmoe {
namespace {

constexpr int kGT = 256;          // threads per CTA
constexpr int kGuRows = 16;       // gate/up row pairs per CTA
constexpr int kGuTok = 2;         // tokens whose digits are staged at once (gate/up)
constexpr int kDnRows = 32;       // down output rows per CTA
constexpr int kDnTok = 16;        // tokens whose activation digits are staged at once (down)
constexpr int kMaxTK = 4096;      // T*K pairs
constexpr int kRtRows = 8;        // router rows per CTA (batched router)
constexpr int kRtTok = 16;        // tokens per CTA (batched router)

// ---- selection, in two kernels.  topk: one CTA per token, the block-wide
// two-stage top-K (ties to the lower index) with renormalised weights and the
// shared-gate sigma.
__global__ void __launch_bounds__(kGT) topk_tokens_kernel(const GroupedParams p) {
  __shared__ int s_idx[32];
  __shared__ float s_w[33];
  __shared__ unsigned long long s_cand[8 * 32];
  const int t = blockIdx.x, tid = threadIdx.x, K = p.K, E = p.E;
  block_topk(p.logits + (size_t)t * (E + 1), E, K, 1, s_cand, s_idx, s_w);
  if (tid < K) {
    int e = s_idx[tid];
    e = (e < 0 || e >= E) ? 0 : e;
    p.route_idx[(size_t)t * K + tid] = e;
    p.route_w[(size_t)t * (K + 1) + tid] = s_w[tid];
    if (p.idx_out) p.idx_out[(size_t)t * K + tid] = e;
    if (p.w_out) p.w_out[(size_t)t * K + tid] = s_w[tid];
  }
  if (tid == K) p.route_w[(size_t)t * (K + 1) + K] = s_w[K];
}

constexpr int kST = 1024;  // threads of the sort kernel

// Exclusive block-wide scan of one value per thread (kST threads); returns the
// exclusive prefix and writes the total to *total.
__device__ __forceinline__ int block_scan_excl(int v, int* s_warp, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) s_warp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < kST / 32 ? s_warp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < kST / 32) s_warp[lane] = w;  // inclusive warp totals
  }
  __syncthreads();
  const int before = warp ? s_warp[warp - 1] : 0;
  *total = s_warp[kST / 32 - 1];
  __syncthreads();
  return before + x - v;
}

// sort: one CTA.  Counting sort of the T*K pairs by expert, stable in (token, k)
// order: the rank of pair i among the pairs of its expert is the number of
// earlier pairs with the same expert.  Active experts in increasing order.
__global__ void __launch_bounds__(kST) sort_pairs_kernel(const GroupedParams p) {
  extern __shared__ __align__(16) int s_mem[];  // [T*K] experts of the pairs, [E] counts, [E] starts
  __shared__ int s_warp[kST / 32];
  const int tid = threadIdx.x, N = p.T * p.K, E = p.E;
  int* s_e = s_mem;
  int* s_cnt = s_mem + N;
  int* s_start = s_cnt + E;
  for (int e = tid; e < E; e += kST) s_cnt[e] = 0;
  __syncthreads();
  for (int i = tid; i < N; i += kST) {
    const int e = __ldcg(p.route_idx + i);
    s_e[i] = e;
    atomicAdd(&s_cnt[e], 1);
  }
  __syncthreads();
  // starts of the experts (exclusive scan of the counts) and slots of the active ones
  const int per = (E + kST - 1) / kST;  // experts per thread, contiguous
  int c = 0, a = 0;
  for (int k = 0; k < per; ++k) {
    const int e = tid * per + k;
    if (e < E) {
      c += s_cnt[e];
      a += s_cnt[e] > 0;
    }
  }
  int tot_c, tot_a;
  int run = block_scan_excl(c, s_warp, &tot_c);
  int slot = block_scan_excl(a, s_warp, &tot_a);
  for (int k = 0; k < per; ++k) {
    const int e = tid * per + k;
    if (e < E) {
      s_start[e] = run;
      if (s_cnt[e] > 0) {
        p.act_expert[slot] = e;
        p.act_off[slot] = run;
        ++slot;
      }
      run += s_cnt[e];
    }
  }
  if (tid == 0) {
    p.act_off[tot_a] = tot_c;
    *p.n_active = tot_a;
  }
  __syncthreads();
  for (int i = tid; i < N; i += kST) {
    const int e = s_e[i];
    int rank = 0;
    for (int j = 0; j < i; ++j) rank += s_e[j] == e;
    const int pos = s_start[e] + rank;
    p.pair_tok[pos] = i;
    p.pair_pos[i] = pos;
  }
}

// ---- router for the batch.  norm_digits: one CTA per token, x = RMSNorm(h)
// (two passes) in fp32 for the router and as digits for the experts.
__global__ void __launch_bounds__(kGT) norm_digits_kernel(const GroupedParams p, const RouterBatch rb, int bits) {
  __shared__ float s_red[kGT / 32];
  const int t = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, H = p.H;
  const float* h = p.h + (size_t)t * H;
  float* x = rb.x + (size_t)t * H;
  float ss = 0.0f;
  for (int i = tid * 4; i < H; i += kGT * 4) {
    const float4 v = __ldcg(reinterpret_cast<const float4*>(h + i));
    ss = fmaf(v.x, v.x, fmaf(v.y, v.y, fmaf(v.z, v.z, fmaf(v.w, v.w, ss))));
  }
  float rstd = 1.0f;
  if (rb.gamma) {
    ss = warp_sum(ss);
    if (lane == 0) s_red[warp] = ss;
    __syncthreads();
    float tot = 0.0f;
#pragma unroll
    for (int w = 0; w < kGT / 32; ++w) tot += s_red[w];
    rstd = 1.0f / sqrtf(tot / (float)H + rb.eps);
  }
  for (int i = tid * 4; i < H; i += kGT * 4) {
    float4 v = __ldcg(reinterpret_cast<const float4*>(h + i));
    if (rb.gamma) {
      const float4 g = __ldg(reinterpret_cast<const float4*>(rb.gamma + i));
      v = make_float4(v.x * rstd * g.x, v.y * rstd * g.y, v.z * rstd * g.z, v.w * rstd * g.w);
    }
    *reinterpret_cast<float4*>(x + i) = v;
  }
  __syncthreads();  // this CTA's x is written (read back through L1-bypassing loads below)
  __threadfence_block();
  uint8_t* limbs = const_cast<uint8_t*>(p.xq_limbs) + (size_t)t * 3 * H;
  float2* cs = const_cast<float2*>(p.xq_cs) + (size_t)t * (H / 32);
  for (int g = warp; g < H / kGroup; g += kGT / 32) {
    const float2 v = __ldcg(reinterpret_cast<const float2*>(x + g * kGroup) + lane);
    if (bits == 4)
      xq_quantize_group<4>(v.x, v.y, g, H / kGroup, limbs, cs);
    else
      xq_quantize_group<2>(v.x, v.y, g, H / kGroup, limbs, cs);
  }
}

// router_gemm: CTA (a, b) computes logits of rows [8a, 8a+8) of [W_r; w_sg] for
// tokens [16b, 16b+16): the rows are staged once, x of each token streams from
// L2.  Warp w sums column slice w (H/8 columns); the 8 slice sums add in fixed order.
__global__ void __launch_bounds__(kGT) router_gemm_kernel(const GroupedParams p, const RouterBatch rb) {
  extern __shared__ __align__(128) uint8_t sm[];
  __shared__ float s_part[kRtTok][kRtRows][kGT / 32];
  __shared__ __align__(8) uint64_t s_bar;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, H = p.H, E = p.E;
  const int r0 = blockIdx.x * kRtRows, n = min(kRtRows, E + 1 - r0);
  const int t0 = blockIdx.y * kRtTok, nt = min(kRtTok, p.T - t0);
  uint16_t* w = reinterpret_cast<uint16_t*>(sm);
  if (tid == 0) {
    const uint32_t bar = smem_addr(&s_bar);
    mbar_init(bar, 1);
    mbar_fence_init();
    const int nr = max(0, min(n, E - r0));  // rows of w_router; the rest is the shared-gate row
    mbar_expect_tx(bar, (uint32_t)n * H * 2);
    if (nr > 0) bulk_g2s(smem_addr(w), rb.w_router + (size_t)r0 * H, (uint32_t)nr * H * 2, bar, l2_policy_evict_first());
    if (nr < n) bulk_g2s(smem_addr(w + (size_t)nr * H), rb.w_sgate, (uint32_t)H * 2, bar, l2_policy_evict_first());
  }
  __syncthreads();
  const bool ok = mbar_wait_bounded(smem_addr(&s_bar), 0, p.err);
  const uint16_t* ws = w + warp * (H / 8);
  for (int j = 0; ok && j < nt; ++j) {
    const float* xs = rb.x + (size_t)(t0 + j) * H + warp * (H / 8);
    float acc[kRtRows];
#pragma unroll
    for (int r = 0; r < kRtRows; ++r) acc[r] = 0.0f;
    for (int k = lane; k < H / 64; k += 32) {
      const float4 xa = __ldcg(reinterpret_cast<const float4*>(xs + 8 * k));
      const float4 xb = __ldcg(reinterpret_cast<const float4*>(xs + 8 * k + 4));
#pragma unroll
      for (int r = 0; r < kRtRows; ++r) {
        if (r < n) {
          const uint4 q = *reinterpret_cast<const uint4*>(ws + (size_t)r * H + 8 * k);
          float a = acc[r];
          a = fmaf(__uint_as_float(q.x << 16), xa.x, a);
          a = fmaf(__uint_as_float(q.x & 0xFFFF0000u), xa.y, a);
          a = fmaf(__uint_as_float(q.y << 16), xa.z, a);
          a = fmaf(__uint_as_float(q.y & 0xFFFF0000u), xa.w, a);
          a = fmaf(__uint_as_float(q.z << 16), xb.x, a);
          a = fmaf(__uint_as_float(q.z & 0xFFFF0000u), xb.y, a);
          a = fmaf(__uint_as_float(q.w << 16), xb.z, a);
          a = fmaf(__uint_as_float(q.w & 0xFFFF0000u), xb.w, a);
          acc[r] = a;
        }
      }
    }
#pragma unroll
    for (int r = 0; r < kRtRows; ++r) acc[r] = warp_sum(acc[r]);
    if (lane == 0)
#pragma unroll
      for (int r = 0; r < kRtRows; ++r) s_part[j][r][warp] = acc[r];
  }
  __syncthreads();
  for (int i = tid; ok && i < nt * n; i += kGT) {
    const int j = i / n, r = i % n;
    float l = 0.0f;
#pragma unroll
    for (int q = 0; q < kGT / 32; ++q) l += s_part[j][r][q];
    const int row = r0 + r;
    if (row < E && rb.bias) l += rb.bias[row];
    const_cast<float*>(p.logits)[(size_t)(t0 + j) * (E + 1) + row] = l;
  }
}

// The group of CTA slot u (u == 0: the shared expert, every token, scheduled
// first because its groups are the largest; u >= 1: active expert u - 1):
// record, number of tokens, and for token j its token index and output row.
struct Group {
  const uint8_t* rec;
  const long long* off;
  int n;      // tokens in the group
  int first;  // routed: first sorted pair; shared: -1
};

__device__ __forceinline__ Group group_of(const GroupedParams& p, int u, int U) {
  Group g;
  (void)U;
  if (u == 0) {
    g.rec = p.shared.base;
    g.off = p.shared.off;
    g.n = p.T;
    g.first = -1;
  } else {
    const int e = __ldcg(p.act_expert + u - 1);
    g.rec = p.routed.base + (long long)e * p.routed.stride;
    g.off = p.routed.off;
    g.first = __ldcg(p.act_off + u - 1);
    g.n = __ldcg(p.act_off + u) - g.first;
  }
  return g;
}

// token and output row (into act / y) of member j of a group
__device__ __forceinline__ void member(const GroupedParams& p, const Group& g, int j, int& tok, int& row) {
  if (g.first < 0) {
    tok = j;
    row = p.T * p.K + j;
  } else {
    const int pr = __ldcg(p.pair_tok + g.first + j);
    tok = pr / p.K;
    row = g.first + j;
  }
}


// ---- gate/up + SwiGLU: CTA (u, b) = active expert slot u, row pairs [16b, 16b+16).
// The rows are staged once; the digits of x of kGuTok tokens of the group at a
// time.  Lane geometry as in the per-token kernel (Geo<NG>): a lane owns GPL
// groups of 64 columns, a warp one row pair per pass (RPP when NG < 32).
template <int BITS, int NG>
__global__ void __launch_bounds__(kGT) grouped_gateup_kernel(const GroupedParams p) {
  using G = Geo<NG>;
  constexpr int LPR = G::kLanesPerRow, RPP = G::kRowsPerPass, GPL = G::kGroupsPerLane;
  constexpr int RB = NG * kGroup * BITS / 8, SB = NG * 2;
  constexpr int NCX = NG * kGroup * BITS / 128;              // chunk scalars of x
  constexpr int DIG = NG * kGroupWords * 4 + NCX * 8;        // staged bytes per token
  constexpr int WB = kGuRows * (2 * RB + 4 * SB);            // staged weight bytes
  extern __shared__ __align__(128) uint8_t sm[];
  __shared__ __align__(8) uint64_t s_wbar;
  __shared__ __align__(8) uint64_t s_dbar;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int U = __ldcg(p.n_active);
  const int u = blockIdx.x;
  if (u > U) return;  // block-uniform
  const Group grp = group_of(p, u, U);
  const int H = p.H, I = p.I;
  const int r0 = blockIdx.y * kGuRows;
  uint8_t* dbuf = sm + WB;
  const uint64_t pol = l2_policy_evict_first();
  if (tid == 0) {
    mbar_init(smem_addr(&s_wbar), 1);
    mbar_init(smem_addr(&s_dbar), 1);
    mbar_fence_init();
    const uint32_t bw = smem_addr(&s_wbar), dst = smem_addr(sm);
    const uint32_t cb = kGuRows * RB, sbb = kGuRows * SB;
    mbar_expect_tx(bw, 2 * cb + 4 * sbb);
    bulk_g2s(dst, grp.rec + grp.off[0] + (long long)r0 * RB, cb, bw, pol);
    bulk_g2s(dst + cb, grp.rec + grp.off[3] + (long long)r0 * RB, cb, bw, pol);
    bulk_g2s(dst + 2 * cb, grp.rec + grp.off[1] + (long long)r0 * SB, sbb, bw, pol);
    bulk_g2s(dst + 2 * cb + sbb, grp.rec + grp.off[2] + (long long)r0 * SB, sbb, bw, pol);
    bulk_g2s(dst + 2 * cb + 2 * sbb, grp.rec + grp.off[4] + (long long)r0 * SB, sbb, bw, pol);
    bulk_g2s(dst + 2 * cb + 3 * sbb, grp.rec + grp.off[5] + (long long)r0 * SB, sbb, bw, pol);
  }
  __syncthreads();
  bool ok = mbar_wait_bounded(smem_addr(&s_wbar), 0, p.err);
  const int sub = lane / LPR, gl = lane % LPR;
  const uint16_t* scl = reinterpret_cast<const uint16_t*>(sm + 2 * kGuRows * RB);
  for (int j0 = 0, it = 0; j0 < grp.n; j0 += kGuTok, ++it) {
    const int nb = min(kGuTok, grp.n - j0);
    if (tid == 0) {
      const uint32_t bd = smem_addr(&s_dbar);
      fence_proxy_async();
      mbar_expect_tx(bd, (uint32_t)nb * DIG);
      for (int jj = 0; jj < nb; ++jj) {
        int tok, row;
        member(p, grp, j0 + jj, tok, row);
        bulk_g2s(smem_addr(dbuf + jj * DIG), p.xq_limbs + (size_t)tok * 3 * H, NG * kGroupWords * 4, bd, pol);
        bulk_g2s(smem_addr(dbuf + jj * DIG + NG * kGroupWords * 4), p.xq_cs + (size_t)tok * (H / 32), NCX * 8, bd, pol);
      }
    }
    if (!mbar_wait_bounded(smem_addr(&s_dbar), (uint32_t)(it & 1), p.err)) ok = false;
    for (int jj = 0; ok && jj < nb; ++jj) {
      int tok, row;
      member(p, grp, j0 + jj, tok, row);
      const uint32_t* xl = reinterpret_cast<const uint32_t*>(dbuf + jj * DIG);
      const float2* xc = reinterpret_cast<const float2*>(dbuf + jj * DIG + NG * kGroupWords * 4);
      uint32_t L[GPL][48];
      float2 cs[GPL];
#pragma unroll
      for (int q = 0; q < GPL; ++q) {
        load_group_limbs(xl, gl + LPR * q, NG, L[q]);
        cs[q] = group_scalars<BITS>(xc, gl + LPR * q);
      }
      for (int pr = warp; pr * RPP < kGuRows; pr += kGT / 32) {
        const int r = pr * RPP + sub;  // row pair within the block
        float ag = 0.0f, au = 0.0f;
#pragma unroll
        for (int q = 0; q < GPL; ++q) {
          const int g = gl + LPR * q;
          uint4 q0, q1, v0, v1;
          load_group_codes<BITS>(sm + r * RB, g, q0, q1);
          load_group_codes<BITS>(sm + kGuRows * RB + r * RB, g, v0, v1);
          const float gs = bf16_to_f32(scl[r * NG + g]), gb = bf16_to_f32(scl[kGuRows * NG + r * NG + g]);
          const float us = bf16_to_f32(scl[2 * kGuRows * NG + r * NG + g]);
          const float ub = bf16_to_f32(scl[3 * kGuRows * NG + r * NG + g]);
          const float Sg = group_dot<BITS>(q0, q1, L[q]);
          const float Su = group_dot<BITS>(v0, v1, L[q]);
          ag = fmaf(gs, cs[q].x * Sg, fmaf(gb, cs[q].y, ag));
          au = fmaf(us, cs[q].x * Su, fmaf(ub, cs[q].y, au));
        }
        for (int o = LPR / 2; o > 0; o >>= 1) {
          ag += __shfl_xor_sync(0xffffffffu, ag, o);
          au += __shfl_xor_sync(0xffffffffu, au, o);
        }
        if (gl == 0) p.act[(size_t)row * I + r0 + r] = ag / (1.0f + expf(-ag)) * au;
      }
    }
    __syncthreads();  // the digit buffer is free for the next tokens
  }
}

// ---- activation digits of every sorted pair and every shared-expert token: one warp per group of 64
template <int BITS>
__global__ void __launch_bounds__(kGT) grouped_actq_kernel(const GroupedParams p) {
  const int I = p.I, NGI = I / kGroup;
  const int gw = blockIdx.x * (kGT / 32) + (threadIdx.x >> 5);
  if (gw >= (p.T * p.K + p.T) * NGI) return;  // warp-uniform
  const int row = gw / NGI, g = gw % NGI;
  const float2 v = __ldcg(reinterpret_cast<const float2*>(p.act + (size_t)row * I + g * kGroup) + (threadIdx.x & 31));
  xq_quantize_group<BITS>(v.x, v.y, g, NGI, p.act_limbs + (size_t)row * 3 * I, p.act_cs + (size_t)row * (I / 32));
}

// ---- down: CTA (u, b) = active expert slot u, output rows [32b, 32b+32).  The
// rows are staged once, the activation digits of up to `tb` group members at a
// time; y[member row][h] holds the unweighted down output.
template <int BITS, int NG>
__global__ void __launch_bounds__(kGT) grouped_down_kernel(const GroupedParams p, int tb) {
  using G = Geo<NG>;
  constexpr int LPR = G::kLanesPerRow, RPP = G::kRowsPerPass, GPL = G::kGroupsPerLane;
  constexpr int RB = NG * kGroup * BITS / 8, SB = NG * 2;
  constexpr int NCA = NG * kGroup * BITS / 128;
  constexpr int DIG = NG * kGroupWords * 4 + NCA * 8;
  constexpr int WB = kDnRows * (RB + 2 * SB);
  extern __shared__ __align__(128) uint8_t sm[];
  __shared__ __align__(8) uint64_t s_wbar;
  __shared__ __align__(8) uint64_t s_dbar;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int U = __ldcg(p.n_active);
  const int u = blockIdx.x;
  if (u > U) return;
  const Group grp = group_of(p, u, U);
  const int H = p.H, I = p.I;
  const int d0 = blockIdx.y * kDnRows;
  uint8_t* dbuf = sm + WB;
  const uint64_t pol = l2_policy_evict_first();
  if (tid == 0) {
    mbar_init(smem_addr(&s_wbar), 1);
    mbar_init(smem_addr(&s_dbar), 1);
    mbar_fence_init();
    const uint32_t bw = smem_addr(&s_wbar), dst = smem_addr(sm);
    mbar_expect_tx(bw, kDnRows * (RB + 2 * SB));
    bulk_g2s(dst, grp.rec + grp.off[6] + (long long)d0 * RB, kDnRows * RB, bw, pol);
    bulk_g2s(dst + kDnRows * RB, grp.rec + grp.off[7] + (long long)d0 * SB, kDnRows * SB, bw, pol);
    bulk_g2s(dst + kDnRows * (RB + SB), grp.rec + grp.off[8] + (long long)d0 * SB, kDnRows * SB, bw, pol);
  }
  __syncthreads();
  bool ok = mbar_wait_bounded(smem_addr(&s_wbar), 0, p.err);
  const int sub = lane / LPR, gl = lane % LPR;
  const uint16_t* scl = reinterpret_cast<const uint16_t*>(sm + kDnRows * RB);
  const uint16_t* bsl = reinterpret_cast<const uint16_t*>(sm + kDnRows * (RB + SB));
  for (int j0 = 0, it = 0; j0 < grp.n; j0 += tb, ++it) {
    const int nb = min(tb, grp.n - j0);
    if (tid == 0) {
      const uint32_t bd = smem_addr(&s_dbar);
      fence_proxy_async();
      mbar_expect_tx(bd, (uint32_t)nb * DIG);
      for (int jj = 0; jj < nb; ++jj) {
        int tok, row;
        member(p, grp, j0 + jj, tok, row);
        bulk_g2s(smem_addr(dbuf + jj * DIG), p.act_limbs + (size_t)row * 3 * I, NG * kGroupWords * 4, bd, pol);
        bulk_g2s(smem_addr(dbuf + jj * DIG + NG * kGroupWords * 4), p.act_cs + (size_t)row * (I / 32), NCA * 8, bd, pol);
      }
    }
    if (!mbar_wait_bounded(smem_addr(&s_dbar), (uint32_t)(it & 1), p.err)) ok = false;
    for (int jj = 0; ok && jj < nb; ++jj) {
      int tok, row;
      member(p, grp, j0 + jj, tok, row);
      const uint32_t* al = reinterpret_cast<const uint32_t*>(dbuf + jj * DIG);
      const float2* ac = reinterpret_cast<const float2*>(dbuf + jj * DIG + NG * kGroupWords * 4);
      uint32_t L[GPL][48];
      float2 cs[GPL];
#pragma unroll
      for (int q = 0; q < GPL; ++q) {
        load_group_limbs(al, gl + LPR * q, NG, L[q]);
        cs[q] = group_scalars<BITS>(ac, gl + LPR * q);
      }
      for (int pr = warp; pr * RPP < kDnRows; pr += kGT / 32) {
        const int r = pr * RPP + sub;
        float acc = 0.0f;
#pragma unroll
        for (int q = 0; q < GPL; ++q) {
          const int g = gl + LPR * q;
          uint4 q0, q1;
          load_group_codes<BITS>(sm + r * RB, g, q0, q1);
          const float sc = bf16_to_f32(scl[r * NG + g]), bi = bf16_to_f32(bsl[r * NG + g]);
          const float S = group_dot<BITS>(q0, q1, L[q]);
          acc = fmaf(sc, cs[q].x * S, fmaf(bi, cs[q].y, acc));
        }
        for (int o = LPR / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (gl == 0) p.y[(size_t)row * H + d0 + r] = acc;
      }
    }
    __syncthreads();
  }
}

// ---- combine, fixed k order: out[t] = h[t] + sum_k w_tk y[pair(t,k)] + sigma_t y_shared[t]
__global__ void __launch_bounds__(kGT) grouped_combine_kernel(const GroupedParams p) {
  const int t = blockIdx.y, h = blockIdx.x * kGT + threadIdx.x;
  if (h >= p.H) return;
  const int K = p.K;
  float acc = 0.0f;
  for (int k = 0; k < K; ++k) {
    const int pos = __ldcg(p.pair_pos + (size_t)t * K + k);
    acc = fmaf(__ldcg(p.route_w + (size_t)t * (K + 1) + k), __ldcg(p.y + (size_t)pos * p.H + h), acc);
  }
  acc = fmaf(__ldcg(p.route_w + (size_t)t * (K + 1) + K), __ldcg(p.y + (size_t)(p.T * K + t) * p.H + h), acc);
  p.out[(size_t)t * p.H + h] = p.h[(size_t)t * p.H + h] + acc;
}

size_t gu_smem(int bits, int H) {
  const int NG = H / kGroup, RB = H * bits / 8, SB = NG * 2;
  return (size_t)kGuRows * (2 * RB + 4 * SB) + (size_t)kGuTok * (NG * kGroupWords * 4 + (H * bits / 128) * 8);
}

// down: staged rows + as many members' digits as fit (at most kDnTok)
int dn_tokens(int bits, int I, size_t* smem) {
  const int NG = I / kGroup, RB = I * bits / 8, SB = NG * 2;
  const size_t wb = (size_t)kDnRows * (RB + 2 * SB), dig = (size_t)NG * kGroupWords * 4 + (size_t)(I * bits / 128) * 8;
  const size_t budget = 220 * 1024;
  if (wb + dig > budget) return 0;
  size_t tb = (budget - wb) / dig;
  tb = tb > (size_t)kDnTok ? (size_t)kDnTok : tb;
  *smem = wb + tb * dig;
  return (int)tb;
}

template <int BITS>
cudaError_t gateup_bits_g(const GroupedParams& p, cudaStream_t s) {
  void (*k)(const GroupedParams) = nullptr;
  switch (p.H / kGroup) {
    case 2: k = grouped_gateup_kernel<BITS, 2>; break;
    case 4: k = grouped_gateup_kernel<BITS, 4>; break;
    case 8: k = grouped_gateup_kernel<BITS, 8>; break;
    case 16: k = grouped_gateup_kernel<BITS, 16>; break;
    case 32: k = grouped_gateup_kernel<BITS, 32>; break;
    case 64: k = grouped_gateup_kernel<BITS, 64>; break;
    case 128: k = grouped_gateup_kernel<BITS, 128>; break;
    default: return cudaErrorInvalidValue;
  }
  const size_t smem = gu_smem(BITS, p.H);
  cudaError_t e = set_smem((const void*)k, smem);
  if (e != cudaSuccess) return e;
  const int umax = (p.E < p.T * p.K ? p.E : p.T * p.K) + 1;
  k<<<dim3(umax, p.I / kGuRows), kGT, smem, s>>>(p);
  return cudaGetLastError();
}

template <int BITS>
cudaError_t down_bits_g(const GroupedParams& p, cudaStream_t s) {
  void (*k)(const GroupedParams, int) = nullptr;
  switch (p.I / kGroup) {
    case 2: k = grouped_down_kernel<BITS, 2>; break;
    case 4: k = grouped_down_kernel<BITS, 4>; break;
    case 8: k = grouped_down_kernel<BITS, 8>; break;
    case 16: k = grouped_down_kernel<BITS, 16>; break;
    case 32: k = grouped_down_kernel<BITS, 32>; break;
    case 64: k = grouped_down_kernel<BITS, 64>; break;
    case 128: k = grouped_down_kernel<BITS, 128>; break;
    default: return cudaErrorInvalidValue;
  }
  size_t smem = 0;
  const int tb = dn_tokens(BITS, p.I, &smem);
  if (tb < 1) return cudaErrorInvalidValue;
  cudaError_t e = set_smem((const void*)k, smem);
  if (e != cudaSuccess) return e;
  const int umax = (p.E < p.T * p.K ? p.E : p.T * p.K) + 1;
  k<<<dim3(umax, p.H / kDnRows), kGT, smem, s>>>(p, tb);
  return cudaGetLastError();
}

}  // namespace

bool grouped_shapes_supported(int bits, int H, int I, int E, int K, int T) {
  if (T * K > kMaxTK || ((size_t)T * K + 2 * (size_t)E) * 4 > 200 * 1024) return false;
  if ((size_t)kRtRows * H * 2 > 200 * 1024) return false;
  if (H % kDnRows || I % kGuRows) return false;
  size_t smem = 0;
  return gu_smem(bits, H) <= 220 * 1024 && dn_tokens(bits, I, &smem) >= 1;
}

cudaError_t launch_grouped_select(const GroupedParams& p, cudaStream_t s) {
  topk_tokens_kernel<<<p.T, kGT, 0, s>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t smem = ((size_t)p.T * p.K + 2 * (size_t)p.E) * sizeof(int);
  if ((e = set_smem((const void*)sort_pairs_kernel, smem)) != cudaSuccess) return e;
  sort_pairs_kernel<<<1, kST, smem, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_grouped_router(const GroupedParams& p, const RouterBatch& rb, int bits, cudaStream_t s) {
  norm_digits_kernel<<<p.T, kGT, 0, s>>>(p, rb, bits);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int R = p.E + 1;
  const size_t smem = (size_t)kRtRows * p.H * 2;
  void (*k)(const GroupedParams, const RouterBatch) = router_gemm_kernel;
  if ((e = set_smem((const void*)k, smem)) != cudaSuccess) return e;
  k<<<dim3((R + kRtRows - 1) / kRtRows, (p.T + kRtTok - 1) / kRtTok), kGT, smem, s>>>(p, rb);
  return cudaGetLastError();
}

cudaError_t launch_grouped_gateup(const GroupedParams& p, int bits, cudaStream_t s) {
  return bits == 4 ? gateup_bits_g<4>(p, s) : gateup_bits_g<2>(p, s);
}

cudaError_t launch_grouped_actq(const GroupedParams& p, int bits, cudaStream_t s) {
  const int warps = (p.T * p.K + p.T) * (p.I / kGroup);
  const int grid = (warps + kGT / 32 - 1) / (kGT / 32);
  if (bits == 4)
    grouped_actq_kernel<4><<<grid, kGT, 0, s>>>(p);
  else
    grouped_actq_kernel<2><<<grid, kGT, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_grouped_down(const GroupedParams& p, int bits, cudaStream_t s) {
  return bits == 4 ? down_bits_g<4>(p, s) : down_bits_g<2>(p, s);
}

cudaError_t launch_grouped_combine(const GroupedParams& p, cudaStream_t s) {
  grouped_combine_kernel<<<dim3((p.H + kGT - 1) / kGT, p.T), kGT, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace fmoe
