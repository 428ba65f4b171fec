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
// Kernels, in stream order:
//   norm_digits : x = RMSNorm(h) per token (fp32 for the router) and its digits
//   router_gemm : partial logits of [W_r; w_sg] x as a split-K tiled product
//   topk_tokens : the slice sums in order, the top-K and weights per token
//   sort_pairs  : the sorted pair list, the active experts and the work units
//                 (runs of at most kUnitToks members of one expert's group)
//   gate/up     : persistent, one CTA per SM; a producer warp stages each item
//                 (a block of rows of one unit's expert) by TMA tensor copies,
//                 eight consumer warps contract it with the members' digits
//                 on the int8 tensor cores (mma.sync) and apply SwiGLU
//   actq        : digits of every member's activations
//   down        : the same scheme over blocks of output rows
//   combine     : out[t] = h[t] + sum_k w_tk y[pair(t,k)] + sigma_t y_shared[t]
// The dequant products use the per-group fold sum_c (q s + b) x = s*sum q x + b*sum x
// with exact integer sums of codes times fixed-point digits of x ("What is
// Flash-MoE", sections 2-3, for the block itself).
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "fmoe_internal.h"

namespace fmoe {
namespace {

// The grouped path's kernels are chained by dependent launch: each waits for its
// predecessor to complete (its writes visible) before anything else, and only then lets
// its successor launch.  At most two kernels of the chain are resident, and the waiting
// one never holds resources that a CTA of its predecessor still needs; what is saved is
// the successor's launch latency.  Every kernel waits, so completion is transitive.
__device__ __forceinline__ void pdl_chain() {
  pdl_wait();
  pdl_trigger();
}

constexpr int kGT = 256;          // threads per CTA
constexpr int kMaxTK = 4096;      // T*K pairs

// ---- int8 tensor-core contraction of codes with activation digits.
// The batched expert products run on mma.sync m16n8k32 (u8 codes x s8 digits,
// s32 accumulate).  A tile is 16 weight rows x 8 columns, a column being one
// limb of one token's digits (3 limbs per token, two tokens per tile); K runs
// over one group of 64 in two k-blocks of 32, so that every group's int32 sums
// are scaled on their own (s * cscale * S + b * sum x, per the fold above).
//
// Lane (gid, q) of the quad layout (gid = lane / 4, q = lane % 4) holds the A
// registers {row gid k-lo, row gid+8 k-lo, row gid k-hi, row gid+8 k-hi} and the
// B registers {k-lo, k-hi} of column gid, k-lo being k-slots 4q..4q+3 and k-hi
// 16+4q..16+4q+3 (A row r is staged row tc_row(r) of its 8-row half).  A code
// word unpacks into those byte registers directly:
//   4-bit, k-block kb: word 2q+kb of the group's row; k-lo = low nibbles
//     (columns 16q + 8kb + 2j), k-hi = high nibbles (the next column each),
//     both entering as 16 x code (tc_unpack_a);
//   2-bit, k-block kb: word q; k-lo = 2-bit pack 2kb (columns 16q + 4j + 2kb),
//     k-hi = pack 2kb+1 (the next column each).
// The digits are stored so that each (k-block, limb, q) is one 8-byte pair
// {k-lo, k-hi}: word ((kb*3 + L)*4 + q)*2 + {0, 1}, byte j; 192 bytes per group.
// Per group one float2 {cscale, sum of x over the group}.

__device__ __forceinline__ void mma_u8s8(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
               : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
               : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Two fp32 fmas in one instruction (element-wise, each rounded once: the same
// results as two fmaf).
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{ .reg .b64 a, b, c, d; mov.b64 a, {%2, %3}; mov.b64 b, {%4, %5}; mov.b64 c, {%6, %7};"
      " fma.rn.f32x2 d, a, b, c; mov.b64 {%0, %1}, d; }"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}

// d = a * b + c with c a separate (unchanged) input, e.g. a constant start value.
__device__ __forceinline__ void mma_u8s8_c(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1, int c) {
  asm volatile("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%10,%10,%10};"
               : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
               : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "r"(c));
}

// Quantises one group of 64 values (lane l holds columns 2l, 2l+1) into the
// layout above: the same fixed-point digits as the per-token format (cscale =
// 2^(e-22) from the group's largest magnitude), only placed differently.
template <int BITS>
__device__ __forceinline__ void tc_quantize_group(float v0, float v1, uint8_t* glimbs, float2* gcs) {
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
  const int c = 2 * lane;  // columns c (k-lo) and c + 1 (k-hi) share k-block, quad lane and byte
  const int q = c >> 4;
  const int kb = BITS == 4 ? (c >> 3) & 1 : (c & 3) >> 1;
  const int j = BITS == 4 ? (c & 7) >> 1 : (c & 15) >> 2;
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int X = __float2int_rn((r ? v1 : v0) * inv);
    const int d2 = ((X + 128) & 255) - 128;
    const int X1 = (X - d2) >> 8;
    const int d1 = ((X1 + 128) & 255) - 128;
    const int d0 = (X1 - d1) >> 8;
    const int d[3] = {d0, d1, d2};
#pragma unroll
    for (int L = 0; L < 3; ++L) glimbs[((((kb * 3 + L) * 4 + q) * 2 + r) << 2) + j] = (uint8_t)(int8_t)d[L];
  }
  const float sx = warp_sum(v0 + v1);
  if (lane == 0) *gcs = make_float2(csc, sx);
}

// ---- selection, in two kernels.  topk: one CTA per token, the block-wide
// two-stage top-K (ties to the lower index) with renormalised weights and the
// shared-gate sigma.
__global__ void __launch_bounds__(kGT) topk_tokens_kernel(const GroupedParams p) {
  pdl_chain();
  __shared__ int s_idx[32];
  __shared__ float s_w[33];
  __shared__ unsigned long long s_cand[8 * 32];
  const int t = blockIdx.x, tid = threadIdx.x, K = p.K, E = p.E, R = E + 1, T = p.T, ns = p.rt_split;
  float* lg = const_cast<float*>(p.logits) + (size_t)t * R;
  for (int r = tid; r < R; r += kGT) {  // the router's slice sums, in slice order, then the bias
    float v[16];
#pragma unroll
    for (int c = 0; c < 16; ++c) v[c] = c < ns ? __ldcg(p.rt_part + ((size_t)c * T + t) * R + r) : 0.0f;
    float l = 0.0f;
#pragma unroll
    for (int c = 0; c < 16; ++c) l += v[c];
    if (r < E && p.rt_bias) l += p.rt_bias[r];
    lg[r] = l;
  }
  __syncthreads();  // the block's own global writes are visible to it after the barrier
  block_topk(lg, E, K, 1, s_cand, s_idx, s_w);
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
// Then the work units of the expert kernels: each group (the shared expert's
// T tokens first, then every active expert's pairs) cut into runs of at most
// kUnitToks members, so that no unit of work is much heavier than another.
// A unit is written out whole (UnitDesc) so that the expert kernels find it
// with one load.
__global__ void __launch_bounds__(kST) sort_pairs_kernel(const GroupedParams p) {
  pdl_chain();
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
  const int C = kUnitToks, nsh = (p.T + C - 1) / C;
  int c = 0, a = 0, w = 0;
  for (int k = 0; k < per; ++k) {
    const int e = tid * per + k;
    if (e < E) {
      c += s_cnt[e];
      a += s_cnt[e] > 0;
      w += (s_cnt[e] + C - 1) / C;
    }
  }
  int tot_c, tot_a, tot_w;
  int run = block_scan_excl(c, s_warp, &tot_c);
  int slot = block_scan_excl(a, s_warp, &tot_a);
  int wpos = nsh + block_scan_excl(w, s_warp, &tot_w);
  for (int k = 0; k < per; ++k) {
    const int e = tid * per + k;
    if (e < E) {
      s_start[e] = run;
      if (s_cnt[e] > 0) {
        p.act_expert[slot] = e;
        p.act_off[slot] = run;
        ++slot;
        for (int j0 = 0; j0 < s_cnt[e]; j0 += C, ++wpos)
          p.units[wpos] = UnitDesc{e, run + j0, min(C, s_cnt[e] - j0), 0, {0, 0, 0, 0}};
      }
      run += s_cnt[e];
    }
  }
  for (int i = tid; i < nsh; i += kST)  // the shared expert's members are all T tokens, rows T*K + t
    p.units[i] = UnitDesc{-1, N + i * C, min(C, p.T - i * C), 0, {0, 0, 0, 0}};
  if (tid == 0) {
    p.act_off[tot_a] = tot_c;
    p.n_active[0] = tot_a;
    p.n_active[1] = nsh + tot_w;
  }
  __syncthreads();
  for (int i = tid; i < N; i += kST) {
    const int e = s_e[i];
    int rank = 0, j = 0;
#pragma unroll 4
    for (; j + 4 <= i; j += 4) {
      const int4 v = *reinterpret_cast<const int4*>(s_e + j);
      rank += (v.x == e) + (v.y == e) + (v.z == e) + (v.w == e);
    }
    for (; j < i; ++j) rank += s_e[j] == e;
    const int pos = s_start[e] + rank;
    p.pair_tok[pos] = i;
    p.pair_pos[i] = pos;
  }
  __syncthreads();  // the units' tokens: from the sorted pairs (routed) or the row (shared)
  const int NW = nsh + tot_w;
  for (int i = tid; i < NW * kUnitToks; i += kST) {
    UnitDesc& d = p.units[i / kUnitToks];
    const int jj = i % kUnitToks;
    if (jj < d.n) d.tok[jj] = d.e < 0 ? d.row0 - N + jj : p.pair_tok[d.row0 + jj] / p.K;
  }
}

// ---- router for the batch.  norm_digits: x = RMSNorm(h) in fp32 for the
// router and as digits for the experts.  CTA (c, t) takes groups
// [c*NG/kNormSplit, (c+1)*NG/kNormSplit) of token t, one warp per group; every
// CTA of the token sums the squares of the whole row (the same order in each).
constexpr int kNormSplit = 4;

__global__ void __launch_bounds__(kGT) norm_digits_kernel(const GroupedParams p, const RouterBatch rb, int bits) {
  pdl_chain();
  __shared__ float s_red[kGT / 32];
  const int t = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, H = p.H, NG = H / kGroup;
  const float* h = p.h + (size_t)t * H;
  float* x = rb.x + (size_t)t * H;
  float rstd = 1.0f;
  if (rb.gamma) {
    float ss = 0.0f;
    for (int i = tid * 4; i < H; i += kGT * 4) {
      const float4 v = __ldcg(reinterpret_cast<const float4*>(h + i));
      ss = fmaf(v.x, v.x, fmaf(v.y, v.y, fmaf(v.z, v.z, fmaf(v.w, v.w, ss))));
    }
    ss = warp_sum(ss);
    if (lane == 0) s_red[warp] = ss;
    __syncthreads();
    float tot = 0.0f;
#pragma unroll
    for (int w = 0; w < kGT / 32; ++w) tot += s_red[w];
    rstd = 1.0f / sqrtf(tot / (float)H + rb.eps);
  }
  const int per = (NG + kNormSplit - 1) / kNormSplit, ge = min(NG, (int)(blockIdx.x + 1) * per);
  uint8_t* limbs = const_cast<uint8_t*>(p.xq_limbs) + (size_t)t * 3 * H;
  float2* cs = const_cast<float2*>(p.xq_cs) + (size_t)t * NG;
  for (int g = blockIdx.x * per + warp; g < ge; g += kGT / 32) {
    const int i = g * kGroup + 2 * lane;
    float2 v = __ldcg(reinterpret_cast<const float2*>(h + i));
    if (rb.gamma) {
      const float2 gm = __ldg(reinterpret_cast<const float2*>(rb.gamma + i));
      v = make_float2(v.x * rstd * gm.x, v.y * rstd * gm.y);
    }
    *reinterpret_cast<float2*>(x + i) = v;
    if (bits == 4)
      tc_quantize_group<4>(v.x, v.y, limbs + g * 192, cs + g);
    else
      tc_quantize_group<2>(v.x, v.y, limbs + g * 192, cs + g);
  }
}

// router_gemm: partial logits of [W_r; w_sg] . x[t] as a split-K tiled product.
// CTA (a, b, c) takes rows [64a, 64a+64), tokens [64b, 64b+64) and the c-th of
// p.rt_split slices of H, staged 256 columns at a time (cp.async); thread
// (ty, tx) sums rows ty + 16i and tokens tx + 16j.  The slice sums go to
// rt_part[c][t][row]; the top-K kernel adds the slices in order and the bias.
constexpr int kRtR = 64, kRtT = 64, kRtK = 256;  // rows, tokens and columns per staged tile

__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_addr(dst)), "l"(src), "r"(valid ? 16 : 0)
               : "memory");
}

__global__ void __launch_bounds__(kGT) router_gemm_kernel(const GroupedParams p, const RouterBatch rb) {
  pdl_chain();
  extern __shared__ __align__(16) uint8_t sm[];
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15, H = p.H, E = p.E, T = p.T, R = E + 1;
  const int r0 = blockIdx.x * kRtR, t0 = blockIdx.y * kRtT, kc = blockIdx.z, KC = H / p.rt_split;
  constexpr int WP = kRtK + 8, XP = kRtK + 4;  // padded row pitches (bf16, fp32)
  uint16_t* ws = reinterpret_cast<uint16_t*>(sm);
  float* xs = reinterpret_cast<float*>(sm + (size_t)kRtR * WP * 2);
  float acc[4][4] = {};
  for (int k0 = kc * KC; k0 < (kc + 1) * KC; k0 += kRtK) {
    const int kn = min(kRtK, (kc + 1) * KC - k0);  // a multiple of 64
    if (k0 != kc * KC) __syncthreads();          // the previous columns are summed
    for (int i = tid; i < kRtR * (kn / 8); i += kGT) {  // rows: W_r, then the shared-gate row, then zeros
      const int r = i / (kn / 8), c = (i % (kn / 8)) * 8, row = r0 + r;
      const uint16_t* src = row < E ? rb.w_router + (size_t)row * H + k0 + c : rb.w_sgate + k0 + c;
      cp_async16(ws + (size_t)r * WP + c, src, row <= E);
    }
    for (int i = tid; i < kRtT * (kn / 4); i += kGT) {
      const int t = i / (kn / 4), c = (i % (kn / 4)) * 4;
      cp_async16(xs + (size_t)t * XP + c, rb.x + (size_t)min(t0 + t, T - 1) * H + k0 + c, t0 + t < T);
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();
    for (int k = 0; k < kn; k += 4) {
      float4 xv[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) xv[j] = *reinterpret_cast<const float4*>(xs + (size_t)(tx + 16 * j) * XP + k);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint2 wv = *reinterpret_cast<const uint2*>(ws + (size_t)(ty + 16 * i) * WP + k);
        const float w0 = __uint_as_float(wv.x << 16), w1 = __uint_as_float(wv.x & 0xFFFF0000u);
        const float w2 = __uint_as_float(wv.y << 16), w3 = __uint_as_float(wv.y & 0xFFFF0000u);
#pragma unroll
        for (int j = 0; j < 4; ++j)
          acc[i][j] = fmaf(w3, xv[j].w, fmaf(w2, xv[j].z, fmaf(w1, xv[j].y, fmaf(w0, xv[j].x, acc[i][j]))));
      }
    }
  }
  float* pc = p.rt_part + (size_t)kc * T * R;  // this slice's partials [T][R]
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int row = r0 + ty + 16 * i, t = t0 + tx + 16 * j;
      if (row < R && t < T) pc[(size_t)t * R + row] = acc[i][j];
    }
}

// ---- the two expert kernels share one schedule.  Persistent, one CTA per SM,
// 8 consumer warps and 1 producer warp.  The items are the row blocks of the
// work units (item i = block i % NB of unit i / NB); CTA c takes the contiguous
// range [c*N/P, (c+1)*N/P), so consecutive items read neighbouring rows of one
// expert and share the unit's digits, which are staged once per unit.  The
// producer stages each item's rows into a ring of `ns` buffers (full / empty
// mbarriers per buffer) and each unit's digits into one of two slots; the
// consumers sum, then reduce their partial tiles and write the outputs.
constexpr int kConsumers = 8;                      // consumer warps
constexpr int kThreads = (kConsumers + 1) * 32;    // + the producer warp
constexpr int kRing = 16;                          // item descriptors in flight (> the largest ns)

struct ItemDesc {
  UnitDesc u;
  int blk;    // row block within the unit
  int useq;   // unit sequence number within this CTA: digit slot useq & 1
  int first;  // first item of its unit here (consumers wait for the digits)
  int last;   // last item of its unit here (consumers release the digit slot)
};

__device__ __forceinline__ UnitDesc load_unit(const GroupedParams& p, int wi) {
  const int4* src = reinterpret_cast<const int4*>(p.units + wi);
  const int4 a = __ldcg(src), b = __ldcg(src + 1);
  return UnitDesc{a.x, a.y, a.z, a.w, {b.x, b.y, b.z, b.w}};
}

// this CTA's items [i0, i0 + count)
__device__ __forceinline__ void item_range(const GroupedParams& p, int NB, int& i0, int& count) {
  const long long n = (long long)__ldcg(p.n_active + 1) * NB, P = gridDim.x, c = blockIdx.x;
  i0 = (int)(c * n / P);
  count = (int)((c + 1) * n / P) - i0;
}

// barrier of the consumer warps that also ORs a predicate over them
__device__ __forceinline__ bool named_sync_or(bool v) {
  uint32_t r;
  asm volatile(
      "{ .reg .pred p, q; setp.ne.u32 p, %1, 0; bar.red.or.pred q, 1, %2, p; selp.u32 %0, 1, 0, q; }"
      : "=r"(r)
      : "r"((uint32_t)v), "n"(kConsumers * 32)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ void mbar_arrive_one(uint32_t bar) {
  asm volatile("{ .reg .b64 st; mbarrier.arrive.shared::cta.b64 st, [%0]; }" ::"r"(bar) : "memory");
}

// The producer loop (lane 0 plans and waits; `issue_w(it, stage)` and
// `issue_d(unit, slot)` are called by the whole warp and arm their barrier on
// lane 0 first).  On a timeout, or when the consumers gave up, it stops
// issuing and waits (bounded) for the copies it has in flight, then returns.
template <typename IW, typename ID>
__device__ __forceinline__ void producer_loop(const GroupedParams& p, int NB, int i0, int count, int ns,
                                              ItemDesc* s_item, uint64_t* wfull, uint64_t* wempty, uint64_t* dfull,
                                              uint64_t* dempty, volatile int* s_abort, IW issue_w, ID issue_d) {
  const int lane = threadIdx.x & 31;
  int prev = -1, useq = -1, issued = 0, dissued = 0;
  bool ok = true;
  UnitDesc u{};
  for (int k = 0; k < count && ok; ++k) {
    const int item = i0 + k, wi = item / NB, blk = item % NB;
    if (lane == 0 && k >= ns) ok = mbar_wait_bounded(smem_addr(&wempty[k % ns]), (uint32_t)(((k / ns) - 1) & 1), p.err);
    if (lane == 0 && *s_abort) ok = false;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (!ok) break;
    const bool first = wi != prev;
    if (first) {
      ++useq;
      prev = wi;
      if (lane == 0) {
        u = load_unit(p, wi);
        if (useq >= 2) ok = mbar_wait_bounded(smem_addr(&dempty[useq & 1]), (uint32_t)(((useq >> 1) - 1) & 1), p.err);
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
    }
    const bool last = k + 1 == count || (item + 1) / NB != wi;
    if (lane == 0) s_item[k % kRing] = ItemDesc{u, blk, useq, first ? 1 : 0, last ? 1 : 0};
    __syncwarp();
    if (first) {
      issue_d(s_item[k % kRing].u, useq & 1);
      dissued = useq + 1;
    }
    issue_w(s_item[k % kRing], k % ns);  // its arrive releases the descriptor to the consumers
    issued = k + 1;
  }
  if (!ok && lane == 0) {  // let every copy in flight land before the CTA can leave
    *s_abort = 1;
    for (int k = issued - ns > 0 ? issued - ns : 0; k < issued; ++k)
      mbar_wait_bounded(smem_addr(&wfull[k % ns]), (uint32_t)((k / ns) & 1), p.err);
    for (int q = dissued - 2 > 0 ? dissued - 2 : 0; q < dissued; ++q)
      mbar_wait_bounded(smem_addr(&dfull[q & 1]), (uint32_t)((q >> 1) & 1), p.err);
  }
}

// Shapes of one staged row and of one token's (or activation row's) digits.
template <int BITS, int NG>
struct TcRows {
  static constexpr int RB = NG * kGroup * BITS / 8;
  static constexpr int LB = NG * 192;               // digit bytes of one token / activation row
  static constexpr int LBP = LB + 96;               // a member's pitch in a digit slot (see tc_sum)
  static constexpr int CB = NG * 8;                 // its per-group scalars
};

// The staged row that mma row gid (and gid + 8) of a tile reads: even rows for
// lanes 0-15, odd rows for lanes 16-31.  An 8-byte shared load is served per
// half-warp; with the 128-byte swizzle (chunk ^= row % 8) rows r and r ^ 1 share
// their pair of chunks, so a half-warp must read rows of distinct r >> 1.
__device__ __forceinline__ int tc_row(int gid) { return ((gid & 3) << 1) | (gid >> 2); }

// Staged rows (codes, and the per-group scale arrays): one tensor copy per array
// brings an item's ROWS rows of RB bytes as lines of LW = min(128, RB) bytes
// ordered (column block, row), with the copy's swizzle: the 16-byte chunk
// index of byte X is XORed with bits 7.. of X (128-byte swizzle: 3 bits,
// 64-byte: 2, 32-byte: 1; 16-byte lines are not swizzled).  Rows gid = 0..7 of
// a tile are consecutive, so the eight rows a quad-layout load reads land in
// distinct chunks.
template <int RB, int ROWS>
struct Sw {
  static constexpr int LW = RB >= 128 ? 128 : RB;
  __device__ static __forceinline__ const uint8_t* at(const uint8_t* buf, int row, int c) {
    constexpr int M = LW == 128 ? 7 : LW == 64 ? 3 : LW == 32 ? 1 : 0;  // swizzle mask of the line index
    const int X = ((c / LW) * ROWS + row) * LW + c % LW;
    return buf + (X ^ (((X >> 7) & M) << 4));
  }
};

template <int BITS, int NG, int ROWS>
using TcSw = Sw<NG * kGroup * BITS / 8, ROWS>;

// A registers of staged rows row_lo (A rows 0-7) and row_hi (rows 8-15) for group g.
template <int BITS, int NG, int ROWS>
__device__ __forceinline__ void tc_load_a(const uint8_t* buf_lo, int row_lo, const uint8_t* buf_hi, int row_hi, int g,
                                          int q, uint32_t (&w)[2][2]) {
  using S = TcSw<BITS, NG, ROWS>;
  if (BITS == 4) {
    const uint2 x = *reinterpret_cast<const uint2*>(S::at(buf_lo, row_lo, g * 32 + 8 * q));
    const uint2 y = *reinterpret_cast<const uint2*>(S::at(buf_hi, row_hi, g * 32 + 8 * q));
    w[0][0] = x.x; w[0][1] = x.y; w[1][0] = y.x; w[1][1] = y.y;
  } else {
    const uint32_t x = *reinterpret_cast<const uint32_t*>(S::at(buf_lo, row_lo, g * 16 + 4 * q));
    const uint32_t y = *reinterpret_cast<const uint32_t*>(S::at(buf_hi, row_hi, g * 16 + 4 * q));
    w[0][0] = w[0][1] = x; w[1][0] = w[1][1] = y;
  }
}

// A registers of k-block kb.  At 4 bits the u8 operands are 16 * code (the low
// nibble moved up, the high nibble masked in place), so the sums come out 16x;
// the column scales carry the 1/16 (tc_colscale).
template <int BITS>
__device__ __forceinline__ void tc_unpack_a(const uint32_t (&w)[2][2], int kb, uint32_t (&a)[4]) {
  if (BITS == 4) {
    a[0] = (w[0][kb] << 4) & 0xF0F0F0F0u;
    a[1] = (w[1][kb] << 4) & 0xF0F0F0F0u;
    a[2] = w[0][kb] & 0xF0F0F0F0u;
    a[3] = w[1][kb] & 0xF0F0F0F0u;
  } else {
    a[0] = (w[0][kb] >> (4 * kb)) & 0x03030303u;
    a[1] = (w[1][kb] >> (4 * kb)) & 0x03030303u;
    a[2] = (w[0][kb] >> (4 * kb + 2)) & 0x03030303u;
    a[3] = (w[1][kb] >> (4 * kb + 2)) & 0x03030303u;
  }
}

// GPW consecutive bf16 values (a warp's groups of one staged scale row) into
// packed registers, two per word.
template <int GPW>
__device__ __forceinline__ void tc_load_scales(const uint16_t* src, uint32_t (&v)[(GPW + 1) / 2]) {
  if constexpr (GPW == 1) {
    v[0] = src[0];
  } else if constexpr (GPW == 2) {
    v[0] = *reinterpret_cast<const uint32_t*>(src);
  } else if constexpr (GPW == 4) {
    const uint2 x = *reinterpret_cast<const uint2*>(src);
    v[0] = x.x;
    v[1] = x.y;
  } else {
#pragma unroll
    for (int i = 0; i < GPW / 8; ++i) {
      const uint4 x = reinterpret_cast<const uint4*>(src)[i];
      v[4 * i] = x.x;
      v[4 * i + 1] = x.y;
      v[4 * i + 2] = x.z;
      v[4 * i + 3] = x.w;
    }
  }
}

template <int GPW>
__device__ __forceinline__ float tc_scale(const uint32_t (&v)[(GPW + 1) / 2], int gi) {
  return __uint_as_float((gi & 1) ? (v[gi >> 1] & 0xFFFF0000u) : (v[gi >> 1] << 16));
}

// The quad lane's two C columns are 2q and 2q + 1; column c = 3t + L is limb L
// of the tile's token t, columns 6 and 7 unused.  Per group the lane needs each
// column's digit scale (0 for a column without a token), and for the limb-0
// column it holds (lane q = 0: column 0, token 0; q = 1: column 3, token 1) the
// token's group sum of x, for the bias term b * sum x (added on limb 0, whose
// weight 2^16 is applied last).  B registers of a column without a token read
// whatever the digit slot holds: any byte is a digit, and the column's scale is 0.
struct TcLane {
  int ta, tb;    // tokens of columns 2q and 2q + 1, clamped to a slot that exists
  bool va, vb;   // whether those columns have a token
  bool bias_a;   // column 2q is limb 0 of a token (q == 0)
  bool bias_b;   // column 2q + 1 is limb 0 of a token (q == 1 with two tokens)
};

__device__ __forceinline__ TcLane tc_lane(int q, int n) {
  TcLane l;
  const int ca = 2 * q, cb = 2 * q + 1;
  l.va = ca < 6 && ca / 3 < n;
  l.vb = cb < 6 && cb / 3 < n;
  l.ta = l.va ? ca / 3 : 0;
  l.tb = l.vb ? cb / 3 : 0;
  l.bias_a = q == 0;
  l.bias_b = q == 1 && l.vb;
  return l;
}

// The int32 sums are read as floats through a biased accumulator: the mma
// starts from the bits of 1.5 * 2^23, so that (for |sum| < 2^22, here below
// 16 * 15 * 128 * 64 at 4 bits) the result's bits are those of the float 1.5 * 2^23 + sum.
// With a power-of-two digit scale s, fma(f, s, -1.5 * 2^23 * s) is then
// exactly sum * s.
constexpr int kMagicBits = 0x4B400000;
constexpr float kMagic = 12582912.0f;

struct TcColScale {
  float sa, sb;  // digit scales of the two columns
  float na, nb;  // -kMagic * scale
  float bx;      // group sum of x / 2^16 for this lane's limb-0 column, else 0
};

// cf: the factor of the codes in the A operand's sums (1/16 at 4 bits, see tc_unpack_a).
__device__ __forceinline__ TcColScale tc_colscale(const float2* csv, int NG, int g, const TcLane& l, float cf) {
  const float2 va = csv[l.ta * (NG + 2) + g], vb = csv[l.tb * (NG + 2) + g];
  TcColScale c;
  c.sa = l.va ? va.x * cf : 0.0f;
  c.sb = l.vb ? vb.x * cf : 0.0f;
  c.na = -kMagic * c.sa;
  c.nb = -kMagic * c.sb;
  c.bx = (l.bias_a ? va.y : l.bias_b ? vb.y : 0.0f) * 0x1p-16f;
  return c;
}

// One group of one 16-row tile from its A words, with row scales s_lo / s_hi
// and biases b_lo / b_hi.
template <int BITS>
__device__ __forceinline__ void tc_tile_group(const uint32_t (&w)[2][2], const uint2 (&b)[2], const TcColScale& cs,
                                              float s_lo, float s_hi, float b_lo, float b_hi, float (&acc)[4],
                                              float (&accb)[2]) {
  int c[4];
  uint32_t a[4];
  tc_unpack_a<BITS>(w, 0, a);
  mma_u8s8_c(c, a, b[0].x, b[0].y, kMagicBits);  // starts from the biased accumulator
  tc_unpack_a<BITS>(w, 1, a);
  mma_u8s8(c, a, b[1].x, b[1].y);
  // the lane's two columns pair up: digit scales {sa, sb}, row scale s_lo (A rows
  // 0-7) or s_hi (rows 8-15)
  const float2 sc = make_float2(cs.sa, cs.sb), nc = make_float2(cs.na, cs.nb);
  const float2 ilo = ffma2(make_float2(__int_as_float(c[0]), __int_as_float(c[1])), sc, nc);
  const float2 ihi = ffma2(make_float2(__int_as_float(c[2]), __int_as_float(c[3])), sc, nc);
  const float2 alo = ffma2(make_float2(s_lo, s_lo), ilo, make_float2(acc[0], acc[1]));
  const float2 ahi = ffma2(make_float2(s_hi, s_hi), ihi, make_float2(acc[2], acc[3]));
  const float2 ab = ffma2(make_float2(b_lo, b_hi), make_float2(cs.bx, cs.bx), make_float2(accb[0], accb[1]));
  acc[0] = alo.x;
  acc[1] = alo.y;
  acc[2] = ahi.x;
  acc[3] = ahi.y;
  accb[0] = ab.x;
  accb[1] = ab.y;
}

// Sums TPW tiles over groups [g0, g0 + GPW) into acc (each tile's C layout,
// bias folded into the limb-0 columns).  Tile i reads rows rlo[i] of buf_lo and
// rhi[i] of buf_hi (staged, ROWS rows each); its row scales and biases come
// from the staged scale arrays sarr = {s_lo, b_lo, s_hi, b_hi} (row rlo[i] for
// the first two, rhi[i] for the others).  B and the column scales are shared
// by the tiles.
template <int BITS, int NG, int ROWS, int GPW, int TPW>
__device__ __forceinline__ void tc_sum(const uint8_t* buf_lo, const uint8_t* buf_hi, const int (&rlo)[TPW],
                                       const int (&rhi)[TPW], const uint8_t* const (&sarr)[4], const uint8_t* db, int n,
                                       int g0, float (&acc)[TPW][4]) {
  constexpr int LBP = TcRows<BITS, NG>::LBP;
  constexpr int GPC = GPW < 8 ? GPW : 8;  // groups whose scales are held at once
  const int lane = threadIdx.x & 31, gid = lane >> 2, q = lane & 3;
  const TcLane ln = tc_lane(q, n);
  // This lane's B column: member slot and limb.  Half-warp 0 reads member 0's
  // three limbs and member 1's limb 0, half-warp 1 member 1's limbs 1 and 2
  // (columns 6 and 7, unused, repeat 4 and 5).  A member's 96 bytes of a group
  // are limb-major; with the members 96 bytes apart modulo 128 (pitch LBP),
  // each half-warp's 8-byte loads fall in distinct banks.
  const int bt = gid < 3 ? 0 : 1, bl = gid < 6 ? gid % 3 : gid - 5;
  const uint8_t* bsrc = db + bt * LBP + (size_t)((bl * 4 + q) * 8);
  const float2* csv = reinterpret_cast<const float2*>(db + kUnitToks * LBP);  // [token][NG + 2] (padded pitch)
  // A addresses.  With 128-byte lines and g0 a multiple of the groups per line
  // (4 at 4-bit, 8 at 2-bit), a lane's rows all have row % 8 == tc_row(gid), so the
  // swizzled byte of group g is row*128 + (g / PER)*ROWS*128 + vx[g % PER], with
  // vx a lane constant: one add per load.  Otherwise the general formula (Sw).
  using SA = TcSw<BITS, NG, ROWS>;
  constexpr int PER = BITS == 4 ? 4 : 8;  // groups per 128-byte line
  constexpr bool FAST = SA::LW == 128 && GPW % PER == 0;
  uint32_t vx[PER];
#pragma unroll
  for (int m = 0; m < PER; ++m)
    vx[m] = (uint32_t)((BITS == 4 ? (m << 5) | (8 * q) : (m << 4) | (4 * q)) ^ (tc_row(gid) << 4));
  const uint8_t* blo[TPW];
  const uint8_t* bhi[TPW];
#pragma unroll
  for (int i = 0; i < TPW; ++i) {
    blo[i] = buf_lo + (size_t)rlo[i] * 128 + (size_t)(g0 / PER) * ROWS * 128;
    bhi[i] = buf_hi + (size_t)rhi[i] * 128 + (size_t)(g0 / PER) * ROWS * 128;
  }
  float accb[TPW][2];
#pragma unroll
  for (int i = 0; i < TPW; ++i) accb[i][0] = accb[i][1] = 0.0f;
#pragma unroll 1  // chunks of GPC groups (more than one only for long rows: keeps registers in bounds)
  for (int gc = 0; gc < GPW; gc += GPC) {
    uint32_t sv[TPW][4][(GPC + 1) / 2];
#pragma unroll
    for (int i = 0; i < TPW; ++i)
#pragma unroll
      for (int a = 0; a < 4; ++a)
        tc_load_scales<GPC>(
            reinterpret_cast<const uint16_t*>(Sw<NG * 2, ROWS>::at(sarr[a], a < 2 ? rlo[i] : rhi[i], (g0 + gc) * 2)),
            sv[i][a]);
#pragma unroll
    for (int gi = 0; gi < GPC; ++gi) {
      const int g = g0 + gc + gi;
      uint2 b[2];
#pragma unroll
      for (int kb = 0; kb < 2; ++kb) b[kb] = *reinterpret_cast<const uint2*>(bsrc + g * 192 + kb * 96);
      const TcColScale cs = tc_colscale(csv, NG, g, ln, BITS == 4 ? 0.0625f : 1.0f);
#pragma unroll
      for (int i = 0; i < TPW; ++i) {
        uint32_t w[2][2];
        if constexpr (FAST) {
          // GPC is a multiple of PER here, so gi % PER is the line position
          const size_t off = (size_t)(gc / PER + gi / PER) * ROWS * 128;
          if (BITS == 4) {
            const uint2 x = *reinterpret_cast<const uint2*>(blo[i] + off + vx[gi % PER]);
            const uint2 y = *reinterpret_cast<const uint2*>(bhi[i] + off + vx[gi % PER]);
            w[0][0] = x.x; w[0][1] = x.y; w[1][0] = y.x; w[1][1] = y.y;
          } else {
            const uint32_t x = *reinterpret_cast<const uint32_t*>(blo[i] + off + vx[gi % PER]);
            const uint32_t y = *reinterpret_cast<const uint32_t*>(bhi[i] + off + vx[gi % PER]);
            w[0][0] = w[0][1] = x; w[1][0] = w[1][1] = y;
          }
        } else {
          tc_load_a<BITS, NG, ROWS>(buf_lo, rlo[i], buf_hi, rhi[i], g, q, w);
        }
        tc_tile_group<BITS>(w, b, cs, tc_scale<GPC>(sv[i][0], gi), tc_scale<GPC>(sv[i][2], gi),
                            tc_scale<GPC>(sv[i][1], gi), tc_scale<GPC>(sv[i][3], gi), acc[i], accb[i]);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < TPW; ++i) {
    if (q == 0) {
      acc[i][0] += accb[i][0];
      acc[i][2] += accb[i][1];
    } else if (q == 1) {
      acc[i][1] += accb[i][0];
      acc[i][3] += accb[i][1];
    }
  }
}

// The tensor maps of a kernel's staged arrays: routed bank first, then the shared expert's.
template <int N>
struct TcMaps {
  CUtensorMap m[N];
};

// cp.async.bulk.tensor of a 4-D box at (0, row, 0, expert) into shared memory.
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* tm, int row, int expert, uint32_t bar,
                                            uint64_t pol) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4, %5}], [%6], %7;" ::"r"(dst),
      "l"(tm), "r"(0), "r"(row), "r"(0), "r"(expert), "r"(bar), "l"(pol)
      : "memory");
}

// ---- gate/up + SwiGLU.  An item is ROWS = 8*TL (gate, up) row pairs: one
// tensor copy per matrix stages the rows (swizzled, see TcSw), four bulk copies
// the scale arrays.  Tile t pairs gate row 8t + tc_row(gid) (A rows 0-7) with
// the same up row (rows 8-15).  The digits are those of x for each member token.  Warp
// w sums tiles [TPW*(w / KS), +TPW) over K slice w % KS; the KS partial tiles
// add in slice order.  act[row][r] = silu(g) * u.
template <int BITS, int NG, int TL>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gateup_kernel(const GroupedParams p, int ns, const __grid_constant__ TcMaps<12> maps) {
  pdl_chain();
  using R = TcRows<BITS, NG>;
  constexpr int RB = R::RB, LB = R::LB, LBP = R::LBP, CB = R::CB, SB = NG * 2;
  constexpr int ROWS = 8 * TL, TPW = TL < 2 ? TL : 2, KS = kConsumers * TPW / TL;  // TPW tiles per warp, KS K slices
  constexpr int GPW = NG / KS >= 1 ? NG / KS : 1;                                  // groups per K slice
  constexpr int CODE = (ROWS * RB + 1023) / 1024 * 1024;  // one matrix's staged rows
  constexpr int SA = (ROWS * SB + 1023) / 1024 * 1024;    // one staged scale array
  constexpr int WB = 2 * CODE + 4 * SA;                   // gate rows, up rows, gate s, gate b, up s, up b
  constexpr int CBP = CB + 16;                            // a token's scalars, padded apart in shared memory
  constexpr int DB = kUnitToks * (LBP + CBP);
  constexpr int TP = 2 * ROWS * 8 + 4;  // floats per slice's partial tiles (gate rows, then up rows)
  extern __shared__ __align__(1024) uint8_t sm_raw[];
  __shared__ __align__(8) uint64_t s_wfull[kRing], s_wempty[kRing], s_dfull[2], s_dempty[2];
  __shared__ ItemDesc s_item[kRing];
  __shared__ int s_abort;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gid = lane >> 2, q = lane & 3;
  const int I = p.I, NB = I / ROWS;
  int i0, count;
  item_range(p, NB, i0, count);
  uint8_t* sm = sm_raw + ((1024u - (smem_addr(sm_raw) & 1023u)) & 1023u);  // swizzled copies want 1 KiB alignment
  uint8_t* dbase = sm + (size_t)ns * WB;
  float* red = reinterpret_cast<float*>(dbase + 2 * DB);  // [2][KS][TP]
  if (tid == 0) {
    for (int i = 0; i < ns; ++i) {
      mbar_init(smem_addr(&s_wfull[i]), 1);
      mbar_init(smem_addr(&s_wempty[i]), kConsumers);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_addr(&s_dfull[i]), 1);
      mbar_init(smem_addr(&s_dempty[i]), kConsumers);
    }
    mbar_fence_init();
    s_abort = 0;
  }
  __syncthreads();

  if (warp == kConsumers) {  // the producer
    const uint64_t pol_w = l2_policy_evict_first(), pol_d = l2_policy_evict_last();
    auto issue_w = [&](const ItemDesc& it, int st) {  // gate rows, up rows, then the four scale arrays
      const int r0 = it.blk * ROWS;
      const uint32_t bw = smem_addr(&s_wfull[st]), dst = smem_addr(sm + (size_t)st * WB);
      if (lane == 0) mbar_expect_tx(bw, 2 * ROWS * RB + 4 * ROWS * SB);
      __syncwarp();
      if (lane < 6) {
        const bool sh = it.u.e < 0;
        const uint32_t off = lane == 0 ? 0u : lane == 1 ? (uint32_t)CODE : (uint32_t)(2 * CODE + (lane - 2) * SA);
        tma_load_4d(dst + off, &maps.m[(sh ? 6 : 0) + lane], r0, sh ? 0 : it.u.e, bw, pol_w);
      }
    };
    auto issue_d = [&](const UnitDesc& u, int slot) {
      const uint32_t bd = smem_addr(&s_dfull[slot]);
      uint8_t* dst = dbase + (size_t)slot * DB;
      if (lane == 0) mbar_expect_tx(bd, (uint32_t)u.n * (LB + CB));
      __syncwarp();
      if (lane < u.n) {
        const int tok = u.tok[lane];
        bulk_g2s(smem_addr(dst + lane * LBP), p.xq_limbs + (size_t)tok * LB, LB, bd, pol_d);
        bulk_g2s(smem_addr(dst + kUnitToks * LBP + lane * CBP), p.xq_cs + (size_t)tok * NG, CB, bd, pol_d);
      }
    };
    producer_loop(p, NB, i0, count, ns, s_item, s_wfull, s_wempty, s_dfull, s_dempty, &s_abort, issue_w, issue_d);
    return;
  }

  const int tg = warp / KS, kp = warp % KS, g0 = kp * GPW;
  const bool kwarp = g0 < NG;  // this warp has groups to sum
  int rows[TPW];               // this lane's row pair in each of its tiles
#pragma unroll
  for (int i = 0; i < TPW; ++i) rows[i] = 8 * (tg * TPW + i) + tc_row(gid);
  // output (row pair r, token t) of item k from slice ks, then the KS slices in order
  auto reduce = [&](int k, int row0, int n, int r0) {
    if (tid < 2 * ROWS * KS) {
      const int o = tid / KS, ks = tid % KS, r = o >> 1, t = o & 1;
      const float* rs = red + ((k & 1) * KS + ks) * TP + 3 * t;
      float gv = 0.0f, uv = 0.0f;
#pragma unroll
      for (int L = 0; L < 3; ++L) {
        const float f = L == 0 ? 65536.0f : L == 1 ? 256.0f : 1.0f;
        gv = fmaf(f, rs[r * 8 + L], gv);
        uv = fmaf(f, rs[(ROWS + r) * 8 + L], uv);
      }
#pragma unroll
      for (int o2 = 1; o2 < KS; o2 <<= 1) {
        gv += __shfl_xor_sync(0xffffffffu, gv, o2);
        uv += __shfl_xor_sync(0xffffffffu, uv, o2);
      }
      if (ks == 0 && t < n) p.act[(size_t)(row0 + t) * I + r0 + r] = gv / (1.0f + expf(-gv)) * uv;
    }
  };
  int p_row0 = 0, p_n = 0, p_r0 = 0;  // the previous item, reduced one step late
  for (int k = 0; k < count; ++k) {
    const int st = k % ns;
    bool ok = mbar_wait_bounded(smem_addr(&s_wfull[st]), (uint32_t)((k / ns) & 1), p.err);
    const ItemDesc it = s_item[k % kRing];
    const int slot = it.useq & 1;
    if (ok && it.first) ok = mbar_wait_bounded(smem_addr(&s_dfull[slot]), (uint32_t)((it.useq >> 1) & 1), p.err);
    ok = __all_sync(0xffffffffu, ok);
    const uint8_t* wb = sm + (size_t)st * WB;
    float acc[TPW][4];
#pragma unroll
    for (int i = 0; i < TPW; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.0f;
    if (ok && kwarp) {
      const uint8_t* const sarr[4] = {wb + 2 * CODE, wb + 2 * CODE + SA, wb + 2 * CODE + 2 * SA, wb + 2 * CODE + 3 * SA};
      tc_sum<BITS, NG, ROWS, GPW, TPW>(wb, wb + CODE, rows, rows, sarr, dbase + (size_t)slot * DB, it.u.n, g0, acc);
    }
    __syncwarp();
    if (lane == 0) {  // this warp is done with the item's rows (and, on its last item, the unit's digits)
      mbar_arrive_one(smem_addr(&s_wempty[st]));
      if (it.last) mbar_arrive_one(smem_addr(&s_dempty[slot]));
    }
    if (k > 0) reduce(k - 1, p_row0, p_n, p_r0);  // its tiles were complete at the last barrier
    float* rw = red + ((k & 1) * KS + kp) * TP;
#pragma unroll
    for (int i = 0; i < TPW; ++i) {
      *reinterpret_cast<float2*>(rw + rows[i] * 8 + 2 * q) = make_float2(acc[i][0], acc[i][1]);
      *reinterpret_cast<float2*>(rw + (ROWS + rows[i]) * 8 + 2 * q) = make_float2(acc[i][2], acc[i][3]);
    }
    // the tiles of item k are in place; item k + 2 writes them again only after the
    // next barrier, by which every thread has reduced them.  A wait that ran out
    // anywhere ends every consumer here.
    if (named_sync_or(!ok)) {
      if (tid == 0) s_abort = 1;
      return;
    }
    p_row0 = it.u.row0;
    p_n = it.u.n;
    p_r0 = it.blk * ROWS;
  }
  if (count > 0) reduce(count - 1, p_row0, p_n, p_r0);
}

// ---- activation digits of every sorted pair and every shared-expert token: one warp per group of 64
template <int BITS>
__global__ void __launch_bounds__(kGT) grouped_actq_kernel(const GroupedParams p) {
  pdl_chain();
  const int I = p.I, NGI = I / kGroup;
  const int gw = blockIdx.x * (kGT / 32) + (threadIdx.x >> 5);
  if (gw >= (p.T * p.K + p.T) * NGI) return;  // warp-uniform
  const int row = gw / NGI, g = gw % NGI;
  const float2 v = __ldcg(reinterpret_cast<const float2*>(p.act + (size_t)row * I + g * kGroup) + (threadIdx.x & 31));
  tc_quantize_group<BITS>(v.x, v.y, p.act_limbs + (size_t)row * 3 * I + g * 192, p.act_cs + (size_t)row * NGI + g);
}

// ---- down.  An item is ROWS = 16*TL output rows: one tensor copy stages the
// rows (swizzled, see TcSw), two bulk copies the scale arrays.  Tile t takes
// rows 16t + tc_row(gid) (A rows 0-7) and 16t + 8 + tc_row(gid) (rows 8-15).
// The digits are those of the members' activations (two copies per member).
// Warps split tiles and K as in gate/up.  y[member row][h] holds the unweighted
// down output.
template <int BITS, int NG, int TL>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_down_kernel(const GroupedParams p, int ns, const __grid_constant__ TcMaps<6> maps) {
  pdl_chain();
  using R = TcRows<BITS, NG>;
  constexpr int RB = R::RB, LB = R::LB, LBP = R::LBP, CB = R::CB, SB = NG * 2;
  constexpr int ROWS = 16 * TL, TPW = TL < 2 ? TL : 2, KS = kConsumers * TPW / TL;
  constexpr int GPW = NG / KS >= 1 ? NG / KS : 1;
  constexpr int CODE = (ROWS * RB + 1023) / 1024 * 1024;
  constexpr int SA = (ROWS * SB + 1023) / 1024 * 1024;
  constexpr int WB = CODE + 2 * SA;  // rows, then s, b
  constexpr int CBP = CB + 16;
  constexpr int DB = kUnitToks * (LBP + CBP);
  constexpr int TP = ROWS * 8 + 4;
  extern __shared__ __align__(1024) uint8_t sm_raw[];
  __shared__ __align__(8) uint64_t s_wfull[kRing], s_wempty[kRing], s_dfull[2], s_dempty[2];
  __shared__ ItemDesc s_item[kRing];
  __shared__ int s_abort;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gid = lane >> 2, q = lane & 3;
  const int H = p.H, NB = H / ROWS;
  int i0, count;
  item_range(p, NB, i0, count);
  uint8_t* sm = sm_raw + ((1024u - (smem_addr(sm_raw) & 1023u)) & 1023u);
  uint8_t* dbase = sm + (size_t)ns * WB;
  float* red = reinterpret_cast<float*>(dbase + 2 * DB);
  if (tid == 0) {
    for (int i = 0; i < ns; ++i) {
      mbar_init(smem_addr(&s_wfull[i]), 1);
      mbar_init(smem_addr(&s_wempty[i]), kConsumers);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_addr(&s_dfull[i]), 1);
      mbar_init(smem_addr(&s_dempty[i]), kConsumers);
    }
    mbar_fence_init();
    s_abort = 0;
  }
  __syncthreads();

  if (warp == kConsumers) {  // the producer
    const uint64_t pol_w = l2_policy_evict_first(), pol_d = l2_policy_evict_last();
    auto issue_w = [&](const ItemDesc& it, int st) {  // rows, then the scale arrays s, b
      const int d0 = it.blk * ROWS;
      const uint32_t bw = smem_addr(&s_wfull[st]), dst = smem_addr(sm + (size_t)st * WB);
      if (lane == 0) mbar_expect_tx(bw, ROWS * RB + 2 * ROWS * SB);
      __syncwarp();
      if (lane < 3) {
        const bool sh = it.u.e < 0;
        const uint32_t off = lane == 0 ? 0u : (uint32_t)(CODE + (lane - 1) * SA);
        tma_load_4d(dst + off, &maps.m[(sh ? 3 : 0) + lane], d0, sh ? 0 : it.u.e, bw, pol_w);
      }
    };
    auto issue_d = [&](const UnitDesc& u, int slot) {
      const uint32_t bd = smem_addr(&s_dfull[slot]);
      uint8_t* dst = dbase + (size_t)slot * DB;
      if (lane == 0) mbar_expect_tx(bd, (uint32_t)u.n * (LB + CB));
      __syncwarp();
      if (lane < u.n) {
        bulk_g2s(smem_addr(dst + lane * LBP), p.act_limbs + (size_t)(u.row0 + lane) * LB, LB, bd, pol_d);
        bulk_g2s(smem_addr(dst + kUnitToks * LBP + lane * CBP), p.act_cs + (size_t)(u.row0 + lane) * NG, CB, bd, pol_d);
      }
    };
    producer_loop(p, NB, i0, count, ns, s_item, s_wfull, s_wempty, s_dfull, s_dempty, &s_abort, issue_w, issue_d);
    return;
  }

  const int tg = warp / KS, kp = warp % KS, g0 = kp * GPW;
  const bool kwarp = g0 < NG;
  int rlo[TPW], rhi[TPW];  // this lane's rows in each of its tiles
#pragma unroll
  for (int i = 0; i < TPW; ++i) {
    rlo[i] = 16 * (tg * TPW + i) + tc_row(gid);
    rhi[i] = rlo[i] + 8;
  }
  // output (row r, token t) of item k from slice ks, then the KS slices in order
  auto reduce = [&](int k, int row0, int n, int d0) {
#pragma unroll
    for (int pass = 0; pass < (2 * ROWS * KS + kConsumers * 32 - 1) / (kConsumers * 32); ++pass) {
      const int idx = pass * kConsumers * 32 + tid;
      if (idx < 2 * ROWS * KS) {
        const int o = idx / KS, ks = idx % KS, r = o >> 1, t = o & 1;
        const float* rs = red + ((k & 1) * KS + ks) * TP + r * 8 + 3 * t;
        float v = fmaf(65536.0f, rs[0], fmaf(256.0f, rs[1], rs[2]));
#pragma unroll
        for (int o2 = 1; o2 < KS; o2 <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o2);
        if (ks == 0 && t < n) p.y[(size_t)(row0 + t) * H + d0 + r] = v;
      }
    }
  };
  int p_row0 = 0, p_n = 0, p_d0 = 0;
  for (int k = 0; k < count; ++k) {
    const int st = k % ns;
    bool ok = mbar_wait_bounded(smem_addr(&s_wfull[st]), (uint32_t)((k / ns) & 1), p.err);
    const ItemDesc it = s_item[k % kRing];
    const int slot = it.useq & 1;
    if (ok && it.first) ok = mbar_wait_bounded(smem_addr(&s_dfull[slot]), (uint32_t)((it.useq >> 1) & 1), p.err);
    ok = __all_sync(0xffffffffu, ok);
    const uint8_t* wb = sm + (size_t)st * WB;
    float acc[TPW][4];
#pragma unroll
    for (int i = 0; i < TPW; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.0f;
    if (ok && kwarp) {
      const uint8_t* const sarr[4] = {wb + CODE, wb + CODE + SA, wb + CODE, wb + CODE + SA};
      tc_sum<BITS, NG, ROWS, GPW, TPW>(wb, wb, rlo, rhi, sarr, dbase + (size_t)slot * DB, it.u.n, g0, acc);
    }
    __syncwarp();
    if (lane == 0) {
      mbar_arrive_one(smem_addr(&s_wempty[st]));
      if (it.last) mbar_arrive_one(smem_addr(&s_dempty[slot]));
    }
    if (k > 0) reduce(k - 1, p_row0, p_n, p_d0);
    float* rw = red + ((k & 1) * KS + kp) * TP;
#pragma unroll
    for (int i = 0; i < TPW; ++i) {
      *reinterpret_cast<float2*>(rw + rlo[i] * 8 + 2 * q) = make_float2(acc[i][0], acc[i][1]);
      *reinterpret_cast<float2*>(rw + rhi[i] * 8 + 2 * q) = make_float2(acc[i][2], acc[i][3]);
    }
    if (named_sync_or(!ok)) {
      if (tid == 0) s_abort = 1;
      return;
    }
    p_row0 = it.u.row0;
    p_n = it.u.n;
    p_d0 = it.blk * ROWS;
  }
  if (count > 0) reduce(count - 1, p_row0, p_n, p_d0);
}

// ---- combine, fixed k order: out[t] = h[t] + sum_k w_tk y[pair(t,k)] + sigma_t y_shared[t].
// CTA (c, t) takes columns [4*kGT*c, 4*kGT*(c+1)) of token t, four per thread;
// the member rows and weights are read once per CTA, and the rows' loads are
// issued eight at a time before their terms are added in k order.
__global__ void __launch_bounds__(kGT) grouped_combine_kernel(const GroupedParams p) {
  pdl_chain();
  __shared__ int s_pos[33];
  __shared__ float s_w[33];
  const int t = blockIdx.y, tid = threadIdx.x, K = p.K, H = p.H;
  if (tid <= K) {
    s_pos[tid] = tid < K ? __ldcg(p.pair_pos + (size_t)t * K + tid) : p.T * K + t;
    s_w[tid] = __ldcg(p.route_w + (size_t)t * (K + 1) + tid);
  }
  __syncthreads();
  const int h = (blockIdx.x * kGT + tid) * 4;
  if (h >= H) return;
  float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  for (int k0 = 0; k0 <= K; k0 += 8) {
    float4 v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (k0 + j <= K) v[j] = __ldcg(reinterpret_cast<const float4*>(p.y + (size_t)s_pos[k0 + j] * H + h));
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (k0 + j <= K) {
        const float w = s_w[k0 + j];
        acc = make_float4(fmaf(w, v[j].x, acc.x), fmaf(w, v[j].y, acc.y), fmaf(w, v[j].z, acc.z), fmaf(w, v[j].w, acc.w));
      }
  }
  const float4 hv = __ldcg(reinterpret_cast<const float4*>(p.h + (size_t)t * H + h));
  *reinterpret_cast<float4*>(p.out + (size_t)t * H + h) =
      make_float4(hv.x + acc.x, hv.y + acc.y, hv.z + acc.z, hv.w + acc.w);
}

constexpr size_t kSmemBudget = 220 * 1024;

// Shared memory of an expert kernel: `ns` staged items of `wb` bytes, two digit
// slots of kUnitToks members, the double-buffered partial tiles (tp floats per
// buffer, all K slices) and 1 KiB to align the staging ring.
size_t tc_smem(int ns, size_t wb, int NG, size_t tp) {
  return (size_t)ns * wb + 2 * (size_t)kUnitToks * ((size_t)NG * 200 + 96 + 16) + 2 * tp * 4 + 1024;
}

size_t round_kib(size_t v) { return (v + 1023) / 1024 * 1024; }

struct TcConfig {
  int tl, ns;
  size_t smem;
};

// gate/up: 16 row pairs per item (TL 2) while two stages fit, else 8 (TL 1),
// with as many stages (<= 6) as fit.
TcConfig gu_config(int bits, int H) {
  const int NG = H / kGroup, RB = H * bits / 8, SB = NG * 2;
  for (int tl : {2, 1}) {
    const int rows = 8 * tl, ks = kConsumers * (tl < 2 ? tl : 2) / tl;
    const size_t wb = 2 * round_kib((size_t)rows * RB) + 4 * round_kib((size_t)rows * SB);
    const size_t tp = (size_t)ks * (2 * rows * 8 + 4);
    for (int n = 6; n >= 2; --n) {
      const size_t sm = tc_smem(n, wb, NG, tp);
      if (sm <= kSmemBudget) return TcConfig{tl, n, sm};
    }
  }
  return TcConfig{0, 0, 0};
}

// down: 128 rows per item (TL 8) with at least 2 stages, else 64, 32 or 16 rows
// (TL 4, 2, 1) with at least 3; at most 8 stages.
TcConfig dn_config(int bits, int I) {
  const int NG = I / kGroup, RB = I * bits / 8, SB = NG * 2;
  for (int tl : {8, 4, 2, 1}) {
    const int rows = 16 * tl, ks = kConsumers * (tl < 2 ? tl : 2) / tl;
    const size_t wb = round_kib((size_t)rows * RB) + 2 * round_kib((size_t)rows * SB);
    const size_t tp = (size_t)ks * (rows * 8 + 4);
    for (int n = 8; n >= (tl == 8 ? 2 : 3); --n) {
      const size_t sm = tc_smem(n, wb, NG, tp);
      if (sm <= kSmemBudget) return TcConfig{tl, n, sm};
    }
  }
  return TcConfig{0, 0, 0};
}

// The tensor map of one staged array of a bank (a code matrix, or a per-group
// scale array): `rows` rows of RB bytes per expert, seen as (LW bytes, rows,
// RB / LW column blocks, experts) so that a box of box_rows rows lands as
// (column block, row) lines; swizzled as Sw assumes.
cudaError_t encode_codes(CUtensorMap* m, const uint8_t* base, int rows, int RB, int nexp, long long stride,
                         int box_rows) {
  static PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      enc = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  if (!enc) return cudaErrorNotSupported;
  const int LW = RB >= 128 ? 128 : RB;
  const cuuint64_t dims[4] = {(cuuint64_t)LW, (cuuint64_t)rows, (cuuint64_t)(RB / LW), (cuuint64_t)nexp};
  const cuuint64_t strides[3] = {(cuuint64_t)RB, (cuuint64_t)LW,
                                 (cuuint64_t)(nexp > 1 ? stride : (long long)rows * RB)};
  const cuuint32_t box[4] = {(cuuint32_t)LW, (cuuint32_t)box_rows, (cuuint32_t)(RB / LW), 1};
  const cuuint32_t es[4] = {1, 1, 1, 1};
  const CUtensorMapSwizzle sw = LW == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                                : LW == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                : LW == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                           : CU_TENSOR_MAP_SWIZZLE_NONE;
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<uint8_t*>(base), dims, strides, box, es,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// Maps of the arrays `subs` (record sub-array indices) of both banks: rows of
// the codes are rb bytes, of the scale arrays 2 * NG bytes.
template <int N>
cudaError_t encode_maps(TcMaps<N>& m, const GroupedParams& p, const int (&subs)[N / 2], bool codes_first, int rows,
                        int rb, int NG, int box_rows) {
  for (int b = 0; b < 2; ++b) {
    const BankRef& bk = b == 0 ? p.routed : p.shared;
    for (int j = 0; j < N / 2; ++j) {
      const int w = (codes_first && j == 0) || (!codes_first && j < 2) ? rb : 2 * NG;
      const cudaError_t e = encode_codes(&m.m[b * (N / 2) + j], bk.base + bk.off[subs[j]], rows, w, b == 0 ? p.E : 1,
                                         b == 0 ? bk.stride : 0, box_rows);
      if (e != cudaSuccess) return e;
    }
  }
  return cudaSuccess;
}

template <int BITS, int NG>
cudaError_t gateup_ng(const GroupedParams& p, const TcConfig& c, bool pdl, cudaStream_t s) {
  TcMaps<12> m;
  static constexpr int subs[6] = {0, 3, 1, 2, 4, 5};  // gate rows, up rows, gate s, gate b, up s, up b
  cudaError_t e = encode_maps(m, p, subs, false, p.I, p.H * BITS / 8, NG, 8 * c.tl);
  if (e != cudaSuccess) return e;
  auto k = c.tl == 2 ? grouped_gateup_kernel<BITS, NG, 2> : grouped_gateup_kernel<BITS, NG, 1>;
  if ((e = set_smem((const void*)k, c.smem)) != cudaSuccess) return e;
  if ((e = set_carveout_max((const void*)k)) != cudaSuccess) return e;
  return launch_pdl(k, dim3(num_sms()), dim3(kThreads), c.smem, s, pdl, p, c.ns, m);
}

template <int BITS, int NG>
cudaError_t down_ng(const GroupedParams& p, const TcConfig& c, bool pdl, cudaStream_t s) {
  TcMaps<6> m;
  static constexpr int subs[3] = {6, 7, 8};  // rows, s, b
  cudaError_t e = encode_maps(m, p, subs, true, p.H, p.I * BITS / 8, NG, 16 * c.tl);
  if (e != cudaSuccess) return e;
  auto k = c.tl == 8   ? grouped_down_kernel<BITS, NG, 8>
           : c.tl == 4 ? grouped_down_kernel<BITS, NG, 4>
           : c.tl == 2 ? grouped_down_kernel<BITS, NG, 2>
                       : grouped_down_kernel<BITS, NG, 1>;
  if ((e = set_smem((const void*)k, c.smem)) != cudaSuccess) return e;
  if ((e = set_carveout_max((const void*)k)) != cudaSuccess) return e;
  return launch_pdl(k, dim3(num_sms()), dim3(kThreads), c.smem, s, pdl, p, c.ns, m);
}

template <int BITS>
cudaError_t gateup_bits_g(const GroupedParams& p, bool pdl, cudaStream_t s) {
  const TcConfig c = gu_config(BITS, p.H);
  if (c.tl == 0 || p.I % (8 * c.tl)) return cudaErrorInvalidValue;
  switch (p.H / kGroup) {
    case 8: return gateup_ng<BITS, 8>(p, c, pdl, s);
    case 16: return gateup_ng<BITS, 16>(p, c, pdl, s);
    case 32: return gateup_ng<BITS, 32>(p, c, pdl, s);
    case 64: return gateup_ng<BITS, 64>(p, c, pdl, s);
    case 128: return gateup_ng<BITS, 128>(p, c, pdl, s);
    default: return cudaErrorInvalidValue;
  }
}

template <int BITS>
cudaError_t down_bits_g(const GroupedParams& p, bool pdl, cudaStream_t s) {
  const TcConfig c = dn_config(BITS, p.I);
  if (c.tl == 0 || p.H % (16 * c.tl)) return cudaErrorInvalidValue;
  switch (p.I / kGroup) {
    case 8: return down_ng<BITS, 8>(p, c, pdl, s);
    case 16: return down_ng<BITS, 16>(p, c, pdl, s);
    case 32: return down_ng<BITS, 32>(p, c, pdl, s);
    case 64: return down_ng<BITS, 64>(p, c, pdl, s);
    case 128: return down_ng<BITS, 128>(p, c, pdl, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

bool grouped_shapes_supported(int bits, int H, int I, int E, int K, int T) {
  if (bits != 2 && bits != 4) return false;  // this path has no 8-bit form (token by token instead)
  if (H < 512 || I < 512) return false;  // scale rows of at least 16 bytes (one tensor-copy line)
  if (T * K > kMaxTK || ((size_t)T * K + 2 * (size_t)E) * 4 > 200 * 1024) return false;
  const TcConfig gu = gu_config(bits, H), dn = dn_config(bits, I);
  return gu.tl > 0 && I % (8 * gu.tl) == 0 && dn.tl > 0 && H % (16 * dn.tl) == 0;
}

cudaError_t launch_grouped_select(const GroupedParams& p, bool pdl, cudaStream_t s) {
  cudaError_t e = set_carveout_max((const void*)topk_tokens_kernel);
  if (e != cudaSuccess) return e;
  if ((e = launch_pdl(topk_tokens_kernel, dim3(p.T), dim3(kGT), 0, s, pdl, p)) != cudaSuccess) return e;
  const size_t smem = ((size_t)p.T * p.K + 2 * (size_t)p.E) * sizeof(int);
  if ((e = set_smem((const void*)sort_pairs_kernel, smem)) != cudaSuccess) return e;
  if ((e = set_carveout_max((const void*)sort_pairs_kernel)) != cudaSuccess) return e;
  return launch_pdl(sort_pairs_kernel, dim3(1), dim3(kST), smem, s, pdl, p);
}

int grouped_router_split(int H, int E, int T) {
  const int blocks = ((E + 1 + kRtR - 1) / kRtR) * ((T + kRtT - 1) / kRtT);
  int n = 1;
  while (n < 16 && blocks * n * 2 <= 148 && H % (2 * n * 64) == 0) n *= 2;
  return n;
}

cudaError_t launch_grouped_router(const GroupedParams& p, const RouterBatch& rb, int bits, bool pdl, cudaStream_t s) {
  cudaError_t e = set_carveout_max((const void*)norm_digits_kernel);
  if (e != cudaSuccess) return e;
  if ((e = launch_pdl(norm_digits_kernel, dim3(kNormSplit, p.T), dim3(kGT), 0, s, pdl, p, rb, bits)) != cudaSuccess)
    return e;
  const size_t smem = (size_t)kRtR * (kRtK + 8) * 2 + (size_t)kRtT * (kRtK + 4) * 4;
  void (*k)(const GroupedParams, const RouterBatch) = router_gemm_kernel;
  if ((e = set_smem((const void*)k, smem)) != cudaSuccess) return e;
  if ((e = set_carveout_max((const void*)k)) != cudaSuccess) return e;
  return launch_pdl(k, dim3((p.E + 1 + kRtR - 1) / kRtR, (p.T + kRtT - 1) / kRtT, p.rt_split), dim3(kGT), smem, s,
                    pdl, p, rb);
}

cudaError_t launch_grouped_gateup(const GroupedParams& p, int bits, bool pdl, cudaStream_t s) {
  return bits == 4 ? gateup_bits_g<4>(p, pdl, s) : gateup_bits_g<2>(p, pdl, s);
}

cudaError_t launch_grouped_actq(const GroupedParams& p, int bits, bool pdl, cudaStream_t s) {
  const int warps = (p.T * p.K + p.T) * (p.I / kGroup);
  const int grid = (warps + kGT / 32 - 1) / (kGT / 32);
  void (*k)(const GroupedParams) = bits == 4 ? grouped_actq_kernel<4> : grouped_actq_kernel<2>;
  const cudaError_t e = set_carveout_max((const void*)k);
  return e != cudaSuccess ? e : launch_pdl(k, dim3(grid), dim3(kGT), 0, s, pdl, p);
}

cudaError_t launch_grouped_down(const GroupedParams& p, int bits, bool pdl, cudaStream_t s) {
  return bits == 4 ? down_bits_g<4>(p, pdl, s) : down_bits_g<2>(p, pdl, s);
}

cudaError_t launch_grouped_combine(const GroupedParams& p, bool pdl, cudaStream_t s) {
  const cudaError_t e = set_carveout_max((const void*)grouped_combine_kernel);
  return e != cudaSuccess ? e
                          : launch_pdl(grouped_combine_kernel, dim3((p.H / 4 + kGT - 1) / kGT, p.T), dim3(kGT), 0, s,
                                       pdl, p);
}

}  // namespace fmoe
