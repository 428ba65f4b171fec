// k_token.cu -- the MoE block for one token: a router kernel and one expert kernel.
//
// What is computed follows the Flash-MoE pages: "What is Flash-MoE"
// (a2a-mcp.org), MoE section (4 of 512 routed experts + one shared expert per
// layer), section 2 (group-wise affine codes, weight = code * scale + bias),
// section 3 (two-pass RMSNorm, fused SwiGLU, one combine pass of the weighted
// experts, the residual and the sigmoid-gated shared expert); the "Flash-MoE"
// wiki summary (jeongsk), per-layer pipeline (routing projection, softmax,
// top-K).
//
// tok_router_kernel: every CTA stages its rows of [W_r; w_sg] before the
// dependency wait, then computes sum(h^2) and its rows' dot products with
// gamma * h in one pass over h (the first pass of the RMSNorm), so that a
// logit is rsqrt(mean(h^2) + eps) * (w . (gamma * h)); the second pass
// applies the scale to the groups of x whose digits this CTA writes.  Its
// shared memory is small, so that under programmatic dependent launch its
// CTAs sit beside the previous token's expert kernel and their row copies
// overlap it.
//
// tok_expert_kernel: one CTA per SM, eight consumer warps and one producer
// warp.  Every CTA selects the experts from the logits itself (block-wide
// top-K), computes an equal share of the shared expert's and of the routed
// experts' gate/up rows (SwiGLU activations out to global memory), publishes
// that by an epoch-tagged flag, waits for every CTA's flag, turns all
// activations into digits, and computes its share of the output rows: down
// projection of every slot, weighted sum, sigma * shared, residual.  The
// producer streams the CTA's rows through a byte ring of shared memory with
// bulk copies (TMA engine): one chunk = a row range of one slot's gate and up
// (six copies) or of every slot's down matrix (three copies per slot); each
// chunk completes on its own "full" mbarrier and is handed back by the
// consumer warps on its "empty" mbarrier, so no block-wide barrier sits in the
// stream.  The shared expert's rows are requested before the dependency wait,
// the routed rows as soon as the routing is known, and the routed down rows
// are asked of L2 right after, to be copied into the ring as gate/up chunks
// free it.
//
// Dot products: sum_c (q_c s + b) x_c = s * sum_c q_c X_c * cscale + b * sum_c x_c
// per group of 64, with the integer sum on dp4a against 24-bit fixed-point
// digits of x (fmoe_device.cuh).
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "fmoe_internal.h"

namespace fmoe {
namespace {

// ------------------------------------------------------------------------------------------ router

constexpr int kRtThreads = 128;
constexpr int kRtMaxRows = 8;
constexpr int kRtSmemBudget = 32 * 1024;  // rows of the router per CTA, bf16

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// grid (ceil((E + 1 - row0) / rpc)): CTA b computes rows [row0 + b*rpc, +rpc) of [W_r; w_sg]
// (row E is the shared-gate vector), and the digits of groups b, b + grid, .. of x.
// kRtMaxF4: float4s of h per thread (H <= kRtMaxF4 * 512).
template <int BITS, int kRtMaxF4>
__global__ void __launch_bounds__(kRtThreads) tok_router_kernel(const TokRouterParams p) {
  extern __shared__ __align__(128) uint8_t sm[];
  __shared__ __align__(8) uint64_t s_bar;
  __shared__ float s_red[kRtThreads / 32][kRtMaxRows + 1];
  __shared__ __align__(16) float s_x[kRtThreads / 32][kGroup];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int H = p.H, E = p.E;
  const int r0 = p.row0 + blockIdx.x * p.rpc;
  const int nrows = max(0, min(p.rpc, E + 1 - r0));
  const uint32_t bar = smem_addr(&s_bar);
  if (tid == 0) {
    mbar_init(bar, 1);
    mbar_fence_init();
    if (nrows > 0) {  // weights: staged before the dependency wait
      const int nr = max(0, min(nrows, E - r0));  // routed rows; the rest is the shared-gate row
      const uint64_t pol = l2_policy_evict_first();
      mbar_expect_tx(bar, (uint32_t)nrows * H * 2);
      if (nr > 0) bulk_g2s(smem_addr(sm), p.w_router + (size_t)r0 * H, (uint32_t)nr * H * 2, bar, pol);
      if (nr < nrows) bulk_g2s(smem_addr(sm + (size_t)nr * H * 2), p.w_sgate, (uint32_t)H * 2, bar, pol);
    }
  }
  // pass 1: sum of squares of h, and each row's dot product with gamma * h.  Every
  // load is issued before any is used (a use waits for its load, and a warp issues in
  // order); columns past H read a clamped address and count 0.  gamma is a weight:
  // loaded before the wait.
  float4 hv[kRtMaxF4], gv[kRtMaxF4];
  if (p.gamma) {
#pragma unroll
    for (int j = 0; j < kRtMaxF4; ++j)
      gv[j] = __ldg(reinterpret_cast<const float4*>(p.gamma + min((tid + j * kRtThreads) * 4, H - 4)));
  } else {
#pragma unroll
    for (int j = 0; j < kRtMaxF4; ++j) gv[j] = make_float4(1.0f, 1.0f, 1.0f, 1.0f);
  }
  __syncthreads();
  pdl_wait();  // h may be the previous kernel's output
  const float* h = p.h;
#pragma unroll
  for (int j = 0; j < kRtMaxF4; ++j)
    hv[j] = __ldcg(reinterpret_cast<const float4*>(h + min((tid + j * kRtThreads) * 4, H - 4)));
  pdl_trigger();  // after the loads of h, so that they go out before the next kernel's weight copies
  if (blockIdx.x == 0 && tid == 0) *p.count = 0u;  // every kernel of the previous token is complete
  float ss = 0.0f;
#pragma unroll
  for (int j = 0; j < kRtMaxF4; ++j) {
    if ((tid + j * kRtThreads) * 4 >= H) hv[j] = make_float4(0.f, 0.f, 0.f, 0.f);
    ss = fmaf(hv[j].x, hv[j].x, ss);
    ss = fmaf(hv[j].y, hv[j].y, ss);
    ss = fmaf(hv[j].z, hv[j].z, ss);
    ss = fmaf(hv[j].w, hv[j].w, ss);
  }
  // v = gamma * h, kept in hv (pass 2 scales it by rstd)
#pragma unroll
  for (int j = 0; j < kRtMaxF4; ++j)
    hv[j] = make_float4(hv[j].x * gv[j].x, hv[j].y * gv[j].y, hv[j].z * gv[j].z, hv[j].w * gv[j].w);
  ss = warp_sum(ss);
  if (lane == 0) s_red[warp][kRtMaxRows] = ss;
  const bool ready = nrows == 0 || mbar_wait_bounded(bar, 0, p.err);
  if (ready) {
    // one row at a time in a loop that is not unrolled over the rows: this code runs
    // once per token, so it is kept short (it is fetched cold every time)
    const uint16_t* wr = reinterpret_cast<const uint16_t*>(sm);
#pragma unroll 1
    for (int r = 0; r < nrows; ++r) {
      float a = 0.0f;
#pragma unroll
      for (int j = 0; j < kRtMaxF4; ++j) {
        const int cc = min((tid + j * kRtThreads) * 4, H - 4);  // columns past H: v is 0 there
        const uint2 w = *reinterpret_cast<const uint2*>(wr + (size_t)r * H + cc);
        a = fmaf(bf_lo(w.x), hv[j].x, a);
        a = fmaf(bf_hi(w.x), hv[j].y, a);
        a = fmaf(bf_lo(w.y), hv[j].z, a);
        a = fmaf(bf_hi(w.y), hv[j].w, a);
      }
      a = warp_sum(a);
      if (lane == 0) s_red[warp][r] = a;
    }
  }
  __syncthreads();
  float sst = 0.0f;
#pragma unroll
  for (int w = 0; w < kRtThreads / 32; ++w) sst += s_red[w][kRtMaxRows];  // same order in every CTA
  const float rstd = p.norm ? 1.0f / sqrtf(sst / (float)H + p.eps) : 1.0f;
  if (ready && tid < nrows) {
    float d = 0.0f;
#pragma unroll
    for (int w = 0; w < kRtThreads / 32; ++w) d += s_red[w][tid];
    const int row = r0 + tid;
    p.logits[row] = fmaf(rstd, d, (row < E && p.bias) ? p.bias[row] : 0.0f);
  }
  // pass 2: x = h * rstd * gamma for the groups whose digits this CTA writes (group b,
  // b + grid, ..), from the registers of pass 1: thread tid holds columns
  // 4 tid + 512 j, i.e. elements 4 (tid % 16) .. + 3 of group tid / 16 + 8 j.  Up to
  // four groups per round are staged in shared memory, then one warp digitises each.
  const int NG = H / kGroup;
  for (int g0 = blockIdx.x; g0 < NG; g0 += gridDim.x * (kRtThreads / 32)) {
    __syncthreads();
#pragma unroll
    for (int w = 0; w < kRtThreads / 32; ++w) {
      const int g = g0 + gridDim.x * w;
      if (g < NG && tid / 16 == g % 8) {
#pragma unroll
        for (int j = 0; j < kRtMaxF4; ++j)
          if (j == g / 8) {
            const float4 v = hv[j];
            *reinterpret_cast<float4*>(&s_x[w][4 * (tid % 16)]) =
                make_float4(v.x * rstd, v.y * rstd, v.z * rstd, v.w * rstd);
          }
      }
    }
    __syncthreads();
    const int g = g0 + gridDim.x * warp;
    if (g < NG) {
      const float2 v = *reinterpret_cast<const float2*>(&s_x[warp][2 * lane]);
      xq_quantize_group<BITS>(v.x, v.y, g, NG, p.xq_limbs, p.xq_cs);
    }
  }
}

// Digits of a given x (the single-expert entry point); one warp per group.  CTA 0
// clears the expert kernel's arrival counter, as the router kernel does.
template <int BITS>
__global__ void __launch_bounds__(kRtThreads) tok_xq_kernel(const float* __restrict__ x, int H, uint8_t* limbs,
                                                           float2* cs, unsigned int* count) {
  pdl_wait();
  pdl_trigger();
  if (blockIdx.x == 0 && threadIdx.x == 0) *count = 0u;
  const int g = blockIdx.x * (kRtThreads / 32) + (threadIdx.x >> 5);
  if (g >= H / kGroup) return;  // warp-uniform
  const float2 v = __ldcg(reinterpret_cast<const float2*>(x + g * kGroup) + (threadIdx.x & 31));
  xq_quantize_group<BITS>(v.x, v.y, g, H / kGroup, limbs, cs);
}

// ------------------------------------------------------------------------------------------ expert kernel

constexpr int kXWarps = 8;                     // consumer warps
constexpr int kXThreads = (kXWarps + 1) * 32;  // + the producer warp
constexpr int kXSlots = 48;                    // chunks in flight at most (barrier pairs); >= 33 + a few
constexpr int kBarCons = 1;                    // named barrier of the consumer warps
constexpr int kBarAll = 2;                     // named barrier of consumers + producer
constexpr int kXMaxDRows = 128;                // output rows per down range
constexpr int kMaxSlots = 33;                  // K + shared
constexpr size_t kXSmemBudget = 184 * 1024;    // dynamic shared memory of the expert kernel
constexpr size_t kXChunkTarget = 32 * 1024;    // bytes per gate/up chunk, about

// The tensor maps of the staged arrays, [0] the routed bank, [1] the shared expert:
//   gu_codes  (RB / 8 u64, I rows, {gate, up}, experts)                 box (RB / 8, gbox, 2, 1)
//   gu_sb     (SB / 8 u64, {scale, bias}, {gate, up}, I rows, experts)  box (SB / 8, 2, 2, sbox, 1)
//   dn_codes  (RBD / 8 u64, H rows, experts)                           box (RBD / 8, dbox, 1)
// A box lands as [outer dims][..][row bytes]: gate/up codes as gate rows then up rows;
// the scale box row by row, each row as gate scales, gate biases, up scales, up biases.
struct TokMaps {
  CUtensorMap gu_codes[2];
  CUtensorMap gu_sb[2];
  CUtensorMap dn_codes[2];
};

// Block-wide top-K of logits [E] by the 256 consumer threads (E <= 1024), in two
// stages: each warp's K largest keys of its logits e = tid + 256 i into cand,
// then warp 0 the K largest candidates, the renormalised weights
// w_k = exp(l_k - l_0) / sum_j exp(l_j - l_0) and, with has_gate, w[K] =
// sigmoid(logits[E]).  Keys order by value, then lower index: one sort's result.
// Larger E: warp 0 alone (rescans).  Ends before the caller's next barrier.
__device__ __forceinline__ void consumer_topk(const float* logits, int E, int K, int has_gate, unsigned long long* cand,
                                              int* idx, float* w) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (E > 1024) {
    if (warp == 0) {
      int ik;
      float wk, sig;
      warp_topk(logits, E, K, has_gate, ik, wk, sig);
      if (lane < K) {
        idx[lane] = ik;
        w[lane] = wk;
      }
      if (lane == 0) w[K] = sig;
    }
    return;
  }
  // every load first (clamped index), then the keys: a use waits for its load
  const float zg = __ldcg(logits + E);
  float lv[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) lv[i] = __ldcg(logits + min(tid + 256 * i, E - 1));
  unsigned long long key[4], best = 0ull;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int e = tid + 256 * i;
    key[i] = e < E ? topk_key(lv[i], e) : 0ull;
    best = key[i] > best ? key[i] : best;
  }
#pragma unroll 1
  for (int k = 0; k < K; ++k) {
    const unsigned long long m = warp_max_key(best);
    if (lane == 0) cand[warp * K + k] = m;
    if (best == m && m != 0ull) {
      best = 0ull;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        key[i] = key[i] == m ? 0ull : key[i];
        best = key[i] > best ? key[i] : best;
      }
    }
  }
  named_bar_sync(kBarCons, kXWarps * 32);
  if (warp != 0) return;
  const int NC = kXWarps * K;  // candidates, <= 256
  unsigned long long ck[8];
  best = 0ull;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    ck[i] = lane + 32 * i < NC ? cand[lane + 32 * i] : 0ull;
    best = ck[i] > best ? ck[i] : best;
  }
  float top = 0.0f, mine = 0.0f;
  int mi = 0;
#pragma unroll 1
  for (int k = 0; k < K; ++k) {
    const unsigned long long m = warp_max_key(best);
    int e = m ? topk_key_index(m) : 0;
    const float v = topk_key_value(m);
    if (e < 0 || e >= E) e = 0;  // only with non-finite logits
    if (k == 0) top = v;
    if (lane == k) {
      mi = e;
      mine = v;
    }
    if (best == m && m != 0ull) {
      best = 0ull;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        ck[i] = ck[i] == m ? 0ull : ck[i];
        best = ck[i] > best ? ck[i] : best;
      }
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

// The CTA's work ranges, in units: shared-expert gate/up units [sh0, sh1) (a unit =
// RPP rows of gate and of up); routed gate/up units [rt0, rt1) of one slot, rslot
// (the CTAs are dealt out to the K slots in equal runs, so that a CTA's routed rows
// belong to one expert); output-row units [d0, d1) (a unit = DR rows).
struct Ranges {
  int sh0, sh1, rslot, rt0, rt1, d0, d1;
};

__device__ __forceinline__ Ranges cta_ranges(int b, int G, int K, int ups, int has_shared, int UD) {
  Ranges r;
  const int US = has_shared ? ups : 0;
  r.sh0 = (int)((long long)b * US / G);
  r.sh1 = (int)((long long)(b + 1) * US / G);
  r.rslot = (int)((long long)b * K / G);
  const int c0 = (int)(((long long)r.rslot * G + K - 1) / K);        // first CTA of the slot
  const int c1 = (int)(((long long)(r.rslot + 1) * G + K - 1) / K);  // one past its last
  r.rt0 = (int)((long long)(b - c0) * ups / (c1 - c0));
  r.rt1 = (int)((long long)(b - c0 + 1) * ups / (c1 - c0));
  r.d0 = (int)((long long)b * UD / G);
  r.d1 = (int)((long long)(b + 1) * UD / G);
  return r;
}

// A gate/up chunk: n units of one slot (K = the shared expert), from unit u0 of the slot.
struct GChunk {
  int slot, u0, n;
};

// The CTA's gate/up chunks in order: the shared expert's, then its routed slot's.
struct GChunkIt {
  int phase, u;
  __device__ __forceinline__ explicit GChunkIt(const Ranges& r) : phase(0), u(r.sh0) {}
  __device__ __forceinline__ bool next(GChunk& c, const Ranges& r, int K, int gmax_s, int gmax_r) {
    if (phase == 0) {
      if (u < r.sh1) {
        c = GChunk{K, u, min(gmax_s, r.sh1 - u)};
        u += c.n;
        return true;
      }
      phase = 1;
      u = r.rt0;
    }
    if (phase == 1 && u < r.rt1) {
      c = GChunk{r.rslot, u, min(gmax_r, r.rt1 - u)};
      u += c.n;
      return true;
    }
    phase = 2;
    return false;
  }
};

// Down chunk jd of the CTA: output-row range jd / NE (rows [d0*DR + range*dbox, +dbox),
// clipped to the CTA's rows), slot order within a range: the shared expert first.
__device__ __forceinline__ int down_slot(int pos, int K, int has_shared) {
  return has_shared ? (pos == 0 ? K : pos - 1) : pos;
}

// Ring placement: a chunk takes the virtual byte range [vs, vs + len), vs the end of
// the previous chunk padded so that the chunk never wraps; its buffer is
// ring + vs % RING.  Placement depends on the lengths only, so producer and
// consumers replay it alike.
struct RingPos {
  uint32_t vhead = 0;
  __device__ __forceinline__ uint32_t place(uint32_t len, uint32_t RING) {
    uint32_t vs = vhead;
    if (vs % RING + len > RING) vs = (vs / RING + 1) * RING;
    vhead = vs + len;
    return vs;
  }
};

// A producer's view of one ring: chunk j uses barrier pair j % NS, and may be issued
// once chunk j - NS is handed back and every older chunk still in use starts at most
// RING bytes before its end.  Every producer lane keeps the same state.
template <int NS>
struct RingProd {
  RingPos rp;
  uint32_t vstart[NS] = {};
  int tail = 0, j = 0;
  uint32_t RING;
  uint64_t* empty;
  // Places a chunk of len bytes; with may_wait false gives up (returns false) instead of
  // waiting; ok turns false when a wait runs out.
  __device__ __forceinline__ bool reserve(uint32_t len, bool may_wait, uint32_t& vs, bool& ok, int* err) {
    RingPos trial = rp;
    vs = trial.place(len, RING);
    while (tail < j && (tail <= j - NS || vs + len > vstart[tail % NS] + RING)) {
      if (!may_wait) return false;
      if (!mbar_wait_bounded(smem_addr(&empty[tail % NS]), (uint32_t)((tail / NS) & 1), err)) {
        ok = false;
        return false;
      }
      ++tail;
    }
    rp = trial;
    vstart[j % NS] = vs;
    return true;
  }
};

template <int BITS, int NG>
struct XCfg {
  using G = Geo<NG>;
  static constexpr int kLPR = G::kLanesPerRow, kRPP = G::kRowsPerPass, kGPL = G::kGroupsPerLane;
  static constexpr bool kRegDigits = kGPL <= 2;  // this lane's digits of x in registers (else read per group)
  static constexpr int kRB = NG * kGroup * BITS / 8;  // bytes of codes per gate/up row
  static constexpr int kSB = NG * 2;                 // bytes of scales per gate/up row
  static constexpr int kXChunks = NG * kGroup * BITS / 128;
  static constexpr int kXDigitBytes = NG * kGroupWords * 4;
};

// Staged layouts.  Gate/up chunk (box of gbox rows): gate codes [gbox][RB] | up codes |
// gate s [gbox][SB] | gate b | up s | up b.  Down chunk (one slot, dbox rows): codes
// [dbox][RBD] | s [dbox][SBD] | b [dbox][SBD], each part 128-byte aligned.
__device__ __forceinline__ uint32_t r128(uint32_t v) { return (v + 127u) & ~127u; }

template <int BITS, int NG, int DPPL>
__global__ void __launch_bounds__(kXThreads, 1) tok_expert_kernel(const TokExpertParams p,
                                                                  const __grid_constant__ TokMaps maps) {
  using C = XCfg<BITS, NG>;
  constexpr int LPR = C::kLPR, RPP = C::kRPP, GPL = C::kGPL;
  constexpr int RB = C::kRB, SB = C::kSB;
  extern __shared__ __align__(128) uint8_t sm[];
  __shared__ __align__(8) uint64_t s_full[kXSlots], s_empty[kXSlots];
  __shared__ __align__(8) uint64_t s_xbar;
  __shared__ __align__(8) uint64_t s_gss, s_gsr;   // gate/up scales: the shared expert's, the routed slot's
  __shared__ __align__(8) uint64_t s_dsp, s_dsr;   // down scales: the shared expert's, the routed ones
  __shared__ int s_idx[32];
  __shared__ float s_w[kMaxSlots];
  __shared__ unsigned long long s_cand[kXWarps * 32];
  __shared__ float s_dpart[2][kXMaxDRows];
  __shared__ int s_abort;
  __shared__ int s_issued;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int K = p.K, NE = K + p.has_shared, H = p.H, I = p.I;
  const int NGD = I / kGroup;
  const int ups = I / RPP;                        // gate/up units per slot
  const int DR = NGD >= 8 ? 1 : 8 / NGD;          // output rows per down unit (16-byte scale rows)
  const int RBD = I * BITS / 8, SBD = NGD * 2;     // bytes of codes / scales per down row
  const int chD = I * BITS / 128;                  // digit chunk scalars per slot
  const int dbox = p.dmax * DR;
  // a gate/up chunk's box: gmax_s units for the shared expert, gmax_r for the routed slot
  auto gbox_of = [&](int slot) { return (slot < K ? p.gmax_r : p.gmax_s) * RPP; };
  auto glen_of = [&](int gbox) { return r128(2u * gbox * RB); };
  const uint32_t dlen = r128((uint32_t)dbox * RBD);
  const int G = gridDim.x, b = blockIdx.x;
  const Ranges rg = cta_ranges(b, G, K, ups, p.has_shared, H / DR);
  const int drows_all = (rg.d1 - rg.d0) * DR;                // this CTA's output rows
  const int nranges = (drows_all + dbox - 1) / dbox;
  const int nd = nranges * NE;                               // down chunks (one per slot and row range)
  uint8_t* xd = sm;                                          // digits of x, then of the activations
  // scales: gate/up rows [sbox_s shared rows + sbox_r routed rows][4][SB] (gate s, gate b,
  // up s, up b of a row together), down [NE][scale, bias][drows][SBD]
  uint8_t* gsc = sm + p.xd_bytes;
  uint8_t* dsc = gsc + r128(4u * (p.sbox_s + p.sbox_r) * SB);
  uint8_t* ring = sm + p.xd_bytes + p.sc_bytes;
  const uint32_t RING = (uint32_t)p.ring_bytes;
  const uint32_t dslot = 2u * p.drows * SBD;                 // bytes per slot in the down scales

  if (tid == 0) {
    for (int i = 0; i < kXSlots; ++i) {
      mbar_init(smem_addr(&s_full[i]), 1);
      mbar_init(smem_addr(&s_empty[i]), kXWarps);
    }
    mbar_init(smem_addr(&s_xbar), 1);
    mbar_init(smem_addr(&s_gss), 1);
    mbar_init(smem_addr(&s_gsr), 1);
    mbar_init(smem_addr(&s_dsp), kXWarps * 32);  // one cp.async arrival per consumer thread
    mbar_init(smem_addr(&s_dsr), kXWarps * 32);
    mbar_fence_init();
    s_abort = 0;
    s_issued = 0;
  }
  __syncthreads();

  if (warp == kXWarps) {
    // ================================================================ producer warp (lane 0 issues)
    // One ring, chunks in order: the gate/up chunks (shared expert, then the routed slot),
    // then the down chunks (per row range, one per slot, the shared expert's first).
    // Every copy is a tensor copy of a whole box: the TMA engine spends about as long on
    // a small copy as on a large one, so copies are few and large.
    const uint64_t pol = l2_policy_evict_first();
    bool ok = true;
    RingProd<kXSlots> rpr;
    rpr.RING = RING;
    rpr.empty = s_empty;
    GChunkIt git(rg);
    GChunk gc;
    bool ghave = git.next(gc, rg, K, p.gmax_s, p.gmax_r);
    auto issue_g = [&](const GChunk& c, uint32_t vs) {
      const int gbox = gbox_of(c.slot);
      const bool routed = c.slot < K;
      if (lane == 0) {
        const uint32_t bar = smem_addr(&s_full[rpr.j % kXSlots]);
        mbar_expect_tx(bar, 2u * gbox * RB);
        tma_4d(smem_addr(ring + vs % RING), &maps.gu_codes[routed ? 0 : 1], c.u0 * RPP, 0, routed ? s_idx[c.slot] : 0,
               bar, pol);
      }
      __syncwarp();
      ++rpr.j;
    };
    auto issue_d = [&](int jd, uint32_t vs) {
      const int range = jd / NE, slot = down_slot(jd % NE, K, p.has_shared);
      const bool routed = slot < K;
      if (lane == 0) {
        const uint32_t bar = smem_addr(&s_full[rpr.j % kXSlots]);
        mbar_expect_tx(bar, (uint32_t)dbox * RBD);
        tma_3d(smem_addr(ring + vs % RING), &maps.dn_codes[routed ? 0 : 1], rg.d0 * DR + range * dbox,
               routed ? s_idx[slot] : 0, bar, pol);
      }
      __syncwarp();
      ++rpr.j;
    };
    // gate/up scales of a segment: one tensor copy of the segment's rows (whole box)
    auto issue_gs = [&](bool routed, int row0, uint32_t dst, uint64_t* bar_) {
      if (lane == 0) {
        const int box = routed ? p.sbox_r : p.sbox_s;
        const uint32_t bar = smem_addr(bar_);
        mbar_expect_tx(bar, 4u * box * SB);
        tma_5d(dst, &maps.gu_sb[routed ? 0 : 1], 0, 0, row0, routed ? s_idx[rg.rslot] : 0, bar, pol);
      }
      __syncwarp();
    };
    // L2 requests for this CTA's down rows of slot `slot` (codes, scales, biases), lanes base..base+2
    auto ask_l2_down = [&](int slot, int base) {
      if (lane >= base && lane < base + 3 && drows_all > 0) {
        const int m = lane - base;
        const bool routed = slot < K;
        const uint8_t* rec = routed ? p.routed.base + (long long)s_idx[slot] * p.routed.stride : p.shared.base;
        const long long* off = routed ? p.routed.off : p.shared.off;
        const long long unit = m == 0 ? RBD : SBD;
        prefetch_l2(rec + off[6 + m] + (long long)rg.d0 * DR * unit, (uint32_t)(drows_all * unit));
      }
    };
    // Before the dependency wait (weights only): the shared expert's gate/up scales and
    // chunks as far as they fit without waiting, and an L2 request for its down rows.
    uint32_t vs;
    if (p.has_shared && rg.sh1 > rg.sh0) issue_gs(false, rg.sh0 * RPP, smem_addr(gsc), &s_gss);
    while (ghave && gc.slot == K && rpr.reserve(glen_of(gbox_of(gc.slot)), false, vs, ok, p.err)) {
      issue_g(gc, vs);
      ghave = git.next(gc, rg, K, p.gmax_s, p.gmax_r);
    }
    if (p.has_shared) ask_l2_down(K, 0);
    pdl_wait();
    pdl_trigger();
    if (lane == 0) {  // the digits of x, written by the previous kernel
      const uint32_t bx = smem_addr(&s_xbar);
      mbar_expect_tx(bx, (uint32_t)(C::kXDigitBytes + C::kXChunks * 8));
      bulk_g2s(smem_addr(xd), p.xq_limbs, C::kXDigitBytes, bx, l2_policy_evict_last());
      bulk_g2s(smem_addr(xd + C::kXDigitBytes), p.xq_cs, C::kXChunks * 8, bx, l2_policy_evict_last());
    }
    named_bar_sync(kBarAll, kXThreads);  // the routing is in s_idx
    if (rg.rt1 > rg.rt0)
      issue_gs(true, rg.rt0 * RPP, smem_addr(gsc + 4u * p.sbox_s * SB), &s_gsr);
    while (ok && ghave && rpr.reserve(glen_of(gbox_of(gc.slot)), true, vs, ok, p.err)) {
      issue_g(gc, vs);
      ghave = git.next(gc, rg, K, p.gmax_s, p.gmax_r);
    }
    // every gate/up chunk is out: ask L2 for the routed down rows, then stage the down chunks
    for (int k = 0; k < K && 3 * k < 32; ++k) ask_l2_down(k, 3 * k);
    for (int jd = 0; ok && jd < nd && rpr.reserve(dlen, true, vs, ok, p.err); ++jd) issue_d(jd, vs);
    if (lane == 0) {
      s_issued = rpr.j;
      if (!ok) s_abort = 1;
    }
  } else {
    // ================================================================ consumer warps
    // Down scale arrays of the CTA's output rows, by cp.async from every consumer thread
    // (the shared expert's before the dependency wait, the routed ones once gate/up is
    // done, while the CTAs wait for one another).  Each thread arrives once per batch.
    const uint32_t dsa = smem_addr(dsc);
    auto cp_rows = [&](uint32_t dst, const uint8_t* src, uint32_t bytes) {
      for (uint32_t o = 16u * tid; o < bytes; o += 16u * kXWarps * 32) cp_async16(dst + o, src + o);
    };
    auto cp_down_scales = [&](int slot) {
      const bool routed = slot < K;
      const uint8_t* rec = routed ? p.routed.base + (long long)s_idx[slot] * p.routed.stride : p.shared.base;
      const long long* off = routed ? p.routed.off : p.shared.off;
#pragma unroll 1
      for (int m = 0; m < 2; ++m)
        cp_rows(dsa + slot * dslot + m * p.drows * SBD, rec + off[7 + m] + (long long)rg.d0 * DR * SBD,
                (uint32_t)drows_all * SBD);
    };
    if (p.has_shared) cp_down_scales(K);
    cp_async_arrive(smem_addr(&s_dsp));
    pdl_wait();  // the router's logits and the digits of x are complete
    pdl_trigger();
    if (p.logits && !p.route_idx) {
      consumer_topk(p.logits, p.E, K, p.has_shared, s_cand, s_idx, s_w);
    } else if (warp == 0) {
      int e = 0;
      float wv = 1.0f;
      if (lane < K) {
        e = p.route_idx ? __ldcg(p.route_idx + lane) : p.fixed_expert;
        wv = p.route_w ? __ldcg(p.route_w + lane) : 1.0f;
      }
      const float zg = (p.has_shared && p.logits) ? __ldcg(p.logits + p.E) : 0.0f;
      if (lane < K) {
        s_idx[lane] = e;
        s_w[lane] = wv;
      }
      if (lane == 0) s_w[K] = p.has_shared ? (p.logits ? 1.0f / (1.0f + expf(-zg)) : 1.0f) : 0.0f;
    }
    if (warp == 0 && lane < K) {
      const int e = s_idx[lane];
      if (e < 0 || e >= p.routed.num_experts) {
        atomicExch(p.err, kDevBadIndex);
        s_idx[lane] = 0;
      }
    }
    __syncwarp();
    named_bar_sync(kBarAll, kXThreads);
    if (b == 0 && tid < K) {
      if (p.idx_out) p.idx_out[tid] = s_idx[tid];
      if (p.w_out) p.w_out[tid] = s_w[tid];
    }

    // this lane's groups of x and their digits, for every gate/up row it computes
    const int sub = lane / LPR, gl = lane % LPR;
    bool ok = mbar_wait_bounded(smem_addr(&s_xbar), 0, p.err);
    const uint32_t* xs = reinterpret_cast<const uint32_t*>(xd);
    const float2* xcs = reinterpret_cast<const float2*>(xd + C::kXDigitBytes);
    uint32_t L[C::kRegDigits ? GPL : 1][48];
    float2 cs[GPL];
#pragma unroll
    for (int q = 0; q < GPL; ++q) {
      const int g = gl + LPR * q;
      if constexpr (C::kRegDigits) load_group_limbs(xs, g, NG, L[q]);
      cs[q] = group_scalars<BITS>(xcs, g);
    }

    // ---- gate/up + SwiGLU: warp w takes tasks w, w + 8, .. of a chunk (a task = RPP rows)
    RingPos rp;
    int jc = 0;  // chunk index (both kinds)
    {
      GChunkIt git(rg);
      GChunk c;
      for (; git.next(c, rg, K, p.gmax_s, p.gmax_r); ++jc) {
        const int gbox = gbox_of(c.slot);
        const uint32_t vs = rp.place(glen_of(gbox), RING);
        const bool routed_c = c.slot < K;
        if (ok && !mbar_wait_bounded(smem_addr(routed_c ? &s_gsr : &s_gss), 0, p.err)) ok = false;
        if (ok && !mbar_wait_bounded(smem_addr(&s_full[jc % kXSlots]), (uint32_t)((jc / kXSlots) & 1), p.err))
          ok = false;
        const uint8_t* buf = ring + vs % RING;
        // this chunk's rows among the CTA's staged scale rows
        const int crow = routed_c ? p.sbox_s + (c.u0 - rg.rt0) * RPP : (c.u0 - rg.sh0) * RPP;
        for (int t = warp; ok && t < c.n; t += kXWarps) {
          const int rr = t * RPP + sub;  // row within the chunk
          const uint16_t* sc = reinterpret_cast<const uint16_t*>(gsc + (size_t)(crow + rr) * 4 * SB);
          float ag = 0.0f, au = 0.0f;
#pragma unroll
          for (int q = 0; q < GPL; ++q) {
            const int g = gl + LPR * q;
            uint4 q0, q1, v0, v1;
            load_group_codes<BITS>(buf + rr * RB, g, q0, q1);
            load_group_codes<BITS>(buf + gbox * RB + rr * RB, g, v0, v1);
            const float gs = bf16_to_f32(sc[g]);
            const float gb = bf16_to_f32(sc[SB / 2 + g]);
            const float us = bf16_to_f32(sc[SB + g]);
            const float ub = bf16_to_f32(sc[3 * SB / 2 + g]);
            float Sg, Su;
            if constexpr (C::kRegDigits) {
              Sg = group_dot<BITS>(q0, q1, L[q]);
              Su = group_dot<BITS>(v0, v1, L[q]);
            } else {
              uint32_t Lt[48];
              load_group_limbs(xs, g, NG, Lt);
              Sg = group_dot<BITS>(q0, q1, Lt);
              Su = group_dot<BITS>(v0, v1, Lt);
            }
            ag = fmaf(gs, cs[q].x * Sg, fmaf(gb, cs[q].y, ag));
            au = fmaf(us, cs[q].x * Su, fmaf(ub, cs[q].y, au));
          }
#pragma unroll
          for (int o = LPR / 2; o > 0; o >>= 1) {
            ag += __shfl_xor_sync(0xffffffffu, ag, o);
            au += __shfl_xor_sync(0xffffffffu, au, o);
          }
          if (gl == 0) p.act[(size_t)c.slot * I + (size_t)c.u0 * RPP + rr] = ag / (1.0f + expf(-ag)) * au;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_addr(&s_empty[jc % kXSlots]));
      }
    }

    // ---- the routed down scales (needed only after the hand-off), then the hand-off:
    // count this CTA in, wait until every CTA is in.  One thread each (consumer threads
    // issue no bulk copies, so their fences do not wait on any).
#pragma unroll 1
    for (int k = 0; k < K; ++k) cp_down_scales(k);
    cp_async_arrive(smem_addr(&s_dsr));
    named_bar_sync(kBarCons, kXWarps * 32);
    if (tid == 0) {
      __threadfence();
      atomicAdd(p.count, 1u);
      if (!count_wait_bounded(p.count, (unsigned)G, p.err)) s_abort = 1;
    }
    named_bar_sync(kBarCons, kXWarps * 32);
    if (s_abort) ok = false;

    // ---- digits of every slot's activations, into the digits region (x is in registers now)
    uint8_t* dl = xd;                                                                  // [NE][NGD * 192]
    float2* dcs = reinterpret_cast<float2*>(xd + (size_t)NE * NGD * kGroupWords * 4);  // [NE][chD]
    {
      // this warp's groups q = warp + 8 i, four at a time; the next four are loaded before
      // the current four are digitised (a use waits for its load)
      const int nq = NE * NGD, mine = (nq - warp + kXWarps - 1) / kXWarps;
      float2 cur[4], nxt[4];
      auto load4 = [&](int i0, float2 (&v)[4]) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int q = min(warp + kXWarps * (i0 + k), nq - 1);
          v[k] = __ldcg(reinterpret_cast<const float2*>(p.act + (size_t)q * kGroup) + lane);
        }
      };
      load4(0, cur);
#pragma unroll 1
      for (int i0 = 0; i0 < mine; i0 += 4) {
        if (i0 + 4 < mine) load4(i0 + 4, nxt);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          if (i0 + k < mine) {
            const int q = warp + kXWarps * (i0 + k), s = q / NGD, g = q - s * NGD;
            xq_quantize_group<BITS>(cur[k].x, cur[k].y, g, NGD, dl + (size_t)s * NGD * kGroupWords * 4,
                                    dcs + (size_t)s * chD);
          }
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) cur[k] = nxt[k];
      }
    }
    named_bar_sync(kBarCons, kXWarps * 32);

    // ---- down + combine.  The (slot, group) pairs split into P parts of at most 64,
    // each taken by 8 / P warps; lane l owns pairs l and l + 32 of its part.
    const int NP = NE * NGD;
    const int P = NP > 64 ? 2 : 1;
    const int part = warp / (kXWarps / P), wi = warp % (kXWarps / P), nw = kXWarps / P;
    const int pb = part == 0 ? 0 : (NP + 1) / 2, pe = P == 1 ? NP : (part == 0 ? (NP + 1) / 2 : NP);
    uint32_t LD[DPPL][48];
    float2 csd[DPPL];
    float wq[DPPL];
    int qs[DPPL], qg[DPPL];
#pragma unroll
    for (int m = 0; m < DPPL; ++m) {
      const int q = pb + lane + 32 * m;
      const bool has = q < pe;
      const int s = has ? q / NGD : 0, g = has ? q - (q / NGD) * NGD : 0;
      load_group_limbs(reinterpret_cast<const uint32_t*>(dl + (size_t)s * NGD * kGroupWords * 4), g, NGD, LD[m]);
      csd[m] = group_scalars<BITS>(dcs + (size_t)s * chD, g);
      wq[m] = has ? s_w[s] : 0.0f;
      qs[m] = s;
      qg[m] = g;
    }
    if (ok && !(mbar_wait_bounded(smem_addr(&s_dsp), 0, p.err) && mbar_wait_bounded(smem_addr(&s_dsr), 0, p.err)))
      ok = false;
    for (int range = 0; range < nranges; ++range) {
      // the range's NE chunks, in issue order; this lane's slots' buffers
      const uint8_t* sbuf[DPPL];
#pragma unroll
      for (int m = 0; m < DPPL; ++m) sbuf[m] = ring;
      const int j0 = jc;
      for (int k = 0; k < NE; ++k, ++jc) {
        const uint32_t vs = rp.place(dlen, RING);
        const int slot = down_slot(k, K, p.has_shared);
#pragma unroll
        for (int m = 0; m < DPPL; ++m)
          if (qs[m] == slot) sbuf[m] = ring + vs % RING;
        if (ok && !mbar_wait_bounded(smem_addr(&s_full[jc % kXSlots]), (uint32_t)((jc / kXSlots) & 1), p.err))
          ok = false;
      }
      const int rows = min(dbox, drows_all - range * dbox);
      for (int rr = wi; ok && rr < rows; rr += nw) {
        float acc = 0.0f;
#pragma unroll
        for (int m = 0; m < DPPL; ++m) {
          const uint8_t* sb = sbuf[m];
          const int g = qg[m];
          const uint4 q0 = *reinterpret_cast<const uint4*>(sb + rr * RBD + g * (kGroup * BITS / 8));
          const uint4 q1 = BITS == 4 ? *reinterpret_cast<const uint4*>(sb + rr * RBD + g * (kGroup * BITS / 8) + 16) : q0;
          const uint8_t* ss_ = dsc + qs[m] * dslot + (size_t)(range * dbox + rr) * SBD;
          const float sc = bf16_to_f32(reinterpret_cast<const uint16_t*>(ss_)[g]);
          const float bi = bf16_to_f32(reinterpret_cast<const uint16_t*>(ss_ + p.drows * SBD)[g]);
          const float S = group_dot<BITS>(q0, q1, LD[m]);
          acc = fmaf(wq[m], fmaf(sc, csd[m].x * S, bi * csd[m].y), acc);
        }
        acc = warp_sum(acc);
        if (lane == 0) s_dpart[part][rr] = acc;
      }
      __syncwarp();
      if (lane == 0)
        for (int k = 0; k < NE; ++k) mbar_arrive(smem_addr(&s_empty[(j0 + k) % kXSlots]));
      named_bar_sync(kBarCons, kXWarps * 32);
      if (ok)
        for (int rr = tid; rr < rows; rr += kXWarps * 32) {
          const int row = rg.d0 * DR + range * dbox + rr;
          const float y = P == 2 ? s_dpart[0][rr] + s_dpart[1][rr] : s_dpart[0][rr];
          p.out[row] = (p.resid ? __ldcg(p.resid + row) : 0.0f) + y;
        }
      named_bar_sync(kBarCons, kXWarps * 32);
    }
    if (!ok && tid == 0) s_abort = 1;
  }
  // A CTA that gave up a wait lets the copies it issued land before it exits.
  __syncthreads();
  if (s_abort && tid == 0) {
    for (int q = s_issued > kXSlots ? s_issued - kXSlots : 0; q < s_issued; ++q)
      mbar_wait_bounded(smem_addr(&s_full[q % kXSlots]), (uint32_t)((q / kXSlots) & 1), p.err);
    mbar_wait_bounded(smem_addr(&s_xbar), 0, p.err);
    if (p.has_shared && rg.sh1 > rg.sh0) mbar_wait_bounded(smem_addr(&s_gss), 0, p.err);
    if (rg.rt1 > rg.rt0) mbar_wait_bounded(smem_addr(&s_gsr), 0, p.err);
  }
  if (s_abort && tid < kXWarps * 32) {  // every consumer thread's cp.async copies
    mbar_wait_bounded(smem_addr(&s_dsp), 0, p.err);
    mbar_wait_bounded(smem_addr(&s_dsr), 0, p.err);
  }
}

size_t round128(size_t v) { return (v + 127) / 128 * 128; }

// The two-kernel path stages every array by tensor copies of whole boxes, which needs:
// rows of at most 2048 bytes of codes, at least 16 bytes of scales, and a record
// layout in which up's arrays sit at one distance from gate's, and each bias array at
// one distance from its scale array.
bool tok_layout_ok(const BankRef& r, int bits, int H, int I) {
  const long long NG = H / kGroup, NGD = I / kGroup;
  if ((long long)H * bits / 8 > 2048 || (long long)I * bits / 8 > 2048 || NG * 2 < 16 || NGD * 2 < 16) return false;
  const long long* o = r.off;
  const long long gu = o[3] - o[0], gus = o[4] - o[1], sb = o[2] - o[1];
  return gu > 0 && gus > 0 && sb > 0 && o[5] - o[2] == gus && o[5] - o[4] == sb && o[8] > o[7];
}

bool encode_tok_maps(TokMaps& M, const TokExpertParams& p, int bits) {
  const int H = p.H, I = p.I, NG = H / kGroup, NGD = I / kGroup;
  const long long RB = (long long)H * bits / 8, SB = NG * 2, RBD = (long long)I * bits / 8;
  const int LPR = NG < 32 ? NG : 32, RPP = 32 / LPR, DR = NGD >= 8 ? 1 : 8 / NGD;
  const int dbox = p.dmax * DR;
  if (p.gmax_r * RPP > 256 || p.gmax_s * RPP > 256 || dbox > 256 || p.sbox_r > 256 || p.sbox_s > 256) return false;
  for (int bk = 0; bk < 2; ++bk) {
    const BankRef& r = bk == 0 ? p.routed : p.shared;
    if (!tok_layout_ok(r, bits, H, I)) return false;
    const long long* o = r.off;
    const cuuint64_t ne = bk == 0 ? (cuuint64_t)p.routed.num_experts : 1;
    const cuuint64_t est = bk == 0 ? (cuuint64_t)r.stride : 16;
    {
      const int gbox = (bk == 0 ? p.gmax_r : p.gmax_s) * RPP;
      const cuuint64_t dims[4] = {(cuuint64_t)(RB / 8), (cuuint64_t)I, 2, ne};
      const cuuint64_t st[3] = {(cuuint64_t)RB, (cuuint64_t)(o[3] - o[0]), est};
      const cuuint32_t box[4] = {(cuuint32_t)(RB / 8), (cuuint32_t)gbox, 2, 1};
      if (!encode_map(&M.gu_codes[bk], r.base + o[0], 4, dims, st, box)) return false;
    }
    {
      const int sbox = bk == 0 ? p.sbox_r : p.sbox_s;
      const cuuint64_t dims[5] = {(cuuint64_t)(SB / 8), 2, 2, (cuuint64_t)I, ne};
      const cuuint64_t st[4] = {(cuuint64_t)(o[2] - o[1]), (cuuint64_t)(o[4] - o[1]), (cuuint64_t)SB, est};
      const cuuint32_t box[5] = {(cuuint32_t)(SB / 8), 2, 2, (cuuint32_t)(sbox > 0 ? sbox : 1), 1};
      if (!encode_map(&M.gu_sb[bk], r.base + o[1], 5, dims, st, box)) return false;
    }
    {
      const cuuint64_t dims[3] = {(cuuint64_t)(RBD / 8), (cuuint64_t)H, ne};
      const cuuint64_t st[2] = {(cuuint64_t)RBD, est};
      const cuuint32_t box[3] = {(cuuint32_t)(RBD / 8), (cuuint32_t)dbox, 1};
      if (!encode_map(&M.dn_codes[bk], r.base + o[6], 3, dims, st, box)) return false;
    }
  }
  return true;
}

template <int BITS, int NG>
cudaError_t expert_ng(const TokExpertParams& p, const TokMaps& m, int dppl, size_t smem, int grid, bool pdl,
                      cudaStream_t s) {
  void (*k)(const TokExpertParams, const TokMaps) =
      dppl == 1 ? tok_expert_kernel<BITS, NG, 1> : tok_expert_kernel<BITS, NG, 2>;
  cudaError_t e = set_smem((const void*)k, smem);
  if (e == cudaSuccess) e = set_carveout_max((const void*)k);
  if (e != cudaSuccess) return e;
  return launch_pdl(k, dim3(grid), dim3(kXThreads), smem, s, pdl, p, m);
}

template <int BITS>
cudaError_t expert_bits(const TokExpertParams& p, const TokMaps& m, int dppl, size_t smem, int grid, bool pdl,
                        cudaStream_t s) {
  switch (p.H / kGroup) {
    case 2: return expert_ng<BITS, 2>(p, m, dppl, smem, grid, pdl, s);
    case 4: return expert_ng<BITS, 4>(p, m, dppl, smem, grid, pdl, s);
    case 8: return expert_ng<BITS, 8>(p, m, dppl, smem, grid, pdl, s);
    case 16: return expert_ng<BITS, 16>(p, m, dppl, smem, grid, pdl, s);
    case 32: return expert_ng<BITS, 32>(p, m, dppl, smem, grid, pdl, s);
    case 64: return expert_ng<BITS, 64>(p, m, dppl, smem, grid, pdl, s);
    case 128: return expert_ng<BITS, 128>(p, m, dppl, smem, grid, pdl, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      enc = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return enc;
}

// One map over 8-byte elements: dims[0] elements per row, then the outer dims with
// their byte strides; box: dims[0] x box_rows x the outer dims' full extents (last: 1).
bool encode_map(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims, const cuuint64_t* strides,
                const cuuint32_t* box) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint32_t es[5] = {1, 1, 1, 1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT64, rank, const_cast<void*>(base), dims, strides, box, es,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}


// Shared memory of the expert kernel: the digits region (x, later the activations) and
// one ring for the staged chunks.  A down range's NE chunks are in the ring together,
// so a range holds at most half of it.
TokPlan plan_token(int bits, int H, int I, int K, int has_shared) {
  TokPlan pl{};
  if (H % kGroup || I % kGroup || H < 2 * kGroup || I < 2 * kGroup || K < 1 || K > 32) return pl;
  const int NG = H / kGroup, NGD = I / kGroup, NE = K + has_shared;
  const int LPR = NG < 32 ? NG : 32, RPP = 32 / LPR;
  const size_t RB = (size_t)H * bits / 8, SB = (size_t)NG * 2;
  const size_t chX = (size_t)H * bits / 128, chD = (size_t)I * bits / 128;
  const size_t xd = round128(std::max((size_t)NG * kGroupWords * 4 + chX * 8,
                                      (size_t)NE * ((size_t)NGD * kGroupWords * 4 + chD * 8)));
  if (xd + 4096 > kXSmemBudget || NE + 4 > kXSlots) return pl;
  size_t ring = (kXSmemBudget - xd) / 128 * 128;
  int grid = num_sms();
  if (grid > kMaxTokenCtas) grid = kMaxTokenCtas;
  const int DR = NGD >= 8 ? 1 : 8 / NGD;
  const size_t RBD = (size_t)I * bits / 8, SBD = (size_t)NGD * 2;
  // gate/up chunks: at most about kXChunkTarget bytes, the CTA's average range split
  // into equal chunks (a tensor copy moves a whole box, so uneven tails would fetch
  // rows of the next range)
  const size_t unitG = RPP * 2 * (RB + 2 * SB);
  const int cap = (int)std::max<size_t>(1, std::min<size_t>(std::min(kXChunkTarget, ring / 4) / unitG, 256 / RPP));
  const int ups = I / RPP;
  if (grid < K) return pl;
  // the routed units of a slot are dealt out to its run of grid / K CTAs
  const int per_r = (ups + grid / K - 1) / (grid / K), per_s = has_shared ? (ups + grid - 1) / grid : 0;
  auto even_r = [&](int avg) {
    avg = std::max(1, avg);
    const int n = (avg + cap - 1) / cap;
    return (avg + n - 1) / n;
  };
  const int gmax_r = even_r(per_r), gmax_s = has_shared ? even_r(per_s) : 1;
  const size_t glen = round128(2 * (size_t)std::max(gmax_r, gmax_s) * RPP * RB);
  // scales of the CTA's rows: gate/up [sbox_s + sbox_r rows][4][SB], down [NE][2][drows][SBD]
  const int UD = H / DR, dshare = (UD + grid - 1) / grid;
  const int sbox_s = per_s * RPP, sbox_r = per_r * RPP;
  const int drows = dshare * DR;
  const size_t sc = round128(4 * (size_t)(sbox_s + sbox_r) * SB) + round128((size_t)NE * 2 * drows * SBD);
  if (xd + sc + glen > kXSmemBudget) return pl;
  ring = (kXSmemBudget - xd - sc) / 128 * 128;
  // down ranges: the CTA's whole share when its NE chunks fit in half the ring
  auto dlen_of = [&](int dm) { return round128((size_t)dm * DR * RBD); };
  int dmax = std::min(dshare, std::min(kXMaxDRows, 256) / DR);
  while (dmax > 1 && (size_t)NE * dlen_of(dmax) > ring / 2) --dmax;
  const int NP = NE * NGD, part = NP > 64 ? (NP + 1) / 2 : NP;
  if (glen > ring || (size_t)NE * dlen_of(dmax) > ring || NP > 128) return pl;
  pl.ok = true;
  pl.grid = grid;
  pl.gmax_s = gmax_s;
  pl.gmax_r = gmax_r;
  pl.dmax = dmax;
  pl.xd_bytes = (int)xd;
  pl.sc_bytes = (int)sc;
  pl.sbox_s = sbox_s;
  pl.sbox_r = sbox_r;
  pl.drows = drows;
  pl.ring_bytes = (int)ring;
  pl.dppl = (part + 31) / 32;
  pl.smem = xd + sc + ring;
  return pl;
}

bool token_path_supported(int bits, int H, int I, int K, int has_shared, const BankRef& routed, const BankRef& shared) {
  if (bits != 2 && bits != 4) return false;  // this path has no 8-bit form
  return plan_token(bits, H, I, K, has_shared).ok && tok_layout_ok(routed, bits, H, I) &&
         tok_layout_ok(shared, bits, H, I);
}

cudaError_t launch_tok_router(TokRouterParams p, int bits, bool pdl, cudaStream_t s) {
  const int rows = p.E + 1 - p.row0;
  int rmax = kRtSmemBudget / (2 * p.H);
  rmax = rmax < 1 ? 1 : (rmax > kRtMaxRows ? kRtMaxRows : rmax);
  const int nsm = num_sms();
  int rpc = (rows + nsm - 1) / nsm;
  rpc = rpc < 1 ? 1 : (rpc > rmax ? rmax : rpc);
  int grid = (rows + rpc - 1) / rpc;
  const int NG = p.H / kGroup;
  if (grid < NG && grid < nsm) grid = NG < nsm ? NG : nsm;  // spread the digit groups too
  p.rpc = rpc;
  const size_t smem = (size_t)rpc * p.H * 2;
  void (*k)(const TokRouterParams) = p.H <= 8 * 4 * kRtThreads
                                        ? (bits == 4 ? tok_router_kernel<4, 8> : tok_router_kernel<2, 8>)
                                        : (bits == 4 ? tok_router_kernel<4, 16> : tok_router_kernel<2, 16>);
  cudaError_t e = set_smem((const void*)k, smem);
  if (e == cudaSuccess) e = set_carveout_max((const void*)k);
  if (e != cudaSuccess) return e;
  return launch_pdl(k, dim3(grid), dim3(kRtThreads), smem, s, pdl, p);
}

cudaError_t launch_tok_xq(const float* x, int H, int bits, uint8_t* limbs, float2* cs, unsigned int* count, bool pdl,
                          cudaStream_t s) {
  const int grid = (H / kGroup + kRtThreads / 32 - 1) / (kRtThreads / 32);
  void (*k)(const float*, int, uint8_t*, float2*, unsigned int*) = bits == 4 ? tok_xq_kernel<4> : tok_xq_kernel<2>;
  cudaError_t e = set_carveout_max((const void*)k);
  if (e != cudaSuccess) return e;
  return launch_pdl(k, dim3(grid), dim3(kRtThreads), 0, s, pdl, x, H, limbs, cs, count);
}

cudaError_t launch_tok_expert(TokExpertParams p, int bits, bool pdl, cudaStream_t s) {
  const TokPlan pl = plan_token(bits, p.H, p.I, p.K, p.has_shared);
  if (!pl.ok) return cudaErrorInvalidValue;
  p.gmax_s = pl.gmax_s;
  p.gmax_r = pl.gmax_r;
  p.dmax = pl.dmax;
  p.xd_bytes = pl.xd_bytes;
  p.sc_bytes = pl.sc_bytes;
  p.sbox_s = pl.sbox_s;
  p.sbox_r = pl.sbox_r;
  p.drows = pl.drows;
  p.ring_bytes = pl.ring_bytes;
  TokMaps m;
  memset(&m, 0, sizeof(m));
  if (!encode_tok_maps(m, p, bits)) return cudaErrorNotSupported;
  return bits == 4 ? expert_bits<4>(p, m, pl.dppl, pl.smem, pl.grid, pdl, s)
                   : expert_bits<2>(p, m, pl.dppl, pl.smem, pl.grid, pdl, s);
}

}  // namespace fmoe
