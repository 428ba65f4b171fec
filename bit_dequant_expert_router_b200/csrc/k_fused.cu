// k_fused.cu -- the whole MoE block as one persistent kernel, for a sequence of steps.
//
// One step is one token through one layer: RMSNorm, router GEMV, softmax/top-K,
// gate/up + SwiGLU of the K routed experts and the shared expert, down and the
// weighted combine with the sigmoid-gated shared expert and the residual
// ("What is Flash-MoE" (a2a-mcp.org), MoE section and sections 2-3; the
// per-layer pipeline of the "Flash-MoE" wiki summary (jeongsk)).  The pages run
// these as separate GPU dispatches with the top-K on the CPU in between; here
// one CTA per SM carries every step of a sequence.
//
// A step has three all-to-all exchanges between CTAs: the router logits (each
// CTA computes a few rows, every CTA needs all of them for the top-K), the
// SwiGLU activations (every CTA needs all of them for its down rows) and, in a
// stack of layers, the output vector (the next layer's input).  Each goes
// through a workspace array of 8-byte words {value, epoch}: the producer stores
// the word once, consumers poll until the epoch of the step appears.  The word
// is a single 64-bit access, so a matching epoch is its own proof that the
// value is current: no grid barrier, counter or memory fence is on the path.
// Arrays alternate by step parity; a CTA cannot run two steps ahead of another
// (each step consumes data of every CTA), so two copies suffice.  Epochs are a
// per-workspace count of steps (WsControl::epoch), advanced by CTA 0 on exit.
//
// The bytes of a step fall into two kinds.  The router rows, the shared
// expert's gate/up rows and the shared expert's down rows do not depend on the
// routing, so a CTA requests its share of them for step s+1 as soon as its
// gate/up work of step s is done.  The routed experts' gate/up rows stream
// through a ring of chunk buffers, and their down rows land in a separate
// region while gate/up is still running, so the down phase computes from
// shared memory.
//
// Dot products use the per-group fold of fmoe_device.cuh:
//   sum_c (q_c s + b) x_c = s * sum_c q_c x_c + b * sum_c x_c
// with exact dp4a integer sums against a 3-digit fixed-point x.
#include "fmoe_internal.h"

namespace fmoe {
namespace {

constexpr int kFW = kFusedWarps;
constexpr int kFT = kFW * 32;

// ---- epoch-tagged words: low 32 bits the value, high 32 bits the epoch
__device__ __forceinline__ void st_tagged(unsigned long long* p, float v, unsigned ep) {
  const unsigned long long w = ((unsigned long long)ep << 32) | __float_as_uint(v);
  asm volatile("st.relaxed.gpu.global.b64 [%0], %1;" ::"l"(p), "l"(w) : "memory");
}

__device__ __forceinline__ void ld_tagged2(const unsigned long long* p, unsigned long long& a, unsigned long long& b) {
  asm volatile("ld.relaxed.gpu.global.v2.b64 {%0, %1}, [%2];" : "=l"(a), "=l"(b) : "l"(p) : "memory");
}

__device__ __forceinline__ unsigned long long ld_tagged(const unsigned long long* p) {
  unsigned long long a;
  asm volatile("ld.relaxed.gpu.global.b64 %0, [%1];" : "=l"(a) : "l"(p) : "memory");
  return a;
}

__device__ __forceinline__ unsigned tag_of(unsigned long long w) { return (unsigned)(w >> 32); }
__device__ __forceinline__ float val_of(unsigned long long w) { return __uint_as_float((unsigned)w); }

// Polls n (even, 16-byte aligned) tagged words until all carry epoch ep; the
// values go to v[0..n).  Bounded by kWaitNs; false (and the error word set) on timeout.
template <int N>
__device__ __forceinline__ bool poll_tagged(const unsigned long long* p, unsigned ep, float (&v)[N], int* err) {
  unsigned long long t0 = 0;
  for (;;) {
    bool all = true;
#pragma unroll
    for (int i = 0; i < N; i += 2) {
      unsigned long long a, b;
      ld_tagged2(p + i, a, b);
      all = all && tag_of(a) == ep && tag_of(b) == ep;
      v[i] = val_of(a);
      v[i + 1] = val_of(b);
    }
    if (all) return true;
    if (t0 == 0) t0 = global_ns();
    else if (global_ns() - t0 > kWaitNs) {
      atomicExch(err, kDevTimeout);
      return false;
    }
    __nanosleep(64);  // back off: polling loads compete with the copies and loads of other warps
  }
}

struct Item {
  int kind;   // 0: router rows, 1: gate/up rows
  int slot;   // gate/up: expert slot (K = shared)
  int row0;
  int rows;
  int rbase;  // gate/up: index of the item's first row among this CTA's gate/up rows
};

// Shapes the copy helpers need (kept out of line: the kernel runs each
// phase once per step, so its code is kept small enough to stay in the
// instruction cache).
struct CopyShape {
  int E, H, K, RB, SB, CU;
  uint64_t pol;
};

// Stages one item into its ring buffer: router rows (the last may be the
// shared-gate row), or `rows` rows of gate and of up of one expert with their
// scales and biases.
__device__ __noinline__ void issue_item_dev(const Item it, uint8_t* buf, uint32_t bar, const FusedLayer* ly,
                                            const int* idx, const long long* off, const CopyShape cs) {
  const uint32_t dst = smem_addr(buf);
  if (it.kind == 0) {
    const int nr = max(0, min(it.rows, cs.E - it.row0));  // rows of w_router; the rest is the shared-gate row
    mbar_expect_tx(bar, (uint32_t)it.rows * cs.H * 2);
    if (nr > 0) bulk_g2s(dst, ly->w_router + (size_t)it.row0 * cs.H, (uint32_t)nr * cs.H * 2, bar, cs.pol);
    if (nr < it.rows) bulk_g2s(dst + (uint32_t)nr * cs.H * 2, ly->w_sgate, (uint32_t)cs.H * 2, bar, cs.pol);
    return;
  }
  const uint8_t* rec = it.slot < cs.K ? ly->routed + (long long)idx[it.slot] * ly->stride : ly->shared;
  const int RB = cs.RB, SB = cs.SB, CU = cs.CU;
  const uint32_t cb = (uint32_t)it.rows * RB, sbb = (uint32_t)it.rows * SB;
  mbar_expect_tx(bar, 2 * cb + 4 * sbb);
  bulk_g2s(dst, rec + off[0] + (long long)it.row0 * RB, cb, bar, cs.pol);
  bulk_g2s(dst + CU * RB, rec + off[3] + (long long)it.row0 * RB, cb, bar, cs.pol);
  bulk_g2s(dst + 2 * CU * RB, rec + off[1] + (long long)it.row0 * SB, sbb, bar, cs.pol);
  bulk_g2s(dst + 2 * CU * RB + CU * SB, rec + off[2] + (long long)it.row0 * SB, sbb, bar, cs.pol);
  bulk_g2s(dst + 2 * CU * RB + 2 * CU * SB, rec + off[4] + (long long)it.row0 * SB, sbb, bar, cs.pol);
  bulk_g2s(dst + 2 * CU * RB + 3 * CU * SB, rec + off[5] + (long long)it.row0 * SB, sbb, bar, cs.pol);
}

// Stages down rows [d0, d0 + nd) of one expert record (codes, scales, biases)
// into its slot region of DN, which holds `dmax` rows.
__device__ __noinline__ void issue_down_dev(uint8_t* base, uint32_t bar, const uint8_t* rec, const long long* off,
                                            int d0, int nd, int dmax, int RBd, int SBd, uint64_t pol) {
  bulk_g2s(smem_addr(base), rec + off[6] + (long long)d0 * RBd, (uint32_t)nd * RBd, bar, pol);
  bulk_g2s(smem_addr(base + (size_t)dmax * RBd), rec + off[7] + (long long)d0 * SBd, (uint32_t)nd * SBd, bar, pol);
  bulk_g2s(smem_addr(base + (size_t)dmax * (RBd + SBd)), rec + off[8] + (long long)d0 * SBd, (uint32_t)nd * SBd, bar,
           pol);
}

// Routing of one token from its tagged logits [E] (+ the shared-gate logit at
// E), E <= 8 * 64: stage 1, every warp w takes the K largest keys of its slice
// of ceil(E/8) logits (two per lane) into cand[w*K + k]; stage 2 (after a block
// barrier), warp 0 takes the K largest of the 8K candidates.  Keys order by
// value, then by lower index (topk_key), so the result is that of one sort of
// all E.  Returns false if the logits did not arrive in time.
__device__ __forceinline__ bool topk_stage1(const unsigned long long* logits, unsigned ep, int E, int K,
                                            unsigned long long* cand, int* err) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int ES = (E + kFW - 1) / kFW;
  const int e0 = warp * ES + lane, e1 = e0 + 32;
  const bool h0 = lane < ES && e0 < E, h1 = lane + 32 < ES && e1 < E;
  unsigned long long w0 = 0, w1 = 0, t0 = 0;
  bool ok = true;
  for (;;) {
    if (h0) w0 = ld_tagged(logits + e0);
    if (h1) w1 = ld_tagged(logits + e1);
    if ((!h0 || tag_of(w0) == ep) && (!h1 || tag_of(w1) == ep)) break;
    if (t0 == 0) t0 = global_ns();
    else if (global_ns() - t0 > kWaitNs) {
      atomicExch(err, kDevTimeout);
      ok = false;
      break;
    }
    __nanosleep(64);
  }
  unsigned long long k0 = h0 ? topk_key(val_of(w0), e0) : 0ull;
  unsigned long long k1 = h1 ? topk_key(val_of(w1), e1) : 0ull;
#pragma unroll 1
  for (int k = 0; k < K; ++k) {
    const unsigned long long m = warp_max_key(k0 > k1 ? k0 : k1);
    if (lane == 0) cand[warp * K + k] = m;
    k0 = k0 == m ? 0ull : k0;
    k1 = k1 == m ? 0ull : k1;
  }
  return __all_sync(0xffffffffu, ok);
}

// Stage 2, warp 0: picks, renormalised weights w_k = exp(l_k - l_0) / sum_j exp(l_j - l_0)
// and sigma = sigmoid(l_E) into idx[0..K), w[0..K], w[K] = sigma.
__device__ __noinline__ bool topk_stage2(const unsigned long long* logits, unsigned ep, int E, int K,
                                         const unsigned long long* cand, int* idx, float* w, int* err) {
  const int lane = threadIdx.x & 31;
  unsigned long long key[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) key[i] = lane + 32 * i < kFW * K ? cand[lane + 32 * i] : 0ull;
  float top = 0.0f, mine = 0.0f;
  int mi = 0;
#pragma unroll 1
  for (int k = 0; k < K; ++k) {
    unsigned long long best = 0ull;
#pragma unroll
    for (int i = 0; i < 8; ++i) best = key[i] > best ? key[i] : best;
    const unsigned long long m = warp_max_key(best);
#pragma unroll
    for (int i = 0; i < 8; ++i) key[i] = key[i] == m ? 0ull : key[i];
    int e = m ? topk_key_index(m) : 0;
    const float v = topk_key_value(m);
    if (e < 0 || e >= E) e = 0;  // only with non-finite logits
    if (k == 0) top = v;
    if (lane == k) {
      mi = e;
      mine = v;
    }
  }
  const float ek = lane < K ? expf(mine - top) : 0.0f;
  const float wk = ek / warp_sum(ek);
  if (lane < K) {
    idx[lane] = mi;
    w[lane] = wk;
  }
  bool ok = true;
  if (lane == 0) {  // the shared-gate logit
    unsigned long long g = 0, t0 = 0;
    for (;;) {
      g = ld_tagged(logits + E);
      if (tag_of(g) == ep) break;
      if (t0 == 0) t0 = global_ns();
      else if (global_ns() - t0 > kWaitNs) {
        atomicExch(err, kDevTimeout);
        ok = false;
        break;
      }
    }
    w[K] = 1.0f / (1.0f + expf(-val_of(g)));
  }
  return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

template <int BITS>
__global__ void __launch_bounds__(kFT, 1) fused_kernel(const __grid_constant__ FusedParams p) {
  extern __shared__ __align__(128) uint8_t sm[];
  __shared__ __align__(8) uint64_t s_full[kFusedMaxRing];
  __shared__ __align__(8) uint64_t s_dnbar;
  __shared__ Item s_item[kFusedMaxItems];
  __shared__ int s_pend[kFusedMaxRing];
  __shared__ int s_idx[32];
  __shared__ unsigned long long s_cand[kFW * 32];  // top-K candidates, K per warp
  __shared__ float s_w[33];
  __shared__ float s_red[kFW];
  __shared__ float s_rpart[2][kFusedMaxRtRows * 8];
  __shared__ float s_gacc[kFusedMaxGuRows * 4 * 2];  // gate/up partial sums [row][k-part][gate, up]
  __shared__ int s_cnt[kFusedMaxRing];                // warps done with a buffer
  __shared__ float s_dpart[kFusedMaxKS * kFusedMaxDnRows];
  __shared__ int s_abort;
  __shared__ int s_nconst, s_nitems;
  __shared__ int s_dnstate;  // down rows of the current step: 0 none in flight, 1 shared issued, 2 all issued

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int P = gridDim.x, b = blockIdx.x;
  const int H = p.H, I = p.I, K = p.K, E = p.E, NE = K + 1;
  const int NGH = H / kGroup, NGI = I / kGroup;
  const int RB = H * BITS / 8, SB = NGH * 2;        // gate/up row: code bytes, scale bytes
  const int RBd = I * BITS / 8, SBd = NGI * 2;      // down row
  const int ncd = I * BITS / 128;                   // chunk scalars of one activation vector
  const int nbuf = p.nbuf, chb = p.chb, CU = p.cu;
  uint8_t* xd = sm;
  uint8_t* dn = sm + p.dn_off;
  uint8_t* ring = sm + p.ring_off;
  float* s_x = reinterpret_cast<float*>(xd);
  uint8_t* s_xl = xd + (size_t)H * 4;
  float2* s_xcs = reinterpret_cast<float2*>(xd + (size_t)H * 4 + (size_t)NGH * kGroupWords * 4);
  uint8_t* s_al = xd;  // down phase: activation digits of every slot, then their chunk scalars
  float2* s_acs = reinterpret_cast<float2*>(xd + (size_t)NE * NGI * kGroupWords * 4);
  const uint64_t pol = l2_policy_evict_first();

  // ---- this CTA's share of every phase (the same for every step)
  const int R = E + 1;  // router rows + the shared-gate row
  const int rr0 = (int)((long long)b * R / P), rr1 = (int)((long long)(b + 1) * R / P);
  const int US = I / p.ru, UR = K * I / p.ru, UD = H / p.rd;
  const int sh0 = (int)((long long)b * US / P) * p.ru, sh1 = (int)((long long)(b + 1) * US / P) * p.ru;
  const int rf0 = (int)((long long)b * UR / P) * p.ru, rf1 = (int)((long long)(b + 1) * UR / P) * p.ru;
  const int d0 = (int)((long long)b * UD / P) * p.rd, d1 = (int)((long long)(b + 1) * UD / P) * p.rd;
  const int nd = d1 - d0;
  const int dn_slot = p.dn_slot_bytes, dmax = p.dn_rows_max;

  if (tid == 0) {
    int n = 0;
    int rb = 0;
    for (int r = rr0; r < rr1; r += p.rt_rows) s_item[n++] = Item{0, 0, r, min(p.rt_rows, rr1 - r), 0};
    for (int r = sh0; r < sh1; r += CU) {
      s_item[n++] = Item{1, K, r, min(CU, sh1 - r), rb};
      rb += min(CU, sh1 - r);
    }
    s_nconst = n;
    for (int f = rf0; f < rf1;) {
      const int slot = f / I, r = f % I;
      const int rows = min(min(CU, rf1 - f), I - r);
      s_item[n++] = Item{1, slot, r, rows, rb};
      rb += rows;
      f += rows;
    }
    s_nitems = n;
    for (int i = 0; i < nbuf; ++i) {
      mbar_init(smem_addr(&s_full[i]), 1);
      s_pend[i] = 0;
      s_cnt[i] = 0;
    }
    mbar_init(smem_addr(&s_dnbar), 2);
    mbar_fence_init();
    s_abort = 0;
    s_dnstate = 0;
  }
  __syncthreads();
  const int n_const = s_nconst, n_items = s_nitems;
  const int n_rt = (rr1 - rr0 + p.rt_rows - 1) / p.rt_rows;

  // ---- copies (one thread per call)
  const CopyShape cshape{E, H, K, RB, SB, CU, pol};
  auto issue_item = [&](int j, const FusedLayer& ly) {
    const int bi = j % nbuf;
    s_pend[bi] = 1;
    issue_item_dev(s_item[j], ring + (size_t)bi * chb, smem_addr(&s_full[bi]), &ly, s_idx, p.off, cshape);
  };
  auto issue_down = [&](int slot, const uint8_t* rec) {
    issue_down_dev(dn + (size_t)slot * dn_slot, smem_addr(&s_dnbar), rec, p.off, d0, nd, dmax, RBd, SBd, pol);
  };
  auto issue_shared_down = [&](const FusedLayer& ly) {
    if (nd == 0) return;
    s_dnstate = 1;
    mbar_expect_tx(smem_addr(&s_dnbar), (uint32_t)nd * (RBd + 2 * SBd));
    issue_down(K, ly.shared);
  };

  // ---- lane geometry
  // gate/up: KS warps share a row (each lane one group of 64 columns), or RPP rows share a warp
  const int KS = NGH >= 32 ? NGH / 32 : 1;
  const int LPR = NGH >= 32 ? 32 : NGH, RPP = 32 / LPR;
  const int gsub = lane / LPR, gl = lane % LPR;
  const int kap = warp % KS;
  const int xg = NGH >= 32 ? kap * 32 + lane : gl;  // this lane's group of x
  // down: (slot, group) pairs, one per lane
  const int NP = NE * NGI;
  int np2 = 1;
  while (np2 < NP) np2 <<= 1;
  const int LPRd = np2 < 32 ? np2 : 32, RPPd = 32 / LPRd, KSd = np2 > 32 ? np2 / 32 : 1;
  const int dsub = lane / LPRd, dl = lane % LPRd, kapd = warp % KSd;
  const int q = kapd * 32 + dl;
  const bool qon = q < NP;
  const int qslot = qon ? q / NGI : 0, qg = qon ? q % NGI : 0;

  uint32_t ph = 0;  // per ring buffer: parity of its next fill
  bool ok = true;

  // After a failed wait: let every copy in flight into this CTA's shared memory
  // land (bounded), then leave.  `sp` is the step's parity.
  auto abort_all = [&](int sp) {
    __syncthreads();
    if (tid == 0) {
      for (int i = 0; i < nbuf; ++i)
        if (s_pend[i]) mbar_wait_bounded(smem_addr(&s_full[i]), (ph >> i) & 1u, p.err);
      if (s_dnstate == 1) mbar_arrive(smem_addr(&s_dnbar));  // the routed half never came
      if (s_dnstate > 0) mbar_wait_bounded(smem_addr(&s_dnbar), (uint32_t)(sp & 1), p.err);
    }
  };

  const int S = p.T * p.L;

  // Step 0's routing-independent rows, before waiting on the previous kernel.
  if (tid == 0) {
    const FusedLayer& ly0 = p.layers[0];
    for (int j = 0; j < n_const && j < nbuf; ++j) issue_item(j, ly0);
    issue_shared_down(ly0);
  }
  pdl_wait();
  pdl_trigger();  // the next kernel's CTAs start only once every CTA of this grid is running
  // Epochs of this launch: base + s + 1 for step s.  Every CTA reads the base
  // here; CTA 0 advances it on exit, after every CTA has consumed its data.
  const unsigned ep_base = *reinterpret_cast<volatile const unsigned*>(p.epoch);

  int s = 0;
  for (; s < S; ++s) {
    const int t = s / p.L, l = s % p.L;
    const FusedLayer& ly = p.layers[l];
    const unsigned ep = ep_base + (unsigned)s + 1u;
    const int par = s & 1;
    const float* hin = (l == 0 ? p.h : p.out) + (size_t)t * H;
    float* hout = p.out + (size_t)t * H;
    unsigned long long* xlog = p.xlog + (size_t)par * (E + 1);
    unsigned long long* xact = p.xact + (size_t)par * NE * I;

    if (s > 0 && tid == 0) issue_shared_down(ly);
    __syncwarp();  // a single lane issuing copies keeps its warp-mates waiting, not spinning beside it

    // ---- x = RMSNorm(h) (two passes: sum of squares, then apply) and its digits,
    // the whole vector in every CTA.  Pass 1 stages h in s_x: the user's input
    // for the first layer, the previous step's tagged output inside a stack.
    float ss = 0.0f;
    if (l == 0) {
#pragma unroll 4
      for (int i = tid * 4; i < H; i += kFT * 4) {
        const float4 v = __ldcg(reinterpret_cast<const float4*>(hin + i));
        *reinterpret_cast<float4*>(s_x + i) = v;
        ss = fmaf(v.x, v.x, fmaf(v.y, v.y, fmaf(v.z, v.z, fmaf(v.w, v.w, ss))));
      }
    } else {
      const unsigned long long* xh = p.xh + (size_t)(par ^ 1) * H;
#pragma unroll 1
      for (int i = tid * 4; i < H; i += kFT * 4) {
        float v[4];
        if (!poll_tagged<4>(xh + i, ep - 1u, v, p.err)) ok = false;
        *reinterpret_cast<float4*>(s_x + i) = make_float4(v[0], v[1], v[2], v[3]);
        ss = fmaf(v[0], v[0], fmaf(v[1], v[1], fmaf(v[2], v[2], fmaf(v[3], v[3], ss))));
      }
    }
    float rstd = 1.0f;
    if (ly.gamma) {
      ss = warp_sum(ss);
      if (lane == 0) s_red[warp] = ss;
    }
    if (!ok) s_abort = 1;
    __syncthreads();
    if (s_abort) break;
    if (ly.gamma) {
      float tot = 0.0f;
#pragma unroll
      for (int w = 0; w < kFW; ++w) tot += s_red[w];
      rstd = 1.0f / sqrtf(tot / (float)H + ly.eps);
    }
    // Pass 2: lane l of a warp owns block (base + l) of 16 elements; the four
    // blocks of a group of 64 sit on four neighbouring lanes.
    const int NB = H / 16;
#pragma unroll 1
    for (int base = warp * 32; base < NB; base += kFT) {
      const int blk = base + lane;
      const bool act = blk < NB;
      float xv[16];
      if (act) {
        const float4* xs4 = reinterpret_cast<const float4*>(s_x + blk * 16);
        float4 v[4] = {xs4[0], xs4[1], xs4[2], xs4[3]};
        if (ly.gamma) {
          const float4* gp = reinterpret_cast<const float4*>(ly.gamma + blk * 16);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float4 g = __ldg(gp + k);
            v[k] = make_float4(v[k].x * rstd * g.x, v[k].y * rstd * g.y, v[k].z * rstd * g.z, v[k].w * rstd * g.w);
          }
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          xv[4 * k] = v[k].x;
          xv[4 * k + 1] = v[k].y;
          xv[4 * k + 2] = v[k].z;
          xv[4 * k + 3] = v[k].w;
        }
        float4* xo = reinterpret_cast<float4*>(s_x + blk * 16);
#pragma unroll
        for (int k = 0; k < 4; ++k) xo[k] = v[k];
      } else {
#pragma unroll
        for (int k = 0; k < 16; ++k) xv[k] = 0.0f;
      }
      xq_quantize_block16<BITS>(xv, blk >> 2, blk & 3, NGH, s_xl, s_xcs, act);
    }
    __syncthreads();

    // ---- router rows: logits of this CTA's rows, published as tagged words.
    // Warp w sums segment w (H/8 columns) of every row of a staged item; the 8
    // segments add in fixed order.
    int j = 0;
    for (; j < n_rt; ++j) {
      const int bi = j % nbuf;
      if (!mbar_wait_bounded(smem_addr(&s_full[bi]), (ph >> bi) & 1u, p.err)) ok = false;
      ph ^= 1u << bi;
      const Item it = s_item[j];
      const uint16_t* wr = reinterpret_cast<const uint16_t*>(ring + (size_t)bi * chb) + warp * (H / 8);
      const float* xs = s_x + warp * (H / 8);
      float* part = s_rpart[j & 1];
      float acc[kFusedMaxRtRows];
#pragma unroll
      for (int r = 0; r < kFusedMaxRtRows; ++r) acc[r] = 0.0f;
#pragma unroll 1
      for (int k = lane; ok && k < H / 64; k += 32) {  // 8 columns per step
        const float4 xa = *reinterpret_cast<const float4*>(xs + 8 * k);
        const float4 xb = *reinterpret_cast<const float4*>(xs + 8 * k + 4);
#pragma unroll
        for (int r = 0; r < kFusedMaxRtRows; ++r) {
          if (r < it.rows) {
            const uint4 w = *reinterpret_cast<const uint4*>(wr + (size_t)r * H + 8 * k);
            float a = acc[r];
            a = fmaf(__uint_as_float(w.x << 16), xa.x, a);
            a = fmaf(__uint_as_float(w.x & 0xFFFF0000u), xa.y, a);
            a = fmaf(__uint_as_float(w.y << 16), xa.z, a);
            a = fmaf(__uint_as_float(w.y & 0xFFFF0000u), xa.w, a);
            a = fmaf(__uint_as_float(w.z << 16), xb.x, a);
            a = fmaf(__uint_as_float(w.z & 0xFFFF0000u), xb.y, a);
            a = fmaf(__uint_as_float(w.w << 16), xb.z, a);
            a = fmaf(__uint_as_float(w.w & 0xFFFF0000u), xb.w, a);
            acc[r] = a;
          }
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int r = 0; r < kFusedMaxRtRows; ++r) acc[r] += __shfl_xor_sync(0xffffffffu, acc[r], o);
      if (lane == 0)
#pragma unroll
        for (int r = 0; r < kFusedMaxRtRows; ++r)
          if (r < it.rows) part[r * 8 + warp] = acc[r];
      __syncthreads();
      if (tid < it.rows) {
        float lg = 0.0f;
#pragma unroll
        for (int sg = 0; sg < 8; ++sg) lg += part[tid * 8 + sg];
        const int row = it.row0 + tid;
        if (row < E && ly.bias) lg += ly.bias[row];
        st_tagged(xlog + row, lg, ep);
      }
      if (tid == 0) {
        s_pend[bi] = 0;
        if (ok && j + nbuf < n_const) {  // more routing-independent rows than buffers
          fence_proxy_async();
          issue_item(j + nbuf, ly);
        }
      }
      __syncwarp();
    }

    // ---- this lane's digits of x, for every gate/up row of the step
    uint32_t L[48];
    load_group_limbs(reinterpret_cast<const uint32_t*>(s_xl), xg, NGH, L);
    float2 csx;
    if (BITS == 4) {
      const float2 a = s_xcs[2 * xg], c = s_xcs[2 * xg + 1];
      csx = make_float2(a.x, a.y + c.y);
    } else {
      csx = s_xcs[xg];
    }

    // ---- gate/up of every staged item of the step: the shared expert's first
    // (while the other CTAs finish their logits), then, once every logit is
    // in and the routing is known, the routed experts'.  Warp-level tasks
    // (k-part, row pass) leave partial sums in s_gacc; warps move on
    // independently, and the last warp done with a buffer refills it.
    bool stop = false;
    for (;; ++j) {
      if (j == n_const) {
        // ---- the routing: every CTA selects the experts itself from the tagged logits
        if (!topk_stage1(xlog, ep, E, K, s_cand, p.err)) ok = false;
        if (!ok) s_abort = 1;
        __syncthreads();
        if (s_abort) {
          stop = true;
          break;
        }
        if (warp == 0 && !topk_stage2(xlog, ep, E, K, s_cand, s_idx, s_w, p.err)) s_abort = 1;
        __syncthreads();
        if (s_abort) {
          stop = true;
          break;
        }
        // routed gate/up rows into every buffer (all consumed by now): item i by
        // lane 0 of warp 1 + i % 7, so the copies go out from several warps at once
        if (lane == 0 && warp > 0) {
          fence_proxy_async();
          for (int jj = n_const + warp - 1; jj < n_items && jj < n_const + nbuf; jj += kFW - 1) issue_item(jj, ly);
        }
        __syncwarp();
        if (warp == 0) {
          if (b == 0 && lane < K && p.idx_out) p.idx_out[(size_t)t * K + lane] = s_idx[lane];
          if (b == 0 && lane < K && p.w_out) p.w_out[(size_t)t * K + lane] = s_w[lane];
          // routed down rows: one slot per lane of warp 0
          if (nd > 0 && lane < K) {
            if (lane == 0) {
              s_dnstate = 2;
              mbar_expect_tx(smem_addr(&s_dnbar), (uint32_t)K * nd * (RBd + 2 * SBd));
            }
            __syncwarp(0xffffffffu >> (32 - K));
            issue_down(lane, ly.routed + (long long)s_idx[lane] * ly.stride);
          }
          __syncwarp();
        }
      }
      if (j >= n_items) break;
      const int limit = j < n_const ? n_const : n_items;
      const int bi = j % nbuf;
      if (!mbar_wait_bounded(smem_addr(&s_full[bi]), (ph >> bi) & 1u, p.err)) ok = false;
      ph ^= 1u << bi;
      const Item it = s_item[j];
      const uint8_t* buf = ring + (size_t)bi * chb;
      const int ntask = (it.rows + RPP - 1) / RPP * KS;
#pragma unroll 1
      for (int task = warp; ok && task < ntask; task += kFW) {
        const int r = (task / KS) * RPP + gsub;
        float ag = 0.0f, au = 0.0f;
        if (r < it.rows) {
          const uint8_t* gr = buf + (size_t)r * RB + xg * (kGroup * BITS / 8);
          const uint8_t* ur = gr + (size_t)CU * RB;
          const uint4 q0 = *reinterpret_cast<const uint4*>(gr);
          const uint4 q1 = BITS == 4 ? *reinterpret_cast<const uint4*>(gr + 16) : q0;
          const uint4 v0 = *reinterpret_cast<const uint4*>(ur);
          const uint4 v1 = BITS == 4 ? *reinterpret_cast<const uint4*>(ur + 16) : v0;
          const uint16_t* sc = reinterpret_cast<const uint16_t*>(buf + 2 * (size_t)CU * RB + (size_t)r * SB);
          const int cs2 = CU * SB / 2;
          const float gs = bf16_to_f32(sc[xg]), gb = bf16_to_f32(sc[cs2 + xg]);
          const float us = bf16_to_f32(sc[2 * cs2 + xg]), ub = bf16_to_f32(sc[3 * cs2 + xg]);
          const float Sg = group_dot<BITS>(q0, q1, L);
          const float Su = group_dot<BITS>(v0, v1, L);
          ag = fmaf(gs, csx.x * Sg, gb * csx.y);
          au = fmaf(us, csx.x * Su, ub * csx.y);
        }
        for (int o = LPR / 2; o > 0; o >>= 1) {
          ag += __shfl_xor_sync(0xffffffffu, ag, o);
          au += __shfl_xor_sync(0xffffffffu, au, o);
        }
        if (gl == 0 && r < it.rows) {
          s_gacc[((it.rbase + r) * 4 + kap) * 2] = ag;
          s_gacc[((it.rbase + r) * 4 + kap) * 2 + 1] = au;
        }
      }
      __syncwarp();
      if (lane == 0) {
        __threadfence_block();
        if (atomicAdd(&s_cnt[bi], 1) == kFW - 1) {
          s_cnt[bi] = 0;
          __threadfence_block();
          s_pend[bi] = 0;
          if (ok && j + nbuf < limit) {
            fence_proxy_async();
            issue_item(j + nbuf, ly);
          }
        }
      }
      __syncwarp();
    }
    if (stop) break;
    if (!ok) s_abort = 1;
    __syncthreads();  // every partial sum of the step is in s_gacc
    if (s_abort) break;
    // SwiGLU of every gate/up row of this CTA, silu(g) * u with silu(z) = z / (1 + exp(-z)),
    // published as tagged words
    for (int jj = n_rt + warp; jj < n_items; jj += kFW) {
      const Item it = s_item[jj];
      if (lane < it.rows) {
        float g = 0.0f, u = 0.0f;
        for (int k = 0; k < KS; ++k) {
          g += s_gacc[((it.rbase + lane) * 4 + k) * 2];
          u += s_gacc[((it.rbase + lane) * 4 + k) * 2 + 1];
        }
        st_tagged(xact + (size_t)it.slot * I + it.row0 + lane, g / (1.0f + expf(-g)) * u, ep);
      }
    }

    // ---- the next step's routing-independent rows, into the drained ring
    if (tid == 0 && s + 1 < S) {
      fence_proxy_async();
      const FusedLayer& ln = p.layers[(s + 1) % p.L];
      for (int jj = 0; jj < n_const && jj < nbuf; ++jj) issue_item(jj, ln);
    }
    __syncwarp();

    // ---- every CTA's activations: poll the tagged words of all K+1 slots and
    // quantise them here (lane per block of 16, four lanes per group of 64)
    const int nblk = NE * I / 16, bps = I / 16;
#pragma unroll 1
    for (int base = warp * 32; base < nblk; base += kFT) {
      const int blk = base + lane;
      const bool act = blk < nblk;
      float av[16];
      if (act) {
        if (!poll_tagged<16>(xact + (size_t)blk * 16, ep, av, p.err)) ok = false;
      } else {
#pragma unroll
        for (int k = 0; k < 16; ++k) av[k] = 0.0f;
      }
      const int slot = act ? blk / bps : 0, bb = act ? blk % bps : 0;
      xq_quantize_block16<BITS>(av, bb >> 2, bb & 3, NGI, s_al + (size_t)slot * NGI * kGroupWords * 4,
                                s_acs + (size_t)slot * ncd, act);
    }
    if (nd > 0 && !mbar_wait_bounded(smem_addr(&s_dnbar), (uint32_t)(s & 1), p.err)) ok = false;
    if (!ok) s_abort = 1;
    __syncthreads();
    if (s_abort) break;
    if (tid == 0) s_dnstate = 0;

    // ---- down + combine from shared memory: lane q owns one (slot, group) pair,
    // four output rows per pass, then one interleaved reduction
    {
      uint32_t A[48];
      load_group_limbs(reinterpret_cast<const uint32_t*>(s_al + (size_t)qslot * NGI * kGroupWords * 4), qg, NGI, A);
      const float2* acs = s_acs + qslot * ncd;
      float2 csa;
      if (BITS == 4) {
        const float2 a = acs[2 * qg], c = acs[2 * qg + 1];
        csa = make_float2(a.x, a.y + c.y);
      } else {
        csa = acs[qg];
      }
      const float wq = qon ? s_w[qslot] : 0.0f;
      const uint8_t* sb = dn + (size_t)qslot * dn_slot;
      const uint16_t* scl = reinterpret_cast<const uint16_t*>(sb + (size_t)dmax * RBd);
      const uint16_t* bsl = reinterpret_cast<const uint16_t*>(sb + (size_t)dmax * (RBd + SBd));
#pragma unroll 1
      for (int pass = warp / KSd; pass * 4 * RPPd < nd; pass += kFW / KSd) {
        float acc[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int r = (pass * 4 + u) * RPPd + dsub;
          acc[u] = 0.0f;
          if (qon && r < nd) {
            const uint8_t* cr = sb + (size_t)r * RBd + qg * (kGroup * BITS / 8);
            const uint4 q0 = *reinterpret_cast<const uint4*>(cr);
            const uint4 q1 = BITS == 4 ? *reinterpret_cast<const uint4*>(cr + 16) : q0;
            const float sc = bf16_to_f32(scl[(size_t)r * NGI + qg]);
            const float bi = bf16_to_f32(bsl[(size_t)r * NGI + qg]);
            const float Sd = group_dot<BITS>(q0, q1, A);
            acc[u] = wq * fmaf(sc, csa.x * Sd, bi * csa.y);
          }
        }
        for (int o = LPRd / 2; o > 0; o >>= 1)
#pragma unroll
          for (int u = 0; u < 4; ++u) acc[u] += __shfl_xor_sync(0xffffffffu, acc[u], o);
        if (dl == 0)
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int r = (pass * 4 + u) * RPPd + dsub;
            if (r < nd) s_dpart[kapd * kFusedMaxDnRows + r] = acc[u];
          }
      }
    }
    __syncthreads();
    // out = h + sum_k w_k y_k + sigma y_shared; inside a stack also the next layer's tagged input
    const bool feed = s + 1 < S && (s + 1) % p.L != 0;
    unsigned long long* xh = p.xh + (size_t)par * H;
    for (int r = tid; r < nd; r += kFT) {
      float y = 0.0f;
      for (int k = 0; k < KSd; ++k) y += s_dpart[k * kFusedMaxDnRows + r];
      const float o = __ldcg(hin + d0 + r) + y;
      hout[d0 + r] = o;
      if (feed) st_tagged(xh + d0 + r, o, ep);
    }
    __syncthreads();  // shared memory of this step (XD, DN) is free
    if (tid == 0) fence_proxy_async();
  }
  if (s < S) abort_all(s);
  if (b == 0 && tid == 0) *reinterpret_cast<volatile unsigned*>(p.epoch) = ep_base + (unsigned)S;
}

}  // namespace

FusedPlan plan_fused(int bits, int H, int I, int E, int K) {
  FusedPlan pl{};
  pl.ok = false;
  if (bits != 2 && bits != 4) return pl;  // this path has no 8-bit form
  if (H % kGroup || I % kGroup || K < 1 || K > 32 || E < K || E > kFW * 64) return pl;
  const int NGH = H / kGroup, NGI = I / kGroup, NE = K + 1;
  if (NGH > 128 || NGI > 128) return pl;
  const int RB = H * bits / 8, SB = NGH * 2, RBd = I * bits / 8, SBd = NGI * 2;
  const int sms = num_sms();
  int P = ((NE * I) + 31) / 32;
  P = P < 2 ? 2 : P;
  P = P > sms ? sms : P;
  pl.P = P;
  pl.ru = SB >= 16 ? 1 : 16 / SB;
  pl.rd = SBd >= 16 ? 1 : 16 / SBd;
  // down pairs per row: one per lane across at most 8 warps
  int np2 = 1;
  while (np2 < NE * NGI) np2 <<= 1;
  if (np2 > 32 * kFusedMaxKS) return pl;
  const int UD = H / pl.rd;
  pl.dn_rows_max = (UD + P - 1) / P * pl.rd;
  if (pl.dn_rows_max > kFusedMaxDnRows) return pl;
  pl.dn_slot_bytes = (pl.dn_rows_max * (RBd + 2 * SBd) + 127) / 128 * 128;
  const size_t xd1 = (size_t)H * 4 + (size_t)NGH * kGroupWords * 4 + (size_t)(H * bits / 128) * 8;
  const size_t xd2 = (size_t)NE * NGI * kGroupWords * 4 + (size_t)NE * (I * bits / 128) * 8;
  const size_t xd = ((xd1 > xd2 ? xd1 : xd2) + 127) / 128 * 128;
  pl.dn_off = (int)xd;
  pl.ring_off = (int)(xd + (size_t)NE * pl.dn_slot_bytes);
  // gate/up chunks of about 18 KiB, a whole number of row units, at most kFusedMaxChunkRows rows
  const int pair = 2 * (RB + 2 * SB);
  int cu = 18432 / pair;
  cu = cu < 1 ? 1 : cu;
  cu = cu > kFusedMaxChunkRows ? kFusedMaxChunkRows : cu;
  cu = cu / pl.ru * pl.ru;
  if (cu < pl.ru) return pl;
  pl.cu = cu;
  pl.chb = ((cu * pair) + 127) / 128 * 128;
  if (pl.chb < H * 2) pl.chb = (H * 2 + 127) / 128 * 128;  // at least one router row per buffer
  int rt = pl.chb / (H * 2);
  pl.rt_rows = rt > kFusedMaxRtRows ? kFusedMaxRtRows : rt;
  const long long budget = kFusedSmemBudget - pl.ring_off;
  if (budget < 2LL * pl.chb) return pl;
  int nbuf = (int)(budget / pl.chb);
  pl.nbuf = nbuf > kFusedMaxRing ? kFusedMaxRing : nbuf;
  pl.smem = (size_t)pl.ring_off + (size_t)pl.nbuf * pl.chb;
  // items per CTA must fit the item table
  const int R = E + 1;
  const int rt_items = ((R + P - 1) / P + pl.rt_rows - 1) / pl.rt_rows;
  const int sh_items = ((I / pl.ru + P - 1) / P * pl.ru + cu - 1) / cu;
  const int rf_items = ((K * I / pl.ru + P - 1) / P * pl.ru + cu - 1) / cu + 2;
  if (rt_items + sh_items + rf_items > kFusedMaxItems) return pl;
  // activation groups counted per CTA must fit s_gdone
  const int gcount = ((I / pl.ru + P - 1) / P * pl.ru) / kGroup + 2 + ((K * I / pl.ru + P - 1) / P * pl.ru) / kGroup + 2;
  if (gcount > 64) return pl;
  const int gu_rows = (I / pl.ru + P - 1) / P * pl.ru + (K * I / pl.ru + P - 1) / P * pl.ru;
  if (gu_rows > kFusedMaxGuRows || (NGH >= 32 && NGH / 32 > 4)) return pl;
  pl.ok = true;
  return pl;
}

cudaError_t launch_fused(const FusedParams& p, const FusedPlan& pl, int bits, bool pdl, cudaStream_t s) {
  void (*k)(const FusedParams) = bits == 4 ? fused_kernel<4> : fused_kernel<2>;
  cudaError_t e = set_smem((const void*)k, pl.smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(k, dim3(pl.P), dim3(kFT), pl.smem, s, pdl, p);
}

}  // namespace fmoe
