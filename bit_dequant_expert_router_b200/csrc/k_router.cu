// k_router.cu -- RMSNorm, activation digits, the router GEMV and the standalone top-K.
//
// RMSNorm follows "What is Flash-MoE" (a2a-mcp.org), section 3: two passes,
// sum of squares then apply.  Routing follows the "Flash-MoE" wiki summary
// (jeongsk), per-layer pipeline: routing projection, then softmax and top-K.
// The pages run the selection on the CPU; here it stays on the GPU: in the
// MoE block the router kernel writes the logits and every CTA of the expert
// kernels selects the experts from them itself (block_topk), so neither a host
// round trip nor a grid-wide handshake sits between the router and the experts.
// The standalone router_topk entry point uses topk_kernel.
#include "fmoe_internal.h"

namespace fmoe {
namespace {

constexpr int kRouterThreads = 256;
constexpr int kRouterMaxRows = 8;  // router rows per CTA

// Block-wide sum of one value per thread (256 threads), same order every call.
__device__ __forceinline__ float block_sum_256(float v, float* s_red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = warp_sum(v);
  if (lane == 0) s_red[warp] = v;
  __syncthreads();
  float r = 0.0f;
#pragma unroll
  for (int w = 0; w < kRouterThreads / 32; ++w) r += s_red[w];
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(256) rmsnorm_kernel(const float* __restrict__ h, const float* __restrict__ gamma,
                                                      float eps, int H, float* __restrict__ y) {
  __shared__ float s_red[8];
  const float* hr = h + (size_t)blockIdx.x * H;
  float* yr = y + (size_t)blockIdx.x * H;
  float ss = 0.0f;  // pass 1: sum of squares
  for (int i = threadIdx.x; i < H; i += blockDim.x) ss = fmaf(hr[i], hr[i], ss);
  ss = block_sum_256(ss, s_red);
  const float rstd = 1.0f / sqrtf(ss / (float)H + eps);
  for (int i = threadIdx.x; i < H; i += blockDim.x)  // pass 2: apply
    yr[i] = hr[i] * rstd * (gamma ? gamma[i] : 1.0f);
}

// Digits of x (fp32 [H]) for the expert kernels; one warp per group of 64.
template <int BITS>
__global__ void __launch_bounds__(256) xq_kernel(const float* __restrict__ x, int H, uint8_t* limbs, float2* cs) {
  const int g = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (g >= H / kGroup) return;  // warp-uniform
  const float2 v = reinterpret_cast<const float2*>(x + g * kGroup)[threadIdx.x & 31];
  xq_quantize_group<BITS>(v.x, v.y, g, H / kGroup, limbs, cs);
}

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// grid (NB, T).  Before waiting on the predecessor, each CTA bulk-copies its
// rows [b*rpc, b*rpc + rpc) of [Wr; wsg] into shared memory (weights only).
// Then x = RMSNorm(h_t) in shared memory, at most one group of the activation
// digits per warp spread over the grid, and its logits as 8 warp tasks (rows x
// segments).  When top_k > 0 the last CTA of the token (atomic ticket) selects
// the experts once for every later kernel.
template <int XQB>
__global__ void __launch_bounds__(kRouterThreads) router_kernel(const RouterParams p) {
  extern __shared__ __align__(128) uint8_t sm[];
  __shared__ float s_red[8];
  __shared__ float s_part[kRouterMaxRows * 8];
  __shared__ int s_last;
  __shared__ __align__(8) uint64_t s_bar;
  const int t = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int H = p.H, E = p.E;
  const int R = E + (p.w_sgate ? 1 : 0);
  const int rpc = p.rows_per_cta;
  const int r0 = blockIdx.x * rpc;
  const int nrows = min(rpc, R - r0);
  uint16_t* wrows = reinterpret_cast<uint16_t*>(sm);
  float* xs = reinterpret_cast<float*>(sm + (size_t)rpc * H * 2);
  const uint32_t bar = smem_addr(&s_bar);

  if (tid == 0) {
    mbar_init(bar, 1);
    mbar_fence_init();
    if (nrows > 0) {
      const int nr = min(nrows, E - r0 > 0 ? E - r0 : 0);  // routed rows in range
      const bool gate_row = p.w_sgate && r0 + nrows > E;
      mbar_expect_tx(bar, (uint32_t)nrows * H * 2);
      if (nr > 0) bulk_g2s(smem_addr(wrows), p.w_router + (size_t)r0 * H, (uint32_t)nr * H * 2, bar, l2_policy_evict_last());
      if (gate_row) bulk_g2s(smem_addr(wrows + (size_t)nr * H), p.w_sgate, (uint32_t)H * 2, bar, l2_policy_evict_last());
    }
  }
  // gamma is a weight: read it (this thread's float4s, H <= 8192) before the wait
  constexpr int kGv = 8192 / (kRouterThreads * 4);
  float4 gv[kGv];
#pragma unroll
  for (int j = 0; j < kGv; ++j) {
    const int i = (tid + j * kRouterThreads) * 4;
    gv[j] = (p.norm && p.gamma && i < H) ? __ldg(reinterpret_cast<const float4*>(p.gamma + i))
                                         : make_float4(1.0f, 1.0f, 1.0f, 1.0f);
  }
  // h may still be written by the kernel waited on below.  An L2 prefetch of it
  // cannot leave stale data behind (every global write lands in L2); when h was
  // written earlier it hides the DRAM latency of the first read after the wait.
  if (blockIdx.x == 0 && tid == 0) prefetch_l2(p.h + (size_t)t * H, (uint32_t)H * 4);
  pdl_wait();
  pdl_trigger();
  // every kernel of the previous token is complete: its routing flag is spent, and the
  // gate/up kernel's group counters are cleared (they return to zero by themselves unless
  // a bounded wait gave up part-way)
  if (p.route_ready && blockIdx.x == 0 && blockIdx.y == 0 && tid == 0) *p.route_ready = 0u;
  if (p.clear && blockIdx.x == 0 && blockIdx.y == 0)
    for (int i = tid; i < p.nclear; i += kRouterThreads) p.clear[i] = 0u;

  const float* h = p.h + (size_t)t * H;
  float ss = 0.0f;
#pragma unroll 4
  for (int i = tid * 4; i < H; i += kRouterThreads * 4) {
    const float4 v = *reinterpret_cast<const float4*>(h + i);
    *reinterpret_cast<float4*>(xs + i) = v;
    ss = fmaf(v.x, v.x, ss);
    ss = fmaf(v.y, v.y, ss);
    ss = fmaf(v.z, v.z, ss);
    ss = fmaf(v.w, v.w, ss);
  }
  if (p.norm) {
    ss = block_sum_256(ss, s_red);
    const float rstd = 1.0f / sqrtf(ss / (float)H + p.eps);
#pragma unroll
    for (int j = 0; j < kGv; ++j) {
      const int i = (tid + j * kRouterThreads) * 4;
      if (i < H) {
        float4 v = *reinterpret_cast<const float4*>(xs + i);
        const float4 g = gv[j];
        v = make_float4(v.x * rstd * g.x, v.y * rstd * g.y, v.z * rstd * g.z, v.w * rstd * g.w);
        *reinterpret_cast<float4*>(xs + i) = v;
      }
    }
  }
  __syncthreads();

  if (XQB != 0 && p.xq_limbs != nullptr) {  // group g by warp g / NB of CTA g % NB
    for (int g = blockIdx.x + gridDim.x * warp; g < H / kGroup; g += gridDim.x * 8) {
      const float2 v = reinterpret_cast<const float2*>(xs + g * kGroup)[lane];
      xq_quantize_group<XQB == 0 ? 4 : XQB>(v.x, v.y, g, H / kGroup, p.xq_limbs + t * p.xq_limb_stride,
                                            p.xq_cs + t * p.xq_cs_stride);
    }
  }

  // Warp w sums column slice w (H/8 columns) of every row of this CTA: x of the
  // slice is read from shared memory once per 8 columns and reused for every
  // row; the 8 slice sums of a row then add in fixed order.
  const bool ready = nrows > 0 && mbar_wait_bounded(bar, 0, p.err);
  if (ready) {
    const uint16_t* wr = wrows + warp * (H / 8);
    const float* xv = xs + warp * (H / 8);
    float acc[kRouterMaxRows];
#pragma unroll
    for (int r = 0; r < kRouterMaxRows; ++r) acc[r] = 0.0f;
#pragma unroll 1
    for (int k = lane; k < H / 64; k += 32) {  // 8 columns per step
      const float4 xa = *reinterpret_cast<const float4*>(xv + 8 * k);
      const float4 xb = *reinterpret_cast<const float4*>(xv + 8 * k + 4);
#pragma unroll
      for (int r = 0; r < kRouterMaxRows; ++r) {
        if (r < nrows) {
          const uint4 w = *reinterpret_cast<const uint4*>(wr + (size_t)r * H + 8 * k);
          float a = acc[r];
          a = fmaf(bf_lo(w.x), xa.x, a);
          a = fmaf(bf_hi(w.x), xa.y, a);
          a = fmaf(bf_lo(w.y), xa.z, a);
          a = fmaf(bf_hi(w.y), xa.w, a);
          a = fmaf(bf_lo(w.z), xb.x, a);
          a = fmaf(bf_hi(w.z), xb.y, a);
          a = fmaf(bf_lo(w.w), xb.z, a);
          a = fmaf(bf_hi(w.w), xb.w, a);
          acc[r] = a;
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
      for (int r = 0; r < kRouterMaxRows; ++r) acc[r] += __shfl_xor_sync(0xffffffffu, acc[r], o);
    if (lane == 0)
#pragma unroll
      for (int r = 0; r < kRouterMaxRows; ++r)
        if (r < nrows) s_part[r * 8 + warp] = acc[r];
  }
  __syncthreads();
  float* logits = p.logits + (size_t)t * (E + 1);
  if (ready && tid < nrows) {
    float l = 0.0f;
#pragma unroll
    for (int w = 0; w < 8; ++w) l += s_part[tid * 8 + w];
    const int row = r0 + tid;
    if (row < E && p.bias) l += p.bias[row];
    logits[row] = l;
  }
  if (p.top_k <= 0) return;

  // ---- the last CTA of this token selects the experts
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = atomicAdd(&p.tickets[t], 1u) == gridDim.x - 1;
  __syncthreads();
  if (!s_last || warp != 0) return;
  __threadfence();
  const int K = p.top_k;
  int ik;
  float wk, sig;
  warp_topk(logits, E, K, p.w_sgate != nullptr, ik, wk, sig);
  if (lane < K) {
    p.route_idx[(size_t)t * K + lane] = ik;
    p.route_w[(size_t)t * (K + 1) + lane] = wk;
    if (p.idx_out) p.idx_out[(size_t)t * K + lane] = ik;
    if (p.w_out) p.w_out[(size_t)t * K + lane] = wk;
  }
  if (lane == 0) {
    p.route_w[(size_t)t * (K + 1) + K] = sig;
    p.tickets[t] = 0u;
  }
  if (p.cache.state != nullptr) cache_lookup_warp(p.cache, ik, K, cache_slot_out(p.cache), p.err);
}

// One warp per token: top-K, renormalised weights and (optionally) full softmax.
__global__ void __launch_bounds__(32) topk_kernel(const TopkParams p) {
  const int t = blockIdx.x, lane = threadIdx.x;
  const float* l = p.logits + (size_t)t * (p.E + 1);
  int ik;
  float wk, sig;
  warp_topk(l, p.E, p.K, 0, ik, wk, sig);
  if (lane < p.K) {
    p.idx[(size_t)t * p.K + lane] = ik;
    p.w[(size_t)t * p.K + lane] = wk;
  }
  if (p.probs) {
    const float m = __shfl_sync(0xffffffffu, __ldcg(l + ik), 0);  // the largest logit
    float z = 0.0f;
    for (int e = lane; e < p.E; e += 32) z += expf(__ldcg(l + e) - m);
    z = warp_sum(z);
    for (int e = lane; e < p.E; e += 32) p.probs[(size_t)t * p.E + e] = expf(__ldcg(l + e) - m) / z;
  }
}

}  // namespace

cudaError_t launch_rmsnorm(const float* h, const float* gamma, float eps, int T, int H, float* y, cudaStream_t s) {
  rmsnorm_kernel<<<T, 256, 0, s>>>(h, gamma, eps, H, y);
  return cudaGetLastError();
}

cudaError_t launch_xq(const float* x, int H, int bits, uint8_t* limbs, float2* cs, cudaStream_t s) {
  const int groups = H / kGroup;
  const int grid = (groups + 7) / 8;
  if (bits == 8)
    xq_kernel<8><<<grid, 256, 0, s>>>(x, H, limbs, cs);
  else if (bits == 4)
    xq_kernel<4><<<grid, 256, 0, s>>>(x, H, limbs, cs);
  else
    xq_kernel<2><<<grid, 256, 0, s>>>(x, H, limbs, cs);
  return cudaGetLastError();
}

cudaError_t launch_router(RouterParams p, int xq_bits, bool pdl, cudaStream_t s) {
  const int R = p.E + (p.w_sgate ? 1 : 0);
  int rmax = 98304 / (2 * p.H);
  rmax = rmax < 1 ? 1 : (rmax > 8 ? 8 : rmax);
  int nb = num_sms();
  if (nb > R) nb = R;
  if ((R + nb - 1) / nb > rmax) nb = (R + rmax - 1) / rmax;
  p.rows_per_cta = (R + nb - 1) / nb;
  const size_t smem = (size_t)p.rows_per_cta * p.H * 2 + (size_t)p.H * 4;
  cudaError_t e;
  void (*k)(RouterParams) = xq_bits == 8   ? router_kernel<8>
                            : xq_bits == 4 ? router_kernel<4>
                            : xq_bits == 2 ? router_kernel<2>
                                           : router_kernel<0>;
  if ((e = set_smem((const void*)k, smem)) != cudaSuccess) return e;
  return launch_pdl(k, dim3(nb, p.T), dim3(kRouterThreads), smem, s, pdl, p);
}

cudaError_t launch_topk(const TopkParams& p, cudaStream_t s) {
  topk_kernel<<<p.T, 32, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace fmoe
