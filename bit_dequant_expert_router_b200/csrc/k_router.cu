// k_router.cu -- RMSNorm, activation digits, and the router GEMV with softmax / top-K.
//
// RMSNorm follows "What is Flash-MoE" (a2a-mcp.org), section 3: two passes,
// sum of squares then apply.  Routing follows the "Flash-MoE" wiki summary
// (jeongsk), per-layer pipeline: routing projection, softmax, top-K -- except
// that the selection runs on the GPU in the last CTA to finish its rows, so no
// host round trip sits between the router and the experts.
#include "fmoe_internal.h"

namespace fmoe {
namespace {

constexpr int kRouterThreads = 256;

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
  xq_quantize_group<BITS>(v.x, v.y, g, limbs, cs);
}

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint4 ldg_nc(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// grid (NB, T).  Each CTA: x = RMSNorm(h_t) in shared memory; its share of the
// activation digits; rows [b*rpc, b*rpc + rpc) of [Wr; wsg] as 8 warp tasks
// (rows x segments).  The last CTA of token t (ticket) selects the top-K.
template <int XQB>
__global__ void __launch_bounds__(kRouterThreads) router_kernel(const RouterParams p) {
  extern __shared__ __align__(16) float smem[];
  __shared__ float s_red[8];
  __shared__ float s_part[8];
  __shared__ int s_last;
  __shared__ int s_sel_idx[32];
  __shared__ float s_sel_val[32];
  const int t = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int H = p.H, E = p.E, K = p.K;
  float* xs = smem;
  const float* h = p.h + (size_t)t * H;

  float ss = 0.0f;
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
    for (int i = tid; i < H; i += kRouterThreads) xs[i] = xs[i] * rstd * (p.gamma ? p.gamma[i] : 1.0f);
  }
  __syncthreads();

  if (XQB != 0 && p.xq_limbs != nullptr) {
    for (int g = blockIdx.x * 8 + warp; g < H / kGroup; g += gridDim.x * 8) {
      const float2 v = reinterpret_cast<const float2*>(xs + g * kGroup)[lane];
      xq_quantize_group<XQB == 0 ? 4 : XQB>(v.x, v.y, g, p.xq_limbs + t * p.xq_limb_stride,
                                            p.xq_cs + t * p.xq_cs_stride);
    }
  }

  const int R = E + (p.w_sgate ? 1 : 0);
  const int rpc = (R + gridDim.x - 1) / gridDim.x;
  const int r0 = blockIdx.x * rpc;
  const int nrows = min(rpc, R - r0);
  const int S = rpc >= 8 ? 1 : 8 / rpc;  // segments per row: 8, 4, 2 or 1
  if (nrows > 0 && warp < nrows * S) {
    const int row = r0 + warp / S, seg = warp % S;
    const uint16_t* wrow = row < E ? p.w_router + (size_t)row * H : p.w_sgate;
    const int seglen = H / S;
    const uint4* wv = reinterpret_cast<const uint4*>(wrow + seg * seglen);
    const float* xv = xs + seg * seglen;
    float acc = 0.0f;
#pragma unroll 4
    for (int k = lane; k < seglen / 8; k += 32) {
      const uint4 w = ldg_nc(wv + k);
      const float4 xa = *reinterpret_cast<const float4*>(xv + 8 * k);
      const float4 xb = *reinterpret_cast<const float4*>(xv + 8 * k + 4);
      acc = fmaf(bf_lo(w.x), xa.x, acc);
      acc = fmaf(bf_hi(w.x), xa.y, acc);
      acc = fmaf(bf_lo(w.y), xa.z, acc);
      acc = fmaf(bf_hi(w.y), xa.w, acc);
      acc = fmaf(bf_lo(w.z), xb.x, acc);
      acc = fmaf(bf_hi(w.z), xb.y, acc);
      acc = fmaf(bf_lo(w.w), xb.z, acc);
      acc = fmaf(bf_hi(w.w), xb.w, acc);
    }
    acc = warp_sum(acc);
    if (lane == 0) s_part[warp] = acc;
  }
  __syncthreads();
  float* logits = p.logits + (size_t)t * (E + 1);
  if (tid < nrows) {
    float l = 0.0f;
    for (int s = 0; s < S; ++s) l += s_part[tid * S + s];
    const int row = r0 + tid;
    if (row < E && p.bias) l += p.bias[row];
    logits[row] = l;
  }

  // ---- last CTA of this token selects
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    const unsigned prev = atomicAdd(&p.tickets[t], 1u);
    s_last = prev == gridDim.x - 1;
  }
  __syncthreads();
  if (!s_last || warp != 0) return;
  __threadfence();
  float* sl = xs;  // x is no longer needed; smem holds max(H, E) floats
  for (int e = lane; e < E; e += 32) sl[e] = __ldcg(logits + e);
  __syncwarp();
  for (int k = 0; k < K; ++k) {
    float bv = -INFINITY;
    int bi = 0x7fffffff;
    for (int e = lane; e < E; e += 32) {
      const float v = sl[e];
      if (v > bv || (v == bv && e < bi)) {
        bv = v;
        bi = e;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > bv || (ov == bv && oi < bi)) {
        bv = ov;
        bi = oi;
      }
    }
    if (bi >= E) bi = 0;  // only reachable with non-finite logits
    if (lane == 0) {
      s_sel_idx[k] = bi;
      s_sel_val[k] = bv;
    }
    if ((bi & 31) == lane) sl[bi] = -INFINITY;
    __syncwarp();
  }
  const float m = s_sel_val[0];
  const float ek = lane < K ? expf(s_sel_val[lane] - m) : 0.0f;
  const float esum = warp_sum(ek);
  if (lane < K) {
    const float wk = ek / esum;
    const int ik = s_sel_idx[lane];
    p.idx[t * K + lane] = ik;
    p.wts[t * (K + 1) + lane] = wk;
    if (p.idx_out) p.idx_out[t * K + lane] = ik;
    if (p.w_out) p.w_out[t * K + lane] = wk;
  }
  if (lane == 0) p.wts[t * (K + 1) + K] = p.w_sgate ? 1.0f / (1.0f + expf(-__ldcg(logits + E))) : 0.0f;
  if (p.probs_out) {
    float z = 0.0f;
    for (int e = lane; e < E; e += 32) z += expf(__ldcg(logits + e) - m);
    z = warp_sum(z);
    for (int e = lane; e < E; e += 32) p.probs_out[(size_t)t * E + e] = expf(__ldcg(logits + e) - m) / z;
  }
  if (lane == 0) p.tickets[t] = 0u;
}

}  // namespace

cudaError_t launch_rmsnorm(const float* h, const float* gamma, float eps, int T, int H, float* y, cudaStream_t s) {
  rmsnorm_kernel<<<T, 256, 0, s>>>(h, gamma, eps, H, y);
  return cudaGetLastError();
}

cudaError_t launch_xq(const float* x, int H, int bits, uint8_t* limbs, float2* cs, cudaStream_t s) {
  const int groups = H / kGroup;
  const int grid = (groups + 7) / 8;
  if (bits == 4)
    xq_kernel<4><<<grid, 256, 0, s>>>(x, H, limbs, cs);
  else
    xq_kernel<2><<<grid, 256, 0, s>>>(x, H, limbs, cs);
  return cudaGetLastError();
}

cudaError_t launch_router(const RouterParams& p, int xq_bits, cudaStream_t s) {
  const int R = p.E + (p.w_sgate ? 1 : 0);
  int nb = num_sms();
  if (nb > R) nb = R;
  if ((R + nb - 1) / nb > 8 && nb < (R + 7) / 8) nb = (R + 7) / 8;
  const size_t smem = sizeof(float) * (size_t)(p.H > p.E ? p.H : p.E);
  dim3 grid(nb, p.T);
  if (xq_bits == 4)
    router_kernel<4><<<grid, kRouterThreads, smem, s>>>(p);
  else if (xq_bits == 2)
    router_kernel<2><<<grid, kRouterThreads, smem, s>>>(p);
  else
    router_kernel<0><<<grid, kRouterThreads, smem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace fmoe
