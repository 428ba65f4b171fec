// k_gdn.cu -- Gated DeltaNet state update of the linear-attention layers, one decode step.
//
// "What is Flash-MoE" (a2a-mcp.org), section 4, and the "Flash-MoE" wiki summary
// (jeongsk), key technique 4: each linear-attention layer keeps a 128 x 128 fp32 state
// per head, 64 heads, and updates it per token with a scaling, a matrix-vector product
// and a rank-1 update (sscal, sgemv and sger in the pages' CPU code).  Per head, with S
// stored [dv][dk] (row i = value coordinate i):
//   S <- alpha S;  u = S k;  S <- S + beta (v - u) k^T;  o = S q.
// Every step touches a row of S only through that row, k, q, v_i, alpha and beta, so the
// kernel gives each state row to one warp and does all four steps on it in registers:
// one read and one write of the state, which is the whole of the HBM traffic (plus the
// small vectors).  A lane holds dk/32 floats of a row, four consecutive ones in each
// 128-column block; the two dot products are lane partial sums (fma, in column order)
// and a butterfly over the warp.
//
// The state is read with the streaming hint and, when the caller says the launch before
// this one on the stream does not write it, before the dependency wait: with dependent
// launch the reads of one layer's state then overlap the tail of the previous kernel.
#include <cstdlib>

#include "fmoe_internal.h"

namespace fmoe {
namespace {

// 8 warps per CTA: CTAs of 4 warps measured slower (3.03 against 2.32 us per step).
constexpr int kGdnWarps = 8;

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

__device__ __forceinline__ float dot4(const float4 a, const float4 b, float acc) {
  acc = fmaf(a.x, b.x, acc);
  acc = fmaf(a.y, b.y, acc);
  acc = fmaf(a.z, b.z, acc);
  return fmaf(a.w, b.w, acc);
}

// NC float4 per lane per row (dk = 128 NC); R consecutive rows per warp.
template <int NC, int R>
__global__ void __launch_bounds__(kGdnWarps * 32) gdn_step_kernel(const GdnParams p) {
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const long long row0 = ((long long)blockIdx.x * kGdnWarps + warp) * R;
  float4 s[R][NC];
  auto load_rows = [&]() {
#pragma unroll
    for (int r = 0; r < R; ++r) {
      if (row0 + r < p.rows) {
        const float4* src = reinterpret_cast<const float4*>(p.state + (row0 + r) * p.dk) + lane;
#pragma unroll
        for (int c = 0; c < NC; ++c) s[r][c] = __ldcs(src + 32 * c);
      }
    }
  };
  if (p.early) load_rows();
  pdl_trigger();
  pdl_wait();
  if (!p.early) load_rows();

  // this warp's small operands, all requested before any arithmetic (one L2 round trip)
  float a[R], b[R], vi[R];
  float4 kk[R][NC], qq[R][NC];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const long long row = row0 + r;
    if (row < p.rows) {
      const int head = (int)(row / p.dv);
      a[r] = __ldg(p.alpha + head);
      b[r] = __ldg(p.beta + head);
      vi[r] = __ldg(p.v + row);
      const float4* k4 = reinterpret_cast<const float4*>(p.k + (long long)head * p.dk) + lane;
      const float4* q4 = reinterpret_cast<const float4*>(p.q + (long long)head * p.dk) + lane;
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        kk[r][c] = __ldg(k4 + 32 * c);
        qq[r][c] = __ldg(q4 + 32 * c);
      }
    }
  }

#pragma unroll
  for (int r = 0; r < R; ++r) {
    const long long row = row0 + r;
    if (row >= p.rows) break;  // uniform over the warp
    float part = 0.0f;
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      s[r][c].x *= a[r];  // S <- alpha S
      s[r][c].y *= a[r];
      s[r][c].z *= a[r];
      s[r][c].w *= a[r];
      part = dot4(s[r][c], kk[r][c], part);
    }
    const float u = warp_sum(part);  // u_i = S[i] . k
    const float d = b[r] * (vi[r] - u);
    part = 0.0f;
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      s[r][c].x = fmaf(d, kk[r][c].x, s[r][c].x);  // S[i] <- S[i] + beta (v_i - u_i) k
      s[r][c].y = fmaf(d, kk[r][c].y, s[r][c].y);
      s[r][c].z = fmaf(d, kk[r][c].z, s[r][c].z);
      s[r][c].w = fmaf(d, kk[r][c].w, s[r][c].w);
      part = dot4(s[r][c], qq[r][c], part);
    }
    const float oi = warp_sum(part);  // o_i = S[i] . q
    float4* dst = reinterpret_cast<float4*>(p.state + row * p.dk) + lane;
#pragma unroll
    for (int c = 0; c < NC; ++c) __stcs(dst + 32 * c, s[r][c]);
    if (lane == 0) p.o[row] = oi;
  }
}

template <int NC, int R>
cudaError_t launch_nc(const GdnParams& p, bool pdl, cudaStream_t s) {
  const long long warps = ((long long)p.rows + R - 1) / R;
  const unsigned blocks = (unsigned)((warps + kGdnWarps - 1) / kGdnWarps);
  return launch_pdl(gdn_step_kernel<NC, R>, dim3(blocks), dim3(kGdnWarps * 32), 0, s, pdl, p);
}

// Rows per warp at dk = 128 (FMOE_GDN_RPW: 1, 2 or 4).  One row per warp measured fastest
// (2.31 us per 64-head step against 2.60 with two and 4.09 with four): every state row of
// the step is requested at once, and no warp works through two rows in turn.
int rows_per_warp() {
  static const int r = [] {  // read once (thread-safe static initialisation)
    const char* e = getenv("FMOE_GDN_RPW");
    return (e && (e[0] == '1' || e[0] == '2' || e[0] == '4')) ? e[0] - '0' : 1;
  }();
  return r;
}

}  // namespace

bool gdn_shape_supported(int dk) { return dk == 128 || dk == 256 || dk == 384 || dk == 512; }

cudaError_t launch_gdn_step(const GdnParams& p, bool pdl, cudaStream_t s) {
  switch (p.dk) {
    case 128: {
      const int r = rows_per_warp();
      return r == 1 ? launch_nc<1, 1>(p, pdl, s) : r == 4 ? launch_nc<1, 4>(p, pdl, s) : launch_nc<1, 2>(p, pdl, s);
    }
    case 256: return launch_nc<2, 1>(p, pdl, s);
    case 384: return launch_nc<3, 1>(p, pdl, s);
    case 512: return launch_nc<4, 1>(p, pdl, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace fmoe
