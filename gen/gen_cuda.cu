/*
 * gen_cuda.cu -- device build of the seeded input generator (fmoe_gen.h).
 * Fills device buffers with the same bytes the host build produces; used by
 * the tests and the benchmark to synthesise multi-GB expert banks in HBM.
 * Compiled with -fmad=false (no FMA contraction).
 */
#include <cuda_runtime.h>

#include "fmoe_gen.h"

namespace {

__global__ void packed_bank_kernel(uint64_t seed, uint64_t layer, uint64_t expert_id0, int ne, int kind, float std,
                                   int bits, int gs, int rows, int cols, unsigned char* base, long long stride,
                                   long long off_qw, long long off_s, long long off_b) {
  const int gpr = cols / gs, wpr = cols * bits / 32, wpg = gs * bits / 32;
  const long long total = (long long)ne * rows * gpr;
  for (long long t = blockIdx.x * (long long)blockDim.x + threadIdx.x; t < total;
       t += (long long)gridDim.x * blockDim.x) {
    const int g = (int)(t % gpr);
    const int r = (int)((t / gpr) % rows);
    const int e = (int)(t / ((long long)gpr * rows));
    const uint64_t key = fg_key(seed, fg_stream_id(layer, expert_id0 + (uint64_t)e, (uint64_t)kind));
    float w[256];
    uint32_t words[32];
    for (int i = 0; i < wpg; ++i) words[i] = 0u;
    fg_draw_group(key, std, cols, r, g, gs, w);
    uint16_t sb, bb;
    fg_quantize_group(w, gs, bits, words, &sb, &bb);
    unsigned char* rec = base + (long long)e * stride;
    uint32_t* qw = (uint32_t*)(rec + off_qw) + (long long)r * wpr + (long long)g * wpg;
    for (int i = 0; i < wpg; ++i) qw[i] = words[i];
    ((uint16_t*)(rec + off_s))[(long long)r * gpr + g] = sb;
    ((uint16_t*)(rec + off_b))[(long long)r * gpr + g] = bb;
  }
}

__global__ void normal_f32_kernel(uint64_t key, float std, long long n, float* out) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
    out[i] = fg_normal(key, (uint64_t)i) * std;
}

__global__ void normal_bf16_kernel(uint64_t key, float std, long long n, uint16_t* out) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
    out[i] = fg_f32_to_bf16(fg_normal(key, (uint64_t)i) * std);
}

int grid_for(long long n) {
  long long b = (n + 255) / 256;
  return (int)(b < 148 * 64 ? (b < 1 ? 1 : b) : 148 * 64);
}

}  // namespace

extern "C" {

/* Fills matrices `kind` (gate/up/down) of experts expert_id0 .. expert_id0+ne-1
 * of `layer`, record e at base + e*stride.  Returns a cudaError_t value. */
int fg_cuda_packed_bank(uint64_t seed, uint64_t layer, uint64_t expert_id0, int ne, int kind, float std, int bits,
                        int gs, int rows, int cols, void* base, long long stride, long long off_qw, long long off_s,
                        long long off_b, cudaStream_t stream) {
  if (gs > 256 || gs * bits / 32 > 32 || cols % gs != 0 || (gs * bits) % 32 != 0) return (int)cudaErrorInvalidValue;
  const long long total = (long long)ne * rows * (cols / gs);
  packed_bank_kernel<<<grid_for(total), 256, 0, stream>>>(seed, layer, expert_id0, ne, kind, std, bits, gs, rows, cols,
                                                          (unsigned char*)base, stride, off_qw, off_s, off_b);
  return (int)cudaGetLastError();
}

int fg_cuda_normal_f32(uint64_t key, float std, long long n, float* out, cudaStream_t stream) {
  if (n <= 0) return 0;
  normal_f32_kernel<<<grid_for(n), 256, 0, stream>>>(key, std, n, out);
  return (int)cudaGetLastError();
}

int fg_cuda_normal_bf16(uint64_t key, float std, long long n, uint16_t* out, cudaStream_t stream) {
  if (n <= 0) return 0;
  normal_bf16_kernel<<<grid_for(n), 256, 0, stream>>>(key, std, n, out);
  return (int)cudaGetLastError();
}

}  // extern "C"
