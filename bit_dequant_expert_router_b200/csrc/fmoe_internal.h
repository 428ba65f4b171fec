// fmoe_internal.h -- host-side declarations shared by the C-ABI layer and the kernel files.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "fmoe_device.cuh"

namespace fmoe {

// Router GEMV + last-CTA softmax/top-K, one grid row (blockIdx.y) per token.
struct RouterParams {
  const float* h;             // [T][H] input (normalised in-kernel when norm != 0)
  const float* gamma;         // [H] or NULL (unit)
  float eps;
  int norm;                   // 1: x = RMSNorm(h); 0: x = h
  const uint16_t* w_router;   // bf16 [E][H]
  const float* bias;          // [E] or NULL
  const uint16_t* w_sgate;    // bf16 [H] or NULL (no shared-gate row)
  int T, H, E, K;
  uint8_t* xq_limbs;          // per-token activation digits, or NULL
  float2* xq_cs;
  long long xq_limb_stride;   // bytes per token
  long long xq_cs_stride;     // float2 per token
  float* logits;              // [T][E+1]
  int32_t* idx;               // [T][K]
  float* wts;                 // [T][K+1]: routing weights, slot K = shared gate sigma
  int32_t* idx_out;           // optional [T][K]
  float* w_out;               // optional [T][K]
  float* probs_out;           // optional [T][E]
  unsigned int* tickets;      // [T], zero on entry, zero on exit
  int* err;
};

struct ExpertParams {
  BankRef routed;
  BankRef shared;
  const int32_t* idx;         // [K] routed slots, or NULL -> fixed_expert
  int fixed_expert;
  int K;                      // routed slots
  int has_shared;             // slot K is the shared expert
  int H, I;
  const uint32_t* xq_limbs;   // gate/up: digits of x (chunk-major)
  const float2* xq_cs;
  float* act;                 // [K+has_shared][I]: gate/up output, down input
  const float* wts;           // down: per-slot weights [K+1] or NULL (all 1)
  const float* resid;         // down: residual [H] or NULL
  float* out;                 // down: [H]
  int* err;
};

cudaError_t launch_rmsnorm(const float* h, const float* gamma, float eps, int T, int H, float* y, cudaStream_t s);
cudaError_t launch_router(const RouterParams& p, int xq_bits, cudaStream_t s);
cudaError_t launch_gateup(const ExpertParams& p, int bits, cudaStream_t s);
cudaError_t launch_down(const ExpertParams& p, int bits, cudaStream_t s);

int num_sms();

}  // namespace fmoe
