/*
 * gen_host.c -- host build of the seeded input generator (fmoe_gen.h).
 * Compiled with -ffp-contract=off so that every float operation is the single
 * correctly rounded IEEE operation that the device build also performs.
 */
#include <stdlib.h>
#include <string.h>

#include "fmoe_gen.h"

uint64_t fg_host_key(uint64_t seed, uint64_t stream) { return fg_key(seed, stream); }

uint64_t fg_host_stream_id(uint64_t layer, uint64_t expert, uint64_t kind) { return fg_stream_id(layer, expert, kind); }

/* Standard-normal draws times `std`, as fp32. */
void fg_host_normal_f32(uint64_t key, float std, int64_t n, float* out) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = fg_normal(key, (uint64_t)i) * std;
}

/* Standard-normal draws times `std`, rounded to bf16. */
void fg_host_normal_bf16(uint64_t key, float std, int64_t n, uint16_t* out) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = fg_f32_to_bf16(fg_normal(key, (uint64_t)i) * std);
}

/* Uniform integers in [0, n) for draws 0..count-1. */
void fg_host_uniform_u32(uint64_t key, uint32_t n, int64_t count, uint32_t* out) {
  for (int64_t i = 0; i < count; ++i) out[i] = fg_uniform_below(key, (uint64_t)i, n);
}

/* One packed [rows][cols] matrix: qw uint32[rows][cols*bits/32],
 * scale/bias bf16[rows][cols/gs]. */
void fg_host_packed(uint64_t key, float std, int bits, int gs, int rows, int cols, uint32_t* qw, uint16_t* scale,
                    uint16_t* bias) {
  const int wpr = cols * bits / 32, gpr = cols / gs, wpg = gs * bits / 32;
#pragma omp parallel for schedule(static)
  for (int r = 0; r < rows; ++r) {
    float w[256];
    uint32_t* qrow = qw + (int64_t)r * wpr;
    memset(qrow, 0, sizeof(uint32_t) * (size_t)wpr);
    for (int g = 0; g < gpr; ++g) {
      fg_draw_group(key, std, cols, r, g, gs, w);
      fg_quantize_group(w, gs, bits, qrow + g * wpg, scale + (int64_t)r * gpr + g, bias + (int64_t)r * gpr + g);
    }
  }
}
