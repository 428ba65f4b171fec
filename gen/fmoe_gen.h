/*
 * fmoe_gen.h -- seeded synthetic-input generator shared by the test harness,
 * the benchmark, the CPU oracle's inputs and the GPU inputs.
 *
 * This header holds no arithmetic of the MoE block itself.  It draws the
 * synthetic "checkpoint" and token inputs that both sides consume:
 *   - a counter-based generator (SplitMix64 finaliser over a Weyl sequence),
 *   - Gaussian draws as Irwin-Hall(12) sums of 16-bit uniforms, which are
 *     integer-exact and therefore bit-identical on the host and the device,
 *   - the offline weight writer: round-to-nearest-even fp32->bf16 and the
 *     min/max affine group quantiser that turns fp32 weights into packed
 *     codes plus bf16 scale/bias (the synthetic stand-in for the weight
 *     conversion scripts of the Flash-MoE repository; it is never on the
 *     inference path).
 *
 * Every operation is integer or a single correctly rounded IEEE fp32
 * add/sub/mul/div/rint, and the translation units that include this header
 * are compiled without FMA contraction, so the host build and the device
 * build produce the same bytes.
 */
#ifndef FMOE_GEN_H
#define FMOE_GEN_H

#include <stdint.h>

#if defined(__CUDACC__)
#define FG_FN static __host__ __device__ __forceinline__
#else
#include <math.h>
#include <string.h>
#define FG_FN static inline
#endif

#define FG_GOLDEN 0x9E3779B97F4A7C15ull

/* SplitMix64 output function applied to an arbitrary 64-bit state. */
FG_FN uint64_t fg_mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

/* Key of an independent stream: (seed, stream id) -> 64-bit key. */
FG_FN uint64_t fg_key(uint64_t seed, uint64_t stream) {
  return fg_mix64(fg_mix64(seed + FG_GOLDEN) ^ (stream * 0xD1B54A32D192ED03ull + FG_GOLDEN));
}

/* Draw number `ctr` of the stream with key `key`. */
FG_FN uint64_t fg_draw(uint64_t key, uint64_t ctr) {
  return fg_mix64(key + (ctr + 1ull) * FG_GOLDEN);
}

FG_FN uint32_t fg_sum16x4(uint64_t v) {
  return (uint32_t)(v & 0xFFFFu) + (uint32_t)((v >> 16) & 0xFFFFu) +
         (uint32_t)((v >> 32) & 0xFFFFu) + (uint32_t)(v >> 48);
}

/* Standard normal number i of stream `key`: Irwin-Hall sum of twelve 16-bit
 * uniforms (u+0.5)/65536, minus 6.  The integer numerator is below 2^24, so
 * the conversion and the power-of-two scaling are exact. */
FG_FN float fg_normal(uint64_t key, uint64_t i) {
  uint32_t s = fg_sum16x4(fg_draw(key, 3u * i)) + fg_sum16x4(fg_draw(key, 3u * i + 1u)) +
               fg_sum16x4(fg_draw(key, 3u * i + 2u));
  return (float)((int32_t)s - 393210) * (1.0f / 65536.0f);
}

/* Uniform integer in [0, n) (n < 2^32) for draw `i`: multiply-shift. */
FG_FN uint32_t fg_uniform_below(uint64_t key, uint64_t i, uint32_t n) {
  return (uint32_t)(((fg_draw(key, i) >> 32) * (uint64_t)n) >> 32);
}

FG_FN uint32_t fg_f32_bits(float f) {
#if defined(__CUDA_ARCH__)
  return __float_as_uint(f);
#else
  uint32_t u;
  memcpy(&u, &f, 4);
  return u;
#endif
}

FG_FN float fg_bits_f32(uint32_t u) {
#if defined(__CUDA_ARCH__)
  return __uint_as_float(u);
#else
  float f;
  memcpy(&f, &u, 4);
  return f;
#endif
}

/* fp32 -> bf16, round to nearest even (inputs here are finite). */
FG_FN uint16_t fg_f32_to_bf16(float f) {
  uint32_t u = fg_f32_bits(f);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

FG_FN float fg_bf16_to_f32(uint16_t b) { return fg_bits_f32((uint32_t)b << 16); }

/* Offline writer for one group of `gs` fp32 weights (gs*bits a multiple of
 * 32): min/max affine code, scale = bf16((max-min)/(2^bits-1)),
 * bias = bf16(min), code = clamp(rint((w - bias)/scale)), packed LSB-first
 * (code j of a word at bits [bits*j, bits*j+bits)).  The group's words are
 * OR-ed into `words`, which the caller zeroes. */
FG_FN void fg_quantize_group(const float* w, int gs, int bits, uint32_t* words, uint16_t* scale_out,
                             uint16_t* bias_out) {
  float mn = w[0], mx = w[0];
  for (int i = 1; i < gs; ++i) {
    mn = w[i] < mn ? w[i] : mn;
    mx = w[i] > mx ? w[i] : mx;
  }
  const int qmax = (1 << bits) - 1;
  const uint16_t sb = fg_f32_to_bf16((mx - mn) / (float)qmax);
  const uint16_t bb = fg_f32_to_bf16(mn);
  const float s = fg_bf16_to_f32(sb), b = fg_bf16_to_f32(bb);
  const int per_word = 32 / bits;
  for (int i = 0; i < gs; ++i) {
    int q = 0;
    if (s > 0.0f) {
      float t = rintf((w[i] - b) / s);
      q = t < 0.0f ? 0 : (t > (float)qmax ? qmax : (int)t);
    }
    words[i / per_word] |= (uint32_t)q << (bits * (i % per_word));
  }
  *scale_out = sb;
  *bias_out = bb;
}

/* Stream id of one synthetic tensor: layer, expert id (28 bits; the shared
 * expert and per-layer vectors use the ids below) and tensor kind. */
#define FG_EXPERT_SHARED 0xFFFFFFFull
#define FG_EXPERT_LAYER 0xFFFFFFEull
enum { FG_GATE = 0, FG_UP = 1, FG_DOWN = 2, FG_ROUTER = 3, FG_SHARED_GATE = 4, FG_GAMMA = 5, FG_PERM = 6 };
FG_FN uint64_t fg_stream_id(uint64_t layer, uint64_t expert, uint64_t kind) {
  return (layer << 36) | ((expert & 0xFFFFFFFull) << 4) | (kind & 0xFull);
}

/* Weights of row r, group g of a [rows][cols] matrix drawn from stream `key`
 * with standard deviation `std`: element (r,c) is normal number r*cols+c. */
FG_FN void fg_draw_group(uint64_t key, float std, int cols, int r, int g, int gs, float* w) {
  const uint64_t base = (uint64_t)r * (uint64_t)cols + (uint64_t)g * (uint64_t)gs;
  for (int i = 0; i < gs; ++i) w[i] = fg_normal(key, base + (uint64_t)i) * std;
}

#endif /* FMOE_GEN_H */
