/*
 * moe_inputs.h -- seeded, counter-based synthetic input generator.
 *
 * This header is the single definition of every synthetic tensor used by the
 * tests and the benchmark.  It is shared, unchanged, by a host build (g++/nvcc
 * host pass) and a device build (nvcc device pass), so host-generated and
 * device-generated tensors are bit-identical by construction: every step below
 * is integer arithmetic, one exact int->float conversion and one IEEE
 * single-precision multiply, followed by an integer round-to-nearest-even to
 * bf16.  It holds none of the layer's arithmetic (no routing, no FFN).
 *
 * Random bits: SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom
 * number generators", OOPSLA 2014; the mixing function and increment are the
 * published ones).  Element i of a stream with key K uses the three 64-bit words
 *     w_c = mix64(K + GOLDEN * (3*i + c + 1)),   c = 0, 1, 2
 * so any element can be generated on its own (random access by index).
 *
 * Normal variates: Irwin-Hall sum of twelve independent uniform 16-bit
 * integers (the four 16-bit chunks of each w_c), centred and scaled by 2^-16:
 *     z = (sum - 12*65535/2) / 65536,   E[z] = 0,  Var[z] = 1 - 2^-32
 * z takes values on a 2^-16 grid in [-6, 6]; its excess kurtosis is -0.1, the
 * textbook twelve-uniform approximation of N(0,1).  A N(0, sigma^2) draw is
 * z * sigma rounded once to fp32, then to bf16 (round to nearest even).
 *
 * Stream keys: key(seed, stream, redraw) = mix64(mix64(seed) ^ mix64((stream << 32) | redraw)).
 * "redraw" selects an independent substream for the same tensor (used when a
 * test harness redraws a token row); it is 0 for every first draw.
 */
#ifndef MOE_INPUTS_H
#define MOE_INPUTS_H

#include <stdint.h>

#if defined(__CUDACC__)
#define MI_FN __host__ __device__ __forceinline__
#else
#define MI_FN static inline
#endif

#define MI_GOLDEN 0x9E3779B97F4A7C15ULL

/* Stream identifiers: one per synthetic tensor. */
enum {
  MI_STREAM_X = 1,          /* activations x[T, D]                      */
  MI_STREAM_WG = 2,         /* router weight W_g[E, D]                  */
  MI_STREAM_GATE_UP = 3,    /* routed experts gate_up_proj[E, 2F, D]    */
  MI_STREAM_DOWN = 4,       /* routed experts down_proj[E, D, F]        */
  MI_STREAM_SH_GATE_UP = 5, /* shared expert gate_up[2Fs, D]            */
  MI_STREAM_SH_DOWN = 6,    /* shared expert down[D, Fs]                */
  MI_STREAM_BIAS = 7,       /* per-expert selection bias[E] (normal)    */
  MI_STREAM_RANK = 8        /* per-expert rank permutation (Zipf bias)  */
};

MI_FN uint64_t mi_mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

MI_FN uint64_t mi_stream_key(uint64_t seed, uint32_t stream, uint32_t redraw) {
  return mi_mix64(mi_mix64(seed) ^ mi_mix64(((uint64_t)stream << 32) | (uint64_t)redraw));
}

/* 64-bit uniform word number `i` of a stream (used for permutations). */
MI_FN uint64_t mi_word(uint64_t key, uint64_t i) {
  return mi_mix64(key + MI_GOLDEN * (i + 1ULL));
}

/* Standard (approximately) normal variate number `i` of a stream, exact in fp32. */
MI_FN float mi_normal(uint64_t key, uint64_t i) {
  int32_t s = 0;
  for (int c = 0; c < 3; ++c) {
    uint64_t w = mi_mix64(key + MI_GOLDEN * (3ULL * i + (uint64_t)c + 1ULL));
    s += (int32_t)(w & 0xFFFFu) + (int32_t)((w >> 16) & 0xFFFFu) +
         (int32_t)((w >> 32) & 0xFFFFu) + (int32_t)((w >> 48) & 0xFFFFu);
  }
  /* |s - 393210| < 2^19, so the conversion and the power-of-two scale are exact. */
  return (float)(s - 393210) * (1.0f / 65536.0f);
}

MI_FN float mi_scale(float z, float sigma) {
#if defined(__CUDA_ARCH__)
  return __fmul_rn(z, sigma);
#else
  return z * sigma;
#endif
}

/* fp32 -> bf16 bits, round to nearest even (inputs here are always finite). */
MI_FN uint16_t mi_f32_to_bf16(float f) {
  union { float f; uint32_t u; } v;
  v.f = f;
  uint32_t u = v.u;
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

MI_FN uint16_t mi_normal_bf16(uint64_t key, uint64_t i, float sigma) {
  return mi_f32_to_bf16(mi_scale(mi_normal(key, i), sigma));
}

#endif /* MOE_INPUTS_H */
