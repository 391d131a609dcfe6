/*
 * synth_def.h -- the counter-based input generator, one definition for the host
 * (gcc) and the device (nvcc) so that both produce the same bits.
 *
 * This module only makes seeded synthetic inputs for the MoE layer (activations x,
 * router weights, expert weights). It holds none of the layer's arithmetic.
 *
 * Definition (every tensor element is a pure function of seed, tensor id, index):
 *
 *   mix64(z)         : the SplitMix64 output function (Steele, Lea & Flood,
 *                      "Fast splittable pseudorandom number generators", OOPSLA 2014;
 *                      constants of Vigna's public-domain splitmix64):
 *                        z ^= z >> 30; z *= 0xBF58476D1CE4E5B9;
 *                        z ^= z >> 27; z *= 0x94D049BB133111EB; z ^= z >> 31
 *   key(seed, tid)   = mix64(seed ^ mix64(tid * G)),  G = 0x9E3779B97F4A7C15
 *   word(key, c)     = mix64(key + c * G)            (c-th output of a SplitMix64
 *                                                     stream whose state starts at key)
 *   element i        : words c = 3i+1, 3i+2, 3i+3 give twelve 16-bit uniforms U_q;
 *                      S = sum U_q  (an Irwin-Hall(12) sum, mean 393210,
 *                      variance 65536^2 - 1);
 *                      z = (float)(S - 393210) * 2^-16   (exact in fp32);
 *                      v = z * sigma                      (one fp32 multiply, RN);
 *                      bf16 tensors store RNE(v) to bf16.
 *
 * z approximates N(0,1) with tails cut at +-6 (the classical sum-of-twelve-uniforms
 * normal generator).
 */
#ifndef SYNTH_DEF_H
#define SYNTH_DEF_H

#include <stdint.h>

#if defined(__CUDACC__)
#define SYNTH_HD __host__ __device__ __forceinline__
#else
#define SYNTH_HD static inline
#endif

#define SYNTH_GOLDEN 0x9E3779B97F4A7C15ULL

/* tensor ids of the layer's inputs */
enum {
  SYNTH_T_X = 1,             /* x [T][H] bf16, sigma 1            */
  SYNTH_T_W_ROUTER = 2,      /* router weight [E][H] fp32          */
  SYNTH_T_W_GATE_UP = 3,     /* routed gate|up [E][2I][H] bf16     */
  SYNTH_T_W_DOWN = 4,        /* routed down [E][H][I] bf16         */
  SYNTH_T_WS_GATE_UP = 5,    /* shared gate|up [2Is][H] bf16       */
  SYNTH_T_WS_DOWN = 6,       /* shared down [H][Is] bf16           */
  SYNTH_T_W_SHARED_GATE = 7, /* shared-expert gate vector [H] bf16 */
  SYNTH_T_ZIPF_PERM = 8,     /* permutation behind the Zipf bias   */
  SYNTH_T_ZERO_ROWS = 9      /* choice of zeroed gate/up channels  */
};

SYNTH_HD uint64_t synth_mix64(uint64_t z) {
  z ^= z >> 30;
  z *= 0xBF58476D1CE4E5B9ULL;
  z ^= z >> 27;
  z *= 0x94D049BB133111EBULL;
  z ^= z >> 31;
  return z;
}

SYNTH_HD uint64_t synth_key(uint64_t seed, uint32_t tid) {
  return synth_mix64(seed ^ synth_mix64((uint64_t)tid * SYNTH_GOLDEN));
}

SYNTH_HD uint64_t synth_word(uint64_t key, uint64_t c) {
  return synth_mix64(key + c * SYNTH_GOLDEN);
}

/* Irwin-Hall(12) standard value of element i, exact in fp32 */
SYNTH_HD float synth_std(uint64_t key, uint64_t i) {
  int32_t s = 0;
  for (int r = 1; r <= 3; ++r) {
    uint64_t w = synth_word(key, 3 * i + (uint64_t)r);
    s += (int32_t)(w & 0xFFFF) + (int32_t)((w >> 16) & 0xFFFF) +
         (int32_t)((w >> 32) & 0xFFFF) + (int32_t)((w >> 48) & 0xFFFF);
  }
  return (float)(s - 393210) * (1.0f / 65536.0f);
}

SYNTH_HD uint32_t synth_f32_bits(float f) {
  union { float f; uint32_t u; } c;
  c.f = f;
  return c.u;
}

/* fp32 -> bf16, round to nearest even (inputs here are finite) */
SYNTH_HD uint16_t synth_bf16_rne(float f) {
  uint32_t u = synth_f32_bits(f);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

#endif /* SYNTH_DEF_H */
