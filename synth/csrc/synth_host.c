/*
 * synth_host.c -- host half of the seeded input generator (see synth_def.h).
 * Plain C with pthreads; built into libsynth_host.so and called through ctypes.
 * It produces inputs only (activations and weights); no step of the MoE layer
 * is computed here.
 */
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include "synth_def.h"

typedef struct {
  void* out;
  uint64_t begin, end;      /* element range of this worker       */
  uint64_t key;
  uint64_t index_offset;    /* flat index of out[0] in the tensor */
  float sigma;
  int bf16;
  /* gate|up zero-row masking (NULL = none) */
  const uint8_t* zero_mask; /* [E][I], 1 = channel zeroed          */
  uint64_t I, H;
} fill_job;

static void* fill_worker(void* arg) {
  fill_job* j = (fill_job*)arg;
  for (uint64_t n = j->begin; n < j->end; ++n) {
    uint64_t idx = j->index_offset + n;
    float v;
    int zeroed = 0;
    if (j->zero_mask) {
      uint64_t row = idx / j->H;              /* row of the [E*2I][H] view */
      uint64_t e = row / (2 * j->I);
      uint64_t ch = (row % (2 * j->I)) % j->I; /* gate row ch or up row I+ch */
      zeroed = j->zero_mask[e * j->I + ch] != 0;
    }
    if (zeroed) {
      v = 0.0f;
    } else {
      float z = synth_std(j->key, idx);
      v = z * j->sigma;
    }
    if (j->bf16)
      ((uint16_t*)j->out)[n] = synth_bf16_rne(v);
    else
      ((float*)j->out)[n] = v;
  }
  return NULL;
}

static void run_fill(void* out, uint64_t n, uint64_t seed, uint32_t tid, float sigma,
                     uint64_t index_offset, int bf16, const uint8_t* zero_mask,
                     uint64_t I, uint64_t H, int nthreads) {
  if (n == 0) return;
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if ((uint64_t)nthreads > n) nthreads = (int)n;
  uint64_t key = synth_key(seed, tid);
  fill_job jobs[256];
  pthread_t th[256];
  uint64_t chunk = (n + (uint64_t)nthreads - 1) / (uint64_t)nthreads;
  int launched = 0;
  for (int t = 0; t < nthreads; ++t) {
    uint64_t b = (uint64_t)t * chunk;
    if (b >= n) break;
    uint64_t e = b + chunk < n ? b + chunk : n;
    fill_job j = {out, b, e, key, index_offset, sigma, bf16, zero_mask, I, H};
    jobs[t] = j;
    launched++;
  }
  for (int t = 1; t < launched; ++t) {
    if (pthread_create(&th[t], NULL, fill_worker, &jobs[t]) != 0) {
      fill_worker(&jobs[t]); /* no thread: do the work here */
      th[t] = 0;
    }
  }
  fill_worker(&jobs[0]);
  for (int t = 1; t < launched; ++t)
    if (th[t]) pthread_join(th[t], NULL);
}

/* Elements [index_offset, index_offset+n) of tensor `tid`, as bf16 bits. */
void synth_fill_bf16(uint16_t* out, uint64_t n, uint64_t seed, uint32_t tid, float sigma,
                     uint64_t index_offset, int nthreads) {
  run_fill(out, n, seed, tid, sigma, index_offset, 1, NULL, 1, 1, nthreads);
}

/* Elements [index_offset, index_offset+n) of tensor `tid`, as fp32. */
void synth_fill_f32(float* out, uint64_t n, uint64_t seed, uint32_t tid, float sigma,
                    uint64_t index_offset, int nthreads) {
  run_fill(out, n, seed, tid, sigma, index_offset, 0, NULL, 1, 1, nthreads);
}

/*
 * Routed gate|up weights [E][2I][H] (bf16), experts [e_begin, e_begin+e_count).
 * zero_mask [E][I] (or NULL): channel ch of expert e is zero in both its gate
 * row ch and its up row I+ch.
 */
void synth_fill_gate_up_bf16(uint16_t* out, uint64_t e_begin, uint64_t e_count, uint64_t I,
                             uint64_t H, uint64_t seed, uint32_t tid, float sigma,
                             const uint8_t* zero_mask, int nthreads) {
  uint64_t per = 2 * I * H;
  run_fill(out, e_count * per, seed, tid, sigma, e_begin * per, 1, zero_mask, I, H,
           nthreads);
}

/* One 64-bit word of stream (seed, tid) at counter c (c >= 1). */
uint64_t synth_word_at(uint64_t seed, uint32_t tid, uint64_t c) {
  return synth_word(synth_key(seed, tid), c);
}

/*
 * Seeded Fisher-Yates permutation of 0..n-1 of stream (seed, tid, sub):
 * for i = n-1 down to 1, j = word(sub*2^32 + (n-1-i) + 1) mod (i+1), swap.
 */
void synth_permutation(int32_t* perm, uint32_t n, uint64_t seed, uint32_t tid, uint32_t sub) {
  uint64_t key = synth_key(seed, tid);
  for (uint32_t i = 0; i < n; ++i) perm[i] = (int32_t)i;
  for (uint32_t s = 0; s + 1 < n; ++s) {
    uint32_t i = n - 1 - s;
    uint64_t w = synth_word(key, ((uint64_t)sub << 32) + (uint64_t)s + 1);
    uint32_t j = (uint32_t)(w % (uint64_t)(i + 1));
    int32_t t = perm[i];
    perm[i] = perm[j];
    perm[j] = t;
  }
}

/* c-th output (c >= 1) of a plain SplitMix64 stream whose state starts at `state`. */
uint64_t synth_splitmix64_at(uint64_t state, uint64_t c) { return synth_word(state, c); }
