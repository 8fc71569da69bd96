/*
 * synth.c -- host side of the seeded synthetic input generator (see
 * synth_core.h).  Test and benchmark infrastructure only; it holds no
 * mixture-of-experts arithmetic.
 */
#include "synth_core.h"

#include <string.h>

uint64_t synth_key_c(uint64_t seed, uint32_t layer, uint32_t tensor, uint32_t item) {
  return synth_key(seed, layer, tensor, item);
}

uint64_t synth_draw_c(uint64_t key, uint64_t i) { return synth_draw(key, i); }

uint16_t synth_double_to_bf16_c(double v) { return synth_double_to_bf16(v); }

int64_t synth_blob_bytes_c(const synth_expert_params* p) { return synth_blob_bytes(p); }

/* Writes `count` consecutive expert blobs, experts expert_begin.., into dst. */
void synth_gen_experts(const synth_expert_params* p, int expert_begin, int count, uint8_t* dst) {
  int64_t words = synth_blob_bytes(p) / 8;
  int64_t total = words * (int64_t)count;
  uint64_t* out = (uint64_t*)dst;
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < total; ++i) {
    int e = expert_begin + (int)(i / words);
    out[i] = synth_blob_word(p, e, i % words);
  }
}

/* n normally distributed bf16 values of the stream (seed, layer, tensor, item). */
void synth_gen_normal_bf16(uint64_t seed, uint32_t layer, uint32_t tensor, uint32_t item, int64_t n,
                           double mean, double std, uint16_t* out) {
  uint64_t key = synth_key(seed, layer, tensor, item);
#pragma omp parallel for schedule(static) if (n > 65536)
  for (int64_t i = 0; i < n; ++i) out[i] = synth_normal_elem(key, i, mean, std);
}

/* n uniform bf16 values in [lo, hi) of the stream (seed, layer, tensor, item). */
void synth_gen_uniform_bf16(uint64_t seed, uint32_t layer, uint32_t tensor, uint32_t item, int64_t n,
                            double lo, double hi, uint16_t* out) {
  uint64_t key = synth_key(seed, layer, tensor, item);
  for (int64_t i = 0; i < n; ++i) out[i] = synth_uniform_bf16(synth_draw(key, (uint64_t)i), lo, hi);
}

/* n raw 64-bit draws of the stream (seed, layer, tensor, item). */
void synth_gen_raw(uint64_t seed, uint32_t layer, uint32_t tensor, uint32_t item, int64_t n, uint64_t* out) {
  uint64_t key = synth_key(seed, layer, tensor, item);
  for (int64_t i = 0; i < n; ++i) out[i] = synth_draw(key, (uint64_t)i);
}
