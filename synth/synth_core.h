/*
 * synth_core.h -- seeded, counter-based synthetic input generator.
 *
 * This module is test and benchmark infrastructure.  It produces the synthetic
 * tensors that stand in for the trained Qwen3.5-397B-A17B weights the Flash-MoE
 * pages run on (the themata summary "Flash-MoE: Running a 397B Parameter Model
 * on a Laptop", Key Takeaways: 60 layers, 512 experts, K=4; the Hysen Labs page
 * of the same title, section "How the SSD expert streaming pipeline works":
 * hidden 4096, one shared expert).  It holds none of
 * the mixture-of-experts arithmetic: it only draws random bits and turns them
 * into bf16 numbers and packed integer codes in the canonical expert-blob format.
 *
 * Both the host library (synth.c) and the device generator (synth_cuda.cu)
 * include this header, so the same (seed, layer, tensor, item, index) gives the
 * same bytes on either side.  Every floating-point step is a single IEEE
 * operation with an explicit rounding (no contraction), so results are
 * bit-identical between gcc and nvcc.
 *
 * Random stream: SplitMix64 (G. Steele, D. Lea, C. Flood, "Fast splittable
 * pseudorandom number generators", OOPSLA 2014; constants as published by
 * S. Vigna).  Draw i of a stream with key k is mix(k + (i+1)*0x9E3779B97F4A7C15),
 * i.e. the i-th output of a SplitMix64 generator seeded with k.
 */
#ifndef SYNTH_CORE_H
#define SYNTH_CORE_H

#include <stdint.h>
#include <stddef.h>

#if defined(__CUDACC__)
#define SYNTH_FN __host__ __device__ static inline
#else
#define SYNTH_FN static inline
#endif

#if defined(__CUDA_ARCH__)
#define SYNTH_DMUL(a, b) __dmul_rn((a), (b))
#define SYNTH_DADD(a, b) __dadd_rn((a), (b))
#else
/* host: compiled with -ffp-contract=off, so these are single roundings */
#define SYNTH_DMUL(a, b) ((a) * (b))
#define SYNTH_DADD(a, b) ((a) + (b))
#endif

/* Tensor identifiers used to key independent streams. */
enum {
  SYNTH_T_CODES = 1,   /* +0 gate, +1 up, +2 down */
  SYNTH_T_SCALE = 4,   /* +0 gate, +1 up, +2 down */
  SYNTH_T_BIAS = 7,    /* +0 gate, +1 up, +2 down */
  SYNTH_T_ROUTER = 10, /* router weight [E][H] */
  SYNTH_T_NORM = 11,   /* RMSNorm weight [H] */
  SYNTH_T_TOKEN = 12   /* token activations [H] */
};

#define SYNTH_GOLDEN 0x9E3779B97F4A7C15ULL

SYNTH_FN uint64_t synth_mix(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

/* Key of the stream for (seed, layer, tensor, item). */
SYNTH_FN uint64_t synth_key(uint64_t seed, uint32_t layer, uint32_t tensor, uint32_t item) {
  uint64_t k = synth_mix(seed + SYNTH_GOLDEN);
  k = synth_mix(k ^ (((uint64_t)layer << 32) | (uint64_t)tensor));
  k = synth_mix(k ^ ((uint64_t)item * SYNTH_GOLDEN + 0x632BE59BD9B4E019ULL));
  return k;
}

SYNTH_FN uint64_t synth_draw(uint64_t key, uint64_t i) {
  return synth_mix(key + (i + 1) * SYNTH_GOLDEN);
}

/* Round a double to bf16, round-to-nearest-even, integer arithmetic only. */
SYNTH_FN uint16_t synth_double_to_bf16(double v) {
  union { double d; uint64_t u; } cv;
  cv.d = v;
  uint64_t b = cv.u;
  uint16_t sign = (uint16_t)((b >> 63) << 15);
  int e = (int)((b >> 52) & 0x7FF);
  uint64_t m = b & ((1ULL << 52) - 1);
  if (e == 0x7FF) return (uint16_t)(sign | 0x7F80 | (m ? 0x40 : 0));
  if (e == 0) return sign; /* zero or double subnormal: far below bf16 range */
  int E = e - 1023;
  uint64_t M = (1ULL << 52) | m; /* 53 significant bits */
  int shift;
  int biased;
  if (E >= -126) {
    shift = 45; /* keep 8 significant bits */
    biased = E + 127;
  } else {
    shift = 45 + (-126 - E);
    biased = 0;
    if (shift > 60) return sign;
  }
  uint64_t q = M >> shift;
  uint64_t rem = M & ((1ULL << shift) - 1);
  uint64_t half = 1ULL << (shift - 1);
  if (rem > half || (rem == half && (q & 1))) q++;
  if (biased == 0) {
    /* subnormal: q holds the mantissa; q == 128 became the smallest normal */
    return (uint16_t)(sign | (uint16_t)q);
  }
  if (q == 256) { q = 128; biased++; }
  if (biased >= 255) return (uint16_t)(sign | 0x7F80);
  return (uint16_t)(sign | (uint16_t)(biased << 7) | (uint16_t)(q & 0x7F));
}

/* Uniform double in [0,1) with 53 random bits. */
SYNTH_FN double synth_unit(uint64_t r) { return (double)(r >> 11) * 0x1p-53; }

/* bf16 value drawn uniformly from [lo, hi). */
SYNTH_FN uint16_t synth_uniform_bf16(uint64_t r, double lo, double hi) {
  double d = SYNTH_DADD(hi, -lo);
  return synth_double_to_bf16(SYNTH_DADD(lo, SYNTH_DMUL(d, synth_unit(r))));
}

/* Approximately normal value: Irwin-Hall sum of eight 16-bit uniforms from two
 * draws, centred and scaled to unit variance (1/sqrt(8*(65536^2-1)/12) below),
 * then mean + std * n, rounded to bf16.  Support is +-4.9 standard deviations. */
#define SYNTH_IH8_INV_STD 1.8688123650118534e-05
SYNTH_FN uint16_t synth_normal_bf16(uint64_t r0, uint64_t r1, double mean, double std) {
  int64_t s = 0;
  for (int j = 0; j < 4; ++j) {
    s += (int64_t)((r0 >> (16 * j)) & 0xFFFF);
    s += (int64_t)((r1 >> (16 * j)) & 0xFFFF);
  }
  double n = SYNTH_DMUL((double)(s - 262140), SYNTH_IH8_INV_STD);
  return synth_double_to_bf16(SYNTH_DADD(mean, SYNTH_DMUL(std, n)));
}

/* ---------------------------------------------------------------------------
 * Canonical expert blob.  For each matrix m in order gate [I][H], up [I][H],
 * down [H][I] (rows x columns):
 *   codes  : R*C*bits/8 bytes, row-major, 32/bits codes per little-endian
 *            uint32; element c of a row sits at bit bits*(c % (32/bits)) of
 *            word c / (32/bits) of that row;
 *   scales : bf16 [R][C/64];
 *   biases : bf16 [R][C/64].
 * Group size is 64 along the input (column) dimension.
 * ------------------------------------------------------------------------- */
typedef struct synth_expert_params {
  uint64_t seed;
  int32_t layer;
  int32_t hidden;
  int32_t inter;
  int32_t bits;
  double scale_lo, scale_hi;
  double bias_lo, bias_hi;
} synth_expert_params;

SYNTH_FN void synth_matrix_shape(const synth_expert_params* p, int m, int64_t* R, int64_t* C) {
  if (m < 2) { *R = p->inter; *C = p->hidden; }
  else { *R = p->hidden; *C = p->inter; }
}

SYNTH_FN int64_t synth_matrix_bytes(const synth_expert_params* p, int m) {
  int64_t R, C;
  synth_matrix_shape(p, m, &R, &C);
  return R * C * p->bits / 8 + 4 * (R * C / 64);
}

SYNTH_FN int64_t synth_blob_bytes(const synth_expert_params* p) {
  return synth_matrix_bytes(p, 0) + synth_matrix_bytes(p, 1) + synth_matrix_bytes(p, 2);
}

/* The 64-bit little-endian word at byte offset 8*w of expert `expert`'s blob. */
SYNTH_FN uint64_t synth_blob_word(const synth_expert_params* p, int expert, int64_t w) {
  int64_t off = w * 8;
  for (int m = 0; m < 3; ++m) {
    int64_t R, C;
    synth_matrix_shape(p, m, &R, &C);
    int64_t cb = R * C * p->bits / 8;
    int64_t nsb = R * C / 64;
    if (off < cb) {
      uint64_t key = synth_key(p->seed, (uint32_t)p->layer, SYNTH_T_CODES + m, (uint32_t)expert);
      return synth_draw(key, (uint64_t)(off / 8));
    }
    off -= cb;
    if (off < 4 * nsb) {
      int is_bias = off >= 2 * nsb;
      int64_t first = (is_bias ? off - 2 * nsb : off) / 2; /* index of first bf16 */
      uint64_t key = synth_key(p->seed, (uint32_t)p->layer,
                               (is_bias ? SYNTH_T_BIAS : SYNTH_T_SCALE) + m, (uint32_t)expert);
      double lo = is_bias ? p->bias_lo : p->scale_lo;
      double hi = is_bias ? p->bias_hi : p->scale_hi;
      uint64_t out = 0;
      for (int j = 0; j < 4; ++j) {
        uint64_t v = synth_uniform_bf16(synth_draw(key, (uint64_t)(first + j)), lo, hi);
        out |= v << (16 * j);
      }
      return out;
    }
    off -= 4 * nsb;
  }
  return 0;
}

/* Element i of a normally distributed bf16 tensor with stream key `key`. */
SYNTH_FN uint16_t synth_normal_elem(uint64_t key, int64_t i, double mean, double std) {
  return synth_normal_bf16(synth_draw(key, (uint64_t)(2 * i)), synth_draw(key, (uint64_t)(2 * i + 1)),
                           mean, std);
}

#endif /* SYNTH_CORE_H */
