// fmoe_requant.cu -- 4-bit -> 2-bit requantisation of canonical expert blobs,
// the conversion the page "Flash-MoE Inference Engine", section "Weight
// Preparation" (step 3, optional 2-bit requantisation) runs as an offline
// script; the page gives no algorithm.  Per 64-column group of every row:
//   w    = fma(q4, s4, b4)                 s4, b4: the group's bf16 scale, bias
//   lo   = min w, hi = max w               (in column order, strict comparisons)
//   s2   = bf16((hi - lo) / 3), b2 = bf16(lo)
//   inv  = s2 > 0 ? 1 / s2 : 0
//   q2   = min(max(rint((w - b2) * inv), 0), 3)
// each step one IEEE fp32 operation rounded to nearest even, so the integer
// codes are decided by exactly the arithmetic the definition states.
//
// One thread per (matrix row, group): 32 bytes of 4-bit codes in (two 16-byte
// loads), 16 bytes of 2-bit codes out; consecutive threads take consecutive
// groups of a row, so a warp reads 1 KB and writes 512 B contiguously.  The
// weights are recomputed for the second pass instead of being held.  About 16
// fp32/integer operations per weight: at the full shape the kernel is bound by
// issue, ~3x above its HBM time, which is fine for a one-off conversion.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "fmoe_internal.h"

namespace fmoe {
namespace {

__device__ __forceinline__ float bf16f(uint16_t v) { return __uint_as_float((uint32_t)v << 16); }
__device__ __forceinline__ uint16_t to_bf16(float f) { return __bfloat16_as_ushort(__float2bfloat16_rn(f)); }

__global__ void requant_kernel(const uint8_t* __restrict__ src, uint8_t* __restrict__ dst, int H, int I,
                               int64_t n_groups) {
  const int64_t per_m = (int64_t)H * I / kGroup;              // groups per matrix
  const int64_t mat4 = (int64_t)H * I / 2 + (int64_t)H * I / 16;  // bytes of a 4-bit matrix (codes, scales, biases)
  const int64_t mat2 = (int64_t)H * I / 4 + (int64_t)H * I / 16;
  for (int64_t gi = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; gi < n_groups;
       gi += (int64_t)gridDim.x * blockDim.x) {
    const int64_t blob = gi / (3 * per_m), rem3 = gi % (3 * per_m);
    const int m = (int)(rem3 / per_m);
    const int64_t rem = rem3 % per_m;
    const int C = m < 2 ? H : I, R = m < 2 ? I : H, ng = C / kGroup;
    const int64_t r = rem / ng, g = rem % ng;
    const uint8_t* in = src + (blob * 3 + m) * mat4;
    uint8_t* out = dst + (blob * 3 + m) * mat2;
    const uint4* cp = reinterpret_cast<const uint4*>(in + r * (C / 2) + 32 * g);
    const uint4 c0 = cp[0], c1 = cp[1];
    const int64_t sb = r * ng + g;
    const float s4 = bf16f(*reinterpret_cast<const uint16_t*>(in + (int64_t)R * C / 2 + 2 * sb));
    const float b4 = bf16f(*reinterpret_cast<const uint16_t*>(in + (int64_t)R * C / 2 + 2 * (int64_t)R * ng + 2 * sb));
    const uint32_t wd[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
    // pass 1: smallest and largest weight, in column order
    float lo = 0.f, hi = 0.f;
#pragma unroll
    for (int c = 0; c < kGroup; ++c) {
      const float w = __fmaf_rn((float)((wd[c / 8] >> (4 * (c % 8))) & 15u), s4, b4);
      if (c == 0) {
        lo = w;
        hi = w;
      } else {
        if (w < lo) lo = w;
        if (w > hi) hi = w;
      }
    }
    const uint16_t s2b = to_bf16(__fdiv_rn(__fsub_rn(hi, lo), 3.0f));
    const uint16_t b2b = to_bf16(lo);
    const float s2 = bf16f(s2b), b2 = bf16f(b2b);
    const float inv = s2 > 0.f ? __fdiv_rn(1.0f, s2) : 0.f;
    // pass 2: codes, 16 per output word
    uint32_t o[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      uint32_t word = 0;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int c = 16 * k + j;
        const float w = __fmaf_rn((float)((wd[c / 8] >> (4 * (c % 8))) & 15u), s4, b4);
        const float q = fminf(fmaxf(rintf(__fmul_rn(__fsub_rn(w, b2), inv)), 0.f), 3.f);
        word |= (uint32_t)q << (2 * j);
      }
      o[k] = word;
    }
    *reinterpret_cast<uint4*>(out + r * (C / 4) + 16 * g) = make_uint4(o[0], o[1], o[2], o[3]);
    *reinterpret_cast<uint16_t*>(out + (int64_t)R * C / 4 + 2 * sb) = s2b;
    *reinterpret_cast<uint16_t*>(out + (int64_t)R * C / 4 + 2 * (int64_t)R * ng + 2 * sb) = b2b;
  }
}

}  // namespace

int launch_requant(const uint8_t* src, uint8_t* dst, int n_blobs, int H, int I, int n_sm, void* stream) {
  const int64_t n_groups = (int64_t)n_blobs * 3 * H * I / kGroup;
  if (n_groups == 0) return 0;
  const int64_t blocks = (n_groups + 255) / 256;
  const int grid = (int)(blocks < 16LL * n_sm ? blocks : 16LL * n_sm);
  requant_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(src, dst, H, I, n_groups);
  return (int)cudaGetLastError();
}

}  // namespace fmoe
