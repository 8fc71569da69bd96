// fmoe_static.cu -- router step (fmoe_route_static) whose scratch lives in a
// fixed device array instead of the context workspace.
//
// Some callers must not allocate device memory per call: a serving loop whose
// device memory is entirely held by its own pool allocator (a cudaMalloc would
// fail or fragment that pool), and latency-critical loops that cannot afford
// cudaFree's implicit device-wide synchronisation.  This variant of the route
// step allocates nothing: its only scratch, the fp32 logits [T][E], is the
// file-scope array below (128 KB, so T * E <= kStaticRouteLogits), whose
// address is looked up once per device.  Every logit is written by the first
// kernel before the second reads it, so nothing has to start at zero.  Calls
// that overlap in time (two streams, or two host threads) share the array and
// race; callers must order them.
//
// Two launches on the caller's stream: (1) logits, one warp per expert row and
// token, with z = RMSNorm(x) formed on the fly when the layer has a norm weight;
// (2) top-K and renormalised weights, one warp per token.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <mutex>

#include "fmoe_internal.h"

namespace fmoe {
namespace {

__device__ __align__(256) float g_route_logits[kStaticRouteLogits];

__device__ __forceinline__ float lo16(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float hi16(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }
__device__ __forceinline__ float round_bf16(float f) { return __bfloat162float(__float2bfloat16_rn(f)); }

constexpr int kWarps = 8;

// Grid-stride over expert rows: warp w of block b takes rows b*kWarps + w, ...
// Shared memory: the per-token RMSNorm factor (T floats).
__global__ void __launch_bounds__(kWarps * 32) static_logits_kernel(const uint16_t* __restrict__ wr,
                                                                     const float* __restrict__ bias,
                                                                     const uint16_t* __restrict__ norm_w, float eps,
                                                                     const uint16_t* __restrict__ x, int T, int H,
                                                                     int E, float* __restrict__ logits) {
  extern __shared__ float s_rms[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (norm_w != nullptr) {
    for (int t = warp; t < T; t += kWarps) {
      const uint4* xr = reinterpret_cast<const uint4*>(x + (size_t)t * H);
      float ss = 0.f;
      for (int c = lane; c < H / 8; c += 32) {
        const uint4 v = xr[c];
        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) ss += lo16(w4[k]) * lo16(w4[k]) + hi16(w4[k]) * hi16(w4[k]);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      if (lane == 0) s_rms[t] = 1.0f / sqrtf(ss / (float)H + eps);
    }
  }
  __syncthreads();
  for (int e = blockIdx.x * kWarps + warp; e < E; e += gridDim.x * kWarps) {
    const uint4* wrow = reinterpret_cast<const uint4*>(wr + (size_t)e * H);
    for (int t = 0; t < T; ++t) {
      const uint4* xr = reinterpret_cast<const uint4*>(x + (size_t)t * H);
      const uint4* nw = reinterpret_cast<const uint4*>(norm_w);
      const float r = norm_w != nullptr ? s_rms[t] : 1.f;
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      for (int c = lane; c < H / 8; c += 32) {
        const uint4 wv = wrow[c], xv = xr[c];
        const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w}, xx[4] = {xv.x, xv.y, xv.z, xv.w};
        uint32_t nn[4] = {0u, 0u, 0u, 0u};
        if (norm_w != nullptr) {
          const uint4 n4 = nw[c];
          nn[0] = n4.x; nn[1] = n4.y; nn[2] = n4.z; nn[3] = n4.w;
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          float zl = lo16(xx[k]), zh = hi16(xx[k]);
          if (norm_w != nullptr) {
            zl = round_bf16(zl * r * lo16(nn[k]));
            zh = round_bf16(zh * r * hi16(nn[k]));
          }
          acc[k] = fmaf(lo16(ww[k]), zl, acc[k]);
          acc[k] = fmaf(hi16(ww[k]), zh, acc[k]);
        }
      }
      float s = (acc[0] + acc[1]) + (acc[2] + acc[3]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (lane == 0) logits[(size_t)t * E + e] = s + (bias != nullptr ? bias[e] : 0.f);
    }
  }
}

// Router order as a 64-bit key: larger logit first (NaN counts as -inf, -0 as
// +0), then lower index.
__device__ __forceinline__ uint64_t order_key(float v, int i) {
  if (v != v) v = -INFINITY;
  const uint32_t u = (v == 0.f) ? 0u : __float_as_uint(v);
  const uint32_t k = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return ((uint64_t)k << 32) | (uint32_t)~i;
}
__device__ __forceinline__ float key_logit(uint64_t key) {
  const uint32_t k = (uint32_t)(key >> 32);
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}
__device__ __forceinline__ uint64_t warp_max_u64(uint64_t v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const uint64_t other = __shfl_xor_sync(0xffffffffu, v, o);
    v = other > v ? other : v;
  }
  return v;
}

__global__ void __launch_bounds__(kWarps * 32) static_topk_kernel(const float* __restrict__ logits, int T, int E,
                                                                   int K, int32_t* __restrict__ idx_out,
                                                                   float* __restrict__ w_out) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * kWarps + warp;
  if (t >= T) return;
  const float* row = logits + (size_t)t * E;
  uint64_t prev = ~0ull;
  float my_logit = -INFINITY;
  int my_idx = 0;
  for (int k = 0; k < K; ++k) {
    uint64_t best = 0ull;
    for (int i = lane; i < E; i += 32) {
      const uint64_t key = order_key(row[i], i);
      if (key < prev && key > best) best = key;
    }
    prev = warp_max_u64(best);
    if (lane == k && prev != 0ull) {
      my_logit = key_logit(prev);
      my_idx = (int)~(uint32_t)prev;
    }
  }
  // renormalised weights over the K picks: exp(l_k - l_0) / sum_j exp(l_j - l_0); an infinite
  // largest logit takes the softmax's limit (equal shares for the picks equal to it)
  const float top0 = __shfl_sync(0xffffffffu, my_logit, 0);
  const float ex = lane >= K ? 0.f : fabsf(top0) != INFINITY ? expf(my_logit - top0) : (my_logit == top0 ? 1.f : 0.f);
  float den = ex;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
  if (lane < K) {
    idx_out[(size_t)t * K + lane] = my_idx;
    w_out[(size_t)t * K + lane] = ex / den;
  }
}

std::mutex g_symbol_mu;
float* g_symbol_addr[kMaxDevices] = {};

}  // namespace

int launch_topk_rows(const float* logits, int T, int E, int K, int32_t* idx_out, float* w_out, void* stream) {
  static_topk_kernel<<<(T + kWarps - 1) / kWarps, kWarps * 32, 0, static_cast<cudaStream_t>(stream)>>>(logits, T, E, K,
                                                                                                  idx_out, w_out);
  return (int)cudaGetLastError();
}

// Looks up the fixed scratch's address on the current device (once per
// device).  fmoe_create calls it, so no later call has to, which matters
// inside a stream capture, where the lookup may load the module.
int route_static_prepare() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return (int)e;
  if (dev < 0 || dev >= kMaxDevices) return (int)cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> g(g_symbol_mu);
  if (g_symbol_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_route_logits);
    if (e != cudaSuccess) return (int)e;
    g_symbol_addr[dev] = static_cast<float*>(p);
  }
  return 0;
}

bool route_static_ready() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  std::lock_guard<std::mutex> g(g_symbol_mu);
  return g_symbol_addr[dev] != nullptr;
}

int launch_route_static(const uint16_t* wr, const float* bias, const uint16_t* norm_w, float eps,
                        const uint16_t* x, int T, int H, int E, int K, int32_t* idx_out, float* w_out, void* stream) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return (int)e;
  if (dev < 0 || dev >= kMaxDevices) return (int)cudaErrorInvalidDevice;
  const int rc = route_static_prepare();
  if (rc != 0) return rc;
  float* scratch = nullptr;
  {
    std::lock_guard<std::mutex> g(g_symbol_mu);
    scratch = g_symbol_addr[dev];
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int blocks = (E + kWarps - 1) / kWarps;
  static_logits_kernel<<<blocks, kWarps * 32, (size_t)T * sizeof(float), st>>>(wr, bias, norm_w, eps, x, T, H, E,
                                                                                scratch);
  e = cudaGetLastError();
  if (e != cudaSuccess) return (int)e;
  static_topk_kernel<<<(T + kWarps - 1) / kWarps, kWarps * 32, 0, st>>>(scratch, T, E, K, idx_out, w_out);
  return (int)cudaGetLastError();
}

}  // namespace fmoe
