/*
 * synth_cuda.cu -- device side of the seeded synthetic input generator (see
 * synth_core.h).  It fills device buffers with exactly the bytes the host
 * generator produces, so that full-size weight sets (tens of GB) never have to
 * be built on the host.  Test and benchmark infrastructure only; it holds no
 * mixture-of-experts arithmetic.
 */
#include <cuda_runtime.h>

#include "synth_core.h"

namespace {

__global__ void gen_experts_kernel(synth_expert_params p, int expert_begin, int64_t words_per_blob,
                                   int64_t total, uint64_t* __restrict__ out) {
  int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += stride) {
    int e = expert_begin + (int)(i / words_per_blob);
    out[i] = synth_blob_word(&p, e, i % words_per_blob);
  }
}

__global__ void gen_normal_kernel(uint64_t key, int64_t n, double mean, double std, uint16_t* __restrict__ out) {
  int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
    out[i] = synth_normal_elem(key, i, mean, std);
}

// Rows r = 0..rows-1 of length n: row r is stream (seed, layer, tensor, item0 + r).
__global__ void gen_normal_rows_kernel(uint64_t seed, uint32_t layer, uint32_t tensor, uint32_t item0, int rows,
                                       int64_t n, double mean, double std, uint16_t* __restrict__ out) {
  const int64_t total = (int64_t)rows * n, stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += stride) {
    const int r = (int)(i / n);
    out[i] = synth_normal_elem(synth_key(seed, layer, tensor, item0 + (uint32_t)r), i % n, mean, std);
  }
}

int grid_for(int64_t n) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t want = (n + 255) / 256;
  int64_t cap = (int64_t)sms * 8;
  return (int)(want < cap ? (want < 1 ? 1 : want) : cap);
}

}  // namespace

extern "C" {

/* Fills dst (device, 8-byte aligned) with `count` expert blobs, experts
 * expert_begin.., asynchronously on `stream`.  Returns a cudaError_t value. */
int synth_cuda_gen_experts(const synth_expert_params* p, int expert_begin, int count, void* dst, void* stream) {
  int64_t words = synth_blob_bytes(p) / 8;
  int64_t total = words * (int64_t)count;
  if (total <= 0) return 0;
  gen_experts_kernel<<<grid_for(total), 256, 0, (cudaStream_t)stream>>>(*p, expert_begin, words, total,
                                                                        (uint64_t*)dst);
  return (int)cudaGetLastError();
}

/* Fills dst (device) with n normal bf16 values of stream (seed, layer, tensor, item). */
int synth_cuda_gen_normal_bf16(uint64_t seed, uint32_t layer, uint32_t tensor, uint32_t item, int64_t n,
                               double mean, double std, void* dst, void* stream) {
  if (n <= 0) return 0;
  uint64_t key = synth_key(seed, layer, tensor, item);
  gen_normal_kernel<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>(key, n, mean, std, (uint16_t*)dst);
  return (int)cudaGetLastError();
}

/* Fills dst (device) with `rows` consecutive rows of n normal bf16 values; row r
 * is the stream (seed, layer, tensor, item0 + r), identical to the single-row call. */
int synth_cuda_gen_normal_rows_bf16(uint64_t seed, uint32_t layer, uint32_t tensor, uint32_t item0, int rows,
                                    int64_t n, double mean, double std, void* dst, void* stream) {
  if (n <= 0 || rows <= 0) return 0;
  gen_normal_rows_kernel<<<grid_for((int64_t)rows * n), 256, 0, (cudaStream_t)stream>>>(seed, layer, tensor, item0,
                                                                                     rows, n, mean, std,
                                                                                     (uint16_t*)dst);
  return (int)cudaGetLastError();
}

}  // extern "C"
