// fmoe_batched.cu -- the mixture-of-experts layer for T tokens at once.
//
// With many tokens per step the expert matrices become real contractions: an
// expert chosen by n tokens multiplies an [rows x K] weight matrix by an
// [K x n] block of token vectors.  The batch-1 kernel (fmoe_decode.cu) reads
// every expert once per token; here each selected expert is read once per 64
// of its tokens.  The steps, all on the caller's stream:
//   norm     z = RMSNorm(h) (or h), bf16
//   router   logits = W_r z (+ bias), bf16 tensor-core GEMM, fp32 accumulate
//   top-K    per token (launch_topk_rows)
//   permute  (token, slot) pairs grouped by expert into segments; the shared
//            expert's segment holds every token; a list of GEMM work items
//   prep     per position: its token's z as fp16, scaled by a power of two so
//            the row's largest magnitude lies in [2^14, 2^15), columns in the
//            order the tensor-core A operand uses
//   gate/up  grouped tcgen05 GEMM (fmoe_grouped_tc.cu): a work item is 128 rows
//            (8 units of 8 gate + 8 up rows) x up to 64 positions of one expert;
//            a = silu(g)*u written per position
//   prep     of a, per position
//   down     grouped tcgen05 GEMM, 128 output rows x up to 64 positions
//   combine  out = h + y_shared + sum_k w_k y_k, fp32, one bf16 rounding
#include <cuda_bf16.h>
#include <algorithm>
#include <type_traits>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "fmoe_internal.h"

namespace fmoe {
namespace {

__device__ __forceinline__ float bflo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bfhi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }
__device__ __forceinline__ uint16_t to_bf16(float f) { return __bfloat16_as_ushort(__float2bfloat16_rn(f)); }
__device__ __forceinline__ float pow2(int k) { return __uint_as_float((uint32_t)(k + 127) << 23); }
__device__ __forceinline__ uint32_t smem_addr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mma_bf16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// 16-byte async copy global -> shared; src_bytes 0 fills zeros.
__device__ __forceinline__ void cp_async16(void* dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_addr(dst)), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// ------------------------------------------------------------------ norm
// One warp per token: z = bf16(h * r * w), r = 1/sqrt(mean(h^2) + eps); a
// copy of h when there is no norm weight.
__global__ void bt_norm_kernel(const uint16_t* __restrict__ h, const uint16_t* __restrict__ norm_w, float eps, int T,
                               int H, uint16_t* __restrict__ z) {
  const int lane = threadIdx.x & 31;
  for (int t = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5); t < T; t += gridDim.x * (blockDim.x / 32)) {
    const uint4* hr = reinterpret_cast<const uint4*>(h + (size_t)t * H);
    uint4* zr = reinterpret_cast<uint4*>(z + (size_t)t * H);
    if (norm_w == nullptr) {
      for (int c = lane; c < H / 8; c += 32) zr[c] = hr[c];
      continue;
    }
    float ss = 0.f;
    for (int c = lane; c < H / 8; c += 32) {
      const uint4 v = hr[c];
      const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) ss = fmaf(bflo(w4[k]), bflo(w4[k]), fmaf(bfhi(w4[k]), bfhi(w4[k]), ss));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float r = 1.0f / sqrtf(ss / (float)H + eps);
    const uint4* nw = reinterpret_cast<const uint4*>(norm_w);
    for (int c = lane; c < H / 8; c += 32) {
      const uint4 v = hr[c], n = nw[c];
      const uint32_t h4[4] = {v.x, v.y, v.z, v.w}, n4[4] = {n.x, n.y, n.z, n.w};
      uint32_t o4[4];
#pragma unroll
      for (int k = 0; k < 4; ++k)
        o4[k] = (uint32_t)to_bf16(bflo(h4[k]) * r * bflo(n4[k])) |
                ((uint32_t)to_bf16(bfhi(h4[k]) * r * bfhi(n4[k])) << 16);
      zr[c] = make_uint4(o4[0], o4[1], o4[2], o4[3]);
    }
  }
}

// ------------------------------------------------------------------ prep
// Element p of every 16 columns of a GEMM input row holds source column pi(p):
// the order in which the tensor-core A operand holds the weights (the 16x256b
// tensor-memory store of an mma.sync-ordered fragment; fmoe_grouped_tc.cu).
__host__ __device__ constexpr int k_perm(int p) { return 2 * (p >> 2) + (p & 1) + 8 * ((p >> 1) & 1); }

__device__ __forceinline__ void load16(const uint16_t* src, float (&v)[16]) {
  const uint4 a = *reinterpret_cast<const uint4*>(src), b = *reinterpret_cast<const uint4*>(src + 8);
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    v[2 * k] = bflo(w[k]);
    v[2 * k + 1] = bfhi(w[k]);
  }
}
__device__ __forceinline__ void load16(const float* src, float (&v)[16]) {
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float4 f = reinterpret_cast<const float4*>(src)[k];
    v[4 * k] = f.x;
    v[4 * k + 1] = f.y;
    v[4 * k + 2] = f.z;
    v[4 * k + 3] = f.w;
  }
}

// One warp per position p: dst[p] = fp16(src[row(p)] * 2^sh) in k_perm order,
// with sh putting the row's largest magnitude in [2^14, 2^15) (any finite row
// fits fp16; bf16 inputs convert exactly unless they are 2^28 times smaller
// than the row's largest), and scale[p] = 2^-sh.  row(p) = rowmap[p], or p.
// sums[(g / 2) * pcap + p][g % 2] = the fp32 sum of the fp16 values of 64-column
// group g of dst[p] (the grouped GEMM's bias term).
template <typename Src>
__global__ void bt_prep_kernel(const Src* __restrict__ src, const int32_t* __restrict__ rowmap, int P, int K,
                               uint16_t* __restrict__ dst, float* __restrict__ scale, float* __restrict__ sums,
                               int pcap) {
  const int lane = threadIdx.x & 31, nb = K / 16;
  for (int p = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5); p < P; p += gridDim.x * (blockDim.x / 32)) {
    const Src* row = src + (size_t)(rowmap ? rowmap[p] : p) * K;
    uint32_t m = 0;
    for (int b = lane; b < nb; b += 32) {
      float v[16];
      load16(row + 16 * b, v);
#pragma unroll
      for (int k = 0; k < 16; ++k) m = max(m, __float_as_uint(fabsf(v[k])));
    }
    m = __reduce_max_sync(0xffffffffu, m);
    const int e = (int)((m >> 23) & 0xFF) - 127;
    const int sh = m == 0 ? 0 : min(14 - max(e, -126), 126);
    const float mul = pow2(sh);
    if (lane == 0) scale[p] = pow2(-sh);
    uint16_t* drow = dst + (size_t)p * K;
    // K is a multiple of 64, so the four 16-column blocks of a group are four
    // consecutive lanes of one pass
    for (int b0 = 0; b0 < nb; b0 += 32) {
      const int b = b0 + lane;
      float gsum = 0.f;
      if (b < nb) {
        float v[16];
        load16(row + 16 * b, v);
        uint32_t o[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const __half2 h = __floats2half2_rn(v[k_perm(2 * k)] * mul, v[k_perm(2 * k + 1)] * mul);
          o[k] = *reinterpret_cast<const uint32_t*>(&h);
          const float2 f = __half22float2(h);
          gsum += f.x + f.y;
        }
        reinterpret_cast<uint4*>(drow + 16 * b)[0] = make_uint4(o[0], o[1], o[2], o[3]);
        reinterpret_cast<uint4*>(drow + 16 * b)[1] = make_uint4(o[4], o[5], o[6], o[7]);
      }
      gsum += __shfl_xor_sync(0xffffffffu, gsum, 1);
      gsum += __shfl_xor_sync(0xffffffffu, gsum, 2);
      if (b < nb && (b & 3) == 0) {
        const int g = b >> 2;
        sums[((size_t)(g >> 1) * pcap + p) * 4 + (g & 1)] = gsum;
      }
    }
  }
}

// ------------------------------------------------------------------ router
// logits[t][e] = sum_h W_r[e][h] z[t][h] (+ bias[e]), bf16 mma.sync with fp32
// accumulation.  A block computes 64 experts x 64 tokens: 64-column chunks of
// both operands are staged in shared memory by cp.async (3 stages, rows padded
// to 36 words so fragment reads are conflict-free); warp (we, wt) owns experts
// 16*we.. and tokens 32*wt.. (4 blocks of 8).
constexpr int kRtRows = 64, kRtStages = 4, kRtRowWords = 36, kRtSplit = 8;
constexpr int kRtStage = 2 * kRtRows * kRtRowWords * 4;
__global__ void __launch_bounds__(256) bt_router_kernel(const uint16_t* __restrict__ wr, const uint16_t* __restrict__ z,
                                                        int T, int E, int H, float* __restrict__ part) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
  const int we = warp & 3, wt = warp >> 2;
  const int e0 = blockIdx.x * kRtRows, t0 = blockIdx.y * kRtRows;
  // K split: block z covers chunks [ch0, ch0 + nch) of the hidden dimension
  const int per = (H / kGroup + kRtSplit - 1) / kRtSplit;
  const int ch0 = blockIdx.z * per, nch = max(0, min(per, H / kGroup - ch0));
  auto load = [&](int ch, int st) {
    uint8_t* sa = smem + st * kRtStage;
    uint8_t* sb = sa + kRtRows * kRtRowWords * 4;
    for (int c = tid; c < 2 * kRtRows * 8; c += 256) {
      const bool is_b = c >= kRtRows * 8;
      const int r = (c % (kRtRows * 8)) / 8, part = c % 8;
      const int row = (is_b ? t0 : e0) + r;
      const bool ok = row < (is_b ? T : E);
      const uint16_t* src = (is_b ? z : wr) + (size_t)(ok ? row : 0) * H + (size_t)(ch0 + ch) * kGroup + part * 8;
      cp_async16((is_b ? sb : sa) + r * kRtRowWords * 4 + part * 16, src, ok ? 16u : 0u);
    }
  };
  float c[4][4] = {};
#pragma unroll
  for (int st = 0; st < kRtStages - 1; ++st) {
    if (st < nch) load(st, st);
    cp_async_commit();
  }
  for (int ch = 0; ch < nch; ++ch) {
    cp_async_wait<kRtStages - 2>();
    __syncthreads();
    if (ch + kRtStages - 1 < nch) load(ch + kRtStages - 1, (ch + kRtStages - 1) % kRtStages);
    cp_async_commit();
    const uint32_t* sa = reinterpret_cast<const uint32_t*>(smem + (ch % kRtStages) * kRtStage);
    const uint32_t* sb = sa + kRtRows * kRtRowWords;
#pragma unroll
    for (int sl = 0; sl < 4; ++sl) {
      const uint32_t* ar = sa + (16 * we + g) * kRtRowWords + 8 * sl + t;
      const uint32_t a0 = ar[0], a1 = ar[8 * kRtRowWords], a2 = ar[4], a3 = ar[8 * kRtRowWords + 4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t* br = sb + (32 * wt + 8 * j + g) * kRtRowWords + 8 * sl + t;
        mma_bf16(c[j], a0, a1, a2, a3, br[0], br[4]);
      }
    }
  }
  cp_async_wait<0>();
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int ta = t0 + 32 * wt + 8 * j + 2 * t;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int e = e0 + 16 * we + g + ((q & 2) ? 8 : 0), tok = ta + (q & 1);
      if (e < E && tok < T) part[((size_t)blockIdx.z * T + tok) * E + e] = c[j][q];
    }
  }
}

// logits = the K-split partials summed in split order, plus the bias.
__global__ void bt_logits_sum_kernel(const float* __restrict__ part, const float* __restrict__ bias, int T, int E,
                                     float* __restrict__ logits) {
  const int64_t n = (int64_t)T * E;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    float acc = part[i];
    for (int k = 1; k < kRtSplit; ++k) acc += part[(size_t)k * n + i];
    logits[i] = acc + (bias != nullptr ? bias[i % E] : 0.f);
  }
}

// ------------------------------------------------------------------ permute
struct PermuteArgs {
  const int32_t* idx;  // [T][K]
  int T, E, K, single_expert;
  int rows_gu, rows_dn;  // matrix rows of gate/up (2I) and down (H)
  int32_t* seg;          // [4][E+1] + n_seg
  int32_t* cursor;       // [E+1]
  int32_t* pos_tok;
  int32_t* pos_of;
  uint32_t* items_gu;
  uint32_t* items_dn;
  int32_t* n_items;
  int max_items_gu, max_items_dn;
  int32_t* small_seg;    // [E+1]
  int bands_gu, bands_dn;  // 16-row bands of gate/up (2I/16) and down (H/16)
};

// Block-wide exclusive scan of three counters per thread (blockDim 1024);
// returns the prefixes and writes the totals to tot[0..2].
__device__ __forceinline__ int3 block_scan3(int3 v, int32_t* scratch, int32_t* tot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int3 inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int x = __shfl_up_sync(0xffffffffu, inc.x, o), y = __shfl_up_sync(0xffffffffu, inc.y, o),
              z = __shfl_up_sync(0xffffffffu, inc.z, o);
    if (lane >= o) {
      inc.x += x;
      inc.y += y;
      inc.z += z;
    }
  }
  if (lane == 31) {
    scratch[3 * warp] = inc.x;
    scratch[3 * warp + 1] = inc.y;
    scratch[3 * warp + 2] = inc.z;
  }
  __syncthreads();
  if (warp == 0) {
    int3 w = lane < nw ? make_int3(scratch[3 * lane], scratch[3 * lane + 1], scratch[3 * lane + 2]) : make_int3(0, 0, 0);
    int3 wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int x = __shfl_up_sync(0xffffffffu, wi.x, o), y = __shfl_up_sync(0xffffffffu, wi.y, o),
                z = __shfl_up_sync(0xffffffffu, wi.z, o);
      if (lane >= o) {
        wi.x += x;
        wi.y += y;
        wi.z += z;
      }
    }
    if (lane < nw) {
      scratch[3 * lane] = wi.x - w.x;
      scratch[3 * lane + 1] = wi.y - w.y;
      scratch[3 * lane + 2] = wi.z - w.z;
    }
    if (lane == nw - 1) {
      tot[0] = wi.x;
      tot[1] = wi.y;
      tot[2] = wi.z;
    }
  }
  __syncthreads();
  return make_int3(scratch[3 * warp] + inc.x - v.x, scratch[3 * warp + 1] + inc.y - v.y,
                   scratch[3 * warp + 2] + inc.z - v.z);
}

// One block of 1024 threads (E + 1 <= 1024).  Counts per expert (lanes that
// hold the same expert add once), one scan for segment starts, segment numbers
// and work-item offsets, a scatter of the T*K routed pairs (positions within an
// expert follow the atomics, so their order varies, but every position is
// computed independently: the results do not depend on it), the shared
// expert's segment after them, and the GEMM work items of every non-empty
// segment in expert order.
__global__ void __launch_bounds__(1024) bt_permute_kernel(PermuteArgs p) {
  extern __shared__ int32_t sh[];
  const int S = p.E + 1;  // segment candidates: experts 0..E-1, then the shared one
  int32_t* cnt = sh;
  int32_t* cur = sh + S;          // scatter cursors
  int32_t* scratch = sh + 2 * S;  // [3 * 32] scan scratch
  int32_t* tot = scratch + 96;    // [3] totals
  const int tid = threadIdx.x, lane = tid & 31;
  int32_t* seg_e = p.seg;
  int32_t* seg_start = p.seg + S;
  int32_t* seg_cnt = p.seg + 2 * S;
  int32_t* seg_item = p.seg + 3 * S;  // first gate/up item of each segment
  const int rbg = (p.rows_gu + kGemmRows - 1) / kGemmRows, rbd = (p.rows_dn + kGemmRows - 1) / kGemmRows;
  if (p.single_expert >= 0) {
    const bool small = p.T <= kGemvTokens;
    if (tid == 0) {
      seg_e[0] = p.single_expert;
      seg_start[0] = 0;
      seg_cnt[0] = p.T;
      p.seg[4 * S] = 1;
      p.small_seg[0] = 0;
    }
    for (int t = tid; t < p.T; t += blockDim.x) p.pos_tok[t] = t;
    const int ntb = small ? 0 : (p.T + kGemmTokens - 1) / kGemmTokens;
    for (int i = tid; i < rbg * ntb; i += blockDim.x) p.items_gu[i] = ((uint32_t)(i / ntb) << 8) | (i % ntb);
    for (int i = tid; i < rbd * ntb; i += blockDim.x) p.items_dn[i] = ((uint32_t)(i / ntb) << 8) | (i % ntb);
    if (tid == 0) {
      p.n_items[0] = rbg * ntb;
      p.n_items[1] = rbd * ntb;
      p.n_items[2] = small ? p.bands_gu : 0;
      p.n_items[3] = small ? p.bands_dn : 0;
    }
    return;
  }
  const int n = p.T * p.K;
  for (int e = tid; e < S; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  for (int base = tid - lane; base < n; base += blockDim.x) {
    const int i = base + lane;
    const int e = i < n ? p.idx[i] : -1;
    const uint32_t same = __match_any_sync(0xffffffffu, e);
    if (e >= 0 && lane == __ffs(same) - 1) atomicAdd(&cnt[e], __popc(same));
  }
  __syncthreads();
  if (tid == 0) cnt[p.E] = p.T;
  __syncthreads();
  // per candidate: positions, a segment if non-empty, its token blocks
  // segments of up to kGemvTokens positions go to the GEMV (no token blocks);
  // the second counter packs segments (low 16 bits) and small ones (high)
  const int c = tid < S ? cnt[tid] : 0;
  const bool small = c > 0 && c <= kGemvTokens;
  const int ntb = small ? 0 : (c + kGemmTokens - 1) / kGemmTokens;
  const int3 pre = block_scan3(make_int3(c, (c > 0 ? 1 : 0) | (small ? 1 << 16 : 0), ntb), scratch, tot);
  const int n_seg = tot[1] & 0xFFFF, n_small = tot[1] >> 16, n_tb = tot[2];
  const int sidx = pre.y & 0xFFFF;
  if (tid < S) {
    cur[tid] = pre.x;
    if (c > 0) {
      seg_e[sidx] = tid;
      seg_start[sidx] = pre.x;
      seg_cnt[sidx] = c;
      seg_item[sidx] = rbg * pre.z;
      if (small) p.small_seg[pre.y >> 16] = sidx;
    }
  }
  if (tid == 0) {
    p.seg[4 * S] = n_seg;
    p.n_items[0] = min(rbg * n_tb, p.max_items_gu);
    p.n_items[1] = min(rbd * n_tb, p.max_items_dn);
    p.n_items[2] = n_small * p.bands_gu;
    p.n_items[3] = n_small * p.bands_dn;
  }
  __syncthreads();
  for (int base = tid - lane; base < n; base += blockDim.x) {
    const int i = base + lane;
    const int e = i < n ? p.idx[i] : -1;
    const uint32_t same = __match_any_sync(0xffffffffu, e);
    const int leader = __ffs(same) - 1;
    int first = 0;
    if (e >= 0 && lane == leader) first = atomicAdd(&cur[e], __popc(same));
    first = __shfl_sync(0xffffffffu, first, leader);
    if (e >= 0) {
      const int pos = first + __popc(same & ((1u << lane) - 1u));
      p.pos_tok[pos] = i / p.K;
      p.pos_of[(i / p.K) * (p.K + 1) + i % p.K] = pos;
    }
  }
  for (int t = tid; t < p.T; t += blockDim.x) {
    const int pos = p.T * p.K + t;
    p.pos_tok[pos] = t;
    p.pos_of[t * (p.K + 1) + p.K] = pos;
  }
  // work items of this thread's segment: segment-major, then row block, then
  // token block (token blocks of one row block run side by side and share the
  // weight tiles in L2)
  if (tid < S && c > 0) {
    const int s = sidx, ig0 = rbg * pre.z, id0 = rbd * pre.z;
    for (int rb = 0; rb < rbg; ++rb)
      for (int tb = 0; tb < ntb; ++tb) {
        const int i = ig0 + rb * ntb + tb;
        if (i < p.max_items_gu) p.items_gu[i] = ((uint32_t)s << 16) | ((uint32_t)rb << 8) | (uint32_t)tb;
      }
    for (int rb = 0; rb < rbd; ++rb)
      for (int tb = 0; tb < ntb; ++tb) {
        const int i = id0 + rb * ntb + tb;
        if (i < p.max_items_dn) p.items_dn[i] = ((uint32_t)s << 16) | ((uint32_t)rb << 8) | (uint32_t)tb;
      }
  }
}

// ------------------------------------------------------------------ small segments: GEMV
// Segments of at most kGemvTokens positions (most experts of a 256-token step)
// are contracted by one warp per 16-row band with mma.sync m16n8k16: the
// packed tile is the A fragment layout, so the exact codes come out of one
// lop3 + sub per pair, and the 8 columns of B are the segment's positions.
// Per 64-column group each position's input is scaled to fp16 by its own
// power of two (exact for bf16), and the group's result is s*2^-sh*sum(q*x')
// + b*sum(x) in fp32, as in the batch-1 kernel: scale and bias never pass
// through fp16.

__device__ __forceinline__ uint32_t gv_lop(uint32_t a, uint32_t mask, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(mask), "r"(c));
  return d;
}
__device__ __forceinline__ uint32_t gv_code2(uint32_t w, uint32_t mask) {  // codes * 4^k, exact fp16 pair
  constexpr uint32_t kMagic = 0x64006400u;  // (1024, 1024)
  uint32_t d;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(gv_lop(w, mask, kMagic)), "r"(kMagic));
  return d;
}
__device__ __forceinline__ void gv_mma(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                       uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ float gv_exp2i(int k) { return __uint_as_float((uint32_t)(k + 127) << 23); }

struct GemvArgs {
  const int32_t* seg;        // segment table ([4][S] + n_seg)
  int S;
  const int32_t* small_seg;  // small segment -> segment index
  const int32_t* n_items;    // device count of (small segment, band) items
  const int32_t* pos_tok;    // position -> token (gate/up input rows)
  const void* src;           // gate/up: z bf16 [T][H] by token; down: a fp32 [P][I] by position
  int K;                     // contraction length (H or I)
  int bits;
  uint32_t* frag;            // [max_small][K/64][8][32]
  float2* info;              // [max_small][K/64][8]
  const uint8_t* experts;    // packed blobs of the layer
  int64_t blob;
  int64_t mat_off;           // byte offset of the matrix in a blob (0: gate/up, else down)
  int bands;                 // 16-row bands of the matrix
  float* out;                // gate/up: a [P][I]; down: y [P][H]
  int ldo;
  uint32_t* status;          // device status word (a timed-out wait sets kStatusTimeoutTc)
};

// B fragments of every small segment: one warp per (segment, group), the
// group's 64 values of each of the segment's (up to 8) positions; lane l holds
// values 2l, 2l+1.  Fragment word (position p, lane column t, slice s, half
// `which`) sits at ((item * 8 + p) * 32) + (t * 4 + s) * 2 + which, laid out
// as the batch-1 kernel's fragments; positions past the segment are zero.
template <typename Src>
__global__ void bt_gv_frag_kernel(GemvArgs g, int n_small_cap) {
  const int lane = threadIdx.x & 31, G = g.K / kGroup;
  const int n_small = *g.n_items / g.bands;  // the GEMV item count is small segments x bands
  const int q = 2 * lane, sl = q / 16, qq = q % 16, which = qq / 8, t = (qq % 8) / 2;
  const int fs = (g.bits == 4) ? (which ? 4 : 0) : ((sl & 1) ? 4 : 0) + (which ? 2 : 0);
  const int total = min(n_small, n_small_cap) * G;
  for (int it = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5); it < total; it += gridDim.x * (blockDim.x / 32)) {
    const int sr = it / G, gr = it % G;
    const int sg = g.small_seg[sr];
    const int pos0 = g.seg[g.S + sg], n = g.seg[2 * g.S + sg];
#pragma unroll 1
    for (int pj = 0; pj < kGemvTokens; ++pj) {
      float lo = 0.f, hi = 0.f;
      if (pj < n) {
        const int c0 = gr * kGroup + 2 * lane;
        if constexpr (sizeof(Src) == 2) {
          const uint32_t v = *reinterpret_cast<const uint32_t*>(static_cast<const uint16_t*>(g.src) +
                                                                (size_t)g.pos_tok[pos0 + pj] * g.K + c0);
          lo = bflo(v);
          hi = bfhi(v);
        } else {
          const float2 v = *reinterpret_cast<const float2*>(static_cast<const float*>(g.src) + (size_t)(pos0 + pj) * g.K + c0);
          lo = v.x;
          hi = v.y;
        }
      }
      const uint32_t m = __reduce_max_sync(0xffffffffu, max(__float_as_uint(fabsf(lo)), __float_as_uint(fabsf(hi))));
      float sum = lo + hi;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      const int e = (int)((m >> 23) & 0xFF) - 127;
      const int sh = m == 0 ? 0 : min(14 - max(e, -126), 126);
      const __half2 h2 = __floats2half2_rn(lo * gv_exp2i(sh - fs), hi * gv_exp2i(sh - fs));
      const size_t base = ((size_t)it * kGemvTokens + pj) * 32;
      g.frag[base + (t * 4 + sl) * 2 + which] = *reinterpret_cast<const uint32_t*>(&h2);
      if (lane == 0) g.info[(size_t)it * kGemvTokens + pj] = make_float2(gv_exp2i(-sh), sum);
    }
  }
}

// One block per (small segment, 8 consecutive 16-row bands): consumer warp w
// contracts band 8o+w; lane 4r+t accumulates rows r and r+8 of the band for
// positions 2t and 2t+1.  A producer warp streams the block's operands through
// a ring of kBsStages shared-memory stages, each holding kBsGroups groups: per
// band one bulk copy of its kBsGroups consecutive tiles (codes + scale/bias),
// plus the segment's B fragments and input info for those groups, copied once
// for all eight bands.  The block's items run as one stream of stages; one
// block per SM (the ring takes ~180 KB of shared memory).
constexpr int kBsWarps = 8;    // consumer warps (bands per item)
constexpr int kBsGroups = 16;  // groups (tiles per band) per stage
constexpr uint64_t kBsWaitNs = 500ull * 1000 * 1000;  // bounded waits: 0.5 s

template <int BITS>
struct BsLayout {
  using Codes = typename std::conditional<BITS == 4, uint4, uint2>::type;  // one lane's codes of a tile
  static constexpr int CODES = 16 * kGroup * BITS / 8;  // a 16-row band's codes for one group
  static constexpr int TILE = CODES + 64;               // + the 16 rows' (scale, bias)
  static constexpr int FRAG = kGemvTokens * 32 * 4;     // one group's B fragments (8 positions)
  static constexpr int INFO = kGemvTokens * 8;          // (2^-sh, sum x) per position
  static constexpr int BAND = kBsGroups * TILE;         // one band's tiles in a stage
  static constexpr int STAGE = kBsWarps * BAND + kBsGroups * (FRAG + INFO);
  static constexpr int STAGES = BITS == 4 ? 2 : 3;
  static constexpr int SMEM = STAGES * STAGE + 2 * STAGES * 8 + 16;
  static_assert(TILE % 16 == 0 && BAND % 128 == 0 && STAGE % 128 == 0, "bulk copy alignment");
  static_assert(SMEM <= 232448, "shared memory");
};

__device__ __forceinline__ uint32_t bs_su32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }
__device__ __forceinline__ uint64_t bs_time() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ bool bs_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait; false after kBsWaitNs or once the block has aborted.
__device__ __forceinline__ bool bs_wait(uint32_t bar, uint32_t parity, const volatile int* abort_flag) {
  if (bs_try(bar, parity)) return true;
  const uint64_t t0 = bs_time();
  for (uint32_t it = 0;; ++it) {
    if (bs_try(bar, parity)) return true;
    if ((it & 15) == 15 && (*abort_flag || bs_time() - t0 > kBsWaitNs)) return false;
    if (it >= 8) __nanosleep(32);
  }
}
__device__ __forceinline__ void bs_bulk(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

template <int BITS, bool GATE_UP>
__global__ void __launch_bounds__(32 * (kBsWarps + 1), 1) bt_gemv_kernel(GemvArgs g) {
  using Ly = BsLayout<BITS>;
  using Codes = typename Ly::Codes;
  constexpr int S = Ly::STAGES;
  extern __shared__ __align__(128) uint8_t bs_smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t base = bs_su32(bs_smem);
  const uint32_t full0 = base + S * Ly::STAGE, empty0 = full0 + 8 * S;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bs_smem + S * Ly::STAGE + 16 * S);
  const int G = g.K / kGroup;
  const int n_small = *g.n_items / g.bands;  // GEMV items are counted as small segments x bands
  const int octets = (g.bands + kBsWarps - 1) / kBsWarps;
  const int n_blk_items = n_small * octets;
  const int n_st = (G + kBsGroups - 1) / kBsGroups;  // stages per item
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(full0 + 8 * s) : "memory");
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(empty0 + 8 * s), "r"(kBsWarps) : "memory");
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (warp == kBsWarps) {
    // ---- producer: lane 0 fills stage q % S with the q-th stage of the block's stream
    if (lane != 0) return;
    int q = 0;
    bool ok = true;
    for (int bi = blockIdx.x; bi < n_blk_items && ok; bi += gridDim.x) {
      const int sr = bi / octets, b0 = (bi % octets) * kBsWarps;
      const int nb = min(kBsWarps, g.bands - b0);
      const uint8_t* tiles = g.experts + (int64_t)g.seg[g.small_seg[sr]] * g.blob + g.mat_off;
      const uint8_t* frag = reinterpret_cast<const uint8_t*>(g.frag) + (size_t)sr * G * Ly::FRAG;
      const uint8_t* info = reinterpret_cast<const uint8_t*>(g.info) + (size_t)sr * G * Ly::INFO;
      for (int j = 0; j < n_st; ++j, ++q) {
        const int s = q % S, gs = j * kBsGroups, ng = min(kBsGroups, G - gs);
        if (q >= S && !bs_wait(empty0 + 8 * s, (uint32_t)((q / S) - 1) & 1u, abort_flag)) {
          ok = false;
          break;
        }
        const uint32_t st = base + s * Ly::STAGE, full = full0 + 8 * s;
        const uint32_t bytes = (uint32_t)(nb * ng * Ly::TILE + ng * (Ly::FRAG + Ly::INFO));
        asm volatile("{ .reg .b64 t; mbarrier.arrive.expect_tx.shared::cta.b64 t, [%0], %1; }" ::"r"(full), "r"(bytes)
                     : "memory");
        for (int b = 0; b < nb; ++b)
          bs_bulk(st + b * Ly::BAND, tiles + ((int64_t)(b0 + b) * G + gs) * Ly::TILE, (uint32_t)(ng * Ly::TILE), full);
        bs_bulk(st + kBsWarps * Ly::BAND, frag + (size_t)gs * Ly::FRAG, (uint32_t)(ng * Ly::FRAG), full);
        bs_bulk(st + kBsWarps * Ly::BAND + kBsGroups * Ly::FRAG, info + (size_t)gs * Ly::INFO,
                (uint32_t)(ng * Ly::INFO), full);
      }
    }
    if (!ok) {
      if (!*abort_flag) atomicOr(g.status, kStatusTimeoutTc);
      *abort_flag = 1;
    }
    // every stage issued but not yet seen complete lands before the block exits (bounded)
    const uint64_t t0 = bs_time();
    for (int v = max(0, q - S); v < q; ++v)
      while (!bs_try(full0 + 8 * (v % S), (uint32_t)(v / S) & 1u) && bs_time() - t0 < kBsWaitNs) __nanosleep(64);
    return;
  }
  // ---- consumers: warp w contracts band b0 + w of each item
  const int r = lane >> 2, t = lane & 3;
  int q = 0;
  for (int bi = blockIdx.x; bi < n_blk_items; bi += gridDim.x) {
    const int sr = bi / octets, band = (bi % octets) * kBsWarps + warp;
    const int sg = g.small_seg[sr];
    const int pos0 = g.seg[g.S + sg], n = g.seg[2 * g.S + sg];
    const bool mine = band < g.bands;
    float a00 = 0.f, a01 = 0.f, a10 = 0.f, a11 = 0.f;  // (row r | r+8) x (position 2t | 2t+1)
    for (int j = 0; j < n_st; ++j, ++q) {
      const int s = q % S, ng = min(kBsGroups, G - j * kBsGroups);
      if (!__all_sync(0xffffffffu, bs_wait(full0 + 8 * s, (uint32_t)(q / S) & 1u, abort_flag))) {
        if (lane == 0) {
          if (!*abort_flag) atomicOr(g.status, kStatusTimeoutTc);
          *abort_flag = 1;
        }
        return;
      }
      const uint8_t* st = bs_smem + s * Ly::STAGE;
      const uint8_t* codes = st + warp * Ly::BAND;
      const uint8_t* frag = st + kBsWarps * Ly::BAND + (r * 32 + t * 8) * 4;
      const uint8_t* info = st + kBsWarps * Ly::BAND + kBsGroups * Ly::FRAG + 2 * t * 8;
      if (mine) {
#pragma unroll 4
        for (int k = 0; k < ng; ++k) {
          const uint8_t* tile = codes + k * Ly::TILE;
          const Codes qv = *reinterpret_cast<const Codes*>(tile + lane * sizeof(Codes));
          const uint2 sb = *reinterpret_cast<const uint2*>(tile + Ly::CODES + r * 8);
          const uint4 f0 = *reinterpret_cast<const uint4*>(frag + k * Ly::FRAG);
          const uint4 f1 = *reinterpret_cast<const uint4*>(frag + k * Ly::FRAG + 16);
          const float4 iv = *reinterpret_cast<const float4*>(info + k * Ly::INFO);  // positions 2t, 2t+1
          const uint32_t bb[8] = {f0.x, f0.y, f0.z, f0.w, f1.x, f1.y, f1.z, f1.w};
          float c[4] = {0.f, 0.f, 0.f, 0.f};
          if constexpr (BITS == 4) {
            const uint32_t w4[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
            for (int sl = 0; sl < 4; ++sl) {
              const uint32_t w = w4[sl], w8 = w >> 8;
              gv_mma(c, gv_code2(w, 0x000F000Fu), gv_code2(w8, 0x000F000Fu), gv_code2(w, 0x00F000F0u),
                     gv_code2(w8, 0x00F000F0u), bb[2 * sl], bb[2 * sl + 1]);
            }
          } else {
            const uint32_t w2[2] = {qv.x, qv.y};
#pragma unroll
            for (int wj = 0; wj < 2; ++wj) {
              const uint32_t w = w2[wj], w8 = w >> 8;
              gv_mma(c, gv_code2(w, 0x00030003u), gv_code2(w8, 0x00030003u), gv_code2(w, 0x000C000Cu),
                     gv_code2(w8, 0x000C000Cu), bb[4 * wj], bb[4 * wj + 1]);
              gv_mma(c, gv_code2(w, 0x00300030u), gv_code2(w8, 0x00300030u), gv_code2(w, 0x00C000C0u),
                     gv_code2(w8, 0x00C000C0u), bb[4 * wj + 2], bb[4 * wj + 3]);
            }
          }
          const float s0 = bflo(sb.x), b0 = bfhi(sb.x), s8 = bflo(sb.y), b8 = bfhi(sb.y);
          a00 = fmaf(s0 * iv.x, c[0], fmaf(b0, iv.y, a00));
          a01 = fmaf(s0 * iv.z, c[1], fmaf(b0, iv.w, a01));
          a10 = fmaf(s8 * iv.x, c[2], fmaf(b8, iv.y, a10));
          a11 = fmaf(s8 * iv.z, c[3], fmaf(b8, iv.w, a11));
        }
      }
      __syncwarp();
      if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(empty0 + 8 * s) : "memory");
    }
    if (!mine) continue;
    const int p0 = 2 * t, p1 = 2 * t + 1;
    if constexpr (GATE_UP) {
      // band rows r (gate) and r + 8 (up) are the same activation j
      const int jj = band * 8 + r;
      if (p0 < n) g.out[(size_t)(pos0 + p0) * g.ldo + jj] = a00 / (1.0f + expf(-a00)) * a10;
      if (p1 < n) g.out[(size_t)(pos0 + p1) * g.ldo + jj] = a01 / (1.0f + expf(-a01)) * a11;
    } else {
      const int row = band * 16 + r;
      if (p0 < n) {
        g.out[(size_t)(pos0 + p0) * g.ldo + row] = a00;
        g.out[(size_t)(pos0 + p0) * g.ldo + row + 8] = a10;
      }
      if (p1 < n) {
        g.out[(size_t)(pos0 + p1) * g.ldo + row] = a01;
        g.out[(size_t)(pos0 + p1) * g.ldo + row + 8] = a11;
      }
    }
  }
}

// ------------------------------------------------------------------ combine
// out[t] = bf16(h[t] + y[shared] + sum_k w[t][k] * y[routed k]), fixed order;
// four consecutive outputs per thread.
__global__ void bt_combine_kernel(const uint16_t* __restrict__ h, const float* __restrict__ y,
                                  const int32_t* __restrict__ pos_of, const float* __restrict__ w, int T, int H, int K,
                                  uint16_t* __restrict__ out) {
  const int64_t n4 = (int64_t)T * H / 4;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (int64_t)gridDim.x * blockDim.x) {
    const int tk = (int)(4 * i / H), c = (int)(4 * i % H);
    const int32_t* po = pos_of + (size_t)tk * (K + 1);
    const uint2 hv = *reinterpret_cast<const uint2*>(h + 4 * i);
    const float4 ys = *reinterpret_cast<const float4*>(y + (size_t)po[K] * H + c);
    float a0 = bflo(hv.x) + ys.x, a1 = bfhi(hv.x) + ys.y, a2 = bflo(hv.y) + ys.z, a3 = bfhi(hv.y) + ys.w;
    for (int k = 0; k < K; ++k) {
      const float wk = w[(size_t)tk * K + k];
      const float4 yk = *reinterpret_cast<const float4*>(y + (size_t)po[k] * H + c);
      a0 = fmaf(wk, yk.x, a0);
      a1 = fmaf(wk, yk.y, a1);
      a2 = fmaf(wk, yk.z, a2);
      a3 = fmaf(wk, yk.w, a3);
    }
    *reinterpret_cast<uint2*>(out + 4 * i) = make_uint2((uint32_t)to_bf16(a0) | ((uint32_t)to_bf16(a1) << 16),
                                                        (uint32_t)to_bf16(a2) | ((uint32_t)to_bf16(a3) << 16));
  }
}

template <int BITS, bool GATE_UP>
int launch_gemv_t(const GemvArgs& v, int n_sm, cudaStream_t st) {
  // the shared-memory opt-in is per device: set it on every launch, like the other kernels
  const cudaError_t e = cudaFuncSetAttribute(bt_gemv_kernel<BITS, GATE_UP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             BsLayout<BITS>::SMEM);
  if (e != cudaSuccess) return (int)e;
  bt_gemv_kernel<BITS, GATE_UP><<<n_sm, 32 * (kBsWarps + 1), BsLayout<BITS>::SMEM, st>>>(v);
  return (int)cudaGetLastError();
}

int launch_gemv(int bits, bool gate_up, const GemvArgs& v, int n_sm, cudaStream_t st) {
  if (bits == 4) return gate_up ? launch_gemv_t<4, true>(v, n_sm, st) : launch_gemv_t<4, false>(v, n_sm, st);
  return gate_up ? launch_gemv_t<2, true>(v, n_sm, st) : launch_gemv_t<2, false>(v, n_sm, st);
}

int grid_of(int64_t work, int per_block, int cap) {
  const int64_t b = (work + per_block - 1) / per_block;
  return (int)(b < 1 ? 1 : (b > cap ? cap : b));
}

}  // namespace

namespace {
// Lays the batched workspace out from `base` (0 to size it); returns its bytes.
size_t carve(uintptr_t base, int H, int E, int K, int I, int T, BatchWs& ws) {
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const uintptr_t p = base + off;
    off += (bytes + 255) / 256 * 256;
    return p;
  };
  const size_t P = (size_t)T * (K + 1);
  const int rbg = (2 * I + kGemmRows - 1) / kGemmRows, rbd = (H + kGemmRows - 1) / kGemmRows;
  // token blocks: at most P/64 full ones plus one partial per segment
  const int max_tb = (int)((P + kGemmTokens - 1) / kGemmTokens) + (E + 1);
  ws.pcap = (int)P;
  ws.max_items_gu = rbg * max_tb;
  ws.max_items_dn = rbd * max_tb;
  ws.z = reinterpret_cast<uint16_t*>(take((size_t)T * H * 2));
  ws.zp = reinterpret_cast<uint16_t*>(take(P * H * 2));
  ws.zsc = reinterpret_cast<float*>(take(P * 4));
  ws.zsum = reinterpret_cast<float*>(take((size_t)((H + 127) / 128) * P * 16));
  ws.logits = reinterpret_cast<float*>(take((size_t)T * E * 4));
  ws.logit_part = reinterpret_cast<float*>(take((size_t)kRtSplit * T * E * 4));
  ws.idx = reinterpret_cast<int32_t*>(take((size_t)T * K * 4));
  ws.w = reinterpret_cast<float*>(take((size_t)T * K * 4));
  ws.seg = reinterpret_cast<int32_t*>(take(((size_t)4 * (E + 1) + 1) * 4));
  ws.cursor = reinterpret_cast<int32_t*>(take((size_t)(E + 1) * 4));
  ws.pos_tok = reinterpret_cast<int32_t*>(take(P * 4));
  ws.pos_of = reinterpret_cast<int32_t*>(take(P * 4));
  ws.items_gu = reinterpret_cast<uint32_t*>(take((size_t)ws.max_items_gu * 4));
  ws.items_dn = reinterpret_cast<uint32_t*>(take((size_t)ws.max_items_dn * 4));
  ws.n_items = reinterpret_cast<int32_t*>(take(4 * 4));
  ws.max_small = (int)std::min<size_t>((size_t)E + 1, P);
  ws.small_seg = reinterpret_cast<int32_t*>(take((size_t)(E + 1) * 4));
  const size_t gmax = (size_t)std::max(H, I) / kGroup;
  ws.gv_frag = reinterpret_cast<uint32_t*>(take((size_t)ws.max_small * gmax * kGemvTokens * 32 * 4));
  ws.gv_info = reinterpret_cast<float2*>(take((size_t)ws.max_small * gmax * kGemvTokens * 8));
  ws.a = reinterpret_cast<float*>(take(P * I * 4));
  ws.ap = reinterpret_cast<uint16_t*>(take(P * I * 2));
  ws.asc = reinterpret_cast<float*>(take(P * 4));
  ws.asum = reinterpret_cast<float*>(take((size_t)((I + 127) / 128) * P * 16));
  ws.y = reinterpret_cast<float*>(take(P * H * 4));
  return off;
}
}  // namespace

size_t batch_ws_bytes(int H, int E, int K, int I, int T) {
  BatchWs ws;
  return carve(0, H, E, K, I, T, ws);
}

int batch_ws_carve(uint8_t* base, int H, int E, int K, int I, int T, BatchWs& ws) {
  carve(reinterpret_cast<uintptr_t>(base), H, E, K, I, T, ws);
  const int P = T * (K + 1);
  int rc = tc_encode_token_maps(ws.zp, H, P, ws.zmap);
  if (rc == 0) rc = tc_encode_token_maps(ws.ap, I, P, ws.amap);
  if (rc == 0) rc = tc_encode_sum_maps(ws.zsum, (H + 127) / 128, P, ws.zsmap);
  if (rc == 0) rc = tc_encode_sum_maps(ws.asum, (I + 127) / 128, P, ws.asmap);
  return rc;
}

int launch_batched(const BatchArgs& a, const BatchWs& ws, int n_sm, void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const bool layer = a.single_expert < 0;
  const int positions = layer ? a.T * (a.K + 1) : a.T;
  bt_norm_kernel<<<grid_of(a.T, 8, 4 * n_sm), 256, 0, st>>>(a.h_in, a.norm_w, a.eps, a.T, a.H, ws.z);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return (int)e;
  if (layer) {
    cudaFuncSetAttribute(bt_router_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kRtStages * kRtStage);
    const dim3 grid((a.E + kRtRows - 1) / kRtRows, (a.T + kRtRows - 1) / kRtRows, kRtSplit);
    bt_router_kernel<<<grid, 256, kRtStages * kRtStage, st>>>(a.router_w, ws.z, a.T, a.E, a.H, ws.logit_part);
    bt_logits_sum_kernel<<<grid_of((int64_t)a.T * a.E, 256, 4 * n_sm), 256, 0, st>>>(ws.logit_part, a.router_bias,
                                                                                  a.T, a.E, ws.logits);
    e = cudaGetLastError();
    if (e != cudaSuccess) return (int)e;
    const int rc = launch_topk_rows(ws.logits, a.T, a.E, a.K, ws.idx, ws.w, stream);
    if (rc != 0) return rc;
  }
  PermuteArgs pa{};
  pa.idx = ws.idx;
  pa.T = a.T;
  pa.E = a.E;
  pa.K = a.K;
  pa.single_expert = a.single_expert;
  pa.rows_gu = 2 * a.I;
  pa.rows_dn = a.H;
  pa.seg = ws.seg;
  pa.cursor = ws.cursor;
  pa.pos_tok = ws.pos_tok;
  pa.pos_of = ws.pos_of;
  pa.items_gu = ws.items_gu;
  pa.items_dn = ws.items_dn;
  pa.n_items = ws.n_items;
  pa.max_items_gu = ws.max_items_gu;
  pa.max_items_dn = ws.max_items_dn;
  pa.small_seg = ws.small_seg;
  pa.bands_gu = 2 * a.I / 16;
  pa.bands_dn = a.H / 16;
  bt_permute_kernel<<<1, 1024, (size_t)(2 * (a.E + 1) + 96 + 3) * 4, st>>>(pa);
  e = cudaGetLastError();
  if (e != cudaSuccess) return (int)e;
  // gate/up: B = each position's token input
  const int pcap = ws.pcap;
  bt_prep_kernel<uint16_t><<<grid_of(positions, 8, 8 * n_sm), 256, 0, st>>>(ws.z, ws.pos_tok, positions, a.H, ws.zp,
                                                                           ws.zsc, ws.zsum, pcap);
  TcArgs g{};
  g.seg = ws.seg;
  g.S = a.E + 1;
  g.items = ws.items_gu;
  g.n_items = ws.n_items;
  g.k_chunks = (a.H + 127) / 128;
  g.rows = 2 * a.I;
  g.ldo = a.I;
  g.bscale = ws.zsc;
  g.out = ws.a;
  g.status = a.status;
  auto mark = [&](int k) {
    if (a.gemm_events[k]) cudaEventRecord(static_cast<cudaEvent_t>(a.gemm_events[k]), st);
  };
  // small segments: B fragments of their positions, then the GEMV
  GemvArgs v{};
  v.seg = ws.seg;
  v.S = a.E + 1;
  v.small_seg = ws.small_seg;
  v.pos_tok = ws.pos_tok;
  v.bits = a.bits;
  v.frag = ws.gv_frag;
  v.info = ws.gv_info;
  v.experts = a.experts;
  v.blob = a.blob_bytes;
  v.status = a.status;
  mark(0);
  v.n_items = ws.n_items + 2;
  v.src = ws.z;
  v.K = a.H;
  v.mat_off = 0;
  v.bands = 2 * a.I / 16;
  v.out = ws.a;
  v.ldo = a.I;
  bt_gv_frag_kernel<uint16_t><<<2 * n_sm, 256, 0, st>>>(v, ws.max_small);
  int rc = launch_tc_gemm(a.bits, true, *a.wmap_gu, ws.zmap, ws.zsmap, g, n_sm, stream);
  if (rc != 0) return rc;
  rc = launch_gemv(a.bits, true, v, n_sm, st);
  if (rc != 0) return rc;
  mark(1);
  // down: B = the position's activation
  bt_prep_kernel<float><<<grid_of(positions, 8, 8 * n_sm), 256, 0, st>>>(ws.a, nullptr, positions, a.I, ws.ap, ws.asc,
                                                                        ws.asum, pcap);
  g.items = ws.items_dn;
  g.n_items = ws.n_items + 1;
  g.k_chunks = (a.I + 127) / 128;
  g.rows = a.H;
  g.ldo = a.H;
  g.bscale = ws.asc;
  g.out = layer ? ws.y : a.y_out;
  mark(2);
  v.n_items = ws.n_items + 3;
  v.src = ws.a;
  v.K = a.I;
  v.mat_off = packed_gu_bytes(a.H, a.I, a.bits);
  v.bands = a.H / 16;
  v.out = g.out;
  v.ldo = a.H;
  bt_gv_frag_kernel<float><<<2 * n_sm, 256, 0, st>>>(v, ws.max_small);
  rc = launch_tc_gemm(a.bits, false, *a.wmap_dn, ws.amap, ws.asmap, g, n_sm, stream);
  if (rc != 0) return rc;
  rc = launch_gemv(a.bits, false, v, n_sm, st);
  if (rc != 0) return rc;
  mark(3);
  if (layer) {
    bt_combine_kernel<<<grid_of((int64_t)a.T * a.H / 4, 256, 8 * n_sm), 256, 0, st>>>(a.h_in, ws.y, ws.pos_of, ws.w, a.T,
                                                                                  a.H, a.K, a.h_out);
    e = cudaGetLastError();
    if (e != cudaSuccess) return (int)e;
    if (a.idx_out) e = cudaMemcpyAsync(a.idx_out, ws.idx, (size_t)a.T * a.K * 4, cudaMemcpyDeviceToDevice, st);
    if (e == cudaSuccess && a.w_out) e = cudaMemcpyAsync(a.w_out, ws.w, (size_t)a.T * a.K * 4, cudaMemcpyDeviceToDevice, st);
    if (e != cudaSuccess) return (int)e;
  }
  return 0;
}

}  // namespace fmoe
