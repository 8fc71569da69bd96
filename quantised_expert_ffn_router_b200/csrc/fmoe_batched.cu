// fmoe_batched.cu -- the mixture-of-experts layer for T tokens at once.
//
// With many tokens per step the expert matrices become real contractions: an
// expert chosen by n tokens multiplies an [rows x K] weight matrix by an
// [K x n] block of token vectors.  The batch-1 kernel (fmoe_decode.cu) reads
// every expert once per token; here each selected expert is read once per 64
// of its tokens.  The steps, all on the caller's stream:
//   norm     z = RMSNorm(h) (or h), bf16
//   frag     per (token, 64-group): fp16 values scaled by a power of two so the
//            group's largest magnitude lies in [2^14, 2^15), plus the group sum
//   router   logits = W_r z (+ bias), bf16 tensor-core GEMM, fp32 accumulate
//   top-K    per token (launch_topk_rows)
//   permute  (token, slot) pairs grouped by expert into segments; the shared
//            expert's segment holds every token; a list of GEMM work items
//   gate/up  grouped GEMM: a work item is 128 rows (8 units of 8 gate + 8 up
//            rows) x 64 positions of one expert; exact integer codes x fp16
//            values on mma.sync, per-group s*sum(q*x) + b*sum(x) epilogue,
//            a = silu(g)*u written per position
//   frag     of a, per (position, 64-group)
//   down     grouped GEMM, 128 output rows x 64 positions per work item
//   combine  out = h + y_shared + sum_k w_k y_k, fp32, one bf16 rounding
#include <cuda_bf16.h>
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

__device__ __forceinline__ uint32_t lop_and_or(uint32_t a, uint32_t mask, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(mask), "r"(c));
  return d;
}
__device__ __forceinline__ uint32_t hsub2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ void mma_f16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                        uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
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

constexpr uint32_t kMagic = 0x64006400u;  // fp16 pair (1024, 1024)
constexpr int kBRowBytes = 144;          // fragment record: 128 B of fp16 values, 8 B info, 8 B pad

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

// ------------------------------------------------------------------ fragments
// One warp per (row, 64-group); lane l holds elements 2l, 2l+1.  The group is
// scaled by 2^sh so its largest magnitude lies in [2^14, 2^15) (any finite
// input fits fp16); element k of the group is further divided by 4^fs(k) where
// the packed layout stores its codes as code * 4^fs (the same positions the
// batch-1 kernel's fragments use).  Output: one 144-byte record per (row,
// group): 64 fp16 values, then (2^-sh, sum of the group) as two floats, then
// 8 bytes of padding -- exactly the shared-memory row the GEMM reads, so the
// copies of a row bring its values and its scale together.
template <typename Src>
__global__ void bt_frag_kernel(const Src* __restrict__ src, int rows, int cols, int bits, uint8_t* __restrict__ dst) {
  const int lane = threadIdx.x & 31;
  const int ng = cols / kGroup;
  const int q = 2 * lane, s = q / 16, which = (q % 16) / 8;
  const int fs = (bits == 4) ? (which ? 4 : 0) : ((s & 1) ? 4 : 0) + (which ? 2 : 0);
  for (int item = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5); item < rows * ng;
       item += gridDim.x * (blockDim.x / 32)) {
    const int r = item / ng, G = item % ng;
    const size_t off = (size_t)r * cols + (size_t)G * kGroup + q;
    float v0, v1;
    if constexpr (sizeof(Src) == 2) {
      const uint32_t p = *reinterpret_cast<const uint32_t*>(src + off);
      v0 = bflo(p);
      v1 = bfhi(p);
    } else {
      const float2 p = *reinterpret_cast<const float2*>(src + off);
      v0 = p.x;
      v1 = p.y;
    }
    uint32_t m = max(__float_as_uint(fabsf(v0)), __float_as_uint(fabsf(v1)));
    m = __reduce_max_sync(0xffffffffu, m);
    float sum = v0 + v1;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    const int e = (int)((m >> 23) & 0xFF) - 127;
    int sh = (m == 0) ? 0 : 14 - max(e, -126);
    sh = min(sh, 126);
    const float scl = pow2(sh - fs);
    uint8_t* row = dst + ((size_t)r * ng + G) * kBRowBytes;
    *reinterpret_cast<__half2*>(row + 4 * lane) = __floats2half2_rn(v0 * scl, v1 * scl);
    if (lane == 0) *reinterpret_cast<float2*>(row + kGroup * 2) = make_float2(pow2(-sh), sum);  // after the values
  }
}

// ------------------------------------------------------------------ router
// logits[t][e] = sum_h W_r[e][h] z[t][h] (+ bias[e]), bf16 mma.sync with fp32
// accumulation.  A block computes 64 experts x 64 tokens: 64-column chunks of
// both operands are staged in shared memory by cp.async (3 stages, rows padded
// to 36 words so fragment reads are conflict-free); warp (we, wt) owns experts
// 16*we.. and tokens 32*wt.. (4 blocks of 8).
constexpr int kRtRows = 64, kRtStages = 4, kRtRowWords = 36, kRtSplit = 4;
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
    if (tid == 0) {
      seg_e[0] = p.single_expert;
      seg_start[0] = 0;
      seg_cnt[0] = p.T;
      p.seg[4 * S] = 1;
    }
    for (int t = tid; t < p.T; t += blockDim.x) p.pos_tok[t] = t;
    const int ntb = (p.T + kGemmTokens - 1) / kGemmTokens;
    for (int i = tid; i < rbg * ntb; i += blockDim.x) p.items_gu[i] = ((uint32_t)(i / ntb) << 8) | (i % ntb);
    for (int i = tid; i < rbd * ntb; i += blockDim.x) p.items_dn[i] = ((uint32_t)(i / ntb) << 8) | (i % ntb);
    if (tid == 0) {
      p.n_items[0] = rbg * ntb;
      p.n_items[1] = rbd * ntb;
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
  const int c = tid < S ? cnt[tid] : 0;
  const int ntb = (c + kGemmTokens - 1) / kGemmTokens;
  const int3 pre = block_scan3(make_int3(c, c > 0 ? 1 : 0, ntb), scratch, tot);
  const int n_seg = tot[1], n_tb = tot[2];
  if (tid < S) {
    cur[tid] = pre.x;
    if (c > 0) {
      seg_e[pre.y] = tid;
      seg_start[pre.y] = pre.x;
      seg_cnt[pre.y] = c;
      seg_item[pre.y] = rbg * pre.z;
    }
  }
  if (tid == 0) {
    p.seg[4 * S] = n_seg;
    p.n_items[0] = min(rbg * n_tb, p.max_items_gu);
    p.n_items[1] = min(rbd * n_tb, p.max_items_dn);
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
    const int s = pre.y, ig0 = rbg * pre.z, id0 = rbd * pre.z;
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

// ------------------------------------------------------------------ grouped GEMM
struct GemmArgs {
  const uint8_t* experts;
  int64_t blob_bytes;
  int64_t region;        // byte offset of the matrix inside a blob (0: gate/up, else down)
  int rows;              // matrix rows (2I gate/up, H down)
  int k_groups;          // 64-column groups along K (H/64 gate/up, I/64 down)
  int ldo;               // elements per output row (I for a, H for y)
  const int32_t* seg;    // segment table
  int n_seg_stride;      // E+1
  const uint32_t* items;
  const int32_t* n_items;
  const int32_t* pos_tok;  // B row of a position (gate/up: its token; null: the position itself)
  const uint8_t* bsrc;     // fragment records [rows][k_groups][144 B]
  float* out;              // gate/up: a [pos][I]; down: y [pos][H]
};

constexpr int kStages = 6;      // 6 x 13.5 KB per block; two blocks per SM keep ~140 KB of copies in flight
constexpr int kBRowWords = kBRowBytes / 4;  // 36: the record's 4 extra words keep fragment reads conflict-free
template <int BITS>
struct GemmSmem {
  static constexpr int TB = 16 * kGroup * BITS / 8 + 64;
  static constexpr int A_BYTES = 8 * TB;
  static constexpr int B_BYTES = kGemmTokens * kBRowBytes;
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int TOTAL = kStages * STAGE;
};

// 4-bit: the four A fragment registers of one 16-column slice from lane word w.
__device__ __forceinline__ void a_frag4(uint32_t w, uint32_t (&a)[4]) {
  const uint32_t w8 = w >> 8;
  a[0] = hsub2(lop_and_or(w, 0x000F000Fu, kMagic), kMagic);
  a[1] = hsub2(lop_and_or(w8, 0x000F000Fu, kMagic), kMagic);
  a[2] = hsub2(lop_and_or(w, 0x00F000F0u, kMagic), kMagic);
  a[3] = hsub2(lop_and_or(w8, 0x00F000F0u, kMagic), kMagic);
}
// 2-bit: fragments of the even and odd slices stored in lane word w.
__device__ __forceinline__ void a_frag2(uint32_t w, uint32_t (&ae)[4], uint32_t (&ao)[4]) {
  const uint32_t w8 = w >> 8;
  ae[0] = hsub2(lop_and_or(w, 0x00030003u, kMagic), kMagic);
  ae[1] = hsub2(lop_and_or(w8, 0x00030003u, kMagic), kMagic);
  ae[2] = hsub2(lop_and_or(w, 0x000C000Cu, kMagic), kMagic);
  ae[3] = hsub2(lop_and_or(w8, 0x000C000Cu, kMagic), kMagic);
  ao[0] = hsub2(lop_and_or(w, 0x00300030u, kMagic), kMagic);
  ao[1] = hsub2(lop_and_or(w8, 0x00300030u, kMagic), kMagic);
  ao[2] = hsub2(lop_and_or(w, 0x00C000C0u, kMagic), kMagic);
  ao[3] = hsub2(lop_and_or(w8, 0x00C000C0u, kMagic), kMagic);
}

// One 128-row x 64-position work item per iteration.  Warp w owns rows
// 16*(8*rb + w) .. +15 (one packed row block); per 64-column group it takes 4
// k-slices x (positions/8) token blocks of mma.sync and folds the group's scale
// and bias: acc += s * C * inv_scale(position, group) + b * sum(position, group).
// All threads stream each group's 8 weight tiles and B records into a ring of
// stages with 16-byte cp.async copies (records are gathered rows, too small
// for bulk copies to pay); a stage is refilled after the block barrier that
// follows its last use.
template <int BITS, bool GATE_UP>
__global__ void __launch_bounds__(256) bt_gemm_kernel(GemmArgs p) {
  using L = GemmSmem<BITS>;
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
  const int S = p.n_seg_stride;
  const int n_items = *p.n_items;
  const int n_rb16 = p.rows / 16;  // packed row blocks of the matrix
  constexpr int kAChunks = L::A_BYTES / 16, kBChunks = kGemmTokens * kBRowBytes / 16;
  constexpr int kAPer = (kAChunks + 255) / 256, kBPer = (kBChunks + 255) / 256;
  for (int it = blockIdx.x; it < n_items; it += gridDim.x) {
    const uint32_t item = p.items[it];
    const int s = (int)(item >> 16), rb = (int)((item >> 8) & 0xFF), tb = (int)(item & 0xFF);
    const int e = p.seg[s], pos0 = p.seg[S + s] + tb * kGemmTokens;
    const int ntok = min(kGemmTokens, p.seg[2 * S + s] - tb * kGemmTokens);
    const uint8_t* mat = p.experts + (int64_t)e * p.blob_bytes + p.region;
    const int my_rb = rb * 8 + warp;  // this warp's packed row block
    const bool active = my_rb < n_rb16;
    const int nb = (ntok + 7) / 8;    // 8-position blocks holding tokens (the rest are skipped)
    // This thread's 16-byte copies of every group: sources at group 0 (a
    // group adds TB to a weight source and 144 to a record source) and fixed
    // shared-memory offsets.  Weight tiles of rows past the matrix and records
    // of positions past the segment are not copied (their columns are unused).
    const uint8_t* asrc[kAPer];
    uint32_t adst[kAPer];
    bool aok[kAPer];
#pragma unroll
    for (int k = 0; k < kAPer; ++k) {
      const int c = tid + 256 * k, w = c / (L::TB / 16), off = (c % (L::TB / 16)) * 16;
      aok[k] = c < kAChunks && rb * 8 + w < n_rb16;
      asrc[k] = mat + (int64_t)(aok[k] ? rb * 8 + w : 0) * p.k_groups * L::TB + off;
      adst[k] = (uint32_t)(w * L::TB + off);
    }
    const uint8_t* bsrc[kBPer];
    uint32_t bdst[kBPer];
    bool bok[kBPer];
#pragma unroll
    for (int k = 0; k < kBPer; ++k) {
      const int c = tid + 256 * k, j = c / (kBRowBytes / 16), part = c % (kBRowBytes / 16);
      bok[k] = c < kBChunks && j < ntok;
      const int row = bok[k] ? (p.pos_tok ? p.pos_tok[pos0 + j] : pos0 + j) : 0;
      bsrc[k] = p.bsrc + (size_t)row * p.k_groups * kBRowBytes + part * 16;
      bdst[k] = (uint32_t)(L::A_BYTES + j * kBRowBytes + part * 16);
    }
    auto load = [&](int gi, int st) {
      uint8_t* base = smem + st * L::STAGE;
#pragma unroll
      for (int k = 0; k < kAPer; ++k)
        if (aok[k]) cp_async16(base + adst[k], asrc[k] + (int64_t)gi * L::TB, 16u);
#pragma unroll
      for (int k = 0; k < kBPer; ++k)
        if (bok[k]) cp_async16(base + bdst[k], bsrc[k] + (size_t)gi * kBRowBytes, 16u);
    };
    float acc[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
    __syncthreads();  // the previous item's stages are no longer read
#pragma unroll
    for (int st = 0; st < kStages - 1; ++st) {
      if (st < p.k_groups) load(st, st);
      cp_async_commit();
    }
    for (int gi = 0; gi < p.k_groups; ++gi) {
      cp_async_wait<kStages - 2>();
      __syncthreads();  // stage gi visible to all; the stage of gi - 1 is free again
      if (gi + kStages - 1 < p.k_groups) load(gi + kStages - 1, (gi + kStages - 1) % kStages);
      cp_async_commit();
      const int st = gi % kStages;
      if (active) {
        const uint8_t* sa = smem + st * L::STAGE;
        const uint32_t* sb = reinterpret_cast<const uint32_t*>(sa + L::A_BYTES);
        const uint8_t* tile = sa + warp * L::TB;
        float c[8][4];
#pragma unroll
        for (int j = 0; j < 8; ++j) c[j][0] = c[j][1] = c[j][2] = c[j][3] = 0.f;
        if (BITS == 4) {
          const uint4 qv = *reinterpret_cast<const uint4*>(tile + lane * 16);
          const uint32_t qw[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
          for (int sl = 0; sl < 4; ++sl) {
            uint32_t a[4];
            a_frag4(qw[sl], a);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              if (j >= nb) break;
              const uint32_t* br = sb + (8 * j + g) * kBRowWords + 8 * sl + t;
              mma_f16(c[j], a[0], a[1], a[2], a[3], br[0], br[4]);
            }
          }
        } else {
          const uint2 qv = *reinterpret_cast<const uint2*>(tile + lane * 8);
          const uint32_t qw[2] = {qv.x, qv.y};
#pragma unroll
          for (int wj = 0; wj < 2; ++wj) {
            uint32_t ae[4], ao[4];
            a_frag2(qw[wj], ae, ao);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              if (j >= nb) break;
              const uint32_t* be = sb + (8 * j + g) * kBRowWords + 8 * (2 * wj) + t;
              const uint32_t* bo = sb + (8 * j + g) * kBRowWords + 8 * (2 * wj + 1) + t;
              mma_f16(c[j], ae[0], ae[1], ae[2], ae[3], be[0], be[4]);
              mma_f16(c[j], ao[0], ao[1], ao[2], ao[3], bo[0], bo[4]);
            }
          }
        }
        const uint2 sbv = *reinterpret_cast<const uint2*>(tile + 16 * kGroup * BITS / 8 + g * 8);
        const float s0 = bflo(sbv.x), b0 = bfhi(sbv.x), s8 = bflo(sbv.y), b8 = bfhi(sbv.y);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (j >= nb) break;
          // the record's info: (2^-scale, sum) right after the 64 values
          const float2 i0 = *reinterpret_cast<const float2*>(sb + (8 * j + 2 * t) * kBRowWords + 32);
          const float2 i1 = *reinterpret_cast<const float2*>(sb + (8 * j + 2 * t + 1) * kBRowWords + 32);
          acc[j][0] = fmaf(s0 * i0.x, c[j][0], fmaf(b0, i0.y, acc[j][0]));
          acc[j][1] = fmaf(s0 * i1.x, c[j][1], fmaf(b0, i1.y, acc[j][1]));
          acc[j][2] = fmaf(s8 * i0.x, c[j][2], fmaf(b8, i0.y, acc[j][2]));
          acc[j][3] = fmaf(s8 * i1.x, c[j][3], fmaf(b8, i1.y, acc[j][3]));
        }
      }
    }
    cp_async_wait<0>();
    if (!active) continue;
    // lane holds rows g, g+8 of its row block for positions 8j + 2t, 8j + 2t + 1
#pragma unroll
    for (int j = 0; j < 8; ++j) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int jt = 8 * j + 2 * t + h;
        if (jt >= ntok) continue;
        float* orow = p.out + (size_t)(pos0 + jt) * p.ldo;
        if (GATE_UP) {
          // row g is gate row 8*my_rb + g, row g + 8 its up row
          const float gv = acc[j][h], uv = acc[j][2 + h];
          orow[my_rb * 8 + g] = gv / (1.0f + expf(-gv)) * uv;
        } else {
          orow[my_rb * 16 + g] = acc[j][h];
          orow[my_rb * 16 + g + 8] = acc[j][2 + h];
        }
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

int grid_of(int64_t work, int per_block, int cap) {
  const int64_t b = (work + per_block - 1) / per_block;
  return (int)(b < 1 ? 1 : (b > cap ? cap : b));
}

template <int BITS>
int launch_gemms(const BatchArgs& a, const BatchWs& ws, int n_sm, cudaStream_t st, int positions) {
  using L = GemmSmem<BITS>;
  cudaFuncSetAttribute(bt_gemm_kernel<BITS, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::TOTAL);
  cudaFuncSetAttribute(bt_gemm_kernel<BITS, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::TOTAL);
  GemmArgs g{};
  g.experts = a.experts;
  g.blob_bytes = a.blob_bytes;
  g.seg = ws.seg;
  g.n_seg_stride = a.E + 1;
  // gate/up: B = z fragments of each position's token
  g.region = 0;
  g.rows = 2 * a.I;
  g.k_groups = a.H / kGroup;
  g.ldo = a.I;
  g.items = ws.items_gu;
  g.n_items = ws.n_items;
  g.pos_tok = ws.pos_tok;
  g.bsrc = ws.zf;
  g.out = ws.a;
  bt_gemm_kernel<BITS, true><<<2 * n_sm, 256, L::TOTAL, st>>>(g);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return (int)e;
  // fragments of a, per position
  bt_frag_kernel<float><<<grid_of((int64_t)positions * (a.I / kGroup), 8, 8 * n_sm), 256, 0, st>>>(
      ws.a, positions, a.I, BITS, ws.af);
  // down: B = a fragments of the position itself
  g.region = packed_gu_bytes(a.H, a.I, BITS);
  g.rows = a.H;
  g.k_groups = a.I / kGroup;
  g.ldo = a.H;
  g.items = ws.items_dn;
  g.n_items = ws.n_items + 1;
  g.pos_tok = nullptr;
  g.bsrc = ws.af;
  g.out = a.single_expert >= 0 ? a.y_out : ws.y;
  bt_gemm_kernel<BITS, false><<<2 * n_sm, 256, L::TOTAL, st>>>(g);
  return (int)cudaGetLastError();
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
  ws.max_items_gu = rbg * max_tb;
  ws.max_items_dn = rbd * max_tb;
  ws.z = reinterpret_cast<uint16_t*>(take((size_t)T * H * 2));
  ws.zf = reinterpret_cast<uint8_t*>(take((size_t)T * (H / kGroup) * kBRowBytes));
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
  ws.n_items = reinterpret_cast<int32_t*>(take(2 * 4));
  ws.a = reinterpret_cast<float*>(take(P * I * 4));
  ws.af = reinterpret_cast<uint8_t*>(take(P * (I / kGroup) * kBRowBytes));
  ws.y = reinterpret_cast<float*>(take(P * H * 4));
  return off;
}
}  // namespace

size_t batch_ws_bytes(int H, int E, int K, int I, int T) {
  BatchWs ws;
  return carve(0, H, E, K, I, T, ws);
}

void batch_ws_carve(uint8_t* base, int H, int E, int K, int I, int T, BatchWs& ws) {
  carve(reinterpret_cast<uintptr_t>(base), H, E, K, I, T, ws);
}

int launch_batched(const BatchArgs& a, const BatchWs& ws, int n_sm, void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const bool layer = a.single_expert < 0;
  const int positions = layer ? a.T * (a.K + 1) : a.T;
  bt_norm_kernel<<<grid_of(a.T, 8, 4 * n_sm), 256, 0, st>>>(a.h_in, a.norm_w, a.eps, a.T, a.H, ws.z);
  bt_frag_kernel<uint16_t><<<grid_of((int64_t)a.T * (a.H / kGroup), 8, 8 * n_sm), 256, 0, st>>>(
      ws.z, a.T, a.H, a.bits, ws.zf);
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
  bt_permute_kernel<<<1, 1024, (size_t)(2 * (a.E + 1) + 96 + 3) * 4, st>>>(pa);
  e = cudaGetLastError();
  if (e != cudaSuccess) return (int)e;
  const int rc = a.bits == 4 ? launch_gemms<4>(a, ws, n_sm, st, positions) : launch_gemms<2>(a, ws, n_sm, st, positions);
  if (rc != 0) return rc;
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
