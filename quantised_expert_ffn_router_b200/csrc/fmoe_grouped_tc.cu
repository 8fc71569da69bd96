// fmoe_grouped_tc.cu -- the grouped per-expert dequant GEMM of the batched
// layer on the 5th-generation tensor cores (tcgen05, tensor memory, TMA).
//
// A work item (from the permute step) is one expert, one block of 128 matrix
// rows and up to 64 positions:  C[128 x n] = W[128 x K] X[n x K]^T  with W the
// packed b-bit tiles of the expert (w = q*s + b per 64-column group, the
// affine dequantisation the Flash-MoE pages apply in their FMA kernel: "Flash-MoE:
// Running a 400 Billion Parameter Model on a MacBook", section "The
// Architecture") and X an fp16 copy of the positions' inputs, each row scaled
// by a power of two (bt_prep_kernel, fmoe_batched.cu).
//
// One persistent block per SM, 15 warps:
//   warp 0      TMA producer.  Per 128-column chunk (one ring stage): one 3-D
//               copy of the item's 8 bands x 2 packed tiles and one 3-D copy of
//               the n' = ceil(n/16)*16 rows x 2 x 64 columns of X (128-byte
//               swizzle; one of four tensor maps by n').  A TMA instruction
//               costs the issuing lane ~0.1 us, so a chunk takes two.
//   warps 1, 14 MMA issuers (warp 1 also allocates tensor memory): one lane
//               each, even / odd chunks, each into its own accumulator (A from
//               tensor memory, B from shared memory, fp32 in tensor memory,
//               M=128, N=ceil(n/16)*16, 8 x K=16 per chunk), committing to the
//               ring / buffer barriers.  A thread issues one tcgen05.mma per
//               ~55 cycles however small N is, so two issuers halve the time
//               the tensor core needs per chunk.
//   warps 2-9   two groups of four that take alternate chunks: a warp turns two
//               bands (32 rows) x 2 tiles into fp16 weights and stores them into
//               the A buffer with tcgen05.st.16x256b, whose thread layout is the
//               mma.sync fragment layout the packed tile is stored in (lane
//               4g+t: rows g and g+8, columns 2t, 2t+1 | 2t+8, 2t+9).
//   warps 10-13 epilogue: add the two accumulators (double-buffered, so it
//               overlaps the next item's main loop), scale each column back by
//               its position's power of two, and write a = silu(g)*u (gate/up)
//               or y (down) in fp32.
//
// K order.  The 16x256b store puts a lane's fragment columns {2t, 2t+1, 2t+8,
// 2t+9} of a 16-column slice at tensor-memory positions 4t..4t+3, so within
// every 16 columns A holds column pi(p) = 2*(p/4) + p%2 + 8*((p/2)%2) at
// position p.  The prep kernel stores X in the same order; the contraction over
// K does not depend on the order.
//
// Exact codes.  A code at bit offset o of a 32-bit word is moved into the
// mantissa of an fp16 constant whose unit in the last place is 2^-o
// (1024, 256, 64, 16 for o = 0, 2, 4, 6), so subtracting the constant leaves
// the code exactly; one fma.rn.f16x2 then gives round_fp16(q*s + b).
//
// Every wait is bounded (globaltimer); on a timeout the block records
// kStatusTimeoutTc in the workspace status word, the other roles stop at their
// next wait, the MMA lane drains its tensor-core work and the block frees its
// tensor memory and exits.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstring>

#include "fmoe_internal.h"

namespace fmoe {
namespace {

constexpr int kTcWarps = 15;
constexpr int kTcThreads = kTcWarps * 32;
constexpr int kTcBBytes = 2 * kGemmTokens * 128;  // X in a stage: 2 halves x up to 64 rows x 128 B (16 KB)
constexpr int kTcABufs = 4;                       // A buffers in tensor memory (64 columns each)
constexpr int kTcXMaps = kGemmTokens / 16;          // input tensor maps, one per box height
constexpr int kTcIssuers = 2;                     // MMA-issuing threads, one accumulator each
constexpr int kTcDCols = kTcIssuers * kGemmTokens;  // accumulator columns per buffer (both issuers)
constexpr int kTcACol0 = 2 * kTcDCols;            // first A column (after two buffers)
constexpr uint32_t kTcTmemCols = 512;
constexpr uint64_t kTcWaitNs = 500ull * 1000 * 1000;  // bounded waits: 0.5 s

template <int BITS>
struct TcL {
  static constexpr int TB = 16 * kGroup * BITS / 8 + 64;  // packed tile bytes
  static constexpr int CODES = 8 * 2 * TB;               // 8 bands x 2 tiles
  static constexpr int STAGE = kTcBBytes + CODES;        // multiple of 1024
  static constexpr int NS = BITS == 4 ? 8 : 10;
  static constexpr int BAR = NS * STAGE;                 // barriers after the ring
  static constexpr int SMEM = BAR + 512 + 1024;          // + alignment slack
  static_assert(STAGE % 1024 == 0, "stage alignment");
};

// ------------------------------------------------------------------ PTX helpers
__device__ __forceinline__ uint32_t su32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }
__device__ __forceinline__ uint64_t gtime() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("{ .reg .b64 st; mbarrier.arrive.shared::cta.b64 st, [%0]; }" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("{ .reg .b64 st; mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1; }" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait; false on timeout or when another role has aborted.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, const volatile int* abort_flag) {
  if (mbar_try(bar, parity)) return true;
  const uint64_t t0 = gtime();
  for (uint32_t it = 0;; ++it) {
    if (mbar_try(bar, parity)) return true;
    if ((it & 15) == 15 && ((abort_flag && *abort_flag) || gtime() - t0 > kTcWaitNs)) return false;
    if (it >= 8) __nanosleep(20);
  }
}
__device__ __forceinline__ void tma_3d(uint32_t dst, const void* map, int x, int y, int z, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(
          dst),
      "l"(map), "r"(x), "r"(y), "r"(z), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem]^T, kind::f16, cta_group::1.
__device__ __forceinline__ void tc_mma(uint32_t d, uint32_t a, uint64_t bdesc, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{ .reg .pred p; setp.ne.b32 p, %4, 0;\n"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %5, %5, %5}, p; }" ::"r"(d),
      "r"(a), "l"(bdesc), "r"(idesc), "r"(acc), "r"(0u)
      : "memory");
}
// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (the layout a 64-column fp16 TMA box with 128-byte swizzle
// writes at a 1024-byte aligned address).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t addr) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) | ((uint64_t)1 << 46) |
         ((uint64_t)2 << 61);
}
// Instruction descriptor: fp32 accumulator, fp16 A and B, both K-major, M=128.
__device__ __forceinline__ uint32_t f16_idesc(int n) {
  return (1u << 4) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

__device__ __forceinline__ void tmem_st16x256x4(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x256b.x4.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_ld16x256x8(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x256b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_ld32x32x32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// ------------------------------------------------------------------ dequantisation
__device__ __forceinline__ uint32_t lop_and_or(uint32_t a, uint32_t mask, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(mask), "r"(c));
  return d;
}
// round_fp16(code * s + b) for the two codes of `w` under `mask`; `magic` is the
// fp16 pair whose last mantissa place is the mask's lowest bit.
__device__ __forceinline__ uint32_t dq2(uint32_t w, uint32_t mask, uint32_t magic, uint32_t s2, uint32_t b2) {
  uint32_t q, d;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(q) : "r"(lop_and_or(w, mask, magic)), "r"(magic));
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(q), "r"(s2), "r"(b2));
  return d;
}
__device__ __forceinline__ uint32_t h2dup_bf16(uint32_t bf_bits) {  // bf16 (low 16 bits) -> fp16 pair
  const float f = __uint_as_float(bf_bits << 16);
  const __half2 h = __floats2half2_rn(f, f);
  return *reinterpret_cast<const uint32_t*>(&h);
}
constexpr uint32_t kM0 = 0x64006400u;  // 1024: codes at bit 0
constexpr uint32_t kM2 = 0x5C005C00u;  // 256:  codes at bit 2
constexpr uint32_t kM4 = 0x54005400u;  // 64:   codes at bit 4
constexpr uint32_t kM6 = 0x4C004C00u;  // 16:   codes at bit 6

// The 16 registers tcgen05.st.16x256b.x4 stores for one packed tile (4 slices
// of 16 columns): per slice {row g cols 2t,2t+1; row g cols 2t+8,2t+9; row g+8
// cols 2t,2t+1; row g+8 cols 2t+8,2t+9}.
template <int BITS>
__device__ __forceinline__ void dequant_tile(const uint8_t* tile, int lane, uint32_t (&r)[16]) {
  const int g = lane >> 2;
  const uint2 sb = *reinterpret_cast<const uint2*>(tile + 16 * kGroup * BITS / 8 + g * 8);
  const uint32_t s0 = h2dup_bf16(sb.x & 0xFFFFu), b0 = h2dup_bf16(sb.x >> 16);
  const uint32_t s8 = h2dup_bf16(sb.y & 0xFFFFu), b8 = h2dup_bf16(sb.y >> 16);
  if constexpr (BITS == 4) {
    const uint4 qv = *reinterpret_cast<const uint4*>(tile + lane * 16);
    const uint32_t qw[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
    for (int sl = 0; sl < 4; ++sl) {
      const uint32_t w = qw[sl], w8 = w >> 8;
      r[4 * sl + 0] = dq2(w, 0x000F000Fu, kM0, s0, b0);
      r[4 * sl + 1] = dq2(w, 0x00F000F0u, kM4, s0, b0);
      r[4 * sl + 2] = dq2(w8, 0x000F000Fu, kM0, s8, b8);
      r[4 * sl + 3] = dq2(w8, 0x00F000F0u, kM4, s8, b8);
    }
  } else {
    const uint2 qv = *reinterpret_cast<const uint2*>(tile + lane * 8);
    const uint32_t qw[2] = {qv.x, qv.y};
#pragma unroll
    for (int wj = 0; wj < 2; ++wj) {
      const uint32_t w = qw[wj], w8 = w >> 8;
      r[8 * wj + 0] = dq2(w, 0x00030003u, kM0, s0, b0);
      r[8 * wj + 1] = dq2(w, 0x000C000Cu, kM2, s0, b0);
      r[8 * wj + 2] = dq2(w8, 0x00030003u, kM0, s8, b8);
      r[8 * wj + 3] = dq2(w8, 0x000C000Cu, kM2, s8, b8);
      r[8 * wj + 4] = dq2(w, 0x00300030u, kM4, s0, b0);
      r[8 * wj + 5] = dq2(w, 0x00C000C0u, kM6, s0, b0);
      r[8 * wj + 6] = dq2(w8, 0x00300030u, kM4, s8, b8);
      r[8 * wj + 7] = dq2(w8, 0x00C000C0u, kM6, s8, b8);
    }
  }
}

struct ItemInfo {
  int e, rb, pos0, ntok, npad;
};
__device__ __forceinline__ ItemInfo item_info(const TcArgs& p, int it) {
  const uint32_t item = p.items[it];
  const int s = (int)(item >> 16), tb = (int)(item & 0xFF);
  ItemInfo f;
  f.rb = (int)((item >> 8) & 0xFF);
  f.e = p.seg[s];
  f.pos0 = p.seg[p.S + s] + tb * kGemmTokens;
  f.ntok = min(kGemmTokens, p.seg[2 * p.S + s] - tb * kGemmTokens);
  f.npad = (f.ntok + 15) & ~15;
  return f;
}

struct XMaps {
  CUtensorMap m[kTcXMaps];  // box heights 16, 32, 48, 64
};

template <int BITS, bool GATE_UP>
__global__ void __launch_bounds__(kTcThreads, 1)
    bt_tc_gemm_kernel(const __grid_constant__ CUtensorMap wmap, const __grid_constant__ XMaps xmaps, TcArgs p) {
  using L = TcL<BITS>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (su32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = su32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // barriers: full[NS], empty[NS], afull[4], aempty[4], dfull[2], dempty[2], drain
  const uint32_t bar0 = sbase + L::BAR;
  auto full = [&](int s) { return bar0 + 8u * s; };
  auto empty = [&](int s) { return bar0 + 8u * (L::NS + s); };
  auto afull = [&](int b) { return bar0 + 8u * (2 * L::NS + b); };
  auto aempty = [&](int b) { return bar0 + 8u * (2 * L::NS + kTcABufs + b); };
  auto dfull = [&](int b) { return bar0 + 8u * (2 * L::NS + 2 * kTcABufs + b); };
  auto dempty = [&](int b) { return bar0 + 8u * (2 * L::NS + 2 * kTcABufs + 2 + b); };
  const uint32_t drain = bar0 + 8u * (2 * L::NS + 2 * kTcABufs + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::BAR + 8 * (2 * L::NS + 2 * kTcABufs + 5));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < L::NS; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);
    }
    for (int b = 0; b < kTcABufs; ++b) {
      mbar_init(afull(b), 4);
      mbar_init(aempty(b), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(dfull(b), kTcIssuers);
      mbar_init(dempty(b), 4);
    }
    mbar_init(drain, kTcIssuers);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(su32(tmem_slot)),
                 "r"(kTcTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int n_items = *p.n_items;
  auto fail = [&]() {
    if (!*abort_flag) atomicOr(p.status, kStatusTimeoutTc);
    *abort_flag = 1;
  };

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      uint32_t c = 0;
      bool ok = true;
      for (int it = blockIdx.x; ok && it < n_items; it += gridDim.x) {
        const ItemInfo f = item_info(p, it);
        const uint32_t bytes = (uint32_t)L::CODES + (uint32_t)f.npad * 256u;
        for (int kc = 0; kc < p.k_chunks; ++kc, ++c) {
          const int s = (int)(c % L::NS);
          const uint32_t ph = (c / L::NS) & 1u;
          if (!mbar_wait(empty(s), ph ^ 1u, abort_flag)) {
            fail();
            ok = false;
            break;
          }
          const uint32_t st = sbase + (uint32_t)s * L::STAGE;
          mbar_expect_tx(full(s), bytes);
          tma_3d(st + kTcBBytes, &wmap, kc * 2 * L::TB / 8, f.rb * 8, f.e, full(s));
          // X rows pos0 .. pos0 + n' - 1, 64-column blocks 2kc and 2kc + 1: [half][n'][128 B]
          tma_3d(st, &xmaps.m[f.npad / 16 - 1], 0, f.pos0, 2 * kc, full(s));
        }
      }
      // copies still in flight land before the block exits
      const uint32_t c0 = c > (uint32_t)L::NS ? c - L::NS : 0u;
      for (uint32_t k = c0; k < c; ++k) mbar_wait(full((int)(k % L::NS)), (k / L::NS) & 1u, nullptr);
    }
  } else if (warp == 1 || warp == 14) {
    // ---------------------------------------------------------------- MMA issuers
    // Everything between two MMAs is a constant offset: per chunk one
    // descriptor add and eight unrolled MMAs.  The ring's full barrier was
    // waited on by the dequantisers whose A-buffer barrier this lane waits on.
    if (lane == 0) {
      const int j = warp == 1 ? 0 : 1;
      const uint64_t bdesc0 = sw128_desc(sbase);
      uint32_t c = 0, ii = 0;
      bool ok = true;
      int it = blockIdx.x;
      ItemInfo f = it < n_items ? item_info(p, it) : ItemInfo{};
      for (; ok && it < n_items; it += gridDim.x, ++ii) {
        const int nit = it + (int)gridDim.x;
        const ItemInfo nf = nit < n_items ? item_info(p, nit) : f;  // loads in flight during this item
        const int d = (int)(ii & 1u);
        if (!mbar_wait(dempty(d), ((ii >> 1) & 1u) ^ 1u, abort_flag)) {
          fail();
          break;
        }
        tc_fence_after();
        const uint32_t idesc = f16_idesc(f.npad);
        const uint32_t dcol = tmem + (uint32_t)(d * kTcDCols + j * kGemmTokens);
        for (int kc = 0; kc < p.k_chunks; ++kc, ++c) {
          if ((kc & 1) != j) continue;
          const int s = (int)(c % L::NS), ab = (int)(c % kTcABufs);
          if (!mbar_wait(afull(ab), (c / kTcABufs) & 1u, abort_flag)) {
            fail();
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t bd = bdesc0 + (uint64_t)((uint32_t)s * (uint32_t)(L::STAGE >> 4));
          const uint32_t ad = tmem + (uint32_t)(kTcACol0 + ab * 64);
          // K step ks: A columns +8, B +32 bytes inside a 64-column half, +n' rows of
          // 128 bytes across halves
          tc_mma(dcol, ad, bd, idesc, kc > 1 ? 1u : 0u);
#pragma unroll
          for (int ks = 1; ks < 4; ++ks) tc_mma(dcol, ad + 8u * ks, bd + (uint64_t)(ks * 2), idesc, 1u);
          const uint64_t bd1 = bd + (uint64_t)(f.npad * 8);
#pragma unroll
          for (int ks = 4; ks < 8; ++ks) tc_mma(dcol, ad + 8u * ks, bd1 + (uint64_t)((ks - 4) * 2), idesc, 1u);
          tc_commit(empty(s));
          tc_commit(aempty(ab));
        }
        if (ok) tc_commit(dfull(d));
        f = nf;
      }
      // all issued tensor-core work completes before tensor memory is freed
      tc_commit(drain);
      mbar_wait(drain, 0, nullptr);
    }
  } else if (warp < 10) {
    // ---------------------------------------------------------------- dequantisers
    const int grp = (warp - 2) >> 2, q = warp & 3;
    uint32_t c = 0;
    bool ok = true;
    for (int it = blockIdx.x; ok && it < n_items; it += gridDim.x) {
      for (int kc = 0; kc < p.k_chunks; ++kc, ++c) {
        if ((int)(c & 1u) != grp) continue;
        const int s = (int)(c % L::NS), ab = (int)(c % kTcABufs);
        const bool got = mbar_wait(full(s), (c / L::NS) & 1u, abort_flag) &&
                         mbar_wait(aempty(ab), ((c / kTcABufs) & 1u) ^ 1u, abort_flag);
        if (!__all_sync(0xffffffffu, got)) {  // the tensor-memory stores below need the whole warp
          if (lane == 0) fail();
          ok = false;
          break;
        }
        tc_fence_after();
        const uint8_t* codes = smem + (size_t)s * L::STAGE + kTcBBytes;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int band = 2 * q + h;
#pragma unroll
          for (int tt = 0; tt < 2; ++tt) {
            uint32_t r[16];
            dequant_tile<BITS>(codes + (band * 2 + tt) * L::TB, lane, r);
            const uint32_t taddr =
                tmem + ((uint32_t)(32 * q + 16 * h) << 16) + (uint32_t)(kTcACol0 + ab * 64 + tt * 32);
            tmem_st16x256x4(taddr, r);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(afull(ab));
      }
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int q = warp & 3;
    uint32_t ii = 0;
    for (int it = blockIdx.x; it < n_items; it += gridDim.x, ++ii) {
      const ItemInfo f = item_info(p, it);
      const int d = (int)(ii & 1u);
      if (!__all_sync(0xffffffffu, mbar_wait(dfull(d), (ii >> 1) & 1u, abort_flag))) {
        if (lane == 0) fail();
        break;
      }
      tc_fence_after();
      const uint32_t dcol = tmem + (uint32_t)(d * kTcDCols);
      const bool two = p.k_chunks > 1;  // the second issuer's accumulator holds chunks 1, 3, ...
      auto sum2 = [&](uint32_t (&a)[32], const uint32_t (&b)[32]) {
#pragma unroll
        for (int k = 0; k < 32; ++k) a[k] = __float_as_uint(__uint_as_float(a[k]) + __uint_as_float(b[k]));
      };
      if constexpr (GATE_UP) {
        // lane 4g+t: gate row j (tensor-memory lane 16*band + g) and its up row
        // (lane 16*band + 8 + g) for positions 8i + 2t, 8i + 2t + 1
        const int g = lane >> 2, t = lane & 3;
#pragma unroll 1
        for (int h = 0; h < 2; ++h) {
          uint32_t r[32], r1[32];
          const uint32_t ta = dcol + ((uint32_t)(32 * q + 16 * h) << 16);
          tmem_ld16x256x8(ta, r);
          if (two) tmem_ld16x256x8(ta + (uint32_t)kGemmTokens, r1);
          tmem_wait_ld();
          if (two) sum2(r, r1);
          const int j = f.rb * 64 + (2 * q + h) * 8 + g;
          if (j >= p.ldo) continue;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
#pragma unroll
            for (int e2 = 0; e2 < 2; ++e2) {
              const int n = 8 * i + 2 * t + e2;
              if (n >= f.ntok) continue;
              const float sc = p.bscale[f.pos0 + n];
              const float gv = __uint_as_float(r[4 * i + e2]) * sc, uv = __uint_as_float(r[4 * i + 2 + e2]) * sc;
              p.out[(size_t)(f.pos0 + n) * p.ldo + j] = gv / (1.0f + expf(-gv)) * uv;
            }
          }
        }
      } else {
        // lane l of warp q: output row 128*rb + 32*q + l, 32 positions per pass
        const int row = f.rb * 128 + 32 * q + lane;
#pragma unroll 1
        for (int h = 0; h < 2; ++h) {
          uint32_t r[32], r1[32];
          const uint32_t ta = dcol + ((uint32_t)(32 * q) << 16) + (uint32_t)(32 * h);
          tmem_ld32x32x32(ta, r);
          if (two) tmem_ld32x32x32(ta + (uint32_t)kGemmTokens, r1);
          tmem_wait_ld();
          if (two) sum2(r, r1);
          if (row < p.rows) {
#pragma unroll
            for (int n = 0; n < 32; ++n) {
              if (32 * h + n >= f.ntok) break;
              p.out[(size_t)(f.pos0 + 32 * h + n) * p.ldo + row] = __uint_as_float(r[n]) * p.bscale[f.pos0 + 32 * h + n];
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(dempty(d));
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTcTmemCols) : "memory");
  }
}

// ------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }
  return fn;
}

template <int BITS, bool GATE_UP>
int launch_one(const TmaDesc& w, const TmaDesc* x, const TcArgs& a, int n_sm, cudaStream_t st) {
  using L = TcL<BITS>;
  cudaError_t e = cudaFuncSetAttribute(bt_tc_gemm_kernel<BITS, GATE_UP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       L::SMEM);
  if (e != cudaSuccess) return (int)e;
  CUtensorMap wm;
  XMaps xm;
  static_assert(sizeof(TmaDesc) == sizeof(CUtensorMap), "tensor map size");
  memcpy(&wm, w.bytes, sizeof wm);
  for (int k = 0; k < kTcXMaps; ++k) memcpy(&xm.m[k], x[k].bytes, sizeof(CUtensorMap));
  bt_tc_gemm_kernel<BITS, GATE_UP><<<n_sm, kTcThreads, L::SMEM, st>>>(wm, xm, a);
  return (int)cudaGetLastError();
}

}  // namespace

int tc_encode_weight_map(const uint8_t* matrix0, int64_t blob_bytes, int n_blobs, int rows, int cols, int bits,
                         TmaDesc* out) {
  auto fn = encode_fn();
  if (fn == nullptr) return (int)cudaErrorNotSupported;
  const int tb = tile_bytes(bits);
  const cuuint64_t band_bytes = (cuuint64_t)(cols / kGroup) * tb;
  const cuuint64_t dims[3] = {band_bytes / 8, (cuuint64_t)(rows / 16), (cuuint64_t)n_blobs};
  const cuuint64_t strides[2] = {band_bytes, (cuuint64_t)blob_bytes};
  const cuuint32_t box[3] = {(cuuint32_t)(2 * tb / 8), 8u, 1u};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  CUtensorMap m;
  const CUresult r = fn(&m, CU_TENSOR_MAP_DATA_TYPE_UINT64, 3, const_cast<uint8_t*>(matrix0), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return (int)cudaErrorInvalidValue;
  memcpy(out->bytes, &m, sizeof m);
  return 0;
}

int tc_encode_token_maps(const uint16_t* base, int cols, int rows, TmaDesc* out) {
  auto fn = encode_fn();
  if (fn == nullptr) return (int)cudaErrorNotSupported;
  // (64 columns, rows, 64-column blocks) view of the row-major [rows][cols] matrix
  const cuuint64_t dims[3] = {64u, (cuuint64_t)rows, (cuuint64_t)(cols / 64)};
  const cuuint64_t strides[2] = {(cuuint64_t)cols * 2, 128u};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  for (int k = 0; k < kTcXMaps; ++k) {
    const cuuint32_t box[3] = {64u, (cuuint32_t)(16 * (k + 1)), 2u};
    CUtensorMap m;
    const CUresult r = fn(&m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<uint16_t*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return (int)cudaErrorInvalidValue;
    memcpy(out[k].bytes, &m, sizeof m);
  }
  return 0;
}

int launch_tc_gemm(int bits, bool gate_up, const TmaDesc& wmap, const TmaDesc* xmaps, const TcArgs& a, int n_sm,
                   void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (bits == 4)
    return gate_up ? launch_one<4, true>(wmap, xmaps, a, n_sm, st) : launch_one<4, false>(wmap, xmaps, a, n_sm, st);
  return gate_up ? launch_one<2, true>(wmap, xmaps, a, n_sm, st) : launch_one<2, false>(wmap, xmaps, a, n_sm, st);
}

}  // namespace fmoe
