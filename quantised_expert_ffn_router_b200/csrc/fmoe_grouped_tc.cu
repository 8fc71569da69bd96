// fmoe_grouped_tc.cu -- the grouped per-expert GEMM of the batched layer on
// the 5th-generation tensor cores (tcgen05, tensor memory, TMA).
//
// A work item (from the permute step) is one expert, one block of 128 matrix
// rows and up to 64 positions:  C[128 x n] = W[128 x K] X[n x K]^T  with W the
// packed b-bit tiles of the expert (w = q*s + b per 64-column group, the
// affine dequantisation the Flash-MoE pages apply in their FMA kernel: "Flash-MoE:
// Running a 400 Billion Parameter Model on a MacBook", section "The
// Architecture") and X an fp16 copy of the positions' inputs, each row scaled
// by a power of two (bt_prep_kernel, fmoe_batched.cu).
//
// The contraction is taken in its factored form, group by group:
//   C[j][n] = sum_g  s[j][g] * (sum_{i in g} q[j][i] X[n][i])  +  b[j][g] * S[n][g]
// The tensor core multiplies the exact integer codes q (fp16) by X and sums
// each 64-column group into its own fp32 accumulator P_g; the epilogue warps
// scale P_g by the group's bf16 scale and add the bias times the group sum
// S[n][g] of X (computed by the prep kernel), in fp32.  Scales and biases
// therefore never pass through fp16, and the only rounding before the fp32
// accumulation is that of X.
//
// One persistent block per SM, 15 warps:
//   warp 0      TMA producer.  Per 128-column chunk (one ring stage, two
//               groups): one 3-D copy of the item's 8 bands x 2 packed tiles,
//               one of the n' = ceil(n/16)*16 rows x 2 x 64 columns of X
//               (128-byte swizzle) and one of the n' rows of group sums.
//   warps 1, 14 MMA issuers (warp 1 also allocates tensor memory): one lane
//               each, even / odd chunks, each into its own pair of group
//               accumulators (A from tensor memory, B from shared memory, fp32
//               in tensor memory, M=128, N=n', 4 x K=16 per group).  A thread
//               issues one tcgen05.mma per ~55 cycles however small N is, so two
//               issuers halve the time the tensor core needs per chunk.
//   warps 2-5   code warps: a warp turns two bands (32 rows) x 2 tiles of every
//               chunk into exact fp16 codes and stores them into the A buffer
//               with tcgen05.st.16x256b, whose thread layout is the mma.sync
//               fragment layout the packed tile is stored in (lane 4g+t: rows g
//               and g+8, columns 2t, 2t+1 | 2t+8, 2t+9).
//   warps 6-13  epilogue, two sets of four: one matrix row per thread (its
//               tensor-memory lane), positions 0-31 (set 0) or 32-63 (set 1).
//               Per chunk: copy the two group accumulators' columns into
//               registers and release them at once (so the issuer can refill
//               them while the arithmetic runs), then fold them with the row's
//               scales and biases (from the packed tiles in the stage) and the
//               group sums into the row's fp32 sums, and release the stage.
//               Per item: scale each column back by its position's power of
//               two and write a = silu(g)*u (gate/up; the up row is 8 lanes
//               below its gate row) or y (down).
//
// K order.  The 16x256b store puts a lane's fragment columns {2t, 2t+1, 2t+8,
// 2t+9} of a 16-column slice at tensor-memory positions 4t..4t+3, so within
// every 16 columns A holds column pi(p) = 2*(p/4) + p%2 + 8*((p/2)%2) at
// position p.  The prep kernel stores X in the same order; the contraction over
// a group does not depend on the order.
//
// Exact codes.  A code at bit offset o of a 32-bit word is moved into the
// mantissa of an fp16 constant whose unit in the last place is 2^-o
// (1024, 256, 64, 16 for o = 0, 2, 4, 6); subtracting the constant leaves the
// code exactly.
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
constexpr int kTcSBytes = kGemmTokens * 16;       // group sums in a stage: up to 64 rows x 4 floats
constexpr int kTcABufs = 4;                       // A buffers in tensor memory (64 columns each)
constexpr int kTcXMaps = kGemmTokens / 16;          // input tensor maps, one per box height
constexpr int kTcIssuers = 2;                     // MMA-issuing threads, one accumulator pair each
constexpr int kTcEpiWarp0 = 6;                    // warps 2-5 turn codes into fp16, warps 6-13 are the epilogue
constexpr int kTcEpiWarps = 8;
constexpr int kTcPCols = 2 * kGemmTokens;         // tensor-memory columns of one issuer's group accumulators
constexpr int kTcPSlots = 4;                      // accumulator pairs per issuer at n' = 16 (64 / n' in general)
constexpr int kTcACol0 = kTcIssuers * kTcPCols;   // first A column
constexpr uint32_t kTcTmemCols = 512;
constexpr uint64_t kTcWaitNs = 500ull * 1000 * 1000;  // bounded waits: 0.5 s
static_assert(kTcACol0 + kTcABufs * 64 <= (int)kTcTmemCols, "tensor memory plan");

template <int BITS>
struct TcL {
  static constexpr int TB = 16 * kGroup * BITS / 8 + 64;  // packed tile bytes
  static constexpr int CB = 16 * kGroup * BITS / 8;       // code bytes of a tile (scales/biases follow)
  static constexpr int CODES = 8 * 2 * TB;               // 8 bands x 2 tiles
  static constexpr int SUMS = kTcBBytes + CODES;         // group sums, after X and the codes
  static constexpr int STAGE = SUMS + kTcSBytes;         // multiple of 1024
  static constexpr int NS = BITS == 4 ? 8 : 10;
  static constexpr int BAR = NS * STAGE;                 // barriers after the ring
  static constexpr int SMEM = BAR + 512 + 1024;          // + alignment slack
  static_assert(STAGE % 1024 == 0 && SUMS % 128 == 0, "stage alignment");
  static_assert(SMEM <= 232448, "shared memory");
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
__device__ __forceinline__ void tmem_ld32x32x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// ------------------------------------------------------------------ exact codes
__device__ __forceinline__ uint32_t lop_and_or(uint32_t a, uint32_t mask, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(mask), "r"(c));
  return d;
}
// The two codes of `w` under `mask` as an exact fp16 pair; `magic` is the fp16
// pair whose last mantissa place is the mask's lowest bit.
__device__ __forceinline__ uint32_t code2(uint32_t w, uint32_t mask, uint32_t magic) {
  uint32_t q;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(q) : "r"(lop_and_or(w, mask, magic)), "r"(magic));
  return q;
}
constexpr uint32_t kM0 = 0x64006400u;  // 1024: codes at bit 0
constexpr uint32_t kM2 = 0x5C005C00u;  // 256:  codes at bit 2
constexpr uint32_t kM4 = 0x54005400u;  // 64:   codes at bit 4
constexpr uint32_t kM6 = 0x4C004C00u;  // 16:   codes at bit 6

// The 16 registers tcgen05.st.16x256b.x4 stores for one packed tile (4 slices
// of 16 columns): per slice {row g cols 2t,2t+1; row g cols 2t+8,2t+9; row g+8
// cols 2t,2t+1; row g+8 cols 2t+8,2t+9}, as exact fp16 codes.
template <int BITS>
__device__ __forceinline__ void code_tile(const uint8_t* tile, int lane, uint32_t (&r)[16]) {
  if constexpr (BITS == 4) {
    const uint4 qv = *reinterpret_cast<const uint4*>(tile + lane * 16);
    const uint32_t qw[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
    for (int sl = 0; sl < 4; ++sl) {
      const uint32_t w = qw[sl], w8 = w >> 8;
      r[4 * sl + 0] = code2(w, 0x000F000Fu, kM0);
      r[4 * sl + 1] = code2(w, 0x00F000F0u, kM4);
      r[4 * sl + 2] = code2(w8, 0x000F000Fu, kM0);
      r[4 * sl + 3] = code2(w8, 0x00F000F0u, kM4);
    }
  } else {
    const uint2 qv = *reinterpret_cast<const uint2*>(tile + lane * 8);
    const uint32_t qw[2] = {qv.x, qv.y};
#pragma unroll
    for (int wj = 0; wj < 2; ++wj) {
      const uint32_t w = qw[wj], w8 = w >> 8;
      r[8 * wj + 0] = code2(w, 0x00030003u, kM0);
      r[8 * wj + 1] = code2(w, 0x000C000Cu, kM2);
      r[8 * wj + 2] = code2(w8, 0x00030003u, kM0);
      r[8 * wj + 3] = code2(w8, 0x000C000Cu, kM2);
      r[8 * wj + 4] = code2(w, 0x00300030u, kM4);
      r[8 * wj + 5] = code2(w, 0x00C000C0u, kM6);
      r[8 * wj + 6] = code2(w8, 0x00300030u, kM4);
      r[8 * wj + 7] = code2(w8, 0x00C000C0u, kM6);
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

// Accumulator pairs per issuer for an item of n' positions: its kTcPCols
// columns hold 64 / n' pairs (1, 2 or 4) of two n'-column group accumulators.
__device__ __forceinline__ int pair_slots(int npad) { return npad <= 16 ? 4 : npad <= 32 ? 2 : 1; }

struct XMaps {
  CUtensorMap m[kTcXMaps];  // box heights 16, 32, 48, 64
};

template <int BITS, bool GATE_UP>
__global__ void __launch_bounds__(kTcThreads, 1)
    bt_tc_gemm_kernel(const __grid_constant__ CUtensorMap wmap, const __grid_constant__ XMaps xmaps,
                      const __grid_constant__ XMaps smaps, TcArgs p) {
  using L = TcL<BITS>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (su32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = su32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // barriers: full[NS], empty[NS], afull[4], aempty[4], pfull[2][4], pempty[2][4], drain
  constexpr int kPB = kTcIssuers * kTcPSlots;
  const uint32_t bar0 = sbase + L::BAR;
  auto full = [&](int s) { return bar0 + 8u * s; };
  auto empty = [&](int s) { return bar0 + 8u * (L::NS + s); };
  auto afull = [&](int b) { return bar0 + 8u * (2 * L::NS + b); };
  auto aempty = [&](int b) { return bar0 + 8u * (2 * L::NS + kTcABufs + b); };
  auto pfull = [&](int j, int k) { return bar0 + 8u * (2 * L::NS + 2 * kTcABufs + j * kTcPSlots + k); };
  auto pempty = [&](int j, int k) { return bar0 + 8u * (2 * L::NS + 2 * kTcABufs + kPB + j * kTcPSlots + k); };
  const uint32_t drain = bar0 + 8u * (2 * L::NS + 2 * kTcABufs + 2 * kPB);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::BAR + 8 * (2 * L::NS + 2 * kTcABufs + 2 * kPB + 1));
  static_assert(8 * (2 * L::NS + 2 * kTcABufs + 2 * kPB + 1) + 8 <= 512, "barrier area");
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < L::NS; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), kTcEpiWarps);  // released by the epilogue warps (after the MMAs that read it)
    }
    for (int b = 0; b < kTcABufs; ++b) {
      mbar_init(afull(b), 4);
      mbar_init(aempty(b), 1);
    }
    for (int j = 0; j < kTcIssuers; ++j)
      for (int k = 0; k < kTcPSlots; ++k) {
        mbar_init(pfull(j, k), 1);
        mbar_init(pempty(j, k), kTcEpiWarps);
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
        const uint32_t bytes = (uint32_t)L::CODES + (uint32_t)f.npad * (256u + 16u);
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
          // their group sums: [n'][4 floats] (groups 2kc, 2kc + 1, two unused)
          tma_3d(st + L::SUMS, &smaps.m[f.npad / 16 - 1], 0, f.pos0, kc, full(s));
        }
      }
      // copies still in flight land before the block exits
      const uint32_t c0 = c > (uint32_t)L::NS ? c - L::NS : 0u;
      for (uint32_t k = c0; k < c; ++k) mbar_wait(full((int)(k % L::NS)), (k / L::NS) & 1u, nullptr);
    }
  } else if (warp == 1 || warp == 14) {
    // ---------------------------------------------------------------- MMA issuers
    // Issuer j takes the chunks kc = j mod 2 of every item, chunk kc into
    // accumulator pair (kc / 2) mod pair_slots(n') of its column range, once
    // the epilogue has copied that pair's previous contents out.  Before an
    // item the issuer waits for every pair it has used, since the pairs of
    // items of different n' overlap.  The ring's full barrier was waited on by
    // the code warps whose A-buffer barrier this lane waits on.
    if (lane == 0) {
      const int j = warp == 1 ? 0 : 1;
      const uint64_t bdesc0 = sw128_desc(sbase);
      const uint32_t pbase = tmem + (uint32_t)(j * kTcPCols);
      uint32_t c = 0, ebits = 0;  // ebits bit k: parity of pair k's uses so far
      bool ok = true;
      for (int it = blockIdx.x; ok && it < n_items; it += gridDim.x) {
        const ItemInfo f = item_info(p, it);
        const uint32_t idesc = f16_idesc(f.npad);
        const int slots = pair_slots(f.npad), width = kTcPCols / slots;
        for (int k = 0; ok && k < kTcPSlots; ++k)
          if (!mbar_wait(pempty(j, k), ((ebits >> k) & 1u) ^ 1u, abort_flag)) {
            fail();
            ok = false;
          }
        for (int kc = 0; ok && kc < p.k_chunks; ++kc, ++c) {
          if ((kc & 1) != j) continue;
          const int s = (int)(c % L::NS), ab = (int)(c % kTcABufs), k = (kc >> 1) % slots;
          if (!mbar_wait(afull(ab), (c / kTcABufs) & 1u, abort_flag) ||
              !mbar_wait(pempty(j, k), ((ebits >> k) & 1u) ^ 1u, abort_flag)) {
            fail();
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t bd = bdesc0 + (uint64_t)((uint32_t)s * (uint32_t)(L::STAGE >> 4));
          const uint32_t ad = tmem + (uint32_t)(kTcACol0 + ab * 64);
          const uint32_t d0 = pbase + (uint32_t)(k * width), d1 = d0 + (uint32_t)(width / 2);
          // group 2kc: A columns 0..31 (K = 64), B the first 64-column half;
          // group 2kc + 1: A columns 32..63, B the second half (n' rows of 128 B on)
          tc_mma(d0, ad, bd, idesc, 0u);
#pragma unroll
          for (int ks = 1; ks < 4; ++ks) tc_mma(d0, ad + 8u * ks, bd + (uint64_t)(ks * 2), idesc, 1u);
          const uint64_t bd1 = bd + (uint64_t)(f.npad * 8);
          tc_mma(d1, ad + 32u, bd1, idesc, 0u);
#pragma unroll
          for (int ks = 5; ks < 8; ++ks) tc_mma(d1, ad + 8u * ks, bd1 + (uint64_t)((ks - 4) * 2), idesc, 1u);
          tc_commit(aempty(ab));
          tc_commit(pfull(j, k));
          ebits ^= 1u << k;
        }
      }
      // all issued tensor-core work completes before tensor memory is freed
      tc_commit(drain);
      mbar_wait(drain, 0, nullptr);
    }
  } else if (warp < kTcEpiWarp0) {
    // ---------------------------------------------------------------- code warps
    const int q = warp & 3;
    uint32_t c = 0;
    bool ok = true;
    for (int it = blockIdx.x; ok && it < n_items; it += gridDim.x) {
      for (int kc = 0; kc < p.k_chunks; ++kc, ++c) {
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
            code_tile<BITS>(codes + (band * 2 + tt) * L::TB, lane, r);
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
    // Thread = tensor-memory lane l = 32q + lane = row 16*band + rho of the
    // item's packed bands; its scale and bias of group tt sit in tile
    // (band, tt) of the stage at byte 8*(rho % 8) + 4*(rho / 8) after the codes.
    // Set h takes positions 32h .. 32h + 31.
    const int q = warp & 3, h = (warp - kTcEpiWarp0) >> 2, l = 32 * q + lane, band = l >> 4, rho = l & 15;
    const uint32_t sb_off = (uint32_t)(kTcBBytes + band * 2 * L::TB + L::CB + 8 * (rho & 7) + 4 * (rho >> 3));
    const uint32_t tlane = (uint32_t)(32 * q) << 16;
    constexpr int kHalf = kGemmTokens / 2;
    uint32_t c = 0, fbits = 0;  // fbits bit 4j + k: parity of issuer j's pair k completions seen
    bool ok = true;
    for (int it = blockIdx.x; ok && it < n_items; it += gridDim.x) {
      const ItemInfo f = item_info(p, it);
      const int nb = min(2, max(0, (f.npad - kHalf * h) / 16));  // 16-column blocks of this set (uniform)
      const int slots = pair_slots(f.npad), width = kTcPCols / slots;
      float acc[kHalf];
#pragma unroll
      for (int n = 0; n < kHalf; ++n) acc[n] = 0.f;
      for (int kc = 0; kc < p.k_chunks; ++kc, ++c) {
        const int j = kc & 1, s = (int)(c % L::NS), k = (kc >> 1) % slots, fb = 4 * j + k;
        const bool got = mbar_wait(pfull(j, k), (fbits >> fb) & 1u, abort_flag) &&
                         mbar_wait(full(s), (c / L::NS) & 1u, abort_flag);
        if (!__all_sync(0xffffffffu, got)) {  // the tensor-memory loads below need the whole warp
          if (lane == 0) fail();
          ok = false;
          break;
        }
        tc_fence_after();
        const uint8_t* stg = smem + (size_t)s * L::STAGE;
        const uint32_t sb0 = *reinterpret_cast<const uint32_t*>(stg + sb_off);
        const uint32_t sb1 = *reinterpret_cast<const uint32_t*>(stg + sb_off + L::TB);
        const float s0 = __uint_as_float(sb0 << 16), b0 = __uint_as_float(sb0 & 0xFFFF0000u);
        const float s1 = __uint_as_float(sb1 << 16), b1 = __uint_as_float(sb1 & 0xFFFF0000u);
        const float2* gs = reinterpret_cast<const float2*>(stg + L::SUMS) + 2 * kHalf * h;  // [n][4] floats
        // one 16-column block of both groups at a time; the accumulators are
        // released as soon as the last block has been copied out
        const uint32_t pcol = tmem + tlane + (uint32_t)(j * kTcPCols + k * width + kHalf * h);
#pragma unroll
        for (int b = 0; b < 2; ++b) {
          if (b < nb) {  // uniform across the warp
            uint32_t r0[16], r1[16];
            tmem_ld32x32x16(pcol + (uint32_t)(16 * b), r0);
            tmem_ld32x32x16(pcol + (uint32_t)(width / 2 + 16 * b), r1);
            tmem_wait_ld();
            if (b == nb - 1) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(pempty(j, k));
            }
#pragma unroll
            for (int n = 0; n < 16; ++n) {
              const float2 g = gs[2 * (16 * b + n)];
              float a = fmaf(s0, __uint_as_float(r0[n]), acc[16 * b + n]);
              a = fmaf(s1, __uint_as_float(r1[n]), a);
              acc[16 * b + n] = fmaf(b0, g.x, fmaf(b1, g.y, a));
            }
          }
        }
        if (nb == 0) {  // a set with no columns in this item still releases its share
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(pempty(j, k));
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty(s));
        fbits ^= 1u << fb;
      }
      if (!ok) break;
      if constexpr (GATE_UP) {
        // rho < 8: gate row j = 64*rb + 8*band + rho; its up row is lane + 8
        const int jrow = f.rb * 64 + band * 8 + (rho & 7);
        const bool writer = rho < 8 && jrow < p.ldo;
#pragma unroll
        for (int n = 0; n < kHalf; ++n) {
          const float uv = __shfl_down_sync(0xffffffffu, acc[n], 8);
          const int pn = kHalf * h + n;
          if (writer && pn < f.ntok) {
            const float sc = p.bscale[f.pos0 + pn];
            const float gv = acc[n] * sc;
            p.out[(size_t)(f.pos0 + pn) * p.ldo + jrow] = gv / (1.0f + expf(-gv)) * (uv * sc);
          }
        }
      } else {
        const int row = f.rb * 128 + l;
        if (row < p.rows) {
#pragma unroll
          for (int n = 0; n < kHalf; ++n) {
            const int pn = kHalf * h + n;
            if (pn < f.ntok) p.out[(size_t)(f.pos0 + pn) * p.ldo + row] = acc[n] * p.bscale[f.pos0 + pn];
          }
        }
      }
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
int launch_one(const TmaDesc& w, const TmaDesc* x, const TmaDesc* sums, const TcArgs& a, int n_sm, cudaStream_t st) {
  using L = TcL<BITS>;
  cudaError_t e = cudaFuncSetAttribute(bt_tc_gemm_kernel<BITS, GATE_UP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       L::SMEM);
  if (e != cudaSuccess) return (int)e;
  CUtensorMap wm;
  XMaps xm, sm;
  static_assert(sizeof(TmaDesc) == sizeof(CUtensorMap), "tensor map size");
  memcpy(&wm, w.bytes, sizeof wm);
  for (int k = 0; k < kTcXMaps; ++k) {
    memcpy(&xm.m[k], x[k].bytes, sizeof(CUtensorMap));
    memcpy(&sm.m[k], sums[k].bytes, sizeof(CUtensorMap));
  }
  bt_tc_gemm_kernel<BITS, GATE_UP><<<n_sm, kTcThreads, L::SMEM, st>>>(wm, xm, sm, a);
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

int tc_encode_sum_maps(const float* base, int chunks, int rows, TmaDesc* out) {
  auto fn = encode_fn();
  if (fn == nullptr) return (int)cudaErrorNotSupported;
  // [chunks][rows][4] floats: (4 floats, rows, chunks); boxes of 16..64 rows of one chunk
  const cuuint64_t dims[3] = {4u, (cuuint64_t)rows, (cuuint64_t)chunks};
  const cuuint64_t strides[2] = {16u, (cuuint64_t)rows * 16u};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  for (int k = 0; k < kTcXMaps; ++k) {
    const cuuint32_t box[3] = {4u, (cuuint32_t)(16 * (k + 1)), 1u};
    CUtensorMap m;
    const CUresult r = fn(&m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return (int)cudaErrorInvalidValue;
    memcpy(out[k].bytes, &m, sizeof m);
  }
  return 0;
}

int launch_tc_gemm(int bits, bool gate_up, const TmaDesc& wmap, const TmaDesc* xmaps, const TmaDesc* smaps,
                   const TcArgs& a, int n_sm, void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (bits == 4)
    return gate_up ? launch_one<4, true>(wmap, xmaps, smaps, a, n_sm, st)
                   : launch_one<4, false>(wmap, xmaps, smaps, a, n_sm, st);
  return gate_up ? launch_one<2, true>(wmap, xmaps, smaps, a, n_sm, st)
                 : launch_one<2, false>(wmap, xmaps, smaps, a, n_sm, st);
}

}  // namespace fmoe
