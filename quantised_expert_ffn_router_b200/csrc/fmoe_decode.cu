// fmoe_decode.cu -- fused single-token mixture-of-experts layer for sm_100a.
//
// One cooperative launch, one block per SM, runs the whole decode step that the
// Flash-MoE pages split over two GPU command buffers and the host (the Hysen
// Labs page "Flash-MoE: Running a 397B Parameter Model on a Laptop", section
// "How the SSD expert streaming pipeline works"): optional RMSNorm, router GEMV,
// softmax + top-K,
// the K routed and the shared SwiGLU experts with inline dequantisation, and the
// weighted combine into the residual.
//
// Work split.  Every block owns (a) router rows b, b+G, ..., (b) gate/up units
// (8 gate + 8 up rows over the full hidden width) u = b, b+G, ... striped over
// the flattened list [shared expert | routed expert 1 | ... | routed expert K],
// (c) output row blocks G-1-b, 2G-1-b, ... of every expert's down projection, so
// the combine is local and needs no atomics.  These become an ordered list of
// tasks of at most 16 tiles each (a router row, a 1024-column K-chunk of a
// unit, a down job).
//
// Roles.  One producer warp walks the list and streams each task's weights
// HBM -> shared memory with bulk-async (TMA) copies into a ring of stages
// (full/empty mbarriers); it also waits (bounded) for every block's router
// rows and runs softmax + top-K itself before the first task that needs a
// routed expert.  Fifteen consumer warps take tasks round-robin and never wait
// for each other: K-chunks of a unit are summed by whichever warp finishes
// last (shared-memory counter, fixed order), which writes a = silu(g)*u and
// publishes the unit's values as tagged words (plus a relaxed count that
// paces readers); a down job waits (bounded) for its expert's activations to
// be published by every block, turns them into fragments once per block and
// reduces its rows.
//
// Inner loop.  A tile is 16 rows x 64 columns (one quantisation group per
// row); its codes go into mma.sync fragments exactly (lop3 into the mantissa
// of 1024, sub.f16x2), the input is a power-of-two-scaled fp16 fragment, the
// tensor pipe accumulates sum(q*x) in fp32, and s*sum(q*x) + b*sum(x) folds
// in the group's scale and bias.
// Every wait is bounded by %globaltimer; on a timeout the block records a status
// bit, drains its outstanding copies and leaves.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "fmoe_internal.h"

namespace fmoe {
namespace {

// ------------------------------------------------------------------ PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ void tma_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}
// smem -> global bulk copy (one bulk group per call), and waits for the
// issuing thread's groups: until their sources are read / until complete.
__device__ __forceinline__ void bulk_store(void* dst, uint32_t src, uint32_t bytes) {
  asm volatile("fence.proxy.async.shared::cta;\n"
               "cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;\n"
               "cp.async.bulk.commit_group;" ::"l"(dst),
               "r"(src), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ uint64_t gtimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
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
__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  // not volatile: the result is the only effect, so independent tiles' chains
  // may be interleaved by the compiler
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ float bf16lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }
__device__ __forceinline__ float bf16f(uint16_t v) { return __uint_as_float((uint32_t)v << 16); }
__device__ __forceinline__ uint16_t f2bf16(float f) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}
// 2^k for k in [-126, 127] as an exact float.
__device__ __forceinline__ float exp2i(int k) { return __uint_as_float((uint32_t)(k + 127) << 23); }

constexpr uint32_t kMagic = 0x64006400u;  // fp16 pair (1024, 1024)

// One 16-column slice of a 4-bit tile: word w -> four fragment registers.
__device__ __forceinline__ void mma_slice4(float (&c)[4], uint32_t w, uint2 b) {
  uint32_t w8 = w >> 8;
  uint32_t a0 = hsub2(lop_and_or(w, 0x000F000Fu, kMagic), kMagic);
  uint32_t a1 = hsub2(lop_and_or(w8, 0x000F000Fu, kMagic), kMagic);
  uint32_t a2 = hsub2(lop_and_or(w, 0x00F000F0u, kMagic), kMagic);
  uint32_t a3 = hsub2(lop_and_or(w8, 0x00F000F0u, kMagic), kMagic);
  mma16816(c, a0, a1, a2, a3, b.x, b.y);
}
// Two 16-column slices of a 2-bit tile from one word.
__device__ __forceinline__ void mma_word2(float (&c)[4], uint32_t w, uint2 be, uint2 bo) {
  uint32_t w8 = w >> 8;
  uint32_t a0 = hsub2(lop_and_or(w, 0x00030003u, kMagic), kMagic);
  uint32_t a1 = hsub2(lop_and_or(w8, 0x00030003u, kMagic), kMagic);
  uint32_t a2 = hsub2(lop_and_or(w, 0x000C000Cu, kMagic), kMagic);
  uint32_t a3 = hsub2(lop_and_or(w8, 0x000C000Cu, kMagic), kMagic);
  mma16816(c, a0, a1, a2, a3, be.x, be.y);
  a0 = hsub2(lop_and_or(w, 0x00300030u, kMagic), kMagic);
  a1 = hsub2(lop_and_or(w8, 0x00300030u, kMagic), kMagic);
  a2 = hsub2(lop_and_or(w, 0x00C000C0u, kMagic), kMagic);
  a3 = hsub2(lop_and_or(w8, 0x00C000C0u, kMagic), kMagic);
  mma16816(c, a0, a1, a2, a3, bo.x, bo.y);
}

// Dot products of one tile (16 rows x 64 columns = one quantisation group per
// row) with the prepared input slice; adds s*sum(q*x) + b*sum(x) for rows g and
// g+8 into acc0 / acc1.
template <int BITS>
__device__ __forceinline__ void tile_dot(const uint8_t* tile, const uint2 (&bf)[4], float2 info, int lane,
                                         float& acc0, float& acc1) {
  float c[4] = {0.f, 0.f, 0.f, 0.f};
  constexpr int CB = 16 * kGroup * BITS / 8;
  if (BITS == 4) {
    uint4 q = *reinterpret_cast<const uint4*>(tile + lane * 16);
    mma_slice4(c, q.x, bf[0]);
    mma_slice4(c, q.y, bf[1]);
    mma_slice4(c, q.z, bf[2]);
    mma_slice4(c, q.w, bf[3]);
  } else {
    uint2 q = *reinterpret_cast<const uint2*>(tile + lane * 8);
    mma_word2(c, q.x, bf[0], bf[1]);
    mma_word2(c, q.y, bf[2], bf[3]);
  }
  uint2 sb = *reinterpret_cast<const uint2*>(tile + CB + (lane >> 2) * 8);
  acc0 = fmaf(bf16lo(sb.x) * info.x, c[0], fmaf(bf16hi(sb.x), info.y, acc0));
  acc1 = fmaf(bf16lo(sb.y) * info.x, c[2], fmaf(bf16hi(sb.y), info.y, acc1));
}


// Publishes {value, tag} with an atomic exchange: atomics are performed at L2,
// so other SMs see the word within about a microsecond, whereas plain stores
// were measured to linger for several microseconds under load.
__device__ __forceinline__ void st_tagged(uint64_t* p, float v, uint32_t tag) {
  const uint64_t w = (uint64_t)__float_as_uint(v) | ((uint64_t)tag << 32);
  asm volatile("{ .reg .b64 old; atom.relaxed.gpu.global.exch.b64 old, [%0], %1; }" ::"l"(p), "l"(w) : "memory");
}
__device__ __forceinline__ uint64_t ld_tagged(const uint64_t* p) {
  uint64_t w;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(w) : "l"(p) : "memory");
  return w;
}
// Two tagged words (16-byte aligned); volatile so a polling loop re-reads them.
__device__ __forceinline__ ulonglong2 ld_tagged2(const uint64_t* p) {
  ulonglong2 w;
  asm volatile("ld.relaxed.gpu.global.v2.u64 {%0, %1}, [%2];" : "=l"(w.x), "=l"(w.y) : "l"(p) : "memory");
  return w;
}
__device__ __forceinline__ float tagged_value(uint64_t w) { return __uint_as_float((uint32_t)w); }
__device__ __forceinline__ uint32_t tagged_tag(uint64_t w) { return (uint32_t)(w >> 32); }

__device__ __forceinline__ void red_relaxed_add(uint32_t* p, uint32_t v) {
  asm volatile("red.relaxed.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t ld_relaxed(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
// Bounded spin until a published count reaches its target (a hint only: the
// values it counts carry their own tags and are re-checked by the reader).
__device__ __forceinline__ bool wait_count(const uint32_t* p, uint32_t target, uint64_t limit,
                                           const volatile int* abort_flag) {
  const uint64_t t0 = gtimer();
  for (uint32_t it = 0;; ++it) {
    if (ld_relaxed(p) >= target) return true;
    if ((it & 7) == 7 && (*abort_flag || gtimer() - t0 > limit)) return false;
    __nanosleep(128);  // leave issue slots to warps with work
  }
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// fp16 B fragments of NG 64-value groups G0..G0+NG-1 (those below g_end), built
// by one warp; lane l holds values 2l and 2l+1 of group k in (lo[k], hi[k]).
// Each group is scaled by 2^sh so its largest magnitude lies in [2^14, 2^15);
// within slice s the values multiplying codes stored as 4^k * q are divided by
// 4^k.  Fragment word for (group G, lane column t, slice s, half which) sits at
// uint32 index ((G*4 + t)*4 + s)*2 + which; info[G] = (2^-sh, sum of the
// group's values, summed in xor-butterfly order).  The NG groups' reductions
// are independent, so they overlap instead of running one after another.
template <int NG>
__device__ __forceinline__ void frag_batch(const float (&lo)[NG], const float (&hi)[NG], int G0, int g_end,
                                           int bits, uint32_t* frag, float2* info, int lane) {
  uint32_t m[NG];
  float sum[NG];
#pragma unroll
  for (int k = 0; k < NG; ++k) {
    m[k] = max(__float_as_uint(fabsf(lo[k])), __float_as_uint(fabsf(hi[k])));
    sum[k] = lo[k] + hi[k];
  }
#pragma unroll
  for (int k = 0; k < NG; ++k) m[k] = __reduce_max_sync(0xffffffffu, m[k]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
    for (int k = 0; k < NG; ++k) sum[k] += __shfl_xor_sync(0xffffffffu, sum[k], o);
  }
  const int q = 2 * lane, s = q / 16, qq = q % 16, which = qq / 8, t = (qq % 8) / 2;
  const int fs = (bits == 4) ? (which ? 4 : 0) : ((s & 1) ? 4 : 0) + (which ? 2 : 0);
#pragma unroll
  for (int k = 0; k < NG; ++k) {
    if (G0 + k < g_end) {
      const int e = (int)((m[k] >> 23) & 0xFF) - 127;  // exponent of the group maximum
      int sh = (m[k] == 0) ? 0 : 14 - max(e, -126);
      sh = min(sh, 126);
      const float scl = exp2i(sh - fs);
      __half2 h2 = __floats2half2_rn(lo[k] * scl, hi[k] * scl);
      frag[(((G0 + k) * 4 + t) * 4 + s) * 2 + which] = *reinterpret_cast<uint32_t*>(&h2);
      if (lane == 0) info[G0 + k] = make_float2(exp2i(-sh), sum[k]);
    }
  }
}

// Dot products of n consecutive tiles (groups G0..G0+n-1 of the input) with the
// fragments in shared memory.
template <int BITS>
__device__ __noinline__ float2 chunk_dot(const uint8_t* tiles, int n, const uint32_t* frag, const float2* info,
                                          int G0, int lane) {
  float acc0 = 0.f, acc1 = 0.f;
  constexpr int TB = 16 * kGroup * BITS / 8 + 64;
  const int t = lane & 3;
#pragma unroll 4
  for (int tt = 0; tt < n; ++tt) {
    const int G = G0 + tt;
    const uint4* fp = reinterpret_cast<const uint4*>(frag + ((G * 4 + t) * 4) * 2);
    const uint4 x = fp[0], y = fp[1];
    const uint2 bf[4] = {make_uint2(x.x, x.y), make_uint2(x.z, x.w), make_uint2(y.x, y.y), make_uint2(y.z, y.w)};
    tile_dot<BITS>(tiles + tt * TB, bf, info[G], lane, acc0, acc1);
  }
  return make_float2(acc0, acc1);
}

// Router order as one 64-bit key: larger logit first, then lower index.  The
// logit bits map to an unsigned key that orders like the float (NaN was
// already mapped to -inf, -0 counts as +0); the low word is ~index, so ties go to the lower
// index.  Key 0 lies below every real entry.
__device__ __forceinline__ uint64_t router_key(float v, int i) {
  const uint32_t u = (v == 0.f) ? 0u : __float_as_uint(v);  // -0 ranks with +0
  const uint32_t k = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return ((uint64_t)k << 32) | (uint32_t)~i;
}
__device__ __forceinline__ float router_key_logit(uint64_t key) {
  const uint32_t k = (uint32_t)(key >> 32);
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// Top-K of the router logits lg[0..E) (shared memory) in router-key order.
// Round k takes the largest key below the previous pick: each lane reduces its
// entries with a tree of independent maxima, then two warp reductions find the
// warp maximum (high word, then low word among the lanes that hold it).
// Nothing is written, so a dry run on any data is harmless.  Lane k < K
// receives pick k.
struct TopPick {
  float logit;
  int expert;
};
__device__ __noinline__ TopPick topk_select(const float* lg, int E, int K, int lane) {
  constexpr int kPer = 16;  // entries per lane per pass
  uint64_t prev = ~0ull;
  TopPick mine = {-INFINITY, 0};
  if (E <= 32 * kPer) {
    // keys computed once, kept in registers
    uint64_t key[kPer];
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int i = j * 32 + lane;
      key[j] = i < E ? router_key(lg[i], i) : 0ull;
    }
#pragma unroll 1
    for (int k = 0; k < K; ++k) {
      uint64_t c[kPer];
#pragma unroll
      for (int j = 0; j < kPer; ++j) c[j] = key[j] < prev ? key[j] : 0ull;
#pragma unroll
      for (int w = kPer / 2; w > 0; w >>= 1) {
#pragma unroll
        for (int j = 0; j < w; ++j) c[j] = c[j] > c[j + w] ? c[j] : c[j + w];
      }
      const uint32_t hmax = __reduce_max_sync(0xffffffffu, (uint32_t)(c[0] >> 32));
      const uint32_t lmax = __reduce_max_sync(0xffffffffu, (uint32_t)(c[0] >> 32) == hmax ? (uint32_t)c[0] : 0u);
      prev = ((uint64_t)hmax << 32) | lmax;
      if (lane == k && prev != 0ull) mine = {router_key_logit(prev), (int)~lmax};
    }
    return mine;
  }
#pragma unroll 1
  for (int k = 0; k < K; ++k) {
    uint64_t best = 0ull;
#pragma unroll 1
    for (int base = 0; base < E; base += 32 * kPer) {
      uint64_t c[kPer];
#pragma unroll
      for (int j = 0; j < kPer; ++j) {
        const int i = base + j * 32 + lane;
        const uint64_t key = i < E ? router_key(lg[i], i) : 0ull;
        c[j] = key < prev ? key : 0ull;
      }
#pragma unroll
      for (int w = kPer / 2; w > 0; w >>= 1) {
#pragma unroll
        for (int j = 0; j < w; ++j) c[j] = c[j] > c[j + w] ? c[j] : c[j + w];
      }
      best = c[0] > best ? c[0] : best;
    }
    const uint32_t hmax = __reduce_max_sync(0xffffffffu, (uint32_t)(best >> 32));
    const uint32_t lmax = __reduce_max_sync(0xffffffffu, (uint32_t)(best >> 32) == hmax ? (uint32_t)best : 0u);
    prev = ((uint64_t)hmax << 32) | lmax;
    if (lane == k && prev != 0ull) mine = {router_key_logit(prev), (int)~lmax};
  }
  return mine;
}

// Spinning warps back off with a short sleep and read the global timer only
// every few rounds, so they take few issue slots from working warps.
__device__ __forceinline__ bool wait_mbar(uint32_t bar, uint32_t parity, uint64_t limit,
                                          const volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = gtimer();
  for (uint32_t it = 0;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 7) == 7 && (*abort_flag || gtimer() - t0 > limit)) return false;
    if (it >= 4) __nanosleep(32);
  }
}
__device__ __forceinline__ bool wait_flag(const volatile int* f, int value, uint64_t limit,
                                          const volatile int* abort_flag) {
  uint64_t t0 = gtimer();
  for (uint32_t it = 0;; ++it) {
    if (*f == value) return true;
    if ((it & 15) == 15 && (*abort_flag || gtimer() - t0 > limit)) return false;
    __nanosleep(64);  // leave issue slots to warps with work
  }
}



// Barrier of the consumer warps that also tells every one of them whether any
// thread arrived with v set, so all take the same branch afterwards.
__device__ __forceinline__ bool consumers_any(bool v) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.or.pred q, 1, %2, p;\n selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(kConsumerWarps * 32)
      : "memory");
  return r != 0;
}

// Weights of layer l: the plan's own for a single-layer launch.
template <bool MULTI>
__device__ __forceinline__ LayerDev layer_of(const DecodePlan& P, int l) {
  if (MULTI) return P.layer_dev[l];
  return LayerDev{P.experts, P.router_w, P.router_bias, P.norm_w};
}

// Expert cache decision for one launch, in the producer warp after top-K
// (lane k < K holds pick k in `sel`).  Every block computes the same result
// from the state the launch started with: a pick whose key has a slot is a
// hit and is read from that slot; the misses are read from host memory and
// take the CLOCK victims among the kCacheWindow slots from the hand (a slot
// holding a hit is never one): first the unreferenced slots in sweep order,
// then, when those run out, the referenced ones (the sweep has cleared them).
__device__ __noinline__ void cache_assign(const DecodePlan& P, Misc* misc, int sel, int lane) {
  const CacheArgs& C = P.cache;
  const int K = P.K, n = C.n_slots;
  const bool pick = lane < K;
  const int have = pick ? C.slot_of[C.key0 + sel] : -1;
  const bool hit = pick && have >= 0;
  const uint32_t hits = __ballot_sync(0xffffffffu, hit), misses = __ballot_sync(0xffffffffu, pick && !hit);
  const uint32_t hand = *C.hand;
  const int W = min(kCacheWindow, n);
  const int ws = (int)((hand + (uint32_t)lane) % (uint32_t)n);
  const int wref = lane < W ? C.ref[ws] : 1;
  bool held = false;  // window position holds one of this launch's hits
  for (int k = 0; k < K; ++k) {
    const int hs = __shfl_sync(0xffffffffu, have, k);
    held = held || (((hits >> k) & 1u) && hs == ws);
  }
  const bool usable = lane < W && !held;
  const uint32_t f0 = __ballot_sync(0xffffffffu, usable && wref == 0);
  const uint32_t f1 = __ballot_sync(0xffffffffu, usable && wref != 0);
  int vpos = -1;
  if (pick && !hit) {
    int r = __popc(misses & ((1u << lane) - 1u));
    uint32_t m = f0;
    if (r >= __popc(f0)) {
      r -= __popc(f0);
      m = f1;
    }
    for (int i = 0; i < r; ++i) m &= m - 1u;
    vpos = __ffs(m) - 1;  // -1 only if fewer than 2K slots (the host refuses that)
  }
  const int victim = vpos >= 0 ? (int)((hand + (uint32_t)vpos) % (uint32_t)n) : -1;
  const int walk = __reduce_max_sync(0xffffffffu, (uint32_t)(vpos + 1));
  if (pick) {
    const int slot = hit ? have : victim;
    misc->cslot[1 + lane] = slot;
    misc->chit[1 + lane] = hit ? 1 : 0;
    misc->slot_src[1 + lane] = hit ? C.slots + (int64_t)slot * P.blob_bytes : C.host + (int64_t)sel * P.blob_bytes;
    misc->slot_dst[1 + lane] = (hit || slot < 0) ? nullptr : C.slots + (int64_t)slot * P.blob_bytes;
  }
  if (lane == 0) {
    misc->chand = (int)hand;
    misc->cwalk = walk;
  }
}

// Applies a launch's cache decision (the last block out, one thread).  After
// an aborted launch the victims' contents are incomplete, so they are dropped
// from the cache instead.
__device__ void cache_update(const DecodePlan& P, const Misc* misc, bool aborted) {
  const CacheArgs& C = P.cache;
  const int K = P.K, n = C.n_slots;
  if (aborted) {
    for (int k = 1; k <= K; ++k) {
      const int v = misc->cslot[k];
      if (misc->chit[k] || v < 0 || v >= n) continue;
      const int old = C.owner[v];
      if (old >= 0) C.slot_of[old] = -1;
      C.owner[v] = -1;
      C.ref[v] = 0;
    }
    return;
  }
  for (int w = 0; w < misc->cwalk; ++w) {  // the sweep clears what it passed
    const int sl = (int)(((uint32_t)misc->chand + (uint32_t)w) % (uint32_t)n);
    bool mine = false;
    for (int k = 1; k <= K; ++k) mine = mine || misc->cslot[k] == sl;
    if (!mine) C.ref[sl] = 0;
  }
  unsigned long long h = 0, m = 0;
  for (int k = 1; k <= K; ++k) {
    const int v = misc->cslot[k], key = C.key0 + misc->slot_e[k];
    if (v < 0 || v >= n) continue;  // no decision recorded (cannot happen after routing)
    if (misc->chit[k]) {
      ++h;
    } else {
      const int old = C.owner[v];
      if (old >= 0) C.slot_of[old] = -1;
      C.owner[v] = key;
      C.slot_of[key] = v;
      ++m;
    }
    C.ref[v] = 1;
  }
  *C.hand = (uint32_t)(((uint32_t)misc->chand + (uint32_t)misc->cwalk) % (uint32_t)n);
  C.stats[0] += h;
  C.stats[1] += m;
}

#ifdef FMOE_TRACE
// Phase timestamps (%globaltimer) of this block for the first kTraceLayers
// layers: SET once by one thread, FIRST by the first of several threads
// (slot starts at 0), LAST by the latest.
__device__ __forceinline__ unsigned long long* trace_slot(const DecodePlan& P, int l, int k) {
  return P.trace + ((size_t)blockIdx.x * kTraceLayers + l) * kTracePoints + k;
}
#define FMOE_TRACE_SET(l, k) \
  do { if (P.trace && (l) < kTraceLayers) *trace_slot(P, l, k) = gtimer(); } while (0)
#define FMOE_TRACE_FIRST(l, k) \
  do { if (P.trace && (l) < kTraceLayers) atomicCAS(trace_slot(P, l, k), 0ull, (unsigned long long)gtimer()); } while (0)
#define FMOE_TRACE_LAST(l, k) \
  do { if (P.trace && (l) < kTraceLayers) atomicMax(trace_slot(P, l, k), (unsigned long long)gtimer()); } while (0)
#else
#define FMOE_TRACE_SET(l, k) do {} while (0)
#define FMOE_TRACE_FIRST(l, k) do {} while (0)
#define FMOE_TRACE_LAST(l, k) do {} while (0)
#endif

// MULTI: one launch runs layers 0..n_layers-1 of a stack for one token.  The
// producer streams on into layer l+1 (its router rows, then the shared
// expert's chunks, which need no routing) while the consumers finish layer l;
// each block publishes its rows of layer l's output as tagged words, and every
// block reads all of them back (until every tag is layer l's) as layer l+1's
// input.  Tags advance by one per layer.
template <int BITS, bool MULTI>
__global__ void __launch_bounds__(kThreads, 1) decode_kernel(const __grid_constant__ DecodePlan P) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int cta = blockIdx.x, G = P.grid;
  constexpr int TB = 16 * kGroup * BITS / 8 + 64;
  Misc* misc = reinterpret_cast<Misc*>(smem + P.off_misc);
  volatile int* abort_flag = &misc->abort;
  uint32_t* tasks = reinterpret_cast<uint32_t*>(smem + P.off_tasks);
  const uint32_t bar_full = smem_u32(smem + P.off_bar);
  const int n_stages_all = P.nstage + P.n_down_max;
  const uint32_t bar_empty = bar_full + 8u * n_stages_all;
  uint16_t* zs = reinterpret_cast<uint16_t*>(smem + P.off_z);
  uint32_t* zfrag = reinterpret_cast<uint32_t*>(smem + P.off_zfrag);
  float2* zinfo = reinterpret_cast<float2*>(smem + P.off_zinfo);
  float* gupart = reinterpret_cast<float*>(smem + P.off_gupart);
  float* dnpart = reinterpret_cast<float*>(smem + P.off_dnpart);
  float* ys = reinterpret_cast<float*>(smem + P.off_y);
  const uint64_t limit = P.timeout_ns;
  const int NL = MULTI ? P.n_layers : 1;

  // this block's share of the work
  const int first_rb = G - 1 - cta;
  const int my_rb = (P.n_slots > 0 && first_rb < P.n_rb) ? (P.n_rb - first_rb + G - 1) / G : 0;
  const bool has_router = P.mode != kModeExpert;
  const int my_rrows = (has_router && cta < P.E) ? (P.E - cta + G - 1) / G : 0;
  const int n_down = P.n_down_max > 0 ? my_rb * P.n_slots * P.dn_chunks : 0;
  float h_res = 0.f;  // residual input of the row this thread combines
  if (tid == 0) FMOE_TRACE_SET(0, 0);

  // ---------------------------------------------------------------- set-up
  // The producer initialises the ring and, before the block barrier, already
  // issues the copies of its first router rows (tasks 0.. of every list, known
  // without reading it): weights do not depend on the previous launch.
  int pre_issued = 0;
  if (warp == kConsumerWarps) {
    for (int i = lane; i < 2 * n_stages_all; i += 32) mbar_init(bar_full + 8u * i, 1);
    misc->last_task[lane] = -1;
    misc->last_task[lane + 32] = -1;
    asm volatile("fence.mbarrier_init.release.cluster;\n fence.proxy.async.shared::cta;" ::: "memory");
    __syncwarp();
    if (has_router && P.router_parts == 1) {
      pre_issued = min(my_rrows, P.n_issuers);
      if (lane < pre_issued) {
        int s, fill;
        task_stage(P.nstage, P.n_issuers, lane, s, fill);  // fill 0
        const uint32_t bytes = (uint32_t)P.H * 2;
        mbar_expect_tx(bar_full + 8u * s, bytes);
        tma_load(smem_u32(smem + P.off_ring + (uint32_t)s * P.stage_bytes), P.router_w + (int64_t)(cta + lane * G) * P.H,
                 bytes, bar_full + 8u * s);
        reinterpret_cast<volatile int*>(misc->last_task)[s] = lane;
      }
    }
    if (lane == 0) FMOE_TRACE_SET(0, 1);
  } else if (warp == 1) {
    misc->aflag[lane] = 0;
    if (lane < 16) {
      misc->rcnt[lane] = 0;
      misc->slot_e[lane] = (lane == 0) ? (P.mode == kModeExpert ? P.expert_id : P.E) : 0;
      misc->slot_w[lane] = (lane == 0) ? 1.f : 0.f;
      misc->slot_src[lane] = (lane == 0) ? P.cache.shared : nullptr;  // cached contexts: the shared expert
      misc->slot_dst[lane] = nullptr;
      misc->cslot[lane] = -1;
      misc->chit[lane] = 1;
    }
    misc->unit_cnt[lane] = 0;
    misc->dn_cnt[lane] = 0;
    if (lane == 0) {
      misc->abort = 0;
      misc->rdone = 0;
    }
  } else if (warp == 2) {
    // this block's ordered task list, global -> shared
    const uint32_t* src = P.tasks + (int64_t)cta * kMaxTasks;
    uint32_t v[kMaxTasks / 32];
#pragma unroll
    for (int k = 0; k < kMaxTasks / 32; ++k) v[k] = src[k * 32 + lane];
#pragma unroll
    for (int k = 0; k < kMaxTasks / 32; ++k) tasks[k * 32 + lane] = v[k];
    if (lane == 0) misc->n_tasks = P.n_tasks[cta];
  }
  __syncthreads();
  const int n_tasks = misc->n_tasks;
  // The next launch may start its weight prefetch as soon as blocks retire.
  if (P.pdl) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  if (warp == kConsumerWarps) {
    // ============================================================ producer warp
    bool routed = false;
    bool waited_grid = false;
    uint32_t tag0 = 0;
    int cur = 0;  // layer being issued
    LayerDev Ld = layer_of<MULTI>(P, 0);
    auto do_routing = [&]() {
      if (!waited_grid) {
        if (P.pdl) asm volatile("griddepcontrol.wait;" ::: "memory");
        tag0 = *reinterpret_cast<volatile uint32_t*>(&P.ws->epoch) + 1u;
      }
      waited_grid = true;
      // Poll the tagged logits until every router row of this layer is
      // published; each round a lane reads experts lane, lane+32, ... (16 loads
      // issued back to back) and stages them in shared memory for top-K.
      const uint32_t tag = tag0 + (uint32_t)cur;
      constexpr int kPollE = 16;  // logits per lane per load round
      float* lg = reinterpret_cast<float*>(smem + P.off_lg);
      const uint64_t t0 = gtimer();
      for (;;) {
        bool mine = true;
        for (int base = 0; base < P.E; base += 32 * kPollE) {
          uint64_t v[kPollE];
#pragma unroll
          for (int k = 0; k < kPollE; ++k) {
            const int i = base + k * 32 + lane;
            v[k] = ld_tagged(P.ws_logits + min(i, P.E - 1));  // past the end: ignored below
          }
#pragma unroll
          for (int k = 0; k < kPollE; ++k) {
            const int i = base + k * 32 + lane;
            if (i < P.E) {
              mine = mine && tagged_tag(v[k]) == tag;
              const float f = tagged_value(v[k]);
              lg[i] = (f != f) ? -INFINITY : f;
            }
          }
        }
        if (__all_sync(0xffffffffu, mine)) {
          if (lane == 0) FMOE_TRACE_SET(cur, 3);
          break;
        }
        __nanosleep(32);
        if (__any_sync(0xffffffffu, *abort_flag != 0 || gtimer() - t0 > limit)) {
          if (lane == 0) {
            atomicOr(&P.ws->status, kStatusTimeoutRouter);
            *abort_flag = 1;
          }
          return false;
        }
      }
      __syncwarp();
      const TopPick pick = topk_select(lg, P.E, P.K, lane);
      const float my_top = pick.logit;
      const int my_sel = pick.expert;
      // renormalised weights over the K selected: p_k / sum_j p_j = e^(l_k - l_0) / sum_j e^(l_j - l_0);
      // an infinite largest logit takes the softmax's limit (equal shares for the picks equal to it)
      const float top0 = __shfl_sync(0xffffffffu, my_top, 0);
      const float ex = lane >= P.K ? 0.f : fabsf(top0) != INFINITY ? expf(my_top - top0) : (my_top == top0 ? 1.f : 0.f);
      float den = ex;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
      if (lane < P.K) {
        const float w = ex / den;
        if (P.mode == kModeLayer) { misc->slot_e[1 + lane] = my_sel; misc->slot_w[1 + lane] = w; }
        if (cta == 0 && P.idx_out) P.idx_out[lane] = my_sel;
        if (cta == 0 && P.w_out) P.w_out[lane] = w;
      }
      __syncwarp();
      if (P.cache.on && P.mode == kModeLayer) {
        cache_assign(P, misc, my_sel, lane);
        __syncwarp();
      }
      if (lane == 0) FMOE_TRACE_SET(cur, 4);
      return true;
    };

    // Copies are issued by n_issuers lanes at once (one bulk copy in flight per
    // lane, each lane refilling only its own stages), in rounds of n_issuers
    // consecutive tasks.  Within a round, tasks that need no routing go first,
    // so a round holding this block's own router rows never waits on routing.
    const int NI = P.n_issuers, per_lane = P.nstage / NI;
    // this lane's next ring position (its copies of the block's router rows
    // issued during set-up took the first one)
    int ring_slot = 0, ring_fill = 0;
    if (lane < pre_issued) ring_advance(per_lane, ring_slot, ring_fill);
    auto issue = [&](int i, uint32_t t) -> int {
      int s, fill;
      if (i < n_tasks - n_down) {
        s = ring_slot * NI + lane;
        fill = ring_fill;
        ring_advance(per_lane, ring_slot, ring_fill);
      } else {
        s = P.nstage + (i - (n_tasks - n_down));
        fill = cur;
      }
      if (fill > 0 && !wait_mbar(bar_empty + 8u * s, (uint32_t)((fill - 1) & 1), limit, abort_flag)) {
        if (!*abort_flag) atomicOr(&P.ws->status, kStatusTimeoutTma);
        *abort_flag = 1;
        return 0;
      }
      const uint32_t dst = smem_u32(smem + P.off_ring + (uint32_t)s * P.stage_bytes);
      const void* src;
      uint32_t bytes;
      const uint32_t ty = task_type(t), idx = task_idx(t), slot = task_slot(t), c = task_chunk(t);
      if (ty == kTaskRouter) {
        const int c0 = (int)c * P.router_part_cols;
        src = Ld.router_w + (int64_t)(cta + (int)idx * G) * P.H + c0;
        bytes = (uint32_t)min(P.router_part_cols, P.H - c0) * 2;
      } else {
        // the expert's blob: resident, or (cached contexts) its cache slot or host copy
        const uint8_t* blob =
            P.cache.on ? misc->slot_src[slot] : Ld.experts + (int64_t)misc->slot_e[slot] * P.blob_bytes;
        if (ty == kTaskGateUp) {
          const int u = cta + (int)idx * G, rb = u % P.units_per_slot;
          const int n = min(chunk_tiles(BITS), P.gu_tiles - (int)c * chunk_tiles(BITS));
          src = blob + ((int64_t)rb * P.gu_tiles + c * chunk_tiles(BITS)) * TB;
          bytes = (uint32_t)(n * TB);
        } else {
          const int rbg = first_rb + (int)idx * G;
          const int n = min(chunk_tiles(BITS), P.dn_tiles - (int)c * chunk_tiles(BITS));
          src = blob + packed_gu_bytes(P.H, P.I, BITS) + ((int64_t)rbg * P.dn_tiles + c * chunk_tiles(BITS)) * TB;
          bytes = (uint32_t)(n * TB);
        }
      }
      mbar_expect_tx(bar_full + 8u * s, bytes);
      tma_load(dst, src, bytes, bar_full + 8u * s);
      // tells the consumer of task i that this fill is the one to wait for
      reinterpret_cast<volatile int*>(misc->last_task)[s] = cur * kMaxTasks + i;
      return 1;
    };
    // Down jobs with stages of their own (the block's last n_down tasks) are all
    // issued as soon as their experts are known, ahead of the gate/up stream:
    // their weights land early and nothing streams any more when the
    // activations are exchanged.
    const int ring_end = n_tasks - n_down;
    bool downs_issued;
    auto issue_downs = [&]() -> bool {
      for (int r = 0; ring_end + r * NI < n_tasks; ++r) {
        const int i = ring_end + r * NI + lane;
        const int ok = (lane < NI && i < n_tasks) ? issue(i, tasks[i]) : 1;
        if (!__all_sync(0xffffffffu, ok)) return false;
      }
      downs_issued = true;
      return true;
    };
    for (cur = 0; cur < NL; ++cur) {
      if (cur > 0) {
        if (__any_sync(0xffffffffu, *abort_flag)) break;
        Ld = layer_of<MULTI>(P, cur);
        routed = false;
      }
      downs_issued = n_down == 0;
      bool failed = P.mode == kModeExpert && !downs_issued && !issue_downs();
      const int pre = cur == 0 ? pre_issued : 0;
      for (int r = 0; r * NI < ring_end && !failed; ++r) {
        if (__any_sync(0xffffffffu, *abort_flag)) break;
        const int i = r * NI + lane;
        const bool mine = lane < NI && i < ring_end && i >= pre;
        const uint32_t t = mine ? tasks[i] : 0u;
        // the shared expert's chunks never wait for routing: they stream in
        // during routing (and, past a launch's first layer, while the
        // previous layer finishes)
        const bool needs_route =
            mine && P.mode == kModeLayer && !routed && task_type(t) != kTaskRouter && task_slot(t) >= 1;
        int ok = 1;
        if (mine && !needs_route) ok = issue(i, t);
        if (!__all_sync(0xffffffffu, ok)) break;
        if (__any_sync(0xffffffffu, needs_route)) {
          if (!do_routing()) break;
          routed = true;
          if (!downs_issued && !issue_downs()) break;
          if (needs_route) ok = issue(i, t);
          if (!__all_sync(0xffffffffu, ok)) break;
          if (lane == 0) FMOE_TRACE_SET(cur, 5);
        }
      }
      if (lane == 0) FMOE_TRACE_SET(cur, 6);
      // a block whose own list needed no routing still owes its down jobs
      if (!downs_issued && !__any_sync(0xffffffffu, *abort_flag)) {
        if (P.mode == kModeLayer && !routed) routed = do_routing();
        if (routed || P.mode != kModeLayer) issue_downs();
      }
      // routing still owed for the output indices, and (cached contexts) by
      // every block, since the last one out records the cache decision
      if (!__any_sync(0xffffffffu, *abort_flag) && !routed && has_router &&
          ((cta == 0 && (P.idx_out || P.w_out)) || (P.cache.on && P.mode == kModeLayer)))
        routed = do_routing();
    }
  } else {
    // ============================================================ consumer warps
    if (P.pdl) asm volatile("griddepcontrol.wait;" ::: "memory");
    const uint32_t tag0 = *reinterpret_cast<volatile uint32_t*>(&P.ws->epoch) + 1u;
    if (tid == 0) misc->tag = tag0 + (uint32_t)(NL - 1);
    // residual rows this block writes at the end
    if (P.mode == kModeLayer && tid < my_rb * 16)
      h_res = bf16f(P.h_in[(first_rb + (tid / 16) * G) * 16 + tid % 16]);
    for (int cur = 0; cur < NL; ++cur) {
      const uint32_t tag = tag0 + (uint32_t)cur;
      const LayerDev Ld = layer_of<MULTI>(P, cur);
      // warps whose first task is a router row (the first tasks of the list)
      const int n_early = (P.mode != kModeExpert && P.n_slots > 0 && my_rrows * P.router_parts <= kConsumerWarps / 2)
                              ? my_rrows * P.router_parts
                              : 0;
      const bool early_router = warp < n_early;
      // thread tid holds columns 8*(tid + j*threads) .. +7, j < kPrepChunks
      constexpr int kCT = kConsumerWarps * 32;
      constexpr int kPrepChunks = (kMaxHidden + 8 * kCT - 1) / (8 * kCT);
      // the layer's RMSNorm weights do not depend on the previous layer: their
      // loads are in flight while the block waits for it
      uint4 nw[kPrepChunks];
#pragma unroll
      for (int j = 0; j < kPrepChunks; ++j) {
        const int c0 = (tid + j * kCT) * 8;
        nw[j] = (Ld.norm_w != nullptr && c0 < P.H) ? *reinterpret_cast<const uint4*>(Ld.norm_w + c0)
                                                   : make_uint4(0u, 0u, 0u, 0u);
      }
      // ---- input: z = RMSNorm(h_in) or h_in (bf16, shared memory) and its fragments
      {
        uint4 hv[kPrepChunks];
        if (!MULTI || cur == 0) {
#pragma unroll
          for (int j = 0; j < kPrepChunks; ++j) {
            const int c0 = (tid + j * kCT) * 8;
            hv[j] = c0 < P.H ? *reinterpret_cast<const uint4*>(P.h_in + c0) : make_uint4(0u, 0u, 0u, 0u);
          }
        } else {
          // The previous layer's output: tagged words that every block's
          // combine publishes.  All of a thread's loads are issued before any
          // tag is examined, and the round is repeated until every tag is the
          // previous layer's.
          const uint32_t want = tag - 1u;
          const uint64_t t0 = gtimer();
          bool ok = true;
          for (uint32_t it = 0;; ++it) {
            ulonglong2 v[kPrepChunks][4];
#pragma unroll
            for (int j = 0; j < kPrepChunks; ++j) {
              const int c0 = min((tid + j * kCT) * 8, P.H - 8);  // past the end: re-read the last chunk, ignored
#pragma unroll
              for (int q = 0; q < 4; ++q) v[j][q] = ld_tagged2(P.ws_h + c0 + 2 * q);
            }
            bool all = true;
#pragma unroll
            for (int j = 0; j < kPrepChunks; ++j) {
              if ((tid + j * kCT) * 8 < P.H) {
#pragma unroll
                for (int q = 0; q < 4; ++q) all = all && tagged_tag(v[j][q].x) == want && tagged_tag(v[j][q].y) == want;
              }
            }
            if (all) {
              // the words hold bf16 values exactly; keep their bf16 bits
#pragma unroll
              for (int j = 0; j < kPrepChunks; ++j) {
                uint32_t hw[4];
#pragma unroll
                for (int q = 0; q < 4; ++q)
                  hw[q] = ((uint32_t)v[j][q].x >> 16) | ((uint32_t)v[j][q].y & 0xFFFF0000u);
                hv[j] = (tid + j * kCT) * 8 < P.H ? make_uint4(hw[0], hw[1], hw[2], hw[3]) : make_uint4(0u, 0u, 0u, 0u);
              }
              break;
            }
            if (*abort_flag || gtimer() - t0 > limit) {
              if (!*abort_flag) atomicOr(&P.ws->status, kStatusTimeoutLayer);
              *abort_flag = 1;
              ok = false;
              break;
            }
            if (it > 0) __nanosleep(128);
          }
          if (consumers_any(!ok || *abort_flag != 0)) break;
        }
        if (Ld.norm_w != nullptr) {
          float ss = 0.f;
#pragma unroll
          for (int j = 0; j < kPrepChunks; ++j) {
            const uint32_t hw[4] = {hv[j].x, hv[j].y, hv[j].z, hv[j].w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              ss = fmaf(bf16lo(hw[k]), bf16lo(hw[k]), ss);
              ss = fmaf(bf16hi(hw[k]), bf16hi(hw[k]), ss);
            }
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
          if (lane == 0) misc->red[warp] = ss;
          asm volatile("bar.sync 1, %0;" ::"r"(kCT) : "memory");
          float tot = 0.f;
          for (int w = 0; w < kConsumerWarps; ++w) tot += misc->red[w];
          const float r = 1.0f / sqrtf(tot / (float)P.H + P.eps);
#pragma unroll
          for (int j = 0; j < kPrepChunks; ++j) {
            const int c0 = (tid + j * kCT) * 8;
            if (c0 < P.H) {
              const uint4 wv = nw[j];
              const uint32_t hw[4] = {hv[j].x, hv[j].y, hv[j].z, hv[j].w};
              const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
              uint32_t zz[4];
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const uint32_t lo = f2bf16(bf16lo(hw[k]) * r * bf16lo(ww[k]));
                const uint32_t hi = f2bf16(bf16hi(hw[k]) * r * bf16hi(ww[k]));
                zz[k] = lo | (hi << 16);
              }
              hv[j] = make_uint4(zz[0], zz[1], zz[2], zz[3]);
            }
          }
        }
#pragma unroll
        for (int j = 0; j < kPrepChunks; ++j) {
          const int c0 = (tid + j * kCT) * 8;
          if (c0 < P.H) *reinterpret_cast<uint4*>(zs + c0) = hv[j];
        }
        asm volatile("bar.sync 1, %0;" ::"r"(kCT) : "memory");
        // The warps whose first task is a router row start it now (the rows
        // need z only); the others build the fp16 fragments, which the gate/up
        // chunks need, and every warp meets at barrier 2 before its first
        // chunk.
        if (P.n_slots > 0 && !early_router) {
          // builder b builds groups 4b..4b+3, then 4(b+B).., so a batch is contiguous
          const int ngz = P.H / kGroup, nb = kConsumerWarps - n_early, b = warp - n_early;
          for (int G0 = 4 * b; G0 < ngz; G0 += 4 * nb) {
            float lo[4], hi[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const uint32_t zz = (G0 + k < ngz) ? *reinterpret_cast<const uint32_t*>(zs + (G0 + k) * kGroup + 2 * lane) : 0u;
              lo[k] = bf16lo(zz);
              hi[k] = bf16hi(zz);
            }
            frag_batch<4>(lo, hi, G0, ngz, BITS, zfrag, zinfo, lane);
          }
        }
        if (!early_router) asm volatile("bar.sync 2, %0;" ::"r"(kCT) : "memory");
      }
      bool frags_seen = !early_router;

      if (tid == 0) FMOE_TRACE_SET(cur, 2);
      // The producer selects the routed experts once per launch, late; running
      // the same selection code here on whatever the logit buffer holds (it
      // writes nothing) brings that code into the instruction cache meanwhile.
      if (warp == kConsumerWarps - 1 && P.mode != kModeExpert && cur == 0) {
        const TopPick dummy = topk_select(reinterpret_cast<const float*>(smem + P.off_lg), P.E, P.K, lane);
        if (dummy.expert < 0) misc->pad[0] = dummy.expert;  // never true; keeps the call
      }
      // ---- task loop: warp w takes tasks w, w+16, ...
      for (int i = warp; i < n_tasks; i += kConsumerWarps) {
        if (!frags_seen && i != warp) {  // an early router warp's first chunk: fragments first
          asm volatile("bar.sync 2, %0;" ::"r"(kCT) : "memory");
          frags_seen = true;
        }
        int s, fill;
        task_stage_of(P.nstage, P.n_issuers, n_tasks, n_down, i, s, fill, cur);
        // A stage's fills are consumed by different warps, so first make sure
        // task i is the stage's current fill (all earlier fills consumed); only
        // then is the parity wait unambiguous.  Every lane observes the phase,
        // so the copied bytes are visible to it.
        const bool issued =
            wait_flag(reinterpret_cast<volatile int*>(misc->last_task) + s, cur * kMaxTasks + i, limit, abort_flag);
        if (!__all_sync(0xffffffffu, issued && wait_mbar(bar_full + 8u * s, (uint32_t)(fill & 1), limit, abort_flag))) {
          if (lane == 0) {
            if (!*abort_flag) atomicOr(&P.ws->status, kStatusTimeoutTma);
            *abort_flag = 1;
          }
          break;
        }
        const uint8_t* stage = smem + P.off_ring + (uint32_t)s * P.stage_bytes;
        const uint32_t t = tasks[i];
        const uint32_t ty = task_type(t), idx = task_idx(t), slot = task_slot(t), c = task_chunk(t);
        // cached contexts: a routed expert read from host memory is also
        // written into its victim slot, tile range by tile range, as it lands
        if (P.cache.on && ty != kTaskRouter && lane == 0 && misc->slot_dst[slot] != nullptr) {
          int64_t off;
          int n;
          if (ty == kTaskGateUp) {
            const int rb = (cta + (int)idx * G) % P.units_per_slot;
            n = min(chunk_tiles(BITS), P.gu_tiles - (int)c * chunk_tiles(BITS));
            off = ((int64_t)rb * P.gu_tiles + c * chunk_tiles(BITS)) * TB;
          } else {
            n = min(chunk_tiles(BITS), P.dn_tiles - (int)c * chunk_tiles(BITS));
            off = packed_gu_bytes(P.H, P.I, BITS) + ((int64_t)(first_rb + (int)idx * G) * P.dn_tiles + c * chunk_tiles(BITS)) * TB;
          }
          bulk_store(misc->slot_dst[slot] + off, smem_u32(stage), (uint32_t)(n * TB));
        }
        // The shared expert's chunks arrive with the router rows (or before
        // them, past a launch's first layer): they wait until this block's
        // router rows are published, so that the router rows have the SM to
        // themselves and the chunks fill the logit exchange instead.  (In a
        // multi-layer launch's first layer the wait measured slower.)
        if (P.mode == kModeLayer && (!MULTI || cur > 0) && ty != kTaskRouter && my_rrows > 0 &&
            !__all_sync(0xffffffffu, wait_flag(&misc->rdone, my_rrows, limit, abort_flag))) {
          if (lane == 0) {
            if (!*abort_flag) atomicOr(&P.ws->status, kStatusTimeoutRouter);
            *abort_flag = 1;
          }
          break;
        }
        if (ty == kTaskRouter) {
          const int c0 = (int)c * P.router_part_cols, width = min(P.router_part_cols, P.H - c0);
          float acc = 0.f;
          for (int col = lane * 8; col < width; col += 256) {
            const uint4 w = *reinterpret_cast<const uint4*>(stage + col * 2);
            const uint4 z = *reinterpret_cast<const uint4*>(zs + c0 + col);
            acc = fmaf(bf16lo(w.x), bf16lo(z.x), acc);
            acc = fmaf(bf16hi(w.x), bf16hi(z.x), acc);
            acc = fmaf(bf16lo(w.y), bf16lo(z.y), acc);
            acc = fmaf(bf16hi(w.y), bf16hi(z.y), acc);
            acc = fmaf(bf16lo(w.z), bf16lo(z.z), acc);
            acc = fmaf(bf16hi(w.z), bf16hi(z.z), acc);
            acc = fmaf(bf16lo(w.w), bf16lo(z.w), acc);
            acc = fmaf(bf16hi(w.w), bf16hi(z.w), acc);
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
          if (lane == 0) {
            // parts of a row are summed, in part order, by whichever warp ends last
            misc->rpart[idx][c] = acc;
            __threadfence_block();
            const int old = atomicAdd(&misc->rcnt[idx], 1);
            if (old == P.router_parts - 1) {
              __threadfence_block();
              const volatile float* rp = misc->rpart[idx];
              float l = 0.f;
              for (int q = 0; q < P.router_parts; ++q) l += rp[q];
              const int e = cta + (int)idx * G;
              if (Ld.router_bias) l += Ld.router_bias[e];
              // fault injection publishes with a stale tag, so no reader accepts it
              st_tagged(P.ws_logits + e, l, (P.flags & FMOE_FLAG_DEBUG_SKIP_ROUTER_RELEASE) ? tag - 1u : tag);
              red_relaxed_add(&P.ws->router_cnt, 1u);
            atomicAdd(&misc->rdone, 1);
            FMOE_TRACE_LAST(cur, 7);
            }
          }
        } else if (ty == kTaskGateUp) {
          if (lane == 0 && slot > 0) FMOE_TRACE_FIRST(cur, 8);
          const int n = min(chunk_tiles(BITS), P.gu_tiles - (int)c * chunk_tiles(BITS));
          const float2 acc = chunk_dot<BITS>(stage, n, zfrag, zinfo, (int)c * chunk_tiles(BITS), lane);
          float acc0 = acc.x, acc1 = acc.y;
          const int u = cta + (int)idx * G, rb = u % P.units_per_slot;
          bool last = true;
          if (P.gu_chunks > 1) {
            float* part = gupart + ((int)idx * P.gu_chunks + (int)c) * 16;
            if ((lane & 3) == 0) { part[lane >> 2] = acc0; part[8 + (lane >> 2)] = acc1; }
            __syncwarp();
            int old = 0;
            if (lane == 0) {
              __threadfence_block();
              old = atomicAdd(&misc->unit_cnt[idx], 1);
              __threadfence_block();
            }
            old = __shfl_sync(0xffffffffu, old, 0);
            last = old == P.gu_chunks - 1;
            if (last && lane < 8) {
              acc0 = 0.f;
              acc1 = 0.f;
              for (int k = 0; k < P.gu_chunks; ++k) {
                const volatile float* pk = gupart + ((int)idx * P.gu_chunks + k) * 16;
                acc0 += pk[lane];
                acc1 += pk[8 + lane];
              }
            }
          }
          if (last) {
            // lanes 0..7 (gu_chunks > 1) or lanes 4g (gu_chunks == 1) hold row g
            const int row = P.gu_chunks > 1 ? lane : (lane >> 2);
            const bool writer = P.gu_chunks > 1 ? lane < 8 : (lane & 3) == 0;
            const float av = writer ? acc0 / (1.0f + expf(-acc0)) * acc1 : 0.f;
            if (writer) st_tagged(P.ws_a + (int64_t)slot * P.I + rb * 8 + row, av, tag);
            if (lane == 0) red_relaxed_add(&P.ws->h_cnt[slot], 1u);
            if (lane == 0) {
              if (slot > 0) FMOE_TRACE_LAST(cur, 9);
              else FMOE_TRACE_LAST(cur, 14);
            }
          }
        } else {
          // activations of this slot as fragments, built once per block in two
          // halves of the slot's groups: the block's two down jobs of a slot
          // usually run on two warps, which then fetch and build a half each.
          if (lane == 0) FMOE_TRACE_FIRST(cur, 15);
          uint32_t* af = reinterpret_cast<uint32_t*>(smem + P.off_afrag + slot * P.afrag_bytes);
          float2* ai = reinterpret_cast<float2*>(smem + P.off_ainfo + slot * P.ainfo_bytes);
          const uint64_t* act = P.ws_a + (int64_t)slot * P.I;
          const int ng = P.I / kGroup, half_g = (ng + 1) / 2;
          int good = 1;
          for (int h = 0; h < 2 && good; ++h) {
            const int gb = h * half_g, ge = min(ng, gb + half_g);
            int* flag = &misc->aflag[2 * (int)slot + h];
            int claimed = 0;
            if (lane == 0 && *reinterpret_cast<volatile int*>(flag) == 0 && atomicCAS(flag, 0, 1) == 0) claimed = 1;
            claimed = __shfl_sync(0xffffffffu, claimed, 0);
            if (!claimed) continue;
            // The slot's activations are tagged words published by every block's
            // gate/up units.  Each lane fetches its pair (2*lane, 2*lane+1) of up
            // to kFetchGroups groups in one round trip and the round is repeated
            // until every tag is current; the published count only paces the
            // retries.  Each group then gets its own power-of-two scale and sum,
            // exactly as the input z does.
            const uint64_t t0 = gtimer();
            for (int g0 = gb; g0 < ge && good; g0 += kFetchGroups) {
              ulonglong2 v[kFetchGroups];
              for (int attempt = 0;; ++attempt) {
                // every load is issued before any result is examined: the loads
                // are volatile, so a check between two of them would wait for
                // the first one's round trip before issuing the second
#pragma unroll
                for (int k = 0; k < kFetchGroups; ++k)  // past the end: re-read the last group, ignored below
                  v[k] = ld_tagged2(act + min(g0 + k, ge - 1) * kGroup + 2 * lane);
                bool mine = true;
#pragma unroll
                for (int k = 0; k < kFetchGroups; ++k)
                  if (g0 + k < ge) mine = mine && tagged_tag(v[k].x) == tag && tagged_tag(v[k].y) == tag;
                if (__all_sync(0xffffffffu, mine)) break;
                // not all published yet: wait for the count, then fetch again
                const bool counted =
                    wait_count(&P.ws->h_cnt[slot], (uint32_t)(P.units_per_slot * (cur + 1)), limit, abort_flag);
                if (__any_sync(0xffffffffu, !counted || *abort_flag != 0 || gtimer() - t0 > limit)) {
                  good = 0;
                  break;
                }
                if (attempt > 0) __nanosleep(256);
              }
              if (!good) break;
              if (lane == 0) FMOE_TRACE_FIRST(cur, 10);
              float lo[kFetchGroups], hi[kFetchGroups];
#pragma unroll
              for (int k = 0; k < kFetchGroups; ++k) {
                lo[k] = tagged_value(v[k].x);
                hi[k] = tagged_value(v[k].y);
              }
              frag_batch<kFetchGroups>(lo, hi, g0, ge, BITS, af, ai, lane);
            }
            if (!good && lane == 0) {
              if (!*abort_flag) atomicOr(&P.ws->status, kStatusTimeoutH);
              *abort_flag = 1;
            }
            if (good) {
              __syncwarp();
              if (lane == 0) {
                __threadfence_block();
                *reinterpret_cast<volatile int*>(flag) = 2;
              }
            }
          }
          // both halves ready (built here or by another warp)
          for (int h = 0; h < 2 && good; ++h) {
            if (h * half_g >= ng) continue;
            if (lane == 0 && !wait_flag(&misc->aflag[2 * (int)slot + h], 2, limit, abort_flag)) {
              if (!*abort_flag) atomicOr(&P.ws->status, kStatusTimeoutH);
              *abort_flag = 1;
              good = 0;
            }
            good = __shfl_sync(0xffffffffu, good, 0);
          }
          __threadfence_block();
          if (!good) break;
          const int n = min(chunk_tiles(BITS), P.dn_tiles - (int)c * chunk_tiles(BITS));
          const float2 acc = chunk_dot<BITS>(stage, n, af, ai, (int)c * chunk_tiles(BITS), lane);
          const float acc0 = acc.x, acc1 = acc.y;
          float* y = ys + ((int)idx * P.n_slots + (int)slot) * 16;
          if (P.dn_chunks == 1) {
            if ((lane & 3) == 0) { y[lane >> 2] = acc0; y[8 + (lane >> 2)] = acc1; }
          } else {
            const int job = (int)idx * P.n_slots + (int)slot;
            float* part = dnpart + (job * P.dn_chunks + (int)c) * 16;
            if ((lane & 3) == 0) { part[lane >> 2] = acc0; part[8 + (lane >> 2)] = acc1; }
            __syncwarp();
            int old = 0;
            if (lane == 0) {
              __threadfence_block();
              old = atomicAdd(&misc->dn_cnt[job], 1);
              __threadfence_block();
            }
            old = __shfl_sync(0xffffffffu, old, 0);
            if (old == P.dn_chunks - 1 && lane < 16) {
              float v = 0.f;
              for (int k = 0; k < P.dn_chunks; ++k) v += reinterpret_cast<volatile float*>(dnpart)[(job * P.dn_chunks + k) * 16 + lane];
              y[lane] = v;
            }
          }
        }
        __syncwarp();
        if (lane == 0) {
          if (P.cache.on) bulk_wait_read();  // a cache fill from this stage has read it
          mbar_arrive(bar_empty + 8u * s);
          if (ty == kTaskDown) FMOE_TRACE_LAST(cur, 11);
        }
      }
      if (!frags_seen) asm volatile("bar.sync 2, %0;" ::"r"(kCT) : "memory");  // an early router warp without chunks
      if (MULTI) {
        // all consumer warps are done with this layer's tasks
        if (consumers_any(*abort_flag != 0)) break;
        if (tid < my_rb * 16) {
          const int jb = tid / 16, row = tid % 16, out_row = (first_rb + jb * G) * 16 + row;
          float acc = h_res + ys[(jb * P.n_slots + 0) * 16 + row];
          for (int k = 1; k < P.n_slots; ++k) acc = fmaf(misc->slot_w[k], ys[(jb * P.n_slots + k) * 16 + row], acc);
          const uint16_t o = f2bf16(acc);
          h_res = bf16f(o);  // the next layer's residual input of this row
          if (cur == NL - 1)
            P.h_out[out_row] = o;
          else
            st_tagged(P.ws_h + out_row, h_res, tag);
        }
        if (tid == 0) FMOE_TRACE_SET(cur, 12);
        if (warp == 1) {
          misc->aflag[lane] = 0;
          misc->unit_cnt[lane] = 0;
          misc->dn_cnt[lane] = 0;
          if (lane < 16) misc->rcnt[lane] = 0;
          if (lane == 0) misc->rdone = 0;
        }
      }
    }
    if (P.cache.on && lane == 0) bulk_wait_all();  // cache fills complete before the block reports out
  }
  __syncthreads();

  // ---------------------------------------------------------------- combine + output
  const bool aborted = *abort_flag != 0;
  if (!MULTI && !aborted && tid < kConsumerWarps * 32) {
    for (int r = tid; r < my_rb * 16; r += kConsumerWarps * 32) {
      const int jb = r / 16, row = r % 16;
      const int out_row = (first_rb + jb * G) * 16 + row;
      if (P.mode == kModeLayer) {
        float acc = h_res + ys[(jb * P.n_slots + 0) * 16 + row];
        for (int k = 1; k < P.n_slots; ++k) acc = fmaf(misc->slot_w[k], ys[(jb * P.n_slots + k) * 16 + row], acc);
        P.h_out[out_row] = f2bf16(acc);
      } else if (P.mode == kModeExpert) {
        P.y_out[out_row] = ys[(jb * P.n_slots + 0) * 16 + row];
      }
    }
  }

  if (tid == 0) FMOE_TRACE_SET(0, 12);
  // ---------------------------------------------------------------- drain + reset
  if (tid == kConsumerWarps * 32) {
    // After an abort the latest copy into every stage must land before the
    // block exits (without one, every issued copy was consumed already).
    for (int s = 0; s < n_stages_all && aborted; ++s) {
      const int uid = misc->last_task[s];
      if (uid < 0) continue;
      int s2, fill;
      task_stage_of(P.nstage, P.n_issuers, n_tasks, n_down, uid % kMaxTasks, s2, fill, uid / kMaxTasks);
      const uint64_t t0 = gtimer();
      while (!mbar_try_wait(bar_full + 8u * s, (uint32_t)(fill & 1)))
        if (gtimer() - t0 > limit) {
          atomicOr(&P.ws->status, kStatusTimeoutTma);
          break;
        }
    }
    FMOE_TRACE_SET(0, 13);
    // the last block out advances the epoch for the next launch
    uint32_t old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(old) : "l"(&P.ws->exit_count) : "memory");
    if (old == (uint32_t)G - 1) {
      P.ws->exit_count = 0;
      P.ws->router_cnt = 0;
      for (int k = 0; k < 16; ++k) P.ws->h_cnt[k] = 0;
      P.ws->epoch = misc->tag;
      if (P.cache.on && P.mode == kModeLayer)
        cache_update(P, misc, aborted || *reinterpret_cast<volatile uint32_t*>(&P.ws->status) != 0u);
    }
  }
}

}  // namespace

using DecodeFn = void (*)(DecodePlan);
DecodeFn decode_fn(int bits, bool multi) {
  if (bits == 4) return multi ? decode_kernel<4, true> : decode_kernel<4, false>;
  return multi ? decode_kernel<2, true> : decode_kernel<2, false>;
}

int decode_occupancy(int bits, bool multi, int smem_bytes, int* blocks_per_sm) {
  DecodeFn kern = decode_fn(bits, multi);
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
  if (err != cudaSuccess) return (int)err;
  return (int)cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks_per_sm, kern, kThreads, smem_bytes);
}

int decode_max_smem_optin(int device) {
  int v = 0;
  cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, device);
  return v;
}

int launch_decode(const DecodePlan& plan, void* stream, bool cooperative, bool pdl) {
  DecodePlan p = plan;
  p.pdl = pdl ? 1 : 0;
  DecodeFn kern = decode_fn(p.bits, p.n_layers > 0);
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)p.smem_bytes);
  if (err != cudaSuccess) return (int)err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = p.smem_bytes;
  cfg.stream = (cudaStream_t)stream;
  cudaLaunchAttribute attrs[2];
  int na = 0;
  if (cooperative) {
    attrs[na].id = cudaLaunchAttributeCooperative;
    attrs[na].val.cooperative = 1;
    ++na;
  }
  if (pdl) {
    attrs[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attrs[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attrs;
  cfg.numAttrs = na;
  return (int)cudaLaunchKernelEx(&cfg, kern, p);
}

int zero_workspace(void* ws, size_t bytes, void* stream) {
  return (int)cudaMemsetAsync(ws, 0, bytes, (cudaStream_t)stream);
}

}  // namespace fmoe
