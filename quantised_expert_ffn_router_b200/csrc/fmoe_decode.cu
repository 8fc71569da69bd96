// fmoe_decode.cu -- fused single-token mixture-of-experts layer for sm_100a.
//
// One cooperative launch, one 512-thread block per SM, runs the whole decode
// step the Flash-MoE pages split over CMD2, the CPU and CMD3 (page 5 "How the
// SSD expert streaming pipeline works"):
//   1. optional RMSNorm of the layer input (every block, redundantly);
//   2. router GEMV: block b owns router rows b, b+G, ...; logits go to a global
//      workspace and a release-counter announces them;
//   3. softmax + top-K: every block waits (bounded) for all logits and selects
//      the same K experts itself, so no second launch is needed;
//   4. SwiGLU experts: the K routed experts and the shared expert are cut into
//      units of 8 gate rows + 8 up rows over the full hidden width; units are
//      striped over all blocks, their weights stream HBM -> shared memory by
//      bulk-async (TMA) copies into a ring of stages, and each warp dequantises
//      its 256-column slice into mma.sync fragments (codes are exact in fp16,
//      the per-group scale and bias are applied as s*sum(q*x) + b*sum(x) after
//      each 64-column group);  a = silu(g)*u goes to the workspace and a
//      per-expert counter is released;
//   5. down projection: block b owns output row blocks G-1-b, 2G-1-b, ... for
//      every expert, preloads those weight tiles at the start, waits (bounded)
//      for an expert's activations to be complete and folds them in;
//   6. combine: h_out = h_in + y_shared + sum_k w_k y_k in fp32, one bf16
//      rounding, written by the block that owns the rows (no atomics).
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
__device__ __forceinline__ uint64_t gtimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void red_release_add(uint32_t* p, uint32_t v) {
  asm volatile("fence.acq_rel.gpu;\n red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
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
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
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

// Input vector -> fp16 B fragments.  Group G of 64 values is scaled by 2^sh so
// its largest magnitude lies in [2^14, 2^15); within slice s of the group the
// values multiplying codes stored as 4^k * q are divided by 4^k.  Fragment
// word for (group G, lane column t, slice s, half which) sits at uint32 index
// ((G*4 + t)*4 + s)*2 + which; info[G] = (2^-sh, sum of the group's values).
template <typename Load>
__device__ __forceinline__ void build_frags(Load load, int C, int bits, uint32_t* frag, float2* info, int tid) {
  const int lane = tid & 31;
  for (int base = 0; base < C / 2; base += kThreads) {
    int p = base + tid;
    if (p - lane + 32 > C / 2) break;  // warp-uniform (C is a multiple of 64)
    float v0 = load(2 * p), v1 = load(2 * p + 1);
    uint32_t m = max(__float_as_uint(fabsf(v0)), __float_as_uint(fabsf(v1)));
    m = __reduce_max_sync(0xffffffffu, m);
    float sum = v0 + v1;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    int e = (int)((m >> 23) & 0xFF) - 127;  // exponent of the group maximum
    int sh = (m == 0) ? 0 : 14 - max(e, -126);
    sh = min(sh, 126);
    int k = (2 * p) % kGroup, s = k / 16, kk = k % 16, which = kk / 8, t = (kk % 8) / 2;
    int fs = (bits == 4) ? (which ? 4 : 0) : ((s & 1) ? 4 : 0) + (which ? 2 : 0);
    float scl = exp2i(sh - fs);
    __half2 h2 = __floats2half2_rn(v0 * scl, v1 * scl);
    int G = (2 * p) / kGroup;
    frag[((G * 4 + t) * 4 + s) * 2 + which] = *reinterpret_cast<uint32_t*>(&h2);
    if (lane == 0) info[G] = make_float2(exp2i(-sh), sum);
  }
}

__device__ __forceinline__ void load_frags(const uint32_t* frag, const float2* info, int kr, int n_groups, int lane,
                                           uint2 (&bf)[4][4], float2 (&inf)[4]) {
  const int t = lane & 3;
#pragma unroll
  for (int gg = 0; gg < 4; ++gg) {
    int G = kr * 4 + gg;
    if (G < n_groups) {
      const uint4* src = reinterpret_cast<const uint4*>(frag + ((G * 4 + t) * 4) * 2);
      uint4 x = src[0], y = src[1];
      bf[gg][0] = make_uint2(x.x, x.y);
      bf[gg][1] = make_uint2(x.z, x.w);
      bf[gg][2] = make_uint2(y.x, y.y);
      bf[gg][3] = make_uint2(y.z, y.w);
      inf[gg] = info[G];
    } else {
      inf[gg] = make_float2(0.f, 0.f);
#pragma unroll
      for (int s = 0; s < 4; ++s) bf[gg][s] = make_uint2(0u, 0u);
    }
  }
}

// Bounded waits: true when satisfied, false after the time limit.
__device__ __forceinline__ bool wait_counter(const uint32_t* p, uint32_t target, uint64_t limit) {
  uint64_t t0 = gtimer();
  for (uint32_t it = 0;; ++it) {
    if (ld_acquire(p) >= target) return true;
    if ((it & 15) == 15 && gtimer() - t0 > limit) return false;
  }
}
__device__ __forceinline__ bool wait_mbar(uint32_t bar, uint32_t parity, uint64_t limit) {
  if (mbar_try_wait(bar, parity)) return true;
  uint64_t t0 = gtimer();
  for (;;) {
    if (mbar_try_wait(bar, parity)) return true;
    if (gtimer() - t0 > limit) return false;
  }
}

template <int BITS>
__global__ void __launch_bounds__(kThreads, 1) decode_kernel(const __grid_constant__ DecodePlan P) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int cta = blockIdx.x, G = P.grid;
  constexpr int TB = 16 * kGroup * BITS / 8 + 64;

  const uint32_t bar_base = smem_u32(smem + P.off_bar);
  const uint32_t bar_router = bar_base + 8u * (P.nstage + kMaxSlots);
  int* slot_e = reinterpret_cast<int*>(smem + P.off_misc);
  float* slot_w = reinterpret_cast<float*>(smem + P.off_misc + 64);
  float* gupart = reinterpret_cast<float*>(smem + P.off_gupart);
  float* dnpart = reinterpret_cast<float*>(smem + P.off_dnpart);
  float* ys = reinterpret_cast<float*>(smem + P.off_y);
  float* rpart = reinterpret_cast<float*>(smem + P.off_rpart);
  uint16_t* zs = reinterpret_cast<uint16_t*>(smem + P.off_z);

  // this block's share of the work
  const int my_units = P.total_units > cta ? (P.total_units - cta + G - 1) / G : 0;
  const int my_stages = (my_units + P.teams_gu - 1) / P.teams_gu;
  const int first_rb = G - 1 - cta;
  const int my_rb = (P.n_slots > 0 && first_rb < P.n_rb) ? (P.n_rb - first_rb + G - 1) / G : 0;
  const bool has_router = P.mode != kModeExpert;
  const int my_rrows = (has_router && cta < P.E) ? (P.E - cta + G - 1) / G : 0;
  const uint64_t limit = P.timeout_ns;

  auto unit_of = [&](int j) { return cta + j * G; };
  // Units of a stage are increasing, so its last unit has its largest slot.
  auto stage_max_slot = [&](int s) {
    int j = min((s + 1) * P.teams_gu, my_units) - 1;
    return unit_of(j) / P.units_per_slot;
  };

  if (tid == 0) {
    for (int i = 0; i < P.nstage + kMaxSlots + 1; ++i) mbar_init(bar_base + 8u * i, 1);
    asm volatile("fence.mbarrier_init.release.cluster;\n fence.proxy.async.shared::cta;" ::: "memory");
    if (P.mode == kModeLayer) { slot_e[0] = P.E; slot_w[0] = 1.f; }
    if (P.mode == kModeExpert) { slot_e[0] = P.expert_id; slot_w[0] = 1.f; }
  }
  __syncthreads();

  // ---------------------------------------------------------------- producer (thread 0)
  int issued = 0;       // stages issued, in order
  uint32_t dn_issued = 0;
  bool router_issued = false;
  auto issue_stage = [&](int s) {
    const int buf = s % P.nstage;
    const uint32_t dst = smem_u32(smem + P.off_ring + (uint32_t)buf * P.stage_bytes);
    const uint32_t bar = bar_base + 8u * buf;
    int n = min(P.teams_gu, my_units - s * P.teams_gu);
    mbar_expect_tx(bar, (uint32_t)(n * P.gu_unit_bytes));
    for (int tau = 0; tau < n; ++tau) {
      int u = unit_of(s * P.teams_gu + tau);
      int slot = u / P.units_per_slot, rb = u % P.units_per_slot;
      const uint8_t* src = P.experts + (int64_t)slot_e[slot] * P.blob_bytes + (int64_t)rb * P.gu_unit_bytes;
      tma_load(dst + (uint32_t)(tau * P.gu_unit_bytes), src, (uint32_t)P.gu_unit_bytes, bar);
    }
  };
  auto issue_down = [&](int slot) {
    if (my_rb == 0) return;
    const uint32_t bar = bar_base + 8u * (P.nstage + slot);
    mbar_expect_tx(bar, (uint32_t)(my_rb * P.dn_job_bytes));
    const uint8_t* ex = P.experts + (int64_t)slot_e[slot] * P.blob_bytes + packed_gu_bytes(P.H, P.I, BITS);
    for (int j = 0; j < my_rb; ++j) {
      int rbg = first_rb + j * G;
      uint32_t dst = smem_u32(smem + P.off_down + (uint32_t)((slot * P.rb_per_cta + j) * P.dn_job_bytes));
      tma_load(dst, ex + (int64_t)rbg * P.dn_job_bytes, (uint32_t)P.dn_job_bytes, bar);
    }
    dn_issued |= 1u << slot;
  };
  auto issue_ready_stages = [&](int upto, bool routed) {
    while (issued < my_stages && issued < upto && (routed || stage_max_slot(issued) == 0)) issue_stage(issued++);
  };

  if (tid == 0) {
    if (my_rrows > 0) {
      mbar_expect_tx(bar_router, (uint32_t)(my_rrows * P.H * 2));
      for (int j = 0; j < my_rrows; ++j)
        tma_load(smem_u32(smem + P.off_router + (uint32_t)(j * P.H * 2)), P.router_w + (int64_t)(cta + j * G) * P.H,
                 (uint32_t)(P.H * 2), bar_router);
      router_issued = true;
    }
    if (P.n_slots > 0) issue_down(0);
    issue_ready_stages(P.nstage, P.mode == kModeExpert);
  }

  // Weights above do not depend on earlier kernels; everything below may.
  if (P.pdl) asm volatile("griddepcontrol.wait;" ::: "memory");
  if (P.pdl) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  int abort = 0;
  int consumed = 0;         // stages consumed
  bool router_consumed = false;
  uint32_t dn_consumed = 0;

  // ---------------------------------------------------------------- input: z and its fragments
  {
    const uint16_t* h = P.h_in;
    if (P.norm_w != nullptr) {
      float ss = 0.f;
      for (int i = tid; i < P.H; i += kThreads) {
        float v = bf16f(h[i]);
        ss = fmaf(v, v, ss);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      if (lane == 0) dnpart[warp] = ss;
      __syncthreads();
      float tot = 0.f;
      for (int w = 0; w < kWarps; ++w) tot += dnpart[w];
      const float r = 1.0f / sqrtf(tot / (float)P.H + P.eps);
      for (int i = tid; i < P.H; i += kThreads) zs[i] = f2bf16(bf16f(h[i]) * r * bf16f(P.norm_w[i]));
    } else {
      for (int i = tid; i < P.H; i += kThreads) zs[i] = h[i];
    }
    for (int i = tid; i < P.router_rows * kWarps; i += kThreads) rpart[i] = 0.f;
    __syncthreads();
    if (P.n_slots > 0)
      build_frags([&](int i) { return bf16f(zs[i]); }, P.H, BITS, reinterpret_cast<uint32_t*>(smem + P.off_zfrag),
                  reinterpret_cast<float2*>(smem + P.off_zinfo), tid);
    __syncthreads();
  }

  // ---------------------------------------------------------------- router GEMV
  if (my_rrows > 0) {
    if (!wait_mbar(bar_router, 0, limit)) {
      abort = 1;
      atomicOr(&P.ws->status, kStatusTimeoutTma);
    }
    const int pairs = my_rrows * P.router_chunks;
    for (int p = warp; p < pairs && !abort; p += kWarps) {
      int j = p / P.router_chunks, ch = p % P.router_chunks;
      int col = ch * 256 + lane * 8;
      float acc = 0.f;
      if (col < P.H) {
        uint4 w = *reinterpret_cast<const uint4*>(smem + P.off_router + (uint32_t)(j * P.H * 2 + col * 2));
        uint4 z = *reinterpret_cast<const uint4*>(zs + col);
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
      if (lane == 0) rpart[j * kWarps + warp] = acc;
    }
    router_consumed = true;
  }
  abort = __syncthreads_or(abort);
  if (!abort && tid < my_rrows) {
    float l = 0.f;
    for (int w = 0; w < kWarps; ++w) l += rpart[tid * kWarps + w];
    int e = cta + tid * G;
    if (P.router_bias) l += P.router_bias[e];
    P.ws_logits[e] = l;
  }
  __syncthreads();
  if (tid == 0 && has_router && !abort && !(P.flags & FMOE_FLAG_DEBUG_SKIP_ROUTER_RELEASE))
    red_release_add(&P.ws->router_arrive, 1u);

  // ---------------------------------------------------------------- routing (softmax + top-K)
  bool routed = (P.mode == kModeExpert);
  auto do_routing = [&]() {
    if (tid == 0 && !wait_counter(&P.ws->router_arrive, (uint32_t)G, limit)) {
      atomicOr(&P.ws->status, kStatusTimeoutRouter);
      abort = 1;
    }
    abort = __syncthreads_or(abort);
    if (abort) return;
    float* lg = reinterpret_cast<float*>(smem + P.off_z);  // z no longer needed
    if (warp == 0) {
      for (int i = lane; i < P.E; i += 32) {
        float v = __ldcg(P.ws_logits + i);
        lg[i] = (v != v) ? -INFINITY : v;
      }
      __syncwarp();
      float top[kMaxTopK];
      int sel[kMaxTopK];
      for (int k = 0; k < P.K; ++k) {
        float bv = -INFINITY;
        int bi = P.E;
        for (int i = lane; i < P.E; i += 32) {
          float v = lg[i];
          if (v > bv || (v == bv && i < bi)) { bv = v; bi = i; }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          float ov = __shfl_xor_sync(0xffffffffu, bv, o);
          int oi = __shfl_xor_sync(0xffffffffu, bi, o);
          if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
        }
        if (bi >= P.E) bi = 0;  // only when every remaining logit is NaN/-inf
        top[k] = bv;
        sel[k] = bi;
        __syncwarp();
        if (lane == 0) lg[bi] = -INFINITY;
        __syncwarp();
      }
      if (lane == 0) {
        float den = 0.f;
        float ex[kMaxTopK];
        for (int k = 0; k < P.K; ++k) { ex[k] = expf(top[k] - top[0]); den += ex[k]; }
        for (int k = 0; k < P.K; ++k) {
          float w = ex[k] / den;
          if (P.mode == kModeLayer) { slot_e[1 + k] = sel[k]; slot_w[1 + k] = w; }
          if (cta == 0 && P.idx_out) P.idx_out[k] = sel[k];
          if (cta == 0 && P.w_out) P.w_out[k] = w;
        }
      }
    }
    __syncthreads();
    if (tid == 0) {
      for (int s = 1; s < P.n_slots; ++s) issue_down(s);
      issue_ready_stages(consumed + P.nstage, true);
    }
  };

  // ---------------------------------------------------------------- down projections of one slot
  const int n_ig = P.I / kGroup;
  auto do_downs = [&](int d) {
    if (tid == 0 && !wait_counter(&P.ws->h_arrive[d], (uint32_t)P.units_per_slot, limit)) {
      atomicOr(&P.ws->status, kStatusTimeoutH);
      abort = 1;
    }
    if (my_rb > 0 && !wait_mbar(bar_base + 8u * (P.nstage + d), 0, limit)) {
      abort = 1;
      atomicOr(&P.ws->status, kStatusTimeoutTma);
    }
    abort = __syncthreads_or(abort);
    if (abort) return;
    dn_consumed |= 1u << d;
    uint32_t* af = reinterpret_cast<uint32_t*>(smem + P.off_afrag + (uint32_t)(d & 1) * P.afrag_bytes);
    float2* ai = reinterpret_cast<float2*>(smem + P.off_ainfo + (uint32_t)(d & 1) * P.ainfo_bytes);
    const float* act = P.ws_a + (int64_t)d * P.I;
    build_frags([&](int i) { return __ldcg(act + i); }, P.I, BITS, af, ai, tid);
    __syncthreads();
    const int kr = warp % P.n_kr_dn, team = warp / P.n_kr_dn;
    if (team < P.teams_dn) {
      uint2 bf[4][4];
      float2 inf[4];
      load_frags(af, ai, kr, n_ig, lane, bf, inf);
      for (int job = team; job < my_rb; job += P.teams_dn) {
        const uint8_t* base = smem + P.off_down + (uint32_t)((d * P.rb_per_cta + job) * P.dn_job_bytes);
        float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
        for (int tt = 0; tt < 4; ++tt)
          if (kr * 4 + tt < P.dn_tiles) tile_dot<BITS>(base + (kr * 4 + tt) * TB, bf[tt], inf[tt], lane, acc0, acc1);
        if ((lane & 3) == 0) {
          dnpart[warp * 16 + (lane >> 2)] = acc0;
          dnpart[warp * 16 + 8 + (lane >> 2)] = acc1;
        }
        if (P.n_kr_dn > 1) asm volatile("bar.sync %0, %1;" ::"r"(1 + team), "r"(P.n_kr_dn * 32) : "memory");
        else __syncwarp();
        if (kr == 0 && lane < 16) {
          float y = 0.f;
          for (int k = 0; k < P.n_kr_dn; ++k) y += dnpart[(team * P.n_kr_dn + k) * 16 + lane];
          ys[(job * P.n_slots + d) * 16 + lane] = y;
        }
        if (P.n_kr_dn > 1) asm volatile("bar.sync %0, %1;" ::"r"(1 + team), "r"(P.n_kr_dn * 32) : "memory");
        else __syncwarp();
      }
    }
  };

  // ---------------------------------------------------------------- gate/up stages, interleaved with downs
  int next_down = 0;
  const int n_zg = P.H / kGroup;
  for (int s = 0; s < my_stages && !abort; ++s) {
    if (!routed && stage_max_slot(s) > 0) {
      do_routing();
      routed = true;
      if (abort) break;
    }
    const int buf = s % P.nstage;
    if (!wait_mbar(bar_base + 8u * buf, (uint32_t)((s / P.nstage) & 1), limit)) {
      abort = 1;
      atomicOr(&P.ws->status, kStatusTimeoutTma);
    }
    const int kr = warp % P.n_kr_gu, team = warp / P.n_kr_gu;
    const int j = s * P.teams_gu + team;
    float* part = gupart + (s & 1) * (kWarps * 16);
    if (!abort && team < P.teams_gu && j < my_units) {
      uint2 bf[4][4];
      float2 inf[4];
      load_frags(reinterpret_cast<const uint32_t*>(smem + P.off_zfrag),
                 reinterpret_cast<const float2*>(smem + P.off_zinfo), kr, n_zg, lane, bf, inf);
      const uint8_t* base = smem + P.off_ring + (uint32_t)buf * P.stage_bytes + (uint32_t)(team * P.gu_unit_bytes);
      float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
      for (int tt = 0; tt < 4; ++tt)
        if (kr * 4 + tt < P.gu_tiles) tile_dot<BITS>(base + (kr * 4 + tt) * TB, bf[tt], inf[tt], lane, acc0, acc1);
      if ((lane & 3) == 0) {
        part[warp * 16 + (lane >> 2)] = acc0;
        part[warp * 16 + 8 + (lane >> 2)] = acc1;
      }
    }
    abort = __syncthreads_or(abort);
    if (abort) break;
    consumed = s + 1;
    if (tid == 0) issue_ready_stages(consumed + P.nstage, routed);
    // reduce the stage's units: a = silu(g) * u
    const int nred = P.teams_gu * 8;
    if (tid < nred) {
      const int tau = tid / 8, i = tid % 8, jj = s * P.teams_gu + tau;
      if (jj < my_units) {
        float g = 0.f, u = 0.f;
        for (int k = 0; k < P.n_kr_gu; ++k) {
          g += part[(tau * P.n_kr_gu + k) * 16 + i];
          u += part[(tau * P.n_kr_gu + k) * 16 + 8 + i];
        }
        const int uu = unit_of(jj), slot = uu / P.units_per_slot, rb = uu % P.units_per_slot;
        const float a = g / (1.0f + expf(-g)) * u;
        P.ws_a[(int64_t)slot * P.I + rb * 8 + i] = a;
      }
    }
    if (nred <= 32) __syncwarp();
    else if (tid < ((nred + 31) / 32) * 32) asm volatile("bar.sync 15, %0;" ::"r"(((nred + 31) / 32) * 32) : "memory");
    if (tid == 0) {
      // publish per slot (units of a stage have non-decreasing slots)
      int n = min(P.teams_gu, my_units - s * P.teams_gu);
      int cur = -1;
      uint32_t cnt = 0;
      for (int tau = 0; tau < n; ++tau) {
        int slot = unit_of(s * P.teams_gu + tau) / P.units_per_slot;
        if (slot != cur) {
          if (cnt) red_release_add(&P.ws->h_arrive[cur], cnt);
          cur = slot;
          cnt = 0;
        }
        ++cnt;
      }
      if (cnt) red_release_add(&P.ws->h_arrive[cur], cnt);
    }
    // downs of slot d once all of this block's units of slots <= d+1 are done
    while (next_down < P.n_slots && !abort) {
      bool last = (s + 1 == my_stages);
      int next_slot = last ? 1 << 30 : unit_of((s + 1) * P.teams_gu) / P.units_per_slot;
      if (next_slot <= next_down + 1) break;
      if (!routed && next_down >= 1) { do_routing(); routed = true; if (abort) break; }
      do_downs(next_down++);
    }
  }
  // Routing still pending: needed for the output indices (block 0) and for the
  // down projections of routed experts.
  if (!abort && !routed && has_router && (cta == 0 || (P.mode == kModeLayer && my_rb > 0))) {
    do_routing();
    routed = true;
  }
  while (!abort && next_down < P.n_slots) do_downs(next_down++);

  // ---------------------------------------------------------------- combine + output
  __syncthreads();
  if (!abort) {
    for (int r = tid; r < my_rb * 16; r += kThreads) {
      const int jb = r / 16, row = r % 16;
      const int out_row = (first_rb + jb * G) * 16 + row;
      if (P.mode == kModeLayer) {
        float acc = bf16f(P.h_in[out_row]) + ys[(jb * P.n_slots + 0) * 16 + row];
        for (int k = 1; k < P.n_slots; ++k) acc = fmaf(slot_w[k], ys[(jb * P.n_slots + k) * 16 + row], acc);
        P.h_out[out_row] = f2bf16(acc);
      } else if (P.mode == kModeExpert) {
        P.y_out[out_row] = ys[(jb * P.n_slots + 0) * 16 + row];
      }
    }
  }

  // ---------------------------------------------------------------- drain + reset
  if (tid == 0) {
    // copies still in flight (only after an abort) must land before the block exits
    for (int s = consumed; s < issued; ++s)
      if (!wait_mbar(bar_base + 8u * (s % P.nstage), (uint32_t)((s / P.nstage) & 1), limit))
        atomicOr(&P.ws->status, kStatusTimeoutTma);
    if (router_issued && !router_consumed && !wait_mbar(bar_router, 0, limit))
      atomicOr(&P.ws->status, kStatusTimeoutTma);
    for (int d = 0; d < kMaxSlots; ++d)
      if ((dn_issued >> d & 1) && !(dn_consumed >> d & 1) && !wait_mbar(bar_base + 8u * (P.nstage + d), 0, limit))
        atomicOr(&P.ws->status, kStatusTimeoutTma);
    uint32_t old;
    asm volatile("fence.acq_rel.gpu;\n atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;"
                 : "=r"(old)
                 : "l"(&P.ws->exit_count)
                 : "memory");
    if (old == (uint32_t)G - 1) {
      P.ws->router_arrive = 0;
      for (int i = 0; i < 16; ++i) P.ws->h_arrive[i] = 0;
      P.ws->exit_count = 0;
      __threadfence();
    }
  }
}

}  // namespace

int decode_occupancy(int bits, int smem_bytes, int* blocks_per_sm) {
  void (*kern)(DecodePlan) = bits == 4 ? decode_kernel<4> : decode_kernel<2>;
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
  void (*kern)(DecodePlan) = p.bits == 4 ? decode_kernel<4> : decode_kernel<2>;
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
  err = cudaLaunchKernelEx(&cfg, kern, p);
  return (int)err;
}

int zero_workspace(void* ws, size_t bytes, void* stream) {
  return (int)cudaMemsetAsync(ws, 0, bytes, (cudaStream_t)stream);
}

}  // namespace fmoe
