// fmoe_api.cu -- C ABI (include/fmoe.h): contexts, argument validation,
// shared-memory plans and kernel launches.  No compute happens on the host.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <set>
#include <string>
#include <vector>

#include "fmoe_internal.h"

using namespace fmoe;

struct fmoe_ctx {
  fmoe_config cfg;
  std::vector<fmoe_layer_desc> layers;
  int device = 0;
  int n_sm = 0;
  bool pdl_ok = true;
  void* ws = nullptr;  // device workspace
  size_t ws_bytes = 0;
  WsHeader* hdr = nullptr;
  uint64_t* logits = nullptr;  // tagged
  uint64_t* act = nullptr;     // tagged
  size_t tagged_bytes = 0;     // logits, activations and layer outputs: the tagged words after the header
  uint64_t tags_used = 0;      // mirrors the device epoch: tags handed out since the last clear
  unsigned long long* trace = nullptr;  // caller's timestamp buffer (FMOE_TRACE builds), or null
  uint32_t* tasks = nullptr;   // device [3 modes][grid][kMaxTasks]
  int32_t* ntasks = nullptr;   // device [3 modes][grid]
  uint16_t* stack_buf[2] = {nullptr, nullptr};  // ping-pong activations, [max_tokens][H] bf16
  LayerDev* layer_dev = nullptr;                // device [n_layers]: weights of every layer (multi-layer launches)
  uint64_t* hwords = nullptr;                   // device [H] tagged: a multi-layer launch's intermediate outputs
  uint16_t* io_in = nullptr;                    // device staging of the *_host calls: [max_tokens][H] bf16 in,
  uint16_t* io_out = nullptr;                   //   [max_tokens][H] bf16 out,
  int32_t* io_idx = nullptr;                    //   [max_tokens][K] expert indices,
  float* io_w = nullptr;                        //   [max_tokens][K] weights
  void* bws_mem = nullptr;  // batched-path workspace (max_tokens > 1)
  BatchWs bws{};
  std::vector<TmaDesc> tc_maps;  // per layer: tensor maps of the packed gate/up and down matrices
  void* gemm_events[4] = {nullptr, nullptr, nullptr, nullptr};  // caller's timing events (fmoe_set_gemm_events)
  DecodePlan plan[3];  // per mode: layer, expert, route (pointers filled per call)
  // host-resident routed experts (fmoe_create_cached)
  bool cached = false;
  int n_cache_slots = 0;
  std::vector<const uint8_t*> host_dev;  // per layer: device address of the page-locked expert blobs
  uint8_t* shared_dev = nullptr;         // [n_layers] packed shared experts in HBM
  uint8_t* cache_slots = nullptr;        // [n_cache_slots] blobs in HBM
  void* cache_state = nullptr;           // slot_of | owner | ref | hand | stats
  int32_t* slot_of = nullptr;
  int32_t* owner = nullptr;
  uint8_t* ref = nullptr;
  uint32_t* hand = nullptr;
  unsigned long long* stats = nullptr;
  std::string err;
};

namespace {

std::mutex g_mu;
std::set<const fmoe_ctx*> g_live;
thread_local std::string g_create_err;

bool alive(const fmoe_ctx* c) {
  std::lock_guard<std::mutex> lk(g_mu);
  return c != nullptr && g_live.count(c) != 0;
}

fmoe_status fail(fmoe_ctx* c, fmoe_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  if (c) c->err = buf;
  else g_create_err = buf;
  return st;
}

bool misaligned(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; }

uint32_t align_up(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }

// Shared-memory layout of the fused kernel for one mode; false if it does not fit.
bool make_plan(const fmoe_config& c, int grid, int mode, int max_smem, DecodePlan& P) {
  memset(&P, 0, sizeof P);
  P.H = c.hidden;
  P.E = c.n_experts;
  P.K = c.top_k;
  P.I = c.inter;
  P.bits = c.bits;
  P.mode = mode;
  P.n_slots = mode == kModeLayer ? c.top_k + 1 : (mode == kModeExpert ? 1 : 0);
  P.grid = grid;
  P.tb = tile_bytes(c.bits);
  P.cb = tile_code_bytes(c.bits);
  P.gu_tiles = c.hidden / kGroup;
  const int ct = chunk_tiles(c.bits);
  P.gu_chunks = (P.gu_tiles + ct - 1) / ct;
  P.dn_tiles = c.inter / kGroup;
  P.dn_chunks = (P.dn_tiles + ct - 1) / ct;
  P.units_per_slot = c.inter / 8;
  P.total_units = P.n_slots * P.units_per_slot;
  P.units_per_cta = (P.total_units + grid - 1) / grid;
  P.n_rb = c.hidden / 16;
  P.rb_per_cta = P.n_slots > 0 ? (P.n_rb + grid - 1) / grid : 0;
  const bool router = mode != kModeExpert;
  P.router_rows = router ? (c.n_experts + grid - 1) / grid : 0;
  // A router row is one task when it fits an expert stage (one copy, one warp);
  // otherwise it is split into up to 4 non-empty parts of whole 64-column groups.
  const int rgroups = c.hidden / kGroup;
  const uint32_t expert_stage = (uint32_t)std::max(std::min(ct, c.hidden / kGroup),
                                                   std::min(ct, c.inter / kGroup)) * tile_bytes(c.bits);
  const int per_part = ((uint32_t)c.hidden * 2 <= expert_stage) ? rgroups : (rgroups + 3) / 4;
  P.router_part_cols = per_part * kGroup;
  P.router_parts = (rgroups + per_part - 1) / per_part;
  const int max_tasks =
      P.router_rows * P.router_parts + P.units_per_cta * P.gu_chunks + P.rb_per_cta * P.n_slots * P.dn_chunks;
  if (max_tasks > kMaxTasks || P.units_per_cta > 32 || P.rb_per_cta * P.n_slots > 32 || P.router_rows > 16)
    return false;

  uint32_t stage = 0;
  if (P.total_units > 0) {
    stage = std::max<uint32_t>(stage, (uint32_t)(std::min(ct, P.gu_tiles) * P.tb));
    stage = std::max<uint32_t>(stage, (uint32_t)(std::min(ct, P.dn_tiles) * P.tb));
  }
  if (router) stage = std::max<uint32_t>(stage, (uint32_t)P.router_part_cols * 2);
  P.stage_bytes = align_up(stage, 128);

  // fixed regions after the ring
  uint32_t off = 0;
  uint32_t fixed = 0;
  auto region = [&](uint32_t bytes) {
    uint32_t o = fixed;
    fixed = align_up(fixed + bytes, 128);
    return o;
  };
  const uint32_t r_z = region((uint32_t)c.hidden * 2);
  const uint32_t r_lg = region(router ? (uint32_t)c.n_experts * 4 : 4u);
  const uint32_t r_zfrag = region((uint32_t)c.hidden * 2);
  const uint32_t r_zinfo = region((uint32_t)(c.hidden / kGroup) * 8);
  P.afrag_bytes = align_up((uint32_t)c.inter * 2, 128);
  P.ainfo_bytes = align_up((uint32_t)(c.inter / kGroup) * 8, 128);
  const uint32_t r_afrag = region((uint32_t)std::max(P.n_slots, 1) * P.afrag_bytes);
  const uint32_t r_ainfo = region((uint32_t)std::max(P.n_slots, 1) * P.ainfo_bytes);
  const uint32_t r_gupart = region((uint32_t)(std::max(P.units_per_cta, 1) * P.gu_chunks * 16 * 4));
  const uint32_t r_dnpart = region((uint32_t)(std::max(P.rb_per_cta * P.n_slots, 1) * P.dn_chunks * 16 * 4));
  const uint32_t r_y = region((uint32_t)(std::max(P.rb_per_cta, 1) * std::max(P.n_slots, 1) * 16 * 4));
  const uint32_t r_tasks = region((uint32_t)kMaxTasks * 4);
  const uint32_t r_misc = region((uint32_t)sizeof(Misc));
  // Down jobs get a stage each after the ring when that leaves the ring at
  // least min_ring_stages(bits) stages (else they share the ring, streamed last).  A
  // ring stage turns over in about one loaded HBM round trip plus one task's
  // processing (~1.5 + ~1.7 us), so keeping HBM busy takes ~180 KB of stages
  // per SM at 4-bit; a shallower ring loses more than early down weights gain.
  // The ring takes as many stages as still fit (<= 64 in all, <= its tasks).
  auto fit_ring = [&](int n_down) {
    const int ring_tasks = std::max(max_tasks - n_down, 1);
    for (int ns = std::min(64 - n_down, ring_tasks); ns >= 1; --ns) {
      const int all = ns + n_down;
      uint32_t total = align_up((uint32_t)all * P.stage_bytes, 128) + fixed + align_up((uint32_t)(2 * all * 8), 128);
      if ((int)total <= max_smem) return ns;
    }
    return 0;
  };
  P.n_down_max = P.n_slots > 0 ? P.rb_per_cta * P.n_slots * P.dn_chunks : 0;
  int nstage = P.n_down_max > 0 && P.n_down_max <= 32 ? fit_ring(P.n_down_max) : 0;
  if (nstage < std::min(min_ring_stages(c.bits), std::max(max_tasks - P.n_down_max, 1))) {
    P.n_down_max = 0;
    nstage = fit_ring(0);
  }
  if (nstage < 1) return false;
  // several issuing lanes (one copy instruction in flight per lane); keep the
  // largest ring that divides evenly among 4..8 of them
  int best_ni = 1, best_ns = nstage;
  if (nstage >= 4) {
    best_ns = 0;
    for (int ni = std::min(8, nstage); ni >= 4; --ni)
      if (nstage / ni * ni > best_ns) {
        best_ns = nstage / ni * ni;
        best_ni = ni;
      }
  } else {
    best_ni = nstage;
  }
  nstage = best_ns;
  P.n_issuers = best_ni;
  P.nstage = nstage;
  P.off_ring = off;
  off = align_up((uint32_t)(nstage + P.n_down_max) * P.stage_bytes, 128);
  P.off_z = off + r_z;
  P.off_lg = off + r_lg;
  P.off_zfrag = off + r_zfrag;
  P.off_zinfo = off + r_zinfo;
  P.off_afrag = off + r_afrag;
  P.off_ainfo = off + r_ainfo;
  P.off_gupart = off + r_gupart;
  P.off_dnpart = off + r_dnpart;
  P.off_y = off + r_y;
  P.off_tasks = off + r_tasks;
  P.off_misc = off + r_misc;
  off += fixed;
  P.off_bar = off;
  off = align_up(off + (uint32_t)(2 * (nstage + P.n_down_max) * 8), 128);
  P.smem_bytes = off;
  return (int)P.smem_bytes <= max_smem;
}

bool plan_all(fmoe_ctx* ctx, int max_smem) {
  const int modes[3] = {kModeLayer, kModeExpert, kModeRoute};
  for (int m = 0; m < 3; ++m)
    if (!make_plan(ctx->cfg, ctx->n_sm, modes[m], max_smem, ctx->plan[m])) return false;
  return true;
}

fmoe_status cuda_fail(fmoe_ctx* c, cudaError_t e, const char* what) {
  return fail(c, FMOE_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

fmoe_status check_ctx_layer(fmoe_ctx* ctx, int32_t layer, int32_t T) {
  if (layer < 0 || layer >= ctx->cfg.n_layers) return fail(ctx, FMOE_ERR_INVALID_ARG, "layer %d out of range", layer);
  if (T < 0 || T > ctx->cfg.max_tokens)
    return fail(ctx, FMOE_ERR_INVALID_ARG, "T=%d outside [0, max_tokens=%d]", T, ctx->cfg.max_tokens);
  return FMOE_OK;
}

// Fills the per-call pointers of a plan.
DecodePlan bind(const fmoe_ctx* ctx, int mode, int layer) {
  DecodePlan P = ctx->plan[mode];
  const fmoe_layer_desc& L = ctx->layers[layer];
  P.experts = static_cast<const uint8_t*>(L.experts_dev);
  P.blob_bytes = expert_bytes(ctx->cfg.hidden, ctx->cfg.inter, ctx->cfg.bits);
  P.router_w = static_cast<const uint16_t*>(L.router_w_dev);
  P.router_bias = L.router_bias_dev;
  P.norm_w = static_cast<const uint16_t*>(L.norm_w_dev);
  P.eps = ctx->cfg.rms_eps;
  P.ws = ctx->hdr;
  P.ws_logits = ctx->logits;
  P.ws_a = ctx->act;
  P.tasks = ctx->tasks + (size_t)mode * ctx->n_sm * kMaxTasks;
  P.n_tasks = ctx->ntasks + (size_t)mode * ctx->n_sm;
  P.flags = ctx->cfg.flags;
  P.trace = ctx->trace;
  P.timeout_ns = (uint64_t)(ctx->cfg.wait_timeout_us ? ctx->cfg.wait_timeout_us : 1000000u) * 1000ull;
  P.cache = CacheArgs{};
  if (ctx->cached) {
    P.experts = ctx->host_dev[layer];
    if (mode == kModeLayer) {
      CacheArgs& C = P.cache;
      C.on = 1;
      C.n_slots = ctx->n_cache_slots;
      C.key0 = layer * ctx->cfg.n_experts;
      C.host = ctx->host_dev[layer];
      C.shared = ctx->shared_dev + (size_t)layer * P.blob_bytes;
      C.slots = ctx->cache_slots;
      C.slot_of = ctx->slot_of;
      C.owner = ctx->owner;
      C.ref = ctx->ref;
      C.hand = ctx->hand;
      C.stats = ctx->stats;
    }
  }
  return P;
}

fmoe_status launch(fmoe_ctx* ctx, const DecodePlan& P, void* stream) {
  // A launch tags its words epoch + 1 .. epoch + layers.  Before the tags would
  // pass 2^32 - 1, the tagged words and the epoch are cleared (stream-ordered),
  // so a tag never wraps to a value that stale words still carry.
  const uint64_t n_tags = (uint64_t)std::max(P.n_layers, 1);
  if (ctx->tags_used + n_tags > 0xFFFFFFFFull) {
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e = cudaMemsetAsync(&ctx->hdr->epoch, 0, sizeof(uint32_t), st);
    if (e == cudaSuccess) e = cudaMemsetAsync(ctx->logits, 0, ctx->tagged_bytes, st);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return cuda_fail(ctx, e, "tag reset");
    }
    ctx->tags_used = 0;
  }
  int rc = launch_decode(P, stream, true, ctx->pdl_ok);
  if (rc != 0 && ctx->pdl_ok) {
    cudaGetLastError();
    rc = launch_decode(P, stream, true, false);
    if (rc == 0) ctx->pdl_ok = false;
  }
  if (rc != 0) {
    cudaGetLastError();
    return cuda_fail(ctx, (cudaError_t)rc, "decode launch");
  }
  ctx->tags_used += n_tags;
  return FMOE_OK;
}

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  auto x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

}  // namespace

namespace fmoe {

// A block's ordered work list: its router row parts; the slot-0 expert's
// gate/up K-chunks (known before routing); the routed experts' gate/up chunks
// in unit order; then every down job, slot by slot.  A down job waits for
// other blocks' activations and holds its ring stage while it waits, so all of
// them come after the last gate/up chunk: the producer has issued every
// gate/up copy before any stage can be held up, and the down weights land
// while the activations are being exchanged.
int build_task_list(const DecodePlan& P, int cta, uint32_t* out) {
  const int G = P.grid;
  const int my_units = P.total_units > cta ? (P.total_units - cta + G - 1) / G : 0;
  const int first_rb = G - 1 - cta;
  const int my_rb = (P.n_slots > 0 && first_rb < P.n_rb) ? (P.n_rb - first_rb + G - 1) / G : 0;
  const int my_rrows = (P.mode != kModeExpert && cta < P.E) ? (P.E - cta + G - 1) / G : 0;
  int n = 0;
  for (int j = 0; j < my_rrows; ++j)
    for (int q = 0; q < P.router_parts; ++q) out[n++] = make_task(kTaskRouter, j, 0, q);
  // the slot-0 expert (shared, or the single expert) needs no routing: its
  // gate/up chunks go first, ahead of every routed chunk
  int j = 0;
  for (; j < my_units && (cta + j * G) / P.units_per_slot == 0; ++j)
    for (int c = 0; c < P.gu_chunks; ++c) out[n++] = make_task(kTaskGateUp, j, 0, c);
  for (; j < my_units; ++j) {
    const int slot = (cta + j * G) / P.units_per_slot;
    for (int c = 0; c < P.gu_chunks; ++c) out[n++] = make_task(kTaskGateUp, j, slot, c);
  }
  for (int d = 0; d < P.n_slots; ++d)
    for (int r = 0; r < my_rb; ++r)
      for (int c = 0; c < P.dn_chunks; ++c) out[n++] = make_task(kTaskDown, r, d, c);
  return n;
}

}  // namespace fmoe

extern "C" {

size_t fmoe_expert_bytes(int32_t hidden, int32_t inter, int32_t bits) {
  if (hidden <= 0 || inter <= 0 || hidden % kGroup || inter % kGroup || (bits != 2 && bits != 4)) return 0;
  return (size_t)expert_bytes(hidden, inter, bits);
}

const char* fmoe_last_error(const fmoe_ctx* ctx) {
  if (ctx == nullptr) return g_create_err.c_str();
  if (!alive(ctx)) return "invalid or destroyed context";
  return ctx->err.c_str();
}

namespace {
// fmoe_create and fmoe_create_cached: cache_slots > 0 makes a context whose
// routed experts stay in page-locked host memory (layers[l].experts_dev is a
// host pointer) behind an HBM cache of that many expert slots.
fmoe_status create_impl(const fmoe_config* cfg, const fmoe_layer_desc* layers, int64_t cache_slots, void* stream,
                        fmoe_ctx** out) {
  if (out) *out = nullptr;
  if (!cfg || !layers || !out) return fail(nullptr, FMOE_ERR_INVALID_ARG, "NULL argument");
  fmoe_config c = *cfg;
  if (c.max_tokens == 0) c.max_tokens = 256;
  const bool cached = cache_slots > 0;
  if (cached) {
    // one launch per layer and token on the batch-1 kernel: the cache is
    // consulted per launch, and the grouped path needs resident weights
    c.flags = (c.flags | FMOE_FLAG_FORCE_PER_TOKEN | FMOE_FLAG_STACK_PER_LAYER) & ~FMOE_FLAG_FORCE_GROUPED;
    if (cfg->flags & FMOE_FLAG_FORCE_GROUPED)
      return fail(nullptr, FMOE_ERR_UNSUPPORTED, "host-resident experts run on the batch-1 kernel only");
    if (cache_slots < 2 * (int64_t)c.top_k)
      return fail(nullptr, FMOE_ERR_INVALID_ARG, "cache_slots=%lld below 2 * top_k", (long long)cache_slots);
    if (c.n_layers > 0 && c.n_experts > 0 && (int64_t)c.n_layers * c.n_experts > INT32_MAX)
      return fail(nullptr, FMOE_ERR_UNSUPPORTED, "n_layers * n_experts above 2^31");
    if (cache_slots > (int64_t)c.n_layers * std::max(c.n_experts, 1)) cache_slots = (int64_t)c.n_layers * c.n_experts;
  }
  if (c.hidden <= 0 || c.hidden % kGroup)
    return fail(nullptr, FMOE_ERR_INVALID_ARG, "hidden=%d must be a positive multiple of 64", c.hidden);
  if (c.inter <= 0 || c.inter % kGroup)
    return fail(nullptr, FMOE_ERR_INVALID_ARG, "inter=%d must be a positive multiple of 64", c.inter);
  if (c.n_experts <= 0) return fail(nullptr, FMOE_ERR_INVALID_ARG, "n_experts=%d", c.n_experts);
  if (c.top_k <= 0 || c.top_k > c.n_experts)
    return fail(nullptr, FMOE_ERR_INVALID_ARG, "top_k=%d must be in [1, n_experts=%d]", c.top_k, c.n_experts);
  if (c.bits != 2 && c.bits != 4) return fail(nullptr, FMOE_ERR_INVALID_ARG, "bits=%d must be 2 or 4", c.bits);
  if (c.group != kGroup) return fail(nullptr, FMOE_ERR_INVALID_ARG, "group=%d must be 64", c.group);
  if (c.n_layers <= 0) return fail(nullptr, FMOE_ERR_INVALID_ARG, "n_layers=%d", c.n_layers);
  if (c.max_tokens < 0) return fail(nullptr, FMOE_ERR_INVALID_ARG, "max_tokens=%d", c.max_tokens);
  if (!(c.rms_eps >= 0.f)) return fail(nullptr, FMOE_ERR_INVALID_ARG, "rms_eps must be >= 0");
  if (c.top_k > kMaxTopK) return fail(nullptr, FMOE_ERR_UNSUPPORTED, "top_k=%d above %d", c.top_k, kMaxTopK);
  if (c.hidden > kMaxHidden || c.inter > 4096)
    return fail(nullptr, FMOE_ERR_UNSUPPORTED, "hidden=%d / inter=%d above 4096", c.hidden, c.inter);
  if (c.n_experts > 65536) return fail(nullptr, FMOE_ERR_UNSUPPORTED, "n_experts=%d above 65536", c.n_experts);
  for (int l = 0; l < c.n_layers; ++l) {
    const fmoe_layer_desc& L = layers[l];
    if (!L.router_w_dev || !L.experts_dev)
      return fail(nullptr, FMOE_ERR_INVALID_ARG, "layer %d: NULL router or experts pointer", l);
    if (misaligned(L.router_w_dev) || misaligned(L.experts_dev) || misaligned(L.router_bias_dev) ||
        misaligned(L.norm_w_dev))
      return fail(nullptr, FMOE_ERR_ALIGNMENT, "layer %d: pointer not 16-byte aligned", l);
  }

  fmoe_ctx* ctx = new fmoe_ctx();
  ctx->cfg = c;
  ctx->layers.assign(layers, layers + c.n_layers);
  auto bail = [&](fmoe_status st) {
    g_create_err = ctx->err;
    if (ctx->ws) cudaFree(ctx->ws);
    if (ctx->bws_mem) cudaFree(ctx->bws_mem);
    if (ctx->shared_dev) cudaFree(ctx->shared_dev);
    if (ctx->cache_slots) cudaFree(ctx->cache_slots);
    if (ctx->cache_state) cudaFree(ctx->cache_state);
    delete ctx;
    return st;
  };
  if (cached) {
    ctx->cached = true;
    ctx->n_cache_slots = (int)std::min<int64_t>(cache_slots, INT32_MAX);
    for (int l = 0; l < c.n_layers; ++l) {
      cudaPointerAttributes at{};
      cudaError_t pe = cudaPointerGetAttributes(&at, layers[l].experts_dev);
      if (pe != cudaSuccess || at.type != cudaMemoryTypeHost || at.devicePointer == nullptr) {
        cudaGetLastError();
        return bail(fail(ctx, FMOE_ERR_INVALID_ARG,
                         "layer %d: experts must be page-locked host memory (cudaHostAlloc / cudaHostRegister)", l));
      }
      ctx->host_dev.push_back(static_cast<const uint8_t*>(at.devicePointer));
    }
  }
  cudaError_t e = cudaGetDevice(&ctx->device);
  if (e != cudaSuccess) return bail(cuda_fail(ctx, e, "cudaGetDevice"));
  cudaDeviceGetAttribute(&ctx->n_sm, cudaDevAttrMultiProcessorCount, ctx->device);
  {
    const int rc = route_static_prepare();  // the allocation-free router's scratch, looked up outside any capture
    if (rc != 0) return bail(cuda_fail(ctx, (cudaError_t)rc, "fixed router scratch lookup"));
  }
  int coop = 0;
  cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, ctx->device);
  if (!coop) return bail(fail(ctx, FMOE_ERR_UNSUPPORTED, "device lacks cooperative launch"));
  const int max_smem = decode_max_smem_optin(ctx->device);
  if (!plan_all(ctx, max_smem))
    return bail(fail(ctx, FMOE_ERR_UNSUPPORTED, "shared-memory plan does not fit (%d bytes available)", max_smem));
  for (int m = 0; m < 4; ++m) {  // three single-layer plans, then the multi-layer kernel with the layer plan
    int blocks = 0;
    int rc = decode_occupancy(c.bits, m == 3, (int)ctx->plan[m == 3 ? kModeLayer : m].smem_bytes, &blocks);
    if (rc != 0) return bail(cuda_fail(ctx, (cudaError_t)rc, "occupancy query"));
    if (blocks < 1) return bail(fail(ctx, FMOE_ERR_UNSUPPORTED, "fused kernel cannot be resident"));
  }

  // workspace: header | tagged words: logits [E], activations [kMaxSlots][I], layer outputs [H] |
  // task lists | 2 x [max_tokens][H] bf16 | per-layer weight table | staging of the host-buffer calls
  size_t off = 256;
  size_t off_logits = off;
  off += ((size_t)c.n_experts * 8 + 255) / 256 * 256;
  size_t off_act = off;
  off += ((size_t)kMaxSlots * c.inter * 8 + 255) / 256 * 256;
  size_t off_hwords = off;
  off += ((size_t)c.hidden * 8 + 255) / 256 * 256;
  ctx->tagged_bytes = off - off_logits;
  size_t off_tasks = off;
  off += ((size_t)3 * ctx->n_sm * kMaxTasks * 4 + 255) / 256 * 256;
  size_t off_ntasks = off;
  off += ((size_t)3 * ctx->n_sm * 4 + 255) / 256 * 256;
  size_t off_stack = off;
  size_t stack_bytes = ((size_t)std::max(c.max_tokens, 1) * c.hidden * 2 + 255) / 256 * 256;
  off += 2 * stack_bytes;
  size_t off_layers = off;
  off += ((size_t)c.n_layers * sizeof(LayerDev) + 255) / 256 * 256;
  const size_t io_rows = (size_t)std::max(c.max_tokens, 1);
  size_t off_io_in = off;
  off += (io_rows * c.hidden * 2 + 255) / 256 * 256;
  size_t off_io_out = off;
  off += (io_rows * c.hidden * 2 + 255) / 256 * 256;
  size_t off_io_idx = off;
  off += (io_rows * c.top_k * 4 + 255) / 256 * 256;
  size_t off_io_w = off;
  off += (io_rows * c.top_k * 4 + 255) / 256 * 256;
  ctx->ws_bytes = off;
  e = cudaMalloc(&ctx->ws, ctx->ws_bytes);
  if (e != cudaSuccess) {
    cudaGetLastError();
    ctx->ws = nullptr;
    return bail(fail(ctx, FMOE_ERR_OOM, "workspace allocation of %zu bytes failed", ctx->ws_bytes));
  }
  uint8_t* base = static_cast<uint8_t*>(ctx->ws);
  ctx->hdr = reinterpret_cast<WsHeader*>(base);
  ctx->logits = reinterpret_cast<uint64_t*>(base + off_logits);
  ctx->act = reinterpret_cast<uint64_t*>(base + off_act);
  ctx->tasks = reinterpret_cast<uint32_t*>(base + off_tasks);
  ctx->ntasks = reinterpret_cast<int32_t*>(base + off_ntasks);
  ctx->stack_buf[0] = reinterpret_cast<uint16_t*>(base + off_stack);
  ctx->stack_buf[1] = reinterpret_cast<uint16_t*>(base + off_stack + stack_bytes);
  ctx->layer_dev = reinterpret_cast<LayerDev*>(base + off_layers);
  ctx->hwords = reinterpret_cast<uint64_t*>(base + off_hwords);
  ctx->io_in = reinterpret_cast<uint16_t*>(base + off_io_in);
  ctx->io_out = reinterpret_cast<uint16_t*>(base + off_io_out);
  ctx->io_idx = reinterpret_cast<int32_t*>(base + off_io_idx);
  ctx->io_w = reinterpret_cast<float*>(base + off_io_w);
  // batched path: sized for max_tokens, only when more than one token is allowed
  const bool grouped_ok = c.n_experts <= kBatchMaxExperts && c.max_tokens <= kBatchMaxTokens;
  if ((c.flags & FMOE_FLAG_FORCE_GROUPED) && !grouped_ok)
    return bail(fail(ctx, FMOE_ERR_UNSUPPORTED, "grouped path: n_experts=%d (max %d), max_tokens=%d (max %d)",
                     c.n_experts, kBatchMaxExperts, c.max_tokens, kBatchMaxTokens));
  if (!cached && (c.max_tokens > 1 || (c.flags & FMOE_FLAG_FORCE_GROUPED)) && grouped_ok) {
    const size_t bb = batch_ws_bytes(c.hidden, c.n_experts, c.top_k, c.inter, std::max(c.max_tokens, 1));
    e = cudaMalloc(&ctx->bws_mem, bb);
    if (e != cudaSuccess) {
      cudaGetLastError();
      ctx->bws_mem = nullptr;
      return bail(fail(ctx, FMOE_ERR_OOM, "batched workspace allocation of %zu bytes failed", bb));
    }
    const int rc = batch_ws_carve(static_cast<uint8_t*>(ctx->bws_mem), c.hidden, c.n_experts, c.top_k, c.inter,
                                  std::max(c.max_tokens, 1), ctx->bws);
    if (rc != 0) return bail(cuda_fail(ctx, (cudaError_t)rc, "batched tensor maps"));
    // GEMM inputs past a step's positions are read into unused columns: keep them finite
    e = cudaMemsetAsync(ctx->bws_mem, 0, bb, (cudaStream_t)stream);
    if (e != cudaSuccess) return bail(cuda_fail(ctx, e, "batched workspace clear"));
    ctx->tc_maps.resize((size_t)2 * c.n_layers);
    const int64_t blob = expert_bytes(c.hidden, c.inter, c.bits);
    for (int l = 0; l < c.n_layers; ++l) {
      const uint8_t* ex = static_cast<const uint8_t*>(ctx->layers[l].experts_dev);
      int r2 = tc_encode_weight_map(ex, blob, c.n_experts + 1, 2 * c.inter, c.hidden, c.bits, &ctx->tc_maps[2 * l]);
      if (r2 == 0)
        r2 = tc_encode_weight_map(ex + packed_gu_bytes(c.hidden, c.inter, c.bits), blob, c.n_experts + 1, c.hidden,
                                  c.inter, c.bits, &ctx->tc_maps[2 * l + 1]);
      if (r2 != 0) return bail(cuda_fail(ctx, (cudaError_t)r2, "expert tensor maps"));
    }
  }
  cudaStream_t st = (cudaStream_t)stream;
  e = cudaMemsetAsync(ctx->ws, 0, ctx->ws_bytes, st);
  if (e != cudaSuccess) return bail(cuda_fail(ctx, e, "workspace clear"));
  {
    std::vector<uint32_t> tl((size_t)3 * ctx->n_sm * kMaxTasks, 0u);
    std::vector<int32_t> nt((size_t)3 * ctx->n_sm, 0);
    for (int m = 0; m < 3; ++m)
      for (int b = 0; b < ctx->n_sm; ++b)
        nt[(size_t)m * ctx->n_sm + b] =
            build_task_list(ctx->plan[m], b, tl.data() + ((size_t)m * ctx->n_sm + b) * kMaxTasks);
    std::vector<LayerDev> ld((size_t)c.n_layers);
    for (int l = 0; l < c.n_layers; ++l) {
      const fmoe_layer_desc& L = ctx->layers[l];
      ld[l] = LayerDev{static_cast<const uint8_t*>(L.experts_dev), static_cast<const uint16_t*>(L.router_w_dev),
                       L.router_bias_dev, static_cast<const uint16_t*>(L.norm_w_dev)};
    }
    e = cudaMemcpyAsync(ctx->tasks, tl.data(), tl.size() * 4, cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) e = cudaMemcpyAsync(ctx->ntasks, nt.data(), nt.size() * 4, cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(ctx->layer_dev, ld.data(), ld.size() * sizeof(LayerDev), cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return bail(cuda_fail(ctx, e, "task table upload"));
  }

  // In-place repack, canonical -> packed, through a bounded staging buffer
  // (host-resident experts: through two, the packed blobs copied back; the
  // shared expert also kept in HBM).
  const size_t blob = (size_t)expert_bytes(c.hidden, c.inter, c.bits);
  const int per_layer = c.n_experts + 1;
  int chunk = (int)std::max<size_t>(1, std::min<size_t>((size_t)per_layer, (size_t)(256u << 20) / blob));
  if (cached) {
    const size_t state = ((size_t)c.n_layers * c.n_experts * 4 + 255) / 256 * 256 +
                         ((size_t)ctx->n_cache_slots * 4 + 255) / 256 * 256 + ((size_t)ctx->n_cache_slots + 255) / 256 * 256 +
                         256 + 256;
    e = cudaMalloc(&ctx->shared_dev, (size_t)c.n_layers * blob);
    if (e == cudaSuccess) e = cudaMalloc(&ctx->cache_slots, (size_t)ctx->n_cache_slots * blob);
    if (e == cudaSuccess) e = cudaMalloc(&ctx->cache_state, state);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return bail(fail(ctx, FMOE_ERR_OOM, "expert cache allocation (%d slots of %zu bytes) failed",
                       ctx->n_cache_slots, blob));
    }
    uint8_t* cs = static_cast<uint8_t*>(ctx->cache_state);
    size_t o = 0;
    ctx->slot_of = reinterpret_cast<int32_t*>(cs + o);
    o += ((size_t)c.n_layers * c.n_experts * 4 + 255) / 256 * 256;
    ctx->owner = reinterpret_cast<int32_t*>(cs + o);
    o += ((size_t)ctx->n_cache_slots * 4 + 255) / 256 * 256;
    ctx->ref = cs + o;
    o += ((size_t)ctx->n_cache_slots + 255) / 256 * 256;
    ctx->hand = reinterpret_cast<uint32_t*>(cs + o);
    o += 256;
    ctx->stats = reinterpret_cast<unsigned long long*>(cs + o);
    // empty cache: no key has a slot, no slot a key, no reference bits, hand at 0
    e = cudaMemsetAsync(ctx->slot_of, 0xFF, (size_t)c.n_layers * c.n_experts * 4, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(ctx->owner, 0xFF, (size_t)ctx->n_cache_slots * 4, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(ctx->ref, 0, (size_t)ctx->n_cache_slots, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(ctx->hand, 0, 512, st);
    if (e != cudaSuccess) return bail(cuda_fail(ctx, e, "expert cache clear"));
  }
  void* tmp = nullptr;
  void* tmp2 = nullptr;
  e = cudaMalloc(&tmp, (size_t)chunk * blob);
  if (e == cudaSuccess && cached) e = cudaMalloc(&tmp2, (size_t)chunk * blob);
  if (e != cudaSuccess) {
    cudaGetLastError();
    if (tmp) cudaFree(tmp);
    return bail(fail(ctx, FMOE_ERR_OOM, "repack staging allocation failed"));
  }
  for (int l = 0; l < c.n_layers && e == cudaSuccess; ++l) {
    uint8_t* ex = static_cast<uint8_t*>(ctx->layers[l].experts_dev);
    for (int e0 = 0; e0 < per_layer; e0 += chunk) {
      int n = std::min(chunk, per_layer - e0);
      uint8_t* dst = cached ? static_cast<uint8_t*>(tmp2) : ex + (size_t)e0 * blob;
      e = cudaMemcpyAsync(tmp, ex + (size_t)e0 * blob, (size_t)n * blob, cudaMemcpyDefault, st);
      if (e != cudaSuccess) break;
      int rc = launch_repack(static_cast<const uint8_t*>(tmp), dst, n, c.hidden, c.inter, c.bits, 1, stream);
      if (rc != 0) { e = (cudaError_t)rc; break; }
      if (cached) {
        e = cudaMemcpyAsync(ex + (size_t)e0 * blob, dst, (size_t)n * blob, cudaMemcpyDeviceToHost, st);
        if (e == cudaSuccess && e0 + n == per_layer)  // the chunk ends with the shared expert
          e = cudaMemcpyAsync(ctx->shared_dev + (size_t)l * blob, dst + (size_t)(n - 1) * blob, blob,
                              cudaMemcpyDeviceToDevice, st);
        // the staging buffers are reused by the next chunk
        if (e == cudaSuccess) e = cudaStreamSynchronize(st);
        if (e != cudaSuccess) break;
      }
    }
  }
  cudaError_t e2 = cudaStreamSynchronize(st);
  cudaFree(tmp);
  if (tmp2) cudaFree(tmp2);
  if (e != cudaSuccess) return bail(cuda_fail(ctx, e, "expert repack"));
  if (e2 != cudaSuccess) return bail(cuda_fail(ctx, e2, "expert repack (sync)"));
  {
    std::lock_guard<std::mutex> lk(g_mu);
    g_live.insert(ctx);
  }
  *out = ctx;
  return FMOE_OK;
}
}  // namespace

fmoe_status fmoe_create(const fmoe_config* cfg, const fmoe_layer_desc* layers, void* stream, fmoe_ctx** out) {
  return create_impl(cfg, layers, 0, stream, out);
}

fmoe_status fmoe_create_cached(const fmoe_config* cfg, const fmoe_layer_desc* layers, int64_t cache_slots,
                               void* stream, fmoe_ctx** out) {
  if (cache_slots <= 0) {
    if (out) *out = nullptr;
    return fail(nullptr, FMOE_ERR_INVALID_ARG, "cache_slots=%lld must be positive", (long long)cache_slots);
  }
  return create_impl(cfg, layers, cache_slots, stream, out);
}

fmoe_status fmoe_cache_stats(fmoe_ctx* ctx, void* stream, uint64_t* hits, uint64_t* misses) {
  if (!alive(ctx)) return fail(nullptr, FMOE_ERR_INVALID_ARG, "invalid or destroyed context");
  if (!ctx->cached) return fail(ctx, FMOE_ERR_INVALID_ARG, "context has no expert cache");
  unsigned long long v[2] = {0, 0};
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = cudaMemcpyAsync(v, ctx->stats, sizeof v, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(ctx, e, "cache statistics");
  if (hits) *hits = v[0];
  if (misses) *misses = v[1];
  return FMOE_OK;
}

fmoe_status fmoe_destroy(fmoe_ctx* ctx) {
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (ctx == nullptr || g_live.erase(ctx) == 0) {
      g_create_err = "fmoe_destroy: invalid or destroyed context";
      return FMOE_ERR_INVALID_ARG;
    }
  }
  if (ctx->ws) cudaFree(ctx->ws);
  if (ctx->bws_mem) cudaFree(ctx->bws_mem);
  if (ctx->shared_dev) cudaFree(ctx->shared_dev);
  if (ctx->cache_slots) cudaFree(ctx->cache_slots);
  if (ctx->cache_state) cudaFree(ctx->cache_state);
  delete ctx;
  return FMOE_OK;
}

// The batched path takes T >= kGroupedMinTokens tokens (any T with
// FORCE_GROUPED) unless FORCE_PER_TOKEN asks for one batch-1 launch per token.
static bool use_batched(const fmoe_ctx* ctx, int32_t T) {
  if (ctx->bws_mem == nullptr) return false;
  if (ctx->cfg.flags & FMOE_FLAG_FORCE_GROUPED) return true;
  if (ctx->cfg.flags & FMOE_FLAG_FORCE_PER_TOKEN) return false;
  return T >= kGroupedMinTokens;
}

static BatchArgs batch_args(const fmoe_ctx* ctx, int32_t layer, int32_t T) {
  const fmoe_config& c = ctx->cfg;
  const fmoe_layer_desc& L = ctx->layers[layer];
  BatchArgs a{};
  a.H = c.hidden;
  a.E = c.n_experts;
  a.K = c.top_k;
  a.I = c.inter;
  a.bits = c.bits;
  a.T = T;
  a.experts = static_cast<const uint8_t*>(L.experts_dev);
  a.blob_bytes = expert_bytes(c.hidden, c.inter, c.bits);
  a.router_w = static_cast<const uint16_t*>(L.router_w_dev);
  a.router_bias = L.router_bias_dev;
  a.norm_w = static_cast<const uint16_t*>(L.norm_w_dev);
  a.eps = c.rms_eps;
  a.single_expert = -1;
  if (!ctx->tc_maps.empty()) {
    a.wmap_gu = &ctx->tc_maps[2 * (size_t)layer];
    a.wmap_dn = &ctx->tc_maps[2 * (size_t)layer + 1];
  }
  a.status = &ctx->hdr->status;
  for (int k = 0; k < 4; ++k) a.gemm_events[k] = ctx->gemm_events[k];
  return a;
}

static fmoe_status run_batched(fmoe_ctx* ctx, const BatchArgs& a, void* stream) {
  const int rc = launch_batched(a, ctx->bws, ctx->n_sm, stream);
  if (rc != 0) {
    cudaGetLastError();
    return cuda_fail(ctx, (cudaError_t)rc, "batched launch");
  }
  return FMOE_OK;
}

fmoe_status fmoe_route(fmoe_ctx* ctx, int32_t layer, const void* x_dev, int32_t T, int32_t* idx_dev, float* w_dev,
                       void* stream) {
  if (!alive(ctx)) return fail(nullptr, FMOE_ERR_INVALID_ARG, "invalid or destroyed context");
  fmoe_status s = check_ctx_layer(ctx, layer, T);
  if (s != FMOE_OK) return s;
  if (T == 0) return FMOE_OK;
  if (!x_dev || !idx_dev || !w_dev) return fail(ctx, FMOE_ERR_INVALID_ARG, "NULL tensor");
  if (misaligned(x_dev) || misaligned(idx_dev) || misaligned(w_dev))
    return fail(ctx, FMOE_ERR_ALIGNMENT, "tensor not 16-byte aligned");
  const int H = ctx->cfg.hidden, K = ctx->cfg.top_k;
  for (int t = 0; t < T; ++t) {
    DecodePlan P = bind(ctx, kModeRoute, layer);
    P.h_in = static_cast<const uint16_t*>(x_dev) + (size_t)t * H;
    P.idx_out = idx_dev + (size_t)t * K;
    P.w_out = w_dev + (size_t)t * K;
    s = launch(ctx, P, stream);
    if (s != FMOE_OK) return s;
  }
  return FMOE_OK;
}

fmoe_status fmoe_route_static(fmoe_ctx* ctx, int32_t layer, const void* x_dev, int32_t T, int32_t* idx_dev,
                              float* w_dev, void* stream) {
  if (!alive(ctx)) return fail(nullptr, FMOE_ERR_INVALID_ARG, "invalid or destroyed context");
  fmoe_status s = check_ctx_layer(ctx, layer, T);
  if (s != FMOE_OK) return s;
  if (T == 0) return FMOE_OK;
  if (!x_dev || !idx_dev || !w_dev) return fail(ctx, FMOE_ERR_INVALID_ARG, "NULL tensor");
  if (misaligned(x_dev) || misaligned(idx_dev) || misaligned(w_dev))
    return fail(ctx, FMOE_ERR_ALIGNMENT, "tensor not 16-byte aligned");
  const fmoe_config& c = ctx->cfg;
  if ((int64_t)T * c.n_experts > kStaticRouteLogits || T > kStaticRouteMaxTokens)
    return fail(ctx, FMOE_ERR_UNSUPPORTED, "T=%d x E=%d exceeds the fixed scratch (%d logits, %d tokens)", T,
                c.n_experts, kStaticRouteLogits, kStaticRouteMaxTokens);
  if (!route_static_ready()) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing((cudaStream_t)stream, &cs) != cudaSuccess) cudaGetLastError();
    if (cs != cudaStreamCaptureStatusNone)
      return fail(ctx, FMOE_ERR_UNSUPPORTED,
                  "first fmoe_route_static call on this device is inside a stream capture; call it (or create a "
                  "context on this device) before capturing");
  }
  const fmoe_layer_desc& L = ctx->layers[layer];
  const int rc = launch_route_static(static_cast<const uint16_t*>(L.router_w_dev), L.router_bias_dev,
                                     static_cast<const uint16_t*>(L.norm_w_dev), c.rms_eps,
                                     static_cast<const uint16_t*>(x_dev), T, c.hidden, c.n_experts, c.top_k, idx_dev,
                                     w_dev, stream);
  if (rc != 0) {
    cudaGetLastError();
    return cuda_fail(ctx, (cudaError_t)rc, "static route launch");
  }
  return FMOE_OK;
}

fmoe_status fmoe_expert_forward(fmoe_ctx* ctx, int32_t layer, int32_t expert, const void* x_dev, int32_t T,
                                float* y_dev, void* stream) {
  if (!alive(ctx)) return fail(nullptr, FMOE_ERR_INVALID_ARG, "invalid or destroyed context");
  fmoe_status s = check_ctx_layer(ctx, layer, T);
  if (s != FMOE_OK) return s;
  if (expert < -1 || expert >= ctx->cfg.n_experts)
    return fail(ctx, FMOE_ERR_INVALID_ARG, "expert %d outside [-1, %d)", expert, ctx->cfg.n_experts);
  if (ctx->cached)
    return fail(ctx, FMOE_ERR_UNSUPPORTED, "host-resident experts: single-expert calls are not supported");
  if (T == 0) return FMOE_OK;
  if (!x_dev || !y_dev) return fail(ctx, FMOE_ERR_INVALID_ARG, "NULL tensor");
  if (misaligned(x_dev) || misaligned(y_dev)) return fail(ctx, FMOE_ERR_ALIGNMENT, "tensor not 16-byte aligned");
  if (use_batched(ctx, T)) {
    BatchArgs a = batch_args(ctx, layer, T);
    a.h_in = static_cast<const uint16_t*>(x_dev);
    a.single_expert = expert < 0 ? ctx->cfg.n_experts : expert;
    a.y_out = y_dev;
    return run_batched(ctx, a, stream);
  }
  const int H = ctx->cfg.hidden;
  for (int t = 0; t < T; ++t) {
    DecodePlan P = bind(ctx, kModeExpert, layer);
    P.expert_id = expert < 0 ? ctx->cfg.n_experts : expert;
    P.h_in = static_cast<const uint16_t*>(x_dev) + (size_t)t * H;
    P.y_out = y_dev + (size_t)t * H;
    s = launch(ctx, P, stream);
    if (s != FMOE_OK) return s;
  }
  return FMOE_OK;
}

static fmoe_status layer_tokens(fmoe_ctx* ctx, int32_t layer, const uint16_t* h_in, int32_t T, uint16_t* h_out,
                                int32_t* idx, float* w, void* stream) {
  if (use_batched(ctx, T)) {
    BatchArgs a = batch_args(ctx, layer, T);
    a.h_in = h_in;
    a.h_out = h_out;
    a.idx_out = idx;
    a.w_out = w;
    return run_batched(ctx, a, stream);
  }
  const int H = ctx->cfg.hidden, K = ctx->cfg.top_k;
  for (int t = 0; t < T; ++t) {
    DecodePlan P = bind(ctx, kModeLayer, layer);
    P.h_in = h_in + (size_t)t * H;
    P.h_out = h_out + (size_t)t * H;
    P.idx_out = idx ? idx + (size_t)t * K : nullptr;
    P.w_out = w ? w + (size_t)t * K : nullptr;
    fmoe_status s = launch(ctx, P, stream);
    if (s != FMOE_OK) return s;
  }
  return FMOE_OK;
}

fmoe_status fmoe_layer_forward(fmoe_ctx* ctx, int32_t layer, const void* h_in_dev, int32_t T, void* h_out_dev,
                               int32_t* idx_out_dev, float* w_out_dev, void* stream) {
  if (!alive(ctx)) return fail(nullptr, FMOE_ERR_INVALID_ARG, "invalid or destroyed context");
  fmoe_status s = check_ctx_layer(ctx, layer, T);
  if (s != FMOE_OK) return s;
  if (T == 0) return FMOE_OK;
  if (!h_in_dev || !h_out_dev) return fail(ctx, FMOE_ERR_INVALID_ARG, "NULL tensor");
  if (misaligned(h_in_dev) || misaligned(h_out_dev) || misaligned(idx_out_dev) || misaligned(w_out_dev))
    return fail(ctx, FMOE_ERR_ALIGNMENT, "tensor not 16-byte aligned");
  const size_t bytes = (size_t)T * ctx->cfg.hidden * 2;
  if (overlaps(h_in_dev, bytes, h_out_dev, bytes)) return fail(ctx, FMOE_ERR_INVALID_ARG, "h_out overlaps h_in");
  return layer_tokens(ctx, layer, static_cast<const uint16_t*>(h_in_dev), T, static_cast<uint16_t*>(h_out_dev),
                      idx_out_dev, w_out_dev, stream);
}

static fmoe_status stack_tokens(fmoe_ctx* ctx, int32_t layer_begin, int32_t layer_end, const void* h_in_dev,
                                int32_t T, void* h_out_dev, void* stream) {
  fmoe_status s = FMOE_OK;
  const int n_layers = layer_end - layer_begin;
  if (n_layers > 1 && !use_batched(ctx, T) && !(ctx->cfg.flags & FMOE_FLAG_STACK_PER_LAYER)) {
    // one launch per token runs every layer of the range
    const int H = ctx->cfg.hidden;
    for (int t = 0; t < T; ++t) {
      DecodePlan P = bind(ctx, kModeLayer, layer_begin);
      P.n_layers = n_layers;
      P.layer_dev = ctx->layer_dev + layer_begin;
      P.ws_h = ctx->hwords;
      P.h_in = static_cast<const uint16_t*>(h_in_dev) + (size_t)t * H;
      P.h_out = static_cast<uint16_t*>(h_out_dev) + (size_t)t * H;
      s = launch(ctx, P, stream);
      if (s != FMOE_OK) return s;
    }
    return FMOE_OK;
  }
  const uint16_t* cur = static_cast<const uint16_t*>(h_in_dev);
  for (int l = layer_begin; l < layer_end; ++l) {
    uint16_t* dst = (l + 1 == layer_end) ? static_cast<uint16_t*>(h_out_dev) : ctx->stack_buf[(l - layer_begin) & 1];
    s = layer_tokens(ctx, l, cur, T, dst, nullptr, nullptr, stream);
    if (s != FMOE_OK) return s;
    cur = dst;
  }
  return FMOE_OK;
}

static fmoe_status check_stack_range(fmoe_ctx* ctx, int32_t layer_begin, int32_t layer_end, int32_t T) {
  if (layer_begin < 0 || layer_end > ctx->cfg.n_layers || layer_begin >= layer_end)
    return fail(ctx, FMOE_ERR_INVALID_ARG, "layer range [%d, %d) invalid", layer_begin, layer_end);
  return check_ctx_layer(ctx, layer_begin, T);
}

fmoe_status fmoe_stack_forward(fmoe_ctx* ctx, int32_t layer_begin, int32_t layer_end, const void* h_in_dev, int32_t T,
                               void* h_out_dev, void* stream) {
  if (!alive(ctx)) return fail(nullptr, FMOE_ERR_INVALID_ARG, "invalid or destroyed context");
  fmoe_status s = check_stack_range(ctx, layer_begin, layer_end, T);
  if (s != FMOE_OK) return s;
  if (T == 0) return FMOE_OK;
  if (!h_in_dev || !h_out_dev) return fail(ctx, FMOE_ERR_INVALID_ARG, "NULL tensor");
  if (misaligned(h_in_dev) || misaligned(h_out_dev)) return fail(ctx, FMOE_ERR_ALIGNMENT, "tensor not 16-byte aligned");
  const size_t bytes = (size_t)T * ctx->cfg.hidden * 2;
  if (overlaps(h_in_dev, bytes, h_out_dev, bytes)) return fail(ctx, FMOE_ERR_INVALID_ARG, "h_out overlaps h_in");
  return stack_tokens(ctx, layer_begin, layer_end, h_in_dev, T, h_out_dev, stream);
}

// Host-buffer variants: the input is copied into the context's staging buffer,
// the device path runs on it, and the results are copied back, all enqueued
// on `stream` (plain cudaMemcpyAsync, one per buffer).
static fmoe_status copy_async(fmoe_ctx* ctx, void* dst, const void* src, size_t bytes, cudaMemcpyKind kind,
                              void* stream) {
  if (bytes == 0) return FMOE_OK;
  cudaError_t e = cudaMemcpyAsync(dst, src, bytes, kind, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) {
    cudaGetLastError();
    return cuda_fail(ctx, e, kind == cudaMemcpyHostToDevice ? "host-to-device copy" : "device-to-host copy");
  }
  return FMOE_OK;
}

namespace {
using PointerAttrsFn = CUresult (*)(unsigned int, CUpointer_attribute*, void**, CUdeviceptr);
PointerAttrsFn pointer_attrs_fn() {
  static PointerAttrsFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuPointerGetAttributes", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PointerAttrsFn>(f);
    cudaGetLastError();
  });
  return fn;
}

// Device address of `bytes` of page-locked, device-mapped host memory at p, or
// null: for pageable memory, a failed query, or a buffer that does not lie
// inside one page-locked allocation (a kernel reading or writing past its end
// would fault; the copy path reports the error on the host instead).  One
// driver query per buffer.
void* mapped_host(const void* p, size_t bytes) {
  if (p == nullptr) return nullptr;
  PointerAttrsFn fn = pointer_attrs_fn();
  if (fn == nullptr) return nullptr;
  unsigned int type = 0;
  CUdeviceptr dev = 0, start = 0;
  size_t size = 0;
  CUpointer_attribute at[4] = {CU_POINTER_ATTRIBUTE_MEMORY_TYPE, CU_POINTER_ATTRIBUTE_DEVICE_POINTER,
                               CU_POINTER_ATTRIBUTE_RANGE_START_ADDR, CU_POINTER_ATTRIBUTE_RANGE_SIZE};
  void* data[4] = {&type, &dev, &start, &size};
  const CUdeviceptr addr = (CUdeviceptr)(uintptr_t)p;
  if (fn(4, at, data, addr) != CUDA_SUCCESS) return nullptr;  // pageable memory: zeros and CUDA_SUCCESS
  if (type != CU_MEMORYTYPE_HOST || dev == 0 || size == 0) return nullptr;
  if (addr < start || bytes > size || addr - start > size - bytes) return nullptr;
  return reinterpret_cast<void*>((uintptr_t)dev);
}

// Reads `bytes` (a multiple of 16) from mapped host memory into device memory:
// a few blocks of 16-byte loads over the host link, one round trip for an 8 KB
// token instead of a copy-engine transfer.
__global__ void stage_in_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, size_t n16) {
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n16; i += (size_t)gridDim.x * blockDim.x)
    dst[i] = src[i];
}

// The input of a host-buffer call into the context's staging buffer.
fmoe_status stage_in(fmoe_ctx* ctx, const void* src_mapped, size_t bytes, void* stream) {
  const size_t n16 = bytes / 16;  // H is a multiple of 64: bf16 rows are multiples of 16 bytes
  const int blocks = (int)std::min<size_t>((n16 + 255) / 256, (size_t)ctx->n_sm);
  stage_in_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<const uint4*>(src_mapped),
                                                                        reinterpret_cast<uint4*>(ctx->io_in), n16);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? FMOE_OK : cuda_fail(ctx, e, "input stage-in launch");
}
}  // namespace

fmoe_status fmoe_layer_forward_host(fmoe_ctx* ctx, int32_t layer, const void* h_in_host, int32_t T, void* h_out_host,
                                    int32_t* idx_out_host, float* w_out_host, void* stream) {
  if (!alive(ctx)) return fail(nullptr, FMOE_ERR_INVALID_ARG, "invalid or destroyed context");
  fmoe_status s = check_ctx_layer(ctx, layer, T);
  if (s != FMOE_OK) return s;
  if (T == 0) return FMOE_OK;
  if (!h_in_host || !h_out_host) return fail(ctx, FMOE_ERR_INVALID_ARG, "NULL buffer");
  const size_t bytes = (size_t)T * ctx->cfg.hidden * 2, kbytes = (size_t)T * ctx->cfg.top_k * 4;
  if (!use_batched(ctx, T)) {
    // page-locked buffers: the input is read over the link by a small kernel
    // and the fused kernel writes its outputs straight into host memory
    void* in = mapped_host(h_in_host, bytes);
    void* out = mapped_host(h_out_host, bytes);
    void* idx = mapped_host(idx_out_host, kbytes);
    void* w = mapped_host(w_out_host, kbytes);
    if (in && out && !misaligned(in) && (!idx_out_host || idx) && (!w_out_host || w)) {
      s = stage_in(ctx, in, bytes, stream);
      if (s == FMOE_OK)
        s = layer_tokens(ctx, layer, ctx->io_in, T, static_cast<uint16_t*>(out), static_cast<int32_t*>(idx),
                         static_cast<float*>(w), stream);
      return s;
    }
  }
  s = copy_async(ctx, ctx->io_in, h_in_host, bytes, cudaMemcpyHostToDevice, stream);
  if (s == FMOE_OK)
    s = layer_tokens(ctx, layer, ctx->io_in, T, ctx->io_out, idx_out_host ? ctx->io_idx : nullptr,
                     w_out_host ? ctx->io_w : nullptr, stream);
  if (s == FMOE_OK) s = copy_async(ctx, h_out_host, ctx->io_out, bytes, cudaMemcpyDeviceToHost, stream);
  if (s == FMOE_OK && idx_out_host) s = copy_async(ctx, idx_out_host, ctx->io_idx, kbytes, cudaMemcpyDeviceToHost, stream);
  if (s == FMOE_OK && w_out_host) s = copy_async(ctx, w_out_host, ctx->io_w, kbytes, cudaMemcpyDeviceToHost, stream);
  return s;
}

fmoe_status fmoe_stack_forward_host(fmoe_ctx* ctx, int32_t layer_begin, int32_t layer_end, const void* h_in_host,
                                    int32_t T, void* h_out_host, void* stream) {
  if (!alive(ctx)) return fail(nullptr, FMOE_ERR_INVALID_ARG, "invalid or destroyed context");
  fmoe_status s = check_stack_range(ctx, layer_begin, layer_end, T);
  if (s != FMOE_OK) return s;
  if (T == 0) return FMOE_OK;
  if (!h_in_host || !h_out_host) return fail(ctx, FMOE_ERR_INVALID_ARG, "NULL buffer");
  const size_t bytes = (size_t)T * ctx->cfg.hidden * 2;
  if (!use_batched(ctx, T)) {  // page-locked buffers: as fmoe_layer_forward_host
    void* in = mapped_host(h_in_host, bytes);
    void* out = mapped_host(h_out_host, bytes);
    if (in && out && !misaligned(in)) {
      s = stage_in(ctx, in, bytes, stream);
      if (s == FMOE_OK) s = stack_tokens(ctx, layer_begin, layer_end, ctx->io_in, T, out, stream);
      return s;
    }
  }
  s = copy_async(ctx, ctx->io_in, h_in_host, bytes, cudaMemcpyHostToDevice, stream);
  if (s == FMOE_OK) s = stack_tokens(ctx, layer_begin, layer_end, ctx->io_in, T, ctx->io_out, stream);
  if (s == FMOE_OK) s = copy_async(ctx, h_out_host, ctx->io_out, bytes, cudaMemcpyDeviceToHost, stream);
  return s;
}

fmoe_status fmoe_unpack_expert(fmoe_ctx* ctx, int32_t layer, int32_t expert, void* dst_dev, void* stream) {
  if (!alive(ctx)) return fail(nullptr, FMOE_ERR_INVALID_ARG, "invalid or destroyed context");
  if (layer < 0 || layer >= ctx->cfg.n_layers) return fail(ctx, FMOE_ERR_INVALID_ARG, "layer %d out of range", layer);
  if (expert < -1 || expert >= ctx->cfg.n_experts)
    return fail(ctx, FMOE_ERR_INVALID_ARG, "expert %d outside [-1, %d)", expert, ctx->cfg.n_experts);
  if (!dst_dev) return fail(ctx, FMOE_ERR_INVALID_ARG, "NULL destination");
  if (misaligned(dst_dev)) return fail(ctx, FMOE_ERR_ALIGNMENT, "destination not 16-byte aligned");
  const size_t blob = (size_t)expert_bytes(ctx->cfg.hidden, ctx->cfg.inter, ctx->cfg.bits);
  const int e = expert < 0 ? ctx->cfg.n_experts : expert;
  const uint8_t* src = ctx->cached ? (e == ctx->cfg.n_experts ? ctx->shared_dev + (size_t)layer * blob
                                                                : ctx->host_dev[layer] + (size_t)e * blob)
                                   : static_cast<const uint8_t*>(ctx->layers[layer].experts_dev) + (size_t)e * blob;
  int rc = launch_repack(src, static_cast<uint8_t*>(dst_dev), 1, ctx->cfg.hidden, ctx->cfg.inter, ctx->cfg.bits, 0,
                         stream);
  if (rc != 0) return cuda_fail(ctx, (cudaError_t)rc, "unpack");
  return FMOE_OK;
}

fmoe_status fmoe_requant_4to2(const void* src_dev, int32_t n_blobs, int32_t hidden, int32_t inter, void* dst_dev,
                              void* stream) {
  if (n_blobs < 0) return fail(nullptr, FMOE_ERR_INVALID_ARG, "n_blobs=%d", n_blobs);
  if (hidden <= 0 || hidden % kGroup || inter <= 0 || inter % kGroup)
    return fail(nullptr, FMOE_ERR_INVALID_ARG, "hidden=%d / inter=%d must be positive multiples of 64", hidden, inter);
  if ((int64_t)hidden * inter > (int64_t)1 << 30)
    return fail(nullptr, FMOE_ERR_UNSUPPORTED, "hidden*inter=%lld above 2^30", (long long)hidden * inter);
  if (n_blobs == 0) return FMOE_OK;
  if (!src_dev || !dst_dev) return fail(nullptr, FMOE_ERR_INVALID_ARG, "NULL blob pointer");
  if (misaligned(src_dev) || misaligned(dst_dev)) return fail(nullptr, FMOE_ERR_ALIGNMENT, "blobs not 16-byte aligned");
  const size_t in_bytes = (size_t)n_blobs * (size_t)expert_bytes(hidden, inter, 4);
  const size_t out_bytes = (size_t)n_blobs * (size_t)expert_bytes(hidden, inter, 2);
  if (overlaps(src_dev, in_bytes, dst_dev, out_bytes))
    return fail(nullptr, FMOE_ERR_INVALID_ARG, "destination overlaps the source blobs");
  int dev = 0, n_sm = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return fail(nullptr, FMOE_ERR_CUDA, "device query: %s", cudaGetErrorString(e));
  const int rc = launch_requant(static_cast<const uint8_t*>(src_dev), static_cast<uint8_t*>(dst_dev), n_blobs, hidden,
                                inter, n_sm, stream);
  if (rc != 0) {
    cudaGetLastError();
    return fail(nullptr, FMOE_ERR_CUDA, "requant launch: %s", cudaGetErrorString((cudaError_t)rc));
  }
  return FMOE_OK;
}

fmoe_status fmoe_set_gemm_events(fmoe_ctx* ctx, void* const* events) {
  if (!alive(ctx)) return fail(nullptr, FMOE_ERR_INVALID_ARG, "invalid or destroyed context");
  if (events == nullptr) {
    for (int k = 0; k < 4; ++k) ctx->gemm_events[k] = nullptr;
    return FMOE_OK;
  }
  for (int k = 0; k < 4; ++k)
    if (events[k] == nullptr) return fail(ctx, FMOE_ERR_INVALID_ARG, "event %d is NULL", k);
  for (int k = 0; k < 4; ++k) ctx->gemm_events[k] = events[k];
  return FMOE_OK;
}

fmoe_status fmoe_set_trace(fmoe_ctx* ctx, void* trace_dev) {
  if (!alive(ctx)) return fail(nullptr, FMOE_ERR_INVALID_ARG, "invalid or destroyed context");
  if (misaligned(trace_dev)) return fail(ctx, FMOE_ERR_ALIGNMENT, "trace buffer not 16-byte aligned");
  ctx->trace = static_cast<unsigned long long*>(trace_dev);
  return FMOE_OK;
}

int32_t fmoe_trace_points(void) { return kTracePoints; }
int32_t fmoe_trace_layers(void) { return kTraceLayers; }

fmoe_status fmoe_debug_set_epoch(fmoe_ctx* ctx, uint32_t epoch, void* stream) {
  if (!alive(ctx)) return fail(nullptr, FMOE_ERR_INVALID_ARG, "invalid or destroyed context");
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = cudaMemcpyAsync(&ctx->hdr->epoch, &epoch, sizeof epoch, cudaMemcpyHostToDevice, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(ctx, e, "epoch write");
  ctx->tags_used = epoch;
  return FMOE_OK;
}

fmoe_status fmoe_poll_status(fmoe_ctx* ctx, void* stream, uint32_t* device_status) {
  if (!alive(ctx)) return fail(nullptr, FMOE_ERR_INVALID_ARG, "invalid or destroyed context");
  cudaStream_t st = (cudaStream_t)stream;
  WsHeader h;
  cudaError_t e = cudaMemcpyAsync(&h, ctx->hdr, sizeof h, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(ctx, e, "status read");
  if (device_status) *device_status = h.status;
  if (h.status != 0) {
    // only the status word: the epoch must keep increasing so that values
    // tagged by earlier launches are never mistaken for new ones
    e = cudaMemsetAsync(&ctx->hdr->status, 0, sizeof(uint32_t), st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(ctx, e, "status reset");
    return fail(ctx, FMOE_ERR_TIMEOUT, "device-side wait timed out (status 0x%x)", h.status);
  }
  return FMOE_OK;
}

}  // extern "C"
