// fmoe_internal.h -- packed expert layout and kernel launch plans shared by the
// host API (fmoe_api.cu) and the kernels (fmoe_repack.cu, fmoe_decode.cu).
//
// Packed tile layout (build-side design; the Flash-MoE pages only size an
// expert at about 6.75 MB and dequantise it with fused multiply-adds: "Flash-MoE:
// Running a 400 Billion Parameter Model on a MacBook", section "The Architecture").
// A tile is 16 weight rows x 64 input columns, i.e. one quantisation group per
// row, laid out for one warp's mma.sync.m16n8k16 A fragments:
//   codes: 32 lanes x (16*64*bits/8/32) bytes, lane l = 4*g + t owns rows g and
//          g+8, columns 2t, 2t+1, 2t+8, 2t+9 of every 16-column slice;
//   s/b  : 8 entries of 8 bytes, entry g = {scale[g], bias[g], scale[g+8],
//          bias[g+8]} as bf16.
// 4-bit (576 B tile): lane word j covers slice j; nibble n of the word holds
//   row g + 8*((n>>1)&1), column 16j + 2t + (n>>2) + 8*(n&1).
// 2-bit (320 B tile): lane word j covers slices 2j and 2j+1; 2-bit field f
//   holds row g + 8*((f&7)>>2), column 16*(2j + ((f&3)>>1)) + 2t + (f>>3) +
//   8*(f&1).
// With these positions one lop3 per register places two codes into the
// mantissas of an fp16 pair (1024 + code * 4^k), and one sub.f16x2 removes the
// 1024, so the codes enter the tensor-core fragment exactly.
//
// Expert = gate/up region then down region, same byte size as the canonical
// blob:
//   gate/up: I/8 row blocks x H/64 tiles; tile rows 0..7 are gate rows
//            8rb..8rb+7 and rows 8..15 the up rows with the same indices;
//   down   : H/16 row blocks x I/64 tiles; tile rows are down rows 16rb..16rb+15.
#pragma once

#include <cstdint>

#include "../../include/fmoe.h"

namespace fmoe {

constexpr int kGroup = 64;
constexpr int kMaxTopK = 8;
constexpr int kMaxSlots = kMaxTopK + 1;  // K routed + 1 shared
constexpr int kConsumerWarps = 15;       // warps that compute (16 warps in all: 4 per SM sub-partition, 128 registers each)
constexpr int kMaxHidden = 4096;         // largest hidden size a context accepts
constexpr int kThreads = (kConsumerWarps + 1) * 32;  // + one producer warp
// Tiles per gate/up or down task, one bulk copy each: 24 x 576 B = 13.5 KB at
// 4-bit, 32 x 320 B = 10 KB at 2-bit.  Larger copies stream HBM faster; fewer
// tasks per unit leave consumer warps idle (32 tiles at 4-bit measured slower).
constexpr __host__ __device__ int chunk_tiles(int bits) { return bits == 4 ? 24 : 32; }
constexpr int kMaxTasks = 96;            // task-list capacity per block (multiple of 32)
constexpr int kStaticRouteLogits = 32768; // fp32 logits in the fixed scratch of fmoe_route_static (128 KB)
constexpr int kStaticRouteMaxTokens = 4096;  // tokens per fmoe_route_static call
constexpr int kMaxDevices = 64;          // devices fmoe_route_static caches a scratch address for
// Ring stages kept when down jobs get stages of their own (~180 KB of ring at
// 4-bit; 100 KB at 2-bit, where the down jobs' own stages pay more).
constexpr __host__ __device__ int min_ring_stages(int bits) { return bits == 4 ? 13 : 10; }
constexpr int kFetchGroups = 8;          // activation groups a warp fetches per round trip
constexpr int kTracePoints = 32;         // FMOE_TRACE builds: %globaltimer stamps per block and layer
constexpr int kTraceLayers = 4;          // ... for the first layers of a launch

inline __host__ __device__ int tile_code_bytes(int bits) { return 16 * kGroup * bits / 8; }
inline __host__ __device__ int tile_bytes(int bits) { return tile_code_bytes(bits) + 64; }

inline __host__ __device__ int64_t canonical_matrix_bytes(int64_t R, int64_t C, int bits) {
  return R * C * bits / 8 + 4 * R * (C / kGroup);
}
inline __host__ __device__ int64_t expert_bytes(int H, int I, int bits) {
  return 2 * canonical_matrix_bytes(I, H, bits) + canonical_matrix_bytes(H, I, bits);
}
inline __host__ __device__ int64_t packed_gu_bytes(int H, int I, int bits) {
  return (int64_t)(I / 8) * (H / kGroup) * tile_bytes(bits);
}

// Device workspace header, followed by the tagged logits, activations and
// layer outputs.  Cross-block results are published as 64-bit words
// {float bits, tag} with tag = epoch + 1 (+ layer in a multi-layer launch), so
// a reader knows a value is from the current launch without any counter, fence
// or atomic on the critical path.  The last block to finish a launch advances
// the epoch by the launch's layer count (exit_count protocol).  The host never
// lets a tag pass 2^32 - 1: before a launch whose tags would, it clears the
// tagged words and the epoch, so tag 0 -- the value of every cleared word --
// is never current.
struct WsHeader {
  uint32_t epoch;           // launches completed on this workspace
  uint32_t exit_count;      // blocks finished in the current launch
  uint32_t status;          // kStatus* bits, cleared by fmoe_poll_status
  uint32_t router_cnt;      // router rows published in this launch (hint for pollers)
  uint32_t h_cnt[16];       // gate/up units published per slot in this launch (hint; cumulative over
                            // the layers of a multi-layer launch)
};
static_assert(sizeof(WsHeader) <= 256, "header");

// device status bits
constexpr uint32_t kStatusTimeoutRouter = 0x1;
constexpr uint32_t kStatusTimeoutH = 0x2;
constexpr uint32_t kStatusTimeoutTma = 0x4;
constexpr uint32_t kStatusTimeoutTc = 0x8;   // a bounded wait of the grouped tensor-core GEMM ran out
constexpr uint32_t kStatusTimeoutLayer = 0x10;  // a multi-layer launch waited too long for the previous layer


enum DecodeMode : int { kModeLayer = 0, kModeExpert = 1, kModeRoute = 2 };

// Task descriptors of a block's ordered work list (one 32-bit word each).
enum TaskType : uint32_t { kTaskRouter = 0, kTaskGateUp = 1, kTaskDown = 2 };
inline __host__ __device__ uint32_t make_task(uint32_t type, uint32_t idx, uint32_t slot, uint32_t chunk) {
  return type | (idx << 2) | (slot << 18) | (chunk << 22);
}
inline __host__ __device__ uint32_t task_type(uint32_t t) { return t & 3u; }
inline __host__ __device__ uint32_t task_idx(uint32_t t) { return (t >> 2) & 0xFFFFu; }
inline __host__ __device__ uint32_t task_slot(uint32_t t) { return (t >> 18) & 0xFu; }
inline __host__ __device__ uint32_t task_chunk(uint32_t t) { return (t >> 22) & 0x3FFu; }

// Shared-memory bookkeeping of the fused kernel.
struct Misc {
  int slot_e[16];
  float slot_w[16];
  int abort;
  uint32_t tag;         // epoch + 1 of this launch
  int n_tasks;          // length of this block's task list
  int rdone;            // router rows of this block published in the current layer
  int pad[12];
  // expert cache (contexts with host-resident experts): per slot the blob base
  // the copies read, the cache slot a miss fills (null on a hit) and the slot
  // index / hit flag the last block out records; the CLOCK hand advance
  const uint8_t* slot_src[16];
  uint8_t* slot_dst[16];
  int cslot[16];
  int chit[16];
  int cwalk;
  int chand;
  int cpad[14];
  int aflag[32];        // per (slot, half) activation fragments: 0 none, 1 building, 2 ready
  int rcnt[16];         // parts finished per router row of this block
  float rpart[16][4];   // partial logits per router row and part
  int unit_cnt[32];     // K-chunks finished per gate/up unit of this block
  int dn_cnt[32];       // K-chunks finished per (row block, slot) down job
  int last_task[64];    // last task issued into each ring stage (-1: none)
  float red[16];        // RMSNorm scratch
};

// Host-resident routed experts with an HBM cache (fmoe_create_cached), as
// the fused kernel sees them for one layer.  Slots are shared by all layers
// (key = layer * E + expert) and replaced by CLOCK (second chance): the hand
// sweeps the slots, a slot whose reference bit is set loses the bit and is
// skipped, the first unreferenced one is the victim; a hit or a fill sets the
// bit.  Every block derives the same decision from the state the launch
// starts with; the last block out applies it.
constexpr int kCacheWindow = 32;  // slots from the hand a launch may sweep
struct CacheArgs {
  int on;
  int n_slots;
  int key0;                  // layer * E
  const uint8_t* host;       // the layer's packed routed blobs, device-mapped page-locked host memory
  const uint8_t* shared;     // the layer's packed shared expert in HBM
  uint8_t* slots;            // [n_slots] blobs in HBM
  int32_t* slot_of;          // [n_layers * E]: cache slot of a key, or -1
  int32_t* owner;            // [n_slots]: key held, or -1
  uint8_t* ref;              // [n_slots]: reference bits
  uint32_t* hand;            // CLOCK hand
  unsigned long long* stats; // [2]: hits, misses
};

// Per-layer weights of a multi-layer launch (device array, one entry per layer).
struct LayerDev {
  const uint8_t* experts;
  const uint16_t* router_w;
  const float* router_bias;
  const uint16_t* norm_w;
};

// Everything the fused single-token kernel needs, computed on the host.
struct DecodePlan {
  // shapes
  int H, E, K, I, bits, mode;
  int n_slots;             // K+1 (layer), 1 (expert), 0 (route)
  int grid;                // blocks (one per SM)
  int tb, cb;              // tile bytes, code bytes per tile
  int gu_tiles;            // H/64 tiles per gate/up row block (unit)
  int gu_chunks;           // tasks per unit (chunk_tiles(bits) tiles each, last may be shorter)
  int dn_tiles;            // I/64 tiles per down row block
  int dn_chunks;           // tasks per down job
  int units_per_slot;      // I/8
  int total_units;         // n_slots * units_per_slot
  int units_per_cta;       // max units per block
  int n_rb;                // H/16 output row blocks
  int rb_per_cta;          // max output row blocks per block
  int router_rows;         // max router rows per block
  int router_parts;        // column parts per router row (one task each)
  int router_part_cols;    // columns per part (multiple of 64; the last part may be shorter)
  int nstage;              // ring stages for router and gate/up tasks (a multiple of n_issuers)
  int n_down_max;          // stages after the ring, one per down job (filled once per launch)
  int n_issuers;           // producer lanes issuing copies; lane l owns stages l, l+n_issuers, ...
  uint32_t stage_bytes;
  // shared-memory layout (byte offsets)
  uint32_t off_ring;
  uint32_t off_z;          // bf16 z [H]
  uint32_t off_lg;         // fp32 logits [E] (routing)
  uint32_t off_zfrag, off_zinfo;
  uint32_t off_afrag, off_ainfo, afrag_bytes, ainfo_bytes;  // per slot
  uint32_t off_gupart;     // [units_per_cta][gu_chunks][16] fp32
  uint32_t off_dnpart;     // [rb_per_cta][n_slots][dn_chunks][16] fp32
  uint32_t off_y;          // [rb_per_cta][n_slots][16] fp32
  uint32_t off_tasks;      // [kMaxTasks] uint32, this block's task list
  uint32_t off_misc;       // slot expert ids / weights / counters / flags
  uint32_t off_bar;        // mbarriers: full[nstage], empty[nstage]
  uint32_t smem_bytes;
  // data
  const uint8_t* experts;  // packed experts of this layer
  int64_t blob_bytes;
  const uint16_t* router_w;
  const float* router_bias;
  const uint16_t* norm_w;
  float eps;
  const uint16_t* h_in;    // [H]
  uint16_t* h_out;         // [H] bf16 (layer mode)
  float* y_out;            // [H] fp32 (expert mode)
  int32_t* idx_out;        // [K] or null
  float* w_out;            // [K] or null
  int expert_id;           // expert mode: 0..E (E = shared)
  WsHeader* ws;
  uint64_t* ws_logits;     // [E] tagged
  uint64_t* ws_a;          // [kMaxSlots][I] tagged
  const uint32_t* tasks;   // [grid][kMaxTasks] ordered task lists (host-built)
  const int32_t* n_tasks;  // [grid]
  uint32_t flags;
  uint64_t timeout_ns;
  int pdl;                 // launched with programmatic stream serialisation
  // multi-layer launch (n_layers > 0): layers 0..n_layers-1 take their weights
  // from layer_dev[l]; layer 0 reads h_in, the last writes h_out, and each
  // layer in between publishes its output as tagged words in ws_h.
  // n_layers == 0: one layer from the fields above.
  int n_layers;
  const LayerDev* layer_dev;
  uint64_t* ws_h;          // [H] tagged
  unsigned long long* trace;  // FMOE_TRACE builds: [grid][kTraceLayers][kTracePoints] stamps, or null
  CacheArgs cache;         // host-resident experts (single-layer launches, layer mode)
};

// Ring position of task i: issued by producer lane i % n_issuers into that
// lane's (i / n_issuers) % (nstage / n_issuers)-th stage, as fill number
// (i / n_issuers) / (nstage / n_issuers) of that stage.
inline __host__ __device__ void task_stage(int nstage, int n_issuers, int i, int& stage, int& fill) {
  const int L = nstage / n_issuers, j = i / n_issuers;
  stage = (j % L) * n_issuers + i % n_issuers;
  fill = j / L;
}

// The same positions, followed one issue at a time by the producer lane that
// owns them: its next ring task goes to stage slot * n_issuers + lane as fill
// `fill`; ring_advance moves to the lane's next stage (nstage / n_issuers of
// them, used round-robin).
inline __host__ __device__ void ring_advance(int per_lane, int& slot, int& fill) {
  if (++slot == per_lane) {
    slot = 0;
    ++fill;
  }
}

// Stage and fill of task i of layer l (0 for a single-layer launch) of a block
// whose last n_down tasks are its down jobs: those sit in dedicated stages after
// the ring (one fill per layer), the other tasks cycle through the ring.  Layer
// by layer, producer lane i % n_issuers issues the same ring_end-task list, so
// its k-th issue of the launch is issue i / n_issuers of layer l plus the
// ceil((ring_end - lane) / n_issuers) issues it made in each earlier layer: a
// stage is always refilled by the same lane, in order.
inline __host__ __device__ void task_stage_of(int nstage, int n_issuers, int n_tasks, int n_down, int i, int& stage,
                                              int& fill, int layer = 0) {
  const int ring_end = n_tasks - n_down;
  if (i >= ring_end) {
    stage = nstage + (i - ring_end);
    fill = layer;
  } else {
    const int lane = i % n_issuers, per_layer = (ring_end - lane + n_issuers - 1) / n_issuers;
    task_stage(nstage, n_issuers, (layer * per_layer + i / n_issuers) * n_issuers + lane, stage, fill);
  }
}

// ---------------------------------------------------------------- batched path
// T tokens at once (fmoe_batched.cu): RMSNorm, router GEMM, top-K, a
// per-expert permutation of the T*(K+1) (token, slot) pairs into segments, a
// grouped gate/up GEMM on tcgen05 (fmoe_grouped_tc.cu: 128 rows x up to 64
// positions per work item, weights dequantised to fp16 in tensor memory,
// silu(g)*u in the epilogue), a grouped down GEMM, and a fixed-order combine.
// Positions 0..T*K-1 hold the routed pairs grouped by expert; positions T*K..
// hold the shared expert.
constexpr int kGemmRows = 128;       // rows per work item (8 packed bands of 16)
constexpr int kGemmTokens = 64;      // tokens (positions) per work item
constexpr int kGroupedMinTokens = 8; // fmoe_layer_forward uses the batched path from this T on
constexpr int kGemvTokens = 8;       // segments up to this many positions take the mma.sync GEMV, not tcgen05
constexpr int kBatchMaxExperts = 1023;  // batched permute: one thread per expert plus the shared one
constexpr int kBatchMaxTokens = 255 * kGemmTokens;  // token blocks per segment fit 8 bits of a work item

// Opaque copy of a TMA tensor map (CUtensorMap: 128 bytes, 64-byte aligned).
struct TmaDesc {
  alignas(64) unsigned char bytes[128];
};

struct BatchWs {              // device buffers, sized for max_tokens at create
  uint16_t* z;                // bf16 [T][H]   (normalised input)
  uint16_t* zp;               // fp16 [T*(K+1)][H] GEMM input of each position (scaled, k-permuted)
  float* zsc;                 // [T*(K+1)] 2^sh that undoes the scaling of zp
  float* zsum;                // [H/128][T*(K+1)][4] sums of zp's 64-column groups (fp32)
  float* logits;              // [T][E]
  float* logit_part;          // [4][T][E] partial router logits (K split)
  int32_t* idx;               // [T][K]
  float* w;                   // [T][K]
  int32_t* seg;               // [4][E+1]: expert, start, count, items-prefix per segment; [4*(E+1)] = n_seg
  int32_t* cursor;            // [E+1] scatter cursors
  int32_t* pos_tok;           // [T*(K+1)] token of each position
  int32_t* pos_of;            // [T][K+1] position of (token, slot); slot K = shared
  uint32_t* items_gu;         // work items (seg, row block, token block)
  uint32_t* items_dn;
  int32_t* n_items;           // [4]: tcgen05 gate/up, down items; GEMV gate/up, down items
  int32_t* small_seg;         // [E+1]: segments of <= kGemvTokens positions, in segment order
  uint32_t* gv_frag;          // [small][H/64][8 positions][32] fp16 pairs: mma.sync B fragments (GEMV)
  float2* gv_info;            // [small][H/64][8]: (2^-shift, group sum) per position and group
  int max_small;              // segments the GEMV buffers hold
  float* a;                   // [T*(K+1)][I] activations
  uint16_t* ap;               // fp16 [T*(K+1)][I] down-GEMM input (scaled, k-permuted)
  float* asc;                 // [T*(K+1)]
  float* asum;                // [I/128][T*(K+1)][4] sums of ap's 64-column groups
  float* y;                   // [T*(K+1)][H] expert outputs
  int max_items_gu, max_items_dn;
  int pcap;                   // positions the buffers hold: max_tokens * (K + 1)
  TmaDesc zmap[4], amap[4];   // zp / ap boxes of 16, 32, 48, 64 rows x 2 x 64 columns, 128-byte swizzle
  TmaDesc zsmap[4], asmap[4]; // zsum / asum boxes of 16, 32, 48, 64 rows x 4 floats
};

struct BatchArgs {
  int H, E, K, I, bits, T;
  const uint8_t* experts;     // packed experts of the layer (E routed + shared)
  int64_t blob_bytes;
  const uint16_t* router_w;
  const float* router_bias;
  const uint16_t* norm_w;
  float eps;
  const uint16_t* h_in;       // [T][H]
  uint16_t* h_out;            // [T][H]
  int32_t* idx_out;           // [T][K] or null
  float* w_out;               // [T][K] or null
  int single_expert;          // >= 0: expert mode on this expert (0..E, E = shared), output y_out
  float* y_out;               // [T][H] fp32 (expert mode)
  const TmaDesc* wmap_gu;     // tensor maps of the layer's packed gate/up and down matrices
  const TmaDesc* wmap_dn;
  uint32_t* status;           // device status word (kStatus* bits)
  void* gemm_events[4];       // cudaEvent_t recorded around the two grouped GEMMs, or null
};

// Bytes of the batched workspace for T tokens; carves it out of `base` and
// encodes its tensor maps (returns a cudaError_t value).
size_t batch_ws_bytes(int H, int E, int K, int I, int T);
int batch_ws_carve(uint8_t* base, int H, int E, int K, int I, int T, BatchWs& ws);

// Grouped tensor-core GEMM (fmoe_grouped_tc.cu).
struct TcArgs {
  const int32_t* seg;         // segment table ([4][S] + n_seg)
  int S;                      // E + 1
  const uint32_t* items;      // work items (seg << 16 | row block << 8 | token block)
  const int32_t* n_items;
  int k_chunks;               // ceil(K / 128)
  int rows;                   // matrix rows (2I gate/up, H down)
  int ldo;                    // output row length (I: a, H: y)
  const float* bscale;        // per position: 2^sh undoing the input scaling
  float* out;                 // gate/up: a [pos][I]; down: y [pos][H]
  uint32_t* status;
};
// Tensor map over the packed matrix at `matrix0` of each of n_blobs experts
// (blob_bytes apart): uint64 elements, 3-D (band bytes/8, rows/16, n_blobs),
// box = 2 tiles x 8 bands.
int tc_encode_weight_map(const uint8_t* matrix0, int64_t blob_bytes, int n_blobs, int rows, int cols, int bits,
                         TmaDesc* out);
// Four tensor maps over an fp16 [rows][cols] matrix seen as (64 columns, rows,
// cols/64 blocks): boxes of 16, 32, 48, 64 rows x 2 blocks, 128-byte swizzle.
int tc_encode_token_maps(const uint16_t* base, int cols, int rows, TmaDesc* out);
// Four tensor maps over fp32 group sums laid out [chunks][rows][4] (per
// 128-column chunk and row: the sums of its two 64-column groups, two unused):
// boxes of 16, 32, 48, 64 rows x 4 floats of one chunk.
int tc_encode_sum_maps(const float* base, int chunks, int rows, TmaDesc* out);
int launch_tc_gemm(int bits, bool gate_up, const TmaDesc& wmap, const TmaDesc* xmaps, const TmaDesc* smaps,
                   const TcArgs& a, int n_sm, void* stream);
int launch_batched(const BatchArgs& a, const BatchWs& ws, int n_sm, void* stream);

// Top-K and renormalised weights of T rows of fp32 logits (one warp per row).
int launch_topk_rows(const float* logits, int T, int E, int K, int32_t* idx_out, float* w_out, void* stream);

// Host-side construction of a block's ordered task list; returns its length.
int build_task_list(const DecodePlan& P, int cta, uint32_t* out);

// host launchers (return cudaError_t as int)
int launch_repack(const uint8_t* src, uint8_t* dst, int n_experts, int H, int I, int bits, int to_packed,
                  void* stream);
int launch_decode(const DecodePlan& plan, void* stream, bool cooperative, bool pdl);
// Router step with its scratch in a fixed device array (fmoe_static.cu); returns
// a cudaError_t value.
int route_static_prepare();  // 0 or a cudaError_t
bool route_static_ready();
int launch_route_static(const uint16_t* wr, const float* bias, const uint16_t* norm_w, float eps,
                        const uint16_t* x, int T, int H, int E, int K, int32_t* idx_out, float* w_out, void* stream);
// 4-bit -> 2-bit requantisation of n canonical blobs (fmoe_requant.cu).
int launch_requant(const uint8_t* src, uint8_t* dst, int n_blobs, int H, int I, int n_sm, void* stream);
int decode_max_smem_optin(int device);
int decode_occupancy(int bits, bool multi, int smem_bytes, int* blocks_per_sm);
int zero_workspace(void* ws, size_t bytes, void* stream);

}  // namespace fmoe
