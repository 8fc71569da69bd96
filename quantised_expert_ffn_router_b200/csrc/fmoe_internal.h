// fmoe_internal.h -- packed expert layout and kernel launch plans shared by the
// host API (fmoe_api.cu) and the kernels (fmoe_repack.cu, fmoe_decode.cu).
//
// Packed tile layout (build-side design; the Flash-MoE pages only say experts
// are ~6.75 MB blobs dequantised by an FMA kernel, page 4 "The Architecture").
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
constexpr int kThreads = 512;            // 16 warps per block
constexpr int kWarps = kThreads / 32;
constexpr int kMaxNStage = 4;

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

// Device workspace header (counters and status), followed by logits and
// activations.  Zero between launches: the last block of every launch resets it.
struct WsHeader {
  uint32_t router_arrive;
  uint32_t exit_count;
  uint32_t status;
  uint32_t pad0;
  uint32_t h_arrive[16];
};
static_assert(sizeof(WsHeader) <= 256, "header");

// device status bits
constexpr uint32_t kStatusTimeoutRouter = 0x1;
constexpr uint32_t kStatusTimeoutH = 0x2;
constexpr uint32_t kStatusTimeoutTma = 0x4;

enum DecodeMode : int { kModeLayer = 0, kModeExpert = 1, kModeRoute = 2 };

// Everything the fused single-token kernel needs, computed on the host.
struct DecodePlan {
  // shapes
  int H, E, K, I, bits, mode;
  int n_slots;             // K+1 (layer), 1 (expert), 0 (route)
  int grid;                // blocks (one per SM)
  int tb, cb;              // tile bytes, code bytes per tile
  int gu_tiles;            // H/64 tiles per gate/up row block
  int gu_unit_bytes;       // gu_tiles * tb
  int n_kr_gu;             // K-ranges (warps) per gate/up unit
  int teams_gu;            // gate/up units processed concurrently (= units per stage)
  int units_per_slot;      // I/8
  int total_units;         // n_slots * units_per_slot
  int dn_tiles;            // I/64 tiles per down row block
  int dn_job_bytes;        // dn_tiles * tb
  int n_kr_dn;             // K-ranges per down job
  int teams_dn;            // down jobs processed concurrently
  int n_rb;                // H/16 output row blocks
  int rb_per_cta;          // max output row blocks per block
  int router_rows;         // max router rows per block
  int router_chunks;       // 256-column chunks per router row
  int nstage;
  // shared-memory layout (byte offsets)
  uint32_t off_ring, stage_bytes;
  uint32_t off_down;       // [slot][rb_local] down jobs
  uint32_t off_router;     // router rows (aliases the routed part of off_down)
  uint32_t off_zfrag, off_zinfo;
  uint32_t off_afrag, off_ainfo, afrag_bytes, ainfo_bytes;  // two buffers
  uint32_t off_z;          // bf16 z [H] (router input; reused for logits)
  uint32_t off_gupart;     // [2][16 warps][16] fp32
  uint32_t off_dnpart;     // [16 warps][16] fp32
  uint32_t off_y;          // [rb_per_cta][n_slots][16] fp32
  uint32_t off_rpart;      // [router_rows][16 warps] fp32
  uint32_t off_misc;       // slot expert ids / weights
  uint32_t off_bar;        // mbarriers
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
  float* ws_logits;        // [E]
  float* ws_a;             // [kMaxSlots][I]
  uint32_t flags;
  uint64_t timeout_ns;
  int pdl;                 // launched with programmatic stream serialisation
};

// host launchers (return cudaError_t as int)
int launch_repack(const uint8_t* src, uint8_t* dst, int n_experts, int H, int I, int bits, int to_packed,
                  void* stream);
int launch_decode(const DecodePlan& plan, void* stream, bool cooperative, bool pdl);
int decode_max_smem_optin(int device);
int decode_occupancy(int bits, int smem_bytes, int* blocks_per_sm);
int zero_workspace(void* ws, size_t bytes, void* stream);

}  // namespace fmoe
