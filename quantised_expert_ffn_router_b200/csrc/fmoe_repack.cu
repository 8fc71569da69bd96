// fmoe_repack.cu -- canonical expert blobs <-> packed tile layout.
//
// The canonical blob is the row-major code/scale/bias format fmoe.h documents;
// the packed layout (fmoe_internal.h) groups each 16-row x 64-column tile's
// codes so a warp loads them with one 16-byte (4-bit) or 8-byte (2-bit) shared
// load per lane and unpacks them straight into mma.sync fragments, with the
// tile's scales and biases next to its codes.  This is the B200 counterpart of
// the pages' offline expert packing ("Flash-MoE Inference Engine", section
// "Weight Preparation", step 2); it runs once, on device, at fmoe_create.
#include <cuda_runtime.h>

#include "fmoe_internal.h"

namespace fmoe {
namespace {

struct Geo {
  int H, I, bits;
  int64_t blob;       // bytes per expert
  int64_t gate_bytes; // canonical bytes of one [I][H] matrix
  int64_t gu_packed;  // packed gate/up region bytes
  int tb, cb;
};

__device__ __forceinline__ void mat_shape(const Geo& g, int m, int& R, int& C) {
  if (m < 2) { R = g.I; C = g.H; } else { R = g.H; C = g.I; }
}

__device__ __forceinline__ int64_t canon_mat_base(const Geo& g, int m) { return (int64_t)m * g.gate_bytes; }

// Byte offset of the 32-bit word holding code (m, r, c) in the packed expert,
// and its bit shift.
__device__ __forceinline__ void packed_code_pos(const Geo& g, int m, int r, int c, int64_t& off, int& shift) {
  int rho, rb;
  int64_t tile;
  int kt = c / kGroup, cc = c % kGroup;
  if (m < 2) {
    rb = r / 8;
    rho = (r % 8) + 8 * m;
    tile = (int64_t)rb * (g.H / kGroup) + kt;
    off = tile * g.tb;
  } else {
    rb = r / 16;
    rho = r % 16;
    tile = (int64_t)rb * (g.I / kGroup) + kt;
    off = g.gu_packed + tile * g.tb;
  }
  int grow = rho % 8, hi = rho / 8;
  if (g.bits == 4) {
    int j = cc / 16, k = cc % 16, rem = k % 8;
    int t = rem / 2;
    int n = (rem % 2) * 4 + hi * 2 + (k / 8);
    int lane = 4 * grow + t;
    off += lane * 16 + j * 4;
    shift = 4 * n;
  } else {
    int j = cc / 32, ss = (cc % 32) / 16, k = cc % 16, rem = k % 8;
    int t = rem / 2;
    int f = (rem % 2) * 8 + hi * 4 + ss * 2 + (k / 8);
    int lane = 4 * grow + t;
    off += lane * 8 + j * 4;
    shift = 2 * f;
  }
}

// Byte offset of the bf16 scale (is_bias = 0) or bias of (m, r, group kt).
__device__ __forceinline__ int64_t packed_sb_pos(const Geo& g, int m, int r, int kt, int is_bias) {
  int64_t off;
  int rho;
  if (m < 2) {
    rho = (r % 8) + 8 * m;
    off = ((int64_t)(r / 8) * (g.H / kGroup) + kt) * g.tb;
  } else {
    rho = r % 16;
    off = g.gu_packed + ((int64_t)(r / 16) * (g.I / kGroup) + kt) * g.tb;
  }
  return off + g.cb + 8 * (rho % 8) + 4 * (rho / 8) + 2 * is_bias;
}

__device__ __forceinline__ uint32_t load_u32(const uint8_t* p) { return *reinterpret_cast<const uint32_t*>(p); }
__device__ __forceinline__ uint16_t load_u16(const uint8_t* p) { return *reinterpret_cast<const uint16_t*>(p); }

// Canonical code words: matrix m, row r, word w (32/bits codes each).
__device__ __forceinline__ bool canon_word_coords(const Geo& g, int64_t i, int& m, int& r, int& wi) {
  for (m = 0; m < 3; ++m) {
    int R, C;
    mat_shape(g, m, R, C);
    int64_t words = (int64_t)R * C * g.bits / 32;
    if (i < words) {
      int per_row = C * g.bits / 32;
      r = (int)(i / per_row);
      wi = (int)(i % per_row);
      return true;
    }
    i -= words;
  }
  return false;
}

// Packed -> canonical, one thread per canonical 32-bit code word, then per scale.
__global__ void unpack_kernel(const uint8_t* __restrict__ src, uint8_t* __restrict__ dst, int n_experts, Geo g) {
  int64_t code_words = 0, groups = 0;
  for (int m = 0; m < 3; ++m) {
    int R = m < 2 ? g.I : g.H, C = m < 2 ? g.H : g.I;
    code_words += (int64_t)R * C * g.bits / 32;
    groups += (int64_t)R * (C / kGroup);
  }
  int64_t per_expert = code_words + groups;
  int64_t total = per_expert * n_experts;
  int per = 32 / g.bits;
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (int64_t)gridDim.x * blockDim.x) {
    int e = (int)(idx / per_expert);
    int64_t i = idx % per_expert;
    const uint8_t* s = src + e * g.blob;
    uint8_t* d = dst + e * g.blob;
    if (i < code_words) {
      int m, r, wi;
      canon_word_coords(g, i, m, r, wi);
      int R, C;
      mat_shape(g, m, R, C);
      uint32_t word = 0;
      for (int f = 0; f < per; ++f) {
        int c = wi * per + f;
        int64_t off;
        int sh;
        packed_code_pos(g, m, r, c, off, sh);
        uint32_t q = (load_u32(s + off) >> sh) & ((1u << g.bits) - 1u);
        word |= q << (g.bits * f);
      }
      int64_t dst_off = canon_mat_base(g, m) + ((int64_t)r * (C * g.bits / 32) + wi) * 4;
      *reinterpret_cast<uint32_t*>(d + dst_off) = word;
    } else {
      int64_t j = i - code_words;
      for (int m = 0; m < 3; ++m) {
        int R, C;
        mat_shape(g, m, R, C);
        int64_t n = (int64_t)R * (C / kGroup);
        if (j < n) {
          int r = (int)(j / (C / kGroup)), kt = (int)(j % (C / kGroup));
          int64_t sbase = canon_mat_base(g, m) + (int64_t)R * C * g.bits / 8;
          *reinterpret_cast<uint16_t*>(d + sbase + 2 * j) = load_u16(s + packed_sb_pos(g, m, r, kt, 0));
          *reinterpret_cast<uint16_t*>(d + sbase + 2 * n + 2 * j) = load_u16(s + packed_sb_pos(g, m, r, kt, 1));
          break;
        }
        j -= n;
      }
    }
  }
}

// Canonical -> packed, one thread per packed 32-bit word (codes or s/b words).
__global__ void pack_kernel(const uint8_t* __restrict__ src, uint8_t* __restrict__ dst, int n_experts, Geo g) {
  const int64_t words_per_expert = g.blob / 4;
  const int64_t total = words_per_expert * n_experts;
  const int tile_words = g.tb / 4, code_words = g.cb / 4;
  const int64_t gu_tiles = (int64_t)(g.I / 8) * (g.H / kGroup);
  const int per = 32 / g.bits;
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (int64_t)gridDim.x * blockDim.x) {
    int e = (int)(idx / words_per_expert);
    int64_t w = idx % words_per_expert;
    const uint8_t* s = src + e * g.blob;
    int64_t tile = w / tile_words;
    int tw = (int)(w % tile_words);
    // tile -> region, row block, k tile
    int m_lo, rows_per_block, rb, kt, C;
    if (tile < gu_tiles) {
      rb = (int)(tile / (g.H / kGroup));
      kt = (int)(tile % (g.H / kGroup));
      rows_per_block = 8;
      m_lo = 0;
      C = g.H;
    } else {
      int64_t t2 = tile - gu_tiles;
      rb = (int)(t2 / (g.I / kGroup));
      kt = (int)(t2 % (g.I / kGroup));
      rows_per_block = 16;
      m_lo = 2;
      C = g.I;
    }
    uint32_t out = 0;
    if (tw < code_words) {
      int lane, j;
      if (g.bits == 4) { lane = tw / 4; j = tw % 4; }
      else { lane = tw / 2; j = tw % 2; }
      int grow = lane / 4, t = lane % 4;
      for (int f = 0; f < per; ++f) {
        int rho, col;
        if (g.bits == 4) {
          rho = grow + 8 * ((f >> 1) & 1);
          col = 16 * j + 2 * t + (f >> 2) + 8 * (f & 1);
        } else {
          rho = grow + 8 * ((f & 7) >> 2);
          col = 16 * (2 * j + ((f & 3) >> 1)) + 2 * t + (f >> 3) + 8 * (f & 1);
        }
        int m, r;
        if (m_lo == 0) { m = rho / 8; r = rb * 8 + rho % 8; }
        else { m = 2; r = rb * rows_per_block + rho; }
        int c = kt * kGroup + col;
        int64_t coff = canon_mat_base(g, m) + ((int64_t)r * (C * g.bits / 32) + c / per) * 4;
        uint32_t q = (load_u32(s + coff) >> (g.bits * (c % per))) & ((1u << g.bits) - 1u);
        out |= q << (g.bits * f);
      }
    } else {
      // s/b word: entry grow = (tw - code_words) / 2, half = which pair
      int k = tw - code_words;
      int grow = k / 2, hi = k % 2;
      int rho = grow + 8 * hi;
      int m, r, R;
      if (m_lo == 0) { m = rho / 8; r = rb * 8 + rho % 8; R = g.I; }
      else { m = 2; r = rb * rows_per_block + rho; R = g.H; }
      int ng = C / kGroup;
      int64_t sbase = canon_mat_base(g, m) + (int64_t)R * C * g.bits / 8;
      uint32_t sc = load_u16(s + sbase + 2 * ((int64_t)r * ng + kt));
      uint32_t bi = load_u16(s + sbase + 2 * (int64_t)R * ng + 2 * ((int64_t)r * ng + kt));
      out = sc | (bi << 16);
    }
    *reinterpret_cast<uint32_t*>(dst + e * g.blob + w * 4) = out;
  }
}

}  // namespace

int launch_repack(const uint8_t* src, uint8_t* dst, int n_experts, int H, int I, int bits, int to_packed,
                  void* stream) {
  Geo g;
  g.H = H;
  g.I = I;
  g.bits = bits;
  g.blob = expert_bytes(H, I, bits);
  g.gate_bytes = canonical_matrix_bytes(I, H, bits);
  g.gu_packed = packed_gu_bytes(H, I, bits);
  g.tb = tile_bytes(bits);
  g.cb = tile_code_bytes(bits);
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaStream_t st = (cudaStream_t)stream;
  if (to_packed)
    pack_kernel<<<sms * 8, 256, 0, st>>>(src, dst, n_experts, g);
  else
    unpack_kernel<<<sms * 8, 256, 0, st>>>(src, dst, n_experts, g);
  return (int)cudaGetLastError();
}

}  // namespace fmoe
