// Packed-code operands of the tcgen05 GEMMs on Lloyd-Max codes: the layout of
// a row's codes in a code stage (as the TMA producer lands them), reading one
// row's codes back, byte-permute helpers, and the host calls that build the
// tensor maps and the weight workspace pool.  Used by the fp16-operand
// qlinear kernel; the W8A16 and 8-bit-operand GEMMs take the byte permute,
// the tensor-map encoder and the workspace pool.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace rbq {
namespace qfast {

// Code-stage geometry of the activation operand.
struct CodeGeo {
  uint32_t rows;         // 128
  uint32_t bits;
  uint32_t offset;       // byte offset of this operand inside a code stage
  uint32_t bytes;        // bytes of this operand landing per code stage (2 K slices)
  uint32_t slice_bytes;  // per-slice sub-buffer stride (even widths), else 0
  uint32_t swz;          // 0 none, 1 = 32B swizzle (4-bit), 2 = 64B swizzle (8-bit)
};

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// Codes 8c .. 8c+7 of a row's LSB-first bitstream of B-bit codes (B = 2, 3),
// one per nibble.
template <int B>
__device__ __forceinline__ uint32_t spread8(const uint32_t* src, int c) {
  if constexpr (B == 2) {
    uint32_t x = (src[c >> 1] >> (16 * (c & 1))) & 0xFFFFu;
    x = (x | (x << 8)) & 0x00FF00FFu;
    x = (x | (x << 4)) & 0x0F0F0F0Fu;
    return (x | (x << 2)) & 0x33333333u;
  } else {
    const int bit = 24 * c, wi = bit >> 5, sh = bit & 31;
    uint32_t u = src[wi] >> sh;
    if (sh > 8) u |= src[wi + 1] << (32 - sh);
    uint32_t x = 0u;
#pragma unroll
    for (int k = 0; k < 8; ++k) x |= ((u >> (3 * k)) & 7u) << (4 * k);
    return x;
  }
}

template <int BITS>
constexpr int slice_words() { return 2 * BITS; }

// Row r's codes of K slice h (0/1) of a code stage -> 2*BITS words.
template <int BITS>
__device__ __forceinline__ void read_slice(const uint8_t* part, const CodeGeo& g, int r, int h,
                                           uint32_t (&dst)[slice_words<BITS>()]) {
  if constexpr ((BITS & 1) == 0) {
    // even width: sub-buffer per slice, rows of 8*BITS bytes, maybe swizzled
    const uint8_t* row = part + h * g.slice_bytes + r * (8 * BITS);
#pragma unroll
    for (int c = 0; c < BITS / 2; ++c) {
      uint32_t pc = c;
      if constexpr (BITS == 4) pc ^= (r >> 2) & 1;   // 32B swizzle
      if constexpr (BITS == 8) pc ^= (r >> 1) & 3;   // 64B swizzle
      const uint4 v = *reinterpret_cast<const uint4*>(row + 16 * pc);
      dst[4 * c] = v.x;
      dst[4 * c + 1] = v.y;
      dst[4 * c + 2] = v.z;
      dst[4 * c + 3] = v.w;
    }
  } else {
    // odd width: one box of two slices, rows of 16*BITS bytes
    const uint2* row = reinterpret_cast<const uint2*>(part + r * (16 * BITS) + h * (8 * BITS));
#pragma unroll
    for (int i = 0; i < BITS; ++i) {
      const uint2 v = row[i];
      dst[2 * i] = v.x;
      dst[2 * i + 1] = v.y;
    }
  }
}

// Host side (rbq_qlinear_fast.cu).
PFN_cuTensorMapEncodeTiled_v12000 encode_fn();
// Geometry of one operand's share of a code stage (two 64-code K slices of
// `rows` rows), starting at `offset`.
CodeGeo make_geo(uint32_t rows, uint32_t bits, uint32_t offset);
// Bytes a code stage reserves for that operand (1024-aligned).
uint32_t geo_span(const CodeGeo& g);
// Tensor map over a [rows, K*bits/8] code matrix with the boxes of `g`.
int encode_codes_map(CUtensorMap* map, const uint8_t* base, int rows, int bits, int K, const CodeGeo& g);
// A memory pool per device for stream-ordered weight workspaces.
cudaMemPool_t workspace_pool(int dev);

}  // namespace qfast
}  // namespace rbq
