// Internal declarations shared by the library's translation units.
// Nothing here is part of the public ABI (include/rbq.h is).
#pragma once

#include <cstdint>
#include <cstddef>
#include <vector>

#include <cuda_runtime.h>

#include "rbq.h"

namespace rbq {

constexpr int kH = 64;            // Hadamard block size (OrbitQuant §2.3: h = 64)
constexpr int kMaxD = 32768;      // largest supported input width (one token row in shared memory)
constexpr int kMaxDevices = 64;

// Device-resident copy of one RPBH draw, laid out for the fused kernels.
struct RpbhDevice {
  bool ready = false;
  int32_t* perm = nullptr;        // pi(k), destination order
  float* sign = nullptr;          // D_k as +-1.0f, destination order
  // Gather table of the token-pair kernel (built on first use): for output
  // position k, at pair_tab_slot(k / 64, k % 64), the byte offset 2 pi(k) of
  // its source in a staged row with the sign D_k in bit 31 (set for -1).
  uint32_t* pair_tab = nullptr;
  // The same in 16 bits for wide rows (d <= 16384), at pair_tab16_slot(k / 64,
  // k % 64): the byte offset 2 pi(k) (< 2^15) with D_k in bit 15.
  uint16_t* pair_tab16 = nullptr;
};

// Slot of output position (block b, index i) in the token-pair kernel's
// tables: the 16-byte chunk index inside the block is XORed with b & 7 so that
// the four blocks a warp reads hit four different bank quads.
__host__ __device__ inline uint32_t pair_tab_slot(int b, int i) {
  return 64u * b + 4u * ((static_cast<uint32_t>(i) >> 2) ^ (static_cast<uint32_t>(b) & 7u)) + (i & 3);
}

// The same for the 16-bit table: 8 entries per 16-byte chunk, the chunk
// index XORed with b & 7.
__host__ __device__ inline uint32_t pair_tab16_slot(int b, int i) {
  return 64u * b + 8u * ((static_cast<uint32_t>(i) >> 3) ^ (static_cast<uint32_t>(b) & 7u)) + (i & 7);
}

}  // namespace rbq

struct rbq_rpbh {
  int d = 0;
  uint64_t seed = 0;
  int flags = 0;                  // RBQ_RPBH_NO_* ablation flags of the draw
  std::vector<int32_t> perm;      // pi
  std::vector<int8_t> sign;       // D
  rbq::RpbhDevice dev[rbq::kMaxDevices];
};

namespace rbq {

// Per (device, d, bits) codebook tables for the kernels.
struct CodebookDevice {
  int d = 0, bits = 0;
  float* bounds = nullptr;        // fp32[2^bits - 1], increasing
  uint16_t* levels_f16 = nullptr; // fp16[2^bits]: levels times sqrt(d) (unit scale)
  float inv_d = 0.f;              // 1/d: undoes the two sqrt(d) factors in qlinear
  // qlinear_int8_levels: levels rounded onto a signed 8-bit grid,
  // RNE(alpha * level), alpha = 127 / max |level| (int8[256], zero padded).
  int8_t* levels_i8 = nullptr;
  double alpha = 0.0;
  // qlinear_fp8_levels: levels times beta = 2^(7 - floor(log2 max |level|))
  // rounded to FP8 E4M3 (round to nearest even), as E4M3 bytes (uint8[256],
  // zero padded); the power-of-two beta leaves only the 3-bit mantissa rounding.
  uint8_t* levels_e4m3 = nullptr;
  double beta = 0.0;
  // Code-search grid: `grid_cells` + 1 cells centred at -R + n*2R/cells;
  // entry n = {boundary inside cell n or +inf, number of boundaries below
  // that cell}.  See build_grid() in rbq_host.cu.
  float2* grid = nullptr;
  int grid_cells = 0;
  float grid_scale = 0.f;         // 1 / (2R)
  // The same over v in [-1, 1] (R = 1, no clamp needed); null when it would
  // need more than kMaxFullGridCells cells.
  float2* grid_full = nullptr;
  int grid_full_cells = 0;
  // The [-R, R] grid again with kGridGuard copies of the end entries before
  // and after, padded to an even entry count, so that one bulk copy (16-byte
  // multiple) brings a guarded grid into shared memory.
  float2* grid_pad = nullptr;
};

constexpr int kGridGuard = 2;
// Entries of a guarded grid of n entries (see CodebookDevice::grid_pad).
__host__ __device__ inline int guarded_grid_entries(int n) { return (n + 2 * kGridGuard + 1) & ~1; }

constexpr int kMaxFullGridCells = 5000;

// Returns the device tables of `r` on the current device, uploading on first use.
int rpbh_device(const rbq_rpbh* r, const RpbhDevice** out);
// Returns the token-pair kernel's gather table of `r` on the current device
// (d words, see RpbhDevice::pair_tab), building it on first use.
int rpbh_pair_tables(const rbq_rpbh* r, const uint32_t** out);
// The 16-bit gather table (d <= 16384; see RpbhDevice::pair_tab16).
int rpbh_pair_tables16(const rbq_rpbh* r, const uint16_t** out);
// Returns the codebook of (d, bits) on the current device, computing and
// uploading it on first use.
int codebook_device(int d, int bits, const CodebookDevice** out);

// The 8-bit integer levels of a codebook (see CodebookDevice::levels_i8).
void int8_levels(const std::vector<double>& levels, std::vector<int8_t>& out, double* alpha);
// The FP8 E4M3 levels of a codebook (see CodebookDevice::levels_e4m3).
void fp8_levels(const std::vector<double>& levels, std::vector<uint8_t>& out, double* beta);

// Records a CUDA error (for rbq_error_string) and maps it to RBQ_ECUDA.
int cuda_fail(cudaError_t e);

// Device error word (bounded waits record here); defined in rbq_host.cu.
int device_error_word_ptr(unsigned int** out);

inline bool aligned(const void* p, size_t a) {
  return (reinterpret_cast<uintptr_t>(p) % a) == 0;
}

}  // namespace rbq
