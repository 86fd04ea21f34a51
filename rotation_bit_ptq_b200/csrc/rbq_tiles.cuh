// Tile order of the persistent tcgen05 GEMMs (rbq_qlinear_int8_fast.cu,
// rbq_qlinear_i8.cu): which output tile a CTA (pair) takes next.
#pragma once

#include <cuda_runtime.h>

namespace rbq {
namespace tiles {

// Order in which a CTA (pair) walks its output tiles, chosen on the host so
// that the operand panels a wave of CTAs touches stay in L2:
//   kOrderM  M fastest: a wave shares a few weight panels; the activation
//            operand is read once if it stays in L2 (it fits in half of it);
//   kOrderN  N fastest: a wave shares a few activation panels; for weights
//            that fit in half of L2 (read once) and a larger activation
//            operand (streamed once instead of once per column of tiles);
//   kOrderGrouped  neither fits: groups of kGroupM row panels, N fastest
//            inside a group, so a wave touches about kGroupM activation and
//            ~waves/kGroupM weight panels.
enum TileOrder { kOrderM = 0, kOrderN = 1, kOrderGrouped = 2 };
constexpr int kGroupM = 8;

__device__ __forceinline__ void tile_coords(int tile, int ntiles_m, int ntiles_n, int order, int& mt, int& nt) {
  if (order == kOrderM) {
    mt = tile % ntiles_m;
    nt = tile / ntiles_m;
  } else if (order == kOrderN) {
    mt = tile / ntiles_n;
    nt = tile % ntiles_n;
  } else {
    const int per_group = kGroupM * ntiles_n;
    const int g = tile / per_group, r = tile - g * per_group;
    const int m0 = g * kGroupM, gm = min(kGroupM, ntiles_m - m0);
    mt = m0 + r % gm;
    nt = r / gm;
  }
}

// The order for operands of a_bytes (activations) and b_bytes (weights) on
// device `dev`: the panels that can stay in L2 get half of it, the rest is
// for the output and the other operand's panels in flight.
inline int tile_order(int dev, long long a_bytes, long long b_bytes) {
  int l2 = 0;
  if (cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, dev) != cudaSuccess || l2 <= 0) l2 = 126 << 20;
  const long long half = static_cast<long long>(l2) / 2;
  if (b_bytes <= half && a_bytes > b_bytes) return kOrderN;
  if (a_bytes <= half) return kOrderM;
  if (b_bytes <= half) return kOrderN;
  return kOrderGrouped;
}

}  // namespace tiles
}  // namespace rbq
