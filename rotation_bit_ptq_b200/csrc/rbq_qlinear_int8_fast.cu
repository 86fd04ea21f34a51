// qlinear_int8, throughput version: the W8A16 linear of the INT8 path.
//
//   INT8-convrot (cloud.baidu.com/article/9430339) §4: rotate, quantise to
//   INT8 per output channel, then run the layer through an INT8-aware operator:
//     Y[m, n] = bf16( scale[n] * sum_k q[n, k] * x'[m, k] ),  x' = bf16(Pi x).
//
// Two kernels per call.
//
// 1. widen_int8_kernel: q [N, K] int8 -> bf16 [N, K] in a stream-ordered
//    workspace.  Integers up to 127 are exact in bf16, so the tensor core sees
//    the same values; an HBM pass over 3 N K bytes.
// 2. qlinear_bf16_kernel: persistent tcgen05 GEMM, K slices of 64, on CTA
//    pairs (256 x 256 output tiles, cta_group::2) when there is more than one
//    128-row tile of rows, else one CTA per SM (128 x 256 tiles).
//      warps 0..3  epilogue: TMEM lane quadrant w, one output row of this
//                  CTA's 128 per thread; multiply by scale[n], round to BF16,
//                  store.
//      warp 4      MMA issuer (the even CTA's, for a pair): one thread, four
//                  kind::f16 (bf16) MMAs per slice from shared memory, one
//                  commit per slice (to both CTAs' stage barriers).
//      warp 5      TMA producer: this CTA's x' tile (128 x 64) and its part
//                  of the weight tile (256 x 64, or 128 x 64 for a pair) of
//                  each slice into the ring (4 stages of 48 KB, or 6 of 32
//                  KB), both 128B-swizzled K-major.  A pair's weight tile
//                  is split between the two CTAs, each loading its part.
//    Two TMEM accumulators (2 x 256 columns) let the epilogue of tile i
//    overlap the MMAs of tile i+1.
//    Fused with the next layer's rotation (qlinear_int8_rotate_next, see
//    rbq_fused.cu) the epilogue does more per element -- an activation, the
//    signs, the 64-point Walsh-Hadamard transform on packed pairs -- so it runs
//    on eight warps (0..3 and 6..9, two per TMEM lane quadrant), each thread
//    finishing two of a tile's four 64-column blocks.
//
// Every mbarrier wait is bounded (see qlinear_fast); a thread whose wait runs
// out raises the shared abort flag and records an error bit.

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include "rbq_internal.h"
#include "rbq_qcodes.cuh"
#include "rbq_sm100.cuh"
#include "rbq_tiles.cuh"

namespace rbq {
namespace q8fast {

using namespace sm100;
using qfast::encode_fn;
using qfast::workspace_pool;
using tiles::tile_coords;
using tiles::tile_order;

constexpr int kBM = 128, kBN = 256, kBK = 64;
constexpr int kATile = kBM * kBK * 2;          // 16 KB
constexpr int kMaxStages = 6;
constexpr int kMmaWarp = 4, kTmaWarp = 5;

// Tile geometry.  Single-SM tiles are 128 x 256: the CTA holds the whole
// 256 x 64 weight tile of each K slice (4 stages of 48 KB).  CTA-pair tiles
// are 256 x 256: one thread of the even CTA issues each MMA for both SMs
// (cta_group::2, M = 256), each CTA holds its own 128 rows of x' and 128 of
// the 256 weight rows (6 stages of 32 KB), and each CTA's tensor memory
// receives its own 128 output rows.  The pair does the same MMA work per SM
// with a third fewer operand bytes arriving per K slice, and the freed shared
// memory deepens the ring.
template <bool PAIR>
struct Geom {
  static constexpr int kTileM = PAIR ? 2 * kBM : kBM;     // output rows per tile
  static constexpr int kBNc = PAIR ? kBN / 2 : kBN;       // weight rows loaded per CTA
  static constexpr int kBTile = kBNc * kBK * 2;           // 16 KB / 32 KB
  static constexpr int kStage = kATile + kBTile;          // 32 KB / 48 KB
  static constexpr int kStages = PAIR ? 6 : 4;
};
static_assert(Geom<true>::kStages * Geom<true>::kStage == Geom<false>::kStages * Geom<false>::kStage,
              "both geometries use the same shared memory");

// Epilogue kinds.
enum Epi {
  kEpiScale = 0,        // W8A16: Y = bf16(acc * scale[n])
  kEpiCodes = 1,        // qlinear on expanded code levels: Y = bf16(acc * s[m] r'[n] / K)
  kEpiRotateNext = 2,   // W8A16 whose output feeds the next rotated layer: per 64-column
                        // block, Y = bf16(H_64 D (act(acc * scale)) / 8), act = identity
  kEpiRotateNextGelu = 3,   // the same with act = GELU
  kEpiCodesRotateNext = 4,      // qlinear on expanded code levels whose output feeds the next rotated
                                // layer: y = acc * s[m] r'[n] / K, then as kEpiRotateNext
  kEpiCodesRotateNextGelu = 5,  // the same with act = GELU
};
__host__ __device__ constexpr bool epi_codes(int epi) { return epi == kEpiCodes || epi >= kEpiCodesRotateNext; }
__host__ __device__ constexpr bool epi_gelu(int epi) {
  return epi == kEpiRotateNextGelu || epi == kEpiCodesRotateNextGelu;
}

// Threads per CTA: 4 epilogue warps + MMA warp + TMA warp; the rotating
// epilogues add 4 more epilogue warps (warps 6..9), two per TMEM lane
// quadrant, so that each thread finishes two of a tile's four Hadamard blocks.
__host__ __device__ constexpr int threads_for(int epi) { return epi >= kEpiRotateNext ? 320 : 192; }
__host__ __device__ constexpr int epi_threads_for(int epi) { return epi >= kEpiRotateNext ? 256 : 128; }

struct Params {
  int M, N, K;
  int order;                  // tile order (TileOrder)
  const float* scale;         // W8A16: per-column scales
  const float* s;             // qlinear: per-row norms
  const uint16_t* rnorm;      // qlinear: BF16 per-column norms
  float inv_k;                // qlinear: 1/K (the fp16 levels carry sqrt(K) each)
  const float* next_sign;     // rotating epilogues: D of the next layer (+-1, output position order)
  uint16_t* Y;
  unsigned int* err;
  int y32;                    // Y 32-byte aligned with N % 16 == 0: 32-byte output stores
};

// 32 bytes (eight words) to global memory in one store; dst 32-byte aligned.
__device__ __forceinline__ void st_v8(void* dst, const uint32_t* w) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(dst), "r"(w[0]), "r"(w[1]),
               "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
               : "memory");
}

// GELU(y) = y Phi(y) with the normal CDF from Abramowitz & Stegun (1964),
// formula 7.1.26 (Hastings' rational approximation of erf, |error| <= 1.5e-7
// for x >= 0): for x = |y| / sqrt 2, t = 1 / (1 + p x),
// erfc(x) ~= t (a1 + t (a2 + t (a3 + t (a4 + t a5)))) exp(-x^2), and
// Phi(y) = 1 - erfc(x) / 2 for y >= 0, erfc(x) / 2 for y < 0.  Phi is within
// 1e-7 of the exact value, far below the BF16 rounding of the layer's output.
// (A reciprocal by Newton-Raphson on the FMA pipe instead of the division
// measured no faster.)
__device__ __forceinline__ float gelu_as7126(float y) {
  const float x = fabsf(y) * 0.70710678118654752f;
  const float t = __fdividef(1.0f, fmaf(0.3275911f, x, 1.0f));
  float poly = fmaf(t, 1.061405429f, -1.453152027f);
  poly = fmaf(t, poly, 1.421413741f);
  poly = fmaf(t, poly, -0.284496736f);
  poly = fmaf(t, poly, 0.254829592f);
  const float half_erfc = 0.5f * t * poly * __expf(-x * x);
  return y * (y >= 0.f ? 1.0f - half_erfc : half_erfc);
}

__device__ __forceinline__ unsigned long long pk2(float a, float b) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void upk2(unsigned long long r, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}
__device__ __forceinline__ unsigned long long add_f2(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ unsigned long long sub_f2(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// In-place unnormalised 64-point Walsh-Hadamard transform (Sylvester order)
// on the pairs P[i] = (z_i, z_{i+32}): strides 1..16 act on both halves of a
// pair alike (one packed add/sub each), stride 32 combines the two halves.
__device__ __forceinline__ void fwht64_pairs(unsigned long long (&P)[32]) {
#pragma unroll
  for (int len = 1; len < 32; len <<= 1) {
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      if ((i & len) == 0) {
        const unsigned long long a = P[i], b = P[i + len];
        P[i] = add_f2(a, b);
        P[i + len] = sub_f2(a, b);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    float lo, hi;
    upk2(P[i], lo, hi);
    P[i] = pk2(lo + hi, lo - hi);        // (z_i, z_{i+32})
  }
}

struct __align__(8) Tail {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t drain;                // abort path only: completion of the MMAs issued
  uint32_t tmem_slot;
  volatile uint32_t abort;
};

constexpr size_t kSmem = 1024 + Geom<false>::kStages * Geom<false>::kStage + sizeof(Tail) + 64;

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, Tail* tl) {
  return mbar_wait_or_abort(bar, parity, &tl->abort);
}
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, Tail* tl) {
  return mbar_warp_wait(bar, parity, &tl->abort);
}

// EPI = kEpiScale: the W8A16 layer (bf16 operands, epilogue x scale[n]);
// kEpiCodes: qlinear on codes expanded beforehand into fp16 levels (x sqrt(K)),
// epilogue x s[m] r'[n] / K; kEpiRotateNext: the W8A16 layer whose weight rows
// come in the order of the next layer's permutation, its epilogue applying the
// activation and the next layer's signs and 64-point Hadamard blocks.
// PAIR: the kernel runs on clusters of two CTAs (see Geom).
template <int EPI, bool PAIR>
__global__ void __launch_bounds__(threads_for(EPI), 1)
    qlinear_bf16_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const Params p) {
  using G = Geom<PAIR>;
  constexpr int kS = G::kStages;
  constexpr bool kQ = epi_codes(EPI);
  constexpr bool kRot = (EPI >= kEpiRotateNext);
  constexpr uint32_t kEpiWarps = epi_threads_for(EPI) / 32;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* ops = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  Tail* tl = reinterpret_cast<Tail*>(ops + kS * G::kStage);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;       // CTA within the pair
  const int tile0 = PAIR ? static_cast<int>(cluster_id_x()) : static_cast<int>(blockIdx.x);
  const int tstep = PAIR ? static_cast<int>(cluster_count_x()) : static_cast<int>(gridDim.x);
  const int ntiles_m = (p.M + G::kTileM - 1) / G::kTileM, ntiles_n = (p.N + kBN - 1) / kBN;
  const int ntiles = ntiles_m * ntiles_n;
  const int KT = p.K / kBK;

  if (tid == 0) {
    for (int s = 0; s < kS; ++s) {
      mbar_init(&tl->full[s], 1);
      mbar_init(&tl->empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tl->acc_full[a], 1);
      // one arrival per epilogue warp (of both CTAs for a pair: the even CTA's
      // MMA thread waits for both halves of the accumulator to be drained)
      mbar_init(&tl->acc_empty[a], (PAIR ? 2u : 1u) * kEpiWarps);
    }
    mbar_init(&tl->drain, 1);
    tl->abort = 0u;
    mbar_fence_init();
  }
  if (warp == kMmaWarp) {
    if constexpr (PAIR) {
      tmem_alloc_pair(&tl->tmem_slot, 512);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(&tl->tmem_slot, 512);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  // A pair's barriers are signalled from both CTAs: both must be initialised.
  if constexpr (PAIR)
    cluster_sync();
  else
    __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tl->tmem_slot;
  // The prologue above reads only constant tables; the operands (written by
  // the kernels before this one on the stream) wait for them.
  griddep_wait();
  griddep_launch_dependents();

  if (warp == kMmaWarp) {
    // ---------------- MMA issuer (the even CTA's, for a pair) ----------------
    if (lane == 0 && rank == 0) {
      constexpr uint32_t kIdesc = idesc_f16(G::kTileM, kBN, !kQ);
      const uint64_t desc0 = sdesc_k_sw128(smem_u32(ops));
      uint32_t s = 0, ph = 0, it = 0;
      bool ok = true;
      for (int tile = tile0; tile < ntiles && ok; tile += tstep, ++it) {
        const uint32_t a = it & 1u, use = it >> 1;
        if (use >= 1) {
          const bool got = PAIR ? mbar_wait_or_abort_cl(&tl->acc_empty[a], (use - 1) & 1, &tl->abort)
                                : wait_or_abort(&tl->acc_empty[a], (use - 1) & 1, tl);
          if (!got) { ok = false; break; }
        }
        tc_fence_after();
        const uint32_t acc = tmem + a * kBN;
        for (int kb = 0; kb < KT; ++kb) {
          if (!wait_or_abort(&tl->full[s], ph, tl)) { ok = false; break; }
          tc_fence_after();
          const uint64_t ad = desc0 + ((s * static_cast<uint32_t>(G::kStage)) >> 4);
          const uint64_t bd = ad + (kATile >> 4);
          if constexpr (PAIR) {
            umma_f16_pair(acc, ad, bd, kIdesc, kb != 0);
            umma_f16_pair(acc, ad + 2, bd + 2, kIdesc, 1u);      // +32 bytes of K per step
            umma_f16_pair(acc, ad + 4, bd + 4, kIdesc, 1u);
            umma_f16_pair(acc, ad + 6, bd + 6, kIdesc, 1u);
            umma_commit_pair(&tl->empty[s], 3);                  // stage s of both CTAs
          } else {
            umma_f16(acc, ad, bd, kIdesc, kb != 0);
            umma_f16(acc, ad + 2, bd + 2, kIdesc, 1u);
            umma_f16(acc, ad + 4, bd + 4, kIdesc, 1u);
            umma_f16(acc, ad + 6, bd + 6, kIdesc, 1u);
            umma_commit(&tl->empty[s]);
          }
          if (++s == kS) { s = 0; ph ^= 1u; }
        }
        if (ok) {
          if constexpr (PAIR)
            umma_commit_pair(&tl->acc_full[a], 3);
          else
            umma_commit(&tl->acc_full[a]);
        }
      }
      if (!ok) atomicOr(p.err, 2u);
    }
  } else if (warp == kTmaWarp) {
    // ---------------- TMA producer ----------------
    // For a pair each CTA loads its own 128 rows of x' and its half of the
    // weight rows; both CTAs' bytes are counted on the even CTA's barrier,
    // which only the even CTA's producer arms.
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB);
      uint32_t s = 0, ph = 0;
      bool first = true, ok = true;
      for (int tile = tile0; tile < ntiles && ok; tile += tstep) {
        int mt, nt;
        tile_coords(tile, ntiles_m, ntiles_n, p.order, mt, nt);
        const int m0 = mt * G::kTileM + static_cast<int>(rank) * kBM;
        const int n0 = nt * kBN + static_cast<int>(rank) * G::kBNc;
        for (int kb = 0; kb < KT; ++kb) {
          if (!first && !wait_or_abort(&tl->empty[s], ph ^ 1u, tl)) { ok = false; break; }
          uint8_t* st = ops + s * G::kStage;
          if constexpr (PAIR) {
            if (rank == 0) mbar_arrive_expect_tx(&tl->full[s], 2 * G::kStage);
            const uint32_t bar = mapa_shared(&tl->full[s], 0);
            tma_load_2d_pair(st, &tmA, kb * kBK, m0, bar);
            tma_load_2d_pair(st + kATile, &tmB, kb * kBK, n0, bar);
          } else {
            mbar_arrive_expect_tx(&tl->full[s], G::kStage);
            tma_load_2d(st, &tmA, kb * kBK, m0, &tl->full[s]);
            tma_load_2d(st + kATile, &tmB, kb * kBK, n0, &tl->full[s]);
          }
          if (++s == kS) { s = 0; ph ^= 1u; first = false; }
        }
      }
      if (!ok) atomicOr(p.err, 16u);
    }
  } else {
    // ---------------- epilogue ----------------
    const int q = warp & 3;                 // TMEM lane quadrant (warps 6..9: 2, 3, 0, 1)
    const int r = 32 * q + lane;            // row within this CTA's 128 rows of the tile
    const int eg = warp < 4 ? 0 : 1;        // rotating epilogues: which two of the four blocks
    // Accumulator drained: one arrival per warp, on the even CTA's barrier.
    auto release_acc = [&](uint32_t a) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if constexpr (PAIR)
          mbar_arrive_cluster(mapa_shared(&tl->acc_empty[a], 0));
        else
          mbar_arrive(&tl->acc_empty[a]);
      }
    };
    uint32_t it = 0;
    for (int tile = tile0; tile < ntiles; tile += tstep, ++it) {
      const uint32_t a = it & 1u, use = it >> 1;
      if (!warp_wait(&tl->acc_full[a], use & 1, tl)) {
        if (lane == 0) atomicOr(p.err, 4u);
        break;
      }
      tc_fence_after();
      int mt, nt;
      tile_coords(tile, ntiles_m, ntiles_n, p.order, mt, nt);
      const int m = mt * G::kTileM + static_cast<int>(rank) * kBM + r;
      if constexpr (kRot) {
        // The tile's 256 columns are four whole blocks of the next layer's
        // rotation (N % 64 == 0, tiles start at multiples of 256): column k is
        // the producing layer's output channel pi(k), so block b of the next
        // layer's rotated input is H_64 D_b act(y) over these 64 columns.
        // This thread's warp group takes blocks 2 eg and 2 eg + 1.
#pragma unroll 1
        for (int blk = 2 * eg; blk < 2 * eg + 2; ++blk) {
          uint32_t v0[32], v1[32];
          __syncwarp();                   // the loads are warp-collective; rows past M only skip the stores
          tmem_ld32(tmem + (static_cast<uint32_t>(32 * q) << 16) + a * kBN + 64 * blk, v0);
          tmem_ld32(tmem + (static_cast<uint32_t>(32 * q) << 16) + a * kBN + 64 * blk + 32, v1);
          tmem_wait_ld();
          const int n0 = nt * kBN + 64 * blk;
          if (m >= p.M || n0 >= p.N) continue;
          // per-column factor: the W8A16 scale, or r'_n (BF16) for the code layer,
          // whose per-row factor s_m / K comes in rs
          const auto colf = [&](int n) {
            if constexpr (kQ) return __uint_as_float(static_cast<uint32_t>(__ldg(p.rnorm + n)) << 16);
            else return __ldg(p.scale + n);
          };
          const float rs = kQ ? p.s[m] * p.inv_k : 1.f;
          unsigned long long P[32];       // (z_i, z_{i+32})
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            float y0 = __uint_as_float(v0[i]) * rs * colf(n0 + i);
            float y1 = __uint_as_float(v1[i]) * rs * colf(n0 + 32 + i);
            if constexpr (epi_gelu(EPI)) {
              y0 = gelu_as7126(y0);
              y1 = gelu_as7126(y1);
            }
            P[i] = pk2(y0 * __ldg(p.next_sign + n0 + i), y1 * __ldg(p.next_sign + n0 + 32 + i));
          }
          fwht64_pairs(P);
          uint4* d4 = reinterpret_cast<uint4*>(p.Y + static_cast<long long>(m) * p.N + n0);
#pragma unroll
          for (int half = 0; half < 2; ++half) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              uint32_t w[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                float a0, a1, b0, b1;
                upk2(P[8 * j + 2 * e], a0, a1);
                upk2(P[8 * j + 2 * e + 1], b0, b1);
                const __nv_bfloat162 h = half ? __floats2bfloat162_rn(a1 * 0.125f, b1 * 0.125f)
                                              : __floats2bfloat162_rn(a0 * 0.125f, b0 * 0.125f);
                w[e] = *reinterpret_cast<const uint32_t*>(&h);
              }
              d4[4 * half + j] = make_uint4(w[0], w[1], w[2], w[3]);
            }
          }
        }
        release_acc(a);
        continue;
      }
      const float rs = kQ ? ((m < p.M) ? p.s[m] * p.inv_k : 0.f) : 1.f;
#pragma unroll 1
      for (int cc = 0; cc < kBN / 32; ++cc) {
        uint32_t v[32];
        tmem_ld32(tmem + (static_cast<uint32_t>(32 * q) << 16) + a * kBN + 32 * cc, v);
        tmem_wait_ld();
        const int nb = nt * kBN + 32 * cc;
        if (m >= p.M || nb >= p.N) continue;
        uint16_t* dst = p.Y + static_cast<long long>(m) * p.N + nb;
        if (nb + 32 <= p.N) {
          uint32_t packed[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            float c0, c1;
            if constexpr (kQ) {
              const uint32_t rr = *reinterpret_cast<const uint32_t*>(p.rnorm + nb + 2 * j);
              c0 = rs * __uint_as_float(rr << 16);
              c1 = rs * __uint_as_float(rr & 0xFFFF0000u);
            } else {
              c0 = __ldg(p.scale + nb + 2 * j);
              c1 = __ldg(p.scale + nb + 2 * j + 1);
            }
            const __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(v[2 * j]) * c0, __uint_as_float(v[2 * j + 1]) * c1);
            packed[j] = *reinterpret_cast<const uint32_t*>(&h);
          }
          // a lane writes 64 bytes of its own row: as two 32-byte stores each
          // fills whole sectors (16-byte stores leave every piece alone in one)
          if (p.y32) {
            st_v8(dst, packed);
            st_v8(dst + 16, packed + 8);
          } else {
            uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
            for (int j = 0; j < 4; ++j)
              d4[j] = make_uint4(packed[4 * j], packed[4 * j + 1], packed[4 * j + 2], packed[4 * j + 3]);
          }
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (nb + j < p.N) {
              const float c = kQ ? rs * __uint_as_float(static_cast<uint32_t>(p.rnorm[nb + j]) << 16) : p.scale[nb + j];
              dst[j] = __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(v[j]) * c));
            }
        }
      }
      release_acc(a);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (tl->abort) {                 // the same value in every thread after the barrier
    drain_after_abort(warp == kMmaWarp && lane == 0 && rank == 0, &tl->drain, PAIR);
    __syncthreads();
  }
  // Neither CTA of a pair leaves while the other may still signal its
  // barriers or the MMAs may still read its shared memory.
  if constexpr (PAIR) cluster_sync();
  if (warp == kMmaWarp) {
    tc_fence_after();
    if constexpr (PAIR)
      tmem_dealloc_pair(tmem, 512);
    else
      tmem_dealloc(tmem, 512);
  }
}

// uint8 q [N, K] with a zero point per row -> bf16 (q - z) [N, K], 16 values
// per thread; |q - z| <= 255 is exact in bf16, so the layer needs no extra
// epilogue term (the asymmetric variant of INT8-convrot's "quantized model
// file": scale and zero point per channel).  K % 16 == 0: a group never
// straddles two rows.
__global__ void __launch_bounds__(256) widen_u8_zp_kernel(const uint8_t* q, const uint8_t* zp, int K,
                                                          long long groups, uint16_t* out) {
  for (long long g = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; g < groups;
       g += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int z = zp[(g * 16) / K];
    const uint4 v = __ldcs(reinterpret_cast<const uint4*>(q) + g);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int a = static_cast<int>((w[i] >> (16 * h)) & 0xFFu) - z;
        const int b = static_cast<int>((w[i] >> (16 * h + 8)) & 0xFFu) - z;
        const __nv_bfloat162 pr = __floats2bfloat162_rn(static_cast<float>(a), static_cast<float>(b));
        o[2 * i + h] = *reinterpret_cast<const uint32_t*>(&pr);
      }
    }
    __stcg(reinterpret_cast<uint4*>(out) + 2 * g, make_uint4(o[0], o[1], o[2], o[3]));
    __stcg(reinterpret_cast<uint4*>(out) + 2 * g + 1, make_uint4(o[4], o[5], o[6], o[7]));
  }
}

// int8 [n] -> bf16 [n], 16 values per thread (16 bytes in, 32 bytes out).
__global__ void __launch_bounds__(256) widen_int8_kernel(const int8_t* q, long long groups, uint16_t* out) {
  for (long long g = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; g < groups;
       g += static_cast<long long>(gridDim.x) * blockDim.x) {
    const uint4 v = __ldcs(reinterpret_cast<const uint4*>(q) + g);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float f0 = static_cast<float>(static_cast<int8_t>((w[i] >> (16 * h)) & 0xFFu));
        const float f1 = static_cast<float>(static_cast<int8_t>((w[i] >> (16 * h + 8)) & 0xFFu));
        const __nv_bfloat162 b = __floats2bfloat162_rn(f0, f1);
        o[2 * i + h] = *reinterpret_cast<const uint32_t*>(&b);
      }
    }
    uint4* dst = reinterpret_cast<uint4*>(out) + 2 * g;
    __stcg(dst, make_uint4(o[0], o[1], o[2], o[3]));
    __stcg(dst + 1, make_uint4(o[4], o[5], o[6], o[7]));
  }
}

// bf16 [rows, K] K-major, box = 64 x box_rows, 128B swizzle.
int encode_bf16_map(CUtensorMap* map, const uint16_t* base, int rows, int K, int box_rows, bool f16 = false) {
  auto fn = encode_fn();
  if (!fn) return RBQ_ECUDA;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kBK), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                        const_cast<uint16_t*>(base), dims, strides, box,
                        estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? RBQ_OK : RBQ_ECUDA;
}

// Resident clusters of two for the pair kernel on device `dev` (0: none
// could be co-scheduled), queried once per device.
template <int EPI>
int pair_clusters(int dev) {
  static int cached[kMaxDevices] = {};        // 0 = not yet asked; else clusters + 1
  if (cached[dev]) return cached[dev] - 1;
  auto kern = qlinear_bf16_kernel<EPI, true>;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(2, 1, 1);
  cfg.blockDim = dim3(threads_for(EPI), 1, 1);
  cfg.dynamicSmemBytes = kSmem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  cached[dev] = n + 1;
  return n;
}

// Launches the GEMM on two fp16/bf16 operands already in memory (K % 64 == 0):
// on CTA pairs (256 x 256 tiles) when there is more than one 128-row tile of
// rows and the device can co-schedule pairs, else on single SMs.
template <int EPI>
int launch_gemm(const uint16_t* A, const uint16_t* B, const Params& p, cudaStream_t st, int sms) {
  constexpr bool kQ = epi_codes(EPI);
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= kMaxDevices) return RBQ_EINVAL;
  bool pair = p.M > kBM;
  if (pair) {
    e = cudaFuncSetAttribute(qlinear_bf16_kernel<EPI, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmem));
    if (e != cudaSuccess) return cuda_fail(e);
    pair = pair_clusters<EPI>(dev) >= 1;
  }
  const int tile_m = pair ? Geom<true>::kTileM : Geom<false>::kTileM;
  Params q = p;
  q.order = tile_order(dev, 2LL * p.M * p.K, 2LL * p.N * p.K);
  q.y32 = (reinterpret_cast<uintptr_t>(p.Y) % 32 == 0 && p.N % 16 == 0) ? 1 : 0;
  CUtensorMap mA, mB;
  int rc = encode_bf16_map(&mA, A, p.M, p.K, kBM, kQ);
  if (rc == RBQ_OK) rc = encode_bf16_map(&mB, B, p.N, p.K, pair ? Geom<true>::kBNc : Geom<false>::kBNc, kQ);
  if (rc != RBQ_OK) return rc;
  const int ntiles = ((p.M + tile_m - 1) / tile_m) * ((p.N + kBN - 1) / kBN);
  cudaLaunchConfig_t cfg{};
  cfg.blockDim = dim3(threads_for(EPI), 1, 1);
  cfg.dynamicSmemBytes = kSmem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (pair) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 2;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.numAttrs = 2;
    int clusters = pair_clusters<EPI>(dev);           // persistent: as many pairs as are resident at once
    if (clusters > ntiles) clusters = ntiles;
    cfg.gridDim = dim3(2 * clusters, 1, 1);
    e = cudaLaunchKernelEx(&cfg, qlinear_bf16_kernel<EPI, true>, mA, mB, q);
  } else {
    auto kern = qlinear_bf16_kernel<EPI, false>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kSmem));
    if (e != cudaSuccess) return cuda_fail(e);
    cfg.gridDim = dim3(ntiles < sms ? ntiles : sms, 1, 1);
    e = cudaLaunchKernelEx(&cfg, kern, mA, mB, q);
  }
  if (e == cudaSuccess) e = cudaGetLastError();
  return e == cudaSuccess ? RBQ_OK : cuda_fail(e);
}

}  // namespace q8fast

// qlinear on expanded operands: `af16` [M, K] and `wf16` [N, K] fp16 levels x
// sqrt(K).  next_sign != null: the epilogue finishes the next layer's rotation
// (N % 64 == 0, the weight rows in the next permutation's order, act given).
int qlinear_f16_operands_gemm(const uint16_t* af16, const float* s, const uint16_t* wf16, const uint16_t* rnorm,
                              float inv_k, int M, int N, int K, uint16_t* Y, unsigned int* err, cudaStream_t st,
                              int sms, const float* next_sign, int act) {
  q8fast::Params p{};
  p.M = M;
  p.N = N;
  p.K = K;
  p.s = s;
  p.rnorm = rnorm;
  p.inv_k = inv_k;
  p.next_sign = next_sign;
  p.Y = Y;
  p.err = err;
  if (!next_sign) return q8fast::launch_gemm<q8fast::kEpiCodes>(af16, wf16, p, st, sms);
  if (act == RBQ_ACT_GELU) return q8fast::launch_gemm<q8fast::kEpiCodesRotateNextGelu>(af16, wf16, p, st, sms);
  return q8fast::launch_gemm<q8fast::kEpiCodesRotateNext>(af16, wf16, p, st, sms);
}

bool qlinear_int8_fast_eligible(int M, int N, int K) {
  return M >= 1 && N >= 8 && (N % 8) == 0 && K >= 64 && (K % 64) == 0;
}

// next_sign != null: the kEpiRotateNext epilogue (N % 64 == 0, act given).
int qlinear_int8_fast_launch(const uint16_t* Xrot, const int8_t* Wq, const float* scale, int M, int N, int K,
                             uint16_t* Y, unsigned int* err, cudaStream_t st, const uint8_t* zero_point,
                             const float* next_sign, int act) {
  using namespace q8fast;
  int dev = 0, sms = 148;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= kMaxDevices) return RBQ_EINVAL;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaMemPool_t pool = workspace_pool(dev);
  if (!pool) return RBQ_ECUDA;
  void* ws = nullptr;
  e = cudaMallocFromPoolAsync(&ws, static_cast<size_t>(N) * K * 2, pool, st);
  if (e != cudaSuccess) return cuda_fail(e);
  uint16_t* wb = static_cast<uint16_t*>(ws);
  const long long groups = static_cast<long long>(N) * K / 16;
  long long blocks = (groups + 255) / 256;
  if (blocks > 16LL * sms) blocks = 16LL * sms;
  if (zero_point)
    widen_u8_zp_kernel<<<static_cast<int>(blocks), 256, 0, st>>>(reinterpret_cast<const uint8_t*>(Wq), zero_point, K,
                                                                 groups, wb);
  else
    widen_int8_kernel<<<static_cast<int>(blocks), 256, 0, st>>>(Wq, groups, wb);
  int rc = RBQ_OK;
  if ((e = cudaGetLastError()) != cudaSuccess) rc = cuda_fail(e);
  if (rc == RBQ_OK) {
    Params p{};
    p.M = M;
    p.N = N;
    p.K = K;
    p.scale = scale;
    p.next_sign = next_sign;
    p.Y = Y;
    p.err = err;
    // programmatic dependent launch: the prologue overlaps the widening kernel's tail
    if (!next_sign) rc = launch_gemm<kEpiScale>(Xrot, wb, p, st, sms);
    else if (act == RBQ_ACT_GELU) rc = launch_gemm<kEpiRotateNextGelu>(Xrot, wb, p, st, sms);
    else rc = launch_gemm<kEpiRotateNext>(Xrot, wb, p, st, sms);
  }
  e = cudaFreeAsync(ws, st);
  if (rc == RBQ_OK && e != cudaSuccess) rc = cuda_fail(e);
  return rc;
}

}  // namespace rbq
