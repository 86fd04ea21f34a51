// qlinear_int8_levels / qlinear_fp8_levels: the quantised linear layer on the
// 8-bit tensor cores.
//
//   OrbitQuant (hotelren.com/news/3376620) §2.2: with the rotation absorbed
//   into the weights it cancels, y[m,n] = s_m r'_n sum_k C_w[q_nk] C_a[p_mk].
//   Here each codebook's levels are first rounded onto a signed 8-bit grid,
//   l[j] = RNE(alpha c_j) with alpha = 127 / max_j |c_j|, so that
//     y[m,n] = s_m r'_n (sum_k l_w[q_nk] l_a[p_mk]) / (alpha_w alpha_a),
//   the sum exact in int32 (|sum| <= K 127^2 < 2^31 for K <= 32768), on
//   tcgen05 kind::i8: twice the fp16 tensor rate and half the operand bytes.
//   The FP8 form rounds beta c_j to E4M3 (beta a power of two, so only the
//   3-bit mantissa rounding remains) and sums in fp32 on kind::f8f6f4:
//     y[m,n] = s_m r'_n (sum_k e_w[q_nk] e_a[p_mk]) / (beta_w beta_a).
//   Both run the same kernels; only the level bytes, the MMA kind and the
//   accumulator type differ.
//
// Three kernels per call.
// 1./2. expand_weights_i8_*: the weight codes [N, K*b/8] and the activation
//    codes [M, K*b/8] become int8 levels [N, K] and [M, K] in one
//    stream-ordered workspace (4-bit codes by byte permutes over a 16-byte
//    register table, other widths through a byte table in shared memory).
//    The activation part (M*K bytes) stays in L2 for the GEMM.
// 3. qlinear_8bit_kernel: persistent, on CTA pairs (256 x 256 output tiles,
//    cta_group::2, 6 stages of 32 KB per CTA: 16 KB of activations and half
//    the weight tile) when there is more than one 128-row tile of rows, else
//    one CTA per SM (128 x 256 tiles, 4 stages of 48 KB); K slices of 128
//    int8 values (one 128-byte swizzle row per operand row):
//      warps 0..3  epilogue: TMEM lane quadrant, one output row per thread;
//                  int32 -> fp32, times s_m r'_n / (alpha_w alpha_a), BF16.
//      warp 4      MMA issuer (one thread; the even CTA's for a pair): four
//                  kind::i8 MMAs per slice (+32 bytes of K per step) into one
//                  of two int32 TMEM accumulators, so the epilogue of tile i
//                  overlaps the MMAs of tile i+1.
//      warp 5      TMA producer (one thread): this CTA's operand tiles of
//                  each slice into the ring, 128B-swizzled K-major (a pair
//                  splits the weight tile between its CTAs, each loading
//                  its own part).
// (Expanding the activation codes inside the GEMM, as the fp16 qlinear kernel
// does, measured slower here: at twice the tensor rate the expansion warps
// set the pace, 57.3 vs 51.4 us at 4608 x 3072 x 3072 W4A4.)
//
// Every mbarrier wait is bounded; a thread whose wait runs out raises a shared
// abort flag, records an error in the library's device error word, and the
// CTA still frees its TMEM.

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include "rbq_internal.h"
#include "rbq_qcodes.cuh"
#include "rbq_sm100.cuh"
#include "rbq_tiles.cuh"

namespace rbq {
namespace qi8 {

using namespace sm100;
using qfast::prmt;

constexpr int kBM = 128, kBN = 256, kBK = 128;  // K values per slice (= bytes per operand row)
constexpr int kATile = kBM * kBK;               // 16 KB int8 activation tile
constexpr int kMaxStages = 6;
constexpr int kThreads = 192;                   // 6 warps
constexpr int kMmaWarp = 4, kTmaWarp = 5;

// Single-SM tiles are 128 x 256 (the CTA holds the whole 256 x 128 weight
// tile of a slice, 4 stages of 48 KB); CTA-pair tiles are 256 x 256 (each CTA
// holds its 128 activation rows and 128 of the 256 weight rows, 6 stages of
// 32 KB; one thread of the even CTA issues the cta_group::2 MMAs), as in the
// fp16 GEMM of rbq_qlinear_int8_fast.cu.  At twice the fp16 tensor rate the
// single SM's 48 KB per slice arrive too slowly; the pair halves the weight
// bytes per SM.
template <bool PAIR>
struct Geom {
  static constexpr int kTileM = PAIR ? 2 * kBM : kBM;
  static constexpr int kBNc = PAIR ? kBN / 2 : kBN;       // weight rows loaded per CTA
  static constexpr int kBTile = kBNc * kBK;               // 16 KB / 32 KB
  static constexpr int kStage = kATile + kBTile;          // 32 KB / 48 KB
  static constexpr int kStages = PAIR ? 6 : 4;
};
static_assert(Geom<true>::kStages * Geom<true>::kStage == Geom<false>::kStages * Geom<false>::kStage,
              "both geometries use the same shared memory");

// Instruction descriptor of kind::i8: s32 accumulator (D format 2), signed
// 8-bit A and B (format 1), both K-major, N>>3 at bit 17, M>>4 at bit 24.
__host__ __device__ constexpr uint32_t idesc_i8(int M, int N) {
  return (2u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// Instruction descriptor of kind::f8f6f4 with E4M3 A and B (format 0) and an
// fp32 accumulator (D format 1), both K-major.
__host__ __device__ constexpr uint32_t idesc_e4m3(int M, int N) {
  return (1u << 4) | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// D[tmem] (+)= A[smem] * B[smem]^T on 8-bit operands: signed integers with an
// int32 accumulator (kFp8 = false) or E4M3 with an fp32 one (kFp8 = true).
template <bool kFp8>
__device__ __forceinline__ void umma_8bit(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  if constexpr (kFp8) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
  } else {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
  }
}
// The same over a CTA pair (M = 256), issued by one thread of the even CTA.
template <bool kFp8>
__device__ __forceinline__ void umma_8bit_pair(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                               uint32_t accumulate) {
  if constexpr (kFp8) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
  } else {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
  }
}

// An accumulator word as fp32.
template <bool kFp8>
__device__ __forceinline__ float acc_value(uint32_t v) {
  if constexpr (kFp8) return __uint_as_float(v);
  else return __int2float_rn(static_cast<int>(v));
}

// The level bytes of codes 0..15 as four words (byte j of word w = level 4w+j).
struct Tab16 {
  uint32_t t0, t1, t2, t3;
};

__device__ __forceinline__ Tab16 make_tab16(const uint8_t* lut) {
  const uint32_t* w = reinterpret_cast<const uint32_t*>(lut);
  return Tab16{w[0], w[1], w[2], w[3]};
}

// Eight 4-bit codes (nibbles of x, LSB first) -> eight level bytes: the low
// three bits of a code pick a byte from the table half its top bit selects.
__device__ __forceinline__ uint2 expand8_4bit_i8(uint32_t x, const Tab16& T) {
  const uint32_t sel = x & 0x77777777u, sel1 = sel >> 16;
  const uint32_t lo0 = prmt(T.t0, T.t1, sel), hi0 = prmt(T.t2, T.t3, sel);
  const uint32_t lo1 = prmt(T.t0, T.t1, sel1), hi1 = prmt(T.t2, T.t3, sel1);
  // byte masks from the top bits: a7 has nibble 2i's bit at byte i's sign
  // bit, a3 nibble 2i+1's; sign-replicating byte selects spread them
  const uint32_t h = (x >> 3) & 0x11111111u;
  const uint32_t a7 = h << 7, a3 = h << 3;
  const uint32_t m0 = prmt(a7, a3, 0xD9C8u), m1 = prmt(a7, a3, 0xFBEAu);
  return make_uint2((hi0 & m0) | (lo0 & ~m0), (hi1 & m1) | (lo1 & ~m1));
}

// ---- the GEMM: both int8 operands by TMA ------------------------------------
struct Params {
  int M, N, K;
  const float* s;
  const uint16_t* rnorm;
  float inv_scale;
  uint16_t* Y;
  unsigned int* err;
  int order;                  // tile order (tiles::TileOrder)
};

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

template <bool kFp8, bool PAIR>
__global__ void __launch_bounds__(kThreads, 1)
    qlinear_8bit_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const Params p) {
  using G = Geom<PAIR>;
  constexpr int kS = G::kStages;
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
  const int KS = p.K / kBK;
  volatile uint32_t* abort = &tl->abort;

  if (tid == 0) {
    for (int s = 0; s < kS; ++s) {
      mbar_init(&tl->full[s], 1);
      mbar_init(&tl->empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tl->acc_full[a], 1);
      mbar_init(&tl->acc_empty[a], PAIR ? 8 : 4);    // one arrival per epilogue warp (of both CTAs)
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
  griddep_wait();
  griddep_launch_dependents();

  if (warp == kMmaWarp) {
    // ---------------- MMA issuer (the even CTA's, for a pair) ----------------
    if (lane == 0 && rank == 0) {
      constexpr uint32_t kIdesc = kFp8 ? idesc_e4m3(G::kTileM, kBN) : idesc_i8(G::kTileM, kBN);
      const uint64_t desc0 = sdesc_k_sw128(smem_u32(ops));
      uint32_t s = 0, ph = 0, it = 0;
      bool ok = true;
      for (int tile = tile0; tile < ntiles && ok; tile += tstep, ++it) {
        const uint32_t a = it & 1u, use = it >> 1;
        if (use >= 1) {
          const bool got = PAIR ? mbar_wait_or_abort_cl(&tl->acc_empty[a], (use - 1) & 1, abort)
                                : mbar_wait_or_abort(&tl->acc_empty[a], (use - 1) & 1, abort);
          if (!got) { ok = false; break; }
        }
        tc_fence_after();
        const uint32_t acc = tmem + a * kBN;
        for (int ks = 0; ks < KS; ++ks) {
          if (!mbar_wait_or_abort(&tl->full[s], ph, abort)) { ok = false; break; }
          tc_fence_after();
          const uint64_t ad = desc0 + ((s * static_cast<uint32_t>(G::kStage)) >> 4);
          const uint64_t bd = ad + (kATile >> 4);
          if constexpr (PAIR) {
            umma_8bit_pair<kFp8>(acc, ad, bd, kIdesc, ks != 0);
            umma_8bit_pair<kFp8>(acc, ad + 2, bd + 2, kIdesc, 1u);     // +32 bytes = 32 values of K
            umma_8bit_pair<kFp8>(acc, ad + 4, bd + 4, kIdesc, 1u);
            umma_8bit_pair<kFp8>(acc, ad + 6, bd + 6, kIdesc, 1u);
            umma_commit_pair(&tl->empty[s], 3);                          // stage s of both CTAs
          } else {
            umma_8bit<kFp8>(acc, ad, bd, kIdesc, ks != 0);
            umma_8bit<kFp8>(acc, ad + 2, bd + 2, kIdesc, 1u);
            umma_8bit<kFp8>(acc, ad + 4, bd + 4, kIdesc, 1u);
            umma_8bit<kFp8>(acc, ad + 6, bd + 6, kIdesc, 1u);
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
    // For a pair each CTA loads its own activation rows and its half of the
    // weight rows; both CTAs' bytes are counted on the even CTA's barrier.
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB);
      uint32_t s = 0, ph = 0;
      bool first = true, ok = true;
      for (int tile = tile0; tile < ntiles && ok; tile += tstep) {
        int mt, nt;
        tiles::tile_coords(tile, ntiles_m, ntiles_n, p.order, mt, nt);
        const int m0 = mt * G::kTileM + static_cast<int>(rank) * kBM;
        const int n0 = nt * kBN + static_cast<int>(rank) * G::kBNc;
        for (int ks = 0; ks < KS; ++ks) {
          if (!first && !mbar_wait_or_abort(&tl->empty[s], ph ^ 1u, abort)) { ok = false; break; }
          uint8_t* st = ops + s * G::kStage;
          if constexpr (PAIR) {
            if (rank == 0) mbar_arrive_expect_tx(&tl->full[s], 2 * G::kStage);
            const uint32_t bar = mapa_shared(&tl->full[s], 0);
            tma_load_2d_pair(st, &tmA, ks * kBK, m0, bar);
            tma_load_2d_pair(st + kATile, &tmB, ks * kBK, n0, bar);
          } else {
            mbar_arrive_expect_tx(&tl->full[s], G::kStage);
            tma_load_2d(st, &tmA, ks * kBK, m0, &tl->full[s]);
            tma_load_2d(st + kATile, &tmB, ks * kBK, n0, &tl->full[s]);
          }
          if (++s == kS) { s = 0; ph ^= 1u; first = false; }
        }
      }
      if (!ok) atomicOr(p.err, 16u);
    }
  } else {
    // ---------------- epilogue ----------------
    const int q = warp;                     // TMEM lane quadrant
    const int r = 32 * q + lane;            // row within this CTA's 128 rows of the tile
    uint32_t it = 0;
    for (int tile = tile0; tile < ntiles; tile += tstep, ++it) {
      const uint32_t a = it & 1u, use = it >> 1;
      if (!mbar_warp_wait(&tl->acc_full[a], use & 1, abort)) {   // warp-uniform: tmem loads follow
        if (lane == 0) atomicOr(p.err, 4u);
        break;
      }
      tc_fence_after();
      int mt, nt;
      tiles::tile_coords(tile, ntiles_m, ntiles_n, p.order, mt, nt);
      const int m = mt * G::kTileM + static_cast<int>(rank) * kBM + r;
      const float rs = (m < p.M) ? p.s[m] * p.inv_scale : 0.f;
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
            const uint32_t rr = *reinterpret_cast<const uint32_t*>(p.rnorm + nb + 2 * j);
            const float r0 = __uint_as_float(rr << 16), r1 = __uint_as_float(rr & 0xFFFF0000u);
            const float f0 = acc_value<kFp8>(v[2 * j]);
            const float f1 = acc_value<kFp8>(v[2 * j + 1]);
            const __nv_bfloat162 h = __floats2bfloat162_rn(f0 * rs * r0, f1 * rs * r1);
            packed[j] = *reinterpret_cast<const uint32_t*>(&h);
          }
          uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            d4[j] = make_uint4(packed[4 * j], packed[4 * j + 1], packed[4 * j + 2], packed[4 * j + 3]);
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            if (nb + j < p.N) {
              const float rv = __uint_as_float(static_cast<uint32_t>(p.rnorm[nb + j]) << 16);
              const float f = acc_value<kFp8>(v[j]);
              dst[j] = __bfloat16_as_ushort(__float2bfloat16_rn(f * rs * rv));
            }
          }
        }
      }
      // accumulator drained: one arrival per warp, on the even CTA's barrier
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if constexpr (PAIR)
          mbar_arrive_cluster(mapa_shared(&tl->acc_empty[a], 0));
        else
          mbar_arrive(&tl->acc_empty[a]);
      }
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

// Codes [rows, K*b/8] -> 8-bit levels [rows, K].  4-bit: a warp expands 128
// pairs of code words (16 codes each: 8 bytes in, 16 out) per step, lane l
// taking pairs l, l+32, l+64, l+96 of the warp's range, so every load and store
// instruction of the warp covers contiguous memory; other widths: a thread per
// 8 codes (b bytes in, 8 out).  K is a multiple of 128, so no group straddles
// two rows.
__global__ void __launch_bounds__(256) expand_weights_i8_4bit(const uint2* codes, long long pairs,
                                                             const int8_t* lut_g, uint4* out) {
  __shared__ __align__(16) uint8_t lut[16];
  if (threadIdx.x < 16) lut[threadIdx.x] = static_cast<uint8_t>(lut_g[threadIdx.x]);
  __syncthreads();
  const Tab16 T = make_tab16(lut);
  const int lane = threadIdx.x & 31;
  const long long warps = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
  for (long long base = (blockIdx.x * static_cast<long long>(blockDim.x >> 5) + (threadIdx.x >> 5)) * 128;
       base < pairs; base += 128 * warps) {
    uint2 v[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const long long g = base + 32 * j + lane;
      v[j] = g < pairs ? __ldcs(codes + g) : make_uint2(0u, 0u);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const long long g = base + 32 * j + lane;
      if (g < pairs) {
        const uint2 w0 = expand8_4bit_i8(v[j].x, T), w1 = expand8_4bit_i8(v[j].y, T);
        __stcg(out + g, make_uint4(w0.x, w0.y, w1.x, w1.y));
      }
    }
  }
}

template <int BITS>
__global__ void __launch_bounds__(256) expand_weights_i8_kernel(const uint8_t* codes, long long groups,
                                                               const int8_t* lut_g, uint2* out) {
  __shared__ __align__(16) uint8_t lut[256];
  for (int i = threadIdx.x; i < 256; i += blockDim.x) lut[i] = static_cast<uint8_t>(lut_g[i]);
  __syncthreads();
  constexpr uint32_t mask = (1u << BITS) - 1u;
  for (long long g = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; g < groups;
       g += static_cast<long long>(gridDim.x) * blockDim.x) {
    uint64_t x = 0;
    if constexpr (BITS == 8) {
      x = __ldcs(reinterpret_cast<const unsigned long long*>(codes) + g);
    } else if constexpr (BITS == 2) {
      x = __ldcs(reinterpret_cast<const unsigned short*>(codes) + g);
    } else {
      const uint8_t* src = codes + g * BITS;
#pragma unroll
      for (int i = 0; i < BITS; ++i) x |= static_cast<uint64_t>(__ldcs(src + i)) << (8 * i);
    }
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int e = 0; e < 8; ++e)
      w[e >> 2] |= static_cast<uint32_t>(lut[(x >> (BITS * e)) & mask]) << (8 * (e & 3));
    __stcg(out + g, make_uint2(w[0], w[1]));
  }
}

int expand_weights(const uint8_t* codes, int bits, int rows, int K, const int8_t* lut, int8_t* out,
                   cudaStream_t st, int sms) {
  const long long elems = static_cast<long long>(rows) * K;
  if (bits == 4) {
    const long long pairs = elems / 16;                     // 16 codes: 8 bytes in, 16 out
    long long blocks = (pairs + 1023) / 1024;               // 8 warps x 128 pairs
    if (blocks > 16LL * sms) blocks = 16LL * sms;
    expand_weights_i8_4bit<<<static_cast<int>(blocks), 256, 0, st>>>(reinterpret_cast<const uint2*>(codes), pairs,
                                                                      lut, reinterpret_cast<uint4*>(out));
  } else {
    const long long groups = elems / 8;
    long long blocks = (groups + 255) / 256;
    if (blocks > 16LL * sms) blocks = 16LL * sms;
    uint2* o = reinterpret_cast<uint2*>(out);
    const int nb = static_cast<int>(blocks);
    switch (bits) {
      case 1: expand_weights_i8_kernel<1><<<nb, 256, 0, st>>>(codes, groups, lut, o); break;
      case 2: expand_weights_i8_kernel<2><<<nb, 256, 0, st>>>(codes, groups, lut, o); break;
      case 3: expand_weights_i8_kernel<3><<<nb, 256, 0, st>>>(codes, groups, lut, o); break;
      case 5: expand_weights_i8_kernel<5><<<nb, 256, 0, st>>>(codes, groups, lut, o); break;
      case 6: expand_weights_i8_kernel<6><<<nb, 256, 0, st>>>(codes, groups, lut, o); break;
      case 7: expand_weights_i8_kernel<7><<<nb, 256, 0, st>>>(codes, groups, lut, o); break;
      default: expand_weights_i8_kernel<8><<<nb, 256, 0, st>>>(codes, groups, lut, o); break;
    }
  }
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? RBQ_OK : cuda_fail(e);
}

// int8 [rows, K] K-major, 256 x 128 boxes, 128B swizzle.
int encode_i8_map(CUtensorMap* map, const int8_t* base, int rows, int K, int box_rows = kBN) {
  auto fn = qfast::encode_fn();
  if (!fn) return RBQ_ECUDA;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kBK), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? RBQ_OK : RBQ_ECUDA;
}

// Resident clusters of two for the pair kernel on device `dev` (0: none
// could be co-scheduled), queried once per device.
template <bool kFp8>
int pair_clusters(int dev) {
  static int cached[kMaxDevices] = {};        // 0 = not yet asked; else clusters + 1
  if (cached[dev]) return cached[dev] - 1;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(2, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, qlinear_8bit_kernel<kFp8, true>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  cached[dev] = n + 1;
  return n;
}

// The GEMM on expanded int8 operands: activations `ai8` [M, K], weights `wi8`
// [N, K]; on CTA pairs when there is more than one 128-row tile of rows.
template <bool kFp8>
int gemm(const int8_t* ai8, const float* s, const int8_t* wi8, const uint16_t* rnorm, int M, int N, int K,
         uint16_t* Y, float inv_scale, unsigned int* err, cudaStream_t st, int sms) {
  Params p{};
  p.M = M;
  p.N = N;
  p.K = K;
  p.s = s;
  p.rnorm = rnorm;
  p.inv_scale = inv_scale;
  p.Y = Y;
  p.err = err;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= kMaxDevices) return RBQ_EINVAL;
  bool pair = M > kBM;
  if (pair) {
    e = cudaFuncSetAttribute(qlinear_8bit_kernel<kFp8, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmem));
    if (e != cudaSuccess) return cuda_fail(e);
    pair = pair_clusters<kFp8>(dev) >= 1;
  }
  const int tile_m = pair ? Geom<true>::kTileM : Geom<false>::kTileM;
  p.order = tiles::tile_order(dev, 1LL * M * K, 1LL * N * K);
  CUtensorMap mA, mB;
  int rc = encode_i8_map(&mA, ai8, M, K, kBM);
  if (rc != RBQ_OK) return rc;
  if ((rc = encode_i8_map(&mB, wi8, N, K, pair ? Geom<true>::kBNc : Geom<false>::kBNc)) != RBQ_OK) return rc;
  const int ntiles = ((M + tile_m - 1) / tile_m) * ((N + kBN - 1) / kBN);
  cudaLaunchConfig_t cfg{};
  cfg.blockDim = dim3(kThreads, 1, 1);
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
    int clusters = pair_clusters<kFp8>(dev);          // persistent: as many pairs as are resident at once
    if (clusters > ntiles) clusters = ntiles;
    cfg.gridDim = dim3(2 * clusters, 1, 1);
    e = cudaLaunchKernelEx(&cfg, qlinear_8bit_kernel<kFp8, true>, mA, mB, p);
  } else {
    auto kern = qlinear_8bit_kernel<kFp8, false>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kSmem));
    if (e != cudaSuccess) return cuda_fail(e);
    cfg.gridDim = dim3(ntiles < sms ? ntiles : sms, 1, 1);
    e = cudaLaunchKernelEx(&cfg, kern, mA, mB, p);
  }
  if (e == cudaSuccess) e = cudaGetLastError();
  return e == cudaSuccess ? RBQ_OK : cuda_fail(e);
}

}  // namespace qi8
}  // namespace rbq

using namespace rbq;

namespace {

// The two 8-bit-level layers: validation, level tables, both expansions, GEMM.
template <bool kFp8>
int qlinear_8bit_levels(const uint8_t* a_codes, const float* s, int bits_a, const uint8_t* w_codes,
                        const uint16_t* rnorm, int bits_w, int M, int N, int K, uint16_t* Y, void* stream) {
  if (M < 0 || N < 0 || K <= 0 || K % 128 || K > kMaxD) return RBQ_EINVAL;
  if (bits_a < 1 || bits_a > 8 || bits_w < 1 || bits_w > 8) return RBQ_EINVAL;
  if (N % 8 || (static_cast<long long>(K) * bits_a / 8) % 16) return RBQ_EINVAL;
  if (M == 0 || N == 0) return RBQ_OK;
  if (!a_codes || !s || !w_codes || !rnorm || !Y) return RBQ_EINVAL;
  if (!aligned(a_codes, 16) || !aligned(w_codes, 16) || !aligned(Y, 16) || !aligned(s, 4) || !aligned(rnorm, 4))
    return RBQ_EALIGN;
  const CodebookDevice *ca = nullptr, *cw = nullptr;
  int rc = codebook_device(K, bits_a, &ca);
  if (rc != RBQ_OK) return rc;
  if ((rc = codebook_device(K, bits_w, &cw)) != RBQ_OK) return rc;
  unsigned int* err = nullptr;
  if ((rc = device_error_word_ptr(&err)) != RBQ_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int dev = 0, sms = 148;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaMemPool_t pool = qfast::workspace_pool(dev);
  if (!pool) return RBQ_ECUDA;
  void* ws = nullptr;
  e = cudaMallocFromPoolAsync(&ws, (static_cast<size_t>(N) + M) * K, pool, st);
  if (e != cudaSuccess) return cuda_fail(e);
  int8_t* wq = static_cast<int8_t*>(ws);
  int8_t* aq = wq + static_cast<size_t>(N) * K;
  // level bytes: two's-complement integers or E4M3 codes, expanded alike
  const int8_t* lut_w = kFp8 ? reinterpret_cast<const int8_t*>(cw->levels_e4m3) : cw->levels_i8;
  const int8_t* lut_a = kFp8 ? reinterpret_cast<const int8_t*>(ca->levels_e4m3) : ca->levels_i8;
  const double scale = kFp8 ? ca->beta * cw->beta : ca->alpha * cw->alpha;
  rc = qi8::expand_weights(w_codes, bits_w, N, K, lut_w, wq, st, sms);
  if (rc == RBQ_OK) rc = qi8::expand_weights(a_codes, bits_a, M, K, lut_a, aq, st, sms);
  if (rc == RBQ_OK)
    rc = qi8::gemm<kFp8>(aq, s, wq, rnorm, M, N, K, Y, static_cast<float>(1.0 / scale), err, st, sms);
  e = cudaFreeAsync(ws, st);
  if (rc == RBQ_OK && e != cudaSuccess) rc = cuda_fail(e);
  return rc;
}

}  // namespace

extern "C" int qlinear_int8_levels(const uint8_t* a_codes, const float* s, int bits_a, const uint8_t* w_codes,
                                   const uint16_t* rnorm, int bits_w, int M, int N, int K, uint16_t* Y,
                                   void* stream) {
  return qlinear_8bit_levels<false>(a_codes, s, bits_a, w_codes, rnorm, bits_w, M, N, K, Y, stream);
}

extern "C" int qlinear_fp8_levels(const uint8_t* a_codes, const float* s, int bits_a, const uint8_t* w_codes,
                                  const uint16_t* rnorm, int bits_w, int M, int N, int K, uint16_t* Y,
                                  void* stream) {
  return qlinear_8bit_levels<true>(a_codes, s, bits_a, w_codes, rnorm, bits_w, M, N, K, Y, stream);
}
