// qlinear, throughput version: persistent, warp-specialised tcgen05 GEMM on
// packed Lloyd-Max codes.
//
//   OrbitQuant (hotelren.com/news/3376620) §2.2: the rotation absorbed into
//   the weights (§2.1) cancels the online one, so
//   y[m,n] = s_m r'_n sum_k C_w[q_nk] C_a[p_mk].
//
// Each CTA (one per SM) walks a static list of 128 x 256 output tiles.
//   warp 0          MMA issuer: one thread waits for a filled stage, issues
//                   four 128x256x16 kind::f16 MMAs into the tile's TMEM
//                   accumulator and commits them to the stage's "empty"
//                   barrier; after the last K slice it commits the
//                   accumulator to the epilogue.
//   warps 4..7      epilogue: TMEM lane quadrant w%4, one output row per
//                   thread; scale by s_m r'_n / K, round to BF16, store.
//   warps 8..19     operand expansion, one row per thread (128 rows of A,
//                   256 rows of B): read the row's 64 codes of the K slice,
//                   turn them into fp16 levels (x sqrt(K)), write the row into
//                   the stage's 128B-swizzled K-major tile.
// Four shared-memory stages decouple expansion from the MMAs; two TMEM
// accumulators (2 x 256 columns) let the epilogue of tile i overlap the MMAs
// of tile i+1.
//
// 4-bit codes are expanded in registers: by symmetry C[15-c] = -C[c], the
// magnitude index m (0..7) selects the two bytes of |C| with byte permutes
// (prmt) from four registers holding the low and high byte planes of the
// eight positive fp16 levels, and the sign lands on the high byte.  Other
// widths read a 2^b-entry fp16 table in shared memory.
//
// Every mbarrier wait is bounded; a thread whose wait runs out raises a
// shared abort flag (so the others stop waiting at once), records an error
// in the library's device error word, and the CTA still frees its TMEM.

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "rbq_internal.h"
#include "rbq_sm100.cuh"

namespace rbq {
namespace qfast {

using namespace sm100;

constexpr int kBM = 128, kBN = 256, kBK = 64, kStages = 4;
constexpr int kATile = kBM * kBK * 2;          // 16 KB
constexpr int kBTile = kBN * kBK * 2;          // 32 KB
constexpr int kStageBytes = kATile + kBTile;   // 48 KB
constexpr int kThreads = 640;                  // 20 warps
constexpr int kExpandFirst = 256;              // first expansion thread
constexpr int kExpandThreads = kBM + kBN;      // 384

struct Params {
  const uint8_t* A;        // activation codes [M, K*bits_a/8]
  const uint8_t* B;        // weight codes     [N, K*bits_b/8]
  int M, N, K;
  int bits_a, bits_b;
  const uint16_t* lut_a;   // fp16 levels x sqrt(K), 2^bits entries
  const uint16_t* lut_b;
  const float* s;
  const uint16_t* rnorm;
  float inv_k;
  uint16_t* Y;
  unsigned int* err;
};

struct __align__(8) Tail {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint32_t tmem_slot;
  volatile uint32_t abort;
  uint16_t lut_a[256];
  uint16_t lut_b[256];
};

constexpr size_t kSmem = 1024 + kStages * kStageBytes + sizeof(Tail);

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, Tail* tl) {
  const long long t0 = clock64();
  for (uint32_t i = 0;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if (tl->abort) return false;
    if (clock64() - t0 > (1ll << 31) || i > (1u << 26)) {
      tl->abort = 1u;
      return false;
    }
  }
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// Byte planes of the eight positive fp16 levels C[8..15]: lo/hi bytes of
// levels 0-3 in p[0]/p[2], of levels 4-7 in p[1]/p[3].
struct Planes4 {
  uint32_t lo0, lo1, hi0, hi1;
};

__device__ __forceinline__ Planes4 make_planes4(const uint16_t* lut) {
  Planes4 p{0, 0, 0, 0};
#pragma unroll
  for (int m = 0; m < 8; ++m) {
    const uint32_t v = lut[8 + m];
    const uint32_t lo = v & 0xFFu, hi = v >> 8;
    if (m < 4) {
      p.lo0 |= lo << (8 * m);
      p.hi0 |= hi << (8 * m);
    } else {
      p.lo1 |= lo << (8 * (m - 4));
      p.hi1 |= hi << (8 * (m - 4));
    }
  }
  return p;
}

// Eight 4-bit codes (x, LSB first) -> eight fp16 levels in four words.
__device__ __forceinline__ void expand8_4bit(uint32_t x, const Planes4& P, uint32_t (&w)[4]) {
  const uint32_t neg = (~x >> 3) & 0x11111111u;           // 1 where c < 8
  const uint32_t m = (x ^ (neg * 7u)) & 0x77777777u;      // c<8: 7-c, else c-8
  // 0xFF bytes where an element is negative, elements 0-3 and 4-7
  const uint32_t a7 = neg << 7, a3 = neg << 3;
  const uint32_t s_lo = prmt(a7, a3, 0xD9C8u);
  const uint32_t s_hi = prmt(a7, a3, 0xFBEAu);
  const uint32_t m_hi = m >> 16;
  const uint32_t lo0 = prmt(P.lo0, P.lo1, m);
  const uint32_t hi0 = prmt(P.hi0, P.hi1, m) ^ (s_lo & 0x80808080u);
  const uint32_t lo1 = prmt(P.lo0, P.lo1, m_hi);
  const uint32_t hi1 = prmt(P.hi0, P.hi1, m_hi) ^ (s_hi & 0x80808080u);
  w[0] = prmt(lo0, hi0, 0x5140u);
  w[1] = prmt(lo0, hi0, 0x7362u);
  w[2] = prmt(lo1, hi1, 0x5140u);
  w[3] = prmt(lo1, hi1, 0x7362u);
}

// One row's 64 codes of a K slice -> 8 swizzled 16-byte chunks of fp16.
template <int BITS>
__device__ __forceinline__ void expand_row(const uint32_t (&src)[16], const Planes4& P, const uint16_t* lut,
                                           uint8_t* tile, int r) {
  if constexpr (BITS == 4) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      uint32_t w[4];
      expand8_4bit(src[c], P, w);
      *reinterpret_cast<uint4*>(tile + sw128_offset(r, c)) = make_uint4(w[0], w[1], w[2], w[3]);
    }
  } else {
    constexpr uint32_t mask = (1u << BITS) - 1u;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      uint32_t w[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t pair = 0u;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int i = 8 * c + 2 * j + e;
          const int bit = i * BITS, wi = bit >> 5, sh = bit & 31;
          uint32_t code = src[wi] >> sh;
          if (sh + BITS > 32) code |= src[wi + 1] << (32 - sh);
          pair |= static_cast<uint32_t>(lut[code & mask]) << (16 * e);
        }
        w[j] = pair;
      }
      *reinterpret_cast<uint4*>(tile + sw128_offset(r, c)) = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
}

template <int BITS>
__device__ __forceinline__ void load_row(const uint8_t* row, int kb, bool valid, uint32_t (&dst)[16]) {
  // 64 codes of slice kb = 8*BITS bytes, 8-byte aligned
  const uint2* p = reinterpret_cast<const uint2*>(row + static_cast<size_t>(kb) * 8 * BITS);
#pragma unroll
  for (int i = 0; i < BITS; ++i) {
    const uint2 v = valid ? __ldg(p + i) : make_uint2(0, 0);
    dst[2 * i] = v.x;
    dst[2 * i + 1] = v.y;
  }
#pragma unroll
  for (int i = 2 * BITS; i < 16; ++i) dst[i] = 0u;
}

template <int BITS>
__device__ __forceinline__ void expand_loop(const Params& p, Tail* tl, uint8_t* stages, bool is_a, int r, int ntiles_m,
                            int ntiles, Planes4 P, const uint16_t* lut, const uint8_t* base, long long pitch,
                            int rows_total) {
  const int KT = p.K / kBK;
  uint32_t cnt = 0;
  for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
    const int mt = tile % ntiles_m, nt = tile / ntiles_m;
    const int row = is_a ? mt * kBM + r : nt * kBN + r;
    const bool valid = row < rows_total;
    const uint8_t* src = base + (valid ? row : 0) * pitch;
    uint32_t cur[16], nxt[16];
    load_row<BITS>(src, 0, valid, cur);
    for (int kb = 0; kb < KT; ++kb) {
      if (kb + 1 < KT) load_row<BITS>(src, kb + 1, valid, nxt);
      const uint32_t s = cnt % kStages;
      if (cnt >= kStages && !wait_or_abort(&tl->empty[s], ((cnt / kStages) - 1) & 1, tl)) return;
      uint8_t* tile_ptr = stages + s * kStageBytes + (is_a ? 0 : kATile);
      expand_row<BITS>(cur, P, lut, tile_ptr, r);
      fence_proxy_async_smem();
      mbar_arrive(&tl->full[s]);
      ++cnt;
#pragma unroll
      for (int i = 0; i < 16; ++i) cur[i] = nxt[i];
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1) qlinear_fast_kernel(Params p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* stages = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  Tail* tl = reinterpret_cast<Tail*>(stages + kStages * kStageBytes);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ntiles_m = (p.M + kBM - 1) / kBM, ntiles_n = (p.N + kBN - 1) / kBN;
  const int ntiles = ntiles_m * ntiles_n;
  const int KT = p.K / kBK;

  for (int i = tid; i < 256; i += kThreads) {
    tl->lut_a[i] = (i < (1 << p.bits_a)) ? p.lut_a[i] : 0;
    tl->lut_b[i] = (i < (1 << p.bits_b)) ? p.lut_b[i] : 0;
  }
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&tl->full[s], kExpandThreads);
      mbar_init(&tl->empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tl->acc_full[a], 1);
      mbar_init(&tl->acc_empty[a], 128);
    }
    tl->abort = 0u;
    mbar_fence_init();
  }
  if (warp == 0) {
    tmem_alloc(&tl->tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tl->tmem_slot;

  if (warp == 0) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t kIdesc = idesc_f16(kBM, kBN, false);
      uint32_t cnt = 0, it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++it) {
        const uint32_t a = it & 1u, use = it >> 1;
        if (use >= 1 && !wait_or_abort(&tl->acc_empty[a], (use - 1) & 1, tl)) { ok = false; break; }
        tc_fence_after();
        const uint32_t acc = tmem + a * kBN;
        for (int kb = 0; kb < KT; ++kb) {
          const uint32_t s = cnt % kStages;
          if (!wait_or_abort(&tl->full[s], (cnt / kStages) & 1, tl)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(stages + s * kStageBytes);
          const uint32_t b0 = a0 + kATile;
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k)
            umma_f16(acc, sdesc_k_sw128(a0 + 32 * k), sdesc_k_sw128(b0 + 32 * k), kIdesc, (kb | k) != 0);
          umma_commit(&tl->empty[s]);
          ++cnt;
        }
        if (ok) umma_commit(&tl->acc_full[a]);
      }
      if (!ok) atomicOr(p.err, 2u);
    }
  } else if (warp >= 4 && warp < 8) {
    // ---------------- epilogue ----------------
    const int q = warp & 3;                 // TMEM lane quadrant
    const int r = 32 * q + lane;            // row within the tile
    uint32_t it = 0;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++it) {
      const uint32_t a = it & 1u, use = it >> 1;
      if (!wait_or_abort(&tl->acc_full[a], use & 1, tl)) {
        if (lane == 0) atomicOr(p.err, 4u);
        break;
      }
      tc_fence_after();
      const int mt = tile % ntiles_m, nt = tile / ntiles_m;
      const int m = mt * kBM + r;
      const float rs = (m < p.M) ? p.s[m] * p.inv_k : 0.f;
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
            const __nv_bfloat162 h =
                __floats2bfloat162_rn(__uint_as_float(v[2 * j]) * rs * r0, __uint_as_float(v[2 * j + 1]) * rs * r1);
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
              dst[j] = __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(v[j]) * rs * rv));
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&tl->acc_empty[a]);
    }
  } else if (warp >= 8) {
    // ---------------- operand expansion ----------------
    const int e = tid - kExpandFirst;
    const bool is_a = e < kBM;
    const int r = is_a ? e : e - kBM;
    const int bits = is_a ? p.bits_a : p.bits_b;
    const uint16_t* lut = is_a ? tl->lut_a : tl->lut_b;
    const Planes4 P = make_planes4(lut);
    const uint8_t* base = is_a ? p.A : p.B;
    const long long pitch = static_cast<long long>(p.K) * bits / 8;
    const int rows_total = is_a ? p.M : p.N;
    switch (bits) {
      case 2: expand_loop<2>(p, tl, stages, is_a, r, ntiles_m, ntiles, P, lut, base, pitch, rows_total); break;
      case 3: expand_loop<3>(p, tl, stages, is_a, r, ntiles_m, ntiles, P, lut, base, pitch, rows_total); break;
      case 4: expand_loop<4>(p, tl, stages, is_a, r, ntiles_m, ntiles, P, lut, base, pitch, rows_total); break;
      case 5: expand_loop<5>(p, tl, stages, is_a, r, ntiles_m, ntiles, P, lut, base, pitch, rows_total); break;
      case 6: expand_loop<6>(p, tl, stages, is_a, r, ntiles_m, ntiles, P, lut, base, pitch, rows_total); break;
      case 7: expand_loop<7>(p, tl, stages, is_a, r, ntiles_m, ntiles, P, lut, base, pitch, rows_total); break;
      case 8: expand_loop<8>(p, tl, stages, is_a, r, ntiles_m, ntiles, P, lut, base, pitch, rows_total); break;
      default: expand_loop<1>(p, tl, stages, is_a, r, ntiles_m, ntiles, P, lut, base, pitch, rows_total); break;
    }
    if (tl->abort && e == 0) atomicOr(p.err, 8u);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace qfast

bool qlinear_fast_eligible(int M, int N, int K) {
  return M >= 1 && N >= 1 && (N % 8) == 0 && (K % 64) == 0 && K >= 64;
}

int qlinear_fast_launch(const uint8_t* a_codes, const float* s, int bits_a, const uint8_t* w_codes,
                        const uint16_t* rnorm, int bits_w, int M, int N, int K, uint16_t* Y,
                        const CodebookDevice* ca, const CodebookDevice* cw, unsigned int* err, cudaStream_t st) {
  qfast::Params p{};
  p.A = a_codes;
  p.B = w_codes;
  p.M = M;
  p.N = N;
  p.K = K;
  p.bits_a = bits_a;
  p.bits_b = bits_w;
  p.lut_a = ca->levels_f16;
  p.lut_b = cw->levels_f16;
  p.s = s;
  p.rnorm = rnorm;
  p.inv_k = ca->inv_d;
  p.Y = Y;
  p.err = err;
  auto kern = qfast::qlinear_fast_kernel;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(qfast::kSmem));
  if (e != cudaSuccess) return cuda_fail(e);
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int ntiles = ((M + qfast::kBM - 1) / qfast::kBM) * ((N + qfast::kBN - 1) / qfast::kBN);
  const int grid = ntiles < sms ? ntiles : sms;
  kern<<<grid, qfast::kThreads, qfast::kSmem, st>>>(p);
  e = cudaGetLastError();
  return e == cudaSuccess ? RBQ_OK : cuda_fail(e);
}

}  // namespace rbq
