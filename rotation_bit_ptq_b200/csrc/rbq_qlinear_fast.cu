// qlinear, throughput version: persistent, warp-specialised tcgen05 GEMM on
// packed Lloyd-Max codes.
//
//   OrbitQuant (hotelren.com/news/3376620) §2.2: the rotation absorbed into
//   the weights (§2.1) cancels the online one, so
//   y[m,n] = s_m r'_n sum_k C_w[q_nk] C_a[p_mk].
//
// Code expansion: expand_codes_kernel turns
// packed codes into fp16 levels (x sqrt(K)) in a stream-ordered workspace, an
// HBM-bound pass over rows*K*(b/8 + 2) bytes with warp-contiguous loads and
// stores.  Expanding each weight tile inside the GEMM instead would redo that
// work for every tile of tokens and saturate the SM's integer pipe.
//
// Each call expands the weight codes [N, K]; then one of two routes:
//  * activations whose fp16 copy (M*K*2 bytes) is at most 2 GiB are
//    expanded the same way and the TMA-fed GEMM of rbq_qlinear_int8_fast.cu
//    (on CTA pairs, epilogue s_m r'_n / K) multiplies the two fp16 operands;
//  * larger activations stay packed and are expanded inside the GEMM below
//    (as does the allocation-free entry point), which needs no workspace for
//    them.
//
// 1. expand_codes_kernel: the weight codes (and, first route, the activation
//    codes in the same launch) to fp16 levels.
// 2. qlinear_fast_kernel: each CTA (one per SM) walks a static list of
//    128 x 256 output tiles.
//      warps 0..3  epilogue: TMEM lane quadrant w, one output row per thread;
//                  scale by s_m r'_n / K, round to BF16, store.
//      warp 4      MMA issuer: one thread waits for a filled operand stage,
//                  issues four 128x256x16 kind::f16 MMAs (both operands from
//                  shared memory) into the tile's TMEM accumulator, commits
//                  them to the stage's "empty" barrier, and after the last K
//                  slice commits the accumulator.  Its own instruction latency
//                  sets the pace, so stage indices and phases advance
//                  incrementally and a completed barrier costs one try_wait.
//      warp 5      TMA producer: one thread loads (a) the activation codes of
//                  two K slices for the tile's 128 rows into a ring of code
//                  stages and (b) the 256 x 64 fp16 weight tile of each K
//                  slice straight into the operand stage, 128B-swizzled as the
//                  tensor core reads it.
//      warps 6..13 activation expansion, a thread per row, two warp groups
//                  taking alternate K slices (warps 6..9 the even ones, 10..13
//                  the odd ones), so two slices are in flight in this stage:
//                  read the row's 64 codes of the slice from the code stage,
//                  turn them into fp16 levels before waiting for the stage,
//                  then write them into the stage's swizzled K-major A tile.
//    Two TMEM accumulators (2 x 256 columns) let the epilogue of tile i
//    overlap the MMAs of tile i+1.  (A variant that kept the activation tile
//    in tensor memory, written with tcgen05.st, measured slower: the stores
//    cost more than the shared-memory traffic they save.)

// 4-bit codes are expanded in registers: by symmetry C[15-c] = -C[c], the
// magnitude index m (0..7) selects the two bytes of |C| with byte permutes
// (prmt) from four registers holding the low and high byte planes of the
// eight positive fp16 levels, and the sign lands on the high byte.  Other
// widths read a 2^b-entry fp16 table in shared memory.
//
// Activation code stages: an even width b is loaded one K slice per box (rows
// of 8b bytes; 4- and 8-bit rows use the 32B / 64B TMA swizzle so that the
// expansion threads, one row each, read them without bank conflicts); an odd
// width is loaded two slices per box (rows of 16b bytes, an odd number of
// 16-byte chunks, conflict-free as is).
//
// Every mbarrier wait is bounded; a thread whose wait runs out raises a
// shared abort flag (so the others stop waiting at once), records an error
// in the library's device error word, and the CTA still frees its TMEM.

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <mutex>

#include "rbq_internal.h"
#include "rbq_sm100.cuh"
#include "rbq_qcodes.cuh"

namespace rbq {
namespace qfast {

using namespace sm100;

constexpr int kBM = 128, kBN = 256, kBK = 64;
constexpr int kATile = kBM * kBK * 2;          // 16 KB fp16 activation tile
constexpr int kBTile = kBN * kBK * 2;          // 32 KB fp16 weight tile
constexpr int kOpStage = kATile + kBTile;      // 48 KB per operand stage (shared memory)
constexpr int kAStages = 4;
constexpr int kMaxF = kAStages, kMaxC = 8;     // operand stages, code stages
// Tensor memory: two fp32 accumulators of kBN columns (512 columns).
constexpr int kThreads = 448;                  // 14 warps
constexpr int kMmaWarp = 4, kTmaWarp = 5;
constexpr int kExpandThreads = 2 * kBM;        // two warp groups of a thread per activation row
constexpr size_t kSmemLimit = 227 * 1024;

struct Params {
  int M, N, K;
  int bits_a;
  int F, C;                          // operand stages, code stages
  uint32_t cstage_bytes;             // bytes per code stage (1024-aligned)
  CodeGeo ga;
  const uint16_t* lut_a;             // fp16 levels x sqrt(K), 2^bits entries
  const float* s;
  const uint16_t* rnorm;
  float inv_k;
  uint16_t* Y;
  unsigned int* err;
  int n_fast;                 // tile order: N fastest (the activation operand is the larger)
};

struct __align__(8) Tail {
  uint64_t full[kMaxF];          // weight tile landed (TMA bytes) and activation tile stored (expansion threads)
  uint64_t empty[kMaxF];         // stage consumed (MMA commit)
  uint64_t cfull[kMaxC];
  uint64_t cempty[kMaxC];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t drain;                // abort path only: completion of the MMAs issued
  uint32_t tmem_slot;
  volatile uint32_t abort;
  uint16_t lut_a[256];
};

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, Tail* tl) {
  return mbar_wait_or_abort(bar, parity, &tl->abort);
}

// Byte planes of the positive fp16 levels C[half + m], m < half <= 8 (the
// codebooks are antisymmetric: C[L-1-c] = -C[c], exactly, also in fp16).
struct Planes4 {
  uint32_t lo0, lo1, hi0, hi1;
};

__device__ __forceinline__ Planes4 make_planes_sym(const uint16_t* lut, int half) {
  Planes4 p{0, 0, 0, 0};
#pragma unroll
  for (int m = 0; m < 8; ++m) {
    const uint32_t v = (m < half) ? lut[half + m] : 0u;
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

__device__ __forceinline__ Planes4 make_planes4(const uint16_t* lut) { return make_planes_sym(lut, 8); }

// Eight codes of width B <= 4, one per nibble (x, LSB first) -> eight fp16
// levels in four words: the top bit of a code picks the half, the rest
// (mirrored in the lower half) indexes the positive levels through byte
// permutes, and the sign lands on the high byte.
template <int B>
__device__ __forceinline__ void expand8_sym(uint32_t x, const Planes4& P, uint32_t (&w)[4]) {
  constexpr uint32_t kMag = (1u << (B - 1)) - 1u;
  const uint32_t neg = (~x >> (B - 1)) & 0x11111111u;     // 1 where c < half
  const uint32_t m = (x ^ (neg * kMag)) & (0x11111111u * kMag);   // c<half: half-1-c, else c-half
  const uint32_t a7 = neg << 7, a3 = neg << 3;            // 0xFF bytes where negative
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
__device__ __forceinline__ void expand8_4bit(uint32_t x, const Planes4& P, uint32_t (&w)[4]) {
  expand8_sym<4>(x, P, w);
}

// Half HF (codes 32 HF .. 32 HF + 31) of one row's 64 codes of a K slice ->
// 16 words of fp16 pairs (k even in the low half), 16 of the row's operand
// columns in tensor memory.
template <int BITS, int HF>
__device__ __forceinline__ void expand_row(const uint32_t (&src)[slice_words<BITS>()], const Planes4& P,
                                           const uint16_t* lut, uint32_t (&out)[16]) {
  if constexpr (BITS == 4) {
#pragma unroll
    for (int c = 4 * HF; c < 4 * HF + 4; ++c) {
      uint32_t w[4];
      expand8_4bit(src[c], P, w);
#pragma unroll
      for (int j = 0; j < 4; ++j) out[4 * (c - 4 * HF) + j] = w[j];
    }
  } else if constexpr (BITS == 2 || BITS == 3) {
#pragma unroll
    for (int c = 4 * HF; c < 4 * HF + 4; ++c) {
      uint32_t w[4];
      expand8_sym<BITS>(spread8<BITS>(src, c), P, w);
#pragma unroll
      for (int j = 0; j < 4; ++j) out[4 * (c - 4 * HF) + j] = w[j];
    }
  } else {
    constexpr uint32_t mask = (1u << BITS) - 1u;
#pragma unroll
    for (int c = 4 * HF; c < 4 * HF + 4; ++c) {
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
#pragma unroll
      for (int j = 0; j < 4; ++j) out[4 * (c - 4 * HF) + j] = w[j];
    }
  }
}

// Waits on a barrier for the whole warp: every lane returns the same answer,
// so a warp leaves its loop together (the epilogue's warp-collective
// tensor-memory loads rely on this).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, Tail* tl) {
  return mbar_warp_wait(bar, parity, &tl->abort);
}

// Row r = 32 (warp % 4) + lane of every activation tile, whole rows of the K
// slices of parity G (2 kp + G): the two warp groups expand alternate slices,
// so two slices are in flight in the expansion stage.
template <int BITS, int G>
__device__ __forceinline__ void expand_loop(const Params& p, Tail* tl, uint8_t* ops, uint8_t* codes, int r,
                                            int ntiles, Planes4 P, const uint16_t* lut) {
  const CodeGeo& g = p.ga;
  const int KP = p.K / (2 * kBK);
  const uint32_t C = static_cast<uint32_t>(p.C);
  uint32_t c = 0, cph = 0, s = G, aph = 0;       // code stage / A stage and their phases
  bool a_first = true;                           // first round of A stages: nothing to wait for
  for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
    for (int kp = 0; kp < KP; ++kp) {
      if (!warp_wait(&tl->cfull[c], cph, tl)) return;
      const uint8_t* part = codes + c * p.cstage_bytes + g.offset;
      uint32_t cur[slice_words<BITS>()];
      read_slice<BITS>(part, g, r, G, cur);
      uint32_t w0[16], w1[16];
      expand_row<BITS, 0>(cur, P, lut, w0);          // before the wait: off the critical path
      expand_row<BITS, 1>(cur, P, lut, w1);
      mbar_arrive(&tl->cempty[c]);                     // the codes are in registers now
      if (++c == C) { c = 0; cph ^= 1u; }
      if (!a_first && !warp_wait(&tl->empty[s], aph ^ 1u, tl)) return;
      uint8_t* tile = ops + s * kOpStage;              // the stage's A tile, 128B-swizzled K-major
#pragma unroll
      for (int q = 0; q < 4; ++q)
        *reinterpret_cast<uint4*>(tile + sw128_offset(r, q)) =
            make_uint4(w0[4 * q], w0[4 * q + 1], w0[4 * q + 2], w0[4 * q + 3]);
#pragma unroll
      for (int q = 0; q < 4; ++q)
        *reinterpret_cast<uint4*>(tile + sw128_offset(r, 4 + q)) =
            make_uint4(w1[4 * q], w1[4 * q + 1], w1[4 * q + 2], w1[4 * q + 3]);
      fence_proxy_async_smem();                        // visible to the tensor core
      mbar_arrive(&tl->full[s]);
      s += 2;                                          // this group's next slice
      if (s >= kAStages) { s -= kAStages; aph ^= 1u; a_first = false; }
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    qlinear_fast_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const Params p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* ops = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* codes = ops + p.F * kOpStage;
  Tail* tl = reinterpret_cast<Tail*>(codes + p.C * p.cstage_bytes);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ntiles_m = (p.M + kBM - 1) / kBM, ntiles_n = (p.N + kBN - 1) / kBN;
  const int ntiles = ntiles_m * ntiles_n;
  const int KT = p.K / kBK;
  const int KP = KT / 2;

  for (int i = tid; i < 256; i += kThreads) tl->lut_a[i] = (i < (1 << p.bits_a)) ? p.lut_a[i] : 0;
  if (tid == 0) {
    for (int s = 0; s < kMaxF; ++s) {
      mbar_init(&tl->full[s], kBM + 1);   // one warp group (a thread per row) + the producer's expect-tx arrival
      mbar_init(&tl->empty[s], 1);
    }
    for (int c = 0; c < p.C; ++c) {
      mbar_init(&tl->cfull[c], 1);
      mbar_init(&tl->cempty[c], kExpandThreads);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tl->acc_full[a], 1);
      mbar_init(&tl->acc_empty[a], 128);
    }
    mbar_init(&tl->drain, 1);
    tl->abort = 0u;
    mbar_fence_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&tl->tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tl->tmem_slot;
  // The prologue above reads only constant tables; the operands (written by
  // the kernels before this one on the stream) wait for them.
  griddep_wait();
  griddep_launch_dependents();

  if (warp == kMmaWarp) {
    // ---------------- MMA issuer ----------------
    // One thread feeds the tensor core, so its own instruction latency sets
    // the pace: stage indices and phases advance incrementally, a barrier
    // that is already complete costs one try_wait, and the operand
    // descriptors step by constants.
    if (lane == 0) {
      constexpr uint32_t kIdesc = idesc_f16(kBM, kBN, false);
      const uint64_t bdesc0 = sdesc_k_sw128(smem_u32(ops));
      constexpr uint32_t F = kMaxF;
      uint32_t s = 0, ph = 0, it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++it) {
        const uint32_t a = it & 1u, use = it >> 1;
        if (use >= 1 && !wait_or_abort(&tl->acc_empty[a], (use - 1) & 1, tl)) { ok = false; break; }
        tc_fence_after();
        const uint32_t acc = tmem + a * kBN;
        for (int kb = 0; kb < KT; ++kb) {
          if (!mbar_try_wait(&tl->full[s], ph) && !wait_or_abort(&tl->full[s], ph, tl)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t a0 = bdesc0 + ((s * static_cast<uint32_t>(kOpStage)) >> 4);   // A, then B
          const uint64_t b0 = a0 + (kATile >> 4);
          umma_f16(acc, a0, b0, kIdesc, kb != 0);
          umma_f16(acc, a0 + 2, b0 + 2, kIdesc, 1u);                      // +32 bytes of K per step
          umma_f16(acc, a0 + 4, b0 + 4, kIdesc, 1u);
          umma_f16(acc, a0 + 6, b0 + 6, kIdesc, 1u);
          umma_commit(&tl->empty[s]);
          if (++s == F) { s = 0; ph ^= 1u; }
        }
        if (ok) umma_commit(&tl->acc_full[a]);
      }
      if (!ok) atomicOr(p.err, 2u);
    }
  } else if (warp == kTmaWarp) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB);
      const uint32_t C = static_cast<uint32_t>(p.C), F = static_cast<uint32_t>(p.F);
      uint32_t c = 0, cph = 0, s = 0, ph = 0;     // code / weight stage and their phases
      bool c_first = true, b_first = true;
      bool ok = true;
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
        const int mt = p.n_fast ? tile / ntiles_n : tile % ntiles_m;
        const int nt = p.n_fast ? tile % ntiles_n : tile / ntiles_m;
        for (int kp = 0; kp < KP && ok; ++kp) {
          if (!c_first && !wait_or_abort(&tl->cempty[c], cph ^ 1u, tl)) {
            ok = false;
            break;
          }
          uint8_t* stage = codes + c * p.cstage_bytes;
          mbar_arrive_expect_tx(&tl->cfull[c], p.ga.bytes);
          if (p.ga.slice_bytes) {
            tma_load_2d(stage + p.ga.offset, &tmA, (2 * kp) * 8 * p.ga.bits, mt * kBM, &tl->cfull[c]);
            tma_load_2d(stage + p.ga.offset + p.ga.slice_bytes, &tmA, (2 * kp + 1) * 8 * p.ga.bits, mt * kBM,
                        &tl->cfull[c]);
          } else {
            tma_load_2d(stage + p.ga.offset, &tmA, kp * 16 * p.ga.bits, mt * kBM, &tl->cfull[c]);
          }
          if (++c == C) { c = 0; cph ^= 1u; c_first = false; }
#pragma unroll 1
          for (int h = 0; h < 2; ++h) {
            if (!b_first && !wait_or_abort(&tl->empty[s], ph ^ 1u, tl)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&tl->full[s], kBTile);
            tma_load_2d(ops + s * kOpStage + kATile, &tmB, (2 * kp + h) * kBK, nt * kBN, &tl->full[s]);
            if (++s == F) { s = 0; ph ^= 1u; b_first = false; }
          }
        }
      }
      if (!ok) atomicOr(p.err, 16u);
    }
  } else if (warp < 4) {
    // ---------------- epilogue ----------------
    const int q = warp;                     // TMEM lane quadrant
    const int r = 32 * q + lane;            // row within the tile
    uint32_t it = 0;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++it) {
      const uint32_t a = it & 1u, use = it >> 1;
      if (!warp_wait(&tl->acc_full[a], use & 1, tl)) {   // warp-uniform: tmem loads follow
        if (lane == 0) atomicOr(p.err, 4u);
        break;
      }
      tc_fence_after();
      const int mt = p.n_fast ? tile / ntiles_n : tile % ntiles_m;
      const int nt = p.n_fast ? tile % ntiles_n : tile / ntiles_m;
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
  } else {
    // ---------------- activation expansion ----------------
    // warps 6..13: lane quarter warp % 4, slice parity (warp - 6) / 4
    const int r = 32 * (warp & 3) + lane;
    const uint16_t* lut = tl->lut_a;
    const Planes4 P = make_planes_sym(lut, p.bits_a <= 4 ? (1 << (p.bits_a - 1)) : 8);
    if (warp < 10) {
      switch (p.bits_a) {
        case 1: expand_loop<1, 0>(p, tl, ops, codes, r, ntiles, P, lut); break;
        case 2: expand_loop<2, 0>(p, tl, ops, codes, r, ntiles, P, lut); break;
        case 3: expand_loop<3, 0>(p, tl, ops, codes, r, ntiles, P, lut); break;
        case 4: expand_loop<4, 0>(p, tl, ops, codes, r, ntiles, P, lut); break;
        case 5: expand_loop<5, 0>(p, tl, ops, codes, r, ntiles, P, lut); break;
        case 6: expand_loop<6, 0>(p, tl, ops, codes, r, ntiles, P, lut); break;
        case 7: expand_loop<7, 0>(p, tl, ops, codes, r, ntiles, P, lut); break;
        default: expand_loop<8, 0>(p, tl, ops, codes, r, ntiles, P, lut); break;
      }
    } else {
      switch (p.bits_a) {
        case 1: expand_loop<1, 1>(p, tl, ops, codes, r, ntiles, P, lut); break;
        case 2: expand_loop<2, 1>(p, tl, ops, codes, r, ntiles, P, lut); break;
        case 3: expand_loop<3, 1>(p, tl, ops, codes, r, ntiles, P, lut); break;
        case 4: expand_loop<4, 1>(p, tl, ops, codes, r, ntiles, P, lut); break;
        case 5: expand_loop<5, 1>(p, tl, ops, codes, r, ntiles, P, lut); break;
        case 6: expand_loop<6, 1>(p, tl, ops, codes, r, ntiles, P, lut); break;
        case 7: expand_loop<7, 1>(p, tl, ops, codes, r, ntiles, P, lut); break;
        default: expand_loop<8, 1>(p, tl, ops, codes, r, ntiles, P, lut); break;
      }
    }
    if (tl->abort && r == 0 && warp < 10) atomicOr(p.err, 8u);
  }

  tc_fence_before();
  __syncthreads();
  if (tl->abort) {                 // the same value in every thread after the barrier
    drain_after_abort(warp == kMmaWarp && lane == 0, &tl->drain);
    __syncthreads();
  }
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---- host side ------------------------------------------------------------

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// Geometry of one operand's share of a code stage, starting at `offset`.
CodeGeo make_geo(uint32_t rows, uint32_t bits, uint32_t offset) {
  CodeGeo g{};
  g.rows = rows;
  g.bits = bits;
  g.offset = offset;
  if ((bits & 1) == 0) {
    const uint32_t sb = rows * 8 * bits;
    g.slice_bytes = (sb + 1023u) & ~1023u;   // each slice buffer swizzle-aligned
    g.bytes = 2 * sb;                        // bytes landing per stage
    g.swz = bits == 4 ? 1 : bits == 8 ? 2 : 0;
  } else {
    g.slice_bytes = 0;
    g.bytes = rows * 16 * bits;
    g.swz = 0;
  }
  return g;
}

uint32_t geo_span(const CodeGeo& g) {
  return g.slice_bytes ? 2 * g.slice_bytes : ((g.bytes + 1023u) & ~1023u);
}

int encode_codes_map(CUtensorMap* map, const uint8_t* base, int rows, int bits, int K, const CodeGeo& g) {
  auto fn = encode_fn();
  if (!fn) return RBQ_ECUDA;
  const cuuint64_t row_bytes = static_cast<cuuint64_t>(K) * bits / 8;
  const cuuint64_t dims[2] = {row_bytes, static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {g.slice_bytes ? 8u * bits : 16u * bits, g.rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUtensorMapSwizzle swz = g.swz == 1 ? CU_TENSOR_MAP_SWIZZLE_32B
                                 : g.swz == 2 ? CU_TENSOR_MAP_SWIZZLE_64B
                                              : CU_TENSOR_MAP_SWIZZLE_NONE;
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? RBQ_OK : RBQ_ECUDA;
}

// fp16 [rows, K] K-major, 256 x 64 tiles, 128B swizzle: the canonical K-major
// operand layout of the tensor core.
int encode_f16_map(CUtensorMap* map, const uint16_t* base, int rows, int K) {
  auto fn = encode_fn();
  if (!fn) return RBQ_ECUDA;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kBK), static_cast<cuuint32_t>(kBN)};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<uint16_t*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? RBQ_OK : RBQ_ECUDA;
}

// ---- code expansion ------------------------------------------------------
// One job: `groups` groups of 8 codes (BITS bytes each; the packed rows are
// contiguous and every row holds K/8 whole groups) -> 16 bytes of fp16
// levels each.  One launch runs one or two jobs (a call's weights and
// activations), each on its own range of blocks; every body is a grid-stride
// loop over its job's blocks in which each warp's loads and stores cover
// contiguous memory.
struct ExpandJob {
  const uint8_t* codes;
  long long groups;
  const uint16_t* lut;      // 2^bits fp16 levels
  uint4* out;
  int bits;
  int blocks;               // blocks of the launch that run this job
};

// 4-bit codes: a group is one 32-bit word.  A warp expands 128 words (512
// bytes in, 2 KB out) per step; lane l takes words l, l+32, l+64 and l+96 of
// the warp's range, so every load and store instruction of the warp is
// contiguous (128 and 512 bytes), not 16-byte pieces 64 bytes apart.
__device__ __forceinline__ void expand_job4(const ExpandJob& j, int jb) {
  Planes4 P;
  {
    uint16_t lut[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) lut[i] = __ldg(j.lut + i);
    P = make_planes4(lut);
  }
  const uint32_t* codes = reinterpret_cast<const uint32_t*>(j.codes);
  const int lane = threadIdx.x & 31;
  const long long warps = static_cast<long long>(j.blocks) * (blockDim.x >> 5);
  for (long long base = (jb * static_cast<long long>(blockDim.x >> 5) + (threadIdx.x >> 5)) * 128;
       base < j.groups; base += 128 * warps) {
    uint32_t x[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const long long g = base + 32 * q + lane;
      x[q] = g < j.groups ? __ldcs(codes + g) : 0u;
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const long long g = base + 32 * q + lane;
      if (g < j.groups) {
        uint32_t w[4];
        expand8_4bit(x[q], P, w);
        __stcg(j.out + g, make_uint4(w[0], w[1], w[2], w[3]));
      }
    }
  }
}

// Widths that divide 8 bits (1, 2, 8): one thread per group, the group read
// as one 16-, 8- or 64-bit word, its 8 levels from the shared table.
template <int BITS>
__device__ __forceinline__ void expand_job_div8(const ExpandJob& j, const uint16_t* lut, int jb) {
  for (long long g = jb * static_cast<long long>(blockDim.x) + threadIdx.x; g < j.groups;
       g += static_cast<long long>(j.blocks) * blockDim.x) {
    uint64_t x;
    if constexpr (BITS == 8) x = __ldcs(reinterpret_cast<const unsigned long long*>(j.codes) + g);
    else if constexpr (BITS == 2) x = __ldcs(reinterpret_cast<const unsigned short*>(j.codes) + g);
    else x = j.codes[g];
    constexpr uint32_t mask = (1u << BITS) - 1u;
    uint32_t w[4];
#pragma unroll
    for (int q = 0; q < 4; ++q)
      w[q] = static_cast<uint32_t>(lut[(x >> (2 * q * BITS)) & mask]) |
             (static_cast<uint32_t>(lut[(x >> ((2 * q + 1) * BITS)) & mask]) << 16);
    __stcg(j.out + g, make_uint4(w[0], w[1], w[2], w[3]));
  }
}

// Widths that do not divide 8 bits (3, 5, 6, 7): one thread per group.  A
// warp's 32 groups are 32*BITS contiguous bytes, loaded as words by the warp
// into its shared buffer `wb` (so the loads are contiguous too) and read back
// by each lane as the 64-bit window that holds its group.
template <int BITS>
__device__ __forceinline__ void expand_job_groups(const ExpandJob& j, const uint16_t* lut, uint32_t* wb, int jb) {
  constexpr int kWords = 8 * BITS;                     // words of a warp's 32 groups
  const uint32_t* codes = reinterpret_cast<const uint32_t*>(j.codes);
  const int lane = threadIdx.x & 31;
  const long long total_words = j.groups * BITS / 4;   // groups % 16 == 0 (K % 128 == 0)
  const long long warps = static_cast<long long>(j.blocks) * (blockDim.x >> 5);
  for (long long g0 = (jb * static_cast<long long>(blockDim.x >> 5) + (threadIdx.x >> 5)) * 32; g0 < j.groups;
       g0 += 32 * warps) {
    const long long w0 = g0 * BITS / 4;                // g0 % 32 == 0: a whole word
    __syncwarp();
#pragma unroll
    for (int q = 0; q < (kWords + 31) / 32; ++q) {
      const int i = 32 * q + lane;
      if (i < kWords) wb[i] = (w0 + i < total_words) ? __ldcs(codes + w0 + i) : 0u;
    }
    __syncwarp();
    const long long g = g0 + lane;
    if (g < j.groups) {
      // bytes [lane*BITS, lane*BITS + BITS) of the buffer; word wi + 2 only
      // feeds bits above the group's 8*BITS (the buffer has 2 spare words)
      const int byte = lane * BITS, wi = byte >> 2, sh = 8 * (byte & 3);
      const uint64_t lo = (static_cast<uint64_t>(wb[wi + 1]) << 32) | wb[wi];
      const uint64_t v = sh ? (lo >> sh) | (static_cast<uint64_t>(wb[wi + 2]) << (64 - sh)) : lo;
      constexpr uint32_t mask = (1u << BITS) - 1u;
      uint32_t o[4];
#pragma unroll
      for (int q = 0; q < 4; ++q)
        o[q] = static_cast<uint32_t>(lut[(v >> (2 * q * BITS)) & mask]) |
               (static_cast<uint32_t>(lut[(v >> ((2 * q + 1) * BITS)) & mask]) << 16);
      __stcg(j.out + g, make_uint4(o[0], o[1], o[2], o[3]));
    }
  }
}

// Blocks [0, j0.blocks) run job 0, the rest job 1 (j1.blocks may be 0).
__global__ void __launch_bounds__(256) expand_codes_kernel(const ExpandJob j0, const ExpandJob j1) {
  griddep_wait();
  griddep_launch_dependents();
  __shared__ uint16_t lut[256];
  __shared__ uint32_t buf[8][64 + 2];                  // per warp (expand_job_groups)
  const bool second = static_cast<int>(blockIdx.x) >= j0.blocks;
  const ExpandJob j = second ? j1 : j0;
  const int jb = second ? static_cast<int>(blockIdx.x) - j0.blocks : static_cast<int>(blockIdx.x);
  if (j.bits == 4) {                                   // block-uniform
    expand_job4(j, jb);
    return;
  }
  for (int i = threadIdx.x; i < 256; i += blockDim.x) lut[i] = (i < (1 << j.bits)) ? j.lut[i] : 0;
  __syncthreads();
  uint32_t* wb = buf[threadIdx.x >> 5];
  switch (j.bits) {
    case 1: expand_job_div8<1>(j, lut, jb); break;
    case 2: expand_job_div8<2>(j, lut, jb); break;
    case 3: expand_job_groups<3>(j, lut, wb, jb); break;
    case 5: expand_job_groups<5>(j, lut, wb, jb); break;
    case 6: expand_job_groups<6>(j, lut, wb, jb); break;
    case 7: expand_job_groups<7>(j, lut, wb, jb); break;
    default: expand_job_div8<8>(j, lut, jb); break;
  }
}

// ---- host side ------------------------------------------------------------

// The job that expands `rows` rows of K codes of `bits` bits (K % 128 == 0).
ExpandJob expand_job(const uint8_t* codes, int bits, int rows, int K, const uint16_t* lut, uint16_t* out, int sms) {
  ExpandJob j{};
  j.codes = codes;
  j.groups = static_cast<long long>(rows) * (K / 8);
  j.lut = lut;
  j.out = reinterpret_cast<uint4*>(out);
  j.bits = bits;
  // 4-bit: 8 warps x 128 groups per block step; other widths 256 groups
  long long blocks = bits == 4 ? (j.groups + 1023) / 1024 : (j.groups + 255) / 256;
  if (blocks > 16LL * sms) blocks = 16LL * sms;
  j.blocks = static_cast<int>(blocks);
  return j;
}

// Launch with programmatic dependent launch allowed: the kernel waits
// (griddep_wait) for the launch before it before touching memory, so only its
// launch latency overlaps that launch's tail, and the GEMM after it waits for
// it the same way.
int launch_expand(const ExpandJob& j0, const ExpandJob& j1, cudaStream_t st) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(j0.blocks + j1.blocks), 1, 1);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, expand_codes_kernel, j0, j1);
  if (e == cudaSuccess) e = cudaGetLastError();
  return e == cudaSuccess ? RBQ_OK : cuda_fail(e);
}

int expand_weights(const uint8_t* codes, int bits, int rows, int K, const uint16_t* lut, uint16_t* out,
                   cudaStream_t st, int sms) {
  ExpandJob none{};
  return launch_expand(expand_job(codes, bits, rows, K, lut, out, sms), none, st);
}

// Weights and activations of one call in one launch.
int expand_both(const uint8_t* w_codes, int bits_w, int N, const uint16_t* lut_w, uint16_t* wf16,
                const uint8_t* a_codes, int bits_a, int M, const uint16_t* lut_a, uint16_t* af16, int K,
                cudaStream_t st, int sms) {
  return launch_expand(expand_job(w_codes, bits_w, N, K, lut_w, wf16, sms),
                       expand_job(a_codes, bits_a, M, K, lut_a, af16, sms), st);
}

// A memory pool per device for the stream-ordered weight workspace; it keeps
// freed blocks cached so repeated calls do not go back to the driver.
cudaMemPool_t workspace_pool(int dev) {
  static cudaMemPool_t pools[kMaxDevices] = {};
  static std::mutex mu;
  if (dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(mu);
  if (!pools[dev]) {
    cudaMemPoolProps props{};
    props.allocType = cudaMemAllocationTypePinned;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    cudaMemPool_t pool = nullptr;
    if (cudaMemPoolCreate(&pool, &props) != cudaSuccess) return nullptr;
    uint64_t keep = ~0ull;
    cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
    pools[dev] = pool;
  }
  return pools[dev];
}

}  // namespace qfast

bool qlinear_fast_eligible(int M, int N, int K, int bits_a, int bits_w) {
  (void)bits_w;
  if (M < 1 || N < 1 || (N % 8) != 0 || K < 128 || (K % 128) != 0) return false;
  // TMA needs 16-byte row strides for the activation codes
  return (static_cast<long long>(K) * bits_a / 8) % 16 == 0;
}

// The GEMM on already-expanded fp16 weights `wf16` [N, K].
int qlinear_fast_gemm(const uint8_t* a_codes, const float* s, int bits_a, const uint16_t* wf16,
                      const uint16_t* rnorm, int M, int N, int K, uint16_t* Y, const CodebookDevice* ca,
                      unsigned int* err, cudaStream_t st, int sms) {
  using namespace qfast;
  Params p{};
  p.M = M;
  p.N = N;
  p.K = K;
  p.bits_a = bits_a;
  p.ga = make_geo(kBM, bits_a, 0);
  p.cstage_bytes = geo_span(p.ga);
  const size_t tail = sizeof(Tail) + 64;
  // The operand ring is fixed at kMaxF stages (their A halves fill the rest of
  // tensor memory); the code ring takes what shared memory is left.
  const int F = kMaxF;
  int C = 2;
  while (C < kMaxC && 1024 + F * kOpStage + (C + 1) * p.cstage_bytes + tail <= kSmemLimit) ++C;
  const size_t smem = 1024 + static_cast<size_t>(F) * kOpStage + static_cast<size_t>(C) * p.cstage_bytes + tail;
  if (smem > kSmemLimit) return RBQ_EINVAL;
  p.F = F;
  p.C = C;
  p.lut_a = ca->levels_f16;
  p.s = s;
  p.rnorm = rnorm;
  p.inv_k = ca->inv_d;
  p.Y = Y;
  p.err = err;
  // walk N fastest when the activation codes outweigh the fp16 weights and
  // would not stay in L2 between waves of CTAs (more than half of its 126 MB)
  const long long a_bytes = static_cast<long long>(M) * K * bits_a / 8;
  p.n_fast = a_bytes > 2LL * N * K && a_bytes > (64LL << 20);
  CUtensorMap mA, mB;
  int rc = encode_codes_map(&mA, a_codes, M, bits_a, K, p.ga);
  if (rc != RBQ_OK) return rc;
  if ((rc = encode_f16_map(&mB, wf16, N, K)) != RBQ_OK) return rc;
  auto kern = qlinear_fast_kernel;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return cuda_fail(e);
  const int ntiles = ((M + kBM - 1) / kBM) * ((N + kBN - 1) / kBN);
  const int grid = ntiles < sms ? ntiles : sms;
  // programmatic dependent launch: the prologue overlaps the weight expansion's tail
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, mA, mB, p);
  if (e == cudaSuccess) e = cudaGetLastError();
  return e == cudaSuccess ? RBQ_OK : cuda_fail(e);
}

// The TMA-fed GEMM on operands expanded beforehand (rbq_qlinear_int8_fast.cu).
int qlinear_f16_operands_gemm(const uint16_t* af16, const float* s, const uint16_t* wf16, const uint16_t* rnorm,
                              float inv_k, int M, int N, int K, uint16_t* Y, unsigned int* err, cudaStream_t st,
                              int sms, const float* next_sign = nullptr, int act = 0);

int qlinear_fast_launch(const uint8_t* a_codes, const float* s, int bits_a, const uint8_t* w_codes,
                        const uint16_t* rnorm, int bits_w, int M, int N, int K, uint16_t* Y,
                        const CodebookDevice* ca, const CodebookDevice* cw, unsigned int* err, cudaStream_t st) {
  int dev = 0, sms = 148;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaMemPool_t pool = qfast::workspace_pool(dev);
  if (!pool) return RBQ_ECUDA;
  // The activation codes get their own pass into fp16 and the GEMM streams
  // both operands by TMA on CTA pairs -- faster than expanding them inside the
  // GEMM at every measured size (587 MB of fp16 activations included) -- while
  // that copy (M*K*2 bytes) is at most 2 GiB of workspace; beyond it the
  // activations are expanded inside the GEMM (qlinear_fast_kernel).
  const size_t a_f16_bytes = static_cast<size_t>(M) * K * 2;
  const bool split = a_f16_bytes <= (static_cast<size_t>(2048) << 20);
  void* ws = nullptr;
  e = cudaMallocFromPoolAsync(&ws, static_cast<size_t>(N) * K * 2 + (split ? a_f16_bytes : 0), pool, st);
  if (e != cudaSuccess) return cuda_fail(e);
  uint16_t* wf16 = static_cast<uint16_t*>(ws);
  int rc = RBQ_OK;
  if (split) {
    uint16_t* af16 = wf16 + static_cast<size_t>(N) * K;
    rc = qfast::expand_both(w_codes, bits_w, N, cw->levels_f16, wf16, a_codes, bits_a, M, ca->levels_f16, af16, K,
                            st, sms);
    if (rc == RBQ_OK) rc = qlinear_f16_operands_gemm(af16, s, wf16, rnorm, ca->inv_d, M, N, K, Y, err, st, sms);
  } else {
    rc = qfast::expand_weights(w_codes, bits_w, N, K, cw->levels_f16, wf16, st, sms);
    if (rc == RBQ_OK) rc = qlinear_fast_gemm(a_codes, s, bits_a, wf16, rnorm, M, N, K, Y, ca, err, st, sms);
  }
  e = cudaFreeAsync(ws, st);
  if (rc == RBQ_OK && e != cudaSuccess) rc = cuda_fail(e);
  return rc;
}

// qlinear whose epilogue finishes the next layer's rotation (next_sign: its D
// in output order; the weight rows and r' in its permutation's order): always
// the expanded-operand route, whatever the activations' size.
int qlinear_rotate_next_launch(const uint8_t* a_codes, const float* s, int bits_a, const uint8_t* w_codes,
                               const uint16_t* rnorm, int bits_w, int M, int N, int K, uint16_t* Y,
                               const CodebookDevice* ca, const CodebookDevice* cw, unsigned int* err,
                               cudaStream_t st, const float* next_sign, int act) {
  int dev = 0, sms = 148;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaMemPool_t pool = qfast::workspace_pool(dev);
  if (!pool) return RBQ_ECUDA;
  void* ws = nullptr;
  e = cudaMallocFromPoolAsync(&ws, (static_cast<size_t>(N) + M) * K * 2, pool, st);
  if (e != cudaSuccess) return cuda_fail(e);
  uint16_t* wf16 = static_cast<uint16_t*>(ws);
  uint16_t* af16 = wf16 + static_cast<size_t>(N) * K;
  int rc = qfast::expand_both(w_codes, bits_w, N, cw->levels_f16, wf16, a_codes, bits_a, M, ca->levels_f16, af16, K,
                              st, sms);
  if (rc == RBQ_OK)
    rc = qlinear_f16_operands_gemm(af16, s, wf16, rnorm, ca->inv_d, M, N, K, Y, err, st, sms, next_sign, act);
  e = cudaFreeAsync(ws, st);
  if (rc == RBQ_OK && e != cudaSuccess) rc = cuda_fail(e);
  return rc;
}

}  // namespace rbq
