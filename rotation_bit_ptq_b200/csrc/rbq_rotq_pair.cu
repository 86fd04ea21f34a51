// Rotate-then-quantise for BF16 rows of width 1024..16384 (d a multiple of
// 256): the token-pair kernel.
//
//   OrbitQuant (hotelren.com/news/3376620) §2.2 / §2.1: x' = Pi_d x, s = ||x'||,
//   codes of x'/(s + eps) in the Lloyd-Max codebook of N(0, 1/d); weights the
//   same with BF16 row norms.  INT8-convrot (cloud.baidu.com/article/9430339)
//   §4: rotate, scale = max|w'|/127, round.  Rotate-only: x' in BF16.
//   Pi_d = blkdiag(H_64 D_1, ..., H_64 D_{d/64}) · P_pi (OrbitQuant §2.3).
//
// Work unit: a tile of R = 2P token rows, P = 8 pairs for d <= 3072 and 4, 2
// or 1 for wider rows (whatever keeps two ring slots in shared memory).
// Thread (p, b) owns output block b of the token pair (p, p+P), p < P,
// holding the pair's values as packed fp32x2 registers, so every butterfly
// stage is one packed add/sub per pair.
// It gathers and transforms one 32-position half-block at a time (strides
// 1..16), parks both halves in its own lane of tensor memory, and runs the
// last stage (stride 32) inside the encoding loop as it reads them back; the
// smaller live register set leaves room for many loads in flight.  A warp
// covers P pairs x 32/P blocks; the P lanes that share a block read the same
// source position of P different rows, which a 16-byte row padding puts in P
// different banks.  Threads whose block is past d/64 (when 32/P does not
// divide the block count) only join the warp's collective steps.
//
// Data movement: whole rows arrive by bulk asynchronous copies (TMA, no
// tensor map needed for contiguous rows), one row per lane of an issuing
// warp, into a ring of tile slots, each completion counted on the slot's
// mbarrier.  The gather table and the code grid are copied first, so they are
// not queued behind the tiles.  The last warp done gathering from a slot
// refills it with a later tile, so the next tiles stream in while the current
// one is transformed and encoded.
//
// Norm: the rotation is orthogonal, so ||Pi x|| = ||x||; every thread sums the
// squares of the 64 inputs it gathered (each input lands in exactly one
// block), the partial sums meet in shared memory, and the wait for them is
// split from the arrival so the butterfly overlaps it.  (INT8 needs max|w'|,
// which exists only after the butterfly, so there the arrival follows it.)
//
// Codes: z (8x the rotated value, H unnormalised) -> v = z / (||z|| + 8 eps).
// A small uniform grid over [-R, R], v clamped into it, gives a cell n whose
// entry holds the count of boundaries below the cell and the boundary inside
// it (or +inf): code = base + (v >= thr) (see rowtile::Enc).

#include <cuda_bf16.h>

#include "rbq_internal.h"
#include "rbq_sm100.cuh"
#include "rbq_rowtile.cuh"

namespace rbq {
namespace pairk {

using namespace sm100;
using namespace rowtile;

// Codes of one block for both tokens: the last butterfly stage (stride 32)
// runs here, on half-blocks read back from tensor memory 16 positions at a
// time.  SAN: the token(s) flagged bad are encoded as the zero vector.
template <int BITS, bool SAN>
__device__ __forceinline__ void encode_block(const Enc& enc, uint32_t tA, uint32_t tB, bool bad0, bool bad1,
                                             uint32_t* w0, uint32_t* w1) {
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    uint32_t va[32], vb[32];
    __syncwarp();
    tmem_ld32(tA + 32u * c, va);
    tmem_ld32(tB + 32u * c, vb);
    tmem_wait_ld();
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const unsigned long long a = pk_u(va[2 * k], va[2 * k + 1]), bb = pk_u(vb[2 * k], vb[2 * k + 1]);
      unsigned long long z = add2(a, bb), y = sub2(a, bb);
      if constexpr (SAN) {
        float z0, z1, y0, y1;
        upk(z, z0, z1);
        upk(y, y0, y1);
        z = pk(bad0 ? 0.f : z0, bad1 ? 0.f : z1);
        y = pk(bad0 ? 0.f : y0, bad1 ? 0.f : y1);
      }
      uint32_t c0, c1, d0, d1;
      enc.codes(z, c0, c1);
      enc.codes(y, d0, d1);
      const int i = 16 * c + k;
      put_code<BITS>(w0, i, c0);
      put_code<BITS>(w1, i, c1);
      put_code<BITS>(w0, i + 32, d0);
      put_code<BITS>(w1, i + 32, d1);
    }
  }
}

template <int MODE, int BITS, int P, bool TAB16>
__global__ void __launch_bounds__(kMaxWarps * 32, 1) rotq_pair_kernel(Params p) {
  constexpr int kTR = 2 * P;                       // rows per tile
  constexpr uint32_t kTabBytes = TAB16 ? 2u : 4u;  // per gather-table entry
  constexpr bool kAsym = (MODE == kInt8Asym);
  constexpr int kParts = kAsym ? 2 : 1;             // partial-result arrays (max, min)
  extern __shared__ unsigned char smem_raw[];
  const uint32_t sraw = smem_u32(smem_raw);
  const uint32_t sbase = (sraw + 127u) & ~127u;
  unsigned char* sm = smem_raw + (sbase - sraw);
  const Layout L = layout(p.d, p.NS, p.grid_entries, kTR, kTabBytes, kParts);
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + L.bars);
  uint64_t* red = full + p.NS;
  uint64_t* tabbar = red + 2 * p.NS;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tabbar + 1);  // TMEM base address
  constexpr bool kLloyd = (MODE == kAct || MODE == kWeightLM);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int NS = p.NS;

  const uint32_t pitch = p.pitch;
  const uint32_t slot_bytes = kTR * pitch;
  const uint32_t ring = sbase + L.ring;

  // The bulk copies of tile `tile` into slot `slot`, shared out over the
  // CTA: row r is copied by lane r / nwarps of warp r % nwarps (at most a few
  // copies per warp, so no warp stalls long on the copy engine), and thread 0
  // posts the expected bytes.  Every thread calls it at the same points, in
  // slot order 0, 1, ..., NS-1, 0, ..., and counts the calls.
  int n_issued = 0;
  auto issue_rows = [&](int tile, int slot) {
    const uint32_t row_bytes = 2u * static_cast<uint32_t>(p.d);
    const long long r0 = static_cast<long long>(tile) * kTR;
    const int rows = static_cast<int>(min(static_cast<long long>(kTR), p.T - r0));
    ++n_issued;
    if (tid == 0) mbar_arrive_expect_tx(&full[slot], static_cast<uint32_t>(rows) * row_bytes);
    for (int r = warp + p.nwarps * lane; r < rows; r += 32 * p.nwarps) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      bulk_load(ring + slot * slot_bytes + r * pitch, p.X + (r0 + r) * p.d, row_bytes, &full[slot]);
    }
  };

  // ---- prologue: the gather table and the guarded code grid start streaming
  //      first; the first tile follows once the barriers are visible to all
  //      (the other slots fill after it has landed, so that it is not slowed
  //      by them) ----
  if (tid == 0) {
    for (int s = 0; s < NS; ++s) mbar_init(&full[s], 1);
    for (int r = 0; r < 2 * NS; ++r) mbar_init(&red[r], p.nwarps);   // one arrival per warp
    mbar_init(tabbar, 1);
    mbar_fence_init();
    const uint32_t gbytes = kLloyd ? 8u * static_cast<uint32_t>(p.grid_entries) : 0u;
    mbar_arrive_expect_tx(tabbar, kTabBytes * p.d + gbytes);
    bulk_load(sbase + L.off, p.tab, kTabBytes * p.d, tabbar);
    if (kLloyd) bulk_load(sbase + L.grid, p.grid, gbytes, tabbar);
  }
  {
    float* part = reinterpret_cast<float*>(sm + L.part);
    for (int i = tid; i < kParts * (2 * NS) * kTR * kMaxWarps; i += blockDim.x) part[i] = 0.f;
  }
  __syncwarp();
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // Everything above touches only this launch's own shared memory and the
  // handle's constant tables; the rows and every output wait for the kernels
  // this launch depends on (launched with programmatic dependent launch, the
  // prologue overlaps their tail).
  griddep_wait();
  griddep_launch_dependents();
  if (blockIdx.x < p.ntiles) issue_rows(blockIdx.x, 0);
  if (!mbar_wait(tabbar, 0)) atomicOr(p.err, 256u);

  // ---------------- consumers ----------------
  const int j = lane / P, pp = lane % P;           // lane = P j + p
  const int b = (32 / P) * warp + j;               // output block of this thread
  // With 8 pairs the host keeps d % 256 == 0, so every block is a whole
  // warp's; otherwise the last warp may hold lanes past the last block.
  const bool act = (P == 8) || b < p.nblk;
  const int bx = b & 7;
  const uint32_t off_addr = sbase + L.off + 64u * kTabBytes * (act ? b : 0);
  const uint32_t part_addr = sbase + L.part;
  const uint32_t part2_addr = part_addr + 4u * (2 * NS) * kTR * kMaxWarps;   // asymmetric INT8: the minima
  const uint32_t gbase = sbase + L.grid + 8u * static_cast<uint32_t>(p.grid_first) - 0x4B000000u * 8u;
  const uint32_t pitchP = static_cast<uint32_t>(P) * pitch;   // token p to token p + P
  // Tensor memory: each thread parks its pair's two half-blocks (2 x 64 words)
  // in its own lane; warps w, w+4, w+8 share a lane quarter, 128 columns each.
  const uint32_t tA = *tmem_slot + (static_cast<uint32_t>(32 * (warp & 3)) << 16) + 128u * (warp >> 2);
  const uint32_t tB = tA + 64u;
  int it = 0;
  for (int tile = blockIdx.x; tile < p.ntiles; tile += gridDim.x, ++it) {
    const int s = it % NS, rb = it % (2 * NS);
    // A timed-out wait ends the whole warp's loop together: the tensor-memory
    // accesses below are warp-collective (.sync.aligned).
    if (__any_sync(0xffffffffu, !mbar_wait(&full[s], (it / NS) & 1))) { atomicOr(p.err, 64u); break; }
    if (it == 0)
      for (int s2 = 1; s2 < NS; ++s2)
        if (blockIdx.x + s2 * static_cast<int>(gridDim.x) < p.ntiles) issue_rows(blockIdx.x + s2 * gridDim.x, s2);

    // ---- gather x[pi(k)] with D_k folded in (tokens p, p+P), one half-block
    //      at a time; butterfly strides 1..16 inside each half; park in TMEM ----
    const uint32_t rowA = ring + s * slot_bytes + pp * pitch;
    unsigned long long acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      unsigned long long R[32];
      if (act && TAB16) {
        // 16-bit entries, 8 per 16-byte chunk: byte offset | sign << 15
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8) {
          const uint32_t c = 16u * (static_cast<uint32_t>(4 * h + q8) ^ static_cast<uint32_t>(bx));
          const uint4 o = lds128(off_addr + c);
          const uint32_t ww[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const uint32_t w = ww[e >> 1];
            const uint32_t S = (e & 1) ? (w & 0x80000000u) : ((w << 16) & 0x80000000u);
            const uint32_t off = ((e & 1) ? (w >> 16) : w) & 0x7FFFu;
            const uint32_t a = rowA + dbg_index(off, 2u * static_cast<uint32_t>(p.d), p.err);
            const float y0 = bf16_signed(lds_u16(a), S);
            const float y1 = bf16_signed(lds_u16(a + pitchP), S);
            R[8 * q8 + e] = pk(y0, y1);
            acc[e & 3] = fma2(R[8 * q8 + e], R[8 * q8 + e], acc[e & 3]);
          }
        }
      } else if (act) {
#pragma unroll
        for (int q4 = 0; q4 < 8; ++q4) {
          const uint32_t c = 16u * (static_cast<uint32_t>(8 * h + q4) ^ static_cast<uint32_t>(bx));
          const uint4 o = lds128(off_addr + c);
          const uint32_t oo[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            // entry = source byte offset | sign << 31: the sign word S feeds the
            // conversion, the entry minus S is the offset
            const uint32_t S = oo[e] & 0x80000000u;
            const uint32_t a = rowA + dbg_index(oo[e] - S, 2u * static_cast<uint32_t>(p.d), p.err);
            const float y0 = bf16_signed(lds_u16(a), S);
            const float y1 = bf16_signed(lds_u16(a + pitchP), S);
            R[4 * q4 + e] = pk(y0, y1);
            acc[e] = fma2(R[4 * q4 + e], R[4 * q4 + e], acc[e]);
          }
        }
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) R[i] = 0ull;      // a lane past the last block: zeros
      }
      if (h == 1) {
        if constexpr (MODE != kInt8 && !kAsym) {
          // ||x||^2 partials of both tokens (||Pi x|| = ||x||): 32/P lanes share a pair
          float a0, a1;
          upk(add2(add2(acc[0], acc[1]), add2(acc[2], acc[3])), a0, a1);
#pragma unroll
          for (int o = P; o < 32; o <<= 1) {
            a0 += __shfl_xor_sync(0xffffffffu, a0, o);
            a1 += __shfl_xor_sync(0xffffffffu, a1, o);
          }
          if (j == 0) {
            sts_f32(part_addr + 4u * ((rb * kTR + pp) * kMaxWarps + warp), a0);
            sts_f32(part_addr + 4u * ((rb * kTR + pp + P) * kMaxWarps + warp), a1);
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&red[rb]);
        }
      }
#pragma unroll
      for (int st = 1; st < 32; st <<= 1) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          if ((i & st) == 0) {
            const unsigned long long a = R[i], c = R[i + st];
            R[i] = add2(a, c);
            R[i + st] = sub2(a, c);
          }
        }
      }
      uint32_t v0[32], v1[32];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        upk_u(R[i], v0[2 * i], v0[2 * i + 1]);
        upk_u(R[16 + i], v1[2 * i], v1[2 * i + 1]);
      }
      __syncwarp();
      tmem_st32((h ? tB : tA), v0);
      tmem_st32((h ? tB : tA) + 32u, v1);
    }
    tmem_wait_st();

    if constexpr (MODE == kInt8 || kAsym) {
      // max |z| (asymmetric: max z and min z, both widened to contain 0) needs
      // the last butterfly stage: z_i = A_i + B_i, z_{i+32} = A_i - B_i
      float m0 = 0.f, m1 = 0.f, n0 = 0.f, n1 = 0.f;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t va[32], vb[32];
        __syncwarp();
        tmem_ld32(tA + 32u * c, va);
        tmem_ld32(tB + 32u * c, vb);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const unsigned long long a = pk_u(va[2 * k], va[2 * k + 1]), bb = pk_u(vb[2 * k], vb[2 * k + 1]);
          float z0, z1, y0, y1;
          upk(add2(a, bb), z0, z1);
          upk(sub2(a, bb), y0, y1);
          if constexpr (kAsym) {
            m0 = fmaxf(m0, fmaxf(z0, y0));
            m1 = fmaxf(m1, fmaxf(z1, y1));
            n0 = fminf(n0, fminf(z0, y0));
            n1 = fminf(n1, fminf(z1, y1));
          } else {
            m0 = fmaxf(m0, fmaxf(fabsf(z0), fabsf(y0)));
            m1 = fmaxf(m1, fmaxf(fabsf(z1), fabsf(y1)));
          }
        }
      }
#pragma unroll
      for (int o = P; o < 32; o <<= 1) {
        m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, o));
        m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, o));
        if constexpr (kAsym) {
          n0 = fminf(n0, __shfl_xor_sync(0xffffffffu, n0, o));
          n1 = fminf(n1, __shfl_xor_sync(0xffffffffu, n1, o));
        }
      }
      if (j == 0) {
        sts_f32(part_addr + 4u * ((rb * kTR + pp) * kMaxWarps + warp), m0);
        sts_f32(part_addr + 4u * ((rb * kTR + pp + P) * kMaxWarps + warp), m1);
        if constexpr (kAsym) {
          sts_f32(part2_addr + 4u * ((rb * kTR + pp) * kMaxWarps + warp), n0);
          sts_f32(part2_addr + 4u * ((rb * kTR + pp + P) * kMaxWarps + warp), n1);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&red[rb]);
    }

    // ---- per-token totals: fixed summation order, identical in every thread ----
    if (__any_sync(0xffffffffu, !mbar_wait(&red[rb], (it / (2 * NS)) & 1))) { atomicOr(p.err, 64u); break; }
    // Every thread arrived on red[rb] after its last read of slot s, so the
    // slot can take the tile NS steps ahead (the barrier's release/acquire
    // orders those reads before the asynchronous overwrite).
    if (tile + NS * static_cast<int>(gridDim.x) < p.ntiles) issue_rows(tile + NS * gridDim.x, s);
    float tot[2], tot2[2];                         // tot2: asymmetric INT8 min z
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      if constexpr (kAsym) {
        const uint32_t pa = part2_addr + 4u * ((rb * kTR + pp + P * h) * kMaxWarps);
        const uint4 q0 = lds128(pa), q1 = lds128(pa + 16), q2 = lds128(pa + 32);
        const uint32_t u[12] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w, q2.x, q2.y, q2.z, q2.w};
        float m = __uint_as_float(u[0]);
#pragma unroll
        for (int w = 1; w < 12; ++w) m = fminf(m, __uint_as_float(u[w]));
        tot2[h] = m;
      } else {
        tot2[h] = 0.f;
      }
      const uint32_t pa = part_addr + 4u * ((rb * kTR + pp + P * h) * kMaxWarps);
      const uint4 q0 = lds128(pa), q1 = lds128(pa + 16), q2 = lds128(pa + 32);
      const float v[12] = {__uint_as_float(q0.x), __uint_as_float(q0.y), __uint_as_float(q0.z),
                           __uint_as_float(q0.w), __uint_as_float(q1.x), __uint_as_float(q1.y),
                           __uint_as_float(q1.z), __uint_as_float(q1.w), __uint_as_float(q2.x),
                           __uint_as_float(q2.y), __uint_as_float(q2.z), __uint_as_float(q2.w)};
      if constexpr (MODE == kInt8 || kAsym) {
        float m = v[0];
#pragma unroll
        for (int w = 1; w < 12; ++w) m = fmaxf(m, v[w]);
        tot[h] = m;
      } else {
        tot[h] = ((v[0] + v[1]) + (v[2] + v[3])) + ((v[4] + v[5]) + (v[6] + v[7])) + ((v[8] + v[9]) + (v[10] + v[11]));
      }
    }

    const long long t0 = static_cast<long long>(tile) * kTR + pp, t1 = t0 + P;
    const bool ok0 = act && t0 < p.T, ok1 = act && t1 < p.T;   // rows to store

    if constexpr (kLloyd) {
      const float s0 = sqrtf(tot[0]), s1 = sqrtf(tot[1]);      // ||x|| = ||Pi x||
      // A non-finite row (or a padding row past T) is encoded as the zero
      // vector, which also keeps every grid index inside the table.
      const bool bad0 = !(tot[0] < INFINITY) || !ok0, bad1 = !(tot[1] < INFINITY) || !ok1;
      // z is 8x the rotated value: v = z / (8 s + 8 eps); a bad row's z is
      // taken as 0 below and its scale as 0, so its v is exactly 0 (the
      // middle cell, code 2^(b-1)) even when its norm is NaN
      const float inv0 = bad0 ? 0.f : 1.0f / (8.0f * s0 + 8e-12f);
      const float inv1 = bad1 ? 0.f : 1.0f / (8.0f * s1 + 8e-12f);
      uint32_t w0[2 * BITS], w1[2 * BITS];
#pragma unroll
      for (int i = 0; i < 2 * BITS; ++i) w0[i] = w1[i] = 0u;
      Enc enc(inv0, inv1, p.grid_cells, p.grid_scale, gbase);
#ifdef RBQ_DEBUG
      enc.dbg_err = p.err;
      enc.dbg_entries = static_cast<uint32_t>(p.grid_entries);
      enc.dbg_first = static_cast<uint32_t>(p.grid_first);
#endif
      // warp-uniform choice: encode_block reads tensor memory collectively
      if (__any_sync(0xffffffffu, bad0 || bad1)) {
        encode_block<BITS, true>(enc, tA, tB, bad0, bad1, w0, w1);
      } else {
        encode_block<BITS, false>(enc, tA, tB, false, false, w0, w1);
      }
      const long long cp = static_cast<long long>(p.d) * BITS / 8;
      unsigned char* out = static_cast<unsigned char*>(p.out) + static_cast<long long>(b) * 8 * BITS;
      if (ok0) store_codes<BITS>(out + t0 * cp, w0, p.st256 != 0);
      if (ok1) store_codes<BITS>(out + t1 * cp, w1, p.st256 != 0);
      if (b == 0) {
        if (MODE == kAct) {
          if (ok0) static_cast<float*>(p.aux)[t0] = s0;
          if (ok1) static_cast<float*>(p.aux)[t1] = s1;
        } else {
          if (ok0) static_cast<__nv_bfloat16*>(p.aux)[t0] = __float2bfloat16_rn(s0);
          if (ok1) static_cast<__nv_bfloat16*>(p.aux)[t1] = __float2bfloat16_rn(s1);
        }
      }
    } else if constexpr (MODE == kInt8) {
      // scale = max|w'| / 127 with w' = z / 8; q = clamp(round(w' / scale), +-127)
      const float sc0 = p.fixed_scale ? *p.fixed_scale : (tot[0] * 0.125f) / 127.0f;
      const float sc1 = p.fixed_scale ? *p.fixed_scale : (tot[1] * 0.125f) / 127.0f;
      const float r0 = (sc0 > 0.f) ? 1.0f / sc0 : 0.f, r1 = (sc1 > 0.f) ? 1.0f / sc1 : 0.f;
      int8_t* out = static_cast<int8_t*>(p.out) + 64 * b;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t va[32], vb[32];
        __syncwarp();
        tmem_ld32(tA + 32u * c, va);
        tmem_ld32(tB + 32u * c, vb);
        tmem_wait_ld();
        uint32_t qa0[4] = {0u, 0u, 0u, 0u}, qa1[4] = {0u, 0u, 0u, 0u};   // positions 16c + k
        uint32_t qb0[4] = {0u, 0u, 0u, 0u}, qb1[4] = {0u, 0u, 0u, 0u};   // positions 32 + 16c + k
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const unsigned long long a = pk_u(va[2 * k], va[2 * k + 1]), bb = pk_u(vb[2 * k], vb[2 * k + 1]);
          float z0, z1, y0, y1;
          upk(add2(a, bb), z0, z1);
          upk(sub2(a, bb), y0, y1);
          const int sh = 8 * (k & 3);
          qa0[k >> 2] |= (static_cast<uint32_t>(max(-127, min(127, __float2int_rn(z0 * 0.125f * r0)))) & 0xFFu) << sh;
          qa1[k >> 2] |= (static_cast<uint32_t>(max(-127, min(127, __float2int_rn(z1 * 0.125f * r1)))) & 0xFFu) << sh;
          qb0[k >> 2] |= (static_cast<uint32_t>(max(-127, min(127, __float2int_rn(y0 * 0.125f * r0)))) & 0xFFu) << sh;
          qb1[k >> 2] |= (static_cast<uint32_t>(max(-127, min(127, __float2int_rn(y1 * 0.125f * r1)))) & 0xFFu) << sh;
        }
        if (ok0) {
          __stcs(reinterpret_cast<uint4*>(out + t0 * p.d + 16 * c), make_uint4(qa0[0], qa0[1], qa0[2], qa0[3]));
          __stcs(reinterpret_cast<uint4*>(out + t0 * p.d + 32 + 16 * c), make_uint4(qb0[0], qb0[1], qb0[2], qb0[3]));
        }
        if (ok1) {
          __stcs(reinterpret_cast<uint4*>(out + t1 * p.d + 16 * c), make_uint4(qa1[0], qa1[1], qa1[2], qa1[3]));
          __stcs(reinterpret_cast<uint4*>(out + t1 * p.d + 32 + 16 * c), make_uint4(qb1[0], qb1[1], qb1[2], qb1[3]));
        }
      }
      if (b == 0) {
        if (ok0 && !p.fixed_scale) static_cast<float*>(p.aux)[t0] = sc0;
        if (ok1 && !p.fixed_scale) static_cast<float*>(p.aux)[t1] = sc1;
      }
    } else if constexpr (kAsym) {
      // the row's range [min w', max w'] widened to contain 0, 255 steps:
      // scale = (hi - lo) / 255, zero point = round(-lo / scale) in 0..255,
      // q = clamp(round(w' / scale) + zero point, 0, 255), w' = z / 8
      float sc[2], rc[2];
      int zp[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float hi = tot[h] * 0.125f, lo = tot2[h] * 0.125f;
        sc[h] = (hi - lo) / 255.0f;
        rc[h] = (sc[h] > 0.f) ? 1.0f / sc[h] : 0.f;
        zp[h] = (sc[h] > 0.f) ? min(255, max(0, __float2int_rn(-lo * rc[h]))) : 0;
      }
      uint8_t* out = static_cast<uint8_t*>(p.out) + 64 * b;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t va[32], vb[32];
        __syncwarp();
        tmem_ld32(tA + 32u * c, va);
        tmem_ld32(tB + 32u * c, vb);
        tmem_wait_ld();
        uint32_t qa0[4] = {0u, 0u, 0u, 0u}, qa1[4] = {0u, 0u, 0u, 0u};   // positions 16c + k
        uint32_t qb0[4] = {0u, 0u, 0u, 0u}, qb1[4] = {0u, 0u, 0u, 0u};   // positions 32 + 16c + k
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const unsigned long long a = pk_u(va[2 * k], va[2 * k + 1]), bb = pk_u(vb[2 * k], vb[2 * k + 1]);
          float z0, z1, y0, y1;
          upk(add2(a, bb), z0, z1);
          upk(sub2(a, bb), y0, y1);
          const int sh = 8 * (k & 3);
          const auto code = [&](float z, int h) {
            return static_cast<uint32_t>(sc[h] > 0.f ? min(255, max(0, __float2int_rn(z * 0.125f * rc[h]) + zp[h])) : 0);
          };
          qa0[k >> 2] |= code(z0, 0) << sh;
          qa1[k >> 2] |= code(z1, 1) << sh;
          qb0[k >> 2] |= code(y0, 0) << sh;
          qb1[k >> 2] |= code(y1, 1) << sh;
        }
        if (ok0) {
          __stcs(reinterpret_cast<uint4*>(out + t0 * p.d + 16 * c), make_uint4(qa0[0], qa0[1], qa0[2], qa0[3]));
          __stcs(reinterpret_cast<uint4*>(out + t0 * p.d + 32 + 16 * c), make_uint4(qb0[0], qb0[1], qb0[2], qb0[3]));
        }
        if (ok1) {
          __stcs(reinterpret_cast<uint4*>(out + t1 * p.d + 16 * c), make_uint4(qa1[0], qa1[1], qa1[2], qa1[3]));
          __stcs(reinterpret_cast<uint4*>(out + t1 * p.d + 32 + 16 * c), make_uint4(qb1[0], qb1[1], qb1[2], qb1[3]));
        }
      }
      if (b == 0) {
        if (ok0) {
          static_cast<float*>(p.aux)[t0] = sc[0];
          p.zero_point[t0] = static_cast<uint8_t>(zp[0]);
        }
        if (ok1) {
          static_cast<float*>(p.aux)[t1] = sc[1];
          p.zero_point[t1] = static_cast<uint8_t>(zp[1]);
        }
      }
    } else {   // kRotate: x' = z / 8 in BF16
      __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out) + 64 * b;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t va[32], vb[32];
        __syncwarp();
        tmem_ld32(tA + 32u * c, va);
        tmem_ld32(tB + 32u * c, vb);
        tmem_wait_ld();
        uint32_t ua0[8], ua1[8], ub0[8], ub1[8];
#pragma unroll
        for (int k2 = 0; k2 < 8; ++k2) {
          float z[2][2], y[2][2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int k = 2 * k2 + e;
            const unsigned long long a = pk_u(va[2 * k], va[2 * k + 1]), bb = pk_u(vb[2 * k], vb[2 * k + 1]);
            upk(add2(a, bb), z[e][0], z[e][1]);
            upk(sub2(a, bb), y[e][0], y[e][1]);
          }
          ua0[k2] = bf2_bits(z[0][0] * 0.125f, z[1][0] * 0.125f);
          ua1[k2] = bf2_bits(z[0][1] * 0.125f, z[1][1] * 0.125f);
          ub0[k2] = bf2_bits(y[0][0] * 0.125f, y[1][0] * 0.125f);
          ub1[k2] = bf2_bits(y[0][1] * 0.125f, y[1][1] * 0.125f);
        }
        if (p.st256) {                 // 32-byte aligned rows: one store per 16 values
          if (ok0) {
            st_v8_cs(out + t0 * p.d + 16 * c, ua0);
            st_v8_cs(out + t0 * p.d + 32 + 16 * c, ub0);
          }
          if (ok1) {
            st_v8_cs(out + t1 * p.d + 16 * c, ua1);
            st_v8_cs(out + t1 * p.d + 32 + 16 * c, ub1);
          }
        } else {
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            if (ok0) {
              __stcs(reinterpret_cast<uint4*>(out + t0 * p.d + 16 * c) + q,
                     make_uint4(ua0[4 * q], ua0[4 * q + 1], ua0[4 * q + 2], ua0[4 * q + 3]));
              __stcs(reinterpret_cast<uint4*>(out + t0 * p.d + 32 + 16 * c) + q,
                     make_uint4(ub0[4 * q], ub0[4 * q + 1], ub0[4 * q + 2], ub0[4 * q + 3]));
            }
            if (ok1) {
              __stcs(reinterpret_cast<uint4*>(out + t1 * p.d + 16 * c) + q,
                     make_uint4(ua1[4 * q], ua1[4 * q + 1], ua1[4 * q + 2], ua1[4 * q + 3]));
              __stcs(reinterpret_cast<uint4*>(out + t1 * p.d + 32 + 16 * c) + q,
                     make_uint4(ub1[4 * q], ub1[4 * q + 1], ub1[4 * q + 2], ub1[4 * q + 3]));
            }
          }
        }
      }
      if (b == 0 && p.aux) {
        if (ok0) static_cast<float*>(p.aux)[t0] = sqrtf(tot[0]);
        if (ok1) static_cast<float*>(p.aux)[t1] = sqrtf(tot[1]);
      }
    }
  }

  // Every bulk copy this CTA issued has landed before it exits: each thread
  // that copies rows waits for the last phase of every slot it wrote (they
  // all have landed on the normal path; after a timed-out wait, when the
  // threads may have left the loop at different tiles, this bounds the exit).
  tc_fence_before();
  __syncthreads();
  if (warp + p.nwarps * lane < kTR) {
    bool ok = true;
    for (int s = 0; s < NS; ++s) {
      const int uses = n_issued > s ? (n_issued - 1 - s) / NS + 1 : 0;
      if (uses && !mbar_wait(&full[s], (uses - 1) & 1)) ok = false;
    }
    if (!ok) atomicOr(p.err, 128u);
  }
  __syncwarp();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(*tmem_slot, 512);
  }
}

}  // namespace pairk

// ---- host side ------------------------------------------------------------

namespace {

template <int MODE, int BITS, int P, bool TAB16>
int launch_pair(const pairk::Params& p, cudaStream_t st) {
  auto kern = pairk::rotq_pair_kernel<MODE, BITS, P, TAB16>;
  const size_t smem =
      rowtile::layout(p.d, p.NS, p.grid_entries, 2 * P, TAB16 ? 2 : 4, MODE == rowtile::kInt8Asym ? 2 : 1).total + 128;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return cuda_fail(e);
  const int sms = rowtile::sm_count();
  const int grid = p.ntiles < sms ? p.ntiles : sms;
  return rowtile::launch_pdl(kern, grid, p.nwarps * 32, smem, st, p);
}

// The 16-bit table is instantiated only for 2-pair tiles, the one geometry
// that needs it (widths of about 11000 to 12288; 1-pair tiles fit the 32-bit
// table up to 16384).
template <int MODE, int BITS>
int launch_pair_p(int P, bool tab16, const pairk::Params& p, cudaStream_t st) {
  switch (P) {
    case 8: return launch_pair<MODE, BITS, 8, false>(p, st);
    case 4: return launch_pair<MODE, BITS, 4, false>(p, st);
    case 2: return tab16 ? launch_pair<MODE, BITS, 2, true>(p, st) : launch_pair<MODE, BITS, 2, false>(p, st);
    default: return launch_pair<MODE, BITS, 1, false>(p, st);
  }
}

template <int MODE>
int launch_pair_bits(int bits, int P, bool tab16, const pairk::Params& p, cudaStream_t st) {
  switch (bits) {
    case 1: return launch_pair_p<MODE, 1>(P, tab16, p, st);
    case 2: return launch_pair_p<MODE, 2>(P, tab16, p, st);
    case 3: return launch_pair_p<MODE, 3>(P, tab16, p, st);
    case 4: return launch_pair_p<MODE, 4>(P, tab16, p, st);
    case 5: return launch_pair_p<MODE, 5>(P, tab16, p, st);
    case 6: return launch_pair_p<MODE, 6>(P, tab16, p, st);
    case 7: return launch_pair_p<MODE, 7>(P, tab16, p, st);
    case 8: return launch_pair_p<MODE, 8>(P, tab16, p, st);
    default: return RBQ_EINVAL;
  }
}

}  // namespace

bool rotq_pair_eligible(int dtype, int d) { return dtype == RBQ_BF16 && d % 256 == 0 && d >= 1024 && d <= 16384; }

// Pairs per tile for width d: the most (8, 4, 2 or 1) whose CTA has at most
// kMaxWarps warps and whose ring keeps at least two slots next to the tables,
// with the 32-bit gather table if it fits, else (2 pairs) the 16-bit one; 0
// when none fits.  Sets the ring slots, the warps and the table width.
int pair_geometry(int d, int grid_entries, int nparts, int* NS, int* nwarps, bool* tab16) {
  const int nblk = d / kH;
  for (int P = 8; P >= 1; P >>= 1) {
    const int w = (P * nblk + 31) / 32;
    if (w > rowtile::kMaxWarps) continue;
    for (int t16 = 0; t16 < (P == 2 ? 2 : 1); ++t16) {
      const int ns = rowtile::slots_that_fit(d, grid_entries, 2 * P, t16 ? 2 : 4, nparts);
      if (ns >= 2) {
        *NS = ns;
        *nwarps = w;
        *tab16 = t16 != 0;
        return P;
      }
    }
  }
  return 0;
}

// Returns RBQ_ECONVERGE when the tables do not fit (the caller then uses
// another kernel); any other code is the call's result.
int rotq_pair_launch(const rbq_rpbh* r, int mode, int bits, long long rows, const void* X, void* out, void* aux,
                     cudaStream_t st, const float* fixed_scale, uint8_t* zero_point) {
  using namespace pairk;
  Params p{};
  p.X = static_cast<const __nv_bfloat16*>(X);
  p.T = rows;
  p.d = r->d;
  p.nblk = r->d / kH;
  p.pitch = 2u * static_cast<uint32_t>(r->d) + 16u;
  p.out = out;
  p.aux = aux;
  p.fixed_scale = fixed_scale;
  p.zero_point = zero_point;
  int rc = device_error_word_ptr(&p.err);
  if (rc != RBQ_OK) return rc;
  const bool lloyd = (mode == kAct || mode == kWeightLM);
  if (lloyd) {
    const CodebookDevice* cb = nullptr;
    if ((rc = codebook_device(r->d, bits, &cb)) != RBQ_OK) return rc;
    p.grid = cb->grid_pad;
    p.grid_entries = guarded_grid_entries(cb->grid_cells + 1);
    p.grid_first = kGridGuard;
    p.grid_cells = static_cast<float>(cb->grid_cells);
    p.grid_scale = cb->grid_scale;
  }
  bool tab16 = false;
  const int P = pair_geometry(r->d, p.grid_entries, mode == kInt8Asym ? 2 : 1, &p.NS, &p.nwarps, &tab16);
  if (P == 0) return RBQ_ECONVERGE;
  // With pi = identity (the ablation handle) the source of step i of every
  // block sits at the same offset of consecutive 128-byte blocks, i.e. in one
  // bank: with fewer than 8 pairs a warp's 32/P blocks would all conflict.
  // The register-staged kernel, whose staging spreads the blocks, takes it.
  if (P < 8 && (r->flags & RBQ_RPBH_NO_PERMUTATION)) return RBQ_ECONVERGE;
  if (tab16) {
    const uint16_t* t = nullptr;
    if ((rc = rpbh_pair_tables16(r, &t)) != RBQ_OK) return rc;
    p.tab = t;
  } else {
    const uint32_t* t = nullptr;
    if ((rc = rpbh_pair_tables(r, &t)) != RBQ_OK) return rc;
    p.tab = t;
  }
  p.ntiles = static_cast<int>((rows + 2 * P - 1) / (2 * P));
  // 32-byte stores need every row's block start 32-byte aligned (rotate-only
  // rows are 2d bytes, a multiple of 512)
  p.st256 = (reinterpret_cast<uintptr_t>(out) % 32 == 0 &&
             ((lloyd && (static_cast<long long>(r->d) * bits / 8) % 32 == 0) || mode == kRotate)) ? 1 : 0;
  switch (mode) {
    case kAct: return launch_pair_bits<kAct>(bits, P, tab16, p, st);
    case kWeightLM: return launch_pair_bits<kWeightLM>(bits, P, tab16, p, st);
    case kInt8: return launch_pair_p<kInt8, 8>(P, tab16, p, st);
    case kInt8Asym: return launch_pair_p<kInt8Asym, 8>(P, tab16, p, st);
    default: return launch_pair_p<kRotate, 8>(P, tab16, p, st);
  }
}

}  // namespace rbq
