// Fused rotate-then-quantise kernel (one kernel, four output modes).
//
//   OrbitQuant (hotelren.com/news/3376620) §2.2, online activations:
//     x' = Pi_d x, s = ||x'||, v = x'/(s+eps), codes = Q_b(v) -> packed + s.
//   OrbitQuant §2.1, offline weights: the same on each row w_i, r' kept BF16.
//   INT8-convrot (cloud.baidu.com/article/9430339) §4: rotate, scale =
//     max|w'|/127, q = round(w'/scale).
//   Rotate-only: x' = Pi_d x in BF16, the activation operand of the W8A16
//     linear (INT8-convrot §3: the transform information is used at inference).
//
// Pi_d = blkdiag(H_64 D_1, ..., H_64 D_{d/64}) · P_pi (OrbitQuant §2.3).  One
// thread owns one 64-wide output block of one token: it gathers its 64 inputs
// x[pi(k)] from the token row staged in shared memory, applies the signs,
// runs the 64-point Walsh-Hadamard butterfly in registers (6 stages), and
// joins the other threads of its token for the norm.

#include <cuda_bf16.h>

#include "rbq_internal.h"
#include "rbq_sm100.cuh"

namespace rbq {
namespace {

using sm100::dbg_index;

enum Mode { kAct = 0, kWeightLM = 1, kInt8 = 2, kRotate = 3, kInt8Asym = 4 };

// Widths up to this use the fast kernel's unclamped [-1, 1] code grid.
constexpr int kFullGridBits = 6;

struct RotqParams {
  const void* X;
  long long T;
  int d, nblk, G;
  const int32_t* perm;
  const float* sign;
  const float* bounds;   // 2^bits - 1 Lloyd-Max boundaries (Lloyd-Max modes)
  void* out;             // packed codes | int8 q | bf16 x'
  void* aux;             // float norms | bf16 row norms | float scales | float norms (optional)
  const float* fixed_scale;   // INT8: one scale for every row (not written back), else null
  uint8_t* zero_point;        // asymmetric INT8: uint8 zero point per row
  unsigned int* err;          // device error word (debug builds' bounds checks)
};

template <typename Tin> __device__ __forceinline__ float to_f32(Tin v);
template <> __device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}

// In-place unnormalised 64-point Walsh-Hadamard transform, Sylvester order:
// out[r] = sum_c (-1)^popcount(r&c) in[c].
__device__ __forceinline__ void fwht64(float (&y)[64]) {
#pragma unroll
  for (int len = 1; len < 64; len <<= 1) {
#pragma unroll
    for (int i = 0; i < 64; ++i) {
      if ((i & len) == 0) {
        const float a = y[i], b = y[i + len];
        y[i] = a + b;
        y[i + len] = a - b;
      }
    }
  }
}

// #{ j : bounds[j] <= v } over 2^BITS - 1 increasing boundaries.
template <int BITS>
__device__ __forceinline__ uint32_t code_of(float v, const float* bounds) {
  uint32_t p = 0;
#pragma unroll
  for (int step = 1 << (BITS - 1); step >= 1; step >>= 1)
    if (v >= bounds[p + step - 1]) p += step;
  return p;
}

template <int MODE, int BITS, typename Tin>
__global__ void __launch_bounds__(512) rotq_kernel(RotqParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int d = p.d, nblk = p.nblk, G = p.G;
  float* rows = reinterpret_cast<float*>(smem_raw);     // [G][d]
  float* red = rows + static_cast<size_t>(G) * d;       // [G][nblk]
  float* tok = red + G * nblk;                           // [G]
  float* bnd = tok + G;                                  // [2^BITS - 1] (256 reserved)
  float* red2 = bnd + 256;                               // [G][nblk] minima (asymmetric INT8)
  float* tok2 = red2 + G * nblk;                         // [G]

  constexpr bool kLloyd = (MODE == kAct || MODE == kWeightLM);
  if (kLloyd) {
    for (int j = threadIdx.x; j < (1 << BITS) - 1; j += blockDim.x) bnd[j] = p.bounds[j];
  }
  const int tid = threadIdx.x;
  const int g = tid / nblk, b = tid - (tid / nblk) * nblk;
  const Tin* X = static_cast<const Tin*>(p.X);

  for (long long t0 = static_cast<long long>(blockIdx.x) * G; t0 < p.T;
       t0 += static_cast<long long>(gridDim.x) * G) {
    __syncthreads();   // previous iteration done with rows/red/tok
    for (int i = tid; i < G * d; i += blockDim.x) {
      const int gg = i / d;
      const long long t = t0 + gg;
      rows[i] = (t < p.T) ? to_f32<Tin>(X[t * d + (i - gg * d)]) : 0.f;
    }
    __syncthreads();

    const long long t = t0 + g;
    float y[64];
#pragma unroll
    for (int i = 0; i < 64; ++i) {
      const int k = 64 * b + i;
      y[i] = p.sign[k] * rows[g * d + dbg_index(static_cast<uint32_t>(p.perm[k]), static_cast<uint32_t>(d), p.err)];
    }
    fwht64(y);
    float acc = (MODE == kInt8Asym) ? -INFINITY : 0.f, acc2 = INFINITY;
#pragma unroll
    for (int i = 0; i < 64; ++i) {
      y[i] *= 0.125f;                                    // 1/sqrt(64): orthonormal H
      if constexpr (MODE == kInt8Asym) {
        acc = fmaxf(acc, y[i]);
        acc2 = fminf(acc2, y[i]);
      } else {
        acc = (MODE == kInt8) ? fmaxf(acc, fabsf(y[i])) : fmaf(y[i], y[i], acc);
      }
    }
    red[g * nblk + b] = acc;
    if constexpr (MODE == kInt8Asym) red2[g * nblk + b] = acc2;
    __syncthreads();
    if (b == 0) {
      if constexpr (MODE == kInt8Asym) {
        float hi = -INFINITY, lo = INFINITY;
        for (int j = 0; j < nblk; ++j) {
          hi = fmaxf(hi, red[g * nblk + j]);
          lo = fminf(lo, red2[g * nblk + j]);
        }
        tok[g] = hi;
        tok2[g] = lo;
      } else {
        float tot = 0.f;
        for (int j = 0; j < nblk; ++j)
          tot = (MODE == kInt8) ? fmaxf(tot, red[g * nblk + j]) : tot + red[g * nblk + j];
        tok[g] = (MODE == kInt8) ? tot : sqrtf(tot);
      }
    }
    __syncthreads();
    if (t >= p.T) continue;
    const float s = tok[g];

    if constexpr (kLloyd) {
      // A row whose norm is not finite is encoded as the zero vector (every
      // v = 0, code 2^(b-1)).
      const bool fin = s < INFINITY;
      const float inv = fin ? 1.0f / (s + 1e-12f) : 0.f;
      uint32_t w[2 * BITS];
#pragma unroll
      for (int i = 0; i < 2 * BITS; ++i) w[i] = 0u;
#pragma unroll
      for (int i = 0; i < 64; ++i) {
        const uint32_t c = code_of<BITS>(fin ? y[i] * inv : 0.f, bnd);
        const int bit = i * BITS, wi = bit >> 5, sh = bit & 31;
        w[wi] |= c << sh;
        if (sh + BITS > 32) w[wi + 1] |= c >> (32 - sh);
      }
      const size_t pitch = static_cast<size_t>(d) * BITS / 8;
      uint2* dst = reinterpret_cast<uint2*>(static_cast<unsigned char*>(p.out) +
                                            static_cast<size_t>(t) * pitch + static_cast<size_t>(b) * 8 * BITS);
#pragma unroll
      for (int i = 0; i < BITS; ++i) dst[i] = make_uint2(w[2 * i], w[2 * i + 1]);
      if (b == 0) {
        if (MODE == kAct) static_cast<float*>(p.aux)[t] = s;
        else static_cast<__nv_bfloat16*>(p.aux)[t] = __float2bfloat16_rn(s);
      }
    } else if constexpr (MODE == kInt8) {
      const float scale = p.fixed_scale ? __ldg(p.fixed_scale) : s / 127.0f;
      int8_t* dst = static_cast<int8_t*>(p.out) + static_cast<size_t>(t) * d + 64 * b;
      uint32_t packed[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) packed[i] = 0u;
#pragma unroll
      for (int i = 0; i < 64; ++i) {
        int q = 0;
        if (scale > 0.f) {
          q = __float2int_rn(__fdiv_rn(y[i], scale));
          q = max(-127, min(127, q));
        }
        packed[i >> 2] |= (static_cast<uint32_t>(q) & 0xFFu) << (8 * (i & 3));
      }
      uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
      for (int i = 0; i < 4; ++i)
        d4[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
      if (b == 0 && !p.fixed_scale) static_cast<float*>(p.aux)[t] = scale;
    } else if constexpr (MODE == kInt8Asym) {
      // the range [min(w'), max(w')] widened to contain 0, 255 steps; the
      // zero point is the code of 0
      const float hi = fmaxf(s, 0.f), lo = fminf(tok2[g], 0.f);
      const float scale = (hi - lo) / 255.0f;
      int z = 0;
      if (scale > 0.f) z = min(255, max(0, __float2int_rn(__fdiv_rn(-lo, scale))));
      uint8_t* dst = static_cast<uint8_t*>(p.out) + static_cast<size_t>(t) * d + 64 * b;
      uint32_t packed[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) packed[i] = 0u;
#pragma unroll
      for (int i = 0; i < 64; ++i) {
        int q = 0;
        if (scale > 0.f) q = min(255, max(0, __float2int_rn(__fdiv_rn(y[i], scale)) + z));
        packed[i >> 2] |= static_cast<uint32_t>(q) << (8 * (i & 3));
      }
      uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
      for (int i = 0; i < 4; ++i)
        d4[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
      if (b == 0) {
        static_cast<float*>(p.aux)[t] = scale;
        p.zero_point[t] = static_cast<uint8_t>(z);
      }
    } else {   // kRotate
      __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.out) + static_cast<size_t>(t) * d + 64 * b;
      uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        uint32_t u[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const __nv_bfloat162 h = __floats2bfloat162_rn(y[8 * i + 2 * j], y[8 * i + 2 * j + 1]);
          u[j] = *reinterpret_cast<const uint32_t*>(&h);
        }
        d4[i] = make_uint4(u[0], u[1], u[2], u[3]);
      }
      if (b == 0 && p.aux) static_cast<float*>(p.aux)[t] = s;
    }
  }
}

// ===========================================================================
// Fast path: BF16 input, 1024 <= d <= 16384.
//
// A CTA owns G tokens at a time (G = 4, 2 or 1 so that G*d/64 threads fit).
// Thread (b, g), tid = b*G + g, produces output block b of token g.
//
//  * Staging: each thread streams 16-byte chunks of its token row from HBM
//    into registers one group ahead, flips the signs of the source positions
//    (a source-side XOR mask: (D P x)_k = D_k x_pi(k) = s'_{pi(k)} x_{pi(k)}
//    with s'_j = D_{pi^-1(j)}), and writes them to shared memory in a
//    chunk-interleaved layout [chunk][token][8 x bf16].  Two stages.
//  * Gather: a per-CTA table holds, for every output position k, the byte
//    offset of source position pi(k) in that layout (swizzled so that the
//    threads of a warp read it without bank conflicts).
//  * Butterfly: the 64 values sit in 32 fp32x2 registers (y_2m, y_2m+1);
//    stride 1 runs inside a pair, strides 2..32 use packed f32x2 add/sub.
//  * Norm: per-thread sum of squares, a shuffle tree over the token's
//    threads in the warp, then the per-warp partials -- a fixed order, so
//    every thread of a token gets the same s.
//  * Codes: one grid lookup and one compare per element (see build_grid()).
// ===========================================================================
namespace fast {

struct Params {
  const __nv_bfloat16* X;
  long long T;
  int d, nblk;
  const int32_t* perm;
  const float* sign;
  const float2* grid;     // Lloyd-Max modes
  int grid_n;             // entries = cells + 1
  float grid_cells, grid_scale;
  void* out;
  void* aux;
  const float* fixed_scale;  // INT8: one scale for every row (not written back), else null
  unsigned int* err;         // device error word (debug builds' bounds checks)
};

__device__ __forceinline__ unsigned long long pk(float a, float b) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void upk(unsigned long long r, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}
__device__ __forceinline__ unsigned long long add2(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ unsigned long long sub2(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ unsigned long long fma2(unsigned long long a, unsigned long long b,
                                                   unsigned long long c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ unsigned long long mul2(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
// 0xFFFFFFFF if a >= b else 0 (IEEE compare: -0 >= -0, NaN never)
__device__ __forceinline__ uint32_t set_ge(float a, float b) {
  uint32_t d;
  asm("set.ge.u32.f32 %0, %1, %2;" : "=r"(d) : "f"(a), "f"(b));
  return d;
}
__device__ __forceinline__ float fma_sat(float a, float b, float c) {
  float d;
  asm("fma.rn.sat.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ uint32_t lds_u16(uint32_t addr) {
  unsigned short v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}
__device__ __forceinline__ void sts128(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}
__device__ __forceinline__ float2 lds_f2(uint32_t addr) {
  float2 v;
  asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint4 ldg_stream(const uint4* p) { return __ldcs(p); }

template <int G>
struct Layout {
  // bytes: stage[2] (G rows of 2d+32) | off (4d) | mask (2d) | red (4*G*32) | grid
  // (the 32-byte pad puts token g's row 8g banks over, so the G threads of an
  // output block read different banks)
  static __host__ __device__ size_t row_pitch(int d) { return 2 * static_cast<size_t>(d) + 32; }
  static __host__ __device__ size_t stage_bytes(int d) { return G * row_pitch(d); }
  static __host__ __device__ size_t off_at(int d) { return 2 * stage_bytes(d); }
  static __host__ __device__ size_t mask_at(int d) { return off_at(d) + 4 * static_cast<size_t>(d); }
  static __host__ __device__ size_t red_at(int d) { return mask_at(d) + 2 * static_cast<size_t>(d); }
  static __host__ __device__ size_t grid_at(int d) { return red_at(d) + 4 * G * 32; }
  static __host__ __device__ size_t total(int d, int grid_n) { return grid_at(d) + 8 * static_cast<size_t>(grid_n); }
};

template <int MODE, int BITS, int G>
__global__ void __launch_bounds__(384, 1) rotq_fast_kernel(Params p) {
  extern __shared__ __align__(16) unsigned char smem[];
  using L = Layout<G>;
  const int d = p.d, nblk = p.nblk;
  const int nthreads = blockDim.x;          // G * nblk rounded up to whole warps
  const int tid = threadIdx.x;
  const int g = tid % G, b = tid / G;
  const bool active = b < nblk;             // padding lanes only join shuffles/barriers
  const uint32_t sbase = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  const uint32_t stage_addr[2] = {sbase, sbase + static_cast<uint32_t>(L::stage_bytes(d))};
  const uint32_t off_addr = sbase + static_cast<uint32_t>(L::off_at(d));
  const uint32_t mask_addr = sbase + static_cast<uint32_t>(L::mask_at(d));
  float* red = reinterpret_cast<float*>(smem + L::red_at(d));
  const uint32_t grid_addr = sbase + static_cast<uint32_t>(L::grid_at(d));
  constexpr bool kLloyd = (MODE == kAct || MODE == kWeightLM);

  // ---- per-CTA tables ------------------------------------------------------
  // mask16[j]: 0x8000 where source position j is sign-flipped, i.e. D_k = -1
  // for the output position k with pi(k) = j.  off[]: byte offset 2*pi(k) of
  // the source of output position k inside a staged row, stored swizzled so
  // that the threads of a warp read their 16-byte groups without conflicts.
  uint16_t* mask16 = reinterpret_cast<uint16_t*>(smem + L::mask_at(d));
  uint32_t* off = reinterpret_cast<uint32_t*>(smem + L::off_at(d));
  for (int k = tid; k < d; k += nthreads) {
    const int j = __ldg(p.perm + k);
    mask16[j] = (__ldg(p.sign + k) < 0.f) ? 0x8000u : 0u;
    const int kb = k >> 6, ki = k & 63;
    const int slot = 64 * kb + 4 * ((ki >> 2) ^ (kb & 15)) + (ki & 3);
    off[slot] = static_cast<uint32_t>(2 * j);
  }
  if (kLloyd) {
    float2* gs = reinterpret_cast<float2*>(smem + L::grid_at(d));
    for (int n = tid; n < p.grid_n; n += nthreads) gs[n] = p.grid[n];
  }
  __syncthreads();   // tables ready

  // ---- staging: 16-byte chunks, token-major rows, chunk index fastest ----
  // Active thread t stages chunks L = t + i*nact (i = 0..7) of the G x (d/8)
  // chunk grid, i.e. 8/G distinct chunk indices per thread; with G = 4 their
  // sign masks stay in registers, otherwise they are read from shared memory.
  // With nact = G*nblk and d/8 = 8*nblk, slot i is token (i*G)>>3, chunk
  // t + ((i*G)&7)*nblk: compile-time in i.
  constexpr bool kRegMasks = (G == 4);         // 2 chunks x 4 words per thread
  constexpr int NM = kRegMasks ? 8 / G : 1;
  uint4 msk[NM];
  if (kRegMasks && active) {
#pragma unroll
    for (int i = 0; i < NM; ++i) msk[i] = lds128(mask_addr + 16 * (tid + ((i * G) & 7) * nblk));
  }
  const long long ngroups = (p.T + G - 1) / G;
  uint4 pre[8];
  auto load_group = [&](long long gi) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int sg = (i * G) >> 3, c = tid + ((i * G) & 7) * nblk;
      const long long row = gi * G + sg;
      const bool valid = active && (gi < ngroups) && (row < p.T);
      pre[i] = valid ? ldg_stream(reinterpret_cast<const uint4*>(p.X + row * d) + c) : make_uint4(0, 0, 0, 0);
    }
  };
  auto store_group = [&](int st) {
    if (!active) return;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int sg = (i * G) >> 3, c = tid + ((i * G) & 7) * nblk;
      uint4 m;
      if constexpr (kRegMasks) m = msk[i % NM];
      else m = lds128(mask_addr + 16 * c);
      const uint4 v = make_uint4(pre[i].x ^ m.x, pre[i].y ^ m.y, pre[i].z ^ m.z, pre[i].w ^ m.w);
      sts128(stage_addr[st] + static_cast<uint32_t>(sg * L::row_pitch(d)) + 16 * c, v);
    }
  };

  long long gi = blockIdx.x;
  load_group(gi);
  store_group(0);
  load_group(gi + gridDim.x);
  __syncthreads();

  const int warp = tid >> 5, lane = tid & 31;
  const int nwarps = (nthreads + 31) >> 5;
  int st = 0;
  for (; gi < ngroups; gi += gridDim.x, st ^= 1) {
    // ---- gather (signs already applied) -> 32 fp32x2 pairs (y_2m, y_2m+1) ----
    unsigned long long P[32];
    if (active) {
      const uint32_t base = stage_addr[st] + static_cast<uint32_t>(g * L::row_pitch(d));
#pragma unroll
      for (int i4 = 0; i4 < 16; ++i4) {
        uint4 o = lds128(off_addr + 4 * (64 * b + 4 * (i4 ^ (b & 15))));
        const uint32_t rb = 2u * static_cast<uint32_t>(d);
        o = make_uint4(dbg_index(o.x, rb, p.err), dbg_index(o.y, rb, p.err), dbg_index(o.z, rb, p.err),
                       dbg_index(o.w, rb, p.err));
        P[2 * i4] = pk(__uint_as_float(lds_u16(base + o.x) << 16), __uint_as_float(lds_u16(base + o.y) << 16));
        P[2 * i4 + 1] = pk(__uint_as_float(lds_u16(base + o.z) << 16), __uint_as_float(lds_u16(base + o.w) << 16));
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) P[j] = 0ull;
    }
    // ---- 64-point Walsh-Hadamard (unnormalised): stride 1 inside a pair,
    //      strides 2..32 between pairs with packed f32x2 ----
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      float lo, hi;
      upk(P[j], lo, hi);
      P[j] = pk(lo + hi, lo - hi);
    }
#pragma unroll
    for (int s = 1; s < 32; s <<= 1) {
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        if ((j & s) == 0) {
          const unsigned long long a = P[j], c = P[j + s];
          P[j] = add2(a, c);
          P[j + s] = sub2(a, c);
        }
      }
    }
    // ---- token reduction: sum of squares (or max |z| for INT8) ----
    float part;
    if (MODE == kInt8) {
      float m = 0.f;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        float lo, hi;
        upk(P[j], lo, hi);
        m = fmaxf(m, fmaxf(fabsf(lo), fabsf(hi)));
      }
      part = m;
    } else {
      unsigned long long acc = 0ull;
#pragma unroll
      for (int j = 0; j < 32; ++j) acc = fma2(P[j], P[j], acc);
      float lo, hi;
      upk(acc, lo, hi);
      part = lo + hi;
    }
    // lanes of the same token in this warp are lane = g (mod G)
#pragma unroll
    for (int o = G; o < 32; o <<= 1) {
      const float other = __shfl_xor_sync(0xffffffffu, part, o);
      part = (MODE == kInt8) ? fmaxf(part, other) : part + other;
    }
    if (lane < G) red[g * 32 + warp] = part;
    __syncthreads();
    float tot = 0.f;
    for (int w = 0; w < nwarps; ++w)
      tot = (MODE == kInt8) ? fmaxf(tot, red[g * 32 + w]) : tot + red[g * 32 + w];

    // ---- refill the other stage (its loads were issued one iteration ago) ----
    store_group(st ^ 1);

    const long long t = gi * G + g;
    if (active && t < p.T) {
      if constexpr (kLloyd && BITS <= kFullGridBits) {
        // z here is 8x the rotated value (H unnormalised): v = z / (||z|| + 8 eps).
        // Grid over v in [-1, 1]: n = round((v + 1)/2 * NC) needs no clamp once
        // z is finite, which holds for every coordinate when ||z|| is finite.
        // A row whose norm is not finite is encoded as the zero vector: z and
        // the scale both 0, so every index lands on the middle cell (a NaN
        // scale would turn into a NaN grid index).
        const float nrm = sqrtf(tot);
        const bool bad = !(nrm < INFINITY);
        if (bad) {
#pragma unroll
          for (int j = 0; j < 32; ++j) P[j] = 0ull;
        }
        const float inv = bad ? 0.f : 1.0f / (nrm + 8e-12f);
        const float kq = inv * (0.5f * p.grid_cells);
        const float cq = 0.5f * p.grid_cells + 8388608.0f;   // + 2^23: round(.) lands in the low bits
        const unsigned long long kq2 = pk(kq, kq), cq2 = pk(cq, cq), inv2 = pk(inv, inv);
        uint32_t w[2 * BITS];
#pragma unroll
        for (int i = 0; i < 2 * BITS; ++i) w[i] = 0u;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          float q0, q1, v0, v1;
          upk(fma2(P[j], kq2, cq2), q0, q1);
          upk(mul2(P[j], inv2), v0, v1);
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int r = 2 * j + e;
            const float2 ent = lds_f2(grid_addr + 8u * dbg_index(__float_as_uint(e ? q1 : q0) - 0x4B000000u,
                                                                 static_cast<uint32_t>(p.grid_n), p.err));
            const uint32_t code = static_cast<uint32_t>(__float_as_int(ent.y)) - set_ge(e ? v1 : v0, ent.x);
            const int bit = r * BITS, wi = bit >> 5, sh = bit & 31;
            if constexpr ((32 % BITS) == 0) {
              w[wi] += code << sh;                 // disjoint fields: add = or
            } else {
              w[wi] |= code << sh;
              if (sh + BITS > 32) w[wi + 1] |= code >> (32 - sh);
            }
          }
        }
        unsigned char* dst = static_cast<unsigned char*>(p.out) + t * (static_cast<long long>(d) * BITS / 8) +
                             static_cast<long long>(b) * 8 * BITS;
        if constexpr ((BITS % 2) == 0) {
#pragma unroll
          for (int i = 0; i < BITS / 2; ++i)
            __stcs(reinterpret_cast<uint4*>(dst) + i, make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]));
        } else {
#pragma unroll
          for (int i = 0; i < BITS; ++i) __stcs(reinterpret_cast<uint2*>(dst) + i, make_uint2(w[2 * i], w[2 * i + 1]));
        }
        if (b == 0) {
          const float sn = nrm * 0.125f;
          if (MODE == kAct) static_cast<float*>(p.aux)[t] = sn;
          else static_cast<__nv_bfloat16*>(p.aux)[t] = __float2bfloat16_rn(sn);
        }
      } else if constexpr (kLloyd) {
        // Clamped grid (wide codebooks): u = sat(v/(2R) + 1/2), n = round(u NC).
        // A row whose norm is not finite is encoded as the zero vector.
        const float nrm = sqrtf(tot);
        const bool bad = !(nrm < INFINITY);
        const float inv = bad ? 0.f : 1.0f / (nrm + 8e-12f);
        const float A = inv * p.grid_scale;
        uint32_t w[2 * BITS];
#pragma unroll
        for (int i = 0; i < 2 * BITS; ++i) w[i] = 0u;
#pragma unroll
        for (int r = 0; r < 64; ++r) {
          float lo, hi;
          upk(P[r >> 1], lo, hi);
          const float z = bad ? 0.f : ((r & 1) ? hi : lo);
          const float u = fma_sat(z, A, 0.5f);
          const float qf = fmaf(u, p.grid_cells, 8388608.0f);   // 2^23: round(u*NC) in the low bits
          const float2 e = lds_f2(grid_addr + 8u * dbg_index(__float_as_uint(qf) - 0x4B000000u,
                                                             static_cast<uint32_t>(p.grid_n), p.err));
          // code = base + (v >= thr): the sign of z*inv - thr, as 0 / -1
          const int below = __float_as_int(fmaf(z, inv, -e.x)) >> 31;
          const uint32_t code = static_cast<uint32_t>(__float_as_int(e.y) + 1 + below);
          const int bit = r * BITS, wi = bit >> 5, sh = bit & 31;
          if constexpr ((32 % BITS) == 0) {
            w[wi] += code << sh;                   // disjoint fields: add = or
          } else {
            w[wi] |= code << sh;
            if (sh + BITS > 32) w[wi + 1] |= code >> (32 - sh);
          }
        }
        unsigned char* dst = static_cast<unsigned char*>(p.out) + t * (static_cast<long long>(d) * BITS / 8) +
                             static_cast<long long>(b) * 8 * BITS;
        if constexpr ((BITS % 2) == 0) {
#pragma unroll
          for (int i = 0; i < BITS / 2; ++i)
            __stcs(reinterpret_cast<uint4*>(dst) + i, make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]));
        } else {
#pragma unroll
          for (int i = 0; i < BITS; ++i) __stcs(reinterpret_cast<uint2*>(dst) + i, make_uint2(w[2 * i], w[2 * i + 1]));
        }
        if (b == 0) {
          const float sn = nrm * 0.125f;
          if (MODE == kAct) static_cast<float*>(p.aux)[t] = sn;
          else static_cast<__nv_bfloat16*>(p.aux)[t] = __float2bfloat16_rn(sn);
        }
      } else if constexpr (MODE == kInt8) {
        const float scale = p.fixed_scale ? __ldg(p.fixed_scale) : (tot * 0.125f) / 127.0f;
        const float rcp = (scale > 0.f) ? 1.0f / scale : 0.f;
        uint32_t q4[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) q4[i] = 0u;
#pragma unroll
        for (int r = 0; r < 64; ++r) {
          float lo, hi;
          upk(P[r >> 1], lo, hi);
          const float z = ((r & 1) ? hi : lo) * 0.125f;
          int q = __float2int_rn(z * rcp);
          q = max(-127, min(127, q));
          q4[r >> 2] |= (static_cast<uint32_t>(q) & 0xFFu) << (8 * (r & 3));
        }
        uint4* dst = reinterpret_cast<uint4*>(static_cast<int8_t*>(p.out) + t * d + 64 * b);
#pragma unroll
        for (int i = 0; i < 4; ++i) __stcs(dst + i, make_uint4(q4[4 * i], q4[4 * i + 1], q4[4 * i + 2], q4[4 * i + 3]));
        if (b == 0 && !p.fixed_scale) static_cast<float*>(p.aux)[t] = scale;
      } else {   // kRotate
        uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + t * d + 64 * b);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          uint32_t u[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            float z0, z1;
            upk(P[4 * i + j], z0, z1);
            const __nv_bfloat162 h = __floats2bfloat162_rn(z0 * 0.125f, z1 * 0.125f);
            u[j] = *reinterpret_cast<const uint32_t*>(&h);
          }
          __stcs(dst + i, make_uint4(u[0], u[1], u[2], u[3]));
        }
        if (b == 0 && p.aux) static_cast<float*>(p.aux)[t] = sqrtf(tot) * 0.125f;
      }
    }
    // next group's loads: issued after the code phase so that the staging
    // registers are not live while the codes are computed
    load_group(gi + 2 * static_cast<long long>(gridDim.x));
    __syncthreads();   // stage st fully read and stage st^1 fully written
  }
}

}  // namespace fast

int sm_count() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

template <int MODE, int BITS, typename Tin>
int launch_one(const RotqParams& p, cudaStream_t st) {
  const int threads = p.G * p.nblk;
  const size_t smem = sizeof(float) * (static_cast<size_t>(p.G) * p.d + 2 * (p.G * p.nblk + p.G) + 256);
  auto kern = rotq_kernel<MODE, BITS, Tin>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return cuda_fail(e);
  const long long groups = (p.T + p.G - 1) / p.G;
  const int grid = static_cast<int>(groups < 8LL * sm_count() ? groups : 8LL * sm_count());
  kern<<<grid, threads, smem, st>>>(p);
  e = cudaGetLastError();
  return e == cudaSuccess ? RBQ_OK : cuda_fail(e);
}

template <int MODE, typename Tin>
int launch_bits(int bits, const RotqParams& p, cudaStream_t st) {
  switch (bits) {
    case 1: return launch_one<MODE, 1, Tin>(p, st);
    case 2: return launch_one<MODE, 2, Tin>(p, st);
    case 3: return launch_one<MODE, 3, Tin>(p, st);
    case 4: return launch_one<MODE, 4, Tin>(p, st);
    case 5: return launch_one<MODE, 5, Tin>(p, st);
    case 6: return launch_one<MODE, 6, Tin>(p, st);
    case 7: return launch_one<MODE, 7, Tin>(p, st);
    case 8: return launch_one<MODE, 8, Tin>(p, st);
    default: return RBQ_EINVAL;
  }
}

template <int MODE>
int launch_mode(int dtype, int bits, const RotqParams& p, cudaStream_t st) {
  if (MODE == kAct || MODE == kWeightLM)
    return dtype == RBQ_BF16 ? launch_bits<MODE, __nv_bfloat16>(bits, p, st)
                             : launch_bits<MODE, float>(bits, p, st);
  return dtype == RBQ_BF16 ? launch_one<MODE, 8, __nv_bfloat16>(p, st)
                           : launch_one<MODE, 8, float>(p, st);
}

// ---- fast path launch --------------------------------------------------------
bool fast_eligible(int dtype, int d) { return dtype == RBQ_BF16 && d >= 1024 && d <= 16384; }

int fast_tokens_per_cta(int nblk) { return (4 * nblk <= 384) ? 4 : (2 * nblk <= 384) ? 2 : 1; }

template <int MODE, int BITS, int G>
int launch_fast_g(const fast::Params& p, cudaStream_t st) {
  const int threads = ((G * p.nblk + 31) / 32) * 32;
  const size_t smem = fast::Layout<G>::total(p.d, p.grid_n);
  auto kern = fast::rotq_fast_kernel<MODE, BITS, G>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return cuda_fail(e);
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem);
  if (e != cudaSuccess) return cuda_fail(e);
  if (per_sm < 1) per_sm = 1;
  const long long groups = (p.T + G - 1) / G;
  const long long cap = static_cast<long long>(per_sm) * sm_count();
  const int grid = static_cast<int>(groups < cap ? groups : cap);
  kern<<<grid, threads, smem, st>>>(p);
  e = cudaGetLastError();
  return e == cudaSuccess ? RBQ_OK : cuda_fail(e);
}

template <int MODE, int BITS>
int launch_fast_bits(const fast::Params& p, cudaStream_t st) {
  switch (fast_tokens_per_cta(p.nblk)) {
    case 4: return launch_fast_g<MODE, BITS, 4>(p, st);
    case 2: return launch_fast_g<MODE, BITS, 2>(p, st);
    default: return launch_fast_g<MODE, BITS, 1>(p, st);
  }
}

template <int MODE>
int launch_fast(int bits, const fast::Params& p, cudaStream_t st) {
  if constexpr (MODE != kAct && MODE != kWeightLM) {
    return launch_fast_bits<MODE, 8>(p, st);
  } else {
  switch (bits) {
    case 1: return launch_fast_bits<MODE, 1>(p, st);
    case 2: return launch_fast_bits<MODE, 2>(p, st);
    case 3: return launch_fast_bits<MODE, 3>(p, st);
    case 4: return launch_fast_bits<MODE, 4>(p, st);
    case 5: return launch_fast_bits<MODE, 5>(p, st);
    case 6: return launch_fast_bits<MODE, 6>(p, st);
    case 7: return launch_fast_bits<MODE, 7>(p, st);
    case 8: return launch_fast_bits<MODE, 8>(p, st);
    default: return RBQ_EINVAL;
  }
  }
}

int run_fast(const rbq_rpbh* r, int mode, int bits, long long rows, const void* X, void* out, void* aux,
             cudaStream_t st, const float* fixed_scale = nullptr) {
  const RpbhDevice* rd = nullptr;
  int rc = rpbh_device(r, &rd);
  if (rc != RBQ_OK) return rc;
  fast::Params p{};
  p.X = static_cast<const __nv_bfloat16*>(X);
  p.T = rows;
  p.d = r->d;
  p.nblk = r->d / kH;
  p.perm = rd->perm;
  p.sign = rd->sign;
  p.out = out;
  p.aux = aux;
  p.fixed_scale = fixed_scale;
  if ((rc = device_error_word_ptr(&p.err)) != RBQ_OK) return rc;
  if (mode == kAct || mode == kWeightLM) {
    const CodebookDevice* cb = nullptr;
    if ((rc = codebook_device(r->d, bits, &cb)) != RBQ_OK) return rc;
    if (bits <= kFullGridBits) {
      if (!cb->grid_full) return RBQ_ECONVERGE;   // caller falls back to the general kernel
      p.grid = cb->grid_full;
      p.grid_n = cb->grid_full_cells + 1;
      p.grid_cells = static_cast<float>(cb->grid_full_cells);
      p.grid_scale = 0.5f;
    } else {
      p.grid = cb->grid;
      p.grid_n = cb->grid_cells + 1;
      p.grid_cells = static_cast<float>(cb->grid_cells);
      p.grid_scale = cb->grid_scale;
    }
  }
  switch (mode) {
    case kAct: return launch_fast<kAct>(bits, p, st);
    case kWeightLM: return launch_fast<kWeightLM>(bits, p, st);
    case kInt8: return launch_fast<kInt8>(8, p, st);
    default: return launch_fast<kRotate>(8, p, st);
  }
}

// Tokens per CTA so that a CTA has at least 128 threads (one per block).
int tokens_per_cta(int nblk) {
  int G = (128 + nblk - 1) / nblk;
  if (G * nblk > 512) G = 512 / nblk;
  return G < 1 ? 1 : G;
}

int prepare(const rbq_rpbh* r, int mode, int bits, long long rows, const void* X, void* out,
            void* aux, RotqParams* p, const float* fixed_scale = nullptr) {
  const RpbhDevice* rd = nullptr;
  int rc = rpbh_device(r, &rd);
  if (rc != RBQ_OK) return rc;
  p->X = X;
  p->T = rows;
  p->d = r->d;
  p->nblk = r->d / kH;
  p->G = tokens_per_cta(p->nblk);
  p->perm = rd->perm;
  p->sign = rd->sign;
  p->bounds = nullptr;
  p->out = out;
  p->aux = aux;
  p->fixed_scale = fixed_scale;
  p->zero_point = nullptr;
  if ((rc = device_error_word_ptr(&p->err)) != RBQ_OK) return rc;
  if (mode == kAct || mode == kWeightLM) {
    const CodebookDevice* cb = nullptr;
    if ((rc = codebook_device(r->d, bits, &cb)) != RBQ_OK) return rc;
    p->bounds = cb->bounds;
  }
  return RBQ_OK;
}

}  // namespace

// The token-pair kernel (rbq_rotq_pair.cu): BF16 rows, d = 1024..16384 in
// steps of 256.  RBQ_ECONVERGE from the launch means "not this kernel".
bool rotq_pair_eligible(int dtype, int d);
int rotq_pair_launch(const rbq_rpbh* r, int mode, int bits, long long rows, const void* X, void* out, void* aux,
                     cudaStream_t st, const float* fixed_scale = nullptr, uint8_t* zero_point = nullptr);

namespace {

// Per-tensor INT8: the largest per-row scale, written to every entry of the
// row-scale array (one block; rows are few compared with the weight bytes).
__global__ void __launch_bounds__(1024) max_broadcast_kernel(float* scale, int n) {
  __shared__ float part[32];
  float m = 0.f;
  for (int i = threadIdx.x; i < n; i += blockDim.x) m = fmaxf(m, scale[i]);
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x < 32) {
    m = (threadIdx.x < (blockDim.x >> 5)) ? part[threadIdx.x] : 0.f;
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (threadIdx.x == 0) part[0] = m;
  }
  __syncthreads();
  m = part[0];
  for (int i = threadIdx.x; i < n; i += blockDim.x) scale[i] = m;
}

}  // namespace

}  // namespace rbq

using namespace rbq;

extern "C" int rotate_quantize_act(const rbq_rpbh* r, const void* X, int dtype, int T, int bits,
                                   void* codes_out, float* norms_out, void* stream) {
  if (!r || T < 0 || (dtype != RBQ_F32 && dtype != RBQ_BF16)) return RBQ_EINVAL;
  const bool rot = (bits == RBQ_ROTATE_ONLY);
  if (!rot && (bits < 1 || bits > 8)) return RBQ_EINVAL;
  if (T == 0) return RBQ_OK;
  if (!X || !codes_out || (!rot && !norms_out)) return RBQ_EINVAL;
  if (!aligned(X, 16) || !aligned(codes_out, 16) || (norms_out && !aligned(norms_out, 4)))
    return RBQ_EALIGN;
  const int mode = rot ? kRotate : kAct;
  if (rotq_pair_eligible(dtype, r->d)) {
    const int prc = rotq_pair_launch(r, mode, rot ? 8 : bits, T, X, codes_out, norms_out,
                                     static_cast<cudaStream_t>(stream));
    if (prc != RBQ_ECONVERGE) return prc;
  }
  if (fast_eligible(dtype, r->d)) {
    const int frc = run_fast(r, mode, bits, T, X, codes_out, norms_out, static_cast<cudaStream_t>(stream));
    if (frc != RBQ_ECONVERGE) return frc;
  }
  RotqParams p;
  int rc = prepare(r, mode, bits, T, X, codes_out, norms_out, &p);
  if (rc != RBQ_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return rot ? launch_mode<kRotate>(dtype, 8, p, st) : launch_mode<kAct>(dtype, bits, p, st);
}

namespace {

// One rotate-then-quantise pass over the weight rows through the first
// kernel that takes this width (fixed_scale: INT8 with one given scale).
int weights_pass(const rbq_rpbh* r, const void* W, int dtype, int d_out, int m, int bits, void* out, void* aux,
                 cudaStream_t st, const float* fixed_scale) {
  if (rotq_pair_eligible(dtype, r->d)) {
    const int prc = rotq_pair_launch(r, m, bits, d_out, W, out, aux, st, fixed_scale);
    if (prc != RBQ_ECONVERGE) return prc;
  }
  if (fast_eligible(dtype, r->d)) {
    const int frc = run_fast(r, m, bits, d_out, W, out, aux, st, fixed_scale);
    if (frc != RBQ_ECONVERGE) return frc;
  }
  RotqParams p;
  int rc = prepare(r, m, bits, d_out, W, out, aux, &p, fixed_scale);
  if (rc != RBQ_OK) return rc;
  return (m == kWeightLM) ? launch_mode<kWeightLM>(dtype, bits, p, st) : launch_mode<kInt8>(dtype, 8, p, st);
}

}  // namespace

extern "C" int quantize_weights(const rbq_rpbh* r, const void* W, int dtype, int d_out, int mode,
                                int bits, void* codes_or_q, void* rownorm_or_scale, void* stream) {
  if (!r || d_out < 0 || (dtype != RBQ_F32 && dtype != RBQ_BF16)) return RBQ_EINVAL;
  if (mode == RBQ_LLOYDMAX) {
    if (bits < 1 || bits > 8) return RBQ_EINVAL;
  } else if (mode == RBQ_INT8_SYM || mode == RBQ_INT8_TENSOR) {
    if (bits != 8) return RBQ_EINVAL;
  } else {
    return RBQ_EINVAL;
  }
  if (d_out == 0) return RBQ_OK;
  if (!W || !codes_or_q || !rownorm_or_scale) return RBQ_EINVAL;
  if (!aligned(W, 16) || !aligned(codes_or_q, 16) || !aligned(rownorm_or_scale, 4))
    return RBQ_EALIGN;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int m = (mode == RBQ_LLOYDMAX) ? kWeightLM : kInt8;
  int rc = weights_pass(r, W, dtype, d_out, m, bits, codes_or_q, rownorm_or_scale, st, nullptr);
  if (rc != RBQ_OK || mode != RBQ_INT8_TENSOR) return rc;
  // per tensor: the largest row scale, then the rows again with that scale
  float* scale = static_cast<float*>(rownorm_or_scale);
  max_broadcast_kernel<<<1, 1024, 0, st>>>(scale, d_out);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e);
  return weights_pass(r, W, dtype, d_out, kInt8, 8, codes_or_q, rownorm_or_scale, st, scale);
}

extern "C" int quantize_weights_int8_asym(const rbq_rpbh* r, const void* W, int dtype, int d_out, uint8_t* q,
                                          float* scale, uint8_t* zero_point, void* stream) {
  if (!r || d_out < 0 || (dtype != RBQ_F32 && dtype != RBQ_BF16)) return RBQ_EINVAL;
  if (d_out == 0) return RBQ_OK;
  if (!W || !q || !scale || !zero_point) return RBQ_EINVAL;
  if (!aligned(W, 16) || !aligned(q, 16) || !aligned(scale, 4)) return RBQ_EALIGN;
  if (rotq_pair_eligible(dtype, r->d)) {
    const int prc = rotq_pair_launch(r, kInt8Asym, 8, d_out, W, q, scale, static_cast<cudaStream_t>(stream),
                                     nullptr, zero_point);
    if (prc != RBQ_ECONVERGE) return prc;
  }
  RotqParams p;
  int rc = prepare(r, kInt8Asym, 8, d_out, W, q, scale, &p);
  if (rc != RBQ_OK) return rc;
  p.zero_point = zero_point;
  return launch_mode<kInt8Asym>(dtype, 8, p, static_cast<cudaStream_t>(stream));
}
