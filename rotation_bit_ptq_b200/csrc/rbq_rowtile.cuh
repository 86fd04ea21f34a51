// Pieces of the row-tile rotate-then-quantise kernel (token pairs): the tile
// geometry and shared-memory layout, packed fp32x2 arithmetic, the code
// search on the shared-memory grid, the code packing and the launch helpers.
//
//   OrbitQuant (hotelren.com/news/3376620) §2.1-§2.3; INT8-convrot
//   (cloud.baidu.com/article/9430339) §4.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "rbq_internal.h"
#include "rbq_sm100.cuh"

namespace rbq {
namespace rowtile {

using namespace sm100;

enum Mode { kAct = 0, kWeightLM = 1, kInt8 = 2, kRotate = 3, kInt8Asym = 4 };

// A tile holds R = 2P token rows (P token pairs): 16 rows for d <= 3072, and
// 8, 4 or 2 rows for wider rows, so that a double-buffered ring still fits.
constexpr int kMaxRows = 16;
constexpr int kMaxWarps = 12;        // partial-sum columns per token (warps of the CTA)
constexpr size_t kSmemLimit = 227 * 1024;

struct Params {
  const __nv_bfloat16* X;
  long long T;
  int d, nblk, nwarps;               // warps of the CTA
  int ntiles;                        // ceil(T / R)
  int NS;                            // ring slots
  uint32_t pitch;                    // bytes per staged row (2d + 16)
  const void* tab;                   // d entries: source byte offset | sign in the top bit, 32-bit
                                     // (pair_tab_slot order) or 16-bit (pair_tab16_slot order)
  const float2* grid;                // Lloyd-Max modes: the code grid as copied into shared memory
  int grid_entries;                  // entries copied (even: one 16-byte-multiple bulk copy)
  int grid_first;                    // index of cell 0 among them (guard entries before it)
  float grid_cells, grid_scale;      // cells, 1 / (2R)
  void* out;
  void* aux;
  unsigned int* err;
  const float* fixed_scale;          // INT8: one scale for every row (not written back), else null
  uint8_t* zero_point;               // asymmetric INT8: one per row
  int st256;                         // output rows 32-byte aligned: 32-byte stores allowed
};

// Shared-memory layout (bytes from the 128-aligned base).
struct Layout {
  uint32_t ring, off, grid, part, bars, total;
};

// tab_bytes: bytes per gather-table entry (4, or 2 for the 16-bit table);
// nparts: partial-result arrays (2 for the asymmetric INT8 mode: max and min).
__host__ __device__ inline Layout layout(int d, int NS, int grid_entries, int R, int tab_bytes, int nparts) {
  Layout L{};
  const uint32_t pitch = 2u * d + 16u;
  L.ring = 0;
  L.off = L.ring + NS * R * pitch;
  L.grid = L.off + static_cast<uint32_t>(tab_bytes) * d;
  L.part = (L.grid + 8u * grid_entries + 15u) & ~15u;
  L.bars = L.part + 4u * nparts * (2 * NS) * R * kMaxWarps;   // nparts x [2NS][R tokens][12 warps]
  L.bars = (L.bars + 7u) & ~7u;
  // full[NS], red[2NS], tab | TMEM base
  L.total = L.bars + 8u * (NS + 2 * NS + 1) + 8u;
  return L;
}

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
__device__ __forceinline__ unsigned long long fma2(unsigned long long a, unsigned long long b, unsigned long long c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ unsigned long long mul2(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
// 0xFFFFFFFF if a >= b else 0 (IEEE: -0 >= -0; NaN never)
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
__device__ __forceinline__ float2 lds_f2(uint32_t addr) {
  float2 v;
  asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr));
  return v;
}
__device__ __forceinline__ float lds_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ void sts_f32(uint32_t addr, float v) {
  asm volatile("st.shared.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}
// Whole contiguous row, global -> shared, completion counted in bytes on `bar`.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}
// bf16 bits (low 16 of u) -> fp32 with the sign word S (0 or 0x80000000)
// folded in: (u << 16) + S flips the sign bit exactly when S is set.
__device__ __forceinline__ float bf16_signed(uint32_t u, uint32_t S) { return __uint_as_float(u * 65536u + S); }


__device__ __forceinline__ unsigned long long pk_u(uint32_t a, uint32_t b) {
  return pk(__uint_as_float(a), __uint_as_float(b));
}
__device__ __forceinline__ void upk_u(unsigned long long r, uint32_t& a, uint32_t& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=r"(a), "=r"(b) : "l"(r));
}
__device__ __forceinline__ uint32_t bf2_bits(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Code of each half of a packed pair z (two tokens) from the shared-memory
// grid over [-R, R] (every cell holds at most one boundary): u = sat(v/(2R) +
// 1/2), n = round(u * cells) through the +2^23 trick, and the cell's entry
// {boundary or +inf, count of boundaries below the cell} gives code = count +
// (v >= boundary), the compare taken as the sign of z*inv - boundary.  Values
// beyond +-R saturate into the end cells, whose entries cover them.  Measured
// alternatives: a grid over all of [-1, 1] needs no clamp but is 20x larger
// and its lookups cost more shared-memory wavefronts than the clamp costs
// arithmetic (2-5 % slower for 2-4 bits); a grid over |v| with a negative v's
// code mirrored fits 128 bytes at 4 bits, so its lookups never conflict, but
// its extra compare and XOR per value cost 7 %; v for both tokens in one
// packed multiply with the cell index from it cost 2 %.
struct Enc {
  float A0, A1, inv0, inv1, cells;
  uint32_t gbase;
#ifdef RBQ_DEBUG
  unsigned int* dbg_err = nullptr;     // debug builds: check every grid entry index
  uint32_t dbg_entries = 0;
  uint32_t dbg_first = 0;
#endif
  __device__ __forceinline__ Enc(float i0, float i1, float nc, float scale, uint32_t gb)
      : A0(i0 * scale), A1(i1 * scale), inv0(i0), inv1(i1), cells(nc), gbase(gb) {}
  // Shared-memory address of the entry for the rounded grid coordinate qf
  // (2^23 + n in the float's low bits; gbase already holds -2^23 entries and
  // the guard entries before entry 0).
  __device__ __forceinline__ uint32_t entry_addr(float qf) const {
#ifdef RBQ_DEBUG
    const uint32_t e = __float_as_uint(qf) - 0x4B000000u + dbg_first;
    return gbase + (0x4B000000u - dbg_first) * 8u + 8u * dbg_index(e, dbg_entries, dbg_err);
#else
    return gbase + __float_as_uint(qf) * 8u;
#endif
  }
  __device__ __forceinline__ void codes(unsigned long long z, uint32_t& c0, uint32_t& c1) const {
    float z0, z1;
    upk(z, z0, z1);
    const float qf0 = fmaf(fma_sat(z0, A0, 0.5f), cells, 8388608.0f);
    const float qf1 = fmaf(fma_sat(z1, A1, 0.5f), cells, 8388608.0f);
    const float2 e0 = lds_f2(entry_addr(qf0));
    const float2 e1 = lds_f2(entry_addr(qf1));
    const int below0 = __float_as_int(fmaf(z0, inv0, -e0.x)) >> 31;
    const int below1 = __float_as_int(fmaf(z1, inv1, -e1.x)) >> 31;
    c0 = static_cast<uint32_t>(__float_as_int(e0.y) + 1 + below0);
    c1 = static_cast<uint32_t>(__float_as_int(e1.y) + 1 + below1);
  }
};

// Packs `code` (already < 2^BITS) into bit i*BITS of the word array w.
template <int BITS>
__device__ __forceinline__ void put_code(uint32_t* w, int i, uint32_t code) {
  const int bit = i * BITS, wi = bit >> 5, sh = bit & 31;
  if constexpr ((32 % BITS) == 0) {
    w[wi] += code << sh;                     // disjoint fields: add = or
  } else {
    w[wi] |= code << sh;
    if (sh + BITS > 32) w[wi + 1] |= code >> (32 - sh);
  }
}

// 32 bytes (eight words) to global memory in one streaming store; dst must be
// 32-byte aligned.
__device__ __forceinline__ void st_v8_cs(void* dst, const uint32_t* w) {
  asm volatile("st.global.cs.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(dst), "r"(w[0]), "r"(w[1]),
               "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
               : "memory");
}

// One block's codes (8*BITS bytes) of one row.  wide: dst is 32-byte aligned,
// so 4- and 8-bit codes go out as 32-byte stores -- the four lanes of a warp
// that hold one row's consecutive blocks then write whole 128-byte lines.
template <int BITS>
__device__ __forceinline__ void store_codes(unsigned char* dst, const uint32_t* w, bool wide = false) {
  if constexpr ((BITS % 4) == 0) {
    if (wide) {
#pragma unroll
      for (int i = 0; i < BITS / 4; ++i) st_v8_cs(dst + 32 * i, w + 8 * i);
      return;
    }
  }
  if constexpr ((BITS % 2) == 0) {
#pragma unroll
    for (int i = 0; i < BITS / 2; ++i)
      __stcs(reinterpret_cast<uint4*>(dst) + i, make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]));
  } else {
#pragma unroll
    for (int i = 0; i < BITS; ++i) __stcs(reinterpret_cast<uint2*>(dst) + i, make_uint2(w[2 * i], w[2 * i + 1]));
  }
}


// ---- host side ----------------------------------------------------------------

inline int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

// Most ring slots of R-row tiles that fit next to the tables (at least 2, at
// most 6), or 0.
inline int slots_that_fit(int d, int grid_entries, int R, int tab_bytes, int nparts) {
  int best = 0;
  for (int ns = 2; ns <= 6; ++ns)
    if (layout(d, ns, grid_entries, R, tab_bytes, nparts).total + 128 <= kSmemLimit) best = ns;
  return best;
}

// Launch with programmatic dependent launch allowed: the kernel may start
// while the previous launch on the stream finishes; it calls griddep_wait()
// before reading anything that launch may have written.
template <typename Kern>
inline int launch_pdl(Kern kern, int grid, int threads, size_t smem, cudaStream_t st, const Params& p) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(threads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, p);
  if (e == cudaSuccess) e = cudaGetLastError();
  return e == cudaSuccess ? RBQ_OK : cuda_fail(e);
}

}  // namespace rowtile
}  // namespace rbq
