// The rotation fused into the matmul that produces its input.
//
//   OrbitQuant (hotelren.com/news/3376620) §6.2 ("performance below
//   expectations") points at fusing the rotation with the matrix-multiply
//   kernels to cut memory traffic; §2.3 defines Pi_d = blkdiag(H_64 D) P_pi.
//
// The next layer's input is x = act(y), y = the producing W8A16 layer's output
// (INT8-convrot §4).  Its rotation gathers x by pi across the whole row, which
// no output tile of the producing GEMM holds -- but the gather can be moved
// offline: with the producing layer's weight rows (and their per-row scales)
// stored in the order of pi, its output column k is y_{pi(k)}, so every 64
// consecutive output columns are the inputs of one block of the next layer's
// rotation, and the GEMM's epilogue finishes it: x'[64b + r] =
// (1/8) sum_i H[r][i] D_{64b+i} act(y_{pi(64b+i)}).  The BF16 y never goes to
// memory and no separate rotation pass runs; the weights are the same INT8
// values and scales, reordered once.
//
// rpbh_gather_rows does the offline reordering (row k of dst = row pi(k) of
// src), and qlinear_int8_rotate_next is the fused layer.
//
// The same for the code layer (OrbitQuant §2.2, y = s_m r'_n sum C_w C_a):
// qlinear_rotate_next writes the next layer's rotated input x' (BF16), and
// quantize_rotated finishes that layer's quantiser -- §2.2 steps 2-4, the
// norm and the Lloyd-Max codes -- on the rotated rows: a light, HBM-bound
// pass with no gather and no butterfly (the step the pages' fusion removes).

#include <cuda_runtime.h>

#include "rbq_internal.h"
#include "rbq_rowtile.cuh"

namespace rbq {
int qlinear_int8_fast_launch(const uint16_t* Xrot, const int8_t* Wq, const float* scale, int M, int N, int K,
                             uint16_t* Y, unsigned int* err, cudaStream_t st, const uint8_t* zero_point,
                             const float* next_sign, int act);
bool qlinear_int8_fast_eligible(int M, int N, int K);
bool qlinear_fast_eligible(int M, int N, int K, int bits_a, int bits_w);
int qlinear_rotate_next_launch(const uint8_t* a_codes, const float* s, int bits_a, const uint8_t* w_codes,
                               const uint16_t* rnorm, int bits_w, int M, int N, int K, uint16_t* Y,
                               const CodebookDevice* ca, const CodebookDevice* cw, unsigned int* err,
                               cudaStream_t st, const float* next_sign, int act);

namespace {

struct QRParams {
  const uint16_t* X;          // BF16 [T, d], rotated rows
  long long T;
  int d;
  const float2* grid;         // the guarded code grid (see CodebookDevice::grid_pad)
  int grid_entries, grid_first;
  float grid_cells, grid_scale;
  uint8_t* codes;             // [T, d*BITS/8]
  float* norms;               // [T]
  unsigned int* err;
  int NS;                     // ring slots
};

// One warp per row, the rows staged in shared memory: a persistent block
// per SM of W warps, each owning S row slots (W x S rows of 2d bytes, about
// 200 KB: 32 rows at d = 3072, 8 at d = 12288), so that many rows per SM are
// in flight at once without any barrier across warps.  Lane 0 of a warp
// brings each of its rows (warp g of the grid takes rows g, g + G, ...) by one
// bulk asynchronous copy, counted on the slot's mbarrier.  For a row: lane i
// sums the squares of its 16-byte chunks i, i + 32, ... (shuffles give every
// lane the same total, s); then re-reads them and encodes each chunk's 8
// values -- v = x' / (s + eps) on the shared-memory grid, as the
// rotate-quantise kernels do -- into BITS bytes at the chunk's place in the
// packed row; the slot then takes the warp's row S steps ahead.  A row whose
// norm is not finite is encoded as the zero vector.
constexpr int kQRMaxWarps = 16;

struct QRLayout {
  uint32_t ring, grid, bars, total;
};
__host__ __device__ inline QRLayout qr_layout(int d, int slots, int grid_entries) {
  QRLayout L{};
  L.ring = 0;                                          // slots x 2d bytes (2d is a multiple of 128)
  L.grid = L.ring + static_cast<uint32_t>(slots) * 2u * d;
  L.bars = (L.grid + 8u * grid_entries + 7u) & ~7u;    // one mbarrier per slot
  L.total = L.bars + 8u * slots;
  return L;
}

template <int BITS>
__global__ void __launch_bounds__(kQRMaxWarps * 32, 1) quantize_rotated_kernel(const QRParams p) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  const uint32_t sraw = rowtile::smem_u32(smem_raw);
  const uint32_t sbase = (sraw + 127u) & ~127u;
  unsigned char* sm = smem_raw + (sbase - sraw);
  const int W = blockDim.x >> 5, S = p.NS;                 // warps, slots per warp
  const QRLayout L = qr_layout(p.d, W * S, p.grid_entries);
  float2* g = reinterpret_cast<float2*>(sm + L.grid);
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + L.bars);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t row_bytes = 2u * static_cast<uint32_t>(p.d);
  const int chunks = p.d / 8;

  for (int i = threadIdx.x; i < p.grid_entries; i += blockDim.x) g[i] = p.grid[i];
  if (threadIdx.x == 0) {
    for (int k = 0; k < W * S; ++k) rowtile::mbar_init(&full[k], 1);
    rowtile::mbar_fence_init();
  }
  __syncthreads();
  const long long G = static_cast<long long>(gridDim.x) * W;            // warps in the grid
  const long long first = static_cast<long long>(blockIdx.x) * W + warp;
  auto issue = [&](long long t, int k) {                // lane 0 only; slot k of this warp
    if (t < p.T) {
      uint64_t* bar = &full[warp * S + k];
      rowtile::mbar_arrive_expect_tx(bar, row_bytes);
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      rowtile::bulk_load(sbase + L.ring + (warp * S + k) * row_bytes, p.X + t * p.d, row_bytes, bar);
    }
  };
  if (lane == 0)
    for (int k = 0; k < S; ++k) issue(first + k * G, k);
  const uint32_t gbase = sbase + L.grid + 8u * static_cast<uint32_t>(p.grid_first) - 0x4B000000u * 8u;

  bool ok = true;
  int it = 0;
  for (long long t = first; t < p.T; t += G, ++it) {
    const int k = it % S;
    if (__any_sync(0xffffffffu, !rowtile::mbar_wait(&full[warp * S + k], (it / S) & 1))) {
      ok = false;
      break;
    }
    const uint32_t rbase = sbase + L.ring + (warp * S + k) * row_bytes;
    float acc = 0.f;
#pragma unroll 4
    for (int c = lane; c < chunks; c += 32) {
      const uint4 v = rowtile::lds128(rbase + 16u * c);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float a = __uint_as_float(w[j] << 16), b = __uint_as_float(w[j] & 0xFFFF0000u);
        acc = fmaf(a, a, acc);
        acc = fmaf(b, b, acc);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    const float s = sqrtf(acc);
    const bool bad = !(acc < INFINITY);             // the same in every lane
    const float inv = bad ? 0.f : 1.0f / (s + 1e-12f);
    rowtile::Enc enc(inv, inv, p.grid_cells, p.grid_scale, gbase);
#ifdef RBQ_DEBUG
    enc.dbg_err = p.err;
    enc.dbg_entries = static_cast<uint32_t>(p.grid_entries);
    enc.dbg_first = static_cast<uint32_t>(p.grid_first);
#endif
    uint8_t* out = p.codes + t * (static_cast<long long>(p.d) * BITS / 8);
    // four chunks per step: their 32 grid lookups are independent, so more of
    // the shared-memory latency overlaps
#pragma unroll 4
    for (int c = lane; c < chunks; c += 32) {
      const uint4 v = rowtile::lds128(rbase + 16u * c);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
      uint32_t pw[2] = {0u, 0u};                    // the chunk's 8 codes, LSB first (8*BITS bits)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float a = bad ? 0.f : __uint_as_float(w[j] << 16);
        const float b = bad ? 0.f : __uint_as_float(w[j] & 0xFFFF0000u);
        uint32_t c0, c1;
        enc.codes(rowtile::pk(a, b), c0, c1);
        rowtile::put_code<BITS>(pw, 2 * j, c0);
        rowtile::put_code<BITS>(pw, 2 * j + 1, c1);
      }
      unsigned char* dst = out + static_cast<long long>(c) * BITS;
      if constexpr (BITS == 8) {
        __stcs(reinterpret_cast<uint2*>(dst), make_uint2(pw[0], pw[1]));
      } else if constexpr (BITS == 4) {
        __stcs(reinterpret_cast<unsigned int*>(dst), pw[0]);
      } else if constexpr (BITS == 2) {
        __stcs(reinterpret_cast<unsigned short*>(dst), static_cast<unsigned short>(pw[0]));
      } else {
#pragma unroll
        for (int q = 0; q < BITS; ++q) dst[q] = static_cast<unsigned char>(pw[q >> 2] >> (8 * (q & 3)));
      }
    }
    if (lane == 0) p.norms[t] = s;
    __syncwarp();                                   // every lane's reads of the slot are done
    if (lane == 0) issue(t + S * G, k);
  }
  if (!ok) {
    // a timed-out wait: copies may still be landing; let them finish before
    // the block's shared memory is released
    if (lane == 0) atomicOr(p.err, 512u);
    const long long t0 = clock64();
    while (clock64() - t0 < 40000) {
    }
  }
}

// Warps per block and row slots per warp: S = 2 while 16 warps x 2 rows fit
// in about 200 KB next to the grid, else one slot per warp and as many warps
// (at most 16) as rows fit; 0 warps when not even one row fits.
inline void qr_geometry(int d, int grid_entries, int* warps, int* slots) {
  const long long budget = rowtile::kSmemLimit - 128 - 8LL * grid_entries - 8LL * 2 * kQRMaxWarps - 64;
  const long long rows = budget / (2LL * d);
  *slots = rows >= 2LL * kQRMaxWarps ? 2 : 1;
  const long long w = rows / *slots;
  *warps = static_cast<int>(w > kQRMaxWarps ? kQRMaxWarps : w);
}

template <int BITS>
int launch_quantize_rotated(QRParams p, cudaStream_t st) {
  int warps = 0;
  qr_geometry(p.d, p.grid_entries, &warps, &p.NS);
  if (warps < 1) return RBQ_EINVAL;
  const size_t smem = qr_layout(p.d, warps * p.NS, p.grid_entries).total + 128;
  if (smem > rowtile::kSmemLimit) return RBQ_EINVAL;
  auto kern = quantize_rotated_kernel<BITS>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return cuda_fail(e);
  const int sms = rowtile::sm_count();
  const long long need = (p.T + warps - 1) / warps;
  const int grid = static_cast<int>(need < sms ? need : sms);
  kern<<<grid, warps * 32, smem, st>>>(p);
  e = cudaGetLastError();
  return e == cudaSuccess ? RBQ_OK : cuda_fail(e);
}

// dst row k = src row perm[k]; one CTA per row, 16-byte vectors when the row
// and both bases allow it.
__global__ void __launch_bounds__(256) gather_rows_kernel(const unsigned char* src, unsigned char* dst,
                                                           const int32_t* perm, long long row_bytes, bool vec16) {
  const long long k = blockIdx.x;
  const unsigned char* s = src + static_cast<long long>(perm[k]) * row_bytes;
  unsigned char* d = dst + k * row_bytes;
  if (vec16) {
    const uint4* s4 = reinterpret_cast<const uint4*>(s);
    uint4* d4 = reinterpret_cast<uint4*>(d);
    for (long long i = threadIdx.x; i < row_bytes / 16; i += blockDim.x) d4[i] = s4[i];
  } else {
    for (long long i = threadIdx.x; i < row_bytes; i += blockDim.x) d[i] = s[i];
  }
}

}  // namespace
}  // namespace rbq

using namespace rbq;

extern "C" int rpbh_gather_rows(const rbq_rpbh* r, const void* src, long long row_bytes, void* dst, void* stream) {
  if (!r || !src || !dst || row_bytes <= 0) return RBQ_EINVAL;
  if (src == dst) return RBQ_EINVAL;
  const RpbhDevice* rd = nullptr;
  int rc = rpbh_device(r, &rd);
  if (rc != RBQ_OK) return rc;
  const bool vec16 = (row_bytes % 16) == 0 && aligned(src, 16) && aligned(dst, 16);
  gather_rows_kernel<<<r->d, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const unsigned char*>(src), static_cast<unsigned char*>(dst), rd->perm, row_bytes, vec16);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? RBQ_OK : cuda_fail(e);
}

extern "C" int qlinear_int8_rotate_next(const uint16_t* Xrot, const int8_t* Wq_next_order,
                                        const float* scale_next_order, int M, int K, const rbq_rpbh* next,
                                        int activation, uint16_t* Xrot_next, void* stream) {
  if (!next || M < 0 || K <= 0 || K % kH || K > kMaxD) return RBQ_EINVAL;
  if (activation != RBQ_ACT_NONE && activation != RBQ_ACT_GELU) return RBQ_EINVAL;
  const int N = next->d;
  if (M == 0) return RBQ_OK;
  if (!Xrot || !Wq_next_order || !scale_next_order || !Xrot_next) return RBQ_EINVAL;
  if (!qlinear_int8_fast_eligible(M, N, K)) return RBQ_EINVAL;
  if (!aligned(Xrot, 16) || !aligned(Wq_next_order, 16) || !aligned(Xrot_next, 16) || !aligned(scale_next_order, 4))
    return RBQ_EALIGN;
  const RpbhDevice* rd = nullptr;
  int rc = rpbh_device(next, &rd);
  if (rc != RBQ_OK) return rc;
  unsigned int* err = nullptr;
  if ((rc = device_error_word_ptr(&err)) != RBQ_OK) return rc;
  return qlinear_int8_fast_launch(Xrot, Wq_next_order, scale_next_order, M, N, K, Xrot_next, err,
                                  static_cast<cudaStream_t>(stream), nullptr, rd->sign, activation);
}

extern "C" int qlinear_rotate_next(const uint8_t* a_codes, const float* s, int bits_a,
                                   const uint8_t* w_codes_next_order, const uint16_t* rnorm_next_order, int bits_w,
                                   int M, int K, const rbq_rpbh* next, int activation, uint16_t* Xrot_next,
                                   void* stream) {
  if (!next || M < 0 || K <= 0 || K % kH || K > kMaxD) return RBQ_EINVAL;
  if (bits_a < 1 || bits_a > 8 || bits_w < 1 || bits_w > 8) return RBQ_EINVAL;
  if (activation != RBQ_ACT_NONE && activation != RBQ_ACT_GELU) return RBQ_EINVAL;
  const int N = next->d;
  if (M == 0) return RBQ_OK;
  if (!a_codes || !s || !w_codes_next_order || !rnorm_next_order || !Xrot_next) return RBQ_EINVAL;
  if (!qlinear_fast_eligible(M, N, K, bits_a, bits_w)) return RBQ_EINVAL;
  if (!aligned(a_codes, 16) || !aligned(w_codes_next_order, 16) || !aligned(Xrot_next, 16) || !aligned(s, 4) ||
      !aligned(rnorm_next_order, 4))
    return RBQ_EALIGN;
  const CodebookDevice *ca = nullptr, *cw = nullptr;
  int rc = codebook_device(K, bits_a, &ca);
  if (rc != RBQ_OK) return rc;
  if ((rc = codebook_device(K, bits_w, &cw)) != RBQ_OK) return rc;
  const RpbhDevice* rd = nullptr;
  if ((rc = rpbh_device(next, &rd)) != RBQ_OK) return rc;
  unsigned int* err = nullptr;
  if ((rc = device_error_word_ptr(&err)) != RBQ_OK) return rc;
  return qlinear_rotate_next_launch(a_codes, s, bits_a, w_codes_next_order, rnorm_next_order, bits_w, M, N, K,
                                    Xrot_next, ca, cw, err, static_cast<cudaStream_t>(stream), rd->sign, activation);
}

extern "C" int quantize_rotated(const void* Xrot, int dtype, int T, int d, int bits, void* codes_out,
                                float* norms_out, void* stream) {
  if (dtype != RBQ_BF16 || T < 0 || d <= 0 || d % kH || d > kMaxD || bits < 1 || bits > 8) return RBQ_EINVAL;
  if (T == 0) return RBQ_OK;
  if (!Xrot || !codes_out || !norms_out) return RBQ_EINVAL;
  if (!aligned(Xrot, 16) || !aligned(codes_out, 8) || !aligned(norms_out, 4)) return RBQ_EALIGN;
  const CodebookDevice* cb = nullptr;
  int rc = codebook_device(d, bits, &cb);
  if (rc != RBQ_OK) return rc;
  QRParams p{};
  p.X = static_cast<const uint16_t*>(Xrot);
  p.T = T;
  p.d = d;
  p.grid = cb->grid_pad;
  p.grid_entries = guarded_grid_entries(cb->grid_cells + 1);
  p.grid_first = kGridGuard;
  p.grid_cells = static_cast<float>(cb->grid_cells);
  p.grid_scale = cb->grid_scale;
  p.codes = static_cast<uint8_t*>(codes_out);
  p.norms = norms_out;
  if ((rc = device_error_word_ptr(&p.err)) != RBQ_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  switch (bits) {
    case 1: return launch_quantize_rotated<1>(p, st);
    case 2: return launch_quantize_rotated<2>(p, st);
    case 3: return launch_quantize_rotated<3>(p, st);
    case 4: return launch_quantize_rotated<4>(p, st);
    case 5: return launch_quantize_rotated<5>(p, st);
    case 6: return launch_quantize_rotated<6>(p, st);
    case 7: return launch_quantize_rotated<7>(p, st);
    default: return launch_quantize_rotated<8>(p, st);
  }
}
