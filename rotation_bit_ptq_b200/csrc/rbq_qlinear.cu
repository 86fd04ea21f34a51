// Quantised linear layers on the 5th-generation tensor cores (tcgen05).
//
//   qlinear       OrbitQuant (hotelren.com/news/3376620) §2.2: with the
//                 rotation absorbed into the weights (§2.1) it cancels, and
//                 y[m,n] = s_m r'_n sum_k C_w[q_nk] C_a[p_mk].
//   qlinear_int8  INT8-convrot (cloud.baidu.com/article/9430339) §4, W8A16:
//                 y[m,n] = scale_n sum_k q_nk x'_mk.
//
// Design: a CTA owns a 128 x 128 output tile whose fp32 accumulator lives in
// tensor memory (128 lanes x 128 columns).  For each 64-wide K slice every
// thread expands one row of A and one row of B into fp16 (qlinear, levels
// scaled by sqrt(K) so they sit near unit size) or bf16 (INT8 path) operand
// tiles in shared memory, in the 128-byte-swizzled K-major layout the tensor
// core reads; one thread then issues four 128x128x16 MMAs and commits them to
// an mbarrier.  Two stages let the expansion of slice k+1 overlap the MMAs of
// slice k.  The epilogue reads TMEM back (one row per thread), applies
// s_m r'_n / K (or scale_n), rounds to BF16 and stores.

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "rbq_internal.h"
#include "rbq_sm100.cuh"

namespace rbq {
namespace {

using namespace sm100;

constexpr int kBM = 128, kBN = 128, kBK = 64, kStages = 2;
constexpr int kTileBytes = kBM * kBK * 2;    // 16 KB per operand tile

struct QParams {
  const uint8_t* A;
  const uint8_t* B;
  long long a_pitch, b_pitch;   // bytes per row
  int M, N, K;
  int bits_a, bits_b;
  const uint16_t* lut_a;        // fp16 level tables (qlinear)
  const uint16_t* lut_b;
  const float* s;               // qlinear: per-row norms
  const uint16_t* rnorm;        // qlinear: BF16 per-column norms
  const float* scale;           // int8: per-column scales
  float inv_k;
  uint16_t* Y;
  unsigned int* err;
};

struct __align__(8) SmemTail {
  uint64_t bar[kStages];
  uint64_t drain;                  // abort path only: completion of the MMAs issued
  uint32_t tmem_slot;
  uint32_t pad;
  uint16_t lut_a[256];
  uint16_t lut_b[256];
};

constexpr size_t kSmemBytes = 1024 + 2 * kStages * kTileBytes + sizeof(SmemTail);

// One 64-code row slice of a packed code row -> 8 swizzled 16-byte chunks.
__device__ __forceinline__ void expand_codes_row(const uint8_t* src, int bits, const uint16_t* lut,
                                                 uint8_t* tile, int r, bool valid) {
  uint32_t w[17];
  if (valid) {
    const uint2* s2 = reinterpret_cast<const uint2*>(src);
    for (int i = 0; i < bits; ++i) {
      const uint2 v = __ldg(s2 + i);
      w[2 * i] = v.x;
      w[2 * i + 1] = v.y;
    }
  } else {
    for (int i = 0; i < 2 * bits; ++i) w[i] = 0u;
  }
  w[2 * bits] = 0u;
  const uint32_t mask = (1u << bits) - 1u;
  for (int c = 0; c < 8; ++c) {
    uint32_t h[4];
    for (int j = 0; j < 4; ++j) {
      uint32_t pair = 0u;
      for (int e = 0; e < 2; ++e) {
        const int i = 8 * c + 2 * j + e;
        const int bit = i * bits, wi = bit >> 5, sh = bit & 31;
        const uint64_t win = (static_cast<uint64_t>(w[wi + 1]) << 32) | w[wi];
        const uint32_t code = static_cast<uint32_t>(win >> sh) & mask;
        const uint32_t v = valid ? lut[code] : 0u;
        pair |= v << (16 * e);
      }
      h[j] = pair;
    }
    *reinterpret_cast<uint4*>(tile + sw128_offset(r, c)) = make_uint4(h[0], h[1], h[2], h[3]);
  }
}

// 64 BF16 values -> 8 swizzled chunks (plain copy).
__device__ __forceinline__ void copy_bf16_row(const uint8_t* src, uint8_t* tile, int r, bool valid) {
  const uint4* s4 = reinterpret_cast<const uint4*>(src);
  for (int c = 0; c < 8; ++c) {
    const uint4 v = valid ? __ldg(s4 + c) : make_uint4(0, 0, 0, 0);
    *reinterpret_cast<uint4*>(tile + sw128_offset(r, c)) = v;
  }
}

// 64 int8 values -> 64 exact BF16 values -> 8 swizzled chunks.
__device__ __forceinline__ void expand_int8_row(const uint8_t* src, uint8_t* tile, int r, bool valid) {
  const uint4* s4 = reinterpret_cast<const uint4*>(src);
  for (int q = 0; q < 4; ++q) {
    const uint4 v = valid ? __ldg(s4 + q) : make_uint4(0, 0, 0, 0);
    const uint32_t word[4] = {v.x, v.y, v.z, v.w};
    for (int half = 0; half < 2; ++half) {
      uint32_t h[4];
      for (int j = 0; j < 4; ++j) {
        const uint32_t wd = word[2 * half + (j >> 1)];
        const int b0 = static_cast<int8_t>((wd >> (16 * (j & 1))) & 0xFF);
        const int b1 = static_cast<int8_t>((wd >> (16 * (j & 1) + 8)) & 0xFF);
        const __nv_bfloat162 pr = __floats2bfloat162_rn(static_cast<float>(b0), static_cast<float>(b1));
        h[j] = *reinterpret_cast<const uint32_t*>(&pr);
      }
      *reinterpret_cast<uint4*>(tile + sw128_offset(r, 2 * q + half)) = make_uint4(h[0], h[1], h[2], h[3]);
    }
  }
}

template <bool kInt8>
__global__ void __launch_bounds__(128, 1) qgemm_kernel(QParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* sm = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  SmemTail* tail = reinterpret_cast<SmemTail*>(sm + 2 * kStages * kTileBytes);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int m0 = blockIdx.y * kBM, n0 = blockIdx.x * kBN;

  if (!kInt8) {
    for (int i = tid; i < 256; i += 128) {
      tail->lut_a[i] = (i < (1 << p.bits_a)) ? p.lut_a[i] : 0;
      tail->lut_b[i] = (i < (1 << p.bits_b)) ? p.lut_b[i] : 0;
    }
  }
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(&tail->bar[s], 1);
    mbar_init(&tail->drain, 1);
    mbar_fence_init();
  }
  if (warp == 0) {
    tmem_alloc(&tail->tmem_slot, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tail->tmem_slot;

  constexpr uint32_t kIdesc = idesc_f16(kBM, kBN, kInt8);
  const int KT = p.K / kBK;
  const int mrow = m0 + tid, nrow = n0 + tid;
  const bool mvalid = mrow < p.M, nvalid = nrow < p.N;
  bool ok = true;

  for (int kt = 0; kt < KT; ++kt) {
    const int st = kt % kStages;
    if (kt >= kStages) ok = ok && mbar_wait(&tail->bar[st], ((kt / kStages) - 1) & 1);
    if (!__syncthreads_and(ok)) { ok = false; break; }
    uint8_t* tA = sm + st * 2 * kTileBytes;
    uint8_t* tB = tA + kTileBytes;
    if (kInt8) {
      copy_bf16_row(p.A + (mvalid ? mrow : 0) * p.a_pitch + kt * 128, tA, tid, mvalid);
      expand_int8_row(p.B + (nvalid ? nrow : 0) * p.b_pitch + kt * 64, tB, tid, nvalid);
    } else {
      expand_codes_row(p.A + (mvalid ? mrow : 0) * p.a_pitch + kt * 8 * p.bits_a, p.bits_a, tail->lut_a, tA,
                       tid, mvalid);
      expand_codes_row(p.B + (nvalid ? nrow : 0) * p.b_pitch + kt * 8 * p.bits_b, p.bits_b, tail->lut_b, tB,
                       tid, nvalid);
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      const uint32_t a0 = smem_u32(tA), b0 = smem_u32(tB);
#pragma unroll
      for (int k = 0; k < kBK / 16; ++k)
        umma_f16(tmem, sdesc_k_sw128(a0 + 32 * k), sdesc_k_sw128(b0 + 32 * k), kIdesc, (kt | k) != 0);
      umma_commit(&tail->bar[st]);
    }
  }
  if (ok && KT > 0) ok = mbar_wait(&tail->bar[(KT - 1) % kStages], ((KT - 1) / kStages) & 1);
  ok = __syncthreads_and(ok);
  tc_fence_after();

  if (ok) {
    const int r = 32 * warp + lane;
    const int m = m0 + r;
    const float rs = kInt8 ? 1.0f : (m < p.M ? p.s[m] * p.inv_k : 0.f);
#pragma unroll 1
    for (int cc = 0; cc < kBN / 32; ++cc) {
      uint32_t v[32];
      tmem_ld32(tmem + (static_cast<uint32_t>(32 * warp) << 16) + 32 * cc, v);
      tmem_wait_ld();
      const int nb = n0 + 32 * cc;
      if (m >= p.M) continue;
      uint16_t* dst = p.Y + static_cast<long long>(m) * p.N + nb;
      if (nb + 32 <= p.N) {
        uint32_t packed[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          float f0 = __uint_as_float(v[2 * j]), f1 = __uint_as_float(v[2 * j + 1]);
          if (kInt8) {
            f0 *= p.scale[nb + 2 * j];
            f1 *= p.scale[nb + 2 * j + 1];
          } else {
            f0 *= rs * __bfloat162float(__ushort_as_bfloat16(p.rnorm[nb + 2 * j]));
            f1 *= rs * __bfloat162float(__ushort_as_bfloat16(p.rnorm[nb + 2 * j + 1]));
          }
          const __nv_bfloat162 h = __floats2bfloat162_rn(f0, f1);
          packed[j] = *reinterpret_cast<const uint32_t*>(&h);
        }
        uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
        for (int j = 0; j < 4; ++j)
          d4[j] = make_uint4(packed[4 * j], packed[4 * j + 1], packed[4 * j + 2], packed[4 * j + 3]);
      } else {
        for (int j = 0; j < 32 && nb + j < p.N; ++j) {
          float f = __uint_as_float(v[j]);
          f *= kInt8 ? p.scale[nb + j] : rs * __bfloat162float(__ushort_as_bfloat16(p.rnorm[nb + j]));
          dst[j] = __bfloat16_as_ushort(__float2bfloat16_rn(f));
        }
      }
    }
  } else {
    if (tid == 0) atomicOr(p.err, 1u);
    drain_after_abort(tid == 0, &tail->drain);    // `ok` is the same in every thread
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 128);
}

template <bool kInt8>
int launch_qgemm(const QParams& p, cudaStream_t st) {
  auto kern = qgemm_kernel<kInt8>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kSmemBytes));
  if (e != cudaSuccess) return cuda_fail(e);
  dim3 grid((p.N + kBN - 1) / kBN, (p.M + kBM - 1) / kBM);
  kern<<<grid, 128, kSmemBytes, st>>>(p);
  e = cudaGetLastError();
  return e == cudaSuccess ? RBQ_OK : cuda_fail(e);
}

}  // namespace
}  // namespace rbq

namespace rbq {
bool qlinear_int8_fast_eligible(int M, int N, int K);
int qlinear_int8_fast_launch(const uint16_t* Xrot, const int8_t* Wq, const float* scale, int M, int N, int K,
                             uint16_t* Y, unsigned int* err, cudaStream_t st, const uint8_t* zero_point = nullptr,
                             const float* next_sign = nullptr, int act = 0);
bool qlinear_fast_eligible(int M, int N, int K, int bits_a, int bits_w);
int qlinear_fast_launch(const uint8_t* a_codes, const float* s, int bits_a, const uint8_t* w_codes,
                        const uint16_t* rnorm, int bits_w, int M, int N, int K, uint16_t* Y,
                        const CodebookDevice* ca, const CodebookDevice* cw, unsigned int* err, cudaStream_t st);
}  // namespace rbq

using namespace rbq;

extern "C" int qlinear(const uint8_t* a_codes, const float* s, int bits_a, const uint8_t* w_codes,
                       const uint16_t* rnorm, int bits_w, int M, int N, int K, uint16_t* Y,
                       void* stream) {
  if (M < 0 || N < 0 || K <= 0 || K % kH || K > kMaxD) return RBQ_EINVAL;
  if (bits_a < 1 || bits_a > 8 || bits_w < 1 || bits_w > 8) return RBQ_EINVAL;
  if (M == 0 || N == 0) return RBQ_OK;
  if (!a_codes || !s || !w_codes || !rnorm || !Y) return RBQ_EINVAL;
  if (N % 8) return RBQ_EINVAL;
  if (!aligned(a_codes, 16) || !aligned(w_codes, 16) || !aligned(Y, 16) || !aligned(s, 4) ||
      !aligned(rnorm, 4))
    return RBQ_EALIGN;
  const CodebookDevice *ca = nullptr, *cw = nullptr;
  int rc = codebook_device(K, bits_a, &ca);
  if (rc != RBQ_OK) return rc;
  if ((rc = codebook_device(K, bits_w, &cw)) != RBQ_OK) return rc;
  unsigned int* err = nullptr;
  if ((rc = device_error_word_ptr(&err)) != RBQ_OK) return rc;
  if (qlinear_fast_eligible(M, N, K, bits_a, bits_w))
    return qlinear_fast_launch(a_codes, s, bits_a, w_codes, rnorm, bits_w, M, N, K, Y, ca, cw, err,
                               static_cast<cudaStream_t>(stream));
  QParams p{};
  p.A = a_codes;
  p.B = w_codes;
  p.a_pitch = static_cast<long long>(K) * bits_a / 8;
  p.b_pitch = static_cast<long long>(K) * bits_w / 8;
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
  return launch_qgemm<false>(p, static_cast<cudaStream_t>(stream));
}

extern "C" int qlinear_int8(const uint16_t* Xrot, const int8_t* Wq, const float* scale, int M, int N,
                            int K, uint16_t* Y, void* stream) {
  if (M < 0 || N < 0 || K <= 0 || K % kH || K > kMaxD) return RBQ_EINVAL;
  if (M == 0 || N == 0) return RBQ_OK;
  if (!Xrot || !Wq || !scale || !Y) return RBQ_EINVAL;
  if (N % 8) return RBQ_EINVAL;
  if (!aligned(Xrot, 16) || !aligned(Wq, 16) || !aligned(Y, 16) || !aligned(scale, 4)) return RBQ_EALIGN;
  unsigned int* err = nullptr;
  int rc = device_error_word_ptr(&err);
  if (rc != RBQ_OK) return rc;
  if (qlinear_int8_fast_eligible(M, N, K))
    return qlinear_int8_fast_launch(Xrot, Wq, scale, M, N, K, Y, err, static_cast<cudaStream_t>(stream));
  QParams p{};
  p.A = reinterpret_cast<const uint8_t*>(Xrot);
  p.B = reinterpret_cast<const uint8_t*>(Wq);
  p.a_pitch = static_cast<long long>(K) * 2;
  p.b_pitch = K;
  p.M = M;
  p.N = N;
  p.K = K;
  p.scale = scale;
  p.Y = Y;
  p.err = err;
  return launch_qgemm<true>(p, static_cast<cudaStream_t>(stream));
}

extern "C" int qlinear_int8_asym(const uint16_t* Xrot, const uint8_t* Wq, const float* scale,
                                 const uint8_t* zero_point, int M, int N, int K, uint16_t* Y, void* stream) {
  if (M < 0 || N < 0 || K <= 0 || K % kH || K > kMaxD) return RBQ_EINVAL;
  if (M == 0 || N == 0) return RBQ_OK;
  if (!Xrot || !Wq || !scale || !zero_point || !Y) return RBQ_EINVAL;
  if (!qlinear_int8_fast_eligible(M, N, K)) return RBQ_EINVAL;
  if (!aligned(Xrot, 16) || !aligned(Wq, 16) || !aligned(Y, 16) || !aligned(scale, 4)) return RBQ_EALIGN;
  unsigned int* err = nullptr;
  const int rc = device_error_word_ptr(&err);
  if (rc != RBQ_OK) return rc;
  return qlinear_int8_fast_launch(Xrot, reinterpret_cast<const int8_t*>(Wq), scale, M, N, K, Y, err,
                                  static_cast<cudaStream_t>(stream), zero_point);
}
