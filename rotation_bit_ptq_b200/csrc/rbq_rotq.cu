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

namespace rbq {
namespace {

enum Mode { kAct = 0, kWeightLM = 1, kInt8 = 2, kRotate = 3 };

struct RotqParams {
  const void* X;
  long long T;
  int d, nblk, G;
  const int32_t* perm;
  const float* sign;
  const float* bounds;   // 2^bits - 1 Lloyd-Max boundaries (Lloyd-Max modes)
  void* out;             // packed codes | int8 q | bf16 x'
  void* aux;             // float norms | bf16 row norms | float scales | float norms (optional)
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
  float* bnd = tok + G;                                  // [2^BITS - 1]

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
      y[i] = p.sign[k] * rows[g * d + p.perm[k]];
    }
    fwht64(y);
    float acc = 0.f;
#pragma unroll
    for (int i = 0; i < 64; ++i) {
      y[i] *= 0.125f;                                    // 1/sqrt(64): orthonormal H
      acc = (MODE == kInt8) ? fmaxf(acc, fabsf(y[i])) : fmaf(y[i], y[i], acc);
    }
    red[g * nblk + b] = acc;
    __syncthreads();
    if (b == 0) {
      float tot = 0.f;
      for (int j = 0; j < nblk; ++j)
        tot = (MODE == kInt8) ? fmaxf(tot, red[g * nblk + j]) : tot + red[g * nblk + j];
      tok[g] = (MODE == kInt8) ? tot : sqrtf(tot);
    }
    __syncthreads();
    if (t >= p.T) continue;
    const float s = tok[g];

    if constexpr (kLloyd) {
      const float inv = 1.0f / (s + 1e-12f);
      uint32_t w[2 * BITS];
#pragma unroll
      for (int i = 0; i < 2 * BITS; ++i) w[i] = 0u;
#pragma unroll
      for (int i = 0; i < 64; ++i) {
        const uint32_t c = code_of<BITS>(y[i] * inv, bnd);
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
      const float scale = s / 127.0f;
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
      if (b == 0) static_cast<float*>(p.aux)[t] = scale;
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
  const size_t smem = sizeof(float) * (static_cast<size_t>(p.G) * p.d + p.G * p.nblk + p.G + 256);
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

// Tokens per CTA so that a CTA has at least 128 threads (one per block).
int tokens_per_cta(int nblk) {
  int G = (128 + nblk - 1) / nblk;
  if (G * nblk > 512) G = 512 / nblk;
  return G < 1 ? 1 : G;
}

int prepare(const rbq_rpbh* r, int mode, int bits, long long rows, const void* X, void* out,
            void* aux, RotqParams* p) {
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
  if (mode == kAct || mode == kWeightLM) {
    const CodebookDevice* cb = nullptr;
    if ((rc = codebook_device(r->d, bits, &cb)) != RBQ_OK) return rc;
    p->bounds = cb->bounds;
  }
  return RBQ_OK;
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
  RotqParams p;
  const int mode = rot ? kRotate : kAct;
  int rc = prepare(r, mode, bits, T, X, codes_out, norms_out, &p);
  if (rc != RBQ_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return rot ? launch_mode<kRotate>(dtype, 8, p, st) : launch_mode<kAct>(dtype, bits, p, st);
}

extern "C" int quantize_weights(const rbq_rpbh* r, const void* W, int dtype, int d_out, int mode,
                                int bits, void* codes_or_q, void* rownorm_or_scale, void* stream) {
  if (!r || d_out < 0 || (dtype != RBQ_F32 && dtype != RBQ_BF16)) return RBQ_EINVAL;
  if (mode == RBQ_LLOYDMAX) {
    if (bits < 1 || bits > 8) return RBQ_EINVAL;
  } else if (mode == RBQ_INT8_SYM) {
    if (bits != 8) return RBQ_EINVAL;
  } else {
    return RBQ_EINVAL;
  }
  if (d_out == 0) return RBQ_OK;
  if (!W || !codes_or_q || !rownorm_or_scale) return RBQ_EINVAL;
  if (!aligned(W, 16) || !aligned(codes_or_q, 16) || !aligned(rownorm_or_scale, 4))
    return RBQ_EALIGN;
  RotqParams p;
  const int m = (mode == RBQ_LLOYDMAX) ? kWeightLM : kInt8;
  int rc = prepare(r, m, bits, d_out, W, codes_or_q, rownorm_or_scale, &p);
  if (rc != RBQ_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return (m == kWeightLM) ? launch_mode<kWeightLM>(dtype, bits, p, st)
                          : launch_mode<kInt8>(dtype, 8, p, st);
}
