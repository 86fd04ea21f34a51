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

#include <cuda_runtime.h>

#include "rbq_internal.h"

namespace rbq {
int qlinear_int8_fast_launch(const uint16_t* Xrot, const int8_t* Wq, const float* scale, int M, int N, int K,
                             uint16_t* Y, unsigned int* err, cudaStream_t st, const uint8_t* zero_point,
                             const float* next_sign, int act);
bool qlinear_int8_fast_eligible(int M, int N, int K);

namespace {

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
