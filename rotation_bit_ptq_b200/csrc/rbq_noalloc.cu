// qlinear_noalloc: the quantised linear of qlinear() for callers that cannot
// allocate device memory.
//
// qlinear() expands the weight codes into an fp16 workspace of N*K*2 bytes
// that it takes from a stream-ordered memory pool on every call.  Some callers
// cannot let a library do that: a host program that owns every byte of the
// device through its own allocator and must not see the driver's pool grow, a
// runtime that forbids allocation on its inference thread, or a plug-in loaded
// into a process whose allocator is not the CUDA one.  This variant runs the
// same two kernels (weight expansion, then the tcgen05 GEMM) but puts the
// workspace, the level tables and a fallback error word in one file-scope
// __device__ array of fixed size.  Nothing is allocated on any call.
//
// The array's name, seen from host code, is a host-side stand-in and not a
// device address; the device address is looked up once per device with
// cudaGetSymbolAddress while that device is current, and only that address is
// handed to the kernels.

#include <cuda_fp16.h>

#include <cmath>
#include <mutex>

#include "rbq_internal.h"

namespace rbq {
int qlinear_fast_gemm(const uint8_t* a_codes, const float* s, int bits_a, const uint16_t* wf16,
                      const uint16_t* rnorm, int M, int N, int K, uint16_t* Y, const CodebookDevice* ca,
                      unsigned int* err, cudaStream_t st, int sms);
bool qlinear_fast_eligible(int M, int N, int K, int bits_a, int bits_w);
namespace qfast {
int expand_weights(const uint8_t* codes, int bits, int rows, int K, const uint16_t* lut, uint16_t* out,
                   cudaStream_t st, int sms);
}  // namespace qfast

namespace {

// Layout of the array: [fp16 weights, up to kWorkspaceBytes][kLutSlots level
// tables of 256 x u16][error word].
constexpr size_t kWorkspaceBytes = size_t(32) << 20;          // N * K <= 16,777,216
constexpr int kLutSlots = 16;
constexpr size_t kLutBytes = 512;
constexpr size_t kLutOffset = kWorkspaceBytes;
constexpr size_t kErrOffset = kLutOffset + kLutSlots * kLutBytes;
constexpr size_t kScratchBytes = kErrOffset + 256;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

// Device address of the array, per device (looked up once, then reused).
unsigned char* g_scratch_addr[kMaxDevices] = {};
std::mutex g_setup_mu;

int scratch_address(int dev, unsigned char** out) {
  std::lock_guard<std::mutex> lk(g_setup_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e);
    if (!p) return RBQ_ECUDA;
    g_scratch_addr[dev] = static_cast<unsigned char*>(p);
  }
  *out = g_scratch_addr[dev];
  return RBQ_OK;
}

// Host copies of the fp16 level tables (levels x sqrt(d), the scaling the
// GEMM's epilogue undoes with 1/d), kept so that repeated calls do not solve
// the Lloyd-Max conditions again.  Entries are never moved or overwritten
// while the cache has room; when it is full the last entry is reused.
struct HostLut {
  int d = 0, bits = 0;
  uint16_t lut[256] = {};
};
constexpr int kLutCache = 64;
HostLut g_luts[kLutCache];
int g_nluts = 0;

int host_lut(int d, int bits, const uint16_t** out) {
  for (int i = 0; i < g_nluts; ++i)
    if (g_luts[i].d == d && g_luts[i].bits == bits) { *out = g_luts[i].lut; return RBQ_OK; }
  double levels[256], bounds[255];
  const int rc = lloydmax_table(d, bits, levels, bounds);
  if (rc != RBQ_OK) return rc;
  HostLut& h = g_luts[g_nluts < kLutCache ? g_nluts++ : (kLutCache - 1)];
  h.d = d;
  h.bits = bits;
  const double sd = std::sqrt(static_cast<double>(d));
  for (int j = 0; j < 256; ++j) {
    const __half v = __float2half_rn(j < (1 << bits) ? static_cast<float>(levels[j] * sd) : 0.f);
    h.lut[j] = *reinterpret_cast<const uint16_t*>(&v);
  }
  *out = h.lut;
  return RBQ_OK;
}

// Which (d, bits) level table each of a device's slots holds.  A table is
// copied into a slot on the first call that needs it on that device (ordered
// on that call's stream before its kernels); later calls find it there and
// copy nothing.  When every slot is taken, slots are reused in turn (never
// the one the same call just took for its other operand).
struct SlotKey {
  int d = 0, bits = 0;
};
SlotKey g_slot_key[kMaxDevices][kLutSlots];
int g_slot_next[kMaxDevices] = {};
std::mutex g_slot_mu;

int level_table_slot(int dev, unsigned char* base, int d, int bits, int avoid, cudaStream_t st, int* slot_out) {
  std::lock_guard<std::mutex> lk(g_slot_mu);
  SlotKey* keys = g_slot_key[dev];
  for (int i = 0; i < kLutSlots; ++i)
    if (keys[i].d == d && keys[i].bits == bits) { *slot_out = i; return RBQ_OK; }
  int slot = -1;
  for (int i = 0; i < kLutSlots && slot < 0; ++i)
    if (keys[i].d == 0 && i != avoid) slot = i;
  if (slot < 0) {
    slot = g_slot_next[dev];
    if (slot == avoid) slot = (slot + 1) % kLutSlots;
    g_slot_next[dev] = (slot + 1) % kLutSlots;
  }
  const uint16_t* lut = nullptr;
  int rc = host_lut(d, bits, &lut);
  if (rc != RBQ_OK) return rc;
  // A copy from pageable host memory returns once the source has been staged,
  // so the host table may change afterwards; the device copy is ordered on
  // `st` before the kernels that read the slot.
  const cudaError_t e = cudaMemcpyAsync(base + kLutOffset + static_cast<size_t>(slot) * kLutBytes, lut, kLutBytes,
                                        cudaMemcpyHostToDevice, st);
  if (e != cudaSuccess) {
    keys[slot] = SlotKey{};
    return cuda_fail(e);
  }
  keys[slot].d = d;
  keys[slot].bits = bits;
  *slot_out = slot;
  return RBQ_OK;
}

}  // namespace
}  // namespace rbq

using namespace rbq;

extern "C" int qlinear_noalloc(const uint8_t* a_codes, const float* s, int bits_a, const uint8_t* w_codes,
                               const uint16_t* rnorm, int bits_w, int M, int N, int K, uint16_t* Y,
                               unsigned int* err, void* stream) {
  if (M < 0 || N < 0 || K <= 0 || K % kH || K > kMaxD) return RBQ_EINVAL;
  if (bits_a < 1 || bits_a > 8 || bits_w < 1 || bits_w > 8) return RBQ_EINVAL;
  if (M == 0 || N == 0) return RBQ_OK;
  if (!a_codes || !s || !w_codes || !rnorm || !Y) return RBQ_EINVAL;
  if (!qlinear_fast_eligible(M, N, K, bits_a, bits_w)) return RBQ_EINVAL;
  if (static_cast<size_t>(N) * static_cast<size_t>(K) * 2 > kWorkspaceBytes) return RBQ_ESCRATCH;
  if (!aligned(a_codes, 16) || !aligned(w_codes, 16) || !aligned(Y, 16) || !aligned(s, 4) ||
      !aligned(rnorm, 4) || (err && !aligned(err, 4)))
    return RBQ_EALIGN;

  int dev = 0, sms = 148;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= kMaxDevices) return RBQ_EINVAL;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return cuda_fail(e);

  unsigned char* base = nullptr;
  int rc = scratch_address(dev, &base);
  if (rc != RBQ_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int slot_a = 0, slot_w = 0;
  if ((rc = level_table_slot(dev, base, K, bits_a, -1, st, &slot_a)) != RBQ_OK) return rc;
  if ((rc = level_table_slot(dev, base, K, bits_w, slot_a, st, &slot_w)) != RBQ_OK) return rc;

  uint16_t* wf16 = reinterpret_cast<uint16_t*>(base);
  uint16_t* dlut_a = reinterpret_cast<uint16_t*>(base + kLutOffset + static_cast<size_t>(slot_a) * kLutBytes);
  uint16_t* dlut_w = reinterpret_cast<uint16_t*>(base + kLutOffset + static_cast<size_t>(slot_w) * kLutBytes);
  unsigned int* werr = err ? err : reinterpret_cast<unsigned int*>(base + kErrOffset);
  // The workspace needs no clearing: the expansion writes every element the
  // GEMM reads.

  CodebookDevice ca{};
  ca.d = K;
  ca.bits = bits_a;
  ca.levels_f16 = dlut_a;
  ca.inv_d = static_cast<float>(1.0 / K);
  rc = qfast::expand_weights(w_codes, bits_w, N, K, dlut_w, wf16, st, sms);
  if (rc != RBQ_OK) return rc;
  return qlinear_fast_gemm(a_codes, s, bits_a, wf16, rnorm, M, N, K, Y, &ca, werr, st, sms);
}
