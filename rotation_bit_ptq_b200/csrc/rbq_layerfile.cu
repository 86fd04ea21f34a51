// Quantised layer files: the "quantized model file" of the INT8-convrot page
// (section 1: the quantised weights, their quantisation parameters and the
// transform info), one file per linear layer.  Host code only; the layout is
// documented in rbq.h.

#include <cstdio>
#include <cstring>
#include <vector>

#include "rbq.h"
#include "rbq_internal.h"

namespace {

constexpr char kMagic[8] = {'R', 'B', 'Q', 'L', 'A', 'Y', 'E', 'R'};
constexpr uint32_t kVersion = 1;
constexpr uint32_t kHeader = 64;

// FNV-1a, 64-bit (Fowler, Noll, Vo): offset basis and prime of the published
// definition.
struct Fnv64 {
  uint64_t h = 0xcbf29ce484222325ull;
  void add(const void* p, size_t n) {
    const auto* b = static_cast<const unsigned char*>(p);
    for (size_t i = 0; i < n; ++i) {
      h ^= b[i];
      h *= 0x100000001b3ull;
    }
  }
};

void put32(unsigned char* p, uint32_t v) {
  for (int i = 0; i < 4; ++i) p[i] = static_cast<unsigned char>(v >> (8 * i));
}
void put64(unsigned char* p, uint64_t v) {
  for (int i = 0; i < 8; ++i) p[i] = static_cast<unsigned char>(v >> (8 * i));
}
uint32_t get32(const unsigned char* p) {
  uint32_t v = 0;
  for (int i = 0; i < 4; ++i) v |= static_cast<uint32_t>(p[i]) << (8 * i);
  return v;
}
uint64_t get64(const unsigned char* p) {
  uint64_t v = 0;
  for (int i = 0; i < 8; ++i) v |= static_cast<uint64_t>(p[i]) << (8 * i);
  return v;
}

struct File {
  FILE* f = nullptr;
  File(const char* path, const char* mode) : f(std::fopen(path, mode)) {}
  ~File() {
    if (f) std::fclose(f);
  }
};

}  // namespace

extern "C" int rbq_layer_sizes(const rbq_layer_info* info, uint64_t* codes_bytes, uint64_t* aux_bytes,
                               uint64_t* zp_bytes) {
  if (!info) return RBQ_EINVAL;
  const rbq_layer_info& I = *info;
  if (I.h != rbq::kH || I.d <= 0 || I.d > rbq::kMaxD || I.d % I.h || I.rows <= 0) return RBQ_EINVAL;
  if (I.rpbh_flags & ~(RBQ_RPBH_NO_PERMUTATION | RBQ_RPBH_NO_SIGNS)) return RBQ_EINVAL;
  const uint64_t rows = static_cast<uint64_t>(I.rows), d = static_cast<uint64_t>(I.d);
  uint64_t c = 0, a = 0, z = 0;
  switch (I.mode) {
    case RBQ_LAYER_LLOYDMAX:
      if (I.bits < 1 || I.bits > 8) return RBQ_EINVAL;
      c = rows * d * static_cast<uint64_t>(I.bits) / 8;
      a = rows * 2;
      break;
    case RBQ_LAYER_INT8_SYM:
    case RBQ_LAYER_INT8_TENSOR:
      if (I.bits != 8) return RBQ_EINVAL;
      c = rows * d;
      a = rows * 4;
      break;
    case RBQ_LAYER_INT8_ASYM:
      if (I.bits != 8) return RBQ_EINVAL;
      c = rows * d;
      a = rows * 4;
      z = rows;
      break;
    default:
      return RBQ_EINVAL;
  }
  if (codes_bytes) *codes_bytes = c;
  if (aux_bytes) *aux_bytes = a;
  if (zp_bytes) *zp_bytes = z;
  return RBQ_OK;
}

extern "C" int rbq_layer_write(const char* path, const rbq_layer_info* info, const void* codes, const void* aux,
                               const void* zero_point) {
  uint64_t nc = 0, na = 0, nz = 0;
  if (!path) return RBQ_EINVAL;
  const int rc = rbq_layer_sizes(info, &nc, &na, &nz);
  if (rc != RBQ_OK) return rc;
  if (!codes || !aux || (nz && !zero_point)) return RBQ_EINVAL;
  File f(path, "wb");
  if (!f.f) return RBQ_EIO;
  Fnv64 sum;
  sum.add(codes, nc);
  sum.add(aux, na);
  if (nz) sum.add(zero_point, nz);
  unsigned char hdr[kHeader] = {};
  std::memcpy(hdr, kMagic, 8);
  put32(hdr + 8, kVersion);
  put32(hdr + 12, kHeader);
  put32(hdr + 16, static_cast<uint32_t>(info->d));
  put32(hdr + 20, static_cast<uint32_t>(info->h));
  put32(hdr + 24, static_cast<uint32_t>(info->rpbh_flags));
  put32(hdr + 28, static_cast<uint32_t>(info->mode));
  put32(hdr + 32, static_cast<uint32_t>(info->bits));
  put32(hdr + 36, static_cast<uint32_t>(info->rows));
  put64(hdr + 40, info->seed);
  put64(hdr + 48, sum.h);
  if (std::fwrite(hdr, 1, kHeader, f.f) != kHeader) return RBQ_EIO;
  if (std::fwrite(codes, 1, nc, f.f) != nc) return RBQ_EIO;
  if (std::fwrite(aux, 1, na, f.f) != na) return RBQ_EIO;
  if (nz && std::fwrite(zero_point, 1, nz, f.f) != nz) return RBQ_EIO;
  if (std::fflush(f.f) != 0) return RBQ_EIO;
  return RBQ_OK;
}

extern "C" int rbq_layer_read(const char* path, rbq_layer_info* info, void* codes, uint64_t codes_cap, void* aux,
                              uint64_t aux_cap, void* zero_point, uint64_t zp_cap) {
  if (!path || !info) return RBQ_EINVAL;
  File f(path, "rb");
  if (!f.f) return RBQ_EIO;
  unsigned char hdr[kHeader];
  if (std::fread(hdr, 1, kHeader, f.f) != kHeader) return RBQ_EIO;
  if (std::memcmp(hdr, kMagic, 8) != 0 || get32(hdr + 8) != kVersion || get32(hdr + 12) != kHeader) return RBQ_EIO;
  rbq_layer_info I{};
  I.d = static_cast<int32_t>(get32(hdr + 16));
  I.h = static_cast<int32_t>(get32(hdr + 20));
  I.rpbh_flags = static_cast<int32_t>(get32(hdr + 24));
  I.mode = static_cast<int32_t>(get32(hdr + 28));
  I.bits = static_cast<int32_t>(get32(hdr + 32));
  I.rows = static_cast<int32_t>(get32(hdr + 36));
  I.seed = get64(hdr + 40);
  const uint64_t want = get64(hdr + 48);
  uint64_t nc = 0, na = 0, nz = 0;
  if (rbq_layer_sizes(&I, &nc, &na, &nz) != RBQ_OK) return RBQ_EIO;   // a header no writer makes
  *info = I;
  if (!codes && !aux && !zero_point) return RBQ_OK;                   // info only
  if (!codes || !aux || (nz && !zero_point)) return RBQ_EINVAL;
  // The payload sizes come from this file's header; a file replaced since the
  // caller sized its buffers (or buffers sized from another description)
  // must not be read past their ends.
  if (nc > codes_cap || na > aux_cap || nz > zp_cap) return RBQ_EINVAL;
  if (std::fread(codes, 1, nc, f.f) != nc) return RBQ_EIO;
  if (std::fread(aux, 1, na, f.f) != na) return RBQ_EIO;
  if (nz && std::fread(zero_point, 1, nz, f.f) != nz) return RBQ_EIO;
  unsigned char extra;
  if (std::fread(&extra, 1, 1, f.f) != 0) return RBQ_EIO;             // trailing bytes: not this format
  Fnv64 sum;
  sum.add(codes, nc);
  sum.add(aux, na);
  if (nz) sum.add(zero_point, nz);
  return sum.h == want ? RBQ_OK : RBQ_EIO;
}
