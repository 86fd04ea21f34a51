// Host half of the boundary: RPBH draws, the Lloyd-Max solver, per-device
// table caches, error reporting.
//
// Sources: OrbitQuant write-up (hotelren.com/news/3376620) §2.3 for the RPBH
// structure and §6.3 for reproducible random draws; §1 and §4.2 for the
// per-d Lloyd-Max codebook of N(0, 1/d).

#include <algorithm>
#include <cmath>
#include <cstring>
#include <map>
#include <mutex>
#include <new>
#include <utility>

#include "rbq_internal.h"

namespace rbq {
namespace {

thread_local cudaError_t g_last_cuda = cudaSuccess;
std::mutex g_mu;

// ---------------------------------------------------------------------------
// SplitMix64 (Steele, Lea & Flood, OOPSLA 2014): Weyl increment, then the
// 64-bit finaliser with shifts 30/27/31.
// ---------------------------------------------------------------------------
struct SplitMix64 {
  uint64_t s;
  explicit SplitMix64(uint64_t seed) : s(seed) {}
  uint64_t next() {
    uint64_t z = (s += 0x9E3779B97F4A7C15ull);
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
  }
};

// floor(u * n / 2^64): multiply-high range reduction.
inline uint32_t mulhi_range(uint64_t u, uint32_t n) {
  return static_cast<uint32_t>((static_cast<unsigned __int128>(u) * n) >> 64);
}

// ---------------------------------------------------------------------------
// Lloyd-Max for N(0,1), positive half.  The optimum is symmetric (unique for
// a log-concave density), so with H = 2^(b-1) positive levels c_0 < ... <
// c_{H-1} the boundaries are t_0 = 0, t_i = (c_{i-1}+c_i)/2, t_H = +inf and
// the centroid map is G_i(c) = (phi(t_i) - phi(t_{i+1})) / (Q(t_i) - Q(t_{i+1}))
// with Q the upper tail.  We solve G(c) = c by Newton's method: dG_i/dt_i =
// phi(t_i)(G_i - t_i)/P_i and dG_i/dt_{i+1} = phi(t_{i+1})(t_{i+1} - G_i)/P_i,
// each t depending on two neighbouring levels with weight 1/2, so the
// Jacobian is tridiagonal.
// ---------------------------------------------------------------------------
constexpr double kInvSqrt2Pi = 0.39894228040143267794;

inline double pdf(double x) { return std::isinf(x) ? 0.0 : kInvSqrt2Pi * std::exp(-0.5 * x * x); }
inline double upper_tail(double x) { return 0.5 * std::erfc(x * 0.70710678118654752440); }

void centroid_map(const std::vector<double>& c, std::vector<double>& t,
                  std::vector<double>& G, std::vector<double>& P) {
  const int H = static_cast<int>(c.size());
  t.assign(H + 1, 0.0);
  for (int i = 1; i < H; ++i) t[i] = 0.5 * (c[i - 1] + c[i]);
  t[H] = INFINITY;
  G.resize(H);
  P.resize(H);
  for (int i = 0; i < H; ++i) {
    P[i] = upper_tail(t[i]) - upper_tail(t[i + 1]);
    G[i] = (pdf(t[i]) - pdf(t[i + 1])) / P[i];
  }
}

int lloydmax_half(int bits, std::vector<double>& c_out) {
  const int H = 1 << (bits - 1);
  std::vector<double> c(H), t, G, P, lo(H), di(H), up(H), rhs(H), cp(H), dp(H);
  for (int i = 0; i < H; ++i) c[i] = (i + 0.5) * (4.0 / H);
  // A few plain fixed-point steps bring the start into Newton's basin.
  for (int it = 0; it < 60; ++it) {
    centroid_map(c, t, G, P);
    c = G;
  }
  bool done = false;
  for (int it = 0; it < 200 && !done; ++it) {
    centroid_map(c, t, G, P);
    for (int i = 0; i < H; ++i) {
      const double a = (i >= 1) ? 0.5 * pdf(t[i]) * (G[i] - t[i]) / P[i] : 0.0;
      const double b = (i + 1 < H) ? 0.5 * pdf(t[i + 1]) * (t[i + 1] - G[i]) / P[i] : 0.0;
      lo[i] = a;               // d G_i / d c_{i-1}
      up[i] = b;               // d G_i / d c_{i+1}
      di[i] = a + b - 1.0;     // d (G_i - c_i) / d c_i
      rhs[i] = c[i] - G[i];    // solve (J - I) delta = -(G - c)
    }
    // Thomas algorithm.
    cp[0] = (H > 1) ? up[0] / di[0] : 0.0;
    dp[0] = rhs[0] / di[0];
    for (int i = 1; i < H; ++i) {
      const double m = di[i] - lo[i] * cp[i - 1];
      cp[i] = (i + 1 < H) ? up[i] / m : 0.0;
      dp[i] = (rhs[i] - lo[i] * dp[i - 1]) / m;
    }
    std::vector<double> delta(H);
    delta[H - 1] = dp[H - 1];
    for (int i = H - 2; i >= 0; --i) delta[i] = dp[i] - cp[i] * delta[i + 1];
    // Damp the step if it would break the ordering 0 < c_0 < ... < c_{H-1}.
    double lam = 1.0;
    for (int tries = 0; tries < 40; ++tries) {
      bool ok = c[0] + lam * delta[0] > 0.0;
      for (int i = 1; i < H && ok; ++i)
        ok = (c[i] + lam * delta[i]) > (c[i - 1] + lam * delta[i - 1]);
      if (ok) break;
      lam *= 0.5;
    }
    double step = 0.0;
    for (int i = 0; i < H; ++i) {
      c[i] += lam * delta[i];
      step = std::fmax(step, std::fabs(lam * delta[i]));
    }
    done = step < 1e-15 * std::fmax(1.0, c[H - 1]);
  }
  centroid_map(c, t, G, P);
  double resid = 0.0;
  for (int i = 0; i < H; ++i) resid = std::fmax(resid, std::fabs(G[i] - c[i]));
  if (!(resid < 1e-12)) return RBQ_ECONVERGE;
  c_out = c;
  return RBQ_OK;
}

struct UnitTable {
  std::vector<double> half;   // positive levels of N(0,1)
};

std::map<int, UnitTable>& unit_cache() {
  static std::map<int, UnitTable> m;
  return m;
}

int unit_half(int bits, std::vector<double>& half) {
  {
    std::lock_guard<std::mutex> lk(g_mu);
    auto it = unit_cache().find(bits);
    if (it != unit_cache().end()) { half = it->second.half; return RBQ_OK; }
  }
  std::vector<double> c;
  const int rc = lloydmax_half(bits, c);
  if (rc != RBQ_OK) return rc;
  std::lock_guard<std::mutex> lk(g_mu);
  unit_cache()[bits].half = c;
  half = c;
  return RBQ_OK;
}

// Full (levels, bounds) of N(0, 1/d) from the positive half of N(0,1).
int full_table(int d, int bits, std::vector<double>& levels, std::vector<double>& bounds) {
  std::vector<double> half;
  const int rc = unit_half(bits, half);
  if (rc != RBQ_OK) return rc;
  const int H = 1 << (bits - 1), L = 2 * H;
  const double sd = std::sqrt(static_cast<double>(d));
  levels.assign(L, 0.0);
  bounds.assign(L - 1, 0.0);
  for (int i = 0; i < H; ++i) {
    levels[H + i] = half[i] / sd;
    levels[H - 1 - i] = -half[i] / sd;
  }
  // Boundaries are the midpoints of the returned levels; antisymmetric levels
  // make the middle one exactly 0.
  for (int j = 0; j < L - 1; ++j) bounds[j] = 0.5 * (levels[j] + levels[j + 1]);
  return RBQ_OK;
}

// fp32 -> fp16 bit pattern, round to nearest even (host side; normal range).
uint16_t f32_to_f16_bits(float f) {
  uint32_t x;
  std::memcpy(&x, &f, 4);
  const uint32_t sign = (x >> 16) & 0x8000u;
  const int32_t exp = static_cast<int32_t>((x >> 23) & 0xFF) - 127 + 15;
  uint32_t man = x & 0x7FFFFFu;
  if (exp <= 0) {            // subnormal half (or zero)
    if (exp < -10) return static_cast<uint16_t>(sign);
    man |= 0x800000u;
    const int shift = 14 - exp;
    uint32_t h = man >> shift;
    const uint32_t rem = man & ((1u << shift) - 1), halfway = 1u << (shift - 1);
    if (rem > halfway || (rem == halfway && (h & 1u))) ++h;
    return static_cast<uint16_t>(sign | h);
  }
  if (exp >= 31) return static_cast<uint16_t>(sign | 0x7C00u);
  uint32_t h = (static_cast<uint32_t>(exp) << 10) | (man >> 13);
  const uint32_t rem = man & 0x1FFFu;
  if (rem > 0x1000u || (rem == 0x1000u && (h & 1u))) ++h;
  return static_cast<uint16_t>(sign | h);
}

// ---------------------------------------------------------------------------
// Code-search grid.  The kernel finds code #{t_j <= v} with one comparison:
// n = round(sat(v / (2R) + 1/2) * NC) picks cell n of a uniform grid whose
// cells are centred at -R + n w (w = 2R/NC, n = 0..NC); each cell holds at most
// one boundary, so the code is the number of boundaries below the cell plus
// (v >= that boundary).  Rounding can put v one cell off near a cell edge;
// that gives the same code as long as no boundary sits near an edge, which is
// checked here (margin 1% of a cell).  NC even puts the boundary at 0 in the
// middle of cell NC/2; the end cells (which also take the clamped values
// beyond +-R) hold no boundary.
// ---------------------------------------------------------------------------
inline float int_bits_as_float(int v) {
  float f;
  std::memcpy(&f, &v, sizeof(f));
  return f;
}

struct Grid {
  int cells = 0;
  double R = 0.0;
  std::vector<float2> lut;
};

bool try_grid(const std::vector<double>& t, int nc, double R, Grid* g) {
  const double w = 2.0 * R / nc;
  std::vector<float2> lut(nc + 1);
  size_t j = 0;   // first boundary not below the current cell's lower edge
  for (int n = 0; n <= nc; ++n) {
    const double lo = -R + (n - 0.5) * w, hi = lo + w;
    if (n == 0) {               // also takes v <= -R: below every boundary
      if (!t.empty() && t.front() < hi + 0.01 * w) return false;
      lut[n] = make_float2(INFINITY, int_bits_as_float(0));
      continue;
    }
    if (n == nc) {              // also takes v >= R: above every boundary
      if (!t.empty() && t.back() >= lo - 0.01 * w) return false;
      lut[n] = make_float2(INFINITY, int_bits_as_float(static_cast<int>(t.size())));
      continue;
    }
    while (j < t.size() && t[j] < lo) ++j;
    size_t k = j;
    int inside = 0;
    double thr = INFINITY;
    while (k < t.size() && t[k] < hi) {
      if (t[k] - lo < 0.01 * w || hi - t[k] < 0.01 * w) return false;
      thr = t[k];
      ++inside;
      ++k;
    }
    if (inside > 1) return false;
    float tf = static_cast<float>(thr);
    if (inside == 1 && thr == 0.0) tf = -0.0f;   // so that -0.0 counts as >= 0
    lut[n] = make_float2(tf, int_bits_as_float(static_cast<int>(j)));
  }
  g->cells = nc;
  g->R = R;
  g->lut = std::move(lut);
  return true;
}

// Full-range variant: R = 1, the largest |v| a unit vector can have, so the
// kernel needs no clamp.  Returns RBQ_ECONVERGE if it would need more than
// `max_cells` cells.
int build_grid_full(const std::vector<double>& bounds, int max_cells, Grid* g) {
  double gap = INFINITY;
  for (size_t j = 1; j < bounds.size(); ++j) gap = std::fmin(gap, bounds[j] - bounds[j - 1]);
  if (bounds.size() == 1) gap = 1.0;
  int nc = static_cast<int>(std::ceil(2.0 / (0.9 * gap)));
  nc += nc & 1;
  if (nc < 4) nc = 4;
  for (; nc <= max_cells; nc += 2)
    if (try_grid(bounds, nc, 1.0, g)) return RBQ_OK;
  return RBQ_ECONVERGE;
}

int build_grid(const std::vector<double>& bounds, Grid* g) {
  double tmax = 0.0, gap = INFINITY;
  for (size_t j = 0; j < bounds.size(); ++j) {
    tmax = std::fmax(tmax, std::fabs(bounds[j]));
    if (j) gap = std::fmin(gap, bounds[j] - bounds[j - 1]);
  }
  if (bounds.size() == 1) gap = 1.0;           // 1 bit: the single boundary 0
  const double R0 = tmax > 0.0 ? tmax * 1.05 : 1.0;
  int nc = static_cast<int>(std::ceil(2.0 * R0 / (0.9 * gap)));
  nc += nc & 1;
  if (nc < 2) nc = 2;
  for (; nc <= 4096; nc += 2)
    for (int step = 0; step < 64; ++step)
      if (try_grid(bounds, nc, R0 * (1.0 + 0.003 * step), g)) return RBQ_OK;
  return RBQ_ECONVERGE;
}

// ---------------------------------------------------------------------------
// Per-device caches.
// ---------------------------------------------------------------------------
std::map<std::pair<int, long long>, CodebookDevice*>& cb_cache() {
  static std::map<std::pair<int, long long>, CodebookDevice*> m;
  return m;
}

unsigned int* g_err_word[kMaxDevices] = {};

template <class T>
int upload(const T* host, size_t n, T** dev) {
  cudaError_t e = cudaMalloc(reinterpret_cast<void**>(dev), n * sizeof(T));
  if (e != cudaSuccess) return cuda_fail(e);
  e = cudaMemcpy(*dev, host, n * sizeof(T), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return cuda_fail(e);
  return RBQ_OK;
}

int current_device(int* dev) {
  const cudaError_t e = cudaGetDevice(dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (*dev < 0 || *dev >= kMaxDevices) return RBQ_EINVAL;
  return RBQ_OK;
}

}  // namespace

int cuda_fail(cudaError_t e) {
  g_last_cuda = e;
  return RBQ_ECUDA;
}

int rpbh_device(const rbq_rpbh* r, const RpbhDevice** out) {
  int dev;
  int rc = current_device(&dev);
  if (rc != RBQ_OK) return rc;
  auto* mr = const_cast<rbq_rpbh*>(r);
  std::lock_guard<std::mutex> lk(g_mu);
  RpbhDevice& D = mr->dev[dev];
  if (!D.ready) {
    std::vector<float> s(r->d);
    for (int k = 0; k < r->d; ++k) s[k] = static_cast<float>(r->sign[k]);
    if ((rc = upload(r->perm.data(), r->perm.size(), &D.perm)) != RBQ_OK) return rc;
    if ((rc = upload(s.data(), s.size(), &D.sign)) != RBQ_OK) return rc;
    D.ready = true;
  }
  *out = &D;
  return RBQ_OK;
}

int rpbh_pair_tables(const rbq_rpbh* r, const uint32_t** out) {
  const RpbhDevice* rd = nullptr;
  int rc = rpbh_device(r, &rd);
  if (rc != RBQ_OK) return rc;
  std::lock_guard<std::mutex> lk(g_mu);
  auto* D = const_cast<RpbhDevice*>(rd);
  if (!D->pair_tab) {
    const int d = r->d;
    std::vector<uint32_t> tab(static_cast<size_t>(d));
    for (int k = 0; k < d; ++k) {
      const uint32_t slot = pair_tab_slot(k / kH, k % kH);
      tab[slot] = 2u * static_cast<uint32_t>(r->perm[k]) | (r->sign[k] < 0 ? 0x80000000u : 0u);
    }
    uint32_t* dev = nullptr;
    if ((rc = upload(tab.data(), tab.size(), &dev)) != RBQ_OK) return rc;
    D->pair_tab = dev;
  }
  *out = D->pair_tab;
  return RBQ_OK;
}

int rpbh_pair_tables16(const rbq_rpbh* r, const uint16_t** out) {
  if (r->d > 16384) return RBQ_EINVAL;
  const RpbhDevice* rd = nullptr;
  int rc = rpbh_device(r, &rd);
  if (rc != RBQ_OK) return rc;
  std::lock_guard<std::mutex> lk(g_mu);
  auto* D = const_cast<RpbhDevice*>(rd);
  if (!D->pair_tab16) {
    const int d = r->d;
    std::vector<uint16_t> tab(static_cast<size_t>(d));
    for (int k = 0; k < d; ++k) {
      const uint32_t slot = pair_tab16_slot(k / kH, k % kH);
      tab[slot] = static_cast<uint16_t>(2u * static_cast<uint32_t>(r->perm[k]) | (r->sign[k] < 0 ? 0x8000u : 0u));
    }
    uint16_t* dev = nullptr;
    if ((rc = upload(tab.data(), tab.size(), &dev)) != RBQ_OK) return rc;
    D->pair_tab16 = dev;
  }
  *out = D->pair_tab16;
  return RBQ_OK;
}

// The grid with kGridGuard copies of each end entry outside it, padded with
// one more copy of the last entry to an even count.
std::vector<float2> guarded(const std::vector<float2>& lut) {
  const int n = static_cast<int>(lut.size());
  std::vector<float2> g(guarded_grid_entries(n));
  for (int i = 0; i < static_cast<int>(g.size()); ++i) g[i] = lut[std::min(std::max(i - kGridGuard, 0), n - 1)];
  return g;
}

void int8_levels(const std::vector<double>& levels, std::vector<int8_t>& out, double* alpha) {
  double cmax = 0.0;
  for (double c : levels) cmax = std::max(cmax, std::fabs(c));
  const double a = 127.0 / cmax;
  out.assign(levels.size(), 0);
  for (size_t j = 0; j < levels.size(); ++j) out[j] = static_cast<int8_t>(std::nearbyint(a * levels[j]));
  *alpha = a;
}

// Round-to-nearest-even onto FP8 E4M3 (OCP "E4M3FN": 1 sign bit, 4 exponent
// bits with bias 7, 3 mantissa bits, subnormals below 2^-6, largest finite
// 448, no infinities) and encode; |x| above 448 saturates (never reached for
// the scaled levels, which stay below 256).
static uint8_t to_e4m3(double x) {
  const uint8_t sign = std::signbit(x) ? 0x80 : 0x00;
  double a = std::fabs(x);
  if (a == 0.0) return sign;
  int E = 0;
  const double f = std::frexp(a, &E);          // a = f 2^E, f in [0.5, 1)
  int e = E - 1;                               // a = m 2^e, m in [1, 2)
  if (e < -6) {                                // subnormal: multiples of 2^-9
    const double q = std::nearbyint(std::ldexp(a, 9));
    if (q >= 8.0) return sign | (1u << 3);     // rounds up to the smallest normal
    return sign | static_cast<uint8_t>(q);
  }
  double q = std::nearbyint(2.0 * f * 8.0);     // 8 .. 16
  if (q == 16.0) { q = 8.0; ++e; }
  if (e > 8 || (e == 8 && q > 14.0)) return sign | 0x7E;   // 448
  return sign | static_cast<uint8_t>(((e + 7) << 3) | (static_cast<int>(q) - 8));
}

void fp8_levels(const std::vector<double>& levels, std::vector<uint8_t>& out, double* beta) {
  double cmax = 0.0;
  for (double c : levels) cmax = std::max(cmax, std::fabs(c));
  int E = 0;
  std::frexp(cmax, &E);                        // cmax in [2^(E-1), 2^E)
  const double b = std::ldexp(1.0, 8 - E);     // b cmax in [128, 256)
  out.assign(levels.size(), 0);
  for (size_t j = 0; j < levels.size(); ++j) out[j] = to_e4m3(b * levels[j]);
  *beta = b;
}

int codebook_device(int d, int bits, const CodebookDevice** out) {
  int dev;
  int rc = current_device(&dev);
  if (rc != RBQ_OK) return rc;
  const auto key = std::make_pair(dev, (static_cast<long long>(d) << 8) | bits);
  {
    std::lock_guard<std::mutex> lk(g_mu);
    auto it = cb_cache().find(key);
    if (it != cb_cache().end()) { *out = it->second; return RBQ_OK; }
  }
  std::vector<double> levels, bounds;
  if ((rc = full_table(d, bits, levels, bounds)) != RBQ_OK) return rc;
  auto* cb = new (std::nothrow) CodebookDevice;
  if (!cb) return RBQ_ENOMEM;
  cb->d = d;
  cb->bits = bits;
  cb->inv_d = static_cast<float>(1.0 / d);
  const int L = 1 << bits;
  std::vector<float> bf(L - 1);
  for (int j = 0; j < L - 1; ++j) bf[j] = static_cast<float>(bounds[j]);
  std::vector<uint16_t> lh(L);
  const double sd = std::sqrt(static_cast<double>(d));
  for (int j = 0; j < L; ++j) lh[j] = f32_to_f16_bits(static_cast<float>(levels[j] * sd));
  if ((rc = upload(bf.data(), bf.size(), &cb->bounds)) != RBQ_OK) { delete cb; return rc; }
  if ((rc = upload(lh.data(), lh.size(), &cb->levels_f16)) != RBQ_OK) { delete cb; return rc; }
  {
    std::vector<int8_t> li;
    int8_levels(levels, li, &cb->alpha);
    li.resize(256, 0);
    if ((rc = upload(li.data(), li.size(), &cb->levels_i8)) != RBQ_OK) { delete cb; return rc; }
    std::vector<uint8_t> lf;
    fp8_levels(levels, lf, &cb->beta);
    lf.resize(256, 0);
    if ((rc = upload(lf.data(), lf.size(), &cb->levels_e4m3)) != RBQ_OK) { delete cb; return rc; }
  }
  Grid grid;
  if ((rc = build_grid(bounds, &grid)) != RBQ_OK) { delete cb; return rc; }
  cb->grid_cells = grid.cells;
  cb->grid_scale = static_cast<float>(1.0 / (2.0 * grid.R));
  if ((rc = upload(grid.lut.data(), grid.lut.size(), &cb->grid)) != RBQ_OK) { delete cb; return rc; }
  const std::vector<float2> pad = guarded(grid.lut);
  if ((rc = upload(pad.data(), pad.size(), &cb->grid_pad)) != RBQ_OK) { delete cb; return rc; }
  Grid full;
  if (build_grid_full(bounds, kMaxFullGridCells, &full) == RBQ_OK) {
    cb->grid_full_cells = full.cells;
    if ((rc = upload(full.lut.data(), full.lut.size(), &cb->grid_full)) != RBQ_OK) { delete cb; return rc; }
  }
  std::lock_guard<std::mutex> lk(g_mu);
  auto ins = cb_cache().emplace(key, cb);
  if (!ins.second) {          // another thread won the race; keep its copy
    cudaFree(cb->bounds);
    cudaFree(cb->levels_f16);
    cudaFree(cb->levels_i8);
    cudaFree(cb->levels_e4m3);
    cudaFree(cb->grid);
    cudaFree(cb->grid_full);
    cudaFree(cb->grid_pad);
    delete cb;
  }
  *out = ins.first->second;
  return RBQ_OK;
}

int device_error_word_ptr(unsigned int** out) {
  int dev;
  int rc = current_device(&dev);
  if (rc != RBQ_OK) return rc;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_err_word[dev]) {
    cudaError_t e = cudaMalloc(reinterpret_cast<void**>(&g_err_word[dev]), sizeof(unsigned int));
    if (e != cudaSuccess) { g_err_word[dev] = nullptr; return cuda_fail(e); }
    e = cudaMemset(g_err_word[dev], 0, sizeof(unsigned int));
    if (e != cudaSuccess) return cuda_fail(e);
  }
  *out = g_err_word[dev];
  return RBQ_OK;
}

}  // namespace rbq

// ===========================================================================
// Public entry points
// ===========================================================================
using namespace rbq;

extern "C" int rpbh_make(int d, int h, uint64_t seed, rbq_rpbh** out) {
  if (!out) return RBQ_EINVAL;
  *out = nullptr;
  if (h != kH || d <= 0 || d > kMaxD || d % h) return RBQ_EINVAL;
  auto* r = new (std::nothrow) rbq_rpbh;
  if (!r) return RBQ_ENOMEM;
  try {
    r->d = d;
    r->seed = seed;
    r->perm.resize(d);
    r->sign.resize(d);
  } catch (...) {
    delete r;
    return RBQ_ENOMEM;
  }
  for (int k = 0; k < d; ++k) r->perm[k] = k;
  SplitMix64 g(seed);
  for (int i = d - 1; i >= 1; --i) {
    const uint32_t j = mulhi_range(g.next(), static_cast<uint32_t>(i + 1));
    std::swap(r->perm[i], r->perm[j]);
  }
  for (int k = 0; k < d; ++k) r->sign[k] = (g.next() >> 63) ? -1 : 1;
  *out = r;
  return RBQ_OK;
}

extern "C" int rpbh_make_ablation(int d, int h, uint64_t seed, int flags, rbq_rpbh** out) {
  if (flags & ~(RBQ_RPBH_NO_PERMUTATION | RBQ_RPBH_NO_SIGNS)) {
    if (out) *out = nullptr;
    return RBQ_EINVAL;
  }
  const int rc = rpbh_make(d, h, seed, out);
  if (rc != RBQ_OK) return rc;
  rbq_rpbh* r = *out;
  r->flags = flags;
  if (flags & RBQ_RPBH_NO_PERMUTATION)
    for (int k = 0; k < d; ++k) r->perm[k] = k;
  if (flags & RBQ_RPBH_NO_SIGNS)
    for (int k = 0; k < d; ++k) r->sign[k] = 1;
  return RBQ_OK;
}

extern "C" void rpbh_free(rbq_rpbh* r) {
  if (!r) return;
  for (auto& D : r->dev) {
    if (!D.ready) continue;
    cudaFree(D.perm);
    cudaFree(D.sign);
    cudaFree(D.pair_tab);
    cudaFree(D.pair_tab16);
  }
  delete r;
}

extern "C" int rpbh_describe(const rbq_rpbh* r, int* d, int* h, uint64_t* seed, int* flags) {
  if (!r) return RBQ_EINVAL;
  if (d) *d = r->d;
  if (h) *h = kH;
  if (seed) *seed = r->seed;
  if (flags) *flags = r->flags;
  return RBQ_OK;
}

extern "C" int rpbh_export(const rbq_rpbh* r, int32_t* perm_host, int8_t* signs_host) {
  if (!r) return RBQ_EINVAL;
  if (perm_host) std::memcpy(perm_host, r->perm.data(), r->perm.size() * sizeof(int32_t));
  if (signs_host) std::memcpy(signs_host, r->sign.data(), r->sign.size());
  return RBQ_OK;
}

extern "C" int rpbh_dim(const rbq_rpbh* r) { return r ? r->d : RBQ_EINVAL; }

extern "C" int lloydmax_table(int d, int bits, double* levels, double* bounds) {
  if (d <= 0 || bits < 1 || bits > 8) return RBQ_EINVAL;
  std::vector<double> lv, bd;
  const int rc = full_table(d, bits, lv, bd);
  if (rc != RBQ_OK) return rc;
  if (levels) std::memcpy(levels, lv.data(), lv.size() * sizeof(double));
  if (bounds) std::memcpy(bounds, bd.data(), bd.size() * sizeof(double));
  return RBQ_OK;
}

extern "C" int rbq_int8_levels(int d, int bits, int8_t* levels, double* alpha) {
  if (d <= 0 || bits < 1 || bits > 8) return RBQ_EINVAL;
  std::vector<double> lv, bd;
  const int rc = full_table(d, bits, lv, bd);
  if (rc != RBQ_OK) return rc;
  std::vector<int8_t> li;
  double a = 0.0;
  int8_levels(lv, li, &a);
  if (levels) std::memcpy(levels, li.data(), li.size());
  if (alpha) *alpha = a;
  return RBQ_OK;
}

extern "C" int rbq_fp8_levels(int d, int bits, uint8_t* levels, double* beta) {
  if (d <= 0 || bits < 1 || bits > 8) return RBQ_EINVAL;
  std::vector<double> lv, bd;
  const int rc = full_table(d, bits, lv, bd);
  if (rc != RBQ_OK) return rc;
  std::vector<uint8_t> lf;
  double b = 0.0;
  fp8_levels(lv, lf, &b);
  if (levels) std::memcpy(levels, lf.data(), lf.size());
  if (beta) *beta = b;
  return RBQ_OK;
}

extern "C" const char* rbq_error_string(int code) {
  switch (code) {
    case RBQ_OK: return "ok";
    case RBQ_EINVAL: return "invalid argument";
    case RBQ_EALIGN: return "misaligned pointer";
    case RBQ_ECUDA: return cudaGetErrorString(g_last_cuda);
    case RBQ_ENOMEM: return "out of host memory";
    case RBQ_ECONVERGE: return "Lloyd-Max solver did not converge";
    case RBQ_EDEVICE: return "kernel reported an internal error (bounded wait expired)";
    case RBQ_ESCRATCH: return "problem exceeds the fixed scratch area (qlinear_noalloc: N*K <= 16777216)";
    case RBQ_EIO: return "layer file could not be opened, read or written, or is not a valid layer file";
    default: return "unknown error code";
  }
}

extern "C" int rbq_device_error(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  unsigned int* w = nullptr;
  int rc = device_error_word_ptr(&w);
  if (rc != RBQ_OK) return rc;
  unsigned int v = 0;
  e = cudaMemcpy(&v, w, sizeof(v), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e);
  if (v) {
    e = cudaMemset(w, 0, sizeof(v));
    if (e != cudaSuccess) return cuda_fail(e);
    return RBQ_EDEVICE;
  }
  return RBQ_OK;
}

extern "C" int rbq_code_grid(int d, int bits, int variant, float* thr, int32_t* base, int* cells,
                             float* scale) {
  if (d <= 0 || bits < 1 || bits > 8 || (variant != 0 && variant != 1)) return RBQ_EINVAL;
  std::vector<double> levels, bounds;
  int rc = full_table(d, bits, levels, bounds);
  if (rc != RBQ_OK) return rc;
  Grid g;
  rc = variant ? build_grid_full(bounds, kMaxFullGridCells, &g) : build_grid(bounds, &g);
  if (rc != RBQ_OK) return rc;
  for (size_t n = 0; n < g.lut.size(); ++n) {
    if (thr) thr[n] = g.lut[n].x;
    if (base) {
      int b;
      std::memcpy(&b, &g.lut[n].y, sizeof(b));
      base[n] = b;
    }
  }
  if (cells) *cells = g.cells;
  if (scale) *scale = static_cast<float>(1.0 / (2.0 * g.R));
  return RBQ_OK;
}
