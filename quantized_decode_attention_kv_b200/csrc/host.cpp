// C-ABI host layer of libtq: argument validation, the Gaussian Lloyd-Max codebook (double),
// the seeded sign vector and QJL matrix (SplitMix64 + Box-Muller), split planning, and the
// calls into the CUDA launchers. Nothing here allocates device memory or synchronises.
#include "../../include/tq.h"
#include "tq_internal.h"

#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

namespace {

thread_local std::string g_err;

int fail(int code, const char *fmt, ...) __attribute__((format(printf, 2, 3)));
int fail(int code, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_err = buf;
  return code;
}

// ---------------------------------------------------------------- SplitMix64
// Steele, Lea & Flood, "Fast splittable pseudorandom number generators" (OOPSLA 2014):
// output k (k >= 0) from seed s is mix(s + (k+1) * 0x9E3779B97F4A7C15).
uint64_t splitmix64_at(uint64_t seed, uint64_t k) {
  uint64_t z = seed + (k + 1) * 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

bool pow2_in(int v, int lo, int hi) { return v >= lo && v <= hi && (v & (v - 1)) == 0; }

// ---------------------------------------------------------------- Lloyd-Max (double)
// Gaussian Lloyd-Max quantiser ("Closing - The Three-Step Summary", Step 2): alternate
// boundaries = midpoints of neighbouring centroids and centroids = conditional means of
// N(0,1) on their cells, until no centroid moves by more than 1e-13.
double npdf(double x) { return std::isinf(x) ? 0.0 : std::exp(-0.5 * x * x) * 0.3989422804014327; }
double ncdf(double x) { return 0.5 * std::erfc(-x * 0.7071067811865476); }

double ninv(double p) { // bisection on the CDF; only the starting point depends on it
  double lo = -40.0, hi = 40.0;
  for (int i = 0; i < 200; ++i) {
    double mid = 0.5 * (lo + hi);
    (ncdf(mid) < p ? lo : hi) = mid;
  }
  return 0.5 * (lo + hi);
}

struct DoubleCodebook {
  double c[16], beta[15];
  int levels;
  bool ok;
  double fix_scale;
};

// Scale S of the centroids as 16-bit fixed-point integers rint(c_j S), |rint(c_j S)| <= 32639,
// chosen among 40000 candidates in [0.6, 1] x the largest admissible one to minimise the
// rounding error sum_j P_j (rint(c_j S) - c_j S)^2 / S^2 (P_j: the probability of level j under
// N(0, 1)); the products are rounded in float32, as the decode kernel forms them.
double fixed_point_scale(const double *c, int L) {
  double cmax = 0.0;
  for (int j = 0; j < L; ++j) cmax = std::fmax(cmax, std::fabs(c[j]));
  double prob[16];
  for (int j = 0; j < L; ++j) {
    const double lo = j == 0 ? -INFINITY : 0.5 * (c[j - 1] + c[j]);
    const double hi = j == L - 1 ? INFINITY : 0.5 * (c[j] + c[j + 1]);
    prob[j] = ncdf(hi) - ncdf(lo);
  }
  const double smax = 32639.0 / cmax;
  double best = smax, best_err = INFINITY;
  constexpr int kCand = 40000;
  for (int i = 0; i < kCand; ++i) {
    const float sf = static_cast<float>(smax * (1.0 - 0.4 * i / kCand));
    double err = 0.0;
    bool fits = true;
    for (int j = 0; j < L; ++j) {
      const float v = static_cast<float>(c[j]) * sf;
      const double r = std::nearbyint(static_cast<double>(v));
      fits = fits && std::fabs(r) <= 32639.0;
      const double e = (r - c[j] * static_cast<double>(sf)) / sf;
      err += prob[j] * e * e;
    }
    if (fits && err < best_err) {
      best_err = err;
      best = sf;
    }
  }
  return best;
}

// The E2M1 codebook on the N(0,1) scale: the 16 ascending levels s * (-6, -4, -3, -2, -1.5, -1,
// -0.5, -0, +0, 0.5, 1, 1.5, 2, 3, 4, 6) of Blackwell's FP4 format (+0 and -0 kept as two
// codes: a coordinate takes the zero of its sign), boundaries at the midpoints (0 between the
// zeros), s minimising the Gaussian MSE by golden-section search over [0.3, 0.8] ("Where This
// Fits in the Inference Stack", Blackwell FP4: can the codes live on the E2M1 grid).
double grid_mse(const double *c, int L) {
  double total = 0.0;
  for (int j = 0; j < L; ++j) {
    const double a = j == 0 ? -INFINITY : 0.5 * (c[j - 1] + c[j]);
    const double b = j == L - 1 ? INFINITY : 0.5 * (c[j] + c[j + 1]);
    const double p = ncdf(b) - ncdf(a);
    const double m1 = npdf(a) - npdf(b);
    const double m2 = p + (std::isinf(a) ? 0.0 : a * npdf(a)) - (std::isinf(b) ? 0.0 : b * npdf(b));
    total += m2 - 2.0 * c[j] * m1 + c[j] * c[j] * p;
  }
  return total;
}

DoubleCodebook compute_e2m1() {
  static const double grid[16] = {-6, -4, -3, -2, -1.5, -1, -0.5, -0.0, 0.0, 0.5, 1, 1.5, 2, 3, 4, 6};
  auto mse_at = [](double s) {
    double c[16];
    for (int j = 0; j < 16; ++j) c[j] = grid[j] * s;
    return grid_mse(c, 16);
  };
  const double g = 0.5 * (std::sqrt(5.0) - 1.0);
  double lo = 0.3, hi = 0.8, a = hi - g * (hi - lo), b = lo + g * (hi - lo);
  double fa = mse_at(a), fb = mse_at(b);
  while (hi - lo > 1e-12) {
    if (fa < fb) {
      hi = b;
      b = a;
      fb = fa;
      a = hi - g * (hi - lo);
      fa = mse_at(a);
    } else {
      lo = a;
      a = b;
      fa = fb;
      b = lo + g * (hi - lo);
      fb = mse_at(b);
    }
  }
  const double s = 0.5 * (lo + hi);
  DoubleCodebook cb{};
  cb.levels = 16;
  cb.ok = true;
  for (int j = 0; j < 16; ++j) cb.c[j] = grid[j] * s;
  for (int j = 0; j < 15; ++j) cb.beta[j] = 0.5 * (cb.c[j] + cb.c[j + 1]);
  cb.beta[7] = 0.0;
  cb.fix_scale = fixed_point_scale(cb.c, 16);
  return cb;
}

const DoubleCodebook &e2m1_codebook() {
  static DoubleCodebook table;
  static std::once_flag once;
  std::call_once(once, [] { table = compute_e2m1(); });
  return table;
}

DoubleCodebook compute_lloyd_max(int wbits) {
  DoubleCodebook cb{};
  const int L = 1 << wbits;
  cb.levels = L;
  double c[16], nc[16], edges[17];
  for (int j = 0; j < L; ++j) c[j] = ninv((j + 0.5) / L);
  cb.ok = false;
  for (int it = 0; it < 200000; ++it) {
    edges[0] = -INFINITY;
    edges[L] = INFINITY;
    for (int j = 0; j + 1 < L; ++j) edges[j + 1] = 0.5 * (c[j] + c[j + 1]);
    double moved = 0.0;
    for (int j = 0; j < L; ++j) {
      nc[j] = (npdf(edges[j]) - npdf(edges[j + 1])) / (ncdf(edges[j + 1]) - ncdf(edges[j]));
      moved = std::fmax(moved, std::fabs(nc[j] - c[j]));
    }
    std::memcpy(c, nc, sizeof(double) * L);
    if (moved < 1e-13) {
      cb.ok = true;
      break;
    }
  }
  // The Gaussian is symmetric, so the fixed point satisfies c_j = -c_{L-1-j}; enforce it
  // exactly so the middle boundary is exactly 0 (a zero coordinate takes the lower level).
  for (int j = 0; j < L / 2; ++j) {
    const double s = 0.5 * (c[L - 1 - j] - c[j]);
    c[L - 1 - j] = s;
    c[j] = -s;
  }
  for (int j = 0; j < L; ++j) cb.c[j] = c[j];
  for (int j = 0; j + 1 < L; ++j) cb.beta[j] = 0.5 * (c[j] + c[j + 1]);
  cb.fix_scale = fixed_point_scale(cb.c, L);
  return cb;
}

const DoubleCodebook &lloyd_max(int wbits) { // wbits in 1..4, computed once
  static DoubleCodebook table[5];
  static std::once_flag once[5];
  std::call_once(once[wbits], [wbits] { table[wbits] = compute_lloyd_max(wbits); });
  return table[wbits];
}

// ---------------------------------------------------------------- validation helpers
bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_qcfg(int d, const tq_qcfg &c, const char *name) {
  if (!pow2_in(d, 16, 256))
    return fail(TQ_ERR_UNSUPPORTED, "d=%d: head_dim must be a power of two in 16..256", d);
  if (c.bits < 1 || c.bits > 4)
    return fail(TQ_ERR_UNSUPPORTED, "%s.bits=%d: bits must be 1..4", name, c.bits);
  if (c.mode != TQ_MSE && c.mode != TQ_PROD && c.mode != TQ_E2M1)
    return fail(TQ_ERR_UNSUPPORTED, "%s.mode=%d: mode must be TQ_MSE, TQ_PROD or TQ_E2M1", name, c.mode);
  if (c.mode == TQ_E2M1 && c.bits != 4)
    return fail(TQ_ERR_UNSUPPORTED, "%s.bits=%d: TQ_E2M1 codes are 4 bits", name, c.bits);
  if (c.mode == TQ_PROD) {
    int m = c.qjl_m == 0 ? d : c.qjl_m;
    if (m < 8 || m > tq::kMaxM || m % 8)
      return fail(TQ_ERR_UNSUPPORTED, "%s.qjl_m=%d: must be 0 or a multiple of 8 in 8..%d",
                  name, c.qjl_m, tq::kMaxM);
  }
  return TQ_OK;
}

int resolve_tensor(const tq_cache &c, int which, tq::TensorArgs *t) {
  const tq_qcfg &q = which == 0 ? c.kc : c.vc;
  const char *name = which == 0 ? "kc" : "vc";
  int st = check_qcfg(c.d, q, name);
  if (st) return st;
  std::memset(t, 0, sizeof *t);
  t->bits = q.bits;
  t->mode = q.mode == TQ_PROD ? TQ_PROD : TQ_MSE; // E2M1 codes are MSE codes on another codebook
  t->wbits = q.mode == TQ_PROD ? q.bits - 1 : q.bits;
  t->m = q.mode == TQ_PROD ? (q.qjl_m == 0 ? c.d : q.qjl_m) : 0;
  t->code_bytes = c.d * t->wbits / 8;
  t->sign_bytes = t->m / 8;
  t->codes = which == 0 ? c.k_codes : c.v_codes;
  t->norm = which == 0 ? c.k_norm : c.v_norm;
  t->signs = which == 0 ? c.k_signs : c.v_signs;
  t->rnorm = which == 0 ? c.k_rnorm : c.v_rnorm;
  t->S = which == 0 ? c.k_qjl : c.v_qjl;
  const char *tn = which == 0 ? "K" : "V";
  if (t->wbits > 0 && (!t->codes || !aligned16(t->codes)))
    return fail(TQ_ERR_INVALID_ARG, "%s codes pointer is NULL or not 16-byte aligned", tn);
  if (!t->norm || !aligned16(t->norm))
    return fail(TQ_ERR_INVALID_ARG, "%s norm pointer is NULL or not 16-byte aligned", tn);
  if (q.mode == TQ_PROD) {
    if (!t->signs || !aligned16(t->signs) || !t->rnorm || !aligned16(t->rnorm) || !t->S ||
        !aligned16(t->S))
      return fail(TQ_ERR_INVALID_ARG,
                  "%s is TQ_PROD: signs, rnorm and qjl pointers must be non-NULL and 16-byte "
                  "aligned", tn);
  }
  tq::Codebook &cb = t->cb;
  std::memset(&cb, 0, sizeof cb);
  if (t->wbits == 0) {
    cb.levels = 1;
  } else {
    const DoubleCodebook &d = q.mode == TQ_E2M1 ? e2m1_codebook() : lloyd_max(t->wbits);
    if (!d.ok) return fail(TQ_ERR_UNSUPPORTED, "Lloyd-Max iteration did not converge");
    cb.levels = d.levels;
    for (int j = 0; j < d.levels; ++j) cb.c[j] = static_cast<float>(d.c[j]);
    for (int j = 0; j + 1 < d.levels; ++j) cb.beta[j] = static_cast<float>(d.beta[j]);
    cb.fix_scale = static_cast<float>(d.fix_scale);
  }
  return TQ_OK;
}

int check_cache(const tq_cache *c) {
  if (!c) return fail(TQ_ERR_INVALID_ARG, "cache is NULL");
  if (c->B < 1 || c->Hkv < 1 || c->T_cap < 1)
    return fail(TQ_ERR_INVALID_ARG, "cache shape B=%d Hkv=%d T_cap=%d must be positive", c->B,
                c->Hkv, c->T_cap);
  if (!pow2_in(c->d, 16, 256))
    return fail(TQ_ERR_UNSUPPORTED, "d=%d: head_dim must be a power of two in 16..256", c->d);
  if ((long long)c->B * c->Hkv * c->T_cap > (1ll << 40))
    return fail(TQ_ERR_INVALID_ARG, "cache too large");
  if (c->B > 65535 || c->Hkv > 4096)
    return fail(TQ_ERR_INVALID_ARG, "B=%d must be <= 65535 and Hkv=%d <= 4096", c->B, c->Hkv);
  return TQ_OK;
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
  return n;
}

int cuda_status(cudaError_t e, const char *what) {
  if (e == cudaSuccess) return TQ_OK;
  return fail(TQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool dtype_ok(int dt) { return dt == TQ_F32 || dt == TQ_BF16 || dt == TQ_F16; }

// Whether the cache's bit-widths and shape take a tensor-core decode kernel: 0 if not,
// kProdFast for the TurboQuant_prod kernel, else (key bits << 4) | value bits.
int fast_path(const tq_cache &c, int Hq) {
  const int kw = c.kc.mode == TQ_PROD ? c.kc.bits - 1 : c.kc.bits;
  const int vw = c.vc.mode == TQ_PROD ? c.vc.bits - 1 : c.vc.bits;
  const int km = c.kc.qjl_m ? c.kc.qjl_m : c.d, vm = c.vc.qjl_m ? c.vc.qjl_m : c.d;
  // the kernels see E2M1 tensors as MSE tensors with their own codebook
  const int kmode = c.kc.mode == TQ_PROD ? TQ_PROD : TQ_MSE, vmode = c.vc.mode == TQ_PROD ? TQ_PROD : TQ_MSE;
  if (tq::prod_decode_supported(c.d, c.kc.mode, c.kc.bits, km, c.vc.mode, c.vc.bits, vm, Hq / c.Hkv))
    return tq::kProdFast;
  return tq::fast_decode_supported(c.d, kmode, kw, vmode, vw, Hq / c.Hkv) ? (kw << 4) | vw : 0;
}

} // namespace

extern "C" {

const char *tq_last_error(void) { return g_err.c_str(); }

int tq_make_codebook(int bits, int d, float *centroids, float *bounds) {
  if (bits < 1 || bits > 4) return fail(TQ_ERR_UNSUPPORTED, "bits=%d: must be 1..4", bits);
  if (!pow2_in(d, 16, 256))
    return fail(TQ_ERR_UNSUPPORTED, "d=%d: head_dim must be a power of two in 16..256", d);
  if (!centroids || !bounds) return fail(TQ_ERR_INVALID_ARG, "output pointer is NULL");
  const DoubleCodebook &cb = lloyd_max(bits);
  if (!cb.ok) return fail(TQ_ERR_UNSUPPORTED, "Lloyd-Max iteration did not converge");
  const double s = 1.0 / std::sqrt(static_cast<double>(d));
  for (int j = 0; j < cb.levels; ++j) centroids[j] = static_cast<float>(cb.c[j] * s);
  for (int j = 0; j + 1 < cb.levels; ++j) bounds[j] = static_cast<float>(cb.beta[j] * s);
  return TQ_OK;
}

int tq_make_signs(uint64_t seed, int d, uint8_t *signs) {
  if (!pow2_in(d, 16, 256))
    return fail(TQ_ERR_UNSUPPORTED, "d=%d: head_dim must be a power of two in 16..256", d);
  if (!signs) return fail(TQ_ERR_INVALID_ARG, "signs is NULL");
  for (int byte = 0; byte < d / 8; ++byte) {
    uint64_t w = splitmix64_at(seed, static_cast<uint64_t>(byte / 8));
    signs[byte] = static_cast<uint8_t>(w >> (8 * (byte % 8)));
  }
  return TQ_OK;
}

int tq_make_qjl_matrix(uint64_t seed, int m, int d, float *S) {
  if (!pow2_in(d, 16, 256))
    return fail(TQ_ERR_UNSUPPORTED, "d=%d: head_dim must be a power of two in 16..256", d);
  if (m < 8 || m > tq::kMaxM || m % 8)
    return fail(TQ_ERR_UNSUPPORTED, "m=%d: must be a multiple of 8 in 8..%d", m, tq::kMaxM);
  if (!S) return fail(TQ_ERR_INVALID_ARG, "S is NULL");
  const long n = static_cast<long>(m) * d;
  const double two_pi = 6.283185307179586;
  for (long k = 0; k < n / 2; ++k) {
    double u0 = static_cast<double>(splitmix64_at(seed, 2 * k) >> 11) * 0x1.0p-53;
    double u1 = static_cast<double>(splitmix64_at(seed, 2 * k + 1) >> 11) * 0x1.0p-53;
    double rho = std::sqrt(-2.0 * std::log(1.0 - u0));
    double th = two_pi * u1;
    S[2 * k] = static_cast<float>(rho * std::cos(th));
    S[2 * k + 1] = static_cast<float>(rho * std::sin(th));
  }
  return TQ_OK;
}

size_t tq_code_bytes(int d, tq_qcfg c) {
  if (check_qcfg(d, c, "cfg")) return 0;
  int w = c.mode == TQ_PROD ? c.bits - 1 : c.bits;
  return static_cast<size_t>(d) * w / 8;
}

size_t tq_sign_bytes(int d, tq_qcfg c) {
  if (check_qcfg(d, c, "cfg")) return 0;
  return c.mode == TQ_PROD ? static_cast<size_t>(c.qjl_m == 0 ? d : c.qjl_m) / 8 : 0;
}

size_t tq_record_bytes(int d, tq_qcfg c) {
  if (check_qcfg(d, c, "cfg")) return 0;
  return tq_code_bytes(d, c) + tq_sign_bytes(d, c) + (c.mode == TQ_PROD ? 4 : 2);
}

// Shared body of the dense and paged writes (cache: the dense descriptor or a paged cache's
// view; pg.bt == nullptr for the dense layout).
static int quantize_impl(const void *K, const void *V, int dtype, int T, int t_offset,
                         const tq_cache *cache, const tq::Paging &pg, void *stream);

int tq_quantize_kv(const void *K, const void *V, int dtype, int T, int t_offset,
                   const tq_cache *cache, void *stream) {
  int st = check_cache(cache);
  if (st) return st;
  return quantize_impl(K, V, dtype, T, t_offset, cache, tq::Paging{nullptr, -1, 0}, stream);
}

static int quantize_impl(const void *K, const void *V, int dtype, int T, int t_offset,
                         const tq_cache *cache, const tq::Paging &pg, void *stream) {
  int st = TQ_OK;
  if (!dtype_ok(dtype)) return fail(TQ_ERR_INVALID_ARG, "dtype=%d is not F32/BF16/F16", dtype);
  if (T < 0 || t_offset < 0 || (long long)t_offset + T > cache->T_cap)
    return fail(TQ_ERR_INVALID_ARG, "positions [%d, %d) fall outside T_cap=%d", t_offset,
                t_offset + T, cache->T_cap);
  if (!K && !V) return fail(TQ_ERR_INVALID_ARG, "K and V are both NULL");
  if ((K && !aligned16(K)) || (V && !aligned16(V)))
    return fail(TQ_ERR_INVALID_ARG, "K/V input pointers must be 16-byte aligned");
  tq::QuantArgs a[2];
  for (int which = 0; which < 2; ++which) {
    const void *x = which == 0 ? K : V;
    if (!x) continue;
    st = resolve_tensor(*cache, which, &a[which].t);
    if (st) return st;
  }
  if (T == 0) return TQ_OK;
  for (int which = 0; which < 2; ++which) {
    const void *x = which == 0 ? K : V;
    if (!x) continue;
    tq::QuantArgs &q = a[which];
    q.x = x;
    q.dtype = dtype;
    q.B = cache->B;
    q.Hkv = cache->Hkv;
    q.T = T;
    q.T_cap = cache->T_cap;
    q.t_offset = t_offset;
    q.d = cache->d;
    q.seed = cache->seed;
    for (int k = 0; k < 4; ++k) q.sign_words[k] = splitmix64_at(cache->seed, static_cast<uint64_t>(k));
    q.pg = pg;
  }
  // 16-bit MSE tensors take the streaming kernel, 16-bit d=64 TurboQuant_prod tensors the
  // tensor-core sketch kernel (each with K and V in one launch); the rest, the per-vector
  // kernel.
  const tq::QuantArgs *fast[2] = {nullptr, nullptr}, *prod[2] = {nullptr, nullptr};
  for (int which = 0; which < 2; ++which) {
    const void *x = which == 0 ? K : V;
    if (!x) continue;
    if (tq::quantize_fast_supported(a[which])) fast[which] = &a[which];
    else if (tq::quantize_prod_supported(a[which])) prod[which] = &a[which];
    // the paged layout is written by the 16-bit MSE and TurboQuant_prod (d = 64, m = 64) kernels
    if (pg.bt && !fast[which] && !prod[which])
      return fail(TQ_ERR_UNSUPPORTED, "paged writes need 16-bit input and a head_dim-128 TurboQuant_mse "
                                      "or head_dim-64 TurboQuant_prod (m = 64) tensor");
  }
  if (fast[0] || fast[1] || prod[0] || prod[1]) {
    const int sms = sm_count();
    if (sms <= 0) return fail(TQ_ERR_CUDA, "cannot query the device's SM count");
    if (fast[0] || fast[1]) {
      st = cuda_status(tq::launch_quantize_fast(fast[0], fast[1], sms, static_cast<cudaStream_t>(stream)),
                       "quantize launch");
      if (st) return st;
    }
    if (prod[0] || prod[1]) {
      st = cuda_status(tq::launch_quantize_prod(prod[0], prod[1], sms, static_cast<cudaStream_t>(stream)),
                       "quantize launch");
      if (st) return st;
    }
  }
  for (int which = 0; which < 2; ++which) {
    const void *x = which == 0 ? K : V;
    if (!x || fast[which] || prod[which]) continue;
    st = cuda_status(tq::launch_quantize(a[which], static_cast<cudaStream_t>(stream)), "quantize launch");
    if (st) return st;
  }
  return TQ_OK;
}

size_t tq_decode_workspace_bytes(int B, int Hq, int T_len, const tq_cache *cache) {
  if (check_cache(cache)) return 0;
  if (Hq < 1 || Hq % cache->Hkv || T_len < 1 || T_len > cache->T_cap) {
    fail(TQ_ERR_INVALID_ARG, "bad Hq=%d or T_len=%d", Hq, T_len);
    return 0;
  }
  if (B != cache->B) {
    fail(TQ_ERR_INVALID_ARG, "B=%d differs from cache B=%d", B, cache->B);
    return 0;
  }
  if (check_qcfg(cache->d, cache->kc, "kc") || check_qcfg(cache->d, cache->vc, "vc")) return 0;
  int sms = sm_count();
  if (sms <= 0) {
    fail(TQ_ERR_CUDA, "cannot query the device's SM count");
    return 0;
  }
  int vm = cache->vc.mode == TQ_PROD ? (cache->vc.qjl_m ? cache->vc.qjl_m : cache->d) : 0;
  return tq::plan_decode(cache->B, Hq, cache->Hkv, cache->d, T_len, vm, sms, false,
                         fast_path(*cache, Hq)).ws_bytes;
}

int tq_decode_attention(const void *q, int dtype, int Hq, int T_len, float scale,
                        const tq_cache *cache, float *out, void *ws, size_t ws_bytes,
                        void *stream) {
  int st = check_cache(cache);
  if (st) return st;
  if (!dtype_ok(dtype)) return fail(TQ_ERR_INVALID_ARG, "dtype=%d is not F32/BF16/F16", dtype);
  if (!q || !out || !aligned16(q) || !aligned16(out))
    return fail(TQ_ERR_INVALID_ARG, "q/out must be non-NULL and 16-byte aligned");
  if (Hq < 1 || Hq % cache->Hkv || Hq > 65535)
    return fail(TQ_ERR_INVALID_ARG, "Hq=%d must be a positive multiple of Hkv=%d (<= 65535)", Hq,
                cache->Hkv);
  if (T_len < 1 || T_len > cache->T_cap)
    return fail(TQ_ERR_INVALID_ARG, "T_len=%d must be in 1..T_cap=%d", T_len, cache->T_cap);
  if (!std::isfinite(scale)) return fail(TQ_ERR_INVALID_ARG, "scale is not finite");
  tq::DecodeArgs a;
  std::memset(&a, 0, sizeof a);
  st = resolve_tensor(*cache, 0, &a.k);
  if (st) return st;
  st = resolve_tensor(*cache, 1, &a.v);
  if (st) return st;
  int sms = sm_count();
  if (sms <= 0) return fail(TQ_ERR_CUDA, "cannot query the device's SM count");
  a.plan = tq::plan_decode(cache->B, Hq, cache->Hkv, cache->d, T_len, a.v.m, sms, false,
                           fast_path(*cache, Hq));
  if (!ws || !aligned16(ws) || ws_bytes < a.plan.ws_bytes)
    return fail(TQ_ERR_WORKSPACE, "workspace needs %zu bytes (16-byte aligned), got %zu",
                a.plan.ws_bytes, ws ? ws_bytes : 0);
  a.q = q;
  a.q_dtype = dtype;
  a.B = cache->B;
  a.Hq = Hq;
  a.Hkv = cache->Hkv;
  a.d = cache->d;
  a.T_len = T_len;
  a.T_cap = cache->T_cap;
  a.scale = scale;
  a.seed = cache->seed;
  a.out = out;
  a.ws = static_cast<float *>(ws);
  return cuda_status(tq::launch_decode(a, static_cast<cudaStream_t>(stream)), "decode launch");
}

// Ragged decode: validation shared by the size query and the call. Returns TQ_OK and the
// longest length, or an error.
static int check_varlen(const tq_cache *cache, int Hq, const int *T_lens, int *T_max) {
  int st = check_cache(cache);
  if (st) return st;
  if (Hq < 1 || Hq % cache->Hkv || Hq > 65535)
    return fail(TQ_ERR_INVALID_ARG, "Hq=%d must be a positive multiple of Hkv=%d (<= 65535)", Hq,
                cache->Hkv);
  if (!T_lens) return fail(TQ_ERR_INVALID_ARG, "T_lens is NULL");
  if (cache->B > tq::kMaxVarlenB)
    return fail(TQ_ERR_UNSUPPORTED, "ragged decode supports B <= %d, got %d", tq::kMaxVarlenB, cache->B);
  int mx = 0;
  for (int b = 0; b < cache->B; ++b) {
    if (T_lens[b] < 1 || T_lens[b] > cache->T_cap)
      return fail(TQ_ERR_INVALID_ARG, "T_lens[%d]=%d must be in 1..T_cap=%d", b, T_lens[b], cache->T_cap);
    mx = std::max(mx, T_lens[b]);
  }
  const int fp = fast_path(*cache, Hq);
  if (fp == 0)
    return fail(TQ_ERR_UNSUPPORTED, "ragged decode needs a tensor-core configuration (d = 128, MSE, "
                                    "3/4-bit K, 2..4-bit V, <= 8 query heads per KV head; or d = 64, "
                                    "2-bit TurboQuant_prod K and V with 64 sketch rows, <= 2 query heads "
                                    "per KV head)");
  *T_max = mx;
  return TQ_OK;
}

// Plan of a ragged call for the configuration's tensor-core kernel.
static void plan_varlen(const tq_cache &c, int Hq, int mx, int sms, const int *T_lens, tq::DecodePlan *p) {
  const int fp = fast_path(c, Hq);
  if (fp == tq::kProdFast)
    tq::plan_prod(c.B, Hq, c.Hkv, mx, sms, p, T_lens);
  else
    tq::plan_fast(c.B, Hq, c.Hkv, mx, sms, fp >> 4, fp & 15, p, T_lens);
}

size_t tq_decode_varlen_workspace_bytes(int Hq, const tq_cache *cache, const int *T_lens) {
  int mx = 0;
  if (check_varlen(cache, Hq, T_lens, &mx)) return 0;
  int sms = sm_count();
  if (sms <= 0) {
    fail(TQ_ERR_CUDA, "cannot query the device's SM count");
    return 0;
  }
  tq::DecodePlan p{};
  plan_varlen(*cache, Hq, mx, sms, T_lens, &p);
  return p.ws_bytes;
}

static int decode_varlen_impl(const void *q, int dtype, int Hq, const int *T_lens, float scale,
                              const tq_cache *cache, const tq::Paging &pg, float *out, void *ws,
                              size_t ws_bytes, void *stream) {
  int mx = 0;
  int st = check_varlen(cache, Hq, T_lens, &mx);
  if (st) return st;
  if (!dtype_ok(dtype)) return fail(TQ_ERR_INVALID_ARG, "dtype=%d is not F32/BF16/F16", dtype);
  if (!q || !out || !aligned16(q) || !aligned16(out))
    return fail(TQ_ERR_INVALID_ARG, "q/out must be non-NULL and 16-byte aligned");
  if (!std::isfinite(scale)) return fail(TQ_ERR_INVALID_ARG, "scale is not finite");
  tq::DecodeArgs a;
  std::memset(&a, 0, sizeof a);
  st = resolve_tensor(*cache, 0, &a.k);
  if (st) return st;
  st = resolve_tensor(*cache, 1, &a.v);
  if (st) return st;
  int sms = sm_count();
  if (sms <= 0) return fail(TQ_ERR_CUDA, "cannot query the device's SM count");
  plan_varlen(*cache, Hq, mx, sms, T_lens, &a.plan);
  if (!ws || !aligned16(ws) || ws_bytes < a.plan.ws_bytes)
    return fail(TQ_ERR_WORKSPACE, "workspace needs %zu bytes (16-byte aligned), got %zu",
                a.plan.ws_bytes, ws ? ws_bytes : 0);
  a.T_lens = T_lens;
  a.pg = pg;
  a.q = q;
  a.q_dtype = dtype;
  a.B = cache->B;
  a.Hq = Hq;
  a.Hkv = cache->Hkv;
  a.d = cache->d;
  a.T_len = mx;
  a.T_cap = cache->T_cap;
  a.scale = scale;
  a.seed = cache->seed;
  a.out = out;
  a.ws = static_cast<float *>(ws);
  return cuda_status(a.plan.path == 2 ? tq::launch_prod_decode(a, static_cast<cudaStream_t>(stream))
                                      : tq::launch_fast_decode(a, static_cast<cudaStream_t>(stream)),
                     "decode launch");
}

int tq_decode_attention_varlen(const void *q, int dtype, int Hq, const int *T_lens, float scale,
                               const tq_cache *cache, float *out, void *ws, size_t ws_bytes,
                               void *stream) {
  return decode_varlen_impl(q, dtype, Hq, T_lens, scale, cache, tq::Paging{nullptr, -1, 0}, out, ws,
                            ws_bytes, stream);
}

// A paged cache seen as the dense descriptor the shared checks and resolvers read (T_cap: one
// sequence's capacity; the pointers: the page pools), plus its paging.
static int paged_view(const tq_paged_cache *pc, tq_cache *view, tq::Paging *pg) {
  if (!pc) return fail(TQ_ERR_INVALID_ARG, "cache is NULL");
  if (pc->B < 1 || pc->Hkv < 1 || pc->num_pages < 1 || pc->max_pages < 1)
    return fail(TQ_ERR_INVALID_ARG, "bad paged cache shape B=%d Hkv=%d num_pages=%d max_pages=%d",
                pc->B, pc->Hkv, pc->num_pages, pc->max_pages);
  if (pc->page_size < 16 || (pc->page_size & (pc->page_size - 1)))
    return fail(TQ_ERR_INVALID_ARG, "page_size=%d must be a power of two >= 16", pc->page_size);
  if (!pc->block_table) return fail(TQ_ERR_INVALID_ARG, "block_table is NULL");
  const bool mse = pc->kc.mode != TQ_PROD && pc->vc.mode != TQ_PROD; // MSE or E2M1 codes
  const bool prod = pc->kc.mode == TQ_PROD && pc->vc.mode == TQ_PROD;
  if (!(mse && pc->d == 128) && !(prod && pc->d == 64))
    return fail(TQ_ERR_UNSUPPORTED, "paged caches hold head_dim-128 TurboQuant_mse or head_dim-64 "
                                    "TurboQuant_prod records (d=%d, modes %d/%d)", pc->d, pc->kc.mode, pc->vc.mode);
  const long long cap = static_cast<long long>(pc->max_pages) * pc->page_size;
  const long long recs = static_cast<long long>(pc->num_pages) * pc->Hkv * pc->page_size;
  if (cap > (1ll << 30) || recs > (1ll << 40))
    return fail(TQ_ERR_INVALID_ARG, "paged cache too large (capacity %lld positions)", cap);
  std::memset(view, 0, sizeof *view);
  view->B = pc->B;
  view->Hkv = pc->Hkv;
  view->T_cap = static_cast<int>(cap);
  view->d = pc->d;
  view->seed = pc->seed;
  view->kc = pc->kc;
  view->vc = pc->vc;
  view->k_codes = pc->k_codes;
  view->v_codes = pc->v_codes;
  view->k_norm = pc->k_norm;
  view->v_norm = pc->v_norm;
  view->k_signs = pc->k_signs;
  view->v_signs = pc->v_signs;
  view->k_rnorm = pc->k_rnorm;
  view->v_rnorm = pc->v_rnorm;
  view->k_qjl = pc->k_qjl;
  view->v_qjl = pc->v_qjl;
  int st = check_cache(view);
  if (st) return st;
  int shift = 0;
  while ((1 << shift) < pc->page_size) ++shift;
  *pg = tq::Paging{pc->block_table, shift, pc->max_pages};
  return TQ_OK;
}

int tq_quantize_kv_paged(const void *K, const void *V, int dtype, int T, int t_offset,
                         const tq_paged_cache *cache, void *stream) {
  tq_cache view;
  tq::Paging pg;
  int st = paged_view(cache, &view, &pg);
  if (st) return st;
  return quantize_impl(K, V, dtype, T, t_offset, &view, pg, stream);
}

size_t tq_decode_paged_workspace_bytes(int Hq, const tq_paged_cache *cache, const int *T_lens) {
  tq_cache view;
  tq::Paging pg;
  if (paged_view(cache, &view, &pg)) return 0;
  return tq_decode_varlen_workspace_bytes(Hq, &view, T_lens);
}

int tq_decode_attention_paged(const void *q, int dtype, int Hq, const int *T_lens, float scale,
                              const tq_paged_cache *cache, float *out, void *ws, size_t ws_bytes,
                              void *stream) {
  tq_cache view;
  tq::Paging pg;
  int st = paged_view(cache, &view, &pg);
  if (st) return st;
  return decode_varlen_impl(q, dtype, Hq, T_lens, scale, &view, pg, out, ws, ws_bytes, stream);
}

int tq_decode_attention_noalloc(const void *q, int dtype, int Hq, int T_len, float scale,
                                const tq_cache *cache, float *out, void *stream) {
  // Same arguments and checks as tq_decode_attention, minus the workspace: the split-K
  // partials go to the library's fixed device scratch, so this call allocates nothing.
  int st = check_cache(cache);
  if (st) return st;
  if (!dtype_ok(dtype)) return fail(TQ_ERR_INVALID_ARG, "dtype=%d is not F32/BF16/F16", dtype);
  if (!q || !out || !aligned16(q) || !aligned16(out))
    return fail(TQ_ERR_INVALID_ARG, "q/out must be non-NULL and 16-byte aligned");
  if (Hq < 1 || Hq % cache->Hkv || Hq > 65535)
    return fail(TQ_ERR_INVALID_ARG, "Hq=%d must be a positive multiple of Hkv=%d (<= 65535)", Hq,
                cache->Hkv);
  if (T_len < 1 || T_len > cache->T_cap)
    return fail(TQ_ERR_INVALID_ARG, "T_len=%d must be in 1..T_cap=%d", T_len, cache->T_cap);
  if (!std::isfinite(scale)) return fail(TQ_ERR_INVALID_ARG, "scale is not finite");
  tq::DecodeArgs a;
  std::memset(&a, 0, sizeof a);
  st = resolve_tensor(*cache, 0, &a.k);
  if (st) return st;
  st = resolve_tensor(*cache, 1, &a.v);
  if (st) return st;
  int sms = sm_count();
  if (sms <= 0) return fail(TQ_ERR_CUDA, "cannot query the device's SM count");
  a.plan = tq::plan_decode(cache->B, Hq, cache->Hkv, cache->d, T_len, a.v.m, sms, false,
                           fast_path(*cache, Hq));
  float *scratch = nullptr;
  size_t cap = 0;
  st = cuda_status(tq::fixed_scratch(&scratch, &cap), "fixed scratch lookup");
  if (st) return st;
  if (a.plan.ws_bytes > cap)
    return fail(TQ_ERR_WORKSPACE,
                "this shape needs %zu bytes of split-K scratch but the fixed scratch holds %zu; "
                "call tq_decode_attention with a caller-owned workspace instead",
                a.plan.ws_bytes, cap);
  a.q = q;
  a.q_dtype = dtype;
  a.B = cache->B;
  a.Hq = Hq;
  a.Hkv = cache->Hkv;
  a.d = cache->d;
  a.T_len = T_len;
  a.T_cap = cache->T_cap;
  a.scale = scale;
  a.seed = cache->seed;
  a.out = out;
  a.ws = scratch;
  return cuda_status(tq::launch_decode(a, static_cast<cudaStream_t>(stream)),
                     "decode (fixed scratch) launch");
}

int tq_prefill_attention(const void *q, int dtype, int Hq, int Lq, int t0, float scale,
                         const tq_cache *cache, float *out, void *stream) {
  int st = check_cache(cache);
  if (st) return st;
  if (!dtype_ok(dtype)) return fail(TQ_ERR_INVALID_ARG, "dtype=%d is not F32/BF16/F16", dtype);
  if (!q || !out || !aligned16(q) || !aligned16(out))
    return fail(TQ_ERR_INVALID_ARG, "q/out must be non-NULL and 16-byte aligned");
  if (Hq < 1 || Hq % cache->Hkv || Hq > 65535)
    return fail(TQ_ERR_INVALID_ARG, "Hq=%d must be a positive multiple of Hkv=%d (<= 65535)", Hq,
                cache->Hkv);
  if (Lq < 1 || t0 < 0 || static_cast<long long>(t0) + Lq > cache->T_cap)
    return fail(TQ_ERR_INVALID_ARG, "Lq=%d, t0=%d: need Lq >= 1, t0 >= 0, t0 + Lq <= T_cap=%d", Lq, t0,
                cache->T_cap);
  if (!std::isfinite(scale)) return fail(TQ_ERR_INVALID_ARG, "scale is not finite");
  tq::PrefillLaunch l;
  std::memset(&l, 0, sizeof l);
  st = resolve_tensor(*cache, 0, &l.k);
  if (st) return st;
  st = resolve_tensor(*cache, 1, &l.v);
  if (st) return st;
  if (!tq::prefill_supported(cache->d, l.k.mode, l.k.wbits, l.v.mode, l.v.wbits, Hq / cache->Hkv))
    return fail(TQ_ERR_UNSUPPORTED,
                "prefill supports head_dim 128, TurboQuant_mse keys of 3/4 bits and values of 2..4 bits, "
                "and Hq/Hkv dividing 128");
  const long long ctas = static_cast<long long>(cache->B) * cache->Hkv *
                         ((Lq + 128 / (Hq / cache->Hkv) - 1) / (128 / (Hq / cache->Hkv)));
  if (ctas > 0x7FFFFFFF) return fail(TQ_ERR_INVALID_ARG, "too many query blocks");
  l.q = q;
  l.q_dtype = dtype;
  l.B = cache->B;
  l.Hq = Hq;
  l.Hkv = cache->Hkv;
  l.Lq = Lq;
  l.t0 = t0;
  l.T_cap = cache->T_cap;
  l.scale = scale;
  l.seed = cache->seed;
  l.out = out;
  l.k_e2m1 = cache->kc.mode == TQ_E2M1;
  return cuda_status(tq::launch_prefill(l, static_cast<cudaStream_t>(stream)), "prefill launch");
}

int tq_device_faults(unsigned *flags) {
  if (!flags) return fail(TQ_ERR_INVALID_ARG, "flags is NULL");
  unsigned prod = 0, pre = 0;
  int st = cuda_status(tq::read_and_clear_prod_faults(&prod), "tq_device_faults");
  if (st) return st;
  st = cuda_status(tq::read_and_clear_prefill_faults(&pre), "tq_device_faults");
  if (st) return st;
  *flags = (prod ? 1u : 0u) | (pre ? 2u : 0u);
  return TQ_OK;
}

int tq_launch_counts(const tq_cache *cache, int dtype, int T, int Hq, int T_len,
                     int *quantize_launches, int *decode_launches) {
  int st = check_cache(cache);
  if (st) return st;
  if (!dtype_ok(dtype)) return fail(TQ_ERR_INVALID_ARG, "dtype=%d is not F32/BF16/F16", dtype);
  if (T < 0 || T > cache->T_cap) return fail(TQ_ERR_INVALID_ARG, "T=%d outside [0, T_cap]", T);
  if (Hq < 1 || Hq % cache->Hkv || Hq > 65535 || T_len < 1 || T_len > cache->T_cap)
    return fail(TQ_ERR_INVALID_ARG, "bad Hq=%d or T_len=%d", Hq, T_len);
  int nq = 0;
  bool any_fast = false, any_prod = false;
  for (int which = 0; which < 2 && T > 0; ++which) {
    tq::QuantArgs q{};
    st = resolve_tensor(*cache, which, &q.t);
    if (st) return st;
    q.dtype = dtype;
    q.B = cache->B;
    q.Hkv = cache->Hkv;
    q.T = T;
    q.d = cache->d;
    if (tq::quantize_fast_supported(q)) any_fast = true;
    else if (tq::quantize_prod_supported(q)) any_prod = true;
    else ++nq;
  }
  if (quantize_launches) *quantize_launches = nq + (any_fast ? 1 : 0) + (any_prod ? 1 : 0);
  // split-K kernel and combine; the TurboQuant_prod kernels add a query-prep kernel (the MSE
  // tensor-core kernel and the generic kernel prepare their queries themselves)
  if (decode_launches) *decode_launches = fast_path(*cache, Hq) == tq::kProdFast ? 3 : 2;
  return TQ_OK;
}

int tq_dequantize(const tq_cache *cache, int which, int T_len, void *out, int dtype,
                  void *stream) {
  int st = check_cache(cache);
  if (st) return st;
  if (which != 0 && which != 1) return fail(TQ_ERR_INVALID_ARG, "which=%d must be 0 or 1", which);
  if (!dtype_ok(dtype)) return fail(TQ_ERR_INVALID_ARG, "dtype=%d is not F32/BF16/F16", dtype);
  if (T_len < 0 || T_len > cache->T_cap)
    return fail(TQ_ERR_INVALID_ARG, "T_len=%d must be in 0..T_cap=%d", T_len, cache->T_cap);
  if (!out || !aligned16(out))
    return fail(TQ_ERR_INVALID_ARG, "out must be non-NULL and 16-byte aligned");
  tq::DequantArgs a;
  std::memset(&a, 0, sizeof a);
  st = resolve_tensor(*cache, which, &a.t);
  if (st) return st;
  if (T_len == 0) return TQ_OK;
  a.out = out;
  a.dtype = dtype;
  a.B = cache->B;
  a.Hkv = cache->Hkv;
  a.T_len = T_len;
  a.T_cap = cache->T_cap;
  a.d = cache->d;
  a.seed = cache->seed;
  return cuda_status(tq::launch_dequantize(a, static_cast<cudaStream_t>(stream)),
                     "dequantize launch");
}

size_t tq_decode_bf16_workspace_bytes(int B, int Hq, int Hkv, int T_len, int d) {
  if (B < 1 || Hkv < 1 || Hq < 1 || Hq % Hkv || T_len < 1 || !pow2_in(d, 16, 256)) {
    fail(TQ_ERR_INVALID_ARG, "bad shape B=%d Hq=%d Hkv=%d T_len=%d d=%d", B, Hq, Hkv, T_len, d);
    return 0;
  }
  int sms = sm_count();
  if (sms <= 0) {
    fail(TQ_ERR_CUDA, "cannot query the device's SM count");
    return 0;
  }
  return tq::plan_decode(B, Hq, Hkv, d, T_len, 0, sms, true).ws_bytes;
}

int tq_decode_attention_bf16(const void *q, int Hq, const void *K, const void *V, int B,
                             int Hkv, int T_cap, int T_len, int d, float scale, float *out,
                             void *ws, size_t ws_bytes, void *stream) {
  if (B < 1 || Hkv < 1 || T_cap < 1 || B > 65535 || Hkv > 4096)
    return fail(TQ_ERR_INVALID_ARG, "shape B=%d Hkv=%d T_cap=%d must be positive (B <= 65535, "
                "Hkv <= 4096)", B, Hkv, T_cap);
  if (!pow2_in(d, 16, 256))
    return fail(TQ_ERR_UNSUPPORTED, "d=%d: head_dim must be a power of two in 16..256", d);
  if (Hq < 1 || Hq % Hkv || Hq > 65535)
    return fail(TQ_ERR_INVALID_ARG, "Hq=%d must be a positive multiple of Hkv=%d (<= 65535)", Hq,
                Hkv);
  if (T_len < 1 || T_len > T_cap)
    return fail(TQ_ERR_INVALID_ARG, "T_len=%d must be in 1..T_cap=%d", T_len, T_cap);
  if (!q || !K || !V || !out || !aligned16(q) || !aligned16(K) || !aligned16(V) ||
      !aligned16(out))
    return fail(TQ_ERR_INVALID_ARG, "q/K/V/out must be non-NULL and 16-byte aligned");
  if (!std::isfinite(scale)) return fail(TQ_ERR_INVALID_ARG, "scale is not finite");
  int sms = sm_count();
  if (sms <= 0) return fail(TQ_ERR_CUDA, "cannot query the device's SM count");
  tq::DecodeBf16Args a;
  std::memset(&a, 0, sizeof a);
  a.plan = tq::plan_decode(B, Hq, Hkv, d, T_len, 0, sms, true);
  if (!ws || !aligned16(ws) || ws_bytes < a.plan.ws_bytes)
    return fail(TQ_ERR_WORKSPACE, "workspace needs %zu bytes (16-byte aligned), got %zu",
                a.plan.ws_bytes, ws ? ws_bytes : 0);
  a.q = q;
  a.K = K;
  a.V = V;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.d = d;
  a.T_len = T_len;
  a.T_cap = T_cap;
  a.scale = scale;
  a.out = out;
  a.ws = static_cast<float *>(ws);
  return cuda_status(tq::launch_decode_bf16(a, static_cast<cudaStream_t>(stream)),
                     "bf16 decode launch");
}

} // extern "C"
