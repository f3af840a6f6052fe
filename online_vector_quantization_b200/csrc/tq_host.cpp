// Host side of libtq: the tables the kernels read (rotation, QJL matrix,
// Lloyd-Max codebooks), parameter objects, argument checking and the C ABI
// entry points.  Device work is enqueued by the launchers in the .cu files.

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include "tq_internal.h"

namespace tq {

static thread_local std::string g_last_error;

tq_status fail(tq_status st, const std::string& msg) {
  g_last_error = msg;
  return st;
}

tq_status cuda_fail(cudaError_t e, const char* what) {
  return fail(TQ_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

// ---------------------------------------------------------------------------
// SplitMix64 (Steele, Lea, Flood 2014): output i of a stream with initial
// state s0 is mix(s0 + (i+1) * 0x9E3779B97F4A7C15).  Streams are named by a
// tag: s0 = seed ^ (tag << 32); tag 0 feeds Pi, tag 1 feeds S.
// ---------------------------------------------------------------------------
static inline uint64_t splitmix_mix(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// Fill out[0..count) with N(0,1) samples: Box-Muller on consecutive uniform
// pairs, u = ((z >> 11) + 0.5) 2^-53, emitting r cos(theta) then r sin(theta).
static void gaussian_stream(uint64_t seed, uint64_t tag, size_t count, double* out) {
  const uint64_t s0 = seed ^ (tag << 32);
  uint64_t ctr = 0;
  auto next_uniform = [&]() {
    ++ctr;
    uint64_t z = splitmix_mix(s0 + ctr * 0x9E3779B97F4A7C15ull);
    return (static_cast<double>(z >> 11) + 0.5) * 0x1.0p-53;
  };
  const double two_pi = 6.283185307179586476925286766559;
  for (size_t i = 0; i < count; i += 2) {
    double u1 = next_uniform();
    double u2 = next_uniform();
    double r = std::sqrt(-2.0 * std::log(u1));
    double th = two_pi * u2;
    out[i] = r * std::cos(th);
    if (i + 1 < count) out[i + 1] = r * std::sin(th);
  }
}

// Householder QR of the column-major copy of g (d x d, row-major input);
// returns Q (row-major) with the signs chosen so that diag(R) > 0.
static void haar_from_gaussian(int d, const std::vector<double>& g, std::vector<double>& q_out) {
  // a: column-major working copy, a[c*d + r] = g[r][c]
  std::vector<double> a(static_cast<size_t>(d) * d), vs(static_cast<size_t>(d) * d, 0.0);
  std::vector<double> beta(d, 0.0), rdiag(d, 0.0);
  for (int r = 0; r < d; ++r)
    for (int c = 0; c < d; ++c) a[static_cast<size_t>(c) * d + r] = g[static_cast<size_t>(r) * d + c];
  for (int k = 0; k < d; ++k) {
    double* col = &a[static_cast<size_t>(k) * d];
    double norm = 0.0;
    for (int r = k; r < d; ++r) norm += col[r] * col[r];
    norm = std::sqrt(norm);
    double alpha = col[k] >= 0 ? -norm : norm;  // R_kk = alpha
    double* v = &vs[static_cast<size_t>(k) * d];
    for (int r = k; r < d; ++r) v[r] = col[r];
    v[k] -= alpha;
    double vtv = 0.0;
    for (int r = k; r < d; ++r) vtv += v[r] * v[r];
    beta[k] = vtv > 0 ? 2.0 / vtv : 0.0;
    rdiag[k] = alpha;
    // apply H_k = I - beta v v^T to the remaining columns
    for (int c = k; c < d; ++c) {
      double* cc = &a[static_cast<size_t>(c) * d];
      double dot = 0.0;
      for (int r = k; r < d; ++r) dot += v[r] * cc[r];
      dot *= beta[k];
      for (int r = k; r < d; ++r) cc[r] -= dot * v[r];
    }
  }
  // Q = H_0 H_1 ... H_{d-1} applied to the identity, column by column
  std::vector<double> qc(static_cast<size_t>(d) * d, 0.0);  // column-major
  for (int c = 0; c < d; ++c) qc[static_cast<size_t>(c) * d + c] = 1.0;
  for (int k = d - 1; k >= 0; --k) {
    const double* v = &vs[static_cast<size_t>(k) * d];
    for (int c = 0; c < d; ++c) {
      double* cc = &qc[static_cast<size_t>(c) * d];
      double dot = 0.0;
      for (int r = k; r < d; ++r) dot += v[r] * cc[r];
      dot *= beta[k];
      for (int r = k; r < d; ++r) cc[r] -= dot * v[r];
    }
  }
  q_out.assign(static_cast<size_t>(d) * d, 0.0);
  for (int c = 0; c < d; ++c) {
    double sgn = rdiag[c] < 0 ? -1.0 : 1.0;
    for (int r = 0; r < d; ++r) q_out[static_cast<size_t>(r) * d + c] = sgn * qc[static_cast<size_t>(c) * d + r];
  }
}

// ---------------------------------------------------------------------------
// Lloyd-Max for f(x) = C (1-x^2)^((d-3)/2) on [-1, 1].  Cell masses by
// composite Gauss-Legendre (nodes from Newton's method on P_n); first
// moments in closed form, int x f = -C/(d-1) (1-x^2)^((d-1)/2).
// ---------------------------------------------------------------------------
struct GaussLegendre {
  std::vector<double> x, w;
  explicit GaussLegendre(int n) : x(n), w(n) {
    const double pi = 3.14159265358979323846264338327950288;
    for (int i = 0; i < n; ++i) {
      double z = std::cos(pi * (i + 0.75) / (n + 0.5));
      double dp = 1.0;
      for (int it = 0; it < 100; ++it) {
        double p0 = 1.0, p1 = z;
        for (int k = 2; k <= n; ++k) {
          double p2 = ((2.0 * k - 1.0) * z * p1 - (k - 1.0) * p0) / k;
          p0 = p1;
          p1 = p2;
        }
        dp = n * (z * p1 - p0) / (z * z - 1.0);
        double dz = p1 / dp;
        z -= dz;
        if (std::fabs(dz) < 1e-17) break;
      }
      x[i] = z;
      w[i] = 2.0 / ((1.0 - z * z) * dp * dp);
    }
  }
};

struct SphereCoordinate {
  int d;
  double log_c;
  double reach;  // |x| beyond which f < exp(-750) f(0)
  explicit SphereCoordinate(int d_) : d(d_) {
    log_c = std::lgamma(0.5 * d) - 0.5 * std::log(3.14159265358979323846) - std::lgamma(0.5 * (d - 1));
    reach = std::min(1.0, std::sqrt(-std::expm1(-1500.0 / std::max(d - 3, 1))));
  }
  double density(double x) const {
    if (std::fabs(x) >= 1.0) return 0.0;
    return std::exp(log_c + 0.5 * (d - 3) * std::log1p(-x * x));
  }
  double moment_prim(double x) const {  // F1(x) with F1' = -x f(x)... sign handled by caller
    if (std::fabs(x) >= 1.0) return 0.0;
    return std::exp(log_c + 0.5 * (d - 1) * std::log1p(-x * x)) / (d - 1);
  }
  double mass(double a, double b, const GaussLegendre& gl) const {
    a = std::max(a, -reach);
    b = std::min(b, reach);
    if (b <= a) return 0.0;
    const int pieces = 24;
    double h = (b - a) / pieces, sum = 0.0;
    for (int p = 0; p < pieces; ++p) {
      double lo = a + p * h, mid = lo + 0.5 * h;
      double part = 0.0;
      for (size_t i = 0; i < gl.x.size(); ++i) part += gl.w[i] * density(mid + 0.5 * h * gl.x[i]);
      sum += 0.5 * h * part;
    }
    return sum;
  }
  double first_moment(double a, double b) const { return moment_prim(a) - moment_prim(b); }
};

// Standard normal quantile by bisection on erfc (start values only).
static double normal_quantile(double p) {
  double lo = -40.0, hi = 40.0;
  for (int i = 0; i < 200; ++i) {
    const double mid = 0.5 * (lo + hi);
    if (0.5 * std::erfc(-mid / std::sqrt(2.0)) < p)
      lo = mid;
    else
      hi = mid;
  }
  return 0.5 * (lo + hi);
}

// The Lloyd map: T_k = (first moment) / (mass) of f over the cell of c_k.
static void lloyd_map(const SphereCoordinate& f, const GaussLegendre& gl, const std::vector<double>& c,
                      std::vector<double>& T, std::vector<double>& m0) {
  const int levels = static_cast<int>(c.size());
  for (int k = 0; k < levels; ++k) {
    const double lo = k == 0 ? -1.0 : 0.5 * (c[k - 1] + c[k]);
    const double hi = k == levels - 1 ? 1.0 : 0.5 * (c[k] + c[k + 1]);
    m0[k] = f.mass(lo, hi, gl);
    T[k] = f.first_moment(lo, hi) / m0[k];
  }
}

// More than 16 levels: the plain iteration's contraction approaches 1, so the
// fixed point c = T(c) is found by Newton's method.  With t_k the midpoints
// and f_k = f(t_k), dT_k/dc_{k+1} = f_k (t_k - T_k) / (2 M0_k) and
// dT_k/dc_{k-1} = f_{k-1} (T_k - t_{k-1}) / (2 M0_k), dT_k/dc_k their sum:
// the Jacobian of c - T(c) is tridiagonal (Thomas algorithm).  Start: the
// high-resolution optimum of a Gaussian of variance 1/d (point density ~
// f^(1/3): Gaussian quantiles of variance 3/d), then 50 plain steps; Newton
// steps are halved while they do not reduce max |c - T(c)| or break the order.
static tq_status lloyd_max_newton(int d, int bits, double* centroids, double* bounds) {
  const int L = 1 << bits;
  SphereCoordinate f(d);
  GaussLegendre gl(48);
  std::vector<double> c(L), T(L), m0(L), cn(L), Tn(L), m0n(L), step(L);
  const double s3 = std::sqrt(3.0 / d);
  for (int k = 0; k < L; ++k) c[k] = s3 * normal_quantile((k + 0.5) / L);
  for (int it = 0; it < 50; ++it) {
    lloyd_map(f, gl, c, T, m0);
    c = T;
  }
  lloyd_map(f, gl, c, T, m0);
  auto max_abs_g = [&](const std::vector<double>& cc, const std::vector<double>& tt) {
    double g = 0.0;
    for (int k = 0; k < L; ++k) g = std::max(g, std::fabs(cc[k] - tt[k]));
    return g;
  };
  std::vector<double> diag(L), sup(L), sub(L), rhs(L);
  for (int it = 0; it < 100; ++it) {
    // J = I - dT, rows k: sub[k] (column k-1), diag[k], sup[k] (column k+1)
    for (int k = 0; k < L; ++k) {
      double up = 0.0, dn = 0.0;
      if (k + 1 < L) {
        const double t = 0.5 * (c[k] + c[k + 1]);
        up = f.density(t) * (t - T[k]) / (2.0 * m0[k]);
      }
      if (k > 0) {
        const double t = 0.5 * (c[k - 1] + c[k]);
        dn = f.density(t) * (T[k] - t) / (2.0 * m0[k]);
      }
      diag[k] = 1.0 - up - dn;
      sup[k] = -up;
      sub[k] = -dn;
      rhs[k] = -(c[k] - T[k]);
    }
    // Thomas algorithm
    for (int k = 1; k < L; ++k) {
      const double w = sub[k] / diag[k - 1];
      diag[k] -= w * sup[k - 1];
      rhs[k] -= w * rhs[k - 1];
    }
    step[L - 1] = rhs[L - 1] / diag[L - 1];
    for (int k = L - 2; k >= 0; --k) step[k] = (rhs[k] - sup[k] * step[k + 1]) / diag[k];
    const double g0 = max_abs_g(c, T);
    double lam = 1.0;
    for (;;) {
      bool ok = true;
      for (int k = 0; k < L; ++k) {
        cn[k] = c[k] + lam * step[k];
        if (k > 0 && !(cn[k] > cn[k - 1])) ok = false;
      }
      if (!(cn[0] > -1.0) || !(cn[L - 1] < 1.0)) ok = false;
      if (ok) {
        lloyd_map(f, gl, cn, Tn, m0n);
        if (max_abs_g(cn, Tn) < g0 || lam < 1e-6) break;
      }
      lam *= 0.5;
      if (lam < 1e-9) return fail(TQ_ERR_ARG, "tq_codebook: Newton iteration did not converge");
    }
    double moved = 0.0, cmax = 0.0;
    for (int k = 0; k < L; ++k) {
      moved = std::max(moved, std::fabs(cn[k] - c[k]));
      cmax = std::max(cmax, std::fabs(cn[k]));
    }
    c.swap(cn);
    T.swap(Tn);
    m0.swap(m0n);
    if (moved <= 1e-15 * cmax) break;
  }
  for (int k = 0; k < L; ++k) centroids[k] = c[k];
  for (int k = 0; k + 1 < L; ++k) bounds[k] = 0.5 * (c[k] + c[k + 1]);
  return TQ_OK;
}

static tq_status lloyd_max(int d, int bits, double* centroids, double* bounds) {
  if (bits > 4) return lloyd_max_newton(d, bits, centroids, bounds);
  const int levels = 1 << bits;
  SphereCoordinate f(d);
  GaussLegendre gl(48);
  std::vector<double> c(levels), nc(levels);
  // start: equally spaced over +-2.5 standard deviations (1/sqrt(d))
  const double sd = 1.0 / std::sqrt(static_cast<double>(d));
  for (int k = 0; k < levels; ++k) c[k] = sd * (-2.5 + 5.0 * (k + 0.5) / levels);
  for (int it = 0; it < 200000; ++it) {
    double moved = 0.0, cmax = 0.0;
    for (int k = 0; k < levels; ++k) {
      double lo = k == 0 ? -1.0 : 0.5 * (c[k - 1] + c[k]);
      double hi = k == levels - 1 ? 1.0 : 0.5 * (c[k] + c[k + 1]);
      nc[k] = f.first_moment(lo, hi) / f.mass(lo, hi, gl);
    }
    for (int k = 0; k < levels; ++k) {
      moved = std::max(moved, std::fabs(nc[k] - c[k]));
      cmax = std::max(cmax, std::fabs(nc[k]));
    }
    c.swap(nc);
    if (moved <= 1e-15 * cmax) break;
  }
  for (int k = 0; k < levels; ++k) centroids[k] = c[k];
  for (int k = 0; k + 1 < levels; ++k) bounds[k] = 0.5 * (c[k] + c[k + 1]);
  return TQ_OK;
}

// Round a positive double to the nearest fp16 value (normal range).
static double round_to_f16(double v) {
  int e = 0;
  std::frexp(v, &e);                       // v = m 2^e, m in [0.5, 1)
  const double ulp = std::ldexp(1.0, e - 11);  // 11 significant bits
  return std::nearbyint(v / ulp) * ulp;
}

// Scale sigma for one codebook: the MMAs see sigma * c_k in fp16 and the
// result is divided by sigma in fp32, so pick sigma (a power of two times a
// factor in [1, 2), searched on a grid) that makes every centroid nearly
// exact in fp16.  One-bit codebooks get sigma = 1/c_1 (values exactly +-1).
static double codebook_sigma(const double* c, int levels) {
  double cmax = 0.0;
  for (int k = 0; k < levels; ++k) cmax = std::max(cmax, std::fabs(c[k]));
  if (levels == 2) return 1.0 / cmax;
  int e = 0;
  std::frexp(cmax, &e);
  const double base = std::ldexp(1.0, 1 - e);  // cmax * base in [1, 2)
  double best_err = 1e300, best = base;
  for (int i = 0; i < (1 << 16); ++i) {
    const double sg = base * (1.0 + i / 65536.0);
    double err = 0.0;
    for (int k = 0; k < levels; ++k) {
      const double v = std::fabs(c[k]) * sg;
      err = std::max(err, std::fabs(round_to_f16(v) - v) / v);
    }
    if (err < best_err) { best_err = err; best = sg; }
  }
  return best;
}

static bool make_format(int bits, int mode, int mixed, FormatSpec* f, std::string* why) {
  if (mode != TQ_MODE_MSE && mode != TQ_MODE_PROD) { *why = "mode must be MSE or PROD"; return false; }
  const bool wide = bits == kWideBits && mode == TQ_MODE_MSE && mixed == 0;
  if ((bits < 1 || bits > 4) && !wide) { *why = "bits must be in 1..4, or 8 in MSE mode (unmixed rows)"; return false; }
  if (mixed != 0 && mixed != 1) { *why = "mixed must be 0 or 1"; return false; }
  f->total_bits = bits;
  f->prod = mode == TQ_MODE_PROD;
  f->mixed = mixed;
  f->mse_bits = f->prod ? bits - 1 : bits;
  if (mixed && f->prod) { *why = "mixed rows are supported in MSE mode only"; return false; }
  if (mixed && bits != 2 && bits != 3) {
    *why = "mixed rows are supported for bits = 2 and 3 (2.5 and 3.5 bits per channel) only";
    return false;
  }
  f->code_bytes = mixed ? 8 * (2 * f->mse_bits + 1) : 16 * f->mse_bits;
  f->qjl_bytes = f->prod ? kSketch / 8 : 0;
  return true;
}

// ---- argument checks shared by the entry points --------------------------

static bool aligned16_ptr(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15) == 0; }

tq_status check_cache(const tq_params* p, const tq_cache* c, const char* who) {
  if (!c) return fail(TQ_ERR_ARG, std::string(who) + ": NULL cache");
  if (c->n_seq < 1 || c->n_kv_heads < 1 || c->capacity < 0 || c->capacity % 64 || c->n_sink < 0)
    return fail(TQ_ERR_ARG, std::string(who) + ": bad cache sizes");
  if (!c->lens || !c->status || !c->k_norms || !c->v_norms || (p->fk.code_bytes && !c->k_codes) ||
      (p->fv.code_bytes && !c->v_codes) || (p->fk.prod && (!c->k_qjl || !c->k_res_norms)) ||
      (p->fv.prod && (!c->v_qjl || !c->v_res_norms)) || (c->n_sink && (!c->k_sink || !c->v_sink)))
    return fail(TQ_ERR_ARG, std::string(who) + ": a cache plane is NULL");
  const void* planes[] = {c->k_codes, c->k_norms, c->k_qjl, c->k_res_norms, c->v_codes,
                          c->v_norms, c->v_qjl, c->v_res_norms, c->k_sink, c->v_sink};
  for (const void* pl : planes)
    if (pl && !aligned16_ptr(pl)) return fail(TQ_ERR_ALIGN, std::string(who) + ": cache planes must be 16-byte aligned");
  return TQ_OK;
}

tq_status check_decode_call(const tq_params* p, const void* q, int q_dtype, const tq_cache* cache, int B, int hq,
                            int max_len, const void* out, int out_dtype, const tq_attn_flags* flags,
                            const char* who, DecodePlan* plan, float* thr, unsigned long long** sv_stats) {
  const std::string w(who);
  if (!p) return fail(TQ_ERR_ARG, w + ": NULL params");
  tq_status st = check_cache(p, cache, who);
  if (st != TQ_OK) return st;
  if (B < 1 || B > cache->n_seq || hq < 1 || max_len < 0 || (q_dtype != TQ_F32 && q_dtype != TQ_BF16) ||
      (out_dtype != TQ_F32 && out_dtype != TQ_BF16))
    return fail(TQ_ERR_ARG, w + ": bad B, hq, max_len or dtype");
  const int hkv = cache->n_kv_heads;
  if (hq % hkv) return fail(TQ_ERR_ARG, w + ": hq must be a multiple of n_kv_heads");
  if (hq / hkv > 8) return fail(TQ_ERR_UNSUPPORTED, w + ": at most 8 query heads per kv-head");
  if (max_len > cache->capacity + cache->n_sink) return fail(TQ_ERR_ARG, w + ": max_len above the cache's capacity");
  if (!q || !out) return fail(TQ_ERR_ARG, w + ": NULL q or out");
  if (!aligned16_ptr(q) || !aligned16_ptr(out)) return fail(TQ_ERR_ALIGN, w + ": q and out must be 16-byte aligned");
  const float t = flags ? flags->sparse_v_threshold : 0.f;
  if (!(t >= 0.f) || t >= 1.f) return fail(TQ_ERR_ARG, w + ": sparse_v_threshold must be in [0, 1)");
  if (flags && flags->reserved != 0) return fail(TQ_ERR_ARG, w + ": flags->reserved must be 0");
  unsigned long long* stats = flags ? flags->sparse_v_stats : nullptr;
  if (stats && (reinterpret_cast<uintptr_t>(stats) & 7))
    return fail(TQ_ERR_ALIGN, w + ": sparse_v_stats must be 8-byte aligned");
  *thr = t;
  *sv_stats = stats;
  *plan = plan_decode(p, B, hq, hkv, max_len);
  return TQ_OK;
}

}  // namespace tq

using namespace tq;

extern "C" {

const char* tq_last_error(void) { return g_last_error.c_str(); }

tq_status tq_codebook(int d, int bits, double* centroids, double* bounds) {
  if (!centroids || !bounds) return fail(TQ_ERR_ARG, "tq_codebook: NULL output");
  if (d < 3 || bits < 1 || bits > 8) return fail(TQ_ERR_ARG, "tq_codebook: need d >= 3 and bits in 1..8");
  return lloyd_max(d, bits, centroids, bounds);
}

tq_status tq_rotation(uint64_t seed, int d, double* pi) {
  if (!pi || d < 1) return fail(TQ_ERR_ARG, "tq_rotation: bad arguments");
  std::vector<double> g(static_cast<size_t>(d) * d), q;
  gaussian_stream(seed, 0, g.size(), g.data());
  haar_from_gaussian(d, g, q);
  std::memcpy(pi, q.data(), q.size() * sizeof(double));
  return TQ_OK;
}

tq_status tq_hadamard_rotation(uint64_t seed, int d, double* pi) {
  if (!pi || d < 1 || (d & (d - 1))) return fail(TQ_ERR_ARG, "tq_hadamard_rotation: d must be a power of two");
  // Sylvester doubling: H_2n = [[H_n, H_n], [H_n, -H_n]]
  std::vector<double> h(static_cast<size_t>(d) * d, 0.0);
  h[0] = 1.0;
  for (int n = 1; n < d; n *= 2)
    for (int i = 0; i < n; ++i)
      for (int j = 0; j < n; ++j) {
        const double v = h[static_cast<size_t>(i) * d + j];
        h[static_cast<size_t>(i) * d + j + n] = v;
        h[static_cast<size_t>(i + n) * d + j] = v;
        h[static_cast<size_t>(i + n) * d + j + n] = -v;
      }
  const uint64_t s0 = seed ^ (uint64_t(2) << 32);
  const double inv = 1.0 / std::sqrt(static_cast<double>(d));
  for (int j = 0; j < d; ++j) {
    const uint64_t z = splitmix_mix(s0 + uint64_t(j + 1) * 0x9E3779B97F4A7C15ull);
    const double s = (z >> 63) ? -inv : inv;
    for (int i = 0; i < d; ++i) pi[static_cast<size_t>(i) * d + j] = h[static_cast<size_t>(i) * d + j] * s;
  }
  return TQ_OK;
}

tq_status tq_qjl_matrix(uint64_t seed, int m, int d, double* s) {
  if (!s || m < 1 || d < 1) return fail(TQ_ERR_ARG, "tq_qjl_matrix: bad arguments");
  gaussian_stream(seed, 1, static_cast<size_t>(m) * d, s);
  return TQ_OK;
}

// The tensor-core quantize kernels take Pi (rotation) and M = S Pi^T (QJL
// sketch of the rotated residual) as B operands: row n = output index, K =
// input index, 16-bit values in the layout a TMA copy with 128-byte swizzle
// produces (two 64-column boxes of 128 rows x 128 B; the 16-byte chunk c of
// row r sits at chunk c ^ (r & 7)).  Pi is split into bf16 terms (two for
// the MSE kernels, three for the prod kernels) and M into two fp16 terms, each
// term rounding what the previous ones left of the fp64 value.
static size_t sw128_offset(int row, int k) {
  return static_cast<size_t>((k >> 6) * 16384 + row * 128 + ((((k & 63) >> 3) ^ (row & 7)) << 4) + (k & 7) * 2);
}

static std::vector<uint8_t> tensor_core_images(const std::vector<double>& pi, const std::vector<double>& m_rowmajor) {
  std::vector<uint8_t> img(static_cast<size_t>(kTcImgCount) * kTcImgBytes, 0);
  auto put = [&](int which, int row, int k, uint16_t bits) {
    std::memcpy(img.data() + static_cast<size_t>(which) * kTcImgBytes + sw128_offset(row, k), &bits, 2);
  };
  auto bf = [](double v, double* back) {
    const __nv_bfloat16 h = __float2bfloat16_rn(static_cast<float>(v));
    *back = static_cast<double>(__bfloat162float(h));
    uint16_t b;
    std::memcpy(&b, &h, 2);
    return b;
  };
  auto hf = [](double v, double* back) {
    const __half h = __float2half_rn(static_cast<float>(v));
    *back = static_cast<double>(__half2float(h));
    uint16_t b;
    std::memcpy(&b, &h, 2);
    return b;
  };
  for (int row = 0; row < kDim; ++row)
    for (int k = 0; k < kDim; ++k) {
      const double p = pi[static_cast<size_t>(row) * kDim + k];
      double h0, h1, h2;
      put(kTcImgPiHi, row, k, bf(p, &h0));
      put(kTcImgPiLo, row, k, bf(p - h0, &h1));
      put(kTcImgPiA, row, k, bf(p, &h0));
      put(kTcImgPiB, row, k, bf(p - h0, &h1));
      put(kTcImgPiC, row, k, bf(p - h0 - h1, &h2));
      const double mv = m_rowmajor[static_cast<size_t>(row) * kDim + k];
      put(kTcImgMHi, row, k, hf(mv, &h0));
      put(kTcImgMLo, row, k, hf(mv - h0, &h1));
    }
  return img;
}

tq_status tq_params_create(const tq_config* cfg, tq_params** out) {
  if (!cfg || !out) return fail(TQ_ERR_ARG, "tq_params_create: NULL argument");
  *out = nullptr;
  if (cfg->d != kDim) return fail(TQ_ERR_UNSUPPORTED, "tq_params_create: d must be 128");
  if (cfg->rotation != TQ_ROT_HAAR && cfg->rotation != TQ_ROT_HADAMARD)
    return fail(TQ_ERR_ARG, "tq_params_create: unknown rotation kind");
  if (cfg->m != kSketch) return fail(TQ_ERR_UNSUPPORTED, "tq_params_create: m must be 128");
  std::string why;
  FormatSpec fk, fv;
  if (!make_format(cfg->bits_k, cfg->mode_k, cfg->mixed_k, &fk, &why) ||
      !make_format(cfg->bits_v, cfg->mode_v, cfg->mixed_v, &fv, &why))
    return fail(TQ_ERR_UNSUPPORTED, "tq_params_create: " + why);

  tq_params* p = new tq_params();
  p->cfg = *cfg;
  p->fk = fk;
  p->fv = fv;
  const int d = kDim, m = kSketch;
  p->pi.resize(static_cast<size_t>(d) * d);
  p->s.resize(static_cast<size_t>(m) * d);
  if (cfg->rotation == TQ_ROT_HADAMARD)
    tq_hadamard_rotation(cfg->seed, d, p->pi.data());
  else
    tq_rotation(cfg->seed, d, p->pi.data());
  tq_qjl_matrix(cfg->seed, m, d, p->s.data());

  // host staging of every device table
  std::vector<float> pi32(d * d), pit32(d * d), s32(m * d), st32(d * m), mt32(d * m);
  std::vector<float> cb32((kMaxBits + 1) * kBookSlots, 0.f), bd32((kMaxBits + 1) * kBookSlots, 0.f);
  std::vector<float> cbs32((kMaxBits + 1) * kBookSlots, 0.f), sig32(kSigSlots, 1.f);
  std::vector<float> cb8_32(256, 0.f), cbs8_32(256, 0.f), bd8_32(256, INFINITY);
  std::vector<double> cb8_64(256, 0.0), pit64(static_cast<size_t>(d) * d);
  std::vector<float> cell8;  // pairs {count, bound}
  for (int r = 0; r < d; ++r)
    for (int c = 0; c < d; ++c) pit64[static_cast<size_t>(c) * d + r] = p->pi[static_cast<size_t>(r) * d + c];
  if (fk.wide() || fv.wide()) {
    double c[256], t[255];
    lloyd_max(d, kWideBits, c, t);
    const double sg = codebook_sigma(c, 256);
    sig32[kWideBits] = static_cast<float>(sg);
    for (int k = 0; k < 256; ++k) {
      cb8_32[k] = static_cast<float>(c[k]);
      cbs8_32[k] = static_cast<float>(c[k] * static_cast<double>(sig32[kWideBits]));
      cb8_64[k] = c[k];
    }
    for (int k = 0; k < 255; ++k) bd8_32[k] = static_cast<float>(t[k]);
    // cells over |u| no wider than the closest two positive bounds, so each
    // holds at most one bound: the code of |u| is the count at the cell's
    // start plus 1 if |u| passes the cell's bound
    double min_gap = INFINITY;
    for (int k = 128; k + 1 < 255; ++k) min_gap = std::min(min_gap, t[k + 1] - t[k]);
    const float w = static_cast<float>(0.99 * min_gap);
    const int n_cells = static_cast<int>(std::ceil(t[254] / w)) + 2;
    if (n_cells > kCell8Max) { delete p; return fail(TQ_ERR_UNSUPPORTED, "tq_params_create: 8-bit code cells"); }
    cell8.resize(2 * static_cast<size_t>(n_cells));
    for (int cidx = 0; cidx < n_cells; ++cidx) {
      const float lo = cidx * w, hi = (cidx + 1) * w;
      int cnt = 0;
      float inside = INFINITY;
      for (int k = 128; k < 255; ++k) {  // the positive bounds t[128..254]
        const float b = static_cast<float>(t[k]);
        if (b <= lo) ++cnt;
        else if (b < hi) inside = std::min(inside, b);
      }
      cell8[2 * cidx] = static_cast<float>(cnt);
      cell8[2 * cidx + 1] = inside;
    }
    p->cell8_n = n_cells;
    p->cell8_inv_w = 1.f / w;
  }
  std::vector<double> cb64((kMaxBits + 1) * kBookSlots, 0.0);
  for (int r = 0; r < d; ++r)
    for (int c = 0; c < d; ++c) {
      pi32[r * d + c] = static_cast<float>(p->pi[r * d + c]);
      pit32[c * d + r] = static_cast<float>(p->pi[r * d + c]);
    }
  for (int i = 0; i < m; ++i)
    for (int j = 0; j < d; ++j) {
      s32[i * d + j] = static_cast<float>(p->s[i * d + j]);
      st32[j * m + i] = static_cast<float>(p->s[i * d + j]);
    }
  // M = S Pi^T (fp64): (S r) = M (Pi r) for a residual r given in the rotated domain
  std::vector<double> mt64(static_cast<size_t>(m) * d);  // M row-major [i][j]
  for (int i = 0; i < m; ++i)
    for (int j = 0; j < d; ++j) {
      double acc = 0.0;
      for (int k = 0; k < d; ++k) acc += p->s[i * d + k] * p->pi[j * d + k];
      mt32[j * m + i] = static_cast<float>(acc);
      mt64[i * d + j] = acc;
    }
  for (int b = 1; b <= kMaxBits; ++b) {
    bool used = false;
    for (int j = 0; j < d; ++j) used |= fk.width(j) == b || fv.width(j) == b;
    if (!used) continue;
    double c[16], t[15];
    lloyd_max(d, b, c, t);
    const double sg = codebook_sigma(c, 1 << b);
    sig32[b] = static_cast<float>(sg);
    for (int k = 0; k < (1 << b); ++k) {
      cb32[b * kBookSlots + k] = static_cast<float>(c[k]);
      cbs32[b * kBookSlots + k] = static_cast<float>(c[k] * static_cast<double>(sig32[b]));
      cb64[b * kBookSlots + k] = c[k];
    }
    for (int k = 0; k + 1 < (1 << b); ++k) bd32[b * kBookSlots + k] = static_cast<float>(t[k]);
    for (int k = (1 << b) - 1; k < kBookSlots; ++k) bd32[b * kBookSlots + k] = INFINITY;
  }

  // one device block, each table 256-byte aligned
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off += (bytes + 255) & ~size_t(255); return o; };
  size_t o_pi = take(pi32.size() * 4), o_pit = take(pit32.size() * 4), o_s = take(s32.size() * 4),
         o_st = take(st32.size() * 4), o_mt = take(mt32.size() * 4), o_pi64 = take(p->pi.size() * 8),
         o_s64 = take(p->s.size() * 8), o_cb = take(cb32.size() * 4), o_bd = take(bd32.size() * 4),
         o_cb64 = take(cb64.size() * 8), o_cbs = take(cbs32.size() * 4), o_sig = take(sig32.size() * 4),
         o_status = take(sizeof(int32_t)), o_img = take(static_cast<size_t>(kTcImgCount) * kTcImgBytes),
         o_cb8 = take(256 * 4), o_cbs8 = take(256 * 4), o_bd8 = take(256 * 4), o_cb864 = take(256 * 8),
         o_cell8 = take(cell8.size() * 4), o_pit64 = take(pit64.size() * 8);
  p->lut_bytes = decode_lut_bytes(p->fk, p->fv);
  const size_t o_lut = take(p->lut_bytes);
  cudaError_t e = cudaGetDevice(&p->device);
  if (e == cudaSuccess) e = cudaMalloc(&p->block, off);
  if (e != cudaSuccess) {
    delete p;
    return e == cudaErrorMemoryAllocation ? fail(TQ_ERR_NOMEM, "tq_params_create: cudaMalloc failed")
                                          : cuda_fail(e, "tq_params_create");
  }
  char* base = static_cast<char*>(p->block);
  p->pi32 = reinterpret_cast<float*>(base + o_pi);
  p->pit32 = reinterpret_cast<float*>(base + o_pit);
  p->s32 = reinterpret_cast<float*>(base + o_s);
  p->st32 = reinterpret_cast<float*>(base + o_st);
  p->mt32 = reinterpret_cast<float*>(base + o_mt);
  p->pi64 = reinterpret_cast<double*>(base + o_pi64);
  p->s64 = reinterpret_cast<double*>(base + o_s64);
  p->cb32 = reinterpret_cast<float*>(base + o_cb);
  p->bd32 = reinterpret_cast<float*>(base + o_bd);
  p->cb64 = reinterpret_cast<double*>(base + o_cb64);
  p->cbs32 = reinterpret_cast<float*>(base + o_cbs);
  p->sig32 = reinterpret_cast<float*>(base + o_sig);
  p->status32 = reinterpret_cast<int32_t*>(base + o_status);
  p->tc_img = reinterpret_cast<uint8_t*>(base + o_img);
  p->lut_img = p->lut_bytes ? reinterpret_cast<uint8_t*>(base + o_lut) : nullptr;
  p->cb8_32 = reinterpret_cast<float*>(base + o_cb8);
  p->cbs8_32 = reinterpret_cast<float*>(base + o_cbs8);
  p->bd8_32 = reinterpret_cast<float*>(base + o_bd8);
  p->cb8_64 = reinterpret_cast<double*>(base + o_cb864);
  p->cell8 = cell8.empty() ? nullptr : reinterpret_cast<float2*>(base + o_cell8);
  p->pit64 = reinterpret_cast<double*>(base + o_pit64);
  const std::vector<uint8_t> img = tensor_core_images(p->pi, mt64);
  e = cudaMemset(p->status32, 0, sizeof(int32_t));
  if (e != cudaSuccess) {
    cudaFree(p->block);
    delete p;
    return cuda_fail(e, "tq_params_create: status word");
  }
  struct { void* dst; const void* src; size_t n; } copies[] = {
      {p->pi32, pi32.data(), pi32.size() * 4},   {p->pit32, pit32.data(), pit32.size() * 4},
      {p->s32, s32.data(), s32.size() * 4},      {p->st32, st32.data(), st32.size() * 4},
      {p->mt32, mt32.data(), mt32.size() * 4},   {p->pi64, p->pi.data(), p->pi.size() * 8},
      {p->s64, p->s.data(), p->s.size() * 8},    {p->cb32, cb32.data(), cb32.size() * 4},
      {p->bd32, bd32.data(), bd32.size() * 4},   {p->cb64, cb64.data(), cb64.size() * 8},
      {p->cbs32, cbs32.data(), cbs32.size() * 4}, {p->sig32, sig32.data(), sig32.size() * 4},
      {p->tc_img, img.data(), img.size()},       {p->cb8_32, cb8_32.data(), 256 * 4},
      {p->cbs8_32, cbs8_32.data(), 256 * 4},     {p->bd8_32, bd8_32.data(), 256 * 4},
      {p->cb8_64, cb8_64.data(), 256 * 8},       {p->cell8, cell8.data(), cell8.size() * 4},
      {p->pit64, pit64.data(), pit64.size() * 8}};
  for (auto& c : copies) {
    if (c.n == 0) continue;
    e = cudaMemcpy(c.dst, c.src, c.n, cudaMemcpyHostToDevice);
    if (e != cudaSuccess) {
      cudaFree(p->block);
      delete p;
      return cuda_fail(e, "tq_params_create: upload");
    }
  }
  if (p->lut_bytes) {
    const tq_status st = build_decode_luts(p);
    if (st != TQ_OK) {
      cudaFree(p->block);
      delete p;
      return st;
    }
  }
  *out = p;
  return TQ_OK;
}

void tq_params_destroy(tq_params* p) {
  if (!p) return;
  if (p->block) cudaFree(p->block);
  delete p;
}

tq_status tq_params_status(const tq_params* p, int32_t* out, int clear) {
  if (!p || !out) return fail(TQ_ERR_ARG, "tq_params_status: bad arguments");
  cudaError_t e = cudaMemcpy(out, p->status32, sizeof(int32_t), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && clear) e = cudaMemset(p->status32, 0, sizeof(int32_t));
  return e == cudaSuccess ? TQ_OK : cuda_fail(e, "tq_params_status");
}

tq_status tq_row_bytes(const tq_params* p, int which, int* code_bytes, int* qjl_bytes) {
  if (!p || !code_bytes || !qjl_bytes || (which != TQ_K && which != TQ_V))
    return fail(TQ_ERR_ARG, "tq_row_bytes: bad arguments");
  const FormatSpec& f = which == TQ_K ? p->fk : p->fv;
  *code_bytes = f.code_bytes;
  *qjl_bytes = f.qjl_bytes;
  return TQ_OK;
}

static bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15) == 0; }

static tq_status check_packed(const FormatSpec& f, const tq_packed* pk, const char* who) {
  if (!pk) return fail(TQ_ERR_ARG, std::string(who) + ": NULL packed planes");
  if ((f.code_bytes && !pk->codes) || !pk->norms || (f.prod && (!pk->qjl || !pk->res_norms)))
    return fail(TQ_ERR_ARG, std::string(who) + ": a required plane is NULL");
  if ((f.code_bytes && !aligned16(pk->codes)) || !aligned16(pk->norms) ||
      (f.prod && (!aligned16(pk->qjl) || !aligned16(pk->res_norms))))
    return fail(TQ_ERR_ALIGN, std::string(who) + ": planes must be 16-byte aligned");
  return TQ_OK;
}

tq_status tq_quantize(const tq_params* p, const void* x, int x_dtype, int64_t n, int which,
                      const tq_packed* out, void* stream) {
  if (!p) return fail(TQ_ERR_ARG, "tq_quantize: NULL params");
  if (n < 0 || (which != TQ_K && which != TQ_V) || (x_dtype != TQ_F32 && x_dtype != TQ_BF16))
    return fail(TQ_ERR_ARG, "tq_quantize: bad n, which or dtype");
  if (n == 0) return TQ_OK;
  if (!x) return fail(TQ_ERR_ARG, "tq_quantize: NULL input");
  if (!aligned16(x)) return fail(TQ_ERR_ALIGN, "tq_quantize: input must be 16-byte aligned");
  const FormatSpec& f = which == TQ_K ? p->fk : p->fv;
  tq_status st = check_packed(f, out, "tq_quantize");
  if (st != TQ_OK) return st;
  return launch_quantize(p, f, x, x_dtype == TQ_BF16, n, out, static_cast<cudaStream_t>(stream));
}

tq_status tq_dequantize(const tq_params* p, const tq_packed* in, int64_t n, int which, float* out,
                        void* stream) {
  if (!p) return fail(TQ_ERR_ARG, "tq_dequantize: NULL params");
  if (n < 0 || (which != TQ_K && which != TQ_V)) return fail(TQ_ERR_ARG, "tq_dequantize: bad n or which");
  if (n == 0) return TQ_OK;
  if (!out) return fail(TQ_ERR_ARG, "tq_dequantize: NULL output");
  const FormatSpec& f = which == TQ_K ? p->fk : p->fv;
  tq_status st = check_packed(f, in, "tq_dequantize");
  if (st != TQ_OK) return st;
  return launch_dequantize(p, f, in, n, out, static_cast<cudaStream_t>(stream));
}

// ---- cache ----------------------------------------------------------------

struct CachePlanes {
  size_t k_codes, k_norms, k_qjl, k_res, v_codes, v_norms, v_qjl, v_res, k_sink, v_sink, total;
};

static bool cache_planes(const tq_params* p, int n_seq, int hkv, int cap, int n_sink, CachePlanes* cp) {
  if (!p || n_seq < 1 || hkv < 1 || cap < 0 || (cap % 64) != 0 || n_sink < 0) return false;
  size_t rows = static_cast<size_t>(n_seq) * hkv * cap;
  size_t sink = static_cast<size_t>(n_seq) * hkv * n_sink * kDim * 2;
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off += (bytes + 255) & ~size_t(255); return o; };
  cp->k_codes = take(rows * p->fk.code_bytes);
  cp->k_norms = take(rows * 4);
  cp->k_qjl = take(rows * p->fk.qjl_bytes);
  cp->k_res = take(p->fk.prod ? rows * 4 : 0);
  cp->v_codes = take(rows * p->fv.code_bytes);
  cp->v_norms = take(rows * 4);
  cp->v_qjl = take(rows * p->fv.qjl_bytes);
  cp->v_res = take(p->fv.prod ? rows * 4 : 0);
  cp->k_sink = take(sink);
  cp->v_sink = take(sink);
  cp->total = off;
  return true;
}

size_t tq_cache_bytes(const tq_params* p, int n_seq, int n_kv_heads, int capacity, int n_sink) {
  CachePlanes cp;
  if (!cache_planes(p, n_seq, n_kv_heads, capacity, n_sink, &cp)) return 0;
  return cp.total;
}

tq_status tq_cache_bind(const tq_params* p, void* base, size_t bytes, int n_seq, int n_kv_heads,
                        int capacity, int n_sink, int32_t* lens, int32_t* status, tq_cache* out) {
  CachePlanes cp;
  if (!out || !base || !lens || !status) return fail(TQ_ERR_ARG, "tq_cache_bind: NULL argument");
  if (!cache_planes(p, n_seq, n_kv_heads, capacity, n_sink, &cp))
    return fail(TQ_ERR_ARG, "tq_cache_bind: bad sizes (capacity must be a multiple of 64)");
  if (bytes < cp.total) return fail(TQ_ERR_CAPACITY, "tq_cache_bind: buffer smaller than tq_cache_bytes");
  if ((reinterpret_cast<uintptr_t>(base) & 255) != 0) return fail(TQ_ERR_ALIGN, "tq_cache_bind: base must be 256-byte aligned");
  char* b = static_cast<char*>(base);
  std::memset(out, 0, sizeof(*out));
  out->n_seq = n_seq;
  out->n_kv_heads = n_kv_heads;
  out->capacity = capacity;
  out->n_sink = n_sink;
  out->k_codes = reinterpret_cast<uint8_t*>(b + cp.k_codes);
  out->k_norms = reinterpret_cast<float*>(b + cp.k_norms);
  out->k_qjl = p->fk.prod ? reinterpret_cast<uint8_t*>(b + cp.k_qjl) : nullptr;
  out->k_res_norms = p->fk.prod ? reinterpret_cast<float*>(b + cp.k_res) : nullptr;
  out->v_codes = reinterpret_cast<uint8_t*>(b + cp.v_codes);
  out->v_norms = reinterpret_cast<float*>(b + cp.v_norms);
  out->v_qjl = p->fv.prod ? reinterpret_cast<uint8_t*>(b + cp.v_qjl) : nullptr;
  out->v_res_norms = p->fv.prod ? reinterpret_cast<float*>(b + cp.v_res) : nullptr;
  out->k_sink = n_sink ? reinterpret_cast<uint16_t*>(b + cp.k_sink) : nullptr;
  out->v_sink = n_sink ? reinterpret_cast<uint16_t*>(b + cp.v_sink) : nullptr;
  out->lens = lens;
  out->status = status;
  return TQ_OK;
}

tq_status tq_append(const tq_params* p, const tq_cache* cache, const int32_t* seq_ids, const void* k,
                    const void* v, int dtype, int n_tok, int n_seq, void* stream) {
  if (!p) return fail(TQ_ERR_ARG, "tq_append: NULL params");
  tq_status st = check_cache(p, cache, "tq_append");
  if (st != TQ_OK) return st;
  if (n_tok < 0 || n_seq < 0 || n_seq > cache->n_seq || (dtype != TQ_F32 && dtype != TQ_BF16))
    return fail(TQ_ERR_ARG, "tq_append: bad n_tok, n_seq or dtype");
  if (n_tok == 0 || n_seq == 0) return TQ_OK;
  if (!seq_ids || !k || !v) return fail(TQ_ERR_ARG, "tq_append: NULL input");
  if (!aligned16(k) || !aligned16(v)) return fail(TQ_ERR_ALIGN, "tq_append: inputs must be 16-byte aligned");
  return launch_append(p, cache, seq_ids, k, v, dtype == TQ_BF16, n_tok, n_seq,
                       static_cast<cudaStream_t>(stream));
}

static tq_status cache_rows(const tq_params* p, const tq_cache* cache, int which, int seq, int kv_head, int row0,
                            int64_t n, const tq_packed* rows, void* stream, int to_cache, const char* who) {
  if (!p) return fail(TQ_ERR_ARG, std::string(who) + ": NULL params");
  tq_status st = check_cache(p, cache, who);
  if (st != TQ_OK) return st;
  if ((which != TQ_K && which != TQ_V) || seq < 0 || seq >= cache->n_seq || kv_head < 0 ||
      kv_head >= cache->n_kv_heads || row0 < 0 || n < 0)
    return fail(TQ_ERR_ARG, std::string(who) + ": bad which, seq, kv_head, row0 or n");
  if (row0 + n > cache->capacity) return fail(TQ_ERR_CAPACITY, std::string(who) + ": rows past the cache's capacity");
  if (n == 0) return TQ_OK;
  st = check_packed(which == TQ_K ? p->fk : p->fv, rows, who);
  if (st != TQ_OK) return st;
  return launch_cache_rows(p, cache, which, seq, kv_head, row0, n, rows, to_cache, static_cast<cudaStream_t>(stream));
}

tq_status tq_cache_write_rows(const tq_params* p, const tq_cache* cache, int which, int seq, int kv_head, int row0,
                              int64_t n, const tq_packed* rows, void* stream) {
  return cache_rows(p, cache, which, seq, kv_head, row0, n, rows, stream, 1, "tq_cache_write_rows");
}

tq_status tq_cache_read_rows(const tq_params* p, const tq_cache* cache, int which, int seq, int kv_head, int row0,
                             int64_t n, const tq_packed* rows, void* stream) {
  return cache_rows(p, cache, which, seq, kv_head, row0, n, rows, stream, 0, "tq_cache_read_rows");
}

size_t tq_decode_workspace_bytes(const tq_params* p, int B, int hq, int n_kv_heads, int max_len) {
  if (!p || B < 1 || hq < 1 || n_kv_heads < 1 || hq % n_kv_heads || max_len < 0) return 0;
  return plan_decode(p, B, hq, n_kv_heads, max_len).ws_total_bytes;
}

tq_status tq_decode_workspace_init(void* workspace, size_t ws_bytes, void* stream) {
  if (!workspace || ws_bytes == 0) return fail(TQ_ERR_ARG, "tq_decode_workspace_init: bad arguments");
  cudaError_t e = cudaMemsetAsync(workspace, 0, ws_bytes, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? TQ_OK : cuda_fail(e, "tq_decode_workspace_init");
}

tq_status tq_decode_attn(const tq_params* p, const void* q, int q_dtype, const tq_cache* cache, int B,
                         int hq, int max_len, void* out, int out_dtype, void* workspace, size_t ws_bytes,
                         const tq_attn_flags* flags, void* stream) {
  DecodePlan plan;
  float thr = 0.f;
  unsigned long long* sv_stats = nullptr;
  tq_status st = check_decode_call(p, q, q_dtype, cache, B, hq, max_len, out, out_dtype, flags, "tq_decode_attn",
                                   &plan, &thr, &sv_stats);
  if (st != TQ_OK) return st;
  if (!workspace) return fail(TQ_ERR_ARG, "tq_decode_attn: NULL workspace");
  if (!aligned16(workspace)) return fail(TQ_ERR_ALIGN, "tq_decode_attn: workspace must be 16-byte aligned");
  if (ws_bytes < plan.ws_total_bytes) return fail(TQ_ERR_CAPACITY, "tq_decode_attn: workspace too small");
  return launch_decode(p, q, q_dtype == TQ_BF16, cache, plan, out, out_dtype == TQ_BF16, workspace, thr, sv_stats,
                       static_cast<cudaStream_t>(stream));
}

size_t tq_search_workspace_bytes(void) { return search_workspace_bytes(); }

tq_status tq_search(const tq_params* p, int which, const tq_packed* db, int64_t n, const void* q, int q_dtype,
                    int n_queries, int k, float* scores, int64_t* rows, void* workspace, size_t ws_bytes,
                    void* stream) {
  if (!p) return fail(TQ_ERR_ARG, "tq_search: NULL params");
  if ((which != TQ_K && which != TQ_V) || (q_dtype != TQ_F32 && q_dtype != TQ_BF16) || n < 0 ||
      n > INT32_MAX - 1 || n_queries < 1 || k < 1)
    return fail(TQ_ERR_ARG, "tq_search: bad which, dtype, n, n_queries or k");
  if (k > search_max_k()) return fail(TQ_ERR_UNSUPPORTED, "tq_search: k above 32");
  if (!q || !scores || !rows || !workspace) return fail(TQ_ERR_ARG, "tq_search: NULL q, scores, rows or workspace");
  if (!aligned16(q) || !aligned16(workspace))
    return fail(TQ_ERR_ALIGN, "tq_search: q and workspace must be 16-byte aligned");
  if (ws_bytes < search_workspace_bytes()) return fail(TQ_ERR_CAPACITY, "tq_search: workspace too small");
  const FormatSpec& f = which == TQ_K ? p->fk : p->fv;
  if (n > 0) {
    tq_status st = check_packed(f, db, "tq_search");
    if (st != TQ_OK) return st;
  } else if (!db) {
    return fail(TQ_ERR_ARG, "tq_search: NULL database");
  }
  return launch_search(p, f, db, n, q, q_dtype == TQ_BF16, n_queries, k, scores, rows, workspace,
                       static_cast<cudaStream_t>(stream));
}

}  // extern "C"
