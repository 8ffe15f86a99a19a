// Host side of libtq: random draws, Lloyd-Max codebooks, codec lifecycle, and
// the argument checking in front of every kernel launch.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <climits>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <new>
#include <string>
#include <vector>

#include "tq_internal.h"
#include "tq_trace.h"

namespace {

thread_local std::string g_last_error;

// ------------------------------------------------------------------ random draws
// splitmix64 (S. Vigna, public domain): the state advances by the golden-ratio
// increment and every output is the state passed through two xor-shift-multiply
// rounds and a final xor-shift.
struct SplitMix64 {
  uint64_t s;
  explicit SplitMix64(uint64_t seed) : s(seed) {}
  uint64_t next() {
    s += 0x9E3779B97F4A7C15ull;
    uint64_t z = s;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
  }
};

constexpr uint64_t kSketchSeedXor = 0x5851F42D4C957F2Dull;

// D: sign i is -1 when the top bit of the i-th output is set.
void draw_signs(uint64_t seed, int d, std::vector<uint32_t>& bits) {
  bits.assign((d + 31) / 32, 0u);
  SplitMix64 g(seed);
  for (int i = 0; i < d; ++i)
    if (g.next() >> 63) bits[i / 32] |= 1u << (i % 32);
}

// S: m x d row-major, one normal per pair of outputs by the Box-Muller cosine
// branch, u1 in (0, 1] and u2 in [0, 1) from the top 53 bits, rounded to fp32.
void draw_sketch(uint64_t seed, int m, int d, std::vector<float>& S) {
  S.resize((size_t)m * d);
  SplitMix64 g(seed ^ kSketchSeedXor);
  const double two_pi = 6.283185307179586476925286766559;
  for (size_t k = 0; k < S.size(); ++k) {
    const double u1 = (double)((g.next() >> 11) + 1) * 0x1.0p-53;
    const double u2 = (double)(g.next() >> 11) * 0x1.0p-53;
    S[k] = (float)(std::sqrt(-2.0 * std::log(u1)) * std::cos(two_pi * u2));
  }
}

// Haar rotation (tq_spec.rotation = TQ_ROTATION_HAAR): G, a d x d matrix of
// iid N(0, 1) drawn like S from splitmix64(seed ^ kHaarSeedXor), row-major;
// its columns are orthonormalised by Gram-Schmidt in fp64 with a second
// reorthogonalisation pass.  The result Q has a positive diagonal in R
// (G = QR), which makes it the unique Haar-distributed orthogonal matrix of
// the QR of G; the rotation is Pi = Q, y = Pi u.  Returned as Pi[j][i]
// (row-major) in fp64.
constexpr uint64_t kHaarSeedXor = 0x2545F4914F6CDD1Dull;

void draw_haar(uint64_t seed, int d, std::vector<double>& Pi) {
  std::vector<double> G((size_t)d * d);
  SplitMix64 g(seed ^ kHaarSeedXor);
  const double two_pi = 6.283185307179586476925286766559;
  for (size_t k = 0; k < G.size(); ++k) {
    const double u1 = (double)((g.next() >> 11) + 1) * 0x1.0p-53;
    const double u2 = (double)(g.next() >> 11) * 0x1.0p-53;
    G[k] = std::sqrt(-2.0 * std::log(u1)) * std::cos(two_pi * u2);
  }
  // columns of G: col c has entries G[r * d + c]
  Pi.assign((size_t)d * d, 0.0);
  std::vector<double> v(d);
  for (int c = 0; c < d; ++c) {
    for (int r = 0; r < d; ++r) v[r] = G[(size_t)r * d + c];
    for (int pass = 0; pass < 2; ++pass) {
      for (int k = 0; k < c; ++k) {
        double dot = 0.0;
        for (int r = 0; r < d; ++r) dot += Pi[(size_t)r * d + k] * v[r];
        for (int r = 0; r < d; ++r) v[r] -= dot * Pi[(size_t)r * d + k];
      }
    }
    double nrm = 0.0;
    for (int r = 0; r < d; ++r) nrm += v[r] * v[r];
    nrm = std::sqrt(nrm);
    for (int r = 0; r < d; ++r) Pi[(size_t)r * d + c] = v[r] / nrm;
  }
}

// ----------------------------------------------------------------- Lloyd-Max
// Gauss-Legendre rule on [-1, 1] by Newton's method on the Legendre recurrence.
struct GaussLegendre {
  std::vector<double> x, w;
  explicit GaussLegendre(int n) : x(n), w(n) {
    const double pi = 3.14159265358979323846;
    for (int i = 0; i < n; ++i) {
      double t = std::cos(pi * (i + 0.75) / (n + 0.5));
      double dp = 1.0;
      for (int it = 0; it < 100; ++it) {
        double p0 = 1.0, p1 = t;
        for (int k = 2; k <= n; ++k) {
          const double p2 = ((2.0 * k - 1.0) * t * p1 - (k - 1.0) * p0) / k;
          p0 = p1;
          p1 = p2;
        }
        dp = n * (t * p1 - p0) / (t * t - 1.0);
        const double dt = p1 / dp;
        t -= dt;
        if (std::fabs(dt) < 1e-16) break;
      }
      x[i] = t;
      w[i] = 2.0 / ((1.0 - t * t) * dp * dp);
    }
  }
};

// The law of z = sqrt(d) u_1 for u uniform on the unit sphere:
//   f_d(z) = C_d (1 - z^2/d)^((d-3)/2),  |z| < sqrt(d).
// With z = sqrt(d) sin(theta) the density becomes C_d sqrt(d) cos^(d-2)(theta),
// a smooth integrand on [-pi/2, pi/2], so Gauss-Legendre converges fast.
struct SphereMarginal {
  int d;
  double sd, cd;
  GaussLegendre gl{32};
  explicit SphereMarginal(int d_) : d(d_), sd(std::sqrt((double)d_)) {
    cd = std::exp(std::lgamma(0.5 * d) - std::lgamma(0.5 * (d - 1))) / std::sqrt(3.14159265358979323846 * d);
  }
  double theta(double z) const {
    const double s = z / sd;
    return std::asin(s > 1 ? 1.0 : (s < -1 ? -1.0 : s));
  }
  // P(a <= z <= b)
  double prob(double a, double b) const {
    const double ta = theta(a), tb = theta(b);
    const int panels = 16;
    const double h = (tb - ta) / panels;
    double acc = 0.0;
    for (int p = 0; p < panels; ++p) {
      const double c = ta + (p + 0.5) * h;
      for (size_t k = 0; k < gl.x.size(); ++k) {
        const double t = c + 0.5 * h * gl.x[k];
        acc += gl.w[k] * std::pow(std::cos(t), d - 2);
      }
    }
    return cd * sd * 0.5 * h * acc;
  }
  // E[z ; a <= z <= b] in closed form: the antiderivative of z f_d(z) is
  //   -C_d d/(d-1) (1 - z^2/d)^((d-1)/2).
  double first_moment(double a, double b) const {
    auto g = [&](double z) {
      const double t = 1.0 - z * z / d;
      return t > 0 ? std::exp(0.5 * (d - 1) * std::log1p(-z * z / d)) : 0.0;
    };
    return cd * d / (d - 1.0) * (g(a) - g(b));
  }
};

}  // namespace

// --------------------------------------------------------------------- errors
void tq_set_error(const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
}

tq_status tq_fail(tq_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

static tq_status cuda_fail(cudaError_t e, const char* what) {
  return tq_fail(TQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

extern "C" const char* tq_status_string(tq_status s) {
  switch (s) {
    case TQ_OK: return "ok";
    case TQ_ERR_INVALID_ARG: return "invalid argument";
    case TQ_ERR_UNSUPPORTED: return "unsupported configuration";
    case TQ_ERR_NO_MEMORY: return "out of memory";
    case TQ_ERR_CUDA: return "CUDA error";
    case TQ_ERR_DEVICE_ASSERT: return "device-side check failed";
    case TQ_ERR_NOT_CONVERGED: return "Lloyd-Max did not converge";
  }
  return "unknown status";
}

extern "C" const char* tq_last_error_string(void) { return g_last_error.c_str(); }

// ------------------------------------------------------------------- codebook
static tq_status lloyd_max(int bits, int d, double tol, int max_iter, std::vector<double>& cen) {
  const SphereMarginal f(d);
  const int L = 1 << bits, h = L / 2;
  std::vector<double> c(h), nc(h), b(h + 1);
  for (int j = 0; j < h; ++j) c[j] = std::min((j + 0.5) * 2.5 / h, 0.9 * f.sd);
  bool done = false;
  for (int it = 0; it < max_iter && !done; ++it) {
    b[0] = 0.0;
    for (int j = 1; j < h; ++j) b[j] = 0.5 * (c[j - 1] + c[j]);
    b[h] = f.sd;
    double delta = 0.0;
    for (int j = 0; j < h; ++j) {
      nc[j] = f.first_moment(b[j], b[j + 1]) / f.prob(b[j], b[j + 1]);
      delta = std::max(delta, std::fabs(nc[j] - c[j]));
    }
    c.swap(nc);
    done = delta < tol;
  }
  if (!done) return tq_fail(TQ_ERR_NOT_CONVERGED, "Lloyd-Max: no convergence in %d iterations", max_iter);
  cen.resize(L);
  for (int j = 0; j < h; ++j) {
    cen[h + j] = c[j];
    cen[h - 1 - j] = -c[j];
  }
  return TQ_OK;
}

extern "C" tq_status tq_make_codebook(int bits, int d, double tol, int max_iter, float* centroids,
                                      float* boundaries) {
  const tqtrace::Range trace("tq_make_codebook");
  if (bits < 1 || bits > 4) return tq_fail(TQ_ERR_INVALID_ARG, "bits must be 1..4 (got %d)", bits);
  if (d < 4) return tq_fail(TQ_ERR_INVALID_ARG, "d must be >= 4 (got %d)", d);
  if (!centroids || !boundaries) return tq_fail(TQ_ERR_INVALID_ARG, "null output pointer");
  if (tol <= 0) tol = 1e-12;
  if (max_iter <= 0) max_iter = 20000;
  std::vector<double> cen;
  const tq_status st = lloyd_max(bits, d, tol, max_iter, cen);
  if (st != TQ_OK) return st;
  const int L = 1 << bits;
  for (int k = 0; k < L; ++k) centroids[k] = (float)cen[k];
  for (int k = 0; k + 1 < L; ++k) boundaries[k] = (float)(0.5 * (cen[k] + cen[k + 1]));
  return TQ_OK;
}

// ---------------------------------------------------------------------- codec
static bool is_pow2(int v) { return v > 0 && (v & (v - 1)) == 0; }

static tq_status check_spec(const tq_spec* s) {
  if (!s) return tq_fail(TQ_ERR_INVALID_ARG, "null spec");
  const int d = s->d;
  if (!(d == 64 || d == 128 || d == 256 || d == 512 || d == 1024 || d == 1536))
    return tq_fail(TQ_ERR_UNSUPPORTED, "d = %d: need 64, 128, 256, 512, 1024 or 1536", d);
  if (s->nseg != 1 && s->nseg != 2) return tq_fail(TQ_ERR_INVALID_ARG, "nseg must be 1 or 2");
  for (int i = 0; i < s->nseg; ++i)
    if (s->seg_bits[i] < 1 || s->seg_bits[i] > 4)
      return tq_fail(TQ_ERR_INVALID_ARG, "seg_bits[%d] = %d not in 1..4", i, s->seg_bits[i]);
  if (s->m < 0 || s->m % 32 != 0 || s->m > TQ_MAX_M)
    return tq_fail(TQ_ERR_INVALID_ARG, "m = %d: need 0 or a multiple of 32 up to %d", s->m, TQ_MAX_M);
  if (s->residual != TQ_RESIDUAL_QJL && s->residual != TQ_RESIDUAL_SIGN)
    return tq_fail(TQ_ERR_INVALID_ARG, "residual = %d: need TQ_RESIDUAL_QJL or TQ_RESIDUAL_SIGN", s->residual);
  if (s->rotation != TQ_ROTATION_RHT && s->rotation != TQ_ROTATION_HAAR)
    return tq_fail(TQ_ERR_INVALID_ARG, "rotation = %d: need TQ_ROTATION_RHT or TQ_ROTATION_HAAR", s->rotation);
  if (s->rotation == TQ_ROTATION_HAAR && d > 256)
    return tq_fail(TQ_ERR_UNSUPPORTED, "TQ_ROTATION_HAAR: d = %d above 256", d);
  if (s->residual == TQ_RESIDUAL_SIGN && (s->nseg != 1 || s->m != d))
    return tq_fail(TQ_ERR_INVALID_ARG, "TQ_RESIDUAL_SIGN needs one segment and m = d (got nseg %d, m %d)", s->nseg,
                   s->m);
  if (s->vq_bits < 0 || s->vq_bits > TQ_MAX_VQ_BITS)
    return tq_fail(TQ_ERR_INVALID_ARG, "vq_bits = %d not in 0..%d", s->vq_bits, TQ_MAX_VQ_BITS);
  if (s->vq_bits > 0 && (s->nseg != 1 || s->residual != TQ_RESIDUAL_QJL))
    return tq_fail(TQ_ERR_UNSUPPORTED, "FibQuant codes (vq_bits %d) need nseg = 1 and TQ_RESIDUAL_QJL", s->vq_bits);
  return TQ_OK;
}

// ------------------------------------------------------- FibQuant, k = 2
// The codebook of the FibQuant page, sections 2.2 (construction) and 2.1 (the
// source): the block (z_2j, z_2j+1) of z = sqrt(d) u, u uniform on S^{d-1},
// has density proportional to (1 - |z|^2 / d)^((d - 4) / 2) on the disc of
// radius sqrt(d).
//  - initial codewords: a planar Fibonacci spiral, codeword n at angle
//    n * g + offset (g the golden angle 2 pi (1 - 1/phi)) and at the radius
//    where the Bennett-Gersho point density, proportional to the square root of
//    the block density, has put a fraction (n + 1/2) / N of the codewords:
//    r_n^2 = d (1 - (1 - (n + 1/2) / N)^(4 / d));
//  - Lloyd refinement: the expectation over the source is taken on M points
//    i = 0..M-1 at angle i * g and at the (i + 1/2) / M quantile of the radius
//    (|z|^2 / d ~ Beta(1, (d - 2) / 2): |z|^2 = d (1 - (1 - (i + 1/2) / M)^(2 / (d - 2))));
//    every iteration assigns each point to its nearest codeword (ties: lower
//    index) and moves every codeword with a nonempty cell to the cell's mean;
//  - restarts r = 0..R-1 turn the spiral by r g / R; the restart with the
//    least mean distortion is kept (ties: the first).
// Sums run in point order in double, so the result does not depend on
// threading; the cache holds one codebook per (vq_bits, d).
constexpr int kVqPoints = 16384;
constexpr int kVqIters = 40;
constexpr int kVqRestarts = 3;

static void fibquant_lloyd(int N, int d, double offset, const std::vector<double>& px, const std::vector<double>& py,
                           std::vector<double>& cx, std::vector<double>& cy, double* distortion) {
  const double pi = 3.14159265358979323846;
  const double g = pi * (3.0 - std::sqrt(5.0));
  cx.resize(N);
  cy.resize(N);
  for (int n = 0; n < N; ++n) {
    const double r = std::sqrt(d * (1.0 - std::pow(1.0 - (n + 0.5) / N, 4.0 / d)));
    const double a = n * g + offset;
    cx[n] = r * std::cos(a);
    cy[n] = r * std::sin(a);
  }
  const size_t M = px.size();
  std::vector<int> own(M);
  std::vector<double> sx(N), sy(N);
  std::vector<long> cnt(N);
  auto assign = [&]() {
    for (size_t i = 0; i < M; ++i) {
      int best = 0;
      double bd = INFINITY;
      for (int n = 0; n < N; ++n) {
        const double dx = px[i] - cx[n], dy = py[i] - cy[n];
        const double e = dx * dx + dy * dy;
        if (e < bd) {
          bd = e;
          best = n;
        }
      }
      own[i] = best;
    }
  };
  for (int it = 0; it < kVqIters; ++it) {
    assign();
    std::fill(sx.begin(), sx.end(), 0.0);
    std::fill(sy.begin(), sy.end(), 0.0);
    std::fill(cnt.begin(), cnt.end(), 0L);
    for (size_t i = 0; i < M; ++i) {
      sx[own[i]] += px[i];
      sy[own[i]] += py[i];
      ++cnt[own[i]];
    }
    for (int n = 0; n < N; ++n)
      if (cnt[n] > 0) {
        cx[n] = sx[n] / (double)cnt[n];
        cy[n] = sy[n] / (double)cnt[n];
      }
  }
  assign();
  double tot = 0.0;
  for (size_t i = 0; i < M; ++i) {
    const double dx = px[i] - cx[own[i]], dy = py[i] - cy[own[i]];
    tot += dx * dx + dy * dy;
  }
  *distortion = tot / (double)M;
}

static const std::vector<float>& fibquant_codebook(int vq_bits, int d) {
  static std::mutex mu;
  static std::map<std::pair<int, int>, std::vector<float>> cache;
  std::lock_guard<std::mutex> lock(mu);
  std::vector<float>& out = cache[{vq_bits, d}];
  if (!out.empty()) return out;
  const double pi = 3.14159265358979323846;
  const double g = pi * (3.0 - std::sqrt(5.0));
  std::vector<double> px(kVqPoints), py(kVqPoints);
  for (int i = 0; i < kVqPoints; ++i) {
    const double r = std::sqrt(d * (1.0 - std::pow(1.0 - (i + 0.5) / kVqPoints, 2.0 / (d - 2))));
    const double a = i * g;
    px[i] = r * std::cos(a);
    py[i] = r * std::sin(a);
  }
  const int N = 1 << vq_bits;
  double best = INFINITY;
  std::vector<double> cx, cy;
  for (int rs = 0; rs < kVqRestarts; ++rs) {
    double dist = 0.0;
    fibquant_lloyd(N, d, rs * g / kVqRestarts, px, py, cx, cy, &dist);
    if (dist < best) {
      best = dist;
      out.resize(2 * (size_t)N);
      for (int n = 0; n < N; ++n) {
        out[2 * n] = (float)cx[n];
        out[2 * n + 1] = (float)cy[n];
      }
    }
  }
  return out;
}

// Mean residual magnitude mu = E|z - cen[code(z)]| under f_d for a published
// codebook (fp32 centroids and boundaries, ascending): per cell, split at its
// centroid,
//   int_cell |z - c| f = c (P(lo, c) - P(c, hi)) - M1(lo, c) + M1(c, hi),
// with P and M1 the probability and first moment of f_d between the limits.
static double residual_mean_magnitude(int d, const std::vector<float>& cen, const std::vector<float>& bnd) {
  const SphereMarginal f(d);
  const double edge = std::sqrt((double)d);
  double mu = 0.0;
  const int L = (int)cen.size();
  for (int k = 0; k < L; ++k) {
    const double lo = k == 0 ? -edge : (double)bnd[k - 1];
    const double hi = k == L - 1 ? edge : (double)bnd[k];
    const double c = (double)cen[k];
    mu += c * (f.prob(lo, c) - f.prob(c, hi)) - f.first_moment(lo, c) + f.first_moment(c, hi);
  }
  return mu;
}

static size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

extern "C" tq_status tq_codec_create(const tq_spec* spec, int device, tq_codec** out) {
  const tqtrace::Range trace("tq_codec_create");
  tq_status st = check_spec(spec);
  if (st != TQ_OK) return st;
  if (!out) return tq_fail(TQ_ERR_INVALID_ARG, "null output pointer");
  if (device < -1) return tq_fail(TQ_ERR_INVALID_ARG, "device %d", device);
  tq_codec* c = new (std::nothrow) tq_codec();
  if (!c) return tq_fail(TQ_ERR_NO_MEMORY, "host allocation");
  c->spec = *spec;
  if (spec->nseg == 1) c->spec.seg_bits[1] = 0;
  c->device = device;
  const int d = spec->d, m = spec->m;
  tq_params& p = c->p;
  std::memset(&p, 0, sizeof p);
  p.out_stride = 1;  // compressed row r is output row r (tq_append changes the map per call)
  p.d = d;
  p.nseg = spec->nseg;
  p.seg_len = d / spec->nseg;
  p.pw = p.seg_len / 32;
  p.m = m;
  p.MS = m / 32;
  p.hblock = is_pow2(d) ? d : TQ_HBLOCK_MAX;
  p.log2_hblock = 0;
  while ((1 << p.log2_hblock) < p.hblock) ++p.log2_hblock;
  p.zscale = (float)std::sqrt((double)d / p.hblock);
  p.inv_sqrt_d = (float)(1.0 / std::sqrt((double)d));
  p.inv_sqrt_p = (float)(1.0 / std::sqrt((double)p.hblock));
  p.qjl_coef = m > 0 ? (float)(std::sqrt(3.14159265358979323846 / 2.0) / m) : 0.0f;
  int W = 0;
  for (int s = 0; s < (spec->vq_bits ? 0 : spec->nseg); ++s) {
    const int bits = spec->seg_bits[s];
    p.bits[s] = bits;
    p.segbase[s] = W;
    W += bits * p.pw;
    std::vector<double> cen;
    st = lloyd_max(bits, d, 1e-12, 20000, cen);
    if (st != TQ_OK) {
      delete c;
      return st;
    }
    const int L = 1 << bits;
    c->cen_host[s].resize(L);
    c->bnd_host[s].resize(L - 1);
    for (int k = 0; k < TQ_MAX_LEVELS; ++k) p.bnd[s][k] = INFINITY;
    for (int k = 0; k < L; ++k) {
      c->cen_host[s][k] = (float)cen[k];
      p.cen[s][k] = c->cen_host[s][k];
      p.cmax = std::max(p.cmax, std::fabs(p.cen[s][k]));
    }
    for (int k = 0; k + 1 < L; ++k) {
      c->bnd_host[s][k] = (float)(0.5 * (cen[k] + cen[k + 1]));
      p.bnd[s][k] = c->bnd_host[s][k];
    }
  }
  if (spec->vq_bits) {
    // FibQuant block codes: no scalar tables (bits 0, every boundary +inf)
    c->spec.seg_bits[0] = 0;
    p.bits[0] = 0;
    for (int k = 0; k < TQ_MAX_LEVELS; ++k) p.bnd[0][k] = p.bnd[1][k] = INFINITY;
    p.vq_bits = spec->vq_bits;
    p.vq_pw = d / 64;
    W = p.vq_bits * p.vq_pw;
    c->vq_host = fibquant_codebook(spec->vq_bits, d);
    for (float v : c->vq_host) p.cmax = std::max(p.cmax, std::fabs(v));
  }
  p.W = W;
  // plane-identity coefficients: alpha_t = 2^-b sum_c cen[c] prod_{k in t} s_k(c)
  p.plane_ok = spec->vq_bits ? 0 : 1;
  for (int s = 0; s < (spec->vq_bits ? 0 : spec->nseg); ++s) {
    const int bits = spec->seg_bits[s], L = 1 << bits;
    p.nterms[s] = tq_term_count[bits];
    for (int t = 0; t < p.nterms[s]; ++t) {
      double a = 0.0;
      for (int code = 0; code < L; ++code) {
        double prod = 1.0;
        for (int k = 0; k < bits; ++k)
          if ((tq_term_mask[bits][t] >> k) & 1) prod *= ((code >> k) & 1) ? 1.0 : -1.0;
        a += (double)c->cen_host[s][code] * prod;
      }
      p.alpha[s][t] = (float)(a / L);
    }
    for (int code = 0; code < L; ++code) {
      double rec = 0.0;
      for (int t = 0; t < p.nterms[s]; ++t) {
        double prod = 1.0;
        for (int k = 0; k < bits; ++k)
          if ((tq_term_mask[bits][t] >> k) & 1) prod *= ((code >> k) & 1) ? 1.0 : -1.0;
        rec += (double)p.alpha[s][t] * prod;
      }
      if (std::fabs(rec - c->cen_host[s][code]) > 1e-6 * (1.0 + std::fabs(c->cen_host[s][code]))) p.plane_ok = 0;
    }
  }
  draw_signs(spec->seed, d, c->dbits_host);
  if (spec->rotation == TQ_ROTATION_HAAR) {
    // the dense Haar rotation replaces H D / sqrt(d): D = I
    std::fill(c->dbits_host.begin(), c->dbits_host.end(), 0u);
    draw_haar(spec->seed, d, c->haar);
    p.haar = 1;
  }
  if (spec->residual == TQ_RESIDUAL_SIGN) {
    // per-element residual sign: S = I (m = d), every row's stored residual
    // scale is the constant mu sqrt(2d/pi), so that the estimator's
    // gamma sqrt(pi/2)/m factor equals mu / sqrt(d)
    c->S_host.assign((size_t)d * d, 0.0f);
    for (int i = 0; i < d; ++i) c->S_host[(size_t)i * d + i] = 1.0f;
    c->mu = residual_mean_magnitude(d, c->cen_host[0], c->bnd_host[0]);
    p.rnorm_const = (float)(c->mu * std::sqrt(2.0 * d / 3.14159265358979323846));
    p.rnorm_is_const = 1;
  } else if (m > 0) {
    draw_sketch(spec->seed, m, d, c->S_host);
  }

  if (device >= 0) {
    int cur = -1;
    cudaError_t e = cudaGetDevice(&cur);
    if (e != cudaSuccess) {
      delete c;
      return cuda_fail(e, "cudaGetDevice");
    }
    if (cur != device) {
      delete c;
      return tq_fail(TQ_ERR_INVALID_ARG, "device %d is not the current device (%d)", device, cur);
    }
    // one block: S [m][d] | St [d][m] | s_l1 [m] | s_l2 [m] | dbits | bimg | dmask | sl1n | sl2n | err
    const int Q = m / 32;
    std::vector<float> St((size_t)d * m), l1(m), l2(m), l1n(m), l2n(m);
    for (int j = 0; j < m; ++j) {
      double a1 = 0, a2 = 0;
      for (int i = 0; i < d; ++i) {
        const double v = c->S_host[(size_t)j * d + i];
        a1 += std::fabs(v);
        a2 += v * v;
      }
      l1n[j] = (float)(a1 * (1 + 1e-6));
      l2n[j] = (float)(std::sqrt(a2) * (1 + 1e-6));
    }
    for (int lane = 0; lane < 32; ++lane)
      for (int q = 0; q < Q; ++q) {
        const int j = lane + 32 * q, col = lane * Q + q;
        for (int i = 0; i < d; ++i) St[(size_t)i * m + col] = c->S_host[(size_t)j * d + i];
        l1[col] = l1n[j];
        l2[col] = l2n[j];
      }
    // fp16 split S = S_hi + S_lo (+ error <= 2^-22 |S| + 2^-25) in the tensor-core operand layout
    std::vector<uint16_t> bimg(2 * (size_t)m * d);
    for (int j = 0; j < m; ++j)
      for (int i = 0; i < d; ++i) {
        const float v = c->S_host[(size_t)j * d + i];
        const __half hi = __float2half_rn(v);
        const __half lo = __float2half_rn(v - __half2float(hi));
        const size_t off = ((size_t)(i / 8) * 16 * m + (size_t)(j / 8) * 128 + (j % 8) * 16 + (i % 8) * 2) / 2;
        bimg[off] = __half_as_ushort(hi);
        bimg[(size_t)m * d + off] = __half_as_ushort(lo);
      }
    std::vector<uint32_t> dmask(d);
    for (int i = 0; i < d; ++i) dmask[i] = ((c->dbits_host[i / 32] >> (i % 32)) & 1u) ? 0x80000000u : 0u;
    const size_t oS = 0, oSt = align256(oS + sizeof(float) * (size_t)m * d);
    const size_t o1 = align256(oSt + sizeof(float) * (size_t)m * d);
    const size_t o2 = align256(o1 + sizeof(float) * m);
    const size_t oD = align256(o2 + sizeof(float) * m);
    const size_t oB = align256(oD + sizeof(uint32_t) * c->dbits_host.size());
    const size_t oM = align256(oB + sizeof(uint16_t) * bimg.size());
    const size_t o1n = align256(oM + sizeof(uint32_t) * d);
    const size_t o2n = align256(o1n + sizeof(float) * m);
    const size_t oE = align256(o2n + sizeof(float) * m);
    const size_t oH = align256(oE + 16);  // Haar: Pi^T [d][d] fp32 (element (i, j) = Pi_ji)
    const size_t oV = align256(oH + (p.haar ? sizeof(float) * (size_t)d * d : 0));  // FibQuant codebook
    const size_t total = align256(oV + sizeof(float) * c->vq_host.size());
    e = cudaMalloc(&c->dev_block, total);
    if (e != cudaSuccess) {
      delete c;
      cudaGetLastError();
      return tq_fail(TQ_ERR_NO_MEMORY, "cudaMalloc(%zu): %s", total, cudaGetErrorString(e));
    }
    char* base = (char*)c->dev_block;
    e = cudaMemset(base, 0, total);
    if (e == cudaSuccess)
      e = cudaMemcpy(base + oD, c->dbits_host.data(), sizeof(uint32_t) * c->dbits_host.size(), cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMemcpy(base + oM, dmask.data(), sizeof(uint32_t) * d, cudaMemcpyHostToDevice);
    if (e == cudaSuccess && m > 0) {
      e = cudaMemcpy(base + oS, c->S_host.data(), sizeof(float) * (size_t)m * d, cudaMemcpyHostToDevice);
      if (e == cudaSuccess) e = cudaMemcpy(base + oSt, St.data(), sizeof(float) * St.size(), cudaMemcpyHostToDevice);
      if (e == cudaSuccess) e = cudaMemcpy(base + o1, l1.data(), sizeof(float) * m, cudaMemcpyHostToDevice);
      if (e == cudaSuccess) e = cudaMemcpy(base + o2, l2.data(), sizeof(float) * m, cudaMemcpyHostToDevice);
      if (e == cudaSuccess) e = cudaMemcpy(base + oB, bimg.data(), sizeof(uint16_t) * bimg.size(), cudaMemcpyHostToDevice);
      if (e == cudaSuccess) e = cudaMemcpy(base + o1n, l1n.data(), sizeof(float) * m, cudaMemcpyHostToDevice);
      if (e == cudaSuccess) e = cudaMemcpy(base + o2n, l2n.data(), sizeof(float) * m, cudaMemcpyHostToDevice);
    }
    if (e == cudaSuccess && p.haar) {
      std::vector<float> PiT((size_t)d * d);
      for (int j = 0; j < d; ++j)
        for (int i = 0; i < d; ++i) PiT[(size_t)i * d + j] = (float)c->haar[(size_t)j * d + i];
      e = cudaMemcpy(base + oH, PiT.data(), sizeof(float) * PiT.size(), cudaMemcpyHostToDevice);
    }
    if (e == cudaSuccess && p.vq_bits)
      e = cudaMemcpy(base + oV, c->vq_host.data(), sizeof(float) * c->vq_host.size(), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) {
      cudaFree(c->dev_block);
      delete c;
      return cuda_fail(e, "codec upload");
    }
    if (p.haar) p.piT = (const float*)(base + oH);
    if (p.vq_bits) p.vq_cb = (const float*)(base + oV);
    p.S = (const float*)(base + oS);
    p.St = (const float*)(base + oSt);
    p.s_l1 = (const float*)(base + o1);
    p.s_l2 = (const float*)(base + o2);
    p.dbits = (const uint32_t*)(base + oD);
    p.bimg = (const uint16_t*)(base + oB);
    p.dmask = (const uint32_t*)(base + oM);
    p.sl1n = (const float*)(base + o1n);
    p.sl2n = (const float*)(base + o2n);
    p.err = (uint32_t*)(base + oE);
    p.exact_rows = (unsigned long long*)(base + oE + 8);
  }
  *out = c;
  return TQ_OK;
}

extern "C" tq_status tq_codec_destroy(tq_codec* c) {
  if (!c) return TQ_OK;
  tq_status st = TQ_OK;
  if (c->dev_block) {
    int cur = -1;
    cudaGetDevice(&cur);
    if (cur != c->device) cudaSetDevice(c->device);
    const cudaError_t e = cudaFree(c->dev_block);
    if (cur != c->device && cur >= 0) cudaSetDevice(cur);
    if (e != cudaSuccess) st = cuda_fail(e, "cudaFree");
  }
  delete c;
  return st;
}

extern "C" tq_status tq_codec_export(const tq_codec* c, float* S, uint32_t* dsigns, float* cen, float* bnd) {
  if (!c) return tq_fail(TQ_ERR_INVALID_ARG, "null codec");
  if (S && c->spec.m > 0) std::copy(c->S_host.begin(), c->S_host.end(), S);
  if (dsigns) std::copy(c->dbits_host.begin(), c->dbits_host.end(), dsigns);
  for (int s = 0; s < c->spec.nseg; ++s) {
    if (cen) cen = std::copy(c->cen_host[s].begin(), c->cen_host[s].end(), cen);
    if (bnd) bnd = std::copy(c->bnd_host[s].begin(), c->bnd_host[s].end(), bnd);
  }
  return TQ_OK;
}

extern "C" tq_status tq_codec_vq_codebook(const tq_codec* c, float* cb) {
  if (!c || !cb) return tq_fail(TQ_ERR_INVALID_ARG, "tq_codec_vq_codebook: null argument");
  if (!c->p.vq_bits) return tq_fail(TQ_ERR_INVALID_ARG, "tq_codec_vq_codebook: the codec has scalar codes");
  std::copy(c->vq_host.begin(), c->vq_host.end(), cb);
  return TQ_OK;
}

extern "C" tq_status tq_codec_rotation(const tq_codec* c, float* Pi) {
  if (!c || !Pi) return tq_fail(TQ_ERR_INVALID_ARG, "tq_codec_rotation: null argument");
  const int d = c->p.d;
  if (c->p.haar) {
    for (size_t k = 0; k < (size_t)d * d; ++k) Pi[k] = (float)c->haar[k];
    return TQ_OK;
  }
  // randomized Hadamard: Pi_ji = H_p[j % p][i % p] D_i / sqrt(p) inside the blocks
  const int hp = c->p.hblock;
  const double sc = 1.0 / std::sqrt((double)hp);
  for (int j = 0; j < d; ++j)
    for (int i = 0; i < d; ++i) {
      double v = 0.0;
      if (j / hp == i / hp) {
        const int par = __builtin_popcount((unsigned)((j % hp) & (i % hp))) & 1;
        const bool neg = (c->dbits_host[i / 32] >> (i % 32)) & 1u;
        v = ((par != 0) != neg ? -1.0 : 1.0) * sc;
      }
      Pi[(size_t)j * d + i] = (float)v;
    }
  return TQ_OK;
}

extern "C" tq_status tq_codec_layout(const tq_codec* c, int* code_words, int* sign_words) {
  if (!c) return tq_fail(TQ_ERR_INVALID_ARG, "null codec");
  if (code_words) *code_words = c->p.W;
  if (sign_words) *sign_words = c->p.MS;
  return TQ_OK;
}

// ------------------------------------------------------------ compute checks
static bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

static size_t dtype_size(tq_dtype dt) { return dt == TQ_F32 ? 4 : 2; }

static tq_status check_device_codec(const tq_codec* c, const char* name) {
  if (!c) return tq_fail(TQ_ERR_INVALID_ARG, "%s: null codec", name);
  if (c->device < 0) return tq_fail(TQ_ERR_INVALID_ARG, "%s: host-only codec", name);
  int cur = -1;
  const cudaError_t e = cudaGetDevice(&cur);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (cur != c->device)
    return tq_fail(TQ_ERR_INVALID_ARG, "%s: current device %d is not the codec's device %d", name, cur, c->device);
  return TQ_OK;
}

static tq_status check_dtype(tq_dtype dt) {
  if (dt != TQ_F32 && dt != TQ_BF16 && dt != TQ_F16) return tq_fail(TQ_ERR_INVALID_ARG, "dtype %d", (int)dt);
  return TQ_OK;
}

static tq_status check_compressed(const tq_codec* c, const tq_compressed* t, const char* name) {
  if (!t) return tq_fail(TQ_ERR_INVALID_ARG, "%s: null tq_compressed", name);
  if (!t->codes || !aligned16(t->codes)) return tq_fail(TQ_ERR_INVALID_ARG, "%s.codes null or not 16-byte aligned", name);
  if (!t->norms || !aligned16(t->norms)) return tq_fail(TQ_ERR_INVALID_ARG, "%s.norms null or not 16-byte aligned", name);
  if (c->p.m > 0) {
    if (!t->signs || !aligned16(t->signs))
      return tq_fail(TQ_ERR_INVALID_ARG, "%s.signs null or not 16-byte aligned (m = %d)", name, c->p.m);
    if (!t->rnorms || !aligned16(t->rnorms))
      return tq_fail(TQ_ERR_INVALID_ARG, "%s.rnorms null or not 16-byte aligned (m = %d)", name, c->p.m);
  }
  return TQ_OK;
}

static tq_status launch_status(cudaError_t e, const char* what) {
  if (e != cudaSuccess) return cuda_fail(e, what);
  return TQ_OK;
}

extern "C" tq_status tq_quantize(const tq_codec* c, const void* x, tq_dtype dt, int64_t n, int64_t ld,
                                 const tq_compressed* out, void* stream) {
  const tqtrace::Range trace("tq_quantize");
  tq_status st = check_device_codec(c, "tq_quantize");
  if (st != TQ_OK) return st;
  if ((st = check_dtype(dt)) != TQ_OK) return st;
  if (n < 0) return tq_fail(TQ_ERR_INVALID_ARG, "tq_quantize: n = %lld", (long long)n);
  if (ld < c->p.d) return tq_fail(TQ_ERR_INVALID_ARG, "tq_quantize: ld %lld < d %d", (long long)ld, c->p.d);
  if ((ld * (int64_t)dtype_size(dt)) % 16 != 0)
    return tq_fail(TQ_ERR_INVALID_ARG, "tq_quantize: row pitch %lld bytes is not a multiple of 16",
                   (long long)(ld * (int64_t)dtype_size(dt)));
  if (n == 0) return TQ_OK;
  if (!x || !aligned16(x)) return tq_fail(TQ_ERR_INVALID_ARG, "tq_quantize: x null or not 16-byte aligned");
  if ((st = check_compressed(c, out, "out")) != TQ_OK) return st;
  cudaError_t e = tq_launch_quantize_tc(c->p, x, dt, n, ld, *out, (cudaStream_t)stream);
  if (e == cudaErrorNotSupported) e = tq_launch_quantize(c->p, x, dt, n, ld, *out, (cudaStream_t)stream);
  return launch_status(e, "tq_quantize launch");
}

// row checks shared by tq_quantize_rope and tq_append
static tq_status check_rows(const tq_codec* c, const void* x, tq_dtype dt, int64_t n, int64_t ld, const char* name) {
  tq_status st = check_device_codec(c, name);
  if (st != TQ_OK) return st;
  if ((st = check_dtype(dt)) != TQ_OK) return st;
  if (n < 0) return tq_fail(TQ_ERR_INVALID_ARG, "%s: n = %lld", name, (long long)n);
  if (ld < c->p.d) return tq_fail(TQ_ERR_INVALID_ARG, "%s: ld %lld < d %d", name, (long long)ld, c->p.d);
  if ((ld * (int64_t)dtype_size(dt)) % 16 != 0)
    return tq_fail(TQ_ERR_INVALID_ARG, "%s: row pitch %lld bytes is not a multiple of 16", name,
                   (long long)(ld * (int64_t)dtype_size(dt)));
  if (n > 0 && (!x || !aligned16(x))) return tq_fail(TQ_ERR_INVALID_ARG, "%s: x null or not 16-byte aligned", name);
  return TQ_OK;
}

static tq_status check_rope(const tq_codec* c, const tq_rope* rope, bool need_positions, const char* name) {
  if (!rope) return tq_fail(TQ_ERR_INVALID_ARG, "%s: rope null", name);
  if (!rope->cos_sin || !aligned16(rope->cos_sin))
    return tq_fail(TQ_ERR_INVALID_ARG, "%s: rope cos_sin null or not 16-byte aligned", name);
  if (rope->max_pos <= 0) return tq_fail(TQ_ERR_INVALID_ARG, "%s: rope max_pos = %d", name, (int)rope->max_pos);
  if (need_positions && (!rope->positions || ((uintptr_t)rope->positions & 3u)))
    return tq_fail(TQ_ERR_INVALID_ARG, "%s: rope positions null or not 4-byte aligned", name);
  if (c->p.d % 2 != 0) return tq_fail(TQ_ERR_UNSUPPORTED, "%s: odd d", name);
  return TQ_OK;
}

extern "C" tq_status tq_rope_cache(double theta, int d, int max_pos, float* cos_sin, void* stream) {
  const tqtrace::Range trace("tq_rope_cache");
  if (!(theta > 1.0) || d <= 0 || d % 2 != 0 || max_pos < 0)
    return tq_fail(TQ_ERR_INVALID_ARG, "tq_rope_cache: theta %g, d %d, max_pos %d", theta, d, max_pos);
  if (max_pos == 0) return TQ_OK;
  if (!cos_sin || !aligned16(cos_sin)) return tq_fail(TQ_ERR_INVALID_ARG, "tq_rope_cache: cos_sin null or misaligned");
  return launch_status(tq_launch_rope_cache(theta, d, max_pos, cos_sin, (cudaStream_t)stream), "tq_rope_cache launch");
}

extern "C" tq_status tq_quantize_rope(const tq_codec* c, const void* x, tq_dtype dt, int64_t n, int64_t ld,
                                      const tq_rope* rope, const tq_compressed* out, void* stream) {
  const tqtrace::Range trace("tq_quantize_rope");
  tq_status st = check_rows(c, x, dt, n, ld, "tq_quantize_rope");
  if (st != TQ_OK) return st;
  if ((st = check_rope(c, rope, true, "tq_quantize_rope")) != TQ_OK) return st;
  if (n == 0) return TQ_OK;
  if ((st = check_compressed(c, out, "out")) != TQ_OK) return st;
  tq_params p = c->p;
  p.rope_cs = rope->cos_sin;
  p.rope_pos = rope->positions;
  p.rope_max_pos = rope->max_pos;
  const cudaError_t e = tq_launch_quantize_tc_rope(p, x, dt, n, ld, *out, (cudaStream_t)stream);
  if (e == cudaErrorNotSupported)
    return tq_fail(TQ_ERR_UNSUPPORTED, "tq_quantize_rope: needs d of 64 or 128, bf16 or fp32 rows and m <= 256");
  return launch_status(e, "tq_quantize_rope launch");
}

extern "C" tq_status tq_append(const tq_codec* c, const void* x, tq_dtype dt, int64_t rows, int64_t ld,
                               const tq_rope* rope, int64_t t, int64_t T, const tq_compressed* cache, void* stream) {
  const tqtrace::Range trace("tq_append");
  tq_status st = check_rows(c, x, dt, rows, ld, "tq_append");
  if (st != TQ_OK) return st;
  if (T <= 0 || t < 0 || t >= T)
    return tq_fail(TQ_ERR_INVALID_ARG, "tq_append: position t = %lld outside [0, T = %lld)", (long long)t,
                   (long long)T);
  if (rope) {
    if ((st = check_rope(c, rope, false, "tq_append")) != TQ_OK) return st;
    if (t >= rope->max_pos)
      return tq_fail(TQ_ERR_INVALID_ARG, "tq_append: t = %lld beyond the RoPE cache (%d positions)", (long long)t,
                     (int)rope->max_pos);
  }
  if (rows == 0) return TQ_OK;
  if ((st = check_compressed(c, cache, "cache")) != TQ_OK) return st;
  tq_params p = c->p;
  p.out_stride = T;  // input row r -> cache row r * T + t
  p.out_offset = t;
  cudaError_t e;
  if (rope) {
    p.rope_cs = rope->cos_sin;
    p.rope_pos = nullptr;
    p.rope_pos_fixed = (int)t;
    p.rope_max_pos = rope->max_pos;
    e = tq_launch_quantize_tc_rope(p, x, dt, rows, ld, *cache, (cudaStream_t)stream);
    if (e == cudaErrorNotSupported)
      return tq_fail(TQ_ERR_UNSUPPORTED, "tq_append with RoPE: needs d of 64 or 128, bf16 or fp32 rows and m <= 256");
  } else {
    e = tq_launch_quantize_tc(p, x, dt, rows, ld, *cache, (cudaStream_t)stream);
    if (e == cudaErrorNotSupported) e = tq_launch_quantize(p, x, dt, rows, ld, *cache, (cudaStream_t)stream);
  }
  return launch_status(e, "tq_append launch");
}

static size_t qprep_bytes(const tq_params& p, size_t nq) { return align256(sizeof(float) * nq * (size_t)(p.d + p.m)); }

// B * Hq (and B * Hkv) index query and head arrays with int arithmetic in the
// kernels and the size helpers: larger products are refused.
static bool heads_fit_int(int B, int Hq, int Hkv) {
  return (int64_t)B * Hq <= INT_MAX && (int64_t)B * Hkv <= INT_MAX;
}

static size_t scores_bytes(const tq_params& p, int B, int Hq, int Hkv) {
  return qprep_bytes(p, (size_t)B * Hq) + align256(tq_scores_tc_bytes(p, B, Hq, Hkv));
}

extern "C" tq_status tq_scores_workspace_size(const tq_codec* kc, int B, int Hq, int Hkv, size_t* bytes) {
  if (!kc || !bytes) return tq_fail(TQ_ERR_INVALID_ARG, "tq_scores_workspace_size: null argument");
  if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv)
    return tq_fail(TQ_ERR_INVALID_ARG, "tq_scores_workspace_size: bad shape B=%d Hq=%d Hkv=%d", B, Hq, Hkv);
  if (!heads_fit_int(B, Hq, Hkv))
    return tq_fail(TQ_ERR_UNSUPPORTED, "tq_scores_workspace_size: B*Hq or B*Hkv above INT_MAX");
  *bytes = scores_bytes(kc->p, B, Hq, Hkv);
  return TQ_OK;
}

static tq_status check_heads(int B, int Hq, int Hkv, int64_t T, const char* name) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || T < 0)
    return tq_fail(TQ_ERR_INVALID_ARG, "%s: bad shape B=%d Hq=%d Hkv=%d T=%lld", name, B, Hq, Hkv, (long long)T);
  if (Hq % Hkv != 0) return tq_fail(TQ_ERR_INVALID_ARG, "%s: Hq %d not a multiple of Hkv %d", name, Hq, Hkv);
  if (Hq / Hkv > 32) return tq_fail(TQ_ERR_UNSUPPORTED, "%s: Hq/Hkv = %d above 32", name, Hq / Hkv);
  if (!heads_fit_int(B, Hq, Hkv)) return tq_fail(TQ_ERR_UNSUPPORTED, "%s: B*Hq or B*Hkv above INT_MAX", name);
  if (T > (int64_t)1 << 31) return tq_fail(TQ_ERR_UNSUPPORTED, "%s: T above 2^31", name);
  return TQ_OK;
}

extern "C" tq_status tq_scores(const tq_codec* kc, const void* q, tq_dtype dt, int B, int Hq, int Hkv, int64_t T,
                               const tq_compressed* K, float* logits, void* workspace, size_t ws_bytes,
                               void* stream) {
  const tqtrace::Range trace("tq_scores");
  tq_status st = check_device_codec(kc, "tq_scores");
  if (st != TQ_OK) return st;
  if ((st = check_dtype(dt)) != TQ_OK) return st;
  if ((st = check_heads(B, Hq, Hkv, T, "tq_scores")) != TQ_OK) return st;
  if (B == 0 || T == 0) return TQ_OK;
  if (!q || !aligned16(q)) return tq_fail(TQ_ERR_INVALID_ARG, "tq_scores: q null or not 16-byte aligned");
  if (!logits || !aligned16(logits)) return tq_fail(TQ_ERR_INVALID_ARG, "tq_scores: logits null or not 16-byte aligned");
  if ((st = check_compressed(kc, K, "K")) != TQ_OK) return st;
  const size_t need = scores_bytes(kc->p, B, Hq, Hkv);
  if (!workspace || !aligned16(workspace) || ws_bytes < need)
    return tq_fail(TQ_ERR_INVALID_ARG, "tq_scores: workspace null, misaligned or smaller than %zu bytes", need);
  const cudaStream_t s = (cudaStream_t)stream;
  float* qprep = (float*)workspace;
  cudaError_t e;
  e = tq_launch_qprep(kc->p, q, dt, B * Hq, qprep, s);
  if (e == cudaSuccess) {
    if (tq_scores_tc_supported(kc->p, Hq, Hkv)) {
      void* ws_tc = (char*)workspace + qprep_bytes(kc->p, (size_t)B * Hq);
      e = tq_launch_scores_tc(kc->p, qprep, B, Hq, Hkv, T, *K, logits, ws_tc, s);
    } else {
      e = tq_launch_scores(kc->p, qprep, B, Hq, Hkv, T, *K, logits, s);
    }
  }
  return launch_status(e, "tq_scores launch");
}

static int device_sms(int device) {
  int v = 0;
  if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, device) != cudaSuccess || v <= 0) v = 148;
  return v;
}

// partials per (b, hq, chunk): acc[d], max, sum, and the values' sketch
// accumulator a[m] when the value codec has m > 0 (QJL-corrected values)
static size_t attend_bytes(const tq_params& kp, const tq_params& vp, int B, int Hq, int nchunk) {
  return qprep_bytes(kp, (size_t)B * Hq) +
         align256(sizeof(float) * (size_t)B * Hq * nchunk * (size_t)(kp.d + 2 + vp.m));
}

extern "C" tq_status tq_attend_workspace_size(const tq_codec* kc, const tq_codec* vc, int B, int Hq, int Hkv,
                                              int64_t T, size_t* bytes) {
  if (!kc || !vc || !bytes) return tq_fail(TQ_ERR_INVALID_ARG, "tq_attend_workspace_size: null argument");
  tq_status st = check_heads(B, Hq, Hkv, T, "tq_attend_workspace_size");
  if (st != TQ_OK) return st;
  const int nchunk = tq_attend_chunks(B, Hq, Hkv, T, device_sms(kc->device < 0 ? 0 : kc->device));
  *bytes = attend_bytes(kc->p, vc->p, B, Hq, nchunk);
  return TQ_OK;
}

extern "C" tq_status tq_attend(const tq_codec* kc, const tq_codec* vc, const void* q, tq_dtype dt, int B, int Hq,
                               int Hkv, int64_t T, float scale, const tq_compressed* K, const tq_compressed* V,
                               void* workspace, size_t ws_bytes, float* out, void* stream) {
  const tqtrace::Range trace("tq_attend");
  tq_status st = check_device_codec(kc, "tq_attend");
  if (st != TQ_OK) return st;
  if ((st = check_device_codec(vc, "tq_attend")) != TQ_OK) return st;
  if (kc->p.d != vc->p.d) return tq_fail(TQ_ERR_INVALID_ARG, "tq_attend: key d %d != value d %d", kc->p.d, vc->p.d);
  if (kc->p.d > 256) return tq_fail(TQ_ERR_UNSUPPORTED, "tq_attend: d = %d above 256", kc->p.d);
  if ((st = check_dtype(dt)) != TQ_OK) return st;
  if ((st = check_heads(B, Hq, Hkv, T, "tq_attend")) != TQ_OK) return st;
  if (B == 0) return TQ_OK;
  if (T < 1) return tq_fail(TQ_ERR_INVALID_ARG, "tq_attend: T must be >= 1");
  if (!std::isfinite(scale) || scale < 0) return tq_fail(TQ_ERR_INVALID_ARG, "tq_attend: scale must be finite and >= 0");
  if (!q || !aligned16(q)) return tq_fail(TQ_ERR_INVALID_ARG, "tq_attend: q null or not 16-byte aligned");
  if (!out || !aligned16(out)) return tq_fail(TQ_ERR_INVALID_ARG, "tq_attend: out null or not 16-byte aligned");
  if ((st = check_compressed(kc, K, "K")) != TQ_OK) return st;
  if (!V || !V->codes || !aligned16(V->codes) || !V->norms || !aligned16(V->norms))
    return tq_fail(TQ_ERR_INVALID_ARG, "tq_attend: V.codes / V.norms null or not 16-byte aligned");
  if (vc->p.m > 0) {
    if ((st = check_compressed(vc, V, "V")) != TQ_OK) return st;
    if (vc->p.m > 128)
      return tq_fail(TQ_ERR_UNSUPPORTED, "tq_attend: QJL-corrected values need a value sketch of m <= 128");
  }
  const int nchunk = tq_attend_chunks(B, Hq, Hkv, T, device_sms(kc->device));
  const size_t need = attend_bytes(kc->p, vc->p, B, Hq, nchunk);
  if (!workspace || !aligned16(workspace) || ws_bytes < need)
    return tq_fail(TQ_ERR_INVALID_ARG, "tq_attend: workspace null, misaligned or smaller than %zu bytes", need);
  if (scale == 0.0f) scale = kc->p.inv_sqrt_d;
  const cudaStream_t s = (cudaStream_t)stream;
  float* qprep = (float*)workspace;
  float* partials = (float*)((char*)workspace + qprep_bytes(kc->p, B * Hq));
  cudaError_t e = tq_launch_qprep(kc->p, q, dt, B * Hq, qprep, s);
  if (e == cudaSuccess)
    e = tq_launch_attend(kc->p, vc->p, qprep, B, Hq, Hkv, T, scale, *K, *V, partials, nchunk, out, s);
  if (e == cudaErrorNotSupported)
    return tq_fail(TQ_ERR_UNSUPPORTED, "tq_attend: no kernel for this key layout with QJL-corrected values");
  return launch_status(e, "tq_attend launch");
}

// ---------------------------------------------------------------- search
static tq_status check_search_codec(const tq_codec* c, const char* name) {
  if (c->p.nseg != 1) return tq_fail(TQ_ERR_UNSUPPORTED, "%s: needs one segment (nseg = %d)", name, c->p.nseg);
  if (c->p.vq_bits) return tq_fail(TQ_ERR_UNSUPPORTED, "%s: needs scalar codes (the codec has FibQuant codes)", name);
  if (c->p.d % 32 != 0 || c->p.d < 64 || c->p.d > 2048)
    return tq_fail(TQ_ERR_UNSUPPORTED, "%s: d = %d (needs a multiple of 32 in [64, 2048])", name, c->p.d);
  if (c->p.m > 512) return tq_fail(TQ_ERR_UNSUPPORTED, "%s: m = %d above 512", name, c->p.m);
  return TQ_OK;
}

extern "C" tq_status tq_search_workspace_size(const tq_codec* c, int nq, int k, size_t* bytes) {
  if (!c || !bytes) return tq_fail(TQ_ERR_INVALID_ARG, "tq_search_workspace_size: null argument");
  if (nq < 0 || k < 1 || k > 32) return tq_fail(TQ_ERR_INVALID_ARG, "tq_search_workspace_size: nq = %d, k = %d", nq, k);
  tq_status st = check_search_codec(c, "tq_search_workspace_size");
  if (st != TQ_OK) return st;
  *bytes = tq_search_bytes(c->p, nq > 0 ? nq : 1, k, device_sms(c->device < 0 ? 0 : c->device));
  return TQ_OK;
}

extern "C" tq_status tq_search_topk(const tq_codec* c, const void* q, tq_dtype dt, int nq, const tq_compressed* X,
                                    int64_t n, int k, int32_t* idx, float* score, void* workspace, size_t ws_bytes,
                                    void* stream) {
  const tqtrace::Range trace("tq_search_topk");
  tq_status st = check_device_codec(c, "tq_search_topk");
  if (st != TQ_OK) return st;
  if ((st = check_search_codec(c, "tq_search_topk")) != TQ_OK) return st;
  if ((st = check_dtype(dt)) != TQ_OK) return st;
  if (nq < 0) return tq_fail(TQ_ERR_INVALID_ARG, "tq_search_topk: nq = %d", nq);
  if (k < 1 || k > 32) return tq_fail(TQ_ERR_INVALID_ARG, "tq_search_topk: k = %d outside [1, 32]", k);
  if (n < k || n >= ((int64_t)1 << 31))
    return tq_fail(TQ_ERR_INVALID_ARG, "tq_search_topk: n = %lld (needs k <= n < 2^31)", (long long)n);
  if (nq == 0) return TQ_OK;
  if (!q || !aligned16(q)) return tq_fail(TQ_ERR_INVALID_ARG, "tq_search_topk: q null or not 16-byte aligned");
  if (!idx || !score) return tq_fail(TQ_ERR_INVALID_ARG, "tq_search_topk: idx / score null");
  if ((st = check_compressed(c, X, "index")) != TQ_OK) return st;
  const size_t need = tq_search_bytes(c->p, nq, k, device_sms(c->device));
  if (!workspace || ((uintptr_t)workspace & 255u) != 0 || ws_bytes < need)
    return tq_fail(TQ_ERR_INVALID_ARG, "tq_search_topk: workspace null, not 256-byte aligned or smaller than %zu bytes",
                   need);
  const cudaStream_t s = (cudaStream_t)stream;
  const int nb = tq_search_batch(nq, k);
  const size_t esz = dtype_size(dt);
  for (int q0 = 0; q0 < nq; q0 += nb) {
    const int cnt = std::min(nb, nq - q0);
    cudaError_t e = tq_launch_qprep(c->p, (const char*)q + (size_t)q0 * c->p.d * esz, dt, cnt, (float*)workspace, s);
    if (e == cudaSuccess) e = tq_launch_search(c->p, (const float*)workspace, cnt, q0, *X, n, k, idx, score, workspace, s);
    if (e != cudaSuccess) return launch_status(e, "tq_search_topk launch");
  }
  return TQ_OK;
}

extern "C" tq_status tq_codec_device_error(const tq_codec* c, void* stream, uint32_t* code) {
  tq_status st = check_device_codec(c, "tq_codec_device_error");
  if (st != TQ_OK) return st;
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "tq_codec_device_error: stream sync");
  uint32_t v = 0;
  e = cudaMemcpy(&v, c->p.err, sizeof v, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "tq_codec_device_error: read");
  if (v != 0) {
    const uint32_t zero = 0;
    e = cudaMemcpy(c->p.err, &zero, sizeof zero, cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_fail(e, "tq_codec_device_error: clear");
  }
  if (code) *code = v;
  if (v != 0) return tq_fail(TQ_ERR_DEVICE_ASSERT, "device error code %u (a bounded wait timed out)", v);
  return TQ_OK;
}

extern "C" tq_status tq_codec_exact_rows(const tq_codec* c, void* stream, int reset, uint64_t* rows) {
  tq_status st = check_device_codec(c, "tq_codec_exact_rows");
  if (st != TQ_OK) return st;
  if (!rows) return tq_fail(TQ_ERR_INVALID_ARG, "tq_codec_exact_rows: null output");
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e == cudaSuccess) e = cudaMemcpy(rows, c->p.exact_rows, sizeof(uint64_t), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess && reset) e = cudaMemset(c->p.exact_rows, 0, sizeof(uint64_t));
  if (e != cudaSuccess) return cuda_fail(e, "tq_codec_exact_rows");
  return TQ_OK;
}
