// Host side of libtq: the quantizer's random draws, Lloyd-Max codebook,
// Haar rotation, and the set-up / inspection entry points of the C ABI.
//
// Method sources (intelliparadigm.com page "TurboQuant 技术概览与核心价值",
// called "TurboQuant article" below):
//   1.2.1 random rotation by QR of a Gaussian matrix; 2.1.2 three rounds of
//   +-1 diagonal and fast Walsh-Hadamard transform; 1.2.2 and 2.2.1-2.2.2
//   Lloyd-Max quantizer on the Beta((d-1)/2,(d-1)/2) coordinate law,
//   precomputed per dimension; 2.3.2 Gaussian QJL projection.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <limits>
#include <new>
#include <thread>
#include <vector>

#include "tq_internal.h"

namespace tq {
namespace {

// ----------------------------------------------------------------- RNG
// SplitMix64 (Steele, Lea, Flood, OOPSLA 2014): output k of the generator
// started from `state` is mix(state + (k+1) * golden_gamma).  A stream of the
// quantizer is keyed by output `stream` of the generator started from seed.
constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;

inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}
inline uint64_t sm64(uint64_t state, uint64_t k) { return mix64(state + (k + 1) * kGamma); }
inline uint64_t stream_key(uint64_t seed, int stream) { return sm64(seed, (uint64_t)stream); }

enum { kStreamD1 = 0, kStreamD2 = 1, kStreamD3 = 2, kStreamS = 3, kStreamHaar = 4 };

// Box-Muller, cosine branch: N(0,1) draw i from words 2i and 2i+1.
inline double gaussian(uint64_t key, uint64_t i) {
  const double u1 = ((double)(sm64(key, 2 * i) >> 11) + 1.0) * 0x1.0p-53;
  const double u2 = (double)(sm64(key, 2 * i + 1) >> 11) * 0x1.0p-53;
  return std::sqrt(-2.0 * std::log(u1)) * std::cos(2.0 * M_PI * u2);
}

// ----------------------------------------------------------------- Lloyd-Max
// Coordinate density f(x) ~ (1-x^2)^((d-3)/2) on [-1,1].  With x = sin(t) the
// bin integrals become integrals of cos(t)^(d-2), smooth on [-pi/2, pi/2],
// which composite Gauss-Legendre handles to full double precision.  The
// first moment has the closed form
//   int_lo^hi x (1-x^2)^((d-3)/2) dx = [(1-lo^2)^((d-1)/2) - (1-hi^2)^((d-1)/2)] / (d-1).
struct GaussLegendre {
  std::vector<double> x, w;
  explicit GaussLegendre(int n) : x(n), w(n) {
    for (int i = 0; i < n; ++i) {
      double z = std::cos(M_PI * (i + 0.75) / (n + 0.5));
      double dp = 0.0;
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
        if (std::fabs(dz) < 1e-16) break;
      }
      x[i] = z;
      w[i] = 2.0 / ((1.0 - z * z) * dp * dp);
    }
  }
};

class CoordLaw {
 public:
  explicit CoordLaw(int d) : d_(d), gl_(24) {
    // Beyond |t| = tcut the integrand is below exp(-700) of its peak.
    const double e = d - 2.0;
    tcut_ = e > 0 ? std::min(M_PI / 2, std::acos(std::exp(-700.0 / e))) : M_PI / 2;
    h_ = std::min(0.25, 0.2 / std::sqrt((double)d));
  }
  // integral of cos(t)^(d-2) over [asin(lo), asin(hi)]
  double mass(double lo, double hi) const {
    double a = std::max(std::asin(std::clamp(lo, -1.0, 1.0)), -tcut_);
    double b = std::min(std::asin(std::clamp(hi, -1.0, 1.0)), tcut_);
    if (!(b > a)) return 0.0;
    int panels = (int)std::ceil((b - a) / h_);
    panels = std::max(1, std::min(panels, 1 << 16));
    const double ph = (b - a) / panels;
    double total = 0.0;
    for (int p = 0; p < panels; ++p) {
      const double c = a + (p + 0.5) * ph, r = 0.5 * ph;
      double s = 0.0;
      for (size_t i = 0; i < gl_.x.size(); ++i) {
        const double t = c + r * gl_.x[i];
        s += gl_.w[i] * std::exp((d_ - 2.0) * std::log(std::cos(t)));
      }
      total += s * r;
    }
    return total;
  }
  double first_moment(double lo, double hi) const {
    auto g = [&](double x) {
      if (std::fabs(x) >= 1.0) return 0.0;
      return std::exp(0.5 * (d_ - 1.0) * std::log1p(-x * x));
    };
    return (g(lo) - g(hi)) / (d_ - 1.0);
  }
  double cdf(double x) const { return mass(-1.0, x) / total(); }
  double total() const {
    if (total_ < 0) total_ = mass(-1.0, 1.0);
    return total_;
  }

 private:
  int d_;
  GaussLegendre gl_;
  double tcut_, h_;
  mutable double total_ = -1.0;
};

void lloyd_max(int d, int w, std::vector<double> &cen, std::vector<double> &thr, double &mse) {
  const int L = 1 << w;
  CoordLaw law(d);
  thr.assign(L - 1, 0.0);
  for (int i = 1; i < L; ++i) {  // equal-probability start: quantiles i/L
    const double q = (double)i / L;
    double lo = -1.0, hi = 1.0;
    for (int it = 0; it < 200 && hi - lo > 1e-17; ++it) {
      const double mid = 0.5 * (lo + hi);
      (law.cdf(mid) < q ? lo : hi) = mid;
    }
    thr[i - 1] = 0.5 * (lo + hi);
  }
  cen.assign(L, 0.0);
  std::vector<double> nc(L), edges(L + 1);
  for (int it = 0; it < 100000; ++it) {
    edges[0] = -1.0;
    edges[L] = 1.0;
    for (int i = 0; i < L - 1; ++i) edges[i + 1] = thr[i];
    for (int i = 0; i < L; ++i)
      nc[i] = law.first_moment(edges[i], edges[i + 1]) / law.mass(edges[i], edges[i + 1]);
    std::vector<double> sym(L);
    for (int i = 0; i < L; ++i) sym[i] = 0.5 * (nc[i] - nc[L - 1 - i]);
    double step = 0.0, big = 0.0;
    for (int i = 0; i < L; ++i) {
      step = std::max(step, std::fabs(sym[i] - cen[i]));
      big = std::max(big, std::fabs(sym[i]));
    }
    cen = sym;
    for (int i = 0; i < L - 1; ++i) thr[i] = 0.5 * (cen[i] + cen[i + 1]);
    if (step <= 1e-14 * big) break;
  }
  edges[0] = -1.0;
  edges[L] = 1.0;
  for (int i = 0; i < L - 1; ++i) edges[i + 1] = thr[i];
  double acc = 0.0, z = law.total();
  for (int i = 0; i < L; ++i) acc += cen[i] * cen[i] * law.mass(edges[i], edges[i + 1]) / z;
  mse = 1.0 / d - acc;
}

// ----------------------------------------------------------------- Haar
// Q of the QR factorization of a Gaussian matrix G (Householder reflections,
// column-major work array), with columns multiplied by sign(diag(R)) so that
// Q is Haar distributed.  Returned row-major.
void haar(int d, uint64_t seed, std::vector<double> &q_out) {
  const uint64_t key = stream_key(seed, kStreamHaar);
  std::vector<double> a((size_t)d * d);  // column-major: a[j*d + i] = G[i][j]
  for (int i = 0; i < d; ++i)
    for (int j = 0; j < d; ++j) a[(size_t)j * d + i] = gaussian(key, (uint64_t)i * d + j);
  std::vector<double> vs((size_t)d * d, 0.0);  // reflector j in column j, rows j..d-1
  std::vector<double> rdiag(d);
  const unsigned hw = std::max(1u, std::min(16u, std::thread::hardware_concurrency()));

  auto parallel_cols = [&](int c0, int c1, auto &&fn) {
    const int cols = c1 - c0;
    if (cols <= 0) return;
    const int nt = (int)std::min<unsigned>(hw, (unsigned)std::max(1, cols / 32));
    if (nt <= 1) {
      for (int c = c0; c < c1; ++c) fn(c);
      return;
    }
    std::vector<std::thread> th;
    for (int t = 0; t < nt; ++t)
      th.emplace_back([&, t] {
        for (int c = c0 + t; c < c1; c += nt) fn(c);
      });
    for (auto &x : th) x.join();
  };

  for (int j = 0; j < d; ++j) {
    double *col = &a[(size_t)j * d];
    double nrm = 0.0;
    for (int i = j; i < d; ++i) nrm += col[i] * col[i];
    nrm = std::sqrt(nrm);
    const double alpha = col[j] >= 0 ? -nrm : nrm;
    double *v = &vs[(size_t)j * d];
    for (int i = j; i < d; ++i) v[i] = col[i];
    v[j] -= alpha;
    double vn = 0.0;
    for (int i = j; i < d; ++i) vn += v[i] * v[i];
    vn = std::sqrt(vn);
    if (vn > 0)
      for (int i = j; i < d; ++i) v[i] /= vn;
    rdiag[j] = alpha;
    parallel_cols(j + 1, d, [&](int c) {
      double *y = &a[(size_t)c * d];
      double s = 0.0;
      for (int i = j; i < d; ++i) s += v[i] * y[i];
      s *= 2.0;
      for (int i = j; i < d; ++i) y[i] -= s * v[i];
    });
  }
  // Q = H_0 H_1 ... H_{d-1}: apply the reflectors to the identity, last first.
  std::vector<double> q((size_t)d * d, 0.0);  // column-major
  for (int i = 0; i < d; ++i) q[(size_t)i * d + i] = 1.0;
  for (int j = d - 1; j >= 0; --j) {
    const double *v = &vs[(size_t)j * d];
    parallel_cols(0, d, [&](int c) {
      double *y = &q[(size_t)c * d];
      double s = 0.0;
      for (int i = j; i < d; ++i) s += v[i] * y[i];
      s *= 2.0;
      for (int i = j; i < d; ++i) y[i] -= s * v[i];
    });
  }
  q_out.assign((size_t)d * d, 0.0);
  for (int c = 0; c < d; ++c) {
    const double sg = rdiag[c] < 0 ? -1.0 : 1.0;
    for (int i = 0; i < d; ++i) q_out[(size_t)i * d + c] = q[(size_t)c * d + i] * sg;
  }
}

bool is_pow2(int d) { return d > 0 && (d & (d - 1)) == 0; }

template <class T>
tq_status upload(T **dst, const T *src, size_t count) {
  if (cudaMalloc((void **)dst, count * sizeof(T)) != cudaSuccess) {
    cudaGetLastError();
    *dst = nullptr;
    return TQ_ERR_NOMEM;
  }
  if (cudaMemcpy(*dst, src, count * sizeof(T), cudaMemcpyHostToDevice) != cudaSuccess) {
    cudaGetLastError();
    return TQ_ERR_CUDA;
  }
  return TQ_OK;
}

// v as 31-bit fixed point under one power-of-two scale 2^e (|v| 2^e < 2^30),
// split into four signed-byte planes: round(v 2^e) = 2^24 a + 2^16 b +
// 2^8 c + d with b, c, d in [-128, 127] and |a| <= 64.
std::vector<int8_t> limb_split(const std::vector<double> &v, int *e_out) {
  double big = 0.0;
  for (double x : v) big = std::max(big, std::fabs(x));
  int E = 0;
  std::frexp(big, &E);  // big < 2^E
  const int e = big > 0.0 ? 30 - E : 0;
  const size_t n = v.size();
  std::vector<int8_t> out(4 * n);
  for (size_t i = 0; i < n; ++i) {
    long t = std::lrint(std::ldexp(v[i], e));
    for (int l = 3; l >= 1; --l) {  // low limbs, balanced
      const long lo = ((t + 128) & 255) - 128;
      out[(size_t)l * n + i] = (int8_t)lo;
      t = (t - lo) / 256;
    }
    out[i] = (int8_t)t;
  }
  *e_out = e;
  return out;
}

void free_device(tq_quantizer *q) {
  cudaFree(q->d_rot_limbs);
  cudaFree(q->d_qjl_limbs);
  q->d_rot_limbs = nullptr;
  q->d_qjl_limbs = nullptr;
  cudaFree(q->d_rot16);
  cudaFree(q->d_rot_bf16);
  cudaFree(q->d_rot_bf16x3);
  q->d_rot_bf16x3 = nullptr;
  cudaFree(q->d_err);
  q->d_rot16 = nullptr;
  q->d_rot_bf16 = nullptr;
  q->d_err = nullptr;
  cudaFree(q->d_diag_bits);
  cudaFree(q->d_rot);
  cudaFree(q->d_qjl16);
  cudaFree(q->d_qjl32);
  cudaFree(q->d_qjl32t);
  q->d_qjl32t = nullptr;
  cudaFree(q->d_rott);
  q->d_rott = nullptr;
  q->d_diag_bits = nullptr;
  q->d_rot = nullptr;
  q->d_qjl16 = nullptr;
  q->d_qjl32 = nullptr;
}

}  // namespace

// Round a double to the nearest IEEE binary16 value (ties to even), directly
// from double (no intermediate float rounding).
uint16_t double_to_half_bits(double v) {
  uint16_t sign = std::signbit(v) ? 0x8000 : 0;
  double a = std::fabs(v);
  if (std::isnan(a)) return sign | 0x7e00;
  if (a >= 65520.0) return sign | 0x7c00;  // at or beyond the rounding edge of 65504
  int e;
  std::frexp(a, &e);  // a = f * 2^e, f in [0.5, 1)
  e -= 1;             // a = g * 2^e, g in [1, 2)
  if (a == 0.0) return sign;
  if (e < -14) {  // subnormal range: units of 2^-24
    double m = std::nearbyint(std::ldexp(a, 24));
    return sign | (uint16_t)m;  // m == 1024 encodes the smallest normal
  }
  double m = std::nearbyint(std::ldexp(a, 10 - e));  // in [1024, 2048]
  if (m >= 2048.0) {
    m = 1024.0;
    e += 1;
  }
  if (e > 15) return sign | 0x7c00;
  return sign | (uint16_t)(((e + 15) << 10) | ((int)m - 1024));
}

double half_bits_to_double(uint16_t h) {
  const double s = (h & 0x8000) ? -1.0 : 1.0;
  const int e = (h >> 10) & 0x1f, m = h & 0x3ff;
  if (e == 0) return s * std::ldexp((double)m, -24);
  if (e == 31) return m ? std::numeric_limits<double>::quiet_NaN() : s * INFINITY;
  return s * std::ldexp(1024.0 + m, e - 25);
}

}  // namespace tq

extern "C" {

const char *tq_status_string(tq_status s) {
  switch (s) {
    case TQ_OK: return "ok";
    case TQ_ERR_INVALID_ARG: return "invalid argument";
    case TQ_ERR_UNSUPPORTED: return "unsupported configuration";
    case TQ_ERR_ALIGNMENT: return "misaligned pointer or leading dimension";
    case TQ_ERR_NOMEM: return "out of memory";
    case TQ_ERR_CUDA: return "CUDA error";
    case TQ_ERR_WORKSPACE: return "workspace missing or too small";
    case TQ_ERR_TOO_LARGE: return "request exceeds the fixed internal scratch buffer";
    case TQ_ERR_TIMEOUT: return "a kernel gave up a bounded wait; the outputs of that call are not valid";
  }
  return "unknown status";
}

// mse: TurboQuant-MSE (all b bits to the codebook, no QJL stage, m = 0);
// otherwise b - 1 codebook bits and an m-row QJL sketch.
static tq_status build_quantizer(int d, int b, int m, uint64_t seed, tq_rotation rot, bool device, bool mse,
                                 tq_quantizer **out) {
  using namespace tq;
  if (!out) return TQ_ERR_INVALID_ARG;
  *out = nullptr;
  if (mse) {
    if (d <= 0 || b < 1 || b > 4 || (rot != TQ_ROT_AUTO && rot != TQ_ROT_HADAMARD && rot != TQ_ROT_HAAR))
      return TQ_ERR_INVALID_ARG;
    m = 0;
  } else {
    if (m == 0) m = d;
    if (d <= 0 || b < 2 || b > 5 || m <= 0 || (rot != TQ_ROT_AUTO && rot != TQ_ROT_HADAMARD && rot != TQ_ROT_HAAR))
      return TQ_ERR_INVALID_ARG;
    if (m != d) return TQ_ERR_UNSUPPORTED;
  }
  if (d % 32 != 0 || d > 4096) return TQ_ERR_UNSUPPORTED;
  if (rot == TQ_ROT_AUTO) rot = is_pow2(d) ? TQ_ROT_HADAMARD : TQ_ROT_HAAR;
  if (rot == TQ_ROT_HADAMARD && !is_pow2(d)) return TQ_ERR_UNSUPPORTED;

  tq_quantizer *q = new (std::nothrow) tq_quantizer();
  if (!q) return TQ_ERR_NOMEM;
  q->d = d;
  q->b = b;
  q->w = mse ? b : b - 1;
  q->m = m;
  q->rotation = rot;
  q->seed = seed;
  q->device = -1;
  if (device && cudaGetDevice(&q->device) != cudaSuccess) {
    cudaGetLastError();
    delete q;
    return TQ_ERR_CUDA;
  }
  lloyd_max(d, q->w, q->centroids, q->thresholds, q->coord_mse);

  // rotation
  q->rot.assign((size_t)d * d, 0.0f);
  if (rot == TQ_ROT_HADAMARD) {
    q->diag.resize(3 * (size_t)d);
    for (int r = 0; r < 3; ++r) {
      const uint64_t key = stream_key(seed, kStreamD1 + r);
      for (int j = 0; j < d; ++j) q->diag[(size_t)r * d + j] = (sm64(key, j) & 1) ? -1 : 1;
    }
    // dense R = H D3 H D2 H D1 in double (column j = R e_j by fast
    // Walsh-Hadamard butterflies), for inspection and for the dense path
    std::vector<double> cur((size_t)d * d, 0.0), col(d);
    const double s = 1.0 / std::sqrt((double)d);
    for (int j = 0; j < d; ++j) {
      std::fill(col.begin(), col.end(), 0.0);
      col[j] = 1.0;
      for (int r = 0; r < 3; ++r) {
        for (int i = 0; i < d; ++i) col[i] *= q->diag[(size_t)r * d + i];
        for (int h = 1; h < d; h <<= 1)
          for (int i = 0; i < d; i += 2 * h)
            for (int k = i; k < i + h; ++k) {
              const double a = col[k], c = col[k + h];
              col[k] = a + c;
              col[k + h] = a - c;
            }
        for (int i = 0; i < d; ++i) col[i] *= s;
      }
      for (int i = 0; i < d; ++i) cur[(size_t)i * d + j] = col[i];
    }
    for (size_t i = 0; i < cur.size(); ++i) q->rot[i] = (float)cur[i];
    q->rot_exact = cur;
  } else {
    std::vector<double> h;
    haar(d, seed, h);
    for (size_t i = 0; i < h.size(); ++i) q->rot[i] = (float)h[i];
  }
  // QJL projection S, fp16-rounded Gaussians
  q->qjl16.resize((size_t)m * d);
  std::vector<float> s32((size_t)m * d);
  {
    const uint64_t key = stream_key(seed, kStreamS);
    for (size_t i = 0; i < q->qjl16.size(); ++i) {
      q->qjl16[i] = double_to_half_bits(gaussian(key, i));
      s32[i] = (float)half_bits_to_double(q->qjl16[i]);
    }
  }

  tq_status st = TQ_OK;
  if (!device) {
    *out = q;
    return TQ_OK;
  }
  if (rot == TQ_ROT_HADAMARD) {
    std::vector<uint32_t> bits(3 * (size_t)d / 32, 0u);
    for (int r = 0; r < 3; ++r)
      for (int j = 0; j < d; ++j)
        if (q->diag[(size_t)r * d + j] < 0) bits[((size_t)r * d + j) / 32] |= 1u << (j % 32);
    st = upload(&q->d_diag_bits, bits.data(), bits.size());
  }
  if (st == TQ_OK) st = upload(&q->d_rot, q->rot.data(), q->rot.size());
  if (st == TQ_OK && m > 0) st = upload(&q->d_qjl16, q->qjl16.data(), q->qjl16.size());
  if (st == TQ_OK && m > 0) st = upload(&q->d_qjl32, s32.data(), s32.size());
  if (st == TQ_OK && m > 0) {
    std::vector<float> st32((size_t)m * d);
    for (int i = 0; i < m; ++i)
      for (int j = 0; j < d; ++j) st32[(size_t)j * m + i] = s32[(size_t)i * d + j];
    st = upload(&q->d_qjl32t, st32.data(), st32.size());
  }
  if (st == TQ_OK && d <= 128) {
    std::vector<float> rt((size_t)d * d);
    for (int i = 0; i < d; ++i)
      for (int j = 0; j < d; ++j) rt[(size_t)j * d + i] = q->rot[(size_t)i * d + j];
    st = upload(&q->d_rott, rt.data(), rt.size());
  }
  if (st == TQ_OK) {
    // Rotation as fp16 pieces for the tensor-core encode.  Hadamard: d^1.5 R
    // is an integer matrix (exact in fp16 when every |entry| <= 2048, else
    // split into two exact pieces).  Haar: R * 2^8 split into hi + lo fp16.
    std::vector<uint16_t> pieces;
    const size_t dd = (size_t)d * d;
    if (rot == TQ_ROT_HADAMARD) {
      const double s15 = std::pow((double)d, 1.5);
      double big = 0.0;
      std::vector<double> kmat(dd);
      for (size_t i = 0; i < dd; ++i) {
        kmat[i] = std::nearbyint((double)q->rot_exact[i] * s15);
        big = std::max(big, std::fabs(kmat[i]));
      }
      q->tc_rho = (float)(1.0 / s15);
      q->tc_rot_pieces = big <= 2048.0 ? 1 : 2;
      pieces.resize(q->tc_rot_pieces * dd);
      for (size_t i = 0; i < dd; ++i) {
        const uint16_t h = double_to_half_bits(kmat[i]);
        pieces[i] = h;
        if (q->tc_rot_pieces == 2) pieces[dd + i] = double_to_half_bits(kmat[i] - half_bits_to_double(h));
      }
      if (big <= 2048.0) {
        // the same integer matrix as two bf16 pieces (8 + 8 significant bits
        // cover integers up to 2^11 exactly), for MMAs that read bf16 keys as-is
        std::vector<uint16_t> bfp(2 * dd);
        auto to_bf16 = [](double v) {
          float f = (float)v;  // exact: an integer below 2^24
          uint32_t b;
          std::memcpy(&b, &f, 4);
          b += 0x7FFFu + ((b >> 16) & 1u);
          return (uint16_t)(b >> 16);
        };
        auto from_bf16 = [](uint16_t h) {
          uint32_t b = (uint32_t)h << 16;
          float f;
          std::memcpy(&f, &b, 4);
          return (double)f;
        };
        for (size_t i = 0; i < dd; ++i) {
          const uint16_t h = to_bf16(kmat[i]);
          bfp[i] = h;
          bfp[dd + i] = to_bf16(kmat[i] - from_bf16(h));
        }
        st = upload(&q->d_rot_bf16, bfp.data(), bfp.size());
      }
    } else {
      if (d <= 128) {
        // the fp32 R as three bf16 pieces (8 + 8 + 8 significant bits: exact),
        // for the gathered tensor-core encode of bf16 keys
        std::vector<uint16_t> b3(3 * dd);
        auto bf = [](float f) {
          uint32_t b;
          std::memcpy(&b, &f, 4);
          b += 0x7FFFu + ((b >> 16) & 1u);
          return (uint16_t)(b >> 16);
        };
        auto fb = [](uint16_t h) {
          uint32_t b = (uint32_t)h << 16;
          float f;
          std::memcpy(&f, &b, 4);
          return f;
        };
        for (size_t i = 0; i < dd; ++i) {
          const float r0 = q->rot[i];
          const uint16_t h0 = bf(r0);
          const float r1 = r0 - fb(h0);  // exact: fewer significant bits than r0
          const uint16_t h1 = bf(r1);
          const float r2 = r1 - fb(h1);
          b3[i] = h0;
          b3[dd + i] = h1;
          b3[2 * dd + i] = bf(r2);
        }
        st = upload(&q->d_rot_bf16x3, b3.data(), b3.size());
      }
      q->tc_rho = 1.0f / 256.0f;
      q->tc_rot_pieces = 2;
      pieces.resize(2 * dd);
      for (size_t i = 0; i < dd; ++i) {
        const double v = (double)q->rot[i] * 256.0;
        const uint16_t h = double_to_half_bits(v);
        pieces[i] = h;
        pieces[dd + i] = double_to_half_bits(v - half_bits_to_double(h));
      }
    }
    if (st == TQ_OK) st = upload(&q->d_rot16, pieces.data(), pieces.size());
  }
  if (st == TQ_OK && d >= 256) {
    // fixed-point limbs of R and S for the dense tensor-core encode
    const size_t dd = (size_t)d * d;
    std::vector<double> rv(dd), sv((size_t)m * d);
    for (size_t i = 0; i < dd; ++i) rv[i] = rot == TQ_ROT_HADAMARD ? q->rot_exact[i] : (double)q->rot[i];
    for (size_t i = 0; i < sv.size(); ++i) sv[i] = half_bits_to_double(q->qjl16[i]);
    const std::vector<int8_t> rl = limb_split(rv, &q->rot_limb_exp);
    st = upload(&q->d_rot_limbs, rl.data(), rl.size());
    if (st == TQ_OK && m > 0) {
      const std::vector<int8_t> sl = limb_split(sv, &q->qjl_limb_exp);
      st = upload(&q->d_qjl_limbs, sl.data(), sl.size());
    }
  }
  if (st == TQ_OK) {
    if (cudaMalloc((void **)&q->d_err, sizeof(int)) != cudaSuccess || cudaMemset(q->d_err, 0, sizeof(int)) != cudaSuccess) {
      cudaGetLastError();
      st = TQ_ERR_NOMEM;
    }
  }
  if (st != TQ_OK) {
    free_device(q);
    delete q;
    return st;
  }

  {
    // centroids as 16-bit fixed point split into two signed bytes (integer scorer)
    double big = 0.0;
    for (double c : q->centroids) big = std::max(big, std::fabs(c));
    int e = 0;
    std::frexp(big, &e);  // big < 2^e
    q->score_cexp = 14 - e;  // |c| * 2^cexp < 2^14: the limbs stay within int8
    const int L = 1 << q->w;
    for (int k = 0; k < L; ++k) {
      const long v = std::lrint(std::ldexp(q->centroids[k], q->score_cexp));
      const long hi = (v + 128) >> 8;  // floor((v + 128) / 256)
      q->score_ch[k] = (int8_t)hi;
      q->score_cl[k] = (int8_t)(v - 256 * hi);
    }
  }
  KernelTables &kt = q->kt;
  kt.d = d;
  kt.w = q->w;
  kt.m = m;
  kt.levels = 1 << q->w;
  for (int i = 0; i < kMaxLevels; ++i) {
    kt.centroids[i] = i < kt.levels ? (float)q->centroids[i] : 0.0f;
    kt.thresholds[i] = i < kt.levels - 1 ? (float)q->thresholds[i] : INFINITY;
  }
  kt.qjl_scale = m > 0 ? (float)(std::sqrt(M_PI / 2.0) / m) : 0.0f;  // no QJL term in TurboQuant-MSE
  kt.diag_bits = q->d_diag_bits;
  kt.rot = q->d_rot;
  kt.qjl16 = q->d_qjl16;
  kt.qjl32 = q->d_qjl32;
  kt.qjl32t = q->d_qjl32t;
  kt.rott = q->d_rott;
  kt.qjl_key = stream_key(seed, kStreamS);
  kt.qjl_otf = 0;
  *out = q;
  return TQ_OK;
}

tq_status tq_codebook(int d, int b, int m, uint64_t seed, tq_rotation rot, tq_quantizer **out) {
  return build_quantizer(d, b, m, seed, rot, true, false, out);
}

tq_status tq_codebook_host(int d, int b, int m, uint64_t seed, tq_rotation rot, tq_quantizer **out) {
  return build_quantizer(d, b, m, seed, rot, false, false, out);
}

tq_status tq_codebook_mse(int d, int b, uint64_t seed, tq_rotation rot, tq_quantizer **out) {
  return build_quantizer(d, b, 0, seed, rot, true, true, out);
}

tq_status tq_codebook_mse_host(int d, int b, uint64_t seed, tq_rotation rot, tq_quantizer **out) {
  return build_quantizer(d, b, 0, seed, rot, false, true, out);
}

void tq_destroy(tq_quantizer *q) {
  if (!q) return;
  if (q->device < 0) {
    delete q;
    return;
  }
  int cur = 0;
  cudaGetDevice(&cur);
  cudaSetDevice(q->device);
  tq::free_device(q);
  cudaSetDevice(cur);
  delete q;
}

tq_status tq_info(const tq_quantizer *q, tq_info_t *info) {
  if (!q || !info) return TQ_ERR_INVALID_ARG;
  info->d = q->d;
  info->b = q->b;
  info->w = q->w;
  info->m = q->m;
  info->rotation = q->rotation;
  info->device = q->device;
  info->seed = q->seed;
  info->code_bytes = (size_t)q->w * q->d / 8;
  info->sign_bytes = (size_t)q->m / 8;
  info->coord_mse = q->coord_mse;
  return TQ_OK;
}

tq_status tq_codebook_get(const tq_quantizer *q, double *centroids, double *thresholds, double *coord_mse) {
  if (!q) return TQ_ERR_INVALID_ARG;
  if (centroids) std::memcpy(centroids, q->centroids.data(), q->centroids.size() * sizeof(double));
  if (thresholds) std::memcpy(thresholds, q->thresholds.data(), q->thresholds.size() * sizeof(double));
  if (coord_mse) *coord_mse = q->coord_mse;
  return TQ_OK;
}

tq_status tq_tables_get(const tq_quantizer *q, float *rotation, int8_t *diag_signs, uint16_t *qjl) {
  if (!q) return TQ_ERR_INVALID_ARG;
  if (rotation) std::memcpy(rotation, q->rot.data(), q->rot.size() * sizeof(float));
  if (diag_signs && !q->diag.empty()) std::memcpy(diag_signs, q->diag.data(), q->diag.size());
  if (qjl) std::memcpy(qjl, q->qjl16.data(), q->qjl16.size() * sizeof(uint16_t));
  return TQ_OK;
}

}  // extern "C"
