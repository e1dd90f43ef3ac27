// Host-side part of libtq: codebook solver, dense rotation factorization,
// quantizer handles and status strings.
//
// The codebook solver integrates the Lemma 1 density of the TurboQuant notes
// ([2026 ICLR] TurboQuant blog notes, Lemma 1) numerically with composite
// Gauss-Legendre quadrature and runs the Lloyd-Max iteration of eq. (4)
// (TurboQuant explainer §5: boundaries at midpoints, centroids at conditional
// means, repeat until stable).
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include "tq_gemm_tc.h"
#include "tq_internal.h"

namespace tq {
namespace {

// ---------------------------------------------------------------- quadrature

struct GaussLegendre {
  static constexpr int kN = 16;
  double x[kN];
  double w[kN];
  GaussLegendre() {
    // Nodes are the roots of P_n, found by Newton's method from the
    // Chebyshev-like starting guesses cos(pi (i + 3/4) / (n + 1/2)); the
    // weights are 2 / ((1 - x^2) P_n'(x)^2).
    const int n = kN;
    for (int i = 0; i < n; ++i) {
      double z = std::cos(M_PI * (i + 0.75) / (n + 0.5));
      double dp = 0.0;
      for (int it = 0; it < 100; ++it) {
        double p0 = 1.0, p1 = 0.0;
        for (int j = 1; j <= n; ++j) {
          double p2 = p1;
          p1 = p0;
          p0 = ((2.0 * j - 1.0) * z * p1 - (j - 1.0) * p2) / j;
        }
        dp = n * (z * p0 - p1) / (z * z - 1.0);
        double dz = p0 / dp;
        z -= dz;
        if (std::fabs(dz) < 1e-16) break;
      }
      x[i] = z;
      w[i] = 2.0 / ((1.0 - z * z) * dp * dp);
    }
  }
};

const GaussLegendre& gl() {
  static GaussLegendre g;
  return g;
}

struct Density {
  double d;
  double logk;
  double half_exp;  // (d - 3) / 2
  explicit Density(int dim)
      : d(dim),
        logk(std::lgamma(dim / 2.0) - 0.5 * std::log(M_PI) - std::lgamma((dim - 1) / 2.0)),
        half_exp((dim - 3) / 2.0) {}
  double operator()(double x) const {
    if (x <= -1.0 || x >= 1.0) return 0.0;
    return std::exp(logk + half_exp * std::log1p(-x * x));
  }
};

// Integrals of f and x f over [a, b] by composite Gauss-Legendre.
void cell_integrals(const Density& f, double a, double b, int panels, double* m0, double* m1) {
  const GaussLegendre& g = gl();
  double s0 = 0.0, s1 = 0.0;
  const double h = (b - a) / panels;
  for (int p = 0; p < panels; ++p) {
    const double lo = a + p * h;
    const double mid = lo + 0.5 * h, half = 0.5 * h;
    for (int i = 0; i < GaussLegendre::kN; ++i) {
      const double t = mid + half * g.x[i];
      const double v = g.w[i] * half * f(t);
      s0 += v;
      s1 += v * t;
    }
  }
  *m0 = s0;
  *m1 = s1;
}

}  // namespace

int solve_codebook(int d, int bits, double* c_out, double* b_out) {
  const int n = 1 << bits;
  const Density f(d);
  // Beyond |x| = 16/sqrt(d) the density is below e^-100 of its peak for the
  // dimensions supported here; integrate over that support only.
  const double lim = std::min(1.0, 16.0 / std::sqrt((double)d));
  std::vector<double> c(n), nc(n), bnd(n + 1);
  const double sig = 1.0 / std::sqrt((double)d);
  for (int i = 0; i < n; ++i) c[i] = sig * 2.5 * ((i + 0.5) / n * 2.0 - 1.0);
  bool converged = false;
  for (int it = 0; it < 200000; ++it) {
    bnd[0] = -lim;
    bnd[n] = lim;
    for (int i = 1; i < n; ++i) bnd[i] = 0.5 * (c[i - 1] + c[i]);
    for (int i = 0; i < n; ++i) {
      double m0, m1;
      cell_integrals(f, bnd[i], bnd[i + 1], 24, &m0, &m1);
      nc[i] = m0 > 0 ? m1 / m0 : 0.5 * (bnd[i] + bnd[i + 1]);
    }
    double delta = 0.0, scale = 0.0;
    for (int i = 0; i < n; ++i) {
      const double v = 0.5 * (nc[i] - nc[n - 1 - i]);  // odd symmetry of the codebook
      delta = std::max(delta, std::fabs(v - c[i]));
      scale = std::max(scale, std::fabs(v));
      c[i] = v;
    }
    if (delta <= 1e-15 * scale) {
      converged = true;
      break;
    }
  }
  if (!converged) return 1;
  for (int i = 0; i < n; ++i) c_out[i] = c[i];
  for (int i = 0; i + 1 < n; ++i) b_out[i] = 0.5 * (c[i] + c[i + 1]);
  return 0;
}

// Dense Haar rotation from a Gaussian draw (TurboQuant explainer §3: QR of an
// iid N(0,1) matrix, keep the orthogonal factor).  Householder QR in double;
// Pi = Q diag(sign(diag R)).  G and Pi are row-major d x d.
int householder_rotation(int d, const double* G, double* Pi) {
  // A is stored column-major: A[col][row].
  std::vector<double> A((size_t)d * d);
  for (int r = 0; r < d; ++r)
    for (int c = 0; c < d; ++c) A[(size_t)c * d + r] = G[(size_t)r * d + c];
  std::vector<double> vs((size_t)d * d, 0.0);  // Householder vectors, column k in vs[k]
  std::vector<double> rdiag(d);
  for (int k = 0; k < d; ++k) {
    double* a = &A[(size_t)k * d];
    double nrm = 0.0;
    for (int i = k; i < d; ++i) nrm += a[i] * a[i];
    nrm = std::sqrt(nrm);
    double* v = &vs[(size_t)k * d];
    if (nrm == 0.0) {
      rdiag[k] = 0.0;
      continue;
    }
    const double alpha = a[k] >= 0 ? -nrm : nrm;  // reflect a[k:] onto alpha e_k
    for (int i = k; i < d; ++i) v[i] = a[i];
    v[k] -= alpha;
    double vv = 0.0;
    for (int i = k; i < d; ++i) vv += v[i] * v[i];
    rdiag[k] = alpha;
    if (vv == 0.0) continue;
    const double inv = 2.0 / vv;
    for (int c = k; c < d; ++c) {
      double* ac = &A[(size_t)c * d];
      double dot = 0.0;
      for (int i = k; i < d; ++i) dot += v[i] * ac[i];
      dot *= inv;
      for (int i = k; i < d; ++i) ac[i] -= dot * v[i];
    }
  }
  // Q = H_0 H_1 ... H_{d-1}: apply the reflectors in reverse to the identity,
  // column by column (Q stored column-major in A).
  std::fill(A.begin(), A.end(), 0.0);
  for (int c = 0; c < d; ++c) A[(size_t)c * d + c] = 1.0;
  for (int k = d - 1; k >= 0; --k) {
    const double* v = &vs[(size_t)k * d];
    double vv = 0.0;
    for (int i = k; i < d; ++i) vv += v[i] * v[i];
    if (vv == 0.0) continue;
    const double inv = 2.0 / vv;
    for (int c = 0; c < d; ++c) {
      double* qc = &A[(size_t)c * d];
      double dot = 0.0;
      for (int i = k; i < d; ++i) dot += v[i] * qc[i];
      dot *= inv;
      if (dot != 0.0)
        for (int i = k; i < d; ++i) qc[i] -= dot * v[i];
    }
  }
  for (int r = 0; r < d; ++r)
    for (int c = 0; c < d; ++c) {
      const double s = rdiag[c] < 0 ? -1.0 : 1.0;
      Pi[(size_t)r * d + c] = A[(size_t)c * d + r] * s;
    }
  return 0;
}

}  // namespace tq

// ====================================================================== C ABI

namespace {

bool fp16_exact(float v) {
  // Round-trip through IEEE binary16 on the host (round to nearest even).
  if (v == 0.0f || !std::isfinite(v)) return std::isfinite(v);
  const float a = std::fabs(v);
  if (a > 65504.0f) return false;
  int e;
  std::frexp(a, &e);  // a = f * 2^e, f in [0.5, 1)
  // binary16 has 11 significant bits for normals (e >= -13), fewer below.
  int sig_bits = 11;
  if (e < -13) sig_bits = 11 - (-13 - e);
  if (sig_bits <= 0) return false;
  const double q = std::ldexp(1.0, e - sig_bits);
  const double r = a / q;
  return r == std::floor(r);
}

uint16_t to_half_bits(float v) {
  // exact conversion for fp16-representable v (checked by fp16_exact)
  uint32_t sign = std::signbit(v) ? 0x8000u : 0u;
  float a = std::fabs(v);
  if (a == 0.0f) return (uint16_t)sign;
  int e;
  double f = std::frexp((double)a, &e);  // a = f 2^e, f in [0.5,1)
  int exp16 = e - 1 + 15;               // a = 1.m * 2^(e-1)
  if (exp16 <= 0) {
    // subnormal: a = mant * 2^-24
    uint32_t mant = (uint32_t)std::ldexp((double)a, 24);
    return (uint16_t)(sign | mant);
  }
  uint32_t mant = (uint32_t)((f * 2.0 - 1.0) * 1024.0);
  return (uint16_t)(sign | ((uint32_t)exp16 << 10) | mant);
}

}  // namespace

extern "C" {

const char* tq_status_string(tq_status s) {
  switch (s) {
    case TQ_OK: return "TQ_OK";
    case TQ_ERR_INVALID_ARG: return "TQ_ERR_INVALID_ARG";
    case TQ_ERR_UNSUPPORTED: return "TQ_ERR_UNSUPPORTED";
    case TQ_ERR_CUDA: return "TQ_ERR_CUDA";
    case TQ_ERR_TIMEOUT: return "TQ_ERR_TIMEOUT";
    case TQ_ERR_INTERNAL: return "TQ_ERR_INTERNAL";
    case TQ_ERR_WORKSPACE: return "TQ_ERR_WORKSPACE";
  }
  return "TQ_ERR_UNKNOWN";
}

const char* tq_version(void) { return "libtq 0.1 (sm_100a)"; }

tq_status tq_build_codebook(int d, int bits, float* centroids, float* boundaries) {
  if (!centroids || !boundaries || d < 4 || d > 4096 || bits < 1 || bits > 4)
    return TQ_ERR_INVALID_ARG;
  double c[tq::kMaxLevels], b[tq::kMaxLevels];
  if (tq::solve_codebook(d, bits, c, b) != 0) return TQ_ERR_INTERNAL;
  const int n = 1 << bits;
  for (int i = 0; i < n; ++i) centroids[i] = (float)c[i];
  for (int i = 0; i + 1 < n; ++i) boundaries[i] = (float)b[i];
  return TQ_OK;
}

tq_status tq_make_rotation(int d, const double* G, float* Pi) {
  if (!G || !Pi || d < 1 || d > 4096) return TQ_ERR_INVALID_ARG;
  std::vector<double> pi((size_t)d * d);
  if (tq::householder_rotation(d, G, pi.data()) != 0) return TQ_ERR_INTERNAL;
  for (size_t i = 0; i < pi.size(); ++i) Pi[i] = (float)pi[i];
  return TQ_OK;
}

tq_status tq_params_destroy(tq_params* p) {
  if (!p) return TQ_OK;
  int cur = 0;
  cudaGetDevice(&cur);
  cudaSetDevice(p->device);
  cudaFree(p->dev_S);
  cudaFree(p->dev_St);
  cudaFree(p->dev_S16);
  cudaFree(p->dev_Pi);
  cudaFree(p->dev_Pi2);
  cudaSetDevice(cur);
  std::free(p->host_Pi);
  delete p;
  return TQ_OK;
}

tq_status tq_params_create(int d, int bits, tq_mode mode, tq_rot rot, int m, const int8_t* signs,
                           const float* S, const double* G, tq_params** out) {
  if (!out) return TQ_ERR_INVALID_ARG;
  *out = nullptr;
  if (d < 1 || d > tq::kMaxDim) return TQ_ERR_INVALID_ARG;
  const int store_flags = (int)mode & ~0xFF;
  mode = (tq_mode)((int)mode & 0xFF);
  if (mode != TQ_MODE_MSE && mode != TQ_MODE_PROD && mode != TQ_MODE_MSE_UNBIASED) return TQ_ERR_INVALID_ARG;
  if (store_flags & ~(int)TQ_STORE_RNORM_F16) return TQ_ERR_INVALID_ARG;
  if ((store_flags & TQ_STORE_RNORM_F16) && mode != TQ_MODE_PROD) return TQ_ERR_INVALID_ARG;
  if (rot != TQ_ROT_HADAMARD && rot != TQ_ROT_DENSE) return TQ_ERR_INVALID_ARG;
  const bool prod = mode == TQ_MODE_PROD;
  if (!prod && (bits < 1 || bits > 4)) return TQ_ERR_INVALID_ARG;
  if (prod && (bits < 2 || bits > 5)) return TQ_ERR_INVALID_ARG;
  int d_pad = d;
  if (rot == TQ_ROT_HADAMARD) {
    d_pad = 1;
    while (d_pad < d) d_pad *= 2;
    if (d_pad < 32) d_pad = 32;
    if (d_pad > tq::kMaxHadamard) return TQ_ERR_UNSUPPORTED;
    if (!signs) return TQ_ERR_INVALID_ARG;
  } else {
    if (d % 32 != 0) return TQ_ERR_UNSUPPORTED;
    if (!G) return TQ_ERR_INVALID_ARG;
  }
  if (prod) {
    if (!S || m < 32 || m > 4096 || m % 32 != 0) return TQ_ERR_INVALID_ARG;
  } else {
    m = 0;
  }
  const int k = prod ? bits - 1 : bits;

  tq_params* p = new tq_params();
  std::memset(&p->q, 0, sizeof(p->q));
  p->bits = bits;
  p->mode = mode;
  cudaGetDevice(&p->device);
  tq::QParams& q = p->q;
  q.d = d;
  q.d_pad = d_pad;
  q.k = k;
  q.m = m;
  q.rot = rot;
  q.unbiased = mode == TQ_MODE_MSE_UNBIASED ? 1 : 0;
  q.rnorm_f16 = (store_flags & TQ_STORE_RNORM_F16) ? 1 : 0;
  q.code_words = k * ((d_pad + 31) / 32);
  q.sign_words = m / 32;
  q.inv_sqrt_dpad = (float)(1.0 / std::sqrt((double)d_pad));
  q.kappa = m ? (float)(std::sqrt(M_PI / 2.0) / m) : 0.0f;

  double c[tq::kMaxLevels], b[tq::kMaxLevels];
  if (tq::solve_codebook(d_pad, k, c, b) != 0) {
    delete p;
    return TQ_ERR_INTERNAL;
  }
  for (int i = 0; i < tq::kMaxLevels; ++i) {
    q.centroids[i] = 0.0f;
    q.boundaries[i] = 3.0e38f;
  }
  for (int i = 0; i < (1 << k); ++i) q.centroids[i] = p->host_centroids[i] = (float)c[i];
  for (int i = 0; i + 1 < (1 << k); ++i) q.boundaries[i] = p->host_boundaries[i] = (float)b[i];

  if (rot == TQ_ROT_HADAMARD) {
    for (int j = 0; j < d_pad; ++j) {
      if (signs[j] != 1 && signs[j] != -1) {
        delete p;
        return TQ_ERR_INVALID_ARG;
      }
      if (signs[j] < 0) q.dmask[j / 32] |= 1u << (j % 32);
    }
  }

  tq_status st = TQ_OK;
  auto fail = [&](tq_status s) {
    tq_params_destroy(p);
    return s;
  };
  if (prod) {
    const size_t n = (size_t)m * d_pad;
    std::vector<float> st_host(n);
    std::vector<uint16_t> s16(n);
    for (int i = 0; i < m; ++i)
      for (int j = 0; j < d_pad; ++j) {
        const float v = S[(size_t)i * d_pad + j];
        if (!fp16_exact(v)) return fail(TQ_ERR_INVALID_ARG);
        st_host[(size_t)j * m + i] = v;
        s16[(size_t)i * d_pad + j] = to_half_bits(v);
      }
    if (cudaMalloc(&p->dev_S, n * 4) != cudaSuccess || cudaMalloc(&p->dev_St, n * 4) != cudaSuccess ||
        cudaMalloc(&p->dev_S16, n * 2) != cudaSuccess)
      return fail(TQ_ERR_CUDA);
    if (cudaMemcpy(p->dev_S, S, n * 4, cudaMemcpyHostToDevice) != cudaSuccess ||
        cudaMemcpy(p->dev_St, st_host.data(), n * 4, cudaMemcpyHostToDevice) != cudaSuccess ||
        cudaMemcpy(p->dev_S16, s16.data(), n * 2, cudaMemcpyHostToDevice) != cudaSuccess)
      return fail(TQ_ERR_CUDA);
    q.S = (const float*)p->dev_S;
    q.St = (const float*)p->dev_St;
    q.S16 = (const uint16_t*)p->dev_S16;
  }
  if (rot == TQ_ROT_DENSE) {
    const size_t n = (size_t)d * d;
    std::vector<double> pi(n);
    tq::householder_rotation(d, G, pi.data());
    p->host_Pi = (float*)std::malloc(n * 4);
    if (!p->host_Pi) return fail(TQ_ERR_INTERNAL);
    for (size_t i = 0; i < n; ++i) p->host_Pi[i] = (float)pi[i];
    if (cudaMalloc(&p->dev_Pi, n * 4) != cudaSuccess) return fail(TQ_ERR_CUDA);
    if (cudaMemcpy(p->dev_Pi, p->host_Pi, n * 4, cudaMemcpyHostToDevice) != cudaSuccess)
      return fail(TQ_ERR_CUDA);
    q.Pi = (const float*)p->dev_Pi;
    // the tensor-core encoder's operand: [hi | lo] fp16 of 2^8 Pi
    std::vector<uint16_t> pi2(2 * n);
    tq::gemm_tc::split_host(p->host_Pi, d, d, pi2.data());
    if (cudaMalloc(&p->dev_Pi2, 2 * n * 2) != cudaSuccess) return fail(TQ_ERR_CUDA);
    if (cudaMemcpy(p->dev_Pi2, pi2.data(), 2 * n * 2, cudaMemcpyHostToDevice) != cudaSuccess)
      return fail(TQ_ERR_CUDA);
    q.Pi2 = (const uint16_t*)p->dev_Pi2;
  }
  (void)st;
  *out = p;
  return TQ_OK;
}

tq_status tq_params_info(const tq_params* p, int* d_pad, int* k, int* code_words, int* sign_words,
                         int* m) {
  if (!p) return TQ_ERR_INVALID_ARG;
  if (d_pad) *d_pad = p->q.d_pad;
  if (k) *k = p->q.k;
  if (code_words) *code_words = p->q.code_words;
  if (sign_words) *sign_words = p->q.sign_words;
  if (m) *m = p->q.m;
  return TQ_OK;
}

tq_status tq_params_tables(const tq_params* p, float* centroids, float* boundaries, float* Pi) {
  if (!p) return TQ_ERR_INVALID_ARG;
  const int n = 1 << p->q.k;
  if (centroids) std::memcpy(centroids, p->host_centroids, n * sizeof(float));
  if (boundaries) std::memcpy(boundaries, p->host_boundaries, (n - 1) * sizeof(float));
  if (Pi) {
    if (!p->host_Pi) return TQ_ERR_INVALID_ARG;
    std::memcpy(Pi, p->host_Pi, (size_t)p->q.d * p->q.d * sizeof(float));
  }
  return TQ_OK;
}

}  // extern "C"

// ------------------------------------------------------------------ attention feature coefficients

#include "tq_attn_params.h"

namespace tq {
namespace attn {

void odd_feature_coefs(const float* centroids, int k, float* alpha, float* alpha_sum) {
  // subsets as bit masks in the kernel's order
  int subsets[8];
  int nf = 0;
  for (int p = 0; p < k; ++p) subsets[nf++] = 1 << p;
  if (k == 3) subsets[nf++] = 0x7;
  if (k == 4) {
    for (int t = 0; t < 4; ++t) subsets[nf++] = 0xF & ~(1 << (3 - t));
  }
  const int n = 1 << (k - 1);
  // rows: idx = n + mu (upper half); columns: features
  double A[8][9];
  for (int r = 0; r < n; ++r) {
    const int idx = n + r;
    for (int f = 0; f < nf; ++f) {
      double v = 1.0;
      for (int p = 0; p < k; ++p)
        if (subsets[f] & (1 << p)) v *= ((idx >> p) & 1) ? 1.0 : -1.0;
      A[r][f] = v;
    }
    A[r][nf] = centroids[idx];
  }
  // Gauss-Jordan elimination with partial pivoting (n <= 8)
  for (int col = 0; col < n; ++col) {
    int piv = col;
    for (int r = col + 1; r < n; ++r)
      if (std::fabs(A[r][col]) > std::fabs(A[piv][col])) piv = r;
    for (int j = 0; j <= n; ++j) std::swap(A[col][j], A[piv][j]);
    const double d = A[col][col];
    for (int j = 0; j <= n; ++j) A[col][j] /= d;
    for (int r = 0; r < n; ++r) {
      if (r == col) continue;
      const double f = A[r][col];
      for (int j = 0; j <= n; ++j) A[r][j] -= f * A[col][j];
    }
  }
  double s = 0.0;
  for (int f = 0; f < 8; ++f) alpha[f] = 0.f;
  for (int f = 0; f < n; ++f) {
    alpha[f] = (float)A[f][n];
    s += A[f][n];
  }
  *alpha_sum = (float)s;
}

}  // namespace attn
}  // namespace tq
