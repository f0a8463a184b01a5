// Host-side calibration: per-block WUSH / WUS / WUSH-diag / Hadamard / identity transforms.
//
// WUSH news article, paragraph 3: the transform combines the Cholesky factor of
// the weights' second moment (W), the SVD components (U, S) and a Hadamard
// matrix (H), is non-orthogonal and block-diagonal.  Paragraph 6: the moments
// come from calibration data (or existing Hessians), the per-block Cholesky and
// SVD run in parallel, and at inference only the activations are transformed.
//
// For block j (b x b): Sigma_X = X_j X_j^T / n, Sigma_W = W_j W_j^T / d_out,
// W' = chol(Sigma_W), W'^T Sigma_X W' = U diag(lambda) U^T (cyclic Jacobi, fp64),
// S = sqrt(lambda) descending, T_X = Hn S^{-1/2} U^T W'^T,
// T_W = Hn S^{1/2} U^T W'^{-1} (Hn = H_b / sqrt(b); WUS drops Hn).
// WUSH-diag (paragraphs 6 and 8: the data-aware component approximated by a
// diagonal matrix) is the same construction on the moments' diagonals:
// T_X = Hn D, T_W = Hn D^{-1}, D = diag((sigma_w,k / sigma_x,k)^{1/4}), each
// diagonal floored at 1e-12 of its largest entry (1 if all are zero).
// Runs in fp64 on the host's cores (OpenMP over blocks); not on the timed path.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

#include "wush.h"

namespace {

constexpr double kEigFloor = 1e-12;
constexpr double kCholJitter = 1e-8;

bool is_pow2(int64_t v) { return v > 0 && (v & (v - 1)) == 0; }

// Moments, absolute maxima and scale exponents have no meaning for NaN or an
// infinity, so calibration refuses such inputs before any work.
template <typename T>
bool all_finite(const T* p, int64_t n) {
  bool ok = true;
#pragma omp parallel for reduction(&& : ok) schedule(static)
  for (int64_t i = 0; i < n; ++i) ok = ok && std::isfinite(p[i]);
  return ok;
}

// Lower Cholesky factor of a (n x n, row-major) into l; false if not positive definite.
bool cholesky(const double* a, double* l, int n) {
  std::memset(l, 0, sizeof(double) * n * n);
  for (int i = 0; i < n; ++i) {
    for (int j = 0; j <= i; ++j) {
      double s = a[i * n + j];
      for (int k = 0; k < j; ++k) s -= l[i * n + k] * l[j * n + k];
      if (i == j) {
        if (!(s > 0.0)) return false;
        l[i * n + i] = std::sqrt(s);
      } else {
        l[i * n + j] = s / l[j * n + j];
      }
    }
  }
  return true;
}

// Inverse of a lower-triangular matrix by forward substitution, column by column.
void lower_inverse(const double* l, double* inv, int n) {
  std::memset(inv, 0, sizeof(double) * n * n);
  for (int c = 0; c < n; ++c) {
    for (int i = c; i < n; ++i) {
      double s = (i == c) ? 1.0 : 0.0;
      for (int k = c; k < i; ++k) s -= l[i * n + k] * inv[k * n + c];
      inv[i * n + c] = s / l[i * n + i];
    }
  }
}

// Symmetric eigen-decomposition by cyclic Jacobi rotations (Golub & Van Loan,
// "Matrix Computations", the cyclic Jacobi method).  a is overwritten; on return
// lam holds the eigenvalues and v (row-major) the eigenvectors as columns.
void jacobi_eigen(double* a, double* v, double* lam, int n) {
  for (int i = 0; i < n; ++i)
    for (int j = 0; j < n; ++j) v[i * n + j] = (i == j) ? 1.0 : 0.0;
  double total = 0.0;
  for (int i = 0; i < n * n; ++i) total += a[i] * a[i];
  for (int sweep = 0; sweep < 100; ++sweep) {
    double off = 0.0;
    for (int p = 0; p < n; ++p)
      for (int q = p + 1; q < n; ++q) off += a[p * n + q] * a[p * n + q];
    if (off <= 1e-32 * total) break;
    for (int p = 0; p < n; ++p) {
      for (int q = p + 1; q < n; ++q) {
        const double apq = a[p * n + q];
        if (apq == 0.0) continue;
        const double theta = (a[q * n + q] - a[p * n + p]) / (2.0 * apq);
        const double t = (theta >= 0 ? 1.0 : -1.0) / (std::fabs(theta) + std::sqrt(1.0 + theta * theta));
        const double c = 1.0 / std::sqrt(1.0 + t * t);
        const double s = t * c;
        // A <- J^T A J with J the (p, q) rotation
        for (int k = 0; k < n; ++k) {
          const double akp = a[k * n + p], akq = a[k * n + q];
          a[k * n + p] = c * akp - s * akq;
          a[k * n + q] = s * akp + c * akq;
        }
        for (int k = 0; k < n; ++k) {
          const double apk = a[p * n + k], aqk = a[q * n + k];
          a[p * n + k] = c * apk - s * aqk;
          a[q * n + k] = s * apk + c * aqk;
        }
        for (int k = 0; k < n; ++k) {
          const double vkp = v[k * n + p], vkq = v[k * n + q];
          v[k * n + p] = c * vkp - s * vkq;
          v[k * n + q] = s * vkp + c * vkq;
        }
      }
    }
  }
  for (int i = 0; i < n; ++i) lam[i] = a[i * n + i];
}

// Fills hn (n x n) with H_n / sqrt(n), H_n[i][j] = (-1)^popcount(i & j).
void normalized_hadamard(double* hn, int n) {
  const double s = 1.0 / std::sqrt(static_cast<double>(n));
  for (int i = 0; i < n; ++i)
    for (int j = 0; j < n; ++j) hn[i * n + j] = (__builtin_popcount(i & j) & 1) ? -s : s;
}

// One block: (sigma_x, sigma_w) -> (t_x, t_w) as fp32.  Returns a wush_status.
int block_pair(const double* sx, const double* sw, int b, int kind, float* tx, float* tw) {
  const int bb = b * b;
  if (kind == WUSH_T_IDENTITY) {
    for (int i = 0; i < bb; ++i) tx[i] = tw[i] = (i / b == i % b) ? 1.0f : 0.0f;
    return WUSH_OK;
  }
  std::vector<double> hn(bb);
  normalized_hadamard(hn.data(), b);
  if (kind == WUSH_T_HADAMARD) {
    for (int i = 0; i < bb; ++i) tx[i] = tw[i] = static_cast<float>(hn[i]);
    return WUSH_OK;
  }
  if (kind == WUSH_T_WUSH_DIAG) {
    double mx = 0.0, mw = 0.0;
    for (int k = 0; k < b; ++k) {
      mx = std::fmax(mx, sx[k * b + k]);
      mw = std::fmax(mw, sw[k * b + k]);
    }
    const double fx = kEigFloor * (mx > 0 ? mx : 1.0), fw = kEigFloor * (mw > 0 ? mw : 1.0);
    std::vector<double> d(b);
    for (int k = 0; k < b; ++k) d[k] = std::pow(std::fmax(sw[k * b + k], fw) / std::fmax(sx[k * b + k], fx), 0.25);
    for (int i = 0; i < b; ++i)
      for (int j = 0; j < b; ++j) {
        tx[i * b + j] = static_cast<float>(hn[i * b + j] * d[j]);
        tw[i * b + j] = static_cast<float>(hn[i * b + j] / d[j]);
      }
    return WUSH_OK;
  }
  std::vector<double> l(bb), linv(bb), m(bb), tmp(bb), u(bb), lam(b);
  if (!cholesky(sw, l.data(), b)) {
    double tr = 0.0;
    for (int i = 0; i < b; ++i) tr += sw[i * b + i];
    std::vector<double> sj(sw, sw + bb);
    for (int i = 0; i < b; ++i) sj[i * b + i] += kCholJitter * tr / b;
    if (!cholesky(sj.data(), l.data(), b)) return WUSH_ERR_NOT_SPD;
  }
  lower_inverse(l.data(), linv.data(), b);
  // m = L^T Sigma_X L
  for (int i = 0; i < b; ++i)
    for (int j = 0; j < b; ++j) {
      double s = 0.0;
      for (int k = 0; k < b; ++k) s += sx[i * b + k] * l[k * b + j];
      tmp[i * b + j] = s;
    }
  for (int i = 0; i < b; ++i)
    for (int j = 0; j < b; ++j) {
      double s = 0.0;
      for (int k = 0; k < b; ++k) s += l[k * b + i] * tmp[k * b + j];
      m[i * b + j] = s;
    }
  for (int i = 0; i < b; ++i)  // symmetrise rounding noise
    for (int j = i + 1; j < b; ++j) m[i * b + j] = m[j * b + i] = 0.5 * (m[i * b + j] + m[j * b + i]);
  jacobi_eigen(m.data(), u.data(), lam.data(), b);
  // order: descending eigenvalues (stable for equal values)
  std::vector<int> order(b);
  for (int i = 0; i < b; ++i) order[i] = i;
  for (int i = 1; i < b; ++i) {
    int k = order[i], j = i - 1;
    while (j >= 0 && lam[order[j]] < lam[k]) { order[j + 1] = order[j]; --j; }
    order[j + 1] = k;
  }
  double lmax = lam[order[0]] > 0 ? lam[order[0]] : 0.0;
  std::vector<double> us(bb), sv(b);
  for (int c = 0; c < b; ++c) {
    const int src = order[c];
    int imax = 0;
    for (int i = 1; i < b; ++i)
      if (std::fabs(u[i * b + src]) > std::fabs(u[imax * b + src])) imax = i;
    const double sgn = u[imax * b + src] < 0 ? -1.0 : 1.0;
    for (int i = 0; i < b; ++i) us[i * b + c] = sgn * u[i * b + src];
    double lv = lam[src];
    if (lv < kEigFloor * lmax) lv = kEigFloor * lmax;
    sv[c] = std::sqrt(lv);
  }
  // a = diag(s^-1/2) U^T L^T  and  c = diag(s^1/2) U^T L^{-1}
  std::vector<double> ax(bb), aw(bb);
  for (int i = 0; i < b; ++i) {
    const double fx = 1.0 / std::sqrt(sv[i]), fw = std::sqrt(sv[i]);
    for (int j = 0; j < b; ++j) {
      double s1 = 0.0, s2 = 0.0;
      for (int k = 0; k < b; ++k) {
        s1 += us[k * b + i] * l[j * b + k];      // (U^T)_{ik} (L^T)_{kj}
        s2 += us[k * b + i] * linv[k * b + j];   // (U^T)_{ik} (L^-1)_{kj}
      }
      ax[i * b + j] = fx * s1;
      aw[i * b + j] = fw * s2;
    }
  }
  for (int i = 0; i < b; ++i)
    for (int j = 0; j < b; ++j) {
      double s1, s2;
      if (kind == WUSH_T_WUSH) {
        s1 = s2 = 0.0;
        for (int k = 0; k < b; ++k) {
          s1 += hn[i * b + k] * ax[k * b + j];
          s2 += hn[i * b + k] * aw[k * b + j];
        }
      } else {
        s1 = ax[i * b + j];
        s2 = aw[i * b + j];
      }
      tx[i * b + j] = static_cast<float>(s1);
      tw[i * b + j] = static_cast<float>(s2);
    }
  return WUSH_OK;
}

// Per-block second moments (1/rows) sum_r x_rj x_rj^T of a [rows, d_in] fp32 matrix.
void block_moments(const float* x, int64_t rows, int64_t d_in, int b, double* out) {
  const int64_t nb = d_in / b;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t j = 0; j < nb; ++j) {
    std::vector<double> acc(static_cast<size_t>(b) * b, 0.0), xv(b);
    for (int64_t r = 0; r < rows; ++r) {
      const float* p = x + r * d_in + j * b;
      for (int k = 0; k < b; ++k) xv[k] = p[k];
      for (int k = 0; k < b; ++k) {
        const double xk = xv[k];
        double* row = &acc[static_cast<size_t>(k) * b];
        for (int l = k; l < b; ++l) row[l] += xk * xv[l];
      }
    }
    double* o = out + j * b * b;
    for (int k = 0; k < b; ++k)
      for (int l = k; l < b; ++l) o[k * b + l] = o[l * b + k] = acc[static_cast<size_t>(k) * b + l] / rows;
  }
}

}  // namespace

extern "C" int wush_calibrate_from_moments(const double* sigma_x, const double* sigma_w, int64_t d_in,
                                           int block, int kind, float* t_x, float* t_w) {
  if (!t_x || !t_w || !is_pow2(block) || block < 2 || block > 256 || d_in <= 0 || d_in % block)
    return WUSH_ERR_INVALID_ARG;
  if (kind < WUSH_T_IDENTITY || kind > WUSH_T_WUSH_DIAG) return WUSH_ERR_UNSUPPORTED;
  if (kind >= WUSH_T_WUS && (!sigma_x || !sigma_w)) return WUSH_ERR_INVALID_ARG;
  const int64_t nb = d_in / block, bb = static_cast<int64_t>(block) * block;
  if (kind >= WUSH_T_WUS && (!all_finite(sigma_x, nb * bb) || !all_finite(sigma_w, nb * bb)))
    return WUSH_ERR_INVALID_ARG;
  int status = WUSH_OK;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t j = 0; j < nb; ++j) {
    const double* sx = sigma_x ? sigma_x + j * bb : nullptr;
    const double* sw = sigma_w ? sigma_w + j * bb : nullptr;
    int st = block_pair(sx, sw, block, kind, t_x + j * bb, t_w + j * bb);
    if (st != WUSH_OK) {
#pragma omp critical
      status = st;
    }
  }
  return status;
}

extern "C" int wush_calibrate(const float* x_calib, int64_t n_calib, const float* w, int64_t d_out,
                              int64_t d_in, int block, int kind, float* t_x, float* t_w) {
  if (!t_x || !t_w || !is_pow2(block) || block < 2 || block > 256 || d_in <= 0 || d_in % block)
    return WUSH_ERR_INVALID_ARG;
  if (kind < WUSH_T_IDENTITY || kind > WUSH_T_WUSH_DIAG) return WUSH_ERR_UNSUPPORTED;
  if (kind == WUSH_T_IDENTITY || kind == WUSH_T_HADAMARD)
    return wush_calibrate_from_moments(nullptr, nullptr, d_in, block, kind, t_x, t_w);
  if (!x_calib || !w || n_calib <= 0 || d_out <= 0) return WUSH_ERR_INVALID_ARG;
  if (!all_finite(x_calib, n_calib * d_in) || !all_finite(w, d_out * d_in)) return WUSH_ERR_INVALID_ARG;
  const size_t n = static_cast<size_t>(d_in / block) * block * block;
  std::vector<double> sx(n), sw(n);
  block_moments(x_calib, n_calib, d_in, block, sx.data());
  block_moments(w, d_out, d_in, block, sw.data());
  return wush_calibrate_from_moments(sx.data(), sw.data(), d_in, block, kind, t_x, t_w);
}

// ---------------------------------------------------------------------------
// Transform sharing (WUSH news article, paragraph 6: share transform matrices
// between similar blocks).  The pages give no algorithm.  Reading: a block's
// feature is its two moments divided by their traces, flattened; k-means (Lloyd)
// groups the features, with centres started at blocks round(i * nb / groups)
// (halves to even), squared Euclidean distance, ties to the lowest group, empty
// groups keeping their centre, until no block changes group (at most 50
// rounds).  Each group's transform comes from its members' mean moments.
extern "C" int wush_calibrate_shared_from_moments(const double* sigma_x, const double* sigma_w, int64_t d_in,
                                                  int block, int kind, int groups, float* t_x, float* t_w,
                                                  int32_t* index) {
  if (!sigma_x || !sigma_w || !t_x || !t_w || !index || !is_pow2(block) || block < 2 || block > 256 || d_in <= 0 ||
      d_in % block)
    return WUSH_ERR_INVALID_ARG;
  if (kind < WUSH_T_WUS || kind > WUSH_T_WUSH_DIAG) return WUSH_ERR_UNSUPPORTED;
  const int64_t nb = d_in / block, bb = static_cast<int64_t>(block) * block, nf = 2 * bb;
  if (groups < 1 || groups > nb) return WUSH_ERR_INVALID_ARG;
  if (!all_finite(sigma_x, nb * bb) || !all_finite(sigma_w, nb * bb)) return WUSH_ERR_INVALID_ARG;
  std::vector<double> feat(static_cast<size_t>(nb * nf));
  for (int64_t j = 0; j < nb; ++j) {
    for (int m = 0; m < 2; ++m) {
      const double* sg = (m == 0 ? sigma_x : sigma_w) + j * bb;
      double tr = 0.0;
      for (int k = 0; k < block; ++k) tr += sg[k * block + k];
      const double dv = tr > 0 ? tr : 1.0;
      for (int64_t e = 0; e < bb; ++e) feat[j * nf + m * bb + e] = sg[e] / dv;
    }
  }
  std::vector<double> centres(static_cast<size_t>(groups * nf));
  for (int g = 0; g < groups; ++g) {
    const int64_t src = static_cast<int64_t>(std::nearbyint(static_cast<double>(g) * nb / groups));
    std::memcpy(&centres[g * nf], &feat[src * nf], sizeof(double) * nf);
  }
  std::vector<int32_t> assign(nb, -1), next(nb);
  for (int it = 0; it < 50; ++it) {
    for (int64_t j = 0; j < nb; ++j) {
      int best = 0;
      double best_d = 0.0;
      for (int g = 0; g < groups; ++g) {
        double d = 0.0;
        for (int64_t f = 0; f < nf; ++f) {
          const double v = feat[j * nf + f] - centres[g * nf + f];
          d += v * v;
        }
        if (g == 0 || d < best_d) { best = g; best_d = d; }
      }
      next[j] = best;
    }
    if (next == assign) break;
    assign = next;
    for (int g = 0; g < groups; ++g) {
      int64_t cnt = 0;
      std::vector<double> acc(nf, 0.0);
      for (int64_t j = 0; j < nb; ++j)
        if (assign[j] == g) {
          ++cnt;
          for (int64_t f = 0; f < nf; ++f) acc[f] += feat[j * nf + f];
        }
      if (cnt)
        for (int64_t f = 0; f < nf; ++f) centres[g * nf + f] = acc[f] / cnt;
    }
  }
  std::vector<double> gx(static_cast<size_t>(groups * bb), 0.0), gw(static_cast<size_t>(groups * bb), 0.0);
  std::vector<int64_t> cnt(groups, 0);
  for (int64_t j = 0; j < nb; ++j) {
    const int g = assign[j];
    index[j] = g;
    ++cnt[g];
    for (int64_t e = 0; e < bb; ++e) {
      gx[g * bb + e] += sigma_x[j * bb + e];
      gw[g * bb + e] += sigma_w[j * bb + e];
    }
  }
  for (int g = 0; g < groups; ++g) {
    if (cnt[g] == 0) {
      // a group left empty (its start tied with an earlier group's) maps no block:
      // its transform comes from its starting block's moments
      const int64_t src = static_cast<int64_t>(std::nearbyint(static_cast<double>(g) * nb / groups));
      std::memcpy(&gx[g * bb], sigma_x + src * bb, sizeof(double) * bb);
      std::memcpy(&gw[g * bb], sigma_w + src * bb, sizeof(double) * bb);
      continue;
    }
    for (int64_t e = 0; e < bb; ++e) {
      gx[g * bb + e] /= static_cast<double>(cnt[g]);
      gw[g * bb + e] /= static_cast<double>(cnt[g]);
    }
  }
  return wush_calibrate_from_moments(gx.data(), gw.data(), static_cast<int64_t>(groups) * block, block, kind, t_x,
                                     t_w);
}

extern "C" int wush_calibrate_shared(const float* x_calib, int64_t n_calib, const float* w, int64_t d_out,
                                     int64_t d_in, int block, int kind, int groups, float* t_x, float* t_w,
                                     int32_t* index) {
  if (!x_calib || !w || n_calib <= 0 || d_out <= 0 || !is_pow2(block) || block < 2 || block > 256 || d_in <= 0 ||
      d_in % block)
    return WUSH_ERR_INVALID_ARG;
  if (!all_finite(x_calib, n_calib * d_in) || !all_finite(w, d_out * d_in)) return WUSH_ERR_INVALID_ARG;
  const size_t n = static_cast<size_t>(d_in / block) * block * block;
  std::vector<double> sx(n), sw(n);
  block_moments(x_calib, n_calib, d_in, block, sx.data());
  block_moments(w, d_out, d_in, block, sw.data());
  return wush_calibrate_shared_from_moments(sx.data(), sw.data(), d_in, block, kind, groups, t_x, t_w, index);
}

// Static NVFP4 per-tensor scale and GEMM alpha (see wush.h): plain fp32 IEEE
// arithmetic, one rounding each.
extern "C" int wush_nvfp4_global_scale(float amax, float* s_g) {
  if (!s_g || !std::isfinite(amax) || amax < 0.0f) return WUSH_ERR_INVALID_ARG;
  const float q = amax / 2688.0f;
  *s_g = q >= 1e-30f ? q : 1.0f;
  return WUSH_OK;
}

extern "C" int wush_nvfp4_alpha(float s_gx, float s_gw, float* alpha) {
  if (!alpha || !std::isfinite(s_gx) || !std::isfinite(s_gw) || !(s_gx > 0.0f) || !(s_gw > 0.0f))
    return WUSH_ERR_INVALID_ARG;
  *alpha = s_gx * s_gw;
  return WUSH_OK;
}
