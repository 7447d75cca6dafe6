// Real-basis Clebsch-Gordan coefficients (host, long double arithmetic).
// See cg_host.h for the conventions.
#include "cg_host.h"

#include <cmath>
#include <complex>
#include <cstdlib>

namespace tpc {
namespace {

using ld = long double;
using cld = std::complex<long double>;

ld fact(int n) {
  ld r = 1.0L;
  for (int k = 2; k <= n; ++k) r *= (ld)k;
  return r;
}

// <j1 m1; j2 m2 | J M> by Racah's formula:
//   delta(M, m1+m2) sqrt((2J+1)(J+j1-j2)!(J-j1+j2)!(j1+j2-J)!/(j1+j2+J+1)!)
//   sqrt((J+M)!(J-M)!(j1-m1)!(j1+m1)!(j2-m2)!(j2+m2)!)
//   sum_k (-1)^k / (k!(j1+j2-J-k)!(j1-m1-k)!(j2+m2-k)!(J-j2+m1+k)!(J-j1-m2+k)!)
ld complex_cg(int j1, int m1, int j2, int m2, int J, int M) {
  if (M != m1 + m2) return 0.0L;
  if (J < std::abs(j1 - j2) || J > j1 + j2) return 0.0L;
  if (std::abs(m1) > j1 || std::abs(m2) > j2 || std::abs(M) > J) return 0.0L;
  ld pre = (ld)(2 * J + 1) * fact(J + j1 - j2) * fact(J - j1 + j2) * fact(j1 + j2 - J) /
           fact(j1 + j2 + J + 1);
  pre *= fact(J + M) * fact(J - M) * fact(j1 - m1) * fact(j1 + m1) * fact(j2 - m2) * fact(j2 + m2);
  ld s = 0.0L;
  for (int k = 0; k <= j1 + j2 - J; ++k) {
    int a[6] = {k, j1 + j2 - J - k, j1 - m1 - k, j2 + m2 - k, J - j2 + m1 + k, J - j1 - m2 + k};
    bool ok = true;
    ld d = 1.0L;
    for (int v : a) {
      if (v < 0) { ok = false; break; }
      d *= fact(v);
    }
    if (!ok) continue;
    s += ((k & 1) ? -1.0L : 1.0L) / d;
  }
  return std::sqrt(pre) * s;
}

// Row m+l (real index), column m'+l (complex index) of the complex->real map.
cld U(int l, int m, int mp) {
  const ld r = 1.0L / std::sqrt(2.0L);
  const ld sgn = (std::abs(m) & 1) ? -1.0L : 1.0L;
  if (m > 0) {
    if (mp == -m) return cld(r, 0);
    if (mp == m) return cld(sgn * r, 0);
  } else if (m == 0) {
    if (mp == 0) return cld(1, 0);
  } else {
    if (mp == m) return cld(0, r);
    if (mp == -m) return cld(0, -sgn * r);
  }
  return cld(0, 0);
}

}  // namespace

bool real_cg(int l1, int l2, int l3, std::vector<double>& R) {
  if (l1 < 0 || l2 < 0 || l3 < std::abs(l1 - l2) || l3 > l1 + l2) return false;
  const int n1 = 2 * l1 + 1, n2 = 2 * l2 + 1, n3 = 2 * l3 + 1;
  std::vector<cld> Rc((size_t)n1 * n2 * n3, cld(0, 0));
  for (int a = -l1; a <= l1; ++a)
    for (int b = -l2; b <= l2; ++b)
      for (int c = -l3; c <= l3; ++c) {
        cld acc(0, 0);
        // U[a][i] is non-zero only for i = +-a, same for b, c
        const int is[2] = {a, -a}, js[2] = {b, -b}, ks[2] = {c, -c};
        for (int ii = 0; ii < (a ? 2 : 1); ++ii)
          for (int jj = 0; jj < (b ? 2 : 1); ++jj)
            for (int kk = 0; kk < (c ? 2 : 1); ++kk) {
              const int i = is[ii], j = js[jj], k = ks[kk];
              if (i + j != k) continue;
              const ld cg = complex_cg(l1, i, l2, j, l3, k);
              if (cg == 0.0L) continue;
              acc += std::conj(U(l1, a, i)) * std::conj(U(l2, b, j)) * U(l3, c, k) * cg;
            }
        Rc[((size_t)(a + l1) * n2 + (b + l2)) * n3 + (c + l3)] = acc;
      }
  ld re = 0, im = 0;
  for (auto& v : Rc) {
    re = std::fmax(re, std::fabs(v.real()));
    im = std::fmax(im, std::fabs(v.imag()));
  }
  const bool use_im = im > re;
  R.assign(Rc.size(), 0.0);
  for (size_t t = 0; t < Rc.size(); ++t) {
    const ld v = use_im ? Rc[t].imag() : Rc[t].real();
    R[t] = std::fabs(v) < 1e-12L ? 0.0 : (double)v;
  }
  for (size_t t = 0; t < R.size(); ++t) {
    if (R[t] != 0.0) {
      if (R[t] < 0)
        for (auto& v : R) v = (v == 0.0) ? 0.0 : -v;
      break;
    }
  }
  return true;
}

std::vector<CgEntry> real_cg_sparse(int l1, int l2, int l3) {
  std::vector<double> R;
  std::vector<CgEntry> out;
  if (!real_cg(l1, l2, l3, R)) return out;
  const int n2 = 2 * l2 + 1, n3 = 2 * l3 + 1;
  for (int a = 0; a < 2 * l1 + 1; ++a)
    for (int b = 0; b < n2; ++b)
      for (int c = 0; c < n3; ++c) {
        const double v = R[((size_t)a * n2 + b) * n3 + c];
        if (v != 0.0) out.push_back({a, b, c, v});
      }
  return out;
}

}  // namespace tpc
