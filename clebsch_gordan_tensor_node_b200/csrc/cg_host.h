// Host-side Clebsch-Gordan coefficients in the real spherical-harmonic basis.
//
// Coupling of LunaTP (§2.1, Eq. 1): the degree-l3 part of x^(l1) (x) y^(l2) is
// sum_{m1,m2} C[m1][m2][m3] x_{m1} y_{m2}, non-zero only for |l1-l2| <= l3 <= l1+l2.
// Sobek (§4.2, Eq. 32) uses the same sparse coefficient in the real basis.
//
// Conventions (fixed here; the pages leave them open):
//   * complex CG from Racah's closed formula, Condon-Shortley phases;
//   * real basis per degree: m<0 sine-type, m=0, m>0 cosine-type, index m+l, so
//     l=1 is ordered (y, z, x);
//   * R[a][b][c] = sum conj(U1[a][i]) conj(U2[b][j]) U3[c][k] C[i][j][k], whose real
//     or imaginary part (whichever is non-zero) is kept;
//   * orthonormal in (m1, m2) for each m3; the first non-zero entry in
//     lexicographic (m1, m2, m3) order is positive; path normalisation 1.
#pragma once

#include <vector>

namespace tpc {

// Dense real coupling tensor R[(m1*(2l2+1) + m2)*(2l3+1) + m3], entries below 1e-12
// in magnitude are set to exactly zero. Returns false if the triangle rule fails.
bool real_cg(int l1, int l2, int l3, std::vector<double>& R);

struct CgEntry {
  int m1, m2, m3;
  double c;
};

// Non-zero entries of real_cg in lexicographic (m1, m2, m3) order.
std::vector<CgEntry> real_cg_sparse(int l1, int l2, int l3);

}  // namespace tpc
