// Build-time emitter of the compile-time CG table used by the kernels.
//
// LunaTP (§4.3, "Sparse expansion") embeds the non-zero coefficients and their
// component indices in the kernel code so that no table is read at run time and
// no zero term is ever visited. This program writes the same real-basis
// coefficients that the run-time planner computes (cg_host.cpp) into a header of
// constexpr structures, grouped for the kernels' access pattern:
//
//   for each (l1, l2, l3): the non-zero (m1, m3) pairs, each with its list of
//   (m2, c) terms, so that cY[m1][m3] = sum_{m2} c * Y[m2] is one short dot
//   product and T[m3] = sum_{m1} cY[m1][m3] x[m1] touches only non-zero pairs.
//
// Usage: cg_gen <lmax> <output-file>
#include <algorithm>
#include <cstdio>
#include <cstdlib>
#include <vector>

#include "cg_host.h"

int main(int argc, char** argv) {
  if (argc != 3) {
    std::fprintf(stderr, "usage: %s <lmax> <out.inc>\n", argv[0]);
    return 2;
  }
  const int lmax = std::atoi(argv[1]);
  FILE* f = std::fopen(argv[2], "w");
  if (!f) return 1;
  std::fprintf(f,
               "// Generated at build time by cg_gen from cg_host.cpp. Do not edit.\n"
               "#pragma once\n"
               "namespace tpc {\nnamespace cgt {\n"
               "constexpr int kLmax = %d;\n"
               "struct Pair { int m1, m3, start, n; };\n"
               "struct Term { int m2; double c; };\n"
               "struct Flat { signed char l1, l2, l3, m1, m2, m3; double c; };\n"
               "template <int L1, int L2, int L3> struct CG;\n",
               lmax);
  std::vector<std::vector<int>> flat_keys;
  std::vector<double> flat_c;
  for (int l1 = 0; l1 <= lmax; ++l1)
    for (int l2 = 0; l2 <= lmax; ++l2)
      for (int l3 = std::abs(l1 - l2); l3 <= std::min(l1 + l2, lmax); ++l3) {
        auto e = tpc::real_cg_sparse(l1, l2, l3);
        std::stable_sort(e.begin(), e.end(), [](const tpc::CgEntry& a, const tpc::CgEntry& b) {
          if (a.m1 != b.m1) return a.m1 < b.m1;
          if (a.m3 != b.m3) return a.m3 < b.m3;
          return a.m2 < b.m2;
        });
        std::vector<int> pm1, pm3, pst, pn;
        for (size_t k = 0; k < e.size(); ++k) {
          if (k == 0 || e[k].m1 != e[k - 1].m1 || e[k].m3 != e[k - 1].m3) {
            pm1.push_back(e[k].m1);
            pm3.push_back(e[k].m3);
            pst.push_back((int)k);
            pn.push_back(0);
          }
          pn.back()++;
        }
        std::fprintf(f, "template <> struct CG<%d, %d, %d> {\n", l1, l2, l3);
        std::fprintf(f, "  static constexpr int npair = %zu;\n  static constexpr Pair pair[%zu] = {",
                     pm1.size(), pm1.size());
        for (size_t p = 0; p < pm1.size(); ++p)
          std::fprintf(f, "%s{%d, %d, %d, %d}", p ? ", " : "", pm1[p], pm3[p], pst[p], pn[p]);
        std::fprintf(f, "};\n  static constexpr int nterm = %zu;\n  static constexpr Term term[%zu] = {",
                     e.size(), e.size());
        for (size_t k = 0; k < e.size(); ++k)
          std::fprintf(f, "%s{%d, %.17g}", k ? ", " : "", e[k].m2, e[k].c);
        std::fprintf(f, "};\n};\n");
        for (auto& t : e) {
          flat_keys.push_back({l1, l2, l3, t.m1, t.m2, t.m3});
          flat_c.push_back(t.c);
        }
      }
  std::fprintf(f, "#ifdef TPC_CG_FLAT\nconstexpr int kFlatCount = %zu;\nconstexpr Flat kFlat[%zu] = {\n",
               flat_c.size(), flat_c.size());
  for (size_t k = 0; k < flat_c.size(); ++k) {
    auto& q = flat_keys[k];
    std::fprintf(f, "  {%d, %d, %d, %d, %d, %d, %.17g},\n", q[0], q[1], q[2], q[3], q[4], q[5], flat_c[k]);
  }
  std::fprintf(f, "};\n#endif\n}  // namespace cgt\n}  // namespace tpc\n");
  std::fclose(f);
  return 0;
}
