// Host planner of the tensor-product convolution (Sobek §4.5: the wrapper
// validates the contract and enumerates valid paths and sparse CG terms; LunaTP
// §4.2: work is partitioned into tasks over receivers, path groups and channel
// blocks).
//
// Path enumeration (the pages fix no order; this order defines the layout of A):
// for each input block in the order written, for l2 = 0..L_sh (parity (-1)^l2),
// for l3 = |l1-l2|..l1+l2, one path to every output block of degree l3 and
// parity p1 p2 (Sobek §2.2 selection rule), in output order. Output blocks
// receive the sum over their paths.
#include "plan.h"

#include <algorithm>
#include <cctype>
#include <cmath>
#include <cstdlib>

#include "cg_host.h"
#include "tpconv.h"

namespace tpc {
namespace {

bool parse_irreps(const char* s, std::vector<Block>& out, std::string& msg) {
  out.clear();
  if (!s) {
    msg = "irreps string is NULL";
    return false;
  }
  std::string str(s);
  size_t pos = 0;
  int off = 0;
  while (pos <= str.size()) {
    size_t end = str.find('+', pos);
    if (end == std::string::npos) end = str.size();
    std::string t;
    for (size_t k = pos; k < end; ++k)
      if (!std::isspace((unsigned char)str[k])) t.push_back(str[k]);
    if (t.empty()) {
      msg = "empty irreps term in '" + str + "'";
      return false;
    }
    int mul = 1;
    size_t x = t.find('x');
    std::string ir = t;
    if (x != std::string::npos) {
      mul = std::atoi(t.substr(0, x).c_str());
      ir = t.substr(x + 1);
      for (size_t k = 0; k < x; ++k)
        if (!std::isdigit((unsigned char)t[k])) mul = -1;
    }
    if (ir.size() < 2 || (ir.back() != 'e' && ir.back() != 'o') || mul <= 0) {
      msg = "bad irreps term '" + t + "'";
      return false;
    }
    for (size_t k = 0; k + 1 < ir.size(); ++k)
      if (!std::isdigit((unsigned char)ir[k])) {
        msg = "bad irreps term '" + t + "'";
        return false;
      }
    const int l = std::atoi(ir.substr(0, ir.size() - 1).c_str());
    const int p = ir.back() == 'e' ? 1 : -1;
    out.push_back({mul, l, p, off});
    off += mul * (2 * l + 1);
    pos = end + 1;
  }
  return !out.empty();
}

// Appends, for every block, its member paths to plist and one tile per run of
// tile_w channels to tiles (each tile refers to the block's path range).
void add_tiles(const std::vector<Block>& blocks, const std::vector<std::vector<int>>& members,
               const std::vector<HostPath>& paths, int tile_w, std::vector<TileD>& tiles,
               std::vector<PathD>& plist) {
  for (size_t b = 0; b < blocks.size(); ++b) {
    const int pbeg = (int)plist.size();
    for (int pi : members[b]) {
      const HostPath& h = paths[pi];
      PathD d{};
      d.l1 = (int8_t)h.l1;
      d.l2 = (int8_t)h.l2;
      d.l3 = (int8_t)h.l3;
      d.x_off = h.x_off;
      d.out_off = h.out_off;
      d.w_off = (int)h.w_off;
      d.mul_in = h.mul_in;
      d.mul_out = h.mul_out;
      plist.push_back(d);
    }
    const int pend = (int)plist.size();
    const Block& bl = blocks[b];
    for (int ch0 = 0; ch0 < bl.mul; ch0 += tile_w)
      tiles.push_back({bl.l, bl.offset, bl.mul, ch0, std::min(tile_w, bl.mul - ch0), pbeg, pend});
  }
}

}  // namespace

int make_plan(const char* irreps_in, int sh_lmax, const char* irreps_out, int n_radial, int mode,
              int dtype, Plan& P, std::string& msg, const int* sh_parity) {
  P = Plan{};
  auto par2 = [&](int l2) { return sh_parity ? sh_parity[l2] : ((l2 & 1) ? -1 : 1); };
  if (mode != TP_UVU && mode != TP_UVW && mode != TP_UVU_PATHS) {
    msg = "mode must be TP_UVU, TP_UVW or TP_UVU_PATHS";
    return TP_EINVAL;
  }
  if (dtype != TP_F32 && dtype != TP_F64) {
    msg = "dtype must be TP_F32 or TP_F64";
    return TP_EINVAL;
  }
  if (sh_lmax < 0 || n_radial <= 0) {
    msg = "sh_lmax must be >= 0 and n_radial > 0";
    return TP_EINVAL;
  }
  if (sh_lmax > 16) {
    msg = "sh_lmax above 16";
    return TP_EINVAL;
  }
  if (!parse_irreps(irreps_in, P.bin, msg) || !parse_irreps(irreps_out, P.bout, msg)) return TP_EINVAL;
  if (mode == TP_UVU_PATHS) {
    // one output block per path (LunaTP Appendix A.1: per-path uvu outputs are
    // concatenated): irreps_out only says which (l, p) exist; the output
    // blocks are the paths' own, in enumeration order
    std::vector<Block> allowed = P.bout;
    P.bout.clear();
    int off = 0;
    for (const Block& b1 : P.bin)
      for (int l2 = 0; l2 <= sh_lmax; ++l2)
        for (int l3 = std::abs(b1.l - l2); l3 <= b1.l + l2; ++l3) {
          const int p3 = b1.p * par2(l2);
          bool ok = false;
          for (const Block& a : allowed) ok |= (a.l == l3 && a.p == p3);
          if (!ok) continue;
          P.bout.push_back({b1.mul, l3, p3, off});
          off += b1.mul * (2 * l3 + 1);
        }
    if (P.bout.empty()) {
      msg = "no path reaches the output irreps";
      return TP_EINVAL;
    }
    P.per_path = true;
    mode = TP_UVU;
  }
  P.mode = mode;
  P.dtype = dtype;
  P.K = n_radial;
  P.sh_lmax = sh_lmax;
  P.dim_y = (sh_lmax + 1) * (sh_lmax + 1);
  for (auto& b : P.bin) P.c_in += b.mul * (2 * b.l + 1);
  for (auto& b : P.bout) P.c_out += b.mul * (2 * b.l + 1);
  long long w = 0;
  for (size_t i1 = 0; i1 < P.bin.size(); ++i1) {
    const Block& b1 = P.bin[i1];
    for (int l2 = 0; l2 <= sh_lmax; ++l2) {
      const int p2 = par2(l2);
      for (int l3 = std::abs(b1.l - l2); l3 <= b1.l + l2; ++l3) {
        const int p3 = b1.p * p2;
        // per-path outputs: the path about to be added owns the next block
        const size_t io0 = P.per_path ? P.paths.size() : 0;
        const size_t io1 = P.per_path ? std::min(P.paths.size() + 1, P.bout.size()) : P.bout.size();
        for (size_t io = io0; io < io1; ++io) {
          const Block& bo = P.bout[io];
          if (bo.l != l3 || bo.p != p3) continue;
          HostPath h{};
          h.l1 = b1.l; h.p1 = b1.p; h.l2 = l2; h.p2 = p2; h.l3 = l3; h.p3 = p3;
          h.i_in = (int)i1; h.i_out = (int)io;
          h.mul_in = b1.mul; h.mul_out = bo.mul;
          h.x_off = b1.offset; h.out_off = bo.offset;
          if (mode == TP_UVU) {
            if (bo.mul != b1.mul) {
              msg = "uvu needs equal input and output multiplicity on every path";
              return TP_EUNSUPPORTED;
            }
            h.n_w = b1.mul;
          } else {
            h.n_w = (long long)b1.mul * bo.mul;
          }
          h.w_off = w;
          h.nnz = (int)real_cg_sparse(h.l1, h.l2, h.l3).size();
          w += h.n_w;
          P.paths.push_back(h);
          P.lmax = std::max(P.lmax, std::max(h.l1, std::max(h.l2, h.l3)));
        }
      }
    }
  }
  P.n_w = w;
  for (auto& b : P.bin) P.lmax = std::max(P.lmax, b.l);
  for (auto& b : P.bout) P.lmax = std::max(P.lmax, b.l);
  P.lmax = std::max(P.lmax, sh_lmax);
  // limits of the compiled kernels: degrees up to kLmax everywhere; up to
  // kLmaxUvu for channelwise fp32 plans with K <= 8
  const bool wide = mode == TP_UVU && dtype == TP_F32 && P.K <= 8;
  if (P.lmax > (wide ? kLmaxUvu : kLmax)) {
    msg = "degree " + std::to_string(P.lmax) + " above the kernels' limit " +
          std::to_string(wide ? kLmaxUvu : kLmax) + " for this mode, dtype and K";
    return TP_EUNSUPPORTED;
  }
  if (P.K > 16) {
    msg = "n_radial above 16 is not compiled";
    return TP_EUNSUPPORTED;
  }
  P.KP = P.K <= 8 ? 8 : 16;
  if ((int)P.paths.size() > kMaxPaths) {
    msg = "more than " + std::to_string(kMaxPaths) + " paths";
    return TP_EUNSUPPORTED;
  }
  if (P.n_w * (long long)P.K >= (1LL << 31) || P.c_in <= 0 || P.c_out <= 0) {
    msg = "weight tensor too large for 32-bit indexing";
    return TP_EUNSUPPORTED;
  }
  bool all_even = true;
  int min_mul = 1 << 30;
  for (const auto* v : {&P.bin, &P.bout})
    for (auto& b : *v) {
      all_even &= (b.mul % 2 == 0);
      min_mul = std::min(min_mul, b.mul);
    }
  // backward kernels: 1 or 2 channels per lane (fp32), 1 (fp64)
  P.CPL = (dtype == TP_F32 && all_even) ? 2 : 1;
  // edge pass: 16-byte gathers when every multiplicity allows them
  {
    const int vw = dtype == TP_F32 ? 4 : 2;
    bool ok = true;
    for (const auto* v : {&P.bin, &P.bout})
      for (auto& b : *v) ok &= (b.mul % vw == 0);
    P.edge_V = ok ? vw : 1;
  }
  // forward: vector width by dtype and block width (every access CPL-aligned);
  // 4 channels per lane measured slower than 2 on the 128-channel workload
  if (dtype == TP_F32)
    P.fwd_CPL = all_even ? 2 : 1;
  else
    P.fwd_CPL = (all_even && min_mul >= 64) ? 2 : 1;
  // degree profile of the forward kernel: (max input l, sh_lmax, max output l)
  // bounded by one of the compiled profiles
  int lin = 0, lout = 0;
  for (auto& b : P.bin) lin = std::max(lin, b.l);
  for (auto& b : P.bout) lout = std::max(lout, b.l);
  const int profs[5][3] = {{2, 2, 2}, {1, 3, 3}, {3, 3, 3}, {4, 4, 4}, {6, 6, 6}};
  for (int k = 0; k < 5; ++k)
    if (lin <= profs[k][0] && sh_lmax <= profs[k][1] && lout <= profs[k][2]) {
      P.prof = k;
      break;
    }
  // the widest profile is compiled for one channel per lane and scalar gathers
  if (P.prof == 4) P.CPL = P.fwd_CPL = P.edge_V = 1;
  // instantiated combinations (uvu_fwd.cu): fp64 with 2 channels per lane only
  // with profiles 0-2
  if (dtype == TP_F64 && P.fwd_CPL == 2 && P.prof == 3) P.fwd_CPL = 1;
  std::vector<std::vector<int>> by_out(P.bout.size()), by_in(P.bin.size());
  for (size_t k = 0; k < P.paths.size(); ++k) {
    by_out[P.paths[k].i_out].push_back((int)k);
    by_in[P.paths[k].i_in].push_back((int)k);
  }
  add_tiles(P.bout, by_out, P.paths, 32 * P.fwd_CPL, P.out_tiles, P.paths_by_out);
  add_tiles(P.bin, by_in, P.paths, 32 * P.CPL, P.in_tiles, P.paths_by_in);
  std::vector<std::vector<int>> all(1);
  for (size_t k = 0; k < P.paths.size(); ++k) all[0].push_back((int)k);
  std::vector<TileD> unused;
  std::vector<Block> one{{1, 0, 1, 0}};
  add_tiles(one, all, P.paths, 1, unused, P.paths_canon);
  add_tiles(P.bout, by_out, P.paths, 32, P.dbl_out_tiles, P.dbl_paths_by_out);
  add_tiles(P.bin, by_in, P.paths, 32, P.dbl_in_tiles, P.dbl_paths_by_in);
  P.dbl_ok = (int)P.dbl_out_tiles.size() <= kMaxTiles && (int)P.dbl_in_tiles.size() <= kMaxTiles;
  if ((int)P.out_tiles.size() > kMaxTiles || (int)P.in_tiles.size() > kMaxTiles) {
    msg = "more than " + std::to_string(kMaxTiles) + " channel tiles";
    return TP_EUNSUPPORTED;
  }
  // forward staging: per output block, the cY slots of its paths, each padded
  // to a 16-byte vector so that the kernel reads them with 16-byte loads
  const int bsz = dtype == TP_F32 ? 4 : 8, vw = 16 / bsz;
  P.cy_stride = vw;
  for (const TileD& t : P.out_tiles) {
    int off = 0;
    for (int k = t.pbeg; k < t.pend; ++k) {
      PathD& d = P.paths_by_out[k];
      auto e = real_cg_sparse(d.l1, d.l2, d.l3);
      std::vector<std::pair<int, int>> pairs;
      for (auto& q : e) pairs.emplace_back(q.m1, q.m3);
      std::sort(pairs.begin(), pairs.end());
      pairs.erase(std::unique(pairs.begin(), pairs.end()), pairs.end());
      d.cy_off = off;
      off += ((int)pairs.size() + vw - 1) / vw * vw;
    }
    P.cy_stride = std::max(P.cy_stride, off);
  }
  // forward: per warp, the staged chunk (senders, radial rows, cY) and an x copy
  // ring of two groups of ring_g edges (every component of the widest input
  // block, 32 lanes x CPL channels). Group size, then chunk, shrink until one
  // CTA of fwd_warps warps fits on an SM.
  {
    // the kernel sizes the ring for its degree profile's widest input block
    const int l1p = profs[P.prof][0], d1 = 2 * l1p + 1, warps = fwd_warps_for(bsz);
    const int budget = 226 * 1024 / ctas_per_sm_for(bsz);
    const int g = fwd_ring_g(bsz, P.fwd_CPL, l1p);
    auto base = [&](int chunk) { return (32 * 4 + 32 * P.KP * bsz + chunk * P.cy_stride * bsz + 15) / 16 * 16; };
    auto per_warp = [&](int chunk) { return base(chunk) + (2 * g * d1 * 32 * P.fwd_CPL * bsz + 15) / 16 * 16; };
    int chunk = std::max(1, std::min(32, (20 * 1024) / (P.cy_stride * bsz)));
    while (per_warp(chunk) * warps > budget && chunk > 1) chunk /= 2;
    if (per_warp(chunk) * warps > budget) {
      msg = "forward staging exceeds shared memory";
      return TP_EUNSUPPORTED;
    }
    P.fwd_chunk = chunk;
    P.fwd_ring_g = g;
    P.fwd_ring_off = base(chunk);
    P.fwd_warp_smem = per_warp(chunk);
  }
  // the same staging for the source pass of the backward (paths by input block)
  P.src_cy_stride = vw;
  P.in_tile_cost.clear();
  for (const TileD& t : P.in_tiles) {
    int off = 0, cost = 0;
    for (int k = t.pbeg; k < t.pend; ++k) {
      PathD& d = P.paths_by_in[k];
      auto e = real_cg_sparse(d.l1, d.l2, d.l3);
      std::vector<std::pair<int, int>> pairs;
      for (auto& q : e) pairs.emplace_back(q.m1, q.m3);
      std::sort(pairs.begin(), pairs.end());
      pairs.erase(std::unique(pairs.begin(), pairs.end()), pairs.end());
      d.cy_off = off;
      off += ((int)pairs.size() + vw - 1) / vw * vw;
      // per edge: the adjoint contraction (one FMA per (m1, m3) pair), x_bar and
      // h (2 per m1), w and the A_bar update (K each) and the radial row, the
      // m_bar components read from the ring
      cost += (int)pairs.size() + 2 * (2 * d.l1 + 1) + 3 * P.K + (2 * d.l3 + 1);
    }
    P.src_cy_stride = std::max(P.src_cy_stride, off);
    P.in_tile_cost.push_back(std::max(1, cost));
  }
  // the second-order source pass's 32-channel tiles, by the same per-edge count
  P.dbl_in_tile_cost.clear();
  for (const TileD& t : P.dbl_in_tiles) {
    int cost = 0;
    for (int k = t.pbeg; k < t.pend; ++k) {
      const PathD& d = P.dbl_paths_by_in[k];
      auto e = real_cg_sparse(d.l1, d.l2, d.l3);
      std::vector<std::pair<int, int>> pairs;
      for (auto& q : e) pairs.emplace_back(q.m1, q.m3);
      std::sort(pairs.begin(), pairs.end());
      pairs.erase(std::unique(pairs.begin(), pairs.end()), pairs.end());
      cost += (int)pairs.size() + 2 * (2 * d.l1 + 1) + 3 * P.K + (2 * d.l3 + 1);
    }
    P.dbl_in_tile_cost.push_back(std::max(1, cost));
  }
  // source pass: per warp, the staged chunk (receivers, radial rows, cY) and an
  // m_bar copy ring of two groups of ring_g edges (every component of the
  // widest output block, 32 lanes x CPL channels). Group size, then chunk,
  // shrink until one CTA of src_warps warps fits on an SM.
  {
    // the kernel sizes the ring for its degree profile's widest output block
    const int l3p = profs[P.prof][2], d3 = 2 * l3p + 1, warps = src_warps_for(bsz);
    const int budget = 226 * 1024 / ctas_per_sm_for(bsz);
    const int g = src_ring_g(bsz, P.CPL, l3p);
    auto base = [&](int chunk) { return (32 * 4 + 32 * P.KP * bsz + chunk * P.src_cy_stride * bsz + 15) / 16 * 16; };
    auto per_warp = [&](int chunk) { return base(chunk) + (2 * g * d3 * 32 * P.CPL * bsz + 15) / 16 * 16; };
    int chunk = std::max(1, std::min(32, (20 * 1024) / (P.src_cy_stride * bsz)));
    while (per_warp(chunk) * warps > budget && chunk > 1) chunk /= 2;
    if (per_warp(chunk) * warps > budget) {
      msg = "source-pass staging exceeds shared memory";
      return TP_EUNSUPPORTED;
    }
    P.src_chunk = chunk;
    P.src_ring_g = g;
    P.src_ring_off = base(chunk);
    P.src_warp_smem = per_warp(chunk);
    // split mode adds the warps' x_bar partials (widest input block of the profile)
    const int d1 = 2 * profs[P.prof][0] + 1;
    P.src_split_ok = (size_t)per_warp(chunk) * warps + (size_t)warps * d1 * 32 * P.CPL * bsz <= 227 * 1024;
  }
  if (mode == TP_UVW) {
    if ((int)P.bout.size() > kMaxBlocks || (int)P.bin.size() > kMaxBlocks) {
      msg = "more than " + std::to_string(kMaxBlocks) + " irrep blocks";
      return TP_EUNSUPPORTED;
    }
    // receiver state S (Sobek §4.2): per output block g, rows (receiver, m3),
    // columns (path of g, q, u); the mixing operand B_g packs A's rows in the
    // same (path, q, u) order
    long long s_off = 0, bf_off = 0;
    P.pack.K = P.K;
    P.pack.bf_uq = 0;
    P.pack.n_w = (int)P.n_w;
    P.pack.n_paths = (int)P.paths.size();
    for (size_t g = 0; g < P.bout.size(); ++g) {
      UvwBlockD b{};
      b.l = P.bout[g].l;
      b.pbeg = (int)P.paths_fwd.size();
      int cols = 0;
      for (int pi : by_out[g]) {
        const HostPath& h = P.paths[pi];
        PathD d{};
        d.l1 = (int8_t)h.l1; d.l2 = (int8_t)h.l2; d.l3 = (int8_t)h.l3;
        d.x_off = h.x_off; d.mul_in = h.mul_in; d.out_off = h.out_off; d.mul_out = h.mul_out;
        d.w_off = (int)h.w_off;
        d.col_off = cols;
        P.pack.paths[pi].w_off = (int)h.w_off;
        P.pack.paths[pi].mi = h.mul_in;
        P.pack.paths[pi].mo = h.mul_out;
        P.pack.paths[pi].colf = cols;
        P.pack.paths[pi].bf_off = bf_off;
        cols += P.K * h.mul_in;
        P.paths_fwd.push_back(d);
      }
      b.pend = (int)P.paths_fwd.size();
      b.dcols = cols;
      for (int pi : by_out[g]) P.pack.paths[pi].dcf = cols;
      b.s_off = s_off;
      b.out_off = P.bout[g].offset;
      b.mul_own = P.bout[g].mul;
      s_off += (long long)(2 * b.l + 1) * cols;
      bf_off += (long long)cols * P.bout[g].mul;
      P.uvw_out.push_back(b);
    }
    P.s_row_elems = s_off;
    // source state S' for x_bar: per input block b, rows (source, m1), columns
    // (path from b, q, w); B'_b packs A's rows in (path, q, w) order
    long long sa_off = 0, ba_off = 0;
    for (size_t b1 = 0; b1 < P.bin.size(); ++b1) {
      UvwBlockD b{};
      b.l = P.bin[b1].l;
      b.pbeg = (int)P.paths_adj.size();
      int cols = 0;
      for (int pi : by_in[b1]) {
        const HostPath& h = P.paths[pi];
        PathD d{};
        d.l1 = (int8_t)h.l1; d.l2 = (int8_t)h.l2; d.l3 = (int8_t)h.l3;
        d.x_off = h.out_off;            // gathered: the grad_out block of the path
        d.mul_in = h.mul_out;
        d.out_off = h.x_off; d.mul_out = h.mul_in;
        d.w_off = (int)h.w_off;
        d.col_off = cols;
        P.pack.paths[pi].cola = cols;
        P.pack.paths[pi].ba_off = ba_off;
        cols += P.K * h.mul_out;
        P.paths_adj.push_back(d);
      }
      b.pend = (int)P.paths_adj.size();
      b.dcols = cols;
      for (int pi : by_in[b1]) P.pack.paths[pi].dca = cols;
      b.s_off = sa_off;
      b.out_off = P.bin[b1].offset;
      b.mul_own = P.bin[b1].mul;
      sa_off += (long long)(2 * b.l + 1) * cols;
      ba_off += (long long)cols * P.bin[b1].mul;
      P.uvw_in.push_back(b);
    }
    P.sa_row_elems = sa_off;
    // tensor-core mixing: fp32, at most 256 channels per block (one 128 x N
    // accumulator in tensor memory; the ring shrinks to fit shared memory), state
    // rows whose width is a multiple of 4 (16-byte TMA strides)
    P.uvw_tc = dtype == TP_F32;
    for (auto& b : P.uvw_out) P.uvw_tc = P.uvw_tc && b.mul_own <= 256 && b.dcols % 4 == 0;
    for (auto& b : P.uvw_in) P.uvw_tc = P.uvw_tc && b.mul_own <= 256 && b.dcols % 4 == 0;
    const size_t bsz2 = dtype == TP_F32 ? 4 : 8;
    if ((size_t)std::max(P.s_row_elems, P.sa_row_elems) * bsz2 > P.state_budget) {
      msg = "one node's uvw state exceeds the state chunk budget";
      return TP_EUNSUPPORTED;
    }
  }
  return TP_OK;
}

int parse_sh_irreps(const char* s, int& sh_lmax, std::vector<int>& parity, std::string& msg) {
  std::vector<Block> b;
  if (!parse_irreps(s, b, msg)) return TP_EINVAL;
  parity.clear();
  for (size_t k = 0; k < b.size(); ++k) {
    if (b[k].l != (int)k || b[k].mul != 1) {
      msg = "spherical-harmonic irreps must be 1x0?+1x1?+... with degrees 0, 1, 2, ... in order";
      return TP_EINVAL;
    }
    parity.push_back(b[k].p);
  }
  sh_lmax = (int)b.size() - 1;
  return TP_OK;
}

int uvw_chunk_rows(const Plan& p, long long n_nodes, int dir) {
  const size_t b = p.dtype == TP_F32 ? 4 : 8;
  const long long per = std::max<long long>(1, (dir == 0 ? p.s_row_elems : p.sa_row_elems));
  long long r = (long long)(p.state_budget / (per * b));
  r = std::max<long long>(1, std::min<long long>(r, std::max<long long>(1, n_nodes)));
  return (int)r;
}

// CTAs per tile in proportion to cost: shares rounded down (at least one CTA
// each, at most cap), then the CTAs left over one at a time to the tile with the
// most cost per CTA. Returns the largest count.
long long deal_ctas(const std::vector<int>& cost, long long grid, long long cap, int* cta) {
  const int t = (int)cost.size();
  double tot = 0;
  for (int k = 0; k < t; ++k) tot += cost[k];
  std::vector<long long> c(t);
  long long used = 0, most = 0;
  for (int k = 0; k < t; ++k) {
    c[k] = std::min(cap, std::max<long long>(1, (long long)(grid * (cost[k] / tot))));
    used += c[k];
  }
  while (used < grid) {
    int best = -1;
    double bv = 0;
    for (int k = 0; k < t; ++k) {
      const double v = cost[k] / (double)c[k];
      if (c[k] < cap && v > bv) {
        bv = v;
        best = k;
      }
    }
    if (best < 0) break;
    ++c[best];
    ++used;
  }
  if (cta) cta[0] = 0;
  for (int k = 0; k < t; ++k) {
    most = std::max(most, c[k]);
    if (cta) cta[k + 1] = cta[k] + (int)c[k];
  }
  return most;
}

int uvu_dbl_src_partition(const Plan& p, long long n_nodes, int* cta) {
  const int t = (int)p.dbl_in_tiles.size();
  if (t == 0) {
    if (cta) cta[0] = 0;
    return 0;
  }
  // several waves of CTAs (the hardware hands the later ones to the SMs that
  // finish first), dealt to the tiles by cost
  const long long grid = std::max<long long>(t, 4LL * kSMs);
  const long long cap = std::max<long long>(1, (n_nodes + kDbWarps - 1) / kDbWarps);
  return (int)(deal_ctas(p.dbl_in_tile_cost, grid, cap, cta) * kDbWarps);
}

int uvu_src_partition(const Plan& p, long long n_nodes, long long max_slots, int* cta, int* split) {
  const int t = (int)p.in_tiles.size();
  if (split) *split = 1;
  if (t == 0) {
    if (cta) cta[0] = 0;
    return 0;
  }
  const int bsz = p.dtype == TP_F32 ? 4 : 8;
  const long long grid = std::max<long long>(t, (long long)kSMs * ctas_per_sm_for(bsz));
  // split mode while one warp per (source, tile) pair would not fill the
  // wave's warps
  const bool sp = p.src_split_ok && n_nodes * t <= grid * src_warps_for(bsz);
  if (split && sp) *split = src_warps_for(bsz);
  const long long w = sp ? 1 : src_warps_for(bsz);   // slots (source streams) per CTA
  const long long cap = std::max<long long>(1, (n_nodes + w - 1) / w);   // CTAs with a source for every stream
  const long long slots = deal_ctas(p.in_tile_cost, grid, cap, cta) * w;
  return (int)std::max<long long>(1, std::min(slots, max_slots));
}

size_t workspace_bytes(const Plan& p, long long n_nodes, int pass) {
  const size_t b = p.dtype == TP_F32 ? 4 : 8;
  size_t bytes = 0;
  if (p.mode == TP_UVU) {
    // first order: the source pass's slots; second order: its own source pass
    if (pass == 1) bytes = (size_t)uvu_src_partition(p, n_nodes, 1LL << 40, nullptr, nullptr) * p.K * p.n_w * b;
    if (pass >= 2) bytes = (size_t)uvu_dbl_src_partition(p, n_nodes, nullptr) * p.K * p.n_w * b;
  } else {
    // packed A (forward operand; plus adjoint operand and packed A_bar in the
    // backward), each 256-byte aligned, and one (forward) or two (backward)
    // state chunks
    const size_t a = ((size_t)p.K * p.n_w * b + 255) / 256 * 256;
    const size_t s0 = ((size_t)uvw_chunk_rows(p, n_nodes, 0) * p.s_row_elems * b + 255) / 256 * 256;
    const size_t s1 = ((size_t)uvw_chunk_rows(p, n_nodes, 1) * p.sa_row_elems * b + 255) / 256 * 256;
    // the tensor-core path adds the low parts of the transposed operands; the
    // backward adds the split-K partials of A_bar
    // the double backward packs A and its direction for all three products
    // (forward, source and S_bar operands; hi/lo on the tensor cores)
    const size_t na = pass == 0   ? (p.uvw_tc ? 2 : 1)
                      : pass == 1 ? (p.uvw_tc ? 4 : 3) + kTnSplits
                                  : 2 * (p.uvw_tc ? 5 : 3) + 1 + kTnSplits;
    bytes = na * a + (pass == 0 ? s0 : 2 * std::max(s0, s1));
  }
  return (bytes + 255) / 256 * 256;
}

void work_model(const Plan& p, long long N, long long E, int pass, double& flops, double& bytes) {
  const double b = p.dtype == TP_F32 ? 4.0 : 8.0;
  double fwd = 0, bwd = 0, dbl = 0;
  for (auto& h : p.paths) {
    const double d1 = 2 * h.l1 + 1, d3 = 2 * h.l3 + 1, nnz = h.nnz, K = p.K;
    if (p.mode == TP_UVU) {
      const double C = h.mul_in;
      fwd += 2.0 * E * C * (K + nnz + d3);
      bwd += 2.0 * E * C * (3 * K + 3 * nnz + 2 * d3);
      // second order: w, w_dot (3K); T, T_dot (3 nnz); m_dot (2 d3); h, h_dot
      // (2 d3); A_bar_dot, phi_bar_dot (4K); x_bar_dot (2 nnz + 2 d1); Y_bar_dot
      // (2 nnz)
      dbl += 2.0 * E * C * (7 * K + 7 * nnz + 4 * d3 + 2 * d1);
    } else {
      // state S (Eqs. 32-33) and mixing m = S A (Eqs. 34-35); the backward
      // recomputes S, forms A_bar = S^T m_bar and S_bar = m_bar A^T (Eq. 36),
      // runs the edge pass (C, T_bar, phi_bar, Y_bar), and builds and mixes the
      // source state of x_bar
      const double ci = h.mul_in, co = h.mul_out;
      const double e = E * (2 * ci * nnz + 2 * K * ci * d3);
      const double r = N * 2 * d3 * K * ci * co;
      fwd += e + r;
      bwd += e + 2 * r + E * (4 * K * ci * d3 + 4 * ci * nnz) + E * (2 * co * nnz + 2 * K * co * d1) +
             N * 2 * d1 * K * co * ci;
      // second order (Sobek §4.4): S and its directional state dS (C_dot, then
      // phi_dot C + phi C_dot); dm = dS A + S dA, dA_bar = dS^T m_bar,
      // S_bar = m_bar A^T, dS_bar = m_bar dA^T (5 mixing products); the edge pass
      // on (S_bar, dS_bar, C, C_dot); the source state S' and dS', and
      // x_bar_dot = dS' A' + S' dA'
      dbl += e + E * (4 * ci * nnz + 4 * K * ci * d3) + 5 * r + E * (10 * K * ci * d3 + 10 * ci * nnz) +
             E * (4 * co * nnz + 6 * K * co * d1) + 2 * N * 2 * d1 * K * co * ci;
    }
  }
  const double in_b = b * ((double)N * p.c_in + (double)E * p.dim_y + (double)E * p.K + (double)p.K * p.n_w);
  if (pass == 0) {
    flops = fwd;
    bytes = in_b + b * (double)N * p.c_out + 4.0 * E + 4.0 * (N + 1);
  } else if (pass == 1) {
    flops = bwd;
    bytes = in_b + b * ((double)N * p.c_out + (double)N * p.c_in + (double)E * p.dim_y + (double)E * p.K +
                        (double)p.K * p.n_w) +
            12.0 * E + 8.0 * (N + 1);
  } else {
    // inputs and their directions, grad_out; m_dot and the four directional adjoints
    flops = dbl;
    bytes = 3 * in_b + b * 2.0 * (double)N * p.c_out + 12.0 * E + 8.0 * (N + 1);
  }
}

}  // namespace tpc
