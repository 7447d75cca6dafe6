// Channelwise (uvu) second-order program of the CG tensor-product convolution.
//
// Along directions (x_dot, Y_dot, phi_dot, A_dot), with the output adjoint
// m_bar held fixed (Sobek §3.3; LunaTP Appendix F, Algorithm 3), per edge
// e = j -> i, path pi and channel u:
//   w      = sum_q phi_q A_q,        w_dot = sum_q phi_dot_q A_q + phi_q A_dot_q
//   T      = CG(x_j, Y_e),           T_dot = CG(x_dot_j, Y_e) + CG(x_j, Y_dot_e)
//   m_dot_i        += w_dot T + w T_dot
//   h      = <m_bar_i, T>,           h_dot = <m_bar_i, T_dot>
//   A_bar_dot_q    += phi_dot_q h + phi_q h_dot
//   phi_bar_dot_eq += A_dot_q h + A_q h_dot
//   x_bar_dot_j    += w_dot D_xT^*(Y_e) m_bar_i + w D_xT^*(Y_dot_e) m_bar_i
//   Y_bar_dot_e    += w_dot D_YT^*(x_j) m_bar_i + w D_YT^*(x_dot_j) m_bar_i
// Bilinearity of T means every term uses the forward's operands and CG
// coefficients; nothing edge-sized is stored. Ownership is that of the first
// backward (Sobek §4.3, §4.4):
//   * receiver pass: one warp per (receiver, 32-channel tile of an output
//     block); m_dot accumulates in registers over the receiver's CSR edges and
//     is stored once;
//   * edge pass: one lane per CSR edge; phi_bar_dot and Y_bar_dot accumulate in
//     that lane's registers over every path and channel (graphs too small to
//     fill the GPU share 32 edges among the warps of a CTA, paths dealt
//     round-robin, partial sums added in warp order);
//   * source pass: one warp per (source, 32-channel tile of an input block)
//     over the source view; x_bar_dot in registers, one fixed order; the same
//     sweep forms h and h_dot and adds A_bar_dot into the warp's own slot of a
//     fixed-size [slots, K, N_w] buffer, summed in slot order afterwards.
#include "common.cuh"
#include "kernels.h"

namespace tpc {
namespace {

constexpr long long kDbSplitGroups = 148LL * kDbWarps;   // 32-edge groups below which the edge pass splits

template <int L1M, int L2M, int L3M>
struct DProf {
  static constexpr int l1 = L1M, l2 = L2M, l3 = L3M;
};

template <int V, typename T>
__device__ __forceinline__ void ldv(T (&v)[V], const T* p) {
  if constexpr (V == 4 && sizeof(T) == 4) {
    const float4 t = __ldg(reinterpret_cast<const float4*>(p));
    v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
  } else if constexpr (V == 2 && sizeof(T) == 8) {
    const double2 t = __ldg(reinterpret_cast<const double2*>(p));
    v[0] = t.x; v[1] = t.y;
  } else {
#pragma unroll
    for (int c = 0; c < V; ++c) v[c] = __ldg(p + c);
  }
}

// ---------------------------------------------------------------- receiver pass

template <typename T, int KP, int L1, int L2, int L3>
__device__ __forceinline__ void recv_path(const UvuDbwdParams<T>& p, const PathD& pd, int e0, int e1, int ch,
                                          T (&acc)[2 * L3 + 1]) {
  using CGp = cgt::CG<L1, L2, L3>;
  constexpr int D1 = 2 * L1 + 1, D2 = 2 * L2 + 1, NP = CGp::npair, Y0 = L2 * L2;
  T a[KP], ad[KP];
#pragma unroll
  for (int q = 0; q < KP; ++q) {
    a[q] = q < p.K ? ldg(p.A + (size_t)q * p.n_w + pd.w_off + ch) : T(0);
    ad[q] = q < p.K ? ldg(p.dA + (size_t)q * p.n_w + pd.w_off + ch) : T(0);
  }
  const int mul = pd.mul_in;
  for (int e = e0; e < e1; ++e) {
    const int j = ldg(p.senders + e);
    if ((unsigned)j >= (unsigned)p.N) {   // uniform over the warp
      raise_error(p.err, kErrIndex);
      continue;
    }
    T w = T(0), wd = T(0);
#pragma unroll
    for (int q = 0; q < KP; ++q) {
      if (q < p.K) {
        const T ph = ldg(p.phi + (size_t)e * p.K + q), phd = ldg(p.dphi + (size_t)e * p.K + q);
        w = fma(ph, a[q], w);
        wd = fma(phd, a[q], fma(ph, ad[q], wd));
      }
    }
    T y[D2], yd[D2];
#pragma unroll
    for (int m = 0; m < D2; ++m) {
      y[m] = ldg(p.Y + (size_t)e * p.dim_y + Y0 + m);
      yd[m] = ldg(p.dY + (size_t)e * p.dim_y + Y0 + m);
    }
    const T* xr = p.x + (size_t)j * p.c_in + pd.x_off + ch;
    const T* xdr = p.dx + (size_t)j * p.c_in + pd.x_off + ch;
    // m_dot += sum cY (w_dot x + w x_dot) + sum cY_dot (w x)
    T u1[D1], u2[D1];
#pragma unroll
    for (int m = 0; m < D1; ++m) {
      const T xv = ldg(xr + m * mul), xdv = ldg(xdr + m * mul);
      u1[m] = fma(wd, xv, w * xdv);
      u2[m] = w * xv;
    }
    static_for<NP>([&](auto P) {
      constexpr int Pi = decltype(P)::value;
      constexpr Pair pr = CGp::pair[Pi];
      const T cy = pair_coef<T, CGp, Pi>(y), cyd = pair_coef<T, CGp, Pi>(yd);
      acc[pr.m3] = fma(cy, u1[pr.m1], fma(cyd, u2[pr.m1], acc[pr.m3]));
    });
  }
}

template <typename T, int KP, int L1M, int L2M, int L3>
__device__ __forceinline__ void recv_tile(const UvuDbwdParams<T>& p, const TileD& tl, int i, int lane) {
  constexpr int D3 = 2 * L3 + 1;
  T acc[D3];
#pragma unroll
  for (int m = 0; m < D3; ++m) acc[m] = T(0);
  const bool active = lane < tl.nch;
  const int ch = tl.ch0 + (active ? lane : 0);   // inactive lanes read a valid channel, never store
  int e0 = ldg(p.rowptr + i), e1 = ldg(p.rowptr + i + 1);
  if (e0 < 0 || e1 < e0 || e1 > p.E) {
    raise_error(p.err, kErrCsr);
    e1 = e0;
  }
  for (int pi = tl.pbeg; pi < tl.pend; ++pi) {
    const PathD& pd = p.paths[pi];
    dispatch_l1l2<L3, L1M, L2M>(pd.l1, pd.l2, [&](auto A1, auto A2) {
      recv_path<T, KP, decltype(A1)::value, decltype(A2)::value, L3>(p, pd, e0, e1, ch, acc);
    });
  }
  if (active) {
    T* o = p.mdot + (size_t)i * p.c_out + tl.off + ch;
#pragma unroll
    for (int m = 0; m < D3; ++m) o[(size_t)m * tl.mul] = acc[m];
  }
}

template <typename T, int KP, class PR>
__global__ void __launch_bounds__(kDbWarps * 32) uvu_dbwd_recv_kernel(const __grid_constant__ UvuDbwdParams<T> p) {
  const int lane = threadIdx.x & 31;
  const long long task = (long long)blockIdx.x * kDbWarps + (threadIdx.x >> 5);
  if (task >= (long long)p.N * p.n_tiles) return;
  const int i = (int)(task / p.n_tiles);
  const TileD& tl = p.tiles[(int)(task - (long long)i * p.n_tiles)];
  dispatch_l<PR::l3>(tl.l, [&](auto L) { recv_tile<T, KP, PR::l1, PR::l2, decltype(L)::value>(p, tl, i, lane); });
}

// ---------------------------------------------------------------- edge pass

template <typename T, int KP, int V, int DY, int L1, int L2, int L3>
__device__ __forceinline__ void edge_path(const UvuDbwdParams<T>& p, const PathD& pd, int e, int j, int i,
                                          const T (&ph)[KP], const T (&phd)[KP], T (&gphi)[KP], T (&gY)[DY]) {
  using CGp = cgt::CG<L1, L2, L3>;
  constexpr int D1 = 2 * L1 + 1, D2 = 2 * L2 + 1, D3 = 2 * L3 + 1, NP = CGp::npair, Y0 = L2 * L2;
  T y[D2], yd[D2];
#pragma unroll
  for (int m = 0; m < D2; ++m) {
    y[m] = ldg(p.Y + (size_t)e * p.dim_y + Y0 + m);
    yd[m] = ldg(p.dY + (size_t)e * p.dim_y + Y0 + m);
  }
  T cy[NP], cyd[NP];
  static_for<NP>([&](auto P) {
    cy[decltype(P)::value] = pair_coef<T, CGp, decltype(P)::value>(y);
    cyd[decltype(P)::value] = pair_coef<T, CGp, decltype(P)::value>(yd);
  });
  const int mul = pd.mul_in;
  const T* xr = p.x + (size_t)j * p.c_in + pd.x_off;
  const T* xdr = p.dx + (size_t)j * p.c_in + pd.x_off;
  const T* gr = p.gout + (size_t)i * p.c_out + pd.out_off;
  for (int u0 = 0; u0 < mul; u0 += V) {
    T a[KP][V], ad[KP][V], xv[D1][V], xdv[D1][V], gv[D3][V];
#pragma unroll
    for (int q = 0; q < KP; ++q) {
      if (q < p.K) {
        ldv<V>(a[q], p.A + (size_t)q * p.n_w + pd.w_off + u0);
        ldv<V>(ad[q], p.dA + (size_t)q * p.n_w + pd.w_off + u0);
      } else {
#pragma unroll
        for (int c = 0; c < V; ++c) a[q][c] = ad[q][c] = T(0);
      }
    }
#pragma unroll
    for (int m = 0; m < D1; ++m) {
      ldv<V>(xv[m], xr + m * mul + u0);
      ldv<V>(xdv[m], xdr + m * mul + u0);
    }
#pragma unroll
    for (int m = 0; m < D3; ++m) ldv<V>(gv[m], gr + m * mul + u0);
    T w[V], wd[V], h[V], hd[V];
#pragma unroll
    for (int c = 0; c < V; ++c) {
      w[c] = wd[c] = h[c] = hd[c] = T(0);
#pragma unroll
      for (int q = 0; q < KP; ++q) {
        w[c] = fma(ph[q], a[q][c], w[c]);
        wd[c] = fma(phd[q], a[q][c], fma(ph[q], ad[q][c], wd[c]));
      }
    }
    static_for<NP>([&](auto P) {
      constexpr int Pi = decltype(P)::value;
      constexpr Pair pr = CGp::pair[Pi];
      T z = T(0);
#pragma unroll
      for (int c = 0; c < V; ++c) {
        const T xg = xv[pr.m1][c] * gv[pr.m3][c], xdg = xdv[pr.m1][c] * gv[pr.m3][c];
        h[c] = fma(cy[Pi], xg, h[c]);
        hd[c] = fma(cyd[Pi], xg, fma(cy[Pi], xdg, hd[c]));
        z = fma(wd[c], xg, fma(w[c], xdg, z));
      }
      // Y_bar_dot[m2] += c sum_u (w_dot x[m1] + w x_dot[m1]) m_bar[m3]
      static_for<pr.n>([&](auto t) {
        constexpr Term tm = CGp::term[pr.start + decltype(t)::value];
        gY[Y0 + tm.m2] = fma(T(tm.c), z, gY[Y0 + tm.m2]);
      });
    });
#pragma unroll
    for (int q = 0; q < KP; ++q)
#pragma unroll
      for (int c = 0; c < V; ++c) gphi[q] = fma(ad[q][c], h[c], fma(a[q][c], hd[c], gphi[q]));
  }
}

template <typename T, int KP, int V, class PR>
__global__ void __launch_bounds__(kDbWarps * 32) uvu_dbwd_edge_kernel(const __grid_constant__ UvuDbwdParams<T> p) {
  constexpr int DY = (PR::l2 + 1) * (PR::l2 + 1);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const bool split = p.split > 1;
  const long long e0 = split ? (long long)blockIdx.x * 32 : ((long long)blockIdx.x * kDbWarps + warp) * 32;
  if (e0 >= p.E) return;   // uniform over the CTA in split mode
  const int e = (int)(e0 + lane);
  const bool live = e < p.E;
  int i = 0, j = 0;
  bool ok = false;
  if (live) {
    int lo = 0, hi = p.N;   // receiver of CSR position e: the last i with rowptr[i] <= e
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (ldg(p.rowptr + mid) <= e) lo = mid; else hi = mid;
    }
    i = lo;
    j = ldg(p.senders + e);
    ok = (unsigned)j < (unsigned)p.N;
    if (!ok) {
      atomicOr(p.err, kErrIndex);
      j = 0;
    }
  }
  T ph[KP], phd[KP], gphi[KP], gY[DY];
#pragma unroll
  for (int q = 0; q < KP; ++q) {
    ph[q] = (live && q < p.K) ? ldg(p.phi + (size_t)e * p.K + q) : T(0);
    phd[q] = (live && q < p.K) ? ldg(p.dphi + (size_t)e * p.K + q) : T(0);
    gphi[q] = T(0);
  }
#pragma unroll
  for (int m = 0; m < DY; ++m) gY[m] = T(0);
  if (live) {
    for (int pi = split ? warp : 0; pi < p.n_paths; pi += split ? p.split : 1) {
      const PathD& pd = p.paths[pi];
      dispatch_l<PR::l1>(pd.l1, [&](auto A1) {
        constexpr int L1 = decltype(A1)::value;
        static_for<PR::l2 + 1>([&](auto A2) {
          static_for<PR::l3 + 1>([&](auto A3) {
            constexpr int L2 = decltype(A2)::value, L3 = decltype(A3)::value;
            if constexpr (triangle(L1, L2, L3)) {
              if (pd.l2 == L2 && pd.l3 == L3)
                edge_path<T, KP, V, DY, L1, L2, L3>(p, pd, e, j, i, ph, phd, gphi, gY);
            }
          });
        });
      });
    }
    if (!ok) {
#pragma unroll
      for (int q = 0; q < KP; ++q) gphi[q] = T(0);
#pragma unroll
      for (int m = 0; m < DY; ++m) gY[m] = T(0);
    }
  }
  if (split) {
    // add the warps' partial sums in warp order: red[warp][v][lane]
    extern __shared__ __align__(16) unsigned char smem_raw[];
    T* red = reinterpret_cast<T*>(smem_raw);
    const int nv = p.K + p.dim_y;
    T* mine = red + (size_t)warp * nv * 32 + lane;
#pragma unroll
    for (int q = 0; q < KP; ++q)
      if (q < p.K) mine[q * 32] = gphi[q];
#pragma unroll
    for (int m = 0; m < DY; ++m)
      if (m < p.dim_y) mine[(p.K + m) * 32] = gY[m];
    __syncthreads();
    for (int t = threadIdx.x; t < nv * 32; t += blockDim.x) {
      const int v = t >> 5, sl = t & 31;
      const long long eo = e0 + sl;
      if (eo >= p.E) continue;
      T acc = red[(size_t)v * 32 + sl];
      for (int w = 1; w < p.split; ++w) acc += red[((size_t)w * nv + v) * 32 + sl];
      if (v < p.K) p.gphi[(size_t)eo * p.K + v] = acc;
      else p.gY[(size_t)eo * p.dim_y + (v - p.K)] = acc;
    }
  } else if (live) {
#pragma unroll
    for (int q = 0; q < KP; ++q)
      if (q < p.K) p.gphi[(size_t)e * p.K + q] = gphi[q];
#pragma unroll
    for (int m = 0; m < DY; ++m)
      if (m < p.dim_y) p.gY[(size_t)e * p.dim_y + m] = gY[m];
  }
}

// ---------------------------------------------------------------- source pass

template <typename T, int KP, int L1, int L2, int L3>
__device__ __forceinline__ void src_path(const UvuDbwdParams<T>& p, const PathD& pd, int k0, int k1, int slot,
                                         int ch, bool active, const T (&xs)[2 * L1 + 1],
                                         const T (&xds)[2 * L1 + 1], T (&gx)[2 * L1 + 1]) {
  using CGp = cgt::CG<L1, L2, L3>;
  constexpr int D1 = 2 * L1 + 1, D2 = 2 * L2 + 1, D3 = 2 * L3 + 1, NP = CGp::npair, Y0 = L2 * L2;
  T a[KP], ad[KP], ab[KP];
#pragma unroll
  for (int q = 0; q < KP; ++q) {
    a[q] = q < p.K ? ldg(p.A + (size_t)q * p.n_w + pd.w_off + ch) : T(0);
    ad[q] = q < p.K ? ldg(p.dA + (size_t)q * p.n_w + pd.w_off + ch) : T(0);
    ab[q] = T(0);
  }
  const int mo = pd.mul_out;
  for (int k = k0; k < k1; ++k) {
    const int e = ldg(p.srcedge + k), i = ldg(p.srcrecv + k);
    if ((unsigned)e >= (unsigned)p.E || (unsigned)i >= (unsigned)p.N) {   // uniform over the warp
      raise_error(p.err, kErrIndex);
      continue;
    }
    T ph[KP], phd[KP], w = T(0), wd = T(0);
#pragma unroll
    for (int q = 0; q < KP; ++q) {
      ph[q] = q < p.K ? ldg(p.phi + (size_t)e * p.K + q) : T(0);
      phd[q] = q < p.K ? ldg(p.dphi + (size_t)e * p.K + q) : T(0);
      w = fma(ph[q], a[q], w);
      wd = fma(phd[q], a[q], fma(ph[q], ad[q], wd));
    }
    T y[D2], yd[D2];
#pragma unroll
    for (int m = 0; m < D2; ++m) {
      y[m] = ldg(p.Y + (size_t)e * p.dim_y + Y0 + m);
      yd[m] = ldg(p.dY + (size_t)e * p.dim_y + Y0 + m);
    }
    T gv[D3];
    const T* gr = p.gout + (size_t)i * p.c_out + pd.out_off + ch;
#pragma unroll
    for (int m = 0; m < D3; ++m) gv[m] = ldg(gr + m * mo);
    // B^x[m1] = sum cY m_bar[m3], its derivative along Y_dot uses cY_dot
    T tp[D1], tdp[D1];
#pragma unroll
    for (int m = 0; m < D1; ++m) tp[m] = tdp[m] = T(0);
    static_for<NP>([&](auto P) {
      constexpr int Pi = decltype(P)::value;
      constexpr Pair pr = CGp::pair[Pi];
      tp[pr.m1] = fma(pair_coef<T, CGp, Pi>(y), gv[pr.m3], tp[pr.m1]);
      tdp[pr.m1] = fma(pair_coef<T, CGp, Pi>(yd), gv[pr.m3], tdp[pr.m1]);
    });
    T h = T(0), hd = T(0);
    static_for<D1>([&](auto M) {
      constexpr int m1 = decltype(M)::value;
      if constexpr (has_m1<CGp>(m1)) {
        gx[m1] = fma(wd, tp[m1], fma(w, tdp[m1], gx[m1]));
        h = fma(xs[m1], tp[m1], h);
        hd = fma(xds[m1], tp[m1], fma(xs[m1], tdp[m1], hd));
      }
    });
#pragma unroll
    for (int q = 0; q < KP; ++q) ab[q] = fma(phd[q], h, fma(ph[q], hd, ab[q]));
  }
  if (active && k1 > k0) {
#pragma unroll
    for (int q = 0; q < KP; ++q)
      if (q < p.K) p.apart[((size_t)slot * p.K + q) * p.n_w + pd.w_off + ch] += ab[q];
  }
}

template <typename T, int KP, class PR, int L1>
__device__ __forceinline__ void src_tile(const UvuDbwdParams<T>& p, const TileD& tl, int slot, int stride, int lane) {
  constexpr int D1 = 2 * L1 + 1;
  const bool active = lane < tl.nch;
  const int ch = tl.ch0 + (active ? lane : 0);
  for (int j = slot; j < p.N; j += stride) {
    int k0 = ldg(p.colptr + j), k1 = ldg(p.colptr + j + 1);
    if (k0 < 0 || k1 < k0 || k1 > p.E) {
      raise_error(p.err, kErrCsr);
      k1 = k0;
    }
    T xs[D1], xds[D1], gx[D1];
    const T* xr = p.x + (size_t)j * p.c_in + tl.off + ch;
    const T* xdr = p.dx + (size_t)j * p.c_in + tl.off + ch;
#pragma unroll
    for (int m = 0; m < D1; ++m) {
      xs[m] = ldg(xr + m * tl.mul);
      xds[m] = ldg(xdr + m * tl.mul);
      gx[m] = T(0);
    }
    for (int pi = tl.pbeg; pi < tl.pend; ++pi) {
      const PathD& pd = p.paths[pi];
      dispatch_l2l3<L1, PR::l2>(pd.l2, pd.l3, [&](auto A2, auto A3) {
        if constexpr (decltype(A3)::value <= PR::l3)
          src_path<T, KP, L1, decltype(A2)::value, decltype(A3)::value>(p, pd, k0, k1, slot, ch, active, xs, xds,
                                                                        gx);
      });
    }
    if (active) {
      T* o = p.gx + (size_t)j * p.c_in + tl.off + ch;
#pragma unroll
      for (int m = 0; m < D1; ++m) o[(size_t)m * tl.mul] = gx[m];
    }
  }
}

template <typename T, int KP, class PR>
__global__ void __launch_bounds__(kDbWarps * 32) uvu_dbwd_src_kernel(const __grid_constant__ UvuDbwdParams<T> p) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  // the host deals the CTAs to the tiles in proportion to their per-edge cost
  int tile = 0;
  while (tile + 1 < p.n_tiles && (int)blockIdx.x >= p.tile_cta[tile + 1]) ++tile;
  if (tile >= p.n_tiles || (int)blockIdx.x >= p.tile_cta[tile + 1]) return;
  const int stride = min((p.tile_cta[tile + 1] - p.tile_cta[tile]) * kDbWarps, p.n_slots);
  const int slot = ((int)blockIdx.x - p.tile_cta[tile]) * kDbWarps + warp;
  if (slot >= stride) return;
  const TileD& tl = p.tiles[tile];
  dispatch_l<PR::l1>(tl.l, [&](auto L) { src_tile<T, KP, PR, decltype(L)::value>(p, tl, slot, stride, lane); });
}

// Wide: the degree-6 profile is compiled (fp32, K <= 8, scalar gathers only).
template <bool Wide, typename F>
cudaError_t by_prof(int prof, F&& f) {
  switch (prof) {
    case 0: return f(DProf<2, 2, 2>{});
    case 1: return f(DProf<1, 3, 3>{});
    case 2: return f(DProf<3, 3, 3>{});
    case 3: return f(DProf<4, 4, 4>{});
    default:
      if constexpr (Wide) return f(DProf<6, 6, 6>{});
      return cudaErrorInvalidValue;
  }
}

template <typename T, int KP>
constexpr bool wide_ok() { return std::is_same<T, float>::value && KP == 8; }

}  // namespace

// One channel per lane (CPL = 1): wider lanes measured slower (register spills
// in the source pass, no gain in the receiver pass).
template <typename T, int KP, int CPL>
cudaError_t launch_uvu_dbwd_recv(const UvuDbwdParams<T>& p, int prof, cudaStream_t s) {
  static_assert(CPL == 1, "the second-order passes run one channel per lane");
  const long long tasks = (long long)p.N * p.n_tiles;
  if (tasks == 0) return cudaSuccess;
  const unsigned blocks = (unsigned)((tasks + kDbWarps - 1) / kDbWarps);
  return by_prof<wide_ok<T, KP>()>(prof, [&](auto PR) {
    uvu_dbwd_recv_kernel<T, KP, decltype(PR)><<<blocks, kDbWarps * 32, 0, s>>>(p);
    return cudaGetLastError();
  });
}

template <typename T, int KP, int V>
cudaError_t launch_uvu_dbwd_edge(const UvuDbwdParams<T>& p0, int prof, cudaStream_t s) {
  if (p0.N == 0 || p0.E == 0) return cudaSuccess;
  UvuDbwdParams<T> p = p0;
  const long long groups = ((long long)p.E + 31) / 32;
  p.split = groups < kDbSplitGroups ? kDbWarps : 1;
  const unsigned blocks = (unsigned)(p.split > 1 ? groups : (groups + kDbWarps - 1) / kDbWarps);
  const size_t smem = p.split > 1 ? sizeof(T) * (size_t)kDbWarps * (p.K + p.dim_y) * 32 : 0;
  return by_prof<wide_ok<T, KP>() && V == 1>(prof, [&](auto PR) {
    auto kern = uvu_dbwd_edge_kernel<T, KP, V, decltype(PR)>;
    static SmemLimit limit;
    if (cudaError_t e = limit.ensure((const void*)kern, smem); e != cudaSuccess) return e;
    kern<<<blocks, kDbWarps * 32, smem, s>>>(p);
    return cudaGetLastError();
  });
}

template <typename T, int KP, int CPL>
cudaError_t launch_uvu_dbwd_src(const UvuDbwdParams<T>& p, int prof, cudaStream_t s) {
  static_assert(CPL == 1, "the second-order passes run one channel per lane");
  cudaError_t err = cudaMemsetAsync(p.apart, 0, sizeof(T) * (size_t)p.n_slots * p.K * p.n_w, s);
  if (err != cudaSuccess) return err;
  if (p.n_slots == 0 || p.n_tiles == 0 || p.N == 0) return cudaSuccess;
  const unsigned blocks = (unsigned)p.tile_cta[p.n_tiles];
  return by_prof<wide_ok<T, KP>()>(prof, [&](auto PR) {
    uvu_dbwd_src_kernel<T, KP, decltype(PR)><<<blocks, kDbWarps * 32, 0, s>>>(p);
    return cudaGetLastError();
  });
}

#define TPC_INST_R(T, KP) \
  template cudaError_t launch_uvu_dbwd_recv<T, KP, 1>(const UvuDbwdParams<T>&, int, cudaStream_t);
#define TPC_INST_S(T, KP) \
  template cudaError_t launch_uvu_dbwd_src<T, KP, 1>(const UvuDbwdParams<T>&, int, cudaStream_t);
#define TPC_INST_E(T, KP, V) \
  template cudaError_t launch_uvu_dbwd_edge<T, KP, V>(const UvuDbwdParams<T>&, int, cudaStream_t);
#if TPC_WANT(0)
TPC_INST_R(float, 8)
#endif
#if TPC_WANT(1)
TPC_INST_S(float, 8)
#endif
#if TPC_WANT(2)
TPC_INST_E(float, 8, 1)
#endif
#if TPC_WANT(3)
TPC_INST_E(float, 8, 4)
#endif
#if TPC_WANT(4)
TPC_INST_R(float, 16)
TPC_INST_S(float, 16)
#endif
#if TPC_WANT(5)
TPC_INST_E(float, 16, 1)
TPC_INST_E(float, 16, 4)
#endif
#if TPC_WANT(6)
TPC_INST_R(double, 8)
TPC_INST_S(double, 8)
#endif
#if TPC_WANT(7)
TPC_INST_E(double, 8, 1)
TPC_INST_E(double, 8, 2)
#endif
#if TPC_WANT(8)
TPC_INST_R(double, 16)
TPC_INST_S(double, 16)
#endif
#if TPC_WANT(9)
TPC_INST_E(double, 16, 1)
TPC_INST_E(double, 16, 2)
#endif
#undef TPC_INST_R
#undef TPC_INST_S
#undef TPC_INST_E

}  // namespace tpc
