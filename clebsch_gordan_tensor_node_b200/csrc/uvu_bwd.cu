// Channelwise (uvu) first backward of the CG tensor-product convolution.
//
// Adjoints (Sobek §3.2; LunaTP Appendix F, Algorithm 2), with m_bar = grad_out:
//   h_{e,pi,u}      = < m_bar_i[pi], T_{pi,u}(x_j, Y_e) >
//   A_bar_{q,pi,u}  = sum_e phi_{e,q} h_{e,pi,u}
//   phi_bar_{e,q}   = sum_{pi,u} A_{q,pi,u} h_{e,pi,u}
//   x_bar_j         = sum_{e: src=j} sum_{pi,u} w_{e,pi,u} D_x T^* m_bar_i
//   Y_bar_e         = sum_{pi,u} w_{e,pi,u} D_Y T^* m_bar_i
// h is consumed where it is formed; no W_bar tensor or edge chunk of it exists
// (Sobek §3.2, §4.3). Ownership follows Sobek §4.3 and LunaTP §4.4:
//   * edge pass: one warp per receiver walks its CSR edges; for each edge it
//     sweeps every path and channel, keeps per-lane partials of phi_bar_e and
//     Y_bar_e in registers, reduces them across the warp once, and writes them
//     (each edge has one owner, no cross-edge reduction);
//   * source pass: one warp per (source j, input block, channel tile) walks the
//     source-CSR view, accumulates x_bar_j in registers (one fixed order, no
//     atomics) and, because the same sweep forms h, the A_bar contributions,
//     which it adds into its own slot of a fixed-size partial buffer
//     [slots, K, N_w] (independent of E);
//   * reduce: A_bar = sum over slots in slot order.
#include "common.cuh"
#include "kernels.h"

namespace tpc {
namespace {

constexpr long long kSplitEdgeGroups = 148LL * kWarpsPerBlock;   // 32-edge groups below which paths split

// ---------------------------------------------------------------- edge pass
//
// One lane owns one edge: a warp takes 32 consecutive CSR edges (of any
// receivers), so phi_bar_e and Y_bar_e accumulate in the owning lane's
// registers over every path and channel and need no cross-lane reduction. Per
// path the lane contracts its Y block with the CG pairs once (cY); the channel
// loop then reads A as a warp-uniform 16-byte broadcast and x_j, m_bar_i as
// per-lane 16-byte gathers, V channels at a time.
//
// Graphs with few edges would leave most SMs idle that way, so there all the
// warps of a CTA share one group of 32 edges and deal the paths round-robin;
// their partial sums are added in warp order in shared memory (split mode).

template <int L1M, int L2M, int L3M>
struct Prof {
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
  } else if constexpr (V == 2 && sizeof(T) == 4) {
    const float2 t = __ldg(reinterpret_cast<const float2*>(p));
    v[0] = t.x; v[1] = t.y;
  } else {
#pragma unroll
    for (int c = 0; c < V; ++c) v[c] = __ldg(p + c);
  }
}

template <typename T, int KP, int V, int DY, int L1, int L2, int L3>
__device__ __forceinline__ void edge_path(const UvuEdgeParams<T>& p, const PathD& pd, int e, int j, int i,
                                          const T (&ph)[KP], T (&gphi)[KP], T (&gY)[DY]) {
  using CGp = cgt::CG<L1, L2, L3>;
  constexpr int D1 = 2 * L1 + 1, D2 = 2 * L2 + 1, D3 = 2 * L3 + 1, NP = CGp::npair, Y0 = L2 * L2;
  T y[D2];
#pragma unroll
  for (int m = 0; m < D2; ++m) y[m] = ldg(p.Y + (size_t)e * p.dim_y + Y0 + m);
  T cy[NP];
  static_for<NP>([&](auto P) { cy[decltype(P)::value] = pair_coef<T, CGp, decltype(P)::value>(y); });
  const int mul = pd.mul_in;
  const T* xr = p.x + (size_t)j * p.c_in + pd.x_off;
  const T* gr = p.gout + (size_t)i * p.c_out + pd.out_off;
  const T* ar = p.A + pd.w_off;
  for (int u0 = 0; u0 < mul; u0 += V) {
    T a[KP][V], xv[D1][V], gv[D3][V];
#pragma unroll
    for (int q = 0; q < KP; ++q) {
      if (q < p.K) {
        ldv<V>(a[q], ar + (size_t)q * p.n_w + u0);
      } else {
#pragma unroll
        for (int c = 0; c < V; ++c) a[q][c] = T(0);
      }
    }
#pragma unroll
    for (int m = 0; m < D1; ++m) ldv<V>(xv[m], xr + m * mul + u0);
#pragma unroll
    for (int m = 0; m < D3; ++m) ldv<V>(gv[m], gr + m * mul + u0);
    T w[V], h[V];
#pragma unroll
    for (int c = 0; c < V; ++c) {
      w[c] = ph[0] * a[0][c];
#pragma unroll
      for (int q = 1; q < KP; ++q) w[c] = fma(ph[q], a[q][c], w[c]);
      h[c] = T(0);
    }
    static_for<NP>([&](auto P) {
      constexpr int Pi = decltype(P)::value;
      constexpr Pair pr = CGp::pair[Pi];
      T z = T(0);
#pragma unroll
      for (int c = 0; c < V; ++c) {
        const T xg = xv[pr.m1][c] * gv[pr.m3][c];
        h[c] = fma(cy[Pi], xg, h[c]);
        z = fma(w[c], xg, z);
      }
      // Y_bar[m2] += c * sum_u w x[m1] m_bar[m3]
      static_for<pr.n>([&](auto t) {
        constexpr Term tm = CGp::term[pr.start + decltype(t)::value];
        gY[Y0 + tm.m2] = fma(T(tm.c), z, gY[Y0 + tm.m2]);
      });
    });
#pragma unroll
    for (int q = 0; q < KP; ++q)
#pragma unroll
      for (int c = 0; c < V; ++c) gphi[q] = fma(a[q][c], h[c], gphi[q]);
  }
}

// fp32 up to degree 2: at most 128 registers, so that two CTAs (16 warps)
// share an SM (a few spilled values); the wider profiles would spill kilobytes
// under that cap and keep one CTA
template <typename T, int KP, int V, class PR>
__global__ void __launch_bounds__(kWarpsPerBlock * 32, sizeof(T) == 4 && PR::l3 <= 2 ? 2 : 1)
uvu_edge_kernel(const __grid_constant__ UvuEdgeParams<T> p) {
  constexpr int DY = (PR::l2 + 1) * (PR::l2 + 1);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const bool split = p.split > 1;
  const long long e0 = split ? (long long)blockIdx.x * 32 : ((long long)blockIdx.x * kWarpsPerBlock + warp) * 32;
  if (e0 >= p.E) return;   // uniform over the CTA in split mode
  const int e = (int)(e0 + lane);
  const bool live = e < p.E;
  // receiver of CSR position e: the last i with rowptr[i] <= e
  int i = 0;
  int j = 0;
  bool ok = false;
  if (live) {
    int lo = 0, hi = p.N;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (ldg(p.rowptr + mid) <= e) lo = mid; else hi = mid;
    }
    i = lo;
    j = ldg(p.senders + e);
    ok = (unsigned)j < (unsigned)p.N;
    if (!ok) atomicOr(p.err, kErrIndex);
    if (!ok) j = 0;
  }
  T ph[KP], gphi[KP], gY[DY];
#pragma unroll
  for (int q = 0; q < KP; ++q) {
    ph[q] = (live && q < p.K) ? ldg(p.phi + (size_t)e * p.K + q) : T(0);
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
              if (pd.l2 == L2 && pd.l3 == L3) edge_path<T, KP, V, DY, L1, L2, L3>(p, pd, e, j, i, ph, gphi, gY);
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
//
// The forward's structure on the source view: a warp owns (source j, input
// block b, channel tile); per chunk of up to 32 outgoing edges, lanes first
// stage each edge's receiver, radial row and the cY values of every path of b
// in shared memory; then every path sweeps the chunk with A in registers and
// the receivers' m_bar rows arriving through an asynchronous copy ring. x_bar_j
// accumulates in registers in one fixed order; the same sweep forms
// h = <x_j, t'> and adds phi h to the warp's slot of the A_bar partial buffer
// (read at the start of the path, so that its latency overlaps the first copy
// group's, and written back at the end). The tiles differ in cost (their
// paths' pair counts and degrees), so the host deals the CTAs of the single
// wave to them in proportion to it; each warp of tile t serves every
// (CTAs of t x warps)-th source. On graphs with too few (source, tile) pairs
// to fill the GPU (split mode) the warps of a CTA share each source instead and
// deal the tile's paths; their x_bar partials are added in warp order in shared
// memory, and the CTA owns the slot (its warps write the columns of their own
// paths).

template <typename T>
struct SrcSmem {
  int* i;
  T* phi;
  T* cy;
  T* ring;   // [2][G][2 lmax_out + 1][32 CPL] m_bar rows in flight
};


template <typename T, int L1, int L2, int L3>
__device__ __forceinline__ void src_stage_cy(const T* yrow, T* dst) {
  using CGp = cgt::CG<L1, L2, L3>;
  T y[2 * L2 + 1];
#pragma unroll
  for (int m = 0; m < 2 * L2 + 1; ++m) y[m] = ldg(yrow + L2 * L2 + m);
  static_for<CGp::npair>([&](auto P) { dst[decltype(P)::value] = pair_coef<T, CGp, decltype(P)::value>(y); });
}

template <typename T>
__device__ __forceinline__ void lds16(T* v, const T* src) {
  if constexpr (sizeof(T) == 4) {
    const float4 t = *reinterpret_cast<const float4*>(src);
    v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
  } else {
    const double2 t = *reinterpret_cast<const double2*>(src);
    v[0] = t.x; v[1] = t.y;
  }
}

// Plain (coherent) load of CPL consecutive scalars that this kernel writes.
template <int CPL, typename T>
__device__ __forceinline__ void load_rw(T (&v)[CPL], const T* p) {
  if constexpr (CPL == 2 && std::is_same<T, float>::value) {
    const float2 t = *reinterpret_cast<const float2*>(p);
    v[0] = t.x; v[1] = t.y;
  } else {
#pragma unroll
    for (int c = 0; c < CPL; ++c) v[c] = p[c];
  }
}

template <typename T, int KP, int CPL, int G, int L1, int L2, int L3>
__device__ __forceinline__ void src_path(const UvuSrcParams<T>& p, const PathD& pd, const SrcSmem<T>& s, int n,
                                         int slot, int chl, bool active, const T (&xs)[2 * L1 + 1][CPL],
                                         T (&gx)[2 * L1 + 1][CPL]) {
  using CGp = cgt::CG<L1, L2, L3>;
  constexpr int D1 = 2 * L1 + 1, D3 = 2 * L3 + 1, NP = CGp::npair;
  constexpr int VW = sizeof(T) == 4 ? 4 : 2;
  T* adst = p.apart + (size_t)slot * p.K * p.n_w + pd.w_off + chl;
  T a[KP][CPL], ab[KP][CPL];
#pragma unroll
  for (int q = 0; q < KP; ++q) {
    if (q < p.K) {
      load_ch<CPL>(a[q], p.A + (size_t)q * p.n_w + pd.w_off + chl);
      if (active) {
        load_rw<CPL>(ab[q], adst + (size_t)q * p.n_w);
      } else {
#pragma unroll
        for (int c = 0; c < CPL; ++c) ab[q][c] = T(0);
      }
    } else {
#pragma unroll
      for (int c = 0; c < CPL; ++c) a[q][c] = ab[q][c] = T(0);
    }
  }
  // m_bar rows of the chunk's receivers go through a two-buffer ring of groups
  // of G edges: the copies of group g + 1 are in flight while group g is
  // contracted. Each lane copies and later reads only its own channels.
  const T* gb = p.gout + pd.out_off + chl;
  const int mo = pd.mul_out, lane = threadIdx.x & 31;
  constexpr int RW = 32 * CPL;   // ring row: one component of one edge
  auto issue = [&](int g0, int buf) {
#pragma unroll
    for (int t = 0; t < G; ++t) {
      if (g0 + t < n) {
        const T* gr = gb + (size_t)s.i[g0 + t] * p.c_out;
        T* dst = s.ring + ((buf * G + t) * D3) * RW + lane * CPL;
#pragma unroll
        for (int m = 0; m < D3; ++m) cp_async_b<CPL * sizeof(T)>(dst + m * RW, gr + m * mo);
      }
    }
  };
  if (n > 0) issue(0, 0);
  cp_commit();
  for (int g0 = 0, buf = 0; g0 < n; g0 += G, buf ^= 1) {
    if (g0 + G < n) issue(g0 + G, buf ^ 1);
    cp_commit();
    cp_wait<1>();   // this group's rows have landed
    const int tn = min(G, n - g0);
#pragma unroll 1
  for (int t = 0; t < tn; ++t) {
    const int k = g0 + t;
    T gv[D3][CPL];
    {
      const T* src = s.ring + ((buf * G + t) * D3) * RW + lane * CPL;
#pragma unroll
      for (int m = 0; m < D3; ++m) {
        if constexpr (CPL == 2 && sizeof(T) == 4) {
          const float2 v2 = *reinterpret_cast<const float2*>(src + m * RW);
          gv[m][0] = v2.x; gv[m][1] = v2.y;
        } else {
#pragma unroll
          for (int c = 0; c < CPL; ++c) gv[m][c] = src[m * RW + c];
        }
      }
    }
    T ph[KP];
#pragma unroll
    for (int q = 0; q < KP; q += VW) lds16(ph + q, s.phi + k * KP + q);
    const T* cyr = s.cy + k * p.cy_stride + pd.cy_off;
    T w[CPL];
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
      w[c] = ph[0] * a[0][c];
#pragma unroll
      for (int q = 1; q < KP; ++q) w[c] = fma(ph[q], a[q][c], w[c]);
    }
    // t'[m1] = sum_{m3} cY[m1][m3] m_bar[m3]   (D_x T^* applied to m_bar)
    T tp[D1][CPL];
    T cyv[VW];
    static_for<NP>([&](auto P) {
      constexpr int Pi = decltype(P)::value;
      constexpr Pair pr = CGp::pair[Pi];
      if constexpr (Pi % VW == 0) lds16(cyv, cyr + Pi);
#pragma unroll
      for (int c = 0; c < CPL; ++c) {
        if constexpr (first_m1<CGp>(Pi))
          tp[pr.m1][c] = cyv[Pi % VW] * gv[pr.m3][c];
        else
          tp[pr.m1][c] = fma(cyv[Pi % VW], gv[pr.m3][c], tp[pr.m1][c]);
      }
    });
    T h[CPL];
#pragma unroll
    for (int c = 0; c < CPL; ++c) h[c] = T(0);
    static_for<D1>([&](auto M) {
      constexpr int m1 = decltype(M)::value;
      if constexpr (has_m1<CGp>(m1)) {
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
          gx[m1][c] = fma(w[c], tp[m1][c], gx[m1][c]);
          h[c] = fma(xs[m1][c], tp[m1][c], h[c]);
        }
      }
    });
#pragma unroll
    for (int q = 0; q < KP; ++q)
#pragma unroll
      for (int c = 0; c < CPL; ++c) ab[q][c] = fma(ph[q], h[c], ab[q][c]);
  }
  }
  cp_wait<0>();
  if (active) {
#pragma unroll
    for (int q = 0; q < KP; ++q)
      if (q < p.K) store_ch<CPL>(adst + (size_t)q * p.n_w, ab[q]);
  }
}

// One warp's share of one input-block tile: sources slot, slot + stride, ...,
// and the paths pbeg + pw, pbeg + pw + ps, ... of each.
template <typename T, int KP, int CPL, class PR, int L1>
__device__ __forceinline__ void src_tile(const UvuSrcParams<T>& p, const TileD& tl, int slot, int stride,
                                         int lane, const SrcSmem<T>& s, int pw, int ps) {
  constexpr int D1 = 2 * L1 + 1;
  const bool active = lane * CPL < tl.nch;
  const int chl = tl.ch0 + (active ? lane * CPL : 0);
  for (int j = slot; j < p.N; j += stride) {
    int k0 = ldg(p.colptr + j), k1 = ldg(p.colptr + j + 1);
    if (k0 < 0 || k1 < k0 || k1 > p.E) {
      raise_error(p.err, kErrCsr);
      k1 = k0;
    }
    T xs[D1][CPL], gx[D1][CPL];
    const T* xr = p.x + (size_t)j * p.c_in + tl.off + chl;
#pragma unroll
    for (int m = 0; m < D1; ++m) {
      load_ch<CPL>(xs[m], xr + m * tl.mul);
#pragma unroll
      for (int c = 0; c < CPL; ++c) gx[m][c] = T(0);
    }
    for (int c0 = k0; c0 < k1; c0 += p.chunk) {
      const int n = min(p.chunk, k1 - c0);
      if (lane < n) {
        const int k = c0 + lane;
        int e = ldg(p.srcedge + k), i = ldg(p.srcrecv + k);
        const bool ok = (unsigned)e < (unsigned)p.E && (unsigned)i < (unsigned)p.N;
        if (!ok) {
          atomicOr(p.err, kErrIndex);
          e = 0;
          i = 0;
        }
        s.i[lane] = i;
        T ph[KP];
        load_phi<KP>(ph, p.phi + (size_t)e * p.K, p.K);
#pragma unroll
        for (int q = 0; q < KP; ++q) s.phi[lane * KP + q] = ok ? ph[q] : T(0);
        const T* yrow = p.Y + (size_t)e * p.dim_y;
        T* cyrow = s.cy + lane * p.cy_stride;
        for (int pi = tl.pbeg + pw; pi < tl.pend; pi += ps) {
          const PathD& pd = p.paths[pi];
          dispatch_l2l3<L1, PR::l2>(pd.l2, pd.l3, [&](auto A2, auto A3) {
            if constexpr (decltype(A3)::value <= PR::l3)
              src_stage_cy<T, L1, decltype(A2)::value, decltype(A3)::value>(yrow, cyrow + pd.cy_off);
          });
        }
      }
      __syncwarp();
      for (int pi = tl.pbeg + pw; pi < tl.pend; pi += ps) {
        const PathD& pd = p.paths[pi];
        dispatch_l2l3<L1, PR::l2>(pd.l2, pd.l3, [&](auto A2, auto A3) {
          if constexpr (decltype(A3)::value <= PR::l3)
            src_path<T, KP, CPL, src_ring_g(sizeof(T), CPL, PR::l3), L1, decltype(A2)::value,
                     decltype(A3)::value>(p, pd, s, n, slot, chl, active, xs, gx);
        });
      }
      __syncwarp();
    }
    if (ps > 1) {
      // split mode: red[warp][m][32 CPL] after the warps' slices, added in warp order
      extern __shared__ __align__(16) unsigned char smem_raw[];
      constexpr int RW = 32 * CPL;
      const int warp = threadIdx.x >> 5;
      T* red = reinterpret_cast<T*>(smem_raw + (size_t)ps * p.warp_smem);
      __syncthreads();   // the previous source's partials have been read
#pragma unroll
      for (int m = 0; m < D1; ++m)
#pragma unroll
        for (int c = 0; c < CPL; ++c) red[(warp * D1 + m) * RW + lane * CPL + c] = gx[m][c];
      __syncthreads();
      if (warp != 0) continue;
      for (int w = 1; w < ps; ++w)
#pragma unroll
        for (int m = 0; m < D1; ++m)
#pragma unroll
          for (int c = 0; c < CPL; ++c) gx[m][c] += red[(w * D1 + m) * RW + lane * CPL + c];
    }
    if (active) {
      T* o = p.gx + (size_t)j * p.c_in + tl.off + chl;
#pragma unroll
      for (int m = 0; m < D1; ++m) store_ch<CPL>(o + m * tl.mul, gx[m]);
    }
  }
}

template <typename T, int KP, int CPL, class PR>
__global__ void __launch_bounds__(src_warps<T>() * 32, ctas_per_sm_for(sizeof(T)))
uvu_src_kernel(const __grid_constant__ UvuSrcParams<T> p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  // every warp of a CTA serves the same input-block tile (one family of path
  // bodies per SM in the instruction cache); the host deals the CTAs to the
  // tiles in proportion to their per-edge cost
  constexpr int W = src_warps<T>();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int tile = 0;
  while (tile + 1 < p.n_tiles && (int)blockIdx.x >= p.tile_cta[tile + 1]) ++tile;
  if (tile >= p.n_tiles || (int)blockIdx.x >= p.tile_cta[tile + 1]) return;
  // split mode: one source stream (slot) per CTA, whose warps deal the paths
  const bool split = p.split > 1;
  const int streams = split ? 1 : W;
  const int stride = min((p.tile_cta[tile + 1] - p.tile_cta[tile]) * streams, p.n_slots);
  const int slot = ((int)blockIdx.x - p.tile_cta[tile]) * streams + (split ? 0 : warp);
  if (slot >= stride) return;   // uniform over the CTA in split mode
  const TileD& tl = p.tiles[tile];
  unsigned char* base = smem_raw + (size_t)warp * p.warp_smem;
  SrcSmem<T> s;
  s.i = reinterpret_cast<int*>(base);
  s.phi = reinterpret_cast<T*>(base + 32 * sizeof(int));
  s.cy = s.phi + 32 * KP;
  s.ring = reinterpret_cast<T*>(base + p.ring_off);
  dispatch_l<PR::l1>(tl.l, [&](auto L) {
    src_tile<T, KP, CPL, PR, decltype(L)::value>(p, tl, slot, stride, lane, s, split ? warp : 0, split ? W : 1);
  });
}

template <typename T>
__global__ void reduce_slots_kernel(const T* __restrict__ part, T* __restrict__ out, int n_slots,
                                    long long n) {
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= n) return;
  T s = T(0);
  for (int k = 0; k < n_slots; ++k) s += part[(size_t)k * n + t];
  out[t] = s;
}

}  // namespace

template <typename T, int KP, int V, class PR>
cudaError_t launch_edge_prof(const UvuEdgeParams<T>& p, unsigned blocks, size_t smem, cudaStream_t s) {
  auto kern = uvu_edge_kernel<T, KP, V, PR>;
  static SmemLimit limit;
  if (cudaError_t e = limit.ensure((const void*)kern, smem); e != cudaSuccess) return e;
  kern<<<blocks, kWarpsPerBlock * 32, smem, s>>>(p);
  return cudaGetLastError();
}

template <typename T, int KP, int V>
cudaError_t launch_uvu_edge(const UvuEdgeParams<T>& p0, int prof, cudaStream_t s) {
  if (p0.N == 0 || p0.E == 0) return cudaSuccess;
  UvuEdgeParams<T> p = p0;
  const long long groups = ((long long)p.E + 31) / 32;
  // split mode while one warp per 32 edges would give fewer than 8 warps per SM
  p.split = groups < kSplitEdgeGroups ? kWarpsPerBlock : 1;
  const unsigned blocks = (unsigned)(p.split > 1 ? groups : (groups + kWarpsPerBlock - 1) / kWarpsPerBlock);
  const size_t smem = p.split > 1 ? sizeof(T) * (size_t)kWarpsPerBlock * (p.K + p.dim_y) * 32 : 0;
  switch (prof) {
    case 0: return launch_edge_prof<T, KP, V, Prof<2, 2, 2>>(p, blocks, smem, s);
    case 1: return launch_edge_prof<T, KP, V, Prof<1, 3, 3>>(p, blocks, smem, s);
    case 2: return launch_edge_prof<T, KP, V, Prof<3, 3, 3>>(p, blocks, smem, s);
    case 3: return launch_edge_prof<T, KP, V, Prof<4, 4, 4>>(p, blocks, smem, s);
    default:   // degrees up to 6: fp32, K <= 8, scalar gathers
      if constexpr (std::is_same<T, float>::value && KP == 8 && V == 1)
        return launch_edge_prof<T, KP, V, Prof<6, 6, 6>>(p, blocks, smem, s);
      return cudaErrorInvalidValue;
  }
}

template <typename T, int KP, int CPL, class PR>
cudaError_t launch_src_prof(const UvuSrcParams<T>& p, unsigned blocks, cudaStream_t s) {
  constexpr int W = src_warps<T>();
  const size_t smem = (size_t)p.warp_smem * W +
                      (p.split > 1 ? sizeof(T) * (size_t)W * (2 * PR::l1 + 1) * 32 * CPL : 0);
  auto kern = uvu_src_kernel<T, KP, CPL, PR>;
  static SmemLimit limit;
  if (cudaError_t e = limit.ensure((const void*)kern, smem); e != cudaSuccess) return e;
  kern<<<blocks, src_warps<T>() * 32, smem, s>>>(p);
  return cudaGetLastError();
}

template <typename T, int KP, int CPL>
cudaError_t launch_uvu_src(const UvuSrcParams<T>& p, int prof, cudaStream_t s) {
  cudaError_t err = cudaMemsetAsync(p.apart, 0, sizeof(T) * (size_t)p.n_slots * p.K * p.n_w, s);
  if (err != cudaSuccess) return err;
  if (p.n_slots == 0 || p.n_tiles == 0 || p.N == 0) return cudaSuccess;
  const unsigned blocks = (unsigned)p.tile_cta[p.n_tiles];
  switch (prof) {
    case 0: return launch_src_prof<T, KP, CPL, Prof<2, 2, 2>>(p, blocks, s);
    case 1: return launch_src_prof<T, KP, CPL, Prof<1, 3, 3>>(p, blocks, s);
    case 2: return launch_src_prof<T, KP, CPL, Prof<3, 3, 3>>(p, blocks, s);
    case 3: return launch_src_prof<T, KP, CPL, Prof<4, 4, 4>>(p, blocks, s);
    default:   // degrees up to 6: fp32, K <= 8, one channel per lane
      if constexpr (std::is_same<T, float>::value && KP == 8 && CPL == 1)
        return launch_src_prof<T, KP, CPL, Prof<6, 6, 6>>(p, blocks, s);
      return cudaErrorInvalidValue;
  }
}

template <typename T>
cudaError_t launch_reduce_slots(const T* part, T* out, int n_slots, long long n, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  reduce_slots_kernel<T><<<(unsigned)((n + 255) / 256), 256, 0, s>>>(part, out, n_slots, n);
  return cudaGetLastError();
}

#define TPC_INST_SRC(T, KP, CPL) \
  template cudaError_t launch_uvu_src<T, KP, CPL>(const UvuSrcParams<T>&, int, cudaStream_t);
#define TPC_INST_EDGE(T, KP, V) \
  template cudaError_t launch_uvu_edge<T, KP, V>(const UvuEdgeParams<T>&, int, cudaStream_t);
#if TPC_WANT(0)
TPC_INST_SRC(float, 8, 1)
#endif
#if TPC_WANT(1)
TPC_INST_SRC(float, 8, 2)
#endif
#if TPC_WANT(2)
TPC_INST_SRC(float, 16, 1)
TPC_INST_SRC(float, 16, 2)
#endif
#if TPC_WANT(9)
TPC_INST_SRC(double, 8, 1)
TPC_INST_SRC(double, 16, 1)
#endif
#if TPC_WANT(3)
TPC_INST_EDGE(float, 8, 1)
#endif
#if TPC_WANT(4)
TPC_INST_EDGE(float, 8, 4)
#endif
#if TPC_WANT(5)
TPC_INST_EDGE(float, 16, 1)
TPC_INST_EDGE(float, 16, 4)
#endif
#if TPC_WANT(6)
TPC_INST_EDGE(double, 8, 1)
#endif
#if TPC_WANT(7)
TPC_INST_EDGE(double, 8, 2)
#endif
#if TPC_WANT(8)
TPC_INST_EDGE(double, 16, 1)
TPC_INST_EDGE(double, 16, 2)
#endif
#undef TPC_INST_SRC
#undef TPC_INST_EDGE
#if TPC_WANT(0)
template cudaError_t launch_reduce_slots<float>(const float*, float*, int, long long, cudaStream_t);
template cudaError_t launch_reduce_slots<double>(const double*, double*, int, long long, cudaStream_t);
#endif

}  // namespace tpc
