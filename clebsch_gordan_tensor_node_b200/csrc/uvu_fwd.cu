// Channelwise (uvu) forward of the edge-conditioned CG tensor-product convolution.
//
// m_i = sum_{j in N(i)} sum_pi w_{ij,pi,u} T_{pi,u}(x_j, Y_ij),
// w_{ij,pi,u} = sum_q phi_{ij,q} A_{q,pi,u}            (Sobek §2.4, Eq. 11-12)
//
// Schedule: the streamed order of Sobek §3.1 -- the scalar w is formed in
// registers and consumed at once; no W and no edge message exists anywhere.
// Work is node-centric as in LunaTP §4.1-4.2: one warp owns one task
// (receiver i, output block g, tile of 32*CPL channels), lanes own CPL adjacent
// channels, the receiver's incoming edges (CSR by receiver) form the inner loop,
// and the output accumulators of block g stay in registers until the single
// store. Paths into g run one after another (outer loop); their A values live in
// registers for the whole edge traversal of that path.
//
// Per edge and path the CG contraction is split into an edge-uniform part and a
// per-channel part: cY[m1][m3] = sum_{m2} c[m1,m2,m3] Y[m2] (a few FMAs shared by
// the warp's CPL channels) and acc[m3] += cY[m1][m3] * (w x[m1]) over the
// non-zero (m1, m3) pairs only; coefficients and indices are compile-time
// constants (LunaTP §4.3, sparse expansion).
#include "common.cuh"
#include "kernels.h"

namespace tpc {
namespace {

template <typename T, int KP, int CPL, int L1, int L2, int L3>
__device__ __forceinline__ void fwd_path(const UvuFwdParams<T>& p, const PathD& pd, int chl,
                                         int e0, int e1, T (&acc)[2 * L3 + 1][CPL]) {
  using CGp = cgt::CG<L1, L2, L3>;
  constexpr int D1 = 2 * L1 + 1, D2 = 2 * L2 + 1, D3 = 2 * L3 + 1;
  T a[KP][CPL];
#pragma unroll
  for (int q = 0; q < KP; ++q) {
    if (q < p.K) {
      load_ch<CPL>(a[q], p.A + (size_t)q * p.n_w + pd.w_off + chl);
    } else {
#pragma unroll
      for (int c = 0; c < CPL; ++c) a[q][c] = T(0);
    }
  }
  const T* xb = p.x + pd.x_off + chl;
  const T* yb = p.Y + L2 * L2;
  const int mul = pd.mul_in;
  for (int e = e0; e < e1; ++e) {
    const int j = ldg(p.senders + e);
    if ((unsigned)j >= (unsigned)p.N) {
      raise_error(p.err, kErrIndex);
      continue;
    }
    T ph[KP];
    load_phi<KP>(ph, p.phi + (size_t)e * p.K, p.K);
    T y[D2];
#pragma unroll
    for (int m = 0; m < D2; ++m) y[m] = ldg(yb + (size_t)e * p.dim_y + m);
    T xv[D1][CPL];
    const T* xr = xb + (size_t)j * p.c_in;
#pragma unroll
    for (int m = 0; m < D1; ++m) load_ch<CPL>(xv[m], xr + m * mul);
    T w[CPL];
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
      w[c] = ph[0] * a[0][c];
#pragma unroll
      for (int q = 1; q < KP; ++q) w[c] = fma(ph[q], a[q][c], w[c]);
    }
    if constexpr (D1 <= D3) {
      // fold w into the inputs, then accumulate straight into acc
#pragma unroll
      for (int m = 0; m < D1; ++m)
#pragma unroll
        for (int c = 0; c < CPL; ++c) xv[m][c] *= w[c];
      static_for<CGp::npair>([&](auto P) {
        constexpr Pair pr = CGp::pair[decltype(P)::value];
        const T cy = pair_coef<T, CGp, decltype(P)::value>(y);
#pragma unroll
        for (int c = 0; c < CPL; ++c) acc[pr.m3][c] = fma(cy, xv[pr.m1][c], acc[pr.m3][c]);
      });
    } else {
      // contract first, then weight the (fewer) output components
      T t[D3][CPL];
      static_for<CGp::npair>([&](auto P) {
        constexpr int Pi = decltype(P)::value;
        constexpr Pair pr = CGp::pair[Pi];
        const T cy = pair_coef<T, CGp, Pi>(y);
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
          if constexpr (first_m3<CGp>(Pi))
            t[pr.m3][c] = cy * xv[pr.m1][c];
          else
            t[pr.m3][c] = fma(cy, xv[pr.m1][c], t[pr.m3][c]);
        }
      });
      static_for<D3>([&](auto M) {
        constexpr int m3 = decltype(M)::value;
        if constexpr (has_m3<CGp>(m3)) {
#pragma unroll
          for (int c = 0; c < CPL; ++c) acc[m3][c] = fma(w[c], t[m3][c], acc[m3][c]);
        }
      });
    }
  }
}

template <typename T, int KP, int CPL, int L3>
__device__ __forceinline__ void fwd_tile(const UvuFwdParams<T>& p, const TileD& tl, int i, int lane) {
  constexpr int D3 = 2 * L3 + 1;
  T acc[D3][CPL];
#pragma unroll
  for (int m = 0; m < D3; ++m)
#pragma unroll
    for (int c = 0; c < CPL; ++c) acc[m][c] = T(0);
  const bool active = lane * CPL < tl.nch;
  // inactive lanes read a valid channel and never store
  const int chl = tl.ch0 + (active ? lane * CPL : 0);
  int e0 = ldg(p.rowptr + i), e1 = ldg(p.rowptr + i + 1);
  if (e0 < 0 || e1 < e0 || e1 > p.E) {
    raise_error(p.err, kErrCsr);
    e1 = e0;
  }
  for (int pi = tl.pbeg; pi < tl.pend; ++pi) {
    const PathD& pd = p.paths[pi];
    dispatch_l1l2<L3>(pd.l1, pd.l2, [&](auto A1, auto A2) {
      fwd_path<T, KP, CPL, decltype(A1)::value, decltype(A2)::value, L3>(p, pd, chl, e0, e1, acc);
    });
  }
  if (active) {
    T* o = p.out + (size_t)i * p.c_out + tl.off + chl;
#pragma unroll
    for (int m = 0; m < D3; ++m) store_ch<CPL>(o + m * tl.mul, acc[m]);
  }
}

template <typename T, int KP, int CPL>
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
uvu_fwd_kernel(const __grid_constant__ UvuFwdParams<T> p) {
  const int lane = threadIdx.x & 31;
  const long long task = (long long)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5);
  if (task >= (long long)p.N * p.n_tiles) return;
  const int i = (int)(task / p.n_tiles);
  const TileD& tl = p.tiles[(int)(task % p.n_tiles)];
  dispatch_l(tl.l, [&](auto L) { fwd_tile<T, KP, CPL, decltype(L)::value>(p, tl, i, lane); });
}

}  // namespace

template <typename T, int KP, int CPL>
cudaError_t launch_uvu_fwd(const UvuFwdParams<T>& p, cudaStream_t s) {
  const long long tasks = (long long)p.N * p.n_tiles;
  if (tasks == 0) return cudaSuccess;
  const long long blocks = (tasks + kWarpsPerBlock - 1) / kWarpsPerBlock;
  uvu_fwd_kernel<T, KP, CPL><<<(unsigned)blocks, kWarpsPerBlock * 32, 0, s>>>(p);
  return cudaGetLastError();
}

#define TPC_INST(T, KP, CPL) \
  template cudaError_t launch_uvu_fwd<T, KP, CPL>(const UvuFwdParams<T>&, cudaStream_t);
#if TPC_WANT(0)
TPC_INST(float, 8, 1)
#endif
#if TPC_WANT(1)
TPC_INST(float, 8, 2)
#endif
#if TPC_WANT(2)
TPC_INST(float, 16, 1)
#endif
#if TPC_WANT(3)
TPC_INST(float, 16, 2)
#endif
#if TPC_WANT(4)
TPC_INST(double, 8, 1)
#endif
#if TPC_WANT(5)
TPC_INST(double, 16, 1)
#endif
#undef TPC_INST

}  // namespace tpc
