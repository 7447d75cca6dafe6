// Fully connected (uvw) path: receiver state S, its backward edge pass, and the
// repacking of A for the channel-mixing GEMMs.
//
// Forward (Sobek §4.2):
//   C_{pi,u,mo}(x_j, Y_ij)   = sum_{mi,my} c^pi x_{j,pi,u,mi} Y_{ij,my}          (Eq. 32)
//   S_{i,pi,q,u,mo}          = sum_{j in N(i)} phi_{ij,q} C_{pi,u,mo}(x_j, Y_ij) (Eq. 33)
//   m^(g)_{i,w,mo}           = sum_{pi in g} sum_{q,u} S_{i,pi,q,u,mo} A_{q,pi,u,w} (Eqs. 34-35)
// S has no output-channel axis. It is built here for a bounded chunk of
// receivers (Sobek §4.2: receiver ranges under a fixed scratch budget), laid out
// per output block g as rows (receiver, mo) x columns (pi, q, u), and mixed by
// one GEMM per block (gemm.cu).
//
// Backward (Sobek §4.3, Eq. 36): A_bar = S^T m_bar and S_bar = m_bar A^T by
// GEMM; the edge pass below differentiates Eq. 33 per edge, in receiver order:
//   phi_bar_{e,q} = sum_{pi,u,mo} S_bar_{i,pi,q,u,mo} C_{pi,u,mo}(x_j, Y_e)
//   Y_bar_e       = sum_pi D_Y C^*[ T_bar ],  T_bar_{pi,u,mo} = sum_q phi_{e,q} S_bar_{i,pi,q,u,mo}
// x_bar is the forward structure on the source view: with the adjoint coupling
// C'_{pi,w,mi} = sum_{my,mo} c^pi Y_{e,my} m_bar_{recv(e),pi,w,mo}, the state
// S'_{j,pi,q,w,mi} = sum_{e: src=j} phi_{e,q} C'_{pi,w,mi} is built by the same
// kernel (direction 1) and x_bar_j = S'_j A'^T by GEMM -- no per-edge adjoint
// tensor and no per-edge read of S_bar.
#include "common.cuh"
#include "kernels.h"

namespace tpc {
namespace {

constexpr int kThreads = 128;      // 4 warps
constexpr int kChunk = 32;         // edges staged per round

template <typename T, int KP>
struct SbSmem {
  T* C;     // [kChunk][DOmax][32]
  T* phi;   // [kChunk][KP]
};

// One path of one owner block: accumulate the state columns (q, channel) of
// this warp's radial indices over the owner's edges, then store them.
template <typename T, int KP, int DIR, int L1, int L2, int L3>
__device__ __forceinline__ void sbuild_path(const UvwSParams<T>& p, const UvwBlockD& bd, const PathD& pd,
                                            int r, int k0, int k1, T* Cs, T* phis) {
  using CGp = cgt::CG<L1, L2, L3>;
  constexpr int D1 = 2 * L1 + 1, D3 = 2 * L3 + 1;
  constexpr int DG = DIR == 0 ? D1 : D3;   // components of the gathered block
  constexpr int DO = DIR == 0 ? D3 : D1;   // components of the owner block
  constexpr int KQ = KP / 4;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gmul = pd.mul_in;              // gathered multiplicity (direction-specific)
  for (int c0 = 0; c0 < gmul; c0 += 32) {
    const bool act = c0 + lane < gmul;
    const int cl = act ? c0 + lane : c0;
    T Sr[KQ][DO];
#pragma unroll
    for (int q = 0; q < KQ; ++q)
#pragma unroll
      for (int m = 0; m < DO; ++m) Sr[q][m] = T(0);
    for (int kc = k0; kc < k1; kc += kChunk) {
      const int n = min(kChunk, k1 - kc);
      // phase A: warp w contracts the CG product of chunk edges w, w+4, ...
      for (int t = warp; t < n; t += 4) {
        const int k = kc + t;
        const int e = p.eid ? ldg(p.eid + k) : k;
        const int nb = ldg(p.nbr + k);
        const bool ok = (unsigned)e < (unsigned)p.E && (unsigned)nb < (unsigned)p.n_feat_rows;
        if (!ok) raise_error(p.err, kErrIndex);
        T y[2 * L2 + 1];
        T g[DG];
#pragma unroll
        for (int m = 0; m < 2 * L2 + 1; ++m) y[m] = ok ? ldg(p.Y + (size_t)e * p.dim_y + L2 * L2 + m) : T(0);
        const T* gr = p.feat + (size_t)(ok ? nb : 0) * p.ld_feat + pd.x_off + cl;
#pragma unroll
        for (int m = 0; m < DG; ++m) g[m] = ldg(gr + (size_t)m * gmul);
        T C[DO];
#pragma unroll
        for (int m = 0; m < DO; ++m) C[m] = T(0);
        static_for<CGp::npair>([&](auto P) {
          constexpr Pair pr = CGp::pair[decltype(P)::value];
          const T cy = pair_coef<T, CGp, decltype(P)::value>(y);
          if constexpr (DIR == 0)
            C[pr.m3] = fma(cy, g[pr.m1], C[pr.m3]);
          else
            C[pr.m1] = fma(cy, g[pr.m3], C[pr.m1]);
        });
#pragma unroll
        for (int m = 0; m < DO; ++m) Cs[(t * DO + m) * 32 + lane] = (act && ok) ? C[m] : T(0);
        if (lane < KP) phis[t * KP + lane] = (ok && lane < p.K) ? ldg(p.phi + (size_t)e * p.K + lane) : T(0);
      }
      __syncthreads();
      // phase B: S[q][m] += phi[q] C[m] for this warp's radial indices
      for (int t = 0; t < n; ++t) {
        T cm[DO];
#pragma unroll
        for (int m = 0; m < DO; ++m) cm[m] = Cs[(t * DO + m) * 32 + lane];
#pragma unroll
        for (int q = 0; q < KQ; ++q) {
          const T ph = phis[t * KP + warp * KQ + q];
#pragma unroll
          for (int m = 0; m < DO; ++m) Sr[q][m] = fma(ph, cm[m], Sr[q][m]);
        }
      }
      __syncthreads();
    }
    if (act) {
      T* dst = p.S + (size_t)p.nr_alloc * bd.s_off + (size_t)(r - p.r0) * DO * bd.dcols + pd.col_off + cl;
#pragma unroll
      for (int q = 0; q < KQ; ++q) {
        const int qq = warp * KQ + q;
        if (qq < p.K) {
#pragma unroll
          for (int m = 0; m < DO; ++m) dst[(size_t)m * bd.dcols + (size_t)qq * gmul] = Sr[q][m];
        }
      }
    }
  }
}

template <typename T, int KP, int DIR>
__global__ void __launch_bounds__(kThreads) uvw_sbuild_kernel(const __grid_constant__ UvwSParams<T> p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  T* Cs = reinterpret_cast<T*>(smem_raw);
  T* phis = Cs + kChunk * (2 * kLmax + 1) * 32;
  const int r = p.r0 + blockIdx.x;
  const UvwBlockD& bd = p.blocks[blockIdx.y];
  if (r >= p.N || bd.pbeg == bd.pend) return;
  int k0 = ldg(p.ptr + r), k1 = ldg(p.ptr + r + 1);
  if (k0 < 0 || k1 < k0 || k1 > p.E) {
    raise_error(p.err, kErrCsr);
    k1 = k0;
  }
  dispatch_l(bd.l, [&](auto LO) {
    constexpr int L = decltype(LO)::value;
    for (int pi = bd.pbeg; pi < bd.pend; ++pi) {
      const PathD& pd = p.paths[pi];
      if constexpr (DIR == 0) {
        dispatch_l1l2<L>(pd.l1, pd.l2, [&](auto A1, auto A2) {
          sbuild_path<T, KP, 0, decltype(A1)::value, decltype(A2)::value, L>(p, bd, pd, r, k0, k1, Cs, phis);
        });
      } else {
        dispatch_l2l3<L>(pd.l2, pd.l3, [&](auto A2, auto A3) {
          sbuild_path<T, KP, 1, L, decltype(A2)::value, decltype(A3)::value>(p, bd, pd, r, k0, k1, Cs, phis);
        });
      }
    }
  });
}

// ---------------------------------------------------------------- edge pass

constexpr int kEdgeChunk = 64;

template <typename T>
__device__ __forceinline__ T wsum(T v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <typename T, int KP, int L1, int L2, int L3>
__device__ __forceinline__ void edge_path(const UvwEdgeParams<T>& p, const UvwBlockD& bd, const PathD& pd,
                                          int r, int ec, int n, T* Sb, T* acc) {
  using CGp = cgt::CG<L1, L2, L3>;
  constexpr int D1 = 2 * L1 + 1, D2 = 2 * L2 + 1, D3 = 2 * L3 + 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int mi = pd.mul_in;
  const int accw = p.K + p.dim_y;
  for (int c0 = 0; c0 < mi; c0 += 32) {
    // stage S_bar of receiver r, this path, channel tile: Sb[q][m3][lane]
    const T* src = p.Sbar + (size_t)p.nr_alloc * bd.s_off + (size_t)(r - p.r0) * D3 * bd.dcols + pd.col_off + c0;
    for (int t = threadIdx.x; t < KP * D3 * 32; t += kThreads) {
      const int c = t & 31, m3 = (t >> 5) % D3, q = (t >> 5) / D3;
      Sb[t] = (q < p.K && c0 + c < mi) ? src[(size_t)m3 * bd.dcols + (size_t)q * mi + c] : T(0);
    }
    __syncthreads();
    const bool act = c0 + lane < mi;
    const int cl = act ? c0 + lane : c0;
    for (int t = warp; t < n; t += 4) {
      const int e = ec + t;
      const int j = ldg(p.senders + e);
      if ((unsigned)j >= (unsigned)p.N) {
        raise_error(p.err, kErrIndex);
        continue;
      }
      T x[D1], y[D2], ph[KP];
      const T* xr = p.x + (size_t)j * p.c_in + pd.x_off + cl;
#pragma unroll
      for (int m = 0; m < D1; ++m) x[m] = act ? ldg(xr + (size_t)m * mi) : T(0);
#pragma unroll
      for (int m = 0; m < D2; ++m) y[m] = ldg(p.Y + (size_t)e * p.dim_y + L2 * L2 + m);
#pragma unroll
      for (int q = 0; q < KP; ++q) ph[q] = q < p.K ? ldg(p.phi + (size_t)e * p.K + q) : T(0);
      T C[D3];
#pragma unroll
      for (int m = 0; m < D3; ++m) C[m] = T(0);
      static_for<CGp::npair>([&](auto P) {
        constexpr Pair pr = CGp::pair[decltype(P)::value];
        const T cy = pair_coef<T, CGp, decltype(P)::value>(y);
        C[pr.m3] = fma(cy, x[pr.m1], C[pr.m3]);
      });
      T tb[D3], gp[KP];
#pragma unroll
      for (int m = 0; m < D3; ++m) tb[m] = T(0);
#pragma unroll
      for (int q = 0; q < KP; ++q) {
        T s = T(0);
#pragma unroll
        for (int m = 0; m < D3; ++m) {
          const T sb = Sb[(q * D3 + m) * 32 + lane];
          tb[m] = fma(ph[q], sb, tb[m]);
          s = fma(sb, C[m], s);
        }
        gp[q] = s;
      }
      T gy[D2];
#pragma unroll
      for (int m = 0; m < D2; ++m) gy[m] = T(0);
      static_for<CGp::npair>([&](auto P) {
        constexpr Pair pr = CGp::pair[decltype(P)::value];
        const T z = x[pr.m1] * tb[pr.m3];
        static_for<pr.n>([&](auto k) {
          constexpr Term tm = CGp::term[pr.start + decltype(k)::value];
          gy[tm.m2] = fma(T(tm.c), z, gy[tm.m2]);
        });
      });
      T* a = acc + t * accw;
#pragma unroll
      for (int q = 0; q < KP; ++q) {
        if (q < p.K) {
          const T v = wsum(gp[q]);
          if (lane == 0) a[q] += v;
        }
      }
#pragma unroll
      for (int m = 0; m < D2; ++m) {
        const T v = wsum(gy[m]);
        if (lane == 0) a[p.K + L2 * L2 + m] += v;
      }
    }
    __syncthreads();
  }
}

template <typename T, int KP>
__global__ void __launch_bounds__(kThreads) uvw_edge_kernel(const __grid_constant__ UvwEdgeParams<T> p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  T* Sb = reinterpret_cast<T*>(smem_raw);                 // [KP][D3max][32]
  T* acc = Sb + KP * (2 * kLmax + 1) * 32;                // [kEdgeChunk][K + dim_y]
  const int r = p.r0 + blockIdx.x;
  if (r >= p.N) return;
  int k0 = ldg(p.rowptr + r), k1 = ldg(p.rowptr + r + 1);
  if (k0 < 0 || k1 < k0 || k1 > p.E) {
    raise_error(p.err, kErrCsr);
    return;
  }
  const int accw = p.K + p.dim_y;
  for (int ec = k0; ec < k1; ec += kEdgeChunk) {
    const int n = min(kEdgeChunk, k1 - ec);
    for (int t = threadIdx.x; t < n * accw; t += kThreads) acc[t] = T(0);
    __syncthreads();
    for (int b = 0; b < p.n_blocks; ++b) {
      const UvwBlockD& bd = p.blocks[b];
      dispatch_l(bd.l, [&](auto L3c) {
        constexpr int L3 = decltype(L3c)::value;
        for (int pi = bd.pbeg; pi < bd.pend; ++pi) {
          const PathD& pd = p.paths[pi];
          dispatch_l1l2<L3>(pd.l1, pd.l2, [&](auto A1, auto A2) {
            edge_path<T, KP, decltype(A1)::value, decltype(A2)::value, L3>(p, bd, pd, r, ec, n, Sb, acc);
          });
        }
      });
    }
    for (int t = threadIdx.x; t < n * accw; t += kThreads) {
      const int el = t / accw, v = t - el * accw;
      const int e = ec + el;
      if (v < p.K)
        p.gphi[(size_t)e * p.K + v] = acc[t];
      else
        p.gY[(size_t)e * p.dim_y + (v - p.K)] = acc[t];
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------- A repacking

// Column (within A's row q) to packed row/col: every element of A [K, N_w] is
// copied to the forward layout B_g [(pi, q, u), w] and the adjoint layout
// B'_b [(pi, q, w), u] (or the reverse for the unpack of A_bar).
// Layouts: Bf (forward, SIMT) [(pi,q,u), w]; Ba (adjoint, SIMT) [(pi,q,w), u];
// Btf / Bta: the same transposed, [w, (pi,q,u)] / [u, (pi,q,w)] (K-major operands
// of the tensor-core GEMM). Any output may be NULL.
template <typename T>
__device__ __forceinline__ T hi_part(T v) {
  if constexpr (sizeof(T) == 4)
    return __uint_as_float(__float_as_uint(v) & 0xFFFFE000u);
  else
    return v;
}

template <typename T>
__global__ void pack_a_kernel(const __grid_constant__ UvwPackParams p, const T* __restrict__ A,
                              T* __restrict__ Bf, T* __restrict__ Ba, T* __restrict__ Btf,
                              T* __restrict__ Bta, T* __restrict__ Btf_lo, T* __restrict__ Bta_lo) {
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)p.K * p.n_w) return;
  const int q = (int)(idx / p.n_w);
  const int col = (int)(idx - (long long)q * p.n_w);
  int lo = 0, hi = p.n_paths;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (p.paths[mid].w_off <= col) lo = mid; else hi = mid;
  }
  const PackPath& pp = p.paths[lo];
  const int rem = col - pp.w_off, u = rem / pp.mo, w = rem - u * pp.mo;
  const T v = A[idx];
  if (Bf) Bf[pp.bf_off + ((size_t)pp.colf + (size_t)q * pp.mi + u) * pp.mo + w] = v;
  if (Ba) Ba[pp.ba_off + ((size_t)pp.cola + (size_t)q * pp.mo + w) * pp.mi + u] = v;
  const T vh = hi_part(v);
  if (Btf) {
    const size_t o = pp.bf_off + (size_t)w * pp.dcf + pp.colf + (size_t)q * pp.mi + u;
    Btf[o] = Btf_lo ? vh : v;
    if (Btf_lo) Btf_lo[o] = v - vh;
  }
  if (Bta) {
    const size_t o = pp.ba_off + (size_t)u * pp.dca + pp.cola + (size_t)q * pp.mo + w;
    Bta[o] = Bta_lo ? vh : v;
    if (Bta_lo) Bta_lo[o] = v - vh;
  }
}

template <typename T>
__global__ void unpack_a_kernel(const __grid_constant__ UvwPackParams p, const T* __restrict__ Bf,
                                T* __restrict__ A) {
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)p.K * p.n_w) return;
  const int q = (int)(idx / p.n_w);
  const int col = (int)(idx - (long long)q * p.n_w);
  int lo = 0, hi = p.n_paths;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (p.paths[mid].w_off <= col) lo = mid; else hi = mid;
  }
  const PackPath& pp = p.paths[lo];
  const int rem = col - pp.w_off, u = rem / pp.mo, w = rem - u * pp.mo;
  A[idx] = Bf[pp.bf_off + ((size_t)pp.colf + (size_t)q * pp.mi + u) * pp.mo + w];
}

}  // namespace

template <typename T, int KP, int DIR>
cudaError_t launch_uvw_sbuild_dir(const UvwSParams<T>& p, cudaStream_t s) {
  if (p.nr <= 0 || p.n_blocks == 0) return cudaSuccess;
  const size_t smem = sizeof(T) * (size_t)(kChunk * (2 * kLmax + 1) * 32 + kChunk * KP);
  dim3 grid(p.nr, p.n_blocks);
  auto k = uvw_sbuild_kernel<T, KP, DIR>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  k<<<grid, kThreads, smem, s>>>(p);
  return cudaGetLastError();
}

template <typename T, int KP>
cudaError_t launch_uvw_edge(const UvwEdgeParams<T>& p, cudaStream_t s) {
  if (p.nr <= 0) return cudaSuccess;
  const size_t smem = sizeof(T) * ((size_t)KP * (2 * kLmax + 1) * 32 + (size_t)kEdgeChunk * (p.K + p.dim_y));
  auto k = uvw_edge_kernel<T, KP>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  k<<<p.nr, kThreads, smem, s>>>(p);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_pack_a(const UvwPackParams& p, const T* A, T* Bf, T* Ba, T* Btf, T* Bta, T* Btf_lo,
                          T* Bta_lo, cudaStream_t s) {
  const long long n = (long long)p.K * p.n_w;
  if (n == 0) return cudaSuccess;
  pack_a_kernel<T><<<(unsigned)((n + 255) / 256), 256, 0, s>>>(p, A, Bf, Ba, Btf, Bta, Btf_lo, Bta_lo);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_unpack_a(const UvwPackParams& p, const T* Bf, T* A, cudaStream_t s) {
  const long long n = (long long)p.K * p.n_w;
  if (n == 0) return cudaSuccess;
  unpack_a_kernel<T><<<(unsigned)((n + 255) / 256), 256, 0, s>>>(p, Bf, A);
  return cudaGetLastError();
}

#define TPC_INST_S(T, KP, DIR) \
  template cudaError_t launch_uvw_sbuild_dir<T, KP, DIR>(const UvwSParams<T>&, cudaStream_t);
#define TPC_INST_E(T, KP) template cudaError_t launch_uvw_edge<T, KP>(const UvwEdgeParams<T>&, cudaStream_t);
#if TPC_WANT(0)
template cudaError_t launch_pack_a<float>(const UvwPackParams&, const float*, float*, float*, float*, float*,
                                          float*, float*, cudaStream_t);
template cudaError_t launch_unpack_a<float>(const UvwPackParams&, const float*, float*, cudaStream_t);
template cudaError_t launch_pack_a<double>(const UvwPackParams&, const double*, double*, double*, double*,
                                           double*, double*, double*, cudaStream_t);
template cudaError_t launch_unpack_a<double>(const UvwPackParams&, const double*, double*, cudaStream_t);
TPC_INST_S(float, 8, 0)
#endif
#if TPC_WANT(1)
TPC_INST_S(float, 8, 1)
#endif
#if TPC_WANT(2)
TPC_INST_E(float, 8)
#endif
#if TPC_WANT(3)
TPC_INST_S(float, 16, 0)
#endif
#if TPC_WANT(4)
TPC_INST_S(float, 16, 1)
#endif
#if TPC_WANT(5)
TPC_INST_E(float, 16)
#endif
#if TPC_WANT(6)
TPC_INST_S(double, 8, 0)
TPC_INST_S(double, 8, 1)
#endif
#if TPC_WANT(7)
TPC_INST_E(double, 8)
#endif
#if TPC_WANT(8)
TPC_INST_S(double, 16, 0)
TPC_INST_S(double, 16, 1)
#endif
#if TPC_WANT(9)
TPC_INST_E(double, 16)
#endif
#undef TPC_INST_S
#undef TPC_INST_E

}  // namespace tpc
