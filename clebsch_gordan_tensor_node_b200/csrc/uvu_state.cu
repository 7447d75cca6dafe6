// Channelwise (uvu) forward in the receiver-factorised order of Sobek §4.2,
// an alternative schedule kept beside the streamed one (uvu_fwd.cu).
//
//   C_{pi,u,mo}(x_j, Y_ij) = sum_{mi,my} c^pi x_{j,pi,u,mi} Y_{ij,my}        (Eq. 32)
//   S_{i,pi,q,u,mo}        = sum_{j in N(i)} phi_{ij,q} C_{pi,u,mo}          (Eq. 33)
//   m_{i,u,mo}            += sum_q A_{q,pi,u} S_{i,pi,q,u,mo}                (Eqs. 34-35,
//                                                                              channelwise)
// For a channelwise path the mixing is diagonal in the channel, so the state of
// one receiver, path and channel (K x (2 l3 + 1) values) stays in one lane's
// registers over the receiver's edges and is mixed once at the end: one warp
// per (receiver, 32-channel tile of an output block), lane = channel. Per edge
// and channel it costs nnz + K (2 l3 + 1) FMAs against the streamed order's
// K + nnz + (2 l3 + 1), which is why the streamed order is the default.
#include "common.cuh"
#include "kernels.h"

namespace tpc {
namespace {

constexpr int kStWarps = 8;

template <typename T, int KP, int L1, int L2, int L3>
__device__ __forceinline__ void state_path(const UvuFwdParams<T>& p, const PathD& pd, int e0, int e1, int ch,
                                           T (&acc)[2 * L3 + 1]) {
  using CGp = cgt::CG<L1, L2, L3>;
  constexpr int D1 = 2 * L1 + 1, D2 = 2 * L2 + 1, D3 = 2 * L3 + 1, NP = CGp::npair, Y0 = L2 * L2;
  T S[KP][D3];
#pragma unroll
  for (int q = 0; q < KP; ++q)
#pragma unroll
    for (int m = 0; m < D3; ++m) S[q][m] = T(0);
  const int mul = pd.mul_in;
  for (int e = e0; e < e1; ++e) {
    const int j = ldg(p.senders + e);
    if ((unsigned)j >= (unsigned)p.N) {   // uniform over the warp
      raise_error(p.err, kErrIndex);
      continue;
    }
    T y[D2];
#pragma unroll
    for (int m = 0; m < D2; ++m) y[m] = ldg(p.Y + (size_t)e * p.dim_y + Y0 + m);
    T xv[D1];
    const T* xr = p.x + (size_t)j * p.c_in + pd.x_off + ch;
#pragma unroll
    for (int m = 0; m < D1; ++m) xv[m] = ldg(xr + m * mul);
    T C[D3];   // Eq. 32 for this edge and channel
#pragma unroll
    for (int m = 0; m < D3; ++m) C[m] = T(0);
    static_for<NP>([&](auto P) {
      constexpr int Pi = decltype(P)::value;
      constexpr Pair pr = CGp::pair[Pi];
      C[pr.m3] = fma(pair_coef<T, CGp, Pi>(y), xv[pr.m1], C[pr.m3]);
    });
#pragma unroll
    for (int q = 0; q < KP; ++q) {   // Eq. 33: S += phi (outer) C
      const T ph = q < p.K ? ldg(p.phi + (size_t)e * p.K + q) : T(0);
#pragma unroll
      for (int m = 0; m < D3; ++m) S[q][m] = fma(ph, C[m], S[q][m]);
    }
  }
#pragma unroll
  for (int q = 0; q < KP; ++q) {     // mixing, once per receiver
    const T a = q < p.K ? ldg(p.A + (size_t)q * p.n_w + pd.w_off + ch) : T(0);
#pragma unroll
    for (int m = 0; m < D3; ++m) acc[m] = fma(a, S[q][m], acc[m]);
  }
}

template <typename T, int KP, int L1M, int L2M, int L3>
__device__ __forceinline__ void state_tile(const UvuFwdParams<T>& p, const TileD& tl, int i, int lane) {
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
      state_path<T, KP, decltype(A1)::value, decltype(A2)::value, L3>(p, pd, e0, e1, ch, acc);
    });
  }
  if (active) {
    T* o = p.out + (size_t)i * p.c_out + tl.off + ch;
#pragma unroll
    for (int m = 0; m < D3; ++m) o[(size_t)m * tl.mul] = acc[m];
  }
}

template <typename T, int KP, int L1M, int L2M, int L3M>
__global__ void __launch_bounds__(kStWarps * 32) uvu_state_fwd_kernel(const __grid_constant__ UvuFwdParams<T> p) {
  const int lane = threadIdx.x & 31;
  const long long task = (long long)blockIdx.x * kStWarps + (threadIdx.x >> 5);
  if (task >= (long long)p.N * p.n_tiles) return;
  const int i = (int)(task / p.n_tiles);
  const TileD& tl = p.tiles[(int)(task - (long long)i * p.n_tiles)];
  dispatch_l<L3M>(tl.l, [&](auto L) { state_tile<T, KP, L1M, L2M, decltype(L)::value>(p, tl, i, lane); });
}

}  // namespace

template <typename T>
cudaError_t launch_uvu_state_fwd(const UvuFwdParams<T>& p, int prof, cudaStream_t s) {
  const long long tasks = (long long)p.N * p.n_tiles;
  if (tasks == 0) return cudaSuccess;
  const unsigned blocks = (unsigned)((tasks + kStWarps - 1) / kStWarps);
  switch (prof) {
    case 0: uvu_state_fwd_kernel<T, 8, 2, 2, 2><<<blocks, kStWarps * 32, 0, s>>>(p); break;
    case 1: uvu_state_fwd_kernel<T, 8, 1, 3, 3><<<blocks, kStWarps * 32, 0, s>>>(p); break;
    case 2: uvu_state_fwd_kernel<T, 8, 3, 3, 3><<<blocks, kStWarps * 32, 0, s>>>(p); break;
    case 3: uvu_state_fwd_kernel<T, 8, 4, 4, 4><<<blocks, kStWarps * 32, 0, s>>>(p); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

#if TPC_WANT(0)
template cudaError_t launch_uvu_state_fwd<float>(const UvuFwdParams<float>&, int, cudaStream_t);
#endif
#if TPC_WANT(1)
template cudaError_t launch_uvu_state_fwd<double>(const UvuFwdParams<double>&, int, cudaStream_t);
#endif

}  // namespace tpc
