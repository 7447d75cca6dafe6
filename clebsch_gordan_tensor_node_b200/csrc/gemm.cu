// Channel-mixing GEMMs of the fully connected (uvw) path, SIMT fp32/fp64.
//
// Sobek §4.2 (Eqs. 34-35): with receiver and output component packed as rows and
// (path, radial index, input channel) as the contracted dimension, the mixing is
// one matrix product per output group, m = S A; Sobek §4.3 (Eq. 36): the
// backward uses S_bar = m_bar A^T and A_bar = S^T m_bar. All three shapes run
// through one tiled kernel; the operands are addressed by small descriptors so
// that output rows (receiver, component) land directly in the ir_mul output.
//
//   op NN:  C[m][n] = sum_k X[m][k] * B[k][n]      (m = S A, x_bar = S' A')
//   op NT:  C[m][k] = sum_n G[m][n] * B[k][n]      (S_bar = m_bar A^T)
//   op TN:  C[k][n] (+)= sum_m X[m][k] * G[m][n]   (A_bar += S^T m_bar)
//
// X and S-like operands are dense row-major [M, D]; B is dense row-major [D, N];
// G is "row-blocked": row m = (owner r, component c) lives at
// base + (r0 + r) * ld_outer + off + c * N (the ir_mul layout of one block).
#include "common.cuh"
#include "kernels.h"

namespace tpc {
namespace {

constexpr int BM = 64, BN = 32, BK = 16, NT = 256;  // tile and threads; thread tile 4 x 2

template <typename T>
__device__ __forceinline__ const T* blocked_row(const T* base, const RowBlocked& rb, int m) {
  const int r = m / rb.dcomp, c = m - r * rb.dcomp;
  return base + (size_t)(rb.r0 + r) * rb.ld_outer + rb.off + (size_t)c * rb.n;
}

template <typename T>
__device__ __forceinline__ T* blocked_row(T* base, const RowBlocked& rb, int m) {
  const int r = m / rb.dcomp, c = m - r * rb.dcomp;
  return base + (size_t)(rb.r0 + r) * rb.ld_outer + rb.off + (size_t)c * rb.n;
}

// One (batch) problem per blockIdx.z.
template <typename T, int OP>
__global__ void __launch_bounds__(NT) gemm_kernel(const __grid_constant__ GemmBatch<T> gb) {
  const GemmProb<T>& p = gb.prob[blockIdx.z];
  // output tile origin
  int M, N, Kd;
  if (OP == 0) { M = p.M; N = p.N; Kd = p.D; }          // C[M,N] = X[M,D] B[D,N]
  else if (OP == 1) { M = p.M; N = p.D; Kd = p.N; }     // C[M,D] = G[M,N] B[D,N]^T
  else { M = p.D; N = p.N; Kd = p.M; }                  // C[D,N] = X[M,D]^T G[M,N]
  const int tm = blockIdx.y * BM, tn = blockIdx.x * BN;
  if (tm >= M || tn >= N) return;
  __shared__ T As[BK][BM + 4];
  __shared__ T Bs[BK][BN + 4];
  const int tid = threadIdx.x;
  const int tx = tid % 16, ty = tid / 16;       // 16 x 16 threads; thread tile rows 4, cols 2
  T acc[4][2];
#pragma unroll
  for (int a = 0; a < 4; ++a) acc[a][0] = acc[a][1] = T(0);
  for (int k0 = 0; k0 < Kd; k0 += BK) {
    // stage A-like tile: As[k][m] (BK x BM = 1024 values, 4 per thread)
#pragma unroll
    for (int t = 0; t < (BK * BM) / NT; ++t) {
      const int idx = tid + t * NT;
      int kk, mm;
      if (OP == 2) { kk = idx / BM; mm = idx % BM; } else { mm = idx / BK; kk = idx % BK; }
      const int gm = tm + mm, gk = k0 + kk;
      T v = T(0);
      if (gm < M && gk < Kd) {
        if (OP == 0) v = p.X[(size_t)gm * p.D + gk];
        else if (OP == 1) v = blocked_row(p.G, p.g, gm)[gk];
        else v = p.X[(size_t)gk * p.D + gm];
      }
      As[kk][mm] = v;
    }
    // stage B-like tile: Bs[k][n] (BK x BN = 512 values, 2 per thread)
#pragma unroll
    for (int t = 0; t < (BK * BN) / NT; ++t) {
      const int idx = tid + t * NT;
      int kk, nn;
      if (OP == 1) { nn = idx / BK; kk = idx % BK; } else { kk = idx / BN; nn = idx % BN; }
      const int gn = tn + nn, gk = k0 + kk;
      T v = T(0);
      if (gn < N && gk < Kd) {
        if (OP == 0) v = p.B[(size_t)gk * p.N + gn];
        else if (OP == 1) v = p.B[(size_t)gn * p.N + gk];
        else v = blocked_row(p.G, p.g, gk)[gn];
      }
      Bs[kk][nn] = v;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      T a[4], b[2];
#pragma unroll
      for (int r = 0; r < 4; ++r) a[r] = As[kk][ty * 4 + r];
      b[0] = Bs[kk][tx * 2];
      b[1] = Bs[kk][tx * 2 + 1];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        acc[r][0] = fma(a[r], b[0], acc[r][0]);
        acc[r][1] = fma(a[r], b[1], acc[r][1]);
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int gm = tm + ty * 4 + r;
    if (gm >= M) continue;
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int gn = tn + tx * 2 + c;
      if (gn >= N) continue;
      if (OP == 0) {
        blocked_row(p.C, p.c, gm)[gn] = acc[r][c];
      } else if (OP == 1) {
        p.C[(size_t)gm * p.D + gn] = acc[r][c];
      } else {
        T* dst = p.C + (size_t)gm * p.N + gn;
        *dst = p.accumulate ? *dst + acc[r][c] : acc[r][c];
      }
    }
  }
}

}  // namespace

template <typename T>
cudaError_t launch_gemm(int op, const GemmBatch<T>& gb, int n_prob, int max_m, int max_n, cudaStream_t s) {
  if (n_prob == 0 || max_m == 0 || max_n == 0) return cudaSuccess;
  dim3 grid((max_n + BN - 1) / BN, (max_m + BM - 1) / BM, n_prob);
  if (op == 0) gemm_kernel<T, 0><<<grid, NT, 0, s>>>(gb);
  else if (op == 1) gemm_kernel<T, 1><<<grid, NT, 0, s>>>(gb);
  else gemm_kernel<T, 2><<<grid, NT, 0, s>>>(gb);
  return cudaGetLastError();
}

template cudaError_t launch_gemm<float>(int, const GemmBatch<float>&, int, int, int, cudaStream_t);
template cudaError_t launch_gemm<double>(int, const GemmBatch<double>&, int, int, int, cudaStream_t);

}  // namespace tpc
