// Channel-mixing GEMMs of the fully connected (uvw) path, SIMT fp32/fp64.
//
// Sobek §4.2 (Eqs. 34-35): with receiver and output component packed as rows and
// (path, radial index, input channel) as the contracted dimension, the mixing is
// one matrix product per output group, m = S A; Sobek §4.3 (Eq. 36): the
// backward uses S_bar = m_bar A^T and A_bar = S^T m_bar. All three shapes run
// through one tiled kernel; the operands are addressed by small descriptors so
// that output rows (receiver, component) land directly in the ir_mul output.
//
//   op NN:  C[m][n] (+)= sum_k X[m][k] * B[k][n]   (m = S A, x_bar = S' A')
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
        T* dst = blocked_row(p.C, p.c, gm) + gn;
        *dst = p.accumulate ? *dst + acc[r][c] : acc[r][c];
      } else if (OP == 1) {
        p.C[(size_t)gm * p.D + gn] = acc[r][c];
      } else {
        T* dst = p.C + (size_t)gm * p.N + gn;
        *dst = p.accumulate ? *dst + acc[r][c] : acc[r][c];
      }
    }
  }
}

// ---------------------------------------------------------------- backward products
//
// The two backward products stream a whole state chunk through a short inner
// dimension (the mul_out channels of one block), so they are bound by memory,
// not arithmetic. Dedicated shapes:
//
//   S_bar = m_bar B^T (op NT): a CTA writes a 64 x 128 tile of S_bar from the
//   64 m_bar rows and 128 B rows it stages once per 32-wide slice of the inner
//   dimension; each thread owns 8 x 4 outputs (32 FMAs per three 16-byte shared
//   loads) and stores rows with 16-byte writes.
//
//   A_bar += S^T m_bar (op TN): split-K. CTA (d tile of 64, n tile of 32, split
//   s) reduces rows [m0, m1) of split s into a partial [64 x 32] tile with the
//   next 32-row slice of S and m_bar held in registers while the current one is
//   contracted from shared memory; the partials of all splits are then added in
//   split order (deterministic) into A_bar.

constexpr int NT_BM = 64, NT_BD = 128, NT_BK = 32;

template <typename T>
__global__ void __launch_bounds__(256) gemm_nt_kernel(const __grid_constant__ GemmBatch<T> gb) {
  const GemmProb<T>& p = gb.prob[blockIdx.z];
  const int M = p.M, Dn = p.D, Kd = p.N;   // C[M, D] = G[M, N] B[D, N]^T
  const int tm = blockIdx.y * NT_BM, tn = blockIdx.x * NT_BD;
  if (tm >= M || tn >= Dn) return;
  constexpr int BK = sizeof(T) == 4 ? NT_BK : NT_BK / 2;   // 48 KiB of static shared memory at most
  __shared__ __align__(16) T Gs[BK][NT_BM + 4];
  __shared__ __align__(16) T Bs[BK][NT_BD + 4];
  const int tid = threadIdx.x, lane = tid & 31, ry = tid >> 5;   // warp ry owns rows ry*8 .. +8
  T acc[8][4];
#pragma unroll
  for (int r = 0; r < 8; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[r][c] = T(0);
  for (int k0 = 0; k0 < Kd; k0 += BK) {
    // G rows: consecutive threads read consecutive k of one row
#pragma unroll
    for (int i = 0; i < NT_BM * BK / 256; ++i) {
      const int idx = tid + 256 * i, row = idx / BK, k = idx % BK;
      const int gm = tm + row, gk = k0 + k;
      Gs[k][row] = (gm < M && gk < Kd) ? blocked_row(p.G, p.g, gm)[gk] : T(0);
    }
#pragma unroll
    for (int i = 0; i < NT_BD * BK / 256; ++i) {
      const int idx = tid + 256 * i, d = idx / BK, k = idx % BK;
      const int gd = tn + d, gk = k0 + k;
      Bs[k][d] = (gd < Dn && gk < Kd) ? p.B[(size_t)gd * Kd + gk] : T(0);
    }
    __syncthreads();
#pragma unroll 8
    for (int k = 0; k < BK; ++k) {
      T a[8], b[4];
#pragma unroll
      for (int r = 0; r < 8; ++r) a[r] = Gs[k][ry * 8 + r];
#pragma unroll
      for (int c = 0; c < 4; ++c) b[c] = Bs[k][lane * 4 + c];
#pragma unroll
      for (int r = 0; r < 8; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[r][c] = fma(a[r], b[c], acc[r][c]);
    }
    __syncthreads();
  }
  const int gn = tn + lane * 4;
  // 16-byte stores where every row of this problem's C starts on a 16-byte boundary
  const bool vec = sizeof(T) == 4 && (Dn & 3) == 0 && (reinterpret_cast<uintptr_t>(p.C) & 15) == 0 && gn + 4 <= Dn;
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    const int gm = tm + ry * 8 + r;
    if (gm >= M) continue;
    T* dst = p.C + (size_t)gm * Dn + gn;
    if (vec) {
      if constexpr (sizeof(T) == 4)
        *reinterpret_cast<float4*>(dst) = make_float4(acc[r][0], acc[r][1], acc[r][2], acc[r][3]);
    } else {
#pragma unroll
      for (int c = 0; c < 4; ++c)
        if (gn + c < Dn) dst[c] = acc[r][c];
    }
  }
}

constexpr int TN_BD = 64, TN_BN = 32, TN_BM = 32;

template <typename T>
__global__ void __launch_bounds__(256) gemm_tn_kernel(const __grid_constant__ GemmBatch<T> gb, const T* c_base,
                                                      T* partial, size_t split_stride, int splits) {
  const GemmProb<T>& p = gb.prob[blockIdx.z];
  const int Dn = p.D, N = p.N, M = p.M;    // C[D, N] = X[M, D]^T G[M, N]
  const int n_tiles = (N + TN_BN - 1) / TN_BN;
  const int td = blockIdx.x * TN_BD, tn = (blockIdx.y % n_tiles) * TN_BN, split = blockIdx.y / n_tiles;
  if (td >= Dn || split >= splits) return;
  const int per = ((M + splits - 1) / splits + TN_BM - 1) / TN_BM * TN_BM;
  const int m0 = split * per, m1 = min(M, m0 + per);
  __shared__ __align__(16) T Xs[TN_BM][TN_BD + 4];
  __shared__ __align__(16) T Gs[TN_BM][TN_BN + 4];
  const int tid = threadIdx.x, dx = tid & 15, ny = tid >> 4;   // outputs d = dx*4 .. +4, n = ny*2 .. +2
  T acc[4][2];
#pragma unroll
  for (int a = 0; a < 4; ++a) acc[a][0] = acc[a][1] = T(0);
  // register staging of one 32-row slice: X 32 x 64 (8 per thread), G 32 x 32 (4 per thread)
  T xr[8], gr[4];
  auto fetch = [&](int mb) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int idx = tid + 256 * i, row = idx / TN_BD, d = idx % TN_BD;
      const int gm = mb + row, gd = td + d;
      xr[i] = (gm < m1 && gd < Dn) ? p.X[(size_t)gm * Dn + gd] : T(0);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int idx = tid + 256 * i, row = idx / TN_BN, n = idx % TN_BN;
      const int gm = mb + row, gn = tn + n;
      gr[i] = (gm < m1 && gn < N) ? blocked_row(p.G, p.g, gm)[gn] : T(0);
    }
  };
  if (m0 < m1) fetch(m0);
  for (int mb = m0; mb < m1; mb += TN_BM) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int idx = tid + 256 * i;
      Xs[idx / TN_BD][idx % TN_BD] = xr[i];
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int idx = tid + 256 * i;
      Gs[idx / TN_BN][idx % TN_BN] = gr[i];
    }
    __syncthreads();
    if (mb + TN_BM < m1) fetch(mb + TN_BM);   // next slice in flight during the arithmetic
#pragma unroll 8
    for (int k = 0; k < TN_BM; ++k) {
      T a[4], b[2];
#pragma unroll
      for (int r = 0; r < 4; ++r) a[r] = Xs[k][dx * 4 + r];
      b[0] = Gs[k][ny * 2];
      b[1] = Gs[k][ny * 2 + 1];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        acc[r][0] = fma(a[r], b[0], acc[r][0]);
        acc[r][1] = fma(a[r], b[1], acc[r][1]);
      }
    }
    __syncthreads();
  }
  // partial tile of this split at the problem's place in the packed A layout
  T* out = partial + (size_t)split * split_stride + (p.C - c_base);
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int gd = td + dx * 4 + r;
    if (gd >= Dn) continue;
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int gn = tn + ny * 2 + c;
      if (gn < N) out[(size_t)gd * N + gn] = acc[r][c];
    }
  }
}

template <typename T>
__global__ void sum_splits_kernel(const T* __restrict__ partial, size_t split_stride, int splits, T* __restrict__ out,
                                  long long n, int accumulate) {
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= n) return;
  T s = accumulate ? out[t] : T(0);
  for (int k = 0; k < splits; ++k) s += partial[(size_t)k * split_stride + t];
  out[t] = s;
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

template <typename T>
cudaError_t launch_gemm_nt(const GemmBatch<T>& gb, int n_prob, int max_m, int max_d, cudaStream_t s) {
  if (n_prob == 0 || max_m == 0 || max_d == 0) return cudaSuccess;
  dim3 grid((max_d + NT_BD - 1) / NT_BD, (max_m + NT_BM - 1) / NT_BM, n_prob);
  gemm_nt_kernel<T><<<grid, 256, 0, s>>>(gb);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_gemm_tn_split(const GemmBatch<T>& gb, int n_prob, int max_d, int max_n, const T* c_base,
                                 T* partial, size_t split_stride, int splits, cudaStream_t s) {
  if (n_prob == 0 || max_d == 0 || max_n == 0) return cudaSuccess;
  const int n_tiles = (max_n + TN_BN - 1) / TN_BN;
  dim3 grid((max_d + TN_BD - 1) / TN_BD, n_tiles * splits, n_prob);
  gemm_tn_kernel<T><<<grid, 256, 0, s>>>(gb, c_base, partial, split_stride, splits);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_sum_splits(const T* partial, size_t split_stride, int splits, T* out, long long n, int accumulate,
                              cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  sum_splits_kernel<T><<<(unsigned)((n + 255) / 256), 256, 0, s>>>(partial, split_stride, splits, out, n, accumulate);
  return cudaGetLastError();
}

template cudaError_t launch_gemm<float>(int, const GemmBatch<float>&, int, int, int, cudaStream_t);
template cudaError_t launch_gemm<double>(int, const GemmBatch<double>&, int, int, int, cudaStream_t);
template cudaError_t launch_gemm_nt<float>(const GemmBatch<float>&, int, int, int, cudaStream_t);
template cudaError_t launch_gemm_nt<double>(const GemmBatch<double>&, int, int, int, cudaStream_t);
template cudaError_t launch_gemm_tn_split<float>(const GemmBatch<float>&, int, int, int, const float*, float*,
                                                 size_t, int, cudaStream_t);
template cudaError_t launch_gemm_tn_split<double>(const GemmBatch<double>&, int, int, int, const double*, double*,
                                                  size_t, int, cudaStream_t);
template cudaError_t launch_sum_splits<float>(const float*, size_t, int, float*, long long, int, cudaStream_t);
template cudaError_t launch_sum_splits<double>(const double*, size_t, int, double*, long long, int, cudaStream_t);

}  // namespace tpc
