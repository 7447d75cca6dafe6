// Launchers of the tensor-product convolution kernels (internal to the library).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"

namespace tpc {

template <typename T, int KP, int CPL, int L1M, int L2M, int L3M>
cudaError_t launch_uvu_fwd(const UvuFwdParams<T>& p, cudaStream_t s);

// V: channels per 16-byte (fp32: 4) or 8/16-byte (fp64: 2) gather; prof: degree profile
template <typename T, int KP, int V>
cudaError_t launch_uvu_edge(const UvuEdgeParams<T>& p, int prof, cudaStream_t s);

template <typename T, int KP, int CPL>
cudaError_t launch_uvu_src(const UvuSrcParams<T>& p, int prof, cudaStream_t s);

template <typename T>
cudaError_t launch_reduce_slots(const T* part, T* out, int n_slots, long long n, cudaStream_t s);

// second-order program of the channelwise path: receiver pass (m_dot), edge
// pass (phi_bar_dot, Y_bar_dot; V channels per gather) and source pass
// (x_bar_dot, A_bar_dot slot partials, zeroed first)
template <typename T, int KP, int CPL>
cudaError_t launch_uvu_dbwd_recv(const UvuDbwdParams<T>& p, int prof, cudaStream_t s);
template <typename T, int KP, int V>
cudaError_t launch_uvu_dbwd_edge(const UvuDbwdParams<T>& p, int prof, cudaStream_t s);
template <typename T, int KP, int CPL>
cudaError_t launch_uvu_dbwd_src(const UvuDbwdParams<T>& p, int prof, cudaStream_t s);

template <typename T, int KP, int DIR>
cudaError_t launch_uvw_sbuild_dir(const UvwSParams<T>& p, cudaStream_t s);

template <typename T, int KP>
cudaError_t launch_uvw_edge(const UvwEdgeParams<T>& p, cudaStream_t s);

// Bf, Ba: SIMT operand layouts; Btf / Bta: transposed (K-major) operands, holding
// the TF32-exact high parts when Btf_lo / Bta_lo are given (which get the rest).
template <typename T>
cudaError_t launch_pack_a(const UvwPackParams& p, const T* A, T* Bf, T* Ba, T* Btf, T* Bta, T* Btf_lo,
                          T* Bta_lo, cudaStream_t s);

template <typename T>
cudaError_t launch_unpack_a(const UvwPackParams& p, const T* Bf, T* A, cudaStream_t s);

// op 0: C (+)= X B (C row-blocked); op 1: C = G B^T (dense); op 2: C (+)= X^T G (dense)
template <typename T>
cudaError_t launch_gemm(int op, const GemmBatch<T>& gb, int n_prob, int max_m, int max_n, cudaStream_t s);
// backward products: S_bar = m_bar B^T, and the split-K A_bar partials with
// their fixed-order sum (kTnSplits partial copies of the packed-A layout)
template <typename T>
cudaError_t launch_gemm_nt(const GemmBatch<T>& gb, int n_prob, int max_m, int max_d, cudaStream_t s);
template <typename T>
cudaError_t launch_gemm_tn_split(const GemmBatch<T>& gb, int n_prob, int max_d, int max_n, const T* c_base,
                                 T* partial, size_t split_stride, int splits, cudaStream_t s);
template <typename T>
cudaError_t launch_sum_splits(const T* partial, size_t split_stride, int splits, T* out, long long n, int accumulate,
                              cudaStream_t s);

// op 0 on tensor cores (fp32, 3xTF32): C (+)= X Bt^T with X [M, D] and Bt [N, D]
// row-major, read through TMA tensor maps (box 32 x 128 for X, 32 x N16 for Bt).
struct TcProb {
  CUtensorMap tx, tbh, tbl;   // X (raw), Bt_hi, Bt_lo
  float* C;
  RowBlocked c;
  int M, N, D, accumulate;    // accumulate: add to C instead of overwriting it
};
struct TcBatch {
  TcProb prob[kMaxGemmBatch];
};
bool tc_gemm_available();
bool tc_make_map(CUtensorMap* map, const float* base, long long rows, long long cols, int box_rows);
cudaError_t launch_gemm_tc(const TcBatch& tb, int n_prob, int max_m, int npmax, int* err, cudaStream_t s);

size_t csr_workspace_bytes(long long n_nodes);
cudaError_t csr_build(int N, int E, const int* src, const int* dst, int* rowptr, int* senders, int* perm,
                      void* ws, int* err, cudaStream_t s);
cudaError_t csr_transpose(int N, int E, const int* rowptr, const int* senders, int* colptr, int* srcedge,
                          int* srcrecv, void* ws, int* err, cudaStream_t s);

}  // namespace tpc

// Explicit instantiations are split over several compilations of the same file
// (-DTPC_SET=k builds only set k) so that the build runs in parallel.
#ifndef TPC_SET
#define TPC_SET -1
#endif
#define TPC_WANT(k) (TPC_SET < 0 || TPC_SET == (k))

#include <string>

namespace tpc {
// Record a host-side failure for tp_last_error_message; returns status.
int set_error_message(int status, const std::string& msg);
// Device address of the current device's error word.
int device_error_word(int** out);
}  // namespace tpc
