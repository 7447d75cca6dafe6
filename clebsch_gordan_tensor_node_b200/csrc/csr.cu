// Receiver CSR and its source transpose, on the device.
//
// LunaTP §4.1 keeps the adjacency as a CSR by destination (edges of node i in
// [rowptr[i], rowptr[i+1])); LunaTP §4.4 and Sobek §4.3 add a source-ordered
// view so that the node-feature gradient has one owner and one fixed order per
// source row. Sobek §4.5 asks for stable views: within a receiver the edges keep
// their input order, within a source the CSR positions stay ascending.
//
// Build: count per row (integer atomics; the counts do not depend on order),
// exclusive scan, scatter with an atomic cursor, then sort each row segment by
// the original index, which restores the stable order exactly. Rows of up to 256
// entries sort in shared memory (one warp per row); longer rows sort in place in
// global memory (one CTA per row). Every result is integer and bit-exact.
#include <climits>

#include "common.cuh"
#include "kernels.h"

namespace tpc {
namespace {

constexpr int kSmallRow = 256;

__global__ void count_kernel(const int* __restrict__ key, const int* __restrict__ other, int n_keys,
                             long long n, int* __restrict__ cnt, int* err) {
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= n) return;
  const int k = key[t];
  const bool bad = (unsigned)k >= (unsigned)n_keys || (other && (unsigned)other[t] >= (unsigned)n_keys);
  if (bad) {
    atomicOr(err, kErrIndex);
    return;
  }
  atomicAdd(cnt + k, 1);
}

// Exclusive scan of cnt[0..n) into ptr[0..n] and cur[0..n); one CTA of 1024 threads.
__global__ void __launch_bounds__(1024) scan_kernel(const int* __restrict__ cnt, int n,
                                                    int* __restrict__ ptr, int* __restrict__ cur) {
  __shared__ long long part[1024];
  const int t = threadIdx.x;
  const long long per = ((long long)n + 1023) / 1024;
  const long long b = t * per, e = b + per < n ? b + per : n;
  long long s = 0;
  for (long long k = b; k < e; ++k) s += cnt[k];
  part[t] = s;
  __syncthreads();
  for (int o = 1; o < 1024; o <<= 1) {
    long long v = t >= o ? part[t - o] : 0;
    __syncthreads();
    part[t] += v;
    __syncthreads();
  }
  long long run = t ? part[t - 1] : 0;
  for (long long k = b; k < e; ++k) {
    ptr[k] = (int)run;
    cur[k] = (int)run;
    run += cnt[k];
  }
  if (t == 1023) ptr[n] = (int)part[1023];
}

__global__ void scatter_kernel(const int* __restrict__ key, const int* __restrict__ other, int n_keys,
                               long long n, int* __restrict__ cur, int* __restrict__ out) {
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= n) return;
  const int k = key[t];
  if ((unsigned)k >= (unsigned)n_keys || (other && (unsigned)other[t] >= (unsigned)n_keys)) return;
  const int pos = atomicAdd(cur + k, 1);
  out[pos] = (int)t;
}

// In-place ascending bitonic sort of v[0..n) where positions >= n act as +inf:
// every comparator puts the minimum at the lower index, so a pair with its upper
// element out of range is a no-op.
__device__ __forceinline__ void cmpx(int* v, int a, int b) {
  const int x = v[a], y = v[b];
  if (x > y) {
    v[a] = y;
    v[b] = x;
  }
}

__global__ void __launch_bounds__(kWarpsPerBlock * 32)
sort_small_rows_kernel(const int* __restrict__ ptr, int n_rows, int* __restrict__ vals) {
  __shared__ int buf[kWarpsPerBlock][kSmallRow];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int r = blockIdx.x * kWarpsPerBlock + w;
  if (r >= n_rows) return;
  const int b = ptr[r], n = ptr[r + 1] - b;
  if (n <= 1 || n > kSmallRow) return;
  int* v = buf[w];
  for (int k = lane; k < n; k += 32) v[k] = vals[b + k];
  int P = 1;
  while (P < n) P <<= 1;
  __syncwarp();
  for (int k = 2; k <= P; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = lane; i < P; i += 32) {
        const int l = (j == (k >> 1)) ? (i ^ (k - 1)) : (i ^ j);
        if (l > i && l < n) cmpx(v, i, l);
      }
      __syncwarp();
    }
  }
  for (int k = lane; k < n; k += 32) vals[b + k] = v[k];
}

__global__ void __launch_bounds__(1024) sort_large_rows_kernel(const int* __restrict__ ptr, int n_rows,
                                                               int* __restrict__ vals) {
  for (int r = blockIdx.x; r < n_rows; r += gridDim.x) {
    const int b = ptr[r], n = ptr[r + 1] - b;
    if (n <= kSmallRow) continue;
    int* v = vals + b;
    int P = 1;
    while (P < n) P <<= 1;
    for (int k = 2; k <= P; k <<= 1) {
      for (int j = k >> 1; j > 0; j >>= 1) {
        for (int i = threadIdx.x; i < P; i += blockDim.x) {
          const int l = (j == (k >> 1)) ? (i ^ (k - 1)) : (i ^ j);
          if (l > i && l < n) cmpx(v, i, l);
        }
        __syncthreads();
      }
    }
  }
}

// Entries past ptr_end[0] exist only when some index was invalid (the error word
// is set); they are filled with -1 so that nothing reads through them.
__global__ void fill_tail_kernel(const int* __restrict__ ptr_end, int n, int* __restrict__ vals) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t < n && t >= ptr_end[0]) vals[t] = -1;
}

__global__ void gather_kernel(const int* __restrict__ idx, const int* __restrict__ src, int n,
                              int* __restrict__ out) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t < n) {
    const int k = idx[t];
    out[t] = k < 0 ? -1 : src[k];
  }
}

// srcrecv[t] = receiver of CSR position srcedge[t] (upper bound search in rowptr).
__global__ void receiver_of_kernel(const int* __restrict__ rowptr, int n_rows,
                                   const int* __restrict__ pos, int n, int* __restrict__ out) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= n) return;
  const int k = pos[t];
  if (k < 0) {
    out[t] = -1;
    return;
  }
  int lo = 0, hi = n_rows;  // find the last i with rowptr[i] <= k
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (rowptr[mid] <= k) lo = mid; else hi = mid;
  }
  out[t] = lo;
}

cudaError_t sort_rows(const int* ptr, int n_rows, int* vals, cudaStream_t s) {
  if (n_rows == 0) return cudaSuccess;
  sort_small_rows_kernel<<<(n_rows + kWarpsPerBlock - 1) / kWarpsPerBlock, kWarpsPerBlock * 32, 0, s>>>(
      ptr, n_rows, vals);
  const int g = n_rows < 148 * 4 ? n_rows : 148 * 4;
  sort_large_rows_kernel<<<g, 1024, 0, s>>>(ptr, n_rows, vals);
  return cudaGetLastError();
}

}  // namespace

size_t csr_workspace_bytes(long long n_nodes) {
  return (((size_t)n_nodes + 1) * 2 * sizeof(int) + 255) / 256 * 256;
}

cudaError_t csr_build(int N, int E, const int* src, const int* dst, int* rowptr, int* senders,
                      int* perm, void* ws, int* err, cudaStream_t s) {
  int* cnt = static_cast<int*>(ws);
  int* cur = cnt + (N + 1);
  cudaError_t e = cudaMemsetAsync(cnt, 0, sizeof(int) * (size_t)(N + 1), s);
  if (e != cudaSuccess) return e;
  if (E > 0) count_kernel<<<(E + 255) / 256, 256, 0, s>>>(dst, src, N, E, cnt, err);
  scan_kernel<<<1, 1024, 0, s>>>(cnt, N, rowptr, cur);
  if (E > 0) scatter_kernel<<<(E + 255) / 256, 256, 0, s>>>(dst, src, N, E, cur, perm);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if ((e = sort_rows(rowptr, N, perm, s)) != cudaSuccess) return e;
  if (E > 0) fill_tail_kernel<<<(E + 255) / 256, 256, 0, s>>>(rowptr + N, E, perm);
  if (E > 0) gather_kernel<<<(E + 255) / 256, 256, 0, s>>>(perm, src, E, senders);
  return cudaGetLastError();
}

cudaError_t csr_transpose(int N, int E, const int* rowptr, const int* senders, int* colptr,
                          int* srcedge, int* srcrecv, void* ws, int* err, cudaStream_t s) {
  int* cnt = static_cast<int*>(ws);
  int* cur = cnt + (N + 1);
  cudaError_t e = cudaMemsetAsync(cnt, 0, sizeof(int) * (size_t)(N + 1), s);
  if (e != cudaSuccess) return e;
  if (E > 0) count_kernel<<<(E + 255) / 256, 256, 0, s>>>(senders, nullptr, N, E, cnt, err);
  scan_kernel<<<1, 1024, 0, s>>>(cnt, N, colptr, cur);
  if (E > 0) scatter_kernel<<<(E + 255) / 256, 256, 0, s>>>(senders, nullptr, N, E, cur, srcedge);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if ((e = sort_rows(colptr, N, srcedge, s)) != cudaSuccess) return e;
  if (E > 0) fill_tail_kernel<<<(E + 255) / 256, 256, 0, s>>>(colptr + N, E, srcedge);
  if (E > 0) receiver_of_kernel<<<(E + 255) / 256, 256, 0, s>>>(rowptr, N, srcedge, E, srcrecv);
  return cudaGetLastError();
}

}  // namespace tpc
