// Shared device-side definitions of the tensor-product convolution kernels.
//
// Layouts (Sobek §4.5: ir_mul, channels contiguous inside each irrep block):
//   x   [N, C_x]      row j: blocks in irreps order, each [2l+1][mul]
//   out [N, C_out]    same layout for the output irreps
//   Y   [E, (L+1)^2]  CSR edge order, blocks l = 0..L, m = -l..l
//   phi [E, K]        CSR edge order
//   A   [K, N_w]      path pi in columns [w_off, w_off + n_w); uvu column = u,
//                     uvw column = u * C_out + w
// Indices are int32; scalars are float or double (the plan's dtype).
#pragma once

#include <atomic>
#include <cstdint>
#include <type_traits>
#include <utility>

#include "cg_table.inc"
#include "tpconv_limits.h"

namespace tpc {

using cgt::Pair;
using cgt::Term;

// ------------------------------------------------------------------ descriptors

struct PathD {          // one coupling path (l1, l2) -> l3
  int8_t l1, l2, l3, pad;
  int x_off;            // input block offset in an x row
  int out_off;          // output block offset in an out row
  int w_off;            // first column of the path in A
  int mul_in;
  int mul_out;
  int cy_off;           // forward: first cY slot of the path in a staged edge row
  int col_off;          // uvw: first column of the path in its owner block's state row
};

struct TileD {          // one channel tile of one irrep block
  int l;                // degree of the block
  int off;              // block offset in its row
  int mul;              // block multiplicity
  int ch0;              // first channel of the tile
  int nch;              // channels in the tile
  int pbeg, pend;       // paths of the block, in the kernel's path array
};

// Device error word bits (read back by tp_get_device_error).
enum : int { kErrIndex = 1, kErrCsr = 2, kErrTimeout = 4 };

template <typename T>
struct UvuFwdParams {
  const T* x; const T* Y; const T* phi; const T* A;
  const int* rowptr; const int* senders;
  T* out; int* err;
  int N, E, K, c_in, c_out, dim_y, n_w;
  int n_tiles;
  int cy_stride;              // cY slots per staged edge (max over tiles, padded)
  int chunk;                  // edges staged per warp at a time (<= 32)
  int warp_smem;              // bytes of shared memory per warp
  int ring_off;               // x copy ring: byte offset in the warp's slice
  int split;                  // 1, or the warps of a CTA that share one task and deal its paths (small graphs)
  TileD tiles[kMaxTiles];     // one per (output block, channel tile)
  PathD paths[kMaxPaths];     // grouped by output block
};

template <typename T>
struct UvuEdgeParams {        // backward: edge-owned grad_phi, grad_Y
  const T* x; const T* Y; const T* phi; const T* A; const T* gout;
  const int* rowptr; const int* senders;
  T* gY; T* gphi; int* err;
  int N, E, K, c_in, c_out, dim_y, n_w;
  int n_paths;
  int split;                  // warps that share one group of 32 edges (paths dealt round-robin)
  PathD paths[kMaxPaths];     // canonical order
};

template <typename T>
struct UvuSrcParams {         // backward: source-owned grad_x, grad_A partials
  const T* x; const T* Y; const T* phi; const T* A; const T* gout;
  const int* colptr; const int* srcedge; const int* srcrecv;
  T* gx; T* apart; int* err;
  int N, E, K, c_in, c_out, dim_y, n_w;
  int n_tiles, n_slots;
  int cy_stride;              // cY slots per staged edge (max over tiles, padded)
  int chunk;                  // edges staged per warp at a time (<= 32)
  int warp_smem;              // bytes of shared memory per warp
  int ring_off;               // m_bar copy ring: byte offset in the warp's slice
  int split;                  // 1, or the warps of a CTA that share each source and deal the tile's paths
  int tile_cta[kMaxTiles + 1];  // CTAs [tile_cta[t], tile_cta[t + 1]) serve tile t
  TileD tiles[kMaxTiles];     // one per (input block, channel tile)
  PathD paths[kMaxPaths];     // grouped by input block
};

// Second-order program of the channelwise path (Sobek §3.3): directions
// (dx, dY, dphi, dA) of the four inputs, the output adjoint gout held fixed.
template <typename T>
struct UvuDbwdParams {
  const T* x; const T* Y; const T* phi; const T* A; const T* gout;
  const T* dx; const T* dY; const T* dphi; const T* dA;
  const int* rowptr; const int* senders;
  const int* colptr; const int* srcedge; const int* srcrecv;
  T* mdot;                    // receiver pass: directional output [N, C_out]
  T* gY; T* gphi;             // edge pass: directional Y_bar [E, dimY], phi_bar [E, K]
  T* gx; T* apart;            // source pass: directional x_bar [N, C_in]; A_bar slot partials
  int* err;
  int N, E, K, c_in, c_out, dim_y, n_w;
  int n_paths, n_tiles, n_slots;
  int split;                  // edge pass: warps sharing one group of 32 edges
  int tile_cta[kMaxTiles + 1];  // source pass: CTAs [tile_cta[t], tile_cta[t + 1]) serve tile t
  TileD tiles[kMaxTiles];     // receiver pass: (output block, 32-channel tile); source pass: input blocks
  PathD paths[kMaxPaths];     // receiver pass: by output block; source pass: by input block; edge pass: canonical
};

// ---- fully connected (uvw) path

constexpr int kMaxBlocks = 32;

struct UvwBlockD {      // owner block of a receiver-state (S) or source-state (S') build
  int l;                // degree of the owner block
  int pbeg, pend;       // its paths in the kernel's path array
  int dcols;            // state columns per owner row: sum over paths of K * gathered mul
  long long s_off;      // region of the block in a state chunk, in units of chunk rows
  int out_off;          // owner block offset in the owner's row (out or grad_x)
  int mul_own;          // multiplicity of the owner block
};

template <typename T>
struct UvwSParams {           // S (dir 0: receivers gather x) or S' (dir 1: sources gather grad_out)
  const T* feat; const T* Y; const T* phi;
  const int* ptr; const int* nbr; const int* eid;   // eid = NULL: edge id = position
  T* S; int* err;
  int N, E, K, ld_feat, dim_y, n_feat_rows;
  int r0, nr, nr_alloc, n_blocks;
  int accumulate;             // add to the state chunk instead of overwriting it
  UvwBlockD blocks[kMaxBlocks];
  PathD paths[kMaxPaths];     // x_off / mul_in describe the gathered block
};

// Edge pass of the uvw backward: input channels staged per tile, warps per
// CTA, and the per-sender row stride in the staging buffer for a tile row of n
// scalars: odd, so that 32 lanes reading one scalar each from their own row
// hit 32 distinct banks.
constexpr int kEdgeTile = 16;
constexpr int kEdgeWarps = 4, kEdgeThreads = 32 * kEdgeWarps;
__host__ __device__ constexpr int edge_slot_stride(int n) { return n | 1; }

template <typename T>
struct UvwEdgeParams {        // backward: edge-owned grad_phi, grad_Y from S_bar
  const T* x; const T* Y; const T* phi; const T* Sbar;   // S_bar columns per path: (u, q)
  const int* rowptr; const int* senders;
  T* gY; T* gphi; int* err;
  int N, E, K, c_in, dim_y;
  int r0, nr, nr_alloc, n_blocks;
  int accumulate;              // add to grad_phi / grad_Y instead of overwriting them
  int vec;                     // 16-byte copies: K == KP; c_in, x_off, mul_in multiples of 16 bytes
  int smem_stage, smem_sbar;   // bytes of one stage buffer (x part, then S_bar part) and its S_bar part
  int smem_red, smem_ct;       // bytes of the per-warp Y_bar region and of the C / T_bar columns
  int8_t path_blk[kMaxPaths];  // owner block of each path
  UvwBlockD blocks[kMaxBlocks];
  PathD paths[kMaxPaths];
};

struct PackPath {       // where the A columns of one path go in the packed GEMM operands
  int w_off, mi, mo, colf, cola;
  int dcf, dca;         // state columns of the path's output block / input block
  long long bf_off, ba_off;
};

struct UvwPackParams {
  int K, n_w, n_paths;
  int bf_uq;            // rows of Bf per path in (u, q) order instead of (q, u)
  PackPath paths[kMaxPaths];
};

struct RowBlocked {     // row m = (owner r, component c) -> (r0 + r) * ld_outer + off + c * n
  int r0, dcomp;
  long long ld_outer;
  int off, n;
};

template <typename T>
struct GemmProb {
  const T* X; const T* B; const T* G; T* C;
  RowBlocked g, c;
  int M, N, D, accumulate;
};

constexpr int kMaxGemmBatch = 16;

template <typename T>
struct GemmBatch {
  GemmProb<T> prob[kMaxGemmBatch];
};

// ------------------------------------------------------------------ compile-time helpers

template <typename F, int... I>
__device__ __forceinline__ void static_for_impl(F&& f, std::integer_sequence<int, I...>) {
  (f(std::integral_constant<int, I>{}), ...);
}

template <int N, typename F>
__device__ __forceinline__ void static_for(F&& f) {
  static_for_impl(f, std::make_integer_sequence<int, N>{});
}

__host__ __device__ constexpr bool triangle(int a, int b, int c) {
  return c >= (a > b ? a - b : b - a) && c <= a + b;
}

// True if pair P of CG<L1,L2,L3> is the first pair that writes output component m3.
template <class CGp>
__host__ __device__ constexpr bool first_m3(int P) {
  for (int k = 0; k < P; ++k)
    if (CGp::pair[k].m3 == CGp::pair[P].m3) return false;
  return true;
}
// True if pair P is the first pair that reads input component m1.
template <class CGp>
__host__ __device__ constexpr bool first_m1(int P) {
  for (int k = 0; k < P; ++k)
    if (CGp::pair[k].m1 == CGp::pair[P].m1) return false;
  return true;
}
// True if component m3 of CG<L1,L2,L3> receives any pair.
template <class CGp>
__host__ __device__ constexpr bool has_m3(int m3) {
  for (int k = 0; k < CGp::npair; ++k)
    if (CGp::pair[k].m3 == m3) return true;
  return false;
}
template <class CGp>
__host__ __device__ constexpr bool has_m1(int m1) {
  for (int k = 0; k < CGp::npair; ++k)
    if (CGp::pair[k].m1 == m1) return true;
  return false;
}

// cY = sum over the terms of pair P of c * y[m2] (y holds the degree-L2 block).
template <typename T, class CGp, int P>
__device__ __forceinline__ T pair_coef(const T* y) {
  constexpr Pair pr = CGp::pair[P];
  T cy = T(CGp::term[pr.start].c) * y[CGp::term[pr.start].m2];
  static_for<pr.n - 1>([&](auto t) {
    constexpr Term tm = CGp::term[pr.start + 1 + decltype(t)::value];
    cy = fma(T(tm.c), y[tm.m2], cy);
  });
  return cy;
}

// Call f(integral_constant<L1>, integral_constant<L2>) for the runtime (l1, l2)
// among the pairs that can couple into L3 (degrees up to LM).
template <int L3, int L1M = kLmax, int L2M = kLmax, typename F>
__device__ __forceinline__ void dispatch_l1l2(int l1, int l2, F&& f) {
  static_for<L1M + 1>([&](auto A1) {
    static_for<L2M + 1>([&](auto A2) {
      constexpr int a = decltype(A1)::value, b = decltype(A2)::value;
      if constexpr (triangle(a, b, L3)) {
        if (l1 == a && l2 == b) f(A1, A2);
      }
    });
  });
}

// Same for (l2, l3) at fixed L1.
template <int L1, int LM = kLmax, typename F>
__device__ __forceinline__ void dispatch_l2l3(int l2, int l3, F&& f) {
  static_for<LM + 1>([&](auto A2) {
    static_for<LM + 1>([&](auto A3) {
      constexpr int b = decltype(A2)::value, c = decltype(A3)::value;
      if constexpr (triangle(L1, b, c)) {
        if (l2 == b && l3 == c) f(A2, A3);
      }
    });
  });
}

// Same for one degree.
template <int LM = kLmax, typename F>
__device__ __forceinline__ void dispatch_l(int l, F&& f) {
  static_for<LM + 1>([&](auto A) {
    if (l == decltype(A)::value) f(A);
  });
}

// ------------------------------------------------------------------ memory helpers

template <typename T>
__device__ __forceinline__ T ldg(const T* p) { return __ldg(p); }

// Asynchronous copy of B bytes (4, 8 or 16) from global to shared memory, and
// its commit / wait (per thread: a thread waits only for its own copies).
template <int B>
__device__ __forceinline__ void cp_async_b(void* dst, const void* src) {
  const unsigned d = (unsigned)__cvta_generic_to_shared(dst);
  if constexpr (B == 16)
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(d), "l"(src) : "memory");
  else
    asm volatile("cp.async.ca.shared.global [%0], [%1], %2;\n" ::"r"(d), "l"(src), "n"(B) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }

// Load CPL consecutive scalars (8-byte aligned when CPL*sizeof(T) == 8).
template <int CPL, typename T>
__device__ __forceinline__ void load_ch(T (&v)[CPL], const T* p) {
  if constexpr (CPL == 2 && std::is_same<T, float>::value) {
    float2 t = __ldg(reinterpret_cast<const float2*>(p));
    v[0] = t.x; v[1] = t.y;
  } else if constexpr (CPL == 4 && std::is_same<T, float>::value) {
    float4 t = __ldg(reinterpret_cast<const float4*>(p));
    v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
  } else if constexpr (CPL == 2 && std::is_same<T, double>::value) {
    double2 t = __ldg(reinterpret_cast<const double2*>(p));
    v[0] = t.x; v[1] = t.y;
  } else {
#pragma unroll
    for (int c = 0; c < CPL; ++c) v[c] = __ldg(p + c);
  }
}

template <int CPL, typename T>
__device__ __forceinline__ void store_ch(T* p, const T (&v)[CPL]) {
  if constexpr (CPL == 2 && std::is_same<T, float>::value) {
    *reinterpret_cast<float2*>(p) = make_float2(v[0], v[1]);
  } else if constexpr (CPL == 4 && std::is_same<T, float>::value) {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  } else if constexpr (CPL == 2 && std::is_same<T, double>::value) {
    *reinterpret_cast<double2*>(p) = make_double2(v[0], v[1]);
  } else {
#pragma unroll
    for (int c = 0; c < CPL; ++c) p[c] = v[c];
  }
}

// K radial values of one edge, zero-padded to KP.
template <int KP, typename T>
__device__ __forceinline__ void load_phi(T (&ph)[KP], const T* row, int K) {
  if (K == KP) {
    if constexpr (std::is_same<T, float>::value && KP % 4 == 0) {
#pragma unroll
      for (int q = 0; q < KP; q += 4) {
        float4 t = __ldg(reinterpret_cast<const float4*>(row + q));
        ph[q] = t.x; ph[q + 1] = t.y; ph[q + 2] = t.z; ph[q + 3] = t.w;
      }
      return;
    } else if constexpr (std::is_same<T, double>::value && KP % 2 == 0) {
#pragma unroll
      for (int q = 0; q < KP; q += 2) {
        double2 t = __ldg(reinterpret_cast<const double2*>(row + q));
        ph[q] = t.x; ph[q + 1] = t.y;
      }
      return;
    }
  }
#pragma unroll
  for (int q = 0; q < KP; ++q) ph[q] = q < K ? __ldg(row + q) : T(0);
}

__device__ __forceinline__ void raise_error(int* err, int bit) {
  if ((threadIdx.x & 31) == 0) atomicOr(err, bit);
}

// Raise a kernel's dynamic shared-memory limit to at least `bytes` on the
// current device. The attribute call costs host time comparable to a small
// kernel, so each launcher keeps one SmemLimit per kernel instantiation and
// the call is made only when a device first needs more than it was given.
struct SmemLimit {
  std::atomic<int> granted[64] = {};
  cudaError_t ensure(const void* kernel, size_t bytes) {
    if (bytes <= 48 * 1024) return cudaSuccess;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64)
      return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (granted[dev].load(std::memory_order_acquire) >= (int)bytes) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess) {
      int cur = granted[dev].load();
      while (cur < (int)bytes && !granted[dev].compare_exchange_weak(cur, (int)bytes)) {
      }
    }
    return e;
  }
};

}  // namespace tpc
