// Compile-time limits shared by the planner and the kernels.
#pragma once

namespace tpc {

constexpr int kLmax = 4;          // largest degree (l1, l2, l3) of the fully connected kernels
constexpr int kLmaxUvu = 6;       // largest degree of the channelwise kernels (fp32, K <= 8 above kLmax)
constexpr int kMaxPaths = 192;    // paths per plan (kernel parameter space)
constexpr int kMaxTiles = 224;    // (block, channel tile) pairs per plan
constexpr int kWarpsPerBlock = 8; // warps per CTA of the warp-task kernels
constexpr int kSMs = 148;         // streaming multiprocessors of a B200
constexpr int kTnSplits = 8;      // split-K partial copies of A_bar in the uvw backward

// Warps per CTA and CTAs per SM of the uvu source pass and forward: one CTA of
// 16 warps for fp32; two CTAs of 4 warps for fp64 (whose path bodies need more
// than 128 registers per thread), which spreads small graphs over twice the SMs.
#ifdef __CUDACC__
__host__ __device__
#endif
constexpr int src_warps_for(int scalar_bytes) { return scalar_bytes == 4 ? 16 : 4; }
#ifdef __CUDACC__
__host__ __device__
#endif
constexpr int ctas_per_sm_for(int scalar_bytes) { return scalar_bytes == 4 ? 1 : 2; }

// Warps per CTA of the second-order passes (one channel per lane).
constexpr int kDbWarps = 8;
template <typename T>
#ifdef __CUDACC__
__host__ __device__
#endif
constexpr int src_warps() { return src_warps_for(sizeof(T)); }

// Warps per CTA of the uvu forward (CTAs per SM as for the source pass).
#ifdef __CUDACC__
__host__ __device__
#endif
constexpr int fwd_warps_for(int scalar_bytes) { return scalar_bytes == 4 ? 16 : 4; }
template <typename T>
#ifdef __CUDACC__
__host__ __device__
#endif
constexpr int fwd_warps() { return fwd_warps_for(sizeof(T)); }

// Edges per group of the forward's x copy ring (two groups per warp in
// flight): 4 while the widest input block has at most 3 components, else 2,
// which leaves shared memory for a full 32-edge staged chunk (the ring restarts
// with every path of every chunk, so long chunks matter more than deep groups).
#ifdef __CUDACC__
__host__ __device__
#endif
constexpr int fwd_ring_g(int scalar_bytes, int cpl, int l1max) { return l1max <= 1 ? 4 : 2; }

// The same for the source pass's m_bar ring (widest output block, degree l3max).
#ifdef __CUDACC__
__host__ __device__
#endif
constexpr int src_ring_g(int scalar_bytes, int cpl, int l3max) { return l3max <= 1 ? 4 : 2; }

}  // namespace tpc
