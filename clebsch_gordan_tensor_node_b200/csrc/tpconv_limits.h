// Compile-time limits shared by the planner and the kernels.
#pragma once

namespace tpc {

constexpr int kLmax = 4;          // largest degree (l1, l2, l3) the kernels are built for
constexpr int kMaxPaths = 192;    // paths per plan (kernel parameter space)
constexpr int kMaxTiles = 96;     // (block, channel tile) pairs per plan
constexpr int kWarpsPerBlock = 8; // warps per CTA of the warp-task kernels
constexpr int kSMs = 148;         // streaming multiprocessors of a B200

// Warps per CTA of the uvu source pass, which runs one CTA per SM: 16 for fp32,
// 8 for fp64 (whose path bodies need more than 128 registers per thread).
#ifdef __CUDACC__
__host__ __device__
#endif
constexpr int src_warps_for(int scalar_bytes) { return scalar_bytes == 4 ? 16 : 8; }
template <typename T>
#ifdef __CUDACC__
__host__ __device__
#endif
constexpr int src_warps() { return src_warps_for(sizeof(T)); }

}  // namespace tpc
