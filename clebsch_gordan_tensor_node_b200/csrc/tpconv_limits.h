// Compile-time limits shared by the planner and the kernels.
#pragma once

namespace tpc {

constexpr int kLmax = 4;          // largest degree (l1, l2, l3) the kernels are built for
constexpr int kMaxPaths = 192;    // paths per plan (kernel parameter space)
constexpr int kMaxTiles = 96;     // (block, channel tile) pairs per plan
constexpr int kWarpsPerBlock = 8; // warps per CTA of the warp-task kernels

}  // namespace tpc
