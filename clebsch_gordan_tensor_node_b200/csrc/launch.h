// Host-side selection of the compiled kernel variant for a plan.
#pragma once

#include <type_traits>

#include "kernels.h"
#include "plan.h"

namespace tpc {

// Channelwise forward in the receiver-factorised order (uvu_state.cu): 32-channel
// tiles of the output blocks, K <= 8, degree profiles 0-3.
template <typename T>
cudaError_t launch_uvu_state_fwd(const UvuFwdParams<T>& p, int prof, cudaStream_t s);

// Edge pass of the uvu backward: radial width KP, gather width V, degree profile.
template <typename T>
cudaError_t launch_uvu_edge_for(const Plan& P, const UvuEdgeParams<T>& p, cudaStream_t s) {
  constexpr bool f32 = std::is_same<T, float>::value;
  constexpr int VW = f32 ? 4 : 2;
  if (P.KP == 8) {
    if (P.edge_V == VW) return launch_uvu_edge<T, 8, VW>(p, P.prof, s);
    return launch_uvu_edge<T, 8, 1>(p, P.prof, s);
  }
  if (P.edge_V == VW) return launch_uvu_edge<T, 16, VW>(p, P.prof, s);
  return launch_uvu_edge<T, 16, 1>(p, P.prof, s);
}

// Source pass of the uvu backward: radial width KP, channels per lane, profile.
// On entry p.n_slots is the most A_bar partial slots the caller's buffer holds;
// on return it is the number the launch used (the tile partition's).
template <typename T>
cudaError_t launch_uvu_src_for(const Plan& P, UvuSrcParams<T>& p, cudaStream_t s) {
  p.n_slots = uvu_src_partition(P, p.N, p.n_slots, p.tile_cta, &p.split);
  p.cy_stride = P.src_cy_stride;
  p.chunk = P.src_chunk;
  p.warp_smem = P.src_warp_smem;
  p.ring_off = P.src_ring_off;
  if constexpr (std::is_same<T, float>::value) {
    if (P.CPL == 2) return P.KP == 8 ? launch_uvu_src<T, 8, 2>(p, P.prof, s) : launch_uvu_src<T, 16, 2>(p, P.prof, s);
  }
  return P.KP == 8 ? launch_uvu_src<T, 8, 1>(p, P.prof, s) : launch_uvu_src<T, 16, 1>(p, P.prof, s);
}

}  // namespace tpc
