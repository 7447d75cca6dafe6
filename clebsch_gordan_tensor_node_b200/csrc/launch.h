// Host-side selection of the compiled kernel variant for a plan.
#pragma once

#include <type_traits>

#include "kernels.h"
#include "plan.h"

namespace tpc {

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

}  // namespace tpc
