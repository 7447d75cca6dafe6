// Channelwise backward for callers that cannot allocate device memory.
//
// tp_conv_backward needs a caller-provided device workspace for the partial sums
// of grad_A. Some callers cannot obtain one at the point where they run the
// backward: a plugin called from another engine's execution step, where
// allocating is forbidden or would synchronise the device; code that runs while
// a stream capture is open; a process confined to a fixed memory reservation
// that it cannot grow. tp_conv_backward_noalloc serves them: it runs the same
// kernels as tp_conv_backward, but the grad_A partials live in one fixed array
// of device memory defined in this file, so the call itself allocates nothing.
//
// The array holds kNoAllocScratchBytes (16 MiB). Every GPU that loads the library
// keeps that much device memory reserved until the process exits. The number of
// partial-sum slots of the source pass is cut so that they fit; the results
// differ from tp_conv_backward only by the order of the grad_A additions.
#include <cstring>
#include <mutex>
#include <string>

#include "kernels.h"
#include "launch.h"
#include "plan.h"
#include "tpconv.h"

struct tp_plan_s {
  tpc::Plan p;
};

// Size of the scratch below: 16 MiB.
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;

// The scratch itself. In host code this name is only a stand-in for the device
// symbol, not a device address: the address comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace tpc {
namespace {

constexpr int kMaxDev = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDev] = {};

// Device address of the scratch on the current device, looked up once per
// device (with that device current) and cached.
int scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return set_error_message(TP_ECUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDev) return set_error_message(TP_EUNSUPPORTED, "device ordinal above 63");
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress((void**)&ptr, g_noalloc_scratch);
    if (e != cudaSuccess)
      return set_error_message(TP_ECUDA, std::string("cudaGetSymbolAddress(no-alloc scratch): ") +
                                             cudaGetErrorString(e));
    g_scratch_ptr[dev] = ptr;
  }
  *out = g_scratch_ptr[dev];
  return TP_OK;
}

template <typename T>
int run(const Plan& P, const void* x, const void* Y, const void* phi, const void* A, const int* rowptr,
        const int* senders, const int* colptr, const int* srcedge, const int* srcrecv, const void* gout,
        int N, int E, void* gx, void* gY, void* gphi, void* gA, void* scratch, int slots, int* err,
        cudaStream_t s) {
  UvuEdgeParams<T> ep;
  ep.x = (const T*)x; ep.Y = (const T*)Y; ep.phi = (const T*)phi; ep.A = (const T*)A;
  ep.gout = (const T*)gout; ep.rowptr = rowptr; ep.senders = senders;
  ep.gY = (T*)gY; ep.gphi = (T*)gphi; ep.err = err;
  ep.N = N; ep.E = E; ep.K = P.K; ep.c_in = P.c_in; ep.c_out = P.c_out; ep.dim_y = P.dim_y;
  ep.n_w = (int)P.n_w; ep.n_paths = (int)P.paths_canon.size();
  std::memset(ep.paths, 0, sizeof(ep.paths));
  std::memcpy(ep.paths, P.paths_canon.data(), P.paths_canon.size() * sizeof(PathD));
  cudaError_t e = launch_uvu_edge_for<T>(P, ep, s);
  if (e != cudaSuccess) return set_error_message(TP_ECUDA, std::string("edge pass: ") + cudaGetErrorString(e));

  UvuSrcParams<T> sp;
  sp.x = (const T*)x; sp.Y = (const T*)Y; sp.phi = (const T*)phi; sp.A = (const T*)A;
  sp.gout = (const T*)gout; sp.colptr = colptr; sp.srcedge = srcedge; sp.srcrecv = srcrecv;
  sp.gx = (T*)gx; sp.apart = (T*)scratch; sp.err = err;
  sp.N = N; sp.E = E; sp.K = P.K; sp.c_in = P.c_in; sp.c_out = P.c_out; sp.dim_y = P.dim_y;
  sp.n_w = (int)P.n_w;
  sp.n_slots = slots;
  std::memset(sp.tiles, 0, sizeof(sp.tiles));
  std::memset(sp.paths, 0, sizeof(sp.paths));
  std::memcpy(sp.tiles, P.in_tiles.data(), P.in_tiles.size() * sizeof(TileD));
  std::memcpy(sp.paths, P.paths_by_in.data(), P.paths_by_in.size() * sizeof(PathD));
  sp.n_tiles = (int)P.in_tiles.size();
  // launch_uvu_src first clears the slots it uses (the scratch keeps the previous
  // call's contents), then accumulates into them
  e = launch_uvu_src_for<T>(P, sp, s);
  if (e != cudaSuccess) return set_error_message(TP_ECUDA, std::string("source pass: ") + cudaGetErrorString(e));
  e = launch_reduce_slots<T>((const T*)scratch, (T*)gA, sp.n_slots, (long long)P.K * P.n_w, s);
  if (e != cudaSuccess) return set_error_message(TP_ECUDA, std::string("grad_A reduction: ") + cudaGetErrorString(e));
  return TP_OK;
}

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace tpc

using namespace tpc;

extern "C" int tp_conv_backward_noalloc(tp_plan_t plan, const void* x, const void* Y, const void* phi,
                                        const void* A, const int32_t* rowptr, const int32_t* senders,
                                        const int32_t* colptr, const int32_t* srcedge,
                                        const int32_t* srcrecv, const void* grad_out, int64_t n_nodes,
                                        int64_t n_edges, void* grad_x, void* grad_Y, void* grad_phi,
                                        void* grad_A, void* stream) {
  if (!plan) return set_error_message(TP_EINVAL, "NULL plan");
  const Plan& P = plan->p;
  if (P.mode != TP_UVU)
    return set_error_message(TP_EUNSUPPORTED, "the no-alloc backward covers channelwise (uvu) plans only");
  if (n_nodes < 0 || n_edges < 0 || n_nodes >= (1LL << 31) - 1 || n_edges >= (1LL << 31) - 1)
    return set_error_message(TP_EINVAL, "N and E must be in [0, 2^31 - 1)");
  if (!x || !A || !rowptr || !colptr || !grad_out || !grad_x || !grad_A ||
      (n_edges > 0 && (!Y || !phi || !senders || !srcedge || !srcrecv || !grad_Y || !grad_phi)))
    return set_error_message(TP_EINVAL, "NULL device pointer");
  const void* f[] = {x, A, grad_out, grad_x, grad_A};
  for (const void* q : f)
    if (!al16(q)) return set_error_message(TP_EINVAL, "floating-point buffers must be 16-byte aligned");
  if (n_edges > 0 && (!al16(Y) || !al16(phi) || !al16(grad_Y) || !al16(grad_phi)))
    return set_error_message(TP_EINVAL, "floating-point buffers must be 16-byte aligned");
  const size_t bsz = P.dtype == TP_F32 ? 4 : 8;
  const size_t per_slot = (size_t)P.K * (size_t)P.n_w * bsz;
  const size_t fit = kNoAllocScratchBytes / per_slot;
  if (fit == 0)
    return set_error_message(TP_EWORKSPACE, "grad_A partials need " + std::to_string(per_slot) +
                                                " bytes per slot (K * N_w * scalar size); the no-alloc "
                                                "scratch holds " + std::to_string(kNoAllocScratchBytes) +
                                                " bytes");
  cudaStream_t s = (cudaStream_t)stream;
  if (n_nodes == 0) {
    cudaError_t e = cudaMemsetAsync(grad_A, 0, per_slot, s);
    return e == cudaSuccess ? TP_OK : set_error_message(TP_ECUDA, "memset grad_A");
  }
  int* err = nullptr;
  int st = device_error_word(&err);
  if (st) return st;
  void* scratch = nullptr;
  if ((st = scratch_address(&scratch))) return st;
  const int slots = (int)std::min<size_t>(fit, 1 << 30);   // the source pass uses at most this many
  return P.dtype == TP_F32
             ? run<float>(P, x, Y, phi, A, rowptr, senders, colptr, srcedge, srcrecv, grad_out, (int)n_nodes,
                          (int)n_edges, grad_x, grad_Y, grad_phi, grad_A, scratch, slots, err, s)
             : run<double>(P, x, Y, phi, A, rowptr, senders, colptr, srcedge, srcrecv, grad_out, (int)n_nodes,
                           (int)n_edges, grad_x, grad_Y, grad_phi, grad_A, scratch, slots, err, s);
}
