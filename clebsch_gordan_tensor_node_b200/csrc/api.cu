// C ABI of the tensor-product convolution library (declarations in tpconv.h).
#include <cstdint>
#include <cstring>
#include <mutex>
#include <string>

#include "cg_host.h"
#include "kernels.h"
#include "launch.h"
#include "plan.h"
#include "tpconv.h"

struct tp_plan_s {
  tpc::Plan p;
};

namespace tpc {
namespace {

thread_local std::string g_msg;

int fail(int status, const std::string& m) {
  g_msg = m;
  return status;
}

int cuda_fail(cudaError_t e, const char* where) {
  return fail(TP_ECUDA, std::string(where) + ": " + cudaGetErrorString(e));
}

// Per-device error word: kernels set bits here instead of trapping.
__device__ int g_error_word;

constexpr int kMaxDevices = 64;
std::mutex g_err_mu;
int* g_err_ptr[kMaxDevices] = {};

int error_word(int** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(TP_EUNSUPPORTED, "device ordinal above 63");
  std::lock_guard<std::mutex> lk(g_err_mu);
  if (!g_err_ptr[dev]) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_error_word);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(error word)");
    g_err_ptr[dev] = static_cast<int*>(ptr);
  }
  *out = g_err_ptr[dev];
  return TP_OK;
}

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_sizes(long long N, long long E) {
  if (N < 0 || E < 0) return fail(TP_EINVAL, "negative node or edge count");
  if (N >= (1LL << 31) - 1 || E >= (1LL << 31) - 1) return fail(TP_EINVAL, "N and E must be below 2^31 - 1");
  return TP_OK;
}

template <typename P>
void copy_tables(P& prm, const std::vector<TileD>& tiles, const std::vector<PathD>& paths) {
  std::memset(prm.tiles, 0, sizeof(prm.tiles));
  std::memset(prm.paths, 0, sizeof(prm.paths));
  std::memcpy(prm.tiles, tiles.data(), tiles.size() * sizeof(TileD));
  std::memcpy(prm.paths, paths.data(), paths.size() * sizeof(PathD));
  prm.n_tiles = (int)tiles.size();
}

template <typename T, int KP, int CPL, bool Full>
cudaError_t fwd_prof(const Plan& P, const UvuFwdParams<T>& p, cudaStream_t s) {
  switch (P.prof) {
    case 0: return launch_uvu_fwd<T, KP, CPL, 2, 2, 2>(p, s);
    case 1: return launch_uvu_fwd<T, KP, CPL, 1, 3, 3>(p, s);
    case 2: return launch_uvu_fwd<T, KP, CPL, 3, 3, 3>(p, s);
    case 3:
      if constexpr (Full) return launch_uvu_fwd<T, KP, CPL, 4, 4, 4>(p, s);
      return cudaErrorInvalidValue;
    default:   // degrees up to 6: fp32, K <= 8, one channel per lane
      if constexpr (std::is_same<T, float>::value && KP == 8 && CPL == 1)
        return launch_uvu_fwd<T, KP, CPL, 6, 6, 6>(p, s);
      return cudaErrorInvalidValue;
  }
}

// Mirrors the instantiation list of uvu_fwd.cu.
template <typename T>
cudaError_t fwd_dispatch(const Plan& P, const UvuFwdParams<T>& p, cudaStream_t s) {
  constexpr bool f32 = std::is_same<T, float>::value;
  if (P.KP == 8) {
    if (P.fwd_CPL == 1) return fwd_prof<T, 8, 1, true>(P, p, s);
    if (P.fwd_CPL == 2) return fwd_prof<T, 8, 2, f32>(P, p, s);
  } else {
    if (P.fwd_CPL == 1) return fwd_prof<T, 16, 1, true>(P, p, s);
    if (P.fwd_CPL == 2) return fwd_prof<T, 16, 2, f32>(P, p, s);
  }
  return cudaErrorInvalidValue;
}


template <typename T>
int forward_uvu(const Plan& P, const void* x, const void* Y, const void* phi, const void* A,
                const int* rowptr, const int* senders, int N, int E, void* out, int* err, cudaStream_t s) {
  UvuFwdParams<T> prm;
  if (P.schedule == TP_SCHED_RECEIVER_STATE) {
    std::memset(&prm, 0, sizeof(prm));
    prm.x = (const T*)x; prm.Y = (const T*)Y; prm.phi = (const T*)phi; prm.A = (const T*)A;
    prm.rowptr = rowptr; prm.senders = senders; prm.out = (T*)out; prm.err = err;
    prm.N = N; prm.E = E; prm.K = P.K; prm.c_in = P.c_in; prm.c_out = P.c_out; prm.dim_y = P.dim_y;
    prm.n_w = (int)P.n_w;
    copy_tables(prm, P.dbl_out_tiles, P.dbl_paths_by_out);
    cudaError_t e = launch_uvu_state_fwd<T>(prm, P.prof, s);
    return e == cudaSuccess ? TP_OK : cuda_fail(e, "uvu receiver-state forward launch");
  }
  prm.x = (const T*)x; prm.Y = (const T*)Y; prm.phi = (const T*)phi; prm.A = (const T*)A;
  prm.rowptr = rowptr; prm.senders = senders; prm.out = (T*)out; prm.err = err;
  prm.N = N; prm.E = E; prm.K = P.K; prm.c_in = P.c_in; prm.c_out = P.c_out; prm.dim_y = P.dim_y;
  prm.n_w = (int)P.n_w;
  prm.cy_stride = P.cy_stride;
  prm.chunk = P.fwd_chunk;
  prm.warp_smem = P.fwd_warp_smem;
  prm.ring_off = P.fwd_ring_off;
  copy_tables(prm, P.out_tiles, P.paths_by_out);
  cudaError_t e = fwd_dispatch<T>(P, prm, s);
  return e == cudaSuccess ? TP_OK : cuda_fail(e, "uvu forward launch");
}

template <typename T>
int backward_uvu(const Plan& P, const void* x, const void* Y, const void* phi, const void* A,
                 const int* rowptr, const int* senders, const int* colptr, const int* srcedge,
                 const int* srcrecv, const void* gout, int N, int E, void* gx, void* gY, void* gphi,
                 void* gA, void* ws, int* err, cudaStream_t s) {
  UvuEdgeParams<T> ep;
  ep.x = (const T*)x; ep.Y = (const T*)Y; ep.phi = (const T*)phi; ep.A = (const T*)A;
  ep.gout = (const T*)gout; ep.rowptr = rowptr; ep.senders = senders;
  ep.gY = (T*)gY; ep.gphi = (T*)gphi; ep.err = err;
  ep.N = N; ep.E = E; ep.K = P.K; ep.c_in = P.c_in; ep.c_out = P.c_out; ep.dim_y = P.dim_y;
  ep.n_w = (int)P.n_w; ep.n_paths = (int)P.paths_canon.size();
  std::memset(ep.paths, 0, sizeof(ep.paths));
  std::memcpy(ep.paths, P.paths_canon.data(), P.paths_canon.size() * sizeof(PathD));
  cudaError_t e = launch_uvu_edge_for<T>(P, ep, s);
  if (e != cudaSuccess) return cuda_fail(e, "uvu edge pass launch");

  UvuSrcParams<T> sp;
  sp.x = (const T*)x; sp.Y = (const T*)Y; sp.phi = (const T*)phi; sp.A = (const T*)A;
  sp.gout = (const T*)gout; sp.colptr = colptr; sp.srcedge = srcedge; sp.srcrecv = srcrecv;
  sp.gx = (T*)gx; sp.apart = (T*)ws; sp.err = err;
  sp.N = N; sp.E = E; sp.K = P.K; sp.c_in = P.c_in; sp.c_out = P.c_out; sp.dim_y = P.dim_y;
  sp.n_w = (int)P.n_w;
  sp.n_slots = 1 << 30;   // the workspace holds the partition's slots
  copy_tables(sp, P.in_tiles, P.paths_by_in);
  e = launch_uvu_src_for<T>(P, sp, s);
  if (e != cudaSuccess) return cuda_fail(e, "uvu source pass launch");
  e = launch_reduce_slots<T>((const T*)ws, (T*)gA, sp.n_slots, (long long)P.K * P.n_w, s);
  return e == cudaSuccess ? TP_OK : cuda_fail(e, "grad_A reduction launch");
}

// Second-order program (Sobek §3.3): receiver, edge and source passes, then the
// fixed-order sum of the A_bar_dot slot partials.
template <typename T>
int double_backward_uvu(const Plan& P, const void* const* in, const int* const* idx, const void* const* dir,
                        int N, int E, void* const* out, void* ws, int* err, cudaStream_t s) {
  UvuDbwdParams<T> p;
  std::memset(&p, 0, sizeof(p));
  p.x = (const T*)in[0]; p.Y = (const T*)in[1]; p.phi = (const T*)in[2]; p.A = (const T*)in[3];
  p.gout = (const T*)in[4];
  p.dx = (const T*)dir[0]; p.dY = (const T*)dir[1]; p.dphi = (const T*)dir[2]; p.dA = (const T*)dir[3];
  p.rowptr = idx[0]; p.senders = idx[1]; p.colptr = idx[2]; p.srcedge = idx[3]; p.srcrecv = idx[4];
  p.mdot = (T*)out[0]; p.gx = (T*)out[1]; p.gY = (T*)out[2]; p.gphi = (T*)out[3]; p.apart = (T*)ws;
  p.err = err;
  p.N = N; p.E = E; p.K = P.K; p.c_in = P.c_in; p.c_out = P.c_out; p.dim_y = P.dim_y; p.n_w = (int)P.n_w;
  const bool k8 = P.KP == 8;
  // receiver pass: m_dot (one channel per lane, 32-channel tiles)
  copy_tables(p, P.dbl_out_tiles, P.dbl_paths_by_out);
  cudaError_t e = k8 ? launch_uvu_dbwd_recv<T, 8, 1>(p, P.prof, s) : launch_uvu_dbwd_recv<T, 16, 1>(p, P.prof, s);
  if (e != cudaSuccess) return cuda_fail(e, "double backward receiver pass");
  // edge pass: phi_bar_dot, Y_bar_dot
  std::memset(p.paths, 0, sizeof(p.paths));
  std::memcpy(p.paths, P.paths_canon.data(), P.paths_canon.size() * sizeof(PathD));
  p.n_paths = (int)P.paths_canon.size();
  constexpr int VW = std::is_same<T, float>::value ? 4 : 2;
  if (P.edge_V == VW)
    e = k8 ? launch_uvu_dbwd_edge<T, 8, VW>(p, P.prof, s) : launch_uvu_dbwd_edge<T, 16, VW>(p, P.prof, s);
  else
    e = k8 ? launch_uvu_dbwd_edge<T, 8, 1>(p, P.prof, s) : launch_uvu_dbwd_edge<T, 16, 1>(p, P.prof, s);
  if (e != cudaSuccess) return cuda_fail(e, "double backward edge pass");
  // source pass: x_bar_dot and the A_bar_dot slot partials, then their sum
  p.n_slots = uvu_dbl_src_partition(P, N, p.tile_cta);
  copy_tables(p, P.dbl_in_tiles, P.dbl_paths_by_in);
  e = k8 ? launch_uvu_dbwd_src<T, 8, 1>(p, P.prof, s) : launch_uvu_dbwd_src<T, 16, 1>(p, P.prof, s);
  if (e != cudaSuccess) return cuda_fail(e, "double backward source pass");
  e = launch_reduce_slots<T>((const T*)ws, (T*)out[4], p.n_slots, (long long)P.K * P.n_w, s);
  return e == cudaSuccess ? TP_OK : cuda_fail(e, "double backward A_bar reduction");
}

// ---------------------------------------------------------------- uvw

bool use_tc(const Plan& P) { return P.uvw_tc; }

template <typename T>
cudaError_t sbuild(const Plan& P, const UvwSParams<T>& p, int dir, cudaStream_t s) {
  if (dir == 0) return P.KP == 8 ? launch_uvw_sbuild_dir<T, 8, 0>(p, s) : launch_uvw_sbuild_dir<T, 16, 0>(p, s);
  return P.KP == 8 ? launch_uvw_sbuild_dir<T, 8, 1>(p, s) : launch_uvw_sbuild_dir<T, 16, 1>(p, s);
}

template <typename T>
void fill_blocks(UvwSParams<T>& p, const std::vector<UvwBlockD>& blocks, const std::vector<PathD>& paths) {
  std::memset(p.blocks, 0, sizeof(p.blocks));
  std::memset(p.paths, 0, sizeof(p.paths));
  std::memcpy(p.blocks, blocks.data(), blocks.size() * sizeof(UvwBlockD));
  std::memcpy(p.paths, paths.data(), paths.size() * sizeof(PathD));
  p.n_blocks = (int)blocks.size();
}

size_t align256(size_t v) { return (v + 255) / 256 * 256; }

// m_g (+)= S_g B_g for every output block of one receiver chunk (rows -> out).
// Tensor-core plans: Bf holds Bt_hi and Blo Bt_lo (transposed, split); the
// SIMT GEMM reads Bf as B [D, N].
template <typename T>
cudaError_t mix_out(const Plan& P, const T* S, const T* Bf, const T* Blo, T* out, int r0, int nr, int nr_alloc,
                    const std::vector<UvwBlockD>& blocks, const std::vector<long long>& b_off, long long ld_out,
                    int accumulate, int* err, cudaStream_t s) {
  if constexpr (std::is_same<T, float>::value) {
    if (use_tc(P)) {
      TcBatch tb;
      int n = 0, mm = 0, npmax = 16;
      for (size_t g = 0; g < blocks.size(); ++g) {
        const UvwBlockD& b = blocks[g];
        const int dc = 2 * b.l + 1, M = nr * dc, N = b.mul_own, D = b.dcols;
        if (M == 0) continue;
        TcProb& q = tb.prob[n];
        const int np = (N + 15) / 16 * 16;
        const float* X = S + (size_t)nr_alloc * b.s_off;
        if (D > 0) {
          if (!tc_make_map(&q.tx, X, M, D, 128) || !tc_make_map(&q.tbh, Bf + b_off[g], N, D, np) ||
              !tc_make_map(&q.tbl, Blo + b_off[g], N, D, np))
            return cudaErrorInvalidValue;
        }
        q.C = out;
        q.c = RowBlocked{r0, dc, ld_out, b.out_off, N};
        q.M = M; q.N = N; q.D = D; q.accumulate = accumulate;
        ++n;
        mm = std::max(mm, M);
        npmax = std::max(npmax, np);
        if (n == kMaxGemmBatch) {
          cudaError_t e = launch_gemm_tc(tb, n, mm, npmax, err, s);
          if (e != cudaSuccess) return e;
          n = mm = 0;
          npmax = 16;
        }
      }
      return launch_gemm_tc(tb, n, mm, npmax, err, s);
    }
  }
  GemmBatch<T> gb;
  int n = 0, mm = 0, mn = 0;
  for (size_t g = 0; g < blocks.size(); ++g) {
    const UvwBlockD& b = blocks[g];
    GemmProb<T>& q = gb.prob[n++];
    const int dc = 2 * b.l + 1;
    q.X = S + (size_t)nr_alloc * b.s_off;
    q.B = Bf + b_off[g];
    q.G = nullptr;
    q.C = out;
    q.c = RowBlocked{r0, dc, ld_out, b.out_off, b.mul_own};
    q.M = nr * dc; q.N = b.mul_own; q.D = b.dcols; q.accumulate = accumulate;
    mm = std::max(mm, q.M);
    mn = std::max(mn, q.N);
    if (n == kMaxGemmBatch || g + 1 == blocks.size()) {
      cudaError_t e = launch_gemm<T>(0, gb, n, mm, mn, s);
      if (e != cudaSuccess) return e;
      n = mm = mn = 0;
    }
  }
  return cudaSuccess;
}

std::vector<long long> block_offsets(const std::vector<UvwBlockD>& blocks) {
  std::vector<long long> off;
  long long o = 0;
  for (auto& g : blocks) {
    off.push_back(o);
    o += (long long)g.dcols * g.mul_own;
  }
  return off;
}

template <typename T>
void state_params(UvwSParams<T>& sp, const Plan& P, const T* feat, const T* Y, const T* phi, const int* ptr,
                  const int* nbr, const int* eid, T* S, int N, int E, int ld_feat, int nr_alloc,
                  const std::vector<UvwBlockD>& blocks, const std::vector<PathD>& paths, int* err) {
  sp.feat = feat; sp.Y = Y; sp.phi = phi;
  sp.ptr = ptr; sp.nbr = nbr; sp.eid = eid; sp.S = S; sp.err = err;
  sp.N = N; sp.E = E; sp.K = P.K; sp.ld_feat = ld_feat; sp.dim_y = P.dim_y; sp.n_feat_rows = N;
  sp.r0 = 0; sp.nr = 0; sp.nr_alloc = nr_alloc; sp.accumulate = 0;
  fill_blocks(sp, blocks, paths);
}

// The uvw edge pass's descriptor and shared-memory layout for one plan.
template <typename T>
int edge_params(const Plan& P, UvwEdgeParams<T>& ep, const T* x, const T* Y, const T* phi, const T* Sb,
                const int* rowptr, const int* senders, T* gY, T* gphi, int N, int E, int NR, int* err) {
  const size_t b = sizeof(T);
  ep.x = x; ep.Y = Y; ep.phi = phi; ep.Sbar = Sb;
  ep.rowptr = rowptr; ep.senders = senders; ep.gY = gY; ep.gphi = gphi; ep.err = err;
  ep.N = N; ep.E = E; ep.K = P.K; ep.c_in = P.c_in; ep.dim_y = P.dim_y; ep.nr_alloc = NR;
  ep.r0 = 0; ep.nr = 0; ep.accumulate = 0;
  std::memset(ep.blocks, 0, sizeof(ep.blocks));
  std::memset(ep.paths, 0, sizeof(ep.paths));
  std::memcpy(ep.blocks, P.uvw_out.data(), P.uvw_out.size() * sizeof(UvwBlockD));
  std::memcpy(ep.paths, P.paths_fwd.data(), P.paths_fwd.size() * sizeof(PathD));
  ep.n_blocks = (int)P.uvw_out.size();
  const int vw = 16 / (int)b;
  bool vec = P.K == P.KP && P.c_in % vw == 0;
  int xs = 0, sbar = 0;
  for (const PathD& pd : P.paths_fwd) {
    vec = vec && pd.x_off % vw == 0 && pd.mul_in % vw == 0;
    const int nc = std::min(kEdgeTile, pd.mul_in);
    xs = std::max(xs, 32 * edge_slot_stride((2 * pd.l1 + 1) * nc));
    sbar = std::max(sbar, (2 * pd.l3 + 1) * nc * P.K);
  }
  for (size_t g = 0; g < P.uvw_out.size(); ++g)
    for (int pi = P.uvw_out[g].pbeg; pi < P.uvw_out[g].pend; ++pi) ep.path_blk[pi] = (int8_t)g;
  // the phi_bar partials [warps][K][32] reuse stage buffer 0 at the end of a round
  xs = std::max(xs, kEdgeWarps * 32 * P.K - sbar);
  ep.vec = vec ? 1 : 0;
  ep.smem_sbar = (int)((sbar * b + 15) / 16 * 16);
  ep.smem_stage = (int)((xs * b + 15) / 16 * 16) + ep.smem_sbar;
  ep.smem_red = (int)((kEdgeWarps * 32 * P.dim_y * b + 15) / 16 * 16);
  ep.smem_ct = (int)(kEdgeWarps * 32 * (2 * kLmax + 1) * b);
  if (2 * (size_t)ep.smem_stage + ep.smem_red + ep.smem_ct + 32 * sizeof(int) > (size_t)227 * 1024)
    return fail(TP_EUNSUPPORTED, "uvw edge pass: staging buffers exceed 227 KiB of shared memory");
  return TP_OK;
}

template <typename T>
cudaError_t edge_pass(const Plan& P, const UvwEdgeParams<T>& ep, cudaStream_t s) {
  return P.KP == 8 ? launch_uvw_edge<T, 8>(ep, s) : launch_uvw_edge<T, 16>(ep, s);
}

// A_bar (+)= X_g^T m_bar_g over one receiver chunk (split-K partials, then their
// fixed-order sum; accumulated over chunks when `acc`), X = S or dS.
template <typename T>
cudaError_t abar_chunk(const Plan& P, const T* X, const T* gout, T* Ab, T* Apart, size_t a_elems,
                       const std::vector<long long>& bf_off, int r0, int nr, int NR, bool acc, cudaStream_t s) {
  GemmBatch<T> gb;
  int n = 0, mm = 0, mn = 0;
  for (size_t g = 0; g < P.uvw_out.size(); ++g) {
    const UvwBlockD& bd = P.uvw_out[g];
    const int dc = 2 * bd.l + 1;
    GemmProb<T>& q = gb.prob[n++];
    q.G = gout;
    q.g = RowBlocked{r0, dc, P.c_out, bd.out_off, bd.mul_own};
    q.M = nr * dc; q.N = bd.mul_own; q.D = bd.dcols;
    q.X = X + (size_t)NR * bd.s_off; q.B = nullptr; q.C = Ab + bf_off[g];
    q.accumulate = acc;
    mm = std::max(mm, q.D); mn = std::max(mn, q.N);
    if (n == kMaxGemmBatch || g + 1 == P.uvw_out.size()) {
      cudaError_t e = launch_gemm_tn_split<T>(gb, n, mm, mn, Ab, Apart, a_elems, kTnSplits, s);
      if (e != cudaSuccess) return e;
      n = mm = mn = 0;
    }
  }
  return launch_sum_splits<T>(Apart, a_elems, kTnSplits, Ab, (long long)P.K * P.n_w, acc, s);
}

// S_bar_g = m_bar_g B_g^T over one receiver chunk (B packed from A or dA in
// (u, q) row order).
template <typename T>
cudaError_t sbar_chunk(const Plan& P, const T* Buq, const T* gout, T* Sb, const std::vector<long long>& bf_off,
                       int r0, int nr, int NR, cudaStream_t s) {
  GemmBatch<T> gb;
  int n = 0, mm = 0, mn = 0;
  for (size_t g = 0; g < P.uvw_out.size(); ++g) {
    const UvwBlockD& bd = P.uvw_out[g];
    const int dc = 2 * bd.l + 1;
    GemmProb<T>& q = gb.prob[n++];
    q.G = gout;
    q.g = RowBlocked{r0, dc, P.c_out, bd.out_off, bd.mul_own};
    q.M = nr * dc; q.N = bd.mul_own; q.D = bd.dcols;
    q.X = nullptr; q.B = Buq + bf_off[g]; q.C = Sb + (size_t)NR * bd.s_off;
    q.accumulate = 0;
    mm = std::max(mm, q.M); mn = std::max(mn, q.D);
    if (n == kMaxGemmBatch || g + 1 == P.uvw_out.size()) {
      cudaError_t e = launch_gemm_nt<T>(gb, n, mm, mn, s);
      if (e != cudaSuccess) return e;
      n = mm = mn = 0;
    }
  }
  return cudaSuccess;
}

template <typename T>
int forward_uvw(const Plan& P, const void* x, const void* Y, const void* phi, const void* A, const int* rowptr,
                const int* senders, int N, int E, void* out, void* ws, int* err, cudaStream_t s) {
  const size_t b = sizeof(T);
  const bool tc = use_tc(P);
  const size_t a = align256((size_t)P.K * P.n_w * b);
  T* Bf = (T*)ws;
  T* Blo = tc ? (T*)((char*)ws + a) : nullptr;
  T* S = (T*)((char*)ws + (tc ? 2 : 1) * a);
  cudaError_t e = launch_pack_a<T>(P.pack, (const T*)A, tc ? nullptr : Bf, nullptr, tc ? Bf : nullptr, nullptr,
                                   Blo, nullptr, s);
  if (e != cudaSuccess) return cuda_fail(e, "pack A");
  const std::vector<long long> bf_off = block_offsets(P.uvw_out);
  const int NR = uvw_chunk_rows(P, N, 0);
  UvwSParams<T> sp;
  state_params(sp, P, (const T*)x, (const T*)Y, (const T*)phi, rowptr, senders, (const int*)nullptr, S, N, E,
               P.c_in, NR, P.uvw_out, P.paths_fwd, err);
  for (int r0 = 0; r0 < N; r0 += NR) {
    sp.r0 = r0;
    sp.nr = std::min(NR, N - r0);
    if ((e = sbuild<T>(P, sp, 0, s)) != cudaSuccess) return cuda_fail(e, "uvw state build");
    if ((e = mix_out<T>(P, S, Bf, Blo, (T*)out, r0, sp.nr, NR, P.uvw_out, bf_off, P.c_out, 0, err, s)) !=
        cudaSuccess)
      return cuda_fail(e, "uvw mixing");
  }
  return TP_OK;
}

template <typename T>
int backward_uvw(const Plan& P, const void* x, const void* Y, const void* phi, const void* A, const int* rowptr,
                 const int* senders, const int* colptr, const int* srcedge, const int* srcrecv, const void* gout,
                 int N, int E, void* gx, void* gY, void* gphi, void* gA, void* ws, int* err, cudaStream_t s) {
  const size_t b = sizeof(T);
  const size_t a = align256((size_t)P.K * P.n_w * b);
  const bool tc = use_tc(P);
  T* Bf = (T*)ws;
  T* Ba = (T*)((char*)ws + a);
  T* Ab = (T*)((char*)ws + 2 * a);
  T* Balo = tc ? (T*)((char*)ws + 3 * a) : nullptr;
  const size_t na = tc ? 4 : 3;
  const int NR = uvw_chunk_rows(P, N, 0), NS = uvw_chunk_rows(P, N, 1);
  const size_t s0 = align256((size_t)NR * P.s_row_elems * b), s1 = align256((size_t)NS * P.sa_row_elems * b);
  T* S = (T*)((char*)ws + na * a);
  T* Sb = (T*)((char*)ws + na * a + std::max(s0, s1));
  T* Apart = (T*)((char*)ws + na * a + 2 * std::max(s0, s1));   // kTnSplits copies of the A_bar layout
  // Bf feeds only S_bar = m_bar Bf^T here: rows in (u, q) order give S_bar the
  // column order of the edge pass
  UvwPackParams pk = P.pack;
  pk.bf_uq = 1;
  cudaError_t e = launch_pack_a<T>(pk, (const T*)A, Bf, tc ? nullptr : Ba, nullptr, tc ? Ba : nullptr, nullptr,
                                   Balo, s);
  if (e != cudaSuccess) return cuda_fail(e, "pack A");
  const std::vector<long long> bf_off = block_offsets(P.uvw_out), ba_off = block_offsets(P.uvw_in);
  // ---- receiver chunks: S, A_bar += S^T m_bar, S_bar = m_bar B^T, edge pass
  UvwSParams<T> sp;
  state_params(sp, P, (const T*)x, (const T*)Y, (const T*)phi, rowptr, senders, (const int*)nullptr, S, N, E,
               P.c_in, NR, P.uvw_out, P.paths_fwd, err);
  UvwEdgeParams<T> ep;
  int st = edge_params(P, ep, (const T*)x, (const T*)Y, (const T*)phi, Sb, rowptr, senders, (T*)gY, (T*)gphi, N, E,
                       NR, err);
  if (st) return st;
  for (int r0 = 0; r0 < N; r0 += NR) {
    const int nr = std::min(NR, N - r0);
    sp.r0 = r0;
    sp.nr = nr;
    if ((e = sbuild<T>(P, sp, 0, s)) != cudaSuccess) return cuda_fail(e, "uvw state build");
    if ((e = abar_chunk<T>(P, S, (const T*)gout, Ab, Apart, a / b, bf_off, r0, nr, NR, r0 > 0, s)) != cudaSuccess)
      return cuda_fail(e, "uvw A_bar product");
    if ((e = sbar_chunk<T>(P, Bf, (const T*)gout, Sb, bf_off, r0, nr, NR, s)) != cudaSuccess)
      return cuda_fail(e, "uvw S_bar product");
    ep.r0 = r0;
    ep.nr = nr;
    if ((e = edge_pass<T>(P, ep, s)) != cudaSuccess) return cuda_fail(e, "uvw edge pass");
  }
  // ---- source chunks: S' over the source view, x_bar = S' B'
  UvwSParams<T> ap;
  state_params(ap, P, (const T*)gout, (const T*)Y, (const T*)phi, colptr, srcrecv, srcedge, S, N, E, P.c_out, NS,
               P.uvw_in, P.paths_adj, err);
  for (int s0r = 0; s0r < N; s0r += NS) {
    ap.r0 = s0r;
    ap.nr = std::min(NS, N - s0r);
    if ((e = sbuild<T>(P, ap, 1, s)) != cudaSuccess) return cuda_fail(e, "uvw source state build");
    if ((e = mix_out<T>(P, S, Ba, Balo, (T*)gx, s0r, ap.nr, NS, P.uvw_in, ba_off, P.c_in, 0, err, s)) !=
        cudaSuccess)
      return cuda_fail(e, "uvw grad_x mixing");
  }
  e = launch_unpack_a<T>(P.pack, Ab, (T*)gA, s);
  return e == cudaSuccess ? TP_OK : cuda_fail(e, "unpack grad_A");
}

// The packed GEMM operands of one [K, N_w] weight tensor (A or its direction).
template <typename T>
struct PackedW {
  T* fwd;      // forward mixing m = S B (tensor cores: B^T hi part)
  T* fwd_lo;   // tensor cores: B^T lo part
  T* adj;      // source mixing x_bar = S' B' (tensor cores: B'^T hi part)
  T* adj_lo;
  T* uq;       // S_bar = m_bar B^T, rows in (u, q) order
};

template <typename T>
cudaError_t pack_w(const Plan& P, const T* W, PackedW<T>& o, char*& cur, size_t a, cudaStream_t s) {
  const bool tc = use_tc(P);
  auto take = [&]() {
    T* p = (T*)cur;
    cur += a;
    return p;
  };
  o.uq = take();
  o.fwd = take();
  o.adj = take();
  o.fwd_lo = tc ? take() : nullptr;
  o.adj_lo = tc ? take() : nullptr;
  UvwPackParams pk = P.pack;
  pk.bf_uq = 1;
  cudaError_t e = tc ? launch_pack_a<T>(pk, W, o.uq, nullptr, o.fwd, o.adj, o.fwd_lo, o.adj_lo, s)
                     : launch_pack_a<T>(pk, W, o.uq, o.adj, nullptr, nullptr, nullptr, nullptr, s);
  if (e != cudaSuccess || tc) return e;
  pk.bf_uq = 0;
  return launch_pack_a<T>(pk, W, o.fwd, nullptr, nullptr, nullptr, nullptr, nullptr, s);
}

// Second-order program of the fully connected path (Sobek §4.4), composed from
// the first-order kernels by multilinearity: with the directional state
// dS = S(dx, Y, phi) + S(x, dY, phi) + S(x, Y, dphi) per receiver chunk,
//   m_dot       = dS A + S dA,             A_bar_dot = dS^T m_bar,
//   phi_bar_dot = E_phi(dx, Y; S_bar) + E_phi(x, dY; S_bar) + E_phi(x, Y; dS_bar),
//   Y_bar_dot   = E_Y(dx, phi; S_bar) + E_Y(x, dphi; S_bar) + E_Y(x, phi; dS_bar),
// with S_bar = m_bar A^T, dS_bar = m_bar dA^T and E the edge pass (its phi_bar
// does not read phi, its Y_bar does not read Y, so each call yields two wanted
// terms); per source chunk x_bar_dot = (S'(dY, phi) + S'(Y, dphi)) A' + S' dA'.
template <typename T>
int double_backward_uvw(const Plan& P, const void* const* in, const int* const* idx, const void* const* dir, int N,
                        int E, void* const* out, void* ws, int* err, cudaStream_t s) {
  const size_t b = sizeof(T);
  const size_t a = align256((size_t)P.K * P.n_w * b);
  const T *x = (const T*)in[0], *Y = (const T*)in[1], *phi = (const T*)in[2], *A = (const T*)in[3],
          *gout = (const T*)in[4];
  const T *dx = (const T*)dir[0], *dY = (const T*)dir[1], *dphi = (const T*)dir[2], *dA = (const T*)dir[3];
  const int *rowptr = idx[0], *senders = idx[1], *colptr = idx[2], *srcedge = idx[3], *srcrecv = idx[4];
  T *mdot = (T*)out[0], *dgx = (T*)out[1], *dgY = (T*)out[2], *dgphi = (T*)out[3], *dgA = (T*)out[4];
  char* cur = (char*)ws;
  PackedW<T> pa, pd;
  cudaError_t e = pack_w<T>(P, A, pa, cur, a, s);
  if (e == cudaSuccess) e = pack_w<T>(P, dA, pd, cur, a, s);
  if (e != cudaSuccess) return cuda_fail(e, "pack A");
  T* Ab = (T*)cur;
  cur += a;
  T* Apart = (T*)cur;
  cur += kTnSplits * a;
  const int NR = uvw_chunk_rows(P, N, 0), NS = uvw_chunk_rows(P, N, 1);
  const size_t sm = std::max(align256((size_t)NR * P.s_row_elems * b), align256((size_t)NS * P.sa_row_elems * b));
  T* S = (T*)cur;
  T* Sb = (T*)(cur + sm);
  const std::vector<long long> bf_off = block_offsets(P.uvw_out), ba_off = block_offsets(P.uvw_in);
  UvwSParams<T> sp;
  state_params(sp, P, x, Y, phi, rowptr, senders, (const int*)nullptr, S, N, E, P.c_in, NR, P.uvw_out, P.paths_fwd,
               err);
  UvwEdgeParams<T> ep;
  int st = edge_params(P, ep, x, Y, phi, Sb, rowptr, senders, dgY, dgphi, N, E, NR, err);
  if (st) return st;
  auto build = [&](UvwSParams<T>& p, const T* feat, const T* y, const T* ph, int acc, int d) {
    p.feat = feat; p.Y = y; p.phi = ph; p.accumulate = acc;
    return sbuild<T>(P, p, d, s);
  };
  for (int r0 = 0; r0 < N; r0 += NR) {
    const int nr = std::min(NR, N - r0);
    sp.r0 = r0;
    sp.nr = nr;
    // directional state dS, then m_dot = dS A and A_bar_dot (+)= dS^T m_bar
    if ((e = build(sp, dx, Y, phi, 0, 0)) != cudaSuccess || (e = build(sp, x, dY, phi, 1, 0)) != cudaSuccess ||
        (e = build(sp, x, Y, dphi, 1, 0)) != cudaSuccess)
      return cuda_fail(e, "uvw directional state");
    if ((e = mix_out<T>(P, S, pa.fwd, pa.fwd_lo, mdot, r0, nr, NR, P.uvw_out, bf_off, P.c_out, 0, err, s)) !=
        cudaSuccess)
      return cuda_fail(e, "uvw directional mixing");
    if ((e = abar_chunk<T>(P, S, gout, Ab, Apart, a / b, bf_off, r0, nr, NR, r0 > 0, s)) != cudaSuccess)
      return cuda_fail(e, "uvw A_bar_dot product");
    // primal state S, m_dot += S dA
    if ((e = build(sp, x, Y, phi, 0, 0)) != cudaSuccess) return cuda_fail(e, "uvw state build");
    if ((e = mix_out<T>(P, S, pd.fwd, pd.fwd_lo, mdot, r0, nr, NR, P.uvw_out, bf_off, P.c_out, 1, err, s)) !=
        cudaSuccess)
      return cuda_fail(e, "uvw mixing");
    // edge pass on S_bar with (dx, Y, phi) and (x, dY, dphi), then on dS_bar
    if ((e = sbar_chunk<T>(P, pa.uq, gout, Sb, bf_off, r0, nr, NR, s)) != cudaSuccess)
      return cuda_fail(e, "uvw S_bar product");
    ep.r0 = r0;
    ep.nr = nr;
    ep.x = dx; ep.Y = Y; ep.phi = phi; ep.accumulate = 0;
    if ((e = edge_pass<T>(P, ep, s)) != cudaSuccess) return cuda_fail(e, "uvw edge pass");
    ep.x = x; ep.Y = dY; ep.phi = dphi; ep.accumulate = 1;
    if ((e = edge_pass<T>(P, ep, s)) != cudaSuccess) return cuda_fail(e, "uvw edge pass");
    if ((e = sbar_chunk<T>(P, pd.uq, gout, Sb, bf_off, r0, nr, NR, s)) != cudaSuccess)
      return cuda_fail(e, "uvw S_bar product");
    ep.x = x; ep.Y = Y; ep.phi = phi; ep.accumulate = 1;
    if ((e = edge_pass<T>(P, ep, s)) != cudaSuccess) return cuda_fail(e, "uvw edge pass");
  }
  UvwSParams<T> ap;
  state_params(ap, P, gout, Y, phi, colptr, srcrecv, srcedge, S, N, E, P.c_out, NS, P.uvw_in, P.paths_adj, err);
  for (int s0r = 0; s0r < N; s0r += NS) {
    ap.r0 = s0r;
    ap.nr = std::min(NS, N - s0r);
    if ((e = build(ap, gout, dY, phi, 0, 1)) != cudaSuccess || (e = build(ap, gout, Y, dphi, 1, 1)) != cudaSuccess)
      return cuda_fail(e, "uvw directional source state");
    if ((e = mix_out<T>(P, S, pa.adj, pa.adj_lo, dgx, s0r, ap.nr, NS, P.uvw_in, ba_off, P.c_in, 0, err, s)) !=
        cudaSuccess)
      return cuda_fail(e, "uvw directional source mixing");
    if ((e = build(ap, gout, Y, phi, 0, 1)) != cudaSuccess) return cuda_fail(e, "uvw source state");
    if ((e = mix_out<T>(P, S, pd.adj, pd.adj_lo, dgx, s0r, ap.nr, NS, P.uvw_in, ba_off, P.c_in, 1, err, s)) !=
        cudaSuccess)
      return cuda_fail(e, "uvw source mixing");
  }
  e = launch_unpack_a<T>(P.pack, Ab, dgA, s);
  return e == cudaSuccess ? TP_OK : cuda_fail(e, "unpack A_bar_dot");
}

}  // namespace

// Shared with other translation units of the library.
int set_error_message(int status, const std::string& m) { return fail(status, m); }
int device_error_word(int** out) { return error_word(out); }

}  // namespace tpc

using namespace tpc;

extern "C" {

int tp_conv_plan(const char* irreps_in, int sh_lmax, const char* irreps_out, int n_radial, int mode,
                 int dtype, tp_plan_t* plan) {
  if (!plan) return fail(TP_EINVAL, "plan output pointer is NULL");
  *plan = nullptr;
  auto* h = new (std::nothrow) tp_plan_s;
  if (!h) return fail(TP_EINVAL, "out of host memory");
  std::string msg;
  const int st = make_plan(irreps_in, sh_lmax, irreps_out, n_radial, mode, dtype, h->p, msg);
  if (st != TP_OK) {
    delete h;
    return fail(st, msg);
  }
  *plan = h;
  return TP_OK;
}

int tp_conv_plan_sh(const char* irreps_in, const char* irreps_sh, const char* irreps_out, int n_radial, int mode,
                    int dtype, tp_plan_t* plan) {
  if (!plan) return fail(TP_EINVAL, "plan output pointer is NULL");
  *plan = nullptr;
  if (!irreps_sh) return fail(TP_EINVAL, "spherical-harmonic irreps string is NULL");
  std::string msg;
  int sh_lmax = 0;
  std::vector<int> parity;
  int st = parse_sh_irreps(irreps_sh, sh_lmax, parity, msg);
  if (st != TP_OK) return fail(st, msg);
  auto* h = new (std::nothrow) tp_plan_s;
  if (!h) return fail(TP_EINVAL, "out of host memory");
  st = make_plan(irreps_in, sh_lmax, irreps_out, n_radial, mode, dtype, h->p, msg, parity.data());
  if (st != TP_OK) {
    delete h;
    return fail(st, msg);
  }
  *plan = h;
  return TP_OK;
}

int tp_conv_plan_destroy(tp_plan_t plan) {
  delete plan;
  return TP_OK;
}

int tp_conv_plan_info(tp_plan_t plan, tp_plan_info_t* info) {
  if (!plan || !info) return fail(TP_EINVAL, "NULL plan or info");
  const Plan& P = plan->p;
  std::memset(info, 0, sizeof(*info));
  info->c_in = P.c_in; info->c_out = P.c_out; info->dim_y = P.dim_y; info->n_radial = P.K;
  info->n_paths = (int)P.paths.size(); info->mode = P.per_path ? TP_UVU_PATHS : P.mode; info->dtype = P.dtype;
  info->sh_lmax = P.sh_lmax; info->lmax = P.lmax; info->n_w = P.n_w;
  return TP_OK;
}

int tp_conv_plan_path(tp_plan_t plan, int index, tp_path_info_t* info) {
  if (!plan || !info) return fail(TP_EINVAL, "NULL plan or info");
  const Plan& P = plan->p;
  if (index < 0 || index >= (int)P.paths.size()) return fail(TP_EINVAL, "path index out of range");
  const HostPath& h = P.paths[index];
  std::memset(info, 0, sizeof(*info));
  info->l1 = h.l1; info->p1 = h.p1; info->l2 = h.l2; info->p2 = h.p2; info->l3 = h.l3; info->p3 = h.p3;
  info->block_in = h.i_in; info->block_out = h.i_out; info->mul_in = h.mul_in; info->mul_out = h.mul_out;
  info->x_off = h.x_off; info->out_off = h.out_off; info->w_off = h.w_off; info->n_w = h.n_w;
  info->nnz = h.nnz;
  return TP_OK;
}

int tp_conv_plan_cg(tp_plan_t plan, int index, int32_t* m1, int32_t* m2, int32_t* m3, double* c,
                    int capacity) {
  if (!plan) return fail(TP_EINVAL, "NULL plan");
  const Plan& P = plan->p;
  if (index < 0 || index >= (int)P.paths.size()) return fail(TP_EINVAL, "path index out of range");
  const HostPath& h = P.paths[index];
  auto e = real_cg_sparse(h.l1, h.l2, h.l3);
  const int n = (int)e.size();
  if (capacity > 0 && (!m1 || !m2 || !m3 || !c)) return fail(TP_EINVAL, "NULL output array");
  for (int k = 0; k < n && k < capacity; ++k) {
    m1[k] = e[k].m1; m2[k] = e[k].m2; m3[k] = e[k].m3; c[k] = e[k].c;
  }
  return n;
}

int tp_conv_plan_set_state_budget(tp_plan_t plan, size_t bytes) {
  if (!plan) return fail(TP_EINVAL, "NULL plan");
  Plan& P = plan->p;
  if (P.mode != TP_UVW) return TP_OK;
  const size_t b = P.dtype == TP_F32 ? 4 : 8;
  const size_t one = (size_t)std::max(P.s_row_elems, P.sa_row_elems) * b;
  if (bytes < one)
    return fail(TP_EINVAL, "state budget " + std::to_string(bytes) + " bytes is below one node's state (" +
                               std::to_string(one) + " bytes)");
  P.state_budget = bytes;
  return TP_OK;
}

int tp_conv_plan_set_schedule(tp_plan_t plan, int schedule) {
  if (!plan) return fail(TP_EINVAL, "NULL plan");
  Plan& P = plan->p;
  if (schedule != TP_SCHED_STREAMED && schedule != TP_SCHED_RECEIVER_STATE)
    return fail(TP_EINVAL, "schedule must be TP_SCHED_STREAMED or TP_SCHED_RECEIVER_STATE");
  if (P.mode != TP_UVU) return schedule == TP_SCHED_RECEIVER_STATE ? TP_OK
                                                                  : fail(TP_EUNSUPPORTED, "fully connected plans "
                                                                                          "use the receiver state");
  if (schedule == TP_SCHED_RECEIVER_STATE && (P.K > 8 || P.prof > 3 || !P.dbl_ok))
    return fail(TP_EUNSUPPORTED, "the receiver-state uvu forward is compiled for K <= 8 and degrees <= 4");
  P.schedule = schedule;
  return TP_OK;
}

int tp_conv_work_model(tp_plan_t plan, int64_t n_nodes, int64_t n_edges, int pass, double* flops,
                       double* bytes) {
  if (!plan || !flops || !bytes) return fail(TP_EINVAL, "NULL argument");
  if (pass < 0 || pass > 2) return fail(TP_EINVAL, "pass must be 0, 1 or 2");
  work_model(plan->p, n_nodes, n_edges, pass, *flops, *bytes);
  return TP_OK;
}

int tp_conv_workspace_size(tp_plan_t plan, int64_t n_nodes, int pass, size_t* bytes) {
  if (!plan || !bytes) return fail(TP_EINVAL, "NULL argument");
  if (pass < 0 || pass > 2) return fail(TP_EINVAL, "pass must be 0, 1 or 2");
  if (n_nodes < 0) return fail(TP_EINVAL, "negative node count");
  *bytes = workspace_bytes(plan->p, n_nodes, pass);
  return TP_OK;
}

int tp_conv_launch_count(tp_plan_t plan, int64_t n_nodes, int pass, int* kernels) {
  if (!plan || !kernels) return fail(TP_EINVAL, "NULL argument");
  if (pass < 0 || pass > 2) return fail(TP_EINVAL, "pass must be 0, 1 or 2");
  if (n_nodes < 0) return fail(TP_EINVAL, "negative node count");
  const Plan& P = plan->p;
  if (n_nodes == 0) {
    *kernels = 0;
    return TP_OK;
  }
  if (P.mode == TP_UVU) {
    // forward; edge pass, source pass, grad_A reduction; receiver, edge and
    // source passes of the second-order program and its A_bar reduction
    *kernels = pass == 0 ? 1 : pass == 1 ? 3 : 4;
    return TP_OK;
  }
  const long long nr = uvw_chunk_rows(P, n_nodes, 0), ns = uvw_chunk_rows(P, n_nodes, 1);
  const long long cr = (n_nodes + nr - 1) / nr, cs = (n_nodes + ns - 1) / ns;
  const long long gout = ((long long)P.uvw_out.size() + kMaxGemmBatch - 1) / kMaxGemmBatch;
  const long long gin = ((long long)P.uvw_in.size() + kMaxGemmBatch - 1) / kMaxGemmBatch;
  if (pass == 0)
    *kernels = (int)(1 + cr * (1 + gout));                       // pack A; per chunk: state, mixing
  else if (pass == 1)   // pack A; per receiver chunk: state, A_bar partials, their sum, S_bar, edge pass;
                        // per source chunk: source-view state, mixing; unpack A_bar
    *kernels = (int)(1 + cr * (1 + gout + 1 + gout + 1) + cs * (1 + gin) + 1);
  else   // pack A and dA (twice each without tensor cores); per receiver chunk: three
         // directional-state builds, mixing, A_bar_dot partials and their sum, the state,
         // mixing, S_bar, two edge passes, dS_bar, one edge pass; per source chunk: three
         // state builds, two mixings; unpack A_bar_dot
    *kernels = (int)((P.uvw_tc ? 2 : 4) + cr * (8 + 5 * gout) + cs * (3 + 2 * gin) + 1);
  return TP_OK;
}

int tp_csr_workspace_size(int64_t n_nodes, size_t* bytes) {
  if (!bytes || n_nodes < 0) return fail(TP_EINVAL, "bad argument");
  *bytes = csr_workspace_bytes(n_nodes);
  return TP_OK;
}

int tp_csr_build(int64_t n_nodes, int64_t n_edges, const int32_t* src, const int32_t* dst,
                 int32_t* rowptr, int32_t* senders, int32_t* perm, void* ws, size_t ws_bytes,
                 void* stream) {
  int st = check_sizes(n_nodes, n_edges);
  if (st) return st;
  if (!rowptr || !ws || (n_edges > 0 && (!src || !dst || !senders || !perm)))
    return fail(TP_EINVAL, "NULL device pointer");
  if (ws_bytes < csr_workspace_bytes(n_nodes)) return fail(TP_EWORKSPACE, "CSR workspace too small");
  int* err = nullptr;
  if ((st = error_word(&err))) return st;
  cudaError_t e = csr_build((int)n_nodes, (int)n_edges, src, dst, rowptr, senders, perm, ws, err,
                            (cudaStream_t)stream);
  return e == cudaSuccess ? TP_OK : cuda_fail(e, "tp_csr_build");
}

int tp_csr_transpose(int64_t n_nodes, int64_t n_edges, const int32_t* rowptr, const int32_t* senders,
                     int32_t* colptr, int32_t* srcedge, int32_t* srcrecv, void* ws, size_t ws_bytes,
                     void* stream) {
  int st = check_sizes(n_nodes, n_edges);
  if (st) return st;
  if (!rowptr || !colptr || !ws || (n_edges > 0 && (!senders || !srcedge || !srcrecv)))
    return fail(TP_EINVAL, "NULL device pointer");
  if (ws_bytes < csr_workspace_bytes(n_nodes)) return fail(TP_EWORKSPACE, "CSR workspace too small");
  int* err = nullptr;
  if ((st = error_word(&err))) return st;
  cudaError_t e = csr_transpose((int)n_nodes, (int)n_edges, rowptr, senders, colptr, srcedge, srcrecv,
                                ws, err, (cudaStream_t)stream);
  return e == cudaSuccess ? TP_OK : cuda_fail(e, "tp_csr_transpose");
}

int tp_conv_forward(tp_plan_t plan, const void* x, const void* Y, const void* phi, const void* A,
                    const int32_t* rowptr, const int32_t* senders, int64_t n_nodes, int64_t n_edges,
                    void* out, void* ws, size_t ws_bytes, void* stream) {
  if (!plan) return fail(TP_EINVAL, "NULL plan");
  const Plan& P = plan->p;
  int st = check_sizes(n_nodes, n_edges);
  if (st) return st;
  if (n_nodes == 0) return TP_OK;
  if (!x || !A || !rowptr || !out || (n_edges > 0 && (!Y || !phi || !senders)))
    return fail(TP_EINVAL, "NULL device pointer");
  if (!al16(x) || !al16(A) || !al16(out) || (n_edges > 0 && (!al16(Y) || !al16(phi))))
    return fail(TP_EINVAL, "floating-point buffers must be 16-byte aligned");
  if (ws_bytes < workspace_bytes(P, n_nodes, 0)) return fail(TP_EWORKSPACE, "workspace too small");
  int* err = nullptr;
  if ((st = error_word(&err))) return st;
  cudaStream_t s = (cudaStream_t)stream;
  if (P.mode == TP_UVW) {
    if (!ws) return fail(TP_EWORKSPACE, "uvw forward needs a workspace");
    return P.dtype == TP_F32
               ? forward_uvw<float>(P, x, Y, phi, A, rowptr, senders, (int)n_nodes, (int)n_edges, out, ws, err, s)
               : forward_uvw<double>(P, x, Y, phi, A, rowptr, senders, (int)n_nodes, (int)n_edges, out, ws, err, s);
  }
  return P.dtype == TP_F32
             ? forward_uvu<float>(P, x, Y, phi, A, rowptr, senders, (int)n_nodes, (int)n_edges, out, err, s)
             : forward_uvu<double>(P, x, Y, phi, A, rowptr, senders, (int)n_nodes, (int)n_edges, out, err, s);
}

int tp_conv_backward(tp_plan_t plan, const void* x, const void* Y, const void* phi, const void* A,
                     const int32_t* rowptr, const int32_t* senders, const int32_t* colptr,
                     const int32_t* srcedge, const int32_t* srcrecv, const void* grad_out,
                     int64_t n_nodes, int64_t n_edges, void* grad_x, void* grad_Y, void* grad_phi,
                     void* grad_A, void* ws, size_t ws_bytes, void* stream) {
  if (!plan) return fail(TP_EINVAL, "NULL plan");
  const Plan& P = plan->p;
  int st = check_sizes(n_nodes, n_edges);
  if (st) return st;
  if (!x || !A || !rowptr || !colptr || !grad_out || !grad_x || !grad_A ||
      (n_edges > 0 && (!Y || !phi || !senders || !srcedge || !srcrecv || !grad_Y || !grad_phi)))
    return fail(TP_EINVAL, "NULL device pointer");
  const void* f[] = {x, A, grad_out, grad_x, grad_A};
  for (const void* q : f)
    if (!al16(q)) return fail(TP_EINVAL, "floating-point buffers must be 16-byte aligned");
  if (n_edges > 0 && (!al16(Y) || !al16(phi) || !al16(grad_Y) || !al16(grad_phi)))
    return fail(TP_EINVAL, "floating-point buffers must be 16-byte aligned");
  if (ws_bytes < workspace_bytes(P, n_nodes, 1) || (!ws && workspace_bytes(P, n_nodes, 1) > 0))
    return fail(TP_EWORKSPACE, "workspace too small");
  int* err = nullptr;
  if ((st = error_word(&err))) return st;
  cudaStream_t s = (cudaStream_t)stream;
  if (n_nodes == 0) {
    cudaError_t e = cudaMemsetAsync(grad_A, 0, (size_t)P.K * P.n_w * (P.dtype == TP_F32 ? 4 : 8), s);
    return e == cudaSuccess ? TP_OK : cuda_fail(e, "memset grad_A");
  }
  if (P.mode == TP_UVW)
    return P.dtype == TP_F32
               ? backward_uvw<float>(P, x, Y, phi, A, rowptr, senders, colptr, srcedge, srcrecv, grad_out,
                                     (int)n_nodes, (int)n_edges, grad_x, grad_Y, grad_phi, grad_A, ws, err, s)
               : backward_uvw<double>(P, x, Y, phi, A, rowptr, senders, colptr, srcedge, srcrecv, grad_out,
                                      (int)n_nodes, (int)n_edges, grad_x, grad_Y, grad_phi, grad_A, ws, err, s);
  return P.dtype == TP_F32
             ? backward_uvu<float>(P, x, Y, phi, A, rowptr, senders, colptr, srcedge, srcrecv, grad_out,
                                   (int)n_nodes, (int)n_edges, grad_x, grad_Y, grad_phi, grad_A, ws, err, s)
             : backward_uvu<double>(P, x, Y, phi, A, rowptr, senders, colptr, srcedge, srcrecv, grad_out,
                                    (int)n_nodes, (int)n_edges, grad_x, grad_Y, grad_phi, grad_A, ws, err, s);
}

int tp_conv_double_backward(tp_plan_t plan, const void* x, const void* Y, const void* phi, const void* A,
                            const int32_t* rowptr, const int32_t* senders, const int32_t* colptr,
                            const int32_t* srcedge, const int32_t* srcrecv, const void* grad_out,
                            const void* dx, const void* dY, const void* dphi, const void* dA, int64_t n_nodes,
                            int64_t n_edges, void* d_out, void* dgrad_x, void* dgrad_Y, void* dgrad_phi,
                            void* dgrad_A, void* ws, size_t ws_bytes, void* stream) {
  if (!plan) return fail(TP_EINVAL, "NULL plan");
  const Plan& P = plan->p;
  int st = check_sizes(n_nodes, n_edges);
  if (st) return st;
  if (!x || !A || !rowptr || !colptr || !grad_out || !dx || !dA || !d_out || !dgrad_x || !dgrad_A ||
      (n_edges > 0 && (!Y || !phi || !senders || !srcedge || !srcrecv || !dY || !dphi || !dgrad_Y || !dgrad_phi)))
    return fail(TP_EINVAL, "NULL device pointer");
  const void* f[] = {x, A, grad_out, dx, dA, d_out, dgrad_x, dgrad_A};
  for (const void* q : f)
    if (!al16(q)) return fail(TP_EINVAL, "floating-point buffers must be 16-byte aligned");
  if (n_edges > 0 && (!al16(Y) || !al16(phi) || !al16(dY) || !al16(dphi) || !al16(dgrad_Y) || !al16(dgrad_phi)))
    return fail(TP_EINVAL, "floating-point buffers must be 16-byte aligned");
  if (P.mode == TP_UVU && !P.dbl_ok) return fail(TP_EUNSUPPORTED, "double backward: more than 96 channel tiles of 32");
  const size_t need = workspace_bytes(P, n_nodes, 2);
  if (ws_bytes < need || (!ws && need > 0)) return fail(TP_EWORKSPACE, "workspace too small");
  int* err = nullptr;
  if ((st = error_word(&err))) return st;
  cudaStream_t s = (cudaStream_t)stream;
  if (n_nodes == 0) {
    cudaError_t e = cudaMemsetAsync(dgrad_A, 0, (size_t)P.K * P.n_w * (P.dtype == TP_F32 ? 4 : 8), s);
    return e == cudaSuccess ? TP_OK : cuda_fail(e, "memset dgrad_A");
  }
  const void* in[] = {x, Y, phi, A, grad_out};
  const int* idx[] = {rowptr, senders, colptr, srcedge, srcrecv};
  const void* dir[] = {dx, dY, dphi, dA};
  void* out[] = {d_out, dgrad_x, dgrad_Y, dgrad_phi, dgrad_A};
  if (P.mode == TP_UVW)
    return P.dtype == TP_F32
               ? double_backward_uvw<float>(P, in, idx, dir, (int)n_nodes, (int)n_edges, out, ws, err, s)
               : double_backward_uvw<double>(P, in, idx, dir, (int)n_nodes, (int)n_edges, out, ws, err, s);
  return P.dtype == TP_F32
             ? double_backward_uvu<float>(P, in, idx, dir, (int)n_nodes, (int)n_edges, out, ws, err, s)
             : double_backward_uvu<double>(P, in, idx, dir, (int)n_nodes, (int)n_edges, out, ws, err, s);
}

int tp_get_device_error(void* stream) {
  int* err = nullptr;
  int st = error_word(&err);
  if (st) return st;
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  int v = 0;
  e = cudaMemcpy(&v, err, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "read error word");
  if (v) {
    const int zero = 0;
    e = cudaMemcpy(err, &zero, sizeof(int), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_fail(e, "clear error word");
  }
  if (v & kErrIndex) return fail(TP_EDEVICE_INDEX, "a kernel met an index outside its range");
  if (v & kErrCsr) return fail(TP_EDEVICE_CSR, "a kernel met a bad row pointer");
  if (v & kErrTimeout) return fail(TP_EDEVICE_TIMEOUT, "a kernel's bounded wait expired");
  return TP_OK;
}

const char* tp_status_string(int status) {
  switch (status) {
    case TP_OK: return "ok";
    case TP_EINVAL: return "invalid argument";
    case TP_EUNSUPPORTED: return "unsupported contract";
    case TP_ECUDA: return "CUDA runtime error";
    case TP_EWORKSPACE: return "workspace too small";
    case TP_EDEVICE_INDEX: return "device: index out of range";
    case TP_EDEVICE_CSR: return "device: bad row pointer";
    case TP_EDEVICE_TIMEOUT: return "device: bounded wait expired";
    default: return "unknown status";
  }
}

const char* tp_last_error_message(void) { return g_msg.c_str(); }

}  // extern "C"
