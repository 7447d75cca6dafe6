// Channelwise (uvu) forward of the edge-conditioned CG tensor-product convolution.
//
// m_i = sum_{j in N(i)} sum_pi w_{ij,pi,u} T_{pi,u}(x_j, Y_ij),
// w_{ij,pi,u} = sum_q phi_{ij,q} A_{q,pi,u}            (Sobek §2.4, Eq. 11-12)
//
// Schedule: the streamed order of Sobek §3.1 -- the scalar w is formed in
// registers and consumed at once; no W and no edge message exists anywhere.
// Work is node-centric as in LunaTP §4.1-4.2: one warp owns one task
// (receiver i, output block g, tile of 32*CPL channels), lanes own CPL adjacent
// channels, the receiver's incoming edges (CSR by receiver) form the inner loop,
// and the output accumulators of block g stay in registers until the single
// store. Paths into g run one after another; their A values live in registers
// for the whole edge traversal of that path.
//
// The CG contraction is split (Sobek §4.2, Eq. 32) into an edge-uniform part
// cY[m1][m3] = sum_{m2} c[m1,m2,m3] Y[m2] and a per-channel part
// acc[m3] += cY[m1][m3] * (w x[m1]) over the non-zero (m1, m3) pairs; the
// coefficients and pair structure are compile-time constants (LunaTP §4.3).
// Edges are processed in chunks of up to 32: first each lane takes one edge of
// the chunk and writes its sender, radial row and the cY values of every path
// of the tile into the warp's shared-memory slice; then the warp sweeps the
// chunk once per path, reading those values as broadcasts while the x rows of
// the next group of senders arrive through an asynchronous copy ring.
//
// Task order: windows of kWin receivers; inside a window all receivers of one
// tile come first, so the warps of a CTA run the same code on neighbouring
// receivers, and the window's x rows are re-read from L2 by the other tiles.
//
// Graphs with too few (receiver, tile) tasks to fill the GPU run in split mode:
// a CTA takes one task and its warps deal the tile's paths round-robin, each
// staging and sweeping the chunk for its own paths; their accumulators are
// added in warp order in shared memory before the one store.
#include "common.cuh"
#include "kernels.h"

namespace tpc {
namespace {

constexpr int kWin = 16;

template <typename T>
struct FwdSmem {
  int* j;
  T* phi;
  T* cy;
  T* ring;   // [2][G][2 lmax_in + 1][32 CPL] x rows in flight (G = fwd_ring_g)
};

template <typename T, int KP>
__device__ __forceinline__ FwdSmem<T> fwd_smem(const UvuFwdParams<T>& p, int warp) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  unsigned char* base = smem_raw + (size_t)warp * p.warp_smem;
  FwdSmem<T> s;
  s.j = reinterpret_cast<int*>(base);
  s.phi = reinterpret_cast<T*>(base + 32 * sizeof(int));
  s.cy = s.phi + 32 * KP;
  s.ring = reinterpret_cast<T*>(base + p.ring_off);
  return s;
}

// Stage the cY values of one path for the calling lane's edge.
template <typename T, int L1, int L2, int L3>
__device__ __forceinline__ void stage_cy(const T* yrow, T* dst) {
  using CGp = cgt::CG<L1, L2, L3>;
  T y[2 * L2 + 1];
#pragma unroll
  for (int m = 0; m < 2 * L2 + 1; ++m) y[m] = ldg(yrow + L2 * L2 + m);
  static_for<CGp::npair>([&](auto P) { dst[decltype(P)::value] = pair_coef<T, CGp, decltype(P)::value>(y); });
}

// 16-byte shared-memory load of VW scalars.
template <typename T>
__device__ __forceinline__ void lds16(T* v, const T* src) {
  if constexpr (sizeof(T) == 4) {
    const float4 t = *reinterpret_cast<const float4*>(src);
    v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
  } else {
    const double2 t = *reinterpret_cast<const double2*>(src);
    v[0] = t.x; v[1] = t.y;
  }
}

template <typename T, int KP, int CPL, int G, int L1, int L2, int L3>
__device__ __forceinline__ void fwd_path(const UvuFwdParams<T>& p, const PathD& pd, const FwdSmem<T>& s,
                                         int n, int chl, T (&acc)[2 * L3 + 1][CPL]) {
  using CGp = cgt::CG<L1, L2, L3>;
  constexpr int D1 = 2 * L1 + 1, D3 = 2 * L3 + 1, NP = CGp::npair;
  constexpr int VW = sizeof(T) == 4 ? 4 : 2;           // scalars per 16-byte shared load
  T a[KP][CPL];
#pragma unroll
  for (int q = 0; q < KP; ++q) {
    if (q < p.K) {
      load_ch<CPL>(a[q], p.A + (size_t)q * p.n_w + pd.w_off + chl);
    } else {
#pragma unroll
      for (int c = 0; c < CPL; ++c) a[q][c] = T(0);
    }
  }
  // x rows of the chunk's senders go through a two-buffer ring of groups of G
  // edges: the copies of group g + 1 are in flight while group g is
  // contracted. Each lane copies and later reads only its own channels.
  const T* xb = p.x + pd.x_off + chl;
  const int mul = pd.mul_in, lane = threadIdx.x & 31;
  constexpr int RW = 32 * CPL;   // ring row: one component of one edge
  auto issue = [&](int g0, int buf) {
#pragma unroll
    for (int t = 0; t < G; ++t) {
      if (g0 + t < n) {
        const T* xr = xb + (size_t)s.j[g0 + t] * p.c_in;
        T* dst = s.ring + ((buf * G + t) * D1) * RW + lane * CPL;
#pragma unroll
        for (int m = 0; m < D1; ++m) cp_async_b<CPL * sizeof(T)>(dst + m * RW, xr + m * mul);
      }
    }
  };
  if (n > 0) issue(0, 0);
  cp_commit();
  for (int g0 = 0, buf = 0; g0 < n; g0 += G, buf ^= 1) {
    if (g0 + G < n) issue(g0 + G, buf ^ 1);
    cp_commit();
    cp_wait<1>();   // this group's rows have landed
    const int tn = min(G, n - g0);
    // the group's edges unrolled: their loads and FMA chains interleave
#pragma unroll
  for (int t = 0; t < G; ++t) {
    if (t >= tn) break;
    const int k = g0 + t;
    T xv[D1][CPL];
    {
      const T* src = s.ring + ((buf * G + t) * D1) * RW + lane * CPL;
#pragma unroll
      for (int m = 0; m < D1; ++m) {
        if constexpr (CPL == 2 && sizeof(T) == 4) {
          const float2 v2 = *reinterpret_cast<const float2*>(src + m * RW);
          xv[m][0] = v2.x; xv[m][1] = v2.y;
        } else {
#pragma unroll
          for (int c = 0; c < CPL; ++c) xv[m][c] = src[m * RW + c];
        }
      }
    }
    T ph[KP];
#pragma unroll
    for (int q = 0; q < KP; q += VW) lds16(ph + q, s.phi + k * KP + q);
    const T* cyr = s.cy + k * p.cy_stride + pd.cy_off;
    T w[CPL];
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
      w[c] = ph[0] * a[0][c];
#pragma unroll
      for (int q = 1; q < KP; ++q) w[c] = fma(ph[q], a[q][c], w[c]);
    }
    T cyv[VW];
    if constexpr (D1 <= D3) {
      // fold w into the inputs, then accumulate straight into acc
#pragma unroll
      for (int m = 0; m < D1; ++m)
#pragma unroll
        for (int c = 0; c < CPL; ++c) xv[m][c] *= w[c];
      static_for<NP>([&](auto P) {
        constexpr int Pi = decltype(P)::value;
        constexpr Pair pr = CGp::pair[Pi];
        if constexpr (Pi % VW == 0) lds16(cyv, cyr + Pi);
#pragma unroll
        for (int c = 0; c < CPL; ++c) acc[pr.m3][c] = fma(cyv[Pi % VW], xv[pr.m1][c], acc[pr.m3][c]);
      });
    } else {
      // contract first, then weight the (fewer) output components
      T t[D3][CPL];
      static_for<NP>([&](auto P) {
        constexpr int Pi = decltype(P)::value;
        constexpr Pair pr = CGp::pair[Pi];
        if constexpr (Pi % VW == 0) lds16(cyv, cyr + Pi);
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
          if constexpr (first_m3<CGp>(Pi))
            t[pr.m3][c] = cyv[Pi % VW] * xv[pr.m1][c];
          else
            t[pr.m3][c] = fma(cyv[Pi % VW], xv[pr.m1][c], t[pr.m3][c]);
        }
      });
      static_for<D3>([&](auto M) {
        constexpr int m3 = decltype(M)::value;
        if constexpr (has_m3<CGp>(m3)) {
#pragma unroll
          for (int c = 0; c < CPL; ++c) acc[m3][c] = fma(w[c], t[m3][c], acc[m3][c]);
        }
      });
    }
  }
  }
  cp_wait<0>();
}

template <typename T, int KP, int CPL, int L1M, int L2M, int L3>
__device__ __forceinline__ void fwd_tile(const UvuFwdParams<T>& p, const TileD& tl, int i, int lane,
                                         const FwdSmem<T>& s, int pw, int ps) {
  constexpr int D3 = 2 * L3 + 1;
  T acc[D3][CPL];
#pragma unroll
  for (int m = 0; m < D3; ++m)
#pragma unroll
    for (int c = 0; c < CPL; ++c) acc[m][c] = T(0);
  const bool active = lane * CPL < tl.nch;
  // inactive lanes read a valid channel and never store
  const int chl = tl.ch0 + (active ? lane * CPL : 0);
  int e0 = ldg(p.rowptr + i), e1 = ldg(p.rowptr + i + 1);
  if (e0 < 0 || e1 < e0 || e1 > p.E) {
    raise_error(p.err, kErrCsr);
    e1 = e0;
  }
  for (int c0 = e0; c0 < e1; c0 += p.chunk) {
    const int n = min(p.chunk, e1 - c0);
    // ---- stage: lane k owns edge c0 + k
    if (lane < n) {
      const int e = c0 + lane;
      int j = ldg(p.senders + e);
      if ((unsigned)j >= (unsigned)p.N) {
        atomicOr(p.err, kErrIndex);
        j = -1;
      }
      s.j[lane] = j;
      T ph[KP];
      load_phi<KP>(ph, p.phi + (size_t)e * p.K, p.K);
#pragma unroll
      for (int q = 0; q < KP; ++q) s.phi[lane * KP + q] = j < 0 ? T(0) : ph[q];
      const T* yrow = p.Y + (size_t)e * p.dim_y;
      T* cyrow = s.cy + lane * p.cy_stride;
      for (int pi = tl.pbeg + pw; pi < tl.pend; pi += ps) {
        const PathD& pd = p.paths[pi];
        dispatch_l1l2<L3, L1M, L2M>(pd.l1, pd.l2, [&](auto A1, auto A2) {
          stage_cy<T, decltype(A1)::value, decltype(A2)::value, L3>(yrow, cyrow + pd.cy_off);
        });
      }
      if (j < 0) s.j[lane] = 0;  // a skipped edge contributes zero (phi = 0)
    }
    __syncwarp();
    // ---- sweep: every path of the tile (of this warp's share) over the staged chunk
    for (int pi = tl.pbeg + pw; pi < tl.pend; pi += ps) {
      const PathD& pd = p.paths[pi];
      dispatch_l1l2<L3, L1M, L2M>(pd.l1, pd.l2, [&](auto A1, auto A2) {
        fwd_path<T, KP, CPL, fwd_ring_g(sizeof(T), CPL, L1M), decltype(A1)::value, decltype(A2)::value, L3>(
            p, pd, s, n, chl, acc);
      });
    }
    __syncwarp();
  }
  if (ps > 1) {
    // split mode: red[warp][m][32 CPL] after the warps' slices, added in warp order
    extern __shared__ __align__(16) unsigned char smem_raw[];
    constexpr int RW = 32 * CPL;
    const int warp = threadIdx.x >> 5;
    T* red = reinterpret_cast<T*>(smem_raw + (size_t)ps * p.warp_smem);
#pragma unroll
    for (int m = 0; m < D3; ++m)
#pragma unroll
      for (int c = 0; c < CPL; ++c) red[(warp * D3 + m) * RW + lane * CPL + c] = acc[m][c];
    __syncthreads();
    if (warp == 0) {
      for (int w = 1; w < ps; ++w)
#pragma unroll
        for (int m = 0; m < D3; ++m)
#pragma unroll
          for (int c = 0; c < CPL; ++c) acc[m][c] += red[(w * D3 + m) * RW + lane * CPL + c];
    }
    if (warp != 0) return;
  }
  if (active) {
    T* o = p.out + (size_t)i * p.c_out + tl.off + chl;
#pragma unroll
    for (int m = 0; m < D3; ++m) store_ch<CPL>(o + m * tl.mul, acc[m]);
  }
}

// fp32: one CTA of 16 warps per SM (a 128-register cap); fp64: two CTAs of 4
// warps. The warps of a CTA work on one tile's path family at a time.
template <typename T, int KP, int CPL, int L1M, int L2M, int L3M>
__global__ void __launch_bounds__(fwd_warps<T>() * 32, ctas_per_sm_for(sizeof(T)))
uvu_fwd_kernel(const __grid_constant__ UvuFwdParams<T> p) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const bool split = p.split > 1;   // split mode: one task per CTA, paths dealt to its warps
  const long long task = split ? (long long)blockIdx.x : (long long)blockIdx.x * fwd_warps<T>() + warp;
  const long long per_win = (long long)kWin * p.n_tiles;
  const long long win = task / per_win;
  const int r = (int)(task - win * per_win);
  const int tile = r / kWin;
  const long long i = win * kWin + (r % kWin);
  if (i >= p.N) return;   // uniform over the CTA in split mode
  const TileD& tl = p.tiles[tile];
  const FwdSmem<T> s = fwd_smem<T, KP>(p, warp);
  dispatch_l<L3M>(tl.l, [&](auto L) {
    fwd_tile<T, KP, CPL, L1M, L2M, decltype(L)::value>(p, tl, (int)i, lane, s, split ? warp : 0,
                                                       split ? p.split : 1);
  });
}

}  // namespace

template <typename T, int KP, int CPL, int L1M, int L2M, int L3M>
cudaError_t launch_uvu_fwd(const UvuFwdParams<T>& p0, cudaStream_t s) {
  UvuFwdParams<T> p = p0;
  const long long wins = ((long long)p.N + kWin - 1) / kWin;
  const long long tasks = wins * kWin * p.n_tiles;
  if (tasks == 0) return cudaSuccess;
  constexpr int W = fwd_warps<T>();
  // split mode while one warp per task would not fill the resident warp slots
  // of one wave (and the warps' accumulators fit beside their slices)
  const size_t red = sizeof(T) * (size_t)W * (2 * L3M + 1) * 32 * CPL;
  const bool small = (long long)p.N * p.n_tiles <= (long long)kSMs * ctas_per_sm_for(sizeof(T)) * W;
  p.split = small && (size_t)p.warp_smem * W + red <= (size_t)227 * 1024 ? W : 1;
  const long long blocks = p.split > 1 ? tasks : (tasks + W - 1) / W;
  const size_t smem = (size_t)p.warp_smem * W + (p.split > 1 ? red : 0);
  auto kern = uvu_fwd_kernel<T, KP, CPL, L1M, L2M, L3M>;
  static SmemLimit limit;
  if (cudaError_t e = limit.ensure((const void*)kern, smem); e != cudaSuccess) return e;
  kern<<<(unsigned)blocks, W * 32, smem, s>>>(p);
  return cudaGetLastError();
}

// degree profiles (max input l, max SH l, max output l): see plan.cpp
#define TPC_INST(T, KP, CPL, A, B, C) \
  template cudaError_t launch_uvu_fwd<T, KP, CPL, A, B, C>(const UvuFwdParams<T>&, cudaStream_t);
#define TPC_INST_P(T, KP, CPL) \
  TPC_INST(T, KP, CPL, 2, 2, 2) TPC_INST(T, KP, CPL, 1, 3, 3) TPC_INST(T, KP, CPL, 3, 3, 3)
#if TPC_WANT(0)
TPC_INST_P(float, 8, 1)
TPC_INST(float, 8, 1, 4, 4, 4)
#endif
#if TPC_WANT(1)
TPC_INST_P(float, 8, 2)
#endif
#if TPC_WANT(9)
TPC_INST(float, 8, 1, 6, 6, 6)
#endif
#if TPC_WANT(2)
TPC_INST(float, 8, 2, 4, 4, 4)
#endif
#if TPC_WANT(3)
TPC_INST_P(float, 16, 1)
TPC_INST(float, 16, 1, 4, 4, 4)
#endif
#if TPC_WANT(4)
TPC_INST_P(float, 16, 2)
TPC_INST(float, 16, 2, 4, 4, 4)
#endif
#if TPC_WANT(5)
TPC_INST_P(double, 8, 1)
TPC_INST(double, 8, 1, 4, 4, 4)
#endif
#if TPC_WANT(6)
TPC_INST_P(double, 8, 2)
#endif
#if TPC_WANT(7)
TPC_INST_P(double, 16, 1)
TPC_INST(double, 16, 1, 4, 4, 4)
#endif
#if TPC_WANT(8)
TPC_INST_P(double, 16, 2)
#endif
#undef TPC_INST_P
#undef TPC_INST

}  // namespace tpc
