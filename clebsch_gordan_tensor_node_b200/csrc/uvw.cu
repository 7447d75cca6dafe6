// Fully connected (uvw) path: receiver state S, its backward edge pass, and the
// repacking of A for the channel-mixing GEMMs.
//
// Forward (Sobek §4.2):
//   C_{pi,u,mo}(x_j, Y_ij)   = sum_{mi,my} c^pi x_{j,pi,u,mi} Y_{ij,my}          (Eq. 32)
//   S_{i,pi,q,u,mo}          = sum_{j in N(i)} phi_{ij,q} C_{pi,u,mo}(x_j, Y_ij) (Eq. 33)
//   m^(g)_{i,w,mo}           = sum_{pi in g} sum_{q,u} S_{i,pi,q,u,mo} A_{q,pi,u,w} (Eqs. 34-35)
// S has no output-channel axis. It is built here for a bounded chunk of
// receivers (Sobek §4.2: receiver ranges under a fixed scratch budget), laid out
// per output block g as rows (receiver, mo) x columns (pi, q, u), and mixed by
// one GEMM per block (gemm.cu).
//
// Backward (Sobek §4.3, Eq. 36): A_bar = S^T m_bar and S_bar = m_bar A^T by
// GEMM; the edge pass below differentiates Eq. 33 per edge, in receiver order:
//   phi_bar_{e,q} = sum_{pi,u,mo} S_bar_{i,pi,q,u,mo} C_{pi,u,mo}(x_j, Y_e)
//   Y_bar_e       = sum_pi D_Y C^*[ T_bar ],  T_bar_{pi,u,mo} = sum_q phi_{e,q} S_bar_{i,pi,q,u,mo}
// x_bar is the forward structure on the source view: with the adjoint coupling
// C'_{pi,w,mi} = sum_{my,mo} c^pi Y_{e,my} m_bar_{recv(e),pi,w,mo}, the state
// S'_{j,pi,q,w,mi} = sum_{e: src=j} phi_{e,q} C'_{pi,w,mi} is built by the same
// kernel (direction 1) and x_bar_j = S'_j A'^T by GEMM -- no per-edge adjoint
// tensor and no per-edge read of S_bar.
#include "common.cuh"
#include "kernels.h"

namespace tpc {
namespace {

constexpr int kThreads = 128;      // 4 warps
constexpr int kChunk = 32;         // edges staged per round

template <typename T, int KP>
struct SbSmem {
  T* C;     // [kChunk][DOmax][32]
  T* phi;   // [kChunk][KP]
};

// One m16n8k8 tensor-core product with tf32 operands and fp32 accumulation.
__device__ __forceinline__ void mma_tf32(float (&d)[4], const unsigned (&a)[4], const unsigned (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}
// x = hi + lo with hi holding the top 19 bits (a tf32 value) and lo the exact
// remainder; the tensor core reads lo's top 19 bits.
__device__ __forceinline__ void split_tf32(float x, unsigned& hi, unsigned& lo) {
  hi = __float_as_uint(x) & 0xFFFFE000u;
  lo = __float_as_uint(x - __uint_as_float(hi));
}

// One path of one owner block: accumulate the state columns (q, channel) of
// this CTA's channel tile over the owner's edges, then store them.
//
// Phase A (all types): the warps contract the CG product C[e][mo][u] of the
// chunk's edges into shared memory, lane = channel u.
// Phase B, fp32: S[q][(mo, u)] += sum_e phi[e][q] C[e][mo][u] is a product with
// 16 rows (q), 32 DO columns and the chunk's edges as inner dimension; it runs
// on the tensor cores as m16n8k8 tf32 products in three parts (hi*hi + hi*lo +
// lo*hi, the fp32-accurate split), warp w owning channels 8w .. 8w + 7 of every
// component. fp64: warp w owns radial indices 4w .. 4w + 3, lane = channel,
// plain FMAs.
template <typename T, int KP, int DIR, int L1, int L2, int L3>
__device__ __forceinline__ void sbuild_path(const UvwSParams<T>& p, const UvwBlockD& bd, const PathD& pd,
                                            int r, int k0, int k1, T* Cs, T* phis) {
  using CGp = cgt::CG<L1, L2, L3>;
  constexpr int D1 = 2 * L1 + 1, D3 = 2 * L3 + 1;
  constexpr int DG = DIR == 0 ? D1 : D3;   // components of the gathered block
  constexpr int DO = DIR == 0 ? D3 : D1;   // components of the owner block
  constexpr int KQ = KP / 4;
  constexpr bool kTC = sizeof(T) == 4;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tig = lane & 3;   // mma fragment coordinates
  const int gmul = pd.mul_in;              // gathered multiplicity (direction-specific)
  for (int c0 = 0; c0 < gmul; c0 += 32) {
    const bool act = c0 + lane < gmul;
    const int cl = act ? c0 + lane : c0;
    T Sr[kTC ? 1 : KQ][DO];                  // fp64 accumulators
    float acc[kTC ? DO : 1][4];              // fp32: [component][mma C fragment]
#pragma unroll
    for (int m = 0; m < DO; ++m) {
      if constexpr (kTC) {
        acc[m][0] = acc[m][1] = acc[m][2] = acc[m][3] = 0.f;
      } else {
#pragma unroll
        for (int q = 0; q < KQ; ++q) Sr[q][m] = T(0);
      }
    }
    for (int kc = k0; kc < k1; kc += kChunk) {
      const int n = min(kChunk, k1 - kc);
      // phase A: warp w contracts the CG product of chunk edges w, w+4, ...
      for (int t = warp; t < n; t += 4) {
        const int k = kc + t;
        const int e = p.eid ? ldg(p.eid + k) : k;
        const int nb = ldg(p.nbr + k);
        const bool ok = (unsigned)e < (unsigned)p.E && (unsigned)nb < (unsigned)p.n_feat_rows;
        if (!ok) raise_error(p.err, kErrIndex);
        T y[2 * L2 + 1];
        T g[DG];
#pragma unroll
        for (int m = 0; m < 2 * L2 + 1; ++m) y[m] = ok ? ldg(p.Y + (size_t)e * p.dim_y + L2 * L2 + m) : T(0);
        const T* gr = p.feat + (size_t)(ok ? nb : 0) * p.ld_feat + pd.x_off + cl;
#pragma unroll
        for (int m = 0; m < DG; ++m) g[m] = ldg(gr + (size_t)m * gmul);
        T C[DO];
#pragma unroll
        for (int m = 0; m < DO; ++m) C[m] = T(0);
        static_for<CGp::npair>([&](auto P) {
          constexpr Pair pr = CGp::pair[decltype(P)::value];
          const T cy = pair_coef<T, CGp, decltype(P)::value>(y);
          if constexpr (DIR == 0)
            C[pr.m3] = fma(cy, g[pr.m1], C[pr.m3]);
          else
            C[pr.m1] = fma(cy, g[pr.m3], C[pr.m1]);
        });
#pragma unroll
        for (int m = 0; m < DO; ++m) Cs[(t * DO + m) * 32 + lane] = (act && ok) ? C[m] : T(0);
        if (lane < KP) phis[t * KP + lane] = (ok && lane < p.K) ? ldg(p.phi + (size_t)e * p.K + lane) : T(0);
      }
      if constexpr (kTC) {
        // zero rows up to the next multiple of 8 edges (the last mma step)
        const int n8 = (n + 7) & ~7;
        for (int t = n + warp; t < n8; t += 4) {
#pragma unroll
          for (int m = 0; m < DO; ++m) Cs[(t * DO + m) * 32 + lane] = T(0);
          if (lane < KP) phis[t * KP + lane] = T(0);
        }
      }
      __syncthreads();
      if constexpr (kTC) {
        // phase B on the tensor cores: A = phi^T (16 x 8 edges), B = C (8 edges x 8 channels)
        const float* Cf = reinterpret_cast<const float*>(Cs);
        const float* Pf = reinterpret_cast<const float*>(phis);
        for (int e0 = 0; e0 < n; e0 += 8) {
          unsigned ah[4], al[4];
          {
            const int ea = e0 + tig, eb = e0 + tig + 4;
            const float v0 = gid < KP ? Pf[ea * KP + gid] : 0.f;
            const float v1 = gid + 8 < KP ? Pf[ea * KP + gid + 8] : 0.f;
            const float v2 = gid < KP ? Pf[eb * KP + gid] : 0.f;
            const float v3 = gid + 8 < KP ? Pf[eb * KP + gid + 8] : 0.f;
            split_tf32(v0, ah[0], al[0]);
            split_tf32(v1, ah[1], al[1]);
            split_tf32(v2, ah[2], al[2]);
            split_tf32(v3, ah[3], al[3]);
          }
#pragma unroll
          for (int m = 0; m < DO; ++m) {
            unsigned bh[2], bl[2];
            split_tf32(Cf[((e0 + tig) * DO + m) * 32 + warp * 8 + gid], bh[0], bl[0]);
            split_tf32(Cf[((e0 + tig + 4) * DO + m) * 32 + warp * 8 + gid], bh[1], bl[1]);
            mma_tf32(acc[m], al, bh);
            mma_tf32(acc[m], ah, bl);
            mma_tf32(acc[m], ah, bh);
          }
        }
      } else {
        // phase B: S[q][m] += phi[q] C[m] for this warp's radial indices
        for (int t = 0; t < n; ++t) {
          T cm[DO];
#pragma unroll
          for (int m = 0; m < DO; ++m) cm[m] = Cs[(t * DO + m) * 32 + lane];
#pragma unroll
          for (int q = 0; q < KQ; ++q) {
            const T ph = phis[t * KP + warp * KQ + q];
#pragma unroll
            for (int m = 0; m < DO; ++m) Sr[q][m] = fma(ph, cm[m], Sr[q][m]);
          }
        }
      }
      __syncthreads();
    }
    T* dst = p.S + (size_t)p.nr_alloc * bd.s_off + (size_t)(r - p.r0) * DO * bd.dcols + pd.col_off;
    // the accumulate choice is taken once, outside the unrolled store loops
    auto store = [&](auto Acc) {
      constexpr bool kAcc = decltype(Acc)::value;
      if constexpr (kTC) {
        // C fragment: rows q = gid, gid + 8; columns u = 8 warp + 2 tig, + 1
        const int u = c0 + warp * 8 + 2 * tig;
#pragma unroll
        for (int m = 0; m < DO; ++m) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int q = gid + 8 * h;
            if (q >= p.K) continue;
            T* row = dst + (size_t)m * bd.dcols + (size_t)q * gmul;
            if (u < gmul) row[u] = kAcc ? row[u] + acc[m][2 * h] : acc[m][2 * h];
            if (u + 1 < gmul) row[u + 1] = kAcc ? row[u + 1] + acc[m][2 * h + 1] : acc[m][2 * h + 1];
          }
        }
      } else if (act) {
#pragma unroll
        for (int q = 0; q < KQ; ++q) {
          const int qq = warp * KQ + q;
          if (qq < p.K) {
#pragma unroll
            for (int m = 0; m < DO; ++m) {
              T* o = dst + (size_t)m * bd.dcols + (size_t)qq * gmul + cl;
              *o = kAcc ? *o + Sr[q][m] : Sr[q][m];
            }
          }
        }
      }
    };
    if (p.accumulate)
      store(std::true_type{});
    else
      store(std::false_type{});
  }
}

template <typename T, int KP, int DIR>
__global__ void __launch_bounds__(kThreads) uvw_sbuild_kernel(const __grid_constant__ UvwSParams<T> p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  T* Cs = reinterpret_cast<T*>(smem_raw);
  T* phis = Cs + kChunk * (2 * kLmax + 1) * 32;
  const int r = p.r0 + blockIdx.x;
  const UvwBlockD& bd = p.blocks[blockIdx.y];
  if (r >= p.N || bd.pbeg == bd.pend) return;
  int k0 = ldg(p.ptr + r), k1 = ldg(p.ptr + r + 1);
  if (k0 < 0 || k1 < k0 || k1 > p.E) {
    raise_error(p.err, kErrCsr);
    k1 = k0;
  }
  dispatch_l(bd.l, [&](auto LO) {
    constexpr int L = decltype(LO)::value;
    for (int pi = bd.pbeg; pi < bd.pend; ++pi) {
      const PathD& pd = p.paths[pi];
      if constexpr (DIR == 0) {
        dispatch_l1l2<L>(pd.l1, pd.l2, [&](auto A1, auto A2) {
          sbuild_path<T, KP, 0, decltype(A1)::value, decltype(A2)::value, L>(p, bd, pd, r, k0, k1, Cs, phis);
        });
      } else {
        dispatch_l2l3<L>(pd.l2, pd.l3, [&](auto A2, auto A3) {
          sbuild_path<T, KP, 1, L, decltype(A2)::value, decltype(A3)::value>(p, bd, pd, r, k0, k1, Cs, phis);
        });
      }
    }
  });
}

// ---------------------------------------------------------------- edge pass
//
// One CTA (kEdgeWarps warps) per receiver r. The receiver's edges go in rounds
// of 32: lane l of every warp owns edge slot l of the round. The work of a
// round is a sequence of stages, one per (path, tile of kEdgeTile input
// channels u); each warp takes an equal share of the tile's channels. For each
// stage the CTA copies into shared memory the gathered x[m1][u] of the 32
// senders and S_bar[mo][u][q] of r, with cp.async, one stage ahead of the
// arithmetic (two buffers). S_bar of r is laid out per path as (mo, u, q) with
// the K radial values contiguous (the backward packs A in that column order),
// so all lanes of a warp read the same S_bar values (shared-memory broadcast)
// while each contracts its own edge:
//   C[mo]        = sum c x[mi] Y[my]                     (per edge, channel u)
//   T_bar[u][mo] = sum_q phi_e[q] S_bar[mo][u][q]
//   phi_bar_e[q] += sum_{u,mo} S_bar[mo][u][q] C[mo]
//   Y_bar_e[my]  += sum c x[mi] T_bar[mo]
// The loops over u and mo are not unrolled (C and T_bar pass through a
// per-lane shared column), which keeps a path's loop body small enough for the
// instruction cache. phi_bar_e accumulates in registers, Y_bar_e in a per-warp
// shared column; the warps' partial sums are added in warp order at the end of
// the round, so the result does not depend on timing.

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  const unsigned d = (unsigned)__cvta_generic_to_shared(dst);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(d), "l"(src) : "memory");
}
template <int B>
__device__ __forceinline__ void cp_async_small(void* dst, const void* src) {   // B = 4 or 8 bytes
  const unsigned d = (unsigned)__cvta_generic_to_shared(dst);
  asm volatile("cp.async.ca.shared.global [%0], [%1], %2;\n" ::"r"(d), "l"(src), "n"(B) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }

struct EdgeStage {
  int pi, c0;   // path and first channel of the tile; pi == n_paths ends the round
};

// Issue the copies of one stage into buffer (Xs, Ss). x goes as single
// scalars into [slot][mi][u] rows of odd stride (conflict-free reads by slot);
// S_bar as 16-byte pieces where the layout allows, else plain loads.
template <typename T>
__device__ __forceinline__ void edge_stage_issue(const UvwEdgeParams<T>& p, const EdgeStage& st, int r,
                                                 const int* js, T* Xs, T* Ss) {
  constexpr int VW = sizeof(T) == 4 ? 4 : 2;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const PathD& pd = p.paths[st.pi];
  const UvwBlockD& bd = p.blocks[p.path_blk[st.pi]];
  const int d1 = 2 * pd.l1 + 1, d3 = 2 * pd.l3 + 1, mi = pd.mul_in;
  const int nc = min(kEdgeTile, mi - st.c0), row = d1 * nc, ss = edge_slot_stride(row);
  const T* xb = p.x + pd.x_off + st.c0;
  const T* sb = p.Sbar + (size_t)p.nr_alloc * bd.s_off + (size_t)(r - p.r0) * d3 * bd.dcols + pd.col_off +
                (size_t)st.c0 * p.K;
  const int srow = nc * p.K;   // S_bar scalars per component in the tile
  for (int sl = warp; sl < 32; sl += kEdgeWarps) {
    const T* src = xb + (size_t)js[sl] * p.c_in;
    T* dst = Xs + sl * ss;
    for (int c = lane; c < row; c += 32) {
      const int m = c / nc, u = c - m * nc;
      if (p.vec)
        cp_async_small<sizeof(T)>(dst + c, src + m * mi + u);
      else
        dst[c] = ldg(src + m * mi + u);
    }
  }
  if (p.vec) {
    const int nsv = srow / VW;
    for (int t = threadIdx.x; t < d3 * nsv; t += kEdgeThreads) {
      const int m = t / nsv, c = (t - m * nsv) * VW;
      cp_async16(Ss + m * srow + c, sb + (size_t)m * bd.dcols + c);
    }
  } else {
    for (int t = threadIdx.x; t < d3 * srow; t += kEdgeThreads) {
      const int m = t / srow, c = t - m * srow;
      Ss[m * srow + c] = ldg(sb + (size_t)m * bd.dcols + c);
    }
  }
}

template <typename T, int L1, int L2, int L3, int KP>
__device__ __forceinline__ void edge_stage_compute(const UvwEdgeParams<T>& p, const PathD& pd, int c0, int e,
                                                   bool ok, const T* Xs, const T* Ss, T* CT,
                                                   const T (&ph)[KP], T (&gphi)[KP], T* gyr) {
  using CGp = cgt::CG<L1, L2, L3>;
  constexpr int D1 = 2 * L1 + 1, D2 = 2 * L2 + 1, D3 = 2 * L3 + 1, NP = CGp::npair, Y0 = L2 * L2;
  constexpr int VW = sizeof(T) == 4 ? 4 : 2;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nc = min(kEdgeTile, pd.mul_in - c0), ss = edge_slot_stride(D1 * nc);
  const int uw = (nc + kEdgeWarps - 1) / kEdgeWarps;
  const int u0 = warp * uw, u1 = min(nc, u0 + uw);
  if (u0 >= u1) return;
  T y[D2], cy[NP], gy[D2];
#pragma unroll
  for (int m = 0; m < D2; ++m) {
    y[m] = ok ? ldg(p.Y + (size_t)e * p.dim_y + Y0 + m) : T(0);
    gy[m] = T(0);
  }
  static_for<NP>([&](auto P) { cy[decltype(P)::value] = pair_coef<T, CGp, decltype(P)::value>(y); });
  const T* xs = Xs + lane * ss;
  const int srow = nc * p.K;
  T* ct = CT + lane;   // this lane's column: C[mo], then T_bar[mo]
#pragma unroll 1
  for (int u = u0; u < u1; ++u) {
    T xv[D1];
#pragma unroll
    for (int m = 0; m < D1; ++m) xv[m] = xs[m * nc + u];
    {
      T C[D3];
#pragma unroll
      for (int m = 0; m < D3; ++m) C[m] = T(0);
      static_for<NP>([&](auto P) {
        constexpr Pair pr = CGp::pair[decltype(P)::value];
        C[pr.m3] = fma(cy[decltype(P)::value], xv[pr.m1], C[pr.m3]);
      });
#pragma unroll
      for (int m = 0; m < D3; ++m) ct[m * 32] = C[m];
    }
    const T* su = Ss + u * p.K;
#pragma unroll 1
    for (int m = 0; m < D3; ++m) {
      const T cm = ct[m * 32];
      const T* sr = su + m * srow;
      T acc[4] = {T(0), T(0), T(0), T(0)};   // four independent chains over q
      if (p.vec) {
#pragma unroll
        for (int q = 0; q < KP; q += VW) {
          if constexpr (VW == 4) {
            const float4 v = *reinterpret_cast<const float4*>(sr + q);
            acc[0] = fma(ph[q], v.x, acc[0]); gphi[q] = fma(v.x, cm, gphi[q]);
            acc[1] = fma(ph[q + 1], v.y, acc[1]); gphi[q + 1] = fma(v.y, cm, gphi[q + 1]);
            acc[2] = fma(ph[q + 2], v.z, acc[2]); gphi[q + 2] = fma(v.z, cm, gphi[q + 2]);
            acc[3] = fma(ph[q + 3], v.w, acc[3]); gphi[q + 3] = fma(v.w, cm, gphi[q + 3]);
          } else {
            const double2 v = *reinterpret_cast<const double2*>(sr + q);
            acc[(q >> 1) & 2] = fma(ph[q], v.x, acc[(q >> 1) & 2]); gphi[q] = fma(v.x, cm, gphi[q]);
            acc[((q >> 1) & 2) + 1] = fma(ph[q + 1], v.y, acc[((q >> 1) & 2) + 1]);
            gphi[q + 1] = fma(v.y, cm, gphi[q + 1]);
          }
        }
      } else {
#pragma unroll
        for (int q = 0; q < KP; ++q) {
          const T v = q < p.K ? sr[q] : T(0);
          acc[q & 3] = fma(ph[q], v, acc[q & 3]);
          gphi[q] = fma(v, cm, gphi[q]);
        }
      }
      ct[m * 32] = (acc[0] + acc[1]) + (acc[2] + acc[3]);
    }
    T tb[D3];
#pragma unroll
    for (int m = 0; m < D3; ++m) tb[m] = ct[m * 32];
    static_for<NP>([&](auto P) {
      constexpr Pair pr = CGp::pair[decltype(P)::value];
      const T z = xv[pr.m1] * tb[pr.m3];
      static_for<pr.n>([&](auto q) {
        constexpr Term tm = CGp::term[pr.start + decltype(q)::value];
        gy[tm.m2] = fma(T(tm.c), z, gy[tm.m2]);
      });
    });
  }
#pragma unroll
  for (int m = 0; m < D2; ++m) gyr[(Y0 + m) * 32] += gy[m];
}

template <typename T>
__device__ __forceinline__ EdgeStage edge_next(const UvwEdgeParams<T>& p, EdgeStage st) {
  st.c0 += kEdgeTile;
  if (st.c0 >= p.paths[st.pi].mul_in) {
    st.c0 = 0;
    ++st.pi;
  }
  return st;
}

template <typename T, int KP>
__global__ void __launch_bounds__(kEdgeThreads, sizeof(T) == 4 ? 3 : 1)
uvw_edge_kernel(const __grid_constant__ UvwEdgeParams<T> p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  T* const buf0 = reinterpret_cast<T*>(smem_raw);   // two stage buffers: x part, then S_bar part
  const int stage_n = p.smem_stage / (int)sizeof(T), xn = (p.smem_stage - p.smem_sbar) / (int)sizeof(T);
  T* Red = reinterpret_cast<T*>(smem_raw + 2 * p.smem_stage);                        // [warps][dim_y][32]
  T* CTs = reinterpret_cast<T*>(smem_raw + 2 * p.smem_stage + p.smem_red);           // [warps][2 kLmax + 1][32]
  int* js = reinterpret_cast<int*>(smem_raw + 2 * p.smem_stage + p.smem_red + p.smem_ct);   // [32]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int r = p.r0 + blockIdx.x;
  if (r >= p.N || p.n_blocks == 0) return;
  const int k0 = ldg(p.rowptr + r), k1 = ldg(p.rowptr + r + 1);
  if (k0 < 0 || k1 < k0 || k1 > p.E) {
    if (threadIdx.x == 0) raise_error(p.err, kErrCsr);
    return;
  }
  const int n_paths = p.blocks[p.n_blocks - 1].pend;
  T* CT = CTs + (size_t)warp * (2 * kLmax + 1) * 32;
  for (int e0 = k0; e0 < k1; e0 += 32) {
    const int e = e0 + lane;
    bool ok = e < k1;
    int j = 0;
    if (ok) {
      j = ldg(p.senders + e);
      if ((unsigned)j >= (unsigned)p.N) {
        if (warp == 0) atomicOr(p.err, kErrIndex);
        ok = false;
        j = 0;
      }
    }
    __syncthreads();   // the previous round is done with js, the buffers and Red
    if (warp == 0) js[lane] = j;
    T ph[KP], gphi[KP];
#pragma unroll
    for (int q = 0; q < KP; ++q) {
      ph[q] = (ok && q < p.K) ? ldg(p.phi + (size_t)e * p.K + q) : T(0);
      gphi[q] = T(0);
    }
    T* gyr = Red + (size_t)warp * p.dim_y * 32 + lane;   // this lane's Y_bar column
    for (int m = 0; m < p.dim_y; ++m) gyr[m * 32] = T(0);
    __syncthreads();   // js visible
    EdgeStage st{0, 0};
    edge_stage_issue(p, st, r, js, buf0, buf0 + xn);
    cp_async_commit();
    for (int s = 0; st.pi < n_paths; ++s) {
      const EdgeStage nx = edge_next(p, st);
      T* cur = buf0 + (s & 1) * stage_n;
      T* nxt = buf0 + ((s + 1) & 1) * stage_n;
      if (nx.pi < n_paths) edge_stage_issue(p, nx, r, js, nxt, nxt + xn);
      cp_async_commit();
      cp_async_wait<1>();   // this stage's copies have landed (own thread)
      __syncthreads();      // ... and every thread's
      const PathD& pd = p.paths[st.pi];
      dispatch_l(pd.l3, [&](auto L3c) {
        constexpr int L3 = decltype(L3c)::value;
        dispatch_l1l2<L3>(pd.l1, pd.l2, [&](auto A1, auto A2) {
          edge_stage_compute<T, decltype(A1)::value, decltype(A2)::value, L3, KP>(
              p, pd, st.c0, e, ok, cur, cur + xn, CT, ph, gphi, gyr);
        });
      });
      __syncthreads();      // buffer cur is free for the stage after next
      st = nx;
    }
    cp_async_wait<0>();
    // ---- add the warps' partial sums in a fixed order (phi_bar via buffer 0)
    T* Rp = buf0;   // [warps][K][32]
#pragma unroll
    for (int q = 0; q < KP; ++q)
      if (q < p.K) Rp[((size_t)warp * p.K + q) * 32 + lane] = gphi[q];
    __syncthreads();
    const int n = min(32, k1 - e0), nv = p.K + p.dim_y;
    for (int t = threadIdx.x; t < nv * 32; t += kEdgeThreads) {
      const int v = t >> 5, sl = t & 31;
      if (sl >= n) continue;
      const size_t eo = (size_t)e0 + sl;
      if (v < p.K) {
        T acc = Rp[(size_t)v * 32 + sl];
#pragma unroll
        for (int w = 1; w < kEdgeWarps; ++w) acc += Rp[((size_t)w * p.K + v) * 32 + sl];
        if (p.accumulate) acc += p.gphi[eo * p.K + v];
        p.gphi[eo * p.K + v] = acc;
      } else {
        const int m = v - p.K;
        T acc = Red[(size_t)m * 32 + sl];
#pragma unroll
        for (int w = 1; w < kEdgeWarps; ++w) acc += Red[((size_t)w * p.dim_y + m) * 32 + sl];
        if (p.accumulate) acc += p.gY[eo * p.dim_y + m];
        p.gY[eo * p.dim_y + m] = acc;
      }
    }
  }
}

// ---------------------------------------------------------------- A repacking

// Column (within A's row q) to packed row/col: every element of A [K, N_w] is
// copied to the forward layout B_g [(pi, q, u), w] and the adjoint layout
// B'_b [(pi, q, w), u] (or the reverse for the unpack of A_bar).
// Layouts: Bf (forward, SIMT) [(pi,q,u), w]; Ba (adjoint, SIMT) [(pi,q,w), u];
// Btf / Bta: the same transposed, [w, (pi,q,u)] / [u, (pi,q,w)] (K-major operands
// of the tensor-core GEMM). Any output may be NULL.
template <typename T>
__device__ __forceinline__ T hi_part(T v) {
  if constexpr (sizeof(T) == 4)
    return __uint_as_float(__float_as_uint(v) & 0xFFFFE000u);
  else
    return v;
}

template <typename T>
__global__ void pack_a_kernel(const __grid_constant__ UvwPackParams p, const T* __restrict__ A,
                              T* __restrict__ Bf, T* __restrict__ Ba, T* __restrict__ Btf,
                              T* __restrict__ Bta, T* __restrict__ Btf_lo, T* __restrict__ Bta_lo) {
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)p.K * p.n_w) return;
  const int q = (int)(idx / p.n_w);
  const int col = (int)(idx - (long long)q * p.n_w);
  int lo = 0, hi = p.n_paths;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (p.paths[mid].w_off <= col) lo = mid; else hi = mid;
  }
  const PackPath& pp = p.paths[lo];
  const int rem = col - pp.w_off, u = rem / pp.mo, w = rem - u * pp.mo;
  const T v = A[idx];
  if (Bf) {
    const size_t rowf = p.bf_uq ? (size_t)u * p.K + q : (size_t)q * pp.mi + u;
    Bf[pp.bf_off + ((size_t)pp.colf + rowf) * pp.mo + w] = v;
  }
  if (Ba) Ba[pp.ba_off + ((size_t)pp.cola + (size_t)q * pp.mo + w) * pp.mi + u] = v;
  const T vh = hi_part(v);
  if (Btf) {
    const size_t o = pp.bf_off + (size_t)w * pp.dcf + pp.colf + (size_t)q * pp.mi + u;
    Btf[o] = Btf_lo ? vh : v;
    if (Btf_lo) Btf_lo[o] = v - vh;
  }
  if (Bta) {
    const size_t o = pp.ba_off + (size_t)u * pp.dca + pp.cola + (size_t)q * pp.mo + w;
    Bta[o] = Bta_lo ? vh : v;
    if (Bta_lo) Bta_lo[o] = v - vh;
  }
}

template <typename T>
__global__ void unpack_a_kernel(const __grid_constant__ UvwPackParams p, const T* __restrict__ Bf,
                                T* __restrict__ A) {
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)p.K * p.n_w) return;
  const int q = (int)(idx / p.n_w);
  const int col = (int)(idx - (long long)q * p.n_w);
  int lo = 0, hi = p.n_paths;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (p.paths[mid].w_off <= col) lo = mid; else hi = mid;
  }
  const PackPath& pp = p.paths[lo];
  const int rem = col - pp.w_off, u = rem / pp.mo, w = rem - u * pp.mo;
  A[idx] = Bf[pp.bf_off + ((size_t)pp.colf + (size_t)q * pp.mi + u) * pp.mo + w];
}

}  // namespace

template <typename T, int KP, int DIR>
cudaError_t launch_uvw_sbuild_dir(const UvwSParams<T>& p, cudaStream_t s) {
  if (p.nr <= 0 || p.n_blocks == 0) return cudaSuccess;
  const size_t smem = sizeof(T) * (size_t)(kChunk * (2 * kLmax + 1) * 32 + kChunk * KP);
  dim3 grid(p.nr, p.n_blocks);
  auto k = uvw_sbuild_kernel<T, KP, DIR>;
  static SmemLimit limit;
  if (cudaError_t e = limit.ensure((const void*)k, smem); e != cudaSuccess) return e;
  k<<<grid, kThreads, smem, s>>>(p);
  return cudaGetLastError();
}

template <typename T, int KP>
cudaError_t launch_uvw_edge(const UvwEdgeParams<T>& p, cudaStream_t s) {
  if (p.nr <= 0) return cudaSuccess;
  const size_t smem = 2 * (size_t)p.smem_stage + p.smem_red + p.smem_ct + 32 * sizeof(int);
  auto k = uvw_edge_kernel<T, KP>;
  static SmemLimit limit;
  if (cudaError_t e = limit.ensure((const void*)k, smem); e != cudaSuccess) return e;
  k<<<p.nr, kEdgeThreads, smem, s>>>(p);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_pack_a(const UvwPackParams& p, const T* A, T* Bf, T* Ba, T* Btf, T* Bta, T* Btf_lo,
                          T* Bta_lo, cudaStream_t s) {
  const long long n = (long long)p.K * p.n_w;
  if (n == 0) return cudaSuccess;
  pack_a_kernel<T><<<(unsigned)((n + 255) / 256), 256, 0, s>>>(p, A, Bf, Ba, Btf, Bta, Btf_lo, Bta_lo);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_unpack_a(const UvwPackParams& p, const T* Bf, T* A, cudaStream_t s) {
  const long long n = (long long)p.K * p.n_w;
  if (n == 0) return cudaSuccess;
  unpack_a_kernel<T><<<(unsigned)((n + 255) / 256), 256, 0, s>>>(p, Bf, A);
  return cudaGetLastError();
}

#define TPC_INST_S(T, KP, DIR) \
  template cudaError_t launch_uvw_sbuild_dir<T, KP, DIR>(const UvwSParams<T>&, cudaStream_t);
#define TPC_INST_E(T, KP) template cudaError_t launch_uvw_edge<T, KP>(const UvwEdgeParams<T>&, cudaStream_t);
#if TPC_WANT(0)
template cudaError_t launch_pack_a<float>(const UvwPackParams&, const float*, float*, float*, float*, float*,
                                          float*, float*, cudaStream_t);
template cudaError_t launch_unpack_a<float>(const UvwPackParams&, const float*, float*, cudaStream_t);
template cudaError_t launch_pack_a<double>(const UvwPackParams&, const double*, double*, double*, double*,
                                           double*, double*, double*, cudaStream_t);
template cudaError_t launch_unpack_a<double>(const UvwPackParams&, const double*, double*, cudaStream_t);
TPC_INST_S(float, 8, 0)
#endif
#if TPC_WANT(1)
TPC_INST_S(float, 8, 1)
#endif
#if TPC_WANT(2)
TPC_INST_E(float, 8)
#endif
#if TPC_WANT(3)
TPC_INST_S(float, 16, 0)
#endif
#if TPC_WANT(4)
TPC_INST_S(float, 16, 1)
#endif
#if TPC_WANT(5)
TPC_INST_E(float, 16)
#endif
#if TPC_WANT(6)
TPC_INST_S(double, 8, 0)
TPC_INST_S(double, 8, 1)
#endif
#if TPC_WANT(7)
TPC_INST_E(double, 8)
#endif
#if TPC_WANT(8)
TPC_INST_S(double, 16, 0)
TPC_INST_S(double, 16, 1)
#endif
#if TPC_WANT(9)
TPC_INST_E(double, 16)
#endif
#undef TPC_INST_S
#undef TPC_INST_E

}  // namespace tpc
