// Tensor-core (tcgen05) channel-mixing GEMM of the fully connected path, fp32.
//
// Sobek §4.2 (Eqs. 34-35): m_g = S_g A_g per output block, rows = (receiver,
// output component), contracted dimension = (path, radial index, input
// channel), columns = output channels. This kernel computes C = X B with
// X [M, D] row-major (the receiver state) and B given transposed as
// Bt [N, D] row-major (both K-major operands), and writes C rows straight into
// the ir_mul output block (row-blocked addressing).
//
// FP32-exact on TF32 tensor cores by the three-term split (Ootomo & Yokota
// 2022): x = x_hi + x_lo with x_hi exactly representable in TF32 (low 13
// mantissa bits cleared) and x_lo = x - x_hi; C = X_hi B_hi + X_hi B_lo +
// X_lo B_hi with fp32 accumulation, the dropped X_lo B_lo term is ~2^-22
// relative.
//
// One CTA (4 warps) owns 128 rows and all N (<= 256, padded to a multiple of
// 16) columns; the fp32 accumulator [128 lanes x N columns] lives in tensor
// memory. K is staged 32 at a time into shared memory, double-buffered, in the
// K-major no-swizzle core-matrix layout (8 rows x 16 bytes per core matrix);
// one elected thread issues tcgen05.mma (kind::tf32, M 128, N, K 8) and
// commits to an mbarrier that gates the reuse of the stage. Every wait is
// bounded: on expiry the kernel sets the error word, waits (bounded) for its
// own MMAs, frees its tensor memory and returns.
#include "common.cuh"
#include "kernels.h"

namespace tpc {
namespace {

constexpr int TM = 128;        // rows per CTA (tensor-memory lanes)
constexpr int KT = 32;         // K per stage
constexpr int NSTAGE = 2;
constexpr long long kSpinLimit = 1ll << 22;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// K-major, no swizzle: element (r, k) of a [rows x KT] tile lives at byte
// ((r / 8) * (KT / 4) + k / 4) * 128 + (r % 8) * 16 + (k % 4) * 4.
__device__ __forceinline__ uint32_t tile_off(int r, int kchunk) {
  return (uint32_t)(((r >> 3) * (KT / 4) + kchunk) * 128 + (r & 7) * 16);
}

// Shared-memory matrix descriptor (sm100): start >> 4 at [0,14), leading byte
// offset >> 4 at [16,30) = distance of the two 16-byte K chunks of one K-8
// step, stride byte offset >> 4 at [32,46) = distance of 8-row groups,
// version 1 at [46,48), no swizzle.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr) {
  const uint64_t lbo = 128 >> 4;
  const uint64_t sbo = ((KT / 4) * 128) >> 4;
  return (uint64_t)((addr >> 4) & 0x3FFF) | (lbo << 16) | (sbo << 32) | (1ull << 46);
}

// Instruction descriptor: D f32, A/B tf32, both K-major, N >> 3, M >> 4.
__device__ __forceinline__ uint32_t instr_desc(int n) {
  return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(TM >> 4) << 24);
}

__device__ __forceinline__ void mma_tf32(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t idesc, int acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}\n" ::"r"(tmem_d),
      "l"(da), "l"(db), "r"(idesc), "r"(acc), "r"(0u), "r"(0u), "r"(0u), "r"(0u));
}

__device__ __forceinline__ void mma_commit(uint32_t mbar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar)
               : "memory");
}

__device__ __forceinline__ void mbar_init(uint32_t mbar, int count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(mbar), "r"(count) : "memory");
}

// Bounded wait for the given phase parity; returns false on expiry.
__device__ __forceinline__ bool mbar_wait(uint32_t mbar, uint32_t parity) {
  for (long long it = 0; it < kSpinLimit; ++it) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(done)
        : "r"(mbar), "r"(parity)
        : "memory");
    if (done) return true;
  }
  return false;
}

__device__ __forceinline__ float tf32_hi(float v) { return __uint_as_float(__float_as_uint(v) & 0xFFFFE000u); }

// Shared memory: per stage X_hi, X_lo [128 x 32] and Bt_hi, Bt_lo [npmax x 32],
// then the stage mbarriers and the tensor-memory base address.
struct TcShared {
  float* a_hi[NSTAGE];
  float* a_lo[NSTAGE];
  float* b_hi[NSTAGE];
  float* b_lo[NSTAGE];
  unsigned long long* mbar;
  uint32_t* tmem_base_p;
};

__device__ __forceinline__ TcShared tc_shared(unsigned char* base, int npmax) {
  TcShared sm;
  size_t off = 0;
  for (int s = 0; s < NSTAGE; ++s) {
    sm.a_hi[s] = reinterpret_cast<float*>(base + off); off += (size_t)TM * KT * 4;
    sm.a_lo[s] = reinterpret_cast<float*>(base + off); off += (size_t)TM * KT * 4;
    sm.b_hi[s] = reinterpret_cast<float*>(base + off); off += (size_t)npmax * KT * 4;
    sm.b_lo[s] = reinterpret_cast<float*>(base + off); off += (size_t)npmax * KT * 4;
  }
  sm.mbar = reinterpret_cast<unsigned long long*>(base + off); off += NSTAGE * 8;
  sm.tmem_base_p = reinterpret_cast<uint32_t*>(base + off);
  return sm;
}

size_t tc_smem_bytes(int npmax) {
  return (size_t)NSTAGE * (2 * TM * KT * 4 + 2 * (size_t)npmax * KT * 4) + NSTAGE * 8 + 16;
}

__global__ void __launch_bounds__(128, 1) tc_gemm_kernel(const __grid_constant__ GemmBatch<float> gb, int npmax,
                                                         int* err) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  const TcShared sm = tc_shared(smem_raw, npmax);
  const GemmProb<float>& p = gb.prob[blockIdx.y];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int M = p.M, N = p.N, D = p.D;
  const int tm = blockIdx.x * TM;
  if (tm >= M) return;
  const int NP = (N + 15) / 16 * 16;          // MMA N (multiple of 16, <= 256)
  int ncols = 32;
  while (ncols < NP) ncols <<= 1;             // tensor-memory columns (power of two >= 32)

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(sm.tmem_base_p)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid == 0) {
    for (int s = 0; s < NSTAGE; ++s) mbar_init(smem_u32(sm.mbar + s), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *sm.tmem_base_p;
  const uint32_t idesc = instr_desc(NP);

  bool ok = true;
  uint32_t phase[NSTAGE] = {0u, 0u};
  int pending[NSTAGE] = {0, 0};
  const int nkt = (D + KT - 1) / KT;
  for (int kt = 0; kt < nkt; ++kt) {
    const int s = kt % NSTAGE;
    if (pending[s]) {                           // the MMAs that read this stage are done
      bool w = true;
      if (tid == 0) w = mbar_wait(smem_u32(sm.mbar + s), phase[s]);
      phase[s] ^= 1u;
      pending[s] = 0;
      ok = __syncthreads_and(w) != 0;           // block-uniform outcome
      if (!ok) break;
    }
    const int k0 = kt * KT;
    // X tile: 128 rows x 32 k; 8 threads per row read 16 bytes each (coalesced)
    for (int t = tid; t < TM * (KT / 4); t += 128) {
      const int r = t >> 3, c = t & 7;
      const int gr = tm + r, gk = k0 + c * 4;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (gr < M) {
        const float* src = p.X + (size_t)gr * D + gk;
        if (gk + 3 < D && ((reinterpret_cast<uintptr_t>(src) & 15u) == 0)) {
          v = __ldg(reinterpret_cast<const float4*>(src));
        } else {
          v.x = gk < D ? src[0] : 0.f;
          v.y = gk + 1 < D ? src[1] : 0.f;
          v.z = gk + 2 < D ? src[2] : 0.f;
          v.w = gk + 3 < D ? src[3] : 0.f;
        }
      }
      const float4 hi = make_float4(tf32_hi(v.x), tf32_hi(v.y), tf32_hi(v.z), tf32_hi(v.w));
      const float4 lo = make_float4(v.x - hi.x, v.y - hi.y, v.z - hi.z, v.w - hi.w);
      const uint32_t off = tile_off(r, c);
      *reinterpret_cast<float4*>(reinterpret_cast<unsigned char*>(sm.a_hi[s]) + off) = hi;
      *reinterpret_cast<float4*>(reinterpret_cast<unsigned char*>(sm.a_lo[s]) + off) = lo;
    }
    // B tile (Bt rows = output columns): NP rows x 32 k
    for (int t = tid; t < NP * (KT / 4); t += 128) {
      const int r = t >> 3, c = t & 7;
      const int gk = k0 + c * 4;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (r < N) {
        const float* src = p.B + (size_t)r * D + gk;
        if (gk + 3 < D && ((reinterpret_cast<uintptr_t>(src) & 15u) == 0)) {
          v = __ldg(reinterpret_cast<const float4*>(src));
        } else {
          v.x = gk < D ? src[0] : 0.f;
          v.y = gk + 1 < D ? src[1] : 0.f;
          v.z = gk + 2 < D ? src[2] : 0.f;
          v.w = gk + 3 < D ? src[3] : 0.f;
        }
      }
      const float4 hi = make_float4(tf32_hi(v.x), tf32_hi(v.y), tf32_hi(v.z), tf32_hi(v.w));
      const float4 lo = make_float4(v.x - hi.x, v.y - hi.y, v.z - hi.z, v.w - hi.w);
      const uint32_t off = tile_off(r, c);
      *reinterpret_cast<float4*>(reinterpret_cast<unsigned char*>(sm.b_hi[s]) + off) = hi;
      *reinterpret_cast<float4*>(reinterpret_cast<unsigned char*>(sm.b_lo[s]) + off) = lo;
    }
    // make the generic-proxy shared stores visible to the tensor core
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncthreads();
    if (tid == 0) {
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const uint32_t ahi = smem_u32(sm.a_hi[s]), alo = smem_u32(sm.a_lo[s]);
      const uint32_t bhi = smem_u32(sm.b_hi[s]), blo = smem_u32(sm.b_lo[s]);
#pragma unroll
      for (int ks = 0; ks < KT / 8; ++ks) {
        const uint32_t o = ks * 2 * 128;   // two 16-byte K chunks per K-8 step
        const int acc = (kt > 0 || ks > 0) ? 1 : 0;
        mma_tf32(tmem, smem_desc(ahi + o), smem_desc(bhi + o), idesc, acc);
        mma_tf32(tmem, smem_desc(ahi + o), smem_desc(blo + o), idesc, 1);
        mma_tf32(tmem, smem_desc(alo + o), smem_desc(bhi + o), idesc, 1);
      }
      mma_commit(smem_u32(sm.mbar + s));
    }
    pending[s] = 1;
  }
  // drain: wait for every stage that still has MMAs in flight (also after an
  // expired wait, so that no MMA is in flight when the tensor memory is freed)
  bool w = true;
  if (tid == 0) {
    for (int s = 0; s < NSTAGE; ++s) {
      if (pending[s]) {
        w = mbar_wait(smem_u32(sm.mbar + s), phase[s]) && w;
        phase[s] ^= 1u;
      }
    }
  }
  ok = (__syncthreads_and(w) != 0) && ok;
  if (!ok && tid == 0) atomicOr(err, kErrTimeout);
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  if (ok && nkt > 0) {
    // epilogue: warp w reads lanes 32w..32w+31; 32 columns per load
    const int row = tm + warp * 32 + lane;
    for (int c0 = 0; c0 < NP; c0 += 32) {
      uint32_t v[32];
      const uint32_t taddr = tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)c0;
      asm volatile(
          "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
          "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
          : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
            "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
            "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
            "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
          : "r"(taddr));
      asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
      if (row < M) {
        const int rb = row / p.c.dcomp, cc = row - rb * p.c.dcomp;
        float* dst = p.C + (size_t)(p.c.r0 + rb) * p.c.ld_outer + p.c.off + (size_t)cc * p.c.n;
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (c0 + j < N) dst[c0 + j] = __uint_as_float(v[j]);
      }
    }
  } else if (nkt == 0) {
    const int row = tm + warp * 32 + lane;
    if (row < M) {
      const int rb = row / p.c.dcomp, cc = row - rb * p.c.dcomp;
      float* dst = p.C + (size_t)(p.c.r0 + rb) * p.c.ld_outer + p.c.off + (size_t)cc * p.c.n;
      for (int j = 0; j < N; ++j) dst[j] = 0.f;
    }
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 0) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(ncols) : "memory");
  }
}

}  // namespace

// C = X Bt^T for every problem of the batch (op 0 of gemm.cu on tensor cores);
// every problem must have 1 <= N <= 256.
cudaError_t launch_gemm_tc(const GemmBatch<float>& gb, int n_prob, int max_m, int* err, cudaStream_t s) {
  if (n_prob == 0 || max_m == 0) return cudaSuccess;
  int npmax = 16;
  for (int k = 0; k < n_prob; ++k) {
    if (gb.prob[k].N < 1 || gb.prob[k].N > 256) return cudaErrorInvalidValue;
    npmax = max(npmax, (gb.prob[k].N + 15) / 16 * 16);
  }
  const size_t smem = tc_smem_bytes(npmax);
  cudaError_t e = cudaFuncSetAttribute(tc_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((max_m + TM - 1) / TM, n_prob);
  tc_gemm_kernel<<<grid, 128, smem, s>>>(gb, npmax, err);
  return cudaGetLastError();
}

}  // namespace tpc
