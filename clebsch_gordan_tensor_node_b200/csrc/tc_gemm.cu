// Tensor-core (tcgen05) channel-mixing GEMM of the fully connected path, fp32.
//
// Sobek §4.2 (Eqs. 34-35): m_g = S_g A_g per output block, rows = (receiver,
// output component), contracted dimension = (path, radial index, input
// channel), columns = output channels. This kernel computes C = X Bt^T with
// X [M, D] row-major (the receiver state, fp32) and Bt [N, D] row-major (A's
// block, transposed and pre-split), both K-major, and writes C rows straight
// into the ir_mul output block (row-blocked addressing).
//
// FP32-exact on TF32 tensor cores by the three-term split (Ootomo & Yokota
// 2022): x = x_hi + x_lo with x_hi exactly representable in TF32 (low 13
// mantissa bits cleared) and x_lo = x - x_hi; C = X_hi B_hi + X_hi B_lo +
// X_lo B_hi with fp32 accumulation (the dropped X_lo B_lo term is ~2^-22
// relative). Bt is split once by the packing kernel; X is split in shared memory.
//
// One CTA (4 warps) owns 128 rows and all N (<= 256, padded to 16) columns;
// the fp32 accumulator lives in tensor memory. K runs through a 2- to 4-stage
// shared-memory pipeline in 32-wide tiles:
//   warp 0 (one lane): TMA producer -- cp.async.bulk.tensor loads of the raw X
//            tile [128 x 32] and the Bt_hi / Bt_lo tiles [N x 32], 128-byte
//            swizzle, out-of-bounds rows/columns zero-filled, completion on the
//            stage's "full" mbarrier (expect_tx);
//   warps 2-3: split the raw X tile in place (hi) and into a second buffer
//            (lo) at the same swizzled offsets, then arrive on "split";
//   warp 1 (one lane): issues tcgen05.mma (kind::tf32, M 128, N, K 8; SW128
//            K-major descriptors, K steps advance the start address by 32 B)
//            and commits to the stage's "empty" mbarrier, and finally to
//            "done";
//   all warps: tensor memory -> registers (tcgen05.ld) -> global.
// Every wait is bounded: on expiry the kernel records kErrTimeout, waits
// (bounded) for its own copies and MMAs, frees its tensor memory and returns.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"

namespace tpc {
namespace {

constexpr int TM = 128;        // rows per CTA (tensor-memory lanes)
constexpr int KT = 32;         // K per stage (one 128-byte swizzle row of fp32)
constexpr int kMaxStages = 4;  // pipeline stages for output blocks of up to 64 channels
constexpr long long kSpinLimit = 1ll << 22;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// sm100 shared-memory descriptor, K-major, 128-byte swizzle: start >> 4,
// leading byte offset 16 B (unused by this layout), stride byte offset 1024 B
// (8 rows of 128 B), version 1, layout type SWIZZLE_128B (2).
__device__ __forceinline__ uint64_t desc_sw128(uint32_t addr) {
  return (uint64_t)((addr >> 4) & 0x3FFF) | (1ull << 16) | ((uint64_t)(1024 >> 4) << 32) | (1ull << 46) |
         (2ull << 61);
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

__device__ __forceinline__ void mbar_arrive(uint32_t mbar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(mbar) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t mbar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(mbar), "r"(bytes) : "memory");
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

__device__ __forceinline__ void tma_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t mbar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
      "[%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(mbar)
      : "memory");
}

__device__ __forceinline__ float tf32_hi(float v) { return __uint_as_float(__float_as_uint(v) & 0xFFFFE000u); }

struct Stage {
  float* xr;  // raw X tile, split in place into X_hi
  float* xl;  // X_lo
  float* bh;  // Bt_hi tile
  float* bl;  // Bt_lo tile
};

// NS: pipeline stages; wider output blocks (npmax up to 256) take fewer stages so
// that the ring stays within shared memory.
template <int NS>
__global__ void __launch_bounds__(128, 1) tc_gemm_kernel(const __grid_constant__ TcBatch tb, int npmax, int* err) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  __shared__ int fail_flag;
  const TcProb& p = tb.prob[blockIdx.y];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int M = p.M, N = p.N, D = p.D;
  const int tm = blockIdx.x * TM;
  if (tm >= M) return;
  // shared memory: NS stages of {X raw/hi, X lo [128 x 32], Bt hi, Bt lo [npmax x 32]},
  // each buffer 1024-byte aligned (128-byte swizzle atoms), then the barriers
  unsigned char* base =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Stage st[NS];
  size_t off = 0;
  for (int s = 0; s < NS; ++s) {
    st[s].xr = reinterpret_cast<float*>(base + off); off += (size_t)TM * KT * 4;
    st[s].xl = reinterpret_cast<float*>(base + off); off += (size_t)TM * KT * 4;
    st[s].bh = reinterpret_cast<float*>(base + off); off += (size_t)npmax * KT * 4;
    st[s].bl = reinterpret_cast<float*>(base + off); off += (size_t)npmax * KT * 4;
  }
  unsigned long long* bar = reinterpret_cast<unsigned long long*>(base + off);  // full, split, empty, done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 3 * NS + 1);
  const int NP = (N + 15) / 16 * 16;
  int ncols = 32;
  while (ncols < NP) ncols <<= 1;

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid == 0) {
    fail_flag = 0;
    for (int s = 0; s < NS; ++s) {
      mbar_init(smem_u32(bar + s), 1);           // full: producer's expect_tx
      mbar_init(smem_u32(bar + NS + s), 64);     // split: 64 splitter threads
      mbar_init(smem_u32(bar + 2 * NS + s), 1);  // empty: MMA commit
    }
    mbar_init(smem_u32(bar + 3 * NS), 1);        // done
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tmem_slot;
  const int nkt = (D + KT - 1) / KT;
  const uint32_t tx_bytes = (uint32_t)(TM * KT * 4 + 2 * NP * KT * 4);

  if (warp == 0) {
    if (lane == 0) {  // ---- TMA producer
      for (int kt = 0; kt < nkt; ++kt) {
        const int s = kt % NS;
        if (kt >= NS && !mbar_wait(smem_u32(bar + 2 * NS + s), ((kt / NS) - 1) & 1)) {
          atomicOr(&fail_flag, 1);
          break;
        }
        const uint32_t fb = smem_u32(bar + s);
        mbar_expect_tx(fb, tx_bytes);
        tma_2d(smem_u32(st[s].xr), &p.tx, kt * KT, tm, fb);
        tma_2d(smem_u32(st[s].bh), &p.tbh, kt * KT, 0, fb);
        tma_2d(smem_u32(st[s].bl), &p.tbl, kt * KT, 0, fb);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {  // ---- MMA issuer
      const uint32_t idesc = instr_desc(NP);
      bool good = true;
      for (int kt = 0; kt < nkt; ++kt) {
        const int s = kt % NS;
        if (!mbar_wait(smem_u32(bar + NS + s), (kt / NS) & 1)) {
          atomicOr(&fail_flag, 1);
          good = false;
          break;
        }
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const uint32_t xh = smem_u32(st[s].xr), xl = smem_u32(st[s].xl);
        const uint32_t bh = smem_u32(st[s].bh), bl = smem_u32(st[s].bl);
#pragma unroll
        for (int ks = 0; ks < KT / 8; ++ks) {
          const uint32_t o = ks * 32;  // K-8 step = 32 bytes inside the swizzled row
          mma_tf32(tmem, desc_sw128(xh + o), desc_sw128(bh + o), idesc, (kt | ks) ? 1 : 0);
          mma_tf32(tmem, desc_sw128(xh + o), desc_sw128(bl + o), idesc, 1);
          mma_tf32(tmem, desc_sw128(xl + o), desc_sw128(bh + o), idesc, 1);
        }
        mma_commit(smem_u32(bar + 2 * NS + s));
      }
      if (good) mma_commit(smem_u32(bar + 3 * NS));
    }
    __syncwarp();
  } else {  // ---- splitters (warps 2-3, 64 threads)
    const int t = tid - 64;
    for (int kt = 0; kt < nkt; ++kt) {
      const int s = kt % NS;
      if (!mbar_wait(smem_u32(bar + s), (kt / NS) & 1)) {
        atomicOr(&fail_flag, 1);
        break;
      }
      float4* xr = reinterpret_cast<float4*>(st[s].xr);
      float4* xl = reinterpret_cast<float4*>(st[s].xl);
      for (int c = t; c < TM * KT / 4; c += 64) {
        const float4 v = xr[c];
        const float4 h = make_float4(tf32_hi(v.x), tf32_hi(v.y), tf32_hi(v.z), tf32_hi(v.w));
        xr[c] = h;
        xl[c] = make_float4(v.x - h.x, v.y - h.y, v.z - h.z, v.w - h.w);
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_arrive(smem_u32(bar + NS + s));
    }
  }
  __syncthreads();
  bool ok = fail_flag == 0 && nkt > 0;
  {
    bool w = true;
    if (ok && tid == 0) w = mbar_wait(smem_u32(bar + 3 * NS), 0);
    ok = (__syncthreads_and(w) != 0) && ok;
  }
  if (ok) {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
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
        if (p.accumulate) {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (c0 + j < N) dst[c0 + j] += __uint_as_float(v[j]);
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (c0 + j < N) dst[c0 + j] = __uint_as_float(v[j]);
        }
      }
    }
  } else if (nkt == 0) {
    const int row = tm + warp * 32 + lane;
    if (row < M && !p.accumulate) {
      const int rb = row / p.c.dcomp, cc = row - rb * p.c.dcomp;
      float* dst = p.C + (size_t)(p.c.r0 + rb) * p.c.ld_outer + p.c.off + (size_t)cc * p.c.n;
      for (int j = 0; j < N; ++j) dst[j] = 0.f;
    }
  } else if (tid == 0) {
    // an expired wait: record it, then wait (bounded) for the last phase of every
    // stage's copies and MMAs so that nothing is in flight when the CTA exits
    atomicOr(err, kErrTimeout);
    for (int s = 0; s < NS && s < nkt; ++s) {
      const int last = (nkt - 1 - s) / NS;  // index of the last use of stage s
      mbar_wait(smem_u32(bar + s), last & 1);
      mbar_wait(smem_u32(bar + 2 * NS + s), last & 1);
    }
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 0) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(ncols) : "memory");
  }
}

using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                              const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                              CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn encode_fn() {
  static EncodeFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeFn>(f);
  }
  return fn;
}

}  // namespace

bool tc_gemm_available() { return encode_fn() != nullptr; }

// 2-D fp32 tensor map of a row-major [rows, cols] matrix, box [box_rows, 32]
// with 128-byte swizzle; cols * 4 must be a multiple of 16.
bool tc_make_map(CUtensorMap* map, const float* base, long long rows, long long cols, int box_rows) {
  EncodeFn fn = encode_fn();
  if (!fn || rows <= 0 || cols <= 0 || (cols * 4) % 16 != 0 || (reinterpret_cast<uintptr_t>(base) & 15u) != 0)
    return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 4};
  const cuuint32_t box[2] = {(cuuint32_t)KT, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t tc_smem_bytes(int npmax, int ns) {
  return 1024 + (size_t)ns * (2 * TM * KT * 4 + 2 * (size_t)npmax * KT * 4) + (3 * ns + 1) * 8 + 16;
}

template <int NS>
cudaError_t launch_tc_ns(const TcBatch& tb, int n_prob, int max_m, int npmax, int* err, cudaStream_t s) {
  const size_t smem = tc_smem_bytes(npmax, NS);
  static SmemLimit limit;
  if (cudaError_t e = limit.ensure((const void*)tc_gemm_kernel<NS>, smem); e != cudaSuccess) return e;
  dim3 grid((max_m + TM - 1) / TM, n_prob);
  tc_gemm_kernel<NS><<<grid, 128, smem, s>>>(tb, npmax, err);
  return cudaGetLastError();
}

// Output blocks up to 256 channels (padded to 16): the deepest ring that fits
// 227 KiB of shared memory, 4 stages up to 64 channels, 3 up to 128, 2 up to 256.
cudaError_t launch_gemm_tc(const TcBatch& tb, int n_prob, int max_m, int npmax, int* err, cudaStream_t s) {
  if (n_prob == 0 || max_m == 0) return cudaSuccess;
  if (npmax > 256) return cudaErrorInvalidValue;
  const size_t cap = 227 * 1024;
  if (tc_smem_bytes(npmax, kMaxStages) <= cap) return launch_tc_ns<kMaxStages>(tb, n_prob, max_m, npmax, err, s);
  if (tc_smem_bytes(npmax, 3) <= cap) return launch_tc_ns<3>(tb, n_prob, max_m, npmax, err, s);
  return launch_tc_ns<2>(tb, n_prob, max_m, npmax, err, s);
}

}  // namespace tpc
