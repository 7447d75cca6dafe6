/*
 * tpconv.h -- C ABI of the edge-conditioned Clebsch-Gordan tensor-product
 * convolution on NVIDIA B200 (sm_100a).
 *
 * The operator (Sobek: Streaming Equivariant Tensor Product Convolutions, §2.4):
 *
 *   m_i = sum_{j in N(i)} sum_{pi} sum_a W_{ij,pi,a} T_{pi,a}(x_j, Y_ij),
 *   W_{ij,pi,a} = sum_q phi_{ij,q} A_{q,pi,a},
 *
 * for every receiver i over its incoming edges j -> i, where T_{pi,a} is the
 * Clebsch-Gordan product of path pi = (l1, l2) -> l3 (LunaTP: Enabling Efficient
 * and Scalable Tensor Product for Equivariant MLIPs, §2.1 Eq. 1) of the sender
 * features x_j with the spherical harmonics Y_ij of the edge, and a is the
 * channel index: a = u (channelwise "uvu", output channel = input channel) or
 * a = (u, w) (fully connected "uvw", Sobek §2.3). It is evaluated in the
 * streamed, receiver-owned schedule of Sobek §3-§4: no per-edge weight,
 * message or adjoint tensor is ever stored.
 *
 * Conventions common to all entry points
 * --------------------------------------
 * Layouts (Sobek §4.5 "ir_mul": channels contiguous inside each irrep block):
 *   x        [N, C_in]   row j = blocks of irreps_in in order, each [2l+1][mul]
 *   out      [N, C_out]  the same for irreps_out
 *   Y        [E, (L+1)^2] per edge, blocks l = 0..L (L = sh_lmax), m = -l..l;
 *                        the real basis has l = 1 ordered (y, z, x)
 *   phi      [E, K]      radial basis values per edge
 *   A        [K, N_w]    path pi owns columns [w_off, w_off + n_w); uvu column u,
 *                        uvw column u * mul_out + w (row-major [K, P, C_in, C_out]
 *                        when all multiplicities agree)
 * Y and phi are in receiver-CSR edge order: the caller permutes them with the
 * perm array of tp_csr_build. All arrays are row-major and contiguous. Floating
 * arrays use the plan's dtype; index arrays are int32 (N, E < 2^31).
 * Every device pointer must be 16-byte aligned (cudaMalloc and PyTorch
 * allocations are).
 *
 * Ownership: the caller owns every buffer, device or host, including the
 * workspace. A plan owns only host memory. No entry point allocates device
 * memory or synchronises unless stated.
 *
 * Streams: `stream` is a cudaStream_t passed as void* (NULL = legacy default
 * stream). Device work is enqueued asynchronously on it.
 *
 * Errors: every entry point returns TP_OK (0) or a negative tp_status.
 * Argument errors are detected on the host before any work is enqueued. Bad
 * data found by a kernel (a sender index outside [0, N), a row pointer that is
 * not monotone) sets a per-device error word instead of trapping; the offending
 * edge is skipped and the call's outputs are then unspecified.
 * tp_get_device_error reads and clears that word. tp_last_error_message gives
 * a description of the last host-side failure of the calling thread.
 */
#ifndef TPCONV_H
#define TPCONV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct tp_plan_s* tp_plan_t;

enum tp_mode { TP_UVU = 0, TP_UVW = 1, TP_UVU_PATHS = 2 };
enum tp_dtype { TP_F32 = 0, TP_F64 = 1 };
enum tp_schedule { TP_SCHED_STREAMED = 0, TP_SCHED_RECEIVER_STATE = 1 };
enum tp_status {
  TP_OK = 0,
  TP_EINVAL = -1,         /* bad argument (null pointer, size, alignment, string) */
  TP_EUNSUPPORTED = -2,   /* valid contract outside what the kernels are built for */
  TP_ECUDA = -3,          /* a CUDA runtime call failed */
  TP_EWORKSPACE = -4,     /* workspace smaller than tp_conv_workspace_size */
  TP_EDEVICE_INDEX = -5,  /* a kernel met an index outside its range */
  TP_EDEVICE_CSR = -6,    /* a kernel met a non-monotone or out-of-range row pointer */
  TP_EDEVICE_TIMEOUT = -7 /* a kernel's bounded wait on its tensor-core work expired */
};

typedef struct {
  int32_t c_in, c_out;    /* row widths of x and out */
  int32_t dim_y;          /* (sh_lmax + 1)^2 */
  int32_t n_radial;       /* K */
  int32_t n_paths;
  int32_t mode, dtype, sh_lmax;
  int32_t lmax;           /* largest degree among inputs, outputs and Y */
  int32_t pad;
  int64_t n_w;            /* columns of A */
} tp_plan_info_t;

typedef struct {
  int32_t l1, p1, l2, p2, l3, p3;   /* degrees and parities (+1 even, -1 odd) */
  int32_t block_in, block_out;      /* indices into irreps_in / irreps_out */
  int32_t mul_in, mul_out;
  int32_t x_off, out_off;           /* block offsets in an x / out row */
  int64_t w_off, n_w;               /* columns of A owned by the path */
  int32_t nnz;                      /* non-zero real CG coefficients */
  int32_t pad;
} tp_path_info_t;

/* Plan one convolution contract (Sobek §4.5: validate the contract, enumerate
 * the valid paths and their sparse CG terms; §2.2 for the selection rule).
 * irreps_in / irreps_out: strings such as "64x0e+64x1o+64x2e". sh_lmax: degree
 * of Y. n_radial: K. mode: TP_UVU, TP_UVW or TP_UVU_PATHS. dtype: TP_F32 or
 * TP_F64. Paths are enumerated for each input block in order, l2 = 0..sh_lmax
 * ascending (Y of parity (-1)^l2), l3 = |l1-l2|..l1+l2 ascending, one path per
 * output block of that degree and parity; output blocks sum their paths.
 * TP_UVU_PATHS is the channelwise product with one output block per path
 * (LunaTP Appendix A.1: the uvu paths' outputs are concatenated): irreps_out
 * only says which (l, p) may be produced (its multiplicities are ignored); the
 * output row holds, in path order, one block of the path's input multiplicity
 * and degree l3 per path (tp_conv_plan_info gives C_out, tp_conv_plan_path the
 * blocks' offsets). Degrees up to 4 are compiled for every mode and dtype, up
 * to 6 for channelwise fp32 plans with K <= 8.
 * Host only (no CUDA call). On success *plan receives a new plan that the
 * caller releases with tp_conv_plan_destroy. Errors: TP_EINVAL (malformed
 * string, bad enum, NULL, no path reaches the outputs), TP_EUNSUPPORTED (uvu
 * with unequal multiplicity on a path, degree above the limit, K above 16,
 * more than 192 paths or 224 channel tiles). */
int tp_conv_plan(const char* irreps_in, int sh_lmax, const char* irreps_out, int n_radial,
                 int mode, int dtype, tp_plan_t* plan);

/* tp_conv_plan with the spherical-harmonic irreps given explicitly, as
 * "1x0e+1x1o+1x2e" (degrees 0..L in order, multiplicity 1): the parity of
 * each degree of Y is taken from the string instead of (-1)^l. Parity only
 * selects the paths (Sobek §2.2: p_out = p_in p_sh); the arithmetic of Y is
 * unchanged. Used by contracts whose edge irreps are all even (LunaTP
 * Appendix A.1, Table 1, case C1). Errors as tp_conv_plan, plus TP_EINVAL for a
 * malformed SH string. */
int tp_conv_plan_sh(const char* irreps_in, const char* irreps_sh, const char* irreps_out, int n_radial,
                    int mode, int dtype, tp_plan_t* plan);

/* Release a plan (NULL is accepted). */
int tp_conv_plan_destroy(tp_plan_t plan);

/* Sizes of a plan. Host only. */
int tp_conv_plan_info(tp_plan_t plan, tp_plan_info_t* info);

/* Description of path `index` (0 <= index < n_paths), in enumeration order. */
int tp_conv_plan_path(tp_plan_t plan, int index, tp_path_info_t* info);

/* The real-basis CG coefficients of path `index` (LunaTP §2.1 Eq. 1; Sobek
 * §4.2 Eq. 32): non-zero entries (m1, m2, m3, c), indices 0..2l, lexicographic.
 * Computed on the host by Racah's formula (Condon-Shortley phases) mapped to
 * the real basis, orthonormal in (m1, m2), the first non-zero entry positive.
 * Writes at most `capacity` entries into the caller's host arrays and returns
 * the number of non-zeros (>= 0), or a negative tp_status. */
int tp_conv_plan_cg(tp_plan_t plan, int index, int32_t* m1, int32_t* m2, int32_t* m3, double* c,
                    int capacity);

/* Bytes of one receiver-state chunk of a fully connected (uvw) plan. The uvw
 * path reduces each receiver's edges into a state S_i with no output-channel
 * axis and mixes it once (Sobek §4.2, Eqs. 33-35); receivers are processed in
 * ranges whose states fit this budget, so the workspace is bounded by it and
 * not by the edge count (Sobek App. B.2, fixed scratch budget). Default 1 GiB.
 * A smaller budget gives more, smaller receiver (and source) chunks: less
 * workspace, more launches (tp_conv_launch_count reports them). Host only.
 * Errors: TP_EINVAL if `bytes` is below the state of one node
 * (the message gives that size). Channelwise (uvu) plans keep no state
 * chunks and accept any value without effect. */
int tp_conv_plan_set_state_budget(tp_plan_t plan, size_t bytes);

/* Evaluation order of the channelwise forward. TP_SCHED_STREAMED (default):
 * Sobek §3.1, the scalar w = phi A formed per edge, path and channel and
 * consumed at once. TP_SCHED_RECEIVER_STATE: Sobek §4.2 (Eqs. 32-35) applied to
 * uvu, the receiver state S_i = sum_e phi_e (outer) C(x_j, Y_e) per path and
 * channel kept in registers over the receiver's edges and mixed with A once per
 * receiver; it costs nnz + K (2 l3 + 1) FMAs per edge and channel against
 * K + nnz + (2 l3 + 1) and exists to compare the two orders. Both give the
 * same result up to rounding order. Fully connected plans always use the
 * receiver state (TP_SCHED_STREAMED is TP_EUNSUPPORTED for them). Errors:
 * TP_EINVAL (unknown schedule), TP_EUNSUPPORTED (receiver state with K > 8 or
 * degrees above 4). Host only. */
int tp_conv_plan_set_schedule(tp_plan_t plan, int schedule);

/* Algorithmic work of one pass (0 forward, 1 backward, 2 double backward) on
 * N nodes and E edges: flops (FMA = 2) of the streamed schedule and compulsory
 * HBM bytes (each input read once, each output written once). Host only. */
int tp_conv_work_model(tp_plan_t plan, int64_t n_nodes, int64_t n_edges, int pass, double* flops,
                       double* bytes);

/* Workspace bytes that tp_conv_forward (pass 0), tp_conv_backward (pass 1) or
 * tp_conv_double_backward (pass 2) need for n_nodes receivers. It does not depend on the edge count (Sobek
 * §3.4, Table 2: tensor-product workspace is bounded, not edge-sized). */
int tp_conv_workspace_size(tp_plan_t plan, int64_t n_nodes, int pass, size_t* bytes);

/* Number of kernels that one tp_conv_forward (pass 0), tp_conv_backward
 * (pass 1) or tp_conv_double_backward (pass 2) call enqueues for n_nodes receivers (memsets not counted). The
 * fully connected path works on receiver chunks of a fixed state budget, so
 * its count grows with n_nodes. Host only. */
int tp_conv_launch_count(tp_plan_t plan, int64_t n_nodes, int pass, int* kernels);

/* Workspace bytes of tp_csr_build / tp_csr_transpose for n_nodes rows. */
int tp_csr_workspace_size(int64_t n_nodes, size_t* bytes);

/* Receiver CSR of a COO edge list (LunaTP §4.1; Sobek §4.5, which prepares a
 * stable CSR before the kernels run). Inputs (device): src[E], dst[E] with
 * edge e = src[e] -> dst[e].
 * Outputs (device): rowptr[N+1]; senders[E] = src of the edge at each CSR
 * position; perm[E] = COO index of the edge at each CSR position. Edges of one
 * receiver keep their input order. ws: device workspace of
 * tp_csr_workspace_size bytes. An index outside [0, N) sets TP_EDEVICE_INDEX
 * in the device error word and drops that edge. */
int tp_csr_build(int64_t n_nodes, int64_t n_edges, const int32_t* src, const int32_t* dst,
                 int32_t* rowptr, int32_t* senders, int32_t* perm, void* ws, size_t ws_bytes,
                 void* stream);

/* Source view of a receiver CSR, for the node-feature gradient (LunaTP §4.4;
 * Sobek §4.3, where x_bar is owned by a second traversal grouped by sender).
 * Inputs (device): rowptr[N+1], senders[E] from tp_csr_build. Outputs
 * (device): colptr[N+1]; srcedge[E] = CSR positions grouped by sender, in
 * ascending order within a sender; srcrecv[E] = receiver of each of them. */
int tp_csr_transpose(int64_t n_nodes, int64_t n_edges, const int32_t* rowptr,
                     const int32_t* senders, int32_t* colptr, int32_t* srcedge, int32_t* srcrecv,
                     void* ws, size_t ws_bytes, void* stream);

/* Forward (Sobek §2.4 Eqs. 11-12, streamed as in §3.1; uvw as the
 * receiver-factorised S then m = S A of §4.2 Eqs. 32-35). Inputs (device): x,
 * Y, phi, A, rowptr, senders as described above. Output (device): out[N, C_out],
 * overwritten; receivers without incoming edges get zeros. ws: device
 * workspace of at least tp_conv_workspace_size(plan, N, 0) bytes (may be NULL
 * when that is 0). */
int tp_conv_forward(tp_plan_t plan, const void* x, const void* Y, const void* phi, const void* A,
                    const int32_t* rowptr, const int32_t* senders, int64_t n_nodes,
                    int64_t n_edges, void* out, void* ws, size_t ws_bytes, void* stream);

/* First backward (Sobek §3.2 and §4.3; LunaTP Appendix F, Algorithm 2). Given
 * grad_out = dL/dout [N, C_out] (device), writes (device, overwritten):
 * grad_x [N, C_in], grad_Y [E, (L+1)^2] and grad_phi [E, K] in CSR edge order,
 * grad_A [K, N_w]. Needs the receiver CSR (rowptr, senders) and its source view
 * (colptr, srcedge, srcrecv). Every reduction has one owner and a fixed order,
 * so results are bitwise reproducible run to run. ws: device workspace of at
 * least tp_conv_workspace_size(plan, N, 1) bytes. */
int tp_conv_backward(tp_plan_t plan, const void* x, const void* Y, const void* phi, const void* A,
                     const int32_t* rowptr, const int32_t* senders, const int32_t* colptr,
                     const int32_t* srcedge, const int32_t* srcrecv, const void* grad_out,
                     int64_t n_nodes, int64_t n_edges, void* grad_x, void* grad_Y, void* grad_phi,
                     void* grad_A, void* ws, size_t ws_bytes, void* stream);

/* Second-order program (Sobek §3.3 and §4.4; LunaTP Appendix F, Algorithm 3):
 * the directional derivative, along v = (dx, dY, dphi, dA), of the forward
 * output and of the four first-order adjoints, with grad_out held fixed:
 *   d_out   = J v                 (J: Jacobian of the forward)
 *   dgrad_* = H v                 (H: Hessian of <grad_out, forward>),
 * per edge e = j -> i, path and channel (w = phi A, T = CG(x_j, Y_e)):
 *   w_dot = dphi A + phi dA,  T_dot = CG(dx_j, Y_e) + CG(x_j, dY_e),
 *   d_out_i += w_dot T + w T_dot,  h = <grad_out_i, T>,  h_dot = <grad_out_i, T_dot>,
 *   dgrad_A += dphi h + phi h_dot,  dgrad_phi_e = dA h + A h_dot,
 *   dgrad_x_j += w_dot D_xT^*(Y) grad_out_i + w D_xT^*(dY) grad_out_i,
 *   dgrad_Y_e = w_dot D_YT^*(x) grad_out_i + w D_YT^*(dx) grad_out_i.
 * For a loss L of the first-order outputs, passing v = (dL/dgrad_x, dL/dgrad_Y,
 * dL/dgrad_phi, dL/dgrad_A) gives dL/d(x, Y, phi, A) in dgrad_* and dL/dgrad_out
 * in d_out (the Hessian is symmetric), which is what a framework's double
 * backward asks for. A direction of grad_out itself would add
 * tp_conv_backward applied to it; callers add that separately.
 * Inputs (device): x, Y, phi, A, grad_out and the CSR views as for
 * tp_conv_backward; directions dx [N, C_in], dY [E, dimY], dphi [E, K] (CSR
 * edge order), dA [K, N_w]. Outputs (device, overwritten): d_out [N, C_out],
 * dgrad_x [N, C_in], dgrad_Y [E, dimY], dgrad_phi [E, K], dgrad_A [K, N_w].
 * ws: at least tp_conv_workspace_size(plan, N, 2) bytes. Results are bitwise
 * reproducible run to run (fixed ownership and order). Fully connected (uvw)
 * plans run the receiver program of Sobek §4.4 through the first-order
 * kernels: the directional state dS = S(dx, Y, phi) + S(x, dY, phi) +
 * S(x, Y, dphi) gives d_out = dS A + S dA and dgrad_A = dS^T grad_out; the
 * edge pass runs on S_bar = grad_out A^T and dS_bar = grad_out dA^T; the
 * source states give dgrad_x = (S'(dY, phi) + S'(Y, dphi)) A' + S' dA'. */
int tp_conv_double_backward(tp_plan_t plan, const void* x, const void* Y, const void* phi, const void* A,
                            const int32_t* rowptr, const int32_t* senders, const int32_t* colptr,
                            const int32_t* srcedge, const int32_t* srcrecv, const void* grad_out,
                            const void* dx, const void* dY, const void* dphi, const void* dA, int64_t n_nodes,
                            int64_t n_edges, void* d_out, void* dgrad_x, void* dgrad_Y, void* dgrad_phi,
                            void* dgrad_A, void* ws, size_t ws_bytes, void* stream);

/* tp_conv_backward for callers that cannot allocate device memory (no
 * counterpart in the pages: it is a service of this library). Plugins run from
 * another engine's execution step, code running while a stream capture is
 * open, or processes held to a fixed memory reservation may be unable to
 * cudaMalloc the workspace tp_conv_backward asks for. This entry point takes
 * the same arguments minus the workspace and allocates nothing: the grad_A
 * partial sums live in a static 16 MiB array of device memory inside the
 * library, which every GPU that loads the library keeps reserved until the
 * process exits. Limits: channelwise (uvu) plans only (else TP_EUNSUPPORTED);
 * one slot of partials takes K * N_w * scalar-size bytes and must fit in the
 * 16 MiB (else TP_EWORKSPACE with the sizes in tp_last_error_message); with
 * fewer slots than tp_conv_backward uses, results differ from it only by the
 * order of the grad_A additions. The first call on each device looks up the
 * array's device address (cudaGetSymbolAddress) with that device current: make
 * that first call before any stream capture. Every call on a device shares the
 * one array and leaves its contents behind (each call clears what it needs
 * first); calls that may overlap on the GPU -- different streams, or threads
 * without ordering -- race on it and give wrong results. The looked-up address
 * is kept for the life of the process (as is the error word's): do not use the
 * library on a device after cudaDeviceReset. The TP_EWORKSPACE limit is a
 * guard: within the planner's limits (at most 96 channel tiles and 192 paths)
 * one slot of a channelwise plan stays below about 2 MiB. */
int tp_conv_backward_noalloc(tp_plan_t plan, const void* x, const void* Y, const void* phi,
                             const void* A, const int32_t* rowptr, const int32_t* senders,
                             const int32_t* colptr, const int32_t* srcedge, const int32_t* srcrecv,
                             const void* grad_out, int64_t n_nodes, int64_t n_edges, void* grad_x,
                             void* grad_Y, void* grad_phi, void* grad_A, void* stream);

/* Synchronise `stream`, then read and clear the device error word of the
 * current device. Returns TP_OK, TP_EDEVICE_INDEX, TP_EDEVICE_CSR or
 * TP_EDEVICE_TIMEOUT or TP_ECUDA. */
int tp_get_device_error(void* stream);

/* Static description of a status code. */
const char* tp_status_string(int status);

/* Description of the calling thread's last host-side failure ("" if none). */
const char* tp_last_error_message(void);

#ifdef __cplusplus
}
#endif

#endif /* TPCONV_H */
