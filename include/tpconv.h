/*
 * tpconv.h -- C ABI of the streaming Clebsch-Gordan tensor-product convolution
 * (B200 / sm_100a).
 *
 * Operator.  "Sobek: streaming edge-conditioned equivariant tensor-product
 * convolution" (arXiv 2607.18074), abstract: an edge-conditioned tensor-product
 * convolution built from a radial projection, a spherical-harmonic coupling and
 * graph aggregation, with fully connected multiplicity mixing, and its
 * backward and double backward.  Written out (the pages print no formula; this
 * is the reading the library implements):
 *
 *   out[r, i3, w, m3] = sum_{e: recv(e)=r} sum_{paths p -> i3} sum_{u, k}
 *                       b_k(|v_e|) Theta[p][k][u][w] T_e[p, u, m3],
 *   T_e[p, u, m3]     = sum_{m1, m2} C_p[m1, m2, m3] x[send(e), i1, u, m1] Y_{l2 m2}(v_e).
 *
 * C_p is the real Clebsch-Gordan tensor of the path (l1, l2, l3) ("The Price of
 * Freedom", Approach: Clebsch-Gordan tensor product and its selection rules),
 * Y the real spherical harmonics in component normalisation, b the radial basis.
 *
 * Schedule.  The abstract's reassociation: edge-local products are consumed
 * into bounded receiver-side state A[r, k, p, u, m3] = sum_e b_ek T_e[p, u, m3]
 * and a node-level contraction with Theta mixes it; no per-edge weights,
 * messages or adjoints are materialised.  Receiver-side state is bounded by
 * receiver chunking (tpconv_options.workspace_cap), never by the edge count.
 *
 * Conventions shared by every entry point
 *   - All tensors are caller-owned, contiguous, row-major.  Floating point is
 *     fp32; indices are int32 (E must stay below 2^31).
 *   - Device pointers are CUDA device memory of the current device; host
 *     pointers are noted as such.
 *   - Feature layout: blocks in irreps-string order, each block [mul][2l+1]
 *     with m fastest (m = -l..l, real basis, Y_1 ~ (y, z, x)).
 *   - Graph: CSR by receiver: rowptr[N+1] (rowptr[0] = 0, non-decreasing),
 *     col[E] = sender of edge e, edge_vec[E][3] = pos[sender] - pos[receiver],
 *     all in CSR order.  Zero-length edge vectors are undefined.
 *   - Theta layout: one block [R][C_in][C_out] per path, in path order (output
 *     block, then input block, then l2); see tpconv_plan_path.
 *   - Outputs are overwritten, never accumulated.  An output pointer may be NULL
 *     when documented as optional: that output is then not computed.
 *   - Calls are asynchronous on the given stream (a cudaStream_t passed as
 *     void*; NULL = legacy default stream).  Argument errors are reported
 *     synchronously through the return code; kernel faults surface at the
 *     caller's next synchronisation.
 *   - Workspace is caller-provided device memory of at least
 *     tpconv_workspace_size() bytes, 256-byte aligned; the library allocates
 *     nothing on the device.
 *   - A plan is immutable after creation and may be used concurrently from
 *     several streams, each with its own workspace.
 */
#ifndef TPCONV_H
#define TPCONV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* status codes */
/* Device set-up (constant tables, kernel attributes) is done once per CUDA
 * context on the first call that needs it; a context destroyed by
 * cudaDeviceReset is set up again on the next call. */
#define TPCONV_OK 0
#define TPCONV_ERR_INVALID_ARG 1        /* null/negative/misaligned argument   */
#define TPCONV_ERR_BAD_IRREPS 2         /* irreps string does not parse         */
#define TPCONV_ERR_UNSUPPORTED 3        /* l > 3, l_sh_max > 3, R > 16, ...     */
#define TPCONV_ERR_WORKSPACE_TOO_SMALL 4
#define TPCONV_ERR_CUDA 5               /* a CUDA runtime call failed           */
#define TPCONV_ERR_GRAPH_INVALID 6      /* validate mode: bad CSR / indices     */
#define TPCONV_ERR_TIMEOUT 7            /* a bounded device wait expired        */
#define TPCONV_ERR_INTERNAL 8           /* self-check failed (e.g. CG table)    */

/* radial basis kinds */
#define TPCONV_RADIAL_GAUSSIAN 0   /* exp(-((r-mu_k)/D)^2), mu_k = p0 + k D, D = (p1-p0)/(R-1) */
#define TPCONV_RADIAL_BESSEL_COS 1 /* sqrt(2/p0) sin(k pi r/p0)/r * (cos(pi r/p0)+1)/2, k=1..R, 0 beyond p0 */

/* precision of the node-level Theta contractions (tensor cores).  The value 2
 * is not a mode: plan creation rejects it with TPCONV_ERR_UNSUPPORTED.  A
 * half-precision operand mode would save nothing here: the contractions read
 * the fp32 node-side state from HBM once either way and are bound by that
 * read, not by the tensor pipe. */
#define TPCONV_GEMM_FP32 0 /* fp32 accuracy: 3xTF32 split on tcgen05      */
#define TPCONV_GEMM_TF32 1 /* single TF32 pass on tcgen05                 */
#define TPCONV_GEMM_SIMT 3 /* plain fp32 FFMA (reference-precision mode)  */

/* operator families (tpconv_options.family).  Both follow "Sobek: streaming
 * edge-conditioned equivariant tensor-product convolution" (arXiv 2607.18074),
 * abstract, which evaluates two operator families without naming them:
 *   FULL         W_e[p] = sum_k b_k(|v_e|) Theta[p][k], a C_in x C_out matrix
 *                (fully connected multiplicity mixing); Theta is
 *                [P][R][C_in][C_out].
 *   CHANNELWISE  W_e[p] = diag(sum_k b_k(|v_e|) Theta[p][k, :]): each channel
 *                keeps its own weight; Theta is [P][R][C].  Every path needs
 *                C_in = C_out, else plan creation returns
 *                TPCONV_ERR_INVALID_ARG.  The edge streams are those of FULL;
 *                the node-level contractions become per-channel sums.
 * The path order and the CG coupling are the same for both. */
#define TPCONV_FAMILY_FULL 0
#define TPCONV_FAMILY_CHANNELWISE 1

/* operations, for tpconv_workspace_size */
#define TPCONV_OP_FORWARD 0
#define TPCONV_OP_BACKWARD 1
#define TPCONV_OP_DOUBLE_BACKWARD 2
#define TPCONV_OP_TRANSPOSE 3

typedef struct tpconv_plan tpconv_plan;

typedef struct tpconv_options {
  int radial;            /* TPCONV_RADIAL_*                                   */
  double radial_p0;      /* Gaussian: r_min; Bessel: r_cut                    */
  double radial_p1;      /* Gaussian: r_max; Bessel: unused                   */
  int gemm;              /* TPCONV_GEMM_*                                     */
  size_t workspace_cap;  /* bytes of node-side state per chunk; 0 = no cap    */
  int validate;          /* 1: check the graph on the device first (syncs)    */
  int family;            /* TPCONV_FAMILY_*                                   */
} tpconv_options;

/* Fill *opt with defaults: Bessel (r_cut 5), GEMM_FP32, no cap, no validation,
 * the FULL family. */
void tpconv_default_options(tpconv_options* opt);

/* Human-readable name of a status code (static storage; never NULL). */
const char* tpconv_status_string(int status);

/*
 * Create a plan (host only; touches no device).
 *   irreps_in, irreps_out: e.g. "64x0e+64x1o+64x2e"; l <= 3 per block.
 *   l_sh_max: highest spherical-harmonic degree, 0..3.
 *   R: radial basis size, 1..16.
 *   opt: NULL for defaults.
 * Paths follow the selection rules |l1-l2| <= l3 <= l1+l2 and
 * p1 (-1)^l2 = p3 ("The Price of Freedom", Approach).  The real CG table is
 * generated in double precision (Racah formula mapped to the real basis) and
 * self-checked for orthogonality; a failure returns TPCONV_ERR_INTERNAL.
 * On success *out owns the plan; release it with tpconv_plan_destroy.
 */
int tpconv_plan_create(tpconv_plan** out, const char* irreps_in, int l_sh_max,
                       const char* irreps_out, int R, const tpconv_options* opt);
int tpconv_plan_destroy(tpconv_plan* plan);

/* Sizes of a plan (host).  Any pointer may be NULL. */
int tpconv_plan_info(const tpconv_plan* plan, int* n_paths, int* dim_in, int* dim_out,
                     int* n_sh, size_t* theta_numel);

/* Path i (host): degrees, multiplicities and the offset of its Theta block. */
int tpconv_plan_path(const tpconv_plan* plan, int i, int* l1, int* l2, int* l3, int* c_in,
                     int* c_out, size_t* theta_offset);

/*
 * The real CG tensor C[m1][m2][m3] of one triple as generated for the device
 * table (host, double).  out must hold (2l1+1)(2l2+1)(2l3+1) doubles.
 * Returns TPCONV_ERR_UNSUPPORTED for l > 3 or a triple outside the triangle.
 */
int tpconv_cg_coefficients(int l1, int l2, int l3, double* out);

/*
 * Bytes of device workspace one call of `op` needs for a graph of N nodes and
 * E edges (host).  Independent of E except for TPCONV_OP_TRANSPOSE.
 */
int tpconv_workspace_size(const tpconv_plan* plan, int op, int64_t N, int64_t E, size_t* bytes);

/*
 * Sender-sorted view of the graph, once per graph (device, async).
 *   perm[E]       out: edge ids (CSR positions) grouped by sender, ascending
 *                      inside a sender (deterministic).
 *   s_rowptr[N+1] out: sender CSR offsets into perm.
 *   s_recv[E]     out: s_recv[j] = receiver of edge perm[j].
 */
int tpconv_graph_transpose(const tpconv_plan* plan, int64_t N, int64_t E, const int32_t* rowptr,
                           const int32_t* col, int32_t* perm, int32_t* s_rowptr, int32_t* s_recv,
                           void* workspace, size_t workspace_bytes, void* stream);

/*
 * Forward (device, async): out[N][dim_out] from x[N][dim_in], theta[theta_numel]
 * and the receiver CSR graph with edge vectors.  The operator of "Sobek"
 * (arXiv 2607.18074), abstract, in the streaming form the abstract describes:
 * a receiver-sorted edge stream accumulates A[r, k, p, u, m3] and a node-level
 * contraction with Theta mixes it (formula at the top of this file).
 */
int tpconv_forward(const tpconv_plan* plan, int64_t N, int64_t E, const int32_t* rowptr,
                   const int32_t* col, const float* edge_vec, const float* x, const float* theta,
                   float* out, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Allocation-free forward (device, async).  No counterpart in the pages: an
 * interface addition of this library for callers that cannot allocate device
 * memory (a host program without a device allocator of its own, a plugin that
 * may not bypass its framework's caching allocator, a fixed-latency loop that
 * must not call cudaMalloc, which can synchronise the device).
 *
 * Same arguments and result as tpconv_forward, without workspace: the
 * workspace is a fixed array of TPCONV_STATIC_SCRATCH_BYTES inside the library
 * (one per device).  Nothing is allocated.  Nothing in it needs to start at
 * zero.
 *   Returns TPCONV_ERR_WORKSPACE_TOO_SMALL, before any device work, when
 *   tpconv_workspace_size(plan, TPCONV_OP_FORWARD, N, E) exceeds
 *   TPCONV_STATIC_SCRATCH_BYTES.  The forward workspace is the node state of
 *   one receiver chunk (bounded by workspace_cap) plus a Theta region that no
 *   cap shrinks: 2 x theta_numel floats with GEMM_FP32, 1 x with GEMM_TF32,
 *   none with GEMM_SIMT or the CHANNELWISE family.  A plan whose Theta region
 *   alone approaches the limit (e.g. 128x{0e,1o,2e,3o} with GEMM_FP32, 24 MB)
 *   fits only with a small cap; tpconv_workspace_size says which.
 *   Calls share the array: calls that overlap in time (other streams, other
 *   host threads) race on it and must be serialised by the caller.
 *   The first call on a device also performs the library's one-time device
 *   set-up (constant tables, kernel attributes), which synchronises the
 *   device: make it before any stream capture.  The array's device address is
 *   looked up on every call (cudaGetSymbolAddress, a host-side query).
 *   Every device on which the library is loaded holds the array until the
 *   process exits, whether or not this entry point is called.
 */
#define TPCONV_STATIC_SCRATCH_BYTES (64u << 20) /* 64 MiB */
int tpconv_forward_static(const tpconv_plan* plan, int64_t N, int64_t E, const int32_t* rowptr,
                          const int32_t* col, const float* edge_vec, const float* x, const float* theta,
                          float* out, void* stream);

/*
 * Backward (device, async) for the cotangent g[N][dim_out] of out: the first
 * differentiation order of the operator ("Sobek", arXiv 2607.18074, abstract:
 * the streaming schedule extends through backward), run as a sender-sorted
 * stream into sender-side state B plus node contractions (dx = B . Theta,
 * dtheta = x^T B) and a receiver-sorted adjoint stream (dvec, dY, db).
 *   dx[N][dim_in], dtheta[theta_numel], dvec[E][3] (CSR order): optional.
 *   dY[E][n_sh], db[E][R]: optional per-edge adjoints of the spherical
 *   harmonics and radial basis (CSR order).
 * perm / s_rowptr / s_recv come from tpconv_graph_transpose; they may be NULL
 * when dx and dtheta are both NULL.
 */
int tpconv_backward(const tpconv_plan* plan, int64_t N, int64_t E, const int32_t* rowptr,
                    const int32_t* col, const int32_t* perm, const int32_t* s_rowptr,
                    const int32_t* s_recv, const float* edge_vec, const float* x,
                    const float* theta, const float* g, float* dx, float* dtheta, float* dvec,
                    float* dY, float* db, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Double backward (device, async): the second differentiation order the
 * abstract of "Sobek" (arXiv 2607.18074) names.  With Psi = <gg_x, dx> + <gg_vec, dvec> +
 * <gg_theta, dtheta> for the first-order gradients of <g, out>, returns
 * d_g = dPsi/dg [N][dim_out], d_x = dPsi/dx, d_vec = dPsi/dedge_vec [E][3] and
 * d_theta = dPsi/dtheta.  Each cotangent gg_* may be NULL (= zero); each
 * output may be NULL (= not computed).
 */
int tpconv_double_backward(const tpconv_plan* plan, int64_t N, int64_t E, const int32_t* rowptr,
                           const int32_t* col, const int32_t* perm, const int32_t* s_rowptr,
                           const int32_t* s_recv, const float* edge_vec, const float* x,
                           const float* theta, const float* g, const float* gg_x,
                           const float* gg_vec, const float* gg_theta, float* d_g, float* d_x,
                           float* d_vec, float* d_theta, void* workspace, size_t workspace_bytes,
                           void* stream);

/*
 * Device-side wait status (host; synchronises the stream).  The tensor-core
 * kernels (Theta contractions and Theta gradient) wait only on their own
 * pipelines (TMA copies into shared memory, tensor-core MMAs), and every such
 * wait is bounded by a time limit.  When one expires the kernel records it,
 * stops issuing work, waits (bounded) for the copies and MMAs it has already
 * issued, frees its tensor memory and returns; its output is then not valid.
 * No kernel of the library waits on another CTA, kernel or GPU.
 *   *status = TPCONV_ERR_TIMEOUT if a wait expired since the previous query
 *   (the record is cleared), else TPCONV_OK.  Returns TPCONV_ERR_CUDA if the
 *   stream or the query itself fails.
 * With tpconv_options.validate set, every forward / backward / double backward
 * ends with this query and returns its status.  Not defined in the pages: an
 * interface addition for failure detection.
 */
int tpconv_get_device_status(const tpconv_plan* plan, void* stream, int* status);

/*
 * Limit of those device waits, in nanoseconds, for calls issued from now on
 * (process-wide; 0 restores the default of 2 s).  Tests use a tiny limit to
 * make the waits run out on purpose and check the error path.
 */
int tpconv_set_wait_limit(uint64_t ns);

/*
 * Diagnostics (host).  Every kernel launch of the library is counted per phase.
 * With profiling enabled, each phase of each call is bracketed by CUDA events
 * recorded on the call's stream; tpconv_profile_read synchronises those events
 * and returns the summed device time of a phase.  Profiling state is process-
 * wide and not thread-safe; it does not change results.
 */
#define TPCONV_PHASE_TRANSPOSE 0   /* sender-sorted view of the graph          */
#define TPCONV_PHASE_FWD_EDGE 1    /* forward receiver edge stream -> A        */
#define TPCONV_PHASE_FWD_NODE 2    /* out = A . Theta                          */
#define TPCONV_PHASE_BWD_NODE_G 3  /* G = g . Theta^T                          */
#define TPCONV_PHASE_BWD_EDGE_R 4  /* receiver adjoint stream -> dvec, dY, db  */
#define TPCONV_PHASE_BWD_EDGE_S 5  /* sender stream -> B                       */
#define TPCONV_PHASE_BWD_NODE_X 6  /* dx = B . Theta, dtheta = x^T B           */
#define TPCONV_PHASE_DBL_EDGE_A 7  /* double backward receiver stream -> A0,A1 */
#define TPCONV_PHASE_DBL_NODE_A 8  /* d_g = A1 . Theta + A0 . gg_theta         */
#define TPCONV_PHASE_DBL_EDGE_R 9  /* double backward adjoint stream -> d_vec  */
#define TPCONV_PHASE_DBL_EDGE_S 10 /* double backward sender stream -> B0, B1  */
#define TPCONV_PHASE_DBL_NODE_X 11 /* d_x, d_theta                             */
#define TPCONV_PHASE_OTHER 12      /* memsets, packing, G for double backward  */
#define TPCONV_N_PHASES 13

int tpconv_profile_enable(int on);  /* 1: record events from now on; 0: stop    */
int tpconv_profile_reset(void);     /* drop recorded events and launch counts   */
/* ms: summed device milliseconds of the phase since the last reset (needs
 * profiling enabled while the calls ran); launches: kernels launched in the
 * phase since the last reset (always counted).  Either pointer may be NULL. */
int tpconv_profile_read(int phase, double* ms, int64_t* launches);

#ifdef __cplusplus
}
#endif

#endif /* TPCONV_H */
