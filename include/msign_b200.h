/*
 * msign_b200.h - C ABI of the B200 (sm_100a) Newton-Schulz msign library.
 *
 * The operation is msign(M) = (M M^T)^{-1/2} M = U V^T, the polar factor of
 * M, approximated by the quintic Newton-Schulz iteration that the Muon
 * optimizer uses.  Sources, cited by page title and section:
 *
 *   [P1] nil9.net blog, flash-muon post: the symmetric X X^T operator
 *        ("matmul_transpose") that computes one triangle and mirrors it.
 *   [P2] "msign算子的Newton-Schulz迭代（上）" (kexue.fm/archives/10922):
 *        definition (eq. 1-2), iteration X0 = M/||M||_F,
 *        X <- aX + bX(X^T X) + cX(X^T X)^2 (eq. 4, 6), Jordan's
 *        coefficients (a,b,c) = (3.4445, -4.7750, 2.0315), T = 5 (eq. 7),
 *        batched routine with bf16 cast, transpose when rows > cols and
 *        eps = 1e-20 under the square root (section 参考实现), per-step
 *        coefficients (section 解开约束, eq. 12).
 *   [P3] "Gram Newton-Schulz" (zifeng-mai.github.io, 2026/04/05): Muon
 *        update (section 1.1), Algorithm 2 "Stabilized Gram Newton-Schulz"
 *        (section 3.4) with its restart (section 3.2), fp16 arithmetic
 *        (section 3.3), and the fused symmetric kernel C <- aAB + bC + gI
 *        (section 4).
 *   [P5] the Mousse post (anti-entrophic.github.io/posts/10054), section
 *        "Mousse": L^(-1/4) msign(L^(-1/4) G R^(-1/4)) R^(-1/4) with
 *        Shampoo-style Kronecker factors L and R.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Matrices are dense and row-major.  A batch of rows x cols matrices lies
 *   back to back (matrix i starts at element i*rows*cols) unless the entry
 *   point takes a batch stride (msign_ns and gram_ns: matrix i starts at
 *   element i*stride).  All pointers passed as matrices are DEVICE pointers
 *   unless stated otherwise.
 * - The caller owns every buffer.  The library allocates nothing: it works
 *   in the caller's workspace, whose size the *_workspace_size() query gives
 *   (a workspace must be 256-byte aligned).  Inputs are never written
 *   unless stated.  Outputs must not overlap the workspace, nor an input
 *   unless the entry point says so (msign_ns and gram_ns accept out == in).
 * - All work is enqueued asynchronously on `stream` (a cudaStream_t; NULL is
 *   the legacy default stream).  Argument checks happen on the host before
 *   anything is enqueued; on any error status nothing has been enqueued,
 *   except for MSIGN_ERR_CUDA, which reports a failed launch.
 * - Kernels never wait without a time limit.  A wait that runs out sets a
 *   device-side error word and the kernel returns; msign_sync_status()
 *   reports it as MSIGN_ERR_TIMEOUT.
 * - Coefficient schedules are HOST arrays.  NULL selects Jordan's triple
 *   for T = 5 steps ([P2] eq. 7).
 * - Empty problems (batch, rows or cols = 0) are valid and do nothing,
 *   except gram_xxt with m = 0 and n > 0, which writes the zero n x n result.
 * - Size limits: batch <= 65535 and every matrix dimension <= 2^30
 *   (mousse_inv_root: n <= 2^20); beyond them an entry point returns
 *   MSIGN_ERR_UNSUPPORTED before enqueuing anything.
 * - Entry points run on the CURRENT device (cudaGetDevice) and every pointer
 *   of a call must belong to it.  The library keeps per-device addresses
 *   (its device error word, the msign_ns_noalloc scratch) for the life of
 *   the process: do not use it across a cudaDeviceReset() or any other
 *   destruction of the device's primary context.
 */
#ifndef MSIGN_B200_H
#define MSIGN_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st *msign_stream_t;

typedef enum {
  MSIGN_OK = 0,
  MSIGN_ERR_INVALID_ARG = 1,  /* null pointer, negative size, bad coefficient count */
  MSIGN_ERR_UNSUPPORTED = 2,  /* dtype combination or size outside what is built */
  MSIGN_ERR_WORKSPACE = 3,    /* workspace missing, too small or misaligned */
  MSIGN_ERR_CUDA = 4,         /* a CUDA call or kernel launch failed */
  MSIGN_ERR_TIMEOUT = 5       /* a kernel's bounded wait ran out (see msign_sync_status) */
} msign_status;

typedef enum {
  MSIGN_BF16 = 0,
  MSIGN_FP16 = 1,
  MSIGN_FP32 = 2
} msign_dtype;

/* Coefficient schedule: steps triples (a_t, b_t, c_t), one per iteration,
 * laid out a_1 b_1 c_1 a_2 b_2 c_2 ... in a HOST array.  abc == NULL means
 * Jordan's triple repeated `steps` times (steps <= 0 then means 5).
 * eps < 0 selects the default of the routine (1e-20 for msign_ns, 1e-7 for
 * gram_ns).
 * init selects the initial normalisation of msign_ns and muon_step:
 *   0  X0 = X / sqrt(sum X^2 + eps) (the msign page's reference routine);
 *   1  additionally, at step 0, rescale X0, X0 X0^T and (X0 X0^T)^2 by n,
 *      n^2 and n^4 with n = (||(X0 X0^T)^2||_F^2 + eps)^(1/8) -- the
 *      sharper bound on the largest singular value from the msign page's
 *      section on improving the initial value (改进初值).  bf16 and fp16
 *      compute only (MSIGN_ERR_UNSUPPORTED with the fp32-accurate path and
 *      with gram_ns).
 * method selects the iteration msign_ns and muon_step run (gram_ns takes 0
 * only):
 *   0  standard Newton-Schulz, always;
 *   1  automatic: Gram Newton-Schulz ([P3] Algorithm 2, the page's restart
 *      after step 2 when T >= 3, fp16 inside, eps as for gram_ns) where it is
 *      expected to be faster, standard Newton-Schulz elsewhere.
 *      msign_ns_route() reports the choice for a shape.
 * Added in ABI 101 (init) and 102 (method); a caller built against an
 * older ABI lacks the later fields.  ABI 103 added the batch strides of
 * msign_ns and gram_ns. */
typedef struct {
  int steps;
  const float *abc;
  float eps;
  int init;
  int method;
} msign_coeffs;

/* Library ABI version (major * 100 + minor). */
int msign_abi_version(void);

/* Fires the failure path of the library's bounded waits, for tests: one
 * kernel thread waits on an mbarrier that nothing completes and on a device
 * counter that nothing increments, each for limit_ns (0 < limit_ns <= 1e9),
 * then returns.  Each expiry sets the device error word, so the next
 * msign_sync_status(stream) returns MSIGN_ERR_TIMEOUT (and clears the word);
 * the context stays usable.  Asynchronous on `stream`.  No counterpart on
 * the pages. */
msign_status msign_selftest_timeout(uint64_t limit_ns, msign_stream_t stream);

/* Human-readable name of a status code (static storage). */
const char *msign_status_string(msign_status status);

/* Waits for `stream`, then reads and clears the device-side error word that
 * bounded waits set.  Returns MSIGN_OK, MSIGN_ERR_TIMEOUT, or
 * MSIGN_ERR_CUDA if the stream reports an error. */
msign_status msign_sync_status(msign_stream_t stream);

/* ------------------------------------------------------------------------
 * Launch records, for benchmarks (no counterpart on the pages).
 *
 * msign_profile_enable(1) makes every later kernel launch of the library
 * record a CUDA event on its stream before and after the kernel, tagged with
 * a kind and with the launch's algorithmic work: useful FLOPs (symmetric
 * outputs count one triangle) and compulsory HBM bytes (operands, epilogue
 * input and outputs once each).  msign_profile_read() waits for the records
 * of one kind and returns their count, summed device time in milliseconds,
 * FLOPs and bytes; msign_profile_reset() drops all records.  Kinds: 0 =
 * tensor-core GEMM, 1 = Frobenius-norm reduction, 2 = cast/orient/scale
 * ingest, 3 = Muon elementwise (momentum, weight update).  Not thread-safe
 * with concurrent library calls on other host threads.
 * ------------------------------------------------------------------------ */
msign_status msign_profile_enable(int enable);

msign_status msign_profile_read(int kind, int *launches, double *total_ms, double *flops, double *bytes);

msign_status msign_profile_reset(void);

/* Diagnostics (no counterpart on the pages): msign_set_chaining(0) makes
 * later msign_ns and muon_step calls on the standard route run each product
 * of an iteration step (X X^T, the A^2 product with its combine b A + c A^2,
 * B X with its a X term) as a launch of its own, so that a profiler sees the
 * three phases apart; msign_set_chaining(1) restores the default, the phases
 * of up to five steps chained in one launch.  Results agree with the chained
 * ones to rounding (X X^T is not split along K then).  Process-wide; returns
 * the previous setting.  Added in ABI 104. */
int msign_set_chaining(int enable);

/* ------------------------------------------------------------------------
 * msign_ns: batched standard Newton-Schulz msign ([P2] eq. 4-7, section
 * 参考实现).
 *
 * For each of `batch` matrices M (rows x cols): cast to the compute dtype,
 * work on M^T when rows > cols, X0 = M / sqrt(sum(M^2) + eps), then for
 * t = 1..T:  A = X X^T;  B = b_t A + c_t A A;  X = a_t X + B X;  finally
 * transpose back and write X in io_dtype.
 *
 *   in, out        device pointers, batch x rows x cols in io_dtype; out may
 *                  be in (the input is read whole into the workspace before
 *                  the first store to out)
 *   in_stride,     elements from the start of one matrix of `in` (`out`) to
 *   out_stride     the next: 0 means rows*cols (back to back), otherwise at
 *                  least rows*cols (MSIGN_ERR_INVALID_ARG else), e.g. every
 *                  other matrix of a larger batch.  Each matrix itself is
 *                  dense row-major.  The pages' routine acts on the last two
 *                  dims of a batch (section 参考实现); a stride lets a caller
 *                  pass a batch that is a view into a larger tensor.
 *   io_dtype       MSIGN_BF16, MSIGN_FP16 or MSIGN_FP32
 *   compute_dtype  MSIGN_BF16: bf16 tensor-core operands, fp32 accumulation,
 *                  fp32 epilogue arithmetic and an fp32 copy of X between
 *                  steps (the input is cast to bf16 first, as the routine of
 *                  [P2] section 参考实现 does).
 *                  MSIGN_FP16: the same with fp16 operands (the input is
 *                  cast to fp16 first); 8x smaller rounding than bf16 at the
 *                  same tensor-core rate ([P3] section 3.3 argues the same
 *                  for Gram NS).
 *                  MSIGN_FP32: fp32-accurate products: every operand is kept
 *                  as two tf32 planes (hi, lo) and each product is
 *                  hi*hi + hi*lo + lo*hi on the tf32 tensor cores with fp32
 *                  accumulation (about 6x the bf16 time).
 *   coeffs         schedule (NULL: Jordan, T = 5, eps = 1e-20, standard NS);
 *                  coeffs->method = 1 lets the call run Gram NS instead (see
 *                  msign_ns_route)
 *   workspace      device scratch of at least msign_ns_workspace_size() bytes
 *                  (enough for either iteration wherever the route picks it)
 * ------------------------------------------------------------------------ */
size_t msign_ns_workspace_size(int64_t batch, int64_t rows, int64_t cols, msign_dtype compute_dtype);

/* The iteration msign_ns runs for these arguments: 0 standard NS, 1 Gram NS,
 * or a negated status for a schedule or dtype msign_ns would reject
 * (-MSIGN_ERR_INVALID_ARG, -MSIGN_ERR_UNSUPPORTED).  Host only.
 *
 * With coeffs->method = 1 the call takes Gram NS when all of these hold:
 * 16-bit compute (Gram NS iterates in fp16; the fp32-accurate path stays
 * standard), init = 0 (the sharper normalisation is a standard-NS option),
 * after orientation (n <= m) n >= 512 and m - n >= 3072, or m - n >= 2048
 * where n <= 2048, and Gram NS's workspace is no larger than
 * msign_ns_workspace_size() (2048 x 4096 alone is not routed for that
 * reason).  [P3] section 2 counts (17 + 3 alpha) n^3 FLOPs for Gram NS
 * against T (3 alpha + 1) n^3 for standard NS with symmetric products,
 * alpha = m / n, so Gram NS does less work whenever alpha > 1; measured on a
 * B200, its chain of n x n fp16 products pays from the widths above (e.g.
 * 0.91 of standard NS's time at 1024 x 4096, 0.98 at 4096 x 7168, 1.04 at
 * 4096 x 6144), and below n = 512 both are latency-bound.  The two results
 * agree within 2e-2 (relative Frobenius).  Changed in ABI 106 (before it:
 * m - n >= 4096 for every n). */
int msign_ns_route(int64_t batch, int64_t rows, int64_t cols, msign_dtype compute_dtype,
                   const msign_coeffs *coeffs);

msign_status msign_ns(const void *in, void *out, msign_dtype io_dtype, msign_dtype compute_dtype,
                      int64_t batch, int64_t rows, int64_t cols, int64_t in_stride, int64_t out_stride,
                      const msign_coeffs *coeffs, void *workspace, size_t workspace_bytes,
                      msign_stream_t stream);

/* ------------------------------------------------------------------------
 * msign_ns_noalloc: msign_ns for callers that cannot allocate device memory.
 * The pages have no counterpart of this entry point.
 *
 * Some callers may not call cudaMalloc where they need msign: plugins hosted
 * by a framework that reserves all GPU memory for its own pool (an
 * allocation outside that pool fails or steals from it), and real-time
 * loops that forbid allocation after start-up (cudaMalloc can synchronise
 * the device and takes an unbounded time).  This variant takes no
 * workspace: it computes exactly what msign_ns does with compute_dtype
 * MSIGN_BF16, in a scratch array built into the library (a file-scope
 * __device__ array of msign_ns_noalloc_max_bytes() = 32 MiB, held on every
 * GPU that loads the library until the process exits).  It makes no device
 * allocation of its own; inputs and outputs are the caller's.
 *
 * - A problem whose msign_ns_workspace_size(batch, rows, cols, MSIGN_BF16)
 *   exceeds the built-in scratch is rejected with MSIGN_ERR_WORKSPACE before
 *   anything is enqueued (e.g. 1024 x 2048 fits, 2048 x 2048 does not).
 * - The first call on a device looks up that device's address of the array
 *   (cudaGetSymbolAddress) with the device current; make that first call
 *   before any stream capture that contains later calls.
 * - All calls on a device share the one array and leave their intermediate
 *   results in it.  Each call clears the part that must start at zero (its
 *   schedule and dependency counters) on its stream before use; every other
 *   part is written before it is read.  Calls whose executions overlap on
 *   the GPU (different streams, or different host threads without ordering)
 *   race on the array and give wrong results: order them on one stream.
 * ------------------------------------------------------------------------ */
size_t msign_ns_noalloc_max_bytes(void);

msign_status msign_ns_noalloc(const void *in, void *out, msign_dtype io_dtype,
                              int64_t batch, int64_t rows, int64_t cols, const msign_coeffs *coeffs,
                              msign_stream_t stream);

/* ------------------------------------------------------------------------
 * msign_ns_host: msign_ns on HOST buffers (no counterpart on the pages).
 *
 * Enqueues on `stream`: the copy of the input from in_host into the
 * workspace, msign_ns in place there (same arguments and results as
 * msign_ns with back-to-back matrices), and the copy of the result to
 * out_host.  in_host and out_host are host pointers to batch x rows x cols
 * values in io_dtype, dense; they must stay valid, and out_host unread,
 * until the stream has passed the call.  With page-locked (pinned) host
 * memory the copies are asynchronous and calls on two streams overlap one
 * call's copies with the other's kernels; pageable memory works, with the
 * copies synchronous to the host.  out_host may equal in_host.
 *   workspace   device scratch of at least msign_ns_host_workspace_size()
 *               bytes (the device copy of the matrices, then msign_ns's
 *               workspace), 256-byte aligned
 * Errors as for msign_ns; the argument checks come before any copy is
 * enqueued.  Added in ABI 105.
 * ------------------------------------------------------------------------ */
size_t msign_ns_host_workspace_size(int64_t batch, int64_t rows, int64_t cols, msign_dtype io_dtype,
                                    msign_dtype compute_dtype);

msign_status msign_ns_host(const void *in_host, void *out_host, msign_dtype io_dtype, msign_dtype compute_dtype,
                           int64_t batch, int64_t rows, int64_t cols, const msign_coeffs *coeffs,
                           void *workspace, size_t workspace_bytes, msign_stream_t stream);

/* ------------------------------------------------------------------------
 * gram_xxt: symmetric Gram product A = X X^T ([P1] flash-muon
 * matmul_transpose; [P3] section 4, triangular scheduling).
 *
 * Only output tiles on or above the diagonal are computed; each is stored
 * and its transpose is stored into the mirrored position from the same
 * fp32 accumulators, so A is bit-exactly symmetric.
 *
 *   X   device pointer, batch x n x m, dtype x_dtype (MSIGN_BF16 or MSIGN_FP16)
 *   A   device pointer, batch x n x n, dtype a_dtype (BF16, FP16 or FP32)
 *   workspace  needed only when X is not 16-byte aligned or m is not a
 *              multiple of 8 (X is then staged into the workspace); the
 *              query returns 0 otherwise.
 * ------------------------------------------------------------------------ */
size_t gram_xxt_workspace_size(int64_t batch, int64_t n, int64_t m, msign_dtype x_dtype, const void *X);

msign_status gram_xxt(const void *X, msign_dtype x_dtype, void *A, msign_dtype a_dtype,
                      int64_t batch, int64_t n, int64_t m,
                      void *workspace, size_t workspace_bytes, msign_stream_t stream);

/* ------------------------------------------------------------------------
 * gram_ns: batched Stabilized Gram Newton-Schulz ([P3] Algorithm 2,
 * sections 3.2-3.4).
 *
 * For each matrix (oriented so that n <= m as in msign_ns):
 * X <- X / (||X||_F + eps); X <- float16(X); then for each segment of steps
 * between restarts: R = X X^T, Q = I; per step Z = b R + c R^2,
 * Q <- QZ + aQ, RZ <- RZ + aR, R <- Z RZ + a RZ; then X <- Q X.  The n x n
 * products are symmetric (polynomials in one Gram matrix) and use the
 * triangle schedule; the a_t terms are added in fp32 epilogues.  Operands
 * are fp16, accumulation fp32.
 *
 *   in, out        device pointers, batch x rows x cols in io_dtype; out may
 *                  be in, as for msign_ns
 *   in_stride,     batch strides in elements, as for msign_ns (0: back to
 *   out_stride     back)
 *   restart_after  HOST array of step numbers after which to restart
 *                  (values in 1..T-1); NULL with n_restart < 0 selects the
 *                  page's schedule {2}; n_restart == 0 means no restart.
 * ------------------------------------------------------------------------ */
size_t gram_ns_workspace_size(int64_t batch, int64_t rows, int64_t cols);

msign_status gram_ns(const void *in, void *out, msign_dtype io_dtype,
                     int64_t batch, int64_t rows, int64_t cols, int64_t in_stride, int64_t out_stride,
                     const msign_coeffs *coeffs, const int *restart_after, int n_restart,
                     void *workspace, size_t workspace_bytes, msign_stream_t stream);

/* ------------------------------------------------------------------------
 * muon_step: one Muon update of a list of weight matrices ([P3] section
 * 1.1; momentum M_0 = 0, no Nesterov term, no weight decay).
 *
 * For each matrix i (rows[i] x cols[i]):
 *   M_i <- momentum * M_i + G_i                           (fp32)
 *   O_i  = msign_ns(M_i)  with bf16 compute, `coeffs` schedule
 *   W_i <- W_i - lr * sqrt(max(1, rows_i / cols_i)) * O_i
 * Matrices of equal (oriented) shape share grouped launches; all shapes in
 * one call are scheduled together.
 * With coeffs->method = 1, a matrix for which muon_step_route(rows_i,
 * cols_i, coeffs) is 1 runs Gram NS instead (4096 x 11008 and 4096 x 14336
 * do; 1024 x 4096 does not): M_i is updated by its own elementwise pass,
 * O_i = gram_ns(M_i) (restart after step 2 when T >= 3) is stored in bf16
 * in place of Gram NS's dead copy of X, and W_i is updated from it.
 * Matrices of equal shape (rows, cols) share one batched Gram-NS chain,
 * after the standard-route groups.
 *
 *   W, M, G     HOST arrays of `num` DEVICE pointers.  W_i in w_dtype
 *               (BF16 or FP32) is updated in place; M_i is fp32 and updated
 *               in place; G_i is in g_dtype (BF16 or FP32) and read only.
 *   rows, cols  HOST arrays of `num` sizes.
 *   workspace   at least muon_step_workspace_size() bytes; a smaller one
 *               (but at least the size for the largest single matrix) makes
 *               the call process the list in several groups.
 * ------------------------------------------------------------------------ */
size_t muon_step_workspace_size(int num, const int64_t *rows, const int64_t *cols);

/* The iteration muon_step runs for one rows x cols matrix: 0 standard NS,
 * 1 Gram NS, or a negated status for a schedule muon_step would reject.
 * Host only.  A matrix takes Gram NS when msign_ns_route(1, rows, cols,
 * MSIGN_BF16, coeffs) is 1, m - n >= 4096 after orientation, and Gram NS's
 * workspace with a bf16 O fits in the matrix's standard-route workspace.
 * The width is larger than msign_ns's because muon_step runs its Gram-NS
 * matrices after the grouped standard-route launch, where a small matrix
 * would otherwise share the launch with the large ones (a Llama layer's
 * 1024 x 4096 k and v stay standard).  Added in ABI 106. */
int muon_step_route(int64_t rows, int64_t cols, const msign_coeffs *coeffs);

msign_status muon_step(int num, void *const *W, float *const *M, const void *const *G,
                       const int64_t *rows, const int64_t *cols,
                       msign_dtype w_dtype, msign_dtype g_dtype,
                       float momentum, float lr, const msign_coeffs *coeffs,
                       void *workspace, size_t workspace_bytes, msign_stream_t stream);

/* ------------------------------------------------------------------------
 * Mousse: msign in a space whitened by Shampoo-style Kronecker factors (the
 * Mousse post, anti-entrophic.github.io/posts/10054, section "Mousse"):
 *
 *   Delta W = -L^(-1/4) msign(L^(-1/4) G R^(-1/4)) R^(-1/4)
 *
 * for a gradient G (rows x cols), L (rows x rows) and R (cols x cols)
 * symmetric positive semidefinite statistics (Shampoo's accumulated G G^T
 * and G^T G are the plain choice; the post leaves their update open).
 * mousse_inv_root computes the roots, which an optimizer refreshes every few
 * steps; mousse_direction is the per-step hot path and returns
 * D = L^(-1/4) msign(L^(-1/4) G R^(-1/4)) R^(-1/4), the update being -lr D.
 * ------------------------------------------------------------------------ */

/* out = (A + eps I)^(-1/4) for each of `batch` symmetric positive
 * semidefinite n x n fp32 matrices A (device, back to back; only the upper
 * triangle of each A is read).  Coupled Newton iteration for inverse p-th
 * roots with p = 4, X_{j+1} = X_j T_j, M_{j+1} = T_j^4 M_j,
 * T_j = (5 I - M_j) / 4, from X_0 = s^(1/4) I, M_0 = s (A + eps I),
 * s = 1 / (||A||_F + eps); every product runs on the tensor cores in
 * fp32-accurate arithmetic (3xTF32, as msign_ns's MSIGN_FP32).
 *
 *   eps    damping >= 0 (a rank-deficient statistic needs eps > 0)
 *   iters  Newton steps (0: 20).  An eigenvalue lambda of A converges once
 *          s (lambda + eps) has been driven to 1: it grows by a factor of
 *          about 2.4 per step while small, then converges quadratically,
 *          so iters ~ log(kappa) / log(2.44) + 4 with kappa =
 *          (||A||_F + eps) / (lambda_min + eps).  2 <= iters <= 1000.
 *   out    device, batch x n x n fp32, exactly symmetric
 *   workspace  at least mousse_inv_root_workspace_size() bytes
 * ------------------------------------------------------------------------ */
size_t mousse_inv_root_workspace_size(int64_t batch, int64_t n);

msign_status mousse_inv_root(const float *A, float *out, int64_t batch, int64_t n, float eps, int iters,
                             void *workspace, size_t workspace_bytes, msign_stream_t stream);

/* out = L_root msign(L_root G R_root) R_root for each of `batch` matrices G
 * (rows x cols, io_dtype, back to back), with L_root = L^(-1/4)
 * (batch x rows x rows fp32) and R_root = R^(-1/4) (batch x cols x cols
 * fp32), e.g. from mousse_inv_root.  The four projection products run with
 * bf16 operands and fp32 accumulation; msign is msign_ns with bf16 compute
 * and the `coeffs` schedule (method must be 0; init 0 or 1).  out is
 * batch x rows x cols in io_dtype and must not overlap G.
 *   workspace  at least mousse_direction_workspace_size() bytes
 * ------------------------------------------------------------------------ */
size_t mousse_direction_workspace_size(int64_t batch, int64_t rows, int64_t cols);

msign_status mousse_direction(const void *G, void *out, msign_dtype io_dtype, int64_t batch, int64_t rows,
                              int64_t cols, const float *L_root, const float *R_root, const msign_coeffs *coeffs,
                              void *workspace, size_t workspace_bytes, msign_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MSIGN_B200_H */
