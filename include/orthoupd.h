/*
 * orthoupd.h -- C ABI of liborthoupd.so: the optimizer step that
 * orthonormalizes each weight matrix's momentum (Muon Newton-Schulz, Gram
 * Newton-Schulz, the Dion3 row-selection rule, Dion / Orth-Dion low-rank
 * steps), as hand-written CUDA kernels for NVIDIA B200 (sm_100a).
 *
 * Sources the calls follow (cited by page title and section):
 *   [D3]  "Dion3: Full-Stack Orthogonal Updates" (arXiv abstract).
 *   [D3s] "Dion3：全栈正交更新" (ai-feeds summary), sections 核心洞察,
 *         核心模块, 输入输出流程, 局限.
 *   [OD]  "Orth-Dion: Eliminating Geometric Mismatch in Distributed Low-Rank
 *         Spectral Optimization" (gist.science), sections Problem Statement,
 *         The Geometric Insight, Orth-Dion, Theoretical Contributions.
 *   [D1]  "Dion: The Distributed Orthonormal Update Revolution Is Here",
 *         Technical details.
 *
 * Conventions shared by every call
 *   - Every call returns an int: OUO_OK (0) or a negative OUO_ERR_* code.
 *     On error, ouo_last_error() returns a message (thread-local).  Argument
 *     validation happens before anything is launched: a failed call has
 *     launched nothing.
 *   - Every call is asynchronous: kernels are enqueued on `stream` (a
 *     cudaStream_t; NULL = the legacy default stream) on the current device.
 *     Results are ready when the stream is synchronized.
 *   - Every pointer inside an ouo_mat, every workspace and every index /
 *     scale / status array marked "device" is caller-owned device memory on
 *     the current device.  The library allocates no device memory and keeps
 *     no pointer after the call returns (a stream-ordered use of the memory
 *     is pending until the stream reaches it).
 *   - Matrices are row-major with a leading dimension `ld` (elements between
 *     consecutive rows, ld >= cols).  Element (i, j) is at ptr + i*ld + j.
 *     Row-major with rows = out-features matches PyTorch's [out, in]
 *     weights.  Pointers must be aligned to their element size.  Matrices
 *     whose rows all start on 16-byte boundaries take 16-byte vector paths;
 *     others are processed element by element (same results).
 *   - A batch is a host array of `nmat` ouo_mat describing independent
 *     matrices.  Matrices of equal shape are processed together; batches may
 *     mix shapes.  nmat <= OUO_MAX_BATCH.
 *   - dtype arguments take OUO_F32 or OUO_BF16.
 *   - `dev_status` (optional, device int*, may be NULL): kernels OR
 *     OUO_STATUS_* bits into it when a bounded wait times out or a
 *     numerical breakdown is met; read it after synchronizing.  It is never
 *     cleared by the library.
 */
#ifndef ORTHOUPD_H
#define ORTHOUPD_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define OUO_VERSION 1

/* return codes */
#define OUO_OK 0
#define OUO_ERR_INVALID_ARG (-1)  /* bad pointer, shape, ld, alignment, value */
#define OUO_ERR_UNSUPPORTED (-2)  /* valid request the library does not take */
#define OUO_ERR_WORKSPACE (-3)    /* workspace missing or too small          */
#define OUO_ERR_CUDA (-4)         /* a CUDA runtime / driver call failed     */
#define OUO_ERR_NO_DEVICE (-5)    /* no sm_100 device current                */

/* bits OR-ed into *dev_status by kernels */
#define OUO_STATUS_TIMEOUT 1      /* a bounded device wait gave up           */
#define OUO_STATUS_BREAKDOWN 2    /* Cholesky breakdown survived the shift   */

/* element types */
#define OUO_F32 0
#define OUO_BF16 1

/* momentum modes */
#define OUO_MOMENTUM_EMA 0        /* M <- mu * M + G                         */
#define OUO_MOMENTUM_ACCUM 1      /* M <- M + G  (error-feedback buffer B)   */

/* Dion3 error-feedback modes */
#define OUO_EF_NONE 0             /* selection only reads the momentum       */
#define OUO_EF_ROWS 1             /* kept rows: M[S] <- mu * B[S]            */

/* arithmetic of the orthogonalization */
#define OUO_PREC_BF16 0  /* bf16 operands for k x n products, tf32 for k x k,
                            fp32 accumulation (tensor cores)                 */
#define OUO_PREC_FP32 1  /* fp32 operands and accumulation (CUDA cores)      */

/* Dion finishing step */
#define OUO_DION_COLNORM 0        /* Dion: column normalization              */
#define OUO_DION_QR 1             /* Orth-Dion: QR orthogonalization         */

#define OUO_MAX_BATCH 4096
#define OUO_MAX_RESTARTS 8
/* size of the fixed scratch array of gram_ns_orthogonalize_noalloc (64 MiB) */
#define OUO_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)

typedef struct ouo_mat {
  void* ptr;     /* device pointer to element (0, 0)                        */
  int64_t rows;
  int64_t cols;
  int64_t ld;    /* elements between consecutive rows (>= cols)             */
} ouo_mat;

/* Newton-Schulz parameters.  ouo_ns_default() fills Muon's quintic
 * coefficients (a, b, c) = (3.4445, -4.7750, 2.0315), 5 iterations, safety
 * 1, eps 1e-7, normalize 1, bf16 precision, one restart after iteration 3. */
typedef struct ouo_ns_params {
  float a, b, c;       /* p(x) = a x + b x^3 + c x^5                         */
  int iters;           /* number of iterations (>= 0)                        */
  float safety;        /* s >= 1: every iteration uses p(x / s)              */
  float eps;           /* X0 = X / (||X||_F + eps)                           */
  int normalize;       /* 1: normalize first; 0: input already normalized    */
  int precision;       /* OUO_PREC_BF16 or OUO_PREC_FP32                     */
  int n_restart;       /* Gram NS only: number of entries in restart_after   */
  int restart_after[OUO_MAX_RESTARTS]; /* iterations t (1 <= t < iters)      */
} ouo_ns_params;

/* Dion / Orth-Dion parameters.  ouo_dion_default(): rank 256, mu 0.95,
 * beta 1, lr 0.01, wd 0, COLNORM, eps 1e-8. */
typedef struct ouo_dion_params {
  int rank;            /* r, 1 <= r <= min(rows, cols); 0 = per matrix, from
                          Q_state[i].rows (ragged ranks)                      */
  float mu;            /* momentum / error-feedback factor                    */
  float beta;          /* error-feedback coefficient (1 = Dion's buffer)      */
  float lr;            /* learning rate                                       */
  float wd;            /* decoupled weight decay                              */
  int norm_mode;       /* OUO_DION_COLNORM or OUO_DION_QR                     */
  float eps;           /* column-normalization guard                          */
} ouo_dion_params;

/* ------------------------------------------------------------------------ */

int ouo_version(void);
const char* ouo_last_error(void);
/* Number of kernels this library has enqueued in this process, all devices
 * and threads together (monotonic; for accounting in benchmarks). */
unsigned long long ouo_launch_count(void);

/* Kernel timing for benchmarks.  ouo_timing_enable(1) creates a pool of CUDA
 * events (on the current device) and from then on brackets every
 * tensor-core GEMM launch with two events on its stream, recording the
 * launch's kind and algorithmic flops (2 M N K per matrix; symmetric
 * outputs M (M + 1) K, the upper triangle).  ouo_timing_enable(0) drops the
 * records and the pool.  At most 4096 launches are recorded.
 * ouo_timing_read(kind, ...) waits for the recorded events and returns the
 * number of launches, their summed device time (ms) and summed flops for
 * one kind (-1 = all): kind = (symmetric ? 4 : 0) + (tf32 ? 2 : 0) +
 * (B operand MN-major ? 1 : 0). */
int ouo_timing_enable(int on);
int ouo_timing_read(int kind, int* launches, double* total_ms, double* flops);

/* Test hook for the failure path of the bounded device waits: launches one
 * block that waits on an mbarrier nothing ever completes, gives up after
 * limit_ns (at most 1 s) and ORs OUO_STATUS_TIMEOUT into *dev_status, the
 * way a stalled GEMM pipeline reports.  Nothing faults or hangs; the
 * context stays usable. */
int ouo_debug_wait_timeout(int* dev_status, unsigned long long limit_ns,
                           void* stream);
void ouo_ns_default(ouo_ns_params* p);
void ouo_dion_default(ouo_dion_params* p);

/*
 * dion_momentum_update -- the momentum step that opens every optimizer step
 * ([D3s] 输入输出流程: "update momentum" first; [OD] Orth-Dion: Dion keeps a
 * residual buffer that the gradient is added to).
 *
 *   mode OUO_MOMENTUM_EMA:   M <- mu * M + G      (fp32 fused multiply-add)
 *   mode OUO_MOMENTUM_ACCUM: M <- M + G
 *
 * M[i]: fp32 momentum, updated in place.  G[i]: gradient of the same shape,
 * dtype g_dtype.  row_sqnorm (optional device double*, may be NULL): receives
 * for every row of every matrix, matrices in batch order, the float64 sum of
 * the squares of the updated fp32 row (length = sum of rows).  Rows are
 * summed in a fixed order, so the result is deterministic.
 */
int dion_momentum_update(const ouo_mat* M, const ouo_mat* G, int nmat,
                         int g_dtype, float mu, int mode, double* row_sqnorm,
                         void* stream);

/*
 * dion3_num_selected -- k = ceil(rho * rows) clamped to [1, rows]: the number
 * of rows the Dion3 rule keeps ([D3s] 核心模块: e.g. 1/8 of the rows).
 * Returns -1 for rows < 1 or rho outside (0, 1].
 */
int64_t dion3_num_selected(int64_t rows, double rho);

/*
 * dion3_select_rows -- the Dion3 rule ([D3] Abstract: orthogonalize only a
 * fraction of the momentum matrix's rows; [D3s] 核心模块: a fraction such as
 * 1/8, the other rows keep the plain momentum, with error feedback).
 *
 * For matrix i with m_i rows and k_i = dion3_num_selected(m_i, rho):
 *   S_i   = the k_i rows with the largest row_sqnorm, equal keys taken in
 *           ascending row order, listed in ascending row order (exact and
 *           deterministic: keys are compared as float64 bit patterns).
 *   idx   (device int32, length sum k_i): S_i of matrix i at offset
 *           sum_{j<i} k_j.
 *   X0[i] (k_i x n_i, dtype x0_dtype): B_i[S_i] / (||B_i[S_i]||_F + eps), the
 *           Frobenius norm taken from the float64 keys.
 *   x0_scale (device float, length nmat): the factor 1 / (||.||_F + eps).
 *   ef_mode OUO_EF_ROWS: B_i[S_i] <- mu * B_i[S_i] afterwards (the kept
 *           rows' orthogonalized share leaves the buffer; other rows keep B).
 * B[i]: fp32 momentum buffer (read; written on kept rows under EF).
 * row_sqnorm: device double*, as produced by dion_momentum_update.
 */
int dion3_select_rows(const ouo_mat* B, const double* row_sqnorm, int nmat,
                      double rho, int ef_mode, float mu, float eps,
                      int32_t* idx, const ouo_mat* X0, int x0_dtype,
                      float* x0_scale, void* stream);

/*
 * ns_orthogonalize -- Muon's quintic Newton-Schulz ([D3] Abstract: the
 * cubic-time Newton-Schulz orthogonalization step of Muon):
 *   X0 = X / (||X||_F + eps)  (if p->normalize), transposed if rows > cols;
 *   iters times: A = X X^T;  X <- a' X + (b' A + c' A^2) X
 * with (a', b', c') = (a / s, b / s^3, c / s^5), s = p->safety.
 * X[i] (dtype x_dtype) is read; O[i] (same shape, dtype o_dtype) is written;
 * O may alias X.  ws / ws_bytes: device workspace of at least
 * ns_workspace_bytes(...) bytes (256-byte aligned).
 */
size_t ns_workspace_bytes(const ouo_mat* X, int nmat, const ouo_ns_params* p);
int ns_orthogonalize(const ouo_mat* X, int x_dtype, const ouo_mat* O,
                     int o_dtype, int nmat, const ouo_ns_params* p, void* ws,
                     size_t ws_bytes, int* dev_status, void* stream);

/*
 * gram_ns_orthogonalize -- Gram Newton-Schulz ([D3] Abstract; [D3s] 核心洞察,
 * 核心模块: iterate on the small symmetric Gram matrix, stabilized by
 * restarts and a safety factor; 局限: restarts repair spurious negative
 * eigenvalues and eigenvector drift).  With X0 as above:
 *   A = X0 X0^T, Q = I;  for t = 1..iters:
 *     H = a' I + b' A + c' A^2;  Q <- H Q;
 *     if t < iters: restart after t ? (X0 <- Q X0, A <- X0 X0^T, Q <- I)
 *                                   : A <- H (H A)
 *   O = Q X0
 * Equal to ns_orthogonalize in exact arithmetic.  Symmetric k x k products
 * compute only upper-triangle tiles and mirror them.  Arguments as for
 * ns_orthogonalize; restarts from p->restart_after.
 */
size_t gram_ns_workspace_bytes(const ouo_mat* X, int nmat,
                               const ouo_ns_params* p);
int gram_ns_orthogonalize(const ouo_mat* X, int x_dtype, const ouo_mat* O,
                          int o_dtype, int nmat, const ouo_ns_params* p,
                          void* ws, size_t ws_bytes, int* dev_status,
                          void* stream);

/*
 * gram_ns_orthogonalize_noalloc -- gram_ns_orthogonalize for callers that
 * cannot allocate device memory (no counterpart on the pages: it is a
 * service of this library).  Such callers include plugins running inside a
 * host framework whose own pool owns all device memory, and latency-critical
 * paths that must not pay cudaMalloc's implicit synchronization; they cannot
 * provide the workspace gram_ns_orthogonalize needs.
 *
 * Same arguments and results as gram_ns_orthogonalize minus the workspace:
 * the library uses a fixed scratch array of OUO_NOALLOC_SCRATCH_BYTES bytes
 * in its own device image instead, and allocates nothing (no cudaMalloc, no
 * allocating library routine).  Every GPU that loads this part of the
 * library holds the array until the process exits.
 *   - A batch whose gram_ns_workspace_bytes() exceeds the array is refused
 *     with OUO_ERR_WORKSPACE before anything is launched.
 *   - Every call looks up the array's device address on the current device
 *     (no allocation).  The first call on a device also loads the library's
 *     device image there; make that first call before any stream capture.
 *     The address is never cached, so a device reset (which reloads the
 *     image, possibly elsewhere) is safe.
 *   - Arguments are checked as gram_ns_orthogonalize checks them (bad ones
 *     give OUO_ERR_INVALID_ARG) before the scratch size is computed.
 *   - Every call shares the array; calls whose kernels overlap on the GPU
 *     (e.g. on two unordered streams) race on it.  Each call overwrites what
 *     it reads, so no state carries over between calls.
 */
int gram_ns_orthogonalize_noalloc(const ouo_mat* X, int x_dtype,
                                  const ouo_mat* O, int o_dtype, int nmat,
                                  const ouo_ns_params* p, int* dev_status,
                                  void* stream);

/*
 * apply_update -- the weight update that ends the step ([D3s] 输入输出流程:
 * "update weights"):
 *   W[i][r] <- (1 - lr * wd) * W[i][r] - lr * scale[i] * O[i][j]
 * for r = idx[off_i + j] (Dion3 kept rows; O[i] is k_i x n_i) or, when idx
 * is NULL, r = j over all rows (O[i] has W[i]'s shape).  W dtype w_dtype,
 * O dtype o_dtype, fp32 arithmetic.  scale: host float array of nmat
 * per-matrix factors, or NULL for 1.
 */
int apply_update(const ouo_mat* W, int w_dtype, const ouo_mat* O, int o_dtype,
                 const int32_t* idx, int nmat, float lr, const float* scale,
                 float wd, void* stream);

/*
 * dion_lowrank_step -- one Dion / Orth-Dion step per matrix ([OD] Problem
 * Statement: rank-r factors from a single power-iteration step; The
 * Geometric Insight: Dion's column normalization; Orth-Dion: QR of the right
 * factor instead, same residual buffer; Theoretical Contributions: the
 * error-feedback coefficient beta; [D1] Technical details):
 *   B = M + G;  P = orth(B Q_prev);  R = B^T P;
 *   Q_new = ColNorm(R) or orth(R);   M <- beta B - (beta - mu) P R^T;
 *   W <- (1 - lr wd) W - lr scale P Q_new^T;  Q_state <- Q_new
 * orth() is the QR factor with positive R diagonal (CholeskyQR2 at fp32
 * accuracy: Gram matrices and solves as split-tf32 tensor-core products,
 * the Cholesky factor and its inverse in fp32).
 * ColNorm(R)_j = R_j / (||R_j|| + eps).
 * M[i]: fp32 m x n buffer (in/out).  G[i]: m x n, dtype g_dtype.
 * Q_state[i]: fp32, stored TRANSPOSED as r x n (row c = column c of Q),
 * in/out; the caller initializes it with orthonormal rows.
 * W[i]: m x n, dtype w_dtype (in/out).  scale: host float[nmat] or NULL.
 * ws / ws_bytes: at least dion_workspace_bytes(...) bytes, 256-byte aligned
 * (about 4 to 5 r (m + n) floats per matrix: the projections and their
 * bf16 copies, the CholeskyQR buffers, Gram and split-K partials; 12.9 GB
 * for the 224-matrix Llama-3-8B-shaped set at r = 256).  The workspace holds no
 * state between calls, except in the row-sharded step below.
 * Matrices of the same (rows, cols, rank) run as one group; when their M,
 * G, Q_state and W each sit evenly strided in memory, every stage of the
 * group is one descriptor of a grouped launch, and a matrix gives the same
 * bits alone as in any batch.
 */
size_t dion_workspace_bytes(const ouo_mat* M, int nmat,
                            const ouo_dion_params* p);
int dion_lowrank_step(const ouo_mat* M, const ouo_mat* G, int g_dtype,
                      const ouo_mat* Q_state, const ouo_mat* W, int w_dtype,
                      int nmat, const ouo_dion_params* p, const float* scale,
                      void* ws, size_t ws_bytes, int* dev_status,
                      void* stream);

/*
 * Per-matrix working ranks ([OD] Ada-Orth-Dion: the working rank of every
 * layer is adjusted to its gradient spectrum).
 *
 * Ragged ranks: with p->rank == 0, dion_lowrank_step and
 * dion_lowrank_step_stats give matrix i the rank r_i = Q_state[i].rows
 * (1 <= r_i <= min(rows, cols)); a nonzero p->rank must equal every
 * Q_state[i].rows as before.  dion_workspace_bytes_ranks sizes the
 * workspace for per-matrix ranks (ranks: host int[nmat]); it returns 0 for
 * invalid arguments.
 *
 * dion_lowrank_step_stats -- dion_lowrank_step that also writes, for every
 * matrix, the Euclidean norms of the r_i rows of R^T = P^T B (the columns of
 * R: the power iteration's estimates of B's leading singular values) to
 * sigma, a device float array of sum_i r_i values, matrix i's after those
 * of the matrices before it.  sigma == NULL is dion_lowrank_step.
 *
 * dion_effective_rank -- per matrix, exp(-sum_j p_j ln p_j) with
 * p_j = sigma_j^2 / sum_k sigma_k^2: the exponential of the Shannon entropy of
 * the energy the rank-r_i factors capture, between 1 (one direction holds
 * all of it) and r_i (evenly spread).  The pages name "a lightweight
 * entropy-based estimator derived from the power iteration factors" without
 * defining it; this is that reading (the effective rank of the estimated
 * spectrum).  sigma: device float[sum r_i] laid out as above; ranks: host
 * int[nmat]; erank: device float[nmat]; all-zero sigma gives 0.  Float64
 * sums in a fixed order.  Asynchronous on `stream`.
 */
size_t dion_workspace_bytes_ranks(const ouo_mat* M, const int* ranks, int nmat,
                                  const ouo_dion_params* p);
int dion_lowrank_step_stats(const ouo_mat* M, const ouo_mat* G, int g_dtype,
                            const ouo_mat* Q_state, const ouo_mat* W,
                            int w_dtype, int nmat, const ouo_dion_params* p,
                            const float* scale, void* ws, size_t ws_bytes,
                            float* sigma, int* dev_status, void* stream);
int dion_effective_rank(const float* sigma, const int* ranks, int nmat,
                        float* erank, void* stream);

/*
 * Row-sharded Dion / Orth-Dion step: the power iteration with the rows of
 * every matrix spread over ranks, the form Dion takes when weights are
 * sharded ([OD] Problem Statement: Dion's communication is the rank-r
 * factors; [D1] Technical details).  Each rank holds a block of rows of M, G
 * and W of each matrix (m_i local rows, any split) and a full copy of
 * Q_state.  A step is four calls on one workspace; after each of the first
 * three the caller sums the float buffer `red` over the ranks in place (an
 * all-reduce) before the next call:
 *   dion_shard_project  B = M + G; P^T = Q^T B^T (r x m_i); red = P^T P.
 *   dion_shard_orth1    red = sum of P^T P: P^T <- L^-1 P^T (CholeskyQR);
 *                       red = P^T P.
 *   dion_shard_orth2    red = sum: P^T <- L^-1 P^T; red = P^T B (r x n).
 *   dion_shard_update   red = sum = R^T: Q_new^T = ColNorm or orth of the rows
 *                       of R^T; M <- beta B - (beta - mu) P R^T;
 *                       W <- (1 - lr wd) W - lr scale P Q_new^T;
 *                       Q_state <- Q_new^T.
 * With one rank (nothing summed) the four calls compute what
 * dion_lowrank_step computes, bit for bit (except for the trace behind a
 * shifted CholeskyQR retry).
 * red: device float[dion_shard_red_floats(...)]; matrix i's block follows
 * those of the matrices before it (256-byte aligned), r_i x r_i packed for
 * P^T P and r_i x n_i (row pitch n_i rounded up to 4) for P^T B.
 * rows_total: host int64[nmat], every matrix's global row count (the
 * shifted-CholeskyQR retry uses it).  ws: dion_shard_workspace_bytes(...)
 * bytes, the same buffer for the four calls of a step (P^T lives in it
 * between them).  Ranks as in dion_lowrank_step: p->rank, or 0 for
 * Q_state[i].rows.  The size queries return 0 for invalid arguments.
 */
size_t dion_shard_workspace_bytes(const ouo_mat* M, const ouo_mat* Q_state,
                                  int nmat, const ouo_dion_params* p);
size_t dion_shard_red_floats(const ouo_mat* M, const ouo_mat* Q_state, int nmat,
                             const ouo_dion_params* p);
int dion_shard_project(const ouo_mat* M, const ouo_mat* G, int g_dtype,
                       const ouo_mat* Q_state, int nmat,
                       const ouo_dion_params* p, void* ws, size_t ws_bytes,
                       float* red, int* dev_status, void* stream);
int dion_shard_orth1(const ouo_mat* M, const ouo_mat* Q_state, int nmat,
                     const ouo_dion_params* p, const int64_t* rows_total,
                     void* ws, size_t ws_bytes, float* red, int* dev_status,
                     void* stream);
int dion_shard_orth2(const ouo_mat* M, const ouo_mat* Q_state, int nmat,
                     const ouo_dion_params* p, const int64_t* rows_total,
                     void* ws, size_t ws_bytes, float* red, int* dev_status,
                     void* stream);
int dion_shard_update(const ouo_mat* M, const ouo_mat* Q_state,
                      const ouo_mat* W, int w_dtype, int nmat,
                      const ouo_dion_params* p, const float* scale, void* ws,
                      size_t ws_bytes, float* red, int* dev_status,
                      void* stream);

#ifdef __cplusplus
}
#endif

#endif /* ORTHOUPD_H */
