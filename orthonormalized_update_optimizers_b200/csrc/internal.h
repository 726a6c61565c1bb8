// Internal interfaces between the translation units of liborthoupd.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <vector>

#include "common.cuh"

namespace ouo {

// ------------------------------------------------------------ batch tables
// Launch-time tables are passed to kernels by value (kernel parameters), so
// a call needs no device allocation and no host-to-device copy.
constexpr int kChunk = 128;  // matrices per launch; larger batches loop

struct MatRef {
  void* p;
  int64_t ld;
};

// Equal-shape matrices of one call, in batch order.
struct Group {
  int64_t rows, cols;
  std::vector<int> members;  // indices into the caller's batch
};

std::vector<Group> group_by_shape(const ouo_mat* mats, int nmat);

// Checks a caller batch: non-null pointers aligned to the element size,
// rows, cols >= 1, ld >= cols.  Returns OUO_OK or OUO_ERR_INVALID_ARG.
int validate_mats(const ouo_mat* mats, int nmat, int dtype, const char* name);
int validate_dtype(int dtype, const char* name);
// True when every row starts on a 16-byte boundary (vector access allowed).
bool vec16(const ouo_mat& m, int dtype);
// Same shapes, element for element.
int validate_same_shapes(const ouo_mat* a, const ouo_mat* b, int nmat,
                         const char* na, const char* nb);

// --------------------------------------------------------- workspace tensors
// A batch of `nb` equal-shape matrices laid out in library workspace as
// [nb][rows][ld] with element size 2 (bf16) or 4 (fp32).
struct Buf {
  char* p = nullptr;
  int dtype = OUO_F32;
  int64_t rows = 0, cols = 0, ld = 0, stride = 0;  // ld, stride in elements
  int64_t nb = 0;
};

// Carves consecutive 256-byte-aligned buffers out of a workspace.
struct Arena {
  char* base;
  size_t cap, used = 0;
  bool measuring;  // only count bytes
  Buf take(int dtype, int64_t nb, int64_t rows, int64_t cols);
};

// C = alpha * A op(B) + beta * C0 + gamma * I, for each of nb matrices.
//   A: M x K, K-major (row i holds A[i, :]).
//   B: K-major: an N x K buffer (row j holds B[:, j]);
//      MN-major (b_mn = 1): a K x N buffer (row l holds B[l, :]).
//   C0 (optional) is M x N.  When tri = 1 the output is symmetric (M = N):
//   only tiles on or above the diagonal are computed, each element with
//   j >= i is written to (i, j) and (j, i), and C0 is read at (j, i), which
//   requires C0 symmetric.
//   Outputs: out_f32 (optionally rounded to tf32) and / or out_bf16.
struct GemmDesc {
  int64_t M = 0, N = 0, K = 0, nb = 0;
  Buf A, B;
  int b_mn = 0;
  float alpha = 1.f, beta = 0.f, gamma = 0.f;
  Buf C0;
  bool has_c0 = false;
  Buf out_f32;
  bool has_f32 = false;
  bool round_tf32 = false;
  Buf out_bf16;
  bool has_bf16 = false;
  bool tri = false;
  // When non-empty, matrix b of the batch is written to direct[b] (caller
  // memory, element type direct_dtype, rows 16-byte aligned) instead of to
  // out_f32 / out_bf16.  Tensor-core path only.
  std::vector<MatRef> direct;
  int direct_dtype = OUO_BF16;
  // With direct outputs: C0 is the output matrix itself (in-place update
  // out = alpha * A op(B) + beta * out).  Non-symmetric outputs only.
  bool c0_from_out = false;
  // Half-stored symmetric matrices (tf32 / bf16 tensor-core path, CTA-pair
  // tiles).  A symmetric matrix is "upper-stored" when every 256 x 256 block
  // on or above the block diagonal holds its values (diagonal blocks in
  // full) and the blocks below may hold anything.
  //   sym_half:  the symmetric output is written upper-stored (off-diagonal
  //              tiles are not mirrored);
  //   a_sym / b_sym: A / B (K-major, symmetric) are upper-stored: K blocks
  //              left of the diagonal are read from the transposed block;
  //   c0_upper:  the symmetric C0 is upper-stored (read at (i, j), j >= i).
  bool sym_half = false, a_sym = false, b_sym = false, c0_upper = false;
  // Per-matrix alpha of direct outputs (one value per batch matrix); empty:
  // `alpha` for every matrix.
  std::vector<float> direct_alpha;
  // Split-K (tensor-core path, one workspace output, no C0, non-symmetric):
  // the K range is cut into up to `ksplit` equal ranges of whole K blocks;
  // range s of matrix b is written to output matrix b * ksplit' + s, where
  // ksplit' = gemm_ksplit_used(K, ksplit, dtype) <= ksplit (no empty range).
  // The output buffer holds nb * ksplit' matrices; the caller sums them.
  int ksplit = 1;
  // Tile shape (CTA pair or not, 128 or 256 columns) chosen for this
  // descriptor alone instead of for the whole grouped launch, so that a
  // matrix is computed the same way whatever it is batched with.
  bool per_desc_tiles = false;
  // With per_desc_tiles: CTA-pair tiles also for an MN-major B (by default
  // only K-major B takes them).  Pairs halve the operand bytes per output
  // element, which is what a short-K GEMM with an in-place C0 runs out of.
  bool pair_mn = false;
  // Split-tf32 passes (tf32 operands, no symmetric operands): the K range is
  // run `npass` times (1 to 3) into one accumulator; in pass q the A
  // operand is A2 instead of A when bit q of a_lo is set (A3 for a_lo2),
  // and B2 instead of B for b_lo.  With A2 / B2 holding the residuals
  // x - tf32(x) of A / B, the passes (A, B), (A, B2), (A2, B) give the
  // product to about fp32 accuracy (the tensor core reads A and B truncated
  // to tf32; the residual-residual term, 2^-20 relative, is left out).
  // A2, A3 / B2 have the shapes, leading dimensions and batch strides of
  // A / B.
  int npass = 1;
  Buf A2, B2, A3;
  int a_lo = 0, b_lo = 0, a_lo2 = 0;
};

// Number of K ranges a split-K GEMM of depth K over `dtype` operands
// (run `npass` times) actually uses for a requested `ksplit` (every range
// non-empty).
int gemm_ksplit_used(int64_t K, int ksplit, int dtype, int npass = 1);

// Whether K-major tensor-core GEMMs with more than 128 output rows and
// columns run on CTA-pair tiles (OUO_CTA_PAIR, default on); upper-stored
// symmetric matrices need them.
bool cta_pairs_enabled();

// Tensor-core GEMM (tcgen05 / TMEM / TMA).  A and B are both bf16
// (kind::f16) or both fp32 read as tf32 (kind::tf32).
int gemm_umma(const GemmDesc& g, cudaStream_t stream, int* status);
// Several equal-kind GEMMs (same operand types, majorness, symmetry,
// epilogue coefficients and output kinds; any sizes) in as few launches as
// possible: one persistent launch covers up to 6 batch segments.
int gemm_umma_grouped(const std::vector<GemmDesc>& gs, cudaStream_t stream,
                      int* status);
// Opt-in event timing of tensor-core GEMM launches (see ouo_timing_enable).
int gemm_timing_enable(int on);
int gemm_timing_read(int kind, int* launches, double* total_ms, double* flops);
// CUDA-core fp32 GEMM for the fp32 precision path.
int gemm_simt(const GemmDesc& g, cudaStream_t stream);

// Argument checks of ns_orthogonalize / gram_ns_orthogonalize (everything
// but the workspace): OUO_OK or the error code, with the message set.
int ns_check_call(const ouo_mat* X, int x_dtype, const ouo_mat* O, int o_dtype,
                  int nmat, const ouo_ns_params* p, int* dev_status);

// ----------------------------------------------------------- other kernels
struct PrepArgs;  // defined in nsprep.cu

// X (caller's, dtype x_dtype) -> workspace X0 (bf16 or fp32), multiplied by
// 1 / (||X||_F + eps) when normalize, transposed when transpose.
int ns_prep(const ouo_mat* X, int x_dtype, const Group& grp, bool transpose,
            bool normalize, float eps, const Buf& x0, double* scratch_sq,
            cudaStream_t stream);
// workspace Y (nb x rows x cols) -> caller's O (dtype o_dtype), transposed
// back when transpose.
int ns_writeout(const Buf& y, const ouo_mat* O, int o_dtype, const Group& grp,
                bool transpose, cudaStream_t stream);
// Fill nb identity matrices (fp32 and / or bf16 copies).
int fill_identity(const Buf& q, cudaStream_t stream);

// --------------------------------------------------- batched CholeskyQR
// One r x L block of rows to orthonormalize (cholqr.cu): Gram matrix S =
// X X^T, Cholesky S = L L^T, Y = L^-1 X (rows orthonormal, the QR factor
// with a positive diagonal).  Every pointer is device memory.
struct CholQrJob {
  const float* X = nullptr;  // r x L, row pitch ldx (16-byte rows preferred)
  int64_t ldx = 0;
  int r = 0;
  int64_t L = 0;
  float* Xlo = nullptr;      // 2 (X - tf32(X)), r x L, row pitch ldx: written
                             // by the Gram, read again by the solve
  float* gpart = nullptr;    // Gram partials, cholqr_gram_part_floats(r, L)
  float* S = nullptr;        // summed Gram, r x r, full symmetric storage
  float* Lb = nullptr;       // R x R (R = r rounded up to 32), ld R: the
                             // strictly lower 32 x 32 blocks of L
  const float* Dd = nullptr; // R x R, ld R: D_i = L_ii^-1 on the diagonal
                             // blocks (nullptr: they are in Lb)
  float* Z = nullptr;        // cholqr_z_floats(r): L^-1 in three planes
  float* Y = nullptr;        // L^-1 X, r x L (apart from X)
  int64_t ldy = 0;
  float* Y2 = nullptr;       // optional copy of Y
  int64_t ldy2 = 0;
  float* Yt = nullptr;       // optional transpose of Y, L x r
  int64_t ldyt = 0;
  uint16_t* Ytb = nullptr;   // optional bf16 copy of the transpose, L x r
  int64_t ldytb = 0;
};
// Split-K ranges of the tensor-core Gram of an r x L block, and the floats
// of its partials ([ranges][r][pitch4(r)]).  A run of jobs whose X, Xlo and
// gpart are evenly strided (X and Xlo by the same step, gpart by
// cholqr_gram_part_floats) is computed by one GEMM descriptor.
int cholqr_gram_ksplit(int r, int64_t L);
int64_t cholqr_gram_part_floats(int r, int64_t L);
// Residuals, split-tf32 Gram partials on the tensor cores and their
// float64 sum S (full symmetric), for every job.  X rows and Xlo on 16-byte
// boundaries.
int cholqr_gram(const std::vector<CholQrJob>& jobs, int* status, cudaStream_t s);
// Whether the one-CTA Cholesky takes rank r (1 <= r <= 256).
bool cholqr_small_rank(int r);
// S -> Lb (strictly lower blocks of L and D_i on the diagonal blocks), one
// CTA per job, r <= 256; breakdown after the shifted retry sets
// OUO_STATUS_BREAKDOWN and writes the identity.
int cholqr_factor(const std::vector<CholQrJob>& jobs, int* status, cudaStream_t s);
// Floats of a job's Z (three R x R planes, R = r rounded up to 32).
size_t cholqr_z_floats(int r);
// Y = L^-1 X (and Y2, Yt, Ytb) for every job, r <= 1024: Z = L^-1, then
// the product on the tensor cores in split-tf32 passes, reading the
// residuals the job's Gram left in Xlo.  A run of jobs whose X, Xlo, Y and
// Z are evenly strided (X and Xlo by the same step, Z by cholqr_z_floats)
// is one GEMM descriptor.
int cholqr_apply(const std::vector<CholQrJob>& jobs, int* status, cudaStream_t s);

// Rows of the sum of `ks` partial matrices (sp floats apart, row pitch
// ldp), with optional row norms (float64, fixed order) and normalized rows
// v / (||v|| + eps).
struct RowsJob {
  const float* part = nullptr;
  int64_t ldp = 0, sp = 0;
  int ks = 1;
  int64_t rows = 0, n = 0;
  float* out = nullptr;      // optional summed rows
  int64_t ldo = 0;
  uint16_t* outb = nullptr;  // optional bf16 copy of the summed rows
  int64_t ldob = 0;
  float* sigma = nullptr;    // optional row norms
  float* qn = nullptr;       // optional normalized rows
  int64_t ldq = 0;
  float* q2 = nullptr;       // optional copy of qn
  int64_t ldq2 = 0;
};
int rows_reduce(const std::vector<RowsJob>& jobs, float eps, cudaStream_t s);

// Cooperative blocked Cholesky for ranks above 256 (chol.cu): S = sum of
// `splits` partial r x r Gram matrices in upper storage.  Leaves the
// strictly lower blocks of L in S (R x R, ld R, R = r rounded up to 32) and
// the inverted diagonal blocks in the diagonal blocks of Linv.  ctl is
// chol_blocked_ctl_bytes(r) bytes of 8-byte aligned scratch.
size_t chol_blocked_ctl_bytes(int r);
int chol_blocked(const float* part, int splits, int r, int64_t L, float* S,
                 float* Linv, void* ctl, int* status, cudaStream_t stream);
int convert_buf(const Buf& src, const Buf& dst, cudaStream_t stream);

}  // namespace ouo
