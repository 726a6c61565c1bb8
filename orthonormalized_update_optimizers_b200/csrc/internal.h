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
};

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

// Blocked Cholesky + triangular inverse (chol.cu): S = sum of `splits`
// partial r x r Gram matrices; writes L^-1 into Linv (R x R, ld R, R = r
// rounded up to 32).  S is R x R scratch (ld R); ctl is
// chol_blocked_ctl_bytes(r) bytes of 8-byte aligned scratch.
size_t chol_blocked_ctl_bytes(int r);
int chol_blocked(const float* part, int splits, int r, int64_t L, float* S,
                 float* Linv, void* ctl, int* status, cudaStream_t stream);
// The same factorization and inverse in one CTA with the blocks in shared
// memory, for 1 <= r <= 256 (chol_smem_fits), from one summed r x r matrix
// S (ld r); no scratch besides Linv.
bool chol_smem_fits(int r);
int chol_smem(const float* S, int r, int64_t L, float* Linv, int* status,
              cudaStream_t stream);
int convert_buf(const Buf& src, const Buf& dst, cudaStream_t stream);

}  // namespace ouo
