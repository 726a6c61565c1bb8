// Dion / Orth-Dion low-rank step.
//
// Source: "Orth-Dion: Eliminating Geometric Mismatch in Distributed Low-Rank
// Spectral Optimization" -- Problem Statement (rank-r factors from a single
// power-iteration step per optimizer step), The Geometric Insight (Dion's
// column normalization of the right factor), Orth-Dion (QR of the right
// factor instead, same power iteration and residual buffer), Theoretical
// Contributions (error-feedback coefficient beta); "Dion: The Distributed
// Orthonormal Update Revolution Is Here", Technical details.
//
// Per matrix (B is the momentum buffer after B = M + G, m x n fp32):
//   Pt = Qt B^T                      (r x m; Qt = Q_prev^T is the state)
//   Pt <- rows orthonormalized       (CholeskyQR2: P = orth(B Q_prev))
//   Rt = Pt B                        (r x n; R = B^T P)
//   Qt_new = rows of Rt normalized   (Dion)  or  rows orthonormalized (Orth-Dion)
//   M <- beta B - (beta - mu) P Rt   (residual buffer / error feedback)
//   W <- (1 - lr wd) W - lr s P Qt_new
//   state <- Qt_new
// Working in the transposed layouts keeps every large product on the
// tcgen05 GEMM (tf32 operands, fp32 accumulation) with K-major A.  The
// orthonormalization works on r x L row blocks X: S = X X^T in fp32 (split
// over L, partial sums added in float64 in a fixed order), S = L L^T by a
// one-CTA Cholesky (r <= 64) or the blocked cooperative Cholesky of chol.cu
// (wider ranks), L inverted, X <- L^-1 X (rows orthonormal; the
// implied R = L^T has a positive diagonal, the unique QR).  Two passes
// (CholeskyQR2).  A failed pivot retries with the shift of shifted
// CholeskyQR (11 (L r + r (r + 1)) u ||X||_F^2); a second failure sets
// OUO_STATUS_BREAKDOWN.
#include <cmath>
#include <cstdlib>

#include "internal.h"

namespace ouo {
namespace {

// --------------------------------------------------------------- Gram S
constexpr int kGT = 32;  // Gram tile

struct GramArgs {
  const float* X;
  int64_t ld;
  int r;
  int64_t L, chunk;
  float* part;  // [splits][r][r]
  int tiles;    // ceil(r / 32)
};

// grid.x: upper tile pairs (ti <= tj), grid.y: split of the L range.
__global__ void __launch_bounds__(256) gram_partial_kernel(const GramArgs a) {
  __shared__ float xi[kGT][kGT + 1];
  __shared__ float xj[kGT][kGT + 1];
  int t = blockIdx.x, ti = 0;
  while (t >= a.tiles - ti) { t -= a.tiles - ti; ++ti; }
  const int tj = ti + t;
  const int64_t l0 = (int64_t)blockIdx.y * a.chunk;
  const int64_t l1 = l0 + a.chunk < a.L ? l0 + a.chunk : a.L;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int64_t k0 = l0; k0 < l1; k0 += kGT) {
    for (int e = threadIdx.x; e < kGT * kGT; e += 256) {
      const int rr = e >> 5, kk = e & 31;
      const int64_t k = k0 + kk;
      const int ri = ti * kGT + rr, rj = tj * kGT + rr;
      xi[kk][rr] = (ri < a.r && k < l1) ? a.X[ri * a.ld + k] : 0.f;
      xj[kk][rr] = (rj < a.r && k < l1) ? a.X[rj * a.ld + k] : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < kGT; ++kk) {
      const float bj = xj[kk][tx];
#pragma unroll
      for (int u = 0; u < 4; ++u) acc[u] = __fmaf_rn(xi[kk][ty + 8 * u], bj, acc[u]);
    }
    __syncthreads();
  }
  float* part = a.part + (size_t)blockIdx.y * a.r * a.r;
  const int j = tj * kGT + tx;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int i = ti * kGT + ty + 8 * u;
    if (i < a.r && j < a.r) {
      part[(size_t)i * a.r + j] = acc[u];
      part[(size_t)j * a.r + i] = acc[u];
    }
  }
}

// ---------------------------------------------------- Cholesky + inverse
// One CTA, ranks up to 128 (by default up to 64; larger ones use the
// blocked kernel in chol.cu).
// S is summed from the partials in float64 (fixed order) and kept as a
// packed lower triangle (fp32) in shared memory.
// Cholesky S = L L^T in place, then L^-1 in place, then written as a full
// lower-triangular r x r row-major fp32 matrix.
__device__ __forceinline__ int tri_at(int i, int j) {  // j <= i
  return i * (i + 1) / 2 + j;
}

struct CholArgs {
  const float* part;
  int splits;
  int r;
  int64_t L;        // length of the rows of X (for the shift)
  float* Linv;      // r x r out, row pitch ldl
  int64_t ldl;
  int* status;
};

__device__ void chol_load(const CholArgs& a, float* tri, float shift) {
  const int n = a.r * (a.r + 1) / 2;
  for (int e = threadIdx.x; e < n; e += blockDim.x) {
    // invert e -> (i, j), j <= i
    int i = (int)((sqrtf(8.f * (float)e + 1.f) - 1.f) * 0.5f);
    while (tri_at(i + 1, 0) <= e) ++i;
    while (tri_at(i, 0) > e) --i;
    const int j = e - tri_at(i, 0);
    double s = 0.0;
    for (int p = 0; p < a.splits; ++p)
      s += (double)a.part[(size_t)p * a.r * a.r + (size_t)i * a.r + j];
    if (i == j) s += (double)shift;
    tri[e] = (float)s;
  }
  __syncthreads();
}

// Right-looking Cholesky in place; returns false if a pivot is not positive.
__device__ bool chol_factor(const CholArgs& a, float* tri, int* s_fail) {
  const int r = a.r;
  if (threadIdx.x == 0) *s_fail = 0;
  __syncthreads();
  for (int k = 0; k < r; ++k) {
    const float piv = tri[tri_at(k, k)];
    if (!(piv > 0.f) || !isfinite(piv)) {
      if (threadIdx.x == 0) *s_fail = 1;
      __syncthreads();
      return false;
    }
    const float d = sqrtf(piv);
    const float inv = 1.0f / d;
    __syncthreads();
    if (threadIdx.x == 0) tri[tri_at(k, k)] = d;
    for (int i = k + 1 + threadIdx.x; i < r; i += blockDim.x) tri[tri_at(i, k)] *= inv;
    __syncthreads();
    // trailing update S[i][j] -= L[i][k] L[j][k], k < j <= i
    const int m = r - k - 1;
    const int cnt = m * (m + 1) / 2;
    for (int e = threadIdx.x; e < cnt; e += blockDim.x) {
      int ii = (int)((sqrtf(8.f * (float)e + 1.f) - 1.f) * 0.5f);
      while ((ii + 1) * (ii + 2) / 2 <= e) ++ii;
      while (ii * (ii + 1) / 2 > e) --ii;
      const int jj = e - ii * (ii + 1) / 2;
      const int i = k + 1 + ii, j = k + 1 + jj;
      tri[tri_at(i, j)] -= tri[tri_at(i, k)] * tri[tri_at(j, k)];
    }
    __syncthreads();
  }
  return true;
}

// In-place inverse of the packed lower-triangular L (column j from the
// last to the first: L^-1[j+1:, j] = -L^-1[j+1:, j+1:] L[j+1:, j] / L[j][j]).
__device__ void tri_invert(const CholArgs& a, float* tri, float* tmp) {
  const int r = a.r;
  for (int j = r - 1; j >= 0; --j) {
    const float djj = 1.0f / tri[tri_at(j, j)];
    // tmp = L[j+1:, j] (original column)
    for (int i = j + 1 + threadIdx.x; i < r; i += blockDim.x) tmp[i] = tri[tri_at(i, j)];
    __syncthreads();
    for (int i = j + 1 + threadIdx.x; i < r; i += blockDim.x) {
      float s = 0.f;
      for (int k = j + 1; k <= i; ++k) s = __fmaf_rn(tri[tri_at(i, k)], tmp[k], s);
      tri[tri_at(i, j)] = -s * djj;
    }
    __syncthreads();
    if (threadIdx.x == 0) tri[tri_at(j, j)] = djj;
    __syncthreads();
  }
}

__global__ void __launch_bounds__(1024) chol_inv_kernel(const CholArgs a) {
  extern __shared__ float sm[];
  __shared__ int s_fail;
  const int r = a.r;
  float* tri = sm;
  float* tmp = sm + r * (r + 1) / 2;
  chol_load(a, tri, 0.f);
  if (!chol_factor(a, tri, &s_fail)) {
    // shifted CholeskyQR: 11 (L r + r (r + 1)) u ||X||_F^2, ||X||_F^2 = tr S
    __shared__ float s_trace;
    __syncthreads();
    if (threadIdx.x == 0) {
      double tr = 0.0;
      for (int i = 0; i < r; ++i)
        for (int p = 0; p < a.splits; ++p)
          tr += (double)a.part[(size_t)p * r * r + (size_t)i * r + i];
      const double u = 5.9604644775390625e-8;  // 2^-24
      s_trace = (float)(11.0 * ((double)a.L * r + (double)r * (r + 1)) * u * tr);
    }
    __syncthreads();
    chol_load(a, tri, s_trace > 0.f ? s_trace : 1e-30f);
    if (!chol_factor(a, tri, &s_fail)) {
      if (threadIdx.x == 0) report_status(a.status, OUO_STATUS_BREAKDOWN);
      // keep going with unit pivots where the factorization failed
      __syncthreads();
      for (int e = threadIdx.x; e < r * (r + 1) / 2; e += blockDim.x) tri[e] = 0.f;
      __syncthreads();
      for (int i = threadIdx.x; i < r; i += blockDim.x) tri[tri_at(i, i)] = 1.f;
      __syncthreads();
    }
  }
  tri_invert(a, tri, tmp);
  for (int e = threadIdx.x; e < r * r; e += blockDim.x) {
    const int i = e / r, j = e - (e / r) * r;
    a.Linv[(int64_t)i * a.ldl + j] = j <= i ? tri[tri_at(i, j)] : 0.f;
  }
}

// ------------------------------------------------------ row normalization
// Q[c][:] = R[c][:] / (||R[c][:]||_2 + eps); one block per row, float64
// sum of squares in a fixed order.
__global__ void __launch_bounds__(256)
rownorm_kernel(const float* R, int64_t ldr, float* Q, int64_t ldq, int64_t n,
               float eps) {
  __shared__ double part[8];
  const int64_t c = blockIdx.x;
  const float* row = R + c * ldr;
  double acc = 0.0;
  for (int64_t j = threadIdx.x; j < n; j += blockDim.x) acc += (double)row[j] * row[j];
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
  __syncthreads();
  double tot = 0.0;
  for (int w = 0; w < 8; ++w) tot += part[w];
  const float inv = (float)(1.0 / (sqrt(tot) + (double)eps));
  for (int64_t j = threadIdx.x; j < n; j += blockDim.x) Q[c * ldq + j] = row[j] * inv;
}

// sigma[c] = ||R[c][:]||_2 (float64 sum of squares in a fixed order).
__global__ void __launch_bounds__(256)
rownorm_only_kernel(const float* R, int64_t ldr, int64_t n, float* sigma) {
  __shared__ double part[8];
  const int64_t c = blockIdx.x;
  const float* row = R + c * ldr;
  double acc = 0.0;
  for (int64_t j = threadIdx.x; j < n; j += blockDim.x) acc += (double)row[j] * row[j];
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double tot = 0.0;
    for (int w = 0; w < 8; ++w) tot += part[w];
    sigma[c] = (float)sqrt(tot);
  }
}

// One block per matrix: exp(-sum p ln p), p_j = sigma_j^2 / sum sigma^2.
struct ERankArgs {
  const float* sigma;
  int64_t off[kChunk + 1];
  float* erank;
};

__global__ void __launch_bounds__(256) erank_kernel(const ERankArgs a) {
  __shared__ double red[256];
  const int i = blockIdx.x;
  const float* s = a.sigma + a.off[i];
  const int64_t r = a.off[i + 1] - a.off[i];
  double e = 0.0;
  for (int64_t j = threadIdx.x; j < r; j += blockDim.x) e += (double)s[j] * s[j];
  red[threadIdx.x] = e;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  const double tot = red[0];
  __syncthreads();
  double h = 0.0;
  if (tot > 0.0) {
    for (int64_t j = threadIdx.x; j < r; j += blockDim.x) {
      const double pj = (double)s[j] * s[j] / tot;
      if (pj > 0.0) h -= pj * log(pj);
    }
  }
  red[threadIdx.x] = h;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) a.erank[i] = tot > 0.0 ? (float)exp(red[0]) : 0.f;
}

// --------------------------------------------------------------- helpers
__global__ void transpose_kernel(const float* src, int64_t lds, float* dst,
                                 int64_t ldd, int64_t rows, int64_t cols) {
  __shared__ float t[32][33];
  const int64_t r0 = (int64_t)blockIdx.y * 32, c0 = (int64_t)blockIdx.x * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 32 x 8
  for (int y = ty; y < 32; y += 8) {
    const int64_t r = r0 + y, c = c0 + tx;
    t[y][tx] = (r < rows && c < cols) ? src[r * lds + c] : 0.f;
  }
  __syncthreads();
  for (int y = ty; y < 32; y += 8) {
    const int64_t r = c0 + y, c = r0 + tx;  // dst is cols x rows
    if (r < cols && c < rows) dst[r * ldd + c] = t[tx][y];
  }
}

__global__ void copy2d_kernel(const float* src, int64_t lds, float* dst,
                              int64_t ldd, int64_t rows, int64_t cols) {
  const int64_t total = rows * cols;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = e / cols, c = e - (e / cols) * cols;
    dst[r * ldd + c] = src[r * lds + c];
  }
}

unsigned grid_1d(int64_t n, int per_block) {
  int64_t b = ceil_div(n, per_block);
  int64_t cap = (int64_t)num_sms() * 8;
  if (b > cap) b = cap;
  return (unsigned)(b < 1 ? 1 : b);
}

// Packed triangle (plus r floats) the one-CTA kernel keeps in shared
// memory: at most 33 KB for the ranks it serves (r <= 128).
size_t chol_smem_bytes(int r) { return ((size_t)r * (r + 1) / 2 + r) * sizeof(float); }

int gram_splits(int r, int64_t L) {
  const int tiles = (int)ceil_div(r, kGT);
  const int pairs = tiles * (tiles + 1) / 2;
  int64_t want = ceil_div((int64_t)num_sms() * 4, pairs);
  int64_t maxs = ceil_div(L, 256);  // at least 256 columns per split
  if (want > maxs) want = maxs;
  if (want < 1) want = 1;
  if (want > 64) want = 64;
  return (int)want;
}

struct DionWs {
  Buf Pa, Pb;   // r x m
  Buf P;        // m x r
  Buf Ra, Rb;   // r x n
  Buf part;     // [64][r][r]
  Buf Linv;     // R x R (R = r rounded up to 32)
  Buf S;        // R x R (blocked Cholesky)
  Buf ctl;      // barrier counter and flags of the blocked Cholesky
};

// Ranks from blocked_chol_min_rank() up take a blocked Cholesky: the
// one-CTA kernel with the blocks in shared memory up to
// smem_chol_max_rank(), the cooperative multi-CTA kernel above it; smaller
// ranks keep the one-CTA packed-triangle kernel.  Per 4096 x 4096
// Orth-Dion step the one-CTA blocked kernel is 7-11% faster than the
// better of the other two from r = 64 to 192, 2% at r = 224 and 4% slower
// at r = 256, where the cooperative kernel's wider phases win.
// OUO_CHOL_BLOCKED_MIN_RANK (1 to 129) and OUO_CHOL_SMEM_MAX_RANK (0 to
// 256; 0 turns the one-CTA blocked kernel off) override the two bounds.
int blocked_chol_min_rank() {
  const char* env = getenv("OUO_CHOL_BLOCKED_MIN_RANK");
  if (env) {
    const int v = atoi(env);
    if (v >= 1 && v <= 129) return v;
  }
  return 64;
}
int smem_chol_max_rank() {
  const char* env = getenv("OUO_CHOL_SMEM_MAX_RANK");
  if (env) {
    const int v = atoi(env);
    if (v >= 0 && v <= 256) return v;
  }
  return 224;
}
int64_t padded_rank(int r) { return ceil_div(r, 32) * 32; }

DionWs carve_dion(Arena& ar, int64_t m, int64_t n, int r) {
  DionWs w;
  w.Pa = ar.take(OUO_F32, 1, r, m);
  w.Pb = ar.take(OUO_F32, 1, r, m);
  w.P = ar.take(OUO_F32, 1, m, r);
  w.Ra = ar.take(OUO_F32, 1, r, n);
  w.Rb = ar.take(OUO_F32, 1, r, n);
  w.part = ar.take(OUO_F32, 64, r, r);
  const int64_t R = padded_rank(r);
  w.Linv = ar.take(OUO_F32, 1, R, R);
  w.S = ar.take(OUO_F32, 1, R, R);
  w.ctl = ar.take(OUO_F32, 1, 1, (int64_t)ceil_div(chol_blocked_ctl_bytes(r), 4));
  return w;
}

Buf caller_buf(const ouo_mat& m, int dtype) {
  Buf b;
  b.p = reinterpret_cast<char*>(m.ptr);
  b.dtype = dtype;
  b.rows = m.rows;
  b.cols = m.cols;
  b.ld = m.ld;
  b.stride = m.rows * m.ld;
  b.nb = 1;
  return b;
}

// Partial Gram matrices of the rows of X (r x L) into w.part: returns the
// number of partials written (their float64 sum is X X^T).
int gram_parts(const Buf& X, const DionWs& w, cudaStream_t s, int* used) {
  const int r = (int)X.rows;
  const int64_t L = X.cols;
  GramArgs ga;
  ga.X = reinterpret_cast<const float*>(X.p);
  ga.ld = X.ld;
  ga.r = r;
  ga.L = L;
  const int splits = gram_splits(r, L);
  ga.chunk = ceil_div(ceil_div(L, splits), kGT) * kGT;
  *used = (int)ceil_div(L, ga.chunk);
  ga.part = reinterpret_cast<float*>(w.part.p);
  ga.tiles = (int)ceil_div(r, kGT);
  dim3 grid((unsigned)(ga.tiles * (ga.tiles + 1) / 2), (unsigned)*used);
  gram_partial_kernel<<<grid, 256, 0, s>>>(ga);
  OUO_CHECK_LAUNCH();
  return OUO_OK;
}

__global__ void sum_parts_kernel(const float* part, int splits, int64_t n, float* out) {
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n;
       e += (int64_t)gridDim.x * blockDim.x) {
    double s = 0.0;
    for (int q = 0; q < splits; ++q) s += (double)part[(size_t)q * n + e];
    out[e] = (float)s;
  }
}

// w.Linv = L^-1 where L L^T = sum of `splits` r x r partials at `part`
// (L_rows: the rows' length, for the shifted retry).
int cholesky_inverse(const float* part, int splits, int r, int64_t L_rows,
                     const DionWs& w, int* status, cudaStream_t s) {
  if (r >= blocked_chol_min_rank() && r <= smem_chol_max_rank() && chol_smem_fits(r)) {
    if (splits > 1) {  // one wide pass sums the partials; the CTA reads S once
      const int64_t n = (int64_t)r * r;
      float* S = reinterpret_cast<float*>(w.S.p);
      sum_parts_kernel<<<grid_1d(n, 256), 256, 0, s>>>(part, splits, n, S);
      OUO_CHECK_LAUNCH();
      part = S;
      splits = 1;
    }
    OUO_TRY(chol_smem(part, r, L_rows, reinterpret_cast<float*>(w.Linv.p), status, s));
  } else if (r >= blocked_chol_min_rank()) {
    OUO_TRY(chol_blocked(part, splits, r, L_rows, reinterpret_cast<float*>(w.S.p),
                         reinterpret_cast<float*>(w.Linv.p), w.ctl.p, status, s));
  } else {
    CholArgs ca;
    ca.part = part;
    ca.splits = splits;
    ca.r = r;
    ca.L = L_rows;
    ca.Linv = reinterpret_cast<float*>(w.Linv.p);
    ca.ldl = w.Linv.ld;
    ca.status = status;
    chol_inv_kernel<<<1, 1024, chol_smem_bytes(r), s>>>(ca);
    OUO_CHECK_LAUNCH();
  }
  return OUO_OK;
}

// dst = Linv src (r x L, fp32 SIMT)
int apply_linv(const DionWs& w, int r, const Buf& src, const Buf& dst, cudaStream_t s) {
  GemmDesc d;
  d.M = r;
  d.N = src.cols;
  d.K = r;
  d.nb = 1;
  d.A = w.Linv;
  d.B = src;
  d.b_mn = 1;
  d.out_f32 = dst;
  d.has_f32 = true;
  return gemm_simt(d, s);
}

// Rows of X (r x L, workspace) made orthonormal into Y: two CholeskyQR
// passes (X -> tmp -> Y); X is clobbered.
int orth_rows(Buf X, Buf tmp, Buf Y, const DionWs& w, cudaStream_t s,
              int* status) {
  const int r = (int)X.rows;
  Buf src = X;
  for (int pass = 0; pass < 2; ++pass) {
    Buf dst = pass == 0 ? tmp : Y;
    int used = 0;
    OUO_TRY(gram_parts(src, w, s, &used));
    OUO_TRY(cholesky_inverse(reinterpret_cast<const float*>(w.part.p), used, r, src.cols,
                             w, status, s));
    OUO_TRY(apply_linv(w, r, src, dst, s));
    src = dst;
  }
  return OUO_OK;
}

int validate_dion(const ouo_dion_params* p) {
  if (!p) return set_error(OUO_ERR_INVALID_ARG, "NULL dion params");
  if (p->norm_mode != OUO_DION_COLNORM && p->norm_mode != OUO_DION_QR)
    return set_error(OUO_ERR_INVALID_ARG, "unknown norm_mode %d", p->norm_mode);
  if (!(p->eps >= 0.f)) return set_error(OUO_ERR_INVALID_ARG, "eps must be >= 0");
  return OUO_OK;
}

size_t dion_plan_bytes(const ouo_mat* M, int nmat, const int* ranks) {
  Arena ar{nullptr, 0, 0, true};
  for (int i = 0; i < nmat; ++i) carve_dion(ar, M[i].rows, M[i].cols, ranks[i]);
  return ar.used + 256;
}

}  // namespace
}  // namespace ouo

extern "C" size_t dion_workspace_bytes(const ouo_mat* M, int nmat,
                                       const ouo_dion_params* p) {
  if (!M || !p || nmat <= 0 || nmat > OUO_MAX_BATCH || p->rank < 1) return 0;
  std::vector<int> ranks((size_t)nmat, p->rank);
  return ouo::dion_plan_bytes(M, nmat, ranks.data());
}

extern "C" size_t dion_workspace_bytes_ranks(const ouo_mat* M, const int* ranks,
                                             int nmat, const ouo_dion_params* p) {
  if (!M || !ranks || !p || nmat <= 0 || nmat > OUO_MAX_BATCH) return 0;
  for (int i = 0; i < nmat; ++i)
    if (ranks[i] < 1) return 0;
  return ouo::dion_plan_bytes(M, nmat, ranks);
}

extern "C" int dion_lowrank_step(const ouo_mat* M, const ouo_mat* G,
                                 int g_dtype, const ouo_mat* Q_state,
                                 const ouo_mat* W, int w_dtype, int nmat,
                                 const ouo_dion_params* p, const float* scale,
                                 void* ws, size_t ws_bytes, int* dev_status,
                                 void* stream) {
  return dion_lowrank_step_stats(M, G, g_dtype, Q_state, W, w_dtype, nmat, p, scale,
                                 ws, ws_bytes, nullptr, dev_status, stream);
}

extern "C" int dion_lowrank_step_stats(const ouo_mat* M, const ouo_mat* G,
                                       int g_dtype, const ouo_mat* Q_state,
                                       const ouo_mat* W, int w_dtype, int nmat,
                                       const ouo_dion_params* p, const float* scale,
                                       void* ws, size_t ws_bytes, float* sigma,
                                       int* dev_status, void* stream) {
  using namespace ouo;
  clear_error();
  if (nmat < 0 || nmat > OUO_MAX_BATCH)
    return set_error(OUO_ERR_INVALID_ARG, "nmat %d out of range", nmat);
  OUO_TRY(validate_dion(p));
  if (nmat == 0) return OUO_OK;
  OUO_TRY(validate_mats(M, nmat, OUO_F32, "M"));
  OUO_TRY(validate_mats(G, nmat, g_dtype, "G"));
  OUO_TRY(validate_mats(Q_state, nmat, OUO_F32, "Q_state"));
  OUO_TRY(validate_mats(W, nmat, w_dtype, "W"));
  OUO_TRY(validate_same_shapes(M, G, nmat, "M", "G"));
  OUO_TRY(validate_same_shapes(M, W, nmat, "M", "W"));
  if (p->rank < 0) return set_error(OUO_ERR_INVALID_ARG, "rank %d < 0", p->rank);
  // per-matrix ranks: p->rank, or Q_state[i].rows when p->rank == 0
  std::vector<int> ranks((size_t)nmat);
  for (int i = 0; i < nmat; ++i) {
    const int r = p->rank ? p->rank : (int)Q_state[i].rows;
    ranks[i] = r;
    if (r < 1 || r > M[i].rows || r > M[i].cols)
      return set_error(OUO_ERR_INVALID_ARG, "rank %d outside [1, min(rows, cols)] for M[%d]",
                       r, i);
    if (Q_state[i].rows != r || Q_state[i].cols != M[i].cols)
      return set_error(OUO_ERR_INVALID_ARG,
                       "Q_state[%d] must be r x cols (%d x %lld, the transposed factor)",
                       i, r, (long long)M[i].cols);
    if (!vec16(M[i], OUO_F32) || !vec16(Q_state[i], OUO_F32) || !vec16(W[i], w_dtype))
      return set_error(OUO_ERR_INVALID_ARG,
                       "dion_lowrank_step needs M, Q_state and W rows on 16-byte "
                       "boundaries (matrix %d)", i);
  }
  if (dev_status && ((uintptr_t)dev_status % 4))
    return set_error(OUO_ERR_INVALID_ARG, "dev_status misaligned");
  if (sigma && ((uintptr_t)sigma % 4))
    return set_error(OUO_ERR_INVALID_ARG, "sigma misaligned");
  const size_t need = dion_plan_bytes(M, nmat, ranks.data());
  if (!ws || ws_bytes < need)
    return set_error(OUO_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given",
                     need, ws_bytes);
  if ((uintptr_t)ws % 256)
    return set_error(OUO_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  OUO_TRY(require_sm100());
  cudaStream_t s = (cudaStream_t)stream;
  // B = M + G for the whole batch
  OUO_TRY(dion_momentum_update(M, G, nmat, g_dtype, p->mu, OUO_MOMENTUM_ACCUM,
                               nullptr, stream));
  Arena ar{reinterpret_cast<char*>(ws), ws_bytes, 0, false};
  const float mu = p->mu, beta = p->beta;
  int64_t sig_off = 0;
  for (int i = 0; i < nmat; ++i) {
    const int64_t m = M[i].rows, n = M[i].cols;
    const int r = ranks[i];
    DionWs w = carve_dion(ar, m, n, r);
    const Buf Bm = caller_buf(M[i], OUO_F32);
    const Buf Qt = caller_buf(Q_state[i], OUO_F32);
    // Pt = Qt B^T  (r x m)
    {
      GemmDesc d;
      d.M = r; d.N = m; d.K = n; d.nb = 1;
      d.A = Qt;
      d.B = Bm;
      d.out_f32 = w.Pa;
      d.has_f32 = true;
      OUO_TRY(gemm_umma(d, s, dev_status));
    }
    // rows of Pt orthonormal (P = orth(B Q_prev)) -> Pa
    OUO_TRY(orth_rows(w.Pa, w.Pb, w.Pa, w, s, dev_status));
    // Rt = Pt B  (r x n)
    {
      GemmDesc d;
      d.M = r; d.N = n; d.K = m; d.nb = 1;
      d.A = w.Pa;
      d.B = Bm;
      d.b_mn = 1;
      d.out_f32 = w.Ra;
      d.has_f32 = true;
      OUO_TRY(gemm_umma(d, s, dev_status));
    }
    // the power iteration's singular-value estimates: ||rows of Rt||
    if (sigma) {
      rownorm_only_kernel<<<r, 256, 0, s>>>(reinterpret_cast<const float*>(w.Ra.p), w.Ra.ld,
                                            n, sigma + sig_off);
      OUO_CHECK_LAUNCH();
    }
    sig_off += r;
    // P = Pt^T (m x r), the K-major left operand of the updates
    {
      dim3 grid((unsigned)ceil_div(m, 32), (unsigned)ceil_div(r, 32));
      transpose_kernel<<<grid, 256, 0, s>>>(reinterpret_cast<const float*>(w.Pa.p),
                                            w.Pa.ld, reinterpret_cast<float*>(w.P.p),
                                            w.P.ld, r, m);
      OUO_CHECK_LAUNCH();
    }
    // M <- beta B - (beta - mu) P Rt   (in place over B)
    {
      GemmDesc d;
      d.M = m; d.N = n; d.K = r; d.nb = 1;
      d.A = w.P;
      d.B = w.Ra;
      d.b_mn = 1;
      d.alpha = -(beta - mu);
      d.beta = beta;
      d.has_c0 = true;
      d.direct = {MatRef{M[i].ptr, M[i].ld}};
      d.direct_dtype = OUO_F32;
      d.c0_from_out = true;
      OUO_TRY(gemm_umma(d, s, dev_status));
    }
    // Qt_new: rows of Rt normalized (Dion) or orthonormalized (Orth-Dion) -> Rb
    Buf Qn = w.Rb;
    if (p->norm_mode == OUO_DION_COLNORM) {
      rownorm_kernel<<<r, 256, 0, s>>>(reinterpret_cast<const float*>(w.Ra.p), w.Ra.ld,
                                       reinterpret_cast<float*>(w.Rb.p), w.Rb.ld, n,
                                       p->eps);
      OUO_CHECK_LAUNCH();
    } else {
      OUO_TRY(orth_rows(w.Ra, w.Rb, w.Ra, w, s, dev_status));
      Qn = w.Ra;
    }
    // W <- (1 - lr wd) W - lr s P Qt_new
    {
      const float sc = scale ? scale[i] : 1.0f;
      GemmDesc d;
      d.M = m; d.N = n; d.K = r; d.nb = 1;
      d.A = w.P;
      d.B = Qn;
      d.b_mn = 1;
      d.alpha = -p->lr * sc;
      d.beta = 1.0f - p->lr * p->wd;
      d.has_c0 = true;
      d.direct = {MatRef{W[i].ptr, W[i].ld}};
      d.direct_dtype = w_dtype;
      d.c0_from_out = true;
      OUO_TRY(gemm_umma(d, s, dev_status));
    }
    // state <- Qt_new
    copy2d_kernel<<<grid_1d((int64_t)r * n, 256), 256, 0, s>>>(
        reinterpret_cast<const float*>(Qn.p), Qn.ld,
        reinterpret_cast<float*>(Q_state[i].ptr), Q_state[i].ld, r, n);
    OUO_CHECK_LAUNCH();
  }
  return OUO_OK;
}

extern "C" int dion_effective_rank(const float* sigma, const int* ranks, int nmat,
                                   float* erank, void* stream) {
  using namespace ouo;
  clear_error();
  if (nmat < 0 || nmat > OUO_MAX_BATCH)
    return set_error(OUO_ERR_INVALID_ARG, "nmat %d out of range", nmat);
  if (nmat == 0) return OUO_OK;
  if (!sigma || !ranks || !erank)
    return set_error(OUO_ERR_INVALID_ARG, "NULL sigma, ranks or erank");
  if ((uintptr_t)sigma % 4 || (uintptr_t)erank % 4)
    return set_error(OUO_ERR_INVALID_ARG, "sigma / erank misaligned");
  for (int i = 0; i < nmat; ++i)
    if (ranks[i] < 1) return set_error(OUO_ERR_INVALID_ARG, "ranks[%d] < 1", i);
  OUO_TRY(require_sm100());
  cudaStream_t s = (cudaStream_t)stream;
  int64_t base = 0;
  for (int c0 = 0; c0 < nmat; c0 += kChunk) {
    const int cn = nmat - c0 < kChunk ? nmat - c0 : kChunk;
    ERankArgs a;
    a.sigma = sigma + base;
    a.erank = erank + c0;
    a.off[0] = 0;
    for (int i = 0; i < cn; ++i) a.off[i + 1] = a.off[i] + ranks[c0 + i];
    erank_kernel<<<cn, 256, 0, s>>>(a);
    OUO_CHECK_LAUNCH();
    base += a.off[cn];
  }
  return OUO_OK;
}

// ------------------------------------------------------ row-sharded step
// The power iteration with the rows of every matrix spread over ranks: the
// r x r Gram matrices of P^T and the r x n product P^T B are the only
// quantities summed across ranks (by the caller, between the calls below);
// everything else is local to a rank's rows, and the right factor is
// formed redundantly on every rank.
namespace ouo {
namespace {

// out[e] = sum_p part[p][e] in float64, fixed order (the reduction the
// Cholesky kernels apply to their partials), rounded to fp32.
int64_t pitch4(int64_t n) { return ceil_div(n, 4) * 4; }

// floats of matrix i's block of `red` (256-byte multiple)
int64_t red_block(int r, int64_t n) {
  const int64_t f = (int64_t)r * r > (int64_t)r * pitch4(n) ? (int64_t)r * r : (int64_t)r * pitch4(n);
  return ceil_div(f, 64) * 64;
}

// Ranks of the batch (p->rank, or Q_state rows with p->rank == 0) and the
// shared shape checks of every sharded call.
int shard_ranks(const ouo_mat* M, const ouo_mat* Q_state, int nmat,
                const ouo_dion_params* p, std::vector<int>& ranks) {
  OUO_TRY(validate_dion(p));
  if (p->rank < 0) return set_error(OUO_ERR_INVALID_ARG, "rank %d < 0", p->rank);
  OUO_TRY(validate_mats(M, nmat, OUO_F32, "M"));
  OUO_TRY(validate_mats(Q_state, nmat, OUO_F32, "Q_state"));
  ranks.assign((size_t)nmat, 0);
  for (int i = 0; i < nmat; ++i) {
    const int r = p->rank ? p->rank : (int)Q_state[i].rows;
    ranks[i] = r;
    if (r < 1 || r > M[i].cols)
      return set_error(OUO_ERR_INVALID_ARG, "rank %d outside [1, cols] for M[%d]", r, i);
    if (Q_state[i].rows != r || Q_state[i].cols != M[i].cols)
      return set_error(OUO_ERR_INVALID_ARG, "Q_state[%d] must be r x cols", i);
    if (!vec16(M[i], OUO_F32) || !vec16(Q_state[i], OUO_F32))
      return set_error(OUO_ERR_INVALID_ARG,
                       "sharded Dion needs M and Q_state rows on 16-byte boundaries (%d)", i);
  }
  return OUO_OK;
}

int shard_common(const ouo_mat* M, const ouo_mat* Q_state, int nmat,
                 const ouo_dion_params* p, void* ws, size_t ws_bytes, float* red,
                 int* dev_status, std::vector<int>& ranks) {
  OUO_TRY(shard_ranks(M, Q_state, nmat, p, ranks));
  if (dev_status && ((uintptr_t)dev_status % 4))
    return set_error(OUO_ERR_INVALID_ARG, "dev_status misaligned");
  if (!red || ((uintptr_t)red % 256))
    return set_error(OUO_ERR_INVALID_ARG, "red must be a 256-byte aligned device buffer");
  const size_t need = dion_plan_bytes(M, nmat, ranks.data());
  if (!ws || ws_bytes < need)
    return set_error(OUO_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given",
                     need, ws_bytes);
  if ((uintptr_t)ws % 256)
    return set_error(OUO_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  return require_sm100();
}

int sum_parts(const DionWs& w, int used, int r, float* out, cudaStream_t s) {
  const int64_t n = (int64_t)r * r;
  sum_parts_kernel<<<grid_1d(n, 256), 256, 0, s>>>(reinterpret_cast<const float*>(w.part.p),
                                                   used, n, out);
  OUO_CHECK_LAUNCH();
  return OUO_OK;
}

}  // namespace
}  // namespace ouo

extern "C" size_t dion_shard_workspace_bytes(const ouo_mat* M, const ouo_mat* Q_state,
                                             int nmat, const ouo_dion_params* p) {
  if (!M || !Q_state || !p || nmat <= 0 || nmat > OUO_MAX_BATCH || p->rank < 0) return 0;
  std::vector<int> ranks((size_t)nmat);
  for (int i = 0; i < nmat; ++i) {
    ranks[i] = p->rank ? p->rank : (int)Q_state[i].rows;
    if (ranks[i] < 1) return 0;
  }
  return ouo::dion_plan_bytes(M, nmat, ranks.data());
}

extern "C" size_t dion_shard_red_floats(const ouo_mat* M, const ouo_mat* Q_state, int nmat,
                                        const ouo_dion_params* p) {
  if (!M || !Q_state || !p || nmat <= 0 || nmat > OUO_MAX_BATCH || p->rank < 0) return 0;
  size_t f = 0;
  for (int i = 0; i < nmat; ++i) {
    const int r = p->rank ? p->rank : (int)Q_state[i].rows;
    if (r < 1) return 0;
    f += (size_t)ouo::red_block(r, M[i].cols);
  }
  return f;
}

extern "C" int dion_shard_project(const ouo_mat* M, const ouo_mat* G, int g_dtype,
                                  const ouo_mat* Q_state, int nmat,
                                  const ouo_dion_params* p, void* ws, size_t ws_bytes,
                                  float* red, int* dev_status, void* stream) {
  using namespace ouo;
  clear_error();
  if (nmat < 0 || nmat > OUO_MAX_BATCH)
    return set_error(OUO_ERR_INVALID_ARG, "nmat %d out of range", nmat);
  if (nmat == 0) return OUO_OK;
  std::vector<int> ranks;
  OUO_TRY(shard_common(M, Q_state, nmat, p, ws, ws_bytes, red, dev_status, ranks));
  OUO_TRY(validate_mats(G, nmat, g_dtype, "G"));
  OUO_TRY(validate_same_shapes(M, G, nmat, "M", "G"));
  cudaStream_t s = (cudaStream_t)stream;
  OUO_TRY(dion_momentum_update(M, G, nmat, g_dtype, p->mu, OUO_MOMENTUM_ACCUM, nullptr,
                               stream));
  Arena ar{reinterpret_cast<char*>(ws), ws_bytes, 0, false};
  int64_t off = 0;
  for (int i = 0; i < nmat; ++i) {
    const int r = ranks[i];
    const int64_t m = M[i].rows, n = M[i].cols;
    DionWs w = carve_dion(ar, m, n, r);
    GemmDesc d;  // P^T = Q^T B^T (r x m local)
    d.M = r; d.N = m; d.K = n; d.nb = 1;
    d.A = caller_buf(Q_state[i], OUO_F32);
    d.B = caller_buf(M[i], OUO_F32);
    d.out_f32 = w.Pa;
    d.has_f32 = true;
    OUO_TRY(gemm_umma(d, s, dev_status));
    int used = 0;
    OUO_TRY(gram_parts(w.Pa, w, s, &used));
    OUO_TRY(sum_parts(w, used, r, red + off, s));
    off += red_block(r, n);
  }
  return OUO_OK;
}

namespace ouo {
namespace {
// orth1 (second = false) and orth2 (second = true)
int shard_orth(const ouo_mat* M, const ouo_mat* Q_state, int nmat,
               const ouo_dion_params* p, const int64_t* rows_total, void* ws,
               size_t ws_bytes, float* red, int* dev_status, void* stream, bool second) {
  clear_error();
  if (nmat < 0 || nmat > OUO_MAX_BATCH)
    return set_error(OUO_ERR_INVALID_ARG, "nmat %d out of range", nmat);
  if (nmat == 0) return OUO_OK;
  if (!rows_total) return set_error(OUO_ERR_INVALID_ARG, "NULL rows_total");
  std::vector<int> ranks;
  OUO_TRY(shard_common(M, Q_state, nmat, p, ws, ws_bytes, red, dev_status, ranks));
  for (int i = 0; i < nmat; ++i)
    if (rows_total[i] < ranks[i] || rows_total[i] < M[i].rows)
      return set_error(OUO_ERR_INVALID_ARG, "rows_total[%d] smaller than rank or local rows", i);
  cudaStream_t s = (cudaStream_t)stream;
  Arena ar{reinterpret_cast<char*>(ws), ws_bytes, 0, false};
  int64_t off = 0;
  for (int i = 0; i < nmat; ++i) {
    const int r = ranks[i];
    const int64_t m = M[i].rows, n = M[i].cols;
    DionWs w = carve_dion(ar, m, n, r);
    OUO_TRY(cholesky_inverse(red + off, 1, r, rows_total[i], w, dev_status, s));
    if (!second) {
      OUO_TRY(apply_linv(w, r, w.Pa, w.Pb, s));
      int used = 0;
      OUO_TRY(gram_parts(w.Pb, w, s, &used));
      OUO_TRY(sum_parts(w, used, r, red + off, s));
    } else {
      OUO_TRY(apply_linv(w, r, w.Pb, w.Pa, s));
      Buf rt;  // P^T B (r x n) into the exchange buffer
      rt.p = reinterpret_cast<char*>(red + off);
      rt.dtype = OUO_F32;
      rt.rows = r;
      rt.cols = n;
      rt.ld = pitch4(n);
      rt.stride = rt.rows * rt.ld;
      rt.nb = 1;
      GemmDesc d;
      d.M = r; d.N = n; d.K = m; d.nb = 1;
      d.A = w.Pa;
      d.B = caller_buf(M[i], OUO_F32);
      d.b_mn = 1;
      d.out_f32 = rt;
      d.has_f32 = true;
      OUO_TRY(gemm_umma(d, s, dev_status));
    }
    off += red_block(r, n);
  }
  return OUO_OK;
}
}  // namespace
}  // namespace ouo

extern "C" int dion_shard_orth1(const ouo_mat* M, const ouo_mat* Q_state, int nmat,
                                const ouo_dion_params* p, const int64_t* rows_total,
                                void* ws, size_t ws_bytes, float* red, int* dev_status,
                                void* stream) {
  return ouo::shard_orth(M, Q_state, nmat, p, rows_total, ws, ws_bytes, red, dev_status,
                         stream, false);
}

extern "C" int dion_shard_orth2(const ouo_mat* M, const ouo_mat* Q_state, int nmat,
                                const ouo_dion_params* p, const int64_t* rows_total,
                                void* ws, size_t ws_bytes, float* red, int* dev_status,
                                void* stream) {
  return ouo::shard_orth(M, Q_state, nmat, p, rows_total, ws, ws_bytes, red, dev_status,
                         stream, true);
}

extern "C" int dion_shard_update(const ouo_mat* M, const ouo_mat* Q_state,
                                 const ouo_mat* W, int w_dtype, int nmat,
                                 const ouo_dion_params* p, const float* scale, void* ws,
                                 size_t ws_bytes, float* red, int* dev_status,
                                 void* stream) {
  using namespace ouo;
  clear_error();
  if (nmat < 0 || nmat > OUO_MAX_BATCH)
    return set_error(OUO_ERR_INVALID_ARG, "nmat %d out of range", nmat);
  if (nmat == 0) return OUO_OK;
  std::vector<int> ranks;
  OUO_TRY(shard_common(M, Q_state, nmat, p, ws, ws_bytes, red, dev_status, ranks));
  OUO_TRY(validate_mats(W, nmat, w_dtype, "W"));
  OUO_TRY(validate_same_shapes(M, W, nmat, "M", "W"));
  for (int i = 0; i < nmat; ++i)
    if (!vec16(W[i], w_dtype))
      return set_error(OUO_ERR_INVALID_ARG, "W rows must be on 16-byte boundaries (%d)", i);
  cudaStream_t s = (cudaStream_t)stream;
  Arena ar{reinterpret_cast<char*>(ws), ws_bytes, 0, false};
  const float mu = p->mu, beta = p->beta;
  int64_t off = 0;
  for (int i = 0; i < nmat; ++i) {
    const int r = ranks[i];
    const int64_t m = M[i].rows, n = M[i].cols;
    DionWs w = carve_dion(ar, m, n, r);
    // R^T (summed over ranks) into the workspace
    copy2d_kernel<<<grid_1d((int64_t)r * n, 256), 256, 0, s>>>(
        red + off, pitch4(n), reinterpret_cast<float*>(w.Ra.p), w.Ra.ld, r, n);
    OUO_CHECK_LAUNCH();
    {
      dim3 grid((unsigned)ceil_div(m, 32), (unsigned)ceil_div(r, 32));
      transpose_kernel<<<grid, 256, 0, s>>>(reinterpret_cast<const float*>(w.Pa.p),
                                            w.Pa.ld, reinterpret_cast<float*>(w.P.p),
                                            w.P.ld, r, m);
      OUO_CHECK_LAUNCH();
    }
    {  // M <- beta B - (beta - mu) P R^T (local rows)
      GemmDesc d;
      d.M = m; d.N = n; d.K = r; d.nb = 1;
      d.A = w.P;
      d.B = w.Ra;
      d.b_mn = 1;
      d.alpha = -(beta - mu);
      d.beta = beta;
      d.has_c0 = true;
      d.direct = {MatRef{M[i].ptr, M[i].ld}};
      d.direct_dtype = OUO_F32;
      d.c0_from_out = true;
      OUO_TRY(gemm_umma(d, s, dev_status));
    }
    Buf Qn = w.Rb;
    if (p->norm_mode == OUO_DION_COLNORM) {
      rownorm_kernel<<<r, 256, 0, s>>>(reinterpret_cast<const float*>(w.Ra.p), w.Ra.ld,
                                       reinterpret_cast<float*>(w.Rb.p), w.Rb.ld, n,
                                       p->eps);
      OUO_CHECK_LAUNCH();
    } else {
      OUO_TRY(orth_rows(w.Ra, w.Rb, w.Ra, w, s, dev_status));
      Qn = w.Ra;
    }
    {  // W <- (1 - lr wd) W - lr s P Q_new^T (local rows)
      const float sc = scale ? scale[i] : 1.0f;
      GemmDesc d;
      d.M = m; d.N = n; d.K = r; d.nb = 1;
      d.A = w.P;
      d.B = Qn;
      d.b_mn = 1;
      d.alpha = -p->lr * sc;
      d.beta = 1.0f - p->lr * p->wd;
      d.has_c0 = true;
      d.direct = {MatRef{W[i].ptr, W[i].ld}};
      d.direct_dtype = w_dtype;
      d.c0_from_out = true;
      OUO_TRY(gemm_umma(d, s, dev_status));
    }
    copy2d_kernel<<<grid_1d((int64_t)r * n, 256), 256, 0, s>>>(
        reinterpret_cast<const float*>(Qn.p), Qn.ld,
        reinterpret_cast<float*>(Q_state[i].ptr), Q_state[i].ld, r, n);
    OUO_CHECK_LAUNCH();
    off += red_block(r, n);
  }
  return OUO_OK;
}
