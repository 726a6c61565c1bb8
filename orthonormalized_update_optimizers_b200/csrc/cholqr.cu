// Batched CholeskyQR pieces of the Dion / Orth-Dion step: every kernel here
// takes a table of independent problems (one per matrix of a batch) and
// runs them in one launch.
//
// Source: "Orth-Dion: Eliminating Geometric Mismatch in Distributed Low-Rank
// Spectral Optimization", Problem Statement (the left factor of the power
// iteration is orthonormalized) and Orth-Dion (the right factor is too, by
// QR, instead of Dion's column normalization).  The QR of a block of r rows
// X (r x L, r <= L) is computed as CholeskyQR: S = X X^T = L L^T, and the
// rows of L^-1 X are orthonormal with the implied triangular factor L^T on
// a positive diagonal, i.e. the unique QR factor.
//
//   gram     on the tensor cores, split-tf32: lo = 2 (X - tf32(X)), then
//            part[s] = tf32(X) [tf32(X) | tf32(lo)]^T over K range s of
//            two passes (one tcgen05 GEMM, split-K so that a single matrix
//            fills the GPU), and S = sym(sum_s part[s]) in float64, fixed
//            order, rounded to fp32 and written in full: X X^T up to the
//            residual-residual term (2^-20 relative) and fp32 accumulation.
//   chol     one CTA per matrix (r <= 256): the lower 32 x 32 blocks of S in
//            shared memory, right-looking blocked Cholesky with one block of
//            look-ahead; writes the strictly lower blocks L_ij and the
//            inverses D_i = L_ii^-1 of the diagonal blocks.  A non-positive
//            pivot restarts once with the shift of shifted CholeskyQR,
//            11 (L r + r (r + 1)) u tr(S); a second failure reports
//            OUO_STATUS_BREAKDOWN and writes the identity.
//   trinv    Z = L^-1 from the blocks of L and the D_i, one CTA per block
//            column, written as Z, Z / 2 and Z - tf32(Z).
//   solve    Y = Z X on the tensor cores in three split-tf32 passes (one
//            tcgen05 GEMM over the batch), then optional copies of Y, its
//            transpose and the transpose's bf16 rounding.
//   rows     out = sum_s part[s] (split-K partial products) row by row, with
//            optional row norms (float64, fixed order) and normalized rows
//            (Dion's column normalization of R, stored transposed).
#include <cmath>

#include "internal.h"

namespace ouo {
namespace {

constexpr int kB = 32;        // Cholesky / solve block

// ------------------------------------------------------------------- gram
__device__ __forceinline__ int find_job(const int64_t* start, int njob, int64_t item) {
  int lo = 0, hi = njob - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (start[mid] <= item) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

// Residual operand of the split-tf32 Gram: lo = 2 (x - tf32(x)), where
// tf32(x) keeps the sign, exponent and top 10 mantissa bits of x (the
// tensor core's reading of an fp32 operand).  x - tf32(x) is exact in fp32,
// and so is the factor 2.  One CTA per row of every job.
struct LoBatch {
  const float* X[kChunk];
  float* lo[kChunk];
  int64_t ld[kChunk], L[kChunk];
  int64_t start[kChunk + 1];  // prefix sums of the jobs' rows
  int njob;
};

__device__ __forceinline__ float resid2(float x) {
  const float h = __uint_as_float(__float_as_uint(x) & 0xffffe000u);
  return 2.f * (x - h);
}

__global__ void __launch_bounds__(256) lo_kernel(const __grid_constant__ LoBatch lb) {
  const int j = find_job(lb.start, lb.njob, blockIdx.x);
  const int64_t row = blockIdx.x - lb.start[j];
  const float* x = lb.X[j] + row * lb.ld[j];
  float* o = lb.lo[j] + row * lb.ld[j];
  const int64_t L = lb.L[j], L4 = L >> 2;
  // rows start on 16-byte boundaries (ld a multiple of 4, aligned bases)
  const float4* x4 = reinterpret_cast<const float4*>(x);
  float4* o4 = reinterpret_cast<float4*>(o);
  for (int64_t c = threadIdx.x; c < L4; c += blockDim.x) {
    const float4 v = x4[c];
    o4[c] = make_float4(resid2(v.x), resid2(v.y), resid2(v.z), resid2(v.w));
  }
  for (int64_t c = 4 * L4 + threadIdx.x; c < L; c += blockDim.x) o[c] = resid2(x[c]);
}

// S = (U + U^T) / 2 with U = sum_s part[s] (float64, s ascending), the
// partials r x r with row pitch pitch4(r), one after another.  With
// U = X^ X^T + 2 X^ lo'^T (X^ = tf32(X), lo' = X - X^), the symmetric part is
// X^ X^T + X^ lo'^T + lo' X^T = X X^T - lo' lo'^T.  S is written in full.
// One CTA per pair of 32 x 32 tiles (bi, bj), bi <= bj: thread (ty, tx)
// sums U at rows bi*32 + ty + 8k, column bj*32 + tx, and at the mirrored
// position, both reads along rows; the mirrored sums meet their partners
// through shared memory.
struct SumBatch {
  const float* part[kChunk];
  float* S[kChunk];
  int r[kChunk], splits[kChunk];
  int64_t start[kChunk + 1];  // prefix sums of the jobs' tile pairs
  int njob;
};

__global__ void __launch_bounds__(256) sum_kernel(const __grid_constant__ SumBatch sb) {
  __shared__ double mir[32][33];
  const int j = find_job(sb.start, sb.njob, blockIdx.x);
  const int r = sb.r[j];
  const int nt = (r + 31) / 32;
  int pr = (int)(blockIdx.x - sb.start[j]);
  int bi = 0;
  while (pr >= nt - bi) { pr -= nt - bi; ++bi; }
  const int bj = bi + pr;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int64_t ldp = (r + 3) & ~3;
  const size_t sp = (size_t)r * ldp;
  const float* p = sb.part[j];
  double u[4] = {0.0, 0.0, 0.0, 0.0}, v[4] = {0.0, 0.0, 0.0, 0.0};
  const int cu = bj * 32 + tx, cv = bi * 32 + tx;
#pragma unroll 4
  for (int q = 0; q < sb.splits[j]; ++q) {
    const float* pq = p + q * sp;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int ru = bi * 32 + ty + 8 * k, rv = bj * 32 + ty + 8 * k;
      if (ru < r && cu < r) u[k] += (double)pq[(size_t)ru * ldp + cu];
      if (rv < r && cv < r) v[k] += (double)pq[(size_t)rv * ldp + cv];
    }
  }
  // v[k] = sum U[bj*32 + ty + 8k][bi*32 + tx]: element (tx, ty + 8k) of
  // the tile (bi, bj) of U^T
#pragma unroll
  for (int k = 0; k < 4; ++k) mir[ty + 8 * k][tx] = v[k];
  __syncthreads();
  float* S = sb.S[j];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int i = bi * 32 + ty + 8 * k, c = bj * 32 + tx;
    const double w = 0.5 * (u[k] + mir[tx][ty + 8 * k]);
    if (i < r && c < r) S[(size_t)i * r + c] = (float)w;
    u[k] = w;
  }
  if (bi == bj) return;
  // the mirrored tile (bj, bi) of S, rows along tx
  __syncthreads();
#pragma unroll
  for (int k = 0; k < 4; ++k) mir[ty + 8 * k][tx] = u[k];
  __syncthreads();
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int i = bj * 32 + ty + 8 * k, c = bi * 32 + tx;
    if (i < r && c < r) S[(size_t)i * r + c] = (float)mir[tx][ty + 8 * k];
  }
}

// ------------------------------------------------------------------- chol
constexpr int kCT = 384;             // threads of the Cholesky CTA
constexpr int kCW = kCT / 32;        // warps
constexpr int kP = 36;               // tile pitch (16-byte rows, conflict-free row reads)
constexpr int kTF = kB * kP;         // floats per tile
constexpr int kMaxNb = 8;            // blocks per side (r <= 256)

struct CholBatch {
  const float* S[kChunk];   // r x r, upper storage, ld r
  float* Lb[kChunk];        // R x R, ld R
  int r[kChunk];
  int64_t L[kChunk];        // length of the rows (for the shift)
  int njob;
  int* status;
};

size_t chol_smem_bytes(int nb) {
  const int ntri = nb * (nb + 1) / 2;
  // lower tiles, D of the current block, the panel (nb - 1 tiles), the
  // factoring warp's column scratch
  return (size_t)(ntri + 2 + (nb > 1 ? nb - 1 : 0)) * kTF * sizeof(float);
}

__device__ __forceinline__ int tri_index(int bi, int bj) { return bi * (bi + 1) / 2 + bj; }

__device__ __forceinline__ int tri_row_of(int t) {
  int bi = (int)((sqrtf(8.f * (float)t + 1.f) - 1.f) * 0.5f);
  while ((bi + 1) * (bi + 2) / 2 <= t) ++bi;
  while (bi * (bi + 1) / 2 > t) --bi;
  return bi;
}

// One warp: factor the 32 x 32 block T (pitch kP, lower triangle used),
// T = L L^T, and write D = L^-1 (lower triangular, zeros above) to Dt
// (pitch kP) and to global memory at g (row pitch ldg).  `col` is 32 x kP
// floats of shared scratch of this warp.  Returns false on a non-positive
// or non-finite pivot (the same in every lane).
//   factor:  row `lane` of the block in registers, right-looking.  Every
//            lane takes the pivot by one shuffle and forms 1/sqrt itself;
//            the scaled column k is broadcast through shared memory (one
//            store per lane, 16-byte reads), not by one shuffle per entry,
//            which would serialize 31 shuffles per pivot.
//   inverse: column `lane` of L^-1 by a column sweep, x[k] = acc[k] /
//            L[k][k], then every later row r loses L[r][k] x[k]; column k of
//            L is read from its transposed copy in `col`.
__device__ __noinline__ bool chol_inv32(const float* T, float* Dt, float* g, int64_t ldg,
                                        float* col) {
  const unsigned full = 0xffffffffu;
  const int lane = threadIdx.x & 31;
  bool ok = true;
  float l[kB];
#pragma unroll
  for (int k = 0; k < kB; k += 4) {
    const float4 v = *reinterpret_cast<const float4*>(T + lane * kP + k);
    l[k] = v.x; l[k + 1] = v.y; l[k + 2] = v.z; l[k + 3] = v.w;
  }
#pragma unroll
  for (int k = 0; k < kB; ++k) {
    const float piv = __shfl_sync(full, l[k], k);
    // a bad pivot is the same in every lane; the sweep runs on (its values
    // are discarded) so that the loop stays fully unrolled
    if (!(piv > 0.f) || !(piv < INFINITY)) ok = false;
    const float rs = rsqrtf(piv);
    l[k] = lane == k ? piv * rs : l[k] * rs;  // L[lane][k] (lanes above k: unused)
    // column k (rows > k) to every lane: col row k holds L[.][k], and its
    // padding column 32 holds 1 / L[k][k]
    col[k * kP + lane] = l[k];
    if (lane == 0) col[k * kP + kB] = rs;
    __syncwarp();
    if (k + 1 < kB) {
      const float lk = l[k];
#pragma unroll
      for (int j4 = ((k + 1) >> 2) << 2; j4 < kB; j4 += 4) {
        const float4 c4 = *reinterpret_cast<const float4*>(col + k * kP + j4);
        const float cj[4] = {c4.x, c4.y, c4.z, c4.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int j = j4 + u;
          if (j > k && lane >= j) l[j] = fmaf(-lk, cj[u], l[j]);
        }
      }
    }
  }
  // col row k now holds column k of L (rows k..31 valid)
  float acc[kB];
#pragma unroll
  for (int r = 0; r < kB; ++r) acc[r] = r == lane ? 1.f : 0.f;
#pragma unroll
  for (int k = 0; k < kB; ++k) {
    const float xk = acc[k] * col[k * kP + kB];
    acc[k] = xk;
#pragma unroll
    for (int r4 = ((k + 1) >> 2) << 2; r4 < kB; r4 += 4) {
      const float4 c4 = *reinterpret_cast<const float4*>(col + k * kP + r4);
      const float cr[4] = {c4.x, c4.y, c4.z, c4.w};
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (r4 + u > k) acc[r4 + u] = fmaf(-cr[u], xk, acc[r4 + u]);
    }
  }
  __syncwarp();
  // acc[r] = D[r][lane]; lanes write column `lane`
#pragma unroll
  for (int r = 0; r < kB; ++r) {
    Dt[r * kP + lane] = acc[r];
    g[(int64_t)r * ldg + lane] = acc[r];
  }
  return ok;
}

// acc[c] += sum_k A[lane][k] B[c0 + c][k], c < 8 (tiles of pitch kP)
__device__ __forceinline__ void rowdot8(const float* A, const float* B, int c0, float (&acc)[8]) {
  const int lane = threadIdx.x & 31;
  float row[kB];
#pragma unroll
  for (int k = 0; k < kB; k += 4) {
    const float4 v = *reinterpret_cast<const float4*>(A + lane * kP + k);
    row[k] = v.x; row[k + 1] = v.y; row[k + 2] = v.z; row[k + 3] = v.w;
  }
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const float* bp = B + (c0 + c) * kP;
#pragma unroll
    for (int k = 0; k < kB; k += 4) {
      const float4 v = *reinterpret_cast<const float4*>(bp + k);
      acc[c] = fmaf(row[k], v.x, acc[c]);
      acc[c] = fmaf(row[k + 1], v.y, acc[c]);
      acc[c] = fmaf(row[k + 2], v.z, acc[c]);
      acc[c] = fmaf(row[k + 3], v.w, acc[c]);
    }
  }
}

// tile -= A B^T over columns c0 .. c0 + 7 (row = lane)
__device__ __forceinline__ void sub_rowdot8(float* Tt, const float* A, const float* B, int c0) {
  const int lane = threadIdx.x & 31;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  rowdot8(A, B, c0, acc);
  float* sp = Tt + lane * kP + c0;
  const float4 s0 = *reinterpret_cast<const float4*>(sp);
  const float4 s1 = *reinterpret_cast<const float4*>(sp + 4);
  *reinterpret_cast<float4*>(sp) =
      make_float4(s0.x - acc[0], s0.y - acc[1], s0.z - acc[2], s0.w - acc[3]);
  *reinterpret_cast<float4*>(sp + 4) =
      make_float4(s1.x - acc[4], s1.y - acc[5], s1.z - acc[6], s1.w - acc[7]);
}

// C -= A B^T for whole 32 x 32 blocks (pitch kP), one warp: lane (lr, lc)
// = (lane / 8, lane % 8) owns rows lr + 4u (u < 8) and columns lc + 8v
// (v < 4), so that its operands come as float4 runs along k: per four k,
// 8 reads of A and 4 of B (bank-conflict free: the rows a read instruction
// touches are four consecutive rows, the columns eight consecutive ones)
// for 128 FMAs.
__device__ __forceinline__ void sub_blk32(float* C, const float* A, const float* B) {
  const int lane = threadIdx.x & 31, lr = lane >> 3, lc = lane & 7;
  float acc[8][4];
#pragma unroll
  for (int u = 0; u < 8; ++u)
#pragma unroll
    for (int v = 0; v < 4; ++v) acc[u][v] = 0.f;
#pragma unroll 2
  for (int k = 0; k < kB; k += 4) {
    float4 b4[4];
#pragma unroll
    for (int v = 0; v < 4; ++v) b4[v] = *reinterpret_cast<const float4*>(B + (lc + 8 * v) * kP + k);
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const float4 a4 = *reinterpret_cast<const float4*>(A + (lr + 4 * u) * kP + k);
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        acc[u][v] = fmaf(a4.x, b4[v].x, acc[u][v]);
        acc[u][v] = fmaf(a4.y, b4[v].y, acc[u][v]);
        acc[u][v] = fmaf(a4.z, b4[v].z, acc[u][v]);
        acc[u][v] = fmaf(a4.w, b4[v].w, acc[u][v]);
      }
    }
  }
#pragma unroll
  for (int u = 0; u < 8; ++u)
#pragma unroll
    for (int v = 0; v < 4; ++v) C[(lr + 4 * u) * kP + lc + 8 * v] -= acc[u][v];
}

__global__ void __launch_bounds__(kCT, 1) chol_kernel(const __grid_constant__ CholBatch cb) {
  extern __shared__ __align__(16) float sm[];
  __shared__ int s_bad;
  __shared__ double s_red[kCW];
  const int job = blockIdx.x;
  const float* S = cb.S[job];
  float* Lb = cb.Lb[job];
  const int r = cb.r[job];
  const int nb = (r + kB - 1) / kB, R = nb * kB;
  const int ntri = nb * (nb + 1) / 2;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto tile = [&](int bi, int bj) { return sm + (size_t)tri_index(bi, bj) * kTF; };
  float* Dt = sm + (size_t)ntri * kTF;
  float* col = Dt + kTF;   // column scratch of the factoring warp
  float* pan = col + kTF;
  auto gblk = [&](int bi, int bj) { return Lb + (size_t)bi * kB * R + (size_t)bj * kB; };

  bool ok = false;
  for (int attempt = 0; attempt < 2 && !ok; ++attempt) {
    double shift = 0.0;
    if (attempt == 1) {
      double t = 0.0;
      for (int i = threadIdx.x; i < r; i += kCT) t += (double)S[(size_t)i * r + i];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) t += __shfl_xor_sync(0xffffffffu, t, off);
      if (lane == 0) s_red[warp] = t;
      __syncthreads();
      double tr = 0.0;
      for (int w = 0; w < kCW; ++w) tr += s_red[w];
      const double u = 5.9604644775390625e-8;  // 2^-24
      shift = 11.0 * ((double)cb.L[job] * r + (double)r * (r + 1)) * u * tr;
      if (!(shift > 0.0)) shift = 1e-30;
      __syncthreads();
    }
    // lower tiles of S (full symmetric storage, ld r): row ii of tile
    // (bi, bj) is 32 consecutive floats of row bi*32 + ii, copied as eight
    // 16-byte asynchronous copies when the rows allow it; identity padding
    // past r
    {
      const bool vec = (r & 3) == 0 && ((uintptr_t)S & 15) == 0;
      for (int e = threadIdx.x; e < ntri * kB * 8; e += kCT) {
        const int tt = e >> 8, w = e & 255, ii = w >> 3, c4 = (w & 7) * 4;
        const int bi = tri_row_of(tt), bj = tt - bi * (bi + 1) / 2;
        const int i = bi * kB + ii, j = bj * kB + c4;
        float* d = sm + (size_t)tt * kTF + ii * kP + c4;
        if (vec && i < r && j + 3 < r) {
          const unsigned da = (unsigned)__cvta_generic_to_shared(d);
          asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(da),
                       "l"(S + (size_t)i * r + j) : "memory");
        } else {
#pragma unroll
          for (int u = 0; u < 4; ++u)
            d[u] = (i < r && j + u < r) ? S[(size_t)i * r + j + u] : (i == j + u ? 1.f : 0.f);
        }
      }
    }
    asm volatile("cp.async.wait_all;\n" ::: "memory");
    __syncthreads();
    if (shift != 0.0) {
      for (int i = threadIdx.x; i < r; i += kCT) {
        float* d = tile(i / kB, i / kB) + (i % kB) * kP + (i % kB);
        *d = (float)((double)*d + shift);
      }
    }
    if (threadIdx.x == 0) s_bad = 0;
    __syncthreads();
    if (warp == 0 && !chol_inv32(tile(0, 0), Dt, gblk(0, 0), R, col) && lane == 0) s_bad = 1;
    __syncthreads();
    bool failed = s_bad != 0;
    for (int p = 0; p < nb && !failed; ++p) {
      const int m = nb - 1 - p;
      if (m == 0) break;
      // panel: pan[b] = S(p+1+b, p) D_p^T, items (block, 8 columns)
      for (int it = warp; it < 4 * m; it += kCW) {
        const int bb = it >> 2, c0 = (it & 3) * 8;
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        rowdot8(tile(p + 1 + bb, p), Dt, c0, acc);
        float* dst = pan + (size_t)bb * kTF + lane * kP + c0;
        *reinterpret_cast<float4*>(dst) = make_float4(acc[0], acc[1], acc[2], acc[3]);
        *reinterpret_cast<float4*>(dst + 4) = make_float4(acc[4], acc[5], acc[6], acc[7]);
      }
      __syncthreads();
      // the panel blocks L_{p+1+b, p} to global memory (16-byte stores)
      for (int e = threadIdx.x; e < m * kB * 8; e += kCT) {
        const int bb = e >> 8, w = e & 255, ii = w >> 3, c4 = (w & 7) * 4;
        *reinterpret_cast<float4*>(gblk(p + 1 + bb, p) + (size_t)ii * R + c4) =
            *reinterpret_cast<const float4*>(pan + (size_t)bb * kTF + ii * kP + c4);
      }
      // look-ahead: warps 0-3 update the next diagonal block, then warp 0
      // factors it while the other warps finish the trailing update
      if (warp < 4) {
        sub_rowdot8(tile(p + 1, p + 1), pan, pan, warp * 8);
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (warp == 0 && !chol_inv32(tile(p + 1, p + 1), Dt, gblk(p + 1, p + 1), R, col) &&
            lane == 0)
          s_bad = 1;
      }
      if (warp > 0) {
        // trailing: S(p+1+bi, p+1+bj) -= pan[bi] pan[bj]^T, bj <= bi, except
        // (0, 0): whole blocks per warp
        const int tasks = m * (m + 1) / 2 - 1;
        for (int it = warp - 1; it < tasks; it += kCW - 1) {
          const int tt = it + 1;
          const int bi = tri_row_of(tt), bj = tt - bi * (bi + 1) / 2;
          sub_blk32(tile(p + 1 + bi, p + 1 + bj), pan + (size_t)bi * kTF, pan + (size_t)bj * kTF);
        }
      }
      __syncthreads();
      failed = s_bad != 0;
    }
    ok = !failed;
    __syncthreads();
  }
  if (!ok) {
    // breakdown survived the shift: L^-1 = I (the solve copies X)
    if (threadIdx.x == 0) report_status(cb.status, OUO_STATUS_BREAKDOWN);
    for (int e = threadIdx.x; e < R * R; e += kCT) {
      const int i = e / R, j = e - (e / R) * R;
      if (j / kB <= i / kB) Lb[e] = i == j ? 1.f : 0.f;
    }
  }
}


// ------------------------------------------------------------------ trinv
// Z = L^-1 (lower triangular) from the strictly lower blocks L_ij of Lb and
// the inverted diagonal blocks D_i (in Dd), block column by block column:
//   Z_jj = D_j,   Z_ij = -D_i sum_{k=j}^{i-1} L_ik Z_kj   (i > j).
// One CTA per (job, block column j), 256 threads; thread (ty, tx) owns
// rows ty + 8u (u < 4), column tx of a 32 x 32 block.  Entries outside the
// r x r matrix, and above the diagonal of a D_i, are read as zero.  The
// column is written as three planes (R x R, ld R, R = 32 ceil(r / 32)):
// Z, Z / 2 and Z - tf32(Z), the A operands of the split-tf32 product
// Y = Z X; blocks above the diagonal are zero.
constexpr int kZP = 33;  // pitch of a 32 x 32 block in shared memory

struct TrinvBatch {
  const float* Lb[kChunk];
  const float* Dd[kChunk];
  float* Z[kChunk];
  int r[kChunk];
  int64_t start[kChunk + 1];  // prefix sums of the jobs' block columns
  int njob;
};

// Ranks above 256 (streaming): the L_ik of a block row are fetched in
// groups of 8 while the column is built; shared memory holds the column,
// 8 L blocks, D_i and T.
size_t trinv_smem_bytes(int nb) { return (size_t)(nb + 8 + 2) * 32 * kZP * sizeof(float); }

__device__ __forceinline__ float tf32_trunc(float x) {
  return __uint_as_float(__float_as_uint(x) & 0xffffe000u);
}

__device__ __forceinline__ void trinv_store(const TrinvBatch& tb, int job, int j, int nb,
                                            const float* zc, int zpitch, int bstride) {
  float* Z0 = tb.Z[job];
  const int R = nb * kB;
  const size_t plane = (size_t)R * R;
  if ((zpitch & 3) == 0) {
    // 16-byte groups: four consecutive columns of a row per thread
    for (int bi = 0; bi < nb; ++bi) {
      for (int e = threadIdx.x; e < 256; e += blockDim.x) {
        const int a = e >> 3, c = (e & 7) * 4;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (bi >= j) v = *reinterpret_cast<const float4*>(zc + (size_t)bi * bstride + a * zpitch + c);
        const size_t off = (size_t)(bi * kB + a) * R + j * kB + c;
        *reinterpret_cast<float4*>(Z0 + off) = v;
        *reinterpret_cast<float4*>(Z0 + plane + off) =
            make_float4(0.5f * v.x, 0.5f * v.y, 0.5f * v.z, 0.5f * v.w);
        *reinterpret_cast<float4*>(Z0 + 2 * plane + off) =
            make_float4(v.x - tf32_trunc(v.x), v.y - tf32_trunc(v.y), v.z - tf32_trunc(v.z),
                        v.w - tf32_trunc(v.w));
      }
    }
    return;
  }
  for (int bi = 0; bi < nb; ++bi) {
    for (int e = threadIdx.x; e < 1024; e += blockDim.x) {
      const int a = e >> 5, c = e & 31;
      const float v = bi >= j ? zc[(size_t)bi * bstride + a * zpitch + c] : 0.f;
      const size_t off = (size_t)(bi * kB + a) * R + j * kB + c;
      Z0[off] = v;
      Z0[plane + off] = 0.5f * v;
      Z0[2 * plane + off] = v - tf32_trunc(v);
    }
  }
}

__global__ void __launch_bounds__(256) trinv_kernel(const __grid_constant__ TrinvBatch tb) {
  extern __shared__ float zs[];
  const int job = find_job(tb.start, tb.njob, blockIdx.x);
  const int j = (int)(blockIdx.x - tb.start[job]);
  const int r = tb.r[job], nb = (r + kB - 1) / kB, R = nb * kB;
  const float* Lb = tb.Lb[job];
  const float* Dd = tb.Dd[job];
  constexpr int kBF = 32 * kZP;  // floats of one block in shared memory
  float* zc = zs;                       // Z_kj, k = 0 .. nb-1
  float* lblk = zc + (size_t)nb * kBF;  // up to 8 L_ik
  float* dblk = lblk + 8 * kBF;         // D_i
  float* tblk = dblk + kBF;             // T
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  auto fetch = [&](float* dst, const float* src, int bi, int bj, bool lower, int e) {
    const int a = e >> 5, c = e & 31;
    const int gi = bi * kB + a, gc = bj * kB + c;
    float v = 0.f;
    if (gi < r && gc < r && (!lower || c <= a)) v = src[(size_t)gi * R + gc];
    dst[a * kZP + c] = v;
  };
  for (int e = threadIdx.x; e < 1024; e += 256) fetch(zc + (size_t)j * kBF, Dd, j, j, true, e);
  __syncthreads();
  for (int i = j + 1; i < nb; ++i) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int k0 = j; k0 < i; k0 += 8) {
      const int kn = i - k0 < 8 ? i - k0 : 8;
      // 4 loads per thread and block, all issued before any is stored
      for (int q0 = 0; q0 < kn; q0 += 4) {
        float v[16];
#pragma unroll
        for (int t = 0; t < 16; ++t) {
          const int q = q0 + (t >> 2), w = threadIdx.x + 256 * (t & 3);
          const int gi = i * kB + (w >> 5), gc = (k0 + q) * kB + (w & 31);
          v[t] = q < kn && gi < r && gc < r ? Lb[(size_t)gi * R + gc] : 0.f;
        }
#pragma unroll
        for (int t = 0; t < 16; ++t) {
          const int q = q0 + (t >> 2), w = threadIdx.x + 256 * (t & 3);
          if (q < kn) lblk[(size_t)q * kBF + (w >> 5) * kZP + (w & 31)] = v[t];
        }
      }
      __syncthreads();
      for (int q = 0; q < kn; ++q) {
        const float* lq = lblk + (size_t)q * kBF;
        const float* zq = zc + (size_t)(k0 + q) * kBF;
#pragma unroll 8
        for (int c = 0; c < 32; ++c) {
          const float zv = zq[c * kZP + tx];
#pragma unroll
          for (int u = 0; u < 4; ++u) acc[u] = fmaf(lq[(ty + 8 * u) * kZP + c], zv, acc[u]);
        }
      }
      __syncthreads();
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) tblk[(ty + 8 * u) * kZP + tx] = acc[u];
    for (int e = threadIdx.x; e < 1024; e += 256) fetch(dblk, Dd, i, i, true, e);
    __syncthreads();
    float z[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
    for (int c = 0; c < 32; ++c) {
      const float tv = tblk[c * kZP + tx];
#pragma unroll
      for (int u = 0; u < 4; ++u) z[u] = fmaf(dblk[(ty + 8 * u) * kZP + c], tv, z[u]);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) zc[(size_t)i * kBF + (ty + 8 * u) * kZP + tx] = -z[u];
    __syncthreads();
  }
  trinv_store(tb, job, j, nb, zc, kZP, kBF);
}

// Ranks up to 256 (nb <= 8), right-looking: once Z_kj is known, every
// T_i (i > k) takes its term L_ik Z_kj, and Z_{k+1,j} = -D_{k+1} T_{k+1}.
// 512 threads: the T_i updates of a step run in parallel on eight groups of
// 64 threads (T_i belongs to group i - j - 1 and stays in its registers),
// each thread a 4 x 4 tile from float4 reads (L and D stored transposed, Z
// and T by rows); the D product is spread over all threads.  All L_ik
// (k >= j) and D_i (i >= j) of the column are loaded once.
constexpr int kP4 = 36;  // pitch of a 32 x 32 block read as float4 rows
constexpr int kB4 = 32 * kP4;
size_t trinv8_smem_bytes(int nb) {
  const int m = nb;  // the column j = 0 needs the most
  return (size_t)(nb + m * (m - 1) / 2 + m + 1) * kB4 * sizeof(float);
}

constexpr int kT8 = 512;  // threads of the right-looking inverse
__global__ void __launch_bounds__(kT8, 1) trinv8_kernel(const __grid_constant__ TrinvBatch tb) {
  extern __shared__ __align__(16) float z8[];
  const int job = find_job(tb.start, tb.njob, blockIdx.x);
  const int j = (int)(blockIdx.x - tb.start[job]);
  const int r = tb.r[job], nb = (r + kB - 1) / kB, R = nb * kB;
  const float* Lb = tb.Lb[job];
  const float* Dd = tb.Dd[job];
  const int m = nb - j;
  float* zc = z8;                              // Z_kj by rows, k = 0 .. nb-1
  float* lt = zc + (size_t)nb * kB4;           // L_ik^T, j <= k < i
  float* dt = lt + (size_t)(m * (m - 1) / 2) * kB4;  // D_i^T, i >= j
  float* tb4 = dt + (size_t)m * kB4;           // T_{k+1} by rows
  auto lidx = [&](int i, int k) {
    const int a = i - j;
    return (size_t)((a * (a - 1)) / 2 + (k - j)) * kB4;
  };
  // loads: transposed copies of L_ik and D_i, Z_jj = D_j by rows; entries
  // outside the r x r matrix, and above a D_i's diagonal, are zero.  Blocks
  // go in groups of 8 (block indices decoded once per block, the same in
  // every thread); each thread issues its 16 loads of a group before it
  // stores any of them.
  {
    const int nl = m * (m - 1) / 2;
    const int nblk = nl + m + 1;
    const int w0 = threadIdx.x;  // elements w0 and w0 + 512 of every block
    int bl_a = 1, bl_q = 0;      // (a, q) of L block index `blk`, walked in order
    for (int b0 = 0; b0 < nblk; b0 += 8) {
      float v[16];
      float* dst[16];
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        const int blk = b0 + t;
        int bi = 0, bj = 0;
        bool lower = false, trans = true, valid = blk < nblk;
        float* base = nullptr;
        if (valid && blk < nl) {
          bi = j + bl_a;
          bj = j + bl_q;
          base = lt + (size_t)blk * kB4;
          if (++bl_q == bl_a) { bl_q = 0; ++bl_a; }
        } else if (valid && blk < nl + m) {
          bi = bj = j + (blk - nl);
          base = dt + (size_t)(blk - nl) * kB4;
          lower = true;
        } else if (valid) {
          bi = bj = j;
          base = zc + (size_t)j * kB4;
          lower = true;
          trans = false;
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int w = w0 + 512 * h, a = w >> 5, c = w & 31;
          const int gi = bi * kB + a, gc = bj * kB + c;
          v[2 * t + h] = valid && gi < r && gc < r && (!lower || c <= a)
                             ? (lower ? Dd : Lb)[(size_t)gi * R + gc] : 0.f;
          dst[2 * t + h] = valid ? base + (trans ? c * kP4 + a : a * kP4 + c) : nullptr;
        }
      }
#pragma unroll
      for (int t = 0; t < 16; ++t)
        if (dst[t]) *dst[t] = v[t];
    }
  }
  __syncthreads();
  const int g = threadIdx.x >> 6, gt = threadIdx.x & 63;
  const int rr = (gt >> 3) * 4, cc = (gt & 7) * 4;
  float acc[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) acc[e] = 0.f;
  // acc += A B on a 4 x 4 tile, A given transposed (At[c][row]), B by rows
  auto mac = [&](const float* At, const float* B) {
#pragma unroll 8
    for (int c = 0; c < 32; ++c) {
      const float4 a4 = *reinterpret_cast<const float4*>(At + c * kP4 + rr);
      const float4 b4 = *reinterpret_cast<const float4*>(B + c * kP4 + cc);
      const float av[4] = {a4.x, a4.y, a4.z, a4.w};
      const float bv[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[4 * u + v] = fmaf(av[u], bv[v], acc[4 * u + v]);
    }
  };
  for (int k = j; k < nb - 1; ++k) {
    const float* zk = zc + (size_t)k * kB4;
    // T_i += L_ik Z_kj for the row i = j + 1 + g this group owns
    const int i = j + 1 + g;
    if (i > k && i < nb) mac(lt + lidx(i, k), zk);
    // T_{k+1} to shared memory by its owner
    const int i1 = k + 1;
    if (g == i1 - j - 1) {
#pragma unroll
      for (int u = 0; u < 4; ++u)
        *reinterpret_cast<float4*>(tb4 + (rr + u) * kP4 + cc) =
            make_float4(acc[4 * u], acc[4 * u + 1], acc[4 * u + 2], acc[4 * u + 3]);
    }
    __syncthreads();
    // Z_{k+1,j} = -D_{k+1} T_{k+1}: thread: row tid >> 4, two columns
    {
      const int row = threadIdx.x >> 4, col = 2 * (threadIdx.x & 15);
      const float* di = dt + (size_t)(i1 - j) * kB4;
      float z0 = 0.f, z1 = 0.f;
#pragma unroll 8
      for (int c = 0; c < 32; ++c) {
        const float d = di[c * kP4 + row];
        const float2 t2 = *reinterpret_cast<const float2*>(tb4 + c * kP4 + col);
        z0 = fmaf(d, t2.x, z0);
        z1 = fmaf(d, t2.y, z1);
      }
      *reinterpret_cast<float2*>(zc + (size_t)i1 * kB4 + row * kP4 + col) = make_float2(-z0, -z1);
    }
    __syncthreads();
  }
  trinv_store(tb, job, j, nb, zc, kP4, kB4);
}

// ------------------------------------------------------------------- post
// Copies of the solve's result Y (r x L): Y2 = Y, Yt = Y^T (L x r) and its
// bf16 rounding Ytb, for the jobs that ask.  One CTA per 32 x 32 tile of Y;
// the transposes go through shared memory so that both sides are read and
// written along rows.
struct PostBatch {
  const float* Y[kChunk];
  int64_t ldy[kChunk];
  float* Y2[kChunk];
  int64_t ldy2[kChunk];
  float* Yt[kChunk];
  int64_t ldyt[kChunk];
  uint16_t* Ytb[kChunk];
  int64_t ldytb[kChunk];
  int r[kChunk];
  int64_t L[kChunk];
  int64_t start[kChunk + 1];  // prefix sums of the jobs' tiles
  int njob;
};

__global__ void __launch_bounds__(256) post_kernel(const __grid_constant__ PostBatch pb) {
  __shared__ float t[32][33];
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int64_t total = pb.start[pb.njob];
  for (int64_t g = blockIdx.x; g < total; g += gridDim.x) {
    const int job = find_job(pb.start, pb.njob, g);
    const int r = pb.r[job];
    const int64_t L = pb.L[job];
    const int64_t ntj = (L + 31) / 32;
    const int64_t tile = g - pb.start[job];
    const int ti = (int)(tile / ntj);
    const int64_t tj = tile - (int64_t)ti * ntj;
    const float* Y = pb.Y[job];
    float* Y2 = pb.Y2[job];
    float* Yt = pb.Yt[job];
    uint16_t* Ytb = pb.Ytb[job];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = ti * 32 + ty + 8 * u;
      const int64_t c = tj * 32 + tx;
      float v = 0.f;
      if (i < r && c < L) {
        v = Y[(int64_t)i * pb.ldy[job] + c];
        if (Y2) Y2[(int64_t)i * pb.ldy2[job] + c] = v;
      }
      t[ty + 8 * u][tx] = v;
    }
    __syncthreads();
    if (Yt || Ytb) {
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int64_t c = tj * 32 + ty + 8 * u;  // row of Y^T
        const int i = ti * 32 + tx;              // column of Y^T
        if (c < L && i < r) {
          const float v = t[tx][ty + 8 * u];
          if (Yt) Yt[c * pb.ldyt[job] + i] = v;
          if (Ytb) Ytb[c * pb.ldytb[job] + i] = f32_to_bf16(v);
        }
      }
    }
    __syncthreads();
  }
}

// ------------------------------------------------------------------- rows
struct RowsBatch {
  RowsJob job[kChunk];
  int64_t start[kChunk + 1];  // first row of every job
  int njob;
  float eps;
};

__global__ void __launch_bounds__(256) rows_kernel(const __grid_constant__ RowsBatch rb) {
  __shared__ double red[8];
  const int j = find_job(rb.start, rb.njob, blockIdx.x);
  const RowsJob& jb = rb.job[j];
  const int64_t c = blockIdx.x - rb.start[j];
  const int64_t n = jb.n;
  const float* src = jb.part + c * jb.ldp;
  const bool vec = (jb.ldp & 3) == 0 && (jb.sp & 3) == 0 && ((uintptr_t)jb.part & 15) == 0 &&
                   (!jb.out || ((jb.ldo & 3) == 0 && ((uintptr_t)jb.out & 15) == 0)) &&
                   (!jb.outb || ((jb.ldob & 3) == 0 && ((uintptr_t)jb.outb & 7) == 0));
  uint16_t* brow = jb.outb ? jb.outb + c * jb.ldob : nullptr;
  const bool want_norm = jb.sigma || jb.qn;
  double ss = 0.0;
  float* orow = jb.out ? jb.out + c * jb.ldo : nullptr;
  if (vec) {
    for (int64_t e = 4 * (int64_t)threadIdx.x; e < (n & ~3LL); e += 4 * blockDim.x) {
      float4 v = *reinterpret_cast<const float4*>(src + e);
      for (int q = 1; q < jb.ks; ++q) {
        const float4 w = *reinterpret_cast<const float4*>(src + q * jb.sp + e);
        v.x += w.x; v.y += w.y; v.z += w.z; v.w += w.w;
      }
      if (orow) *reinterpret_cast<float4*>(orow + e) = v;
      if (brow) {
        uint2 u;
        u.x = pack_bf16x2(v.x, v.y);
        u.y = pack_bf16x2(v.z, v.w);
        *reinterpret_cast<uint2*>(brow + e) = u;
      }
      if (want_norm)
        ss += (double)v.x * v.x + (double)v.y * v.y + (double)v.z * v.z + (double)v.w * v.w;
    }
  }
  for (int64_t e = (vec ? (n & ~3LL) : 0) + threadIdx.x; e < n; e += blockDim.x) {
    float v = src[e];
    for (int q = 1; q < jb.ks; ++q) v += src[q * jb.sp + e];
    if (orow) orow[e] = v;
    if (brow) brow[e] = f32_to_bf16(v);
    if (want_norm) ss += (double)v * v;
  }
  if (!want_norm) return;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  double tot = 0.0;
  for (int w = 0; w < 8; ++w) tot += red[w];
  const double nrm = sqrt(tot);
  if (jb.sigma && threadIdx.x == 0) jb.sigma[c] = (float)nrm;
  if (!jb.qn) return;
  const float inv = (float)(1.0 / (nrm + (double)rb.eps));
  // the summed row is read back from where this thread wrote it (orow), or
  // summed again from the partials
  for (int64_t e = threadIdx.x; e < n; e += blockDim.x) {
    float v;
    if (orow) {
      v = orow[e];
    } else {
      v = src[e];
      for (int q = 1; q < jb.ks; ++q) v += src[q * jb.sp + e];
    }
    const float qv = v * inv;
    jb.qn[c * jb.ldq + e] = qv;
    if (jb.q2) jb.q2[c * jb.ldq2 + e] = qv;
  }
}

unsigned grid_cap(int64_t n, int per_block) {
  int64_t b = ceil_div(n, per_block);
  const int64_t cap = (int64_t)num_sms() * 8;
  if (b > cap) b = cap;
  return (unsigned)(b < 1 ? 1 : b);
}

int set_smem_attr(const void* fn, size_t bytes) {
  static int done[64][4] = {{0}};
  int dev = 0;
  OUO_CHECK_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return set_error(OUO_ERR_UNSUPPORTED, "device ordinal %d", dev);
  const int slot = fn == (const void*)chol_kernel ? 0 : fn == (const void*)trinv_kernel ? 1 : 2;
  if (!done[dev][slot]) {
    const size_t b = slot == 0 ? chol_smem_bytes(kMaxNb)
                   : slot == 1 ? trinv_smem_bytes(1024 / kB) : trinv8_smem_bytes(8);
    OUO_CHECK_CUDA(cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)b));
    done[dev][slot] = 1;
  }
  (void)bytes;
  return OUO_OK;
}

}  // namespace

namespace {
// Distance in floats from a to b (addresses compared as integers: the two
// may lie in different allocations), and whether b sits d * step floats
// after a.
int64_t fdist(const void* a, const void* b) {
  return ((int64_t)(uintptr_t)b - (int64_t)(uintptr_t)a) / (int64_t)sizeof(float);
}
bool at_step(const void* a, const void* b, int64_t d, int64_t step) {
  return (int64_t)(uintptr_t)b - (int64_t)(uintptr_t)a == d * step * (int64_t)sizeof(float);
}
}  // namespace

int cholqr_gram_ksplit(int r, int64_t L) {
  (void)r;
  // K ranges of at least 32 tf32 K blocks (the two passes counted), at
  // most 64: a lone matrix spreads over enough CTAs to keep the Gram short,
  // and a large batch writes few partials.  Depends on L alone.
  const int64_t nkv = 2 * ceil_div(L, (int64_t)32);
  int64_t want = nkv / 32;
  if (want < 1) want = 1;
  if (want > 64) want = 64;
  return gemm_ksplit_used(L, (int)want, OUO_F32, 2);
}

int64_t cholqr_gram_part_floats(int r, int64_t L) {
  return (int64_t)cholqr_gram_ksplit(r, L) * r * ((r + 3) & ~3);
}

int cholqr_gram(const std::vector<CholQrJob>& jobs, int* status, cudaStream_t s) {
  if (jobs.empty()) return OUO_OK;
  // residuals
  for (size_t c0 = 0; c0 < jobs.size(); c0 += kChunk) {
    const int cn = (int)(jobs.size() - c0 < (size_t)kChunk ? jobs.size() - c0 : kChunk);
    LoBatch lb;
    lb.njob = cn;
    lb.start[0] = 0;
    for (int i = 0; i < cn; ++i) {
      const CholQrJob& jb = jobs[c0 + i];
      if ((jb.ldx & 3) || ((uintptr_t)jb.X & 15) || ((uintptr_t)jb.Xlo & 15))
        return set_error(OUO_ERR_INVALID_ARG, "Gram operands need 16-byte rows");
      lb.X[i] = jb.X;
      lb.lo[i] = jb.Xlo;
      lb.ld[i] = jb.ldx;
      lb.L[i] = jb.L;
      lb.start[i + 1] = lb.start[i] + jb.r;
    }
    lo_kernel<<<(unsigned)lb.start[cn], 256, 0, s>>>(lb);
    OUO_CHECK_LAUNCH();
  }
  // partial Gram matrices: one two-pass GEMM descriptor per run of jobs
  // that sit evenly strided in memory (the members of a group)
  std::vector<GemmDesc> ds;
  size_t k = 0;
  while (k < jobs.size()) {
    const CholQrJob& j0 = jobs[k];
    const int ks = cholqr_gram_ksplit(j0.r, j0.L);
    const int64_t ldp = (j0.r + 3) & ~3;
    const int64_t pf = (int64_t)ks * j0.r * ldp;
    size_t e = k + 1;
    int64_t xs = 0, ls = 0;
    if (e < jobs.size()) {
      xs = fdist(j0.X, jobs[e].X);
      ls = fdist(j0.Xlo, jobs[e].Xlo);
    }
    while (e < jobs.size()) {
      const CholQrJob& je = jobs[e];
      const int64_t d = (int64_t)(e - k);
      if (je.r != j0.r || je.L != j0.L || je.ldx != j0.ldx || xs < j0.r * j0.ldx ||
          xs != ls || !at_step(j0.X, je.X, d, xs) || !at_step(j0.Xlo, je.Xlo, d, ls) ||
          !at_step(j0.gpart, je.gpart, d, pf))
        break;
      ++e;
    }
    const int64_t cnt = (int64_t)(e - k);
    if (cnt == 1) xs = j0.r * j0.ldx;
    GemmDesc d;
    d.M = j0.r; d.N = j0.r; d.K = j0.L; d.nb = cnt;
    Buf x;
    x.p = reinterpret_cast<char*>(const_cast<float*>(j0.X));
    x.dtype = OUO_F32;
    x.rows = j0.r;
    x.cols = j0.L;
    x.ld = j0.ldx;
    x.stride = xs;
    x.nb = cnt;
    d.A = x;
    d.B = x;
    d.B2 = x;
    d.B2.p = reinterpret_cast<char*>(j0.Xlo);
    d.npass = 2;
    d.b_lo = 2;  // pass 1 reads B from the residuals
    d.has_f32 = true;
    Buf o;
    o.p = reinterpret_cast<char*>(j0.gpart);
    o.dtype = OUO_F32;
    o.rows = j0.r;
    o.cols = j0.r;
    o.ld = ldp;
    o.stride = j0.r * ldp;
    o.nb = cnt * ks;
    d.out_f32 = o;
    d.ksplit = ks;
    d.per_desc_tiles = true;
    ds.push_back(d);
    k = e;
  }
  OUO_TRY(gemm_umma_grouped(ds, s, status));
  for (size_t c0 = 0; c0 < jobs.size(); c0 += kChunk) {
    const int cn = (int)(jobs.size() - c0 < (size_t)kChunk ? jobs.size() - c0 : kChunk);
    SumBatch sb;
    sb.njob = cn;
    sb.start[0] = 0;
    for (int i = 0; i < cn; ++i) {
      const CholQrJob& jb = jobs[c0 + i];
      sb.part[i] = jb.gpart;
      sb.S[i] = jb.S;
      sb.r[i] = jb.r;
      sb.splits[i] = cholqr_gram_ksplit(jb.r, jb.L);
      const int64_t nt = ceil_div(jb.r, 32);
      sb.start[i + 1] = sb.start[i] + nt * (nt + 1) / 2;
    }
    sum_kernel<<<(unsigned)sb.start[cn], 256, 0, s>>>(sb);
    OUO_CHECK_LAUNCH();
  }
  return OUO_OK;
}

bool cholqr_small_rank(int r) { return r >= 1 && r <= kMaxNb * kB; }

int cholqr_factor(const std::vector<CholQrJob>& jobs, int* status, cudaStream_t s) {
  OUO_TRY(set_smem_attr((const void*)chol_kernel, 0));
  for (size_t c0 = 0; c0 < jobs.size(); c0 += kChunk) {
    const int cn = (int)(jobs.size() - c0 < (size_t)kChunk ? jobs.size() - c0 : kChunk);
    CholBatch cb;
    cb.njob = cn;
    cb.status = status;
    int nbmax = 1;
    for (int i = 0; i < cn; ++i) {
      const CholQrJob& jb = jobs[c0 + i];
      if (!cholqr_small_rank(jb.r))
        return set_error(OUO_ERR_UNSUPPORTED, "one-CTA Cholesky takes r <= %d", kMaxNb * kB);
      cb.S[i] = jb.S;
      cb.Lb[i] = jb.Lb;
      cb.r[i] = jb.r;
      cb.L[i] = jb.L;
      const int nb = (int)ceil_div(jb.r, kB);
      if (nb > nbmax) nbmax = nb;
    }
    chol_kernel<<<cn, kCT, chol_smem_bytes(nbmax), s>>>(cb);
    OUO_CHECK_LAUNCH();
  }
  return OUO_OK;
}

size_t cholqr_z_floats(int r) {
  const size_t R = (size_t)ceil_div(r, kB) * kB;
  return 3 * R * R;
}

int cholqr_apply(const std::vector<CholQrJob>& jobs, int* status, cudaStream_t s) {
  if (jobs.empty()) return OUO_OK;
  OUO_TRY(set_smem_attr((const void*)trinv_kernel, 0));
  OUO_TRY(set_smem_attr((const void*)trinv8_kernel, 0));
  // Z = L^-1 in three planes: ranks up to 256 on the right-looking kernel,
  // larger ones on the streaming kernel
  for (int big = 0; big < 2; ++big) {
    std::vector<const CholQrJob*> sel;
    for (const CholQrJob& jb : jobs) {
      const int nb = (int)ceil_div(jb.r, kB);
      if (nb * kB > 1024) return set_error(OUO_ERR_UNSUPPORTED, "triangular solve takes r <= 1024");
      if (!jb.Z || jb.Y == jb.X)
        return set_error(OUO_ERR_INVALID_ARG, "solve needs Z and an output apart from X");
      if ((nb > 8) == (big == 1)) sel.push_back(&jb);
    }
    for (size_t c0 = 0; c0 < sel.size(); c0 += kChunk) {
      const int cn = (int)(sel.size() - c0 < (size_t)kChunk ? sel.size() - c0 : kChunk);
      TrinvBatch tb;
      tb.njob = cn;
      tb.start[0] = 0;
      int nbmax = 1;
      for (int i = 0; i < cn; ++i) {
        const CholQrJob& jb = *sel[c0 + i];
        const int nb = (int)ceil_div(jb.r, kB);
        if (nb > nbmax) nbmax = nb;
        tb.Lb[i] = jb.Lb;
        tb.Dd[i] = jb.Dd ? jb.Dd : jb.Lb;
        tb.Z[i] = jb.Z;
        tb.r[i] = jb.r;
        tb.start[i + 1] = tb.start[i] + nb;
      }
      if (big) trinv_kernel<<<(unsigned)tb.start[cn], 256, trinv_smem_bytes(nbmax), s>>>(tb);
      else trinv8_kernel<<<(unsigned)tb.start[cn], kT8, trinv8_smem_bytes(nbmax), s>>>(tb);
      OUO_CHECK_LAUNCH();
    }
  }
  // Y = Z X in three split-tf32 passes, (Z, X), (Z / 2, 2 lo), (Z - tf32(Z), X):
  // tf32(Z) tf32(X) + tf32(Z) lo + (Z - tf32(Z)) tf32(X).  One descriptor per
  // run of jobs laid out evenly (the members of a group).
  std::vector<GemmDesc> ds;
  size_t k = 0;
  while (k < jobs.size()) {
    const CholQrJob& j0 = jobs[k];
    const int64_t zf = (int64_t)cholqr_z_floats(j0.r);
    size_t e = k + 1;
    int64_t xs = 0, ys = 0, ls = 0, zs = 0;
    if (e < jobs.size()) {
      xs = fdist(j0.X, jobs[e].X);
      ys = fdist(j0.Y, jobs[e].Y);
      ls = fdist(j0.Xlo, jobs[e].Xlo);
      zs = fdist(j0.Z, jobs[e].Z);
    }
    while (e < jobs.size()) {
      const CholQrJob& je = jobs[e];
      const int64_t d = (int64_t)(e - k);
      if (je.r != j0.r || je.L != j0.L || je.ldx != j0.ldx || je.ldy != j0.ldy ||
          xs < j0.r * j0.ldx || ys < j0.r * j0.ldy || xs != ls || zs != zf ||
          !at_step(j0.X, je.X, d, xs) || !at_step(j0.Xlo, je.Xlo, d, ls) ||
          !at_step(j0.Y, je.Y, d, ys) || !at_step(j0.Z, je.Z, d, zs))
        break;
      ++e;
    }
    const int64_t cnt = (int64_t)(e - k);
    if (cnt == 1) {
      xs = j0.r * j0.ldx;
      ys = j0.r * j0.ldy;
    }
    const int64_t R = ceil_div(j0.r, kB) * kB;
    GemmDesc d;
    d.M = j0.r; d.N = j0.L; d.K = j0.r; d.nb = cnt;
    Buf z;
    z.p = reinterpret_cast<char*>(j0.Z);
    z.dtype = OUO_F32;
    z.rows = j0.r;
    z.cols = j0.r;
    z.ld = R;
    z.stride = zf;
    z.nb = cnt;
    d.A = z;
    d.A2 = z;
    d.A2.p = reinterpret_cast<char*>(j0.Z + R * R);
    d.A3 = z;
    d.A3.p = reinterpret_cast<char*>(j0.Z + 2 * R * R);
    Buf x;
    x.p = reinterpret_cast<char*>(const_cast<float*>(j0.X));
    x.dtype = OUO_F32;
    x.rows = j0.r;
    x.cols = j0.L;
    x.ld = j0.ldx;
    x.stride = xs;
    x.nb = cnt;
    d.B = x;
    d.B2 = x;
    d.B2.p = reinterpret_cast<char*>(j0.Xlo);
    d.b_mn = 1;
    d.npass = 3;
    d.a_lo = 2;   // pass 1: Z / 2 against the residuals (stored doubled)
    d.b_lo = 2;
    d.a_lo2 = 4;  // pass 2: Z - tf32(Z) against X
    d.has_f32 = true;
    Buf o;
    o.p = reinterpret_cast<char*>(j0.Y);
    o.dtype = OUO_F32;
    o.rows = j0.r;
    o.cols = j0.L;
    o.ld = j0.ldy;
    o.stride = ys;
    o.nb = cnt;
    d.out_f32 = o;
    d.per_desc_tiles = true;
    d.pair_mn = true;
    ds.push_back(d);
    k = e;
  }
  OUO_TRY(gemm_umma_grouped(ds, s, status));
  // copies and transposes of Y
  std::vector<const CholQrJob*> post;
  for (const CholQrJob& jb : jobs)
    if (jb.Y2 || jb.Yt || jb.Ytb) post.push_back(&jb);
  for (size_t c0 = 0; c0 < post.size(); c0 += kChunk) {
    const int cn = (int)(post.size() - c0 < (size_t)kChunk ? post.size() - c0 : kChunk);
    PostBatch pb;
    pb.njob = cn;
    pb.start[0] = 0;
    for (int i = 0; i < cn; ++i) {
      const CholQrJob& jb = *post[c0 + i];
      pb.Y[i] = jb.Y;
      pb.ldy[i] = jb.ldy;
      pb.Y2[i] = jb.Y2;
      pb.ldy2[i] = jb.ldy2;
      pb.Yt[i] = jb.Yt;
      pb.ldyt[i] = jb.ldyt;
      pb.Ytb[i] = jb.Ytb;
      pb.ldytb[i] = jb.ldytb;
      pb.r[i] = jb.r;
      pb.L[i] = jb.L;
      pb.start[i + 1] = pb.start[i] + ceil_div(jb.r, 32) * ceil_div(jb.L, 32);
    }
    post_kernel<<<grid_cap(pb.start[cn], 1), 256, 0, s>>>(pb);
    OUO_CHECK_LAUNCH();
  }
  return OUO_OK;
}

int rows_reduce(const std::vector<RowsJob>& jobs, float eps, cudaStream_t s) {
  for (size_t c0 = 0; c0 < jobs.size(); c0 += kChunk) {
    const int cn = (int)(jobs.size() - c0 < (size_t)kChunk ? jobs.size() - c0 : kChunk);
    RowsBatch rb;
    rb.njob = cn;
    rb.eps = eps;
    rb.start[0] = 0;
    for (int i = 0; i < cn; ++i) {
      rb.job[i] = jobs[c0 + i];
      rb.start[i + 1] = rb.start[i] + jobs[c0 + i].rows;
    }
    if (rb.start[cn] == 0) continue;
    rows_kernel<<<(unsigned)rb.start[cn], 256, 0, s>>>(rb);
    OUO_CHECK_LAUNCH();
  }
  return OUO_OK;
}

}  // namespace ouo
