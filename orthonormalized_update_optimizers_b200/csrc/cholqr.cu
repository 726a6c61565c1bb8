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
//   trsm     Y = L^-1 X by block forward substitution, one CTA per 32-column
//            strip of X: Y_i = D_i (X_i - sum_{k<i} L_ik Y_k).  Optional
//            second copy and transposed copy of Y.
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
        // trailing: S(p+1+bi, p+1+bj) -= pan[bi] pan[bj]^T, bj <= bi, except (0, 0)
        const int tasks = m * (m + 1) / 2 - 1;
        for (int it = warp - 1; it < 4 * tasks; it += kCW - 1) {
          const int tt = (it >> 2) + 1, c0 = (it & 3) * 8;
          const int bi = tri_row_of(tt), bj = tt - bi * (bi + 1) / 2;
          sub_rowdot8(tile(p + 1 + bi, p + 1 + bj), pan + (size_t)bi * kTF,
                      pan + (size_t)bj * kTF, c0);
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

// ------------------------------------------------------------------- trsm
constexpr int kSP = 36;  // row pitch of the strip and block buffers (floats)

struct TrsmBatch {
  CholQrJob job[kChunk];
  int64_t start[kChunk + 1];  // first strip of every job
  int njob;
};

__device__ __forceinline__ void cp_async16(float* dst, const float* src) {
  const unsigned d = (unsigned)__cvta_generic_to_shared(dst);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(d), "l"(src) : "memory");
}

// Y = L^-1 X on one 32-column strip, block row by block row:
//   Y_i = D_i X_i;  X_j -= L_ji Y_i for the blocks j > i below.
// The products run in rounds: a round is D_i X_i, or up to four updates
// L_ji Y_i, one per group of 64 threads (a thread owns rows ro, ro+8,
// ro+16, ro+24 and four columns of a 32 x 32 block).  The blocks of L a
// round needs are copied into shared memory (cp.async) one round ahead.
__global__ void __launch_bounds__(256) trsm_kernel(const __grid_constant__ TrsmBatch tb) {
  extern __shared__ __align__(16) float sm[];
  const int job = find_job(tb.start, tb.njob, blockIdx.x);
  const CholQrJob& jb = tb.job[job];
  const int64_t c0g = (blockIdx.x - tb.start[job]) * kB;  // first column of the strip
  const int r = jb.r, nb = (r + kB - 1) / kB, R = nb * kB;
  float* xs = sm;                                   // R x kSP
  float* blk = sm + (size_t)R * kSP;                // [2][4][32][kSP]
  const int tid = threadIdx.x, grp = tid >> 6, t64 = tid & 63;
  const int ro = t64 >> 3, cc = 4 * (t64 & 7);
  const int64_t ncol = jb.L - c0g < kB ? jb.L - c0g : kB;
  const float* Lb = jb.Lb;
  const float* Dd = jb.Dd ? jb.Dd : jb.Lb;
  // rounds: for every block row i, one D round, then ceil((nb-1-i)/4)
  // update rounds
  auto round_of = [&](int t, int* i, int* j0) {
    for (int b = 0; b < nb; ++b) {
      const int nu = (nb - 1 - b + 3) / 4;
      if (t == 0) { *i = b; *j0 = -1; return; }
      if (t <= nu) { *i = b; *j0 = b + 1 + 4 * (t - 1); return; }
      t -= 1 + nu;
    }
    *i = -1;
    *j0 = -1;
  };
  int nrounds = 0;
  for (int b = 0; b < nb; ++b) nrounds += 1 + (nb - 1 - b + 3) / 4;
  auto prefetch = [&](int t) {
    if (t >= nrounds) return;
    int i, j0;
    round_of(t, &i, &j0);
    float* dst = blk + (size_t)(t & 1) * 4 * kB * kSP;
    // thread: row tid >> 3, 16-byte column group tid & 7 of each block
    const int br = tid >> 3, bc = 4 * (tid & 7);
    if (j0 < 0) {
      cp_async16(dst + br * kSP + bc, Dd + (size_t)(i * kB + br) * R + i * kB + bc);
    } else {
      for (int g = 0; g < 4 && j0 + g < nb; ++g)
        cp_async16(dst + (size_t)g * kB * kSP + br * kSP + bc,
                   Lb + (size_t)((j0 + g) * kB + br) * R + i * kB + bc);
    }
  };
  prefetch(0);
  asm volatile("cp.async.commit_group;\n" ::: "memory");
  // strip in: xs[i][c] = X[i][c0g + c], zero past r or L
  {
    const bool vec = (jb.ldx & 3) == 0 && ((uintptr_t)jb.X & 15) == 0 && ncol == kB;
    for (int e = tid; e < R * 8; e += 256) {
      const int i = e >> 3, c = (e & 7) * 4;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (i < r) {
        const float* src = jb.X + (int64_t)i * jb.ldx + c0g + c;
        if (vec) {
          v = *reinterpret_cast<const float4*>(src);
        } else {
          float t4[4] = {0.f, 0.f, 0.f, 0.f};
          for (int q = 0; q < 4; ++q)
            if (c + q < ncol) t4[q] = src[q];
          v = make_float4(t4[0], t4[1], t4[2], t4[3]);
        }
      }
      *reinterpret_cast<float4*>(xs + i * kSP + c) = v;
    }
  }
  for (int t = 0; t < nrounds; ++t) {
    prefetch(t + 1);
    asm volatile("cp.async.commit_group;\n" ::: "memory");
    asm volatile("cp.async.wait_group 1;\n" ::: "memory");
    __syncthreads();
    int i, j0;
    round_of(t, &i, &j0);
    const float* bb = blk + (size_t)(t & 1) * 4 * kB * kSP + (size_t)grp * kB * kSP;
    const bool active = j0 < 0 ? grp == 0 : j0 + grp < nb;
    float acc[4][4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int v = 0; v < 4; ++v) acc[u][v] = 0.f;
    if (active) {
      const float* yi = xs + (size_t)(i * kB) * kSP + cc;
#pragma unroll 2
      for (int k = 0; k < kB; k += 4) {
        float a[4][4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float4 w = *reinterpret_cast<const float4*>(bb + (ro + 8 * u) * kSP + k);
          a[u][0] = w.x; a[u][1] = w.y; a[u][2] = w.z; a[u][3] = w.w;
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float4 y = *reinterpret_cast<const float4*>(yi + (k + q) * kSP);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            acc[u][0] = fmaf(a[u][q], y.x, acc[u][0]);
            acc[u][1] = fmaf(a[u][q], y.y, acc[u][1]);
            acc[u][2] = fmaf(a[u][q], y.z, acc[u][2]);
            acc[u][3] = fmaf(a[u][q], y.w, acc[u][3]);
          }
        }
      }
    }
    if (j0 < 0) {
      __syncthreads();  // every read of X_i is done before Y_i replaces it
      if (active) {
#pragma unroll
        for (int u = 0; u < 4; ++u)
          *reinterpret_cast<float4*>(xs + (size_t)(i * kB + ro + 8 * u) * kSP + cc) =
              make_float4(acc[u][0], acc[u][1], acc[u][2], acc[u][3]);
      }
    } else if (active) {
      const int jb2 = j0 + grp;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        float* xp = xs + (size_t)(jb2 * kB + ro + 8 * u) * kSP + cc;
        float4 x = *reinterpret_cast<float4*>(xp);
        x.x -= acc[u][0]; x.y -= acc[u][1]; x.z -= acc[u][2]; x.w -= acc[u][3];
        *reinterpret_cast<float4*>(xp) = x;
      }
    }
    __syncthreads();
  }
  asm volatile("cp.async.wait_group 0;\n" ::: "memory");
  // out: Y (and its copy) row-major, Y^T (L x r)
  for (int e = tid; e < r * 8; e += 256) {
    const int i = e >> 3, c = (e & 7) * 4;
    const float4 v = *reinterpret_cast<const float4*>(xs + i * kSP + c);
    const float vv[4] = {v.x, v.y, v.z, v.w};
    float* outs[2] = {jb.Y, jb.Y2};
    const int64_t lds[2] = {jb.ldy, jb.ldy2};
#pragma unroll
    for (int o = 0; o < 2; ++o) {
      if (!outs[o]) continue;
      float* dst = outs[o] + (int64_t)i * lds[o] + c0g + c;
      if (ncol == kB && (lds[o] & 3) == 0 && ((uintptr_t)outs[o] & 15) == 0) {
        *reinterpret_cast<float4*>(dst) = v;
      } else {
        for (int q = 0; q < 4; ++q)
          if (c + q < ncol) dst[q] = vv[q];
      }
    }
  }
  if (jb.Yt || jb.Ytb) {
    for (int c = 0; c < ncol; ++c)
      for (int i = tid; i < r; i += 256) {
        const float v = xs[i * kSP + c];
        if (jb.Yt) jb.Yt[(c0g + c) * jb.ldyt + i] = v;
        if (jb.Ytb) jb.Ytb[(c0g + c) * jb.ldytb + i] = f32_to_bf16(v);
      }
  }
}

size_t trsm_smem_bytes(int R) { return ((size_t)R * kSP + 2 * 4 * kB * kSP) * sizeof(float); }

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
  const int slot = fn == (const void*)chol_kernel ? 0 : 1;
  if (!done[dev][slot]) {
    OUO_CHECK_CUDA(cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        slot == 0 ? (int)chol_smem_bytes(kMaxNb)
                                                  : (int)trsm_smem_bytes(1024)));
    done[dev][slot] = 1;
  }
  (void)bytes;
  return OUO_OK;
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
      xs = jobs[e].X - j0.X;
      ls = jobs[e].Xlo - j0.Xlo;
    }
    while (e < jobs.size()) {
      const CholQrJob& je = jobs[e];
      const int64_t d = (int64_t)(e - k);
      if (je.r != j0.r || je.L != j0.L || je.ldx != j0.ldx || xs < j0.r * j0.ldx ||
          xs != ls || je.X != j0.X + d * xs || je.Xlo != j0.Xlo + d * ls ||
          je.gpart != j0.gpart + d * pf)
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

int cholqr_apply(const std::vector<CholQrJob>& jobs, cudaStream_t s) {
  OUO_TRY(set_smem_attr((const void*)trsm_kernel, 0));
  for (size_t c0 = 0; c0 < jobs.size(); c0 += kChunk) {
    const int cn = (int)(jobs.size() - c0 < (size_t)kChunk ? jobs.size() - c0 : kChunk);
    TrsmBatch tb;
    tb.njob = cn;
    tb.start[0] = 0;
    int Rmax = kB;
    for (int i = 0; i < cn; ++i) {
      const CholQrJob& jb = jobs[c0 + i];
      const int R = (int)(ceil_div(jb.r, kB) * kB);
      if (R > 1024) return set_error(OUO_ERR_UNSUPPORTED, "triangular solve takes r <= 1024");
      if (R > Rmax) Rmax = R;
      tb.job[i] = jb;
      tb.start[i + 1] = tb.start[i] + ceil_div(jb.L, kB);
    }
    trsm_kernel<<<(unsigned)tb.start[cn], 256, trsm_smem_bytes(Rmax), s>>>(tb);
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
