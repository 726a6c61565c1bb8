// Blocked Cholesky factorization for CholeskyQR on ranks above 256: one
// cooperative multi-CTA launch (chol_blocked).  Ranks up to 256 take the
// one-CTA kernel of cholqr.cu.
//
// Source: "Orth-Dion: Eliminating Geometric Mismatch in Distributed Low-Rank
// Spectral Optimization", Orth-Dion (the right factor, and in Dion the left
// factor, is orthonormalized by QR); the QR is computed as CholeskyQR: the
// Gram matrix S = X X^T of the r x L row block X is factored S = L L^T and the
// rows L^-1 X are orthonormal, with the implied R = L^T on a positive
// diagonal (the unique QR).
//
// S arrives as `splits` partial Gram matrices in upper storage (entry (i, j)
// valid for j >= i), summed here in float64 in a fixed order.  The r x r
// problem is padded to R = 32 * ceil(r / 32) with an identity block and
// processed in 32 x 32 blocks:
//   for each block column p:
//     the diagonal block S_pp = L_pp L_pp^T is factored and inverted
//       (D_p = L_pp^-1) by one warp, in registers, in every CTA that needs
//       it (identical bits), and published by CTA 0;
//     the blocks below it become L_ip = S_ip D_p^T;
//     the trailing lower blocks are updated S_ij -= L_ip L_jp^T.
// The strictly lower blocks L_ij stay in S and the inverted diagonal blocks
// D_p go to the diagonal blocks of Linv: the form the block inverse of
// cholqr.cu reads.  Phases are separated by a grid barrier whose wait is
// bounded in time (a barrier that runs out sets OUO_STATUS_TIMEOUT and
// every later barrier passes at once).  A non-positive pivot restarts the
// factorization once with the shift of shifted CholeskyQR,
// 11 (L r + r (r + 1)) u tr(S); a second failure sets OUO_STATUS_BREAKDOWN
// and returns L = I.
#include <atomic>
#include <cmath>

#include "internal.h"

namespace ouo {
namespace {

constexpr int kNb = 32;
constexpr int kCholThreads = 256;

struct CholBArgs {
  const float* part;  // [splits][r][r]
  int splits;
  int r, R, nblk;     // size, padded size, blocks per side
  int64_t L;          // row length of X (for the shift)
  float* S;           // R x R scratch (ld R), lower blocks used
  float* Linv;        // R x R output (ld R), lower triangular
  unsigned* bar;      // grid barrier counter, zero at launch
  int* flags;         // [0] pivot failed, [1] barrier timed out
  double* diag;       // unshifted diagonal of S (r values)
  int* status;
};

// Grid-wide barrier over all CTAs of the cooperative launch; the wait is
// bounded and gives up for good once any CTA has timed out.
__device__ void grid_barrier(const CholBArgs& a) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const unsigned n = gridDim.x;
    const unsigned ticket = atomicAdd(a.bar, 1u);
    const unsigned target = (ticket / n + 1u) * n;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
      const unsigned v = *reinterpret_cast<volatile unsigned*>(a.bar);
      if (v >= target) break;
      if (*reinterpret_cast<volatile int*>(&a.flags[1])) break;
      if (globaltimer_ns() - t0 > kWaitLimitNs) {
        atomicExch(&a.flags[1], 1);
        break;
      }
    }
    __threadfence();
  }
  __syncthreads();
}

__device__ __forceinline__ float* blk(float* base, int R, int bi, int bj) {
  return base + (size_t)bi * kNb * R + (size_t)bj * kNb;
}

// 32 x 32 block from global (ld R) into shared memory tile [32][33].
__device__ __forceinline__ void load_blk(float (*t)[kNb + 1], const float* g, int R) {
  for (int e = threadIdx.x; e < kNb * kNb; e += blockDim.x) {
    const int i = e >> 5, j = e & 31;
    t[i][j] = g[(size_t)i * R + j];
  }
}

// S = sum of the partials (float64, fixed order) + shift on the diagonal,
// padded with an identity block; the upper blocks of Linv are zeroed.
__device__ void assemble(const CholBArgs& a, float shift) {
  const size_t total = (size_t)a.R * a.R;
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (size_t)gridDim.x * blockDim.x) {
    const int i = (int)(e / a.R), j = (int)(e - (e / a.R) * a.R);
    if (j > i) {
      a.Linv[e] = 0.f;
      continue;
    }
    float v;
    if (i < a.r) {
      double s = 0.0;  // (i, j), j <= i, is stored at (j, i)
      for (int p = 0; p < a.splits; ++p)
        s += (double)a.part[(size_t)p * a.r * a.r + (size_t)j * a.r + i];
      if (i == j) {
        a.diag[i] = s;
        s += (double)shift;
      }
      v = (float)s;
    } else {
      v = i == j ? 1.f : 0.f;
    }
    a.S[e] = v;
  }
}

// Warp 0 factors the 32 x 32 lower block at g (ld R), one row per lane in
// registers: l = row `lane` of L_pp, x = column `lane` of D_p = L_pp^-1.
// Every CTA that runs it computes the same bits.  Returns false on a bad
// pivot (the same in every lane).
__device__ __forceinline__ bool warp_chol32(const float* g, int R, float (&l)[kNb],
                                            float (&x)[kNb]) {
  const unsigned full = 0xffffffffu;
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int j = 0; j < kNb; ++j) l[j] = g[(size_t)lane * R + j];
#pragma unroll
  for (int k = 0; k < kNb; ++k) {
    const float piv = __shfl_sync(full, l[k], k);
    if (!(piv > 0.f) || !isfinite(piv)) return false;
    const float d = sqrtf(piv);
    const float inv = 1.0f / d;
    if (lane > k) l[k] *= inv;
    else if (lane == k) l[k] = d;
#pragma unroll
    for (int j = k + 1; j < kNb; ++j) {
      const float ljk = __shfl_sync(full, l[k], j);  // L[j][k] from lane j
      if (j <= lane) l[j] -= l[k] * ljk;
    }
  }
  // lane c: column c of L^-1 by forward substitution
#pragma unroll
  for (int r = 0; r < kNb; ++r) {
    float s = r == lane ? 1.f : 0.f;
#pragma unroll
    for (int k = 0; k < r; ++k) s -= __shfl_sync(full, l[k], r) * x[k];
    const float lrr = __shfl_sync(full, l[r], r);
    x[r] = r < lane ? 0.f : s / lrr;
  }
  return true;
}

// Factor diagonal block p (every CTA that needs D_p, and CTA 0, which
// writes D_p into the diagonal block of Linv); D_p goes to the shared tile
// sd as sd[i][k] = D_p[i][k].  L_pp itself is not stored: later phases read
// only the off-diagonal blocks of L, and other CTAs may still be reading
// S_pp.  Returns false on a bad pivot.
__device__ bool factor_diag(const CholBArgs& a, int p, float (*sd)[kNb + 1]) {
  __shared__ int s_ok;
  if (threadIdx.x < 32) {
    float l[kNb], x[kNb];
    const bool ok = warp_chol32(blk(a.S, a.R, p, p), a.R, l, x);
    const int lane = threadIdx.x;
    if (lane == 0) s_ok = ok ? 1 : 0;
    if (ok) {
#pragma unroll
      for (int i = 0; i < kNb; ++i) sd[i][lane] = x[i];
      if (blockIdx.x == 0) {
        float* d = blk(a.Linv, a.R, p, p);
#pragma unroll
        for (int i = 0; i < kNb; ++i) d[(size_t)i * a.R + lane] = x[i];
      }
    } else if (blockIdx.x == 0 && lane == 0) {
      atomicExch(&a.flags[0], 1);
    }
  }
  __syncthreads();
  return s_ok != 0;
}

// out(32 x 32) (+)= A(32 x 32) * B^T(32 x 32), thread owns 4 entries of a row.
__device__ __forceinline__ void mma_bt(float (*A)[kNb + 1], float (*B)[kNb + 1],
                                       float acc[4]) {
  const int i = threadIdx.x >> 3, j0 = (threadIdx.x & 7) * 4;
#pragma unroll 8
  for (int k = 0; k < kNb; ++k) {
    const float av = A[i][k];
#pragma unroll
    for (int u = 0; u < 4; ++u) acc[u] = fmaf(av, B[j0 + u][k], acc[u]);
  }
}

// L_ip = S_ip D_p^T for the blocks below diagonal block p (D_p in sd).
__device__ void panel(const CholBArgs& a, int p, float (*sd)[kNb + 1]) {
  __shared__ float sa[kNb][kNb + 1];
  const int i = threadIdx.x >> 3, j0 = (threadIdx.x & 7) * 4;
  for (int bi = p + 1 + blockIdx.x; bi < a.nblk; bi += gridDim.x) {
    float* g = blk(a.S, a.R, bi, p);
    load_blk(sa, g, a.R);
    __syncthreads();
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    mma_bt(sa, sd, acc);
    __syncthreads();
#pragma unroll
    for (int u = 0; u < 4; ++u) g[(size_t)i * a.R + j0 + u] = acc[u];
  }
}

// S_ij -= L_ip L_jp^T for p < j <= i.
__device__ void trailing(const CholBArgs& a, int p) {
  __shared__ float li[kNb][kNb + 1];
  __shared__ float lj[kNb][kNb + 1];
  const int m = a.nblk - p - 1;
  const int tasks = m * (m + 1) / 2;
  const int i = threadIdx.x >> 3, j0 = (threadIdx.x & 7) * 4;
  for (int t = blockIdx.x; t < tasks; t += gridDim.x) {
    // t -> (bi, bj), bj <= bi, row-major over the lower triangle
    int bi = (int)((sqrtf(8.f * (float)t + 1.f) - 1.f) * 0.5f);
    while ((bi + 1) * (bi + 2) / 2 <= t) ++bi;
    while (bi * (bi + 1) / 2 > t) --bi;
    const int bj = t - bi * (bi + 1) / 2;
    const int gi = p + 1 + bi, gj = p + 1 + bj;
    load_blk(li, blk(a.S, a.R, gi, p), a.R);
    load_blk(lj, blk(a.S, a.R, gj, p), a.R);
    __syncthreads();
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    mma_bt(li, lj, acc);
    __syncthreads();
    float* g = blk(a.S, a.R, gi, gj);
#pragma unroll
    for (int u = 0; u < 4; ++u) g[(size_t)i * a.R + j0 + u] -= acc[u];
  }
}

// Transposed 32 x 32 block into shared memory: t[c][r] = g[r][c].

// tr(S) from the diagonal kept by assemble(); every CTA forms the same sum
// in the same (fixed) order.
__device__ double trace_of_s(const CholBArgs& a) {
  __shared__ double part[kCholThreads];
  double t = 0.0;
  for (int i = threadIdx.x; i < a.r; i += blockDim.x)
    t += *reinterpret_cast<volatile double*>(&a.diag[i]);
  part[threadIdx.x] = t;
  __syncthreads();
  for (int w = kCholThreads / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) part[threadIdx.x] += part[threadIdx.x + w];
    __syncthreads();
  }
  const double tr = part[0];
  __syncthreads();
  return tr;
}

__global__ void __launch_bounds__(kCholThreads) chol_blocked_kernel(const CholBArgs a) {
  __shared__ float sd[kNb][kNb + 1];
  bool ok = false;
  for (int attempt = 0; attempt < 2 && !ok; ++attempt) {
    float shift = 0.f;
    if (attempt == 1) {
      const double u = 5.9604644775390625e-8;  // 2^-24
      const double tr = trace_of_s(a);
      shift = (float)(11.0 * ((double)a.L * a.r + (double)a.r * (a.r + 1)) * u * tr);
      if (!(shift > 0.f)) shift = 1e-30f;
    }
    assemble(a, shift);
    grid_barrier(a);
    bool failed = false;
    for (int p = 0; p < a.nblk; ++p) {
      // CTAs with panel work factor the diagonal block themselves (same
      // bits everywhere); CTA 0 always does and publishes it
      const bool busy = blockIdx.x == 0 || p + 1 + (int)blockIdx.x < a.nblk;
      if (busy && factor_diag(a, p, sd)) panel(a, p, sd);
      grid_barrier(a);
      if (*reinterpret_cast<volatile int*>(&a.flags[0])) {
        failed = true;
        break;
      }
      if (p + 1 < a.nblk) {
        trailing(a, p);
        grid_barrier(a);
      }
    }
    if (failed && attempt == 0) {
      // every CTA has read the failure flag before CTA 0 clears it
      grid_barrier(a);
      if (blockIdx.x == 0 && threadIdx.x == 0) atomicExch(&a.flags[0], 0);
    }
    ok = !failed;
  }
  if (!ok) {
    if (blockIdx.x == 0 && threadIdx.x == 0) report_status(a.status, OUO_STATUS_BREAKDOWN);
    const size_t total = (size_t)a.R * a.R;
    for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
         e += (size_t)gridDim.x * blockDim.x) {
      const int i = (int)(e / a.R), j = (int)(e - (e / a.R) * a.R);
      a.Linv[e] = i == j ? 1.f : 0.f;
      if (j / kNb < i / kNb) a.S[e] = 0.f;  // L = I
    }
  }
  if (blockIdx.x == 0 && threadIdx.x == 0 &&
      *reinterpret_cast<volatile int*>(&a.flags[1]))
    report_status(a.status, OUO_STATUS_TIMEOUT);
}

}  // namespace

size_t chol_blocked_ctl_bytes(int r) { return 64 + (size_t)r * sizeof(double); }

int chol_blocked(const float* part, int splits, int r, int64_t L, float* S,
                 float* Linv, void* ctl, int* status, cudaStream_t stream) {
  CholBArgs a;
  a.part = part;
  a.splits = splits;
  a.r = r;
  a.nblk = (int)ceil_div(r, kNb);
  a.R = a.nblk * kNb;
  a.L = L;
  a.S = S;
  a.Linv = Linv;
  a.bar = reinterpret_cast<unsigned*>(ctl);
  a.flags = reinterpret_cast<int*>(reinterpret_cast<char*>(ctl) + 16);
  a.diag = reinterpret_cast<double*>(reinterpret_cast<char*>(ctl) + 64);
  a.status = status;
  OUO_CHECK_CUDA(cudaMemsetAsync(ctl, 0, 64, stream));
  // every CTA must be resident at once: at most one per SM times the
  // occupancy, and no more than the widest phase needs
  static std::atomic<int> per_sm[64];  // zero-initialized (static storage)
  int dev = 0;
  OUO_CHECK_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64)
    return set_error(OUO_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  int resident = per_sm[dev].load(std::memory_order_relaxed);
  if (!resident) {
    OUO_CHECK_CUDA(cudaOccupancyMaxActiveBlocksPerMultiprocessor(
        &resident, chol_blocked_kernel, kCholThreads, 0));
    if (resident < 1)
      return set_error(OUO_ERR_UNSUPPORTED, "blocked Cholesky kernel does not fit");
    per_sm[dev].store(resident, std::memory_order_relaxed);
  }
  const int m = a.nblk - 1;
  int want = m * (m + 1) / 2;
  if (want < 1) want = 1;
  int grid = num_sms() * (resident < 2 ? resident : 2);
  if (grid > want) grid = want;
  void* args[] = {&a};
  OUO_CHECK_CUDA(cudaLaunchCooperativeKernel((const void*)chol_blocked_kernel,
                                             dim3((unsigned)grid), dim3(kCholThreads),
                                             args, 0, stream));
  OUO_CHECK_LAUNCH();
  return OUO_OK;
}

}  // namespace ouo
