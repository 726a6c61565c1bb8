// fp32 GEMM on CUDA cores for the fp32 precision path of Newton-Schulz
// (operands and accumulation in fp32; tensor-core tf32 would miss the 1e-4
// relative accuracy that path is held to).  64 x 64 output tiles, 16-deep
// k-slices staged in shared memory, 4 x 4 outputs per thread.  Symmetric
// outputs (tri) compute only tiles on or above the diagonal and mirror.
#include "internal.h"

namespace ouo {
namespace {

constexpr int TM = 64, TN = 64, TK = 16;

struct SimtArgs {
  int64_t M, N, K;
  int tri, b_mn, has_c0, has_f32, has_bf16, round_tf32;
  float alpha, beta, gamma;
  const float* A; int64_t lda, sa;
  const float* B; int64_t ldb, sb;
  const float* C0; int64_t ldc0, sc0;
  float* Of; int64_t ldof, sof;
  uint16_t* Ob; int64_t ldob, sob;
  int64_t tiles_m, tiles_n;
};

__device__ __forceinline__ void tri_tile(int64_t t, int64_t T, int64_t* ti,
                                         int64_t* tj) {
  int64_t i = 0, rem = t;
  while (rem >= T - i) { rem -= T - i; ++i; }
  *ti = i;
  *tj = i + rem;
}

__device__ __forceinline__ void put(const SimtArgs& a, int64_t b, int64_t i,
                                    int64_t j, float v) {
  if (a.has_f32) {
    float w = a.round_tf32 ? round_tf32(v) : v;
    a.Of[b * a.sof + i * a.ldof + j] = w;
  }
  if (a.has_bf16) a.Ob[b * a.sob + i * a.ldob + j] = f32_to_bf16(v);
}

__global__ void __launch_bounds__(256) simt_gemm_kernel(const SimtArgs a) {
  __shared__ float As[TK][TM + 4];
  __shared__ float Bs[TK][TN + 4];
  const int64_t b = blockIdx.z;
  int64_t ti, tj;
  if (a.tri) {
    tri_tile(blockIdx.x, a.tiles_m, &ti, &tj);
  } else {
    ti = blockIdx.x / a.tiles_n;
    tj = blockIdx.x % a.tiles_n;
  }
  const int64_t row0 = ti * TM, col0 = tj * TN;
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const float* A = a.A + b * a.sa;
  const float* B = a.B + b * a.sb;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  for (int64_t k0 = 0; k0 < a.K; k0 += TK) {
    for (int e = tid; e < TM * TK; e += 256) {
      int r = e / TK, kk = e % TK;
      int64_t gi = row0 + r, gk = k0 + kk;
      As[kk][r] = (gi < a.M && gk < a.K) ? A[gi * a.lda + gk] : 0.f;
    }
    if (!a.b_mn) {
      for (int e = tid; e < TN * TK; e += 256) {
        int c = e / TK, kk = e % TK;
        int64_t gj = col0 + c, gk = k0 + kk;
        Bs[kk][c] = (gj < a.N && gk < a.K) ? B[gj * a.ldb + gk] : 0.f;
      }
    } else {
      for (int e = tid; e < TN * TK; e += 256) {
        int kk = e / TN, c = e % TN;
        int64_t gj = col0 + c, gk = k0 + kk;
        Bs[kk][c] = (gj < a.N && gk < a.K) ? B[gk * a.ldb + gj] : 0.f;
      }
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < TK; ++kk) {
      float av[4], bv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) av[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) bv[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = __fmaf_rn(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t gi = row0 + ty * 4 + i, gj = col0 + tx * 4 + j;
      if (gi >= a.M || gj >= a.N) continue;
      if (a.tri && gj < gi) continue;
      float v = a.alpha * acc[i][j];
      if (a.has_c0) {
        const float* c0 = a.C0 + b * a.sc0;
        v += a.beta * (a.tri ? c0[gj * a.ldc0 + gi] : c0[gi * a.ldc0 + gj]);
      }
      if (gi == gj) v += a.gamma;
      put(a, b, gi, gj, v);
      if (a.tri && gi != gj) put(a, b, gj, gi, v);
    }
  }
}

}  // namespace

int gemm_simt(const GemmDesc& g, cudaStream_t stream) {
  if (g.A.dtype != OUO_F32 || g.B.dtype != OUO_F32 ||
      (g.has_c0 && g.C0.dtype != OUO_F32))
    return set_error(OUO_ERR_UNSUPPORTED, "fp32 GEMM needs fp32 operands");
  if (g.tri && g.M != g.N)
    return set_error(OUO_ERR_INVALID_ARG, "symmetric GEMM needs M == N");
  SimtArgs a;
  a.M = g.M; a.N = g.N; a.K = g.K;
  a.tri = g.tri; a.b_mn = g.b_mn; a.has_c0 = g.has_c0;
  a.has_f32 = g.has_f32; a.has_bf16 = g.has_bf16; a.round_tf32 = g.round_tf32;
  a.alpha = g.alpha; a.beta = g.beta; a.gamma = g.gamma;
  a.A = reinterpret_cast<const float*>(g.A.p); a.lda = g.A.ld; a.sa = g.A.stride;
  a.B = reinterpret_cast<const float*>(g.B.p); a.ldb = g.B.ld; a.sb = g.B.stride;
  a.C0 = g.has_c0 ? reinterpret_cast<const float*>(g.C0.p) : nullptr;
  a.ldc0 = g.C0.ld; a.sc0 = g.C0.stride;
  a.Of = g.has_f32 ? reinterpret_cast<float*>(g.out_f32.p) : nullptr;
  a.ldof = g.out_f32.ld; a.sof = g.out_f32.stride;
  a.Ob = g.has_bf16 ? reinterpret_cast<uint16_t*>(g.out_bf16.p) : nullptr;
  a.ldob = g.out_bf16.ld; a.sob = g.out_bf16.stride;
  a.tiles_m = ceil_div(g.M, TM);
  a.tiles_n = ceil_div(g.N, TN);
  int64_t tiles = g.tri ? a.tiles_m * (a.tiles_m + 1) / 2 : a.tiles_m * a.tiles_n;
  if (tiles > 0x7fffffff || g.nb > 65535)
    return set_error(OUO_ERR_UNSUPPORTED, "fp32 GEMM grid too large");
  dim3 grid((unsigned)tiles, 1, (unsigned)g.nb);
  simt_gemm_kernel<<<grid, 256, 0, stream>>>(a);
  OUO_CHECK_LAUNCH();
  return OUO_OK;
}

}  // namespace ouo
