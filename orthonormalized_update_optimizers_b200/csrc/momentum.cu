// Momentum update (HBM-bound): M <- mu M + G  or  M <- M + G, with the
// float64 sum of squares of every updated row fused in.
//
// Source: "Dion3：全栈正交更新", 输入输出流程 (a step starts by updating the
// momentum); "Orth-Dion: ...", Orth-Dion (Dion's residual buffer receives the
// gradient).  The row sums feed the Dion3 row-selection rule.
//
// Layout: one warp per matrix row, 16-byte vector loads and stores, a
// persistent grid (a multiple of the SM count) striding over all rows of all
// matrices of the batch.  Each lane accumulates its squares in float64 in a
// fixed order and the warp reduces them with a fixed butterfly, so the row
// sums are deterministic.
#include "internal.h"

namespace ouo {
namespace {

struct MomentumArgs {
  int nmat;
  int g_bf16;
  int mode;
  float mu;
  double* row_sqnorm;  // already offset to this launch's first row
  int64_t row_start[kChunk + 1];
  int64_t cols[kChunk];
  float* M[kChunk];
  int64_t ldm[kChunk];
  const void* G[kChunk];
  int64_t ldg[kChunk];
  uint8_t vec[kChunk];  // rows of M and G start on 16-byte boundaries
};

__device__ __forceinline__ float4 load_g4(const void* g, int64_t j, int bf16) {
  if (bf16) {
    uint2 v = *reinterpret_cast<const uint2*>(
        reinterpret_cast<const uint16_t*>(g) + j);
    return make_float4(__uint_as_float(v.x << 16),
                       __uint_as_float(v.x & 0xffff0000u),
                       __uint_as_float(v.y << 16),
                       __uint_as_float(v.y & 0xffff0000u));
  }
  return *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(g) + j);
}

__device__ __forceinline__ float load_g1(const void* g, int64_t j, int bf16) {
  if (bf16) return bf16_to_f32(reinterpret_cast<const uint16_t*>(g)[j]);
  return reinterpret_cast<const float*>(g)[j];
}

__device__ __forceinline__ float mom(float m, float g, float mu, int mode) {
  return mode == OUO_MOMENTUM_EMA ? __fmaf_rn(mu, m, g) : __fadd_rn(m, g);
}

__global__ void __launch_bounds__(256)
momentum_kernel(const __grid_constant__ MomentumArgs a) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  const int64_t total = a.row_start[a.nmat];
  for (int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
       row < total; row += warps) {
    int lo = 0, hi = a.nmat - 1;
    while (lo < hi) {
      int mid = (lo + hi + 1) >> 1;
      if (a.row_start[mid] <= row) lo = mid; else hi = mid - 1;
    }
    const int64_t r = row - a.row_start[lo];
    const int64_t n = a.cols[lo];
    float* m = a.M[lo] + r * a.ldm[lo];
    const void* g = a.g_bf16
        ? (const void*)(reinterpret_cast<const uint16_t*>(a.G[lo]) + r * a.ldg[lo])
        : (const void*)(reinterpret_cast<const float*>(a.G[lo]) + r * a.ldg[lo]);
    double acc = 0.0;
    const int64_t n4 = a.vec[lo] ? (n >> 2) : 0;
    int64_t q = lane;
    // four 16-byte vectors in flight per lane
    for (; q + 96 < n4; q += 128) {
      float4 mv[4], gv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        mv[u] = *reinterpret_cast<const float4*>(m + 4 * (q + 32 * u));
        gv[u] = load_g4(g, 4 * (q + 32 * u), a.g_bf16);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        float4 o;
        o.x = mom(mv[u].x, gv[u].x, a.mu, a.mode);
        o.y = mom(mv[u].y, gv[u].y, a.mu, a.mode);
        o.z = mom(mv[u].z, gv[u].z, a.mu, a.mode);
        o.w = mom(mv[u].w, gv[u].w, a.mu, a.mode);
        *reinterpret_cast<float4*>(m + 4 * (q + 32 * u)) = o;
        acc += (double)o.x * (double)o.x;
        acc += (double)o.y * (double)o.y;
        acc += (double)o.z * (double)o.z;
        acc += (double)o.w * (double)o.w;
      }
    }
    for (; q < n4; q += 32) {
      float4 mv = *reinterpret_cast<const float4*>(m + 4 * q);
      float4 gv = load_g4(g, 4 * q, a.g_bf16);
      float4 o;
      o.x = mom(mv.x, gv.x, a.mu, a.mode);
      o.y = mom(mv.y, gv.y, a.mu, a.mode);
      o.z = mom(mv.z, gv.z, a.mu, a.mode);
      o.w = mom(mv.w, gv.w, a.mu, a.mode);
      *reinterpret_cast<float4*>(m + 4 * q) = o;
      acc += (double)o.x * (double)o.x;
      acc += (double)o.y * (double)o.y;
      acc += (double)o.z * (double)o.z;
      acc += (double)o.w * (double)o.w;
    }
    for (int64_t j = 4 * n4 + lane; j < n; j += 32) {
      float o = mom(m[j], load_g1(g, j, a.g_bf16), a.mu, a.mode);
      m[j] = o;
      acc += (double)o * (double)o;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
      acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0 && a.row_sqnorm) a.row_sqnorm[row] = acc;
  }
}

}  // namespace
}  // namespace ouo

extern "C" int dion_momentum_update(const ouo_mat* M, const ouo_mat* G,
                                    int nmat, int g_dtype, float mu, int mode,
                                    double* row_sqnorm, void* stream) {
  using namespace ouo;
  clear_error();
  if (nmat < 0 || nmat > OUO_MAX_BATCH)
    return set_error(OUO_ERR_INVALID_ARG, "nmat %d out of range", nmat);
  if (nmat == 0) return OUO_OK;
  if (mode != OUO_MOMENTUM_EMA && mode != OUO_MOMENTUM_ACCUM)
    return set_error(OUO_ERR_INVALID_ARG, "unknown momentum mode %d", mode);
  OUO_TRY(validate_mats(M, nmat, OUO_F32, "M"));
  OUO_TRY(validate_mats(G, nmat, g_dtype, "G"));
  OUO_TRY(validate_same_shapes(M, G, nmat, "M", "G"));
  if (row_sqnorm && ((uintptr_t)row_sqnorm % 8))
    return set_error(OUO_ERR_INVALID_ARG, "row_sqnorm not 8-byte aligned");
  OUO_TRY(require_sm100());
  cudaStream_t s = (cudaStream_t)stream;
  int64_t row_base = 0;
  for (int c0 = 0; c0 < nmat; c0 += kChunk) {
    int cn = nmat - c0 < kChunk ? nmat - c0 : kChunk;
    MomentumArgs a;
    a.nmat = cn;
    a.g_bf16 = g_dtype == OUO_BF16;
    a.mode = mode;
    a.mu = mu;
    a.row_sqnorm = row_sqnorm ? row_sqnorm + row_base : nullptr;
    int64_t acc = 0;
    for (int i = 0; i < cn; ++i) {
      const ouo_mat& mm = M[c0 + i];
      a.row_start[i] = acc;
      a.cols[i] = mm.cols;
      a.M[i] = reinterpret_cast<float*>(mm.ptr);
      a.ldm[i] = mm.ld;
      a.G[i] = G[c0 + i].ptr;
      a.ldg[i] = G[c0 + i].ld;
      a.vec[i] = vec16(mm, OUO_F32) && vec16(G[c0 + i], g_dtype);
      acc += mm.rows;
    }
    a.row_start[cn] = acc;
    int64_t warps_needed = acc;
    int64_t blocks = ceil_div(warps_needed, 8);
    int64_t cap = (int64_t)num_sms() * 8;  // 8 blocks x 8 warps per SM
    if (blocks > cap) blocks = cap;
    momentum_kernel<<<(unsigned)blocks, 256, 0, s>>>(a);
    OUO_CHECK_LAUNCH();
    row_base += acc;
  }
  return OUO_OK;
}
