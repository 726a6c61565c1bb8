// Dion3 row selection (exact, deterministic top-k), the gather of the kept
// rows with Frobenius scaling and error feedback, and the weight update.
//
// Sources: "Dion3: Full-Stack Orthogonal Updates", Abstract (orthogonalize
// only a fraction of the momentum matrix's rows); "Dion3：全栈正交更新",
// 核心模块 (e.g. 1/8 of the rows; the others keep the plain momentum; error
// feedback) and 输入输出流程 (select rows -> Gram NS -> update weights).
//
// Selection: one CTA per matrix.  Keys are non-negative float64 sums of
// squares, so their bit patterns order like the values; an 8-pass radix
// select over 8-bit digits finds the k-th largest key T exactly, then two
// ordered block scans keep every key > T and the lowest-indexed keys == T,
// emitting indices in ascending order.  No floating-point atomics, so the
// result does not depend on scheduling.
#include "internal.h"

namespace ouo {
namespace {

constexpr int kSelThreads = 1024;

struct SelectArgs {
  int nmat;
  const double* keys;          // row_sqnorm, at this launch's first row
  int32_t* idx;                // at this launch's first kept row
  float* x0_scale;             // at this launch's first matrix
  float eps;
  int64_t key_start[kChunk];   // first key of matrix i (relative)
  int64_t rows[kChunk];
  int64_t k[kChunk];
  int64_t sel_start[kChunk];   // first kept row of matrix i (relative)
};

// Exclusive block-wide prefix sum of `v` over kSelThreads threads; returns the
// prefix and writes the block total to *total.  Fixed order.
__device__ int block_exclusive_scan(int v, int* total, int* sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += y;
  }
  if (lane == 31) sh[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = sh[lane];
    int ws = w;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, ws, off);
      if (lane >= off) ws += y;
    }
    sh[32 + lane] = ws - w;  // exclusive warp offsets
    if (lane == 31) sh[64] = ws;
  }
  __syncthreads();
  int res = sh[32 + warp] + x - v;
  *total = sh[64];
  __syncthreads();
  return res;
}

__global__ void __launch_bounds__(kSelThreads)
select_kernel(const __grid_constant__ SelectArgs a) {
  __shared__ int hist[256];
  __shared__ int sh[80];
  __shared__ unsigned long long s_prefix;
  __shared__ long long s_krem;
  __shared__ double s_part[32];
  const int mat = blockIdx.x;
  const int tid = threadIdx.x;
  const int64_t m = a.rows[mat];
  const int64_t k = a.k[mat];
  const unsigned long long* keys =
      reinterpret_cast<const unsigned long long*>(a.keys + a.key_start[mat]);

  unsigned long long prefix = 0, mask = 0;
  long long krem = k;
  for (int pass = 0; pass < 8; ++pass) {
    const int shift = 56 - 8 * pass;
    for (int d = tid; d < 256; d += kSelThreads) hist[d] = 0;
    __syncthreads();
    for (int64_t i = tid; i < m; i += kSelThreads) {
      unsigned long long key = keys[i];
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255ull], 1);
    }
    __syncthreads();
    if (tid == 0) {
      long long cum = 0;
      int sel = 0;
      for (int d = 255; d >= 0; --d) {
        if (cum + hist[d] >= krem) { sel = d; break; }
        cum += hist[d];
      }
      s_krem = krem - cum;
      s_prefix = prefix | ((unsigned long long)sel << shift);
    }
    __syncthreads();
    prefix = s_prefix;
    krem = s_krem;
    mask |= 255ull << shift;
    __syncthreads();
  }
  const unsigned long long T = prefix;  // the k-th largest key, exactly
  int eq_base = 0, out_base = 0;
  double sum = 0.0;
  int32_t* out = a.idx + a.sel_start[mat];
  for (int64_t c = 0; c < m; c += kSelThreads) {
    const int64_t i = c + tid;
    unsigned long long key = i < m ? keys[i] : 0ull;
    int is_eq = (i < m && key == T) ? 1 : 0;
    int is_gt = (i < m && key > T) ? 1 : 0;
    int eq_tot;
    int eq_rank = eq_base + block_exclusive_scan(is_eq, &eq_tot, sh);
    int sel = is_gt | (is_eq & (eq_rank < krem ? 1 : 0));
    int sel_tot;
    int pos = out_base + block_exclusive_scan(sel, &sel_tot, sh);
    if (sel) {
      out[pos] = (int32_t)i;
      sum += __longlong_as_double((long long)key);
    }
    eq_base += eq_tot;
    out_base += sel_tot;
  }
  // deterministic block reduction of the kept keys
#pragma unroll
  for (int off = 16; off > 0; off >>= 1)
    sum += __shfl_xor_sync(0xffffffffu, sum, off);
  if ((tid & 31) == 0) s_part[tid >> 5] = sum;
  __syncthreads();
  if (tid < 32) {
    double v = s_part[tid];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
      v += __shfl_xor_sync(0xffffffffu, v, off);
    if (tid == 0) a.x0_scale[mat] = (float)(1.0 / (sqrt(v) + (double)a.eps));
  }
}

struct GatherArgs {
  int nmat;
  int x0_bf16;
  int ef;
  float mu;
  const int32_t* idx;        // at this launch's first kept row
  const float* x0_scale;     // at this launch's first matrix
  int64_t sel_start[kChunk + 1];
  int64_t cols[kChunk];
  float* B[kChunk];
  int64_t ldb[kChunk];
  void* X0[kChunk];
  int64_t ldx[kChunk];
  uint8_t vec[kChunk];
};

// One warp per kept row: X0[j] = B[idx[j]] * scale (bf16 or fp32) and, under
// error feedback, B[idx[j]] <- mu * B[idx[j]].
__global__ void __launch_bounds__(256)
gather_kernel(const __grid_constant__ GatherArgs a) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  const int64_t total = a.sel_start[a.nmat];
  for (int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
       row < total; row += warps) {
    int lo = 0, hi = a.nmat - 1;
    while (lo < hi) {
      int mid = (lo + hi + 1) >> 1;
      if (a.sel_start[mid] <= row) lo = mid; else hi = mid - 1;
    }
    const int64_t j = row - a.sel_start[lo];
    const int64_t r = a.idx[row];
    const int64_t n = a.cols[lo];
    const float s = a.x0_scale[lo];
    float* b = a.B[lo] + r * a.ldb[lo];
    const int64_t n4 = a.vec[lo] ? (n >> 2) : 0;
    if (a.x0_bf16) {
      uint16_t* x = reinterpret_cast<uint16_t*>(a.X0[lo]) + j * a.ldx[lo];
      int64_t q = lane;
      // four 16-byte vectors in flight per lane
      for (; q + 96 < n4; q += 128) {
        float4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) v[u] = *reinterpret_cast<const float4*>(b + 4 * (q + 32 * u));
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          uint2 o;
          o.x = pack_bf16x2(v[u].x * s, v[u].y * s);
          o.y = pack_bf16x2(v[u].z * s, v[u].w * s);
          *reinterpret_cast<uint2*>(x + 4 * (q + 32 * u)) = o;
          if (a.ef)
            *reinterpret_cast<float4*>(b + 4 * (q + 32 * u)) =
                make_float4(a.mu * v[u].x, a.mu * v[u].y, a.mu * v[u].z, a.mu * v[u].w);
        }
      }
      for (; q < n4; q += 32) {
        float4 v = *reinterpret_cast<const float4*>(b + 4 * q);
        uint2 o;
        o.x = pack_bf16x2(v.x * s, v.y * s);
        o.y = pack_bf16x2(v.z * s, v.w * s);
        *reinterpret_cast<uint2*>(x + 4 * q) = o;
        if (a.ef) {
          float4 e = make_float4(a.mu * v.x, a.mu * v.y, a.mu * v.z, a.mu * v.w);
          *reinterpret_cast<float4*>(b + 4 * q) = e;
        }
      }
      for (int64_t c = 4 * n4 + lane; c < n; c += 32) {
        float v = b[c];
        x[c] = f32_to_bf16(v * s);
        if (a.ef) b[c] = a.mu * v;
      }
    } else {
      float* x = reinterpret_cast<float*>(a.X0[lo]) + j * a.ldx[lo];
      int64_t q = lane;
      for (; q + 96 < n4; q += 128) {
        float4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) v[u] = *reinterpret_cast<const float4*>(b + 4 * (q + 32 * u));
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          *reinterpret_cast<float4*>(x + 4 * (q + 32 * u)) =
              make_float4(v[u].x * s, v[u].y * s, v[u].z * s, v[u].w * s);
          if (a.ef)
            *reinterpret_cast<float4*>(b + 4 * (q + 32 * u)) =
                make_float4(a.mu * v[u].x, a.mu * v[u].y, a.mu * v[u].z, a.mu * v[u].w);
        }
      }
      for (; q < n4; q += 32) {
        float4 v = *reinterpret_cast<const float4*>(b + 4 * q);
        *reinterpret_cast<float4*>(x + 4 * q) =
            make_float4(v.x * s, v.y * s, v.z * s, v.w * s);
        if (a.ef) {
          float4 e = make_float4(a.mu * v.x, a.mu * v.y, a.mu * v.z, a.mu * v.w);
          *reinterpret_cast<float4*>(b + 4 * q) = e;
        }
      }
      for (int64_t c = 4 * n4 + lane; c < n; c += 32) {
        float v = b[c];
        x[c] = v * s;
        if (a.ef) b[c] = a.mu * v;
      }
    }
  }
}

struct ApplyArgs {
  int nmat;
  int w_bf16, o_bf16;
  float decay;                 // 1 - lr * wd
  const int32_t* idx;          // NULL: all rows; else at launch's first row
  int64_t row_start[kChunk + 1];
  int64_t cols[kChunk];
  float lrs[kChunk];           // lr * scale[i]
  void* W[kChunk];
  int64_t ldw[kChunk];
  const void* O[kChunk];
  int64_t ldo[kChunk];
  uint8_t vec[kChunk];
};

__device__ __forceinline__ void load4(const void* p, int64_t j, int bf16,
                                      float v[4]) {
  if (bf16) {
    uint2 u = *reinterpret_cast<const uint2*>(
        reinterpret_cast<const uint16_t*>(p) + j);
    v[0] = __uint_as_float(u.x << 16);
    v[1] = __uint_as_float(u.x & 0xffff0000u);
    v[2] = __uint_as_float(u.y << 16);
    v[3] = __uint_as_float(u.y & 0xffff0000u);
  } else {
    float4 u = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(p) + j);
    v[0] = u.x; v[1] = u.y; v[2] = u.z; v[3] = u.w;
  }
}

__device__ __forceinline__ void store4(void* p, int64_t j, int bf16,
                                       const float v[4]) {
  if (bf16) {
    uint2 u;
    u.x = pack_bf16x2(v[0], v[1]);
    u.y = pack_bf16x2(v[2], v[3]);
    *reinterpret_cast<uint2*>(reinterpret_cast<uint16_t*>(p) + j) = u;
  } else {
    *reinterpret_cast<float4*>(reinterpret_cast<float*>(p) + j) =
        make_float4(v[0], v[1], v[2], v[3]);
  }
}

__device__ __forceinline__ float load1(const void* p, int64_t j, int bf16) {
  return bf16 ? bf16_to_f32(reinterpret_cast<const uint16_t*>(p)[j])
              : reinterpret_cast<const float*>(p)[j];
}

__device__ __forceinline__ void store1(void* p, int64_t j, int bf16, float v) {
  if (bf16) reinterpret_cast<uint16_t*>(p)[j] = f32_to_bf16(v);
  else reinterpret_cast<float*>(p)[j] = v;
}

// One warp per row of O: W[r] = decay * W[r] - lr * scale * O[j].
__global__ void __launch_bounds__(256)
apply_kernel(const __grid_constant__ ApplyArgs a) {
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
    const int64_t j = row - a.row_start[lo];
    const int64_t r = a.idx ? (int64_t)a.idx[row] : j;
    const int64_t n = a.cols[lo];
    const float lrs = a.lrs[lo];
    char* w = reinterpret_cast<char*>(a.W[lo]) + r * a.ldw[lo] * (a.w_bf16 ? 2 : 4);
    const char* o = reinterpret_cast<const char*>(a.O[lo]) + j * a.ldo[lo] * (a.o_bf16 ? 2 : 4);
    const int64_t n4 = a.vec[lo] ? (n >> 2) : 0;
    int64_t q = lane;
    // four vectors of W and of O in flight per lane
    for (; q + 96 < n4; q += 128) {
      float wv[4][4], ov[4][4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        load4(w, 4 * (q + 32 * u), a.w_bf16, wv[u]);
        load4(o, 4 * (q + 32 * u), a.o_bf16, ov[u]);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
#pragma unroll
        for (int t = 0; t < 4; ++t) wv[u][t] = __fmaf_rn(-lrs, ov[u][t], a.decay * wv[u][t]);
        store4(w, 4 * (q + 32 * u), a.w_bf16, wv[u]);
      }
    }
    for (; q < n4; q += 32) {
      float wv[4], ov[4];
      load4(w, 4 * q, a.w_bf16, wv);
      load4(o, 4 * q, a.o_bf16, ov);
#pragma unroll
      for (int u = 0; u < 4; ++u) wv[u] = __fmaf_rn(-lrs, ov[u], a.decay * wv[u]);
      store4(w, 4 * q, a.w_bf16, wv);
    }
    for (int64_t c = 4 * n4 + lane; c < n; c += 32) {
      float wv = load1(w, c, a.w_bf16);
      store1(w, c, a.w_bf16, __fmaf_rn(-lrs, load1(o, c, a.o_bf16), a.decay * wv));
    }
  }
}

unsigned grid_for_rows(int64_t rows) {
  int64_t blocks = ceil_div(rows, 8);
  int64_t cap = (int64_t)num_sms() * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  return (unsigned)blocks;
}

}  // namespace
}  // namespace ouo

extern "C" int dion3_select_rows(const ouo_mat* B, const double* row_sqnorm,
                                 int nmat, double rho, int ef_mode, float mu,
                                 float eps, int32_t* idx, const ouo_mat* X0,
                                 int x0_dtype, float* x0_scale, void* stream) {
  using namespace ouo;
  clear_error();
  if (nmat < 0 || nmat > OUO_MAX_BATCH)
    return set_error(OUO_ERR_INVALID_ARG, "nmat %d out of range", nmat);
  if (nmat == 0) return OUO_OK;
  if (!(rho > 0.0) || rho > 1.0)
    return set_error(OUO_ERR_INVALID_ARG, "rho %g outside (0, 1]", rho);
  if (ef_mode != OUO_EF_NONE && ef_mode != OUO_EF_ROWS)
    return set_error(OUO_ERR_INVALID_ARG, "unknown ef_mode %d", ef_mode);
  if (!row_sqnorm || !idx || !x0_scale)
    return set_error(OUO_ERR_INVALID_ARG,
                     "row_sqnorm, idx and x0_scale are required");
  if (((uintptr_t)row_sqnorm) % 8 || ((uintptr_t)idx) % 4 ||
      ((uintptr_t)x0_scale) % 4)
    return set_error(OUO_ERR_INVALID_ARG, "misaligned key / index / scale array");
  OUO_TRY(validate_mats(B, nmat, OUO_F32, "B"));
  OUO_TRY(validate_mats(X0, nmat, x0_dtype, "X0"));
  for (int i = 0; i < nmat; ++i) {
    int64_t k = dion3_num_selected(B[i].rows, rho);
    if (X0[i].rows != k || X0[i].cols != B[i].cols)
      return set_error(OUO_ERR_INVALID_ARG,
                       "X0[%d] must be %lld x %lld (k = ceil(rho * rows))", i,
                       (long long)k, (long long)B[i].cols);
  }
  OUO_TRY(require_sm100());
  cudaStream_t s = (cudaStream_t)stream;
  int64_t key_base = 0, sel_base = 0;
  for (int c0 = 0; c0 < nmat; c0 += kChunk) {
    int cn = nmat - c0 < kChunk ? nmat - c0 : kChunk;
    SelectArgs sa;
    GatherArgs ga;
    sa.nmat = cn;
    sa.keys = row_sqnorm + key_base;
    sa.idx = idx + sel_base;
    sa.x0_scale = x0_scale + c0;
    sa.eps = eps;
    ga.nmat = cn;
    ga.x0_bf16 = x0_dtype == OUO_BF16;
    ga.ef = ef_mode == OUO_EF_ROWS;
    ga.mu = mu;
    ga.idx = idx + sel_base;
    ga.x0_scale = x0_scale + c0;
    int64_t kacc = 0, racc = 0;
    for (int i = 0; i < cn; ++i) {
      const ouo_mat& b = B[c0 + i];
      int64_t k = dion3_num_selected(b.rows, rho);
      sa.key_start[i] = racc;
      sa.rows[i] = b.rows;
      sa.k[i] = k;
      sa.sel_start[i] = kacc;
      ga.sel_start[i] = kacc;
      ga.cols[i] = b.cols;
      ga.B[i] = reinterpret_cast<float*>(b.ptr);
      ga.ldb[i] = b.ld;
      ga.X0[i] = X0[c0 + i].ptr;
      ga.ldx[i] = X0[c0 + i].ld;
      ga.vec[i] = vec16(b, OUO_F32) && vec16(X0[c0 + i], x0_dtype);
      kacc += k;
      racc += b.rows;
    }
    ga.sel_start[cn] = kacc;
    select_kernel<<<cn, kSelThreads, 0, s>>>(sa);
    OUO_CHECK_LAUNCH();
    gather_kernel<<<grid_for_rows(kacc), 256, 0, s>>>(ga);
    OUO_CHECK_LAUNCH();
    key_base += racc;
    sel_base += kacc;
  }
  return OUO_OK;
}

extern "C" int apply_update(const ouo_mat* W, int w_dtype, const ouo_mat* O,
                            int o_dtype, const int32_t* idx, int nmat,
                            float lr, const float* scale, float wd,
                            void* stream) {
  using namespace ouo;
  clear_error();
  if (nmat < 0 || nmat > OUO_MAX_BATCH)
    return set_error(OUO_ERR_INVALID_ARG, "nmat %d out of range", nmat);
  if (nmat == 0) return OUO_OK;
  OUO_TRY(validate_mats(W, nmat, w_dtype, "W"));
  OUO_TRY(validate_mats(O, nmat, o_dtype, "O"));
  for (int i = 0; i < nmat; ++i) {
    if (O[i].cols != W[i].cols || (!idx && O[i].rows != W[i].rows) ||
        O[i].rows > W[i].rows)
      return set_error(OUO_ERR_INVALID_ARG, "O[%d] shape does not fit W[%d]",
                       i, i);
  }
  if (idx && ((uintptr_t)idx) % 4)
    return set_error(OUO_ERR_INVALID_ARG, "idx not 4-byte aligned");
  OUO_TRY(require_sm100());
  cudaStream_t s = (cudaStream_t)stream;
  int64_t base = 0;
  for (int c0 = 0; c0 < nmat; c0 += kChunk) {
    int cn = nmat - c0 < kChunk ? nmat - c0 : kChunk;
    ApplyArgs a;
    a.nmat = cn;
    a.w_bf16 = w_dtype == OUO_BF16;
    a.o_bf16 = o_dtype == OUO_BF16;
    a.decay = 1.0f - lr * wd;
    a.idx = idx ? idx + base : nullptr;
    int64_t acc = 0;
    for (int i = 0; i < cn; ++i) {
      a.row_start[i] = acc;
      a.cols[i] = W[c0 + i].cols;
      a.lrs[i] = lr * (scale ? scale[c0 + i] : 1.0f);
      a.W[i] = W[c0 + i].ptr;
      a.ldw[i] = W[c0 + i].ld;
      a.O[i] = O[c0 + i].ptr;
      a.ldo[i] = O[c0 + i].ld;
      a.vec[i] = vec16(W[c0 + i], w_dtype) && vec16(O[c0 + i], o_dtype);
      acc += O[c0 + i].rows;
    }
    a.row_start[cn] = acc;
    apply_kernel<<<grid_for_rows(acc), 256, 0, s>>>(a);
    OUO_CHECK_LAUNCH();
    base += acc;
  }
  return OUO_OK;
}
