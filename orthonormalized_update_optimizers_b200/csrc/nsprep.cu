// Newton-Schulz input preparation and output write-out (HBM-bound copies).
//
// ns_prep:     X0 = X / (||X||_F + eps) into library workspace (bf16 or
//              fp32), transposed when X has more rows than columns.  The
//              Frobenius norm is a float64 sum of squares, rows summed by one
//              warp each and rows combined per matrix in a fixed order.
// ns_writeout: the workspace result back to the caller's O (any dtype),
//              transposed back when needed.
// Also: identity fill and dtype conversion of workspace buffers.
#include "internal.h"

namespace ouo {
namespace {

struct RowSqArgs {
  int nmat;
  int x_bf16;
  double* out;                   // one float64 per row of the launch
  int64_t row_start[kChunk + 1];
  int64_t cols;
  const void* X[kChunk];
  int64_t ldx[kChunk];
};

__global__ void __launch_bounds__(256)
rowsq_kernel(const __grid_constant__ RowSqArgs a) {
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
    double acc = 0.0;
    if (a.x_bf16) {
      const uint16_t* x = reinterpret_cast<const uint16_t*>(a.X[lo]) + r * a.ldx[lo];
      for (int64_t c = lane; c < a.cols; c += 32) {
        double v = bf16_to_f32(x[c]);
        acc += v * v;
      }
    } else {
      const float* x = reinterpret_cast<const float*>(a.X[lo]) + r * a.ldx[lo];
      for (int64_t c = lane; c < a.cols; c += 32) {
        double v = x[c];
        acc += v * v;
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
      acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) a.out[row] = acc;
  }
}

// One block per matrix: scale[b] = 1 / (sqrt(sum of its rows) + eps).
__global__ void __launch_bounds__(256)
matscale_kernel(const double* rowsq, int64_t rows, float eps, float* scale) {
  __shared__ double part[8];
  const int b = blockIdx.x;
  double acc = 0.0;
  for (int64_t r = threadIdx.x; r < rows; r += blockDim.x) acc += rowsq[b * rows + r];
#pragma unroll
  for (int off = 16; off > 0; off >>= 1)
    acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double v = 0.0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) v += part[w];
    scale[b] = (float)(1.0 / (sqrt(v) + (double)eps));
  }
}

struct CopyArgs {
  int nmat;
  int src_bf16, dst_bf16;
  int transpose;       // dst[b][c][r] = src[r][c]
  int to_caller;       // 0: src caller -> dst workspace; 1: src workspace -> dst caller
  const float* scale;  // per matrix of the launch, or NULL
  int64_t rows, cols;  // of the caller-side matrix
  // caller side
  void* C[kChunk];
  int64_t ldc[kChunk];
  // workspace side
  char* wbase;
  int64_t wld, wstride;
};

__device__ __forceinline__ float ld_elem(const char* p, int64_t i, int bf16) {
  return bf16 ? bf16_to_f32(reinterpret_cast<const uint16_t*>(p)[i])
              : reinterpret_cast<const float*>(p)[i];
}
__device__ __forceinline__ void st_elem(char* p, int64_t i, int bf16, float v) {
  if (bf16) reinterpret_cast<uint16_t*>(p)[i] = f32_to_bf16(v);
  else reinterpret_cast<float*>(p)[i] = v;
}

// 32 x 32 tiles through shared memory; grid.z = matrix, grid.y / grid.x tile
// rows / tile cols of the caller-side matrix (grid-stride when large).
__global__ void __launch_bounds__(256)
copy_kernel(const __grid_constant__ CopyArgs a) {
  __shared__ float tile[32][33];
  const int b = blockIdx.z;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 32 x 8
  const float s = a.scale ? a.scale[b] : 1.0f;
  const int wes = a.to_caller ? (a.src_bf16 ? 2 : 4) : (a.dst_bf16 ? 2 : 4);
  char* w = a.wbase + (size_t)b * a.wstride * wes;
  char* c = reinterpret_cast<char*>(a.C[b]);
  const int64_t tiles_r = (a.rows + 31) / 32, tiles_c = (a.cols + 31) / 32;
  for (int64_t tr = blockIdx.y; tr < tiles_r; tr += gridDim.y) {
    for (int64_t tc = blockIdx.x; tc < tiles_c; tc += gridDim.x) {
      const int64_t r0 = tr * 32, c0 = tc * 32;
      if (!a.transpose) {
        for (int yy = ty; yy < 32; yy += 8) {
          int64_t r = r0 + yy, cc = c0 + tx;
          if (r < a.rows && cc < a.cols) {
            if (a.to_caller) {
              float v = ld_elem(w, r * a.wld + cc, a.src_bf16);
              st_elem(c, r * a.ldc[b] + cc, a.dst_bf16, v);
            } else {
              float v = ld_elem(c, r * a.ldc[b] + cc, a.src_bf16) * s;
              st_elem(w, r * a.wld + cc, a.dst_bf16, v);
            }
          }
        }
      } else if (!a.to_caller) {
        // caller X (rows x cols) -> workspace X0 (cols x rows)
        for (int yy = ty; yy < 32; yy += 8) {
          int64_t r = r0 + yy, cc = c0 + tx;
          tile[yy][tx] = (r < a.rows && cc < a.cols)
              ? ld_elem(c, r * a.ldc[b] + cc, a.src_bf16) * s : 0.f;
        }
        __syncthreads();
        for (int yy = ty; yy < 32; yy += 8) {
          int64_t wr = c0 + yy, wc = r0 + tx;  // workspace row = caller col
          if (wr < a.cols && wc < a.rows)
            st_elem(w, wr * a.wld + wc, a.dst_bf16, tile[tx][yy]);
        }
        __syncthreads();
      } else {
        // workspace Y (cols x rows) -> caller O (rows x cols)
        for (int yy = ty; yy < 32; yy += 8) {
          int64_t wr = c0 + yy, wc = r0 + tx;
          tile[yy][tx] = (wr < a.cols && wc < a.rows)
              ? ld_elem(w, wr * a.wld + wc, a.src_bf16) : 0.f;
        }
        __syncthreads();
        for (int yy = ty; yy < 32; yy += 8) {
          int64_t r = r0 + yy, cc = c0 + tx;
          if (r < a.rows && cc < a.cols)
            st_elem(c, r * a.ldc[b] + cc, a.dst_bf16, tile[tx][yy]);
        }
        __syncthreads();
      }
    }
  }
}

struct RowCopyArgs {
  int nmat;
  int src_bf16, dst_bf16;
  int to_caller;       // 0: caller -> workspace, 1: workspace -> caller
  const float* scale;  // per matrix of the launch, or NULL
  int64_t rows, cols;
  void* C[kChunk];
  int64_t ldc[kChunk];
  uint8_t vec[kChunk];  // caller rows start on 16-byte boundaries
  char* wbase;
  int64_t wld, wstride;
};

__device__ __forceinline__ void load4v(const char* p, int bf16, float v[4]) {
  if (bf16) {
    uint2 u = *reinterpret_cast<const uint2*>(p);
    v[0] = __uint_as_float(u.x << 16);
    v[1] = __uint_as_float(u.x & 0xffff0000u);
    v[2] = __uint_as_float(u.y << 16);
    v[3] = __uint_as_float(u.y & 0xffff0000u);
  } else {
    float4 f = *reinterpret_cast<const float4*>(p);
    v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
  }
}

__device__ __forceinline__ void store4v(char* p, int bf16, const float v[4]) {
  if (bf16) {
    uint2 u;
    u.x = pack_bf16x2(v[0], v[1]);
    u.y = pack_bf16x2(v[2], v[3]);
    *reinterpret_cast<uint2*>(p) = u;
  } else {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  }
}

// Row-to-row copy without transposition: one warp per row, 4 elements per
// lane per step with 8- or 16-byte accesses where the caller rows allow.
__global__ void __launch_bounds__(256)
rowcopy_kernel(const __grid_constant__ RowCopyArgs a) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  const int64_t total = a.rows * a.nmat;
  const int ses = a.src_bf16 ? 2 : 4, des = a.dst_bf16 ? 2 : 4;
  for (int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
       row < total; row += warps) {
    const int64_t b = row / a.rows, r = row - b * a.rows;
    const float s = a.scale ? a.scale[b] : 1.0f;
    const char* src;
    char* dst;
    if (a.to_caller) {
      src = a.wbase + ((size_t)b * a.wstride + (size_t)r * a.wld) * ses;
      dst = reinterpret_cast<char*>(a.C[b]) + (size_t)r * a.ldc[b] * des;
    } else {
      src = reinterpret_cast<const char*>(a.C[b]) + (size_t)r * a.ldc[b] * ses;
      dst = a.wbase + ((size_t)b * a.wstride + (size_t)r * a.wld) * des;
    }
    const int64_t n4 = a.vec[b] ? (a.cols >> 2) : 0;
    for (int64_t q = lane; q < n4; q += 32) {
      float v[4];
      load4v(src + 4 * q * ses, a.src_bf16, v);
      v[0] *= s; v[1] *= s; v[2] *= s; v[3] *= s;
      store4v(dst + 4 * q * des, a.dst_bf16, v);
    }
    for (int64_t c = 4 * n4 + lane; c < a.cols; c += 32)
      st_elem(dst, c, a.dst_bf16, ld_elem(src, c, a.src_bf16) * s);
  }
}

unsigned rows_grid(int64_t rows) {
  int64_t blocks = ceil_div(rows, 8);
  int64_t cap = (int64_t)num_sms() * 8;
  if (blocks > cap) blocks = cap;
  return (unsigned)(blocks < 1 ? 1 : blocks);
}

dim3 copy_grid(int64_t rows, int64_t cols, int nmat) {
  int64_t tr = ceil_div(rows, 32), tc = ceil_div(cols, 32);
  int64_t want = (int64_t)num_sms() * 8;
  int64_t per = want / (nmat > 0 ? nmat : 1);
  if (per < 1) per = 1;
  int64_t gx = tc < per ? tc : per;
  int64_t gy = ceil_div(per, gx);
  if (gy > tr) gy = tr;
  if (gy > 65535) gy = 65535;
  if (gx < 1) gx = 1;
  if (gy < 1) gy = 1;
  return dim3((unsigned)gx, (unsigned)gy, (unsigned)nmat);
}

__global__ void identity_kernel(char* p, int bf16, int64_t rows, int64_t cols,
                                int64_t ld, int64_t stride, int64_t nb) {
  const int64_t per = rows * cols;
  const int64_t total = per * nb;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    int64_t b = e / per, rem = e - b * per, r = rem / cols, c = rem - r * cols;
    st_elem(p, b * stride + r * ld + c, bf16, r == c ? 1.f : 0.f);
  }
}

__global__ void convert_kernel(const char* src, int sbf16, char* dst, int dbf16,
                               int64_t rows, int64_t cols, int64_t sld,
                               int64_t sstride, int64_t dld, int64_t dstride,
                               int64_t nb) {
  const int64_t per = rows * cols;
  const int64_t total = per * nb;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    int64_t b = e / per, rem = e - b * per, r = rem / cols, c = rem - r * cols;
    st_elem(dst, b * dstride + r * dld + c, dbf16,
            ld_elem(src, b * sstride + r * sld + c, sbf16));
  }
}

}  // namespace

int ns_prep(const ouo_mat* X, int x_dtype, const Group& grp, bool transpose,
            bool normalize, float eps, const Buf& x0, double* scratch,
            cudaStream_t stream) {
  const int nb = (int)grp.members.size();
  float* scales = reinterpret_cast<float*>(scratch + (size_t)nb * grp.rows);
  for (int c0 = 0; c0 < nb; c0 += kChunk) {
    int cn = nb - c0 < kChunk ? nb - c0 : kChunk;
    if (normalize) {
      RowSqArgs ra;
      ra.nmat = cn;
      ra.x_bf16 = x_dtype == OUO_BF16;
      ra.out = scratch + (size_t)c0 * grp.rows;
      ra.cols = grp.cols;
      for (int i = 0; i < cn; ++i) {
        const ouo_mat& m = X[grp.members[c0 + i]];
        ra.row_start[i] = (int64_t)i * grp.rows;
        ra.X[i] = m.ptr;
        ra.ldx[i] = m.ld;
      }
      ra.row_start[cn] = (int64_t)cn * grp.rows;
      int64_t blocks = ceil_div(ra.row_start[cn], 8);
      int64_t cap = (int64_t)num_sms() * 8;
      rowsq_kernel<<<(unsigned)(blocks < cap ? blocks : cap), 256, 0, stream>>>(ra);
      OUO_CHECK_LAUNCH();
      matscale_kernel<<<cn, 256, 0, stream>>>(scratch + (size_t)c0 * grp.rows,
                                              grp.rows, eps, scales + c0);
      OUO_CHECK_LAUNCH();
    }
    if (!transpose) {
      RowCopyArgs ra;
      ra.nmat = cn;
      ra.src_bf16 = x_dtype == OUO_BF16;
      ra.dst_bf16 = x0.dtype == OUO_BF16;
      ra.to_caller = 0;
      ra.scale = normalize ? scales + c0 : nullptr;
      ra.rows = grp.rows;
      ra.cols = grp.cols;
      for (int i = 0; i < cn; ++i) {
        const ouo_mat& m = X[grp.members[c0 + i]];
        ra.C[i] = m.ptr;
        ra.ldc[i] = m.ld;
        ra.vec[i] = vec16(m, x_dtype);
      }
      ra.wbase = x0.p + (size_t)c0 * x0.stride * elem_size(x0.dtype);
      ra.wld = x0.ld;
      ra.wstride = x0.stride;
      rowcopy_kernel<<<rows_grid(grp.rows * cn), 256, 0, stream>>>(ra);
      OUO_CHECK_LAUNCH();
      continue;
    }
    CopyArgs ca;
    ca.nmat = cn;
    ca.src_bf16 = x_dtype == OUO_BF16;
    ca.dst_bf16 = x0.dtype == OUO_BF16;
    ca.transpose = transpose;
    ca.to_caller = 0;
    ca.scale = normalize ? scales + c0 : nullptr;
    ca.rows = grp.rows;
    ca.cols = grp.cols;
    for (int i = 0; i < cn; ++i) {
      const ouo_mat& m = X[grp.members[c0 + i]];
      ca.C[i] = m.ptr;
      ca.ldc[i] = m.ld;
    }
    ca.wbase = x0.p + (size_t)c0 * x0.stride * elem_size(x0.dtype);
    ca.wld = x0.ld;
    ca.wstride = x0.stride;
    copy_kernel<<<copy_grid(grp.rows, grp.cols, cn), 256, 0, stream>>>(ca);
    OUO_CHECK_LAUNCH();
  }
  return OUO_OK;
}

int ns_writeout(const Buf& y, const ouo_mat* O, int o_dtype, const Group& grp,
                bool transpose, cudaStream_t stream) {
  const int nb = (int)grp.members.size();
  for (int c0 = 0; c0 < nb; c0 += kChunk) {
    int cn = nb - c0 < kChunk ? nb - c0 : kChunk;
    if (!transpose) {
      RowCopyArgs ra;
      ra.nmat = cn;
      ra.src_bf16 = y.dtype == OUO_BF16;
      ra.dst_bf16 = o_dtype == OUO_BF16;
      ra.to_caller = 1;
      ra.scale = nullptr;
      ra.rows = grp.rows;
      ra.cols = grp.cols;
      for (int i = 0; i < cn; ++i) {
        const ouo_mat& m = O[grp.members[c0 + i]];
        ra.C[i] = m.ptr;
        ra.ldc[i] = m.ld;
        ra.vec[i] = vec16(m, o_dtype);
      }
      ra.wbase = y.p + (size_t)c0 * y.stride * elem_size(y.dtype);
      ra.wld = y.ld;
      ra.wstride = y.stride;
      rowcopy_kernel<<<rows_grid(grp.rows * cn), 256, 0, stream>>>(ra);
      OUO_CHECK_LAUNCH();
      continue;
    }
    CopyArgs ca;
    ca.nmat = cn;
    ca.src_bf16 = y.dtype == OUO_BF16;
    ca.dst_bf16 = o_dtype == OUO_BF16;
    ca.transpose = transpose;
    ca.to_caller = 1;
    ca.scale = nullptr;
    ca.rows = grp.rows;
    ca.cols = grp.cols;
    for (int i = 0; i < cn; ++i) {
      const ouo_mat& m = O[grp.members[c0 + i]];
      ca.C[i] = m.ptr;
      ca.ldc[i] = m.ld;
    }
    ca.wbase = y.p + (size_t)c0 * y.stride * elem_size(y.dtype);
    ca.wld = y.ld;
    ca.wstride = y.stride;
    copy_kernel<<<copy_grid(grp.rows, grp.cols, cn), 256, 0, stream>>>(ca);
    OUO_CHECK_LAUNCH();
  }
  return OUO_OK;
}

int fill_identity(const Buf& q, cudaStream_t stream) {
  int64_t total = q.rows * q.cols * q.nb;
  int64_t blocks = ceil_div(total, 256);
  int64_t cap = (int64_t)num_sms() * 8;
  identity_kernel<<<(unsigned)(blocks < cap ? blocks : cap), 256, 0, stream>>>(
      q.p, q.dtype == OUO_BF16, q.rows, q.cols, q.ld, q.stride, q.nb);
  OUO_CHECK_LAUNCH();
  return OUO_OK;
}

int convert_buf(const Buf& src, const Buf& dst, cudaStream_t stream) {
  int64_t total = src.rows * src.cols * src.nb;
  int64_t blocks = ceil_div(total, 256);
  int64_t cap = (int64_t)num_sms() * 8;
  convert_kernel<<<(unsigned)(blocks < cap ? blocks : cap), 256, 0, stream>>>(
      src.p, src.dtype == OUO_BF16, dst.p, dst.dtype == OUO_BF16, src.rows,
      src.cols, src.ld, src.stride, dst.ld, dst.stride, src.nb);
  OUO_CHECK_LAUNCH();
  return OUO_OK;
}

}  // namespace ouo
