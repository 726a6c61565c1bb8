// Tensor-core GEMM for sm_100a: tcgen05.mma with fp32 accumulators in TMEM,
// operands staged in shared memory by TMA (no multicast), warp-specialized
// and persistent over output tiles.
//
//   C[b] = alpha * A[b] op(B[b]) + beta * C0[b] + gamma * I
//
// Roles (192 threads): warp 0 lane 0 issues TMA loads into a ring of
// shared-memory stages; warp 1 lane 0 issues tcgen05.mma (one thread per
// CTA) into one of two TMEM accumulators; warps 2-5 drain the other
// accumulator (tcgen05.ld, one TMEM lane quarter per warp) and run the
// epilogue.  Every wait is an mbarrier wait bounded in time; a wait that runs
// out sets OUO_STATUS_TIMEOUT and the CTA winds down cleanly (drains its MMAs,
// frees TMEM, returns).
//
// Symmetric outputs (the Gram matrix X X^T and the products of commuting
// symmetric matrices in Gram Newton-Schulz) are computed with a triangular
// tile scheduler: only 128 x BN tiles that reach the diagonal or above are
// scheduled, and each element (i, j >= i) is written to (i, j) and (j, i).
// This is the symmetric-GEMM idea of "Dion3：全栈正交更新", 核心模块 (upper
// triangle only, transposed write-back), restated for tcgen05.
//
// Tile: 128 (M) x BN (N), K staged 128 bytes per stage (64 bf16 or 32 tf32
// elements) with the 128-byte swizzle.  A is always K-major.  B is K-major
// (an N x K buffer) or MN-major (a K x N buffer, e.g. X in Q X).
#include <cuda.h>

#include <cstring>
#include <mutex>

#include "internal.h"
#include "umma.cuh"

namespace ouo {
namespace {

constexpr int kEpiWarps = 8;                 // two per TMEM lane quarter
constexpr int kThreads = 64 + 32 * kEpiWarps;  // producer, MMA, epilogue
constexpr uint32_t kTileM = 128;
constexpr uint32_t kRowBytes = 128;  // one swizzle row: K bytes per stage
// Epilogue staging: a 32 x 32 fp32 chunk per warp, 16-byte groups XOR-
// swizzled by row so that row-wise and column-wise accesses are both free
// of bank conflicts.
__device__ __forceinline__ int stg_idx(int row, int col) {
  return row * 32 + ((((col >> 2) ^ row) & 7) << 2) + (col & 3) +
         ((col >> 5) << 5);
}

struct UmmaArgs {
  CUtensorMap tmA;
  CUtensorMap tmB;
  int64_t M, N, K, nb;
  int64_t tiles_m, tiles_n, tiles_per_mat, total_tiles;
  int tri;
  float alpha, beta, gamma;
  int has_c0, c0_bf16, has_f32, round_tf32, has_bf16;
  const void* C0;
  int64_t ldc0, sc0;
  float* Of;
  int64_t ldof, sof;
  uint16_t* Ob;
  int64_t ldob, sob;
  int* status;
};

template <int BN>
struct Cfg {
  static constexpr uint32_t kABytes = kTileM * kRowBytes;       // 16 KB
  static constexpr uint32_t kBBytes = (uint32_t)BN * kRowBytes;  // 16/32 KB
  static constexpr uint32_t kStageBytes = kABytes + kBBytes;
  static constexpr int kStages = BN == 256 ? 4 : 6;
  static constexpr uint32_t kTmemCols = 2 * BN;
  // per epilogue warp: a 32 x 32 fp32 staging buffer
  static constexpr uint32_t kEpiBytes = kEpiWarps * 32 * 32 * 4;
  static constexpr size_t kSmem =
      1024 + (size_t)kStages * kStageBytes + 256 + kEpiBytes;
};

// First column tile of row tile i that reaches the diagonal.
__device__ __forceinline__ int64_t tri_jmin(int64_t i, int BN) {
  return (i * (int64_t)kTileM) / BN;
}

__device__ __forceinline__ void decode_tile(const UmmaArgs& a, int BN,
                                            int64_t tile, int64_t* b,
                                            int64_t* ti, int64_t* tj) {
  *b = tile / a.tiles_per_mat;
  int64_t t = tile - *b * a.tiles_per_mat;
  if (!a.tri) {
    *ti = t / a.tiles_n;
    *tj = t - *ti * a.tiles_n;
    return;
  }
  int64_t i = 0;
  while (true) {
    int64_t cnt = a.tiles_n - tri_jmin(i, BN);
    if (t < cnt) break;
    t -= cnt;
    ++i;
  }
  *ti = i;
  *tj = tri_jmin(i, BN) + t;
}

__device__ __forceinline__ void store_out(const UmmaArgs& a, int64_t b,
                                          int64_t i, int64_t j, float v) {
  if (a.has_f32)
    a.Of[b * a.sof + i * a.ldof + j] = a.round_tf32 ? round_tf32(v) : v;
  if (a.has_bf16) a.Ob[b * a.sob + i * a.ldob + j] = f32_to_bf16(v);
}

// Stores 4 consecutive elements (row, col .. col+3); element t only when
// bit t of `mask` is set.  Full masks use one 16-byte (fp32) or 8-byte
// (bf16) store: workspace rows are 16-byte aligned and col is a multiple of 4.
__device__ __forceinline__ void store4(const UmmaArgs& a, int64_t b,
                                       int64_t row, int64_t col, float4 w,
                                       uint32_t mask) {
  if (mask == 0xFu) {
    if (a.has_f32) {
      float4 o = w;
      if (a.round_tf32) {
        o.x = round_tf32(o.x); o.y = round_tf32(o.y);
        o.z = round_tf32(o.z); o.w = round_tf32(o.w);
      }
      *reinterpret_cast<float4*>(a.Of + b * a.sof + row * a.ldof + col) = o;
    }
    if (a.has_bf16) {
      uint2 u;
      u.x = pack_bf16x2(w.x, w.y);
      u.y = pack_bf16x2(w.z, w.w);
      *reinterpret_cast<uint2*>(a.Ob + b * a.sob + row * a.ldob + col) = u;
    }
    return;
  }
  const float e[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int t = 0; t < 4; ++t)
    if (mask & (1u << t)) store_out(a, b, row, col + t, e[t]);
}

__device__ __forceinline__ float load_c0(const UmmaArgs& a, int64_t b,
                                         int64_t i, int64_t j) {
  const int64_t off = b * a.sc0 + i * a.ldc0 + j;
  return a.c0_bf16 ? bf16_to_f32(reinterpret_cast<const uint16_t*>(a.C0)[off])
                   : reinterpret_cast<const float*>(a.C0)[off];
}

template <int BN, int FMT /*1 bf16, 2 tf32*/, int B_MN>
__global__ void __launch_bounds__(kThreads, 1)
umma_gemm_kernel(const __grid_constant__ UmmaArgs a) {
  using C = Cfg<BN>;
  constexpr uint32_t kEs = FMT == 1 ? 2 : 4;           // element bytes
  constexpr uint32_t kBK = kRowBytes / kEs;            // K elements per stage
  constexpr uint32_t kInstK = 32 / kEs;                // K per MMA (32 bytes)
  constexpr uint32_t kChunkCols = kRowBytes / kEs;     // MN-major chunk width
  constexpr uint32_t kChunkBytes = kBK * kRowBytes;    // one MN-major chunk
  constexpr uint32_t kIdesc = ptx::instr_desc(FMT, B_MN, BN);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kStages * C::kStageBytes);
  uint64_t* empty = full + C::kStages;
  uint64_t* tfull = empty + C::kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  float* epi_smem =
      reinterpret_cast<float*>(smem + C::kStages * C::kStageBytes + 256);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(&tfull[s], 1);
      ptx::mbar_init(&tempty[s], kEpiWarps);  // one arrival per epilogue warp
    }
    ptx::mbar_init(drain, 1);
    *abort_flag = 0;
    ptx::fence_barrier_init();
    ptx::prefetch_tmap(&a.tmA);
    ptx::prefetch_tmap(&a.tmB);
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_holder, C::kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int64_t nk = (a.K + kBK - 1) / kBK;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ producer
    uint32_t stage = 0, phase = 0;
    bool ok = true;
    int64_t issued = 0;
    for (int64_t tile = blockIdx.x; ok && tile < a.total_tiles;
         tile += gridDim.x) {
      int64_t b, ti, tj;
      decode_tile(a, BN, tile, &b, &ti, &tj);
      for (int64_t kb = 0; kb < nk; ++kb) {
        if (!ptx::mbar_wait(&empty[stage], phase ^ 1, abort_flag)) {
          ok = false;
          break;
        }
        ptx::mbar_arrive_expect_tx(&full[stage], C::kStageBytes);
        uint8_t* sa = smem + stage * C::kStageBytes;
        uint8_t* sb = sa + C::kABytes;
        ptx::tma_load_3d(sa, &a.tmA, &full[stage], (int32_t)(kb * kBK),
                         (int32_t)(ti * kTileM), (int32_t)b);
        if (!B_MN) {
          ptx::tma_load_3d(sb, &a.tmB, &full[stage], (int32_t)(kb * kBK),
                           (int32_t)(tj * BN), (int32_t)b);
        } else {
#pragma unroll
          for (uint32_t c = 0; c < (uint32_t)BN / kChunkCols; ++c)
            ptx::tma_load_3d(sb + c * kChunkBytes, &a.tmB, &full[stage],
                             (int32_t)(tj * BN + c * kChunkCols),
                             (int32_t)(kb * kBK), (int32_t)b);
        }
        ++issued;
        if (++stage == (uint32_t)C::kStages) { stage = 0; phase ^= 1; }
      }
    }
    if (!ok) {
      *abort_flag = 1;
      report_status(a.status, OUO_STATUS_TIMEOUT);
    }
    // Loads still in flight complete on their own; before the CTA exits,
    // wait (bounded) for the last fill of every stage to land.
    if (!ok) {
      for (int s = 0; s < C::kStages; ++s) {
        const int64_t fills = issued / C::kStages + (s < issued % C::kStages ? 1 : 0);
        if (fills > 0)
          ptx::mbar_wait_timed(&full[s], (uint32_t)((fills - 1) & 1), 100000000ull);
      }
    }
  } else if (warp == 1 && lane == 0) {
    // ----------------------------------------------------------- MMA issuer
    uint32_t stage = 0, phase = 0;
    bool ok = true;
    int64_t local = 0;
    for (int64_t tile = blockIdx.x; ok && tile < a.total_tiles;
         tile += gridDim.x, ++local) {
      const uint32_t buf = (uint32_t)(local & 1);
      const uint32_t tphase = (uint32_t)((local >> 1) & 1);
      if (!ptx::mbar_wait(&tempty[buf], tphase ^ 1, abort_flag)) {
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      const uint32_t d = tmem_base + buf * BN;
      for (int64_t kb = 0; kb < nk; ++kb) {
        if (!ptx::mbar_wait(&full[stage], phase, abort_flag)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t sa = ptx::smem_u32(smem + stage * C::kStageBytes);
        const uint32_t sb = sa + C::kABytes;
#pragma unroll
        for (uint32_t kk = 0; kk < kBK / kInstK; ++kk) {
          const uint64_t ad = ptx::smem_desc_sw128(sa + kk * 32, 16, 1024);
          const uint64_t bd =
              B_MN ? ptx::smem_desc_sw128(sb + kk * kInstK * kRowBytes,
                                          kChunkBytes, 1024)
                   : ptx::smem_desc_sw128(sb + kk * 32, 16, 1024);
          const uint32_t acc = (kb > 0 || kk > 0) ? 1u : 0u;
          if (FMT == 1) ptx::mma_bf16(d, ad, bd, kIdesc, acc);
          else ptx::mma_tf32(d, ad, bd, kIdesc, acc);
        }
        ptx::mma_commit(&empty[stage]);
        if (++stage == (uint32_t)C::kStages) { stage = 0; phase ^= 1; }
      }
      if (!ok) break;
      ptx::mma_commit(&tfull[buf]);
    }
    if (!ok) {
      *abort_flag = 1;
      report_status(a.status, OUO_STATUS_TIMEOUT);
    }
    // all MMAs of this thread complete before TMEM is released
    ptx::mma_commit(drain);
    ptx::mbar_wait_timed(drain, 0, kWaitLimitNs);
  } else if (warp >= 2) {
    // ------------------------------------------------------------- epilogue
    const uint32_t q = (uint32_t)(warp & 3);  // TMEM lanes 32q .. 32q+31
    int64_t local = 0;
    for (int64_t tile = blockIdx.x; tile < a.total_tiles;
         tile += gridDim.x, ++local) {
      int64_t b, ti, tj;
      decode_tile(a, BN, tile, &b, &ti, &tj);
      const uint32_t buf = (uint32_t)(local & 1);
      const uint32_t tphase = (uint32_t)((local >> 1) & 1);
      if (!ptx::mbar_wait(&tfull[buf], tphase, abort_flag)) {
        *abort_flag = 1;
        report_status(a.status, OUO_STATUS_TIMEOUT);
        break;
      }
      ptx::tc_fence_after();
      // This warp owns tile rows q*32 .. q*32+31 (TMEM lanes) and one half
      // of the columns; each chunk is 32 rows x 32 columns.  Values are
      // finished with row = lane (where the symmetric C0 read (j, i) is
      // coalesced), staged in shared memory, and written back with 16-byte
      // stores: 8 lanes per 128-byte row, 4 rows per instruction, for the
      // direct tile (i, j) and, for symmetric outputs, the mirrored tile
      // (j, i).  Chunks entirely below the diagonal of a symmetric output
      // are skipped; chunks fully inside and above it store without masks.
      const int64_t row_base = ti * kTileM + q * 32;
      const int64_t gi = row_base + lane;
      float* stg = epi_smem + (warp - 2) * (32 * 32);
      const int sub_r = lane >> 3, sub_c = 4 * (lane & 7);
      const uint32_t half = (uint32_t)((warp - 2) >> 2);
#pragma unroll 1
      for (uint32_t c0 = half * (BN / 2); c0 < (half + 1) * (BN / 2); c0 += 32) {
        const int64_t gj0 = tj * BN + c0;
        if (a.tri && gj0 + 31 < row_base) continue;  // below the diagonal
        if (row_base >= a.M || gj0 >= a.N) continue;  // outside the output
        const bool full_chunk = row_base + 32 <= a.M && gj0 + 32 <= a.N &&
                                (!a.tri || gj0 >= row_base + 31);
        float v[32];
        ptx::tmem_ld32(tmem_base + ((q * 32u) << 16) + buf * BN + c0, v);
        if (a.tri) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int64_t gj = gj0 + j;
            float r = a.alpha * v[j];
            if (a.has_c0 && (full_chunk || (gi < a.M && gj < a.N && gj >= gi)))
              r += a.beta * load_c0(a, b, gj, gi);
            if (gi == gj) r += a.gamma;
            v[j] = r;
          }
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] *= a.alpha;
        }
        // direct tile: stage row-major [row][col]
#pragma unroll
        for (int j = 0; j < 32; j += 4)
          *reinterpret_cast<float4*>(stg + stg_idx(lane, j)) =
              make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
        __syncwarp();
#pragma unroll 2
        for (int it = 0; it < 8; ++it) {
          const int rr = it * 4 + sub_r;
          const int64_t gr = row_base + rr, gc = gj0 + sub_c;
          float4 w = *reinterpret_cast<const float4*>(stg + stg_idx(rr, sub_c));
          uint32_t mask = 0xFu;
          if (!full_chunk) {
            mask = 0;
#pragma unroll
            for (int t = 0; t < 4; ++t)
              if (gr < a.M && gc + t < a.N && (!a.tri || gc + t >= gr)) mask |= 1u << t;
          }
          if (!a.tri && mask && (a.has_c0 || a.gamma != 0.f)) {
            float e[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int t = 0; t < 4; ++t) {
              if (!(mask & (1u << t))) continue;
              if (a.has_c0) e[t] += a.beta * load_c0(a, b, gr, gc + t);
              if (gr == gc + t) e[t] += a.gamma;
            }
            w = make_float4(e[0], e[1], e[2], e[3]);
          }
          if (mask) store4(a, b, gr, gc, w, mask);
        }
        __syncwarp();
        if (a.tri) {
          // mirrored tile: stage transposed [col][row], store row gj
#pragma unroll
          for (int j = 0; j < 32; ++j) stg[stg_idx(j, lane)] = v[j];
          __syncwarp();
#pragma unroll 2
          for (int it = 0; it < 8; ++it) {
            const int rr = it * 4 + sub_r;           // source column offset
            const int64_t dst_r = gj0 + rr;          // = source column gj
            const int64_t dst_c = row_base + sub_c;  // = source rows gi
            float4 w = *reinterpret_cast<const float4*>(stg + stg_idx(rr, sub_c));
            uint32_t mask = 0xFu;
            if (!full_chunk) {
              mask = 0;
#pragma unroll
              for (int t = 0; t < 4; ++t)
                if (dst_c + t < a.M && dst_r < a.N && dst_r >= dst_c + t) mask |= 1u << t;
            }
            if (mask) store4(a, b, dst_r, dst_c, w, mask);
          }
          __syncwarp();
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&tempty[buf]);
    }
  }
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// ------------------------------------------------------------------- host

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t,
                                  void*, const cuuint64_t*, const cuuint64_t*,
                                  const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000,
                                         cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 3-D map over a workspace batch [nb][rows][ld]: dims (cols, rows, nb), box
// (box_cols, box_rows, 1), 128-byte swizzle, zero fill out of bounds.
int make_map(CUtensorMap* map, const Buf& t, uint32_t box_cols,
             uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn)
    return set_error(OUO_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  const size_t es = elem_size(t.dtype);
  cuuint64_t dims[3] = {(cuuint64_t)t.cols, (cuuint64_t)t.rows,
                        (cuuint64_t)t.nb};
  cuuint64_t strides[2] = {(cuuint64_t)(t.ld * es), (cuuint64_t)(t.stride * es)};
  cuuint32_t box[3] = {box_cols, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map,
                  t.dtype == OUO_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                      : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                  3, t.p, dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return set_error(OUO_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return OUO_OK;
}

template <int BN, int FMT, int B_MN>
int launch(const GemmDesc& g, UmmaArgs& a, cudaStream_t stream) {
  using C = Cfg<BN>;
  constexpr uint32_t es = FMT == 1 ? 2 : 4;
  constexpr uint32_t bk = kRowBytes / es;
  OUO_TRY(make_map(&a.tmA, g.A, bk, kTileM));
  if (!B_MN) OUO_TRY(make_map(&a.tmB, g.B, bk, BN));
  else OUO_TRY(make_map(&a.tmB, g.B, kRowBytes / es, bk));
  a.tiles_m = ceil_div(g.M, kTileM);
  a.tiles_n = ceil_div(g.N, BN);
  if (g.tri) {
    int64_t cnt = 0;
    for (int64_t i = 0; i < a.tiles_m; ++i) cnt += a.tiles_n - (i * (int64_t)kTileM) / BN;
    a.tiles_per_mat = cnt;
  } else {
    a.tiles_per_mat = a.tiles_m * a.tiles_n;
  }
  a.total_tiles = a.tiles_per_mat * g.nb;
  auto kern = umma_gemm_kernel<BN, FMT, B_MN>;
  static bool configured[64] = {false};
  int dev = 0;
  OUO_CHECK_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64 || !configured[dev]) {
    OUO_CHECK_CUDA(cudaFuncSetAttribute(
        kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::kSmem));
    if (dev >= 0 && dev < 64) configured[dev] = true;
  }
  int64_t grid = a.total_tiles < num_sms() ? a.total_tiles : num_sms();
  if (grid < 1) return OUO_OK;
  kern<<<(unsigned)grid, kThreads, C::kSmem, stream>>>(a);
  OUO_CHECK_LAUNCH();
  return OUO_OK;
}

}  // namespace

int gemm_umma(const GemmDesc& g, cudaStream_t stream, int* status) {
  if (g.A.dtype != g.B.dtype)
    return set_error(OUO_ERR_UNSUPPORTED, "tensor-core GEMM needs equal operand types");
  if (g.tri && (g.M != g.N || g.b_mn))
    return set_error(OUO_ERR_INVALID_ARG, "symmetric GEMM needs M == N, K-major B");
  if (g.M < 1 || g.N < 1 || g.K < 1 || g.nb < 1) return OUO_OK;
  UmmaArgs a;
  memset(&a, 0, sizeof(a));
  a.M = g.M; a.N = g.N; a.K = g.K; a.nb = g.nb;
  a.tri = g.tri;
  a.alpha = g.alpha; a.beta = g.beta; a.gamma = g.gamma;
  a.has_c0 = g.has_c0;
  a.c0_bf16 = g.has_c0 && g.C0.dtype == OUO_BF16;
  a.C0 = g.has_c0 ? g.C0.p : nullptr;
  a.ldc0 = g.C0.ld; a.sc0 = g.C0.stride;
  a.has_f32 = g.has_f32; a.round_tf32 = g.round_tf32;
  a.Of = g.has_f32 ? reinterpret_cast<float*>(g.out_f32.p) : nullptr;
  a.ldof = g.out_f32.ld; a.sof = g.out_f32.stride;
  a.has_bf16 = g.has_bf16;
  a.Ob = g.has_bf16 ? reinterpret_cast<uint16_t*>(g.out_bf16.p) : nullptr;
  a.ldob = g.out_bf16.ld; a.sob = g.out_bf16.stride;
  a.status = status;
  const bool wide = g.N > 128;
  if (g.A.dtype == OUO_BF16) {
    if (g.b_mn) return wide ? launch<256, 1, 1>(g, a, stream) : launch<128, 1, 1>(g, a, stream);
    return wide ? launch<256, 1, 0>(g, a, stream) : launch<128, 1, 0>(g, a, stream);
  }
  if (g.b_mn) return wide ? launch<256, 2, 1>(g, a, stream) : launch<128, 2, 1>(g, a, stream);
  return wide ? launch<256, 2, 0>(g, a, stream) : launch<128, 2, 0>(g, a, stream);
}

}  // namespace ouo
