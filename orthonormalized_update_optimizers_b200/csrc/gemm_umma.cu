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
//
// CTA-pair mode (CG = 2, BN = 256): the launch is made of clusters of two
// CTAs on neighbouring SMs that share one 256 x 256 tile.  Each CTA stages
// its own 128 rows of A and its own half (128 columns) of B, so an SM moves
// two thirds of the operand bytes of the single-CTA 128 x 256 tile for the
// same number of MMA cycles.  The even CTA issues tcgen05.mma.cta_group::2
// (M = 256) over both CTAs' shared memory; both CTAs' TMA loads complete on
// the even CTA's stage barrier, MMA completion is multicast to the stage and
// accumulator barriers of both CTAs (tcgen05.commit multicast), and each CTA
// drains its own 128 TMEM lanes.  TMA loads never multicast.
#include <cuda.h>

#include <cstdlib>
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
// bf16 staging for TMA stores: 64-byte rows, 16-byte chunks XOR (row / 2) % 4
// (the 64-byte swizzle pattern).
__device__ __forceinline__ int stg16_idx(int row, int col) {
  return row * 32 + ((((col >> 3) ^ (row >> 1)) & 3) << 3) + (col & 7);
}

// Epilogue staging: a 32 x 32 fp32 chunk per warp, 16-byte groups XOR-
// swizzled by row so that row-wise and column-wise accesses are both free
// of bank conflicts.
__device__ __forceinline__ int stg_idx(int row, int col) {
  return row * 32 + ((((col >> 2) ^ row) & 7) << 2) + (col & 3) +
         ((col >> 5) << 5);
}

// One segment of a launch: a batch range [b0, b0 + nb) of one group of
// equal-shape matrices, with its own operand maps, sizes and outputs.
struct Segment {
  CUtensorMap tmA;
  CUtensorMap tmB;
  CUtensorMap tmC;  // workspace output (TMA-store epilogue)
  int64_t M, N, K;
  int64_t nb, b0;
  int64_t tiles_n, tiles_per_mat, tile_start;  // tile_start: first tile id
  const void* C0;
  int64_t ldc0, sc0;
  float* Of;
  int64_t ldof, sof;
  uint16_t* Ob;
  int64_t ldob, sob;
  int direct;  // outputs go to dptr[dbase + b]
  int dbase;
  int b4d;  // MN-major B: tmB is 4-D, one TMA load brings every chunk of a stage
  // upper-stored symmetric operands: maps of the same matrices read with
  // rows and columns exchanged (MN-major tiles; 4-D when the matrix splits
  // into whole 32-column chunks, else one 3-D load per chunk)
  CUtensorMap tmAt;
  CUtensorMap tmBt;
  int t4d;
  // split-K: the K blocks of every output tile are divided into `ksplit`
  // ranges of `kbc` blocks; range s of matrix b is written to output matrix
  // b * ksplit + s (workspace outputs only), to be summed by the caller
  int ksplit;
  int64_t kbc;
  int64_t tiles_2d;  // output tiles of one matrix (tiles_per_mat / ksplit)
  // split-tf32 passes: the K blocks are walked `npass` times; pass q reads
  // A from UmmaArgs::lo_map[segment][0] when bit q of a_lo is set (from
  // lo_map[segment][2] for a_lo2), B from lo_map[segment][1] for b_lo
  int npass, a_lo, b_lo, a_lo2;
};

constexpr int kMaxSeg = 6;

struct UmmaArgs {
  Segment seg[kMaxSeg];
  int nseg;
  int64_t total_tiles;
  int tri;
  float alpha, beta, gamma;
  int has_c0, c0_bf16, has_f32, round_tf32, has_bf16;
  int c0_out;  // C0 is read from the (direct) output itself
  int a_sym, b_sym, c0_upper, sym_half;  // upper-stored symmetric matrices
  int tma_out;  // single workspace output written by TMA stores
  int* status;
  void* dptr[kChunk];
  int64_t dld[kChunk];
  // per-matrix alpha of direct outputs (has_dalpha), else `alpha` for all
  float dalpha[kChunk];
  int has_dalpha;
  // residual operands of the split-tf32 passes, per segment (A2, B2, A3);
  // kept out of Segment so that the fields every tile reads stay compact
  CUtensorMap lo_map[kMaxSeg][3];
};
static_assert(sizeof(UmmaArgs) <= 32764, "kernel parameters above the 32 KB limit");

// UPD: in-place rank-r updates (K = r, short main loops): fewer operand
// stages, four staging buffers per epilogue warp, so that three C0 boxes
// per warp are in flight.
template <int BN, int CG, int UPD = 0>
struct Cfg {
  static constexpr uint32_t kTileRows = kTileM * CG;  // rows of one scheduled tile
  static constexpr uint32_t kBRows = (uint32_t)BN / CG;  // B rows (N) staged per CTA
  static constexpr uint32_t kABytes = kTileM * kRowBytes;      // 16 KB
  static constexpr uint32_t kBBytes = kBRows * kRowBytes;      // 16/32 KB
  static constexpr uint32_t kStageBytes = kABytes + kBBytes;
  static constexpr int kStages = UPD ? 3 : (CG == 2 ? 5 : (BN == 256 ? 4 : 6));
  // epilogue staging buffers per warp: two where shared memory allows, so a
  // bulk store can still be reading one while the next chunk fills the other
  static constexpr int kStg = UPD ? 4 : (CG == 2 ? 2 : 1);
  static constexpr uint32_t kTmemCols = 2 * BN;
  // per epilogue warp: a 32 x 32 fp32 staging buffer
  static constexpr uint32_t kEpiBytes = kEpiWarps * kStg * 32 * 32 * 4;
  static constexpr size_t kSmem =
      1024 + (size_t)kStages * kStageBytes + 512 + kEpiBytes;
};

// First column tile of row tile i (tiles of TR rows) that reaches the
// diagonal.
__host__ __device__ __forceinline__ int64_t tri_jmin(int64_t i, int BN, int TR) {
  return (i * (int64_t)TR) / BN;
}

// Launch-wide tile id -> (segment, matrix within the segment, tile row,
// tile column).
__device__ __forceinline__ int decode_tile(const UmmaArgs& a, int BN, int TR,
                                           int64_t tile, int64_t* b,
                                           int64_t* ti, int64_t* tj,
                                           int64_t* ks) {
  int g = 0;
  while (g + 1 < a.nseg && tile >= a.seg[g + 1].tile_start) ++g;
  const Segment& sg = a.seg[g];
  int64_t t = tile - sg.tile_start;
  *b = t / sg.tiles_per_mat;
  t -= *b * sg.tiles_per_mat;
  *ks = 0;
  if (!a.tri) {
    *ks = t / sg.tiles_2d;
    t -= *ks * sg.tiles_2d;
    *ti = t / sg.tiles_n;
    *tj = t - *ti * sg.tiles_n;
    return g;
  }
  int64_t i = 0;
  while (true) {
    int64_t cnt = sg.tiles_n - tri_jmin(i, BN, TR);
    if (t < cnt) break;
    t -= cnt;
    ++i;
  }
  *ti = i;
  *tj = tri_jmin(i, BN, TR) + t;
  return g;
}

// Output element addresses: workspace batch [b0 + b] or a caller matrix.
__device__ __forceinline__ float* out_f32_at(const UmmaArgs& a,
                                             const Segment& sg, int64_t b,
                                             int64_t i, int64_t j) {
  return sg.direct
      ? reinterpret_cast<float*>(a.dptr[sg.dbase + b]) + i * a.dld[sg.dbase + b] + j
      : sg.Of + (sg.b0 + b) * sg.sof + i * sg.ldof + j;
}
__device__ __forceinline__ uint16_t* out_bf16_at(const UmmaArgs& a,
                                                 const Segment& sg, int64_t b,
                                                 int64_t i, int64_t j) {
  return sg.direct
      ? reinterpret_cast<uint16_t*>(a.dptr[sg.dbase + b]) + i * a.dld[sg.dbase + b] + j
      : sg.Ob + (sg.b0 + b) * sg.sob + i * sg.ldob + j;
}

// Output bases of one matrix of a segment (workspace or caller memory).
struct TileOut {
  float* f;
  uint16_t* h;
  int64_t ldf, ldh;
};

__device__ __forceinline__ TileOut tile_out(const UmmaArgs& a,
                                            const Segment& sg, int64_t b) {
  TileOut o;
  o.f = a.has_f32 ? out_f32_at(a, sg, b, 0, 0) : nullptr;
  o.h = a.has_bf16 ? out_bf16_at(a, sg, b, 0, 0) : nullptr;
  o.ldf = sg.direct ? a.dld[sg.dbase + b] : sg.ldof;
  o.ldh = sg.direct ? a.dld[sg.dbase + b] : sg.ldob;
  return o;
}

__device__ __forceinline__ void store_elem(const UmmaArgs& a, const TileOut& o,
                                           int64_t i, int64_t j, float v) {
  if (a.has_f32) o.f[i * o.ldf + j] = a.round_tf32 ? round_tf32(v) : v;
  if (a.has_bf16) o.h[i * o.ldh + j] = f32_to_bf16(v);
}

// Stores 4 consecutive elements (row, col .. col+3); element t only when
// bit t of `mask` is set.  Full masks use one 16-byte (fp32) or 8-byte
// (bf16) store: output rows are 16-byte aligned and col is a multiple of 4.
__device__ __forceinline__ void store4t(const UmmaArgs& a, const TileOut& o,
                                        int64_t row, int64_t col, float4 w,
                                        uint32_t mask) {
  if (mask == 0xFu) {
    if (a.has_f32) {
      float4 v = w;
      if (a.round_tf32) {
        v.x = round_tf32(v.x); v.y = round_tf32(v.y);
        v.z = round_tf32(v.z); v.w = round_tf32(v.w);
      }
      *reinterpret_cast<float4*>(o.f + row * o.ldf + col) = v;
    }
    if (a.has_bf16) {
      uint2 u;
      u.x = pack_bf16x2(w.x, w.y);
      u.y = pack_bf16x2(w.z, w.w);
      *reinterpret_cast<uint2*>(o.h + row * o.ldh + col) = u;
    }
    return;
  }
  const float e[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int t = 0; t < 4; ++t)
    if (mask & (1u << t)) store_elem(a, o, row, col + t, e[t]);
}

// In-place updates read their C0 from the output location.
__device__ __forceinline__ float load_out1(const UmmaArgs& a, const TileOut& o,
                                           int64_t i, int64_t j) {
  return a.has_f32 ? o.f[i * o.ldf + j] : bf16_to_f32(o.h[i * o.ldh + j]);
}

__device__ __forceinline__ void load_out4(const UmmaArgs& a, const TileOut& o,
                                          int64_t i, int64_t j, float e[4]) {
  if (a.has_f32) {
    float4 f = *reinterpret_cast<const float4*>(o.f + i * o.ldf + j);
    e[0] = f.x; e[1] = f.y; e[2] = f.z; e[3] = f.w;
  } else {
    uint2 u = *reinterpret_cast<const uint2*>(o.h + i * o.ldh + j);
    e[0] = __uint_as_float(u.x << 16);
    e[1] = __uint_as_float(u.x & 0xffff0000u);
    e[2] = __uint_as_float(u.y << 16);
    e[3] = __uint_as_float(u.y & 0xffff0000u);
  }
}

__device__ __forceinline__ float load_c0(const Segment& sg, int64_t b,
                                         int64_t i, int64_t j, int bf16) {
  const int64_t off = (sg.b0 + b) * sg.sc0 + i * sg.ldc0 + j;
  return bf16 ? bf16_to_f32(reinterpret_cast<const uint16_t*>(sg.C0)[off])
              : reinterpret_cast<const float*>(sg.C0)[off];
}

// Four consecutive C0 elements (i, j .. j+3); workspace rows are 16-byte
// aligned and j is a multiple of 4.
__device__ __forceinline__ void load_c0x4(const Segment& sg, int64_t b,
                                          int64_t i, int64_t j, float e[4],
                                          int bf16) {
  const int64_t off = (sg.b0 + b) * sg.sc0 + i * sg.ldc0 + j;
  if (bf16) {
    uint2 u = *reinterpret_cast<const uint2*>(
        reinterpret_cast<const uint16_t*>(sg.C0) + off);
    e[0] = __uint_as_float(u.x << 16);
    e[1] = __uint_as_float(u.x & 0xffff0000u);
    e[2] = __uint_as_float(u.y << 16);
    e[3] = __uint_as_float(u.y & 0xffff0000u);
  } else {
    float4 f = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(sg.C0) + off);
    e[0] = f.x; e[1] = f.y; e[2] = f.z; e[3] = f.w;
  }
}

template <int BN, int FMT /*1 bf16, 2 tf32*/, int B_MN, int CG /*CTAs per tile*/, int UPD>
__global__ void __launch_bounds__(kThreads, 1)
umma_gemm_kernel(const __grid_constant__ UmmaArgs a) {
  using C = Cfg<BN, CG, UPD>;
  constexpr int TR = (int)C::kTileRows;
  constexpr uint32_t kEs = FMT == 1 ? 2 : 4;           // element bytes
  constexpr uint32_t kBK = kRowBytes / kEs;            // K elements per stage
  constexpr uint32_t kInstK = 32 / kEs;                // K per MMA (32 bytes)
  constexpr uint32_t kChunkCols = kRowBytes / kEs;     // MN-major chunk width
  constexpr uint32_t kChunkBytes = kBK * kRowBytes;    // one MN-major chunk
  constexpr uint32_t kIdesc = ptx::instr_desc(FMT, B_MN, BN, kTileM * CG);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kStages * C::kStageBytes +
                                               C::kEpiBytes);
  uint64_t* empty = full + C::kStages;
  uint64_t* tfull = empty + C::kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  // per stage: bit 0 = A tile MN-major (transposed block), bit 1 = B tile
  volatile uint32_t* stage_fmt = reinterpret_cast<volatile uint32_t*>(tmem_holder + 2);
  // in-place TMA epilogue: one barrier per staging buffer of every epilogue
  // warp, completed by the TMA load of a C0 box into that buffer
  uint64_t* c0bar = reinterpret_cast<uint64_t*>(
      (reinterpret_cast<uintptr_t>(stage_fmt + C::kStages) + 7) & ~(uintptr_t)7);
  // per-warp 4 KB staging buffers, 1024-byte aligned (the TMA swizzle
  // patterns are computed from absolute shared-memory address bits)
  float* epi_smem = reinterpret_cast<float*>(smem + C::kStages * C::kStageBytes);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // CTA pair: rank 0 issues the MMAs and owns the stage and accumulator-free
  // barriers both CTAs signal; a scheduled tile is shared by the pair.
  const uint32_t rank = CG == 2 ? ptx::cluster_ctarank() : 0u;
  const int64_t tile0 = blockIdx.x / CG, tile_step = gridDim.x / CG;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(&tfull[s], 1);
      ptx::mbar_init(&tempty[s], kEpiWarps * CG);  // one arrival per epilogue warp
    }
    ptx::mbar_init(drain, 1);
    for (int i = 0; i < kEpiWarps * C::kStg; ++i) ptx::mbar_init(&c0bar[i], 1);
    *abort_flag = 0;
    ptx::fence_barrier_init();
    for (int g = 0; g < a.nseg; ++g) {
      ptx::prefetch_tmap(&a.seg[g].tmA);
      ptx::prefetch_tmap(&a.seg[g].tmB);
    }
  }
  if (warp == 1) {
    if (CG == 2) {
      ptx::tmem_alloc2(tmem_holder, C::kTmemCols);
      ptx::tmem_relinquish2();
    } else {
      ptx::tmem_alloc(tmem_holder, C::kTmemCols);
      ptx::tmem_relinquish();
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  // the peer's barriers are initialized before anything signals them
  if (CG == 2) ptx::cluster_sync();
  ptx::tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ producer
    uint32_t stage = 0, phase = 0;
    bool ok = true;
    int64_t issued = 0;
    for (int64_t tile = tile0; ok && tile < a.total_tiles;
         tile += tile_step) {
      int64_t b, ti, tj, ks;
      const int g = decode_tile(a, BN, TR, tile, &b, &ti, &tj, &ks);
      const Segment& sg = a.seg[g];
      const int64_t nkr = (sg.K + kBK - 1) / kBK;  // K blocks of one pass
      const int64_t nk = nkr * sg.npass;
      const int64_t kb0 = ks * sg.kbc;
      const int64_t kb1 = kb0 + sg.kbc < nk ? kb0 + sg.kbc : nk;
      const int32_t z = (int32_t)(sg.b0 + b);
      const int32_t arow = (int32_t)(ti * TR + rank * kTileM);
      const int32_t bcol = (int32_t)(tj * BN + rank * C::kBRows);
      // pass and K block within the pass, advanced by counting (no division
      // per stage); the operands of the pass
      int64_t pass = kb0 >= nkr ? kb0 / nkr : 0;
      int64_t kb = kb0 - pass * nkr;
      for (int64_t kbv = kb0; kbv < kb1; ++kbv, ++kb) {
        if (kb == nkr) {
          kb = 0;
          ++pass;
        }
        if (!ptx::mbar_wait(&empty[stage], phase ^ 1, abort_flag)) {
          ok = false;
          break;
        }
        const CUtensorMap* mA = ((sg.a_lo2 >> pass) & 1) ? &a.lo_map[g][2]
                                : ((sg.a_lo >> pass) & 1) ? &a.lo_map[g][0] : &sg.tmA;
        const CUtensorMap* mB = ((sg.b_lo >> pass) & 1) ? &a.lo_map[g][1] : &sg.tmB;
        // Upper-stored symmetric operands: a K stage left of the tile's block
        // diagonal (256-wide blocks, pair tiles) comes from the transposed
        // block.  Both CTAs of a pair take the same decision.
        const int64_t cblk = (kb * (int64_t)kBK) / 256;
        const bool at = CG == 2 && a.a_sym && cblk < ti;
        const bool bt = CG == 2 && a.b_sym && cblk < tj;
        if (rank == 0) stage_fmt[stage] = (at ? 1u : 0u) | (bt ? 2u : 0u);
        // the stage barrier of the pair's even CTA counts both CTAs' bytes
        if (rank == 0) ptx::mbar_arrive_expect_tx(&full[stage], CG * C::kStageBytes);
        const uint32_t fb = CG == 2 ? ptx::mapa(ptx::smem_u32(&full[stage]), 0) : 0u;
        auto load = [&](void* dst, const CUtensorMap* m, int32_t c0, int32_t c1) {
          if (CG == 2) ptx::tma_load_3d_pair(dst, m, fb, c0, c1, z);
          else ptx::tma_load_3d(dst, m, &full[stage], c0, c1, z);
        };
        uint8_t* sa = smem + stage * C::kStageBytes;
        uint8_t* sb = sa + C::kABytes;
        // transposed tile: rows = this K stage, columns = the tile's 128
        // rows (M or N), as 32-column MN-major chunks
        auto load_t = [&](uint8_t* dst, const CUtensorMap* m, int32_t col0) {
          if (CG == 2) {
            if (sg.t4d) {
              ptx::tma_load_4d_pair(dst, m, fb, 0, (int32_t)(kb * kBK), col0 / 32, z);
            } else {
#pragma unroll
              for (uint32_t c = 0; c < kTileM / 32; ++c)
                load(dst + c * kChunkBytes, m, col0 + (int32_t)(c * 32), (int32_t)(kb * kBK));
            }
          }
        };
        if (at) load_t(sa, &sg.tmAt, arow);
        else load(sa, mA, (int32_t)(kb * kBK), arow);
        if (bt) {
          load_t(sb, &sg.tmBt, bcol);
        } else if (!B_MN) {
          load(sb, mB, (int32_t)(kb * kBK), bcol);
        } else if (CG == 1 && sg.b4d) {
          // (chunk column, K row, chunk, matrix): the chunks land back to
          // back, the layout the per-chunk loads produce
          ptx::tma_load_4d(sb, mB, &full[stage], 0, (int32_t)(kb * kBK),
                           (int32_t)(bcol / kChunkCols), z);
        } else {
#pragma unroll
          for (uint32_t c = 0; c < C::kBRows / kChunkCols; ++c)
            load(sb + c * kChunkBytes, mB, (int32_t)(bcol + c * kChunkCols),
                 (int32_t)(kb * kBK));
        }
        ++issued;
        if (++stage == (uint32_t)C::kStages) { stage = 0; phase ^= 1; }
      }
    }
    if (!ok) {
      *abort_flag = 1;
      report_status(a.status, OUO_STATUS_TIMEOUT);
      // Loads still in flight complete on their own; before the CTA exits,
      // wait (bounded) for the last fill of every stage to land.  The odd
      // CTA of a pair signals the even CTA's barriers and cannot observe
      // them: it waits a fixed 2 ms, far longer than a tile load takes.
      if (CG == 2 && rank != 0) {
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 2000000ull) {
        }
        issued = 0;
      }
      for (int s = 0; s < C::kStages; ++s) {
        const int64_t fills = issued / C::kStages + (s < issued % C::kStages ? 1 : 0);
        if (fills > 0)
          ptx::mbar_wait_timed(&full[s], (uint32_t)((fills - 1) & 1), 100000000ull);
      }
    }
  } else if (warp == 1 && lane == 0 && rank == 0) {
    // ----------------------------------------------------------- MMA issuer
    uint32_t stage = 0, phase = 0;
    bool ok = true;
    int64_t local = 0;
    for (int64_t tile = tile0; ok && tile < a.total_tiles;
         tile += tile_step, ++local) {
      int64_t b, ti, tj, ks;
      const int g = decode_tile(a, BN, TR, tile, &b, &ti, &tj, &ks);
      const int64_t nk = (a.seg[g].K + kBK - 1) / kBK * a.seg[g].npass;
      const int64_t kb0 = ks * a.seg[g].kbc;
      const int64_t kb1 = kb0 + a.seg[g].kbc < nk ? kb0 + a.seg[g].kbc : nk;
      const uint32_t buf = (uint32_t)(local & 1);
      const uint32_t tphase = (uint32_t)((local >> 1) & 1);
      if (!ptx::mbar_wait(&tempty[buf], tphase ^ 1, abort_flag)) {
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      const uint32_t d = tmem_base + buf * BN;
      for (int64_t kb = kb0; kb < kb1; ++kb) {
        if (!ptx::mbar_wait(&full[stage], phase, abort_flag)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t sa = ptx::smem_u32(smem + stage * C::kStageBytes);
        const uint32_t sb = sa + C::kABytes;
        const uint32_t fmt = stage_fmt[stage];
        const bool a_mn = (fmt & 1u) != 0;
        const bool b_mn = B_MN || (fmt & 2u) != 0;
        const uint32_t idesc = kIdesc | (a_mn ? (1u << 15) : 0u) | (b_mn ? (1u << 16) : 0u);
        // MN-major tiles: chunks of one 128-byte row across kBK K rows; tf32
        // takes the 32-byte-atom swizzle (4-row groups)
        auto mn_desc = [&](uint32_t base, uint32_t kk) {
          return FMT == 2 ? ptx::smem_desc_sw128_32b(base + kk * kInstK * kRowBytes,
                                                     kChunkBytes, 512)
                          : ptx::smem_desc_sw128(base + kk * kInstK * kRowBytes,
                                                 kChunkBytes, 1024);
        };
#pragma unroll
        for (uint32_t kk = 0; kk < kBK / kInstK; ++kk) {
          const uint64_t ad = a_mn ? mn_desc(sa, kk) : ptx::smem_desc_sw128(sa + kk * 32, 16, 1024);
          const uint64_t bd = b_mn ? mn_desc(sb, kk) : ptx::smem_desc_sw128(sb + kk * 32, 16, 1024);
          const uint32_t acc = (kb > kb0 || kk > 0) ? 1u : 0u;
          if (CG == 2) {
            if (FMT == 1) ptx::mma2_bf16(d, ad, bd, idesc, acc);
            else ptx::mma2_tf32(d, ad, bd, idesc, acc);
          } else {
            if (FMT == 1) ptx::mma_bf16(d, ad, bd, idesc, acc);
            else ptx::mma_tf32(d, ad, bd, idesc, acc);
          }
        }
        // frees the stage in both CTAs of a pair
        if (CG == 2) ptx::mma2_commit(&empty[stage], 0x3);
        else ptx::mma_commit(&empty[stage]);
        if (++stage == (uint32_t)C::kStages) { stage = 0; phase ^= 1; }
      }
      if (!ok) break;
      if (CG == 2) ptx::mma2_commit(&tfull[buf], 0x3);
      else ptx::mma_commit(&tfull[buf]);
    }
    if (!ok) {
      *abort_flag = 1;
      report_status(a.status, OUO_STATUS_TIMEOUT);
    }
    // all MMAs of this thread complete before TMEM (of both CTAs of a pair)
    // is released
    if (CG == 2) ptx::mma2_commit(drain, 0x1);
    else ptx::mma_commit(drain);
    ptx::mbar_wait_timed(drain, 0, kWaitLimitNs);
  } else if (warp >= 2) {
    // ------------------------------------------------------------- epilogue
    const uint32_t q = (uint32_t)(warp & 3);  // TMEM lanes 32q .. 32q+31
    int64_t local = 0;
    // accumulator-free barrier of the pair's even CTA (cluster address)
    const uint32_t tempty_lead = CG == 2 ? ptx::mapa(ptx::smem_u32(tempty), 0) : 0u;
    uint32_t nstores = 0;  // bulk stores issued by this warp
    uint32_t c0ph = 0u;    // bit s: parity of the C0 box loads waited for in buffer s
    uint32_t c0pend = 0u;  // bit s: a C0 box load into buffer s not yet waited for
    for (int64_t tile = tile0; tile < a.total_tiles;
         tile += tile_step, ++local) {
      int64_t b, ti, tj, ks;
      const int g = decode_tile(a, BN, TR, tile, &b, &ti, &tj, &ks);
      const Segment& sg = a.seg[g];
      const uint32_t buf = (uint32_t)(local & 1);
      const uint32_t tphase = (uint32_t)((local >> 1) & 1);
      constexpr int kCh = BN / 64;  // 32-column chunks per warp (half a tile)
      // In-place update through the TMA (non-symmetric outputs): the C0 box
      // of a 32 x 32 chunk is loaded by the TMA into a staging buffer (the
      // layout of the store box), the finished chunk alpha acc + beta C0
      // replaces it there, and a bulk tensor store writes it back.  Up to
      // kStg - 1 chunks ahead are in flight (one with a single buffer); the
      // first ones are requested before the accumulator is waited for, so
      // that they load while the tile's MMAs run.  Loads and stores are
      // async bulk copies: no per-thread global access in the epilogue.
      const bool inplace = a.tma_out && a.c0_out;
      constexpr int kAhead = C::kStg > 1 ? C::kStg - 1 : 1;
      const int64_t ip_row = ti * TR + rank * kTileM + q * 32;
      const uint32_t ip_half = (uint32_t)((warp - 2) >> 2);
      float* const ip_stg = epi_smem + (warp - 2) * (C::kStg * 32 * 32);
      uint64_t* const ip_bars = c0bar + (warp - 2) * C::kStg;
      const int32_t ip_z = (int32_t)(sg.b0 + b);
      const uint32_t ip_box = a.has_bf16 ? 2048u : 4096u;
      const uint32_t ip_base = nstores;  // chunk c stages in buffer (ip_base + c) % kStg
      int nch = 0;  // chunks of this warp inside the output
      if (inplace) {
        for (int c = 0; c < kCh; ++c)
          if (ip_row < sg.M && tj * BN + ip_half * (BN / 2) + c * 32 < sg.N) nch = c + 1;
      }
      auto c0_issue = [&](int c) {  // lane 0
        const uint32_t sb = (ip_base + (uint32_t)c) & (C::kStg - 1);
        ptx::mbar_arrive_expect_tx(&ip_bars[sb], ip_box);
        ptx::tma_load_3d(ip_stg + sb * (32 * 32), &sg.tmC, &ip_bars[sb],
                         (int32_t)(tj * BN + ip_half * (BN / 2) + c * 32), (int32_t)ip_row, ip_z);
        c0pend |= 1u << sb;
      };
      // loads in flight land before the CTA's shared memory goes away
      auto c0_drain = [&]() {
        if (lane == 0)
          for (int i = 0; i < C::kStg; ++i)
            if ((c0pend >> i) & 1u)
              ptx::mbar_wait_timed(&ip_bars[i], (c0ph >> i) & 1u, 100000000ull);
      };
      if (inplace && nch > 0 && lane == 0) {
        ptx::bulk_wait_read0();  // earlier stores have read their buffers
        for (int c = 0; c < nch && c < kAhead; ++c) c0_issue(c);
      }
      // one lane polls the barrier; the warp follows through __syncwarp
      int ok = 1;
      if (lane == 0) ok = ptx::mbar_wait(&tfull[buf], tphase, abort_flag) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) {
        if (lane == 0) {
          *abort_flag = 1;
          report_status(a.status, OUO_STATUS_TIMEOUT);
        }
        c0_drain();
        break;
      }
      ptx::tc_fence_after();
      if (inplace) {
        const bool obf = a.has_bf16 != 0;
        const float alpha = a.has_dalpha ? a.dalpha[sg.dbase + b] : a.alpha;
        bool ok_c0 = true;
#pragma unroll 1
        for (int c = 0; c < nch; ++c) {
          const uint32_t sb = (ip_base + (uint32_t)c) & (C::kStg - 1);
          const uint32_t ph = (c0ph >> sb) & 1u;
          float* stg = ip_stg + sb * (32 * 32);
          uint16_t* stg16 = reinterpret_cast<uint16_t*>(stg);
          const int64_t gj0 = tj * BN + ip_half * (BN / 2) + c * 32;
          float v[32];
          ptx::tmem_ld32(tmem_base + ((q * 32u) << 16) + buf * BN + ip_half * (BN / 2) + c * 32, v);
          // C0 of this chunk has landed
          int okw = 1;
          if (lane == 0) okw = ptx::mbar_wait(&ip_bars[sb], ph, abort_flag) ? 1 : 0;
          okw = __shfl_sync(0xffffffffu, okw, 0);
          if (!okw) {
            if (lane == 0) {
              *abort_flag = 1;
              report_status(a.status, OUO_STATUS_TIMEOUT);
            }
            ok_c0 = false;
            break;
          }
          c0ph ^= 1u << sb;
          c0pend &= ~(1u << sb);
          if (!obf) {
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
              float4* pp = reinterpret_cast<float4*>(stg + stg_idx(lane, j));
              const float4 e = *pp;
              *pp = make_float4(alpha * v[j] + a.beta * e.x, alpha * v[j + 1] + a.beta * e.y,
                                alpha * v[j + 2] + a.beta * e.z, alpha * v[j + 3] + a.beta * e.w);
            }
          } else {
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
              uint4* pp = reinterpret_cast<uint4*>(stg16 + stg16_idx(lane, 8 * qq));
              const uint4 e = *pp;
              const uint32_t ew[4] = {e.x, e.y, e.z, e.w};
              uint32_t ow[4];
#pragma unroll
              for (int h = 0; h < 4; ++h) {
                const float lo = __uint_as_float(ew[h] << 16), hi = __uint_as_float(ew[h] & 0xffff0000u);
                ow[h] = pack_bf16x2(alpha * v[8 * qq + 2 * h] + a.beta * lo,
                                    alpha * v[8 * qq + 2 * h + 1] + a.beta * hi);
              }
              *pp = make_uint4(ow[0], ow[1], ow[2], ow[3]);
            }
          }
          ptx::fence_async_shared();
          __syncwarp();
          if (lane == 0) {
            ptx::tma_store_3d(&sg.tmC, stg, (int32_t)gj0, (int32_t)ip_row, ip_z);
            ptx::bulk_commit();
            // the next load reuses the buffer of chunk c + kAhead - kStg,
            // whose store must have finished reading it
            if (c + kAhead < nch) {
              if (C::kStg == 1) ptx::bulk_wait_read0();
              else ptx::bulk_wait_read1();
              c0_issue(c + kAhead);
            }
          }
          ++nstores;
        }
        if (!ok_c0) {
          c0_drain();
          break;
        }
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (CG == 2) ptx::mbar_arrive_cluster(tempty_lead + buf * 8u);
          else ptx::mbar_arrive(&tempty[buf]);
        }
        continue;
      }
      if (a.tma_out) {
        // Finished values (row = lane) are staged in the TMA's swizzled box
        // layout (fp32: 128-byte rows, 16-byte chunks XOR row % 8; bf16:
        // 64-byte rows, chunks XOR (row / 2) % 4) and written by one lane
        // with a bulk tensor store; rows and columns past the matrix are
        // clipped by the TMA.  Symmetric outputs: the mirrored box (j, i)
        // is a second store from a transposed staging; a chunk on the
        // diagonal is made symmetric in place and stored once.
        const int64_t row_base = ti * TR + rank * kTileM + q * 32;
        const int64_t gi = row_base + lane;
        float* const stg_base = epi_smem + (warp - 2) * (C::kStg * 32 * 32);
        float* stg = stg_base;
        uint16_t* stg16 = reinterpret_cast<uint16_t*>(stg);
        // Stores rotate over the warp's staging buffers; before a buffer is
        // refilled, the store that last read it must have finished reading
        // (with two buffers that is every store but the latest one).
        auto next_stg = [&]() {
          if (C::kStg == 2) {
            if (lane == 0) ptx::bulk_wait_read1();
            stg = stg_base + (nstores & 1u) * (32 * 32);
          } else {
            if (lane == 0) ptx::bulk_wait_read0();
          }
          stg16 = reinterpret_cast<uint16_t*>(stg);
          __syncwarp();
        };
        const uint32_t half = (uint32_t)((warp - 2) >> 2);
        const int32_t z = (int32_t)((sg.b0 + b) * sg.ksplit + ks);
        const bool obf = a.has_bf16 != 0;
#pragma unroll 1
        for (uint32_t c0 = half * (BN / 2); c0 < (half + 1) * (BN / 2); c0 += 32) {
          const int64_t gj0 = tj * BN + c0;
          if (a.tri && gj0 + 31 < row_base) continue;  // below the diagonal
          if (row_base >= sg.M || gj0 >= sg.N) continue;
          float v[32];
          ptx::tmem_ld32(tmem_base + ((q * 32u) << 16) + buf * BN + c0, v);
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] *= a.alpha;
          if (a.has_c0) {
            float c0v[32];
            if (a.tri && !a.c0_upper) {
              const int64_t gic = gi < sg.M ? gi : sg.M - 1;
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                const int64_t gjc = gj0 + j < sg.N ? gj0 + j : sg.N - 1;
                c0v[j] = load_c0(sg, b, gjc, gic, a.c0_bf16);
              }
            } else if (gi < sg.M && gj0 + 32 <= sg.N) {
#pragma unroll
              for (int j = 0; j < 32; j += 4) load_c0x4(sg, b, gi, gj0 + j, c0v + j, a.c0_bf16);
            } else {
              const int64_t gic = gi < sg.M ? gi : sg.M - 1;
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                const int64_t gjc = gj0 + j < sg.N ? gj0 + j : sg.N - 1;
                c0v[j] = load_c0(sg, b, gic, gjc, a.c0_bf16);
              }
            }
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] += a.beta * c0v[j];
          }
          if (gi >= gj0 && gi < gj0 + 32) {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (gi == gj0 + j) v[j] += a.gamma;
          }
          if (a.round_tf32 && !obf) {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = round_tf32(v[j]);
          }
          const bool diag = a.tri && gj0 == row_base;
          next_stg();
          if (!obf) {
#pragma unroll
            for (int j = 0; j < 32; j += 4)
              *reinterpret_cast<float4*>(stg + stg_idx(lane, j)) =
                  make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
          } else {
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
              uint4 u;
              u.x = pack_bf16x2(v[8 * qq + 0], v[8 * qq + 1]);
              u.y = pack_bf16x2(v[8 * qq + 2], v[8 * qq + 3]);
              u.z = pack_bf16x2(v[8 * qq + 4], v[8 * qq + 5]);
              u.w = pack_bf16x2(v[8 * qq + 6], v[8 * qq + 7]);
              *reinterpret_cast<uint4*>(stg16 + stg16_idx(lane, 8 * qq)) = u;
            }
          }
          if (diag) {
            // lower triangle of the chunk := its upper triangle, transposed
            __syncwarp();
            for (int j = 0; j < lane; ++j) {
              if (!obf) stg[stg_idx(lane, j)] = stg[stg_idx(j, lane)];
              else stg16[stg16_idx(lane, j)] = stg16[stg16_idx(j, lane)];
            }
          }
          ptx::fence_async_shared();
          __syncwarp();
          if (lane == 0) {
            ptx::tma_store_3d(&sg.tmC, stg, (int32_t)gj0, (int32_t)row_base, z);
            ptx::bulk_commit();
          }
          ++nstores;
          // upper-stored outputs: only tiles on the block diagonal mirror
          if (a.tri && !diag && !(a.sym_half && tj != ti)) {
            next_stg();
            if (!obf) {
#pragma unroll
              for (int j = 0; j < 32; ++j) stg[stg_idx(j, lane)] = v[j];
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j) stg16[stg16_idx(j, lane)] = f32_to_bf16(v[j]);
            }
            ptx::fence_async_shared();
            __syncwarp();
            if (lane == 0) {
              ptx::tma_store_3d(&sg.tmC, stg, (int32_t)row_base, (int32_t)gj0, z);
              ptx::bulk_commit();
            }
            ++nstores;
          }
        }
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (CG == 2) ptx::mbar_arrive_cluster(tempty_lead + buf * 8u);
          else ptx::mbar_arrive(&tempty[buf]);
        }
        continue;
      }
      // Direct (or dual) outputs, symmetric or not.
      // This warp owns tile rows q*32 .. q*32+31 (TMEM lanes) and one half
      // of the columns; each chunk is 32 rows x 32 columns.  Values are
      // finished with row = lane (where the symmetric C0 read (j, i) is
      // coalesced), staged in shared memory, and written back with 16-byte
      // stores: 8 lanes per 128-byte row, 4 rows per instruction, for the
      // direct tile (i, j) and, for symmetric outputs, the mirrored tile
      // (j, i).  Chunks entirely below the diagonal of a symmetric output
      // are skipped; chunks fully inside and above it store without masks.
      const int64_t row_base = ti * TR + rank * kTileM + q * 32;
      const int64_t gi = row_base + lane;
      float* stg = epi_smem + (warp - 2) * (C::kStg * 32 * 32);
      const int sub_r = lane >> 3, sub_c = 4 * (lane & 7);
      const TileOut to = tile_out(a, sg, b);
      const uint32_t half = (uint32_t)((warp - 2) >> 2);
#pragma unroll 1
      for (uint32_t c0 = half * (BN / 2); c0 < (half + 1) * (BN / 2); c0 += 32) {
        const int64_t gj0 = tj * BN + c0;
        if (a.tri && gj0 + 31 < row_base) continue;  // below the diagonal
        if (row_base >= sg.M || gj0 >= sg.N) continue;  // outside the output
        const bool full_chunk = row_base + 32 <= sg.M && gj0 + 32 <= sg.N &&
                                (!a.tri || gj0 >= row_base + 31);
        float v[32];
        ptx::tmem_ld32(tmem_base + ((q * 32u) << 16) + buf * BN + c0, v);
        if (a.tri) {
          if (a.has_c0) {
            // 32 independent loads (clamped into the matrix, so they can be
            // issued together), used only where the element is kept; an
            // upper-stored C0 is read at (i, j), otherwise at (j, i)
            const int64_t gic = gi < sg.M ? gi : sg.M - 1;
            float c0v[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int64_t gjc = gj0 + j < sg.N ? gj0 + j : sg.N - 1;
              c0v[j] = a.c0_upper ? load_c0(sg, b, gic, gjc, a.c0_bf16)
                                  : load_c0(sg, b, gjc, gic, a.c0_bf16);
            }
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = a.alpha * v[j] + a.beta * c0v[j];
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] *= a.alpha;
          }
          if (gi >= gj0 && gi < gj0 + 32) {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (gi == gj0 + j) v[j] += a.gamma;
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
              if (gr < sg.M && gc + t < sg.N && (!a.tri || gc + t >= gr)) mask |= 1u << t;
          }
          if (!a.tri && mask) {
            if (a.has_c0) {
              float e[4];
              if (a.c0_out) {
                if (mask == 0xFu) {
                  load_out4(a, to, gr, gc, e);
                } else {
#pragma unroll
                  for (int t = 0; t < 4; ++t)
                    e[t] = (mask & (1u << t)) ? load_out1(a, to, gr, gc + t) : 0.f;
                }
              } else if (mask == 0xFu) {
                load_c0x4(sg, b, gr, gc, e, a.c0_bf16);
              } else {
#pragma unroll
                for (int t = 0; t < 4; ++t)
                  e[t] = (mask & (1u << t)) ? load_c0(sg, b, gr, gc + t, a.c0_bf16) : 0.f;
              }
              w.x += a.beta * e[0];
              w.y += a.beta * e[1];
              w.z += a.beta * e[2];
              w.w += a.beta * e[3];
            }
            if (a.gamma != 0.f && gr >= gc && gr < gc + 4) {
              if (gr == gc) w.x += a.gamma;
              if (gr == gc + 1) w.y += a.gamma;
              if (gr == gc + 2) w.z += a.gamma;
              if (gr == gc + 3) w.w += a.gamma;
            }
          }
          if (mask) store4t(a, to, gr, gc, w, mask);
        }
        __syncwarp();
        if (a.tri && !(a.sym_half && tj != ti)) {
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
                if (dst_c + t < sg.M && dst_r < sg.N && dst_r >= dst_c + t) mask |= 1u << t;
            }
            if (mask) store4t(a, to, dst_r, dst_c, w, mask);
          }
          __syncwarp();
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (CG == 2) ptx::mbar_arrive_cluster(tempty_lead + buf * 8u);
        else ptx::mbar_arrive(&tempty[buf]);
      }
    }
    // bulk stores complete before the CTA (and its shared memory) goes away
    if (lane == 0) ptx::bulk_wait0();
    __syncwarp();
  }
  __syncthreads();
  // a pair frees TMEM only after the even CTA's MMAs (which write both
  // CTAs' TMEM) and both CTAs' epilogues (which signal the even CTA) are done
  if (CG == 2) {
    __syncwarp();
    ptx::cluster_sync();
  }
  if (warp == 1) {
    ptx::tc_fence_after();
    if (CG == 2) ptx::tmem_dealloc2(tmem_base, C::kTmemCols);
    else ptx::tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// ------------------------------------------------------------------- host

// ------------------------------------------------ per-launch timing (opt-in)
// While enabled, every launch of the tensor-core GEMM is bracketed by two
// CUDA events on its stream and its algorithmic flops (symmetric outputs:
// the upper triangle only) are recorded per kernel kind.  Events come from a
// pool created when timing is switched on.
// kinds: (tri ? 4 : 0) + (tf32 ? 2 : 0) + b_mn
constexpr int kTimingMax = 4096;
struct TimingRec {
  cudaEvent_t e0, e1;
  int kind;
  double flops;
};
std::mutex g_tmu;
bool g_timing = false;
std::vector<TimingRec> g_recs;
std::vector<cudaEvent_t> g_pool;
size_t g_next = 0;

int timing_record_begin(cudaStream_t s, TimingRec* r) {
  if (g_next + 2 > g_pool.size()) return 0;
  r->e0 = g_pool[g_next++];
  r->e1 = g_pool[g_next++];
  cudaEventRecord(r->e0, s);
  return 1;
}

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
// (box_cols, box_rows, 1), 128-byte swizzle (16-byte atoms, or 32-byte
// atoms for MN-major tf32 operands), zero fill out of bounds.
int make_map(CUtensorMap* map, const Buf& t, uint32_t box_cols,
             uint32_t box_rows,
             CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
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
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return set_error(OUO_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return OUO_OK;
}

// 4-D map of an MN-major operand whose columns split into whole chunks:
// dims (chunk columns, rows, chunk index, matrix), the chunk index striding
// by one chunk's bytes.  A box of `nchunks` chunks is one TMA load that
// fills consecutive chunk tiles in shared memory.
int make_map4(CUtensorMap* map, const Buf& t, uint32_t chunk_cols, uint32_t box_rows,
              uint32_t nchunks, CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = encode_fn();
  if (!fn)
    return set_error(OUO_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  const size_t es = elem_size(t.dtype);
  cuuint64_t dims[4] = {(cuuint64_t)chunk_cols, (cuuint64_t)t.rows,
                        (cuuint64_t)(t.cols / chunk_cols), (cuuint64_t)t.nb};
  cuuint64_t strides[3] = {(cuuint64_t)(t.ld * es), (cuuint64_t)(chunk_cols * es),
                           (cuuint64_t)(t.stride * es)};
  cuuint32_t box[4] = {chunk_cols, box_rows, nchunks, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map,
                  t.dtype == OUO_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                      : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                  4, t.p, dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return set_error(OUO_ERR_CUDA, "cuTensorMapEncodeTiled (4-D) failed (%d)", (int)r);
  return OUO_OK;
}

int64_t tiles_per_matrix(const GemmDesc& g, int BN, int TR) {
  const int64_t tm = ceil_div(g.M, (int64_t)TR), tn = ceil_div(g.N, BN);
  if (!g.tri) return tm * tn;
  int64_t cnt = 0;
  for (int64_t i = 0; i < tm; ++i) cnt += tn - tri_jmin(i, BN, TR);
  return cnt;
}

// Launch configuration of one kernel instance; CTA pairs are clusters of 2.
cudaLaunchConfig_t launch_cfg(unsigned grid, size_t smem, cudaStream_t stream,
                              int cg, cudaLaunchAttribute* attr) {
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)cg;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cfg;
}

template <int BN, int FMT, int B_MN, int CG, int UPD = 0>
int launch(const std::vector<GemmDesc>& gs, cudaStream_t stream, int* status) {
  using C = Cfg<BN, CG, UPD>;
  constexpr int TR = (int)C::kTileRows;
  constexpr uint32_t es = FMT == 1 ? 2 : 4;
  constexpr uint32_t bk = kRowBytes / es;
  auto kern = umma_gemm_kernel<BN, FMT, B_MN, CG, UPD>;
  // per device: shared-memory opt-in done, and how many CTAs (pairs: CTA
  // pairs) of this kernel can be resident at once -- a persistent grid
  // larger than that would run its last CTAs after the others finish
  static std::mutex setup_mu;
  static int resident[64] = {0};  // 0: not yet set up on that device
  int dev = 0;
  OUO_CHECK_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64)
    return set_error(OUO_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  int cap_slots = 0;
  {
  std::lock_guard<std::mutex> setup_lock(setup_mu);
  if (!resident[dev]) {
    OUO_CHECK_CUDA(cudaFuncSetAttribute(
        kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::kSmem));
    int n = num_sms();
    if (CG == 2) {
      cudaLaunchAttribute attr[1];
      cudaLaunchConfig_t cfg = launch_cfg(
          (unsigned)(2 * num_sms()), C::kSmem, stream, CG, attr);
      int clusters = 0;
      OUO_CHECK_CUDA(cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg));
      if (clusters < 1)
        return set_error(OUO_ERR_UNSUPPORTED, "no CTA pair of the GEMM kernel fits on this device");
      n = clusters;
    }
    resident[dev] = n;
  }
  cap_slots = resident[dev];
  }
  const GemmDesc& g0 = gs[0];
  UmmaArgs a;
  memset(&a, 0, sizeof(a));
  a.tri = g0.tri;
  a.alpha = g0.alpha; a.beta = g0.beta; a.gamma = g0.gamma;
  a.has_c0 = g0.has_c0;
  a.c0_bf16 = g0.has_c0 && g0.C0.dtype == OUO_BF16;
  a.has_f32 = g0.has_f32; a.round_tf32 = g0.round_tf32;
  a.has_bf16 = g0.has_bf16;
  a.status = status;
  a.has_dalpha = !g0.direct_alpha.empty() ? 1 : 0;
  if (!g0.direct.empty()) {
    a.has_f32 = g0.direct_dtype == OUO_F32;
    a.has_bf16 = g0.direct_dtype == OUO_BF16;
    a.round_tf32 = 0;
    a.c0_out = g0.c0_from_out ? 1 : 0;
    if (a.c0_out) a.has_c0 = 1;
  }
  // single workspace output: TMA-store epilogue
  a.tma_out = (g0.direct.empty() && (g0.has_f32 != g0.has_bf16)) ? 1 : 0;
  // in-place update through the TMA: C0 is the output matrix itself
  if (a.tma_out && g0.c0_from_out) {
    a.c0_out = 1;
    a.has_c0 = 1;
  }
  a.a_sym = g0.a_sym; a.b_sym = g0.b_sym;
  a.c0_upper = g0.c0_upper; a.sym_half = g0.sym_half;
  if ((a.a_sym || a.b_sym) && !(CG == 2 && FMT == 2 && !B_MN))
    return set_error(OUO_ERR_INVALID_ARG, "upper-stored operands need tf32 K-major pair tiles");
  if ((a.sym_half || a.c0_upper) && CG != 2)
    return set_error(OUO_ERR_INVALID_ARG, "upper-stored symmetric outputs need pair tiles");
  int ndirect = 0;
  auto flush = [&]() -> int {
    if (a.nseg == 0) return OUO_OK;
    a.total_tiles = 0;
    for (int s = 0; s < a.nseg; ++s) {
      a.seg[s].tile_start = a.total_tiles;
      a.total_tiles += a.seg[s].tiles_per_mat * a.seg[s].nb;
    }
    // one CTA (or CTA pair) per resident slot, at most one per tile
    const int64_t slots = a.total_tiles < cap_slots ? a.total_tiles : cap_slots;
    if (slots >= 1) {
      TimingRec rec;
      bool timed = false;
      if (g_timing) {
        std::lock_guard<std::mutex> lock(g_tmu);
        timed = timing_record_begin(stream, &rec) != 0;
      }
      if (CG == 1) {
        kern<<<(unsigned)slots, kThreads, C::kSmem, stream>>>(a);
      } else {
        cudaLaunchAttribute attr[1];
        cudaLaunchConfig_t cfg = launch_cfg(
            (unsigned)(CG * slots), C::kSmem, stream, CG, attr);
        OUO_CHECK_CUDA(cudaLaunchKernelEx(&cfg, kern, a));
      }
      OUO_CHECK_LAUNCH();
      if (timed) {
        cudaEventRecord(rec.e1, stream);
        rec.kind = (a.tri ? 4 : 0) + (FMT == 2 ? 2 : 0) + B_MN;
        rec.flops = 0.0;
        for (int sgi = 0; sgi < a.nseg; ++sgi) {
          const Segment& sg = a.seg[sgi];
          const double per = a.tri ? (double)sg.M * (double)(sg.M + 1) * (double)sg.K
                                   : 2.0 * (double)sg.M * (double)sg.N * (double)sg.K;
          rec.flops += per * (double)sg.nb * (double)sg.npass;
        }
        std::lock_guard<std::mutex> lock(g_tmu);
        g_recs.push_back(rec);
      }
    }
    a.nseg = 0;
    ndirect = 0;
    return OUO_OK;
  };
  for (const GemmDesc& g : gs) {
    if (g.M < 1 || g.N < 1 || g.K < 1 || g.nb < 1) continue;
    Segment proto;
    memset(&proto, 0, sizeof(proto));
    OUO_TRY(make_map(&proto.tmA, g.A, bk, kTileM));
    const CUtensorMapSwizzle mn_swz =
        FMT == 2 ? CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B : CU_TENSOR_MAP_SWIZZLE_128B;
    // one 4-D load per stage when the columns split into whole chunks (a
    // partial last chunk would be zero-filled whole by the chunk dimension)
    // (OUO_TMA_4D=0 keeps the per-chunk loads)
    const char* env4 = getenv("OUO_TMA_4D");
    const bool b4d = B_MN && CG == 1 && g.N % (kRowBytes / es) == 0 &&
                     !(env4 && env4[0] == '0');
    auto make_b = [&](CUtensorMap* m, const Buf& b) -> int {
      if (!B_MN) return make_map(m, b, bk, C::kBRows);
      if (b4d) return make_map4(m, b, kRowBytes / es, bk, C::kBRows / (kRowBytes / es), mn_swz);
      return make_map(m, b, kRowBytes / es, bk, mn_swz);
    };
    OUO_TRY(make_b(&proto.tmB, g.B));
    CUtensorMap lo_a, lo_b, lo_a3;
    memset(&lo_a, 0, sizeof(lo_a));
    memset(&lo_b, 0, sizeof(lo_b));
    memset(&lo_a3, 0, sizeof(lo_a3));
    proto.npass = g.npass < 1 ? 1 : g.npass;
    if (proto.npass > 1) {
      if (FMT != 2 || proto.npass > 3 || g.a_sym || g.b_sym)
        return set_error(OUO_ERR_INVALID_ARG, "split-tf32 passes: tf32, 2 or 3 passes, "
                                              "no upper-stored operands");
      proto.a_lo = g.a_lo & ((1 << proto.npass) - 1);
      proto.a_lo2 = g.a_lo2 & ((1 << proto.npass) - 1) & ~proto.a_lo;
      proto.b_lo = g.b_lo & ((1 << proto.npass) - 1);
      if (proto.a_lo) OUO_TRY(make_map(&lo_a, g.A2, bk, kTileM));
      if (proto.a_lo2) OUO_TRY(make_map(&lo_a3, g.A3, bk, kTileM));
      if (proto.b_lo) OUO_TRY(make_b(&lo_b, g.B2));
    }
    proto.M = g.M; proto.N = g.N; proto.K = g.K;
    proto.b4d = b4d ? 1 : 0;
    if (g.a_sym || g.b_sym) {
      // the same matrices read transposed, as 32-column MN-major chunks
      constexpr uint32_t cc = kRowBytes / 4;  // tf32 chunk columns
      proto.t4d = g.K % cc == 0 ? 1 : 0;
      const Buf* ops[2] = {&g.A, &g.B};
      CUtensorMap* maps[2] = {&proto.tmAt, &proto.tmBt};
      const bool want[2] = {g.a_sym, g.b_sym};
      for (int q = 0; q < 2; ++q) {
        if (!want[q]) continue;
        if (proto.t4d) OUO_TRY(make_map4(maps[q], *ops[q], cc, bk, kTileM / cc, mn_swz));
        else OUO_TRY(make_map(maps[q], *ops[q], cc, bk, mn_swz));
      }
    }
    proto.tiles_n = ceil_div(g.N, BN);
    proto.tiles_2d = tiles_per_matrix(g, BN, TR);
    {
      const int64_t nk = ceil_div(g.K, (int64_t)bk) * proto.npass;
      int64_t ksp = g.ksplit < 1 ? 1 : g.ksplit;
      if (ksp > nk) ksp = nk;
      proto.kbc = ceil_div(nk, ksp);
      proto.ksplit = (int)ceil_div(nk, proto.kbc);  // every range non-empty
    }
    proto.tiles_per_mat = proto.tiles_2d * proto.ksplit;
    proto.C0 = (g.has_c0 && !g.c0_from_out) ? g.C0.p : nullptr;
    proto.ldc0 = g.C0.ld; proto.sc0 = g.C0.stride;
    proto.Of = g.has_f32 ? reinterpret_cast<float*>(g.out_f32.p) : nullptr;
    proto.ldof = g.out_f32.ld; proto.sof = g.out_f32.stride;
    proto.Ob = g.has_bf16 ? reinterpret_cast<uint16_t*>(g.out_bf16.p) : nullptr;
    proto.ldob = g.out_bf16.ld; proto.sob = g.out_bf16.stride;
    proto.direct = g.direct.empty() ? 0 : 1;
    if (a.tma_out) {
      const Buf& ob = g.has_f32 ? g.out_f32 : g.out_bf16;
      OUO_TRY(make_map(&proto.tmC, ob, 32, 32,
                       g.has_f32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B));
    }
    int64_t b0 = 0;
    while (b0 < g.nb) {
      const bool tabled = proto.direct || a.has_dalpha;  // per-matrix table slots
      if (a.nseg == kMaxSeg || (tabled && ndirect == kChunk)) OUO_TRY(flush());
      int64_t nb = g.nb - b0;
      if (tabled && nb > kChunk - ndirect) nb = kChunk - ndirect;
      a.lo_map[a.nseg][0] = lo_a;
      a.lo_map[a.nseg][1] = lo_b;
      a.lo_map[a.nseg][2] = lo_a3;
      Segment& sg = a.seg[a.nseg++];
      sg = proto;
      sg.b0 = b0;
      sg.nb = nb;
      if (tabled) {
        sg.dbase = ndirect;
        for (int64_t i = 0; i < nb; ++i) {
          a.dptr[ndirect + i] = proto.direct ? g.direct[b0 + i].p : nullptr;
          a.dld[ndirect + i] = proto.direct ? g.direct[b0 + i].ld : 0;
          a.dalpha[ndirect + i] = a.has_dalpha ? g.direct_alpha[b0 + i] : g.alpha;
        }
        ndirect += (int)nb;
      }
      b0 += nb;
    }
  }
  return flush();
}

}  // namespace

int gemm_timing_enable(int on) {
  std::lock_guard<std::mutex> lock(g_tmu);
  for (cudaEvent_t e : g_pool) cudaEventDestroy(e);
  g_pool.clear();
  g_recs.clear();
  g_next = 0;
  g_timing = false;
  if (!on) return OUO_OK;
  for (int i = 0; i < 2 * kTimingMax; ++i) {
    cudaEvent_t e;
    OUO_CHECK_CUDA(cudaEventCreate(&e));
    g_pool.push_back(e);
  }
  g_timing = true;
  return OUO_OK;
}

int gemm_timing_read(int kind, int* launches, double* total_ms, double* flops) {
  std::lock_guard<std::mutex> lock(g_tmu);
  int n = 0;
  double ms = 0.0, fl = 0.0;
  for (const TimingRec& r : g_recs) {
    if (kind >= 0 && r.kind != kind) continue;
    OUO_CHECK_CUDA(cudaEventSynchronize(r.e1));
    float t = 0.f;
    OUO_CHECK_CUDA(cudaEventElapsedTime(&t, r.e0, r.e1));
    ++n;
    ms += t;
    fl += r.flops;
  }
  if (launches) *launches = n;
  if (total_ms) *total_ms = ms;
  if (flops) *flops = fl;
  return OUO_OK;
}

int gemm_ksplit_used(int64_t K, int ksplit, int dtype, int npass) {
  const int64_t bk = kRowBytes / (dtype == OUO_BF16 ? 2 : 4);
  const int64_t nk = ceil_div(K, bk) * (npass < 1 ? 1 : npass);
  int64_t ksp = ksplit < 1 ? 1 : ksplit;
  if (ksp > nk) ksp = nk;
  const int64_t kbc = ceil_div(nk, ksp);
  return (int)ceil_div(nk, kbc);
}

int cta_pair_mode() {
  const char* env = getenv("OUO_CTA_PAIR");
  return env && env[0] >= '0' && env[0] <= '2' ? env[0] - '0' : 1;
}

bool cta_pairs_enabled() { return cta_pair_mode() > 0; }

// One launch kind: operand type, B majorness, CTA pairs, tile width.
int launch_kind(const std::vector<GemmDesc>& gs, bool pair, bool wide, cudaStream_t stream,
                int* status) {
  const GemmDesc& g0 = gs[0];
  // in-place updates through the TMA (one output matrix, C0 = itself)
  const bool upd = g0.c0_from_out && g0.direct.empty() && g0.has_f32 != g0.has_bf16;
  if (g0.A.dtype == OUO_BF16) {
    if (g0.b_mn) {
      if (pair && upd) return launch<256, 1, 1, 2, 1>(gs, stream, status);
      if (pair) return launch<256, 1, 1, 2>(gs, stream, status);
      return wide ? launch<256, 1, 1, 1>(gs, stream, status) : launch<128, 1, 1, 1>(gs, stream, status);
    }
    if (pair) return launch<256, 1, 0, 2>(gs, stream, status);
    return wide ? launch<256, 1, 0, 1>(gs, stream, status) : launch<128, 1, 0, 1>(gs, stream, status);
  }
  if (g0.b_mn) {
    if (pair && upd) return launch<256, 2, 1, 2, 1>(gs, stream, status);
    if (pair) return launch<256, 2, 1, 2>(gs, stream, status);
    return wide ? launch<256, 2, 1, 1>(gs, stream, status) : launch<128, 2, 1, 1>(gs, stream, status);
  }
  if (pair) return launch<256, 2, 0, 2>(gs, stream, status);
  return wide ? launch<256, 2, 0, 1>(gs, stream, status) : launch<128, 2, 0, 1>(gs, stream, status);
}

int gemm_umma_grouped(const std::vector<GemmDesc>& gs, cudaStream_t stream,
                      int* status) {
  if (gs.empty()) return OUO_OK;
  const GemmDesc& g0 = gs[0];
  bool wide = false, tall = false, per_desc = false;
  for (const GemmDesc& g : gs) {
    if (g.A.dtype != g.B.dtype || g.A.dtype != g0.A.dtype)
      return set_error(OUO_ERR_UNSUPPORTED, "tensor-core GEMM needs equal operand types");
    if (g.tri != g0.tri || g.b_mn != g0.b_mn || g.has_c0 != g0.has_c0 ||
        g.has_f32 != g0.has_f32 || g.has_bf16 != g0.has_bf16 ||
        g.round_tf32 != g0.round_tf32 || g.direct.empty() != g0.direct.empty() ||
        g.c0_from_out != g0.c0_from_out || g.sym_half != g0.sym_half ||
        g.a_sym != g0.a_sym || g.b_sym != g0.b_sym || g.c0_upper != g0.c0_upper ||
        (g.alpha != g0.alpha && g0.direct_alpha.empty()) || g.beta != g0.beta ||
        g.gamma != g0.gamma || g.direct_alpha.empty() != g0.direct_alpha.empty() ||
        (g.has_c0 && g.C0.dtype != g0.C0.dtype) ||
        (!g.direct.empty() && g.direct_dtype != g0.direct_dtype))
      return set_error(OUO_ERR_INVALID_ARG, "grouped GEMM descriptors differ");
    if (g.tri && (g.M != g.N || g.b_mn))
      return set_error(OUO_ERR_INVALID_ARG, "symmetric GEMM needs M == N, K-major B");
    if (!g.direct.empty() && (int64_t)g.direct.size() != g.nb)
      return set_error(OUO_ERR_INVALID_ARG, "direct output table size mismatch");
    if (g.c0_from_out && (g.tri || (g.direct.empty() && g.has_f32 == g.has_bf16)))
      return set_error(OUO_ERR_INVALID_ARG,
                       "in-place C0 needs non-symmetric direct outputs or one output matrix");
    if (!g.direct_alpha.empty() && (int64_t)g.direct_alpha.size() != g.nb)
      return set_error(OUO_ERR_INVALID_ARG, "direct alpha table size mismatch");
    if (g.ksplit > 1 && (g.tri || !g.direct.empty() || g.has_c0 || g.has_f32 == g.has_bf16))
      return set_error(OUO_ERR_INVALID_ARG,
                       "split-K needs one workspace output, no C0, non-symmetric");
    wide = wide || g.N > 128;
    tall = tall || g.M > 128;
    per_desc = per_desc || g.per_desc_tiles;
  }
  // CTA pairs (256 x 256 tiles) for wide outputs with more than 128 rows and
  // K-major B.  OUO_CTA_PAIR=0 selects single-CTA 128 x BN tiles throughout;
  // OUO_CTA_PAIR=2 also puts MN-major B (Q X) on pairs.
  const int pair_mode = cta_pair_mode();
  auto pair_of = [&](bool w, bool t, bool mn_ok) {
    return w && t && pair_mode > 0 && (!g0.b_mn || pair_mode == 2 || mn_ok);
  };
  if (!per_desc) return launch_kind(gs, pair_of(wide, tall, false), wide, stream, status);
  // every descriptor keeps its own tile shape: one launch per shape in use
  for (int kind = 0; kind < 3; ++kind) {
    std::vector<GemmDesc> part;
    for (const GemmDesc& g : gs) {
      const bool w = g.N > 128, pr = pair_of(w, g.M > 128, g.pair_mn);
      const int k = pr ? 2 : (w ? 1 : 0);
      if (k == kind) part.push_back(g);
    }
    if (!part.empty()) OUO_TRY(launch_kind(part, kind == 2, kind >= 1, stream, status));
  }
  return OUO_OK;
}

int gemm_umma(const GemmDesc& g, cudaStream_t stream, int* status) {
  return gemm_umma_grouped(std::vector<GemmDesc>{g}, stream, status);
}

}  // namespace ouo
