// Dion / Orth-Dion low-rank step, batched across the matrices of a call.
//
// Source: "Orth-Dion: Eliminating Geometric Mismatch in Distributed Low-Rank
// Spectral Optimization" -- Problem Statement (rank-r factors from a single
// power-iteration step per optimizer step), The Geometric Insight (Dion's
// column normalization of the right factor), Orth-Dion (QR of the right
// factor instead, same power iteration and residual buffer), Theoretical
// Contributions (error-feedback coefficient beta); "Dion: The Distributed
// Orthonormal Update Revolution Is Here", Technical details.
//
// Per matrix (B is the momentum buffer after B = M + G, m x n fp32; the
// state Qt is the right factor transposed, r x n):
//   Pt = Qt B^T                      (r x m)
//   Pt <- rows orthonormalized       (CholeskyQR2: P = orth(B Q_prev))
//   Rt = Pt B                        (r x n; R = B^T P)
//   Qt_new = rows of Rt normalized   (Dion)  or  rows orthonormalized (Orth-Dion)
//   M <- beta B - (beta - mu) P Rt   (residual buffer / error feedback)
//   W <- (1 - lr wd) W - lr s P Qt_new
//   state <- Qt_new
// Every stage is one batched launch over all matrices (or a few, for very
// large batches): the momentum pass; the two projections on the tensor
// cores (tf32 operands, fp32 accumulation), grouped by shape and split
// along K when a matrix alone has too few output tiles to fill the GPU; the
// CholeskyQR passes (Gram matrices, one Cholesky CTA per matrix, block
// triangular solves; cholqr.cu); the row reductions / column
// normalization; and the two in-place rank-r updates.  Per-matrix choices
// (split counts, Gram chunks, tile shapes) depend only on that matrix's
// shape and rank, so a batch computes what one call per matrix computes,
// bit for bit.
#include <cmath>
#include <cstdlib>
#include <map>
#include <tuple>

#include "internal.h"

namespace ouo {
namespace {

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

int64_t pitch4(int64_t n) { return ceil_div(n, 4) * 4; }
int pad32(int r) { return (int)(ceil_div(r, 32) * 32); }

// Split-K of a projection with an M x N fp32 output and depth K: only a
// matrix whose own output tiles cannot fill the GPU is split, into ranges
// of at least 1024 along K.  Depends on the shape alone.
int proj_ksplit(int64_t M, int64_t N, int64_t K) {
  const int64_t ctas = ceil_div(M, 128) * ceil_div(N, 256);
  if (ctas >= 64) return 1;
  int64_t ks = ceil_div(128, ctas);
  int64_t kmax = K / 1024;
  if (kmax < 1) kmax = 1;
  if (ks > kmax) ks = kmax;
  if (ks > 8) ks = 8;
  return gemm_ksplit_used(K, (int)ks, OUO_F32);
}

// Matrices of one (rows, cols, rank) in a call, with their workspace.
struct DGroup {
  int64_t m = 0, n = 0;
  int r = 0;
  std::vector<int> members;  // indices into the caller's batch
  int ks1 = 1, ks2 = 1;      // K splits of Pt = Qt B^T and Rt = Pt B
  Buf Pt, P, Rt, Qn;         // r x m, m x r, r x n, r x n per member
  Buf Pb, Rtb;               // bf16 copies of P and Rt (the M update's operands)
  Buf T;                     // r x max(m, n): the first CholeskyQR pass's output
  Buf kp1, kp2;              // split-K partials (the same memory)
  float* lo = nullptr;       // Gram residual operands (the same memory again)
  Buf S, Lb, Ld;             // r x r summed Gram; R x R factors
  float* Z = nullptr;        // L^-1 planes, cholqr_z_floats(r) per member
  float* gpart = nullptr;    // Gram partials, gstride floats per member
  int64_t gstride = 0;
  char* ctl = nullptr;       // cooperative Cholesky control (r > 256)
  size_t ctl_stride = 0;
};

Buf view(const Buf& b, int64_t first, int64_t nb) {
  Buf v = b;
  v.p = b.p ? b.p + (size_t)first * b.stride * elem_size(b.dtype) : nullptr;
  v.nb = nb;
  return v;
}

Buf take_bytes(Arena& ar, size_t bytes) {
  Buf b = ar.take(OUO_F32, 1, 1, (int64_t)ceil_div((int64_t)bytes, 4));
  return b;
}

std::vector<DGroup> plan(const ouo_mat* M, int nmat, const int* ranks, Arena& ar) {
  std::vector<DGroup> gs;
  std::map<std::tuple<int64_t, int64_t, int>, int> where;
  for (int i = 0; i < nmat; ++i) {
    auto key = std::make_tuple(M[i].rows, M[i].cols, ranks[i]);
    auto it = where.find(key);
    if (it == where.end()) {
      where[key] = (int)gs.size();
      DGroup g;
      g.m = M[i].rows;
      g.n = M[i].cols;
      g.r = ranks[i];
      gs.push_back(g);
      gs.back().members.push_back(i);
    } else {
      gs[it->second].members.push_back(i);
    }
  }
  for (DGroup& g : gs) {
    const int64_t nb = (int64_t)g.members.size();
    const int64_t m = g.m, n = g.n;
    const int r = g.r, R = pad32(r);
    g.ks1 = proj_ksplit(r, m, n);
    g.ks2 = proj_ksplit(r, n, m);
    g.Pt = ar.take(OUO_F32, nb, r, m);
    g.P = ar.take(OUO_F32, nb, m, r);
    g.Rt = ar.take(OUO_F32, nb, r, n);
    g.Qn = ar.take(OUO_F32, nb, r, n);
    g.Pb = ar.take(OUO_BF16, nb, m, r);
    g.Rtb = ar.take(OUO_BF16, nb, r, n);
    g.T = ar.take(OUO_F32, nb, r, m > n ? m : n);
    {
      // the two partial sets and the Gram residuals are used one after the
      // other: one region (residuals of member i at i times the stride of
      // the Gram's input, at most the largest of the inputs' strides)
      const int64_t f1 = g.ks1 > 1 ? g.ks1 * (int64_t)r * pitch4(m) : 0;
      const int64_t f2 = g.ks2 > 1 ? g.ks2 * (int64_t)r * pitch4(n) : 0;
      int64_t f = f1 > f2 ? f1 : f2;
      const int64_t xs[5] = {g.Pt.stride, g.Rt.stride, g.Qn.stride, g.T.stride,
                             (int64_t)r * pitch4(n)};
      for (int64_t x : xs) f = x > f ? x : f;
      Buf region = take_bytes(ar, (size_t)nb * (size_t)f * 4 + 256);
      g.lo = reinterpret_cast<float*>(region.p);
      g.kp1 = Buf();
      g.kp1.p = region.p;
      g.kp1.dtype = OUO_F32;
      g.kp1.rows = r;
      g.kp1.cols = m;
      g.kp1.ld = pitch4(m);
      g.kp1.stride = r * pitch4(m);
      g.kp1.nb = nb * g.ks1;
      g.kp2 = g.kp1;
      g.kp2.cols = n;
      g.kp2.ld = pitch4(n);
      g.kp2.stride = r * pitch4(n);
      g.kp2.nb = nb * g.ks2;
    }
    const int64_t gp_m = cholqr_gram_part_floats(r, m), gp_n = cholqr_gram_part_floats(r, n);
    g.gstride = gp_m > gp_n ? gp_m : gp_n;
    g.gpart = reinterpret_cast<float*>(take_bytes(ar, (size_t)nb * g.gstride * 4).p);
    g.S = ar.take(OUO_F32, nb, r, r);
    g.Lb = ar.take(OUO_F32, nb, R, R);
    g.Z = reinterpret_cast<float*>(take_bytes(ar, (size_t)nb * cholqr_z_floats(r) * 4).p);
    if (!cholqr_small_rank(r)) {
      g.Ld = ar.take(OUO_F32, nb, R, R);
      g.ctl_stride = align_up(chol_blocked_ctl_bytes(r), 256);
      g.ctl = take_bytes(ar, (size_t)nb * g.ctl_stride).p;
    }
  }
  return gs;
}

size_t plan_bytes(const ouo_mat* M, int nmat, const int* ranks) {
  Arena ar{nullptr, 0, 0, true};
  plan(M, nmat, ranks, ar);
  return ar.used + 256;
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

// The members' caller matrices as one evenly strided batch, when they are
// laid out that way (same ld, equal byte steps, 16-byte multiple, no
// overlap); false otherwise.
bool caller_uniform(const ouo_mat* mats, const std::vector<int>& mem, int dtype, Buf* out) {
  const ouo_mat& f = mats[mem[0]];
  const int64_t es = (int64_t)elem_size(dtype);
  if (mem.size() == 1) {
    *out = caller_buf(f, dtype);
    return true;
  }
  const int64_t step = reinterpret_cast<const char*>(mats[mem[1]].ptr) -
                       reinterpret_cast<const char*>(f.ptr);
  if (step <= 0 || step % 16 || step % es || step < f.rows * f.ld * es) return false;
  for (size_t k = 0; k < mem.size(); ++k) {
    const ouo_mat& x = mats[mem[k]];
    if (x.ld != f.ld || reinterpret_cast<const char*>(x.ptr) !=
                            reinterpret_cast<const char*>(f.ptr) + (int64_t)k * step)
      return false;
  }
  *out = caller_buf(f, dtype);
  out->stride = step / es;
  out->nb = (int64_t)mem.size();
  return true;
}

// Descriptors of one GEMM stage for a group whose A and / or B operands are
// caller matrices: one descriptor over the whole group when the caller
// operands are evenly strided, else one per member.
void add_descs(std::vector<GemmDesc>& out, const GemmDesc& proto, const DGroup& g,
               const ouo_mat* Acall, const ouo_mat* Bcall, const Buf& Aws, const Buf& Bws,
               const Buf& Ows) {
  const int64_t nb = (int64_t)g.members.size();
  Buf A = Aws, B = Bws;
  bool uniform = true;
  if (Acall) uniform = uniform && caller_uniform(Acall, g.members, OUO_F32, &A);
  if (Bcall) uniform = uniform && caller_uniform(Bcall, g.members, OUO_F32, &B);
  if (uniform) {
    GemmDesc d = proto;
    d.nb = nb;
    d.A = A;
    d.B = B;
    d.out_f32 = Ows;
    out.push_back(d);
    return;
  }
  const int64_t per = Ows.nb / nb;  // outputs per member (K splits)
  for (int64_t k = 0; k < nb; ++k) {
    GemmDesc d = proto;
    d.nb = 1;
    d.A = Acall ? caller_buf(Acall[g.members[k]], OUO_F32) : view(Aws, k, 1);
    d.B = Bcall ? caller_buf(Bcall[g.members[k]], OUO_F32) : view(Bws, k, 1);
    d.out_f32 = view(Ows, k * per, per);
    out.push_back(d);
  }
}

// Which CholeskyQR jobs of a pass take the one-CTA Cholesky.
int orth_factor(std::vector<CholQrJob>& jobs, const std::vector<const DGroup*>& owner,
                const std::vector<int64_t>& mem, int* status, cudaStream_t s) {
  std::vector<CholQrJob> small;
  for (size_t k = 0; k < jobs.size(); ++k) {
    if (cholqr_small_rank(jobs[k].r)) {
      small.push_back(jobs[k]);
      continue;
    }
    const DGroup& g = *owner[k];
    const int64_t i = mem[k];
    OUO_TRY(chol_blocked(jobs[k].S, 1, jobs[k].r, jobs[k].L, jobs[k].Lb,
                         const_cast<float*>(jobs[k].Dd), g.ctl + (size_t)i * g.ctl_stride,
                         status, s));
  }
  return cholqr_factor(small, status, s);
}

// One CholeskyQR pass over every job: Gram, Cholesky, triangular solve.
// With `gram_done`, S already holds the (summed) Gram matrices.
int orth_pass(std::vector<CholQrJob>& jobs, const std::vector<const DGroup*>& owner,
              const std::vector<int64_t>& mem, int* status, cudaStream_t s, bool gram_done) {
  if (jobs.empty()) return OUO_OK;
  if (!gram_done) OUO_TRY(cholqr_gram(jobs, status, s));
  OUO_TRY(orth_factor(jobs, owner, mem, status, s));
  return cholqr_apply(jobs, status, s);
}

// A CholeskyQR job on member i of group g (rows X, length L; the members'
// inputs `xstride` floats apart), factor buffers from the group.  Gram
// partials and residuals are laid out evenly over the members, so that
// the group's Gram is one GEMM descriptor.
CholQrJob orth_job(const DGroup& g, int64_t i, const float* X, int64_t ldx, int64_t L,
                   int64_t xstride) {
  CholQrJob j;
  j.X = X;
  j.ldx = ldx;
  j.r = g.r;
  j.L = L;
  j.Xlo = g.lo + i * xstride;
  j.gpart = g.gpart + i * cholqr_gram_part_floats(g.r, L);
  j.Z = g.Z + i * (int64_t)cholqr_z_floats(g.r);
  j.S = reinterpret_cast<float*>(view(g.S, i, 1).p);
  j.Lb = reinterpret_cast<float*>(view(g.Lb, i, 1).p);
  j.Dd = g.Ld.p ? reinterpret_cast<const float*>(view(g.Ld, i, 1).p) : nullptr;
  return j;
}

float* fp(const Buf& b, int64_t i) { return reinterpret_cast<float*>(view(b, i, 1).p); }

// Stage: Pt = Qt B^T for every matrix (split-K partials summed into Pt).
int stage_project(const std::vector<DGroup>& gs, const ouo_mat* M, const ouo_mat* Q,
                  int* status, cudaStream_t s) {
  std::vector<GemmDesc> ds;
  std::vector<RowsJob> red;
  for (const DGroup& g : gs) {
    GemmDesc d;
    d.M = g.r; d.N = g.m; d.K = g.n;
    d.has_f32 = true;
    d.ksplit = g.ks1;
    d.per_desc_tiles = true;
    add_descs(ds, d, g, Q, M, Buf(), Buf(), g.ks1 > 1 ? g.kp1 : g.Pt);
    if (g.ks1 > 1) {
      for (int64_t i = 0; i < (int64_t)g.members.size(); ++i) {
        RowsJob rj;
        rj.part = fp(g.kp1, i * g.ks1);
        rj.ldp = g.kp1.ld;
        rj.sp = g.kp1.stride;
        rj.ks = g.ks1;
        rj.rows = g.r;
        rj.n = g.m;
        rj.out = fp(g.Pt, i);
        rj.ldo = g.Pt.ld;
        red.push_back(rj);
      }
    }
  }
  OUO_TRY(gemm_umma_grouped(ds, s, status));
  return rows_reduce(red, 0.f, s);
}

// Stage: passes pass_from .. pass_to - 1 of CholeskyQR2 on every Pt: the
// first pass solves Pt into T, the second T back into Pt and also writes
// P = Pt^T and its bf16 copy.
int stage_orth_p(const std::vector<DGroup>& gs, int* status, cudaStream_t s, int pass_from,
                 int pass_to) {
  for (int pass = pass_from; pass < pass_to; ++pass) {
    std::vector<CholQrJob> jobs;
    std::vector<const DGroup*> own;
    std::vector<int64_t> mem;
    for (const DGroup& g : gs) {
      for (int64_t i = 0; i < (int64_t)g.members.size(); ++i) {
        CholQrJob j = pass == 0 ? orth_job(g, i, fp(g.Pt, i), g.Pt.ld, g.m, g.Pt.stride)
                                : orth_job(g, i, fp(g.T, i), g.T.ld, g.m, g.T.stride);
        j.Y = pass == 0 ? fp(g.T, i) : fp(g.Pt, i);
        j.ldy = pass == 0 ? g.T.ld : g.Pt.ld;
        if (pass == 1) {
          j.Yt = fp(g.P, i);
          j.ldyt = g.P.ld;
          j.Ytb = reinterpret_cast<uint16_t*>(view(g.Pb, i, 1).p);
          j.ldytb = g.Pb.ld;
        }
        jobs.push_back(j);
        own.push_back(&g);
        mem.push_back(i);
      }
    }
    OUO_TRY(orth_pass(jobs, own, mem, status, s, false));
  }
  return OUO_OK;
}

// Stage: Rt = Pt B into `dst(g, i)` (Rt of the workspace, or the
// caller-summed buffer of the row-sharded step), split-K partials summed.
template <class Dst>
int stage_rproject(const std::vector<DGroup>& gs, const ouo_mat* M, Dst dst, int* status,
                   cudaStream_t s) {
  std::vector<GemmDesc> ds;
  std::vector<RowsJob> red;
  for (const DGroup& g : gs) {
    GemmDesc d;
    d.M = g.r; d.N = g.n; d.K = g.m;
    d.b_mn = 1;
    d.has_f32 = true;
    d.ksplit = g.ks2;
    d.per_desc_tiles = true;
    d.pair_mn = true;  // the two CTAs of a pair share each B (momentum) tile
    if (g.ks2 > 1) {
      add_descs(ds, d, g, nullptr, M, g.Pt, Buf(), g.kp2);
      for (int64_t i = 0; i < (int64_t)g.members.size(); ++i) {
        RowsJob rj;
        rj.part = fp(g.kp2, i * g.ks2);
        rj.ldp = g.kp2.ld;
        rj.sp = g.kp2.stride;
        rj.ks = g.ks2;
        rj.rows = g.r;
        rj.n = g.n;
        int64_t ld = 0;
        rj.out = dst(g, i, &ld);
        rj.ldo = ld;
        red.push_back(rj);
      }
    } else {
      // outputs straight into dst: per member when dst is not one batch
      std::vector<GemmDesc> one;
      add_descs(one, d, g, nullptr, M, g.Pt, Buf(), g.Rt);
      int64_t ld0 = 0;
      float* base = dst(g, 0, &ld0);
      if (base == fp(g.Rt, 0)) {
        for (auto& x : one) ds.push_back(x);
      } else {
        for (int64_t i = 0; i < (int64_t)g.members.size(); ++i) {
          GemmDesc di = d;
          di.nb = 1;
          di.A = view(g.Pt, i, 1);
          di.B = caller_buf(M[g.members[i]], OUO_F32);
          int64_t ld = 0;
          Buf o;
          o.p = reinterpret_cast<char*>(dst(g, i, &ld));
          o.dtype = OUO_F32;
          o.rows = g.r;
          o.cols = g.n;
          o.ld = ld;
          o.stride = g.r * ld;
          o.nb = 1;
          di.out_f32 = o;
          ds.push_back(di);
        }
      }
    }
  }
  OUO_TRY(gemm_umma_grouped(ds, s, status));
  return rows_reduce(red, 0.f, s);
}

// Stage: from Rt (rt(g, i), row pitch ldr): sigma (optional), and Q_new^T
// into Qn and the caller's state -- column normalization (Dion) or
// CholeskyQR2 (Orth-Dion).
template <class Rtp>
int stage_qnew(const std::vector<DGroup>& gs, Rtp rt, const ouo_mat* Q_state,
               const ouo_dion_params* p, float* sigma, const std::vector<int64_t>& sig_off,
               int* status, cudaStream_t s) {
  std::vector<RowsJob> rows;
  for (const DGroup& g : gs) {
    for (int64_t i = 0; i < (int64_t)g.members.size(); ++i) {
      const int bi = g.members[i];
      const bool colnorm = p->norm_mode == OUO_DION_COLNORM;
      int64_t ld = 0;
      RowsJob rj;
      rj.part = rt(g, i, &ld);
      rj.ldp = ld;
      rj.sp = 0;
      rj.ks = 1;
      rj.rows = g.r;
      rj.n = g.n;
      rj.outb = reinterpret_cast<uint16_t*>(view(g.Rtb, i, 1).p);  // the M update's operand
      rj.ldob = g.Rtb.ld;
      rj.sigma = sigma ? sigma + sig_off[bi] : nullptr;
      if (colnorm) {
        rj.qn = fp(g.Qn, i);
        rj.ldq = g.Qn.ld;
        rj.q2 = reinterpret_cast<float*>(Q_state[bi].ptr);
        rj.ldq2 = Q_state[bi].ld;
      }
      rows.push_back(rj);
    }
  }
  OUO_TRY(rows_reduce(rows, p->eps, s));
  if (p->norm_mode == OUO_DION_COLNORM) return OUO_OK;
  for (int pass = 0; pass < 2; ++pass) {
    std::vector<CholQrJob> jobs;
    std::vector<const DGroup*> own;
    std::vector<int64_t> mem;
    for (const DGroup& g : gs) {
      for (int64_t i = 0; i < (int64_t)g.members.size(); ++i) {
        int64_t ld = 0, xst = 0;
        float* x = nullptr;
        if (pass == 0) {
          x = rt(g, i, &ld);
          // residuals spaced like the inputs when those are evenly spaced
          // (the workspace's Rt), so that the group is one Gram descriptor
          xst = (int64_t)g.r * ld;
          if (g.members.size() > 1) {
            int64_t l1 = 0;
            const int64_t d = rt(g, 1, &l1) - rt(g, 0, &l1);
            if (d >= xst && d <= g.Rt.stride) xst = d;
          }
        } else {
          x = fp(g.T, i);
          ld = g.T.ld;
          xst = g.T.stride;
        }
        CholQrJob j = orth_job(g, i, x, ld, g.n, xst);
        j.Y = pass == 0 ? fp(g.T, i) : fp(g.Qn, i);
        j.ldy = pass == 0 ? g.T.ld : g.Qn.ld;
        if (pass == 1) {
          const int bi = g.members[i];
          j.Y2 = reinterpret_cast<float*>(Q_state[bi].ptr);
          j.ldy2 = Q_state[bi].ld;
        }
        jobs.push_back(j);
        own.push_back(&g);
        mem.push_back(i);
      }
    }
    OUO_TRY(orth_pass(jobs, own, mem, status, s, false));
  }
  return OUO_OK;
}

// Stage: M <- beta B - (beta - mu) P Rt and W <- (1 - lr wd) W - lr s P Qn,
// in place in the caller's matrices.  Both are rank-r updates whose C0 is
// the output itself: the GEMM's TMA epilogue loads each C0 box, adds the
// product and stores it back (bulk copies only).  With K = r the operand
// tiles weigh as much as the output they update, so both run on CTA-pair
// tiles (half the operand bytes per output), and the M update takes bf16
// operands (P and Rt rounded once: its product is scaled by beta - mu and
// lands in the momentum buffer, so the rounding is far inside the
// tolerance).  The weight update keeps tf32 operands, so that Orth-Dion's
// update stays a partial isometry to fp32-level accuracy.  Outputs are
// described to the TMA as one evenly strided batch per group when the
// caller's matrices are laid out that way, else one matrix per segment.
int stage_update(const std::vector<DGroup>& gs, const ouo_mat* M, const ouo_mat* W,
                 int w_dtype, const ouo_dion_params* p, const float* scale, int* status,
                 cudaStream_t s) {
  std::vector<GemmDesc> dm, dw;
  for (const DGroup& g : gs) {
    const int64_t nb = (int64_t)g.members.size();
    GemmDesc d;
    d.M = g.m; d.N = g.n; d.K = g.r;
    d.b_mn = 1;
    d.has_c0 = true;
    d.c0_from_out = true;
    d.per_desc_tiles = true;
    d.pair_mn = true;
    // M update (fp32 output)
    GemmDesc x = d;
    x.alpha = -(p->beta - p->mu);
    x.beta = p->beta;
    x.has_f32 = true;
    Buf mo;
    if (caller_uniform(M, g.members, OUO_F32, &mo)) {
      x.nb = nb;
      x.A = g.Pb;
      x.B = g.Rtb;
      x.out_f32 = mo;
      dm.push_back(x);
    } else {
      for (int64_t k = 0; k < nb; ++k) {
        GemmDesc xi = x;
        xi.nb = 1;
        xi.A = view(g.Pb, k, 1);
        xi.B = view(g.Rtb, k, 1);
        xi.out_f32 = caller_buf(M[g.members[k]], OUO_F32);
        dm.push_back(xi);
      }
    }
    // W update (caller dtype), per-matrix alpha = -lr * scale
    GemmDesc y = d;
    y.beta = 1.0f - p->lr * p->wd;
    y.alpha = -p->lr;
    y.has_f32 = w_dtype == OUO_F32;
    y.has_bf16 = w_dtype == OUO_BF16;
    Buf wo;
    auto alpha_of = [&](int64_t k) { return -p->lr * (scale ? scale[g.members[k]] : 1.0f); };
    if (caller_uniform(W, g.members, w_dtype, &wo)) {
      y.nb = nb;
      y.A = g.P;
      y.B = g.Qn;
      (w_dtype == OUO_F32 ? y.out_f32 : y.out_bf16) = wo;
      for (int64_t k = 0; k < nb; ++k) y.direct_alpha.push_back(alpha_of(k));
      dw.push_back(y);
    } else {
      for (int64_t k = 0; k < nb; ++k) {
        GemmDesc yi = y;
        yi.nb = 1;
        yi.A = view(g.P, k, 1);
        yi.B = view(g.Qn, k, 1);
        (w_dtype == OUO_F32 ? yi.out_f32 : yi.out_bf16) =
            caller_buf(W[g.members[k]], w_dtype);
        yi.direct_alpha.push_back(alpha_of(k));
        dw.push_back(yi);
      }
    }
  }
  OUO_TRY(gemm_umma_grouped(dm, s, status));
  return gemm_umma_grouped(dw, s, status);
}

int validate_dion(const ouo_dion_params* p) {
  if (!p) return set_error(OUO_ERR_INVALID_ARG, "NULL dion params");
  if (p->norm_mode != OUO_DION_COLNORM && p->norm_mode != OUO_DION_QR)
    return set_error(OUO_ERR_INVALID_ARG, "unknown norm_mode %d", p->norm_mode);
  if (!(p->eps >= 0.f)) return set_error(OUO_ERR_INVALID_ARG, "eps must be >= 0");
  return OUO_OK;
}

}  // namespace
}  // namespace ouo

extern "C" size_t dion_workspace_bytes(const ouo_mat* M, int nmat,
                                       const ouo_dion_params* p) {
  if (!M || !p || nmat <= 0 || nmat > OUO_MAX_BATCH || p->rank < 1) return 0;
  std::vector<int> ranks((size_t)nmat, p->rank);
  return ouo::plan_bytes(M, nmat, ranks.data());
}

extern "C" size_t dion_workspace_bytes_ranks(const ouo_mat* M, const int* ranks,
                                             int nmat, const ouo_dion_params* p) {
  if (!M || !ranks || !p || nmat <= 0 || nmat > OUO_MAX_BATCH) return 0;
  for (int i = 0; i < nmat; ++i)
    if (ranks[i] < 1) return 0;
  return ouo::plan_bytes(M, nmat, ranks);
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
  std::vector<int64_t> sig_off((size_t)nmat);
  int64_t so = 0;
  for (int i = 0; i < nmat; ++i) {
    const int r = p->rank ? p->rank : (int)Q_state[i].rows;
    ranks[i] = r;
    sig_off[i] = so;
    so += r;
    if (r < 1 || r > M[i].rows || r > M[i].cols)
      return set_error(OUO_ERR_INVALID_ARG, "rank %d outside [1, min(rows, cols)] for M[%d]",
                       r, i);
    if (r > 1024)
      return set_error(OUO_ERR_UNSUPPORTED, "rank %d above 1024 (M[%d])", r, i);
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
  const size_t need = plan_bytes(M, nmat, ranks.data());
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
  const std::vector<DGroup> gs = plan(M, nmat, ranks.data(), ar);
  auto rt_ws = [](const DGroup& g, int64_t i, int64_t* ld) {
    *ld = g.Rt.ld;
    return fp(g.Rt, i);
  };
  OUO_TRY(stage_project(gs, M, Q_state, dev_status, s));
  OUO_TRY(stage_orth_p(gs, dev_status, s, 0, 2));
  OUO_TRY(stage_rproject(gs, M, rt_ws, dev_status, s));
  OUO_TRY(stage_qnew(gs, rt_ws, Q_state, p, sigma, sig_off, dev_status, s));
  return stage_update(gs, M, W, w_dtype, p, scale, dev_status, s);
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
// formed redundantly on every rank.  The four calls run the same batched
// stages as dion_lowrank_step, so one rank reproduces it bit for bit.
namespace ouo {
namespace {

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
    if (r > 1024)
      return set_error(OUO_ERR_UNSUPPORTED, "rank %d above 1024 (M[%d])", r, i);
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
  const size_t need = plan_bytes(M, nmat, ranks.data());
  if (!ws || ws_bytes < need)
    return set_error(OUO_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given",
                     need, ws_bytes);
  if ((uintptr_t)ws % 256)
    return set_error(OUO_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  return require_sm100();
}

// Offsets (floats) of every batch matrix's block of `red`.
std::vector<int64_t> red_offsets(const ouo_mat* M, const std::vector<int>& ranks) {
  std::vector<int64_t> off(ranks.size());
  int64_t o = 0;
  for (size_t i = 0; i < ranks.size(); ++i) {
    off[i] = o;
    o += red_block(ranks[i], M[i].cols);
  }
  return off;
}

// The Gram matrices of every member's rows in `which` (Pt, or T after the
// first solve), summed into S = the matrix's block of red.
int gram_into_red(const std::vector<DGroup>& gs, Buf DGroup::*which, float* red,
                  const std::vector<int64_t>& off, int64_t (*rows_of)(const DGroup&),
                  int* status, cudaStream_t s) {
  std::vector<CholQrJob> jobs;
  for (const DGroup& g : gs) {
    const Buf& x = g.*which;
    for (int64_t i = 0; i < (int64_t)g.members.size(); ++i) {
      CholQrJob j = orth_job(g, i, fp(x, i), x.ld, rows_of(g), x.stride);
      j.S = red + off[g.members[i]];
      jobs.push_back(j);
    }
  }
  return cholqr_gram(jobs, status, s);
}

int64_t local_rows(const DGroup& g) { return g.m; }

// orth1 (second = false) and orth2 (second = true): Cholesky of the summed
// Gram matrices in red, the solve on the local rows (Pt into T, then T
// back into Pt, as in the unsharded step), then red = the next pass's Gram
// matrices (orth1) or P^T B (orth2).
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
  const std::vector<DGroup> gs = plan(M, nmat, ranks.data(), ar);
  const std::vector<int64_t> off = red_offsets(M, ranks);
  std::vector<CholQrJob> jobs;
  std::vector<const DGroup*> own;
  std::vector<int64_t> mem;
  for (const DGroup& g : gs) {
    for (int64_t i = 0; i < (int64_t)g.members.size(); ++i) {
      const int bi = g.members[i];
      // the shift of a retry takes the global row count
      const Buf& x = second ? g.T : g.Pt;
      const Buf& y = second ? g.Pt : g.T;
      CholQrJob j = orth_job(g, i, fp(x, i), x.ld, rows_total[bi], x.stride);
      j.S = red + off[bi];
      j.Y = fp(y, i);
      j.ldy = y.ld;
      if (second) {
        j.Yt = fp(g.P, i);
        j.ldyt = g.P.ld;
        j.Ytb = reinterpret_cast<uint16_t*>(view(g.Pb, i, 1).p);
        j.ldytb = g.Pb.ld;
      }
      // the solve runs over the local rows
      jobs.push_back(j);
      own.push_back(&g);
      mem.push_back(i);
    }
  }
  OUO_TRY(orth_factor(jobs, own, mem, dev_status, s));
  for (CholQrJob& j : jobs) j.L = 0;
  {
    size_t k = 0;
    for (const DGroup& g : gs)
      for (int64_t i = 0; i < (int64_t)g.members.size(); ++i) jobs[k++].L = g.m;
  }
  OUO_TRY(cholqr_apply(jobs, dev_status, s));
  if (!second) return gram_into_red(gs, &DGroup::T, red, off, local_rows, dev_status, s);
  auto dst = [&](const DGroup& g, int64_t i, int64_t* ld) {
    *ld = pitch4(g.n);
    return red + off[g.members[i]];
  };
  return stage_rproject(gs, M, dst, dev_status, s);
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
  return ouo::plan_bytes(M, nmat, ranks.data());
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
  const std::vector<DGroup> gs = plan(M, nmat, ranks.data(), ar);
  OUO_TRY(stage_project(gs, M, Q_state, dev_status, s));
  return gram_into_red(gs, &DGroup::Pt, red, red_offsets(M, ranks), local_rows, dev_status, s);
}

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
  const std::vector<DGroup> gs = plan(M, nmat, ranks.data(), ar);
  const std::vector<int64_t> off = red_offsets(M, ranks);
  // R^T (summed over the ranks) is read where the caller left it
  auto rt_red = [&](const DGroup& g, int64_t i, int64_t* ld) {
    *ld = pitch4(g.n);
    return red + off[g.members[i]];
  };
  std::vector<int64_t> no_sig((size_t)nmat, 0);
  OUO_TRY(stage_qnew(gs, rt_red, Q_state, p, nullptr, no_sig, dev_status, s));
  return stage_update(gs, M, W, w_dtype, p, scale, dev_status, s);
}
