// Host orchestration of standard and Gram Newton-Schulz over a batch.
//
// Sources: "Dion3: Full-Stack Orthogonal Updates", Abstract (Muon's
// cubic-time Newton-Schulz; Gram Newton-Schulz lowers its FLOP cost);
// "Dion3：全栈正交更新", 核心洞察 / 核心模块 (iterate on the symmetric Gram
// matrix; restarts and safety factors keep it stable) and 局限 (restarts fix
// spurious negative eigenvalues and eigenvector drift; fp16 / bf16 need
// care).
//
// Per group of equal-shape matrices (k x n after orientation, k <= n):
//   prep   X0 = X / (||X||_F + eps) into workspace (transposed if needed)
//   Gram:  A = X0 X0^T;  for t: H = a'I + b'A + c'A^2;  Q <- H Q  (Q = H on
//          the first iteration of a segment);  restart: X0 <- Q X0,
//          A = X0 X0^T;  otherwise A <- H (H A);  finally O = Q X0.
//   Std:   for t: A = X X^T;  B = b'A + c'A^2;  X <- a'X + B X.
//
// Precision (OUO_PREC_BF16): products with an n-long contraction or output
// (X X^T, Q X, B X) take bf16 operands; the k x k products (A^2, H Q, H A,
// H T) take tf32 operands, stored already rounded to tf32; every
// accumulation is fp32 in TMEM.  Rounding A itself to bf16 measurably breaks
// the 2e-2 accuracy bound on 512 x 4096 inputs; tf32 keeps it below 1e-2.
// OUO_PREC_FP32 runs every product in fp32 on CUDA cores.
#include <algorithm>
#include <cmath>

#include <cstdlib>

#include "internal.h"

namespace ouo {
namespace {

struct Coeffs {
  float a, b, c;
};

Coeffs scaled(const ouo_ns_params& p) {
  double s = p.safety;
  Coeffs c;
  c.a = (float)((double)p.a / s);
  c.b = (float)((double)p.b / (s * s * s));
  c.c = (float)((double)p.c / (s * s * s * s * s));
  return c;
}

struct Oriented {
  int64_t k, n;
  bool transpose;
};

Oriented orient(const Group& g) {
  Oriented o;
  o.transpose = g.rows > g.cols;
  o.k = o.transpose ? g.cols : g.rows;
  o.n = o.transpose ? g.rows : g.cols;
  return o;
}

struct GroupWs {
  Buf x0, x1, y;       // k x n: current / alternate X, final output
  Buf kk[3];           // k x k fp32 (A, H/Q rotation)
  Buf A, T;            // k x k fp32
  Buf qbf;             // k x k bf16 copy of Q (bf16 path)
  Buf bm;              // standard NS: b'A + c'A^2 (bf16 or fp32)
  double* scratch;     // rows doubles per matrix + one float per matrix
};

GroupWs carve(Arena& ar, const Group& g, const Oriented& o, bool gram,
              int precision, int o_dtype) {
  GroupWs w;
  const int64_t nb = (int64_t)g.members.size();
  const bool bf = precision == OUO_PREC_BF16;
  const int xd = bf ? OUO_BF16 : OUO_F32;
  w.x0 = ar.take(xd, nb, o.k, o.n);
  w.x1 = ar.take(xd, nb, o.k, o.n);
  w.y = ar.take(bf ? o_dtype : OUO_F32, nb, o.k, o.n);
  w.A = ar.take(OUO_F32, nb, o.k, o.k);
  if (gram) {
    for (int i = 0; i < 3; ++i) w.kk[i] = ar.take(OUO_F32, nb, o.k, o.k);
    w.T = ar.take(OUO_F32, nb, o.k, o.k);
    if (bf) w.qbf = ar.take(OUO_BF16, nb, o.k, o.k);
  } else {
    w.bm = ar.take(bf ? OUO_BF16 : OUO_F32, nb, o.k, o.k);
  }
  // float64 row sums (rows of the caller's matrix) + float scales
  Buf s = ar.take(OUO_F32, 1, 1, nb * g.rows * 2 + nb);
  w.scratch = reinterpret_cast<double*>(s.p);
  return w;
}

GemmDesc syrk(const Buf& X, const Buf& out, bool bf) {
  GemmDesc d;
  d.M = d.N = X.rows;
  d.K = X.cols;
  d.nb = X.nb;
  d.A = X;
  d.B = X;
  d.tri = true;
  d.out_f32 = out;
  d.has_f32 = true;
  d.round_tf32 = bf;
  return d;
}

// out = alpha * L R + beta * C0 + gamma * I for commuting symmetric k x k L, R
GemmDesc symprod(const Buf& L, const Buf& R, float alpha, const Buf* C0,
                 float beta, float gamma, bool bf) {
  GemmDesc d;
  d.M = d.N = d.K = L.rows;
  d.nb = L.nb;
  d.A = L;
  d.B = R;
  d.alpha = alpha;
  if (C0) {
    d.C0 = *C0;
    d.has_c0 = true;
    d.beta = beta;
  }
  d.gamma = gamma;
  d.tri = true;
  d.round_tf32 = bf;
  return d;
}

// out = alpha * L X + beta * C0, L k x k (K-major), X k x n (MN-major)
GemmDesc apply_left(const Buf& L, const Buf& X, const Buf& out, float alpha,
                    const Buf* C0, float beta) {
  GemmDesc d;
  d.M = L.rows;
  d.N = X.cols;
  d.K = L.cols;
  d.nb = L.nb;
  d.A = L;
  d.B = X;
  d.b_mn = 1;
  d.alpha = alpha;
  if (C0) {
    d.C0 = *C0;
    d.has_c0 = true;
    d.beta = beta;
  }
  if (out.dtype == OUO_BF16) {
    d.out_bf16 = out;
    d.has_bf16 = true;
  } else {
    d.out_f32 = out;
    d.has_f32 = true;
  }
  return d;
}

bool is_restart(const ouo_ns_params& p, int t) {
  for (int i = 0; i < p.n_restart; ++i)
    if (p.restart_after[i] == t) return true;
  return false;
}

// Index among {0, 1, 2} equal to neither a nor b (a and b may be equal or -1).
int free_idx(int a, int b) {
  for (int i = 0; i < 3; ++i)
    if (i != a && i != b) return i;
  return -1;
}

// One stage of the iteration over all groups: a single grouped tensor-core
// launch (bf16 path) or one CUDA-core GEMM per group (fp32 path).
// Upper-stored symmetric k x k matrices (tensor-core path on CTA-pair
// tiles): Gram matrices and symmetric products skip the mirrored write of
// tiles off the block diagonal, and every symmetric fp32 k x k operand (and
// symmetric C0) is read through its upper blocks.  A product that also
// writes a bf16 copy (the Q of Q X, read whole as a dense operand) keeps
// full storage.  Used when the launches run on pair tiles: the bf16 path,
// pairs enabled, and some k above 128 (so every symmetric launch of the
// call, which covers all groups, takes pairs).
// OUO_SYM_HALF=0 keeps full storage.
bool half_mode(const std::vector<GroupWs>& ws, bool bf) {
  if (!bf || !cta_pairs_enabled()) return false;
  const char* env = getenv("OUO_SYM_HALF");
  if (env && env[0] == '0') return false;
  for (const GroupWs& w : ws)
    if (w.A.rows > 128) return true;
  return false;
}

void mark_half(std::vector<GemmDesc>& ds, bool half) {
  if (!half) return;
  for (GemmDesc& d : ds) {
    if (!d.tri) continue;
    d.sym_half = !d.has_bf16;
    if (d.A.dtype == OUO_F32 && d.A.rows == d.A.cols) d.a_sym = d.b_sym = true;
    if (d.has_c0) d.c0_upper = true;
  }
}

int run_stage(const std::vector<GemmDesc>& ds, bool bf, cudaStream_t s,
              int* status, bool half = false) {
  if (bf && half) {
    std::vector<GemmDesc> hd = ds;
    mark_half(hd, true);
    return gemm_umma_grouped(hd, s, status);
  }
  if (bf) return gemm_umma_grouped(ds, s, status);
  for (const GemmDesc& d : ds) OUO_TRY(gemm_simt(d, s));
  return OUO_OK;
}

// The final product: groups writing to caller memory and groups writing to
// workspace differ in output kind, so they go in separate grouped launches.
int run_final(const std::vector<GemmDesc>& ds, bool bf, cudaStream_t s,
              int* status) {
  if (!bf) return run_stage(ds, bf, s, status);
  std::vector<GemmDesc> dir, ws;
  for (const GemmDesc& d : ds) (d.direct.empty() ? ws : dir).push_back(d);
  if (!dir.empty()) OUO_TRY(gemm_umma_grouped(dir, s, status));
  if (!ws.empty()) OUO_TRY(gemm_umma_grouped(ws, s, status));
  return OUO_OK;
}

struct Plan {
  std::vector<GroupWs> ws;
  std::vector<std::vector<MatRef>> direct;  // per group; empty = write-out
  int o_dtype;
};

// Attaches the caller's output table (if any) to the final product of group i.
void final_output(GemmDesc& d, const Plan& pl, size_t i, bool bf) {
  if (bf && !pl.direct[i].empty()) {
    d.direct = pl.direct[i];
    d.direct_dtype = pl.o_dtype;
  }
}

// Gram Newton-Schulz, all groups in lockstep (they share the schedule).
int gram_all(const ouo_ns_params& p, Plan& pl, cudaStream_t s, int* status) {
  const bool bf = p.precision == OUO_PREC_BF16;
  const bool half = half_mode(pl.ws, bf);
  const Coeffs c = scaled(p);
  const size_t ng = pl.ws.size();
  int xi = 0;  // current X is x0 (0) or x1 (1)
  auto Xc = [&](GroupWs& w) -> Buf& { return xi ? w.x1 : w.x0; };
  auto Xa = [&](GroupWs& w) -> Buf& { return xi ? w.x0 : w.x1; };
  std::vector<GemmDesc> ds(ng);
  for (size_t i = 0; i < ng; ++i) ds[i] = syrk(Xc(pl.ws[i]), pl.ws[i].A, bf);
  OUO_TRY(run_stage(ds, bf, s, status, half));
  int q = -1;  // buffer holding Q; -1 while Q = I
  for (int t = 1; t <= p.iters; ++t) {
    const bool last = t == p.iters;
    const bool restart = !last && is_restart(p, t);
    const bool need_qbf = bf && (last || restart);
    const int h = free_idx(q, -1);
    // H = c' A A + b' A + a' I
    for (size_t i = 0; i < ng; ++i) {
      GroupWs& w = pl.ws[i];
      ds[i] = symprod(w.A, w.A, c.c, &w.A, c.b, c.a, bf);
      ds[i].out_f32 = w.kk[h];
      ds[i].has_f32 = true;
      if (q < 0 && need_qbf) {
        ds[i].out_bf16 = w.qbf;
        ds[i].has_bf16 = true;
      }
    }
    OUO_TRY(run_stage(ds, bf, s, status, half));
    if (q < 0) {
      q = h;  // Q = H I
    } else {
      const int nq = free_idx(q, h);
      for (size_t i = 0; i < ng; ++i) {
        GroupWs& w = pl.ws[i];
        ds[i] = symprod(w.kk[h], w.kk[q], 1.f, nullptr, 0.f, 0.f, bf);
        ds[i].out_f32 = w.kk[nq];
        ds[i].has_f32 = true;
        if (need_qbf) {
          ds[i].out_bf16 = w.qbf;
          ds[i].has_bf16 = true;
        }
      }
      OUO_TRY(run_stage(ds, bf, s, status, half));
      q = nq;
    }
    if (last) break;
    if (restart) {
      for (size_t i = 0; i < ng; ++i) {
        GroupWs& w = pl.ws[i];
        ds[i] = apply_left(bf ? w.qbf : w.kk[q], Xc(w), Xa(w), 1.f, nullptr, 0.f);
      }
      OUO_TRY(run_stage(ds, bf, s, status, half));
      xi ^= 1;
      for (size_t i = 0; i < ng; ++i) ds[i] = syrk(Xc(pl.ws[i]), pl.ws[i].A, bf);
      OUO_TRY(run_stage(ds, bf, s, status, half));
      q = -1;
    } else {
      // A <- H (H A)
      for (size_t i = 0; i < ng; ++i) {
        GroupWs& w = pl.ws[i];
        ds[i] = symprod(w.kk[h], w.A, 1.f, nullptr, 0.f, 0.f, bf);
        ds[i].out_f32 = w.T;
        ds[i].has_f32 = true;
      }
      OUO_TRY(run_stage(ds, bf, s, status, half));
      for (size_t i = 0; i < ng; ++i) {
        GroupWs& w = pl.ws[i];
        ds[i] = symprod(w.kk[h], w.T, 1.f, nullptr, 0.f, 0.f, bf);
        ds[i].out_f32 = w.A;
        ds[i].has_f32 = true;
      }
      OUO_TRY(run_stage(ds, bf, s, status, half));
    }
  }
  if (q < 0) {
    // no iteration: the output is X0 itself
    for (size_t i = 0; i < ng; ++i) {
      OUO_TRY(convert_buf(Xc(pl.ws[i]), pl.ws[i].y, s));
      pl.direct[i].clear();
    }
  } else {
    for (size_t i = 0; i < ng; ++i) {
      GroupWs& w = pl.ws[i];
      ds[i] = apply_left(bf ? w.qbf : w.kk[q], Xc(w), w.y, 1.f, nullptr, 0.f);
      final_output(ds[i], pl, i, bf);
    }
    OUO_TRY(run_final(ds, bf, s, status));
  }
  return OUO_OK;
}

// Standard quintic Newton-Schulz, all groups in lockstep.
int std_all(const ouo_ns_params& p, Plan& pl, cudaStream_t s, int* status) {
  const bool bf = p.precision == OUO_PREC_BF16;
  const bool half = half_mode(pl.ws, bf);
  const Coeffs c = scaled(p);
  const size_t ng = pl.ws.size();
  int xi = 0;
  auto Xc = [&](GroupWs& w) -> Buf& { return xi ? w.x1 : w.x0; };
  auto Xa = [&](GroupWs& w) -> Buf& { return xi ? w.x0 : w.x1; };
  std::vector<GemmDesc> ds(ng);
  for (int t = 1; t <= p.iters; ++t) {
    for (size_t i = 0; i < ng; ++i) ds[i] = syrk(Xc(pl.ws[i]), pl.ws[i].A, bf);
    OUO_TRY(run_stage(ds, bf, s, status, half));
    // B = c' A A + b' A
    for (size_t i = 0; i < ng; ++i) {
      GroupWs& w = pl.ws[i];
      ds[i] = symprod(w.A, w.A, c.c, &w.A, c.b, 0.f, bf);
      ds[i].round_tf32 = false;
      if (w.bm.dtype == OUO_BF16) {
        ds[i].out_bf16 = w.bm;
        ds[i].has_bf16 = true;
      } else {
        ds[i].out_f32 = w.bm;
        ds[i].has_f32 = true;
      }
    }
    OUO_TRY(run_stage(ds, bf, s, status, half));
    // X <- a' X + B X   (the last iteration writes the output)
    const bool last = t == p.iters;
    for (size_t i = 0; i < ng; ++i) {
      GroupWs& w = pl.ws[i];
      Buf& X = Xc(w);
      ds[i] = apply_left(w.bm, X, last ? w.y : Xa(w), 1.f, &X, c.a);
      if (last) final_output(ds[i], pl, i, bf);
    }
    OUO_TRY(last ? run_final(ds, bf, s, status) : run_stage(ds, bf, s, status));
    xi ^= 1;
  }
  if (p.iters == 0) {
    for (size_t i = 0; i < ng; ++i) {
      OUO_TRY(convert_buf(Xc(pl.ws[i]), pl.ws[i].y, s));
      pl.direct[i].clear();
    }
  }
  return OUO_OK;
}

// True when a group's matrices can serve directly as the (read-only) X0
// operand of Gram NS: no
// normalization, no transposition, the arithmetic's own element type, rows
// on 16-byte boundaries, matrices equally spaced in memory (a batched
// [nb][rows][ld] block with a 16-byte multiple stride), and no output of the
// call overlapping the block (X0 is read again by later stages).
bool caller_x0(const ouo_mat* X, int x_dtype, const ouo_mat* O, int o_dtype,
               int nmat, const Group& g, const Oriented& o,
               const ouo_ns_params& p, bool gram, Buf* out) {
  const int want = p.precision == OUO_PREC_BF16 ? OUO_BF16 : OUO_F32;
  if (p.normalize || o.transpose || x_dtype != want) return false;
  // Standard NS and a second Gram restart write into the X0 buffer; only a
  // Gram schedule with at most one restart leaves it read-only.
  if (!gram) return false;
  int restarts = 0;
  for (int t = 1; t < p.iters; ++t) restarts += is_restart(p, t) ? 1 : 0;
  if (restarts > 1) return false;
  const size_t es = elem_size(x_dtype);
  const ouo_mat& f = X[g.members[0]];
  for (int m : g.members)
    if (!vec16(X[m], x_dtype) || X[m].ld != f.ld) return false;
  int64_t stride_b = 0;
  if (g.members.size() > 1) {
    stride_b = (int64_t)((const char*)X[g.members[1]].ptr - (const char*)f.ptr);
    if (stride_b <= 0 || stride_b % 16 || stride_b < f.rows * f.ld * (int64_t)es)
      return false;
    for (size_t i = 1; i < g.members.size(); ++i)
      if ((const char*)X[g.members[i]].ptr - (const char*)f.ptr != (int64_t)i * stride_b)
        return false;
  }
  const char* lo = (const char*)f.ptr;
  const char* hi = (const char*)X[g.members.back()].ptr + f.rows * f.ld * es;
  for (int i = 0; i < nmat; ++i) {
    const char* olo = (const char*)O[i].ptr;
    const char* ohi = olo + O[i].rows * O[i].ld * elem_size(o_dtype);
    if (olo < hi && lo < ohi) return false;
  }
  Buf b;
  b.p = const_cast<char*>(lo);
  b.dtype = x_dtype;
  b.rows = f.rows;
  b.cols = f.cols;
  b.ld = f.ld;
  b.stride = g.members.size() > 1 ? stride_b / (int64_t)es : f.rows * f.ld;
  b.nb = (int64_t)g.members.size();
  *out = b;
  return true;
}

int validate_params(const ouo_ns_params* p) {
  if (!p) return set_error(OUO_ERR_INVALID_ARG, "NULL ns params");
  if (p->iters < 0 || p->iters > 1000)
    return set_error(OUO_ERR_INVALID_ARG, "iters %d out of range", p->iters);
  if (!(p->safety >= 1.0f) || !std::isfinite(p->safety))
    return set_error(OUO_ERR_INVALID_ARG, "safety must be >= 1");
  if (!(p->eps >= 0.0f))
    return set_error(OUO_ERR_INVALID_ARG, "eps must be >= 0");
  if (p->precision != OUO_PREC_BF16 && p->precision != OUO_PREC_FP32)
    return set_error(OUO_ERR_INVALID_ARG, "unknown precision %d", p->precision);
  if (p->n_restart < 0 || p->n_restart > OUO_MAX_RESTARTS)
    return set_error(OUO_ERR_INVALID_ARG, "n_restart out of range");
  if (!std::isfinite(p->a) || !std::isfinite(p->b) || !std::isfinite(p->c))
    return set_error(OUO_ERR_INVALID_ARG, "non-finite coefficients");
  return OUO_OK;
}

size_t plan_bytes(const ouo_mat* X, int nmat, const ouo_ns_params* p,
                  bool gram, int o_dtype) {
  Arena ar{nullptr, 0, 0, true};
  for (const Group& g : group_by_shape(X, nmat))
    carve(ar, g, orient(g), gram, p->precision, o_dtype);
  return ar.used + 256;
}

}  // namespace

int ns_check_call(const ouo_mat* X, int x_dtype, const ouo_mat* O, int o_dtype,
                  int nmat, const ouo_ns_params* p, int* dev_status) {
  if (nmat < 0 || nmat > OUO_MAX_BATCH)
    return set_error(OUO_ERR_INVALID_ARG, "nmat %d out of range", nmat);
  OUO_TRY(validate_params(p));
  if (nmat == 0) return OUO_OK;
  OUO_TRY(validate_mats(X, nmat, x_dtype, "X"));
  OUO_TRY(validate_mats(O, nmat, o_dtype, "O"));
  OUO_TRY(validate_same_shapes(X, O, nmat, "X", "O"));
  if (dev_status && ((uintptr_t)dev_status % 4))
    return set_error(OUO_ERR_INVALID_ARG, "dev_status misaligned");
  return OUO_OK;
}

namespace {

int run_ns(const ouo_mat* X, int x_dtype, const ouo_mat* O, int o_dtype,
           int nmat, const ouo_ns_params* p, void* ws, size_t ws_bytes,
           int* dev_status, void* stream, bool gram) {
  clear_error();
  OUO_TRY(ns_check_call(X, x_dtype, O, o_dtype, nmat, p, dev_status));
  if (nmat == 0) return OUO_OK;
  const size_t need = plan_bytes(X, nmat, p, gram, o_dtype);
  if (!ws || ws_bytes < need)
    return set_error(OUO_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given",
                     need, ws_bytes);
  if ((uintptr_t)ws % 256)
    return set_error(OUO_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  OUO_TRY(require_sm100());
  cudaStream_t s = (cudaStream_t)stream;
  Arena ar{reinterpret_cast<char*>(ws), ws_bytes, 0, false};
  const std::vector<Group> groups = group_by_shape(X, nmat);
  Plan pl;
  pl.o_dtype = o_dtype;
  for (const Group& g : groups) {
    const Oriented o = orient(g);
    pl.ws.push_back(carve(ar, g, o, gram, p->precision, o_dtype));
    Buf direct_x0;
    if (caller_x0(X, x_dtype, O, o_dtype, nmat, g, o, *p, gram, &direct_x0)) {
      // the caller's batch already is the layout X0 needs: read it in place
      pl.ws.back().x0 = direct_x0;
    } else {
      OUO_TRY(ns_prep(X, x_dtype, g, o.transpose, p->normalize != 0, p->eps,
                      pl.ws.back().x0, pl.ws.back().scratch, s));
    }
    // The last product writes straight into the caller's O when the layout
    // allows (no transposition, 16-byte aligned rows, tensor-core path).
    std::vector<MatRef> direct;
    bool can_direct = p->precision == OUO_PREC_BF16 && !o.transpose;
    for (int m : g.members) can_direct = can_direct && vec16(O[m], o_dtype);
    if (can_direct)
      for (int m : g.members) direct.push_back(MatRef{O[m].ptr, O[m].ld});
    pl.direct.push_back(direct);
  }
  if (gram) OUO_TRY(gram_all(*p, pl, s, dev_status));
  else OUO_TRY(std_all(*p, pl, s, dev_status));
  for (size_t i = 0; i < groups.size(); ++i)
    if (pl.direct[i].empty())
      OUO_TRY(ns_writeout(pl.ws[i].y, O, o_dtype, groups[i], orient(groups[i]).transpose, s));
  return OUO_OK;
}

}  // namespace
}  // namespace ouo

extern "C" size_t ns_workspace_bytes(const ouo_mat* X, int nmat,
                                     const ouo_ns_params* p) {
  if (!X || !p || nmat <= 0) return 0;
  return ouo::plan_bytes(X, nmat, p, false, OUO_F32);
}

extern "C" size_t gram_ns_workspace_bytes(const ouo_mat* X, int nmat,
                                          const ouo_ns_params* p) {
  if (!X || !p || nmat <= 0) return 0;
  return ouo::plan_bytes(X, nmat, p, true, OUO_F32);
}

extern "C" int ns_orthogonalize(const ouo_mat* X, int x_dtype, const ouo_mat* O,
                                int o_dtype, int nmat, const ouo_ns_params* p,
                                void* ws, size_t ws_bytes, int* dev_status,
                                void* stream) {
  return ouo::run_ns(X, x_dtype, O, o_dtype, nmat, p, ws, ws_bytes, dev_status,
                     stream, false);
}

extern "C" int gram_ns_orthogonalize(const ouo_mat* X, int x_dtype,
                                     const ouo_mat* O, int o_dtype, int nmat,
                                     const ouo_ns_params* p, void* ws,
                                     size_t ws_bytes, int* dev_status,
                                     void* stream) {
  return ouo::run_ns(X, x_dtype, O, o_dtype, nmat, p, ws, ws_bytes, dev_status,
                     stream, true);
}
