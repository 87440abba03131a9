// The complex-phase gate's forward in 16-token chunks: per-CTA programs.
//
// "Semidirect Fourier Delta Attention" §3, eqs. (13)-(14): S' = Lambda_t S,
// Lambda_t = diag(lambda_t), lambda_t = alpha_t exp(i theta_t);
// S_t = S' + beta_t k_t (conj(v_t) - k_t^* S')^T; o_t = scale S_t^* q_t. The
// chunk-WY form of §2.2 eqs. (9)-(10) carries over with conjugates where k^*
// and q^* stand (rows i, j in 0..C-1 of a chunk; entry state S;
// G_{i<-j} = prod_{s=j+1..i} diag(lambda_s); gamma_i = G_{i<-(-1)};
// sigma_j = G_{C-1<-j}):
//   A_ij = beta_i k_i^* G_{i<-j} k_j (j < i),   M_ij = q_i^* G_{i<-j} k_j (j <= i)
//   T = (I + A)^-1,  W = T diag(beta) Khat,  Utilde = T diag(beta) conj(V)
//   U = Utilde - W S,  conj(O) = scale (Qhat S + M U),
//   S <- diag(gamma_{C-1}) S + Kbar^T U,
// with Khat_i = gamma_i conj(k_i), Qhat_i = gamma_i conj(q_i), Kbar_j = sigma_j k_j.
// Two programs:
//   prep (per chunk and head): lambda, gamma, sigma, A and M (per-pair running
//        products of lambda over at most 15 tokens), T by forward substitution,
//        then W, Kbar, Qhat (token-major [T, H, d_k]), Utilde ([T, H, d_v]),
//        M and gamma_{C-1} per checkpoint slot;
//   scan (per sequence, head, tile of DVT complex columns): per chunk
//        U = Utilde - W S, the outputs, the state update.
// Complex numbers are interleaved (real, imaginary) fp32 pairs, in global and
// in shared memory. The same executor contract as ckda_bwd_chunk.cuh: each
// phase is par<N>(x, f) over independent items, then a barrier, so the
// programs also run as plain host loops in the tests.
#pragma once

#include <math.h>

#include "ckda_bwd_chunk.cuh"

namespace ckda {
namespace cplx {

using bwdc::C;
using bwdc::par;

struct cf {
  float r, i;
};
CKDA_PROG cf cmul(cf a, cf b) { return cf{a.r * b.r - a.i * b.i, a.r * b.i + a.i * b.r}; }
// conj(a) b
CKDA_PROG cf cmulc(cf a, cf b) { return cf{a.r * b.r + a.i * b.i, a.r * b.i - a.i * b.r}; }
CKDA_PROG cf cadd(cf a, cf b) { return cf{a.r + b.r, a.i + b.i}; }
CKDA_PROG cf csub(cf a, cf b) { return cf{a.r - b.r, a.i - b.i}; }
CKDA_PROG cf cscale(float s, cf a) { return cf{s * a.r, s * a.i}; }
CKDA_PROG cf cconj(cf a) { return cf{a.r, -a.i}; }
CKDA_PROG cf cld(const float *p) { return cf{p[0], p[1]}; }
// read-only global data
CKDA_PROG cf cldg(const float *p) { return cf{CKDA_LDG(p), CKDA_LDG(p + 1)}; }
CKDA_PROG void cst(float *p, cf x) {
  p[0] = x.r;
  p[1] = x.i;
}

// Pointers and sizes of one call: q, k [T_total, H, d_k] and v, o [T_total,
// H, d_v] complex; alpha, theta [T_total, H, d_k] and beta [T_total, H] fp32;
// states [N, H, d_k, d_v] complex (s0, sf may be null).
struct Args {
  const float *q, *k, *v, *alpha, *theta, *beta, *s0;
  float *sf, *o;
  int H, DVF;
  float scale;
};

// Workspace (complex unless noted): W, Kbar, Qhat [T_total H][d_k];
// Utilde [T_total H][d_v]; M [slots][H][C][C]; gamma_{C-1} [slots][H][d_k].
struct Ws {
  float *wt, *kb, *qh, *ut, *mm, *gc;
};

template <int DK, int DVT>
struct PrepLayout {
  static constexpr int KS = 2 * (DK + 1), VS = 2 * (DVT + 1), CS = 2 * (C + 1);
  // C x DK complex: q, k, lambda, gamma, sigma; C x DVT complex: conj(v)
  static constexpr int Q = 0, K = Q + C * KS, LM = K + C * KS, GM = LM + C * KS,
                       SG = GM + C * KS, V = SG + C * KS;
  // C x C complex: A, M, T; the Gram phase's per-group partials; beta [C]
  static constexpr int NG = 2;  // channel groups of the Gram phase
  static constexpr int A = V + C * VS, M = A + C * CS, TT = M + C * CS, PG = TT + C * CS,
                       BE = PG + 4 * C * C * NG;
  static constexpr int FLOATS = BE + C;
  static constexpr size_t BYTES = (size_t)FLOATS * sizeof(float);
};

template <class X, int DK, int DVT>
CKDA_PROG void prep_program(X &x, const Args &a, const Ws &w, float *sm, int h, int t0, int L,
                            int slot) {
  using Ly = PrepLayout<DK, DVT>;
  constexpr int KS = Ly::KS, VS = Ly::VS, CS = Ly::CS;
  const int H = a.H, DVF = a.DVF;
  float *be = sm + Ly::BE;
  // stage q, k (complex), lambda = alpha (cos theta, sin theta), beta; rows
  // L..C-1 are inert (q = k = 0, lambda = 1, beta = 0)
  par<C * DK>(x, [&](int e) {
    const int i = e / DK, c = e - i * DK;
    cf qv{0.f, 0.f}, kv{0.f, 0.f}, lv{1.f, 0.f};
    if (i < L) {
      const size_t g = ((size_t)(t0 + i) * H + h) * DK + c;
      qv = cldg(a.q + 2 * g);
      kv = cldg(a.k + 2 * g);
      const float al = CKDA_LDG(a.alpha + g), th = CKDA_LDG(a.theta + g);
      lv = cf{al * cosf(th), al * sinf(th)};
    }
    cst(sm + Ly::Q + i * KS + 2 * c, qv);
    cst(sm + Ly::K + i * KS + 2 * c, kv);
    cst(sm + Ly::LM + i * KS + 2 * c, lv);
    if (e < C) be[e] = e < L ? CKDA_LDG(a.beta + (size_t)(t0 + e) * H + h) : 0.f;
  });
  par<DK>(x, [&](int c) {  // gamma (prefix products), sigma (suffix products)
    cf g{1.f, 0.f};
    for (int i = 0; i < C; ++i) {
      g = cmul(g, cld(sm + Ly::LM + i * KS + 2 * c));
      cst(sm + Ly::GM + i * KS + 2 * c, g);
    }
    g = cf{1.f, 0.f};
    for (int j = C - 1; j >= 0; --j) {
      cst(sm + Ly::SG + j * KS + 2 * c, g);
      g = cmul(g, cld(sm + Ly::LM + j * KS + 2 * c));
    }
  });
  // A (without beta) and M: item (pair, channel group g) sums channels g, g + NG, ...;
  // then the NG partials are added in a fixed order
  constexpr int NG = Ly::NG;
  par<C * C * NG>(x, [&](int e) {
    const int g = e % NG, p = e / NG, i = p / C, j = p - i * C;
    cf ak{0.f, 0.f}, m{0.f, 0.f};
    if (j <= i) {
      for (int c = g; c < DK; c += NG) {
        cf gp{1.f, 0.f};
        for (int s = j + 1; s <= i; ++s) gp = cmul(gp, cld(sm + Ly::LM + s * KS + 2 * c));
        const cf gk = cmul(gp, cld(sm + Ly::K + j * KS + 2 * c));
        ak = cadd(ak, cmulc(cld(sm + Ly::K + i * KS + 2 * c), gk));
        m = cadd(m, cmulc(cld(sm + Ly::Q + i * KS + 2 * c), gk));
      }
    }
    cst(sm + Ly::PG + 4 * e, ak);
    cst(sm + Ly::PG + 4 * e + 2, m);
  });
  par<C * C>(x, [&](int e) {
    const int i = e / C, j = e - i * C;
    cf ak{0.f, 0.f}, m{0.f, 0.f};
CKDA_UNROLL
    for (int g = 0; g < NG; ++g) {
      ak = cadd(ak, cld(sm + Ly::PG + 4 * (e * NG + g)));
      m = cadd(m, cld(sm + Ly::PG + 4 * (e * NG + g) + 2));
    }
    if (j >= i) ak = cf{0.f, 0.f};
    cst(sm + Ly::A + i * CS + 2 * j, ak);
    cst(sm + Ly::M + i * CS + 2 * j, m);
    w.mm[(((size_t)slot * H + h) * C * C + e) * 2] = m.r;
    w.mm[(((size_t)slot * H + h) * C * C + e) * 2 + 1] = m.i;
  });
  par<C>(x, [&](int j) {  // column j of T = (I + diag(beta) A)^-1
    float *tt = sm + Ly::TT;
    for (int i = 0; i < j; ++i) cst(tt + i * CS + 2 * j, cf{0.f, 0.f});
    cst(tt + j * CS + 2 * j, cf{1.f, 0.f});
    for (int i = j + 1; i < C; ++i) {
      cf s{0.f, 0.f};
      for (int m = j; m < i; ++m)
        s = cadd(s, cmul(cld(sm + Ly::A + i * CS + 2 * m), cld(tt + m * CS + 2 * j)));
      cst(tt + i * CS + 2 * j, cscale(-be[i], s));
    }
  });
  // W = T diag(beta) Khat, Kbar, Qhat; gamma_{C-1}
  par<C * DK>(x, [&](int e) {
    const int i = e / DK, c = e - i * DK;
    if (e < DK) {
      const cf g = cld(sm + Ly::GM + (C - 1) * KS + 2 * c);
      cst(w.gc + (((size_t)slot * H + h) * DK + c) * 2, g);
    }
    if (i >= L) return;
    cf wt{0.f, 0.f};
    for (int m = 0; m <= i; ++m) {
      const cf kh =
          cmul(cld(sm + Ly::GM + m * KS + 2 * c), cconj(cld(sm + Ly::K + m * KS + 2 * c)));
      wt = cadd(wt, cscale(be[m], cmul(cld(sm + Ly::TT + i * CS + 2 * m), kh)));
    }
    const size_t o = (((size_t)(t0 + i) * H + h) * DK + c) * 2;
    cst(w.wt + o, wt);
    cst(w.kb + o, cmul(cld(sm + Ly::SG + i * KS + 2 * c), cld(sm + Ly::K + i * KS + 2 * c)));
    cst(w.qh + o,
        cmul(cld(sm + Ly::GM + i * KS + 2 * c), cconj(cld(sm + Ly::Q + i * KS + 2 * c))));
  });
  // Utilde = T diag(beta) conj(V), one column tile at a time
  for (int c0 = 0; c0 < DVF; c0 += DVT) {
    par<C * DVT>(x, [&](int e) {
      const int i = e / DVT, v = e - i * DVT;
      const cf vv = i < L ? cldg(a.v + (((size_t)(t0 + i) * H + h) * DVF + c0 + v) * 2)
                          : cf{0.f, 0.f};
      cst(sm + Ly::V + i * VS + 2 * v, cconj(vv));
    });
    par<C * DVT>(x, [&](int e) {
      const int i = e / DVT, v = e - i * DVT;
      cf u{0.f, 0.f};
      for (int m = 0; m <= i; ++m)
        u = cadd(u, cscale(be[m], cmul(cld(sm + Ly::TT + i * CS + 2 * m),
                                       cld(sm + Ly::V + m * VS + 2 * v))));
      if (i < L) cst(w.ut + (((size_t)(t0 + i) * H + h) * DVF + c0 + v) * 2, u);
    });
  }
}

template <int DK, int DVT>
struct ScanLayout {
  static constexpr int KS = 2 * (DK + 1), VS = 2 * (DVT + 1), CS = 2 * (C + 1);
  // two sets of a chunk's factors (chunk i in set i & 1; chunk i + 1's
  // asynchronous copies land while chunk i is worked on, and are waited for
  // at chunk i + 1's start): C x DK complex W, Kbar, Qhat;
  // C x DVT complex Utilde (then U); C x C complex M; gamma_{C-1} [DK]
  // complex; offsets within a set
  static constexpr int WT = 0, KB = WT + C * KS, QH = KB + C * KS, UT = QH + C * KS,
                       M = UT + C * VS, GC = M + C * CS, SET = GC + 2 * DK;
  // DK x DVT complex state; the sets; partial products of W S and Qhat S (4
  // quarters of C x DVT complex each)
  static constexpr int S = 0, SETS = S + DK * VS, PW = SETS + 2 * SET, PQ = PW + 8 * C * DVT;
  static constexpr int FLOATS = PQ + 8 * C * DVT;
  static constexpr size_t BYTES = (size_t)FLOATS * sizeof(float);
};

template <class X, int DK, int DVT>
CKDA_PROG void scan_program(X &x, const Args &a, const Ws &w, float *sm, int h, int n, int tile,
                            int bos, int eos, int slot0) {
  using Ly = ScanLayout<DK, DVT>;
  constexpr int KS = Ly::KS, VS = Ly::VS, CS = Ly::CS, NV = DVT / 4;
  constexpr int NP = (C / 2) * NV * 4;                       // items of the W S, Qhat S pass
  constexpr int NL = DK * DVT > C * DK ? DK * DVT : C * DK;  // items of a load phase
  const int c0 = tile * DVT, H = a.H, DVF = a.DVF;
  const int nck = (eos - bos + C - 1) / C;
  const size_t st_base = ((size_t)n * H + h) * DK * DVF + c0;  // complex elements
  float *S = sm + Ly::S;
  const cf zero{0.f, 0.f};
  // one complex element (two floats) copied in the background
  auto acopy = [&](float *dst, const float *src) {
    x.acopy4(dst, src);
    x.acopy4(dst + 1, src + 1);
  };
  // item e of starting the copies of chunk ci's factors into set ci & 1
  // (rows past its end are written as zero at once)
  auto load = [&](int e, int ci) {
    float *f = sm + Ly::SETS + (ci & 1) * Ly::SET;
    const int t0 = bos + C * ci, L = eos - t0 < C ? eos - t0 : C;
    const size_t sl = (size_t)(slot0 + ci) * H + h;
    if (e < C * DK) {
      const int i = e / DK, c = e - i * DK;
      const size_t o = (((size_t)(t0 + i) * H + h) * DK + c) * 2;
      if (i < L) {
        acopy(f + Ly::WT + i * KS + 2 * c, w.wt + o);
        acopy(f + Ly::KB + i * KS + 2 * c, w.kb + o);
        acopy(f + Ly::QH + i * KS + 2 * c, w.qh + o);
      } else {
        cst(f + Ly::WT + i * KS + 2 * c, zero);
        cst(f + Ly::KB + i * KS + 2 * c, zero);
        cst(f + Ly::QH + i * KS + 2 * c, zero);
      }
    }
    if (e < C * DVT) {
      const int i = e / DVT, v = e - i * DVT;
      if (i < L)
        acopy(f + Ly::UT + i * VS + 2 * v, w.ut + (((size_t)(t0 + i) * H + h) * DVF + c0 + v) * 2);
      else
        cst(f + Ly::UT + i * VS + 2 * v, zero);
    }
    if (e < C * C) acopy(f + Ly::M + (e / C) * CS + 2 * (e % C), w.mm + (sl * C * C + e) * 2);
    if (e < DK) acopy(f + Ly::GC + 2 * e, w.gc + (sl * DK + e) * 2);
  };
  par<NL>(x, [&](int e) {  // the initial state; chunk 0's factors
    if (e < DK * DVT) {
      const int c = e / DVT, v = e - c * DVT;
      // plain load: the final state may overwrite the initial one in place
      const cf s = a.s0 ? cld(a.s0 + (st_base + (size_t)c * DVF + v) * 2) : zero;
      cst(S + c * VS + 2 * v, s);
    }
    if (nck > 0) load(e, 0);
  });
  x.commit();
  for (int ci = 0; ci < nck; ++ci) {
    const int t0 = bos + C * ci, L = eos - t0 < C ? eos - t0 : C;
    float *f = sm + Ly::SETS + (ci & 1) * Ly::SET;
    float *U = f + Ly::UT;
    x.template wait_copies<0>();  // chunk ci has landed
    // W S and Qhat S in one pass over S: item (row pair, 4 columns, quarter q)
    // sums channels q, q + 4, ... in 2 x 4 complex register tiles; chunk
    // ci + 1's factors load meanwhile
    par<NL>(x, [&](int e) {
      if (e < NP) {
        const int q = e % 4, rest = e / 4, vg = rest % NV, ip = rest / NV;
        const int i0 = 2 * ip, v0 = 4 * vg;
        cf aw[2][4], aq[2][4];
CKDA_UNROLL
        for (int r = 0; r < 2; ++r)
CKDA_UNROLL
          for (int j = 0; j < 4; ++j) aw[r][j] = aq[r][j] = zero;
        for (int c = q; c < DK; c += 4) {
          const cf w0 = cld(f + Ly::WT + i0 * KS + 2 * c);
          const cf w1 = cld(f + Ly::WT + (i0 + 1) * KS + 2 * c);
          const cf q0 = cld(f + Ly::QH + i0 * KS + 2 * c);
          const cf q1 = cld(f + Ly::QH + (i0 + 1) * KS + 2 * c);
CKDA_UNROLL
          for (int j = 0; j < 4; ++j) {
            const cf sv = cld(S + c * VS + 2 * (v0 + j));
            aw[0][j] = cadd(aw[0][j], cmul(w0, sv));
            aw[1][j] = cadd(aw[1][j], cmul(w1, sv));
            aq[0][j] = cadd(aq[0][j], cmul(q0, sv));
            aq[1][j] = cadd(aq[1][j], cmul(q1, sv));
          }
        }
CKDA_UNROLL
        for (int r = 0; r < 2; ++r)
CKDA_UNROLL
          for (int j = 0; j < 4; ++j) {
            cst(sm + Ly::PW + ((e * 2 + r) * 4 + j) * 2, aw[r][j]);
            cst(sm + Ly::PQ + ((e * 2 + r) * 4 + j) * 2, aq[r][j]);
          }
      }
      if (ci + 1 < nck) load(e, ci + 1);
    });
    x.commit();
    // the four quarters of (row i, column v) in a fixed order
    auto quarters = [&](int base, int i, int v) {
      const int e0 = (((i / 2) * NV + v / 4) * 4) * 2 + (i % 2), j = v % 4;
      cf s = zero;
CKDA_UNROLL
      for (int q4 = 0; q4 < 4; ++q4) s = cadd(s, cld(sm + base + ((e0 + 2 * q4) * 4 + j) * 2));
      return s;
    };
    par<C * DVT>(x, [&](int e) {  // U = Utilde - W S (rows past the end stay zero)
      const int i = e / DVT, v = e - i * DVT;
      if (i < L) cst(U + i * VS + 2 * v, csub(cld(U + i * VS + 2 * v), quarters(Ly::PW, i, v)));
    });
    par<C * DVT>(x, [&](int e) {  // o = conj(scale (Qhat S + M U))
      const int i = e / DVT, v = e - i * DVT;
      if (i >= L) return;
      cf s = quarters(Ly::PQ, i, v);
      for (int j = 0; j <= i; ++j)
        s = cadd(s, cmul(cld(f + Ly::M + i * CS + 2 * j), cld(U + j * VS + 2 * v)));
      cst(a.o + (((size_t)(t0 + i) * H + h) * DVF + c0 + v) * 2, cconj(cscale(a.scale, s)));
    });
    // S <- diag(gamma_{C-1}) S + Kbar^T U, in 2 x 4 complex register tiles
    par<(DK / 2) * NV>(x, [&](int e) {
      const int cg = e / NV, vg = e - cg * NV, cc = 2 * cg, v0 = 4 * vg;
      cf acc[2][4];
CKDA_UNROLL
      for (int r = 0; r < 2; ++r) {
        const cf g = cld(f + Ly::GC + 2 * (cc + r));
CKDA_UNROLL
        for (int j = 0; j < 4; ++j) acc[r][j] = cmul(g, cld(S + (cc + r) * VS + 2 * (v0 + j)));
      }
CKDA_UNROLL
      for (int i = 0; i < C; ++i) {
        const cf k0 = cld(f + Ly::KB + i * KS + 2 * cc);
        const cf k1 = cld(f + Ly::KB + i * KS + 2 * (cc + 1));
CKDA_UNROLL
        for (int j = 0; j < 4; ++j) {
          const cf uv = cld(U + i * VS + 2 * (v0 + j));
          acc[0][j] = cadd(acc[0][j], cmul(k0, uv));
          acc[1][j] = cadd(acc[1][j], cmul(k1, uv));
        }
      }
CKDA_UNROLL
      for (int r = 0; r < 2; ++r)
CKDA_UNROLL
        for (int j = 0; j < 4; ++j) cst(S + (cc + r) * VS + 2 * (v0 + j), acc[r][j]);
    });
  }
  if (a.sf) {
    par<DK * DVT>(x, [&](int e) {
      const int c = e / DVT, v = e - c * DVT;
      cst(a.sf + (st_base + (size_t)c * DVF + v) * 2, cld(S + c * VS + 2 * v));
    });
  }
}

}  // namespace cplx
}  // namespace ckda
