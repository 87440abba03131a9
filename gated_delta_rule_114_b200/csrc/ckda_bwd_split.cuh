// The chunkwise backward pass, split by what depends on the carried state.
//
// Built from the per-chunk pieces of ckda_bwd_chunk.cuh (the chunk-WY reverse
// of "Semidirect Fourier Delta Attention" §2.2 eqs. (9)-(10) in 16-token
// chunks): the work that does not depend on S or dS runs in CTAs of its own,
// in parallel over all chunks, and the two sequential scans keep only their
// state products. With T = (I + diag(beta) Abar)^-1 and per chunk
//   W = T diag(beta) Khat,  Utilde = T diag(beta) V,  Kbar = sigma * k,
//   Wb = T^T Kbar,  X = T^T (scale M^T dO),  Qs = scale Qhat,  BK = diag(beta) Khat,
// the forward over chunks is S <- diag(gamma_C) S + Kbar^T U with
// U = Utilde - W S, and the reverse is dR = X + Wb dS_C,
// dS <- diag(gamma_C) dS_C + Qs^T dO - BK^T dR. Four programs:
//   prep   (per chunk and head)            the factors above, Abar, gamma_C;
//   scan1  (per sequence, head, col. tile) entry states S per chunk, and U;
//   scan2  (per sequence, head, col. tile) exit-state gradients dS_C, and dR;
//   grads  (per chunk and head)            all gradients from (S, dS_C, U, dR).
// Per-chunk values (S, dS_C, gamma_C, Abar) sit in checkpoint slots
// (slot = floor(cu[n] / C) + n + chunk, at most floor(T_total / C) + N
// slots); per-token values in token-major [T_total, H, .] fp32 arrays.
#pragma once

#include "ckda_bwd_chunk.cuh"

namespace ckda {
namespace bwdc {

// Workspace arrays of the split form (all fp32).
struct SplitWs {
  float *cks, *ckd;              // [slots][H][DK][DVF]: S entering, dS leaving each chunk
  float *gc;                     // [slots][H][DK]: gamma over the whole chunk
  float *ab;                     // [slots][H][C][C]: Abar
  float *wt, *kb, *wb, *qs, *bk; // [T_total H][DK]: W, Kbar, Wb, Qs, BK
  float *ut, *xt, *uu, *dr;      // [T_total H][DVF]: Utilde, X, U, dR
};

// Sequence n and chunk ci of checkpoint slot g (slots of sequence n start at
// floor(start_n / C) + n); false when no sequence starts a chunk there.
CKDA_PROG bool slot_chunk(const int32_t *cu, int N, int T, int g, int &n, int &ci) {
  int lo = 0, hi = N - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) / 2;
    const int b = cu ? cu[mid] : mid * T;
    if (b / C + mid <= g) lo = mid; else hi = mid - 1;
  }
  const int b = cu ? cu[lo] : lo * T;
  n = lo;
  ci = g - (b / C + lo);
  return ci >= 0;
}

// Prep works on one (chunk, head) for all of d_v, one DVT tile of v and dO at a time.
template <int DK, int DVT>
struct PrepLayout {
  static constexpr int dk = DK, dvt = DVT;
  static constexpr int KS = DK + 1, VS = DVT + 1, CS = C + 1;
  static constexpr int Q = 0, K = Q + C * KS, AL = K + C * KS, GM = AL + C * KS,
                       SG = GM + C * KS;
  static constexpr int V = SG + C * KS, DO = V + C * VS, RD = DO + C * VS;
  static constexpr int AB = RD + C * VS, M = AB + C * CS, TT = M + C * CS;
  static constexpr int NG = 4;  // channel groups of the Gram phase
  static constexpr int PG = TT + C * CS, BE = PG + 2 * C * C * NG;
  static constexpr int FLOATS = BE + C;
  static constexpr size_t BYTES = (size_t)FLOATS * sizeof(float);
};

template <class X, class IOL, typename IOT, int DK, int DVT>
CKDA_PROG void prep_program(X &x, const Args<IOT> &a, const SplitWs &w, float *sm, int h,
                            int t0, int L, int slot) {
  using Ly = PrepLayout<DK, DVT>;
  constexpr int KS = Ly::KS, VS = Ly::VS, CS = Ly::CS;
  const int H = a.H, DVF = a.DVF;
  const float scale = a.scale;
  const float *be = sm + Ly::BE, *tt = sm + Ly::TT;
  stage<X, IOL, IOT, Ly>(x, a, sm, h, 0, t0, L, true);
  chunk_gates<X, Ly>(x, sm);
  chunk_grams_solve<X, Ly>(x, sm);
  // the d_k-wide factors, gamma_C and Abar
  par<C * DK>(x, [&](int e) {
    const int i = e / DK, c = e - i * DK;
    if (e < DK) w.gc[((size_t)slot * H + h) * DK + c] = sm[Ly::GM + (C - 1) * KS + c];
    if (e < C * C) w.ab[((size_t)slot * H + h) * C * C + e] = sm[Ly::AB + (e / C) * CS + e % C];
    if (i >= L) return;
    float wt = 0.f, wb = 0.f;
    for (int m = 0; m <= i; ++m)
      wt += tt[i * CS + m] * be[m] * sm[Ly::GM + m * KS + c] * sm[Ly::K + m * KS + c];
    for (int j = i; j < C; ++j)
      wb += tt[j * CS + i] * sm[Ly::SG + j * KS + c] * sm[Ly::K + j * KS + c];
    const float gm = sm[Ly::GM + i * KS + c], kc = sm[Ly::K + i * KS + c];
    const size_t o = ((size_t)(t0 + i) * H + h) * DK + c;
    w.wt[o] = wt;
    w.kb[o] = sm[Ly::SG + i * KS + c] * kc;
    w.wb[o] = wb;
    w.qs[o] = scale * gm * sm[Ly::Q + i * KS + c];
    w.bk[o] = be[i] * gm * kc;
  });
  // Utilde = T diag(beta) V and X = T^T (scale M^T dO), one column tile at a time
  for (int c0 = 0; c0 < DVF; c0 += DVT) {
    if (c0 > 0) {
      par<C * DVT>(x, [&](int e) {
        const int i = e / DVT, v = e - i * DVT;
        float vv = 0.f, dd = 0.f;
        if (i < L) {
          const size_t g = ((size_t)(t0 + i) * H + h) * DVF + c0 + v;
          vv = IOL::ldg(a.v + g);
          dd = IOL::ldg(a.d_o + g);
        }
        sm[Ly::V + i * VS + v] = vv;
        sm[Ly::DO + i * VS + v] = dd;
      });
    }
    par<C * DVT>(x, [&](int e) {  // Utilde; Y = scale M^T dO into the R rows
      const int i = e / DVT, v = e - i * DVT;
      float u = 0.f, y = 0.f;
      for (int m = 0; m <= i; ++m) u += tt[i * CS + m] * be[m] * sm[Ly::V + m * VS + v];
      for (int l = i; l < C; ++l) y += sm[Ly::M + l * CS + i] * sm[Ly::DO + l * VS + v];
      sm[Ly::RD + i * VS + v] = scale * y;
      if (i < L) w.ut[((size_t)(t0 + i) * H + h) * DVF + c0 + v] = u;
    });
    par<C * DVT>(x, [&](int e) {  // X = T^T Y
      const int j = e / DVT, v = e - j * DVT;
      float s = 0.f;
      for (int i = j; i < C; ++i) s += tt[i * CS + j] * sm[Ly::RD + i * VS + v];
      if (j < L) w.xt[((size_t)(t0 + j) * H + h) * DVF + c0 + v] = s;
    });
  }
}

// Shared memory of the two scans: one state (or state gradient) tile and the
// chunks' per-token factors.
template <int DK, int DVT>
struct ScanLayout {
  static constexpr int KS = DK + 1, VS = DVT + 1;
  // three sets of a chunk's factors: the k-th chunk a scan visits sits in set
  // k % 3, its copies started two chunks ahead (asynchronous copies, waited
  // for at the chunk's start), so their latency overlaps two chunks' work.
  // Per set: three C x DK, two C x DVT, gamma_C, and the raw I/O-type pairs of
  // a C x DVT tile (dO in bf16, converted in place once it has landed);
  // offsets within a set
  static constexpr int F0 = 0, F1 = F0 + C * KS, F2 = F1 + C * KS, R0 = F2 + C * KS,
                       R1 = R0 + C * VS, GC = R1 + C * VS, RAW = GC + DK,
                       SET = RAW + C * DVT / 2;
  static constexpr int NSETS = 3;
  static constexpr int S = 0, SETS = S + DK * VS;
  static constexpr int P = SETS + NSETS * SET;  // partial products, C x DVT x 4
  static constexpr int FLOATS = P + 4 * C * DVT;
  static constexpr size_t BYTES = (size_t)FLOATS * sizeof(float);
};

// Partial products of the C x DVT result A B (A: C x DK rows of stride DK + 1;
// B: the DK x DVT state tile, rows of stride DVT + 1): item e (row pair, 4
// columns, quarter q; PartialItems of them) sums channels q, q + 4, ... in
// a 2 x 4 register tile into P; rows_state_sum adds the quarters in order.
template <int DK, int DVT>
CKDA_PROG void rows_state_partial_item(int e, float *P, const float *A, const float *B) {
  constexpr int KS = DK + 1, VS = DVT + 1, NV = DVT / 4;
  {
    const int q = e % 4, rest = e / 4, vg = rest % NV, ip = rest / NV;
    const int i0 = 2 * ip, v0 = 4 * vg;
    float acc[2][4] = {};
    for (int c = q; c < DK; c += 4) {
      const float a0 = A[i0 * KS + c], a1 = A[(i0 + 1) * KS + c];
CKDA_UNROLL
      for (int j = 0; j < 4; ++j) {
        const float b = B[c * VS + v0 + j];
        acc[0][j] += a0 * b;
        acc[1][j] += a1 * b;
      }
    }
CKDA_UNROLL
    for (int r = 0; r < 2; ++r)
CKDA_UNROLL
      for (int j = 0; j < 4; ++j) P[(e * 2 + r) * 4 + j] = acc[r][j];
  }
}

// items of rows_state_partial_item
template <int DVT>
struct PartialItems {
  static constexpr int value = (C / 2) * (DVT / 4) * 4;
};

// (A B)[i][v] from the partial products of rows_state_partial_item
template <int DVT>
CKDA_PROG float rows_state_sum(const float *P, int i, int v) {
  constexpr int NV = DVT / 4;
  const int e0 = (((i / 2) * NV + v / 4) * 4) * 2 + (i % 2), j = v % 4;
  float s = 0.f;
CKDA_UNROLL
  for (int q = 0; q < 4; ++q) s += P[(e0 + 2 * q) * 4 + j];
  return s;
}

// The scans' state update over one chunk, in 4 x 4 register tiles (each item
// owns rows 4cg..4cg+3 and columns 4vg..4vg+3 of the d_k x DVT tile):
//   Z[c][v] <- g[c] Z[c][v] + sum_i A[i][c] B[i][v]   (minus sum_i A2[i][c] B2[i][v]
// when A2 is given), rows of A, A2 with stride KS and of B, B2 and Z with stride VS.
template <int DK, int DVT, class X>
CKDA_PROG void state_update(X &x, float *Z, const float *g, const float *A, const float *B,
                            const float *A2, const float *B2) {
  constexpr int KS = DK + 1, VS = DVT + 1, NV = DVT / 4;
  static_assert(DK % 4 == 0 && DVT % 4 == 0, "4 x 4 tiles");
  par<(DK / 4) * NV>(x, [&](int e) {
    const int c0 = 4 * (e / NV), v0 = 4 * (e % NV);
    float acc[4][4];
CKDA_UNROLL
    for (int r = 0; r < 4; ++r)
CKDA_UNROLL
      for (int j = 0; j < 4; ++j) acc[r][j] = g[c0 + r] * Z[(c0 + r) * VS + v0 + j];
CKDA_UNROLL
    for (int i = 0; i < C; ++i) {
      float av[4], bv[4];
CKDA_UNROLL
      for (int r = 0; r < 4; ++r) av[r] = A[i * KS + c0 + r];
CKDA_UNROLL
      for (int j = 0; j < 4; ++j) bv[j] = B[i * VS + v0 + j];
CKDA_UNROLL
      for (int r = 0; r < 4; ++r)
CKDA_UNROLL
        for (int j = 0; j < 4; ++j) acc[r][j] += av[r] * bv[j];
      if (A2) {
CKDA_UNROLL
        for (int r = 0; r < 4; ++r) av[r] = A2[i * KS + c0 + r];
CKDA_UNROLL
        for (int j = 0; j < 4; ++j) bv[j] = B2[i * VS + v0 + j];
CKDA_UNROLL
        for (int r = 0; r < 4; ++r)
CKDA_UNROLL
          for (int j = 0; j < 4; ++j) acc[r][j] -= av[r] * bv[j];
      }
    }
CKDA_UNROLL
    for (int r = 0; r < 4; ++r)
CKDA_UNROLL
      for (int j = 0; j < 4; ++j) Z[(c0 + r) * VS + v0 + j] = acc[r][j];
  });
}

template <class X, class IOL, typename IOT, int DK, int DVT>
CKDA_PROG void scan1_program(X &x, const Args<IOT> &a, const SplitWs &w, float *sm, int h,
                             int n, int tile, int bos, int eos, int slot0) {
  using Ly = ScanLayout<DK, DVT>;
  constexpr int KS = Ly::KS, VS = Ly::VS, NP = PartialItems<DVT>::value;
  constexpr int NL = DK * DVT > C * DK ? DK * DVT : C * DK;  // items of a load phase
  const int c0 = tile * DVT, H = a.H, DVF = a.DVF;
  const int nck = (eos - bos + C - 1) / C;
  const size_t st_base = ((size_t)n * H + h) * DK * DVF + c0;
  float *S = sm + Ly::S;
  // item e of starting the copies of chunk ci's W, Kbar, Utilde and gamma_C
  // into set ci % 3 (rows past its end are written as zero at once)
  auto load = [&](int e, int ci) {
    if (ci >= nck) return;
    float *f = sm + Ly::SETS + (ci % Ly::NSETS) * Ly::SET;
    const int t0 = bos + C * ci, L = eos - t0 < C ? eos - t0 : C;
    if (e < C * DK) {
      const int i = e / DK, c = e - i * DK;
      const size_t o = ((size_t)(t0 + i) * H + h) * DK + c;
      if (i < L) {
        x.acopy4(f + Ly::F0 + i * KS + c, w.wt + o);
        x.acopy4(f + Ly::F1 + i * KS + c, w.kb + o);
      } else {
        f[Ly::F0 + i * KS + c] = 0.f;
        f[Ly::F1 + i * KS + c] = 0.f;
      }
    }
    if (e < C * DVT) {
      const int i = e / DVT, v = e - i * DVT;
      if (i < L)
        x.acopy4(f + Ly::R0 + i * VS + v, w.ut + ((size_t)(t0 + i) * H + h) * DVF + c0 + v);
      else
        f[Ly::R0 + i * VS + v] = 0.f;
    }
    if (e < DK) x.acopy4(f + Ly::GC + e, w.gc + ((size_t)(slot0 + ci) * H + h) * DK + e);
  };
  par<NL>(x, [&](int e) {  // the initial state; chunks 0 and 1 start coming in
    if (e < DK * DVT) {
      const int c = e / DVT, v = e - c * DVT;
      S[c * VS + v] = a.s0 ? a.s0[st_base + (size_t)c * DVF + v] : 0.f;
    }
    load(e, 0);
    load(e, 1);
  });
  x.commit();
  for (int ci = 0; ci < nck; ++ci) {
    const int t0 = bos + C * ci, L = eos - t0 < C ? eos - t0 : C;
    const size_t slot = (size_t)(slot0 + ci) * H + h;
    float *f = sm + Ly::SETS + (ci % Ly::NSETS) * Ly::SET;
    float *WT = f + Ly::F0, *KB = f + Ly::F1, *U = f + Ly::R0, *GC = f + Ly::GC;
    // chunk ci has landed (only chunk ci + 1's group may still be in flight)
    if (ci == 0) x.template wait_copies<0>();
    else x.template wait_copies<1>();
    // checkpoint S; the partial products of W S; chunk ci + 2's copies start
    par<NL>(x, [&](int e) {
      if (e < DK * DVT) {
        const int c = e / DVT, v = e - c * DVT;
        w.cks[slot * DK * DVF + (size_t)c * DVF + c0 + v] = S[c * VS + v];
      }
      if (e < NP) rows_state_partial_item<DK, DVT>(e, sm + Ly::P, WT, S);
      load(e, ci + 2);
    });
    x.commit();
    par<C * DVT>(x, [&](int e) {  // U = Utilde - W S
      const int i = e / DVT, v = e - i * DVT;
      const float s = U[i * VS + v] - rows_state_sum<DVT>(sm + Ly::P, i, v);
      U[i * VS + v] = s;
      if (i < L) w.uu[((size_t)(t0 + i) * H + h) * DVF + c0 + v] = s;
    });
    // S <- diag(gamma_C) S + Kbar^T U
    state_update<DK, DVT>(x, S, GC, KB, U, nullptr, nullptr);
  }
}

template <class X, class IOL, typename IOT, int DK, int DVT>
CKDA_PROG void scan2_program(X &x, const Args<IOT> &a, const SplitWs &w, float *sm, int h,
                             int n, int tile, int bos, int eos, int slot0) {
  using Ly = ScanLayout<DK, DVT>;
  constexpr int KS = Ly::KS, VS = Ly::VS, NP = PartialItems<DVT>::value;
  constexpr int NL = DK * DVT > C * DK ? DK * DVT : C * DK;  // items of a load phase
  constexpr bool RAW_DO = sizeof(IOT) != sizeof(float);  // dO arrives as bf16 pairs
  const int c0 = tile * DVT, H = a.H, DVF = a.DVF;
  const int nck = (eos - bos + C - 1) / C;
  const size_t st_base = ((size_t)n * H + h) * DK * DVF + c0;
  float *DS = sm + Ly::S;
  // item e of starting the copies of the k-th chunk from the end (chunk
  // nck - 1 - k): Wb, Qs, BK, X, dO and gamma_C into set k % 3 (rows past its
  // end are written as zero at once)
  auto load = [&](int e, int k) {
    if (k >= nck) return;
    const int ci = nck - 1 - k;
    float *f = sm + Ly::SETS + (k % Ly::NSETS) * Ly::SET;
    const int t0 = bos + C * ci, L = eos - t0 < C ? eos - t0 : C;
    if (e < C * DK) {
      const int i = e / DK, c = e - i * DK;
      const size_t o = ((size_t)(t0 + i) * H + h) * DK + c;
      if (i < L) {
        x.acopy4(f + Ly::F0 + i * KS + c, w.wb + o);
        x.acopy4(f + Ly::F1 + i * KS + c, w.qs + o);
        x.acopy4(f + Ly::F2 + i * KS + c, w.bk + o);
      } else {
        f[Ly::F0 + i * KS + c] = 0.f;
        f[Ly::F1 + i * KS + c] = 0.f;
        f[Ly::F2 + i * KS + c] = 0.f;
      }
    }
    if (e < C * DVT) {
      const int i = e / DVT, v = e - i * DVT;
      const size_t o = ((size_t)(t0 + i) * H + h) * DVF + c0 + v;
      if (i < L) {
        x.acopy4(f + Ly::R0 + i * VS + v, w.xt + o);
        if constexpr (RAW_DO) {  // a pair of bf16 per 4-byte copy
          if ((v & 1) == 0)
            x.acopy4(f + Ly::RAW + i * (DVT / 2) + v / 2, reinterpret_cast<const float *>(a.d_o + o));
        } else {
          x.acopy4(f + Ly::R1 + i * VS + v, reinterpret_cast<const float *>(a.d_o + o));
        }
      } else {
        f[Ly::R0 + i * VS + v] = 0.f;
        f[Ly::R1 + i * VS + v] = 0.f;
        if constexpr (RAW_DO) if ((v & 1) == 0) f[Ly::RAW + i * (DVT / 2) + v / 2] = 0.f;
      }
    }
    if (e < DK) x.acopy4(f + Ly::GC + e, w.gc + ((size_t)(slot0 + ci) * H + h) * DK + e);
  };
  par<NL>(x, [&](int e) {  // the final-state gradient; the last two chunks start coming in
    if (e < DK * DVT) {
      const int c = e / DVT, v = e - c * DVT;
      DS[c * VS + v] = a.dsf ? a.dsf[st_base + (size_t)c * DVF + v] : 0.f;
    }
    load(e, 0);
    load(e, 1);
  });
  x.commit();
  for (int k = 0; k < nck; ++k) {
    const int ci = nck - 1 - k;
    const int t0 = bos + C * ci, L = eos - t0 < C ? eos - t0 : C;
    const size_t slot = (size_t)(slot0 + ci) * H + h;
    float *f = sm + Ly::SETS + (k % Ly::NSETS) * Ly::SET;
    float *WB = f + Ly::F0, *QS = f + Ly::F1, *BK = f + Ly::F2, *DR = f + Ly::R0,
          *DO = f + Ly::R1, *GC = f + Ly::GC;
    // this chunk has landed (only the next one's group may still be in flight)
    if (k == 0) x.template wait_copies<0>();
    else x.template wait_copies<1>();
    // checkpoint dS_C; the partial products of Wb dS_C; the copies of the
    // chunk two ahead start
    par<NL>(x, [&](int e) {
      if (e < DK * DVT) {
        const int c = e / DVT, v = e - c * DVT;
        w.ckd[slot * DK * DVF + (size_t)c * DVF + c0 + v] = DS[c * VS + v];
      }
      if (e < NP) rows_state_partial_item<DK, DVT>(e, sm + Ly::P, WB, DS);
      load(e, k + 2);
    });
    x.commit();
    par<C * DVT>(x, [&](int e) {  // dR = X + Wb dS_C; dO to fp32 (bf16 pairs)
      const int j = e / DVT, v = e - j * DVT;
      const float s = DR[j * VS + v] + rows_state_sum<DVT>(sm + Ly::P, j, v);
      DR[j * VS + v] = s;
      if (j < L) w.dr[((size_t)(t0 + j) * H + h) * DVF + c0 + v] = s;
      if constexpr (RAW_DO) {
        const float pair = f[Ly::RAW + j * (DVT / 2) + v / 2];
        DO[j * VS + v] = IOL::pair_half(pair, v & 1);
      }
    });
    // dS <- diag(gamma_C) dS_C + Qs^T dO - BK^T dR
    state_update<DK, DVT>(x, DS, GC, QS, DO, BK, DR);
  }
  if (a.ds0) {
    par<DK * DVT>(x, [&](int e) {
      const int c = e / DVT, v = e - c * DVT;
      a.ds0[st_base + (size_t)c * DVF + v] = DS[c * VS + v];
    });
  }
}

// Shared memory of the gradient program: one (chunk, head), the columns in
// tiles of GT. Rows are padded to an odd stride so that a warp reading down a
// column, or along rows indexed by its lanes, touches distinct banks.
template <int DK, int GT>
struct GradLayout {
  static constexpr int dk = DK, dvt = GT;
  static constexpr int KS = DK + 1, VS = GT + 1, CS = C + 1;
  // C x DK: q, k, alpha; gamma, sigma; the column sums of dO S^T, dR S^T and
  // U dS_C^T, overwritten by the gate-gradient coefficients E0 (over XQ) and
  // EX (over XB)
  static constexpr int Q = 0, K = Q + C * KS, AL = K + C * KS, GM = AL + C * KS,
                       SG = GM + C * KS, XQ = SG + C * KS, XK = XQ + C * KS, XB = XK + C * KS,
                       KH = XB + C * KS;  // KH: Khat = gamma * k
  static constexpr int E0 = XQ, EX = XB;
  // C x GT: v, dO, Khat S then w, U, dR of the current column tile
  static constexpr int V = KH + C * KS, DO = V + C * VS, KSW = DO + C * VS, U = KSW + C * VS,
                       DR = U + C * VS;
  // DK x GT: the tile of the entry state and of the exit-state gradient
  static constexpr int S = DR + C * VS, DS = S + DK * VS;
  // C x C: Abar, dM and dAbar (summed over the tiles)
  static constexpr int AB = DS + DK * VS, DM = AB + C * CS, DA = DM + C * CS;
  // beta [C], dbeta [C], sum_v S dS_C per channel [DK]; partial products of Khat S
  static constexpr int BE = DA + C * CS, DB = BE + C, SDS = DB + C, P = SDS + DK;
  static constexpr int FLOATS = P + 4 * C * GT;
  static constexpr size_t BYTES = (size_t)FLOATS * sizeof(float);
};

// The gradients of one (chunk, head) from the scans' outputs (S, dS_C, U, dR
// per chunk). dv is written tile by tile; everything that sums over the
// columns (dM, dAbar, dbeta and the state-side terms of dq, dk, dalpha)
// accumulates over the column tiles in a fixed order, then dq, dk (with the
// gated Gram terms), dalpha and dbeta are written once.
template <class X, class IOL, typename IOT, int DK, int GT>
CKDA_PROG void grads_program(X &x, const Args<IOT> &a, const SplitWs &w, float *sm, int h,
                             int t0, int L, int slot) {
  using Ly = GradLayout<DK, GT>;
  constexpr int KS = Ly::KS, VS = Ly::VS, CS = Ly::CS, NQ = DK / 4;
  const int H = a.H, DVF = a.DVF;
  const float scale = a.scale;
  const size_t sl = (size_t)slot * H + h;
  const float *be = sm + Ly::BE;
  const float *al = sm + Ly::AL, *kk = sm + Ly::K, *qq = sm + Ly::Q;
  // q, k, alpha, beta (rows L..C-1 inert); zero the sums; Abar
  par<C * DK>(x, [&](int e) {
    const int i = e / DK, c = e - i * DK;
    float qv = 0.f, kv = 0.f, av = 1.f;
    if (i < L) {
      const size_t g = ((size_t)(t0 + i) * H + h) * DK + c;
      qv = IOL::ldg(a.q + g);
      kv = IOL::ldg(a.k + g);
      av = CKDA_LDG(a.alpha + g);
    }
    sm[Ly::Q + i * KS + c] = qv;
    sm[Ly::K + i * KS + c] = kv;
    sm[Ly::AL + i * KS + c] = av;
    sm[Ly::XQ + i * KS + c] = 0.f;
    sm[Ly::XK + i * KS + c] = 0.f;
    sm[Ly::XB + i * KS + c] = 0.f;
    if (e < C * C) {
      sm[Ly::AB + (e / C) * CS + e % C] = CKDA_LDG(w.ab + sl * C * C + e);
      sm[Ly::DM + (e / C) * CS + e % C] = 0.f;
      sm[Ly::DA + (e / C) * CS + e % C] = 0.f;
    }
    if (e < C) {
      sm[Ly::BE + e] = e < L ? CKDA_LDG(a.beta + (size_t)(t0 + e) * H + h) : 0.f;
      sm[Ly::DB + e] = 0.f;
    }
    if (e < DK) sm[Ly::SDS + e] = 0.f;
  });
  chunk_gates<X, Ly>(x, sm);
  par<C * DK>(x, [&](int e) {  // Khat = gamma * k
    const int i = e / DK, c = e - i * DK;
    sm[Ly::KH + i * KS + c] = sm[Ly::GM + i * KS + c] * kk[i * KS + c];
  });
  for (int c0 = 0; c0 < DVF; c0 += GT) {
    // the tile's S, dS_C and rows of U, dR, v, dO (rows L..C-1 zero)
    par<DK * GT>(x, [&](int e) {
      const int c = e / GT, v = e - c * GT;
      const size_t o = sl * DK * DVF + (size_t)c * DVF + c0 + v;
      sm[Ly::S + c * VS + v] = CKDA_LDG(w.cks + o);
      sm[Ly::DS + c * VS + v] = CKDA_LDG(w.ckd + o);
      if (e < C * GT) {
        const int i = e / GT, u = e - i * GT;
        const bool in = i < L;
        const size_t r = ((size_t)(t0 + i) * H + h) * DVF + c0 + u;
        sm[Ly::U + i * VS + u] = in ? CKDA_LDG(w.uu + r) : 0.f;
        sm[Ly::DR + i * VS + u] = in ? CKDA_LDG(w.dr + r) : 0.f;
        sm[Ly::V + i * VS + u] = in ? IOL::ldg(a.v + r) : 0.f;
        sm[Ly::DO + i * VS + u] = in ? IOL::ldg(a.d_o + r) : 0.f;
      }
    });
    // Khat S in 2 x 4 register tiles (split d_k sums); then
    // w = V - Khat S - Abar U (into the Khat S rows) and dv = diag(beta) dR
    par<PartialItems<GT>::value>(
        x, [&](int e) { rows_state_partial_item<DK, GT>(e, sm + Ly::P, sm + Ly::KH, sm + Ly::S); });
    par<C * GT>(x, [&](int e) {
      const int i = e / GT, v = e - i * GT;
      float s = rows_state_sum<GT>(sm + Ly::P, i, v);
      for (int m = 0; m < i; ++m) s += sm[Ly::AB + i * CS + m] * sm[Ly::U + m * VS + v];
      sm[Ly::KSW + i * VS + v] = sm[Ly::V + i * VS + v] - s;
      if (i < L)
        IOL::st(a.dv + ((size_t)(t0 + i) * H + h) * DVF + c0 + v, be[i] * sm[Ly::DR + i * VS + v]);
    });
    // the tile's share of dO U^T, dR U^T and dR . w
    par<C * C>(x, [&](int e) {
      const int i = e / C, j = e - i * C;
      if (j == 0) {
        float s = 0.f;
        for (int v = 0; v < GT; ++v) s += sm[Ly::DR + i * VS + v] * sm[Ly::KSW + i * VS + v];
        sm[Ly::DB + i] += s;
      }
      if (j <= i) {
        float m = 0.f, d = 0.f;
        for (int v = 0; v < GT; ++v) {
          const float u = sm[Ly::U + j * VS + v];
          m += sm[Ly::DO + i * VS + v] * u;
          d += sm[Ly::DR + i * VS + v] * u;
        }
        sm[Ly::DM + i * CS + j] += m;
        sm[Ly::DA + i * CS + j] += d;
      }
    });
    // the tile's share of dO S^T, dR S^T, U dS_C^T and of sum_v S dS_C, per
    // (rows 2rp, 2rp + 1; channels cq + t DK/4): each S, dS_C load serves both rows
    par<(C / 2) * NQ>(x, [&](int e) {
      const int rp = e / NQ, cq = e - rp * NQ, r0 = 2 * rp;
      float xq[2][4] = {}, xk[2][4] = {}, xb[2][4] = {}, sd[4] = {};
      for (int v = 0; v < GT; ++v) {
        float dov[2], drv[2], uv[2];
CKDA_UNROLL
        for (int r = 0; r < 2; ++r) {
          dov[r] = sm[Ly::DO + (r0 + r) * VS + v];
          drv[r] = sm[Ly::DR + (r0 + r) * VS + v];
          uv[r] = sm[Ly::U + (r0 + r) * VS + v];
        }
CKDA_UNROLL
        for (int t = 0; t < 4; ++t) {
          const int c = cq + t * NQ;
          const float sv = sm[Ly::S + c * VS + v], dsv = sm[Ly::DS + c * VS + v];
CKDA_UNROLL
          for (int r = 0; r < 2; ++r) {
            xq[r][t] += dov[r] * sv;
            xk[r][t] += drv[r] * sv;
            xb[r][t] += uv[r] * dsv;
          }
          sd[t] += sv * dsv;
        }
      }
CKDA_UNROLL
      for (int t = 0; t < 4; ++t) {
        const int c = cq + t * NQ;
CKDA_UNROLL
        for (int r = 0; r < 2; ++r) {
          sm[Ly::XQ + (r0 + r) * KS + c] += xq[r][t];
          sm[Ly::XK + (r0 + r) * KS + c] += xk[r][t];
          sm[Ly::XB + (r0 + r) * KS + c] += xb[r][t];
        }
        if (rp == 0) sm[Ly::SDS + c] += sd[t];
      }
    });
  }
  // dM = scale dO U^T (j <= i), dAbar = -diag(beta) dR U^T (j < i)
  par<C * C>(x, [&](int e) {
    const int i = e / C, j = e - i * C;
    sm[Ly::DM + i * CS + j] *= scale;
    sm[Ly::DA + i * CS + j] = j < i ? -be[i] * sm[Ly::DA + i * CS + j] : 0.f;
  });
  // per (row r, channels cq + t DK/4): dQhat = scale (dO S^T), dKhat =
  // -diag(beta) (dR S^T), dKbar = U dS_C^T; E0, EX over their sums; dq and dk
  // with the gated Gram terms, written once
  par<C * NQ>(x, [&](int e) {
    const int r = e / NQ, cq = e - r * NQ;
    float dq[4], dk[4];
    const float dmrr = sm[Ly::DM + r * CS + r];
CKDA_UNROLL
    for (int t = 0; t < 4; ++t) {
      const int c = cq + t * NQ;
      const float dqh = scale * sm[Ly::XQ + r * KS + c], dkh = -be[r] * sm[Ly::XK + r * KS + c];
      const float xb = sm[Ly::XB + r * KS + c];
      const float gm = sm[Ly::GM + r * KS + c], sg = sm[Ly::SG + r * KS + c];
      sm[Ly::E0 + r * KS + c] = qq[r * KS + c] * dqh + kk[r * KS + c] * dkh;
      sm[Ly::EX + r * KS + c] = kk[r * KS + c] * xb;
      dq[t] = gm * dqh + dmrr * kk[r * KS + c];
      dk[t] = gm * dkh + sg * xb;
    }
    float g[4] = {1.f, 1.f, 1.f, 1.f};  // G_{r<-j} per channel
    for (int j = r - 1; j >= 0; --j) {
      const float dm = sm[Ly::DM + r * CS + j], da = sm[Ly::DA + r * CS + j];
CKDA_UNROLL
      for (int t = 0; t < 4; ++t) {
        const int c = cq + t * NQ;
        g[t] *= al[(j + 1) * KS + c];
        const float gk = g[t] * kk[j * KS + c];
        dq[t] += dm * gk;
        dk[t] += da * gk;
      }
    }
CKDA_UNROLL
    for (int t = 0; t < 4; ++t) g[t] = 1.f;  // G_{i<-r} per channel
    for (int i = r; i < C; ++i) {
      const float dm = sm[Ly::DM + i * CS + r], da = sm[Ly::DA + i * CS + r];
CKDA_UNROLL
      for (int t = 0; t < 4; ++t) {
        const int c = cq + t * NQ;
        if (i > r) g[t] *= al[i * KS + c];
        dk[t] += g[t] * (dm * qq[i * KS + c] + da * kk[i * KS + c]);
      }
    }
    if (r < L) {
      const size_t o = ((size_t)(t0 + r) * H + h) * DK;
CKDA_UNROLL
      for (int t = 0; t < 4; ++t) {
        IOL::st(a.dq + o + cq + t * NQ, dq[t]);
        IOL::st(a.dk + o + cq + t * NQ, dk[t]);
      }
    }
  });
  // dalpha, one channel per item; dbeta
  par<DK>(x, [&](int c) {
    float da[C];
    gate_grad_channel<Ly>(sm, c, sm[Ly::SDS + c], da);
CKDA_UNROLL
    for (int i = 0; i < C; ++i)  // static indices keep da in registers
      if (i < L) a.dalpha[((size_t)(t0 + i) * H + h) * DK + c] = da[i];
    if (c < L) a.dbeta[(size_t)(t0 + c) * H + h] = sm[Ly::DB + c];
  });
}

}  // namespace bwdc
}  // namespace ckda
