// The chunkwise backward pass of the CKDA recurrence: per-chunk pieces.
//
// Forward of one chunk of C tokens (rows i, j in 0..C-1; entry state S;
// G_{i<-j} = prod_{s=j+1..i} diag(alpha_s); gamma_i = G_{i<-(-1)} the prefix
// product; sigma_j = G_{C-1<-j} the suffix product; A = diag(beta) Abar):
//   Abar_ij = k_i^T G_{i<-j} k_j (j < i),   M_ij = q_i^T G_{i<-j} k_j (j <= i)
//   T = (I + A)^-1,  U = T diag(beta) (V - Khat S),  Khat_i = gamma_i * k_i
//   O = scale (Qhat S + M U),  S_C = diag(gamma_{C-1}) S + Kbar^T U,
// the chunk-WY / UT form of "Semidirect Fourier Delta Attention" §2.2
// eqs. (9)-(10). Its reverse, given dO and dS_C (the exit-state gradient):
//   dU = scale M^T dO + Kbar dS_C,   dR = T^T dU,   dv = diag(beta) dR
//   dS = scale Qhat^T dO + diag(gamma_{C-1}) dS_C - Khat^T diag(beta) dR
//   dbeta_i = dR_i . (V - Khat S - Abar U)_i
//   dM = scale dO U^T (j <= i),  dAbar = -diag(beta) dR U^T (j < i)
//   dq_i = scale gamma_i * (S dO_i) + sum_j dM_ij G_{i<-j} k_j
//   dk   = gamma * dKhat + sigma * dKbar + the gated Gram terms of M and Abar
// and, for the gates, every alpha_{s,c} sits in products G_{i<-j,c} with
// j < s <= i (j = the chunk entry for gamma, i = the chunk exit for sigma):
//   dalpha_{s,c} = sum_{j < s <= i} E_{ij,c} G_{s-1<-j,c} G_{i<-s,c},
// E_{ij,c} the coefficient of G_{i<-j,c}, evaluated per channel with two
// running products and no division, so zero and negative gates need nothing
// special. Only dS crosses chunks.
//
// This file holds the pieces one chunk needs (staging, gate products, Grams
// and the UT solve, the per-channel gate gradient); ckda_bwd_split.cuh
// composes them into the four programs of the backward. The columns of S and
// dS are independent; everything that sums over columns (dq, dk, dalpha,
// dbeta) is linear in per-column terms, so the gradient program adds the
// column tiles of one chunk in a fixed order.
//
// Every program is a fixed sequence of data-parallel phases. par<N>(x, f)
// runs one phase on executor X: f(i) for every i in [0, N), the calls
// independent of one another, then a barrier. Every value that outlives a
// phase sits in the shared-memory block `sm` (or in global memory), so the
// same source runs as a CUDA kernel (threads stride over i, __syncthreads
// between phases) and, for tests, as plain host loops. Gate products inside a 16-token chunk are
// short running products (at most 15 factors), so every factor keeps its sign
// and its zeros exactly. fp32 throughout.
#pragma once

#include <stddef.h>
#include <stdint.h>

#ifndef CKDA_PROG
#ifdef __CUDACC__
#define CKDA_PROG __device__ __forceinline__
#define CKDA_UNROLL _Pragma("unroll")
#define CKDA_LDG(p) __ldg(p)
#else
#define CKDA_PROG inline
#define CKDA_UNROLL
#define CKDA_LDG(p) (*(p))
#endif
#endif


namespace ckda {
namespace bwdc {

constexpr int C = 16;  // tokens per chunk

// One phase: f(i) for every i in [0, N), the calls independent of one
// another, then a barrier. N is a compile-time count so that a CUDA thread
// can unroll its share of the items and issue all of their loads at once.
template <int N, class X, class F>
CKDA_PROG void par(X &x, F f) {
  x.template run<N>(f);
}

// Pointers and sizes of one call. Token-major [T_total, H, .] tensors (q, k,
// v, dO and dq, dk, dv in the I/O type; alpha, dalpha [T_total, H, d_k] and
// beta, dbeta [T_total, H] fp32); states [N, H, d_k, d_v] fp32.
template <typename IOT>
struct Args {
  const IOT *q, *k, *v;
  const float *alpha, *beta, *s0;
  const IOT *d_o;
  const float *dsf;
  IOT *dq, *dk, *dv;
  float *dalpha, *dbeta, *ds0;
  int H, DVF;  // heads; full d_v
  float scale;
};

// Stage chunk rows [t0, t0 + L) of head h; rows L..C-1 are inert padding
// (q = k = v = dO = 0, alpha = 1, beta = 0).
template <class X, class IOL, typename IOT, class Ly>
CKDA_PROG void stage(X &x, const Args<IOT> &a, float *sm, int h, int c0, int t0, int L,
                     bool with_do) {
  constexpr int DK = Ly::dk, DVT = Ly::dvt;
  constexpr int NW = DK > DVT ? DK : DVT;  // items per row: the wider of d_k and the tile
  par<C * NW>(x, [&](int e) {
    const int i = e / NW, c = e - i * NW;
    if (c < DK) {
      float qv = 0.f, kv = 0.f, av = 1.f;
      if (i < L) {
        const size_t g = ((size_t)(t0 + i) * a.H + h) * DK + c;
        qv = IOL::ldg(a.q + g);
        kv = IOL::ldg(a.k + g);
        av = CKDA_LDG(a.alpha + g);
      }
      sm[Ly::Q + i * Ly::KS + c] = qv;
      sm[Ly::K + i * Ly::KS + c] = kv;
      sm[Ly::AL + i * Ly::KS + c] = av;
    }
    if (c < DVT) {
      float vv = 0.f, dd = 0.f;
      if (i < L) {
        const size_t g = ((size_t)(t0 + i) * a.H + h) * a.DVF + c0 + c;
        vv = IOL::ldg(a.v + g);
        if (with_do) dd = IOL::ldg(a.d_o + g);
      }
      sm[Ly::V + i * Ly::VS + c] = vv;
      sm[Ly::DO + i * Ly::VS + c] = dd;
    }
    if (e < C) sm[Ly::BE + e] = e < L ? CKDA_LDG(a.beta + (size_t)(t0 + e) * a.H + h) : 0.f;
  });
}

// gamma_i = prod_{s<=i} alpha_s and sigma_j = prod_{s>j} alpha_s per channel
template <class X, class Ly>
CKDA_PROG void chunk_gates(X &x, float *sm) {
  constexpr int DK = Ly::dk, KS = Ly::KS;
  const float *al = sm + Ly::AL;
  par<DK>(x, [&](int c) {
    float g = 1.f;
    for (int i = 0; i < C; ++i) {
      g *= al[i * KS + c];
      sm[Ly::GM + i * KS + c] = g;
    }
    g = 1.f;
    for (int j = C - 1; j >= 0; --j) {
      sm[Ly::SG + j * KS + c] = g;
      g *= al[j * KS + c];
    }
  });
}

// Abar and M, then T = (I + diag(beta) Abar)^-1. A (row i, column j, channel
// group g) item sums channels g, g + NG, g + 2 NG, ... (strided so that the
// groups of one pair read different banks); a second phase adds the NG
// partials in a fixed order. Needs Ly::PG, 2 C C NG floats.
template <class X, class Ly>
CKDA_PROG void chunk_grams_solve(X &x, float *sm) {
  constexpr int DK = Ly::dk, KS = Ly::KS, CS = Ly::CS, NG = Ly::NG;
  const float *al = sm + Ly::AL, *kk = sm + Ly::K, *qq = sm + Ly::Q, *be = sm + Ly::BE;
  par<C * C * NG>(x, [&](int e) {
    const int g = e % NG, p = e / NG, i = p / C, j = p - i * C;
    float ab = 0.f, m = 0.f;
    if (j <= i) {
      for (int c = g; c < DK; c += NG) {
        float gp = 1.f;
        for (int s = j + 1; s <= i; ++s) gp *= al[s * KS + c];
        const float gk = gp * kk[j * KS + c];
        ab += kk[i * KS + c] * gk;
        m += qq[i * KS + c] * gk;
      }
    }
    sm[Ly::PG + 2 * e] = ab;
    sm[Ly::PG + 2 * e + 1] = m;
  });
  par<C * C>(x, [&](int e) {
    const int i = e / C, j = e - i * C;
    float ab = 0.f, m = 0.f;
CKDA_UNROLL
    for (int g = 0; g < NG; ++g) {
      ab += sm[Ly::PG + 2 * (e * NG + g)];
      m += sm[Ly::PG + 2 * (e * NG + g) + 1];
    }
    sm[Ly::AB + i * CS + j] = j < i ? ab : 0.f;
    sm[Ly::M + i * CS + j] = m;
  });
  par<C>(x, [&](int j) {  // column j of T by forward substitution
    float *tt = sm + Ly::TT;
    const float *ab = sm + Ly::AB;
    for (int i = 0; i < j; ++i) tt[i * CS + j] = 0.f;
    tt[j * CS + j] = 1.f;
    for (int i = j + 1; i < C; ++i) {
      float s = 0.f;
      for (int m = j; m < i; ++m) s += ab[i * CS + m] * tt[m * CS + j];
      tt[i * CS + j] = -be[i] * s;
    }
  });
}

// dalpha of one channel c over the chunk: positions p = 0..C, 0 the chunk
// entry and p = i + 1 token row i; E(p, q) the coefficient of G over
// positions (q, p]. F_s(p) = sum_{q<s} G_{s-1<-q} E(p, q) grows as
// F_{s+1} = alpha_s F_s + E(., s); dalpha_s = sum_{p>=s} G_{p<-s} F_s(p), a
// Horner pass from p = C down.
template <class Ly>
CKDA_PROG void gate_grad_channel(const float *sm, int c, float sds, float *out) {
  constexpr int KS = Ly::KS, CS = Ly::CS;
  const float *al = sm + Ly::AL, *kk = sm + Ly::K, *qq = sm + Ly::Q;
  const float *dm = sm + Ly::DM, *da = sm + Ly::DA;
  const float *e0 = sm + Ly::E0, *ex = sm + Ly::EX;
  float F[C + 1];
  // s = 1: F(p) = E(p, 0), the entry column (gamma); exit row adds diag(gamma) S
CKDA_UNROLL
  for (int p = 1; p <= C; ++p) F[p] = e0[(p - 1) * KS + c];
  F[C] += sds;
  F[0] = 0.f;
CKDA_UNROLL
  for (int s = 1; s <= C; ++s) {
    if (s > 1) {
      const int j = s - 2;  // token row of position q = s - 1
      const float a = al[j * KS + c], kj = kk[j * KS + c];
CKDA_UNROLL
      for (int p = s; p <= C; ++p) {
        const int i = p - 1;  // token row of position p (i > j)
        float e = kj * (qq[i * KS + c] * dm[i * CS + j] + kk[i * KS + c] * da[i * CS + j]);
        if (p == C) e += ex[j * KS + c];  // sigma_j: exit coefficient
        F[p] = a * F[p] + e;
      }
    }
    float hsum = F[C];
CKDA_UNROLL
    for (int p = C - 1; p >= s; --p) hsum = al[p * KS + c] * hsum + F[p];
    out[s - 1] = hsum;
  }
}

}  // namespace bwdc
}  // namespace ckda
