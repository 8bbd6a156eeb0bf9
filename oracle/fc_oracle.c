/*
 * fc_oracle.c -- plain FP64 reference for irreducible-Cartesian tensor
 * products, the receiver-sorted edge convolution and the node-local
 * product ladder ("the oracle").
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or
 * calls this file: only the tests, the smoke check and the CPU-baseline leg
 * of the benchmark do.  It shares no code, table or constant with the CUDA
 * library; both sides read the same seeded inputs and nothing else.
 *
 * Everything is done on dense 3^l Cartesian arrays, by explicit outer
 * products, index contractions, averages over index permutations and trace
 * removal, exactly as the defining formulas read.  It is deliberately slow.
 *
 * Sources (FlashCart: Fast Cartesian Tensor Products for Equivariant
 * Interatomic Potentials, arXiv 2610.06409):
 *   - STF spaces, 2l+1 components, parity          Sec. 2 "Irreducible Cartesian tensors"
 *   - admissible paths, n = (l1+l2-l3)/2           Sec. 2, App. B
 *   - independent components (p_z <= 1) and the
 *     trace relation that rebuilds the rest       Sec. 3 "Symbolic construction"
 *   - direction tensor T_l(r)                      App. B, equation after Eq. B1's lead-in
 *   - Cartesian product, distinct placements       App. B Eq. (B1)
 *   - permutation average vs distinct placements   App. C "Symbolic construction"
 *   - weighted product VJP                         App. C Eq. (C1)
 *   - VJP-of-VJP of the weighted product           App. C Eq. (C2), Algorithm 3
 *   - derivatives of the direction tensors         App. C, paragraph after Eq. (C2)
 *   - receiver-sorted convolution                  Sec. 4 Eq. (1)
 *   - array layout off(l) + (c P_l + eta) d + k    App. D "Data layout"
 *   - ladder product + channel mixing              Sec. 5 Eq. (2), App. E
 *   - full ladder (paths kept, path+channel mix)   Sec. 5 Eq. (2)
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *   - C_{l1 l2 l3} of Eq. (B1) is "defined elsewhere".  Here it is fixed so
 *     that (T_l1(r) (x) T_l2(r))_l3 = T_l3(r) for every admissible path
 *     (computed at r = z-hat from the z...z entry).
 *   - order of the 2l+1 components inside a rank block: p_z = 0 first with
 *     p_x descending, then p_z = 1 with p_x descending.
 *   - order of paths: by l3, then l1, then l2.
 *   - weights w[E][P][C] are channel-contiguous.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_MAXL 6                 /* highest rank held densely            */
#define ORC_MAXD 729               /* 3^ORC_MAXL                            */
#define ORC_MAXPERM 720            /* ORC_MAXL!                             */

/* ------------------------------------------------------------------ */
/* small integer helpers                                               */
/* ------------------------------------------------------------------ */

static int pow3(int l) {
  int p = 1;
  for (int i = 0; i < l; ++i) p *= 3;
  return p;
}

static double fact(int n) {
  double f = 1.0;
  for (int i = 2; i <= n; ++i) f *= i;
  return f;
}

/* n!! with (-1)!! = 0!! = 1 */
static double dfact(int n) {
  double f = 1.0;
  for (int i = n; i > 1; i -= 2) f *= i;
  return f;
}

/* multi-index <-> flat position, row-major, digit 0/1/2 = x/y/z */
static void unflat(int l, int f, int *idx) {
  for (int j = l - 1; j >= 0; --j) {
    idx[j] = f % 3;
    f /= 3;
  }
}

static int flat(int l, const int *idx) {
  int f = 0;
  for (int j = 0; j < l; ++j) f = 3 * f + idx[j];
  return f;
}

/* ------------------------------------------------------------------ */
/* permutation tables (all l! orderings of l index slots)               */
/* ------------------------------------------------------------------ */

static int g_nperm[ORC_MAXL + 1];
static unsigned char g_perm[ORC_MAXL + 1][ORC_MAXPERM][ORC_MAXL];

static void build_perms(int l) {
  /* lexicographic enumeration */
  int a[ORC_MAXL];
  for (int i = 0; i < l; ++i) a[i] = i;
  int n = 0;
  for (;;) {
    for (int i = 0; i < l; ++i) g_perm[l][n][i] = (unsigned char)a[i];
    ++n;
    int i = l - 2;
    while (i >= 0 && a[i] >= a[i + 1]) --i;
    if (i < 0) break;
    int j = l - 1;
    while (a[j] <= a[i]) --j;
    int t = a[i]; a[i] = a[j]; a[j] = t;
    for (int p = i + 1, q = l - 1; p < q; ++p, --q) { t = a[p]; a[p] = a[q]; a[q] = t; }
  }
  g_nperm[l] = n;
}

static void init_path_norms(void);

__attribute__((constructor)) static void orc_init(void) {
  for (int l = 0; l <= ORC_MAXL; ++l) build_perms(l);
  init_path_norms();
}

/* ------------------------------------------------------------------ */
/* dense tensor primitives                                             */
/* ------------------------------------------------------------------ */

/* out = average over all l! permutations of the index slots of `in` */
void orc_permavg(int l, const double *in, double *out) {
  int D = pow3(l), idx[ORC_MAXL], pidx[ORC_MAXL];
  int np = g_nperm[l];
  for (int f = 0; f < D; ++f) {
    unflat(l, f, idx);
    double s = 0.0;
    for (int p = 0; p < np; ++p) {
      for (int j = 0; j < l; ++j) pidx[j] = idx[g_perm[l][p][j]];
      s += in[flat(l, pidx)];
    }
    out[f] = s / np;
  }
}

/* x .q. y : contract the last q slots of x (rank a) with the first q slots
 * of y (rank b).  Result rank a+b-2q, slots = x's free slots then y's. */
static void contract(int a, const double *x, int b, const double *y, int q,
                     double *out) {
  int r = a + b - 2 * q;
  int D = pow3(r), K = pow3(q);
  int idx[ORC_MAXL + 2], k[ORC_MAXL], xi[ORC_MAXL], yi[ORC_MAXL];
  for (int fo = 0; fo < D; ++fo) {
    unflat(r, fo, idx);
    double s = 0.0;
    for (int fk = 0; fk < K; ++fk) {
      unflat(q, fk, k);
      for (int j = 0; j < a - q; ++j) xi[j] = idx[j];
      for (int j = 0; j < q; ++j) xi[a - q + j] = k[j];
      for (int j = 0; j < q; ++j) yi[j] = k[j];
      for (int j = 0; j < b - q; ++j) yi[q + j] = idx[a - q + j];
      s += x[flat(a, xi)] * y[flat(b, yi)];
    }
    out[fo] = s;
  }
}

/* out (rank r+2m) = t (rank r) (x) delta (x) ... (x) delta (m factors),
 * the deltas occupying the last 2m slots pairwise */
static void outer_delta(int r, const double *t, int m, double *out) {
  int R = r + 2 * m, D = pow3(R), idx[ORC_MAXL];
  for (int f = 0; f < D; ++f) {
    unflat(R, f, idx);
    double d = 1.0;
    for (int s = 0; s < m; ++s)
      if (idx[r + 2 * s] != idx[r + 2 * s + 1]) { d = 0.0; break; }
    out[f] = (d == 0.0) ? 0.0 : t[flat(r, idx)];
  }
}

/* trace over the first two slots: out (rank l-2) */
static void trace_once(int l, const double *S, double *out) {
  int D = pow3(l - 2), idx[ORC_MAXL], full[ORC_MAXL];
  for (int f = 0; f < D; ++f) {
    unflat(l - 2, f, idx);
    double s = 0.0;
    for (int k = 0; k < 3; ++k) {
      full[0] = k; full[1] = k;
      for (int j = 0; j < l - 2; ++j) full[2 + j] = idx[j];
      s += S[flat(l, full)];
    }
    out[f] = s;
  }
}

/* number of distinct ways to place m deltas and a symmetric rank-(l-2m)
 * block on l slots: l! / ((l-2m)! m! 2^m)  (App. B, after the T_l formula) */
static double count_delta_placements(int l, int m) {
  return fact(l) / (fact(l - 2 * m) * fact(m) * pow(2.0, m));
}

/* Symmetric trace-free part of a SYMMETRIC rank-l tensor S:
 * sum_m (-1)^m (2l-2m-1)!!/(2l-1)!! {Tr^m(S) (x) I^m}, braces = sum over
 * distinct placements = count x permutation average.  This is the trace
 * removal written in App. B for the direction tensor, applied to a general
 * symmetric tensor (the r-hat powers replaced by the tensor's traces). */
void orc_detrace(int l, const double *S, double *out) {
  int D = pow3(l);
  double T[ORC_MAXD], Tn[ORC_MAXD], P[ORC_MAXD], A[ORC_MAXD];
  memcpy(T, S, sizeof(double) * pow3(l));
  for (int f = 0; f < D; ++f) out[f] = 0.0;
  for (int m = 0; 2 * m <= l; ++m) {
    outer_delta(l - 2 * m, T, m, P);
    orc_permavg(l, P, A);
    double c = ((m & 1) ? -1.0 : 1.0) * dfact(2 * l - 2 * m - 1) /
               dfact(2 * l - 1) * count_delta_placements(l, m);
    for (int f = 0; f < D; ++f) out[f] += c * A[f];
    if (2 * m + 2 <= l) {
      trace_once(l - 2 * m, T, Tn);
      memcpy(T, Tn, sizeof(double) * pow3(l - 2 * m - 2));
    }
  }
}

/* ------------------------------------------------------------------ */
/* independent components (Sec. 3): p_z <= 1                            */
/* ------------------------------------------------------------------ */

/* component c of rank l -> index counts (px, py, pz) */
void orc_comp_pxyz(int l, int c, int *px, int *py, int *pz) {
  if (c <= l) {
    *pz = 0; *py = c; *px = l - c;
  } else {
    int j = c - (l + 1);
    *pz = 1; *py = j; *px = l - 1 - j;
  }
}

static int comp_index(int l, int px, int py, int pz) {
  (void)px;
  return (pz == 0) ? py : (l + 1) + py;
}

/* value of entry with counts (px,py,pz): stored if pz <= 1, otherwise the
 * trace relation x_{px,py,pz} = -x_{px+2,py,pz-2} - x_{px,py+2,pz-2} */
static double comp_value(int l, const double *comps, int px, int py, int pz) {
  if (pz <= 1) return comps[comp_index(l, px, py, pz)];
  return -comp_value(l, comps, px + 2, py, pz - 2) -
         comp_value(l, comps, px, py + 2, pz - 2);
}

/* rebuild all 3^l entries from the 2l+1 independent components */
void orc_stf_dense(int l, const double *comps, double *dense) {
  int D = pow3(l), idx[ORC_MAXL];
  for (int f = 0; f < D; ++f) {
    unflat(l, f, idx);
    int n[3] = {0, 0, 0};
    for (int j = 0; j < l; ++j) n[idx[j]]++;
    dense[f] = comp_value(l, comps, n[0], n[1], n[2]);
  }
}

/* read the 2l+1 independent components off a dense tensor */
void orc_stf_extract(int l, const double *dense, double *comps) {
  int idx[ORC_MAXL];
  for (int c = 0; c < 2 * l + 1; ++c) {
    int px, py, pz, j = 0;
    orc_comp_pxyz(l, c, &px, &py, &pz);
    for (int t = 0; t < px; ++t) idx[j++] = 0;
    for (int t = 0; t < py; ++t) idx[j++] = 1;
    for (int t = 0; t < pz; ++t) idx[j++] = 2;
    comps[c] = dense[flat(l, idx)];
  }
}

/* ------------------------------------------------------------------ */
/* direction tensor T_l(r-hat) (App. B)                                 */
/* ------------------------------------------------------------------ */

/* rank-k outer power of u */
static void outer_power(int k, const double *u, double *out) {
  int D = pow3(k), idx[ORC_MAXL];
  for (int f = 0; f < D; ++f) {
    unflat(k, f, idx);
    double p = 1.0;
    for (int j = 0; j < k; ++j) p *= u[idx[j]];
    out[f] = p;
  }
}

static void unit(const double *r, double *u) {
  double n = sqrt(r[0] * r[0] + r[1] * r[1] + r[2] * r[2]);
  u[0] = r[0] / n; u[1] = r[1] / n; u[2] = r[2] / n;
}

/* T_l = (2l-1)!!/l! sum_m (-1)^m (2l-2m-1)!!/(2l-1)!! {u^(l-2m) (x) I^m},
 * u taken as given (callers pass a unit vector) */
static void direction_dense_u(int l, const double *u, double *out) {
  int D = pow3(l);
  double Pw[ORC_MAXD], P[ORC_MAXD], A[ORC_MAXD];
  for (int f = 0; f < D; ++f) out[f] = 0.0;
  double pre = dfact(2 * l - 1) / fact(l);
  for (int m = 0; 2 * m <= l; ++m) {
    outer_power(l - 2 * m, u, Pw);
    outer_delta(l - 2 * m, Pw, m, P);
    orc_permavg(l, P, A);
    double c = pre * ((m & 1) ? -1.0 : 1.0) * dfact(2 * l - 2 * m - 1) /
               dfact(2 * l - 1) * count_delta_placements(l, m);
    for (int f = 0; f < D; ++f) out[f] += c * A[f];
  }
}

void orc_direction_dense(int l, const double *r, double *dense) {
  double u[3];
  unit(r, u);
  direction_dense_u(l, u, dense);
}

void orc_direction(int l, const double *r, double *comps) {
  double d[ORC_MAXD];
  orc_direction_dense(l, r, d);
  orc_stf_extract(l, d, comps);
}

/* Partial derivatives of the components of T_l(u), u taken as free (not
 * normalised): order 1 gives d T_c / d u_i in d1[i][c]; order 2 gives
 * d^2 T_c / d u_i d u_j in d2[3 i + j][c].  Product rule on the outer
 * powers of each term of the direction-tensor sum: a slot holding u_i is
 * replaced by 1 (and for order 2 a second, different slot holding u_j). */
static void direction_du(int l, const double *u, int order,
                         double d1[3][2 * ORC_MAXL + 1],
                         double d2[9][2 * ORC_MAXL + 1]) {
  int D = pow3(l), idx[ORC_MAXL];
  int nd = order == 1 ? 3 : 9;
  double acc[9][ORC_MAXD];
  double Pw[ORC_MAXD], P[ORC_MAXD], A[ORC_MAXD];
  double pre = dfact(2 * l - 1) / fact(l);
  for (int j = 0; j < nd; ++j)
    for (int f = 0; f < D; ++f) acc[j][f] = 0.0;
  for (int m = 0; 2 * m <= l; ++m) {
    int k = l - 2 * m;
    double c = pre * ((m & 1) ? -1.0 : 1.0) * dfact(2 * l - 2 * m - 1) /
               dfact(2 * l - 1) * count_delta_placements(l, m);
    for (int j = 0; j < nd; ++j) {
      int di = order == 1 ? j : j / 3, dj = order == 1 ? -1 : j % 3;
      int Dk = pow3(k);
      for (int f = 0; f < Dk; ++f) {
        unflat(k, f, idx);
        double s = 0.0;
        for (int s1 = 0; s1 < k; ++s1) {
          if (idx[s1] != di) continue;
          if (order == 1) {
            double p = 1.0;
            for (int t = 0; t < k; ++t)
              if (t != s1) p *= u[idx[t]];
            s += p;
          } else {
            for (int s2 = 0; s2 < k; ++s2) {
              if (s2 == s1 || idx[s2] != dj) continue;
              double p = 1.0;
              for (int t = 0; t < k; ++t)
                if (t != s1 && t != s2) p *= u[idx[t]];
              s += p;
            }
          }
        }
        Pw[f] = s;
      }
      outer_delta(k, Pw, m, P);
      orc_permavg(l, P, A);
      for (int f = 0; f < D; ++f) acc[j][f] += c * A[f];
    }
  }
  for (int j = 0; j < nd; ++j) orc_stf_extract(l, acc[j], order == 1 ? d1[j] : d2[j]);
}

/* d T_l(r/|r|) / d r as a (2l+1) x 3 matrix, by the product rule on the
 * outer powers and the chain rule through u = r/|r|:
 * du/dr = (I - u u^T)/|r|. */
void orc_direction_jac(int l, const double *r, double *jac) {
  double u[3], nr = sqrt(r[0] * r[0] + r[1] * r[1] + r[2] * r[2]);
  unit(r, u);
  double comps[3][2 * ORC_MAXL + 1];
  direction_du(l, u, 1, comps, NULL);
  double proj[3][3];
  for (int a = 0; a < 3; ++a)
    for (int b = 0; b < 3; ++b)
      proj[a][b] = ((a == b) ? 1.0 : 0.0) - u[a] * u[b];
  for (int c = 0; c < 2 * l + 1; ++c)
    for (int b = 0; b < 3; ++b) {
      double s = 0.0;
      for (int j = 0; j < 3; ++j) s += comps[j][c] * proj[j][b];
      jac[c * 3 + b] = s / nr;
    }
}

/* Hessian-vector product of F(r) = <ybar, T_l(r/|r|)> (ybar: 2l+1 weights of
 * the components): out = (d^2 F / dr dr) v.  With u = r/|r|, P = I - u u^T,
 * G = dF/du, H_u = d^2 F / du du and the gradient dF/dr = P G / |r|,
 * differentiating along r + t v (du/dt = P v/|r| =: w, d|r|/dt = u.v,
 * dP/dt = -(w u^T + u w^T)) gives
 *   out = [-(w (u.G) + u (w.G)) + P H_u w] / |r| - P G (u.v) / |r|^2. */
void orc_direction_hvp(int l, const double *r, const double *ybar,
                       const double *v, double *out) {
  double u[3], nr = sqrt(r[0] * r[0] + r[1] * r[1] + r[2] * r[2]);
  unit(r, u);
  double d1[3][2 * ORC_MAXL + 1], d2[9][2 * ORC_MAXL + 1];
  direction_du(l, u, 1, d1, NULL);
  direction_du(l, u, 2, NULL, d2);
  double G[3], Hu[3][3];
  for (int i = 0; i < 3; ++i) {
    G[i] = 0.0;
    for (int c = 0; c < 2 * l + 1; ++c) G[i] += ybar[c] * d1[i][c];
    for (int j = 0; j < 3; ++j) {
      Hu[i][j] = 0.0;
      for (int c = 0; c < 2 * l + 1; ++c) Hu[i][j] += ybar[c] * d2[3 * i + j][c];
    }
  }
  double uv = u[0] * v[0] + u[1] * v[1] + u[2] * v[2];
  double w[3], PG[3], Hw[3];
  for (int i = 0; i < 3; ++i) w[i] = (v[i] - u[i] * uv) / nr;
  double uG = u[0] * G[0] + u[1] * G[1] + u[2] * G[2];
  double wG = w[0] * G[0] + w[1] * G[1] + w[2] * G[2];
  for (int i = 0; i < 3; ++i) {
    PG[i] = G[i] - u[i] * uG;
    Hw[i] = Hu[i][0] * w[0] + Hu[i][1] * w[1] + Hu[i][2] * w[2];
  }
  double uHw = u[0] * Hw[0] + u[1] * Hw[1] + u[2] * Hw[2];
  for (int i = 0; i < 3; ++i)
    out[i] = (-(w[i] * uG + u[i] * wG) + Hw[i] - u[i] * uHw) / nr - PG[i] * uv / (nr * nr);
}

/* ------------------------------------------------------------------ */
/* Cartesian product along an admissible path (App. B Eq. B1)           */
/* ------------------------------------------------------------------ */

int orc_admissible(int l1, int l2, int l3) {
  if (l1 < 0 || l2 < 0 || l3 < 0) return 0;
  if (l3 < abs(l1 - l2) || l3 > l1 + l2) return 0;
  if ((l1 + l2 + l3) & 1) return 0;
  if (l1 > ORC_MAXL || l2 > ORC_MAXL || l3 > ORC_MAXL) return 0;
  return 1;
}

/* Unnormalised Eq. (B1) sum on dense inputs:
 * sum_{m=0}^{mmax} (-2)^m (2l3-2m-1)!!/(2l3-1)!! {(x .(n+m). y) (x) I^m},
 * braces = number of distinct placements x permutation average, with
 * (l1-n-m)! (l2-n-m)! m! 2^m placements of the same value among l3! */
static void product_b1(int l1, int l2, int l3, const double *xd,
                       const double *yd, double *out) {
  int n = (l1 + l2 - l3) / 2;
  int mmax = (l1 < l2 ? l1 : l2) - n;
  int D = pow3(l3);
  double Q[ORC_MAXD], P[ORC_MAXD], A[ORC_MAXD];
  for (int f = 0; f < D; ++f) out[f] = 0.0;
  for (int m = 0; m <= mmax; ++m) {
    contract(l1, xd, l2, yd, n + m, Q);
    outer_delta(l3 - 2 * m, Q, m, P);
    orc_permavg(l3, P, A);
    double count = fact(l3) / (fact(l1 - n - m) * fact(l2 - n - m) *
                               fact(m) * pow(2.0, m));
    double c = pow(-2.0, m) * dfact(2 * l3 - 2 * m - 1) / dfact(2 * l3 - 1) *
               count;
    for (int f = 0; f < D; ++f) out[f] += c * A[f];
  }
}

/* Second, independent route (App. C): permutation average of the
 * n-contracted product, generic trace removal, times binom(l3, l1-n). */
static void product_symdetrace(int l1, int l2, int l3, const double *xd,
                               const double *yd, double *out) {
  int n = (l1 + l2 - l3) / 2;
  double Q[ORC_MAXD], S[ORC_MAXD];
  contract(l1, xd, l2, yd, n, Q);
  orc_permavg(l3, Q, S);
  orc_detrace(l3, S, out);
  double b = fact(l3) / (fact(l1 - n) * fact(l2 - n));
  for (int f = 0; f < pow3(l3); ++f) out[f] *= b;
}

/* C_{l1 l2 l3}: normalisation chosen so that T_l1 (x) T_l2 -> T_l3.
 * Both sides are axially symmetric about z-hat and STF, so they agree
 * everywhere once their z...z entries agree, and T_l3(z-hat)_{z..z} = 1. */
static double g_norm[ORC_MAXL + 1][ORC_MAXL + 1][ORC_MAXL + 1];
static int g_norm_done[ORC_MAXL + 1][ORC_MAXL + 1][ORC_MAXL + 1];

static double compute_path_norm(int l1, int l2, int l3) {
  double zhat[3] = {0.0, 0.0, 1.0};
  double t1[ORC_MAXD], t2[ORC_MAXD], u[ORC_MAXD];
  direction_dense_u(l1, zhat, t1);
  direction_dense_u(l2, zhat, t2);
  product_b1(l1, l2, l3, t1, t2, u);
  int idx[ORC_MAXL];
  for (int j = 0; j < l3; ++j) idx[j] = 2;
  return 1.0 / u[flat(l3, idx)];
}

/* ranks <= 4 are filled once at load; higher ranks on first use */
static void init_path_norms(void) {
  for (int l1 = 0; l1 <= 4; ++l1)
    for (int l2 = 0; l2 <= 4; ++l2)
      for (int l3 = 0; l3 <= 4; ++l3)
        if (orc_admissible(l1, l2, l3)) {
          g_norm[l1][l2][l3] = compute_path_norm(l1, l2, l3);
          g_norm_done[l1][l2][l3] = 1;
        }
}

double orc_path_norm(int l1, int l2, int l3) {
  if (!orc_admissible(l1, l2, l3)) return 0.0;
  if (l1 <= 4 && l2 <= 4 && l3 <= 4) return g_norm[l1][l2][l3];
  double c;
#pragma omp critical(orc_norm)
  {
    if (!g_norm_done[l1][l2][l3]) {
      g_norm[l1][l2][l3] = compute_path_norm(l1, l2, l3);
      g_norm_done[l1][l2][l3] = 1;
    }
    c = g_norm[l1][l2][l3];
  }
  return c;
}

/* Dense normalised product from independent components.
 * route 0: Eq. (B1); route 1: symmetrise + generic trace removal. */
int orc_product_dense(int l1, int l2, int l3, const double *xc,
                      const double *yc, double *out, int route) {
  if (!orc_admissible(l1, l2, l3)) return 1;
  double xd[ORC_MAXD], yd[ORC_MAXD];
  orc_stf_dense(l1, xc, xd);
  orc_stf_dense(l2, yc, yd);
  if (route == 0)
    product_b1(l1, l2, l3, xd, yd, out);
  else
    product_symdetrace(l1, l2, l3, xd, yd, out);
  double c = orc_path_norm(l1, l2, l3);
  for (int f = 0; f < pow3(l3); ++f) out[f] *= c;
  return 0;
}

/* the 2l3+1 independent output components f(x, y) */
int orc_product(int l1, int l2, int l3, const double *xc, const double *yc,
                double *out) {
  double d[ORC_MAXD];
  if (orc_product_dense(l1, l2, l3, xc, yc, d, 0)) return 1;
  orc_stf_extract(l3, d, out);
  return 0;
}

/* from dense y (already a direction tensor) -- avoids re-expanding it */
static void product_xc_yd(int l1, int l2, int l3, const double *xc,
                          const double *yd, double *out) {
  double xd[ORC_MAXD], d[ORC_MAXD];
  orc_stf_dense(l1, xc, xd);
  product_b1(l1, l2, l3, xd, yd, d);
  double c = orc_path_norm(l1, l2, l3);
  for (int f = 0; f < pow3(l3); ++f) d[f] *= c;
  orc_stf_extract(l3, d, out);
}

/* Bilinear coefficients of one path, found by evaluating the product on
 * unit independent-component vectors: K[a][b1][b2] = f_a(e_b1, e_b2).
 * Used for the derivatives of Eq. (C1), where d f_a / d x_b1 = f_a(e_b1, y)
 * by bilinearity. */
void orc_path_coeffs(int l1, int l2, int l3, double *K) {
  int n1 = 2 * l1 + 1, n2 = 2 * l2 + 1, n3 = 2 * l3 + 1;
  double e1[2 * ORC_MAXL + 1], e2[2 * ORC_MAXL + 1], f[2 * ORC_MAXL + 1];
  for (int b1 = 0; b1 < n1; ++b1)
    for (int b2 = 0; b2 < n2; ++b2) {
      for (int i = 0; i < n1; ++i) e1[i] = (i == b1);
      for (int i = 0; i < n2; ++i) e2[i] = (i == b2);
      orc_product(l1, l2, l3, e1, e2, f);
      for (int a = 0; a < n3; ++a) K[(a * n1 + b1) * n2 + b2] = f[a];
    }
}

/* ------------------------------------------------------------------ */
/* odd-J (parity-changing) products: App. B, paragraph after Eq. (B1),  */
/* and Sec. 7 "Limitations" -- the same construction with one          */
/* Levi-Civita contraction, the output a pseudo-tensor                  */
/* ------------------------------------------------------------------ */

/* (l1, l2) -> l3 with l1, l2 >= 1, |l1 - l2| <= l3 <= l1 + l2 - 1 and
 * l1 + l2 + l3 odd: n = (l1 + l2 - l3 - 1)/2 index pairs contracted, one
 * index of each input through the Levi-Civita symbol. */
int orc_odd_admissible(int l1, int l2, int l3) {
  if (l1 < 1 || l2 < 1 || l3 < 0) return 0;
  if (l3 < abs(l1 - l2) || l3 > l1 + l2 - 1) return 0;
  if (!((l1 + l2 + l3) & 1)) return 0;
  if (l1 > ORC_MAXL || l2 > ORC_MAXL || l3 + 1 > ORC_MAXL) return 0;
  return 1;
}

/* epsilon_{abc} for a, b, c in {0, 1, 2} */
static double levi_civita(int a, int b, int c) {
  return 0.5 * (double)((a - b) * (b - c) * (c - a));
}

/* Contract n pairs (x's last n slots with y's first n), then x's last free
 * slot p and y's first free slot q through epsilon_{p q c}, c the new last
 * slot; symmetrise over the l3 free slots (permutation average) and remove
 * the traces.  No further factor: the plain symmetric trace-free part. */
static void product_odd(int l1, int l2, int l3, const double *xd, const double *yd,
                        double *out) {
  int n = (l1 + l2 - l3 - 1) / 2;
  int a = l1 - n, b = l2 - n;   /* free slots of x and of y after the pairs */
  double Q[ORC_MAXD], Z[ORC_MAXD], S[ORC_MAXD];
  contract(l1, xd, l2, yd, n, Q);   /* rank a + b = l3 + 1 */
  int D = pow3(l3), idx[ORC_MAXL], qi[ORC_MAXL];
  for (int f = 0; f < D; ++f) {
    unflat(l3, f, idx);
    double sum = 0.0;
    for (int pp = 0; pp < 3; ++pp)
      for (int qq = 0; qq < 3; ++qq) {
        double e = levi_civita(pp, qq, idx[l3 - 1]);
        if (e == 0.0) continue;
        for (int j = 0; j < a - 1; ++j) qi[j] = idx[j];
        qi[a - 1] = pp;
        qi[a] = qq;
        for (int j = 0; j < b - 1; ++j) qi[a + 1 + j] = idx[a - 1 + j];
        sum += e * Q[flat(a + b, qi)];
      }
    Z[f] = sum;
  }
  orc_permavg(l3, Z, S);
  orc_detrace(l3, S, out);
}

/* dense odd product from independent components */
int orc_product_odd_dense(int l1, int l2, int l3, const double *xc, const double *yc,
                          double *out) {
  if (!orc_odd_admissible(l1, l2, l3)) return 1;
  double xd[ORC_MAXD], yd[ORC_MAXD];
  orc_stf_dense(l1, xc, xd);
  orc_stf_dense(l2, yc, yd);
  product_odd(l1, l2, l3, xd, yd, out);
  return 0;
}

int orc_product_odd(int l1, int l2, int l3, const double *xc, const double *yc, double *out) {
  double d[ORC_MAXD];
  if (orc_product_odd_dense(l1, l2, l3, xc, yc, d)) return 1;
  orc_stf_extract(l3, d, out);
  return 0;
}

/* K[a][b1][b2] = f_a(e_b1, e_b2) of an odd path (bilinear, as above) */
void orc_path_coeffs_odd(int l1, int l2, int l3, double *K) {
  int n1 = 2 * l1 + 1, n2 = 2 * l2 + 1, n3 = 2 * l3 + 1;
  double e1[2 * ORC_MAXL + 1], e2[2 * ORC_MAXL + 1], f[2 * ORC_MAXL + 1];
  for (int b1 = 0; b1 < n1; ++b1)
    for (int b2 = 0; b2 < n2; ++b2) {
      for (int i = 0; i < n1; ++i) e1[i] = (i == b1);
      for (int i = 0; i < n2; ++i) e2[i] = (i == b2);
      orc_product_odd(l1, l2, l3, e1, e2, f);
      for (int a = 0; a < n3; ++a) K[(a * n1 + b1) * n2 + b2] = f[a];
    }
}

/* odd paths ordered by l3, then l1, then l2 */
int orc_paths_odd(int lin, int ledge, int lout, int *l1s, int *l2s, int *l3s) {
  int n = 0;
  for (int l3 = 0; l3 <= lout; ++l3)
    for (int l1 = 0; l1 <= lin; ++l1)
      for (int l2 = 0; l2 <= ledge; ++l2)
        if (orc_odd_admissible(l1, l2, l3)) {
          if (l1s) { l1s[n] = l1; l2s[n] = l2; l3s[n] = l3; }
          ++n;
        }
  return n;
}

/* ------------------------------------------------------------------ */
/* path lists                                                           */
/* ------------------------------------------------------------------ */

/* all admissible (l1 <= lin, l2 <= ledge) -> l3 <= lout, ordered by l3,
 * then l1, then l2 */
int orc_paths(int lin, int ledge, int lout, int *l1s, int *l2s, int *l3s) {
  int n = 0;
  for (int l3 = 0; l3 <= lout; ++l3)
    for (int l1 = 0; l1 <= lin; ++l1)
      for (int l2 = 0; l2 <= ledge; ++l2)
        if (orc_admissible(l1, l2, l3)) {
          if (l1s) { l1s[n] = l1; l2s[n] = l2; l3s[n] = l3; }
          ++n;
        }
  return n;
}

#define ORC_MAXP 128

typedef struct {
  int odd;                  /* 1: the odd-J paths, 0: the natural-parity ones */
  int P, l1[ORC_MAXP], l2[ORC_MAXP], l3[ORC_MAXP];
  int eta[ORC_MAXP];        /* position of the path within its l3 */
  int Pl[ORC_MAXL + 1];     /* paths per output rank */
  int zoff[ORC_MAXL + 1];   /* off(l)/C of the output row (App. D) */
  int zrow;                 /* output row length / C */
} path_set;

static void make_paths_par(int lin, int ledge, int lout, int sum_paths, int odd,
                           path_set *ps) {
  ps->odd = odd;
  ps->P = odd ? orc_paths_odd(lin, ledge, lout, ps->l1, ps->l2, ps->l3)
              : orc_paths(lin, ledge, lout, ps->l1, ps->l2, ps->l3);
  for (int l = 0; l <= ORC_MAXL; ++l) ps->Pl[l] = 0;
  for (int p = 0; p < ps->P; ++p) ps->eta[p] = ps->Pl[ps->l3[p]]++;
  int off = 0;
  for (int l = 0; l <= lout; ++l) {
    ps->zoff[l] = off;
    off += (2 * l + 1) * (sum_paths ? 1 : ps->Pl[l]);
  }
  ps->zrow = off;
}

static void make_paths(int lin, int ledge, int lout, int sum_paths, path_set *ps) {
  make_paths_par(lin, ledge, lout, sum_paths, 0, ps);
}

static void path_coeffs_of(const path_set *ps, int p, double *K) {
  if (ps->odd)
    orc_path_coeffs_odd(ps->l1[p], ps->l2[p], ps->l3[p], K);
  else
    orc_path_coeffs(ps->l1[p], ps->l2[p], ps->l3[p], K);
}

/* ------------------------------------------------------------------ */
/* receiver-sorted edge convolution, Eq. (1)                           */
/* ------------------------------------------------------------------ */

/* x: [N][(lin+1)^2 C], entry l^2 C + c C + k (P_l = 1 for node features)
 * w: [E][P][C];  z: [N][zrow C], entry C*(zoff(l3) + c P_l3 + eta) + k, or
 * C*(zoff(l3) + c) + k when paths are summed.
 * Only edges whose receiver has recv_mask != 0 contribute (NULL = all);
 * z rows of other receivers are left at zero. */
static int edge_conv_par(int odd, int lin, int ledge, int lout, int C, int sum_paths, int N,
                         int E, const int32_t *recv, const int32_t *send,
                         const double *vec, const double *x, const double *w,
                         const unsigned char *recv_mask, double *z) {
  if (lin > 5 || ledge > 5 || lout > 5) return 1;
  path_set ps;
  make_paths_par(lin, ledge, lout, sum_paths, odd, &ps);
  int xrow = (lin + 1) * (lin + 1);
  memset(z, 0, sizeof(double) * (size_t)N * ps.zrow * C);
  /* direction tensors per edge, dense (shared by every channel) */
  size_t ystride = 0;
  for (int l = 0; l <= ledge; ++l) ystride += pow3(l);
  double *yd = (double *)malloc(sizeof(double) * (size_t)(E > 0 ? E : 1) * ystride);
  for (int e = 0; e < E; ++e) {
    size_t o = (size_t)e * ystride;
    for (int l = 0; l <= ledge; ++l) {
      orc_direction_dense(l, vec + 3 * e, yd + o);
      o += pow3(l);
    }
  }
  int yoff[ORC_MAXL + 1], o = 0;
  for (int l = 0; l <= ledge; ++l) { yoff[l] = o; o += pow3(l); }

#pragma omp parallel for schedule(dynamic, 1)
  for (int k = 0; k < C; ++k) {
    double xc[2 * ORC_MAXL + 1], f[2 * ORC_MAXL + 1];
    for (int e = 0; e < E; ++e) {
      int u = recv[e], v = send[e];
      if (recv_mask && !recv_mask[u]) continue;
      for (int p = 0; p < ps.P; ++p) {
        int l1 = ps.l1[p], l2 = ps.l2[p], l3 = ps.l3[p];
        for (int c = 0; c < 2 * l1 + 1; ++c)
          xc[c] = x[((size_t)v * xrow + l1 * l1 + c) * C + k];
        if (odd) {
          double xd[ORC_MAXD], d[ORC_MAXD];
          orc_stf_dense(l1, xc, xd);
          product_odd(l1, l2, l3, xd, yd + (size_t)e * ystride + yoff[l2], d);
          orc_stf_extract(l3, d, f);
        } else {
          product_xc_yd(l1, l2, l3, xc, yd + (size_t)e * ystride + yoff[l2], f);
        }
        double wk = w[((size_t)e * ps.P + p) * C + k];
        for (int c = 0; c < 2 * l3 + 1; ++c) {
          int slot = sum_paths ? ps.zoff[l3] + c
                               : ps.zoff[l3] + c * ps.Pl[l3] + ps.eta[p];
          z[((size_t)u * ps.zrow + slot) * C + k] += wk * f[c];
        }
      }
    }
  }
  free(yd);
  return 0;
}

int orc_edge_conv(int lin, int ledge, int lout, int C, int sum_paths, int N,
                  int E, const int32_t *recv, const int32_t *send,
                  const double *vec, const double *x, const double *w,
                  const unsigned char *recv_mask, double *z) {
  return edge_conv_par(0, lin, ledge, lout, C, sum_paths, N, E, recv, send, vec, x, w,
                       recv_mask, z);
}

/* the same sum over the odd-J paths (pseudo-tensor outputs), same layouts
 * with the odd path list */
int orc_edge_conv_odd(int lin, int ledge, int lout, int C, int sum_paths, int N,
                      int E, const int32_t *recv, const int32_t *send,
                      const double *vec, const double *x, const double *w,
                      const unsigned char *recv_mask, double *z) {
  return edge_conv_par(1, lin, ledge, lout, C, sum_paths, N, E, recv, send, vec, x, w,
                       recv_mask, z);
}

/* ------------------------------------------------------------------ */
/* its vector-Jacobian product, Eq. (C1) summed as in Sec. 4            */
/* ------------------------------------------------------------------ */

/* g has the layout of z.  x_bar[v] = sum_e w VJP1(g_u, y_e),
 * w_bar[e,p,k] = <g_u, f(x_v, y_e)>, y_bar[e] = sum_{p,k} w VJP2(g_u, x_v),
 * r_bar[e] = (d y_e / d r_e)^T y_bar[e].  Gradients are taken with respect
 * to the independent components as free variables (App. C).
 * Only edges with edge_mask != 0 contribute (NULL = all); any output pointer
 * may be NULL. */
static int edge_conv_vjp_par(int odd, int lin, int ledge, int lout, int C, int sum_paths,
                             int N, int E, const int32_t *recv, const int32_t *send,
                             const double *vec, const double *x, const double *w,
                             const double *g, const unsigned char *edge_mask,
                             double *x_bar, double *w_bar, double *r_bar) {
  if (lin > 5 || ledge > 5 || lout > 5) return 1;
  path_set ps;
  make_paths_par(lin, ledge, lout, sum_paths, odd, &ps);
  int xrow = (lin + 1) * (lin + 1);
  int yrow = (ledge + 1) * (ledge + 1);
  /* per-path coefficient tensors */
  double *K[ORC_MAXP];
  for (int p = 0; p < ps.P; ++p) {
    int n1 = 2 * ps.l1[p] + 1, n2 = 2 * ps.l2[p] + 1, n3 = 2 * ps.l3[p] + 1;
    K[p] = (double *)malloc(sizeof(double) * n1 * n2 * n3);
    path_coeffs_of(&ps, p, K[p]);
  }
  /* direction tensor components per edge */
  double *y = (double *)malloc(sizeof(double) * (size_t)(E > 0 ? E : 1) * yrow);
  for (int e = 0; e < E; ++e)
    for (int l = 0; l <= ledge; ++l)
      orc_direction(l, vec + 3 * e, y + (size_t)e * yrow + l * l);

  if (x_bar) memset(x_bar, 0, sizeof(double) * (size_t)N * xrow * C);
  if (w_bar) memset(w_bar, 0, sizeof(double) * (size_t)E * ps.P * C);

  /* x_bar and w_bar: channels are independent */
#pragma omp parallel for schedule(dynamic, 1)
  for (int k = 0; k < C; ++k) {
    double gc[2 * ORC_MAXL + 1], xc[2 * ORC_MAXL + 1];
    for (int e = 0; e < E; ++e) {
      if (edge_mask && !edge_mask[e]) continue;
      int u = recv[e], v = send[e];
      for (int p = 0; p < ps.P; ++p) {
        int l1 = ps.l1[p], l2 = ps.l2[p], l3 = ps.l3[p];
        int n1 = 2 * l1 + 1, n2 = 2 * l2 + 1, n3 = 2 * l3 + 1;
        for (int c = 0; c < n3; ++c) {
          int slot = sum_paths ? ps.zoff[l3] + c
                               : ps.zoff[l3] + c * ps.Pl[l3] + ps.eta[p];
          gc[c] = g[((size_t)u * ps.zrow + slot) * C + k];
        }
        for (int c = 0; c < n1; ++c)
          xc[c] = x[((size_t)v * xrow + l1 * l1 + c) * C + k];
        const double *ye = y + (size_t)e * yrow + l2 * l2;
        double wk = w[((size_t)e * ps.P + p) * C + k];
        const double *Kp = K[p];
        if (w_bar) {
          double s = 0.0;
          for (int a = 0; a < n3; ++a)
            for (int b1 = 0; b1 < n1; ++b1)
              for (int b2 = 0; b2 < n2; ++b2)
                s += gc[a] * Kp[(a * n1 + b1) * n2 + b2] * xc[b1] * ye[b2];
          w_bar[((size_t)e * ps.P + p) * C + k] = s;
        }
        if (x_bar) {
          for (int b1 = 0; b1 < n1; ++b1) {
            double s = 0.0;
            for (int a = 0; a < n3; ++a)
              for (int b2 = 0; b2 < n2; ++b2)
                s += gc[a] * Kp[(a * n1 + b1) * n2 + b2] * ye[b2];
            x_bar[((size_t)v * xrow + l1 * l1 + b1) * C + k] += wk * s;
          }
        }
      }
    }
  }

  /* y_bar and r_bar: edges are independent */
  if (r_bar) {
#pragma omp parallel for schedule(dynamic, 16)
    for (int e = 0; e < E; ++e) {
      r_bar[3 * e] = r_bar[3 * e + 1] = r_bar[3 * e + 2] = 0.0;
      if (edge_mask && !edge_mask[e]) continue;
      int u = recv[e], v = send[e];
      double yb[(ORC_MAXL + 1) * (ORC_MAXL + 1)];
      for (int i = 0; i < yrow; ++i) yb[i] = 0.0;
      for (int k = 0; k < C; ++k)
        for (int p = 0; p < ps.P; ++p) {
          int l1 = ps.l1[p], l2 = ps.l2[p], l3 = ps.l3[p];
          int n1 = 2 * l1 + 1, n2 = 2 * l2 + 1, n3 = 2 * l3 + 1;
          double wk = w[((size_t)e * ps.P + p) * C + k];
          const double *Kp = K[p];
          for (int b2 = 0; b2 < n2; ++b2) {
            double s = 0.0;
            for (int a = 0; a < n3; ++a) {
              int slot = sum_paths ? ps.zoff[l3] + a
                                   : ps.zoff[l3] + a * ps.Pl[l3] + ps.eta[p];
              double ga = g[((size_t)u * ps.zrow + slot) * C + k];
              for (int b1 = 0; b1 < n1; ++b1)
                s += ga * Kp[(a * n1 + b1) * n2 + b2] *
                     x[((size_t)v * xrow + l1 * l1 + b1) * C + k];
            }
            yb[l2 * l2 + b2] += wk * s;
          }
        }
      for (int l = 0; l <= ledge; ++l) {
        double jac[(2 * ORC_MAXL + 1) * 3];
        orc_direction_jac(l, vec + 3 * e, jac);
        for (int c = 0; c < 2 * l + 1; ++c)
          for (int b = 0; b < 3; ++b)
            r_bar[3 * e + b] += yb[l * l + c] * jac[c * 3 + b];
      }
    }
  }
  for (int p = 0; p < ps.P; ++p) free(K[p]);
  free(y);
  return 0;
}

int orc_edge_conv_vjp(int lin, int ledge, int lout, int C, int sum_paths,
                      int N, int E, const int32_t *recv, const int32_t *send,
                      const double *vec, const double *x, const double *w,
                      const double *g, const unsigned char *edge_mask,
                      double *x_bar, double *w_bar, double *r_bar) {
  return edge_conv_vjp_par(0, lin, ledge, lout, C, sum_paths, N, E, recv, send, vec, x, w, g,
                           edge_mask, x_bar, w_bar, r_bar);
}

/* the VJP of orc_edge_conv_odd (same formulas, odd-path coefficients) */
int orc_edge_conv_odd_vjp(int lin, int ledge, int lout, int C, int sum_paths,
                          int N, int E, const int32_t *recv, const int32_t *send,
                          const double *vec, const double *x, const double *w,
                          const double *g, const unsigned char *edge_mask,
                          double *x_bar, double *w_bar, double *r_bar) {
  return edge_conv_vjp_par(1, lin, ledge, lout, C, sum_paths, N, E, recv, send, vec, x, w, g,
                           edge_mask, x_bar, w_bar, r_bar);
}

/* ------------------------------------------------------------------ */
/* VJP-of-VJP of the edge convolution (App. C Eq. C2, Algorithm 3)       */
/* ------------------------------------------------------------------ */

/* Gradients of  Lv = <vx, x_bar> + <vw, w_bar> + <vr, r_bar>  (x_bar, w_bar,
 * r_bar the VJP of orc_edge_conv_vjp for the incoming gradient g) with
 * respect to g, x, w and the edge vectors.  Per edge, path and channel, with
 * y the direction tensors and vy = (d y / d r) vr their derivative along vr
 * (the cotangent of y_bar):
 *   g_hat  += w [f(vx, y) + f(x, vy)] + vw f(x, y)      (summed per receiver)
 *   x_hat  += VJP1(g, w vy + vw y)                      (summed per sender)
 *   w_hat   = <g, f(vx, y) + f(x, vy)>
 *   y_hat  += VJP2(g, w vx + vw x)
 * and, through the direction tensors,
 *   r_hat   = (d y / d r)^T y_hat + (d^2 <y_bar, y> / dr dr) vr
 * with y_bar = sum w VJP2(g, x) the edge's first-order direction gradient.
 * vx, vw, vr may be NULL (zero cotangent); outputs may be NULL (skipped).
 * With edge_mask only the listed edges contribute (others' w_hat, r_hat 0). */
int orc_edge_conv_vjp2(int lin, int ledge, int lout, int C, int sum_paths,
                       int N, int E, const int32_t *recv, const int32_t *send,
                       const double *vec, const double *x, const double *w,
                       const double *g, const double *vx, const double *vw,
                       const double *vr, const unsigned char *edge_mask,
                       double *g_hat, double *x_hat, double *w_hat,
                       double *r_hat) {
  if (lin > 5 || ledge > 5 || lout > 5) return 1;
  path_set ps;
  make_paths(lin, ledge, lout, sum_paths, &ps);
  int xrow = (lin + 1) * (lin + 1);
  int yrow = (ledge + 1) * (ledge + 1);
  double *K[ORC_MAXP];
  for (int p = 0; p < ps.P; ++p) {
    int n1 = 2 * ps.l1[p] + 1, n2 = 2 * ps.l2[p] + 1, n3 = 2 * ps.l3[p] + 1;
    K[p] = (double *)malloc(sizeof(double) * n1 * n2 * n3);
    orc_path_coeffs(ps.l1[p], ps.l2[p], ps.l3[p], K[p]);
  }
  /* direction tensors and their derivative along vr, per edge */
  size_t En = (size_t)(E > 0 ? E : 1);
  double *y = (double *)malloc(sizeof(double) * En * yrow);
  double *vy = (double *)malloc(sizeof(double) * En * yrow);
  for (int e = 0; e < E; ++e)
    for (int l = 0; l <= ledge; ++l) {
      orc_direction(l, vec + 3 * e, y + (size_t)e * yrow + l * l);
      double jac[(2 * ORC_MAXL + 1) * 3];
      orc_direction_jac(l, vec + 3 * e, jac);
      for (int c = 0; c < 2 * l + 1; ++c) {
        double t = 0.0;
        if (vr)
          for (int b = 0; b < 3; ++b) t += jac[c * 3 + b] * vr[3 * e + b];
        vy[(size_t)e * yrow + l * l + c] = t;
      }
    }
  if (g_hat) memset(g_hat, 0, sizeof(double) * (size_t)N * ps.zrow * C);
  if (x_hat) memset(x_hat, 0, sizeof(double) * (size_t)N * xrow * C);
  if (w_hat) memset(w_hat, 0, sizeof(double) * (size_t)E * ps.P * C);

  /* g_hat, x_hat, w_hat: channels are independent */
#pragma omp parallel for schedule(dynamic, 1)
  for (int k = 0; k < C; ++k) {
    double gc[2 * ORC_MAXL + 1], xc[2 * ORC_MAXL + 1], vxc[2 * ORC_MAXL + 1];
    double fxy[2 * ORC_MAXL + 1], sv[2 * ORC_MAXL + 1], zc[2 * ORC_MAXL + 1];
    for (int e = 0; e < E; ++e) {
      if (edge_mask && !edge_mask[e]) continue;
      int u = recv[e], v = send[e];
      for (int p = 0; p < ps.P; ++p) {
        int l1 = ps.l1[p], l2 = ps.l2[p], l3 = ps.l3[p];
        int n1 = 2 * l1 + 1, n2 = 2 * l2 + 1, n3 = 2 * l3 + 1;
        int slot[2 * ORC_MAXL + 1];
        for (int c = 0; c < n3; ++c) {
          slot[c] = sum_paths ? ps.zoff[l3] + c : ps.zoff[l3] + c * ps.Pl[l3] + ps.eta[p];
          gc[c] = g[((size_t)u * ps.zrow + slot[c]) * C + k];
        }
        for (int c = 0; c < n1; ++c) {
          xc[c] = x[((size_t)v * xrow + l1 * l1 + c) * C + k];
          vxc[c] = vx ? vx[((size_t)v * xrow + l1 * l1 + c) * C + k] : 0.0;
        }
        const double *ye = y + (size_t)e * yrow + l2 * l2;
        const double *vye = vy + (size_t)e * yrow + l2 * l2;
        size_t wi = ((size_t)e * ps.P + p) * C + k;
        double wk = w[wi], vwk = vw ? vw[wi] : 0.0;
        const double *Kp = K[p];
        /* f(x, y) and s = f(vx, y) + f(x, vy) */
        for (int a = 0; a < n3; ++a) {
          double t0 = 0.0, t1 = 0.0;
          for (int b1 = 0; b1 < n1; ++b1)
            for (int b2 = 0; b2 < n2; ++b2) {
              double kk = Kp[(a * n1 + b1) * n2 + b2];
              t0 += kk * xc[b1] * ye[b2];
              t1 += kk * (vxc[b1] * ye[b2] + xc[b1] * vye[b2]);
            }
          fxy[a] = t0;
          sv[a] = t1;
        }
        if (g_hat)
          for (int a = 0; a < n3; ++a)
            g_hat[((size_t)u * ps.zrow + slot[a]) * C + k] += wk * sv[a] + vwk * fxy[a];
        if (w_hat) {
          double t = 0.0;
          for (int a = 0; a < n3; ++a) t += gc[a] * sv[a];
          w_hat[wi] = t;
        }
        if (x_hat) {
          for (int b2 = 0; b2 < n2; ++b2) zc[b2] = wk * vye[b2] + vwk * ye[b2];
          for (int b1 = 0; b1 < n1; ++b1) {
            double t = 0.0;
            for (int a = 0; a < n3; ++a)
              for (int b2 = 0; b2 < n2; ++b2)
                t += gc[a] * Kp[(a * n1 + b1) * n2 + b2] * zc[b2];
            x_hat[((size_t)v * xrow + l1 * l1 + b1) * C + k] += t;
          }
        }
      }
    }
  }

  /* r_hat: edges are independent */
  if (r_hat) {
#pragma omp parallel for schedule(dynamic, 16)
    for (int e = 0; e < E; ++e) {
      r_hat[3 * e] = r_hat[3 * e + 1] = r_hat[3 * e + 2] = 0.0;
      if (edge_mask && !edge_mask[e]) continue;
      int u = recv[e], v = send[e];
      double yh[(ORC_MAXL + 1) * (ORC_MAXL + 1)], yb[(ORC_MAXL + 1) * (ORC_MAXL + 1)];
      for (int i = 0; i < yrow; ++i) yh[i] = yb[i] = 0.0;
      for (int k = 0; k < C; ++k)
        for (int p = 0; p < ps.P; ++p) {
          int l1 = ps.l1[p], l2 = ps.l2[p], l3 = ps.l3[p];
          int n1 = 2 * l1 + 1, n2 = 2 * l2 + 1, n3 = 2 * l3 + 1;
          size_t wi = ((size_t)e * ps.P + p) * C + k;
          double wk = w[wi], vwk = vw ? vw[wi] : 0.0;
          const double *Kp = K[p];
          for (int b2 = 0; b2 < n2; ++b2) {
            double th = 0.0, tb = 0.0;
            for (int a = 0; a < n3; ++a) {
              int slot = sum_paths ? ps.zoff[l3] + a : ps.zoff[l3] + a * ps.Pl[l3] + ps.eta[p];
              double ga = g[((size_t)u * ps.zrow + slot) * C + k];
              for (int b1 = 0; b1 < n1; ++b1) {
                size_t xi = ((size_t)v * xrow + l1 * l1 + b1) * C + k;
                double kg = ga * Kp[(a * n1 + b1) * n2 + b2];
                th += kg * (wk * (vx ? vx[xi] : 0.0) + vwk * x[xi]);
                tb += kg * wk * x[xi];
              }
            }
            yh[l2 * l2 + b2] += th;
            yb[l2 * l2 + b2] += tb;
          }
        }
      for (int l = 0; l <= ledge; ++l) {
        double jac[(2 * ORC_MAXL + 1) * 3], hv[3];
        orc_direction_jac(l, vec + 3 * e, jac);
        for (int c = 0; c < 2 * l + 1; ++c)
          for (int b = 0; b < 3; ++b) r_hat[3 * e + b] += yh[l * l + c] * jac[c * 3 + b];
        if (vr && l > 0) {
          orc_direction_hvp(l, vec + 3 * e, yb + l * l, vr + 3 * e, hv);
          for (int b = 0; b < 3; ++b) r_hat[3 * e + b] += hv[b];
        }
      }
    }
  }
  for (int p = 0; p < ps.P; ++p) free(K[p]);
  free(y);
  free(vy);
  return 0;
}

/* ------------------------------------------------------------------ */
/* node-local product ladder, Sec. 5 Eq. (2) with path-reduced products */
/* ------------------------------------------------------------------ */

/* For v = 1 .. order-1:
 *   B_v[n,l3,c,k] = sum_{paths -> l3} W_v[p,k] f_p(A_v[n,l1,:,k], A_1[n,l2,:,k])_c
 *   A_{v+1}[n,l,c,k] = sum_k' mix[v][l][k][k'] B_v[n,l,c,k']
 * z = A_1 + ... + A_order.  All ranks l <= L, layout of node features.
 * path_w: [order-1][P][C]; mix: [order-1][L+1][C][C] (out k, in k');
 * states: [order-1][N][(L+1)^2 C] = A_2 .. A_order.
 * Only nodes with node_mask != 0 are computed (NULL = all); the others stay 0. */
static void ladder_tp(const path_set *ps, int C, int row, const double *Av,
                      const double *A1, const double *W, double *B) {
  /* one node: Av, A1, B are [row][C] */
  double xc[2 * ORC_MAXL + 1], yc[2 * ORC_MAXL + 1], f[2 * ORC_MAXL + 1];
  for (int i = 0; i < row * C; ++i) B[i] = 0.0;
  for (int k = 0; k < C; ++k)
    for (int p = 0; p < ps->P; ++p) {
      int l1 = ps->l1[p], l2 = ps->l2[p], l3 = ps->l3[p];
      for (int c = 0; c < 2 * l1 + 1; ++c) xc[c] = Av[(l1 * l1 + c) * C + k];
      for (int c = 0; c < 2 * l2 + 1; ++c) yc[c] = A1[(l2 * l2 + c) * C + k];
      orc_product(l1, l2, l3, xc, yc, f);
      for (int c = 0; c < 2 * l3 + 1; ++c)
        B[(l3 * l3 + c) * C + k] += W[p * C + k] * f[c];
    }
}

static void ladder_mix(int L, int C, const double *mix, const double *B,
                       double *A) {
  for (int l = 0; l <= L; ++l)
    for (int c = 0; c < 2 * l + 1; ++c)
      for (int k = 0; k < C; ++k) {
        double s = 0.0;
        for (int kp = 0; kp < C; ++kp)
          s += mix[((size_t)l * C + k) * C + kp] * B[(l * l + c) * C + kp];
        A[(l * l + c) * C + k] = s;
      }
}

int orc_ladder(int L, int C, int order, int N, const double *A1,
               const double *path_w, const double *mix,
               const unsigned char *node_mask, double *states, double *z) {
  if (L > 4 || order < 1) return 1;
  path_set ps;
  make_paths(L, L, L, 1, &ps);
  int row = (L + 1) * (L + 1);
  size_t nrow = (size_t)row * C;
  if (states && order > 1)
    memset(states, 0, sizeof(double) * (size_t)(order - 1) * N * nrow);
  memset(z, 0, sizeof(double) * (size_t)N * nrow);
#pragma omp parallel for schedule(dynamic, 1)
  for (int n = 0; n < N; ++n) {
    if (node_mask && !node_mask[n]) continue;
    double *Av = (double *)malloc(sizeof(double) * nrow);
    double *B = (double *)malloc(sizeof(double) * nrow);
    double *An = (double *)malloc(sizeof(double) * nrow);
    const double *a1 = A1 + (size_t)n * nrow;
    memcpy(Av, a1, sizeof(double) * nrow);
    for (size_t i = 0; i < nrow; ++i) z[(size_t)n * nrow + i] = a1[i];
    for (int v = 1; v < order; ++v) {
      ladder_tp(&ps, C, row, Av, a1, path_w + (size_t)(v - 1) * ps.P * C, B);
      ladder_mix(L, C, mix + (size_t)(v - 1) * (L + 1) * C * C, B, An);
      memcpy(Av, An, sizeof(double) * nrow);
      if (states)
        memcpy(states + ((size_t)(v - 1) * N + n) * nrow, An,
               sizeof(double) * nrow);
      for (size_t i = 0; i < nrow; ++i) z[(size_t)n * nrow + i] += An[i];
    }
    free(Av); free(B); free(An);
  }
  return 0;
}

/* Full correlation ladder, Sec. 5 Eq. (2): the products keep every path
 * separate and a learned map mixes paths and channels per output rank.
 *   phi_1[l,c,j] = sum_k W1[l][j][k] A[l,c,k]
 *   B_q[eta,c,k] = f_eta(phi_{q-1}[l1,:,k], A[l2,:,k])_c          (q = 2 .. order)
 *   phi_q[l,c,j] = sum_{eta -> l} sum_k Wq[l][j][eta_l C + k] B_q[eta,c,k]
 *   z = phi_1 + ... + phi_order
 * W1: [L+1][C][C]; Wq: [order-1] blocks of C*P*C, each the rank blocks
 * [C][P_l C] one after the other (rank l at C * C * sum_{l'<l} P_l'), eta_l
 * the path's position among the paths into rank l.
 * states: [order][N][(L+1)^2 C] = phi_1 .. phi_order (may be NULL). */
int orc_full_ladder(int L, int C, int order, int N, const double *A,
                    const double *W1, const double *Wq,
                    const unsigned char *node_mask, double *states, double *z) {
  if (L > 4 || order < 1) return 1;
  path_set ps;
  make_paths(L, L, L, 0, &ps);
  int row = (L + 1) * (L + 1);
  size_t nrow = (size_t)row * C;
  int rankoff[ORC_MAXL + 2];
  rankoff[0] = 0;
  for (int l = 0; l <= L; ++l) rankoff[l + 1] = rankoff[l] + ps.Pl[l];
  if (states) memset(states, 0, sizeof(double) * (size_t)order * N * nrow);
  memset(z, 0, sizeof(double) * (size_t)N * nrow);
#pragma omp parallel for schedule(dynamic, 1)
  for (int n = 0; n < N; ++n) {
    if (node_mask && !node_mask[n]) continue;
    const double *a = A + (size_t)n * nrow;
    double *phi = (double *)malloc(sizeof(double) * nrow);
    double *nxt = (double *)malloc(sizeof(double) * nrow);
    double *B = (double *)malloc(sizeof(double) * (size_t)ps.P * (2 * L + 1) * C);
    double xc[2 * ORC_MAXL + 1], yc[2 * ORC_MAXL + 1], f[2 * ORC_MAXL + 1];
    /* phi_1 */
    for (int l = 0; l <= L; ++l)
      for (int c = 0; c < 2 * l + 1; ++c)
        for (int j = 0; j < C; ++j) {
          double t = 0.0;
          for (int k = 0; k < C; ++k)
            t += W1[((size_t)l * C + j) * C + k] * a[(l * l + c) * C + k];
          phi[(l * l + c) * C + j] = t;
        }
    for (int q = 1; q <= order; ++q) {
      if (q > 1) {
        /* B: per path p, component c, channel k at ((p * (2L+1)) + c) * C + k */
        for (int p = 0; p < ps.P; ++p) {
          int l1 = ps.l1[p], l2 = ps.l2[p], l3 = ps.l3[p];
          for (int k = 0; k < C; ++k) {
            for (int i = 0; i < 2 * l1 + 1; ++i) xc[i] = phi[(l1 * l1 + i) * C + k];
            for (int i = 0; i < 2 * l2 + 1; ++i) yc[i] = a[(l2 * l2 + i) * C + k];
            orc_product(l1, l2, l3, xc, yc, f);
            for (int c = 0; c < 2 * l3 + 1; ++c)
              B[((size_t)p * (2 * L + 1) + c) * C + k] = f[c];
          }
        }
        const double *Wqq = Wq + (size_t)(q - 2) * C * ps.P * C;
        for (int l = 0; l <= L; ++l) {
          int K = ps.Pl[l] * C;
          const double *Wl = Wqq + (size_t)C * C * rankoff[l];
          for (int c = 0; c < 2 * l + 1; ++c)
            for (int j = 0; j < C; ++j) {
              double t = 0.0;
              for (int p = 0; p < ps.P; ++p) {
                if (ps.l3[p] != l) continue;
                for (int k = 0; k < C; ++k)
                  t += Wl[(size_t)j * K + ps.eta[p] * C + k] *
                       B[((size_t)p * (2 * L + 1) + c) * C + k];
              }
              nxt[(l * l + c) * C + j] = t;
            }
        }
        memcpy(phi, nxt, sizeof(double) * nrow);
      }
      if (states) memcpy(states + ((size_t)(q - 1) * N + n) * nrow, phi, sizeof(double) * nrow);
      for (size_t i = 0; i < nrow; ++i) z[(size_t)n * nrow + i] += phi[i];
    }
    free(phi); free(nxt); free(B);
  }
  return 0;
}

/* Reverse accumulation through the full ladder (orc_full_ladder above).
 * gz: [N][(L+1)^2 C], the gradient of z.  Every phi_q feeds z directly, so
 * its gradient starts at gz; going down from q = order:
 *   Wq_bar[l][j][eta C + k] += sum_c phibar_q[l,c,j] B_q[eta,c,k]
 *   Bbar_q[eta,c,k]          = sum_j Wq[l][j][eta C + k] phibar_q[l,c,j]
 *   phibar_{q-1}[l1,b1,k]   += sum_{a,b2} Bbar_q[eta,a,k] K[a][b1][b2] A[l2,b2,k]
 *   A_bar[l2,b2,k]          += sum_{a,b1} Bbar_q[eta,a,k] K[a][b1][b2] phi_{q-1}[l1,b1,k]
 * with K the path's coefficient tensor (f_a = sum K[a][b1][b2] x_b1 y_b2,
 * bilinear, App. C Eq. C1), and at the first map
 *   W1_bar[l][j][k] += sum_c phibar_1[l,c,j] A[l,c,k],
 *   A_bar[l,c,k]    += sum_j W1[l][j][k] phibar_1[l,c,j].
 * Weight gradients sum over the nodes that node_mask selects (NULL = all);
 * A_bar rows of other nodes are 0.  W1_bar like W1, Wq_bar like Wq. */
int orc_full_ladder_vjp(int L, int C, int order, int N, const double *A,
                        const double *W1, const double *Wq, const double *gz,
                        const unsigned char *node_mask, double *A_bar,
                        double *W1_bar, double *Wq_bar) {
  if (L > 4 || order < 1) return 1;
  path_set ps;
  make_paths(L, L, L, 0, &ps);
  int row = (L + 1) * (L + 1);
  size_t nrow = (size_t)row * C;
  int rankoff[ORC_MAXL + 2];
  rankoff[0] = 0;
  for (int l = 0; l <= L; ++l) rankoff[l + 1] = rankoff[l] + ps.Pl[l];
  double *K[ORC_MAXP];
  for (int p = 0; p < ps.P; ++p) {
    int n1 = 2 * ps.l1[p] + 1, n2 = 2 * ps.l2[p] + 1, n3 = 2 * ps.l3[p] + 1;
    K[p] = (double *)malloc(sizeof(double) * n1 * n2 * n3);
    orc_path_coeffs(ps.l1[p], ps.l2[p], ps.l3[p], K[p]);
  }
  size_t w1_n = (size_t)(L + 1) * C * C;
  size_t wq_n = (size_t)(order > 1 ? order - 1 : 1) * C * ps.P * C;
  size_t bsz = (size_t)ps.P * (2 * L + 1) * C;
  memset(A_bar, 0, sizeof(double) * (size_t)N * nrow);
  if (W1_bar) memset(W1_bar, 0, sizeof(double) * w1_n);
  if (Wq_bar && order > 1) memset(Wq_bar, 0, sizeof(double) * (size_t)(order - 1) * C * ps.P * C);

#pragma omp parallel
  {
    double *w1b = (double *)calloc(w1_n, sizeof(double));
    double *wqb = (double *)calloc(wq_n, sizeof(double));
    double *phi = (double *)malloc(sizeof(double) * (size_t)order * nrow);
    double *B = (double *)malloc(sizeof(double) * (size_t)order * bsz);
    double *pb = (double *)malloc(sizeof(double) * nrow);
    double *pbn = (double *)malloc(sizeof(double) * nrow);
    double *Bb = (double *)malloc(sizeof(double) * bsz);
    double xc[2 * ORC_MAXL + 1], yc[2 * ORC_MAXL + 1], f[2 * ORC_MAXL + 1];
#pragma omp for schedule(dynamic, 1)
    for (int n = 0; n < N; ++n) {
      if (node_mask && !node_mask[n]) continue;
      const double *a = A + (size_t)n * nrow;
      double *ab = A_bar + (size_t)n * nrow;
      /* forward, keeping phi_q (index q-1) and B_q (index q-1, q >= 2) */
      for (int l = 0; l <= L; ++l)
        for (int c = 0; c < 2 * l + 1; ++c)
          for (int j = 0; j < C; ++j) {
            double t = 0.0;
            for (int k = 0; k < C; ++k)
              t += W1[((size_t)l * C + j) * C + k] * a[(l * l + c) * C + k];
            phi[(l * l + c) * C + j] = t;
          }
      for (int q = 2; q <= order; ++q) {
        const double *prev = phi + (size_t)(q - 2) * nrow;
        double *Bq = B + (size_t)(q - 1) * bsz;
        double *cur = phi + (size_t)(q - 1) * nrow;
        for (int p = 0; p < ps.P; ++p) {
          int l1 = ps.l1[p], l2 = ps.l2[p], l3 = ps.l3[p];
          for (int k = 0; k < C; ++k) {
            for (int i = 0; i < 2 * l1 + 1; ++i) xc[i] = prev[(l1 * l1 + i) * C + k];
            for (int i = 0; i < 2 * l2 + 1; ++i) yc[i] = a[(l2 * l2 + i) * C + k];
            orc_product(l1, l2, l3, xc, yc, f);
            for (int c = 0; c < 2 * l3 + 1; ++c) Bq[((size_t)p * (2 * L + 1) + c) * C + k] = f[c];
          }
        }
        const double *Wqq = Wq + (size_t)(q - 2) * C * ps.P * C;
        for (int l = 0; l <= L; ++l) {
          int Kl = ps.Pl[l] * C;
          const double *Wl = Wqq + (size_t)C * C * rankoff[l];
          for (int c = 0; c < 2 * l + 1; ++c)
            for (int j = 0; j < C; ++j) {
              double t = 0.0;
              for (int p = 0; p < ps.P; ++p) {
                if (ps.l3[p] != l) continue;
                for (int k = 0; k < C; ++k)
                  t += Wl[(size_t)j * Kl + ps.eta[p] * C + k] * Bq[((size_t)p * (2 * L + 1) + c) * C + k];
              }
              cur[(l * l + c) * C + j] = t;
            }
        }
      }
      /* reverse */
      memcpy(pb, gz + (size_t)n * nrow, sizeof(double) * nrow);
      for (int q = order; q >= 2; --q) {
        const double *prev = phi + (size_t)(q - 2) * nrow;
        const double *Bq = B + (size_t)(q - 1) * bsz;
        const double *Wqq = Wq + (size_t)(q - 2) * C * ps.P * C;
        double *wqg = wqb + (size_t)(q - 2) * C * ps.P * C;
        for (int p = 0; p < ps.P; ++p) {
          int l = ps.l3[p];
          int Kl = ps.Pl[l] * C;
          const double *Wl = Wqq + (size_t)C * C * rankoff[l];
          double *Wg = wqg + (size_t)C * C * rankoff[l];
          for (int j = 0; j < C; ++j)
            for (int k = 0; k < C; ++k) {
              double s = 0.0;
              for (int c = 0; c < 2 * l + 1; ++c)
                s += pb[(l * l + c) * C + j] * Bq[((size_t)p * (2 * L + 1) + c) * C + k];
              Wg[(size_t)j * Kl + ps.eta[p] * C + k] += s;
            }
          for (int c = 0; c < 2 * l + 1; ++c)
            for (int k = 0; k < C; ++k) {
              double s = 0.0;
              for (int j = 0; j < C; ++j)
                s += Wl[(size_t)j * Kl + ps.eta[p] * C + k] * pb[(l * l + c) * C + j];
              Bb[((size_t)p * (2 * L + 1) + c) * C + k] = s;
            }
        }
        /* phi_{q-1} feeds z and step q */
        memcpy(pbn, gz + (size_t)n * nrow, sizeof(double) * nrow);
        for (int p = 0; p < ps.P; ++p) {
          int l1 = ps.l1[p], l2 = ps.l2[p], l3 = ps.l3[p];
          int n1 = 2 * l1 + 1, n2 = 2 * l2 + 1, n3 = 2 * l3 + 1;
          const double *Kp = K[p];
          for (int k = 0; k < C; ++k)
            for (int aa = 0; aa < n3; ++aa) {
              double g = Bb[((size_t)p * (2 * L + 1) + aa) * C + k];
              for (int b1 = 0; b1 < n1; ++b1)
                for (int b2 = 0; b2 < n2; ++b2) {
                  double kk = Kp[(aa * n1 + b1) * n2 + b2];
                  pbn[(l1 * l1 + b1) * C + k] += g * kk * a[(l2 * l2 + b2) * C + k];
                  ab[(l2 * l2 + b2) * C + k] += g * kk * prev[(l1 * l1 + b1) * C + k];
                }
            }
        }
        memcpy(pb, pbn, sizeof(double) * nrow);
      }
      /* the first map */
      for (int l = 0; l <= L; ++l)
        for (int j = 0; j < C; ++j)
          for (int k = 0; k < C; ++k) {
            double s = 0.0;
            for (int c = 0; c < 2 * l + 1; ++c)
              s += pb[(l * l + c) * C + j] * a[(l * l + c) * C + k];
            w1b[((size_t)l * C + j) * C + k] += s;
          }
      for (int l = 0; l <= L; ++l)
        for (int c = 0; c < 2 * l + 1; ++c)
          for (int k = 0; k < C; ++k) {
            double s = 0.0;
            for (int j = 0; j < C; ++j)
              s += W1[((size_t)l * C + j) * C + k] * pb[(l * l + c) * C + j];
            ab[(l * l + c) * C + k] += s;
          }
    }
#pragma omp critical(orc_full_ladder_reduce)
    {
      if (W1_bar)
        for (size_t i = 0; i < w1_n; ++i) W1_bar[i] += w1b[i];
      if (Wq_bar && order > 1)
        for (size_t i = 0; i < (size_t)(order - 1) * C * ps.P * C; ++i) Wq_bar[i] += wqb[i];
    }
    free(w1b); free(wqb); free(phi); free(B); free(pb); free(pbn); free(Bb);
  }
  for (int p = 0; p < ps.P; ++p) free(K[p]);
  return 0;
}

/* Reverse accumulation through the ladder above.  gz: [N][(L+1)^2 C].
 * A1_bar like A1; path_w_bar like path_w; mix_bar like mix.  Weight
 * gradients sum over the nodes that node_mask selects (NULL = all). */
int orc_ladder_vjp(int L, int C, int order, int N, const double *A1,
                   const double *path_w, const double *mix, const double *gz,
                   const unsigned char *node_mask, double *A1_bar,
                   double *path_w_bar, double *mix_bar) {
  if (L > 4 || order < 1) return 1;
  path_set ps;
  make_paths(L, L, L, 1, &ps);
  int row = (L + 1) * (L + 1);
  size_t nrow = (size_t)row * C;
  int S = order - 1;
  double *K[ORC_MAXP];
  for (int p = 0; p < ps.P; ++p) {
    int n1 = 2 * ps.l1[p] + 1, n2 = 2 * ps.l2[p] + 1, n3 = 2 * ps.l3[p] + 1;
    K[p] = (double *)malloc(sizeof(double) * n1 * n2 * n3);
    orc_path_coeffs(ps.l1[p], ps.l2[p], ps.l3[p], K[p]);
  }
  memset(A1_bar, 0, sizeof(double) * (size_t)N * nrow);
  size_t pw_n = (size_t)(S > 0 ? S : 1) * ps.P * C;
  size_t mx_n = (size_t)(S > 0 ? S : 1) * (L + 1) * C * C;
  if (path_w_bar && S > 0) memset(path_w_bar, 0, sizeof(double) * S * ps.P * C);
  if (mix_bar && S > 0) memset(mix_bar, 0, sizeof(double) * mx_n);

#pragma omp parallel
  {
    double *pwb = (double *)calloc(pw_n, sizeof(double));
    double *mxb = (double *)calloc(mx_n, sizeof(double));
    double *A = (double *)malloc(sizeof(double) * (size_t)order * nrow);
    double *Bs = (double *)malloc(sizeof(double) * (size_t)(S > 0 ? S : 1) * nrow);
    double *Ab = (double *)malloc(sizeof(double) * (size_t)order * nrow);
    double *Bb = (double *)malloc(sizeof(double) * nrow);
#pragma omp for schedule(dynamic, 1)
    for (int n = 0; n < N; ++n) {
      if (node_mask && !node_mask[n]) continue;
      const double *a1 = A1 + (size_t)n * nrow;
      /* forward, keeping A_v and B_v */
      memcpy(A, a1, sizeof(double) * nrow);
      for (int v = 1; v < order; ++v) {
        ladder_tp(&ps, C, row, A + (size_t)(v - 1) * nrow, a1,
                  path_w + (size_t)(v - 1) * ps.P * C, Bs + (size_t)(v - 1) * nrow);
        ladder_mix(L, C, mix + (size_t)(v - 1) * (L + 1) * C * C,
                   Bs + (size_t)(v - 1) * nrow, A + (size_t)v * nrow);
      }
      /* every A_v feeds z directly */
      for (int v = 0; v < order; ++v)
        memcpy(Ab + (size_t)v * nrow, gz + (size_t)n * nrow, sizeof(double) * nrow);
      for (int v = order - 1; v >= 1; --v) {
        /* step v (0-based v-1) maps A_v -> A_{v+1};  here A index v is A_{v+1} */
        const double *Abn = Ab + (size_t)v * nrow;       /* d/dA_{v+1} */
        const double *Bv = Bs + (size_t)(v - 1) * nrow;
        const double *mx = mix + (size_t)(v - 1) * (L + 1) * C * C;
        double *mxg = mxb + (size_t)(v - 1) * (L + 1) * C * C;
        for (int l = 0; l <= L; ++l)
          for (int c = 0; c < 2 * l + 1; ++c)
            for (int kp = 0; kp < C; ++kp) {
              double s = 0.0;
              for (int k = 0; k < C; ++k)
                s += mx[((size_t)l * C + k) * C + kp] * Abn[(l * l + c) * C + k];
              Bb[(l * l + c) * C + kp] = s;
            }
        for (int l = 0; l <= L; ++l)
          for (int k = 0; k < C; ++k)
            for (int kp = 0; kp < C; ++kp) {
              double s = 0.0;
              for (int c = 0; c < 2 * l + 1; ++c)
                s += Abn[(l * l + c) * C + k] * Bv[(l * l + c) * C + kp];
              mxg[((size_t)l * C + k) * C + kp] += s;
            }
        const double *Av = A + (size_t)(v - 1) * nrow;
        double *Avb = Ab + (size_t)(v - 1) * nrow;
        double *A1b = Ab; /* A_1 is A index 0 */
        const double *W = path_w + (size_t)(v - 1) * ps.P * C;
        double *Wb = pwb + (size_t)(v - 1) * ps.P * C;
        for (int k = 0; k < C; ++k)
          for (int p = 0; p < ps.P; ++p) {
            int l1 = ps.l1[p], l2 = ps.l2[p], l3 = ps.l3[p];
            int n1 = 2 * l1 + 1, n2 = 2 * l2 + 1, n3 = 2 * l3 + 1;
            const double *Kp = K[p];
            double wk = W[p * C + k];
            double s = 0.0;
            for (int a = 0; a < n3; ++a) {
              double ga = Bb[(l3 * l3 + a) * C + k];
              for (int b1 = 0; b1 < n1; ++b1)
                for (int b2 = 0; b2 < n2; ++b2)
                  s += ga * Kp[(a * n1 + b1) * n2 + b2] *
                       Av[(l1 * l1 + b1) * C + k] * a1[(l2 * l2 + b2) * C + k];
            }
            Wb[p * C + k] += s;
            for (int b1 = 0; b1 < n1; ++b1) {
              double t = 0.0;
              for (int a = 0; a < n3; ++a)
                for (int b2 = 0; b2 < n2; ++b2)
                  t += Bb[(l3 * l3 + a) * C + k] * Kp[(a * n1 + b1) * n2 + b2] *
                       a1[(l2 * l2 + b2) * C + k];
              Avb[(l1 * l1 + b1) * C + k] += wk * t;
            }
            for (int b2 = 0; b2 < n2; ++b2) {
              double t = 0.0;
              for (int a = 0; a < n3; ++a)
                for (int b1 = 0; b1 < n1; ++b1)
                  t += Bb[(l3 * l3 + a) * C + k] * Kp[(a * n1 + b1) * n2 + b2] *
                       Av[(l1 * l1 + b1) * C + k];
              A1b[(l2 * l2 + b2) * C + k] += wk * t;
            }
          }
      }
      memcpy(A1_bar + (size_t)n * nrow, Ab, sizeof(double) * nrow);
    }
#pragma omp critical(orc_ladder_reduce)
    {
      if (path_w_bar && S > 0)
        for (size_t i = 0; i < (size_t)S * ps.P * C; ++i) path_w_bar[i] += pwb[i];
      if (mix_bar && S > 0)
        for (size_t i = 0; i < mx_n; ++i) mix_bar[i] += mxb[i];
    }
    free(pwb); free(mxb); free(A); free(Bs); free(Ab); free(Bb);
  }
  for (int p = 0; p < ps.P; ++p) free(K[p]);
  return 0;
}

/* ------------------------------------------------------------------ */
/* misc                                                                 */
/* ------------------------------------------------------------------ */

int orc_max_rank(void) { return ORC_MAXL; }

int orc_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
