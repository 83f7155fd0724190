/*
 * cgtp_oracle.c -- FP64 reference implementation of the Clebsch-Gordan
 * tensor-product (CGTP) convolution.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load this library.  The CUDA
 * product path shares no code, table or helper with it.
 *
 * Everything here is written as the plain definition, in double precision,
 * with loops a reader can check against the definitions by eye:
 *   - complex Clebsch-Gordan coefficients from Racah's closed-form sum,
 *   - real CG coefficients by the unitary complex->real change of basis
 *     that matches the real spherical harmonics below,
 *   - real spherical harmonics from associated Legendre functions in
 *     (theta, phi), component normalisation, m = -l..l, no Condon-Shortley
 *     phase,
 *   - a brute-force periodic neighbour search over all atom pairs and images,
 *   - the forward and backward CGTP convolution as nested sums,
 *   - the gradient of the harmonics with respect to the edge vector (forward-
 *     mode differentiation of the harmonics above), and the force and
 *     strain-derivative (virial) assembly from it (the steps after the
 *     backward: forces = -dE/dpos, stress = dE/d strain / volume).
 *
 * Source of the operation: LunaTP (arXiv 2610.18393), Abstract (the CGTP
 * convolution), Table 1 (irreps configurations and hence the path set) and
 * Table 11 (the outputs x', and the gradients x-bar, y-bar, w-bar).
 * The pages never print the formula; the reading taken (uvu weights per
 * edge, sum over neighbours into the receiver) is the plain one and is
 * listed with every other reading in the design notes.
 *
 * Parity pins for every function live in tests/test_oracle_*.py.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------ */
/* deliberate-fault switch used only by the mutation tests, default 0   */
/* ------------------------------------------------------------------ */
static int g_fault = 0;
void orc_set_fault(int f) { g_fault = f; }
int orc_get_fault(void) { return g_fault; }

/* Threads of a parallel loop: the caller's count when positive, else the
 * process default read once (never changed here, so a one-thread call does
 * not lower later ones).  Loops write disjoint outputs, so results do not
 * depend on the count. */
static int orc_threads(int nthreads) {
#ifdef _OPENMP
  static int deflt = 0;
  if (deflt == 0) deflt = omp_get_max_threads();
  return nthreads > 0 ? nthreads : deflt;
#else
  (void)nthreads;
  return 1;
#endif
}

int orc_max_threads(void) {
#ifdef _OPENMP
  return orc_threads(0);
#else
  return 1;
#endif
}

static double fact(int n) {
  double f = 1.0;
  for (int i = 2; i <= n; ++i) f *= (double)i;
  return f;
}

/* Complex CG <j1 m1 j2 m2 | J M>, Condon-Shortley convention, from Racah's
 * closed-form sum over k (integer angular momenta only). */
double orc_cg_complex(int j1, int m1, int j2, int m2, int J, int M) {
  if (M != m1 + m2) return 0.0;
  if (J < abs(j1 - j2) || J > j1 + j2) return 0.0;
  if (abs(m1) > j1 || abs(m2) > j2 || abs(M) > J) return 0.0;
  double pre = sqrt((2.0 * J + 1.0) * fact(J + j1 - j2) * fact(J - j1 + j2) *
                    fact(j1 + j2 - J) / fact(j1 + j2 + J + 1));
  pre *= sqrt(fact(J + M) * fact(J - M) * fact(j1 - m1) * fact(j1 + m1) *
              fact(j2 - m2) * fact(j2 + m2));
  double s = 0.0;
  for (int k = 0; k <= j1 + j2 + J; ++k) {
    int a1 = j1 + j2 - J - k, a2 = j1 - m1 - k, a3 = j2 + m2 - k;
    int a4 = J - j2 + m1 + k, a5 = J - j1 - m2 + k;
    if (a1 < 0 || a2 < 0 || a3 < 0 || a4 < 0 || a5 < 0) continue;
    double t = 1.0 / (fact(k) * fact(a1) * fact(a2) * fact(a3) * fact(a4) * fact(a5));
    s += (k & 1) ? -t : t;
  }
  return pre * s;
}

/* Row m (real index) of the complex->real change of basis for degree l:
 *   real Y_{l,m}  = sum_{m'} U[m][m'] * complex Y_{l,m'}
 *   m > 0 : ( Y_{-m} + (-1)^m Y_{m} ) / sqrt2
 *   m = 0 : Y_0
 *   m < 0 : i ( Y_{m} - (-1)^m Y_{-m} ) / sqrt2
 * Stored as separate real/imaginary parts, [2l+1][2l+1], index = m + l. */
static void u_matrix(int l, double* ure, double* uim) {
  int n = 2 * l + 1;
  const double s = 1.0 / sqrt(2.0);
  memset(ure, 0, sizeof(double) * n * n);
  memset(uim, 0, sizeof(double) * n * n);
  for (int m = -l; m <= l; ++m) {
    int r = m + l;
    double sg = (abs(m) & 1) ? -1.0 : 1.0; /* (-1)^m */
    if (m > 0) {
      ure[r * n + (-m + l)] = s;
      ure[r * n + (m + l)] = sg * s;
    } else if (m == 0) {
      ure[r * n + l] = 1.0;
    } else {
      uim[r * n + (m + l)] = s;
      uim[r * n + (-m + l)] = -sg * s;
    }
  }
  if (g_fault == 2) { /* mutation: the (-1)^m factor dropped from the m>0 rows */
    for (int m = 1; m <= l; ++m) ure[(m + l) * n + (m + l)] = s;
  }
}

/* Real CG block C[m1][m2][m3] (each index 0..2l+1 for m=-l..l) for the
 * coupling l1 (x) l2 -> l3, in the real basis of orc_sph_harm.
 *   C = sum U3[m3][m3'] conj(U1[m1][m1']) conj(U2[m2][m2']) CG[m1',m2',m3']
 * The result is purely real or purely imaginary; the non-vanishing part is
 * kept, scaled so that sum C^2 = 2 l3 + 1, and its sign fixed so that the
 * first entry (lexicographic in m1, m2, m3) with |C| > 1e-12 is positive.
 * Returns 0 on success, -1 if the coupling is not allowed by the triangle rule. */
int orc_real_cg(int l1, int l2, int l3, double* C) {
  if (l3 < abs(l1 - l2) || l3 > l1 + l2) return -1;
  int n1 = 2 * l1 + 1, n2 = 2 * l2 + 1, n3 = 2 * l3 + 1;
  double *u1r = malloc(sizeof(double) * n1 * n1), *u1i = malloc(sizeof(double) * n1 * n1);
  double *u2r = malloc(sizeof(double) * n2 * n2), *u2i = malloc(sizeof(double) * n2 * n2);
  double *u3r = malloc(sizeof(double) * n3 * n3), *u3i = malloc(sizeof(double) * n3 * n3);
  double *cre = calloc((size_t)n1 * n2 * n3, sizeof(double));
  double *cim = calloc((size_t)n1 * n2 * n3, sizeof(double));
  u_matrix(l1, u1r, u1i);
  u_matrix(l2, u2r, u2i);
  u_matrix(l3, u3r, u3i);
  for (int a = 0; a < n1; ++a)
    for (int b = 0; b < n2; ++b)
      for (int c = 0; c < n3; ++c) {
        double sre = 0.0, sim = 0.0;
        for (int mp1 = -l1; mp1 <= l1; ++mp1)
          for (int mp2 = -l2; mp2 <= l2; ++mp2) {
            int mp3 = mp1 + mp2;
            if (mp3 < -l3 || mp3 > l3) continue;
            double cg = orc_cg_complex(l1, mp1, l2, mp2, l3, mp3);
            if (cg == 0.0) continue;
            /* conj(U1[a][mp1]) * conj(U2[b][mp2]) * U3[c][mp3] */
            double ar = u1r[a * n1 + mp1 + l1], ai = -u1i[a * n1 + mp1 + l1];
            double br = u2r[b * n2 + mp2 + l2], bi = -u2i[b * n2 + mp2 + l2];
            double cr = u3r[c * n3 + mp3 + l3], ci = u3i[c * n3 + mp3 + l3];
            double abr = ar * br - ai * bi, abi = ar * bi + ai * br;
            double pr = abr * cr - abi * ci, pi = abr * ci + abi * cr;
            sre += pr * cg;
            sim += pi * cg;
          }
        cre[(a * n2 + b) * n3 + c] = sre;
        cim[(a * n2 + b) * n3 + c] = sim;
      }
  double nre = 0.0, nim = 0.0;
  int nt = n1 * n2 * n3;
  for (int t = 0; t < nt; ++t) {
    nre += cre[t] * cre[t];
    nim += cim[t] * cim[t];
  }
  const double* src = (nre >= nim) ? cre : cim;
  double nrm = (nre >= nim) ? nre : nim;
  double scale = sqrt((double)n3 / nrm);
  for (int t = 0; t < nt; ++t) C[t] = src[t] * scale;
  for (int t = 0; t < nt; ++t) {
    if (fabs(C[t]) > 1e-12) {
      if (C[t] < 0)
        for (int q = 0; q < nt; ++q) C[q] = -C[q];
      break;
    }
  }
  for (int t = 0; t < nt; ++t)
    if (fabs(C[t]) < 1e-14) C[t] = 0.0;
  free(u1r); free(u1i); free(u2r); free(u2i); free(u3r); free(u3i);
  free(cre); free(cim);
  return 0;
}

/* Real spherical harmonics, component normalisation (sum_m Y_lm^2 = 2l+1):
 *   Y_l0      = sqrt(2l+1) P_l(cos th)
 *   Y_l,m>0   = sqrt(2l+1) sqrt(2 (l-m)!/(l+m)!) P_l^m(cos th) cos(m phi)
 *   Y_l,-m<0  = sqrt(2l+1) sqrt(2 (l-m)!/(l+m)!) P_l^m(cos th) sin(m phi)
 * with P_l^m WITHOUT the Condon-Shortley phase.  So Y_1 = sqrt3 (y, z, x).
 * r is [E][3] (not necessarily unit); Y is [E][(L+1)^2], index l^2 + l + m.
 * A zero vector gives Y_00 = 1 and every other component 0. */
void orc_sph_harm(int L, int64_t E, const double* r, double* Y) {
  int D = (L + 1) * (L + 1);
  for (int64_t e = 0; e < E; ++e) {
    double x = r[3 * e], y = r[3 * e + 1], z = r[3 * e + 2];
    double* out = Y + e * D;
    double rr = sqrt(x * x + y * y + z * z);
    if (rr == 0.0) {
      for (int t = 0; t < D; ++t) out[t] = 0.0;
      out[0] = 1.0;
      continue;
    }
    double ct = z / rr;
    if (ct > 1.0) ct = 1.0;
    if (ct < -1.0) ct = -1.0;
    double th = acos(ct);
    double ph = atan2(y, x);
    double st = sin(th);
    double P[13][13];
    memset(P, 0, sizeof(P));
    /* P_m^m = (2m-1)!! st^m, then the upward recurrence in l */
    for (int m = 0; m <= L; ++m) {
      double pmm = 1.0;
      for (int k = 1; k <= m; ++k) pmm *= (2.0 * k - 1.0) * st;
      P[m][m] = pmm;
      if (m + 1 <= L) P[m + 1][m] = ct * (2.0 * m + 1.0) * pmm;
      for (int l = m + 2; l <= L; ++l)
        P[l][m] = ((2.0 * l - 1.0) * ct * P[l - 1][m] - (l + m - 1.0) * P[l - 2][m]) / (l - m);
    }
    for (int l = 0; l <= L; ++l) {
      double nl = sqrt(2.0 * l + 1.0);
      out[l * l + l] = nl * P[l][0];
      for (int m = 1; m <= l; ++m) {
        double nm = nl * sqrt(2.0 * fact(l - m) / fact(l + m));
        out[l * l + l + m] = nm * P[l][m] * cos(m * ph);
        out[l * l + l - m] = nm * P[l][m] * sin(m * ph);
      }
    }
  }
}

/* ------------------------------------------------------------------ */
/* gradient of the real spherical harmonics with respect to r           */
/* ------------------------------------------------------------------ */
/* Forward-mode differentiation of orc_sph_harm above: every quantity of that
 * computation carries its value and its derivatives with respect to
 * (x, y, z), propagated through each elementary operation by the chain rule
 * (exact up to rounding).  J is [E][(L+1)^2][3], J[e][t][k] = dY_t/dr_k.
 * r = 0 gives J = 0.  Undefined exactly on the z axis (x = y = 0, r != 0),
 * where phi = atan2(y, x) has no derivative; returns -1 if such an edge
 * occurs, else 0.  This is the step from dL/dY to dL/dr on the way to the
 * forces (forces = minus the position gradient of the energy, the BranchIP
 * page's force definition). */
typedef struct {
  double v, d[3];
} dual3;

static dual3 dconst(double v) {
  dual3 a = {v, {0.0, 0.0, 0.0}};
  return a;
}
static dual3 dadd(dual3 a, dual3 b) {
  dual3 c = {a.v + b.v, {a.d[0] + b.d[0], a.d[1] + b.d[1], a.d[2] + b.d[2]}};
  return c;
}
static dual3 dsub(dual3 a, dual3 b) {
  dual3 c = {a.v - b.v, {a.d[0] - b.d[0], a.d[1] - b.d[1], a.d[2] - b.d[2]}};
  return c;
}
static dual3 dmul(dual3 a, dual3 b) {
  dual3 c;
  c.v = a.v * b.v;
  for (int k = 0; k < 3; ++k) c.d[k] = a.d[k] * b.v + a.v * b.d[k];
  return c;
}
static dual3 dscale(double s, dual3 a) {
  dual3 c = {s * a.v, {s * a.d[0], s * a.d[1], s * a.d[2]}};
  return c;
}
static dual3 ddiv(dual3 a, dual3 b) {
  dual3 c;
  c.v = a.v / b.v;
  for (int k = 0; k < 3; ++k) c.d[k] = (a.d[k] * b.v - a.v * b.d[k]) / (b.v * b.v);
  return c;
}
/* f(a) with f' given: value f(a.v), derivative f'(a.v) * a.d */
static dual3 dapply(dual3 a, double f, double fprime) {
  dual3 c = {f, {fprime * a.d[0], fprime * a.d[1], fprime * a.d[2]}};
  return c;
}
static dual3 dsqrt(dual3 a) { return dapply(a, sqrt(a.v), 0.5 / sqrt(a.v)); }
static dual3 dacos(dual3 a) { return dapply(a, acos(a.v), -1.0 / sqrt(1.0 - a.v * a.v)); }
static dual3 dsin(dual3 a) { return dapply(a, sin(a.v), cos(a.v)); }
static dual3 dcos(dual3 a) { return dapply(a, cos(a.v), -sin(a.v)); }
static dual3 datan2(dual3 y, dual3 x) {
  /* d atan2(y, x) = (x dy - y dx) / (x^2 + y^2) */
  dual3 c;
  double q = x.v * x.v + y.v * y.v;
  c.v = atan2(y.v, x.v);
  for (int k = 0; k < 3; ++k) c.d[k] = (x.v * y.d[k] - y.v * x.d[k]) / q;
  if (g_fault == 3) /* mutation: the phi dependence of the gradient dropped */
    for (int k = 0; k < 3; ++k) c.d[k] = 0.0;
  return c;
}

int orc_sph_harm_grad(int L, int64_t E, const double* r, double* J) {
  int D = (L + 1) * (L + 1), bad = 0;
  for (int64_t e = 0; e < E; ++e) {
    double* out = J + e * D * 3;
    for (int t = 0; t < 3 * D; ++t) out[t] = 0.0;
    dual3 x = {r[3 * e], {1.0, 0.0, 0.0}};
    dual3 y = {r[3 * e + 1], {0.0, 1.0, 0.0}};
    dual3 z = {r[3 * e + 2], {0.0, 0.0, 1.0}};
    dual3 rr = dsqrt(dadd(dadd(dmul(x, x), dmul(y, y)), dmul(z, z)));
    if (rr.v == 0.0) continue;
    if (x.v == 0.0 && y.v == 0.0) {
      bad = 1;
      continue;
    }
    dual3 ct = ddiv(z, rr);
    dual3 th = dacos(ct);
    dual3 ph = datan2(y, x);
    dual3 st = dsin(th);
    dual3 P[13][13];
    for (int a = 0; a < 13; ++a)
      for (int b = 0; b < 13; ++b) P[a][b] = dconst(0.0);
    /* the same recurrences as orc_sph_harm, on dual numbers */
    for (int m = 0; m <= L; ++m) {
      dual3 pmm = dconst(1.0);
      for (int k = 1; k <= m; ++k) pmm = dmul(pmm, dscale(2.0 * k - 1.0, st));
      P[m][m] = pmm;
      if (m + 1 <= L) P[m + 1][m] = dscale(2.0 * m + 1.0, dmul(ct, pmm));
      for (int l = m + 2; l <= L; ++l)
        P[l][m] = dscale(1.0 / (l - m), dsub(dscale(2.0 * l - 1.0, dmul(ct, P[l - 1][m])),
                                             dscale(l + m - 1.0, P[l - 2][m])));
    }
    for (int l = 0; l <= L; ++l) {
      double nl = sqrt(2.0 * l + 1.0);
      dual3 y0 = dscale(nl, P[l][0]);
      for (int k = 0; k < 3; ++k) out[(l * l + l) * 3 + k] = y0.d[k];
      for (int m = 1; m <= l; ++m) {
        double nm = nl * sqrt(2.0 * fact(l - m) / fact(l + m));
        dual3 mph = dscale((double)m, ph);
        dual3 yc = dscale(nm, dmul(P[l][m], dcos(mph)));
        dual3 ys = dscale(nm, dmul(P[l][m], dsin(mph)));
        for (int k = 0; k < 3; ++k) {
          out[(l * l + l + m) * 3 + k] = yc.d[k];
          out[(l * l + l - m) * 3 + k] = ys.d[k];
        }
      }
    }
  }
  return bad ? -1 : 0;
}

/* Forces from the edge-vector gradient G = dL/dr [E][3], with
 * r_e = pos[col[e]] - pos[i] (+ image shift) for the edges e of receiver i:
 *   F[a] = -dL/dpos[a] = sum_{e of receiver a} G[e] - sum_{e with col[e] = a} G[e].
 * Plain loops over the edges. */
void orc_edge_forces(int64_t n_atoms, const int64_t* rowptr, const int32_t* col, const double* G,
                     double* F) {
  for (int64_t a = 0; a < 3 * n_atoms; ++a) F[a] = 0.0;
  for (int64_t i = 0; i < n_atoms; ++i)
    for (int64_t e = rowptr[i]; e < rowptr[i + 1]; ++e)
      for (int k = 0; k < 3; ++k) {
        F[3 * i + k] += G[3 * e + k];
        F[3 * (int64_t)col[e] + k] -= (g_fault == 4 ? -1.0 : 1.0) * G[3 * e + k]; /* 4: sign mutation */
      }
}

/* Strain derivative of the loss from G = dL/dr [E][3]: straining every
 * edge vector (and with it the cell) as r_e -> (1 + eps) r_e gives
 *   V[3a+b] = dL/d eps_ab = sum_e G[e][a] r[e][b].
 * The stress is V / volume.  Chain rule through the edge vectors, plain loop. */
void orc_edge_virial(int64_t E, const double* r, const double* G, double* V) {
  for (int k = 0; k < 9; ++k) V[k] = 0.0;
  for (int64_t e = 0; e < E; ++e)
    for (int a = 0; a < 3; ++a)
      for (int b = 0; b < 3; ++b) {
        int k = g_fault == 5 ? 3 * b + a : 3 * a + b; /* 5: transposed mutation */
        V[k] += G[3 * e + a] * r[3 * e + b];
      }
}

/* ------------------------------------------------------------------ */
/* brute-force periodic neighbour list                                  */
/* ------------------------------------------------------------------ */
/* Edge i <- j with image n exists iff (i,j,n) != (i,i,0) and
 *   d = (pos_j + n*box) - pos_i   (component-wise, FP64, in that order),
 *   d.x*d.x + d.y*d.y + d.z*d.z < rc*rc   (strict, FP64).
 * Images |n_a| <= ceil(rc / box_a).  Edges are ordered by (i, j, nx, ny, nz).
 * Pass 1 (rowptr only) when col == NULL; pass 2 fills col / shift / vec.
 * rowptr has N+1 entries.  Returns the edge count. */
int64_t orc_neighbor_list(int64_t N, const double* pos, const double* box, double rc,
                          int64_t* rowptr, int32_t* col, int32_t* shift, double* vec) {
  int K[3];
  for (int a = 0; a < 3; ++a) K[a] = (int)ceil(rc / box[a]);
  double rc2 = rc * rc;
  if (col == NULL) {
    rowptr[0] = 0;
#pragma omp parallel for schedule(dynamic, 16)
    for (int64_t i = 0; i < N; ++i) {
      int64_t cnt = 0;
      for (int64_t j = 0; j < N; ++j)
        for (int nx = -K[0]; nx <= K[0]; ++nx)
          for (int ny = -K[1]; ny <= K[1]; ++ny)
            for (int nz = -K[2]; nz <= K[2]; ++nz) {
              if (i == j && nx == 0 && ny == 0 && nz == 0) continue;
              double dx = (pos[3 * j] + (double)nx * box[0]) - pos[3 * i];
              double dy = (pos[3 * j + 1] + (double)ny * box[1]) - pos[3 * i + 1];
              double dz = (pos[3 * j + 2] + (double)nz * box[2]) - pos[3 * i + 2];
              double d2 = dx * dx + dy * dy + dz * dz;
              if (d2 < rc2) cnt++;
            }
      rowptr[i + 1] = cnt;
    }
    for (int64_t i = 0; i < N; ++i) rowptr[i + 1] += rowptr[i];
    return rowptr[N];
  }
#pragma omp parallel for schedule(dynamic, 16)
  for (int64_t i = 0; i < N; ++i) {
    int64_t e = rowptr[i];
    for (int64_t j = 0; j < N; ++j)
      for (int nx = -K[0]; nx <= K[0]; ++nx)
        for (int ny = -K[1]; ny <= K[1]; ++ny)
          for (int nz = -K[2]; nz <= K[2]; ++nz) {
            if (i == j && nx == 0 && ny == 0 && nz == 0) continue;
            double dx = (pos[3 * j] + (double)nx * box[0]) - pos[3 * i];
            double dy = (pos[3 * j + 1] + (double)ny * box[1]) - pos[3 * i + 1];
            double dz = (pos[3 * j + 2] + (double)nz * box[2]) - pos[3 * i + 2];
            double d2 = dx * dx + dy * dy + dz * dz;
            if (d2 < rc2) {
              col[e] = (int32_t)j;
              shift[3 * e] = nx;
              shift[3 * e + 1] = ny;
              shift[3 * e + 2] = nz;
              vec[3 * e] = dx;
              vec[3 * e + 1] = dy;
              vec[3 * e + 2] = dz;
              e++;
            }
          }
  }
  return rowptr[N];
}

/* ------------------------------------------------------------------ */
/* CGTP convolution                                                     */
/* ------------------------------------------------------------------ */
/* Path table, one row of 8 int32 per path p:
 *   [0] l1  [1] l2  [2] l3  [3] mul (channels u of the hidden irrep)
 *   [4] x_off : offset of the hidden irrep block in a row of x
 *   [5] k0    : W column of channel u=0 of this path (column k0+u)
 *   [6] o_off : offset in a row of out of channel u=0 of this path
 *               (channel u, component m3 at o_off + u*(2l3+1) + m3)
 *   [7] c_off : offset of this path's real CG block [n1][n2][n3] in cg
 * Hidden feature of channel u, component m1: x[j][x_off + u*(2l1+1) + m1].
 * Edge SH of degree l2, component m2:        Y[e][l2*l2 + m2].
 *
 * forward:  out[i][o_off + u n3 + m3] =
 *    sum_{e in row i} W[e][k0+u] sum_{m1,m2} C[m1][m2][m3] x[col e][..m1] Y[e][..m2]
 */
enum { PI_L1, PI_L2, PI_L3, PI_MUL, PI_XOFF, PI_K0, PI_OOFF, PI_COFF, PI_N };

void orc_forward(int64_t n_recv, const int64_t* rowptr, const int32_t* col, int D_in, int D_e,
                 int D_out, int U, const double* x, const double* Y, const double* W, int npaths,
                 const int32_t* paths, const double* cg, double* out, int nthreads) {
  const int nt = orc_threads(nthreads);
  (void)nt;
#pragma omp parallel for schedule(dynamic, 4) num_threads(nt)
  for (int64_t i = 0; i < n_recv; ++i) {
    double* oi = out + i * (int64_t)D_out;
    for (int t = 0; t < D_out; ++t) oi[t] = 0.0;
    for (int64_t e = rowptr[i]; e < rowptr[i + 1]; ++e) {
      int64_t j = col[e];
      for (int p = 0; p < npaths; ++p) {
        const int32_t* P = paths + PI_N * p;
        int l1 = P[PI_L1], l2 = P[PI_L2], l3 = P[PI_L3];
        int n1 = 2 * l1 + 1, n2 = 2 * l2 + 1, n3 = 2 * l3 + 1;
        const double* C = cg + P[PI_COFF];
        for (int u = 0; u < P[PI_MUL]; ++u) {
          double w = W[e * U + P[PI_K0] + u];
          const double* xj = x + j * (int64_t)D_in + P[PI_XOFF] + u * n1;
          const double* ye = Y + e * (int64_t)D_e + l2 * l2;
          for (int m3 = 0; m3 < n3; ++m3) {
            double s = 0.0;
            for (int m1 = 0; m1 < n1; ++m1)
              for (int m2 = 0; m2 < n2; ++m2) {
                if (g_fault == 1 && m2 > 0) continue; /* mutation: dropped terms */
                s += C[(m1 * n2 + m2) * n3 + m3] * xj[m1] * ye[m2];
              }
            oi[P[PI_OOFF] + u * n3 + m3] += w * s;
          }
        }
      }
    }
  }
}

/* backward: given g = dL/dout, the three gradients of the trilinear map
 *   grad_x[j][x_off+u n1+m1] = sum_{e: col e = j} sum_{p,u} W[e][k0+u]
 *                                sum_{m2,m3} C Y[e][m2] g[row e][o_off+u n3+m3]
 *   grad_W[e][k0+u]          = sum_{m1,m2,m3} C x[col e][m1] Y[e][m2] g[row e][m3]
 *   grad_Y[e][l2^2+m2]       = sum_{p with this l2} sum_u W[e][k0+u]
 *                                sum_{m1,m3} C x[col e][m1] g[row e][m3]
 * Any of the three outputs may be NULL.  grad_x is accumulated by sender
 * through a transpose of the edge list, so the threaded loop has no race. */
void orc_backward(int64_t n_recv, int64_t n_send, int64_t E, const int64_t* rowptr,
                  const int32_t* col, int D_in, int D_e, int D_out, int U, const double* x,
                  const double* Y, const double* W, const double* g, int npaths,
                  const int32_t* paths, const double* cg, double* grad_x, double* grad_W,
                  double* grad_Y, int nthreads) {
  const int nt = orc_threads(nthreads);
  (void)nt;
  int64_t* recv_of = malloc(sizeof(int64_t) * (E > 0 ? E : 1));
  for (int64_t i = 0; i < n_recv; ++i)
    for (int64_t e = rowptr[i]; e < rowptr[i + 1]; ++e) recv_of[e] = i;

  if (grad_W || grad_Y) {
#pragma omp parallel for schedule(dynamic, 64) num_threads(nt)
    for (int64_t e = 0; e < E; ++e) {
      int64_t i = recv_of[e], j = col[e];
      if (grad_W)
        for (int k = 0; k < U; ++k) grad_W[e * U + k] = 0.0;
      if (grad_Y)
        for (int t = 0; t < D_e; ++t) grad_Y[e * D_e + t] = 0.0;
      for (int p = 0; p < npaths; ++p) {
        const int32_t* P = paths + PI_N * p;
        int l1 = P[PI_L1], l2 = P[PI_L2], l3 = P[PI_L3];
        int n1 = 2 * l1 + 1, n2 = 2 * l2 + 1, n3 = 2 * l3 + 1;
        const double* C = cg + P[PI_COFF];
        for (int u = 0; u < P[PI_MUL]; ++u) {
          int k = P[PI_K0] + u;
          double w = W[e * U + k];
          const double* xj = x + j * (int64_t)D_in + P[PI_XOFF] + u * n1;
          const double* ye = Y + e * (int64_t)D_e + l2 * l2;
          const double* gi = g + i * (int64_t)D_out + P[PI_OOFF] + u * n3;
          for (int m1 = 0; m1 < n1; ++m1)
            for (int m2 = 0; m2 < n2; ++m2)
              for (int m3 = 0; m3 < n3; ++m3) {
                double c = C[(m1 * n2 + m2) * n3 + m3];
                if (c == 0.0) continue;
                if (grad_W) grad_W[e * U + k] += c * xj[m1] * ye[m2] * gi[m3];
                if (grad_Y) grad_Y[e * D_e + l2 * l2 + m2] += c * w * xj[m1] * gi[m3];
              }
        }
      }
    }
  }

  if (grad_x) {
    /* transpose: edges grouped by sender, ascending edge id within a sender */
    int64_t* tptr = calloc((size_t)n_send + 1, sizeof(int64_t));
    int64_t* tedge = malloc(sizeof(int64_t) * (E > 0 ? E : 1));
    for (int64_t e = 0; e < E; ++e) tptr[col[e] + 1]++;
    for (int64_t j = 0; j < n_send; ++j) tptr[j + 1] += tptr[j];
    int64_t* fill = malloc(sizeof(int64_t) * (n_send > 0 ? n_send : 1));
    for (int64_t j = 0; j < n_send; ++j) fill[j] = tptr[j];
    for (int64_t e = 0; e < E; ++e) tedge[fill[col[e]]++] = e;
    free(fill);
#pragma omp parallel for schedule(dynamic, 4) num_threads(nt)
    for (int64_t j = 0; j < n_send; ++j) {
      double* dxj = grad_x + j * (int64_t)D_in;
      for (int t = 0; t < D_in; ++t) dxj[t] = 0.0;
      for (int64_t t = tptr[j]; t < tptr[j + 1]; ++t) {
        int64_t e = tedge[t], i = recv_of[e];
        for (int p = 0; p < npaths; ++p) {
          const int32_t* P = paths + PI_N * p;
          int l1 = P[PI_L1], l2 = P[PI_L2], l3 = P[PI_L3];
          int n1 = 2 * l1 + 1, n2 = 2 * l2 + 1, n3 = 2 * l3 + 1;
          const double* C = cg + P[PI_COFF];
          for (int u = 0; u < P[PI_MUL]; ++u) {
            double w = W[e * U + P[PI_K0] + u];
            const double* ye = Y + e * (int64_t)D_e + l2 * l2;
            const double* gi = g + i * (int64_t)D_out + P[PI_OOFF] + u * n3;
            for (int m1 = 0; m1 < n1; ++m1) {
              double s = 0.0;
              for (int m2 = 0; m2 < n2; ++m2)
                for (int m3 = 0; m3 < n3; ++m3) s += C[(m1 * n2 + m2) * n3 + m3] * ye[m2] * gi[m3];
              dxj[P[PI_XOFF] + u * n1 + m1] += w * s;
            }
          }
        }
      }
    }
    free(tptr);
    free(tedge);
  }
  free(recv_of);
}
