/*
 * oracle.c -- plain, slow, fp64 CPU reference for mesh gradient / block-CSR
 * Hessian assembly.  TEST INFRASTRUCTURE ONLY: nothing in the product library
 * links, calls or includes this file; only the test suite, the smoke check and
 * the benchmark's CPU-baseline leg load it.
 *
 * What it follows
 *   Page "Locality-Aware Automatic Differentiation on the GPU for Mesh-Based
 *   Computations" (reading note), section 方法 (method): a scalar objective
 *   F(x) = sum_j f_j(x_j) over local terms, each with a dense local gradient
 *   g_j and Hessian H_j, assembled as g = sum_j S_j^T g_j and
 *   H = sum_j S_j^T H_j S_j (S_j = selection matrix of the term's stencil);
 *   key design 3: the block sparsity of H is fixed by mesh connectivity and
 *   is preallocated as CSR; key design 4: runtime vertex-vertex pairs add
 *   off-diagonal blocks.
 *
 * How it computes it (deliberately the plain definition, no blocking, fusion
 * or reordering):
 *   1. every term evaluates a hand-derived closed form of E, g_j, H_j;
 *   2. each (row, col) block of S_j^T H_j S_j is appended to a COO list;
 *   3. the COO list is sorted by (row, col, emission order) and equal keys
 *      are summed in that order;
 *   4. the merged blocks are placed into the CSR pattern; a block whose key
 *      is absent from the pattern is an error.
 *   g is accumulated per vertex in term order.
 *
 * Readings of points the pages leave open (each also listed in the design
 * notes): the exact Hessian is assembled (no per-term PSD projection); the CSR
 * stores both triangles, 0-based int32, columns strictly ascending, diagonal
 * block always present, blocks contiguous and row-major inside a block;
 * g and x are [V][dof] interleaved.
 *
 * Energies (the page names the applications -- mass-spring cloth,
 * parameterization -- but prints no formulas; these are the standard forms):
 *   spring / pair  E = 1/2 k (|xi - xj| - L0)^2
 *   inertia        E = 1/2 w |xi - xt_i|^2          (w = m / h^2)
 *   sym. Dirichlet E = A (|J|_F^2 + |J^-1|_F^2),  J = [u1-u0, u2-u0] Dm^-1
 *   ARAP           E = A |J - R(J)|_F^2, R(J) the closest rotation
 *   area           E = 1/2 k (A - A0)^2 / A0  (3D triangle area A)
 *   vertex-face    E = 1/2 k (d - r)^2, d the signed distance of a vertex
 *                  to a triangle's plane
 *
 * Parity pins: every function here is pinned by tests/test_oracle.py against
 * closed-form values, finite differences, symmetry, translation / rotation
 * invariance and a brute-force pattern.  No function is "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OR_OK 0
#define OR_ERR_ARG -1
#define OR_ERR_CAPACITY -2
#define OR_ERR_NOT_IN_PATTERN -3
#define OR_ERR_OOM -4

/* Optional planted mistakes, compiled in only by the mutation test
 * (-DOR_MUTANT=n) to show that the pins catch each of them. */
#ifndef OR_MUTANT
#define OR_MUTANT 0
#endif

/* ------------------------------------------------------------------------ */
/* local terms: closed forms                                                 */
/* ------------------------------------------------------------------------ */

/* Spring between xi and xj in R^dof:  E = 1/2 k (l - L0)^2, l = |xi - xj|.
 * With n = (xi - xj)/l:
 *   dE/dxi = k (l - L0) n = -dE/dxj
 *   K = d2E/dxi2 = k [ n n^T + (1 - L0/l) (I - n n^T) ]
 *   H (2dof x 2dof, row-major) = [[K, -K], [-K, K]]                        */
void or_spring_local(int dof, const double* xi, const double* xj, double L0,
                     double k, double* E, double* g, double* H) {
  double d[3], l2 = 0.0;
  for (int a = 0; a < dof; ++a) {
    d[a] = xi[a] - xj[a];
    l2 += d[a] * d[a];
  }
  double l = sqrt(l2);
  double n[3];
  for (int a = 0; a < dof; ++a) n[a] = d[a] / l;
  double s = l - L0;
  *E = 0.5 * k * s * s;
  for (int a = 0; a < dof; ++a) {
    g[a] = k * s * n[a];
#if OR_MUTANT == 1 /* planted: wrong sign on the second endpoint */
    g[dof + a] = k * s * n[a];
#else
    g[dof + a] = -k * s * n[a];
#endif
  }
  double t = 1.0 - L0 / l;
#if OR_MUTANT == 2 /* planted: dropped geometric-stiffness term */
  t = 0.0;
#endif
  int N = 2 * dof;
  for (int a = 0; a < dof; ++a)
    for (int b = 0; b < dof; ++b) {
      double K = k * (n[a] * n[b] + t * ((a == b ? 1.0 : 0.0) - n[a] * n[b]));
      H[a * N + b] = K;
      H[(dof + a) * N + (dof + b)] = K;
      H[a * N + (dof + b)] = -K;
      H[(dof + a) * N + b] = -K;
    }
}

/* Inertia of one vertex: E = 1/2 w |xi - xt|^2, g = w (xi - xt), H = w I. */
void or_inertia_local(int dof, const double* xi, const double* xt, double w,
                      double* E, double* g, double* H) {
  double e = 0.0;
  for (int a = 0; a < dof; ++a) {
    double r = xi[a] - xt[a];
    e += r * r;
    g[a] = w * r;
    for (int b = 0; b < dof; ++b) H[a * dof + b] = (a == b) ? w : 0.0;
  }
  *E = 0.5 * w * e;
}

/* Symmetric Dirichlet energy of one triangle in 2D (UV):
 *   J = [u1-u0, u2-u0] M,  M = Dm^-1 (row-major 2x2), area A
 *   a = |J|_F^2, d = det J, |J^-1|_F^2 = a / d^2
 *   E = A (a + a / d^2)
 *   P = dE/dJ = A [ 2 (1 + d^-2) J - 2 a d^-3 C ],  C = cof J
 *   with j = vec J = (J00, J01, J10, J11), c = vec C and the constant
 *   Hessian Dd of det (Dd[0][3] = Dd[3][0] = 1, Dd[1][2] = Dd[2][1] = -1):
 *   HJ = A [ 2 (1 + d^-2) I4 - 4 d^-3 (j c^T + c j^T) + 6 a d^-4 c c^T
 *            - 2 a d^-3 Dd ]
 *   dJ[al][ga]/du_k[be] = delta(al,be) w_k[ga] with w1 = M row 0,
 *   w2 = M row 1, w0 = -(w1 + w2); so g_k[al] = sum_ga P[al][ga] w_k[ga] and
 *   H_kl[al][be] = sum_{ga,de} HJ[(al,ga),(be,de)] w_k[ga] w_l[de].
 * Output g[6] = (u0, u1, u2) interleaved, H 6x6 row-major.                  */
void or_symdir_local(const double* u0, const double* u1, const double* u2,
                     const double* M, double A, double* E, double* g,
                     double* H) {
  double Ds[2][2] = {{u1[0] - u0[0], u2[0] - u0[0]},
                     {u1[1] - u0[1], u2[1] - u0[1]}};
  double J[2][2];
  for (int al = 0; al < 2; ++al)
    for (int ga = 0; ga < 2; ++ga)
      J[al][ga] = Ds[al][0] * M[0 * 2 + ga] + Ds[al][1] * M[1 * 2 + ga];
  double a = J[0][0] * J[0][0] + J[0][1] * J[0][1] + J[1][0] * J[1][0] +
             J[1][1] * J[1][1];
  double d = J[0][0] * J[1][1] - J[0][1] * J[1][0];
  double C[2][2] = {{J[1][1], -J[1][0]}, {-J[0][1], J[0][0]}};
  double di = 1.0 / d;
  *E = A * (a + a * di * di);
  double P[2][2];
  for (int al = 0; al < 2; ++al)
    for (int ga = 0; ga < 2; ++ga)
      P[al][ga] = A * (2.0 * (1.0 + di * di) * J[al][ga] -
                       2.0 * a * di * di * di * C[al][ga]);
  double j[4] = {J[0][0], J[0][1], J[1][0], J[1][1]};
  double c[4] = {C[0][0], C[0][1], C[1][0], C[1][1]};
  double Dd[4][4] = {{0, 0, 0, 1}, {0, 0, -1, 0}, {0, -1, 0, 0}, {1, 0, 0, 0}};
  double HJ[4][4];
  for (int p = 0; p < 4; ++p)
    for (int q = 0; q < 4; ++q) {
      double v = 2.0 * (1.0 + di * di) * (p == q ? 1.0 : 0.0);
      v -= 4.0 * di * di * di * (j[p] * c[q] + c[p] * j[q]);
      v += 6.0 * a * di * di * di * di * c[p] * c[q];
      v -= 2.0 * a * di * di * di * Dd[p][q];
      HJ[p][q] = A * v;
    }
  double w[3][2];
  w[1][0] = M[0];
  w[1][1] = M[1];
  w[2][0] = M[2];
  w[2][1] = M[3];
  w[0][0] = -(w[1][0] + w[2][0]);
  w[0][1] = -(w[1][1] + w[2][1]);
  for (int kk = 0; kk < 3; ++kk)
    for (int al = 0; al < 2; ++al)
      g[2 * kk + al] = P[al][0] * w[kk][0] + P[al][1] * w[kk][1];
  for (int kk = 0; kk < 3; ++kk)
    for (int ll = 0; ll < 3; ++ll)
      for (int al = 0; al < 2; ++al)
        for (int be = 0; be < 2; ++be) {
          double s = 0.0;
          for (int ga = 0; ga < 2; ++ga)
            for (int de = 0; de < 2; ++de)
              s += HJ[2 * al + ga][2 * be + de] * w[kk][ga] * w[ll][de];
#if OR_MUTANT == 3 /* planted: transposed off-diagonal vertex block */
          if (kk != ll) {
            s = 0.0;
            for (int ga = 0; ga < 2; ++ga)
              for (int de = 0; de < 2; ++de)
                s += HJ[2 * be + ga][2 * al + de] * w[kk][ga] * w[ll][de];
          }
#endif
          H[(2 * kk + al) * 6 + (2 * ll + be)] = s;
        }
}

/* As-rigid-as-possible (ARAP) parameterization energy of one triangle:
 *   E = A |J - R(J)|_F^2,   J = [u1-u0, u2-u0] Dm^-1 (as for SymDir),
 * R(J) the rotation closest to J.  With j = (J00, J01, J10, J11),
 * p = J00 + J11 and q = J10 - J01, the closest rotation is
 * R = [[p, -q], [q, p]] / s with s = sqrt(p^2 + q^2) (the maximiser of
 * tr(R^T J) over rotations, whose maximum is s), so
 *   E = A (|J|^2 - 2 s + 2).
 * For det J > 0, s = sigma_1 + sigma_2 and E = A sum_i (sigma_i - 1)^2.
 *   dE/dj  = A (2 j - 2 ds/dj),   ds/dj = (p dp + q dq) / s,
 *   dp = (1, 0, 0, 1),  dq = (0, -1, 1, 0),
 *   d2E/dj2 = A (2 I - 2 d2s),
 *   d2s = (q^2 dp dp^T - p q (dp dq^T + dq dp^T) + p^2 dq dq^T) / s^3.
 * The map to the corners is SymDir's: g_k = P w_k, H_kl as there.
 * s > 0 whenever det J > 0 (s^2 = |J|^2 + 2 det J).
 * Output g[6] = (u0, u1, u2) interleaved, H 6x6 row-major.                  */
void or_arap_local(const double* u0, const double* u1, const double* u2,
                   const double* M, double A, double* E, double* g, double* H) {
  double Ds[2][2] = {{u1[0] - u0[0], u2[0] - u0[0]},
                     {u1[1] - u0[1], u2[1] - u0[1]}};
  double J[2][2];
  for (int al = 0; al < 2; ++al)
    for (int ga = 0; ga < 2; ++ga)
      J[al][ga] = Ds[al][0] * M[0 * 2 + ga] + Ds[al][1] * M[1 * 2 + ga];
  double j[4] = {J[0][0], J[0][1], J[1][0], J[1][1]};
  double p = j[0] + j[3];
  double q = j[2] - j[1];
  double s = sqrt(p * p + q * q);
  double a = j[0] * j[0] + j[1] * j[1] + j[2] * j[2] + j[3] * j[3];
  *E = A * (a - 2.0 * s + 2.0);
  const double dp[4] = {1.0, 0.0, 0.0, 1.0};
  const double dq[4] = {0.0, -1.0, 1.0, 0.0};
  double Pj[4];
  for (int r = 0; r < 4; ++r) Pj[r] = A * (2.0 * j[r] - 2.0 * (p * dp[r] + q * dq[r]) / s);
  double s3 = s * s * s;
  double HJ[4][4];
  for (int r = 0; r < 4; ++r)
    for (int c = 0; c < 4; ++c) {
#if OR_MUTANT == 8 /* planted: sign of the mixed p-q term of d2s flipped */
      double d2s = (q * q * dp[r] * dp[c] + p * q * (dp[r] * dq[c] + dq[r] * dp[c]) +
                    p * p * dq[r] * dq[c]) / s3;
#else
      double d2s = (q * q * dp[r] * dp[c] - p * q * (dp[r] * dq[c] + dq[r] * dp[c]) +
                    p * p * dq[r] * dq[c]) / s3;
#endif
      HJ[r][c] = A * (2.0 * (r == c ? 1.0 : 0.0) - 2.0 * d2s);
    }
  double w[3][2];
  w[1][0] = M[0];
  w[1][1] = M[1];
  w[2][0] = M[2];
  w[2][1] = M[3];
  w[0][0] = -(w[1][0] + w[2][0]);
  w[0][1] = -(w[1][1] + w[2][1]);
  for (int kk = 0; kk < 3; ++kk)
    for (int al = 0; al < 2; ++al)
      g[2 * kk + al] = Pj[2 * al] * w[kk][0] + Pj[2 * al + 1] * w[kk][1];
  for (int kk = 0; kk < 3; ++kk)
    for (int ll = 0; ll < 3; ++ll)
      for (int al = 0; al < 2; ++al)
        for (int be = 0; be < 2; ++be) {
          double t = 0.0;
          for (int ga = 0; ga < 2; ++ga)
            for (int de = 0; de < 2; ++de)
              t += HJ[2 * al + ga][2 * be + de] * w[kk][ga] * w[ll][de];
          H[(2 * kk + al) * 6 + (2 * ll + be)] = t;
        }
}

/* Area preservation of one triangle in 3D (a face term with a 9-variable
 * stencil): A = 1/2 |n|, n = e1 x e2, e1 = x1 - x0, e2 = x2 - x0,
 *   E = 1/2 k (A - A0)^2 / A0.
 * With [a] the cross-product matrix ([a] b = a x b), nh = n / |n|:
 *   dn/dx0 = [e2 - e1], dn/dx1 = -[e2], dn/dx2 = [e1]   (Jn, 3 x 9)
 *   dA = 1/2 Jn^T nh
 *   d2A = 1/2 ( Jn^T (I - nh nh^T) Jn / |n|  +  B ),
 *   B: n is bilinear in (e1, e2) with d2 n_c / de1_a de2_b = eps_cab, so
 *   sum_c nh_c d2 n_c is the form de1^T Q de2' + de1'^T Q de2 with
 *   Q[a][b] = sum_c eps_cab nh_c; e1 and e2 take x with coefficients
 *   p1 = (-1, 1, 0) and p2 = (-1, 0, 1), so block (i, j) of B is
 *   p1_i p2_j Q + p2_i p1_j Q^T.
 *   g = k (A - A0) / A0 dA,   H = k / A0 (dA dA^T + (A - A0) d2A).
 * Output g[9] = (x0, x1, x2), H 9x9 row-major.                             */
static void cross_mat(const double* a, double C[3][3]) {
  C[0][0] = 0.0;   C[0][1] = -a[2]; C[0][2] = a[1];
  C[1][0] = a[2];  C[1][1] = 0.0;   C[1][2] = -a[0];
  C[2][0] = -a[1]; C[2][1] = a[0];  C[2][2] = 0.0;
}

void or_area_local(const double* x0, const double* x1, const double* x2, double A0, double k,
                   double* E, double* g, double* H) {
  double e1[3], e2[3], d21[3], n[3];
  for (int a = 0; a < 3; ++a) {
    e1[a] = x1[a] - x0[a];
    e2[a] = x2[a] - x0[a];
    d21[a] = e2[a] - e1[a];
  }
  n[0] = e1[1] * e2[2] - e1[2] * e2[1];
  n[1] = e1[2] * e2[0] - e1[0] * e2[2];
  n[2] = e1[0] * e2[1] - e1[1] * e2[0];
  double l = sqrt(n[0] * n[0] + n[1] * n[1] + n[2] * n[2]);
  double nh[3] = {n[0] / l, n[1] / l, n[2] / l};
  double A = 0.5 * l;
  double C0[3][3], C1[3][3], C2[3][3];
  cross_mat(d21, C0);
  cross_mat(e2, C1);
  cross_mat(e1, C2);
  double Jn[3][9];
  for (int r = 0; r < 3; ++r)
    for (int c = 0; c < 3; ++c) {
      Jn[r][c] = C0[r][c];
      Jn[r][3 + c] = -C1[r][c];
      Jn[r][6 + c] = C2[r][c];
    }
  double dA[9];
  for (int q = 0; q < 9; ++q) {
    double s = 0.0;
    for (int r = 0; r < 3; ++r) s += Jn[r][q] * nh[r];
    dA[q] = 0.5 * s;
  }
  double P[3][3];  /* I - nh nh^T */
  for (int r = 0; r < 3; ++r)
    for (int c = 0; c < 3; ++c) P[r][c] = (r == c ? 1.0 : 0.0) - nh[r] * nh[c];
  double Q[3][3];
  for (int a = 0; a < 3; ++a)
    for (int b = 0; b < 3; ++b) {
      double s = 0.0;
      for (int c = 0; c < 3; ++c) {
        int eps = 0;
        if ((c == 0 && a == 1 && b == 2) || (c == 1 && a == 2 && b == 0) ||
            (c == 2 && a == 0 && b == 1))
          eps = 1;
        if ((c == 0 && a == 2 && b == 1) || (c == 1 && a == 0 && b == 2) ||
            (c == 2 && a == 1 && b == 0))
          eps = -1;
        s += eps * nh[c];
      }
      Q[a][b] = s;
    }
  const double p1[3] = {-1.0, 1.0, 0.0}, p2[3] = {-1.0, 0.0, 1.0};
  double d2A[9][9];
  for (int i = 0; i < 9; ++i)
    for (int j = 0; j < 9; ++j) {
      double s = 0.0;
      for (int r = 0; r < 3; ++r)
        for (int c = 0; c < 3; ++c) s += Jn[r][i] * P[r][c] * Jn[c][j];
      s /= l;
      int vi = i / 3, ai = i % 3, vj = j / 3, aj = j % 3;
      s += p1[vi] * p2[vj] * Q[ai][aj] + p2[vi] * p1[vj] * Q[aj][ai];
      d2A[i][j] = 0.5 * s;
    }
  double dev = A - A0;
  *E = 0.5 * k * dev * dev / A0;
  for (int q = 0; q < 9; ++q) g[q] = k * dev / A0 * dA[q];
  for (int i = 0; i < 9; ++i)
    for (int j = 0; j < 9; ++j) {
#if OR_MUTANT == 7 /* planted: bilinear part of d2A dropped */
      int vi = i / 3, ai = i % 3, vj = j / 3, aj = j % 3;
      double Bij = 0.5 * (p1[vi] * p2[vj] * Q[ai][aj] + p2[vi] * p1[vj] * Q[aj][ai]);
      H[i * 9 + j] = k / A0 * (dA[i] * dA[j] + dev * (d2A[i][j] - Bij));
#else
      H[i * 9 + j] = k / A0 * (dA[i] * dA[j] + dev * d2A[i][j]);
#endif
    }
}

/* Vertex-face term (a 4-vertex stencil p, a, b, c; 12 variables): the
 * signed distance from p to the plane of the triangle (a, b, c),
 *   d = u . nh,  u = p - a,  n = e1 x e2,  e1 = b - a,  e2 = c - a,  nh = n/|n|,
 * penalised as E = 1/2 k (d - r)^2.
 * With m = |n|:
 *   dd/du = nh,   dd/dn = w = (I - nh nh^T) u / m,
 *   d2d/du dn = (I - nh nh^T) / m,   d2d/du2 = 0,
 *   d2d/dn2 = (-(u nh^T + nh u^T) - d I + 3 d nh nh^T) / m^2.
 * u takes (p, a, b, c) with Ju = [I, -I, 0, 0]; n takes them with
 * Jn = [0, [e2 - e1], -[e2], [e1]] ([a] the cross-product matrix), and n is
 * bilinear in (e1, e2), which adds sum_c w_c d2 n_c: the form with
 * Q[a][b] = sum_c eps_cab w_c and corner coefficients p1 = (0, -1, 1, 0) on
 * e1 and p2 = (0, -1, 0, 1) on e2, block (i, j) = p1_i p2_j Q + p2_i p1_j Q^T.
 *   g = k (d - r) grad d,   H = k (grad d grad d^T + (d - r) hess d).
 * Output g[12] = (p, a, b, c), H 12x12 row-major.                          */
void or_vf_local(const double* p, const double* a, const double* b, const double* c, double r,
                 double k, double* E, double* g, double* H) {
  double u[3], e1[3], e2[3], d21[3], n[3];
  for (int q = 0; q < 3; ++q) {
    u[q] = p[q] - a[q];
    e1[q] = b[q] - a[q];
    e2[q] = c[q] - a[q];
    d21[q] = e2[q] - e1[q];
  }
  n[0] = e1[1] * e2[2] - e1[2] * e2[1];
  n[1] = e1[2] * e2[0] - e1[0] * e2[2];
  n[2] = e1[0] * e2[1] - e1[1] * e2[0];
  double m = sqrt(n[0] * n[0] + n[1] * n[1] + n[2] * n[2]);
  double nh[3] = {n[0] / m, n[1] / m, n[2] / m};
  double d = u[0] * nh[0] + u[1] * nh[1] + u[2] * nh[2];
  double P[3][3]; /* I - nh nh^T */
  for (int i = 0; i < 3; ++i)
    for (int j = 0; j < 3; ++j) P[i][j] = (i == j ? 1.0 : 0.0) - nh[i] * nh[j];
  double w[3];
  for (int i = 0; i < 3; ++i) w[i] = (P[i][0] * u[0] + P[i][1] * u[1] + P[i][2] * u[2]) / m;
  /* Jz = [Ju; Jn], 6 x 12 */
  double C0[3][3], C1[3][3], C2[3][3];
  cross_mat(d21, C0);
  cross_mat(e2, C1);
  cross_mat(e1, C2);
  double Jz[6][12];
  memset(Jz, 0, sizeof(Jz));
  for (int i = 0; i < 3; ++i) {
    Jz[i][i] = 1.0;
    Jz[i][3 + i] = -1.0;
    for (int j = 0; j < 3; ++j) {
      Jz[3 + i][3 + j] = C0[i][j];
      Jz[3 + i][6 + j] = -C1[i][j];
      Jz[3 + i][9 + j] = C2[i][j];
    }
  }
  double dz[6] = {nh[0], nh[1], nh[2], w[0], w[1], w[2]};
  double Dz[6][6];
  for (int i = 0; i < 3; ++i)
    for (int j = 0; j < 3; ++j) {
      Dz[i][j] = 0.0;
      Dz[i][3 + j] = P[i][j] / m;
      Dz[3 + i][j] = P[j][i] / m;
      Dz[3 + i][3 + j] = (-(u[i] * nh[j] + nh[i] * u[j]) - d * (i == j ? 1.0 : 0.0) +
                          3.0 * d * nh[i] * nh[j]) / (m * m);
    }
  double gd[12];
  for (int q = 0; q < 12; ++q) {
    double t = 0.0;
    for (int z = 0; z < 6; ++z) t += Jz[z][q] * dz[z];
    gd[q] = t;
  }
  double Q[3][3];
  for (int i = 0; i < 3; ++i)
    for (int j = 0; j < 3; ++j) {
      double t = 0.0;
      for (int cc = 0; cc < 3; ++cc) {
        int eps = 0;
        if ((cc == 0 && i == 1 && j == 2) || (cc == 1 && i == 2 && j == 0) ||
            (cc == 2 && i == 0 && j == 1))
          eps = 1;
        if ((cc == 0 && i == 2 && j == 1) || (cc == 1 && i == 0 && j == 2) ||
            (cc == 2 && i == 1 && j == 0))
          eps = -1;
        t += eps * w[cc];
      }
      Q[i][j] = t;
    }
  const double p1[4] = {0.0, -1.0, 1.0, 0.0}, p2[4] = {0.0, -1.0, 0.0, 1.0};
  double dev = d - r;
  *E = 0.5 * k * dev * dev;
  for (int q = 0; q < 12; ++q) g[q] = k * dev * gd[q];
  for (int i = 0; i < 12; ++i)
    for (int j = 0; j < 12; ++j) {
      double t = 0.0;
      for (int y = 0; y < 6; ++y)
        for (int z = 0; z < 6; ++z) t += Jz[y][i] * Dz[y][z] * Jz[z][j];
      int vi = i / 3, ai = i % 3, vj = j / 3, aj = j % 3;
#if OR_MUTANT != 9 /* planted (9): bilinear part of n dropped */
      t += p1[vi] * p2[vj] * Q[ai][aj] + p2[vi] * p1[vj] * Q[aj][ai];
#endif
      H[i * 12 + j] = k * (gd[i] * gd[j] + dev * t);
    }
}

/* ------------------------------------------------------------------------ */
/* COO machinery                                                             */
/* ------------------------------------------------------------------------ */

typedef struct {
  int32_t r, c;
  int64_t seq; /* emission order, makes the sort and the merge order fixed */
} or_key;

static int or_key_cmp(const void* pa, const void* pb) {
  const or_key* a = (const or_key*)pa;
  const or_key* b = (const or_key*)pb;
  if (a->r != b->r) return a->r < b->r ? -1 : 1;
  if (a->c != b->c) return a->c < b->c ? -1 : 1;
  if (a->seq != b->seq) return a->seq < b->seq ? -1 : 1;
  return 0;
}

/* Block sparsity pattern from topology (key design 3: fixed by connectivity
 * and the declared 1-ring neighbourhood; key design 4: plus runtime pairs):
 * {(i,i)} U {(a,b) : a != b share a face} U {(i,j),(j,i) : (i,j) a pair}.
 * Built as COO -> sort -> unique.  Returns nnzb, or OR_ERR_CAPACITY with
 * *needed set when cap is too small.                                        */
int or_pattern(int32_t V, int32_t nF, const int32_t* F, int32_t nP,
               const int32_t* P, int32_t* row_ptr, int32_t* col_idx,
               int64_t cap, int64_t* needed) {
  if (V < 0 || nF < 0 || nP < 0) return OR_ERR_ARG;
  int64_t n = (int64_t)V + 6 * (int64_t)nF + 2 * (int64_t)nP;
  or_key* keys = (or_key*)malloc(sizeof(or_key) * (size_t)(n > 0 ? n : 1));
  if (!keys) return OR_ERR_OOM;
  int64_t m = 0;
  for (int32_t i = 0; i < V; ++i) {
    keys[m].r = i;
    keys[m].c = i;
    keys[m].seq = m;
    ++m;
  }
  for (int32_t f = 0; f < nF; ++f)
    for (int p = 0; p < 3; ++p)
      for (int q = 0; q < 3; ++q) {
        if (p == q) continue;
        int32_t a = F[3 * f + p], b = F[3 * f + q];
        if (a < 0 || a >= V || b < 0 || b >= V || a == b) {
          free(keys);
          return OR_ERR_ARG;
        }
        keys[m].r = a;
        keys[m].c = b;
        keys[m].seq = m;
        ++m;
      }
  for (int32_t p = 0; p < nP; ++p) {
    int32_t i = P[2 * p], j = P[2 * p + 1];
    if (i < 0 || i >= V || j < 0 || j >= V || i == j) {
      free(keys);
      return OR_ERR_ARG;
    }
    keys[m].r = i;
    keys[m].c = j;
    keys[m].seq = m;
    ++m;
    keys[m].r = j;
    keys[m].c = i;
    keys[m].seq = m;
    ++m;
  }
  qsort(keys, (size_t)m, sizeof(or_key), or_key_cmp);
  int64_t u = 0;
  for (int64_t e = 0; e < m; ++e)
    if (e == 0 || keys[e].r != keys[e - 1].r || keys[e].c != keys[e - 1].c)
      ++u;
  if (needed) *needed = u;
  if (u > cap) {
    free(keys);
    return OR_ERR_CAPACITY;
  }
  for (int32_t i = 0; i <= V; ++i) row_ptr[i] = 0;
  u = 0;
  for (int64_t e = 0; e < m; ++e)
    if (e == 0 || keys[e].r != keys[e - 1].r || keys[e].c != keys[e - 1].c) {
      col_idx[u++] = keys[e].c;
      row_ptr[keys[e].r + 1] += 1;
    }
  for (int32_t i = 0; i < V; ++i) row_ptr[i + 1] += row_ptr[i];
  free(keys);
  return (int)u;
}

/* Unique undirected mesh edges (i < j), sorted by (i, j).  Returns E or an
 * error; *needed is set like or_pattern.                                    */
int or_edges(int32_t V, int32_t nF, const int32_t* F, int32_t* ij, int64_t cap,
             int64_t* needed) {
  int64_t n = 3 * (int64_t)nF;
  or_key* keys = (or_key*)malloc(sizeof(or_key) * (size_t)(n > 0 ? n : 1));
  if (!keys) return OR_ERR_OOM;
  int64_t m = 0;
  for (int32_t f = 0; f < nF; ++f)
    for (int p = 0; p < 3; ++p) {
      int32_t a = F[3 * f + p], b = F[3 * f + (p + 1) % 3];
      if (a < 0 || a >= V || b < 0 || b >= V || a == b) {
        free(keys);
        return OR_ERR_ARG;
      }
      keys[m].r = a < b ? a : b;
      keys[m].c = a < b ? b : a;
      keys[m].seq = m;
      ++m;
    }
  qsort(keys, (size_t)m, sizeof(or_key), or_key_cmp);
  int64_t u = 0;
  for (int64_t e = 0; e < m; ++e)
    if (e == 0 || keys[e].r != keys[e - 1].r || keys[e].c != keys[e - 1].c)
      ++u;
  if (needed) *needed = u;
  if (u > cap) {
    free(keys);
    return OR_ERR_CAPACITY;
  }
  u = 0;
  for (int64_t e = 0; e < m; ++e)
    if (e == 0 || keys[e].r != keys[e - 1].r || keys[e].c != keys[e - 1].c) {
      ij[2 * u] = keys[e].r;
      ij[2 * u + 1] = keys[e].c;
      ++u;
    }
  free(keys);
  return (int)u;
}

/* ------------------------------------------------------------------------ */
/* assembly                                                                  */
/* ------------------------------------------------------------------------ */

typedef struct {
  or_key* keys;
  double* vals; /* bs doubles per entry */
  int64_t n, cap;
  int bs;
} or_coo;

static int coo_push(or_coo* c, int32_t r, int32_t col, const double* blk) {
  if (c->n == c->cap) return OR_ERR_OOM;
  c->keys[c->n].r = r;
  c->keys[c->n].c = col;
  c->keys[c->n].seq = c->n;
  memcpy(c->vals + (size_t)c->n * c->bs, blk, sizeof(double) * c->bs);
  c->n += 1;
  return OR_OK;
}

/* Emit S^T H_j S for a term on `nv` vertices `vid` with local Hessian H of
 * size (nv*dof)^2 row-major: block (p, q) goes to global (vid[p], vid[q]). */
static int emit_blocks(or_coo* c, int dof, int nv, const int32_t* vid,
                       const double* H) {
  int N = nv * dof;
  double blk[9];
  for (int p = 0; p < nv; ++p)
    for (int q = 0; q < nv; ++q) {
      for (int a = 0; a < dof; ++a)
        for (int b = 0; b < dof; ++b)
          blk[a * dof + b] = H[(p * dof + a) * N + (q * dof + b)];
      int rc = coo_push(c, vid[p], vid[q], blk);
      if (rc) return rc;
    }
  return OR_OK;
}

/* Full assembly.  All float inputs are fp64 (the caller widens the stored
 * run-dtype values).  mask bits: 1 spring, 2 inertia, 4 symmetric Dirichlet,
 * 8 pairs.  Outputs: g [V][dof] (overwritten), H_vals [nnzb][dof][dof]
 * (overwritten; blocks absent from every term are zero), *energy.          */
/* mask bits: 1 spring, 2 inertia, 4 symmetric Dirichlet (dof 2, with Minv
 * and area = rest area), 8 pairs, 16 area preservation (dof 3, with area =
 * rest area A0 and stiffness ka), 32 ARAP (dof 2, with Minv and area, like
 * symmetric Dirichlet), 64 vertex-face terms (dof 3: term t couples vertex
 * vf[2t] with the corners of face vf[2t+1], rest offset vf_rest[t],
 * stiffness kc; the pattern must hold the blocks between the vertex and the
 * corners). */
int or_eval3(int32_t V, int dof, const double* x, unsigned mask,
             /* springs */ int32_t nE, const int32_t* edges, const double* L0,
             double k,
             /* inertia */ const double* xt, double w,
             /* faces */ int32_t nF, const int32_t* F,
             const double* Minv, const double* area,
             /* pairs */ int32_t nP, const int32_t* pairs, const double* prest,
             double kp,
             /* area preservation */ double ka,
             /* vertex-face */ int32_t nVF, const int32_t* vf, const double* vf_rest,
             double kc,
             /* pattern */ const int32_t* row_ptr, const int32_t* col_idx,
             /* out */ double* g, double* H_vals, double* energy);

int or_eval2(int32_t V, int dof, const double* x, unsigned mask,
             int32_t nE, const int32_t* edges, const double* L0, double k,
             const double* xt, double w, int32_t nF, const int32_t* F,
             const double* Minv, const double* area, int32_t nP, const int32_t* pairs,
             const double* prest, double kp, double ka, const int32_t* row_ptr,
             const int32_t* col_idx, double* g, double* H_vals, double* energy) {
  return or_eval3(V, dof, x, mask & ~64u, nE, edges, L0, k, xt, w, nF, F, Minv, area, nP, pairs,
                  prest, kp, ka, 0, NULL, NULL, 0.0, row_ptr, col_idx, g, H_vals, energy);
}

int or_eval3(int32_t V, int dof, const double* x, unsigned mask,
             /* springs */ int32_t nE, const int32_t* edges, const double* L0,
             double k,
             /* inertia */ const double* xt, double w,
             /* faces */ int32_t nF, const int32_t* F,
             const double* Minv, const double* area,
             /* pairs */ int32_t nP, const int32_t* pairs, const double* prest,
             double kp,
             /* area preservation */ double ka,
             /* vertex-face */ int32_t nVF, const int32_t* vf, const double* vf_rest,
             double kc,
             /* pattern */ const int32_t* row_ptr, const int32_t* col_idx,
             /* out */ double* g, double* H_vals, double* energy) {
  if (dof != 2 && dof != 3) return OR_ERR_ARG;
  if ((mask & 64) && dof != 3) return OR_ERR_ARG;
  if ((mask & 4) && dof != 2) return OR_ERR_ARG;
  if ((mask & 16) && dof != 3) return OR_ERR_ARG;
  if ((mask & 32) && dof != 2) return OR_ERR_ARG;
  int bs = dof * dof;
  int64_t n = 0;
  if (mask & 1) n += 4 * (int64_t)nE;
  if (mask & 2) n += V;
  if (mask & 4) n += 9 * (int64_t)nF;
  if (mask & 8) n += 4 * (int64_t)nP;
  if (mask & 16) n += 9 * (int64_t)nF;
  if (mask & 32) n += 9 * (int64_t)nF;
  if (mask & 64) n += 16 * (int64_t)nVF;
  or_coo c;
  c.bs = bs;
  c.cap = n > 0 ? n : 1;
  c.n = 0;
  c.keys = (or_key*)malloc(sizeof(or_key) * (size_t)c.cap);
  c.vals = (double*)malloc(sizeof(double) * (size_t)c.cap * bs);
  if (!c.keys || !c.vals) {
    free(c.keys);
    free(c.vals);
    return OR_ERR_OOM;
  }
  for (int64_t i = 0; i < (int64_t)V * dof; ++i) g[i] = 0.0;
  double Etot = 0.0, E, gl[12], Hl[144];
  int rc = OR_OK;
  if (mask & 1)
    for (int32_t e = 0; e < nE && !rc; ++e) {
      int32_t vid[2] = {edges[2 * e], edges[2 * e + 1]};
      or_spring_local(dof, x + (size_t)vid[0] * dof, x + (size_t)vid[1] * dof,
                      L0[e], k, &E, gl, Hl);
      Etot += E;
      for (int p = 0; p < 2; ++p)
        for (int a = 0; a < dof; ++a) g[(size_t)vid[p] * dof + a] += gl[p * dof + a];
      rc = emit_blocks(&c, dof, 2, vid, Hl);
    }
  if (mask & 2)
    for (int32_t i = 0; i < V && !rc; ++i) {
      or_inertia_local(dof, x + (size_t)i * dof, xt + (size_t)i * dof, w, &E,
                       gl, Hl);
      Etot += E;
      for (int a = 0; a < dof; ++a) g[(size_t)i * dof + a] += gl[a];
      rc = emit_blocks(&c, dof, 1, &i, Hl);
    }
  if (mask & 4)
    for (int32_t f = 0; f < nF && !rc; ++f) {
      const int32_t* vid = F + 3 * f;
      or_symdir_local(x + (size_t)vid[0] * 2, x + (size_t)vid[1] * 2,
                      x + (size_t)vid[2] * 2, Minv + 4 * (size_t)f, area[f], &E,
                      gl, Hl);
      Etot += E;
      for (int p = 0; p < 3; ++p)
        for (int a = 0; a < 2; ++a) g[(size_t)vid[p] * 2 + a] += gl[p * 2 + a];
      rc = emit_blocks(&c, 2, 3, vid, Hl);
    }
  if (mask & 32)
    for (int32_t f = 0; f < nF && !rc; ++f) {
      const int32_t* vid = F + 3 * f;
      or_arap_local(x + (size_t)vid[0] * 2, x + (size_t)vid[1] * 2, x + (size_t)vid[2] * 2,
                    Minv + 4 * (size_t)f, area[f], &E, gl, Hl);
      Etot += E;
      for (int p = 0; p < 3; ++p)
        for (int a = 0; a < 2; ++a) g[(size_t)vid[p] * 2 + a] += gl[p * 2 + a];
      rc = emit_blocks(&c, 2, 3, vid, Hl);
    }
  if (mask & 16)
    for (int32_t f = 0; f < nF && !rc; ++f) {
      const int32_t* vid = F + 3 * f;
      or_area_local(x + (size_t)vid[0] * 3, x + (size_t)vid[1] * 3, x + (size_t)vid[2] * 3,
                    area[f], ka, &E, gl, Hl);
      Etot += E;
      for (int p = 0; p < 3; ++p)
        for (int a = 0; a < 3; ++a) g[(size_t)vid[p] * 3 + a] += gl[p * 3 + a];
      rc = emit_blocks(&c, 3, 3, vid, Hl);
    }
  if (mask & 64)
    for (int32_t t = 0; t < nVF && !rc; ++t) {
      const int32_t f = vf[2 * t + 1];
      if (f < 0 || f >= nF) {
        rc = OR_ERR_ARG;
        break;
      }
      int32_t vid[4] = {vf[2 * t], F[3 * f], F[3 * f + 1], F[3 * f + 2]};
      or_vf_local(x + (size_t)vid[0] * 3, x + (size_t)vid[1] * 3, x + (size_t)vid[2] * 3,
                  x + (size_t)vid[3] * 3, vf_rest[t], kc, &E, gl, Hl);
      Etot += E;
      for (int q = 0; q < 4; ++q)
        for (int a = 0; a < 3; ++a) g[(size_t)vid[q] * 3 + a] += gl[q * 3 + a];
      rc = emit_blocks(&c, 3, 4, vid, Hl);
    }
  if (mask & 8)
    for (int32_t p = 0; p < nP && !rc; ++p) {
      int32_t vid[2] = {pairs[2 * p], pairs[2 * p + 1]};
      or_spring_local(dof, x + (size_t)vid[0] * dof, x + (size_t)vid[1] * dof,
                      prest[p], kp, &E, gl, Hl);
      Etot += E;
      for (int q = 0; q < 2; ++q)
        for (int a = 0; a < dof; ++a) g[(size_t)vid[q] * dof + a] += gl[q * dof + a];
      rc = emit_blocks(&c, dof, 2, vid, Hl);
    }
  if (rc) {
    free(c.keys);
    free(c.vals);
    return rc;
  }
  *energy = Etot;
  /* sort an index permutation by (r, c, seq), then merge equal keys in order */
  qsort(c.keys, (size_t)c.n, sizeof(or_key), or_key_cmp);
  int64_t nnzb = row_ptr[V];
  for (int64_t i = 0; i < nnzb * bs; ++i) H_vals[i] = 0.0;
  int64_t e = 0;
  while (e < c.n) {
    int32_t r = c.keys[e].r, col = c.keys[e].c;
    double acc[9] = {0};
    while (e < c.n && c.keys[e].r == r && c.keys[e].c == col) {
      const double* v = c.vals + (size_t)c.keys[e].seq * bs;
      for (int t = 0; t < bs; ++t) acc[t] += v[t];
      ++e;
    }
#if OR_MUTANT == 4 /* planted: merge keeps only the last contribution */
    {
      const double* v = c.vals + (size_t)c.keys[e - 1].seq * bs;
      for (int t = 0; t < bs; ++t) acc[t] = v[t];
    }
#endif
    /* locate (r, col) in the pattern by a linear walk of row r */
    int64_t pos = -1;
    for (int64_t q = row_ptr[r]; q < row_ptr[r + 1]; ++q)
      if (col_idx[q] == col) {
        pos = q;
        break;
      }
    if (pos < 0) {
      rc = OR_ERR_NOT_IN_PATTERN;
      break;
    }
    for (int t = 0; t < bs; ++t) H_vals[pos * bs + t] = acc[t];
  }
  free(c.keys);
  free(c.vals);
  return rc;
}

/* Matrix-free product reference: y = H v with H the assembled block CSR
 * (the parameterization workload's Hessian-vector product).               */
int or_eval(int32_t V, int dof, const double* x, unsigned mask, int32_t nE,
            const int32_t* edges, const double* L0, double k, const double* xt, double w,
            int32_t nF, const int32_t* F, const double* Minv, const double* area, int32_t nP,
            const int32_t* pairs, const double* prest, double kp, const int32_t* row_ptr,
            const int32_t* col_idx, double* g, double* H_vals, double* energy) {
  return or_eval2(V, dof, x, mask & ~16u, nE, edges, L0, k, xt, w, nF, F, Minv, area, nP, pairs,
                  prest, kp, 0.0, row_ptr, col_idx, g, H_vals, energy);
}

int or_bsr_mv(int32_t V, int dof, const int32_t* row_ptr,
              const int32_t* col_idx, const double* H_vals, const double* v,
              double* y) {
  int bs = dof * dof;
  for (int32_t i = 0; i < V; ++i) {
    for (int a = 0; a < dof; ++a) {
      double s = 0.0;
      for (int32_t q = row_ptr[i]; q < row_ptr[i + 1]; ++q) {
        int32_t j = col_idx[q];
        for (int b = 0; b < dof; ++b)
          s += H_vals[(size_t)q * bs + a * dof + b] * v[(size_t)j * dof + b];
      }
      y[(size_t)i * dof + a] = s;
    }
  }
  return OR_OK;
}

/* ------------------------------------------------------------------------ */
/* vector-valued objective: residuals and the sparse Jacobian                */
/* ------------------------------------------------------------------------ */
/* Page "Locality-Aware Automatic Differentiation on the GPU for Mesh-Based
 * Computations", section 方法: a vector-valued objective assembles the sparse
 * Jacobian J = sum_j P_j^T J_j S_j, with S_j the term's stencil selection
 * and P_j placing the term's residuals in the global residual vector.
 *
 * Residual form of each mesh term, chosen so that F = 1/2 |r|^2 equals the
 * scalar energy above (so J^T r = g and J^T J is the Gauss-Newton part of H):
 *   spring  r = sqrt(k) (l - L0)                       1 residual
 *           dr/dxi = sqrt(k) n^T = -dr/dxj
 *   inertia r = sqrt(w) (xi - xt)                      dof residuals
 *           dr/dxi = sqrt(w) I
 *   SymDir  r = sqrt(2A) (vec J, vec J^-1)             8 residuals
 *           d(vec J)[2al+ga]/du_k[be] = delta(al,be) w_k[ga]
 *           d(J^-1)[m][n]/du_k[be] = -J^-1[m][be] (w_k^T J^-1)[n]
 *           (from d(J^-1) = -J^-1 dJ J^-1), vec J^-1 = (m, n) -> 2m+n.
 * Rows: the active term types in the order springs (edge order), inertia
 * (vertex order, dof rows each), faces (face order, 8 rows each).  Columns:
 * vertex * dof + component, ascending within each row (the stencil's
 * vertices sorted by index).                                                 */

/* Residuals r[1] and the 1 x 2dof Jacobian of one spring (xi, xj order). */
void or_spring_res(int dof, const double* xi, const double* xj, double L0, double k,
                   double* r, double* Jl) {
  double d[3], l2 = 0.0;
  for (int a = 0; a < dof; ++a) {
    d[a] = xi[a] - xj[a];
    l2 += d[a] * d[a];
  }
  double l = sqrt(l2), sk = sqrt(k);
  r[0] = sk * (l - L0);
  for (int a = 0; a < dof; ++a) {
    Jl[a] = sk * d[a] / l;
    Jl[dof + a] = -sk * d[a] / l;
  }
}

/* Residuals r[8] and the 8 x 6 Jacobian (row-major, columns u0, u1, u2
 * interleaved) of one symmetric Dirichlet face. */
void or_symdir_res(const double* u0, const double* u1, const double* u2, const double* M,
                   double A, double* r, double* Jl) {
  double J[2][2];
  for (int al = 0; al < 2; ++al)
    for (int ga = 0; ga < 2; ++ga)
      J[al][ga] = (u1[al] - u0[al]) * M[0 * 2 + ga] + (u2[al] - u0[al]) * M[1 * 2 + ga];
  double d = J[0][0] * J[1][1] - J[0][1] * J[1][0];
  double Ji[2][2] = {{J[1][1] / d, -J[0][1] / d}, {-J[1][0] / d, J[0][0] / d}};
  double s = sqrt(2.0 * A);
#if OR_MUTANT == 5 /* planted: residual scale sqrt(A) (F = E / 2) */
  s = sqrt(A);
#endif
  for (int p = 0; p < 4; ++p) r[p] = s * J[p / 2][p % 2];
  for (int p = 0; p < 4; ++p) r[4 + p] = s * Ji[p / 2][p % 2];
  double w[3][2];
  w[1][0] = M[0];
  w[1][1] = M[1];
  w[2][0] = M[2];
  w[2][1] = M[3];
  w[0][0] = -(w[1][0] + w[2][0]);
  w[0][1] = -(w[1][1] + w[2][1]);
  for (int kk = 0; kk < 3; ++kk) {
    double wJi[2];  /* w_k^T J^-1 */
    for (int n = 0; n < 2; ++n) wJi[n] = w[kk][0] * Ji[0][n] + w[kk][1] * Ji[1][n];
    for (int be = 0; be < 2; ++be) {
      int col = 2 * kk + be;
      for (int al = 0; al < 2; ++al)
        for (int ga = 0; ga < 2; ++ga)
          Jl[(2 * al + ga) * 6 + col] = s * (al == be ? w[kk][ga] : 0.0);
      for (int m = 0; m < 2; ++m)
        for (int n = 0; n < 2; ++n) {
#if OR_MUTANT == 6 /* planted: d(J^-1) with the factors' indices swapped */
          Jl[(4 + 2 * m + n) * 6 + col] = -s * Ji[be][m] * wJi[n];
#else
          Jl[(4 + 2 * m + n) * 6 + col] = -s * Ji[m][be] * wJi[n];
#endif
        }
    }
  }
}

typedef struct {
  int32_t col;
  double v;
} or_cv;

static int or_cv_cmp(const void* pa, const void* pb) {
  const or_cv* a = (const or_cv*)pa;
  const or_cv* b = (const or_cv*)pb;
  return (a->col > b->col) - (a->col < b->col);
}

/* Writes one row: the entries (vertex vid[s], component c) -> Jrow[s*dof+c]
 * for the nv stencil vertices, sorted by column. */
static void put_row(int dof, int nv, const int32_t* vid, const double* Jrow, int64_t* q,
                    int32_t* col_idx, double* vals) {
  or_cv e[9];
  int n = 0;
  for (int s = 0; s < nv; ++s)
    for (int c = 0; c < dof; ++c) {
      e[n].col = vid[s] * dof + c;
      e[n].v = Jrow[s * dof + c];
      ++n;
    }
  qsort(e, (size_t)n, sizeof(or_cv), or_cv_cmp);
  for (int t = 0; t < n; ++t) {
    col_idx[*q] = e[t].col;
    vals[*q] = e[t].v;
    ++*q;
  }
}

/* Residual vector r and CSR Jacobian (row_ptr[nrows+1], col_idx, vals) of
 * the active mesh terms (mask bits 1 spring, 2 inertia, 4 SymDir).  The
 * caller sizes the outputs with or_jacobian_shape.  Inertia rows hold their
 * single nonzero.  Returns OR_OK or an error. */
int or_jacobian_shape(int32_t V, int dof, unsigned mask, int32_t nE, int32_t nF,
                      int64_t* nrows, int64_t* nnz) {
  int64_t r = 0, z = 0;
  if (mask & 1u) { r += nE; z += (int64_t)nE * 2 * dof; }
  if (mask & 2u) { r += (int64_t)V * dof; z += (int64_t)V * dof; }
  if (mask & 4u) {
    if (dof != 2) return OR_ERR_ARG;
    r += (int64_t)nF * 8;
    z += (int64_t)nF * 8 * 6;
  }
  *nrows = r;
  *nnz = z;
  return OR_OK;
}

int or_jacobian(int32_t V, int dof, const double* x, unsigned mask, int32_t nE,
                const int32_t* edges, const double* L0, double k, const double* xt, double w,
                int32_t nF, const int32_t* F, const double* Minv, const double* area,
                double* r, int64_t* row_ptr, int32_t* col_idx, double* vals) {
  if (dof < 2 || dof > 3 || ((mask & 4u) && dof != 2)) return OR_ERR_ARG;
  int64_t row = 0, q = 0;
  row_ptr[0] = 0;
  if (mask & 1u) {
    for (int32_t e = 0; e < nE; ++e) {
      int32_t vid[2] = {edges[2 * e], edges[2 * e + 1]};
      double Jl[6];
      or_spring_res(dof, x + (size_t)vid[0] * dof, x + (size_t)vid[1] * dof, L0[e], k,
                    r + row, Jl);
      put_row(dof, 2, vid, Jl, &q, col_idx, vals);
      row_ptr[++row] = q;
    }
  }
  if (mask & 2u) {
    double sw = sqrt(w);
    for (int32_t v = 0; v < V; ++v)
      for (int a = 0; a < dof; ++a) {
        r[row] = sw * (x[(size_t)v * dof + a] - xt[(size_t)v * dof + a]);
        col_idx[q] = v * dof + a;
        vals[q] = sw;
        ++q;
        row_ptr[++row] = q;
      }
  }
  if (mask & 4u) {
    for (int32_t f = 0; f < nF; ++f) {
      const int32_t* vid = F + 3 * (size_t)f;
      double Jl[48];
      or_symdir_res(x + (size_t)vid[0] * 2, x + (size_t)vid[1] * 2, x + (size_t)vid[2] * 2,
                    Minv + 4 * (size_t)f, area[f], r + row, Jl);
      for (int p = 0; p < 8; ++p) {
        put_row(2, 3, vid, Jl + 6 * p, &q, col_idx, vals);
        row_ptr[++row] = q;
      }
    }
  }
  return OR_OK;
}
