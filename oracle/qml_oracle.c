/*
 * qml_oracle.c -- TEST INFRASTRUCTURE, not part of the product.
 *
 * A plain, slow, gate-by-gate complex128 simulator of the hardware-efficient
 * ansatz (HEA) and of its adjoint-method gradient.  It exists only so that the
 * tests, the smoke check and the benchmark's CPU-baseline leg have something
 * obviously correct to compare the CUDA path with.  Only tests/,
 * __graft_entry__.smoke() and bench.py (cpu_baseline / --impl reference) may
 * load it.  It shares no code, header, table or schedule with the CUDA
 * library, and the CUDA library never calls it.
 *
 * Sources (the method is described on five web summaries of Kawase,
 * "Fast and memory-efficient classical simulation of quantum machine learning
 * via forward and backward gate fusion", arXiv 2603.02804):
 *   [Deep-dive]  the Chinese blog "深度解析：正向与反向门融合驱动的高效量子机器学习仿真",
 *                §1.2 (state vector in C^{2^n}; E(theta) = <psi_M|O|psi_M>;
 *                adjoint gradient Re<lambda_j|dU_j/dtheta_j|psi_{j-1}>;
 *                lambda_{j-1} = U_j^dagger lambda_j), §2.1 (HEA = Rx, Ry, Rz
 *                single-qubit rotations plus CZ entanglers).
 *   [Gist-EN]    gist.science "Fast and memory-efficient classical simulation
 *                of quantum machine learning via forward and backward gate
 *                fusion", Technical Summary §2 (adjoint backward walks the
 *                gates in reverse, rebuilding each gate's input state).
 *
 * Readings where the pages are silent (each one is listed with its reason in
 * the design notes of the repository):
 *   - R_P(t) = exp(-i t P / 2) for P in {X, Y, Z};
 *   - a layer is Rx(theta[l][q][0]), Ry(theta[l][q][1]), Rz(theta[l][q][2])
 *     on every qubit q, then CZ(q, q+1) for q = 0 .. n-2 (open chain); other
 *     bond lists, and CNOT(control, target) instead of CZ on each bond (the
 *     pages name CNOT gates as the other entangler they fuse, [Deep-dive]
 *     sec. 3.2), are options;
 *   - the input x is angle-encoded once, Ry(x_q) on |0...0>, before layer 0;
 *   - qubit q is bit q of the amplitude index (qubit 0 = least significant);
 *   - the observable is Z on qubit 0;
 *   - the gradient carries the factor 2 that the printed adjoint formula
 *     omits: dL/dtheta_j = 2 Re<lambda_j| dU_j/dtheta_j |psi_{j-1}> with
 *     lambda_M = (dL/dE) Z0 psi_M.  This is the derivative of
 *     <psi|O|psi>, and the tests pin it against parameter shift.
 *
 * Everything is fp64 / complex128.  OpenMP parallelises over samples, or
 * over amplitude pairs when the state is large; neither changes what is
 * computed, only which core does it.
 */
#include <complex.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef double complex cplx;

enum { PX = 0, PY = 1, PZ = 2 };
enum { G_ROT = 0, G_CZ = 1, G_CNOT = 2 };
/* Entangler kinds: CZ on each bond, or CNOT(control, target) on each bond. */
enum { ENT_CZ = 0, ENT_CNOT = 1 };

typedef struct {
  cplx m[2][2];
} mat2;

/* One gate of the circuit, in the order it is applied. */
typedef struct {
  int kind;    /* G_ROT, G_CZ or G_CNOT */
  int pauli;   /* PX, PY, PZ for G_ROT */
  int q, q2;   /* target qubit; second qubit for CZ; control (q) and target (q2) for CNOT */
  double angle;
  long param;  /* index into theta[L][n][3], or -1 for a fixed (encoding) gate */
} gate;

/* States larger than this are updated with an amplitude-parallel loop. */
#define PAR_AMP_MIN_QUBITS 16

/* ---------------------------------------------------------------- 2x2 algebra */

static mat2 pauli(int p) {
  mat2 r;
  memset(&r, 0, sizeof r);
  if (p == PX) { r.m[0][1] = 1; r.m[1][0] = 1; }
  if (p == PY) { r.m[0][1] = -I; r.m[1][0] = I; }
  if (p == PZ) { r.m[0][0] = 1; r.m[1][1] = -1; }
  return r;
}

static mat2 mat_mul(mat2 a, mat2 b) {
  mat2 r;
  for (int i = 0; i < 2; ++i)
    for (int j = 0; j < 2; ++j) r.m[i][j] = a.m[i][0] * b.m[0][j] + a.m[i][1] * b.m[1][j];
  return r;
}

static mat2 mat_scale(mat2 a, cplx s) {
  for (int i = 0; i < 2; ++i)
    for (int j = 0; j < 2; ++j) a.m[i][j] *= s;
  return a;
}

static mat2 dagger(mat2 a) {
  mat2 r;
  for (int i = 0; i < 2; ++i)
    for (int j = 0; j < 2; ++j) r.m[i][j] = conj(a.m[j][i]);
  return r;
}

/* R_P(t) = exp(-i t P / 2) = cos(t/2) I - i sin(t/2) P, since P^2 = I. */
static mat2 rotation(int p, double t) {
  mat2 P = pauli(p), r;
  double c = cos(0.5 * t), s = sin(0.5 * t);
  for (int i = 0; i < 2; ++i)
    for (int j = 0; j < 2; ++j) r.m[i][j] = (i == j ? c : 0.0) - I * s * P.m[i][j];
  return r;
}

/* d/dt R_P(t) = (-i/2) P R_P(t). */
static mat2 rotation_derivative(int p, double t) {
  return mat_scale(mat_mul(pauli(p), rotation(p, t)), -0.5 * I);
}

/* ------------------------------------------------------------ state kernels */

/* psi <- (u acting on qubit q) psi */
static void apply_1q(cplx* psi, int n, int q, mat2 u) {
  const size_t half = (size_t)1 << (n - 1);
  const size_t bit = (size_t)1 << q;
#pragma omp parallel for schedule(static) if (n >= PAR_AMP_MIN_QUBITS)
  for (size_t k = 0; k < half; ++k) {
    /* k enumerates the indices with bit q cleared */
    size_t i0 = ((k >> q) << (q + 1)) | (k & (bit - 1));
    size_t i1 = i0 | bit;
    cplx a = psi[i0], b = psi[i1];
    psi[i0] = u.m[0][0] * a + u.m[0][1] * b;
    psi[i1] = u.m[1][0] * a + u.m[1][1] * b;
  }
}

/* psi <- CZ(q1, q2) psi: amplitudes with both bits set change sign. */
static void apply_cz(cplx* psi, int n, int q1, int q2) {
  const size_t N = (size_t)1 << n;
  const size_t m = ((size_t)1 << q1) | ((size_t)1 << q2);
#pragma omp parallel for schedule(static) if (n >= PAR_AMP_MIN_QUBITS)
  for (size_t i = 0; i < N; ++i)
    if ((i & m) == m) psi[i] = -psi[i];
}

/* psi <- CNOT(c, t) psi: where bit c is set, the amplitudes with bit t = 0
 * and bit t = 1 trade places (X on the target, controlled by c). */
static void apply_cnot(cplx* psi, int n, int c, int t) {
  const size_t half = (size_t)1 << (n - 1);
  const size_t tbit = (size_t)1 << t, cbit = (size_t)1 << c;
#pragma omp parallel for schedule(static) if (n >= PAR_AMP_MIN_QUBITS)
  for (size_t k = 0; k < half; ++k) {
    size_t i0 = ((k >> t) << (t + 1)) | (k & (tbit - 1));
    if (!(i0 & cbit)) continue;
    cplx a = psi[i0];
    psi[i0] = psi[i0 | tbit];
    psi[i0 | tbit] = a;
  }
}

/* <lambda| (d acting on qubit q) |phi>, summed pair by pair (no temporary). */
static cplx local_braket(const cplx* lam, const cplx* phi, int n, int q, mat2 d) {
  const size_t half = (size_t)1 << (n - 1);
  const size_t bit = (size_t)1 << q;
  double re = 0.0, im = 0.0;
#pragma omp parallel for schedule(static) reduction(+ : re, im) if (n >= PAR_AMP_MIN_QUBITS)
  for (size_t k = 0; k < half; ++k) {
    size_t i0 = ((k >> q) << (q + 1)) | (k & (bit - 1));
    size_t i1 = i0 | bit;
    cplx a = phi[i0], b = phi[i1];
    cplx t = conj(lam[i0]) * (d.m[0][0] * a + d.m[0][1] * b) +
             conj(lam[i1]) * (d.m[1][0] * a + d.m[1][1] * b);
    re += creal(t);
    im += cimag(t);
  }
  return re + I * im;
}

/* E = <psi| Z0 |psi> = sum_i |psi_i|^2 (+1 if bit 0 of i is 0, else -1). */
static double expect_z0(const cplx* psi, int n) {
  const size_t N = (size_t)1 << n;
  double e = 0.0;
#pragma omp parallel for schedule(static) reduction(+ : e) if (n >= PAR_AMP_MIN_QUBITS)
  for (size_t i = 0; i < N; ++i) {
    double p = creal(psi[i]) * creal(psi[i]) + cimag(psi[i]) * cimag(psi[i]);
    e += (i & 1) ? -p : p;
  }
  return e;
}

/*
 * Observable H = sum_k coef[k] P_k, P_k a tensor product of one-qubit Paulis:
 * character paulis[k*n + q] in {'I','X','Y','Z'} is the factor on qubit q.
 * This is the general observable O of E(theta) = <psi|O|psi> ([Deep-dive]
 * sec. 1.2); the Pauli strings are applied as explicit 2x2 matrices, one qubit
 * at a time.  out <- H psi, using tmp as scratch.  Returns -1 on a bad letter.
 */
static int pauli_index(char c) {
  return c == 'X' ? PX : c == 'Y' ? PY : c == 'Z' ? PZ : c == 'I' ? -1 : -2;
}

static int apply_observable(const cplx* psi, cplx* out, cplx* tmp, int n, int nterms, const char* paulis,
                            const double* coef) {
  const size_t N = (size_t)1 << n;
  for (size_t i = 0; i < N; ++i) out[i] = 0;
  for (int k = 0; k < nterms; ++k) {
    memcpy(tmp, psi, sizeof(cplx) * N);
    for (int q = 0; q < n; ++q) {
      int p = pauli_index(paulis[(size_t)k * n + q]);
      if (p == -2) return -1;
      if (p >= 0) apply_1q(tmp, n, q, pauli(p));
    }
    for (size_t i = 0; i < N; ++i) out[i] += coef[k] * tmp[i];
  }
  return 0;
}

/* Re <a|b> */
static double re_inner(const cplx* a, const cplx* b, int n) {
  const size_t N = (size_t)1 << n;
  double e = 0.0;
#pragma omp parallel for schedule(static) reduction(+ : e) if (n >= PAR_AMP_MIN_QUBITS)
  for (size_t i = 0; i < N; ++i) e += creal(conj(a[i]) * b[i]);
  return e;
}

/* ----------------------------------------------------------------- circuit */

/* Number of gates: n encoding rotations + L * (3n rotations + (n-1) CZ). */
/* Entangler of every layer: CZ on each bond (a, b) of a list, in list order.
 * bonds == NULL means the open chain CZ(q, q+1), q = 0 .. n-2. */
static int n_bonds_of(int n, int nbonds, const int* bonds) { return bonds ? nbonds : n - 1; }

/* Gate count: the encoding, then per layer (the encoding again when data is
 * re-uploaded) 3n rotations and the entangler's CZ gates. */
static long circuit_len(int n, int L, int nb, int reupload) {
  return (long)n + (long)L * ((reupload ? 4 : 3) * (long)n + nb);
}

/* The circuit as a flat, ordered gate list for one sample.  With reupload,
 * every layer starts with the angle encoding Ry(x_q) on every qubit again
 * (data re-uploading); those gates carry no parameter. */
static void build_circuit(gate* g, int n, int L, const double* x, const double* theta, int nbonds,
                          const int* bonds, int reupload, int ent) {
  long k = 0;
  for (int q = 0; q < n; ++q) { /* angle encoding Ry(x_q)|0> */
    gate e = {G_ROT, PY, q, -1, x[q], -1};
    g[k++] = e;
  }
  const int nb = n_bonds_of(n, nbonds, bonds);
  for (int l = 0; l < L; ++l) {
    if (reupload)
      for (int q = 0; q < n; ++q) {
        gate e = {G_ROT, PY, q, -1, x[q], -1};
        g[k++] = e;
      }
    for (int q = 0; q < n; ++q)
      for (int a = 0; a < 3; ++a) { /* Rx, then Ry, then Rz */
        long pi = ((long)l * n + q) * 3 + a;
        gate r = {G_ROT, a, q, -1, theta[pi], pi};
        g[k++] = r;
      }
    for (int e = 0; e < nb; ++e) { /* entangler: CZ or CNOT(control, target) per bond, in list order */
      gate c = {ent == ENT_CNOT ? G_CNOT : G_CZ, 0, bonds ? bonds[2 * e] : e, bonds ? bonds[2 * e + 1] : e + 1,
                0.0, -1};
      g[k++] = c;
    }
  }
}

static int bad_bonds(int n, int nbonds, const int* bonds) {
  if (!bonds) return 0;
  if (nbonds < 0) return 1;
  for (int e = 0; e < nbonds; ++e) {
    int a = bonds[2 * e], b = bonds[2 * e + 1];
    if (a < 0 || b < 0 || a >= n || b >= n || a == b) return 1;
  }
  return 0;
}

static void apply_gate(cplx* psi, int n, const gate* g, int inverse) {
  if (g->kind == G_CZ) {
    apply_cz(psi, n, g->q, g->q2); /* CZ is its own inverse */
  } else if (g->kind == G_CNOT) {
    apply_cnot(psi, n, g->q, g->q2); /* so is CNOT */
  } else {
    mat2 u = rotation(g->pauli, g->angle);
    apply_1q(psi, n, g->q, inverse ? dagger(u) : u);
  }
}

static void zero_state(cplx* psi, int n) {
  memset(psi, 0, sizeof(cplx) * ((size_t)1 << n));
  psi[0] = 1.0;
}

/* ----------------------------------------------------------------- exports */

int oracle_version(void) { return 5; }

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

static int bad_args(int n, int L, int B) { return n < 1 || n > 30 || L < 0 || B < 0; }

/*
 * Forward pass for B samples with observable H (nterms > 0; see
 * apply_observable) or Z0 (nterms == 0).
 *   x      [B][n]     encoding angles
 *   theta  [L][n][3]  rotation angles (Rx, Ry, Rz per qubit per layer)
 *   expect [B]        out: <H> of the final state             (may be NULL)
 *   psi    [B][2^n][2] out: final state as (re, im) doubles    (may be NULL)
 * Returns 0, or -1 on bad arguments / allocation failure.
 */
int oracle_forward_ent(int n, int L, int B, const double* x, const double* theta, int reupload, int ent,
                       int nbonds, const int* bonds, int nterms, const char* paulis, const double* coef,
                       double* expect, double* psi_out) {
  if (bad_args(n, L, B) || nterms < 0 || (nterms > 0 && (!paulis || !coef)) || bad_bonds(n, nbonds, bonds)) return -1;
  if (ent != ENT_CZ && ent != ENT_CNOT) return -1;
  const size_t N = (size_t)1 << n;
  const long ng = circuit_len(n, L, n_bonds_of(n, nbonds, bonds), reupload);
  int err = 0;
  const int outer = n < PAR_AMP_MIN_QUBITS;
#pragma omp parallel for schedule(dynamic, 1) if (outer) reduction(| : err)
  for (int b = 0; b < B; ++b) {
    gate* g = (gate*)malloc(sizeof(gate) * (size_t)ng);
    cplx* psi = (cplx*)malloc(sizeof(cplx) * N);
    cplx* hp = nterms ? (cplx*)malloc(sizeof(cplx) * N) : NULL;
    cplx* tmp = nterms ? (cplx*)malloc(sizeof(cplx) * N) : NULL;
    if (!g || !psi || (nterms && (!hp || !tmp))) {
      err |= 1;
    } else {
      build_circuit(g, n, L, x + (size_t)b * n, theta, nbonds, bonds, reupload, ent);
      zero_state(psi, n);
      for (long k = 0; k < ng; ++k) apply_gate(psi, n, &g[k], 0);
      if (expect) {
        if (!nterms) {
          expect[b] = expect_z0(psi, n);
        } else if (apply_observable(psi, hp, tmp, n, nterms, paulis, coef)) {
          err |= 1;
        } else {
          expect[b] = re_inner(psi, hp, n);
        }
      }
      if (psi_out) memcpy(psi_out + (size_t)b * N * 2, psi, sizeof(cplx) * N);
    }
    free(g);
    free(psi);
    free(hp);
    free(tmp);
  }
  return err ? -1 : 0;
}

/* Forward pass with CZ entanglers. */
int oracle_forward_gen(int n, int L, int B, const double* x, const double* theta, int reupload, int nbonds,
                       const int* bonds, int nterms, const char* paulis, const double* coef, double* expect,
                       double* psi_out) {
  return oracle_forward_ent(n, L, B, x, theta, reupload, ENT_CZ, nbonds, bonds, nterms, paulis, coef, expect,
                            psi_out);
}

/* Forward pass with the CZ chain and an observable. */
int oracle_forward_obs(int n, int L, int B, const double* x, const double* theta, int nterms, const char* paulis,
                       const double* coef, double* expect, double* psi_out) {
  return oracle_forward_gen(n, L, B, x, theta, 0, 0, NULL, nterms, paulis, coef, expect, psi_out);
}

/* Forward pass with the CZ chain and the Z0 observable. */
int oracle_forward(int n, int L, int B, const double* x, const double* theta, double* expect,
                   double* psi_out) {
  return oracle_forward_gen(n, L, B, x, theta, 0, 0, NULL, 0, NULL, NULL, expect, psi_out);
}

/*
 * Adjoint-method gradient for B samples with observable H (nterms > 0) or Z0
 * (nterms == 0).
 *   g      [B]        dL/dE_b, the loss seed per sample
 *   grad   [L][n][3]  out: sum_b g_b dE_b/dtheta (overwritten)
 *   expect [B]        out: <H> per sample (may be NULL)
 *   psi0   [B][2^n][2] out: the state after walking the whole circuit back
 *                     to the start, which must be |0...0> (may be NULL)
 *
 * Per sample: run the circuit forward to psi_M, set lambda = g_b H psi_M,
 * then walk the gates in reverse.  For a rotation U_j:
 *     psi    <- U_j^dagger psi                     (psi is now psi_{j-1})
 *     grad_j += 2 Re <lambda| dU_j/dtheta |psi>    (lambda is still lambda_j)
 *     lambda <- U_j^dagger lambda                  (lambda_{j-1})
 * and for CZ both states are multiplied by CZ.
 */
int oracle_adjoint_ent(int n, int L, int B, const double* x, const double* theta, int reupload, int ent,
                       int nbonds, const int* bonds, int nterms, const char* paulis, const double* coef,
                       const double* gseed, double* grad, double* expect, double* psi0_out) {
  if (bad_args(n, L, B) || nterms < 0 || (nterms > 0 && (!paulis || !coef)) || bad_bonds(n, nbonds, bonds)) return -1;
  if (ent != ENT_CZ && ent != ENT_CNOT) return -1;
  const size_t N = (size_t)1 << n;
  const long ng = circuit_len(n, L, n_bonds_of(n, nbonds, bonds), reupload);
  const long P = (long)L * n * 3;
  int err = 0;
  double* per = (double*)calloc((size_t)(B > 0 ? B : 1) * (size_t)(P > 0 ? P : 1), sizeof(double));
  if (!per) return -1;
  const int outer = n < PAR_AMP_MIN_QUBITS;
#pragma omp parallel for schedule(dynamic, 1) if (outer) reduction(| : err)
  for (int b = 0; b < B; ++b) {
    gate* g = (gate*)malloc(sizeof(gate) * (size_t)ng);
    cplx* psi = (cplx*)malloc(sizeof(cplx) * N);
    cplx* lam = (cplx*)malloc(sizeof(cplx) * N);
    cplx* tmp = nterms ? (cplx*)malloc(sizeof(cplx) * N) : NULL;
    if (!g || !psi || !lam || (nterms && !tmp)) {
      err |= 1;
    } else {
      double* gb = per + (size_t)b * P;
      build_circuit(g, n, L, x + (size_t)b * n, theta, nbonds, bonds, reupload, ent);
      zero_state(psi, n);
      for (long k = 0; k < ng; ++k) apply_gate(psi, n, &g[k], 0);
      /* lambda_M = dL/dE * H psi_M  (the derivative of <psi|H|psi> w.r.t. <psi|) */
      if (!nterms) {
        if (expect) expect[b] = expect_z0(psi, n);
        for (size_t i = 0; i < N; ++i) lam[i] = gseed[b] * ((i & 1) ? -psi[i] : psi[i]);
      } else if (apply_observable(psi, lam, tmp, n, nterms, paulis, coef)) {
        err |= 1;
      } else {
        if (expect) expect[b] = re_inner(psi, lam, n);
        for (size_t i = 0; i < N; ++i) lam[i] *= gseed[b];
      }
      for (long k = ng - 1; k >= 0 && !err; --k) {
        const gate* gk = &g[k];
        if (gk->kind == G_CZ) {
          apply_cz(psi, n, gk->q, gk->q2);
          apply_cz(lam, n, gk->q, gk->q2);
          continue;
        }
        if (gk->kind == G_CNOT) {
          apply_cnot(psi, n, gk->q, gk->q2);
          apply_cnot(lam, n, gk->q, gk->q2);
          continue;
        }
        mat2 ud = dagger(rotation(gk->pauli, gk->angle));
        apply_1q(psi, n, gk->q, ud);
        if (gk->param >= 0) {
          mat2 d = rotation_derivative(gk->pauli, gk->angle);
          gb[gk->param] += 2.0 * creal(local_braket(lam, psi, n, gk->q, d));
        }
        apply_1q(lam, n, gk->q, ud);
      }
      if (psi0_out) memcpy(psi0_out + (size_t)b * N * 2, psi, sizeof(cplx) * N);
    }
    free(g);
    free(psi);
    free(lam);
    free(tmp);
  }
  if (!err) {
    /* sum over samples in a fixed order */
    for (long p = 0; p < P; ++p) {
      double s = 0.0;
      for (int b = 0; b < B; ++b) s += per[(size_t)b * P + p];
      grad[p] = s;
    }
  }
  free(per);
  return err ? -1 : 0;
}

/* Adjoint gradient with CZ entanglers. */
int oracle_adjoint_gen(int n, int L, int B, const double* x, const double* theta, int reupload, int nbonds,
                       const int* bonds, int nterms, const char* paulis, const double* coef, const double* gseed,
                       double* grad, double* expect, double* psi0_out) {
  return oracle_adjoint_ent(n, L, B, x, theta, reupload, ENT_CZ, nbonds, bonds, nterms, paulis, coef, gseed, grad,
                            expect, psi0_out);
}

/* Adjoint gradient with the CZ chain and an observable. */
int oracle_adjoint_obs(int n, int L, int B, const double* x, const double* theta, int nterms, const char* paulis,
                       const double* coef, const double* gseed, double* grad, double* expect, double* psi0_out) {
  return oracle_adjoint_gen(n, L, B, x, theta, 0, 0, NULL, nterms, paulis, coef, gseed, grad, expect, psi0_out);
}

/* Adjoint gradient with the CZ chain and the Z0 observable. */
int oracle_adjoint(int n, int L, int B, const double* x, const double* theta, const double* gseed,
                   double* grad, double* expect, double* psi0_out) {
  return oracle_adjoint_gen(n, L, B, x, theta, 0, 0, NULL, 0, NULL, NULL, gseed, grad, expect, psi0_out);
}

/*
 * bf16 storage rounding, as defined by IEEE-754 round-to-nearest-even when
 * an fp32 value is narrowed to 8 significand bits (bfloat16 = the top 16 bits
 * of an fp32).  NaN inputs map to a quiet NaN with the sign kept.  This is the
 * conversion the memory-save mode applies to stored state vectors
 * ([Gist-EN] Technical Summary §2, "Memory-Saving Mode").
 */
static uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu)) return (uint16_t)((u >> 16) | 0x0040u);
  uint32_t lower = u & 0xffffu;
  uint32_t upper = u >> 16;
  if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) upper += 1u;
  return (uint16_t)upper;
}

void oracle_bf16_round(const float* in, uint16_t* out, size_t count) {
  for (size_t i = 0; i < count; ++i) out[i] = f32_to_bf16_rne(in[i]);
}

void oracle_bf16_widen(const uint16_t* in, float* out, size_t count) {
  for (size_t i = 0; i < count; ++i) {
    uint32_t u = (uint32_t)in[i] << 16;
    memcpy(&out[i], &u, sizeof u);
  }
}
