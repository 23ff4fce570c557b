/*
 * mw_oracle.c -- plain fp64 CPU oracle for the 2-D TM Maxwell FDTD forward,
 * exact discrete adjoint and model gradients (adjoint-state method).
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the checker the CUDA library is
 * compared against.  Only the test suite, the smoke check and the CPU
 * baseline leg of the benchmark may load it.  It shares no code, header,
 * table or constant with the CUDA library: every coefficient below is
 * written out here from the mathematics.
 *
 * Source of the method: the page "tide-GPR 0.0.9 ... tide/csrc/maxwell.cu"
 * (file header comment "EXACT DISCRETE Adjoint State Method for Maxwell TM
 * equations": forward leapfrog, adjoint equations, gradient formulas
 * dJ/dCa = sum_n Ey^n lambda^{n+1}, dJ/dCb = sum_n curlH^n lambda^{n+1}),
 * its forward H / E kernels (CPML memory update m = b m + a d, output d/k + m),
 * its source / receiver kernels, its per-shot gradient + combine strategy and
 * its epsilon/sigma chain-rule kernel.
 *
 * Readings where the page is silent (each is pinned by a test, see the
 * header of each function):
 *   - staggered Taylor stencil coefficients (the stencil header is not on
 *     the page);
 *   - every array cell of every field is updated and fields are zero outside
 *     the array, which makes D_x^T = -D_x^h exact;
 *   - the adjoint is the literal transpose of the forward step, CPML band
 *     included (the page's adjoint kernels apply the forward-form recursion
 *     at the other node; the sibling PR "DeepWave-KAUST/sweep #125" documents
 *     that defect class);
 *   - CPML profile: quadratic d, kappa = 1, linear alpha, R = 1e-3;
 *   - snapshot storage in bfloat16 or FP8 E4M3 rounds the fp32 value to
 *     nearest, ties to even, E4M3 saturating to +-448 (orc_quant_bf16,
 *     orc_fp8_encode; pinned to the format definitions and to torch's casts).
 *
 * Layout: row-major [shot][y][x], y = depth (z), x = columns, cell index
 * j = y*nx + x.  Hx lives at (y+1/2, x), Hz at (y, x+1/2), Ey at (y, x).
 * A state is 7 field arrays [7][S][ny][nx]:
 *   0 Ey, 1 Hx, 2 Hz, 3 m_ey_x (Hz nodes), 4 m_ey_z (Hx nodes),
 *   5 m_hz_x (E nodes, x), 6 m_hx_z (E nodes, z).
 * An adjoint state has the same 7 arrays holding the adjoints of the same
 * variables (lambda form: the adjoint of each forward variable itself).
 *
 * Parity pins (tests/test_oracle_*.py): dot tests of the record map and of
 * the state map (<= 1e-12), central finite differences of Ca / Cb / eps / sigma
 * gradients on a 16x16 grid (<= 1e-6), exact discrete energy invariant,
 * CFL growth threshold, reciprocity, stencil order of accuracy against the
 * Taylor conditions solved in exact rationals, plane-wave phase speed,
 * CPML absorption, checkpoint replay equal to full storage.
 */
#include <math.h>
#include <stdint.h>
#ifdef _OPENMP
#include <omp.h>
#endif
#include <stdlib.h>
#include <string.h>

#define NFIELD 7

/* vacuum permittivity, value printed on the maxwell.cu page (EP0 macro) */
static const double ORC_EPS0 = 8.8541878128e-12;
/* vacuum permeability, CODATA 2018 */
static const double ORC_MU0 = 1.25663706212e-6;

/* ------------------------------------------------------------------------ */
/* Stencil coefficients.  Staggered first-derivative weights c_k, k = 1..P,
 * solving sum_k c_k (2k-1)^(2m+1) = [m == 0] for m = 0..P-1 (Taylor
 * conditions on a half-integer staggered grid).  Pinned by a test that solves
 * the same conditions in exact rationals and by an order-of-accuracy test. */
int orc_coeffs(int order, double *c) {
  c[0] = c[1] = c[2] = c[3] = 0.0;
  switch (order) {
    case 2: c[0] = 1.0; return 1;
    case 4: c[0] = 9.0 / 8.0; c[1] = -1.0 / 24.0; return 2;
    case 6: c[0] = 75.0 / 64.0; c[1] = -25.0 / 384.0; c[2] = 3.0 / 640.0; return 3;
    case 8:
      c[0] = 1225.0 / 1024.0; c[1] = -245.0 / 3072.0;
      c[2] = 49.0 / 5120.0;   c[3] = -5.0 / 7168.0;
      return 4;
    default: return 0;
  }
}

/* ------------------------------------------------------------------------ */
/* Model coefficients from (eps_r, sigma, mu_r).  The forms are the ones whose
 * derivatives the page's chain-rule kernel uses (dCa/deps = (1-Ca)Cb/dt,
 * dCb/deps = -Cb^2/dt, dCa/dsigma = -(1+Ca)Cb/2, dCb/dsigma = -Cb^2/2):
 *   Ca = (1 - s dt/(2 eps)) / (1 + s dt/(2 eps)),  Cb = dt / (eps + s dt / 2),
 *   Cq = dt / (mu0 mu_r),  eps = eps0 eps_r.
 * Pinned: finite differences of these formulas against the chain rule, the
 * sigma = 0 limit, the Crank-Nicolson decay factor, and the plane-wave speed. */
void orc_model(int64_t n, const double *eps_r, const double *sigma,
               const double *mu_r, double dt, double *ca, double *cb,
               double *cq) {
  for (int64_t i = 0; i < n; ++i) {
    double eps = ORC_EPS0 * eps_r[i];
    double s = sigma ? sigma[i] : 0.0;
    double a = s * dt / (2.0 * eps);
    ca[i] = (1.0 - a) / (1.0 + a);
    cb[i] = dt / (eps + 0.5 * s * dt);
    if (cq) cq[i] = dt / (ORC_MU0 * (mu_r ? mu_r[i] : 1.0));
  }
}

/* dJ/d eps_r and dJ/d sigma from dJ/dCa, dJ/dCb (chain rule of orc_model;
 * the eps_r gradient carries the eps0 factor as on the page). */
void orc_eps_sigma_grad(int64_t n, const double *ca, const double *cb,
                        double dt, const double *gca, const double *gcb,
                        double *g_eps_r, double *g_sigma) {
  for (int64_t i = 0; i < n; ++i) {
    double dca_de = (1.0 - ca[i]) * cb[i] / dt;
    double dcb_de = -cb[i] * cb[i] / dt;
    double dca_ds = -0.5 * (1.0 + ca[i]) * cb[i];
    double dcb_ds = -0.5 * cb[i] * cb[i];
    if (g_eps_r) g_eps_r[i] = ORC_EPS0 * (gca[i] * dca_de + gcb[i] * dcb_de);
    if (g_sigma) g_sigma[i] = gca[i] * dca_ds + gcb[i] * dcb_ds;
  }
}

/* Largest stable dt of the staggered leapfrog in a medium whose fastest wave
 * speed is vmax: dt_max = 1 / (vmax * sum|c_k| * sqrt(1/dx^2 + 1/dy^2))
 * (von Neumann bound at the grid Nyquist wavenumber; the page only says a
 * stability warning exists).  Pinned by growth / boundedness runs and by a
 * power iteration on the spatial operator. */
double orc_cfl_dt(int order, double dy, double dx, double vmax) {
  double c[4];
  int P = orc_coeffs(order, c);
  double s = 0.0;
  for (int k = 0; k < P; ++k) s += fabs(c[k]);
  return 1.0 / (vmax * s * sqrt(1.0 / (dx * dx) + 1.0 / (dy * dy)));
}

/* Wave speed of light in vacuum implied by eps0, mu0. */
double orc_c0(void) { return 1.0 / sqrt(ORC_EPS0 * ORC_MU0); }

/* CPML profile along one axis of n nodes with an n_pml-cell band on both
 * sides.  Integer node i sits at i, half node i at i + 1/2 (grid units).
 * Distance into the band u: left band measured from the inner edge n_pml,
 * right band from n - 1 - n_pml.  With L = n_pml * h and s = min(u/n_pml, 1):
 *   d = d_max s^2,  d_max = -3 vmax ln(R) / (2 L),  kappa = 1,
 *   alpha = pi f0 (1 - s),  b = exp(-(d + alpha) dt),
 *   a = d (b - 1) / (d + alpha)   (a = 0 where d = 0).
 * Outside the band a = b = 0 and k = 1, so the CPML operator is the identity.
 * Parity unpinned for its reflection quality (no page prints numbers); its
 * absorption is checked by a property test. */
void orc_cpml(int n, int n_pml, double h, double dt, double vmax, double f0,
              double R, double *a, double *ah, double *b, double *bh,
              double *k, double *kh) {
  for (int half = 0; half < 2; ++half) {
    double *aa = half ? ah : a, *bb = half ? bh : b, *kk = half ? kh : k;
    for (int i = 0; i < n; ++i) {
      double pos = i + (half ? 0.5 : 0.0);
      double u = 0.0;
      if (n_pml > 0) {
        double left = (double)n_pml - pos;
        double right = pos - (double)(n - 1 - n_pml);
        if (left > 0.0) u = left;
        if (right > 0.0) u = right;
      }
      kk[i] = 1.0;
      if (u <= 0.0) {
        aa[i] = 0.0;
        bb[i] = 0.0;
        continue;
      }
      double L = n_pml * h;
      double s = u / (double)n_pml;
      if (s > 1.0) s = 1.0;
      double dmax = -3.0 * vmax * log(R) / (2.0 * L);
      double d = dmax * s * s;
      double alpha = M_PI * f0 * (1.0 - s);
      double bv = exp(-(d + alpha) * dt);
      bb[i] = bv;
      aa[i] = (d > 0.0) ? d * (bv - 1.0) / (d + alpha) : 0.0;
    }
  }
}

/* ------------------------------------------------------------------------ */
/* Simulation description shared by forward and adjoint. */
typedef struct {
  int ny, nx, order, n_shots, n_src, n_rec;
  double dy, dx;
  int model_batched; /* 0: ca/cb [ny][nx] shared by shots; 1: [S][ny][nx] */
  int cq_is_array;   /* 0: cq[0] scalar; 1: cq has the shape of ca */
  const double *ca, *cb, *cq;
  /* CPML profiles: y-axis (rows) then x-axis (columns); "h" = half node */
  const double *ay, *ayh, *by, *byh, *ky, *kyh;
  const double *ax, *axh, *bx, *bxh, *kx, *kxh;
  const int64_t *src_idx; /* [S][n_src], flat cell index, -1 inactive */
  const int64_t *rec_idx; /* [S][n_rec] */
} orc_sim;

/* Field value with zero extension outside the array. */
static inline double at(const double *F, int ny, int nx, int y, int x) {
  if (y < 0 || y >= ny || x < 0 || x >= nx) return 0.0;
  return F[(int64_t)y * nx + x];
}

/* D_x^h F at the half node (y, x+1/2):  r sum_k c_k (F[x+k] - F[x-k+1]). */
static inline double d_xh(const double *F, int ny, int nx, int y, int x,
                          const double *c, int P, double r) {
  double s = 0.0;
  for (int k = 1; k <= P; ++k)
    s += c[k - 1] * (at(F, ny, nx, y, x + k) - at(F, ny, nx, y, x - k + 1));
  return r * s;
}
/* D_z^h F at the half node (y+1/2, x). */
static inline double d_zh(const double *F, int ny, int nx, int y, int x,
                          const double *c, int P, double r) {
  double s = 0.0;
  for (int k = 1; k <= P; ++k)
    s += c[k - 1] * (at(F, ny, nx, y + k, x) - at(F, ny, nx, y - k + 1, x));
  return r * s;
}
/* D_x F at the integer node (y, x) from half-node values:
 *   r sum_k c_k (F[x+k-1] - F[x-k]). */
static inline double d_x(const double *F, int ny, int nx, int y, int x,
                         const double *c, int P, double r) {
  double s = 0.0;
  for (int k = 1; k <= P; ++k)
    s += c[k - 1] * (at(F, ny, nx, y, x + k - 1) - at(F, ny, nx, y, x - k));
  return r * s;
}
/* D_z F at the integer node (y, x). */
static inline double d_z(const double *F, int ny, int nx, int y, int x,
                         const double *c, int P, double r) {
  double s = 0.0;
  for (int k = 1; k <= P; ++k)
    s += c[k - 1] * (at(F, ny, nx, y + k - 1, x) - at(F, ny, nx, y - k, x));
  return r * s;
}

static inline const double *model_ptr(const orc_sim *m, const double *p,
                                      int s) {
  return m->model_batched ? p + (int64_t)s * m->ny * m->nx : p;
}
static inline double cq_at(const orc_sim *m, int s, int64_t j) {
  if (!m->cq_is_array) return m->cq[0];
  return model_ptr(m, m->cq, s)[j];
}

/* One forward time step t for all shots, in the page's order:
 * H update, E update (optionally saving Ey^t and curl^t), source injection,
 * receiver sampling.  `state` is [7][S][ny][nx]. */
/* Born source of the linearised step (NULL for the plain forward): the
 * perturbation dCa, dCb (model-shaped) and the background's E^t, curl^t. */
typedef struct {
  const double *dca, *dcb, *e0, *c0;
} orc_born_src;

static void forward_step(const orc_sim *m, int t, const double *f,
                         double *state, double *rec, double *snap_ey,
                         double *snap_curl, const orc_born_src *born) {
  const int ny = m->ny, nx = m->nx, S = m->n_shots;
  const int64_t N = (int64_t)ny * nx;
  double c[4];
  const int P = orc_coeffs(m->order, c);
  const double rdy = 1.0 / m->dy, rdx = 1.0 / m->dx;

  /* 1. H update: Hx -= Cq psi_z(D_z^h Ey), Hz += Cq psi_x(D_x^h Ey) */
#pragma omp parallel for collapse(2) schedule(static)
  for (int s = 0; s < S; ++s) {
    for (int y = 0; y < ny; ++y) {
      const double *ey = state + (0 * (int64_t)S + s) * N;
      double *hx = state + (1 * (int64_t)S + s) * N;
      double *hz = state + (2 * (int64_t)S + s) * N;
      double *mex = state + (3 * (int64_t)S + s) * N;
      double *mez = state + (4 * (int64_t)S + s) * N;
      for (int x = 0; x < nx; ++x) {
        int64_t j = (int64_t)y * nx + x;
        double cq = cq_at(m, s, j);
        double dz = d_zh(ey, ny, nx, y, x, c, P, rdy);
        mez[j] = m->byh[y] * mez[j] + m->ayh[y] * dz;
        hx[j] -= cq * (dz / m->kyh[y] + mez[j]);
        double dx = d_xh(ey, ny, nx, y, x, c, P, rdx);
        mex[j] = m->bxh[x] * mex[j] + m->axh[x] * dx;
        hz[j] += cq * (dx / m->kxh[x] + mex[j]);
      }
    }
  }
  /* 2. E update: curl = psi_x(D_x Hz) - psi_z(D_z Hx); Ey = Ca Ey + Cb curl */
#pragma omp parallel for collapse(2) schedule(static)
  for (int s = 0; s < S; ++s) {
    for (int y = 0; y < ny; ++y) {
      double *ey = state + (0 * (int64_t)S + s) * N;
      const double *hx = state + (1 * (int64_t)S + s) * N;
      const double *hz = state + (2 * (int64_t)S + s) * N;
      double *mhx = state + (5 * (int64_t)S + s) * N;
      double *mhz = state + (6 * (int64_t)S + s) * N;
      const double *ca = model_ptr(m, m->ca, s), *cb = model_ptr(m, m->cb, s);
      for (int x = 0; x < nx; ++x) {
        int64_t j = (int64_t)y * nx + x;
        double cx = d_x(hz, ny, nx, y, x, c, P, rdx);
        mhx[j] = m->bx[x] * mhx[j] + m->ax[x] * cx;
        double cz = d_z(hx, ny, nx, y, x, c, P, rdy);
        mhz[j] = m->by[y] * mhz[j] + m->ay[y] * cz;
        double curl = (cx / m->kx[x] + mhx[j]) - (cz / m->ky[y] + mhz[j]);
        if (snap_ey) snap_ey[((int64_t)t * S + s) * N + j] = ey[j];
        if (snap_curl) snap_curl[((int64_t)t * S + s) * N + j] = curl;
        ey[j] = ca[j] * ey[j] + cb[j] * curl;
        if (born) {
          /* linearised step: d(Ca E + Cb curl) = Ca dE + Cb dcurl + dCa E0 + dCb curl0 */
          const int64_t k = ((int64_t)t * S + s) * N + j;
          ey[j] += model_ptr(m, born->dca, s)[j] * born->e0[k] +
                   model_ptr(m, born->dcb, s)[j] * born->c0[k];
        }
      }
    }
  }
  /* 3. sources, in order (duplicates add up); 4. receivers */
  for (int s = 0; s < S; ++s) {
    double *ey = state + (int64_t)s * N;
    for (int k = 0; k < m->n_src; ++k) {
      int64_t i = m->src_idx[(int64_t)s * m->n_src + k];
      if (i >= 0 && f) ey[i] += f[((int64_t)t * S + s) * m->n_src + k];
    }
    for (int k = 0; k < m->n_rec; ++k) {
      int64_t i = m->rec_idx[(int64_t)s * m->n_rec + k];
      if (rec) rec[((int64_t)t * S + s) * m->n_rec + k] = (i >= 0) ? ey[i] : 0.0;
    }
  }
}

/* Forward over nt steps.  state [7][S][ny][nx] in/out (zero it for a run
 * from rest); rec [nt][S][n_rec] (may be NULL); snap_* [nt][S][ny][nx]
 * (may be NULL). */
int orc_forward(const orc_sim *m, int nt, const double *f, double *state,
                double *rec, double *snap_ey, double *snap_curl) {
  double c[4];
  if (!orc_coeffs(m->order, c)) return -1;
  for (int t = 0; t < nt; ++t)
    forward_step(m, t, f, state, rec, snap_ey, snap_curl, NULL);
  return 0;
}

/* Born (linearised) forward: the derivative of the records with respect to
 * (Ca, Cb) in the direction (dCa, dCb).  The perturbation state starts at
 * zero and takes the forward step without sources, plus the term
 * dCa E0^t + dCb curl0^t from the background's snapshots (the E^t and
 * curl^t of the step, [nt][S][ny][nx]); records are sampled as in the
 * forward.  Its transpose maps a record residual to the gradients
 * sum_t E0^t lambda^{t+1}, sum_t curl0^t lambda^{t+1} of the adjoint. */
int orc_born(const orc_sim *m, int nt, const double *snap_ey0, const double *snap_curl0,
             const double *dca, const double *dcb, double *state, double *rec) {
  double c[4];
  if (!orc_coeffs(m->order, c)) return -1;
  const orc_born_src b = {dca, dcb, snap_ey0, snap_curl0};
  for (int t = 0; t < nt; ++t) forward_step(m, t, NULL, state, rec, NULL, NULL, &b);
  return 0;
}

/* One adjoint step t: the literal transpose of forward_step, applied in
 * reverse order.  adj [7][S][ny][nx] holds the adjoints of the 7 state
 * variables after step t on entry and before step t on exit.  `work` holds
 * 2 arrays of [S][ny][nx]. */
static void adjoint_step(const orc_sim *m, int t, const double *res,
                         const double *snap_ey, const double *snap_curl,
                         double *adj, double *gca, double *gcb, double *grad_f,
                         double *work) {
  const int ny = m->ny, nx = m->nx, S = m->n_shots;
  const int64_t N = (int64_t)ny * nx;
  double c[4];
  const int P = orc_coeffs(m->order, c);
  const double rdy = 1.0 / m->dy, rdx = 1.0 / m->dx;
  double *px_all = work, *pz_all = work + (int64_t)S * N;

  /* transpose of receivers then sources */
  for (int s = 0; s < S; ++s) {
    double *le = adj + (int64_t)s * N;
    for (int k = 0; k < m->n_rec; ++k) {
      int64_t i = m->rec_idx[(int64_t)s * m->n_rec + k];
      if (i >= 0) le[i] += res[((int64_t)t * S + s) * m->n_rec + k];
    }
    if (grad_f) {
      for (int k = 0; k < m->n_src; ++k) {
        int64_t i = m->src_idx[(int64_t)s * m->n_src + k];
        grad_f[((int64_t)t * S + s) * m->n_src + k] = (i >= 0) ? le[i] : 0.0;
      }
    }
  }

  /* transpose of the E update (Ey' = Ca Ey + Cb curl): gradients, then the
   * curl's adjoint g = Cb lambda_E through the E-node CPML recursions. */
#pragma omp parallel for collapse(2) schedule(static)
  for (int s = 0; s < S; ++s) {
    for (int y = 0; y < ny; ++y) {
      double *le = adj + (0 * (int64_t)S + s) * N;
      double *lmhx = adj + (5 * (int64_t)S + s) * N;
      double *lmhz = adj + (6 * (int64_t)S + s) * N;
      double *px = px_all + (int64_t)s * N, *pz = pz_all + (int64_t)s * N;
      const double *ca = model_ptr(m, m->ca, s), *cb = model_ptr(m, m->cb, s);
      (void)ca;
      for (int x = 0; x < nx; ++x) {
        int64_t j = (int64_t)y * nx + x;
        double lam = le[j]; /* lambda^{t+1} */
        if (gca && snap_ey) gca[(int64_t)s * N + j] += snap_ey[((int64_t)t * S + s) * N + j] * lam;
        if (gcb && snap_curl) gcb[(int64_t)s * N + j] += snap_curl[((int64_t)t * S + s) * N + j] * lam;
        double g = cb[j] * lam; /* adjoint of curl */
        /* curl = (cx/kx + m_hz_x') - (cz/ky + m_hx_z') */
        double M = lmhx[j] + g;
        px[j] = g / m->kx[x] + m->ax[x] * M; /* adjoint of cx */
        lmhx[j] = m->bx[x] * M;
        double Mz = lmhz[j] - g;
        pz[j] = -g / m->ky[y] + m->ay[y] * Mz; /* adjoint of cz */
        lmhz[j] = m->by[y] * Mz;
      }
    }
  }
  /* cx = D_x Hz, cz = D_z Hx:  lambda_H += D^T p = -D^h p */
#pragma omp parallel for collapse(2) schedule(static)
  for (int s = 0; s < S; ++s) {
    for (int y = 0; y < ny; ++y) {
      double *lhx = adj + (1 * (int64_t)S + s) * N;
      double *lhz = adj + (2 * (int64_t)S + s) * N;
      const double *px = px_all + (int64_t)s * N, *pz = pz_all + (int64_t)s * N;
      for (int x = 0; x < nx; ++x) {
        int64_t j = (int64_t)y * nx + x;
        lhz[j] -= d_xh(px, ny, nx, y, x, c, P, rdx);
        lhx[j] -= d_zh(pz, ny, nx, y, x, c, P, rdy);
      }
    }
  }
  /* Ca term, then transpose of the H update through the H-node CPML
   * recursions:  Hz' = Hz + Cq psi(D_x^h Ey),  Hx' = Hx - Cq psi(D_z^h Ey). */
#pragma omp parallel for collapse(2) schedule(static)
  for (int s = 0; s < S; ++s) {
    for (int y = 0; y < ny; ++y) {
      double *le = adj + (0 * (int64_t)S + s) * N;
      const double *lhx = adj + (1 * (int64_t)S + s) * N;
      const double *lhz = adj + (2 * (int64_t)S + s) * N;
      double *lmex = adj + (3 * (int64_t)S + s) * N;
      double *lmez = adj + (4 * (int64_t)S + s) * N;
      double *qx = px_all + (int64_t)s * N, *qz = pz_all + (int64_t)s * N;
      const double *ca = model_ptr(m, m->ca, s);
      for (int x = 0; x < nx; ++x) {
        int64_t j = (int64_t)y * nx + x;
        double cq = cq_at(m, s, j);
        le[j] = ca[j] * le[j];
        double v = cq * lhz[j]; /* adjoint of psi_x output */
        double M = lmex[j] + v;
        qx[j] = v / m->kxh[x] + m->axh[x] * M; /* adjoint of D_x^h Ey */
        lmex[j] = m->bxh[x] * M;
        double v2 = -cq * lhx[j];
        double M2 = lmez[j] + v2;
        qz[j] = v2 / m->kyh[y] + m->ayh[y] * M2; /* adjoint of D_z^h Ey */
        lmez[j] = m->byh[y] * M2;
      }
    }
  }
  /* lambda_E += (D^h)^T q = -D q */
#pragma omp parallel for collapse(2) schedule(static)
  for (int s = 0; s < S; ++s) {
    for (int y = 0; y < ny; ++y) {
      double *le = adj + (0 * (int64_t)S + s) * N;
      const double *qx = px_all + (int64_t)s * N, *qz = pz_all + (int64_t)s * N;
      for (int x = 0; x < nx; ++x) {
        int64_t j = (int64_t)y * nx + x;
        le[j] -= d_x(qx, ny, nx, y, x, c, P, rdx) + d_z(qz, ny, nx, y, x, c, P, rdy);
      }
    }
  }
}

/* Adjoint over nt steps, t = nt-1 ... 0, with stored snapshots.
 * res [nt][S][n_rec]; snap_* [nt][S][ny][nx] (NULL disables that gradient);
 * adj [7][S][ny][nx] in/out (zero for a misfit gradient); gca, gcb
 * [S][ny][nx] accumulated (+=); grad_f [nt][S][n_src] or NULL. */
int orc_adjoint(const orc_sim *m, int nt, const double *res,
                const double *snap_ey, const double *snap_curl, double *adj,
                double *gca, double *gcb, double *grad_f) {
  double c[4];
  if (!orc_coeffs(m->order, c)) return -1;
  const int64_t SN = (int64_t)m->n_shots * m->ny * m->nx;
  double *work = (double *)calloc((size_t)(2 * SN), sizeof(double));
  if (!work) return -2;
  for (int t = nt - 1; t >= 0; --t)
    adjoint_step(m, t, res, snap_ey, snap_curl, adj, gca, gcb, grad_f, work);
  free(work);
  return 0;
}

/* Checkpointed forward + adjoint: the forward saves the whole state every C
 * steps; the adjoint replays each segment [kC, min(kC+C, nt)) from its
 * checkpoint into a C-step snapshot buffer and sweeps it backwards.  In fp64
 * this gives bit-for-bit the result of orc_forward + orc_adjoint with full
 * storage (same operations in the same order).  state0 [7][S][ny][nx] is the
 * initial state (NULL = zero); rec may be NULL. */
int orc_fwd_adj_ckpt(const orc_sim *m, int nt, int C, const double *f,
                     const double *state0, double *rec, const double *res_in,
                     double *gca, double *gcb, double *grad_f) {
  double c[4];
  if (!orc_coeffs(m->order, c) || C <= 0) return -1;
  const int64_t SN = (int64_t)m->n_shots * m->ny * m->nx;
  const int64_t SZ = NFIELD * SN;
  const int nseg = (nt + C - 1) / C;
  double *ck = (double *)malloc((size_t)(nseg > 0 ? nseg : 1) * SZ * sizeof(double));
  double *st = (double *)calloc((size_t)SZ, sizeof(double));
  double *sey = (double *)malloc((size_t)C * SN * sizeof(double));
  double *scu = (double *)malloc((size_t)C * SN * sizeof(double));
  double *adj = (double *)calloc((size_t)SZ, sizeof(double));
  double *work = (double *)calloc((size_t)(2 * SN), sizeof(double));
  if (!ck || !st || !sey || !scu || !adj || !work) {
    free(ck); free(st); free(sey); free(scu); free(adj); free(work);
    return -2;
  }
  if (state0) memcpy(st, state0, (size_t)SZ * sizeof(double));
  for (int t = 0; t < nt; ++t) {
    if (t % C == 0) memcpy(ck + (int64_t)(t / C) * SZ, st, (size_t)SZ * sizeof(double));
    forward_step(m, t, f, st, rec, NULL, NULL, NULL);
  }
  if (res_in) {
    for (int k = nseg - 1; k >= 0; --k) {
      int t0 = k * C, t1 = t0 + C < nt ? t0 + C : nt;
      memcpy(st, ck + (int64_t)k * SZ, (size_t)SZ * sizeof(double));
      /* replay: snapshots of step t go to slot t - t0 */
      for (int t = t0; t < t1; ++t)
        forward_step(m, t - t0, f + (int64_t)t0 * m->n_shots * m->n_src, st,
                     NULL, sey, scu, NULL);
      for (int t = t1 - 1; t >= t0; --t)
        adjoint_step(m, t - t0, res_in + (int64_t)t0 * m->n_shots * m->n_rec,
                     sey, scu, adj, gca, gcb,
                     grad_f ? grad_f + (int64_t)t0 * m->n_shots * m->n_src : NULL,
                     work);
    }
  }
  free(ck); free(st); free(sey); free(scu); free(adj); free(work);
  return 0;
}

/* Shot sum of per-shot gradients, fp64, shots in order 0..S-1 (the page's
 * combine_grad kernel, here over every cell). */
void orc_combine(int S, int64_t n, const double *g_shot, double *g) {
  for (int64_t i = 0; i < n; ++i) {
    double acc = 0.0;
    for (int s = 0; s < S; ++s) acc += g_shot[(int64_t)s * n + i];
    g[i] = acc;
  }
}

/* Residual and misfit J = 1/2 sum (d - d_obs)^2. */
double orc_residual(int64_t n, const double *d, const double *d_obs,
                    double *res) {
  double J = 0.0;
  for (int64_t i = 0; i < n; ++i) {
    double r = d[i] - d_obs[i];
    if (res) res[i] = r;
    J += 0.5 * r * r;
  }
  return J;
}

/* ---- snapshot storage formats ----------------------------------------------
 * The page stores the snapshots E^n, curl^n rounded to a narrower format
 * (forward_kernel_e_with_storage_bf16 / _fp8 and the matching backward
 * kernels' loads; the helpers "FP8 E4M3 (1 sign, 4 exponent, 3 mantissa)"
 * with saturation to the largest finite value).  The GPU computes in fp32,
 * so the stored value is the fp32 value rounded to the format; the oracle
 * rounds its fp64 value to fp32 first, then to the format.  Both encoders
 * below are written from the format definitions:
 *   bfloat16: the top 16 bits of an fp32, round to nearest, ties to even;
 *   E4M3: sign, 4-bit exponent (bias 7), 3-bit mantissa; subnormals
 *     m * 2^-9 (exponent field 0); normals (1 + m/8) 2^(e-7); the code
 *     S.1111.111 is NaN, so the largest finite value is 448 (S.1111.110);
 *     round to nearest, ties to even, saturating to +-448.
 */
static double fp32_round(double x) { return (double)(float)x; }

/* bfloat16 rounding of n values (fp64 in, fp64 out holding bf16 values). */
void orc_quant_bf16(int64_t n, const double *in, double *out) {
  for (int64_t i = 0; i < n; ++i) {
    float f = (float)in[i];
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu)) {
      u |= 0x00400000u;  /* NaN stays NaN */
    } else {
      const uint32_t lsb = (u >> 16) & 1u;
      u += 0x7fffu + lsb;
    }
    u &= 0xffff0000u;
    memcpy(&f, &u, 4);
    out[i] = (double)f;
  }
}

/* E4M3 code of one finite value a >= 0 (already an fp32 value). */
static unsigned fp8_code_abs(double a) {
  if (a >= 448.0) return 0x7eu;
  if (a == 0.0) return 0u;
  int e2;
  frexp(a, &e2);     /* a = m 2^e2, m in [0.5, 1): floor(log2 a) = e2 - 1 */
  int E = e2 - 1;
  if (E < -6) E = -6; /* subnormal range: quantum 2^-9 like the first binade */
  const double quantum = ldexp(1.0, E - 3);
  const double q = rint(a / quantum); /* exact quotient; ties to even */
  /* codes are contiguous across binades: ((E + 7) << 3) + (q - 8), and for
   * the subnormal binade (E = -6) code = q (0..8) */
  long code = (long)((E + 7) * 8) + (long)q - 8;
  if (E == -6) code = (long)q;
  if (code > 0x7e) code = 0x7e;
  return (unsigned)code;
}

/* E4M3 codes of n values (rounded to fp32 first). */
void orc_fp8_encode(int64_t n, const double *in, uint8_t *codes) {
  for (int64_t i = 0; i < n; ++i) {
    const double x = fp32_round(in[i]);
    if (x != x) {
      codes[i] = 0x7f;
      continue;
    }
    const unsigned sign = (x < 0.0 || (x == 0.0 && signbit(x))) ? 0x80u : 0u;
    codes[i] = (uint8_t)(sign | fp8_code_abs(fabs(x)));
  }
}

/* Values of n E4M3 codes. */
void orc_fp8_decode(int64_t n, const uint8_t *codes, double *out) {
  for (int64_t i = 0; i < n; ++i) {
    const unsigned c = codes[i];
    const unsigned e = (c >> 3) & 0xfu, m = c & 7u;
    double v;
    if (e == 15 && m == 7) {
      v = NAN;
    } else if (e == 0) {
      v = ldexp((double)m, -9);
    } else {
      v = ldexp(1.0 + m / 8.0, (int)e - 7);
    }
    out[i] = (c & 0x80u) ? -v : v;
  }
}

int orc_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
