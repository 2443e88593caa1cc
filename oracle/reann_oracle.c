/*
 * reann_oracle.c -- plain, slow, fp64 CPU oracle of the REANN energy+force
 * evaluation and of velocity-Verlet MD with it.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or
 * calls this file; only the tests, the smoke check and the benchmark's CPU
 * baseline do.  It shares no code, header or table with the CUDA library.
 *
 * What it computes follows "Efficient Parallelization of Message Passing
 * Neural Network Potentials for Large-Scale Molecular Dynamics" (Xia and
 * Jiang), section "REANN Architecture" (Eqs. 1-2) and section
 * "Parallelization Algorithm" (Eqs. 3-5), read as follows where the page
 * leaves details to its absent Supporting Information:
 *
 *   pairs      d_ij = x_j - x_i reduced to the minimum image per axis,
 *              r2 = (dx*dx + dy*dy) + dz*dz (no fused multiply-add), listed
 *              iff r2 < (r_c + skin)^2; the box must be at least twice the
 *              list radius.  One neighbour list serves every layer
 *              (section "Parallelization Algorithm", Fig. 2).
 *   orbital    for an active pair (r_ij < r_c) and primitive n = 0..N_phi-1:
 *              phi_n(r) = exp(-alpha (r - mu_n)^2) * f_c(r),
 *              mu_n = r_c n / (N_phi - 1), f_c(r) = (cos(pi r / r_c) + 1) / 2;
 *              angular factor Y_tau(d) = dx^lx dy^ly dz^lz for every
 *              tau = (lx, ly, lz) with l = lx + ly + lz <= L.
 *   density    (Eq. 1) A^t_{i,n,tau} = sum_j c^t_{j,(n,l)} phi_n(r_ij) Y_tau(d_ij),
 *              rho^t_{i,(n,l)} = sum_{|tau| = l} l!/(lx! ly! lz!) (A^t_{i,n,tau})^2.
 *              Feature (n, l) sits at index l*N_phi + n; D = N_phi (L+1).
 *   pair form  (density_form = 1; the dimension N_phi (N_phi+1)(L+1)/2 that
 *              section "REANN Architecture" states for the density vector)
 *              rho^t_{i,(n,m,l)} = sum_{|tau| = l} l!/tau! A_{i,n,tau} A_{i,m,tau}
 *              for n <= m, at index l*P + pair(n, m), P = N_phi (N_phi+1)/2,
 *              pair(n, m) = n N_phi - n (n-1)/2 + (m - n); the diagonal n = m
 *              is the square form.  Messages c keep one value per (n, l).
 *   messages   c^0_j is the element row C0[Z_j]; for 1 <= t <= T-1,
 *              c^t_i = M^{t-1}_{Z_i}(rho^{t-1}_i)  (Eq. 2).
 *   energy     E_i = N_{Z_i}(rho^{T-1}_i), E = sum_i E_i (Eq. 3 input).
 *   networks   y = W3 tanh(W2 tanh(W1 ((x - shift) / scale) + b1) + b2) + b3,
 *              one network per layer and per element of the centre atom.
 *   forces     F = -dE/dx by a reverse sweep: the energy network's gradient
 *              (Eq. 3), then per layer t = T-1..0 the density derivative with
 *              respect to the orbitals (direct term of Eq. 4) and to the
 *              neighbours' coefficients (message term of Eq. 4), chained into
 *              layer t-1 through the coefficient network (Eq. 5); dc^0/dx = 0.
 *
 * Everything is fp64.  Loops are written out in the order of the equations;
 * the only parallelism is OpenMP over centre atoms, with per-thread
 * accumulators where a loop scatters.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_MAX_TUPLES 10
#define ORACLE_MAX_L 2

typedef struct {
    int32_t n_elements;
    int32_t T;
    int32_t n_radial;
    int32_t l_max;
    int32_t hidden1;
    int32_t hidden2;
    double r_cut;
    double skin;
    double alpha;
    int32_t density_form; /* 0: squares per (n, l) (Eq. 1); 1: pair products per (n <= m, l) */
} oracle_cfg;

enum { ORACLE_OK = 0, ORACLE_ERR_ARG = 1, ORACLE_ERR_BOX = 2, ORACLE_ERR_CAPACITY = 3, ORACLE_ERR_MEM = 4 };

/* Cartesian angular tuples (lx, ly, lz), grouped by l = 0, 1, 2. */
static const int TUPLE[ORACLE_MAX_TUPLES][3] = {
    {0, 0, 0},
    {1, 0, 0}, {0, 1, 0}, {0, 0, 1},
    {2, 0, 0}, {0, 2, 0}, {0, 0, 2}, {1, 1, 0}, {1, 0, 1}, {0, 1, 1},
};

static int n_tuples(int L) { return (L + 1) * (L + 2) * (L + 3) / 6; }

/* number of density features per atom (network input width) */
static int n_feat(const oracle_cfg *c) {
    int NP = c->n_radial;
    return c->density_form == 1 ? NP * (NP + 1) / 2 * (c->l_max + 1) : NP * (c->l_max + 1);
}

/* index of the pair (n, m), n <= m, among the N_phi (N_phi+1)/2 pairs */
static int pair_index(int NP, int n, int m) { return n * NP - n * (n - 1) / 2 + (m - n); }
static int tuple_l(int tau) { return TUPLE[tau][0] + TUPLE[tau][1] + TUPLE[tau][2]; }

static double factorial(int k) {
    double f = 1.0;
    for (int i = 2; i <= k; ++i) f *= i;
    return f;
}

/* multinomial weight l! / (lx! ly! lz!) */
static double tuple_weight(int tau) {
    const int *t = TUPLE[tau];
    return factorial(t[0] + t[1] + t[2]) / (factorial(t[0]) * factorial(t[1]) * factorial(t[2]));
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------------ */
/* Pair search                                                              */

/* Minimum-image displacement x_j - x_i, per axis d -= L * rint(d / L). */
static void min_image(const double *xi, const double *xj, const double *box, double d[3]) {
    for (int a = 0; a < 3; ++a) {
        double v = xj[a] - xi[a];
        v = v - box[a] * rint(v / box[a]);
        d[a] = v;
    }
}

static double dist2(const double d[3]) {
    double s = d[0] * d[0] + d[1] * d[1];
    return s + d[2] * d[2];
}

static int check_box(const double *box, double r_list) {
    for (int a = 0; a < 3; ++a)
        if (!(box[a] > 0.0) || box[a] < 2.0 * r_list) return ORACLE_ERR_BOX;
    return ORACLE_OK;
}

/*
 * All ordered pairs (i, j), i != j, with r2 < (r_cut + skin)^2, by testing
 * every pair.  Rows come out sorted by i, then j.  `centres` (may be NULL)
 * restricts the rows to the listed centre atoms, in that order.
 * counts[r] receives the row length of row r; pairs are written to pj as
 * neighbour indices (row-major).  Returns ORACLE_ERR_CAPACITY and the total
 * in *nnz when cap is too small.
 */
int oracle_pairs_brute(int64_t n, const double *x, const double *box, double r_cut, double skin,
                       int64_t n_centres, const int64_t *centres,
                       int64_t cap, int64_t *counts, int32_t *pj, int64_t *nnz) {
    double rl = r_cut + skin;
    double thr = rl * rl;
    if (n < 0 || !x || !box || !counts || !nnz) return ORACLE_ERR_ARG;
    int rc = check_box(box, rl);
    if (rc) return rc;
    int64_t rows = centres ? n_centres : n;

    #pragma omp parallel for schedule(dynamic, 64)
    for (int64_t r = 0; r < rows; ++r) {
        int64_t i = centres ? centres[r] : r;
        int64_t c = 0;
        for (int64_t j = 0; j < n; ++j) {
            if (j == i) continue;
            double d[3];
            min_image(&x[3 * i], &x[3 * j], box, d);
            if (dist2(d) < thr) ++c;
        }
        counts[r] = c;
    }
    int64_t total = 0;
    for (int64_t r = 0; r < rows; ++r) total += counts[r];
    *nnz = total;
    if (total > cap || !pj) return pj ? ORACLE_ERR_CAPACITY : ORACLE_OK;

    int64_t *start = (int64_t *)malloc(sizeof(int64_t) * (rows + 1));
    if (!start) return ORACLE_ERR_MEM;
    start[0] = 0;
    for (int64_t r = 0; r < rows; ++r) start[r + 1] = start[r] + counts[r];

    #pragma omp parallel for schedule(dynamic, 64)
    for (int64_t r = 0; r < rows; ++r) {
        int64_t i = centres ? centres[r] : r;
        int64_t o = start[r];
        for (int64_t j = 0; j < n; ++j) {
            if (j == i) continue;
            double d[3];
            min_image(&x[3 * i], &x[3 * j], box, d);
            if (dist2(d) < thr) pj[o++] = (int32_t)j;
        }
    }
    free(start);
    return ORACLE_OK;
}

/*
 * A second, independent pair search (cell list) used only to pin the brute
 * force one.  Bins are at least r_list wide; a bin's neighbourhood is the
 * set of distinct bins within one step along each axis (all bins along an
 * axis with fewer than three).  Each row is sorted by j with insertion sort.
 * Same output contract as oracle_pairs_brute over all atoms.
 */
int oracle_pairs_cells(int64_t n, const double *x, const double *box, double r_cut, double skin,
                       int64_t cap, int64_t *counts, int32_t *pj, int64_t *nnz) {
    double rl = r_cut + skin;
    double thr = rl * rl;
    int rc = check_box(box, rl);
    if (rc) return rc;
    int m[3];
    for (int a = 0; a < 3; ++a) {
        m[a] = (int)floor(box[a] / rl);
        if (m[a] < 1) m[a] = 1;
    }
    int64_t nb = (int64_t)m[0] * m[1] * m[2];
    int64_t *bin = (int64_t *)malloc(sizeof(int64_t) * (n > 0 ? n : 1));
    int64_t *head = (int64_t *)malloc(sizeof(int64_t) * (nb + 1));
    int64_t *list = (int64_t *)malloc(sizeof(int64_t) * (n > 0 ? n : 1));
    if (!bin || !head || !list) return ORACLE_ERR_MEM;
    for (int64_t b = 0; b <= nb; ++b) head[b] = 0;
    for (int64_t i = 0; i < n; ++i) {
        int c[3];
        for (int a = 0; a < 3; ++a) {
            double u = x[3 * i + a] - box[a] * floor(x[3 * i + a] / box[a]);
            int k = (int)floor(u / box[a] * m[a]);
            if (k >= m[a]) k = m[a] - 1;
            if (k < 0) k = 0;
            c[a] = k;
        }
        bin[i] = ((int64_t)c[0] * m[1] + c[1]) * m[2] + c[2];
        head[bin[i] + 1]++;
    }
    for (int64_t b = 0; b < nb; ++b) head[b + 1] += head[b];
    {
        int64_t *fill = (int64_t *)calloc((size_t)(nb > 0 ? nb : 1), sizeof(int64_t));
        for (int64_t i = 0; i < n; ++i) list[head[bin[i]] + fill[bin[i]]++] = i;
        free(fill);
    }
    int pass_ok = 1;
    int64_t total = 0;
    for (int pass = 0; pass < 2 && pass_ok; ++pass) {
        int64_t *start = NULL;
        if (pass == 1) {
            start = (int64_t *)malloc(sizeof(int64_t) * (n + 1));
            start[0] = 0;
            for (int64_t i = 0; i < n; ++i) start[i + 1] = start[i] + counts[i];
        }
        #pragma omp parallel for schedule(dynamic, 64)
        for (int64_t i = 0; i < n; ++i) {
            int64_t b = bin[i];
            int c[3] = {(int)(b / ((int64_t)m[1] * m[2])), (int)((b / m[2]) % m[1]), (int)(b % m[2])};
            int off[3][3], no[3];
            for (int a = 0; a < 3; ++a) {
                if (m[a] >= 3) {
                    no[a] = 3;
                    for (int s = 0; s < 3; ++s) off[a][s] = (c[a] + s - 1 + m[a]) % m[a];
                } else {
                    no[a] = m[a];
                    for (int s = 0; s < m[a]; ++s) off[a][s] = s;
                }
            }
            int64_t cnt = 0;
            int64_t o = pass ? start[i] : 0;
            for (int s0 = 0; s0 < no[0]; ++s0)
                for (int s1 = 0; s1 < no[1]; ++s1)
                    for (int s2 = 0; s2 < no[2]; ++s2) {
                        int64_t nbb = ((int64_t)off[0][s0] * m[1] + off[1][s1]) * m[2] + off[2][s2];
                        for (int64_t q = head[nbb]; q < head[nbb + 1]; ++q) {
                            int64_t j = list[q];
                            if (j == i) continue;
                            double d[3];
                            min_image(&x[3 * i], &x[3 * j], box, d);
                            if (dist2(d) < thr) {
                                if (pass) pj[o + cnt] = (int32_t)j;
                                ++cnt;
                            }
                        }
                    }
            if (!pass) {
                counts[i] = cnt;
            } else {
                int32_t *row = &pj[start[i]];
                for (int64_t a = 1; a < cnt; ++a) {
                    int32_t v = row[a];
                    int64_t k = a - 1;
                    while (k >= 0 && row[k] > v) { row[k + 1] = row[k]; --k; }
                    row[k + 1] = v;
                }
            }
        }
        if (pass == 0) {
            total = 0;
            for (int64_t i = 0; i < n; ++i) total += counts[i];
            *nnz = total;
            if (total > cap || !pj) pass_ok = 0;
        }
        free(start);
    }
    free(bin); free(head); free(list);
    if (!pass_ok) return pj ? ORACLE_ERR_CAPACITY : ORACLE_OK;
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* Weights                                                                  */

typedef struct {
    const float *shift, *scale, *W1, *b1, *W2, *b2, *W3, *b3;
    int n_out;
} net_view;

typedef struct {
    const float *C0;
    net_view *coef;   /* [(T-1) * n_elements] */
    net_view *energy; /* [n_elements] */
    int64_t total;
} weight_view;

static int64_t net_size(const oracle_cfg *c, int n_out) {
    int D = n_feat(c);
    return 2 * D + (int64_t)c->hidden1 * D + c->hidden1 + (int64_t)c->hidden2 * c->hidden1 + c->hidden2 +
           (int64_t)n_out * c->hidden2 + n_out;
}

static const float *bind_net(const oracle_cfg *c, const float *p, int n_out, net_view *v) {
    int D = n_feat(c);
    v->n_out = n_out;
    v->shift = p; p += D;
    v->scale = p; p += D;
    v->W1 = p; p += (int64_t)c->hidden1 * D;
    v->b1 = p; p += c->hidden1;
    v->W2 = p; p += (int64_t)c->hidden2 * c->hidden1;
    v->b2 = p; p += c->hidden2;
    v->W3 = p; p += (int64_t)n_out * c->hidden2;
    v->b3 = p; p += n_out;
    return p;
}

int64_t oracle_weight_count(const oracle_cfg *c) {
    int D = c->n_radial * (c->l_max + 1);
    return (int64_t)c->n_elements * D + (int64_t)(c->T - 1) * c->n_elements * net_size(c, D) +
           (int64_t)c->n_elements * net_size(c, 1);
}

static int bind_weights(const oracle_cfg *c, const float *w, weight_view *v) {
    int D = c->n_radial * (c->l_max + 1);
    v->C0 = w;
    const float *p = w + (int64_t)c->n_elements * D;
    v->coef = (net_view *)malloc(sizeof(net_view) * (size_t)((c->T > 1 ? c->T - 1 : 1) * c->n_elements));
    v->energy = (net_view *)malloc(sizeof(net_view) * (size_t)c->n_elements);
    if (!v->coef || !v->energy) return ORACLE_ERR_MEM;
    for (int t = 0; t < c->T - 1; ++t)
        for (int e = 0; e < c->n_elements; ++e) p = bind_net(c, p, D, &v->coef[t * c->n_elements + e]);
    for (int e = 0; e < c->n_elements; ++e) p = bind_net(c, p, 1, &v->energy[e]);
    v->total = p - w;
    return ORACLE_OK;
}

static void free_weights(weight_view *v) { free(v->coef); free(v->energy); }

static int check_cfg(const oracle_cfg *c) {
    if (!c || c->n_elements < 1 || c->T < 1 || c->n_radial < 2 || c->l_max < 0 || c->l_max > ORACLE_MAX_L ||
        c->hidden1 < 1 || c->hidden2 < 1 || !(c->r_cut > 0) || !(c->skin >= 0) || !(c->alpha > 0) ||
        c->density_form < 0 || c->density_form > 1 || n_feat(c) > 256)
        return ORACLE_ERR_ARG;
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* Atomic network and its vector-Jacobian product                           */

/* hidden activations a1[H1], a2[H2] are returned for reuse by the VJP */
static void net_forward(const oracle_cfg *c, const net_view *v, const double *x, double *a1, double *a2, double *y) {
    int D = n_feat(c), H1 = c->hidden1, H2 = c->hidden2;
    double xt[256];
    for (int f = 0; f < D; ++f) xt[f] = (x[f] - (double)v->shift[f]) / (double)v->scale[f];
    for (int h = 0; h < H1; ++h) {
        double z = v->b1[h];
        for (int f = 0; f < D; ++f) z += (double)v->W1[(int64_t)h * D + f] * xt[f];
        a1[h] = tanh(z);
    }
    for (int h = 0; h < H2; ++h) {
        double z = v->b2[h];
        for (int k = 0; k < H1; ++k) z += (double)v->W2[(int64_t)h * H1 + k] * a1[k];
        a2[h] = tanh(z);
    }
    for (int o = 0; o < v->n_out; ++o) {
        double z = v->b3[o];
        for (int k = 0; k < H2; ++k) z += (double)v->W3[(int64_t)o * H2 + k] * a2[k];
        y[o] = z;
    }
}

/* gx = (dy/dx)^T gy, given the activations of net_forward at the same x */
static void net_vjp(const oracle_cfg *c, const net_view *v, const double *a1, const double *a2, const double *gy,
                    double *gx) {
    int D = n_feat(c), H1 = c->hidden1, H2 = c->hidden2;
    double g2[512], g1[512];
    for (int k = 0; k < H2; ++k) {
        double s = 0.0;
        for (int o = 0; o < v->n_out; ++o) s += (double)v->W3[(int64_t)o * H2 + k] * gy[o];
        g2[k] = s * (1.0 - a2[k] * a2[k]);
    }
    for (int k = 0; k < H1; ++k) {
        double s = 0.0;
        for (int h = 0; h < H2; ++h) s += (double)v->W2[(int64_t)h * H1 + k] * g2[h];
        g1[k] = s * (1.0 - a1[k] * a1[k]);
    }
    for (int f = 0; f < D; ++f) {
        double s = 0.0;
        for (int h = 0; h < H1; ++h) s += (double)v->W1[(int64_t)h * D + f] * g1[h];
        gx[f] = s / (double)v->scale[f];
    }
}

/* ------------------------------------------------------------------------ */
/* Orbitals                                                                 */

/* phi_n(r) and dphi_n/dr for n = 0..N_phi-1 */
static void radial(const oracle_cfg *c, double r, double *phi, double *dphi) {
    const double pi = 3.14159265358979323846;
    double fc = 0.5 * (cos(pi * r / c->r_cut) + 1.0);
    double dfc = -0.5 * (pi / c->r_cut) * sin(pi * r / c->r_cut);
    for (int n = 0; n < c->n_radial; ++n) {
        double mu = c->r_cut * n / (double)(c->n_radial - 1);
        double g = exp(-c->alpha * (r - mu) * (r - mu));
        phi[n] = g * fc;
        if (dphi) dphi[n] = g * (-2.0 * c->alpha * (r - mu) * fc + dfc);
    }
}

static double ipow(double v, int k) {
    double p = 1.0;
    for (int i = 0; i < k; ++i) p *= v;
    return p;
}

/* Y_tau(d) and its gradient with respect to d */
static void angular(int ntau, const double d[3], double *Y, double (*dY)[3]) {
    for (int tau = 0; tau < ntau; ++tau) {
        const int *e = TUPLE[tau];
        Y[tau] = ipow(d[0], e[0]) * ipow(d[1], e[1]) * ipow(d[2], e[2]);
        if (dY) {
            dY[tau][0] = e[0] ? e[0] * ipow(d[0], e[0] - 1) * ipow(d[1], e[1]) * ipow(d[2], e[2]) : 0.0;
            dY[tau][1] = e[1] ? e[1] * ipow(d[0], e[0]) * ipow(d[1], e[1] - 1) * ipow(d[2], e[2]) : 0.0;
            dY[tau][2] = e[2] ? e[2] * ipow(d[0], e[0]) * ipow(d[1], e[1]) * ipow(d[2], e[2] - 1) : 0.0;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Density of one layer (Eq. 1)                                             */

/*
 * A[i][n*ntau + tau] and rho[i][*] of layer t for every centre (n_feat
 * features: l*N_phi + n, or l*P + pair(n, m) in the pair form), given the
 * neighbour list and the coefficients c[j][l*N_phi + n] of layer t.
 */
static void density_layer(const oracle_cfg *c, int64_t n, const double *x, const double *box, const int64_t *row,
                          const int32_t *col, const double *coef, double *A, double *rho) {
    int D = c->n_radial * (c->l_max + 1), ntau = n_tuples(c->l_max), NP = c->n_radial, DR = n_feat(c);
    int P = NP * (NP + 1) / 2;
    #pragma omp parallel for schedule(dynamic, 64)
    for (int64_t i = 0; i < n; ++i) {
        double *Ai = &A[i * NP * ntau];
        for (int k = 0; k < NP * ntau; ++k) Ai[k] = 0.0;
        for (int64_t q = row[i]; q < row[i + 1]; ++q) {
            int64_t j = col[q];
            double d[3];
            min_image(&x[3 * i], &x[3 * j], box, d);
            double r = sqrt(dist2(d));
            if (!(r < c->r_cut)) continue;
            double phi[64], Y[ORACLE_MAX_TUPLES];
            radial(c, r, phi, NULL);
            angular(ntau, d, Y, NULL);
            for (int nn = 0; nn < NP; ++nn)
                for (int tau = 0; tau < ntau; ++tau)
                    Ai[nn * ntau + tau] += coef[j * D + tuple_l(tau) * NP + nn] * phi[nn] * Y[tau];
        }
        for (int f = 0; f < DR; ++f) rho[i * DR + f] = 0.0;
        if (c->density_form == 1) {
            for (int nn = 0; nn < NP; ++nn)
                for (int mm = nn; mm < NP; ++mm)
                    for (int tau = 0; tau < ntau; ++tau)
                        rho[i * DR + tuple_l(tau) * P + pair_index(NP, nn, mm)] +=
                            tuple_weight(tau) * Ai[nn * ntau + tau] * Ai[mm * ntau + tau];
        } else {
            for (int nn = 0; nn < NP; ++nn)
                for (int tau = 0; tau < ntau; ++tau)
                    rho[i * DR + tuple_l(tau) * NP + nn] +=
                        tuple_weight(tau) * Ai[nn * ntau + tau] * Ai[nn * ntau + tau];
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Full evaluation                                                          */

/*
 * Energy and forces.  Inputs: n atoms, x[n][3] (A), types[n] in
 * [0, n_elements), box[3] (A, orthorhombic, periodic), the neighbour list
 * (row[n+1], col[nnz]; must contain every pair closer than r_cut), and the
 * float32 weight blob.  Outputs: *energy (eV), atom_energy[n] (eV, may be
 * NULL), forces[n][3] (eV/A, may be NULL).  When rho_out / coef_out / A_out
 * are non-NULL they receive every layer's rho^t [T][n][D], c^t [T][n][D]
 * and A^t [T][n][N_phi*ntau].
 */
int oracle_energy_forces(const oracle_cfg *c, const float *weights, int64_t weight_count, int64_t n,
                         const double *x, const int32_t *types, const double *box, const int64_t *row,
                         const int32_t *col, double *energy, double *atom_energy, double *forces,
                         double *rho_out, double *coef_out, double *A_out) {
    int rc = check_cfg(c);
    if (rc) return rc;
    if (c->hidden1 > 512 || c->hidden2 > 512 || c->n_radial > 21) return ORACLE_ERR_ARG;
    if (weight_count != oracle_weight_count(c)) return ORACLE_ERR_ARG;
    for (int64_t i = 0; i < n; ++i)
        if (types[i] < 0 || types[i] >= c->n_elements) return ORACLE_ERR_ARG;
    weight_view w;
    if (bind_weights(c, weights, &w)) return ORACLE_ERR_MEM;

    int T = c->T, D = c->n_radial * (c->l_max + 1), NP = c->n_radial, ntau = n_tuples(c->l_max), DR = n_feat(c);
    int P = NP * (NP + 1) / 2;
    int64_t nA = (int64_t)NP * ntau;
    double *rho = (double *)malloc(sizeof(double) * T * n * DR + 1);
    double *coef = (double *)malloc(sizeof(double) * T * n * D + 1);
    double *A = (double *)malloc(sizeof(double) * T * n * nA + 1);
    double *Ei = (double *)malloc(sizeof(double) * n + 1);
    if (!rho || !coef || !A || !Ei) return ORACLE_ERR_MEM;

    /* forward: c^0 from the element table, then layers 0..T-1 */
    for (int64_t i = 0; i < n; ++i)
        for (int f = 0; f < D; ++f) coef[i * D + f] = w.C0[types[i] * D + f];
    for (int t = 0; t < T; ++t) {
        density_layer(c, n, x, box, row, col, &coef[t * n * D], &A[t * n * nA], &rho[t * n * DR]);
        if (t + 1 < T) {
            #pragma omp parallel for schedule(static)
            for (int64_t i = 0; i < n; ++i) {
                double a1[512], a2[512];
                net_forward(c, &w.coef[t * c->n_elements + types[i]], &rho[(t * n + i) * DR], a1, a2,
                            &coef[((t + 1) * n + i) * D]);
            }
        }
    }
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        double a1[512], a2[512];
        net_forward(c, &w.energy[types[i]], &rho[((T - 1) * n + i) * DR], a1, a2, &Ei[i]);
    }
    double E = 0.0;
    for (int64_t i = 0; i < n; ++i) E += Ei[i];
    if (energy) *energy = E;
    if (atom_energy)
        for (int64_t i = 0; i < n; ++i) atom_energy[i] = Ei[i];

    if (forces) {
        int nth = oracle_num_threads();
        double *g = (double *)malloc(sizeof(double) * n * DR + 1);       /* dE/drho^t */
        double *gc = (double *)malloc(sizeof(double) * n * D + 1);       /* dE/dc^t */
        double *gx_t = (double *)calloc((size_t)nth * n * 3 + 1, sizeof(double));
        double *gc_t = (double *)calloc((size_t)nth * n * D + 1, sizeof(double));
        if (!g || !gc || !gx_t || !gc_t) return ORACLE_ERR_MEM;

        /* Eq. 3: dE/drho^{T-1} through the energy network */
        #pragma omp parallel for schedule(static)
        for (int64_t i = 0; i < n; ++i) {
            double a1[512], a2[512], y, one = 1.0;
            const net_view *v = &w.energy[types[i]];
            net_forward(c, v, &rho[((T - 1) * n + i) * DR], a1, a2, &y);
            net_vjp(c, v, a1, a2, &one, &g[i * DR]);
        }
        for (int t = T - 1; t >= 0; --t) {
            const double *ct = &coef[t * n * D];
            const double *At = &A[t * n * nA];
            memset(gc_t, 0, sizeof(double) * (size_t)nth * n * D);
            /* Eq. 4 for centre i and active neighbour j:
             *   dE/dA_{i,n,tau} = 2 w_tau A_{i,n,tau} dE/drho_{i,(n,l)}
             *     (pair form: w_tau sum_m (1 + [m = n]) A_{i,m,tau} dE/drho_{i,(min, max of n m, l)})
             *   message term:  dE/dc_{j,(n,l)} += sum_tau dE/dA_{i,n,tau} phi_n Y_tau
             *   direct term:   dE/dd_ij = sum_{n,tau} dE/dA_{i,n,tau} c_{j,(n,l)} d(phi_n Y_tau)/dd
             *                  with dd_ij/dx_j = +1 and dd_ij/dx_i = -1 */
            #pragma omp parallel for schedule(dynamic, 64)
            for (int64_t i = 0; i < n; ++i) {
                int th = 0;
#ifdef _OPENMP
                th = omp_get_thread_num();
#endif
                double *gx = &gx_t[(int64_t)th * n * 3];
                double *gcl = &gc_t[(int64_t)th * n * D];
                double GA[21 * ORACLE_MAX_TUPLES];
                for (int nn = 0; nn < NP; ++nn)
                    for (int tau = 0; tau < ntau; ++tau) {
                        if (c->density_form == 1) {
                            double s = 0.0;
                            for (int mm = 0; mm < NP; ++mm) {
                                int a = nn < mm ? nn : mm, b = nn < mm ? mm : nn;
                                s += (mm == nn ? 2.0 : 1.0) * At[i * nA + mm * ntau + tau] *
                                     g[i * DR + tuple_l(tau) * P + pair_index(NP, a, b)];
                            }
                            GA[nn * ntau + tau] = tuple_weight(tau) * s;
                        } else {
                            GA[nn * ntau + tau] = 2.0 * tuple_weight(tau) * At[i * nA + nn * ntau + tau] *
                                                  g[i * DR + tuple_l(tau) * NP + nn];
                        }
                    }
                for (int64_t q = row[i]; q < row[i + 1]; ++q) {
                    int64_t j = col[q];
                    double d[3];
                    min_image(&x[3 * i], &x[3 * j], box, d);
                    double r = sqrt(dist2(d));
                    if (!(r < c->r_cut)) continue;
                    double phi[64], dphi[64], Y[ORACLE_MAX_TUPLES], dY[ORACLE_MAX_TUPLES][3];
                    radial(c, r, phi, dphi);
                    angular(ntau, d, Y, dY);
                    double V[3] = {0.0, 0.0, 0.0};
                    for (int nn = 0; nn < NP; ++nn)
                        for (int tau = 0; tau < ntau; ++tau) {
                            int f = tuple_l(tau) * NP + nn;
                            double ga = GA[nn * ntau + tau];
                            gcl[j * D + f] += ga * phi[nn] * Y[tau];
                            double cj = ct[j * D + f];
                            for (int a = 0; a < 3; ++a)
                                V[a] += ga * cj * (dphi[nn] * (d[a] / r) * Y[tau] + phi[nn] * dY[tau][a]);
                        }
                    for (int a = 0; a < 3; ++a) {
                        gx[j * 3 + a] += V[a];
                        gx[i * 3 + a] -= V[a];
                    }
                }
            }
            /* reduce the per-thread message gradients: dE/dc^t */
            #pragma omp parallel for schedule(static)
            for (int64_t k = 0; k < n * D; ++k) {
                double s = 0.0;
                for (int th = 0; th < nth; ++th) s += gc_t[(int64_t)th * n * D + k];
                gc[k] = s;
            }
            /* Eq. 5: dE/drho^{t-1} = (dc^t/drho^{t-1})^T dE/dc^t; c^0 is constant */
            if (t >= 1) {
                #pragma omp parallel for schedule(static)
                for (int64_t i = 0; i < n; ++i) {
                    double a1[512], a2[512], y[64];
                    const net_view *v = &w.coef[(t - 1) * c->n_elements + types[i]];
                    net_forward(c, v, &rho[((t - 1) * n + i) * DR], a1, a2, y);
                    net_vjp(c, v, a1, a2, &gc[i * D], &g[i * DR]);
                }
            }
        }
        for (int64_t i = 0; i < n; ++i)
            for (int a = 0; a < 3; ++a) {
                double s = 0.0;
                for (int th = 0; th < nth; ++th) s += gx_t[(int64_t)th * n * 3 + i * 3 + a];
                forces[i * 3 + a] = -s;
            }
        free(g); free(gc); free(gx_t); free(gc_t);
    }
    if (rho_out) memcpy(rho_out, rho, sizeof(double) * T * n * DR);
    if (coef_out) memcpy(coef_out, coef, sizeof(double) * T * n * D);
    if (A_out) memcpy(A_out, A, sizeof(double) * T * n * nA);
    free(rho); free(coef); free(A); free(Ei);
    free_weights(&w);
    return ORACLE_OK;
}

/*
 * A second formula for rho^t used only to pin density_layer: by the
 * multinomial theorem, sum_{|tau|=l} l!/tau! Y_tau(d_j) Y_tau(d_k) = (d_j . d_k)^l,
 * so rho_{i,(n,l)} = sum_{j,k} a_j a_k (d_ij . d_ik)^l with
 * a_j = c_{j,(n,l)} phi_n(r_ij), over the active neighbours j, k of i.
 * Pair form: rho_{i,(n,m,l)} = sum_{j,k} a_{j,n} b_{k,m} (d_ij . d_ik)^l with
 * b_{k,m} = c_{k,(m,l)} phi_m(r_ik).  No Cartesian tuple appears.
 */
int oracle_rho_pairwise(const oracle_cfg *c, int64_t n, const double *x, const double *box, const int64_t *row,
                        const int32_t *col, const double *coef, double *rho) {
    int rc = check_cfg(c);
    if (rc) return rc;
    int D = c->n_radial * (c->l_max + 1), NP = c->n_radial, DR = n_feat(c), P = NP * (NP + 1) / 2;
    #pragma omp parallel for schedule(dynamic, 16)
    for (int64_t i = 0; i < n; ++i) {
        int64_t deg = row[i + 1] - row[i];
        double *dv = (double *)malloc(sizeof(double) * 3 * (deg + 1));
        double *ph = (double *)malloc(sizeof(double) * NP * (deg + 1));
        int64_t *nb = (int64_t *)malloc(sizeof(int64_t) * (deg + 1));
        int64_t m = 0;
        for (int64_t q = row[i]; q < row[i + 1]; ++q) {
            double d[3];
            min_image(&x[3 * i], &x[3 * col[q]], box, d);
            double r = sqrt(dist2(d));
            if (!(r < c->r_cut)) continue;
            radial(c, r, &ph[m * NP], NULL);
            for (int a = 0; a < 3; ++a) dv[3 * m + a] = d[a];
            nb[m++] = col[q];
        }
        for (int f = 0; f < DR; ++f) rho[i * DR + f] = 0.0;
        for (int64_t p = 0; p < m; ++p)
            for (int64_t q = 0; q < m; ++q) {
                double dot = dv[3 * p] * dv[3 * q] + dv[3 * p + 1] * dv[3 * q + 1] + dv[3 * p + 2] * dv[3 * q + 2];
                for (int l = 0; l <= c->l_max; ++l)
                    for (int nn = 0; nn < NP; ++nn)
                        for (int mm = nn; mm < (c->density_form == 1 ? NP : nn + 1); ++mm) {
                            int fn = l * NP + nn, fm = l * NP + mm;
                            int f = c->density_form == 1 ? l * P + pair_index(NP, nn, mm) : fn;
                            rho[i * DR + f] += coef[nb[p] * D + fn] * ph[p * NP + nn] * coef[nb[q] * D + fm] *
                                               ph[q * NP + mm] * ipow(dot, l);
                        }
            }
        free(dv); free(ph); free(nb);
    }
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* Velocity-Verlet MD                                                       */

static int brute_csr(int64_t n, const double *x, const double *box, double r_cut, double skin, int64_t **row,
                     int32_t **col) {
    int64_t *counts = (int64_t *)malloc(sizeof(int64_t) * (n + 1));
    int64_t nnz = 0;
    int rc = oracle_pairs_brute(n, x, box, r_cut, skin, 0, NULL, 0, counts, NULL, &nnz);
    if (rc) { free(counts); return rc; }
    *col = (int32_t *)malloc(sizeof(int32_t) * (nnz + 1));
    rc = oracle_pairs_brute(n, x, box, r_cut, skin, 0, NULL, nnz, counts, *col, &nnz);
    if (rc) { free(counts); free(*col); return rc; }
    *row = (int64_t *)malloc(sizeof(int64_t) * (n + 1));
    (*row)[0] = 0;
    for (int64_t i = 0; i < n; ++i) (*row)[i + 1] = (*row)[i] + counts[i];
    free(counts);
    return ORACLE_OK;
}

/*
 * nsteps of velocity Verlet with time step dt (fs): v += F/m dt/2;
 * x += v dt; wrap x into [0, L); recompute F (fresh brute-force list every
 * step); v += F/m dt/2.  x [n][3] in A and v [n][3] in A/fs are updated in
 * place; masses are per element in amu.  epot[s] and ekin[s] (eV) are
 * recorded for s = 0..nsteps (s = 0 is the initial state).  The unit of
 * acceleration is 1 eV/(A amu) = 1/103.6426965 A/fs^2.
 */
/*
 * Velocity Verlet (NVE) and, with a thermostat, canonical sampling by
 * stochastic velocity rescaling (Bussi, Donadio and Parrinello, J. Chem. Phys.
 * 126, 014101 (2007)): after each step the kinetic energy K is replaced by
 *   K' = K + (1 - c) (Kt (R1^2 + S) / Nf - K) + 2 R1 sqrt(c (1 - c) K Kt / Nf),
 * c = exp(-dt / tau), Kt = Nf kB T / 2, Nf = 3 n - 3, by scaling every velocity
 * by sqrt(K' / K).  R1 (standard normal) and S (a sum of Nf - 1 squared
 * standard normals) are inputs, two per step, so that any two implementations
 * given the same numbers take the same steps.  work[s] accumulates K' - K, the
 * energy the thermostat has added up to step s.
 */
static int md_run(const oracle_cfg *c, const float *weights, int64_t weight_count, int64_t n, double *x, double *v,
                  const int32_t *types, const double *box, const double *mass, double dt, int32_t nsteps,
                  const double *thermo, const double *noise, double *epot, double *ekin, double *work) {
    const double conv = 1.0 / 103.6426965, kB = 8.617333262e-5;
    double *F = (double *)malloc(sizeof(double) * 3 * n + 1);
    int64_t *row = NULL;
    int32_t *col = NULL;
    double E = 0.0, W = 0.0;
    int rc = brute_csr(n, x, box, c->r_cut, c->skin, &row, &col);
    if (rc) { free(F); return rc; }
    rc = oracle_energy_forces(c, weights, weight_count, n, x, types, box, row, col, &E, NULL, F, NULL, NULL, NULL);
    free(row); free(col);
    if (rc) { free(F); return rc; }
    for (int s = 0; s <= nsteps; ++s) {
        if (s > 0) {
            for (int64_t i = 0; i < n; ++i)
                for (int a = 0; a < 3; ++a) {
                    v[3 * i + a] += 0.5 * dt * conv * F[3 * i + a] / mass[types[i]];
                    x[3 * i + a] += dt * v[3 * i + a];
                    x[3 * i + a] -= box[a] * floor(x[3 * i + a] / box[a]);
                }
            rc = brute_csr(n, x, box, c->r_cut, c->skin, &row, &col);
            if (rc) { free(F); return rc; }
            rc = oracle_energy_forces(c, weights, weight_count, n, x, types, box, row, col, &E, NULL, F, NULL, NULL,
                                      NULL);
            free(row); free(col);
            if (rc) { free(F); return rc; }
            for (int64_t i = 0; i < n; ++i)
                for (int a = 0; a < 3; ++a) v[3 * i + a] += 0.5 * dt * conv * F[3 * i + a] / mass[types[i]];
        }
        double K = 0.0;
        for (int64_t i = 0; i < n; ++i)
            for (int a = 0; a < 3; ++a) K += 0.5 * mass[types[i]] * v[3 * i + a] * v[3 * i + a];
        K *= 103.6426965;   /* eV */
        if (thermo && s > 0 && K > 0.0) {
            const double T = thermo[0], tau = thermo[1];
            const double Nf = (double)(3 * n - 3), Kt = 0.5 * Nf * kB * T;
            const double cc = tau > 0.0 ? exp(-dt / tau) : 0.0;
            const double R1 = noise[2 * (s - 1)], S = noise[2 * (s - 1) + 1];
            const double Kn =
                K + (1.0 - cc) * (Kt * (R1 * R1 + S) / Nf - K) + 2.0 * R1 * sqrt(cc * (1.0 - cc) * K * Kt / Nf);
            const double alpha = sqrt(Kn / K);
            for (int64_t i = 0; i < 3 * n; ++i) v[i] *= alpha;
            W += Kn - K;
            K = Kn;
        }
        if (epot) epot[s] = E;
        if (ekin) ekin[s] = K;
        if (work) work[s] = W;
    }
    free(F);
    return ORACLE_OK;
}

int oracle_md_verlet(const oracle_cfg *c, const float *weights, int64_t weight_count, int64_t n, double *x,
                     double *v, const int32_t *types, const double *box, const double *mass, double dt,
                     int32_t nsteps, double *epot, double *ekin) {
    return md_run(c, weights, weight_count, n, x, v, types, box, mass, dt, nsteps, NULL, NULL, epot, ekin, NULL);
}

/* thermo = {T (K), tau (fs; +inf: no coupling, 0: full resampling)}, noise [nsteps][2] */
int oracle_md_nvt(const oracle_cfg *c, const float *weights, int64_t weight_count, int64_t n, double *x, double *v,
                  const int32_t *types, const double *box, const double *mass, double dt, int32_t nsteps,
                  const double *thermo, const double *noise, double *epot, double *ekin, double *work) {
    if (!thermo || !noise || n < 2 || !(thermo[0] > 0.0) || !(thermo[1] >= 0.0)) return ORACLE_ERR_ARG;
    return md_run(c, weights, weight_count, n, x, v, types, box, mass, dt, nsteps, thermo, noise, epot, ekin, work);
}
