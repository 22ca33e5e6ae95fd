/*
 * Test infrastructure, not product code: a plain, slow fp64 CPU restatement
 * of the edge-aware attention layer of "Efficient Edge-aware Attention
 * Network for Graph Generation" (FlexAttentionGT).  Only the tests, the
 * smoke check and the benchmark's CPU-baseline leg load this file; the CUDA
 * library shares no code with it.
 *
 * What the pages fix (AI summary page, method paragraph; blog summary,
 * "Design Strategy of the Edge-aware Attention Layer"):
 *   - scaled dot-product attention per head replaces the per-channel outer
 *     product of the graph transformer;
 *   - edge features E_ij and the graph's global features y enter the score
 *     through a head-wise FiLM applied inside the score modification;
 *   - the graph mask is respected (mask modification);
 *   - one attention call yields both the node aggregation and the
 *     *normalised* attention coefficients (identity concatenated to V);
 *   - edges get a lightweight residual update from those coefficients.
 * Where the pages stop, the readings below are the plain ones:
 *   gamma,beta = E_ij Wfe + y_b Wfy + bf  (columns 0..H-1 gamma, H..2H-1 beta)
 *   s'   = (q_i . k_j / sqrt(dh)) * (1 + gamma_h) + beta_h
 *   a    = masked softmax over j of s' (valid pair: M_i and M_j; a = 0 else)
 *   O_ih = sum_j a_ij v_jh
 *   E'   = E + sum_h a^h We[h,:]         (no bias)
 *   X'   = X + M_i (O_i Wo + bo)
 * Weights are [in, out] row-major (Y = X W).  Every loop below follows these
 * formulas in the order written; there is no blocking or reordering.
 *
 * Two ablation variants of the layer (AI summary page: the method
 * paragraph's ablation of unnormalised coefficients, and the "Light Edge"
 * bullet), selected by `variant`:
 *   ORC_LIGHT_EDGE   no per-edge modulation: gamma, beta = y_b Wfy + bf (Wfe
 *                    is not used and its gradient is zero);
 *   ORC_UNNORMALISED the edge update takes the unnormalised coefficients, the
 *                    modulated scores themselves: E' = E + sum_h s'^h We[h,:]
 *                    on valid pairs (invalid pairs keep E); nodes unchanged.
 *
 * Parity pins (tests/test_oracle_pins.py): zero-FiLM special case against
 * torch's float64 scaled_dot_product_attention; the gamma = -1 closed form
 * (uniform attention); row sums; masked-entry invariance; permutation
 * equivariance; a brute-force per-pair Python evaluation without max
 * subtraction; the [V | I] formulation; beta-shift invariance; the Light
 * Edge case (Wfe = 0) against scaled dot-product attention at a per-graph,
 * per-head temperature, with its vanishing key-bias gradient; and fp64
 * central finite differences of orc_forward for every gradient orc_backward
 * returns.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

typedef struct { int B, n, dx, de, dy, H, dh; } orc_dims;
enum { ORC_LAYER = 0, ORC_LIGHT_EDGE = 1, ORC_UNNORMALISED = 2 };
typedef struct {
    const double *Wq, *bq, *Wk, *bk, *Wv, *bv, *Wfe, *Wfy, *bf, *We, *Wo, *bo;
} orc_weights;
typedef struct {
    double *Wq, *bq, *Wk, *bk, *Wv, *bv, *Wfe, *Wfy, *bf, *We, *Wo, *bo;
} orc_grads;

/* Y[r, :] = X[r, :] W + b for r in [0, rows): X [rows, in], W [in, out]. */
static void linear(const double *X, const double *W, const double *b, double *Y,
                   long rows, int in, int out)
{
    #pragma omp parallel for schedule(static)
    for (long r = 0; r < rows; ++r) {
        for (int o = 0; o < out; ++o) {
            double acc = b ? b[o] : 0.0;
            for (int k = 0; k < in; ++k) acc += X[r * in + k] * W[(long)k * out + o];
            Y[r * out + o] = acc;
        }
    }
}

/* Per-head FiLM coefficients of pair (b,i,j): f[k] = E_bij . Wfe[:,k] + g_b[k]. */
static void film(const orc_dims *d, const double *E, const double *Wfe, const double *g,
                 int b, int i, int j, double *f)
{
    const double *e = E + (((long)b * d->n + i) * d->n + j) * d->de;
    for (int k = 0; k < 2 * d->H; ++k) {
        double acc = g[(long)b * 2 * d->H + k];
        for (int c = 0; c < d->de; ++c) acc += e[c] * Wfe[(long)c * 2 * d->H + k];
        f[k] = acc;
    }
}

/* Raw score s = q_i^h . k_j^h / sqrt(dh). */
static double raw_score(const orc_dims *d, const double *Q, const double *K,
                        int b, int h, int i, int j)
{
    const int hd = d->H * d->dh;
    const double *q = Q + ((long)b * d->n + i) * hd + h * d->dh;
    const double *k = K + ((long)b * d->n + j) * hd + h * d->dh;
    double acc = 0.0;
    for (int t = 0; t < d->dh; ++t) acc += q[t] * k[t];
    return acc / sqrt((double)d->dh);
}

/* Node projections Q, K, V [B*n, H*dh] and the global FiLM term g [B, 2H]. */
static void project(const orc_dims *d, const double *X, const double *y, const orc_weights *w,
                    double *Q, double *K, double *V, double *g)
{
    const long rows = (long)d->B * d->n;
    const int hd = d->H * d->dh;
    linear(X, w->Wq, w->bq, Q, rows, d->dx, hd);
    linear(X, w->Wk, w->bk, K, rows, d->dx, hd);
    linear(X, w->Wv, w->bv, V, rows, d->dx, hd);
    linear(y, w->Wfy, w->bf, g, d->B, d->dy, 2 * d->H);
}

/*
 * Masked softmax of row (b,i), head h, over j: a[j] for j in [0,n), and the
 * row's max m and normaliser l.  Returns 0 and a = 0 when row i is masked.
 * sp[j] holds the modulated scores s'_ij on entry (ignored at invalid j).
 */
static int masked_softmax(const orc_dims *d, const unsigned char *M, int b, int i,
                          const double *sp, double *a, double *m_out, double *l_out)
{
    const unsigned char *mb = M + (long)b * d->n;
    for (int j = 0; j < d->n; ++j) a[j] = 0.0;
    if (!mb[i]) { *m_out = 0.0; *l_out = 0.0; return 0; }
    double m = -INFINITY;
    for (int j = 0; j < d->n; ++j)
        if (mb[j] && sp[j] > m) m = sp[j];
    double l = 0.0;
    for (int j = 0; j < d->n; ++j)
        if (mb[j]) l += exp(sp[j] - m);
    for (int j = 0; j < d->n; ++j)
        if (mb[j]) a[j] = exp(sp[j] - m) / l;
    *m_out = m; *l_out = l;
    return 1;
}

/* Attention coefficients of row (b,i) for all heads: arow [H][n]; plus the
 * raw scores s [H][n] and FiLM coefficients f [n][2H] used on the way. */
static void row_attention(const orc_dims *d, const double *E, const unsigned char *M,
                          const double *Q, const double *K, const double *Wfe, const double *g,
                          int b, int i, double *arow, double *srow, double *frow, double *lse)
{
    const int n = d->n, H = d->H;
    double *sp = (double *)malloc(sizeof(double) * n);
    for (int j = 0; j < n; ++j) film(d, E, Wfe, g, b, i, j, frow + (long)j * 2 * H);
    for (int h = 0; h < H; ++h) {
        for (int j = 0; j < n; ++j) {
            double s = raw_score(d, Q, K, b, h, i, j);
            double gam = frow[(long)j * 2 * H + h];
            double bet = frow[(long)j * 2 * H + H + h];
            srow[(long)h * n + j] = s;
            sp[j] = s * (1.0 + gam) + bet;
        }
        double m, l;
        int valid = masked_softmax(d, M, b, i, sp, arow + (long)h * n, &m, &l);
        if (lse) lse[h] = valid ? m + log(l) : -INFINITY;
    }
    free(sp);
}

/*
 * Forward.  All arrays fp64, row-major, contiguous:
 *   X [B,n,dx]  E [B,n,n,de]  y [B,dy]  M [B,n] (0/1)
 *   Xout [B,n,dx]  Eout [B,n,n,de]
 *   A   [B,H,n,n]  (nullable) normalised coefficients a^h_ij
 *   O   [B,n,H*dh] (nullable) node aggregation before the output projection
 *   LSE [B,H,n]   (nullable) m + log l per valid row, -inf on masked rows
 * Returns 0.
 */
int orc_forward_variant(const orc_dims *d, int variant, const double *X, const double *E, const double *y,
                        const unsigned char *M, const orc_weights *w,
                        double *Xout, double *Eout, double *A, double *O, double *LSE)
{
    const int B = d->B, n = d->n, H = d->H, dh = d->dh, hd = H * dh, de = d->de, dx = d->dx;
    const long rows = (long)B * n;
    /* Light Edge: the per-edge FiLM map is absent (zero) */
    double *Wfe0 = (double *)calloc((size_t)de * 2 * H, sizeof(double));
    const double *Wfe = variant == ORC_LIGHT_EDGE ? Wfe0 : w->Wfe;
    double *Q = (double *)malloc(sizeof(double) * rows * hd);
    double *K = (double *)malloc(sizeof(double) * rows * hd);
    double *V = (double *)malloc(sizeof(double) * rows * hd);
    double *g = (double *)malloc(sizeof(double) * B * 2 * H);
    double *Ob = (double *)malloc(sizeof(double) * rows * hd);
    project(d, X, y, w, Q, K, V, g);

    #pragma omp parallel for schedule(dynamic, 1)
    for (long r = 0; r < rows; ++r) {
        const int b = (int)(r / n), i = (int)(r % n);
        double *arow = (double *)malloc(sizeof(double) * H * n);
        double *srow = (double *)malloc(sizeof(double) * H * n);
        double *frow = (double *)malloc(sizeof(double) * n * 2 * H);
        double lse[64];
        row_attention(d, E, M, Q, K, Wfe, g, b, i, arow, srow, frow, lse);
        /* node aggregation O_ih = sum_j a_ij v_jh */
        for (int h = 0; h < H; ++h)
            for (int t = 0; t < dh; ++t) {
                double acc = 0.0;
                for (int j = 0; j < n; ++j)
                    acc += arow[(long)h * n + j] * V[((long)b * n + j) * hd + h * dh + t];
                Ob[r * hd + h * dh + t] = acc;
            }
        /* edge residual E'_ij = E_ij + sum_h coef^h_ij We[h,:], coef = a (the layer) or,
           unnormalised, the modulated score s' on valid pairs and 0 elsewhere */
        for (int j = 0; j < n; ++j) {
            const long e0 = (((long)b * n + i) * n + j) * de;
            const int valid = M[(long)b * n + i] && M[(long)b * n + j];
            for (int c = 0; c < de; ++c) {
                double acc = E[e0 + c];
                for (int h = 0; h < H; ++h) {
                    double coef = arow[(long)h * n + j];
                    if (variant == ORC_UNNORMALISED) {
                        const double sp = srow[(long)h * n + j] * (1.0 + frow[(long)j * 2 * H + h]) +
                                          frow[(long)j * 2 * H + H + h];
                        coef = valid ? sp : 0.0;
                    }
                    acc += coef * w->We[(long)h * de + c];
                }
                Eout[e0 + c] = acc;
            }
        }
        if (A)
            for (int h = 0; h < H; ++h)
                for (int j = 0; j < n; ++j)
                    A[(((long)b * H + h) * n + i) * n + j] = arow[(long)h * n + j];
        if (LSE)
            for (int h = 0; h < H; ++h) LSE[((long)b * H + h) * n + i] = lse[h];
        free(arow); free(srow); free(frow);
    }
    /* node residual X' = X + M (O Wo + bo) */
    #pragma omp parallel for schedule(static)
    for (long r = 0; r < rows; ++r) {
        const int b = (int)(r / n), i = (int)(r % n);
        const double mi = M[(long)b * n + i] ? 1.0 : 0.0;
        for (int o = 0; o < dx; ++o) {
            double acc = w->bo[o];
            for (int k = 0; k < hd; ++k) acc += Ob[r * hd + k] * w->Wo[(long)k * dx + o];
            Xout[r * dx + o] = X[r * dx + o] + (mi != 0.0 ? acc : 0.0);
        }
    }
    if (O) memcpy(O, Ob, sizeof(double) * rows * hd);
    free(Q); free(K); free(V); free(g); free(Ob); free(Wfe0);
    return 0;
}

int orc_forward(const orc_dims *d, const double *X, const double *E, const double *y,
                const unsigned char *M, const orc_weights *w,
                double *Xout, double *Eout, double *A, double *O, double *LSE)
{
    return orc_forward_variant(d, ORC_LAYER, X, E, y, M, w, Xout, Eout, A, O, LSE);
}

/*
 * Backward of orc_forward, given the upstream gradients dXout [B,n,dx] and
 * dEout [B,n,n,de].  Writes dX, dE, dy (same shapes as X, E, y) and every
 * weight gradient in gr (same shapes as the weights; overwritten).
 *
 * Chain rule through the forward formulas, written out:
 *   dO_i   = M_i dX'_i Wo^T;  dWo = sum_i M_i O_i^T dX'_i;  dbo = sum_i M_i dX'_i
 *   u_ij^h = We[h,:] . dE'_ij;  dA_ij^h = dO_ih . v_jh + u_ij^h
 *   D_ih   = sum_j a_ij^h dA_ij^h;  dS'_ij = a_ij (dA_ij - D_ih)   (softmax)
 *   dgamma = dS' s;  dbeta = dS';  ds = dS' (1 + gamma)
 *   dq_i   = sum_j ds_ij k_j / sqrt(dh);  dk_j = sum_i ds_ij q_i / sqrt(dh)
 *   dv_j   = sum_i a_ij dO_i
 *   df     = [dgamma | dbeta];  dE = dE' + df Wfe^T;  dWfe = sum E_ij^T df_ij
 *   dg_b   = sum_ij df_ij;  dWfy = sum_b y_b^T dg_b;  dbf = sum_b dg_b;  dy_b = dg_b Wfy^T
 *   dWe    = sum_ij a_ij^T dE'_ij
 *   dX     = dX' + dQ Wq^T + dK Wk^T + dV Wv^T;  dW{q,k,v} = X^T d{Q,K,V};  db = sum d{Q,K,V}
 * Row work (D, dq, dE, per-row weight-gradient parts) runs per (b,i); column
 * work (dk, dv) per (b,j), recomputing a_ij; per-row parts are summed in row
 * order afterwards.
 *
 * Variants.  Light Edge: Wfe is zero in every formula above and its gradient
 * dWfe is zero (the map is not a parameter of that layer).  Unnormalised: the
 * edge update reads s' itself, so the edge path reaches s' without the
 * softmax:  D_ih = sum_j a_ij dO_ih . v_jh  (node path only),
 *   dS'_ij = a_ij (dO_ih . v_jh - D_ih) + [valid_ij] u_ij,
 *   dWe = sum_ij [valid_ij] s'_ij^T dE'_ij;  everything downstream of dS' as above.
 */
int orc_backward_variant(const orc_dims *d, int variant, const double *X, const double *E, const double *y,
                         const unsigned char *M, const orc_weights *w,
                         const double *dXout, const double *dEout,
                         double *dX, double *dE, double *dy, orc_grads *gr)
{
    const int B = d->B, n = d->n, H = d->H, dh = d->dh, hd = H * dh, de = d->de;
    const int dx = d->dx, dyd = d->dy, F = 2 * H;
    const long rows = (long)B * n;
    const int unnorm = variant == ORC_UNNORMALISED;
    double *Wfe0 = (double *)calloc((size_t)de * F, sizeof(double));
    const double *Wfe = variant == ORC_LIGHT_EDGE ? Wfe0 : w->Wfe;
    const double rs = 1.0 / sqrt((double)dh);
    double *Q = (double *)malloc(sizeof(double) * rows * hd);
    double *K = (double *)malloc(sizeof(double) * rows * hd);
    double *V = (double *)malloc(sizeof(double) * rows * hd);
    double *g = (double *)malloc(sizeof(double) * B * F);
    double *O = (double *)calloc((size_t)rows * hd, sizeof(double));
    double *dO = (double *)calloc((size_t)rows * hd, sizeof(double));
    double *dQ = (double *)calloc((size_t)rows * hd, sizeof(double));
    double *dK = (double *)calloc((size_t)rows * hd, sizeof(double));
    double *dV = (double *)calloc((size_t)rows * hd, sizeof(double));
    double *Dst = (double *)calloc((size_t)rows * H, sizeof(double));
    double *LSE = (double *)malloc(sizeof(double) * rows * H);
    /* per-row parts of dWfe [de,F], dWe [H,de], dg [F] */
    const long part = (long)de * F + (long)H * de + F;
    double *parts = (double *)calloc((size_t)rows * part, sizeof(double));
    project(d, X, y, w, Q, K, V, g);

    /* ---- row pass: a, O, dO, D, dS', dq, dE, row parts ---- */
    #pragma omp parallel for schedule(dynamic, 1)
    for (long r = 0; r < rows; ++r) {
        const int b = (int)(r / n), i = (int)(r % n);
        const double mi = M[r] ? 1.0 : 0.0;
        double *arow = (double *)malloc(sizeof(double) * H * n);
        double *srow = (double *)malloc(sizeof(double) * H * n);
        double *frow = (double *)malloc(sizeof(double) * n * F);
        double *dA = (double *)malloc(sizeof(double) * H * n);
        double *df = (double *)calloc((size_t)n * F, sizeof(double));
        double lse[64];
        row_attention(d, E, M, Q, K, Wfe, g, b, i, arow, srow, frow, lse);
        for (int h = 0; h < H; ++h) LSE[r * H + h] = lse[h];
        for (int h = 0; h < H; ++h)
            for (int t = 0; t < dh; ++t) {
                double acc = 0.0;
                for (int j = 0; j < n; ++j)
                    acc += arow[(long)h * n + j] * V[((long)b * n + j) * hd + h * dh + t];
                O[r * hd + h * dh + t] = acc;
            }
        /* dO_i = M_i dX'_i Wo^T */
        for (int k = 0; k < hd; ++k) {
            double acc = 0.0;
            for (int o = 0; o < dx; ++o) acc += dXout[r * dx + o] * w->Wo[(long)k * dx + o];
            dO[r * hd + k] = mi * acc;
        }
        /* dA and D (the unnormalised variant: the node term only in dA and D, u added to dS') */
        double *urow = (double *)malloc(sizeof(double) * n);
        for (int h = 0; h < H; ++h) {
            double D = 0.0;
            for (int j = 0; j < n; ++j) {
                const double *dep = dEout + (((long)b * n + i) * n + j) * de;
                double u = 0.0;
                for (int c = 0; c < de; ++c) u += w->We[(long)h * de + c] * dep[c];
                double dov = 0.0;
                for (int t = 0; t < dh; ++t)
                    dov += dO[r * hd + h * dh + t] * V[((long)b * n + j) * hd + h * dh + t];
                urow[j] = (M[r] && M[(long)b * n + j]) ? u : 0.0;
                dA[(long)h * n + j] = unnorm ? dov : dov + u;
                D += arow[(long)h * n + j] * dA[(long)h * n + j];
            }
            Dst[r * H + h] = D;
            for (int j = 0; j < n; ++j) {
                const double a = arow[(long)h * n + j];
                const double dsp = a * (dA[(long)h * n + j] - D) + (unnorm ? urow[j] : 0.0);
                const double gam = frow[(long)j * F + h];
                const double s = srow[(long)h * n + j];
                df[(long)j * F + h] = dsp * s;          /* dgamma */
                df[(long)j * F + H + h] = dsp;          /* dbeta  */
                const double ds = dsp * (1.0 + gam);
                for (int t = 0; t < dh; ++t)
                    dQ[r * hd + h * dh + t] += ds * K[((long)b * n + j) * hd + h * dh + t] * rs;
            }
        }
        /* dE = dE' + df Wfe^T; row parts of dWfe, dWe, dg */
        double *pWfe = parts + r * part;
        double *pWe = pWfe + (long)de * F;
        double *pg = pWe + (long)H * de;
        for (int j = 0; j < n; ++j) {
            const long e0 = (((long)b * n + i) * n + j) * de;
            const int valid = M[r] && M[(long)b * n + j];
            for (int c = 0; c < de; ++c) {
                double acc = dEout[e0 + c];
                for (int k = 0; k < F; ++k) acc += df[(long)j * F + k] * Wfe[(long)c * F + k];
                dE[e0 + c] = acc;
                for (int k = 0; k < F; ++k) pWfe[(long)c * F + k] += E[e0 + c] * df[(long)j * F + k];
                for (int h = 0; h < H; ++h) {
                    double coef = arow[(long)h * n + j];
                    if (unnorm) {
                        const double sp = srow[(long)h * n + j] * (1.0 + frow[(long)j * F + h]) + frow[(long)j * F + H + h];
                        coef = valid ? sp : 0.0;
                    }
                    pWe[(long)h * de + c] += coef * dEout[e0 + c];
                }
            }
            for (int k = 0; k < F; ++k) pg[k] += df[(long)j * F + k];
        }
        free(arow); free(srow); free(frow); free(dA); free(df); free(urow);
    }

    /* ---- column pass: dk_j, dv_j (recompute a_ij, dS'_ij over all i) ---- */
    #pragma omp parallel for schedule(dynamic, 1)
    for (long r = 0; r < rows; ++r) {
        const int b = (int)(r / n), j = (int)(r % n);
        const unsigned char *mb = M + (long)b * n;
        double f[64];
        if (!mb[j]) continue;
        for (int i = 0; i < n; ++i) {
            if (!mb[i]) continue;
            const long ri = (long)b * n + i;
            film(d, E, Wfe, g, b, i, j, f);
            const double *dep = dEout + ((ri * n) + j) * de;
            for (int h = 0; h < H; ++h) {
                const double s = raw_score(d, Q, K, b, h, i, j);
                const double sp = s * (1.0 + f[h]) + f[H + h];
                const double a = exp(sp - LSE[ri * H + h]);
                double u = 0.0;
                for (int c = 0; c < de; ++c) u += w->We[(long)h * de + c] * dep[c];
                double dov = 0.0;
                for (int t = 0; t < dh; ++t) dov += dO[ri * hd + h * dh + t] * V[r * hd + h * dh + t];
                const double dsp = unnorm ? a * (dov - Dst[ri * H + h]) + u : a * (dov + u - Dst[ri * H + h]);
                const double ds = dsp * (1.0 + f[h]);
                for (int t = 0; t < dh; ++t) {
                    dK[r * hd + h * dh + t] += ds * Q[ri * hd + h * dh + t] * rs;
                    dV[r * hd + h * dh + t] += a * dO[ri * hd + h * dh + t];
                }
            }
        }
    }

    /* ---- sums over rows, in row order ---- */
    memset(gr->Wfe, 0, sizeof(double) * de * F);
    memset(gr->We, 0, sizeof(double) * H * de);
    double *dg = (double *)calloc((size_t)B * F, sizeof(double));
    for (long r = 0; r < rows; ++r) {
        const int b = (int)(r / n);
        const double *pWfe = parts + r * part, *pWe = pWfe + (long)de * F, *pg = pWe + (long)H * de;
        for (long t = 0; t < (long)de * F; ++t) gr->Wfe[t] += pWfe[t];
        for (long t = 0; t < (long)H * de; ++t) gr->We[t] += pWe[t];
        for (int k = 0; k < F; ++k) dg[(long)b * F + k] += pg[k];
    }
    /* global FiLM term: g_b = y_b Wfy + bf */
    memset(gr->Wfy, 0, sizeof(double) * dyd * F);
    memset(gr->bf, 0, sizeof(double) * F);
    for (int b = 0; b < B; ++b) {
        for (int k = 0; k < F; ++k) {
            gr->bf[k] += dg[(long)b * F + k];
            for (int c = 0; c < dyd; ++c) gr->Wfy[(long)c * F + k] += y[(long)b * dyd + c] * dg[(long)b * F + k];
        }
        for (int c = 0; c < dyd; ++c) {
            double acc = 0.0;
            for (int k = 0; k < F; ++k) acc += dg[(long)b * F + k] * w->Wfy[(long)c * F + k];
            dy[(long)b * dyd + c] = acc;
        }
    }
    /* output projection */
    memset(gr->Wo, 0, sizeof(double) * hd * dx);
    memset(gr->bo, 0, sizeof(double) * dx);
    for (long r = 0; r < rows; ++r) {
        if (!M[r]) continue;
        for (int o = 0; o < dx; ++o) {
            gr->bo[o] += dXout[r * dx + o];
            for (int k = 0; k < hd; ++k) gr->Wo[(long)k * dx + o] += O[r * hd + k] * dXout[r * dx + o];
        }
    }
    /* node projections */
    const double *Wn[3] = {w->Wq, w->Wk, w->Wv};
    double *dWn[3] = {gr->Wq, gr->Wk, gr->Wv};
    double *dbn[3] = {gr->bq, gr->bk, gr->bv};
    const double *dN[3] = {dQ, dK, dV};
    for (int p = 0; p < 3; ++p) {
        memset(dWn[p], 0, sizeof(double) * dx * hd);
        memset(dbn[p], 0, sizeof(double) * hd);
        for (long r = 0; r < rows; ++r)
            for (int k = 0; k < hd; ++k) {
                dbn[p][k] += dN[p][r * hd + k];
                for (int c = 0; c < dx; ++c) dWn[p][(long)c * hd + k] += X[r * dx + c] * dN[p][r * hd + k];
            }
    }
    #pragma omp parallel for schedule(static)
    for (long r = 0; r < rows; ++r)
        for (int c = 0; c < dx; ++c) {
            double acc = dXout[r * dx + c];
            for (int p = 0; p < 3; ++p)
                for (int k = 0; k < hd; ++k) acc += dN[p][r * hd + k] * Wn[p][(long)c * hd + k];
            dX[r * dx + c] = acc;
        }
    /* padded / invalid pairs: dE = dE' was written by the row pass for every pair */
    if (variant == ORC_LIGHT_EDGE) memset(gr->Wfe, 0, sizeof(double) * de * F);
    free(Q); free(K); free(V); free(g); free(O); free(dO); free(dQ); free(dK); free(dV);
    free(Dst); free(LSE); free(parts); free(dg); free(Wfe0);
    return 0;
}

int orc_backward(const orc_dims *d, const double *X, const double *E, const double *y,
                 const unsigned char *M, const orc_weights *w,
                 const double *dXout, const double *dEout,
                 double *dX, double *dE, double *dy, orc_grads *gr)
{
    return orc_backward_variant(d, ORC_LAYER, X, E, y, M, w, dXout, dEout, dX, dE, dy, gr);
}
