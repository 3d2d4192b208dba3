/*
 * oal_oracle.c -- plain fp64 CPU oracle for OAL causal grouped positive-quadratic attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or calls this file:
 * only the test suite, the smoke check and the CPU-baseline leg of the benchmark use it.
 * It shares no code, header, table or helper with the CUDA library.
 *
 * Source of every formula: "OAL: 按 QK 离群贡献分组的正二次注意力核" (daiwk auto-research
 * reproduction note of arXiv 2610.13674), section 核心公式 (core formulas):
 *   eq. (2)  s_g = sum_{r in G_g} q_r k_r / sqrt(d_h),   sbar = [1, s_1, ..., s_G]
 *   eq. (3)  kappa(q, k) = eps + sbar^T L L^T sbar  (> 0)
 *   eq. (4)  H0_i = sum_{j<=i} [v_j; 1],  H1_{i,r} = sum_{j<=i} k_{j,r} [v_j; 1],
 *            H2_{i,rt} = sum_{j<=i} k_{j,r} k_{j,t} [v_j; 1]
 *   eq. (5)  u_i = a H0_i + (1/sqrt(d_h)) sum_r b_r q_{i,r} H1_{i,r}
 *                 + (1/d_h) sum_{r,t} C_rt q_{i,r} q_{i,t} H2_{i,rt},
 *            yhat_i = u_{i,1:dv} / u_{i,dv+1}
 *
 * Readings where the page is silent (each is also listed in the design notes):
 *  - a, b_r, C_rt are not printed.  Expanding eq. (3) with sbar_0 = 1 gives
 *    a = eps + M_00, b_r = 2 M_{0,g(r)}, C_rt = M_{g(r),g(t)} with M = L L^T; this is the
 *    only choice that makes eq. (5) equal eq. (3) summed over j <= i.
 *  - causality is inclusive (j <= i), as written in eq. (4).
 *  - group ids run 1..G; index 0 of sbar is the constant 1.
 *  - L is used exactly as given (M = L L^T over the leading (G+1)x(G+1) block of a
 *    (Gmax+1)x(Gmax+1) row-major array); it need not be triangular.
 *  - GQA: query head h reads key/value head floor(h * Hkv / Hq).
 *
 * Two independent evaluations are provided: the dense O(T^2) definition (eqs. 2-3, summed
 * over j <= i and normalised) and the H0/H1/H2 recurrence (eqs. 4-5), run token by token
 * with full (unpacked) d_h x d_h second-order states.  The same two evaluations exist for the
 * ungrouped Hadamard form (free a, b_r, C_rt in eq. (5)).  The gradients of the dense grouped
 * form, the contribution statistic of eq. (1), and a one-head kappa matrix complete the file.
 *
 * Layouts (all row-major, contiguous):
 *   q [B][Hq][T][dh], k [B][Hkv][T][dh], v [B][Hkv][T][dv], y [B][Hq][T][dv]
 *   group_id [Hq][dh] (values 1..G[h]), L [Hq][Gmax+1][Gmax+1], G [Hq]
 *   states H0 [B][Hkv][dv+1], H1 [B][Hkv][dh][dv+1], H2 [B][Hkv][dh][dh][dv+1]
 * Return value: 0 on success, -1 on bad arguments, -2 on allocation failure.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

/* M = L L^T over the leading (G+1)x(G+1) block; L row-major with leading dimension ld. */
static void gram_llt(const double* L, int G, int ld, double* M)
{
    for (int a = 0; a <= G; ++a)
        for (int b = 0; b <= G; ++b) {
            double acc = 0.0;
            for (int m = 0; m <= G; ++m) acc += L[a * ld + m] * L[b * ld + m];
            M[a * (G + 1) + b] = acc;
        }
}

static int check_args(int B, int Hq, int Hkv, int T, int dh, int dv, const int* gid,
                      const int* G, int Gmax)
{
    if (B < 0 || Hq <= 0 || Hkv <= 0 || T < 0 || dh <= 0 || dv <= 0 || Gmax < 1) return -1;
    if (Hq % Hkv != 0) return -1;
    for (int h = 0; h < Hq; ++h) {
        if (G[h] < 1 || G[h] > Gmax) return -1;
        for (int r = 0; r < dh; ++r)
            if (gid[h * dh + r] < 1 || gid[h * dh + r] > G[h]) return -1;
    }
    return 0;
}

/* kappa(q_i, k_j) for one head, every (i, j) pair, no causal mask: eqs. (2)-(3). */
int oal_oracle_kappa(int Tq, int Tk, int dh, const double* q, const double* k,
                     const int* gid, const double* L, int G, int Gmax, double eps,
                     double* kappa)
{
    if (G < 1 || G > Gmax || dh <= 0) return -1;
    double* M = (double*)malloc(sizeof(double) * (G + 1) * (G + 1));
    double* sbar = (double*)malloc(sizeof(double) * (G + 1));
    if (!M || !sbar) { free(M); free(sbar); return -2; }
    gram_llt(L, G, Gmax + 1, M);
    const double inv_sqrt_d = 1.0 / sqrt((double)dh);
    for (int i = 0; i < Tq; ++i)
        for (int j = 0; j < Tk; ++j) {
            sbar[0] = 1.0;
            for (int g = 1; g <= G; ++g) sbar[g] = 0.0;
            for (int r = 0; r < dh; ++r)
                sbar[gid[r]] += q[i * dh + r] * k[j * dh + r] * inv_sqrt_d;
            double quad = 0.0;
            for (int a = 0; a <= G; ++a)
                for (int b = 0; b <= G; ++b) quad += sbar[a] * M[a * (G + 1) + b] * sbar[b];
            kappa[i * Tk + j] = eps + quad;
        }
    free(M);
    free(sbar);
    return 0;
}

/* Dense causal form: yhat_i = sum_{j<=i} kappa_ij v_j / sum_{j<=i} kappa_ij.
 * den (optional, [B][Hq][T]) receives the normaliser sum_{j<=i} kappa_ij. */
int oal_oracle_dense(int B, int Hq, int Hkv, int T, int dh, int dv, const double* q,
                     const double* k, const double* v, const int* gid, const double* L,
                     const int* G, int Gmax, double eps, double* y, double* den)
{
    if (check_args(B, Hq, Hkv, T, dh, dv, gid, G, Gmax)) return -1;
    const int group = Hq / Hkv;
    int status = 0;
#pragma omp parallel for schedule(dynamic) reduction(min : status)
    for (int bh = 0; bh < B * Hq; ++bh) {
        const int b = bh / Hq, h = bh % Hq, kv = h / group;
        const double* qh = q + ((size_t)b * Hq + h) * T * dh;
        const double* kh = k + ((size_t)b * Hkv + kv) * T * dh;
        const double* vh = v + ((size_t)b * Hkv + kv) * T * dv;
        double* yh = y + ((size_t)b * Hq + h) * T * dv;
        double* kap = (double*)malloc(sizeof(double) * (T > 0 ? T : 1));
        double* num = (double*)malloc(sizeof(double) * dv);
        if (!kap || !num) { free(kap); free(num); status = -2; continue; }
        for (int i = 0; i < T; ++i) {
            /* one query row against keys 0..i */
            oal_oracle_kappa(1, i + 1, dh, qh + (size_t)i * dh, kh, gid + h * dh,
                             L + (size_t)h * (Gmax + 1) * (Gmax + 1), G[h], Gmax, eps, kap);
            double z = 0.0;
            for (int n = 0; n < dv; ++n) num[n] = 0.0;
            for (int j = 0; j <= i; ++j) {
                z += kap[j];
                for (int n = 0; n < dv; ++n) num[n] += kap[j] * vh[(size_t)j * dv + n];
            }
            for (int n = 0; n < dv; ++n) yh[(size_t)i * dv + n] = num[n] / z;
            if (den) den[((size_t)b * Hq + h) * T + i] = z;
        }
        free(kap);
        free(num);
    }
    return status;
}

/* Eqs. (4)-(5) for one (batch, query head) over T tokens, with the readout coefficients of
 * eq. (5) given explicitly: a, b [dh], C [dh][dh] (row r, column t).  h0/h1/h2 hold the state
 * of the tokens before this call and advance in place; vv and u are scratch of dv+1 doubles.
 * y receives yhat_i = u_i[:dv] / u_i[dv] by plain IEEE division, so a zero or negative
 * normaliser (possible once the coefficients are free) shows up as it falls out of the
 * arithmetic.  uo, when not NULL, receives u_i itself [T][dv+1]. */
static void recur_head(int T, int dh, int dv, const double* qh, const double* kh,
                       const double* vh, double a, const double* bco, const double* Cco,
                       double* h0, double* h1, double* h2, double* vv, double* u, double* yh,
                       double* uo)
{
    const int w = dv + 1;
    const double inv_sqrt_d = 1.0 / sqrt((double)dh), inv_d = 1.0 / (double)dh;
    for (int i = 0; i < T; ++i) {
        const double* ki = kh + (size_t)i * dh;
        const double* qi = qh + (size_t)i * dh;
        for (int n = 0; n < dv; ++n) vv[n] = vh[(size_t)i * dv + n];
        vv[dv] = 1.0;
        /* eq. (4): add token i to the prefix sums */
        for (int n = 0; n < w; ++n) h0[n] += vv[n];
        for (int r = 0; r < dh; ++r)
            for (int n = 0; n < w; ++n) h1[(size_t)r * w + n] += ki[r] * vv[n];
        for (int r = 0; r < dh; ++r)
            for (int t = 0; t < dh; ++t) {
                const double kk = ki[r] * ki[t];
                double* row = h2 + ((size_t)r * dh + t) * w;
                for (int n = 0; n < w; ++n) row[n] += kk * vv[n];
            }
        /* eq. (5): read out and normalise */
        for (int n = 0; n < w; ++n) u[n] = a * h0[n];
        for (int r = 0; r < dh; ++r) {
            const double c1 = inv_sqrt_d * bco[r] * qi[r];
            for (int n = 0; n < w; ++n) u[n] += c1 * h1[(size_t)r * w + n];
        }
        for (int r = 0; r < dh; ++r)
            for (int t = 0; t < dh; ++t) {
                const double c2 = inv_d * Cco[r * dh + t] * qi[r] * qi[t];
                const double* row = h2 + ((size_t)r * dh + t) * w;
                for (int n = 0; n < w; ++n) u[n] += c2 * row[n];
            }
        for (int n = 0; n < dv; ++n) yh[(size_t)i * dv + n] = u[n] / u[dv];
        if (uo)
            for (int n = 0; n < w; ++n) uo[(size_t)i * w + n] = u[n];
    }
}

/* Shared driver of the two recurrent entry points: per (batch, query head), load the state,
 * take the coefficients from coef_of(h), run recur_head, and let the first head of each GQA
 * group write the state out.  Each query head keeps a private copy of its key/value head's
 * state, exactly as eq. (4) defines it per head; heads of one group end with identical
 * states. */
typedef int (*coef_fn)(int h, int dh, const void* ctx, double* a, double* bco, double* Cco);

static int recurrent_driver(int B, int Hq, int Hkv, int T, int dh, int dv, const double* q,
                            const double* k, const double* v, coef_fn coef_of, const void* ctx,
                            const double* H0_in, const double* H1_in, const double* H2_in,
                            double* H0_out, double* H1_out, double* H2_out, double* y,
                            double* u_all)
{
    const int have_in = (H0_in != NULL) && (H1_in != NULL) && (H2_in != NULL);
    const int have_out = (H0_out != NULL) && (H1_out != NULL) && (H2_out != NULL);
    if (!have_in && (H0_in || H1_in || H2_in)) return -1;
    if (!have_out && (H0_out || H1_out || H2_out)) return -1;
    const int group = Hq / Hkv;
    const int w = dv + 1;
    const size_t n0 = (size_t)w, n1 = (size_t)dh * w, n2 = (size_t)dh * dh * w;
    int status = 0;
#pragma omp parallel for schedule(dynamic) reduction(min : status)
    for (int bh = 0; bh < B * Hq; ++bh) {
        const int b = bh / Hq, h = bh % Hq, kv = h / group;
        const double* qh = q + ((size_t)b * Hq + h) * T * dh;
        const double* kh = k + ((size_t)b * Hkv + kv) * T * dh;
        const double* vh = v + ((size_t)b * Hkv + kv) * T * dv;
        double* yh = y + ((size_t)b * Hq + h) * T * dv;
        double* uh = u_all ? u_all + ((size_t)b * Hq + h) * T * w : NULL;
        double* h0 = (double*)calloc(n0, sizeof(double));
        double* h1 = (double*)calloc(n1, sizeof(double));
        double* h2 = (double*)calloc(n2, sizeof(double));
        double* bco = (double*)malloc(sizeof(double) * dh);
        double* Cco = (double*)malloc(sizeof(double) * dh * dh);
        double* vv = (double*)malloc(sizeof(double) * w);
        double* u = (double*)malloc(sizeof(double) * w);
        double a = 0.0;
        if (!h0 || !h1 || !h2 || !bco || !Cco || !vv || !u || coef_of(h, dh, ctx, &a, bco, Cco)) {
            free(h0); free(h1); free(h2); free(bco); free(Cco); free(vv); free(u);
            status = -2;
            continue;
        }
        const size_t s = (size_t)b * Hkv + kv;
        if (have_in) {
            memcpy(h0, H0_in + s * n0, n0 * sizeof(double));
            memcpy(h1, H1_in + s * n1, n1 * sizeof(double));
            memcpy(h2, H2_in + s * n2, n2 * sizeof(double));
        }
        recur_head(T, dh, dv, qh, kh, vh, a, bco, Cco, h0, h1, h2, vv, u, yh, uh);
        if (have_out && (h % group) == 0) {
            memcpy(H0_out + s * n0, h0, n0 * sizeof(double));
            memcpy(H1_out + s * n1, h1, n1 * sizeof(double));
            memcpy(H2_out + s * n2, h2, n2 * sizeof(double));
        }
        free(h0); free(h1); free(h2); free(bco); free(Cco); free(vv); free(u);
    }
    return status;
}

/* Coefficients of eq. (5) from M = L L^T and the group ids (the expansion of eq. (3) with
 * sbar_0 = 1): a = eps + M_00, b_r = 2 M_{0,g(r)}, C_rt = M_{g(r),g(t)}. */
struct grouped_ctx {
    const int* gid;
    const double* L;
    const int* G;
    int Gmax;
    double eps;
};

static int grouped_coef(int h, int dh, const void* ctx_, double* a, double* bco, double* Cco)
{
    const struct grouped_ctx* c = (const struct grouped_ctx*)ctx_;
    const int Gh = c->G[h];
    double* M = (double*)malloc(sizeof(double) * (Gh + 1) * (Gh + 1));
    if (!M) return -2;
    gram_llt(c->L + (size_t)h * (c->Gmax + 1) * (c->Gmax + 1), Gh, c->Gmax + 1, M);
    const int* g = c->gid + h * dh;
    *a = c->eps + M[0];
    for (int r = 0; r < dh; ++r) bco[r] = 2.0 * M[0 * (Gh + 1) + g[r]];
    for (int r = 0; r < dh; ++r)
        for (int t = 0; t < dh; ++t) Cco[r * dh + t] = M[g[r] * (Gh + 1) + g[t]];
    free(M);
    return 0;
}

/* Recurrent form, eqs. (4)-(5), one token at a time, grouped kernel of eq. (3).
 * H*_in (all three or none) give the state of the tokens before this call; NULL starts from
 * zero (a fresh prefill).  H*_out (all three or none) receive the state after all T tokens;
 * they must not alias the inputs. */
int oal_oracle_recurrent(int B, int Hq, int Hkv, int T, int dh, int dv, const double* q,
                         const double* k, const double* v, const int* gid, const double* L,
                         const int* G, int Gmax, double eps, const double* H0_in,
                         const double* H1_in, const double* H2_in, double* H0_out,
                         double* H1_out, double* H2_out, double* y)
{
    if (check_args(B, Hq, Hkv, T, dh, dv, gid, G, Gmax)) return -1;
    const struct grouped_ctx ctx = {gid, L, G, Gmax, eps};
    return recurrent_driver(B, Hq, Hkv, T, dh, dv, q, k, v, grouped_coef, &ctx, H0_in, H1_in,
                            H2_in, H0_out, H1_out, H2_out, y, NULL);
}

/*
 * Ungrouped Hadamard form.  The abstract of arXiv 2610.13674 starts from the second-order
 * Taylor kernel and relaxes its globally shared coefficients into dimension-specific linear
 * terms and cross-dimensional quadratic terms; eq. (5) of the core-formula section is that
 * form's readout with free a, b_r, C_rt.  Summing eq. (4)'s definitions inside eq. (5) gives
 * the kernel it evaluates,
 *   kappa(q, k) = a + sum_r b_r x_r + sum_{r,t} C_rt x_r x_t,   x_r = q_r k_r / sqrt(d_h),
 * which need not be positive, so the normaliser may vanish or change sign.
 * Coefficient layouts: a [Hq], b [Hq][dh], C [Hq][dh][dh] (row r, column t).
 */
struct hadamard_ctx {
    const double* a;
    const double* b;
    const double* C;
};

static int hadamard_coef(int h, int dh, const void* ctx_, double* a, double* bco, double* Cco)
{
    const struct hadamard_ctx* c = (const struct hadamard_ctx*)ctx_;
    *a = c->a[h];
    memcpy(bco, c->b + (size_t)h * dh, sizeof(double) * dh);
    memcpy(Cco, c->C + (size_t)h * dh * dh, sizeof(double) * dh * dh);
    return 0;
}

static int check_shape(int B, int Hq, int Hkv, int T, int dh, int dv)
{
    return (B < 0 || Hq <= 0 || Hkv <= 0 || T < 0 || dh <= 0 || dv <= 0 || Hq % Hkv) ? -1 : 0;
}

/* Recurrent evaluation of the Hadamard form: eqs. (4)-(5) with the given coefficients.
 * u (optional, [B][Hq][T][dv+1]) receives the unnormalised readout. */
int oal_oracle_hadamard_recurrent(int B, int Hq, int Hkv, int T, int dh, int dv,
                                  const double* q, const double* k, const double* v,
                                  const double* a, const double* b, const double* C,
                                  const double* H0_in, const double* H1_in, const double* H2_in,
                                  double* H0_out, double* H1_out, double* H2_out, double* y,
                                  double* u)
{
    if (check_shape(B, Hq, Hkv, T, dh, dv)) return -1;
    const struct hadamard_ctx ctx = {a, b, C};
    return recurrent_driver(B, Hq, Hkv, T, dh, dv, q, k, v, hadamard_coef, &ctx, H0_in, H1_in,
                            H2_in, H0_out, H1_out, H2_out, y, u);
}

/* Dense evaluation of the Hadamard form: kappa of every causal pair (j <= i) from x = q∘k,
 * then u_i = sum_{j<=i} kappa_ij [v_j; 1] and yhat_i = u_i[:dv] / u_i[dv].
 * u (optional, [B][Hq][T][dv+1]) receives u_i. */
int oal_oracle_hadamard_dense(int B, int Hq, int Hkv, int T, int dh, int dv, const double* q,
                              const double* k, const double* v, const double* a,
                              const double* b, const double* C, double* y, double* u)
{
    if (check_shape(B, Hq, Hkv, T, dh, dv)) return -1;
    const int group = Hq / Hkv, w = dv + 1;
    const double inv_sqrt_d = 1.0 / sqrt((double)dh);
    int status = 0;
#pragma omp parallel for schedule(dynamic) reduction(min : status)
    for (int bh = 0; bh < B * Hq; ++bh) {
        const int bb = bh / Hq, h = bh % Hq, kv = h / group;
        const double* qh = q + ((size_t)bb * Hq + h) * T * dh;
        const double* kh = k + ((size_t)bb * Hkv + kv) * T * dh;
        const double* vh = v + ((size_t)bb * Hkv + kv) * T * dv;
        const double* bh_ = b + (size_t)h * dh;
        const double* Ch = C + (size_t)h * dh * dh;
        double* x = (double*)malloc(sizeof(double) * dh);
        double* acc = (double*)malloc(sizeof(double) * w);
        if (!x || !acc) { free(x); free(acc); status = -2; continue; }
        for (int i = 0; i < T; ++i) {
            for (int n = 0; n < w; ++n) acc[n] = 0.0;
            for (int j = 0; j <= i; ++j) {
                for (int r = 0; r < dh; ++r)
                    x[r] = qh[(size_t)i * dh + r] * kh[(size_t)j * dh + r] * inv_sqrt_d;
                double kap = a[h];
                for (int r = 0; r < dh; ++r) kap += bh_[r] * x[r];
                for (int r = 0; r < dh; ++r)
                    for (int t = 0; t < dh; ++t) kap += Ch[r * dh + t] * x[r] * x[t];
                for (int n = 0; n < dv; ++n) acc[n] += kap * vh[(size_t)j * dv + n];
                acc[dv] += kap;
            }
            double* yi = y + (((size_t)bb * Hq + h) * T + i) * dv;
            for (int n = 0; n < dv; ++n) yi[n] = acc[n] / acc[dv];
            if (u)
                for (int n = 0; n < w; ++n) u[(((size_t)bb * Hq + h) * T + i) * w + n] = acc[n];
        }
        free(x);
        free(acc);
    }
    return status;
}

/* Dense causal form for selected outputs only: row n is (b = rows_b[n], h = rows_h[n],
 * i = rows_i[n]); y [nrows][dv] receives yhat_i of that head.  Same definition as
 * oal_oracle_dense, one row at a time, so single rows of very long sequences stay cheap. */
int oal_oracle_dense_rows(int B, int Hq, int Hkv, int T, int dh, int dv, const double* q,
                          const double* k, const double* v, const int* gid, const double* L,
                          const int* G, int Gmax, double eps, int nrows, const int* rows_b,
                          const int* rows_h, const int* rows_i, double* y)
{
    if (check_args(B, Hq, Hkv, T, dh, dv, gid, G, Gmax)) return -1;
    for (int n = 0; n < nrows; ++n)
        if (rows_b[n] < 0 || rows_b[n] >= B || rows_h[n] < 0 || rows_h[n] >= Hq ||
            rows_i[n] < 0 || rows_i[n] >= T)
            return -1;
    const int group = Hq / Hkv;
    int status = 0;
#pragma omp parallel for schedule(dynamic) reduction(min : status)
    for (int n = 0; n < nrows; ++n) {
        const int b = rows_b[n], h = rows_h[n], i = rows_i[n], kv = h / group;
        const double* qi = q + (((size_t)b * Hq + h) * T + i) * dh;
        const double* kh = k + ((size_t)b * Hkv + kv) * T * dh;
        const double* vh = v + ((size_t)b * Hkv + kv) * T * dv;
        double* kap = (double*)malloc(sizeof(double) * (i + 1));
        double* num = (double*)calloc(dv, sizeof(double));
        if (!kap || !num) { free(kap); free(num); status = -2; continue; }
        oal_oracle_kappa(1, i + 1, dh, qi, kh, gid + h * dh,
                         L + (size_t)h * (Gmax + 1) * (Gmax + 1), G[h], Gmax, eps, kap);
        double z = 0.0;
        for (int j = 0; j <= i; ++j) {
            z += kap[j];
            for (int c = 0; c < dv; ++c) num[c] += kap[j] * vh[(size_t)j * dv + c];
        }
        for (int c = 0; c < dv; ++c) y[(size_t)n * dv + c] = num[c] / z;
        free(kap);
        free(num);
    }
    return status;
}

/*
 * Contribution statistic, eq. (1) of the same section:
 *   chi_{p,r} = (1/|Omega_p|) sum over causal pairs (i, j), j <= i, of |q_{p,i,r} k_{p,j,r}| / sqrt(d_h)
 * for prompt p = (b, query head h); |Omega_p| = T (T + 1) / 2, the number of causal pairs
 * (the page does not define Omega; this is the reading).  chi_r of eq. (1) is the mean of
 * chi_{p,r} over prompts.  Plain double loop over every causal pair, O(T^2 dh) per head.
 * Layouts: q [B][Hq][T][dh], k [B][Hkv][T][dh], chi [B][Hq][dh].
 */
int oal_oracle_chi(int B, int Hq, int Hkv, int T, int dh, const double* q, const double* k,
                   double* chi)
{
    if (B < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv || T < 1 || dh < 1) return -1;
    const int group = Hq / Hkv;
    const double pairs = 0.5 * (double)T * (double)(T + 1), rs = 1.0 / sqrt((double)dh);
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < Hq; ++h) {
            const double* qh = q + ((size_t)b * Hq + h) * T * dh;
            const double* kh = k + ((size_t)b * Hkv + h / group) * T * dh;
            for (int r = 0; r < dh; ++r) {
                double acc = 0.0;
                for (int i = 0; i < T; ++i)
                    for (int j = 0; j <= i; ++j)
                        acc += fabs(qh[(size_t)i * dh + r] * kh[(size_t)j * dh + r] * rs);
                chi[((size_t)b * Hq + h) * dh + r] = acc / pairs;
            }
        }
    return 0;
}

/* kappa of one pair (eqs. (2)-(3)) for the backward pass; also leaves sbar and M sbar. */
static double pair_kappa(const double* qi, const double* kj, const int* g, int dh, int gs,
                         const double* M, double eps, double inv_sqrt_d, double* sbar,
                         double* Ms)
{
    sbar[0] = 1.0;
    for (int c = 1; c < gs; ++c) sbar[c] = 0.0;
    for (int r = 0; r < dh; ++r) sbar[g[r]] += qi[r] * kj[r] * inv_sqrt_d;
    double kap = eps;
    for (int c = 0; c < gs; ++c) {
        Ms[c] = 0.0;
        for (int e = 0; e < gs; ++e) Ms[c] += M[c * gs + e] * sbar[e];
        kap += sbar[c] * Ms[c];
    }
    return kap;
}

/*
 * Gradients of the dense causal form of the grouped kernel (eqs. (2)-(3), summed over
 * j <= i and normalised), for the joint training of the kernel coefficients with the model
 * that the page's pipeline describes (LoRA and kernel parameters trained together).
 * Given dy = dLoss/dyhat [B][Hq][T][dv], with
 *   D_i = sum_{j<=i} kappa_ij,  yhat_i = sum_{j<=i} kappa_ij v_j / D_i,
 * the chain rule gives, per causal pair,
 *   dkappa_ij = dy_i . (v_j - yhat_i) / D_i,     dv_j += kappa_ij dy_i / D_i,
 *   dkappa/dsbar = 2 M sbar (M = L L^T symmetric), ds_g/dq_ir = [g(r) = g] k_jr / sqrt(d_h),
 *   dM += dkappa_ij sbar sbar^T,  deps += dkappa_ij,
 * and dL = (dM + dM^T) L.  Outputs: dq [B][Hq][T][dh], dk [B][Hkv][T][dh] and
 * dv [B][Hkv][T][dv] (summed over the query heads of each GQA group), dL [Hq][Gmax+1][Gmax+1]
 * (zero outside each head's leading (G+1)x(G+1) block), deps (one scalar: eps is shared).
 * Two passes over the pairs of each row: the first forms D_i and yhat_i, the second the
 * gradients.  Parallel over (batch, key/value head); the per-(batch, head) dM and deps are
 * reduced in a fixed order afterwards, so the result does not depend on the thread count.
 */
int oal_oracle_dense_backward(int B, int Hq, int Hkv, int T, int dh, int dv, const double* q,
                              const double* k, const double* v, const int* gid, const double* L,
                              const int* G, int Gmax, double eps, const double* dy, double* dq,
                              double* dk, double* dvv, double* dL, double* deps)
{
    if (check_args(B, Hq, Hkv, T, dh, dv, gid, G, Gmax)) return -1;
    const int group = Hq / Hkv, g1 = Gmax + 1;
    const double inv_sqrt_d = 1.0 / sqrt((double)dh);
    memset(dq, 0, sizeof(double) * (size_t)B * Hq * T * dh);
    memset(dk, 0, sizeof(double) * (size_t)B * Hkv * T * dh);
    memset(dvv, 0, sizeof(double) * (size_t)B * Hkv * T * dv);
    memset(dL, 0, sizeof(double) * (size_t)Hq * g1 * g1);
    double* dM_all = (double*)calloc((size_t)B * Hq * g1 * g1, sizeof(double));
    double* de_all = (double*)calloc((size_t)B * Hq + 1, sizeof(double));
    if (!dM_all || !de_all) { free(dM_all); free(de_all); return -2; }
    int status = 0;
#pragma omp parallel for schedule(dynamic) reduction(min : status)
    for (int bkv = 0; bkv < B * Hkv; ++bkv) {
        const int b = bkv / Hkv, kv = bkv % Hkv;
        const double* kh = k + (size_t)bkv * T * dh;
        const double* vh = v + (size_t)bkv * T * dv;
        double* dkh = dk + (size_t)bkv * T * dh;
        double* dvh = dvv + (size_t)bkv * T * dv;
        double* M = (double*)malloc(sizeof(double) * g1 * g1);
        double* sbar = (double*)malloc(sizeof(double) * g1);
        double* Ms = (double*)malloc(sizeof(double) * g1);
        double* yi = (double*)malloc(sizeof(double) * dv);
        if (!M || !sbar || !Ms || !yi) {
            free(M); free(sbar); free(Ms); free(yi);
            status = -2;
            continue;
        }
        for (int h = kv * group; h < (kv + 1) * group; ++h) {
            const int gs = G[h] + 1;
            const int* g = gid + h * dh;
            gram_llt(L + (size_t)h * g1 * g1, G[h], g1, M);
            const double* qh = q + ((size_t)b * Hq + h) * T * dh;
            const double* dyh = dy + ((size_t)b * Hq + h) * T * dv;
            double* dqh = dq + ((size_t)b * Hq + h) * T * dh;
            double* dM = dM_all + ((size_t)b * Hq + h) * g1 * g1;
            double de = 0.0;
            for (int i = 0; i < T; ++i) {
                const double* qi = qh + (size_t)i * dh;
                const double* gi = dyh + (size_t)i * dv;
                double* dqi = dqh + (size_t)i * dh;
                /* pass 1: normaliser and output of row i */
                double D = 0.0;
                for (int n = 0; n < dv; ++n) yi[n] = 0.0;
                for (int j = 0; j <= i; ++j) {
                    const double kap = pair_kappa(qi, kh + (size_t)j * dh, g, dh, gs, M, eps,
                                                  inv_sqrt_d, sbar, Ms);
                    D += kap;
                    for (int n = 0; n < dv; ++n) yi[n] += kap * vh[(size_t)j * dv + n];
                }
                for (int n = 0; n < dv; ++n) yi[n] /= D;
                /* pass 2: gradients through every pair of row i */
                for (int j = 0; j <= i; ++j) {
                    const double* kj = kh + (size_t)j * dh;
                    const double kap = pair_kappa(qi, kj, g, dh, gs, M, eps, inv_sqrt_d, sbar,
                                                  Ms);
                    double dkap = 0.0;
                    for (int n = 0; n < dv; ++n) {
                        dkap += gi[n] * (vh[(size_t)j * dv + n] - yi[n]);
                        dvh[(size_t)j * dv + n] += kap * gi[n] / D;
                    }
                    dkap /= D;
                    for (int r = 0; r < dh; ++r) {
                        const double wr = dkap * 2.0 * Ms[g[r]] * inv_sqrt_d;
                        dqi[r] += wr * kj[r];
                        dkh[(size_t)j * dh + r] += wr * qi[r];
                    }
                    for (int c = 0; c < gs; ++c)
                        for (int e = 0; e < gs; ++e) dM[c * g1 + e] += dkap * sbar[c] * sbar[e];
                    de += dkap;
                }
            }
            de_all[(size_t)b * Hq + h] = de;
        }
        free(M); free(sbar); free(Ms); free(yi);
    }
    if (status == 0) {
        double acc = 0.0;
        for (int h = 0; h < Hq; ++h) {
            const int gs = G[h] + 1;
            const double* Lh = L + (size_t)h * g1 * g1;
            double* dLh = dL + (size_t)h * g1 * g1;
            for (int b = 0; b < B; ++b) {
                const double* dM = dM_all + ((size_t)b * Hq + h) * g1 * g1;
                /* dL_am += sum_c (dM_ac + dM_ca) L_cm */
                for (int a = 0; a < gs; ++a)
                    for (int m = 0; m < gs; ++m) {
                        double s = 0.0;
                        for (int c = 0; c < gs; ++c)
                            s += (dM[a * g1 + c] + dM[c * g1 + a]) * Lh[c * g1 + m];
                        dLh[a * g1 + m] += s;
                    }
                acc += de_all[(size_t)b * Hq + h];
            }
        }
        *deps = acc;
    }
    free(dM_all);
    free(de_all);
    return status;
}
