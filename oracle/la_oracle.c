/*
 * la_oracle.c -- plain, slow, fp64 CPU oracle for causal linear attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark may load this library.  It shares no code,
 * header, table or helper with the CUDA path, and it includes nothing from it.
 *
 * What it computes (all arithmetic in double precision, inputs given as
 * doubles, layouts row-major [B,H,N,D]; every (b,h) slice is independent):
 *
 *   phi      -- the feature maps.
 *               elu(x)+1 ("Transformers are RNNs", the linear-attention
 *               feature map it proposes; alpha = 1): x+1 for x>0, exp(x) else.
 *               BASED second-order Taylor map ("Simple linear attention
 *               language models balance the recall-throughput tradeoff",
 *               Knowl 3, the equation phi(q).phi(k) = 1 + q.k + (q.k)^2/2):
 *               [1 | x/d'^(1/4) | x_a x_b / (sqrt(2) sqrt(d'))], the second
 *               block row-major in (a, b), so 1 + d' + d'^2 features.
 *               The same map with each symmetric pair of second-order
 *               features folded into one (the count behind the BASED page's
 *               state-size expression, Knowl 7: 1 + 3d'/2 + d'^2/2 features):
 *               [1 | x/d'^(1/4) | x_a^2 / (sqrt(2) sqrt(d')) for each a |
 *               x_a x_b / sqrt(d') for a < b, row-major], so that
 *               phi_sym(q).phi_sym(k) = phi(q).phi(k) term by term.
 *   forward_brute      -- the masked parallel form, Knowl 3 eq. for y_i:
 *               a_ij = phi(q_i).phi(k_j) for j <= i,
 *               y_i  = sum_j a_ij v_j / sum_j a_ij,           O(N^2 F).
 *   forward_rows       -- the same, for selected positions of one slice.
 *   forward_recurrent  -- the recurrent form, Knowl 3 eqs. for s_i, z_i, y_i:
 *               s_i = s_{i-1} + phi(k_i)^T v_i, z_i = z_{i-1} + phi(k_i)^T,
 *               y_i = phi(q_i) s_i / phi(q_i) z_i   (state includes token i),
 *               optionally from a given state, returning the final state
 *               (Knowl 5: the prefill may write its final state for decode).
 *   forward_recurrent_decay / forward_brute_decay / decode_step_decay --
 *               the gated form: a scalar forget gate a_i = exp(g_i) per
 *               token multiplies the state before token i is added,
 *               s_i = a_i s_{i-1} + phi(k_i)^T v_i, z_i = a_i z_{i-1} + phi(k_i)^T
 *               (the gated update C_t = F_t C_{t-1} + k_t v_t^T of the reader
 *               comment on linear RNNs, and the scalar-times-identity state
 *               matrix a_t I of the comment on the state-space duality, on the
 *               'Transformers are RNNs' discussion page; the input-dependent
 *               decay of the BASED page, Knowl 10).  The pages give no
 *               normaliser for it; the same gate decays z, so y_i stays a
 *               weighted mean of the v_j with weights
 *               (prod_{l=j+1..i} a_l) phi(q_i).phi(k_j).
 *   swa_forward        -- causal sliding-window softmax attention (Knowl 4):
 *               query i attends to keys max(0,i-w+1)..i with softmax weights
 *               of scale q_i.k_j, and the log-sum-exp of those scores.
 *   decode_step        -- one step of that recurrence on a given state,
 *               output taken from the updated state (Knowl 5, recurrent
 *               generation kernel description).
 *   backward_brute / backward_recurrent -- gradients of y with respect to
 *               q, k, v for an upstream gradient dO.  The pages give no
 *               backward pass; it is the derivative of the Knowl 3 parallel
 *               form, written out by hand:
 *                 g_i    = dO_i / den_i,   dden_i = -g_i . y_i,
 *                 da_ij  = g_i . v_j + dden_i                (j <= i),
 *                 dv_j   = sum_{i>=j} a_ij g_i,
 *                 dphiq_i = sum_{j<=i} da_ij phi(k_j),
 *                 dphik_j = sum_{i>=j} da_ij phi(q_i),
 *               then dq = J_phi(q)^T dphiq and dk = J_phi(k)^T dphik.
 *               The recurrent version scans s,z forward for dq and
 *               R_j = sum_{i>=j} phi(q_i) g_i^T, r_j = sum_{i>=j} phi(q_i) dden_i
 *               backward for dk, dv.
 *   backward_brute_decay / backward_recurrent_decay -- the same for the
 *               gated form, with w_ij = (prod_{l=j+1..i} a_l) a_ij in place of
 *               a_ij, and dL/dg_l for the log gates.  The brute version sums
 *               dL/dw_ij w_ij over the pairs j < l <= i that g_l scales.  The
 *               recurrent version scans the gated s, z forward and the gated
 *               R_j = phi(q_j) g_j^T + a_{j+1} R_{j+1} backward; with
 *               B_m = g_1 + .. + g_m, w_ij = exp(B_i - B_j) a_ij, so
 *               dL/dB_m = phi(q_m).dphiq_m - phi(k_m).dphik_m (the row sum of
 *               w dL/dw minus the column sum) and dL/dg_l = sum_{m>=l} dL/dB_m.
 *
 * Parallelism: OpenMP over (b,h) slices only; each slice is computed in the
 * plain order above.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_ELU1 0
#define ORC_TAYLOR2 1
#define ORC_TAYLOR2_SYM 2

int orc_feature_dim(int fmap, int dqk)
{
    if (fmap == ORC_ELU1) return dqk;
    if (fmap == ORC_TAYLOR2) return 1 + dqk + dqk * dqk;
    if (fmap == ORC_TAYLOR2_SYM) return 1 + dqk + dqk + dqk * (dqk - 1) / 2;
    return -1;
}

/* phi(x) for one vector x[dqk] -> out[F]. */
void orc_phi(int fmap, int dqk, const double *x, double *out)
{
    if (fmap == ORC_ELU1) {
        for (int a = 0; a < dqk; ++a)
            out[a] = x[a] > 0.0 ? x[a] + 1.0 : exp(x[a]);
        return;
    }
    /* Taylor: constant, first-order coordinates, then second-order products. */
    const double c1 = pow((double)dqk, 0.25);            /* d'^(1/4)          */
    const double c2 = sqrt(2.0) * sqrt((double)dqk);     /* sqrt(2) sqrt(d')  */
    out[0] = 1.0;
    for (int a = 0; a < dqk; ++a) out[1 + a] = x[a] / c1;
    if (fmap == ORC_TAYLOR2_SYM) {
        /* squares, then each unordered pair a < b once; the pair feature
           stands for the two equal features (a,b), (b,a) of the full map,
           so it carries sqrt(2) times their value: sqrt(2)/c2 = 1/sqrt(d'). */
        for (int a = 0; a < dqk; ++a) out[1 + dqk + a] = x[a] * x[a] / c2;
        int f = 1 + 2 * dqk;
        for (int a = 0; a < dqk; ++a)
            for (int b = a + 1; b < dqk; ++b) out[f++] = x[a] * x[b] / sqrt((double)dqk);
        return;
    }
    for (int a = 0; a < dqk; ++a)
        for (int b = 0; b < dqk; ++b)
            out[1 + dqk + a * dqk + b] = x[a] * x[b] / c2;
}

/* dx = J_phi(x)^T dphi  (vector-Jacobian product of the feature map). */
void orc_phi_vjp(int fmap, int dqk, const double *x, const double *dphi, double *dx)
{
    if (fmap == ORC_ELU1) {
        for (int a = 0; a < dqk; ++a)
            dx[a] = dphi[a] * (x[a] > 0.0 ? 1.0 : exp(x[a]));
        return;
    }
    const double c1 = pow((double)dqk, 0.25);
    const double c2 = sqrt(2.0) * sqrt((double)dqk);
    if (fmap == ORC_TAYLOR2_SYM) {
        /* d/dx_c of x_c^2/c2 is 2 x_c/c2; of x_a x_b/sqrt(d') it is
           x_b/sqrt(d') for c = a and x_a/sqrt(d') for c = b. */
        for (int c = 0; c < dqk; ++c) dx[c] = dphi[1 + c] / c1 + dphi[1 + dqk + c] * 2.0 * x[c] / c2;
        int f = 1 + 2 * dqk;
        for (int a = 0; a < dqk; ++a)
            for (int b = a + 1; b < dqk; ++b, ++f) {
                dx[a] += dphi[f] * x[b] / sqrt((double)dqk);
                dx[b] += dphi[f] * x[a] / sqrt((double)dqk);
            }
        return;
    }
    /* phi_{1+a} = x_a / c1;  phi_{1+d'+a d'+b} = x_a x_b / c2. */
    for (int c = 0; c < dqk; ++c) {
        double s = dphi[1 + c] / c1;
        for (int b = 0; b < dqk; ++b) {
            const double d_cb = dphi[1 + dqk + c * dqk + b];  /* d/dx_c of x_c x_b */
            const double d_bc = dphi[1 + dqk + b * dqk + c];  /* d/dx_c of x_b x_c */
            s += (d_cb + d_bc) * x[b] / c2;
        }
        dx[c] = s;
    }
}

static double dot(const double *a, const double *b, int n)
{
    double s = 0.0;
    for (int i = 0; i < n; ++i) s += a[i] * b[i];
    return s;
}

/* Feature vectors of all N rows of one slice: out[N][F]. */
static double *phi_rows(int fmap, int N, int dqk, const double *x)
{
    const int F = orc_feature_dim(fmap, dqk);
    double *out = (double *)malloc(sizeof(double) * (size_t)N * (size_t)F);
    for (int i = 0; i < N; ++i) orc_phi(fmap, dqk, x + (size_t)i * dqk, out + (size_t)i * F);
    return out;
}

/* ---------------------------------------------------------------- forward */

/* Masked parallel form for one slice at the listed positions. */
static void brute_slice_rows(int fmap, int N, int dqk, int dv,
                             const double *q, const double *k, const double *v,
                             const double *phik, const int64_t *rows, int nrows,
                             double *o, double *den)
{
    const int F = orc_feature_dim(fmap, dqk);
    double *phiq = (double *)malloc(sizeof(double) * (size_t)F);
    double *num = (double *)malloc(sizeof(double) * (size_t)dv);
    for (int r = 0; r < nrows; ++r) {
        const int64_t i = rows[r];
        orc_phi(fmap, dqk, q + (size_t)i * dqk, phiq);
        double d = 0.0;
        for (int c = 0; c < dv; ++c) num[c] = 0.0;
        for (int64_t j = 0; j <= i; ++j) {
            const double a = dot(phiq, phik + (size_t)j * F, F);
            d += a;
            for (int c = 0; c < dv; ++c) num[c] += a * v[(size_t)j * dv + c];
        }
        for (int c = 0; c < dv; ++c) o[(size_t)r * dv + c] = num[c] / d;
        if (den) den[r] = d;
    }
    (void)N;
    free(phiq);
    free(num);
}

void orc_forward_brute(int fmap, int B, int H, int N, int dqk, int dv,
                       const double *q, const double *k, const double *v,
                       double *o, double *den)
{
    const int BH = B * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < BH; ++bh) {
        const double *qs = q + (size_t)bh * N * dqk;
        const double *ks = k + (size_t)bh * N * dqk;
        const double *vs = v + (size_t)bh * N * dv;
        double *phik = phi_rows(fmap, N, dqk, ks);
        int64_t *rows = (int64_t *)malloc(sizeof(int64_t) * (size_t)N);
        for (int i = 0; i < N; ++i) rows[i] = i;
        brute_slice_rows(fmap, N, dqk, dv, qs, ks, vs, phik, rows, N,
                         o + (size_t)bh * N * dv, den ? den + (size_t)bh * N : NULL);
        free(rows);
        free(phik);
    }
}

/* Brute force at selected positions of slice bh (for sampled checks of
 * large workloads).  o_rows[nrows][dv], den_rows[nrows] (nullable). */
void orc_forward_rows(int fmap, int N, int dqk, int dv,
                      const double *q, const double *k, const double *v,
                      const int64_t *rows, int nrows, double *o_rows, double *den_rows)
{
    /* Only phi(k_j) for j <= max row is needed. */
    int64_t last = 0;
    for (int r = 0; r < nrows; ++r) if (rows[r] > last) last = rows[r];
    double *phik = phi_rows(fmap, (int)(last + 1), dqk, k);
    brute_slice_rows(fmap, N, dqk, dv, q, k, v, phik, rows, nrows, o_rows, den_rows);
    free(phik);
}

/* The recurrence over one slice.  g (nullable) holds a log-decay per token:
 * with it the state is first multiplied by a_i = exp(g_i) (the gated form). */
static void recurrent_slice(int fmap, int N, int dqk, int dv,
                            const double *q, const double *k, const double *v, const double *g,
                            double *s, double *z, double *o, double *den)
{
    const int F = orc_feature_dim(fmap, dqk);
    double *phiq = (double *)malloc(sizeof(double) * (size_t)F);
    double *phik = (double *)malloc(sizeof(double) * (size_t)F);
    for (int i = 0; i < N; ++i) {
        orc_phi(fmap, dqk, q + (size_t)i * dqk, phiq);
        orc_phi(fmap, dqk, k + (size_t)i * dqk, phik);
        const double *vi = v + (size_t)i * dv;
        if (g) {
            /* gated: s_{i-1} <- a_i s_{i-1}, z_{i-1} <- a_i z_{i-1} */
            const double a = exp(g[i]);
            for (int f = 0; f < F; ++f) {
                for (int c = 0; c < dv; ++c) s[(size_t)f * dv + c] *= a;
                z[f] *= a;
            }
        }
        /* s_i = s_{i-1} + phi(k_i)^T v_i ; z_i = z_{i-1} + phi(k_i)^T */
        for (int f = 0; f < F; ++f) {
            for (int c = 0; c < dv; ++c) s[(size_t)f * dv + c] += phik[f] * vi[c];
            z[f] += phik[f];
        }
        /* y_i = phi(q_i) s_i / phi(q_i) z_i */
        const double d = dot(phiq, z, F);
        for (int c = 0; c < dv; ++c) {
            double n = 0.0;
            for (int f = 0; f < F; ++f) n += phiq[f] * s[(size_t)f * dv + c];
            o[(size_t)i * dv + c] = n / d;
        }
        if (den) den[i] = d;
    }
    free(phiq);
    free(phik);
}

/* Recurrent form over all slices.  s0/z0 (nullable) give a starting state
 * [B,H,F,dv] / [B,H,F]; s_out/z_out (nullable) receive the final state. */
void orc_forward_recurrent_decay(int fmap, int B, int H, int N, int dqk, int dv,
                                 const double *q, const double *k, const double *v, const double *g,
                                 const double *s0, const double *z0,
                                 double *o, double *den, double *s_out, double *z_out);

void orc_forward_recurrent(int fmap, int B, int H, int N, int dqk, int dv,
                           const double *q, const double *k, const double *v,
                           const double *s0, const double *z0,
                           double *o, double *den, double *s_out, double *z_out)
{
    orc_forward_recurrent_decay(fmap, B, H, N, dqk, dv, q, k, v, NULL, s0, z0, o, den, s_out, z_out);
}

/* The same with a log-decay per token, g [B,H,N] (nullable: no decay). */
void orc_forward_recurrent_decay(int fmap, int B, int H, int N, int dqk, int dv,
                                 const double *q, const double *k, const double *v, const double *g,
                                 const double *s0, const double *z0,
                                 double *o, double *den, double *s_out, double *z_out)
{
    const int BH = B * H;
    const int F = orc_feature_dim(fmap, dqk);
#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < BH; ++bh) {
        double *s = (double *)calloc((size_t)F * dv, sizeof(double));
        double *z = (double *)calloc((size_t)F, sizeof(double));
        if (s0) memcpy(s, s0 + (size_t)bh * F * dv, sizeof(double) * (size_t)F * dv);
        if (z0) memcpy(z, z0 + (size_t)bh * F, sizeof(double) * (size_t)F);
        recurrent_slice(fmap, N, dqk, dv,
                        q + (size_t)bh * N * dqk, k + (size_t)bh * N * dqk, v + (size_t)bh * N * dv,
                        g ? g + (size_t)bh * N : NULL,
                        s, z, o + (size_t)bh * N * dv, den ? den + (size_t)bh * N : NULL);
        if (s_out) memcpy(s_out + (size_t)bh * F * dv, s, sizeof(double) * (size_t)F * dv);
        if (z_out) memcpy(z_out + (size_t)bh * F, z, sizeof(double) * (size_t)F);
        free(s);
        free(z);
    }
}

/* One decode step for BH independent heads: q,k [BH,dqk], v [BH,dv];
 * s [BH,F,dv], z [BH,F] updated in place; y [BH,dv] from the updated state. */
void orc_decode_step_decay(int fmap, int BH, int dqk, int dv,
                           const double *q, const double *k, const double *v, const double *g,
                           double *s, double *z, double *y)
{
    const int F = orc_feature_dim(fmap, dqk);
#pragma omp parallel for schedule(static)
    for (int bh = 0; bh < BH; ++bh)
        recurrent_slice(fmap, 1, dqk, dv, q + (size_t)bh * dqk, k + (size_t)bh * dqk,
                        v + (size_t)bh * dv, g ? g + bh : NULL, s + (size_t)bh * F * dv, z + (size_t)bh * F,
                        y + (size_t)bh * dv, NULL);
}

void orc_decode_step(int fmap, int BH, int dqk, int dv,
                     const double *q, const double *k, const double *v,
                     double *s, double *z, double *y)
{
    orc_decode_step_decay(fmap, BH, dqk, dv, q, k, v, NULL, s, z, y);
}

/* Gated masked form by brute force, one slice per (b,h):
 *   w_ij = (prod_{l=j+1..i} exp(g_l)) phi(q_i).phi(k_j)   (j <= i),
 *   y_i  = sum_j w_ij v_j / sum_j w_ij.
 * The product is taken factor by factor, walking j down from i. */
void orc_forward_brute_decay(int fmap, int B, int H, int N, int dqk, int dv,
                             const double *q, const double *k, const double *v, const double *g,
                             double *o, double *den)
{
    const int BH = B * H;
    const int F = orc_feature_dim(fmap, dqk);
#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < BH; ++bh) {
        const double *qs = q + (size_t)bh * N * dqk, *vs = v + (size_t)bh * N * dv, *gs = g + (size_t)bh * N;
        double *phik = phi_rows(fmap, N, dqk, k + (size_t)bh * N * dqk);
        double *phiq = (double *)malloc(sizeof(double) * (size_t)F);
        double *num = (double *)malloc(sizeof(double) * (size_t)dv);
        for (int i = 0; i < N; ++i) {
            orc_phi(fmap, dqk, qs + (size_t)i * dqk, phiq);
            double d = 0.0, prod = 1.0;
            for (int c = 0; c < dv; ++c) num[c] = 0.0;
            for (int j = i; j >= 0; --j) {
                if (j < i) prod *= exp(gs[j + 1]);
                const double w = prod * dot(phiq, phik + (size_t)j * F, F);
                d += w;
                for (int c = 0; c < dv; ++c) num[c] += w * vs[(size_t)j * dv + c];
            }
            for (int c = 0; c < dv; ++c) o[((size_t)bh * N + i) * dv + c] = num[c] / d;
            if (den) den[(size_t)bh * N + i] = d;
        }
        free(phik);
        free(phiq);
        free(num);
    }
}

/* --------------------------------------------------------------- backward */

void orc_backward_brute(int fmap, int B, int H, int N, int dqk, int dv,
                        const double *q, const double *k, const double *v,
                        const double *dout, double *dq, double *dk, double *dvv)
{
    const int BH = B * H;
    const int F = orc_feature_dim(fmap, dqk);
#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < BH; ++bh) {
        const double *qs = q + (size_t)bh * N * dqk;
        const double *ks = k + (size_t)bh * N * dqk;
        const double *vs = v + (size_t)bh * N * dv;
        const double *dos = dout + (size_t)bh * N * dv;
        double *dqs = dq + (size_t)bh * N * dqk;
        double *dks = dk + (size_t)bh * N * dqk;
        double *dvs = dvv + (size_t)bh * N * dv;
        double *phiq = phi_rows(fmap, N, dqk, qs);
        double *phik = phi_rows(fmap, N, dqk, ks);
        double *A = (double *)calloc((size_t)N * N, sizeof(double));   /* a_ij, j<=i */
        double *dA = (double *)calloc((size_t)N * N, sizeof(double));
        double *g = (double *)malloc(sizeof(double) * (size_t)N * dv);
        double *dphiq = (double *)calloc((size_t)N * F, sizeof(double));
        double *dphik = (double *)calloc((size_t)N * F, sizeof(double));
        for (int i = 0; i < N; ++i) {
            double d = 0.0;
            for (int j = 0; j <= i; ++j) {
                A[(size_t)i * N + j] = dot(phiq + (size_t)i * F, phik + (size_t)j * F, F);
                d += A[(size_t)i * N + j];
            }
            /* y_i, then g_i = dO_i / den_i and dden_i = -g_i . y_i */
            double gy = 0.0;
            for (int c = 0; c < dv; ++c) {
                double n = 0.0;
                for (int j = 0; j <= i; ++j) n += A[(size_t)i * N + j] * vs[(size_t)j * dv + c];
                const double y = n / d;
                g[(size_t)i * dv + c] = dos[(size_t)i * dv + c] / d;
                gy += g[(size_t)i * dv + c] * y;
            }
            const double dden = -gy;
            for (int j = 0; j <= i; ++j)
                dA[(size_t)i * N + j] = dot(g + (size_t)i * dv, vs + (size_t)j * dv, dv) + dden;
        }
        for (int j = 0; j < N; ++j)
            for (int c = 0; c < dv; ++c) {
                double s = 0.0;
                for (int i = j; i < N; ++i) s += A[(size_t)i * N + j] * g[(size_t)i * dv + c];
                dvs[(size_t)j * dv + c] = s;
            }
        for (int i = 0; i < N; ++i)
            for (int j = 0; j <= i; ++j) {
                const double da = dA[(size_t)i * N + j];
                for (int f = 0; f < F; ++f) {
                    dphiq[(size_t)i * F + f] += da * phik[(size_t)j * F + f];
                    dphik[(size_t)j * F + f] += da * phiq[(size_t)i * F + f];
                }
            }
        for (int i = 0; i < N; ++i) {
            orc_phi_vjp(fmap, dqk, qs + (size_t)i * dqk, dphiq + (size_t)i * F, dqs + (size_t)i * dqk);
            orc_phi_vjp(fmap, dqk, ks + (size_t)i * dqk, dphik + (size_t)i * F, dks + (size_t)i * dqk);
        }
        free(phiq); free(phik); free(A); free(dA); free(g); free(dphiq); free(dphik);
    }
}

void orc_backward_recurrent(int fmap, int B, int H, int N, int dqk, int dv,
                            const double *q, const double *k, const double *v,
                            const double *dout, double *dq, double *dk, double *dvv)
{
    const int BH = B * H;
    const int F = orc_feature_dim(fmap, dqk);
#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < BH; ++bh) {
        const double *qs = q + (size_t)bh * N * dqk;
        const double *ks = k + (size_t)bh * N * dqk;
        const double *vs = v + (size_t)bh * N * dv;
        const double *dos = dout + (size_t)bh * N * dv;
        double *dqs = dq + (size_t)bh * N * dqk;
        double *dks = dk + (size_t)bh * N * dqk;
        double *dvs = dvv + (size_t)bh * N * dv;
        double *s = (double *)calloc((size_t)F * dv, sizeof(double));
        double *z = (double *)calloc((size_t)F, sizeof(double));
        double *g = (double *)malloc(sizeof(double) * (size_t)N * dv);
        double *dden = (double *)malloc(sizeof(double) * (size_t)N);
        double *phiq = (double *)malloc(sizeof(double) * (size_t)F);
        double *phik = (double *)malloc(sizeof(double) * (size_t)F);
        double *dphi = (double *)malloc(sizeof(double) * (size_t)F);
        /* Forward-order scan: s_i, z_i include token i. */
        for (int i = 0; i < N; ++i) {
            orc_phi(fmap, dqk, qs + (size_t)i * dqk, phiq);
            orc_phi(fmap, dqk, ks + (size_t)i * dqk, phik);
            for (int f = 0; f < F; ++f) {
                for (int c = 0; c < dv; ++c) s[(size_t)f * dv + c] += phik[f] * vs[(size_t)i * dv + c];
                z[f] += phik[f];
            }
            const double d = dot(phiq, z, F);
            double gy = 0.0;
            for (int c = 0; c < dv; ++c) {
                double n = 0.0;
                for (int f = 0; f < F; ++f) n += phiq[f] * s[(size_t)f * dv + c];
                g[(size_t)i * dv + c] = dos[(size_t)i * dv + c] / d;
                gy += g[(size_t)i * dv + c] * (n / d);
            }
            dden[i] = -gy;
            /* dphi(q_i) = s_i g_i + z_i dden_i */
            for (int f = 0; f < F; ++f)
                dphi[f] = dot(s + (size_t)f * dv, g + (size_t)i * dv, dv) + z[f] * dden[i];
            orc_phi_vjp(fmap, dqk, qs + (size_t)i * dqk, dphi, dqs + (size_t)i * dqk);
        }
        /* Reverse-order scan: R_j = sum_{i>=j} phi(q_i) g_i^T (reusing s), r_j (reusing z). */
        memset(s, 0, sizeof(double) * (size_t)F * dv);
        memset(z, 0, sizeof(double) * (size_t)F);
        for (int j = N - 1; j >= 0; --j) {
            orc_phi(fmap, dqk, qs + (size_t)j * dqk, phiq);
            orc_phi(fmap, dqk, ks + (size_t)j * dqk, phik);
            for (int f = 0; f < F; ++f) {
                for (int c = 0; c < dv; ++c) s[(size_t)f * dv + c] += phiq[f] * g[(size_t)j * dv + c];
                z[f] += phiq[f] * dden[j];
            }
            /* dphi(k_j) = R_j v_j + r_j ; dv_j = R_j^T phi(k_j) */
            for (int f = 0; f < F; ++f)
                dphi[f] = dot(s + (size_t)f * dv, vs + (size_t)j * dv, dv) + z[f];
            orc_phi_vjp(fmap, dqk, ks + (size_t)j * dqk, dphi, dks + (size_t)j * dqk);
            for (int c = 0; c < dv; ++c) {
                double a = 0.0;
                for (int f = 0; f < F; ++f) a += s[(size_t)f * dv + c] * phik[f];
                dvs[(size_t)j * dv + c] = a;
            }
        }
        free(s); free(z); free(g); free(dden); free(phiq); free(phik); free(dphi);
    }
}

/* ------------------------------------------------ sliding-window attention */

/* Causal sliding-window softmax attention ("Simple linear attention language
 * models balance the recall-throughput tradeoff", Knowl 4): query i attends
 * to keys max(0, i-w+1) .. i (0-based),
 *   o_i = sum_j exp(s_ij - m_i) v_j / sum_j exp(s_ij - m_i),
 *   s_ij = scale q_i.k_j,  m_i = max_j s_ij,  lse_i = m_i + log sum_j exp(s_ij - m_i).
 * One slice per (b,h); plain loops. */
void orc_swa_forward(int B, int H, int N, int dqk, int dv, int w, double scale,
                     const double *q, const double *k, const double *v, double *o, double *lse)
{
    const int BH = B * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < BH; ++bh) {
        const double *qs = q + (size_t)bh * N * dqk, *ks = k + (size_t)bh * N * dqk, *vs = v + (size_t)bh * N * dv;
        double *os = o + (size_t)bh * N * dv;
        double *sc = (double *)malloc(sizeof(double) * (size_t)w);
        for (int i = 0; i < N; ++i) {
            const int j0 = i - w + 1 > 0 ? i - w + 1 : 0;
            double m = -INFINITY;
            for (int j = j0; j <= i; ++j) {
                sc[j - j0] = scale * dot(qs + (size_t)i * dqk, ks + (size_t)j * dqk, dqk);
                if (sc[j - j0] > m) m = sc[j - j0];
            }
            double den = 0.0;
            for (int c = 0; c < dv; ++c) os[(size_t)i * dv + c] = 0.0;
            for (int j = j0; j <= i; ++j) {
                const double e = exp(sc[j - j0] - m);
                den += e;
                for (int c = 0; c < dv; ++c) os[(size_t)i * dv + c] += e * vs[(size_t)j * dv + c];
            }
            for (int c = 0; c < dv; ++c) os[(size_t)i * dv + c] /= den;
            if (lse) lse[(size_t)bh * N + i] = m + log(den);
        }
        free(sc);
    }
}

/* Gradients of the gated masked form by brute force, one slice per (b,h):
 *   w_ij = (prod_{l=j+1..i} exp(g_l)) phi(q_i).phi(k_j),  y_i = sum_j w_ij v_j / sum_j w_ij,
 *   g_i = dO_i / den_i,  dden_i = -g_i . y_i,  dw_ij = g_i . v_j + dden_i,
 *   dv_j = sum_{i>=j} w_ij g_i,
 *   dphiq_i = sum_{j<=i} dw_ij e_ij phi(k_j),  dphik_j = sum_{i>=j} dw_ij e_ij phi(q_i)   (e_ij = w_ij / a_ij),
 *   dg_l = sum over the pairs j < l <= i of dw_ij w_ij   (g_l scales every such w_ij),
 * then dq, dk through the feature map's Jacobian.  O(N^3) for dg. */
void orc_backward_brute_decay(int fmap, int B, int H, int N, int dqk, int dv,
                              const double *q, const double *k, const double *v, const double *g,
                              const double *dout, double *dq, double *dk, double *dvo, double *dg)
{
    const int BH = B * H;
    const int F = orc_feature_dim(fmap, dqk);
#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < BH; ++bh) {
        const double *qs = q + (size_t)bh * N * dqk, *ks = k + (size_t)bh * N * dqk;
        const double *vs = v + (size_t)bh * N * dv, *gs = g + (size_t)bh * N, *dos = dout + (size_t)bh * N * dv;
        double *phiq = phi_rows(fmap, N, dqk, qs), *phik = phi_rows(fmap, N, dqk, ks);
        double *e = (double *)calloc((size_t)N * N, sizeof(double));   /* e_ij, j <= i */
        double *w = (double *)calloc((size_t)N * N, sizeof(double));   /* w_ij */
        double *gi = (double *)malloc(sizeof(double) * (size_t)N * dv);
        double *dd = (double *)malloc(sizeof(double) * (size_t)N);
        double *dphiq = (double *)calloc((size_t)N * F, sizeof(double));
        double *dphik = (double *)calloc((size_t)N * F, sizeof(double));
        for (int i = 0; i < N; ++i) {
            double prod = 1.0;
            for (int j = i; j >= 0; --j) {
                if (j < i) prod *= exp(gs[j + 1]);
                e[(size_t)i * N + j] = prod;
                w[(size_t)i * N + j] = prod * dot(phiq + (size_t)i * F, phik + (size_t)j * F, F);
            }
            double den = 0.0;
            for (int j = 0; j <= i; ++j) den += w[(size_t)i * N + j];
            double gy = 0.0;
            for (int c = 0; c < dv; ++c) {
                double num = 0.0;
                for (int j = 0; j <= i; ++j) num += w[(size_t)i * N + j] * vs[(size_t)j * dv + c];
                gi[(size_t)i * dv + c] = dos[(size_t)i * dv + c] / den;
                gy += gi[(size_t)i * dv + c] * (num / den);
            }
            dd[i] = -gy;
        }
        double *dgs = dg + (size_t)bh * N;
        for (int l = 0; l < N; ++l) dgs[l] = 0.0;
        for (int i = 0; i < N; ++i)
            for (int j = 0; j <= i; ++j) {
                const double dw = dot(gi + (size_t)i * dv, vs + (size_t)j * dv, dv) + dd[i];
                const double ee = e[(size_t)i * N + j], ww = w[(size_t)i * N + j];
                for (int f = 0; f < F; ++f) {
                    dphiq[(size_t)i * F + f] += dw * ee * phik[(size_t)j * F + f];
                    dphik[(size_t)j * F + f] += dw * ee * phiq[(size_t)i * F + f];
                }
                for (int l = j + 1; l <= i; ++l) dgs[l] += dw * ww;
            }
        for (int j = 0; j < N; ++j)
            for (int c = 0; c < dv; ++c) {
                double acc = 0.0;
                for (int i = j; i < N; ++i) acc += w[(size_t)i * N + j] * gi[(size_t)i * dv + c];
                dvo[((size_t)bh * N + j) * dv + c] = acc;
            }
        for (int i = 0; i < N; ++i) {
            orc_phi_vjp(fmap, dqk, qs + (size_t)i * dqk, dphiq + (size_t)i * F, dq + ((size_t)bh * N + i) * dqk);
            orc_phi_vjp(fmap, dqk, ks + (size_t)i * dqk, dphik + (size_t)i * F, dk + ((size_t)bh * N + i) * dqk);
        }
        free(phiq); free(phik); free(e); free(w); free(gi); free(dd); free(dphiq); free(dphik);
    }
}

/* Gated gradients by scans (the header's backward_recurrent_decay). */
void orc_backward_recurrent_decay(int fmap, int B, int H, int N, int dqk, int dv,
                                  const double *q, const double *k, const double *v, const double *gate,
                                  const double *dout, double *dq, double *dk, double *dvv, double *dgate)
{
    const int BH = B * H;
    const int F = orc_feature_dim(fmap, dqk);
#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < BH; ++bh) {
        const double *qs = q + (size_t)bh * N * dqk;
        const double *ks = k + (size_t)bh * N * dqk;
        const double *vs = v + (size_t)bh * N * dv;
        const double *gs = gate + (size_t)bh * N;
        const double *dos = dout + (size_t)bh * N * dv;
        double *dqs = dq + (size_t)bh * N * dqk;
        double *dks = dk + (size_t)bh * N * dqk;
        double *dvs = dvv + (size_t)bh * N * dv;
        double *dgs = dgate + (size_t)bh * N;
        double *s = (double *)calloc((size_t)F * dv, sizeof(double));
        double *z = (double *)calloc((size_t)F, sizeof(double));
        double *g = (double *)malloc(sizeof(double) * (size_t)N * dv);
        double *dden = (double *)malloc(sizeof(double) * (size_t)N);
        double *dB = (double *)malloc(sizeof(double) * (size_t)N);   /* dL/dB_m */
        double *phiq = (double *)malloc(sizeof(double) * (size_t)F);
        double *phik = (double *)malloc(sizeof(double) * (size_t)F);
        double *dphi = (double *)malloc(sizeof(double) * (size_t)F);
        /* Forward-order scan: the gated s_i, z_i include token i. */
        for (int i = 0; i < N; ++i) {
            orc_phi(fmap, dqk, qs + (size_t)i * dqk, phiq);
            orc_phi(fmap, dqk, ks + (size_t)i * dqk, phik);
            const double a = exp(gs[i]);
            for (int f = 0; f < F; ++f) {
                for (int c = 0; c < dv; ++c)
                    s[(size_t)f * dv + c] = a * s[(size_t)f * dv + c] + phik[f] * vs[(size_t)i * dv + c];
                z[f] = a * z[f] + phik[f];
            }
            const double d = dot(phiq, z, F);
            double gy = 0.0;
            for (int c = 0; c < dv; ++c) {
                double n = 0.0;
                for (int f = 0; f < F; ++f) n += phiq[f] * s[(size_t)f * dv + c];
                g[(size_t)i * dv + c] = dos[(size_t)i * dv + c] / d;
                gy += g[(size_t)i * dv + c] * (n / d);
            }
            dden[i] = -gy;
            /* dphi(q_i) = s_i g_i + z_i dden_i */
            for (int f = 0; f < F; ++f)
                dphi[f] = dot(s + (size_t)f * dv, g + (size_t)i * dv, dv) + z[f] * dden[i];
            dB[i] = dot(phiq, dphi, F);
            orc_phi_vjp(fmap, dqk, qs + (size_t)i * dqk, dphi, dqs + (size_t)i * dqk);
        }
        /* Reverse-order scan: R_j = phi(q_j) g_j^T + a_{j+1} R_{j+1} (reusing s), r_j (reusing z). */
        memset(s, 0, sizeof(double) * (size_t)F * dv);
        memset(z, 0, sizeof(double) * (size_t)F);
        for (int j = N - 1; j >= 0; --j) {
            orc_phi(fmap, dqk, qs + (size_t)j * dqk, phiq);
            orc_phi(fmap, dqk, ks + (size_t)j * dqk, phik);
            const double a_next = j + 1 < N ? exp(gs[j + 1]) : 0.0;
            for (int f = 0; f < F; ++f) {
                for (int c = 0; c < dv; ++c)
                    s[(size_t)f * dv + c] = a_next * s[(size_t)f * dv + c] + phiq[f] * g[(size_t)j * dv + c];
                z[f] = a_next * z[f] + phiq[f] * dden[j];
            }
            /* dphi(k_j) = R_j v_j + r_j ; dv_j = R_j^T phi(k_j) */
            for (int f = 0; f < F; ++f)
                dphi[f] = dot(s + (size_t)f * dv, vs + (size_t)j * dv, dv) + z[f];
            dB[j] -= dot(phik, dphi, F);
            orc_phi_vjp(fmap, dqk, ks + (size_t)j * dqk, dphi, dks + (size_t)j * dqk);
            for (int c = 0; c < dv; ++c) {
                double acc = 0.0;
                for (int f = 0; f < F; ++f) acc += s[(size_t)f * dv + c] * phik[f];
                dvs[(size_t)j * dv + c] = acc;
            }
        }
        /* dL/dg_l = sum_{m>=l} dL/dB_m */
        double suffix = 0.0;
        for (int l = N - 1; l >= 0; --l) {
            suffix += dB[l];
            dgs[l] = suffix;
        }
        free(s); free(z); free(g); free(dden); free(dB); free(phiq); free(phik); free(dphi);
    }
}
