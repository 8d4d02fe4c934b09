/*
 * bimamba_oracle.c -- plain, slow, fp64 CPU definition of the bidirectional
 * Mamba mixer layer of DiffuMamba's masked-diffusion denoiser.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * CPU-baseline leg of the bench may load this library.  The product path (the
 * CUDA library under bidirectional_mamba_denoiser_b200/csrc) shares no code,
 * header, table or helper with this file and never calls it.
 *
 * Sources ("DiffuMamba: High-Throughput Diffusion LMs with Mamba Backbone",
 * arXiv 2511.15927v4; "Training Hybrid Block Diffusion Language Models with
 * Partial Bidirectionality", arXiv 2607.02805, abstract):
 *
 *   per batch row b, channel d, direction r in {0 = forward, 1 = reverse}:
 *     u_0[t] = silu(cb_0[d] + sum_k w_0[d][k] * x[t-3+k]),  x[i<0]  = 0
 *     u_1[t] = silu(cb_1[d] + sum_k w_1[d][k] * x[t+3-k]),  x[i>=L] = 0
 *         -- short depthwise conv of width 4, causal for the forward layer
 *            and anti-causal for the reverse one (DiffuMamba §3.2, text under
 *            Eq. (4)-(5); App. C Table 8, "mamba conv dimension 4").
 *     delta_r[t] = softplus(dt_r[t] + bias_r[d])
 *     forward: h = 0, t = 0..L-1;   reverse: h = 0, t = L-1..0
 *       h_n    = exp(delta_r[t] * A_r[d][n]) * h_n + delta_r[t] * B_r[t][n] * u_r[t]
 *       y_r[t] = sum_n C_r[t][n] * h_n + D_r[d] * u_r[t]
 *         -- the selective scan that Eq. (4) (i = 1..L) and Eq. (5)
 *            (i = L..1) write schematically, repeated as Eq. (7)-(8) in
 *            App. A.1; exp(delta*A), delta*B is the discretisation of the
 *            Mamba scan cited there (Gu & Dao, 2024).
 *     out[t] = (y_0[t] + y_1[t]) * silu(z[t])
 *         -- Eq. (6) / Eq. (9) add the two directional streams; silu(z) is
 *            the Mamba mixer's output gate.
 *
 *   block step (DiffuMamba §4.3, block-cached decoding: right-to-left state
 *   updates stay inside the current block while the cached states are carried
 *   forward across blocks; the follow-up paper's abstract: restricting the
 *   reverse scan to the active block makes caching across blocks exact):
 *     forward: starts from the cached (h, last three x of the prefix);
 *     reverse: the block alone -- h = 0 after the block's last token and the
 *              anti-causal conv zero-padded past the block end.
 *
 * Readings taken where the pages are silent: D multiplies the direction's own
 * scan input u_r; x and z are shared by both directions; the conv bias may be
 * absent (NULL reads as 0); initial states are zero.
 *
 * Precision: double throughout, libm exp/log1p, built without fast-math.
 *
 * Layouts (row-major, contiguous, double):
 *   x, z, dt_0, dt_1 : [batch][L][D]     B_0, C_0, B_1, C_1 : [batch][L][N]
 *   A : [2][D][N]    Dskip, dt_bias, conv_b : [2][D]    conv_w : [2][D][4]
 *   state h : [batch][D][N]     conv tail : [batch][3][D] = x[P-3], x[P-2], x[P-1]
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define OR_FWD_ONLY 1u
#define OR_REV_ONLY 2u

/* Test-only planted mistakes (0 = none).  The test suite sets one at a time to
 * show that some pin fails for each; nothing else sets it.
 *   1 D skip dropped              2 sign of A flipped
 *   3 forward conv taps reversed  4 reverse direction walks forwards
 *   5 reverse conv made causal    6 dt bias dropped
 *   7 B and C swapped             8 C reads the state before the update
 *   9 delta missing on the B term 10 gate is silu of the sum, not silu(z)
 *  11 block step ignores the cached conv tail
 *  12 block step ignores the cached state
 *  13 last state dropped          14 conv bias dropped
 *  15 reverse output added after the gate */
static int g_mutation = 0;
void oracle_set_mutation(int m) { g_mutation = m; }
int oracle_get_mutation(void) { return g_mutation; }

void oracle_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

static double softplus(double v) {
    /* log(1 + e^v) in the form that cannot overflow */
    return (v > 0.0 ? v : 0.0) + log1p(exp(-fabs(v)));
}

static double silu(double v) { return v / (1.0 + exp(-v)); }

typedef struct {
    const double *x, *z, *dt[2], *B[2], *C[2];
    const double *A, *Dskip, *dt_bias, *conv_w, *conv_b;
    int D, N;
} problem_t;

/* One direction r over the tokens [0, L) of the column (batch row b,
 * channel d).  h holds the state on entry and on exit.  tail, used only by
 * the forward direction, supplies x[-3..-1] (NULL = zeros).  Writes y[t]
 * (stride 1) and, if not NULL, the scan input u[t] and step size dl[t]. */
static void scan_dir(const problem_t *p, int r, int b, int d, long L,
                     const double *tail, double *h,
                     double *y, double *u_out, double *dl_out) {
    const int D = p->D, N = p->N;
    const long bx = (long)b * L * D, bn = (long)b * L * N;
    const double *w = p->conv_w + ((long)r * D + d) * 4;
    const double cb = (p->conv_b && g_mutation != 14) ? p->conv_b[r * D + d] : 0.0;
    const double bias = p->dt_bias[r * D + d];
    const double Dd = p->Dskip[r * D + d];
    const double *Arow = p->A + ((long)r * D + d) * N;
    const int nst = (g_mutation == 13) ? N - 1 : N;
    for (long s = 0; s < L; ++s) {
        long t = (r == 0 || g_mutation == 4) ? s : L - 1 - s;
        double c = cb;
        for (int k = 0; k < 4; ++k) {
            long i;
            if (r == 0) i = (g_mutation == 3) ? t - k : t - 3 + k;
            else        i = (g_mutation == 5) ? t - 3 + k : t + 3 - k;
            double xv = 0.0;
            if (i >= 0 && i < L) xv = p->x[bx + i * D + d];
            else if (r == 0 && tail && i < 0 && g_mutation != 11) xv = tail[(3 + i) * D];
            c += w[k] * xv;
        }
        const double u = silu(c);
        const double dtv = p->dt[r][bx + t * D + d];
        const double dl = softplus(g_mutation == 6 ? dtv : dtv + bias);
        const double *Bt = p->B[r] + bn + t * N;
        const double *Ct = p->C[r] + bn + t * N;
        double acc = 0.0;
        for (int n = 0; n < nst; ++n) {
            const double a = (g_mutation == 2) ? -Arow[n] : Arow[n];
            const double bt = (g_mutation == 7) ? Ct[n] : Bt[n];
            const double ct = (g_mutation == 7) ? Bt[n] : Ct[n];
            const double drive = (g_mutation == 9) ? bt * u : dl * bt * u;
            const double hprev = h[n];
            h[n] = exp(dl * a) * h[n] + drive;
            acc += ct * ((g_mutation == 8) ? hprev : h[n]);
        }
        y[t] = acc + ((g_mutation == 1) ? 0.0 : Dd * u);
        if (u_out) u_out[t] = u;
        if (dl_out) dl_out[t] = dl;
    }
}

static void gate_store(const problem_t *p, int b, int d, long L, unsigned flags,
                       const double *yf, const double *yb, double *out) {
    const int D = p->D;
    const long bx = (long)b * L * D;
    for (long t = 0; t < L; ++t) {
        const double zv = p->z[bx + t * D + d];
        const double f = (flags & OR_REV_ONLY) ? 0.0 : yf[t];
        const double r = (flags & OR_FWD_ONLY) ? 0.0 : yb[t];
        double o;
        if (g_mutation == 10) o = silu(f + r) * zv;
        else if (g_mutation == 15) o = f * silu(zv) + r;
        else o = (f + r) * silu(zv);
        out[bx + t * D + d] = o;
    }
}

static int bad_dims(int batch, long L, int D, int N) {
    return batch <= 0 || L <= 0 || D <= 0 || N <= 0;
}

/* Full-sequence layer.  out [batch][L][D]; y_fwd / y_rev, if not NULL,
 * receive the two directions' y before the gate.  Returns 0, or -1 on bad
 * sizes or allocation failure. */
int oracle_layer_fwd(int batch, long L, int D, int N,
                     const double *x, const double *z,
                     const double *dt_0, const double *dt_1,
                     const double *B_0, const double *C_0,
                     const double *B_1, const double *C_1,
                     const double *A, const double *Dskip, const double *dt_bias,
                     const double *conv_w, const double *conv_b,
                     unsigned flags, double *out, double *y_fwd, double *y_rev) {
    if (bad_dims(batch, L, D, N)) return -1;
    problem_t p = {x, z, {dt_0, dt_1}, {B_0, B_1}, {C_0, C_1},
                   A, Dskip, dt_bias, conv_w, conv_b, D, N};
    int err = 0;
    #pragma omp parallel for collapse(2) schedule(dynamic, 1) reduction(|:err)
    for (int b = 0; b < batch; ++b) {
        for (int d = 0; d < D; ++d) {
            double *yf = (double *)malloc(sizeof(double) * (size_t)L);
            double *yb = (double *)malloc(sizeof(double) * (size_t)L);
            double *h = (double *)malloc(sizeof(double) * (size_t)N);
            if (!yf || !yb || !h) { err |= 1; free(yf); free(yb); free(h); continue; }
            memset(h, 0, sizeof(double) * (size_t)N);
            scan_dir(&p, 0, b, d, L, NULL, h, yf, NULL, NULL);
            memset(h, 0, sizeof(double) * (size_t)N);
            scan_dir(&p, 1, b, d, L, NULL, h, yb, NULL, NULL);
            gate_store(&p, b, d, L, flags, yf, yb, out);
            const long bx = (long)b * L * D;
            for (long t = 0; t < L; ++t) {
                if (y_fwd) y_fwd[bx + t * D + d] = yf[t];
                if (y_rev) y_rev[bx + t * D + d] = yb[t];
            }
            free(yf); free(yb); free(h);
        }
    }
    return err ? -1 : 0;
}

/* The conv+SiLU outputs u and step sizes delta of both directions,
 * [2][batch][L][D] each.  (C and z are not read.) */
int oracle_features(int batch, long L, int D, int N,
                    const double *x, const double *dt_0, const double *dt_1,
                    const double *B_0, const double *B_1,
                    const double *A, const double *Dskip, const double *dt_bias,
                    const double *conv_w, const double *conv_b,
                    double *u, double *delta) {
    if (bad_dims(batch, L, D, N)) return -1;
    problem_t p = {x, NULL, {dt_0, dt_1}, {B_0, B_1}, {B_0, B_1},
                   A, Dskip, dt_bias, conv_w, conv_b, D, N};
    int err = 0;
    #pragma omp parallel for collapse(2) schedule(dynamic, 1) reduction(|:err)
    for (int b = 0; b < batch; ++b) {
        for (int d = 0; d < D; ++d) {
            double *y = (double *)malloc(sizeof(double) * (size_t)L * 3);
            double *h = (double *)malloc(sizeof(double) * (size_t)N);
            if (!y || !h) { err |= 1; free(y); free(h); continue; }
            for (int r = 0; r < 2; ++r) {
                memset(h, 0, sizeof(double) * (size_t)N);
                scan_dir(&p, r, b, d, L, NULL, h, y, y + L, y + 2 * L);
                const long base = ((long)r * batch + b) * L * D;
                for (long t = 0; t < L; ++t) {
                    u[base + t * D + d] = y[L + t];
                    delta[base + t * D + d] = y[2 * L + t];
                }
            }
            free(y); free(h);
        }
    }
    return err ? -1 : 0;
}

/* Forward-only scan over a prefix of P tokens from a zero state.  Returns the
 * final state h [batch][D][N] and the conv tail [batch][3][D] (x[P-3..P-1],
 * zero where the position is negative).  This is the cache a block step
 * starts from. */
int oracle_prefix_state(int batch, long P, int D, int N,
                        const double *x, const double *dt_0, const double *B_0,
                        const double *A, const double *Dskip, const double *dt_bias,
                        const double *conv_w, const double *conv_b,
                        double *h_out, double *tail_out) {
    if (bad_dims(batch, P, D, N)) return -1;
    problem_t p = {x, NULL, {dt_0, dt_0}, {B_0, B_0}, {B_0, B_0},
                   A, Dskip, dt_bias, conv_w, conv_b, D, N};
    int err = 0;
    #pragma omp parallel for collapse(2) schedule(dynamic, 1) reduction(|:err)
    for (int b = 0; b < batch; ++b) {
        for (int d = 0; d < D; ++d) {
            double *y = (double *)malloc(sizeof(double) * (size_t)P);
            if (!y) { err |= 1; continue; }
            double *h = h_out + ((long)b * D + d) * N;
            memset(h, 0, sizeof(double) * (size_t)N);
            scan_dir(&p, 0, b, d, P, NULL, h, y, NULL, NULL);
            for (int j = 0; j < 3; ++j) {
                const long i = P - 3 + j;
                tail_out[((long)b * 3 + j) * D + d] = (i >= 0) ? x[((long)b * P + i) * D + d] : 0.0;
            }
            free(y);
        }
    }
    return err ? -1 : 0;
}

/* Block step: G tokens of block input ([batch][G][D] / [batch][G][N]).
 * The forward direction starts from (h_in, tail_in); the reverse direction
 * sees the block alone.  out [batch][G][D].  If h_out is not NULL the state
 * after the block is written there (h_out may equal h_in), and likewise the
 * new conv tail (tail_out may equal tail_in). */
int oracle_block_step(int batch, long G, int D, int N,
                      const double *h_in, const double *tail_in,
                      const double *x, const double *z,
                      const double *dt_0, const double *dt_1,
                      const double *B_0, const double *C_0,
                      const double *B_1, const double *C_1,
                      const double *A, const double *Dskip, const double *dt_bias,
                      const double *conv_w, const double *conv_b,
                      unsigned flags, double *out,
                      double *h_out, double *tail_out,
                      double *y_fwd, double *y_rev) {
    if (bad_dims(batch, G, D, N)) return -1;
    problem_t p = {x, z, {dt_0, dt_1}, {B_0, B_1}, {C_0, C_1},
                   A, Dskip, dt_bias, conv_w, conv_b, D, N};
    double *new_tail = NULL;
    if (tail_out) {
        new_tail = (double *)malloc(sizeof(double) * (size_t)batch * 3 * (size_t)D);
        if (!new_tail) return -1;
    }
    int err = 0;
    #pragma omp parallel for collapse(2) schedule(dynamic, 1) reduction(|:err)
    for (int b = 0; b < batch; ++b) {
        for (int d = 0; d < D; ++d) {
            double *yf = (double *)malloc(sizeof(double) * (size_t)G);
            double *yb = (double *)malloc(sizeof(double) * (size_t)G);
            double *h = (double *)malloc(sizeof(double) * (size_t)N);
            if (!yf || !yb || !h) { err |= 1; free(yf); free(yb); free(h); continue; }
            const double *hin = h_in + ((long)b * D + d) * N;
            for (int n = 0; n < N; ++n) h[n] = (g_mutation == 12) ? 0.0 : hin[n];
            scan_dir(&p, 0, b, d, G, tail_in + (long)b * 3 * D + d, h, yf, NULL, NULL);
            if (h_out) {
                double *ho = h_out + ((long)b * D + d) * N;
                for (int n = 0; n < N; ++n) ho[n] = h[n];
            }
            memset(h, 0, sizeof(double) * (size_t)N);
            scan_dir(&p, 1, b, d, G, NULL, h, yb, NULL, NULL);
            gate_store(&p, b, d, G, flags, yf, yb, out);
            const long bx = (long)b * G * D;
            for (long t = 0; t < G; ++t) {
                if (y_fwd) y_fwd[bx + t * D + d] = yf[t];
                if (y_rev) y_rev[bx + t * D + d] = yb[t];
            }
            if (new_tail) {
                /* last three x of (old tail ++ block) */
                for (int j = 0; j < 3; ++j) {
                    const long i = G - 3 + j;   /* position relative to block start */
                    new_tail[((long)b * 3 + j) * D + d] =
                        (i >= 0) ? x[bx + i * D + d] : tail_in[((long)b * 3 + (3 + i)) * D + d];
                }
            }
            free(yf); free(yb); free(h);
        }
    }
    if (new_tail) {
        if (!err) memcpy(tail_out, new_tail, sizeof(double) * (size_t)batch * 3 * (size_t)D);
        free(new_tail);
    }
    return err ? -1 : 0;
}
