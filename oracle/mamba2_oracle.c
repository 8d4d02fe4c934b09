/*
 * mamba2_oracle.c -- plain, slow, fp64 CPU definition of the bidirectional
 * Mamba-2 mixer at the shape of DiffuMamba's own denoiser.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * CPU-baseline leg of the bench may load this library.  The product path (the
 * CUDA library under bidirectional_mamba_denoiser_b200/csrc) shares no code,
 * header, table or helper with this file and never calls it.
 *
 * Sources ("DiffuMamba: High-Throughput Diffusion LMs with Mamba Backbone",
 * arXiv 2511.15927v4): §3.2 Eq. (4)-(6) (two Mamba mixers, one per
 * direction, outputs added); App. C Table 8 (Mamba-2 mixers, state dimension
 * 128, conv dimension 4, expansion 2, no weight tie between directions);
 * App. C Table 12 (d_inner = 3840, d_state = 128, a conv over conv_ch = 4096
 * channels, the projected width D_in = 8056 = 2*3840 + 2*128 + 120, i.e. one
 * group of B and C shared by 120 heads, each with its own step size).
 * The Mamba-2 state-space layer itself is the one the pages cite (Dao & Gu,
 * 2024): per head a scalar decay exp(delta*A), a state of headdim x d_state.
 *
 *   per batch row b, direction r in {0 = forward, 1 = reverse}, conv channel c
 *   in [0, H*P + 2N) of that direction's projected xBC:
 *     v_r[t][c] = silu(cb_r[c] + sum_k w_r[c][k] * xbc_r[t-3+k][c])   (r = 0)
 *     v_r[t][c] = silu(cb_r[c] + sum_k w_r[c][k] * xbc_r[t+3-k][c])   (r = 1)
 *        with xbc_r[i] = 0 outside [0, L)  -- width-4 causal / anti-causal
 *        conv over x, B and C together (Table 12's conv_ch).
 *     x_r[t][h][p] = v_r[t][h*P + p],  B_r[t][n] = v_r[t][H*P + n],
 *     C_r[t][n]    = v_r[t][H*P + N + n]
 *     delta_r[t][h] = softplus(dt_r[t][h] + dt_bias_r[h])
 *     per head h, S = 0 (P x N), t = 0..L-1 (r = 0) or L-1..0 (r = 1):
 *       S[p][n]      = exp(delta_r[t][h] * A_r[h]) * S[p][n]
 *                      + delta_r[t][h] * x_r[t][h][p] * B_r[t][n]
 *       y_r[t][h][p] = sum_n C_r[t][n] * S[p][n] + D_r[h] * x_r[t][h][p]
 *     out[t][h*P + p] = (y_0[t][h][p] + y_1[t][h][p]) * silu(z[t][h*P + p])
 *
 * Readings taken where the pages are silent: the two directions' outputs are
 * added and gated once by silu(z) (the same combine as the d_state-16 layer
 * of this library); the gated RMSNorm and out_proj of a Mamba-2 block belong
 * to the projections around the mixer and are not part of it; D is one
 * scalar per head; initial states are zero.
 *
 * Precision: double throughout, libm exp/log1p, built without fast-math.
 *
 * Layouts (row-major, contiguous, double):
 *   xbc_0, xbc_1 : [batch][L][H*P + 2N]   z : [batch][L][H*P]
 *   dt_0, dt_1   : [batch][L][H]
 *   A, Dskip, dt_bias : [2][H]    conv_w : [2][H*P + 2N][4]    conv_b : [2][H*P + 2N]
 */
#include <math.h>
#include <stddef.h>
#include <stdlib.h>
#include <string.h>

#define OR2_FWD_ONLY 1u
#define OR2_REV_ONLY 2u

/* Test-only planted mistakes (0 = none); the test suite sets one at a time
 * to show that some pin fails for each.
 *   1 B and C skip the conv           2 A taken from the next head
 *   3 delta taken from the next head  4 reverse conv made causal
 *   5 C reads the state before the update
 *   6 D skip dropped                  7 B read from the C slice
 *   8 dt bias dropped                 9 reverse direction walks forwards
 *  10 delta missing on the drive     11 gate is silu of the sum times z
 *  12 x channels laid out p-major (p*H + h) instead of head-major */
static int g_mutation2 = 0;
void oracle2_set_mutation(int m) { g_mutation2 = m; }

static double softplus2(double v) { return (v > 0.0 ? v : 0.0) + log1p(exp(-fabs(v))); }
static double silu2(double v) { return v / (1.0 + exp(-v)); }

typedef struct {
    const double *xbc[2], *z, *dt[2];
    const double *A, *Dskip, *dt_bias, *conv_w, *conv_b;
    int H, P, N;
    long L;
} problem2_t;

/* Conv + SiLU of channel c of direction r at token t (batch row b). */
static double feature(const problem2_t *q, int r, int b, long t, int c) {
    const int CH = q->H * q->P + 2 * q->N;
    const double *w = q->conv_w + ((long)r * CH + c) * 4;
    const double *col = q->xbc[r] + (long)b * q->L * CH + c;
    double acc = q->conv_b ? q->conv_b[r * CH + c] : 0.0;
    for (int k = 0; k < 4; ++k) {
        long i;
        if (r == 0 || g_mutation2 == 4) i = t - 3 + k;
        else i = t + 3 - k;
        if (i >= 0 && i < q->L) acc += w[k] * col[i * CH];
    }
    return silu2(acc);
}

/* Raw (unconvolved) value of channel c, for mutation 1. */
static double raw(const problem2_t *q, int r, int b, long t, int c) {
    const int CH = q->H * q->P + 2 * q->N;
    return q->xbc[r][(long)b * q->L * CH + t * CH + c];
}

/* One direction of head h of batch row b: y [L][P]. */
static void scan_head(const problem2_t *q, int r, int b, int h, double *S, double *y) {
    const int H = q->H, P = q->P, N = q->N;
    const long L = q->L;
    const int hA = (g_mutation2 == 2) ? (h + 1) % H : h;
    const int hD = (g_mutation2 == 3) ? (h + 1) % H : h;
    const double a_h = q->A[r * H + hA];
    const double d_h = q->Dskip[r * H + h];
    const double bias = q->dt_bias[r * H + hD];
    double *xv = (double *)malloc(sizeof(double) * (size_t)P);
    double *Bv = (double *)malloc(sizeof(double) * (size_t)N);
    double *Cv = (double *)malloc(sizeof(double) * (size_t)N);
    memset(S, 0, sizeof(double) * (size_t)P * (size_t)N);
    for (long s = 0; s < L; ++s) {
        const long t = (r == 0 || g_mutation2 == 9) ? s : L - 1 - s;
        for (int p = 0; p < P; ++p) {
            const int c = (g_mutation2 == 12) ? p * H + h : h * P + p;
            xv[p] = feature(q, r, b, t, c);
        }
        for (int n = 0; n < N; ++n) {
            const int cb = H * P + ((g_mutation2 == 7) ? N + n : n);
            const int cc = H * P + N + n;
            Bv[n] = (g_mutation2 == 1) ? raw(q, r, b, t, cb) : feature(q, r, b, t, cb);
            Cv[n] = (g_mutation2 == 1) ? raw(q, r, b, t, cc) : feature(q, r, b, t, cc);
        }
        const double dtv = q->dt[r][(long)b * L * H + t * H + hD];
        const double dl = softplus2(g_mutation2 == 8 ? dtv : dtv + bias);
        const double decay = exp(dl * a_h);
        for (int p = 0; p < P; ++p) {
            double acc = 0.0;
            for (int n = 0; n < N; ++n) {
                double *sp = S + (long)p * N + n;
                const double before = *sp;
                const double drive = (g_mutation2 == 10) ? xv[p] * Bv[n] : dl * xv[p] * Bv[n];
                *sp = decay * *sp + drive;
                acc += Cv[n] * ((g_mutation2 == 5) ? before : *sp);
            }
            y[t * P + p] = acc + ((g_mutation2 == 6) ? 0.0 : d_h * xv[p]);
        }
    }
    free(xv); free(Bv); free(Cv);
}

/* Full-sequence layer.  out [batch][L][H*P]; y_fwd / y_rev, if not NULL,
 * receive the two directions' y before the gate.  Returns 0, or -1 on bad
 * sizes or allocation failure. */
int oracle2_layer_fwd(int batch, long L, int H, int P, int N,
                      const double *xbc_0, const double *xbc_1, const double *z,
                      const double *dt_0, const double *dt_1,
                      const double *A, const double *Dskip, const double *dt_bias,
                      const double *conv_w, const double *conv_b,
                      unsigned flags, double *out, double *y_fwd, double *y_rev) {
    if (batch <= 0 || L <= 0 || H <= 0 || P <= 0 || N <= 0) return -1;
    problem2_t q = {{xbc_0, xbc_1}, z, {dt_0, dt_1}, A, Dskip, dt_bias, conv_w, conv_b, H, P, N, L};
    const int HP = H * P;
    int err = 0;
    #pragma omp parallel for collapse(2) schedule(dynamic, 1) reduction(|:err)
    for (int b = 0; b < batch; ++b) {
        for (int h = 0; h < H; ++h) {
            double *S = (double *)malloc(sizeof(double) * (size_t)P * (size_t)N);
            double *yf = (double *)malloc(sizeof(double) * (size_t)L * (size_t)P);
            double *yb = (double *)malloc(sizeof(double) * (size_t)L * (size_t)P);
            if (!S || !yf || !yb) { err |= 1; free(S); free(yf); free(yb); continue; }
            scan_head(&q, 0, b, h, S, yf);
            scan_head(&q, 1, b, h, S, yb);
            for (long t = 0; t < L; ++t) {
                for (int p = 0; p < P; ++p) {
                    const long o = (long)b * L * HP + t * HP + (long)h * P + p;
                    const double f = (flags & OR2_REV_ONLY) ? 0.0 : yf[t * P + p];
                    const double rv = (flags & OR2_FWD_ONLY) ? 0.0 : yb[t * P + p];
                    const double zv = z[o];
                    out[o] = (g_mutation2 == 11) ? silu2(f + rv) * zv : (f + rv) * silu2(zv);
                    if (y_fwd) y_fwd[o] = yf[t * P + p];
                    if (y_rev) y_rev[o] = yb[t * P + p];
                }
            }
            free(S); free(yf); free(yb);
        }
    }
    return err ? -1 : 0;
}
