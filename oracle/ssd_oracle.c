/*
 * ssd_oracle.c -- CPU oracle for the Mamba-2 selective-state (SSD) causal layer.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, obviously correct
 * statement of what the GPU path computes.  Only the test-suite, the smoke
 * check and the CPU-baseline leg of the benchmark may load it.  It shares no
 * code, header, table or helper with the CUDA library, and the library never
 * calls it.
 *
 * Everything is computed in IEEE double precision.  Inputs are taken as the
 * exact values of the I/O tensors (bf16 and fp32 values are exactly
 * representable in float), outputs are written as double, except the conv
 * output, which is an ABI-visible tensor and is rounded to the I/O dtype
 * (round-to-nearest-even), exactly as the GPU library stores it.
 *
 * Sources (web pages this layer is described on):
 *  - "Video-Ma2mba" verdict record for arXiv 2411.19460 (pith.science),
 *    pith_extraction.core_discovery: the Markov state recurrence of Mamba-2,
 *    Eq. (1)  h_t = A_t h_{t-1} + B_t x_t.
 *  - same record, skeptic_critique.load_bearing_attack and concrete_test:
 *    a causal Conv1d of kernel 4 precedes the SSD, output at t depends on
 *    inputs t-3..t; exact resume needs that conv buffer as well.
 *  - same record, pith_extraction.key_machinery ("Algorithm 1", Sckpt):
 *    the SSD state is stored every s time steps.
 *  - same record, desk_editor.letter: the pseudocode's re-initialisation of h
 *    inside the time loop is a typo; h is initialised once.
 *  - Video-Ma2mba-0.3B model card (ailist.pro), Architecture table: Mamba-2
 *    language model, bfloat16.
 * The discretised per-head form used here -- A_t = exp(dt_t * A_h),
 * input term dt_t * B_t x_t^T, output y_t = C_t^T h_t + D_h x_t -- is the
 * plainest reading of Eq. (1) for a Mamba-2 head (the pages give Eq. (1)
 * without dt, C or D).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_CONV_K 4

/* ---- rounding of a double to the I/O dtype (round to nearest, ties to even) */

/* bfloat16: 8 significant bits, exponent range of fp32. */
static double round_to_bf16(double d)
{
    if (!isfinite(d) || d == 0.0) return d;
    int e;
    (void)frexp(fabs(d), &e);           /* |d| = m * 2^e, m in [0.5, 1) */
    int q = e - 8;                      /* spacing of 8-bit significands */
    if (e - 1 < -126) q = -133;         /* subnormal range: fixed spacing */
    double r = nearbyint(ldexp(fabs(d), -q)); /* default mode: ties to even */
    double out = ldexp(r, q);
    if (out > 3.3895313892515355e38) out = INFINITY;
    return copysign(out, d);
}

double oracle_round_bf16(double d) { return round_to_bf16(d); }

static double round_io(double d, int io_round)
{
    if (io_round == 1) return (double)(float)d;   /* fp32, C conversion is RNE */
    if (io_round == 2) return round_to_bf16(d);
    return d;
}

/* ---- causal depthwise conv1d (kernel 4) + SiLU ------------------------------
 * v[t,c] = silu(bias_c + sum_{k=0..3} w[c,k] * u[t-3+k, c]),  silu(z) = z/(1+e^-z)
 * u at t < 0 comes from tail_in (row r holds position r-3), or is zero.
 * tail_out[r] = u at position L-3+r (taken from tail_in when that is < 0).
 * Layouts: u, v [b][L][Cch] row-major; w [Cch][4]; bias [Cch]; tails [b][3][Cch].
 */
void oracle_conv(int b, int64_t L, int Cch,
                 const float *u, const float *w, const float *bias,
                 const float *tail_in, int io_round,
                 float *v, float *tail_out)
{
    #pragma omp parallel for schedule(static)
    for (int64_t job = 0; job < (int64_t)b * Cch; ++job) {
        const int bi = (int)(job / Cch);
        const int c = (int)(job % Cch);
        const float *ub = u + (int64_t)bi * L * Cch;
        const float *tb = tail_in ? tail_in + (int64_t)bi * 3 * Cch : NULL;
        for (int64_t t = 0; t < L; ++t) {
            double z = bias ? (double)bias[c] : 0.0;
            for (int k = 0; k < ORACLE_CONV_K; ++k) {
                int64_t tt = t - (ORACLE_CONV_K - 1) + k;
                double val;
                if (tt >= 0) val = ub[tt * Cch + c];
                else val = tb ? (double)tb[(3 + tt) * Cch + c] : 0.0;
                z += (double)w[c * ORACLE_CONV_K + k] * val;
            }
            double silu = z / (1.0 + exp(-z));
            v[((int64_t)bi * L + t) * Cch + c] = (float)round_io(silu, io_round);
        }
        if (tail_out) {
            for (int r = 0; r < 3; ++r) {
                int64_t pos = L - 3 + r;
                float val;
                if (pos >= 0) val = ub[pos * Cch + c];
                else val = tb ? tb[(3 + pos) * Cch + c] : 0.0f;
                tail_out[((int64_t)bi * 3 + r) * Cch + c] = val;
            }
        }
    }
}

/* ---- selective state recurrence, one step per token ------------------------
 * For every batch row bi and every selected head h (group g = h*G/H):
 *   state S[p][n] = h0 (once, before the loop; zeros when h0 is NULL)
 *   for t = 0..L-1:
 *     a = exp(dt[t,h] * A[h])
 *     S[p][n] = a * S[p][n] + dt[t,h] * x[t,h,p] * B[t,g,n]
 *     y[t,h,p] = sum_n C[t,g,n] * S[p][n] + D[h] * x[t,h,p]
 *     if (t+1) % s == 0: ckpt[(t+1)/s - 1] = S
 *   h_final = S
 * Strided inputs (element strides):
 *   x[bi*x_bs + t*x_rs + h*P + p], B[bi*B_bs + t*B_rs + g*N + n], same for C,
 *   dt[(bi*L + t)*H + h], A[H], D[H] (nullable), h0[b][H][P][N] (nullable;
 *   double, so that a state handed over from an earlier call resumes exactly).
 * heads/n_heads select a subset of heads (heads == NULL: all H, in order);
 * outputs are compact over the selection:
 *   y[b][L][n_heads][P], h_final[b][n_heads][P][N], h_ckpt[b][L/s][n_heads][P][N].
 */
void oracle_scan(int b, int64_t L, int H, int P, int N, int G, int64_t s,
                 const float *x, int64_t x_bs, int64_t x_rs,
                 const float *B, int64_t B_bs, int64_t B_rs,
                 const float *C, int64_t C_bs, int64_t C_rs,
                 const float *dt, const float *A, const float *D,
                 const double *h0, const int *heads, int n_heads,
                 double *y, double *h_final, double *h_ckpt)
{
    if (!heads) n_heads = H;
    const int64_t n_ckpt = s > 0 ? L / s : 0;
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t job = 0; job < (int64_t)b * n_heads; ++job) {
        const int bi = (int)(job / n_heads);
        const int hs = (int)(job % n_heads);
        const int h = heads ? heads[hs] : hs;
        const int g = (int)((int64_t)h * G / H);
        double *S = (double *)malloc(sizeof(double) * (size_t)P * N);
        for (int i = 0; i < P * N; ++i)
            S[i] = h0 ? h0[(((int64_t)bi * H + h) * P) * N + i] : 0.0;
        const double Ah = A[h];
        const double Dh = D ? (double)D[h] : 0.0;
        for (int64_t t = 0; t < L; ++t) {
            const float *xt = x + bi * x_bs + t * x_rs + (int64_t)h * P;
            const float *Bt = B + bi * B_bs + t * B_rs + (int64_t)g * N;
            const float *Ct = C + bi * C_bs + t * C_rs + (int64_t)g * N;
            const double dtv = dt[((int64_t)bi * L + t) * H + h];
            const double a = exp(dtv * Ah);
            double *yt = y + (((int64_t)bi * L + t) * n_heads + hs) * P;
            for (int p = 0; p < P; ++p) {
                const double xp = xt[p];
                const double u = dtv * xp;
                double acc = 0.0;
                double *Sp = S + (int64_t)p * N;
                for (int n = 0; n < N; ++n) {
                    Sp[n] = a * Sp[n] + u * (double)Bt[n];
                    acc += (double)Ct[n] * Sp[n];
                }
                yt[p] = acc + Dh * xp;
            }
            if (h_ckpt && s > 0 && (t + 1) % s == 0) {
                const int64_t k = (t + 1) / s - 1;
                double *dst = h_ckpt + (((int64_t)bi * n_ckpt + k) * n_heads + hs) * P * N;
                memcpy(dst, S, sizeof(double) * (size_t)P * N);
            }
        }
        if (h_final)
            memcpy(h_final + ((int64_t)bi * n_heads + hs) * P * N, S,
                   sizeof(double) * (size_t)P * N);
        free(S);
    }
}

/* ---- reverse mode of the recurrence (gradients of a scalar loss) -----------
 * The loss is any scalar whose gradients with respect to the outputs are
 * dy = dLoss/dy [b][L][H][P] and dh_final = dLoss/dh_final [b][H][P][N]
 * (nullable: zero).  Walking the tokens backwards with the running adjoint
 * G = dLoss/dh_t (P x N), seeded with dh_final:
 *   G += dy_t C_t^T                                  (y_t reads h_t)
 *   dC_t[n]  = sum_p dy_t[p] h_t[p][n]
 *   dx_t[p]  = D dy_t[p] + dt_t sum_n G[p][n] B_t[n]
 *   dB_t[n]  = dt_t sum_p G[p][n] x_t[p]
 *   ddt_t    = sum_{p,n} G[p][n] (x_t[p] B_t[n] + A a_t h_{t-1}[p][n])
 *   dA      += sum_{p,n} G[p][n] dt_t a_t h_{t-1}[p][n]
 *   dD      += sum_p dy_t[p] x_t[p]
 *   G       *= a_t                                   (h_t = a_t h_{t-1} + ...)
 * and dh0 = G after token 0.  This needs h_{t-1} and h_t on the way back.
 * With h_ckpt == NULL (or s == 0) they are all recomputed once from h0 and
 * kept ("full backprop").  Otherwise the sequence is cut into cells of s
 * tokens, walked last cell first, and each cell's states are recomputed from
 * the checkpoint that starts it (h0 for the first cell) -- the grid-cell
 * recompute of "Algorithm 1" (MA-GC) in the Video-Ma2mba verdict record,
 * pith_extraction.key_machinery.  Both modes run the same reverse sweep.
 * Outputs (double): dx [b][L][H][P]; dB_h, dC_h [b][L][H][N] per head (the
 * group's gradient is the sum over its heads); ddt [b][L][H]; dA_b, dD_b
 * [b][H] per batch row (the parameter gradient is the sum over rows);
 * dh0 [b][H][P][N].  h_ckpt is [b][L/s][H][P][N] as the forward writes it.
 */
void oracle_scan_backward(int b, int64_t L, int H, int P, int N, int G, int64_t s,
                          const float *x, int64_t x_bs, int64_t x_rs,
                          const float *B, int64_t B_bs, int64_t B_rs,
                          const float *C, int64_t C_bs, int64_t C_rs,
                          const float *dt, const float *A, const float *D,
                          const double *h0, const double *h_ckpt,
                          const double *dy, const double *dh_final,
                          double *dx, double *dB_h, double *dC_h, double *ddt,
                          double *dA_b, double *dD_b, double *dh0)
{
    const int use_ckpt = (h_ckpt != NULL && s > 0);
    const int64_t cell = use_ckpt ? s : (L > 0 ? L : 1);
    const int64_t n_cells = L > 0 ? (L + cell - 1) / cell : 0;
    const int64_t n_ckpt = s > 0 ? L / s : 0;
    const int64_t PN = (int64_t)P * N;
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t job = 0; job < (int64_t)b * H; ++job) {
        const int bi = (int)(job / H);
        const int h = (int)(job % H);
        const int grp = (int)((int64_t)h * G / H);
        const double Ah = A[h];
        const double Dh = D ? (double)D[h] : 0.0;
        double *st = (double *)malloc(sizeof(double) * (size_t)((cell + 1) * PN));
        double *Gs = (double *)malloc(sizeof(double) * (size_t)PN);
        for (int64_t i = 0; i < PN; ++i)
            Gs[i] = dh_final ? dh_final[((int64_t)bi * H + h) * PN + i] : 0.0;
        double dA_acc = 0.0, dD_acc = 0.0;
        for (int64_t k = n_cells - 1; k >= 0; --k) {
            const int64_t t0 = k * cell;
            const int64_t t1 = (t0 + cell < L) ? t0 + cell : L;
            /* the cell's starting state */
            for (int64_t i = 0; i < PN; ++i) {
                double v = 0.0;
                if (k == 0) v = h0 ? h0[((int64_t)bi * H + h) * PN + i] : 0.0;
                else v = h_ckpt[(((int64_t)bi * n_ckpt + (k - 1)) * H + h) * PN + i];
                st[i] = v;
            }
            /* recompute h_t for the cell: st[(t - t0 + 1) * PN] holds h_t */
            for (int64_t t = t0; t < t1; ++t) {
                const float *xt = x + bi * x_bs + t * x_rs + (int64_t)h * P;
                const float *Bt = B + bi * B_bs + t * B_rs + (int64_t)grp * N;
                const double dtv = dt[((int64_t)bi * L + t) * H + h];
                const double step_decay = exp(dtv * Ah);
                const double *prev = st + (t - t0) * PN;
                double *cur = st + (t - t0 + 1) * PN;
                for (int p = 0; p < P; ++p)
                    for (int n = 0; n < N; ++n)
                        cur[(int64_t)p * N + n] = step_decay * prev[(int64_t)p * N + n] + dtv * (double)xt[p] * (double)Bt[n];
            }
            /* reverse sweep */
            for (int64_t t = t1 - 1; t >= t0; --t) {
                const float *xt = x + bi * x_bs + t * x_rs + (int64_t)h * P;
                const float *Bt = B + bi * B_bs + t * B_rs + (int64_t)grp * N;
                const float *Ct = C + bi * C_bs + t * C_rs + (int64_t)grp * N;
                const double dtv = dt[((int64_t)bi * L + t) * H + h];
                const double a_t = exp(dtv * Ah);
                const double *dyt = dy + (((int64_t)bi * L + t) * H + h) * P;
                const double *hprev = st + (t - t0) * PN;
                const double *hcur = st + (t - t0 + 1) * PN;
                for (int p = 0; p < P; ++p)
                    for (int n = 0; n < N; ++n)
                        Gs[(int64_t)p * N + n] += dyt[p] * (double)Ct[n];
                double *dCt = dC_h + (((int64_t)bi * L + t) * H + h) * N;
                double *dBt = dB_h + (((int64_t)bi * L + t) * H + h) * N;
                for (int n = 0; n < N; ++n) {
                    double c_acc = 0.0, b_acc = 0.0;
                    for (int p = 0; p < P; ++p) {
                        c_acc += dyt[p] * hcur[(int64_t)p * N + n];
                        b_acc += Gs[(int64_t)p * N + n] * (double)xt[p];
                    }
                    dCt[n] = c_acc;
                    dBt[n] = dtv * b_acc;
                }
                double *dxt = dx + (((int64_t)bi * L + t) * H + h) * P;
                double ddt_acc = 0.0, dA_t = 0.0;
                for (int p = 0; p < P; ++p) {
                    double acc = 0.0;
                    for (int n = 0; n < N; ++n) {
                        const double gv = Gs[(int64_t)p * N + n];
                        acc += gv * (double)Bt[n];
                        ddt_acc += gv * ((double)xt[p] * (double)Bt[n]);
                        dA_t += gv * a_t * hprev[(int64_t)p * N + n];
                    }
                    dxt[p] = Dh * dyt[p] + dtv * acc;
                    dD_acc += dyt[p] * (double)xt[p];
                }
                ddt[((int64_t)bi * L + t) * H + h] = ddt_acc + Ah * dA_t;
                dA_acc += dtv * dA_t;
                for (int64_t i = 0; i < PN; ++i) Gs[i] *= a_t;
            }
        }
        dA_b[(int64_t)bi * H + h] = dA_acc;
        dD_b[(int64_t)bi * H + h] = dD_acc;
        if (dh0) memcpy(dh0 + ((int64_t)bi * H + h) * PN, Gs, sizeof(double) * (size_t)PN);
        free(st);
        free(Gs);
    }
}

/* ---- gated RMS normalisation of the layer output ------------------------
 * The Mamba-2 block's output norm (not on the pages, which end at y; the
 * plainest block surroundings): for every row r and channel c of d,
 *   v[c]   = y[r,c] * silu(z[r,c]),   silu(z) = z / (1 + e^-z)
 *   ms_g   = (1/group) * sum_{c' in group g} v[c']^2     (groups of `group`
 *            consecutive channels)
 *   out[r,c] = v[c] / sqrt(ms_g + eps) * w[c]
 * rounded to the I/O dtype.  Rows are y[r*y_rs + c], z[r*z_rs + c],
 * out[r*out_rs + c]; w is [d].
 */
void oracle_gated_rmsnorm(int64_t rows, int d, int group,
                          const float *y, int64_t y_rs, const float *z, int64_t z_rs,
                          const float *w, double eps, int io_round,
                          float *out, int64_t out_rs)
{
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        double *v = (double *)malloc(sizeof(double) * (size_t)d);
        for (int c = 0; c < d; ++c) {
            const double zc = z[r * z_rs + c];
            v[c] = (double)y[r * y_rs + c] * (zc / (1.0 + exp(-zc)));
        }
        for (int g0 = 0; g0 < d; g0 += group) {
            double ss = 0.0;
            for (int c = g0; c < g0 + group; ++c) ss += v[c] * v[c];
            const double scale = 1.0 / sqrt(ss / group + eps);
            for (int c = g0; c < g0 + group; ++c)
                out[r * out_rs + c] = (float)round_io(v[c] * scale * (double)w[c], io_round);
        }
        free(v);
    }
}

/* Number of OpenMP threads the oracle would use (for reporting). */
int oracle_num_threads(void)
{
    int n = 1;
    #pragma omp parallel
    {
        #pragma omp single
        {
#ifdef _OPENMP
            extern int omp_get_num_threads(void);
            n = omp_get_num_threads();
#endif
        }
    }
    return n;
}
