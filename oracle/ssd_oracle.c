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

/* ---- reverse mode of the whole layer: conv1d + SiLU, then the recurrence --
 * Forward, as oracle_conv followed by oracle_scan:
 *   z[t,c] = bias_c + sum_k w[c,k] u[t-3+k,c],   v[t,c] = round_io(silu(z[t,c]))
 *   x = v[:, 0 : H*P], B = v[:, H*P : H*P+G*N], C = v[:, H*P+G*N : H*P+2*G*N]
 *   the recurrence of oracle_scan from h0, y, h_final;
 *   tail_out[r] = u at position L-3+r (tail_in[3+pos] when pos < 0).
 * Given the loss gradients dy [b][L][H][P], dh_final [b][H][P][N] and
 * dtail_out [b][3][Cch] (each nullable: zero), the reverse mode, token by
 * token from the last:
 *   the scan part as in oracle_scan_backward, giving dx, dB, dC (summed over
 *   the heads of each group, heads in increasing order), ddt, dA, dD, dh0;
 *   dv = [dx | dB | dC] per channel; dz = dv * silu'(z),
 *   silu'(z) = sig(z) (1 + z (1 - sig(z))),  sig(z) = 1 / (1 + e^-z);
 *   dbias_c += dz[t,c];  dw[c,k] += dz[t,c] u[t-3+k,c];
 *   du[t-3+k,c] += w[c,k] dz[t,c]  (dtail_in[3+t-3+k] when t-3+k < 0).
 * The rounding of v to the I/O dtype is taken as the identity in the reverse
 * mode (its derivative is 1 almost everywhere in the limit of fine rounding).
 * Cells (MA-GC's grid-cell recompute on the sequence axis, "Algorithm 1" of
 * the Video-Ma2mba verdict record, pith_extraction.key_machinery, with the
 * conv buffer that skeptic_critique.headline says exactness needs): with
 * h_ckpt [b][L/s][H][P][N] and conv_ckpt [b][L/s][3][Cch] (both, and s > 0)
 * the sequence is cut into cells of s tokens, walked last first; cell k
 * rebuilds z, v and the states from ITS OWN rows of u, the conv buffer
 * conv_ckpt[k-1] (the 3 rows of u before the cell; tail_in for k = 0) and the
 * state h_ckpt[k-1] (h0 for k = 0).  Without them: one cell over the whole
 * sequence ("full backprop").  The gradient that reaches a cell's conv buffer
 * is the gradient of those rows of u.  Every sum runs over tokens in
 * decreasing order in both modes, so with exact checkpoints the two agree
 * bitwise.
 * Outputs (double): du [b][L][Cch], dtail_in [b][3][Cch], dw_b [b][Cch][4] and
 * dbias_b [b][Cch] per batch row, ddt [b][L][H], dA_b and dD_b [b][H] per batch
 * row, dh0 [b][H][P][N].  u, w, bias, tail_in, conv_ckpt are float holding
 * exact values; dt, A, D as for oracle_scan.
 */
void oracle_layer_backward(int b, int64_t L, int H, int P, int N, int G, int64_t s,
                           const float *u, const float *w, const float *bias, const float *tail_in,
                           const float *dt, const float *A, const float *D,
                           const double *h0, const double *h_ckpt, const float *conv_ckpt,
                           const double *dy, const double *dh_final, const double *dtail_out,
                           int io_round,
                           double *du, double *dtail_in, double *dw_b, double *dbias_b,
                           double *ddt, double *dA_b, double *dD_b, double *dh0)
{
    const int use_cells = (h_ckpt != NULL && conv_ckpt != NULL && s > 0);
    const int64_t cell = use_cells ? s : (L > 0 ? L : 1);
    const int64_t n_cells = L > 0 ? (L + cell - 1) / cell : 0;
    const int64_t n_ckpt = s > 0 ? L / s : 0;
    const int64_t PN = (int64_t)P * N;
    const int HP = H * P, GN = G * N;
    const int Cch = HP + 2 * GN;
    #pragma omp parallel for schedule(dynamic, 1)
    for (int bi = 0; bi < b; ++bi) {
        const float *ub = u + (int64_t)bi * L * Cch;
        double *dub = du + (int64_t)bi * L * Cch;
        double *dtb = dtail_in + (int64_t)bi * 3 * Cch;
        double *dwb = dw_b + (int64_t)bi * Cch * 4;
        double *dbb = dbias_b + (int64_t)bi * Cch;
        double *z = (double *)malloc(sizeof(double) * (size_t)(cell * Cch));
        double *v = (double *)malloc(sizeof(double) * (size_t)(cell * Cch));
        double *dv = (double *)malloc(sizeof(double) * (size_t)(cell * Cch));
        double *ext = (double *)malloc(sizeof(double) * (size_t)(3 * Cch));
        double *st = (double *)malloc(sizeof(double) * (size_t)(H * (cell + 1) * PN));
        double *Gs = (double *)malloc(sizeof(double) * (size_t)(H * PN));
        double *dA_acc = (double *)calloc((size_t)H, sizeof(double));
        double *dD_acc = (double *)calloc((size_t)H, sizeof(double));
        for (int64_t i = 0; i < L * Cch; ++i) dub[i] = 0.0;
        for (int i = 0; i < 3 * Cch; ++i) dtb[i] = 0.0;
        for (int i = 0; i < Cch * 4; ++i) dwb[i] = 0.0;
        for (int i = 0; i < Cch; ++i) dbb[i] = 0.0;
        for (int h = 0; h < H; ++h)
            for (int64_t i = 0; i < PN; ++i)
                Gs[h * PN + i] = dh_final ? dh_final[((int64_t)bi * H + h) * PN + i] : 0.0;
        /* tail_out copies rows of u (or of tail_in): their gradients start the sums */
        if (dtail_out) {
            for (int r = 0; r < 3; ++r) {
                const int64_t at = L - 3 + r;
                for (int c = 0; c < Cch; ++c) {
                    const double g = dtail_out[((int64_t)bi * 3 + r) * Cch + c];
                    if (at >= 0) dub[at * Cch + c] += g;
                    else dtb[(3 + at) * Cch + c] += g;
                }
            }
        }
        for (int64_t k = n_cells - 1; k >= 0; --k) {
            const int64_t t0 = k * cell;
            const int64_t t1 = (t0 + cell < L) ? t0 + cell : L;
            const int64_t nt = t1 - t0;
            /* the cell's conv buffer: the 3 rows of u before it */
            for (int r = 0; r < 3; ++r)
                for (int c = 0; c < Cch; ++c) {
                    double val = 0.0;
                    if (k == 0) val = tail_in ? (double)tail_in[((int64_t)bi * 3 + r) * Cch + c] : 0.0;
                    else val = conv_ckpt[(((int64_t)bi * n_ckpt + (k - 1)) * 3 + r) * Cch + c];
                    ext[r * Cch + c] = val;
                }
            /* conv + SiLU of the cell from its own rows and its buffer */
            for (int64_t t = t0; t < t1; ++t)
                for (int c = 0; c < Cch; ++c) {
                    double zz = bias ? (double)bias[c] : 0.0;
                    for (int kk = 0; kk < ORACLE_CONV_K; ++kk) {
                        const int64_t tt = t - (ORACLE_CONV_K - 1) + kk;
                        const double val = tt >= t0 ? (double)ub[tt * Cch + c] : ext[(3 + tt - t0) * Cch + c];
                        zz += (double)w[c * ORACLE_CONV_K + kk] * val;
                    }
                    z[(t - t0) * Cch + c] = zz;
                    v[(t - t0) * Cch + c] = round_io(zz / (1.0 + exp(-zz)), io_round);
                    dv[(t - t0) * Cch + c] = 0.0;
                }
            /* each head: its states over the cell from the cell's starting state, then the reverse sweep */
            for (int h = 0; h < H; ++h) {
                const int grp = (int)((int64_t)h * G / H);
                const double Ah = A[h];
                const double Dh = D ? (double)D[h] : 0.0;
                double *sth = st + (int64_t)h * (cell + 1) * PN;
                double *Gh = Gs + (int64_t)h * PN;
                for (int64_t i = 0; i < PN; ++i) {
                    if (k == 0) sth[i] = h0 ? h0[((int64_t)bi * H + h) * PN + i] : 0.0;
                    else sth[i] = h_ckpt[(((int64_t)bi * n_ckpt + (k - 1)) * H + h) * PN + i];
                }
                for (int64_t j = 0; j < nt; ++j) {
                    const double *xt = v + j * Cch + (int64_t)h * P;
                    const double *Bt = v + j * Cch + HP + (int64_t)grp * N;
                    const double dtv = dt[((int64_t)bi * L + t0 + j) * H + h];
                    const double a_s = exp(dtv * Ah);
                    const double *prev = sth + j * PN;
                    double *cur = sth + (j + 1) * PN;
                    for (int p = 0; p < P; ++p)
                        for (int n = 0; n < N; ++n)
                            cur[(int64_t)p * N + n] = a_s * prev[(int64_t)p * N + n] + dtv * xt[p] * Bt[n];
                }
                for (int64_t j = nt - 1; j >= 0; --j) {
                    const int64_t t = t0 + j;
                    const double *xt = v + j * Cch + (int64_t)h * P;
                    const double *Bt = v + j * Cch + HP + (int64_t)grp * N;
                    const double *Ct = v + j * Cch + HP + GN + (int64_t)grp * N;
                    const double dtv = dt[((int64_t)bi * L + t) * H + h];
                    const double a_t = exp(dtv * Ah);
                    const double *dyt = dy ? dy + (((int64_t)bi * L + t) * H + h) * P : NULL;
                    const double *hprev = sth + j * PN;
                    const double *hcur = sth + (j + 1) * PN;
                    if (dyt)
                        for (int p = 0; p < P; ++p)
                            for (int n = 0; n < N; ++n) Gh[(int64_t)p * N + n] += dyt[p] * Ct[n];
                    double *dvt = dv + j * Cch;
                    for (int n = 0; n < N; ++n) {
                        double c_acc = 0.0, b_acc = 0.0;
                        for (int p = 0; p < P; ++p) {
                            if (dyt) c_acc += hcur[(int64_t)p * N + n] * dyt[p];
                            b_acc += Gh[(int64_t)p * N + n] * xt[p];
                        }
                        dvt[HP + GN + grp * N + n] += c_acc;
                        dvt[HP + grp * N + n] += dtv * b_acc;
                    }
                    double ddt_acc = 0.0, dA_t = 0.0;
                    for (int p = 0; p < P; ++p) {
                        double acc = 0.0;
                        for (int n = 0; n < N; ++n) {
                            const double gv = Gh[(int64_t)p * N + n];
                            acc += gv * Bt[n];
                            ddt_acc += gv * (xt[p] * Bt[n]);
                            dA_t += gv * a_t * hprev[(int64_t)p * N + n];
                        }
                        const double dyp = dyt ? dyt[p] : 0.0;
                        dvt[h * P + p] = Dh * dyp + dtv * acc;
                        dD_acc[h] += dyp * xt[p];
                    }
                    ddt[((int64_t)bi * L + t) * H + h] = Ah * dA_t + ddt_acc;
                    dA_acc[h] += dtv * dA_t;
                    for (int64_t i = 0; i < PN; ++i) Gh[i] *= a_t;
                }
            }
            /* conv + SiLU, reverse, tokens of the cell from the last */
            for (int64_t j = nt - 1; j >= 0; --j) {
                const int64_t t = t0 + j;
                for (int c = 0; c < Cch; ++c) {
                    const double zz = z[j * Cch + c];
                    const double sg = 1.0 / (1.0 + exp(-zz));
                    const double dz = dv[j * Cch + c] * (sg * (1.0 + zz * (1.0 - sg)));
                    dbb[c] += dz;
                    for (int kk = ORACLE_CONV_K - 1; kk >= 0; --kk) {
                        const int64_t tt = t - (ORACLE_CONV_K - 1) + kk;
                        const double val = tt >= t0 ? (double)ub[tt * Cch + c] : ext[(3 + tt - t0) * Cch + c];
                        const double wv = w[c * ORACLE_CONV_K + kk];
                        dwb[c * ORACLE_CONV_K + kk] += dz * val;
                        if (tt >= 0) dub[tt * Cch + c] += wv * dz;   /* a row of this cell or of the one before */
                        else dtb[(3 + tt) * Cch + c] += wv * dz;
                    }
                }
            }
        }
        for (int h = 0; h < H; ++h) {
            dA_b[(int64_t)bi * H + h] = dA_acc[h];
            dD_b[(int64_t)bi * H + h] = dD_acc[h];
            if (dh0) memcpy(dh0 + ((int64_t)bi * H + h) * PN, Gs + (int64_t)h * PN, sizeof(double) * (size_t)PN);
        }
        free(z); free(v); free(dv); free(ext); free(st); free(Gs); free(dA_acc); free(dD_acc);
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
