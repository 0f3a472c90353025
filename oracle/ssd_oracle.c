/*
 * ssd_oracle.c -- plain fp64 CPU oracle of the Mamba-2 selective-SSM layer core.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls
 * this file; only the tests, the package smoke check and the benchmark's CPU
 * baseline leg use it.  It shares no code, header or constant with the CUDA
 * library: it is the token-by-token definition of the layer, written for a
 * reader to check by eye, and deliberately NOT the chunked algorithm.
 *
 * What is computed (all arithmetic in double; inputs arrive already widened):
 *
 *  - Causal depthwise conv1d over the concatenated channels [x | B | C] with a
 *    kernel of 4 taps, plus bias, then SiLU.  "Nemotron-H 스타일 Hybrid
 *    Mamba-Transformer 3B 모델 구현 타당성 분석", table 1.4 (Mamba-2 구성:
 *    conv_kernel 4, activation SiLU, n_groups 8); "Nemotron-Mamba3架构深度解析"
 *    §2.2 (local Conv1D(kernel4) before the selective SSM).
 *  - dt = softplus(dt_raw + dt_bias): the input-dependent step size of the
 *    selective SSM ("EP6. 트랜스포머 대체 신경망 연구" §6 원리 2: A, B, C, Δ
 *    vary with the input token; "Nemotron-Mamba3架构深度解析" §2.2).
 *  - Scalar-per-head transition a = exp(dt * A[h]) times the identity
 *    ("Mamba-3: 추론을 우선한 상태 공간 모델", opening section: Mamba-2 reduced
 *    the diagonal transition to a scalar times the identity).
 *  - State update S[h] <- a * S[h] + dt * x[h] (outer) B[g]  (P x N per head),
 *    read-out y = S[h] . C[g] + D[h] * x[h], gate y * SiLU(z).  Heads share
 *    B and C in groups of H/G contiguous heads (table 1.4, n_groups).
 *  - Decode is the same body for one token, with the conv history taken from
 *    and written back to a rolling 3-column conv state ("Mamba-3" blog: decode
 *    is a fixed-size state update per token; "Bamba-9B" page, 추론 효율성 /
 *    부록: decode is memory-bound).
 *
 * Readings where the pages are silent:
 *  - conv channel order is x, then B (G*N), then C (G*N); tap k=3 multiplies
 *    the current token (causal cross-correlation); history before token 0 is
 *    zero unless an initial conv state is given;
 *  - the D skip uses the post-conv x; no RMSNorm before the gate;
 *  - head h uses group h / (H/G);
 *  - A is the (negative) transition rate itself, not its log.
 *
 * Layouts (row-major, all double):
 *   x, z        [Bt][L][H*P]        dt_raw   [Bt][L][H]
 *   Bm, Cm      [Bt][L][G*N]        A, D, dt_bias [H]
 *   conv_w      [conv_dim][4]       conv_b   [conv_dim]    conv_dim = H*P + 2*G*N
 *   state       [Bt][H][P][N]       conv_state [Bt][conv_dim][3] (oldest first)
 *   y           [Bt][L][H*P]
 */
#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    long batch, seqlen;
    int nheads, headdim, d_state, ngroups;
} oracle_dims;

/* softplus(v) = log(1 + e^v), written so that large v does not overflow. */
static double o_softplus(double v) {
    if (v > 30.0) return v + log1p(exp(-v));
    return log1p(exp(v));
}

/* SiLU(v) = v * sigmoid(v) = v / (1 + e^-v). */
static double o_silu(double v) { return v / (1.0 + exp(-v)); }

/* ---------------------------------------------------------------------------
 * Causal depthwise conv + bias + SiLU of one channel sequence.
 *   in[t]   t = 0..L-1 : the pre-conv channel values
 *   hist[j] j = 0..2   : tokens -3, -2, -1 (NULL = zeros)
 *   out[t] = silu(b + sum_{k=0..3} w[k] * in[t-3+k])
 * Exported on its own so that a test can compare it with a library FIR.
 * ------------------------------------------------------------------------- */
void oracle_conv_silu(long L, const double* in, long in_stride, const double* hist,
                      const double* w, double b, double* out) {
    for (long t = 0; t < L; t++) {
        double acc = b;
        for (int k = 0; k < 4; k++) {
            long s = t - 3 + k;
            double v;
            if (s >= 0) v = in[s * in_stride];
            else v = hist ? hist[s + 3] : 0.0;
            acc += w[k] * v;
        }
        out[t] = o_silu(acc);
    }
}

typedef struct {
    const oracle_dims* d;
    const double *x, *dt_raw, *Bm, *Cm, *z, *A, *D, *dt_bias, *conv_w, *conv_b;
    const double *init_state, *init_conv_state;
    const unsigned char* unit_mask;
    double *y, *final_state;
    int tid, nthreads;
} prefill_job;

/* One (batch b, head h) sequence, token by token. */
static void prefill_unit(const prefill_job* j, long b, int h) {
    const oracle_dims* d = j->d;
    const long L = d->seqlen;
    const int H = d->nheads, P = d->headdim, N = d->d_state, G = d->ngroups;
    const int HP = H * P, GN = G * N;
    const long conv_dim = (long)HP + 2L * GN;
    const int g = h / (H / G);
    const long cx = (long)h * P, cb = HP + (long)g * N, cc = HP + (long)GN + (long)g * N;

    double* ux = malloc(sizeof(double) * (size_t)L * P);
    double* uB = malloc(sizeof(double) * (size_t)L * N);
    double* uC = malloc(sizeof(double) * (size_t)L * N);
    double* S = malloc(sizeof(double) * (size_t)P * N);
    double* tmp = malloc(sizeof(double) * (size_t)L);

    /* post-conv channels used by this head */
    for (int p = 0; p < P; p++) {
        long c = cx + p;
        const double* hist = j->init_conv_state ? j->init_conv_state + ((size_t)b * conv_dim + c) * 3 : NULL;
        oracle_conv_silu(L, j->x + (size_t)b * L * HP + c, HP, hist, j->conv_w + c * 4, j->conv_b[c], tmp);
        for (long t = 0; t < L; t++) ux[t * P + p] = tmp[t];
    }
    for (int n = 0; n < N; n++) {
        long c = cb + n;
        const double* hist = j->init_conv_state ? j->init_conv_state + ((size_t)b * conv_dim + c) * 3 : NULL;
        oracle_conv_silu(L, j->Bm + (size_t)b * L * GN + (size_t)g * N + n, GN, hist, j->conv_w + c * 4,
                         j->conv_b[c], tmp);
        for (long t = 0; t < L; t++) uB[t * N + n] = tmp[t];
        c = cc + n;
        hist = j->init_conv_state ? j->init_conv_state + ((size_t)b * conv_dim + c) * 3 : NULL;
        oracle_conv_silu(L, j->Cm + (size_t)b * L * GN + (size_t)g * N + n, GN, hist, j->conv_w + c * 4,
                         j->conv_b[c], tmp);
        for (long t = 0; t < L; t++) uC[t * N + n] = tmp[t];
    }

    /* S starts at the initial state, or zero */
    for (int i = 0; i < P * N; i++)
        S[i] = j->init_state ? j->init_state[((size_t)b * H + h) * P * N + i] : 0.0;

    for (long t = 0; t < L; t++) {
        const double dt = o_softplus(j->dt_raw[((size_t)b * L + t) * H + h] + j->dt_bias[h]);
        const double a = exp(dt * j->A[h]);
        const double* xt = ux + t * P;
        const double* Bt = uB + t * N;
        const double* Ct = uC + t * N;
        for (int p = 0; p < P; p++) {
            double* Sp = S + (size_t)p * N;
            double acc = 0.0;
            for (int n = 0; n < N; n++) {
                Sp[n] = a * Sp[n] + dt * xt[p] * Bt[n];
                acc += Sp[n] * Ct[n];
            }
            const double yv = acc + j->D[h] * xt[p];
            const double zv = j->z[((size_t)b * L + t) * HP + cx + p];
            j->y[((size_t)b * L + t) * HP + cx + p] = yv * o_silu(zv);
        }
    }
    memcpy(j->final_state + ((size_t)b * H + h) * P * N, S, sizeof(double) * (size_t)P * N);
    free(ux); free(uB); free(uC); free(S); free(tmp);
}

static void* prefill_worker(void* arg) {
    const prefill_job* j = (const prefill_job*)arg;
    const long units = j->d->batch * j->d->nheads;
    for (long u = j->tid; u < units; u += j->nthreads) {
        if (j->unit_mask && !j->unit_mask[u]) continue;
        prefill_unit(j, u / j->d->nheads, (int)(u % j->d->nheads));
    }
    return NULL;
}

/* ---------------------------------------------------------------------------
 * Prefill of Bt sequences of L tokens.
 *   init_state / init_conv_state: NULL means zeros.
 *   unit_mask [Bt*H] (NULL = all): which (b, h) pairs to compute; y and
 *   final_state entries of skipped pairs are left untouched.
 *   conv_state_out [Bt][conv_dim][3] = pre-conv inputs of tokens L-3..L-1
 *   (falling back to the initial conv history when L < 3).
 * Work is split over (b, h) pairs across nthreads POSIX threads.
 * ------------------------------------------------------------------------- */
void oracle_prefill(const oracle_dims* d, const double* x, const double* dt_raw, const double* Bm,
                    const double* Cm, const double* z, const double* A, const double* D,
                    const double* dt_bias, const double* conv_w, const double* conv_b,
                    const double* init_state, const double* init_conv_state,
                    const unsigned char* unit_mask, double* y, double* final_state,
                    double* conv_state_out, int nthreads) {
    const long L = d->seqlen;
    const int H = d->nheads, P = d->headdim, N = d->d_state, G = d->ngroups;
    const int HP = H * P, GN = G * N;
    const long conv_dim = (long)HP + 2L * GN;
    if (nthreads < 1) nthreads = 1;

    if (conv_state_out) {
        for (long b = 0; b < d->batch; b++) {
            for (long c = 0; c < conv_dim; c++) {
                for (int jj = 0; jj < 3; jj++) {
                    long s = L - 3 + jj;
                    double v;
                    if (s >= 0) {
                        if (c < HP) v = x[((size_t)b * L + s) * HP + c];
                        else if (c < HP + GN) v = Bm[((size_t)b * L + s) * GN + (c - HP)];
                        else v = Cm[((size_t)b * L + s) * GN + (c - HP - GN)];
                    } else {
                        v = init_conv_state ? init_conv_state[((size_t)b * conv_dim + c) * 3 + (s + 3)] : 0.0;
                    }
                    conv_state_out[((size_t)b * conv_dim + c) * 3 + jj] = v;
                }
            }
        }
    }

    prefill_job* jobs = malloc(sizeof(prefill_job) * (size_t)nthreads);
    pthread_t* th = malloc(sizeof(pthread_t) * (size_t)nthreads);
    for (int t = 0; t < nthreads; t++) {
        prefill_job j = {d, x, dt_raw, Bm, Cm, z, A, D, dt_bias, conv_w, conv_b,
                         init_state, init_conv_state, unit_mask, y, final_state, t, nthreads};
        jobs[t] = j;
    }
    if (nthreads == 1) {
        prefill_worker(&jobs[0]);
    } else {
        for (int t = 0; t < nthreads; t++) pthread_create(&th[t], NULL, prefill_worker, &jobs[t]);
        for (int t = 0; t < nthreads; t++) pthread_join(th[t], NULL);
    }
    free(jobs); free(th);
}

/* ---------------------------------------------------------------------------
 * One decode step for Bt sequences (one new token each).
 *   x, z [Bt][H*P]; dt_raw [Bt][H]; Bm, Cm [Bt][G*N]
 *   conv_state [Bt][conv_dim][3] in/out; state [Bt][H][P][N] in/out; y [Bt][H*P]
 *   unit_mask as in oracle_prefill (states of skipped pairs are not advanced;
 *   the conv state is always rolled for every channel).
 * Order: (1) every channel's conv output from the window [3 stored columns,
 * new value]; (2) roll the window; (3) per (b, h) the state update and y.
 * ------------------------------------------------------------------------- */
void oracle_decode_step(const oracle_dims* d, const double* x, const double* dt_raw, const double* Bm,
                        const double* Cm, const double* z, const double* A, const double* D,
                        const double* dt_bias, const double* conv_w, const double* conv_b,
                        double* conv_state, double* state, const unsigned char* unit_mask, double* y) {
    const int H = d->nheads, P = d->headdim, N = d->d_state, G = d->ngroups;
    const int HP = H * P, GN = G * N;
    const long conv_dim = (long)HP + 2L * GN;
    double* u = malloc(sizeof(double) * (size_t)conv_dim);

    for (long b = 0; b < d->batch; b++) {
        for (long c = 0; c < conv_dim; c++) {
            double* cs = conv_state + ((size_t)b * conv_dim + c) * 3;
            double xin;
            if (c < HP) xin = x[(size_t)b * HP + c];
            else if (c < HP + GN) xin = Bm[(size_t)b * GN + (c - HP)];
            else xin = Cm[(size_t)b * GN + (c - HP - GN)];
            const double win[4] = {cs[0], cs[1], cs[2], xin};
            double acc = conv_b[c];
            for (int k = 0; k < 4; k++) acc += conv_w[c * 4 + k] * win[k];
            u[c] = o_silu(acc);
            cs[0] = win[1];
            cs[1] = win[2];
            cs[2] = win[3];
        }
        for (int h = 0; h < H; h++) {
            if (unit_mask && !unit_mask[b * H + h]) continue;
            const int g = h / (H / G);
            const double* xt = u + (size_t)h * P;
            const double* Bt = u + HP + (size_t)g * N;
            const double* Ct = u + HP + GN + (size_t)g * N;
            const double dt = o_softplus(dt_raw[(size_t)b * H + h] + dt_bias[h]);
            const double a = exp(dt * A[h]);
            double* S = state + ((size_t)b * H + h) * P * N;
            for (int p = 0; p < P; p++) {
                double acc = 0.0;
                for (int n = 0; n < N; n++) {
                    S[(size_t)p * N + n] = a * S[(size_t)p * N + n] + dt * xt[p] * Bt[n];
                    acc += S[(size_t)p * N + n] * Ct[n];
                }
                const double yv = acc + D[h] * xt[p];
                y[(size_t)b * HP + (size_t)h * P + p] = yv * o_silu(z[(size_t)b * HP + (size_t)h * P + p]);
            }
        }
    }
    free(u);
}

/* ===========================================================================
 * Backward (gradients) of the prefill, for training.
 *
 * "Nemotron-H 스타일 Hybrid Mamba-Transformer 3B 모델 구현 타당성 분석" trains the
 * hybrid from scratch (§3.1, the change list ends with a forward/backward check
 * of the new Mamba-2 layer; §3.2 phase 2 tests the forward/backward pass).  The
 * backward is the reverse-mode derivative of the recurrence above, written as
 * its adjoint recurrence token by token, in double:
 *
 *   loss = sum dy . y + sum d_final . final_state     (d_final may be NULL = 0)
 *
 *   going backward in t, with lam the adjoint of S (starting at d_final):
 *     g      = dy_t * silu(z_t)                   adjoint of yv_t
 *     dz_t   = dy_t * yv_t * silu'(z_t)
 *     lam   += g (outer) C_t                      yv_t = S_t C_t + D x_t
 *     dC_t  += sum_p g[p] S_t[p, :]
 *     dx_t  += D g + dt_t * lam B_t
 *     dB_t  += dt_t * x_t lam
 *     ddt_t += sum_{p,n} lam x_t B_t + (sum lam . S_{t-1}) a_t A
 *     dA    += (sum lam . S_{t-1}) a_t dt_t
 *     dD    += g . x_t
 *     lam    = a_t lam                            S_t = a_t S_{t-1} + dt_t x_t B_t
 *   d_init_state = lam after token 0;
 *   ddt_raw = ddt * sigmoid(dt_raw + dt_bias)     (softplus' = sigmoid);
 *   the conv: the post-conv gradients du of each channel go through SiLU'
 *   (dv = du silu'(v), v the pre-activation) and the taps:
 *     d xBC[s] += w[k] dv[s+3-k],  dw[k] += dv[t] xBC[t-3+k],  db += dv[t],
 *   with xBC[-3..-1] the initial conv history (its gradient d_init_conv_state).
 *
 * The reverse sweep needs S_{t-1} for every t.  It keeps S only at every
 * RECOMP_SEG-th token and recomputes the states inside a segment from that
 * checkpoint (the same forward steps again, so the values are the same).
 *
 * Work is split over (b, group) units, since the heads of a group share B, C
 * and their conv channels; sums over the batch (dA, dD, ddt_bias, dconv_w,
 * dconv_b) are reduced after the threads join, in batch order.
 * ========================================================================= */

#define RECOMP_SEG 64

static double o_sigmoid(double v) { return 1.0 / (1.0 + exp(-v)); }

/* d silu(v) / dv = s (1 + v (1 - s)), s = sigmoid(v). */
static double o_dsilu(double v) {
    const double s = o_sigmoid(v);
    return s * (1.0 + v * (1.0 - s));
}

/* Pre-activation of the causal conv of one channel: v[t] = b + sum_k w[k] in[t-3+k]. */
static void conv_pre(long L, const double* in, long in_stride, const double* hist, const double* w, double b,
                     double* v) {
    for (long t = 0; t < L; t++) {
        double pre = b;
        for (int k = 0; k < 4; k++) {
            long s = t - 3 + k;
            pre += w[k] * (s >= 0 ? in[s * in_stride] : (hist ? hist[s + 3] : 0.0));
        }
        v[t] = pre;
    }
}

/* Backward of one channel's conv + SiLU.  du[t] = gradient of the post-conv
 * value; v[t] its pre-activation.  Writes d_in[t * in_stride] (the pre-conv
 * input's gradient), adds to dw[0..3], db, and writes d_hist[0..2] if given. */
static void conv_backward(long L, const double* in, long in_stride, const double* hist, const double* w,
                          const double* v, const double* du, double* d_in, long d_stride, double* dw, double* db,
                          double* d_hist, double* dv /* scratch [L] */) {
    for (long t = 0; t < L; t++) dv[t] = du[t] * o_dsilu(v[t]);
    for (long s = -3; s < L; s++) {
        double acc = 0.0;
        for (int k = 0; k < 4; k++) {
            long t = s + 3 - k;
            if (t >= 0 && t < L) acc += w[k] * dv[t];
        }
        if (s >= 0) d_in[s * d_stride] = acc;
        else if (d_hist) d_hist[s + 3] = acc;
    }
    for (long t = 0; t < L; t++) {
        *db += dv[t];
        for (int k = 0; k < 4; k++) {
            long s = t - 3 + k;
            dw[k] += dv[t] * (s >= 0 ? in[s * in_stride] : (hist ? hist[s + 3] : 0.0));
        }
    }
}

typedef struct {
    const oracle_dims* d;
    const double *x, *dt_raw, *Bm, *Cm, *z, *A, *D, *dt_bias, *conv_w, *conv_b;
    const double *init_state, *init_conv_state, *dy, *d_final;
    double *dx, *ddt_raw, *dB, *dC, *dz, *d_init_state, *d_init_conv_state;
    /* per-batch partial sums: [batch][H] and [batch][conv_dim][4], [batch][conv_dim] */
    double *pdA, *pdD, *pddt_bias, *pdconv_w, *pdconv_b;
    int tid, nthreads;
} backward_job;

/* One (batch b, group g) unit: every head of the group and the group's channels. */
static void backward_unit(const backward_job* j, long b, int g) {
    const oracle_dims* d = j->d;
    const long L = d->seqlen;
    const int H = d->nheads, P = d->headdim, N = d->d_state, G = d->ngroups;
    const int HP = H * P, GN = G * N, hpg = H / G;
    const long conv_dim = (long)HP + 2L * GN;
    const long nseg = (L + RECOMP_SEG - 1) / RECOMP_SEG;
    const double* xb = j->x + (size_t)b * L * HP;
    const double* Bb = j->Bm + (size_t)b * L * GN + (size_t)g * N;
    const double* Cb = j->Cm + (size_t)b * L * GN + (size_t)g * N;
    const double* hist_b = j->init_conv_state ? j->init_conv_state + (size_t)b * conv_dim * 3 : NULL;
    double* dhist_b = j->d_init_conv_state ? j->d_init_conv_state + (size_t)b * conv_dim * 3 : NULL;

    double* vB = malloc(sizeof(double) * (size_t)L * N);   /* pre-activations, [t][n] */
    double* vC = malloc(sizeof(double) * (size_t)L * N);
    double* uB = malloc(sizeof(double) * (size_t)L * N);   /* post-conv values */
    double* uC = malloc(sizeof(double) * (size_t)L * N);
    double* duB = calloc((size_t)L * N, sizeof(double));   /* their gradients, summed over the group's heads */
    double* duC = calloc((size_t)L * N, sizeof(double));
    double* vx = malloc(sizeof(double) * (size_t)L * P);
    double* ux = malloc(sizeof(double) * (size_t)L * P);
    double* dux = malloc(sizeof(double) * (size_t)L * P);
    double* dtv = malloc(sizeof(double) * (size_t)L);
    double* av = malloc(sizeof(double) * (size_t)L);
    double* ddt = malloc(sizeof(double) * (size_t)L);
    double* ckpt = malloc(sizeof(double) * (size_t)nseg * P * N);      /* S before each segment */
    double* seg = malloc(sizeof(double) * (size_t)(RECOMP_SEG + 1) * P * N); /* S_{t0-1} .. S_{t0+len-1} */
    double* lam = malloc(sizeof(double) * (size_t)P * N);
    double* g_ = malloc(sizeof(double) * (size_t)P);
    double* tmp = malloc(sizeof(double) * (size_t)L);
    double* tmp2 = malloc(sizeof(double) * (size_t)L);
    double* tmp3 = malloc(sizeof(double) * (size_t)L);

    /* post-conv B and C of the group */
    for (int n = 0; n < N; n++) {
        long c = HP + (long)g * N + n;
        conv_pre(L, Bb + n, GN, hist_b ? hist_b + c * 3 : NULL, j->conv_w + c * 4, j->conv_b[c], tmp);
        for (long t = 0; t < L; t++) { vB[t * N + n] = tmp[t]; uB[t * N + n] = o_silu(tmp[t]); }
        c = HP + (long)GN + (long)g * N + n;
        conv_pre(L, Cb + n, GN, hist_b ? hist_b + c * 3 : NULL, j->conv_w + c * 4, j->conv_b[c], tmp);
        for (long t = 0; t < L; t++) { vC[t * N + n] = tmp[t]; uC[t * N + n] = o_silu(tmp[t]); }
    }

    for (int h = g * hpg; h < (g + 1) * hpg; h++) {
        const long cx = (long)h * P;
        for (int p = 0; p < P; p++) {
            long c = cx + p;
            conv_pre(L, xb + c, HP, hist_b ? hist_b + c * 3 : NULL, j->conv_w + c * 4, j->conv_b[c], tmp);
            for (long t = 0; t < L; t++) { vx[t * P + p] = tmp[t]; ux[t * P + p] = o_silu(tmp[t]); }
        }
        for (long t = 0; t < L; t++) {
            dtv[t] = o_softplus(j->dt_bias[h] + j->dt_raw[((size_t)b * L + t) * H + h]);
            av[t] = exp(dtv[t] * j->A[h]);
            ddt[t] = 0.0;
        }
        memset(dux, 0, sizeof(double) * (size_t)L * P);

        /* forward sweep: checkpoints of S before each segment */
        double* S = seg;
        for (int i = 0; i < P * N; i++)
            S[i] = j->init_state ? j->init_state[((size_t)b * H + h) * P * N + i] : 0.0;
        for (long t = 0; t < L; t++) {
            if (t % RECOMP_SEG == 0) memcpy(ckpt + (size_t)(t / RECOMP_SEG) * P * N, S, sizeof(double) * P * N);
            for (int p = 0; p < P; p++)
                for (int n = 0; n < N; n++)
                    S[p * N + n] = av[t] * S[p * N + n] + dtv[t] * ux[t * P + p] * uB[t * N + n];
        }

        /* reverse sweep */
        for (int i = 0; i < P * N; i++)
            lam[i] = j->d_final ? j->d_final[((size_t)b * H + h) * P * N + i] : 0.0;
        double dA_h = 0.0, dD_h = 0.0;
        for (long sg = nseg - 1; sg >= 0; sg--) {
            const long t0 = sg * RECOMP_SEG;
            const long len = (t0 + RECOMP_SEG <= L) ? RECOMP_SEG : L - t0;
            /* seg[i] = S_{t0-1+i}, i = 0..len */
            memcpy(seg, ckpt + (size_t)sg * P * N, sizeof(double) * P * N);
            for (long i = 0; i < len; i++) {
                const long t = t0 + i;
                const double* Sprev = seg + (size_t)i * P * N;
                double* Snew = seg + (size_t)(i + 1) * P * N;
                for (int p = 0; p < P; p++)
                    for (int n = 0; n < N; n++)
                        Snew[p * N + n] = av[t] * Sprev[p * N + n] + dtv[t] * ux[t * P + p] * uB[t * N + n];
            }
            for (long i = len - 1; i >= 0; i--) {
                const long t = t0 + i;
                const double* Sprev = seg + (size_t)i * P * N;
                const double* St = seg + (size_t)(i + 1) * P * N;
                const double* xt = ux + t * P;
                const double* Bt = uB + t * N;
                const double* Ct = uC + t * N;
                for (int p = 0; p < P; p++) {
                    double acc = 0.0;
                    for (int n = 0; n < N; n++) acc += St[p * N + n] * Ct[n];
                    const double yv = j->D[h] * xt[p] + acc;
                    const size_t yi = ((size_t)b * L + t) * HP + cx + p;
                    const double zv = j->z[yi];
                    g_[p] = j->dy[yi] * o_silu(zv);
                    j->dz[yi] = j->dy[yi] * yv * o_dsilu(zv);
                    dD_h += g_[p] * xt[p];
                    dux[t * P + p] += j->D[h] * g_[p];
                }
                for (int p = 0; p < P; p++)
                    for (int n = 0; n < N; n++) {
                        lam[p * N + n] += g_[p] * Ct[n];
                        duC[t * N + n] += g_[p] * St[p * N + n];
                    }
                double dxB = 0.0, lamS = 0.0;
                for (int p = 0; p < P; p++) {
                    double lb = 0.0;
                    for (int n = 0; n < N; n++) {
                        lb += lam[p * N + n] * Bt[n];
                        duB[t * N + n] += dtv[t] * xt[p] * lam[p * N + n];
                        lamS += lam[p * N + n] * Sprev[p * N + n];
                    }
                    dux[t * P + p] += dtv[t] * lb;
                    dxB += xt[p] * lb;
                }
                ddt[t] += dxB + lamS * av[t] * j->A[h];
                dA_h += lamS * av[t] * dtv[t];
                for (int i2 = 0; i2 < P * N; i2++) lam[i2] *= av[t];
            }
        }
        if (j->d_init_state)
            memcpy(j->d_init_state + ((size_t)b * H + h) * P * N, lam, sizeof(double) * P * N);
        j->pdA[(size_t)b * H + h] = dA_h;
        j->pdD[(size_t)b * H + h] = dD_h;
        double dbias = 0.0;
        for (long t = 0; t < L; t++) {
            const size_t i = ((size_t)b * L + t) * H + h;
            const double v = ddt[t] * o_sigmoid(j->dt_raw[i] + j->dt_bias[h]);
            j->ddt_raw[i] = v;
            dbias += v;
        }
        j->pddt_bias[(size_t)b * H + h] = dbias;

        /* the head's x channels through the conv */
        for (int p = 0; p < P; p++) {
            const long c = cx + p;
            for (long t = 0; t < L; t++) { tmp[t] = vx[t * P + p]; tmp2[t] = dux[t * P + p]; }
            double* dw = j->pdconv_w + ((size_t)b * conv_dim + c) * 4;
            double* db = j->pdconv_b + (size_t)b * conv_dim + c;
            conv_backward(L, xb + c, HP, hist_b ? hist_b + c * 3 : NULL, j->conv_w + c * 4, tmp, tmp2,
                          j->dx + (size_t)b * L * HP + c, HP, dw, db, dhist_b ? dhist_b + c * 3 : NULL, tmp3);
        }
    }

    /* the group's B and C channels through the conv */
    for (int n = 0; n < N; n++) {
        for (int which = 0; which < 2; which++) {
            const long c = HP + (long)which * GN + (long)g * N + n;
            const double* v = which ? vC : vB;
            const double* du = which ? duC : duB;
            for (long t = 0; t < L; t++) { tmp[t] = v[t * N + n]; tmp2[t] = du[t * N + n]; }
            const double* in = (which ? Cb : Bb) + n;
            double* d_in = (which ? j->dC : j->dB) + (size_t)b * L * GN + (size_t)g * N + n;
            double* dw = j->pdconv_w + ((size_t)b * conv_dim + c) * 4;
            double* db = j->pdconv_b + (size_t)b * conv_dim + c;
            conv_backward(L, in, GN, hist_b ? hist_b + c * 3 : NULL, j->conv_w + c * 4, tmp, tmp2, d_in, GN, dw,
                          db, dhist_b ? dhist_b + c * 3 : NULL, tmp3);
        }
    }

    free(vB); free(vC); free(uB); free(uC); free(duB); free(duC); free(vx); free(ux); free(dux);
    free(dtv); free(av); free(ddt); free(ckpt); free(seg); free(lam); free(g_); free(tmp); free(tmp2); free(tmp3);
}

static void* backward_worker(void* arg) {
    const backward_job* j = (const backward_job*)arg;
    const long units = j->d->batch * j->d->ngroups;
    for (long u = j->tid; u < units; u += j->nthreads) backward_unit(j, u / j->d->ngroups, (int)(u % j->d->ngroups));
    return NULL;
}

/* ---------------------------------------------------------------------------
 * Gradients of the prefill.  Inputs as oracle_prefill, plus
 *   dy [Bt][L][H*P] (gradient of y) and d_final [Bt][H][P][N] (NULL = zero).
 * Outputs (all written, none accumulated into):
 *   dx, dz [Bt][L][H*P]; ddt_raw [Bt][L][H]; dB, dC [Bt][L][G*N];
 *   dA, dD, ddt_bias [H]; dconv_w [conv_dim][4]; dconv_b [conv_dim];
 *   d_init_state [Bt][H][P][N] and d_init_conv_state [Bt][conv_dim][3]
 *   (each NULL = not wanted; they are the gradients for the given initial
 *   states, or for zero ones when those are NULL).
 * The conv_state output carries no gradient (it is a copy of the inputs).
 * ------------------------------------------------------------------------- */
void oracle_prefill_backward(const oracle_dims* d, const double* x, const double* dt_raw, const double* Bm,
                             const double* Cm, const double* z, const double* A, const double* D,
                             const double* dt_bias, const double* conv_w, const double* conv_b,
                             const double* init_state, const double* init_conv_state, const double* dy,
                             const double* d_final, double* dx, double* ddt_raw, double* dB, double* dC,
                             double* dz, double* dA, double* dD, double* ddt_bias, double* dconv_w,
                             double* dconv_b, double* d_init_state, double* d_init_conv_state, int nthreads) {
    const int H = d->nheads, P = d->headdim, N = d->d_state, G = d->ngroups;
    const long conv_dim = (long)H * P + 2L * G * N;
    const long Bt = d->batch;
    if (nthreads < 1) nthreads = 1;
    double* pdA = calloc((size_t)Bt * H, sizeof(double));
    double* pdD = calloc((size_t)Bt * H, sizeof(double));
    double* pddt_bias = calloc((size_t)Bt * H, sizeof(double));
    double* pdconv_w = calloc((size_t)Bt * conv_dim * 4, sizeof(double));
    double* pdconv_b = calloc((size_t)Bt * conv_dim, sizeof(double));

    backward_job* jobs = malloc(sizeof(backward_job) * (size_t)nthreads);
    pthread_t* th = malloc(sizeof(pthread_t) * (size_t)nthreads);
    for (int t = 0; t < nthreads; t++) {
        backward_job j = {d, x, dt_raw, Bm, Cm, z, A, D, dt_bias, conv_w, conv_b, init_state, init_conv_state,
                          dy, d_final, dx, ddt_raw, dB, dC, dz, d_init_state, d_init_conv_state,
                          pdA, pdD, pddt_bias, pdconv_w, pdconv_b, t, nthreads};
        jobs[t] = j;
    }
    if (nthreads == 1) {
        backward_worker(&jobs[0]);
    } else {
        for (int t = 0; t < nthreads; t++) pthread_create(&th[t], NULL, backward_worker, &jobs[t]);
        for (int t = 0; t < nthreads; t++) pthread_join(th[t], NULL);
    }

    for (int h = 0; h < H; h++) {
        dA[h] = dD[h] = ddt_bias[h] = 0.0;
        for (long b = 0; b < Bt; b++) {
            dA[h] += pdA[(size_t)b * H + h];
            dD[h] += pdD[(size_t)b * H + h];
            ddt_bias[h] += pddt_bias[(size_t)b * H + h];
        }
    }
    for (long c = 0; c < conv_dim; c++) {
        dconv_b[c] = 0.0;
        for (int k = 0; k < 4; k++) dconv_w[c * 4 + k] = 0.0;
        for (long b = 0; b < Bt; b++) {
            dconv_b[c] += pdconv_b[(size_t)b * conv_dim + c];
            for (int k = 0; k < 4; k++) dconv_w[c * 4 + k] += pdconv_w[((size_t)b * conv_dim + c) * 4 + k];
        }
    }
    free(jobs); free(th); free(pdA); free(pdD); free(pddt_bias); free(pdconv_w); free(pdconv_b);
}

/* ===========================================================================
 * MIMO decode step (Mamba-3's multi-input multi-output SSM).
 *
 * "Mamba-3: 추론을 우선한 상태 공간 모델" (opening section, third change; 아키텍처:
 * the MIMO projection widens B and C) replaces the single-input single-output
 * SSM by several SSMs modelled in parallel, at almost no cost to decode
 * latency.  The page gives no equations; the plainest reading, kept on the
 * Mamba-2 scalar decay (the new discretisation and complex states are other
 * changes), is a rank-R input and R read-outs per head:
 *
 *   dt = softplus(dt_raw + dt_bias[h]),  a = exp(dt A[h])
 *   S[h] <- a S[h] + dt sum_{k<R} x_k[h] (outer) B_k[g]
 *   y_k[h] = (S[h] C_k[g] + D[h] x_k[h]) silu(z_k[h])        k = 0..R-1
 *
 * with no short conv (the same page: Mamba-3 drops it).  R = 1 is the Mamba-2
 * decode step without its conv.
 * Layouts: x, z, y [Bt][H][R][P]; dt_raw [Bt][H]; Bm, Cm [Bt][G][R][N];
 * state [Bt][H][P][N] (in/out).
 * ------------------------------------------------------------------------- */
void oracle_mimo_decode_step(const oracle_dims* d, int R, const double* x, const double* dt_raw,
                             const double* Bm, const double* Cm, const double* z, const double* A,
                             const double* D, const double* dt_bias, double* state, double* y) {
    const int H = d->nheads, P = d->headdim, N = d->d_state, G = d->ngroups;
    for (long b = 0; b < d->batch; b++) {
        for (int h = 0; h < H; h++) {
            const int g = h / (H / G);
            const double dt = o_softplus(dt_raw[(size_t)b * H + h] + dt_bias[h]);
            const double a = exp(dt * A[h]);
            double* S = state + ((size_t)b * H + h) * P * N;
            const double* xh = x + ((size_t)b * H + h) * R * P;
            const double* zh = z + ((size_t)b * H + h) * R * P;
            const double* Bg = Bm + ((size_t)b * G + g) * R * N;
            const double* Cg = Cm + ((size_t)b * G + g) * R * N;
            for (int p = 0; p < P; p++) {
                for (int n = 0; n < N; n++) {
                    double in = 0.0;
                    for (int k = 0; k < R; k++) in += xh[k * P + p] * Bg[k * N + n];
                    S[(size_t)p * N + n] = a * S[(size_t)p * N + n] + dt * in;
                }
            }
            for (int k = 0; k < R; k++) {
                for (int p = 0; p < P; p++) {
                    double acc = 0.0;
                    for (int n = 0; n < N; n++) acc += S[(size_t)p * N + n] * Cg[k * N + n];
                    const double yv = acc + D[h] * xh[k * P + p];
                    y[(((size_t)b * H + h) * R + k) * P + p] = yv * o_silu(zh[k * P + p]);
                }
            }
        }
    }
}
