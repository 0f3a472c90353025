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
