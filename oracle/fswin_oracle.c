/*
 * fp64 CPU oracle for FlashSwin windowed attention with window-local 2D RoPE.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call
 * this file; only the test suite, the smoke check and the CPU-baseline leg of the
 * benchmark use it.  It shares no code with the CUDA library.
 *
 * What it computes is the plain definition of the method described in
 * "FLASHSWIN: Unlocking Large Windows and Dense Tokens in Swin Vision Transformers
 * with Memory Efficient Attention" (arxivdaily.com/papers/2610.04664, English
 * abstract; thelatestinai.com/papers/2610.04664, Figure 1B and Figure S4):
 * exact softmax attention inside every M x M window of a cyclically shifted
 * token grid, with the queries and keys rotated by a window-local learnable 2D
 * RoPE whose inverse frequencies are theta.  "Exact" means the result has a plain
 * definition, so every step below is that definition written out, one query row
 * at a time, in double precision.
 *
 * Readings where the pages are silent (each one is also listed in the design
 * notes of the repository):
 *  - softmax scale 1/sqrt(d);
 *  - RoPE pairs are adjacent channels (2k, 2k+1); the first d/2 channels rotate
 *    with the in-window column j (x axis, theta[h][0][k]), the last d/2 with the
 *    in-window row i (y axis, theta[h][1][k]); positions are 0..M-1 in the rolled
 *    frame;
 *  - the cyclic shift takes rolled token (r, c) from original position
 *    ((r+s) mod H, (c+s) mod W) and writes outputs back there;
 *  - with s > 0, query and key attend only when their region labels agree:
 *    label = 3*l(r) + l(c), l(x) = 0 for x < X-M, 1 for x < X-s, 2 otherwise;
 *    masked scores are -infinity (never an additive constant);
 *  - log-sum-exp is the natural logarithm;
 *  - a grid whose H or W is not a multiple of M is first padded at the bottom
 *    and right to Hp = ceil(H/M)*M, Wp = ceil(W/M)*M with zero tokens (zero q,
 *    k, v and upstream gradient), as a Swin layer pads its input before the
 *    shift; the roll, the windows and the region labels then refer to the
 *    padded grid, padded tokens take part in the softmax like any other token,
 *    and only the H x W real positions are written back.
 *
 * Gradients are those of L = sum(O * dO) for the upstream gradient dO.
 *
 * Optional low-rank additive bias (the FlashBias-T variant of the same pages:
 * thelatestinai.com/papers/2610.04664, Table 2 and Table S1 captions, "a
 * trainable rank-16 bias factorization" whose parameters grow with M).  Reading
 * where the pages are silent: per head h the bias of the window's N x N
 * (query position, key position) pairs is U_h W_h^T with U_h, W_h of shape
 * [N][rank], N = M*M, positions t = i*M + j in the rolled frame, shared by every
 * window of the batch like Swin's relative position bias; it is added to the
 * scaled score before the shift mask, so S_tu = scale q'_t.k'_u + U_t.W_u.  Its
 * gradients are dU_t = sum dS_tu W_u and dW_u = sum dS_tu U_t, summed over every
 * window of the batch (padded tokens of a padded grid included, as in the
 * softmax).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int B, H, W, heads, d, M, s;
} fso_shape;

/* Input tensors are either raw bf16 bit patterns (upcast exactly) or doubles. */
enum { FSO_BF16 = 0, FSO_F64 = 1 };

typedef struct {
    const void* p;
    int dtype;
} fso_in;

static double fso_load(fso_in x, int64_t i) {
    if (x.dtype == FSO_F64) return ((const double*)x.p)[i];
    uint32_t bits = ((uint32_t)((const uint16_t*)x.p)[i]) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* Region index of one axis coordinate x in the rolled frame (extent X). */
int fso_axis_region(int X, int M, int s, int x) {
    if (s == 0) return 0;
    if (x < X - M) return 0;
    if (x < X - s) return 1;
    return 2;
}

/* Fills out[H*W] with the region label of every rolled token. */
int fso_labels(int H, int W, int M, int s, int* out) {
    for (int r = 0; r < H; ++r)
        for (int c = 0; c < W; ++c)
            out[r * W + c] = 3 * fso_axis_region(H, M, s, r) + fso_axis_region(W, M, s, c);
    return 0;
}

int fso_check_shape(const fso_shape* sh) {
    if (!sh) return 1;
    if (sh->B < 0 || sh->H <= 0 || sh->W <= 0 || sh->heads <= 0 || sh->d <= 0 || sh->M <= 0) return 2;
    if (sh->d % 4) return 2;
    if (sh->H < sh->M || sh->W < sh->M) return 2;
    if (sh->s < 0 || sh->s >= sh->M) return 2;
    return 0;
}

/* Rotate the channel pairs of one token vector x (length d) in place by the
 * angles pos_x * theta_h[0][k] (first half) and pos_y * theta_h[1][k] (second half). */
static void rope_rotate(double* x, int d, int pos_x, int pos_y, const double* theta_h, int inverse) {
    int q = d / 4;
    for (int ax = 0; ax < 2; ++ax) {
        int base = ax == 0 ? 0 : d / 2;
        int pos = ax == 0 ? pos_x : pos_y;
        for (int k = 0; k < q; ++k) {
            double phi = (double)pos * theta_h[ax * q + k];
            double cs = cos(phi), sn = sin(phi);
            if (inverse) sn = -sn;
            double a = x[base + 2 * k], b = x[base + 2 * k + 1];
            x[base + 2 * k] = a * cs - b * sn;
            x[base + 2 * k + 1] = a * sn + b * cs;
        }
    }
}

/* Low-rank bias factors: u, w [heads][M*M][rank]; u == NULL: no bias. */
typedef struct {
    const double *u, *w;
    int rank;
} fso_bias;

typedef struct {
    const fso_shape* sh;
    fso_in q, k, v, dout;
    const double* theta;
    fso_bias bias;
    const int64_t* units;
    int64_t n_units;
    double *o, *lse, *dq, *dk, *dv, *dth, *du, *dw;
    int tid, nthreads;
    int status;
} fso_job;

/* Padded grid extent: X rounded up to a multiple of M. */
static int fso_padded(int X, int M) { return (X + M - 1) / M * M; }

/* One (batch, window, head) unit.  Outputs are in window-local token order
 * t = i*M + j (padded tokens included). */
static int fso_one_unit(const fso_job* jb, int64_t unit, double* o, double* lse, double* dq, double* dk,
                        double* dv, double* dth, double* du, double* dw) {
    const fso_shape* sh = jb->sh;
    const int H = sh->H, W = sh->W, heads = sh->heads, d = sh->d, M = sh->M, s = sh->s;
    const int Hp = fso_padded(H, M), Wp = fso_padded(W, M);
    const int nWw = Wp / M, nW = (Hp / M) * nWw, N = M * M;
    const int64_t b = unit / ((int64_t)nW * heads);
    const int64_t rem = unit % ((int64_t)nW * heads);
    const int w = (int)(rem / heads), h = (int)(rem % heads);
    if (b < 0 || b >= sh->B) return 3;
    const int wr = w / nWw, wc = w % nWw;
    const double* th = jb->theta + (int64_t)h * 2 * (d / 4);
    const double scale = 1.0 / sqrt((double)d);
    const int bwd = jb->dout.p != NULL && dq != NULL;
    const int rank = jb->bias.u ? jb->bias.rank : 0;
    const double* ub = rank ? jb->bias.u + (int64_t)h * N * rank : NULL; /* this head's factors */
    const double* wb = rank ? jb->bias.w + (int64_t)h * N * rank : NULL;

    double* buf = (double*)calloc((size_t)N * d * 6 + (size_t)N * 3, sizeof(double));
    if (!buf) return 4;
    double *qr = buf, *kr = qr + (size_t)N * d, *vv = kr + (size_t)N * d, *go = vv + (size_t)N * d;
    double *dqr = go + (size_t)N * d, *dkr = dqr + (size_t)N * d;
    double *srow = dkr + (size_t)N * d, *prow = srow + N;
    int* lab = (int*)(prow + N);
    if (bwd) memset(dv, 0, sizeof(double) * (size_t)N * d);
    if (bwd && rank) {
        memset(du, 0, sizeof(double) * (size_t)N * rank);
        memset(dw, 0, sizeof(double) * (size_t)N * rank);
    }

    /* Step 1: roll and partition; step 2: rotate q and k. */
    for (int t = 0; t < N; ++t) {
        int i = t / M, j = t % M;
        int r = wr * M + i, c = wc * M + j;
        int ro = (r + s) % Hp, co = (c + s) % Wp;
        if (ro < H && co < W) { /* a padded token keeps the zeros of calloc */
            int64_t base = ((((int64_t)b * H + ro) * W + co) * heads + h) * d;
            for (int e = 0; e < d; ++e) {
                qr[(size_t)t * d + e] = fso_load(jb->q, base + e);
                kr[(size_t)t * d + e] = fso_load(jb->k, base + e);
                vv[(size_t)t * d + e] = fso_load(jb->v, base + e);
                if (bwd) go[(size_t)t * d + e] = fso_load(jb->dout, base + e);
            }
        }
        rope_rotate(qr + (size_t)t * d, d, j, i, th, 0);
        rope_rotate(kr + (size_t)t * d, d, j, i, th, 0);
        lab[t] = 3 * fso_axis_region(Hp, M, s, r) + fso_axis_region(Wp, M, s, c);
    }

    /* Steps 3-5, one query row at a time. */
    for (int t = 0; t < N; ++t) {
        double mx = -INFINITY;
        for (int u = 0; u < N; ++u) {
            if (s > 0 && lab[t] != lab[u]) {
                srow[u] = -INFINITY;
                continue;
            }
            double acc = 0.0, bias = 0.0;
            for (int e = 0; e < d; ++e) acc += qr[(size_t)t * d + e] * kr[(size_t)u * d + e];
            for (int x = 0; x < rank; ++x) bias += ub[(size_t)t * rank + x] * wb[(size_t)u * rank + x];
            srow[u] = scale * acc + bias;
            if (srow[u] > mx) mx = srow[u];
        }
        double sum = 0.0;
        for (int u = 0; u < N; ++u) sum += srow[u] == -INFINITY ? 0.0 : exp(srow[u] - mx);
        double l = mx + log(sum);
        lse[t] = l;
        for (int u = 0; u < N; ++u) prow[u] = srow[u] == -INFINITY ? 0.0 : exp(srow[u] - l);
        double* ot = o + (size_t)t * d;
        for (int e = 0; e < d; ++e) ot[e] = 0.0;
        for (int u = 0; u < N; ++u)
            if (prow[u] != 0.0)
                for (int e = 0; e < d; ++e) ot[e] += prow[u] * vv[(size_t)u * d + e];
        if (!bwd) continue;
        double Dt = 0.0;
        for (int e = 0; e < d; ++e) Dt += go[(size_t)t * d + e] * ot[e];
        for (int u = 0; u < N; ++u) {
            if (srow[u] == -INFINITY) continue;
            double dp = 0.0;
            for (int e = 0; e < d; ++e) dp += go[(size_t)t * d + e] * vv[(size_t)u * d + e];
            double ds = prow[u] * (dp - Dt);
            for (int e = 0; e < d; ++e) {
                dqr[(size_t)t * d + e] += scale * ds * kr[(size_t)u * d + e];
                dkr[(size_t)u * d + e] += scale * ds * qr[(size_t)t * d + e];
                dv[(size_t)u * d + e] += prow[u] * go[(size_t)t * d + e];
            }
            for (int x = 0; x < rank; ++x) {
                du[(size_t)t * rank + x] += ds * wb[(size_t)u * rank + x];
                dw[(size_t)u * rank + x] += ds * ub[(size_t)t * rank + x];
            }
        }
    }

    if (bwd) {
        /* d theta from the rotated vectors and their gradients, then undo the rotation. */
        const int qq = d / 4;
        for (int x = 0; x < 2 * qq; ++x) dth[x] = 0.0;
        for (int t = 0; t < N; ++t) {
            int i = t / M, j = t % M;
            for (int ax = 0; ax < 2; ++ax) {
                int base = ax == 0 ? 0 : d / 2;
                int pos = ax == 0 ? j : i;
                for (int k = 0; k < qq; ++k) {
                    size_t a = (size_t)t * d + base + 2 * k, bb = a + 1;
                    double g = (dqr[bb] * qr[a] - dqr[a] * qr[bb]) + (dkr[bb] * kr[a] - dkr[a] * kr[bb]);
                    dth[ax * qq + k] += (double)pos * g;
                }
            }
            for (int e = 0; e < d; ++e) {
                dq[(size_t)t * d + e] = dqr[(size_t)t * d + e];
                dk[(size_t)t * d + e] = dkr[(size_t)t * d + e];
            }
            rope_rotate(dq + (size_t)t * d, d, j, i, th, 1);
            rope_rotate(dk + (size_t)t * d, d, j, i, th, 1);
        }
    }
    free(buf);
    return 0;
}

static void* fso_worker(void* arg) {
    fso_job* jb = (fso_job*)arg;
    const fso_shape* sh = jb->sh;
    const size_t N = (size_t)sh->M * sh->M, d = (size_t)sh->d, q = (size_t)sh->d / 4;
    const size_t rk = jb->bias.u ? (size_t)jb->bias.rank : 0;
    for (int64_t n = jb->tid; n < jb->n_units; n += jb->nthreads) {
        int st = fso_one_unit(jb, jb->units[n], jb->o + n * N * d, jb->lse + n * N,
                              jb->dq ? jb->dq + n * N * d : NULL, jb->dk ? jb->dk + n * N * d : NULL,
                              jb->dv ? jb->dv + n * N * d : NULL, jb->dth ? jb->dth + n * 2 * q : NULL,
                              jb->du ? jb->du + n * N * rk : NULL, jb->dw ? jb->dw + n * N * rk : NULL);
        if (st) {
            jb->status = st;
            break;
        }
    }
    return NULL;
}

/*
 * Forward (and, when dout and dq/dk/dv/dth are all non-NULL, backward) for a list
 * of units.  unit = (b*nW + w)*heads + h with windows w = wr*(Wp/M) + wc in the
 * rolled frame of the padded grid.  Per unit outputs, window-local token order t = i*M + j:
 *   o, dq, dk, dv: [n_units][M*M][d];  lse: [n_units][M*M];
 *   dth: [n_units][2][d/4], this unit's share of d theta for its head;
 *   du, dw: [n_units][M*M][rank], the unit's shares of the bias gradients (with a bias).
 */
int fso_units(const fso_shape* sh, fso_in q, fso_in k, fso_in v, fso_in dout, const double* theta,
              fso_bias bias, const int64_t* units, int64_t n_units, double* o, double* lse, double* dq, double* dk,
              double* dv, double* dth, double* du, double* dw, int nthreads) {
    int st = fso_check_shape(sh);
    if (st) return st;
    if (bias.u && (!bias.w || bias.rank < 1)) return 2;
    if (bias.u && dq && (!du || !dw)) return 1;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    pthread_t tids[256];
    fso_job jobs[256];
    for (int t = 0; t < nthreads; ++t) {
        fso_job jb = {sh, q, k, v, dout, theta, bias, units, n_units, o, lse, dq, dk, dv, dth, du, dw, t, nthreads, 0};
        jobs[t] = jb;
    }
    if (nthreads == 1) {
        fso_worker(&jobs[0]);
        return jobs[0].status;
    }
    for (int t = 0; t < nthreads; ++t) pthread_create(&tids[t], NULL, fso_worker, &jobs[t]);
    for (int t = 0; t < nthreads; ++t) pthread_join(tids[t], NULL);
    for (int t = 0; t < nthreads; ++t)
        if (jobs[t].status) return jobs[t].status;
    return 0;
}

/*
 * Whole-tensor forward/backward.  Outputs at original token positions (padded
 * tokens are dropped):
 *   o, dq, dk, dv: [B][H][W][heads][d];  lse: [B][H][W][heads];
 *   dtheta: [heads][2][d/4], summed over units in increasing unit order;
 *   du, dw: [heads][M*M][rank] with a bias, summed over units in the same order.
 * Backward outputs may be NULL (forward only).
 */
int fso_full(const fso_shape* sh, fso_in q, fso_in k, fso_in v, fso_in dout, const double* theta, fso_bias bias,
             double* o, double* lse, double* dq, double* dk, double* dv, double* dtheta, double* du, double* dw,
             int nthreads) {
    int st = fso_check_shape(sh);
    if (st) return st;
    if (bias.u && (!bias.w || bias.rank < 1)) return 2;
    const int H = sh->H, W = sh->W, heads = sh->heads, d = sh->d, M = sh->M, s = sh->s;
    const int Hp = fso_padded(H, M), Wp = fso_padded(W, M);
    const int nWw = Wp / M, nW = (Hp / M) * nWw, N = M * M, qq = d / 4;
    const int64_t n_units = (int64_t)sh->B * nW * heads;
    const int bwd = dout.p != NULL && dq && dk && dv && dtheta && (!bias.u || (du && dw));
    const int rk = bias.u ? bias.rank : 0;
    int64_t* units = (int64_t*)malloc(sizeof(int64_t) * (size_t)(n_units > 0 ? n_units : 1));
    double* uo = (double*)calloc((size_t)(n_units > 0 ? n_units : 1) * N * d, sizeof(double));
    double* ul = (double*)calloc((size_t)(n_units > 0 ? n_units : 1) * N, sizeof(double));
    double *udq = NULL, *udk = NULL, *udv = NULL, *uth = NULL, *udu = NULL, *udw = NULL;
    if (bwd && rk) {
        udu = (double*)calloc((size_t)(n_units > 0 ? n_units : 1) * N * rk, sizeof(double));
        udw = (double*)calloc((size_t)(n_units > 0 ? n_units : 1) * N * rk, sizeof(double));
        if (!udu || !udw) {
            st = 4;
            goto done;
        }
    }
    if (bwd) {
        udq = (double*)calloc((size_t)(n_units > 0 ? n_units : 1) * N * d, sizeof(double));
        udk = (double*)calloc((size_t)(n_units > 0 ? n_units : 1) * N * d, sizeof(double));
        udv = (double*)calloc((size_t)(n_units > 0 ? n_units : 1) * N * d, sizeof(double));
        uth = (double*)calloc((size_t)(n_units > 0 ? n_units : 1) * 2 * qq, sizeof(double));
    }
    if (!units || !uo || !ul || (bwd && (!udq || !udk || !udv || !uth))) {
        st = 4;
        goto done;
    }
    for (int64_t n = 0; n < n_units; ++n) units[n] = n;
    st = fso_units(sh, q, k, v, bwd ? dout : (fso_in){NULL, 0}, theta, bias, units, n_units, uo, ul, udq, udk, udv,
                   uth, udu, udw, nthreads);
    if (st) goto done;
    for (int64_t n = 0; n < n_units; ++n) {
        int64_t b = n / ((int64_t)nW * heads), rem = n % ((int64_t)nW * heads);
        int w = (int)(rem / heads), h = (int)(rem % heads);
        int wr = w / nWw, wc = w % nWw;
        for (int t = 0; t < N; ++t) {
            int ro = (wr * M + t / M + s) % Hp, co = (wc * M + t % M + s) % Wp;
            if (ro >= H || co >= W) continue;
            int64_t tok = (((int64_t)b * H + ro) * W + co) * heads + h;
            lse[tok] = ul[(size_t)n * N + t];
            for (int e = 0; e < d; ++e) {
                size_t src = ((size_t)n * N + t) * d + e;
                o[tok * d + e] = uo[src];
                if (bwd) {
                    dq[tok * d + e] = udq[src];
                    dk[tok * d + e] = udk[src];
                    dv[tok * d + e] = udv[src];
                }
            }
        }
    }
    if (bwd) {
        for (int x = 0; x < heads * 2 * qq; ++x) dtheta[x] = 0.0;
        for (int64_t n = 0; n < n_units; ++n) {
            int h = (int)((n % ((int64_t)nW * heads)) % heads);
            for (int x = 0; x < 2 * qq; ++x) dtheta[h * 2 * qq + x] += uth[(size_t)n * 2 * qq + x];
        }
    }
    if (bwd && rk) {
        for (int64_t x = 0; x < (int64_t)heads * N * rk; ++x) du[x] = dw[x] = 0.0;
        for (int64_t n = 0; n < n_units; ++n) {
            int h = (int)((n % ((int64_t)nW * heads)) % heads);
            for (int64_t x = 0; x < (int64_t)N * rk; ++x) {
                du[(int64_t)h * N * rk + x] += udu[(size_t)n * N * rk + x];
                dw[(int64_t)h * N * rk + x] += udw[(size_t)n * N * rk + x];
            }
        }
    }
done:
    free(units);
    free(uo);
    free(ul);
    free(udq);
    free(udk);
    free(udv);
    free(uth);
    free(udu);
    free(udw);
    return st;
}
