/*
 * rodref.c -- plain, slow, obviously-correct CPU oracle for the Rodimus+ token mixers.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may link, load or call this
 * library: only the tests, the smoke check and the benchmark's CPU-baseline leg use it.
 * It shares no code, header, table or helper with the CUDA library.
 *
 * Everything is computed in IEEE double precision with plain loops, in the order the
 * definitions are written. Inputs arrive as float arrays: the GPU path receives bf16 or
 * fp32 values, and every bf16 and fp32 value is exactly representable as a float, so the
 * oracle sees exactly the numbers the kernels see and widens them to double on use.
 * Work is split only across independent units ((batch, head) pairs for the recurrence,
 * output rows for attention) with POSIX threads; each unit is computed sequentially.
 *
 * Sources (web pages; cited by title and section):
 *  [CodeFuse]  "ICLR 2025 | Rodimus*: a hybrid attention mechanism balancing performance and
 *              efficiency" (CodeFuse article): the Rodimus block compresses the history into a
 *              fixed-size hidden state, updated recurrently at inference (O(1) space); SKA shares
 *              one key matrix across all heads and keeps per-head values (Fig. 4 and the SKA
 *              paragraph); Rodimus+ uses SKA inside sliding-window attention (SW-SKA).
 *  [Setup]     "Rodimus* ... what problem does it solve" setup/benchmark blog, §3 (module
 *              config): the sliding window only looks at the most recent 4096 tokens; keys are
 *              shared across heads and values are kept per head.
 *  [SALA]      sparse + linear attention blog: §2.1 sliding-window attention (each query looks
 *              only at recent keys), §2.2 linear attention state O_i = phi(q_i) * sum_j phi(k_j)^T v_j
 *              with a d x d state, §3.3 ring-buffer window cache and in-place state update at
 *              decode, §4.3 first tip (store the KV cache in FP8: half the memory, a faster
 *              decode, at some loss of detail), §4.3 third tip (a decay factor makes old state
 *              weights fall exponentially).
 *
 * Readings taken where the pages are silent or garbled (the DDTS gate equation in [CodeFuse]
 * is stripped from the extracted text):
 *  - the gates g_t are inputs, one per key channel, and decay the ROWS of the d_k x d_v state:
 *        S_t = diag(g_t) S_{t-1} + k_t^T v_t,   o_t = q_t S_t   (readout after the update);
 *    no scale and no normaliser are applied to the recurrence output.
 *  - the window of query t holds W keys including t itself: j in [t-W+1, t], clipped at 0.
 *    W = 1 then gives o_t = v_t and W >= T gives full causal attention.
 *  - softmax attention uses o = sum_j p_j v_j / sum_j p_j with p_j = exp(s_j - max s).
 *  - FP8 window cache ([SALA] §4.3 names FP8 and nothing more): the OCP E4M3 format (1 sign
 *    bit, 4 exponent bits with bias 7, 3 mantissa bits, no infinities, S.1111.111 is NaN, the
 *    largest finite value 448), one fp32 scale per cache, stored code = e4m3(x / scale) with x
 *    and the quotient in fp32 (the precision the kernel decides in), rounded to the nearest
 *    code with ties to the even code and saturated at +-448; the attention reads
 *    value(code) * scale. The new token is written to the cache first and read back like the
 *    other window entries.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define RODREF_OK 0
#define RODREF_EINVAL (-1)
#define RODREF_ENOMEM (-2)

/* ------------------------------------------------------------------------------------------
 * tiny work-splitting helper: run fn(arg, unit) for unit in [0, n_units) on nthreads threads
 * ---------------------------------------------------------------------------------------- */
typedef void (*unit_fn)(const void* arg, int64_t unit);

typedef struct {
    unit_fn fn;
    const void* arg;
    int64_t n_units;
    int tid;
    int nthreads;
} worker_t;

static void* worker_main(void* p) {
    worker_t* w = (worker_t*)p;
    for (int64_t u = w->tid; u < w->n_units; u += w->nthreads) w->fn(w->arg, u);
    return NULL;
}

static int run_units(unit_fn fn, const void* arg, int64_t n_units, int nthreads) {
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    if (n_units < nthreads) nthreads = (int)(n_units > 0 ? n_units : 1);
    if (nthreads == 1) {
        for (int64_t u = 0; u < n_units; ++u) fn(arg, u);
        return RODREF_OK;
    }
    pthread_t th[256];
    worker_t w[256];
    int started = 0;
    for (int i = 0; i < nthreads; ++i) {
        w[i].fn = fn; w[i].arg = arg; w[i].n_units = n_units; w[i].tid = i; w[i].nthreads = nthreads;
        if (pthread_create(&th[i], NULL, worker_main, &w[i]) != 0) break;
        ++started;
    }
    for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
    /* units a failed thread would have taken are done here, sequentially */
    for (int i = started; i < nthreads; ++i) worker_main(&w[i]);
    return RODREF_OK;
}

/* ------------------------------------------------------------------------------------------
 * Gated linear recurrence (the Rodimus semantic-compression state) -- [CodeFuse] Rodimus block
 * (recurrent inference form keeps only a fixed-size state); [SALA] §2.2 (state = sum of k^T v,
 * readout q * state) and §4.3 tip 3 (per-step decay of the old state).
 *
 * One step for one (batch, head):
 *     S[c][j] <- g[c] * S[c][j] + k[c] * v[j]        c < dk, j < dv
 *     o[j]     = sum_c q[c] * S[c][j]                 (S after the update)
 * ---------------------------------------------------------------------------------------- */
static void gla_step(const float* q, const float* k, const float* v, const float* g,
                     double* S, double* o, int64_t dk, int64_t dv) {
    for (int64_t c = 0; c < dk; ++c) {
        const double gc = (double)g[c];
        const double kc = (double)k[c];
        double* row = S + c * dv;
        for (int64_t j = 0; j < dv; ++j) row[j] = gc * row[j] + kc * (double)v[j];
    }
    for (int64_t j = 0; j < dv; ++j) {
        double acc = 0.0;
        for (int64_t c = 0; c < dk; ++c) acc += (double)q[c] * S[c * dv + j];
        o[j] = acc;
    }
}

typedef struct {
    const float *q, *k, *v, *g;
    double *state, *o;
    int64_t T, dk, dv;
} gla_args_t;

/* one unit = one (batch, head) pair, walked sequentially in t */
static void gla_unit(const void* p, int64_t bh) {
    const gla_args_t* a = (const gla_args_t*)p;
    const int64_t T = a->T, dk = a->dk, dv = a->dv;
    double* S = a->state + bh * dk * dv;
    for (int64_t t = 0; t < T; ++t) {
        const int64_t tk = (bh * T + t) * dk, tv = (bh * T + t) * dv;
        gla_step(a->q + tk, a->k + tk, a->v + tv, a->g + tk, S, a->o + tv, dk, dv);
    }
}

/*
 * q, k, g: [B,H,T,dk]; v: [B,H,T,dv] (row-major, contiguous).
 * state: [B,H,dk,dv], read as the initial state and overwritten with the final state.
 * o: [B,H,T,dv].
 */
int rodref_gla_prefill(const float* q, const float* k, const float* v, const float* g,
                       double* state, double* o, int64_t B, int64_t H, int64_t T,
                       int64_t dk, int64_t dv, int nthreads) {
    if (!q || !k || !v || !g || !state || !o) return RODREF_EINVAL;
    if (B < 0 || H < 0 || T < 0 || dk < 1 || dv < 1) return RODREF_EINVAL;
    gla_args_t a = {q, k, v, g, state, o, T, dk, dv};
    return run_units(gla_unit, &a, B * H, nthreads);
}

/* ------------------------------------------------------------------------------------------
 * Backward of the recurrence (the chunkwise-parallel algorithm is stated for training too,
 * [CodeFuse] Rodimus block): reverse-mode differentiation of gla_step, written out.
 * Loss gradients dO_t (of every o_t) and dS_final (of the final state S_T, may be absent).
 *   dq_t[c]  = sum_j dO_t[j] S_t[c][j]                       (S_t after step t)
 *   dS_t     = q_t^T dO_t + diag(g_{t+1}) dS_{t+1},  dS_T starting from dS_final
 *   dk_t[c]  = sum_j dS_t[c][j] v_t[j];   dv_t[j] = sum_c dS_t[c][j] k_t[c]
 *   dg_t[c]  = sum_j dS_t[c][j] S_{t-1}[c][j]
 *   dS_0     = diag(g_1) dS_1  (gradient of the initial state)
 * The states S_{t-1} the reverse sweep needs are recomputed per block of 64 steps from
 * checkpoints saved by the forward sweep.
 * ---------------------------------------------------------------------------------------- */
typedef struct {
    const float *q, *k, *v, *g, *dO, *dSf;
    const double* state0;
    double *dq, *dk, *dv, *dg, *dstate0;
    int64_t T, dk_, dv_;
} gla_bwd_args_t;

#define GLA_BWD_BLOCK 64

static void gla_bwd_unit(const void* p, int64_t bh) {
    const gla_bwd_args_t* a = (const gla_bwd_args_t*)p;
    const int64_t T = a->T, dk = a->dk_, dv = a->dv_, DD = dk * dv;
    const int64_t nblk = (T + GLA_BWD_BLOCK - 1) / GLA_BWD_BLOCK;
    double* ckpt = malloc((size_t)((nblk + 1) * DD) * sizeof(double));
    double* Sb = malloc((size_t)((GLA_BWD_BLOCK + 1) * DD) * sizeof(double));
    double* dS = malloc((size_t)DD * sizeof(double));
    if (!ckpt || !Sb || !dS) { free(ckpt); free(Sb); free(dS); return; }
    /* forward sweep: checkpoints (state before each block) and dq */
    double* S = Sb;
    memcpy(S, a->state0 + bh * DD, (size_t)DD * sizeof(double));
    for (int64_t t = 0; t < T; ++t) {
        if (t % GLA_BWD_BLOCK == 0) memcpy(ckpt + (t / GLA_BWD_BLOCK) * DD, S, (size_t)DD * sizeof(double));
        const int64_t tk = (bh * T + t) * dk, tv = (bh * T + t) * dv;
        for (int64_t c = 0; c < dk; ++c)
            for (int64_t j = 0; j < dv; ++j)
                S[c * dv + j] = (double)a->g[tk + c] * S[c * dv + j] + (double)a->k[tk + c] * (double)a->v[tv + j];
        for (int64_t c = 0; c < dk; ++c) {
            double acc = 0.0;
            for (int64_t j = 0; j < dv; ++j) acc += (double)a->dO[tv + j] * S[c * dv + j];
            a->dq[tk + c] = acc;
        }
    }
    /* reverse sweep */
    for (int64_t i = 0; i < DD; ++i) dS[i] = a->dSf ? (double)a->dSf[bh * DD + i] : 0.0;
    for (int64_t blk = nblk - 1; blk >= 0; --blk) {
        const int64_t t0 = blk * GLA_BWD_BLOCK, t1 = t0 + GLA_BWD_BLOCK < T ? t0 + GLA_BWD_BLOCK : T;
        memcpy(Sb, ckpt + blk * DD, (size_t)DD * sizeof(double));   /* Sb[i] = S before step t0+i */
        for (int64_t t = t0; t < t1; ++t) {
            const double* Sp = Sb + (t - t0) * DD;
            double* Sn = Sb + (t - t0 + 1) * DD;
            const int64_t tk = (bh * T + t) * dk, tv = (bh * T + t) * dv;
            for (int64_t c = 0; c < dk; ++c)
                for (int64_t j = 0; j < dv; ++j)
                    Sn[c * dv + j] = (double)a->g[tk + c] * Sp[c * dv + j] + (double)a->k[tk + c] * (double)a->v[tv + j];
        }
        for (int64_t t = t1 - 1; t >= t0; --t) {
            const double* Sprev = Sb + (t - t0) * DD;
            const int64_t tk = (bh * T + t) * dk, tv = (bh * T + t) * dv;
            for (int64_t c = 0; c < dk; ++c)
                for (int64_t j = 0; j < dv; ++j) dS[c * dv + j] += (double)a->q[tk + c] * (double)a->dO[tv + j];
            for (int64_t c = 0; c < dk; ++c) {
                double acck = 0.0, accg = 0.0;
                for (int64_t j = 0; j < dv; ++j) {
                    acck += dS[c * dv + j] * (double)a->v[tv + j];
                    accg += dS[c * dv + j] * Sprev[c * dv + j];
                }
                a->dk[tk + c] = acck;
                a->dg[tk + c] = accg;
            }
            for (int64_t j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int64_t c = 0; c < dk; ++c) acc += dS[c * dv + j] * (double)a->k[tk + c];
                a->dv[tv + j] = acc;
            }
            for (int64_t c = 0; c < dk; ++c)
                for (int64_t j = 0; j < dv; ++j) dS[c * dv + j] *= (double)a->g[tk + c];
        }
    }
    memcpy(a->dstate0 + bh * DD, dS, (size_t)DD * sizeof(double));
    free(ckpt);
    free(Sb);
    free(dS);
}

/*
 * q, k, g, dq, dk, dg: [B,H,T,dk]; v, dO, dv: [B,H,T,dv]; state0, dstate0: [B,H,dk,dv];
 * dS_final: [B,H,dk,dv] or NULL (no loss on the final state).
 */
int rodref_gla_backward(const float* q, const float* k, const float* v, const float* g,
                        const double* state0, const float* dO, const float* dS_final, double* dq,
                        double* dk_out, double* dv_out, double* dg, double* dstate0, int64_t B,
                        int64_t H, int64_t T, int64_t dk, int64_t dv, int nthreads) {
    if (!q || !k || !v || !g || !state0 || !dO || !dq || !dk_out || !dv_out || !dg || !dstate0)
        return RODREF_EINVAL;
    if (B < 0 || H < 0 || T < 0 || dk < 1 || dv < 1) return RODREF_EINVAL;
    gla_bwd_args_t a = {q, k, v, g, dO, dS_final, state0, dq, dk_out, dv_out, dg, dstate0, T, dk, dv};
    return run_units(gla_bwd_unit, &a, B * H, nthreads);
}

/*
 * One decode step for N sequences: q, k, g: [N,H,dk]; v: [N,H,dv];
 * state [N,H,dk,dv] updated in place; o: [N,H,dv]. Identical to a prefill with T = 1.
 */
int rodref_gla_decode_step(const float* q, const float* k, const float* v, const float* g,
                           double* state, double* o, int64_t N, int64_t H, int64_t dk,
                           int64_t dv, int nthreads) {
    return rodref_gla_prefill(q, k, v, g, state, o, N, H, 1, dk, dv, nthreads);
}

/* ------------------------------------------------------------------------------------------
 * Sliding-window shared-key softmax attention (SW-SKA) -- [CodeFuse] Fig. 4 / SKA paragraph
 * (one K for all heads, per-head V), [Setup] §3 (window = most recent W tokens), [SALA] §2.1.
 *
 * For query t of head h in batch b, with window J_t = [max(0, t-W+1), t]:
 *     s_j = scale * sum_c q[b,h,t,c] * k[b,j,c]
 *     p_j = exp(s_j - max_{j' in J_t} s_j')
 *     o[b,h,t,:] = sum_j p_j v[b,h,j,:] / sum_j p_j
 * and the row's log-sum-exp  lse = log sum_j exp(s_j) = max_j s_j + log sum_j p_j  (natural log),
 * the statistic a backward pass keeps from the forward.
 * ---------------------------------------------------------------------------------------- */
static double softmax_row(const float* qrow, const float* kbase, const float* vbase,
                        int64_t j0, int64_t j1, int64_t dk, int64_t dv, double scale,
                        double* s, double* out) {
    /* kbase row j is kbase + j*dk; vbase row j is vbase + j*dv; keys j0..j1 inclusive */
    double m = -INFINITY;
    for (int64_t j = j0; j <= j1; ++j) {
        double acc = 0.0;
        const float* kr = kbase + j * dk;
        for (int64_t c = 0; c < dk; ++c) acc += (double)qrow[c] * (double)kr[c];
        s[j - j0] = scale * acc;
        if (s[j - j0] > m) m = s[j - j0];
    }
    double l = 0.0;
    for (int64_t i = 0; i < dv; ++i) out[i] = 0.0;
    for (int64_t j = j0; j <= j1; ++j) {
        const double p = exp(s[j - j0] - m);
        l += p;
        const float* vr = vbase + j * dv;
        for (int64_t i = 0; i < dv; ++i) out[i] += p * (double)vr[i];
    }
    for (int64_t i = 0; i < dv; ++i) out[i] /= l;
    return m + log(l);
}

typedef struct {
    const float *q, *k, *v;
    double* o;
    int64_t B, H, T, dk, dv, W;
    double scale;
    const int64_t* rows;
    double* lse; /* optional: one per output row */
} ska_args_t;

static void ska_unit(const void* p, int64_t r) {
    const ska_args_t* a = (const ska_args_t*)p;
    const int64_t flat = a->rows ? a->rows[r] : r; /* ((b*H + h)*T + t) */
    const int64_t t = flat % a->T;
    const int64_t bh = flat / a->T;
    const int64_t b = bh / a->H;
    int64_t j0 = t - a->W + 1;
    if (j0 < 0) j0 = 0;
    double* s = (double*)malloc((size_t)(t - j0 + 1) * sizeof(double));
    if (!s) {
        for (int64_t i = 0; i < a->dv; ++i) a->o[r * a->dv + i] = NAN;
        if (a->lse) a->lse[r] = NAN;
        return;
    }
    const double lse = softmax_row(a->q + flat * a->dk, a->k + b * a->T * a->dk, a->v + bh * a->T * a->dv,
                                   j0, t, a->dk, a->dv, a->scale, s, a->o + r * a->dv);
    if (a->lse) a->lse[r] = lse;
    free(s);
}

/*
 * q: [B,H,T,dk]; k: [B,T,dk] (shared by the H heads); v: [B,H,T,dv].
 * rows == NULL: o is [B,H,T,dv] (every output row), lse (if not NULL) [B,H,T].
 * rows != NULL: o is [n_rows, dv] and lse [n_rows]; row r is output row rows[r] = (b*H + h)*T + t.
 */
int rodref_swska_prefill_lse(const float* q, const float* k, const float* v, double* o, double* lse,
                             int64_t B, int64_t H, int64_t T, int64_t dk, int64_t dv, int64_t W,
                             double scale, const int64_t* rows, int64_t n_rows, int nthreads) {
    if (!q || !k || !v || !o) return RODREF_EINVAL;
    if (B < 0 || H < 0 || T < 0 || dk < 1 || dv < 1 || W < 1) return RODREF_EINVAL;
    const int64_t total = B * H * T;
    if (rows) {
        for (int64_t r = 0; r < n_rows; ++r)
            if (rows[r] < 0 || rows[r] >= total) return RODREF_EINVAL;
    } else {
        n_rows = total;
    }
    ska_args_t a = {q, k, v, o, B, H, T, dk, dv, W, scale, rows, lse};
    return run_units(ska_unit, &a, n_rows, nthreads);
}

/* the same without the log-sum-exp */
int rodref_swska_prefill(const float* q, const float* k, const float* v, double* o,
                         int64_t B, int64_t H, int64_t T, int64_t dk, int64_t dv, int64_t W,
                         double scale, const int64_t* rows, int64_t n_rows, int nthreads) {
    return rodref_swska_prefill_lse(q, k, v, o, NULL, B, H, T, dk, dv, W, scale, rows, n_rows, nthreads);
}

/*
 * SW-SKA decode with a ring-buffer window cache -- [SALA] §3.3 (self-made circular buffer,
 * window rolls at every decode step), [CodeFuse] SKA (one shared K cache per sequence).
 *
 * For each sequence n with new position P = pos[n]:
 *   1. write the new token into slot P mod W:  k_cache[n, P mod W, :] = k_new[n, :],
 *      v_cache[n, h, P mod W, :] = v_new[n, h, :] for every head h;
 *   2. attend over the tokens at positions p = max(0, P-W+1) .. P, whose keys sit in
 *      slot p mod W, with the same softmax as above.
 * q: [N,H,dk]; k_new: [N,dk]; v_new: [N,H,dv]; k_cache: [N,W,dk]; v_cache: [N,H,W,dv];
 * o: [N,H,dv]. The caches are updated in place.
 */
typedef struct {
    const float *q, *k_new, *v_new;
    float *k_cache, *v_cache;
    const int64_t* pos;
    double* o;
    int64_t H, dk, dv, W;
    double scale;
} ska_dec_args_t;

static void ska_dec_unit(const void* p, int64_t nh) {
    const ska_dec_args_t* a = (const ska_dec_args_t*)p;
    const int64_t n = nh / a->H, h = nh % a->H;
    const int64_t P = a->pos[n];
    const int64_t p0 = P - a->W + 1 > 0 ? P - a->W + 1 : 0;
    const int64_t cnt = P - p0 + 1;
    const float* kc = a->k_cache + n * a->W * a->dk;
    const float* vc = a->v_cache + (n * a->H + h) * a->W * a->dv;
    const float* qr = a->q + nh * a->dk;
    double* out = a->o + nh * a->dv;
    double* s = (double*)malloc((size_t)cnt * sizeof(double));
    if (!s) { for (int64_t i = 0; i < a->dv; ++i) out[i] = NAN; return; }
    double m = -INFINITY;
    for (int64_t pp = p0; pp <= P; ++pp) {
        const float* kr = kc + (pp % a->W) * a->dk;
        double acc = 0.0;
        for (int64_t c = 0; c < a->dk; ++c) acc += (double)qr[c] * (double)kr[c];
        s[pp - p0] = a->scale * acc;
        if (s[pp - p0] > m) m = s[pp - p0];
    }
    double l = 0.0;
    for (int64_t i = 0; i < a->dv; ++i) out[i] = 0.0;
    for (int64_t pp = p0; pp <= P; ++pp) {
        const double pr = exp(s[pp - p0] - m);
        l += pr;
        const float* vr = vc + (pp % a->W) * a->dv;
        for (int64_t i = 0; i < a->dv; ++i) out[i] += pr * (double)vr[i];
    }
    for (int64_t i = 0; i < a->dv; ++i) out[i] /= l;
    free(s);
}

int rodref_swska_decode(const float* q, const float* k_new, const float* v_new, float* k_cache,
                        float* v_cache, const int64_t* pos, double* o, int64_t N, int64_t H,
                        int64_t dk, int64_t dv, int64_t W, double scale, int nthreads) {
    if (!q || !k_new || !v_new || !k_cache || !v_cache || !pos || !o) return RODREF_EINVAL;
    if (N < 0 || H < 1 || dk < 1 || dv < 1 || W < 1) return RODREF_EINVAL;
    for (int64_t n = 0; n < N; ++n)
        if (pos[n] < 0) return RODREF_EINVAL;
    /* step 1: ring-buffer write of the new token */
    for (int64_t n = 0; n < N; ++n) {
        const int64_t slot = pos[n] % W;
        memcpy(k_cache + (n * W + slot) * dk, k_new + n * dk, (size_t)dk * sizeof(float));
        for (int64_t h = 0; h < H; ++h)
            memcpy(v_cache + ((n * H + h) * W + slot) * dv, v_new + (n * H + h) * dv,
                   (size_t)dv * sizeof(float));
    }
    /* step 2: attention over the window */
    ska_dec_args_t a = {q, k_new, v_new, k_cache, v_cache, pos, o, H, dk, dv, W, scale};
    return run_units(ska_dec_unit, &a, N * H, nthreads);
}

/* Backward of SW-SKA prefill (training path; same attention as rodref_swska_prefill). For the
 * loss gradient dO of every output row, per (b, h, t) with window J_t and p = softmax(s):
 *   D_t = sum_j p_tj (dO_t . v_j)  (= dO_t . o_t),   dS_tj = p_tj (dO_t . v_j - D_t)
 *   dq_t  = scale sum_j dS_tj k_j
 *   dk_j  = scale sum_h sum_t dS_tj q_t      (one K shared by the heads: summed over them)
 *   dv_j  = sum_t p_tj dO_t                  (per head)
 * Units are (b, h) pairs; each writes its dq and dv and a private dk partial, and the partials
 * are summed over heads afterwards. */
typedef struct {
    const float *q, *k, *v, *dO;
    double *dq, *dkp, *dv;
    int64_t H, T, dk, dv_, W;
    double scale;
} ska_bwd_args_t;

static void ska_bwd_unit(const void* p, int64_t bh) {
    const ska_bwd_args_t* a = (const ska_bwd_args_t*)p;
    const int64_t H = a->H, T = a->T, dk = a->dk, dv = a->dv_, W = a->W, b = bh / H;
    double* s = malloc((size_t)(W + 1) * sizeof(double));
    double* pr = malloc((size_t)(W + 1) * sizeof(double));
    double* dp = malloc((size_t)(W + 1) * sizeof(double));
    double* dkp = a->dkp + bh * T * dk;
    if (!s || !pr || !dp) { free(s); free(pr); free(dp); return; }
    for (int64_t i = 0; i < T * dk; ++i) dkp[i] = 0.0;
    for (int64_t i = 0; i < T * dv; ++i) a->dv[bh * T * dv + i] = 0.0;
    for (int64_t t = 0; t < T; ++t) {
        const int64_t j0 = t - W + 1 > 0 ? t - W + 1 : 0;
        const float* qt = a->q + (bh * T + t) * dk;
        const float* dot = a->dO + (bh * T + t) * dv;
        double m = -INFINITY;
        for (int64_t j = j0; j <= t; ++j) {
            double acc = 0.0;
            for (int64_t c = 0; c < dk; ++c) acc += (double)qt[c] * (double)a->k[(b * T + j) * dk + c];
            s[j - j0] = a->scale * acc;
            if (s[j - j0] > m) m = s[j - j0];
        }
        double l = 0.0;
        for (int64_t j = j0; j <= t; ++j) { pr[j - j0] = exp(s[j - j0] - m); l += pr[j - j0]; }
        double D = 0.0;
        for (int64_t j = j0; j <= t; ++j) {
            pr[j - j0] /= l;
            double acc = 0.0;
            for (int64_t i = 0; i < dv; ++i) acc += (double)dot[i] * (double)a->v[(bh * T + j) * dv + i];
            dp[j - j0] = acc;
            D += pr[j - j0] * acc;
        }
        double* dqt = a->dq + (bh * T + t) * dk;
        for (int64_t c = 0; c < dk; ++c) dqt[c] = 0.0;
        for (int64_t j = j0; j <= t; ++j) {
            const double dS = pr[j - j0] * (dp[j - j0] - D);
            for (int64_t c = 0; c < dk; ++c) {
                dqt[c] += a->scale * dS * (double)a->k[(b * T + j) * dk + c];
                dkp[j * dk + c] += a->scale * dS * (double)qt[c];
            }
            for (int64_t i = 0; i < dv; ++i) a->dv[(bh * T + j) * dv + i] += pr[j - j0] * (double)dot[i];
        }
    }
    free(s);
    free(pr);
    free(dp);
}

/* q [B,H,T,dk], k [B,T,dk], v [B,H,T,dv], dO [B,H,T,dv] -> dq [B,H,T,dk], dk [B,T,dk],
 * dv [B,H,T,dv] (float64). */
int rodref_swska_backward(const float* q, const float* k, const float* v, const float* dO,
                          double* dq, double* dk_out, double* dv_out, int64_t B, int64_t H,
                          int64_t T, int64_t dk, int64_t dv, int64_t W, double scale, int nthreads) {
    if (!q || !k || !v || !dO || !dq || !dk_out || !dv_out) return RODREF_EINVAL;
    if (B < 0 || H < 1 || T < 0 || dk < 1 || dv < 1 || W < 1) return RODREF_EINVAL;
    double* dkp = malloc((size_t)(B * H * T * dk + 1) * sizeof(double));
    if (!dkp) return RODREF_EINVAL;
    ska_bwd_args_t a = {q, k, v, dO, dq, dkp, dv_out, H, T, dk, dv, W, scale};
    run_units(ska_bwd_unit, &a, B * H, nthreads);
    for (int64_t b = 0; b < B; ++b)
        for (int64_t i = 0; i < T * dk; ++i) {
            double acc = 0.0;
            for (int64_t h = 0; h < H; ++h) acc += dkp[(b * H + h) * T * dk + i];
            dk_out[b * T * dk + i] = acc;
        }
    free(dkp);
    return 0;
}

/* Decode over a paged window cache (SALA blog §3.3: paged KV cache in small blocks): the ring's
 * W slots are cut into pps pages of `page` slots; slot s of sequence n lives in physical page
 * t = table[n*pps + s/page] at row s mod page of the pools k_pool [P][page][dk] and
 * v_pool [P][H][page][dv]. The step is the ring-buffer decode on the logical cache: gather the
 * window from the pages, run rodref_swska_decode, and write the new token's rows back to its
 * page. */
int rodref_swska_decode_paged(const float* q, const float* k_new, const float* v_new, float* k_pool,
                              float* v_pool, const int32_t* table, int64_t page, int64_t pps,
                              const int64_t* pos, double* o, int64_t N, int64_t H, int64_t dk,
                              int64_t dv, int64_t W, double scale, int nthreads) {
    if (!table || !k_pool || !v_pool || !pos || page < 1 || pps < 1 || page * pps != W || N < 0 || H < 1)
        return RODREF_EINVAL;
    float* kc = malloc((size_t)(N * W * dk + 1) * sizeof(float));
    float* vc = malloc((size_t)(N * H * W * dv + 1) * sizeof(float));
    if (!kc || !vc) { free(kc); free(vc); return RODREF_EINVAL; }
    for (int64_t n = 0; n < N; ++n)
        for (int64_t s = 0; s < W; ++s) {
            const int64_t t = table[n * pps + s / page], r = s % page;
            memcpy(kc + (n * W + s) * dk, k_pool + (t * page + r) * dk, (size_t)dk * sizeof(float));
            for (int64_t h = 0; h < H; ++h)
                memcpy(vc + ((n * H + h) * W + s) * dv, v_pool + ((t * H + h) * page + r) * dv,
                       (size_t)dv * sizeof(float));
        }
    const int rc = rodref_swska_decode(q, k_new, v_new, kc, vc, pos, o, N, H, dk, dv, W, scale, nthreads);
    if (rc == 0)
        for (int64_t n = 0; n < N; ++n) {
            const int64_t s = pos[n] % W, t = table[n * pps + s / page], r = s % page;
            memcpy(k_pool + (t * page + r) * dk, kc + (n * W + s) * dk, (size_t)dk * sizeof(float));
            for (int64_t h = 0; h < H; ++h)
                memcpy(v_pool + ((t * H + h) * page + r) * dv, vc + ((n * H + h) * W + s) * dv,
                       (size_t)dv * sizeof(float));
        }
    free(kc);
    free(vc);
    return rc;
}

/* Prefill -> decode hand-off (SALA blog §3.3: decode keeps the most recent W tokens in a
 * circular buffer; the ring rule is the one rodref_swska_decode writes by): every position p in
 * [max(0, T-W), T) of the prefill's shared keys k [B,T,dk] and per-head values v [B,H,T,dv] is
 * copied to slot p mod W of k_cache [B,W,dk] and v_cache [B,H,W,dv]. Other slots are untouched. */
int rodref_swska_cache_fill(const float* k, const float* v, float* k_cache, float* v_cache,
                            int64_t B, int64_t H, int64_t T, int64_t dk, int64_t dv, int64_t W) {
    if (!k || !v || !k_cache || !v_cache) return RODREF_EINVAL;
    if (B < 0 || H < 1 || T < 0 || dk < 1 || dv < 1 || W < 1) return RODREF_EINVAL;
    const int64_t p0 = T > W ? T - W : 0;
    for (int64_t b = 0; b < B; ++b)
        for (int64_t p = p0; p < T; ++p) {
            const int64_t slot = p % W;
            memcpy(k_cache + (b * W + slot) * dk, k + (b * T + p) * dk, (size_t)dk * sizeof(float));
            for (int64_t h = 0; h < H; ++h)
                memcpy(v_cache + ((b * H + h) * W + slot) * dv, v + ((b * H + h) * T + p) * dv,
                       (size_t)dv * sizeof(float));
        }
    return 0;
}

/* ---- FP8 (E4M3) window cache ([SALA] §4.3; format and rounding: the reading in the header) --- */

/* value of an E4M3 code, from the format's definition: exponent field 0 is subnormal
 * (mantissa/8 * 2^-6), otherwise (1 + mantissa/8) * 2^(exponent - 7); S.1111.111 is NaN */
double rodref_e4m3_decode(uint8_t code) {
    const int sign = code >> 7, e = (code >> 3) & 15, m = code & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

/* The 256 code values, evaluated from rodref_e4m3_decode once before any worker thread starts
 * (every entry point below fills it first; filling twice writes the same numbers). */
static double e4m3_table[256];
static int e4m3_table_ready = 0;
static void e4m3_fill_table(void) {
    if (e4m3_table_ready) return;
    for (int c = 0; c < 256; ++c) e4m3_table[c] = rodref_e4m3_decode((uint8_t)c);
    e4m3_table_ready = 1;
}

/* nearest E4M3 code to the fp32 value x: the non-negative finite codes 0x00 .. 0x7E have
 * increasing values, so bisection finds the last code whose value is <= |x|; of it and the next
 * code the closer one wins, a tie goes to the even code; magnitudes beyond 448 take 448
 * (saturation); the sign bit is x's; NaN gives 0x7F */
uint8_t rodref_e4m3_encode(float x) {
    e4m3_fill_table();
    if (isnan(x)) return 0x7F;
    const double a = fabs((double)x);
    int best;
    if (a >= 448.0) {
        best = 0x7E;
    } else {
        int lo = 0, hi = 0x7E;  /* value(lo) <= a < value(hi) */
        while (hi - lo > 1) {
            const int mid = (lo + hi) / 2;
            if (e4m3_table[mid] <= a) lo = mid; else hi = mid;
        }
        const double dl = a - e4m3_table[lo], dh = e4m3_table[hi] - a;
        best = dl < dh ? lo : (dh < dl ? hi : ((lo & 1) == 0 ? lo : hi));
    }
    return (uint8_t)(best | (signbit(x) ? 0x80 : 0));
}

int rodref_e4m3_encode_array(const float* x, uint8_t* out, int64_t n, float scale) {
    if (!x || !out || n < 0 || !(scale > 0.f)) return RODREF_EINVAL;
    for (int64_t i = 0; i < n; ++i) out[i] = rodref_e4m3_encode(x[i] / scale);
    return 0;
}

int rodref_e4m3_decode_array(const uint8_t* c, double* out, int64_t n) {
    if (!c || !out || n < 0) return RODREF_EINVAL;
    e4m3_fill_table();
    for (int64_t i = 0; i < n; ++i) out[i] = e4m3_table[c[i]];
    return 0;
}

/* Decode with FP8 ring caches: k_cache [N,W,dk] and v_cache [N,H,W,dv] hold E4M3 codes. For
 * each sequence n with P = pos[n] >= 0: the new token's codes e4m3(k_new / k_scale) and
 * e4m3(v_new[h] / v_scale) go to slot P mod W, then o[n,h] is the softmax attention of q[n,h]
 * over positions max(0, P-W+1) .. P read back from their slots as value(code) * scale.
 * pos < 0: o = NaN and the caches are left untouched. */
typedef struct {
    const float *q, *k_new, *v_new;
    uint8_t *kc, *vc;
    const int64_t* pos;
    double* o;
    int64_t H, dk, dv, W;
    double scale, k_scale, v_scale;
} ska_dec8_args_t;

static void ska_dec8_unit(const void* p, int64_t n) {
    const ska_dec8_args_t* a = (const ska_dec8_args_t*)p;
    const int64_t H = a->H, dk = a->dk, dv = a->dv, W = a->W, P = a->pos[n];
    if (P < 0) {
        for (int64_t i = 0; i < H * dv; ++i) a->o[n * H * dv + i] = NAN;
        return;
    }
    const int64_t slot = P % W;
    for (int64_t c = 0; c < dk; ++c)
        a->kc[(n * W + slot) * dk + c] = rodref_e4m3_encode(a->k_new[n * dk + c] / (float)a->k_scale);
    for (int64_t h = 0; h < H; ++h)
        for (int64_t c = 0; c < dv; ++c)
            a->vc[((n * H + h) * W + slot) * dv + c] =
                rodref_e4m3_encode(a->v_new[(n * H + h) * dv + c] / (float)a->v_scale);
    const int64_t p0 = P - W + 1 > 0 ? P - W + 1 : 0, cnt = P - p0 + 1;
    double* s = malloc((size_t)cnt * sizeof(double));
    if (!s) return;
    for (int64_t h = 0; h < H; ++h) {
        const float* qv = a->q + (n * H + h) * dk;
        double m = -INFINITY;
        for (int64_t i = 0; i < cnt; ++i) {
            const int64_t sl = (p0 + i) % W;
            double acc = 0.0;
            for (int64_t c = 0; c < dk; ++c)
                acc += (double)qv[c] * e4m3_table[a->kc[(n * W + sl) * dk + c]] * a->k_scale;
            s[i] = a->scale * acc;
            if (s[i] > m) m = s[i];
        }
        double l = 0.0;
        for (int64_t i = 0; i < cnt; ++i) {
            s[i] = exp(s[i] - m);
            l += s[i];
        }
        double* on = a->o + (n * H + h) * dv;
        for (int64_t c = 0; c < dv; ++c) on[c] = 0.0;
        for (int64_t i = 0; i < cnt; ++i) {
            const int64_t sl = (p0 + i) % W;
            for (int64_t c = 0; c < dv; ++c)
                on[c] += s[i] * e4m3_table[a->vc[((n * H + h) * W + sl) * dv + c]] * a->v_scale;
        }
        for (int64_t c = 0; c < dv; ++c) on[c] /= l;
    }
    free(s);
}

int rodref_swska_decode_fp8(const float* q, const float* k_new, const float* v_new, uint8_t* k_cache,
                            uint8_t* v_cache, const int64_t* pos, double* o, int64_t N, int64_t H,
                            int64_t dk, int64_t dv, int64_t W, double scale, double k_scale,
                            double v_scale, int nthreads) {
    if (!q || !k_new || !v_new || !k_cache || !v_cache || !pos || !o) return RODREF_EINVAL;
    if (N < 0 || H < 1 || dk < 1 || dv < 1 || W < 1 || !(k_scale > 0) || !(v_scale > 0)) return RODREF_EINVAL;
    e4m3_fill_table();
    ska_dec8_args_t a = {q, k_new, v_new, k_cache, v_cache, pos, o, H, dk, dv, W, scale, k_scale, v_scale};
    return run_units(ska_dec8_unit, &a, N, nthreads);
}

/* Prefill -> decode hand-off into FP8 rings: positions [max(0, T-W), T) of k [B,T,dk] and
 * v [B,H,T,dv] go to slot p mod W as e4m3(x / scale); other slots are untouched. */
int rodref_swska_cache_fill_fp8(const float* k, const float* v, uint8_t* k_cache, uint8_t* v_cache,
                                int64_t B, int64_t H, int64_t T, int64_t dk, int64_t dv, int64_t W,
                                float k_scale, float v_scale) {
    if (!k || !v || !k_cache || !v_cache) return RODREF_EINVAL;
    if (B < 0 || H < 1 || T < 0 || dk < 1 || dv < 1 || W < 1 || !(k_scale > 0.f) || !(v_scale > 0.f))
        return RODREF_EINVAL;
    const int64_t first = T > W ? T - W : 0;  /* the oldest position still in the window */
    for (int64_t b = 0; b < B; ++b)
        for (int64_t p = first; p < T; ++p) {
            const int64_t ring_slot = p % W;
            for (int64_t c = 0; c < dk; ++c)
                k_cache[(b * W + ring_slot) * dk + c] = rodref_e4m3_encode(k[(b * T + p) * dk + c] / k_scale);
            for (int64_t h = 0; h < H; ++h)
                for (int64_t c = 0; c < dv; ++c)
                    v_cache[((b * H + h) * W + ring_slot) * dv + c] =
                        rodref_e4m3_encode(v[((b * H + h) * T + p) * dv + c] / v_scale);
        }
    return 0;
}

int rodref_abi_version(void) { return 1; }
