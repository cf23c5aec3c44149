/*
 * TEST INFRASTRUCTURE ONLY: the fp64 CPU oracle of the RWKV-4 WKV recurrence.
 * Only the tests, the smoke check and the benchmark's CPU-baseline leg load
 * this file's library; the CUDA path never links, includes or calls it, and
 * it includes nothing from the CUDA path.
 *
 * What it computes (per channel c of each batch row, independently):
 *   w = w_c (a decay, normally -exp(time_decay_c)), u = u_c (the bonus),
 *   A_t = sum_{i<t} e^{(t-1-i) w + k_i} v_i     (numerator state before step t)
 *   D_t = sum_{i<t} e^{(t-1-i) w + k_i}         (denominator state)
 *   wkv_t = (A_t + e^{u+k_t} v_t) / (D_t + e^{u+k_t})
 *   A_{t+1} = e^w A_t + e^{k_t} v_t,  D_{t+1} = e^w D_t + e^{k_t}.
 * The state is carried as a triple (a, b, p) with A = a e^p and D = b e^p:
 * the per-channel numerator / denominator / max of "RWKV in a self-built
 * engine: a second non-attention paradigm (WKV/RNN)" (Methods table,
 * "Precision" row; Reproducibility / Provenance, "Implementation"), with the
 * standard max-trick that keeps every exponent it evaluates <= 0.  Here all
 * arithmetic is fp64 (the pages carry the state in fp32; the oracle uses a
 * wider type so that it sits far inside the GPU path's tolerance).
 *
 * A state given on entry is the state after the previous call's last token,
 * so it enters output t with weight e^{t w}; splitting T into two calls with
 * the state carried across gives the result of one call.  The empty state is
 * (0, 0, -1e38).
 *
 * One step, as the pages name its parts (output, then state update):
 *   q  = max(p, u + k_t)
 *   y  = (e^{p-q} a + e^{u+k_t-q} v_t) / (e^{p-q} b + e^{u+k_t-q})
 *   q' = max(p + w, k_t)
 *   a  = e^{p+w-q'} a + e^{k_t-q'} v_t ;  b = e^{p+w-q'} b + e^{k_t-q'} ;  p = q'
 */
#include <math.h>
#include <pthread.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>

#define ORACLE_EMPTY_MAX (-1e38)

typedef struct {
    int64_t B, T, C;
    const double *w, *u, *k, *v, *state_in;
    double *y, *state_out;
    int64_t ch_begin, ch_end;   /* range of flat channel ids b*C + c */
} oracle_job;

static void run_channel(const oracle_job* j, int64_t b, int64_t c) {
    const int64_t BC = j->B * j->C;
    const int64_t ch = b * j->C + c;
    const double w = j->w[c], u = j->u[c];
    double a = 0.0, d = 0.0, p = ORACLE_EMPTY_MAX;
    if (j->state_in) {
        a = j->state_in[0 * BC + ch];
        d = j->state_in[1 * BC + ch];
        p = j->state_in[2 * BC + ch];
    }
    for (int64_t t = 0; t < j->T; ++t) {
        const int64_t idx = (b * j->T + t) * j->C + c;
        const double kt = j->k[idx], vt = j->v[idx];
        /* output at step t */
        const double q = fmax(p, u + kt);
        const double e_state = exp(p - q);
        const double e_bonus = exp(u + kt - q);
        if (j->y) j->y[idx] = (e_state * a + e_bonus * vt) / (e_state * d + e_bonus);
        /* state update */
        const double q2 = fmax(p + w, kt);
        const double e_decay = exp(p + w - q2);
        const double e_new = exp(kt - q2);
        a = e_decay * a + e_new * vt;
        d = e_decay * d + e_new;
        p = q2;
    }
    if (j->state_out) {
        j->state_out[0 * BC + ch] = a;
        j->state_out[1 * BC + ch] = d;
        j->state_out[2 * BC + ch] = p;
    }
}

static void* run_job(void* arg) {
    const oracle_job* j = (const oracle_job*)arg;
    for (int64_t ch = j->ch_begin; ch < j->ch_end; ++ch) run_channel(j, ch / j->C, ch % j->C);
    return NULL;
}

/*
 * Forward over T steps.
 *   w, u:        [C]
 *   k, v, y:     [B][T][C] (C fastest); y may be NULL
 *   state_in:    [3][B][C] planes (num, den, max) or NULL for the empty state
 *   state_out:   [3][B][C] or NULL; may equal state_in
 *   nthreads:    channels are split over this many threads (<= 1: caller's thread)
 * Returns 0, or -1 on bad sizes / thread failure.
 */
int wkv4_oracle_forward(int64_t B, int64_t T, int64_t C, const double* w, const double* u,
                        const double* k, const double* v, const double* state_in, double* y,
                        double* state_out, int nthreads) {
    if (B < 0 || T < 0 || C < 0) return -1;
    const int64_t n_ch = B * C;
    if (n_ch == 0) return 0;
    double* tmp_state = NULL;
    double* out = state_out;
    if (state_out && state_out == state_in) {
        /* keep the input planes readable until every channel has started */
        tmp_state = (double*)malloc(sizeof(double) * 3 * (size_t)n_ch);
        if (!tmp_state) return -1;
        out = tmp_state;
    }
    if (nthreads < 1) nthreads = 1;
    if (nthreads > n_ch) nthreads = (int)n_ch;
    oracle_job* jobs = (oracle_job*)calloc((size_t)nthreads, sizeof(oracle_job));
    pthread_t* th = (pthread_t*)calloc((size_t)nthreads, sizeof(pthread_t));
    int rc = 0;
    if (!jobs || !th) { rc = -1; goto done; }
    for (int i = 0; i < nthreads; ++i) {
        oracle_job j = {B, T, C, w, u, k, v, state_in, y, out,
                        n_ch * i / nthreads, n_ch * (i + 1) / nthreads};
        jobs[i] = j;
    }
    if (nthreads == 1) {
        run_job(&jobs[0]);
    } else {
        int started = 0;
        for (; started < nthreads; ++started)
            if (pthread_create(&th[started], NULL, run_job, &jobs[started]) != 0) { rc = -1; break; }
        for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
    }
    if (rc == 0 && tmp_state) {
        for (int64_t i = 0; i < 3 * n_ch; ++i) state_out[i] = tmp_state[i];
    }
done:
    free(jobs);
    free(th);
    free(tmp_state);
    return rc;
}
