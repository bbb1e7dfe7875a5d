/*
 * moda_oracle.c -- plain fp64 CPU reference for mixture-of-depths attention (MoDA).
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the oracle that the CUDA path is checked
 * against.  Only the test suite, the smoke check and the benchmark's CPU-baseline leg
 * may load it.  It shares no code, header, table or helper with the CUDA library.
 *
 * What it computes (hyper.ai summary of arXiv 2603.15619, section "Mixture-of-Depths
 * Attention (MoDA)"): every query head attends, in ONE softmax whose scores are all
 * normalised together, to (a) the sequence keys/values of the current layer and (b)
 * the depth keys/values that earlier sublayers wrote for the query's own token.  The
 * section "Hardware-efficient implementation" of the same page says the logits of the
 * sequence and depth blocks feed a single softmax state before normalisation, and
 * the shijienb.com article (section "second half") calls it a unified softmax.  The
 * result is therefore exact attention over an enlarged key set, and this file writes
 * that definition out directly:
 *
 *   visible sequence keys of row (b,h,t):  S(t) = {s <= t} (causal) or {0..T-1}
 *   z_s = scale * <q[b,h,t], k[b,g,s]>      for s in S(t),   g = h / (Hq/Hkv)
 *   y_j = scale * <q[b,h,t], kd[b,g,t,j]>   for j < L        (own token only)
 *   m   = max(z, y),  Z = sum exp(z - m) + sum exp(y - m)
 *   out = (sum exp(z_s - m) v[b,g,s] + sum exp(y_j - m) vd[b,g,t,j]) / Z
 *   lse = m + ln Z
 *
 * Two passes per row (max, then sums), no online rescaling, fp64 throughout.
 *
 * Backward (the pages give no backward design; this is the gradient of the definition
 * above w.r.t. q, k, v, kd, vd given dO, with P = exp(logit - lse) over every visible
 * key and D = <dO, out>):
 *   dS   = P * (<dO, value> - D)
 *   dq  += scale * dS * key
 *   dk[s] += scale * dS * q,   dv[s]  += P * dO      (summed over rows that see s)
 *   dkd[t,j] += scale * dS * q, dvd[t,j] += P * dO   (summed over the G heads of g)
 *
 * Layouts (row-major, contiguous):
 *   q, out, dout, dq : [B][Hq][T][d]
 *   k, v, dk, dv     : [B][Hkv][T][d]
 *   kd, vd, dkd, dvd : [B][Hkv][T][L][d]
 *   lse              : [B][Hq][T]
 *
 * Token windows: every entry point works on the query tokens [t0, t0+nt) of a problem
 * whose sequence K/V span T tokens.  Window-sized arrays (q, dout, out, lse, dq, kd, vd,
 * dkd, dvd) hold only those nt tokens, in the layouts above with T replaced by nt; k, v,
 * dk, dv always span all T tokens.  The full problem is the window t0=0, nt=T.  This lets
 * a test check sampled rows of a 64K-token problem without materialising its whole
 * depth cache in fp64.
 *
 * Depth-only attention (Flash Depth Attention, the pages' other operator: hyper.ai
 * summary, section "Depth-stream mechanisms" -- a layer's input is attention over the
 * key/value pairs that earlier layers wrote for the SAME token; shijienb.com article,
 * first half, names its kernel Flash Depth Attention): the same definition with no
 * sequence keys, S(t) = {}.  The moda_oracle_depth_* entry points run it (causal = -1
 * internally; k, v, dk, dv absent).
 *
 * Parallelism: rows (forward) or tokens of one (b, kv-head) group (backward) are handed
 * to POSIX threads through an atomic counter; each unit's arithmetic is the plain loop
 * above.  In the backward each thread sums its rows' sequence-key gradients into private
 * buffers that are added into dk/dv when the group is done.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    const double *q, *k, *v, *kd, *vd, *dout;
    const double *out_given; /* backward only: if set, D = <dO, out_given> (see below) */
    double *out, *lse, *dq, *dk, *dv, *dkd, *dvd;
    int64_t nunits;
    int B, Hq, Hkv, T, L, d, causal;
    int t0, nt; /* query-token window */
    double scale;
    volatile int64_t next;
} job_t;

static double dot(const double *a, const double *b, int d) {
    double s = 0.0;
    for (int c = 0; c < d; ++c) s += a[c] * b[c];
    return s;
}

/* Number of visible sequence keys for token t (causal < 0: depth-only, none). */
static int n_seq(int t, int T, int causal) {
    if (causal < 0) return 0;
    return causal ? t + 1 : T;
}

/* Offsets of window-sized arrays: row (b,h,w) of q/out, token (b,g,w) of kd/vd. */
static int64_t qrow(const job_t *J, int b, int h, int w) {
    return ((int64_t)b * J->Hq + h) * J->nt + w;
}
static int64_t dtok(const job_t *J, int b, int g, int w) {
    return ((int64_t)b * J->Hkv + g) * J->nt + w;
}

/* Forward for the row (b, h, token t0+w).  scratch holds T + L doubles and receives the
 * row's logits (sequence keys first, then depth keys).  Writes out_row[d], *lse_row. */
static void forward_row(const job_t *J, int b, int h, int w, double *scratch,
                        double *out_row, double *lse_row) {
    const int d = J->d, T = J->T, L = J->L, G = J->Hq / J->Hkv, g = h / G;
    const int t = J->t0 + w;
    const int ns = n_seq(t, T, J->causal);
    const double *qr = J->q + qrow(J, b, h, w) * d;
    const double *kb = ns ? J->k + ((int64_t)b * J->Hkv + g) * T * d : NULL;
    const double *vb = ns ? J->v + ((int64_t)b * J->Hkv + g) * T * d : NULL;
    const double *kdt = L ? J->kd + dtok(J, b, g, w) * L * d : NULL;
    const double *vdt = L ? J->vd + dtok(J, b, g, w) * L * d : NULL;

    /* pass 1: logits and their maximum */
    double m = -INFINITY;
    for (int s = 0; s < ns; ++s) {
        scratch[s] = J->scale * dot(qr, kb + (int64_t)s * d, d);
        if (scratch[s] > m) m = scratch[s];
    }
    for (int j = 0; j < L; ++j) {
        scratch[ns + j] = J->scale * dot(qr, kdt + (int64_t)j * d, d);
        if (scratch[ns + j] > m) m = scratch[ns + j];
    }
    /* pass 2: normaliser and weighted sum of values */
    double Z = 0.0;
    for (int c = 0; c < d; ++c) out_row[c] = 0.0;
    for (int s = 0; s < ns; ++s) {
        const double p = exp(scratch[s] - m);
        const double *vr = vb + (int64_t)s * d;
        Z += p;
        for (int c = 0; c < d; ++c) out_row[c] += p * vr[c];
    }
    for (int j = 0; j < L; ++j) {
        const double p = exp(scratch[ns + j] - m);
        const double *vr = vdt + (int64_t)j * d;
        Z += p;
        for (int c = 0; c < d; ++c) out_row[c] += p * vr[c];
    }
    for (int c = 0; c < d; ++c) out_row[c] /= Z;
    *lse_row = m + log(Z);
}

static int64_t take(job_t *J) { return __atomic_fetch_add(&J->next, 1, __ATOMIC_RELAXED); }

static void *forward_worker(void *arg) {
    job_t *J = (job_t *)arg;
    double *scratch = (double *)malloc(sizeof(double) * ((size_t)J->T + (size_t)J->L + 1));
    for (int64_t u; (u = take(J)) < J->nunits;) {
        const int w = (int)(u % J->nt);
        const int h = (int)((u / J->nt) % J->Hq);
        const int b = (int)(u / ((int64_t)J->nt * J->Hq));
        forward_row(J, b, h, w, scratch, J->out + u * J->d, J->lse + u);
    }
    free(scratch);
    return NULL;
}

/* Per-thread state of the backward: row scratch and private key-gradient buffers.  The
 * rows of one (b, g) group are dealt out token by token among the threads; every row
 * adds to the sequence-key gradients dk/dv of every key it sees, so each thread sums
 * those contributions into its own [nkeys][d] buffers, and the buffers are added into
 * dk/dv once every thread has finished the group.  dq rows and the depth gradients of a
 * token (dkd/dvd, summed over the G heads of the token's group) belong to exactly one
 * token, so one thread writes them directly. */
typedef struct {
    job_t *J;
    double *scratch, *o_row, *dk_acc, *dv_acc;
    int b, g, tid, nthreads;
    int64_t nkeys;
} bwd_ctx_t;

/* Backward for the G rows (heads of group g) of token t0+w: adds their contributions to
 * dq (own rows), dkd/dvd (own token) and the thread's dk/dv buffers. */
static void backward_token(bwd_ctx_t *C, int w) {
    job_t *J = C->J;
    const int b = C->b, g = C->g;
    const int d = J->d, T = J->T, L = J->L, G = J->Hq / J->Hkv;
    const int64_t kvoff = ((int64_t)b * J->Hkv + g) * T * d;
    const int has_seq = J->causal >= 0;
    const double *kb = has_seq ? J->k + kvoff : NULL, *vb = has_seq ? J->v + kvoff : NULL;
    double *dkb = C->dk_acc, *dvb = C->dv_acc;
    double *scratch = C->scratch, *o_row = C->o_row;
    for (int h = g * G; h < (g + 1) * G; ++h) {
        const int64_t r = qrow(J, b, h, w);
        const double *qr = J->q + r * d, *dor = J->dout + r * d;
        double *dqr = J->dq + r * d;
        const int64_t doff = dtok(J, b, g, w) * L * d;
        const double *kdt = L ? J->kd + doff : NULL, *vdt = L ? J->vd + doff : NULL;
        double *dkdt = L ? J->dkd + doff : NULL, *dvdt = L ? J->dvd + doff : NULL;
        const int ns = n_seq(J->t0 + w, T, J->causal);
        double lse;
        forward_row(J, b, h, w, scratch, o_row, &lse);
        if (J->out) { memcpy(J->out + r * d, o_row, sizeof(double) * d); J->lse[r] = lse; }
        const double D = dot(dor, J->out_given ? J->out_given + r * d : o_row, d);
        /* sequence keys: logits are in scratch[0..ns) from forward_row */
        for (int s = 0; s < ns; ++s) {
            const double P = exp(scratch[s] - lse);
            const double dP = dot(dor, vb + (int64_t)s * d, d);
            const double dS = P * (dP - D);
            const double *kr = kb + (int64_t)s * d;
            double *dkr = dkb + (int64_t)s * d, *dvr = dvb + (int64_t)s * d;
            for (int c = 0; c < d; ++c) {
                dqr[c] += J->scale * dS * kr[c];
                dkr[c] += J->scale * dS * qr[c];
                dvr[c] += P * dor[c];
            }
        }
        /* depth keys of the row's own token: logits in scratch[ns..ns+L) */
        for (int j = 0; j < L; ++j) {
            const double P = exp(scratch[ns + j] - lse);
            const double dP = dot(dor, vdt + (int64_t)j * d, d);
            const double dS = P * (dP - D);
            const double *kr = kdt + (int64_t)j * d;
            double *dkr = dkdt + (int64_t)j * d, *dvr = dvdt + (int64_t)j * d;
            for (int c = 0; c < d; ++c) {
                dqr[c] += J->scale * dS * kr[c];
                dkr[c] += J->scale * dS * qr[c];
                dvr[c] += P * dor[c];
            }
        }
    }
}

/* Thread `tid` of `nthreads` takes the window's tokens tid, tid + nthreads, ... (a fixed
 * interleaving: causal rows grow in cost with t, so every thread gets a similar mix). */
static void *backward_worker(void *arg) {
    bwd_ctx_t *C = (bwd_ctx_t *)arg;
    for (int w = C->tid; w < C->J->nt; w += C->nthreads) backward_token(C, w);
    return NULL;
}

/* The whole backward: one (b, g) group after another, each group's window tokens shared
 * out among the threads, then the threads' key-gradient buffers summed into dk/dv. */
static void run_backward(job_t *J, int nthreads) {
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    if (nthreads > J->nt) nthreads = J->nt;
    const int has_seq = J->causal >= 0;
    /* keys that window rows can see: [0, t0+nt) when causal, all T otherwise */
    const int64_t nkeys = !has_seq ? 0 : (J->causal ? J->t0 + J->nt : J->T);
    const size_t kbytes = sizeof(double) * (size_t)nkeys * (size_t)J->d;
    pthread_t th[256];
    bwd_ctx_t C[256];
    for (int i = 0; i < nthreads; ++i) {
        C[i].J = J;
        C[i].scratch = (double *)malloc(sizeof(double) * ((size_t)J->T + (size_t)J->L + 1));
        C[i].o_row = (double *)malloc(sizeof(double) * (size_t)J->d);
        C[i].dk_acc = nkeys ? (double *)malloc(kbytes) : NULL;
        C[i].dv_acc = nkeys ? (double *)malloc(kbytes) : NULL;
        C[i].nkeys = nkeys;
        C[i].tid = i;
        C[i].nthreads = nthreads;
    }
    for (int b = 0; b < J->B; ++b) {
        for (int g = 0; g < J->Hkv; ++g) {
            for (int i = 0; i < nthreads; ++i) {
                C[i].b = b;
                C[i].g = g;
                if (nkeys) { memset(C[i].dk_acc, 0, kbytes); memset(C[i].dv_acc, 0, kbytes); }
            }
            for (int i = 1; i < nthreads; ++i) pthread_create(&th[i], NULL, backward_worker, &C[i]);
            backward_worker(&C[0]);
            for (int i = 1; i < nthreads; ++i) pthread_join(th[i], NULL);
            if (nkeys) {
                const int64_t kvoff = ((int64_t)b * J->Hkv + g) * J->T * J->d;
                const int64_t n = nkeys * J->d;
                for (int i = 0; i < nthreads; ++i)
                    for (int64_t e = 0; e < n; ++e) {
                        J->dk[kvoff + e] += C[i].dk_acc[e];
                        J->dv[kvoff + e] += C[i].dv_acc[e];
                    }
            }
        }
    }
    for (int i = 0; i < nthreads; ++i) {
        free(C[i].scratch); free(C[i].o_row); free(C[i].dk_acc); free(C[i].dv_acc);
    }
}

/* Forward threading: rows handed out through the job's atomic counter. */
static void run(job_t *J, void *(*fn)(void *), int nthreads) {
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    if ((int64_t)nthreads > J->nunits) nthreads = (int)(J->nunits > 0 ? J->nunits : 1);
    pthread_t th[256];
    J->next = 0;
    for (int i = 1; i < nthreads; ++i) pthread_create(&th[i], NULL, fn, J);
    fn(J);
    for (int i = 1; i < nthreads; ++i) pthread_join(th[i], NULL);
}

static int bad_dims(int B, int Hq, int Hkv, int T, int L, int d, int t0, int nt) {
    if (B < 1 || Hq < 1 || Hkv < 1 || T < 1 || L < 0 || d < 1) return 1;
    if (Hq % Hkv != 0) return 1;
    if (t0 < 0 || nt < 1 || t0 + nt > T) return 1;
    return 0;
}

/* Forward over the query tokens [t0, t0+nt).  Returns 0 on success, 1 on bad sizes. */
int moda_oracle_forward(const double *q, const double *k, const double *v,
                        const double *kd, const double *vd, double *out, double *lse,
                        int B, int Hq, int Hkv, int T, int L, int d, int t0, int nt,
                        double scale, int causal, int nthreads) {
    if (bad_dims(B, Hq, Hkv, T, L, d, t0, nt)) return 1;
    job_t J = {0};
    J.q = q; J.k = k; J.v = v; J.kd = kd; J.vd = vd; J.out = out; J.lse = lse;
    J.B = B; J.Hq = Hq; J.Hkv = Hkv; J.T = T; J.L = L; J.d = d; J.causal = causal;
    J.t0 = t0; J.nt = nt; J.scale = scale;
    J.nunits = (int64_t)B * Hq * nt;
    run(&J, forward_worker, nthreads);
    return 0;
}

/* Backward over the rows whose token lies in [t0, t0+nt).  Gradient buffers are zeroed,
 * then receive the contributions of those rows only, so:
 *   dq (window rows) and dkd/dvd (window tokens) are exact;
 *   with causal=1 and t0+nt=T, dk/dv of every key s >= t0 are exact (only rows of
 *   tokens t >= s see key s); the full backward is the window t0=0, nt=T.
 * If out/lse are non-NULL the oracle's own forward results are written there too. */
/* Backward whose row terms D = <dO, out> use a caller-given `out` (window-sized, like q)
 * instead of the oracle's own exact output; every other quantity (the logits, P from the
 * exact log-sum-exp, the value products) is computed exactly as in moda_oracle_backward.
 * A backward that receives only the forward's rounded output (the operator's backward
 * interface takes `out` as an input) can at best compute D from it, and this mode is the
 * exact result of that; with out_given = the oracle's own out it equals
 * moda_oracle_backward. */
int moda_oracle_backward_given_out(const double *q, const double *k, const double *v,
                                   const double *kd, const double *vd, const double *dout,
                                   const double *out_given, double *dq, double *dk,
                                   double *dv, double *dkd, double *dvd, int B, int Hq,
                                   int Hkv, int T, int L, int d, int t0, int nt,
                                   double scale, int causal, int nthreads);

int moda_oracle_backward(const double *q, const double *k, const double *v,
                         const double *kd, const double *vd, const double *dout,
                         double *dq, double *dk, double *dv, double *dkd, double *dvd,
                         double *out, double *lse, int B, int Hq, int Hkv, int T, int L,
                         int d, int t0, int nt, double scale, int causal, int nthreads) {
    if (bad_dims(B, Hq, Hkv, T, L, d, t0, nt)) return 1;
    const size_t nq = (size_t)B * Hq * nt * d, nk = (size_t)B * Hkv * T * d;
    const size_t nd = (size_t)B * Hkv * nt * (size_t)L * d;
    memset(dq, 0, nq * sizeof(double));
    memset(dk, 0, nk * sizeof(double));
    memset(dv, 0, nk * sizeof(double));
    if (nd) { memset(dkd, 0, nd * sizeof(double)); memset(dvd, 0, nd * sizeof(double)); }
    job_t J = {0};
    J.q = q; J.k = k; J.v = v; J.kd = kd; J.vd = vd; J.dout = dout;
    J.dq = dq; J.dk = dk; J.dv = dv; J.dkd = dkd; J.dvd = dvd; J.out = out; J.lse = lse;
    J.B = B; J.Hq = Hq; J.Hkv = Hkv; J.T = T; J.L = L; J.d = d; J.causal = causal;
    J.t0 = t0; J.nt = nt; J.scale = scale;
    run_backward(&J, nthreads);
    return 0;
}

int moda_oracle_backward_given_out(const double *q, const double *k, const double *v,
                                   const double *kd, const double *vd, const double *dout,
                                   const double *out_given, double *dq, double *dk,
                                   double *dv, double *dkd, double *dvd, int B, int Hq,
                                   int Hkv, int T, int L, int d, int t0, int nt,
                                   double scale, int causal, int nthreads) {
    if (bad_dims(B, Hq, Hkv, T, L, d, t0, nt) || !out_given) return 1;
    const size_t nq = (size_t)B * Hq * nt * d, nk = (size_t)B * Hkv * T * d;
    const size_t nd = (size_t)B * Hkv * nt * (size_t)L * d;
    memset(dq, 0, nq * sizeof(double));
    memset(dk, 0, nk * sizeof(double));
    memset(dv, 0, nk * sizeof(double));
    if (nd) { memset(dkd, 0, nd * sizeof(double)); memset(dvd, 0, nd * sizeof(double)); }
    job_t J = {0};
    J.q = q; J.k = k; J.v = v; J.kd = kd; J.vd = vd; J.dout = dout; J.out_given = out_given;
    J.dq = dq; J.dk = dk; J.dv = dv; J.dkd = dkd; J.dvd = dvd;
    J.B = B; J.Hq = Hq; J.Hkv = Hkv; J.T = T; J.L = L; J.d = d; J.causal = causal;
    J.t0 = t0; J.nt = nt; J.scale = scale;
    run_backward(&J, nthreads);
    return 0;
}

/* Normalised joint-softmax weights of one row (b, h, t) of a full problem (t0=0, nt=T):
 * w_seq[0..n) for the n visible sequence keys in key order, w_depth[0..L) for the
 * token's depth keys.  A debug view used by the tests. */
int moda_oracle_row_weights(const double *q, const double *k, const double *kd, int b,
                            int h, int t, int B, int Hq, int Hkv, int T, int L, int d,
                            double scale, int causal, double *w_seq, double *w_depth) {
    if (bad_dims(B, Hq, Hkv, T, L, d, 0, T)) return 1;
    if (b < 0 || b >= B || h < 0 || h >= Hq || t < 0 || t >= T) return 1;
    const int G = Hq / Hkv, g = h / G, ns = n_seq(t, T, causal);
    const double *qr = q + (((int64_t)b * Hq + h) * T + t) * d;
    const double *kb = k + ((int64_t)b * Hkv + g) * T * d;
    const double *kdt = kd + ((((int64_t)b * Hkv + g) * T + t) * L) * d;
    double m = -INFINITY, Z = 0.0;
    for (int s = 0; s < ns; ++s) {
        w_seq[s] = scale * dot(qr, kb + (int64_t)s * d, d);
        if (w_seq[s] > m) m = w_seq[s];
    }
    for (int j = 0; j < L; ++j) {
        w_depth[j] = scale * dot(qr, kdt + (int64_t)j * d, d);
        if (w_depth[j] > m) m = w_depth[j];
    }
    for (int s = 0; s < ns; ++s) { w_seq[s] = exp(w_seq[s] - m); Z += w_seq[s]; }
    for (int j = 0; j < L; ++j) { w_depth[j] = exp(w_depth[j] - m); Z += w_depth[j]; }
    for (int s = 0; s < ns; ++s) w_seq[s] /= Z;
    for (int j = 0; j < L; ++j) w_depth[j] /= Z;
    return 0;
}

/* Depth-only attention forward over the query tokens [t0, t0+nt): every row attends to
 * its own token's L >= 1 depth keys only.  Returns 0 on success, 1 on bad sizes. */
int moda_oracle_depth_forward(const double *q, const double *kd, const double *vd,
                              double *out, double *lse, int B, int Hq, int Hkv, int T, int L,
                              int d, int t0, int nt, double scale, int nthreads) {
    if (bad_dims(B, Hq, Hkv, T, L, d, t0, nt) || L < 1) return 1;
    job_t J = {0};
    J.q = q; J.kd = kd; J.vd = vd; J.out = out; J.lse = lse;
    J.B = B; J.Hq = Hq; J.Hkv = Hkv; J.T = T; J.L = L; J.d = d; J.causal = -1;
    J.t0 = t0; J.nt = nt; J.scale = scale;
    J.nunits = (int64_t)B * Hq * nt;
    run(&J, forward_worker, nthreads);
    return 0;
}

/* Depth-only attention backward over the window's rows: dq, dkd, dvd (all exact for the
 * window).  out_given: NULL for the exact row terms D = <dO, out>, else D is taken from
 * the given (window-sized) out, as in moda_oracle_backward_given_out.  If out/lse are
 * non-NULL the oracle's own forward results are written there too. */
int moda_oracle_depth_backward(const double *q, const double *kd, const double *vd,
                               const double *dout, const double *out_given, double *dq,
                               double *dkd, double *dvd, double *out, double *lse, int B,
                               int Hq, int Hkv, int T, int L, int d, int t0, int nt,
                               double scale, int nthreads) {
    if (bad_dims(B, Hq, Hkv, T, L, d, t0, nt) || L < 1) return 1;
    const size_t nq = (size_t)B * Hq * nt * d;
    const size_t nd = (size_t)B * Hkv * nt * (size_t)L * d;
    memset(dq, 0, nq * sizeof(double));
    memset(dkd, 0, nd * sizeof(double));
    memset(dvd, 0, nd * sizeof(double));
    job_t J = {0};
    J.q = q; J.kd = kd; J.vd = vd; J.dout = dout; J.out_given = out_given;
    J.dq = dq; J.dkd = dkd; J.dvd = dvd; J.out = out; J.lse = lse;
    J.B = B; J.Hq = Hq; J.Hkv = Hkv; J.T = T; J.L = L; J.d = d; J.causal = -1;
    J.t0 = t0; J.nt = nt; J.scale = scale;
    run_backward(&J, nthreads);
    return 0;
}
