/*
 * gdn_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, token-by-token fp64 CPU implementation of the Gated-Delta-Net
 * (GDN) linear-attention recurrence.  Only the test-suite, the smoke check and
 * the benchmark's CPU-baseline leg may load this library; the product path
 * (the CUDA library) never does, and the two share no code.
 *
 * Definition followed.  The librediffusion PR #21 page ("What's added") names
 * the operation -- a GDN (Gated-Delta-Net) linear-attention recurrence kernel
 * -- but none of the pages prints its formula.  The update below is the gated
 * delta rule (the standard Gated DeltaNet recurrence), per head, with S a
 * dv x dk matrix:
 *
 *     S_t = a_t * S_{t-1} * (I - b_t k_t k_t^T) + b_t v_t k_t^T
 *     o_t = S_t q_t
 *
 * It is evaluated literally, one token at a time, with the product by
 * (I - b k k^T) expanded as S - b (S k) k^T (same value, O(dk*dv) per token
 * instead of forming the dk x dk matrix).  No chunking, no blocking, no
 * reordering.  The library's state layout is S^T, i.e. [dk][dv] row-major,
 * so state_in/state_out are read/written transposed (readings, stated in the
 * design notes: the stored state H = S^T; o_t uses S_t, i.e. the state that
 * already includes token t; no 1/sqrt(dk) scale).
 *
 * The bidirectional form (the "gdn_bidi" kernel named in the PR #21 review, and
 * the full-sequence bidirectional SANA-WM release on the flashdreams SANA-WM
 * page, "Bidirectional variant") is read as
 *     o = fwd(x).o + flip_t( fwd(flip_t(x)).o )
 * where flip_t reverses q, k, v, beta and decay together along time, the
 * reverse scan starts from a zero state, and state_in applies to the forward
 * scan only.  state_out then holds {forward final, reverse final}.
 *
 * The streaming rollout (the causal linear-attention KV cache of the LongSANA
 * diffusers PR #12723, "PR feature") is n_chunks causal calls with each
 * chunk's final state fed as the next chunk's initial state.
 *
 * Parallelism: independent (b, h, direction) scans are spread over POSIX
 * threads.  Each scan is computed by exactly the same sequential code, so the
 * thread count never changes a result bit.
 */
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    /* one scan: a single (b, h) head in one direction */
    const double *q, *k, *v, *beta, *decay; /* q,k: [T][dk]; v: [T][dv]; gates: [T] */
    const double *h0;                        /* [dk][dv] (S^T) or NULL = zero      */
    double *h_final;                         /* [dk][dv] or NULL                     */
    double *o;                               /* [T][dv]; written (=) or added (+=)   */
    int T, dk, dv;
    int reverse;                             /* walk t = T-1 .. 0                    */
    int accumulate;                          /* o += instead of o =                  */
} scan_job;

/* One scan of the recurrence.  S is held as S[i][j], i < dv (value index),
 * j < dk (key index), exactly the orientation of the defining formula. */
static int run_scan(const scan_job *J)
{
    const int dk = J->dk, dv = J->dv, T = J->T;
    double *S = (double *)calloc((size_t)dv * dk, sizeof(double));
    double *y = (double *)malloc((size_t)dv * sizeof(double));
    if (!S || !y) { free(S); free(y); return -1; }

    if (J->h0) /* state_in is S^T, [dk][dv] */
        for (int i = 0; i < dv; ++i)
            for (int j = 0; j < dk; ++j)
                S[(size_t)i * dk + j] = J->h0[(size_t)j * dv + i];

    for (int s = 0; s < T; ++s) {
        const int t = J->reverse ? (T - 1 - s) : s;
        const double *kt = J->k + (size_t)t * dk;
        const double *qt = J->q + (size_t)t * dk;
        const double *vt = J->v + (size_t)t * dv;
        const double a = J->decay[t];
        const double b = J->beta[t];

        /* y = S_{t-1} k_t */
        for (int i = 0; i < dv; ++i) {
            double acc = 0.0;
            for (int j = 0; j < dk; ++j) acc += S[(size_t)i * dk + j] * kt[j];
            y[i] = acc;
        }
        /* S_t = a (S_{t-1} - b y k^T) + b v k^T */
        for (int i = 0; i < dv; ++i)
            for (int j = 0; j < dk; ++j) {
                double *sij = &S[(size_t)i * dk + j];
                *sij = a * (*sij - b * y[i] * kt[j]) + b * vt[i] * kt[j];
            }
        /* o_t = S_t q_t */
        double *ot = J->o + (size_t)t * dv;
        for (int i = 0; i < dv; ++i) {
            double acc = 0.0;
            for (int j = 0; j < dk; ++j) acc += S[(size_t)i * dk + j] * qt[j];
            if (J->accumulate) ot[i] += acc; else ot[i] = acc;
        }
    }

    if (J->h_final)
        for (int i = 0; i < dv; ++i)
            for (int j = 0; j < dk; ++j)
                J->h_final[(size_t)j * dv + i] = S[(size_t)i * dk + j];
    free(S);
    free(y);
    return 0;
}

typedef struct {
    scan_job *jobs;
    int n_jobs;
    int next;
    int failed;
    pthread_mutex_t mu;
} job_queue;

static void *worker(void *arg)
{
    job_queue *Q = (job_queue *)arg;
    for (;;) {
        pthread_mutex_lock(&Q->mu);
        int i = Q->next++;
        pthread_mutex_unlock(&Q->mu);
        if (i >= Q->n_jobs) break;
        if (run_scan(&Q->jobs[i]) != 0) {
            pthread_mutex_lock(&Q->mu);
            Q->failed = 1;
            pthread_mutex_unlock(&Q->mu);
        }
    }
    return NULL;
}

/* Runs the jobs on up to n_threads threads.  Jobs that write the same o rows
 * must not run concurrently; callers run the accumulating (reverse) jobs in a
 * second batch. */
static int run_jobs(scan_job *jobs, int n_jobs, int n_threads)
{
    if (n_jobs <= 0) return 0;
    if (n_threads < 1) n_threads = 1;
    if (n_threads > n_jobs) n_threads = n_jobs;
    job_queue Q;
    Q.jobs = jobs; Q.n_jobs = n_jobs; Q.next = 0; Q.failed = 0;
    pthread_mutex_init(&Q.mu, NULL);
    if (n_threads == 1) {
        worker(&Q);
    } else {
        pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)n_threads);
        if (!th) { pthread_mutex_destroy(&Q.mu); return -1; }
        for (int i = 0; i < n_threads; ++i) pthread_create(&th[i], NULL, worker, &Q);
        for (int i = 0; i < n_threads; ++i) pthread_join(th[i], NULL);
        free(th);
    }
    pthread_mutex_destroy(&Q.mu);
    return Q.failed ? -1 : 0;
}

/*
 * oracle_gdn_forward: the whole [B,H] batch.
 *   q, k   : [B,H,T,dk]      v, o : [B,H,T,dv]      beta, decay : [B,H,T]
 *   state_in  : [B,H,dk,dv] (S^T) or NULL (zero); forward scan only.
 *   state_out : NULL, or [B,H,dk,dv] (causal) / [2,B,H,dk,dv] (bidi: fwd, rev).
 *   bidi      : 0 = causal scan, 1 = forward + re-reversed reverse scan.
 * Returns 0, or -1 on bad arguments / allocation failure.
 */
int oracle_gdn_forward(const double *q, const double *k, const double *v,
                       const double *beta, const double *decay,
                       const double *state_in, double *state_out, double *o,
                       int B, int H, int T, int dk, int dv, int bidi, int n_threads)
{
    if (!q || !k || !v || !beta || !decay || !o) return -1;
    if (B <= 0 || H <= 0 || T <= 0 || dk <= 0 || dv <= 0) return -1;
    const int BH = B * H;
    const size_t st = (size_t)dk * dv;
    scan_job *jobs = (scan_job *)calloc((size_t)BH, sizeof(scan_job));
    if (!jobs) return -1;
    int rc = 0;
    for (int dir = 0; dir < (bidi ? 2 : 1) && rc == 0; ++dir) {
        for (int bh = 0; bh < BH; ++bh) {
            scan_job *J = &jobs[bh];
            J->q = q + (size_t)bh * T * dk;
            J->k = k + (size_t)bh * T * dk;
            J->v = v + (size_t)bh * T * dv;
            J->beta = beta + (size_t)bh * T;
            J->decay = decay + (size_t)bh * T;
            J->h0 = (dir == 0 && state_in) ? state_in + (size_t)bh * st : NULL;
            J->h_final = state_out ? state_out + ((size_t)dir * BH + bh) * st : NULL;
            J->o = o + (size_t)bh * T * dv;
            J->T = T; J->dk = dk; J->dv = dv;
            J->reverse = dir;
            J->accumulate = dir; /* the reverse scan adds onto the forward one */
        }
        rc = run_jobs(jobs, BH, n_threads);
    }
    free(jobs);
    return rc;
}

/*
 * oracle_gdn_rollout: n_chunks consecutive causal chunks, chunk-major inputs
 *   q, k : [n_chunks,B,H,Tc,dk]   v, o : [n_chunks,B,H,Tc,dv]
 *   beta, decay : [n_chunks,B,H,Tc]
 *   state_in : [B,H,dk,dv] or NULL;  state_out : [B,H,dk,dv] or NULL
 *   chunk_states : NULL or [n_chunks,B,H,dk,dv], the state after each chunk.
 * Each chunk's final state is the next chunk's initial state.
 */
int oracle_gdn_rollout(const double *q, const double *k, const double *v,
                       const double *beta, const double *decay,
                       const double *state_in, double *state_out, double *chunk_states,
                       double *o, int B, int H, int n_chunks, int Tc, int dk, int dv,
                       int n_threads)
{
    if (!q || !k || !v || !beta || !decay || !o) return -1;
    if (B <= 0 || H <= 0 || n_chunks <= 0 || Tc <= 0 || dk <= 0 || dv <= 0) return -1;
    const size_t BH = (size_t)B * H;
    const size_t st = (size_t)dk * dv;
    double *cur = (double *)calloc(BH * st, sizeof(double));
    double *nxt = (double *)calloc(BH * st, sizeof(double));
    if (!cur || !nxt) { free(cur); free(nxt); return -1; }
    if (state_in) memcpy(cur, state_in, BH * st * sizeof(double));
    int rc = 0;
    for (int c = 0; c < n_chunks && rc == 0; ++c) {
        const size_t tok = (size_t)c * BH * Tc;
        rc = oracle_gdn_forward(q + tok * dk, k + tok * dk, v + tok * dv,
                                beta + tok, decay + tok, cur, nxt, o + tok * dv,
                                B, H, Tc, dk, dv, 0, n_threads);
        if (chunk_states) memcpy(chunk_states + (size_t)c * BH * st, nxt, BH * st * sizeof(double));
        double *tmp = cur; cur = nxt; nxt = tmp;
    }
    if (rc == 0 && state_out) memcpy(state_out, cur, BH * st * sizeof(double));
    free(cur);
    free(nxt);
    return rc;
}
