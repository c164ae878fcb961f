/*
 * WKV-7 oracle: the plain sequential recurrence in double precision, on the CPU.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or load
 * this file; only the test suite, the smoke check and the benchmark's CPU
 * baseline leg use it.  It shares no code, header or constant with the CUDA
 * library: it parses its own arguments and computes everything from scratch.
 *
 * What it computes (per sequence n, head h; S is a D x D matrix, row index i is
 * the value channel, column index j is the key channel):
 *
 *   w_j   = exp(-exp(l_j))                                      (decay)
 *   sa_i  = sum_j S_ij a_j                                      (uses S_{t-1})
 *   S_ij <- S_ij w_j + sa_i b_j + v_i k_j                       (state update)
 *   y_i   = sum_j S_ij r_j                                      (uses S_t)
 *
 * Sources:
 *  - State update S_t = S_{t-1}(diag(w_t) - k^T (a (.) k)) + v^T k: the note
 *    "RWKV-7 Goose: Expressive Dynamic State Evolution" (myWiki, peng-rwkv7),
 *    section "Generalized Delta rule", the full state-update formula.  Written
 *    with a = -kk and b = kk*a_lr the rank-one term is (S a) b^T, which is the
 *    argument order of the WKV call in the forward listing of
 *    "RWKV hxa07D architecture explainer" (zenn.dev/openmose), where the
 *    kernel receives (r, log_neglog_w, k, v, -kk, kk*a).
 *  - Decay w = exp(-exp(log_neglog_w)): the same listing, where w is formed
 *    from log_neglog_w by two exponentials and the kernel is handed the inner
 *    argument.
 *  - Read-out after the update (y_t = S_t r_t): "RWKV-7 Goose architecture
 *    analysis" (youngju.dev), section "Dynamic State Evolution", whose
 *    per-token loop updates the state and then reads the output from it.
 *  - Padding / variable length: the same WKV call takes an attention mask "for
 *    variable length and padding"; here sequences are given by offsets into a
 *    packed token axis and each sequence starts from its own initial state.
 *
 * Gated read-out (wkv7_oracle_gate), the steps the hxa07D forward listing
 * applies to the WKV result before its output projection ("RWKV hxa07D
 * architecture explainer", forward listing after the WKV call, and its section
 * 9 on the scaling, the r-k-v term and the output gate):
 *
 *   u     = sum_d r_d k_d rk[h][d]                              (per token, head)
 *   z_i   = (y_i / sqrt(D) + u v_i) g_i
 *
 * with y the recurrence output above, r, k, v the same inputs, rk a per-head
 * vector and g the gate.
 *
 * Prologue (wkv7_oracle_prologue), the steps the same forward listing takes
 * between the projections and the WKV call, with the key and value projections
 * producing H_kv heads that are shared by H / H_kv consecutive query heads
 * (the listing's repeat of k/v heads when n_kv_heads < n_heads):
 *
 *   k, v  = the key and value rows of kv head h / (H / H_kv)
 *   w_d   = exp(-exp(l_d))
 *   kk    = k / max(||k||_2, 1e-12)                 (normalise over the head)
 *   k'    = k (1 - w + a_lr)                        (the key handed to the call)
 *   a     = -kk,  b = kk a_lr                       (the pair handed to the call)
 *
 * with a_lr the per-channel in-context learning rate (the listing's sigmoid
 * output "a").  The gated read-out after a prologue uses k' and the repeated v.
 *
 * Backward (wkv7_oracle_backward): the gradient of a scalar loss
 * L = sum_t <dy_t, y_t> + <dsT, S_T> with respect to every input of the
 * recurrence above, by the chain rule through each step (the pages print no
 * backward; this is the derivative of the forward definition).  Writing
 * G = dL/dS_t and sweeping t = T .. 1 from G = dsT:
 *
 *   G    += dy_t r_t^T                      (y_t = S_t r_t)
 *   dr_t  = S_t^T dy_t
 *   dv_t  = G k_t,            dk_t = G^T v_t
 *   q     = G b_t,            p    = S_{t-1} a_t
 *   da_t  = S_{t-1}^T q,      db_t = G^T p
 *   dw_t[j] = sum_i G[i][j] S_{t-1}[i][j]
 *   dl_t[j] = dw_t[j] * (-exp(l_t[j]) w_t[j])   (w = exp(-exp(l)))
 *   G     <- G diag(w_t) + q a_t^T          (dL/dS_{t-1})
 *
 * and ds0 = G at the end.  Every state S_0 .. S_T of the unit is kept.
 *
 * Layouts (all double, contiguous, the fastest index last):
 *  dense  (seq_offsets == NULL): r, w_log, k, v, a, b, y are [B][T][H][D]
 *  packed (seq_offsets != NULL): they are [T][H][D] with T the packed length and
 *          sequence n occupying tokens [seq_offsets[n], seq_offsets[n+1]).
 *  s0, sT: [B][H][D][D] with S[i][j], i = value, j = key.  s0 == NULL means a
 *          zero initial state; sT == NULL means the final state is not stored.
 */
#include <math.h>
#include <pthread.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    const double *r, *w_log, *k, *v, *a, *b, *s0;
    double *y, *sT;
    int B, T, H, D;
    const int32_t *seq_offsets;
    long next_unit; /* shared work counter, guarded by lock */
    pthread_mutex_t lock;
    int status;
} oracle_job;

/* One (sequence, head) unit: tokens [t_begin, t_end) of the token axis. */
static void run_unit(const oracle_job *job, int n, int h, long t_begin, long t_end,
                     long token_stride, double *S, double *sa, double *w) {
    const int D = job->D;
    const long head_off = (long)h * D;
    if (job->s0) {
        memcpy(S, job->s0 + ((long)n * job->H + h) * D * D, sizeof(double) * D * D);
    } else {
        memset(S, 0, sizeof(double) * D * D);
    }
    for (long t = t_begin; t < t_end; ++t) {
        const long off = t * token_stride + head_off;
        const double *r = job->r + off, *wl = job->w_log + off, *k = job->k + off;
        const double *v = job->v + off, *a = job->a + off, *b = job->b + off;
        for (int j = 0; j < D; ++j) w[j] = exp(-exp(wl[j]));
        for (int i = 0; i < D; ++i) {
            double acc = 0.0;
            for (int j = 0; j < D; ++j) acc += S[i * D + j] * a[j];
            sa[i] = acc;
        }
        for (int i = 0; i < D; ++i)
            for (int j = 0; j < D; ++j)
                S[i * D + j] = S[i * D + j] * w[j] + sa[i] * b[j] + v[i] * k[j];
        if (job->y) {
            double *y = job->y + off;
            for (int i = 0; i < D; ++i) {
                double acc = 0.0;
                for (int j = 0; j < D; ++j) acc += S[i * D + j] * r[j];
                y[i] = acc;
            }
        }
    }
    if (job->sT) memcpy(job->sT + ((long)n * job->H + h) * D * D, S, sizeof(double) * D * D);
}

static void *worker(void *arg) {
    oracle_job *job = (oracle_job *)arg;
    const int D = job->D;
    double *S = (double *)malloc(sizeof(double) * D * D);
    double *sa = (double *)malloc(sizeof(double) * D);
    double *w = (double *)malloc(sizeof(double) * D);
    if (!S || !sa || !w) {
        pthread_mutex_lock(&job->lock);
        job->status = -2;
        pthread_mutex_unlock(&job->lock);
        free(S); free(sa); free(w);
        return NULL;
    }
    const long n_units = (long)job->B * job->H;
    for (;;) {
        pthread_mutex_lock(&job->lock);
        long u = job->next_unit++;
        pthread_mutex_unlock(&job->lock);
        if (u >= n_units) break;
        const int n = (int)(u / job->H), h = (int)(u % job->H);
        long t_begin, t_end, token_stride;
        if (job->seq_offsets) {
            t_begin = job->seq_offsets[n];
            t_end = job->seq_offsets[n + 1];
            token_stride = (long)job->H * D;
        } else {
            /* dense [B][T][H][D] viewed as a packed axis of B*T tokens */
            t_begin = (long)n * job->T;
            t_end = t_begin + job->T;
            token_stride = (long)job->H * D;
        }
        run_unit(job, n, h, t_begin, t_end, token_stride, S, sa, w);
    }
    free(S); free(sa); free(w);
    return NULL;
}

/*
 * Returns 0 on success, -1 on an invalid argument, -2 on allocation failure.
 * n_threads <= 0 means one thread.  y may be NULL (no outputs stored).
 */
int wkv7_oracle_forward(const double *r, const double *w_log, const double *k,
                        const double *v, const double *a, const double *b,
                        const double *s0, double *y, double *sT,
                        int B, int T, int H, int D, const int32_t *seq_offsets,
                        int n_threads) {
    if (!r || !w_log || !k || !v || !a || !b) return -1;
    if (B <= 0 || T < 0 || H <= 0 || D <= 0) return -1;
    if (seq_offsets) {
        if (seq_offsets[0] != 0 || seq_offsets[B] != T) return -1;
        for (int n = 0; n < B; ++n)
            if (seq_offsets[n + 1] < seq_offsets[n]) return -1;
    }
    oracle_job job;
    job.r = r; job.w_log = w_log; job.k = k; job.v = v; job.a = a; job.b = b;
    job.s0 = s0; job.y = y; job.sT = sT;
    job.B = B; job.T = T; job.H = H; job.D = D;
    job.seq_offsets = seq_offsets;
    job.next_unit = 0;
    job.status = 0;
    pthread_mutex_init(&job.lock, NULL);
    if (n_threads <= 1) {
        worker(&job);
    } else {
        pthread_t *tid = (pthread_t *)malloc(sizeof(pthread_t) * n_threads);
        if (!tid) { pthread_mutex_destroy(&job.lock); return -2; }
        int started = 0;
        for (int i = 0; i < n_threads; ++i) {
            if (pthread_create(&tid[i], NULL, worker, &job) != 0) break;
            ++started;
        }
        if (started == 0) worker(&job);
        for (int i = 0; i < started; ++i) pthread_join(tid[i], NULL);
        free(tid);
    }
    pthread_mutex_destroy(&job.lock);
    return job.status;
}

/*
 * One recurrent decoding step (a single token per sequence), the RNN mode of
 * "RWKV-7 Goose architecture analysis", section on RNN-mode inference: the
 * state [B][H][D][D] is read from s_in and written to s_out (they may alias);
 * inputs and y are [B][H][D].
 */
int wkv7_oracle_decode_step(const double *r, const double *w_log, const double *k,
                            const double *v, const double *a, const double *b,
                            const double *s_in, double *y, double *s_out,
                            int B, int H, int D, int n_threads) {
    if (!s_out) return -1;
    if (s_in && s_in != s_out)
        memmove(s_out, s_in, sizeof(double) * (size_t)B * H * D * D);
    else if (!s_in)
        memset(s_out, 0, sizeof(double) * (size_t)B * H * D * D);
    /* a dense call with T = 1 whose initial and final state are the same buffer */
    return wkv7_oracle_forward(r, w_log, k, v, a, b, s_out, y, s_out, B, 1, H, D, NULL,
                               n_threads);
}

/*
 * Gated read-out over `ntok` tokens of H heads: y, r, k, v, g, z are
 * [ntok][H][D]; rk is [H][D].  z may alias y.  Returns 0, or -1 on bad sizes.
 */
int wkv7_oracle_gate(const double *y, const double *r, const double *k, const double *v,
                     const double *rk, const double *g, double *z, long ntok, int H, int D) {
    if (ntok < 0 || H <= 0 || D <= 0) return -1;
    const double scale = 1.0 / sqrt((double)D);
    for (long t = 0; t < ntok; ++t) {
        for (int h = 0; h < H; ++h) {
            const long base = (t * H + h) * (long)D;
            double u = 0.0;
            for (int d = 0; d < D; ++d) u += r[base + d] * k[base + d] * rk[(long)h * D + d];
            for (int i = 0; i < D; ++i) z[base + i] = (y[base + i] * scale + u * v[base + i]) * g[base + i];
        }
    }
    return 0;
}

/* The prologue above, per token and head.  k, v: [ntok][H_kv][D]; w_log, a_lr
 * and the outputs k_out, v_out, a_out, b_out: [ntok][H][D]. */
int wkv7_oracle_prologue(const double *k, const double *v, const double *w_log, const double *a_lr,
                         double *k_out, double *v_out, double *a_out, double *b_out, long ntok, int H, int H_kv,
                         int D) {
    if (ntok < 0 || H <= 0 || H_kv <= 0 || D <= 0 || H % H_kv != 0) return -1;
    const int rep = H / H_kv;
    for (long t = 0; t < ntok; ++t) {
        for (int h = 0; h < H; ++h) {
            const long src = (t * H_kv + h / rep) * (long)D;
            const long dst = (t * H + h) * (long)D;
            double ss = 0.0;
            for (int d = 0; d < D; ++d) ss += k[src + d] * k[src + d];
            const double nrm = sqrt(ss);
            const double den = nrm > 1e-12 ? nrm : 1e-12;
            for (int d = 0; d < D; ++d) {
                const double w = exp(-exp(w_log[dst + d]));
                const double kk = k[src + d] / den;
                k_out[dst + d] = k[src + d] * (1.0 - w + a_lr[dst + d]);
                v_out[dst + d] = v[src + d];
                a_out[dst + d] = -kk;
                b_out[dst + d] = kk * a_lr[dst + d];
            }
        }
    }
    return 0;
}

typedef struct {
    const double *r, *w_log, *k, *v, *a, *b, *s0, *dy, *dsT;
    double *dr, *dw_log, *dk, *dv, *da, *db, *ds0;
    int B, T, H, D;
    const int32_t *seq_offsets;
    long next_unit;
    pthread_mutex_t lock;
    int status;
} oracle_bwd_job;

static int bwd_unit(const oracle_bwd_job *jb, int n, int h) {
    const int D = jb->D, H = jb->H;
    long t0, t1;
    if (jb->seq_offsets) {
        t0 = jb->seq_offsets[n];
        t1 = jb->seq_offsets[n + 1];
    } else {
        t0 = (long)n * jb->T;
        t1 = t0 + jb->T;
    }
    const long len = t1 - t0, DD = (long)D * D, stride = (long)H * D, hoff = (long)h * D;
    double *S = (double *)malloc(sizeof(double) * DD * (len + 1)); /* S_0 .. S_len */
    double *G = (double *)malloc(sizeof(double) * DD);
    double *w = (double *)malloc(sizeof(double) * D);
    double *q = (double *)malloc(sizeof(double) * D);
    double *pv = (double *)malloc(sizeof(double) * D);
    if (!S || !G || !w || !q || !pv) {
        free(S); free(G); free(w); free(q); free(pv);
        return -2;
    }
    const long sb = ((long)n * H + h) * DD;
    if (jb->s0) memcpy(S, jb->s0 + sb, sizeof(double) * DD);
    else memset(S, 0, sizeof(double) * DD);
    /* forward, keeping every state */
    for (long t = 0; t < len; ++t) {
        const long off = (t0 + t) * stride + hoff;
        const double *Sp = S + t * DD;
        double *Sn = S + (t + 1) * DD;
        for (int j = 0; j < D; ++j) w[j] = exp(-exp(jb->w_log[off + j]));
        for (int i = 0; i < D; ++i) {
            double acc = 0.0;
            for (int j = 0; j < D; ++j) acc += Sp[i * D + j] * jb->a[off + j];
            pv[i] = acc;
        }
        for (int i = 0; i < D; ++i)
            for (int j = 0; j < D; ++j)
                Sn[i * D + j] = Sp[i * D + j] * w[j] + pv[i] * jb->b[off + j] + jb->v[off + i] * jb->k[off + j];
    }
    /* backward */
    if (jb->dsT) memcpy(G, jb->dsT + sb, sizeof(double) * DD);
    else memset(G, 0, sizeof(double) * DD);
    for (long t = len - 1; t >= 0; --t) {
        const long off = (t0 + t) * stride + hoff;
        const double *Sp = S + t * DD, *St = S + (t + 1) * DD;
        const double *r = jb->r + off, *k = jb->k + off, *v = jb->v + off, *a = jb->a + off, *b = jb->b + off;
        const double *dy = jb->dy + off, *wl = jb->w_log + off;
        for (int i = 0; i < D; ++i)
            for (int j = 0; j < D; ++j) G[i * D + j] += dy[i] * r[j];
        for (int j = 0; j < D; ++j) {
            double acc = 0.0;
            for (int i = 0; i < D; ++i) acc += St[i * D + j] * dy[i];
            jb->dr[off + j] = acc;
        }
        for (int i = 0; i < D; ++i) {
            double gk = 0.0, gb = 0.0, sa = 0.0;
            for (int j = 0; j < D; ++j) {
                gk += G[i * D + j] * k[j];
                gb += G[i * D + j] * b[j];
                sa += Sp[i * D + j] * a[j];
            }
            jb->dv[off + i] = gk;
            q[i] = gb;
            pv[i] = sa;
        }
        for (int j = 0; j < D; ++j) {
            double gv = 0.0, sq = 0.0, gp = 0.0, gs = 0.0;
            for (int i = 0; i < D; ++i) {
                gv += G[i * D + j] * v[i];
                sq += Sp[i * D + j] * q[i];
                gp += G[i * D + j] * pv[i];
                gs += G[i * D + j] * Sp[i * D + j];
            }
            jb->dk[off + j] = gv;
            jb->da[off + j] = sq;
            jb->db[off + j] = gp;
            w[j] = exp(-exp(wl[j]));
            jb->dw_log[off + j] = gs * (-exp(wl[j]) * w[j]);
        }
        for (int i = 0; i < D; ++i)
            for (int j = 0; j < D; ++j) G[i * D + j] = G[i * D + j] * w[j] + q[i] * a[j];
    }
    memcpy(jb->ds0 + sb, G, sizeof(double) * DD);
    free(S); free(G); free(w); free(q); free(pv);
    return 0;
}

static void *bwd_worker(void *arg) {
    oracle_bwd_job *jb = (oracle_bwd_job *)arg;
    const long n_units = (long)jb->B * jb->H;
    for (;;) {
        pthread_mutex_lock(&jb->lock);
        long u = jb->next_unit++;
        pthread_mutex_unlock(&jb->lock);
        if (u >= n_units) break;
        if (bwd_unit(jb, (int)(u / jb->H), (int)(u % jb->H)) != 0) {
            pthread_mutex_lock(&jb->lock);
            jb->status = -2;
            pthread_mutex_unlock(&jb->lock);
        }
    }
    return NULL;
}

/* Layouts as for wkv7_oracle_forward; dy and the input gradients share the
 * layout of r, dsT and ds0 that of the states.  s0 == NULL: zero initial state;
 * dsT == NULL: no gradient on the final state. */
int wkv7_oracle_backward(const double *r, const double *w_log, const double *k, const double *v, const double *a,
                         const double *b, const double *s0, const double *dy, const double *dsT, double *dr,
                         double *dw_log, double *dk, double *dv, double *da, double *db, double *ds0, int B, int T,
                         int H, int D, const int32_t *seq_offsets, int n_threads) {
    if (B <= 0 || T < 0 || H <= 0 || D <= 0) return -1;
    if (seq_offsets) {
        if (seq_offsets[0] != 0 || seq_offsets[B] != T) return -1;
        for (int n = 0; n < B; ++n)
            if (seq_offsets[n + 1] < seq_offsets[n]) return -1;
    }
    oracle_bwd_job jb;
    jb.r = r; jb.w_log = w_log; jb.k = k; jb.v = v; jb.a = a; jb.b = b; jb.s0 = s0; jb.dy = dy; jb.dsT = dsT;
    jb.dr = dr; jb.dw_log = dw_log; jb.dk = dk; jb.dv = dv; jb.da = da; jb.db = db; jb.ds0 = ds0;
    jb.B = B; jb.T = T; jb.H = H; jb.D = D; jb.seq_offsets = seq_offsets;
    jb.next_unit = 0;
    jb.status = 0;
    pthread_mutex_init(&jb.lock, NULL);
    if (n_threads < 1) n_threads = 1;
    if (n_threads > 256) n_threads = 256;
    pthread_t tid[256];
    int started = 0;
    for (int i = 0; i < n_threads - 1; ++i) {
        if (pthread_create(&tid[i], NULL, bwd_worker, &jb) != 0) break;
        ++started;
    }
    bwd_worker(&jb);
    for (int i = 0; i < started; ++i) pthread_join(tid[i], NULL);
    pthread_mutex_destroy(&jb.lock);
    return jb.status;
}
