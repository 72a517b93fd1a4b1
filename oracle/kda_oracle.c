/*
 * KDA (Kimi Delta Attention) reference recurrence -- TEST INFRASTRUCTURE ONLY.
 *
 * This is the oracle: a plain, slow, sequential fp64 CPU loop that the CUDA
 * library is checked against.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark may load it; the library never does.  It
 * shares no code, header or helper with the CUDA path.
 *
 * What it computes, per (sequence b, head h), for t = 0 .. T-1, with the state
 * S in R^{d_k x d_v} (rows = key channels, columns = value channels):
 *
 *   (1) forget   S~  = Diag(alpha_t) S_{t-1}
 *   (2) predict  vh  = S~^T k_t
 *   (3) correct  e   = v_t - vh
 *   (4) write    S_t = S~ + beta_t k_t e^T
 *   (5) read     o_t = S_t^T (scale q_t)
 *
 * This is the five-step update of "Module 03 -- KDA I: The Delta-Rule
 * Recurrence", section 2 ("The five-step update"), with the query scale of the
 * statement that opens "Kimi Delta Attention (KDA)" (brain.bigb.es) applied to
 * q at the read only, in the d_k x d_v layout of that page's five-line code
 * ("KDA: one gate per key channel").
 *
 * Modes (for the tests' pins only):
 *   KDA_REF_EXACT            the recurrence above.
 *   KDA_REF_DROP_CORRECTION  vh := 0, i.e. S_t = Diag(alpha) S + beta k v^T.
 *                            With alpha = beta = 1 this is additive linear
 *                            attention ("Dropping the softmax turns attention
 *                            into a state", brain.bigb.es).
 *   KDA_REF_SWAP_ORDER       the wrong operator order that "Module 03",
 *                            section 3 warns about:
 *                            S_t = Diag(alpha) (I - beta k k^T) S + beta k v^T.
 *   KDA_REF_PREDICT_FIRST    a planted mistake: the prediction reads the
 *                            undecayed S_{t-1} ("Predicting before forgetting",
 *                            "Gated DeltaNet: sometimes everything should
 *                            fade", brain.bigb.es).
 *
 * Decoupled erase and write gates (kda_ref_forward_gdn2): "From Fast Weight
 * Programmers to KDA" (jonahsamost.bearblog.dev), section "Gated DeltaNet-2",
 * replaces beta_t by a per-key-channel erase gate b_t and a per-value-channel
 * write gate w_t.  That page writes the state as d_v x d_k; in the d_k x d_v
 * layout used here its update reads
 *
 *   (1) forget   S~  = Diag(alpha_t) S_{t-1}
 *   (2) predict  vh  = S~^T (b_t * k_t)          retrieval through the gated key
 *   (3) correct  e   = w_t * v_t - vh            the residual of the gated value
 *   (4) write    S_t = S~ + k_t e^T              stored at the original key
 *   (5) read     o_t = S_t^T (scale q_t)
 *
 * (* is the elementwise product).  b_t = beta_t 1, w_t = beta_t 1 gives the
 * KDA update above.
 *
 * Layouts (row-major, contiguous):
 *   q, k, alpha : [B, T, H, d_k]      v, o : [B, T, H, d_v]
 *   beta        : [B, T, H]           s0, s_final : [B, H, d_k, d_v]
 * s0 may be NULL (zero initial state).  s_final may be NULL.
 * Work is split over (b, h) across n_threads POSIX threads (<= 0: one per
 * online core).  Returns 0 on success, -1 on bad arguments, -2 on allocation
 * failure.
 */
#include <pthread.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#define KDA_REF_EXACT 0
#define KDA_REF_DROP_CORRECTION 1
#define KDA_REF_SWAP_ORDER 2
#define KDA_REF_PREDICT_FIRST 3

typedef struct {
    const double *q, *k, *v, *alpha, *beta, *s0;
    const double *erase, *wgate;   /* GDN-2 gates [B,T,H,d_k], [B,T,H,d_v], or NULL */
    double *o, *s_final;
    int B, T, H, dk, dv, mode;
    double scale;
    int next_item;          /* next (b, h) index to hand out */
    int failed;
    pthread_mutex_t lock;
} ref_job;

static int run_head(ref_job *J, int b, int h)
{
    const int dk = J->dk, dv = J->dv, T = J->T, H = J->H;
    double *S = (double *)malloc(sizeof(double) * (size_t)dk * dv);
    double *vh = (double *)malloc(sizeof(double) * (size_t)dv);
    double *e = (double *)malloc(sizeof(double) * (size_t)dv);
    if (!S || !vh || !e) {
        free(S); free(vh); free(e);
        return -2;
    }
    const size_t sbase = ((size_t)b * H + h) * (size_t)dk * dv;
    if (J->s0)
        memcpy(S, J->s0 + sbase, sizeof(double) * (size_t)dk * dv);
    else
        memset(S, 0, sizeof(double) * (size_t)dk * dv);

    for (int t = 0; t < T; ++t) {
        const size_t row = ((size_t)b * T + t) * H + h;   /* token-head index */
        const double *qt = J->q + row * dk;
        const double *kt = J->k + row * dk;
        const double *at = J->alpha + row * dk;
        const double *vt = J->v + row * dv;
        const double bt = J->beta ? J->beta[row] : 0.0;
        double *ot = J->o + row * dv;

        if (J->erase) {
            /* GDN-2: (1) forget, (2) predict through b * k, (3) correct, (4) write */
            const double *bk = J->erase + row * dk;
            const double *wv = J->wgate + row * dv;
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j)
                    S[(size_t)i * dv + j] *= at[i];
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int i = 0; i < dk; ++i) acc += S[(size_t)i * dv + j] * (bk[i] * kt[i]);
                vh[j] = acc;
            }
            for (int j = 0; j < dv; ++j) e[j] = wv[j] * vt[j] - vh[j];
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j)
                    S[(size_t)i * dv + j] += kt[i] * e[j];
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int i = 0; i < dk; ++i) acc += S[(size_t)i * dv + j] * (J->scale * qt[i]);
                ot[j] = acc;
            }
            continue;
        }

        if (J->mode == KDA_REF_SWAP_ORDER) {
            /* (I - beta k k^T) applied to the undecayed state ... */
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int i = 0; i < dk; ++i) acc += S[(size_t)i * dv + j] * kt[i];
                vh[j] = acc;
            }
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j)
                    S[(size_t)i * dv + j] -= bt * kt[i] * vh[j];
            /* ... and only then the decay, then the write of beta k v^T. */
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j)
                    S[(size_t)i * dv + j] = at[i] * S[(size_t)i * dv + j] + bt * kt[i] * vt[j];
        } else {
            if (J->mode == KDA_REF_PREDICT_FIRST) {
                for (int j = 0; j < dv; ++j) {
                    double acc = 0.0;
                    for (int i = 0; i < dk; ++i) acc += S[(size_t)i * dv + j] * kt[i];
                    vh[j] = acc;
                }
            }
            /* (1) forget: row i of S is key channel i */
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j)
                    S[(size_t)i * dv + j] *= at[i];
            /* (2) predict */
            if (J->mode == KDA_REF_EXACT) {
                for (int j = 0; j < dv; ++j) {
                    double acc = 0.0;
                    for (int i = 0; i < dk; ++i) acc += S[(size_t)i * dv + j] * kt[i];
                    vh[j] = acc;
                }
            } else if (J->mode == KDA_REF_DROP_CORRECTION) {
                for (int j = 0; j < dv; ++j) vh[j] = 0.0;
            }
            /* (3) correct */
            for (int j = 0; j < dv; ++j) e[j] = vt[j] - vh[j];
            /* (4) write */
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j)
                    S[(size_t)i * dv + j] += bt * kt[i] * e[j];
        }
        /* (5) read */
        for (int j = 0; j < dv; ++j) {
            double acc = 0.0;
            for (int i = 0; i < dk; ++i) acc += S[(size_t)i * dv + j] * (J->scale * qt[i]);
            ot[j] = acc;
        }
    }
    if (J->s_final)
        memcpy(J->s_final + sbase, S, sizeof(double) * (size_t)dk * dv);
    free(S); free(vh); free(e);
    return 0;
}

static void *worker(void *arg)
{
    ref_job *J = (ref_job *)arg;
    const int n_items = J->B * J->H;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        const int item = J->next_item++;
        pthread_mutex_unlock(&J->lock);
        if (item >= n_items) break;
        if (run_head(J, item / J->H, item % J->H) != 0) {
            pthread_mutex_lock(&J->lock);
            J->failed = 1;
            pthread_mutex_unlock(&J->lock);
        }
    }
    return NULL;
}

static int run_job(ref_job *Jp, int n_threads);

int kda_ref_forward(const double *q, const double *k, const double *v,
                    const double *alpha, const double *beta, const double *s0,
                    double *o, double *s_final, int B, int T, int H, int dk,
                    int dv, double scale, int mode, int n_threads)
{
    if (!q || !k || !v || !alpha || !beta || !o) return -1;
    if (B < 0 || T < 0 || H < 0 || dk <= 0 || dv <= 0) return -1;
    if (mode < KDA_REF_EXACT || mode > KDA_REF_PREDICT_FIRST) return -1;
    ref_job J;
    J.q = q; J.k = k; J.v = v; J.alpha = alpha; J.beta = beta; J.s0 = s0;
    J.erase = NULL; J.wgate = NULL;
    J.o = o; J.s_final = s_final;
    J.B = B; J.T = T; J.H = H; J.dk = dk; J.dv = dv; J.mode = mode;
    J.scale = scale;
    return run_job(&J, n_threads);
}

/* GDN-2: erase [B,T,H,d_k] and write [B,T,H,d_v] gates instead of beta. */
int kda_ref_forward_gdn2(const double *q, const double *k, const double *v,
                         const double *alpha, const double *erase, const double *wgate,
                         const double *s0, double *o, double *s_final, int B, int T,
                         int H, int dk, int dv, double scale, int n_threads)
{
    if (!q || !k || !v || !alpha || !erase || !wgate || !o) return -1;
    if (B < 0 || T < 0 || H < 0 || dk <= 0 || dv <= 0) return -1;
    ref_job J;
    J.q = q; J.k = k; J.v = v; J.alpha = alpha; J.beta = NULL; J.s0 = s0;
    J.erase = erase; J.wgate = wgate;
    J.o = o; J.s_final = s_final;
    J.B = B; J.T = T; J.H = H; J.dk = dk; J.dv = dv; J.mode = KDA_REF_EXACT;
    J.scale = scale;
    return run_job(&J, n_threads);
}

static int run_job(ref_job *Jp, int n_threads)
{
    ref_job J = *Jp;
    J.next_item = 0; J.failed = 0;
    pthread_mutex_init(&J.lock, NULL);
    const int B = J.B, H = J.H;

    const int n_items = B * H;
    if (n_threads <= 0) n_threads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (n_threads < 1) n_threads = 1;
    if (n_threads > n_items) n_threads = n_items;
    if (n_threads <= 1) {
        worker(&J);
    } else {
        pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)n_threads);
        if (!th) { pthread_mutex_destroy(&J.lock); return -2; }
        int started = 0;
        for (; started < n_threads; ++started)
            if (pthread_create(&th[started], NULL, worker, &J) != 0) break;
        if (started == 0) worker(&J);
        for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
        free(th);
    }
    pthread_mutex_destroy(&J.lock);
    return J.failed ? -2 : 0;
}
