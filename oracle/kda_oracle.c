/*
 * KDA recurrence oracle -- TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT PATH.
 *
 * A plain, slow, fp64, token-by-token CPU implementation of the Kimi Delta Attention
 * (KDA) recurrence.  Only the tests, the package's smoke check and the benchmark's
 * CPU-baseline leg may load it.  It shares no code, header or helper with the CUDA
 * library; the two only consume the same seeded input bytes.
 *
 * What it computes, per (batch b, head h), with state S in R^{dk x dv}:
 *
 *     S   <- S0 (or 0)
 *     for t = 1..T:
 *         S[i][:] <- exp(g_t[i]) * S[i][:]            per-channel forget gate (decay first)
 *         p       <- S^T k_t                          prediction from the decayed memory
 *         u       <- beta_t * (v_t - p)               delta-rule residual
 *         S       <- S + k_t u^T                      rank-1 correction
 *         o_t     <- S^T q_t                          read-out from the updated state
 *
 * which is S_t = (I - beta_t k_t k_t^T) Diag(exp g_t) S_{t-1} + beta_t k_t v_t^T and
 * o_t = S_t^T q_t.  Sources on the pages:
 *   - "Day 21" course page (ai.air7.fun), interview item D19: linear attention keeps a
 *     fixed d x d state, KDA adds a delta-rule residual update and a per-channel decay gate;
 *   - same page, quiz Q8: the state is built from k^T v products (so S is dk x dv and the
 *     read-out is S^T q);
 *   - same page, quiz Q9: the old memory first predicts the current value, and only the
 *     residual v - S k overwrites the state (the page writes it without the gate; the
 *     gated form applies the decay before the prediction, as in Gated DeltaNet, which the
 *     podcast show-notes list under section 2.1);
 *   - skill card (skillsmp.com), quick facts: the log-decay is a bounded scaled sigmoid,
 *     g in [-5, 0).  The oracle takes g as given and does not clamp it.
 * Readings the pages leave open (no 1/sqrt(d) query scale; o_t from the post-update
 * state; beta one scalar per token and head) are the plainest ones and are pinned by
 * the single-token closed form o_1 = beta (q.k) v in the tests.
 *
 * Layouts (row-major, contiguous): q,k,g [B,T,H,dk]; v,o [B,T,H,dv]; beta [B,T,H];
 * S0, ST [B,H,dk,dv].  S0 may be NULL (zero state), ST may be NULL (not returned).
 * Intermediate states (kda_oracle_forward_states): S_mid [B,H,T/interval,dk,dv].
 * Decode: q,k,g [B,H,dk]; v,o [B,H,dv]; beta [B,H]; S [B,H,dk,dv] updated in place.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* One token of the recurrence on one head's state S (dk x dv, row-major). */
static void oracle_token(double* S, const double* q, const double* k, const double* v,
                         const double* g, double beta, double* o, double* p, long dk, long dv)
{
    long i, c;
    /* decay: S <- Diag(exp g) S */
    for (i = 0; i < dk; ++i) {
        double a = exp(g[i]);
        for (c = 0; c < dv; ++c) S[i * dv + c] *= a;
    }
    /* prediction p = S^T k */
    for (c = 0; c < dv; ++c) p[c] = 0.0;
    for (i = 0; i < dk; ++i)
        for (c = 0; c < dv; ++c) p[c] += S[i * dv + c] * k[i];
    /* residual u = beta (v - p), stored back into p */
    for (c = 0; c < dv; ++c) p[c] = beta * (v[c] - p[c]);
    /* S <- S + k u^T */
    for (i = 0; i < dk; ++i)
        for (c = 0; c < dv; ++c) S[i * dv + c] += k[i] * p[c];
    /* o = S^T q */
    for (c = 0; c < dv; ++c) o[c] = 0.0;
    for (i = 0; i < dk; ++i)
        for (c = 0; c < dv; ++c) o[c] += S[i * dv + c] * q[i];
}

/*
 * The whole sequence for every (b, h).  When S_mid is not NULL it also records the state
 * after every `interval` tokens: the boundaries at which a prefix cache can resume the
 * recurrence (podcast show-notes (scripod.com), outline item 5.3.1 "KDA-Aware Prefix Cache
 * Management"; the channel post on the K3 report (t.iss.one), online-inference paragraph:
 * prefixes are reused at 512-token boundaries).  S_mid is [B, H, T / interval, dk, dv] and
 * entry n holds the state after tokens 1 .. (n+1)*interval.
 */
static int oracle_forward_impl(const double* q, const double* k, const double* v, const double* g,
                               const double* beta, const double* S0, double* o, double* ST,
                               double* S_mid, long interval, long B, long T, long H, long dk,
                               long dv, int nthreads)
{
    long bh;
    const long n_mid = (S_mid && interval > 0) ? T / interval : 0;
    if (B < 0 || T < 0 || H < 0 || dk <= 0 || dv <= 0) return -1;
    if (S_mid && interval <= 0) return -1;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (bh = 0; bh < B * H; ++bh) {
        long b = bh / H, h = bh % H, t;
        double* S = (double*)malloc(sizeof(double) * (size_t)(dk * dv + dv));
        double* p = S + dk * dv;
        if (S0) memcpy(S, S0 + bh * dk * dv, sizeof(double) * (size_t)(dk * dv));
        else memset(S, 0, sizeof(double) * (size_t)(dk * dv));
        for (t = 0; t < T; ++t) {
            long row = (b * T + t) * H + h;
            oracle_token(S, q + row * dk, k + row * dk, v + row * dv, g + row * dk, beta[row],
                         o + row * dv, p, dk, dv);
            if (n_mid > 0 && (t + 1) % interval == 0)
                memcpy(S_mid + (bh * n_mid + (t + 1) / interval - 1) * dk * dv, S,
                       sizeof(double) * (size_t)(dk * dv));
        }
        if (ST) memcpy(ST + bh * dk * dv, S, sizeof(double) * (size_t)(dk * dv));
        free(S);
    }
    return 0;
}

int kda_oracle_forward(const double* q, const double* k, const double* v, const double* g,
                       const double* beta, const double* S0, double* o, double* ST,
                       long B, long T, long H, long dk, long dv, int nthreads)
{
    return oracle_forward_impl(q, k, v, g, beta, S0, o, ST, NULL, 0, B, T, H, dk, dv, nthreads);
}

int kda_oracle_forward_states(const double* q, const double* k, const double* v, const double* g,
                              const double* beta, const double* S0, double* o, double* ST,
                              double* S_mid, long interval, long B, long T, long H, long dk,
                              long dv, int nthreads)
{
    if (!S_mid) return -1;
    return oracle_forward_impl(q, k, v, g, beta, S0, o, ST, S_mid, interval, B, T, H, dk, dv,
                               nthreads);
}

int kda_oracle_decode_step(const double* q, const double* k, const double* v, const double* g,
                           const double* beta, double* S, double* o, long B, long H, long dk,
                           long dv, int nthreads)
{
    long bh;
    if (B < 0 || H < 0 || dk <= 0 || dv <= 0) return -1;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(static)
#endif
    for (bh = 0; bh < B * H; ++bh) {
        double* p = (double*)malloc(sizeof(double) * (size_t)dv);
        oracle_token(S + bh * dk * dv, q + bh * dk, k + bh * dk, v + bh * dv, g + bh * dk,
                     beta[bh], o + bh * dv, p, dk, dv);
        free(p);
    }
    return 0;
}

int kda_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
