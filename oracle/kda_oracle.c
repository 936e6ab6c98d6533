/*
 * kda_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * Plain, slow, float64 CPU restatement of the Kimi Delta Attention (KDA)
 * recurrence, used to check the CUDA library.  Only tests/, the smoke entry
 * point and the bench's cpu_baseline / reference arm may load it; the
 * product path never does.  It shares no code, header or constant with the
 * CUDA library.
 *
 * Definition followed ("You could have come up with Kimi Delta Attention",
 * gokawiil.com repost, the five-equation KDA state update at the top of the
 * article; the same five steps are listed in the GeekNews summary, section
 * "Kimi Delta Attention: per-channel decay"):
 *
 *     S~_t  = S_{t-1} Diag(alpha_t)            (forget, per key channel)
 *     vhat_t = S~_t k_t                         (predict)
 *     e_t    = beta_t (v_t - vhat_t)            (correct)
 *     S_t    = S~_t + e_t k_t^T                 (write)
 *     o_t    = S_t (d_k^{-1/2} q_t)             (read, post-write state)
 *
 * S is d_v x d_k (maps key space to value space; key channels are columns).
 * The gate is stored as g = log(alpha) (GeekNews summary, end of the
 * "diagonal-plus-low-rank transition" section), so alpha = exp(g).  Gate
 * modes: per channel (g has d_k entries per token/head), scalar (one entry,
 * broadcast to every channel: Gated DeltaNet), none (alpha = 1: DeltaNet).
 *
 * Each step is its own loop nest over the whole state, in the order above;
 * nothing is fused, blocked or reordered.  OpenMP only splits independent
 * (sequence, head) pairs across threads.
 *
 * Parity pins: tests/test_oracle_pins.py.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORACLE_GATE_CHANNEL = 0, ORACLE_GATE_SCALAR = 1, ORACLE_GATE_NONE = 2 };

/* One (sequence, value head) pair: walk its tokens in order.
 * Token t of the pair lives at packed row (start + t); every per-token array
 * is [rows, heads, width] row-major: q and k have Hk heads (value head h reads
 * q/k head hk), v, g, beta and the state have H. */
static void oracle_one_pair(int64_t start, int64_t len, int h, int H, int hk, int Hk, int dk, int dv,
                            int gate_mode, const double* q, const double* k,
                            const double* v, const double* g, const double* beta,
                            const double* S0 /* dv*dk or NULL */, double* out,
                            double* ST /* dv*dk or NULL */, double* S, double* alpha,
                            double* vhat, double* e)
{
    const double scale = 1.0 / sqrt((double)dk);
    if (S0) memcpy(S, S0, sizeof(double) * (size_t)dv * dk);
    else memset(S, 0, sizeof(double) * (size_t)dv * dk);

    for (int64_t t = 0; t < len; ++t) {
        const int64_t row = start + t;
        const double* kt = k + (row * Hk + hk) * dk;
        const double* qt = q + (row * Hk + hk) * dk;
        const double* vt = v + (row * H + h) * dv;
        const double bt = beta[row * H + h];

        /* alpha_t = exp(g_t) per channel */
        for (int c = 0; c < dk; ++c) {
            if (gate_mode == ORACLE_GATE_CHANNEL) alpha[c] = exp(g[(row * H + h) * dk + c]);
            else if (gate_mode == ORACLE_GATE_SCALAR) alpha[c] = exp(g[row * H + h]);
            else alpha[c] = 1.0;
        }
        /* 1. forget: S~ = S Diag(alpha)  (scales column c by alpha_c) */
        for (int r = 0; r < dv; ++r)
            for (int c = 0; c < dk; ++c) S[r * dk + c] *= alpha[c];
        /* 2. predict: vhat = S~ k */
        for (int r = 0; r < dv; ++r) {
            double acc = 0.0;
            for (int c = 0; c < dk; ++c) acc += S[r * dk + c] * kt[c];
            vhat[r] = acc;
        }
        /* 3. correct: e = beta (v - vhat) */
        for (int r = 0; r < dv; ++r) e[r] = bt * (vt[r] - vhat[r]);
        /* 4. write: S = S~ + e k^T */
        for (int r = 0; r < dv; ++r)
            for (int c = 0; c < dk; ++c) S[r * dk + c] += e[r] * kt[c];
        /* 5. read: o = S (d_k^{-1/2} q) */
        double* ot = out + (row * H + h) * dv;
        for (int r = 0; r < dv; ++r) {
            double acc = 0.0;
            for (int c = 0; c < dk; ++c) acc += S[r * dk + c] * (scale * qt[c]);
            ot[r] = acc;
        }
    }
    if (ST) memcpy(ST, S, sizeof(double) * (size_t)dv * dk);
}

/*
 * kda_oracle_forward: run the recurrence over num_seqs packed sequences.
 *   seq_start[n], seq_len[n] : token rows [seq_start[n], seq_start[n]+seq_len[n])
 *                              of the packed token axis belong to sequence n.
 *   q, k : [rows, Hk, dk]    v, out : [rows, H, dv]
 *   H a multiple of Hk: value head h reads q/k head h / (H / Hk) -- groups of
 *   consecutive value heads share one query/key head.
 *   g    : [rows, H, dk] (channel) | [rows, H] (scalar) | NULL (none)
 *   beta : [rows, H]
 *   S0   : [num_seqs, H, dv, dk] or NULL (zero initial state)
 *   ST   : [num_seqs, H, dv, dk] or NULL (final state not wanted)
 *   nthreads <= 0 : OpenMP default.
 * Returns 0 on success, -1 on a bad argument, -2 if memory runs out.
 */
int kda_oracle_forward(int num_seqs, const int64_t* seq_start, const int64_t* seq_len,
                       int H, int Hk, int dk, int dv, int gate_mode, const double* q,
                       const double* k, const double* v, const double* g,
                       const double* beta, const double* S0, double* out, double* ST,
                       int nthreads)
{
    if (num_seqs < 0 || H <= 0 || Hk <= 0 || H % Hk != 0 || dk <= 0 || dv <= 0) return -1;
    if (gate_mode < 0 || gate_mode > 2) return -1;
    if (gate_mode != ORACLE_GATE_NONE && g == NULL) return -1;
    if (!q || !k || !v || !beta || !out || !seq_start || !seq_len) return -1;
    for (int n = 0; n < num_seqs; ++n)
        if (seq_len[n] < 0 || seq_start[n] < 0) return -1;

    const int64_t pairs = (int64_t)num_seqs * H;
    int failed = 0;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
#pragma omp parallel for schedule(dynamic, 1) reduction(| : failed)
    for (int64_t p = 0; p < pairs; ++p) {
        const int n = (int)(p / H), h = (int)(p % H);
        const int hk = h / (H / Hk);
        const size_t soff = (size_t)p * dv * dk;
        double* S = (double*)malloc(sizeof(double) * (size_t)dv * dk);
        double* alpha = (double*)malloc(sizeof(double) * (size_t)dk);
        double* vhat = (double*)malloc(sizeof(double) * (size_t)dv);
        double* e = (double*)malloc(sizeof(double) * (size_t)dv);
        if (S && alpha && vhat && e)
            oracle_one_pair(seq_start[n], seq_len[n], h, H, hk, Hk, dk, dv, gate_mode, q, k, v, g,
                            beta, S0 ? S0 + soff : NULL, out, ST ? ST + soff : NULL, S,
                            alpha, vhat, e);
        else
            failed = 1;
        free(S);
        free(alpha);
        free(vhat);
        free(e);
    }
    return failed ? -2 : 0;
}

/* Number of OpenMP threads a parallel region would use (for reporting). */
int kda_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
