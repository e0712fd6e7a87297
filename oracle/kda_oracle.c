/*
 * KDA oracle: plain fp64 CPU token-by-token recurrence.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the correctness oracle for the CUDA
 * path.  Only the test suite, the smoke check and the CPU-baseline leg of the
 * benchmark may load it.  It shares no code, header or constant with the
 * library under gated_delta_rule_124_b200/.
 *
 * What it computes (Kimi Linear, aiwiki.ai; sections "Background: from the
 * delta rule to gated DeltaNet", "Kimi Delta Attention" and "The constrained
 * DPLR form and the chunkwise algorithm"):
 *
 *   KDA is the gated delta rule whose scalar forget gate is replaced by a
 *   diagonal, per-channel gate.  Per (sequence, head) it keeps a state
 *   S (dk x dv) and, for every token t,
 *
 *       S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *       o_t = S_t^T q_t
 *
 *   with alpha_t = exp(g_t) given per channel as g = log(alpha).
 *
 * The update is evaluated in the order the formula is written: decay first
 * (Sbar = Diag(alpha) S), then the delta-rule correction against the decayed
 * state ("read what the state predicts for k, store the difference"):
 *
 *       p     = Sbar^T k
 *       S_t   = Sbar + beta k (v - p)^T
 *
 * which is algebraically the same matrix as the formula above, expanded as a
 * rank-1 update instead of a dk x dk product.  The output uses the state after
 * the update.  No query scale is applied (none is stated).
 *
 * Layouts (all row-major, C order):
 *   q, k, g   [total_tokens, H, dk]
 *   v, o      [total_tokens, H, dv]
 *   beta      [total_tokens, H]
 *   states    [num_seqs, H, dk, dv]   (S[c][j] multiplies k_c on the left)
 *   cu_seqlens [num_seqs + 1], cu_seqlens[0] = 0, non-decreasing,
 *              cu_seqlens[num_seqs] = total_tokens.
 *
 * Every floating-point value is double.  Inputs that were bf16 or fp32 on the
 * GPU side are widened to double exactly by the caller, so input rounding is
 * never counted as kernel error.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Return codes: 0 ok, 1 invalid argument, 2 out of memory. */

static int check_cu(const int32_t* cu, int num_seqs, int total_tokens) {
    if (cu[0] != 0 || cu[num_seqs] != total_tokens) return 1;
    for (int s = 0; s < num_seqs; ++s)
        if (cu[s + 1] < cu[s]) return 1;
    return 0;
}

/* One token of the recurrence on one (sequence, head) state S[dk][dv].
 * a, kv, vv, qv are that token's alpha (already exp'd), k, v, q rows; p is
 * dv doubles of scratch.  Writes o_row (dv) when it is not NULL. */
static void kda_token(double* S, const double* a, const double* kv, const double* vv,
                      const double* qv, double beta, int dk, int dv, double* p,
                      double* o_row) {
    /* decay: Sbar = Diag(alpha) S */
    for (int c = 0; c < dk; ++c)
        for (int j = 0; j < dv; ++j) S[(size_t)c * dv + j] *= a[c];
    /* prediction of the decayed state for key k: p = Sbar^T k */
    for (int j = 0; j < dv; ++j) {
        double acc = 0.0;
        for (int c = 0; c < dk; ++c) acc += kv[c] * S[(size_t)c * dv + j];
        p[j] = acc;
    }
    /* store the difference: S = Sbar + k (beta (v - p))^T */
    for (int j = 0; j < dv; ++j) p[j] = beta * (vv[j] - p[j]);
    for (int c = 0; c < dk; ++c)
        for (int j = 0; j < dv; ++j) S[(size_t)c * dv + j] += kv[c] * p[j];
    /* read-out with the updated state: o = S^T q */
    if (o_row) {
        for (int j = 0; j < dv; ++j) {
            double acc = 0.0;
            for (int c = 0; c < dk; ++c) acc += qv[c] * S[(size_t)c * dv + j];
            o_row[j] = acc;
        }
    }
}

/*
 * Full forward over packed sequences.  initial_state may be NULL (zeros);
 * final_state may be NULL.  num_threads <= 0 lets OpenMP choose.
 */
int kda_ref_forward(const double* q, const double* k, const double* v, const double* g,
                    const double* beta, const double* initial_state,
                    const int32_t* cu_seqlens, int num_seqs, int total_tokens, int H,
                    int dk, int dv, double* o, double* final_state, int num_threads) {
    if (!q || !k || !v || !g || !beta || !cu_seqlens || !o) return 1;
    if (num_seqs < 1 || total_tokens < 0 || H < 1 || dk < 1 || dv < 1) return 1;
    if (check_cu(cu_seqlens, num_seqs, total_tokens)) return 1;
    int err = 0;
    const int units = num_seqs * H;
#ifdef _OPENMP
    if (num_threads > 0) omp_set_num_threads(num_threads);
#pragma omp parallel for schedule(dynamic, 1) reduction(| : err)
#endif
    for (int unit = 0; unit < units; ++unit) {
        const int s = unit / H, h = unit % H;
        double* S = (double*)malloc(sizeof(double) * (size_t)dk * dv);
        double* p = (double*)malloc(sizeof(double) * (size_t)dv);
        double* a = (double*)malloc(sizeof(double) * (size_t)dk);
        if (!S || !p || !a) {
            free(S); free(p); free(a);
            err |= 2;
            continue;
        }
        const size_t st = ((size_t)s * H + h) * dk * dv;
        if (initial_state)
            memcpy(S, initial_state + st, sizeof(double) * (size_t)dk * dv);
        else
            memset(S, 0, sizeof(double) * (size_t)dk * dv);
        for (int t = cu_seqlens[s]; t < cu_seqlens[s + 1]; ++t) {
            const size_t rk = ((size_t)t * H + h) * dk;
            const size_t rv = ((size_t)t * H + h) * dv;
            for (int c = 0; c < dk; ++c) a[c] = exp(g[rk + c]);
            kda_token(S, a, k + rk, v + rv, q + rk, beta[(size_t)t * H + h], dk, dv, p,
                      o + rv);
        }
        if (final_state) memcpy(final_state + st, S, sizeof(double) * (size_t)dk * dv);
        free(S); free(p); free(a);
    }
    return err ? 2 : 0;
}

/*
 * One recurrent decode step: one token per (sequence, head), state updated in
 * place.  q, k, g [N, H, dk]; v, o [N, H, dv]; beta [N, H]; state [N, H, dk, dv].
 */
int kda_ref_decode_step(const double* q, const double* k, const double* v, const double* g,
                        const double* beta, double* state, double* o, int N, int H, int dk,
                        int dv, int num_threads) {
    if (!q || !k || !v || !g || !beta || !state || !o) return 1;
    if (N < 0 || H < 1 || dk < 1 || dv < 1) return 1;
    int err = 0;
    const int units = N * H;
#ifdef _OPENMP
    if (num_threads > 0) omp_set_num_threads(num_threads);
#pragma omp parallel for schedule(static) reduction(| : err)
#endif
    for (int unit = 0; unit < units; ++unit) {
        double* p = (double*)malloc(sizeof(double) * (size_t)dv);
        double* a = (double*)malloc(sizeof(double) * (size_t)dk);
        if (!p || !a) {
            free(p); free(a);
            err |= 2;
            continue;
        }
        const size_t rk = (size_t)unit * dk, rv = (size_t)unit * dv;
        for (int c = 0; c < dk; ++c) a[c] = exp(g[rk + c]);
        kda_token(state + (size_t)unit * dk * dv, a, k + rk, v + rv, q + rk, beta[unit], dk,
                  dv, p, o + rv);
        free(p); free(a);
    }
    return err ? 2 : 0;
}

/* Threads an OpenMP parallel region would use (1 without OpenMP). */
int kda_ref_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
