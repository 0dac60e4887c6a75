/*
 * CPU oracle for the gated delta rule with a fake-quantized (QDQ) state.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, plain reference that the
 * CUDA path is checked against.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load it; the product path never does.  It
 * shares no code, header, table or constant with the CUDA library.
 *
 * Arithmetic: the recurrence runs in fp64 with plain loops; the QDQ codecs run
 * on the fp32-cast state in IEEE fp32 (compile without fast-math and with
 * -ffp-contract=off so every fp32 operation rounds once, as the GPU's
 * explicitly rounded intrinsics do).
 *
 * Sources (the GatedDeltaNet / KDA state-QAT pages of the "linear_attention"
 * QAT series):
 *  - token recurrence (the "recurrent suffix", recurrent_decode):
 *      H_t = diag(alpha_t) H_{t-1};  u_t = beta_t (v_t - H_t^T k_t);
 *      H_t += k_t u_t^T;  o_t = H_t^T q_t / sqrt(d_k)
 *    with H = S^T stored [d_k, d_v] (row = key, column = value), alpha_t =
 *    exp(g_t), g_t a scalar (GDN) or a d_k-vector (KDA "vector gate");
 *  - state QDQ at every 64-token chunk boundary of the prefix and after every
 *    decode token (PR #2497 "GDN state/W QAT foundation", What section; PR
 *    #2519 decode QAT);
 *  - FP8: "amax at each boundary over each full-key by 64-value-column tile,
 *    independently per sequence and head", scale = amax / 448 with a zero
 *    guard, num_bits (4,3) = E4M3 (PR #2497, What and Usage sections);
 *  - INT8: groups of 32 along the last axis (16 and 64 also allowed), scale =
 *    amax / 127, round half to even, clamp (PR #2519 commit notes, recipe
 *    linear_attention_state_int8_block32_dynamic);
 *  - fp32 working values for the state and gates (PR #2519 commit notes).
 *
 * Readings where the pages are silent (each listed in the design notes):
 *  - the incoming state is not quantized; QDQ follows the update of the last
 *    token of each chunk (counted from each sequence's own start, the final
 *    partial chunk included) and every decode token; outputs use the pre-QDQ
 *    state;
 *  - INT8 clamps to [-127, 127]; FP8 saturates to +-448 (E4M3FN, no inf);
 *  - the scale and x/scale are IEEE fp32 divisions.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define OR_QDQ_NONE 0
#define OR_QDQ_FP8_TILE 1
#define OR_QDQ_INT8_GROUP 2

/* ---------------------------------------------------------------------------
 * E4M3FN rounding, written from the format's definition (OCP 8-bit floating
 * point, E4M3 variant "FN": 4 exponent bits with bias 7, 3 mantissa bits, no
 * infinities, only S.1111.111 is NaN).  Largest finite value 1.75 * 2^8 = 448,
 * smallest normal 2^-6, subnormal spacing 2^-9.  Rounding is to nearest with
 * ties to an even mantissa; magnitudes above 448 saturate to 448.
 * ------------------------------------------------------------------------- */
float or_e4m3_rne_satfinite(float y)
{
    if (y != y) return y; /* NaN passes through */
    double a = fabs((double)y);
    double r;
    if (a >= 448.0) {
        r = 448.0;
    } else {
        int e2;
        (void)frexp(a, &e2);          /* a = m * 2^e2, m in [0.5, 1) */
        int binade = e2 - 1;          /* a in [2^binade, 2^(binade+1)) */
        double quantum = (binade < -6) ? ldexp(1.0, -9) : ldexp(1.0, binade - 3);
        if (a == 0.0) quantum = ldexp(1.0, -9);
        /* a / quantum is an exact power-of-two scaling; nearbyint rounds to
         * nearest with ties to even under the default rounding mode, and an
         * even multiple of the quantum is an even mantissa. */
        double n = nearbyint(a / quantum);
        r = n * quantum;
        if (r > 448.0) r = 448.0;
    }
    return (float)copysign(r, (double)y);
}

/* ---------------------------------------------------------------------------
 * Dynamic FP8 E4M3 QDQ of one fp32 state X[d_k][d_v] (row = key, column =
 * value), one scale per tile of all d_k rows by `tile_cols` value columns.
 * codes/scales (optional) receive the E4M3 value of each element and the
 * scale of each tile (0 for a zero tile).
 * ------------------------------------------------------------------------- */
static void qdq_fp8_tile(float *X, int d_k, int d_v, int tile_cols,
                         float *codes, float *scales)
{
    for (int c0 = 0; c0 < d_v; c0 += tile_cols) {
        float m = 0.0f;
        for (int i = 0; i < d_k; ++i)
            for (int j = c0; j < c0 + tile_cols; ++j) {
                float a = fabsf(X[(size_t)i * d_v + j]);
                if (a > m) m = a;
            }
        if (scales) scales[c0 / tile_cols] = 0.0f;
        if (m == 0.0f) { /* zero guard: an all-zero tile stays zero */
            for (int i = 0; i < d_k; ++i)
                for (int j = c0; j < c0 + tile_cols; ++j) {
                    X[(size_t)i * d_v + j] = 0.0f;
                    if (codes) codes[(size_t)i * d_v + j] = 0.0f;
                }
            continue;
        }
        float s = m / 448.0f;
        if (scales) scales[c0 / tile_cols] = s;
        for (int i = 0; i < d_k; ++i)
            for (int j = c0; j < c0 + tile_cols; ++j) {
                float t = X[(size_t)i * d_v + j] / s;
                float c = or_e4m3_rne_satfinite(t);
                float y = c * s;
                X[(size_t)i * d_v + j] = y;
                if (codes) codes[(size_t)i * d_v + j] = c;
            }
    }
}

/* ---------------------------------------------------------------------------
 * Dynamic INT8 QDQ with groups of `group` consecutive elements.  axis = 1:
 * groups run along the value axis (the last axis of the canonical [d_k, d_v]
 * layout); axis = 0: along the key axis (the other reading of "last axis").
 * codes receive the integer code of each element (as a float); scales one
 * value per group, ordered row-major over (row, group) for axis 1 and
 * (group, column) for axis 0.
 * ------------------------------------------------------------------------- */
static void qdq_int8_group(float *X, int d_k, int d_v, int group, int axis,
                           float *codes, float *scales)
{
    int n_outer = axis == 1 ? d_k : d_v;       /* lines that are grouped */
    int n_inner = axis == 1 ? d_v : d_k;       /* length of a line */
    int n_groups = n_inner / group;
    for (int line = 0; line < n_outer; ++line)
        for (int gi = 0; gi < n_groups; ++gi) {
            size_t idx[64];
            for (int e = 0; e < group; ++e) {
                int pos = gi * group + e;
                idx[e] = axis == 1 ? (size_t)line * d_v + pos
                                   : (size_t)pos * d_v + line;
            }
            float m = 0.0f;
            for (int e = 0; e < group; ++e) {
                float a = fabsf(X[idx[e]]);
                if (a > m) m = a;
            }
            size_t sidx = axis == 1 ? (size_t)line * n_groups + gi
                                    : (size_t)gi * d_v + line;
            if (scales) scales[sidx] = 0.0f;
            if (m == 0.0f) {
                for (int e = 0; e < group; ++e) {
                    X[idx[e]] = 0.0f;
                    if (codes) codes[idx[e]] = 0.0f;
                }
                continue;
            }
            float s = m / 127.0f;
            if (scales) scales[sidx] = s;
            for (int e = 0; e < group; ++e) {
                float t = X[idx[e]] / s;
                float c = rintf(t);               /* ties to even */
                if (c > 127.0f) c = 127.0f;
                if (c < -127.0f) c = -127.0f;
                float y = c * s;
                X[idx[e]] = y;
                if (codes) codes[idx[e]] = c;
            }
        }
}

/* Public codec entry: QDQ of `count` consecutive [d_k, d_v] fp32 states.
 * codes: same size as X (may be NULL); scales: per state, d_v/64 (FP8) or
 * d_k*d_v/group (INT8) entries (may be NULL).  Returns 0, or -1 on a bad
 * argument. */
int or_qdq(float *X, long count, int d_k, int d_v, int mode, int group,
           int axis, float *codes, float *scales)
{
    if (mode == OR_QDQ_NONE) return 0;
    if (d_k <= 0 || d_v <= 0) return -1;
    if (mode == OR_QDQ_FP8_TILE) {
        if (d_v % 64) return -1;
        int nsc = d_v / 64;
        for (long s = 0; s < count; ++s)
            qdq_fp8_tile(X + s * (size_t)d_k * d_v, d_k, d_v, 64,
                         codes ? codes + s * (size_t)d_k * d_v : NULL,
                         scales ? scales + s * (size_t)nsc : NULL);
        return 0;
    }
    if (mode == OR_QDQ_INT8_GROUP) {
        if (group <= 0 || group > 64) return -1;
        if ((axis == 1 ? d_v : d_k) % group) return -1;
        size_t nsc = (size_t)d_k * d_v / group;
        for (long s = 0; s < count; ++s)
            qdq_int8_group(X + s * (size_t)d_k * d_v, d_k, d_v, group, axis,
                           codes ? codes + s * (size_t)d_k * d_v : NULL,
                           scales ? scales + s * nsc : NULL);
        return 0;
    }
    return -1;
}

/* ---------------------------------------------------------------------------
 * Token recurrence for packed sequences.
 *
 *  q, k:  fp64 [total_T, H, d_k];  v: fp64 [total_T, H, d_v]
 *  g:     fp64 [total_T, H] (per_key_gate = 0) or [total_T, H, d_k] (= 1),
 *         natural-log gates, alpha = exp(g)
 *  beta:  fp64 [total_T, H]
 *  state_in: fp64 [n_seq, H, d_k, d_v] or NULL (zero state)
 *  cu_seqlens: int32 [n_seq + 1], sequence s owns tokens [cu[s], cu[s+1])
 *  boundary_every: QDQ after token t (local index) when (t + 1) is a multiple
 *         of it or t is the sequence's last token; 64 for the chunked
 *         prefix, 1 for decode tokens.
 *  o:     fp64 [total_T, H, d_v]; state_out fp64 [n_seq, H, d_k, d_v]
 *  codes_out / scales_out (optional): the codes and scales of the last QDQ
 *         of each (sequence, head), laid out like or_qdq's outputs per state.
 * Returns 0, or -1 on a bad argument.
 * ------------------------------------------------------------------------- */
int or_gdn_recurrence(const double *q, const double *k, const double *v,
                      const double *g, const double *beta,
                      const double *state_in, const int32_t *cu_seqlens,
                      int n_seq, int H, int d_k, int d_v, int per_key_gate,
                      int qdq_mode, int qdq_group, int qdq_axis,
                      int boundary_every, double *o, double *state_out,
                      float *codes_out, float *scales_out, int n_threads)
{
    if (n_seq < 0 || H <= 0 || d_k <= 0 || d_v <= 0 || boundary_every <= 0)
        return -1;
    for (int s = 0; s < n_seq; ++s)
        if (cu_seqlens[s + 1] < cu_seqlens[s]) return -1;
    const double scale = 1.0 / sqrt((double)d_k);
    const size_t ss = (size_t)d_k * d_v;
    size_t nsc = 0;
    if (qdq_mode == OR_QDQ_FP8_TILE) nsc = (size_t)d_v / 64;
    if (qdq_mode == OR_QDQ_INT8_GROUP) nsc = ss / (size_t)qdq_group;
    long units = (long)n_seq * H;
    int bad = 0;

#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#pragma omp parallel for schedule(dynamic, 1) reduction(|: bad)
#endif
    for (long unit = 0; unit < units; ++unit) {
        int s = (int)(unit / H), h = (int)(unit % H);
        double *Hm = (double *)malloc(ss * sizeof(double));
        float *X = (float *)malloc(ss * sizeof(float));
        double *alpha = (double *)malloc((size_t)d_k * sizeof(double));
        double *a = (double *)malloc((size_t)d_v * sizeof(double));
        double *u = (double *)malloc((size_t)d_v * sizeof(double));
        if (!Hm || !X || !alpha || !a || !u) { bad |= 1; goto done; }

        if (state_in)
            memcpy(Hm, state_in + (size_t)unit * ss, ss * sizeof(double));
        else
            memset(Hm, 0, ss * sizeof(double));

        int t0 = cu_seqlens[s], L = cu_seqlens[s + 1] - cu_seqlens[s];
        for (int t = 0; t < L; ++t) {
            size_t tok = (size_t)(t0 + t) * H + h;
            const double *qt = q + tok * d_k, *kt = k + tok * d_k;
            const double *vt = v + tok * d_v;
            const double bt = beta[tok];
            /* decay: H <- diag(alpha_t) H, alpha acting on the key rows */
            for (int i = 0; i < d_k; ++i)
                alpha[i] = exp(per_key_gate ? g[tok * d_k + i] : g[tok]);
            for (int i = 0; i < d_k; ++i)
                for (int j = 0; j < d_v; ++j)
                    Hm[(size_t)i * d_v + j] *= alpha[i];
            /* a = H^T k ; u = beta (v - a) */
            for (int j = 0; j < d_v; ++j) a[j] = 0.0;
            for (int i = 0; i < d_k; ++i)
                for (int j = 0; j < d_v; ++j)
                    a[j] += Hm[(size_t)i * d_v + j] * kt[i];
            for (int j = 0; j < d_v; ++j) u[j] = bt * (vt[j] - a[j]);
            /* H <- H + k u^T */
            for (int i = 0; i < d_k; ++i)
                for (int j = 0; j < d_v; ++j)
                    Hm[(size_t)i * d_v + j] += kt[i] * u[j];
            /* o = H^T q / sqrt(d_k), from the updated (pre-QDQ) state */
            double *ot = o + tok * d_v;
            for (int j = 0; j < d_v; ++j) ot[j] = 0.0;
            for (int i = 0; i < d_k; ++i)
                for (int j = 0; j < d_v; ++j)
                    ot[j] += Hm[(size_t)i * d_v + j] * qt[i];
            for (int j = 0; j < d_v; ++j) ot[j] *= scale;
            /* QDQ at a chunk boundary / after a decode token */
            int boundary = ((t + 1) % boundary_every == 0) || (t == L - 1);
            if (boundary && qdq_mode != OR_QDQ_NONE) {
                for (size_t e = 0; e < ss; ++e) X[e] = (float)Hm[e];
                float *cd = codes_out ? codes_out + (size_t)unit * ss : NULL;
                float *sc = scales_out ? scales_out + (size_t)unit * nsc : NULL;
                if (or_qdq(X, 1, d_k, d_v, qdq_mode, qdq_group, qdq_axis,
                           cd, sc) != 0) { bad |= 1; break; }
                for (size_t e = 0; e < ss; ++e) Hm[e] = (double)X[e];
            }
        }
        memcpy(state_out + (size_t)unit * ss, Hm, ss * sizeof(double));
    done:
        free(Hm); free(X); free(alpha); free(a); free(u);
    }
    return bad ? -1 : 0;
}

/* Elementwise E4M3 rounding of n fp32 values (for tests). */
void or_e4m3_array(const float *in, float *out, long n)
{
    for (long i = 0; i < n; ++i) out[i] = or_e4m3_rne_satfinite(in[i]);
}

/* Number of threads OpenMP would use (1 without OpenMP). */
int or_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
