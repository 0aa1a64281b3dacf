/*
 * moe_oracle.c -- plain CPU oracle for the forward pass of one mixture-of-experts layer.
 *
 * TEST INFRASTRUCTURE ONLY. The product library never links, loads or calls this file.
 * Only the test suite, the smoke check and the bench's CPU-baseline leg use it. It shares
 * no code, header, table or helper with the CUDA path.
 *
 * What is computed, and where the pages say so
 * (Comet: Fine-grained Computation-communication Overlapping for Mixture-of-Experts):
 *   - §2.1 "MoE Structure": each token is routed to a few selected experts, each selected
 *     expert runs its feed-forward network on the token, and the top-k expert outputs are
 *     gathered back and reduced.                       -> oracle_router_logits,
 *                                                        oracle_topk_gates,
 *                                                        oracle_expert_ffn_row,
 *                                                        oracle_combine
 *   - §2.2.1 and §3.1.2: the routed tokens are reorganised so that each computation tile
 *     sees only the rows it needs; layer0 and layer1 run as grouped GEMMs over the
 *     experts.                                         -> oracle_dispatch
 *   - §2.2.2: routing is decided at run time, so the per-expert row counts vary.
 *
 * Readings taken where the pages are silent:
 *   - router: logits = x . W_g (+ an optional per-expert bias), W_g stored [H, E];
 *   - selection: the k largest logits, ties broken toward the lower expert id;
 *   - gates: softmax over the k selected logits (equal, in exact arithmetic, to a softmax
 *     over all E followed by renormalisation over the selected k); a second mode keeps
 *     the full-E softmax values without renormalisation; a third (a load-balancing bias
 *     that steers the selection only, not on the pages) selects by logit + bias and takes
 *     the gates from the logits without the bias;
 *   - experts: SwiGLU with W1 [E, H, 2F] (columns [0,F) gate, [F,2F) up) or a plain
 *     activation with W1 [E, H, F]; W2 is [E, F, H];
 *   - no capacity limit: every routed (token, expert) pair is computed;
 *   - rows of one expert are ordered by ascending token id; each expert's row block is
 *     padded up to a multiple of the tile height; pad rows carry the index -1.
 *
 * Precision:
 *   - inputs are bf16 bit patterns, widened to float exactly;
 *   - the router logits decide integers (the selected experts), so they are computed in
 *     the precision and order the GPU router uses: fp32, one accumulator, h ascending.
 *     A bf16 x bf16 product is exact in fp32, so fused and unfused multiply-add agree;
 *   - everything else (gates, expert FFN, combine) is computed in fp64.
 *
 * Build: gcc -O2 -std=c11 -fPIC -shared -ffp-contract=off -fopenmp. No fast-math.
 * OpenMP only splits independent tokens or rows across threads; it never changes the
 * order of any sum.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_ACT_SWIGLU 0
#define ORACLE_ACT_GELU_TANH 1
#define ORACLE_ACT_RELU 2
#define ORACLE_ACT_IDENTITY 3

#define ORACLE_GATE_SOFTMAX_TOPK 0
#define ORACLE_GATE_SOFTMAX_ALL 1
#define ORACLE_GATE_SELECT_BIAS 2

/* ---------------------------------------------------------------------------------------
 * bf16 helpers
 * ------------------------------------------------------------------------------------- */

/* bf16 is the upper half of an IEEE binary32 word, so widening is a 16-bit shift. */
static float bf16_to_float(uint16_t b)
{
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Round a double to the nearest bf16 value (8 significant bits), ties to even.
 * Only normal-range values are expected here; zero passes through. */
double oracle_round_to_bf16(double v)
{
    if (v == 0.0 || !isfinite(v)) return v;
    int e;
    double m = frexp(v, &e);          /* v = m * 2^e, 0.5 <= |m| < 1 */
    double scaled = ldexp(m, 8);      /* 8 significant bits to the left of the point */
    double r = nearbyint(scaled);     /* default rounding mode: nearest, ties to even */
    return ldexp(r, e - 8);
}

/* ---------------------------------------------------------------------------------------
 * Router (§2.1: tokens are routed to selected experts)
 * ------------------------------------------------------------------------------------- */

/* logits[t][e] = sum_h x[t][h] * Wg[h][e]  (+ bias[e]),
 * in fp32 with a single accumulator and h ascending. x: [T,H], Wg: [H,E], bias: [E] or NULL. */
void oracle_router_logits(int T, int H, int E, const uint16_t *x, const uint16_t *Wg,
                          const float *bias, float *logits)
{
#pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t) {
        for (int e = 0; e < E; ++e) {
            float acc = 0.0f;
            for (int h = 0; h < H; ++h) {
                float p = bf16_to_float(x[(size_t)t * H + h]) * bf16_to_float(Wg[(size_t)h * E + e]);
                acc = acc + p;
            }
            if (bias) acc = acc + bias[e];
            logits[(size_t)t * E + e] = acc;
        }
    }
}

/* Top-k selection and gate weights for one token.
 * Selection: repeatedly take the largest remaining key; on equal keys the lower expert id
 * wins (scan ascending, replace only on strictly greater). Equal compares as floats, so +0
 * and -0 tie. The key is the logit, or for SELECT_BIAS the fp32 sum l[e] + bias[e] (the
 * same single addition that adds the bias to the logits in the other modes).
 * Gates (fp64):
 *   SOFTMAX_TOPK: w_j = exp(l_j - l_0) / sum_i exp(l_i - l_0), i, j over the selected k;
 *   SOFTMAX_ALL : w_j = exp(l_j - l_0) / sum_e exp(l_e - l_0), e over all E
 *                 (l_0 is the largest logit in both cases);
 *   SELECT_BIAS : as SOFTMAX_TOPK on the logits without the bias, shifted by the largest
 *                 of them. */
static float sel_key(int gate, const float *l, const float *bias, int e)
{
    return (gate == ORACLE_GATE_SELECT_BIAS && bias) ? l[e] + bias[e] : l[e];
}

static void topk_one(int E, int k, int gate, const float *l, const float *bias, int32_t *idx,
                     double *w, unsigned char *taken)
{
    memset(taken, 0, (size_t)E);
    for (int j = 0; j < k; ++j) {
        int best = -1;
        for (int e = 0; e < E; ++e) {
            if (taken[e]) continue;
            if (best < 0 || sel_key(gate, l, bias, e) > sel_key(gate, l, bias, best)) best = e;
        }
        taken[best] = 1;
        idx[j] = best;
    }
    double m = (double)l[idx[0]];
    if (gate == ORACLE_GATE_SELECT_BIAS)
        for (int j = 1; j < k; ++j)
            if ((double)l[idx[j]] > m) m = (double)l[idx[j]];
    double denom = 0.0;
    if (gate == ORACLE_GATE_SOFTMAX_ALL) {
        for (int e = 0; e < E; ++e) denom += exp((double)l[e] - m);
    } else {
        for (int j = 0; j < k; ++j) denom += exp((double)l[idx[j]] - m);
    }
    for (int j = 0; j < k; ++j) w[j] = exp((double)l[idx[j]] - m) / denom;
}

/* logits: [T,E] fp32 -> idx: [T,k] int32 (in selection order), w: [T,k] fp64.
 * bias [E] (or NULL) is used by SELECT_BIAS only; the logits then exclude it. */
int oracle_topk_gates_bias(int T, int E, int k, int gate, const float *logits, const float *bias,
                           int32_t *idx, double *w)
{
    if (T < 0 || E < 1 || k < 1 || k > E) return -1;
    int bad = 0;
#pragma omp parallel
    {
        unsigned char *taken = (unsigned char *)malloc((size_t)E);
#pragma omp for schedule(static)
        for (int t = 0; t < T; ++t) {
            if (!taken) {
#pragma omp atomic write
                bad = 1;
                continue;
            }
            topk_one(E, k, gate, logits + (size_t)t * E, bias, idx + (size_t)t * k,
                     w + (size_t)t * k, taken);
        }
        free(taken);
    }
    return bad ? -2 : 0;
}

int oracle_topk_gates(int T, int E, int k, int gate, const float *logits, int32_t *idx, double *w)
{
    return oracle_topk_gates_bias(T, E, k, gate, logits, NULL, idx, w);
}

/* ---------------------------------------------------------------------------------------
 * Dispatch (§2.2.1, §3.1.2: reorganise routed tokens into expert-contiguous tiles)
 * ------------------------------------------------------------------------------------- */

/* Counting sort of the T*k routed pairs by expert, stable in token id.
 *   counts[e]      number of pairs routed to e                              [E]
 *   offsets[e]     exclusive prefix sum of counts                           [E+1]
 *   poff[e]        exclusive prefix sum of counts rounded up to m_tile      [E+1]
 *   gather_idx[r]  token of padded row r, -1 for a pad row                 [gather_len]
 *   inv_pos[t][j]  padded row that holds pair (t, j)                        [T,k]
 *   tile_expert/tile_row0/tile_nvalid: one entry per m_tile block of rows  [tile_cap]
 * Returns the number of tiles, or a negative value on bad arguments. */
int oracle_dispatch(int T, int E, int k, int m_tile, const int32_t *idx, int32_t *counts,
                    int32_t *offsets, int32_t *poff, int32_t *gather_idx, int64_t gather_len,
                    int32_t *inv_pos, int32_t *tile_expert, int32_t *tile_row0,
                    int32_t *tile_nvalid, int64_t tile_cap)
{
    if (T < 0 || E < 1 || k < 1 || m_tile < 1) return -1;
    for (int e = 0; e < E; ++e) counts[e] = 0;
    for (int64_t p = 0; p < (int64_t)T * k; ++p) {
        int e = idx[p];
        if (e < 0 || e >= E) return -2;
        counts[e] += 1;
    }
    offsets[0] = 0;
    poff[0] = 0;
    for (int e = 0; e < E; ++e) {
        offsets[e + 1] = offsets[e] + counts[e];
        int padded = ((counts[e] + m_tile - 1) / m_tile) * m_tile;
        poff[e + 1] = poff[e] + padded;
    }
    if ((int64_t)poff[E] > gather_len) return -3;
    for (int64_t r = 0; r < gather_len; ++r) gather_idx[r] = -1;

    int32_t *cursor = (int32_t *)calloc((size_t)E, sizeof(int32_t));
    if (!cursor) return -4;
    for (int t = 0; t < T; ++t) {
        for (int j = 0; j < k; ++j) {
            int e = idx[(size_t)t * k + j];
            int r = poff[e] + cursor[e];
            cursor[e] += 1;
            gather_idx[r] = t;
            inv_pos[(size_t)t * k + j] = r;
        }
    }
    free(cursor);

    int64_t nt = 0;
    for (int e = 0; e < E; ++e) {
        for (int i = 0; i * m_tile < counts[e]; ++i) {
            if (nt >= tile_cap) return -5;
            int left = counts[e] - i * m_tile;
            tile_expert[nt] = e;
            tile_row0[nt] = poff[e] + i * m_tile;
            tile_nvalid[nt] = left < m_tile ? left : m_tile;
            nt += 1;
        }
    }
    return (int)nt;
}

/* ---------------------------------------------------------------------------------------
 * Expert FFN (§2.1: the selected experts' feed-forward computation)
 * ------------------------------------------------------------------------------------- */

static double act_apply(int act, double z)
{
    switch (act) {
    case ORACLE_ACT_GELU_TANH: {
        const double c = sqrt(2.0 / acos(-1.0));
        return 0.5 * z * (1.0 + tanh(c * (z + 0.044715 * z * z * z)));
    }
    case ORACLE_ACT_RELU:
        return z > 0.0 ? z : 0.0;
    case ORACLE_ACT_IDENTITY:
    default:
        return z;
    }
}

static double silu(double z) { return z / (1.0 + exp(-z)); }

/* One expert applied to one token row, fp64 throughout.
 *   SwiGLU: g_f = sum_h x_h W1[h][f], u_f = sum_h x_h W1[h][F+f], a_f = silu(g_f) * u_f
 *           (W1 row stride 2F);
 *   other : a_f = act(sum_h x_h W1[h][f])  (W1 row stride F);
 *   y_n = sum_f a_f W2[f][n]  (W2 row stride H).
 * round_a_bf16 != 0 rounds a_f to bf16 first (a diagnostic of the GPU's bf16 h tensor).
 * scratch must hold 2F doubles. */
static void ffn_row(int H, int F, int act, int round_a_bf16, const uint16_t *xrow,
                    const uint16_t *W1e, const uint16_t *W2e, double *y, double *scratch)
{
    const int gated = (act == ORACLE_ACT_SWIGLU);
    const int w1_cols = gated ? 2 * F : F;
    double *z = scratch; /* w1_cols pre-activations */
    for (int c = 0; c < w1_cols; ++c) z[c] = 0.0;
    for (int h = 0; h < H; ++h) {
        double xh = (double)bf16_to_float(xrow[h]);
        const uint16_t *wrow = W1e + (size_t)h * w1_cols;
        for (int c = 0; c < w1_cols; ++c) z[c] += xh * (double)bf16_to_float(wrow[c]);
    }
    /* activation in place: a_f is written to z[f] */
    for (int f = 0; f < F; ++f) {
        double a = gated ? silu(z[f]) * z[F + f] : act_apply(act, z[f]);
        z[f] = round_a_bf16 ? oracle_round_to_bf16(a) : a;
    }
    for (int n = 0; n < H; ++n) y[n] = 0.0;
    for (int f = 0; f < F; ++f) {
        double a = z[f];
        const uint16_t *wrow = W2e + (size_t)f * H;
        for (int n = 0; n < H; ++n) y[n] += a * (double)bf16_to_float(wrow[n]);
    }
}

static size_t w1_expert_elems(int H, int F, int act)
{
    return (size_t)H * (size_t)(act == ORACLE_ACT_SWIGLU ? 2 * F : F);
}

/* Public single-row entry (used by tests for dense special cases). */
void oracle_expert_ffn_row(int H, int F, int act, int round_a_bf16, const uint16_t *xrow,
                           const uint16_t *W1e, const uint16_t *W2e, double *y)
{
    double *scratch = (double *)malloc(sizeof(double) * 2 * (size_t)F);
    if (!scratch) return;
    ffn_row(H, F, act, round_a_bf16, xrow, W1e, W2e, y, scratch);
    free(scratch);
}

/* ---------------------------------------------------------------------------------------
 * Combine (§2.1: gather and reduce the top-k outputs)
 * ------------------------------------------------------------------------------------- */

/* out[t][n] = sum_{j=0..k-1} ys[inv_pos[t][j]][n], j ascending, fp64.
 * ys holds bf16 rows that already carry the gate weight. */
void oracle_combine(int T, int H, int k, const uint16_t *ys, const int32_t *inv_pos, double *out)
{
#pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t) {
        for (int n = 0; n < H; ++n) {
            double s = 0.0;
            for (int j = 0; j < k; ++j) {
                int r = inv_pos[(size_t)t * k + j];
                s += (double)bf16_to_float(ys[(size_t)r * H + n]);
            }
            out[(size_t)t * H + n] = s;
        }
    }
}

/* ---------------------------------------------------------------------------------------
 * Whole layer
 * ------------------------------------------------------------------------------------- */

/* The layer in the pages' order: route -> dispatch into expert-contiguous rows ->
 * per-expert FFN over its rows -> weighted top-k reduce per token.
 * out: [T,H] fp64. idx_out [T,k] and w_out [T,k] are optional (NULL to skip).
 * Returns 0 on success. Memory use is about (T*k + E*m_tile) * H doubles, so this entry
 * is meant for small layers; large layers use oracle_moe_tokens on a token sample. */
int oracle_moe_forward(int T, int H, int F, int E, int k, int act, int gate, int m_tile,
                       int round_a_bf16, const uint16_t *x, const uint16_t *Wg, const float *bias,
                       const uint16_t *W1, const uint16_t *W2, double *out, int32_t *idx_out,
                       double *w_out)
{
    if (T < 0 || H < 1 || F < 1 || E < 1 || k < 1 || k > E || m_tile < 1) return -1;
    if (T == 0) return 0;
    const size_t TK = (size_t)T * k;
    const int64_t gather_len = (int64_t)TK + (int64_t)E * (m_tile - 1);
    const int64_t tile_cap = gather_len / m_tile + E;
    int rc = 0;

    float *logits = (float *)malloc(sizeof(float) * (size_t)T * E);
    int32_t *idx = (int32_t *)malloc(sizeof(int32_t) * TK);
    double *w = (double *)malloc(sizeof(double) * TK);
    int32_t *counts = (int32_t *)malloc(sizeof(int32_t) * (size_t)E);
    int32_t *offsets = (int32_t *)malloc(sizeof(int32_t) * (size_t)(E + 1));
    int32_t *poff = (int32_t *)malloc(sizeof(int32_t) * (size_t)(E + 1));
    int32_t *gather_idx = (int32_t *)malloc(sizeof(int32_t) * (size_t)gather_len);
    int32_t *inv_pos = (int32_t *)malloc(sizeof(int32_t) * TK);
    int32_t *t_e = (int32_t *)malloc(sizeof(int32_t) * (size_t)tile_cap);
    int32_t *t_r = (int32_t *)malloc(sizeof(int32_t) * (size_t)tile_cap);
    int32_t *t_n = (int32_t *)malloc(sizeof(int32_t) * (size_t)tile_cap);
    double *y = (double *)malloc(sizeof(double) * (size_t)gather_len * H);
    if (!logits || !idx || !w || !counts || !offsets || !poff || !gather_idx || !inv_pos || !t_e ||
        !t_r || !t_n || !y) {
        rc = -4;
        goto done;
    }

    /* 1. route (with a selection-only bias the logits exclude it) */
    oracle_router_logits(T, H, E, x, Wg, gate == ORACLE_GATE_SELECT_BIAS ? NULL : bias, logits);
    rc = oracle_topk_gates_bias(T, E, k, gate, logits, bias, idx, w);
    if (rc) goto done;

    /* 2. dispatch */
    rc = oracle_dispatch(T, E, k, m_tile, idx, counts, offsets, poff, gather_idx, gather_len,
                         inv_pos, t_e, t_r, t_n, tile_cap);
    if (rc < 0) goto done;
    rc = 0;

    /* 3. experts: every real row of every expert, in expert-sorted order */
    {
        const size_t w1e = w1_expert_elems(H, F, act);
        const size_t w2e = (size_t)F * H;
        int bad = 0;
#pragma omp parallel
        {
            double *scratch = (double *)malloc(sizeof(double) * 2 * (size_t)F);
#pragma omp for schedule(dynamic, 4)
            for (int64_t r = 0; r < (int64_t)poff[E]; ++r) {
                int t = gather_idx[r];
                if (t < 0) continue;
                if (!scratch) {
#pragma omp atomic write
                    bad = 1;
                    continue;
                }
                /* the expert that owns padded row r */
                int e = 0;
                while (!(r >= poff[e] && r < poff[e + 1])) ++e;
                ffn_row(H, F, act, round_a_bf16, x + (size_t)t * H, W1 + (size_t)e * w1e,
                        W2 + (size_t)e * w2e, y + (size_t)r * H, scratch);
            }
            free(scratch);
        }
        if (bad) {
            rc = -4;
            goto done;
        }
    }

    /* 4. combine: out[t] = sum_j w[t][j] * y[inv_pos[t][j]], j ascending */
#pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t) {
        for (int n = 0; n < H; ++n) {
            double s = 0.0;
            for (int j = 0; j < k; ++j) {
                int r = inv_pos[(size_t)t * k + j];
                s += w[(size_t)t * k + j] * y[(size_t)r * H + n];
            }
            out[(size_t)t * H + n] = s;
        }
    }
    if (idx_out) memcpy(idx_out, idx, sizeof(int32_t) * TK);
    if (w_out) memcpy(w_out, w, sizeof(double) * TK);

done:
    free(logits);
    free(idx);
    free(w);
    free(counts);
    free(offsets);
    free(poff);
    free(gather_idx);
    free(inv_pos);
    free(t_e);
    free(t_r);
    free(t_n);
    free(y);
    return rc;
}

/* The layer output for a list of tokens, straight from the definition in §2.1:
 *   out[t] = sum_j w_j * FFN_{e_j}(x_t)
 * with no permutation at all. Tokens are independent, so a sample of tokens of a large
 * layer is checked exactly as the whole layer would be.
 * out: [ntok,H] fp64; idx_out [ntok,k] and w_out [ntok,k] optional. */
int oracle_moe_tokens(int T, int H, int F, int E, int k, int act, int gate, int round_a_bf16,
                      const uint16_t *x, const uint16_t *Wg, const float *bias, const uint16_t *W1,
                      const uint16_t *W2, int ntok, const int32_t *tokens, double *out,
                      int32_t *idx_out, double *w_out)
{
    if (H < 1 || F < 1 || E < 1 || k < 1 || k > E || ntok < 0) return -1;
    for (int i = 0; i < ntok; ++i)
        if (tokens[i] < 0 || tokens[i] >= T) return -2;
    const size_t w1e = w1_expert_elems(H, F, act);
    const size_t w2e = (size_t)F * H;
    int bad = 0;
#pragma omp parallel
    {
        float *l = (float *)malloc(sizeof(float) * (size_t)E);
        unsigned char *taken = (unsigned char *)malloc((size_t)E);
        int32_t *sel = (int32_t *)malloc(sizeof(int32_t) * (size_t)k);
        double *w = (double *)malloc(sizeof(double) * (size_t)k);
        double *y = (double *)malloc(sizeof(double) * (size_t)H);
        double *scratch = (double *)malloc(sizeof(double) * 2 * (size_t)F);
        const int ok = l && taken && sel && w && y && scratch;
#pragma omp for schedule(dynamic, 1)
        for (int i = 0; i < ntok; ++i) {
            if (!ok) {
#pragma omp atomic write
                bad = 1;
                continue;
            }
            {
                int t = tokens[i];
                oracle_router_logits(1, H, E, x + (size_t)t * H, Wg,
                                     gate == ORACLE_GATE_SELECT_BIAS ? NULL : bias, l);
                topk_one(E, k, gate, l, bias, sel, w, taken);
                double *o = out + (size_t)i * H;
                for (int n = 0; n < H; ++n) o[n] = 0.0;
                for (int j = 0; j < k; ++j) {
                    int e = sel[j];
                    ffn_row(H, F, act, round_a_bf16, x + (size_t)t * H, W1 + (size_t)e * w1e,
                            W2 + (size_t)e * w2e, y, scratch);
                    for (int n = 0; n < H; ++n) o[n] += w[j] * y[n];
                }
                if (idx_out) memcpy(idx_out + (size_t)i * k, sel, sizeof(int32_t) * (size_t)k);
                if (w_out) memcpy(w_out + (size_t)i * k, w, sizeof(double) * (size_t)k);
            }
        }
        free(l);
        free(taken);
        free(sel);
        free(w);
        free(y);
        free(scratch);
    }
    return bad ? -4 : 0;
}

/* ---------------------------------------------------------------------------------------
 * Shared expert (a model feature outside the pages: Qwen2-MoE's shared expert)
 * ------------------------------------------------------------------------------------- */

/* For each listed token: out[i] = g_t * FFN_s(x_t), with FFN_s a SwiGLU FFN
 * (W1s [H, 2Fs]: columns [0,Fs) gate, [Fs,2Fs) up; W2s [Fs, H]) and the token's gate
 * g_t = 1 / (1 + exp(-sum_h x_t[h] w_sg[h])) (fp64), or g_t = 1 without w_sg (NULL).
 * The layer with a shared expert is the routed layer's output plus this term.
 * out: [ntok, H] fp64. */
int oracle_shared_tokens(int T, int H, int Fs, const uint16_t *x, const uint16_t *W1s,
                         const uint16_t *W2s, const uint16_t *w_sg, int ntok, const int32_t *tokens,
                         double *out)
{
    if (H < 1 || Fs < 1 || ntok < 0) return -1;
    for (int i = 0; i < ntok; ++i)
        if (tokens[i] < 0 || tokens[i] >= T) return -2;
    int bad = 0;
#pragma omp parallel
    {
        double *y = (double *)malloc(sizeof(double) * (size_t)H);
        double *scratch = (double *)malloc(sizeof(double) * 2 * (size_t)Fs);
#pragma omp for schedule(dynamic, 1)
        for (int i = 0; i < ntok; ++i) {
            if (!y || !scratch) {
#pragma omp atomic write
                bad = 1;
                continue;
            }
            const uint16_t *xr = x + (size_t)tokens[i] * H;
            double g = 1.0;
            if (w_sg) {
                double z = 0.0;
                for (int h = 0; h < H; ++h)
                    z += (double)bf16_to_float(xr[h]) * (double)bf16_to_float(w_sg[h]);
                g = 1.0 / (1.0 + exp(-z));
            }
            ffn_row(H, Fs, ORACLE_ACT_SWIGLU, 0, xr, W1s, W2s, y, scratch);
            for (int n = 0; n < H; ++n) out[(size_t)i * H + n] = g * y[n];
        }
        free(y);
        free(scratch);
    }
    return bad ? -4 : 0;
}

/* ---------------------------------------------------------------------------------------
 * FP8 experts (a precision variant outside the pages; the pages fix no precision)
 *
 * Reading taken:
 *   - element format: e4m3 of the OCP 8-bit floating-point formats: 1 sign bit, 4 exponent
 *     bits (bias 7), 3 mantissa bits, no infinities, S.1111.111 is NaN, so the largest
 *     finite magnitude is 1.75 * 2^8 = 448; exponent field 0 holds m * 2^-9, m = 1..7;
 *   - conversion: nearest value, ties to the even code; magnitudes above 448 and infinities
 *     saturate to 448; NaN stays NaN;
 *   - scaling: one fp32 scale per token row of x and of h (over the K values of the row),
 *     one per output column of W1 and W2 (over K): r = 448 / amax, s = amax / 448, both
 *     rounded to fp32, code = e4m3(v * r) with the product rounded to fp32; a vector whose
 *     r is not finite (amax zero or tiny) takes r = s = 1;
 *   - GEMMs: exact products of the decoded codes, summed, times s_row * s_col;
 *   - between the layers h is held in bf16, as in the bf16 path, and then quantised per row.
 *     A bf16 rounding can only move a value onto an e4m3 rounding midpoint, never across
 *     one, so it shows in the codes only through ties; the pins include such a tie.
 * ------------------------------------------------------------------------------------- */

double oracle_e4m3_decode(uint8_t c)
{
    const int s = c >> 7, ef = (c >> 3) & 15, m = c & 7;
    if (ef == 15 && m == 7) return NAN;
    const double v = ef == 0 ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, ef - 7);
    return s ? -v : v;
}

uint8_t oracle_e4m3_encode(float v)
{
    if (isnan(v)) return 0x7F;
    const uint8_t sign = signbit(v) ? 0x80 : 0x00;
    const double a = fabs((double)v);
    if (a > 448.0) return sign | 0x7E;
    int code;
    if (a < ldexp(1.0, -6)) {
        /* subnormal range: the nearest multiple of 2^-9 (8 * 2^-9 is the smallest normal,
         * whose code is 8) */
        code = (int)nearbyint(ldexp(a, 9));
    } else {
        int e;
        frexp(a, &e); /* a in [2^(e-1), 2^e) */
        const int ex = e - 1;
        const int m = (int)nearbyint((ldexp(a, -ex) - 1.0) * 8.0); /* 0..8; 8 carries */
        code = ((ex + 7) << 3) + m;
    }
    return (uint8_t)(sign | code);
}

void oracle_e4m3_encode_n(int64_t n, const float *v, uint8_t *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_e4m3_encode(v[i]);
}

void oracle_e4m3_decode_n(int64_t n, const uint8_t *c, double *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_e4m3_decode(c[i]);
}

/* scales of one vector with largest magnitude amax: *r = 448 / amax, *s = amax / 448 */
static void fp8_scales(float amax, float *r, float *s)
{
    *r = 448.0f / amax;
    *s = amax / 448.0f;
    if (!isfinite(*r)) {
        *r = 1.0f;
        *s = 1.0f;
    }
}

/* n values v[i * stride] -> codes q[i * qstride] and the vector's dequantisation scale */
static float quant_vec(int n, const float *v, ptrdiff_t stride, uint8_t *q, ptrdiff_t qstride)
{
    float amax = 0.0f;
    for (int i = 0; i < n; ++i) {
        const float a = fabsf(v[(ptrdiff_t)i * stride]);
        if (a > amax) amax = a;
    }
    float r, s;
    fp8_scales(amax, &r, &s);
    for (int i = 0; i < n; ++i) q[(ptrdiff_t)i * qstride] = oracle_e4m3_encode(v[(ptrdiff_t)i * stride] * r);
    return s;
}

/* Row quantisation of a bf16 matrix src [rows, cols] -> dst [rows, cols] codes, scale [rows]. */
void oracle_quant_rows_fp8(int rows, int cols, const uint16_t *src, uint8_t *dst, float *scale)
{
#pragma omp parallel
    {
        float *v = (float *)malloc(sizeof(float) * (size_t)cols);
#pragma omp for schedule(static)
        for (int r = 0; r < rows; ++r) {
            if (!v) continue;
            for (int c = 0; c < cols; ++c) v[c] = bf16_to_float(src[(size_t)r * cols + c]);
            scale[r] = quant_vec(cols, v, 1, dst + (size_t)r * cols, 1);
        }
        free(v);
    }
}

/* Column quantisation of expert weights W [E, K, N] (N contiguous): per column n of expert
 * e, the K values W[e][:, n] -> Wq[e][n][:] (the transpose: K contiguous), scale [E, N]. */
void oracle_quant_cols_fp8(int E, int K, int N, const uint16_t *W, uint8_t *Wq, float *scale)
{
#pragma omp parallel
    {
        float *v = (float *)malloc(sizeof(float) * (size_t)K);
#pragma omp for schedule(static)
        for (int64_t en = 0; en < (int64_t)E * N; ++en) {
            if (!v) continue;
            const int64_t e = en / N, n = en % N;
            const uint16_t *col = W + (size_t)e * K * N + n;
            for (int kk = 0; kk < K; ++kk) v[kk] = bf16_to_float(col[(size_t)kk * N]);
            scale[en] = quant_vec(K, v, 1, Wq + (size_t)en * K, 1);
        }
        free(v);
    }
}

/* One expert on one token with e4m3 operands (xq, sx: the token's quantised row):
 *   z_c = (sum_h dec(xq_h) * dec(W1q[c][h])) * sx * s1[c]     (W1q [w1_cols, H], fp64);
 *   a_f = silu(z_f) * z_{F+f} (SwiGLU) or act(z_f), rounded to bf16 (the stored h);
 *   hq, sh = the row quantisation of a;
 *   y_n = (sum_f dec(hq_f) * dec(W2q[n][f])) * sh * s2[n]      (W2q [H, F]).
 * dec: the 256-entry decode table. z must hold 2F doubles, hf F floats, hq F bytes. */
static void ffn_row_fp8(int H, int F, int act, const double *dec, const uint8_t *xq, float sx,
                        const uint8_t *W1q, const float *s1, const uint8_t *W2q, const float *s2,
                        double *y, double *z, float *hf, uint8_t *hq)
{
    const int gated = (act == ORACLE_ACT_SWIGLU);
    const int w1_cols = gated ? 2 * F : F;
    for (int c = 0; c < w1_cols; ++c) {
        const uint8_t *wr = W1q + (size_t)c * H;
        double acc = 0.0;
        for (int h = 0; h < H; ++h) acc += dec[xq[h]] * dec[wr[h]];
        z[c] = acc * (double)sx * (double)s1[c];
    }
    for (int f = 0; f < F; ++f) {
        const double a = gated ? silu(z[f]) * z[f + F] : act_apply(act, z[f]);
        hf[f] = (float)oracle_round_to_bf16(a);
    }
    const float sh = quant_vec(F, hf, 1, hq, 1);
    for (int n = 0; n < H; ++n) {
        const uint8_t *wr = W2q + (size_t)n * F;
        double acc = 0.0;
        for (int f = 0; f < F; ++f) acc += dec[hq[f]] * dec[wr[f]];
        y[n] = acc * (double)sh * (double)s2[n];
    }
}

/* The layer output for a list of tokens with e4m3 experts: the routing of oracle_moe_tokens
 * (bf16 x and W_g, fp32 logits), then out[t] = sum_j w_j * FFN8_{e_j}(x_t) with the token's
 * row quantised as above. W1q [E, w1_cols, H] with scales s1 [E, w1_cols]; W2q [E, H, F]
 * with s2 [E, H] (as oracle_quant_cols_fp8 writes them). out [ntok, H] fp64. */
int oracle_moe_tokens_fp8(int T, int H, int F, int E, int k, int act, int gate, const uint16_t *x,
                          const uint16_t *Wg, const float *bias, const uint8_t *W1q,
                          const float *s1, const uint8_t *W2q, const float *s2, int ntok,
                          const int32_t *tokens, double *out, int32_t *idx_out, double *w_out)
{
    if (H < 1 || F < 1 || E < 1 || k < 1 || k > E || ntok < 0) return -1;
    for (int i = 0; i < ntok; ++i)
        if (tokens[i] < 0 || tokens[i] >= T) return -2;
    const int w1_cols = act == ORACLE_ACT_SWIGLU ? 2 * F : F;
    double dec[256];
    for (int c = 0; c < 256; ++c) dec[c] = oracle_e4m3_decode((uint8_t)c);
    int bad = 0;
#pragma omp parallel
    {
        float *l = (float *)malloc(sizeof(float) * (size_t)E);
        unsigned char *taken = (unsigned char *)malloc((size_t)E);
        int32_t *sel = (int32_t *)malloc(sizeof(int32_t) * (size_t)k);
        double *w = (double *)malloc(sizeof(double) * (size_t)k);
        double *y = (double *)malloc(sizeof(double) * (size_t)H);
        double *z = (double *)malloc(sizeof(double) * 2 * (size_t)F);
        float *xf = (float *)malloc(sizeof(float) * (size_t)H);
        uint8_t *xq = (uint8_t *)malloc((size_t)H);
        float *hf = (float *)malloc(sizeof(float) * (size_t)F);
        uint8_t *hq = (uint8_t *)malloc((size_t)F);
        const int ok = l && taken && sel && w && y && z && xf && xq && hf && hq;
#pragma omp for schedule(dynamic, 1)
        for (int i = 0; i < ntok; ++i) {
            if (!ok) {
#pragma omp atomic write
                bad = 1;
                continue;
            }
            const int t = tokens[i];
            const uint16_t *xr = x + (size_t)t * H;
            oracle_router_logits(1, H, E, xr, Wg, gate == ORACLE_GATE_SELECT_BIAS ? NULL : bias, l);
            topk_one(E, k, gate, l, bias, sel, w, taken);
            for (int h = 0; h < H; ++h) xf[h] = bf16_to_float(xr[h]);
            const float sx = quant_vec(H, xf, 1, xq, 1);
            double *o = out + (size_t)i * H;
            for (int n = 0; n < H; ++n) o[n] = 0.0;
            for (int j = 0; j < k; ++j) {
                const int e = sel[j];
                ffn_row_fp8(H, F, act, dec, xq, sx, W1q + (size_t)e * w1_cols * H,
                            s1 + (size_t)e * w1_cols, W2q + (size_t)e * H * F, s2 + (size_t)e * H,
                            y, z, hf, hq);
                for (int n = 0; n < H; ++n) o[n] += y[n] * w[j];
            }
            if (idx_out) memcpy(idx_out + (size_t)i * k, sel, sizeof(int32_t) * (size_t)k);
            if (w_out) memcpy(w_out + (size_t)i * k, w, sizeof(double) * (size_t)k);
        }
        free(l);
        free(taken);
        free(sel);
        free(w);
        free(y);
        free(z);
        free(xf);
        free(xq);
        free(hf);
        free(hq);
    }
    return bad ? -4 : 0;
}

/* ---------------------------------------------------------------------------------------
 * Block-scaled FP8 experts (MX form; a precision variant outside the pages). Oracle only:
 * the CUDA path for this form is not built.
 *
 * Reading taken (the block format of the Open Compute Project's microscaling formats: e4m3
 * elements sharing one e8m0 scale per 32 values; the conversion is this reading's):
 *   - a block is 32 consecutive values along the GEMM's K dimension (a row of x or h; a
 *     column of W1 or W2 along its input dimension);
 *   - the block's scale is the smallest power of two 2^X with amax / 2^X <= 448 (amax: the
 *     block's largest magnitude; 448 = 1.75 * 2^8, e4m3's largest finite value), so no
 *     element saturates: X = floor(log2(amax)) - 8, plus 1 when amax / 2^that exceeds 448;
 *     X is clamped to [-127, 127] and stored as the e8m0 byte X + 127 (255 is NaN). (The
 *     specification's own conversion takes X = floor(log2(amax)) - 8 and saturates the
 *     elements that land in (448, 512); on a test layer that gave a larger error than
 *     per-row scales, which this rule avoids);
 *   - each element is e4m3(v / 2^X) (oracle_e4m3_encode: nearest, ties to even);
 *   - a block of zeros takes X = -127;
 *   - GEMMs: for each output, the sum over blocks of 2^(Xa + Xw) times the exact sum of the
 *     block's decoded code products (fp64);
 *   - between the layers h is held in bf16, then quantised per 32-value block of its row.
 * ------------------------------------------------------------------------------------- */

double oracle_e8m0_decode(uint8_t b)
{
    if (b == 255) return NAN;
    return ldexp(1.0, (int)b - 127);
}

/* one block of n <= 32 values v[i * stride] -> codes q[i], returns the e8m0 scale byte */
static uint8_t mx_quant_block(int n, const float *v, ptrdiff_t stride, uint8_t *q)
{
    double amax = 0.0;
    for (int i = 0; i < n; ++i) {
        const double a = fabs((double)v[(ptrdiff_t)i * stride]);
        if (a > amax) amax = a;
    }
    int X = -127;
    if (amax > 0.0) {
        int e;
        frexp(amax, &e); /* amax in [2^(e-1), 2^e): floor(log2 amax) = e - 1 */
        X = (e - 1) - 8;
        if (ldexp(amax, -X) > 448.0) X += 1; /* exact: scaling by a power of two */
        if (X < -127) X = -127;
        if (X > 127) X = 127;
    }
    for (int i = 0; i < n; ++i) {
        const double scaled = ldexp((double)v[(ptrdiff_t)i * stride], -X); /* exact: a power of two */
        q[i] = oracle_e4m3_encode((float)scaled);
    }
    return (uint8_t)(X + 127);
}

/* values [rows, cols] fp32 -> codes [rows, cols], scales [rows, cols / 32] (cols % 32 == 0) */
int oracle_mx_quant_rows_f32(int rows, int cols, const float *v, uint8_t *q, uint8_t *scale)
{
    if (rows < 0 || cols < 0 || cols % 32 != 0) return -1;
    for (int r = 0; r < rows; ++r)
        for (int b = 0; b < cols / 32; ++b)
            scale[(size_t)r * (cols / 32) + b] =
                mx_quant_block(32, v + (size_t)r * cols + b * 32, 1, q + (size_t)r * cols + b * 32);
    return 0;
}

/* bf16 matrix src [rows, cols] -> codes [rows, cols], scales [rows, cols / 32] */
int oracle_mx_quant_rows(int rows, int cols, const uint16_t *src, uint8_t *q, uint8_t *scale)
{
    if (rows < 0 || cols < 0 || cols % 32 != 0) return -1;
    float v[32];
    for (int r = 0; r < rows; ++r)
        for (int b = 0; b < cols / 32; ++b) {
            for (int i = 0; i < 32; ++i) v[i] = bf16_to_float(src[(size_t)r * cols + b * 32 + i]);
            scale[(size_t)r * (cols / 32) + b] = mx_quant_block(32, v, 1, q + (size_t)r * cols + b * 32);
        }
    return 0;
}

/* expert weights W [E, K, N] bf16 (N contiguous) -> per column n of expert e, its K values in
 * blocks of 32: codes Wq [E, N, K] (K contiguous), scales [E, N, K / 32] */
int oracle_mx_quant_cols(int E, int K, int N, const uint16_t *W, uint8_t *Wq, uint8_t *scale)
{
    if (E < 0 || K < 0 || N < 0 || K % 32 != 0) return -1;
    float v[32];
    for (int64_t en = 0; en < (int64_t)E * N; ++en) {
        const int64_t e = en / N, n = en % N;
        const uint16_t *col = W + (size_t)e * K * N + n;
        for (int b = 0; b < K / 32; ++b) {
            for (int i = 0; i < 32; ++i) v[i] = bf16_to_float(col[(size_t)(b * 32 + i) * N]);
            scale[(size_t)en * (K / 32) + b] = mx_quant_block(32, v, 1, Wq + (size_t)en * K + b * 32);
        }
    }
    return 0;
}

/* sum over the K / 32 blocks of 2^(Xa + Xb) * sum of the block's decoded code products */
static double mx_dot(int K, const double *dec, const uint8_t *qa, const uint8_t *sa,
                     const uint8_t *qb, const uint8_t *sb)
{
    double acc = 0.0;
    for (int b = 0; b < K / 32; ++b) {
        double part = 0.0;
        for (int i = 0; i < 32; ++i) part += dec[qa[b * 32 + i]] * dec[qb[b * 32 + i]];
        acc += part * oracle_e8m0_decode(sa[b]) * oracle_e8m0_decode(sb[b]);
    }
    return acc;
}

/* One expert on one token with MX operands (xq, xs: the token's row codes and scales;
 * W1q [w1_cols, H] with W1s [w1_cols, H / 32]; W2q [H, F] with W2s [H, F / 32]):
 *   z_c = mx_dot over H; a = SwiGLU or act(z), rounded to bf16 (the stored h);
 *   hq, hs = the MX quantisation of a; y_n = mx_dot over F. */
static void ffn_row_mx(int H, int F, int act, const double *dec, const uint8_t *xq,
                       const uint8_t *xs, const uint8_t *W1q, const uint8_t *W1s,
                       const uint8_t *W2q, const uint8_t *W2s, double *y, double *z, float *hf,
                       uint8_t *hq, uint8_t *hs)
{
    const int gated = (act == ORACLE_ACT_SWIGLU);
    const int w1_cols = gated ? 2 * F : F;
    for (int c = 0; c < w1_cols; ++c)
        z[c] = mx_dot(H, dec, xq, xs, W1q + (size_t)c * H, W1s + (size_t)c * (H / 32));
    for (int f = 0; f < F; ++f) {
        const double a = gated ? silu(z[f]) * z[f + F] : act_apply(act, z[f]);
        hf[f] = (float)oracle_round_to_bf16(a);
    }
    for (int b = 0; b < F / 32; ++b) hs[b] = mx_quant_block(32, hf + b * 32, 1, hq + b * 32);
    for (int n = 0; n < H; ++n)
        y[n] = mx_dot(F, dec, hq, hs, W2q + (size_t)n * F, W2s + (size_t)n * (F / 32));
}

/* The layer output for a list of tokens with MX experts: the routing of oracle_moe_tokens
 * (bf16 x and W_g, fp32 logits), then out[t] = sum_j w_j * FFN_MX_{e_j}(x_t) with the token's
 * row quantised per block of 32. W1q [E, w1_cols, H], W1s [E, w1_cols, H / 32]; W2q [E, H, F],
 * W2s [E, H, F / 32] (as oracle_mx_quant_cols writes them). out [ntok, H] fp64. */
int oracle_moe_tokens_mx(int T, int H, int F, int E, int k, int act, int gate, const uint16_t *x,
                         const uint16_t *Wg, const float *bias, const uint8_t *W1q,
                         const uint8_t *W1s, const uint8_t *W2q, const uint8_t *W2s, int ntok,
                         const int32_t *tokens, double *out, int32_t *idx_out, double *w_out)
{
    if (H < 1 || F < 1 || E < 1 || k < 1 || k > E || ntok < 0 || H % 32 || F % 32) return -1;
    for (int i = 0; i < ntok; ++i)
        if (tokens[i] < 0 || tokens[i] >= T) return -2;
    const int w1_cols = act == ORACLE_ACT_SWIGLU ? 2 * F : F;
    double dec[256];
    for (int c = 0; c < 256; ++c) dec[c] = oracle_e4m3_decode((uint8_t)c);
    int bad = 0;
#pragma omp parallel
    {
        float *l = (float *)malloc(sizeof(float) * (size_t)E);
        unsigned char *taken = (unsigned char *)malloc((size_t)E);
        int32_t *sel = (int32_t *)malloc(sizeof(int32_t) * (size_t)k);
        double *w = (double *)malloc(sizeof(double) * (size_t)k);
        double *y = (double *)malloc(sizeof(double) * (size_t)H);
        double *z = (double *)malloc(sizeof(double) * 2 * (size_t)F);
        float *xf = (float *)malloc(sizeof(float) * (size_t)H);
        uint8_t *xq = (uint8_t *)malloc((size_t)H);
        uint8_t *xs = (uint8_t *)malloc((size_t)H / 32);
        float *hf = (float *)malloc(sizeof(float) * (size_t)F);
        uint8_t *hq = (uint8_t *)malloc((size_t)F);
        uint8_t *hs = (uint8_t *)malloc((size_t)F / 32);
        const int ok = l && taken && sel && w && y && z && xf && xq && xs && hf && hq && hs;
#pragma omp for schedule(dynamic, 1)
        for (int i = 0; i < ntok; ++i) {
            if (!ok) {
#pragma omp atomic write
                bad = 1;
                continue;
            }
            const int t = tokens[i];
            const uint16_t *xr = x + (size_t)t * H;
            oracle_router_logits(1, H, E, xr, Wg, gate == ORACLE_GATE_SELECT_BIAS ? NULL : bias, l);
            topk_one(E, k, gate, l, bias, sel, w, taken);
            for (int h = 0; h < H; ++h) xf[h] = bf16_to_float(xr[h]);
            for (int b = 0; b < H / 32; ++b) xs[b] = mx_quant_block(32, xf + b * 32, 1, xq + b * 32);
            double *o = out + (size_t)i * H;
            for (int n = 0; n < H; ++n) o[n] = 0.0;
            for (int j = 0; j < k; ++j) {
                const int e = sel[j];
                ffn_row_mx(H, F, act, dec, xq, xs, W1q + (size_t)e * w1_cols * H,
                           W1s + (size_t)e * w1_cols * (H / 32), W2q + (size_t)e * H * F,
                           W2s + (size_t)e * H * (F / 32), y, z, hf, hq, hs);
                for (int n = 0; n < H; ++n) o[n] += y[n] * w[j];
            }
            if (idx_out) memcpy(idx_out + (size_t)i * k, sel, sizeof(int32_t) * (size_t)k);
            if (w_out) memcpy(w_out + (size_t)i * k, w, sizeof(double) * (size_t)k);
        }
        free(l);
        free(taken);
        free(sel);
        free(w);
        free(y);
        free(z);
        free(xf);
        free(xq);
        free(xs);
        free(hf);
        free(hq);
        free(hs);
    }
    return bad ? -4 : 0;
}

/* ---------------------------------------------------------------------------------------
 * Backward pass (training; a next-work item beyond the pages, which describe the forward)
 *
 * The forward is out[t] = sum_j w_j(t) y_{e_j}(x_t), y_e(x) = FFN_e(x) as in ffn_row, the
 * selection fixed (piecewise constant in the inputs, so it carries no gradient), the gates
 * w = softmax over the selected logits. Given dy = dL/dout (bf16 [T, H]), for each token t
 * and selection j (e = e_j), in fp64 (the logits that feed the gates are the forward's fp32
 * ones):
 *   dw_j   = dy[t] . y_e(x_t)
 *   dl_j   = w_j (dw_j - sum_i w_i dw_i)             (softmax over the selected logits)
 *   gy     = w_j dy[t]                                (gradient at the expert output)
 *   dW2[e] += a^T gy,  da = gy W2[e]^T                (a: the expert's hidden activation)
 *   SwiGLU: dg_f = da_f u_f silu'(g_f), du_f = da_f silu(g_f); others: dz_f = da_f act'(z_f)
 *   dW1[e] += x_t^T dz,  dx[t] += dz W1[e]^T
 *   router: dx[t] += dl_j W_g[:, e],  dW_g[:, e] += x_t dl_j,  dbias[e] += dl_j
 *           (SELECT_BIAS: the gates do not see the bias, so dbias stays 0)
 * silu'(g) = s (1 + g (1 - s)), s = 1 / (1 + e^-g). Gate mode SOFTMAX_ALL is not covered.
 * ------------------------------------------------------------------------------------- */

static double act_grad(int act, double z)
{
    switch (act) {
    case ORACLE_ACT_GELU_TANH: {
        const double c = sqrt(2.0 / acos(-1.0));
        const double k3 = 4.4715e-2; /* the cubic coefficient of the tanh form */
        const double th = tanh(c * (z + k3 * z * z * z));
        return 0.5 * (1.0 + th) + 0.5 * z * (1.0 - th * th) * c * (1.0 + 3.0 * k3 * z * z);
    }
    case ORACLE_ACT_RELU:
        return z > 0.0 ? 1.0 : 0.0;
    case ORACLE_ACT_IDENTITY:
    default:
        return 1.0;
    }
}

/* One (token, expert) pair: adds its contributions to dx_t [H], dW1e, dW2e (when not NULL)
 * and returns dw = dy . y. gscale is the gate w_j. z, a, da: scratch of 2F, F, F doubles. */
static double pair_backward(int H, int F, int act, const uint16_t *xr, const uint16_t *dyr,
                            double gscale, const uint16_t *W1e, const uint16_t *W2e, double *dx_t,
                            double *dW1e, double *dW2e, double *z, double *a, double *da)
{
    const int gated = (act == ORACLE_ACT_SWIGLU);
    const int w1_cols = gated ? 2 * F : F;
    for (int c = 0; c < w1_cols; ++c) z[c] = 0.0;
    for (int h = 0; h < H; ++h) {
        const double xh = (double)bf16_to_float(xr[h]);
        const uint16_t *wrow = W1e + (size_t)h * w1_cols;
        for (int c = 0; c < w1_cols; ++c) z[c] += xh * (double)bf16_to_float(wrow[c]);
    }
    for (int f = 0; f < F; ++f) a[f] = gated ? z[F + f] * silu(z[f]) : act_apply(act, z[f]);
    /* dw = dy . (a W2); da = w dy W2^T; dW2 += a^T (w dy) */
    double dw = 0.0;
    for (int f = 0; f < F; ++f) {
        const uint16_t *wrow = W2e + (size_t)f * H;
        double s = 0.0;
        for (int n = 0; n < H; ++n) s += (double)bf16_to_float(dyr[n]) * (double)bf16_to_float(wrow[n]);
        dw += a[f] * s;
        da[f] = gscale * s;
        if (dW2e) {
            double *drow = dW2e + (size_t)f * H;
            for (int n = 0; n < H; ++n) drow[n] += a[f] * gscale * (double)bf16_to_float(dyr[n]);
        }
    }
    /* dz (in place of z's gradient: reuse a as the gate part, z[F..] for up when gated) */
    double *dz = z; /* the pre-activations are read before being overwritten below */
    if (gated) {
        for (int f = 0; f < F; ++f) {
            const double g = z[f], u = z[F + f];
            const double s = 1.0 / (1.0 + exp(-g));
            const double dg = da[f] * u * s * (1.0 + g * (1.0 - s));
            const double du = da[f] * g * s;
            dz[f] = dg;
            dz[F + f] = du;
        }
    } else {
        for (int f = 0; f < F; ++f) dz[f] = da[f] * act_grad(act, z[f]);
    }
    for (int h = 0; h < H; ++h) {
        const double xh = (double)bf16_to_float(xr[h]);
        const uint16_t *wrow = W1e + (size_t)h * w1_cols;
        double s = 0.0;
        for (int c = 0; c < w1_cols; ++c) s += dz[c] * (double)bf16_to_float(wrow[c]);
        dx_t[h] += s;
        if (dW1e) {
            double *drow = dW1e + (size_t)h * w1_cols;
            for (int c = 0; c < w1_cols; ++c) drow[c] += xh * dz[c];
        }
    }
    return dw;
}

/* Gradients of the whole layer (all T tokens): dx [T,H], dWg [H,E], dbias [E],
 * dW1 [E,H,w1_cols], dW2 [E,F,H], all fp64; dy [T,H] bf16. Tokens are taken in order, so
 * the weight-gradient sums run over tokens ascending. Returns -3 for SOFTMAX_ALL. */
int oracle_moe_backward(int T, int H, int F, int E, int k, int act, int gate, const uint16_t *x,
                        const uint16_t *Wg, const float *bias, const uint16_t *W1,
                        const uint16_t *W2, const uint16_t *dy, double *dx, double *dWg,
                        double *dbias, double *dW1, double *dW2)
{
    if (T < 0 || H < 1 || F < 1 || E < 1 || k < 1 || k > E) return -1;
    if (gate == ORACLE_GATE_SOFTMAX_ALL) return -3;
    const size_t w1e = w1_expert_elems(H, F, act);
    const size_t w2e = (size_t)F * H;
    memset(dx, 0, sizeof(double) * (size_t)T * H);
    memset(dWg, 0, sizeof(double) * (size_t)H * E);
    memset(dbias, 0, sizeof(double) * (size_t)E);
    memset(dW1, 0, sizeof(double) * w1e * E);
    memset(dW2, 0, sizeof(double) * w2e * E);
    float *l = (float *)malloc(sizeof(float) * (size_t)E);
    unsigned char *taken = (unsigned char *)malloc((size_t)E);
    int32_t *sel = (int32_t *)malloc(sizeof(int32_t) * (size_t)k);
    double *w = (double *)malloc(sizeof(double) * (size_t)k);
    double *dw = (double *)malloc(sizeof(double) * (size_t)k);
    double *z = (double *)malloc(sizeof(double) * 2 * (size_t)F);
    double *a = (double *)malloc(sizeof(double) * (size_t)F);
    double *da = (double *)malloc(sizeof(double) * (size_t)F);
    int rc = (l && taken && sel && w && dw && z && a && da) ? 0 : -4;
    for (int t = 0; t < T && rc == 0; ++t) {
        const uint16_t *xr = x + (size_t)t * H, *dyr = dy + (size_t)t * H;
        oracle_router_logits(1, H, E, xr, Wg, gate == ORACLE_GATE_SELECT_BIAS ? NULL : bias, l);
        topk_one(E, k, gate, l, bias, sel, w, taken);
        double *dxt = dx + (size_t)t * H;
        for (int j = 0; j < k; ++j) {
            const int e = sel[j];
            dw[j] = pair_backward(H, F, act, xr, dyr, w[j], W1 + (size_t)e * w1e, W2 + (size_t)e * w2e,
                                  dxt, dW1 + (size_t)e * w1e, dW2 + (size_t)e * w2e, z, a, da);
        }
        double wdw = 0.0;
        for (int j = 0; j < k; ++j) wdw += w[j] * dw[j];
        for (int j = 0; j < k; ++j) {
            const int e = sel[j];
            const double dl = (dw[j] - wdw) * w[j];
            for (int h = 0; h < H; ++h) {
                const size_t he = (size_t)h * E + e;
                dxt[h] += dl * (double)bf16_to_float(Wg[he]);
                dWg[he] += (double)bf16_to_float(xr[h]) * dl;
            }
            if (gate != ORACLE_GATE_SELECT_BIAS) dbias[e] += dl;
        }
    }
    free(l);
    free(taken);
    free(sel);
    free(w);
    free(dw);
    free(z);
    free(a);
    free(da);
    return rc;
}

/* dx for a list of tokens only (each token's input gradient needs nothing of the others):
 * dx_out [ntok, H] fp64. */
int oracle_moe_backward_dx_tokens(int T, int H, int F, int E, int k, int act, int gate,
                                  const uint16_t *x, const uint16_t *Wg, const float *bias,
                                  const uint16_t *W1, const uint16_t *W2, const uint16_t *dy,
                                  int ntok, const int32_t *tokens, double *dx_out)
{
    if (T < 0 || H < 1 || F < 1 || E < 1 || k < 1 || k > E || ntok < 0) return -1;
    if (gate == ORACLE_GATE_SOFTMAX_ALL) return -3;
    for (int i = 0; i < ntok; ++i)
        if (tokens[i] < 0 || tokens[i] >= T) return -2;
    const size_t w1e = w1_expert_elems(H, F, act);
    const size_t w2e = (size_t)F * H;
    int bad = 0;
#pragma omp parallel
    {
        float *l = (float *)malloc(sizeof(float) * (size_t)E);
        unsigned char *taken = (unsigned char *)malloc((size_t)E);
        int32_t *sel = (int32_t *)malloc(sizeof(int32_t) * (size_t)k);
        double *w = (double *)malloc(sizeof(double) * (size_t)k);
        double *dw = (double *)malloc(sizeof(double) * (size_t)k);
        double *z = (double *)malloc(sizeof(double) * 2 * (size_t)F);
        double *a = (double *)malloc(sizeof(double) * (size_t)F);
        double *da = (double *)malloc(sizeof(double) * (size_t)F);
        const int ok = l && taken && sel && w && dw && z && a && da;
#pragma omp for schedule(dynamic, 1)
        for (int i = 0; i < ntok; ++i) {
            if (!ok) {
#pragma omp atomic write
                bad = 1;
                continue;
            }
            const int t = tokens[i];
            const uint16_t *xr = x + (size_t)t * H, *dyr = dy + (size_t)t * H;
            oracle_router_logits(1, H, E, xr, Wg, gate == ORACLE_GATE_SELECT_BIAS ? NULL : bias, l);
            topk_one(E, k, gate, l, bias, sel, w, taken);
            double *dxt = dx_out + (size_t)i * H;
            for (int h = 0; h < H; ++h) dxt[h] = 0.0;
            for (int j = 0; j < k; ++j) {
                const int e = sel[j];
                dw[j] = pair_backward(H, F, act, xr, dyr, w[j], W1 + (size_t)e * w1e,
                                      W2 + (size_t)e * w2e, dxt, NULL, NULL, z, a, da);
            }
            double wdw = 0.0;
            for (int j = 0; j < k; ++j) wdw += w[j] * dw[j];
            for (int j = 0; j < k; ++j) {
                const double dl = w[j] * (dw[j] - wdw);
                for (int h = 0; h < H; ++h)
                    dxt[h] += dl * (double)bf16_to_float(Wg[(size_t)h * E + sel[j]]);
            }
        }
        free(l);
        free(taken);
        free(sel);
        free(w);
        free(dw);
        free(z);
        free(a);
        free(da);
    }
    return bad ? -4 : 0;
}
