/*
 * sf_oracle.c -- CPU oracle of the Sparse-First sparse training step.
 *
 * TEST INFRASTRUCTURE ONLY. Only the test suite, the smoke check and the benchmark's CPU
 * baseline leg may load this library. The product (the CUDA library and its Python binding)
 * never calls it, and it shares no code, header, table or constant with the CUDA path.
 *
 * What it restates: the Sparse-First fine-tuning page (tensorwirelabs.com,
 * paper-sparse-first), sections 2.1 to 2.4:
 *   - 2.1 Observing activity: the per-window charge rule and the row masks;
 *   - 2.2 Masked backward pass: dW = dX^T A, skipping all-empty 32-row tiles;
 *   - 2.3 (storage): W = s*q + delta, fp16 moments only for active rows,
 *         fused update that rebuilds the fp32 weight and writes back q, delta and live weights;
 *   - 2.4 (coupled pairs): the mixed gradient of each matrix goes through Adam with bias
 *         correction, and weight decay carries a factor cos(alpha).
 * Code is plain loops, single threaded, slow on purpose so that it can be read against the
 * text. Where the text leaves a step open, the reading taken is stated beside the code.
 *
 * Precision. The weight gradient and the embedding-row gradient, which the pages do not tie to
 * a precision, are summed in fp64. The update works in fp32 because the pages rebuild "the fp32
 * weight" and keep fp16 moments; its operation order is fixed below and the file is built with
 * -ffp-contract=off so that no multiply-add is fused behind the reader's back.
 *
 * Parity status: every exported function is pinned by tests/test_oracle_pins.py against closed
 * forms, invariants, library routines (numpy / torch) or brute force. None is unpinned.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

/* ------------------------------------------------------------------------------------------ */
/* Number formats, written from the IEEE 754 binary16 and bfloat16 bit layouts.              */
/* ------------------------------------------------------------------------------------------ */

/* bfloat16 is the upper half of an IEEE binary32: widening is exact. */
float orc_bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* binary32 -> bfloat16, round to nearest, ties to even (NaN stays a quiet NaN). */
uint16_t orc_f32_to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu) != 0)
        return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t keep = u >> 16;            /* the 16 bits that survive */
    uint32_t drop = u & 0xFFFFu;        /* the 16 bits that are rounded away */
    if (drop > 0x8000u || (drop == 0x8000u && (keep & 1u)))
        keep += 1;                      /* a carry into the exponent is the correct overflow */
    return (uint16_t)keep;
}

/* binary16 -> binary32: sign, 5-bit exponent (bias 15), 10-bit fraction. Exact. */
float orc_f16_to_f32(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1F;
    int frac = h & 0x3FF;
    float mag;
    if (e == 0)
        mag = ldexpf((float)frac, -24);                 /* subnormal: frac * 2^-24 */
    else if (e == 31)
        mag = frac ? NAN : INFINITY;
    else
        mag = ldexpf((float)(1024 + frac), e - 25);     /* (1 + frac/1024) * 2^(e-15) */
    return sign ? -mag : mag;
}

/* binary32 -> binary16, round to nearest, ties to even; overflow gives infinity. */
uint16_t orc_f32_to_f16(float f)
{
    uint16_t sign = signbit(f) ? 0x8000u : 0u;
    float a = fabsf(f);
    if (isnan(a))
        return (uint16_t)(sign | 0x7E00u);
    if (a >= 65520.0f)                  /* halfway between 65504 and 2^16 rounds to 2^16: inf */
        return (uint16_t)(sign | 0x7C00u);
    if (a < 0x1p-14f) {                 /* subnormal range: units of 2^-24 */
        float units = rintf(a * 0x1p24f);               /* scaling by 2^24 is exact */
        return (uint16_t)(sign | (uint16_t)units);      /* 1024 units is the smallest normal */
    }
    int ex;
    frexpf(a, &ex);                     /* a = fr * 2^ex, fr in [0.5, 1) */
    int E = ex - 1;                     /* a in [2^E, 2^(E+1)) */
    float sig = rintf(ldexpf(a, 10 - E));               /* in [1024, 2048], exact scaling */
    if (sig == 2048.0f) {
        sig = 1024.0f;
        E += 1;
    }
    return (uint16_t)(sign | (uint16_t)((E + 15) << 10) | (uint16_t)((int)sig - 1024));
}

/* ------------------------------------------------------------------------------------------ */
/* 2.1 Observing activity: the charge rule and the row mask.                                   */
/* ------------------------------------------------------------------------------------------ */

/*
 * One observation window for a matrix of R rows. h[r] is the row's activity in the window
 * (its token hit count for the embedding, its output magnitude for a projection), hmax the
 * busiest row's. Section 2.1 states the rule in words: the new charge is half the old one plus
 * half the row's share of the window, share = h / hmax. Readings: an empty window (hmax == 0) gives share 0 (pure decay);
 * the share is an fp32 division; both halvings are exact, so the new charge is rounded once.
 * Row r is active while its charge is at least the threshold (0.01 on the pages), compared in
 * fp32. Bit i of words[w] is row 32*w + i.
 */
static void orc_charge_fold(int R, float *charge, const float *h, float hmax, float thr,
                            uint32_t *words)
{
    for (int w = 0; w < R / 32; ++w)
        words[w] = 0;
    for (int r = 0; r < R; ++r) {
        float share = (hmax == 0.0f) ? 0.0f : h[r] / hmax;
        charge[r] = 0.5f * charge[r] + 0.5f * share;
        if (charge[r] >= thr)
            words[r / 32] |= 1u << (r % 32);
    }
}

/* Embedding conductor: h[r] = number of times token id r occurs in the window.
 * Returns the number of ids outside [0, R) (they are ignored). h_scratch holds R floats. */
int orc_window_tokens(int R, float *charge, const int32_t *tok, int n, float thr,
                      uint32_t *words, float *h_scratch)
{
    int bad = 0;
    for (int r = 0; r < R; ++r)
        h_scratch[r] = 0.0f;
    for (int i = 0; i < n; ++i) {
        if (tok[i] < 0 || tok[i] >= R) {
            ++bad;
            continue;
        }
        h_scratch[tok[i]] += 1.0f;       /* counts stay exact below 2^24 */
    }
    float hmax = 0.0f;
    for (int r = 0; r < R; ++r)
        if (h_scratch[r] > hmax)
            hmax = h_scratch[r];
    orc_charge_fold(R, charge, h_scratch, hmax, thr, words);
    return bad;
}

/* Projection row tracker. Y is the forward output, T tokens x R rows, bf16, row-major.
 * Reading of "output magnitudes": a row's magnitude is the largest |Y[t, r]| over the
 * window's tokens, taken on the bf16 values widened to fp32 (exact, independent of order).
 * Section 2.1 speaks of magnitudes of outputs and says nothing of outputs that are not finite.
 * Reading for those: a NaN output carries no magnitude and is skipped; an infinite output counts
 * as the largest finite bfloat16 magnitude (bits 0x7F7F), so the row is as active as a row can
 * be and every charge stays finite. Returns the number of non-finite outputs seen. */
int orc_window_outputs(int R, float *charge, const uint16_t *Y, int T, float thr,
                       uint32_t *words, float *h_scratch)
{
    const float largest = orc_bf16_to_f32(0x7F7Fu);
    int nonfinite = 0;
    for (int r = 0; r < R; ++r) {
        float m = 0.0f;
        for (int t = 0; t < T; ++t) {
            float a = fabsf(orc_bf16_to_f32(Y[(size_t)t * R + r]));
            if (isnan(a)) {
                ++nonfinite;
                continue;
            }
            if (isinf(a)) {
                ++nonfinite;
                a = largest;
            }
            if (a > m)
                m = a;
        }
        h_scratch[r] = m;
    }
    float hmax = 0.0f;
    for (int r = 0; r < R; ++r)
        if (h_scratch[r] > hmax)
            hmax = h_scratch[r];
    orc_charge_fold(R, charge, h_scratch, hmax, thr, words);
    return nonfinite;
}

/* The charge rule of one window from the rows' activities h[R] given directly (the busiest row
 * is found here). window_tokens and window_outputs are this rule applied to the activities they
 * count; split across several processes, each counts its share of the window's tokens and the
 * shares are combined (summed hit counts, largest magnitude) before the rule is applied once. */
void orc_window_activity(int R, float *charge, const float *h, float thr, uint32_t *words)
{
    float hmax = 0.0f;
    for (int r = 0; r < R; ++r)
        if (h[r] > hmax)
            hmax = h[r];
    orc_charge_fold(R, charge, h, hmax, thr, words);
}

/* The row tracker's activities alone: h[r] = largest |Y[t, r]| over the T tokens, with the
 * reading for non-finite outputs of orc_window_outputs. Returns the number of non-finite outputs. */
int orc_row_magnitudes(int R, const uint16_t *Y, int T, float *h)
{
    const float largest = orc_bf16_to_f32(0x7F7Fu);
    int nonfinite = 0;
    for (int r = 0; r < R; ++r) {
        float m = 0.0f;
        for (int t = 0; t < T; ++t) {
            float a = fabsf(orc_bf16_to_f32(Y[(size_t)t * R + r]));
            if (isnan(a)) {
                ++nonfinite;
                continue;
            }
            if (isinf(a)) {
                ++nonfinite;
                a = largest;
            }
            if (a > m)
                m = a;
        }
        h[r] = m;
    }
    return nonfinite;
}

/* The per-step lists every later stage reads: active rows ascending, and the 32-row tiles that
 * hold at least one active row, ascending. Returns nothing; counts go to n_rows / n_tiles. */
void orc_mask_lists(int R, const uint32_t *words, int32_t *rows, int32_t *n_rows,
                    int32_t *tiles, int32_t *n_tiles)
{
    int nr = 0, nt = 0;
    for (int w = 0; w < R / 32; ++w) {
        if (words[w] == 0)
            continue;
        tiles[nt++] = w;
        for (int i = 0; i < 32; ++i)
            if (words[w] & (1u << i))
                rows[nr++] = 32 * w + i;
    }
    *n_rows = nr;
    *n_tiles = nt;
}

/*
 * Moments exist only for active rows (section 2.3). Reading: a row that turns active starts
 * with zero moments and a zero step count; a row that turns inactive drops its moments. The
 * oracle keeps moments per row (dense R x C arrays), so "dropping" writes zeros and the row
 * restarts from zero if it comes back. Rows whose activity did not change are left alone.
 */
void orc_moments_follow_mask(int R, int C, const uint32_t *old_words, const uint32_t *new_words,
                             uint16_t *m, uint16_t *v, int32_t *step)
{
    for (int r = 0; r < R; ++r) {
        int was = (old_words[r / 32] >> (r % 32)) & 1;
        int now = (new_words[r / 32] >> (r % 32)) & 1;
        if (was == now)
            continue;
        for (int c = 0; c < C; ++c) {
            m[(size_t)r * C + c] = 0;
            v[(size_t)r * C + c] = 0;
        }
        step[r] = 0;
    }
}

/* ------------------------------------------------------------------------------------------ */
/* 2.2 Masked backward pass.                                                                   */
/* ------------------------------------------------------------------------------------------ */

/*
 * dW = dX^T A for a projection with R output rows and C input columns over T tokens.
 * dX is T x R (upstream gradient of the outputs), A is T x C (the inputs), both bf16 row-major.
 * Per section 2.2 the mask is checked per tile of 32 rows: an all-empty tile does nothing at
 * all, and inside an active tile only active rows are written. dW is R x C fp64; rows that are
 * not active are never touched. Each entry is the fp64 sum over tokens in ascending order.
 */
void orc_masked_dw(int T, int R, int C, const uint16_t *dX, const uint16_t *A,
                   const uint32_t *words, double *dW)
{
    for (int w = 0; w < R / 32; ++w) {
        if (words[w] == 0)
            continue;                                   /* all-empty tile: no work, no write */
        for (int i = 0; i < 32; ++i) {
            if (!(words[w] & (1u << i)))
                continue;                               /* inactive row of an active tile */
            int r = 32 * w + i;
            for (int c = 0; c < C; ++c) {
                double acc = 0.0;
                for (int t = 0; t < T; ++t)
                    acc += (double)orc_bf16_to_f32(dX[(size_t)t * R + r]) *
                           (double)orc_bf16_to_f32(A[(size_t)t * C + c]);
                dW[(size_t)r * C + c] = acc;
            }
        }
    }
}

/*
 * Embedding-row gradient (sections 1 and 2.2): a row can only have gradient if its token is in
 * the batch, and the mask keeps active rows only. G[r, :] = sum of dY[t, :] over tokens t with id r, summed in
 * fp64 in ascending t. Active rows with no token get zeros; inactive rows are not touched.
 * dY is n x H bf16 row-major, G is V x H fp64.
 */
void orc_embed_grad(int n, const int32_t *tok, int H, const uint16_t *dY, int V,
                    const uint32_t *words, double *G)
{
    for (int r = 0; r < V; ++r)
        if ((words[r / 32] >> (r % 32)) & 1)
            for (int c = 0; c < H; ++c)
                G[(size_t)r * H + c] = 0.0;
    for (int t = 0; t < n; ++t) {
        int r = tok[t];
        if (r < 0 || r >= V || !((words[r / 32] >> (r % 32)) & 1))
            continue;                                   /* token of an inactive row: dropped */
        for (int c = 0; c < H; ++c)
            G[(size_t)r * H + c] += (double)orc_bf16_to_f32(dY[(size_t)t * H + c]);
    }
}

/* ------------------------------------------------------------------------------------------ */
/* 2.3 int8 weights with a per-row scale and an fp32 residual.                                */
/* ------------------------------------------------------------------------------------------ */

/*
 * Quantise one row: W = s*q + delta. Reading of the dropped formula: symmetric per-row absmax,
 * s = max|W| / 127, q = round-half-even(W / s) clamped to [-127, 127], delta = W - s*q computed
 * with one rounding (a fused multiply-add). A row of zeros gets s = 0, q = 0, delta = W.
 */
static void orc_quantize_row(int C, const float *W, int8_t *q, float *s, float *delta)
{
    float amax = 0.0f;
    for (int c = 0; c < C; ++c)
        if (fabsf(W[c]) > amax)
            amax = fabsf(W[c]);
    float sc = amax / 127.0f;
    *s = sc;
    for (int c = 0; c < C; ++c) {
        if (sc == 0.0f) {
            q[c] = 0;
            delta[c] = W[c];
            continue;
        }
        float k = rintf(W[c] / sc);                     /* default rounding: ties to even */
        if (k > 127.0f) k = 127.0f;
        if (k < -127.0f) k = -127.0f;
        q[c] = (int8_t)k;
        delta[c] = fmaf(-sc, k, W[c]);
    }
}

void orc_quantize_rows(int R, int C, const float *W, int8_t *q, float *s, float *delta)
{
    for (int r = 0; r < R; ++r)
        orc_quantize_row(C, W + (size_t)r * C, q + (size_t)r * C, s + r, delta + (size_t)r * C);
}

/* ------------------------------------------------------------------------------------------ */
/* 2.3 + 2.4 The fused sparse update with the coupled pair mix.                                */
/* ------------------------------------------------------------------------------------------ */

/* Bias-correction factor 1 / (1 - beta^t) for the fp32 beta given, with beta^t formed by t
 * successive fp64 multiplications and the quotient rounded once to fp32. */
float orc_bias_correction(float beta, int t)
{
    double p = 1.0;
    for (int i = 0; i < t; ++i)
        p *= (double)beta;
    return (float)(1.0 / (1.0 - p));
}

/*
 * One update of the active rows of matrix a (R x C). Storage per section 2.3: q int8, s fp32
 * per row, delta fp32, live bf16 (the weights the next forward pass reads), moments m and v in
 * fp16 (kept here as dense R x C arrays that only active rows use), step counts per row.
 *
 * g is a's gradient (R x C fp32, active rows meaningful). For a matrix in a coupled pair
 * (gate-up, query-output, key-value; section 2.4) pg / pwords give the partner's gradient and
 * mask; the effective gradient is c_self*g + c_partner*g_partner, where the partner's row
 * contributes only when that row is active in the partner (an inactive row has no gradient).
 * Unpaired matrices pass pg = NULL. The pages' formula for the two coefficients is not in the
 * text; the caller supplies them.
 *
 * Order of operations per element (all fp32, one rounding per line):
 *   W   = fma(s, q, delta)                       rebuild the weight
 *   g  <- clamp(g, -clip, clip) if clip > 0      element clip, off by default
 *   gt  = fma(c_partner, g_partner, c_self * g)  effective gradient
 *   m1  = fma(beta1, m, (1-beta1) * gt)          m, v read from fp16
 *   v1  = fma(beta2, v, (1-beta2) * (gt * gt))
 *   u   = (m1 * bc1(t)) / (sqrt(v1 * bc2(t)) + eps)      t = step count after increment
 *   W'  = fma(-lr, u, W);  W' = fma(-lr*wd, W, W') if wd != 0   (decoupled decay)
 *   m, v <- fp16(m1), fp16(v1)
 * then per row: s' = max|W'| / 127, q' = rint(W'/s') clamped, delta' = fma(-s', q', W'),
 * live = bf16(W'). The Adam step uses m1 and v1 before their fp16 rounding.
 * one_minus_b1 / one_minus_b2 are passed in so that both sides use the same fp32 constants.
 */
void orc_update(int R, int C, int8_t *q, float *s, float *delta, uint16_t *m, uint16_t *v,
                int32_t *step, uint16_t *live, const uint32_t *words, const float *g,
                const uint32_t *pwords, const float *pg, float c_self, float c_partner,
                float lr, float beta1, float beta2, float one_minus_b1, float one_minus_b2,
                float eps, float wd, float clip, float *row_scratch)
{
    for (int r = 0; r < R; ++r) {
        if (!((words[r / 32] >> (r % 32)) & 1))
            continue;                                   /* inactive rows return immediately */
        int partner_live = pg != NULL && ((pwords[r / 32] >> (r % 32)) & 1);
        int t = step[r] + 1;
        step[r] = t;
        float bc1 = orc_bias_correction(beta1, t);
        float bc2 = orc_bias_correction(beta2, t);
        for (int c = 0; c < C; ++c) {
            size_t i = (size_t)r * C + c;
            float W = fmaf(s[r], (float)q[i], delta[i]);
            float ga = g[i];
            float gb = partner_live ? pg[i] : 0.0f;
            if (clip > 0.0f) {
                ga = fminf(fmaxf(ga, -clip), clip);
                gb = fminf(fmaxf(gb, -clip), clip);
            }
            float gt = fmaf(c_partner, gb, c_self * ga);
            float m1 = fmaf(beta1, orc_f16_to_f32(m[i]), one_minus_b1 * gt);
            float v1 = fmaf(beta2, orc_f16_to_f32(v[i]), one_minus_b2 * (gt * gt));
            float u = (m1 * bc1) / (sqrtf(v1 * bc2) + eps);
            float Wn = fmaf(-lr, u, W);
            if (wd != 0.0f)
                Wn = fmaf(-lr * wd, W, Wn);
            m[i] = orc_f32_to_f16(m1);
            v[i] = orc_f32_to_f16(v1);
            row_scratch[c] = Wn;
        }
        orc_quantize_row(C, row_scratch, q + (size_t)r * C, s + r, delta + (size_t)r * C);
        for (int c = 0; c < C; ++c)
            live[(size_t)r * C + c] = orc_f32_to_bf16(row_scratch[c]);
    }
}

/* Array forms of the four conversions, for the format pins. */
void orc_convert(int kind, long n, const void *in, void *out)
{
    for (long i = 0; i < n; ++i) {
        switch (kind) {
        case 0: ((float *)out)[i] = orc_bf16_to_f32(((const uint16_t *)in)[i]); break;
        case 1: ((uint16_t *)out)[i] = orc_f32_to_bf16(((const float *)in)[i]); break;
        case 2: ((float *)out)[i] = orc_f16_to_f32(((const uint16_t *)in)[i]); break;
        case 3: ((uint16_t *)out)[i] = orc_f32_to_f16(((const float *)in)[i]); break;
        default: return;
        }
    }
}

/* The fp32 weight the update rebuilds (section 2.3): W = fma(s, q, delta), one rounding. */
void orc_rebuild_rows(int R, int C, const int8_t *q, const float *s, const float *delta, float *W)
{
    for (int r = 0; r < R; ++r)
        for (int c = 0; c < C; ++c) {
            size_t i = (size_t)r * C + c;
            W[i] = fmaf(s[r], (float)q[i], delta[i]);
        }
}

/* ------------------------------------------------------------------------------------------ */
/* 2.6 Checkpoint and rewind of the active rows.                                               */
/* ------------------------------------------------------------------------------------------ */

/*
 * Section 2.6 saves rows of the active set only. Reading taken: a checkpoint is a
 * snapshot, at save time, of every active row's storage and optimizer state: its row id, q, s,
 * delta, m, v and step count. Rows are saved in ascending row order. Returns the rows saved.
 * Buffers hold cap rows (rows beyond cap are not saved; the return value says how many were).
 */
int orc_checkpoint_save(int R, int C, const int8_t *q, const float *s, const float *delta,
                        const uint16_t *m, const uint16_t *v, const int32_t *step,
                        const uint32_t *words, int cap, int32_t *rows, int8_t *cq, float *cs,
                        float *cdelta, uint16_t *cm, uint16_t *cv, int32_t *cstep)
{
    int k = 0;
    for (int r = 0; r < R; ++r) {
        if (!((words[r / 32] >> (r % 32)) & 1))
            continue;
        if (k >= cap)
            return k;
        rows[k] = r;
        cs[k] = s[r];
        cstep[k] = step[r];
        for (int c = 0; c < C; ++c) {
            size_t i = (size_t)r * C + c, j = (size_t)k * C + c;
            cq[j] = q[i];
            cdelta[j] = delta[i];
            cm[j] = m[i];
            cv[j] = v[i];
        }
        ++k;
    }
    return k;
}

/*
 * Rewind: every saved row gets back its q, s and delta, and its live weights are rebuilt from
 * them (bf16 of fma(s, q, delta)). Moments exist only for active rows (section 2.3), so a saved
 * row gets its moments and step count back only if it is active now; otherwise they stay
 * dropped. Rows that were not saved are left as they are.
 */
void orc_checkpoint_restore(int R, int C, int8_t *q, float *s, float *delta, uint16_t *m,
                            uint16_t *v, int32_t *step, uint16_t *live, const uint32_t *words,
                            int n, const int32_t *rows, const int8_t *cq, const float *cs,
                            const float *cdelta, const uint16_t *cm, const uint16_t *cv,
                            const int32_t *cstep)
{
    (void)R;
    for (int k = 0; k < n; ++k) {
        int r = rows[k];
        int active = (words[r / 32] >> (r % 32)) & 1;
        s[r] = cs[k];
        if (active)
            step[r] = cstep[k];
        for (int c = 0; c < C; ++c) {
            size_t i = (size_t)r * C + c, j = (size_t)k * C + c;
            q[i] = cq[j];
            delta[i] = cdelta[j];
            live[i] = orc_f32_to_bf16(fmaf(cs[k], (float)cq[j], cdelta[j]));
            if (active) {
                m[i] = cm[j];
                v[i] = cv[j];
            }
        }
    }
}
