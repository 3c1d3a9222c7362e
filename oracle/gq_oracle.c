/*
 * gq_oracle.c -- plain, slow, sequential CPU oracle for bucketed gradient quantization.
 *
 * TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU-baseline leg
 * load it; the CUDA product path never does, and the two share no code.
 *
 * Page references ([P1], [P2], [P3]) are defined in gq_oracle.h.  Every loop runs over the
 * elements of a bucket in index order.  Floating point is IEEE binary32/binary64 with
 * round-to-nearest and no contraction (built with -ffp-contract=off).  The pages fix no
 * precision; the level fits and rounding decisions are taken in binary32 (the precision of
 * the gradients and of the CUDA kernels), and every fit decision is taken from exact integer
 * data (fixed-point positions and sums), so that it does not depend on summation order.
 *
 * Pins (checked by the CPU test suite, not by re-typing these formulas):
 *   - Philox4x32-10 against the published known-answer vectors of the generator;
 *   - stochastic rounding against the 0.7 example of [P3] and Monte Carlo mean / variance;
 *   - ORQ's greedy against an independent naive greedy on the raw values;
 *   - BinGrad-b's split against brute force over all thresholds;
 *   - BinGrad-pb's pair against brute force over the admissible grid pairs, its range against
 *     BinGrad-b's ("wider range", [P2] "Proposed method"), its per-value bias against BinGrad-b's
 *     error, and the ordering of quantization errors BinGrad-b <= BinGrad-pb stated in [P2]
 *     "Key findings";
 *   - QSGD/TernGrad against hand-computed closed forms;
 *   - packing against a bit-by-bit unpacker; error feedback against its telescoping sum;
 *   - base-s packing against a big-integer construction of the digit stream, the round trip,
 *     and its bits per code against log2(s) (the compression ratios of [P2] "Key findings");
 *   - nearest-level QSGD against brute force over the levels and its tie rule; the scaled sign
 *     against the exact rational mean of |u|, its sign rule and its error-feedback sum;
 *   - QSGD-l2's scale against the exact norm and its unbiasedness; Elias gamma against the
 *     published codeword table, the stream against a bit string built from it, the offsets,
 *     the round trip and the expected length.
 * The pages state BinGrad-pb's properties (wider range, less bias, larger error than BinGrad-b)
 * but not its formula: the reading below is pinned to those properties.
 */
#include "gq_oracle.h"

#include <float.h>
#include <math.h>
#include <stdlib.h>
#include <string.h>

#define OR_GRIDPTS 64      /* candidate grid points j = 0..63 */
#define OR_TOPCELL 62      /* cells 0..62 lie between grid points */
#define OR_ORQ_FBITS 16    /* fraction bits of ORQ fixed-point positions */
#define OR_PB_FBITS 16     /* fraction bits of BinGrad-pb fixed-point positions */

/* ------------------------------------------------------------------------------------------ */
/* Philox4x32-10 (counter-based generator, Salmon et al., "Parallel Random Numbers: As Easy as */
/* 1, 2, 3", SC'11).  Written from the published definition: ten rounds of two 32x32->64      */
/* multiplications, the key bumped by the two Weyl constants between rounds.                   */
/* ------------------------------------------------------------------------------------------ */
void or_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4])
{
    uint32_t x0 = ctr[0], x1 = ctr[1], x2 = ctr[2], x3 = ctr[3];
    uint32_t k0 = key[0], k1 = key[1];
    for (int round = 0; round < 10; ++round) {
        if (round > 0) {
            k0 += 0x9E3779B9u;
            k1 += 0xBB67AE85u;
        }
        uint64_t p0 = (uint64_t)0xD2511F53u * (uint64_t)x0;
        uint64_t p1 = (uint64_t)0xCD9E8D57u * (uint64_t)x2;
        uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        uint32_t y0 = hi1 ^ x1 ^ k0;
        uint32_t y1 = lo1;
        uint32_t y2 = hi0 ^ x3 ^ k1;
        uint32_t y3 = lo0;
        x0 = y0; x1 = y1; x2 = y2; x3 = y3;
    }
    out[0] = x0; out[1] = x1; out[2] = x2; out[3] = x3;
}

/*
 * Randomness of the rounding step.  [P2] "Proposed method" and [P3] (stochastic quantization)
 * only ask for random rounding; the draw is keyed on (seed, step, worker, global element
 * index) so that it is reproducible and independent of the launch shape.  Reading: key =
 * (seed low word, seed high word), counter = (i/4 low word, i/4 high word, step low word,
 * worker); element i takes output word i mod 4; U = rz(word) * 2^-32, rz(word) the largest
 * binary32 value not above the word (its 24 leading significant bits).  Then
 * P(U < p) = ceil(p * 2^32) * 2^-32 for every p in [0, 1]: exactly p for every binary32 p
 * >= 2^-9, within 2^-32 below that, which is what keeps the rounding unbiased ([P3]).
 */
static float uniform_from_word(uint32_t word)
{
    int len = 0;
    for (uint32_t t = word; t; t >>= 1) ++len;
    if (len > 24) word &= ~((1u << (len - 24)) - 1u); /* keep the 24 leading significant bits */
    return (float)word * 0x1p-32f;                     /* exact: at most 24 significant bits */
}

float or_uniform(uint64_t seed, uint64_t step, uint32_t worker, int64_t i)
{
    uint64_t blk = (uint64_t)i >> 2;
    uint32_t ctr[4] = {(uint32_t)blk, (uint32_t)(blk >> 32), (uint32_t)step, worker};
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    uint32_t out[4];
    or_philox4x32_10(ctr, key, out);
    uint32_t word = out[(uint64_t)i & 3u];
    return uniform_from_word(word);
}

/* floor(log2(m)) for finite m > 0, read from the binary32 encoding. */
int or_fexpo(float m)
{
    uint32_t bits;
    memcpy(&bits, &m, sizeof bits);
    int ex = (int)((bits >> 23) & 0xffu);
    if (ex != 0) return ex - 127;
    uint32_t mant = bits & 0x7fffffu;
    int msb = 31;
    while (msb > 0 && !((mant >> msb) & 1u)) --msb;
    return msb - 149;
}

/* Saturate to [0, 1]; NaN becomes 0. */
static float sat01(float x)
{
    if (!(x > 0.0f)) return 0.0f;
    if (x > 1.0f) return 1.0f;
    return x;
}

/* ------------------------------------------------------------------------------------------ */
/* Clipping.  [P2] "Proposed method": gradients are clipped in the distributed setting,        */
/* notably for ORQ with few levels.  Reading: per bucket, symmetric about zero at +-c*sigma,   */
/* sigma the population standard deviation of the bucket's values.  sigma is computed from    */
/* exact integer sums of the values in fixed point with 20 fraction bits below the bucket's    */
/* largest magnitude, so that it does not depend on summation order.                           */
/* ------------------------------------------------------------------------------------------ */
float or_clip_threshold(const float *v, int n, float c)
{
    float m0 = 0.0f;
    for (int i = 0; i < n; ++i) {
        float a = fabsf(v[i]);
        if (a > m0) m0 = a;
    }
    if (!(m0 > 0.0f) || n <= 0) return 0.0f;
    int e = 20 - or_fexpo(m0);
    int64_t sx = 0, sxx = 0;
    for (int i = 0; i < n; ++i) {
        int64_t x = llrint(ldexp((double)v[i], e));
        sx += x;
        sxx += x * x;
    }
    double mean = (double)sx / (double)n;
    double var = (double)sxx / (double)n - mean * mean;
    if (var < 0.0) var = 0.0;
    double sigma = ldexp(sqrt(var), -e);
    return (float)((double)c * sigma);
}

/* ------------------------------------------------------------------------------------------ */
/* The 64-point candidate grid shared by ORQ and BinGrad-pb: uniform from the bucket minimum   */
/* to its maximum, both ends included (g_j = min + j*(max-min)/63, g_63 = max).  A value's     */
/* position on the grid is kept in fixed point, floor((u - min) * 63/(max-min) * 2^F),        */
/* clamped to [0, 63*2^F]; its cell is min(position >> F, 62).                                 */
/* ------------------------------------------------------------------------------------------ */
typedef struct {
    float mn, mx, step, scale;
    float grid[OR_GRIDPTS];
} or_gridinfo;

/* Returns 0 when the bucket is constant (min == max). */
static int grid_setup(const float *u, int n, int fbits, or_gridinfo *gi)
{
    float mn = u[0], mx = u[0];
    for (int i = 1; i < n; ++i) {
        if (u[i] < mn) mn = u[i];
        if (u[i] > mx) mx = u[i];
    }
    /* canonical zero: -0 + +0 = +0 */
    mn = mn + 0.0f;
    mx = mx + 0.0f;
    gi->mn = mn;
    gi->mx = mx;
    if (!(mx > mn)) return 0;
    float range = mx - mn;
    gi->step = range / 63.0f;
    gi->scale = (63.0f / range) * (float)(1 << fbits);
    for (int j = 0; j < OR_GRIDPTS - 1; ++j) gi->grid[j] = mn + (float)j * gi->step;
    gi->grid[OR_GRIDPTS - 1] = mx;
    return 1;
}

static int32_t grid_pos(const or_gridinfo *gi, float u, int fbits)
{
    int32_t top = (int32_t)63 << fbits;
    float y = (u - gi->mn) * gi->scale;
    if (!(y > 0.0f)) return 0;
    if (y >= (float)top) return top;
    return (int32_t)y;
}

static int pos_cell(int32_t pos, int fbits)
{
    int c = pos >> fbits;
    return c > OR_TOPCELL ? OR_TOPCELL : c;
}

int or_grid(const float *u, int n, float grid[64])
{
    or_gridinfo gi;
    if (!grid_setup(u, n, OR_ORQ_FBITS, &gi)) return 0;
    memcpy(grid, gi.grid, sizeof gi.grid);
    return 1;
}

/* ------------------------------------------------------------------------------------------ */
/* ORQ-s.  [P2] "Proposed method" / abstract: unbiased multi-level quantization whose levels   */
/* are chosen greedily to minimise the expected quantization variance.  Reading: the levels    */
/* start as {min, max} (grid indices 0 and 63); each of s-2 rounds adds the grid index whose   */
/* addition gives the smallest total variance sum (b - x)(x - a) over the bucket, ties to the  */
/* smallest index; x in fixed point with 16 fraction bits per cell, the bracket [a, b] of a    */
/* value being the chosen levels around its cell.                                              */
/* ------------------------------------------------------------------------------------------ */

/* Index k of the bracket [lv[k], lv[k+1]] holding cell c (lv sorted, lv[0]=0, lv[nl-1]=63). */
static int bracket_of(const int *lv, int nl, int c)
{
    int k = 0;
    while (k + 2 < nl && lv[k + 1] <= c) ++k;
    return k;
}

static __int128 orq_total_variance(const int32_t *pos, const int *cell, int n, const int *lv, int nl)
{
    __int128 tot = 0;
    for (int i = 0; i < n; ++i) {
        int k = bracket_of(lv, nl, cell[i]);
        int64_t a = (int64_t)lv[k] << OR_ORQ_FBITS;
        int64_t b = (int64_t)lv[k + 1] << OR_ORQ_FBITS;
        tot += (__int128)(b - pos[i]) * (__int128)(pos[i] - a);
    }
    return tot;
}

/* Sorted insertion of c into lv[0..nl). */
static void insert_level(int *lv, int nl, int c)
{
    int k = nl;
    while (k > 0 && lv[k - 1] > c) {
        lv[k] = lv[k - 1];
        --k;
    }
    lv[k] = c;
}

/* Greedy selection; idx_out[0..s) receives the sorted grid indices.  Returns the final total
 * variance in units of (cell * 2^-22)^2 as a double (0 for a constant bucket). */
static double orq_select_pos(const int32_t *pos, const int *cell, int n, int s, int *lv)
{
    int nl = 2;
    lv[0] = 0;
    lv[1] = OR_GRIDPTS - 1;
    __int128 best_v = orq_total_variance(pos, cell, n, lv, nl);
    for (int round = 0; round < s - 2; ++round) {
        int best_c = -1;
        for (int c = 1; c < OR_GRIDPTS - 1; ++c) {
            int used = 0;
            for (int k = 0; k < nl; ++k) used |= (lv[k] == c);
            if (used) continue;
            int trial[OR_GRIDPTS];
            memcpy(trial, lv, sizeof(int) * (size_t)nl);
            insert_level(trial, nl, c);
            __int128 v = orq_total_variance(pos, cell, n, trial, nl + 1);
            if (best_c < 0 || v < best_v) {
                best_c = c;
                best_v = v;
            }
        }
        insert_level(lv, nl, best_c);
        ++nl;
    }
    return (double)best_v;
}

double or_orq_select(const float *u, int n, int s, int *idx_out)
{
    or_gridinfo gi;
    if (!grid_setup(u, n, OR_ORQ_FBITS, &gi)) {
        for (int k = 0; k < s; ++k) idx_out[k] = 0;
        return 0.0;
    }
    int32_t *pos = (int32_t *)malloc(sizeof(int32_t) * (size_t)n);
    int *cell = (int *)malloc(sizeof(int) * (size_t)n);
    for (int i = 0; i < n; ++i) {
        pos[i] = grid_pos(&gi, u[i], OR_ORQ_FBITS);
        cell[i] = pos_cell(pos[i], OR_ORQ_FBITS);
    }
    double v = orq_select_pos(pos, cell, n, s, idx_out);
    free(pos);
    free(cell);
    return v;
}

static void orq_bucket(const or_config *cfg, int worker, uint64_t step, int64_t base,
                       const float *u, int n, uint8_t *code, float *q, float *table,
                       float *blo, float *bhi, float *bp)
{
    int s = cfg->levels;
    or_gridinfo gi;
    if (!grid_setup(u, n, OR_ORQ_FBITS, &gi)) {
        /* constant bucket: every level is the common value, every code 0 */
        for (int k = 0; k < s; ++k) table[k] = gi.mn;
        for (int i = 0; i < n; ++i) {
            code[i] = 0;
            q[i] = gi.mn;
            if (bp) {
                blo[i] = gi.mn;
                bhi[i] = gi.mn;
                bp[i] = 0.0f;
            }
        }
        return;
    }
    int32_t *pos = (int32_t *)malloc(sizeof(int32_t) * (size_t)n);
    int *cell = (int *)malloc(sizeof(int) * (size_t)n);
    for (int i = 0; i < n; ++i) {
        pos[i] = grid_pos(&gi, u[i], OR_ORQ_FBITS);
        cell[i] = pos_cell(pos[i], OR_ORQ_FBITS);
    }
    int lv[OR_GRIDPTS];
    orq_select_pos(pos, cell, n, s, lv);
    for (int k = 0; k < s; ++k) table[k] = gi.grid[lv[k]];
    /* unbiased rounding inside the bracket [a, b]: up with probability (u - a)/(b - a) */
    for (int i = 0; i < n; ++i) {
        int k = bracket_of(lv, s, cell[i]);
        float a = table[k], b = table[k + 1];
        float rinv = 1.0f / (b - a);
        float p = sat01((u[i] - a) * rinv);
        float U = or_uniform(cfg->seed, step, (uint32_t)worker, base + i);
        int c = k + (U < p ? 1 : 0);
        code[i] = (uint8_t)c;
        q[i] = table[c];
        if (bp) {
            blo[i] = a;
            bhi[i] = b;
            bp[i] = p;
        }
    }
    free(pos);
    free(cell);
}

/* ------------------------------------------------------------------------------------------ */
/* QSGD-s / TernGrad.  [P3]: scale by the maximum magnitude and round stochastically to the    */
/* nearest representable levels; TernGrad uses the three levels {-m, 0, m}.  Reading: per      */
/* bucket, m = max|u|, s uniform levels m*(2k-(s-1))/(s-1), k = 0..s-1 (TernGrad is s = 3).    */
/* The message carries m only.                                                                 */
/* ------------------------------------------------------------------------------------------ */
static float qsgd_ratio(int code, int s)
{
    return (float)(2 * code - (s - 1)) / (float)(s - 1);
}

/*
 * nearest = 1: deterministic rounding ([P3] "Deterministic vs stochastic rounding": every value
 * goes to its nearest representable level; simple, but biased).  Same levels and message as
 * QSGD.  Reading: nearest in the binary32 position y below, ties (y - k = 1/2) to the upper
 * level; no random draw.
 */
static float or_l2_scale_fwd(const float *u, int n);

static void qsgd_bucket(const or_config *cfg, int worker, uint64_t step, int64_t base,
                        const float *u, int n, uint8_t *code, float *q, float *table,
                        float *blo, float *bhi, float *bp, int nearest)
{
    int s = cfg->levels;
    float m = 0.0f;
    for (int i = 0; i < n; ++i) {
        float a = fabsf(u[i]);
        if (a > m) m = a;
    }
    if (cfg->scheme == OR_QSGD_L2) m = or_l2_scale_fwd(u, n);
    table[0] = m;
    float inv_m = m > 0.0f ? 1.0f / m : 0.0f;
    float h = (float)(s - 1) * 0.5f;
    for (int i = 0; i < n; ++i) {
        float y = (u[i] * inv_m + 1.0f) * h;   /* position in level units, 0 .. s-1 */
        /* k = trunc(y) clamped to [0, s-2]; y may be infinite (1/m overflows for a subnormal
         * m) or NaN (0 * inf), so the clamp is taken before any conversion to int */
        int k = 0;
        if (y > 0.0f) k = (y >= (float)(s - 2)) ? s - 2 : (int)y;
        float p = y - (float)k;
        int up;
        if (nearest) {
            up = p >= 0.5f;
        } else {
            float U = or_uniform(cfg->seed, step, (uint32_t)worker, base + i);
            up = U < p;
        }
        int c = k + up;
        code[i] = (uint8_t)c;
        q[i] = m * qsgd_ratio(c, s);
        if (bp) {
            blo[i] = m * qsgd_ratio(k, s);
            bhi[i] = m * qsgd_ratio(k + 1, s);
            bp[i] = nearest ? (float)up : sat01(p);
        }
    }
}

/* ------------------------------------------------------------------------------------------ */
/* Scaled sign.  [P3] "Ternary and binary quantization": SignSGD transmits only the signs of   */
/* the gradient (32x compression) and needs error feedback.  The pages fix no scale.  Reading: */
/* per bucket the two levels are -m1 and +m1, m1 the mean of |u| (for fixed signs the scale    */
/* that minimises the squared error), code 1 for u >= 0 (zeros of either sign go up).  m1 is   */
/* computed from an exact integer sum of |u| in fixed point with 45 fraction bits below the    */
/* bucket's largest magnitude (each term below 2^46, so the sum of up to 2^17 terms is exact  */
/* in int64), so that it does not depend on summation order:                                  */
/*   m1 = binary32(((binary64) S * 2^-E) / n),  S = sum of round(|u| * 2^E),  E = 45 - e,     */
/* e = floor(log2 max|u|).  The level table holds {-m1, +m1}.                                  */
/* ------------------------------------------------------------------------------------------ */
float or_sign_scale(const float *u, int n)
{
    float m0 = 0.0f;
    for (int i = 0; i < n; ++i) {
        float a = fabsf(u[i]);
        if (a > m0) m0 = a;
    }
    if (!(m0 > 0.0f) || n <= 0) return m0 > 0.0f ? m0 : 0.0f;  /* zero bucket: 0; NaN/inf: unspecified */
    if (!(m0 <= FLT_MAX)) return m0;
    int E = 45 - or_fexpo(m0);
    int64_t S = 0;
    for (int i = 0; i < n; ++i) S += llrint(ldexp(fabs((double)u[i]), E));
    return (float)(ldexp((double)S, -E) / (double)n);
}

/* ------------------------------------------------------------------------------------------ */
/* QSGD as originally published (Alistarh et al., "QSGD: Communication-Efficient SGD via      */
/* Gradient Quantization and Encoding", NIPS 2017) scales by the l2 norm of the vector; [P3]   */
/* "QSGD" describes it as the generalisation of stochastic quantization whose codes are then    */
/* Elias-coded.  Reading: per bucket, m = ||u||_2 replaces max |u| in QSGD's levels and         */
/* rounding (every |u| <= m, so every value lies inside the level range), computed from the    */
/* same exact fixed-point sums as the clip's sigma (20 fraction bits below the largest          */
/* magnitude): m = binary32(sqrt((binary64) SXX) * 2^-e).                                       */
/* ------------------------------------------------------------------------------------------ */
float or_l2_scale(const float *u, int n)
{
    float m0 = 0.0f;
    for (int i = 0; i < n; ++i) {
        float a = fabsf(u[i]);
        if (a > m0) m0 = a;
    }
    if (!(m0 > 0.0f) || n <= 0) return 0.0f;
    if (!(m0 <= FLT_MAX)) return m0;
    int e = 20 - or_fexpo(m0);
    int64_t sxx = 0;
    for (int i = 0; i < n; ++i) {
        int64_t x = llrint(ldexp((double)u[i], e));
        sxx += x * x;
    }
    return (float)ldexp(sqrt((double)sxx), -e);
}

static void sign_bucket(const float *u, int n, uint8_t *code, float *q, float *table,
                        float *blo, float *bhi, float *bp)
{
    float m1 = or_sign_scale(u, n);
    table[0] = -m1;
    table[1] = m1;
    for (int i = 0; i < n; ++i) {
        int up = u[i] >= 0.0f;
        code[i] = (uint8_t)up;
        q[i] = up ? m1 : -m1;
        if (bp) {
            blo[i] = -m1;
            bhi[i] = m1;
            bp[i] = (float)up;
        }
    }
}

/* ------------------------------------------------------------------------------------------ */
/* BinGrad-b.  [P2]: the biased binary scheme that minimises variance; its two levels adapt to */
/* the gradient distribution.  Reading: the SSE-optimal two-level split (1-D two-means) with  */
/* the levels at the means of each side, deterministic assignment (hence biased).  Sums are   */
/* exact int64 in fixed point with 46 fraction bits below the bucket's largest magnitude; the  */
/* split maximises J(k) = S_k^2/k + (S_n - S_k)^2/(n - k) (equivalently minimises the SSE),    */
/* evaluated in binary64, ties to the smallest k, over splits between distinct values.         */
/* ------------------------------------------------------------------------------------------ */
static int cmp_float(const void *a, const void *b)
{
    float x = *(const float *)a, y = *(const float *)b;
    return (x > y) - (x < y);
}

void or_bingrad_b_fit(const float *u, int n, float *a_out, float *b_out, float *thr, int *split)
{
    float m = 0.0f;
    for (int i = 0; i < n; ++i) {
        float a = fabsf(u[i]);
        if (a > m) m = a;
    }
    if (!(m > 0.0f)) {
        *a_out = 0.0f;
        *b_out = 0.0f;
        *thr = 0.0f;
        *split = 0;
        return;
    }
    float *srt = (float *)malloc(sizeof(float) * (size_t)n);
    memcpy(srt, u, sizeof(float) * (size_t)n);
    qsort(srt, (size_t)n, sizeof(float), cmp_float);
    int e = 46 - or_fexpo(m);
    int64_t *S = (int64_t *)malloc(sizeof(int64_t) * (size_t)(n + 1));
    S[0] = 0;
    for (int i = 0; i < n; ++i) S[i + 1] = S[i] + llrint(ldexp((double)srt[i], e));
    int best = -1;
    double best_j = 0.0;
    for (int k = 1; k < n; ++k) {
        if (!(srt[k - 1] < srt[k])) continue;
        double l = (double)S[k];
        double r = (double)(S[n] - S[k]);
        double j = l * l / (double)k + r * r / (double)(n - k);
        if (best < 0 || j > best_j) {
            best = k;
            best_j = j;
        }
    }
    if (best < 0) {
        /* every value equal: one level, no split */
        *a_out = srt[0] + 0.0f;
        *b_out = srt[0] + 0.0f;
        *thr = srt[0] + 0.0f;
        *split = 0;
    } else {
        *a_out = (float)ldexp((double)S[best] / (double)best, -e);
        *b_out = (float)ldexp((double)(S[n] - S[best]) / (double)(n - best), -e);
        *thr = srt[best];
        *split = best;
    }
    free(S);
    free(srt);
}

static void bingrad_b_bucket(const float *u, int n, uint8_t *code, float *q, float *table,
                             float *blo, float *bhi, float *bp)
{
    float a, b, thr;
    int split;
    or_bingrad_b_fit(u, n, &a, &b, &thr, &split);
    table[0] = a;
    table[1] = b;
    for (int i = 0; i < n; ++i) {
        int c = (split > 0 && u[i] >= thr) ? 1 : 0;
        code[i] = (uint8_t)c;
        q[i] = c ? b : a;
        if (bp) {
            blo[i] = a;
            bhi[i] = b;
            bp[i] = (float)c;
        }
    }
}

/* ------------------------------------------------------------------------------------------ */
/* BinGrad-pb.  [P2] "Proposed method": the binary variant that, unlike BinGrad-b, reduces bias */
/* through a wider range; [P2] "Key findings": its quantization error is larger than           */
/* BinGrad-b's.  Reading ("partially biased"): two levels (g_A, g_B) from the 64-point grid,    */
/* at least as far apart as BinGrad-b's levels (a_b, b_b) on the same bucket: g_A <= a_b and    */
/* g_B >= b_b (A at most the largest grid index whose point is <= a_b, 0 when there is none; B  */
/* at least the smallest whose point is >= b_b, 63 when there is none).  Values between the     */
/* levels are rounded stochastically (unbiased), values outside are clamped to the nearer       */
/* level (biased).  Among the admissible pairs the one that minimises the expected squared      */
/* error                                                                                        */
/*   sum_{x<a} (a-x)^2 + sum_{a<=x<b} (b-x)(x-a) + sum_{x>=b} (x-b)^2                           */
/* is taken, in fixed point with 16 fraction bits per cell (exact int128), ties to the smallest */
/* (A, B).  The range condition makes the span at least BinGrad-b's and every clamped value's   */
/* bias at most its BinGrad-b error; the expected error is never below BinGrad-b's, since       */
/* (b-x)(x-a) >= min(x-a, b-x)^2 for every x between the levels.                                */
/* ------------------------------------------------------------------------------------------ */
static void pb_limits(const or_gridinfo *gi, const float *u, int n, int *Amax, int *Bmin)
{
    float a, b, thr;
    int split;
    or_bingrad_b_fit(u, n, &a, &b, &thr, &split);
    int am = 0, bm = OR_GRIDPTS - 1;
    for (int j = 0; j < OR_GRIDPTS; ++j)
        if (gi->grid[j] <= a) am = j;
    for (int j = OR_GRIDPTS - 1; j >= 0; --j)
        if (gi->grid[j] >= b) bm = j;
    *Amax = am;
    *Bmin = bm;
}

static void pb_select_pos(const int32_t *pos, int n, int Amax, int Bmin, int *A_out, int *B_out)
{
    int bestA = -1, bestB = -1;
    __int128 best_e = 0;
    for (int A = 0; A <= Amax && A < OR_GRIDPTS - 1; ++A) {
        for (int B = (Bmin > A + 1 ? Bmin : A + 1); B < OR_GRIDPTS; ++B) {
            int64_t a = (int64_t)A << OR_PB_FBITS, b = (int64_t)B << OR_PB_FBITS;
            __int128 e = 0;
            for (int i = 0; i < n; ++i) {
                int64_t x = pos[i];
                if (x < a) e += (__int128)(a - x) * (a - x);
                else if (x >= b) e += (__int128)(x - b) * (x - b);
                else e += (__int128)(b - x) * (x - a);
            }
            if (bestA < 0 || e < best_e) {
                bestA = A;
                bestB = B;
                best_e = e;
            }
        }
    }
    *A_out = bestA;
    *B_out = bestB;
}

void or_bingrad_pb_fit(const float *u, int n, int *A, int *B, float *ga, float *gb)
{
    or_gridinfo gi;
    if (!grid_setup(u, n, OR_PB_FBITS, &gi)) {
        *A = 0;
        *B = 0;
        *ga = gi.mn;
        *gb = gi.mn;
        return;
    }
    int32_t *pos = (int32_t *)malloc(sizeof(int32_t) * (size_t)n);
    for (int i = 0; i < n; ++i) pos[i] = grid_pos(&gi, u[i], OR_PB_FBITS);
    int Amax, Bmin;
    pb_limits(&gi, u, n, &Amax, &Bmin);
    pb_select_pos(pos, n, Amax, Bmin, A, B);
    *ga = gi.grid[*A];
    *gb = gi.grid[*B];
    free(pos);
}

static void bingrad_pb_bucket(const or_config *cfg, int worker, uint64_t step, int64_t base,
                              const float *u, int n, uint8_t *code, float *q, float *table,
                              float *blo, float *bhi, float *bp)
{
    or_gridinfo gi;
    if (!grid_setup(u, n, OR_PB_FBITS, &gi)) {
        table[0] = gi.mn;
        table[1] = gi.mn;
        for (int i = 0; i < n; ++i) {
            code[i] = 0;
            q[i] = gi.mn;
            if (bp) {
                blo[i] = gi.mn;
                bhi[i] = gi.mn;
                bp[i] = 0.0f;
            }
        }
        return;
    }
    int32_t *pos = (int32_t *)malloc(sizeof(int32_t) * (size_t)n);
    for (int i = 0; i < n; ++i) pos[i] = grid_pos(&gi, u[i], OR_PB_FBITS);
    int A, B, Amax, Bmin;
    pb_limits(&gi, u, n, &Amax, &Bmin);
    pb_select_pos(pos, n, Amax, Bmin, &A, &B);
    float a = gi.grid[A], b = gi.grid[B];
    table[0] = a;
    table[1] = b;
    float rinv = 1.0f / (b - a);
    int32_t pa = (int32_t)A << OR_PB_FBITS, pbv = (int32_t)B << OR_PB_FBITS;
    for (int i = 0; i < n; ++i) {
        int c;
        float p;
        if (pos[i] < pa) {
            c = 0;
            p = 0.0f;
        } else if (pos[i] >= pbv) {
            c = 1;
            p = 1.0f;
        } else {
            p = sat01((u[i] - a) * rinv);
            float U = or_uniform(cfg->seed, step, (uint32_t)worker, base + i);
            c = U < p ? 1 : 0;
        }
        code[i] = (uint8_t)c;
        q[i] = c ? b : a;
        if (bp) {
            blo[i] = a;
            bhi[i] = b;
            bp[i] = p;
        }
    }
    free(pos);
}

/* ------------------------------------------------------------------------------------------ */
/* Sizes and message layout.                                                                   */
/* ------------------------------------------------------------------------------------------ */
int or_bits(int levels)
{
    int b = 0;
    while ((1 << b) < levels) ++b;
    return b;
}

int or_table_len(int scheme, int levels)
{
    if (scheme == OR_QSGD || scheme == OR_TERNGRAD || scheme == OR_QSGD_NEAREST || scheme == OR_QSGD_L2) return 1;
    if (scheme == OR_BINGRAD_B || scheme == OR_BINGRAD_PB || scheme == OR_SIGNSGD) return 2;
    return levels;
}

int64_t or_num_buckets(const or_config *cfg)
{
    return (cfg->n + cfg->bucket - 1) / cfg->bucket;
}

/*
 * A worker's message: the packed codes of every bucket, bucket after bucket (d*b/32 words
 * each), then the level tables, bucket after bucket (L floats each), the second region
 * starting on a 16-byte boundary and the total rounded up to 16 bytes.
 */
void or_message_layout(const or_config *cfg, int64_t *bytes, int64_t *codes_off, int64_t *levels_off)
{
    int64_t nb = or_num_buckets(cfg);
    int64_t words = (int64_t)cfg->bucket * or_bits(cfg->levels) / 32;
    int64_t cbytes = nb * words * 4;
    int64_t lbytes = nb * or_table_len(cfg->scheme, cfg->levels) * 4;
    cbytes = (cbytes + 15) / 16 * 16;
    lbytes = (lbytes + 15) / 16 * 16;
    *codes_off = 0;
    *levels_off = cbytes;
    *bytes = cbytes + lbytes;
}

/*
 * Dense packing of one bucket (b bits per code): the code of element e occupies bits
 * b*e .. b*e + b - 1 of the bucket's d*b/32 words, read as one little-endian bit string (bit k
 * is bit k % 32 of word k / 32).  Codes of padding elements (e >= n) are 0.
 */
void or_pack_bucket(const or_config *cfg, const uint8_t *code, int n, uint32_t *words)
{
    int b = or_bits(cfg->levels);
    int d = cfg->bucket;
    memset(words, 0, sizeof(uint32_t) * (size_t)(d * b / 32));
    for (int e = 0; e < n; ++e)
        for (int j = 0; j < b; ++j) {
            int64_t k = (int64_t)b * e + j;
            if ((code[e] >> j) & 1) words[k / 32] |= 1u << (k % 32);
        }
}

void or_unpack_bucket(const or_config *cfg, const uint32_t *words, int n, uint8_t *code)
{
    int b = or_bits(cfg->levels);
    for (int e = 0; e < n; ++e) {
        int v = 0;
        for (int j = 0; j < b; ++j) {
            int64_t k = (int64_t)b * e + j;
            v |= (int)((words[k / 32] >> (k % 32)) & 1u) << j;
        }
        code[e] = (uint8_t)v;
    }
}

float or_dequant(const or_config *cfg, const float *table, int code)
{
    if (cfg->scheme == OR_QSGD || cfg->scheme == OR_TERNGRAD || cfg->scheme == OR_QSGD_NEAREST ||
        cfg->scheme == OR_QSGD_L2)
        return table[0] * qsgd_ratio(code, cfg->levels);
    return table[code];
}

/* ------------------------------------------------------------------------------------------ */
/* One bucket of one worker.                                                                   */
/* ------------------------------------------------------------------------------------------ */
static int bucket_len(const or_config *cfg, int64_t bucket);

static int encode_bucket_ex(const or_config *cfg, int worker, uint64_t step, int64_t bucket,
                            const float *v, int n, uint8_t *code, float *q, float *table,
                            float *u_out, float *blo, float *bhi, float *bp)
{
    if (n <= 0) return 0;
    int64_t base = bucket * (int64_t)cfg->bucket;
    float *u = (float *)malloc(sizeof(float) * (size_t)n);
    memcpy(u, v, sizeof(float) * (size_t)n);
    if (cfg->clip_sigma > 0.0f) {
        float t = or_clip_threshold(v, n, cfg->clip_sigma);
        for (int i = 0; i < n; ++i) {
            if (u[i] < -t) u[i] = -t;
            if (u[i] > t) u[i] = t;
        }
    }
    switch (cfg->scheme) {
    case OR_QSGD:
    case OR_TERNGRAD:
        qsgd_bucket(cfg, worker, step, base, u, n, code, q, table, blo, bhi, bp, 0);
        break;
    case OR_QSGD_NEAREST:
        qsgd_bucket(cfg, worker, step, base, u, n, code, q, table, blo, bhi, bp, 1);
        break;
    case OR_QSGD_L2:
        qsgd_bucket(cfg, worker, step, base, u, n, code, q, table, blo, bhi, bp, 0);
        break;
    case OR_SIGNSGD:
        sign_bucket(u, n, code, q, table, blo, bhi, bp);
        break;
    case OR_BINGRAD_B:
        bingrad_b_bucket(u, n, code, q, table, blo, bhi, bp);
        break;
    case OR_BINGRAD_PB:
        bingrad_pb_bucket(cfg, worker, step, base, u, n, code, q, table, blo, bhi, bp);
        break;
    case OR_ORQ:
        orq_bucket(cfg, worker, step, base, u, n, code, q, table, blo, bhi, bp);
        break;
    default:
        free(u);
        return 1;
    }
    if (u_out) memcpy(u_out, u, sizeof(float) * (size_t)n);
    free(u);
    return 0;
}

int or_encode_bucket(const or_config *cfg, int worker, uint64_t step, int64_t bucket,
                     const float *v, int n, uint8_t *code, float *q, float *table)
{
    return encode_bucket_ex(cfg, worker, step, bucket, v, n, code, q, table, NULL, NULL, NULL, NULL);
}

/*
 * Quantization error of one worker's vector over the buckets [b0, b1): out[0] = sum of the
 * expected squared rounding error p (b - u)^2 + (1 - p) (a - u)^2 of every element (u the
 * value quantized, [a, b] its bracket, p its probability of rounding up; for unbiased rounding
 * this is the variance (b - u)(u - a) that ORQ minimises), out[1] = sum of u^2, out[2] = sum of
 * the realised (Q(u) - u)^2 for this step's draws.  binary64, elements in index order.
 */
int or_quant_error(const or_config *cfg, int worker, uint64_t step, int64_t b0, int64_t b1,
                   const float *g, const float *r, double *out)
{
    int d = cfg->bucket;
    float *v = (float *)malloc(sizeof(float) * (size_t)d);
    float *u = (float *)malloc(sizeof(float) * (size_t)d);
    float *q = (float *)malloc(sizeof(float) * (size_t)d);
    float *blo = (float *)malloc(sizeof(float) * (size_t)d);
    float *bhi = (float *)malloc(sizeof(float) * (size_t)d);
    float *bp = (float *)malloc(sizeof(float) * (size_t)d);
    uint8_t *code = (uint8_t *)malloc((size_t)d);
    float table[16];
    double e = 0.0, uu = 0.0, qq = 0.0;
    int rc = 0;
    for (int64_t bk = b0; bk < b1 && rc == 0; ++bk) {
        int n = bucket_len(cfg, bk);
        int64_t base = bk * d;
        for (int i = 0; i < n; ++i) v[i] = (cfg->error_feedback && r) ? g[base + i] + r[base + i] : g[base + i];
        rc = encode_bucket_ex(cfg, worker, step, bk, v, n, code, q, table, u, blo, bhi, bp);
        for (int i = 0; i < n; ++i) {
            double P = (double)sat01(bp[i]);
            double dh = (double)bhi[i] - (double)u[i];
            double dl = (double)blo[i] - (double)u[i];
            double dq = (double)q[i] - (double)u[i];
            e += P * dh * dh + (1.0 - P) * dl * dl;
            uu += (double)u[i] * (double)u[i];
            qq += dq * dq;
        }
    }
    out[0] = e;
    out[1] = uu;
    out[2] = qq;
    free(v);
    free(u);
    free(q);
    free(blo);
    free(bhi);
    free(bp);
    free(code);
    return rc;
}

/* ------------------------------------------------------------------------------------------ */
/* Whole-vector calls.                                                                         */
/* ------------------------------------------------------------------------------------------ */
static int bucket_len(const or_config *cfg, int64_t bucket)
{
    int64_t lo = bucket * (int64_t)cfg->bucket;
    int64_t hi = lo + cfg->bucket;
    if (hi > cfg->n) hi = cfg->n;
    return (int)(hi - lo);
}

/* Error feedback ([P1] "Quantization Schemes", [P3]): quantize v = g + r, keep r' = v - Q(v). */
int or_encode(const or_config *cfg, int worker, uint64_t step, int64_t b0, int64_t b1,
              const float *g, float *r, uint8_t *msg)
{
    int d = cfg->bucket;
    int L = or_table_len(cfg->scheme, cfg->levels);
    int64_t words = (int64_t)d * or_bits(cfg->levels) / 32;
    int64_t bytes, coff, loff;
    or_message_layout(cfg, &bytes, &coff, &loff);
    float *v = (float *)malloc(sizeof(float) * (size_t)d);
    float *q = (float *)malloc(sizeof(float) * (size_t)d);
    uint8_t *code = (uint8_t *)malloc((size_t)d);
    int rc = 0;
    for (int64_t bk = b0; bk < b1 && rc == 0; ++bk) {
        int n = bucket_len(cfg, bk);
        int64_t base = bk * d;
        for (int i = 0; i < n; ++i) v[i] = (cfg->error_feedback && r) ? g[base + i] + r[base + i] : g[base + i];
        float *table = (float *)(msg + loff) + bk * L;
        rc = or_encode_bucket(cfg, worker, step, bk, v, n, code, q, table);
        if (cfg->error_feedback && r)
            for (int i = 0; i < n; ++i) r[base + i] = v[i] - q[i];
        or_pack_bucket(cfg, code, n, (uint32_t *)(msg + coff) + bk * words);
    }
    free(v);
    free(q);
    free(code);
    return rc;
}

/* Dequantize and aggregate ([P1] "How Gradient Quantization Works"): the mean over workers,
 * summed in worker order in binary32, then multiplied by 1/W. */
int or_decode_accumulate(const or_config *cfg, const uint8_t *const *msgs, int nmsgs,
                         int64_t b0, int64_t b1, float *avg)
{
    int d = cfg->bucket;
    int L = or_table_len(cfg->scheme, cfg->levels);
    int64_t words = (int64_t)d * or_bits(cfg->levels) / 32;
    int64_t bytes, coff, loff;
    or_message_layout(cfg, &bytes, &coff, &loff);
    float inv_w = 1.0f / (float)nmsgs;
    uint8_t *code = (uint8_t *)malloc((size_t)d);
    float *acc = (float *)malloc(sizeof(float) * (size_t)d);
    for (int64_t bk = b0; bk < b1; ++bk) {
        int n = bucket_len(cfg, bk);
        for (int i = 0; i < n; ++i) acc[i] = 0.0f;
        for (int w = 0; w < nmsgs; ++w) {
            const uint32_t *cw = (const uint32_t *)(msgs[w] + coff) + bk * words;
            const float *table = (const float *)(msgs[w] + loff) + bk * L;
            or_unpack_bucket(cfg, cw, n, code);
            for (int i = 0; i < n; ++i) acc[i] = acc[i] + or_dequant(cfg, table, code[i]);
        }
        for (int i = 0; i < n; ++i) avg[bk * d + i] = acc[i] * inv_w;
    }
    free(code);
    free(acc);
    return 0;
}

/* One bucket of the whole step.  g[w] / r_in[w] hold the n values of bucket `bucket` of
 * worker w (r_in NULL when error feedback is off).  Outputs (each may be NULL): r_out[w] the new
 * residuals, words[w] the packed codes (d*b/32 words), tables[w] the level table (L floats),
 * avg the n averaged values. */
int or_fused_bucket(const or_config *cfg, uint64_t step, int64_t bucket, int n,
                    const float *const *g, const float *const *r_in, float *const *r_out,
                    uint32_t *const *words, float *const *tables, float *avg)
{
    int W = cfg->workers;
    float inv_w = 1.0f / (float)W;
    float *v = (float *)malloc(sizeof(float) * (size_t)(n > 0 ? n : 1));
    float *q = (float *)malloc(sizeof(float) * (size_t)(n > 0 ? n : 1));
    float *acc = (float *)malloc(sizeof(float) * (size_t)(n > 0 ? n : 1));
    uint8_t *code = (uint8_t *)malloc((size_t)(n > 0 ? n : 1));
    float table[16];
    int rc = 0;
    for (int i = 0; i < n; ++i) acc[i] = 0.0f;
    for (int w = 0; w < W && rc == 0; ++w) {
        int ef = cfg->error_feedback && r_in && r_in[w];
        for (int i = 0; i < n; ++i) v[i] = ef ? g[w][i] + r_in[w][i] : g[w][i];
        rc = or_encode_bucket(cfg, w, step, bucket, v, n, code, q, table);
        if (ef && r_out && r_out[w])
            for (int i = 0; i < n; ++i) r_out[w][i] = v[i] - q[i];
        if (words && words[w]) or_pack_bucket(cfg, code, n, words[w]);
        if (tables && tables[w])
            memcpy(tables[w], table, sizeof(float) * (size_t)or_table_len(cfg->scheme, cfg->levels));
        for (int i = 0; i < n; ++i) acc[i] = acc[i] + q[i];
    }
    if (avg)
        for (int i = 0; i < n; ++i) avg[i] = acc[i] * inv_w;
    free(v);
    free(q);
    free(acc);
    free(code);
    return rc;
}

/* The whole step for W workers over the bucket range [b0, b1): every worker quantized
 * (messages optional), the dequantized values averaged in worker order. */
int or_fused_step(const or_config *cfg, uint64_t step, int64_t b0, int64_t b1,
                  const float *const *g, float *const *r, uint8_t *const *msgs, float *avg)
{
    int d = cfg->bucket;
    int W = cfg->workers;
    int L = or_table_len(cfg->scheme, cfg->levels);
    int64_t words = (int64_t)d * or_bits(cfg->levels) / 32;
    int64_t bytes, coff, loff;
    or_message_layout(cfg, &bytes, &coff, &loff);
    const float *gb[64];
    const float *rb[64];
    float *ro[64];
    uint32_t *wb[64];
    float *tb[64];
    int ef = cfg->error_feedback && r;
    int rc = 0;
    for (int64_t bk = b0; bk < b1 && rc == 0; ++bk) {
        int n = bucket_len(cfg, bk);
        int64_t base = bk * d;
        for (int w = 0; w < W; ++w) {
            gb[w] = g[w] + base;
            rb[w] = ef ? r[w] + base : NULL;
            ro[w] = ef ? r[w] + base : NULL;
            wb[w] = (msgs && msgs[w]) ? (uint32_t *)(msgs[w] + coff) + bk * words : NULL;
            tb[w] = (msgs && msgs[w]) ? (float *)(msgs[w] + loff) + bk * L : NULL;
        }
        rc = or_fused_bucket(cfg, step, bk, n, gb, ef ? rb : NULL, ef ? ro : NULL, wb, tb, avg + base);
    }
    return rc;
}

/* ------------------------------------------------------------------------------------------ */
/* Base-s packing of the codes (grouped digits).  [P2] "Key findings" quotes compression     */
/* ratios of 20.2 (3 levels) and 10.1 (9 levels), which are 32 / log2(s): a code of s          */
/* levels carries log2(s) bits, which b = ceil(log2 s) bits waste for s = 3, 5, 9.  Reading:    */
/* g consecutive codes of a bucket form one base-s number V = sum_k code[g*i + k] * s^k (codes  */
/* past the bucket's end count as 0), stored in B bits, with s^g <= 2^B:                      */
/*   s = 3: g = 5, B = 8 (243 <= 256, 1.6 bits per code)                                      */
/*   s = 5: g = 3, B = 7 (125 <= 128, 2.33 bits per code)                                     */
/*   s = 9: g = 5, B = 16 (59049 <= 65536, 3.2 bits per code)                                 */
/* The group values follow each other in a little-endian bit string, group i at bits          */
/* B*i .. B*i + B - 1 of the bucket's ceil(ceil(d/g) * B / 32) words; the level tables are     */
/* those of the dense message, after the codes region (16-byte aligned, as there).            */
/* ------------------------------------------------------------------------------------------ */
int or_entropy_groups(int levels, int *g, int *B)
{
    switch (levels) {
    case 3: *g = 5; *B = 8; return 1;
    case 5: *g = 3; *B = 7; return 1;
    case 9: *g = 5; *B = 16; return 1;
    default: return 0;
    }
}

int64_t or_entropy_words(const or_config *cfg)
{
    int g, B;
    if (!or_entropy_groups(cfg->levels, &g, &B)) return 0;
    int64_t groups = (cfg->bucket + g - 1) / g;
    return (groups * B + 31) / 32;
}

void or_entropy_layout(const or_config *cfg, int64_t *bytes, int64_t *codes_off, int64_t *levels_off)
{
    int64_t nb = or_num_buckets(cfg);
    int64_t cbytes = nb * or_entropy_words(cfg) * 4;
    int64_t lbytes = nb * or_table_len(cfg->scheme, cfg->levels) * 4;
    cbytes = (cbytes + 15) / 16 * 16;
    lbytes = (lbytes + 15) / 16 * 16;
    *codes_off = 0;
    *levels_off = cbytes;
    *bytes = cbytes + lbytes;
}

/* Dense message -> base-s message (same buckets, same level tables). */
void or_entropy_pack(const or_config *cfg, const uint8_t *msg, uint8_t *emsg)
{
    int g, B;
    if (!or_entropy_groups(cfg->levels, &g, &B)) return;
    int d = cfg->bucket, s = cfg->levels;
    int64_t nb = or_num_buckets(cfg), dw = (int64_t)d * or_bits(s) / 32, ew = or_entropy_words(cfg);
    int64_t bytes, coff, loff, ebytes, ecoff, eloff;
    or_message_layout(cfg, &bytes, &coff, &loff);
    or_entropy_layout(cfg, &ebytes, &ecoff, &eloff);
    memset(emsg, 0, (size_t)ebytes);
    uint8_t *code = (uint8_t *)malloc((size_t)d);
    for (int64_t bk = 0; bk < nb; ++bk) {
        or_unpack_bucket(cfg, (const uint32_t *)(msg + coff) + bk * dw, d, code);
        uint32_t *out = (uint32_t *)(emsg + ecoff) + bk * ew;
        for (int64_t i = 0; g * i < d; ++i) {
            uint32_t v = 0;
            for (int k = g - 1; k >= 0; --k) {
                int64_t e = g * i + k;
                v = v * (uint32_t)s + (e < d ? code[e] : 0u);
            }
            for (int j = 0; j < B; ++j) {
                int64_t bit = B * i + j;
                if ((v >> j) & 1u) out[bit / 32] |= 1u << (bit % 32);
            }
        }
    }
    free(code);
    memcpy(emsg + eloff, msg + loff, (size_t)(nb * or_table_len(cfg->scheme, s) * 4));
}

/* Base-s message -> dense message. */
void or_entropy_unpack(const or_config *cfg, const uint8_t *emsg, uint8_t *msg)
{
    int g, B;
    if (!or_entropy_groups(cfg->levels, &g, &B)) return;
    int d = cfg->bucket, s = cfg->levels;
    int64_t nb = or_num_buckets(cfg), dw = (int64_t)d * or_bits(s) / 32, ew = or_entropy_words(cfg);
    int64_t bytes, coff, loff, ebytes, ecoff, eloff;
    or_message_layout(cfg, &bytes, &coff, &loff);
    or_entropy_layout(cfg, &ebytes, &ecoff, &eloff);
    memset(msg, 0, (size_t)bytes);
    uint8_t *code = (uint8_t *)malloc((size_t)d);
    for (int64_t bk = 0; bk < nb; ++bk) {
        const uint32_t *in = (const uint32_t *)(emsg + ecoff) + bk * ew;
        for (int64_t i = 0; g * i < d; ++i) {
            uint32_t v = 0;
            for (int j = 0; j < B; ++j) {
                int64_t bit = B * i + j;
                v |= ((in[bit / 32] >> (bit % 32)) & 1u) << j;
            }
            for (int k = 0; k < g; ++k) {
                int64_t e = g * i + k;
                if (e < d) code[e] = (uint8_t)(v % (uint32_t)s);
                v /= (uint32_t)s;
            }
        }
        or_pack_bucket(cfg, code, d, (uint32_t *)(msg + coff) + bk * dw);
    }
    free(code);
    memcpy(msg + loff, emsg + eloff, (size_t)(nb * or_table_len(cfg->scheme, s) * 4));
}

static float or_l2_scale_fwd(const float *u, int n) { return or_l2_scale(u, n); }

/* ------------------------------------------------------------------------------------------ */
/* Elias integer coding.  [P3] "QSGD": the quantized values are encoded with Elias integer     */
/* coding for further lossless compression.  Elias gamma (P. Elias, "Universal codeword sets   */
/* and representations of the integers", IEEE Trans. Inf. Theory 21(2), 1975): an integer     */
/* x >= 1 with N = floor(log2 x) is written as N zero bits followed by the N + 1 bits of x,    */
/* most significant first.  Reading, for the QSGD family with an odd number of levels s (a    */
/* zero level, z0 = (s-1)/2): code c becomes the signed level z = c - z0, zigzag-mapped to     */
/* x = 2z + 1 (z >= 0) or -2z (z < 0), so that the zero level costs one bit.                   */
/* Message: [8 bytes: T, the stream's bit count][8 zero bytes][ceil(n/d) uint64: the first     */
/* stream bit of each bucket, padded to 16 bytes][the level tables, as in the dense message,   */
/* padded to 16 bytes][the stream: the valid codes of every bucket in element order, bit k of  */
/* the stream is bit k % 32 of word k / 32, the bits after T zero, padded to 16 bytes].        */
/* ------------------------------------------------------------------------------------------ */
int or_elias_gamma_len(uint32_t x)
{
    int N = 0;
    while ((x >> (N + 1)) != 0u) ++N;
    return 2 * N + 1;
}

static int elias_supported(const or_config *cfg)
{
    int s = cfg->levels;
    int qs = cfg->scheme == OR_QSGD || cfg->scheme == OR_TERNGRAD || cfg->scheme == OR_QSGD_NEAREST ||
             cfg->scheme == OR_QSGD_L2;
    return qs && (s % 2) == 1;
}

static uint32_t elias_symbol(int code, int s)
{
    int z = code - (s - 1) / 2;
    return z >= 0 ? (uint32_t)(2 * z + 1) : (uint32_t)(-2 * z);
}

static int elias_code(uint32_t x, int s)
{
    int z = (x & 1u) ? (int)((x - 1u) / 2u) : -(int)(x / 2u);
    return z + (s - 1) / 2;
}

int or_elias_layout(const or_config *cfg, int64_t *cap_bytes, int64_t *offsets_off, int64_t *tables_off,
                    int64_t *stream_off)
{
    if (!elias_supported(cfg)) return 0;
    int s = cfg->levels;
    int64_t nb = or_num_buckets(cfg);
    int L = or_table_len(cfg->scheme, s);
    int maxbits = or_elias_gamma_len((uint32_t)s);   /* the largest symbol is s (z = z0) */
    int64_t obytes = (nb * 8 + 15) / 16 * 16;
    int64_t tbytes = (nb * L * 4 + 15) / 16 * 16;
    int64_t sbytes = ((cfg->n * maxbits + 31) / 32 * 4 + 15) / 16 * 16;
    *offsets_off = 16;
    *tables_off = 16 + obytes;
    *stream_off = 16 + obytes + tbytes;
    *cap_bytes = *stream_off + sbytes;
    return 1;
}

int64_t or_elias_pack(const or_config *cfg, const uint8_t *msg, uint8_t *emsg)
{
    int64_t cap, ooff, toff, soff;
    if (!or_elias_layout(cfg, &cap, &ooff, &toff, &soff)) return -1;
    int s = cfg->levels, d = cfg->bucket;
    int64_t nb = or_num_buckets(cfg), dw = (int64_t)d * or_bits(s) / 32;
    int L = or_table_len(cfg->scheme, s);
    int64_t bytes, coff, loff;
    or_message_layout(cfg, &bytes, &coff, &loff);
    memset(emsg, 0, (size_t)cap);
    uint64_t *offs = (uint64_t *)(emsg + ooff);
    uint32_t *stream = (uint32_t *)(emsg + soff);
    uint8_t *code = (uint8_t *)malloc((size_t)d);
    uint64_t k = 0;
    for (int64_t bk = 0; bk < nb; ++bk) {
        int n = bucket_len(cfg, bk);
        offs[bk] = k;
        or_unpack_bucket(cfg, (const uint32_t *)(msg + coff) + bk * dw, n, code);
        for (int e = 0; e < n; ++e) {
            uint32_t x = elias_symbol(code[e], s);
            int len = or_elias_gamma_len(x), N = len / 2;
            k += (uint64_t)N;                                  /* N zeros */
            for (int j = N; j >= 0; --j, ++k)                  /* x, most significant bit first */
                if ((x >> j) & 1u) stream[k / 32] |= 1u << (k % 32);
        }
    }
    free(code);
    memcpy(emsg, &k, sizeof k);
    memcpy(emsg + toff, msg + loff, (size_t)(nb * L * 4));
    return soff + ((int64_t)(k + 31) / 32 * 4 + 15) / 16 * 16;
}

int or_elias_unpack(const or_config *cfg, const uint8_t *emsg, uint8_t *msg)
{
    int64_t cap, ooff, toff, soff;
    if (!or_elias_layout(cfg, &cap, &ooff, &toff, &soff)) return 0;
    int s = cfg->levels, d = cfg->bucket;
    int64_t nb = or_num_buckets(cfg), dw = (int64_t)d * or_bits(s) / 32;
    int L = or_table_len(cfg->scheme, s);
    int64_t bytes, coff, loff;
    or_message_layout(cfg, &bytes, &coff, &loff);
    memset(msg, 0, (size_t)bytes);
    const uint64_t *offs = (const uint64_t *)(emsg + ooff);
    const uint32_t *stream = (const uint32_t *)(emsg + soff);
    uint8_t *code = (uint8_t *)malloc((size_t)d);
    for (int64_t bk = 0; bk < nb; ++bk) {
        int n = bucket_len(cfg, bk);
        uint64_t k = offs[bk];
        for (int e = 0; e < n; ++e) {
            int N = 0;
            while (N < 31 && ((stream[k / 32] >> (k % 32)) & 1u) == 0u) { ++N; ++k; }
            uint32_t x = 0;
            for (int j = 0; j <= N; ++j, ++k) x = (x << 1) | ((stream[k / 32] >> (k % 32)) & 1u);
            code[e] = (uint8_t)elias_code(x, s);
        }
        or_pack_bucket(cfg, code, n, (uint32_t *)(msg + coff) + bk * dw);
    }
    free(code);
    memcpy(msg + loff, emsg + toff, (size_t)(nb * L * 4));
    return 1;
}

/* ------------------------------------------------------------------------------------------ */
/* TernGrad with one scale per parameter tensor.  [P3] "Ternary and binary quantization":     */
/* TernGrad sends three levels {-m, 0, +m} with a single scaling factor per layer.  The        */
/* gradient is the concatenation of nseg tensors; tensor t holds elements [off[t], off[t+1]).  */
/* Reading: m_t = max |v| over the tensor's elements (v = g + r with error feedback, no clip);  */
/* element i of tensor t is rounded between the two of {-m_t, 0, +m_t} around it exactly as    */
/* TernGrad per bucket does (position y = (v / m_t + 1), bracket k = trunc(y) clamped to       */
/* [0, 1], up with probability y - k against the element's Philox draw).  The message holds    */
/* the 2-bit codes in the bucket layout of the dense message (bucket size d), then the nseg    */
/* scales (float); both regions start on 16-byte boundaries.                                   */
/* ------------------------------------------------------------------------------------------ */
void or_tg_layer_layout(const or_config *cfg, int nseg, int64_t *bytes, int64_t *codes_off, int64_t *scales_off)
{
    int64_t nb = or_num_buckets(cfg);
    int64_t cbytes = (nb * (int64_t)cfg->bucket * 2 / 32 * 4 + 15) / 16 * 16;
    int64_t sbytes = ((int64_t)nseg * 4 + 15) / 16 * 16;
    *codes_off = 0;
    *scales_off = cbytes;
    *bytes = cbytes + sbytes;
}

static int tg_segment_of(const int64_t *off, int nseg, int64_t i)
{
    int t = 0;
    while (t + 1 < nseg && off[t + 1] <= i) ++t;
    return t;
}

int or_tg_layer_encode(const or_config *cfg, const int64_t *off, int nseg, int worker, uint64_t step,
                       const float *g, float *r, uint8_t *msg)
{
    int64_t n = cfg->n, bytes, coff, soff;
    int d = cfg->bucket;
    if (nseg < 1 || off[0] != 0 || off[nseg] != n) return 1;
    or_tg_layer_layout(cfg, nseg, &bytes, &coff, &soff);
    memset(msg, 0, (size_t)bytes);
    float *v = (float *)malloc(sizeof(float) * (size_t)(n > 0 ? n : 1));
    for (int64_t i = 0; i < n; ++i) v[i] = (cfg->error_feedback && r) ? g[i] + r[i] : g[i];
    float *scales = (float *)(msg + soff);
    for (int t = 0; t < nseg; ++t) {
        float m = 0.0f;
        for (int64_t i = off[t]; i < off[t + 1]; ++i) {
            float a = fabsf(v[i]);
            if (a > m) m = a;
        }
        scales[t] = m;
    }
    or_config c3 = *cfg;
    c3.levels = 3;
    int64_t nb = or_num_buckets(cfg);
    int64_t words = (int64_t)d * 2 / 32;
    uint8_t *code = (uint8_t *)malloc((size_t)d);
    for (int64_t bk = 0; bk < nb; ++bk) {
        int64_t base = bk * d;
        int nv = (int)((n - base) < d ? (n - base) : d);
        for (int e = 0; e < nv; ++e) {
            int64_t i = base + e;
            float m = scales[tg_segment_of(off, nseg, i)];
            float inv_m = m > 0.0f ? 1.0f / m : 0.0f;
            float y = (v[i] * inv_m + 1.0f) * 1.0f;  /* h = (s - 1) / 2 = 1 */
            int k = 0;
            if (y > 0.0f) k = (y >= 1.0f) ? 1 : (int)y;
            float p = y - (float)k;
            float U = or_uniform(cfg->seed, step, (uint32_t)worker, i);
            int c = k + (U < p ? 1 : 0);
            code[e] = (uint8_t)c;
            float q = m * qsgd_ratio(c, 3);
            if (cfg->error_feedback && r) r[i] = v[i] - q;
        }
        or_pack_bucket(&c3, code, nv, (uint32_t *)(msg + coff) + bk * words);
    }
    free(code);
    free(v);
    return 0;
}

int or_tg_layer_decode_accumulate(const or_config *cfg, const int64_t *off, int nseg, const uint8_t *const *msgs,
                                  int nmsgs, float *avg)
{
    int64_t n = cfg->n, bytes, coff, soff;
    int d = cfg->bucket;
    or_tg_layer_layout(cfg, nseg, &bytes, &coff, &soff);
    or_config c3 = *cfg;
    c3.levels = 3;
    int64_t nb = or_num_buckets(cfg);
    int64_t words = (int64_t)d * 2 / 32;
    float inv_w = 1.0f / (float)nmsgs;
    uint8_t *code = (uint8_t *)malloc((size_t)d);
    float *acc = (float *)malloc(sizeof(float) * (size_t)d);
    for (int64_t bk = 0; bk < nb; ++bk) {
        int64_t base = bk * d;
        int nv = (int)((n - base) < d ? (n - base) : d);
        for (int e = 0; e < nv; ++e) acc[e] = 0.0f;
        for (int w = 0; w < nmsgs; ++w) {
            const float *scales = (const float *)(msgs[w] + soff);
            or_unpack_bucket(&c3, (const uint32_t *)(msgs[w] + coff) + bk * words, nv, code);
            for (int e = 0; e < nv; ++e)
                acc[e] = acc[e] + scales[tg_segment_of(off, nseg, base + e)] * qsgd_ratio(code[e], 3);
        }
        for (int e = 0; e < nv; ++e) avg[base + e] = acc[e] * inv_w;
    }
    free(code);
    free(acc);
    return 0;
}
