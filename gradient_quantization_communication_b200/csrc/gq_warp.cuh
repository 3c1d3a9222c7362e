// gq_warp.cuh -- register-resident quantization kernels for buckets of d = 128, 256, 512.
//
// Included by one translation unit per scheme (gq_warp_*.cu), which instantiates warp_dispatch
// for that scheme only, so that the instantiations compile in parallel.
//
// One warp owns one bucket index at a time and walks its items (bucket, worker) in order.  The
// g and r of each item (2 x d floats) are staged into the warp's shared memory by bulk
// asynchronous copies (TMA, 1-D, into this CTA only) completed on an mbarrier: as soon as an item's
// values are in registers the copy of the next item is issued into the same buffer, so the
// copy engine keeps 4 KB per warp in flight during the whole fit and no registers are spent on
// prefetching.  Lane l then holds EPL = d/32 values in registers, slot
// t being element 128*(t/4) + 4*l + t%4 of the bucket, so that the four values of a slot
// group share one Philox call and every global store is a coalesced 16-byte access.  In the
// fused step the W workers of a bucket are consecutive items: the dequantized values are
// summed in registers in worker order and the average leaves the chip once.
//
// Level fits per bucket:
//   QSGD / TernGrad : m = max|u|, s uniform levels on [-m, m]
//   ORQ             : shared-memory histogram of grid positions with 16 fraction bits (8
//                     columns per cell, one packed shared atomic per value), exact prefix
//                     sums, s-2 incremental greedy rounds, per-bracket reciprocal table
//   BinGrad-b       : warp bitonic sort, exact int64 prefix sums, screened argmax of J(k)
//   BinGrad-pb      : BinGrad-b's levels (as above) bound the pair from inside; the cells'
//                     prefix moments of 16-bit positions read off the sorted values; per
//                     column the least E over the admissible A (E is convex in A)
//   QSGD-nearest    : the QSGD levels, rounding to the nearest level (no draws)
//   QSGD-l2         : the QSGD levels scaled by ||u||_2 (exact fixed-point sum of squares)
//   SignSGD         : m1 = mean |u| from an exact fixed-point warp sum, levels -m1 and +m1
// The last bucket, when ragged, is handled by a one-warp launch of the same code with guarded
// plain loads, so the main kernel carries no tail logic.
#pragma once

#include "gq_bases.cuh"
#include "gq_round.cuh"

namespace gq {
namespace {

constexpr int kWarpsPerCta = 4;
constexpr int kHistCols = 8;
// Items staged ahead per warp (bulk-copy buffers of 2 x d floats each).
#ifndef GQ_WARP_STAGES
#define GQ_WARP_STAGES 1
#endif
constexpr int kStages = GQ_WARP_STAGES;

template <int EPL>
struct alignas(16) StageBuf {
    float g[32 * EPL];
    float r[32 * EPL];
};

// ORQ histogram word of one (cell, column): count << kHistCountShift | sum of 16-bit fractions.
// A column collects at most 4 lanes x 16 values = 64 entries, so the fraction sum stays below
// 64 * 2^16 = 2^22 and the count (<= 64) fits above it.
constexpr int kHistCountShift = 22;
// Base-s messages: the bucket's codes as bytes (512 bytes and 32 bytes of zeros past them for
// the last group's missing codes), then the word buffer of its base-s words (at most 52).
constexpr int kCodeBytesWords = 512 / 4 + 8;
constexpr int kBaseOutWords = 56;
struct alignas(16) FitORQ {
    uint32_t hist[64 * kHistCols];  // [cell][column]; cell 63 holds the values at the top grid point
    float4 ctab[64];                // cell -> {lower, upper, 1/(upper-lower), bracket}; 63 repeats 62
    float4 btab[GQ_MAX_LEVELS];     // bracket k -> {level k, level k+1, 1/difference, k}
    float lev[GQ_MAX_LEVELS];       // chosen levels in increasing order
    uint32_t P1[64];                // sum of positions over cells < k (< 2^31 for d <= 512)
    int P0[64];                     // count over cells < k
    uint32_t codes[kCodeBytesWords + kBaseOutWords];  // base-s messages: codes as bytes, output words
};
struct alignas(16) FitQSGD {
    float2 pair[GQ_MAX_QSGD_LEVELS];  // {level k, level k+1}
    float qr[GQ_MAX_QSGD_LEVELS];     // the level ratios (2k - (s-1)) / (s-1), copied once
    uint32_t codes[kCodeBytesWords + kBaseOutWords];  // base-s messages: codes as bytes, output words
};
struct alignas(16) FitPB {
    unsigned long long q2[64];  // at a cell's first value in sorted order: sum of squared positions before it
    unsigned int q1[64];        // ... sum of positions before it (< 2^31 for d <= 512)
    int q0[64];                 // ... 1 + count before it; 0 for an empty cell
    long long al[64], be[64];   // per-index terms of E(A, B)
    unsigned long long ga16[64], de16[64];  // ... pre-multiplied by 2^16
};

struct alignas(16) FitB {
    int unused;
};

template <int S> struct FitFor { using type = FitQSGD; };
template <> struct FitFor<GQ_ORQ> { using type = FitORQ; };
template <> struct FitFor<GQ_BINGRAD_PB> { using type = FitPB; };
template <> struct FitFor<GQ_BINGRAD_B> { using type = FitB; };

template <int EPL, int SCHEME>
struct alignas(16) WarpSmem {
    StageBuf<EPL> stage[kStages];
    unsigned long long bar[kStages];
    typename FitFor<SCHEME>::type fit;
};

__device__ __forceinline__ int slot_elem(int t, int lane) { return 128 * (t >> 2) + 4 * lane + (t & 3); }

// ---------------------------------------------------------------------------------------------
// Round + pack + residual + accumulate for one worker-bucket, chunk by chunk.
// ---------------------------------------------------------------------------------------------
// BITS < 0 selects the error mode of gq_quant_error: nothing is written, the error terms of
// the bucket's elements are added to *ea.
// IO >> 2 = s selects base-s messages: the codes go to `codes` (the warp's shared bytes) chunk by
// chunk and the bucket's base-s words are built from them after the last chunk.
template <int EPL, bool FUSED, bool RANDOM, bool TAIL, int BITS, int IO = 0, class R>
__device__ __forceinline__ void emit(const KParams &p, const R &rule, int64_t beta, int w, int lane, uint32_t vmask,
                                     const float (&v)[EPL], const float (&u)[EPL], const int (&pos)[EPL],
                                     float (&acc)[EPL], ErrAcc *ea = nullptr, uint32_t *codes = nullptr)
{
    const int64_t base = beta * (int64_t)(32 * EPL);
    if constexpr (BITS < 0) {
        const uint32_t worker = p.worker0 + (uint32_t)w;
#pragma unroll
        for (int m = 0; m < EPL / 4; ++m) {
            const float uu[4] = {u[4 * m], u[4 * m + 1], u[4 * m + 2], u[4 * m + 3]};
            const int pp[4] = {pos[4 * m], pos[4 * m + 1], pos[4 * m + 2], pos[4 * m + 3]};
            const uint32_t valid = TAIL ? (vmask >> (4 * m)) & 0xfu : 0xfu;
            err_chunk<RANDOM, !TAIL>(p, rule, (uint64_t)(base >> 2) + (uint64_t)(32 * m), worker, lane, valid, uu, pp,
                                     *ea);
        }
        return;
    }
    constexpr bool kHasR = (IO & 1) != 0, kHasMsg = (IO & 2) != 0;
    constexpr int kBaseS = IO >> 2;
    constexpr int kCodeWords = kBaseS ? 32 : 4 * (BITS > 0 ? BITS : 0);  // words per chunk when known
    float *r = p.r[w];
    unsigned char *msg = p.msg[w];
    uint32_t *out = (kHasMsg || msg) ? reinterpret_cast<uint32_t *>(msg) + beta * p.codes_words : nullptr;
    uint32_t *cw = kBaseS ? ((kHasMsg || msg) ? codes : nullptr) : out;
    const uint32_t worker = p.worker0 + (uint32_t)w;
#pragma unroll
    for (int m = 0; m < EPL / 4; ++m) {
        const float vv[4] = {v[4 * m], v[4 * m + 1], v[4 * m + 2], v[4 * m + 3]};
        const float uu[4] = {u[4 * m], u[4 * m + 1], u[4 * m + 2], u[4 * m + 3]};
        const int pp[4] = {pos[4 * m], pos[4 * m + 1], pos[4 * m + 2], pos[4 * m + 3]};
        const uint32_t valid = TAIL ? (vmask >> (4 * m)) & 0xfu : 0xfu;
        float q[4];
        round_chunk<RANDOM, !TAIL, BITS, IO>(p, rule, (uint64_t)(base >> 2) + (uint64_t)(32 * m), worker, lane, valid,
                                             vv, uu, pp, (kHasR || r) ? r + base + 128 * m : nullptr,
                                             (kHasMsg || cw) ? cw + m * (kCodeWords ? kCodeWords : 4 * p.bits) : nullptr, q);
        if (FUSED) {
#pragma unroll
            for (int c = 0; c < 4; ++c)
                if (!TAIL || ((valid >> c) & 1u)) acc[4 * m + c] = __fadd_rn(acc[4 * m + c], q[c]);
        }
    }
    if constexpr (kBaseS != 0) {
        if (kHasMsg || out) {
            __syncwarp();
            base_s_store<kBaseS, 32 * EPL>(codes, codes + kCodeBytesWords, out, (int)p.codes_words, lane);
        }
    }
}

// Level table of the message (L floats per bucket).
__device__ __forceinline__ void store_table(const KParams &p, int w, int64_t beta, int lane, float value)
{
    unsigned char *msg = p.msg[w];
    if (msg && lane < p.L) reinterpret_cast<float *>(msg + p.levels_off)[beta * p.L + lane] = value;
}

__device__ __forceinline__ void flag_nonfinite(const KParams &p, int lane)
{
    if (lane == 0) atomicOr(p.status, kStatusNonFinite);
}

// ORQ tables from the chosen grid indices (mask, s bits): the level table of the message, the
// bracket table (one entry per pair of adjacent levels) and the per-cell bracket table the
// rounding pass reads (cell j lies in bracket k = #{chosen indices <= j} - 1; cell 63, the top
// grid point, in bracket s - 2 like cell 62).  IO bit 1: the message buffer is known present.
template <int IO>
__device__ __forceinline__ void build_orq_tables(const KParams &p, FitORQ &sm, int w, int64_t beta, int lane,
                                                 unsigned long long mask, float mn, float mx, float step)
{
    const uint32_t mlo = (uint32_t)mask, mhi = (uint32_t)(mask >> 32);
    const uint32_t lt = (1u << lane) - 1u, le = lt | (1u << lane);
    const int nlo = __popc(mlo);
    unsigned char *msg = p.msg[w];
    float *mtab = ((IO & 2) || msg) ? reinterpret_cast<float *>(msg + p.levels_off) + beta * p.L : nullptr;
    // lanes own grid indices lane and lane + 32; a chosen one stores its level at its rank
    const bool ch0 = (mlo >> lane) & 1u, ch1 = (mhi >> lane) & 1u;
    const int r0 = __popc(mlo & lt), r1 = nlo + __popc(mhi & lt);
    const float lv0 = __fadd_rn(mn, __fmul_rn((float)lane, step));
    const float lv1 = lane == 31 ? mx : __fadd_rn(mn, __fmul_rn((float)(lane + 32), step));
    if (ch0) sm.lev[r0] = lv0;
    if (ch1) sm.lev[r1] = lv1;
    if ((IO & 2) || mtab) {
        if (ch0) mtab[r0] = lv0;
        if (ch1) mtab[r1] = lv1;
    }
    __syncwarp();
    if (lane < p.s - 1) {
        const float lo = sm.lev[lane], hi = sm.lev[lane + 1];
        sm.btab[lane] = make_float4(lo, hi, __frcp_rn(__fsub_rn(hi, lo)), __int_as_float(lane));
    }
    __syncwarp();
    sm.ctab[lane] = sm.btab[__popc(mlo & le) - 1];
    sm.ctab[lane + 32] = sm.btab[min(nlo + __popc(mhi & le) - 1, p.s - 2)];
    __syncwarp();
}

// ---------------------------------------------------------------------------------------------
// Per-scheme fits (u: the values to quantize; v: the error-fed values the residual refers to)
// ---------------------------------------------------------------------------------------------
// L2: the scale is ||u||_2 instead of max|u|, from the exact int64 sum of the squares of
// round(u * 2^e), e = 20 - floor(log2 max|u|) (the clip's fixed point):
// m = fp32(sqrt(SXX) * 2^-e) in binary64.
template <int EPL, bool FUSED, bool TAIL, int BITS, int IO = 0, bool NEAREST = false, bool L2 = false>
__device__ void fit_qsgd(const KParams &p, FitQSGD &sm, int64_t beta, int w, int lane, uint32_t vmask, bool check,
                         const float (&v)[EPL], const float (&u)[EPL], float (&acc)[EPL], ErrAcc *ea = nullptr)
{
    float m = 0.0f;
#pragma unroll
    for (int t = 0; t < EPL; ++t)
        if (!TAIL || ((vmask >> t) & 1u)) m = fmax_nan(m, fabsf(u[t]));
    m = warp_redux_max_abs(m);
    if (check && !(m <= FLT_MAX)) flag_nonfinite(p, lane);
    if constexpr (L2) {
        if (m > 0.0f && m <= FLT_MAX) {
            const int e = 20 - fexpo(m);
            const double sc = pow2d(e);
            long long sxx = 0;
#pragma unroll
            for (int t = 0; t < EPL; ++t)
                if (!TAIL || ((vmask >> t) & 1u)) {
                    const long long X = fixed_point(u[t], sc);
                    sxx += X * X;
                }
            sxx = warp_sum(sxx);
            m = __double2float_rn(__dmul_rn(__dsqrt_rn(__ll2double_rn(sxx)), pow2d(-e)));
        } else if (!(m > 0.0f)) {
            m = 0.0f;  // zero bucket (NaN: unspecified, flagged)
        }
    }
    const int s = p.s;
    __syncwarp();
    for (int k = lane; k < s - 1; k += 32) sm.pair[k] = make_float2(__fmul_rn(m, sm.qr[k]), __fmul_rn(m, sm.qr[k + 1]));
    __syncwarp();
    RoundQSGDT<NEAREST> rule;
    rule.inv_m = m > 0.0f ? __frcp_rn(m) : 0.0f;
    rule.h = __fmul_rn((float)(s - 1), 0.5f);
    rule.kmax = s - 2;
    rule.pair = sm.pair;
    int pos[EPL];
#pragma unroll
    for (int t = 0; t < EPL; ++t) pos[t] = 0;
    emit<EPL, FUSED, !NEAREST, TAIL, BITS, IO>(p, rule, beta, w, lane, vmask, v, u, pos, acc, ea, sm.codes);
    store_table(p, w, beta, lane, m);
}

// Scaled sign: m1 = mean |u| of the valid elements from an exact int64 sum of
// round(|u| * 2^E), E = 45 - floor(log2 max|u|) (every term below 2^46, at most 512 of them),
// m1 = fp32((S * 2^-E) / n) in binary64; table {-m1, +m1}.
template <int EPL, bool FUSED, bool TAIL, int BITS, int IO = 0>
__device__ void fit_sign(const KParams &p, int64_t beta, int w, int lane, uint32_t vmask, bool check, int nvalid,
                         const float (&v)[EPL], const float (&u)[EPL], float (&acc)[EPL], ErrAcc *ea = nullptr)
{
    float m = 0.0f;
#pragma unroll
    for (int t = 0; t < EPL; ++t)
        if (!TAIL || ((vmask >> t) & 1u)) m = fmax_nan(m, fabsf(u[t]));
    m = warp_redux_max_abs(m);
    if (check && !(m <= FLT_MAX)) flag_nonfinite(p, lane);
    RoundSign rule;
    rule.m1 = m > 0.0f ? m : 0.0f;  // zero bucket: 0; non-finite: unspecified (flagged)
    if (m > 0.0f && m <= FLT_MAX) {
        const int E = 45 - fexpo(m);
        const double sc = pow2d(E);
        long long S = 0;
#pragma unroll
        for (int t = 0; t < EPL; ++t)
            if (!TAIL || ((vmask >> t) & 1u)) S += fixed_point(fabsf(u[t]), sc);
        S = warp_sum(S);
        rule.m1 = __double2float_rn(__ddiv_rn(__dmul_rn(__ll2double_rn(S), pow2d(-E)), (double)nvalid));
    }
    int pos[EPL];
#pragma unroll
    for (int t = 0; t < EPL; ++t) pos[t] = 0;
    emit<EPL, FUSED, false, TAIL, BITS, IO>(p, rule, beta, w, lane, vmask, v, u, pos, acc, ea);
    store_table(p, w, beta, lane, lane == 0 ? -rule.m1 : rule.m1);
}

template <int EPL, bool FUSED, bool TAIL, int BITS, int IO = 0>
__device__ void fit_orq(const KParams &p, FitORQ &sm, int64_t beta, int w, int lane, uint32_t vmask, bool check,
                        const float (&v)[EPL], const float (&u)[EPL], float (&acc)[EPL], ErrAcc *ea = nullptr)
{
    float mn = INFINITY, mx = -INFINITY;
    if (TAIL) {
#pragma unroll
        for (int t = 0; t < EPL; ++t)
            if ((vmask >> t) & 1u) {
                mn = fmin_nan(mn, u[t]);
                mx = fmax_nan(mx, u[t]);
            }
    } else {
        mn = fmin3_nan(u[0], u[1], u[2]);
        mx = fmax3_nan(u[0], u[1], u[2]);
#pragma unroll
        for (int t = 3; t < EPL; t += 2) {
            mn = t + 1 < EPL ? fmin3_nan(mn, u[t], u[t + 1]) : fmin_nan(mn, u[t]);
            mx = t + 1 < EPL ? fmax3_nan(mx, u[t], u[t + 1]) : fmax_nan(mx, u[t]);
        }
    }
    mn = warp_redux_min(mn);
    mx = warp_redux_max(mx);
    if (check && !(mn >= -FLT_MAX && mx <= FLT_MAX)) flag_nonfinite(p, lane);
    mn = __fadd_rn(mn, 0.0f);
    mx = __fadd_rn(mx, 0.0f);
    int pos[EPL];
    if (!(mx > mn)) {  // constant bucket (or NaN): one level, code 0
#pragma unroll
        for (int t = 0; t < EPL; ++t) pos[t] = 0;
        emit<EPL, FUSED, false, TAIL, BITS, IO>(p, RoundConst{mn}, beta, w, lane, vmask, v, u, pos, acc, ea, sm.codes);
        store_table(p, w, beta, lane, mn);
        return;
    }
    const float range = __fsub_rn(mx, mn);
    const float step = __fdiv_rn(range, 63.0f);
    const float scale = __fmul_rn(__fdiv_rn(63.0f, range), (float)(1 << kOrqFBits));
    // histogram: 8 columns per cell, lane l adds into column l % 8 with one shared atomic per
    // value (count and fraction packed); the rounding pass needs only the cell of each value.
    // A valid value lies in [mn, mx], so its product below is >= 0 (or NaN, which converts to
    // 0); it exceeds 63 * 2^16 only when 63 / range overflows to +inf (a range below 63 / FLT_MAX),
    // hence the upper clamp.  The cell is the position's integer part, 63 for the top grid point.
    const int col = lane & (kHistCols - 1);
#pragma unroll
    for (int t = 0; t < EPL; ++t) {
        int ps = min(__float2int_rz(__fmul_rn(__fsub_rn(u[t], mn), scale)), 63 << kOrqFBits);
        if (TAIL) ps = max(ps, 0);  // the invalid slots hold anything
        const int cell = ps >> kOrqFBits;
        pos[t] = cell;
        if (!TAIL || ((vmask >> t) & 1u))
            atomicAdd(&sm.hist[cell * kHistCols + col], (uint32_t)(ps & 0xffff) | (1u << kHistCountShift));
    }
    __syncwarp();
    // lane l reduces cells 2l and 2l+1 (16 consecutive words), clearing them; the four 16-byte
    // reads are rotated by l/2 so that a quarter-warp touches 8 distinct bank groups
    uint32_t t0 = 0, t1 = 0, c0 = 0, c1 = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int q4 = (k + (lane >> 1)) & 3;
        uint4 *ph = reinterpret_cast<uint4 *>(sm.hist + lane * 16) + q4;
        const uint4 x = *ph;
        *ph = make_uint4(0u, 0u, 0u, 0u);
        const uint32_t st = x.x + x.y + x.z + x.w;
        const uint32_t sc = (x.x >> kHistCountShift) + (x.y >> kHistCountShift) + (x.z >> kHistCountShift) +
                            (x.w >> kHistCountShift);
        if (q4 < 2) {
            t0 += st;
            c0 += sc;
        } else {
            t1 += st;
            c1 += sc;
        }
    }
    // per cell: total < 2^32 (count <= 512 at bit 22 plus fractions < 2^25), fraction sum = total
    // minus the counts' share
    const uint32_t f0 = t0 - (c0 << kHistCountShift), f1 = t1 - (c1 << kHistCountShift);
    // sums of positions of the two cells; the top grid point (cell 63) belongs to cell 62 with
    // fraction 2^16, i.e. position 63 * 2^16, which is what s1 holds for lane 31
    uint32_t s0 = c0 * ((uint32_t)(2 * lane) << kOrqFBits) + f0;
    uint32_t s1 = c1 * ((uint32_t)(2 * lane + 1) << kOrqFBits) + f1;
    if (lane == 31) {
        c0 += c1;
        s0 += s1;
        c1 = 0u;
        s1 = 0u;
    }
    // one exclusive prefix over the cell pairs of the packed (sum << 16 | count): counts stay
    // below 2^16 and sums below 2^31 for d <= 512
    const unsigned long long own = ((unsigned long long)(s0 + s1) << 16) | (c0 + c1);
    const unsigned long long ex = warp_inclusive_scan(own, lane) - own;
    const int ec = (int)(ex & 0xffffu);
    const uint32_t es = (uint32_t)(ex >> 16);
    reinterpret_cast<int2 *>(sm.P0)[lane] = make_int2(ec, ec + (int)c0);
    reinterpret_cast<uint2 *>(sm.P1)[lane] = make_uint2(es, es + s0);
    __syncwarp();
    const unsigned long long mask = orq_greedy(sm.P0, sm.P1, p.s, lane);
    build_orq_tables<IO>(p, sm, w, beta, lane, mask, mn, mx, step);
    emit<EPL, FUSED, true, TAIL, BITS, IO>(p, RoundORQ{sm.ctab}, beta, w, lane, vmask, v, u, pos, acc, ea, sm.codes);
    __syncwarp();
}

// BinGrad-b's levels of the bucket (m = max|u| over the valid values, already reduced): the
// sorted values' exact fixed-point prefix sums and the screened argmax of J; {a, b, split value,
// split found}.  Also used by BinGrad-pb, whose levels must be at least as far apart.
// The sorted values are left in key (position lane*EPL + r, the invalid ones last as +inf) when
// m > 0.
template <int EPL, bool TAIL>
__device__ __forceinline__ RoundB bingrad_b_levels(int lane, uint32_t vmask, int nvalid, float m, const float (&u)[EPL],
                                                   float (&key)[EPL])
{
    RoundB rule{0.0f, 0.0f, 0.0f, false};
    if (!(m > 0.0f)) return rule;
#pragma unroll
    for (int t = 0; t < EPL; ++t) key[t] = (!TAIL || ((vmask >> t) & 1u)) ? u[t] : INFINITY;
    warp_bitonic_sort<EPL>(key, lane);
    const int e = 46 - fexpo(m);
    // fixed point round(x * 2^e) in binary32: the scaling by 2^e (as 2^(e/2) * 2^(e - e/2),
    // both representable for e in [-81, 195]) is exact, except for products that fall below
    // 2^-126, which round to 0 either way
    const float s1 = pow2f(e >> 1), s2 = pow2f(e - (e >> 1));
    // inclusive prefix of the fixed-point values inside the lane, then across lanes
    long long pre[EPL];
    long long run = 0;
#pragma unroll
    for (int r = 0; r < EPL; ++r) {
        const int i = lane * EPL + r;
        run += (!TAIL || i < nvalid) ? __float2ll_rn(__fmul_rn(__fmul_rn(key[r], s1), s2)) : 0ll;
        pre[r] = run;
    }
    const long long incl = warp_inclusive_scan(run, lane);
    const long long lane_excl = incl - run;
    const long long total = __shfl_sync(kFull, incl, 31);
    const float prev_last = __shfl_up_sync(kFull, key[EPL - 1], 1);
    // Screening: a binary32 estimate of J for every admissible split (two conversions of
    // exact integers, two squares, two reciprocals within 1 ulp, two products and a sum:
    // within 8 * 2^-24 of J), then the fp64 J only for the splits whose estimate reaches
    // M (1 - 2^-18), M the largest estimate: every split whose fp64 J is the largest is
    // among them, so the choice (ties to the smallest split) is the exhaustive one.
    float est[EPL];
    float emax = 0.0f;
#pragma unroll
    for (int r = 0; r < EPL; ++r) {
        const int i = lane * EPL + r;  // split: positions < i on the left
        const float prev = r > 0 ? key[r - 1] : prev_last;
        est[r] = -1.0f;
        if (i >= 1 && i < nvalid && prev < key[r]) {
            const long long Sl = lane_excl + (r > 0 ? pre[r - 1] : 0ll);
            const float l = __ll2float_rn(Sl), rr = __ll2float_rn(total - Sl);
            est[r] = __fadd_rn(__fmul_rn(__fmul_rn(l, l), rcp_approx((float)i)),
                               __fmul_rn(__fmul_rn(rr, rr), rcp_approx((float)(nvalid - i))));
            emax = fmaxf(emax, est[r]);
        }
    }
    // the estimates are >= +0, so their bit patterns order like unsigned integers
    const float thr = __fmul_rn(__uint_as_float(__reduce_max_sync(kFull, __float_as_uint(emax))), 1.0f - 0x1p-18f);
    double best_j = -1.0;
    int best_i = 0x7fffffff;
#pragma unroll
    for (int r = 0; r < EPL; ++r) {
        if (est[r] >= thr) {
            const int i = lane * EPL + r;
            const long long Sl = lane_excl + (r > 0 ? pre[r - 1] : 0ll);
            const double l = __ll2double_rn(Sl);
            const double rr = __ll2double_rn(total - Sl);
            const double J = __dadd_rn(__ddiv_rn(__dmul_rn(l, l), (double)i),
                                       __ddiv_rn(__dmul_rn(rr, rr), (double)(nvalid - i)));
            if (J > best_j) {
                best_j = J;
                best_i = i;
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const double oj = __shfl_xor_sync(kFull, best_j, o);
        const int oi = __shfl_xor_sync(kFull, best_i, o);
        if (oj > best_j || (oj == best_j && oi < best_i)) {
            best_j = oj;
            best_i = oi;
        }
    }
    if (best_i == 0x7fffffff) {
        // every value equal: a single level, code 0
        const float v0 = __fadd_rn(__shfl_sync(kFull, key[0], 0), 0.0f);
        return RoundB{v0, v0, v0, false};
    }
    // owner lane publishes the threshold value and the left sum
    float tv = 0.0f;
    long long sl = 0;
#pragma unroll
    for (int r = 0; r < EPL; ++r)
        if (lane * EPL + r == best_i) {
            tv = key[r];
            sl = lane_excl + (r > 0 ? pre[r - 1] : 0ll);
        }
    const int owner = best_i / EPL;
    tv = __shfl_sync(kFull, tv, owner);
    sl = __shfl_sync(kFull, sl, owner);
    const double inv_sc = pow2d(-e);
    const float a = __double2float_rn(__dmul_rn(__ddiv_rn(__ll2double_rn(sl), (double)best_i), inv_sc));
    const float b = __double2float_rn(__dmul_rn(__ddiv_rn(__ll2double_rn(total - sl), (double)(nvalid - best_i)), inv_sc));
    return RoundB{a, b, tv, true};
}

template <int EPL, bool FUSED, bool TAIL, int BITS, int IO = 0>
__device__ void fit_bingrad_b(const KParams &p, FitB &, int64_t beta, int w, int lane, uint32_t vmask, bool check,
                              int nvalid, const float (&v)[EPL], const float (&u)[EPL], float (&acc)[EPL], ErrAcc *ea = nullptr)
{
    float m = 0.0f;
#pragma unroll
    for (int t = 0; t < EPL; ++t)
        if (!TAIL || ((vmask >> t) & 1u)) m = fmax_nan(m, fabsf(u[t]));
    m = warp_redux_max_abs(m);
    if (check && !(m <= FLT_MAX)) flag_nonfinite(p, lane);
    int pos[EPL];
#pragma unroll
    for (int t = 0; t < EPL; ++t) pos[t] = 0;
    float key[EPL];
    const RoundB rule = bingrad_b_levels<EPL, TAIL>(lane, vmask, nvalid, m, u, key);
    emit<EPL, FUSED, false, TAIL, BITS, IO>(p, rule, beta, w, lane, vmask, v, u, pos, acc, ea);
    store_table(p, w, beta, lane, lane == 0 ? rule.a : rule.b);
}

// BinGrad-pb: the grid pair (A, B) at least as wide as BinGrad-b's levels (g_A <= a_b, g_B >= b_b)
// with the least expected squared error; clamped outside [g_A, g_B], stochastic inside.
template <int EPL, bool FUSED, bool TAIL, int BITS, int IO = 0>
__device__ void fit_bingrad_pb(const KParams &p, FitPB &sm, int64_t beta, int w, int lane, uint32_t vmask, bool check,
                               int nvalid, const float (&v)[EPL], const float (&u)[EPL], float (&acc)[EPL],
                               ErrAcc *ea = nullptr)
{
    float mn = INFINITY, mx = -INFINITY;
#pragma unroll
    for (int t = 0; t < EPL; ++t)
        if (!TAIL || ((vmask >> t) & 1u)) {
            mn = fmin_nan(mn, u[t]);
            mx = fmax_nan(mx, u[t]);
        }
    mn = warp_redux_min(mn);
    mx = warp_redux_max(mx);
    if (check && !(mn >= -FLT_MAX && mx <= FLT_MAX)) flag_nonfinite(p, lane);
    mn = __fadd_rn(mn, 0.0f);
    mx = __fadd_rn(mx, 0.0f);
    int pos[EPL];
    if (!(mx > mn)) {
#pragma unroll
        for (int t = 0; t < EPL; ++t) pos[t] = 0;
        emit<EPL, FUSED, false, TAIL, BITS, IO>(p, RoundConst{mn}, beta, w, lane, vmask, v, u, pos, acc, ea);
        store_table(p, w, beta, lane, mn);
        return;
    }
    const float range = __fsub_rn(mx, mn);
    const float step = __fdiv_rn(range, 63.0f);
    const float scale = __fmul_rn(__fdiv_rn(63.0f, range), (float)(1 << kPbFBits));
    // the admissible pairs: A <= Amax, the largest grid index whose point is <= a_b (0 if none);
    // B >= Bmin, the smallest whose point is >= b_b (63 if none).  mx > mn makes max|u| > 0, so
    // the level search sorts the values into key.
    int Amax, Bmin;
    float key[EPL];
    {
        const RoundB bl = bingrad_b_levels<EPL, TAIL>(lane, vmask, nvalid, fmaxf(fabsf(mn), fabsf(mx)), u, key);
        const float g0 = grid_point(mn, mx, step, lane), g1 = grid_point(mn, mx, step, lane + 32);
        const unsigned long long le = (unsigned long long)__ballot_sync(kFull, g0 <= bl.a) |
                                      ((unsigned long long)__ballot_sync(kFull, g1 <= bl.a) << 32);
        const unsigned long long ge = (unsigned long long)__ballot_sync(kFull, g0 >= bl.b) |
                                      ((unsigned long long)__ballot_sync(kFull, g1 >= bl.b) << 32);
        Amax = le ? 63 - __clzll(le) : 0;
        Bmin = ge ? __ffsll(ge) - 1 : 63;
    }
#pragma unroll
    for (int t = 0; t < EPL; ++t) pos[t] = grid_pos<kPbFBits>(u[t], mn, scale);
    // Q0, Q1, Q2 (count, sum of positions, of squared positions over the cells < k) from the
    // sorted values: the position is monotone in the value, so the cells are too, and Q(k) is the
    // prefix before the first value whose cell is >= k.  Each nonempty cell records the prefix at
    // its first value; no two values add into one shared counter.
    unsigned long long tx_all, ty_all;
    {
        int cell[EPL];
        unsigned int x1[EPL];
        unsigned long long x2[EPL];
        unsigned int run1 = 0u;  // at most 512 * 63 * 2^16 < 2^32
        unsigned long long run2 = 0ull;
#pragma unroll
        for (int r = 0; r < EPL; ++r) {
            const bool valid = !TAIL || lane * EPL + r < nvalid;
            const int ps = grid_pos<kPbFBits>(key[r], mn, scale);
            cell[r] = valid ? min(ps >> kPbFBits, kTopCell) : 64;
            x1[r] = run1;
            x2[r] = run2;
            if (valid) {
                run1 += (unsigned int)ps;
                run2 += (unsigned long long)ps * (unsigned long long)ps;
            }
        }
        const unsigned int in1 = warp_inclusive_scan(run1, lane);
        const unsigned long long in2 = warp_inclusive_scan(run2, lane);
        tx_all = __shfl_sync(kFull, in1, 31);
        ty_all = __shfl_sync(kFull, in2, 31);
        const unsigned int ex1 = in1 - run1;
        const unsigned long long ex2 = in2 - run2;
        const int prev_cell = __shfl_up_sync(kFull, cell[EPL - 1], 1);
#pragma unroll
        for (int r = 0; r < EPL; ++r) {
            const int cp = r > 0 ? cell[r - 1] : (lane > 0 ? prev_cell : -1);
            if (cell[r] != cp && cell[r] < 64) {
                sm.q0[cell[r]] = lane * EPL + r + 1;
                sm.q1[cell[r]] = ex1 + x1[r];
                sm.q2[cell[r]] = ex2 + x2[r];
            }
        }
    }
    __syncwarp();
    // the per-index terms of E(A,B) = al[A] + be[B] + a*ga[B] + b*de[A]   (a = A*2^16, b = B*2^16)
    {
        const unsigned long long tc_all = (unsigned long long)(TAIL ? nvalid : 32 * EPL);
        const unsigned long long nonempty = (unsigned long long)__ballot_sync(kFull, sm.q0[lane] != 0) |
                                            ((unsigned long long)__ballot_sync(kFull, sm.q0[lane + 32] != 0) << 32);
        unsigned long long uQ0[2], uQ1[2], uQ2[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const unsigned long long later = nonempty & (~0ull << (lane + 32 * h));
            if (later) {
                const int c = __ffsll(later) - 1;
                uQ0[h] = (unsigned long long)(sm.q0[c] - 1);
                uQ1[h] = sm.q1[c];
                uQ2[h] = sm.q2[c];
            } else {
                uQ0[h] = tc_all;
                uQ1[h] = tx_all;
                uQ2[h] = ty_all;
            }
        }
        __syncwarp();
        sm.q0[lane] = 0;
        sm.q0[lane + 32] = 0;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int K = lane + 32 * h;
            const unsigned long long k = (unsigned long long)K << kPbFBits;
            // modular 64-bit arithmetic: every E(A,B) fits in int64, so wrapped partial terms cancel
            sm.al[K] = (long long)(k * k * uQ0[h] - 3ull * k * uQ1[h] + 2ull * uQ2[h]);
            sm.be[K] = (long long)(3ull * k * uQ1[h] - 2ull * uQ2[h] + ty_all - 2ull * k * tx_all + k * k * (tc_all - uQ0[h]));
            sm.ga16[K] = (uQ1[h] - k * uQ0[h]) << kPbFBits;
            sm.de16[K] = (k * uQ0[h] - uQ1[h]) << kPbFBits;
        }
    }
    __syncwarp();
    // The least E over the admissible pairs (A <= Amax, B >= Bmin, A < B), ties to the smallest
    // (A, B), column by column (pb_column_argmin): lane l takes B = Bmin + l and Bmin + l + 32.
    // With ga, de pre-multiplied by 2^16, E = al[A] + be[B] + A * ga16[B] + B * de16[A]
    // (mod 2^64; the exact E fits in int64).  The column minima then go to the warp's reduction.
    long long best_e = 0x7fffffffffffffffll;
    int best_ab = 0x7fffffff;
#pragma unroll 1
    for (int pass = 0; pass < 2; ++pass) {
        const int B = Bmin + lane + 32 * pass;
        const int Ahi = min(Amax, B - 1);
        if (B > 63) break;
        if (Ahi < 0) continue;  // B = 0
        const unsigned long long beB = (unsigned long long)sm.be[B], gaB = sm.ga16[B];
        auto E = [&](int A) {
            return (long long)((unsigned long long)sm.al[A] + beB + (unsigned long long)(unsigned)A * gaB +
                               (unsigned long long)(unsigned)B * sm.de16[A]);
        };
        long long es;
        const int ab = pb_column_argmin(E, Ahi, es) * 64 + B;
        if (es < best_e || (es == best_e && ab < best_ab)) {
            best_e = es;
            best_ab = ab;
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const long long oe = __shfl_xor_sync(kFull, best_e, o);
        const int oab = __shfl_xor_sync(kFull, best_ab, o);
        if (oe < best_e || (oe == best_e && oab < best_ab)) {
            best_e = oe;
            best_ab = oab;
        }
    }
    const int A = best_ab >> 6, B = best_ab & 63;
    RoundPB rule;
    rule.a = grid_point(mn, mx, step, A);
    rule.b = grid_point(mn, mx, step, B);
    rule.rinv = __frcp_rn(__fsub_rn(rule.b, rule.a));
    rule.pa = A << kPbFBits;
    rule.pb = B << kPbFBits;
    emit<EPL, FUSED, true, TAIL, BITS, IO>(p, rule, beta, w, lane, vmask, v, u, pos, acc, ea);
    store_table(p, w, beta, lane, lane == 0 ? rule.a : rule.b);
}

// ---------------------------------------------------------------------------------------------
// One item: clip, fit, round, write
// ---------------------------------------------------------------------------------------------
template <int EPL, int SCHEME, bool FUSED, bool TAIL, int BITS, int IO = 0>
__device__ __forceinline__ void process(const KParams &p, typename FitFor<SCHEME>::type &fit, int64_t beta, int w,
                                        int lane, int nvalid, uint32_t vmask, const float (&v)[EPL], float (&acc)[EPL],
                                        ErrAcc *ea = nullptr)
{
    float u[EPL];
    bool check = true;  // the fit flags non-finite values unless the clip pass already did
    if (p.clip > 0.0f) {
        float am = 0.0f;
#pragma unroll
        for (int t = 0; t < EPL; ++t)
            if (!TAIL || ((vmask >> t) & 1u)) am = fmax_nan(am, fabsf(v[t]));
        am = warp_redux_max_abs(am);
        if (!(am <= FLT_MAX)) flag_nonfinite(p, lane);
        check = false;
        float T = 0.0f;
        if (am > 0.0f) {
            const int e = 20 - fexpo(am);
            const double sc = pow2d(e);
            long long sx = 0, sxx = 0;
#pragma unroll
            for (int t = 0; t < EPL; ++t)
                if (!TAIL || ((vmask >> t) & 1u)) {
                    const long long X = fixed_point(v[t], sc);
                    sx += X;
                    sxx += X * X;
                }
            sx = warp_sum(sx);
            sxx = warp_sum(sxx);
            T = clip_threshold_from_sums(sx, sxx, nvalid, e, p.clip);
        }
#pragma unroll
        for (int t = 0; t < EPL; ++t) {
            float x = v[t];
            x = x < -T ? -T : x;
            x = x > T ? T : x;
            u[t] = x;
        }
    } else {
#pragma unroll
        for (int t = 0; t < EPL; ++t) u[t] = v[t];
    }
    if constexpr (SCHEME == GQ_QSGD || SCHEME == GQ_TERNGRAD)
        fit_qsgd<EPL, FUSED, TAIL, BITS, IO>(p, fit, beta, w, lane, vmask, check, v, u, acc, ea);
    else if constexpr (SCHEME == GQ_QSGD_NEAREST)
        fit_qsgd<EPL, FUSED, TAIL, BITS, IO, true>(p, fit, beta, w, lane, vmask, check, v, u, acc, ea);
    else if constexpr (SCHEME == GQ_QSGD_L2)
        fit_qsgd<EPL, FUSED, TAIL, BITS, IO, false, true>(p, fit, beta, w, lane, vmask, check, v, u, acc, ea);
    else if constexpr (SCHEME == GQ_SIGNSGD)
        fit_sign<EPL, FUSED, TAIL, BITS, IO>(p, beta, w, lane, vmask, check, nvalid, v, u, acc, ea);
    else if constexpr (SCHEME == GQ_ORQ)
        fit_orq<EPL, FUSED, TAIL, BITS, IO>(p, fit, beta, w, lane, vmask, check, v, u, acc, ea);
    else if constexpr (SCHEME == GQ_BINGRAD_B)
        fit_bingrad_b<EPL, FUSED, TAIL, BITS, IO>(p, fit, beta, w, lane, vmask, check, nvalid, v, u, acc, ea);
    else
        fit_bingrad_pb<EPL, FUSED, TAIL, BITS, IO>(p, fit, beta, w, lane, vmask, check, nvalid, v, u, acc, ea);
}

// ---------------------------------------------------------------------------------------------
// The kernels
// ---------------------------------------------------------------------------------------------
// Resident CTAs per SM the register allocation is sized for (4 x 4 warps: 128 registers; at
// 5 x 4 warps the 96-register cap spills and measured slower).
#ifndef GQ_WARP_MIN_BLOCKS
#define GQ_WARP_MIN_BLOCKS 4
#endif
// BinGrad keeps the sorted slice and its prefix sums (BinGrad-b) or the pair search state
// (BinGrad-pb) in registers: 3 and 4 CTAs per SM are the most that compile without spills.
#ifndef GQ_BINB_MIN_BLOCKS
#define GQ_BINB_MIN_BLOCKS 3
#endif
#ifndef GQ_BINPB_MIN_BLOCKS
#define GQ_BINPB_MIN_BLOCKS 3
#endif
template <int EPL, int SCHEME, int WARPS>
constexpr int min_blocks()
{
    return SCHEME == GQ_BINGRAD_B    ? GQ_BINB_MIN_BLOCKS
           : SCHEME == GQ_BINGRAD_PB ? GQ_BINPB_MIN_BLOCKS
                                     : GQ_WARP_MIN_BLOCKS * 4 / WARPS;
}

// Fits with a byte buffer of codes (base-s messages) have it cleared once.
template <class F, class = void> struct HasCodes { static constexpr bool value = false; };
template <class F> struct HasCodes<F, decltype((void)sizeof(((F *)nullptr)->codes))> { static constexpr bool value = true; };

template <int SCHEME, class Fit>
__device__ __forceinline__ void init_fit(const KParams &p, Fit &fit, int lane)
{
    if constexpr (SCHEME == GQ_QSGD || SCHEME == GQ_TERNGRAD || SCHEME == GQ_QSGD_NEAREST || SCHEME == GQ_QSGD_L2) {
        for (int k = lane; k < p.s; k += 32) fit.qr[k] = p.qratio[k];
    }
    if constexpr (SCHEME == GQ_ORQ) {
        for (int i = lane; i < 64 * kHistCols; i += 32) fit.hist[i] = 0u;
    }
    if constexpr (HasCodes<Fit>::value) {
        for (int i = lane; i < kCodeBytesWords + kBaseOutWords; i += 32) fit.codes[i] = 0u;
    }
    if constexpr (SCHEME == GQ_BINGRAD_PB) {
        for (int i = lane; i < 64; i += 32) fit.q0[i] = 0;
    }
}

__device__ __forceinline__ void store_avg4(float *ab, int m, int lane, const float *acc, float inv_w)
{
    __stcs(reinterpret_cast<float4 *>(ab + 128 * m + 4 * lane),
           make_float4(__fmul_rn(acc[0], inv_w), __fmul_rn(acc[1], inv_w), __fmul_rn(acc[2], inv_w),
                       __fmul_rn(acc[3], inv_w)));
}

// Full buckets 0 .. nfull-1: every warp walks its items (bucket, worker), bulk copies one item
// ahead.
// IO = 3: every worker has a residual and a message buffer (known at compile time, so the
// rounding pass is straight-line code); IO = 0: checked at run time.
template <int EPL, int SCHEME, bool FUSED, int BITS, int IO>
__global__ void __launch_bounds__(kWarpsPerCta * 32, (min_blocks<EPL, SCHEME, kWarpsPerCta>()))
    k_warp(const __grid_constant__ KParams p, int64_t nfull)
{
    using Smem = WarpSmem<EPL, SCHEME>;
    constexpr int D = 32 * EPL;
    constexpr unsigned kBytes = D * 4;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    const int lane = threadIdx.x & 31;
    const int wib = threadIdx.x >> 5;
    Smem &sm = reinterpret_cast<Smem *>(smem_raw)[wib];
    init_fit<SCHEME>(p, sm.fit, lane);
    if (lane == 0) {
        for (int k = 0; k < kStages; ++k) mbar_init(&sm.bar[k], 1);
        fence_barrier_init();
    }
    __syncwarp();

    const int64_t first = (int64_t)blockIdx.x * kWarpsPerCta + wib;
    const int64_t stride = (int64_t)gridDim.x * kWarpsPerCta;
    if (first >= nfull) return;
    const int W = p.W;
    const int64_t nitems = ((nfull - 1 - first) / stride + 1) * W;
    const bool ef = (IO & 1) || p.r[0] != nullptr;
    const unsigned tx = ef ? 2 * kBytes : kBytes;
    auto issue = [&](int64_t beta, int w, int k) {  // lane 0
        fence_proxy_async();
        mbar_arrive_expect_tx(&sm.bar[k], tx);
        bulk_load(sm.stage[k].g, p.g[w] + beta * D, kBytes, &sm.bar[k]);
        if (ef) bulk_load(sm.stage[k].r, p.r[w] + beta * D, kBytes, &sm.bar[k]);
    };
    // producer position: kStages items ahead of the consumer
    int64_t pbeta = first;
    int pw = 0;
    for (int k = 0; k < kStages; ++k) {
        if (lane == 0 && (int64_t)k < nitems) issue(pbeta, pw, k);
        if (++pw == W) {
            pw = 0;
            pbeta += stride;
        }
    }

    int64_t beta = first;
    int w = 0;
    unsigned parity = 0;  // bit k: phase parity awaited next on buffer k
    float acc[EPL];
    for (int64_t it = 0; it < nitems; ++it) {
        const int k = kStages == 1 ? 0 : (int)(it % kStages);
        if (!mbar_wait_warp(&sm.bar[k], (parity >> k) & 1u)) {
            // a copy did not complete in time: report it, give every copy still in flight one
            // more bounded wait so that none can land after the warp has left, and stop
            if (lane == 0) atomicOr(p.status, kStatusTimeout);
            for (int j = 0; j < kStages; ++j)
                if ((int64_t)j + it < nitems) mbar_wait_warp(&sm.bar[(k + j) % kStages], (parity >> ((k + j) % kStages)) & 1u);
            return;
        }
        parity ^= 1u << k;
        float v[EPL];
#pragma unroll
        for (int m = 0; m < EPL / 4; ++m) {
            float4 x = *reinterpret_cast<const float4 *>(sm.stage[k].g + 128 * m + 4 * lane);
            if (ef) {
                const float4 y = *reinterpret_cast<const float4 *>(sm.stage[k].r + 128 * m + 4 * lane);
                x = make_float4(__fadd_rn(x.x, y.x), __fadd_rn(x.y, y.y), __fadd_rn(x.z, y.z), __fadd_rn(x.w, y.w));
            }
            v[4 * m + 0] = x.x;
            v[4 * m + 1] = x.y;
            v[4 * m + 2] = x.z;
            v[4 * m + 3] = x.w;
        }
        __syncwarp();
        // the buffer is free again: fetch the item kStages ahead while this one is processed
        if (lane == 0 && it + kStages < nitems) issue(pbeta, pw, k);
        if (++pw == W) {
            pw = 0;
            pbeta += stride;
        }
        const bool last_w = w == W - 1;
        if (w == 0) {
#pragma unroll
            for (int t = 0; t < EPL; ++t) acc[t] = 0.0f;
        }
        process<EPL, SCHEME, FUSED, false, BITS, IO>(p, sm.fit, beta, w, lane, D, 0xffffffffu, v, acc);
        if (FUSED && last_w) {
#pragma unroll
            for (int m = 0; m < EPL / 4; ++m) store_avg4(p.avg + beta * D, m, lane, acc + 4 * m, p.inv_w);
        }
        if (last_w) {
            w = 0;
            beta += stride;
        } else {
            ++w;
        }
    }
}

// gq_quant_error: one warp per bucket, grid-stride, plain 16-byte loads; the bucket's three
// error sums (fixed summation order) go to part[3 * bucket + k].
template <int EPL, int SCHEME>
__global__ void __launch_bounds__(kWarpsPerCta * 32) k_warp_err(const __grid_constant__ KParams p, double *part)
{
    using Fit = typename FitFor<SCHEME>::type;
    constexpr int D = 32 * EPL;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
    Fit &fit = reinterpret_cast<Fit *>(smem_raw)[wib];
    init_fit<SCHEME>(p, fit, lane);
    __syncwarp();
    const float *g = p.g[0];
    const float *r = p.r[0];
    float acc[EPL];
    for (int64_t beta = (int64_t)blockIdx.x * kWarpsPerCta + wib; beta < p.nb; beta += (int64_t)gridDim.x * kWarpsPerCta) {
        const int nvalid = beta == p.nb - 1 ? p.tail : D;
        const float *gb = g + beta * D;
        const float *rb = r ? r + beta * D : nullptr;
        float v[EPL];
        ErrAcc ea{0.0, 0.0, 0.0};
        if (nvalid == D) {
#pragma unroll
            for (int m = 0; m < EPL / 4; ++m) {
                float4 x = __ldg(reinterpret_cast<const float4 *>(gb + 128 * m + 4 * lane));
                if (rb) {
                    const float4 y = __ldg(reinterpret_cast<const float4 *>(rb + 128 * m + 4 * lane));
                    x = make_float4(__fadd_rn(x.x, y.x), __fadd_rn(x.y, y.y), __fadd_rn(x.z, y.z), __fadd_rn(x.w, y.w));
                }
                v[4 * m + 0] = x.x;
                v[4 * m + 1] = x.y;
                v[4 * m + 2] = x.z;
                v[4 * m + 3] = x.w;
            }
            process<EPL, SCHEME, false, false, -1>(p, fit, beta, 0, lane, D, 0xffffffffu, v, acc, &ea);
        } else {
            uint32_t vmask = 0;
#pragma unroll
            for (int t = 0; t < EPL; ++t) {
                const int e = slot_elem(t, lane);
                float x = 0.0f;
                if (e < nvalid) {
                    vmask |= 1u << t;
                    x = gb[e];
                    if (rb) x = __fadd_rn(x, rb[e]);
                }
                v[t] = x;
            }
            process<EPL, SCHEME, false, true, -1>(p, fit, beta, 0, lane, nvalid, vmask, v, acc, &ea);
        }
        ea = warp_sum_err(ea);
        if (lane == 0) {
            part[3 * beta + 0] = ea.e;
            part[3 * beta + 1] = ea.uu;
            part[3 * beta + 2] = ea.qq;
        }
        __syncwarp();
    }
}

template <int EPL, int SCHEME>
cudaError_t launch_err(const KParams &p, double *part, cudaStream_t stream)
{
    using Fit = typename FitFor<SCHEME>::type;
    auto kern = k_warp_err<EPL, SCHEME>;
    const size_t smem = sizeof(Fit) * kWarpsPerCta;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0, per_sm = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kWarpsPerCta * 32, smem);
    if (per_sm < 1) per_sm = 1;
    const int64_t need = (p.nb + kWarpsPerCta - 1) / kWarpsPerCta;
    const int64_t cap = (int64_t)sms * per_sm;
    kern<<<(int)(need < cap ? need : cap), kWarpsPerCta * 32, smem, stream>>>(p, part);
    return cudaGetLastError();
}

template <int SCHEME>
cudaError_t warp_dispatch_err(const KParams &p, double *part, cudaStream_t stream)
{
    switch (p.d) {
    case 128: return launch_err<4, SCHEME>(p, part, stream);
    case 256: return launch_err<8, SCHEME>(p, part, stream);
    default: return launch_err<16, SCHEME>(p, part, stream);
    }
}

// The ragged last bucket (n not a multiple of d): guarded plain loads, one warp per worker
// (warp k takes workers k, k + nwarps, ...).  Each warp's dequantized values are parked in
// shared memory (qbuf[w][e]) and summed afterwards in worker order, which gives the same bits
// as the register sum of the main kernel: every partial sum starts from +0.
template <int EPL, int SCHEME, bool FUSED, int IO = 0>
__global__ void __launch_bounds__(512) k_warp_tail(const __grid_constant__ KParams p)
{
    using Fit = typename FitFor<SCHEME>::type;
    constexpr int D = 32 * EPL;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    Fit &fit = reinterpret_cast<Fit *>(smem_raw)[wid];
    float *qbuf = reinterpret_cast<float *>(smem_raw + sizeof(Fit) * nwarps);  // [W][D]
    init_fit<SCHEME>(p, fit, lane);
    __syncwarp();
    const int64_t beta = p.nb - 1;
    const int nvalid = p.tail;
    uint32_t vmask = 0;
#pragma unroll
    for (int t = 0; t < EPL; ++t) vmask |= (slot_elem(t, lane) < nvalid ? 1u : 0u) << t;
    for (int w = wid; w < p.W; w += nwarps) {
        const float *gb = p.g[w] + beta * D;
        const float *rb = p.r[w] ? p.r[w] + beta * D : nullptr;
        float v[EPL], acc[EPL];
#pragma unroll
        for (int t = 0; t < EPL; ++t) {
            const int e = slot_elem(t, lane);
            float x = 0.0f;
            if (e < nvalid) {
                x = gb[e];
                if (rb) x = __fadd_rn(x, rb[e]);
            }
            v[t] = x;
            acc[t] = 0.0f;
        }
        process<EPL, SCHEME, FUSED, true, 0, IO>(p, fit, beta, w, lane, nvalid, vmask, v, acc);
        if (FUSED) {
#pragma unroll
            for (int t = 0; t < EPL; ++t) qbuf[w * D + slot_elem(t, lane)] = acc[t];
        }
    }
    if (FUSED) {
        __syncthreads();
        float *ab = p.avg + beta * D;
        for (int e = threadIdx.x; e < nvalid; e += blockDim.x) {
            float sum = 0.0f;
            for (int w = 0; w < p.W; ++w) sum = __fadd_rn(sum, qbuf[w * D + e]);
            ab[e] = __fmul_rn(sum, p.inv_w);
        }
    }
}

// The base-s level count a code width can carry (s = 3, 5, 9 for b = 2, 3, 4), 0 for none.
template <int SCHEME, int BITS>
constexpr int base_s_for()
{
    if constexpr (SCHEME == GQ_ORQ || SCHEME == GQ_QSGD || SCHEME == GQ_TERNGRAD || SCHEME == GQ_QSGD_NEAREST ||
                  SCHEME == GQ_QSGD_L2)
        return BITS == 2 ? 3 : BITS == 3 ? 5 : BITS == 4 ? 9 : 0;
    return 0;
}

template <int EPL, int SCHEME, bool FUSED, int BITS>
cudaError_t launch_one(const KParams &p, cudaStream_t stream)
{
    constexpr int D = 32 * EPL;
    constexpr int SB = base_s_for<SCHEME, BITS>();
    const bool bases = SB != 0 && p.fmt_s == SB;  // base-s messages (the plan checked s)
    if (p.fmt_s != 0 && !bases) return cudaErrorInvalidValue;
    const int64_t nfull = p.tail == D ? p.nb : p.nb - 1;
    if (nfull > 0) {
        bool all_io = true;
        for (int w = 0; w < p.W; ++w) all_io = all_io && p.r[w] != nullptr && p.msg[w] != nullptr;
        auto kern = bases ? (all_io ? k_warp<EPL, SCHEME, FUSED, BITS, 3 | (SB << 2)> : k_warp<EPL, SCHEME, FUSED, BITS, (SB << 2)>)
                          : (all_io ? k_warp<EPL, SCHEME, FUSED, BITS, 3> : k_warp<EPL, SCHEME, FUSED, BITS, 0>);
        const size_t smem = sizeof(WarpSmem<EPL, SCHEME>) * kWarpsPerCta;
        int sms = 0, per_sm = 0;
        cudaError_t e = kernel_occupancy(reinterpret_cast<const void *>(kern), kWarpsPerCta * 32, smem, &per_sm, &sms);
        if (e != cudaSuccess) return e;
        const int64_t need = (nfull + kWarpsPerCta - 1) / kWarpsPerCta;
        const int64_t cap = (int64_t)sms * per_sm;
        const int grid = (int)(need < cap ? need : cap);
        kern<<<grid, kWarpsPerCta * 32, smem, stream>>>(p, nfull);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if (nfull < p.nb) {
        using Fit = typename FitFor<SCHEME>::type;
        auto tail = bases ? k_warp_tail<EPL, SCHEME, FUSED, (SB << 2)> : k_warp_tail<EPL, SCHEME, FUSED, 0>;
        const int nwarps = p.W < 16 ? p.W : 16;
        const size_t smem = sizeof(Fit) * nwarps + (FUSED ? (size_t)p.W * D * 4 : 0);
        int sms = 0, per_sm = 0;
        cudaError_t e = kernel_occupancy(reinterpret_cast<const void *>(tail), 32 * nwarps, smem, &per_sm, &sms);
        if (e != cudaSuccess) return e;
        tail<<<1, 32 * nwarps, smem, stream>>>(p);
        return cudaGetLastError();
    }
    return cudaSuccess;
}

// The code width is a template parameter of the main kernel (packing with constant shifts).
template <int SCHEME, int EPL, bool FUSED>
cudaError_t dispatch_bits(const KParams &p, cudaStream_t stream)
{
    if constexpr (SCHEME == GQ_BINGRAD_B || SCHEME == GQ_BINGRAD_PB || SCHEME == GQ_SIGNSGD) {
        return launch_one<EPL, SCHEME, FUSED, 1>(p, stream);
    } else if constexpr (SCHEME == GQ_ORQ) {
        switch (p.bits) {
        case 1: return launch_one<EPL, SCHEME, FUSED, 1>(p, stream);
        case 2: return launch_one<EPL, SCHEME, FUSED, 2>(p, stream);
        case 3: return launch_one<EPL, SCHEME, FUSED, 3>(p, stream);
        default: return launch_one<EPL, SCHEME, FUSED, 4>(p, stream);
        }
    } else {
        switch (p.bits) {
        case 1: return launch_one<EPL, SCHEME, FUSED, 1>(p, stream);
        case 2: return launch_one<EPL, SCHEME, FUSED, 2>(p, stream);
        case 3: return launch_one<EPL, SCHEME, FUSED, 3>(p, stream);
        case 4: return launch_one<EPL, SCHEME, FUSED, 4>(p, stream);
        default: return launch_one<EPL, SCHEME, FUSED, 8>(p, stream);
        }
    }
}

template <int SCHEME>
cudaError_t warp_dispatch(const KParams &p, bool fused, cudaStream_t stream)
{
    switch (p.d) {
    case 128: return fused ? dispatch_bits<SCHEME, 4, true>(p, stream) : dispatch_bits<SCHEME, 4, false>(p, stream);
    case 256: return fused ? dispatch_bits<SCHEME, 8, true>(p, stream) : dispatch_bits<SCHEME, 8, false>(p, stream);
    default: return fused ? dispatch_bits<SCHEME, 16, true>(p, stream) : dispatch_bits<SCHEME, 16, false>(p, stream);
    }
}

}  // namespace

}  // namespace gq
