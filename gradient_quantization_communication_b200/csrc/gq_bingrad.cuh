// gq_bingrad.cuh -- BinGrad-b's split search for the register path without sorting the bucket.
//
// BinGrad-b takes the split k (the k smallest values on the left) that maximises
//   J(k) = S_k^2 / k + (T - S_k)^2 / (n - k)
// over the splits between distinct values, S_k the exact fixed-point sum of the k smallest
// values and T the bucket's total (ties to the smallest k); the levels are the two side means.
// Sorting all d values costs far more than the rest of the step, so the search here orders only
// the values that can hold the best split:
//
//  1. The values are binned on a 64-point grid over [min, max] (cell = integer part of the
//     16-fraction-bit grid position, one packed shared atomic per value as in the ORQ fit).
//     Every bin is a run of the sorted order, so the splits at bin boundaries are known
//     exactly in k (prefix counts) and to within a few grid units in S (prefix position sums):
//     S lies in an interval whose width follows from the position's rounding (at most 1.5
//     units per value) and the fixed-point rounding (half a unit per value).
//  2. J is jointly convex in (k, S), so over a boundary's S interval it is largest at an end,
//     and over all splits inside a bin it is largest at a corner of the region the bin's
//     position sum allows (the t smallest of its c values sum to at most t/c of the bin's sum
//     and at least the sum less c - t values at the bin's upper edge).  The best lower bound
//     over the boundaries, LB, is beaten only by boundaries and bins whose upper bound reaches
//     it (with a 2^-15 relative margin, far above the binary32 error of these bounds).
//  3. The bins between the first and the last such candidate form a window.  Its values are
//     gathered into shared memory bin by bin; each is ranked within its own bin (the bins are
//     already in order) and stored at its sorted place; then every split in the window is
//     screened with a binary32 estimate and the near-best ones are evaluated exactly (binary64
//     J of the exact fixed-point sums, as the exhaustive search does), starting from the exact
//     sum of the values below the window.
// Everything outside the window is provably below LB, so the choice is the exhaustive one.  A
// bucket whose range is too narrow for the grid is treated as a single bin.  All loops are
// rolled: the code stays small enough for the instruction cache next to the emit.
#pragma once

#include "gq_round.cuh"

namespace gq {
namespace {

constexpr int kBHistShift = 22;    // packed histogram word: count << 22 | sum of 16-bit fractions

struct alignas(16) FitB {
    uint32_t hist[64 * 8];  // [cell][column]: count << 22 | fraction sum (<= 64 values per column)
    int P0[72];             // values in cells < j (P0[64] = n)
    uint32_t P1[72];        // sum of their 16-bit grid positions (< 2^31 for d <= 512)
    int fill[64];           // gather counters per cell
    float win[520];         // the window's values in cell order; then the split estimates
    float srt[512];         // the window sorted
    unsigned char wcell[512];  // cell of each gathered value
};

// J estimate in binary32 (within about 2^-21 of J for positive k < n).
__device__ __forceinline__ float j_est(float S, float T, float k, float nk)
{
    const float r = __fsub_rn(T, S);
    return __fadd_rn(__fmul_rn(__fmul_rn(S, S), rcp_approx(k)), __fmul_rn(__fmul_rn(r, r), rcp_approx(nk)));
}

// Fixed-point value round(x * 2^e) (e = 46 - floor(log2 max|u|)) computed exactly in binary32 as
// x * 2^(e/2) * 2^(e - e/2): both factors are representable for e in [-81, 195] and the products
// are exact except below 2^-126, which rounds to 0 either way.
__device__ __forceinline__ long long bfixed(float x, float s1, float s2)
{
    return __float2ll_rn(__fmul_rn(__fmul_rn(x, s1), s2));
}

// BinGrad-b's levels {a, b, split value, split found} of the valid values u (m = max|u| > 0,
// reduced over the warp), as the exhaustive search over the sorted bucket would give them.
template <int EPL, bool TAIL>
__device__ __forceinline__ RoundB bingrad_b_pruned(FitB &sm, int lane, uint32_t vmask, int nvalid, float m,
                                                   const float (&u)[EPL])
{
    float mn = INFINITY, mx = -INFINITY;
#pragma unroll
    for (int t = 0; t < EPL; ++t)
        if (!TAIL || ((vmask >> t) & 1u)) {
            mn = fminf(mn, u[t]);
            mx = fmaxf(mx, u[t]);
        }
    mn = __fadd_rn(warp_redux_min(mn), 0.0f);
    mx = __fadd_rn(warp_redux_max(mx), 0.0f);
    if (!(mx > mn)) return RoundB{mn, mn, mn, false};  // every value equal: one level, code 0
    const int n = nvalid;
    const float range = __fsub_rn(mx, mn);
    const float scale = __fmul_rn(__fdiv_rn(63.0f, range), 65536.0f);
    const bool narrow = !(scale <= 0x1p100f);  // a range too narrow for the grid: one bin
    const int ee = 46 - fexpo(m);
    const float f1 = pow2f(ee >> 1), f2 = pow2f(ee - (ee >> 1));

    // 1. histogram of the grid positions, prefix counts P0 and position sums P1 per cell
    const int col = lane & 7;
    int cell[EPL];
#pragma unroll
    for (int t = 0; t < EPL; ++t) {
        int ps = min(__float2int_rz(__fmul_rn(__fsub_rn(u[t], mn), scale)), 63 << 16);
        if (TAIL || narrow) ps = max(ps, 0);
        if (narrow) ps = 0;
        cell[t] = ps >> 16;
        if (!TAIL || ((vmask >> t) & 1u)) atomicAdd(&sm.hist[cell[t] * 8 + col], (uint32_t)(ps & 0xffff) | (1u << kBHistShift));
    }
    __syncwarp();
    {
        uint32_t t0 = 0, t1 = 0, c0 = 0, c1 = 0;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int q4 = (k + (lane >> 1)) & 3;
            uint4 *ph = reinterpret_cast<uint4 *>(sm.hist + lane * 16) + q4;
            const uint4 x = *ph;
            *ph = make_uint4(0u, 0u, 0u, 0u);
            const uint32_t st = x.x + x.y + x.z + x.w;
            const uint32_t sc = (x.x >> kBHistShift) + (x.y >> kBHistShift) + (x.z >> kBHistShift) + (x.w >> kBHistShift);
            if (q4 < 2) {
                t0 += st;
                c0 += sc;
            } else {
                t1 += st;
                c1 += sc;
            }
        }
        const uint32_t s0 = c0 * ((uint32_t)(2 * lane) << 16) + (t0 - (c0 << kBHistShift));
        const uint32_t s1 = c1 * ((uint32_t)(2 * lane + 1) << 16) + (t1 - (c1 << kBHistShift));
        const unsigned long long own = ((unsigned long long)(s0 + s1) << 16) | (c0 + c1);
        const unsigned long long ex = warp_inclusive_scan(own, lane) - own;
        const int e0 = (int)(ex & 0xffffu);
        const uint32_t es = (uint32_t)(ex >> 16);
        reinterpret_cast<int2 *>(sm.P0)[lane] = make_int2(e0, e0 + (int)c0);
        reinterpret_cast<uint2 *>(sm.P1)[lane] = make_uint2(es, es + s0);
        if (lane == 31) {
            sm.P0[64] = e0 + (int)(c0 + c1);
            sm.P1[64] = es + s0 + s1;
        }
        sm.fill[lane] = 0;
        sm.fill[lane + 32] = 0;
    }

    // 2. the exact total T in fixed point
    long long tsum = 0;
#pragma unroll
    for (int t = 0; t < EPL; ++t)
        if (!TAIL || ((vmask >> t) & 1u)) tsum += bfixed(u[t], f1, f2);
    const long long T = warp_sum(tsum);
    __syncwarp();
    const float Tf = __ll2float_rn(T);
    const float nf = (float)n;

    // 3. bounds -> window [jlo, jhi].  S of the k smallest values, k = P0[j] + t, the t of them
    //    in cell j: S in k Mx + sig (P1[j] + their position sum) -+ (sig * 1.5 + 0.5) k, with
    //    Mx = mn 2^e, sig = 2^e / scale (fixed-point units per grid unit); 64 more units of
    //    slack cover the binary64 rounding of these products.
    int jlo = 0, jhi = 0;
    if (!narrow) {
        const double Mx = __dmul_rn((double)mn, pow2d(ee));
        const double sig = __ddiv_rn(pow2d(ee), (double)scale);
        const double wk = __dadd_rn(__dmul_rn(sig, 1.5), 0.5);
        const float Tn = __fmul_rn(__fmul_rn(Tf, Tf), rcp_approx(nf));  // T^2 / n: J's least value for any k
        float lb = 0.0f;
        float ubb[2], ubc[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int j = 2 * lane + h;  // boundary j (split k = P0[j]) and cell j
            const int k = sm.P0[j], kn = sm.P0[j + 1];
            const double pj = (double)sm.P1[j];
            ubb[h] = -1.0f;
            ubc[h] = -1.0f;
            if (k > 0 && k < n) {
                const double c = __dadd_rn(__dmul_rn((double)k, Mx), __dmul_rn(sig, pj));
                const double hw = __dadd_rn(__dmul_rn(wk, (double)k), 64.0);
                const float lo = __double2float_rn(__dsub_rn(c, hw)), hi = __double2float_rn(__dadd_rn(c, hw));
                const float kf = (float)k, nkf = __fsub_rn(nf, kf);
                const float jl = j_est(lo, Tf, kf, nkf), jh = j_est(hi, Tf, kf, nkf);
                // least J over [lo, hi]: T^2/n when the minimiser kT/n lies inside, else the nearer end
                const float smin = __fmul_rn(__fmul_rn(kf, Tf), rcp_approx(nf));
                lb = fmaxf(lb, (smin >= lo && smin <= hi) ? Tn : fminf(jl, jh));
                ubb[h] = fmaxf(jl, jh);
            }
            const int c = kn - k;
            if (c >= 2) {
                // interior splits t = 1 .. c-1: the t smallest of the cell's c values have
                // position sum at most t F / c (F the cell's sum) and at least max(t L,
                // F - (c - t) U), L and U the cell's edges; J's largest value over that region
                // lies at a corner: t = 1 and t = c - 1 on both ends, and the lower end's kink
                // t = (c U - F) / (U - L)
                const double F = (double)(sm.P1[j + 1] - sm.P1[j]);
                const double L = (double)((unsigned)j << 16), U = (double)((unsigned)(j + 1) << 16);
                const double tk = __dmul_rn(__dsub_rn(__dmul_rn((double)c, U), F), 1.0 / 65536.0);
                // rcp_approx is within 2^-22 of 1/c, so the factor 1 + 2^-20 makes fc >= F / c
                const double fc = __dmul_rn(__dmul_rn(F, (double)rcp_approx((float)c)), 1.0 + 0x1p-20);
                float u4 = 0.0f;
                for (int side = 0; side < 3; ++side) {
                    double t = side == 0 ? 1.0 : (side == 1 ? (double)(c - 1) : tk);
                    if (side == 2 && !(tk > 1.0 && tk < (double)(c - 1))) t = 1.0;  // no kink inside
                    const double kk = __dadd_rn((double)k, t);
                    const double base = __dadd_rn(__dmul_rn(kk, Mx), __dmul_rn(sig, pj));
                    const double hw = __dadd_rn(__dmul_rn(wk, kk), 64.0);
                    const double plo = fmax(__dmul_rn(t, L), __dsub_rn(F, __dmul_rn(__dsub_rn((double)c, t), U)));
                    const double phi = __dmul_rn(t, fc);
                    const float lo = __double2float_rn(__dsub_rn(__dadd_rn(base, __dmul_rn(sig, plo)), hw));
                    const float hi = __double2float_rn(__dadd_rn(__dadd_rn(base, __dmul_rn(sig, phi)), hw));
                    const float kf = __double2float_rn(kk), nkf = __fsub_rn(nf, kf);
                    u4 = fmaxf(u4, fmaxf(j_est(lo, Tf, kf, nkf), j_est(hi, Tf, kf, nkf)));
                }
                ubc[h] = u4;
            }
        }
        lb = __uint_as_float(__reduce_max_sync(kFull, __float_as_uint(lb)));
        const float cut = __fmul_rn(lb, 1.0f - 0x1p-15f);
        // candidate boundaries and cells; bit l of the h-mask stands for j = 2 l + h
        const uint32_t b0 = __ballot_sync(kFull, ubb[0] >= cut), b1 = __ballot_sync(kFull, ubb[1] >= cut);
        const uint32_t c0m = __ballot_sync(kFull, ubc[0] >= cut), c1m = __ballot_sync(kFull, ubc[1] >= cut);
        auto first = [](uint32_t m0, uint32_t m1) {  // smallest j, 64 if none
            const int a = m0 ? 2 * (__ffs(m0) - 1) : 64, b = m1 ? 2 * (__ffs(m1) - 1) + 1 : 64;
            return min(a, b);
        };
        auto last = [](uint32_t m0, uint32_t m1) {  // largest j, -1 if none
            const int a = m0 ? 2 * (31 - __clz(m0)) : -1, b = m1 ? 2 * (31 - __clz(m1)) + 1 : -1;
            return max(a, b);
        };
        // window: cells jlo .. jhi, splits P0[jlo] .. P0[jhi + 1]; a candidate boundary j needs
        // jlo <= j and jhi >= j - 1
        jlo = min(first(c0m, c1m), first(b0, b1));
        jhi = max(last(c0m, c1m), last(b0, b1) - 1);
    }
    const int k0 = sm.P0[jlo];
    const int mw = sm.P0[jhi + 1] - k0;

    // 4. gather the window bin by bin; exact sum of the values below it
    long long below = 0;
#pragma unroll
    for (int t = 0; t < EPL; ++t) {
        const bool valid = !TAIL || ((vmask >> t) & 1u);
        if (valid && cell[t] < jlo) below += bfixed(u[t], f1, f2);
        if (valid && cell[t] >= jlo && cell[t] <= jhi) {
            const int slot = sm.P0[cell[t]] - k0 + atomicAdd(&sm.fill[cell[t]], 1);
            sm.win[slot] = u[t];
            sm.wcell[slot] = (unsigned char)cell[t];
        }
    }
    const long long S0 = warp_sum(below);
    __syncwarp();
    // 5. rank each value within its bin (equal values by slot) and store it at its sorted place
    for (int i = lane; i < mw; i += 32) {
        const float x = sm.win[i];
        const int c = sm.wcell[i];
        const int lo = sm.P0[c] - k0, hi = sm.P0[c + 1] - k0;
        int rank = 0;
        for (int j = lo; j < hi; ++j) {
            const float y = sm.win[j];
            rank += (y < x || (y == x && j < i)) ? 1 : 0;
        }
        sm.srt[lo + rank] = x;
    }
    __syncwarp();
    // 6. every split q = 0 .. mw of the window (k = k0 + q, S = S0 + the q smallest window
    //    values), between distinct values (q = 0 and q = mw are bin boundaries): binary32
    //    estimates first (kept in sm.win), then binary64 J for those near the largest
    float emax = 0.0f;
    long long carry = S0;
    for (int q0 = 0; q0 <= mw; q0 += 32) {
        const int q = q0 + lane;
        const float x = q < mw ? sm.srt[q] : INFINITY;
        const long long X = q < mw ? bfixed(x, f1, f2) : 0ll;
        const long long incl = warp_inclusive_scan(X, lane);
        const long long S = carry + incl - X;
        carry += __shfl_sync(kFull, incl, 31);
        const int k = k0 + q;
        const bool ok = q <= mw && k > 0 && k < n && (q == 0 || q == mw || sm.srt[q - 1] < x);
        float est = -1.0f;
        if (ok) {
            est = j_est(__ll2float_rn(S), Tf, (float)k, __fsub_rn(nf, (float)k));
            emax = fmaxf(emax, est);
        }
        if (q <= mw) sm.win[q] = est;
    }
    const float thr = __fmul_rn(__uint_as_float(__reduce_max_sync(kFull, __float_as_uint(emax))), 1.0f - 0x1p-18f);
    __syncwarp();
    double best_j = -1.0;
    int best_q = 0x7fffffff;
    long long best_s = 0;
    carry = S0;
    for (int q0 = 0; q0 <= mw; q0 += 32) {
        const int q = q0 + lane;
        const float x = q < mw ? sm.srt[q] : INFINITY;
        const long long X = q < mw ? bfixed(x, f1, f2) : 0ll;
        const long long incl = warp_inclusive_scan(X, lane);
        const long long S = carry + incl - X;
        carry += __shfl_sync(kFull, incl, 31);
        const float est = q <= mw ? sm.win[q] : -1.0f;
        if (est >= thr && est >= 0.0f) {
            const int k = k0 + q;
            const double l = __ll2double_rn(S);
            const double rr = __ll2double_rn(T - S);
            const double J = __dadd_rn(__ddiv_rn(__dmul_rn(l, l), (double)k), __ddiv_rn(__dmul_rn(rr, rr), (double)(n - k)));
            if (J > best_j) {  // q rises within a lane: ties keep the smallest
                best_j = J;
                best_q = q;
                best_s = S;
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const double oj = __shfl_xor_sync(kFull, best_j, o);
        const int oq = __shfl_xor_sync(kFull, best_q, o);
        const long long os = __shfl_xor_sync(kFull, best_s, o);
        if (oj > best_j || (oj == best_j && oq < best_q)) {
            best_j = oj;
            best_q = oq;
            best_s = os;
        }
    }
    // the split value: the smallest value right of the split
    float thv = best_q < mw ? sm.srt[best_q] : INFINITY;
    if (best_q == mw) {
#pragma unroll
        for (int t = 0; t < EPL; ++t)
            if ((!TAIL || ((vmask >> t) & 1u)) && cell[t] > jhi) thv = fminf(thv, u[t]);
        thv = warp_redux_min(thv);
    }
    __syncwarp();
    const int k = k0 + best_q;
    const double inv_sc = pow2d(-ee);
    const float a = __double2float_rn(__dmul_rn(__ddiv_rn(__ll2double_rn(best_s), (double)k), inv_sc));
    const float b = __double2float_rn(__dmul_rn(__ddiv_rn(__ll2double_rn(T - best_s), (double)(n - k)), inv_sc));
    return RoundB{a, b, thv, true};
}

}  // namespace
}  // namespace gq
