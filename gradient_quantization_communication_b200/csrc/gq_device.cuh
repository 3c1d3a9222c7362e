// gq_device.cuh -- device building blocks shared by the quantization kernels.
//
// Arithmetic that decides a code is written with explicit round-to-nearest intrinsics
// (__fadd_rn, __fmul_rn, __fdiv_rn, __dmul_rn ...) and the library is compiled with
// -fmad=false, so that every binary32/binary64 operation rounds on its own, exactly as IEEE
// arithmetic without contraction.  Every level-fit decision is taken from exact integer data
// (min/max, fixed-point positions and int64 sums), which makes it independent of the order in
// which a warp or a block reduces.
#pragma once

#include <cfloat>
#include <cstdint>
#include <cuda_runtime.h>

#include "gq_internal.h"

namespace gq {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kGridPts = 64;          // candidate grid points j = 0..63 (both ends included)
constexpr int kTopCell = 62;          // cells 0..62 lie between grid points
constexpr int kOrqFBits = 16;         // fraction bits of ORQ fixed-point grid positions
constexpr int kPbFBits = 16;          // fraction bits of BinGrad-pb fixed-point grid positions

// ---------------------------------------------------------------------------------------------
// Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3",
// SC'11): ten rounds, each two 32x32->64-bit products of counter words 0 and 2 with the round
// multipliers, the high halves xor-ed with the other counter words and the round key; the key
// advances by the two Weyl increments between rounds.  The ten round keys are computed once on
// the host (KParams::rk0 / rk1), so a round costs two wide multiplies and two xors.
// philox_rounds_2_to_10 runs the last nine rounds on the state left by round 1, which draws4
// computes.
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ uint4 philox_rounds_2_to_10(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3,
                                               const uint32_t *rk0, const uint32_t *rk1)
{
#pragma unroll
    for (int round = 0; round < 9; ++round) {
        const unsigned long long p0 = (unsigned long long)0xD2511F53u * c0;
        const unsigned long long p1 = (unsigned long long)0xCD9E8D57u * c2;
        const uint32_t y0 = (uint32_t)(p1 >> 32) ^ c1 ^ rk0[round];
        const uint32_t y2 = (uint32_t)(p0 >> 32) ^ c3 ^ rk1[round];
        c1 = (uint32_t)p1;
        c3 = (uint32_t)p0;
        c0 = y0;
        c2 = y2;
    }
    return make_uint4(c0, c1, c2, c3);
}

// The four draws of the 4-element group starting at global element index 4*blk: the counter is
// (blk low word, blk high word, step low word, worker), the key the two words of the seed.
// Counter word 2 is the step for every group, so the first round's product of it (step_m1)
// comes precomputed from the host.
__device__ __forceinline__ uint4 draws4(const KParams &p, uint64_t blk, uint32_t worker)
{
    const uint32_t c0 = (uint32_t)blk, c1 = (uint32_t)(blk >> 32);
    const unsigned long long p0 = (unsigned long long)0xD2511F53u * c0;
    const uint32_t y0 = (uint32_t)(p.step_m1 >> 32) ^ c1 ^ p.rk0[0];
    const uint32_t y2 = (uint32_t)(p0 >> 32) ^ worker ^ p.rk1[0];
    return philox_rounds_2_to_10(y0, (uint32_t)p.step_m1, y2, (uint32_t)p0, p.rk0 + 1, p.rk1 + 1);
}

// Uniform in [0, 1) from one Philox output word: the word converted to binary32 rounding toward
// zero, times 2^-32 (exact).  P(U < p) = ceil(p * 2^32) * 2^-32: exactly p for binary32 p >= 2^-9.
__device__ __forceinline__ float unit_float(uint32_t word)
{
    return __fmul_rn(__uint2float_rz(word), 0x1p-32f);
}

// ---------------------------------------------------------------------------------------------
// Small arithmetic helpers
// ---------------------------------------------------------------------------------------------
// floor(log2(m)) for finite m > 0, subnormals included.
__device__ __forceinline__ int fexpo(float m)
{
    const uint32_t bits = __float_as_uint(m);
    const int ex = (int)((bits >> 23) & 0xffu);
    if (ex != 0) return ex - 127;
    const uint32_t mant = bits & 0x7fffffu;
    return (31 - __clz(mant)) - 149;
}

// 2^e as a double, e in [-1022, 1023].
__device__ __forceinline__ double pow2d(int e)
{
    return __longlong_as_double((long long)(1023 + e) << 52);
}

// 2^e as a float, e in [-126, 127].
__device__ __forceinline__ float pow2f(int e)
{
    return __uint_as_float((uint32_t)(127 + e) << 23);
}

// Reciprocal within 1 ulp (hardware approximation; positive normal inputs).
__device__ __forceinline__ float rcp_approx(float x)
{
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// Saturate to [0, 1]; NaN and -0 become +0.
__device__ __forceinline__ float sat01(float x)
{
    x = (x > 0.0f) ? x : 0.0f;
    return (x > 1.0f) ? 1.0f : x;
}

// max that propagates NaN (any NaN operand gives NaN).
__device__ __forceinline__ float fmax_nan(float a, float b)
{
    float r;
    asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
    return r;
}

// min that propagates NaN.
__device__ __forceinline__ float fmin_nan(float a, float b)
{
    float r;
    asm("min.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
    return r;
}

// Three-operand forms (one instruction each on sm_100).
__device__ __forceinline__ float fmax3_nan(float a, float b, float c)
{
    float r;
    asm("max.NaN.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}
__device__ __forceinline__ float fmin3_nan(float a, float b, float c)
{
    float r;
    asm("min.NaN.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// Round to nearest even, float64 -> int64.
__device__ __forceinline__ long long fixed_point(float x, double scale)
{
    return __double2ll_rn(__dmul_rn((double)x, scale));
}

// ---------------------------------------------------------------------------------------------
// Warp reductions (butterfly; all lanes receive the result)
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ float warp_max(float x)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(kFull, x, o));
    return x;
}
__device__ __forceinline__ float warp_min(float x)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fminf(x, __shfl_xor_sync(kFull, x, o));
    return x;
}
// Order-preserving map of binary32 onto int32 (NaN of either sign lands beyond +-inf, so a
// NaN anywhere surfaces in the max or the min): lets a single REDUX find a float min / max.
__device__ __forceinline__ int float_key(float f)
{
    const int b = __float_as_int(f);
    return b ^ ((b >> 31) & 0x7fffffff);
}
__device__ __forceinline__ float key_float(int k) { return __int_as_float(k ^ ((k >> 31) & 0x7fffffff)); }
__device__ __forceinline__ float warp_redux_min(float x) { return key_float(__reduce_min_sync(kFull, float_key(x))); }
__device__ __forceinline__ float warp_redux_max(float x) { return key_float(__reduce_max_sync(kFull, float_key(x))); }
// max of non-negative values (or NaN): their bit patterns order like unsigned integers.
__device__ __forceinline__ float warp_redux_max_abs(float x)
{
    return __uint_as_float(__reduce_max_sync(kFull, __float_as_uint(x)));
}
__device__ __forceinline__ long long warp_sum(long long x)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(kFull, x, o);
    return x;
}
// Inclusive prefix sum over lanes.
template <typename T>
__device__ __forceinline__ T warp_inclusive_scan(T x, int lane)
{
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const T y = __shfl_up_sync(kFull, x, o);
        if (lane >= o) x += y;
    }
    return x;
}

// ---------------------------------------------------------------------------------------------
// Clipping threshold c*sigma of a bucket from its exact fixed-point moments.
// sx, sxx: sums of X = round(v * 2^(20 - floor(log2 m0))) and of X^2 over the n valid values.
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ float clip_threshold_from_sums(long long sx, long long sxx, int n, int e, float c)
{
    const double dn = (double)n;
    const double mean = __ddiv_rn(__ll2double_rn(sx), dn);
    double var = __dsub_rn(__ddiv_rn(__ll2double_rn(sxx), dn), __dmul_rn(mean, mean));
    if (var < 0.0) var = 0.0;
    const double sigma = __dmul_rn(__dsqrt_rn(var), pow2d(-e));
    return __double2float_rn(__dmul_rn((double)c, sigma));
}

// ---------------------------------------------------------------------------------------------
// ORQ greedy over the prefix sums of the fixed-point histogram.
// P0[k] / P1[k]: count / sum of positions of the elements in cells < k (k = 0..63).
// Adding grid index C between the chosen neighbours A < C < B lowers the bucket's variance
// sum (b-x)(x-a) by 2^16 * Delta(C) with
//   Delta(C) = (B-C) * sum_{A<=cell<C} (x - A) + (C-A) * sum_{C<=cell<B} (B - x)
// (x in units of 2^-16 cell).  Each round takes the largest Delta, ties to the smallest C.
// Returns the 64-bit mask of chosen grid indices.
// ---------------------------------------------------------------------------------------------
// One side of Delta: the sum over the values between grid indices K and C (either order) of
// their distance to K, in units of 2^-16 cell,
//   side(K, C) = (P1[C] - P1[K]) - K * 2^16 * (P0[C] - P0[K]),
// so that Delta(C) = (B-C) * side(A, C) + (C-A) * side(B, C).  The true value is non-negative;
// with 32-bit prefix sums (buckets of up to 512 values: every prefix sum is below
// 512 * 63 * 2^16 < 2^31) it is below 2^31 and exact in wrap-around arithmetic.
__device__ __forceinline__ uint32_t orq_side(int K, int P0K, int P0C, uint32_t P1K, uint32_t P1C)
{
    return (P1C - P1K) - (uint32_t)(K << kOrqFBits) * (uint32_t)(P0C - P0K);
}
__device__ __forceinline__ long long orq_side(int K, int P0K, int P0C, long long P1K, long long P1C)
{
    return (P1C - P1K) - (long long)(K << kOrqFBits) * (long long)(P0C - P0K);
}
// Ranking key of candidate C: Delta << 6 | 63 - C (the largest key has the largest Delta, ties
// to the smallest C).  With 32-bit sides the shift rides on the small factors: (B-C)*64 and
// (C-A)*64 are below 2^12, so two 32 x 32 -> 64 multiply-adds give the key exactly (< 2^59).
__device__ __forceinline__ unsigned long long orq_key(int A, int C, int B, uint32_t lows, uint32_t highs)
{
    return (unsigned long long)((uint32_t)(B - C) << 6) * lows +
           ((unsigned long long)((uint32_t)(C - A) << 6) * highs + (unsigned long long)(63 - C));
}
__device__ __forceinline__ unsigned long long orq_key(int A, int C, int B, long long lows, long long highs)
{
    const unsigned long long delta = (unsigned long long)((long long)(B - C) * lows + (long long)(C - A) * highs);
    return (delta << 6) | (unsigned long long)(63 - C);
}

// Incremental form: lane l owns candidates C = l and l + 32 with their current neighbours
// A < C < B, the two sides side(A, C), side(B, C) and the ranking key in registers.  Adding level
// L to the bracket (A, B) of a candidate changes one neighbour and one side: for L < C the lower
// one, for L > C the upper one, and both are side(L, C).  An index that is chosen (or never a
// candidate: 0 and 63) gets key 0 and the empty bracket A = B = C, which no later level splits.
template <class T>
__device__ __forceinline__ unsigned long long orq_greedy(const int *P0, const T *P1, int s, int lane)
{
    unsigned long long mask = 1ull | (1ull << 63);
    int A[2], B[2], P0C[2];
    T P1C[2], lows[2], highs[2];
    unsigned long long key[2];
    const int P0lo = P0[0], P0hi = P0[63];
    const T P1lo = P1[0], P1hi = P1[63];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int C = lane + 32 * h;
        const bool cand = C >= 1 && C <= 62;
        A[h] = cand ? 0 : C;
        B[h] = cand ? 63 : C;
        P0C[h] = P0[C];
        P1C[h] = P1[C];
        lows[h] = orq_side(0, P0lo, P0C[h], P1lo, P1C[h]);
        highs[h] = orq_side(63, P0hi, P0C[h], P1hi, P1C[h]);
        key[h] = cand ? orq_key(0, C, 63, lows[h], highs[h]) : 0ull;
    }
    for (int round = 0; round < s - 2; ++round) {
        const unsigned long long best = key[0] > key[1] ? key[0] : key[1];
        // warp argmax of the 64-bit key: high words first, then low words among the lanes that tie
        const unsigned hi = __reduce_max_sync(kFull, (unsigned)(best >> 32));
        const unsigned lo = __reduce_max_sync(kFull, (unsigned)(best >> 32) == hi ? (unsigned)best : 0u);
        const int L = 63 - (int)(lo & 63u);
        mask |= 1ull << L;
        if (round + 1 == s - 2) break;
        const int P0L = P0[L];
        const T P1L = P1[L];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            // branch-free: the split bracket's candidates take L as one neighbour and side(L, C)
            // as that side; the chosen index itself gets key 0 and the empty bracket
            const int C = lane + 32 * h;
            const bool split = A[h] < L && L < B[h];
            const bool self = C == L;
            const bool below = L < C;
            const T x = orq_side(L, P0L, P0C[h], P1L, P1C[h]);
            A[h] = split ? (self ? C : (below ? L : A[h])) : A[h];
            B[h] = split ? (self ? C : (below ? B[h] : L)) : B[h];
            lows[h] = (split && below) ? x : lows[h];
            highs[h] = (split && !below && !self) ? x : highs[h];
            const unsigned long long nk = orq_key(A[h], C, B[h], lows[h], highs[h]);
            key[h] = split ? (self ? 0ull : nk) : key[h];
        }
    }
    return mask;
}

// Grid point j of the 64-point grid [mn, mx]: mn + j*step for j < 63, mx for j = 63.
__device__ __forceinline__ float grid_point(float mn, float mx, float step, int j)
{
    return j == 63 ? mx : __fadd_rn(mn, __fmul_rn((float)j, step));
}

// Bitonic sort of the 32*EPL keys, position i = lane*EPL + r, ascending, in the form whose
// comparators all put the minimum at the lower index: each merge of blocks of k keys starts by
// comparing i with its mirror i ^ (k-1), then i with i ^ j for j = k/4 .. 1.  Inside a lane a
// compare-exchange is one min and one max; across lanes (partner lane l ^ m) the lower lane keeps
// the minimum, a choice that depends on the lane only.
template <int EPL>
__device__ __forceinline__ void warp_bitonic_sort(float (&key)[EPL], int lane)
{
    constexpr int N = 32 * EPL;
#pragma unroll
    for (int k = 2; k <= N; k <<= 1) {
        if (k <= EPL) {
#pragma unroll
            for (int r = 0; r < EPL; ++r) {
                const int q = r ^ (k - 1);
                if (q > r) {
                    const float a = key[r], b = key[q];
                    key[r] = fminf(a, b);
                    key[q] = fmaxf(a, b);
                }
            }
        } else {
            // partner of (lane, r) is (lane ^ m, EPL-1-r); pairs (r, EPL-1-r) are updated together
            const int m = k / EPL - 1;
            const bool take_min = (lane & ((k / EPL) >> 1)) == 0;
#pragma unroll
            for (int r = 0; r < EPL / 2; ++r) {
                const float o1 = __shfl_xor_sync(kFull, key[EPL - 1 - r], m);
                const float o2 = __shfl_xor_sync(kFull, key[r], m);
                key[r] = take_min ? fminf(key[r], o1) : fmaxf(key[r], o1);
                key[EPL - 1 - r] = take_min ? fminf(key[EPL - 1 - r], o2) : fmaxf(key[EPL - 1 - r], o2);
            }
        }
#pragma unroll
        for (int j = k >> 2; j > 0; j >>= 1) {
            if (j >= EPL) {
                const bool take_min = (lane & (j / EPL)) == 0;
#pragma unroll
                for (int r = 0; r < EPL; ++r) {
                    const float o = __shfl_xor_sync(kFull, key[r], j / EPL);
                    key[r] = take_min ? fminf(key[r], o) : fmaxf(key[r], o);
                }
            } else {
#pragma unroll
                for (int r = 0; r < EPL; ++r) {
                    if ((r & j) == 0) {
                        const float a = key[r], b = key[r ^ j];
                        key[r] = fminf(a, b);
                        key[r ^ j] = fmaxf(a, b);
                    }
                }
            }
        }
    }
}

// The half-cleaner stages j = JTOP, JTOP/2, .., 1 of the same network on the 32*EPL keys
// (position lane*EPL + r): i against i ^ j, the minimum at the lower index.  Applied to a block
// whose two halves hold the outcome of a merge's first stages, it finishes the merge.
template <int EPL, int JTOP>
__device__ __forceinline__ void warp_halfclean(float (&key)[EPL], int lane)
{
#pragma unroll
    for (int j = JTOP; j > 0; j >>= 1) {
        if (j >= EPL) {
            const bool take_min = (lane & (j / EPL)) == 0;
#pragma unroll
            for (int r = 0; r < EPL; ++r) {
                const float o = __shfl_xor_sync(kFull, key[r], j / EPL);
                key[r] = take_min ? fminf(key[r], o) : fmaxf(key[r], o);
            }
        } else {
#pragma unroll
            for (int r = 0; r < EPL; ++r) {
                if ((r & j) == 0) {
                    const float a = key[r], b = key[r ^ j];
                    key[r] = fminf(a, b);
                    key[r ^ j] = fmaxf(a, b);
                }
            }
        }
    }
}

// BinGrad-pb, one column of the pair search: the smallest minimiser over A in [0, Ahi] (Ahi >= 0)
// of E(A) = E(A, B) for a fixed B, and its value in es.  E(a, b) is convex in a for a fixed b: a
// value x contributes (x - a)(b - x), of slope -(b - x) <= 0, while a <= x, and (a - x)^2, of
// slope 2(a - x) >= 0, past it (nothing that depends on a when x > b).  So the differences
// E(A+1) - E(A) never decrease and the first A whose difference is >= 0 (Ahi if none) is the
// answer: the last difference decides whether it is Ahi, else a bisection finds it.  E is exact
// (int64), so the choice is the one an exhaustive scan with ties to the smallest A makes.
template <class EF>
__device__ __forceinline__ int pb_column_argmin(const EF &E, int Ahi, long long &es)
{
    es = E(Ahi);
    if (Ahi == 0) return 0;
    const long long eb = E(Ahi - 1);
    if (es < eb) return Ahi;
    int lo = 0, hi = Ahi - 1;  // the difference at hi is >= 0
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (E(mid + 1) - E(mid) >= 0) hi = mid;
        else lo = mid + 1;
    }
    es = lo == Ahi - 1 ? eb : E(lo);
    return lo;
}

// Fixed-point grid position, floor((u - mn) * scale) clamped to [0, 63 * 2^F].
template <int F>
__device__ __forceinline__ int grid_pos(float u, float mn, float scale)
{
    const int y = __float2int_rz(__fmul_rn(__fsub_rn(u, mn), scale));
    return min(max(y, 0), 63 << F);
}

// ---------------------------------------------------------------------------------------------
// Bulk asynchronous copies (TMA, 1-D, into this CTA only) into shared memory, completed on an mbarrier.
// Every wait is bounded: after kWaitLimitNs of global time it gives up and reports failure.
// ---------------------------------------------------------------------------------------------
constexpr unsigned long long kWaitLimitNs = 1000000000ull;  // one second

__device__ __forceinline__ uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(unsigned long long *bar, unsigned count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

// Make barrier initialisation (generic proxy) visible to the copy engine (async proxy).
__device__ __forceinline__ void fence_barrier_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Order this thread's earlier generic accesses of shared memory before later async-proxy writes.
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void mbar_arrive_expect_tx(unsigned long long *bar, unsigned bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

// 1-D bulk copy global -> shared of `bytes` (multiple of 16, both addresses 16-byte aligned).
__device__ __forceinline__ void bulk_load(void *dst, const void *src, unsigned bytes, unsigned long long *bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(unsigned long long *bar, unsigned parity)
{
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ unsigned long long global_ns()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// Warp-uniform bounded wait for the phase `parity` of `bar`; false if it timed out.
__device__ __forceinline__ bool mbar_wait_warp(unsigned long long *bar, unsigned parity,
                                               unsigned long long limit_ns = kWaitLimitNs)
{
    if (__all_sync(kFull, mbar_try_wait(bar, parity))) return true;
    const unsigned long long t0 = global_ns();
    for (;;) {
        if (__all_sync(kFull, mbar_try_wait(bar, parity))) return true;
        const bool late = global_ns() - t0 > limit_ns;
        if (__any_sync(kFull, late)) return false;
    }
}

}  // namespace gq
