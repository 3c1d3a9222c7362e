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
constexpr int kOrqFBits = 22;         // fraction bits of ORQ fixed-point grid positions
constexpr int kPbFBits = 16;          // fraction bits of BinGrad-pb fixed-point grid positions

// ---------------------------------------------------------------------------------------------
// Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3",
// SC'11): ten rounds, each two 32x32->64-bit products of counter words 0 and 2 with the
// round multipliers, the high halves xor-ed with the other counter words and the round key;
// the key advances by the two Weyl increments between rounds.
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ uint4 philox4x32_10(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3,
                                               uint32_t k0, uint32_t k1)
{
#pragma unroll
    for (int round = 0; round < 10; ++round) {
        if (round > 0) {
            k0 += 0x9E3779B9u;
            k1 += 0xBB67AE85u;
        }
        const uint32_t lo0 = 0xD2511F53u * c0;
        const uint32_t hi0 = __umulhi(0xD2511F53u, c0);
        const uint32_t lo1 = 0xCD9E8D57u * c2;
        const uint32_t hi1 = __umulhi(0xCD9E8D57u, c2);
        const uint32_t y0 = hi1 ^ c1 ^ k0;
        const uint32_t y2 = hi0 ^ c3 ^ k1;
        c0 = y0;
        c1 = lo1;
        c2 = y2;
        c3 = lo0;
    }
    return make_uint4(c0, c1, c2, c3);
}

// The four draws of the 4-element group starting at global element index 4*blk: the counter is
// (blk low word, blk high word, step low word, worker), the key the two words of the seed.
__device__ __forceinline__ uint4 draws4(const KParams &p, uint64_t blk, uint32_t worker)
{
    return philox4x32_10((uint32_t)blk, (uint32_t)(blk >> 32), p.step_lo, worker, p.key0, p.key1);
}

// Uniform in [0, 1) at 24-bit resolution from one Philox output word.
__device__ __forceinline__ float unit_float(uint32_t word)
{
    return __fmul_rn(__uint2float_rn(word >> 8), 0x1p-24f);
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
__device__ __forceinline__ float warp_max_nan(float x)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmax_nan(x, __shfl_xor_sync(kFull, x, o));
    return x;
}
__device__ __forceinline__ long long warp_sum(long long x)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(kFull, x, o);
    return x;
}
__device__ __forceinline__ unsigned long long warp_max_u64(unsigned long long x)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const unsigned long long y = __shfl_xor_sync(kFull, x, o);
        x = y > x ? y : x;
    }
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
// sum (b-x)(x-a) by 2^22 * Delta(C) with
//   Delta(C) = (B-C) * sum_{A<=cell<C} (x - A) + (C-A) * sum_{C<=cell<B} (B - x)
// (x in units of 2^-22 cell).  Each round takes the largest Delta, ties to the smallest C.
// Returns the 64-bit mask of chosen grid indices.
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ unsigned long long orq_greedy(const int *P0, const long long *P1, int s, int lane)
{
    unsigned long long mask = 1ull | (1ull << 63);
    for (int round = 0; round < s - 2; ++round) {
        unsigned long long best = 0;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int C = lane + 32 * h;
            if (C >= 1 && C <= 62 && !((mask >> C) & 1ull)) {
                const unsigned long long below = mask & ((1ull << C) - 1ull);
                const unsigned long long above = mask & ~((2ull << C) - 1ull);
                const int A = 63 - __clzll((long long)below);
                const int B = __ffsll((long long)above) - 1;
                const long long lows = (P1[C] - P1[A]) - ((long long)A << kOrqFBits) * (long long)(P0[C] - P0[A]);
                const long long highs = ((long long)B << kOrqFBits) * (long long)(P0[B] - P0[C]) - (P1[B] - P1[C]);
                const long long delta = (long long)(B - C) * lows + (long long)(C - A) * highs;
                const unsigned long long key = ((unsigned long long)delta << 6) | (unsigned long long)(63 - C);
                best = key > best ? key : best;
            }
        }
        best = warp_max_u64(best);
        mask |= 1ull << (63 - (int)(best & 63ull));
    }
    return mask;
}

// Grid point j of the 64-point grid [mn, mx]: mn + j*step for j < 63, mx for j = 63.
__device__ __forceinline__ float grid_point(float mn, float mx, float step, int j)
{
    return j == 63 ? mx : __fadd_rn(mn, __fmul_rn((float)j, step));
}

// Fixed-point grid position, floor((u - mn) * scale) clamped to [0, 63 * 2^F].
template <int F>
__device__ __forceinline__ int grid_pos(float u, float mn, float scale)
{
    const int y = __float2int_rz(__fmul_rn(__fsub_rn(u, mn), scale));
    return min(max(y, 0), 63 << F);
}

}  // namespace gq
