// gq_entropy.cuh -- conversion of one chunk of a bucket between the dense codes (b bits per
// code) and base-s groups (g codes per B-bit number V = sum_k code[k] * s^k).
//
// A chunk is CG consecutive groups, chosen so that both its dense bits (CG * g * b) and its
// base-s bits (CG * B) are whole 32-bit words: every chunk starts on a word in both strings
// and converts in registers with compile-time shifts only.
//   s = 3: g = 5, B = 8,  b = 2, CG = 16: 5 dense words <-> 4 base-s words
//   s = 5: g = 3, B = 7,  b = 3, CG = 32: 9 dense words <-> 7 base-s words
//   s = 9: g = 5, B = 16, b = 4, CG = 8:  5 dense words <-> 4 base-s words
// Inside a chunk, groups are converted several at a time in one 32-bit register (SWAR): the
// digit planes of up to three groups are combined with one multiply-add per digit (the fields
// are wide enough that no sum carries into the next field), and unpacking divides two 16-bit
// lanes at once by the constant s with an exact multiply-shift.
//
// Plain C++ on 32-bit unsigned integers (host and device), so that it also compiles for the CPU.
#pragma once

#include <cstdint>

#if defined(__CUDACC__)
#define GQ_HD __host__ __device__ __forceinline__
#else
#define GQ_HD inline
#endif

namespace gq {
namespace entropy {

template <int S>
struct Base;
template <>
struct Base<3> {
    static constexpr int g = 5, B = 8, b = 2, CG = 16;
};
template <>
struct Base<5> {
    static constexpr int g = 3, B = 7, b = 3, CG = 32;
};
template <>
struct Base<9> {
    static constexpr int g = 5, B = 16, b = 4, CG = 8;
};

// `width` bits of the word string `w` starting at bit `pos` (pos + width <= 32 * words of w).
template <int POS, int WIDTH, int N>
GQ_HD uint32_t extract(const uint32_t (&w)[N])
{
    constexpr int q = POS / 32, r = POS % 32;
    constexpr uint32_t mask = WIDTH >= 32 ? 0xffffffffu : (1u << WIDTH) - 1u;
    if constexpr (r + WIDTH <= 32) return (w[q] >> r) & mask;
    const uint64_t two = (uint64_t)w[q] | ((uint64_t)w[q + 1] << 32);
    return (uint32_t)(two >> r) & mask;
}

// OR `y` (WIDTH bits) into the word string `w` at bit `pos`.
template <int POS, int WIDTH, int N>
GQ_HD void deposit(uint32_t (&w)[N], uint32_t y)
{
    constexpr int q = POS / 32, r = POS % 32;
    w[q] |= y << r;
    if constexpr (r + WIDTH > 32) w[q + 1] |= y >> (32 - r);
}

// ---- s = 5 -------------------------------------------------------------------------------
// three groups of 9 dense bits (codes c0 | c1 << 3 | c2 << 6) -> three 7-bit values
GQ_HD uint32_t pack5_run(uint32_t x)
{
    constexpr uint32_t m = 0x001C0E07u;  // a 3-bit digit at bits 0, 9 and 18
    const uint32_t f = (x & m) + 5u * ((x >> 3) & m) + 25u * ((x >> 6) & m);  // fields <= 124 (< 512)
    return (f & 0x7Fu) | ((f >> 2) & 0x3F80u) | ((f >> 4) & 0x1FC000u);
}

// two 7-bit values -> two groups of 9 dense bits.  floor(t / 5) = ((t + 1) * 51) >> 8 for
// 0 <= t <= 127 (51 / 256 under-estimates 1/5 by 1/1280, which the +1 covers up to t = 127).
GQ_HD uint32_t unpack5_run(uint32_t x)
{
    const uint32_t v = (x & 0x7Fu) | ((x << 9) & 0x7F0000u);           // lanes at bits 0 and 16
    const uint32_t q = ((v * 51u + 0x00330033u) >> 8) & 0x001F001Fu;   // floor(v / 5) <= 25
    const uint32_t c0 = v - 5u * q;
    const uint32_t q2 = ((q * 51u + 0x00330033u) >> 8) & 0x00070007u;  // floor(q / 5) <= 5
    const uint32_t c1 = q - 5u * q2;
    const uint32_t dd = c0 | (c1 << 3) | (q2 << 6);                    // 9-bit lanes
    return (dd & 0x1FFu) | ((dd >> 7) & 0x3FE00u);
}

// ---- s = 3 -------------------------------------------------------------------------------
// three groups of 10 dense bits (five 2-bit codes) -> three 8-bit values
GQ_HD uint32_t pack3_run(uint32_t x)
{
    constexpr uint32_t m = 0x00300C03u;  // a 2-bit digit at bits 0, 10 and 20
    uint32_t f = (x >> 8) & m;           // Horner from the highest digit; fields <= 363 (< 1024)
    f = f * 3u + ((x >> 6) & m);
    f = f * 3u + ((x >> 4) & m);
    f = f * 3u + ((x >> 2) & m);
    f = f * 3u + (x & m);
    return (f & 0xFFu) | ((f >> 2) & 0xFF00u) | ((f >> 4) & 0xFF0000u);
}

// two 8-bit values -> two groups of 10 dense bits.  floor(t / 3) = ((t + 1) * 85) >> 8 for
// 0 <= t <= 255.
GQ_HD uint32_t unpack3_run(uint32_t x)
{
    constexpr uint32_t k = 0x00550055u;  // 85 in each lane (the +1)
    const uint32_t v = (x & 0xFFu) | ((x << 8) & 0xFF0000u);
    const uint32_t q1 = ((v * 85u + k) >> 8) & 0x007F007Fu;   // <= 85
    const uint32_t q2 = ((q1 * 85u + k) >> 8) & 0x001F001Fu;  // <= 28
    const uint32_t q3 = ((q2 * 85u + k) >> 8) & 0x000F000Fu;  // <= 9
    const uint32_t q4 = ((q3 * 85u + k) >> 8) & 0x00030003u;  // <= 3
    const uint32_t dd = (v - 3u * q1) | ((q1 - 3u * q2) << 2) | ((q2 - 3u * q3) << 4) | ((q3 - 3u * q4) << 6) |
                        (q4 << 8);
    return (dd & 0x3FFu) | ((dd >> 6) & 0xFFC00u);
}

// ---- s = 9 -------------------------------------------------------------------------------
// one group of 20 dense bits (five 4-bit codes) -> one 16-bit value: digit pairs in bytes,
// then byte pairs in 16-bit lanes
GQ_HD uint32_t pack9_one(uint32_t x)
{
    const uint32_t y = (x & 0x000F0F0Fu) + 9u * ((x >> 4) & 0x000F0F0Fu);   // d0+9d1 | d2+9d3 | d4
    const uint32_t z = (y & 0x00FF00FFu) + 81u * ((y >> 8) & 0x00FF00FFu);  // low | d4 << 16
    return ((z & 0xFFFFu) + 6561u * (z >> 16)) & 0xFFFFu;
}

// one 16-bit value -> one group of 20 dense bits.  floor(t / 9) = (t * 477218589) >> 32 for
// t < 2^16 (477218589 = ceil(2^32 / 9), relative excess 1.2e-9).
GQ_HD uint32_t unpack9_one(uint32_t v)
{
    uint32_t dd = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t q = (uint32_t)(((uint64_t)v * 477218589u) >> 32);
        dd |= (v - 9u * q) << (4 * j);
        v = q;
    }
    return dd | (v << 16);
}

// ---- chunks ------------------------------------------------------------------------------
template <int S, bool PACK>
struct Chunk {
    using C = Base<S>;
    static constexpr int kDenseWords = C::CG * C::g * C::b / 32;
    static constexpr int kBaseWords = C::CG * C::B / 32;
    static constexpr int kSrcWords = PACK ? kDenseWords : kBaseWords;
    static constexpr int kDstWords = PACK ? kBaseWords : kDenseWords;
    static_assert(C::CG * C::g * C::b % 32 == 0 && C::CG * C::B % 32 == 0, "chunks are whole words");
};

template <int R, int S, bool PACK>
struct Runs;

// s = 5: 32 groups; pack in runs of three (the last of two), unpack in runs of two
template <int R>
struct Runs<R, 5, true> {
    template <int NS, int ND>
    GQ_HD static void go(const uint32_t (&in)[NS], uint32_t (&out)[ND])
    {
        constexpr int gk = 3 * R, n = 32 - gk < 3 ? 32 - gk : 3;
        deposit<7 * gk, 7 * n>(out, pack5_run(extract<9 * gk, 9 * n>(in)));
        if constexpr (gk + n < 32) Runs<R + 1, 5, true>::go(in, out);
    }
};
template <int R>
struct Runs<R, 5, false> {
    template <int NS, int ND>
    GQ_HD static void go(const uint32_t (&in)[NS], uint32_t (&out)[ND])
    {
        deposit<18 * R, 18>(out, unpack5_run(extract<14 * R, 14>(in)));
        if constexpr (R + 1 < 16) Runs<R + 1, 5, false>::go(in, out);
    }
};
// s = 3: 16 groups; pack in runs of three (the last of one), unpack in runs of two
template <int R>
struct Runs<R, 3, true> {
    template <int NS, int ND>
    GQ_HD static void go(const uint32_t (&in)[NS], uint32_t (&out)[ND])
    {
        constexpr int gk = 3 * R, n = 16 - gk < 3 ? 16 - gk : 3;
        deposit<8 * gk, 8 * n>(out, pack3_run(extract<10 * gk, 10 * n>(in)));
        if constexpr (gk + n < 16) Runs<R + 1, 3, true>::go(in, out);
    }
};
template <int R>
struct Runs<R, 3, false> {
    template <int NS, int ND>
    GQ_HD static void go(const uint32_t (&in)[NS], uint32_t (&out)[ND])
    {
        deposit<20 * R, 20>(out, unpack3_run(extract<16 * R, 16>(in)));
        if constexpr (R + 1 < 8) Runs<R + 1, 3, false>::go(in, out);
    }
};
// s = 9: 8 groups, one at a time
template <int R>
struct Runs<R, 9, true> {
    template <int NS, int ND>
    GQ_HD static void go(const uint32_t (&in)[NS], uint32_t (&out)[ND])
    {
        deposit<16 * R, 16>(out, pack9_one(extract<20 * R, 20>(in)));
        if constexpr (R + 1 < 8) Runs<R + 1, 9, true>::go(in, out);
    }
};
template <int R>
struct Runs<R, 9, false> {
    template <int NS, int ND>
    GQ_HD static void go(const uint32_t (&in)[NS], uint32_t (&out)[ND])
    {
        deposit<20 * R, 20>(out, unpack9_one(extract<16 * R, 16>(in)));
        if constexpr (R + 1 < 8) Runs<R + 1, 9, false>::go(in, out);
    }
};

// One chunk: in = its source words (words past the bucket's end read as 0), out = its
// destination words.
template <int S, bool PACK>
GQ_HD void convert_chunk(const uint32_t (&in)[Chunk<S, PACK>::kSrcWords], uint32_t (&out)[Chunk<S, PACK>::kDstWords])
{
#pragma unroll
    for (int k = 0; k < Chunk<S, PACK>::kDstWords; ++k) out[k] = 0u;
    Runs<0, S, PACK>::go(in, out);
}

}  // namespace entropy
}  // namespace gq
