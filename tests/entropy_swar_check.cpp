// Exhaustive host check of the chunk conversions of gq_entropy.cuh (the code the base-s kernels
// run, compiled here for the CPU) against plain digit arithmetic: every valid input of each
// SWAR run, the range of every output for invalid inputs, and random whole chunks both ways.
// Exit status 0 when everything agrees.
#include <cstdio>
#include <cstdlib>
#include <cstdint>
#include <random>
#include "gq_entropy.cuh"
using namespace gq::entropy;

static uint32_t naive_pack(int s, int b, int g, uint32_t x) {  // g codes of b bits -> V
    uint32_t v = 0; for (int k = g - 1; k >= 0; --k) v = v * s + ((x >> (b * k)) & ((1u << b) - 1)); return v; }
static uint32_t naive_unpack(int s, int b, int g, uint32_t v) {
    uint32_t x = 0; for (int k = 0; k < g; ++k) { x |= (v % s) << (b * k); v /= s; } return x; }

int main() {
    long bad = 0;
    // s=5 pack: all valid digit combos for 3 groups
    for (uint32_t i = 0; i < 1953125u; ++i) {
        uint32_t t = i, x = 0;
        for (int k = 0; k < 9; ++k) { x |= (t % 5) << (3 * k); t /= 5; }
        uint32_t want = 0;
        for (int gI = 0; gI < 3; ++gI) want |= naive_pack(5, 3, 3, (x >> (9 * gI)) & 0x1FF) << (7 * gI);
        if (pack5_run(x) != want) { if (bad++ < 5) printf("pack5 %u\n", x); }
    }
    for (uint32_t x = 0; x < (1u << 27); x += 97) if (pack5_run(x) >> 21) { if (bad++ < 5) printf("pack5 range\n"); }
    for (uint32_t x = 0; x < (1u << 14); ++x) {
        uint32_t v0 = x & 0x7F, v1 = x >> 7;
        uint32_t y = unpack5_run(x);
        if (y >> 18) { if (bad++ < 5) printf("unpack5 range %u\n", x); }
        if (v0 < 125 && v1 < 125) {
            uint32_t want = naive_unpack(5, 3, 3, v0) | naive_unpack(5, 3, 3, v1) << 9;
            if (y != want) { if (bad++ < 5) printf("unpack5 %u %u %u\n", x, y, want); }
        }
    }
    printf("s5 done bad=%ld\n", bad);
    for (uint32_t i = 0; i < 14348907u; ++i) {
        uint32_t t = i, x = 0;
        for (int k = 0; k < 15; ++k) { x |= (t % 3) << (2 * k); t /= 3; }
        uint32_t want = 0;
        for (int gI = 0; gI < 3; ++gI) want |= naive_pack(3, 2, 5, (x >> (10 * gI)) & 0x3FF) << (8 * gI);
        if (pack3_run(x) != want) { if (bad++ < 5) printf("pack3 %u\n", x); }
    }
    for (uint32_t x = 0; x < (1u << 30); x += 101) if (pack3_run(x) >> 24) { if (bad++ < 5) printf("pack3 range\n"); }
    for (uint32_t x = 0; x < (1u << 16); ++x) {
        uint32_t v0 = x & 0xFF, v1 = x >> 8;
        uint32_t y = unpack3_run(x);
        if (y >> 20) { if (bad++ < 5) printf("unpack3 range\n"); }
        if (v0 < 243 && v1 < 243) {
            uint32_t want = naive_unpack(3, 2, 5, v0) | naive_unpack(3, 2, 5, v1) << 10;
            if (y != want) { if (bad++ < 5) printf("unpack3 %u\n", x); }
        }
    }
    printf("s3 done bad=%ld\n", bad);
    for (uint32_t i = 0; i < 59049u; ++i) {
        uint32_t t = i, x = 0;
        for (int k = 0; k < 5; ++k) { x |= (t % 9) << (4 * k); t /= 9; }
        if (pack9_one(x) != naive_pack(9, 4, 5, x)) { if (bad++ < 5) printf("pack9 %u\n", x); }
    }
    for (uint32_t x = 0; x < (1u << 20); ++x) if (pack9_one(x) >> 16) { if (bad++ < 5) printf("pack9 range\n"); }
    for (uint32_t v = 0; v < (1u << 16); ++v) {
        uint32_t y = unpack9_one(v);
        if (y >> 20) { if (bad++ < 5) printf("unpack9 range\n"); }
        if (v < 59049 && y != naive_unpack(9, 4, 5, v)) { if (bad++ < 5) printf("unpack9 %u\n", v); }
    }
    printf("s9 done bad=%ld\n", bad);
    // chunk level: random valid chunks round trip and match a naive bit-string conversion
    std::mt19937_64 rng(1);
    auto chunk_test = [&](auto tagS) {
        constexpr int S = decltype(tagS)::value;
        using C = Base<S>; using P = Chunk<S, true>; using U = Chunk<S, false>;
        for (int it = 0; it < 20000; ++it) {
            uint32_t dense[P::kSrcWords] = {0}, base[P::kDstWords], back[U::kDstWords], want[P::kDstWords] = {0};
            for (int gI = 0; gI < C::CG; ++gI) {
                uint32_t v = 0, p = 1;
                for (int k = 0; k < C::g; ++k) {
                    uint32_t c = rng() % S; int bit = (gI * C::g + k) * C::b;
                    for (int j = 0; j < C::b; ++j) if ((c >> j) & 1) dense[(bit + j) / 32] |= 1u << ((bit + j) % 32);
                    v += c * p; p *= S;
                }
                for (int j = 0; j < C::B; ++j) { int bit = gI * C::B + j; if ((v >> j) & 1) want[bit / 32] |= 1u << (bit % 32); }
            }
            convert_chunk<S, true>(dense, base);
            convert_chunk<S, false>(base, back);
            for (int k = 0; k < P::kDstWords; ++k) if (base[k] != want[k]) { if (bad++ < 5) printf("chunk pack S=%d\n", S); }
            for (int k = 0; k < U::kDstWords; ++k) if (back[k] != dense[k]) { if (bad++ < 5) printf("chunk unpack S=%d\n", S); }
        }
    };
    chunk_test(std::integral_constant<int, 3>{});
    chunk_test(std::integral_constant<int, 5>{});
    chunk_test(std::integral_constant<int, 9>{});
    printf("chunks done bad=%ld\n", bad);
    return bad != 0;
}
