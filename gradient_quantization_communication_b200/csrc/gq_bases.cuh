// gq_bases.cuh -- base-s messages written by the quantization kernel and read by the decode,
// so that the dense message never exists.
//
// The review "[Paper Review] Optimal Gradient Quantization Condition for Communication-Efficient
// Distributed Training" ("Key findings") quotes compression ratios of 32 / log2(s).  The format
// is that of gq_entropy_pack (gq_entropy.cuh): per bucket, g codes form one base-s number
// V = sum_k code[g*i + k] * s^k of B bits, the group values follow each other in the bucket's
// ceil(ceil(d/g) * B / 32) words, least significant bit first, codes past the bucket's d-th
// count as 0, and the level tables follow the codes region unchanged.
//
// Writer: the encode stores each chunk's codes as bytes in the warp's shared memory (element
// order, one 32-bit word per lane and chunk) instead of packing them; after the bucket's last
// chunk every lane builds whole output words from the bytes (base_word) and stores them.
// Reader: the four codes of a lane (elements 4l .. 4l+3 of a chunk) lie in at most two groups,
// whose 2B <= 32 bits one 64-bit window of two words holds (base_codes4).
#pragma once

#include "gq_entropy.cuh"

namespace gq {

template <int S>
struct BaseS {
    static constexpr int g = entropy::Base<S>::g;
    static constexpr int B = entropy::Base<S>::B;
};

// Word w of a bucket's base-s string, built from its codes as bytes c8[0 .. G*g) (the bytes
// past the bucket's d-th are 0); G = ceil(d / g) groups.
template <int S>
__device__ __forceinline__ uint32_t base_word(const unsigned char *c8, int w, int G)
{
    constexpr int g = BaseS<S>::g, B = BaseS<S>::B;
    constexpr int NG = 32 / B + 2;  // groups that can touch one word
    const int bit0 = 32 * w;
    const int j0 = bit0 / B;
    unsigned long long acc = 0ull;  // the groups j0 .. j0 + NG - 1 from bit B * j0 on
#pragma unroll
    for (int k = 0; k < NG; ++k) {
        const int j = j0 + k;
        if (j < G && B * j < bit0 + 32) {
            uint32_t V = 0u;
#pragma unroll
            for (int q = g - 1; q >= 0; --q) V = V * (uint32_t)S + (uint32_t)c8[j * g + q];
            acc |= (unsigned long long)V << (B * k);
        }
    }
    return (uint32_t)(acc >> (bit0 - B * j0));
}

// The codes of elements e, e+1, e+2, e+3 of a bucket (e a multiple of 4, e + 3 < d) from its
// base-s words (nw of them).
template <int S>
__device__ __forceinline__ void base_codes4(const uint32_t *words, int nw, int e, int (&code)[4])
{
    constexpr int g = BaseS<S>::g, B = BaseS<S>::B;
    const int j0 = e / g;
    const int bit = B * j0, wi = bit >> 5, sh = bit & 31;
    const uint32_t lo = __ldg(words + wi);
    const uint32_t hi = wi + 1 < nw ? __ldg(words + wi + 1) : 0u;
    const unsigned long long two = ((unsigned long long)hi << 32 | lo) >> sh;
    constexpr uint32_t mask = (1u << B) - 1u;
    const uint32_t V0 = (uint32_t)two & mask, V1 = (uint32_t)(two >> B) & mask;
    const int k0 = e - j0 * g;  // digit of element e in group j0
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int k = k0 + q;  // < 2g: group j0 while k < g, else group j0 + 1
        uint32_t V = k < g ? V0 : V1;
        const int kk = k < g ? k : k - g;
#pragma unroll
        for (int t = 0; t < g - 1; ++t)
            if (t < kk) V /= (uint32_t)S;
        code[q] = (int)(V % (uint32_t)S);
    }
}

}  // namespace gq
