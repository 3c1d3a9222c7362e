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
// chunk each lane forms the values of every 32nd group and puts them in place (base_s_store).
// Reader: the four codes of a lane (elements 4l .. 4l+3 of a chunk) lie in at most two groups,
// whose 2B <= 32 bits one 64-bit window of two words holds (base_pos); their digits come from a
// shared table (base_run4).
#pragma once

#include "gq_entropy.cuh"

namespace gq {

template <int S>
struct BaseS {
    static constexpr int g = entropy::Base<S>::g;
    static constexpr int B = entropy::Base<S>::B;
};

// The bucket's base-s words from its codes as bytes (c32: the bytes as words, zero past the
// bucket's d-th code and for at least one word more), through the warp's buffer obuf (whose
// bytes past the last group's value must be 0 on entry; they stay 0), to out (nw words,
// global).  Lane l computes the values of groups l, l + 32, ... and stores each as a byte
// (B = 7, 8) or half-word (B = 16); then each lane writes whole output words: for B = 8 and 16
// the buffer's words themselves, for B = 7 the 7-bit values of the six groups that reach the
// word, closed up.  Every lane of the warp takes part.
template <int S, int D>
__device__ __forceinline__ void base_s_store(const uint32_t *c32, uint32_t *obuf, uint32_t *out, int nw, int lane)
{
    constexpr int g = BaseS<S>::g, B = BaseS<S>::B;
    constexpr int G = (D + g - 1) / g;
#pragma unroll
    for (int j0 = 0; j0 < G; j0 += 32) {
        const int j = j0 + lane;
        if (j < G) {
            const int b0 = j * g;  // the group's first code byte
            const uint32_t w0 = c32[b0 >> 2], w1 = c32[(b0 >> 2) + 1];
            const uint32_t x = __byte_perm(w0, w1, 0x3210u + 0x1111u * (uint32_t)(b0 & 3));  // bytes b0 .. b0+3
            uint32_t V;
            if constexpr (S == 5) {
                // b0 + 5 b1 + 25 b2 is the byte at bit 16 of (b0 + b1 2^8 + b2 2^16)(25 + 5 2^8 + 2^16):
                // with codes below 5 the lower bytes of the product (at most 100 and 120) never carry
                V = (((x & 0xffffffu) * 0x10519u) >> 16) & 0xffu;
            } else if constexpr (S == 3) {
                // b0 + 3 b1 + 9 b2 + 27 b3 is the byte at bit 24 of the product with
                // 27 + 9 2^8 + 3 2^16 + 2^24 (lower bytes at most 54, 72, 78: no carry), then 81 b4
                const uint32_t b4 = __byte_perm(w0, w1, 0x4444u + 0x1111u * (uint32_t)(b0 & 3)) & 0xffu;
                V = ((x * 0x0103091Bu) >> 24) + 81u * b4;
            } else {
                const uint32_t b4 = __byte_perm(w0, w1, 0x4444u + 0x1111u * (uint32_t)(b0 & 3)) & 0xffu;
                V = b4;
#pragma unroll
                for (int q = 3; q >= 0; --q) V = V * (uint32_t)S + ((x >> (8 * q)) & 0xffu);
            }
            if constexpr (B == 16) reinterpret_cast<unsigned short *>(obuf)[j] = (unsigned short)V;
            else reinterpret_cast<unsigned char *>(obuf)[j] = (unsigned char)V;  // B = 8, and B = 7 as bytes
        }
    }
    __syncwarp();
    if constexpr (B == 7) {
        // word k holds bits 32k .. 32k+31: groups j0 .. j0+5 (j0 = floor(32k / 7)), from bit
        // 32k - 7 j0; their 7-bit values are gathered from the bytes and closed up
        for (int k = lane; k < nw; k += 32) {
            const int j0 = (32 * k) / 7, off = 32 * k - 7 * j0;
            const uint32_t a0 = obuf[j0 >> 2], a1 = obuf[(j0 >> 2) + 1], a2 = obuf[(j0 >> 2) + 2];
            const uint32_t sel = 0x3210u + 0x1111u * (uint32_t)(j0 & 3);
            const uint32_t xl = __byte_perm(a0, a1, sel), xh = __byte_perm(a1, a2, sel);  // values j0..j0+3, j0+4..
            const uint32_t t = (xl & 0x007f007fu) | ((xl & 0x7f007f00u) >> 1);  // v0|v1<<7 and v2|v3<<7 at 0, 16
            const uint32_t lo28 = (t & 0x3fffu) | ((t >> 16) << 14);
            const uint32_t hi14 = (xh & 0x7fu) | ((xh >> 1) & 0x3f80u);
            const unsigned long long acc = (unsigned long long)lo28 | ((unsigned long long)hi14 << 28);
            __stcs(out + k, (uint32_t)(acc >> off));
        }
    } else {
        for (int k = lane; k < nw; k += 32) __stcs(out + k, obuf[k]);
    }
    __syncwarp();
}

// Digits of one base-s group value, packed 4 bits each (digit k at bits 4k .. 4k+3): the decode
// reads them from a shared table instead of dividing.  s = 3 and 5 index the value itself
// (243 and 125 entries); s = 9 splits V = 729 hi + lo into a 729-entry table of three digits
// and an 81-entry table of two.
// The tables cover every B-bit pattern (values past s^g - 1 decode to digits that are merely
// wrong), so no message can index past them.
template <int S>
struct DigitTab {
    static constexpr int kLo = S == 9 ? 729 : (1 << BaseS<S>::B);
    static constexpr int kHi = S == 9 ? 90 : 1;  // 65535 / 729 < 90
    uint32_t lo[kLo];  // up to five digits: 20 bits
    uint32_t hi[kHi];
};

template <int S>
__device__ __forceinline__ void build_digit_tab(DigitTab<S> &t)
{
    constexpr int nd = S == 9 ? 3 : BaseS<S>::g;  // digits in the low table
    for (int v = threadIdx.x; v < DigitTab<S>::kLo; v += blockDim.x) {
        uint32_t x = (uint32_t)v, packed = 0u;
        for (int k = 0; k < nd; ++k) {
            packed |= (x % (uint32_t)S) << (4 * k);
            x /= (uint32_t)S;
        }
        t.lo[v] = packed;
    }
    if constexpr (S == 9) {
        for (int v = threadIdx.x; v < 90; v += blockDim.x) t.hi[v] = (uint32_t)((v % 9) | (((v / 9) & 15) << 4));
    }
}

// All g digits of a group value, packed 4 bits each.
template <int S>
__device__ __forceinline__ uint32_t group_digits(const DigitTab<S> &t, uint32_t V)
{
    if constexpr (S == 9) return t.lo[V % 729u] | (t.hi[V / 729u] << 12);
    else return t.lo[V];
}

// Where the codes of elements e .. e+3 of a bucket (e a multiple of 4, e + 3 < d) lie in its
// base-s words: at most two groups hold them, in words wi and wi + 1 from bit sh; element e is
// digit k0 of the first.
struct BasePos {
    int wi, sh, k0;
};
template <int S>
__device__ __forceinline__ BasePos base_pos(int e)
{
    constexpr int g = BaseS<S>::g, B = BaseS<S>::B;
    const int j0 = e / g, bit = B * j0;
    return BasePos{bit >> 5, bit & 31, e - j0 * g};
}
// The four codes from the two words (lo, hi) at that place, 4 bits each: code q of the four at
// bits 4q .. 4q+3 of the result (the bits above are the next codes, or 0).  Both groups lie in
// the low 2B <= 32 bits of the pair shifted down by sh.
template <int S>
__device__ __forceinline__ uint32_t base_run4(const DigitTab<S> &t, uint32_t lo, uint32_t hi, const BasePos &ps)
{
    constexpr int g = BaseS<S>::g, B = BaseS<S>::B;
    static_assert(2 * B <= 32 && 4 * g < 32, "two groups in one word, a group's digits below bit 32");
    const uint32_t two = __funnelshift_r(lo, hi, ps.sh);
    constexpr uint32_t mask = (1u << B) - 1u;
    // element e + q is digit k0 + q of the first group, or digit k0 + q - g of the second
    const uint32_t d1 = group_digits<S>(t, two & mask), d2 = group_digits<S>(t, (two >> B) & mask);
    return (d1 >> (4 * ps.k0)) | (d2 << (4 * (g - ps.k0)));
}

}  // namespace gq
