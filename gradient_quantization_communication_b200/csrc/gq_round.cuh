// gq_round.cuh -- per-element rounding rules of the five schemes and the 128-element chunk
// step shared by the register path (d <= 512) and the shared-memory path (d >= 1024):
// draw, round, dequantize, write the residual, pack the codes densely (shuffles and integer
// multiply-adds).
//
// Every stochastic rule compares U (in [0, 1)) with the unsaturated probability p: U < p has
// the same truth value as U < clamp(p, 0, 1) for every p, NaN included, so no clamp is needed.
#pragma once

#include "gq_device.cuh"

namespace gq {

// QSGD / TernGrad: position y = (u/m + 1) * (s-1)/2 in level units, bracket k = trunc(y)
// clamped to [0, s-2], up with probability y - k.  pair[k] = {level k, level k+1}.
// NEAREST (QSGD-nearest): up iff y - k >= 1/2, no draw; the bracket's probability is then 0 or 1.
template <bool NEAREST>
struct RoundQSGDT {
    float inv_m, h;
    int kmax;
    const float2 *pair;
    __device__ __forceinline__ void round(float u, int, uint32_t word, int &code, float &q) const
    {
        const float y = __fmul_rn(__fadd_rn(__fmul_rn(u, inv_m), 1.0f), h);
        const int k = min(max(__float2int_rz(y), 0), kmax);
        const float pu = __fsub_rn(y, (float)k);
        const bool up = NEAREST ? pu >= 0.5f : unit_float(word) < pu;
        const float2 lp = pair[k];
        code = k + (up ? 1 : 0);
        q = up ? lp.y : lp.x;
    }
    __device__ __forceinline__ void bracket(float u, int, float &lo, float &hi, float &pu) const
    {
        const float y = __fmul_rn(__fadd_rn(__fmul_rn(u, inv_m), 1.0f), h);
        const int k = min(max(__float2int_rz(y), 0), kmax);
        pu = __fsub_rn(y, (float)k);
        if (NEAREST) pu = pu >= 0.5f ? 1.0f : 0.0f;
        lo = pair[k].x;
        hi = pair[k].y;
    }
};
using RoundQSGD = RoundQSGDT<false>;

// Scaled sign: code 1 (level +m1) for u >= 0, both zeros included; code 0 (level -m1) below.
struct RoundSign {
    float m1;
    __device__ __forceinline__ void round(float u, int, uint32_t, int &code, float &q) const
    {
        const bool up = u >= 0.0f;
        code = up ? 1 : 0;
        q = up ? m1 : -m1;
    }
    __device__ __forceinline__ void bracket(float u, int, float &lo, float &hi, float &pu) const
    {
        lo = -m1;
        hi = m1;
        pu = u >= 0.0f ? 1.0f : 0.0f;
    }
};

// ORQ: the bracket of the value's grid cell (the cell is passed in place of the position),
// one entry per cell: ctab[cell] = {lower, upper, 1/(upper-lower), bracket index as bits};
// up with probability (u - lower) / (upper - lower).
struct RoundORQ {
    const float4 *ctab;
    __device__ __forceinline__ void round(float u, int cell, uint32_t word, int &code, float &q) const
    {
        const float4 b = ctab[cell];
        const float pu = __fmul_rn(__fsub_rn(u, b.x), b.z);
        const bool up = unit_float(word) < pu;
        code = __float_as_int(b.w) + (up ? 1 : 0);
        q = up ? b.y : b.x;
    }
    __device__ __forceinline__ void bracket(float u, int cell, float &lo, float &hi, float &pu) const
    {
        const float4 b = ctab[cell];
        lo = b.x;
        hi = b.y;
        pu = __fmul_rn(__fsub_rn(u, b.x), b.z);
    }
};

// Constant bucket: one level, code 0.
struct RoundConst {
    float lv;
    __device__ __forceinline__ void round(float, int, uint32_t, int &code, float &q) const
    {
        code = 0;
        q = lv;
    }
    __device__ __forceinline__ void bracket(float, int, float &lo, float &hi, float &pu) const
    {
        lo = lv;
        hi = lv;
        pu = 0.0f;
    }
};

// BinGrad-b: deterministic, code 1 at or above the split value.
struct RoundB {
    float a, b, thr;
    bool split;
    __device__ __forceinline__ void round(float u, int, uint32_t, int &code, float &q) const
    {
        const bool up = split && u >= thr;
        code = up ? 1 : 0;
        q = up ? b : a;
    }
    __device__ __forceinline__ void bracket(float u, int, float &lo, float &hi, float &pu) const
    {
        lo = a;
        hi = b;
        pu = (split && u >= thr) ? 1.0f : 0.0f;
    }
};

// BinGrad-pb: clamped below the lower / at or above the upper grid level, stochastic between.
struct RoundPB {
    float a, b, rinv;
    int pa, pb;
    __device__ __forceinline__ void round(float u, int pos, uint32_t word, int &code, float &q) const
    {
        bool up;
        if (pos < pa) up = false;
        else if (pos >= pb) up = true;
        else up = unit_float(word) < __fmul_rn(__fsub_rn(u, a), rinv);
        code = up ? 1 : 0;
        q = up ? b : a;
    }
    __device__ __forceinline__ void bracket(float u, int pos, float &lo, float &hi, float &pu) const
    {
        lo = a;
        hi = b;
        if (pos < pa) pu = 0.0f;
        else if (pos >= pb) pu = 1.0f;
        else pu = __fmul_rn(__fsub_rn(u, a), rinv);
    }
};

// Dense packing of one 128-element chunk: the code of element e occupies bits [b*e, b*e + b)
// of the chunk's 4b words (least significant bit first).  Lane l's four codes form the 4b-bit
// field at bit 4b*l; pairs, quads and octets of lanes merge their fields with shuffles (the
// fields do not overlap, so the merges are additions, done by the integer multiply-add unit),
// and lane 8g stores the b words of octet g.  8-bit codes are stored by every lane, one word
// each.  Every lane of the warp must take part.
// BITS: bits per code when known at compile time, 0 to read it from p.bits.
template <int BITS>
__device__ __forceinline__ void pack_chunk(const KParams &p, int lane, const int (&code)[4], uint32_t *cw)
{
    // (BITS < 0 only in never-run instantiations; BITS == 8 never reaches the shifts below)
    const int b = BITS > 0 ? (BITS == 8 ? 1 : BITS) : p.bits;
    if (BITS == 8 || (BITS == 0 && b == 8)) {
        // 8-bit codes: lane l's four codes are word l of the chunk
        __stcs(cw + lane, (uint32_t)code[0] | ((uint32_t)code[1] << 8) | ((uint32_t)code[2] << 16) |
                              ((uint32_t)code[3] << 24));
        return;
    }
    const uint32_t f1 = 1u << b, f2 = 1u << (2 * b), f3 = 1u << (3 * b);
    const uint32_t y = (uint32_t)code[0] + (uint32_t)code[1] * f1 + (uint32_t)code[2] * f2 + (uint32_t)code[3] * f3;
    const uint32_t z = y + __shfl_down_sync(kFull, y, 1) * (1u << (4 * b));  // 8b bits
    const uint32_t z2 = __shfl_down_sync(kFull, z, 2);
    const unsigned long long v = (unsigned long long)z2 * (1ull << (8 * b)) + z;  // 16b bits
    const unsigned long long v2 = __shfl_down_sync(kFull, v, 4);
    if ((lane & 7) == 0) {
        uint32_t *o = cw + b * (lane >> 3);
        if (b == 1) {
            __stcs(o, (uint32_t)v + (uint32_t)v2 * 65536u);
        } else if (b == 2) {
            __stcs(reinterpret_cast<uint2 *>(o), make_uint2((uint32_t)v, (uint32_t)v2));
        } else if (b == 3) {
            __stcs(o, (uint32_t)v);
            __stcs(o + 1, (uint32_t)(v >> 32) + (uint32_t)v2 * 65536u);
            __stcs(o + 2, (uint32_t)(v2 >> 16));
        } else {
            __stcs(reinterpret_cast<uint4 *>(o), make_uint4((uint32_t)v, (uint32_t)(v >> 32), (uint32_t)v2,
                                                            (uint32_t)(v2 >> 32)));
        }
    }
}

// One 128-element chunk of a bucket: lane l holds elements 4l .. 4l+3 of the chunk
// (v: error-fed values, u: clipped values, pos: grid positions; valid: 4-bit mask, ignored
// when ALLVALID).
//   blk   global element index of the chunk's first element, divided by 4
//   rout  residual of the chunk's first element (NULL: no residual), 16-byte aligned
//   cw    packed words of the chunk (4b words, 16-byte aligned), NULL: no message
// Returns the dequantized values in q.
// BITS: bits per code when known at compile time, 0 to read it from p.bits.
// IO: bit 0 set if rout is known non-NULL, bit 1 if cw is (no run-time test then); IO >= 4
// (base-s messages): cw is the chunk's 32 words of codes as bytes in shared memory, element
// order, instead of its packed words.
template <bool RANDOM, bool ALLVALID, int BITS, int IO = 0, class R>
__device__ __forceinline__ void round_chunk(const KParams &p, const R &rule, uint64_t blk, uint32_t worker, int lane,
                                            uint32_t valid, const float (&v)[4], const float (&u)[4],
                                            const int (&pos)[4], float *rout, uint32_t *cw, float (&q)[4])
{
    uint4 rnd = make_uint4(0u, 0u, 0u, 0u);
    if (RANDOM) rnd = draws4(p, blk + (uint64_t)lane, worker);
    const uint32_t words[4] = {rnd.x, rnd.y, rnd.z, rnd.w};
    int code[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        rule.round(u[c], pos[c], words[c], code[c], q[c]);
        if (!ALLVALID && !((valid >> c) & 1u)) code[c] = 0;
    }
    if ((IO & 1) || rout) {
        if (ALLVALID || valid == 0xfu) {
            __stcs(reinterpret_cast<float4 *>(rout + 4 * lane),
                   make_float4(__fsub_rn(v[0], q[0]), __fsub_rn(v[1], q[1]), __fsub_rn(v[2], q[2]), __fsub_rn(v[3], q[3])));
        } else {
#pragma unroll
            for (int c = 0; c < 4; ++c)
                if ((valid >> c) & 1u) rout[4 * lane + c] = __fsub_rn(v[c], q[c]);
        }
    }
    if constexpr (IO >= 4) {
        if ((IO & 2) || cw)
            cw[lane] = (uint32_t)code[0] | ((uint32_t)code[1] << 8) | ((uint32_t)code[2] << 16) | ((uint32_t)code[3] << 24);
    } else {
        if ((IO & 2) || cw) pack_chunk<BITS>(p, lane, code, cw);
    }
}

// Running binary64 sums of the quantization error (see gq_quant_error): expected squared
// rounding error p (b-u)^2 + (1-p) (a-u)^2, u^2, realised (Q(u)-u)^2.
struct ErrAcc {
    double e, uu, qq;
};

template <bool RANDOM, bool ALLVALID, class R>
__device__ __forceinline__ void err_chunk(const KParams &p, const R &rule, uint64_t blk, uint32_t worker, int lane,
                                          uint32_t valid, const float (&u)[4], const int (&pos)[4], ErrAcc &ea)
{
    uint4 rnd = make_uint4(0u, 0u, 0u, 0u);
    if (RANDOM) rnd = draws4(p, blk + (uint64_t)lane, worker);
    const uint32_t words[4] = {rnd.x, rnd.y, rnd.z, rnd.w};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        if (ALLVALID || ((valid >> c) & 1u)) {
            float lo, hi, pu, q;
            int code;
            rule.bracket(u[c], pos[c], lo, hi, pu);
            rule.round(u[c], pos[c], words[c], code, q);
            const double P = (double)sat01(pu);
            const double du = (double)u[c];
            const double dh = __dsub_rn((double)hi, du), dl = __dsub_rn((double)lo, du), dq = __dsub_rn((double)q, du);
            ea.e = __dadd_rn(ea.e, __dadd_rn(__dmul_rn(__dmul_rn(P, dh), dh), __dmul_rn(__dmul_rn(__dsub_rn(1.0, P), dl), dl)));
            ea.uu = __dadd_rn(ea.uu, __dmul_rn(du, du));
            ea.qq = __dadd_rn(ea.qq, __dmul_rn(dq, dq));
        }
    }
}

// Warp sum of an ErrAcc in a fixed butterfly order (every lane gets the same bits).
__device__ __forceinline__ ErrAcc warp_sum_err(ErrAcc a)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        a.e = __dadd_rn(a.e, __shfl_xor_sync(kFull, a.e, o));
        a.uu = __dadd_rn(a.uu, __shfl_xor_sync(kFull, a.uu, o));
        a.qq = __dadd_rn(a.qq, __shfl_xor_sync(kFull, a.qq, o));
    }
    return a;
}

}  // namespace gq
