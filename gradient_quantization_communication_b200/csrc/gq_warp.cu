// gq_warp.cu -- register-resident quantization kernels for buckets of d = 128, 256, 512.
//
// One warp owns one bucket index.  Lane l holds EPL = d/32 values in registers, slot t being
// element 128*(t/4) + 4*l + t%4 of the bucket, so every load and store is a coalesced 16-byte
// access and the four values of a slot group share one Philox call.  For the fused step the
// warp walks the W workers of its bucket in worker order, quantizes each, writes the residual
// (and optionally the message) and accumulates the dequantized values in registers; the
// average leaves the chip once, after the last worker.  Level fits per bucket:
//   QSGD / TernGrad : m = max|u|, s uniform levels on [-m, m]
//   ORQ             : lane-private shared-memory histogram of 22-bit fixed-point grid
//                     positions -> exact int64 prefix sums -> s-2 greedy rounds
//   BinGrad-b       : warp bitonic sort -> exact int64 prefix sums -> argmax of J(k)
//   BinGrad-pb      : shared-memory moments of 16-bit positions -> exact search of all
//                     2016 grid pairs
#include "gq_round.cuh"

namespace gq {
namespace {

constexpr int kWarpsPerCta = 4;

// ---------------------------------------------------------------------------------------------
// Per-warp shared memory, one layout per scheme
// ---------------------------------------------------------------------------------------------
struct alignas(16) SmemORQ {
    uint32_t hist[64 * 32];  // [cell][lane]: (count << 27) + sum of 22-bit fractions
    long long P1[64];        // sum of positions over cells < k
    int P0[64];              // count over cells < k
    float4 tab[16];          // bracket k: {lower level, upper level, 1/(upper-lower), 0}
    float lev[16];           // ascending levels
    unsigned char lut[64];   // cell -> bracket
};
struct alignas(16) SmemQSGD {
    float lev[16];
};
struct alignas(16) SmemPB {
    unsigned long long s1[64], s2[64];  // per cell: sum of positions, of squared positions
    unsigned int cnt[64];               // per cell: count
    long long al[64], be[64], ga[64], de[64];
};
struct alignas(16) SmemB {
    float lev[4];
};

template <int S> struct SmemFor { using type = SmemQSGD; };
template <> struct SmemFor<GQ_ORQ> { using type = SmemORQ; };
template <> struct SmemFor<GQ_BINGRAD_PB> { using type = SmemPB; };
template <> struct SmemFor<GQ_BINGRAD_B> { using type = SmemB; };

__device__ __forceinline__ int slot_elem(int t, int lane) { return 128 * (t >> 2) + 4 * lane + (t & 3); }

// ---------------------------------------------------------------------------------------------
// Loads: v = g (+ r)
// ---------------------------------------------------------------------------------------------
template <int EPL>
__device__ __forceinline__ void load_bucket(const float *g, const float *r, int64_t base, int nvalid,
                                            bool full, int lane, float (&v)[EPL])
{
    const float *gb = g + base;
    if (full) {
#pragma unroll
        for (int m = 0; m < EPL / 4; ++m) {
            const float4 x = __ldcs(reinterpret_cast<const float4 *>(gb + 128 * m + 4 * lane));
            v[4 * m + 0] = x.x;
            v[4 * m + 1] = x.y;
            v[4 * m + 2] = x.z;
            v[4 * m + 3] = x.w;
        }
        if (r) {
            const float *rb = r + base;
#pragma unroll
            for (int m = 0; m < EPL / 4; ++m) {
                const float4 y = __ldcs(reinterpret_cast<const float4 *>(rb + 128 * m + 4 * lane));
                v[4 * m + 0] = __fadd_rn(v[4 * m + 0], y.x);
                v[4 * m + 1] = __fadd_rn(v[4 * m + 1], y.y);
                v[4 * m + 2] = __fadd_rn(v[4 * m + 2], y.z);
                v[4 * m + 3] = __fadd_rn(v[4 * m + 3], y.w);
            }
        }
    } else {
#pragma unroll
        for (int t = 0; t < EPL; ++t) {
            const int e = slot_elem(t, lane);
            float x = 0.0f;
            if (e < nvalid) {
                x = gb[e];
                if (r) x = __fadd_rn(x, r[base + e]);
            }
            v[t] = x;
        }
    }
}

// ---------------------------------------------------------------------------------------------
// Round + pack + residual + accumulate for one worker-bucket, chunk by chunk.
// ---------------------------------------------------------------------------------------------
template <int EPL, bool FUSED, bool RANDOM, class R>
__device__ __forceinline__ void emit(const KParams &p, const R &rule, int64_t beta, int w, int lane, uint32_t vmask,
                                     const float (&v)[EPL], const float (&u)[EPL], const int (&pos)[EPL],
                                     float (&acc)[EPL])
{
    const int64_t base = beta * (int64_t)(32 * EPL);
    float *r = p.r[w];
    unsigned char *msg = p.msg[w];
    uint32_t *cw = msg ? reinterpret_cast<uint32_t *>(msg) + beta * p.codes_words : nullptr;
    const uint32_t worker = p.worker0 + (uint32_t)w;
#pragma unroll
    for (int m = 0; m < EPL / 4; ++m) {
        const float vv[4] = {v[4 * m], v[4 * m + 1], v[4 * m + 2], v[4 * m + 3]};
        const float uu[4] = {u[4 * m], u[4 * m + 1], u[4 * m + 2], u[4 * m + 3]};
        const int pp[4] = {pos[4 * m], pos[4 * m + 1], pos[4 * m + 2], pos[4 * m + 3]};
        const uint32_t valid = (vmask >> (4 * m)) & 0xfu;
        float q[4];
        round_chunk<RANDOM>(p, rule, (uint64_t)(base >> 2) + (uint64_t)(32 * m), worker, lane, valid, vv, uu, pp,
                            r ? r + base + 128 * m : nullptr, cw ? cw + m * 4 * p.bits : nullptr, q);
        if (FUSED) {
#pragma unroll
            for (int c = 0; c < 4; ++c)
                if ((valid >> c) & 1u) acc[4 * m + c] = __fadd_rn(acc[4 * m + c], q[c]);
        }
    }
}

// Level table of the message (L floats per bucket).
__device__ __forceinline__ void store_table(const KParams &p, int w, int64_t beta, int lane, float value)
{
    unsigned char *msg = p.msg[w];
    if (msg && lane < p.L) reinterpret_cast<float *>(msg + p.levels_off)[beta * p.L + lane] = value;
}

// ---------------------------------------------------------------------------------------------
// Per-scheme fits
// ---------------------------------------------------------------------------------------------
template <int EPL, bool FUSED>
__device__ void fit_qsgd(const KParams &p, SmemQSGD &sm, int64_t beta, int w, int lane, bool full, uint32_t vmask,
                         const float (&v)[EPL], const float (&u)[EPL], float (&acc)[EPL])
{
    float m = 0.0f;
#pragma unroll
    for (int t = 0; t < EPL; ++t)
        if ((vmask >> t) & 1u) m = fmaxf(m, fabsf(u[t]));
    m = warp_max(m);
    const int s = p.s;
    __syncwarp();
    if (lane < s) sm.lev[lane] = __fmul_rn(m, __fdiv_rn((float)(2 * lane - (s - 1)), (float)(s - 1)));
    __syncwarp();
    RoundQSGD rule;
    rule.inv_m = m > 0.0f ? __fdiv_rn(1.0f, m) : 0.0f;
    rule.h = __fmul_rn((float)(s - 1), 0.5f);
    rule.s = s;
    rule.lev = sm.lev;
    int pos[EPL];
#pragma unroll
    for (int t = 0; t < EPL; ++t) pos[t] = 0;
    emit<EPL, FUSED, true>(p, rule, beta, w, lane, vmask, v, u, pos, acc);
    store_table(p, w, beta, lane, m);
}

template <int EPL, bool FUSED>
__device__ void fit_orq(const KParams &p, SmemORQ &sm, int64_t beta, int w, int lane, bool full, uint32_t vmask,
                        const float (&v)[EPL], const float (&u)[EPL], float (&acc)[EPL])
{
    float mn = INFINITY, mx = -INFINITY;
#pragma unroll
    for (int t = 0; t < EPL; ++t)
        if ((vmask >> t) & 1u) {
            mn = fminf(mn, u[t]);
            mx = fmaxf(mx, u[t]);
        }
    mn = __fadd_rn(warp_min(mn), 0.0f);
    mx = __fadd_rn(warp_max(mx), 0.0f);
    int pos[EPL];
    if (!(mx > mn)) {
#pragma unroll
        for (int t = 0; t < EPL; ++t) pos[t] = 0;
        RoundConst rule{mn};
        emit<EPL, FUSED, false>(p, rule, beta, w, lane, vmask, v, u, pos, acc);
        store_table(p, w, beta, lane, mn);
        return;
    }
    const float range = __fsub_rn(mx, mn);
    const float step = __fdiv_rn(range, 63.0f);
    const float scale = __fmul_rn(__fdiv_rn(63.0f, range), (float)(1 << kOrqFBits));
    // lane-private histogram: no two lanes ever touch the same word
#pragma unroll
    for (int t = 0; t < EPL; ++t) {
        pos[t] = grid_pos<kOrqFBits>(u[t], mn, scale);
        if ((vmask >> t) & 1u) {
            const int cell = min(pos[t] >> kOrqFBits, kTopCell);
            sm.hist[cell * 32 + lane] += (1u << 27) + (uint32_t)(pos[t] - (cell << kOrqFBits));
        }
    }
    __syncwarp();
    // column sums for cells lane and lane+32 (skewed so that the 32 lanes hit 32 banks), then clear
    uint32_t ca = 0, fa = 0, cb = 0, fb = 0;
#pragma unroll 8
    for (int k = 0; k < 32; ++k) {
        const int col = (lane + k) & 31;
        const uint32_t xa = sm.hist[lane * 32 + col];
        const uint32_t xb = sm.hist[(lane + 32) * 32 + col];
        sm.hist[lane * 32 + col] = 0u;
        sm.hist[(lane + 32) * 32 + col] = 0u;
        ca += xa >> 27;
        fa += xa & 0x7ffffffu;
        cb += xb >> 27;
        fb += xb & 0x7ffffffu;
    }
    const long long sa = (long long)ca * ((long long)lane << kOrqFBits) + (long long)fa;
    const long long sb = (long long)cb * ((long long)(lane + 32) << kOrqFBits) + (long long)fb;
    // exclusive prefix over cells 0..63
    const int ica = warp_inclusive_scan((int)ca, lane);
    const long long isa = warp_inclusive_scan(sa, lane);
    const int icb = warp_inclusive_scan((int)cb, lane);
    const long long isb = warp_inclusive_scan(sb, lane);
    const int tca = __shfl_sync(kFull, ica, 31);
    const long long tsa = __shfl_sync(kFull, isa, 31);
    sm.P0[lane] = ica - (int)ca;
    sm.P1[lane] = isa - sa;
    sm.P0[lane + 32] = tca + icb - (int)cb;
    sm.P1[lane + 32] = tsa + isb - sb;
    __syncwarp();
    const unsigned long long mask = orq_greedy(sm.P0, sm.P1, p.s, lane);
    // levels, cell -> bracket table, brackets
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int j = lane + 32 * h;
        const unsigned long long upto = (j == 63) ? ~0ull : ((2ull << j) - 1ull);
        if ((mask >> j) & 1ull) sm.lev[__popcll(mask & ((1ull << j) - 1ull))] = grid_point(mn, mx, step, j);
        if (j <= kTopCell) sm.lut[j] = (unsigned char)(__popcll(mask & upto) - 1);
    }
    __syncwarp();
    if (lane < p.s - 1) {
        const float lo = sm.lev[lane], hi = sm.lev[lane + 1];
        sm.tab[lane] = make_float4(lo, hi, __fdiv_rn(1.0f, __fsub_rn(hi, lo)), 0.0f);
    }
    __syncwarp();
    RoundORQ rule{sm.lut, sm.tab, sm.lev};
    emit<EPL, FUSED, true>(p, rule, beta, w, lane, vmask, v, u, pos, acc);
    store_table(p, w, beta, lane, lane < p.s ? sm.lev[lane] : 0.0f);
    __syncwarp();
}

// Bitonic sort of the 32*EPL keys, position i = lane*EPL + r.
template <int EPL>
__device__ __forceinline__ void warp_bitonic_sort(float (&key)[EPL], int lane)
{
    constexpr int N = 32 * EPL;
#pragma unroll
    for (int k = 2; k <= N; k <<= 1) {
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
            if (j >= EPL) {
                const int lm = j / EPL;
#pragma unroll
                for (int r = 0; r < EPL; ++r) {
                    const int i = lane * EPL + r;
                    const float o = __shfl_xor_sync(kFull, key[r], lm);
                    const bool up = (i & k) == 0;
                    const bool lower = (i & j) == 0;
                    key[r] = (lower == up) ? fminf(key[r], o) : fmaxf(key[r], o);
                }
            } else {
#pragma unroll
                for (int r = 0; r < EPL; ++r) {
                    if ((r & j) == 0) {
                        const int i = lane * EPL + r;
                        const bool up = (i & k) == 0;
                        const float a = key[r], b = key[r ^ j];
                        key[r] = up ? fminf(a, b) : fmaxf(a, b);
                        key[r ^ j] = up ? fmaxf(a, b) : fminf(a, b);
                    }
                }
            }
        }
    }
}

template <int EPL, bool FUSED>
__device__ void fit_bingrad_b(const KParams &p, SmemB &, int64_t beta, int w, int lane, bool full, uint32_t vmask,
                              int nvalid, const float (&v)[EPL], const float (&u)[EPL], float (&acc)[EPL])
{
    float m = 0.0f;
#pragma unroll
    for (int t = 0; t < EPL; ++t)
        if ((vmask >> t) & 1u) m = fmaxf(m, fabsf(u[t]));
    m = warp_max(m);
    int pos[EPL];
#pragma unroll
    for (int t = 0; t < EPL; ++t) pos[t] = 0;
    RoundB rule{0.0f, 0.0f, 0.0f, false};
    if (m > 0.0f) {
        float key[EPL];
#pragma unroll
        for (int t = 0; t < EPL; ++t) key[t] = ((vmask >> t) & 1u) ? u[t] : INFINITY;
        warp_bitonic_sort<EPL>(key, lane);
        const int e = 46 - fexpo(m);
        const double sc = pow2d(e);
        // inclusive prefix of the fixed-point values inside the lane, then across lanes
        long long pre[EPL];
        long long run = 0;
#pragma unroll
        for (int r = 0; r < EPL; ++r) {
            const int i = lane * EPL + r;
            run += (i < nvalid) ? fixed_point(key[r], sc) : 0ll;
            pre[r] = run;
        }
        const long long incl = warp_inclusive_scan(run, lane);
        const long long lane_excl = incl - run;
        const long long total = __shfl_sync(kFull, incl, 31);
        const float prev_last = __shfl_up_sync(kFull, key[EPL - 1], 1);
        double best_j = -1.0;
        int best_i = 0x7fffffff;
#pragma unroll
        for (int r = 0; r < EPL; ++r) {
            const int i = lane * EPL + r;  // split: positions < i on the left
            const float prev = r > 0 ? key[r - 1] : prev_last;
            if (i >= 1 && i < nvalid && prev < key[r]) {
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
            rule = RoundB{v0, v0, v0, false};
        } else {
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
            const float b = __double2float_rn(
                __dmul_rn(__ddiv_rn(__ll2double_rn(total - sl), (double)(nvalid - best_i)), inv_sc));
            rule = RoundB{a, b, tv, true};
        }
    }
    emit<EPL, FUSED, false>(p, rule, beta, w, lane, vmask, v, u, pos, acc);
    store_table(p, w, beta, lane, lane == 0 ? rule.a : rule.b);
}

template <int EPL, bool FUSED>
__device__ void fit_bingrad_pb(const KParams &p, SmemPB &sm, int64_t beta, int w, int lane, bool full, uint32_t vmask,
                               const float (&v)[EPL], const float (&u)[EPL], float (&acc)[EPL])
{
    float mn = INFINITY, mx = -INFINITY;
#pragma unroll
    for (int t = 0; t < EPL; ++t)
        if ((vmask >> t) & 1u) {
            mn = fminf(mn, u[t]);
            mx = fmaxf(mx, u[t]);
        }
    mn = __fadd_rn(warp_min(mn), 0.0f);
    mx = __fadd_rn(warp_max(mx), 0.0f);
    int pos[EPL];
    if (!(mx > mn)) {
#pragma unroll
        for (int t = 0; t < EPL; ++t) pos[t] = 0;
        RoundConst rule{mn};
        emit<EPL, FUSED, false>(p, rule, beta, w, lane, vmask, v, u, pos, acc);
        store_table(p, w, beta, lane, mn);
        return;
    }
    const float range = __fsub_rn(mx, mn);
    const float step = __fdiv_rn(range, 63.0f);
    const float scale = __fmul_rn(__fdiv_rn(63.0f, range), (float)(1 << kPbFBits));
#pragma unroll
    for (int t = 0; t < EPL; ++t) {
        pos[t] = grid_pos<kPbFBits>(u[t], mn, scale);
        if ((vmask >> t) & 1u) {
            const int cell = min(pos[t] >> kPbFBits, kTopCell);
            const unsigned long long x = (unsigned long long)pos[t];
            atomicAdd(&sm.cnt[cell], 1u);
            atomicAdd(&sm.s1[cell], x);
            atomicAdd(&sm.s2[cell], x * x);
        }
    }
    __syncwarp();
    // prefix sums Q0, Q1, Q2 over cells < k, then the per-index terms of
    // E(A,B) = al[A] + be[B] + a*ga[B] + b*de[A]   (a = A*2^16, b = B*2^16)
    const long long c0 = sm.cnt[lane], c1 = sm.cnt[lane + 32];
    const long long x0 = (long long)sm.s1[lane], x1 = (long long)sm.s1[lane + 32];
    const long long y0 = (long long)sm.s2[lane], y1 = (long long)sm.s2[lane + 32];
    __syncwarp();
    sm.cnt[lane] = 0u;
    sm.cnt[lane + 32] = 0u;
    sm.s1[lane] = 0ull;
    sm.s1[lane + 32] = 0ull;
    sm.s2[lane] = 0ull;
    sm.s2[lane + 32] = 0ull;
    const long long ic0 = warp_inclusive_scan(c0, lane), ic1 = warp_inclusive_scan(c1, lane);
    const long long ix0 = warp_inclusive_scan(x0, lane), ix1 = warp_inclusive_scan(x1, lane);
    const long long iy0 = warp_inclusive_scan(y0, lane), iy1 = warp_inclusive_scan(y1, lane);
    const long long tc = __shfl_sync(kFull, ic0, 31), tx = __shfl_sync(kFull, ix0, 31), ty = __shfl_sync(kFull, iy0, 31);
    const long long tc_all = __shfl_sync(kFull, tc + ic1, 31);
    const long long tx_all = __shfl_sync(kFull, tx + ix1, 31);
    const long long ty_all = __shfl_sync(kFull, ty + iy1, 31);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int K = lane + 32 * h;
        const long long Q0 = h ? tc + ic1 - c1 : ic0 - c0;
        const long long Q1 = h ? tx + ix1 - x1 : ix0 - x0;
        const long long Q2 = h ? ty + iy1 - y1 : iy0 - y0;
        const unsigned long long k = (unsigned long long)K << kPbFBits;
        // modular 64-bit arithmetic: every E(A,B) fits in int64, so wrapped partial terms cancel
        const unsigned long long uQ0 = Q0, uQ1 = Q1, uQ2 = Q2;
        sm.al[K] = (long long)(k * k * uQ0 - 3ull * k * uQ1 + 2ull * uQ2);
        sm.be[K] = (long long)(3ull * k * uQ1 - 2ull * uQ2 + (unsigned long long)ty_all - 2ull * k * (unsigned long long)tx_all +
                               k * k * ((unsigned long long)tc_all - uQ0));
        sm.ga[K] = (long long)(uQ1 - k * uQ0);
        sm.de[K] = (long long)(k * uQ0 - uQ1);
    }
    __syncwarp();
    // exhaustive search over A < B, ties to the smallest (A, B)
    unsigned long long best_e = ~0ull;
    int best_ab = 0x7fffffff;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int B = lane + 32 * h;
        const unsigned long long bb = (unsigned long long)B << kPbFBits;
        const unsigned long long beB = sm.be[B], gaB = sm.ga[B];
        for (int A = 0; A < B; ++A) {
            const unsigned long long aa = (unsigned long long)A << kPbFBits;
            const unsigned long long e = (unsigned long long)sm.al[A] + beB + aa * gaB + bb * (unsigned long long)sm.de[A];
            const int ab = A * 64 + B;
            if ((long long)e < (long long)best_e || ((long long)e == (long long)best_e && ab < best_ab) || best_ab == 0x7fffffff) {
                best_e = e;
                best_ab = ab;
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const unsigned long long oe = __shfl_xor_sync(kFull, best_e, o);
        const int oab = __shfl_xor_sync(kFull, best_ab, o);
        if (oab != 0x7fffffff &&
            (best_ab == 0x7fffffff || (long long)oe < (long long)best_e || ((long long)oe == (long long)best_e && oab < best_ab))) {
            best_e = oe;
            best_ab = oab;
        }
    }
    const int A = best_ab >> 6, B = best_ab & 63;
    RoundPB rule;
    rule.a = grid_point(mn, mx, step, A);
    rule.b = grid_point(mn, mx, step, B);
    rule.rinv = __fdiv_rn(1.0f, __fsub_rn(rule.b, rule.a));
    rule.pa = A << kPbFBits;
    rule.pb = B << kPbFBits;
    emit<EPL, FUSED, true>(p, rule, beta, w, lane, vmask, v, u, pos, acc);
    store_table(p, w, beta, lane, lane == 0 ? rule.a : rule.b);
}

// ---------------------------------------------------------------------------------------------
// The kernel
// ---------------------------------------------------------------------------------------------
template <int EPL, int SCHEME, bool FUSED>
__global__ void __launch_bounds__(kWarpsPerCta * 32) k_warp(const __grid_constant__ KParams p)
{
    using Sm = typename SmemFor<SCHEME>::type;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int lane = threadIdx.x & 31;
    const int wib = threadIdx.x >> 5;
    Sm &sm = reinterpret_cast<Sm *>(smem_raw)[wib];
    if constexpr (SCHEME == GQ_ORQ) {
        for (int i = lane; i < 64 * 32; i += 32) sm.hist[i] = 0u;
    }
    if constexpr (SCHEME == GQ_BINGRAD_PB) {
        for (int i = lane; i < 64; i += 32) {
            sm.cnt[i] = 0u;
            sm.s1[i] = 0ull;
            sm.s2[i] = 0ull;
        }
    }
    __syncwarp();

    constexpr int D = 32 * EPL;
    const int64_t first = (int64_t)blockIdx.x * kWarpsPerCta + wib;
    const int64_t stride = (int64_t)gridDim.x * kWarpsPerCta;
    for (int64_t beta = first; beta < p.nb; beta += stride) {
        const int nvalid = (beta == p.nb - 1) ? p.tail : D;
        const bool full = nvalid == D;
        uint32_t vmask = 0;
#pragma unroll
        for (int t = 0; t < EPL; ++t) vmask |= (slot_elem(t, lane) < nvalid ? 1u : 0u) << t;
        float acc[EPL];
#pragma unroll
        for (int t = 0; t < EPL; ++t) acc[t] = 0.0f;
        for (int w = 0; w < p.W; ++w) {
            float v[EPL];
            load_bucket<EPL>(p.g[w], p.r[w], beta * D, nvalid, full, lane, v);
            // non-finite input: flag it (NaN-propagating max of |v|)
            float am = 0.0f;
#pragma unroll
            for (int t = 0; t < EPL; ++t)
                if ((vmask >> t) & 1u) am = fmax_nan(am, fabsf(v[t]));
            am = warp_max_nan(am);
            if (!(am <= FLT_MAX) && lane == 0) atomicOr(p.status, kStatusNonFinite);
            // clip to +-c*sigma
            float u[EPL];
            if (p.clip > 0.0f) {
                float T = 0.0f;
                if (am > 0.0f) {
                    const int e = 20 - fexpo(am);
                    const double sc = pow2d(e);
                    long long sx = 0, sxx = 0;
#pragma unroll
                    for (int t = 0; t < EPL; ++t)
                        if ((vmask >> t) & 1u) {
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
                fit_qsgd<EPL, FUSED>(p, sm, beta, w, lane, full, vmask, v, u, acc);
            else if constexpr (SCHEME == GQ_ORQ)
                fit_orq<EPL, FUSED>(p, sm, beta, w, lane, full, vmask, v, u, acc);
            else if constexpr (SCHEME == GQ_BINGRAD_B)
                fit_bingrad_b<EPL, FUSED>(p, sm, beta, w, lane, full, vmask, nvalid, v, u, acc);
            else
                fit_bingrad_pb<EPL, FUSED>(p, sm, beta, w, lane, full, vmask, v, u, acc);
        }
        if constexpr (FUSED) {
            float *ab = p.avg + beta * D;
            if (full) {
#pragma unroll
                for (int m = 0; m < EPL / 4; ++m)
                    __stcs(reinterpret_cast<float4 *>(ab + 128 * m + 4 * lane),
                           make_float4(__fmul_rn(acc[4 * m], p.inv_w), __fmul_rn(acc[4 * m + 1], p.inv_w),
                                       __fmul_rn(acc[4 * m + 2], p.inv_w), __fmul_rn(acc[4 * m + 3], p.inv_w)));
            } else {
#pragma unroll
                for (int t = 0; t < EPL; ++t)
                    if ((vmask >> t) & 1u) ab[slot_elem(t, lane)] = __fmul_rn(acc[t], p.inv_w);
            }
        }
    }
}

template <int EPL, int SCHEME, bool FUSED>
cudaError_t launch_one(const KParams &p, cudaStream_t stream)
{
    using Sm = typename SmemFor<SCHEME>::type;
    auto kern = k_warp<EPL, SCHEME, FUSED>;
    const size_t smem = sizeof(Sm) * kWarpsPerCta;
    static bool configured = false;  // per instantiation; attribute setting is idempotent
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    int dev = 0, sms = 0, per_sm = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kWarpsPerCta * 32, smem);
    if (per_sm < 1) per_sm = 1;
    const int64_t need = (p.nb + kWarpsPerCta - 1) / kWarpsPerCta;
    const int64_t cap = (int64_t)sms * per_sm;
    const int grid = (int)(need < cap ? need : cap);
    if (grid <= 0) return cudaSuccess;
    kern<<<grid, kWarpsPerCta * 32, smem, stream>>>(p);
    return cudaGetLastError();
}

template <int EPL, bool FUSED>
cudaError_t dispatch_scheme(const KParams &p, cudaStream_t stream)
{
    switch (p.scheme) {
    case GQ_QSGD:
    case GQ_TERNGRAD: return launch_one<EPL, GQ_QSGD, FUSED>(p, stream);
    case GQ_BINGRAD_B: return launch_one<EPL, GQ_BINGRAD_B, FUSED>(p, stream);
    case GQ_BINGRAD_PB: return launch_one<EPL, GQ_BINGRAD_PB, FUSED>(p, stream);
    default: return launch_one<EPL, GQ_ORQ, FUSED>(p, stream);
    }
}

template <bool FUSED>
cudaError_t dispatch_bucket(const KParams &p, cudaStream_t stream)
{
    switch (p.d) {
    case 128: return dispatch_scheme<4, FUSED>(p, stream);
    case 256: return dispatch_scheme<8, FUSED>(p, stream);
    default: return dispatch_scheme<16, FUSED>(p, stream);
    }
}

}  // namespace

cudaError_t launch_warp_encode(const KParams &p, bool fused, cudaStream_t stream)
{
    return fused ? dispatch_bucket<true>(p, stream) : dispatch_bucket<false>(p, stream);
}

}  // namespace gq
