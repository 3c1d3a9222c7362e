// gq_decode.cu -- Dequantize + Aggregate: avg[i] = (sum_w level_w(code_w[i])) * (1/W).
//
// A warp item is CPI consecutive 128-element chunks of one bucket (CPI = min(d, 512) / 128),
// grid-stride over the items of the vector.  Lane l decodes elements 4l .. 4l+3 of each chunk:
// per worker it needs the one or two words holding its four codes in each chunk (codes are
// packed densely, b bits each, in element order).  A worker's code and level-table addresses
// are formed once per item; the chunks then sit at fixed offsets from them.  The level lookup
// is a register shuffle within segments of 2^b lanes: every segment holds the bucket's level
// table in its first L lanes, and a shuffle of width 2^b takes its source lane modulo 2^b, so
// the code needs no masking (8-bit codes of the QSGD family look their ratio up in a shared
// table instead).  For 1, 2, 4 and 8 workers the item's code words of every worker come into
// shared memory by bulk copies one item ahead (k_decode_staged); for other counts the loads of a
// group of workers are issued together before any of them is used (k_decode).  The sum runs in
// worker order in registers and the average is written once, with 16-byte stores.
#include "gq_bases.cuh"
#include "gq_device.cuh"

namespace gq {
namespace {

constexpr int kDecodeWarps = 4;

// Any worker count (the counts 1, 2, 4 and 8 go to k_decode_staged below): the loads of four
// workers are issued before any of them is used.
template <bool QSGD, int BITS, int CPI>
__global__ void __launch_bounds__(kDecodeWarps * 32) k_decode(const __grid_constant__ KParams p)
{
    constexpr int kDecodeGroup = 4;  // workers whose loads are in flight together
    const int W = p.W;
    constexpr int kWidth = 1 << BITS;
    constexpr int kChunkWords = 4 * BITS;  // words of one chunk's codes
    const int lane = threadIdx.x & 31;
    const int slot = lane & (kWidth - 1);  // this lane's place in its 2^b-lane segment
    const int64_t nitems = (p.n + 128 * CPI - 1) / (128 * CPI);
    const int64_t first = (int64_t)blockIdx.x * kDecodeWarps + (threadIdx.x >> 5);
    const int64_t stride = (int64_t)gridDim.x * kDecodeWarps;
    const int log2d = 31 - __clz(p.d);
    const int bitoff = 4 * BITS * lane, wi = bitoff >> 5, sh = bitoff & 31;
    const bool cross = sh + 4 * BITS > 32;  // the field crosses a word boundary (b = 3 only)
    const bool has_level = slot < p.L;
    const float qr = (QSGD && slot < p.s) ? p.qratio[slot] : 0.0f;
    // 8-bit codes (QSGD family, 129 .. 256 levels): the level ratios in shared memory
    __shared__ float qtab[BITS == 8 ? 256 : 1];
    if (BITS == 8) {
        for (int k = threadIdx.x; k < p.s; k += blockDim.x) qtab[k] = p.qratio[k];
        __syncthreads();
    }
    for (int64_t it = first; it < nitems; it += stride) {
        const int64_t e0 = it * (128 * CPI);
        const int64_t bk = e0 >> log2d;
        // code word of this lane in the item's first chunk, and the bucket's level-table entry
        const int64_t wbase = bk * p.codes_words + (int64_t)((e0 & (p.d - 1)) >> 7) * kChunkWords + wi;
        const int64_t tbase = QSGD ? bk : bk * p.L + slot;
        int nlive = (int)((p.n - e0 + 127) >> 7);
        nlive = nlive < CPI ? nlive : CPI;
        float acc[CPI][4];
#pragma unroll
        for (int c = 0; c < CPI; ++c) acc[c][0] = acc[c][1] = acc[c][2] = acc[c][3] = 0.0f;
        for (int w0 = 0; w0 < W; w0 += kDecodeGroup) {
            uint32_t x[kDecodeGroup][CPI], y[kDecodeGroup][CPI];
            float lv[kDecodeGroup];
#pragma unroll
            for (int k = 0; k < kDecodeGroup; ++k) {
                lv[k] = 0.0f;
#pragma unroll
                for (int c = 0; c < CPI; ++c) x[k][c] = y[k][c] = 0u;
                if (w0 + k < W) {
                    const unsigned char *msg = p.msg[w0 + k];
                    const uint32_t *cw = reinterpret_cast<const uint32_t *>(msg) + wbase;
#pragma unroll
                    for (int c = 0; c < CPI; ++c) {
                        if (c < nlive) {
                            x[k][c] = __ldg(cw + c * kChunkWords);
                            if (BITS == 3 && cross) y[k][c] = __ldg(cw + c * kChunkWords + 1);
                        }
                    }
                    if (QSGD || has_level) lv[k] = __ldg(reinterpret_cast<const float *>(msg + p.levels_off) + tbase);
                }
            }
#pragma unroll
            for (int k = 0; k < kDecodeGroup; ++k) {
                if (BITS == 8 && w0 + k < W) {
#pragma unroll
                    for (int c = 0; c < CPI; ++c)
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            acc[c][e] = __fadd_rn(acc[c][e], __fmul_rn(lv[k], qtab[(x[k][c] >> (8 * e)) & 0xffu]));
                } else if (w0 + k < W) {
                    const float level = QSGD ? __fmul_rn(lv[k], qr) : lv[k];
#pragma unroll
                    for (int c = 0; c < CPI; ++c) {
                        uint32_t f = x[k][c] >> sh;
                        if (BITS == 3 && cross) f |= y[k][c] << (32 - sh);
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            acc[c][e] = __fadd_rn(acc[c][e], __shfl_sync(kFull, level, (int)(f >> (BITS * e)), kWidth));
                    }
                }
            }
        }
#pragma unroll
        for (int c = 0; c < CPI; ++c) {
            const int64_t e = e0 + 128 * c + 4 * lane;
            if (e + 3 < p.n) {
                __stcs(reinterpret_cast<float4 *>(p.avg + e),
                       make_float4(__fmul_rn(acc[c][0], p.inv_w), __fmul_rn(acc[c][1], p.inv_w),
                                   __fmul_rn(acc[c][2], p.inv_w), __fmul_rn(acc[c][3], p.inv_w)));
            } else {
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    if (e + q < p.n) p.avg[e + q] = __fmul_rn(acc[c][q], p.inv_w);
            }
        }
    }
}

// The same decode and sum for a worker count known at compile time (1, 2, 4 or 8), with each item's
// code words staged in the warp's shared memory: one 1-D bulk copy (into this CTA only) per worker and
// item, one item ahead on a two-stage mbarrier pipeline, so that the lanes read their code words
// from shared memory instead of waiting on global loads.  The level tables (a few floats per
// worker and bucket, not 16-byte aligned) are loaded into registers one item ahead.  An item's
// copy spans its CPI chunks of the bucket's codes, which exist in full even when the vector ends
// inside them; the message and every chunk start on 16 bytes.  Every wait is bounded: a copy that
// does not land in time sets kStatusTimeout, the warp waits (bounded) for its other copy in
// flight and stops.
template <bool QSGD, int BITS, int CPI, int WK>
struct DecodeStage {
    static constexpr int kChunkWords = BITS == 8 ? 32 : 4 * BITS;
    static constexpr int kItemWords = CPI * kChunkWords;
    uint32_t w[2][WK][kItemWords];
    unsigned long long bar[2];
};

template <bool QSGD, int BITS, int CPI, int WK>
__global__ void __launch_bounds__(kDecodeWarps * 32) k_decode_staged(const __grid_constant__ KParams p)
{
    using Stage = DecodeStage<QSGD, BITS, CPI, WK>;
    constexpr int kWidth = BITS == 8 ? 32 : 1 << BITS;
    constexpr int kChunkWords = Stage::kChunkWords;
    constexpr int kItemWords = Stage::kItemWords;
    constexpr unsigned kItemBytes = kItemWords * 4u;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
    Stage &sm = reinterpret_cast<Stage *>(smem_raw)[wib];
    const int slot = lane & (kWidth - 1);
    const int64_t nitems = (p.n + 128 * CPI - 1) / (128 * CPI);
    const int64_t first = (int64_t)blockIdx.x * kDecodeWarps + wib;
    const int64_t stride = (int64_t)gridDim.x * kDecodeWarps;
    const int log2d = 31 - __clz(p.d);
    const int bitoff = 4 * (BITS == 8 ? 8 : BITS) * lane, wi = bitoff >> 5, sh = bitoff & 31;
    const bool cross = BITS == 3 && sh + 12 > 32;  // the field crosses a word boundary (b = 3 only)
    const bool has_level = slot < p.L;
    const float qr = (QSGD && slot < p.s) ? p.qratio[slot] : 0.0f;
    __shared__ float qtab[BITS == 8 ? 256 : 1];
    if (BITS == 8) {
        for (int k = threadIdx.x; k < p.s; k += blockDim.x) qtab[k] = p.qratio[k];
        __syncthreads();
    }
    if (first >= nitems) return;
    if (lane == 0) {
        mbar_init(&sm.bar[0], 1);
        mbar_init(&sm.bar[1], 1);
        fence_barrier_init();
    }
    __syncwarp();
    auto issue = [&](int64_t it, int k) {  // lane 0: the item's code words of every worker
        const int64_t e0 = it * (128 * CPI);
        const int64_t off = (e0 >> log2d) * p.codes_words + (int64_t)((e0 & (p.d - 1)) >> 7) * kChunkWords;
        fence_proxy_async();
        mbar_arrive_expect_tx(&sm.bar[k], WK * kItemBytes);
#pragma unroll
        for (int w = 0; w < WK; ++w)
            bulk_load(sm.w[k][w], reinterpret_cast<const uint32_t *>(p.msg[w]) + off, kItemBytes, &sm.bar[k]);
    };
    auto levels = [&](int64_t it, float (&lv)[WK]) {
        const int64_t bk = (it * (128 * CPI)) >> log2d;
        const int64_t tbase = QSGD ? bk : bk * p.L + slot;
#pragma unroll
        for (int w = 0; w < WK; ++w)
            lv[w] = (QSGD || has_level) ? __ldg(reinterpret_cast<const float *>(p.msg[w] + p.levels_off) + tbase) : 0.0f;
    };
    if (lane == 0) issue(first, 0);
    float lv[WK];
    levels(first, lv);
    unsigned parity = 0;  // bit k: phase parity awaited next on stage k
    int k = 0;
    for (int64_t it = first; it < nitems; it += stride) {
        const int64_t nxt = it + stride;
        if (lane == 0 && nxt < nitems) issue(nxt, k ^ 1);
        if (!mbar_wait_warp(&sm.bar[k], (parity >> k) & 1u)) {
            // report it, give both copies still in flight one more bounded wait so that none can
            // land after the warp has left, and stop
            if (lane == 0) atomicOr(p.status, kStatusTimeout);
            mbar_wait_warp(&sm.bar[k], (parity >> k) & 1u);
            if (nxt < nitems) mbar_wait_warp(&sm.bar[k ^ 1], (parity >> (k ^ 1)) & 1u);
            return;
        }
        parity ^= 1u << k;
        float lvn[WK];
        if (nxt < nitems) levels(nxt, lvn);
        const int64_t e0 = it * (128 * CPI);
        int nlive = (int)((p.n - e0 + 127) >> 7);
        nlive = nlive < CPI ? nlive : CPI;
        float acc[CPI][4];
#pragma unroll
        for (int c = 0; c < CPI; ++c) acc[c][0] = acc[c][1] = acc[c][2] = acc[c][3] = 0.0f;
#pragma unroll
        for (int w = 0; w < WK; ++w) {
            const uint32_t *cw = sm.w[k][w];
            if (BITS == 8) {
#pragma unroll
                for (int c = 0; c < CPI; ++c) {
                    const uint32_t x = cw[c * kChunkWords + lane];
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        acc[c][e] = __fadd_rn(acc[c][e], __fmul_rn(lv[w], qtab[(x >> (8 * e)) & 0xffu]));
                }
            } else {
                const float level = QSGD ? __fmul_rn(lv[w], qr) : lv[w];
#pragma unroll
                for (int c = 0; c < CPI; ++c) {
                    uint32_t f = cw[c * kChunkWords + wi] >> sh;
                    if (cross) f |= cw[c * kChunkWords + wi + 1] << (32 - sh);
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        acc[c][e] = __fadd_rn(acc[c][e], __shfl_sync(kFull, level, (int)(f >> (BITS * e)), kWidth));
                }
            }
        }
#pragma unroll
        for (int c = 0; c < CPI; ++c) {
            const int64_t e = e0 + 128 * c + 4 * lane;
            if (c < nlive && e + 3 < p.n) {
                __stcs(reinterpret_cast<float4 *>(p.avg + e),
                       make_float4(__fmul_rn(acc[c][0], p.inv_w), __fmul_rn(acc[c][1], p.inv_w),
                                   __fmul_rn(acc[c][2], p.inv_w), __fmul_rn(acc[c][3], p.inv_w)));
            } else if (c < nlive) {
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    if (e + q < p.n) p.avg[e + q] = __fmul_rn(acc[c][q], p.inv_w);
            }
        }
        __syncwarp();  // every lane has read stage k before it is filled again
#pragma unroll
        for (int w = 0; w < WK; ++w) lv[w] = lvn[w];
        k ^= 1;
    }
}

// Base-s messages (s = 3, 5, 9; d <= 512): the same items and sum, with each lane's four codes
// of a chunk taken from the one or two base-s groups that hold them (base_run4); the code words
// of kBaseGroup workers are loaded before any is decoded.
constexpr int kBaseGroup = 4;
template <bool QSGD, int S, int CPI>
__global__ void __launch_bounds__(kDecodeWarps * 32) k_decode_base(const __grid_constant__ KParams p)
{
    constexpr int BITS = S == 3 ? 2 : S == 5 ? 3 : 4;  // the level lookup's segment: 2^b lanes
    constexpr int kWidth = 1 << BITS;
    const int lane = threadIdx.x & 31;
    const int slot = lane & (kWidth - 1);
    const int64_t nitems = (p.n + 128 * CPI - 1) / (128 * CPI);
    const int64_t first = (int64_t)blockIdx.x * kDecodeWarps + (threadIdx.x >> 5);
    const int64_t stride = (int64_t)gridDim.x * kDecodeWarps;
    const int log2d = 31 - __clz(p.d);
    const int nw = (int)p.codes_words;
    const bool has_level = slot < p.L;
    const float qr = (QSGD && slot < p.s) ? p.qratio[slot] : 0.0f;
    __shared__ DigitTab<S> tab;
    build_digit_tab<S>(tab);
    __syncthreads();
    for (int64_t it = first; it < nitems; it += stride) {
        const int64_t e0 = it * (128 * CPI);
        const int64_t bk = e0 >> log2d;
        const int eb = (int)(e0 & (p.d - 1)) + 4 * lane;  // this lane's first element in the bucket
        const int64_t tbase = QSGD ? bk : bk * p.L + slot;
        int nlive = (int)((p.n - e0 + 127) >> 7);
        nlive = nlive < CPI ? nlive : CPI;
        float acc[CPI][4];
        BasePos ps[CPI];
#pragma unroll
        for (int c = 0; c < CPI; ++c) {
            acc[c][0] = acc[c][1] = acc[c][2] = acc[c][3] = 0.0f;
            ps[c] = base_pos<S>(eb + 128 * c);
        }
        // the loads of a group of workers go out before any is used
        for (int w0 = 0; w0 < p.W; w0 += kBaseGroup) {
            uint32_t lo[kBaseGroup][CPI], hi[kBaseGroup][CPI];
            float lv[kBaseGroup];
#pragma unroll
            for (int k = 0; k < kBaseGroup; ++k) {
                lv[k] = 0.0f;
#pragma unroll
                for (int c = 0; c < CPI; ++c) lo[k][c] = hi[k][c] = 0u;
                if (w0 + k < p.W) {
                    const unsigned char *msg = p.msg[w0 + k];
                    const uint32_t *words = reinterpret_cast<const uint32_t *>(msg) + bk * p.codes_words;
#pragma unroll
                    for (int c = 0; c < CPI; ++c) {
                        if (c < nlive) {
                            lo[k][c] = __ldg(words + ps[c].wi);
                            if (ps[c].wi + 1 < nw) hi[k][c] = __ldg(words + ps[c].wi + 1);
                        }
                    }
                    if (QSGD || has_level) lv[k] = __ldg(reinterpret_cast<const float *>(msg + p.levels_off) + tbase);
                }
            }
#pragma unroll
            for (int k = 0; k < kBaseGroup; ++k) {
                if (w0 + k < p.W) {
                    const float level = QSGD ? __fmul_rn(lv[k], qr) : lv[k];
#pragma unroll
                    for (int c = 0; c < CPI; ++c) {
                        const uint32_t run = base_run4<S>(tab, lo[k][c], hi[k][c], ps[c]);
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            acc[c][e] = __fadd_rn(acc[c][e], __shfl_sync(kFull, level, (int)(run >> (4 * e)), kWidth));
                    }
                }
            }
        }
#pragma unroll
        for (int c = 0; c < CPI; ++c) {
            const int64_t e = e0 + 128 * c + 4 * lane;
            if (e + 3 < p.n) {
                __stcs(reinterpret_cast<float4 *>(p.avg + e),
                       make_float4(__fmul_rn(acc[c][0], p.inv_w), __fmul_rn(acc[c][1], p.inv_w),
                                   __fmul_rn(acc[c][2], p.inv_w), __fmul_rn(acc[c][3], p.inv_w)));
            } else {
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    if (e + q < p.n) p.avg[e + q] = __fmul_rn(acc[c][q], p.inv_w);
            }
        }
    }
}

// Base-s words staged like the dense ones (1, 2, 4 or 8 workers, d <= 512 so that an item is a
// bucket).  A bucket's nw words start on any word, so each worker's copy takes the 16-byte units
// that hold them, at most nw + 6 words (the codes region ends on 16 bytes), and the lanes index
// from the bucket's offset in them.  A lane's second word is read only inside the bucket, as in
// k_decode_base.
template <int S, int CPI>
struct BaseStageDims {
    static constexpr int kWords = ((CPI * 128 + BaseS<S>::g - 1) / BaseS<S>::g * BaseS<S>::B + 31) / 32;
    static constexpr int kStageWords = (kWords + 6 + 3) & ~3;
};
template <int S, int CPI, int WK>
struct BaseDecodeStage {
    uint32_t w[2][WK][BaseStageDims<S, CPI>::kStageWords];
    unsigned long long bar[2];
};

template <bool QSGD, int S, int CPI, int WK>
__global__ void __launch_bounds__(kDecodeWarps * 32) k_decode_base_staged(const __grid_constant__ KParams p)
{
    using Stage = BaseDecodeStage<S, CPI, WK>;
    constexpr int BITS = S == 3 ? 2 : S == 5 ? 3 : 4;  // the level lookup's segment: 2^b lanes
    constexpr int kWidth = 1 << BITS;
    constexpr int nw = BaseStageDims<S, CPI>::kWords;  // the bucket's words (the host checked p.codes_words)
    extern __shared__ __align__(128) unsigned char smem_raw[];
    const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
    Stage &sm = reinterpret_cast<Stage *>(smem_raw)[wib];
    const int slot = lane & (kWidth - 1);
    const int64_t nitems = (p.n + 128 * CPI - 1) / (128 * CPI);
    const int64_t first = (int64_t)blockIdx.x * kDecodeWarps + wib;
    const int64_t stride = (int64_t)gridDim.x * kDecodeWarps;
    const bool has_level = slot < p.L;
    const float qr = (QSGD && slot < p.s) ? p.qratio[slot] : 0.0f;
    __shared__ DigitTab<S> tab;
    build_digit_tab<S>(tab);
    __syncthreads();
    if (first >= nitems) return;
    if (lane == 0) {
        mbar_init(&sm.bar[0], 1);
        mbar_init(&sm.bar[1], 1);
        fence_barrier_init();
    }
    __syncwarp();
    BasePos ps[CPI];
#pragma unroll
    for (int c = 0; c < CPI; ++c) ps[c] = base_pos<S>(4 * lane + 128 * c);
    auto span = [&](int64_t it, int64_t &a0, int &off, int &words) {
        const int64_t sw = it * nw;  // item = bucket
        a0 = sw & ~int64_t(3);
        off = (int)(sw - a0);
        words = (int)(((sw + nw + 3) & ~int64_t(3)) - a0);
    };
    auto issue = [&](int64_t it, int k) {  // lane 0
        int64_t a0;
        int off, words;
        span(it, a0, off, words);
        fence_proxy_async();
        mbar_arrive_expect_tx(&sm.bar[k], (unsigned)(WK * words * 4));
#pragma unroll
        for (int w = 0; w < WK; ++w)
            bulk_load(sm.w[k][w], reinterpret_cast<const uint32_t *>(p.msg[w]) + a0, (unsigned)(words * 4), &sm.bar[k]);
    };
    auto levels = [&](int64_t it, float (&lv)[WK]) {
        const int64_t tbase = QSGD ? it : it * p.L + slot;
#pragma unroll
        for (int w = 0; w < WK; ++w)
            lv[w] = (QSGD || has_level) ? __ldg(reinterpret_cast<const float *>(p.msg[w] + p.levels_off) + tbase) : 0.0f;
    };
    if (lane == 0) issue(first, 0);
    float lv[WK];
    levels(first, lv);
    unsigned parity = 0;
    int k = 0;
    for (int64_t it = first; it < nitems; it += stride) {
        const int64_t nxt = it + stride;
        if (lane == 0 && nxt < nitems) issue(nxt, k ^ 1);
        if (!mbar_wait_warp(&sm.bar[k], (parity >> k) & 1u)) {
            if (lane == 0) atomicOr(p.status, kStatusTimeout);
            mbar_wait_warp(&sm.bar[k], (parity >> k) & 1u);
            if (nxt < nitems) mbar_wait_warp(&sm.bar[k ^ 1], (parity >> (k ^ 1)) & 1u);
            return;
        }
        parity ^= 1u << k;
        float lvn[WK];
        if (nxt < nitems) levels(nxt, lvn);
        const int64_t e0 = it * (128 * CPI);
        int nlive = (int)((p.n - e0 + 127) >> 7);
        nlive = nlive < CPI ? nlive : CPI;
        int64_t a0;
        int off, words;
        span(it, a0, off, words);
        float acc[CPI][4];
#pragma unroll
        for (int c = 0; c < CPI; ++c) acc[c][0] = acc[c][1] = acc[c][2] = acc[c][3] = 0.0f;
#pragma unroll
        for (int w = 0; w < WK; ++w) {
            const uint32_t *bw = sm.w[k][w] + off;
            const float level = QSGD ? __fmul_rn(lv[w], qr) : lv[w];
#pragma unroll
            for (int c = 0; c < CPI; ++c) {
                const uint32_t lo = bw[ps[c].wi];
                const uint32_t hi = ps[c].wi + 1 < nw ? bw[ps[c].wi + 1] : 0u;
                const uint32_t run = base_run4<S>(tab, lo, hi, ps[c]);
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    acc[c][e] = __fadd_rn(acc[c][e], __shfl_sync(kFull, level, (int)(run >> (4 * e)), kWidth));
            }
        }
#pragma unroll
        for (int c = 0; c < CPI; ++c) {
            const int64_t e = e0 + 128 * c + 4 * lane;
            if (c < nlive && e + 3 < p.n) {
                __stcs(reinterpret_cast<float4 *>(p.avg + e),
                       make_float4(__fmul_rn(acc[c][0], p.inv_w), __fmul_rn(acc[c][1], p.inv_w),
                                   __fmul_rn(acc[c][2], p.inv_w), __fmul_rn(acc[c][3], p.inv_w)));
            } else if (c < nlive) {
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    if (e + q < p.n) p.avg[e + q] = __fmul_rn(acc[c][q], p.inv_w);
            }
        }
        __syncwarp();  // every lane has read stage k before it is filled again
#pragma unroll
        for (int w = 0; w < WK; ++w) lv[w] = lvn[w];
        k ^= 1;
    }
}

template <class K>
cudaError_t launch_items(K kern, const KParams &p, int cpi, size_t smem, cudaStream_t stream)
{
    int sms = 0, per_sm = 0;
    const cudaError_t e = kernel_occupancy(reinterpret_cast<const void *>(kern), kDecodeWarps * 32, smem, &per_sm, &sms);
    if (e != cudaSuccess) return e;
    const int64_t nitems = (p.n + 128 * cpi - 1) / (128 * cpi);
    const int64_t need = (nitems + kDecodeWarps - 1) / kDecodeWarps;
    const int64_t cap = (int64_t)sms * per_sm;
    const int grid = (int)(need < cap ? need : cap);
    if (grid <= 0) return cudaSuccess;
    kern<<<grid, kDecodeWarps * 32, smem, stream>>>(p);
    return cudaGetLastError();
}

template <bool QSGD, int BITS, int CPI, int WK>
cudaError_t launch_staged(const KParams &p, cudaStream_t stream)
{
    return launch_items(k_decode_staged<QSGD, BITS, CPI, WK>, p, CPI,
                        sizeof(DecodeStage<QSGD, BITS, CPI, WK>) * kDecodeWarps, stream);
}

template <bool QSGD, int BITS, int CPI>
cudaError_t launch(const KParams &p, cudaStream_t stream)
{
    if (p.W == 8) return launch_staged<QSGD, BITS, CPI, 8>(p, stream);
    if (p.W == 4) return launch_staged<QSGD, BITS, CPI, 4>(p, stream);
    if (p.W == 2) return launch_staged<QSGD, BITS, CPI, 2>(p, stream);
    if (p.W == 1) return launch_staged<QSGD, BITS, CPI, 1>(p, stream);
    return launch_items(k_decode<QSGD, BITS, CPI>, p, CPI, 0, stream);
}

// Chunks per item: a whole bucket for d = 128, 256, four chunks of it for larger buckets.
template <bool QSGD, int BITS>
cudaError_t launch_cpi(const KParams &p, cudaStream_t stream)
{
    switch (p.d) {
    case 128: return launch<QSGD, BITS, 1>(p, stream);
    case 256: return launch<QSGD, BITS, 2>(p, stream);
    default: return launch<QSGD, BITS, 4>(p, stream);
    }
}

template <bool QSGD, int S, int CPI>
cudaError_t launch_base(const KParams &p, cudaStream_t stream)
{
    if (p.codes_words == BaseStageDims<S, CPI>::kWords && CPI * 128 == p.d) {
        switch (p.W) {
        case 8: return launch_items(k_decode_base_staged<QSGD, S, CPI, 8>, p, CPI, sizeof(BaseDecodeStage<S, CPI, 8>) * kDecodeWarps, stream);
        case 4: return launch_items(k_decode_base_staged<QSGD, S, CPI, 4>, p, CPI, sizeof(BaseDecodeStage<S, CPI, 4>) * kDecodeWarps, stream);
        case 2: return launch_items(k_decode_base_staged<QSGD, S, CPI, 2>, p, CPI, sizeof(BaseDecodeStage<S, CPI, 2>) * kDecodeWarps, stream);
        case 1: return launch_items(k_decode_base_staged<QSGD, S, CPI, 1>, p, CPI, sizeof(BaseDecodeStage<S, CPI, 1>) * kDecodeWarps, stream);
        default: break;
        }
    }
    auto kern = k_decode_base<QSGD, S, CPI>;
    int dev = 0, sms = 0, per_sm = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kDecodeWarps * 32, 0);
    if (per_sm < 1) per_sm = 1;
    const int64_t nitems = (p.n + 128 * CPI - 1) / (128 * CPI);
    const int64_t need = (nitems + kDecodeWarps - 1) / kDecodeWarps;
    const int64_t cap = (int64_t)sms * per_sm;
    const int grid = (int)(need < cap ? need : cap);
    if (grid <= 0) return cudaSuccess;
    kern<<<grid, kDecodeWarps * 32, 0, stream>>>(p);
    return cudaGetLastError();
}

template <bool QSGD, int S>
cudaError_t launch_base_cpi(const KParams &p, cudaStream_t stream)
{
    switch (p.d) {
    case 128: return launch_base<QSGD, S, 1>(p, stream);
    case 256: return launch_base<QSGD, S, 2>(p, stream);
    default: return launch_base<QSGD, S, 4>(p, stream);
    }
}

template <bool QSGD>
cudaError_t launch_base_s(const KParams &p, cudaStream_t stream)
{
    switch (p.fmt_s) {
    case 3: return launch_base_cpi<QSGD, 3>(p, stream);
    case 5: return launch_base_cpi<QSGD, 5>(p, stream);
    case 9: return launch_base_cpi<QSGD, 9>(p, stream);
    default: return cudaErrorInvalidValue;
    }
}

template <bool QSGD>
cudaError_t launch_bits(const KParams &p, cudaStream_t stream)
{
    switch (p.bits) {
    case 1: return launch_cpi<QSGD, 1>(p, stream);
    case 2: return launch_cpi<QSGD, 2>(p, stream);
    case 3: return launch_cpi<QSGD, 3>(p, stream);
    case 4: return launch_cpi<QSGD, 4>(p, stream);
    default:
        if constexpr (QSGD) return launch_cpi<QSGD, 8>(p, stream);  // 8-bit codes: QSGD family only
        else return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_decode(const KParams &p, cudaStream_t stream)
{
    const bool qsgd =
        p.scheme == GQ_QSGD || p.scheme == GQ_TERNGRAD || p.scheme == GQ_QSGD_NEAREST || p.scheme == GQ_QSGD_L2;
    if (p.fmt_s != 0) return qsgd ? launch_base_s<true>(p, stream) : launch_base_s<false>(p, stream);
    return qsgd ? launch_bits<true>(p, stream) : launch_bits<false>(p, stream);
}

}  // namespace gq
