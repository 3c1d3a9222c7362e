// gq_cta.cu -- quantization of large buckets (d = 1024 .. 32768): one CTA per bucket index.
//
// The CTA (NW warps: 8, or 16 for d >= 16384) walks the items (bucket, worker) of its bucket
// index in worker order; W = 1 for gq_encode and gq_quant_error.  For each item it stages
// v = g + r in shared memory (16-byte coalesced evict-first loads; the next item's g and r are
// brought into L2 by bulk prefetches while this one is processed), reduces the bucket
// statistics across its warps, fits the levels and then rounds, packs and writes the residual
// chunk by chunk (warp k takes the 128-element chunks k, k + NW, ...).  In the fused step the
// dequantized values are added, in worker order, to a running sum kept on chip: in shared
// memory when it fits beside the staged bucket (d <= 8192), else in the average's own slice,
// which stays in L2 while the CTA works on the bucket; the last worker writes the average.
// Fits:
//   QSGD / TernGrad : block max of |u|
//   ORQ             : per warp, the packed 8-column histogram of the register path (one shared
//                     atomic per value), reduced every 512 values into the warp's cell totals;
//                     warp 0 sums the warps' totals and runs the greedy
//   BinGrad-b       : sort of u in place (runs of 512 sorted by the warps in registers, then
//                     merged: the stages of distance >= 512 in shared memory, the rest in
//                     registers), exact int64 block scan, argmax of J(k) screened in binary32;
//                     the final pass re-reads g and r because the sort overwrote v
//   BinGrad-pb      : BinGrad-b's levels first (as above: the final pass re-reads g and r),
//                     which bound the pair from inside; the cells' prefix moments read off the
//                     sorted values; per column B the least E over the admissible A (convex in A)
// The per-element rules and the chunk step are those of the register path (gq_round.cuh), so
// both paths produce identical codes.
#include "gq_round.cuh"

namespace gq {
namespace {

template <int NW>
struct alignas(16) CtaShared {
    float redf[3][NW];
    long long redl[3][NW];
    double redd[NW];
    double rede[3][NW];
    int redi[NW];
    unsigned long long cs1[64], cs2[64];  // block histogram: sum of positions, of squares
    unsigned int ccnt[64];                // block histogram: count
    long long P1[64];
    int P0[64];
    long long al[64], be[64], ga[64], de[64];
    float4 ctab[64];
    float2 pair[GQ_MAX_QSGD_LEVELS];
    float lev[16];
    float rinv[16];
    float bcast_f[4];
    long long bcast_l[2];
};

// --- block reductions (every thread receives the result) -------------------------------------
template <int NW>
__device__ float block_max(float x, CtaShared<NW> &sh, int slot)
{
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    x = warp_max(x);
    if (lane == 0) sh.redf[slot][wid] = x;
    __syncthreads();
    float y = sh.redf[slot][lane & (NW - 1)];
    y = warp_max(y);
    __syncthreads();
    return y;
}
template <int NW>
__device__ float block_min(float x, CtaShared<NW> &sh, int slot)
{
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    x = warp_min(x);
    if (lane == 0) sh.redf[slot][wid] = x;
    __syncthreads();
    float y = sh.redf[slot][lane & (NW - 1)];
    y = warp_min(y);
    __syncthreads();
    return y;
}
template <int NW>
__device__ long long block_sum(long long x, CtaShared<NW> &sh, int slot)
{
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    x = warp_sum(x);
    if (lane == 0) sh.redl[slot][wid] = x;
    __syncthreads();
    long long y = lane < NW ? sh.redl[slot][lane] : 0ll;
    y = warp_sum(y);
    __syncthreads();
    return y;
}

// The three staging statistics in one exchange: NaN-propagating max |v|, min v and max v.
template <int NW>
__device__ void block_stats(float &am, float &lo, float &hi, CtaShared<NW> &sh)
{
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    am = warp_redux_max_abs(am);
    lo = warp_redux_min(lo);
    hi = warp_redux_max(hi);
    if (lane == 0) {
        sh.redf[0][wid] = am;
        sh.redf[1][wid] = lo;
        sh.redf[2][wid] = hi;
    }
    __syncthreads();
    am = warp_redux_max_abs(sh.redf[0][lane & (NW - 1)]);
    lo = warp_redux_min(sh.redf[1][lane & (NW - 1)]);
    hi = warp_redux_max(sh.redf[2][lane & (NW - 1)]);
    __syncthreads();
}

// --- ORQ: per-warp histogram -------------------------------------------------------------------
// wh[0 .. 511]: [cell][column] words count << 22 | sum of 16-bit fractions (a column sees at most
// 64 values between reductions); wh[512 .. 575]: the warp's cell counts; wh[576 .. 639]: the
// warp's cell fraction sums (cell 63, the top grid point, is folded into cell 62 with fraction
// 2^16).
constexpr int kWarpHistWords = 64 * 8 + 64 + 64;
constexpr int kCtaHistShift = 22;

__device__ __forceinline__ void reduce_warp_hist(uint32_t *wh, int lane)
{
    __syncwarp();
    uint32_t t0 = 0, t1 = 0, c0 = 0, c1 = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int q4 = (k + (lane >> 1)) & 3;
        uint4 *ph = reinterpret_cast<uint4 *>(wh + lane * 16) + q4;
        const uint4 x = *ph;
        *ph = make_uint4(0u, 0u, 0u, 0u);
        const uint32_t st = x.x + x.y + x.z + x.w;
        const uint32_t sc = (x.x >> kCtaHistShift) + (x.y >> kCtaHistShift) + (x.z >> kCtaHistShift) +
                            (x.w >> kCtaHistShift);
        if (q4 < 2) {
            t0 += st;
            c0 += sc;
        } else {
            t1 += st;
            c1 += sc;
        }
    }
    uint32_t f0 = t0 - (c0 << kCtaHistShift), f1 = t1 - (c1 << kCtaHistShift);
    if (lane == 31) {  // cell 63 -> cell 62, fraction 2^16 each
        c0 += c1;
        f0 += c1 << kOrqFBits;
        c1 = 0u;
        f1 = 0u;
    }
    wh[512 + 2 * lane] += c0;
    wh[512 + 2 * lane + 1] += c1;
    wh[576 + 2 * lane] += f0;
    wh[576 + 2 * lane + 1] += f1;
    __syncwarp();
}

// BinGrad-b's levels of the staged bucket (m = max|u| > 0): sorts the clipped values in place
// (padding +inf; the staged values are lost), exact int64 block scan of their fixed-point
// values, argmax of J(k) ties to the smallest k.  {a, b, split value, split found}.  Also used by
// BinGrad-pb, whose levels must be at least as far apart.
template <int NW, class Clip>
__device__ RoundB cta_bingrad_b_levels(float *vs, int d, int nvalid, float m, const Clip &clipped, CtaShared<NW> &sh)
{
    constexpr int kCtaThreads = NW * 32;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    RoundB rb{0.0f, 0.0f, 0.0f, false};
    // sort u in place (padding = +inf), by the register path's network (every comparator puts
    // the minimum at the lower index): the warps sort runs of 512 keys in registers; each merge of
    // blocks of k >= 1024 keys then takes its mirror stage (i against i ^ (k-1)) and its
    // half-cleaners down to distance 512 in shared memory, and the stages below 512, which stay
    // inside a run, in registers again
    constexpr int kRun = 512;
    for (int i = tid; i < d; i += kCtaThreads) vs[i] = i < nvalid ? clipped(vs[i]) : INFINITY;
    __syncthreads();
    const int nruns = d / kRun;
    auto run_io = [&](int run, float (&key)[16], bool load) {
        float4 *q = reinterpret_cast<float4 *>(vs + run * kRun + 16 * lane);
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            if (load) {
                const float4 x = q[v];
                key[4 * v] = x.x;
                key[4 * v + 1] = x.y;
                key[4 * v + 2] = x.z;
                key[4 * v + 3] = x.w;
            } else {
                q[v] = make_float4(key[4 * v], key[4 * v + 1], key[4 * v + 2], key[4 * v + 3]);
            }
        }
    };
    for (int run = wid; run < nruns; run += NW) {
        float key[16];
        run_io(run, key, true);
        warp_bitonic_sort<16>(key, lane);
        run_io(run, key, false);
    }
    __syncthreads();
    for (int k = 2 * kRun; k <= d; k <<= 1) {
        for (int i = tid; i < d; i += kCtaThreads) {  // mirror stage
            const int ixj = i ^ (k - 1);
            if (ixj > i) {
                const float a = vs[i], b = vs[ixj];
                vs[i] = fminf(a, b);
                vs[ixj] = fmaxf(a, b);
            }
        }
        __syncthreads();
        for (int j = k >> 2; j >= kRun; j >>= 1) {
            for (int i = tid; i < d; i += kCtaThreads) {
                const int ixj = i ^ j;
                if (ixj > i) {
                    const float a = vs[i], b = vs[ixj];
                    vs[i] = fminf(a, b);
                    vs[ixj] = fmaxf(a, b);
                }
            }
            __syncthreads();
        }
        for (int run = wid; run < nruns; run += NW) {
            float key[16];
            run_io(run, key, true);
            warp_halfclean<16, kRun / 2>(key, lane);
            run_io(run, key, false);
        }
        __syncthreads();
    }
    // exact prefix sums of the fixed-point values: thread t owns positions [t*seg, (t+1)*seg)
    const int e2 = 46 - fexpo(m);
    const double sc = pow2d(e2);
    const int seg = d / kCtaThreads;
    long long run = 0;
    for (int i = tid * seg; i < tid * seg + seg; ++i) run += (i < nvalid) ? fixed_point(vs[i], sc) : 0ll;
    const long long incl = warp_inclusive_scan(run, lane);
    if (lane == 31) sh.redl[0][wid] = incl;
    __syncthreads();
    long long wpre = 0, total = 0;
    for (int k = 0; k < NW; ++k) {
        const long long t = sh.redl[0][k];
        if (k < wid) wpre += t;
        total += t;
    }
    __syncthreads();
    const long long S0 = wpre + incl - run;  // sum of positions before tid*seg
    // Screening, as in the register path: a binary32 estimate of J for every admissible split
    // (within 8 * 2^-24 of J), then the fp64 J only for the splits whose estimate reaches
    // M (1 - 2^-18), M the block's largest estimate; every split whose fp64 J is the largest is
    // among them, so the choice (ties to the smallest split) is the exhaustive one.
    float emax = 0.0f;
    {
        long long S = S0;
        for (int i = tid * seg; i < tid * seg + seg; ++i) {
            if (i >= 1 && i < nvalid && vs[i - 1] < vs[i]) {
                const float l = __ll2float_rn(S), rr = __ll2float_rn(total - S);
                emax = fmaxf(emax, __fadd_rn(__fmul_rn(__fmul_rn(l, l), rcp_approx((float)i)),
                                             __fmul_rn(__fmul_rn(rr, rr), rcp_approx((float)(nvalid - i)))));
            }
            if (i < nvalid) S += fixed_point(vs[i], sc);
        }
    }
    const float thr = __fmul_rn(block_max(emax, sh, 2), 1.0f - 0x1p-18f);
    double best_j = -1.0;
    int best_i = 0x7fffffff;
    long long best_s = 0;
    {
        long long S = S0;
        for (int i = tid * seg; i < tid * seg + seg; ++i) {
            if (i >= 1 && i < nvalid && vs[i - 1] < vs[i]) {
                const float l = __ll2float_rn(S), rr = __ll2float_rn(total - S);
                const float est = __fadd_rn(__fmul_rn(__fmul_rn(l, l), rcp_approx((float)i)),
                                            __fmul_rn(__fmul_rn(rr, rr), rcp_approx((float)(nvalid - i))));
                if (est >= thr) {
                    const double ld = __ll2double_rn(S);
                    const double rd = __ll2double_rn(total - S);
                    const double J = __dadd_rn(__ddiv_rn(__dmul_rn(ld, ld), (double)i),
                                               __ddiv_rn(__dmul_rn(rd, rd), (double)(nvalid - i)));
                    if (J > best_j) {
                        best_j = J;
                        best_i = i;
                        best_s = S;
                    }
                }
            }
            if (i < nvalid) S += fixed_point(vs[i], sc);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const double oj = __shfl_xor_sync(kFull, best_j, o);
        const int oi = __shfl_xor_sync(kFull, best_i, o);
        const long long os = __shfl_xor_sync(kFull, best_s, o);
        if (oj > best_j || (oj == best_j && oi < best_i)) {
            best_j = oj;
            best_i = oi;
            best_s = os;
        }
    }
    if (lane == 0) {
        sh.redd[wid] = best_j;
        sh.redi[wid] = best_i;
        sh.redl[1][wid] = best_s;
    }
    __syncthreads();
    best_j = sh.redd[lane & (NW - 1)];
    best_i = sh.redi[lane & (NW - 1)];
    best_s = sh.redl[1][lane & (NW - 1)];
#pragma unroll
    for (int o = NW / 2; o > 0; o >>= 1) {
        const double oj = __shfl_xor_sync(kFull, best_j, o);
        const int oi = __shfl_xor_sync(kFull, best_i, o);
        const long long os = __shfl_xor_sync(kFull, best_s, o);
        if (oj > best_j || (oj == best_j && oi < best_i)) {
            best_j = oj;
            best_i = oi;
            best_s = os;
        }
    }
    if (best_i == 0x7fffffff) {
        const float v0 = __fadd_rn(vs[0], 0.0f);
        rb = RoundB{v0, v0, v0, false};
    } else {
        const double inv_sc = pow2d(-e2);
        const float a = __double2float_rn(__dmul_rn(__ddiv_rn(__ll2double_rn(best_s), (double)best_i), inv_sc));
        const float b = __double2float_rn(
            __dmul_rn(__ddiv_rn(__ll2double_rn(total - best_s), (double)(nvalid - best_i)), inv_sc));
        rb = RoundB{a, b, vs[best_i], true};
    }
    __syncthreads();
    return rb;
}

// Largest bucket whose running sum of the fused step stays in shared memory beside the staged
// bucket; larger ones keep it in the average's slice of global memory (L2-resident).
constexpr int kAccSmemMax = 8192;

// Bulk prefetch of [p, p + bytes) into L2 (bytes a multiple of 16, p 16-byte aligned), in
// pieces of at most 32 KB.
__device__ __forceinline__ void prefetch_l2(const void *p, unsigned bytes)
{
    const char *c = static_cast<const char *>(p);
    for (unsigned off = 0; off < bytes; off += 32768u) {
        const unsigned len = bytes - off < 32768u ? bytes - off : 32768u;
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(c + off), "r"(len) : "memory");
    }
}

// ERR: the error mode of gq_quant_error; nothing is written but part[3 * bucket + k].
template <int SCHEME, bool ERR, int NW>
__global__ void __launch_bounds__(NW * 32) k_cta(const __grid_constant__ KParams p, double *part)
{
    constexpr int kCtaWarps = NW, kCtaThreads = NW * 32;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    __shared__ CtaShared<NW> sh;
    const int d = p.d;
    const bool fused = !ERR && p.avg != nullptr;
    const bool acc_smem = fused && d <= kAccSmemMax;
    float *vs = reinterpret_cast<float *>(smem_raw);  // d floats
    float *accs = acc_smem ? vs + d : nullptr;         // the running sum (d floats) when it fits
    uint32_t *hist_all = reinterpret_cast<uint32_t *>(smem_raw + (size_t)d * 4 * (acc_smem ? 2 : 1));  // ORQ
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    uint32_t *wh = hist_all + wid * kWarpHistWords;

    if constexpr (SCHEME == GQ_ORQ) {
        for (int i = lane; i < kWarpHistWords; i += 32) wh[i] = 0u;
    }
    for (int i = tid; i < 64; i += kCtaThreads) {
        sh.ccnt[i] = 0u;
        sh.cs1[i] = 0ull;
        sh.cs2[i] = 0ull;
    }
    __syncthreads();

    const int nchunks = d >> 7;
    const int W = p.W;

    ErrAcc ea{0.0, 0.0, 0.0};
    for (int64_t beta = blockIdx.x; beta < p.nb; beta += gridDim.x) {
      const int64_t base = beta * (int64_t)d;
      const int nvalid = (beta == p.nb - 1) ? p.tail : d;
      for (int w = 0; w < W; ++w) {
        const float *g = p.g[w];
        float *r = p.r[w];
        unsigned char *msg = p.msg[w];
        const uint32_t worker = p.worker0 + (uint32_t)w;
        if (tid == 0) {
            // the next item's g and r into L2 while this one is processed
            const bool same = w + 1 < W;
            const int64_t nbeta = same ? beta : beta + gridDim.x;
            const int nw = same ? w + 1 : 0;
            if (nbeta < p.nb) {
                const int nv = nbeta == p.nb - 1 ? p.tail : d;
                const unsigned bytes = (unsigned)(nv * 4) & ~15u;
                if (bytes) {
                    prefetch_l2(p.g[nw] + nbeta * d, bytes);
                    if (p.r[nw]) prefetch_l2(p.r[nw] + nbeta * d, bytes);
                }
            }
        }
        // ---- stage v = g + r in shared memory; NaN-propagating max |v|, min v, max v ------------
        float am = 0.0f, vlo = INFINITY, vhi = -INFINITY;
        for (int i4 = tid; i4 < (d >> 2); i4 += kCtaThreads) {
            const int e = 4 * i4;
            float4 x;
            if (e + 3 < nvalid) {
                x = __ldcs(reinterpret_cast<const float4 *>(g + base + e));
                if (r) {
                    const float4 y = __ldcs(reinterpret_cast<const float4 *>(r + base + e));
                    x.x = __fadd_rn(x.x, y.x);
                    x.y = __fadd_rn(x.y, y.y);
                    x.z = __fadd_rn(x.z, y.z);
                    x.w = __fadd_rn(x.w, y.w);
                }
                am = fmax_nan(am, fmax_nan(fmax_nan(fabsf(x.x), fabsf(x.y)), fmax_nan(fabsf(x.z), fabsf(x.w))));
                vlo = fmin3_nan(vlo, fmin3_nan(x.x, x.y, x.z), x.w);
                vhi = fmax3_nan(vhi, fmax3_nan(x.x, x.y, x.z), x.w);
            } else {
                float t[4];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    t[c] = 0.0f;
                    if (e + c < nvalid) {
                        t[c] = g[base + e + c];
                        if (r) t[c] = __fadd_rn(t[c], r[base + e + c]);
                        am = fmax_nan(am, fabsf(t[c]));
                        vlo = fmin_nan(vlo, t[c]);
                        vhi = fmax_nan(vhi, t[c]);
                    }
                }
                x = make_float4(t[0], t[1], t[2], t[3]);
            }
            reinterpret_cast<float4 *>(vs)[i4] = x;
        }
        block_stats(am, vlo, vhi, sh);
        if (!(am <= FLT_MAX) && tid == 0) atomicOr(p.status, kStatusNonFinite);

        // ---- clip threshold ---------------------------------------------------------------------
        float T = INFINITY;
        const bool clip = p.clip > 0.0f;
        if (clip) {
            T = 0.0f;
            if (am > 0.0f) {
                const int e = 20 - fexpo(am);
                const double sc = pow2d(e);
                long long sx = 0, sxx = 0;
                for (int i = tid; i < nvalid; i += kCtaThreads) {
                    const long long X = fixed_point(vs[i], sc);
                    sx += X;
                    sxx += X * X;
                }
                sx = block_sum(sx, sh, 0);
                sxx = block_sum(sxx, sh, 1);
                T = clip_threshold_from_sums(sx, sxx, nvalid, e, p.clip);
            }
        }
        auto clipped = [&](float x) {
            if (!clip) return x;
            x = x < -T ? -T : x;
            return x > T ? T : x;
        };

        // ---- fit ------------------------------------------------------------------------------
        RoundQSGD rq;
        RoundORQ ro{sh.ctab};
        RoundB rb{0.0f, 0.0f, 0.0f, false};
        RoundPB rp;
        bool constant = false;
        float mn = 0.0f, mx = 0.0f, scale = 0.0f;
        if constexpr (SCHEME == GQ_QSGD) {
            float m = am;  // without clipping u = v
            if (clip) {
                m = 0.0f;
                for (int i = tid; i < nvalid; i += kCtaThreads) m = fmaxf(m, fabsf(clipped(vs[i])));
                m = block_max(m, sh, 0);
            }
            const int s = p.s;
            for (int k = tid; k < s - 1; k += kCtaThreads)
                sh.pair[k] = make_float2(__fmul_rn(m, p.qratio[k]), __fmul_rn(m, p.qratio[k + 1]));
            if (tid == 0) sh.bcast_f[0] = m;
            __syncthreads();
            rq.inv_m = m > 0.0f ? __frcp_rn(m) : 0.0f;
            rq.h = __fmul_rn((float)(s - 1), 0.5f);
            rq.kmax = s - 2;
            rq.pair = sh.pair;
        } else if constexpr (SCHEME == GQ_ORQ || SCHEME == GQ_BINGRAD_PB) {
            float lo = vlo, hi = vhi;  // without clipping u = v
            if (clip) {
                lo = INFINITY;
                hi = -INFINITY;
                for (int i = tid; i < nvalid; i += kCtaThreads) {
                    const float x = clipped(vs[i]);
                    lo = fminf(lo, x);
                    hi = fmaxf(hi, x);
                }
                lo = block_min(lo, sh, 0);
                hi = block_max(hi, sh, 1);
            }
            mn = __fadd_rn(lo, 0.0f);
            mx = __fadd_rn(hi, 0.0f);
            constant = !(mx > mn);
            if (!constant) {
                const float range = __fsub_rn(mx, mn);
                const float step = __fdiv_rn(range, 63.0f);
                if constexpr (SCHEME == GQ_ORQ) {
                    scale = __fmul_rn(__fdiv_rn(63.0f, range), (float)(1 << kOrqFBits));
                    // warp k: chunks k, k+8, ...; its histogram is reduced every 4 chunks (16
                    // values per lane, 64 per column)
                    const int col = lane & 7;
                    int pending = 0;
                    for (int ch = wid; ch < nchunks; ch += kCtaWarps) {
                        const float4 x = reinterpret_cast<const float4 *>(vs)[ch * 32 + lane];
                        const float xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            const int e = ch * 128 + 4 * lane + c;
                            if (e < nvalid) {
                                const int ps = grid_pos<kOrqFBits>(clipped(xs[c]), mn, scale);
                                atomicAdd(&wh[(ps >> kOrqFBits) * 8 + col], (uint32_t)(ps & 0xffff) | (1u << kCtaHistShift));
                            }
                        }
                        if (++pending == 4) {
                            reduce_warp_hist(wh, lane);
                            pending = 0;
                        }
                    }
                    if (pending) reduce_warp_hist(wh, lane);
                    __syncthreads();
                    if (wid == 0) {
                        // the warps' cell totals -> block histogram (count, sum of positions)
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const int j = lane + 32 * h;
                            uint32_t cnt = 0u;
                            unsigned long long fr = 0ull;
                            for (int w = 0; w < kCtaWarps; ++w) {
                                uint32_t *ow = hist_all + w * kWarpHistWords;
                                cnt += ow[512 + j];
                                fr += ow[576 + j];
                                ow[512 + j] = 0u;
                                ow[576 + j] = 0u;
                            }
                            sh.ccnt[j] = cnt;
                            sh.cs1[j] = (unsigned long long)cnt * ((unsigned long long)j << kOrqFBits) + fr;
                        }
                        __syncwarp();
                        const long long c0 = sh.ccnt[lane], c1 = sh.ccnt[lane + 32];
                        const long long s0 = (long long)sh.cs1[lane], s1 = (long long)sh.cs1[lane + 32];
                        const long long ic0 = warp_inclusive_scan(c0, lane), ic1 = warp_inclusive_scan(c1, lane);
                        const long long is0 = warp_inclusive_scan(s0, lane), is1 = warp_inclusive_scan(s1, lane);
                        const long long tc = __shfl_sync(kFull, ic0, 31), ts = __shfl_sync(kFull, is0, 31);
                        sh.P0[lane] = (int)(ic0 - c0);
                        sh.P1[lane] = is0 - s0;
                        sh.P0[lane + 32] = (int)(tc + ic1 - c1);
                        sh.P1[lane + 32] = ts + is1 - s1;
                        sh.ccnt[lane] = 0u;
                        sh.ccnt[lane + 32] = 0u;
                        sh.cs1[lane] = 0ull;
                        sh.cs1[lane + 32] = 0ull;
                        __syncwarp();
                        const unsigned long long mask = orq_greedy(sh.P0, sh.P1, p.s, lane);
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const int j = lane + 32 * h;
                            if ((mask >> j) & 1ull) sh.lev[__popcll(mask & ((1ull << j) - 1ull))] = grid_point(mn, mx, step, j);
                        }
                        __syncwarp();
                        if (lane < p.s - 1) sh.rinv[lane] = __frcp_rn(__fsub_rn(sh.lev[lane + 1], sh.lev[lane]));
                        __syncwarp();
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const int j = lane + 32 * h;
                            if (j <= kTopCell) {
                                const int k = __popcll(mask & ((2ull << j) - 1ull)) - 1;
                                sh.ctab[j] = make_float4(sh.lev[k], sh.lev[k + 1], sh.rinv[k], __int_as_float(k));
                            }
                        }
                    }
                    __syncthreads();
                } else {
                    scale = __fmul_rn(__fdiv_rn(63.0f, range), (float)(1 << kPbFBits));
                    // BinGrad-b's levels bound the pair from inside: A <= Amax, the largest grid
                    // index whose point is <= a_b (0 if none), B >= Bmin, the smallest whose point
                    // is >= b_b (63 if none).  The sort leaves the clipped values permuted in vs,
                    // which the histogram below does not mind; the final pass re-reads g and r.
                    const RoundB bl = cta_bingrad_b_levels<NW>(vs, d, nvalid, fmaxf(fabsf(mn), fabsf(mx)), clipped, sh);
                    int Amax, Bmin;
                    {
                        const float g0 = grid_point(mn, mx, step, lane), g1 = grid_point(mn, mx, step, lane + 32);
                        const unsigned long long le = (unsigned long long)__ballot_sync(kFull, g0 <= bl.a) |
                                                      ((unsigned long long)__ballot_sync(kFull, g1 <= bl.a) << 32);
                        const unsigned long long ge = (unsigned long long)__ballot_sync(kFull, g0 >= bl.b) |
                                                      ((unsigned long long)__ballot_sync(kFull, g1 >= bl.b) << 32);
                        Amax = le ? 63 - __clzll(le) : 0;
                        Bmin = ge ? __ffsll(ge) - 1 : 63;
                    }
                    // Q0, Q1, Q2 over the cells < k from the sorted values (the level search left them
                    // sorted in vs, valid ones first): the position is monotone in the value, so the
                    // cells are too, and Q(k) is the prefix before the first value whose cell is
                    // >= k.  Thread t walks positions [t*seg, (t+1)*seg); each nonempty cell records
                    // the prefix at its first value (count + 1 in ccnt, sums in cs1, cs2).
                    {
                        const int seg = d / kCtaThreads;
                        unsigned long long r1 = 0ull, r2 = 0ull;
                        for (int i = tid * seg; i < tid * seg + seg && i < nvalid; ++i) {
                            const unsigned long long ps = (unsigned long long)grid_pos<kPbFBits>(vs[i], mn, scale);
                            r1 += ps;
                            r2 += ps * ps;
                        }
                        unsigned long long i1 = warp_inclusive_scan(r1, lane), i2 = warp_inclusive_scan(r2, lane);
                        if (lane == 31) {
                            sh.redl[0][wid] = (long long)i1;
                            sh.redl[1][wid] = (long long)i2;
                        }
                        __syncthreads();
                        unsigned long long w1 = 0ull, w2 = 0ull, t1 = 0ull, t2 = 0ull;
                        for (int k = 0; k < NW; ++k) {
                            const unsigned long long a1 = (unsigned long long)sh.redl[0][k], a2 = (unsigned long long)sh.redl[1][k];
                            if (k < wid) {
                                w1 += a1;
                                w2 += a2;
                            }
                            t1 += a1;
                            t2 += a2;
                        }
                        unsigned long long x1 = w1 + i1 - r1, x2 = w2 + i2 - r2;
                        const int i0 = tid * seg;
                        int prev = (i0 > 0 && i0 - 1 < nvalid)
                                       ? min(grid_pos<kPbFBits>(vs[i0 - 1], mn, scale) >> kPbFBits, kTopCell)
                                       : -1;
                        for (int i = i0; i < i0 + seg && i < nvalid; ++i) {
                            const int ps = grid_pos<kPbFBits>(vs[i], mn, scale);
                            const int c = min(ps >> kPbFBits, kTopCell);
                            if (c != prev) {
                                sh.ccnt[c] = (unsigned int)(i + 1);
                                sh.cs1[c] = x1;
                                sh.cs2[c] = x2;
                            }
                            prev = c;
                            x1 += (unsigned long long)ps;
                            x2 += (unsigned long long)ps * (unsigned long long)ps;
                        }
                        if (tid == 0) {
                            sh.bcast_l[0] = (long long)t1;
                            sh.bcast_l[1] = (long long)t2;
                        }
                    }
                    __syncthreads();
                    if (wid == 0) {
                        const unsigned long long tc_all = (unsigned long long)nvalid;
                        const unsigned long long tx_all = (unsigned long long)sh.bcast_l[0];
                        const unsigned long long ty_all = (unsigned long long)sh.bcast_l[1];
                        const unsigned long long nonempty =
                            (unsigned long long)__ballot_sync(kFull, sh.ccnt[lane] != 0u) |
                            ((unsigned long long)__ballot_sync(kFull, sh.ccnt[lane + 32] != 0u) << 32);
                        unsigned long long Q0[2], Q1[2], Q2[2];
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const unsigned long long later = nonempty & (~0ull << (lane + 32 * h));
                            if (later) {
                                const int c = __ffsll(later) - 1;
                                Q0[h] = (unsigned long long)(sh.ccnt[c] - 1u);
                                Q1[h] = sh.cs1[c];
                                Q2[h] = sh.cs2[c];
                            } else {
                                Q0[h] = tc_all;
                                Q1[h] = tx_all;
                                Q2[h] = ty_all;
                            }
                        }
                        __syncwarp();
                        sh.ccnt[lane] = 0u;
                        sh.ccnt[lane + 32] = 0u;
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const int K = lane + 32 * h;
                            const unsigned long long uQ0 = Q0[h], uQ1 = Q1[h], uQ2 = Q2[h];
                            const unsigned long long k = (unsigned long long)K << kPbFBits;
                            sh.al[K] = (long long)(k * k * uQ0 - 3ull * k * uQ1 + 2ull * uQ2);
                            sh.be[K] = (long long)(3ull * k * uQ1 - 2ull * uQ2 + ty_all - 2ull * k * tx_all +
                                                   k * k * (tc_all - uQ0));
                            sh.ga[K] = (long long)(uQ1 - k * uQ0);
                            sh.de[K] = (long long)(k * uQ0 - uQ1);
                        }
                    }
                    __syncthreads();
                    // thread B < 64 finds column B's least E over A <= min(Amax, B - 1)
                    // (pb_column_argmin; E exact mod 2^64), ties to the smallest (A, B)
                    long long best_e = 0x7fffffffffffffffll;
                    int best_ab = 0x7fffffff;
                    {
                        const int B = tid;
                        const int Ahi = min(Amax, B - 1);
                        if (B < 64 && B >= Bmin && Ahi >= 0) {
                            const unsigned long long beB = sh.be[B], gaB = (unsigned long long)sh.ga[B] << kPbFBits;
                            const unsigned long long bb = (unsigned long long)B << kPbFBits;
                            auto E = [&](int A) {
                                return (long long)((unsigned long long)sh.al[A] + beB + (unsigned long long)(unsigned)A * gaB +
                                                   bb * (unsigned long long)sh.de[A]);
                            };
                            long long es;
                            best_ab = pb_column_argmin(E, Ahi, es) * 64 + B;
                            best_e = es;
                        }
                    }
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) {
                        const long long oe = __shfl_xor_sync(kFull, best_e, o);
                        const int oab = __shfl_xor_sync(kFull, best_ab, o);
                        if (oe < best_e || (oe == best_e && oab < best_ab)) {
                            best_e = oe;
                            best_ab = oab;
                        }
                    }
                    if (lane == 0) {
                        sh.redl[0][wid] = best_e;
                        sh.redi[wid] = best_ab;
                    }
                    __syncthreads();
                    best_e = sh.redl[0][lane & (NW - 1)];
                    best_ab = sh.redi[lane & (NW - 1)];
#pragma unroll
                    for (int o = NW / 2; o > 0; o >>= 1) {
                        const long long oe = __shfl_xor_sync(kFull, best_e, o);
                        const int oab = __shfl_xor_sync(kFull, best_ab, o);
                        if (oe < best_e || (oe == best_e && oab < best_ab)) {
                            best_e = oe;
                            best_ab = oab;
                        }
                    }
                    __syncthreads();
                    const int A = best_ab >> 6, Bs = best_ab & 63;
                    rp.a = grid_point(mn, mx, step, A);
                    rp.b = grid_point(mn, mx, step, Bs);
                    rp.rinv = __frcp_rn(__fsub_rn(rp.b, rp.a));
                    rp.pa = A << kPbFBits;
                    rp.pb = Bs << kPbFBits;
                }
            }
        } else {  // BinGrad-b
            float m = am;  // without clipping u = v
            if (clip) {
                m = 0.0f;
                for (int i = tid; i < nvalid; i += kCtaThreads) m = fmaxf(m, fabsf(clipped(vs[i])));
                m = block_max(m, sh, 0);
            }
            if (m > 0.0f) rb = cta_bingrad_b_levels<NW>(vs, d, nvalid, m, clipped, sh);
        }

        // ---- round, pack, write residual and message ---------------------------------------------
        uint32_t *cw = msg ? reinterpret_cast<uint32_t *>(msg) + beta * p.codes_words : nullptr;
        for (int ch = wid; ch < nchunks; ch += kCtaWarps) {
            const int e0 = ch * 128 + 4 * lane;
            float v4[4];
            if constexpr (SCHEME == GQ_BINGRAD_B || SCHEME == GQ_BINGRAD_PB) {
                // the sort overwrote the staged values: read g (+ r) again
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    v4[c] = 0.0f;
                    if (e0 + c < nvalid) {
                        v4[c] = g[base + e0 + c];
                        if (r) v4[c] = __fadd_rn(v4[c], r[base + e0 + c]);
                    }
                }
            } else {
                const float4 x = reinterpret_cast<const float4 *>(vs)[ch * 32 + lane];
                v4[0] = x.x;
                v4[1] = x.y;
                v4[2] = x.z;
                v4[3] = x.w;
            }
            float u4[4];
            int pos4[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                u4[c] = clipped(v4[c]);
                pos4[c] = 0;
                if constexpr (SCHEME == GQ_ORQ)
                    pos4[c] = constant ? 0 : min(grid_pos<kOrqFBits>(u4[c], mn, scale) >> kOrqFBits, kTopCell);
                if constexpr (SCHEME == GQ_BINGRAD_PB) pos4[c] = constant ? 0 : grid_pos<kPbFBits>(u4[c], mn, scale);
            }
            uint32_t valid = 0;
#pragma unroll
            for (int c = 0; c < 4; ++c) valid |= (e0 + c < nvalid ? 1u : 0u) << c;
            const uint64_t blk = (uint64_t)(base >> 2) + (uint64_t)(32 * ch);
            float *rout = r ? r + base + 128 * ch : nullptr;
            uint32_t *cwc = cw ? cw + ch * 4 * p.bits : nullptr;
            float q[4];
            if constexpr (ERR) {
                if constexpr (SCHEME == GQ_QSGD) {
                    err_chunk<true, false>(p, rq, blk, worker, lane, valid, u4, pos4, ea);
                } else if constexpr (SCHEME == GQ_ORQ) {
                    if (constant) err_chunk<false, false>(p, RoundConst{mn}, blk, worker, lane, valid, u4, pos4, ea);
                    else err_chunk<true, false>(p, ro, blk, worker, lane, valid, u4, pos4, ea);
                } else if constexpr (SCHEME == GQ_BINGRAD_PB) {
                    if (constant) err_chunk<false, false>(p, RoundConst{mn}, blk, worker, lane, valid, u4, pos4, ea);
                    else err_chunk<true, false>(p, rp, blk, worker, lane, valid, u4, pos4, ea);
                } else {
                    err_chunk<false, false>(p, rb, blk, worker, lane, valid, u4, pos4, ea);
                }
            } else {
                if constexpr (SCHEME == GQ_QSGD) {
                    round_chunk<true, false, 0>(p, rq, blk, worker, lane, valid, v4, u4, pos4, rout, cwc, q);
                } else if constexpr (SCHEME == GQ_ORQ) {
                    if (constant)
                        round_chunk<false, false, 0>(p, RoundConst{mn}, blk, worker, lane, valid, v4, u4, pos4, rout, cwc, q);
                    else
                        round_chunk<true, false, 0>(p, ro, blk, worker, lane, valid, v4, u4, pos4, rout, cwc, q);
                } else if constexpr (SCHEME == GQ_BINGRAD_PB) {
                    if (constant)
                        round_chunk<false, false, 0>(p, RoundConst{mn}, blk, worker, lane, valid, v4, u4, pos4, rout, cwc, q);
                    else
                        round_chunk<true, false, 0>(p, rp, blk, worker, lane, valid, v4, u4, pos4, rout, cwc, q);
                } else {
                    round_chunk<false, false, 0>(p, rb, blk, worker, lane, valid, v4, u4, pos4, rout, cwc, q);
                }
                if (fused) {
                    // running sum in worker order from +0; the last worker writes the average.  The
                    // element's sum is read and written by this thread only.
                    float *ab = (acc_smem ? accs : p.avg + base) + e0;
                    float *out = p.avg + base + e0;
                    const bool last = w == W - 1;
                    if (valid == 0xfu) {
                        float4 a = w == 0 ? make_float4(0.0f, 0.0f, 0.0f, 0.0f) : *reinterpret_cast<const float4 *>(ab);
                        a = make_float4(__fadd_rn(a.x, q[0]), __fadd_rn(a.y, q[1]), __fadd_rn(a.z, q[2]), __fadd_rn(a.w, q[3]));
                        if (last)
                            __stcs(reinterpret_cast<float4 *>(out), make_float4(__fmul_rn(a.x, p.inv_w), __fmul_rn(a.y, p.inv_w),
                                                                                __fmul_rn(a.z, p.inv_w), __fmul_rn(a.w, p.inv_w)));
                        else
                            *reinterpret_cast<float4 *>(ab) = a;
                    } else {
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            if ((valid >> c) & 1u) {
                                const float a = __fadd_rn(w == 0 ? 0.0f : ab[c], q[c]);
                                if (last) out[c] = __fmul_rn(a, p.inv_w);
                                else ab[c] = a;
                            }
                        }
                    }
                }
            }
        }
        if constexpr (ERR) {
            // bucket sums: warps in a fixed butterfly, then warp 0 .. 7 in order
            ea = warp_sum_err(ea);
            if (lane == 0) {
                sh.rede[0][wid] = ea.e;
                sh.rede[1][wid] = ea.uu;
                sh.rede[2][wid] = ea.qq;
            }
            __syncthreads();
            if (tid < 3) {
                double t = 0.0;
                for (int k = 0; k < kCtaWarps; ++k) t = __dadd_rn(t, sh.rede[tid][k]);
                part[3 * beta + tid] = t;
            }
            ea = ErrAcc{0.0, 0.0, 0.0};
        }
        // ---- level table --------------------------------------------------------------------------
        if (msg && tid < p.L) {
            float lv;
            if constexpr (SCHEME == GQ_QSGD) lv = sh.bcast_f[0];
            else if constexpr (SCHEME == GQ_ORQ) lv = constant ? mn : sh.lev[tid];
            else if constexpr (SCHEME == GQ_BINGRAD_PB) lv = constant ? mn : (tid == 0 ? rp.a : rp.b);
            else lv = tid == 0 ? rb.a : rb.b;
            reinterpret_cast<float *>(msg + p.levels_off)[beta * p.L + tid] = lv;
        }
        __syncthreads();
      }
    }
}

template <int SCHEME, bool ERR, int NW>
cudaError_t launch(const KParams &p, double *part, cudaStream_t stream)
{
    auto kern = k_cta<SCHEME, ERR, NW>;
    const bool acc_smem = !ERR && p.avg != nullptr && p.d <= kAccSmemMax;
    const size_t smem = (size_t)p.d * 4 * (acc_smem ? 2 : 1) +
                        (SCHEME == GQ_ORQ ? (size_t)NW * kWarpHistWords * 4 : 0);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0, per_sm = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, NW * 32, smem);
    if (per_sm < 1) per_sm = 1;
    const int64_t cap = (int64_t)sms * per_sm;
    const int grid = (int)(p.nb < cap ? p.nb : cap);
    if (grid <= 0) return cudaSuccess;
    kern<<<grid, NW * 32, smem, stream>>>(p, part);
    return cudaGetLastError();
}

// 8 warps per CTA, 16 for the largest buckets (one CTA fits per SM there).
template <int SCHEME, bool ERR>
cudaError_t launch_nw(const KParams &p, double *part, cudaStream_t stream)
{
    return p.d >= 16384 ? launch<SCHEME, ERR, 16>(p, part, stream) : launch<SCHEME, ERR, 8>(p, part, stream);
}

template <bool ERR>
cudaError_t dispatch(const KParams &p, double *part, cudaStream_t stream)
{
    switch (p.scheme) {
    case GQ_QSGD:
    case GQ_TERNGRAD: return launch_nw<GQ_QSGD, ERR>(p, part, stream);
    case GQ_BINGRAD_B: return launch_nw<GQ_BINGRAD_B, ERR>(p, part, stream);
    case GQ_BINGRAD_PB: return launch_nw<GQ_BINGRAD_PB, ERR>(p, part, stream);
    default: return launch_nw<GQ_ORQ, ERR>(p, part, stream);
    }
}

}  // namespace

cudaError_t launch_cta_encode(const KParams &p, cudaStream_t stream) { return dispatch<false>(p, nullptr, stream); }

cudaError_t launch_cta_err(const KParams &p, double *part, cudaStream_t stream) { return dispatch<true>(p, part, stream); }

}  // namespace gq
