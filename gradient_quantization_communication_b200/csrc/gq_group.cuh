// gq_group.cuh -- ORQ and QSGD / TernGrad for buckets of d = 1024 .. 32768 without clipping: a
// bucket is spread over a group of G = d / 512 warps, each of which holds 512 of its values in
// registers exactly as the register path holds a whole bucket of 512.
//
// Included by gq_group_orq.cu and gq_group_qsgd.cu (one scheme each, compiled in parallel).
//
// CTAs of NW warps: 4 for d <= 2048, 8 for 4096, 16 above.  Up to NW warps a CTA holds NW / G
// groups, each synchronised by its own named barrier (d = 1024: two per CTA of 4; 2048, 4096 and
// 8192: one).  For G > NW a bucket takes a cluster of C = G / NW CTAs (d = 16384: 2, 32768: 4),
// synchronised by cluster barriers, and the statistics cross CTAs through distributed shared
// memory (plain loads of the peer CTA's shared memory).
// Only what the fit needs crosses warps:
//   QSGD / TernGrad : each warp's max |u| -> the group's max (one exchange);
//   ORQ             : each warp's min and max -> the group's; then each warp's 64 cell counts
//                     and sums of 16-bit grid positions -> the group's histogram, from which
//                     the group's first warp (in a cluster, every CTA's first warp, on the same
//                     totals) runs the greedy and builds the bracket table the others read.
// Warp k of a group rounds elements 512k .. 512k+511 of the bucket, so it writes the codes,
// residual and fused sum of a 512-element slice at the same global index with the per-element
// rules, Philox counters and dense code layout of the other paths (the launcher passes
// codes_words = 16 b, the code words of one slice).  Group rank 0 writes the level table.
//
// Each warp stages its slice of the next item with a 1-D bulk copy while it works on the
// current one (as the register path does).  Every exchange slot is double-buffered by item
// parity: a slot is rewritten two items later, after a barrier that every reader of its
// previous contents has passed.  Across CTAs the threads that wrote a slot fence it at cluster
// scope and every thread then arrives at the cluster barrier without a release of its own.  A
// copy that does not complete within the wait limit is reported at the next exchange; the whole
// group then stops at the same point (after a last cluster barrier, so that no CTA leaves while
// a peer may still read its shared memory).
// The ragged last bucket is a second launch of the same kernel (TAIL): one group, guarded
// plain loads, the invalid slots masked out of the statistics and the stores.
#pragma once

#include "gq_warp.cuh"

namespace gq {
namespace {

// Warps per CTA: 4 for G <= 4 (one or two groups per CTA; more CTAs per SM hide the groups'
// barrier waits better: 5 % faster at d = 2048 than 8), 8 for G = 8, and 16 from G = 16 on (one
// CTA per SM and per d = 8192 bucket, clusters of 2 and 4 CTAs for 16384 and 32768: 20 % faster
// at d = 8192 than clusters of two 8-warp CTAs, 3-5 % at 32768).
template <int G> constexpr int group_cta_warps() { return G <= 4 ? 4 : (G >= 16 ? 16 : 8); }
constexpr int kSliceEPL = 16;   // values per lane: a warp holds 512 values

struct alignas(16) FitGroupORQ {
    uint32_t hist[64 * kHistCols];  // per warp, as in the register path
    float4 ctab[64];
    float4 btab[GQ_MAX_LEVELS];
    float lev[GQ_MAX_LEVELS];
    long long P1[64];  // the group's prefix sums of positions (up to 32768 * 63 * 2^16 < 2^37)
    int P0[64];
};

template <int SCHEME> struct GroupFitFor { using type = FitQSGD; };
template <> struct GroupFitFor<GQ_ORQ> { using type = FitGroupORQ; };

template <int SCHEME>
struct alignas(16) GroupWarpSmem {
    StageBuf<kSliceEPL> stage;
    unsigned long long bar;
    typename GroupFitFor<SCHEME>::type fit;
};

// The CTA's exchange slots, [item parity][...].
template <int NW>
struct alignas(16) GroupXchg {
    float2 stat[2][NW];            // per warp: {min, max} (ORQ) or {max |u|, 0} (QSGD)
    int fail[2][NW];               // per warp: its copy timed out
    uint4 cells[2][NW][32];        // per warp and lane l: counts and position sums of cells 2l, 2l+1
    unsigned long long cta_s[2][32][2];     // clusters: the CTA's sums of cells 2l, 2l+1
    unsigned int cta_c[2][32][2];           // clusters: the CTA's counts
};

// --- barriers and distributed shared memory ----------------------------------------------------
__device__ __forceinline__ void named_bar(int id, int nthreads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
__device__ __forceinline__ void cluster_bar()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Cluster barrier whose arrival orders nothing: the threads that wrote exchange slots fenced
// them first (fence_cluster), the wait acquires.
__device__ __forceinline__ void cluster_bar_relaxed()
{
    asm volatile("barrier.cluster.arrive.relaxed.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void fence_cluster() { asm volatile("fence.acq_rel.cluster;" ::: "memory"); }
// Address of the same shared-memory object in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t peer_addr(const void *p, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
    return r;
}
__device__ __forceinline__ float2 ld_peer_f2(uint32_t a)
{
    float2 v;
    asm volatile("ld.shared::cluster.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(a) : "memory");
    return v;
}
__device__ __forceinline__ int ld_peer_s32(uint32_t a)
{
    int v;
    asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
    return v;
}
__device__ __forceinline__ uint2 ld_peer_u2(uint32_t a)
{
    uint2 v;
    asm volatile("ld.shared::cluster.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a) : "memory");
    return v;
}
__device__ __forceinline__ ulonglong2 ld_peer_u64x2(uint32_t a)
{
    ulonglong2 v;
    asm volatile("ld.shared::cluster.v2.u64 {%0, %1}, [%2];" : "=l"(v.x), "=l"(v.y) : "r"(a) : "memory");
    return v;
}

// Rank 0 of the group writes the level table; the rest of the table logic is the register path's.
__device__ __forceinline__ void group_orq_tables(const KParams &p, FitGroupORQ &sm, int w, int64_t beta, int lane,
                                                 bool writer, unsigned long long mask, float mn, float mx, float step)
{
    const uint32_t mlo = (uint32_t)mask, mhi = (uint32_t)(mask >> 32);
    const uint32_t lt = (1u << lane) - 1u, le = lt | (1u << lane);
    const int nlo = __popc(mlo);
    unsigned char *msg = p.msg[w];
    float *mtab = (writer && msg) ? reinterpret_cast<float *>(msg + p.levels_off) + beta * p.L : nullptr;
    const bool ch0 = (mlo >> lane) & 1u, ch1 = (mhi >> lane) & 1u;
    const int r0 = __popc(mlo & lt), r1 = nlo + __popc(mhi & lt);
    const float lv0 = __fadd_rn(mn, __fmul_rn((float)lane, step));
    const float lv1 = lane == 31 ? mx : __fadd_rn(mn, __fmul_rn((float)(lane + 32), step));
    if (ch0) sm.lev[r0] = lv0;
    if (ch1) sm.lev[r1] = lv1;
    if (mtab) {
        if (ch0) mtab[r0] = lv0;
        if (ch1) mtab[r1] = lv1;
    }
    __syncwarp();
    if (lane < p.s - 1) {
        const float lo = sm.lev[lane], hi = sm.lev[lane + 1];
        sm.btab[lane] = make_float4(lo, hi, __frcp_rn(__fsub_rn(hi, lo)), __int_as_float(lane));
    }
    __syncwarp();
    sm.ctab[lane] = sm.btab[__popc(mlo & le) - 1];
    sm.ctab[lane + 32] = sm.btab[min(nlo + __popc(mhi & le) - 1, p.s - 2)];
    __syncwarp();
}

// Buckets b0 .. b1-1 (TAIL: the ragged last bucket alone, b0 = nb - 1, b1 = nb).
template <int SCHEME, int G, int NW, bool FUSED, bool TAIL>
__global__ void __launch_bounds__(NW * 32, 16 / NW) k_group(const __grid_constant__ KParams p, int64_t b0, int64_t b1)
{
    constexpr int kGroupWarps = NW;
    constexpr int C = G > kGroupWarps ? G / kGroupWarps : 1;    // CTAs per bucket
    constexpr int GPC = G < kGroupWarps ? kGroupWarps / G : 1;  // groups per CTA
    constexpr int EPL = kSliceEPL;
    constexpr int D = G * 32 * EPL;
    constexpr unsigned kBytes = 32 * EPL * 4;
    using Smem = GroupWarpSmem<SCHEME>;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    GroupXchg<NW> &xg = *reinterpret_cast<GroupXchg<NW> *>(smem_raw);
    const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
    Smem &sm = reinterpret_cast<Smem *>(smem_raw + sizeof(GroupXchg<NW>))[wib];
    const int gid = C > 1 ? 0 : wib / G;                                         // group within the CTA
    const uint32_t crank = C > 1 ? (uint32_t)(blockIdx.x % C) : 0u;             // CTA within the cluster
    const int rk = C > 1 ? (int)crank * kGroupWarps + wib : wib % G;           // warp within the group
    const int64_t first = b0 + (C > 1 ? (int64_t)(blockIdx.x / C) : (int64_t)blockIdx.x * GPC + gid);
    const int64_t stride = C > 1 ? (int64_t)(gridDim.x / C) : (int64_t)gridDim.x * GPC;
    // the group's first exchange: named barrier of its warps, or the cluster's barrier
    auto sync_group = [&]() {
        if constexpr (C > 1) cluster_bar_relaxed();
        else named_bar(1 + gid, 32 * G);
    };
    // TAIL: the valid slots of the warp's slice
    uint32_t vmask = 0xffffffffu;
    if constexpr (TAIL) {
        vmask = 0u;
#pragma unroll
        for (int t = 0; t < EPL; ++t) vmask |= (rk * (32 * EPL) + slot_elem(t, lane) < p.tail ? 1u : 0u) << t;
    }

    init_fit<SCHEME>(p, sm.fit, lane);
    if (lane == 0) {
        mbar_init(&sm.bar, 1);
        fence_barrier_init();
    }
    __syncwarp();
    if (first >= b1) return;  // the whole group (or cluster) leaves together
    const int W = p.W;
    const int64_t nitems = ((b1 - 1 - first) / stride + 1) * W;
    const bool ef = p.r[0] != nullptr;
    const unsigned tx = ef ? 2 * kBytes : kBytes;
    auto issue = [&](int64_t beta, int w) {  // lane 0
        const int64_t off = beta * D + (int64_t)rk * (32 * EPL);
        fence_proxy_async();
        mbar_arrive_expect_tx(&sm.bar, tx);
        bulk_load(sm.stage.g, p.g[w] + off, kBytes, &sm.bar);
        if (ef) bulk_load(sm.stage.r, p.r[w] + off, kBytes, &sm.bar);
    };
    if (!TAIL && lane == 0) issue(first, 0);
    int64_t pbeta = first;
    int pw = 1;
    if (pw == W) {
        pw = 0;
        pbeta += stride;
    }

    int64_t beta = first;
    int w = 0;
    unsigned parity = 0;
    float acc[EPL];
    for (int64_t it = 0; it < nitems; ++it) {
        const bool ok = TAIL || mbar_wait_warp(&sm.bar, parity);
        float v[EPL];
        if constexpr (TAIL) {
            const int64_t off = beta * D + (int64_t)rk * (32 * EPL);
            const float *g = p.g[w] + off;
            const float *r = ef ? p.r[w] + off : nullptr;
#pragma unroll
            for (int t = 0; t < EPL; ++t) {
                const int e = slot_elem(t, lane);
                float x = 0.0f;
                if ((vmask >> t) & 1u) {
                    x = g[e];
                    if (r) x = __fadd_rn(x, r[e]);
                }
                v[t] = x;
            }
        } else if (ok) {
            parity ^= 1u;
#pragma unroll
            for (int m = 0; m < EPL / 4; ++m) {
                float4 x = *reinterpret_cast<const float4 *>(sm.stage.g + 128 * m + 4 * lane);
                if (ef) {
                    const float4 y = *reinterpret_cast<const float4 *>(sm.stage.r + 128 * m + 4 * lane);
                    x = make_float4(__fadd_rn(x.x, y.x), __fadd_rn(x.y, y.y), __fadd_rn(x.z, y.z), __fadd_rn(x.w, y.w));
                }
                v[4 * m + 0] = x.x;
                v[4 * m + 1] = x.y;
                v[4 * m + 2] = x.z;
                v[4 * m + 3] = x.w;
            }
        } else {
#pragma unroll
            for (int t = 0; t < EPL; ++t) v[t] = 0.0f;
        }
        __syncwarp();
        const bool issued = !TAIL && ok && it + 1 < nitems;
        if (issued && lane == 0) issue(pbeta, pw);
        if (++pw == W) {
            pw = 0;
            pbeta += stride;
        }
        const int par = (int)(it & 1);
        const int64_t sigma = beta * G + rk;  // the warp's 512-element slice
        const bool writer = rk == 0;
        if (w == 0) {
#pragma unroll
            for (int t = 0; t < EPL; ++t) acc[t] = 0.0f;
        }

        // ---- first exchange: the group's statistics (and whether every copy arrived) -----------
        float s0, s1;
        if constexpr (SCHEME == GQ_ORQ) {
            float mn = INFINITY, mx = -INFINITY;
            if constexpr (TAIL) {
#pragma unroll
                for (int t = 0; t < EPL; ++t)
                    if ((vmask >> t) & 1u) {
                        mn = fmin_nan(mn, v[t]);
                        mx = fmax_nan(mx, v[t]);
                    }
            } else {
                mn = fmin3_nan(v[0], v[1], v[2]);
                mx = fmax3_nan(v[0], v[1], v[2]);
#pragma unroll
                for (int t = 3; t < EPL; t += 2) {
                    mn = t + 1 < EPL ? fmin3_nan(mn, v[t], v[t + 1]) : fmin_nan(mn, v[t]);
                    mx = t + 1 < EPL ? fmax3_nan(mx, v[t], v[t + 1]) : fmax_nan(mx, v[t]);
                }
            }
            s0 = warp_redux_min(mn);
            s1 = warp_redux_max(mx);
        } else {
            float m = 0.0f;
#pragma unroll
            for (int t = 0; t < EPL; ++t)
                if (!TAIL || ((vmask >> t) & 1u)) m = fmax_nan(m, fabsf(v[t]));
            s0 = warp_redux_max_abs(m);
            s1 = 0.0f;
        }
        if (lane == 0) {
            xg.stat[par][wib] = make_float2(s0, s1);
            xg.fail[par][wib] = ok ? 0 : 1;
            if (C > 1) fence_cluster();
        }
        __syncwarp();
        sync_group();
        float2 st = make_float2(SCHEME == GQ_ORQ ? INFINITY : 0.0f, -INFINITY);
        int failed = 0;
        if constexpr (C > 1) {
#pragma unroll
            for (int h = 0; h < (G + 31) / 32; ++h) {
                const int j = lane + 32 * h;
                if (j < G) {
                    const uint32_t rr = (uint32_t)(j / kGroupWarps);
                    const float2 o = ld_peer_f2(peer_addr(&xg.stat[par][j % kGroupWarps], rr));
                    failed |= ld_peer_s32(peer_addr(&xg.fail[par][j % kGroupWarps], rr));
                    if (SCHEME == GQ_ORQ) {
                        st.x = h ? key_float(min(float_key(st.x), float_key(o.x))) : o.x;
                        st.y = h ? key_float(max(float_key(st.y), float_key(o.y))) : o.y;
                    } else {
                        st.x = h ? __uint_as_float(max(__float_as_uint(st.x), __float_as_uint(o.x))) : o.x;
                    }
                }
            }
        } else {
            if (lane < G) {
                st = xg.stat[par][gid * G + lane];
                failed = xg.fail[par][gid * G + lane];
            }
        }
        if (__any_sync(kFull, failed != 0)) {
            // a copy of the group did not arrive in time: report it, let every copy still in
            // flight land (bounded), and stop the whole group here
            if (lane == 0 && !ok) atomicOr(p.status, kStatusTimeout);
            if constexpr (C > 1) cluster_bar();
            if (!ok || issued) mbar_wait_warp(&sm.bar, parity);
            return;
        }

        if constexpr (SCHEME == GQ_ORQ) {
            float mn = warp_redux_min(st.x), mx = warp_redux_max(st.y);
            if (writer && !(mn >= -FLT_MAX && mx <= FLT_MAX)) flag_nonfinite(p, lane);
            mn = __fadd_rn(mn, 0.0f);
            mx = __fadd_rn(mx, 0.0f);
            int pos[EPL];
            if (!(mx > mn)) {  // constant bucket (or NaN): one level, code 0 -- the whole group
#pragma unroll
                for (int t = 0; t < EPL; ++t) pos[t] = 0;
                emit<EPL, FUSED, false, TAIL, 0>(p, RoundConst{mn}, sigma, w, lane, vmask, v, v, pos, acc);
                if (writer) store_table(p, w, beta, lane, mn);
            } else {
                const float range = __fsub_rn(mx, mn);
                const float step = __fdiv_rn(range, 63.0f);
                const float scale = __fmul_rn(__fdiv_rn(63.0f, range), (float)(1 << kOrqFBits));
                // the warp's histogram, as in the register path
                const int col = lane & (kHistCols - 1);
#pragma unroll
                for (int t = 0; t < EPL; ++t) {
                    int ps = min(__float2int_rz(__fmul_rn(__fsub_rn(v[t], mn), scale)), 63 << kOrqFBits);
                    if (TAIL) ps = max(ps, 0);  // the invalid slots hold 0, maybe outside [mn, mx]
                    const int cell = ps >> kOrqFBits;
                    pos[t] = cell;
                    if (!TAIL || ((vmask >> t) & 1u))
                        atomicAdd(&sm.fit.hist[cell * kHistCols + col], (uint32_t)(ps & 0xffff) | (1u << kHistCountShift));
                }
                __syncwarp();
                uint32_t t0 = 0, t1 = 0, c0 = 0, c1 = 0;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int q4 = (k + (lane >> 1)) & 3;
                    uint4 *ph = reinterpret_cast<uint4 *>(sm.fit.hist + lane * 16) + q4;
                    const uint4 x = *ph;
                    *ph = make_uint4(0u, 0u, 0u, 0u);
                    const uint32_t sx = x.x + x.y + x.z + x.w;
                    const uint32_t sc = (x.x >> kHistCountShift) + (x.y >> kHistCountShift) +
                                        (x.z >> kHistCountShift) + (x.w >> kHistCountShift);
                    if (q4 < 2) {
                        t0 += sx;
                        c0 += sc;
                    } else {
                        t1 += sx;
                        c1 += sc;
                    }
                }
                const uint32_t f0 = t0 - (c0 << kHistCountShift), f1 = t1 - (c1 << kHistCountShift);
                uint32_t w0 = c0 * ((uint32_t)(2 * lane) << kOrqFBits) + f0;
                uint32_t w1 = c1 * ((uint32_t)(2 * lane + 1) << kOrqFBits) + f1;
                if (lane == 31) {  // the top grid point belongs to cell 62 (position 63 * 2^16)
                    c0 += c1;
                    w0 += w1;
                    c1 = 0u;
                    w1 = 0u;
                }
                // ---- second exchange: the group's histogram ---------------------------------
                // The leader (group rank 0; in a cluster every CTA's warp 0) sums the cells, runs
                // the greedy and builds the tables; the other warps wait for them at a barrier.
                xg.cells[par][wib][lane] = make_uint4(c0, c1, w0, w1);
                const int bar_id = C > 1 ? 1 : 1 + gid;
                const int bar_n = 32 * (C > 1 ? kGroupWarps : G);
                const int wfirst = C > 1 ? 0 : gid * G;  // the first warp of the group in this CTA
                const bool leads = wib == wfirst;
                Smem &lead = reinterpret_cast<Smem *>(smem_raw + sizeof(GroupXchg<NW>))[wfirst];
                named_bar(bar_id, bar_n);
                unsigned int C0 = 0u, C1 = 0u;
                unsigned long long S0 = 0ull, S1 = 0ull;
                if (leads) {
#pragma unroll
                    for (int j = 0; j < (C > 1 ? kGroupWarps : G); ++j) {
                        const uint4 x = xg.cells[par][wfirst + j][lane];
                        C0 += x.x;
                        C1 += x.y;
                        S0 += x.z;
                        S1 += x.w;
                    }
                }
                if constexpr (C > 1) {
                    if (leads) {
                        xg.cta_c[par][lane][0] = C0;
                        xg.cta_c[par][lane][1] = C1;
                        xg.cta_s[par][lane][0] = S0;
                        xg.cta_s[par][lane][1] = S1;
                        fence_cluster();
                    }
                    cluster_bar_relaxed();
                    if (leads) {
                        C0 = C1 = 0u;
                        S0 = S1 = 0ull;
#pragma unroll
                        for (int rr = 0; rr < C; ++rr) {
                            const uint2 c = ld_peer_u2(peer_addr(&xg.cta_c[par][lane][0], (uint32_t)rr));
                            const ulonglong2 s = ld_peer_u64x2(peer_addr(&xg.cta_s[par][lane][0], (uint32_t)rr));
                            C0 += c.x;
                            C1 += c.y;
                            S0 += s.x;
                            S1 += s.y;
                        }
                    }
                }
                if (leads) {
                    // exclusive prefix over the cell pairs of (sum << 16 | count): counts up to
                    // 32768 and sums below 2^37 fit the packed 64-bit word
                    const unsigned long long own = ((S0 + S1) << 16) | (unsigned long long)(C0 + C1);
                    const unsigned long long ex = warp_inclusive_scan(own, lane) - own;
                    const int ec = (int)(ex & 0xffffull);
                    const long long es = (long long)(ex >> 16);
                    sm.fit.P0[2 * lane] = ec;
                    sm.fit.P0[2 * lane + 1] = ec + (int)C0;
                    sm.fit.P1[2 * lane] = es;
                    sm.fit.P1[2 * lane + 1] = es + (long long)S0;
                    __syncwarp();
                    const unsigned long long mask = orq_greedy(sm.fit.P0, sm.fit.P1, p.s, lane);
                    group_orq_tables(p, sm.fit, w, beta, lane, writer, mask, mn, mx, step);
                }
                named_bar(bar_id, bar_n);
                emit<EPL, FUSED, true, TAIL, 0>(p, RoundORQ{lead.fit.ctab}, sigma, w, lane, vmask, v, v, pos, acc);
                __syncwarp();
            }
        } else {
            const float m = warp_redux_max_abs(st.x);
            if (writer && !(m <= FLT_MAX)) flag_nonfinite(p, lane);
            const int s = p.s;
            for (int k = lane; k < s - 1; k += 32)
                sm.fit.pair[k] = make_float2(__fmul_rn(m, sm.fit.qr[k]), __fmul_rn(m, sm.fit.qr[k + 1]));
            __syncwarp();
            RoundQSGDT<false> rule;
            rule.inv_m = m > 0.0f ? __frcp_rn(m) : 0.0f;
            rule.h = __fmul_rn((float)(s - 1), 0.5f);
            rule.kmax = s - 2;
            rule.pair = sm.fit.pair;
            int pos[EPL];
#pragma unroll
            for (int t = 0; t < EPL; ++t) pos[t] = 0;
            emit<EPL, FUSED, true, TAIL, 0>(p, rule, sigma, w, lane, vmask, v, v, pos, acc);
            if (writer) store_table(p, w, beta, lane, m);
            __syncwarp();
        }

        const bool last_w = w == W - 1;
        if (FUSED && last_w) {
            if constexpr (TAIL) {
#pragma unroll
                for (int t = 0; t < EPL; ++t)
                    if ((vmask >> t) & 1u) p.avg[sigma * (32 * EPL) + slot_elem(t, lane)] = __fmul_rn(acc[t], p.inv_w);
            } else {
#pragma unroll
                for (int m = 0; m < EPL / 4; ++m) store_avg4(p.avg + sigma * (32 * EPL), m, lane, acc + 4 * m, p.inv_w);
            }
        }
        if (last_w) {
            w = 0;
            beta += stride;
        } else {
            ++w;
        }
    }
    if constexpr (C > 1) cluster_bar();  // no CTA leaves while a peer may still read its slots
}

template <int SCHEME, int G, bool FUSED, bool TAIL>
cudaError_t launch_group_g(const KParams &p0, int64_t b0, int64_t b1, cudaStream_t stream)
{
    constexpr int kGroupWarps = group_cta_warps<G>();
    constexpr int C = G > kGroupWarps ? G / kGroupWarps : 1;
    constexpr int GPC = G < kGroupWarps ? kGroupWarps / G : 1;
    KParams p = p0;
    p.codes_words = (int64_t)(32 * kSliceEPL) * p.bits / 32;  // code words of one 512-element slice
    auto kern = k_group<SCHEME, G, kGroupWarps, FUSED, TAIL>;
    const int64_t nbk = b1 - b0;
    const size_t smem = sizeof(GroupXchg<kGroupWarps>) + sizeof(GroupWarpSmem<SCHEME>) * kGroupWarps;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    cfg.blockDim = dim3(kGroupWarps * 32, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    int64_t groups;
    if constexpr (C > 1) {
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = C;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        cfg.gridDim = dim3((unsigned)(C * sms), 1, 1);
        int nclusters = 0;
        e = cudaOccupancyMaxActiveClusters(&nclusters, kern, &cfg);
        if (e != cudaSuccess) return e;
        if (nclusters < 1) return cudaErrorInvalidConfiguration;
        groups = nbk < nclusters ? nbk : nclusters;
        cfg.gridDim = dim3((unsigned)(groups * C), 1, 1);
    } else {
        int per_sm = 0;
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kGroupWarps * 32, smem);
        if (per_sm < 1) per_sm = 1;
        const int64_t cap = (int64_t)sms * per_sm * GPC;
        groups = nbk < cap ? nbk : cap;
        cfg.gridDim = dim3((unsigned)((groups + GPC - 1) / GPC), 1, 1);
        cfg.attrs = nullptr;
        cfg.numAttrs = 0;
    }
    e = cudaLaunchKernelEx(&cfg, kern, p, b0, b1);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <int SCHEME, bool FUSED, bool TAIL>
cudaError_t launch_group_range(const KParams &p, int64_t b0, int64_t b1, cudaStream_t stream)
{
    switch (p.d) {
    case 1024: return launch_group_g<SCHEME, 2, FUSED, TAIL>(p, b0, b1, stream);
    case 2048: return launch_group_g<SCHEME, 4, FUSED, TAIL>(p, b0, b1, stream);
    case 4096: return launch_group_g<SCHEME, 8, FUSED, TAIL>(p, b0, b1, stream);
    case 8192: return launch_group_g<SCHEME, 16, FUSED, TAIL>(p, b0, b1, stream);
    case 16384: return launch_group_g<SCHEME, 32, FUSED, TAIL>(p, b0, b1, stream);
    default: return launch_group_g<SCHEME, 64, FUSED, TAIL>(p, b0, b1, stream);
    }
}

// Every bucket of p: the full ones, then the ragged last one (if any) in a one-group launch.
template <int SCHEME, bool FUSED>
cudaError_t launch_group_fused(const KParams &p, cudaStream_t stream)
{
    const int64_t nfull = p.tail == p.d ? p.nb : p.nb - 1;
    if (nfull > 0) {
        const cudaError_t e = launch_group_range<SCHEME, FUSED, false>(p, 0, nfull, stream);
        if (e != cudaSuccess) return e;
    }
    return nfull < p.nb ? launch_group_range<SCHEME, FUSED, true>(p, nfull, p.nb, stream) : cudaSuccess;
}

}  // namespace
}  // namespace gq
