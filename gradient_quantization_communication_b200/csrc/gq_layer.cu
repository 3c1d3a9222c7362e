// gq_layer.cu -- TernGrad with one scale per parameter tensor (scheme GQ_TERNGRAD_LAYER).
//
// The glossary "Gradient Quantization" (section Ternary and binary quantization) says TernGrad
// sends three levels with a single scaling factor per layer.  The gradient is the concatenation
// of nseg tensors, tensor t holding elements [off[t], off[t+1]).  Per worker, m_t = max |v| over
// tensor t (v = g + r), and every element is rounded between the two of {-m_t, 0, +m_t} around
// it exactly as per-bucket TernGrad rounds (position y = v / m_t + 1, bracket k = trunc(y)
// clamped to [0, 1], up with probability y - k against the element's Philox draw).
//
// The message is the dense message's codes region (2-bit codes, bucket after bucket: since a
// bucket is a whole number of 128-element chunks, chunk c's codes are words 8c .. 8c+7) followed
// by the nseg scales.  Three kernels:
//   k_layer_max     grid (x, W): every warp a contiguous run of 512-element slices, |v| per
//                   element, a running maximum per lane and tensor, published by atomicMax
//                   (float bits, NaN above +inf) into the plan's scale scratch, zeroed before;
//                   the lanes that end on one tensor reduce first, so that a tensor's word sees
//                   about one atomic per warp;
//   k_layer_encode  every warp a contiguous run of 128-element chunks: per worker v, the
//                   tensor's scale (its reciprocal once per chunk when the lane's four elements
//                   share a tensor), the rounding, the residual, the packed codes; the W
//                   dequantized values are summed in registers in worker order and the average
//                   written once (fused); the scales are copied into each message, and the codes
//                   of the last bucket's chunks past n are written as zeros;
//   k_layer_decode  the same runs of chunks: the W messages' codes and scales, summed in worker
//                   order.
// A lane finds the tensor of its first element once by binary search over the offsets; its
// elements rise, so after that it only walks forward over the tensor boundaries it reaches.
#include "gq_round.cuh"

namespace gq {
namespace {

constexpr int kLayerWarps = 4;

// Largest t with off[t] <= i (the tensor holding element i; empty tensors are skipped).
__device__ __forceinline__ int segment_of(const int64_t *off, int nseg, int64_t i)
{
    int lo = 0, hi = nseg - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (__ldg(off + mid) <= i) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

__device__ __forceinline__ float scale_of(const unsigned int *bits, int t) { return __uint_as_float(bits[t]); }

// Largest |v| per worker and tensor: grid.y = worker; each warp a contiguous run of slices of
// 512 elements (lane l: elements 4l .. 4l+3 of each of four 128-element chunks), so that a lane's
// elements rise and it keeps one running maximum per tensor across slices.  A lane publishes its
// maximum (atomicMax on the bits: |v| >= 0 orders like its bits, NaN above everything) when its
// tensor changes; at the end the warp first reduces the maxima of the lanes that share a tensor,
// so that a tensor's word sees about one atomic per warp instead of one per lane and slice.
__global__ void __launch_bounds__(kLayerWarps * 32) k_layer_max(const __grid_constant__ KParams p)
{
    const int lane = threadIdx.x & 31;
    const int w = blockIdx.y;
    const float *g = p.g[w];
    const float *r = p.r[w];
    unsigned int *smax = p.seg_max + (int64_t)w * p.nseg;
    const int64_t nslices = (p.n + 511) / 512;
    const int64_t nwarps = (int64_t)gridDim.x * kLayerWarps;
    const int64_t per = (nslices + nwarps - 1) / nwarps;
    const int64_t s0 = ((int64_t)blockIdx.x * kLayerWarps + (threadIdx.x >> 5)) * per;
    const int64_t s1 = s0 + per < nslices ? s0 + per : nslices;
    int cur = -1;
    float run = 0.0f;
    // the lane's tensor and the next tensor's first element, advanced as its elements rise
    int t = s0 < s1 ? segment_of(p.seg_off, p.nseg, min(s0 * 512 + 4 * lane, p.n - 1)) : 0;
    int64_t nextb = t + 1 < p.nseg ? __ldg(p.seg_off + t + 1) : INT64_MAX;
    for (int64_t sl = s0; sl < s1; ++sl) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int64_t i0 = sl * 512 + 128 * j + 4 * lane;
            if (i0 >= p.n) break;
            float v[4];
            if (i0 + 3 < p.n) {
                float4 x = __ldg(reinterpret_cast<const float4 *>(g + i0));
                if (r) {
                    const float4 y = __ldg(reinterpret_cast<const float4 *>(r + i0));
                    x = make_float4(__fadd_rn(x.x, y.x), __fadd_rn(x.y, y.y), __fadd_rn(x.z, y.z), __fadd_rn(x.w, y.w));
                }
                v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
            } else {
#pragma unroll
                for (int c = 0; c < 4; ++c) v[c] = i0 + c < p.n ? (r ? __fadd_rn(g[i0 + c], r[i0 + c]) : g[i0 + c]) : 0.0f;
            }
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                if (i0 + c >= p.n) break;
                while (i0 + c >= nextb) {  // empty tensors are passed over
                    ++t;
                    nextb = t + 1 < p.nseg ? __ldg(p.seg_off + t + 1) : INT64_MAX;
                }
                if (t != cur) {
                    if (cur >= 0) atomicMax(smax + cur, __float_as_uint(run));
                    cur = t;
                    run = 0.0f;
                }
                run = fmax_nan(run, fabsf(v[c]));
            }
        }
    }
    const int c0 = __shfl_sync(kFull, cur, 0);
    if (__all_sync(kFull, cur == c0)) {
        const unsigned m = __reduce_max_sync(kFull, __float_as_uint(run));
        if (lane == 0 && c0 >= 0) atomicMax(smax + c0, m);
    } else if (cur >= 0) {
        atomicMax(smax + cur, __float_as_uint(run));
    }
}

// Encode (and, fused, average): a warp per 128-element chunk, lane l elements 4l .. 4l+3.
template <bool FUSED>
__global__ void __launch_bounds__(kLayerWarps * 32) k_layer_encode(const __grid_constant__ KParams p)
{
    const int lane = threadIdx.x & 31;
    const int64_t nchunks = (p.n + 127) / 128;
    const int64_t gtid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    // the scales into every message (and the region's padding), by the first threads
    for (int w = 0; w < p.W; ++w)
        if (p.msg[w]) {
            float *tab = reinterpret_cast<float *>(p.msg[w] + p.levels_off);
            const int pad = (p.nseg + 3) / 4 * 4;
            for (int64_t t = gtid; t < pad; t += (int64_t)gridDim.x * blockDim.x)
                tab[t] = t < p.nseg ? scale_of(p.seg_max + (int64_t)w * p.nseg, (int)t) : 0.0f;
        }
    // each warp a contiguous run of chunks, so that a lane's elements rise and its tensor index
    // only advances (no search per chunk)
    const int64_t nwarps = (int64_t)gridDim.x * kLayerWarps;
    const int64_t per = (nchunks + nwarps - 1) / nwarps;
    const int64_t c0 = ((int64_t)blockIdx.x * kLayerWarps + (threadIdx.x >> 5)) * per;
    const int64_t c1 = c0 + per < nchunks ? c0 + per : nchunks;
    int t = c0 < c1 ? segment_of(p.seg_off, p.nseg, min(c0 * 128 + 4 * lane, p.n - 1)) : 0;
    int64_t nextb = t + 1 < p.nseg ? __ldg(p.seg_off + t + 1) : INT64_MAX;
    for (int64_t ch = c0; ch < c1; ++ch) {
        const int64_t i0 = ch * 128 + 4 * lane;
        uint32_t valid = 0;
#pragma unroll
        for (int c = 0; c < 4; ++c) valid |= (i0 + c < p.n ? 1u : 0u) << c;
        int seg[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            while (i0 + c >= nextb && i0 + c < p.n) {  // empty tensors are passed over
                ++t;
                nextb = t + 1 < p.nseg ? __ldg(p.seg_off + t + 1) : INT64_MAX;
            }
            seg[c] = t;
        }
        const bool one_seg = seg[0] == seg[3];  // the common case: one scale for the lane's four
        float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        for (int w = 0; w < p.W; ++w) {
            const float *g = p.g[w];
            float *r = p.r[w];
            float v[4];
            if (valid == 0xfu) {
                float4 x = __ldcs(reinterpret_cast<const float4 *>(g + i0));
                if (r) {
                    const float4 y = __ldcs(reinterpret_cast<const float4 *>(r + i0));
                    x = make_float4(__fadd_rn(x.x, y.x), __fadd_rn(x.y, y.y), __fadd_rn(x.z, y.z), __fadd_rn(x.w, y.w));
                }
                v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
            } else {
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    v[c] = ((valid >> c) & 1u) ? (r ? __fadd_rn(g[i0 + c], r[i0 + c]) : g[i0 + c]) : 0.0f;
            }
            const uint4 rnd = draws4(p, (uint64_t)(i0 >> 2), p.worker0 + (uint32_t)w);
            const uint32_t words[4] = {rnd.x, rnd.y, rnd.z, rnd.w};
            const unsigned int *smax = p.seg_max + (int64_t)w * p.nseg;
            int code[4];
            float q[4];
            const float m0 = scale_of(smax, seg[0]);
            const float inv_m0 = m0 > 0.0f ? __frcp_rn(m0) : 0.0f;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float m = one_seg ? m0 : scale_of(smax, seg[c]);
                const float inv_m = one_seg ? inv_m0 : (m > 0.0f ? __frcp_rn(m) : 0.0f);
                const float y = __fadd_rn(__fmul_rn(v[c], inv_m), 1.0f);  // (v / m + 1) * (s - 1) / 2, s = 3
                const int k = min(max(__float2int_rz(y), 0), 1);
                const float pu = __fsub_rn(y, (float)k);
                const int cd = k + (unit_float(words[c]) < pu ? 1 : 0);
                code[c] = ((valid >> c) & 1u) ? cd : 0;
                q[c] = __fmul_rn(m, p.qratio[cd]);
                if (!(m <= FLT_MAX) && ((valid >> c) & 1u)) atomicOr(p.status, kStatusNonFinite);
            }
            if (r) {
                if (valid == 0xfu) {
                    __stcs(reinterpret_cast<float4 *>(r + i0), make_float4(__fsub_rn(v[0], q[0]), __fsub_rn(v[1], q[1]),
                                                                           __fsub_rn(v[2], q[2]), __fsub_rn(v[3], q[3])));
                } else {
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        if ((valid >> c) & 1u) r[i0 + c] = __fsub_rn(v[c], q[c]);
                }
            }
            if (p.msg[w]) pack_chunk<2>(p, lane, code, reinterpret_cast<uint32_t *>(p.msg[w]) + ch * 8);
            if (FUSED) {
#pragma unroll
                for (int c = 0; c < 4; ++c) acc[c] = __fadd_rn(acc[c], q[c]);
            }
        }
        if (FUSED) {
            if (valid == 0xfu) {
                __stcs(reinterpret_cast<float4 *>(p.avg + i0),
                       make_float4(__fmul_rn(acc[0], p.inv_w), __fmul_rn(acc[1], p.inv_w), __fmul_rn(acc[2], p.inv_w),
                                   __fmul_rn(acc[3], p.inv_w)));
            } else {
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    if ((valid >> c) & 1u) p.avg[i0 + c] = __fmul_rn(acc[c], p.inv_w);
            }
        }
    }
    // the codes of the last bucket past n (bucket sizes are multiples of 128)
    const int64_t nchunks_msg = (p.n + p.d - 1) / p.d * (p.d / 128);
    for (int64_t ch = nchunks + (int64_t)blockIdx.x * kLayerWarps + (threadIdx.x >> 5); ch < nchunks_msg;
         ch += (int64_t)gridDim.x * kLayerWarps)
        if (lane < 8)
            for (int w = 0; w < p.W; ++w)
                if (p.msg[w]) reinterpret_cast<uint32_t *>(p.msg[w])[ch * 8 + lane] = 0u;
}

// Decode + average of W messages: a warp per chunk, lane l elements 4l .. 4l+3 (its 8 code
// bits are bits 8 (l % 4) .. of word l / 4 of the chunk's 8 words).
__global__ void __launch_bounds__(kLayerWarps * 32) k_layer_decode(const __grid_constant__ KParams p)
{
    const int lane = threadIdx.x & 31;
    const int64_t nchunks = (p.n + 127) / 128;
    // contiguous runs of chunks per warp: the lane's tensor index only advances
    const int64_t nwarps = (int64_t)gridDim.x * kLayerWarps;
    const int64_t per = (nchunks + nwarps - 1) / nwarps;
    const int64_t c0 = ((int64_t)blockIdx.x * kLayerWarps + (threadIdx.x >> 5)) * per;
    const int64_t c1 = c0 + per < nchunks ? c0 + per : nchunks;
    int t = c0 < c1 ? segment_of(p.seg_off, p.nseg, min(c0 * 128 + 4 * lane, p.n - 1)) : 0;
    int64_t nextb = t + 1 < p.nseg ? __ldg(p.seg_off + t + 1) : INT64_MAX;
    for (int64_t ch = c0; ch < c1; ++ch) {
        const int64_t i0 = ch * 128 + 4 * lane;
        if (i0 >= p.n) continue;
        int seg[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            while (i0 + c >= nextb && i0 + c < p.n) {  // empty tensors are passed over
                ++t;
                nextb = t + 1 < p.nseg ? __ldg(p.seg_off + t + 1) : INT64_MAX;
            }
            seg[c] = t;
        }
        float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        for (int w = 0; w < p.W; ++w) {
            const unsigned char *msg = p.msg[w];
            const uint32_t word = __ldg(reinterpret_cast<const uint32_t *>(msg) + ch * 8 + (lane >> 2));
            const uint32_t f = word >> (8 * (lane & 3));
            const float *tab = reinterpret_cast<const float *>(msg + p.levels_off);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int cd = (int)((f >> (2 * c)) & 3u);
                acc[c] = __fadd_rn(acc[c], __fmul_rn(__ldg(tab + seg[c]), p.qratio[cd < 3 ? cd : 2]));
            }
        }
        if (i0 + 3 < p.n) {
            __stcs(reinterpret_cast<float4 *>(p.avg + i0),
                   make_float4(__fmul_rn(acc[0], p.inv_w), __fmul_rn(acc[1], p.inv_w), __fmul_rn(acc[2], p.inv_w),
                               __fmul_rn(acc[3], p.inv_w)));
        } else {
#pragma unroll
            for (int c = 0; c < 4; ++c)
                if (i0 + c < p.n) p.avg[i0 + c] = __fmul_rn(acc[c], p.inv_w);
        }
    }
}

int grid_for(const void *kern, int64_t items)
{
    int dev = 0, sms = 0, per_sm = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kLayerWarps * 32, 0);
    if (per_sm < 1) per_sm = 1;
    const int64_t need = (items + kLayerWarps - 1) / kLayerWarps;
    const int64_t cap = (int64_t)sms * per_sm;
    return (int)(need < cap ? (need > 0 ? need : 1) : cap);
}

}  // namespace

// Scales (into p.seg_max, zeroed here) then the encode of p.W workers; fused when p.avg is set.
cudaError_t launch_layer_encode(const KParams &p, cudaStream_t stream)
{
    cudaError_t e = cudaMemsetAsync(p.seg_max, 0, sizeof(unsigned int) * (size_t)p.nseg * p.W, stream);
    if (e != cudaSuccess) return e;
    // grid (x, W): the x blocks of a worker share the resident CTAs of the device with the others
    const int64_t nslices = (p.n + 511) / 512;
    const int per_worker = (grid_for(reinterpret_cast<const void *>(k_layer_max), nslices * p.W) + p.W - 1) / p.W;
    k_layer_max<<<dim3((unsigned)per_worker, (unsigned)p.W), kLayerWarps * 32, 0, stream>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int64_t nchunks = (p.n + 127) / 128;
    if (p.avg) {
        k_layer_encode<true><<<grid_for(reinterpret_cast<const void *>(k_layer_encode<true>), nchunks), kLayerWarps * 32, 0,
                               stream>>>(p);
    } else {
        k_layer_encode<false><<<grid_for(reinterpret_cast<const void *>(k_layer_encode<false>), nchunks), kLayerWarps * 32, 0,
                                stream>>>(p);
    }
    return cudaGetLastError();
}

cudaError_t launch_layer_decode(const KParams &p, cudaStream_t stream)
{
    const int64_t nchunks = (p.n + 127) / 128;
    k_layer_decode<<<grid_for(reinterpret_cast<const void *>(k_layer_decode), nchunks), kLayerWarps * 32, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace gq
