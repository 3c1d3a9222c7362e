// gq_decode.cu -- Dequantize + Aggregate: avg[i] = (sum_w level_w(code_w[i])) * (1/W).
//
// One warp owns two 128-element chunks at a time (grid-stride over the chunks of the vector),
// for any bucket size.  Lane l decodes elements 4l .. 4l+3 of each chunk: per worker it needs
// the one or two words holding its four codes (codes are packed densely, b bits each, in
// element order).  The level lookup is a register shuffle within segments of 2^b lanes: every
// segment holds the bucket's level table in its first L lanes, and a shuffle of width 2^b takes
// its source lane modulo 2^b, so the code needs no masking.  The loads of 8 workers and both
// chunks are issued together before any of them is used; the sum then runs in worker order in
// registers and the average is written once, with a 16-byte store.
#include "gq_device.cuh"

namespace gq {
namespace {

constexpr int kDecodeWarps = 4;
constexpr int kDecodeGroup = 8;  // workers whose loads are in flight together

template <bool QSGD, int BITS>
__global__ void __launch_bounds__(kDecodeWarps * 32) k_decode(const __grid_constant__ KParams p)
{
    constexpr int kWidth = 1 << BITS;
    const int lane = threadIdx.x & 31;
    const int slot = lane & (kWidth - 1);  // this lane's place in its 2^b-lane segment
    const int64_t nchunks = (p.n + 127) / 128;
    const int64_t first = (int64_t)blockIdx.x * kDecodeWarps + (threadIdx.x >> 5);
    const int64_t stride = (int64_t)gridDim.x * kDecodeWarps;
    const int log2d = 31 - __clz(p.d);
    const int chunks_per_bucket = p.d >> 7;
    const int bitoff = 4 * BITS * lane, wi = bitoff >> 5, sh = bitoff & 31;
    const bool cross = sh + 4 * BITS > 32;  // the field crosses a word boundary (b = 3 only)
    const bool has_level = slot < p.L;
    const float qr = (QSGD && slot < p.s) ? p.qratio[slot] : 0.0f;
    for (int64_t ch0 = first; ch0 < nchunks; ch0 += 2 * stride) {
        int64_t bk[2], woff[2];
        bool live[2];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int64_t ch = ch0 + i * stride;
            live[i] = ch < nchunks;
            bk[i] = (ch * 128) >> log2d;
            woff[i] = bk[i] * p.codes_words + (int64_t)(ch & (chunks_per_bucket - 1)) * 4 * BITS + wi;
        }
        float acc[2][4] = {{0.0f, 0.0f, 0.0f, 0.0f}, {0.0f, 0.0f, 0.0f, 0.0f}};
        for (int w0 = 0; w0 < p.W; w0 += kDecodeGroup) {
            uint32_t x[2][kDecodeGroup], y[2][kDecodeGroup];
            float lv[2][kDecodeGroup];
#pragma unroll
            for (int k = 0; k < kDecodeGroup; ++k) {
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    x[i][k] = 0u;
                    y[i][k] = 0u;
                    lv[i][k] = 0.0f;
                    if (live[i] && w0 + k < p.W) {
                        const unsigned char *msg = p.msg[w0 + k];
                        const uint32_t *cw = reinterpret_cast<const uint32_t *>(msg) + woff[i];
                        const float *tables = reinterpret_cast<const float *>(msg + p.levels_off);
                        x[i][k] = __ldg(cw);
                        if (BITS == 3 && cross) y[i][k] = __ldg(cw + 1);
                        if (QSGD) lv[i][k] = __ldg(tables + bk[i]);
                        else if (has_level) lv[i][k] = __ldg(tables + bk[i] * p.L + slot);
                    }
                }
            }
#pragma unroll
            for (int k = 0; k < kDecodeGroup; ++k) {
                if (w0 + k < p.W) {
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        const float level = QSGD ? __fmul_rn(lv[i][k], qr) : lv[i][k];
                        uint32_t f = x[i][k] >> sh;
                        if (BITS == 3 && cross) f |= y[i][k] << (32 - sh);
#pragma unroll
                        for (int c = 0; c < 4; ++c)
                            acc[i][c] = __fadd_rn(acc[i][c], __shfl_sync(kFull, level, (int)(f >> (BITS * c)), kWidth));
                    }
                }
            }
        }
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            if (!live[i]) continue;
            const int64_t e = (ch0 + i * stride) * 128 + 4 * lane;
            if (e + 3 < p.n) {
                __stcs(reinterpret_cast<float4 *>(p.avg + e),
                       make_float4(__fmul_rn(acc[i][0], p.inv_w), __fmul_rn(acc[i][1], p.inv_w),
                                   __fmul_rn(acc[i][2], p.inv_w), __fmul_rn(acc[i][3], p.inv_w)));
            } else {
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    if (e + c < p.n) p.avg[e + c] = __fmul_rn(acc[i][c], p.inv_w);
            }
        }
    }
}

template <bool QSGD, int BITS>
cudaError_t launch(const KParams &p, cudaStream_t stream)
{
    auto kern = k_decode<QSGD, BITS>;
    int dev = 0, sms = 0, per_sm = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kDecodeWarps * 32, 0);
    if (per_sm < 1) per_sm = 1;
    const int64_t nchunks = (p.n + 127) / 128;
    const int64_t need = (nchunks + 2 * kDecodeWarps - 1) / (2 * kDecodeWarps);
    const int64_t cap = (int64_t)sms * per_sm;
    const int grid = (int)(need < cap ? need : cap);
    if (grid <= 0) return cudaSuccess;
    kern<<<grid, kDecodeWarps * 32, 0, stream>>>(p);
    return cudaGetLastError();
}

template <bool QSGD>
cudaError_t launch_bits(const KParams &p, cudaStream_t stream)
{
    switch (p.bits) {
    case 1: return launch<QSGD, 1>(p, stream);
    case 2: return launch<QSGD, 2>(p, stream);
    case 3: return launch<QSGD, 3>(p, stream);
    default: return launch<QSGD, 4>(p, stream);
    }
}

}  // namespace

cudaError_t launch_decode(const KParams &p, cudaStream_t stream)
{
    const bool qsgd =
        p.scheme == GQ_QSGD || p.scheme == GQ_TERNGRAD || p.scheme == GQ_QSGD_NEAREST || p.scheme == GQ_QSGD_L2;
    return qsgd ? launch_bits<true>(p, stream) : launch_bits<false>(p, stream);
}

}  // namespace gq
