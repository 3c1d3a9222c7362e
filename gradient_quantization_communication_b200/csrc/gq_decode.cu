// gq_decode.cu -- Dequantize + Aggregate: avg[i] = (sum_w level_w(code_w[i])) * (1/W).
//
// One warp owns a tile of 512 consecutive elements (four 128-element chunks), for any bucket
// size.  Per worker and chunk lane l reads the one or two words holding the codes of its
// elements 128m + 4l + c (codes are packed densely, b bits each, in element order) and looks
// the levels up with a register shuffle (lane k holds level k of the bucket).  The
// sum runs in worker order in registers; the average is written once, with 16-byte stores.
#include "gq_device.cuh"

namespace gq {
namespace {

constexpr int kDecodeWarps = 8;

template <bool QSGD>
__global__ void __launch_bounds__(kDecodeWarps * 32) k_decode(const __grid_constant__ KParams p)
{
    const int lane = threadIdx.x & 31;
    const int64_t ntiles = (p.n + 511) / 512;
    const int64_t first = (int64_t)blockIdx.x * kDecodeWarps + (threadIdx.x >> 5);
    const int64_t stride = (int64_t)gridDim.x * kDecodeWarps;
    const int log2d = 31 - __clz(p.d);
    const int chunks_per_bucket = p.d >> 7;
    for (int64_t tile = first; tile < ntiles; tile += stride) {
        float acc[16];
#pragma unroll
        for (int t = 0; t < 16; ++t) acc[t] = 0.0f;
        for (int w = 0; w < p.W; ++w) {
            const unsigned char *msg = p.msg[w];
            const uint32_t *codes = reinterpret_cast<const uint32_t *>(msg);
            const float *tables = reinterpret_cast<const float *>(msg + p.levels_off);
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int64_t e0 = tile * 512 + 128 * m;
                if (e0 >= p.n) break;
                const int64_t bk = e0 >> log2d;
                const int cb = (int)((e0 >> 7) & (chunks_per_bucket - 1));
                const uint32_t *cw = codes + bk * p.codes_words + (int64_t)cb * 4 * p.bits;
                // lane k holds level k of this bucket
                float lv = 0.0f;
                if (QSGD) {
                    const float mscale = __ldg(tables + bk);
                    if (lane < p.s) lv = __fmul_rn(mscale, p.qratio[lane]);
                } else if (lane < p.L) {
                    lv = __ldg(tables + bk * p.L + lane);
                }
                // lane l's four codes: the 4b-bit field at bit 4b*l of the chunk (it crosses a
                // word boundary only for b = 3)
                const int b = p.bits;
                const int bitoff = 4 * b * lane, wi = bitoff >> 5, sh = bitoff & 31;
                uint32_t x = __ldg(cw + wi) >> sh;
                if (sh + 4 * b > 32) x |= __ldg(cw + wi + 1) << (32 - sh);
                const uint32_t cmask = (1u << b) - 1u;
                const uint32_t code0 = x & cmask, code1 = (x >> b) & cmask, code2 = (x >> (2 * b)) & cmask,
                               code3 = (x >> (3 * b)) & cmask;
                acc[4 * m + 0] = __fadd_rn(acc[4 * m + 0], __shfl_sync(kFull, lv, (int)code0));
                acc[4 * m + 1] = __fadd_rn(acc[4 * m + 1], __shfl_sync(kFull, lv, (int)code1));
                acc[4 * m + 2] = __fadd_rn(acc[4 * m + 2], __shfl_sync(kFull, lv, (int)code2));
                acc[4 * m + 3] = __fadd_rn(acc[4 * m + 3], __shfl_sync(kFull, lv, (int)code3));
            }
        }
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const int64_t e = tile * 512 + 128 * m + 4 * lane;
            if (e + 3 < p.n) {
                __stcs(reinterpret_cast<float4 *>(p.avg + e),
                       make_float4(__fmul_rn(acc[4 * m], p.inv_w), __fmul_rn(acc[4 * m + 1], p.inv_w),
                                   __fmul_rn(acc[4 * m + 2], p.inv_w), __fmul_rn(acc[4 * m + 3], p.inv_w)));
            } else {
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    if (e + c < p.n) p.avg[e + c] = __fmul_rn(acc[4 * m + c], p.inv_w);
            }
        }
    }
}

template <bool QSGD>
cudaError_t launch(const KParams &p, cudaStream_t stream)
{
    int dev = 0, sms = 0, per_sm = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_decode<QSGD>, kDecodeWarps * 32, 0);
    if (per_sm < 1) per_sm = 1;
    const int64_t ntiles = (p.n + 511) / 512;
    const int64_t need = (ntiles + kDecodeWarps - 1) / kDecodeWarps;
    const int64_t cap = (int64_t)sms * per_sm;
    const int grid = (int)(need < cap ? need : cap);
    if (grid <= 0) return cudaSuccess;
    k_decode<QSGD><<<grid, kDecodeWarps * 32, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const KParams &p, cudaStream_t stream)
{
    return (p.scheme == GQ_QSGD || p.scheme == GQ_TERNGRAD) ? launch<true>(p, stream) : launch<false>(p, stream);
}

}  // namespace gq
