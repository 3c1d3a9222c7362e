// gq_err.cu -- the two-pass fixed-order reduction of gq_quant_error's per-bucket sums.
//
// part[3 * b + k] holds the three binary64 sums of bucket b.  Pass 1: CTA c adds buckets
// [4096 c, 4096 (c + 1)) (thread t: buckets 4096 c + t, + 256, ... in order, then a fixed tree
// over the 256 threads) into tmp[3 c + k].  Pass 2: one CTA adds the tmp rows the same way into
// out[k].  The result depends only on the per-bucket sums, never on the launch shape.  Given a
// status word, pass 2 writes NaN to out[0..2] instead when any status bit is set (a kernel
// stopped early, so some rows were not written by this call).
#include "gq_device.cuh"

namespace gq {
namespace {

constexpr int kRedThreads = 256;
constexpr int kRedChunk = 4096;

__device__ __forceinline__ void block_tree_sum3(double (&v)[3], double (*sh)[kRedThreads])
{
    const int t = threadIdx.x;
#pragma unroll
    for (int k = 0; k < 3; ++k) sh[k][t] = v[k];
    __syncthreads();
    for (int h = kRedThreads / 2; h > 0; h >>= 1) {
        if (t < h) {
#pragma unroll
            for (int k = 0; k < 3; ++k) sh[k][t] = __dadd_rn(sh[k][t], sh[k][t + h]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int k = 0; k < 3; ++k) v[k] = sh[k][0];
}

__global__ void __launch_bounds__(kRedThreads) k_err_pass(const double *in, int64_t rows, int64_t rows_per_cta,
                                                          double *out, const unsigned int *status)
{
    __shared__ double sh[3][kRedThreads];
    const int64_t r0 = (int64_t)blockIdx.x * rows_per_cta;
    int64_t r1 = r0 + rows_per_cta;
    if (r1 > rows) r1 = rows;
    double v[3] = {0.0, 0.0, 0.0};
    for (int64_t r = r0 + threadIdx.x; r < r1; r += kRedThreads) {
#pragma unroll
        for (int k = 0; k < 3; ++k) v[k] = __dadd_rn(v[k], in[3 * r + k]);
    }
    block_tree_sum3(v, sh);
    if (threadIdx.x < 3) {
        const bool failed = status && *status != 0u;
        out[3 * blockIdx.x + threadIdx.x] = failed ? __longlong_as_double(0x7ff8000000000000ll) : v[threadIdx.x];
    }
}

}  // namespace

int64_t err_scratch_doubles(int64_t nb) { return 3 * (nb + (nb + kRedChunk - 1) / kRedChunk); }

cudaError_t launch_err_reduce(const double *part, int64_t nb, double *tmp, double *out, cudaStream_t stream,
                              const unsigned int *status)
{
    if (nb <= 0) return cudaMemsetAsync(out, 0, 3 * sizeof(double), stream);
    const int64_t nc = (nb + kRedChunk - 1) / kRedChunk;
    k_err_pass<<<(unsigned)nc, kRedThreads, 0, stream>>>(part, nb, kRedChunk, tmp, nullptr);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    k_err_pass<<<1, kRedThreads, 0, stream>>>(tmp, nc, nc, out, status);
    return cudaGetLastError();
}

}  // namespace gq
