// gq_internal.h -- kernel parameter block and launch entry points shared by the library's
// translation units (not part of the public ABI).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "gq.h"

namespace gq {

// Everything a quantization kernel needs, passed by value as a __grid_constant__ parameter.
struct KParams {
    int scheme;          // gq_scheme_t
    int s;               // levels
    int bits;            // ceil(log2 s)
    int L;               // floats per level table in the message
    int d;               // bucket size (power of two)
    int W;               // workers handled by this launch
    int64_t n;           // elements per worker
    int64_t nb;          // buckets per worker
    int tail;            // valid elements of the last bucket (1..d)
    float clip;          // c of the +-c*sigma clip, 0 = off
    uint32_t key0, key1; // Philox key (seed)
    uint32_t rk0[10];    // Philox round keys: key0 + i * 0x9E3779B9
    uint32_t rk1[10];    //                    key1 + i * 0xBB67AE85
    uint32_t step_lo;    // step, low word
    unsigned long long step_m1;  // 0xCD9E8D57 * step_lo (Philox round-1 product of counter word 2)
    uint32_t worker0;    // Philox worker index of worker slot 0
    float inv_w;         // 1/W for the average
    float qratio[GQ_MAX_QSGD_LEVELS];  // QSGD level k = m * qratio[k], qratio[k] = (2k-(s-1))/(s-1)
    int64_t codes_words; // words of packed codes per bucket (d*b/32)
    int64_t levels_off;  // byte offset of the level tables inside a message
    const float *g[GQ_MAX_WORKERS];
    float *r[GQ_MAX_WORKERS];          // NULL when error feedback is off
    unsigned char *msg[GQ_MAX_WORKERS];// NULL: do not write the message
    float *avg;                        // fused kernels only
    unsigned int *status;              // plan status word
    int fmt_s;                         // base-s messages of s levels (3, 5, 9), 0 = dense; codes_words
                                       // then counts the bucket's base-s words
    const int64_t *seg_off;            // GQ_TERNGRAD_LAYER: nseg + 1 tensor offsets (device)
    int nseg;
    unsigned int *seg_max;             // GQ_TERNGRAD_LAYER: W x nseg scales (float bits, device scratch)
};

// Status bits raised by kernels.
constexpr unsigned kStatusNonFinite = 1u;
constexpr unsigned kStatusTimeout = 2u;  // a bounded wait on a bulk copy gave up

// Register-resident path (d = 128, 256, 512): one warp per bucket index.
// The ragged last bucket (when n is not a multiple of d) goes to a one-warp launch of the same
// code with guarded loads, so the main kernel carries no tail logic.
cudaError_t launch_warp_encode(const KParams &p, bool fused, cudaStream_t stream);
// Shared-memory path (d = 1024 .. 32768): one CTA per bucket index walking the p.W workers;
// with p.avg set, the average of the dequantized values is accumulated on chip and written.
cudaError_t launch_cta_encode(const KParams &p, cudaStream_t stream);
// d = 1024 .. 32768, ORQ or QSGD / TernGrad, no clipping: every bucket spread over a group of
// d / 512 warps (gq_group.cuh); the ragged last one in a second, one-group launch.
cudaError_t launch_group_orq(const KParams &p, bool fused, cudaStream_t stream);
cudaError_t launch_group_qsgd(const KParams &p, bool fused, cudaStream_t stream);
// Dequantize + aggregate for any d.
cudaError_t launch_decode(const KParams &p, cudaStream_t stream);
// GQ_TERNGRAD_LAYER: the tensors' scales (into p.seg_max), then the encode of p.W workers (the
// average too when p.avg is set); and the decode + average of p.W messages.
cudaError_t launch_layer_encode(const KParams &p, cudaStream_t stream);
cudaError_t launch_layer_decode(const KParams &p, cudaStream_t stream);

// gq_quant_error: per-bucket binary64 error sums into part[3 * bucket + k] (one worker, nothing
// else written), then their fixed-order reduction into out[3].  The scratch holds
// err_scratch_doubles(nb) doubles: the nb bucket rows followed by the rows of the first pass.
// With a status word, the reduction writes NaN to out[0..2] when any of its bits is set.
cudaError_t launch_warp_err(const KParams &p, double *part, cudaStream_t stream);
cudaError_t launch_cta_err(const KParams &p, double *part, cudaStream_t stream);
int64_t err_scratch_doubles(int64_t nb);
cudaError_t launch_err_reduce(const double *part, int64_t nb, double *tmp, double *out, cudaStream_t stream,
                              const unsigned int *status = nullptr);
// Resident CTAs per SM of kernel `kern` at `threads` threads and `smem` bytes of dynamic shared
// memory on the current device (at least 1), and the device's SM count; the kernel's dynamic
// shared memory limit is raised to `smem` first.  Cached per kernel, block shape and device: the
// queries cost microseconds each, more than the launch of a small step.
cudaError_t kernel_occupancy(const void *kern, int threads, size_t smem, int *per_sm, int *sms);

// One warp waiting, with the kernels' bounded wait, on a barrier that nothing completes; raises
// kStatusTimeout in *status after limit_ns.
cudaError_t launch_wait_selftest(unsigned int *status, unsigned long long limit_ns, cudaStream_t stream);

}  // namespace gq
