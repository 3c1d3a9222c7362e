// gq_noalloc.cu -- gq_quant_error_noalloc: the quantization-error measurement of
// gq_quant_error for callers that cannot allocate device memory.
//
// Who needs it: code that runs where cudaMalloc is off limits -- inside a framework's own
// caching allocator or memory pool (which may not be re-entered), in a process whose device
// memory is fully reserved up front, or in a plugin that is handed buffers but no allocator.
// Such callers cannot create a plan (gq_plan_create allocates the status word and the error
// scratch), so this entry point takes the configuration directly and keeps its scratch in a
// file-scope __device__ array instead: every GPU that loads the library holds that array
// (about 384 KB) until the process exits.
//
// The scratch is shared by every call on a device and keeps the last call's contents.  What
// must start at zero (the status word the kernels OR into) is cleared at the start of every
// call; the per-bucket rows are always fully written before they are read.  Two calls whose
// work overlaps on the GPU (different streams, or different host threads) race on the array.
#include <cstring>
#include <mutex>

#include "gq_internal.h"

namespace {

// Largest number of buckets (ceil(n / d)) a call may have.
constexpr int64_t kMaxBuckets = GQ_NOALLOC_MAX_BUCKETS;
constexpr int64_t kStatusBytes = 256;  // the status word, padded to keep the rows 256-byte aligned

// [status word | padding][per-bucket rows: 3 doubles each][first-pass rows: 3 doubles each]
constexpr size_t kScratchBytes = kStatusBytes + sizeof(double) * 3 * (kMaxBuckets + (kMaxBuckets + 4095) / 4096);
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
unsigned char *g_scratch_ptr[kMaxDevices];  // device address of g_noalloc_scratch, per device
std::mutex g_setup_mutex;

// Device address of the scratch array on the current device (looked up once per device: in
// host code the array's name is only a host-side stand-in, never a device address).
gq_status_t scratch_address(int dev, unsigned char **out)
{
    if (dev < 0 || dev >= kMaxDevices) return GQ_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return GQ_ERR_CUDA;
        g_scratch_ptr[dev] = static_cast<unsigned char *>(p);
    }
    *out = g_scratch_ptr[dev];
    return GQ_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" GQ_API gq_status_t gq_quant_error_noalloc(const gq_config_t *cfg, uint32_t worker, uint64_t step,
                                                     const float *grad, const float *residual, double *out,
                                                     void *stream)
{
    const gq_status_t st = gq_config_check(cfg);
    if (st != GQ_OK) return st;
    if (!out) return GQ_ERR_INVALID;
    gq_config_t c = *cfg;
    if (c.scheme == GQ_TERNGRAD && c.levels == 0) c.levels = 3;
    if ((c.scheme == GQ_BINGRAD_B || c.scheme == GQ_BINGRAD_PB || c.scheme == GQ_SIGNSGD) && c.levels == 0)
        c.levels = 2;
    const int64_t nb = (c.n + c.bucket - 1) / c.bucket;
    if (nb > kMaxBuckets) return GQ_ERR_UNSUPPORTED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (c.n == 0) return cudaMemsetAsync(out, 0, 3 * sizeof(double), s) == cudaSuccess ? GQ_OK : GQ_ERR_CUDA;
    if (!grad || !aligned16(grad)) return GQ_ERR_INVALID;
    if ((c.error_feedback != 0) != (residual != nullptr)) return GQ_ERR_INVALID;
    if (residual && !aligned16(residual)) return GQ_ERR_INVALID;

    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return GQ_ERR_CUDA;
    unsigned char *scratch = nullptr;
    const gq_status_t sa = scratch_address(dev, &scratch);
    if (sa != GQ_OK) return sa;
    unsigned int *status = reinterpret_cast<unsigned int *>(scratch);
    double *part = reinterpret_cast<double *>(scratch + kStatusBytes);
    if (cudaMemsetAsync(status, 0, sizeof(unsigned int), s) != cudaSuccess) return GQ_ERR_CUDA;

    size_t msg_bytes = 0, codes_off = 0, levels_off = 0;
    if (gq_message_layout(&c, &msg_bytes, &codes_off, &levels_off) != GQ_OK) return GQ_ERR_INVALID;
    int bits = 0;
    while ((1 << bits) < c.levels) ++bits;
    gq::KParams p;
    memset(&p, 0, sizeof p);
    p.scheme = c.scheme;
    p.s = c.levels;
    p.bits = bits;
    p.L = (c.scheme == GQ_QSGD || c.scheme == GQ_TERNGRAD || c.scheme == GQ_QSGD_NEAREST || c.scheme == GQ_QSGD_L2) ? 1
          : (c.scheme == GQ_BINGRAD_B || c.scheme == GQ_BINGRAD_PB || c.scheme == GQ_SIGNSGD) ? 2
                                                                                               : c.levels;
    p.d = c.bucket;
    p.W = 1;
    p.n = c.n;
    p.nb = nb;
    p.tail = (int)(c.n - (nb - 1) * c.bucket);
    p.clip = c.clip_sigma;
    p.key0 = (uint32_t)c.seed;
    p.key1 = (uint32_t)(c.seed >> 32);
    for (int i = 0; i < 10; ++i) {
        p.rk0[i] = p.key0 + (uint32_t)i * 0x9E3779B9u;
        p.rk1[i] = p.key1 + (uint32_t)i * 0xBB67AE85u;
    }
    p.step_lo = (uint32_t)step;
    p.step_m1 = 0xCD9E8D57ull * (unsigned long long)p.step_lo;
    p.worker0 = worker;
    p.inv_w = 1.0f;
    for (int k = 0; k < c.levels; ++k) p.qratio[k] = (float)(2 * k - (c.levels - 1)) / (float)(c.levels - 1);
    p.codes_words = (int64_t)c.bucket * bits / 32;
    p.levels_off = (int64_t)levels_off;
    p.g[0] = grad;
    p.r[0] = const_cast<float *>(residual);  // read only in this mode
    p.status = status;
    cudaError_t e = c.bucket <= 512 ? gq::launch_warp_err(p, part, s) : gq::launch_cta_err(p, part, s);
    if (e != cudaSuccess) return GQ_ERR_CUDA;
    return gq::launch_err_reduce(part, nb, part + 3 * nb, out, s) == cudaSuccess ? GQ_OK : GQ_ERR_CUDA;
}
