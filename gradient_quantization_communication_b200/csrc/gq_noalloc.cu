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
// call; the per-bucket rows are fully written before they are read unless a kernel stops
// early (a bounded wait that gave up), and then the status word is set and the reduction
// writes NaN to all three outputs instead of summing rows left by an earlier call.  Two calls
// whose work overlaps on the GPU (different streams, or different host threads) race on the
// array.
//
// In host code the array's name is a host-side stand-in, never a device address: the address
// is looked up with cudaGetSymbolAddress with the device current.  The lookup is cached per
// device together with the identity of the context it was made in (cuCtxGetId, reached through
// cudaGetDriverEntryPoint, so the library needs no link to the driver library); a call made in
// another context of that device (after cudaDeviceReset, say) looks the address up again.
#include <cuda.h>
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
struct ScratchEntry {
    unsigned long long ctx_id;  // context the address belongs to (0: none looked up yet)
    unsigned char *ptr;         // device address of g_noalloc_scratch in that context
};
ScratchEntry g_scratch[kMaxDevices];
std::mutex g_setup_mutex;

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);
CtxGetCurrentFn g_ctx_get_current = nullptr;
CtxGetIdFn g_ctx_get_id = nullptr;

// Identity of the calling thread's current context (unique for the life of the process).
gq_status_t current_context_id(unsigned long long *id)
{
    if (!g_ctx_get_current || !g_ctx_get_id) {
        void *f1 = nullptr, *f2 = nullptr;
        cudaDriverEntryPointQueryResult q1, q2;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &q1) != cudaSuccess ||
            q1 != cudaDriverEntryPointSuccess || !f1)
            return GQ_ERR_CUDA;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &q2) != cudaSuccess ||
            q2 != cudaDriverEntryPointSuccess || !f2)
            return GQ_ERR_CUDA;
        g_ctx_get_current = reinterpret_cast<CtxGetCurrentFn>(f1);
        g_ctx_get_id = reinterpret_cast<CtxGetIdFn>(f2);
    }
    CUcontext ctx = nullptr;
    if (g_ctx_get_current(&ctx) != CUDA_SUCCESS || !ctx) return GQ_ERR_CUDA;
    return g_ctx_get_id(ctx, id) == CUDA_SUCCESS ? GQ_OK : GQ_ERR_CUDA;
}

// Device address of the scratch array on the current device.  In host code the array's name is
// only a host-side stand-in, never a device address, so it is looked up with
// cudaGetSymbolAddress, once per device and context: the first call on a device (and the first
// after that device's context was replaced) does the lookup and must come before any stream
// capture; later calls reuse it.
gq_status_t scratch_address(int dev, unsigned char **out)
{
    if (dev < 0 || dev >= kMaxDevices) return GQ_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    unsigned long long id = 0;
    const gq_status_t st = current_context_id(&id);
    if (st != GQ_OK) return st;
    if (g_scratch[dev].ctx_id != id || !g_scratch[dev].ptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return GQ_ERR_CUDA;
        g_scratch[dev].ptr = static_cast<unsigned char *>(p);
        g_scratch[dev].ctx_id = id;
    }
    *out = g_scratch[dev].ptr;
    return GQ_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" GQ_API gq_status_t gq_quant_error_noalloc(const gq_config_t *cfg, uint32_t worker, uint64_t step,
                                                     const float *grad, const float *residual, double *out,
                                                     void *stream)
{
    if (!cfg || !out) return GQ_ERR_INVALID;
    gq_config_t c = *cfg;
    c.workers = 1;  // one worker's gradient: the configured worker count plays no part
    const gq_status_t st = gq_config_check(&c);
    if (st != GQ_OK) return st;
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
    // the reduction reads the status word: a kernel that stopped early (or saw a non-finite
    // value) makes all three outputs NaN
    return gq::launch_err_reduce(part, nb, part + 3 * nb, out, s, status) == cudaSuccess ? GQ_OK : GQ_ERR_CUDA;
}
