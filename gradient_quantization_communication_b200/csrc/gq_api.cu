// gq_api.cu -- host side of the C ABI declared in include/gq.h: argument checks, the plan,
// kernel selection and the status word.
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "gq_internal.h"

struct gq_plan {
    gq_config_t cfg;  // normalised (levels filled in)
    int bits;
    int L;
    int64_t nb;
    int tail;
    size_t msg_bytes, codes_off, levels_off;
    int device;
    unsigned int *status;  // device word
    double *err_scratch;   // gq_quant_error: per-bucket sums and first-pass rows
    int64_t *seg_off;      // GQ_TERNGRAD_LAYER: the tensors' offsets (device), NULL until set
    int nseg;
    unsigned int *seg_max; // GQ_TERNGRAD_LAYER: W x nseg scales (device scratch)
    int fmt_s;             // base-s messages of s levels (GQ_FORMAT_BASE_S), 0 = dense
    int64_t base_words;    // base-s words per bucket
};

namespace gq {

cudaError_t kernel_occupancy(const void *kern, int threads, size_t smem, int *per_sm, int *sms)
{
    // The dynamic shared memory limit is the kernel's own state on the device, shared by every
    // launch of it: it is raised to the largest size asked for so far and never lowered, so that
    // a cached answer for a larger size stays launchable after a smaller one.
    struct Occ {
        const void *kern;
        int threads, device;
        size_t smem;
        int per_sm, sms;
    };
    struct Limit {
        const void *kern;
        int device;
        size_t smem;
    };
    static std::mutex mu;
    static std::vector<Occ> occ;
    static std::vector<Limit> limits;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    Limit *lim = nullptr;
    for (Limit &x : limits)
        if (x.kern == kern && x.device == dev) lim = &x;
    if (smem > 0 && (!lim || lim->smem < smem)) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        if (lim) lim->smem = smem;
        else limits.push_back(Limit{kern, dev, smem});
    }
    for (const Occ &x : occ)
        if (x.kern == kern && x.threads == threads && x.smem == smem && x.device == dev) {
            *per_sm = x.per_sm;
            *sms = x.sms;
            return cudaSuccess;
        }
    int n_sm = 0, per = 0;
    e = cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, kern, threads, smem);
    if (e != cudaSuccess) return e;
    if (per < 1) per = 1;
    *per_sm = per;
    *sms = n_sm;
    occ.push_back(Occ{kern, threads, dev, smem, per, n_sm});
    return cudaSuccess;
}

}  // namespace gq

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int bits_for(int s)
{
    int b = 0;
    while ((1 << b) < s) ++b;
    return b;
}

int table_len(int scheme, int s)
{
    if (scheme == GQ_QSGD || scheme == GQ_TERNGRAD || scheme == GQ_QSGD_NEAREST || scheme == GQ_QSGD_L2) return 1;
    if (scheme == GQ_BINGRAD_B || scheme == GQ_BINGRAD_PB || scheme == GQ_SIGNSGD) return 2;
    return s;
}

// Validates *in and writes the normalised configuration to *out.
gq_status_t normalise(const gq_config_t *in, gq_config_t *out)
{
    if (!in) return GQ_ERR_INVALID;
    gq_config_t c = *in;
    switch (c.scheme) {
    case GQ_ORQ:
        if (c.levels < 2 || c.levels > GQ_MAX_LEVELS) return GQ_ERR_INVALID;
        break;
    case GQ_QSGD:
    case GQ_QSGD_NEAREST:
    case GQ_QSGD_L2:
        // 2 .. 16 levels take 1 .. 4-bit codes; 129 .. 256 levels take 8-bit codes
        if (c.levels < 2 || (c.levels > GQ_MAX_LEVELS && c.levels <= 128) || c.levels > GQ_MAX_QSGD_LEVELS)
            return GQ_ERR_INVALID;
        break;
    case GQ_TERNGRAD:
        if (c.levels == 0) c.levels = 3;
        if (c.levels != 3) return GQ_ERR_INVALID;
        break;
    case GQ_BINGRAD_B:
    case GQ_BINGRAD_PB:
    case GQ_SIGNSGD:
        if (c.levels == 0) c.levels = 2;
        if (c.levels != 2) return GQ_ERR_INVALID;
        break;
    case GQ_TERNGRAD_LAYER:
        if (c.levels == 0) c.levels = 3;
        if (c.levels != 3) return GQ_ERR_INVALID;
        break;
    default: return GQ_ERR_INVALID;
    }
    if (c.bucket < GQ_MIN_BUCKET || c.bucket > GQ_MAX_BUCKET || (c.bucket & (c.bucket - 1)) != 0) return GQ_ERR_INVALID;
    if (c.workers < 1 || c.workers > GQ_MAX_WORKERS) return GQ_ERR_INVALID;
    if (c.error_feedback != 0 && c.error_feedback != 1) return GQ_ERR_INVALID;
    if (!(c.clip_sigma >= 0.0f) || !std::isfinite(c.clip_sigma)) return GQ_ERR_INVALID;
    if (c.n < 0 || c.n >= (int64_t(1) << 40)) return GQ_ERR_INVALID;
    // the biased baselines are built for the register path only
    if ((c.scheme == GQ_QSGD_NEAREST || c.scheme == GQ_SIGNSGD || c.scheme == GQ_QSGD_L2) && c.bucket > 512)
        return GQ_ERR_UNSUPPORTED;
    if (c.scheme == GQ_TERNGRAD_LAYER && c.clip_sigma > 0.0f) return GQ_ERR_UNSUPPORTED;
    *out = c;
    return GQ_OK;
}

void layout(const gq_config_t &c, size_t *bytes, size_t *codes_off, size_t *levels_off)
{
    const int64_t nb = (c.n + c.bucket - 1) / c.bucket;
    int64_t cbytes = nb * (int64_t)c.bucket * bits_for(c.levels) / 8;
    int64_t lbytes = nb * table_len(c.scheme, c.levels) * 4;
    cbytes = (cbytes + 15) / 16 * 16;
    lbytes = (lbytes + 15) / 16 * 16;
    if (bytes) *bytes = (size_t)(cbytes + lbytes);
    if (codes_off) *codes_off = 0;
    if (levels_off) *levels_off = (size_t)cbytes;
}

gq::KParams base_params(const gq_plan &pl, uint64_t step)
{
    gq::KParams p;
    std::memset(&p, 0, sizeof p);
    p.scheme = pl.cfg.scheme;
    p.s = pl.cfg.levels;
    p.bits = pl.bits;
    p.L = pl.L;
    p.d = pl.cfg.bucket;
    p.W = 1;
    p.n = pl.cfg.n;
    p.nb = pl.nb;
    p.tail = pl.tail;
    p.clip = pl.cfg.clip_sigma;
    p.key0 = (uint32_t)pl.cfg.seed;
    p.key1 = (uint32_t)(pl.cfg.seed >> 32);
    for (int i = 0; i < 10; ++i) {
        p.rk0[i] = p.key0 + (uint32_t)i * 0x9E3779B9u;
        p.rk1[i] = p.key1 + (uint32_t)i * 0xBB67AE85u;
    }
    p.step_lo = (uint32_t)step;
    p.step_m1 = 0xCD9E8D57ull * (unsigned long long)p.step_lo;
    p.worker0 = 0;
    p.inv_w = 1.0f;
    for (int k = 0; k < pl.cfg.levels; ++k)
        p.qratio[k] = (float)(2 * k - (pl.cfg.levels - 1)) / (float)(pl.cfg.levels - 1);
    p.codes_words = pl.fmt_s ? pl.base_words : (int64_t)pl.cfg.bucket * pl.bits / 32;
    p.fmt_s = pl.fmt_s;
    p.levels_off = (int64_t)pl.levels_off;
    p.status = pl.status;
    p.seg_off = pl.seg_off;
    p.nseg = pl.nseg;
    p.seg_max = pl.seg_max;
    return p;
}

gq_status_t check_device(const gq_plan &pl)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return GQ_ERR_CUDA;
    return dev == pl.device ? GQ_OK : GQ_ERR_INVALID;
}

gq_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? GQ_OK : GQ_ERR_CUDA; }

// NVTX range around an entry point (free when no profiler is attached): shows the call on the
// host timeline next to the kernels it enqueues.
struct Range {
    explicit Range(const char *name) { nvtxRangePushA(name); }
    ~Range() { nvtxRangePop(); }
};

}  // namespace

extern "C" {

gq_status_t gq_config_check(const gq_config_t *cfg)
{
    gq_config_t c;
    return normalise(cfg, &c);
}

gq_status_t gq_message_layout(const gq_config_t *cfg, size_t *bytes, size_t *codes_off, size_t *levels_off)
{
    gq_config_t c;
    const gq_status_t st = normalise(cfg, &c);
    if (st != GQ_OK) return st;
    if (c.scheme == GQ_TERNGRAD_LAYER) return GQ_ERR_UNSUPPORTED;  // sized by the tensors: gq_plan_message_layout
    layout(c, bytes, codes_off, levels_off);
    return GQ_OK;
}

gq_status_t gq_plan_create(const gq_config_t *cfg, gq_plan_t *out)
{
    if (!out) return GQ_ERR_INVALID;
    *out = nullptr;
    gq_config_t c;
    const gq_status_t st = normalise(cfg, &c);
    if (st != GQ_OK) return st;
    gq_plan *pl = new (std::nothrow) gq_plan;
    if (!pl) return GQ_ERR_NOMEM;
    pl->cfg = c;
    pl->bits = bits_for(c.levels);
    pl->L = table_len(c.scheme, c.levels);
    pl->nb = (c.n + c.bucket - 1) / c.bucket;
    pl->tail = c.n > 0 ? (int)(c.n - (pl->nb - 1) * c.bucket) : 0;
    layout(c, &pl->msg_bytes, &pl->codes_off, &pl->levels_off);
    pl->status = nullptr;
    pl->err_scratch = nullptr;
    pl->seg_off = nullptr;
    pl->nseg = 0;
    pl->seg_max = nullptr;
    pl->fmt_s = 0;
    pl->base_words = 0;
    if (c.scheme == GQ_TERNGRAD_LAYER) pl->msg_bytes = pl->codes_off = pl->levels_off = 0;  // until the segments
    const size_t err_bytes = (size_t)gq::err_scratch_doubles(pl->nb) * sizeof(double);
    if (cudaGetDevice(&pl->device) != cudaSuccess || cudaMalloc(&pl->status, sizeof(unsigned int)) != cudaSuccess ||
        cudaMemset(pl->status, 0, sizeof(unsigned int)) != cudaSuccess ||
        (err_bytes && cudaMalloc(&pl->err_scratch, err_bytes) != cudaSuccess)) {
        if (pl->status) cudaFree(pl->status);
        if (pl->err_scratch) cudaFree(pl->err_scratch);
        delete pl;
        return GQ_ERR_CUDA;
    }
    *out = pl;
    return GQ_OK;
}

gq_status_t gq_plan_destroy(gq_plan_t plan)
{
    if (!plan) return GQ_ERR_INVALID;
    cudaError_t e = cudaFree(plan->status);
    if (plan->err_scratch) {
        const cudaError_t e2 = cudaFree(plan->err_scratch);
        if (e == cudaSuccess) e = e2;
    }
    if (plan->seg_off) {
        const cudaError_t e2 = cudaFree(plan->seg_off);
        if (e == cudaSuccess) e = e2;
    }
    if (plan->seg_max) {
        const cudaError_t e2 = cudaFree(plan->seg_max);
        if (e == cudaSuccess) e = e2;
    }
    delete plan;
    return from_cuda(e);
}

// Buckets above 512: the group kernels take ORQ and QSGD / TernGrad without clipping; everything
// else goes to the CTA kernel.
static cudaError_t launch_large(const gq::KParams &p, bool fused, cudaStream_t s)
{
    const bool group = p.clip == 0.0f && (p.scheme == GQ_ORQ || p.scheme == GQ_QSGD || p.scheme == GQ_TERNGRAD);
    if (!group) return gq::launch_cta_encode(p, s);
    return p.scheme == GQ_ORQ ? gq::launch_group_orq(p, fused, s) : gq::launch_group_qsgd(p, fused, s);
}

gq_status_t gq_encode(gq_plan_t plan, uint32_t worker, uint64_t step, const float *grad, float *residual, void *msg,
                      void *stream)
{
    Range range("gq_encode");
    if (!plan) return GQ_ERR_INVALID;
    if (plan->cfg.n == 0) return GQ_OK;  // nothing to read or write: pointers may be NULL
    if (!grad || !msg || !aligned16(grad) || !aligned16(msg)) return GQ_ERR_INVALID;
    if ((plan->cfg.error_feedback != 0) != (residual != nullptr)) return GQ_ERR_INVALID;
    if (residual && !aligned16(residual)) return GQ_ERR_INVALID;
    if (plan->cfg.scheme == GQ_TERNGRAD_LAYER && !plan->seg_off) return GQ_ERR_INVALID;
    gq_status_t st = check_device(*plan);
    if (st != GQ_OK) return st;
    gq::KParams p = base_params(*plan, step);
    p.worker0 = worker;
    p.g[0] = grad;
    p.r[0] = residual;
    p.msg[0] = static_cast<unsigned char *>(msg);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (plan->cfg.scheme == GQ_TERNGRAD_LAYER) return from_cuda(gq::launch_layer_encode(p, s));
    if (plan->cfg.bucket <= 512) return from_cuda(gq::launch_warp_encode(p, false, s));
    return from_cuda(launch_large(p, false, s));
}

gq_status_t gq_decode_accumulate(gq_plan_t plan, const void *const *msgs, int nmsgs, float *avg, void *stream)
{
    Range range("gq_decode_accumulate");
    if (!plan || nmsgs < 1 || nmsgs > GQ_MAX_WORKERS) return GQ_ERR_INVALID;
    if (plan->cfg.n == 0) return GQ_OK;  // nothing to read or write: pointers may be NULL
    if (!msgs || !avg || !aligned16(avg)) return GQ_ERR_INVALID;
    for (int w = 0; w < nmsgs; ++w)
        if (!msgs[w] || !aligned16(msgs[w])) return GQ_ERR_INVALID;
    if (plan->cfg.scheme == GQ_TERNGRAD_LAYER && !plan->seg_off) return GQ_ERR_INVALID;
    gq_status_t st = check_device(*plan);
    if (st != GQ_OK) return st;
    gq::KParams p = base_params(*plan, 0);
    p.W = nmsgs;
    p.inv_w = 1.0f / (float)nmsgs;
    for (int w = 0; w < nmsgs; ++w) p.msg[w] = static_cast<unsigned char *>(const_cast<void *>(msgs[w]));
    p.avg = avg;
    if (plan->cfg.scheme == GQ_TERNGRAD_LAYER) return from_cuda(gq::launch_layer_decode(p, static_cast<cudaStream_t>(stream)));
    return from_cuda(gq::launch_decode(p, static_cast<cudaStream_t>(stream)));
}

gq_status_t gq_fused_step(gq_plan_t plan, uint64_t step, const float *const *grads, float *const *residuals,
                          void *const *msgs, float *avg, void *stream)
{
    Range range("gq_fused_step");
    if (!plan) return GQ_ERR_INVALID;
    if (plan->cfg.n == 0) return GQ_OK;  // nothing to read or write: pointers may be NULL
    if (!grads || !avg || !aligned16(avg)) return GQ_ERR_INVALID;
    const int W = plan->cfg.workers;
    const bool ef = plan->cfg.error_feedback != 0;
    if (ef != (residuals != nullptr)) return GQ_ERR_INVALID;
    for (int w = 0; w < W; ++w) {
        if (!grads[w] || !aligned16(grads[w])) return GQ_ERR_INVALID;
        if (ef && (!residuals[w] || !aligned16(residuals[w]))) return GQ_ERR_INVALID;
        if (msgs && (!msgs[w] || !aligned16(msgs[w]))) return GQ_ERR_INVALID;
    }
    if (plan->cfg.scheme == GQ_TERNGRAD_LAYER && !plan->seg_off) return GQ_ERR_INVALID;
    gq_status_t st = check_device(*plan);
    if (st != GQ_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    gq::KParams p = base_params(*plan, step);
    p.W = W;
    p.inv_w = 1.0f / (float)W;
    for (int w = 0; w < W; ++w) {
        p.g[w] = grads[w];
        p.r[w] = ef ? residuals[w] : nullptr;
        p.msg[w] = msgs ? static_cast<unsigned char *>(msgs[w]) : nullptr;
    }
    p.avg = avg;
    if (plan->cfg.scheme == GQ_TERNGRAD_LAYER) return from_cuda(gq::launch_layer_encode(p, s));
    if (plan->cfg.bucket <= 512) return from_cuda(gq::launch_warp_encode(p, true, s));
    return from_cuda(launch_large(p, true, s));
}

gq_status_t gq_quant_error(gq_plan_t plan, uint32_t worker, uint64_t step, const float *grad, const float *residual,
                           double *out, void *stream)
{
    Range range("gq_quant_error");
    if (!plan || !out) return GQ_ERR_INVALID;
    if (plan->cfg.scheme == GQ_TERNGRAD_LAYER) return GQ_ERR_UNSUPPORTED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (plan->cfg.n == 0) return from_cuda(cudaMemsetAsync(out, 0, 3 * sizeof(double), s));
    if (!grad || !aligned16(grad)) return GQ_ERR_INVALID;
    if ((plan->cfg.error_feedback != 0) != (residual != nullptr)) return GQ_ERR_INVALID;
    if (residual && !aligned16(residual)) return GQ_ERR_INVALID;
    gq_status_t st = check_device(*plan);
    if (st != GQ_OK) return st;
    gq::KParams p = base_params(*plan, step);
    p.worker0 = worker;
    p.g[0] = grad;
    p.r[0] = const_cast<float *>(residual);  // read only in this mode
    double *part = plan->err_scratch;
    cudaError_t e = plan->cfg.bucket <= 512 ? gq::launch_warp_err(p, part, s) : gq::launch_cta_err(p, part, s);
    if (e != cudaSuccess) return GQ_ERR_CUDA;
    return from_cuda(gq::launch_err_reduce(part, plan->nb, part + 3 * plan->nb, out, s));
}

gq_status_t gq_plan_set_segments(gq_plan_t plan, const int64_t *offsets, int nseg)
{
    if (!plan || !offsets || nseg < 1 || plan->cfg.scheme != GQ_TERNGRAD_LAYER) return GQ_ERR_INVALID;
    if (offsets[0] != 0 || offsets[nseg] != plan->cfg.n) return GQ_ERR_INVALID;
    for (int t = 0; t < nseg; ++t)
        if (offsets[t + 1] < offsets[t]) return GQ_ERR_INVALID;
    const gq_status_t st = check_device(*plan);
    if (st != GQ_OK) return st;
    if (plan->seg_off) cudaFree(plan->seg_off);
    if (plan->seg_max) cudaFree(plan->seg_max);
    plan->seg_off = nullptr;
    plan->seg_max = nullptr;
    plan->nseg = 0;
    if (cudaMalloc(&plan->seg_off, sizeof(int64_t) * (size_t)(nseg + 1)) != cudaSuccess ||
        cudaMalloc(&plan->seg_max, sizeof(unsigned int) * (size_t)nseg * plan->cfg.workers) != cudaSuccess ||
        cudaMemcpy(plan->seg_off, offsets, sizeof(int64_t) * (size_t)(nseg + 1), cudaMemcpyHostToDevice) != cudaSuccess) {
        if (plan->seg_off) cudaFree(plan->seg_off);
        if (plan->seg_max) cudaFree(plan->seg_max);
        plan->seg_off = nullptr;
        plan->seg_max = nullptr;
        return GQ_ERR_CUDA;
    }
    plan->nseg = nseg;
    const int64_t cbytes = (plan->nb * (int64_t)plan->cfg.bucket * 2 / 8 + 15) / 16 * 16;
    const int64_t sbytes = ((int64_t)nseg * 4 + 15) / 16 * 16;
    plan->codes_off = 0;
    plan->levels_off = (size_t)cbytes;
    plan->msg_bytes = (size_t)(cbytes + sbytes);
    return GQ_OK;
}

gq_status_t gq_plan_set_format(gq_plan_t plan, int format)
{
    if (!plan) return GQ_ERR_INVALID;
    if (plan->cfg.scheme == GQ_TERNGRAD_LAYER)  // its message is dense and sized by the tensors
        return format == GQ_FORMAT_DENSE ? GQ_OK : (format == GQ_FORMAT_BASE_S ? GQ_ERR_UNSUPPORTED : GQ_ERR_INVALID);
    if (format == GQ_FORMAT_DENSE) {
        plan->fmt_s = 0;
        plan->base_words = 0;
        layout(plan->cfg, &plan->msg_bytes, &plan->codes_off, &plan->levels_off);
        return GQ_OK;
    }
    if (format != GQ_FORMAT_BASE_S) return GQ_ERR_INVALID;
    const gq_config_t &c = plan->cfg;
    const bool family = c.scheme == GQ_ORQ || c.scheme == GQ_QSGD || c.scheme == GQ_TERNGRAD ||
                        c.scheme == GQ_QSGD_NEAREST || c.scheme == GQ_QSGD_L2;
    if (!family || c.bucket > 512 || (c.levels != 3 && c.levels != 5 && c.levels != 9)) return GQ_ERR_UNSUPPORTED;
    size_t bytes = 0, coff = 0, loff = 0;
    const gq_status_t st = gq_entropy_layout(&c, &bytes, &coff, &loff);
    if (st != GQ_OK) return st;
    const int g = c.levels == 5 ? 3 : 5, B = c.levels == 3 ? 8 : c.levels == 5 ? 7 : 16;
    plan->fmt_s = c.levels;
    plan->base_words = (((int64_t)c.bucket + g - 1) / g * B + 31) / 32;
    plan->msg_bytes = bytes;
    plan->codes_off = coff;
    plan->levels_off = loff;
    return GQ_OK;
}

gq_status_t gq_plan_message_layout(gq_plan_t plan, size_t *bytes, size_t *codes_off, size_t *levels_off)
{
    if (!plan) return GQ_ERR_INVALID;
    if (plan->cfg.scheme == GQ_TERNGRAD_LAYER && !plan->seg_off) return GQ_ERR_INVALID;
    if (bytes) *bytes = plan->msg_bytes;
    if (codes_off) *codes_off = plan->codes_off;
    if (levels_off) *levels_off = plan->levels_off;
    return GQ_OK;
}

gq_status_t gq_selftest_bounded_wait(gq_plan_t plan, int64_t limit_ns, void *stream)
{
    if (!plan) return GQ_ERR_INVALID;
    const gq_status_t st = check_device(*plan);
    if (st != GQ_OK) return st;
    const int64_t lim = limit_ns < 1000000 ? 1000000 : (limit_ns > 1000000000 ? 1000000000 : limit_ns);
    return from_cuda(gq::launch_wait_selftest(plan->status, (unsigned long long)lim, static_cast<cudaStream_t>(stream)));
}

gq_status_t gq_plan_status(gq_plan_t plan, void *stream)
{
    if (!plan) return GQ_ERR_INVALID;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    unsigned int flags = 0;
    if (cudaMemcpyAsync(&flags, plan->status, sizeof flags, cudaMemcpyDeviceToHost, s) != cudaSuccess) return GQ_ERR_CUDA;
    if (cudaMemsetAsync(plan->status, 0, sizeof(unsigned int), s) != cudaSuccess) return GQ_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return GQ_ERR_CUDA;
    if (flags & gq::kStatusTimeout) return GQ_ERR_TIMEOUT;
    if (flags & gq::kStatusNonFinite) return GQ_ERR_NONFINITE;
    return GQ_OK;
}

const char *gq_status_string(gq_status_t status)
{
    switch (status) {
    case GQ_OK: return "ok";
    case GQ_ERR_INVALID: return "invalid argument";
    case GQ_ERR_UNSUPPORTED: return "unsupported configuration";
    case GQ_ERR_CUDA: return "CUDA error";
    case GQ_ERR_NONFINITE: return "non-finite input value";
    case GQ_ERR_NOMEM: return "out of host memory";
    case GQ_ERR_TIMEOUT: return "a bounded wait for a bulk copy timed out";
    }
    return "unknown status";
}

const char *gq_version(void) { return "0.1.0"; }

}  // extern "C"
