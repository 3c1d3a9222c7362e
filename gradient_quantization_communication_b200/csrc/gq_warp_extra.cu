// gq_warp_extra.cu -- instantiation of the register-path kernels for the biased baselines
// (GQ_QSGD_NEAREST, GQ_SIGNSGD) and for QSGD with l2 scaling (GQ_QSGD_L2).
#include "gq_warp.cuh"

namespace gq {

cudaError_t launch_warp_extra(const KParams &p, bool fused, cudaStream_t stream)
{
    switch (p.scheme) {
    case GQ_QSGD_NEAREST: return warp_dispatch<GQ_QSGD_NEAREST>(p, fused, stream);
    case GQ_SIGNSGD: return warp_dispatch<GQ_SIGNSGD>(p, fused, stream);
    default: return warp_dispatch<GQ_QSGD_L2>(p, fused, stream);
    }
}

cudaError_t launch_warp_err_extra(const KParams &p, double *part, cudaStream_t stream)
{
    switch (p.scheme) {
    case GQ_QSGD_NEAREST: return warp_dispatch_err<GQ_QSGD_NEAREST>(p, part, stream);
    case GQ_SIGNSGD: return warp_dispatch_err<GQ_SIGNSGD>(p, part, stream);
    default: return warp_dispatch_err<GQ_QSGD_L2>(p, part, stream);
    }
}

}  // namespace gq
