// gq_warp_biased.cu -- instantiation of the register-path kernels for the biased baselines
// GQ_QSGD_NEAREST and GQ_SIGNSGD.
#include "gq_warp.cuh"

namespace gq {

cudaError_t launch_warp_biased(const KParams &p, bool fused, cudaStream_t stream)
{
    return p.scheme == GQ_QSGD_NEAREST ? warp_dispatch<GQ_QSGD_NEAREST>(p, fused, stream)
                                       : warp_dispatch<GQ_SIGNSGD>(p, fused, stream);
}

cudaError_t launch_warp_err_biased(const KParams &p, double *part, cudaStream_t stream)
{
    return p.scheme == GQ_QSGD_NEAREST ? warp_dispatch_err<GQ_QSGD_NEAREST>(p, part, stream)
                                       : warp_dispatch_err<GQ_SIGNSGD>(p, part, stream);
}

}  // namespace gq
