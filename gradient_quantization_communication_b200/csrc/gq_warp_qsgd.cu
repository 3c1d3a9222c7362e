// gq_warp_qsgd.cu -- instantiation of the register-path kernels for GQ_QSGD.
#include "gq_warp.cuh"

namespace gq {

cudaError_t launch_warp_qsgd(const KParams &p, bool fused, cudaStream_t stream)
{
    return warp_dispatch<GQ_QSGD>(p, fused, stream);
}

cudaError_t launch_warp_err_qsgd(const KParams &p, double *part, cudaStream_t stream)
{
    return warp_dispatch_err<GQ_QSGD>(p, part, stream);
}

}  // namespace gq
