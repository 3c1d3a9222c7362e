// gq_warp_orq.cu -- instantiation of the register-path kernels for GQ_ORQ.
#include "gq_warp.cuh"

namespace gq {

cudaError_t launch_warp_orq(const KParams &p, bool fused, cudaStream_t stream)
{
    return warp_dispatch<GQ_ORQ>(p, fused, stream);
}

cudaError_t launch_warp_err_orq(const KParams &p, double *part, cudaStream_t stream)
{
    return warp_dispatch_err<GQ_ORQ>(p, part, stream);
}

}  // namespace gq
