// gq_warp_bin.cu -- instantiation of the register-path kernels for GQ_BINGRAD_B, GQ_BINGRAD_PB.
#include "gq_warp.cuh"

namespace gq {

cudaError_t launch_warp_bingrad(const KParams &p, bool fused, cudaStream_t stream)
{
    return p.scheme == GQ_BINGRAD_B ? warp_dispatch<GQ_BINGRAD_B>(p, fused, stream)
                                    : warp_dispatch<GQ_BINGRAD_PB>(p, fused, stream);
}

cudaError_t launch_warp_err_bingrad(const KParams &p, double *part, cudaStream_t stream)
{
    return p.scheme == GQ_BINGRAD_B ? warp_dispatch_err<GQ_BINGRAD_B>(p, part, stream)
                                    : warp_dispatch_err<GQ_BINGRAD_PB>(p, part, stream);
}

}  // namespace gq
