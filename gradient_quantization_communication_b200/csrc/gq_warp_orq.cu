// gq_warp_orq.cu -- instantiation of the register-path kernels for GQ_ORQ.
#include "gq_warp.cuh"

namespace gq {

cudaError_t launch_warp_orq(const KParams &p, bool fused, cudaStream_t stream)
{
    return warp_dispatch<GQ_ORQ>(p, fused, stream);
}

}  // namespace gq
