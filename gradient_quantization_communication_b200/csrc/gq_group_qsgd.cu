// gq_group_orq.cu -- instantiation of the group kernels for GQ_QSGD and GQ_TERNGRAD.
#include "gq_group.cuh"

namespace gq {

cudaError_t launch_group_qsgd(const KParams &p, bool fused, cudaStream_t stream)
{
    return fused ? launch_group_fused<GQ_QSGD, true>(p, stream) : launch_group_fused<GQ_QSGD, false>(p, stream);
}

}  // namespace gq
