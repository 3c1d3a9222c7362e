// gq_group_orq.cu -- instantiation of the group kernels for GQ_ORQ.
#include "gq_group.cuh"

namespace gq {

cudaError_t launch_group_orq(const KParams &p, bool fused, cudaStream_t stream)
{
    return fused ? launch_group_fused<GQ_ORQ, true>(p, stream) : launch_group_fused<GQ_ORQ, false>(p, stream);
}

}  // namespace gq
