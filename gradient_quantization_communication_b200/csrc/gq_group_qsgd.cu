// gq_group_orq.cu -- instantiation of the group kernels for GQ_QSGD and GQ_TERNGRAD.
#include "gq_group.cuh"

namespace gq {

cudaError_t launch_group_qsgd(const KParams &p, int64_t nfull, bool fused, cudaStream_t stream)
{
    return fused ? launch_group_fused<GQ_QSGD, true>(p, nfull, stream) : launch_group_fused<GQ_QSGD, false>(p, nfull, stream);
}

}  // namespace gq
