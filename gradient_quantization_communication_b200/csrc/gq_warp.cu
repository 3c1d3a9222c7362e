// gq_warp.cu -- entry of the register path (d = 128, 256, 512): picks the per-scheme launcher.
#include "gq_internal.h"

namespace gq {

cudaError_t launch_warp_orq(const KParams &p, bool fused, cudaStream_t stream);
cudaError_t launch_warp_qsgd(const KParams &p, bool fused, cudaStream_t stream);
cudaError_t launch_warp_bingrad(const KParams &p, bool fused, cudaStream_t stream);
cudaError_t launch_warp_err_orq(const KParams &p, double *part, cudaStream_t stream);
cudaError_t launch_warp_err_qsgd(const KParams &p, double *part, cudaStream_t stream);
cudaError_t launch_warp_err_bingrad(const KParams &p, double *part, cudaStream_t stream);
cudaError_t launch_warp_extra(const KParams &p, bool fused, cudaStream_t stream);
cudaError_t launch_warp_err_extra(const KParams &p, double *part, cudaStream_t stream);

cudaError_t launch_warp_encode(const KParams &p, bool fused, cudaStream_t stream)
{
    switch (p.scheme) {
    case GQ_QSGD:
    case GQ_TERNGRAD: return launch_warp_qsgd(p, fused, stream);
    case GQ_BINGRAD_B:
    case GQ_BINGRAD_PB: return launch_warp_bingrad(p, fused, stream);
    case GQ_QSGD_NEAREST:
    case GQ_SIGNSGD:
    case GQ_QSGD_L2: return launch_warp_extra(p, fused, stream);
    default: return launch_warp_orq(p, fused, stream);
    }
}

cudaError_t launch_warp_err(const KParams &p, double *part, cudaStream_t stream)
{
    switch (p.scheme) {
    case GQ_QSGD:
    case GQ_TERNGRAD: return launch_warp_err_qsgd(p, part, stream);
    case GQ_BINGRAD_B:
    case GQ_BINGRAD_PB: return launch_warp_err_bingrad(p, part, stream);
    case GQ_QSGD_NEAREST:
    case GQ_SIGNSGD:
    case GQ_QSGD_L2: return launch_warp_err_extra(p, part, stream);
    default: return launch_warp_err_orq(p, part, stream);
    }
}

}  // namespace gq
