// One translation unit per L (compiled with -DETP_L=<L>), so the specialisations
// build in parallel.
#include "etp_frame.cuh"

#ifndef ETP_L
#error "compile with -DETP_L=<0..3>"
#endif

namespace etp {
template cudaError_t launch_forward<ETP_L>(bool, const FwdArgs&, dim3, size_t, cudaStream_t);
template cudaError_t launch_backward<ETP_L>(bool, const BwdArgs&, dim3, size_t, cudaStream_t);
}  // namespace etp
