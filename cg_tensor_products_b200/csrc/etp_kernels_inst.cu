// One translation unit per L (compiled with -DETP_L=<L>), so the specialisations
// build in parallel.
#include "etp_frame.cuh"

#ifndef ETP_L
#error "compile with -DETP_L=<0..3>"
#endif

namespace etp {
template cudaError_t launch_forward<ETP_L>(bool, const FwdArgs&, dim3, size_t, cudaStream_t);
template cudaError_t launch_backward<ETP_L>(bool, const BwdArgs&, dim3, size_t, cudaStream_t);
template size_t smem_bytes<ETP_L>(bool, int, int, bool, bool);
template cudaError_t launch_edge_frames<ETP_L>(int, const float*, float*, cudaStream_t);

// The fault flag of this specialisation's kernels.
template <>
int read_and_clear_fault<ETP_L>() {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, frame::g_fault, sizeof(int)) != cudaSuccess) return -1;
    const int zero = 0;
    cudaMemcpyToSymbol(frame::g_fault, &zero, sizeof(int));
    return v;
}
template int blocks_per_sm<ETP_L>(bool, bool, bool, int, size_t);
}  // namespace etp
