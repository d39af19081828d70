// etp_build_reverse_csr_static: the reverse-CSR build without a caller-supplied
// workspace and without any device allocation.
//
// Some callers cannot allocate device memory at the point where they need the
// reverse CSR: a plugin living inside a host program that owns the whole GPU
// memory budget (an MD engine that hands its force field fixed buffers and
// nothing else), or a time-critical loop where a cudaMalloc - which may
// synchronise the device - is not acceptable. For them this entry point takes
// its scratch from one file-scope __device__ array of fixed size instead of a
// workspace argument. Everything else (inputs, outputs, stream) is still the
// caller's.
//
// The array is part of the library image: every GPU on which the library's
// kernels are loaded holds ETP_STATIC_SCRATCH_BYTES of it until the process
// exits. All calls share it. Its contents persist from call to call; the only
// part that must start at zero (the per-source counters) is cleared by every
// call on the stream, and the rest is fully written before it is read. Two
// calls whose work overlaps on the GPU (different streams, or different host
// threads, with no ordering between them) race on the array and give wrong
// results.
//
// The device address of the array is obtained once per device: the first call
// made with a device current runs cudaGetSymbolAddress for that device (host
// code cannot use the array's name as a device pointer: on the host it names a
// shadow variable). That first call should come before any stream capture
// begins on the device.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "etp.h"
#include "etp_internal.h"

namespace {

constexpr size_t kStaticScratchBytes =
    etp::radix_workspace_bytes_for(ETP_STATIC_MAX_NODES, ETP_STATIC_MAX_EDGES);
static_assert(kStaticScratchBytes == ETP_STATIC_SCRATCH_BYTES, "etp.h states the scratch size");

static __device__ __align__(256) unsigned char g_reverse_csr_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set up once per device).
cudaError_t scratch_address(void** out) {
    int dev = -1;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        err = cudaGetSymbolAddress(&p, g_reverse_csr_scratch);
        if (err != cudaSuccess) return err;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" ETP_API etp_status etp_build_reverse_csr_static(int N, int E, const int32_t* row_ptr, const int32_t* src,
                                                           int32_t* rev_ptr, int32_t* rev_perm,
                                                           int32_t* dst_of_edge, etp_stream_t stream) {
    if (N < 0 || E < 0) return ETP_ERR_INVALID_ARG;
    if (N > ETP_STATIC_MAX_NODES || E > ETP_STATIC_MAX_EDGES) return ETP_ERR_TOO_LARGE;
    if (N == 0 && E > 0) return ETP_ERR_INVALID_ARG;
    const uintptr_t mis4 = 3u;
    if (!rev_ptr || (reinterpret_cast<uintptr_t>(rev_ptr) & mis4)) return ETP_ERR_INVALID_ARG;
    if (E > 0 && (!row_ptr || !src || !rev_perm || (reinterpret_cast<uintptr_t>(row_ptr) & mis4) ||
                  (reinterpret_cast<uintptr_t>(src) & mis4) || (reinterpret_cast<uintptr_t>(rev_perm) & mis4)))
        return ETP_ERR_INVALID_ARG;
    if (dst_of_edge && (reinterpret_cast<uintptr_t>(dst_of_edge) & mis4)) return ETP_ERR_INVALID_ARG;
    void* ws = nullptr;
    if (scratch_address(&ws) != cudaSuccess) return ETP_ERR_CUDA;
    // always the radix path: its scratch need grows with N and E, so the array sized
    // for the limits covers every admitted call
    cudaError_t err = etp::build_reverse_csr(N, E, row_ptr, src, rev_ptr, rev_perm, dst_of_edge, ws,
                                             reinterpret_cast<cudaStream_t>(stream), false);
    return err == cudaSuccess ? ETP_OK : ETP_ERR_CUDA;
}
