// Internal interface between the C ABI (etp_api.cu) and the kernel translation units.
#pragma once

#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

namespace etp {

constexpr int kThreadsPerBlock = 64;  // 2 warps; forward and backward kernels

struct FwdArgs {
    int N, E;
    const int32_t* row_ptr;  // over row ranks when `order` is given
    const int32_t* src;
    const float* r;
    const float* frames;  // may be null: frames built in the kernel
    const float4* x;
    const float4* w;
    float4* out;
    int C4;      // C / 4
    int team;    // lanes per team = min(32, C/2), a power of two
    int slices;  // teams per task = C / (2 team): 1, or 2 when C = 128
    int ntasks;  // equal contiguous ranges of positions
    const int32_t* order;     // may be null: row rank -> destination node (locality order)
    const int32_t* pos_edge;  // may be null: position -> edge (the ranks' rows in sequence)
    float4* part;             // partial rows [ntasks][2][D][C] of rows cut by task boundaries
};

struct BwdArgs {
    int N, E;
    const int32_t* row_ptr;
    const int32_t* src;
    const int32_t* rev_ptr;
    const int32_t* rev_perm;
    const int32_t* dst;  // may be null
    const float* r;
    const float* frames;  // may be null: frames built in the kernel
    const float4* x;
    const float4* w;
    const float4* g;
    float4* grad_x;  // may be null
    float4* grad_w;  // may be null
    float* grad_r;   // may be null
    int C4;
    int team;
    int slices;
    int ntasks;
    const int32_t* order;  // may be null: source row rank -> node (rev_ptr is then over ranks)
    float4* part;          // partial rows [ntasks][2][D][C] of grad_x rows cut by task boundaries
};

// Launch geometry shared by the forward and backward kernels: teams of
// min(32, C/2) lanes, each lane two channels; C/(2 team) teams per task (a
// contiguous range of edges); as many tasks as fill the GPU once.
struct LaunchShape {
    int team, slices, tasks_per_block, ntasks;
    size_t smem_bytes;
    dim3 grid;
};
LaunchShape launch_shape(int C, int L, bool o3, bool backward, bool framed, int E, int N, int waves = 1);

template <int L>
size_t smem_bytes(bool o3, int C, int T, bool backward, bool framed);
template <int L>
int read_and_clear_fault();
template <int L>
int blocks_per_sm(bool o3, bool backward, bool framed, int C, size_t smem);

template <int L>
cudaError_t launch_forward(bool o3, const FwdArgs& a, dim3 grid, size_t smem, cudaStream_t s);
template <int L>
cudaError_t launch_backward(bool o3, const BwdArgs& a, dim3 grid, size_t smem, cudaStream_t s);
template <int L>
cudaError_t launch_edge_frames(int E, const float* r, float* frames, cudaStream_t s);
// The second pass of the segment sums (rows cut by task boundaries, rows without
// positions) over rows of row4 float4s; ptr: the CSR pointer the tasks ran over.
cudaError_t launch_combine_rows(const int32_t* ptr, const int32_t* order, int N, int E, int ntasks, int row4,
                                const float4* part, float4* rows, cudaStream_t s);
// Bytes of the partial-row buffer of one launch shape: two rows of D x C floats
// per task, then one int per task, the task's last row when that row is cut at
// the task's end and begins in it (the task that starts its combine), else -1.
inline size_t partial_rows_bytes(int ntasks, int D, int C) {
    return 2 * (size_t)ntasks * D * C * sizeof(float) + (size_t)ntasks * sizeof(int32_t);
}

// Reverse CSR workspace. Up to kOnePassMaxNodes sources (and a bounded table)
// the grouping is one stable counting pass over a (source, tile) count table;
// otherwise a radix sort of the source ids, 8 bits per pass, whose workspace is
// per-source counts, two key buffers, one value buffer and the table of per-tile
// digit histograms (tiles of kRadixTile edges) with a row of digit totals.
constexpr int kRadixTile = 1024;
constexpr int kOnePassMaxNodes = 8192;
constexpr long long kOnePassMaxEntries = 1ll << 22;
constexpr int kScanChunk = 8192;  // table entries scanned per block
constexpr size_t align16_bytes(size_t b) { return (b + 15) & ~size_t(15); }
constexpr long long radix_tiles(long long E) { return (E + kRadixTile - 1) / kRadixTile; }
constexpr bool reverse_csr_one_pass(long long N, long long E) {
    return N >= 1 && N <= kOnePassMaxNodes && E > 0 && (N + 1) * radix_tiles(E) <= kOnePassMaxEntries;
}
constexpr size_t radix_workspace_bytes_for(long long N, long long E) {
    return align16_bytes(4 * (size_t)(N + 1)) + 3 * align16_bytes(4 * (size_t)E) +
           align16_bytes(4 * (256 * ((size_t)radix_tiles(E) + 1) + 1));
}
constexpr size_t one_pass_workspace_bytes_for(long long N, long long E) {
    return align16_bytes(4 * (size_t)((N + 1) * radix_tiles(E))) +
           align16_bytes(4 * (size_t)((N + 1) * radix_tiles(E) / kScanChunk + 2));
}
constexpr size_t reverse_csr_workspace_bytes_for(long long N, long long E) {
    return reverse_csr_one_pass(N, E) ? one_pass_workspace_bytes_for(N, E) : radix_workspace_bytes_for(N, E);
}
size_t reverse_csr_workspace_bytes(int N, int E);
// one_pass: allow the one-pass grouping when it applies (the workspace must then
// hold reverse_csr_workspace_bytes_for); false: always the radix sort (workspace
// radix_workspace_bytes_for).
cudaError_t build_reverse_csr(int N, int E, const int32_t* row_ptr, const int32_t* src, int32_t* rev_ptr,
                              int32_t* rev_perm, int32_t* dst, void* ws, cudaStream_t s, bool one_pass = true);
// Locality schedule: nodes sorted stably by the Morton code of their cell
// (spatial_order), and the forward and reverse CSRs with rows in a given node
// order (build_ordered_csr; dst = destination of every edge).
size_t spatial_order_workspace_bytes(int N);
cudaError_t spatial_order(int N, const float* pos, float cell, int32_t* order, void* ws, cudaStream_t s);
size_t ordered_csr_workspace_bytes(int N, int E);
cudaError_t build_ordered_csr(int N, int E, const int32_t* row_ptr, const int32_t* src, const int32_t* order,
                              int32_t* ord_ptr, int32_t* ord_edge, int32_t* rev_ptr, int32_t* rev_perm, int32_t* dst,
                              void* ws, cudaStream_t s);
size_t radial_workspace_bytes(int E, int nb, int hidden, int PC);
// Tensor-core path of the radial forward (hidden width 64, P*C a multiple of 16).
bool radial_tc_supported(int nb, int hidden, int PC);
size_t radial_tc_prepare_bytes(int PC);
cudaError_t radial_tc_forward(int E, int nb, int PC, float rc, const float* r, const float* W1, const float* W2,
                              float* w, void* ws, cudaStream_t s);
size_t radial_tc_backward_prepare_bytes(int PC);
cudaError_t radial_tc_backward(int E, int PC, float rc, const float* r, const float* W1, const float* W2,
                               const float* grad_w, float* gZ, float* grad_r, void* prep, cudaStream_t s);
// grad_W2 partial sums over `splits` edge splits on the tensor cores: part [splits][64][PC].
int radial_tc_grad_w2_splits(int E, int PC);
cudaError_t radial_tc_grad_w2(int E, int PC, const float* grad_w, const float* H, float* part, int splits,
                              cudaStream_t s);
int radial_tc_read_and_clear_fault();
cudaError_t radial_forward(int E, int nb, int hidden, int PC, float rc, const float* r, const float* W1,
                           const float* W2, float* w, void* ws, cudaStream_t s);
cudaError_t radial_backward(int E, int nb, int hidden, int PC, float rc, const float* r, const float* W1,
                            const float* W2, const float* grad_w, float* grad_W1, float* grad_W2, float* grad_r,
                            void* ws, cudaStream_t s);
// Radial weights fused into the tensor product (etp_fused.cu): n_basis 8, hidden 64.
bool fused_supported(int nb, int hidden);
size_t fused_workspace_bytes(int L, bool o3, int C, int E);
size_t fused_smem_bytes(int L, bool o3, int C);
cudaError_t fused_forward(int L, bool o3, int C, int N, int E, const int32_t* row_ptr, const int32_t* src,
                          const float* r, const float* x, const float* W1, const float* W2, float rc, float* out,
                          void* ws, cudaStream_t s);
int fused_read_and_clear_fault();
// VJP of the VJP (etp_double.cu).
cudaError_t double_backward(int L, bool o3, int C, int N, int E, const int32_t* row_ptr, const int32_t* src,
                            const int32_t* rev_ptr, const int32_t* rev_perm, const int32_t* dst, const float* r,
                            const float* x, const float* w, const float* g, const float* gg_x, const float* gg_w,
                            const float* gg_r, float* grad_g, float* grad_x, float* grad_w, float* grad_r,
                            void* part, size_t part_bytes, cudaStream_t s);
size_t double_backward_partial_bytes(int L, bool o3, int C, int N, int E);
// Cartesian edge convolution (etp_cart.cu): features in independent STF components.
cudaError_t cart_forward(int L, bool o3, int C, int N, int E, const int32_t* row_ptr, const int32_t* src,
                         const float* r, const float* x, const float* w, float* out, void* part, size_t part_bytes,
                         cudaStream_t s);
cudaError_t cart_backward(int L, bool o3, int C, int N, int E, const int32_t* row_ptr, const int32_t* rev_ptr,
                          const int32_t* rev_perm, const int32_t* dst, const float* r, const float* x, const float* w,
                          const float* g, float* grad_x, float* grad_w, float* grad_r, void* part, size_t part_bytes,
                          cudaStream_t s);
size_t cart_partial_bytes(int L, bool o3, int C, int N, int E);

// node-local product (etp_nodeprod.cu): out = B(K), w [K-1][P][C]; cart selects the
// Cartesian couplings
cudaError_t node_product(int L, bool o3, bool cart, int C, int N, int K, const float* x, const float* w, float* out,
                         cudaStream_t s);
// FP32 operations per node, channel and step of that kernel's arithmetic
int node_product_ops(int L, bool o3, bool cart);
cudaError_t assemble_forces(int N, int E, const int32_t* row_ptr, const int32_t* rev_ptr, const int32_t* rev_perm,
                            const float* r, const float* grad_r, float* forces, float* virial, cudaStream_t s);
cudaError_t validate_csr(int N, int E, const int32_t* row_ptr, const int32_t* src, int32_t* flag, cudaStream_t s);

}  // namespace etp
