// Launch geometry of the forward and backward kernels (host side).
#include <atomic>

#include "etp_frame.cuh"

namespace etp {
namespace {

// Resident blocks per SM of each kernel specialisation, per device (computed once).
std::atomic<int> g_occupancy[16][4][2][2][2][8];
std::atomic<int> g_sms[16];

int log2i(int t) {
    int k = 0;
    while ((1 << k) < t) ++k;
    return k;
}

// Second pass of the segment sums, after the forward or backward kernel on the
// same stream. (1) A row cut by task boundaries is stored by the block of the
// task where it begins (found from the task's record after the partial rows):
// the sum, in task order, of that task's slot 1 and the slot 0 of each
// following task up to the one where the row ends. (2) Rows
// without positions are zeroed, one warp per row. Every output row is thus
// written exactly once, in a fixed order: no atomics, bitwise repeatable.
__global__ void __launch_bounds__(256) etp_combine_rows_kernel(const int32_t* __restrict__ ptr,
                                                               const int32_t* __restrict__ order, int N, int E,
                                                               int ntasks, int row4, const float4* __restrict__ part,
                                                               float4* __restrict__ rows) {
    const int32_t* rec = reinterpret_cast<const int32_t*>(part + (size_t)ntasks * 2 * row4);
    for (int t = blockIdx.x; t < ntasks; t += gridDim.x) {
        const int R = rec[t];  // the task's last row if it goes on past the task and begins in it
        if (R < 0) continue;
        const int hi = __ldg(ptr + R + 1);
        const int node = order ? __ldg(order + R) : R;
        for (int f = threadIdx.x; f < row4; f += blockDim.x) {
            float4 acc = part[((size_t)t * 2 + 1) * row4 + f];
            for (int u = t + 1; u < ntasks; ++u) {
                int u0, u1;
                frame::task_range(E, u, ntasks, u0, u1);
                if (u0 >= hi) break;
                if (u0 < u1) {
                    const float4 v = part[(size_t)u * 2 * row4 + f];
                    acc.x += v.x;
                    acc.y += v.y;
                    acc.z += v.z;
                    acc.w += v.w;
                }
                if (u1 >= hi) break;
            }
            rows[(size_t)node * row4 + f] = acc;
        }
    }
    const int lane = threadIdx.x & 31;
    const int warps = gridDim.x * (blockDim.x >> 5);
    for (int j = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); j < N; j += warps) {
        if (__ldg(ptr + j + 1) > __ldg(ptr + j)) continue;
        float4* dst = rows + (size_t)(order ? __ldg(order + j) : j) * row4;
        for (int f = lane; f < row4; f += 32) dst[f] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
}

}  // namespace

LaunchShape launch_shape(int C, int L, bool o3, bool backward, bool framed, int E, int N, int waves) {
    LaunchShape s;
    s.team = C / 2 < 32 ? C / 2 : 32;
    s.slices = C / (2 * s.team);
    s.tasks_per_block = (frame::kThreads / s.team) / s.slices;
    switch (L) {
        case 0: s.smem_bytes = smem_bytes<0>(o3, C, s.team, backward, framed); break;
        case 1: s.smem_bytes = smem_bytes<1>(o3, C, s.team, backward, framed); break;
        case 2: s.smem_bytes = smem_bytes<2>(o3, C, s.team, backward, framed); break;
        default: s.smem_bytes = smem_bytes<3>(o3, C, s.team, backward, framed); break;
    }
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 16) dev = 0;
    int sms = g_sms[dev].load();
    if (sms == 0) {
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1) sms = 1;
        g_sms[dev].store(sms);
    }
    std::atomic<int>& occ = g_occupancy[dev][L & 3][o3 ? 1 : 0][backward ? 1 : 0][framed ? 1 : 0][log2i(C) % 8];
    int bps = occ.load();
    if (bps == 0) {
        switch (L) {
            case 0: bps = blocks_per_sm<0>(o3, backward, framed, C, s.smem_bytes); break;
            case 1: bps = blocks_per_sm<1>(o3, backward, framed, C, s.smem_bytes); break;
            case 2: bps = blocks_per_sm<2>(o3, backward, framed, C, s.smem_bytes); break;
            default: bps = blocks_per_sm<3>(o3, backward, framed, C, s.smem_bytes); break;
        }
        occ.store(bps);
    }
    // `waves` waves of tasks (one, unless a locality schedule asks for more), at
    // least 16 edges each and no more tasks than rows: a row longer than a task
    // is cut more than once, and its pieces are then summed in a run-dependent
    // order (still correct, not bitwise repeatable).
    long long cap = (long long)sms * bps * s.tasks_per_block * (waves < 1 ? 1 : waves);
    long long want = ((long long)E + 15) / 16;
    if (want > N) want = N;
    long long nt = want < cap ? want : cap;
    s.ntasks = (int)(nt < 1 ? 1 : nt);
    s.grid = dim3((unsigned)((s.ntasks + s.tasks_per_block - 1) / s.tasks_per_block), 1, 1);
    return s;
}

cudaError_t launch_combine_rows(const int32_t* ptr, const int32_t* order, int N, int E, int ntasks, int row4,
                                const float4* part, float4* rows, cudaStream_t s) {
    int blocks = ntasks;
    const int row_blocks = (N + 7) / 8;  // eight warps per block, one row each
    if (blocks < row_blocks) blocks = row_blocks < 4 * 148 ? row_blocks : 4 * 148;
    if (blocks < 1) blocks = 1;
    etp_combine_rows_kernel<<<blocks, 256, 0, s>>>(ptr, order, N, E, ntasks, row4, part, rows);
    return cudaGetLastError();
}

}  // namespace etp
