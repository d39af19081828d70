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

}  // namespace etp
