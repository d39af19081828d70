// Forward and backward kernels of the edge tensor product.
//
// Work decomposition (both kernels): a "team" of T = C/4 lanes (a power of two,
// at most 32, so C <= 128) owns one node and all C channels of it; lane t holds
// channels 4t..4t+3 as float4 registers. A warp holds 32/T teams. Nothing is exchanged between
// teams, so the segment sums need no atomics: each team writes its node's
// output exactly once.
//
// Forward (row i of the CSR by destination, edges e in row order):
//   Y = harmonics of r_e (registers), x_j = x[src e] (registers, from L2),
//   per path p: u = sum_nnz (CG * Y_m2) x_j[l1 m1]  (the sparse CG list of p is a
//   compile-time constant, so each coefficient is an immediate),
//   acc[l3 m3] += w[e,p] * u[m3];   out[i] = acc at the end of the row.
// Backward (row j of the reverse CSR, i.e. the edges whose source is j):
//   t_p[m1] = sum_nnz (CG * Y_m2) g[dst e, l3 m3]  (g = grad_out),
//   grad_x acc[l1 m1] += w[e,p] t_p[m1],  grad_w[e,p] = sum_m1 x_j[l1 m1] t_p[m1],
//   dL/dY_{l2 m2} += CG * <w[e,p] x_j[l1 m1], g[l3 m3]> (summed over the team's
//   channels with shuffles), grad_r[e] = sum dL/dY * dY/dr.
// Passages: "High-performance training and inference for deep equivariant
// interatomic potentials", section "제안 방법" (fused kernel, sparse 3-j
// coefficients, no materialised intermediates); "FlashCart 如何让等变原子间势更快
// 更准?", section "FlashCart 用笛卡尔内核替代球谐耦合" (aggregation of edge
// contributions inside the kernel).
#pragma once

#include "etp_device.cuh"
#include "etp_internal.h"

namespace etp {

constexpr int kThreads = kThreadsPerBlock;

// Row of edge e: largest i with row_ptr[i] <= e (rows without edges are skipped).
__device__ __forceinline__ int row_of_edge(const int32_t* __restrict__ row_ptr, int N, int e) {
    int lo = 0, hi = N;  // invariant: row_ptr[lo] <= e < row_ptr[hi]
    while (hi - lo > 1) {
        int mid = (lo + hi) >> 1;
        if (__ldg(row_ptr + mid) <= e)
            lo = mid;
        else
            hi = mid;
    }
    return lo;
}

template <int L, bool O3>
__global__ void __launch_bounds__(kThreads) etp_fwd_kernel(FwdArgs a) {
    using PS = PathSet<L, O3>;
    constexpr int D = PS::D;
    constexpr int P = PS::P;
    const int lane = threadIdx.x & 31;
    const int T = a.team;
    const int tl = lane & (T - 1);
    const int warp = (blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int row = warp * (32 / T) + lane / T;
    if (row >= a.N) return;
    const int cg = tl;  // float4 channel group
    const int C4 = a.C4;
    const uint64_t pol = l2_evict_first_policy();

    int e0 = __ldg(a.row_ptr + row), e1 = __ldg(a.row_ptr + row + 1);
    e0 = max(e0, 0);
    e1 = min(e1, a.E);

    float4 acc[D];
#pragma unroll
    for (int k = 0; k < D; ++k) acc[k] = f4_zero();

    for (int e = e0; e < e1; ++e) {
        const int j = __ldg(a.src + e);
        if ((unsigned)j >= (unsigned)a.N) continue;
        float Y[D];
        sh_eval<L>(__ldg(a.r + 3 * (size_t)e), __ldg(a.r + 3 * (size_t)e + 1), __ldg(a.r + 3 * (size_t)e + 2), Y);
        float4 xv[D];
        const float4* xj = a.x + (size_t)j * D * C4 + cg;
#pragma unroll
        for (int k = 0; k < D; ++k) xv[k] = __ldg(xj + k * C4);
        const float4* we = a.w + (size_t)e * P * C4 + cg;
        static_for<0, P>([&](auto pc) {
            constexpr int p = decltype(pc)::value;
            constexpr Path pt = PS::path(p);
            constexpr int l1 = pt.l1, l2 = pt.l2, l3 = pt.l3;
            constexpr int off = etp_gen::kCgOff[l1][l2][l3];
            constexpr int cnt = etp_gen::kCgCnt[l1][l2][l3];
            const float4 wv = ld_stream(we + p * C4, pol);
            float4 u[2 * l3 + 1];
#pragma unroll
            for (int m = 0; m < 2 * l3 + 1; ++m) u[m] = f4_zero();
            static_for<0, cnt>([&](auto kc) {
                constexpr etp_gen::CgNz z = etp_gen::kCg[off + decltype(kc)::value];
                const float coef = (float)z.v * Y[l2 * l2 + z.m2];
                f4_fma(u[z.m3], coef, xv[l1 * l1 + z.m1]);
            });
#pragma unroll
            for (int m = 0; m < 2 * l3 + 1; ++m) f4_fma(acc[l3 * l3 + m], wv, u[m]);
        });
    }
    float4* o = a.out + (size_t)row * D * C4 + cg;
#pragma unroll
    for (int k = 0; k < D; ++k) o[k * C4] = acc[k];
}

template <int L, bool O3>
__global__ void __launch_bounds__(kThreads) etp_bwd_kernel(BwdArgs a) {
    using PS = PathSet<L, O3>;
    constexpr int D = PS::D;
    constexpr int P = PS::P;
    const int lane = threadIdx.x & 31;
    const int T = a.team;
    const int tl = lane & (T - 1);
    const int warp = (blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int node = warp * (32 / T) + lane / T;
    // Teams past the end keep running (with no edges) so that every lane of the
    // warp takes part in the shuffles below.
    const bool live = node < a.N;
    const int cg = tl;
    const int C4 = a.C4;
    const bool want_r = a.grad_r != nullptr;
    const uint64_t pol = l2_evict_first_policy();

    int q0 = 0, q1 = 0;
    if (live) {
        q0 = max(__ldg(a.rev_ptr + node), 0);
        q1 = min(__ldg(a.rev_ptr + node + 1), a.E);
    }
    // All teams of the warp iterate to the longest team's count; shorter teams idle.
    int nq = max(q1 - q0, 0);
    int nmax = nq;
    for (int s = 16; s >= 1; s >>= 1) nmax = max(nmax, __shfl_xor_sync(0xffffffffu, nmax, s));

    float4 xv[D], gx[D];
    if (live) {
        const float4* xj = a.x + (size_t)node * D * C4 + cg;
#pragma unroll
        for (int k = 0; k < D; ++k) xv[k] = __ldg(xj + k * C4);
    } else {
#pragma unroll
        for (int k = 0; k < D; ++k) xv[k] = f4_zero();
    }
#pragma unroll
    for (int k = 0; k < D; ++k) gx[k] = f4_zero();

    for (int s = 0; s < nmax; ++s) {
        const bool act = s < nq;
        int e = act ? __ldg(a.rev_perm + q0 + s) : 0;
        bool ok = act && (unsigned)e < (unsigned)a.E;
        int i = 0;
        if (ok) {
            i = a.dst ? __ldg(a.dst + e) : row_of_edge(a.row_ptr, a.N, e);
            ok = (unsigned)i < (unsigned)a.N;
        }
        float dLdY[D];
#pragma unroll
        for (int k = 0; k < D; ++k) dLdY[k] = 0.f;
        if (ok) {
            const float rx = __ldg(a.r + 3 * (size_t)e), ry = __ldg(a.r + 3 * (size_t)e + 1),
                        rz = __ldg(a.r + 3 * (size_t)e + 2);
            float Y[D];
            sh_eval<L>(rx, ry, rz, Y);
            float4 gv[D];
            const float4* gi = a.g + (size_t)i * D * C4 + cg;
#pragma unroll
            for (int k = 0; k < D; ++k) gv[k] = __ldg(gi + k * C4);
            const float4* we = a.w + (size_t)e * P * C4 + cg;
            float4* gwe = a.grad_w ? a.grad_w + (size_t)e * P * C4 + cg : nullptr;
            static_for<0, P>([&](auto pc) {
                constexpr int p = decltype(pc)::value;
                constexpr Path pt = PS::path(p);
                constexpr int l1 = pt.l1, l2 = pt.l2, l3 = pt.l3;
                constexpr int off = etp_gen::kCgOff[l1][l2][l3];
                constexpr int cnt = etp_gen::kCgCnt[l1][l2][l3];
                const float4 wv = ld_stream(we + p * C4, pol);
                float4 t[2 * l1 + 1];
                float4 wx[2 * l1 + 1];
#pragma unroll
                for (int m = 0; m < 2 * l1 + 1; ++m) {
                    t[m] = f4_zero();
                    wx[m] = f4_mul(wv, xv[l1 * l1 + m]);
                }
                static_for<0, cnt>([&](auto kc) {
                    constexpr etp_gen::CgNz z = etp_gen::kCg[off + decltype(kc)::value];
                    const float coef = (float)z.v * Y[l2 * l2 + z.m2];
                    f4_fma(t[z.m1], coef, gv[l3 * l3 + z.m3]);
                    dLdY[l2 * l2 + z.m2] = fmaf((float)z.v, f4_dot(wx[z.m1], gv[l3 * l3 + z.m3]),
                                                dLdY[l2 * l2 + z.m2]);
                });
                float4 gw = f4_zero();
#pragma unroll
                for (int m = 0; m < 2 * l1 + 1; ++m) {
                    f4_fma(gx[l1 * l1 + m], wv, t[m]);
                    f4_fma(gw, xv[l1 * l1 + m], t[m]);
                }
                if (gwe) st_stream(gwe + p * C4, gw, pol);
            });
        }
        if (want_r) {
            // sum dL/dY over the team's lanes (all lanes of the warp take part)
#pragma unroll
            for (int k = 0; k < D; ++k) {
                float v = dLdY[k];
                for (int sft = 1; sft < T; sft <<= 1) v += __shfl_xor_sync(0xffffffffu, v, sft);
                dLdY[k] = v;
            }
            if (ok && tl == 0) {
                float Y[D], dY[D][3];
                sh_eval_grad<L>(__ldg(a.r + 3 * (size_t)e), __ldg(a.r + 3 * (size_t)e + 1),
                                __ldg(a.r + 3 * (size_t)e + 2), Y, dY);
                float g0 = 0.f, g1 = 0.f, g2 = 0.f;
#pragma unroll
                for (int k = 0; k < D; ++k) {
                    g0 = fmaf(dLdY[k], dY[k][0], g0);
                    g1 = fmaf(dLdY[k], dY[k][1], g1);
                    g2 = fmaf(dLdY[k], dY[k][2], g2);
                }
                a.grad_r[3 * (size_t)e] = g0;
                a.grad_r[3 * (size_t)e + 1] = g1;
                a.grad_r[3 * (size_t)e + 2] = g2;
            }
        }
    }
    if (live && a.grad_x) {
        float4* o = a.grad_x + (size_t)node * D * C4 + cg;
#pragma unroll
        for (int k = 0; k < D; ++k) o[k * C4] = gx[k];
    }
}

template <int L>
cudaError_t launch_forward(bool o3, const FwdArgs& a, dim3 grid, cudaStream_t s) {
    if (o3)
        etp_fwd_kernel<L, true><<<grid, kThreads, 0, s>>>(a);
    else
        etp_fwd_kernel<L, false><<<grid, kThreads, 0, s>>>(a);
    return cudaGetLastError();
}

template <int L>
cudaError_t launch_backward(bool o3, const BwdArgs& a, dim3 grid, cudaStream_t s) {
    if (o3)
        etp_bwd_kernel<L, true><<<grid, kThreads, 0, s>>>(a);
    else
        etp_bwd_kernel<L, false><<<grid, kThreads, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace etp
