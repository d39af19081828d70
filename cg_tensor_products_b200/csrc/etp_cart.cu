// Cartesian edge convolution: the same edge tensor product with Cartesian
// couplings, features held as symmetric traceless (STF) tensors in their 2l + 1
// independent components, each path's contraction written out as explicit sums
// (compile-time sparse tables from the build-time generator).
//
// Passage: "FlashCart 如何让等变原子间势更快更准?", sections "FlashCart 用笛卡尔内核替代
// 球谐耦合" (Cartesian kernels in place of spherical-harmonic couplings; the speed comes
// from memory access and the aggregation of edge contributions) and
// "生成内核在高阶下胜过球谐基线" (edge convolution, forward and VJP, compared with
// spherical kernels at equal rank). The pages print no formula; the reading here:
//   - a rank-l feature is an STF tensor, stored by its entries with at most one z
//     index: (x^l, x^(l-1) y, .., y^l, x^(l-1) z, .., y^(l-1) z) for l >= 1;
//   - the edge attribute of rank l is the STF part of u (x) .. (x) u, u = r / |r|
//     (rank 0: 1; |r| < 1e-12: zero for l >= 1):
//       l = 1: (x, y, z);  l = 2: (x^2 - 1/3, xy, y^2 - 1/3, xz, yz);
//       l = 3: (x^3 - 3x/5, x^2 y - y/5, x y^2 - x/5, y^3 - 3y/5, x^2 z - z/5, xyz, y^2 z - z/5);
//   - path (l1, l2 -> l3): k index pairs contracted (one more through the
//     Levi-Civita symbol when l1 + l2 + l3 is odd), STF part of the rest, no
//     normalisation constant; its table Cc[i1][i2][i3] in independent components;
//   - out[i][l3] = sum over row i of sum_p w[e, p] * sum Cc_p[i1][i2][i3] Y[i2] x[src][i1].
// The VJP: grad_x (reverse CSR), grad_w and grad_r = (I - u u^T) grad_u / |r| per edge.
//
// Layout as the spherical kernels: x, out [N][(L+1)^2][C] (l blocks ascending, the
// independent components above), w [E][P][C]; a team of lanes over the channels
// (two per lane), equal contiguous ranges of edges, node rows summed in registers
// and stored once (a row cut by a range boundary leaves partial rows that the
// row-combine pass sums in range order).
#include <cuda_runtime.h>

#include <cstdint>

#include "etp_frame.cuh"

namespace etp {
namespace cart {

using frame::f2_fma;
using frame::f2_mul;
using frame::f2_zero;

constexpr int kThreads = 64;

struct Args {
    int N, E;
    const int32_t* row_ptr;
    const int32_t* src;
    const int32_t* rev_ptr;
    const int32_t* rev_perm;
    const int32_t* dst;  // may be null
    const float* r;
    const float2* x;
    const float2* w;
    const float2* g;
    float2* out;     // forward
    float2* grad_x;  // may be null
    float2* grad_w;  // may be null
    float* grad_r;   // may be null
    int C2, team, slices, ntasks;
    float2* part;    // partial rows [ntasks][2][D][C] of rows cut by task boundaries
};

// Edge attribute (independent STF components, blocks l = 0..L) of the unit vector
// (ux, uy, uz), and, with GRAD, its gradient in u (dY[k] = d Y_k / d u).
template <int L, bool GRAD>
__device__ __forceinline__ void cart_attr(float ux, float uy, float uz, bool zero, float (&Y)[(L + 1) * (L + 1)],
                                          float3 (&dY)[(L + 1) * (L + 1)]) {
    constexpr int D = (L + 1) * (L + 1);
#pragma unroll
    for (int k = 0; k < D; ++k) {
        Y[k] = 0.f;
        if constexpr (GRAD) dY[k] = make_float3(0.f, 0.f, 0.f);
    }
    Y[0] = 1.f;
    if (zero) return;
    if constexpr (L >= 1) {
        Y[1] = ux, Y[2] = uy, Y[3] = uz;
        if constexpr (GRAD) {
            dY[1] = make_float3(1.f, 0.f, 0.f);
            dY[2] = make_float3(0.f, 1.f, 0.f);
            dY[3] = make_float3(0.f, 0.f, 1.f);
        }
    }
    if constexpr (L >= 2) {
        const float t = 1.f / 3.f;
        Y[4] = ux * ux - t, Y[5] = ux * uy, Y[6] = uy * uy - t, Y[7] = ux * uz, Y[8] = uy * uz;
        if constexpr (GRAD) {
            dY[4] = make_float3(2.f * ux, 0.f, 0.f);
            dY[5] = make_float3(uy, ux, 0.f);
            dY[6] = make_float3(0.f, 2.f * uy, 0.f);
            dY[7] = make_float3(uz, 0.f, ux);
            dY[8] = make_float3(0.f, uz, uy);
        }
    }
    if constexpr (L >= 3) {
        const float f = 0.2f;
        Y[9] = ux * ux * ux - 3.f * f * ux;
        Y[10] = ux * ux * uy - f * uy;
        Y[11] = ux * uy * uy - f * ux;
        Y[12] = uy * uy * uy - 3.f * f * uy;
        Y[13] = ux * ux * uz - f * uz;
        Y[14] = ux * uy * uz;
        Y[15] = uy * uy * uz - f * uz;
        if constexpr (GRAD) {
            dY[9] = make_float3(3.f * ux * ux - 3.f * f, 0.f, 0.f);
            dY[10] = make_float3(2.f * ux * uy, ux * ux - f, 0.f);
            dY[11] = make_float3(uy * uy - f, 2.f * ux * uy, 0.f);
            dY[12] = make_float3(0.f, 3.f * uy * uy - 3.f * f, 0.f);
            dY[13] = make_float3(2.f * ux * uz, 0.f, ux * ux - f);
            dY[14] = make_float3(uy * uz, ux * uz, ux * uy);
            dY[15] = make_float3(0.f, 2.f * uy * uz, uy * uy - f);
        }
    }
}

struct Team {
    int T, S, tl, tb, task, slice, cp;
    unsigned tmask;
};
__device__ __forceinline__ Team team_of(const Args& a) {
    Team t;
    const int lane = threadIdx.x & 31;
    t.T = a.team;
    t.S = a.slices;
    t.tl = lane & (t.T - 1);
    t.tb = threadIdx.x / t.T;
    const int gt = blockIdx.x * (kThreads / t.T) + t.tb;
    t.task = gt / t.S;
    t.slice = gt - t.task * t.S;
    t.cp = t.slice * t.T + t.tl;
    const unsigned ones = t.T == 32 ? 0xffffffffu : ((1u << t.T) - 1u);
    t.tmask = ones << (lane & ~(t.T - 1) & 31);
    return t;
}

// Lane-owned double buffers in dynamic shared memory: per team [2][R][T] pairs,
// R = P weight entries + D node-row entries (the forward's source row, the
// backward's destination row). The next edge's rows are copied in (8-byte
// cp.async per lane and entry) while this edge is computed; each lane reads only
// its own entries, so no cross-lane synchronisation is needed.
template <int L, bool O3>
constexpr int buf_rows() {
    return PathSet<L, O3>::P + (L + 1) * (L + 1);
}
// The buffered kernels serve L <= 2. At L = 3 the buffers (51 KB per block) and
// the registers they take cost more occupancy than the hidden latency gains
// (measured: micro_l3 forward 0.89 -> 1.04 ms, VJP 4.08 -> 4.61 ms with them;
// micro_l2 0.38 -> 0.32 and 0.88 -> 0.75 ms): the direct kernels, which load
// each edge's rows where they use them, serve L = 3.
template <int L>
constexpr bool prefetch_rows() {
    return L <= 2;
}
template <int L, bool O3>
constexpr size_t buf_bytes() {
    return prefetch_rows<L>() ? (size_t)kThreads * 2 * buf_rows<L, O3>() * sizeof(float2) : 0;
}
__device__ __forceinline__ void cp_async_wait_one() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

// The unit vector of an edge, and whether it has none.
__device__ __forceinline__ float4 unit_of(const float* r, int e) {
    const float3 rv = frame::load_r(r, e);
    const float n2 = rv.x * rv.x + rv.y * rv.y + rv.z * rv.z;
    if (!(n2 >= 1e-24f)) return make_float4(0.f, 0.f, 0.f, 0.f);  // w = 0: no direction
    const float inv = rsqrtf(n2);
    return make_float4(rv.x * inv, rv.y * inv, rv.z * inv, inv);
}

// ---------------------------------------------------------------------------
// Direct form: each edge's rows read where they are used (L = 3).
template <int L, bool O3>
__global__ void __launch_bounds__(kThreads) etp_cart_fwd_direct_kernel(Args a) {
    using namespace frame;
    constexpr int D = (L + 1) * (L + 1);
    constexpr int P = PathSet<L, O3>::P;
    const Team tm = team_of(a);
    if (tm.task >= a.ntasks) return;
    int k0, k1;
    task_range(a.E, tm.task, a.ntasks, k0, k1);
    if (k0 >= k1) return;
    const int C2 = a.C2;
    int row = segment_of(a.row_ptr, a.N, k0);
    int row_lo = __ldg(a.row_ptr + row), row_hi = __ldg(a.row_ptr + row + 1);
    float2 acc[D];
#pragma unroll
    for (int k = 0; k < D; ++k) acc[k] = f2_zero();
    for (int e = k0; e < k1; ++e) {
        while (e >= row_hi && row < a.N - 1) {
            if (row_hi > max(row_lo, k0)) {
                store_row<D>(row_slot(a.out, a.part, row, row_lo, row_hi, k0, k1, tm.task, D * C2, tm.cp), C2, acc);
#pragma unroll
                for (int k = 0; k < D; ++k) acc[k] = f2_zero();
            }
            ++row;
            row_lo = row_hi;
            row_hi = __ldg(a.row_ptr + row + 1);
        }
        const int j = __ldg(a.src + e);
        if ((unsigned)j >= (unsigned)a.N) continue;
        const float4 u = unit_of(a.r, e);
        float Y[D];
        float3 dY[D];
        cart_attr<L, false>(u.x, u.y, u.z, u.w == 0.f, Y, dY);
        const float2* xs = a.x + (size_t)j * D * C2 + tm.cp;
        const float2* wrow = a.w + (size_t)e * P * C2 + tm.cp;
        float2 xv[D];
#pragma unroll
        for (int k = 0; k < D; ++k) xv[k] = __ldg(xs + k * C2);
        static_for<0, P>([&](auto pc) {
            constexpr int p = decltype(pc)::value;
            constexpr Path pt = PathSet<L, O3>::path(p);
            constexpr int off = etp_gen::kCartOff[pt.l1][pt.l2][pt.l3], cnt = etp_gen::kCartCnt[pt.l1][pt.l2][pt.l3];
            float2 t[2 * pt.l3 + 1];
#pragma unroll
            for (int m = 0; m < 2 * pt.l3 + 1; ++m) t[m] = f2_zero();
            static_for<0, cnt>([&](auto kc) {
                constexpr etp_gen::CgNz z = etp_gen::kCart[off + decltype(kc)::value];
                f2_fma(t[z.m3], (float)z.v * Y[pt.l2 * pt.l2 + z.m2], xv[pt.l1 * pt.l1 + z.m1]);
            });
            const float2 wp = __ldg(wrow + p * C2);
#pragma unroll
            for (int m = 0; m < 2 * pt.l3 + 1; ++m) acc[pt.l3 * pt.l3 + m] = __ffma2_rn(wp, t[m], acc[pt.l3 * pt.l3 + m]);
        });
    }
    store_row<D>(row_slot(a.out, a.part, row, row_lo, row_hi, k0, k1, tm.task, D * C2, tm.cp), C2, acc);
    if (tm.slice == 0 && tm.tl == 0) tail_record(a.part, a.ntasks, D * C2, tm.task, row, row_lo, row_hi, k0, k1);
}

// Buffered form (L <= 2).
template <int L, bool O3>
__global__ void __launch_bounds__(kThreads) etp_cart_fwd_buffered_kernel(Args a) {
    using namespace frame;
    constexpr int D = (L + 1) * (L + 1);
    constexpr int P = PathSet<L, O3>::P;
    const Team tm = team_of(a);
    if (tm.task >= a.ntasks) return;
    int k0, k1;
    task_range(a.E, tm.task, a.ntasks, k0, k1);
    if (k0 >= k1) return;
    const int C2 = a.C2;
    constexpr int R = buf_rows<L, O3>();
    extern __shared__ __align__(16) float2 cbuf[];
    float2* mine = cbuf + (size_t)tm.tb * 2 * R * tm.T + tm.tl;  // entry r of buffer b at (b R + r) T
    auto issue = [&](int e, int j, int b) {                       // edge e's weights and source row j
        j = (unsigned)j < (unsigned)a.N ? j : 0;
        const float2* wrow = a.w + (size_t)e * P * C2 + tm.cp;
        const float2* xs = a.x + (size_t)j * D * C2 + tm.cp;
        float2* dstb = mine + b * R * tm.T;
#pragma unroll
        for (int p = 0; p < P; ++p) cp_async8(dstb + p * tm.T, wrow + p * C2);
#pragma unroll
        for (int k = 0; k < D; ++k) cp_async8(dstb + (P + k) * tm.T, xs + k * C2);
        cp_async_commit();
    };
    int j_cur = __ldg(a.src + k0);  // source indices of this edge and the next
    int j_nx = k0 + 1 < k1 ? __ldg(a.src + k0 + 1) : 0;
    issue(k0, j_cur, 0);
    int row = segment_of(a.row_ptr, a.N, k0);
    int row_lo = __ldg(a.row_ptr + row), row_hi = __ldg(a.row_ptr + row + 1);
    float2 acc[D];
#pragma unroll
    for (int k = 0; k < D; ++k) acc[k] = f2_zero();
    for (int e = k0, it = 0; e < k1; ++e, ++it) {
        while (e >= row_hi && row < a.N - 1) {
            if (row_hi > max(row_lo, k0)) {
                store_row<D>(row_slot(a.out, a.part, row, row_lo, row_hi, k0, k1, tm.task, D * C2, tm.cp), C2, acc);
#pragma unroll
                for (int k = 0; k < D; ++k) acc[k] = f2_zero();
            }
            ++row;
            row_lo = row_hi;
            row_hi = __ldg(a.row_ptr + row + 1);
        }
        const int b = it & 1;
        const int j_after = e + 2 < k1 ? __ldg(a.src + e + 2) : 0;
        if (e + 1 < k1) {
            issue(e + 1, j_nx, b ^ 1);
            cp_async_wait_one();  // this edge's buffer (all but the copies just issued)
        } else {
            cp_async_wait_all();
        }
        const int j = j_cur;
        j_cur = j_nx;
        j_nx = j_after;
        if ((unsigned)j >= (unsigned)a.N) continue;
        const float4 u = unit_of(a.r, e);
        float Y[D];
        float3 dY[D];
        cart_attr<L, false>(u.x, u.y, u.z, u.w == 0.f, Y, dY);
        const float2* wbuf = mine + b * R * tm.T;
        float2 xv[D];
#pragma unroll
        for (int k = 0; k < D; ++k) xv[k] = wbuf[(P + k) * tm.T];
        static_for<0, P>([&](auto pc) {
            constexpr int p = decltype(pc)::value;
            constexpr Path pt = PathSet<L, O3>::path(p);
            constexpr int off = etp_gen::kCartOff[pt.l1][pt.l2][pt.l3], cnt = etp_gen::kCartCnt[pt.l1][pt.l2][pt.l3];
            float2 t[2 * pt.l3 + 1];
#pragma unroll
            for (int m = 0; m < 2 * pt.l3 + 1; ++m) t[m] = f2_zero();
            static_for<0, cnt>([&](auto kc) {
                constexpr etp_gen::CgNz z = etp_gen::kCart[off + decltype(kc)::value];
                f2_fma(t[z.m3], (float)z.v * Y[pt.l2 * pt.l2 + z.m2], xv[pt.l1 * pt.l1 + z.m1]);
            });
            const float2 wp = wbuf[p * tm.T];
#pragma unroll
            for (int m = 0; m < 2 * pt.l3 + 1; ++m) acc[pt.l3 * pt.l3 + m] = __ffma2_rn(wp, t[m], acc[pt.l3 * pt.l3 + m]);
        });
    }
    store_row<D>(row_slot(a.out, a.part, row, row_lo, row_hi, k0, k1, tm.task, D * C2, tm.cp), C2, acc);
    if (tm.slice == 0 && tm.tl == 0) tail_record(a.part, a.ntasks, D * C2, tm.task, row, row_lo, row_hi, k0, k1);
}

template <int L, bool O3>
__global__ void __launch_bounds__(kThreads) etp_cart_bwd_direct_kernel(Args a) {
    using namespace frame;
    constexpr int D = (L + 1) * (L + 1);
    constexpr int P = PathSet<L, O3>::P;
    const Team tm = team_of(a);
    if (tm.task >= a.ntasks) return;
    int k0, k1;
    task_range(a.E, tm.task, a.ntasks, k0, k1);
    if (k0 >= k1) return;
    const int C2 = a.C2;
    int row = segment_of(a.rev_ptr, a.N, k0);
    int row_lo = __ldg(a.rev_ptr + row), row_hi = __ldg(a.rev_ptr + row + 1);
    const int pos_end = __ldg(a.rev_ptr + a.N);
    float2 gx[D];
#pragma unroll
    for (int k = 0; k < D; ++k) gx[k] = f2_zero();
    for (int q = k0; q < k1; ++q) {
        while (q >= row_hi && row < a.N - 1) {
            if (row_hi > max(row_lo, k0)) {
                if (a.grad_x)
                    store_row<D>(row_slot(a.grad_x, a.part, row, row_lo, row_hi, k0, k1, tm.task, D * C2, tm.cp), C2,
                                 gx);
#pragma unroll
                for (int k = 0; k < D; ++k) gx[k] = f2_zero();
            }
            ++row;
            row_lo = row_hi;
            row_hi = __ldg(a.rev_ptr + row + 1);
        }
        const int e = __ldg(a.rev_perm + q);
        if ((unsigned)e >= (unsigned)a.E) continue;
        const int i = a.dst ? __ldg(a.dst + e) : row_of_edge(a.row_ptr, a.N, e);
        const bool ok = (unsigned)i < (unsigned)a.N && q < pos_end;
        float2* gwe = a.grad_w ? a.grad_w + (size_t)e * P * C2 + tm.cp : nullptr;
        float4 u = make_float4(0.f, 0.f, 0.f, 0.f);
        float s0 = 0.f, s1 = 0.f, s2 = 0.f;  // dL/du, this lane's channels
        if (ok) {
            u = unit_of(a.r, e);
            float Y[D];
            float3 dY[D];
            cart_attr<L, true>(u.x, u.y, u.z, u.w == 0.f, Y, dY);
            const float2* xs = a.x + (size_t)row * D * C2 + tm.cp;
            const float2* gs = a.g + (size_t)i * D * C2 + tm.cp;
            const float2* wrow = a.w + (size_t)e * P * C2 + tm.cp;
            float2 xv[D], gv[D], dy[D];
#pragma unroll
            for (int k = 0; k < D; ++k) {
                xv[k] = __ldg(xs + k * C2);
                gv[k] = __ldg(gs + k * C2);
                dy[k] = f2_zero();
            }
            static_for<0, P>([&](auto pc) {
                constexpr int p = decltype(pc)::value;
                constexpr Path pt = PathSet<L, O3>::path(p);
                constexpr int off = etp_gen::kCartOff[pt.l1][pt.l2][pt.l3];
                constexpr int cnt = etp_gen::kCartCnt[pt.l1][pt.l2][pt.l3];
                const float2 wp = __ldg(wrow + p * C2);
                float2 zp[2 * pt.l1 + 1], dyp[2 * pt.l2 + 1], gw = f2_zero();
#pragma unroll
                for (int m = 0; m < 2 * pt.l1 + 1; ++m) zp[m] = f2_zero();
#pragma unroll
                for (int m = 0; m < 2 * pt.l2 + 1; ++m) dyp[m] = f2_zero();
                static_for<0, cnt>([&](auto kc) {
                    constexpr etp_gen::CgNz z = etp_gen::kCart[off + decltype(kc)::value];
                    const float2 gval = gv[pt.l3 * pt.l3 + z.m3];
                    const float2 xg = f2_mul(xv[pt.l1 * pt.l1 + z.m1], gval);
                    const float t = (float)z.v * Y[pt.l2 * pt.l2 + z.m2];
                    f2_fma(zp[z.m1], t, gval);
                    f2_fma(gw, t, xg);
                    f2_fma(dyp[z.m2], (float)z.v, xg);
                });
#pragma unroll
                for (int m = 0; m < 2 * pt.l1 + 1; ++m) gx[pt.l1 * pt.l1 + m] = __ffma2_rn(wp, zp[m], gx[pt.l1 * pt.l1 + m]);
#pragma unroll
                for (int m = 0; m < 2 * pt.l2 + 1; ++m) dy[pt.l2 * pt.l2 + m] = __ffma2_rn(wp, dyp[m], dy[pt.l2 * pt.l2 + m]);
                if (gwe) gwe[p * C2] = gw;
            });
#pragma unroll
            for (int k = 1; k < D; ++k) {
                const float d = dy[k].x + dy[k].y;
                s0 = fmaf(d, dY[k].x, s0);
                s1 = fmaf(d, dY[k].y, s1);
                s2 = fmaf(d, dY[k].z, s2);
            }
        } else if (gwe) {
            for (int p = 0; p < P; ++p) gwe[p * C2] = f2_zero();
        }
        if (a.grad_r) {
            for (int o = 1; o < tm.T; o <<= 1) {
                s0 += __shfl_xor_sync(tm.tmask, s0, o);
                s1 += __shfl_xor_sync(tm.tmask, s1, o);
                s2 += __shfl_xor_sync(tm.tmask, s2, o);
            }
            if (tm.tl == 0) {
                // grad_r = (I - u u^T) dL/du / |r|   (u.w = 1/|r|, 0 without a direction)
                const float ud = u.x * s0 + u.y * s1 + u.z * s2;
                const float g0 = (s0 - ud * u.x) * u.w, g1 = (s1 - ud * u.y) * u.w, g2 = (s2 - ud * u.z) * u.w;
                float* gr = a.grad_r + 3 * (size_t)e;
                if (tm.S == 1) {
                    gr[0] = g0, gr[1] = g1, gr[2] = g2;
                } else {  // the channel slices' parts onto the zeroed output
                    atomicAdd(gr, g0), atomicAdd(gr + 1, g1), atomicAdd(gr + 2, g2);
                }
            }
        }
    }
    if (a.grad_x) {
        store_row<D>(row_slot(a.grad_x, a.part, row, row_lo, row_hi, k0, k1, tm.task, D * C2, tm.cp), C2, gx);
        if (tm.slice == 0 && tm.tl == 0) tail_record(a.part, a.ntasks, D * C2, tm.task, row, row_lo, row_hi, k0, k1);
    }
}

template <int L, bool O3>
__global__ void __launch_bounds__(kThreads) etp_cart_bwd_buffered_kernel(Args a) {
    using namespace frame;
    constexpr int D = (L + 1) * (L + 1);
    constexpr int P = PathSet<L, O3>::P;
    const Team tm = team_of(a);
    if (tm.task >= a.ntasks) return;
    int k0, k1;
    task_range(a.E, tm.task, a.ntasks, k0, k1);
    if (k0 >= k1) return;
    const int C2 = a.C2;
    constexpr int R = buf_rows<L, O3>();
    extern __shared__ __align__(16) float2 cbuf[];
    float2* mine = cbuf + (size_t)tm.tb * 2 * R * tm.T + tm.tl;  // entry r of buffer b at (b R + r) T
    auto dst_of = [&](int e) -> int {
        if ((unsigned)e >= (unsigned)a.E) return -1;
        return a.dst ? __ldg(a.dst + e) : row_of_edge(a.row_ptr, a.N, e);
    };
    auto issue = [&](int e, int i, int b) {  // edge e's weights and destination row i
        e = (unsigned)e < (unsigned)a.E ? e : 0;
        i = (unsigned)i < (unsigned)a.N ? i : 0;
        const float2* wrow = a.w + (size_t)e * P * C2 + tm.cp;
        const float2* gs = a.g + (size_t)i * D * C2 + tm.cp;
        float2* dstb = mine + b * R * tm.T;
#pragma unroll
        for (int p = 0; p < P; ++p) cp_async8(dstb + p * tm.T, wrow + p * C2);
#pragma unroll
        for (int k = 0; k < D; ++k) cp_async8(dstb + (P + k) * tm.T, gs + k * C2);
        cp_async_commit();
    };
    // this edge and the next, and their destination rows
    int e_cur = __ldg(a.rev_perm + k0);
    int i_cur = dst_of(e_cur);
    int e_nx = k0 + 1 < k1 ? __ldg(a.rev_perm + k0 + 1) : 0;
    int i_nx = k0 + 1 < k1 ? dst_of(e_nx) : 0;
    issue(e_cur, i_cur, 0);
    int row = segment_of(a.rev_ptr, a.N, k0);
    int row_lo = __ldg(a.rev_ptr + row), row_hi = __ldg(a.rev_ptr + row + 1);
    const int pos_end = __ldg(a.rev_ptr + a.N);
    float2 gx[D];
#pragma unroll
    for (int k = 0; k < D; ++k) gx[k] = f2_zero();
    for (int q = k0, it = 0; q < k1; ++q, ++it) {
        while (q >= row_hi && row < a.N - 1) {
            if (row_hi > max(row_lo, k0)) {
                if (a.grad_x)
                    store_row<D>(row_slot(a.grad_x, a.part, row, row_lo, row_hi, k0, k1, tm.task, D * C2, tm.cp), C2,
                                 gx);
#pragma unroll
                for (int k = 0; k < D; ++k) gx[k] = f2_zero();
            }
            ++row;
            row_lo = row_hi;
            row_hi = __ldg(a.rev_ptr + row + 1);
        }
        const int b = it & 1;
        const int e_after = q + 2 < k1 ? __ldg(a.rev_perm + q + 2) : 0;
        const int i_after = q + 2 < k1 ? dst_of(e_after) : 0;
        if (q + 1 < k1) {
            issue(e_nx, i_nx, b ^ 1);
            cp_async_wait_one();  // this edge's buffer (all but the copies just issued)
        } else {
            cp_async_wait_all();
        }
        const int e = e_cur, i = i_cur;
        e_cur = e_nx, i_cur = i_nx;
        e_nx = e_after, i_nx = i_after;
        if ((unsigned)e >= (unsigned)a.E) continue;
        const bool ok = (unsigned)i < (unsigned)a.N && q < pos_end;
        float2* gwe = a.grad_w ? a.grad_w + (size_t)e * P * C2 + tm.cp : nullptr;
        float4 u = make_float4(0.f, 0.f, 0.f, 0.f);
        float s0 = 0.f, s1 = 0.f, s2 = 0.f;  // dL/du, this lane's channels
        if (ok) {
            u = unit_of(a.r, e);
            // the attribute's gradient is formed after the paths (fewer live registers)
            float Y[D];
            float3 dY[D];
            cart_attr<L, false>(u.x, u.y, u.z, u.w == 0.f, Y, dY);
            const float2* xs = a.x + (size_t)row * D * C2 + tm.cp;
            const float2* wbuf = mine + b * R * tm.T;
            float2 xv[D], dy[D];
#pragma unroll
            for (int k = 0; k < D; ++k) {
                xv[k] = __ldg(xs + k * C2);
                dy[k] = f2_zero();
            }
            static_for<0, P>([&](auto pc) {
                constexpr int p = decltype(pc)::value;
                constexpr Path pt = PathSet<L, O3>::path(p);
                constexpr int off = etp_gen::kCartOff[pt.l1][pt.l2][pt.l3];
                constexpr int cnt = etp_gen::kCartCnt[pt.l1][pt.l2][pt.l3];
                const float2 wp = wbuf[p * tm.T];
                float2 zp[2 * pt.l1 + 1], dyp[2 * pt.l2 + 1], gw = f2_zero();
#pragma unroll
                for (int m = 0; m < 2 * pt.l1 + 1; ++m) zp[m] = f2_zero();
#pragma unroll
                for (int m = 0; m < 2 * pt.l2 + 1; ++m) dyp[m] = f2_zero();
                // this path's copies of the l3 block of g and the l2 block of Y: opaque to the compiler, so that it
                // does not keep the products of every path alive at once (they differ per path only by the table)
                float2 gl[2 * pt.l3 + 1];
                float yl[2 * pt.l2 + 1];
#pragma unroll
                for (int m = 0; m < 2 * pt.l3 + 1; ++m) {
                    gl[m] = wbuf[(P + pt.l3 * pt.l3 + m) * tm.T];  // the destination's g row, in the buffer
                    asm volatile("" : "+f"(gl[m].x), "+f"(gl[m].y));
                }
#pragma unroll
                for (int m = 0; m < 2 * pt.l2 + 1; ++m) {
                    yl[m] = Y[pt.l2 * pt.l2 + m];
                    asm volatile("" : "+f"(yl[m]));
                }
                static_for<0, cnt>([&](auto kc) {
                    constexpr etp_gen::CgNz z = etp_gen::kCart[off + decltype(kc)::value];
                    const float2 gval = gl[z.m3];
                    const float2 xg = f2_mul(xv[pt.l1 * pt.l1 + z.m1], gval);
                    const float t = (float)z.v * yl[z.m2];
                    f2_fma(zp[z.m1], t, gval);
                    f2_fma(gw, t, xg);
                    f2_fma(dyp[z.m2], (float)z.v, xg);
                });
#pragma unroll
                for (int m = 0; m < 2 * pt.l1 + 1; ++m) gx[pt.l1 * pt.l1 + m] = __ffma2_rn(wp, zp[m], gx[pt.l1 * pt.l1 + m]);
#pragma unroll
                for (int m = 0; m < 2 * pt.l2 + 1; ++m) dy[pt.l2 * pt.l2 + m] = __ffma2_rn(wp, dyp[m], dy[pt.l2 * pt.l2 + m]);
                if (gwe) gwe[p * C2] = gw;
            });
            cart_attr<L, true>(u.x, u.y, u.z, u.w == 0.f, Y, dY);
#pragma unroll
            for (int k = 1; k < D; ++k) {
                const float d = dy[k].x + dy[k].y;
                s0 = fmaf(d, dY[k].x, s0);
                s1 = fmaf(d, dY[k].y, s1);
                s2 = fmaf(d, dY[k].z, s2);
            }
        } else if (gwe) {
            for (int p = 0; p < P; ++p) gwe[p * C2] = f2_zero();
        }
        if (a.grad_r) {
            for (int o = 1; o < tm.T; o <<= 1) {
                s0 += __shfl_xor_sync(tm.tmask, s0, o);
                s1 += __shfl_xor_sync(tm.tmask, s1, o);
                s2 += __shfl_xor_sync(tm.tmask, s2, o);
            }
            if (tm.tl == 0) {
                // grad_r = (I - u u^T) dL/du / |r|   (u.w = 1/|r|, 0 without a direction)
                const float ud = u.x * s0 + u.y * s1 + u.z * s2;
                const float g0 = (s0 - ud * u.x) * u.w, g1 = (s1 - ud * u.y) * u.w, g2 = (s2 - ud * u.z) * u.w;
                float* gr = a.grad_r + 3 * (size_t)e;
                if (tm.S == 1) {
                    gr[0] = g0, gr[1] = g1, gr[2] = g2;
                } else {  // the channel slices' parts onto the zeroed output
                    atomicAdd(gr, g0), atomicAdd(gr + 1, g1), atomicAdd(gr + 2, g2);
                }
            }
        }
    }
    if (a.grad_x) {
        store_row<D>(row_slot(a.grad_x, a.part, row, row_lo, row_hi, k0, k1, tm.task, D * C2, tm.cp), C2, gx);
        if (tm.slice == 0 && tm.tl == 0) tail_record(a.part, a.ntasks, D * C2, tm.task, row, row_lo, row_hi, k0, k1);
    }
}

}  // namespace cart

// ---------------------------------------------------------------------------
namespace {

// Tasks of the forward or backward kernel: one wave, at least 16 edges each, no
// more tasks than rows.
// The kernel of a specialisation: the buffered form for L <= 2, the direct form at L = 3.
template <int L, bool O3>
const void* cart_kernel(bool backward) {
    if constexpr (cart::prefetch_rows<L>())
        return backward ? (const void*)cart::etp_cart_bwd_buffered_kernel<L, O3>
                        : (const void*)cart::etp_cart_fwd_buffered_kernel<L, O3>;
    else
        return backward ? (const void*)cart::etp_cart_bwd_direct_kernel<L, O3>
                        : (const void*)cart::etp_cart_fwd_direct_kernel<L, O3>;
}

template <int L, bool O3>
int cart_tasks(int C, int N, int E, bool backward) {
    const void* k = cart_kernel<L, O3>(backward);
    const int T = C / 2 < 32 ? C / 2 : 32, slices = C / (2 * T);
    int dev = 0, sms = 1, bps = 1;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
                                                   cudaSuccess || sms < 1)
        sms = 1;
    const size_t sm = cart::buf_bytes<L, O3>();
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&bps, k, cart::kThreads, sm) != cudaSuccess || bps < 1) bps = 1;
    const long long cap = (long long)sms * bps * (cart::kThreads / T) / slices;
    long long want = ((long long)E + 15) / 16;
    if (want > N) want = N;
    const long long nt = want < cap ? want : cap;
    return (int)(nt < 1 ? 1 : nt);
}

template <int L, bool O3>
cudaError_t launch_cart(cart::Args a, bool backward, size_t part_bytes, cudaStream_t s) {
    const void* k = cart_kernel<L, O3>(backward);
    const int C = 2 * a.C2, D = (L + 1) * (L + 1);
    a.ntasks = cart_tasks<L, O3>(C, a.N, a.E, backward);
    float2* rows = backward ? a.grad_x : a.out;
    if (rows && part_bytes < partial_rows_bytes(a.ntasks, D, C)) return cudaErrorInvalidValue;
    const int teams_per_block = cart::kThreads / a.team;
    const long long teams = (long long)a.ntasks * a.slices;
    const unsigned blocks = (unsigned)((teams + teams_per_block - 1) / teams_per_block);
    void* args[] = {&a};
    const size_t sm = cart::buf_bytes<L, O3>();
    cudaError_t err = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (err != cudaSuccess) return err;
    err = cudaLaunchKernel(k, dim3(blocks), dim3(cart::kThreads), args, sm, s);
    if (err != cudaSuccess || !rows) return err;
    return launch_combine_rows(backward ? a.rev_ptr : a.row_ptr, nullptr, a.N, a.E, a.ntasks, D * C / 4,
                               reinterpret_cast<const float4*>(a.part), reinterpret_cast<float4*>(rows), s);
}

cudaError_t dispatch_cart(int L, bool o3, const cart::Args& a, bool backward, size_t part_bytes, cudaStream_t s) {
    switch (L * 2 + (o3 ? 1 : 0)) {
        case 0: return launch_cart<0, false>(a, backward, part_bytes, s);
        case 1: return launch_cart<0, true>(a, backward, part_bytes, s);
        case 2: return launch_cart<1, false>(a, backward, part_bytes, s);
        case 3: return launch_cart<1, true>(a, backward, part_bytes, s);
        case 4: return launch_cart<2, false>(a, backward, part_bytes, s);
        case 5: return launch_cart<2, true>(a, backward, part_bytes, s);
        case 6: return launch_cart<3, false>(a, backward, part_bytes, s);
        default: return launch_cart<3, true>(a, backward, part_bytes, s);
    }
}

int cart_tasks_for(int L, bool o3, int C, int N, int E, bool backward) {
    switch (L * 2 + (o3 ? 1 : 0)) {
        case 0: return cart_tasks<0, false>(C, N, E, backward);
        case 1: return cart_tasks<0, true>(C, N, E, backward);
        case 2: return cart_tasks<1, false>(C, N, E, backward);
        case 3: return cart_tasks<1, true>(C, N, E, backward);
        case 4: return cart_tasks<2, false>(C, N, E, backward);
        case 5: return cart_tasks<2, true>(C, N, E, backward);
        case 6: return cart_tasks<3, false>(C, N, E, backward);
        default: return cart_tasks<3, true>(C, N, E, backward);
    }
}

}  // namespace

size_t cart_partial_bytes(int L, bool o3, int C, int N, int E) {
    if (E <= 0 || N <= 0) return 0;
    const int a = cart_tasks_for(L, o3, C, N, E, false), b = cart_tasks_for(L, o3, C, N, E, true);
    return partial_rows_bytes(a > b ? a : b, (L + 1) * (L + 1), C);
}

cudaError_t cart_forward(int L, bool o3, int C, int N, int E, const int32_t* row_ptr, const int32_t* src,
                         const float* r, const float* x, const float* w, float* out, void* part, size_t part_bytes,
                         cudaStream_t s) {
    const int D = (L + 1) * (L + 1);
    if (E == 0) return cudaMemsetAsync(out, 0, sizeof(float) * (size_t)N * D * C, s);
    const int team = C / 2 < 32 ? C / 2 : 32;
    cart::Args a{N, E, row_ptr, src, nullptr, nullptr, nullptr, r, reinterpret_cast<const float2*>(x),
                 reinterpret_cast<const float2*>(w), nullptr, reinterpret_cast<float2*>(out), nullptr, nullptr,
                 nullptr, C / 2, team, C / (2 * team), 1, static_cast<float2*>(part)};
    return dispatch_cart(L, o3, a, false, part_bytes, s);
}

cudaError_t cart_backward(int L, bool o3, int C, int N, int E, const int32_t* row_ptr, const int32_t* rev_ptr,
                          const int32_t* rev_perm, const int32_t* dst, const float* r, const float* x, const float* w,
                          const float* g, float* grad_x, float* grad_w, float* grad_r, void* part,
                          size_t part_bytes, cudaStream_t s) {
    const int D = (L + 1) * (L + 1);
    const int team = C / 2 < 32 ? C / 2 : 32, slices = C / (2 * team);
    cudaError_t err;
    // with two channel slices, grad_r is the sum of the slices' two terms (added onto zero: order-free)
    if (grad_r && slices > 1 && (err = cudaMemsetAsync(grad_r, 0, sizeof(float) * 3 * (size_t)E, s)) != cudaSuccess)
        return err;
    if (E == 0) return grad_x ? cudaMemsetAsync(grad_x, 0, sizeof(float) * (size_t)N * D * C, s) : cudaSuccess;
    cart::Args a{N, E, row_ptr, nullptr, rev_ptr, rev_perm, dst, r, reinterpret_cast<const float2*>(x),
                 reinterpret_cast<const float2*>(w), reinterpret_cast<const float2*>(g), nullptr,
                 reinterpret_cast<float2*>(grad_x), reinterpret_cast<float2*>(grad_w), grad_r, C / 2, team, slices, 1,
                 static_cast<float2*>(part)};
    return dispatch_cart(L, o3, a, true, part_bytes, s);
}

}  // namespace etp
