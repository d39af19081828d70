// Node-local product: features of higher correlation order built from one node's
// own features by repeated weighted products, the ranks kept at or below L after
// every step.
//
// Passages: "FlashCart 如何让等变原子间势更快更准?", section "FlashCart 用笛卡尔内核替代
// 球谐耦合" (features built recursively and brought back to a fixed width at each
// step) and section "生成内核在高阶下胜过球谐基线" (the node-local product at 4096
// nodes x 128 channels, rank 3, order 4; weighted products applied one step at a
// time, only ranks up to the chosen maximum kept). The pages give no formula; the
// reading here:
//   B(1) = x;  B(k+1)_l3[c] = sum_{p = (l1, l2, l3)} w[k-1, p, c] couple_p(B(k)_l1[c], x_l2[c]),
//   k = 1 .. K-1, output B(K); the plan's paths (l1, l2 and l3 in 0..L, triangle
//   rule, natural parities when the plan has them); couple_p the real
//   Clebsch-Gordan coupling, or the Cartesian coupling of STF tensors held by their
//   independent components (the tables of the Cartesian edge convolution).
//
// Layout: x, out [N][(L+1)^2][C]; w [K-1][P][C], shared by every node. One thread
// owns two channels of one node: its x, B(k) and B(k+1) live in registers, so the
// whole ladder reads x once and writes B(K) once. The arithmetic is grouped by
// operand ranks (l1, l2): every product B_l1[m1] x_l2[m2] that some path uses is
// formed once (one packed multiply) and scattered, with its compile-time
// coefficients, into the accumulators of all paths (l1, l2, *); each path's sum is
// then weighted into B(k+1)_l3. Every step is a packed fp32x2 instruction for the
// thread's two channels (the coefficient as a register pair). Channels never mix:
// no shared memory, no synchronisation, no atomics.
#include <cuda_runtime.h>

#include <cstdint>

#include "etp_device.cuh"
#include "etp_frame.cuh"
#include "etp_internal.h"

namespace etp {
namespace nodeprod {

constexpr int kThreads = 64;
constexpr int kMaxGroups = (etp_gen::kLmax + 1) * (etp_gen::kLmax + 1);
constexpr int kMaxPairs = kMaxGroups * (2 * etp_gen::kLmax + 1) * (2 * etp_gen::kLmax + 1);
constexpr int kMaxTerms = etp_gen::kCgTotal > etp_gen::kCartTotal ? etp_gen::kCgTotal : etp_gen::kCartTotal;

// One coefficient: accumulator slot (offset of its path's block + m3) and value.
struct Term {
    int slot;
    float v;
};
// One product B_l1[m1] x_l2[m2] and its coefficients terms[first .. first + count).
struct Pair {
    int m1, m2, first, count;
};
// The paths (l1, l2, l3) that share the operand ranks (l1, l2), with the offsets of
// their accumulator blocks, and their pairs pairs[pair0 .. pair0 + npairs).
struct Group {
    int l1, l2, npaths;
    int path[4], l3[4], toff[4];
    int tdim, pair0, npairs;
};
struct Table {
    int ngroups, npairs, nterms;
    Group g[kMaxGroups];
    Pair pr[kMaxPairs];
    Term tm[kMaxTerms];
};

template <bool CART>
constexpr etp_gen::CgNz coupling_entry(int l1, int l2, int l3, int q) {
    return CART ? etp_gen::kCart[etp_gen::kCartOff[l1][l2][l3] + q] : etp_gen::kCg[etp_gen::kCgOff[l1][l2][l3] + q];
}
template <bool CART>
constexpr int coupling_count(int l1, int l2, int l3) {
    return CART ? etp_gen::kCartCnt[l1][l2][l3] : etp_gen::kCgCnt[l1][l2][l3];
}

template <int L, bool O3, bool CART>
constexpr Table make_table() {
    using PS = PathSet<L, O3>;
    Table t{};
    for (int l1 = 0; l1 <= L; ++l1)
        for (int l2 = 0; l2 <= L; ++l2) {
            Group G{};
            G.l1 = l1;
            G.l2 = l2;
            for (int p = 0; p < PS::P; ++p) {
                const Path pt = PS::path(p);
                if (pt.l1 != l1 || pt.l2 != l2) continue;
                G.path[G.npaths] = p;
                G.l3[G.npaths] = pt.l3;
                G.toff[G.npaths] = G.tdim;
                G.tdim += 2 * pt.l3 + 1;
                ++G.npaths;
            }
            if (G.npaths == 0) continue;
            G.pair0 = t.npairs;
            for (int m1 = 0; m1 <= 2 * l1; ++m1)
                for (int m2 = 0; m2 <= 2 * l2; ++m2) {
                    const int first = t.nterms;
                    for (int k = 0; k < G.npaths; ++k) {
                        const int cnt = coupling_count<CART>(l1, l2, G.l3[k]);
                        for (int q = 0; q < cnt; ++q) {
                            const etp_gen::CgNz z = coupling_entry<CART>(l1, l2, G.l3[k], q);
                            if (z.m1 == m1 && z.m2 == m2) t.tm[t.nterms++] = Term{G.toff[k] + z.m3, (float)z.v};
                        }
                    }
                    if (t.nterms > first) t.pr[t.npairs++] = Pair{m1, m2, first, t.nterms - first};
                }
            G.npairs = t.npairs - G.pair0;
            t.g[t.ngroups++] = G;
        }
    return t;
}

template <int L, bool O3, bool CART>
constexpr Table kTable = make_table<L, O3, CART>();

// FP32 operations per node, channel and step: one multiply per product, one FMA per
// coefficient, one FMA per weighted output component.
template <int L, bool O3, bool CART>
constexpr int ops_per_step() {
    constexpr Table t = make_table<L, O3, CART>();
    int n = t.npairs + t.nterms;
    for (int g = 0; g < t.ngroups; ++g) n += t.g[g].tdim;
    return n;
}

template <int L, bool O3, bool CART>
__global__ void __launch_bounds__(kThreads) etp_node_product_kernel(int N, int K, int C2, const float2* __restrict__ x,
                                                                    const float2* __restrict__ w,
                                                                    float2* __restrict__ out) {
    using frame::f2_fma;
    using frame::f2_mul;
    using frame::f2_zero;
    constexpr int D = (L + 1) * (L + 1);
    constexpr int P = PathSet<L, O3>::P;
    constexpr int NG = kTable<L, O3, CART>.ngroups;
    const long long tid = (long long)blockIdx.x * kThreads + threadIdx.x;
    if (tid >= (long long)N * C2) return;
    const int n = (int)(tid / C2), cp = (int)(tid % C2);
    const float2* xs = x + (size_t)n * D * C2 + cp;
    float2 xv[D], B[D];
#pragma unroll
    for (int k = 0; k < D; ++k) {
        xv[k] = __ldg(xs + k * C2);
        B[k] = xv[k];
    }
    for (int step = 0; step + 1 < K; ++step) {
        const float2* ws = w + (size_t)step * P * C2 + cp;
        float2 nb[D];
#pragma unroll
        for (int k = 0; k < D; ++k) nb[k] = f2_zero();
        static_for<0, NG>([&](auto gc) {
            constexpr Group G = kTable<L, O3, CART>.g[decltype(gc)::value];
            float2 t[G.tdim];
#pragma unroll
            for (int k = 0; k < G.tdim; ++k) t[k] = f2_zero();
            static_for<0, G.npairs>([&](auto pc) {
                constexpr Pair pr = kTable<L, O3, CART>.pr[G.pair0 + decltype(pc)::value];
                const float2 q = f2_mul(B[G.l1 * G.l1 + pr.m1], xv[G.l2 * G.l2 + pr.m2]);
                static_for<0, pr.count>([&](auto qc) {
                    constexpr Term tm = kTable<L, O3, CART>.tm[pr.first + decltype(qc)::value];
                    t[tm.slot] = __ffma2_rn(make_float2(tm.v, tm.v), q, t[tm.slot]);
                });
            });
            static_for<0, G.npaths>([&](auto kc) {
                constexpr int k = decltype(kc)::value;
                const float2 wp = __ldg(ws + G.path[k] * C2);
#pragma unroll
                for (int m = 0; m < 2 * G.l3[k] + 1; ++m) f2_fma(nb[G.l3[k] * G.l3[k] + m], wp, t[G.toff[k] + m]);
            });
        });
#pragma unroll
        for (int k = 0; k < D; ++k) B[k] = nb[k];
    }
    float2* os = out + (size_t)n * D * C2 + cp;
#pragma unroll
    for (int k = 0; k < D; ++k) os[k * C2] = B[k];
}

template <int L, bool O3, bool CART>
cudaError_t launch(int N, int K, int C, const float* x, const float* w, float* out, cudaStream_t s) {
    const int C2 = C / 2;
    const long long threads = (long long)N * C2;
    const long long blocks = (threads + kThreads - 1) / kThreads;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
    etp_node_product_kernel<L, O3, CART><<<(unsigned)blocks, kThreads, 0, s>>>(
        N, K, C2, reinterpret_cast<const float2*>(x), reinterpret_cast<const float2*>(w),
        reinterpret_cast<float2*>(out));
    return cudaGetLastError();
}

template <int L, bool O3>
cudaError_t launch_form(bool cart, int N, int K, int C, const float* x, const float* w, float* out, cudaStream_t s) {
    return cart ? launch<L, O3, true>(N, K, C, x, w, out, s) : launch<L, O3, false>(N, K, C, x, w, out, s);
}

template <int L, bool O3>
int ops_form(bool cart) {
    return cart ? ops_per_step<L, O3, true>() : ops_per_step<L, O3, false>();
}

}  // namespace nodeprod

cudaError_t node_product(int L, bool o3, bool cart, int C, int N, int K, const float* x, const float* w, float* out,
                         cudaStream_t s) {
    if (N == 0) return cudaSuccess;
    switch (L * 2 + (o3 ? 1 : 0)) {
        case 0: return nodeprod::launch_form<0, false>(cart, N, K, C, x, w, out, s);
        case 1: return nodeprod::launch_form<0, true>(cart, N, K, C, x, w, out, s);
        case 2: return nodeprod::launch_form<1, false>(cart, N, K, C, x, w, out, s);
        case 3: return nodeprod::launch_form<1, true>(cart, N, K, C, x, w, out, s);
        case 4: return nodeprod::launch_form<2, false>(cart, N, K, C, x, w, out, s);
        case 5: return nodeprod::launch_form<2, true>(cart, N, K, C, x, w, out, s);
        case 6: return nodeprod::launch_form<3, false>(cart, N, K, C, x, w, out, s);
        default: return nodeprod::launch_form<3, true>(cart, N, K, C, x, w, out, s);
    }
}

int node_product_ops(int L, bool o3, bool cart) {
    switch (L * 2 + (o3 ? 1 : 0)) {
        case 0: return nodeprod::ops_form<0, false>(cart);
        case 1: return nodeprod::ops_form<0, true>(cart);
        case 2: return nodeprod::ops_form<1, false>(cart);
        case 3: return nodeprod::ops_form<1, true>(cart);
        case 4: return nodeprod::ops_form<2, false>(cart);
        case 5: return nodeprod::ops_form<2, true>(cart);
        case 6: return nodeprod::ops_form<3, false>(cart);
        default: return nodeprod::ops_form<3, true>(cart);
    }
}

}  // namespace etp
