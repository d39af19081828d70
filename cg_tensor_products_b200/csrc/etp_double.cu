// VJP of the VJP (double backward) of the edge tensor product, in the edge frame.
//
// For cotangents gg_x, gg_w, gg_r of the first VJP's outputs (grad_x, grad_w,
// grad_r), the gradients of <gg_x, grad_x> + <gg_w, grad_w> + <gg_r, grad_r> with
// respect to g (= grad_out), x, w and r. The tensor product is linear in x, w, g and
// in the harmonics Y, so every term is a first-order contraction with one input
// replaced by its cotangent, or Y by its directional derivative dY/dr . gg_r, plus
// one term through the Hessian of Y. In the edge frame (R u = z, x' = D(R) x,
// g' = D(R) g[dst], M = sum_p w_p B_p) a move of r along v turns the frame by the
// angles w = (v'_y, -v'_x), v' = R v / |r|, about the frame's x and y axes, which
// act on the harmonics through the generators K_x, K_y (K_w = w_x K_x + w_y K_y):
//
//   grad_g[dst] += D^T ( M(w) ggx' + M(gg_w) x' + [M(w), K_w] x' )
//   grad_x[src] += D^T ( M(gg_w)^T g' + [M(w)^T, K_w] g' )
//   grad_w_p    += g'^T B_p ggx' + g'^T B_p (K_w x') + (K_w g')^T B_p x'
//   grad_r      += R^T (c0, c1, c2) / |r|  with, summed over channels and written with
//                  f_a(v, s) = <K_a v, s>,  y = M x', z = M^T g', y5 = M ggx', y6 = M(gg_w) x',
//                  z2 = M(gg_w)^T g', yy = [M, K_w] x', zz = [M^T, K_w] g':
//     c0 = -f_y(ggx', z) + f_y(x', v'_z z - z2 - zz) + f_y(g', v'_z y - y5 - y6 - yy)
//     c1 =  f_x(ggx', z) + f_x(x', z2 + zz - v'_z z) + f_x(g', y5 + y6 + yy - v'_z y)
//     c2 = -w_x (f_x(x', z) + f_x(g', y)) - w_y (f_y(x', z) + f_y(g', y))
//   (the first-order grad_r with x <- gg_x and with w <- gg_w, plus the Hessian term
//   d/dr [grad_r . gg_r], whose frame components follow from the frame turning
//   with r at second order).
// Passage: "FlashCart 如何让等变原子间势更快更准?", section "生成内核在高阶下胜过球谐基线":
// the VJP of the VJP is timed beside the forward and the VJP (force-loss training
// differentiates the forces, built from grad_r, with respect to the parameters).
//
// Two kernels, laid out like the first-order ones: edge-balanced tasks of
// contiguous edges, a team of lanes over the channels (two per lane), node rows
// summed in registers and stored once (a row cut by a task boundary leaves partial
// rows that the row-combine pass sums in task order):
//   dd_dst: CSR order, grad_g;
//   dd_src: reverse-CSR order, grad_x, and per edge grad_w and grad_r.
// The frame vectors of an edge sit in lane-owned shared memory (registers), and so
// do the edge's weight and cotangent-weight rows, copied in asynchronously at the
// start of the edge (their latency hides behind the frame work).
#include <cuda_runtime.h>

#include <cstdint>

#include "etp_frame.cuh"

namespace etp {
namespace dd {

using frame::f2_add;
using frame::f2_dup;
using frame::f2_fma;
using frame::f2_mul;
using frame::f2_zero;
using frame::Frame;

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
    const float2* ggx;  // may be null (zero)
    const float2* ggw;  // may be null (zero)
    const float* ggr;   // may be null (zero)
    float2* grad_g;     // may be null
    float2* grad_x;     // may be null
    float2* grad_w;     // may be null
    float* grad_r;      // may be null
    int C2;             // channel pairs
    int team, slices, ntasks;
    float2* part;       // partial rows [ntasks][2][D][C] of rows cut by task boundaries
};

__device__ __forceinline__ float2 f2_sub(float2 a, float2 b) { return make_float2(a.x - b.x, a.y - b.y); }
__device__ __forceinline__ float2 f2_scale(float s, float2 a) { return make_float2(s * a.x, s * a.y); }

// out = (wx K_x + wy K_y) in, for one block of degree l
template <int l>
__device__ __forceinline__ void gen_apply(float wx, float wy, const float2* in, float2* out) {
    constexpr int d = 2 * l + 1;
#pragma unroll
    for (int a = 0; a < d; ++a) out[a] = f2_zero();
    if constexpr (l > 0) {
        static_for<0, d>([&](auto ac) {
            constexpr int a = decltype(ac)::value;
            static_for<0, d>([&](auto bc) {
                constexpr int b = decltype(bc)::value;
                constexpr float kx = (float)etp_gen::kGen[0][l][a][b];
                constexpr float ky = (float)etp_gen::kGen[1][l][a][b];
                if constexpr (kx != 0.f || ky != 0.f) {
                    const float k = kx * wx + ky * wy;
                    f2_fma(out[a], k, in[b]);
                }
            });
        });
    }
}

// f_a(v, s) = <K_a v, s> for one block of degree l, per channel of the pair
template <int l, int axis>
__device__ __forceinline__ float2 gform(const float2* v, const float2* s) {
    const float2 t = frame::gen_form<l, axis>(v, s);  // -<K_a v, s>
    return make_float2(-t.x, -t.y);
}

// Combined frame weights of the (l1, l3) group, read from a global weight row
// (this lane's channel pair of every path; p-th path at p * C2).
template <int L, bool O3, int l1, int l3>
__device__ __forceinline__ void group_weights_g(const float2* __restrict__ wrow, int C2, float2 (&We)[4],
                                                float2 (&Wo)[4]) {
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        We[m] = f2_zero();
        Wo[m] = f2_zero();
    }
    if (wrow == nullptr) return;
    static_for<0, L + 1>([&](auto l2c) {
        constexpr int l2 = decltype(l2c)::value;
        if constexpr (PathSet<L, O3>::allowed(l1, l2, l3)) {
            constexpr int p = frame::path_index<L, O3>(l1, l2, l3);
            const float2 w = __ldg(wrow + p * C2);
            constexpr bool odd = (l1 + l2 + l3) % 2 == 1;
            static_for<0, frame::cmin(l1, l3) + 1>([&](auto mc) {
                constexpr int mu = decltype(mc)::value;
                constexpr float b = (float)etp_gen::kFrameB[l1][l2][l3][mu];
                if constexpr (b != 0.f) {
                    if constexpr (odd)
                        f2_fma(Wo[mu], b, w);
                    else
                        f2_fma(We[mu], b, w);
                }
            });
        }
    });
}

// Products of the frame components that B_p couples, symmetrised in +-mu, for a
// (g-like, x-like) pair of blocks l3 / l1; added to Pe / Po.
template <int l1, int l3>
__device__ __forceinline__ void add_products(const float2* gl3, const float2* xl1, float2 (&Pe)[4], float2 (&Po)[4]) {
    constexpr int mn = frame::cmin(l1, l3);
    static_for<0, mn + 1>([&](auto mc) {
        constexpr int mu = decltype(mc)::value;
        const float2 a1 = gl3[l3 + mu], a2 = gl3[l3 - mu];
        const float2 b1 = xl1[l1 + mu], b2 = xl1[l1 - mu];
        if constexpr (mu == 0) {
            f2_fma(Pe[0], a1, b1);
        } else {
            f2_fma(Pe[mu], a1, b1);
            f2_fma(Pe[mu], a2, b2);
            f2_fma(Po[mu], a1, b2);
            frame::f2_fms(Po[mu], a2, b1);
        }
    });
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
    t.tb = threadIdx.x / t.T;  // team in block
    const int gt = blockIdx.x * (kThreads / t.T) + t.tb;
    t.task = gt / t.S;
    t.slice = gt - t.task * t.S;
    t.cp = t.slice * t.T + t.tl;
    const unsigned ones = t.T == 32 ? 0xffffffffu : ((1u << t.T) - 1u);
    t.tmask = ones << (lane & ~(t.T - 1) & 31);
    return t;
}

__device__ __forceinline__ void load_fit(float* fit) {
    for (int k = threadIdx.x; k < frame::kFitFloats; k += blockDim.x) fit[k] = frame::c_fit.v[k];
    __syncthreads();
}

// Per team in shared memory: the Wigner buffers, then lane-owned frame vectors
// [v][k] float2 (the destination kernel: x', ggx' + K_w x'; the source kernel:
// x', ggx', g', K_w x', K_w g').
// After those, lane-owned rows of the edge's weights and cotangent weights
// ([p][lane] float2 each), filled by per-lane asynchronous copies at the start of
// the edge so that the frame work hides their latency; in the source kernel the
// destination's g row arrives the same way, in the slot of its frame vector.
template <int L, bool O3>
constexpr int dst_team_floats(int T) {
    return frame::kTeamFloats + (2 * (L + 1) * (L + 1) + 2 * PathSet<L, O3>::P) * T * 2;
}
// The source kernel buffers the cotangent-weight row too for L <= 2; at L = 3 that
// row (8.5 KB more per team) would leave room for three blocks per SM instead of
// four, so there gg_w is read where it is used.
template <int L>
constexpr bool src_buffers_ggw() {
    return L <= 2;
}
template <int L, bool O3>
constexpr int src_team_floats(int T) {
    return frame::kTeamFloats + (3 * (L + 1) * (L + 1) + (src_buffers_ggw<L>() ? 2 : 1) * PathSet<L, O3>::P) * T * 2;
}

// This lane's channel pair of every path of two weight rows, into lane-owned
// shared memory (rows at p * T), by 8-byte asynchronous copies; one commit group.
template <int P>
__device__ __forceinline__ void copy_weight_rows(float2* wbuf, float2* gwbuf, const float2* wrow, const float2* gwrow,
                                                 int C2, int T) {
#pragma unroll
    for (int p = 0; p < P; ++p) {
        frame::cp_async8(wbuf + p * T, wrow + p * C2);
        if (gwrow) frame::cp_async8(gwbuf + p * T, gwrow + p * C2);
    }
}

// ---------------------------------------------------------------------------
// grad_g: destination order.
template <int L, bool O3>
__global__ void __launch_bounds__(kThreads) etp_dd_dst_kernel(Args a) {
    using namespace frame;
    constexpr int D = (L + 1) * (L + 1);
    extern __shared__ __align__(16) float smem[];
    load_fit(smem);
    const Team tm = team_of(a);
    if (tm.task >= a.ntasks) return;  // whole teams leave together
    int k0, k1;
    task_range(a.E, tm.task, a.ntasks, k0, k1);
    if (k0 >= k1) return;
    constexpr int P = PathSet<L, O3>::P;
    const int C2 = a.C2, T = tm.T;
    float* ybuf = smem + kFitStride + tm.tb * dst_team_floats<L, O3>(T);
    float* dbuf = ybuf + kYbufFloats;
    float2* vec = reinterpret_cast<float2*>(ybuf + kTeamFloats) + tm.tl;  // [v][k] at (v * D + k) * T
    auto V = [&](int v, int k) -> float2& { return vec[(v * D + k) * T]; };
    float2* wbuf = vec + 2 * D * T;  // [p] at p * T
    float2* gwbuf = wbuf + P * T;
    int row = segment_of(a.row_ptr, a.N, k0);
    int row_lo = __ldg(a.row_ptr + row), row_hi = __ldg(a.row_ptr + row + 1);
    float2 acc[D];
#pragma unroll
    for (int k = 0; k < D; ++k) acc[k] = f2_zero();
    for (int e = k0; e < k1; ++e) {
        while (e >= row_hi && row < a.N - 1) {
            if (row_hi > max(row_lo, k0)) {
                if (a.grad_g)
                    store_row<D>(row_slot(a.grad_g, a.part, row, row_lo, row_hi, k0, k1, tm.task, D * C2, tm.cp), C2,
                                 acc);
#pragma unroll
                for (int k = 0; k < D; ++k) acc[k] = f2_zero();
            }
            ++row;
            row_lo = row_hi;
            row_hi = __ldg(a.row_ptr + row + 1);
        }
        const int j = __ldg(a.src + e);
        if ((unsigned)j >= (unsigned)a.N) continue;  // an invalid source contributes nothing (team-uniform)
        const float3 rv = load_r(a.r, e);
        const Frame f = make_frame(rv.x, rv.y, rv.z);
        const float2* xs = a.x + (size_t)j * D * C2 + tm.cp;
        const float2* gxs = a.ggx ? a.ggx + (size_t)j * D * C2 + tm.cp : nullptr;
        const float2* wrow = a.w + (size_t)e * P * C2 + tm.cp;
        const float2* gwrow = a.ggw ? a.ggw + (size_t)e * P * C2 + tm.cp : nullptr;
        copy_weight_rows<P>(wbuf, gwbuf, wrow, gwrow, C2, T);
        cp_async_commit();
        if (!f.degenerate) {
            team_wigner<L>(f, tm.tl, tm.T, tm.tmask, ybuf, dbuf, smem);
            float wx = 0.f, wy = 0.f;
            if (a.ggr) {
                const float gx0 = __ldg(a.ggr + 3 * (size_t)e), gy0 = __ldg(a.ggr + 3 * (size_t)e + 1),
                            gz0 = __ldg(a.ggr + 3 * (size_t)e + 2);
                const float vx = (f.R[0] * gx0 + f.R[1] * gy0 + f.R[2] * gz0) * f.inv_rho;
                const float vy = (f.R[3] * gx0 + f.R[4] * gy0 + f.R[5] * gz0) * f.inv_rho;
                wx = vy;
                wy = -vx;
            }
            {  // x' (vector 0) and ggx' + K_w x' (vector 1) into this lane's shared-memory rows
                float2 v[D], u[D];
#pragma unroll
                for (int k = 0; k < D; ++k) v[k] = __ldg(xs + k * C2);
                rotate_all<L>(f, dbuf, v, u);
#pragma unroll
                for (int k = 0; k < D; ++k) {
                    V(0, k) = u[k];
                    v[k] = gxs ? __ldg(gxs + k * C2) : f2_zero();
                }
                float2 gp[D];
                rotate_all<L>(f, dbuf, v, gp);
                static_for<0, L + 1>([&](auto lc) {
                    constexpr int l = decltype(lc)::value;
                    float2 t[2 * l + 1];
                    gen_apply<l>(wx, wy, u + l * l, t);
#pragma unroll
                    for (int m = 0; m < 2 * l + 1; ++m) V(1, l * l + m) = f2_add(gp[l * l + m], t[m]);
                });
            }
            cp_async_wait_all();  // this lane's weight rows
            static_for<0, L + 1>([&](auto l3c) {
                constexpr int l3 = decltype(l3c)::value;
                constexpr int d3 = 2 * l3 + 1;
                float2 y[d3], y3[d3];
#pragma unroll
                for (int m = 0; m < d3; ++m) y[m] = y3[m] = f2_zero();
                static_for<0, L + 1>([&](auto l1c) {
                    constexpr int l1 = decltype(l1c)::value;
                    if constexpr (has_type<L, O3>(l1, l3, 0) || has_type<L, O3>(l1, l3, 1)) {
                        float2 xp[2 * l1 + 1], sum[2 * l1 + 1];
#pragma unroll
                        for (int m = 0; m < 2 * l1 + 1; ++m) {
                            xp[m] = V(0, l1 * l1 + m);
                            sum[m] = V(1, l1 * l1 + m);
                        }
                        float2 We[4], Wo[4];
                        group_weights<L, O3, l1, l3>(wbuf, T, We, Wo);
                        apply_M<L, O3, l1, l3>(We, Wo, sum, y);
                        apply_M<L, O3, l1, l3>(We, Wo, xp, y3);
                        if (gwrow) {
                            group_weights<L, O3, l1, l3>(gwbuf, T, We, Wo);
                            apply_M<L, O3, l1, l3>(We, Wo, xp, y);
                        }
                    }
                });
                float2 ky[d3];
                gen_apply<l3>(wx, wy, y3, ky);
#pragma unroll
                for (int m = 0; m < d3; ++m) y[m] = f2_sub(y[m], ky[m]);
                rotate<l3, true, true>(f, dbuf, y, acc + l3 * l3);
            });
        } else {
            // no direction: only the paths (l, 0, l) act, each as the identity; no derivative in r
            cp_async_wait_all();
            static_for<0, L + 1>([&](auto lc) {
                constexpr int l = decltype(lc)::value;
                constexpr int p0 = path_index<L, O3>(l, 0, l);
                const float2 w0 = __ldg(wrow + p0 * C2);
                const float2 gw0 = gwrow ? __ldg(gwrow + p0 * C2) : f2_zero();
#pragma unroll
                for (int m = 0; m < 2 * l + 1; ++m) {
                    if (gxs) f2_fma(acc[l * l + m], w0, __ldg(gxs + (l * l + m) * C2));
                    f2_fma(acc[l * l + m], gw0, __ldg(xs + (l * l + m) * C2));
                }
            });
        }
    }
    if (a.grad_g) {
        store_row<D>(row_slot(a.grad_g, a.part, row, row_lo, row_hi, k0, k1, tm.task, D * C2, tm.cp), C2, acc);
        if (tm.slice == 0 && tm.tl == 0) tail_record(a.part, a.ntasks, D * C2, tm.task, row, row_lo, row_hi, k0, k1);
    }
}


template <int L, bool O3>
__global__ void __launch_bounds__(kThreads) etp_dd_src_kernel(Args a) {
    using namespace frame;
    constexpr int D = (L + 1) * (L + 1);
    constexpr int P = PathSet<L, O3>::P;
    extern __shared__ __align__(16) float smem[];
    load_fit(smem);
    const Team tm = team_of(a);
    if (tm.task >= a.ntasks) return;
    int k0, k1;
    task_range(a.E, tm.task, a.ntasks, k0, k1);
    if (k0 >= k1) return;
    const int C2 = a.C2, T = tm.T;
    float* ybuf = smem + kFitStride + tm.tb * src_team_floats<L, O3>(T);
    float* dbuf = ybuf + kYbufFloats;
    float2* vec = reinterpret_cast<float2*>(ybuf + kTeamFloats) + tm.tl;  // [v][k] at (v * D + k) * T
    auto V = [&](int v, int k) -> float2& { return vec[(v * D + k) * T]; };
    enum { XP = 0, GXP = 1, GP = 2 };  // x', ggx', g' (the g row is copied into the g' slot, then rotated)
    float2* wbuf = vec + 3 * D * T;  // [p] at p * T
    float2* gwbuf = wbuf + P * T;

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
        const bool write_r = a.grad_r && tm.tl == 0;
        if (!ok) {  // an edge of an invalid CSR: nothing, zero per-edge gradients
            if (gwe)
                for (int p = 0; p < P; ++p) gwe[p * C2] = f2_zero();
            if (write_r && tm.slice == 0) a.grad_r[3 * (size_t)e] = a.grad_r[3 * (size_t)e + 1] = a.grad_r[3 * (size_t)e + 2] = 0.f;
            continue;
        }
        const float3 rv = load_r(a.r, e);
        const Frame f = make_frame(rv.x, rv.y, rv.z);
        const float2* xs = a.x + (size_t)row * D * C2 + tm.cp;
        const float2* gxs = a.ggx ? a.ggx + (size_t)row * D * C2 + tm.cp : nullptr;
        const float2* gs = a.g + (size_t)i * D * C2 + tm.cp;
        const float2* wrow = a.w + (size_t)e * P * C2 + tm.cp;
        const float2* gwrow = a.ggw ? a.ggw + (size_t)e * P * C2 + tm.cp : nullptr;
        if (f.degenerate) {
            // no direction: the (l, 0, l) paths, each the identity; grad_r = 0
            static_for<0, L + 1>([&](auto lc) {
                constexpr int l = decltype(lc)::value;
                constexpr int p0 = path_index<L, O3>(l, 0, l);
                const float2 gw0 = gwrow ? __ldg(gwrow + p0 * C2) : f2_zero();
                float2 pw = f2_zero();
#pragma unroll
                for (int m = 0; m < 2 * l + 1; ++m) {
                    const float2 gv = __ldg(gs + (l * l + m) * C2);
                    f2_fma(gx[l * l + m], gw0, gv);
                    if (gxs) f2_fma(pw, __ldg(gxs + (l * l + m) * C2), gv);
                }
                if (gwe) gwe[p0 * C2] = pw;
            });
            if (gwe) {
                static_for<0, P>([&](auto pc) {
                    constexpr int p = decltype(pc)::value;
                    if constexpr (PathSet<L, O3>::path(p).l2 > 0) gwe[p * C2] = f2_zero();
                });
            }
            if (write_r && tm.slice == 0) a.grad_r[3 * (size_t)e] = a.grad_r[3 * (size_t)e + 1] = a.grad_r[3 * (size_t)e + 2] = 0.f;
            continue;
        }
        // this edge's weight rows and g row, in flight while the frame is built
        copy_weight_rows<P>(wbuf, gwbuf, wrow, src_buffers_ggw<L>() ? gwrow : nullptr, C2, T);
#pragma unroll
        for (int k = 0; k < D; ++k) cp_async8(&V(GP, k), gs + k * C2);
        cp_async_commit();
        team_wigner<L>(f, tm.tl, T, tm.tmask, ybuf, dbuf, smem);
        float wx = 0.f, wy = 0.f, vz = 0.f;
        if (a.ggr) {
            const float gx0 = __ldg(a.ggr + 3 * (size_t)e), gy0 = __ldg(a.ggr + 3 * (size_t)e + 1),
                        gz0 = __ldg(a.ggr + 3 * (size_t)e + 2);
            const float vx = (f.R[0] * gx0 + f.R[1] * gy0 + f.R[2] * gz0) * f.inv_rho;
            const float vy = (f.R[3] * gx0 + f.R[4] * gy0 + f.R[5] * gz0) * f.inv_rho;
            vz = (f.R[6] * gx0 + f.R[7] * gy0 + f.R[8] * gz0) * f.inv_rho;
            wx = vy;
            wy = -vx;
        }
        // frame vectors x', ggx', g' (K_w x' and K_w g' are formed block by block where used)
        {
            float2 u[D], v[D], up[D], vp[D];
#pragma unroll
            for (int k = 0; k < D; ++k) {
                u[k] = __ldg(xs + k * C2);
                v[k] = gxs ? __ldg(gxs + k * C2) : f2_zero();
            }
            rotate_all2<L>(f, dbuf, u, v, up, vp);
            cp_async_wait_all();  // this lane's weight rows and g row
#pragma unroll
            for (int k = 0; k < D; ++k) {
                V(XP, k) = up[k];
                V(GXP, k) = vp[k];
                u[k] = V(GP, k);
            }
            rotate_all<L>(f, dbuf, u, v);
#pragma unroll
            for (int k = 0; k < D; ++k) V(GP, k) = v[k];
        }
        float2 c0 = f2_zero(), c1 = f2_zero(), c2 = f2_zero();
        // (1) blocks l1: z = M^T g', zt = M^T K_w g', z2 = M(gg_w)^T g'; grad_x; the x-side forms
        static_for<0, L + 1>([&](auto l1c) {
            constexpr int l1 = decltype(l1c)::value;
            constexpr int d1 = 2 * l1 + 1;
            float2 z[d1], zt[d1], z2[d1], gp3[7], gt3[7];
#pragma unroll
            for (int m = 0; m < d1; ++m) z[m] = zt[m] = z2[m] = f2_zero();
            static_for<0, L + 1>([&](auto l3c) {
                constexpr int l3 = decltype(l3c)::value;
                if constexpr (has_type<L, O3>(l1, l3, 0) || has_type<L, O3>(l1, l3, 1)) {
#pragma unroll
                    for (int m = 0; m < 2 * l3 + 1; ++m) gp3[m] = V(GP, l3 * l3 + m);
                    gen_apply<l3>(wx, wy, gp3, gt3);
                    float2 We[4], Wo[4];
                    group_weights<L, O3, l1, l3>(wbuf, T, We, Wo);
                    apply_MT<L, O3, l1, l3>(We, Wo, gp3, z);
                    apply_MT<L, O3, l1, l3>(We, Wo, gt3, zt);
                    if (gwrow) {
                        if constexpr (src_buffers_ggw<L>())
                            group_weights<L, O3, l1, l3>(gwbuf, T, We, Wo);
                        else
                            group_weights_g<L, O3, l1, l3>(gwrow, C2, We, Wo);
                        apply_MT<L, O3, l1, l3>(We, Wo, gp3, z2);
                    }
                }
            });
            float2 kz[d1], zz[d1], xp1[d1], gxp1[d1];
            gen_apply<l1>(wx, wy, z, kz);
#pragma unroll
            for (int m = 0; m < d1; ++m) {
                zz[m] = f2_sub(zt[m], kz[m]);
                xp1[m] = V(XP, l1 * l1 + m);
                gxp1[m] = V(GXP, l1 * l1 + m);
            }
            float2 t0[d1], t1[d1], sgx[d1];
#pragma unroll
            for (int m = 0; m < d1; ++m) {
                t0[m] = f2_sub(f2_sub(f2_scale(vz, z[m]), z2[m]), zz[m]);  // v'_z z - z2 - zz
                t1[m] = f2_sub(f2_add(z2[m], zz[m]), f2_scale(vz, z[m]));  // z2 + zz - v'_z z
                sgx[m] = f2_add(z2[m], zz[m]);
            }
            c0 = f2_add(c0, f2_sub(gform<l1, 1>(xp1, t0), gform<l1, 1>(gxp1, z)));
            c1 = f2_add(c1, f2_add(gform<l1, 0>(gxp1, z), gform<l1, 0>(xp1, t1)));
            c2 = f2_sub(c2, f2_add(f2_scale(wx, gform<l1, 0>(xp1, z)), f2_scale(wy, gform<l1, 1>(xp1, z))));
            rotate<l1, true, true>(f, dbuf, sgx, gx + l1 * l1);
        });
        // (2) blocks l3: y = M x', yt = M K_w x', y56 = M ggx' + M(gg_w) x'; grad_w; the g-side forms
        static_for<0, L + 1>([&](auto l3c) {
            constexpr int l3 = decltype(l3c)::value;
            constexpr int d3 = 2 * l3 + 1;
            float2 y[d3], yt[d3], y56[d3], gp3[d3], gt3[d3];
#pragma unroll
            for (int m = 0; m < d3; ++m) {
                y[m] = yt[m] = y56[m] = f2_zero();
                gp3[m] = V(GP, l3 * l3 + m);
            }
            gen_apply<l3>(wx, wy, gp3, gt3);
            static_for<0, L + 1>([&](auto l1c) {
                constexpr int l1 = decltype(l1c)::value;
                if constexpr (has_type<L, O3>(l1, l3, 0) || has_type<L, O3>(l1, l3, 1)) {
                    constexpr int d1 = 2 * l1 + 1;
                    float2 xp1[d1], xt1[d1], gxp1[d1];
#pragma unroll
                    for (int m = 0; m < d1; ++m) {
                        xp1[m] = V(XP, l1 * l1 + m);
                        gxp1[m] = V(GXP, l1 * l1 + m);
                    }
                    gen_apply<l1>(wx, wy, xp1, xt1);
                    float2 We[4], Wo[4];
                    group_weights<L, O3, l1, l3>(wbuf, T, We, Wo);
                    apply_M<L, O3, l1, l3>(We, Wo, xp1, y);
                    apply_M<L, O3, l1, l3>(We, Wo, xt1, yt);
                    apply_M<L, O3, l1, l3>(We, Wo, gxp1, y56);
                    if (gwrow) {
                        if constexpr (src_buffers_ggw<L>())
                            group_weights<L, O3, l1, l3>(gwbuf, T, We, Wo);
                        else
                            group_weights_g<L, O3, l1, l3>(gwrow, C2, We, Wo);
                        apply_M<L, O3, l1, l3>(We, Wo, xp1, y56);
                    }
                    if (gwe) {
                        float2 Pe[4], Po[4];
#pragma unroll
                        for (int m = 0; m < 4; ++m) Pe[m] = Po[m] = f2_zero();
                        add_products<l1, l3>(gp3, gxp1, Pe, Po);
                        add_products<l1, l3>(gp3, xt1, Pe, Po);
                        add_products<l1, l3>(gt3, xp1, Pe, Po);
                        static_for<0, L + 1>([&](auto l2c) {
                            constexpr int l2 = decltype(l2c)::value;
                            if constexpr (PathSet<L, O3>::allowed(l1, l2, l3)) {
                                constexpr int p = path_index<L, O3>(l1, l2, l3);
                                constexpr bool odd = (l1 + l2 + l3) % 2 == 1;
                                float2 gw = f2_zero();
                                static_for<0, cmin(l1, l3) + 1>([&](auto mc) {
                                    constexpr int mu = decltype(mc)::value;
                                    constexpr float b = (float)etp_gen::kFrameB[l1][l2][l3][mu];
                                    if constexpr (b != 0.f) f2_fma(gw, b, odd ? Po[mu] : Pe[mu]);
                                });
                                gwe[p * C2] = gw;
                            }
                        });
                    }
                }
            });
            float2 ky[d3], s0[d3], s1[d3];
            gen_apply<l3>(wx, wy, y, ky);
#pragma unroll
            for (int m = 0; m < d3; ++m) {
                const float2 yy = f2_sub(yt[m], ky[m]);
                s0[m] = f2_sub(f2_sub(f2_scale(vz, y[m]), y56[m]), yy);  // v'_z y - y5 - y6 - yy
                s1[m] = f2_sub(f2_add(y56[m], yy), f2_scale(vz, y[m]));  // y5 + y6 + yy - v'_z y
            }
            c0 = f2_add(c0, gform<l3, 1>(gp3, s0));
            c1 = f2_add(c1, gform<l3, 0>(gp3, s1));
            c2 = f2_sub(c2, f2_add(f2_scale(wx, gform<l3, 0>(gp3, y)), f2_scale(wy, gform<l3, 1>(gp3, y))));
        });
        if (a.grad_r) {
            float s0 = c0.x + c0.y, s1 = c1.x + c1.y, s2 = c2.x + c2.y;
            for (int o = 1; o < T; o <<= 1) {
                s0 += __shfl_xor_sync(tm.tmask, s0, o);
                s1 += __shfl_xor_sync(tm.tmask, s1, o);
                s2 += __shfl_xor_sync(tm.tmask, s2, o);
            }
            if (tm.tl == 0) {
                s0 *= f.inv_rho, s1 *= f.inv_rho, s2 *= f.inv_rho;
                float* gr = a.grad_r + 3 * (size_t)e;
                const float g0 = f.R[0] * s0 + f.R[3] * s1 + f.R[6] * s2;
                const float g1 = f.R[1] * s0 + f.R[4] * s1 + f.R[7] * s2;
                const float g2 = f.R[2] * s0 + f.R[5] * s1 + f.R[8] * s2;
                if (tm.S == 1) {
                    gr[0] = g0, gr[1] = g1, gr[2] = g2;
                } else {  // the slices' parts onto the zeroed output
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
size_t smem_for(bool src_side, int T) {
    const int teams = kThreads / T;
    return sizeof(float) *
           (size_t)(frame::kFitStride + teams * (src_side ? src_team_floats<L, O3>(T) : dst_team_floats<L, O3>(T)));
}

}  // namespace dd

// ---------------------------------------------------------------------------
// host side
namespace {

// Tasks of the destination-side (src_side false) or source-side kernel: one wave,
// at least 16 edges each, no more tasks than rows (as in the first-order kernels).
template <int L, bool O3>
int dd_tasks(int C, int N, int E, bool src_side) {
    const int T = C / 2 < 32 ? C / 2 : 32, slices = C / (2 * T);
    const size_t sm = dd::smem_for<L, O3>(src_side, T);
    const void* k = src_side ? (const void*)dd::etp_dd_src_kernel<L, O3> : (const void*)dd::etp_dd_dst_kernel<L, O3>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    int dev = 0, sms = 1, bps = 1;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
                                                   cudaSuccess || sms < 1)
        sms = 1;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&bps, k, dd::kThreads, sm) != cudaSuccess || bps < 1) bps = 1;
    const long long cap = (long long)sms * bps * (dd::kThreads / T) / slices;
    long long want = ((long long)E + 15) / 16;
    if (want > N) want = N;
    const long long nt = want < cap ? want : cap;
    return (int)(nt < 1 ? 1 : nt);
}

template <int L, bool O3>
cudaError_t launch_dd(dd::Args a, size_t part_bytes, cudaStream_t s) {
    const int T = a.team, C = 2 * a.C2, D = (L + 1) * (L + 1);
    const int teams_per_block = dd::kThreads / T;
    cudaError_t err;
    void* args[] = {&a};
    for (int side = 0; side < 2; ++side) {
        float2* rows = side ? a.grad_x : a.grad_g;
        if (side ? !(a.grad_x || a.grad_w || a.grad_r) : !a.grad_g) continue;
        a.ntasks = dd_tasks<L, O3>(C, a.N, a.E, side != 0);
        if (rows && part_bytes < partial_rows_bytes(a.ntasks, D, C)) return cudaErrorInvalidValue;
        const size_t sm = dd::smem_for<L, O3>(side != 0, T);
        const void* k = side ? (const void*)dd::etp_dd_src_kernel<L, O3> : (const void*)dd::etp_dd_dst_kernel<L, O3>;
        if ((err = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm)) != cudaSuccess)
            return err;
        const long long teams = (long long)a.ntasks * a.slices;
        const unsigned blocks = (unsigned)((teams + teams_per_block - 1) / teams_per_block);
        if ((err = cudaLaunchKernel(k, dim3(blocks), dim3(dd::kThreads), args, sm, s)) != cudaSuccess) return err;
        if (rows &&
            (err = launch_combine_rows(side ? a.rev_ptr : a.row_ptr, nullptr, a.N, a.E, a.ntasks, D * C / 4,
                                       reinterpret_cast<const float4*>(a.part), reinterpret_cast<float4*>(rows), s)) !=
                cudaSuccess)
            return err;
    }
    return cudaSuccess;
}

}  // namespace

cudaError_t double_backward(int L, bool o3, int C, int N, int E, const int32_t* row_ptr, const int32_t* src,
                            const int32_t* rev_ptr, const int32_t* rev_perm, const int32_t* dst, const float* r,
                            const float* x, const float* w, const float* g, const float* gg_x, const float* gg_w,
                            const float* gg_r, float* grad_g, float* grad_x, float* grad_w, float* grad_r,
                            void* part, size_t part_bytes, cudaStream_t s) {
    const int D = (L + 1) * (L + 1);
    cudaError_t err;
    const int team = C / 2 < 32 ? C / 2 : 32, slices = C / (2 * team);
    // with two channel slices, grad_r is the sum of the slices' two terms (added onto zero: order-free)
    if (grad_r && slices > 1 && (err = cudaMemsetAsync(grad_r, 0, sizeof(float) * 3 * (size_t)E, s)) != cudaSuccess)
        return err;
    if (E == 0) {
        if (grad_g && (err = cudaMemsetAsync(grad_g, 0, sizeof(float) * (size_t)N * D * C, s)) != cudaSuccess)
            return err;
        if (grad_x && (err = cudaMemsetAsync(grad_x, 0, sizeof(float) * (size_t)N * D * C, s)) != cudaSuccess)
            return err;
        return cudaSuccess;
    }
    dd::Args a{N,
               E,
               row_ptr,
               src,
               rev_ptr,
               rev_perm,
               dst,
               r,
               reinterpret_cast<const float2*>(x),
               reinterpret_cast<const float2*>(w),
               reinterpret_cast<const float2*>(g),
               reinterpret_cast<const float2*>(gg_x),
               reinterpret_cast<const float2*>(gg_w),
               gg_r,
               reinterpret_cast<float2*>(grad_g),
               reinterpret_cast<float2*>(grad_x),
               reinterpret_cast<float2*>(grad_w),
               grad_r,
               C / 2,
               team,
               slices,
               1,
               static_cast<float2*>(part)};
    switch (L * 2 + (o3 ? 1 : 0)) {
        case 0: return launch_dd<0, false>(a, part_bytes, s);
        case 1: return launch_dd<0, true>(a, part_bytes, s);
        case 2: return launch_dd<1, false>(a, part_bytes, s);
        case 3: return launch_dd<1, true>(a, part_bytes, s);
        case 4: return launch_dd<2, false>(a, part_bytes, s);
        case 5: return launch_dd<2, true>(a, part_bytes, s);
        case 6: return launch_dd<3, false>(a, part_bytes, s);
        default: return launch_dd<3, true>(a, part_bytes, s);
    }
}

size_t double_backward_partial_bytes(int L, bool o3, int C, int N, int E) {
    if (E <= 0 || N <= 0) return 0;
    int nd = 1, ns = 1;
    switch (L * 2 + (o3 ? 1 : 0)) {
        case 0: nd = dd_tasks<0, false>(C, N, E, false), ns = dd_tasks<0, false>(C, N, E, true); break;
        case 1: nd = dd_tasks<0, true>(C, N, E, false), ns = dd_tasks<0, true>(C, N, E, true); break;
        case 2: nd = dd_tasks<1, false>(C, N, E, false), ns = dd_tasks<1, false>(C, N, E, true); break;
        case 3: nd = dd_tasks<1, true>(C, N, E, false), ns = dd_tasks<1, true>(C, N, E, true); break;
        case 4: nd = dd_tasks<2, false>(C, N, E, false), ns = dd_tasks<2, false>(C, N, E, true); break;
        case 5: nd = dd_tasks<2, true>(C, N, E, false), ns = dd_tasks<2, true>(C, N, E, true); break;
        case 6: nd = dd_tasks<3, false>(C, N, E, false), ns = dd_tasks<3, false>(C, N, E, true); break;
        default: nd = dd_tasks<3, true>(C, N, E, false), ns = dd_tasks<3, true>(C, N, E, true); break;
    }
    return partial_rows_bytes(nd > ns ? nd : ns, (L + 1) * (L + 1), C);
}

}  // namespace etp
