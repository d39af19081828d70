// Forward and backward kernels of the edge tensor product, evaluated in the
// edge-aligned frame.
//
// Identity used (exact in exact arithmetic, from the equivariance of every
// coupling): for an edge with unit vector u and a rotation R with R u = z,
//     CG_p(x, Y(u)) = D_l3(R)^T B_p D_l1(R) x,
// where D_l(R) is the Wigner matrix of the real harmonics (Y_l(R r) = D_l Y_l(r))
// and B_p[m3, m1] = sqrt(2 l2 + 1) CG_p[m1, 0, m3] is a compile-time constant that
// is nonzero only at m1 = +-m3 (111 entries for L = 3 against 611 in CG_p). So per
// edge and channel the message is: rotate x_src into the frame, apply the
// weighted sparse B's, rotate back. The derivative with respect to the edge
// direction follows from the rotation generators J_a (a = x, y in the frame):
//     dL/de_a = -(J_a g')^T (M x') - (M^T g')^T (J_a x'),   M = sum_p w_p B_p,
// and grad_r = R^T (dL/de_y, -dL/de_x, 0) / |r|.
//
// Passages: "High-performance training and inference for deep equivariant
// interatomic potentials", section "제안 방법" (fused tensor-product kernel,
// sparse 3-j coefficients, no materialised intermediates); "Scaling the leading
// accuracy of deep equivariant models to biomolecular simulations of realistic
// size", section "提出的方法" (the tensor product as a single contraction);
// "FlashCart 如何让等变原子间势更快更准?", section "FlashCart 用笛卡尔内核替代球谐耦合"
// (the speed comes from memory access and the aggregation of edge contributions).
// The frame rotation itself is not described on the pages; it gives the same
// result as the plain sparse contraction and is this library's choice.
//
// Work decomposition: a task is an equal contiguous range of edges (CSR order
// forward, reverse-CSR order backward), whatever the degree distribution. A team
// of T = min(32, C/2) lanes handles a slice of 2T channels of the task's edges
// (lane t holds channels 2(sT + t), 2(sT + t) + 1 as a float2); with C = 128 a
// task has two slices, the two warps of one block. Node sums accumulate in
// registers and are stored once per row; a row cut by a task boundary leaves one
// partial row per task, which a second launch sums in task order (no atomics).
// Per edge, one lane
// bulk-copies the next edge's weights (and frame record, and in the forward the
// source row) into the other of two shared-memory buffers; each team expands its
// edge's Wigner matrices into shared memory, from the record or built from r.
#pragma once

#include "etp_device.cuh"
#include "etp.h"
#include "etp_internal.h"

namespace etp {

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

namespace frame {

constexpr int kThreads = kThreadsPerBlock;  // 2 warps
constexpr int kYbufFloats = 7 * 12;         // harmonics l = 2, 3 at the 7 fitting points
constexpr int kDbufFloats = 192;            // D_2 (5 rows) then D_3 (7 rows), rows of 8 duplicated pairs
constexpr int kTeamFloats = kYbufFloats + kDbufFloats;
constexpr int kFitFloats = 24 + 2 * 49;     // points (padded) + A_2^-1, A_3^-1 (7 x 7 each)
constexpr int kFitStride = 128;             // shared-memory floats reserved for the fit table
// Team buffers are read with 16-byte vector loads: every offset must keep 16-byte alignment.
static_assert(kFitStride >= kFitFloats && kFitStride % 4 == 0, "fit table stride");
static_assert(kYbufFloats % 4 == 0 && kTeamFloats % 4 == 0, "team buffer alignment");
constexpr int kHeaderFloats = kFitStride + 8;  // fit table, then the grad_r slice partials
static_assert(kHeaderFloats % 4 == 0, "header alignment");
// Shared memory of one task group (the S teams of a task): 32 floats of
// mbarriers, then two edge-weight buffers of P*C floats and `rows` node-row
// buffers of D*C floats (all 16-byte aligned: P*C and D*C are multiples of 4).
constexpr int kBarFloats = 32;
// Edge frame record (floats): D_2 row-major [0, 25), D_3 row-major [25, 74), R
// row-major [76, 85), 1/|r| at 85, the zero-length flag (1 or 0) at 86. With
// frames given, a group also holds two records, one per weight buffer.
constexpr int kFrameFloats = 88;
constexpr int kFrameD3 = 25, kFrameR = 76, kFrameInvRho = 85, kFrameDegen = 86;
static_assert(kFrameFloats % 4 == 0 && kFrameR % 4 == 0, "frame record alignment");
static_assert(kFrameFloats == ETP_FRAME_FLOATS, "etp.h states the record size");
constexpr int group_floats(int P, int D, int C, int rows, bool framed) {
    return kBarFloats + 2 * P * C + rows * D * C + (framed ? 2 * kFrameFloats : 0);
}
// The backward's per-team buffers add this lane-owned x and grad_out rows (D x T float2 each).
constexpr int bwd_team_floats(int D, int T) { return kTeamFloats + 2 * D * T * 2; }

// ---------------------------------------------------------------------------
// compile-time tables
template <int L, bool O3>
constexpr int path_index(int l1, int l2, int l3) {
    int n = 0;
    for (int a = 0; a <= L; ++a)
        for (int b = 0; b <= L; ++b)
            for (int c = 0; c <= L; ++c)
                if (PathSet<L, O3>::allowed(a, b, c)) {
                    if (a == l1 && b == l2 && c == l3) return n;
                    ++n;
                }
    return -1;
}
constexpr int cmin(int a, int b) { return a < b ? a : b; }
// does (l1, *, l3) have an allowed path with l1 + l2 + l3 of the given parity?
template <int L, bool O3>
constexpr bool has_type(int l1, int l3, int odd) {
    for (int b = 0; b <= L; ++b)
        if (PathSet<L, O3>::allowed(l1, b, l3) && (l1 + b + l3) % 2 == odd) return true;
    return false;
}

// Two channels per lane: packed fp32x2 arithmetic (one instruction for both
// channels, each half rounded exactly as fmaf / fadd / fmul).
__device__ __forceinline__ float2 f2_dup(float s) { return make_float2(s, s); }
// scalar (usually a compile-time constant, kept as an immediate) times a pair
__device__ __forceinline__ void f2_fma(float2& acc, float s, float2 v) {
    acc.x = fmaf(s, v.x, acc.x);
    acc.y = fmaf(s, v.y, acc.y);
}
__device__ __forceinline__ void f2_fma(float2& acc, float2 a, float2 b) { acc = __ffma2_rn(a, b, acc); }
__device__ __forceinline__ void f2_fms(float2& acc, float2 a, float2 b) {  // acc -= a * b
    acc.x = fmaf(-a.x, b.x, acc.x);
    acc.y = fmaf(-a.y, b.y, acc.y);
}
__device__ __forceinline__ float2 f2_mul(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 f2_add(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 f2_zero() { return make_float2(0.f, 0.f); }

// Shared-memory read that the compiler must issue where it stands: the Wigner
// entries are re-read at each use instead of being kept live in registers.
__device__ __forceinline__ float lds(const float* p) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"((unsigned)__cvta_generic_to_shared(p)));
    return v;
}
__device__ __forceinline__ float4 lds4(const float* p) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"((unsigned)__cvta_generic_to_shared(p)));
    return v;
}

__device__ __forceinline__ void st_stream2(float2* p, float2 v, uint64_t pol) {
    asm volatile("st.global.L2::cache_hint.v2.f32 [%0], {%1, %2}, %3;" ::"l"(p), "f"(v.x), "f"(v.y), "l"(pol)
                 : "memory");
}

// ---------------------------------------------------------------------------
// The edge frame: R (rows e1, e2, u) with R u = z, from the orthonormal basis of
// Duff, Burgess, Christensen, Hery, Kensler, Liani, Villemin, "Building an
// Orthonormal Basis, Revisited" (JCGT 2017); (e1, e2, u) is right-handed, so R
// is a proper rotation. An edge shorter than 1e-12 has no direction: it gets
// u = z (R = I) and `degenerate` set (its harmonics are Y_0 = 1 only).
struct Frame {
    float R[9];
    float inv_rho;
    bool degenerate;
};

__device__ __forceinline__ float3 load_r(const float* r, int e) {
    return make_float3(__ldg(r + 3 * (size_t)e), __ldg(r + 3 * (size_t)e + 1), __ldg(r + 3 * (size_t)e + 2));
}

__device__ __forceinline__ Frame make_frame(float rx, float ry, float rz) {
    Frame f;
    const float n2 = rx * rx + ry * ry + rz * rz;
    f.degenerate = !(n2 >= 1e-24f);
    const float inv = f.degenerate ? 0.f : rsqrtf(n2);
    const float x = f.degenerate ? 0.f : rx * inv, y = f.degenerate ? 0.f : ry * inv;
    const float z = f.degenerate ? 1.f : rz * inv;
    const float s = copysignf(1.f, z);
    const float a = -__frcp_rn(s + z);
    const float b = x * y * a;
    f.R[0] = 1.f + s * x * x * a;
    f.R[1] = s * b;
    f.R[2] = -s * x;
    f.R[3] = b;
    f.R[4] = s + y * y * a;
    f.R[5] = -y;
    f.R[6] = x;
    f.R[7] = y;
    f.R[8] = z;
    f.inv_rho = inv;
    return f;
}

// D_1(R) in the (y, z, x) component order of the l = 1 harmonics.
__device__ __forceinline__ float d1(const Frame& f, int a, int b) {
    const int pa = a == 0 ? 1 : (a == 1 ? 2 : 0), pb = b == 0 ? 1 : (b == 1 ? 2 : 0);
    return f.R[pa * 3 + pb];
}

// Wigner matrices D_2, D_3 of the frame into the team's shared buffer: harmonics
// at the rotated fitting points R p_k, then D_l = [Y_l(R p_k)]_k A_l^-1.
template <int L>
__device__ __forceinline__ void team_wigner(const Frame& f, int tl, int T, unsigned tmask, float* __restrict__ ybuf,
                                            float* __restrict__ dbuf, const float* __restrict__ fit) {
    if constexpr (L >= 2) {
        constexpr int NP = 2 * L + 1;  // points needed
        __syncwarp(tmask);             // the previous edge's readers are done
        for (int k = tl; k < NP; k += T) {
            const float px = fit[3 * k], py = fit[3 * k + 1], pz = fit[3 * k + 2];
            const float qx = f.R[0] * px + f.R[1] * py + f.R[2] * pz;
            const float qy = f.R[3] * px + f.R[4] * py + f.R[5] * pz;
            const float qz = f.R[6] * px + f.R[7] * py + f.R[8] * pz;
            float Y[(L + 1) * (L + 1)];
            sh_unit<L, float>(qx, qy, qz, Y);
#pragma unroll
            for (int c = 4; c < (L + 1) * (L + 1); ++c) ybuf[k * 12 + (c - 4)] = Y[c];
        }
        __syncwarp(tmask);
        const float* inv2 = fit + 24;
        const float* inv3 = fit + 24 + 49;
        for (int idx = tl; idx < 25; idx += T) {
            const int a = idx / 5, b = idx - 5 * (idx / 5);
            float v = 0.f;
#pragma unroll
            for (int k = 0; k < 5; ++k) v = fmaf(ybuf[k * 12 + a], inv2[k * 7 + b], v);
            reinterpret_cast<float2*>(dbuf + a * 16)[b] = make_float2(v, v);
        }
        if constexpr (L >= 3) {
            for (int idx = tl; idx < 49; idx += T) {
                const int a = idx / 7, b = idx - 7 * (idx / 7);
                float v = 0.f;
#pragma unroll
                for (int k = 0; k < 7; ++k) v = fmaf(ybuf[k * 12 + 5 + a], inv3[k * 7 + b], v);
                reinterpret_cast<float2*>(dbuf + 80 + a * 16)[b] = make_float2(v, v);
            }
        }
        __syncwarp(tmask);
    }
}

// out = D_l in  (TRANS = false)   or   out (+)= D_l^T in  (TRANS = true, ACC adds)
// D_2, D_3 rows are 16 floats apart in the team buffer (8 duplicated pairs),
// read as float4 = two pairs.
template <int l, bool TRANS, bool ACC>
__device__ __forceinline__ void rotate(const Frame& f, const float* __restrict__ dbuf, const float2* in, float2* out) {
    constexpr int d = 2 * l + 1;
    float2 tmp[d];
#pragma unroll
    for (int a = 0; a < d; ++a) tmp[a] = f2_zero();
    if constexpr (l == 0) {
        tmp[0] = in[0];
    } else {
#pragma unroll
        for (int a = 0; a < d; ++a) {
            float2 row[8];
            if constexpr (l == 1) {
#pragma unroll
                for (int b = 0; b < d; ++b) row[b] = f2_dup(d1(f, a, b));
            } else {
                const float* base = dbuf + (l == 2 ? 0 : 80) + a * 16;
#pragma unroll
                for (int h = 0; h < (d + 1) / 2; ++h) {
                    const float4 q = lds4(base + 4 * h);
                    row[2 * h] = make_float2(q.x, q.y);
                    row[2 * h + 1] = make_float2(q.z, q.w);
                }
            }
#pragma unroll
            for (int b = 0; b < d; ++b) {
                if constexpr (TRANS)
                    tmp[b] = __ffma2_rn(row[b], in[a], tmp[b]);
                else
                    tmp[a] = __ffma2_rn(row[b], in[b], tmp[a]);
            }
        }
    }
#pragma unroll
    for (int a = 0; a < d; ++a) {
        if constexpr (ACC)
            out[a] = f2_add(out[a], tmp[a]);
        else
            out[a] = tmp[a];
    }
}

// Two vectors rotated by the same D_l (each row loaded once, two FMA streams).
template <int l>
__device__ __forceinline__ void rotate2(const Frame& f, const float* __restrict__ dbuf, const float2* in1,
                                        const float2* in2, float2* out1, float2* out2) {
    constexpr int d = 2 * l + 1;
    if constexpr (l == 0) {
        out1[0] = in1[0];
        out2[0] = in2[0];
    } else {
#pragma unroll
        for (int a = 0; a < d; ++a) {
            float2 row[8];
            if constexpr (l == 1) {
#pragma unroll
                for (int b = 0; b < d; ++b) row[b] = f2_dup(d1(f, a, b));
            } else {
                const float* base = dbuf + (l == 2 ? 0 : 80) + a * 16;
#pragma unroll
                for (int h = 0; h < (d + 1) / 2; ++h) {
                    const float4 q = lds4(base + 4 * h);
                    row[2 * h] = make_float2(q.x, q.y);
                    row[2 * h + 1] = make_float2(q.z, q.w);
                }
            }
            float2 t1 = f2_zero(), t2 = f2_zero();
#pragma unroll
            for (int b = 0; b < d; ++b) {
                t1 = __ffma2_rn(row[b], in1[b], t1);
                t2 = __ffma2_rn(row[b], in2[b], t2);
            }
            out1[a] = t1;
            out2[a] = t2;
        }
    }
}
template <int L>
__device__ __forceinline__ void rotate_all2(const Frame& f, const float* dbuf, const float2* in1, const float2* in2,
                                            float2* out1, float2* out2) {
    static_for<0, L + 1>([&](auto lc) {
        constexpr int l = decltype(lc)::value;
        rotate2<l>(f, dbuf, in1 + l * l, in2 + l * l, out1 + l * l, out2 + l * l);
    });
}

// Rotate every l block of a [D] float2 vector into the frame.
template <int L>
__device__ __forceinline__ void rotate_all(const Frame& f, const float* dbuf, const float2* in, float2* out) {
    static_for<0, L + 1>([&](auto lc) {
        constexpr int l = decltype(lc)::value;
        rotate<l, false, false>(f, dbuf, in + l * l, out + l * l);
    });
}

// ---------------------------------------------------------------------------
// Streaming of the per-edge weights and node rows with the bulk-copy (TMA) engine:
// one producer lane per task group issues cp.async.bulk copies of whole rows
// (an edge's weights are P*C contiguous floats, a node row D*C) into shared
// memory, completing on an mbarrier by transaction count; consumers wait on the
// barrier's phase. Every wait is bounded: on time-out the kernel raises a fault
// flag and carries on with whatever the buffer holds (stays in bounds, finishes).
__device__ __forceinline__ unsigned smem_u32(const void* p) { return (unsigned)__cvta_generic_to_shared(p); }
__device__ __forceinline__ float2 lds2(const float2* p) {
    float2 v;
    asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(smem_u32(p)));
    return v;
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_fence_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, unsigned bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}
// 16-byte-aligned addresses, bytes a multiple of 16
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, unsigned bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}
// The same with an L2 evict-first hint: for the edge weights, read once per pass,
// so that they do not push the node rows (read by many edges) out of L2.
__device__ __forceinline__ void bulk_g2s_stream(void* dst, const void* src, unsigned bytes, uint64_t* bar,
                                                uint64_t pol) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(pol)
        : "memory");
}
// Per-lane 8-byte asynchronous copies (the backward's node rows: each lane copies
// and later reads only its own channels, so no cross-lane synchronisation).
__device__ __forceinline__ void cp_async8(void* smem, const void* gmem) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(smem_u32(smem)), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

constexpr int kWaitLimit = 1 << 20;  // polls of mbarrier.try_wait before giving up
__device__ int g_fault;              // set when a bounded wait ran out (never expected)
// Wait for a phase of `bar`; `live` turns false (and the flag is raised) when the
// bound runs out, after which the caller's later waits return at once.
__device__ __forceinline__ void mbar_wait(uint64_t* bar, unsigned parity, bool& live) {
    if (!live) return;
    for (int i = 0; i < kWaitLimit; ++i) {
        unsigned done;
        asm volatile(
            "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
            : "=r"(done)
            : "r"(smem_u32(bar)), "r"(parity)
            : "memory");
        if (done) return;
    }
    live = false;
    atomicOr(&g_fault, 1);
}

// Combined frame weights of the (l1, l3) group for this lane's channels:
// We[mu] = sum over even paths (l1, l2, l3) of b_p(mu) w_p, Wo[mu] likewise for
// odd paths. `wrow` is the edge's weight row in shared memory as float2, offset
// to this lane's channel pair.
template <int L, bool O3, int l1, int l3>
__device__ __forceinline__ void group_weights(const float2* wrow, int C2, float2 (&We)[4], float2 (&Wo)[4]) {
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        We[m] = f2_zero();
        Wo[m] = f2_zero();
    }
    static_for<0, L + 1>([&](auto l2c) {
        constexpr int l2 = decltype(l2c)::value;
        if constexpr (PathSet<L, O3>::allowed(l1, l2, l3)) {
            constexpr int p = path_index<L, O3>(l1, l2, l3);
            const float2 w = lds2(wrow + p * C2);
            constexpr bool odd = (l1 + l2 + l3) % 2 == 1;
            static_for<0, cmin(l1, l3) + 1>([&](auto mc) {
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

// y[l3] += M_{l3 l1} x'[l1]
template <int L, bool O3, int l1, int l3>
__device__ __forceinline__ void apply_M(const float2 (&We)[4], const float2 (&Wo)[4], const float2* xp, float2* y) {
    constexpr int mn = cmin(l1, l3);
    if constexpr (has_type<L, O3>(l1, l3, 0)) {
        static_for<-mn, mn + 1>([&](auto mc) {
            constexpr int m = decltype(mc)::value;
            f2_fma(y[l3 + m], We[m < 0 ? -m : m], xp[l1 + m]);
        });
    }
    if constexpr (has_type<L, O3>(l1, l3, 1)) {
        static_for<1, mn + 1>([&](auto mc) {
            constexpr int mu = decltype(mc)::value;
            f2_fma(y[l3 + mu], Wo[mu], xp[l1 - mu]);
            f2_fms(y[l3 - mu], Wo[mu], xp[l1 + mu]);
        });
    }
}

// z[l1] += M_{l3 l1}^T g'[l3]
template <int L, bool O3, int l1, int l3>
__device__ __forceinline__ void apply_MT(const float2 (&We)[4], const float2 (&Wo)[4], const float2* gp, float2* z) {
    constexpr int mn = cmin(l1, l3);
    if constexpr (has_type<L, O3>(l1, l3, 0)) {
        static_for<-mn, mn + 1>([&](auto mc) {
            constexpr int m = decltype(mc)::value;
            f2_fma(z[l1 + m], We[m < 0 ? -m : m], gp[l3 + m]);
        });
    }
    if constexpr (has_type<L, O3>(l1, l3, 1)) {
        static_for<1, mn + 1>([&](auto mc) {
            constexpr int mu = decltype(mc)::value;
            f2_fma(z[l1 - mu], Wo[mu], gp[l3 + mu]);
            f2_fms(z[l1 + mu], Wo[mu], gp[l3 - mu]);
        });
    }
}

// -(J_a v)^T s for a block of degree l, per channel of the lane:
//   -sum_{m,m'} J[m][m'] v[m'] s[m] = -sum_{m < m'} J[m][m'] (v[m'] s[m] - v[m] s[m'])   (J antisymmetric)
template <int l, int axis>
__device__ __forceinline__ float2 gen_form(const float2* v, const float2* s) {
    float2 acc = f2_zero();
    static_for<0, 2 * l + 1>([&](auto ac) {
        constexpr int a = decltype(ac)::value;
        static_for<a + 1, 2 * l + 1>([&](auto bc) {
            constexpr int b = decltype(bc)::value;
            constexpr float J = (float)etp_gen::kGen[axis][l][a][b];
            if constexpr (J != 0.f) {
                float2 t = f2_mul(v[b], s[a]);
                f2_fms(t, v[a], s[b]);
                f2_fma(acc, -J, t);
            }
        });
    });
    return acc;
}

// ---------------------------------------------------------------------------
// Work decomposition: equal contiguous ranges of edges ("tasks"), one per team
// (or per pair of slice teams when C = 128, the block's two warps). Rows inside a
// range are stored once; rows cut by a range boundary go through the partial-row
// slots (store_row, row_slot, tail_record below).
struct Geometry {
    int T, S, team_in_block, task, slice, tl;
    unsigned tmask;
};

__device__ __forceinline__ Geometry geometry(int team_lanes, int slices) {
    Geometry g;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    g.T = team_lanes;
    g.S = slices;
    g.tl = lane & (team_lanes - 1);
    g.team_in_block = warp * (32 / team_lanes) + lane / team_lanes;
    const int tasks_per_block = (kThreads / team_lanes) / slices;
    g.task = blockIdx.x * tasks_per_block + g.team_in_block / slices;
    g.slice = g.team_in_block % slices;
    const unsigned ones = team_lanes == 32 ? 0xffffffffu : ((1u << team_lanes) - 1u);
    g.tmask = ones << (lane & ~(team_lanes - 1) & 31);
    return g;
}

// [k0, k1): the task's share of n items.
__device__ __forceinline__ void task_range(long long n, int task, int ntasks, int& k0, int& k1) {
    k0 = (int)(n * task / ntasks);
    k1 = (int)(n * (task + 1) / ntasks);
}

// largest i in [0, n) with ptr[i] <= k (ptr nondecreasing, ptr[0] <= k)
__device__ __forceinline__ int segment_of(const int32_t* __restrict__ ptr, int n, int k) {
    int lo = 0, hi = n;
    while (hi - lo > 1) {
        int mid = (lo + hi) >> 1;
        if (__ldg(ptr + mid) <= k)
            lo = mid;
        else
            hi = mid;
    }
    return lo;
}


// One finished row of a task, stored with plain stores: into the output when the
// task holds all of the row's positions, else into the task's slot of the
// partial-row buffer (slot 0: the row began before the task; slot 1: it goes on
// past it). etp_combine_rows_kernel then sums each cut row's pieces in task order.
template <int D>
__device__ __forceinline__ void store_row(float2* dst, int C2, const float2 (&acc)[D]) {
#pragma unroll
    for (int k = 0; k < D; ++k) dst[k * C2] = acc[k];
}

// The task's record after the partial rows: its last row (rank) when that row
// goes on past the task and begins in it, else -1 (one lane per task writes it).
__device__ __forceinline__ void tail_record(float2* part, int ntasks, int DC2, int task, int row, int lo, int hi,
                                            int k0, int k1) {
    int32_t* rec = reinterpret_cast<int32_t*>(part + (size_t)ntasks * 2 * DC2);
    rec[task] = (hi > k1 && lo >= k0) ? row : -1;
}

// Where a task's finished row [lo, hi) of positions goes (this lane's channel
// pair): the output row, or the task's partial slot.
__device__ __forceinline__ float2* row_slot(float2* rows, float2* part, int node, int lo, int hi, int k0, int k1,
                                            int task, int DC2, int cp) {
    if (lo >= k0 && hi <= k1) return rows + (size_t)node * DC2 + cp;
    return part + ((size_t)task * 2 + (lo < k0 ? 0 : 1)) * DC2 + cp;
}

// The fitting points and inverses as one constant-memory table, built at
// compile time from the generated constants: points (21, padded to 24), then
// A_2^-1 and A_3^-1 (7 x 7 each).
struct FitTable {
    float v[kFitFloats];
};
constexpr FitTable make_fit_table() {
    FitTable t{};
    for (int k = 0; k < kFitFloats; ++k) {
        float v = 0.f;
        if (k < 21)
            v = (float)etp_gen::kFitPoints[k / 3][k % 3];
        else if (k >= 24 && k < 24 + 49)
            v = (float)etp_gen::kFitInv[2][(k - 24) / 7][(k - 24) % 7];
        else if (k >= 24 + 49)
            v = (float)etp_gen::kFitInv[3][(k - 73) / 7][(k - 73) % 7];
        t.v[k] = v;
    }
    return t;
}
static __constant__ FitTable c_fit = make_fit_table();

__device__ __forceinline__ void load_fit_tables(float* fit) {
    for (int k = threadIdx.x; k < kFitFloats; k += kThreads) fit[k] = c_fit.v[k];
    __syncthreads();
}

// The frame of an edge read back from its record in shared memory.
__device__ __forceinline__ Frame frame_of(const float* fb) {
    Frame f;
    const float4 q0 = lds4(fb + kFrameR), q1 = lds4(fb + kFrameR + 4), q2 = lds4(fb + kFrameR + 8);
    f.R[0] = q0.x, f.R[1] = q0.y, f.R[2] = q0.z, f.R[3] = q0.w;
    f.R[4] = q1.x, f.R[5] = q1.y, f.R[6] = q1.z, f.R[7] = q1.w;
    f.R[8] = q2.x;
    f.inv_rho = q2.y;
    f.degenerate = q2.z != 0.f;
    return f;
}

// The record's D_2, D_3 copied into the team's rotation buffer as duplicated
// pairs (the layout `rotate` reads).
template <int L>
__device__ __forceinline__ void expand_wigner(const float* fb, int tl, int T, unsigned tmask, float* dbuf) {
    if constexpr (L >= 2) {
        constexpr int n = L >= 3 ? kFrameD3 + 49 : kFrameD3;
        for (int idx = tl; idx < n; idx += T) {
            const float v = lds(fb + idx);
            int off;
            if (idx < kFrameD3) {
                const int a = idx / 5;
                off = a * 16 + 2 * (idx - 5 * a);
            } else {
                const int k = idx - kFrameD3, a = k / 7;
                off = 80 + a * 16 + 2 * (k - 7 * a);
            }
            *reinterpret_cast<float2*>(dbuf + off) = make_float2(v, v);
        }
        __syncwarp(tmask);
    }
}

// ---------------------------------------------------------------------------
// One thread's Wigner matrices D_2 (row-major 5 x 5) and D_3 (7 x 7) of the frame
// f, fitted from the harmonics at the rotated fixed points (zero for a degenerate
// frame, and not computed above L).
template <int L>
__device__ __forceinline__ void thread_wigner(const Frame& f, float (&d2)[25], float (&d3)[49]) {
#pragma unroll
    for (int i = 0; i < 25; ++i) d2[i] = 0.f;
#pragma unroll
    for (int i = 0; i < 49; ++i) d3[i] = 0.f;
    if constexpr (L >= 2) {
        if (!f.degenerate) {
#pragma unroll
            for (int k = 0; k < 2 * L + 1; ++k) {
                const float px = c_fit.v[3 * k], py = c_fit.v[3 * k + 1], pz = c_fit.v[3 * k + 2];
                const float qx = f.R[0] * px + f.R[1] * py + f.R[2] * pz;
                const float qy = f.R[3] * px + f.R[4] * py + f.R[5] * pz;
                const float qz = f.R[6] * px + f.R[7] * py + f.R[8] * pz;
                float Y[(L + 1) * (L + 1)];
                sh_unit<L, float>(qx, qy, qz, Y);
                if (k < 5) {
#pragma unroll
                    for (int a = 0; a < 5; ++a)
#pragma unroll
                        for (int b = 0; b < 5; ++b)
                            d2[a * 5 + b] = fmaf(Y[4 + a], c_fit.v[24 + k * 7 + b], d2[a * 5 + b]);
                }
                if constexpr (L >= 3) {
#pragma unroll
                    for (int a = 0; a < 7; ++a)
#pragma unroll
                        for (int b = 0; b < 7; ++b)
                            d3[a * 7 + b] = fmaf(Y[9 + a], c_fit.v[73 + k * 7 + b], d3[a * 7 + b]);
                }
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Edge frames: one thread per edge builds the edge's record (R, 1/|r|, the
// zero-length flag, and D_2, D_3 of R fitted from the harmonics at the fixed
// points, in the same operation order as the in-kernel build); the block's
// records are staged in shared memory and leave as one contiguous write.
constexpr int kFrameBlock = 128;
template <int L>
__global__ void __launch_bounds__(kFrameBlock) etp_edge_frames_kernel(int E, const float* __restrict__ r,
                                                                       float4* __restrict__ frames) {
    __shared__ __align__(16) float stage[kFrameBlock * kFrameFloats];
    const int e0 = blockIdx.x * kFrameBlock;
    const int e = e0 + threadIdx.x;
    if (e < E) {
        const float3 rv = load_r(r, e);
        const Frame f = make_frame(rv.x, rv.y, rv.z);
        float d2[25], d3[49];
        thread_wigner<L>(f, d2, d3);
        float4* rec = reinterpret_cast<float4*>(stage + threadIdx.x * kFrameFloats);
        float v[kFrameFloats];
#pragma unroll
        for (int i = 0; i < kFrameFloats; ++i) v[i] = 0.f;
#pragma unroll
        for (int i = 0; i < 25; ++i) v[i] = d2[i];
#pragma unroll
        for (int i = 0; i < 49; ++i) v[kFrameD3 + i] = d3[i];
#pragma unroll
        for (int i = 0; i < 9; ++i) v[kFrameR + i] = f.R[i];
        v[kFrameInvRho] = f.inv_rho;
        v[kFrameDegen] = f.degenerate ? 1.f : 0.f;
#pragma unroll
        for (int i = 0; i < kFrameFloats / 4; ++i) rec[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    }
    __syncthreads();
    const int n = min(kFrameBlock, E - e0) * (kFrameFloats / 4);
    float4* dst = frames + (size_t)e0 * (kFrameFloats / 4);
    const float4* st = reinterpret_cast<const float4*>(stage);
    for (int i = threadIdx.x; i < n; i += kFrameBlock) dst[i] = st[i];
}

}  // namespace frame


// ===========================================================================
// Forward: task = a contiguous range of CSR (destination-ordered) edges. Per edge,
// the producer lane bulk-copies the next edge's weight row and source row into
// the other of two buffers while the group computes this edge. C2T is the
// compile-time channel-pair count (0: taken from the arguments). FR: the edges'
// frame records are given (copied with the weights) instead of built here.
template <int L, bool O3, int C2T, bool FR>
__global__ void __launch_bounds__(frame::kThreads, 4) etp_fwd_frame_kernel(FwdArgs a) {
    using namespace frame;
    constexpr int D = (L + 1) * (L + 1);
    constexpr int P = PathSet<L, O3>::P;
    extern __shared__ __align__(16) float smem[];
    if constexpr (!FR) load_fit_tables(smem);
    const Geometry G = geometry(a.team, a.slices);
    if (G.task >= a.ntasks) return;  // the slice teams of a task leave together
    int k0, k1;
    task_range(a.E, G.task, a.ntasks, k0, k1);
    if (k0 >= k1) return;
    const int C2 = C2T ? C2T : a.C4 * 2, C = 2 * C2;
    const int ngroups = (kThreads / G.T) / G.S;
    const int gfloats = group_floats(P, D, C, 2, FR);
    float* gbase = smem + kHeaderFloats + (G.team_in_block / G.S) * gfloats;
    uint64_t* bar = reinterpret_cast<uint64_t*>(gbase);
    float* wbuf = gbase + kBarFloats;
    float* xbuf = wbuf + 2 * P * C;
    float* fbuf = xbuf + 2 * D * C;  // two frame records (FR)
    float* team = smem + kHeaderFloats + ngroups * gfloats + G.team_in_block * kTeamFloats;
    float* ybuf = team;
    float* dbuf = team + kYbufFloats;
    const bool producer = G.slice == 0 && G.tl == 0;
    const int cp = G.slice * G.T + G.tl;
    float2* out2 = reinterpret_cast<float2*>(a.out);
    float2* part2 = reinterpret_cast<float2*>(a.part);
    auto group_sync = [&] {
        if (G.S == 2)
            __syncthreads();  // the block is exactly this task's two warps
        else
            __syncwarp(G.tmask);
    };
    const unsigned wbytes = 4u * P * C, xbytes = 4u * D * C, fbytes = FR ? 4u * kFrameFloats : 0u;
    const uint64_t pol_w = l2_evict_first_policy();
    // position q -> edge, and row rank -> node: the identity, or a locality order
    // (rows taken in the order's sequence, each row's edges contiguous)
    // (an out-of-range edge of the map counts as an edge with an invalid source)
    auto edge_at = [&](int q) -> int { return a.pos_edge ? __ldg(a.pos_edge + q) : q; };
    auto node_of = [&](int rank) -> int { return a.order ? __ldg(a.order + rank) : rank; };
    auto src_of = [&](int e) -> int { return (unsigned)e < (unsigned)a.E ? __ldg(a.src + e) : -1; };
    auto issue = [&](int e, int j, int slot) {
        e = (unsigned)e < (unsigned)a.E ? e : 0;
        j = (unsigned)j < (unsigned)a.N ? j : 0;
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        mbar_expect_tx(&bar[slot], wbytes + xbytes + fbytes);
        bulk_g2s_stream(wbuf + slot * P * C, reinterpret_cast<const float*>(a.w) + (size_t)e * P * C, wbytes, &bar[slot],
                        pol_w);
        bulk_g2s(xbuf + slot * D * C, reinterpret_cast<const float*>(a.x) + (size_t)j * D * C, xbytes, &bar[slot]);
        if constexpr (FR)
            bulk_g2s(fbuf + slot * kFrameFloats, a.frames + (size_t)e * kFrameFloats, fbytes, &bar[slot]);
    };
    if (producer) {
        mbar_init(&bar[0], 1);
        mbar_init(&bar[1], 1);
        mbar_fence_init();
    }
    group_sync();
    // edges one to three positions ahead, source indices one and two ahead and the
    // next edge vector are loaded an edge early, so their latency (and that of the
    // position -> edge map before them) hides behind an edge of compute
    const int e0 = edge_at(k0);
    int e_next = k0 + 1 < k1 ? edge_at(k0 + 1) : 0;
    int e_next2 = k0 + 2 < k1 ? edge_at(k0 + 2) : 0;
    int j_cur = src_of(e0);
    int j_next = k0 + 1 < k1 ? src_of(e_next) : 0;
    float3 r_cur = FR ? make_float3(0.f, 0.f, 1.f) : load_r(a.r, (unsigned)e0 < (unsigned)a.E ? e0 : 0);
    if (producer) issue(e0, j_cur, 0);
    bool live = true;

    int row = segment_of(a.row_ptr, a.N, k0);
    int row_lo = __ldg(a.row_ptr + row), row_hi = __ldg(a.row_ptr + row + 1);
    int node = node_of(row);  // loaded a row early: used when the row is stored
    float2 acc[D];
#pragma unroll
    for (int k = 0; k < D; ++k) acc[k] = f2_zero();

    for (int q = k0, it = 0; q < k1; ++q, ++it) {
        while (q >= row_hi && row < a.N - 1) {  // the edge opens a later row: store the finished one
            if (row_hi > max(row_lo, k0)) {
                store_row<D>(row_slot(out2, part2, node, row_lo, row_hi, k0, k1, G.task, D * C2, cp), C2, acc);
#pragma unroll
                for (int k = 0; k < D; ++k) acc[k] = f2_zero();
            }
            ++row;
            row_lo = row_hi;
            row_hi = __ldg(a.row_ptr + row + 1);
            node = node_of(row);
        }
        const int slot = it & 1;
        if (producer && q + 1 < k1) issue(e_next, j_next, slot ^ 1);
        const int e_next3 = q + 3 < k1 ? edge_at(q + 3) : 0;
        const int j_after = q + 2 < k1 ? src_of(e_next2) : 0;
        const float3 r_next =
            (!FR && q + 1 < k1) ? load_r(a.r, (unsigned)e_next < (unsigned)a.E ? e_next : 0) : r_cur;
        const bool valid = (unsigned)j_cur < (unsigned)a.N;  // an invalid source contributes nothing
        Frame f;
        if constexpr (FR) {
            mbar_wait(&bar[slot], (it >> 1) & 1, live);
            const float* fb = fbuf + slot * kFrameFloats;
            f = frame_of(fb);
            if (!f.degenerate) expand_wigner<L>(fb, G.tl, G.T, G.tmask, dbuf);
        } else {
            f = make_frame(r_cur.x, r_cur.y, r_cur.z);
            if (!f.degenerate) team_wigner<L>(f, G.tl, G.T, G.tmask, ybuf, dbuf, smem);
            mbar_wait(&bar[slot], (it >> 1) & 1, live);
        }
        const float2* xs = reinterpret_cast<const float2*>(xbuf + slot * D * C) + cp;
        const float2* ws = reinterpret_cast<const float2*>(wbuf + slot * P * C) + cp;
        if (valid && !f.degenerate) {
            float2 xp[D];
            {
                float2 xv[D];
#pragma unroll
                for (int k = 0; k < D; ++k) xv[k] = lds2(xs + k * C2);
                rotate_all<L>(f, dbuf, xv, xp);
            }
            static_for<0, L + 1>([&](auto l3c) {
                constexpr int l3 = decltype(l3c)::value;
                float2 y[2 * l3 + 1];
#pragma unroll
                for (int m = 0; m < 2 * l3 + 1; ++m) y[m] = f2_zero();
                static_for<0, L + 1>([&](auto l1c) {
                    constexpr int l1 = decltype(l1c)::value;
                    if constexpr (has_type<L, O3>(l1, l3, 0) || has_type<L, O3>(l1, l3, 1)) {
                        float2 We[4], Wo[4];
                        group_weights<L, O3, l1, l3>(ws, C2, We, Wo);
                        apply_M<L, O3, l1, l3>(We, Wo, xp + l1 * l1, y);
                    }
                });
                rotate<l3, true, true>(f, dbuf, y, acc + l3 * l3);
            });
        } else if (valid) {
            // no direction: only the paths (l, 0, l) act, each as the identity
            static_for<0, L + 1>([&](auto lc) {
                constexpr int l = decltype(lc)::value;
                const float2 w = lds2(ws + path_index<L, O3>(l, 0, l) * C2);
#pragma unroll
                for (int m = 0; m < 2 * l + 1; ++m) f2_fma(acc[l * l + m], w, lds2(xs + (l * l + m) * C2));
            });
        }
        group_sync();  // this slot's buffers are free for the edge after next
        j_cur = j_next;
        j_next = j_after;
        e_next = e_next2;
        e_next2 = e_next3;
        r_cur = r_next;
    }
    store_row<D>(row_slot(out2, part2, node, row_lo, row_hi, k0, k1, G.task, D * C2, cp), C2, acc);
    if (G.slice == 0 && G.tl == 0) tail_record(part2, a.ntasks, D * C2, G.task, row, row_lo, row_hi, k0, k1);
}

// ===========================================================================
// Backward: task = a contiguous range of reverse-CSR (source-ordered) positions.
// Weight rows are bulk-copied into two buffers like the forward's; the node rows
// (x of the source, grad_out of the destination) are copied lane by lane
// (cp.async) into lane-owned buffers, refilled for the next edge as soon as this
// edge has read them. FR: frame records given, as in the forward.
template <int L, bool O3, int C2T, bool FR>
__global__ void __launch_bounds__(frame::kThreads, L <= 2 ? 6 : 4) etp_bwd_frame_kernel(BwdArgs a) {
    using namespace frame;
    constexpr int D = (L + 1) * (L + 1);
    constexpr int P = PathSet<L, O3>::P;
    extern __shared__ __align__(16) float smem[];
    if constexpr (!FR) load_fit_tables(smem);
    const Geometry G = geometry(a.team, a.slices);
    if (G.task >= a.ntasks) return;  // the slice teams of a task leave together
    int k0, k1;
    task_range(a.E, G.task, a.ntasks, k0, k1);
    if (k0 >= k1) return;
    const int C2 = C2T ? C2T : a.C4 * 2, C = 2 * C2;
    const int ngroups = (kThreads / G.T) / G.S;
    float* comb = smem + kFitStride;  // slice partials of grad_r, double-buffered by edge parity
    const int gfloats = group_floats(P, D, C, 0, FR);
    float* gbase = smem + kHeaderFloats + (G.team_in_block / G.S) * gfloats;
    uint64_t* bar = reinterpret_cast<uint64_t*>(gbase);  // [0], [1]: weight buffers
    float* wbuf = gbase + kBarFloats;
    float* fbuf = wbuf + 2 * P * C;  // two frame records (FR)
    float* team = smem + kHeaderFloats + ngroups * gfloats + G.team_in_block * bwd_team_floats(D, G.T);
    float* ybuf = team;
    float* dbuf = team + kYbufFloats;
    float2* xrow = reinterpret_cast<float2*>(team + kTeamFloats);  // this lane's channels of x[src], D x T
    float2* grow = xrow + D * G.T;                                  // and of grad_out[dst]
    const bool producer = G.slice == 0 && G.tl == 0;
    const int cp = G.slice * G.T + G.tl;
    const uint64_t pol_w = l2_evict_first_policy();
    float2* gw2 = reinterpret_cast<float2*>(a.grad_w);
    float2* gx2 = reinterpret_cast<float2*>(a.grad_x);
    float2* part2 = reinterpret_cast<float2*>(a.part);
    const bool want_w = a.grad_w != nullptr;
    const bool want_r = a.grad_r != nullptr;
    auto group_sync = [&] {
        if (G.S == 2)
            __syncthreads();  // the block is exactly this task's two warps
        else
            __syncwarp(G.tmask);
    };

    // position q of the reverse order -> edge; out-of-range edges and rows map to
    // valid addresses and are marked invalid (they contribute and store nothing)
    auto edge_at = [&](int q) -> int { return __ldg(a.rev_perm + q); };
    auto node_of = [&](int rank) -> int { return a.order ? __ldg(a.order + rank) : rank; };  // source row -> node
    auto valid_edge = [&](int e) { return (unsigned)e < (unsigned)a.E; };
    auto dst_of = [&](int e) -> int {
        if (!valid_edge(e)) return -1;
        return a.dst ? __ldg(a.dst + e) : row_of_edge(a.row_ptr, a.N, e);
    };
    const unsigned wbytes = 4u * P * C, fbytes = FR ? 4u * kFrameFloats : 0u;
    auto issue_w = [&](int e, int slot) {
        e = valid_edge(e) ? e : 0;
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        mbar_expect_tx(&bar[slot], wbytes + fbytes);
        bulk_g2s_stream(wbuf + slot * P * C, reinterpret_cast<const float*>(a.w) + (size_t)e * P * C, wbytes, &bar[slot],
                        pol_w);
        if constexpr (FR)
            bulk_g2s(fbuf + slot * kFrameFloats, a.frames + (size_t)e * kFrameFloats, fbytes, &bar[slot]);
    };
    const float2* x2 = reinterpret_cast<const float2*>(a.x);
    const float2* g2 = reinterpret_cast<const float2*>(a.g);
    auto copy_x = [&](int node) {
        const float2* xs = x2 + (size_t)node * D * C2 + cp;
#pragma unroll
        for (int k = 0; k < D; ++k) cp_async8(xrow + k * G.T + G.tl, xs + k * C2);
        cp_async_commit();
    };
    auto copy_g = [&](int i) {
        const float2* gs = g2 + (size_t)((unsigned)i < (unsigned)a.N ? i : 0) * D * C2 + cp;
#pragma unroll
        for (int k = 0; k < D; ++k) cp_async8(grow + k * G.T + G.tl, gs + k * C2);
        cp_async_commit();
    };

    int row = segment_of(a.rev_ptr, a.N, k0);  // source row of position k0
    int row_lo = __ldg(a.rev_ptr + row), row_hi = __ldg(a.rev_ptr + row + 1);
    // the nodes of this source row and the next, loaded a row early
    int node = node_of(row), node_nx = row + 1 < a.N ? node_of(row + 1) : 0;
    // positions from rev_ptr[N] on hold the edges whose source is out of range (an
    // invalid CSR): they contribute nothing and get zero grad_w and grad_r
    const int pos_end = __ldg(a.rev_ptr + a.N);
    // the edge of the next position and the destination and vector of the next
    // edge are loaded an edge early (the position after next: two early)
    int e_cur = edge_at(k0);
    int i_cur = dst_of(e_cur);
    int e_next = k0 + 1 < k1 ? edge_at(k0 + 1) : 0;
    float3 r_cur = FR ? make_float3(0.f, 0.f, 1.f) : load_r(a.r, valid_edge(e_cur) ? e_cur : 0);
    if (producer) {
        mbar_init(&bar[0], 1);
        mbar_init(&bar[1], 1);
        mbar_fence_init();
    }
    group_sync();
    if (producer) issue_w(e_cur, 0);
    copy_x(node);
    copy_g(i_cur);
    bool live = true;

    float2 gx[D];
#pragma unroll
    for (int k = 0; k < D; ++k) gx[k] = f2_zero();

    for (int q = k0, it = 0; q < k1; ++q, ++it) {
        while (q >= row_hi && row < a.N - 1) {  // the position opens a later source row: store the finished one
            if (row_hi > max(row_lo, k0)) {
                if (gx2) store_row<D>(row_slot(gx2, part2, node, row_lo, row_hi, k0, k1, G.task, D * C2, cp), C2, gx);
#pragma unroll
                for (int k = 0; k < D; ++k) gx[k] = f2_zero();
            }
            ++row;
            row_lo = row_hi;
            row_hi = __ldg(a.rev_ptr + row + 1);
            node = node_nx;
            node_nx = row + 1 < a.N ? node_of(row + 1) : 0;
        }
        // the next position's source row, edge and destination (for the prefetches)
        const bool has_next = q + 1 < k1;
        const int slot = it & 1;
        if (producer && has_next) issue_w(e_next, slot ^ 1);
        int row_next = row;
        if (has_next) {
            int hi = row_hi;
            while (q + 1 >= hi && row_next < a.N - 1) hi = __ldg(a.rev_ptr + (++row_next) + 1);
        }
        const int e_after = q + 2 < k1 ? edge_at(q + 2) : 0;
        const int i_next = has_next ? dst_of(e_next) : 0;
        const float3 r_next = (!FR && has_next) ? load_r(a.r, valid_edge(e_next) ? e_next : 0) : r_cur;
        const bool ok = valid_edge(e_cur) && (unsigned)i_cur < (unsigned)a.N && q < pos_end;
        Frame f;
        if constexpr (FR) {
            cp_async_wait_all();  // this edge's node rows (this lane's copies)
            mbar_wait(&bar[slot], (it >> 1) & 1, live);
            const float* fb = fbuf + slot * kFrameFloats;
            f = frame_of(fb);
            if (ok && !f.degenerate) expand_wigner<L>(fb, G.tl, G.T, G.tmask, dbuf);
        } else {
            f = ok ? make_frame(r_cur.x, r_cur.y, r_cur.z) : make_frame(0.f, 0.f, 1.f);
            if (ok && !f.degenerate) team_wigner<L>(f, G.tl, G.T, G.tmask, ybuf, dbuf, smem);
            cp_async_wait_all();  // this edge's node rows (this lane's copies)
            mbar_wait(&bar[slot], (it >> 1) & 1, live);
        }
        const float2* ws = reinterpret_cast<const float2*>(wbuf + slot * P * C) + cp;
        float2* gwe = (want_w && valid_edge(e_cur)) ? gw2 + (size_t)e_cur * P * C2 + cp : nullptr;
        float2 sx2 = f2_zero(), sy2 = f2_zero();  // dL/de_x, dL/de_y per channel of this lane
        if (ok && !f.degenerate) {
            float2 xp[D], gpa[D], z[D];
            {
                float2 v[D], u[D];
#pragma unroll
                for (int k = 0; k < D; ++k) v[k] = lds2(xrow + k * G.T + G.tl);
#pragma unroll
                for (int k = 0; k < D; ++k) u[k] = lds2(grow + k * G.T + G.tl);
                rotate_all2<L>(f, dbuf, v, u, xp, gpa);
            }
            // next source's x row, behind this edge's reads
            if (has_next && row_next != row) copy_x(row_next == row + 1 ? node_nx : node_of(row_next));
            if (has_next) copy_g(i_next);
#pragma unroll
            for (int k = 0; k < D; ++k) z[k] = f2_zero();
            static_for<0, L + 1>([&](auto l3c) {
                constexpr int l3 = decltype(l3c)::value;
                constexpr int d3 = 2 * l3 + 1;
                float2 y[d3];
                const float2* gp = gpa + l3 * l3;
#pragma unroll
                for (int m = 0; m < d3; ++m) y[m] = f2_zero();
                static_for<0, L + 1>([&](auto l1c) {
                    constexpr int l1 = decltype(l1c)::value;
                    if constexpr (has_type<L, O3>(l1, l3, 0) || has_type<L, O3>(l1, l3, 1)) {
                        float2 We[4], Wo[4];
                        group_weights<L, O3, l1, l3>(ws, C2, We, Wo);
                        apply_M<L, O3, l1, l3>(We, Wo, xp + l1 * l1, y);
                        apply_MT<L, O3, l1, l3>(We, Wo, gp, z + l1 * l1);
                        if (gwe) {
                            // products of the frame components coupled by B_p, symmetrised in +-mu
                            constexpr int mn = cmin(l1, l3);
                            float2 Pe[4], Po[4];
                            static_for<0, mn + 1>([&](auto mc) {
                                constexpr int mu = decltype(mc)::value;
                                const float2 a1 = gp[l3 + mu], a2 = gp[l3 - mu];
                                const float2 b1 = xp[l1 * l1 + l1 + mu], b2 = xp[l1 * l1 + l1 - mu];
                                if constexpr (mu == 0) {
                                    Pe[0] = f2_mul(a1, b1);
                                    Po[0] = f2_zero();
                                } else {
                                    Pe[mu] = __ffma2_rn(a1, b1, f2_mul(a2, b2));
                                    Po[mu] = f2_mul(a1, b2);
                                    f2_fms(Po[mu], a2, b1);
                                }
                            });
                            static_for<0, L + 1>([&](auto l2c) {
                                constexpr int l2 = decltype(l2c)::value;
                                if constexpr (PathSet<L, O3>::allowed(l1, l2, l3)) {
                                    constexpr int p = path_index<L, O3>(l1, l2, l3);
                                    constexpr bool odd = (l1 + l2 + l3) % 2 == 1;
                                    float2 gw = f2_zero();
                                    static_for<0, mn + 1>([&](auto mc) {
                                        constexpr int mu = decltype(mc)::value;
                                        constexpr float b = (float)etp_gen::kFrameB[l1][l2][l3][mu];
                                        if constexpr (b != 0.f) f2_fma(gw, b, odd ? Po[mu] : Pe[mu]);
                                    });
                                    st_stream2(gwe + p * C2, gw, pol_w);
                                }
                            });
                        }
                    }
                });
                if (want_r) {
                    sx2 = f2_add(sx2, gen_form<l3, 0>(gp, y));
                    sy2 = f2_add(sy2, gen_form<l3, 1>(gp, y));
                }
            });
            static_for<0, L + 1>([&](auto l1c) {
                constexpr int l1 = decltype(l1c)::value;
                if (want_r) {
                    sx2 = f2_add(sx2, gen_form<l1, 0>(xp + l1 * l1, z + l1 * l1));
                    sy2 = f2_add(sy2, gen_form<l1, 1>(xp + l1 * l1, z + l1 * l1));
                }
                rotate<l1, true, true>(f, dbuf, z + l1 * l1, gx + l1 * l1);
            });
        } else {
            // an invalid edge contributes nothing; a degenerate one (no direction)
            // only through the paths (l, 0, l), each the identity, and has grad_r = 0
            if (ok) {
                static_for<0, L + 1>([&](auto lc) {
                    constexpr int l = decltype(lc)::value;
                    constexpr int p0 = path_index<L, O3>(l, 0, l);
                    const float2 w = lds2(ws + p0 * C2);
                    float2 gw = f2_zero();
#pragma unroll
                    for (int m = 0; m < 2 * l + 1; ++m) {
                        const float2 gv = lds2(grow + (l * l + m) * G.T + G.tl);
                        f2_fma(gx[l * l + m], w, gv);
                        f2_fma(gw, lds2(xrow + (l * l + m) * G.T + G.tl), gv);
                    }
                    if (gwe) st_stream2(gwe + p0 * C2, gw, pol_w);
                });
                if (gwe) {
                    static_for<0, P>([&](auto pc) {
                        constexpr int p = decltype(pc)::value;
                        constexpr Path pt = PathSet<L, O3>::path(p);
                        if constexpr (pt.l2 > 0) st_stream2(gwe + p * C2, f2_zero(), pol_w);
                    });
                }
            } else if (gwe) {
                static_for<0, P>([&](auto pc) { st_stream2(gwe + decltype(pc)::value * C2, f2_zero(), pol_w); });
            }
            if (has_next && row_next != row) copy_x(row_next == row + 1 ? node_nx : node_of(row_next));
            if (has_next) copy_g(i_next);
        }
        // sum dL/de over the lane's channels and the team's lanes; the second
        // slice (C = 128) hands its sum over through shared memory at the sync
        float sx = sx2.x + sx2.y, sy = sy2.x + sy2.y;
        if (want_r) {
            for (int s = 1; s < G.T; s <<= 1) {
                sx += __shfl_xor_sync(G.tmask, sx, s);
                sy += __shfl_xor_sync(G.tmask, sy, s);
            }
            if (G.S == 2 && G.slice == 1 && G.tl == 0) {
                comb[(it & 1) * 2] = sx;
                comb[(it & 1) * 2 + 1] = sy;
            }
        }
        group_sync();  // weight buffer free for the edge after next; slice partials visible
        if (want_r && valid_edge(e_cur) && G.slice == 0 && G.tl == 0) {  // zero when !ok (sx = sy = 0)
            if (G.S == 2) {
                sx += comb[(it & 1) * 2];
                sy += comb[(it & 1) * 2 + 1];
            }
            // grad_r = R^T (dL/de_y, -dL/de_x, 0) / |r|   (0 for a degenerate edge: inv_rho = 0)
            const float gu0 = sy * f.inv_rho, gu1 = -sx * f.inv_rho;
            float* gr = a.grad_r + 3 * (size_t)e_cur;
            gr[0] = f.R[0] * gu0 + f.R[3] * gu1;
            gr[1] = f.R[1] * gu0 + f.R[4] * gu1;
            gr[2] = f.R[2] * gu0 + f.R[5] * gu1;
        }
        e_cur = e_next;
        i_cur = i_next;
        e_next = e_after;
        r_cur = r_next;
    }
    cp_async_wait_all();
    if (gx2) {
        store_row<D>(row_slot(gx2, part2, node, row_lo, row_hi, k0, k1, G.task, D * C2, cp), C2, gx);
        if (G.slice == 0 && G.tl == 0) tail_record(part2, a.ntasks, D * C2, G.task, row, row_lo, row_hi, k0, k1);
    }
}

namespace frame {
template <int L, bool O3>
constexpr size_t smem_bytes_for(int C, int T, bool backward, bool framed) {
    constexpr int D = (L + 1) * (L + 1);
    constexpr int P = PathSet<L, O3>::P;
    const int teams = kThreads / T;
    const int S = C / (2 * T);
    const int groups = teams / S;
    return sizeof(float) * (size_t)(kHeaderFloats + groups * group_floats(P, D, C, backward ? 0 : 2, framed) +
                                    teams * (backward ? bwd_team_floats(D, T) : kTeamFloats));
}
}  // namespace frame

template <int L>
size_t smem_bytes(bool o3, int C, int T, bool backward, bool framed) {
    return o3 ? frame::smem_bytes_for<L, true>(C, T, backward, framed)
              : frame::smem_bytes_for<L, false>(C, T, backward, framed);
}

// Kernel of a specialisation: compile-time channel pairs for C = 128 and C = 64;
// frame records given or built in the kernel.
template <int L, bool O3, int C2T>
const void* kernel_of(bool backward, bool framed) {
    if (framed)
        return backward ? (const void*)etp_bwd_frame_kernel<L, O3, C2T, true>
                        : (const void*)etp_fwd_frame_kernel<L, O3, C2T, true>;
    return backward ? (const void*)etp_bwd_frame_kernel<L, O3, C2T, false>
                    : (const void*)etp_fwd_frame_kernel<L, O3, C2T, false>;
}
template <int L>
const void* kernel_for(bool o3, bool backward, bool framed, int C2) {
    if (C2 == 64) return o3 ? kernel_of<L, true, 64>(backward, framed) : kernel_of<L, false, 64>(backward, framed);
    if (C2 == 32) return o3 ? kernel_of<L, true, 32>(backward, framed) : kernel_of<L, false, 32>(backward, framed);
    return o3 ? kernel_of<L, true, 0>(backward, framed) : kernel_of<L, false, 0>(backward, framed);
}

template <int L>
int blocks_per_sm(bool o3, bool backward, bool framed, int C, size_t smem) {
    int n = 0;
    const void* k = kernel_for<L>(o3, backward, framed, C / 2);
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k, frame::kThreads, smem) != cudaSuccess) n = 1;
    return n < 1 ? 1 : n;
}

template <int L>
cudaError_t launch_forward(bool o3, const FwdArgs& a, dim3 grid, size_t smem, cudaStream_t s) {
    void* args[] = {const_cast<FwdArgs*>(&a)};
    return cudaLaunchKernel(kernel_for<L>(o3, false, a.frames != nullptr, a.C4 * 2), grid, dim3(frame::kThreads), args,
                            smem, s);
}

template <int L>
cudaError_t launch_backward(bool o3, const BwdArgs& a, dim3 grid, size_t smem, cudaStream_t s) {
    void* args[] = {const_cast<BwdArgs*>(&a)};
    return cudaLaunchKernel(kernel_for<L>(o3, true, a.frames != nullptr, a.C4 * 2), grid, dim3(frame::kThreads), args,
                            smem, s);
}

template <int L>
cudaError_t launch_edge_frames(int E, const float* r, float* frames, cudaStream_t s) {
    if (E == 0) return cudaSuccess;
    const unsigned blocks = (unsigned)((E + frame::kFrameBlock - 1) / frame::kFrameBlock);
    frame::etp_edge_frames_kernel<L><<<blocks, frame::kFrameBlock, 0, s>>>(E, r, reinterpret_cast<float4*>(frames));
    return cudaGetLastError();
}

}  // namespace etp
