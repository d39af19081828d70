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
// Work decomposition: a team of T lanes owns one node and a slice of 2T channels
// (lane t holds channels 2(sT + t), 2(sT + t) + 1 as a float2). T = min(32, C/2);
// with C = 128 a node has two slices, i.e. two warps of the same block. Each
// team computes its edge's Wigner matrices cooperatively into its own shared
// memory. Forward: teams walk the destination row (CSR), accumulate in
// registers, store the node once. Backward: teams walk the source row (reverse
// CSR) and store grad_x once; grad_w and grad_r are per edge. No atomics.
#pragma once

#include "etp_device.cuh"
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
constexpr int kDbufFloats = 96;             // D_2 (5 rows x 8) then D_3 (7 rows x 8)
constexpr int kTeamFloats = kYbufFloats + kDbufFloats;
constexpr int kFitFloats = 24 + 2 * 49;     // points (padded) + A_2^-1, A_3^-1 (7 x 7 each)
constexpr int kFitStride = 128;             // shared-memory floats reserved for the fit table
// Team buffers are read with 16-byte vector loads: every offset must keep 16-byte alignment.
static_assert(kFitStride >= kFitFloats && kFitStride % 4 == 0, "fit table stride");
static_assert(kYbufFloats % 4 == 0 && kTeamFloats % 4 == 0, "team buffer alignment");
constexpr int kHeaderFloats = kFitStride + 8;  // fit table, then the grad_r slice partials
constexpr int kRingFwd = 24;                   // weight-ring slots (paths) per team, forward
constexpr int kRingBwd = 8;                    // and backward (its node rows take more room)
// Floats of one team's shared buffers: harmonics and Wigner matrices, `rows`
// node-row buffers of D x T float2, and the weight ring.
constexpr int team_floats(int D, int T, int rows, int ring) {
    return kTeamFloats + rows * D * T * 2 + ring * T * 2;
}
static_assert(kHeaderFloats % 4 == 0, "header alignment");

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

__device__ __forceinline__ void f2_fma(float2& acc, float s, float2 v) {
    acc.x = fmaf(s, v.x, acc.x);
    acc.y = fmaf(s, v.y, acc.y);
}
__device__ __forceinline__ void f2_fma(float2& acc, float2 a, float2 b) {
    acc.x = fmaf(a.x, b.x, acc.x);
    acc.y = fmaf(a.y, b.y, acc.y);
}
__device__ __forceinline__ void f2_fms(float2& acc, float2 a, float2 b) {  // acc -= a * b
    acc.x = fmaf(-a.x, b.x, acc.x);
    acc.y = fmaf(-a.y, b.y, acc.y);
}
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

__device__ __forceinline__ Frame make_frame(float rx, float ry, float rz) {
    Frame f;
    const float n2 = rx * rx + ry * ry + rz * rz;
    f.degenerate = !(n2 >= 1e-24f);
    const float inv = f.degenerate ? 0.f : rsqrtf(n2);
    const float x = f.degenerate ? 0.f : rx * inv, y = f.degenerate ? 0.f : ry * inv;
    const float z = f.degenerate ? 1.f : rz * inv;
    const float s = copysignf(1.f, z);
    const float a = -1.f / (s + z);
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
        constexpr int n2 = 25, n3 = L >= 3 ? 49 : 0;
        const float* inv2 = fit + 24;
        const float* inv3 = fit + 24 + 49;
        for (int idx = tl; idx < n2 + n3; idx += T) {
            const bool is3 = idx >= n2;
            const int j = is3 ? idx - n2 : idx;
            const int d = is3 ? 7 : 5;
            const int a = j / d, b = j - a * d;
            const float* inv = is3 ? inv3 : inv2;
            const int yoff = is3 ? 5 : 0;
            float v = 0.f;
#pragma unroll
            for (int k = 0; k < NP; ++k) v = fmaf(ybuf[k * 12 + yoff + a], inv[k * 7 + b], v);
            dbuf[(is3 ? 40 : 0) + a * 8 + b] = v;
        }
        __syncwarp(tmask);
    }
}

// out = D_l in  (TRANS = false)   or   out (+)= D_l^T in  (TRANS = true, ACC adds)
// D_2, D_3 rows are 8 floats apart in the team buffer and read as two float4.
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
            float row[8];
            if constexpr (l == 1) {
#pragma unroll
                for (int b = 0; b < d; ++b) row[b] = d1(f, a, b);
            } else {
                const float4 lo = lds4(dbuf + (l == 2 ? 0 : 40) + a * 8);
                const float4 hi = lds4(dbuf + (l == 2 ? 0 : 40) + a * 8 + 4);
                row[0] = lo.x, row[1] = lo.y, row[2] = lo.z, row[3] = lo.w;
                row[4] = hi.x, row[5] = hi.y, row[6] = hi.z, row[7] = hi.w;
            }
#pragma unroll
            for (int b = 0; b < d; ++b) {
                if constexpr (TRANS)
                    f2_fma(tmp[b], row[b], in[a]);
                else
                    f2_fma(tmp[a], row[b], in[b]);
            }
        }
    }
#pragma unroll
    for (int a = 0; a < d; ++a) {
        if constexpr (ACC) {
            out[a].x += tmp[a].x;
            out[a].y += tmp[a].y;
        } else {
            out[a] = tmp[a];
        }
    }
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
// Streaming of the per-edge weights: every lane copies its own two channels of
// each path into a ring of shared-memory slots with cp.async, a fixed number of
// paths (DIST) ahead of their use, in the order the kernels consume them
// (l3 outer, l1, l2 inner). Each consumption step issues one copy group and
// waits until the group holding the step's own path has landed, so that DIST
// copies stay in flight without holding registers. A lane reads back only what
// it copied itself, so no cross-lane synchronisation is needed. The next edge's
// node row (x for the forward, grad_out for the backward) rides in the group of
// the first step of the current edge.
__device__ __forceinline__ unsigned smem_u32(const void* p) { return (unsigned)__cvta_generic_to_shared(p); }
__device__ __forceinline__ void cp_async8(const void* smem, const void* gmem) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(smem_u32(smem)), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
__device__ __forceinline__ float2 lds2(const float2* p) {
    float2 v;
    asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(smem_u32(p)));
    return v;
}

// Consumption order of the paths within an edge (l3 outer, l1, l2 inner).
template <int L, bool O3>
struct Order {
    static constexpr int P = PathSet<L, O3>::P;
    static constexpr int path_at(int k) {
        int n = 0;
        for (int c = 0; c <= L; ++c)
            for (int a = 0; a <= L; ++a)
                for (int b = 0; b <= L; ++b)
                    if (PathSet<L, O3>::allowed(a, b, c)) {
                        if (n == k) return path_index<L, O3>(a, b, c);
                        ++n;
                    }
        return -1;
    }
    static constexpr int pos(int l1, int l2, int l3) {
        int n = 0;
        for (int c = 0; c <= L; ++c)
            for (int a = 0; a <= L; ++a)
                for (int b = 0; b <= L; ++b)
                    if (PathSet<L, O3>::allowed(a, b, c)) {
                        if (a == l1 && b == l2 && c == l3) return n;
                        ++n;
                    }
        return -1;
    }
};

// Parts of an edge's weights in consumption order: NQ parts of PP paths. PP is
// odd, so the lane-major slots (lane t's paths at t * PP + k) are read and
// written without shared-memory bank conflicts.
template <int L, bool O3>
struct Parts {
    static constexpr int P = PathSet<L, O3>::P;
    static constexpr int NQ0 = P < 4 ? P : 4;
    static constexpr int PP = ((P + NQ0 - 1) / NQ0) | 1;
    static constexpr int NQ = (P + PP - 1) / PP;
    static constexpr int begin(int q) { return q * PP; }
    static constexpr int end(int q) { return (q + 1) * PP < P ? (q + 1) * PP : P; }
    static constexpr int ring_float2(int T) { return (NQ + 1) * PP * T; }
};

// The weight pipe of one team: a ring of NQ + 1 part slots. Part q of the next
// edge is issued when part q of the current edge starts (one edge of lead), into
// the slot the previous part has just released; one cp.async group per part.
// Group bookkeeping (groups numbered in issue order, part q of edge i is group
// i NQ + q): at the start of an edge the groups of its part 0 (which also holds
// its node rows) are complete after wait_group(NQ - 1); at the start of part q,
// after issuing the group of the next edge's part q, wait_group(NQ) leaves the
// current part complete.
template <int L, bool O3>
struct Pipe {
    using PT = Parts<L, O3>;
    static constexpr int P = PT::P, NQ = PT::NQ, PP = PT::PP;
    float2* ring;          // (NQ + 1) slots of PP x T float2, lane-major
    int T, tl, C2;
    int slot0;             // slot of part 0 of the current edge
    const float2* w_next;  // this lane's weights of the next edge, or nullptr

    __device__ __forceinline__ float2* lane_slot(int slot) { return ring + (slot * T + tl) * PP; }

    template <int q>
    __device__ __forceinline__ void issue_part(const float2* w, int slot) {
        float2* dst = lane_slot(slot);
        static_for<PT::begin(q), PT::end(q)>([&](auto kc) {
            constexpr int k = decltype(kc)::value;
            cp_async8(dst + (k - PT::begin(q)), w + Order<L, O3>::path_at(k) * C2);
        });
    }

    // First edge: all its parts, its node rows (issued by `rows`) in the first group.
    template <class Rows>
    __device__ __forceinline__ void prologue(const float2* w_first, Rows&& rows) {
        slot0 = 0;
        static_for<0, NQ>([&](auto qc) {
            constexpr int q = decltype(qc)::value;
            if (w_first) issue_part<q>(w_first, q);
            if constexpr (q == 0) rows();
            cp_async_commit();
        });
    }

    __device__ __forceinline__ void edge_begin() { cp_async_wait<NQ - 1>(); }

    // Start of part q of the current edge: issue the next edge's part q (and at
    // q = 0 its node rows), wait for the current part.
    template <int q, class Rows>
    __device__ __forceinline__ void part_begin(Rows&& next_rows) {
        if (w_next) issue_part<q>(w_next, (slot0 + q + NQ) % (NQ + 1));
        if constexpr (q == 0) next_rows();
        cp_async_commit();
        cp_async_wait<NQ>();
    }

    // Weight of consumption position k (its part has begun).
    template <int k>
    __device__ __forceinline__ float2 w_at() {
        constexpr int q = k / PP;
        return lds2(lane_slot((slot0 + q) % (NQ + 1)) + (k - q * PP));
    }

    __device__ __forceinline__ void edge_end(const float2* next_after) {
        slot0 = (slot0 + NQ) % (NQ + 1);
        w_next = next_after;
    }
};

// Combined frame weights of the (l1, l3) group for this lane's channels:
// We[mu] = sum over even paths (l1, l2, l3) of b_p(mu) w_p, Wo[mu] likewise for
// odd paths; degenerate edges keep only l2 = 0. Part boundaries inside the group
// advance the pipe.
template <int L, bool O3, int l1, int l3, class Rows>
__device__ __forceinline__ void group_weights(Pipe<L, O3>& pp, Rows&& next_rows, bool degenerate, float2 (&We)[4],
                                              float2 (&Wo)[4]) {
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        We[m] = f2_zero();
        Wo[m] = f2_zero();
    }
    static_for<0, L + 1>([&](auto l2c) {
        constexpr int l2 = decltype(l2c)::value;
        if constexpr (PathSet<L, O3>::allowed(l1, l2, l3)) {
            constexpr int k = Order<L, O3>::pos(l1, l2, l3);
            constexpr int PP = Parts<L, O3>::PP;
            if constexpr (k % PP == 0) pp.template part_begin<k / PP>(next_rows);
            float2 w = pp.template w_at<k>();
            if (l2 > 0 && degenerate) w = f2_zero();
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

// sum over the lane's channels of  -(J_a v)^T s  for a block of degree l:  -sum J[m][m'] v[m'] s[m]
template <int l, int axis>
__device__ __forceinline__ float gen_form(const float2* v, const float2* s) {
    float acc = 0.f;
    static_for<0, 2 * l + 1>([&](auto ac) {
        constexpr int a = decltype(ac)::value;
        static_for<0, 2 * l + 1>([&](auto bc) {
            constexpr int b = decltype(bc)::value;
            constexpr float J = (float)etp_gen::kGen[axis][l][a][b];
            if constexpr (J != 0.f) {
                acc = fmaf(-J, v[b].x * s[a].x, acc);
                acc = fmaf(-J, v[b].y * s[a].y, acc);
            }
        });
    });
    return acc;
}

// ---------------------------------------------------------------------------
// Work decomposition: equal contiguous ranges of edges ("tasks"), one per team
// (or per pair of slice teams when C = 128, the block's two warps). Rows cut by a
// range boundary are combined by vector reductions on a zeroed output; rows
// inside a range are stored once.
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

__device__ __forceinline__ void red_add2(float2* p, float2 v) {
    asm volatile("red.global.add.v2.f32 [%0], {%1, %2};" ::"l"(p), "f"(v.x), "f"(v.y) : "memory");
}

// Store a row accumulator: plainly when the task owns the whole row, else by
// vector reduction onto the zeroed output.
template <int D>
__device__ __forceinline__ void flush_row(float2* row, int C2, const float2 (&acc)[D], bool whole) {
#pragma unroll
    for (int k = 0; k < D; ++k) {
        if (whole)
            row[k * C2] = acc[k];
        else
            red_add2(row + k * C2, acc[k]);
    }
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

}  // namespace frame


// ===========================================================================
// Forward: task = a contiguous range of CSR (destination-ordered) edges.
template <int L, bool O3>
__global__ void __launch_bounds__(frame::kThreads, 4) etp_fwd_frame_kernel(FwdArgs a) {
    using namespace frame;
    using PT = Parts<L, O3>;
    constexpr int D = (L + 1) * (L + 1);
    constexpr int P = PT::P;
    extern __shared__ __align__(16) float smem[];
    load_fit_tables(smem);
    const Geometry G = geometry(a.team, a.slices);
    if (G.task >= a.ntasks) return;  // the slice teams of a task leave together
    int k0, k1;
    task_range(a.E, G.task, a.ntasks, k0, k1);
    if (k0 >= k1) return;
    float* team = smem + kHeaderFloats + G.team_in_block * team_floats(D, G.T, 1, PT::ring_float2(G.T) / G.T);
    float* ybuf = team;
    float* dbuf = team + kYbufFloats;
    float2* xbuf = reinterpret_cast<float2*>(team + kYbufFloats + kDbufFloats);
    float2* ring = xbuf + D * G.T;
    const int C2 = a.C4 * 2;
    const int cp = G.slice * G.T + G.tl;
    const float2* x2 = reinterpret_cast<const float2*>(a.x);
    const float2* w2 = reinterpret_cast<const float2*>(a.w);
    float2* out2 = reinterpret_cast<float2*>(a.out);

    auto w_of = [&](int e) -> const float2* { return e < k1 ? w2 + (size_t)e * P * C2 + cp : nullptr; };
    auto copy_x = [&](int j) {  // an out-of-range source reads row 0 and is zeroed later
        const float2* src = x2 + (size_t)((unsigned)j < (unsigned)a.N ? j : 0) * D * C2 + cp;
#pragma unroll
        for (int k = 0; k < D; ++k) cp_async8(xbuf + k * G.T + G.tl, src + k * C2);
    };

    int row = segment_of(a.row_ptr, a.N, k0);
    int row_lo = __ldg(a.row_ptr + row), row_hi = __ldg(a.row_ptr + row + 1);
    int j_cur = __ldg(a.src + k0);
    Pipe<L, O3> pp{ring, G.T, G.tl, C2, 0, w_of(k0 + 1)};
    pp.prologue(w_of(k0), [&] { copy_x(j_cur); });

    float2 acc[D];
#pragma unroll
    for (int k = 0; k < D; ++k) acc[k] = f2_zero();

    for (int e = k0; e < k1; ++e) {
        while (e >= row_hi && row < a.N - 1) {  // the edge opens a later row: store the finished one
            if (row_hi > max(row_lo, k0)) {
                flush_row<D>(out2 + (size_t)row * D * C2 + cp, C2, acc, row_lo >= k0);
#pragma unroll
                for (int k = 0; k < D; ++k) acc[k] = f2_zero();
            }
            ++row;
            row_lo = row_hi;
            row_hi = __ldg(a.row_ptr + row + 1);
        }
        const bool has_next = e + 1 < k1;
        const int j_next = has_next ? __ldg(a.src + e + 1) : 0;
        pp.edge_begin();
        const Frame f = make_frame(__ldg(a.r + 3 * (size_t)e), __ldg(a.r + 3 * (size_t)e + 1),
                                   __ldg(a.r + 3 * (size_t)e + 2));
        team_wigner<L>(f, G.tl, G.T, G.tmask, ybuf, dbuf, smem);
        float2 xp[D];
        {
            float2 xv[D];
            const bool valid = (unsigned)j_cur < (unsigned)a.N;  // an invalid source contributes nothing
#pragma unroll
            for (int k = 0; k < D; ++k) xv[k] = valid ? lds2(xbuf + k * G.T + G.tl) : f2_zero();
            rotate_all<L>(f, dbuf, xv, xp);
        }
        auto next_rows = [&] {
            if (has_next) copy_x(j_next);
        };
        static_for<0, L + 1>([&](auto l3c) {
            constexpr int l3 = decltype(l3c)::value;
            float2 y[2 * l3 + 1];
#pragma unroll
            for (int m = 0; m < 2 * l3 + 1; ++m) y[m] = f2_zero();
            static_for<0, L + 1>([&](auto l1c) {
                constexpr int l1 = decltype(l1c)::value;
                if constexpr (has_type<L, O3>(l1, l3, 0) || has_type<L, O3>(l1, l3, 1)) {
                    float2 We[4], Wo[4];
                    group_weights<L, O3, l1, l3>(pp, next_rows, f.degenerate, We, Wo);
                    apply_M<L, O3, l1, l3>(We, Wo, xp + l1 * l1, y);
                }
            });
            rotate<l3, true, true>(f, dbuf, y, acc + l3 * l3);
        });
        pp.edge_end(w_of(e + 2));
        j_cur = j_next;
    }
    cp_async_wait_all();
    flush_row<D>(out2 + (size_t)row * D * C2 + cp, C2, acc, row_lo >= k0 && row_hi <= k1);
}

// ===========================================================================
// Backward: task = a contiguous range of reverse-CSR (source-ordered) positions.
template <int L, bool O3>
__global__ void __launch_bounds__(frame::kThreads, 4) etp_bwd_frame_kernel(BwdArgs a) {
    using namespace frame;
    using PT = Parts<L, O3>;
    constexpr int D = (L + 1) * (L + 1);
    constexpr int P = PT::P;
    extern __shared__ __align__(16) float smem[];
    load_fit_tables(smem);
    const Geometry G = geometry(a.team, a.slices);
    if (G.task >= a.ntasks) return;  // the slice teams of a task leave together
    int k0, k1;
    task_range(a.E, G.task, a.ntasks, k0, k1);
    if (k0 >= k1) return;
    float* comb = smem + kFitStride;  // slice partials of grad_r, double-buffered by edge parity
    float* team = smem + kHeaderFloats + G.team_in_block * team_floats(D, G.T, 2, PT::ring_float2(G.T) / G.T);
    float* ybuf = team;
    float* dbuf = team + kYbufFloats;
    float2* xbuf = reinterpret_cast<float2*>(team + kYbufFloats + kDbufFloats);
    float2* gbuf = xbuf + D * G.T;
    float2* ring = gbuf + D * G.T;
    const int C2 = a.C4 * 2;
    const int cp = G.slice * G.T + G.tl;
    const uint64_t pol_w = l2_evict_first_policy();
    const float2* x2 = reinterpret_cast<const float2*>(a.x);
    const float2* g2 = reinterpret_cast<const float2*>(a.g);
    const float2* w2 = reinterpret_cast<const float2*>(a.w);
    float2* gw2 = reinterpret_cast<float2*>(a.grad_w);
    float2* gx2 = reinterpret_cast<float2*>(a.grad_x);
    const bool want_w = a.grad_w != nullptr;
    const bool want_r = a.grad_r != nullptr;

    // position q of the reverse order -> edge; out-of-range edges and rows map to
    // valid addresses and are marked invalid (they contribute and store nothing)
    auto edge_at = [&](int q) -> int { return __ldg(a.rev_perm + q); };
    auto valid_edge = [&](int e) { return (unsigned)e < (unsigned)a.E; };
    auto dst_of = [&](int e) -> int {
        if (!valid_edge(e)) return -1;
        return a.dst ? __ldg(a.dst + e) : row_of_edge(a.row_ptr, a.N, e);
    };
    auto w_of = [&](int q) -> const float2* {
        if (q >= k1) return nullptr;
        const int e = edge_at(q);
        return w2 + (size_t)(valid_edge(e) ? e : 0) * P * C2 + cp;
    };
    auto copy_rows = [&](int j, int i) {
        const float2* xs = x2 + (size_t)j * D * C2 + cp;
        const float2* gs = g2 + (size_t)((unsigned)i < (unsigned)a.N ? i : 0) * D * C2 + cp;
#pragma unroll
        for (int k = 0; k < D; ++k) {
            cp_async8(xbuf + k * G.T + G.tl, xs + k * C2);
            cp_async8(gbuf + k * G.T + G.tl, gs + k * C2);
        }
    };

    int row = segment_of(a.rev_ptr, a.N, k0);  // source node of position k0
    int row_lo = __ldg(a.rev_ptr + row), row_hi = __ldg(a.rev_ptr + row + 1);
    int e_cur = edge_at(k0);
    int i_cur = dst_of(e_cur);
    Pipe<L, O3> pp{ring, G.T, G.tl, C2, 0, w_of(k0 + 1)};
    pp.prologue(w_of(k0), [&] { copy_rows(row, i_cur); });

    float2 gx[D];
#pragma unroll
    for (int k = 0; k < D; ++k) gx[k] = f2_zero();

    for (int q = k0, it = 0; q < k1; ++q, ++it) {
        while (q >= row_hi && row < a.N - 1) {  // the position opens a later source row: store the finished one
            if (row_hi > max(row_lo, k0)) {
                if (gx2) flush_row<D>(gx2 + (size_t)row * D * C2 + cp, C2, gx, row_lo >= k0);
#pragma unroll
                for (int k = 0; k < D; ++k) gx[k] = f2_zero();
            }
            ++row;
            row_lo = row_hi;
            row_hi = __ldg(a.rev_ptr + row + 1);
        }
        // the next position's source row and destination (for the row prefetch)
        const bool has_next = q + 1 < k1;
        int row_next = row, e_next = 0, i_next = 0;
        if (has_next) {
            int hi = row_hi;
            while (q + 1 >= hi && row_next < a.N - 1) hi = __ldg(a.rev_ptr + (++row_next) + 1);
            e_next = edge_at(q + 1);
            i_next = dst_of(e_next);
        }
        const bool ok = valid_edge(e_cur) && (unsigned)i_cur < (unsigned)a.N;
        pp.edge_begin();
        Frame f = make_frame(0.f, 0.f, 1.f);
        if (ok)
            f = make_frame(__ldg(a.r + 3 * (size_t)e_cur), __ldg(a.r + 3 * (size_t)e_cur + 1),
                           __ldg(a.r + 3 * (size_t)e_cur + 2));
        team_wigner<L>(f, G.tl, G.T, G.tmask, ybuf, dbuf, smem);
        float2 xp[D], gp[D], z[D];
        {
            float2 v[D];
#pragma unroll
            for (int k = 0; k < D; ++k) v[k] = ok ? lds2(xbuf + k * G.T + G.tl) : f2_zero();
            rotate_all<L>(f, dbuf, v, xp);
#pragma unroll
            for (int k = 0; k < D; ++k) v[k] = ok ? lds2(gbuf + k * G.T + G.tl) : f2_zero();
            rotate_all<L>(f, dbuf, v, gp);
        }
#pragma unroll
        for (int k = 0; k < D; ++k) z[k] = f2_zero();
        auto next_rows = [&] {
            if (has_next) copy_rows(row_next, i_next);
        };
        float2* gwe = (want_w && ok) ? gw2 + (size_t)e_cur * P * C2 + cp : nullptr;
        float sx = 0.f, sy = 0.f;  // dL/de_x, dL/de_y over this lane's channels
        static_for<0, L + 1>([&](auto l3c) {
            constexpr int l3 = decltype(l3c)::value;
            constexpr int d3 = 2 * l3 + 1;
            float2 y[d3];
#pragma unroll
            for (int m = 0; m < d3; ++m) y[m] = f2_zero();
            static_for<0, L + 1>([&](auto l1c) {
                constexpr int l1 = decltype(l1c)::value;
                if constexpr (has_type<L, O3>(l1, l3, 0) || has_type<L, O3>(l1, l3, 1)) {
                    float2 We[4], Wo[4];
                    group_weights<L, O3, l1, l3>(pp, next_rows, f.degenerate, We, Wo);
                    apply_M<L, O3, l1, l3>(We, Wo, xp + l1 * l1, y);
                    apply_MT<L, O3, l1, l3>(We, Wo, gp + l3 * l3, z + l1 * l1);
                    if (gwe) {
                        // products of the frame components coupled by B_p, symmetrised in +-mu
                        constexpr int mn = cmin(l1, l3);
                        float2 Pe[4], Po[4];
                        static_for<0, mn + 1>([&](auto mc) {
                            constexpr int mu = decltype(mc)::value;
                            const float2 a1 = gp[l3 * l3 + l3 + mu], a2 = gp[l3 * l3 + l3 - mu];
                            const float2 b1 = xp[l1 * l1 + l1 + mu], b2 = xp[l1 * l1 + l1 - mu];
                            if constexpr (mu == 0) {
                                Pe[0] = make_float2(a1.x * b1.x, a1.y * b1.y);
                                Po[0] = f2_zero();
                            } else {
                                Pe[mu] = make_float2(fmaf(a1.x, b1.x, a2.x * b2.x), fmaf(a1.y, b1.y, a2.y * b2.y));
                                Po[mu] = make_float2(fmaf(a1.x, b2.x, -a2.x * b1.x), fmaf(a1.y, b2.y, -a2.y * b1.y));
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
                                if (l2 > 0 && f.degenerate) gw = f2_zero();
                                st_stream2(gwe + p * C2, gw, pol_w);
                            }
                        });
                    }
                }
            });
            if (want_r) {
                sx += gen_form<l3, 0>(gp + l3 * l3, y);
                sy += gen_form<l3, 1>(gp + l3 * l3, y);
            }
        });
        static_for<0, L + 1>([&](auto l1c) {
            constexpr int l1 = decltype(l1c)::value;
            if (want_r) {
                sx += gen_form<l1, 0>(xp + l1 * l1, z + l1 * l1);
                sy += gen_form<l1, 1>(xp + l1 * l1, z + l1 * l1);
            }
            rotate<l1, true, true>(f, dbuf, z + l1 * l1, gx + l1 * l1);
        });
        if (want_r) {
            // sum over the team's lanes, then over the task's two slices (the block's two warps)
            for (int s = 1; s < G.T; s <<= 1) {
                sx += __shfl_xor_sync(G.tmask, sx, s);
                sy += __shfl_xor_sync(G.tmask, sy, s);
            }
            if (G.S == 2) {
                float* slot = comb + (it & 1) * 2;
                if (G.slice == 1 && G.tl == 0) {
                    slot[0] = sx;
                    slot[1] = sy;
                }
                __syncthreads();
                if (G.slice == 0) {
                    sx += slot[0];
                    sy += slot[1];
                }
            }
            if (ok && G.slice == 0 && G.tl == 0) {
                // grad_r = R^T (dL/de_y, -dL/de_x, 0) / |r|
                const float gu0 = sy * f.inv_rho, gu1 = -sx * f.inv_rho;
                float* gr = a.grad_r + 3 * (size_t)e_cur;
                gr[0] = f.R[0] * gu0 + f.R[3] * gu1;
                gr[1] = f.R[1] * gu0 + f.R[4] * gu1;
                gr[2] = f.R[2] * gu0 + f.R[5] * gu1;
            }
        }
        pp.edge_end(w_of(q + 2));
        e_cur = e_next;
        i_cur = i_next;
    }
    cp_async_wait_all();
    if (gx2) flush_row<D>(gx2 + (size_t)row * D * C2 + cp, C2, gx, row_lo >= k0 && row_hi <= k1);
}

namespace frame {
template <int L, bool O3>
constexpr size_t smem_bytes_for(int T, bool backward) {
    constexpr int D = (L + 1) * (L + 1);
    const int teams = kThreads / T;
    return sizeof(float) *
           (size_t)(kHeaderFloats + teams * team_floats(D, T, backward ? 2 : 1, Parts<L, O3>::ring_float2(T) / T));
}
}  // namespace frame

template <int L>
size_t smem_bytes(bool o3, int T, bool backward) {
    return o3 ? frame::smem_bytes_for<L, true>(T, backward) : frame::smem_bytes_for<L, false>(T, backward);
}

template <int L>
int blocks_per_sm(bool o3, bool backward, size_t smem) {
    int n = 0;
    const void* k;
    if (backward)
        k = o3 ? (const void*)etp_bwd_frame_kernel<L, true> : (const void*)etp_bwd_frame_kernel<L, false>;
    else
        k = o3 ? (const void*)etp_fwd_frame_kernel<L, true> : (const void*)etp_fwd_frame_kernel<L, false>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, 160 * 1024);
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k, frame::kThreads, smem) != cudaSuccess) n = 1;
    return n < 1 ? 1 : n;
}

template <int L>
cudaError_t launch_forward(bool o3, const FwdArgs& a, dim3 grid, size_t smem, cudaStream_t s) {
    if (o3)
        etp_fwd_frame_kernel<L, true><<<grid, frame::kThreads, smem, s>>>(a);
    else
        etp_fwd_frame_kernel<L, false><<<grid, frame::kThreads, smem, s>>>(a);
    return cudaGetLastError();
}

template <int L>
cudaError_t launch_backward(bool o3, const BwdArgs& a, dim3 grid, size_t smem, cudaStream_t s) {
    if (o3)
        etp_bwd_frame_kernel<L, true><<<grid, frame::kThreads, smem, s>>>(a);
    else
        etp_bwd_frame_kernel<L, false><<<grid, frame::kThreads, smem, s>>>(a);
    return cudaGetLastError();
}

}  // namespace etp
