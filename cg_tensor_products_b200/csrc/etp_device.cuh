// Device building blocks shared by the forward and backward kernels: compile-time
// path sets and coupling lists, a compile-time loop, and the real spherical
// harmonics of an edge vector (values, and values with their r-derivative).
#pragma once

#include <cuda_runtime.h>

#include <cstdint>
#include <type_traits>
#include <utility>

#include "generated/etp_tables.h"

namespace etp {

// ---------------------------------------------------------------------------
// compile-time loop: f(std::integral_constant<int, i>) for i in [Begin, End)
template <int Off, class F, int... I>
__host__ __device__ __forceinline__ void static_for_impl(F&& f, std::integer_sequence<int, I...>) {
    (f(std::integral_constant<int, Off + I>{}), ...);
}
template <int Begin, int End, class F>
__host__ __device__ __forceinline__ void static_for(F&& f) {
    if constexpr (End > Begin) static_for_impl<Begin>(f, std::make_integer_sequence<int, End - Begin>{});
}

// ---------------------------------------------------------------------------
// Paths (l1, l2, l3) of the tensor product of irreps 0..L with harmonics 0..L
// into irreps 0..L: the SO(3) triangle rule, and with O3 also l1+l2+l3 even
// (natural parities). Lexicographic order.
struct Path {
    int l1, l2, l3;
};

template <int L, bool O3>
struct PathSet {
    static constexpr bool allowed(int a, int b, int c) {
        return c >= (a > b ? a - b : b - a) && c <= a + b && (!O3 || (a + b + c) % 2 == 0);
    }
    static constexpr int count() {
        int n = 0;
        for (int a = 0; a <= L; ++a)
            for (int b = 0; b <= L; ++b)
                for (int c = 0; c <= L; ++c) n += allowed(a, b, c) ? 1 : 0;
        return n;
    }
    static constexpr int P = count();
    static constexpr Path path(int p) {
        int n = 0;
        for (int a = 0; a <= L; ++a)
            for (int b = 0; b <= L; ++b)
                for (int c = 0; c <= L; ++c)
                    if (allowed(a, b, c)) {
                        if (n == p) return Path{a, b, c};
                        ++n;
                    }
        return Path{-1, -1, -1};
    }
    static constexpr int D = (L + 1) * (L + 1);
};

// ---------------------------------------------------------------------------
// compile-time square root (Newton's iteration in double), for normalisation
// constants only
constexpr double csqrt(double x) {
    if (x <= 0) return 0;
    double g = x > 1 ? x : 1;
    for (int i = 0; i < 100; ++i) g = 0.5 * (g + x / g);
    return g;
}
constexpr double cfact(int n) { return n <= 1 ? 1.0 : n * cfact(n - 1); }
constexpr double dfact(int n) { return n <= 1 ? 1.0 : n * dfact(n - 2); }  // n!!
// K_lm = sqrt((2l+1) (l-m)!/(l+m)!) * (sqrt2 if m > 0)
constexpr double sh_norm(int l, int m) {
    return csqrt((2.0 * l + 1.0) * cfact(l - m) / cfact(l + m)) * (m > 0 ? csqrt(2.0) : 1.0);
}

// Forward-mode dual number: a value and its derivative along the 3 edge-vector axes.
struct Dual3 {
    float v, d0, d1, d2;
};
__device__ __forceinline__ Dual3 operator+(Dual3 a, Dual3 b) { return {a.v + b.v, a.d0 + b.d0, a.d1 + b.d1, a.d2 + b.d2}; }
__device__ __forceinline__ Dual3 operator-(Dual3 a, Dual3 b) { return {a.v - b.v, a.d0 - b.d0, a.d1 - b.d1, a.d2 - b.d2}; }
__device__ __forceinline__ Dual3 operator*(Dual3 a, Dual3 b) {
    return {a.v * b.v, a.d0 * b.v + a.v * b.d0, a.d1 * b.v + a.v * b.d1, a.d2 * b.v + a.v * b.d2};
}
__device__ __forceinline__ Dual3 operator*(float s, Dual3 a) { return {s * a.v, s * a.d0, s * a.d1, s * a.d2}; }
template <class T>
__device__ __forceinline__ T sh_const(float c);
template <>
__device__ __forceinline__ float sh_const<float>(float c) { return c; }
template <>
__device__ __forceinline__ Dual3 sh_const<Dual3>(float c) { return {c, 0.f, 0.f, 0.f}; }

// Real spherical harmonics of a unit vector u, blocks l = 0..L, m = -l..l:
//   Y_lm = K_lm * Pi_l^|m|(u_z) * {Re (u_x + i u_y)^m (m > 0), 1 (m = 0), Im (u_x + i u_y)^|m| (m < 0)}
// with Pi_l^m = d^m P_l / dz^m from the three-term recurrence
//   Pi_m^m = (2m-1)!!,  Pi_{m+1}^m = (2m+1) z Pi_m^m,
//   (l-m) Pi_l^m = (2l-1) z Pi_{l-1}^m - (l+m-1) Pi_{l-2}^m,
// and (u_x + i u_y)^m by repeated complex multiplication.
template <int L, class T>
__device__ __forceinline__ void sh_unit(T ux, T uy, T uz, T (&Y)[(L + 1) * (L + 1)]) {
    T Cm[L + 1], Sm[L + 1];
    Cm[0] = sh_const<T>(1.f);
    Sm[0] = sh_const<T>(0.f);
#pragma unroll
    for (int m = 1; m <= L; ++m) {
        Cm[m] = ux * Cm[m - 1] - uy * Sm[m - 1];
        Sm[m] = ux * Sm[m - 1] + uy * Cm[m - 1];
    }
    T Pi[L + 1][L + 1];
    static_for<0, L + 1>([&](auto mc) {
        constexpr int m = decltype(mc)::value;
        Pi[m][m] = sh_const<T>((float)dfact(2 * m - 1));
        if constexpr (m + 1 <= L) Pi[m + 1][m] = (float)(2 * m + 1) * (uz * Pi[m][m]);
        static_for<m + 2, L + 1>([&](auto lc) {
            constexpr int l = decltype(lc)::value;
            constexpr float a = (float)((2.0 * l - 1.0) / (l - m));
            constexpr float b = (float)((l + m - 1.0) / (l - m));
            Pi[l][m] = a * (uz * Pi[l - 1][m]) - b * Pi[l - 2][m];
        });
    });
    static_for<0, L + 1>([&](auto lc) {
        constexpr int l = decltype(lc)::value;
        static_for<-l, l + 1>([&](auto mc) {
            constexpr int m = decltype(mc)::value;
            constexpr int mu = m < 0 ? -m : m;
            constexpr float k = (float)sh_norm(l, mu);
            if constexpr (m == 0)
                Y[l * l + l] = k * Pi[l][0];
            else if constexpr (m > 0)
                Y[l * l + l + m] = k * (Pi[l][mu] * Cm[mu]);
            else
                Y[l * l + l + m] = k * (Pi[l][mu] * Sm[mu]);
        });
    });
}

// Y_lm(r / |r|) for all l <= L; |r| < 1e-12 gives Y_0 = 1 and the rest 0.
template <int L>
__device__ __forceinline__ void sh_eval(float rx, float ry, float rz, float (&Y)[(L + 1) * (L + 1)]) {
    float n2 = rx * rx + ry * ry + rz * rz;
    bool ok = n2 >= 1e-24f;
    float inv = ok ? rsqrtf(n2) : 0.f;
    sh_unit<L, float>(rx * inv, ry * inv, rz * inv, Y);
    if (!ok) {
#pragma unroll
        for (int k = 1; k < (L + 1) * (L + 1); ++k) Y[k] = 0.f;
    }
}

// dY_lm/dr (3 components each) for the unnormalised edge vector r: the
// harmonics are evaluated on dual numbers seeded with du/dr = (I - u u^T)/|r|.
template <int L>
__device__ __forceinline__ void sh_eval_grad(float rx, float ry, float rz, float (&Y)[(L + 1) * (L + 1)],
                                             float (&dY)[(L + 1) * (L + 1)][3]) {
    constexpr int D = (L + 1) * (L + 1);
    float n2 = rx * rx + ry * ry + rz * rz;
    bool ok = n2 >= 1e-24f;
    float inv = ok ? rsqrtf(n2) : 0.f;
    float ux = rx * inv, uy = ry * inv, uz = rz * inv;
    Dual3 dx{ux, (1.f - ux * ux) * inv, -ux * uy * inv, -ux * uz * inv};
    Dual3 dy{uy, -uy * ux * inv, (1.f - uy * uy) * inv, -uy * uz * inv};
    Dual3 dz{uz, -uz * ux * inv, -uz * uy * inv, (1.f - uz * uz) * inv};
    Dual3 Yd[D];
    sh_unit<L, Dual3>(dx, dy, dz, Yd);
#pragma unroll
    for (int k = 0; k < D; ++k) {
        bool keep = ok || k == 0;
        Y[k] = keep ? Yd[k].v : 0.f;
        dY[k][0] = ok ? Yd[k].d0 : 0.f;
        dY[k][1] = ok ? Yd[k].d1 : 0.f;
        dY[k][2] = ok ? Yd[k].d2 : 0.f;
    }
}

// ---------------------------------------------------------------------------
// float4 helpers
__device__ __forceinline__ float4 f4_zero() { return make_float4(0.f, 0.f, 0.f, 0.f); }
__device__ __forceinline__ void f4_fma(float4& acc, float s, float4 v) {
    acc.x = fmaf(s, v.x, acc.x);
    acc.y = fmaf(s, v.y, acc.y);
    acc.z = fmaf(s, v.z, acc.z);
    acc.w = fmaf(s, v.w, acc.w);
}
__device__ __forceinline__ void f4_fma(float4& acc, float4 a, float4 b) {
    acc.x = fmaf(a.x, b.x, acc.x);
    acc.y = fmaf(a.y, b.y, acc.y);
    acc.z = fmaf(a.z, b.z, acc.z);
    acc.w = fmaf(a.w, b.w, acc.w);
}
__device__ __forceinline__ float4 f4_mul(float4 a, float4 b) {
    return make_float4(a.x * b.x, a.y * b.y, a.z * b.z, a.w * b.w);
}
__device__ __forceinline__ float f4_dot(float4 a, float4 b) {
    return fmaf(a.w, b.w, fmaf(a.z, b.z, fmaf(a.y, b.y, a.x * b.x)));
}

// L2 policy for data touched exactly once (per-edge weights and their
// gradients): evict first, so that node features stay resident in L2.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
    uint64_t pol;
    asm("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
// Streaming load: no L1 allocation, L2 evict-first.
__device__ __forceinline__ float4 ld_stream(const float4* p, uint64_t pol) {
    float4 v;
    asm("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.f32 {%0, %1, %2, %3}, [%4], %5;"
        : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
        : "l"(p), "l"(pol));
    return v;
}
// Streaming store: L2 evict-first.
__device__ __forceinline__ void st_stream(float4* p, float4 v, uint64_t pol) {
    asm volatile("st.global.L2::cache_hint.v4.f32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(p), "f"(v.x), "f"(v.y),
                 "f"(v.z), "f"(v.w), "l"(pol)
                 : "memory");
}

}  // namespace etp
