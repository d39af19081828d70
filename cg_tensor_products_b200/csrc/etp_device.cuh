// Device building blocks shared by the kernels: compile-time path sets, a
// compile-time loop, the real spherical harmonics of a unit vector (used to fit
// the Wigner matrices of each edge frame) and the L2 evict-first cache policy.
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

template <class T>
__device__ __forceinline__ T sh_const(float c);
template <>
__device__ __forceinline__ float sh_const<float>(float c) { return c; }

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

// L2 policy for data touched exactly once (per-edge weights and their
// gradients): evict first, so that node features stay resident in L2.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
    uint64_t pol;
    asm("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
}  // namespace etp
