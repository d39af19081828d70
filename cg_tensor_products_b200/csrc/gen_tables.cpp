// Build-time generator of the real Clebsch-Gordan tables compiled into the kernels.
//
// Usage: gen_tables <output header>
//
// The pages call for Wigner 3-j / Clebsch-Gordan contraction coefficients held
// in compressed sparse form ("High-performance training and inference for deep
// equivariant interatomic potentials", section "제안 방법") and for
// Clebsch-Gordan tensor products of node irreps with edge spherical harmonics
// ("Machine Learning Interatomic Potentials: Advancing Open-Source Software ...",
// section "방법론 및 아키텍처", item 2). They print no coefficient, so this
// program computes them:
//
//   1. complex CG <l1 m1 l2 m2 | l3 m3> by Racah's closed formula (Condon-Shortley
//      phase), in long double;
//   2. change of basis to the real spherical harmonics of the kernels
//      (component normalisation, no Condon-Shortley phase, m = -l..l, cos for
//      m > 0, sin for m < 0):
//         Y_{l,m>0} = ((-1)^m Y_l^m + Y_l^-m) / sqrt2,   Y_{l,0} = Y_l^0,
//         Y_{l,-mu} = ((-1)^mu Y_l^mu - Y_l^-mu) / (i sqrt2);
//      with U that real<-complex matrix, the real coupling is
//         CG[m1,m2,m3] = sum U3[m3,M] <l1 mu1 l2 mu2|l3 M> conj(U1[m1,mu1]) conj(U2[m2,mu2]),
//      which is real or purely imaginary; the nonzero part is kept;
//   3. normalisation sum_{m1,m2} CG^2 = 1 for every m3, and the sign that makes
//      the first nonzero entry in lexicographic (m1, m2, m3) order positive;
//   4. entries below 1e-15 are exact zeros and are left out of the sparse list.
//
// The output header lists, for every (l1, l2, l3) with l <= kLmax on the SO(3)
// triangle, the nonzero entries (m1, m2, m3, value) with indices 0..2l.
#include <cmath>
#include <complex>
#include <cstdio>
#include <cstdlib>
#include <vector>

namespace {

constexpr int kLmax = 3;
using ld = long double;
using cld = std::complex<ld>;

ld fact(int n) {
    ld f = 1;
    for (int k = 2; k <= n; ++k) f *= k;
    return f;
}

// <j1 m1 j2 m2 | J M>, Racah's formula.
ld cg_complex(int j1, int m1, int j2, int m2, int J, int M) {
    if (m1 + m2 != M) return 0;
    if (std::abs(m1) > j1 || std::abs(m2) > j2 || std::abs(M) > J) return 0;
    if (J < std::abs(j1 - j2) || J > j1 + j2) return 0;
    ld pre = std::sqrt((2 * J + 1) * fact(J + j1 - j2) * fact(J - j1 + j2) * fact(j1 + j2 - J) /
                       fact(j1 + j2 + J + 1));
    pre *= std::sqrt(fact(J + M) * fact(J - M) * fact(j1 - m1) * fact(j1 + m1) * fact(j2 - m2) *
                     fact(j2 + m2));
    ld sum = 0;
    for (int k = 0; k <= j1 + j2 + J; ++k) {
        int a = j1 + j2 - J - k, b = j1 - m1 - k, c = j2 + m2 - k;
        int d = J - j2 + m1 + k, e = J - j1 - m2 + k;
        if (a < 0 || b < 0 || c < 0 || d < 0 || e < 0) continue;
        ld term = 1 / (fact(k) * fact(a) * fact(b) * fact(c) * fact(d) * fact(e));
        sum += (k % 2 ? -term : term);
    }
    return pre * sum;
}

// U[m][mu] (indices m + l, mu + l): real harmonic m as a combination of complex mu.
std::vector<cld> real_from_complex(int l) {
    int d = 2 * l + 1;
    std::vector<cld> U(d * d, cld(0, 0));
    const ld s = 1 / std::sqrt((ld)2);
    for (int m = -l; m <= l; ++m) {
        int r = m + l;
        if (m == 0) {
            U[r * d + l] = 1;
        } else if (m > 0) {
            U[r * d + (m + l)] = cld((m % 2 ? -s : s), 0);
            U[r * d + (-m + l)] = cld(s, 0);
        } else {
            int mu = -m;
            // ((-1)^mu Y^mu - Y^-mu) / (i sqrt2) = -i (-1)^mu s Y^mu + i s Y^-mu
            U[r * d + (mu + l)] = cld(0, (mu % 2 ? s : -s));
            U[r * d + (-mu + l)] = cld(0, s);
        }
    }
    return U;
}

struct Nz {
    int m1, m2, m3;
    ld v;
};

std::vector<Nz> real_cg(int l1, int l2, int l3) {
    std::vector<Nz> out;
    if (l3 < std::abs(l1 - l2) || l3 > l1 + l2) return out;
    int d1 = 2 * l1 + 1, d2 = 2 * l2 + 1, d3 = 2 * l3 + 1;
    auto U1 = real_from_complex(l1), U2 = real_from_complex(l2), U3 = real_from_complex(l3);
    std::vector<cld> T(d1 * d2 * d3, cld(0, 0));
    for (int a = 0; a < d1; ++a)
        for (int b = 0; b < d2; ++b)
            for (int c = 0; c < d3; ++c) {
                cld acc(0, 0);
                for (int mu1 = -l1; mu1 <= l1; ++mu1)
                    for (int mu2 = -l2; mu2 <= l2; ++mu2) {
                        int M = mu1 + mu2;
                        if (std::abs(M) > l3) continue;
                        ld cc = cg_complex(l1, mu1, l2, mu2, l3, M);
                        if (cc == 0) continue;
                        acc += U3[c * d3 + (M + l3)] * cc * std::conj(U1[a * d1 + (mu1 + l1)]) *
                               std::conj(U2[b * d2 + (mu2 + l2)]);
                    }
                T[(a * d2 + b) * d3 + c] = acc;
            }
    ld re = 0, im = 0;
    for (auto& z : T) {
        re += z.real() * z.real();
        im += z.imag() * z.imag();
    }
    bool use_re = re >= im;
    ld other = use_re ? im : re, main = use_re ? re : im;
    if (other > 1e-24L * main) {
        std::fprintf(stderr, "coupling (%d,%d,%d) is not real up to a phase\n", l1, l2, l3);
        std::exit(1);
    }
    std::vector<ld> V(T.size());
    for (size_t k = 0; k < T.size(); ++k) V[k] = use_re ? T[k].real() : T[k].imag();
    // normalisation per m3
    for (int c = 0; c < d3; ++c) {
        ld n2 = 0;
        for (int a = 0; a < d1; ++a)
            for (int b = 0; b < d2; ++b) n2 += V[(a * d2 + b) * d3 + c] * V[(a * d2 + b) * d3 + c];
        if (std::fabs(n2 - main / d3) > 1e-15L * main) {
            std::fprintf(stderr, "coupling (%d,%d,%d) is not an isometry\n", l1, l2, l3);
            std::exit(1);
        }
    }
    ld scale = 1 / std::sqrt(main / d3);
    ld first = 0;
    for (auto v : V)
        if (std::fabs(v * scale) > 1e-15L) {
            first = v;
            break;
        }
    if (first < 0) scale = -scale;
    for (int a = 0; a < d1; ++a)
        for (int b = 0; b < d2; ++b)
            for (int c = 0; c < d3; ++c) {
                ld v = V[(a * d2 + b) * d3 + c] * scale;
                if (std::fabs(v) > 1e-15L) out.push_back({a, b, c, v});
            }
    return out;
}

}  // namespace

int main(int argc, char** argv) {
    if (argc != 2) {
        std::fprintf(stderr, "usage: %s <output header>\n", argv[0]);
        return 2;
    }
    FILE* f = std::fopen(argv[1], "w");
    if (!f) return 1;
    std::fprintf(f, "// Generated by gen_tables.cpp at build time. Do not edit.\n");
    std::fprintf(f, "// Real Clebsch-Gordan couplings (Racah formula, complex-to-real basis change),\n");
    std::fprintf(f, "// normalised per m3, first nonzero entry positive; zeros omitted.\n");
    std::fprintf(f, "#pragma once\n\nnamespace etp_gen {\n\n");
    std::fprintf(f, "constexpr int kLmax = %d;\n\n", kLmax);
    std::fprintf(f, "struct CgNz {\n    int m1, m2, m3;\n    double v;\n};\n\n");
    int off[kLmax + 1][kLmax + 1][kLmax + 1], cnt[kLmax + 1][kLmax + 1][kLmax + 1];
    std::vector<Nz> all;
    for (int a = 0; a <= kLmax; ++a)
        for (int b = 0; b <= kLmax; ++b)
            for (int c = 0; c <= kLmax; ++c) {
                auto v = real_cg(a, b, c);
                off[a][b][c] = (int)all.size();
                cnt[a][b][c] = (int)v.size();
                all.insert(all.end(), v.begin(), v.end());
            }
    std::fprintf(f, "constexpr int kCgTotal = %d;\n\n", (int)all.size());
    std::fprintf(f, "constexpr CgNz kCg[kCgTotal] = {\n");
    for (auto& z : all) std::fprintf(f, "    {%d, %d, %d, %.21Lg},\n", z.m1, z.m2, z.m3, z.v);
    std::fprintf(f, "};\n\n");
    for (int pass = 0; pass < 2; ++pass) {
        std::fprintf(f, "constexpr int %s[%d][%d][%d] = {\n", pass ? "kCgCnt" : "kCgOff", kLmax + 1,
                     kLmax + 1, kLmax + 1);
        for (int a = 0; a <= kLmax; ++a) {
            std::fprintf(f, "    {");
            for (int b = 0; b <= kLmax; ++b) {
                std::fprintf(f, "{");
                for (int c = 0; c <= kLmax; ++c)
                    std::fprintf(f, "%d%s", pass ? cnt[a][b][c] : off[a][b][c], c < kLmax ? ", " : "");
                std::fprintf(f, "}%s", b < kLmax ? ", " : "");
            }
            std::fprintf(f, "},\n");
        }
        std::fprintf(f, "};\n\n");
    }
    std::fprintf(f, "}  // namespace etp_gen\n");
    std::fclose(f);
    return 0;
}
