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
//
// It also writes the tables of the edge-aligned frame used by the kernels. For
// an edge with unit vector u, a rotation R with R u = z maps the harmonics to
// Y(z) = sqrt(2l+1) delta_{m,0}; by the equivariance of every coupling,
//   CG_p(x, Y(u)) = D_l3(R)^T B_p D_l1(R) x,   B_p[m3, m1] = sqrt(2 l2 + 1) CG_p[m1, 0, m3],
// and B_p is nonzero only at m1 = m3 (l1+l2+l3 even) or m1 = -m3 (odd), with
// B_p[m, m] = B_p[-m, -m] = b_p(|m|) (even) or B_p[mu, -mu] = -B_p[-mu, mu] = b_p(mu)
// (odd). Written: b_p(mu) for mu = 0..min(l1, l3); the real-basis rotation
// generators J_x, J_y (d/de Y(exp(e [a]x) r) = J_a Y(r)), obtained from the
// Condon-Shortley ladder operators, (a x r).grad = i a.L, L_+- Y^m =
// sqrt((l -+ m)(l +- m + 1)) Y^(m+-1), through the same change of basis; and, for
// the Wigner matrices D_l(R) (Y_l(R r) = D_l(R) Y_l(r)), 7 fixed unit vectors p_k
// and A_l^-1 with A_l = [Y_l(p_1) .. Y_l(p_2l+1)], so that
// D_l(R) = [Y_l(R p_1) .. Y_l(R p_2l+1)] A_l^-1.
#include <cmath>
#include <complex>
#include <cstdio>
#include <cstdlib>
#include <algorithm>
#include <functional>
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

// ---------------------------------------------------------------------------
// Real spherical harmonics of a unit vector (component normalisation, no
// Condon-Shortley phase), long double: Y_lm = K_lm Pi_l^|m|(z) {Re,1,Im}(x+iy)^|m|.
std::vector<ld> real_sh(int L, ld x, ld y, ld z) {
    std::vector<ld> Y((L + 1) * (L + 1));
    std::vector<ld> Cm(L + 1), Sm(L + 1);
    Cm[0] = 1;
    Sm[0] = 0;
    for (int m = 1; m <= L; ++m) {
        Cm[m] = x * Cm[m - 1] - y * Sm[m - 1];
        Sm[m] = x * Sm[m - 1] + y * Cm[m - 1];
    }
    std::vector<std::vector<ld>> Pi(L + 1, std::vector<ld>(L + 1, 0));
    for (int m = 0; m <= L; ++m) {
        ld df = 1;
        for (int k = 2 * m - 1; k > 1; k -= 2) df *= k;
        Pi[m][m] = df;
        if (m + 1 <= L) Pi[m + 1][m] = (2 * m + 1) * z * Pi[m][m];
        for (int l = m + 2; l <= L; ++l) Pi[l][m] = ((2 * l - 1) * z * Pi[l - 1][m] - (l + m - 1) * Pi[l - 2][m]) / (l - m);
    }
    for (int l = 0; l <= L; ++l)
        for (int m = -l; m <= l; ++m) {
            int mu = std::abs(m);
            ld k = std::sqrt((2 * l + 1) * fact(l - mu) / fact(l + mu)) * (mu ? std::sqrt((ld)2) : 1);
            ld az = m > 0 ? Cm[mu] : (m < 0 ? Sm[mu] : 1);
            Y[l * l + l + m] = k * Pi[l][mu] * az;
        }
    return Y;
}

// Gauss-Jordan inverse with partial pivoting (n <= 7).
bool invert(std::vector<ld>& A, int n) {
    std::vector<ld> I(n * n, 0);
    for (int i = 0; i < n; ++i) I[i * n + i] = 1;
    for (int c = 0; c < n; ++c) {
        int piv = c;
        for (int r = c + 1; r < n; ++r)
            if (std::fabs(A[r * n + c]) > std::fabs(A[piv * n + c])) piv = r;
        if (std::fabs(A[piv * n + c]) < 1e-12L) return false;
        for (int k = 0; k < n; ++k) {
            std::swap(A[c * n + k], A[piv * n + k]);
            std::swap(I[c * n + k], I[piv * n + k]);
        }
        ld d = A[c * n + c];
        for (int k = 0; k < n; ++k) {
            A[c * n + k] /= d;
            I[c * n + k] /= d;
        }
        for (int r = 0; r < n; ++r)
            if (r != c) {
                ld f = A[r * n + c];
                for (int k = 0; k < n; ++k) {
                    A[r * n + k] -= f * A[c * n + k];
                    I[r * n + k] -= f * I[c * n + k];
                }
            }
    }
    A = I;
    return true;
}

// Real-basis generator J_a (a = 0: x, 1: y) of degree l: U J^C U^dagger with
// J^C_x[m, m+-1] = (i/2) c_+-(m), J^C_y[m, m+1] = c_+(m)/2, J^C_y[m, m-1] = -c_-(m)/2.
std::vector<ld> real_generator(int l, int axis) {
    int d = 2 * l + 1;
    std::vector<cld> Jc(d * d, cld(0, 0));
    for (int m = -l; m <= l; ++m) {
        ld cp = std::sqrt((ld)(l - m) * (l + m + 1)), cm = std::sqrt((ld)(l + m) * (l - m + 1));
        if (m + 1 <= l) Jc[(m + l) * d + (m + 1 + l)] = axis == 0 ? cld(0, cp / 2) : cld(cp / 2, 0);
        if (m - 1 >= -l) Jc[(m + l) * d + (m - 1 + l)] = axis == 0 ? cld(0, cm / 2) : cld(-cm / 2, 0);
    }
    auto U = real_from_complex(l);
    std::vector<ld> J(d * d);
    for (int a = 0; a < d; ++a)
        for (int b = 0; b < d; ++b) {
            cld acc(0, 0);
            for (int i = 0; i < d; ++i)
                for (int j = 0; j < d; ++j) acc += U[a * d + i] * Jc[i * d + j] * std::conj(U[b * d + j]);
            if (std::fabs(acc.imag()) > 1e-15L) {
                std::fprintf(stderr, "generator l=%d axis=%d is not real\n", l, axis);
                std::exit(1);
            }
            J[a * d + b] = std::fabs(acc.real()) < 1e-15L ? 0 : acc.real();
        }
    for (int a = 0; a < d; ++a)
        for (int b = 0; b < d; ++b)
            if (std::fabs(J[a * d + b] + J[b * d + a]) > 1e-15L) {
                std::fprintf(stderr, "generator l=%d axis=%d is not antisymmetric\n", l, axis);
                std::exit(1);
            }
    return J;
}

// ---------------------------------------------------------------------------
// Cartesian couplings in independent components. A symmetric traceless (STF)
// tensor of rank l is held by its 2l + 1 entries with at most one z index,
// ordered (x^l, x^(l-1) y, .., y^l, x^(l-1) z, .., y^(l-1) z) by the counts (a, b, c)
// of x, y, z indices; the other entries follow from tracelessness,
// T(a, b, c) = -T(a + 2, b, c - 2) - T(a, b + 2, c - 2). The path (l1, l2 -> l3)
// contracts the last k indices of the first operand with the first k of the
// second, k = (l1 + l2 - l3 - odd) / 2 with odd = (l1 + l2 + l3) mod 2; when odd,
// the first operand's last free index and the second's first free index go
// through the Levi-Civita symbol into a new last index; the STF part of the l3
// remaining indices is the result, with no normalisation constant. In
// independent components the coupling is a sparse tensor Cc[i1][i2][i3].
struct Cnt3 {
    int a, b, c;
};
std::vector<Cnt3> compact_counts(int l) {
    std::vector<Cnt3> v;
    for (int b = 0; b <= l; ++b) v.push_back({l - b, b, 0});
    for (int b = 0; b + 1 <= l; ++b) v.push_back({l - 1 - b, b, 1});
    return v;
}
int ipow3(int l) {
    int n = 1;
    for (int k = 0; k < l; ++k) n *= 3;
    return n;
}
// digits of full index t (rank l, first index most significant)
std::vector<int> digits(int t, int l) {
    std::vector<int> d(l);
    for (int k = l - 1; k >= 0; --k) {
        d[k] = t % 3;
        t /= 3;
    }
    return d;
}
Cnt3 counts_of(const std::vector<int>& d) {
    Cnt3 c{0, 0, 0};
    for (int v : d) (v == 0 ? c.a : (v == 1 ? c.b : c.c))++;
    return c;
}
// full STF tensor of rank l from independent components
std::vector<ld> stf_expand(int l, const std::vector<ld>& comp) {
    auto cc = compact_counts(l);
    std::function<ld(int, int, int)> T = [&](int a, int b, int c) -> ld {
        if (c <= 1) {
            for (size_t i = 0; i < cc.size(); ++i)
                if (cc[i].a == a && cc[i].b == b && cc[i].c == c) return comp[i];
            return 0;
        }
        return -T(a + 2, b, c - 2) - T(a, b + 2, c - 2);
    };
    std::vector<ld> full(ipow3(l));
    for (int t = 0; t < ipow3(l); ++t) {
        Cnt3 c = counts_of(digits(t, l));
        full[t] = l == 0 ? comp[0] : T(c.a, c.b, c.c);
    }
    return full;
}
// STF projection of a rank-l tensor (l <= 3)
std::vector<ld> stf_project(int l, const std::vector<ld>& T) {
    if (l <= 1) return T;
    const int n = ipow3(l);
    std::vector<ld> S(n, 0);
    for (int t = 0; t < n; ++t) {  // symmetrise: average over index permutations
        auto d = digits(t, l);
        std::vector<int> perm(l);
        for (int k = 0; k < l; ++k) perm[k] = k;
        int np = 0;
        ld acc = 0;
        do {
            int u = 0;
            for (int k = 0; k < l; ++k) u = u * 3 + d[perm[k]];
            acc += T[u];
            ++np;
        } while (std::next_permutation(perm.begin(), perm.end()));
        S[t] = acc / np;
    }
    std::vector<ld> out(S);
    if (l == 2) {
        const ld tr = (S[0] + S[4] + S[8]) / 3;
        for (int i = 0; i < 3; ++i) out[i * 3 + i] -= tr;
    } else {  // l == 3: S_ijk - (delta_ij t_k + delta_ik t_j + delta_jk t_i) / 5, t_k = S_llk
        ld tv[3];
        for (int k = 0; k < 3; ++k) tv[k] = S[(0 * 3 + 0) * 3 + k] + S[(1 * 3 + 1) * 3 + k] + S[(2 * 3 + 2) * 3 + k];
        for (int i = 0; i < 3; ++i)
            for (int j = 0; j < 3; ++j)
                for (int k = 0; k < 3; ++k) {
                    ld v = 0;
                    if (i == j) v += tv[k];
                    if (i == k) v += tv[j];
                    if (j == k) v += tv[i];
                    out[(i * 3 + j) * 3 + k] -= v / 5;
                }
    }
    return out;
}
ld levi(int a, int b, int c) {
    if (a == b || b == c || a == c) return 0;
    return ((a + 1) % 3 == b) ? 1 : -1;  // cyclic (0 1 2), (1 2 0), (2 0 1): +1
}
// the path's contraction of full tensors A (rank l1) and B (rank l2), before STF
std::vector<ld> cart_contract(int l1, int l2, int l3, const std::vector<ld>& A, const std::vector<ld>& B) {
    const int odd = (l1 + l2 + l3) % 2, k = (l1 + l2 - l3 - odd) / 2;
    std::vector<ld> out(ipow3(l3), 0);
    for (int ta = 0; ta < ipow3(l1); ++ta) {
        if (A[ta] == 0) continue;
        auto da = digits(ta, l1);
        for (int tb = 0; tb < ipow3(l2); ++tb) {
            if (B[tb] == 0) continue;
            auto db = digits(tb, l2);
            bool match = true;
            for (int t = 0; t < k && match; ++t) match = da[l1 - k + t] == db[t];
            if (!match) continue;
            std::vector<int> fa(da.begin(), da.begin() + (l1 - k)), fb(db.begin() + k, db.end());
            const ld ab = A[ta] * B[tb];
            if (!odd) {
                int u = 0;
                for (int v : fa) u = u * 3 + v;
                for (int v : fb) u = u * 3 + v;
                out[u] += ab;
            } else {
                for (int n = 0; n < 3; ++n) {
                    const ld e = levi(fa.back(), fb.front(), n);
                    if (e == 0) continue;
                    int u = 0;
                    for (size_t q = 0; q + 1 < fa.size(); ++q) u = u * 3 + fa[q];
                    for (size_t q = 1; q < fb.size(); ++q) u = u * 3 + fb[q];
                    u = u * 3 + n;
                    out[u] += e * ab;
                }
            }
        }
    }
    return out;
}
std::vector<Nz> cart_coupling(int l1, int l2, int l3) {
    std::vector<Nz> out;
    if (l3 < std::abs(l1 - l2) || l3 > l1 + l2) return out;
    const int d1 = 2 * l1 + 1, d2 = 2 * l2 + 1;
    auto c3 = compact_counts(l3);
    for (int i1 = 0; i1 < d1; ++i1)
        for (int i2 = 0; i2 < d2; ++i2) {
            std::vector<ld> e1(d1, 0), e2(d2, 0);
            e1[i1] = 1;
            e2[i2] = 1;
            auto R = stf_project(l3, cart_contract(l1, l2, l3, stf_expand(l1, e1), stf_expand(l2, e2)));
            for (int i3 = 0; i3 < 2 * l3 + 1; ++i3) {
                ld v;
                if (l3 == 0) {
                    v = R[0];
                } else {
                    int u = 0;
                    for (int q = 0; q < c3[i3].a; ++q) u = u * 3 + 0;
                    for (int q = 0; q < c3[i3].b; ++q) u = u * 3 + 1;
                    for (int q = 0; q < c3[i3].c; ++q) u = u * 3 + 2;
                    v = R[u];
                }
                if (std::fabs(v) > 1e-15L) out.push_back({i1, i2, i3, v});
            }
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
    // --- edge-aligned frame: b_p(mu) --------------------------------------
    std::fprintf(f, "// b[l1][l2][l3][mu]: the m2 = 0 slice of the coupling in the edge frame (see gen_tables.cpp)\n");
    std::fprintf(f, "constexpr double kFrameB[%d][%d][%d][%d] = {\n", kLmax + 1, kLmax + 1, kLmax + 1, kLmax + 1);
    for (int a = 0; a <= kLmax; ++a) {
        std::fprintf(f, "    {");
        for (int b = 0; b <= kLmax; ++b) {
            std::fprintf(f, "{");
            for (int c = 0; c <= kLmax; ++c) {
                std::vector<ld> dense((2 * a + 1) * (2 * b + 1) * (2 * c + 1), 0);
                int d2 = 2 * b + 1, d3 = 2 * c + 1;
                for (auto& z : real_cg(a, b, c)) dense[(z.m1 * d2 + z.m2) * d3 + z.m3] = z.v;
                auto at = [&](int m1, int m3) { return dense[((m1 + a) * d2 + b) * d3 + (m3 + c)] * std::sqrt((ld)(2 * b + 1)); };
                const bool odd = (a + b + c) % 2 == 1;
                const int mn = a < c ? a : c;
                // structure check: B nonzero only at m1 = +-m3 with the stated symmetry
                for (int m1 = -a; m1 <= a; ++m1)
                    for (int m3 = -c; m3 <= c; ++m3) {
                        ld v = at(m1, m3);
                        bool allowed = odd ? (m1 == -m3 && m3 != 0) : (m1 == m3);
                        if (!allowed && std::fabs(v) > 1e-15L) {
                            std::fprintf(stderr, "frame coupling (%d,%d,%d) has an entry off its pattern\n", a, b, c);
                            return 1;
                        }
                    }
                std::fprintf(f, "{");
                for (int mu = 0; mu <= kLmax; ++mu) {
                    ld v = 0;
                    if (mu <= mn && !(c < std::abs(a - b) || c > a + b)) {
                        if (!odd) {
                            v = at(mu, mu);
                            if (std::fabs(at(-mu, -mu) - v) > 1e-15L) { std::fprintf(stderr, "even symmetry\n"); return 1; }
                        } else if (mu > 0) {
                            v = at(-mu, mu);
                            if (std::fabs(at(mu, -mu) + v) > 1e-15L) { std::fprintf(stderr, "odd symmetry\n"); return 1; }
                        }
                    }
                    std::fprintf(f, "%.21Lg%s", v, mu < kLmax ? ", " : "");
                }
                std::fprintf(f, "}%s", c < kLmax ? ", " : "");
            }
            std::fprintf(f, "}%s", b < kLmax ? ", " : "");
        }
        std::fprintf(f, "},\n");
    }
    std::fprintf(f, "};\n\n");
    // --- generators J_x, J_y -------------------------------------------------
    std::fprintf(f, "// kGen[axis][l][a][b]: real-basis rotation generators (axis 0: x, 1: y), d/de Y(exp(e[a]x) r) = J Y(r)\n");
    std::fprintf(f, "constexpr double kGen[2][%d][7][7] = {\n", kLmax + 1);
    for (int ax = 0; ax < 2; ++ax) {
        std::fprintf(f, "    {");
        for (int l = 0; l <= kLmax; ++l) {
            auto J = real_generator(l, ax);
            int d = 2 * l + 1;
            std::fprintf(f, "{");
            for (int a = 0; a < 7; ++a) {
                std::fprintf(f, "{");
                for (int b = 0; b < 7; ++b) std::fprintf(f, "%.21Lg%s", (a < d && b < d) ? J[a * d + b] : (ld)0, b < 6 ? ", " : "");
                std::fprintf(f, "}%s", a < 6 ? ", " : "");
            }
            std::fprintf(f, "}%s", l < kLmax ? ", " : "");
        }
        std::fprintf(f, "},\n");
    }
    std::fprintf(f, "};\n\n");
    // --- Wigner fitting points and inverses ---------------------------------
    {
        unsigned long long st = 0x9E3779B97F4A7C15ull;
        auto uni = [&]() {
            st = st * 6364136223846793005ull + 1442695040888963407ull;
            return (ld)((st >> 11) & ((1ull << 53) - 1)) / (ld)(1ull << 53);
        };
        ld best = 1e300L;
        std::vector<ld> best_pts, best_inv[kLmax + 1];
        for (int trial = 0; trial < 4000; ++trial) {
            std::vector<ld> pts(3 * 7);
            for (int k = 0; k < 7; ++k) {
                ld zz = 2 * uni() - 1, ph = 2 * 3.14159265358979323846264338327950288L * uni();
                ld rr = std::sqrt(1 - zz * zz);
                pts[3 * k] = rr * std::cos(ph);
                pts[3 * k + 1] = rr * std::sin(ph);
                pts[3 * k + 2] = zz;
            }
            ld worst = 0;
            std::vector<ld> inv[kLmax + 1];
            bool ok = true;
            for (int l = 2; l <= kLmax && ok; ++l) {
                int d = 2 * l + 1;
                std::vector<ld> A(d * d);
                for (int k = 0; k < d; ++k) {
                    auto Y = real_sh(l, pts[3 * k], pts[3 * k + 1], pts[3 * k + 2]);
                    for (int m = 0; m < d; ++m) A[m * d + k] = Y[l * l + m];  // column k = Y_l(p_k)
                }
                ld na = 0;
                for (auto v : A) na += v * v;
                std::vector<ld> Ai = A;
                if (!invert(Ai, d)) { ok = false; break; }
                ld ni = 0;
                for (auto v : Ai) ni += v * v;
                ld cond = std::sqrt(na * ni);
                if (cond > worst) worst = cond;
                inv[l] = Ai;
            }
            if (ok && worst < best) {
                best = worst;
                best_pts = pts;
                for (int l = 2; l <= kLmax; ++l) best_inv[l] = inv[l];
            }
        }
        std::fprintf(f, "// Wigner matrices by fitting: D_l(R) = [Y_l(R p_1) .. Y_l(R p_2l+1)] A_l^-1 (Frobenius condition %.3Lf)\n", best);
        std::fprintf(f, "constexpr double kFitPoints[7][3] = {\n");
        for (int k = 0; k < 7; ++k)
            std::fprintf(f, "    {%.21Lg, %.21Lg, %.21Lg},\n", best_pts[3 * k], best_pts[3 * k + 1], best_pts[3 * k + 2]);
        std::fprintf(f, "};\n");
        std::fprintf(f, "// kFitInv[l][k][b] = (A_l^-1)[k][b], zero-padded to 7 x 7 (l = 2, 3; rows 0, 1 unused)\n");
        std::fprintf(f, "constexpr double kFitInv[%d][7][7] = {\n", kLmax + 1);
        for (int l = 0; l <= kLmax; ++l) {
            int d = 2 * l + 1;
            std::fprintf(f, "    {");
            for (int k = 0; k < 7; ++k) {
                std::fprintf(f, "{");
                for (int b = 0; b < 7; ++b)
                    std::fprintf(f, "%.21Lg%s", (l >= 2 && k < d && b < d) ? best_inv[l][k * d + b] : (ld)0, b < 6 ? ", " : "");
                std::fprintf(f, "}%s", k < 6 ? ", " : "");
            }
            std::fprintf(f, "},\n");
        }
        std::fprintf(f, "};\n\n");
    }
    // --- Cartesian couplings in independent STF components ------------------
    {
        int coff[kLmax + 1][kLmax + 1][kLmax + 1], ccnt[kLmax + 1][kLmax + 1][kLmax + 1];
        std::vector<Nz> call;
        for (int a = 0; a <= kLmax; ++a)
            for (int b = 0; b <= kLmax; ++b)
                for (int c = 0; c <= kLmax; ++c) {
                    auto v = cart_coupling(a, b, c);
                    coff[a][b][c] = (int)call.size();
                    ccnt[a][b][c] = (int)v.size();
                    call.insert(call.end(), v.begin(), v.end());
                }
        std::fprintf(f, "// Cartesian couplings Cc[i1][i2][i3] in independent STF components (counts of x, y, z\n");
        std::fprintf(f, "// indices: c = 0 entries by ascending y count, then c = 1 entries); see gen_tables.cpp.\n");
        std::fprintf(f, "constexpr int kCartTotal = %d;\n", (int)call.size());
        std::fprintf(f, "constexpr CgNz kCart[kCartTotal] = {\n");
        for (auto& z : call) std::fprintf(f, "    {%d, %d, %d, %.21Lg},\n", z.m1, z.m2, z.m3, z.v);
        std::fprintf(f, "};\n\n");
        for (int pass = 0; pass < 2; ++pass) {
            std::fprintf(f, "constexpr int %s[%d][%d][%d] = {\n", pass ? "kCartCnt" : "kCartOff", kLmax + 1, kLmax + 1,
                         kLmax + 1);
            for (int a = 0; a <= kLmax; ++a) {
                std::fprintf(f, "    {");
                for (int b = 0; b <= kLmax; ++b) {
                    std::fprintf(f, "{");
                    for (int c = 0; c <= kLmax; ++c)
                        std::fprintf(f, "%d%s", pass ? ccnt[a][b][c] : coff[a][b][c], c < kLmax ? ", " : "");
                    std::fprintf(f, "}%s", b < kLmax ? ", " : "");
                }
                std::fprintf(f, "},\n");
            }
            std::fprintf(f, "};\n\n");
        }
    }
    std::fprintf(f, "}  // namespace etp_gen\n");
    std::fclose(f);
    return 0;
}
