// Radial weights of the edges: w = SiLU(bessel(|r|) W1) W2 and its vector-Jacobian
// product, so that the tensor product's weights, their gradients and the forces
// through the edge lengths all run on the device.
//
// ("High-performance training and inference for deep equivariant interatomic
// potentials", section "제안 방법": the per-edge weights of the Allegro tensor product
// are a learned function of the edge length; this is the plain reading of that
// function: Bessel basis b_n(d) = sqrt(2/r_c) sin(n pi d / r_c) / d, a hidden layer
// with SiLU, a linear output layer, no biases.)
//
// Layout (row-major): W1 [n_basis][hidden], W2 [hidden][P*C], w / grad_w [E][P*C],
// hidden activations H [E][hidden]. With a hidden width of 64 the forward, dL/dH and
// grad_W2 run on the tensor cores (etp_radial_tc.cu); the other dense products run in FP32 on the
// SIMT pipes (tiled, 64 x 64 outputs per block, exact fp32 FMAs); their reductions over
// the edges are split across blocks into partial sums that a second kernel adds
// in a fixed order, so every result repeats bit for bit.
#include <cuda_runtime.h>

#include <cstdint>

#include "etp_internal.h"

namespace etp {
namespace {

constexpr int kTile = 64, kTileK = 16, kGemmThreads = 256;
constexpr float kPi = 3.14159265358979323846f;

// C[M][N] = sum_k A(m, k) B(k, n) over k in this block's split of [0, K).
// A(m, k) = TA ? A[k * lda + m] : A[m * lda + k];  B(k, n) = TB ? B[n * ldb + k] : B[k * ldb + n].
// gridDim.z splits K into equal chunks; split z writes its partial to C + z * M * N.
template <bool TA, bool TB>
__global__ void __launch_bounds__(kGemmThreads) gemm_tiled(int M, int N, int K, const float* __restrict__ A, int lda,
                                                           const float* __restrict__ B, int ldb,
                                                           float* __restrict__ C) {
    __shared__ float As[kTileK][kTile + 4];
    __shared__ float Bs[kTileK][kTile + 4];
    const int m0 = blockIdx.x * kTile, n0 = blockIdx.y * kTile;  // M (edges) on x: up to 2^31 - 1 blocks
    const int kchunk = (K + gridDim.z - 1) / gridDim.z;
    const int kb = blockIdx.z * kchunk, ke = min(K, kb + kchunk);
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;  // 16 x 16 threads, 4 x 4 outputs each
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
    for (int k0 = kb; k0 < ke; k0 += kTileK) {
        for (int idx = threadIdx.x; idx < kTileK * kTile; idx += kGemmThreads) {
            int kk, mm;
            if (TA) {  // consecutive threads along m (contiguous in A)
                kk = idx / kTile, mm = idx % kTile;
            } else {   // consecutive threads along k
                mm = idx / kTileK, kk = idx % kTileK;
            }
            const int m = m0 + mm, k = k0 + kk;
            As[kk][mm] = (m < M && k < ke) ? (TA ? A[(size_t)k * lda + m] : A[(size_t)m * lda + k]) : 0.f;
            int kn, nn;
            if (TB) {
                nn = idx / kTileK, kn = idx % kTileK;
            } else {
                kn = idx / kTile, nn = idx % kTile;
            }
            const int n = n0 + nn, k2 = k0 + kn;
            Bs[kn][nn] = (n < N && k2 < ke) ? (TB ? B[(size_t)n * ldb + k2] : B[(size_t)k2 * ldb + n]) : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < kTileK; ++kk) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
    float* Cz = C + (size_t)blockIdx.z * M * N;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int m = m0 + ty * 4 + i;
        if (m >= M) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int n = n0 + tx * 4 + j;
            if (n < N) Cz[(size_t)m * N + n] = acc[i][j];
        }
    }
}

// out[i] = sum_z part[z * n + i], z in order.
__global__ void sum_splits(const float* __restrict__ part, int splits, long long n, float* __restrict__ out) {
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
        float s = 0.f;
        for (int z = 0; z < splits; ++z) s += part[(size_t)z * n + i];
        out[i] = s;
    }
}

// Per edge: d = |r|, the Bessel basis b (and db/dd) and the pre-activations
// z = b W1; writes H = SiLU(z) and, when asked, b and z. One block per group of
// edges, one thread per (edge, hidden unit); the basis of each edge once, in
// shared memory.
constexpr int kEdgesPerBlock = 4;
__device__ __forceinline__ void edge_basis(const float* r, int e, float rc, int nb, float* b, float* db, float* dlen) {
    const float x = __ldg(r + 3 * (size_t)e), y = __ldg(r + 3 * (size_t)e + 1), z = __ldg(r + 3 * (size_t)e + 2);
    const float d = sqrtf(x * x + y * y + z * z);
    *dlen = d;
    const float c = sqrtf(2.f / rc);
    for (int n = 1; n <= nb; ++n) {
        const float k = (float)n * kPi / rc;
        if (!(d >= 1e-12f)) {  // limit at d = 0
            b[n - 1] = c * k;
            db[n - 1] = 0.f;
        } else {
            float s, co;
            sincosf(k * d, &s, &co);
            b[n - 1] = c * s / d;
            db[n - 1] = c * (k * co / d - s / (d * d));
        }
    }
}

__global__ void radial_hidden(int E, const float* __restrict__ r, const float* __restrict__ W1, int nb, int hidden,
                              float rc, float* __restrict__ H, float* __restrict__ Zout, float* __restrict__ Bout) {
    extern __shared__ float sb[];  // [kEdgesPerBlock][nb]
    const int e0 = blockIdx.x * kEdgesPerBlock;
    if (threadIdx.x < kEdgesPerBlock && e0 + (int)threadIdx.x < E) {
        float db[32], d;
        edge_basis(r, e0 + threadIdx.x, rc, nb, sb + threadIdx.x * nb, db, &d);
        if (Bout)
            for (int n = 0; n < nb; ++n) Bout[(size_t)(e0 + threadIdx.x) * nb + n] = sb[threadIdx.x * nb + n];
    }
    __syncthreads();
    for (int t = threadIdx.x; t < kEdgesPerBlock * hidden; t += blockDim.x) {
        const int le = t / hidden, k = t % hidden, e = e0 + le;
        if (e >= E) continue;
        float z = 0.f;
        for (int n = 0; n < nb; ++n) z = fmaf(sb[le * nb + n], __ldg(W1 + n * hidden + k), z);
        H[(size_t)e * hidden + k] = z / (1.f + expf(-z));
        if (Zout) Zout[(size_t)e * hidden + k] = z;
    }
}

// Per edge, from dL/dH: dL/dz = dL/dH * SiLU'(z) (written to gZ), dL/db = dL/dz W1^T,
// dL/dd = dL/db . db/dd, and grad_r[e] += dL/dd r / |r|. One block of `hidden`
// threads (a multiple of 32, at most 256) per edge.
__global__ void radial_edge_backward(int E, const float* __restrict__ r, const float* __restrict__ W1, int nb,
                                     int hidden, float rc, const float* __restrict__ Z,
                                     const float* __restrict__ gH, float* __restrict__ gZ,
                                     float* __restrict__ grad_r) {
    __shared__ float red[8][33];  // [warp][basis function], nb <= 32
    __shared__ float basis[2][32];
    __shared__ float dlen;
    const int e = blockIdx.x, k = threadIdx.x, lane = k & 31, wid = k >> 5;
    if (k == 0) edge_basis(r, e, rc, nb, basis[0], basis[1], &dlen);
    __syncthreads();
    const float z = Z[(size_t)e * hidden + k];
    const float s = 1.f / (1.f + expf(-z));
    const float g = gH[(size_t)e * hidden + k] * (s * (1.f + z * (1.f - s)));
    gZ[(size_t)e * hidden + k] = g;
    for (int n = 0; n < nb; ++n) {
        float v = g * __ldg(W1 + n * hidden + k);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) red[wid][n] = v;
    }
    __syncthreads();
    if (k == 0) {
        float dd = 0.f;
        for (int n = 0; n < nb; ++n) {
            float gb = 0.f;
            for (int w = 0; w < (int)(blockDim.x >> 5); ++w) gb += red[w][n];
            dd = fmaf(gb, basis[1][n], dd);
        }
        const float d = dlen;
        if (d >= 1e-12f) {
            const float f = dd / d;
            grad_r[3 * (size_t)e] += f * __ldg(r + 3 * (size_t)e);
            grad_r[3 * (size_t)e + 1] += f * __ldg(r + 3 * (size_t)e + 1);
            grad_r[3 * (size_t)e + 2] += f * __ldg(r + 3 * (size_t)e + 2);
        }
    }
}

// grad_W1 partial sums: part[split][n][k] = sum_e B[e][n] gZ[e][k] over this block's
// split of the edges. 256 threads = (256 / hidden) edge lanes x hidden units; each
// thread keeps its nb (<= 32) sums in registers, then the edge lanes are added in a
// fixed order through shared memory.
constexpr int kW1Threads = 256;
__global__ void __launch_bounds__(kW1Threads) radial_grad_w1(int E, int nb, int hidden, int edges_per_split,
                                                             const float* __restrict__ Bm, const float* __restrict__ gZ,
                                                             float* __restrict__ part) {
    extern __shared__ float red[];  // [lanes][nb][hidden]
    const int lanes = kW1Threads / hidden, el = threadIdx.x / hidden, k = threadIdx.x % hidden;
    const int e_begin = blockIdx.x * edges_per_split, e_end = min(E, e_begin + edges_per_split);
    float acc[32];
#pragma unroll
    for (int n = 0; n < 32; ++n) acc[n] = 0.f;
    if (el < lanes) {
        for (int e = e_begin + el; e < e_end; e += lanes) {
            const float g = __ldg(gZ + (size_t)e * hidden + k);
#pragma unroll
            for (int n = 0; n < 32; ++n)
                if (n < nb) acc[n] = fmaf(__ldg(Bm + (size_t)e * nb + n), g, acc[n]);
        }
#pragma unroll
        for (int n = 0; n < 32; ++n)
            if (n < nb) red[(el * nb + n) * hidden + k] = acc[n];
    }
    __syncthreads();
    for (int o = threadIdx.x; o < nb * hidden; o += kW1Threads) {
        float v = 0.f;
        for (int l = 0; l < lanes; ++l) v += red[l * nb * hidden + o];
        part[(size_t)blockIdx.x * nb * hidden + o] = v;
    }
}

// Edge splits of the grad_W1 reduction: two blocks per SM, at least 256 edges each.
inline int grad_w1_splits(int E) {
    int s = (E + 255) / 256;
    return s > 296 ? 296 : (s < 1 ? 1 : s);
}

inline size_t a16(size_t b) { return (b + 15) & ~size_t(15); }

// Splits of a K = E reduction: enough blocks to fill the GPU once, each split at
// least 4096 edges.
inline int edge_splits(int E, int tiles) {
    int s = (148 * 4 + tiles - 1) / (tiles > 0 ? tiles : 1);
    const int by_size = (E + 4095) / 4096;
    if (s > by_size) s = by_size;
    if (s > 64) s = 64;
    return s < 1 ? 1 : s;
}

// Edge splits of the grad_W2 reduction: the tensor-core kernel's when it runs.
inline int grad_w2_splits(int E, int nb, int hidden, int PC) {
    if (radial_tc_supported(nb, hidden, PC)) return radial_tc_grad_w2_splits(E, PC);
    return edge_splits(E, ((hidden + kTile - 1) / kTile) * ((PC + kTile - 1) / kTile));
}

template <bool TA, bool TB>
cudaError_t gemm(int M, int N, int K, const float* A, int lda, const float* B, int ldb, float* C, int splits,
                 cudaStream_t s) {
    dim3 grid((M + kTile - 1) / kTile, (N + kTile - 1) / kTile, splits);
    gemm_tiled<TA, TB><<<grid, kGemmThreads, 0, s>>>(M, N, K, A, lda, B, ldb, C);
    return cudaGetLastError();
}

}  // namespace

size_t radial_workspace_bytes(int E, int nb, int hidden, int PC) {
    const int s2 = grad_w2_splits(E, nb, hidden, PC);
    const int s1 = grad_w1_splits(E);
    const size_t bwd = 4 * a16(sizeof(float) * (size_t)E * hidden) + a16(sizeof(float) * (size_t)E * nb) +
                       a16(sizeof(float) * (size_t)s2 * hidden * PC) + a16(sizeof(float) * (size_t)s1 * nb * hidden);
    const bool tc = radial_tc_supported(nb, hidden, PC);
    const size_t bwd_all = bwd + (tc ? a16(radial_tc_backward_prepare_bytes(PC)) : 0);
    const size_t fwd_tc = tc ? radial_tc_prepare_bytes(PC) : 0;
    return bwd_all > fwd_tc ? bwd_all : fwd_tc;
}

cudaError_t radial_forward(int E, int nb, int hidden, int PC, float rc, const float* r, const float* W1,
                           const float* W2, float* w, void* ws, cudaStream_t s) {
    if (E == 0) return cudaSuccess;
    if (radial_tc_supported(nb, hidden, PC)) return radial_tc_forward(E, nb, PC, rc, r, W1, W2, w, ws, s);
    float* H = static_cast<float*>(ws);
    radial_hidden<<<(E + kEdgesPerBlock - 1) / kEdgesPerBlock, 256, sizeof(float) * kEdgesPerBlock * nb, s>>>(
        E, r, W1, nb, hidden, rc, H, nullptr, nullptr);
    // w [E][PC] = H [E][hidden] W2 [hidden][PC]
    return gemm<false, false>(E, PC, hidden, H, hidden, W2, PC, w, 1, s);
}

cudaError_t radial_backward(int E, int nb, int hidden, int PC, float rc, const float* r, const float* W1,
                            const float* W2, const float* grad_w, float* grad_W1, float* grad_W2, float* grad_r,
                            void* ws, cudaStream_t s) {
    char* p = static_cast<char*>(ws);
    float* H = reinterpret_cast<float*>(p);
    p += a16(sizeof(float) * (size_t)E * hidden);
    float* Z = reinterpret_cast<float*>(p);
    p += a16(sizeof(float) * (size_t)E * hidden);
    float* gH = reinterpret_cast<float*>(p);
    p += a16(sizeof(float) * (size_t)E * hidden);
    float* gZ = reinterpret_cast<float*>(p);
    p += a16(sizeof(float) * (size_t)E * hidden);
    float* Bm = reinterpret_cast<float*>(p);
    p += a16(sizeof(float) * (size_t)E * nb);
    float* part2 = reinterpret_cast<float*>(p);
    const int s2 = grad_w2_splits(E, nb, hidden, PC);
    p += a16(sizeof(float) * (size_t)s2 * hidden * PC);
    float* part1 = reinterpret_cast<float*>(p);
    const int s1 = grad_w1_splits(E);
    cudaError_t err;
    if (E == 0) {  // no edges: the parameter gradients are zero
        if ((err = cudaMemsetAsync(grad_W1, 0, sizeof(float) * nb * hidden, s)) != cudaSuccess) return err;
        return cudaMemsetAsync(grad_W2, 0, sizeof(float) * (size_t)hidden * PC, s);
    }
    const bool tc = radial_tc_supported(nb, hidden, PC);
    radial_hidden<<<(E + kEdgesPerBlock - 1) / kEdgesPerBlock, 256, sizeof(float) * kEdgesPerBlock * nb, s>>>(
        E, r, W1, nb, hidden, rc, H, tc ? nullptr : Z, Bm);
    if (tc) {  // dL/dH on the tensor cores, with dL/dz, dL/dd and grad_r fused into its epilogue
        p += a16(sizeof(float) * (size_t)s1 * nb * hidden);
        if ((err = radial_tc_backward(E, PC, rc, r, W1, W2, grad_w, gZ, grad_r, p, s)) != cudaSuccess) return err;
    } else {
        // dL/dH [E][hidden] = grad_w [E][PC] W2^T
        if ((err = gemm<false, true>(E, hidden, PC, grad_w, PC, W2, PC, gH, 1, s)) != cudaSuccess) return err;
        radial_edge_backward<<<E, hidden, 0, s>>>(E, r, W1, nb, hidden, rc, Z, gH, gZ, grad_r);
    }
    // grad_W2 [hidden][PC] = H^T grad_w, grad_W1 [nb][hidden] = B^T dL/dz: reductions over the edges
    if (tc)
        err = radial_tc_grad_w2(E, PC, grad_w, H, part2, s2, s);
    else
        err = gemm<true, false>(hidden, PC, E, H, hidden, grad_w, PC, part2, s2, s);
    if (err != cudaSuccess) return err;
    sum_splits<<<256, 256, 0, s>>>(part2, s2, (long long)hidden * PC, grad_W2);
    const int per1 = (E + s1 - 1) / s1;
    radial_grad_w1<<<s1, kW1Threads, sizeof(float) * (kW1Threads / hidden) * nb * hidden, s>>>(E, nb, hidden, per1,
                                                                                               Bm, gZ, part1);
    sum_splits<<<16, 256, 0, s>>>(part1, s1, (long long)nb * hidden, grad_W1);
    return cudaGetLastError();
}

}  // namespace etp
