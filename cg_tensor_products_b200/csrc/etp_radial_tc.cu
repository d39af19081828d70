// Radial weights on the 5th-generation tensor cores: w [E][PC] = H [E][64] W2 [64][PC]
// with H = SiLU(bessel(|r|) W1), computed in one kernel per tile of 128 edges.
//
// FP32 accuracy from TF32 tensor-core products by the three-term split
// (x = x_hi + x_lo with x_hi = TF32(x), x_lo = TF32(x - x_hi)):
//     A B ~ A_hi B_hi + A_hi B_lo + A_lo B_hi,
// whose dropped term A_lo B_lo and rounding of the halves leave a relative error
// near 2^-21 per product, below the 1e-5 tolerance of the forward.
//
// Per CTA (4 warps) and tile of 128 edges:
//   1. each thread builds its edge's row of H (Bessel basis, first layer, SiLU),
//      splits it into TF32 halves and stores both into shared memory in the
//      tensor core's K-major layout without swizzle: 8-row x 16-byte core matrices,
//      LBO = 128 B between core matrices along K, SBO = 2048 B between 8-row groups;
//   2. per chunk of up to 128 output columns, one thread bulk-copies the chunk of
//      W2^T (halves pre-split by radial_tc_prepare into the same layout) into shared
//      memory, issues 8 K-steps x 3 products of tcgen05.mma (M = 128, N = chunk,
//      K = 8, kind::tf32) into a TMEM accumulator and commits them to an mbarrier;
//   3. the 4 warps read the accumulator back (tcgen05.ld, warp w owns TMEM lanes
//      32w..32w+31, i.e. edges), stage it in shared memory and store w in whole
//      row segments.
// Every wait is bounded; on time-out the kernel raises its fault flag and leaves.
#include <cuda_runtime.h>

#include <cstdint>

#include "etp_internal.h"

namespace etp {
namespace rtc {

constexpr int kRows = 128;                    // edges per tile (MMA M)
constexpr int kHidden = 64;                   // K of the product (the hidden width)
constexpr int kChunk = 128;                   // output columns per MMA group (N)
constexpr int kThreads = 128;
constexpr uint32_t kLBO = 128, kSBO = 2048;   // bytes: next K core matrix, next 8-row group
constexpr uint32_t kTileBytes = kRows * kHidden * 4;  // 32 KB: one operand half of a tile
constexpr int kWaitLimit = 1 << 22;
constexpr float kPi = 3.14159265358979323846f;

__device__ int g_fault;

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

// Byte offset of element (row, k) of a K-major, unswizzled operand tile.
__host__ __device__ constexpr uint32_t tile_offset(int row, int k) {
    return (uint32_t)((row >> 3) * kSBO + (k >> 2) * kLBO + (row & 7) * 16 + (k & 3) * 4);
}

__device__ __forceinline__ float tf32_round(float x) {
    uint32_t y;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(y) : "f"(x));
    return __uint_as_float(y);
}

// Shared-memory matrix descriptor: start address, LBO, SBO (all >> 4), version 1,
// no swizzle.
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((kLBO >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((kSBO >> 4) & 0x3FFFu) << 32) | ((uint64_t)1 << 46);
}

// Instruction descriptor: D f32, A and B tf32, both K-major, N, M = 128.
__device__ __forceinline__ uint32_t instr_desc(int n) {
    return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(kRows >> 4) << 24);
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ bool mbar_wait(uint64_t* bar, unsigned parity) {
    for (int i = 0; i < kWaitLimit; ++i) {
        unsigned done;
        asm volatile(
            "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
            : "=r"(done)
            : "r"(smem_u32(bar)), "r"(parity)
            : "memory");
        if (done) return true;
    }
    return false;
}

// Fills the W2^T operand halves: chunk c (columns 128c ..) is a 128 x 64 tile in
// the K-major layout; rows past the end are zero. hi / lo: [n_chunks][32 KB].
__global__ void radial_tc_prepare(const float* __restrict__ W2, int PC, int n_chunks, float* __restrict__ hi,
                                  float* __restrict__ lo) {
    const long long total = (long long)n_chunks * kRows * kHidden;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const int c = (int)(i / (kRows * kHidden)), rem = (int)(i % (kRows * kHidden));
        const int n = rem / kHidden, k = rem % kHidden;
        const int col = c * kChunk + n;
        const float v = col < PC ? W2[(size_t)k * PC + col] : 0.f;
        const float h = tf32_round(v);
        const size_t off = (size_t)c * (kTileBytes / 4) + tile_offset(n, k) / 4;
        hi[off] = h;
        lo[off] = tf32_round(v - h);
    }
}

__global__ void __launch_bounds__(kThreads, 1)
    radial_tc_forward(int E, int PC, int nb, float rc, const float* __restrict__ r, const float* __restrict__ W1,
                      const float* __restrict__ Bhi, const float* __restrict__ Blo, float* __restrict__ w) {
    extern __shared__ __align__(1024) unsigned char smem[];
    // [A_hi 32 KB][A_lo 32 KB][B_hi 32 KB][B_lo 32 KB][2 mbarriers][TMEM address]
    unsigned char* a_hi = smem;
    unsigned char* a_lo = smem + kTileBytes;
    unsigned char* b_hi = smem + 2 * kTileBytes;
    unsigned char* b_lo = smem + 3 * kTileBytes;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 4 * kTileBytes);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + 4 * kTileBytes + 16);
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    const int m0 = blockIdx.x * kRows;

    if (warp == 0) {  // 128 fp32 accumulator columns
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(128)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (t == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }

    // 1. the tile's rows of H, split into TF32 halves
    {
        const int e = m0 + t;
        float b[32];
        if (e < E) {
            const float x = __ldg(r + 3 * (size_t)e), y = __ldg(r + 3 * (size_t)e + 1), z = __ldg(r + 3 * (size_t)e + 2);
            const float d = sqrtf(x * x + y * y + z * z);
            const float c = sqrtf(2.f / rc);
            for (int n = 0; n < nb; ++n) {
                const float k = (float)(n + 1) * kPi / rc;
                b[n] = d >= 1e-12f ? c * sinf(k * d) / d : c * k;
            }
        }
        for (int k = 0; k < kHidden; ++k) {
            float h = 0.f;
            if (e < E) {
                float zz = 0.f;
                for (int n = 0; n < nb; ++n) zz = fmaf(b[n], __ldg(W1 + n * kHidden + k), zz);
                h = zz / (1.f + expf(-zz));
            }
            const float hh = tf32_round(h);
            *reinterpret_cast<float*>(a_hi + tile_offset(t, k)) = hh;
            *reinterpret_cast<float*>(a_lo + tile_offset(t, k)) = tf32_round(h - hh);
        }
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // generic-proxy writes -> tensor core
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = *tmem_slot;

    const int n_chunks = (PC + kChunk - 1) / kChunk;
    bool live = true;
    for (int c = 0; c < n_chunks && live; ++c) {
        const int n = min(kChunk, PC - c * kChunk);  // a multiple of 16
        if (t == 0) {
            asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(&bars[0])),
                         "r"(2 * kTileBytes)
                         : "memory");
            asm volatile(
                "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                    smem_u32(b_hi)),
                "l"(Bhi + (size_t)c * (kTileBytes / 4)), "r"(kTileBytes), "r"(smem_u32(&bars[0]))
                : "memory");
            asm volatile(
                "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                    smem_u32(b_lo)),
                "l"(Blo + (size_t)c * (kTileBytes / 4)), "r"(kTileBytes), "r"(smem_u32(&bars[0]))
                : "memory");
            if (!mbar_wait(&bars[0], c & 1)) {
                live = false;
                mbar_wait(&bars[0], c & 1);  // give the copies in flight one more bounded wait before leaving
            } else {
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                const uint32_t idesc = instr_desc(n);
                const unsigned char* A[3] = {a_hi, a_hi, a_lo};
                const unsigned char* B[3] = {b_hi, b_lo, b_hi};
                int issued = 0;
                for (int s = 0; s < kHidden / 8; ++s) {
                    for (int q = 0; q < 3; ++q, ++issued) {
                        const uint64_t da = smem_desc(smem_u32(A[q]) + s * 2 * kLBO);
                        const uint64_t db = smem_desc(smem_u32(B[q]) + s * 2 * kLBO);
                        const uint32_t acc = issued > 0 ? 1u : 0u;
                        asm volatile(
                            "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
                            " tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n}" ::"r"(tmem),
                            "l"(da), "l"(db), "r"(idesc), "r"(acc)
                            : "memory");
                    }
                }
                asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                                 smem_u32(&bars[1]))
                             : "memory");
            }
        }
        // everyone: the accumulator of this chunk
        live = __syncthreads_and(live ? 1 : 0) != 0;
        if (!live) break;
        if (!mbar_wait(&bars[1], c & 1)) {
            live = false;
            mbar_wait(&bars[1], c & 1);  // the MMAs write TMEM: wait once more before it is freed
        }
        live = __syncthreads_and(live ? 1 : 0) != 0;
        if (!live) break;
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        // 3. epilogue through shared memory (the B buffers are free once the MMAs are
        // done): each half of the chunk (64 columns) is staged row by row with a
        // 65-float stride (conflict-free), then each warp stores whole row segments.
        float* stage = reinterpret_cast<float*>(b_hi);
        for (int h0 = 0; h0 < n; h0 += 64) {
            const int hn = min(64, n - h0);
            for (int j = 0; j < hn; j += 16) {
                uint32_t v[16];
                asm volatile(
                    "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
                    "%13, %14, %15}, [%16];"
                    : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
                      "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]),
                      "=r"(v[15])
                    : "r"(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)(h0 + j)));
                asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
                for (int q = 0; q < 16; ++q) stage[t * 65 + j + q] = __uint_as_float(v[q]);
            }
            __syncthreads();
            for (int rr = 0; rr < 32; ++rr) {
                const int row = warp * 32 + rr, e = m0 + row;
                if (e < E && 2 * lane < hn) {
                    const float2 val = make_float2(stage[row * 65 + 2 * lane], stage[row * 65 + 2 * lane + 1]);
                    *reinterpret_cast<float2*>(w + (size_t)e * PC + c * kChunk + h0 + 2 * lane) = val;
                }
            }
            __syncthreads();
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // staging reads before the next bulk copy
        asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
        __syncthreads();  // accumulator and B buffers free for the next chunk
    }
    if (!live && t == 0) atomicOr(&g_fault, 1);
    __syncthreads();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(128) : "memory");
}

}  // namespace rtc

size_t radial_tc_prepare_bytes(int PC) {
    const int n_chunks = (PC + rtc::kChunk - 1) / rtc::kChunk;
    return 2 * (size_t)n_chunks * rtc::kTileBytes;
}

bool radial_tc_supported(int nb, int hidden, int PC) { return hidden == rtc::kHidden && nb <= 32 && PC % 16 == 0; }

cudaError_t radial_tc_forward(int E, int nb, int PC, float rc, const float* r, const float* W1, const float* W2,
                              float* w, void* ws, cudaStream_t s) {
    if (E == 0) return cudaSuccess;
    const int n_chunks = (PC + rtc::kChunk - 1) / rtc::kChunk;
    float* hi = static_cast<float*>(ws);
    float* lo = hi + (size_t)n_chunks * (rtc::kTileBytes / 4);
    rtc::radial_tc_prepare<<<256, 256, 0, s>>>(W2, PC, n_chunks, hi, lo);
    const size_t smem = 4 * (size_t)rtc::kTileBytes + 64;
    cudaError_t err = cudaFuncSetAttribute(rtc::radial_tc_forward, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)smem);
    if (err != cudaSuccess) return err;
    rtc::radial_tc_forward<<<(E + rtc::kRows - 1) / rtc::kRows, rtc::kThreads, smem, s>>>(E, PC, nb, rc, r, W1, hi, lo,
                                                                                         w);
    return cudaGetLastError();
}

int radial_tc_read_and_clear_fault() {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, rtc::g_fault, sizeof(int)) != cudaSuccess) return -1;
    const int zero = 0;
    cudaMemcpyToSymbol(rtc::g_fault, &zero, sizeof(int));
    return v;
}

}  // namespace etp
