// Radial weights on the 5th-generation tensor cores: w [E][PC] = H [E][64] W2 [64][PC]
// with H = SiLU(bessel(|r|) W1), computed in one kernel per tile of 128 edges.
//
// FP32 accuracy from TF32 tensor-core products by the three-term split
// (x = x_hi + x_lo with x_hi = TF32(x), x_lo = TF32(x - x_hi)):
//     A B ~ A_hi B_hi + A_hi B_lo + A_lo B_hi,
// whose dropped term A_lo B_lo and rounding of the halves leave a relative error
// near 2^-21 per product, below the 1e-5 tolerance of the forward.
//
// Per CTA (9 warps, one persistent CTA per SM: 226 KB of shared memory) and tile of
// 128 edges, the tiles of a CTA taken in turn:
//   1. the 8 epilogue warps build the tile's rows of H (Bessel basis, first layer,
//      SiLU; two threads per edge), split them into TF32 halves and store both into
//      tensor memory (tcgen05.st; TMEM lane = edge, one column per hidden unit; two
//      buffers, so the next tile's H is built while this tile's last chunk multiplies);
//   2. per chunk of up to 128 output columns, one thread of the ninth warp
//      bulk-copies the chunk of W2^T (halves pre-split by radial_tc_prepare into the
//      K-major shared-memory layout without swizzle: 8-row x 16-byte core matrices,
//      LBO = 128 B between core matrices along K, SBO = 2048 B between 8-row groups)
//      into one of three slots, issues 8 K-steps x 3 products of tcgen05.mma
//      (M = 128, N = chunk, K = 8, kind::tf32, A from tensor memory) into one of two
//      TMEM accumulators and commits them to an mbarrier;
//   3. the 8 epilogue warps read the accumulator back (tcgen05.ld; warps w and w + 4
//      own TMEM lanes 32w..32w+31, i.e. edges, and half of the columns each), hand it
//      back to the MMA thread by an mbarrier, and store w in whole 128-byte row
//      segments through a per-warp stage. No block barrier inside the chunk loop.
// The VJP's two dense products, dL/dH = grad_w W2^T and grad_W2 = H^T grad_w, follow
// below as warp-specialised kernels with the same operand layout and split.
// Every wait is bounded; on time-out the kernel raises its fault flag and leaves.
#include <cuda_runtime.h>

#include <cstdint>

#include "etp_internal.h"

namespace etp {
namespace rtc {

constexpr int kRows = 128;                    // edges per tile (MMA M)
constexpr int kBasis = 8;                     // Bessel functions (compile-time: registers, unrolled)
constexpr int kHidden = 64;                   // K of the product (the hidden width)
constexpr int kChunk = 128;                   // output columns per MMA group (N)
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

// Shared memory: three W2 slots of two TF32 halves (192 KB), the epilogue stage (8
// warps x 32 rows x 32 floats, 16-byte units XOR-swizzled by the row so that a phase
// of 8 lanes writing one row each, or reading 8 units of one row, touches 8 distinct
// bank quads), 7 mbarriers, the TMEM address, a flag. The H operand lives in tensor
// memory, next to the two accumulators.
constexpr int kEpiWarps = 8;                   // two per TMEM lane quarter, each half of a chunk's columns
constexpr int kFwdThreads = (kEpiWarps + 1) * 32;
constexpr int kSlots = 3;
constexpr uint32_t kSlotBytes = 2 * kTileBytes;
constexpr uint32_t kStageFloats = kEpiWarps * 32 * 32;
constexpr uint32_t kOffStage = kSlots * kSlotBytes;
constexpr uint32_t kOffW1 = kOffStage + kStageFloats * 4;
constexpr uint32_t kOffBars = kOffW1 + kBasis * kHidden * 4;
constexpr uint32_t kSmemBytes = kOffBars + 128;
// TMEM columns: accumulators 0..127 and 128..255; H's TF32 halves of two tiles (hi, lo): 256.., 384..
constexpr uint32_t kTmemCols = 512;
static_assert(kOffBars % 16 == 0 && kSmemBytes <= 232448, "radial tensor-core kernel shared memory");

__device__ __forceinline__ void load_b(const float* Bhi, const float* Blo, int c, unsigned char* slot_hi,
                                       unsigned char* slot_lo, uint64_t* bar) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(2 * kTileBytes)
                 : "memory");
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(slot_hi)),
                 "l"(Bhi + (size_t)c * (kTileBytes / 4)), "r"(kTileBytes), "r"(smem_u32(bar))
                 : "memory");
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(slot_lo)),
                 "l"(Blo + (size_t)c * (kTileBytes / 4)), "r"(kTileBytes), "r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive_one(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
        "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]),
        "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]),
        "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
}

// The H operand of one tile (128 edges x 64 hidden units, both TF32 halves) from the
// edge lengths: two epilogue threads per edge, 32 hidden units each, written into tensor
// memory (tcgen05.st; TMEM lane = edge) at columns col_hi / col_lo.
__device__ __forceinline__ void build_h(int t, int warp, int m0, int E, float rc, const float* __restrict__ r,
                                        const float* w1s, uint32_t tmem, uint32_t col_hi, uint32_t col_lo) {
    const int row = t & (kRows - 1), k0 = (t >> 7) * (kHidden / 2);
    const int e = m0 + row;
    float b[kBasis];
#pragma unroll
    for (int n = 0; n < kBasis; ++n) b[n] = 0.f;
    if (e < E) {
        const float x = __ldg(r + 3 * (size_t)e), y = __ldg(r + 3 * (size_t)e + 1), z = __ldg(r + 3 * (size_t)e + 2);
        const float d = sqrtf(x * x + y * y + z * z);
        const float c = sqrtf(2.f / rc);
#pragma unroll
        for (int n = 0; n < kBasis; ++n) {
            const float k = (float)(n + 1) * kPi / rc;
            b[n] = d >= 1e-12f ? c * sinf(k * d) / d : c * k;
        }
    }
    uint32_t vh[32], vl[32];
#pragma unroll
    for (int k = 0; k < 32; ++k) {
        float h = 0.f;
        if (e < E) {
            float zz = 0.f;
#pragma unroll
            for (int n = 0; n < kBasis; ++n) zz = fmaf(b[n], w1s[n * kHidden + k0 + k], zz);
            h = zz / (1.f + expf(-zz));
        }
        const float hh = tf32_round(h);
        vh[k] = __float_as_uint(hh);
        vl[k] = __float_as_uint(tf32_round(h - hh));
    }
    const uint32_t lanebase = (uint32_t)((warp & 3) * 32) << 16;
    tmem_st32(tmem + lanebase + col_hi + k0, vh);
    tmem_st32(tmem + lanebase + col_lo + k0, vl);
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Persistent warp-specialised pipeline: one CTA per SM walks tiles blockIdx.x,
// blockIdx.x + gridDim.x, .., and the chunks of all its tiles form one sequence g (tile
// major), with no block barrier in the loop. The MMA warp (one thread) issues chunk g
// into accumulator g % 2 once its W2 slot (g % 3) is filled (bar_b), the epilogue has
// drained chunk g - 2 from that accumulator (bar_free, one arrival per epilogue warp)
// and, for a tile's first chunk, the tile's H is in tensor memory (bar_h, H buffer
// tile % 2); the products read A from tensor memory (the A-from-TMEM form of
// tcgen05.mma) and only W2 from shared memory. It commits to bar_m and refills the slot
// of chunk g - 1 with chunk g + 2 once chunk g - 1's products are done. Each epilogue
// warp (TMEM lane quarter w % 4, column half w / 4) builds the next tile's H while the
// current tile's last chunk multiplies, waits for bar_m, reads its 32 rows x 64 columns
// into registers, frees the accumulator, and writes the rows out through its own stage:
// every store instruction writes four whole 128-byte row segments.
__global__ void __launch_bounds__(kFwdThreads, 1)
    radial_tc_forward(int E, int PC, int nb, float rc, const float* __restrict__ r, const float* __restrict__ W1,
                        const float* __restrict__ Bhi, const float* __restrict__ Blo, float* __restrict__ w) {
    extern __shared__ __align__(1024) unsigned char smem[];
    float* stage = reinterpret_cast<float*>(smem + kOffStage);
    float* w1s = reinterpret_cast<float*>(smem + kOffW1);
    uint64_t* bar_b = reinterpret_cast<uint64_t*>(smem + kOffBars);  // [3]
    uint64_t* bar_m = bar_b + 3;                                        // [2]
    uint64_t* bar_free = bar_b + 5;                                     // [2]
    uint64_t* bar_h = bar_b + 7;                                        // [2] H buffer written
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffBars + 96);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffBars + 100);
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    const int n_tiles = (E + kRows - 1) / kRows;
    const int n_local = n_tiles > (int)blockIdx.x ? (n_tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
    const int n_chunks = (PC + kChunk - 1) / kChunk;
    const int total = n_local * n_chunks;  // this CTA's chunks, tile-major
    constexpr int kMmaWarp = kEpiWarps;
    auto slot_hi = [&](int s) { return smem + (uint32_t)s * kSlotBytes; };
    auto slot_lo = [&](int s) { return smem + (uint32_t)s * kSlotBytes + kTileBytes; };
    auto hcol = [&](int hb, int lo) { return (uint32_t)(256 + 128 * hb + 64 * lo); };
    if (warp == kMmaWarp) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
        if (lane == 0) {
            for (int i = 0; i < 5; ++i) mbar_init(&bar_b[i], 1);
            for (int i = 0; i < 2; ++i) mbar_init(&bar_free[i], kEpiWarps);
            for (int i = 0; i < 2; ++i) mbar_init(&bar_h[i], kEpiWarps);
            *abort_flag = 0;
            asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
            for (int g = 0; g < kSlots && g < total; ++g)
                load_b(Bhi, Blo, g % n_chunks, slot_hi(g), slot_lo(g), &bar_b[g]);
        }
    }
    for (int i = t; i < kBasis * kHidden; i += kFwdThreads) w1s[i] = __ldg(W1 + i);
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = *tmem_slot;
    if (warp == kMmaWarp) {
        if (lane == 0) {
            int committed = -1, loaded = min(kSlots, total) - 1;
            for (int g = 0; g < total && !*abort_flag; ++g) {
                const int i = g / n_chunks, c = g - i * n_chunks;
                const int sb = g & 1, u = g >> 1, sl = g % kSlots, ul = g / kSlots;
                if (!mbar_wait(&bar_b[sl], ul & 1) || (g >= 2 && !mbar_wait(&bar_free[sb], (u - 1) & 1)) ||
                    (c == 0 && !mbar_wait(&bar_h[i & 1], (i >> 1) & 1))) {
                    *abort_flag = 1;
                    break;
                }
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                const int n = min(kChunk, PC - c * kChunk);
                const uint32_t idesc = instr_desc(n);
                const uint32_t d_tmem = tmem + (uint32_t)sb * 128;
                const uint32_t At[3] = {tmem + hcol(i & 1, 0), tmem + hcol(i & 1, 0), tmem + hcol(i & 1, 1)};
                const uint32_t B[3] = {smem_u32(slot_hi(sl)), smem_u32(slot_lo(sl)), smem_u32(slot_hi(sl))};
                for (int s = 0; s < kHidden / 8; ++s) {
                    for (int q = 0; q < 3; ++q) {
                        const uint64_t db = smem_desc(B[q] + s * 2 * kLBO);
                        const uint32_t acc = (s | q) ? 1u : 0u;
                        asm volatile(
                            "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
                            " tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n}" ::"r"(d_tmem),
                            "r"(At[q] + 8 * s), "l"(db), "r"(idesc), "r"(acc)
                            : "memory");
                    }
                }
                asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                                 smem_u32(&bar_m[sb]))
                             : "memory");
                committed = g;
                if (g >= 1 && g + 2 < total) {
                    if (!mbar_wait(&bar_m[sb ^ 1], ((g - 1) >> 1) & 1)) {
                        *abort_flag = 1;
                        break;
                    }
                    const int s2 = (g + 2) % kSlots;
                    load_b(Bhi, Blo, (g + 2) % n_chunks, slot_hi(s2), slot_lo(s2), &bar_b[s2]);
                    loaded = g + 2;
                }
            }
            if (*abort_flag) {
                atomicOr(&g_fault, 1);
                if (committed >= 0) mbar_wait(&bar_m[committed & 1], (committed >> 1) & 1);
                if (committed >= 1) mbar_wait(&bar_m[(committed - 1) & 1], ((committed - 1) >> 1) & 1);
                for (int g = committed + 1; g <= loaded; ++g) mbar_wait(&bar_b[g % kSlots], (g / kSlots) & 1);
            }
        }
    } else {
        const int q = warp & 3, hf = warp >> 2;
        float* st = stage + warp * 32 * 32;
        if (n_local > 0) {
            build_h(t, warp, (int)blockIdx.x * kRows, E, rc, r, w1s, tmem, hcol(0, 0), hcol(0, 1));
            asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
            __syncwarp();
            if (lane == 0) mbar_arrive_one(&bar_h[0]);
        }
        for (int g = 0; g < total; ++g) {
            const int i = g / n_chunks, c = g - i * n_chunks;
            const int m0 = ((int)blockIdx.x + i * (int)gridDim.x) * kRows;
            if (c == n_chunks - 1 && i + 1 < n_local) {  // the next tile's H, while this tile's last chunk multiplies
                build_h(t, warp, ((int)blockIdx.x + (i + 1) * (int)gridDim.x) * kRows, E, rc, r, w1s, tmem,
                        hcol((i + 1) & 1, 0), hcol((i + 1) & 1, 1));
                asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
                __syncwarp();
                if (lane == 0) mbar_arrive_one(&bar_h[(i + 1) & 1]);
            }
            const int sb = g & 1, u = g >> 1;
            const int n = min(kChunk, PC - c * kChunk);
            const int hn = max(0, min(64, n - 64 * hf));
            const bool got = mbar_wait(&bar_m[sb], u & 1);
            if (__any_sync(0xffffffffu, !got || *abort_flag)) {
                if (lane == 0) {
                    *abort_flag = 1;
                    atomicOr(&g_fault, 1);
                }
                break;
            }
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            uint32_t v[64];
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                if (jj * 16 < hn)
                    asm volatile(
                        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
                        "%12, %13, %14, %15}, [%16];"
                        : "=r"(v[16 * jj]), "=r"(v[16 * jj + 1]), "=r"(v[16 * jj + 2]), "=r"(v[16 * jj + 3]),
                          "=r"(v[16 * jj + 4]), "=r"(v[16 * jj + 5]), "=r"(v[16 * jj + 6]), "=r"(v[16 * jj + 7]),
                          "=r"(v[16 * jj + 8]), "=r"(v[16 * jj + 9]), "=r"(v[16 * jj + 10]), "=r"(v[16 * jj + 11]),
                          "=r"(v[16 * jj + 12]), "=r"(v[16 * jj + 13]), "=r"(v[16 * jj + 14]), "=r"(v[16 * jj + 15])
                        : "r"(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(sb * 128 + 64 * hf + 16 * jj)));
                else
#pragma unroll
                    for (int ii = 0; ii < 16; ++ii) v[16 * jj + ii] = 0u;
            }
            asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
            asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
            __syncwarp();
            if (lane == 0) mbar_arrive_one(&bar_free[sb]);
            const int e_base = m0 + q * 32;
            const size_t col0 = (size_t)c * kChunk + 64 * hf;
#pragma unroll
            for (int sbk = 0; sbk < 2; ++sbk) {
                if (32 * sbk >= hn) break;
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    *reinterpret_cast<float4*>(st + lane * 32 + 4 * (j ^ (lane & 7))) =
                        make_float4(__uint_as_float(v[32 * sbk + 4 * j]), __uint_as_float(v[32 * sbk + 4 * j + 1]),
                                    __uint_as_float(v[32 * sbk + 4 * j + 2]), __uint_as_float(v[32 * sbk + 4 * j + 3]));
                __syncwarp();
                const int jj = lane & 7;
#pragma unroll
                for (int rr = 0; rr < 8; ++rr) {
                    const int row = 4 * rr + (lane >> 3), e = e_base + row;
                    const int col = 32 * sbk + 4 * jj;
                    if (e < E && col < hn)
                        *reinterpret_cast<float4*>(w + (size_t)e * PC + col0 + col) =
                            *reinterpret_cast<const float4*>(st + row * 32 + 4 * (jj ^ (row & 7)));
                }
                __syncwarp();
            }
        }
    }
    __syncthreads();
    if (warp == kMmaWarp) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
    }
}

// ---------------------------------------------------------------------------
// Shared by the two VJP kernels below: warp-specialised pipelines in which 8
// producer warps split operand chunks into TF32 halves in shared memory and one
// more warp issues the MMAs. A chunk's slot is handed over by mbarriers: `full`
// (8 arrivals, one per producer warp, after each thread's proxy fence) and `empty`
// (the tcgen05.commit of the chunk's MMAs). No block-wide barrier inside the loop.
constexpr int kProducers = 256;               // 8 producer warps
constexpr int kPipeThreads = kProducers + 32; // + the MMA warp

// grad_w is read once: stream it past L2 (evict first) and L1.
__device__ __forceinline__ float4 ld_stream(const float* p, uint64_t policy) {
    float4 v;
    asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.f32 {%0, %1, %2, %3}, [%4], %5;"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "l"(p), "l"(policy));
    return v;
}

__device__ __forceinline__ uint64_t evict_first_policy() {
    uint64_t policy;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(policy));
    return policy;
}

__device__ __forceinline__ void st_split(unsigned char* hi, unsigned char* lo, float a, float b, float c, float d) {
    const float4 h = make_float4(tf32_round(a), tf32_round(b), tf32_round(c), tf32_round(d));
    *reinterpret_cast<float4*>(hi) = h;
    *reinterpret_cast<float4*>(lo) =
        make_float4(tf32_round(a - h.x), tf32_round(b - h.y), tf32_round(c - h.z), tf32_round(d - h.w));
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// A producer warp's hand-over of a filled slot: every thread's generic-proxy stores
// are made visible to the tensor core's proxy, then one lane arrives.
__device__ __forceinline__ void hand_over(uint64_t* full, int lane) {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncwarp();
    if (lane == 0) mbar_arrive(full);
}

__device__ __forceinline__ void mma_tf32(uint32_t d_tmem, uint64_t da, uint64_t db, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n .reg .pred pp;\n setp.ne.b32 pp, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, pp;\n}" ::"r"(d_tmem),
        "l"(da), "l"(db), "r"(idesc), "r"(acc)
        : "memory");
}

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// Shared-memory descriptor with explicit LBO / SBO (bytes), no swizzle.
__device__ __forceinline__ uint64_t smem_desc_bo(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | ((uint64_t)1 << 46);
}

// ---------------------------------------------------------------------------
// Backward: dL/dH [E][64] = grad_w [E][PC] W2^T on the tensor cores (M = 128 edges,
// N = 64 hidden units, K = PC in chunks of 64), with the per-edge rest of the VJP
// fused into the epilogue: dL/dz = dL/dH * SiLU'(z) (written out for grad_W1),
// dL/db = dL/dz W1^T, dL/dd = dL/db . db/dd and grad_r[e] += dL/dd r / |r|.
// The producers read the tile's grad_w chunk row segment by row segment (16 lanes x
// 16 bytes per edge), keep the next chunk in flight in registers, and store the
// TF32 halves K-major with LBO = 144 B between core matrices along K: the pad of
// 16 B puts the 8 lanes of a store phase (consecutive K groups of one edge) on 8
// distinct bank quads. W2 chunks (64 rows x 64 K, halves pre-split) arrive by bulk
// copies into two B slots.
constexpr int kKChunk = 64;
constexpr uint32_t kBwTileB = 64 * kKChunk * 4;                 // 16 KB: one half of a W2 chunk
constexpr uint32_t kBwLBO = 144, kBwSBO = 16 * kBwLBO;          // A: padded K-major, 64 K per row group
constexpr uint32_t kBwAHalf = 16 * kBwSBO;                      // 128 edges x 64 K, one TF32 half
constexpr uint32_t kBwOffB = 4 * kBwAHalf;                      // after the two A slots [slot][half]
constexpr uint32_t kBwOffW1 = kBwOffB + 4 * kBwTileB;           // after the two B slots [slot][half]
constexpr uint32_t kBwOffBars = kBwOffW1 + kBasis * kHidden * 4;
constexpr uint32_t kBwSmem = kBwOffBars + 64;
static_assert(kBwSmem <= 232448 && kBwOffBars % 16 == 0 && kBwLBO % 128 == 16, "radial backward shared memory");

// W2 [64][PC] as K-major B chunks: chunk q holds rows h = 0..63, K = columns 64q..64q+63.
__global__ void radial_tc_prepare_w2(const float* __restrict__ W2, int PC, int n_kc, float* __restrict__ hi,
                                     float* __restrict__ lo) {
    const long long total = (long long)n_kc * kHidden * kKChunk;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const int q = (int)(i / (kHidden * kKChunk)), rem = (int)(i % (kHidden * kKChunk));
        const int h = rem / kKChunk, k = rem % kKChunk, col = q * kKChunk + k;
        const float v = col < PC ? W2[(size_t)h * PC + col] : 0.f;
        const float vh = tf32_round(v);
        const size_t off = (size_t)q * (kBwTileB / 4) + tile_offset(h, k) / 4;
        hi[off] = vh;
        lo[off] = tf32_round(v - vh);
    }
}

__device__ __forceinline__ void load_w2(const float* Bhi, const float* Blo, int q, unsigned char* dst_hi,
                                        unsigned char* dst_lo, uint64_t* bar) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(2 * kBwTileB)
                 : "memory");
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst_hi)),
                 "l"(Bhi + (size_t)q * (kBwTileB / 4)), "r"(kBwTileB), "r"(smem_u32(bar))
                 : "memory");
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst_lo)),
                 "l"(Blo + (size_t)q * (kBwTileB / 4)), "r"(kBwTileB), "r"(smem_u32(bar))
                 : "memory");
}

__global__ void __launch_bounds__(kPipeThreads, 1)
    radial_tc_backward(int E, int PC, float rc, const float* __restrict__ r, const float* __restrict__ W1,
                       const float* __restrict__ Bhi, const float* __restrict__ Blo,
                       const float* __restrict__ grad_w, float* __restrict__ gZ, float* __restrict__ grad_r) {
    extern __shared__ __align__(1024) unsigned char smem[];
    float* w1s = reinterpret_cast<float*>(smem + kBwOffW1);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kBwOffBars);  // [2] A slot written
    uint64_t* empty = full + 2;                                         // [2] MMAs of a slot done
    uint64_t* bfull = full + 4;                                         // [2] W2 chunk arrived
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kBwOffBars + 48);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kBwOffBars + 52);
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    const int m0 = blockIdx.x * kRows;
    const int n_kc = (PC + kKChunk - 1) / kKChunk;
    auto a_half = [&](int s, int lo) { return smem + (uint32_t)(s * 2 + lo) * kBwAHalf; };
    auto b_half = [&](int s, int lo) { return smem + kBwOffB + (uint32_t)(s * 2 + lo) * kBwTileB; };

    if (warp == 0) {  // 64 fp32 accumulator columns (dL/dH of the tile)
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(64)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    for (int i = t; i < kBasis * kHidden; i += kPipeThreads) w1s[i] = __ldg(W1 + i);
    int issued[2] = {-1, -1};  // (thread 0) the last W2 chunk copied into each B slot
    if (t == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&full[i], kProducers / 32);
            mbar_init(&empty[i], 1);
            mbar_init(&bfull[i], 1);
        }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        for (int q = 0; q < 2 && q < n_kc; ++q) {
            load_w2(Bhi, Blo, q, b_half(q, 0), b_half(q, 1), &bfull[q]);
            issued[q] = q;
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = *tmem_slot;
    int last = -1;  // (MMA thread) the last chunk whose MMAs were committed

    if (warp < kProducers / 32) {
        // this thread's share of a chunk: 8 float4, edge i / 16 of the tile and column
        // group i % 16 of the chunk for i = t + 256 j
        const uint64_t policy = evict_first_policy();
        float4 g[2][8];
        auto load = [&](int b, int q) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int i = t + kProducers * j, e = m0 + (i >> 4), pc = q * kKChunk + 4 * (i & 15);
                g[b][j] = (e < E && pc < PC) ? ld_stream(grad_w + (size_t)e * PC + pc, policy)
                                             : make_float4(0.f, 0.f, 0.f, 0.f);
            }
        };
        if (n_kc > 0) load(0, 0);
        if (n_kc > 1) load(1, 1);
        bool stop = false;
        for (int q0 = 0; q0 < n_kc && !stop; q0 += 2) {
#pragma unroll
            for (int b = 0; b < 2; ++b) {
                const int q = q0 + b;
                // warp-uniform decisions: the hand-over below synchronises the warp
                if (q >= n_kc || __any_sync(0xffffffffu, *abort_flag != 0)) {
                    stop = true;
                    break;
                }
                if (q >= 2) {  // slot b was read by the MMAs of chunk q - 2
                    if (!__all_sync(0xffffffffu, mbar_wait(&empty[b], ((q - 2) >> 1) & 1))) {
                        if (lane == 0) atomicOr((int*)abort_flag, 1);
                        stop = true;
                        break;
                    }
                    if (t == 0) {
                        load_w2(Bhi, Blo, q, b_half(b, 0), b_half(b, 1), &bfull[b]);
                        issued[b] = q;
                    }
                }
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int i = t + kProducers * j, el = i >> 4;
                    const uint32_t off = (uint32_t)(el >> 3) * kBwSBO + (uint32_t)(i & 15) * kBwLBO + (el & 7) * 16;
                    st_split(a_half(b, 0) + off, a_half(b, 1) + off, g[b][j].x, g[b][j].y, g[b][j].z, g[b][j].w);
                }
                if (q + 2 < n_kc) load(b, q + 2);  // in flight while this chunk is multiplied
                hand_over(&full[b], lane);
            }
        }
    } else if (lane == 0) {  // the MMA warp
        const uint32_t idesc = instr_desc(kHidden);  // N = 64
        for (int q = 0; q < n_kc; ++q) {
            const int b = q & 1;
            if (*abort_flag) break;
            if (!mbar_wait(&full[b], (q >> 1) & 1) || !mbar_wait(&bfull[b], (q >> 1) & 1)) {
                atomicOr((int*)abort_flag, 1);
                break;
            }
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            const uint32_t A[3] = {smem_u32(a_half(b, 0)), smem_u32(a_half(b, 0)), smem_u32(a_half(b, 1))};
            const uint32_t B[3] = {smem_u32(b_half(b, 0)), smem_u32(b_half(b, 1)), smem_u32(b_half(b, 0))};
            for (int s = 0; s < kKChunk / 8; ++s)
                for (int p = 0; p < 3; ++p)
                    mma_tf32(tmem, smem_desc_bo(A[p] + s * 2 * kBwLBO, kBwLBO, kBwSBO),
                             smem_desc_bo(B[p] + s * 2 * kLBO, kLBO, kSBO), idesc, (q | s | p) ? 1u : 0u);
            mma_commit(&empty[b]);
            last = q;
        }
    }
    // the accumulator is complete once the last chunk's MMAs are
    if (warp < 4 && !*abort_flag && n_kc > 0 && !mbar_wait(&empty[(n_kc - 1) & 1], ((n_kc - 1) >> 1) & 1))
        atomicOr((int*)abort_flag, 1);
    __syncthreads();
    const int e = m0 + t;
    if (!*abort_flag && warp < 4) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        uint32_t g[64];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj)
            asm volatile(
                "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
                "%14, %15}, [%16];"
                : "=r"(g[16 * jj]), "=r"(g[16 * jj + 1]), "=r"(g[16 * jj + 2]), "=r"(g[16 * jj + 3]),
                  "=r"(g[16 * jj + 4]), "=r"(g[16 * jj + 5]), "=r"(g[16 * jj + 6]), "=r"(g[16 * jj + 7]),
                  "=r"(g[16 * jj + 8]), "=r"(g[16 * jj + 9]), "=r"(g[16 * jj + 10]), "=r"(g[16 * jj + 11]),
                  "=r"(g[16 * jj + 12]), "=r"(g[16 * jj + 13]), "=r"(g[16 * jj + 14]), "=r"(g[16 * jj + 15])
                : "r"(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)(16 * jj)));
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
        if (e < E) {
            const float x = __ldg(r + 3 * (size_t)e), y = __ldg(r + 3 * (size_t)e + 1), z = __ldg(r + 3 * (size_t)e + 2);
            const float d = sqrtf(x * x + y * y + z * z);
            const float c = sqrtf(2.f / rc);
            float b[kBasis], db[kBasis], gb[kBasis];
#pragma unroll
            for (int n = 0; n < kBasis; ++n) {
                const float kk = (float)(n + 1) * kPi / rc;
                gb[n] = 0.f;
                if (d >= 1e-12f) {
                    float sn, cs;
                    sincosf(kk * d, &sn, &cs);
                    b[n] = c * sn / d;
                    db[n] = c * (kk * cs / d - sn / (d * d));
                } else {
                    b[n] = c * kk;
                    db[n] = 0.f;
                }
            }
            float4* gz_row = reinterpret_cast<float4*>(gZ + (size_t)e * kHidden);
#pragma unroll
            for (int k4 = 0; k4 < kHidden; k4 += 4) {
                float out[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int k = k4 + j;
                    float zz = 0.f;
#pragma unroll
                    for (int n = 0; n < kBasis; ++n) zz = fmaf(b[n], w1s[n * kHidden + k], zz);
                    const float sg = 1.f / (1.f + expf(-zz));
                    const float gz = __uint_as_float(g[k]) * (sg * (1.f + zz * (1.f - sg)));
                    out[j] = gz;
#pragma unroll
                    for (int n = 0; n < kBasis; ++n) gb[n] = fmaf(gz, w1s[n * kHidden + k], gb[n]);
                }
                gz_row[k4 / 4] = make_float4(out[0], out[1], out[2], out[3]);
            }
            float dd = 0.f;
#pragma unroll
            for (int n = 0; n < kBasis; ++n) dd = fmaf(gb[n], db[n], dd);
            if (d >= 1e-12f) {
                const float f = dd / d;
                grad_r[3 * (size_t)e] += f * x;
                grad_r[3 * (size_t)e + 1] += f * y;
                grad_r[3 * (size_t)e + 2] += f * z;
            }
        }
    }
    __syncthreads();
    if (*abort_flag) {  // leave nothing in flight on the freed TMEM and shared memory: one bounded wait each
        if (t == 0) atomicOr(&g_fault, 1);
        if (t == kProducers && last >= 0) mbar_wait(&empty[last & 1], (last >> 1) & 1);
        if (t == 0)
            for (int b = 0; b < 2; ++b)
                if (issued[b] >= 0) mbar_wait(&bfull[b], (issued[b] >> 1) & 1);
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(64) : "memory");
}

// ---------------------------------------------------------------------------
// grad_W2 [64][PC] = H^T grad_w: a reduction over the edges, computed transposed on
// the tensor cores as D [pc][h] = sum_e grad_w[e][pc] H[e][h] (M = 128 columns of w
// per accumulator, N = 64 hidden units, K = edges). Both operands lie edge by edge in
// memory, so they are transposed on the way into shared memory: each producer thread
// loads a 4-edge x 4-column block as four float4 rows, transposes it in registers and
// stores four 16-byte runs along K. The operands are K-major with the 8 core matrices
// of a 32-edge chunk adjacent along K (LBO = 128 B) and row groups kGwSBO = 1040 B
// apart: the pad of 16 B puts the 8 lanes of a store phase (two row groups per 4
// lanes) on 8 distinct bank quads.
//
// Per CTA (one per SM): 256 columns of w (two accumulators of 64 TMEM columns) and
// one split of the edges, in chunks of 32 edges. Each producer thread holds its part
// of the next chunk of grad_w and H in registers (loaded while the current chunk is
// converted and multiplied), splits it into TF32 halves and stores them into one of
// two operand slots; the MMA warp issues 4 K-steps x 2 tiles x 3 products per chunk.
// The split's partial sums are written to part [split][64][PC]; the caller adds the
// splits in a fixed order.
constexpr int kGwEdges = 32;                        // edges per chunk (4 K-steps)
constexpr int kGwCols = 256;                        // columns of w per CTA (2 x M = 128)
constexpr uint32_t kGwSBO = kGwEdges * 4 * 8 + 16;  // one row group of a chunk, padded
constexpr uint32_t kGwAHalf = 16 * kGwSBO;          // 128 columns x 32 edges, one TF32 half
constexpr uint32_t kGwBHalf = 8 * kGwSBO;           // 64 hidden units x 32 edges
constexpr uint32_t kGwOffB = 2 * 2 * 2 * kGwAHalf;  // [slot][half][tile] A, then [slot][half] B
constexpr uint32_t kGwOffBars = kGwOffB + 2 * 2 * kGwBHalf;
constexpr uint32_t kGwSmem = kGwOffBars + 64;
static_assert(kGwSmem <= 232448 && kGwOffBars % 16 == 0 && kGwSBO % 128 == 16, "grad_W2 kernel shared memory");

// Rows 4 e4 .. 4 e4 + 3 (edges) of a 4 x 4 block whose column j is row `row0 + j` of
// the operand: column j goes to K-major position (row0 + j, 4 e4 .. 4 e4 + 3).
__device__ __forceinline__ void st_block(unsigned char* hi, unsigned char* lo, int row0, int e4, const float4 (&v)[4]) {
    const uint32_t base = (uint32_t)(row0 >> 3) * kGwSBO + (uint32_t)e4 * kLBO + (uint32_t)(row0 & 7) * 16;
    st_split(hi + base, lo + base, v[0].x, v[1].x, v[2].x, v[3].x);
    st_split(hi + base + 16, lo + base + 16, v[0].y, v[1].y, v[2].y, v[3].y);
    st_split(hi + base + 32, lo + base + 32, v[0].z, v[1].z, v[2].z, v[3].z);
    st_split(hi + base + 48, lo + base + 48, v[0].w, v[1].w, v[2].w, v[3].w);
}

__global__ void __launch_bounds__(kPipeThreads, 1)
    radial_tc_grad_w2(int E, int PC, int chunks_per_split, const float* __restrict__ grad_w,
                      const float* __restrict__ H, float* __restrict__ part) {
    extern __shared__ __align__(1024) unsigned char smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kGwOffBars);  // [2] slot written
    uint64_t* empty = full + 2;                                         // [2] MMAs of a slot done
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kGwOffBars + 32);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kGwOffBars + 36);
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    const int pc0 = blockIdx.x * kGwCols;
    const int n_tiles = PC - pc0 > kRows ? 2 : 1;
    const int n_chunks = (E + kGwEdges - 1) / kGwEdges;
    const int c_begin = blockIdx.y * chunks_per_split;
    const int nq = max(0, min(n_chunks, c_begin + chunks_per_split) - c_begin);
    auto a_half = [&](int slot, int lo, int mt) { return smem + (uint32_t)((slot * 2 + lo) * 2 + mt) * kGwAHalf; };
    auto b_half = [&](int slot, int lo) { return smem + kGwOffB + (uint32_t)(slot * 2 + lo) * kGwBHalf; };

    if (warp == 0) {  // two accumulators of 64 fp32 columns
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(128)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (t == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&full[i], kProducers / 32);
            mbar_init(&empty[i], 1);
        }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = *tmem_slot;
    int last = -1;  // (MMA thread) the last chunk whose MMAs were committed

    if (warp < kProducers / 32) {
        // this thread's share of a chunk: two 4 x 4 blocks of grad_w (edge quad i / 64,
        // column group i % 64 for i = t + 256 j) and, for t < 128, one of H (edge quad
        // t / 16, hidden group t % 16)
        const uint64_t policy = evict_first_policy();
        float4 g[2][2][4], hv[2][4];
        auto load = [&](int b, int q) {
            const int e0 = (c_begin + q) * kGwEdges;
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int i = t + kProducers * j, pc = pc0 + 4 * (i & 63);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int e = e0 + 4 * (i >> 6) + k;
                    g[b][j][k] = (e < E && pc < PC) ? ld_stream(grad_w + (size_t)e * PC + pc, policy)
                                                    : make_float4(0.f, 0.f, 0.f, 0.f);
                }
            }
            if (t < 128) {
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int e = e0 + 4 * (t >> 4) + k;
                    hv[b][k] = e < E ? __ldg(reinterpret_cast<const float4*>(H + (size_t)e * kHidden + 4 * (t & 15)))
                                     : make_float4(0.f, 0.f, 0.f, 0.f);
                }
            }
        };
        if (nq > 0) load(0, 0);
        if (nq > 1) load(1, 1);
        bool stop = false;
        for (int q0 = 0; q0 < nq && !stop; q0 += 2) {
#pragma unroll
            for (int b = 0; b < 2; ++b) {
                const int q = q0 + b;
                // warp-uniform decisions: the hand-over below synchronises the warp
                if (q >= nq || __any_sync(0xffffffffu, *abort_flag != 0)) {
                    stop = true;
                    break;
                }
                if (q >= 2 && !__all_sync(0xffffffffu, mbar_wait(&empty[b], ((q - 2) >> 1) & 1))) {
                    if (lane == 0) atomicOr((int*)abort_flag, 1);  // slot b still read by chunk q - 2
                    stop = true;
                    break;
                }
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int i = t + kProducers * j, grp = i & 63;
                    st_block(a_half(b, 0, grp >> 5), a_half(b, 1, grp >> 5), 4 * (grp & 31), i >> 6, g[b][j]);
                }
                if (t < 128) st_block(b_half(b, 0), b_half(b, 1), 4 * (t & 15), t >> 4, hv[b]);
                if (q + 2 < nq) load(b, q + 2);  // in flight while this chunk is multiplied
                hand_over(&full[b], lane);
            }
        }
    } else if (lane == 0) {  // the MMA warp
        const uint32_t idesc = instr_desc(kHidden);  // M = 128, N = 64, both K-major
        for (int q = 0; q < nq; ++q) {
            const int b = q & 1;
            if (*abort_flag) break;
            if (!mbar_wait(&full[b], (q >> 1) & 1)) {
                atomicOr((int*)abort_flag, 1);
                break;
            }
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            for (int s = 0; s < kGwEdges / 8; ++s)
                for (int mt = 0; mt < n_tiles; ++mt) {
                    // A_hi B_hi + A_hi B_lo + A_lo B_hi
                    const uint32_t A[3] = {smem_u32(a_half(b, 0, mt)), smem_u32(a_half(b, 0, mt)),
                                           smem_u32(a_half(b, 1, mt))};
                    const uint32_t B[3] = {smem_u32(b_half(b, 0)), smem_u32(b_half(b, 1)), smem_u32(b_half(b, 0))};
                    for (int p = 0; p < 3; ++p)
                        mma_tf32(tmem + (uint32_t)(mt * kHidden), smem_desc_bo(A[p] + s * 2 * kLBO, kLBO, kGwSBO),
                                 smem_desc_bo(B[p] + s * 2 * kLBO, kLBO, kGwSBO), idesc, (q | s | p) ? 1u : 0u);
                }
            mma_commit(&empty[b]);
            last = q;
        }
    }
    // all MMAs are complete once the last chunk's are
    if (warp < kProducers / 32 && !*abort_flag && nq > 0 && !mbar_wait(&empty[(nq - 1) & 1], ((nq - 1) >> 1) & 1))
        atomicOr((int*)abort_flag, 1);
    __syncthreads();
    const int mt = warp >> 2, pc = pc0 + mt * kRows + (warp & 3) * 32 + lane;
    if (!*abort_flag && warp < kProducers / 32 && mt < n_tiles) {
        float* out = part + (size_t)blockIdx.y * kHidden * PC;
        if (nq == 0) {  // an empty split contributes zeros
            if (pc < PC)
                for (int h = 0; h < kHidden; ++h) out[(size_t)h * PC + pc] = 0.f;
        } else {
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            uint32_t v[64];
#pragma unroll
            for (int jj = 0; jj < 4; ++jj)
                asm volatile(
                    "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
                    "%13, %14, %15}, [%16];"
                    : "=r"(v[16 * jj]), "=r"(v[16 * jj + 1]), "=r"(v[16 * jj + 2]), "=r"(v[16 * jj + 3]),
                      "=r"(v[16 * jj + 4]), "=r"(v[16 * jj + 5]), "=r"(v[16 * jj + 6]), "=r"(v[16 * jj + 7]),
                      "=r"(v[16 * jj + 8]), "=r"(v[16 * jj + 9]), "=r"(v[16 * jj + 10]), "=r"(v[16 * jj + 11]),
                      "=r"(v[16 * jj + 12]), "=r"(v[16 * jj + 13]), "=r"(v[16 * jj + 14]), "=r"(v[16 * jj + 15])
                    : "r"(tmem + ((uint32_t)((warp & 3) * 32) << 16) + (uint32_t)(mt * kHidden + 16 * jj)));
            asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
            if (pc < PC)
#pragma unroll
                for (int h = 0; h < kHidden; ++h) out[(size_t)h * PC + pc] = __uint_as_float(v[h]);
        }
    }
    __syncthreads();
    if (*abort_flag) {
        if (t == 0) atomicOr(&g_fault, 1);
        if (t == kProducers && last >= 0) mbar_wait(&empty[last & 1], (last >> 1) & 1);  // nothing left in flight
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(128) : "memory");
}

}  // namespace rtc

int radial_tc_grad_w2_splits(int E, int PC) {
    const int n_cta = (PC + rtc::kGwCols - 1) / rtc::kGwCols;
    const int n_chunks = (E + rtc::kGwEdges - 1) / rtc::kGwEdges;
    int s = 148 / n_cta;                     // one wave of one CTA per SM
    const int by_size = n_chunks / 8;        // at least 8 chunks (256 edges) per split
    if (s > by_size) s = by_size;
    return s < 1 ? 1 : s;
}

cudaError_t radial_tc_grad_w2(int E, int PC, const float* grad_w, const float* H, float* part, int splits,
                              cudaStream_t s) {
    const int n_chunks = (E + rtc::kGwEdges - 1) / rtc::kGwEdges;
    const int per = (n_chunks + splits - 1) / splits;
    cudaError_t err = cudaFuncSetAttribute(rtc::radial_tc_grad_w2, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)rtc::kGwSmem);
    if (err != cudaSuccess) return err;
    dim3 grid((PC + rtc::kGwCols - 1) / rtc::kGwCols, splits);
    rtc::radial_tc_grad_w2<<<grid, rtc::kPipeThreads, rtc::kGwSmem, s>>>(E, PC, per, grad_w, H, part);
    return cudaGetLastError();
}

size_t radial_tc_prepare_bytes(int PC) {
    const int n_chunks = (PC + rtc::kChunk - 1) / rtc::kChunk;
    return 2 * (size_t)n_chunks * rtc::kTileBytes;
}

bool radial_tc_supported(int nb, int hidden, int PC) {
    return hidden == rtc::kHidden && nb == rtc::kBasis && PC % 16 == 0;
}

cudaError_t radial_tc_forward(int E, int nb, int PC, float rc, const float* r, const float* W1, const float* W2,
                              float* w, void* ws, cudaStream_t s) {
    if (E == 0) return cudaSuccess;
    const int n_chunks = (PC + rtc::kChunk - 1) / rtc::kChunk;
    float* hi = static_cast<float*>(ws);
    float* lo = hi + (size_t)n_chunks * (rtc::kTileBytes / 4);
    rtc::radial_tc_prepare<<<256, 256, 0, s>>>(W2, PC, n_chunks, hi, lo);
    const size_t smem = rtc::kSmemBytes;
    cudaError_t err = cudaFuncSetAttribute(rtc::radial_tc_forward, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)smem);
    if (err != cudaSuccess) return err;
    const int tiles = (E + rtc::kRows - 1) / rtc::kRows;
    rtc::radial_tc_forward<<<tiles < 148 ? tiles : 148, rtc::kFwdThreads, smem, s>>>(E, PC, nb, rc, r, W1, hi, lo, w);
    return cudaGetLastError();
}

size_t radial_tc_backward_prepare_bytes(int PC) {
    const int n_kc = (PC + rtc::kKChunk - 1) / rtc::kKChunk;
    return 2 * (size_t)n_kc * rtc::kBwTileB;
}

cudaError_t radial_tc_backward(int E, int PC, float rc, const float* r, const float* W1, const float* W2,
                               const float* grad_w, float* gZ, float* grad_r, void* prep, cudaStream_t s) {
    if (E == 0) return cudaSuccess;
    const int n_kc = (PC + rtc::kKChunk - 1) / rtc::kKChunk;
    float* hi = static_cast<float*>(prep);
    float* lo = hi + (size_t)n_kc * (rtc::kBwTileB / 4);
    rtc::radial_tc_prepare_w2<<<256, 256, 0, s>>>(W2, PC, n_kc, hi, lo);
    cudaError_t err = cudaFuncSetAttribute(rtc::radial_tc_backward, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)rtc::kBwSmem);
    if (err != cudaSuccess) return err;
    rtc::radial_tc_backward<<<(E + rtc::kRows - 1) / rtc::kRows, rtc::kPipeThreads, rtc::kBwSmem, s>>>(
        E, PC, rc, r, W1, hi, lo, grad_w, gZ, grad_r);
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
