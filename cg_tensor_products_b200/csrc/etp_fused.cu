// Radial weights fused into the tensor product (forward): the per-edge weights
// w[e] = SiLU(b(|r_e|) W1) W2 are produced on the tensor cores tile by tile and
// consumed from tensor memory by the tensor product in the same kernel; w never
// exists in global memory.
//
// Passages: "High-performance training and inference for deep equivariant
// interatomic potentials", section "제안 방법" (a fused tensor-product kernel
// without materialised intermediates; the per-edge weights of the Allegro tensor
// product are a learned function of the edge length); "Scaling the leading
// accuracy of deep equivariant models to biomolecular simulations of realistic
// size", section "提出的方法" (the tensor product as a single contraction).
//
// Decomposition. A CTA (one per SM) owns a contiguous range of CSR edges, split
// into four equal contiguous warp ranges; tile i holds the i-th 32-edge chunk of
// every warp range, so TMEM lane 32w + t is edge t of warp w's chunk. Per tile:
//   1. each consumer thread (warps 0-3, one edge each) builds its edge's frame and
//      Wigner matrices in registers and its row of the hidden layer
//      H = SiLU(b(|r|) W1), split into TF32 halves, into the A operand (128 x 64,
//      K-major);
//   2. the channels are taken in slices of cs channels; for slice s the B operand
//      is the matching columns of W2 for all P paths (N = P cs, padded to 16;
//      pre-split and pre-arranged in global memory, brought in by bulk copies into
//      two shared-memory slots) and one thread issues 8 K-steps x 3 products of
//      tcgen05.mma (3xTF32) into one of three TMEM accumulators;
//   3. the consumers read their edge's weights of the slice from TMEM
//      (tcgen05.ld), rotate x[src] into the edge frame, apply the sparse
//      couplings, rotate back, and sum the messages of equal destinations across
//      the warp in a fixed order (a transpose through shared memory, one column
//      per lane). A row that continues into the warp's next chunk is carried in a
//      per-warp scratch row; a finished row is stored once, or, when another
//      warp range holds part of it, added by a vector reduction onto the zeroed
//      output (two addends: the result is still bitwise repeatable).
// The slices' MMAs run while the consumers work on earlier slices (three TMEM
// accumulators, two operand slots). Every wait is bounded; on time-out the kernel
// raises its fault flag, stops issuing work, and leaves with nothing in flight.
#include <cuda_runtime.h>

#include <cstdint>

#include "etp_frame.cuh"
#include "etp_tcgen05.cuh"

namespace etp {
namespace fused {

constexpr int kRows = 128;                    // edges per tile (MMA M)
constexpr int kBasis = 8;                     // Bessel functions
constexpr int kHidden = 64;                   // hidden width (MMA K)
constexpr int kAccBufs = 3;                   // TMEM accumulators in flight
constexpr uint32_t kLBO = 128, kSBO = 2048;   // K-major operand: K = 64 per 8-row group
constexpr uint32_t kAHalf = kRows * kHidden * 4;  // 32 KB
constexpr int kWaitLimit = 1 << 22;
constexpr float kPi = 3.14159265358979323846f;

__device__ int g_fault;

// Paths in "l3-major" order (l3 ascending, plan order inside): within a channel
// pair's block of TMEM columns, the paths into one l3 are contiguous, so each l3
// group of weights is one TMEM load.
template <int L, bool O3>
struct L3Order {
    using PS = PathSet<L, O3>;
    static constexpr int P = PS::P;
    static constexpr int start(int l3) {
        int n = 0;
        for (int p = 0; p < P; ++p)
            if (PS::path(p).l3 < l3) ++n;
        return n;
    }
    static constexpr int count(int l3) { return start(l3 + 1) - start(l3); }
    static constexpr int pos(int p) {  // position of plan path p
        const int l3 = PS::path(p).l3;
        int n = start(l3);
        for (int q = 0; q < p; ++q)
            if (PS::path(q).l3 == l3) ++n;
        return n;
    }
    static constexpr int cols_pow2(int l3) {  // TMEM load width for the group (pairs: 2 columns a path)
        const int c = 2 * count(l3);
        return c <= 8 ? 8 : (c <= 16 ? 16 : 32);
    }
};

struct FwdArgs {
    int N, E;
    const int32_t* row_ptr;
    const int32_t* src;
    const float* r;
    const float* x;
    const float* W1;   // [8][64]
    const float* w2s;  // slices: [S][2 halves][Npad x 64, K-major]
    float* out;
    float* carry;      // [ntasks][4 warps][C/2 pairs][32]
    float rc;
    int C, cs, S, Npad, ntasks;
};

// out (+)= D_l in  (TR = false)  or  D_l^T in  (TR = true); the Wigner matrices
// are this thread's registers (D_1 from the frame's rotation).
template <int l, bool TR>
__device__ __forceinline__ void rot_reg(const frame::Frame& f, const float (&d2)[25], const float (&d3)[49],
                                        const float2* in, float2* out) {
    constexpr int d = 2 * l + 1;
    if constexpr (l == 0) {
        out[0] = in[0];
    } else {
#pragma unroll
        for (int a = 0; a < d; ++a) {
            float2 acc = frame::f2_zero();
#pragma unroll
            for (int b = 0; b < d; ++b) {
                const int ra = TR ? b : a, cb = TR ? a : b;
                float m;
                if constexpr (l == 1)
                    m = frame::d1(f, ra, cb);
                else if constexpr (l == 2)
                    m = d2[ra * 5 + cb];
                else
                    m = d3[ra * 7 + cb];
                frame::f2_fma(acc, m, in[b]);
            }
            out[a] = acc;
        }
    }
}

// Combined frame weights of the (l1, l3) group from the l3 group's weights v
// (column 2j: channel c, 2j + 1: channel c + 1 of the group's j-th path).
template <int L, bool O3, int l1, int l3, int NC>
__device__ __forceinline__ void group_weights_reg(const float (&v)[NC], float2 (&We)[4], float2 (&Wo)[4]) {
    using O = L3Order<L, O3>;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        We[m] = frame::f2_zero();
        Wo[m] = frame::f2_zero();
    }
    static_for<0, L + 1>([&](auto l2c) {
        constexpr int l2 = decltype(l2c)::value;
        if constexpr (PathSet<L, O3>::allowed(l1, l2, l3)) {
            constexpr int jj = O::pos(frame::path_index<L, O3>(l1, l2, l3)) - O::start(l3);
            static_assert(2 * jj + 1 < NC, "group load width");
            const float2 w = make_float2(v[2 * jj], v[2 * jj + 1]);
            constexpr bool odd = (l1 + l2 + l3) % 2 == 1;
            static_for<0, frame::cmin(l1, l3) + 1>([&](auto mc) {
                constexpr int mu = decltype(mc)::value;
                constexpr float b = (float)etp_gen::kFrameB[l1][l2][l3][mu];
                if constexpr (b != 0.f) {
                    if constexpr (odd)
                        frame::f2_fma(Wo[mu], b, w);
                    else
                        frame::f2_fma(We[mu], b, w);
                }
            });
        }
    });
}

__device__ __forceinline__ bool wait_live(uint64_t* bar, unsigned parity, bool& live) {
    if (!live) return false;
    if (!tc::mbar_wait(bar, parity, kWaitLimit)) {
        live = false;
        atomicOr(&g_fault, 1);
    }
    return live;
}

__device__ __forceinline__ void red_add(float* p, float v) {
    asm volatile("red.global.add.f32 [%0], %1;" ::"l"(p), "f"(v) : "memory");
}

// Shared memory: A (two TF32 halves, 64 KB), two B slots of 2 x Npad x 256 B, the
// consumers' transpose stage (NW warps x 32 rows of 2D + 1 floats), W1, the
// mbarriers and the TMEM address.
struct Smem {
    uint32_t slot_bytes, off_b, off_stage, off_w1, off_bars, total;
};
__host__ __device__ constexpr Smem smem_layout(int Npad, int D, int NW) {
    Smem s{};
    s.slot_bytes = 2u * (uint32_t)Npad * (kHidden * 4);
    s.off_b = 2 * kAHalf;
    s.off_stage = s.off_b + 2 * s.slot_bytes;
    s.off_w1 = s.off_stage + (uint32_t)((NW * 32 * (2 * D + 1) * 4 + 15) / 16 * 16);
    s.off_bars = s.off_w1 + kBasis * kHidden * 4;
    s.total = s.off_bars + 16 * 8;
    return s;
}
// Consumer warps: eight (two per TMEM lane quarter, splitting the channel pairs)
// where the stage fits in shared memory, else four.
// (Nine warps put three on one scheduler, whose register file then allows 168 per
// thread: enough for L <= 2, not for the L = 3 Wigner matrices.)
template <int L>
constexpr int consumer_warps() { return L <= 2 ? 8 : 4; }

template <int L, bool O3>
__global__ void __launch_bounds__(consumer_warps<L>() * 32 + 32, 1) etp_fused_fwd_kernel(FwdArgs a) {
    using namespace frame;
    using O = L3Order<L, O3>;
    constexpr int D = (L + 1) * (L + 1);
    constexpr int P = PathSet<L, O3>::P;
    constexpr int STR = 2 * D + 1;
    constexpr int NW = consumer_warps<L>();  // consumer warps
    constexpr int NH = NW / 4;               // consumer warps per TMEM lane quarter
    constexpr int kConsumers = NW * 32;
    constexpr bool kPrefetchX = L <= 2;      // registers for the next pair's x
    extern __shared__ __align__(1024) unsigned char smem[];
    const Smem lay = smem_layout(a.Npad, D, NW);
    unsigned char* A_hi = smem;
    unsigned char* A_lo = smem + kAHalf;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + lay.off_bars);
    uint64_t* a_full = bars + 0;       // consumers wrote A (one arrival per consumer thread)
    uint64_t* a_empty = bars + 1;      // the tile's MMAs are done (commit)
    uint64_t* b_full = bars + 2;       // [2] slice operand arrived (bulk copy)
    uint64_t* b_empty = bars + 4;      // [2] slice MMAs done (commit)
    uint64_t* acc_full = bars + 6;     // [3] accumulator ready (commit)
    uint64_t* acc_empty = bars + 9;    // [3] consumers done with it (one arrival per consumer warp)
    uint64_t* done_bar = bars + 12;    // every MMA done (commit, once)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 13);
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;

    // the CTA's edges [k0, k1), four warp ranges, tiles of one 32-edge chunk each
    const int task = blockIdx.x;
    int k0, k1;
    task_range(a.E, task, a.ntasks, k0, k1);
    const long long len = (long long)k1 - k0;
    const int per_warp = (int)((len + 3) / 4);
    const int ntiles = (per_warp + 31) / 32;
    const int S = a.S;
    const int G = ntiles * S;

    float* w1s = reinterpret_cast<float*>(smem + lay.off_w1);
    for (int k = t; k < kBasis * kHidden; k += kConsumers + 32) w1s[k] = __ldg(a.W1 + k);
    if (warp == NW) tc::tmem_alloc(tmem_slot, 512);
    if (t == kConsumers) {
        tc::mbar_init(a_full, kConsumers);
        tc::mbar_init(a_empty, 1);
        for (int i = 0; i < 2; ++i) tc::mbar_init(&b_full[i], 1), tc::mbar_init(&b_empty[i], 1);
        for (int i = 0; i < kAccBufs; ++i) tc::mbar_init(&acc_full[i], 1), tc::mbar_init(&acc_empty[i], NW);
        tc::mbar_init(done_bar, 1);
        tc::mbar_fence_init();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    bool live = true;

    if (warp == NW) {
        // ---------------- bulk copies of the slice operands and the MMAs ----------------
        if (lane == 0 && G > 0) {
            auto load = [&](int g) {
                const int slot = g & 1, s = g % S;
                unsigned char* dst = smem + lay.off_b + slot * lay.slot_bytes;
                const unsigned char* srcp = reinterpret_cast<const unsigned char*>(a.w2s) + (size_t)s * lay.slot_bytes;
                tc::mbar_expect_tx(&b_full[slot], lay.slot_bytes);
                tc::bulk_g2s(dst, srcp, lay.slot_bytes / 2, &b_full[slot]);
                tc::bulk_g2s(dst + lay.slot_bytes / 2, srcp + lay.slot_bytes / 2, lay.slot_bytes / 2, &b_full[slot]);
            };
            int issued = 0;  // slice operands whose copies were issued
            load(0);
            issued = 1;
            if (G > 1) load(1), issued = 2;
            const uint32_t idesc = tc::idesc_tf32(kRows, a.Npad);
            int committed = 0;
            for (int g = 0; g < G && live; ++g) {
                const int i = g / S, s = g - i * S, slot = g & 1, buf = g % kAccBufs;
                if (s == 0 && !wait_live(a_full, i & 1, live)) break;
                if (!wait_live(&b_full[slot], (g >> 1) & 1, live)) break;
                if (g >= kAccBufs && !wait_live(&acc_empty[buf], ((g / kAccBufs) + 1) & 1, live)) break;
                tc::fence_after_sync();
                const uint32_t d_tmem = tmem + (uint32_t)(buf * a.Npad);
                const uint32_t bh = tc::smem_u32(smem + lay.off_b + slot * lay.slot_bytes);
                const uint32_t bl = bh + lay.slot_bytes / 2;
                const uint32_t ah = tc::smem_u32(A_hi), al = tc::smem_u32(A_lo);
                for (int ks = 0; ks < kHidden / 8; ++ks) {
                    const uint32_t o = ks * 2 * kLBO;
                    tc::mma_tf32(d_tmem, tc::smem_desc(ah + o, kLBO, kSBO), tc::smem_desc(bh + o, kLBO, kSBO), idesc,
                                 ks ? 1u : 0u);
                    tc::mma_tf32(d_tmem, tc::smem_desc(ah + o, kLBO, kSBO), tc::smem_desc(bl + o, kLBO, kSBO), idesc, 1u);
                    tc::mma_tf32(d_tmem, tc::smem_desc(al + o, kLBO, kSBO), tc::smem_desc(bh + o, kLBO, kSBO), idesc, 1u);
                }
                tc::mma_commit(&acc_full[buf]);
                tc::mma_commit(&b_empty[slot]);
                if (s == S - 1) tc::mma_commit(a_empty);
                committed = g + 1;
                // refill the other slot with operand g + 1 once the MMAs of g - 1 are done
                if (g >= 1 && g + 1 < G) {
                    if (!wait_live(&b_empty[(g + 1) & 1], ((g - 1) >> 1) & 1, live)) break;
                    load(g + 1);
                    issued = g + 2;
                }
            }
            // leave nothing in flight: every MMA, and every copy that was issued
            if (committed > 0) {
                tc::mma_commit(done_bar);
                tc::mbar_wait(done_bar, 0, kWaitLimit);
            }
            for (int g = committed; g < issued; ++g) tc::mbar_wait(&b_full[g & 1], (g >> 1) & 1, kWaitLimit);
        }
    } else {
        // ---------------- consumers: one edge per thread ----------------
        // warp = quarter + 4 half: the quarter fixes the TMEM lanes (edges), the half
        // the channel pairs of each slice (pairs q with q % NH == half)
        const int quarter = warp & 3, half = warp >> 2;
        const int ra = k0 + (int)(len * quarter / 4), rb = k0 + (int)(len * (quarter + 1) / 4);
        const float2* x2 = reinterpret_cast<const float2*>(a.x);
        const int C2 = a.C / 2, pairs = a.cs / 2;
        float* stage = reinterpret_cast<float*>(smem + lay.off_stage) + warp * 32 * STR;
        float* carry = a.carry + ((size_t)(task * 4 + quarter) * C2) * 32 + lane;
        const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
        int cur_row = ra < rb ? segment_of(a.row_ptr, a.N, ra) : 0;
        bool carried = false;  // warp-uniform: this chunk's first row continues the previous chunk's last
        unsigned char* arow_hi = A_hi + tc::kmajor_offset(quarter * 32 + lane, 0, kLBO, kSBO);
        unsigned char* arow_lo = A_lo + tc::kmajor_offset(quarter * 32 + lane, 0, kLBO, kSBO);
        const int kh0 = half * (kHidden / NH), kh1 = kh0 + kHidden / NH;  // this warp's hidden units of A
        // this warp's channel pairs: gp = s * pairs + q with gp % NH == half

        for (int i = 0; i < ntiles; ++i) {
            const int cb = ra + 32 * i, ce = min(cb + 32, rb);
            const int nrows = max(0, ce - cb);
            const int e = cb + lane;
            const bool has = lane < nrows;
            // row of this edge: forward from the warp's current row
            int d = cur_row, rs = 0, re = 0, j = 0;
            if (has) {
                re = __ldg(a.row_ptr + d + 1);
                for (int steps = 0; re <= e && d < a.N - 1; ++steps) {
                    if (steps == 16) {  // many rows in one chunk (short or empty rows): search instead
                        d = segment_of(a.row_ptr, a.N, e);
                        re = __ldg(a.row_ptr + d + 1);
                        break;
                    }
                    re = __ldg(a.row_ptr + (++d) + 1);
                }
                rs = __ldg(a.row_ptr + d);
                j = __ldg(a.src + e);
            }
            const bool valid = has && (unsigned)j < (unsigned)a.N;
            const int d_next = __shfl_down_sync(0xffffffffu, d, 1);
            const bool is_end = has && (lane == nrows - 1 || d_next != d);
            const unsigned end_mask = __ballot_sync(0xffffffffu, is_end);
            // the last row goes on in the warp's next chunk: carried, not stored
            const unsigned cont_mask = __ballot_sync(0xffffffffu, is_end && lane == nrows - 1 && re > ce && ce < rb);
            // the row lies wholly in this warp range: stored once, else reduced onto the output
            const unsigned whole_mask = __ballot_sync(0xffffffffu, has && rs >= ra && re <= rb);
            const bool one_segment = nrows > 0 && end_mask == (1u << (nrows - 1));
            if (nrows > 0) cur_row = __shfl_sync(0xffffffffu, d, nrows - 1);
            const float2* xrow = x2 + (size_t)(valid ? j : 0) * D * C2;

            // frame and Wigner matrices of the edge
            const float3 rv = has ? load_r(a.r, e) : make_float3(0.f, 0.f, 1.f);
            const Frame f = make_frame(rv.x, rv.y, rv.z);
            float d2[25], d3[49];
            thread_wigner<L>(f, d2, d3);

            // this warp's share of the hidden layer into the A operand (once the previous tile's MMAs are done)
            {
                float b[kBasis];
                const float dist = sqrtf(rv.x * rv.x + rv.y * rv.y + rv.z * rv.z);
                const float c = sqrtf(2.f / a.rc);
#pragma unroll
                for (int n = 0; n < kBasis; ++n) {
                    const float k = (float)(n + 1) * kPi / a.rc;
                    b[n] = dist >= 1e-12f ? c * sinf(k * dist) / dist : c * k;
                }
                if (i > 0) wait_live(a_empty, (i - 1) & 1, live);
#pragma unroll 2
                for (int k4 = kh0; k4 < kh1; k4 += 4) {
                    float h[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int n = 0; n < kBasis; ++n) {
                        const float4 wv = *reinterpret_cast<const float4*>(w1s + n * kHidden + k4);
                        h[0] = fmaf(b[n], wv.x, h[0]), h[1] = fmaf(b[n], wv.y, h[1]);
                        h[2] = fmaf(b[n], wv.z, h[2]), h[3] = fmaf(b[n], wv.w, h[3]);
                    }
#pragma unroll
                    for (int u = 0; u < 4; ++u) h[u] = has ? h[u] / (1.f + expf(-h[u])) : 0.f;
                    float4 hh, hl;
                    hh.x = tc::tf32_round(h[0]), hh.y = tc::tf32_round(h[1]);
                    hh.z = tc::tf32_round(h[2]), hh.w = tc::tf32_round(h[3]);
                    hl.x = tc::tf32_round(h[0] - hh.x), hl.y = tc::tf32_round(h[1] - hh.y);
                    hl.z = tc::tf32_round(h[2] - hh.z), hl.w = tc::tf32_round(h[3] - hh.w);
                    *reinterpret_cast<float4*>(arow_hi + (k4 >> 2) * kLBO) = hh;
                    *reinterpret_cast<float4*>(arow_lo + (k4 >> 2) * kLBO) = hl;
                }
                tc::fence_proxy_async();
                tc::mbar_arrive(a_full);
            }

            // x of the source for a channel pair (zero for an invalid source)
            auto load_x = [&](int gp, float2 (&xv)[D]) {
#pragma unroll
                for (int k = 0; k < D; ++k) xv[k] = valid ? __ldg(xrow + (size_t)k * C2 + gp) : f2_zero();
            };
            float2 xn[D];
            if constexpr (kPrefetchX) load_x(half, xn);
            const int npairs = S * pairs;

            for (int s = 0; s < S; ++s) {
                const int g = i * S + s, buf = g % kAccBufs;
                wait_live(&acc_full[buf], (g / kAccBufs) & 1, live);
                tc::fence_after_sync();
                for (int gp = s * pairs + ((half - s * pairs) % NH + NH) % NH; gp < (s + 1) * pairs; gp += NH) {
                    // channel pair gp: channels 2 gp, 2 gp + 1, TMEM pair block q of the slice
                    const int q = gp - s * pairs;
                    const uint32_t colq = lane_base + (uint32_t)(buf * a.Npad + q * 2 * P);
                    const bool col = lane < 2 * D;
                    // the row carried in from the previous chunk: loaded now, used after the pair's compute
                    const float cin = (carried && col) ? carry[(size_t)gp * 32] : 0.f;
                    float2 xv[D];
                    if constexpr (kPrefetchX) {
#pragma unroll
                        for (int k = 0; k < D; ++k) xv[k] = xn[k];
                        if (gp + NH < npairs) load_x(gp + NH, xn);  // this warp's next pair in the tile
                    } else {
                        load_x(gp, xv);
                    }
                    float2 xp[D];
                    static_for<0, L + 1>([&](auto lc) {
                        constexpr int l = decltype(lc)::value;
                        rot_reg<l, false>(f, d2, d3, xv + l * l, xp + l * l);
                    });
                    float* srow = stage + lane * STR;
                    // the pair's weights, one TMEM load per l3 group: all in flight together
                    // (L <= 2), or group by group (L = 3: registers)
                    constexpr int kAll = O::cols_pow2(0) + (L >= 1 ? O::cols_pow2(1) : 0) +
                                         (L >= 2 ? O::cols_pow2(2) : 0);
                    float vall[L <= 2 ? kAll : 1];
                    if constexpr (L <= 2) {
                        static_for<0, L + 1>([&](auto l3c) {
                            constexpr int l3 = decltype(l3c)::value;
                            constexpr int off = l3 == 0 ? 0 : (l3 == 1 ? O::cols_pow2(0) : O::cols_pow2(0) + O::cols_pow2(1));
                            tc::tmem_ld<O::cols_pow2(l3)>(colq + 2 * O::start(l3),
                                                          *reinterpret_cast<float(*)[O::cols_pow2(l3)]>(vall + off));
                        });
                        tc::tmem_wait_ld(vall);
                    }
                    static_for<0, L + 1>([&](auto l3c) {
                        constexpr int l3 = decltype(l3c)::value;
                        constexpr int NC = O::cols_pow2(l3);
                        float v[NC];
                        if constexpr (L <= 2) {
                            constexpr int off = l3 == 0 ? 0 : (l3 == 1 ? O::cols_pow2(0) : O::cols_pow2(0) + O::cols_pow2(1));
#pragma unroll
                            for (int u = 0; u < NC; ++u) v[u] = vall[off + u];
                        } else {
                            tc::tmem_ld<NC>(colq + 2 * O::start(l3), v);
                            tc::tmem_wait_ld(v);
                        }
                        float2 y[2 * l3 + 1], msg[2 * l3 + 1];
#pragma unroll
                        for (int m = 0; m < 2 * l3 + 1; ++m) y[m] = f2_zero();
                        if (!f.degenerate) {
                            static_for<0, L + 1>([&](auto l1c) {
                                constexpr int l1 = decltype(l1c)::value;
                                if constexpr (has_type<L, O3>(l1, l3, 0) || has_type<L, O3>(l1, l3, 1)) {
                                    float2 We[4], Wo[4];
                                    group_weights_reg<L, O3, l1, l3, NC>(v, We, Wo);
                                    apply_M<L, O3, l1, l3>(We, Wo, xp + l1 * l1, y);
                                }
                            });
                            rot_reg<l3, true>(f, d2, d3, y, msg);
                        } else {
                            // no direction: only the path (l3, 0, l3) acts, as the identity
                            constexpr int jj = O::pos(path_index<L, O3>(l3, 0, l3)) - O::start(l3);
                            const float2 w = make_float2(v[2 * jj], v[2 * jj + 1]);
#pragma unroll
                            for (int m = 0; m < 2 * l3 + 1; ++m) msg[m] = f2_mul(w, xv[l3 * l3 + m]);
                        }
#pragma unroll
                        for (int m = 0; m < 2 * l3 + 1; ++m) {
                            srow[2 * (l3 * l3 + m)] = msg[m].x;
                            srow[2 * (l3 * l3 + m) + 1] = msg[m].y;
                        }
                    });
                    __syncwarp();
                    // sum the rows of equal destination, in row order; lane k < 2D owns column k
                    // (component k / 2, channel 2 gp + k % 2); rows without an edge hold zeros
                    float vr[32];
#pragma unroll
                    for (int rr = 0; rr < 32; ++rr) vr[rr] = stage[rr * STR + (col ? lane : 0)];
                    __syncwarp();  // the stage is rewritten by the next pair
                    float* optr = a.out + (size_t)(lane >> 1) * a.C + 2 * gp + (lane & 1);
                    auto finish = [&](int rr, float acc) {  // the segment that ends at row rr
                        const int dd = __shfl_sync(0xffffffffu, d, rr);
                        if (col) {
                            if ((cont_mask >> rr) & 1u) {
                                carry[(size_t)gp * 32] = acc;
                            } else {
                                float* o = optr + (size_t)dd * D * a.C;
                                if ((whole_mask >> rr) & 1u)
                                    *o = acc;
                                else
                                    red_add(o, acc);
                            }
                        }
                    };
                    if (one_segment) {
#pragma unroll
                        for (int w = 16; w >= 1; w >>= 1)
#pragma unroll
                            for (int rr = 0; rr < w; ++rr) vr[rr] += vr[rr + w];
                        finish(nrows - 1, cin + vr[0]);
                    } else if (nrows > 0) {
                        float acc = cin;
#pragma unroll
                        for (int rr = 0; rr < 32; ++rr) {
                            acc += vr[rr];
                            if ((end_mask >> rr) & 1u) {
                                finish(rr, acc);
                                acc = 0.f;
                            }
                        }
                    }
                }
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&acc_empty[buf]);
            }
            carried = cont_mask != 0;
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == NW) {
        __syncwarp();
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, 512);
    }
}

// W2 [64][P*C] -> per slice s the B operand of the slice's MMA: row n of N = Npad
// (pair q = n / 2P, path j = (n % 2P) / 2 in l3-major order, channel 2q + n % 2 of
// the slice; zero past P * cs), K = the 64 hidden units, TF32 halves hi then lo.
struct PathOrder {
    int plan_path_of_pos[64];
};
__global__ void fused_prepare_w2(const float* __restrict__ W2, int C, int P, int cs, int S, int Npad, PathOrder order,
                                 float* __restrict__ out) {
    const long long per_half = (long long)Npad * kHidden;
    const long long total = (long long)S * per_half;
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
         idx += (long long)gridDim.x * blockDim.x) {
        const int s = (int)(idx / per_half), rem = (int)(idx % per_half);
        const int n = rem / kHidden, k = rem % kHidden;
        float v = 0.f;
        if (n < P * cs) {
            const int q = n / (2 * P), jpos = (n % (2 * P)) / 2, h = n & 1;
            const int c = s * cs + 2 * q + h;
            v = W2[(size_t)k * P * C + (size_t)order.plan_path_of_pos[jpos] * C + c];
        }
        const float hi = tc::tf32_round(v);
        float* base = out + (size_t)s * 2 * per_half;
        const uint32_t off = tc::kmajor_offset(n, k, kLBO, kSBO) / 4;
        base[off] = hi;
        base[per_half + off] = tc::tf32_round(v - hi);
    }
}

}  // namespace fused

// ---------------------------------------------------------------------------
// host side
namespace {

int slice_channels(int L, int C) {
    const int cap = L == 0 ? 32 : (L == 1 ? 16 : (L == 2 ? 8 : 4));
    return C < cap ? C : cap;
}

template <int L, bool O3>
struct FusedSpec {
    static constexpr int P = PathSet<L, O3>::P;
    static int Npad(int cs) { return (P * cs + 15) / 16 * 16; }
    static void plan_path_of_pos(int* out) {
        for (int p = 0; p < P; ++p) out[fused::L3Order<L, O3>::pos(p)] = p;
    }
    static constexpr int max_col_read(int cs, int npad) {
        return (fused::kAccBufs - 1) * npad + (cs / 2 - 1) * 2 * P + 2 * fused::L3Order<L, O3>::start(L) +
               fused::L3Order<L, O3>::cols_pow2(L);
    }
};

constexpr int kMaxFusedTasks = 512;

struct FusedGeometry {
    int cs, S, Npad, P, D;
    size_t w2_bytes, carry_bytes;
};

FusedGeometry fused_geometry(int L, bool o3, int C, int E) {
    FusedGeometry g{};
    g.cs = slice_channels(L, C);
    g.S = C / g.cs;
    g.D = (L + 1) * (L + 1);
    switch (L * 2 + (o3 ? 1 : 0)) {
        case 0: g.P = FusedSpec<0, false>::P; break;
        case 1: g.P = FusedSpec<0, true>::P; break;
        case 2: g.P = FusedSpec<1, false>::P; break;
        case 3: g.P = FusedSpec<1, true>::P; break;
        case 4: g.P = FusedSpec<2, false>::P; break;
        case 5: g.P = FusedSpec<2, true>::P; break;
        case 6: g.P = FusedSpec<3, false>::P; break;
        default: g.P = FusedSpec<3, true>::P; break;
    }
    g.Npad = (g.P * g.cs + 15) / 16 * 16;
    const fused::Smem lay = fused::smem_layout(g.Npad, g.D, 4);
    g.w2_bytes = (size_t)g.S * lay.slot_bytes;
    long long tasks = ((long long)E + fused::kRows - 1) / fused::kRows;
    if (tasks > kMaxFusedTasks) tasks = kMaxFusedTasks;
    if (tasks < 1) tasks = 1;
    g.carry_bytes = (size_t)tasks * 4 * (C / 2) * 32 * sizeof(float);
    return g;
}

template <int L, bool O3>
cudaError_t launch_fused(const FusedGeometry& g, int C, int N, int E, const int32_t* row_ptr, const int32_t* src,
                         const float* r, const float* x, const float* W1, const float* W2, float rc, float* out,
                         void* ws, cudaStream_t s) {
    using Spec = FusedSpec<L, O3>;
    if (Spec::max_col_read(g.cs, g.Npad) > 512 || g.Npad > 256) return cudaErrorInvalidConfiguration;
    char* p = static_cast<char*>(ws);
    float* w2s = reinterpret_cast<float*>(p);
    float* carry = reinterpret_cast<float*>(p + align16_bytes(g.w2_bytes));
    fused::PathOrder order{};
    Spec::plan_path_of_pos(order.plan_path_of_pos);
    const long long prep_total = (long long)g.S * g.Npad * fused::kHidden;
    const long long prep_blocks = (prep_total + 255) / 256;
    fused::fused_prepare_w2<<<(unsigned)(prep_blocks < 1184 ? prep_blocks : 1184), 256, 0, s>>>(
        W2, C, Spec::P, g.cs, g.S, g.Npad, order, w2s);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    if ((err = cudaMemsetAsync(out, 0, sizeof(float) * (size_t)N * g.D * C, s)) != cudaSuccess) return err;
    if (E == 0) return cudaSuccess;
    int dev = 0, sms = 1;
    if ((err = cudaGetDevice(&dev)) != cudaSuccess) return err;
    if ((err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return err;
    long long ntasks = ((long long)E + fused::kRows - 1) / fused::kRows;
    if (ntasks > sms) ntasks = sms;
    if (ntasks > kMaxFusedTasks) ntasks = kMaxFusedTasks;
    fused::FwdArgs a{N, E, row_ptr, src, r, x, W1, w2s, out, carry, rc, C, g.cs, g.S, g.Npad, (int)ntasks};
    constexpr int NW = fused::consumer_warps<L>();
    const fused::Smem lay = fused::smem_layout(g.Npad, g.D, NW);
    const void* k = (const void*)fused::etp_fused_fwd_kernel<L, O3>;
    if ((err = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)lay.total)) != cudaSuccess)
        return err;
    void* args[] = {&a};
    return cudaLaunchKernel(k, dim3((unsigned)ntasks), dim3(NW * 32 + 32), args, lay.total, s);
}

}  // namespace

bool fused_supported(int nb, int hidden) { return nb == fused::kBasis && hidden == fused::kHidden; }

size_t fused_workspace_bytes(int L, bool o3, int C, int E) {
    const FusedGeometry g = fused_geometry(L, o3, C, E);
    return align16_bytes(g.w2_bytes) + align16_bytes(g.carry_bytes);
}

size_t fused_smem_bytes(int L, bool o3, int C) {
    const FusedGeometry g = fused_geometry(L, o3, C, 1);
    return fused::smem_layout(g.Npad, g.D, L <= 2 ? fused::consumer_warps<2>() : fused::consumer_warps<3>()).total;
}

cudaError_t fused_forward(int L, bool o3, int C, int N, int E, const int32_t* row_ptr, const int32_t* src,
                          const float* r, const float* x, const float* W1, const float* W2, float rc, float* out,
                          void* ws, cudaStream_t s) {
    const FusedGeometry g = fused_geometry(L, o3, C, E);
    if (g.S * g.cs != C) return cudaErrorInvalidValue;
    switch (L * 2 + (o3 ? 1 : 0)) {
        case 0: return launch_fused<0, false>(g, C, N, E, row_ptr, src, r, x, W1, W2, rc, out, ws, s);
        case 1: return launch_fused<0, true>(g, C, N, E, row_ptr, src, r, x, W1, W2, rc, out, ws, s);
        case 2: return launch_fused<1, false>(g, C, N, E, row_ptr, src, r, x, W1, W2, rc, out, ws, s);
        case 3: return launch_fused<1, true>(g, C, N, E, row_ptr, src, r, x, W1, W2, rc, out, ws, s);
        case 4: return launch_fused<2, false>(g, C, N, E, row_ptr, src, r, x, W1, W2, rc, out, ws, s);
        case 5: return launch_fused<2, true>(g, C, N, E, row_ptr, src, r, x, W1, W2, rc, out, ws, s);
        case 6: return launch_fused<3, false>(g, C, N, E, row_ptr, src, r, x, W1, W2, rc, out, ws, s);
        default: return launch_fused<3, true>(g, C, N, E, row_ptr, src, r, x, W1, W2, rc, out, ws, s);
    }
}

int fused_read_and_clear_fault() {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, fused::g_fault, sizeof(int)) != cudaSuccess) return -1;
    if (v) {
        const int z = 0;
        if (cudaMemcpyToSymbol(fused::g_fault, &z, sizeof(int)) != cudaSuccess) return -1;
    }
    return v;
}

}  // namespace etp
