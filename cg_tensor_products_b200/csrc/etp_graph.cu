// Graph preprocessing on the device: the reverse CSR (edges grouped by source,
// stable in edge id), the destination of every edge, a CSR validator, and the
// locality schedule (a spatial order of the nodes and the forward and reverse
// CSRs taken in that order).
//
// Up to kOnePassMaxNodes sources the grouping is one stable counting pass: the
// count of every (source, tile of kTile edges) pair in a source-major table, one
// exclusive scan of that table (which also yields rev_ptr: the entry of tile 0 of
// each source), and a stable scatter of each tile. An out-of-range source counts
// as source N, so every position is written.
//
// Otherwise the reverse grouping is a least-significant-digit radix sort of the source ids
// with the edge ids as values, 8 bits per pass. Each pass is a stable counting
// sort over tiles of kTile edges: (1) a per-tile digit histogram, (2) an
// exclusive scan of the histogram table in (digit, tile) order (a parallel
// column scan, then the digit totals), (3) a stable scatter in which four warps split a tile into quarters, offset each other by
// their digit counts, and walk their quarter in order, ranking equal digits
// inside each 32-edge chunk with __match_any_sync. Stability of every pass makes the result
// unique: ties (equal sources) stay in increasing edge id, so the output is
// bit-exact and independent of scheduling. rev_ptr is the exclusive scan of the
// per-source edge counts.
#include <cuda_runtime.h>

#include <cstdint>

#include "etp_internal.h"

namespace etp {
namespace {

constexpr int kTile = kRadixTile;
constexpr int kScanThreads = 1024;

__global__ void count_sources(const int32_t* __restrict__ src, int E, int N, int32_t* __restrict__ cnt) {
    for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < E; e += gridDim.x * blockDim.x) {
        int j = src[e];
        if ((unsigned)j < (unsigned)N) atomicAdd(cnt + j, 1);
    }
}

// Exclusive scan of in[0..n) into out[0..n], out[n] = total; one block, in
// chunks of 4 * kScanThreads. in and out may alias.
__global__ void __launch_bounds__(kScanThreads) scan_exclusive(const int32_t* in, int32_t* out, int n) {
    __shared__ int32_t warp_sums[kScanThreads / 32];
    __shared__ int32_t carry_s;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    if (tid == 0) carry_s = 0;
    __syncthreads();
    for (int base = 0; base < n; base += 4 * kScanThreads) {
        int v[4];
        int local = 0;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            int idx = base + tid * 4 + k;
            v[k] = idx < n ? in[idx] : 0;
            local += v[k];
        }
        int incl = local;
#pragma unroll
        for (int s = 1; s < 32; s <<= 1) {
            int t = __shfl_up_sync(0xffffffffu, incl, s);
            if (lane >= s) incl += t;
        }
        if (lane == 31) warp_sums[wid] = incl;
        __syncthreads();
        if (wid == 0) {
            int ws = warp_sums[lane];
#pragma unroll
            for (int s = 1; s < 32; s <<= 1) {
                int t = __shfl_up_sync(0xffffffffu, ws, s);
                if (lane >= s) ws += t;
            }
            warp_sums[lane] = ws;  // inclusive over warps
        }
        __syncthreads();
        int carry = carry_s;
        int run = carry + (wid ? warp_sums[wid - 1] : 0) + incl - local;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            int idx = base + tid * 4 + k;
            if (idx < n) out[idx] = run;
            run += v[k];
        }
        __syncthreads();
        if (tid == kScanThreads - 1) carry_s = run;
        __syncthreads();
    }
    if (tid == 0) out[n] = carry_s;
}

// Exclusive scan, in place, of the per-tile digit counts in tile-major order
// hist[t * 256 + d], in the order (digit, tile), in two launches.
// (1) scan_digit_column: block d scans its digit's column over the tiles (in
// chunks of 1024 tiles, one per thread, carrying the running total) and leaves
// the column total in hist[256 * n_tiles + d].
__global__ void __launch_bounds__(1024) scan_digit_column(int32_t* hist, int n_tiles) {
    __shared__ int32_t warp_sums[32];
    __shared__ int32_t carry_s;
    const int d = blockIdx.x, tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    if (tid == 0) carry_s = 0;
    __syncthreads();
    for (int base = 0; base < n_tiles; base += 1024) {
        const int t = base + tid;
        const int v = t < n_tiles ? hist[(size_t)t * 256 + d] : 0;
        int incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += u;
        }
        if (lane == 31) warp_sums[wid] = incl;
        __syncthreads();
        if (wid == 0) {
            int ws = warp_sums[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int u = __shfl_up_sync(0xffffffffu, ws, o);
                if (lane >= o) ws += u;
            }
            warp_sums[lane] = ws;  // inclusive over warps
        }
        __syncthreads();
        const int carry = carry_s;
        if (t < n_tiles) hist[(size_t)t * 256 + d] = carry + (wid ? warp_sums[wid - 1] : 0) + incl - v;
        __syncthreads();
        if (tid == 0) carry_s = carry + warp_sums[31];
        __syncthreads();
    }
    if (tid == 0) hist[256 * (size_t)n_tiles + d] = carry_s;
}

// (2) scan_digit_totals: the 256 column totals become the digits' start offsets
// (exclusive scan in place); hist[256 * n_tiles + 256] = the total. tile_scatter
// adds a tile's column entry and its digit's start.
__global__ void __launch_bounds__(256) scan_digit_totals(int32_t* hist, int n_tiles) {
    __shared__ int32_t tot[256];
    const int d = threadIdx.x;
    int32_t* col = hist + 256 * (size_t)n_tiles;
    tot[d] = col[d];
    __syncthreads();
    for (int s = 1; s < 256; s <<= 1) {  // inclusive scan of the totals
        const int v = d >= s ? tot[d - s] : 0;
        __syncthreads();
        tot[d] += v;
        __syncthreads();
    }
    col[d] = d ? tot[d - 1] : 0;
    if (d == 255) col[256] = tot[255];
}

// hist[t * 256 + d] = number of edges of tile t whose key has digit d.
__global__ void __launch_bounds__(256) tile_histogram(const int32_t* __restrict__ keys, int E, int shift,
                                                      int32_t* __restrict__ hist) {
    __shared__ int32_t h[256];
    h[threadIdx.x] = 0;
    __syncthreads();
    const int t = blockIdx.x;
    const int lo = t * kTile, hi = min(E, lo + kTile);
    for (int e = lo + threadIdx.x; e < hi; e += 256) atomicAdd(h + ((keys[e] >> shift) & 255), 1);
    __syncthreads();
    hist[(size_t)t * 256 + threadIdx.x] = h[threadIdx.x];
}

// Stable scatter of one tile per block of 4 warps (one block per tile): warp w
// takes the w-th quarter of the tile; (1) each warp counts its digits, (2) the
// per-digit counts are prefix-summed over the warps on top of the tile's scanned
// offsets (column entry plus digit start), (3) each
// warp walks its quarter in order, ranking equal digits inside 32-edge chunks
// with __match_any_sync. vals_in == nullptr means the identity (value = edge id).
__global__ void __launch_bounds__(128) tile_scatter(const int32_t* __restrict__ keys_in,
                                                    const int32_t* __restrict__ vals_in, int E, int shift,
                                                    const int32_t* __restrict__ offsets,
                                                    int32_t* __restrict__ keys_out, int32_t* __restrict__ vals_out) {
    __shared__ int32_t cnt[4][256];
    const int wid = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x;
    constexpr int kQuarter = kTile / 4;
    const int lo = t * kTile + wid * kQuarter, hi = min(E, lo + kQuarter);
    for (int d = lane; d < 256; d += 32) cnt[wid][d] = 0;
    __syncwarp();
    for (int c = lo; c < hi; c += 32) {
        const int e = c + lane;
        if (e < hi) atomicAdd(&cnt[wid][(keys_in[e] >> shift) & 255], 1);
    }
    __syncthreads();
    for (int d = threadIdx.x; d < 256; d += 128) {  // warp-exclusive prefix per digit
        int run = offsets[(size_t)t * 256 + d] + offsets[256 * (size_t)gridDim.x + d];
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            const int v = cnt[w][d];
            cnt[w][d] = run;
            run += v;
        }
    }
    __syncthreads();
    int32_t* base = cnt[wid];
    const unsigned lt = (1u << lane) - 1u;
    for (int c = lo; c < hi; c += 32) {
        const int e = c + lane;
        const bool act = e < hi;
        const int key = act ? keys_in[e] : 0;
        const int val = act ? (vals_in ? vals_in[e] : e) : 0;
        const int d = act ? ((key >> shift) & 255) : 256 + lane;  // inactive lanes match nobody
        const unsigned peers = __match_any_sync(0xffffffffu, d);
        if (act) {
            const int pos = base[d] + __popc(peers & lt);
            keys_out[pos] = key;
            vals_out[pos] = val;
        }
        __syncwarp();
        if (act && lane == __ffs(peers) - 1) base[d] += __popc(peers);
        __syncwarp();
    }
}

// ---------------------------------------------------------------------------
// One-pass grouping. Bucket of an edge: its source, or N when out of range.
__device__ __forceinline__ int bucket_of(int j, int N) { return (unsigned)j < (unsigned)N ? j : N; }

// table[b * n_tiles + t] = edges of tile t in bucket b, for b = 0..N.
// (dynamic shared memory: N + 1 counters)
__global__ void __launch_bounds__(256) tile_counts(const int32_t* __restrict__ src, int E, int N, int n_tiles,
                                                   int32_t* __restrict__ table) {
    extern __shared__ int32_t h[];
    for (int b = threadIdx.x; b <= N; b += 256) h[b] = 0;
    __syncthreads();
    const int t = blockIdx.x;
    const int lo = t * kTile, hi = min(E, lo + kTile);
    for (int e = lo + threadIdx.x; e < hi; e += 256) atomicAdd(h + bucket_of(src[e], N), 1);
    __syncthreads();
    for (int b = threadIdx.x; b <= N; b += 256) table[(size_t)b * n_tiles + t] = h[b];
}

// Block-wide exclusive scan of one value per thread (1024 threads); returns the
// thread's exclusive prefix and writes the block total to *total.
__device__ __forceinline__ int block_exclusive_1024(int v, int32_t* warp_tot, int* total) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int s = 1; s < 32; s <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, incl, s);
        if (lane >= s) incl += u;
    }
    if (lane == 31) warp_tot[wid] = incl;
    __syncthreads();
    if (wid == 0) {
        int w = warp_tot[lane];
#pragma unroll
        for (int s = 1; s < 32; s <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, w, s);
            if (lane >= s) w += u;
        }
        warp_tot[lane] = w;  // inclusive over warps
    }
    __syncthreads();
    const int excl = (wid ? warp_tot[wid - 1] : 0) + incl - v;
    *total = warp_tot[31];
    return excl;
}

// In-place exclusive scan of each chunk of kScanChunk entries (8 per thread);
// part[chunk] = the chunk's total.
__global__ void __launch_bounds__(1024) scan_chunks(int32_t* __restrict__ a, long long n,
                                                    int32_t* __restrict__ part) {
    __shared__ int32_t warp_tot[32];
    const long long base = (long long)blockIdx.x * kScanChunk + 8ll * threadIdx.x;
    int v[8];
    int sum = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        v[k] = base + k < n ? a[base + k] : 0;
        sum += v[k];
    }
    int total;
    int run = block_exclusive_1024(sum, warp_tot, &total);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        if (base + k < n) a[base + k] = run;
        run += v[k];
    }
    if (threadIdx.x == 0) part[blockIdx.x] = total;
}

// Exclusive scan of the chunk totals (one block, in place; part[nb] = total), then
// rev_ptr[b] = scanned table entry of (b, tile 0) for b = 0..N.
__global__ void __launch_bounds__(1024) scan_parts_rev_ptr(int32_t* __restrict__ part, int nb,
                                                           const int32_t* __restrict__ table, int n_tiles, int N,
                                                           int32_t* __restrict__ rev_ptr) {
    __shared__ int32_t warp_tot[32];
    __shared__ int32_t carry;
    if (threadIdx.x == 0) carry = 0;
    __syncthreads();
    for (int b0 = 0; b0 < nb; b0 += 1024) {
        const int i = b0 + threadIdx.x;
        const int v = i < nb ? part[i] : 0;
        int total;
        const int ex = block_exclusive_1024(v, warp_tot, &total);
        const int c = carry;
        if (i < nb) part[i] = c + ex;
        __syncthreads();
        if (threadIdx.x == 0) carry = c + total;
        __syncthreads();
    }
    if (threadIdx.x == 0) part[nb] = carry;
    __syncthreads();
    for (int b = threadIdx.x; b <= N; b += 1024) {
        const long long idx = (long long)b * n_tiles;
        rev_ptr[b] = table[idx] + part[idx / kScanChunk];
    }
}

// Stable scatter of one tile per block of 4 warps (as tile_scatter, with the
// bucket of the full source id): rev_perm[pos] = edge id. Dynamic shared memory:
// 4 x (N + 1) counters.
__global__ void __launch_bounds__(128) tile_scatter_one_pass(const int32_t* __restrict__ src, int E, int N,
                                                             int n_tiles, const int32_t* __restrict__ table,
                                                             const int32_t* __restrict__ part,
                                                             int32_t* __restrict__ rev_perm) {
    extern __shared__ int32_t cnt[];  // [4][N + 1]
    const int stride = N + 1;
    const int wid = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x;
    constexpr int kQuarter = kTile / 4;
    const int lo = t * kTile + wid * kQuarter, hi = min(E, lo + kQuarter);
    int32_t* base = cnt + wid * stride;
    for (int b = lane; b <= N; b += 32) base[b] = 0;
    __syncwarp();
    for (int c = lo; c < hi; c += 32) {
        const int e = c + lane;
        if (e < hi) atomicAdd(&base[bucket_of(src[e], N)], 1);
    }
    __syncthreads();
    for (int b = threadIdx.x; b <= N; b += 128) {  // warp-exclusive prefix per bucket
        const long long idx = (long long)b * n_tiles + t;
        int run = table[idx] + part[idx / kScanChunk];
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            const int v = cnt[w * stride + b];
            cnt[w * stride + b] = run;
            run += v;
        }
    }
    __syncthreads();
    const unsigned lt = (1u << lane) - 1u;
    for (int c = lo; c < hi; c += 32) {
        const int e = c + lane;
        const bool act = e < hi;
        const int b = act ? bucket_of(src[e], N) : N + 1 + lane;  // inactive lanes match nobody
        const unsigned peers = __match_any_sync(0xffffffffu, b);
        if (act) rev_perm[base[b] + __popc(peers & lt)] = e;
        __syncwarp();
        if (act && lane == __ffs(peers) - 1) base[b] += __popc(peers);
        __syncwarp();
    }
}

__global__ void iota(int32_t* __restrict__ out, int n) {
    for (int k = blockIdx.x * blockDim.x + threadIdx.x; k < n; k += gridDim.x * blockDim.x) out[k] = k;
}

__global__ void edge_rows(const int32_t* __restrict__ row_ptr, int N, int E, int32_t* __restrict__ dst) {
    for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < E; e += gridDim.x * blockDim.x) {
        int lo = 0, hi = N;  // row_ptr[lo] <= e < row_ptr[hi] on a valid CSR
        while (hi - lo > 1) {
            int mid = (lo + hi) >> 1;
            if (row_ptr[mid] <= e)
                lo = mid;
            else
                hi = mid;
        }
        dst[e] = lo;
    }
}

__global__ void validate(const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ src, int N, int E,
                         int32_t* __restrict__ flag) {
    const int tid = blockIdx.x * blockDim.x + threadIdx.x, stride = gridDim.x * blockDim.x;
    int bits = 0;
    if (tid == 0 && (row_ptr[0] != 0 || row_ptr[N] != E)) bits |= 1;
    for (int i = tid; i < N; i += stride)
        if (row_ptr[i] > row_ptr[i + 1]) bits |= 2;
    for (int e = tid; e < E; e += stride) {
        int j = src[e];
        if (j < 0 || j >= N) bits |= 4;
    }
    if (bits) atomicOr(flag, bits);
}

// ---------------------------------------------------------------------------
// Spatial order. The bounding box is reduced on order-preserving unsigned codes of
// the coordinates (a float's bits with the sign flipped, or all bits flipped when
// negative: unsigned order = float order), with atomicMin / atomicMax.
__device__ __forceinline__ unsigned float_code(float f) {
    const unsigned u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float code_float(unsigned c) {
    return __uint_as_float((c & 0x80000000u) ? (c & 0x7fffffffu) : ~c);
}

__global__ void bbox_init(unsigned* box) {
    if (threadIdx.x < 3) box[threadIdx.x] = 0xffffffffu;  // min codes
    else if (threadIdx.x < 6) box[threadIdx.x] = 0u;      // max codes
}

// NaN coordinates are skipped (their nodes land in cell 0 on that axis).
__global__ void __launch_bounds__(256) bbox_reduce(const float* __restrict__ pos, int N, unsigned* __restrict__ box) {
    unsigned lo[3] = {0xffffffffu, 0xffffffffu, 0xffffffffu}, hi[3] = {0u, 0u, 0u};
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < N; i += gridDim.x * blockDim.x) {
#pragma unroll
        for (int a = 0; a < 3; ++a) {
            const float v = pos[3 * (size_t)i + a];
            if (v == v) {
                const unsigned c = float_code(v);
                lo[a] = min(lo[a], c);
                hi[a] = max(hi[a], c);
            }
        }
    }
#pragma unroll
    for (int a = 0; a < 3; ++a) {
#pragma unroll
        for (int o = 16; o; o >>= 1) {
            lo[a] = min(lo[a], __shfl_xor_sync(0xffffffffu, lo[a], o));
            hi[a] = max(hi[a], __shfl_xor_sync(0xffffffffu, hi[a], o));
        }
    }
    if ((threadIdx.x & 31) == 0) {
#pragma unroll
        for (int a = 0; a < 3; ++a) {
            atomicMin(box + a, lo[a]);
            atomicMax(box + 3 + a, hi[a]);
        }
    }
}

// 10 bits spread to every third bit (bit k -> bit 3k).
__device__ __forceinline__ unsigned spread3(unsigned v) {
    v &= 0x3ffu;
    v = (v | (v << 16)) & 0x030000ffu;
    v = (v | (v << 8)) & 0x0300f00fu;
    v = (v | (v << 4)) & 0x030c30c3u;
    v = (v | (v << 2)) & 0x09249249u;
    return v;
}

// Morton code of the node's cell: cells of side max(cell, largest extent / 1024)
// from the box's low corner, 10 bits per axis (x in the lowest bit of each triple).
__global__ void morton_keys(const float* __restrict__ pos, int N, const unsigned* __restrict__ box, float cell,
                            int32_t* __restrict__ keys) {
    const float lx = code_float(box[0]), ly = code_float(box[1]), lz = code_float(box[2]);
    const float ext = fmaxf(fmaxf(code_float(box[3]) - lx, code_float(box[4]) - ly), code_float(box[5]) - lz);
    const float side = fmaxf(cell, ext * (1.0f / 1023.0f));
    const float inv = side > 0.f ? 1.0f / side : 0.f;
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < N; i += gridDim.x * blockDim.x) {
        const float lo3[3] = {lx, ly, lz};
        unsigned c[3];
#pragma unroll
        for (int a = 0; a < 3; ++a) {
            const float t = (pos[3 * (size_t)i + a] - lo3[a]) * inv;  // NaN fails both tests below: cell 0
            c[a] = t >= 1023.f ? 1023u : (t > 0.f ? (unsigned)t : 0u);
        }
        keys[i] = (int32_t)(spread3(c[0]) | (spread3(c[1]) << 1) | (spread3(c[2]) << 2));
    }
}

// ---------------------------------------------------------------------------
// Locality schedule from an order of the nodes.
__global__ void invert_order(const int32_t* __restrict__ order, int N, int32_t* __restrict__ rank) {
    for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < N; j += gridDim.x * blockDim.x) rank[order[j]] = j;
}

// deg[j] = in-degree of the node of rank j
__global__ void ordered_degrees(const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ order, int N,
                                int32_t* __restrict__ deg) {
    for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < N; j += gridDim.x * blockDim.x) {
        const int i = order[j];
        deg[j] = row_ptr[i + 1] - row_ptr[i];
    }
}

// The position of edge e in the ordered forward CSR: its row's start there plus
// its offset inside the row (rows keep their edges in CSR order).
__global__ void ordered_positions(const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ dst,
                                  const int32_t* __restrict__ rank, const int32_t* __restrict__ ord_ptr, int E,
                                  int32_t* __restrict__ ord_edge) {
    for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < E; e += gridDim.x * blockDim.x) {
        const int i = dst[e];
        ord_edge[ord_ptr[rank[i]] + (e - row_ptr[i])] = e;
    }
}

// Source keys of the ordered reverse CSR: the source's rank; an out-of-range
// source keeps its value, so it is grouped after every valid one as before.
__global__ void source_ranks(const int32_t* __restrict__ src, const int32_t* __restrict__ rank, int N, int E,
                             int32_t* __restrict__ keys) {
    for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < E; e += gridDim.x * blockDim.x) {
        const int j = src[e];
        keys[e] = (unsigned)j < (unsigned)N ? rank[j] : j;
    }
}

inline size_t align16(size_t b) { return (b + 15) & ~size_t(15); }
inline int grid_for(long long n, int threads) {
    long long b = (n + threads - 1) / threads;
    if (b < 1) b = 1;
    if (b > 148 * 32) b = 148 * 32;
    return (int)b;
}
inline int radix_passes(int N) {
    int bits = 0;
    while (bits < 31 && (1ll << bits) < (long long)N) ++bits;  // keys are in [0, N)
    return (bits + 7) / 8;
}

// Stable LSD radix sort of the ids 0..n-1 by keys (8 bits per pass, `passes`
// passes from the lowest digit); the sorted ids end in out. keys_a, keys_b,
// vals_spare: n entries each; hist: 256 * (tiles + 1) + 1.
void radix_sort_ids(const int32_t* keys, int n, int passes, int32_t* keys_a, int32_t* keys_b, int32_t* vals_spare,
                    int32_t* hist, int32_t* out, cudaStream_t s) {
    const int n_tiles = (n + kTile - 1) / kTile;
    // values ping-pong between vals_spare and out, ending in out
    int32_t* vbuf[2] = {passes % 2 ? out : vals_spare, passes % 2 ? vals_spare : out};
    int32_t* kbuf[2] = {keys_a, keys_b};
    const int32_t* kin = keys;
    const int32_t* vin = nullptr;
    for (int pass = 0; pass < passes; ++pass) {
        const int shift = 8 * pass;
        tile_histogram<<<n_tiles, 256, 0, s>>>(kin, n, shift, hist);
        scan_digit_column<<<256, 1024, 0, s>>>(hist, n_tiles);
        scan_digit_totals<<<1, 256, 0, s>>>(hist, n_tiles);
        int32_t* kout = kbuf[pass & 1];
        int32_t* vout = vbuf[pass & 1];
        tile_scatter<<<n_tiles, 128, 0, s>>>(kin, vin, n, shift, hist, kout, vout);
        kin = kout;
        vin = vout;
    }
}

}  // namespace

size_t reverse_csr_workspace_bytes(int N, int E) { return reverse_csr_workspace_bytes_for(N, E); }

cudaError_t build_reverse_csr(int N, int E, const int32_t* row_ptr, const int32_t* src, int32_t* rev_ptr,
                              int32_t* rev_perm, int32_t* dst, void* ws, cudaStream_t s, bool one_pass) {
    if (one_pass && reverse_csr_one_pass(N, E)) {
        const int n_tiles = (int)radix_tiles(E);
        const long long n = (long long)(N + 1) * n_tiles;
        const int nb = (int)((n + kScanChunk - 1) / kScanChunk);
        int32_t* table = static_cast<int32_t*>(ws);
        int32_t* part = reinterpret_cast<int32_t*>(static_cast<char*>(ws) + align16(sizeof(int32_t) * (size_t)n));
        const size_t count_smem = sizeof(int32_t) * ((size_t)N + 1), scatter_smem = 4 * count_smem;
        if (scatter_smem > 48 * 1024) {  // above the default limit: opt in (a host-side attribute; cheap)
            cudaError_t e = cudaFuncSetAttribute(tile_scatter_one_pass, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 (int)scatter_smem);
            if (e != cudaSuccess) return e;
        }
        tile_counts<<<n_tiles, 256, count_smem, s>>>(src, E, N, n_tiles, table);
        scan_chunks<<<nb, 1024, 0, s>>>(table, n, part);
        scan_parts_rev_ptr<<<1, 1024, 0, s>>>(part, nb, table, n_tiles, N, rev_ptr);
        tile_scatter_one_pass<<<n_tiles, 128, scatter_smem, s>>>(src, E, N, n_tiles, table, part, rev_perm);
        if (dst) edge_rows<<<grid_for(E, 256), 256, 0, s>>>(row_ptr, N, E, dst);
        return cudaGetLastError();
    }
    char* p = static_cast<char*>(ws);
    int32_t* cnt = reinterpret_cast<int32_t*>(p);
    p += align16(sizeof(int32_t) * ((size_t)N + 1));
    int32_t* keys_a = reinterpret_cast<int32_t*>(p);
    p += align16(sizeof(int32_t) * (size_t)E);
    int32_t* keys_b = reinterpret_cast<int32_t*>(p);
    p += align16(sizeof(int32_t) * (size_t)E);
    int32_t* vals_spare = reinterpret_cast<int32_t*>(p);
    p += align16(sizeof(int32_t) * (size_t)E);
    int32_t* hist = reinterpret_cast<int32_t*>(p);

    cudaError_t err;
    // rev_ptr: exclusive scan of per-source counts
    if ((err = cudaMemsetAsync(cnt, 0, sizeof(int32_t) * ((size_t)N + 1), s)) != cudaSuccess) return err;
    if (E > 0) count_sources<<<grid_for(E, 256), 256, 0, s>>>(src, E, N, cnt);
    scan_exclusive<<<1, kScanThreads, 0, s>>>(cnt, rev_ptr, N);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    if (dst && E > 0) edge_rows<<<grid_for(E, 256), 256, 0, s>>>(row_ptr, N, E, dst);
    if (E == 0) return cudaGetLastError();

    const int passes = radix_passes(N);
    if (passes == 0) {  // a single node: every edge has source 0
        iota<<<grid_for(E, 256), 256, 0, s>>>(rev_perm, E);
        return cudaGetLastError();
    }
    radix_sort_ids(src, E, passes, keys_a, keys_b, vals_spare, hist, rev_perm, s);
    return cudaGetLastError();
}

size_t spatial_order_workspace_bytes(int N) {
    return align16(8 * sizeof(unsigned)) + 4 * align16(sizeof(int32_t) * (size_t)N) +
           align16(sizeof(int32_t) * (256 * ((size_t)radix_tiles(N) + 1) + 1));
}

cudaError_t spatial_order(int N, const float* pos, float cell, int32_t* order, void* ws, cudaStream_t s) {
    char* p = static_cast<char*>(ws);
    unsigned* box = reinterpret_cast<unsigned*>(p);
    p += align16(8 * sizeof(unsigned));
    int32_t* keys = reinterpret_cast<int32_t*>(p);
    p += align16(sizeof(int32_t) * (size_t)N);
    int32_t* keys_a = reinterpret_cast<int32_t*>(p);
    p += align16(sizeof(int32_t) * (size_t)N);
    int32_t* keys_b = reinterpret_cast<int32_t*>(p);
    p += align16(sizeof(int32_t) * (size_t)N);
    int32_t* spare = reinterpret_cast<int32_t*>(p);
    p += align16(sizeof(int32_t) * (size_t)N);
    int32_t* hist = reinterpret_cast<int32_t*>(p);
    bbox_init<<<1, 32, 0, s>>>(box);
    bbox_reduce<<<grid_for(N, 256), 256, 0, s>>>(pos, N, box);
    morton_keys<<<grid_for(N, 256), 256, 0, s>>>(pos, N, box, cell, keys);
    radix_sort_ids(keys, N, 4, keys_a, keys_b, spare, hist, order, s);  // 30-bit keys
    return cudaGetLastError();
}

size_t ordered_csr_workspace_bytes(int N, int E) {
    return align16(sizeof(int32_t) * (size_t)N) + align16(sizeof(int32_t) * (size_t)E) +
           reverse_csr_workspace_bytes_for(N, E);
}

cudaError_t build_ordered_csr(int N, int E, const int32_t* row_ptr, const int32_t* src, const int32_t* order,
                              int32_t* ord_ptr, int32_t* ord_edge, int32_t* rev_ptr, int32_t* rev_perm, int32_t* dst,
                              void* ws, cudaStream_t s) {
    char* p = static_cast<char*>(ws);
    int32_t* rank = reinterpret_cast<int32_t*>(p);
    p += align16(sizeof(int32_t) * (size_t)N);
    int32_t* keys = reinterpret_cast<int32_t*>(p);
    p += align16(sizeof(int32_t) * (size_t)E);
    invert_order<<<grid_for(N, 256), 256, 0, s>>>(order, N, rank);
    ordered_degrees<<<grid_for(N, 256), 256, 0, s>>>(row_ptr, order, N, ord_ptr);
    scan_exclusive<<<1, kScanThreads, 0, s>>>(ord_ptr, ord_ptr, N);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess || E == 0) {
        if (err == cudaSuccess) err = cudaMemsetAsync(rev_ptr, 0, sizeof(int32_t) * ((size_t)N + 1), s);
        return err;
    }
    edge_rows<<<grid_for(E, 256), 256, 0, s>>>(row_ptr, N, E, dst);
    ordered_positions<<<grid_for(E, 256), 256, 0, s>>>(row_ptr, dst, rank, ord_ptr, E, ord_edge);
    source_ranks<<<grid_for(E, 256), 256, 0, s>>>(src, rank, N, E, keys);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    return build_reverse_csr(N, E, row_ptr, keys, rev_ptr, rev_perm, nullptr, p, s);
}

cudaError_t validate_csr(int N, int E, const int32_t* row_ptr, const int32_t* src, int32_t* flag,
                         cudaStream_t s) {
    cudaError_t err = cudaMemsetAsync(flag, 0, sizeof(int32_t), s);
    if (err != cudaSuccess) return err;
    long long work = (long long)(N > E ? N : E);
    validate<<<grid_for(work, 256), 256, 0, s>>>(row_ptr, src, N, E, flag);
    return cudaGetLastError();
}

}  // namespace etp
