/* etp.h - C ABI of the B200 edge-wise equivariant tensor product library.
 *
 * One operation, its vector-Jacobian product, and the graph preprocessing they
 * need. For every directed edge e = (i <- j) of a CSR-by-destination graph:
 *
 *   Y(r_e)            real spherical harmonics of the edge vector, l2 = 0..L
 *   msg_e[l3 m3, c]   = sum_{p = (l1,l2,l3)} w[e,p,c] sum_{m1,m2} CG_p[m1,m2,m3] Y_{l2 m2}(r_e) x[j, l1 m1, c]
 *   out[i]            = sum over the edges e of row i of msg_e
 *
 * Passages this follows (the pages name the operation; they print no formula):
 *   - "High-performance training and inference for deep equivariant interatomic
 *     potentials", section "제안 방법": a fused tensor-product kernel whose Wigner
 *     3-j contraction coefficients are held in compressed sparse form without
 *     materialised intermediates;
 *   - "Scaling the leading accuracy of deep equivariant models to biomolecular
 *     simulations of realistic size", section "提出的方法": strided memory layout
 *     and a tensor product done as a single contraction;
 *   - "FlashCart 如何让等变原子间势更快更准?", sections "FlashCart 用笛卡尔内核替代
 *     球谐耦合" (speed comes from memory access and the aggregation of edge
 *     contributions) and "生成内核在高阶下胜过球谐基线" (edge convolution, forward
 *     and vector-Jacobian product);
 *   - "Machine Learning Interatomic Potentials: Advancing Open-Source Software
 *     for Efficient and Scalable Molecular Simulation", section "방법론 및
 *     아키텍처", item 2: dedicated kernels for Clebsch-Gordan tensor products.
 *
 * Conventions (the readings this library fixes where the pages are silent):
 *   - harmonics: component normalisation (sum_m Y_lm^2 = 2l+1), no Condon-Shortley
 *     phase, m = -l..l, Y_1 = sqrt(3) (y, z, x)/|r|; |r| < 1e-12 gives Y_0 = 1,
 *     Y_{l>0} = 0 and zero derivative;
 *   - CG_p: real coupling with sum_{m1,m2} CG^2 = 1 per m3, first nonzero entry in
 *     lexicographic (m1, m2, m3) order positive; no further path normalisation;
 *   - paths: every (l1, l2, l3) on the SO(3) triangle |l1-l2| <= l3 <= l1+l2,
 *     lexicographic; with parity letters in the irreps strings only the paths
 *     with l1+l2+l3 even (O(3), natural parities);
 *   - edge vector r_e points from the destination i to the source j;
 *   - paths into the same l3 are summed into one block; plain segment sum, no
 *     neighbour normalisation; rows without edges give zeros.
 *
 * Layout (all row-major, channel fastest, "D" = (L+1)^2 components, l blocks
 * ascending, m = -l..l inside a block):
 *   x, out, grad_out, grad_x : float32 [N][D][C]
 *   w, grad_w                : float32 [E][P][C]    (P paths in plan order)
 *   r, grad_r                : float32 [E][3]
 *   row_ptr int32 [N+1] (row_ptr[0] = 0, row_ptr[N] = E, nondecreasing),
 *   src int32 [E] (source node of each edge, in [0, N)).
 * Device pointers must be 16-byte aligned for x, w, out, grad_out, grad_x,
 * grad_w and frames (they are moved in 16-byte units).
 *
 * Ownership and execution: the caller owns every buffer. A plan owns only host
 * tables (the coupling values are compile-time constants of the kernels).
 * etp_edge_frames / etp_forward / etp_backward / etp_build_reverse_csr /
 * etp_validate_csr enqueue
 * work on the given stream and return without synchronising; they allocate no
 * memory; they overwrite their outputs.
 *
 * Errors: arguments that can be checked on the host (NULL pointers, negative
 * sizes, misalignment, unsupported irreps, L, C or dtype, a too-small workspace)
 * are rejected before any launch. The CSR's contents live on the device and are
 * not read by the host: etp_validate_csr checks them and reports through a
 * device flag. The kernels never trap and never wait on a flag; on an invalid
 * CSR they stay inside the given buffers (edges and rows out of range are
 * skipped) and their results are unspecified. A failed launch returns
 * ETP_ERR_CUDA (cudaGetLastError is consumed).
 */
#ifndef ETP_H_
#define ETP_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ETP_API __attribute__((visibility("default")))
#else
#define ETP_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct etp_plan_s* etp_plan_t;
typedef struct CUstream_st* etp_stream_t; /* a cudaStream_t; NULL is the legacy default stream */

typedef enum { ETP_F32 = 0 } etp_dtype;

typedef enum {
    ETP_OK = 0,
    ETP_ERR_INVALID_ARG = 1, /* NULL, negative size, misaligned pointer, bad string   */
    ETP_ERR_UNSUPPORTED = 2, /* irreps / L / C / dtype without a compiled kernel        */
    ETP_ERR_BAD_CSR = 3,     /* reserved for callers that map the validation flag      */
    ETP_ERR_CUDA = 4,        /* a CUDA launch or query failed                           */
    ETP_ERR_ALLOC = 5,       /* host allocation of a plan failed                        */
    ETP_ERR_WORKSPACE = 6,   /* workspace smaller than etp_reverse_csr_workspace_size   */
    ETP_ERR_TOO_LARGE = 7    /* N or E above the fixed scratch of the _static variant   */
} etp_status;

/* Bits of the flag written by etp_validate_csr. */
#define ETP_CSR_BAD_ENDPOINTS 1 /* row_ptr[0] != 0 or row_ptr[N] != E */
#define ETP_CSR_NOT_MONOTONE 2  /* row_ptr[i] > row_ptr[i+1] for some i */
#define ETP_CSR_SRC_RANGE 4     /* some src[e] outside [0, N) */

/* Create a plan for the tensor product of node irreps `irreps_in` with the edge
 * harmonics l2 = 0..sh_lmax into `irreps_out`, C channels each, in `dtype`.
 * Irreps strings: "0..L", "0+1+...+L", or with parity letters "0e+1o+2e+..."
 * (natural parities only). Compiled kernels: irreps_in = irreps_out = l 0..L,
 * sh_lmax = L, L in 0..3; C in {4, 8, 16, 32, 64, 128} (C/4 lanes own a node,
 * at most one warp); ETP_F32. Anything else: ETP_ERR_UNSUPPORTED (a malformed
 * string: ETP_ERR_INVALID_ARG). On success *plan is set; free it with
 * etp_plan_destroy. Host only: needs no GPU. */
ETP_API etp_status etp_plan_create(etp_plan_t* plan, const char* irreps_in, int sh_lmax,
                           const char* irreps_out, int C, etp_dtype dtype);

/* Plan shape. Any output pointer may be NULL. paths_l1l2l3, when given, receives
 * 3*n_paths ints (l1, l2, l3 of each path in kernel order). Host only. */
ETP_API etp_status etp_plan_info(etp_plan_t plan, int* n_paths, int* dim_in, int* dim_sh, int* dim_out,
                         int* paths_l1l2l3);

/* The coupling coefficients compiled into the kernels, in sparse form: for path p
 * the entries k in [path_off[p], path_off[p+1]) couple m1[k], m2[k], m3[k]
 * (indices 0..2l inside the l1, l2, l3 blocks) with value val[k]. Call with all
 * arrays NULL to get *nnz; then pass path_off (n_paths+1 ints) and nnz-sized
 * arrays. Host only. */
ETP_API etp_status etp_plan_couplings(etp_plan_t plan, int* nnz, int* path_off, int* m1, int* m2, int* m3,
                              double* val);

/* Free a plan (NULL is accepted). */
ETP_API etp_status etp_plan_destroy(etp_plan_t plan);

/* Floats in the frame record of one edge (see etp_edge_frames). */
#define ETP_FRAME_FLOATS 88

/* Edge frames: for every edge, the rotation R that takes the edge direction to
 * the z axis, 1/|r|, a zero-length flag, and the Wigner matrices D_2(R), D_3(R)
 * of the real harmonics, written as a record of ETP_FRAME_FLOATS floats.
 * The tensor product is evaluated in this frame: there the harmonics of the edge
 * are those of z, nonzero for m2 = 0 only, so each path couples the rotated x
 * through few coefficients (this library's reading of the pages' sparse
 * Clebsch-Gordan contraction: the rotation is a change of basis, the result the
 * same). The records depend on r only; computed once, they serve both
 * etp_forward and etp_backward for the same r, which then skip building the
 * frames themselves. The record layout is private to the library.
 * frames: device float32 [E][ETP_FRAME_FLOATS], 16-byte aligned, owned by the
 * caller; r: [E][3]. E = 0 launches nothing. */
ETP_API etp_status etp_edge_frames(etp_plan_t plan, int E, const float* r, float* frames, etp_stream_t stream);

/* Whether precomputed frame records pay for this plan and edge count: 1 when the
 * records (E x ETP_FRAME_FLOATS x 4 bytes) stay small enough to be read back from
 * L2 by both kernels (at most 64 MB; the 1024-node micro-benchmark graph: 46 MB),
 * else 0 (then the kernels build the frames themselves, cheaper than streaming the
 * records from HBM: 440 MB at 1.25 M edges). Host only. */
ETP_API etp_status etp_plan_frames_advised(etp_plan_t plan, int E, int* use_records);

/* Bytes of device workspace the tensor-product calls need for this plan and graph
 * size: etp_forward, etp_backward, etp_double_backward, etp_cart_forward and
 * etp_cart_backward (ordered = 0), and with ordered = 1 also etp_forward_ordered
 * and etp_backward_ordered; with or without frame records. Host only; it reads
 * the current device's multiprocessor count and the kernels' occupancy. 0 when
 * E = 0. */
ETP_API etp_status etp_tp_workspace_size(etp_plan_t plan, int N, int E, int ordered, size_t* bytes);

/* Forward: out[i] = sum_{e in row i} msg_e (see above), for all N rows.
 * x: [N][D][C], w: [E][P][C], r: [E][3], out: [N][D][C] device pointers.
 * frames: NULL (the kernel builds each edge's frame from r), or the records
 * etp_edge_frames wrote for this r and plan's L (then r is not read and may be
 * NULL). N >= 0, E >= 0; with N = 0 nothing is launched; with E = 0 out is
 * zeroed.
 * Segment sums without atomics: the edges are split into equal contiguous tasks;
 * each row is summed in registers in edge order and stored once. A row cut by task
 * boundaries leaves one partial row per task in `workspace` (at least
 * etp_tp_workspace_size bytes, 16-byte aligned, owned by the caller; may be NULL
 * when E = 0), and a second launch on the same stream adds them up in task order
 * and zeroes the rows without edges. Every output is written once, in a fixed
 * order: results repeat bit for bit. */
ETP_API etp_status etp_forward(etp_plan_t plan, int N, int E, const int32_t* row_ptr, const int32_t* src,
                       const float* r, const float* frames, const float* x, const float* w, float* out,
                       void* workspace, size_t workspace_bytes, etp_stream_t stream);

/* Vector-Jacobian product for the cotangent grad_out = dLoss/d(out), [N][D][C]:
 *   grad_x[j, l1 m1, c] = sum_{e: src e = j} sum_p w[e,p,c] sum_{m2,m3} CG_p Y_{l2 m2}(r_e) grad_out[dst e, l3 m3, c]
 *   grad_w[e, p, c]     = sum_{m1,m2,m3} CG_p Y_{l2 m2}(r_e) x[src e, l1 m1, c] grad_out[dst e, l3 m3, c]
 *   grad_r[e]           = sum_{l2 m2} dLoss/dY_{l2 m2}(e) dY_{l2 m2}/dr_e   (through Y only; r_e . grad_r[e] = 0)
 * rev_ptr [N+1] / rev_perm [E] group the edges by source, as written by
 * etp_build_reverse_csr; dst_of_edge [E] (may be NULL: then the row of each edge
 * is found by binary search in row_ptr). frames: as in etp_forward (with
 * frames, r is not read and may be NULL). Each of grad_x, grad_w, grad_r may be
 * NULL to skip it. All outputs are overwritten (sources without edges get zero
 * grad_x). An edge whose source or row is out of range (a CSR that
 * etp_validate_csr flags) adds nothing to grad_x and gets zero grad_w and grad_r.
 * workspace: as in etp_forward, for the source rows of grad_x (may be NULL when
 * grad_x is NULL or E = 0); grad_x is summed without atomics and repeats bit for
 * bit, like out. */
ETP_API etp_status etp_backward(etp_plan_t plan, int N, int E, const int32_t* row_ptr, const int32_t* src,
                        const int32_t* rev_ptr, const int32_t* rev_perm, const int32_t* dst_of_edge,
                        const float* r, const float* frames, const float* x, const float* w,
                        const float* grad_out, float* grad_x, float* grad_w, float* grad_r,
                        void* workspace, size_t workspace_bytes, etp_stream_t stream);

/* VJP of the VJP (double backward). With (grad_x, grad_w, grad_r) = etp_backward's
 * outputs for (x, w, r; grad_out) and cotangents gg_x [N][D][C], gg_w [E][P][C],
 * gg_r [E][3] of those outputs, computes the gradients of
 *     <gg_x, grad_x> + <gg_w, grad_w> + <gg_r, grad_r>
 * with respect to grad_out (grad_grad_out [N][D][C]), x (grad_x [N][D][C]), w
 * (grad_w [E][P][C]) and r (grad_r [E][3]). Force-loss training differentiates the
 * forces, built from grad_r, with respect to the parameters, which takes this
 * product ("FlashCart 如何让等变原子间势更快更准?", section "生成内核在高阶下胜过球谐
 * 基线": the VJP of the VJP is timed beside the forward and the VJP). It includes
 * the term through the Hessian of the harmonics (through gg_r). Each of gg_x,
 * gg_w, gg_r may be NULL (zero); each output may be NULL (skipped); outputs are
 * overwritten (nodes without edges get zeros). Graph arguments as in etp_backward
 * (rev_ptr, rev_perm from etp_build_reverse_csr; dst_of_edge may be NULL). r is
 * always read. Edges shorter than 1e-12 have no direction: only the (l, 0, l)
 * paths act and every derivative in r is zero there. Allocates nothing. Node sums
 * as in etp_forward: rows cut by a task boundary leave partial rows in `workspace`
 * (etp_tp_workspace_size bytes; may be NULL when neither grad_grad_out nor grad_x
 * is wanted, or E = 0), summed in task order by a second launch; for C = 128,
 * grad_r is the sum of two channel halves added onto zero (exact in either order).
 * Results repeat bit for bit. */
ETP_API etp_status etp_double_backward(etp_plan_t plan, int N, int E, const int32_t* row_ptr, const int32_t* src,
                                       const int32_t* rev_ptr, const int32_t* rev_perm, const int32_t* dst_of_edge,
                                       const float* r, const float* x, const float* w, const float* grad_out,
                                       const float* gg_x, const float* gg_w, const float* gg_r,
                                       float* grad_grad_out, float* grad_x, float* grad_w, float* grad_r,
                                       void* workspace, size_t workspace_bytes, etp_stream_t stream);

/* Cartesian edge convolution: the same edge tensor product with Cartesian
 * couplings ("FlashCart 如何让等变原子间势更快更准?", sections "FlashCart 用笛卡尔内核替
 * 代球谐耦合" and "生成内核在高阶下胜过球谐基线": Cartesian kernels in place of
 * spherical-harmonic couplings, compared at equal rank). A rank-l feature is a
 * symmetric traceless (STF) tensor held by its 2l + 1 entries with at most one z
 * index, in the order x^l, x^(l-1) y, .., y^l, x^(l-1) z, .., y^(l-1) z (rank 1:
 * x, y, z); x, out, grad_out, grad_x are [N][(L+1)^2][C] with these blocks for
 * l = 0..L. The edge attribute of rank l is the STF part of u (x) .. (x) u,
 * u = r_e / |r_e| (zero for l >= 1 when |r_e| < 1e-12). Path (l1, l2 -> l3), in the
 * plan's path order: k = (l1 + l2 - l3 - odd) / 2 index pairs contracted, the
 * first operand's last k indices with the second's first k; for l1 + l2 + l3 odd
 * (odd = 1) the first operand's last free index and the second's first free index
 * go through the Levi-Civita symbol into a new last index; the STF part of the
 * result; no normalisation constant. Then
 *   out[i] = sum over row i of sum_p w[e,p,:] coupling_p(x[src e], attribute_l2(r_e)).
 * The couplings are compile-time sparse tables of explicit sums; the pages give no
 * formula, so these are this library's reading. Arguments, layouts, ownership and
 * errors as etp_forward / etp_backward (no frame records; the same workspace); the
 * VJP writes grad_x (sources without edges: zero), grad_w and grad_r (derivative
 * through the edge attribute), each optional. */
ETP_API etp_status etp_cart_forward(etp_plan_t plan, int N, int E, const int32_t* row_ptr, const int32_t* src,
                                    const float* r, const float* x, const float* w, float* out, void* workspace,
                                    size_t workspace_bytes, etp_stream_t stream);
ETP_API etp_status etp_cart_backward(etp_plan_t plan, int N, int E, const int32_t* row_ptr, const int32_t* src,
                                     const int32_t* rev_ptr, const int32_t* rev_perm, const int32_t* dst_of_edge,
                                     const float* r, const float* x, const float* w, const float* grad_out,
                                     float* grad_x, float* grad_w, float* grad_r, void* workspace,
                                     size_t workspace_bytes, etp_stream_t stream);

/* Node-local product: features of higher correlation order from one node's own
 * features ("FlashCart 如何让等变原子间势更快更准?", section "FlashCart 用笛卡尔内核替代
 * 球谐耦合": equivariant features built recursively, brought back to a fixed width at
 * every step; section "生成内核在高阶下胜过球谐基线": the node-local product at 4096
 * nodes x 128 channels, rank 3, order 4, weighted products applied step by step and
 * only ranks up to the maximum kept). The pages give no formula; this library's
 * reading, with the plan's paths p = (l1, l2, l3) (l1 a rank of B, l2 a rank of x):
 *   B(1) = x,  B(k+1)_l3[c] = sum_p w[k-1, p, c] couple_p(B(k)_l1[c], x_l2[c]),  k = 1 .. K-1,
 *   out = B(K)   (K: the correlation order, the number of factors of x).
 * Channels do not mix; w is shared by all nodes. cartesian = 0: spherical
 * components and the plan's real Clebsch-Gordan couplings (x, out laid out as for
 * etp_forward); cartesian = 1: STF tensors in the independent components and
 * couplings of etp_cart_forward (a general STF second operand, not only the edge
 * attribute).
 * x: float32 [N][D][C] device; w: float32 [K-1][P][C] device (may be NULL when
 * K = 1); out: float32 [N][D][C] device, written in full, must not overlap x or w.
 * All three 16-byte aligned and owned by the caller; nothing is allocated. The call
 * is asynchronous on `stream`; results repeat bit for bit (no atomics).
 * Errors: ETP_ERR_INVALID_ARG for a NULL plan, N < 0, K < 1, cartesian not 0 or 1, or
 * a NULL or misaligned pointer that is needed; N = 0 returns ETP_OK at once. */
ETP_API etp_status etp_node_product(etp_plan_t plan, int N, int K, int cartesian, const float* x, const float* w,
                                    float* out, etp_stream_t stream);
/* The kernel's FP32 operations per node, channel and step (one multiply per operand
 * product it forms, one FMA per coupling coefficient, one FMA per weighted output
 * component): the cost model of etp_node_product, whose work is this times
 * N * C * (K - 1). */
ETP_API etp_status etp_node_product_ops(etp_plan_t plan, int cartesian, int* ops_per_step);

/* Radial weights: the tensor product's per-edge weights as a function of the edge
 * length. The pages make these weights a learned function of |r| ("High-performance
 * training and inference for deep equivariant interatomic potentials", section
 * "제안 방법": the Allegro tensor product with per-edge weights; the water systems of
 * section "주요 결과"); this library's plain reading, with d = |r_e|:
 *   b_n(d) = sqrt(2/r_cut) sin(n pi d / r_cut) / d,  n = 1..n_basis  (b_n(0) = its limit)
 *   w[e] = SiLU(b(d_e) W1) W2,   SiLU(z) = z / (1 + exp(-z)),   no biases, no envelope,
 * W1: float32 [n_basis][hidden], W2: float32 [hidden][P*C] (row-major), w: float32
 * [E][P][C] as etp_forward takes it. 1 <= n_basis <= 32; hidden a multiple of 32 in
 * [32, 256]; r_cut > 0. With n_basis = 8, hidden = 64 and P*C a multiple of 16 the
 * dense products run on the tensor cores, each FP32 product as three TF32 products
 * (hi*hi + hi*lo + lo*hi of the operands' TF32 halves: relative error near 2^-21);
 * otherwise as FP32 FMAs. Every sum over edges is taken in a fixed order (results
 * repeat bit for bit).
 * workspace: device memory of etp_radial_workspace_size bytes, 16-byte aligned,
 * owned by the caller. */
ETP_API etp_status etp_radial_workspace_size(etp_plan_t plan, int E, int n_basis, int hidden, size_t* bytes);
ETP_API etp_status etp_radial_forward(etp_plan_t plan, int E, int n_basis, int hidden, float r_cut,
                                      const float* r, const float* W1, const float* W2, float* w,
                                      void* workspace, size_t workspace_bytes, etp_stream_t stream);
/* VJP of etp_radial_forward for grad_w = dL/dw [E][P][C] (16-byte aligned): overwrites grad_W1 [n_basis][hidden]
 * and grad_W2 [hidden][P*C], and ADDS the derivative through the edge lengths,
 * (dL/dd) r / |r|, to grad_r [E][3] (so that grad_r can first hold etp_backward's
 * derivative through the harmonics; the sum is then the full dL/dr for
 * etp_assemble_forces). */
ETP_API etp_status etp_radial_backward(etp_plan_t plan, int E, int n_basis, int hidden, float r_cut,
                                       const float* r, const float* W1, const float* W2, const float* grad_w,
                                       float* grad_W1, float* grad_W2, float* grad_r, void* workspace,
                                       size_t workspace_bytes, etp_stream_t stream);

/* Radial weights fused into the tensor product, forward: the same result as
 * etp_radial_forward followed by etp_forward,
 *   out[i] = sum_{e in row i} sum_p w[e,p,:] (coupling of x[src e] with Y(r_e))_p,
 *   w[e] = SiLU(b(|r_e|) W1) W2   (as etp_radial_forward),
 * without the per-edge weights ever being stored: they are produced on the tensor
 * cores 128 edges at a time (each FP32 product as three TF32 products) and read by
 * the tensor product straight from tensor memory. ("High-performance training and
 * inference for deep equivariant interatomic potentials", section "제안 방법": a
 * fused tensor-product kernel without materialised intermediates, whose per-edge
 * weights are a learned function of the edge length.)
 * n_basis = 8 and hidden = 64 only (ETP_ERR_UNSUPPORTED otherwise); W1 [8][64],
 * W2 [64][P*C] row-major as in etp_radial_forward; r [E][3], x [N][D][C], out
 * [N][D][C]. workspace: device memory of etp_fused_workspace_size bytes, 16-byte
 * aligned, owned by the caller (the rearranged W2 and per-warp carry rows),
 * reusable once the stream has passed the call. Node sums are taken in a fixed
 * order; a row shared by two CTAs is completed by a reduction of its two parts
 * onto the zeroed output (bitwise repeatable while no row is longer than a CTA's
 * range of edges, about E / number of SMs). */
ETP_API etp_status etp_fused_workspace_size(etp_plan_t plan, int E, int n_basis, int hidden, size_t* bytes);
ETP_API etp_status etp_fused_forward(etp_plan_t plan, int N, int E, const int32_t* row_ptr, const int32_t* src,
                                     const float* r, const float* x, int n_basis, int hidden, float r_cut,
                                     const float* W1, const float* W2, float* out, void* workspace,
                                     size_t workspace_bytes, etp_stream_t stream);

/* Atom forces and per-atom virials from per-edge energy derivatives.
 * The pages evaluate models on energies and forces ("FlashCart 如何让等变原子间势更快更准?",
 * section "560 万参数模型胜过 1.89 亿参数 transformer"); forces are minus the position
 * gradient of the energy. With r_e = pos[src e] - pos[dst e] (plus a fixed periodic
 * shift) and grad_r[e] = dE/dr_e (etp_backward's grad_r, plus whatever other terms
 * of dE/dr_e the caller adds):
 *   forces[k]          = sum_{e: dst e = k} grad_r[e] - sum_{e: src e = k} grad_r[e]
 *   virial[k][a][b]    = sum_{e: dst e = k} grad_r[e][a] * r[e][b]
 * (summed over k, the virial is dE/d(eps_ab) under the strain r -> (I + eps) r of
 * every edge vector; each edge's term is assigned to its destination atom).
 * row_ptr [N+1] and src define the CSR by destination; rev_ptr [N+1], rev_perm [E]
 * are etp_build_reverse_csr's output for it. forces: float32 [N][3]; virial:
 * float32 [N][3][3] or NULL (then r may be NULL). Every sum is taken in a fixed
 * order: results repeat bit for bit. Overwrites its outputs; allocates nothing. */
ETP_API etp_status etp_assemble_forces(int N, int E, const int32_t* row_ptr, const int32_t* rev_ptr,
                                       const int32_t* rev_perm, const float* r, const float* grad_r,
                                       float* forces, float* virial, etp_stream_t stream);

/* Bytes of device workspace etp_build_reverse_csr needs for (N, E). */
ETP_API etp_status etp_reverse_csr_workspace_size(int N, int E, size_t* bytes);

/* Group edges by source, stably in edge id (a counting sort; deterministic):
 *   rev_ptr[j]..rev_ptr[j+1] indexes rev_perm, the edges with src = j in increasing id;
 *   dst_of_edge[e] = the CSR row that holds e (may be NULL to skip).
 * workspace: device memory of at least etp_reverse_csr_workspace_size bytes,
 * 16-byte aligned, owned by the caller, free to reuse once the stream has passed
 * this call. Needs a valid CSR (see etp_validate_csr). */
ETP_API etp_status etp_build_reverse_csr(int N, int E, const int32_t* row_ptr, const int32_t* src,
                                 int32_t* rev_ptr, int32_t* rev_perm, int32_t* dst_of_edge,
                                 void* workspace, size_t workspace_bytes, etp_stream_t stream);

/* Locality schedule. With node features larger than L2 and node ids in no spatial
 * order, the per-edge gathers of x[src] (forward) and grad_out[dst] (backward)
 * miss L2 often. A locality schedule takes the rows in a spatial order of the
 * nodes and splits the work into several waves of tasks, so that the tasks in
 * flight at any time hold nearby rows and share their neighbours' rows in L2.
 * Results are the same as etp_forward's and etp_backward's up to the rounding of
 * rows cut by a task boundary (the two split the edges differently); each repeats
 * bit for bit. The pages measure on spatially coherent systems
 * ("FlashCart 如何让等变原子间势更快更准?", section "FlashCart 用笛卡尔内核替代球谐耦合":
 * the speed comes from memory access and the aggregation of edge contributions);
 * the schedule is this library's way to keep those accesses local when the ids
 * are not. */

/* Bytes of device workspace etp_build_locality_schedule needs for (N, E). */
ETP_API etp_status etp_locality_schedule_workspace_size(int N, int E, size_t* bytes);

/* Build the locality schedule of a CSR graph from node positions:
 *   order [N]: the node ids sorted stably by the Morton (Z-order) code of their
 *     cell: cubic cells of side max(cell, largest bounding-box extent / 1023),
 *     10 bits per axis (ties keep increasing id; NaN coordinates fall in cell 0);
 *   ord_ptr [N+1], ord_edge [E]: the forward CSR with its rows taken in that
 *     order: positions ord_ptr[k]..ord_ptr[k+1] hold the edges of row order[k],
 *     in CSR order;
 *   rev_ptr [N+1], rev_perm [E]: the reverse CSR with its sources taken in that
 *     order (positions rev_ptr[k]..rev_ptr[k+1]: the edges whose source is
 *     order[k], in increasing edge id; edges with an out-of-range source last);
 *   dst_of_edge [E]: the CSR row of every edge.
 * pos: device float32 [N][3]; cell > 0 and finite (the radial cutoff is a good
 * choice). workspace: at least etp_locality_schedule_workspace_size bytes, 16-byte
 * aligned, owned by the caller. Deterministic (counting and radix sorts). Needs a
 * valid CSR (see etp_validate_csr). N = 0 launches nothing. */
ETP_API etp_status etp_build_locality_schedule(int N, int E, const int32_t* row_ptr, const int32_t* src,
                                               const float* pos, float cell, int32_t* order, int32_t* ord_ptr,
                                               int32_t* ord_edge, int32_t* rev_ptr, int32_t* rev_perm,
                                               int32_t* dst_of_edge, void* workspace, size_t workspace_bytes,
                                               etp_stream_t stream);

/* etp_forward on a locality schedule: the same result, out[i] = sum over the
 * edges of row i, with the rows visited in the schedule's order. order, ord_ptr,
 * ord_edge: as written by etp_build_locality_schedule for this graph (an entry of
 * ord_edge out of [0, E) counts as an edge with an invalid source). src, r,
 * frames, x, w, out: as in etp_forward (indexed by edge and node id, unchanged). */
ETP_API etp_status etp_forward_ordered(etp_plan_t plan, int N, int E, const int32_t* order, const int32_t* ord_ptr,
                                       const int32_t* ord_edge, const int32_t* src, const float* r,
                                       const float* frames, const float* x, const float* w, float* out,
                                       void* workspace, size_t workspace_bytes, etp_stream_t stream);

/* etp_backward on a locality schedule: the same outputs, with the sources visited
 * in the schedule's order. order, rev_ptr, rev_perm, dst_of_edge: as written by
 * etp_build_locality_schedule (dst_of_edge is required). The other arguments as
 * in etp_backward. */
ETP_API etp_status etp_backward_ordered(etp_plan_t plan, int N, int E, const int32_t* order,
                                        const int32_t* rev_ptr, const int32_t* rev_perm,
                                        const int32_t* dst_of_edge, const float* r, const float* frames,
                                        const float* x, const float* w, const float* grad_out, float* grad_x,
                                        float* grad_w, float* grad_r, void* workspace, size_t workspace_bytes,
                                        etp_stream_t stream);

/* Limits of etp_build_reverse_csr_static and the size of its scratch array. */
#define ETP_STATIC_MAX_NODES (1 << 18)
#define ETP_STATIC_MAX_EDGES (1 << 18)
#define ETP_STATIC_SCRATCH_BYTES 4457504 /* device bytes held on every GPU that loads the library */

/* etp_build_reverse_csr without a workspace argument and without allocating:
 * for callers that cannot allocate device memory where they need the reverse
 * CSR (a plugin inside a host program that owns the GPU memory budget, or a
 * time-critical loop that must not call cudaMalloc, which may synchronise the
 * device). The pages have no counterpart of this call; it is a deployment
 * convenience of this library.
 * Same arguments, outputs and result as etp_build_reverse_csr. The scratch is a
 * fixed file-scope device array of ETP_STATIC_SCRATCH_BYTES, present on every GPU
 * that loads the library until the process exits. N > ETP_STATIC_MAX_NODES or
 * E > ETP_STATIC_MAX_EDGES returns ETP_ERR_TOO_LARGE before any launch. The
 * first call on a device (the current device) looks up the array's device
 * address for that device; make that first call before any stream capture on
 * it. The address is kept for the life of the process: after cudaDeviceReset
 * (or any other teardown of the device's primary context) this call must not be
 * used on that device again. All calls share the one array: calls whose work overlaps on the GPU
 * (unordered streams or threads) race and give wrong results; calls ordered on
 * one stream are safe. */
ETP_API etp_status etp_build_reverse_csr_static(int N, int E, const int32_t* row_ptr, const int32_t* src,
                                                int32_t* rev_ptr, int32_t* rev_perm, int32_t* dst_of_edge,
                                                etp_stream_t stream);

/* Check a CSR on the device: zeroes *d_flag (a device int) and ORs in the
 * ETP_CSR_* bits of every violation found. Read the flag after the stream has
 * passed this call. */
ETP_API etp_status etp_validate_csr(int N, int E, const int32_t* row_ptr, const int32_t* src, int32_t* d_flag,
                            etp_stream_t stream);

/* Kernel fault report: every wait inside the kernels (on an asynchronous bulk
 * copy) is bounded; if one ever runs out, the kernel raises a flag, finishes its
 * work with the data it has (staying inside its buffers) and returns, instead of
 * hanging. This call synchronises the current device, returns the flag in
 * *fault (0: no wait ran out since the last call) and clears it. */
ETP_API etp_status etp_device_fault(int* fault);

/* A static description of a status code. */
ETP_API const char* etp_status_string(etp_status status);

#ifdef __cplusplus
}
#endif

#endif /* ETP_H_ */
