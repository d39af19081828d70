// C ABI of the edge tensor product library (declared in include/etp.h):
// plan lifecycle, host-side argument checks, and launches on the caller's stream.
#include <cuda_runtime.h>

#include <cctype>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <new>
#include <string>
#include <vector>

#include "etp.h"
#include "etp_device.cuh"
#include "etp_internal.h"

struct etp_plan_s {
    int L;
    bool o3;
    int C;
    int P;
    int D;
    std::vector<int> paths;  // 3 * P
};

namespace {

struct Irrep {
    int l;
    int parity;  // 0: none, +1: even, -1: odd
};

// "a..b" | "l[e|o]+l[e|o]+..." ; whitespace ignored. false on a malformed string.
bool parse_irreps(const char* s, std::vector<Irrep>& out) {
    out.clear();
    std::string t;
    for (const char* c = s; *c; ++c)
        if (!std::isspace((unsigned char)*c)) t.push_back(*c);
    if (t.empty()) return false;
    size_t dots = t.find("..");
    if (dots != std::string::npos) {
        std::string a = t.substr(0, dots), b = t.substr(dots + 2);
        if (a.empty() || b.empty() || a.size() > 3 || b.size() > 3) return false;
        for (char c : a + b)
            if (!std::isdigit((unsigned char)c)) return false;
        int lo = std::stoi(a), hi = std::stoi(b);
        if (lo > hi) return false;
        for (int l = lo; l <= hi; ++l) out.push_back({l, 0});
        return true;
    }
    size_t pos = 0;
    while (pos <= t.size()) {
        size_t plus = t.find('+', pos);
        std::string tok = t.substr(pos, plus == std::string::npos ? std::string::npos : plus - pos);
        if (tok.empty()) return false;
        int par = 0;
        if (tok.back() == 'e' || tok.back() == 'o') {
            par = tok.back() == 'e' ? 1 : -1;
            tok.pop_back();
        }
        if (tok.empty() || tok.size() > 3) return false;
        for (char c : tok)
            if (!std::isdigit((unsigned char)c)) return false;
        out.push_back({std::stoi(tok), par});
        if (plus == std::string::npos) break;
        pos = plus + 1;
    }
    for (size_t k = 1; k < out.size(); ++k)
        if (out[k].l <= out[k - 1].l || (out[k].parity == 0) != (out[0].parity == 0)) return false;
    return true;
}

// irreps 0..L each once; parities absent everywhere, or natural everywhere.
// Returns L, or -1 if the list is not of that form.
int full_range(const std::vector<Irrep>& v, int* parity_mode) {
    for (size_t k = 0; k < v.size(); ++k) {
        if (v[k].l != (int)k) return -1;
        int natural = (k % 2 == 0) ? 1 : -1;
        if (v[k].parity != 0 && v[k].parity != natural) return -1;
    }
    *parity_mode = v[0].parity != 0 ? 1 : 0;
    return (int)v.size() - 1;
}

template <int L, bool O3>
void fill_paths(std::vector<int>& out) {
    using PS = etp::PathSet<L, O3>;
    out.clear();
    for (int p = 0; p < PS::P; ++p) {
        etp::Path pt = PS::path(p);
        out.push_back(pt.l1);
        out.push_back(pt.l2);
        out.push_back(pt.l3);
    }
}

void plan_paths(int L, bool o3, std::vector<int>& out) {
    switch (L * 2 + (o3 ? 1 : 0)) {
        case 0: fill_paths<0, false>(out); break;
        case 1: fill_paths<0, true>(out); break;
        case 2: fill_paths<1, false>(out); break;
        case 3: fill_paths<1, true>(out); break;
        case 4: fill_paths<2, false>(out); break;
        case 5: fill_paths<2, true>(out); break;
        case 6: fill_paths<3, false>(out); break;
        default: fill_paths<3, true>(out); break;
    }
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

etp_status cuda_status(cudaError_t e) { return e == cudaSuccess ? ETP_OK : ETP_ERR_CUDA; }


}  // namespace

extern "C" {

etp_status etp_plan_create(etp_plan_t* plan, const char* irreps_in, int sh_lmax, const char* irreps_out, int C,
                           etp_dtype dtype) {
    if (!plan || !irreps_in || !irreps_out) return ETP_ERR_INVALID_ARG;
    *plan = nullptr;
    std::vector<Irrep> ins, outs;
    if (!parse_irreps(irreps_in, ins) || !parse_irreps(irreps_out, outs)) return ETP_ERR_INVALID_ARG;
    if ((ins[0].parity == 0) != (outs[0].parity == 0)) return ETP_ERR_INVALID_ARG;
    if (sh_lmax < 0 || C <= 0) return ETP_ERR_INVALID_ARG;
    if (dtype != ETP_F32) return ETP_ERR_UNSUPPORTED;
    int pm_in = 0, pm_out = 0;
    int L_in = full_range(ins, &pm_in), L_out = full_range(outs, &pm_out);
    if (L_in < 0 || L_out != L_in || sh_lmax != L_in || L_in > etp_gen::kLmax) return ETP_ERR_UNSUPPORTED;
    if (C % 4 != 0) return ETP_ERR_UNSUPPORTED;
    int C4 = C / 4;
    if (C4 > 32 || (C4 & (C4 - 1)) != 0) return ETP_ERR_UNSUPPORTED;
    etp_plan_s* p = new (std::nothrow) etp_plan_s();
    if (!p) return ETP_ERR_ALLOC;
    p->L = L_in;
    p->o3 = pm_in != 0;
    p->C = C;
    p->D = (L_in + 1) * (L_in + 1);
    try {
        plan_paths(p->L, p->o3, p->paths);
    } catch (...) {
        delete p;
        return ETP_ERR_ALLOC;
    }
    p->P = (int)p->paths.size() / 3;
    *plan = p;
    return ETP_OK;
}

etp_status etp_plan_info(etp_plan_t plan, int* n_paths, int* dim_in, int* dim_sh, int* dim_out, int* paths_l1l2l3) {
    if (!plan) return ETP_ERR_INVALID_ARG;
    if (n_paths) *n_paths = plan->P;
    if (dim_in) *dim_in = plan->D;
    if (dim_sh) *dim_sh = plan->D;
    if (dim_out) *dim_out = plan->D;
    if (paths_l1l2l3) std::memcpy(paths_l1l2l3, plan->paths.data(), sizeof(int) * plan->paths.size());
    return ETP_OK;
}

etp_status etp_plan_couplings(etp_plan_t plan, int* nnz, int* path_off, int* m1, int* m2, int* m3, double* val) {
    if (!plan || !nnz) return ETP_ERR_INVALID_ARG;
    int total = 0;
    for (int p = 0; p < plan->P; ++p) {
        const int a = plan->paths[3 * p], b = plan->paths[3 * p + 1], c = plan->paths[3 * p + 2];
        total += etp_gen::kCgCnt[a][b][c];
    }
    *nnz = total;
    const bool want = path_off || m1 || m2 || m3 || val;
    if (!want) return ETP_OK;
    if (!path_off || !m1 || !m2 || !m3 || !val) return ETP_ERR_INVALID_ARG;
    int k = 0;
    path_off[0] = 0;
    for (int p = 0; p < plan->P; ++p) {
        const int a = plan->paths[3 * p], b = plan->paths[3 * p + 1], c = plan->paths[3 * p + 2];
        const int off = etp_gen::kCgOff[a][b][c], cnt = etp_gen::kCgCnt[a][b][c];
        for (int q = 0; q < cnt; ++q, ++k) {
            m1[k] = etp_gen::kCg[off + q].m1;
            m2[k] = etp_gen::kCg[off + q].m2;
            m3[k] = etp_gen::kCg[off + q].m3;
            val[k] = etp_gen::kCg[off + q].v;
        }
        path_off[p + 1] = k;
    }
    return ETP_OK;
}

etp_status etp_plan_destroy(etp_plan_t plan) {
    delete plan;
    return ETP_OK;
}

etp_status etp_edge_frames(etp_plan_t plan, int E, const float* r, float* frames, etp_stream_t stream) {
    if (!plan || E < 0) return ETP_ERR_INVALID_ARG;
    if (E == 0) return ETP_OK;
    if (!r || !frames || !aligned4(r) || !aligned16(frames)) return ETP_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t err;
    switch (plan->L) {
        case 0: err = etp::launch_edge_frames<0>(E, r, frames, s); break;
        case 1: err = etp::launch_edge_frames<1>(E, r, frames, s); break;
        case 2: err = etp::launch_edge_frames<2>(E, r, frames, s); break;
        default: err = etp::launch_edge_frames<3>(E, r, frames, s); break;
    }
    return cuda_status(err);
}

etp_status etp_plan_frames_advised(etp_plan_t plan, int E, int* use_records) {
    if (!plan || E < 0 || !use_records) return ETP_ERR_INVALID_ARG;
    const size_t bytes = (size_t)E * ETP_FRAME_FLOATS * sizeof(float);
    // L <= 1 kernels use no Wigner matrices beyond the rotation itself: records never pay
    *use_records = (plan->L >= 2 && bytes <= (size_t)64 << 20) ? 1 : 0;
    return ETP_OK;
}

namespace {

// Waves of tasks of a locality schedule: the tasks in flight hold about
// 1/waves of the rows, in the schedule's order.
constexpr int kOrderedWaves = 8;

// Bytes of partial rows the forward (backward) of this plan, graph size and
// schedule needs, the larger of the two frame variants.
size_t partial_bytes(etp_plan_t plan, int N, int E, bool backward, bool ordered) {
    if (E <= 0 || N <= 0) return 0;
    size_t b = 0;
    for (int framed = 0; framed < 2; ++framed) {
        const etp::LaunchShape sh =
            etp::launch_shape(plan->C, plan->L, plan->o3, backward, framed != 0, E, N, ordered ? kOrderedWaves : 1);
        const size_t v = etp::partial_rows_bytes(sh.ntasks, plan->D, plan->C);
        b = v > b ? v : b;
    }
    return b;
}

etp_status forward_impl(etp_plan_t plan, int N, int E, const int32_t* row_ptr, const int32_t* src, const float* r,
                        const float* frames, const float* x, const float* w, float* out, const int32_t* order,
                        const int32_t* pos_edge, void* workspace, size_t workspace_bytes, etp_stream_t stream) {
    if (!plan || N < 0 || E < 0) return ETP_ERR_INVALID_ARG;
    if (N == 0) return E == 0 ? ETP_OK : ETP_ERR_INVALID_ARG;
    if (!row_ptr || !x || !out || !aligned4(row_ptr) || !aligned16(x) || !aligned16(out)) return ETP_ERR_INVALID_ARG;
    if (E > 0 && (!src || !w || !aligned4(src) || !aligned16(w))) return ETP_ERR_INVALID_ARG;
    if (E > 0 && (frames ? !aligned16(frames) : (!r || !aligned4(r)))) return ETP_ERR_INVALID_ARG;
    if ((order && !aligned4(order)) || (pos_edge && !aligned4(pos_edge))) return ETP_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (E == 0) return cuda_status(cudaMemsetAsync(out, 0, sizeof(float) * (size_t)N * plan->D * plan->C, s));
    const etp::LaunchShape sh = etp::launch_shape(plan->C, plan->L, plan->o3, false, frames != nullptr, E, N,
                                                  order ? kOrderedWaves : 1);
    if (!workspace || !aligned16(workspace)) return ETP_ERR_INVALID_ARG;
    if (workspace_bytes < etp::partial_rows_bytes(sh.ntasks, plan->D, plan->C)) return ETP_ERR_WORKSPACE;
    cudaError_t err;
    etp::FwdArgs a{N,
                   E,
                   row_ptr,
                   src,
                   r,
                   frames,
                   reinterpret_cast<const float4*>(x),
                   reinterpret_cast<const float4*>(w),
                   reinterpret_cast<float4*>(out),
                   plan->C / 4,
                   sh.team,
                   sh.slices,
                   sh.ntasks,
                   order,
                   pos_edge,
                   static_cast<float4*>(workspace)};
    switch (plan->L) {
        case 0: err = etp::launch_forward<0>(plan->o3, a, sh.grid, sh.smem_bytes, s); break;
        case 1: err = etp::launch_forward<1>(plan->o3, a, sh.grid, sh.smem_bytes, s); break;
        case 2: err = etp::launch_forward<2>(plan->o3, a, sh.grid, sh.smem_bytes, s); break;
        default: err = etp::launch_forward<3>(plan->o3, a, sh.grid, sh.smem_bytes, s); break;
    }
    if (err != cudaSuccess) return cuda_status(err);
    return cuda_status(etp::launch_combine_rows(row_ptr, order, N, E, sh.ntasks, plan->D * plan->C / 4,
                                                static_cast<const float4*>(workspace), reinterpret_cast<float4*>(out),
                                                s));
}

etp_status backward_impl(etp_plan_t plan, int N, int E, const int32_t* row_ptr, const int32_t* src,
                         const int32_t* rev_ptr, const int32_t* rev_perm, const int32_t* dst_of_edge, const float* r,
                         const float* frames, const float* x, const float* w, const float* grad_out, float* grad_x,
                         float* grad_w, float* grad_r, const int32_t* order, void* workspace,
                         size_t workspace_bytes, etp_stream_t stream) {
    if (!plan || N < 0 || E < 0) return ETP_ERR_INVALID_ARG;
    if (N == 0) return E == 0 ? ETP_OK : ETP_ERR_INVALID_ARG;
    if (!rev_ptr || !x || !grad_out || !aligned4(rev_ptr) || !aligned16(x) || !aligned16(grad_out))
        return ETP_ERR_INVALID_ARG;
    if (row_ptr ? !aligned4(row_ptr) : !dst_of_edge) return ETP_ERR_INVALID_ARG;  // one of them finds the rows
    if (order && !aligned4(order)) return ETP_ERR_INVALID_ARG;
    if (grad_x && !aligned16(grad_x)) return ETP_ERR_INVALID_ARG;
    if (E > 0) {
        if (!rev_perm || !w || !aligned4(rev_perm) || !aligned16(w)) return ETP_ERR_INVALID_ARG;
        if (src && !aligned4(src)) return ETP_ERR_INVALID_ARG;
        if (frames ? !aligned16(frames) : (!r || !aligned4(r))) return ETP_ERR_INVALID_ARG;
        if ((grad_w && !aligned16(grad_w)) || (grad_r && !aligned4(grad_r)) ||
            (dst_of_edge && !aligned4(dst_of_edge)))
            return ETP_ERR_INVALID_ARG;
    } else {
        grad_w = nullptr;
        grad_r = nullptr;
    }
    if (!grad_x && !grad_w && !grad_r) return ETP_OK;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (E == 0)
        return grad_x ? cuda_status(cudaMemsetAsync(grad_x, 0, sizeof(float) * (size_t)N * plan->D * plan->C, s))
                      : ETP_OK;
    const etp::LaunchShape sh = etp::launch_shape(plan->C, plan->L, plan->o3, true, frames != nullptr, E, N,
                                                  order ? kOrderedWaves : 1);
    if (grad_x) {
        if (!workspace || !aligned16(workspace)) return ETP_ERR_INVALID_ARG;
        if (workspace_bytes < etp::partial_rows_bytes(sh.ntasks, plan->D, plan->C)) return ETP_ERR_WORKSPACE;
    }
    cudaError_t err;
    etp::BwdArgs a{N,
                   E,
                   row_ptr,
                   src,
                   rev_ptr,
                   rev_perm,
                   dst_of_edge,
                   r,
                   frames,
                   reinterpret_cast<const float4*>(x),
                   reinterpret_cast<const float4*>(w),
                   reinterpret_cast<const float4*>(grad_out),
                   reinterpret_cast<float4*>(grad_x),
                   reinterpret_cast<float4*>(grad_w),
                   grad_r,
                   plan->C / 4,
                   sh.team,
                   sh.slices,
                   sh.ntasks,
                   order,
                   grad_x ? static_cast<float4*>(workspace) : nullptr};
    switch (plan->L) {
        case 0: err = etp::launch_backward<0>(plan->o3, a, sh.grid, sh.smem_bytes, s); break;
        case 1: err = etp::launch_backward<1>(plan->o3, a, sh.grid, sh.smem_bytes, s); break;
        case 2: err = etp::launch_backward<2>(plan->o3, a, sh.grid, sh.smem_bytes, s); break;
        default: err = etp::launch_backward<3>(plan->o3, a, sh.grid, sh.smem_bytes, s); break;
    }
    if (err != cudaSuccess || !grad_x) return cuda_status(err);
    return cuda_status(etp::launch_combine_rows(rev_ptr, order, N, E, sh.ntasks, plan->D * plan->C / 4,
                                                static_cast<const float4*>(workspace),
                                                reinterpret_cast<float4*>(grad_x), s));
}

}  // namespace

etp_status etp_tp_workspace_size(etp_plan_t plan, int N, int E, int ordered, size_t* bytes) {
    if (!plan || N < 0 || E < 0 || !bytes) return ETP_ERR_INVALID_ARG;
    size_t m = partial_bytes(plan, N, E, false, ordered != 0);
    const size_t more[] = {partial_bytes(plan, N, E, true, ordered != 0),
                           etp::double_backward_partial_bytes(plan->L, plan->o3, plan->C, N, E),
                           etp::cart_partial_bytes(plan->L, plan->o3, plan->C, N, E)};
    for (size_t v : more) m = v > m ? v : m;
    *bytes = m;
    return ETP_OK;
}

etp_status etp_forward(etp_plan_t plan, int N, int E, const int32_t* row_ptr, const int32_t* src, const float* r,
                       const float* frames, const float* x, const float* w, float* out, void* workspace,
                       size_t workspace_bytes, etp_stream_t stream) {
    return forward_impl(plan, N, E, row_ptr, src, r, frames, x, w, out, nullptr, nullptr, workspace, workspace_bytes,
                        stream);
}

etp_status etp_forward_ordered(etp_plan_t plan, int N, int E, const int32_t* order, const int32_t* ord_ptr,
                               const int32_t* ord_edge, const int32_t* src, const float* r, const float* frames,
                               const float* x, const float* w, float* out, void* workspace,
                               size_t workspace_bytes, etp_stream_t stream) {
    if (N > 0 && (!order || (E > 0 && !ord_edge))) return ETP_ERR_INVALID_ARG;
    return forward_impl(plan, N, E, ord_ptr, src, r, frames, x, w, out, order, ord_edge, workspace, workspace_bytes,
                        stream);
}

etp_status etp_backward(etp_plan_t plan, int N, int E, const int32_t* row_ptr, const int32_t* src,
                        const int32_t* rev_ptr, const int32_t* rev_perm, const int32_t* dst_of_edge, const float* r,
                        const float* frames, const float* x, const float* w, const float* grad_out, float* grad_x,
                        float* grad_w, float* grad_r, void* workspace, size_t workspace_bytes, etp_stream_t stream) {
    if (!row_ptr || (E > 0 && !src)) return ETP_ERR_INVALID_ARG;
    return backward_impl(plan, N, E, row_ptr, src, rev_ptr, rev_perm, dst_of_edge, r, frames, x, w, grad_out, grad_x,
                         grad_w, grad_r, nullptr, workspace, workspace_bytes, stream);
}

etp_status etp_backward_ordered(etp_plan_t plan, int N, int E, const int32_t* order, const int32_t* rev_ptr,
                                const int32_t* rev_perm, const int32_t* dst_of_edge, const float* r,
                                const float* frames, const float* x, const float* w, const float* grad_out,
                                float* grad_x, float* grad_w, float* grad_r, void* workspace,
                                size_t workspace_bytes, etp_stream_t stream) {
    if (N > 0 && (!order || (E > 0 && !dst_of_edge))) return ETP_ERR_INVALID_ARG;
    return backward_impl(plan, N, E, nullptr, nullptr, rev_ptr, rev_perm, dst_of_edge, r, frames, x, w, grad_out,
                         grad_x, grad_w, grad_r, order, workspace, workspace_bytes, stream);
}

etp_status etp_double_backward(etp_plan_t plan, int N, int E, const int32_t* row_ptr, const int32_t* src,
                               const int32_t* rev_ptr, const int32_t* rev_perm, const int32_t* dst_of_edge,
                               const float* r, const float* x, const float* w, const float* grad_out,
                               const float* gg_x, const float* gg_w, const float* gg_r, float* grad_grad_out,
                               float* grad_x, float* grad_w, float* grad_r, void* workspace,
                               size_t workspace_bytes, etp_stream_t stream) {
    if (!plan || N < 0 || E < 0) return ETP_ERR_INVALID_ARG;
    if (N == 0) return E == 0 ? ETP_OK : ETP_ERR_INVALID_ARG;
    if (!row_ptr || !rev_ptr || !x || !grad_out || !aligned4(row_ptr) || !aligned4(rev_ptr) || !aligned16(x) ||
        !aligned16(grad_out))
        return ETP_ERR_INVALID_ARG;
    if ((gg_x && !aligned16(gg_x)) || (grad_grad_out && !aligned16(grad_grad_out)) || (grad_x && !aligned16(grad_x)))
        return ETP_ERR_INVALID_ARG;
    if (E > 0) {
        if (!src || !rev_perm || !w || !r || !aligned4(src) || !aligned4(rev_perm) || !aligned16(w) || !aligned4(r))
            return ETP_ERR_INVALID_ARG;
        if ((gg_w && !aligned16(gg_w)) || (gg_r && !aligned4(gg_r)) || (grad_w && !aligned16(grad_w)) ||
            (grad_r && !aligned4(grad_r)) || (dst_of_edge && !aligned4(dst_of_edge)))
            return ETP_ERR_INVALID_ARG;
    } else {
        grad_w = nullptr;
        grad_r = nullptr;
    }
    if (!grad_grad_out && !grad_x && !grad_w && !grad_r) return ETP_OK;
    if (E > 0 && (grad_grad_out || grad_x)) {
        if (!workspace || !aligned16(workspace)) return ETP_ERR_INVALID_ARG;
        if (workspace_bytes < etp::double_backward_partial_bytes(plan->L, plan->o3, plan->C, N, E))
            return ETP_ERR_WORKSPACE;
    }
    return cuda_status(etp::double_backward(plan->L, plan->o3, plan->C, N, E, row_ptr, src, rev_ptr, rev_perm,
                                            dst_of_edge, r, x, w, grad_out, gg_x, gg_w, gg_r, grad_grad_out, grad_x,
                                            grad_w, grad_r, workspace, workspace_bytes,
                                            reinterpret_cast<cudaStream_t>(stream)));
}

etp_status etp_cart_forward(etp_plan_t plan, int N, int E, const int32_t* row_ptr, const int32_t* src, const float* r,
                            const float* x, const float* w, float* out, void* workspace, size_t workspace_bytes,
                            etp_stream_t stream) {
    if (!plan || N < 0 || E < 0) return ETP_ERR_INVALID_ARG;
    if (N == 0) return E == 0 ? ETP_OK : ETP_ERR_INVALID_ARG;
    if (!row_ptr || !x || !out || !aligned4(row_ptr) || !aligned16(x) || !aligned16(out)) return ETP_ERR_INVALID_ARG;
    if (E > 0 && (!src || !w || !r || !aligned4(src) || !aligned16(w) || !aligned4(r))) return ETP_ERR_INVALID_ARG;
    if (E > 0) {
        if (!workspace || !aligned16(workspace)) return ETP_ERR_INVALID_ARG;
        if (workspace_bytes < etp::cart_partial_bytes(plan->L, plan->o3, plan->C, N, E)) return ETP_ERR_WORKSPACE;
    }
    return cuda_status(etp::cart_forward(plan->L, plan->o3, plan->C, N, E, row_ptr, src, r, x, w, out, workspace,
                                         workspace_bytes, reinterpret_cast<cudaStream_t>(stream)));
}

etp_status etp_cart_backward(etp_plan_t plan, int N, int E, const int32_t* row_ptr, const int32_t* src,
                             const int32_t* rev_ptr, const int32_t* rev_perm, const int32_t* dst_of_edge,
                             const float* r, const float* x, const float* w, const float* grad_out, float* grad_x,
                             float* grad_w, float* grad_r, void* workspace, size_t workspace_bytes,
                             etp_stream_t stream) {
    if (!plan || N < 0 || E < 0) return ETP_ERR_INVALID_ARG;
    if (N == 0) return E == 0 ? ETP_OK : ETP_ERR_INVALID_ARG;
    if (!row_ptr || !rev_ptr || !x || !grad_out || !aligned4(row_ptr) || !aligned4(rev_ptr) || !aligned16(x) ||
        !aligned16(grad_out))
        return ETP_ERR_INVALID_ARG;
    if (grad_x && !aligned16(grad_x)) return ETP_ERR_INVALID_ARG;
    if (E > 0) {
        if (!src || !rev_perm || !w || !r || !aligned4(src) || !aligned4(rev_perm) || !aligned16(w) || !aligned4(r))
            return ETP_ERR_INVALID_ARG;
        if ((grad_w && !aligned16(grad_w)) || (grad_r && !aligned4(grad_r)) ||
            (dst_of_edge && !aligned4(dst_of_edge)))
            return ETP_ERR_INVALID_ARG;
    } else {
        grad_w = nullptr;
        grad_r = nullptr;
    }
    if (!grad_x && !grad_w && !grad_r) return ETP_OK;
    if (E > 0 && grad_x) {
        if (!workspace || !aligned16(workspace)) return ETP_ERR_INVALID_ARG;
        if (workspace_bytes < etp::cart_partial_bytes(plan->L, plan->o3, plan->C, N, E)) return ETP_ERR_WORKSPACE;
    }
    return cuda_status(etp::cart_backward(plan->L, plan->o3, plan->C, N, E, row_ptr, rev_ptr, rev_perm, dst_of_edge,
                                          r, x, w, grad_out, grad_x, grad_w, grad_r, workspace, workspace_bytes,
                                          reinterpret_cast<cudaStream_t>(stream)));
}

etp_status etp_node_product(etp_plan_t plan, int N, int K, int cartesian, const float* x, const float* w,
                            float* out, etp_stream_t stream) {
    if (!plan || N < 0 || K < 1 || (cartesian != 0 && cartesian != 1)) return ETP_ERR_INVALID_ARG;
    if (N == 0) return ETP_OK;
    if (!x || !out || !aligned16(x) || !aligned16(out)) return ETP_ERR_INVALID_ARG;
    if (K > 1 && (!w || !aligned16(w))) return ETP_ERR_INVALID_ARG;
    return cuda_status(etp::node_product(plan->L, plan->o3, cartesian != 0, plan->C, N, K, x, w, out,
                                         reinterpret_cast<cudaStream_t>(stream)));
}

etp_status etp_node_product_ops(etp_plan_t plan, int cartesian, int* ops_per_step) {
    if (!plan || !ops_per_step || (cartesian != 0 && cartesian != 1)) return ETP_ERR_INVALID_ARG;
    *ops_per_step = etp::node_product_ops(plan->L, plan->o3, cartesian != 0);
    return ETP_OK;
}

etp_status etp_assemble_forces(int N, int E, const int32_t* row_ptr, const int32_t* rev_ptr, const int32_t* rev_perm,
                               const float* r, const float* grad_r, float* forces, float* virial, etp_stream_t stream) {
    if (N < 0 || E < 0) return ETP_ERR_INVALID_ARG;
    if (N == 0) return E == 0 ? ETP_OK : ETP_ERR_INVALID_ARG;
    if (!row_ptr || !rev_ptr || !forces || !aligned4(row_ptr) || !aligned4(rev_ptr) || !aligned4(forces))
        return ETP_ERR_INVALID_ARG;
    if (virial && !aligned4(virial)) return ETP_ERR_INVALID_ARG;
    if (E > 0 && (!rev_perm || !grad_r || !aligned4(rev_perm) || !aligned4(grad_r))) return ETP_ERR_INVALID_ARG;
    if (E > 0 && virial && (!r || !aligned4(r))) return ETP_ERR_INVALID_ARG;
    return cuda_status(etp::assemble_forces(N, E, row_ptr, rev_ptr, rev_perm, r, grad_r, forces, virial,
                                            reinterpret_cast<cudaStream_t>(stream)));
}

namespace {
bool radial_shape_ok(int n_basis, int hidden, float r_cut) {
    return n_basis >= 1 && n_basis <= 32 && hidden >= 32 && hidden <= 256 && hidden % 32 == 0 && r_cut > 0.f;
}
}  // namespace

etp_status etp_radial_workspace_size(etp_plan_t plan, int E, int n_basis, int hidden, size_t* bytes) {
    if (!plan || E < 0 || !bytes || !radial_shape_ok(n_basis, hidden, 1.f)) return ETP_ERR_INVALID_ARG;
    *bytes = etp::radial_workspace_bytes(E, n_basis, hidden, plan->P * plan->C);
    return ETP_OK;
}

etp_status etp_radial_forward(etp_plan_t plan, int E, int n_basis, int hidden, float r_cut, const float* r,
                              const float* W1, const float* W2, float* w, void* workspace, size_t workspace_bytes,
                              etp_stream_t stream) {
    if (!plan || E < 0 || !radial_shape_ok(n_basis, hidden, r_cut)) return ETP_ERR_INVALID_ARG;
    if (E == 0) return ETP_OK;
    if (!r || !W1 || !W2 || !w || !workspace || !aligned4(r) || !aligned4(W1) || !aligned4(W2) || !aligned16(w) ||
        !aligned16(workspace))
        return ETP_ERR_INVALID_ARG;
    if (workspace_bytes < etp::radial_workspace_bytes(E, n_basis, hidden, plan->P * plan->C)) return ETP_ERR_WORKSPACE;
    return cuda_status(etp::radial_forward(E, n_basis, hidden, plan->P * plan->C, r_cut, r, W1, W2, w, workspace,
                                           reinterpret_cast<cudaStream_t>(stream)));
}

etp_status etp_radial_backward(etp_plan_t plan, int E, int n_basis, int hidden, float r_cut, const float* r,
                               const float* W1, const float* W2, const float* grad_w, float* grad_W1, float* grad_W2,
                               float* grad_r, void* workspace, size_t workspace_bytes, etp_stream_t stream) {
    if (!plan || E < 0 || !radial_shape_ok(n_basis, hidden, r_cut)) return ETP_ERR_INVALID_ARG;
    if (!W1 || !W2 || !grad_W1 || !grad_W2 || !aligned4(W1) || !aligned4(W2) || !aligned4(grad_W1) ||
        !aligned4(grad_W2))
        return ETP_ERR_INVALID_ARG;
    if (E > 0 && (!r || !grad_w || !grad_r || !workspace || !aligned4(r) || !aligned16(grad_w) || !aligned4(grad_r) ||
                  !aligned16(workspace)))
        return ETP_ERR_INVALID_ARG;
    if (E > 0 && workspace_bytes < etp::radial_workspace_bytes(E, n_basis, hidden, plan->P * plan->C))
        return ETP_ERR_WORKSPACE;
    return cuda_status(etp::radial_backward(E, n_basis, hidden, plan->P * plan->C, r_cut, r, W1, W2, grad_w, grad_W1,
                                            grad_W2, grad_r, workspace, reinterpret_cast<cudaStream_t>(stream)));
}

etp_status etp_fused_workspace_size(etp_plan_t plan, int E, int n_basis, int hidden, size_t* bytes) {
    if (!plan || E < 0 || !bytes) return ETP_ERR_INVALID_ARG;
    if (!etp::fused_supported(n_basis, hidden)) return ETP_ERR_UNSUPPORTED;
    *bytes = etp::fused_workspace_bytes(plan->L, plan->o3, plan->C, E);
    return ETP_OK;
}

etp_status etp_fused_forward(etp_plan_t plan, int N, int E, const int32_t* row_ptr, const int32_t* src,
                             const float* r, const float* x, int n_basis, int hidden, float r_cut, const float* W1,
                             const float* W2, float* out, void* workspace, size_t workspace_bytes,
                             etp_stream_t stream) {
    if (!plan || N < 0 || E < 0 || !(r_cut > 0.f)) return ETP_ERR_INVALID_ARG;
    if (!etp::fused_supported(n_basis, hidden)) return ETP_ERR_UNSUPPORTED;
    if (N == 0) return E == 0 ? ETP_OK : ETP_ERR_INVALID_ARG;
    if (!row_ptr || !x || !out || !W1 || !W2 || !workspace || !aligned4(row_ptr) || !aligned16(x) ||
        !aligned16(out) || !aligned4(W1) || !aligned4(W2) || !aligned16(workspace))
        return ETP_ERR_INVALID_ARG;
    if (E > 0 && (!src || !r || !aligned4(src) || !aligned4(r))) return ETP_ERR_INVALID_ARG;
    if (workspace_bytes < etp::fused_workspace_bytes(plan->L, plan->o3, plan->C, E)) return ETP_ERR_WORKSPACE;
    return cuda_status(etp::fused_forward(plan->L, plan->o3, plan->C, N, E, row_ptr, src, r, x, W1, W2, r_cut, out,
                                          workspace, reinterpret_cast<cudaStream_t>(stream)));
}

etp_status etp_reverse_csr_workspace_size(int N, int E, size_t* bytes) {
    if (N < 0 || E < 0 || !bytes) return ETP_ERR_INVALID_ARG;
    *bytes = etp::reverse_csr_workspace_bytes(N, E);
    return ETP_OK;
}

etp_status etp_build_reverse_csr(int N, int E, const int32_t* row_ptr, const int32_t* src, int32_t* rev_ptr,
                                 int32_t* rev_perm, int32_t* dst_of_edge, void* workspace, size_t workspace_bytes,
                                 etp_stream_t stream) {
    if (N < 0 || E < 0) return ETP_ERR_INVALID_ARG;
    if (N == 0 && E > 0) return ETP_ERR_INVALID_ARG;
    if (!rev_ptr || !workspace || !aligned4(rev_ptr) || !aligned16(workspace)) return ETP_ERR_INVALID_ARG;
    if (E > 0 && (!row_ptr || !src || !rev_perm || !aligned4(row_ptr) || !aligned4(src) || !aligned4(rev_perm)))
        return ETP_ERR_INVALID_ARG;
    if (dst_of_edge && !aligned4(dst_of_edge)) return ETP_ERR_INVALID_ARG;
    if (workspace_bytes < etp::reverse_csr_workspace_bytes(N, E)) return ETP_ERR_WORKSPACE;
    return cuda_status(etp::build_reverse_csr(N, E, row_ptr, src, rev_ptr, rev_perm, dst_of_edge, workspace,
                                              reinterpret_cast<cudaStream_t>(stream)));
}

etp_status etp_locality_schedule_workspace_size(int N, int E, size_t* bytes) {
    if (N < 0 || E < 0 || !bytes) return ETP_ERR_INVALID_ARG;
    const size_t a = etp::spatial_order_workspace_bytes(N), b = etp::ordered_csr_workspace_bytes(N, E);
    *bytes = a > b ? a : b;
    return ETP_OK;
}

etp_status etp_build_locality_schedule(int N, int E, const int32_t* row_ptr, const int32_t* src, const float* pos,
                                       float cell, int32_t* order, int32_t* ord_ptr, int32_t* ord_edge,
                                       int32_t* rev_ptr, int32_t* rev_perm, int32_t* dst_of_edge, void* workspace,
                                       size_t workspace_bytes, etp_stream_t stream) {
    if (N < 0 || E < 0 || !(cell > 0.f) || !std::isfinite(cell)) return ETP_ERR_INVALID_ARG;
    if (N == 0) return E == 0 ? ETP_OK : ETP_ERR_INVALID_ARG;
    if (!row_ptr || !pos || !order || !ord_ptr || !rev_ptr || !workspace) return ETP_ERR_INVALID_ARG;
    if (!aligned4(row_ptr) || !aligned4(pos) || !aligned4(order) || !aligned4(ord_ptr) || !aligned4(rev_ptr) ||
        !aligned16(workspace))
        return ETP_ERR_INVALID_ARG;
    if (E > 0 && (!src || !ord_edge || !rev_perm || !dst_of_edge || !aligned4(src) || !aligned4(ord_edge) ||
                  !aligned4(rev_perm) || !aligned4(dst_of_edge)))
        return ETP_ERR_INVALID_ARG;
    size_t need = 0;
    etp_locality_schedule_workspace_size(N, E, &need);
    if (workspace_bytes < need) return ETP_ERR_WORKSPACE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t err = etp::spatial_order(N, pos, cell, order, workspace, s);
    if (err != cudaSuccess) return cuda_status(err);
    return cuda_status(etp::build_ordered_csr(N, E, row_ptr, src, order, ord_ptr, ord_edge, rev_ptr, rev_perm,
                                              dst_of_edge, workspace, s));
}

etp_status etp_validate_csr(int N, int E, const int32_t* row_ptr, const int32_t* src, int32_t* d_flag,
                            etp_stream_t stream) {
    if (N < 0 || E < 0 || !row_ptr || !d_flag || (E > 0 && !src)) return ETP_ERR_INVALID_ARG;
    if (!aligned4(row_ptr) || !aligned4(d_flag) || (src && !aligned4(src))) return ETP_ERR_INVALID_ARG;
    return cuda_status(etp::validate_csr(N, E, row_ptr, src, d_flag, reinterpret_cast<cudaStream_t>(stream)));
}

etp_status etp_device_fault(int* fault) {
    if (!fault) return ETP_ERR_INVALID_ARG;
    if (cudaDeviceSynchronize() != cudaSuccess) return ETP_ERR_CUDA;
    const int f0 = etp::read_and_clear_fault<0>(), f1 = etp::read_and_clear_fault<1>();
    const int f2 = etp::read_and_clear_fault<2>(), f3 = etp::read_and_clear_fault<3>();
    const int f4 = etp::radial_tc_read_and_clear_fault(), f5 = etp::fused_read_and_clear_fault();
    if (f0 < 0 || f1 < 0 || f2 < 0 || f3 < 0 || f4 < 0 || f5 < 0) return ETP_ERR_CUDA;
    *fault = f0 | f1 | f2 | f3 | f4 | f5;
    return ETP_OK;
}

const char* etp_status_string(etp_status status) {
    switch (status) {
        case ETP_OK: return "ok";
        case ETP_ERR_INVALID_ARG: return "invalid argument (null, negative size, misaligned pointer or bad string)";
        case ETP_ERR_UNSUPPORTED: return "unsupported irreps, L, C or dtype (no compiled kernel)";
        case ETP_ERR_BAD_CSR: return "malformed CSR graph";
        case ETP_ERR_CUDA: return "CUDA launch or runtime error";
        case ETP_ERR_ALLOC: return "host allocation failed";
        case ETP_ERR_WORKSPACE: return "workspace too small";
        case ETP_ERR_TOO_LARGE: return "N or E above the fixed scratch limit of the static-scratch variant";
    }
    return "unknown status";
}

}  // extern "C"
