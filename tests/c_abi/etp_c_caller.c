/* A plain C caller of libetp.so: the library used with no Python and no PyTorch.
 *
 *   etp_c_caller host               plan creation, queries and host-side argument
 *                                   checks only (no GPU needed)
 *   etp_c_caller run IN OUT         reads a problem from IN (binary, see read_problem),
 *                                   allocates device memory with the CUDA runtime, builds
 *                                   the reverse CSR and the edge frames, runs the forward
 *                                   and the VJP, assembles forces from grad_r, and writes
 *                                   out, grad_x, grad_w, grad_r, rev_ptr, rev_perm and
 *                                   forces to OUT.
 * Exit status 0 on success; a message on stderr otherwise. Test infrastructure. */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime.h>

#include "etp.h"

#define CHECK(cond, msg)                                      \
    do {                                                      \
        if (!(cond)) {                                        \
            fprintf(stderr, "etp_c_caller: %s (line %d)\n", msg, __LINE__); \
            return 1;                                         \
        }                                                     \
    } while (0)
#define ETP(call) CHECK((call) == ETP_OK, #call)
#define CUDA(call) CHECK((call) == cudaSuccess, #call)

static int host_checks(void) {
    etp_plan_t plan = NULL;
    int P = 0, din = 0, dsh = 0, dout = 0, nnz = 0;
    ETP(etp_plan_create(&plan, "0..3", 3, "0..3", 128, ETP_F32));
    ETP(etp_plan_info(plan, &P, &din, &dsh, &dout, NULL));
    CHECK(P == 34 && din == 16 && dsh == 16 && dout == 16, "plan shape");
    ETP(etp_plan_couplings(plan, &nnz, NULL, NULL, NULL, NULL, NULL));
    CHECK(nnz > 0, "coupling count");
    CHECK(etp_forward(plan, -1, 0, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL) == ETP_ERR_INVALID_ARG,
          "negative N rejected");
    CHECK(etp_edge_frames(NULL, 4, NULL, NULL, NULL) == ETP_ERR_INVALID_ARG, "NULL plan rejected");
    etp_plan_t bad = NULL;
    CHECK(etp_plan_create(&bad, "0..4", 4, "0..4", 128, ETP_F32) == ETP_ERR_UNSUPPORTED, "L = 4 unsupported");
    CHECK(etp_plan_create(&bad, "0..2", 2, "0..2", 6, ETP_F32) == ETP_ERR_UNSUPPORTED, "C = 6 unsupported");
    CHECK(strlen(etp_status_string(ETP_ERR_CUDA)) > 0, "status string");
    int ops = 0;
    ETP(etp_node_product_ops(plan, 0, &ops));
    CHECK(ops == 1023, "node-local product cost model (spherical, L = 3)");
    ETP(etp_node_product_ops(plan, 1, &ops));
    CHECK(ops == 1128, "node-local product cost model (Cartesian, L = 3)");
    CHECK(etp_node_product(plan, 4, 0, 0, NULL, NULL, NULL, NULL) == ETP_ERR_INVALID_ARG, "node product K < 1 rejected");
    CHECK(etp_node_product(plan, 0, 3, 1, NULL, NULL, NULL, NULL) == ETP_OK, "node product with no nodes");
    ETP(etp_plan_destroy(plan));
    return 0;
}

/* IN: int32 N, E, L, C, o3 flag; int32 row_ptr[N+1], src[E]; float32 r[E*3],
 * x[N*D*C], w[E*P*C], g[N*D*C]. */
typedef struct {
    int32_t N, E, L, C, o3, D, P;
    int32_t *row_ptr, *src;
    float *r, *x, *w, *g;
} problem;

static int read_all(FILE* f, void* p, size_t bytes) { return fread(p, 1, bytes, f) == bytes; }

static int read_problem(const char* path, problem* pr) {
    FILE* f = fopen(path, "rb");
    CHECK(f, "open input");
    int32_t hdr[5];
    CHECK(read_all(f, hdr, sizeof hdr), "read header");
    pr->N = hdr[0], pr->E = hdr[1], pr->L = hdr[2], pr->C = hdr[3], pr->o3 = hdr[4];
    pr->D = (pr->L + 1) * (pr->L + 1);
    size_t nd = (size_t)pr->N * pr->D * pr->C;
    pr->row_ptr = malloc(4 * ((size_t)pr->N + 1));
    pr->src = malloc(4 * (size_t)pr->E + 4);
    pr->r = malloc(12 * (size_t)pr->E + 4);
    pr->x = malloc(4 * nd);
    pr->g = malloc(4 * nd);
    CHECK(pr->row_ptr && pr->src && pr->r && pr->x && pr->g, "host allocation");
    CHECK(read_all(f, pr->row_ptr, 4 * ((size_t)pr->N + 1)), "read row_ptr");
    CHECK(read_all(f, pr->src, 4 * (size_t)pr->E), "read src");
    CHECK(read_all(f, pr->r, 12 * (size_t)pr->E), "read r");
    CHECK(read_all(f, pr->x, 4 * nd), "read x");
    long pos = ftell(f);
    fseek(f, 0, SEEK_END);
    long end = ftell(f);
    fseek(f, pos, SEEK_SET);
    size_t wbytes = (size_t)(end - pos) - 4 * nd;
    pr->P = (int32_t)(wbytes / (4 * (size_t)pr->E * pr->C));
    pr->w = malloc(wbytes + 4);
    CHECK(pr->w, "host allocation");
    CHECK(read_all(f, pr->w, wbytes), "read w");
    CHECK(read_all(f, pr->g, 4 * nd), "read g");
    fclose(f);
    return 0;
}

static void* dev_copy(const void* h, size_t bytes) {
    void* d = NULL;
    if (cudaMalloc(&d, bytes ? bytes : 16) != cudaSuccess) return NULL;
    if (bytes && cudaMemcpy(d, h, bytes, cudaMemcpyHostToDevice) != cudaSuccess) return NULL;
    return d;
}

static int run(const char* in, const char* out_path) {
    problem pr;
    if (read_problem(in, &pr)) return 1;
    char irreps[64];
    if (pr.o3)
        snprintf(irreps, sizeof irreps, "%s", pr.L == 0 ? "0e" : pr.L == 1 ? "0e+1o" : pr.L == 2 ? "0e+1o+2e" : "0e+1o+2e+3o");
    else
        snprintf(irreps, sizeof irreps, "0..%d", pr.L);
    etp_plan_t plan = NULL;
    ETP(etp_plan_create(&plan, irreps, pr.L, irreps, pr.C, ETP_F32));
    int P = 0;
    ETP(etp_plan_info(plan, &P, NULL, NULL, NULL, NULL));
    CHECK(P == pr.P, "path count of the input");
    const int N = pr.N, E = pr.E, D = pr.D, C = pr.C;
    const size_t nd = (size_t)N * D * C, ew = (size_t)E * P * C;
    int32_t* d_row_ptr = dev_copy(pr.row_ptr, 4 * ((size_t)N + 1));
    int32_t* d_src = dev_copy(pr.src, 4 * (size_t)E);
    float* d_r = dev_copy(pr.r, 12 * (size_t)E);
    float* d_x = dev_copy(pr.x, 4 * nd);
    float* d_w = dev_copy(pr.w, 4 * ew);
    float* d_g = dev_copy(pr.g, 4 * nd);
    CHECK(d_row_ptr && d_src && d_r && d_x && d_w && d_g, "device inputs");
    float *d_out, *d_gx, *d_gw, *d_gr, *d_frames, *d_forces;
    int32_t *d_rev_ptr, *d_rev_perm, *d_dst, *d_flag;
    void* d_ws;
    size_t ws_bytes = 0;
    ETP(etp_reverse_csr_workspace_size(N, E, &ws_bytes));
    size_t tp_bytes = 0;
    ETP(etp_tp_workspace_size(plan, N, E, 0, &tp_bytes));
    if (tp_bytes > ws_bytes) ws_bytes = tp_bytes; /* one workspace, used by one call at a time on one stream */
    CUDA(cudaMalloc((void**)&d_out, 4 * nd));
    CUDA(cudaMalloc((void**)&d_gx, 4 * nd));
    CUDA(cudaMalloc((void**)&d_gw, 4 * ew + 16));
    CUDA(cudaMalloc((void**)&d_gr, 12 * (size_t)E + 16));
    CUDA(cudaMalloc((void**)&d_frames, 4 * (size_t)ETP_FRAME_FLOATS * E + 16));
    CUDA(cudaMalloc((void**)&d_rev_ptr, 4 * ((size_t)N + 1)));
    CUDA(cudaMalloc((void**)&d_rev_perm, 4 * (size_t)E + 16));
    CUDA(cudaMalloc((void**)&d_dst, 4 * (size_t)E + 16));
    CUDA(cudaMalloc((void**)&d_flag, 4));
    CUDA(cudaMalloc((void**)&d_forces, 12 * (size_t)N));
    CUDA(cudaMalloc(&d_ws, ws_bytes + 16));
    cudaStream_t s;
    CUDA(cudaStreamCreate(&s));
    etp_stream_t es = (etp_stream_t)s;
    ETP(etp_validate_csr(N, E, d_row_ptr, d_src, d_flag, es));
    ETP(etp_build_reverse_csr(N, E, d_row_ptr, d_src, d_rev_ptr, d_rev_perm, d_dst, d_ws, ws_bytes, es));
    ETP(etp_edge_frames(plan, E, d_r, d_frames, es));
    ETP(etp_forward(plan, N, E, d_row_ptr, d_src, NULL, d_frames, d_x, d_w, d_out, d_ws, ws_bytes, es));
    ETP(etp_backward(plan, N, E, d_row_ptr, d_src, d_rev_ptr, d_rev_perm, d_dst, NULL, d_frames, d_x, d_w, d_g,
                     d_gx, d_gw, d_gr, d_ws, ws_bytes, es));
    ETP(etp_assemble_forces(N, E, d_row_ptr, d_rev_ptr, d_rev_perm, NULL, d_gr, d_forces, NULL, es));
    CUDA(cudaStreamSynchronize(s));
    int flag = -1, fault = -1;
    CUDA(cudaMemcpy(&flag, d_flag, 4, cudaMemcpyDeviceToHost));
    CHECK(flag == 0, "the input CSR is valid");
    ETP(etp_device_fault(&fault));
    CHECK(fault == 0, "no bounded wait ran out");
    float* h = malloc(4 * (ew > nd ? ew : nd) + 16);
    int32_t* hi = malloc(4 * ((size_t)(E > N + 1 ? E : N + 1)) + 16);
    CHECK(h && hi, "host allocation");
    FILE* f = fopen(out_path, "wb");
    CHECK(f, "open output");
    CUDA(cudaMemcpy(h, d_out, 4 * nd, cudaMemcpyDeviceToHost));
    fwrite(h, 4, nd, f);
    CUDA(cudaMemcpy(h, d_gx, 4 * nd, cudaMemcpyDeviceToHost));
    fwrite(h, 4, nd, f);
    CUDA(cudaMemcpy(h, d_gw, 4 * ew, cudaMemcpyDeviceToHost));
    fwrite(h, 4, ew, f);
    CUDA(cudaMemcpy(h, d_gr, 12 * (size_t)E, cudaMemcpyDeviceToHost));
    fwrite(h, 4, 3 * (size_t)E, f);
    CUDA(cudaMemcpy(hi, d_rev_ptr, 4 * ((size_t)N + 1), cudaMemcpyDeviceToHost));
    fwrite(hi, 4, (size_t)N + 1, f);
    CUDA(cudaMemcpy(hi, d_rev_perm, 4 * (size_t)E, cudaMemcpyDeviceToHost));
    fwrite(hi, 4, (size_t)E, f);
    CUDA(cudaMemcpy(h, d_forces, 12 * (size_t)N, cudaMemcpyDeviceToHost));
    fwrite(h, 4, 3 * (size_t)N, f);
    fclose(f);
    cudaStreamDestroy(s);
    ETP(etp_plan_destroy(plan));
    return 0;
}

int main(int argc, char** argv) {
    if (argc == 2 && !strcmp(argv[1], "host")) return host_checks();
    if (argc == 4 && !strcmp(argv[1], "run")) return run(argv[2], argv[3]);
    fprintf(stderr, "usage: %s host | run IN OUT\n", argv[0]);
    return 2;
}
