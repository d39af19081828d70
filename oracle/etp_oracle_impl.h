/* Loop bodies of the FP64 oracle, included twice by etp_oracle.c: once with
 * ORACLE_IN_T = double and once with ORACLE_IN_T = float (the element type of
 * x, w and g as stored; the arithmetic is double in both).
 *
 * TEST INFRASTRUCTURE ONLY: see etp_oracle.c.
 *
 * Notation: edge e goes from source j = src[e] to destination i (the CSR row
 * that holds e). The coupling of path p is given as its nonzero entries k in
 * [path_off[p], path_off[p+1]): value cg_val[k] connecting input component
 * cg_in[k] (absolute index into x's component axis), harmonic component
 * cg_sh[k] (absolute index into Y) and output component cg_out[k].
 */

/* out[s] = sum_{e in row rows[s]} sum_p sum_k w[e,p,c] cg Y[e,b] x[src e, a, c]
 * (one block of d_out*C doubles per requested row). */
void ORACLE_FN(oracle_forward)(
    int64_t n_rows, const int64_t *rows, const int32_t *row_ptr, const int32_t *src,
    int C, int d_in, int d_sh, int d_out, int P, const int32_t *path_off,
    const int32_t *cg_in, const int32_t *cg_sh, const int32_t *cg_out, const double *cg_val,
    const double *Y, const ORACLE_IN_T *x, const ORACLE_IN_T *w, double *out)
{
    int64_t s;
#pragma omp parallel for schedule(dynamic, 4)
    for (s = 0; s < n_rows; ++s) {
        int64_t i = rows[s];
        double *o = out + s * (int64_t)d_out * C;
        for (int64_t t = 0; t < (int64_t)d_out * C; ++t) o[t] = 0.0;
        for (int64_t e = row_ptr[i]; e < row_ptr[i + 1]; ++e) {
            int64_t j = src[e];
            for (int p = 0; p < P; ++p) {
                for (int c = 0; c < C; ++c) {
                    double wpc = (double)w[(e * P + p) * (int64_t)C + c];
                    for (int k = path_off[p]; k < path_off[p + 1]; ++k) {
                        double xv = (double)x[(j * d_in + cg_in[k]) * (int64_t)C + c];
                        o[(int64_t)cg_out[k] * C + c] += wpc * cg_val[k] * Y[e * d_sh + cg_sh[k]] * xv;
                    }
                }
            }
        }
    }
}

/* grad_x[s] for source node nodes[s]:
 *   sum_{e: src e = j} sum_p sum_k w[e,p,c] cg Y[e,b] g[dst e, o, c]   into component a.
 * rev_ptr/rev_perm list the edges of each source; dst[e] is the row of e. */
void ORACLE_FN(oracle_grad_x)(
    int64_t n_nodes, const int64_t *nodes, const int32_t *rev_ptr, const int32_t *rev_perm,
    const int32_t *dst, int C, int d_in, int d_sh, int d_out, int P, const int32_t *path_off,
    const int32_t *cg_in, const int32_t *cg_sh, const int32_t *cg_out, const double *cg_val,
    const double *Y, const ORACLE_IN_T *w, const ORACLE_IN_T *g, double *grad_x)
{
    int64_t s;
#pragma omp parallel for schedule(dynamic, 4)
    for (s = 0; s < n_nodes; ++s) {
        int64_t j = nodes[s];
        double *gx = grad_x + s * (int64_t)d_in * C;
        for (int64_t t = 0; t < (int64_t)d_in * C; ++t) gx[t] = 0.0;
        for (int64_t q = rev_ptr[j]; q < rev_ptr[j + 1]; ++q) {
            int64_t e = rev_perm[q];
            int64_t i = dst[e];
            for (int p = 0; p < P; ++p) {
                for (int c = 0; c < C; ++c) {
                    double wpc = (double)w[(e * P + p) * (int64_t)C + c];
                    for (int k = path_off[p]; k < path_off[p + 1]; ++k) {
                        double gv = (double)g[(i * d_out + cg_out[k]) * (int64_t)C + c];
                        gx[(int64_t)cg_in[k] * C + c] += wpc * cg_val[k] * Y[e * d_sh + cg_sh[k]] * gv;
                    }
                }
            }
        }
    }
}

/* For each requested edge e = edges[s] (source j, destination i):
 *   grad_w[s, p, c] = sum_k cg Y[e,b] x[j,a,c] g[i,o,c]
 *   dL/dY_b        = sum_p sum_c w[e,p,c] sum_{k: sh comp b} cg x[j,a,c] g[i,o,c]
 *   grad_r[s, t]   = sum_b dL/dY_b dY[e,b,t]
 * Either output may be NULL. */
void ORACLE_FN(oracle_grad_wr)(
    int64_t n_edges, const int64_t *edges, const int32_t *src, const int32_t *dst,
    int C, int d_in, int d_sh, int d_out, int P, const int32_t *path_off,
    const int32_t *cg_in, const int32_t *cg_sh, const int32_t *cg_out, const double *cg_val,
    const double *Y, const double *dY, const ORACLE_IN_T *x, const ORACLE_IN_T *w,
    const ORACLE_IN_T *g, double *grad_w, double *grad_r)
{
    int64_t s;
#pragma omp parallel for schedule(dynamic, 16)
    for (s = 0; s < n_edges; ++s) {
        int64_t e = edges[s];
        int64_t j = src[e], i = dst[e];
        double dLdY[64];
        for (int b = 0; b < d_sh; ++b) dLdY[b] = 0.0;
        for (int p = 0; p < P; ++p) {
            for (int c = 0; c < C; ++c) {
                double wpc = (double)w[(e * P + p) * (int64_t)C + c];
                double gw = 0.0;
                for (int k = path_off[p]; k < path_off[p + 1]; ++k) {
                    double xv = (double)x[(j * d_in + cg_in[k]) * (int64_t)C + c];
                    double gv = (double)g[(i * d_out + cg_out[k]) * (int64_t)C + c];
                    gw += cg_val[k] * Y[e * d_sh + cg_sh[k]] * xv * gv;
                    dLdY[cg_sh[k]] += wpc * cg_val[k] * xv * gv;
                }
                if (grad_w) grad_w[(s * P + p) * (int64_t)C + c] = gw;
            }
        }
        if (grad_r) {
            for (int t = 0; t < 3; ++t) {
                double acc = 0.0;
                for (int b = 0; b < d_sh; ++b) acc += dLdY[b] * dY[(e * d_sh + b) * 3 + t];
                grad_r[s * 3 + t] = acc;
            }
        }
    }
}
