/* FP64 CPU oracle of the edge-wise equivariant tensor product with neighbour
 * aggregation and its vector-Jacobian product.
 *
 * TEST INFRASTRUCTURE ONLY. This file is compiled into oracle/_build and loaded
 * by oracle/__init__.py; only tests/, __graft_entry__.smoke() and bench.py's CPU
 * baseline leg may call it. It shares no code, header or table with the CUDA
 * library.
 *
 * What it computes (the plain definition, no blocking or fusion):
 *   for every edge e = (i <- j) in the CSR-by-destination graph,
 *     msg_e[l3 m3, c] = sum_{p=(l1,l2,l3)} w[e,p,c] sum_{m1,m2} CG_p[m1,m2,m3] Y_{l2 m2}(r_e) x[j, l1 m1, c]
 *   out[i] = sum over the row of i of msg_e;
 * and for a cotangent g = dL/d(out) the transposed sums for grad_x, grad_w and
 * the derivative through Y for grad_r.
 * Passages: "High-performance training and inference for deep equivariant
 * interatomic potentials", section "제안 방법" (Wigner 3-j contraction of the
 * Allegro tensor product); "FlashCart 如何让等变原子间势更快更准?", sections
 * "FlashCart 用笛卡尔内核替代球谐耦合" (aggregation of edge contributions) and
 * "生成内核在高阶下胜过球谐基线" (edge convolution forward and vector-Jacobian
 * product); "Machine Learning Interatomic Potentials: Advancing Open-Source
 * Software ...", section "방법론 및 아키텍처" item 2 (Clebsch-Gordan tensor
 * products). Y, dY/dr and the CG entries are computed by oracle/sh.py and
 * oracle/cg.py and passed in.
 */
#include <stdint.h>
#include <stddef.h>

#define ORACLE_IN_T double
#define ORACLE_FN(name) name##_f64
#include "etp_oracle_impl.h"
#undef ORACLE_IN_T
#undef ORACLE_FN

#define ORACLE_IN_T float
#define ORACLE_FN(name) name##_f32
#include "etp_oracle_impl.h"
#undef ORACLE_IN_T
#undef ORACLE_FN

#ifdef _OPENMP
#include <omp.h>
int oracle_num_threads(void) { return omp_get_max_threads(); }
#else
int oracle_num_threads(void) { return 1; }
#endif
