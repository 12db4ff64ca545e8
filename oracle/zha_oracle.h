/*
 * ZHA oracle: declarations.
 *
 * TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT. Only tests/, the smoke check in
 * __graft_entry__.py and the cpu_baseline leg of bench.py may load this code.
 * It shares no code, header, table or helper with the CUDA library in
 * tree_indexed_sparse_append_b200/.
 *
 * Every array is row-major double. Node keys of level l are [n_l][R][d],
 * node biases [n_l][R]. Node j of level l summarizes nodes C*j .. C*j+C-1 of
 * level l-1 (level 0 = the original keys).
 */
#ifndef ZHA_ORACLE_H
#define ZHA_ORACLE_H

#ifdef __cplusplus
extern "C" {
#endif

#define ORC_MAX_LEVELS 16

enum { ORC_TOP_P = 0, ORC_TOP_K = 1 };

int orc_summarize(int n_children, int R, int d, double beta,
                  const double *child_keys, long long ck_stride_child, long long ck_stride_ref,
                  const double *child_bias, long long cb_stride_child,
                  const double *refs, int store_f32,
                  double *out_keys, double *out_bias);

int orc_build_level1(long long n_keys, int d, const double *K, int R, const double *refs,
                     int C, double beta, int store_f32, long long node_begin, long long node_end,
                     double *keys1, double *bias1, int threads);

int orc_build_level_up(int d, int R, const double *child_keys, const double *child_bias,
                       const double *refs, int C, double beta, int store_f32,
                       long long node_begin, long long node_end,
                       double *keys, double *bias, int threads);

int orc_search(int depth, const long long *n_nodes,
               const double *const *level_keys, const double *const *level_bias,
               int R, int d, int C, double beta, int top_width,
               const double *query, int mode, double p, int k,
               long long *sel, long long max_sel, long long *n_sel,
               long long *frontier, long long *opened, int *start_level,
               long long *keys_read, long long *work,
               double *tie_gap, double *tie_sum);

int orc_attend(long long n_keys, int d, double beta, const double *K, const double *V,
               const double *q, const long long *sel, long long n_sel, int C, long long n1,
               double *out, double *lse);

int orc_dense_scan(long long n_keys, int d, double beta, const double *K, const double *q,
                   int mode, double p, int k, long long *sel, long long max_sel,
                   long long *n_sel, double *tie_gap, double *tie_sum);

double orc_kept_mass(long long n_keys, int d, double beta, const double *K, const double *q,
                     const long long *sel, long long n_sel, int C, long long n1);

#ifdef __cplusplus
}
#endif
#endif
