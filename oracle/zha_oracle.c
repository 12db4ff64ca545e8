/*
 * ZHA oracle: a plain, slow, double-precision CPU restatement of the method.
 *
 * TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT. Only tests/, the smoke check in
 * __graft_entry__.py and the cpu_baseline leg of bench.py may load it. It shares
 * no code with the CUDA library and neither side includes the other.
 *
 * What it follows (page "How does a tree of summaries search a context? How ZHA
 * works", learn.chabulab.com, unless noted):
 *   - node summary: section "What does a node summarize?" (the summarize function
 *     and the paragraph on tangents that follows it);
 *   - tree shape, chunk fill, keys kept for the final attention: section "How is
 *     the tree built?";
 *   - node score, frontier softmax, top-p prefix, expansion: section "Run a small
 *     tree yourself" (the buildTree and route functions of tree.ts) and section
 *     "How does top-p differ from top-K?";
 *   - top-K opens exactly K nodes per level: sections "Try it" (item 3) and "How
 *     does top-p differ from top-K?";
 *   - final attention over exactly the chosen original keys: sections "How is the
 *     tree built?" and "Common misunderstandings";
 *   - the full-scan indexer used for comparison: page "Zyphra AI Introduces ZHA, a
 *     Path to True Subquadratic Attention" (DeepSeek Sparse Attention scores every
 *     token).
 *
 * Readings taken where the pages leave a step open (each is listed with its
 * reason in the design notes of the repository):
 *   - the walk starts at the lowest level holding at most top_width nodes (the
 *     demo stops building at 64 top nodes), or at the deepest level built;
 *   - keys not yet covered by a level-1 node (the tail) are always read;
 *   - a node whose parent group is not full (an orphan) joins the frontier of its
 *     own level;
 *   - top-K takes the K largest scores of the whole frontier of a level;
 *   - ties in mass are broken by ascending node id; p >= 1 opens every node;
 *   - node keys and biases may be rounded to fp32 when stored (store_f32: bit 0
 *     keys, bit 1 biases), and the next level is summarized from the stored values;
 *   - the bias is taken against the key as stored, as the demo does.
 *
 * Parity pins live in tests/ (closed forms, invariants, brute force, and the
 * printed output of the page's demo).
 */
#include "zha_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* store flags: bit 0 rounds node keys through fp32, bit 1 rounds node biases */
#define ORC_ROUND_KEYS 1
#define ORC_ROUND_BIAS 2

static double stored(double x, int round_f32) { return round_f32 ? (double)(float)x : x; }

static double dot(const double *a, const double *b, int d) {
    double s = 0.0;
    for (int t = 0; t < d; ++t) s += a[t] * b[t];
    return s;
}

static double max_of(const double *s, long long n) {
    double m = -INFINITY;
    for (long long i = 0; i < n; ++i)
        if (s[i] > m) m = s[i];
    return m;
}

/* log(sum_i exp(s_i)), max-subtracted */
static double log_sum_exp(const double *s, long long n) {
    double m = max_of(s, n);
    double z = 0.0;
    for (long long i = 0; i < n; ++i) z += exp(s[i] - m);
    return m + log(z);
}

/* softmax of n scores into w, max-subtracted */
static void softmax(const double *s, long long n, double *w) {
    double m = max_of(s, n);
    double z = 0.0;
    for (long long i = 0; i < n; ++i) {
        w[i] = exp(s[i] - m);
        z += w[i];
    }
    for (long long i = 0; i < n; ++i) w[i] /= z;
}

/*
 * One node from its children, for every reference query r:
 *   s_i    = beta * <key_{i,r}, q_r> + bias_{i,r}
 *   w      = softmax(s)
 *   key_r  = sum_i w_i key_{i,r}
 *   bias_r = logsumexp(s) - beta * <key_r, q_r>
 * Child i's key for reference r is child_keys[i*ck_stride_child + r*ck_stride_ref];
 * leaves pass ck_stride_ref = 0 (one key serves every reference) and a NULL bias.
 */
int orc_summarize(int n_children, int R, int d, double beta,
                  const double *child_keys, long long ck_stride_child, long long ck_stride_ref,
                  const double *child_bias, long long cb_stride_child,
                  const double *refs, int store_f32,
                  double *out_keys, double *out_bias) {
    if (n_children <= 0 || R <= 0 || d <= 0) return -1;
    double *s = (double *)malloc(sizeof(double) * (size_t)n_children);
    double *w = (double *)malloc(sizeof(double) * (size_t)n_children);
    double *acc = (double *)malloc(sizeof(double) * (size_t)d);
    if (!s || !w || !acc) {
        free(s); free(w); free(acc);
        return -2;
    }
    for (int r = 0; r < R; ++r) {
        const double *q = refs + (long long)r * d;
        for (int i = 0; i < n_children; ++i) {
            const double *k = child_keys + i * ck_stride_child + r * ck_stride_ref;
            double b = child_bias ? child_bias[i * cb_stride_child + r] : 0.0;
            s[i] = beta * dot(k, q, d) + b;
        }
        softmax(s, n_children, w);
        for (int t = 0; t < d; ++t) acc[t] = 0.0;
        for (int i = 0; i < n_children; ++i) {
            const double *k = child_keys + i * ck_stride_child + r * ck_stride_ref;
            for (int t = 0; t < d; ++t) acc[t] += w[i] * k[t];
        }
        double *key = out_keys + (long long)r * d;
        for (int t = 0; t < d; ++t) key[t] = stored(acc[t], store_f32 & ORC_ROUND_KEYS);
        out_bias[r] = stored(log_sum_exp(s, n_children) - beta * dot(key, q, d),
                             store_f32 & ORC_ROUND_BIAS);
    }
    free(s); free(w); free(acc);
    return 0;
}

/* Level-1 nodes [node_begin, node_end): node j summarizes keys C*j .. C*j+C-1. */
int orc_build_level1(long long n_keys, int d, const double *K, int R, const double *refs,
                     int C, double beta, int store_f32, long long node_begin, long long node_end,
                     double *keys1, double *bias1, int threads) {
    if (C <= 0 || node_end * C > n_keys || node_begin < 0) return -1;
    int err = 0;
    (void)threads;
#pragma omp parallel for schedule(dynamic, 16) num_threads(threads > 0 ? threads : 1) reduction(| : err)
    for (long long j = node_begin; j < node_end; ++j) {
        err |= orc_summarize(C, R, d, beta, K + j * C * d, d, 0, NULL, 0, refs, store_f32,
                             keys1 + j * R * d, bias1 + j * R);
    }
    return err ? -2 : 0;
}

/* Level-l nodes [node_begin, node_end) from level l-1 (keys [.][R][d], biases [.][R]). */
int orc_build_level_up(int d, int R, const double *child_keys, const double *child_bias,
                       const double *refs, int C, double beta, int store_f32,
                       long long node_begin, long long node_end,
                       double *keys, double *bias, int threads) {
    if (C <= 0 || node_begin < 0) return -1;
    int err = 0;
    (void)threads;
#pragma omp parallel for schedule(dynamic, 16) num_threads(threads > 0 ? threads : 1) reduction(| : err)
    for (long long j = node_begin; j < node_end; ++j) {
        err |= orc_summarize(C, R, d, beta, child_keys + j * C * R * d, (long long)R * d, d,
                             child_bias + j * C * R, R, refs, store_f32,
                             keys + j * R * d, bias + j * R);
    }
    return err ? -2 : 0;
}

/* ---------------------------------------------------------------------------
 * Traversal.
 */
typedef struct {
    double mass;
    long long id;
} ranked;

/* mass descending, then node id ascending */
static int by_mass_then_id(const void *a, const void *b) {
    const ranked *x = (const ranked *)a, *y = (const ranked *)b;
    if (x->mass > y->mass) return -1;
    if (x->mass < y->mass) return 1;
    return (x->id > y->id) - (x->id < y->id);
}

static int by_id(const void *a, const void *b) {
    long long x = *(const long long *)a, y = *(const long long *)b;
    return (x > y) - (x < y);
}

/*
 * Given the frontier's scores, rank them and count how many to open.
 * Also returns the closeness of the decision to a tie: the relative gap
 * between the last opened and the first unopened mass, and (top-p) the
 * distance of the running sum before/after the last opened node from p,
 * relative to p.
 */
static long long choose(ranked *rk, const double *score, const long long *ids, long long F,
                        int mode, double p, int k, double *gap, double *sumdist) {
    double *w = (double *)malloc(sizeof(double) * (size_t)F);
    softmax(score, F, w);
    for (long long i = 0; i < F; ++i) {
        rk[i].mass = w[i];
        rk[i].id = ids[i];
    }
    free(w);
    qsort(rk, (size_t)F, sizeof(ranked), by_mass_then_id);
    long long c;
    *gap = INFINITY;
    *sumdist = INFINITY;
    if (mode == ORC_TOP_K) {
        c = k < F ? k : F;
    } else if (p >= 1.0) {
        c = F;
    } else {
        double total = 0.0;
        c = 0;
        while (c < F) {
            double before = total;
            total += rk[c].mass;
            ++c;
            if (total >= p) {
                double a = (p - before) / p, b = (total - p) / p;
                *sumdist = a < b ? a : b;
                break;
            }
        }
    }
    if (c < F) *gap = (rk[c - 1].mass - rk[c].mass) / rk[c - 1].mass;
    return c;
}

/*
 * One walk of one query down one tree.
 *   n_nodes[0] = keys in the tree, n_nodes[l] = nodes at level l (1..depth),
 *   level_keys[l] / level_bias[l] = that level's arrays (index 0 unused).
 * Output: sel = opened level-1 node ids ascending (n_sel of them); frontier[l]
 * and opened[l] = sizes per level; keys_read = C*|sel| + tail; work =
 * R * sum(frontier) + keys_read; tie_gap / tie_sum = the smallest tie measures
 * met on the way (INFINITY when none applies).
 */
int orc_search(int depth, const long long *n_nodes,
               const double *const *level_keys, const double *const *level_bias,
               int R, int d, int C, double beta, int top_width,
               const double *query, int mode, double p, int k,
               long long *sel, long long max_sel, long long *n_sel,
               long long *frontier, long long *opened, int *start_level,
               long long *keys_read, long long *work,
               double *tie_gap, double *tie_sum) {
    if (depth < 1 || depth >= ORC_MAX_LEVELS || C < 1 || top_width < 1) return -1;
    if (mode == ORC_TOP_K && k < 1) return -1;
    if (mode == ORC_TOP_P && !(p > 0.0)) return -1;

    int s = depth;
    for (int l = 1; l <= depth; ++l)
        if (n_nodes[l] <= top_width) {
            s = l;
            break;
        }
    *start_level = s;
    for (int l = 0; l < ORC_MAX_LEVELS; ++l) frontier[l] = opened[l] = 0;
    *tie_gap = INFINITY;
    *tie_sum = INFINITY;

    long long cap = n_nodes[1] > n_nodes[s] ? n_nodes[1] : n_nodes[s];
    for (int l = 1; l <= depth; ++l)
        if (n_nodes[l] > cap) cap = n_nodes[l];
    if (cap < 1) cap = 1;
    long long *F = (long long *)malloc(sizeof(long long) * (size_t)cap);
    long long *next = (long long *)malloc(sizeof(long long) * (size_t)cap);
    double *score = (double *)malloc(sizeof(double) * (size_t)cap);
    ranked *rk = (ranked *)malloc(sizeof(ranked) * (size_t)cap);
    if (!F || !next || !score || !rk) {
        free(F); free(next); free(score); free(rk);
        return -2;
    }

    long long nF = n_nodes[s];
    for (long long j = 0; j < nF; ++j) F[j] = j;
    long long total_frontier = 0, chosen = 0;
    int rc = 0;

    for (int l = s; l >= 1; --l) {
        frontier[l] = nF;
        total_frontier += nF;
        long long c = 0;
        if (nF > 0) {
            const double *keys = level_keys[l];
            const double *bias = level_bias[l];
            for (long long i = 0; i < nF; ++i) {
                double best = -INFINITY;
                for (int r = 0; r < R; ++r) {
                    double v = beta * dot(keys + (F[i] * R + r) * d, query, d) + bias[F[i] * R + r];
                    if (v > best) best = v;
                }
                score[i] = best;
            }
            double g, sd;
            c = choose(rk, score, F, nF, mode, p, k, &g, &sd);
            if (g < *tie_gap) *tie_gap = g;
            if (sd < *tie_sum) *tie_sum = sd;
        }
        opened[l] = c;
        if (l == 1) {
            if (c > max_sel) {
                rc = -3;
                break;
            }
            for (long long i = 0; i < c; ++i) sel[i] = rk[i].id;
            qsort(sel, (size_t)c, sizeof(long long), by_id);
            chosen = c;
            break;
        }
        /* next frontier: children of the opened nodes, then level l-1 orphans */
        for (long long i = 0; i < c; ++i) next[i] = rk[i].id;
        qsort(next, (size_t)c, sizeof(long long), by_id);
        long long nn = 0;
        for (long long i = 0; i < c; ++i)
            for (int ch = 0; ch < C; ++ch) F[nn++] = next[i] * C + ch;
        for (long long j = (long long)C * n_nodes[l]; j < n_nodes[l - 1]; ++j) F[nn++] = j;
        nF = nn;
    }

    long long tail = n_nodes[0] - (long long)C * n_nodes[1];
    *n_sel = chosen;
    *keys_read = chosen * C + tail;
    *work = (long long)R * total_frontier + *keys_read;
    free(F); free(next); free(score); free(rk);
    return rc;
}

/* ---------------------------------------------------------------------------
 * Final attention over exactly the chosen keys: the chunks in sel plus the
 * tail [C*n1, n_keys).  out = sum_i softmax(beta <q,k_i>) v_i, lse = log sum exp.
 */
int orc_attend(long long n_keys, int d, double beta, const double *K, const double *V,
               const double *q, const long long *sel, long long n_sel, int C, long long n1,
               double *out, double *lse) {
    long long tail = n_keys - (long long)C * n1;
    long long n = n_sel * C + tail;
    if (n <= 0) return -1;
    long long *idx = (long long *)malloc(sizeof(long long) * (size_t)n);
    double *s = (double *)malloc(sizeof(double) * (size_t)n);
    double *w = (double *)malloc(sizeof(double) * (size_t)n);
    if (!idx || !s || !w) {
        free(idx); free(s); free(w);
        return -2;
    }
    long long m = 0;
    for (long long i = 0; i < n_sel; ++i)
        for (int c = 0; c < C; ++c) idx[m++] = sel[i] * C + c;
    for (long long i = (long long)C * n1; i < n_keys; ++i) idx[m++] = i;
    for (long long i = 0; i < n; ++i) s[i] = beta * dot(K + idx[i] * d, q, d);
    softmax(s, n, w);
    for (int t = 0; t < d; ++t) out[t] = 0.0;
    for (long long i = 0; i < n; ++i)
        for (int t = 0; t < d; ++t) out[t] += w[i] * V[idx[i] * d + t];
    *lse = log_sum_exp(s, n);
    free(idx); free(s); free(w);
    return 0;
}

/* ---------------------------------------------------------------------------
 * Full-scan indexer (the comparison): score every key, softmax over all of
 * them, then the same top-p prefix / top-K rule as a tree level, over keys.
 * sel = chosen key indices ascending.
 */
int orc_dense_scan(long long n_keys, int d, double beta, const double *K, const double *q,
                   int mode, double p, int k, long long *sel, long long max_sel,
                   long long *n_sel, double *tie_gap, double *tie_sum) {
    if (n_keys <= 0) return -1;
    double *s = (double *)malloc(sizeof(double) * (size_t)n_keys);
    long long *ids = (long long *)malloc(sizeof(long long) * (size_t)n_keys);
    ranked *rk = (ranked *)malloc(sizeof(ranked) * (size_t)n_keys);
    if (!s || !ids || !rk) {
        free(s); free(ids); free(rk);
        return -2;
    }
    for (long long i = 0; i < n_keys; ++i) {
        s[i] = beta * dot(K + i * d, q, d);
        ids[i] = i;
    }
    long long c = choose(rk, s, ids, n_keys, mode, p, k, tie_gap, tie_sum);
    int rc = 0;
    if (c > max_sel) {
        rc = -3;
    } else {
        for (long long i = 0; i < c; ++i) sel[i] = rk[i].id;
        qsort(sel, (size_t)c, sizeof(long long), by_id);
        *n_sel = c;
    }
    free(s); free(ids); free(rk);
    return rc;
}

/* Share of the dense attention of q that the chosen keys hold. */
double orc_kept_mass(long long n_keys, int d, double beta, const double *K, const double *q,
                     const long long *sel, long long n_sel, int C, long long n1) {
    double *s = (double *)malloc(sizeof(double) * (size_t)n_keys);
    double *w = (double *)malloc(sizeof(double) * (size_t)n_keys);
    if (!s || !w) {
        free(s); free(w);
        return NAN;
    }
    for (long long i = 0; i < n_keys; ++i) s[i] = beta * dot(K + i * d, q, d);
    softmax(s, n_keys, w);
    double kept = 0.0;
    for (long long i = 0; i < n_sel; ++i)
        for (int c = 0; c < C; ++c) kept += w[sel[i] * C + c];
    for (long long i = (long long)C * n1; i < n_keys; ++i) kept += w[i];
    free(s); free(w);
    return kept;
}
