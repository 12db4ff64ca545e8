/*
 * zha.h: C ABI of the B200 library for Zyphra Hierarchical Attention (ZHA).
 *
 * ZHA keeps, beside an unchanged KV cache, a tree of compressed key summaries.
 * A node summarizes C consecutive nodes of the level below (C consecutive keys at
 * level 1) and holds, for each of R reference queries q_r, one tangent of the
 * region's log-sum-exp attention: a key and a bias. A query walks the tree from
 * the top, opening nodes level by level by top-p mass or top-K, and ordinary
 * attention then runs over exactly the original keys of the opened level-1
 * nodes.
 *
 * Sources (page, then section):
 *   [P1] "How does a tree of summaries search a context? How ZHA works"
 *        (learn.chabulab.com): "How is the tree built?", "What does a node
 *        summarize?", "How does top-p differ from top-K?", "Run a small tree
 *        yourself", "Common misunderstandings".
 *   [P4] "Subquadratic Attention with a Hierarchical Tree-Structured Indexer",
 *        abstract (tree of recursively compressed key summaries, traversed from
 *        the top down; sublinear routing plus final attention).
 *   [P3] "Zyphra AI Introduces ZHA, a Path to True Subquadratic Attention"
 *        (full-scan indexers score every token).
 *
 * Conventions for every call:
 *   - Pointers named K, V, Q, k_new, v_new, refs, sel, sel_count, out, lse and
 *     stats are DEVICE pointers (CUDA global memory of the current device), owned
 *     by the caller. The library never frees them.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream): arguments are checked on the host before anything is
 *     launched; results are ready when the stream reaches that point.
 *   - Every call returns ZHA_OK (0) or a negative ZHA_ERR_* code and records a
 *     message readable with zha_last_error() (per host thread). No call aborts
 *     the process, and no exception crosses this boundary.
 *   - Errors the device finds (e.g. a walk opening more chunks than max_sel)
 *     are recorded in the tree and returned by zha_sync_status().
 *   - Layouts are row-major. B = batch (sequences), H_kv = KV heads, H_q = query
 *     heads (a multiple of H_kv; query head h uses KV head h / (H_q / H_kv)),
 *     d = head dimension, n_q = queries per query head. A "walk" is one query
 *     vector of one query head; walk w = (b * H_q + h) * n_q + i, so that the
 *     walks of tree t = b * H_kv + h_kv are the contiguous ids
 *     t * G .. t * G + G - 1 with G = (H_q / H_kv) * n_q.
 */
#ifndef ZHA_H
#define ZHA_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ZHA_MAX_DEPTH 12

typedef enum {
    ZHA_OK = 0,
    ZHA_ERR_INVALID = -1,  /* bad argument: NULL pointer, shape, dtype, range */
    ZHA_ERR_CAPACITY = -2, /* append past capacity; a walk needed more than max_sel */
    ZHA_ERR_OOM = -3,      /* device allocation failed */
    ZHA_ERR_CUDA = -4,     /* a CUDA call or launch failed (message has the CUDA error) */
    ZHA_ERR_INTERNAL = -5, /* a device-side consistency check failed */
    ZHA_ERR_TIMEOUT = -6   /* reserved for bounded device-side waits */
} zha_status;

typedef enum { ZHA_F32 = 0, ZHA_BF16 = 1 } zha_dtype;
typedef enum { ZHA_TOP_P = 0, ZHA_TOP_K = 1 } zha_mode;

/* Shape and parameters of a set of trees (one per sequence and KV head). */
typedef struct {
    int batch;          /* B >= 1 */
    int n_kv_heads;     /* H_kv >= 1 */
    int d;              /* head dimension: 64, 128 or 256 */
    int R;              /* reference queries per tree, 1..16 */
    int chunk;          /* C: children per node, 2..64 */
    int depth;          /* levels built, 1..ZHA_MAX_DEPTH; or 0: grow with the keys
                           (see zha_build) */
    int top_width;      /* a walk starts at the lowest level holding at most this
                           many nodes (the deepest level if none does); >= 1.
                           [P1] "Run a small tree yourself": the demo's top level
                           has at most 64 nodes. */
    long long capacity; /* keys per tree that K and V can hold, >= 1 */
    float sharpness;    /* beta: scale of every query-key dot product, both in the
                           summaries and in the final attention (1/sqrt(d) for a
                           standard attention head) */
    zha_dtype kv_dtype; /* element type of K, V, k_new, v_new and out */
} zha_config;

/* Per-walk counters written by zha_search when `stats` is not NULL.
   [P1] "Try it" / "Run a small tree yourself": the demo counts one comparison
   per reference query per frontier node, plus one per key read. */
typedef struct {
    int start_level;                /* level the walk started at */
    int frontier[ZHA_MAX_DEPTH + 1];/* nodes scored at each level (index = level) */
    int opened[ZHA_MAX_DEPTH + 1];  /* nodes opened at each level */
    long long keys_read;            /* C * opened level-1 nodes + tail keys */
    long long work;                 /* R * sum(frontier) + keys_read */
} zha_stats;

/* Opaque handle: the level arrays of B * H_kv trees, plus scratch for searches.
   Owned by the library; freed by zha_destroy. */
typedef struct zha_tree zha_tree;

/*
 * zha_build: build every level of every tree over the first n_keys keys.
 *   [P1] "How is the tree built?" and "What does a node summarize?": node j of
 *   level l summarizes nodes C*j .. C*j+C-1 of level l-1 (keys at level 1); for
 *   each reference r, with child scores s_i = beta*<key_{i,r}, q_r> + bias_{i,r}
 *   (bias 0 for keys), the node keeps key_r = sum_i softmax(s)_i key_{i,r} and
 *   bias_r = logsumexp(s) - beta*<key_r, q_r>. Level l has floor(n_{l-1}/C)
 *   nodes; keys past the last full chunk (the tail) have no node yet.
 * K, V:  [B][H_kv][capacity][d] of cfg->kv_dtype, the caller's KV cache. The tree
 *        keeps these pointers: zha_append writes new keys and values into them,
 *        and zha_build, zha_append and zha_attend read them. Both must stay
 *        valid until zha_destroy.
 * refs:  [H_kv][R][d] fp32, the reference queries of each KV head (shared by all
 *        sequences). Kept by pointer like K and V.
 * n_keys: 0 .. capacity.
 * out:   receives the new handle (set to NULL on error).
 * Node storage is allocated here for `capacity` keys: level l holds
 * floor(capacity / C^l) nodes of R*d + round_up(R, 4) fp32 each (keys [R][d],
 * then biases [R], then padding).
 * Depth. With cfg->depth >= 1 the tree has exactly that many levels. With
 * cfg->depth == 0 its depth grows with the keys ([P4], abstract: the depth of
 * the tree of summaries grows with the context): the tree has every level that
 * holds at least one node, D = max(1, floor(log_C n)) levels, at most
 * ZHA_MAX_DEPTH and at most the levels `capacity` can fill (storage for those
 * is allocated here). An append that completes a group of C nodes at the top
 * level makes their parent and so starts level D + 1. zha_depth returns D.
 * Errors: ZHA_ERR_INVALID (NULL pointer, shape out of range, n_keys > capacity),
 * ZHA_ERR_OOM, ZHA_ERR_CUDA.
 */
int zha_build(const zha_config *cfg, void *K, void *V, const float *refs, long long n_keys,
              void *stream, zha_tree **out);

/*
 * zha_append: append one key and one value to every tree at position n (the
 * current key count), then make the nodes whose chunk this fills: the level-1
 * node if (n+1) % C == 0, its parent if that completes a group of C at level 1,
 * and so on up to `depth` (for a growing tree, up to the deepest level its
 * capacity allows, which raises the depth when a new top node is made). [P1]
 * "How is the tree built?": a node is created each time a chunk fills. The
 * result equals zha_build over the n+1 keys.
 * k_new, v_new: [B][H_kv][d] of kv_dtype (device).
 * Errors: ZHA_ERR_INVALID (NULL), ZHA_ERR_CAPACITY (n == capacity), ZHA_ERR_CUDA.
 */
int zha_append(zha_tree *tree, const void *k_new, const void *v_new, void *stream);

/*
 * zha_rebuild: summarize every level of every tree again, in place, from the
 * first n keys of the cache and the reference queries as they are now in device
 * memory. [P1] "What does a node summarize?" and "How is the tree built?" (the
 * same summaries as zha_build); [P1] "Does the model have to be retrained?": the
 * reference queries are learned, and each update of them (made in place in the
 * refs array the tree was built with) needs the summaries made again.
 * The result equals zha_build over the same keys and refs, bit for bit. The
 * node storage is reused: nothing is allocated, and the call only launches the
 * build kernels (level 1, then each level from the one below, on `stream`).
 * Errors: ZHA_ERR_INVALID (NULL tree), ZHA_ERR_CUDA.
 */
int zha_rebuild(zha_tree *tree, void *stream);

/*
 * zha_search: walk every query down its tree ([P1] "Run a small tree yourself",
 * route; "How does top-p differ from top-K?").
 *   1. The frontier starts as every node of the start level (see top_width).
 *   2. Each frontier node scores max_r (beta*<key_r, q> + bias_r) ([P1] "What
 *      does a node summarize?": a tangent per reference, take the highest).
 *   3. mass = softmax of the scores over the whole frontier of the walk.
 *   4. Top-p: open the shortest prefix of the nodes ordered by mass (descending,
 *      ties by ascending node id) whose mass sums to at least p; p >= 1 opens
 *      all. Top-K: open the K nodes first in that order (all if fewer).
 *   5. The next frontier is the children of the opened nodes plus the nodes of
 *      the level below whose parent does not exist yet (orphans); at level 1 the
 *      opened nodes are the result.
 * Q:        [B][H_q][n_q][d] of q_dtype.
 * sel:      [walks][max_sel] int32: opened level-1 node ids, ascending; entries
 *           past sel_count are unspecified.
 * sel_count:[walks] int32. Keys [C*n_1, n) (the tail) are always attended too.
 * stats:    NULL or [walks] zha_stats.
 * mode/p/k: ZHA_TOP_P with 0 < p (p >= 1 opens everything), or ZHA_TOP_K with
 *           k >= 1.
 * Scratch memory is taken from the tree (grown on first use for this many
 * walks; see zha_reserve).
 * Errors: ZHA_ERR_INVALID, ZHA_ERR_OOM, ZHA_ERR_CUDA; a walk that opens more than
 * max_sel level-1 nodes keeps the first max_sel (ascending) and makes
 * zha_sync_status return ZHA_ERR_CAPACITY.
 */
int zha_search(zha_tree *tree, const void *Q, zha_dtype q_dtype, int n_q_heads, int n_q,
               zha_mode mode, float p, int k, int *sel, int *sel_count, int max_sel,
               zha_stats *stats, void *stream);

/*
 * zha_attend: attention of every walk over exactly its chosen keys: the keys of
 * the level-1 nodes in sel plus the tail keys [C*n_1, n) ([P1] "How is the tree
 * built?" and "Common misunderstandings": the final attention runs on the
 * original keys and values). out = sum_i softmax_i(beta*<q, k_i>) v_i,
 * lse = logsumexp_i(beta*<q, k_i>), both accumulated in fp32.
 * Q:   [B][H_q][n_q][d] of q_dtype; sel/sel_count as written by zha_search.
 * out: [B][H_q][n_q][d] of out_dtype (the fp32 result, rounded to nearest even
 *      for ZHA_BF16); lse: [walks] fp32 (may be NULL).
 * A walk with no key at all (n == 0) gets out = 0 and lse = -inf.
 * Errors: ZHA_ERR_INVALID, ZHA_ERR_OOM, ZHA_ERR_CUDA; a sel id out of range makes
 * zha_sync_status return ZHA_ERR_INTERNAL (the id is skipped).
 */
int zha_attend(zha_tree *tree, const void *Q, zha_dtype q_dtype, int n_q_heads, int n_q,
               const int *sel, const int *sel_count, int max_sel, void *out, zha_dtype out_dtype,
               float *lse, void *stream);

/*
 * zha_dense_scan: the full-scan indexer the tree walk is compared with ([P3]:
 * sparse attention indexers such as DeepSeek Sparse Attention score every token).
 * Every key of the walk's tree is scored, s_j = beta*<q, k_j>, and the selection
 * rule of one tree level is applied to the keys: softmax over all n keys, then the
 * shortest prefix of the keys ordered by mass (descending, ties by ascending key
 * index) whose mass reaches p (ZHA_TOP_P; p >= 1 takes every key), or the k first
 * in that order (ZHA_TOP_K).
 * Q:         [B][H_q][n_q][d] of q_dtype; at most 32 walks per tree
 *            ((H_q / H_kv) * n_q <= 32).
 * sel:       [walks][max_sel] int32: selected key indices, ascending.
 * sel_count: [walks] int32.
 * Scratch of 8 * walks * n bytes (+ the queries in fp32) is taken from the tree.
 * Errors as zha_search; a walk selecting more than max_sel keys keeps the first
 * max_sel (ascending) and makes zha_sync_status return ZHA_ERR_CAPACITY.
 */
int zha_dense_scan(zha_tree *tree, const void *Q, zha_dtype q_dtype, int n_q_heads, int n_q,
                   zha_mode mode, float p, int k, int *sel, int *sel_count, int max_sel,
                   void *stream);

/*
 * zha_chunk_mass: how concentrated each query's dense attention is over chunks of
 * keys ([P1] "How does top-p differ from top-K?": measured at about 64K tokens,
 * 90% of the attention sits in a median of 2.3% to 15% of the 16-key chunks,
 * depending on the task; no counterpart in the tree walk itself). For every
 * walk: the softmax of beta*<q, k_j> over all n keys of its tree, summed over
 * consecutive chunks of `group` keys (the last chunk may be partial), and the
 * fewest chunks whose summed mass reaches p, taken by mass, largest first, ties
 * to the lower chunk index (p >= 1 takes every chunk).
 * Q:     [B][H_q][n_q][d] of q_dtype; at most 32 walks per tree.
 * group: keys per chunk, >= 1 (16 in the measurement quoted above).
 * sel:   [walks][max_sel] int32: the chunk indices taken, ascending.
 * count: [walks] int32: how many; count / ceil(n / group) is the walk's share.
 * Scratch of 4 * walks * n + 8 * walks * ceil(n / group) bytes (+ the queries in
 * fp32) is taken from the tree.
 * Errors as zha_dense_scan (a walk taking more than max_sel chunks keeps the
 * first max_sel and makes zha_sync_status return ZHA_ERR_CAPACITY).
 */
int zha_chunk_mass(zha_tree *tree, const void *Q, zha_dtype q_dtype, int n_q_heads, int n_q, int group, float p,
                   int *sel, int *count, int max_sel, void *stream);

/*
 * zha_ref_grad: the loss that teaches the reference queries, and its gradient
 * ([P1] "Does the model have to be retrained?": the model stays frozen and the
 * reference queries are learned by comparing how the tree splits attention with
 * how the model does, by KL distillation). At every level l the tree splits a
 * query's attention as softmax_j(max_r(beta*<key_{j,r}, q> + bias_{j,r})); the
 * teacher splits it as the dense attention mass under each node, over the
 * C^l * n_l keys the level covers. loss = mean over the walks of the sum over
 * levels of KL(teacher || tree); grad = d loss / d refs, for the refs the tree
 * was built with (after updating them in place, zha_rebuild makes the nodes again).
 * Q:    [B][H_q][n_q][d] of q_dtype; at most 32 walks per tree.
 * loss: device float[1]; grad: device float [H_kv][R][d] (both overwritten).
 * Scratch of about 4 * walks * (n + 4 * n_1) + 4 * trees * R * (d + 1) * (sum of
 * the level sizes) bytes is taken from the tree's second scratch block (the one
 * zha_dense_scan and zha_chunk_mass use), grown with cudaMalloc when too small
 * and kept for later calls.
 * Errors: ZHA_ERR_INVALID, ZHA_ERR_OOM, ZHA_ERR_CUDA.
 */
int zha_ref_grad(zha_tree *tree, const void *Q, zha_dtype q_dtype, int n_q_heads, int n_q, float *loss, float *grad,
                 void *stream);

/* ---------------------------------------------------------------------------
 * Context-parallel walk. [P4] abstract: the method aims at contexts of
 * hundreds of millions of tokens, more than one GPU holds. The keys of each
 * tree are then split across processes in runs of whole top-level nodes
 * (C^depth keys each; the last process also holds the keys past the last full
 * top node, so it has the orphans and the tail). Each process builds its shard
 * with zha_build over its keys (fixed depth): because the runs align with the
 * top nodes, the shard's level-l nodes are, bit for bit, the nodes
 * key_begin / C^l onward of the tree over all keys. The walk of zha_search
 * ([P1] "Run a small tree yourself", route; "How does top-p differ from top-K?")
 * is then taken one level at a time, with an exchange between the steps that
 * the caller makes over its process group (an all-gather, in process order):
 *   zha_cp_begin   once: queries, the start level (from the whole tree's
 *                  counts) and this shard's start frontier;
 *   zha_cp_export  per level: score this shard's frontier and write each
 *                  walk's (global node id, score) list, ids ascending;
 *   zha_cp_select  per level, after the all-gather: choose over the gathered
 *                  lists exactly as zha_search chooses over the whole frontier
 *                  (same selector, same order, so the same nodes), keep the
 *                  opened nodes this shard holds, and make its next frontier;
 *                  at level 1 write this shard's chosen chunks and end.
 * Every process makes the same sequence of calls and exchanges. The final
 * attention ([P1] "Common misunderstandings": ordinary attention over the
 * chosen original keys) is zha_attend on each shard (its chosen chunks, and on
 * the last process the tail), merged across processes by zha_lse_combine.
 */

/*
 * zha_cp_begin: start a context-parallel walk of Q on this shard.
 * key_begin: index of the shard's first key in the whole sequence, a multiple
 *   of C^depth; global_counts[0..depth] (host): keys and nodes per level of
 *   the tree over all keys (the sum of the shards' counts); n_counts = depth + 1.
 * *start_level receives the level the walk starts at (the lowest holding at
 *   most top_width nodes in the whole tree, else depth).
 * Errors: ZHA_ERR_INVALID (a growing tree, misaligned key_begin, counts below
 * this shard's), ZHA_ERR_OOM, ZHA_ERR_CUDA.
 */
int zha_cp_begin(zha_tree *tree, const void *Q, zha_dtype q_dtype, int n_q_heads, int n_q, long long key_begin,
                 const long long *global_counts, int n_counts, int *start_level, void *stream);

/*
 * zha_cp_export: score this shard's frontier at the current level and write,
 * per walk w, counts[w] pairs ids[w][i] (global node id, ascending) and
 * scores[w][i] (max over r of beta*<key_r, q> + bias_r), rows of list_stride.
 * A frontier longer than list_stride keeps its first list_stride entries and
 * makes zha_sync_status return ZHA_ERR_CAPACITY (the shard's level-1 node count
 * always suffices). *level receives the level exported.
 */
int zha_cp_export(zha_tree *tree, int *ids, float *scores, int *counts, long long list_stride, int *level,
                  void *stream);

/*
 * zha_cp_select: the choice at the current level over the whole frontier.
 * ids, scores: [n_parts][walks][list_stride], counts: [n_parts][walks] (device),
 *   the exports of every process in process order (the all-gather of
 *   zha_cp_export's outputs).
 * mode, p, k: as zha_search. At level 1, sel [walks][max_sel] and sel_count
 *   receive this shard's chosen chunks (local level-1 ids: chunk c covers the
 *   shard's keys C*c .. C*c+C-1), as zha_search writes them for a whole tree.
 * *level receives the next level to export, or 0 when the walk is complete.
 * Scratch of about 16 * walks * n_parts * list_stride bytes is taken from the
 * tree's second scratch block (grown when too small).
 */
int zha_cp_select(zha_tree *tree, int n_parts, const int *ids, const float *scores, const int *counts,
                  long long list_stride, zha_mode mode, float p, int k, int *sel, int *sel_count, int max_sel,
                  int *level, void *stream);

/*
 * zha_lse_combine: attention over the union of disjoint key sets from the
 * attentions over each: outs [n_parts][walks][d] fp32 and lses [n_parts][walks]
 * (each part's out and lse, as zha_attend returns them; lse = -inf for a part
 * without keys) give out = sum_p exp(lse_p - lse) out_p and lse = logsumexp_p
 * lse_p. out: [walks][d] of out_dtype; lse: [walks] fp32 or NULL. No tree.
 */
int zha_lse_combine(int n_parts, long long walks, int d, const float *outs, const float *lses, void *out,
                    zha_dtype out_dtype, float *lse, void *stream);

/*
 * zha_reserve: allocate the search and attend scratch for up to max_walks walks
 * and selections of up to max_sel chunks now, so that later calls with at most
 * these sizes allocate nothing (e.g. before capturing them in a CUDA graph).
 */
int zha_reserve(zha_tree *tree, long long max_walks, int max_sel);

/*
 * zha_level: device pointer to the node array of one level (1..depth) of all
 * trees, laid out [B*H_kv][level_capacity][node_floats] fp32 with node_floats =
 * R*d + round_up(R, 4) (keys [R][d], biases [R], padding); the live node count
 * per tree is written to *n_nodes and the per-tree capacity to *level_capacity.
 * The pointer stays owned by the tree. For inspection and tests.
 */
int zha_level(const zha_tree *tree, int level, const float **nodes, long long *n_nodes,
              long long *level_capacity, int *node_floats);

/* ---------------------------------------------------------------------------
 * Diagnostics (not on the hot path): kernel timing, launch counts and the size of
 * the last search's frontiers, used by the benchmark's roofline figures.
 */
typedef enum {
    ZHA_K_BUILD = 0,          /* node summaries (build and append) */
    ZHA_K_APPEND = 1,         /* key/value write of zha_append */
    ZHA_K_SEARCH_INIT = 2,    /* walk set-up */
    ZHA_K_SCORE = 3,          /* frontier scoring, one launch per level */
    ZHA_K_SELECT = 4,         /* top-p / top-K selection and expansion, one per level */
    ZHA_K_ATTEND_PLAN = 5,    /* split of each walk's keys into work items */
    ZHA_K_ATTEND_PARTIAL = 6, /* gathered attention over the chosen keys */
    ZHA_K_ATTEND_COMBINE = 7, /* log-sum-exp merge of partial results (when a separate launch) */
    ZHA_K_SCORE_TC = 8,       /* tensor-core scoring of whole levels (prefill), with its tile preparation */
    ZHA_K_KINDS = 9
} zha_kernel_kind;

typedef struct {
    long long launches; /* launches recorded */
    double ms;          /* summed device time between the CUDA events around them */
} zha_kernel_time;

/* zha_profile: enable (1) or disable (0) recording a CUDA event pair on the
 * launching stream around every kernel this tree launches. */
int zha_profile(zha_tree *tree, int enable);

/* zha_profile_read: waits for `stream`, writes the per-kind totals recorded since
 * the last read into out[ZHA_K_KINDS] and clears them. */
int zha_profile_read(zha_tree *tree, zha_kernel_time *out, void *stream);

/* Kernels launched by this library in this process, all trees together. */
long long zha_kernel_launches(void);

/*
 * zha_test_wait_limit: test hook for the bounded waits of the tensor-core scorer
 * (prefill scoring, trees of at least 1,024 bf16 walks at d = 128). Every wait
 * of those kernels on a copy or an MMA gives up after wait_ns nanoseconds
 * (0 restores the default of 1 s), records ZHA_ERR_TIMEOUT for zha_sync_status,
 * waits (again bounded) for the copies and MMAs its CTA issued, frees its tensor
 * memory and returns. With stall = 1, every later dense scoring launch of this
 * tree first waits on a barrier that nothing arrives at, before issuing any copy
 * or MMA, so that wait runs out: the results of that search are undefined and
 * zha_sync_status returns ZHA_ERR_TIMEOUT. stall = 0 turns it off. Not for
 * production use.
 */
int zha_test_wait_limit(zha_tree *tree, long long wait_ns, int stall);

/* Size of the frontiers of the last zha_search on this tree. */
typedef struct {
    int start_level;
    long long union_nodes[ZHA_MAX_DEPTH + 1]; /* sum over trees of |union of the walks' frontiers| per level */
    long long walk_nodes[ZHA_MAX_DEPTH + 1];  /* sum over walks of |frontier| per level */
} zha_search_info;

/* zha_last_search_info: waits for `stream` and counts the frontier bits the last
 * zha_search left in its scratch. Valid until the next search on this tree. */
int zha_last_search_info(zha_tree *tree, zha_search_info *out, void *stream);

/* Keys currently in every tree (n). */
long long zha_num_keys(const zha_tree *tree);

/* Levels the trees currently have (cfg->depth, or for a growing tree the
   deepest level holding a node, at least 1); -1 for a NULL handle. */
int zha_depth(const zha_tree *tree);

/* Waits for the tree's pending work on `stream`, then returns and clears the
   first device-side error recorded since the last call (ZHA_OK if none). */
int zha_sync_status(zha_tree *tree, void *stream);

/*
 * zha_attend_noalloc: zha_attend for callers that cannot let the library
 * allocate device memory (no counterpart in the paper: it only changes where
 * the attention's working memory comes from).
 *
 * zha_attend grows the tree's scratch with cudaMalloc when a call needs more
 * than it holds. Some callers cannot allow that once they run: a server that
 * gives all device memory to its own pool at start-up, or a latency-critical
 * loop that cannot take the synchronisation cudaMalloc / cudaFree may cause.
 * This call computes exactly what zha_attend computes (same arguments, same
 * kernels, same results) but takes its scratch from one static device array of
 * 32 MiB that the library holds on every GPU it is loaded on until the process
 * exits. It calls no cudaMalloc, cudaFree or other allocating routine.
 *
 * Size limit: the scratch needed is (16,384 + walks) * 1.0625 * (4 * d + 20)
 * + walks * (4 * d + 32) bytes, give or take alignment (9.5 MB at 256 walks and
 * d = 128; 32 MiB holds about 21,000 walks at d = 128, 40,000 at d = 64 and
 * 8,000 at d = 256); a call needing more than 32 MiB fails with
 * ZHA_ERR_CAPACITY and a message giving both sizes, launching nothing.
 * Every call looks the array's device address up (cudaGetSymbolAddress, with
 * the tree's device current), so the address stays right after a context reset;
 * the first call on a device may load the library's module, so make it before
 * any stream capture.
 * Sharing: every call on a device uses the same array, and each call overwrites
 * what the last one left there. Calls that can overlap on the GPU (different
 * streams, different trees, or different host threads without ordering) race on
 * it and give wrong results: order them on one stream, or use zha_attend.
 * Profiling (zha_profile) does not time this call; zha_kernel_launches counts it.
 * Errors: as zha_attend, plus ZHA_ERR_CAPACITY (scratch limit above) and
 * ZHA_ERR_INVALID when the current device is not the tree's.
 */
int zha_attend_noalloc(zha_tree *tree, const void *Q, zha_dtype q_dtype, int n_q_heads, int n_q,
                       const int *sel, const int *sel_count, int max_sel, void *out,
                       zha_dtype out_dtype, float *lse, void *stream);

/* Frees the tree's node storage and scratch. NULL is a no-op. Pending work that
   uses the tree must have finished. */
void zha_destroy(zha_tree *tree);

/* Message of the last failed call on this host thread ("" if none). */
const char *zha_last_error(void);

/* Library version string. */
const char *zha_version(void);

#ifdef __cplusplus
}
#endif
#endif /* ZHA_H */
