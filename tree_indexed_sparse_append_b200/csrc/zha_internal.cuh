// Internal declarations shared by the CUDA translation units of libzha.
// Nothing here is part of the public ABI (include/zha.h).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/zha.h"

namespace zha {

constexpr unsigned FULL = 0xffffffffu;

// Device-side error codes recorded in the tree's status word (first one wins).
enum : int { DEV_OK = 0, DEV_CAPACITY = 1, DEV_BAD_INDEX = 2, DEV_TIMEOUT = 3 };

__device__ __forceinline__ void report(int *status, int code) {
    if (status) atomicCAS(status, DEV_OK, code);
}

// Kernels of one call chain (append, search, attend) are launched with
// programmatic stream serialization (launch_chained): each first waits until the
// grids before it have completed and their writes are visible (chain_start), so
// nothing is read early and results are the same as with plain stream order;
// each CTA lets the next grid be scheduled when its own work is done
// (chain_done), so the next launch's latency overlaps this grid's tail.
__device__ __forceinline__ void chain_start() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void chain_done() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---------------------------------------------------------------------------
// Loads. Node data is streamed once per launch: keep it out of L1.
__device__ __forceinline__ float4 ld_stream4(const float *p) {
    float4 v;
    asm("ld.global.nc.L1::no_allocate.v4.f32 {%0,%1,%2,%3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "l"(p));
    return v;
}
__device__ __forceinline__ float2 ld_stream2(const float *p) {
    float2 v;
    asm("ld.global.nc.L1::no_allocate.v2.f32 {%0,%1}, [%2];" : "=f"(v.x), "=f"(v.y) : "l"(p));
    return v;
}
__device__ __forceinline__ uint4 ld_stream_u4(const void *p) {
    uint4 v;
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// EPL consecutive floats owned by one lane.
template <int EPL>
__device__ __forceinline__ void load_f32(const float *p, float (&v)[EPL]) {
    if constexpr (EPL == 2) {
        float2 a = ld_stream2(p);
        v[0] = a.x;
        v[1] = a.y;
    } else {
#pragma unroll
        for (int i = 0; i < EPL; i += 4) {
            float4 a = ld_stream4(p + i);
            v[i] = a.x;
            v[i + 1] = a.y;
            v[i + 2] = a.z;
            v[i + 3] = a.w;
        }
    }
}

// EPL consecutive elements of T (float or bf16) as floats, through L1 (reused).
template <int EPL>
__device__ __forceinline__ void load_cached(const float *p, float (&v)[EPL]) {
#pragma unroll
    for (int i = 0; i < EPL; ++i) v[i] = __ldg(p + i);
}
template <int EPL>
__device__ __forceinline__ void load_cached(const __nv_bfloat16 *p, float (&v)[EPL]) {
    // EPL bf16 = 2*EPL bytes, loaded as 32-bit words (2 elements each)
    static_assert(EPL % 2 == 0, "bf16 lanes own an even number of columns");
    const unsigned *w = reinterpret_cast<const unsigned *>(p);
    unsigned u[EPL / 2];
    if constexpr (EPL == 8) {
        uint4 x = __ldg(reinterpret_cast<const uint4 *>(p));
        u[0] = x.x; u[1] = x.y; u[2] = x.z; u[3] = x.w;
    } else if constexpr (EPL == 4) {
        uint2 x = __ldg(reinterpret_cast<const uint2 *>(p));
        u[0] = x.x; u[1] = x.y;
    } else {
#pragma unroll
        for (int i = 0; i < EPL / 2; ++i) u[i] = __ldg(w + i);
    }
#pragma unroll
    for (int i = 0; i < EPL / 2; ++i) {
        v[2 * i] = __uint_as_float(u[i] << 16);
        v[2 * i + 1] = __uint_as_float(u[i] & 0xffff0000u);
    }
}

__device__ __forceinline__ float to_float(float x) { return x; }
__device__ __forceinline__ float to_float(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ void from_float(float x, float *p) { *p = x; }
__device__ __forceinline__ void from_float(float x, __nv_bfloat16 *p) { *p = __float2bfloat16_rn(x); }

// ---------------------------------------------------------------------------
// Warp reductions.
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) x += __shfl_xor_sync(FULL, x, o);
    return x;
}
__device__ __forceinline__ double warp_sum(double x) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) x += __shfl_xor_sync(FULL, x, o);
    return x;
}
__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) x = fmaxf(x, __shfl_xor_sync(FULL, x, o));
    return x;
}

__host__ __device__ constexpr int ilog2(int x) { return x <= 1 ? 0 : 1 + ilog2(x / 2); }

// Sums RP per-lane values across the warp so that afterwards every lane holds
// one complete sum: that of row (lane >> (5 - log2 RP)). Each halving step
// swaps half of the remaining values with the partner lane, so RP rows cost
// RP - 1 + (5 - log2 RP) shuffles instead of 5 * RP.
template <int RP, typename F = float>
__device__ __forceinline__ F transpose_reduce(F (&v)[RP], int lane) {
    constexpr int LG = ilog2(RP);
#pragma unroll
    for (int step = 0; step < LG; ++step) {
        const int off = 16 >> step;
        const int half = RP >> (step + 1);
        const bool upper = (lane & off) != 0;
#pragma unroll
        for (int i = 0; i < half; ++i) {
            F send = upper ? v[i] : v[i + half];
            F keep = upper ? v[i + half] : v[i];
            v[i] = keep + __shfl_xor_sync(FULL, send, off);
        }
    }
    F x = v[0];
#pragma unroll
    for (int off = 16 >> LG; off >= 1; off >>= 1) x += __shfl_xor_sync(FULL, x, off);
    return x;
}

// ---------------------------------------------------------------------------
// Monotone map of an fp32 score to an unsigned key (larger score, larger key).
__device__ __forceinline__ uint32_t order_key(float s) {
    uint32_t b = __float_as_uint(s);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float key_to_float(uint32_t k) {
    uint32_t b = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
    return __uint_as_float(b);
}

// Frontier masses are summed as unsigned fixed point with 40 fractional bits:
// the sums are exact and independent of the order of addition. e * 2^40 is exact
// in fp32 (a power-of-two scale), so converting it rounds that exact value.
__device__ __forceinline__ unsigned long long mass_fixed(float e) {
    return __float2ull_rn(e * 1099511627776.0f);
}

}  // namespace zha

// ---------------------------------------------------------------------------
// Host side: the tree handle.
struct zha_tree {
    zha_config cfg;
    int T;                                  // trees = batch * n_kv_heads
    int NF;                                 // floats per node
    int device;
    long long n;                            // keys per tree
    int max_depth;                          // levels with storage (cfg.depth unless the tree grows)
    int grow;                               // 1: cfg.depth follows the key count
    long long n_nodes[ZHA_MAX_DEPTH + 1];   // live nodes per tree, per level
    long long cap_nodes[ZHA_MAX_DEPTH + 1]; // node capacity per tree, per level
    float *nodes[ZHA_MAX_DEPTH + 1];        // [T][cap_nodes[l]][NF]
    void *K;
    void *V;
    const float *refs;
    int *d_status;

    // scratch (grown on demand)
    void *ws;
    size_t ws_bytes;
    long long ws_walks;
    int ws_max_sel;

    // scratch of the full-scan indexer (grown on demand)
    void *dws;
    size_t dws_bytes;

    // diagnostics
    struct zha_profiler *prof;  // NULL unless zha_profile(tree, 1)
    unsigned long long tc_wait_ns;  // limit of the tensor-core scorer's waits (0: 1 s)
    int tc_stall;                   // test hook of zha_test_wait_limit

    // context-parallel walk (zha_cp_begin / zha_cp_export / zha_cp_select)
    int cp_active, cp_level, cp_start, cp_cur, cp_G;
    long long cp_W;
    long long cp_off[ZHA_MAX_DEPTH + 1];  // global id of the shard's first node, per level
    long long last_W;
    int last_G, last_start, last_max_sel;
};

namespace zha {

// Scratch carved out of tree->ws for one search / attend of W walks.
struct Scratch {
    float *qf;                 // [W][D] queries as fp32
    float *S;                  // [W][Sstride] node scores, indexed by node id
    uint32_t *gkey;            // [W][Sstride] frontier keys too many for shared memory
    int *L[2];                 // [W][Lstride] frontier lists (ping-pong)
    int *cnt[2];               // [W] frontier counts
    unsigned *M[ZHA_MAX_DEPTH + 1];  // per level: [T][words_l][G] membership bits
    unsigned *U[ZHA_MAX_DEPTH + 1];  // per level: [T][words_l] union bits
    size_t M_bytes, U_bytes;
    unsigned *M_base, *U_base;
    int *item_off;             // [W + 1] attend items per walk (prefix)
    int *group_off;            // [W + 1] attend item groups per walk (prefix)
    int *seg;                  // [1] keys per attend item of the call
    int *item_walk;            // [max_items] walk of each attend item
    int *walk_done;            // [W] attend groups finished per walk
    int *group_done;           // [max_groups] attend items finished per group
    float *partial;            // [max_items][D + 4]
    float *gpartial;           // [max_groups][D + 4]
    unsigned char *tc;         // tensor-core scoring: A tiles (NULL when the walks per tree are few)
    unsigned char *tc_b;       //   B tiles of the level being scored
    int *tc_counts, *tc_lists; //   per B tile: how many walks, and which, have one of its nodes in their frontier
    long long Sstride, Lstride, max_items, max_groups;
};

int reserve(zha_tree *t, long long walks, int max_sel, Scratch *s);

// Packed lists of a context-parallel level step (carved from the tree's second
// scratch block): per walk P = n_parts * list stride slots.
struct CpScratch {
    int *pids;
    float *pscores;
    int *pcount;
    int *opened;
    int *ocount;
    uint32_t *stage;
    long long P;
};

// Byte offsets of the attention's scratch for W walks of head dimension D, in
// one block of `bytes` (offsets 256-byte aligned); its size depends on W and D only.
struct AttendLayout {
    size_t item_off, group_off, seg, item_walk, walk_done, group_done, partial, gpartial, bytes;
    long long max_items, max_groups;
};
AttendLayout attend_layout(long long W, int D);
// Points the attention fields of s into the block at base laid out by L.
void attend_carve(const AttendLayout &L, void *base, Scratch *s);

// Tensor-core scoring of a whole level (zha_score_tc.cu), used for trees of at
// least TC_MIN_G walks, levels of at most TC_MAX_NODES nodes, d = 128 and bf16
// queries; other calls score on the CUDA cores.
// Larger levels are scored sparsely on the tensor cores: per tile of nodes, only
// the walks whose frontier holds one of its nodes (zha_score_tc.cu).
constexpr int TC_MIN_G = 1024;
constexpr long long TC_MAX_NODES = 8192;
struct TcLayout {
    size_t a_off, b_off, counts_off, lists_off, bytes;
};
// scratch of tensor-core scoring for trees of G walks: A tiles, the B tiles of the
// widest level (maxn_b nodes), membership lists for a sparse level of maxn_sparse
// nodes (0: none)
TcLayout tc_layout(int T, long long G, long long maxn_b, long long maxn_sparse, int R);
bool tc_applicable(const zha_tree *t, int G, const void *Q, zha_dtype q_dtype, int level);
bool tc_sparse_applicable(const zha_tree *t, int G, const void *Q, zha_dtype q_dtype, int level);
cudaError_t launch_score_tc_queries(const zha_tree *t, const void *Q, int G, unsigned char *ws, cudaStream_t st);
cudaError_t launch_score_tc(const zha_tree *t, int level, int G, unsigned char *atiles, unsigned char *btiles,
                            float *S, long long Sstride, cudaStream_t st);
cudaError_t launch_score_tc_sparse(const zha_tree *t, int level, int G, const void *Q, const unsigned *M,
                                   long long words, int *counts, int *lists, float *S, long long Sstride,
                                   cudaStream_t st);
// Records an error message for zha_last_error (this host thread); returns code.
int set_error(int code, const char *msg);
// Grows the tree's second scratch block (full-scan indexer, chunk-mass profile,
// split-loss gradient) to at least `need` bytes; returns a ZHA_ status.
int grow_dense_scratch(zha_tree *t, size_t need);

// kernel launchers (return cudaError_t of the launch)
cudaError_t launch_build_level(const zha_tree *t, int level, long long j0, long long j1,
                               cudaStream_t st);
cudaError_t launch_append_kv(const zha_tree *t, const void *k_new, const void *v_new,
                             cudaStream_t st);
cudaError_t launch_search(const zha_tree *t, const Scratch &s, const void *Q, zha_dtype q_dtype,
                          int G, long long W, int mode, float p, int k, int *sel, int *sel_count,
                          int max_sel, zha_stats *stats, int start_level, cudaStream_t st);
cudaError_t launch_search_init(const zha_tree *t, const Scratch &s, const void *Q, zha_dtype q_dtype, int G,
                               long long W, zha_stats *stats, int start_level, cudaStream_t st);
cudaError_t launch_score_level(const zha_tree *t, const Scratch &s, int l, int G, cudaStream_t st);
cudaError_t launch_cp_export(const zha_tree *t, const Scratch &s, int cur, int level, bool start, long long off,
                             long long W, int *ids, float *scores, int *counts, long long stride, cudaStream_t st);
cudaError_t launch_cp_select(const zha_tree *t, const Scratch &s, int cur, int level, int G, long long W, int n_parts,
                             const int *ids, const float *scores, const int *counts, long long stride, int mode,
                             float p, int k, const CpScratch &cs, long long lo, int *sel, int *sel_count,
                             int max_sel, cudaStream_t st);
cudaError_t launch_lse_combine(int n_parts, long long W, int D, const float *outs, const float *lses, void *out,
                               zha_dtype out_dtype, float *lse, cudaStream_t st);
// Final attention on the tensor cores for trees walked by many bf16 queries
// (zha_attend_tc.cu): applicability, scratch bytes, and the launch (scratch at ws).
bool attend_tc_applicable(const zha_tree *t, int G, zha_dtype q_dtype);
size_t attend_tc_scratch(const zha_tree *t, int G, long long W);
cudaError_t launch_attend_tc(const zha_tree *t, int G, long long W, const void *Q, const int *sel,
                             const int *sel_count, int max_sel, void *out, zha_dtype out_dtype, float *lse,
                             void *ws, cudaStream_t st);
cudaError_t launch_attend(const zha_tree *t, const Scratch &s, const void *Q, zha_dtype q_dtype,
                          int G, long long W, const int *sel, const int *sel_count, int max_sel,
                          void *out, zha_dtype out_dtype, float *lse, cudaStream_t st);

// Top-p / top-K over all N candidates of each walk (scores S [W][N]), ids out.
cudaError_t launch_select_all(const zha_tree *t, const float *S, uint32_t *gkey, long long N, long long W, int G,
                              int mode, float p, int k, int *sel, int *sel_count, int max_sel, cudaStream_t st);
cudaError_t launch_dense_scan(const zha_tree *t, const void *Q, zha_dtype q_dtype, int G, long long W, int mode,
                              float p, int k, int *sel, int *sel_count, int max_sel, float *qf, float *S,
                              uint32_t *gkey, cudaStream_t st);
// Queries to fp32 (qf [W][d]) and every key's score beta*<q, k> into S [W][n]
// (at most 32 walks per tree).
cudaError_t launch_dense_scores(const zha_tree *t, const void *Q, zha_dtype q_dtype, int G, long long W, float *qf,
                                float *S, cudaStream_t st);
// Sc[w][c] = log sum_j exp(S[w][c*group + j]) over the chunk's keys (rows of N).
cudaError_t launch_chunk_lse(const zha_tree *t, const float *S, long long N, int group, long long nch, long long W,
                             float *Sc, cudaStream_t st);
// Chunk-mass profile: dense scores into S [W][N], chunk log-sum-exps into
// Sc [W][ceil(N / group)], then top-p over each walk's chunks.
cudaError_t launch_chunk_mass(const zha_tree *t, const void *Q, zha_dtype q_dtype, int G, long long W, int group,
                              float p, int *sel, int *count, int max_sel, float *qf, float *S, float *Sc,
                              uint32_t *gkey, cudaStream_t st);

int num_sms();

// Launches kernel<<<grid, block, smem, st>>>(args...) with programmatic stream
// serialization allowed (the kernel must begin with chain_start()).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_chained(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                                  Args... args) {
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Sets n ints to zero (a chained launch, where a memset would break the chain).
cudaError_t launch_clear(const zha_tree *t, int *p, long long n, cudaStream_t st);

// Every kernel launch is bracketed by probe_begin / probe_end: they count the
// launch and, when the tree is being profiled, record a CUDA event pair.
void probe_begin(const zha_tree *t, int kind, cudaStream_t st);
void probe_end(const zha_tree *t, int kind, cudaStream_t st);

struct Probe {
    const zha_tree *t;
    int kind;
    cudaStream_t st;
    Probe(const zha_tree *t_, int k, cudaStream_t s) : t(t_), kind(k), st(s) { probe_begin(t, kind, st); }
    ~Probe() { probe_end(t, kind, st); }
};

}  // namespace zha
