// Top-down walk of every query through its tree.
//
// Page "How does a tree of summaries search a context? How ZHA works":
//   - section "What does a node summarize?": a node's score for a query q is
//     max over references r of (beta * <key_r, q> + bias_r);
//   - section "Run a small tree yourself" (route in tree.ts): the scores of the
//     whole frontier of a walk go through one softmax; top-p opens the shortest
//     prefix of the mass-ordered frontier holding at least p; the children of
//     the opened nodes form the next frontier; opened level-1 nodes name the
//     keys to read;
//   - section "How does top-p differ from top-K?": top-K opens exactly K nodes.
// Readings where the pages are silent: ties in mass go to the lower node id;
// p >= 1 opens every node; nodes whose parent does not exist yet (orphans) join
// their level's frontier; the walk starts at the lowest level with at most
// top_width nodes.
//
// Design (one launch pair per level, no grid-wide synchronisation):
//   score_level  Tree-major and load-balanced: a grid-stride loop over
//                (tree, 4-node group) items of the union of the frontiers of the
//                tree's walks (the GQA heads and queries that share the tree).
//                Each node (R*d fp32 keys + R biases, 4 KB at R=8, d=128) is
//                streamed from HBM once with 128-bit L1-bypassing loads and
//                scored against every walk whose frontier holds it (a ballot over
//                per-walk membership bits; for trees of at most 4 walks their
//                queries are loaded with the node). Dot products reduce with a
//                warp transpose-reduce (R rows in R-1+5-log2 R shuffles).
//   select_level One CTA per walk. Exact selection without sorting: histogram
//                passes over 256 buckets (1/8-nat buckets below the frontier's
//                maximum, then 1/2048-nat buckets inside the crossing one, then
//                the raw score bytes), each bucket carrying its count and its
//                softmax mass in 40-bit fixed point (integer sums: exact and
//                order-independent); a crossing bucket of at most 32 keys is
//                ranked directly by one warp. Ties at the boundary score open
//                in ascending node id. Opened nodes are
//                compacted in id order by block scans; their children and the
//                orphans of the level below form the next frontier (membership
//                bits per walk and a per-tree union).
//   select_warp_kernel  Levels whose frontiers hold at most 64 nodes (start
//                levels of 64 nodes or fewer), or at most 512 in calls of many
//                walks: one warp per walk, keys in registers, a bitonic sort
//                across the warp, the same cutoff rule and the same fixed-point
//                masses, so it opens the same nodes.
#include <algorithm>
#include <cmath>

#include "zha_internal.cuh"

namespace zha {
namespace {


// ---------------------------------------------------------------------------
// block-wide helpers
template <typename V>
__device__ __forceinline__ V warp_incl_scan(V x, int lane) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        V y = __shfl_up_sync(FULL, x, o);
        if (lane >= o) x += y;
    }
    return x;
}

// inclusive scan across a block of NT threads; `sh` holds NT / 32 values
template <int NT, typename V>
__device__ __forceinline__ V block_incl_scan(V x, V *sh, V *total) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    V inc = warp_incl_scan(x, lane);
    if (lane == 31) sh[w] = inc;
    __syncthreads();
    if (w == 0) {
        V s = lane < NT / 32 ? sh[lane] : V(0);
        s = warp_incl_scan(s, lane);
        if (lane < NT / 32) sh[lane] = s;
    }
    __syncthreads();
    V base = w > 0 ? sh[w - 1] : V(0);
    if (total) *total = sh[NT / 32 - 1];
    __syncthreads();
    return base + inc;
}

// Inclusive scans of a 64-bit and a 32-bit value across a block of NT threads in
// one pass (one set of barriers; the two shuffle chains overlap). `shm` and `shc`
// hold NT / 32 values each; `total_m` gets the block's sum of m.
template <int NT>
__device__ __forceinline__ void block_incl_scan_mc(unsigned long long &m, unsigned &c, unsigned long long *shm,
                                                   unsigned *shc, unsigned long long *total_m) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned long long ym = __shfl_up_sync(FULL, m, o);
        const unsigned yc = __shfl_up_sync(FULL, c, o);
        if (lane >= o) {
            m += ym;
            c += yc;
        }
    }
    if (lane == 31) {
        shm[w] = m;
        shc[w] = c;
    }
    __syncthreads();
    if (w == 0) {
        unsigned long long x = lane < NT / 32 ? shm[lane] : 0ull;
        unsigned y = lane < NT / 32 ? shc[lane] : 0u;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const unsigned long long yx = __shfl_up_sync(FULL, x, o);
            const unsigned yy = __shfl_up_sync(FULL, y, o);
            if (lane >= o) {
                x += yx;
                y += yy;
            }
        }
        if (lane < NT / 32) {
            shm[lane] = x;
            shc[lane] = y;
        }
    }
    __syncthreads();
    if (w > 0) {
        m += shm[w - 1];
        c += shc[w - 1];
    }
    *total_m = shm[NT / 32 - 1];
    __syncthreads();
}

template <int EPL>
__device__ __forceinline__ void load_q(const float *p, float (&v)[EPL]) {
    if constexpr (EPL == 2) {
        float2 a = __ldg(reinterpret_cast<const float2 *>(p));
        v[0] = a.x;
        v[1] = a.y;
    } else {
#pragma unroll
        for (int i = 0; i < EPL; i += 4) {
            float4 a = __ldg(reinterpret_cast<const float4 *>(p + i));
            v[i] = a.x;
            v[i + 1] = a.y;
            v[i + 2] = a.z;
            v[i + 3] = a.w;
        }
    }
}

// OR without a returned value: a reduction the issuing thread does not wait for
// (many walks set bits in the same union words, so these are contended).
__device__ __forceinline__ void red_or(unsigned *p, unsigned v) {
    asm volatile("red.relaxed.gpu.global.or.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Sets bits [lo, hi) of one walk's membership row and of its tree's union.
// Trees of more than 8 walks (prefill) read the union word first: every walk of
// the tree sets bits in the same words, and skipping the ones already set keeps
// those reductions from queueing at a few L2 slices (bits are only ever set
// during a search, so a stale read costs at most a redundant reduction). With
// few walks the read would only add its latency.
__device__ __forceinline__ void set_bits(unsigned *M_tree, unsigned *U_tree, int G, int g, long long lo,
                                         long long hi) {
    for (long long w = lo >> 5; w <= (hi - 1) >> 5; ++w) {
        const long long b0 = lo > (w << 5) ? lo : (w << 5);
        const long long b1 = hi < ((w + 1) << 5) ? hi : ((w + 1) << 5);
        const int n = (int)(b1 - b0);
        const unsigned mask = (n == 32 ? FULL : ((1u << n) - 1u)) << (int)(b0 - (w << 5));
        red_or(&M_tree[w * G + g], mask);
        if (G <= 8 || (__ldcg(&U_tree[w]) & mask) != mask) red_or(&U_tree[w], mask);
    }
}

// ---------------------------------------------------------------------------
struct InitArgs {
    const void *Q;
    int q_bf16, D;
    long long W;
    float *qf;
    int *n_par;           // frontier descriptor: parents opened (unused at the start level)
    unsigned *M, *U;      // start level
    long long words;
    int G;
    long long n_s;
    zha_stats *stats;
    int start_level;
    // membership and union words of every level, cleared here except the start
    // level's (written below)
    unsigned *M_all, *U_all;
    long long M_all_words, U_all_words;
};

__global__ void search_init_kernel(InitArgs a) {
    chain_start();
    {
        const long long i0 = (long long)blockIdx.x * blockDim.x + threadIdx.x;
        const long long stride = (long long)gridDim.x * blockDim.x;
        const unsigned *Ms = a.M, *Us = a.U;
        const long long Mn = a.words * a.G * (a.W / a.G), Un = a.words * (a.W / a.G);
        for (long long i = i0; i < a.M_all_words; i += stride) {
            unsigned *p = a.M_all + i;
            if (p < Ms || p >= Ms + Mn) *p = 0u;
        }
        for (long long i = i0; i < a.U_all_words; i += stride) {
            unsigned *p = a.U_all + i;
            if (p < Us || p >= Us + Un) *p = 0u;
        }
    }
    const long long walk = blockIdx.x;
    const int t = (int)(walk / a.G), g = (int)(walk % a.G);
    for (int e = threadIdx.x; e < a.D; e += blockDim.x) {
        const long long i = walk * a.D + e;
        a.qf[i] = a.q_bf16 ? __bfloat162float(static_cast<const __nv_bfloat16 *>(a.Q)[i])
                           : static_cast<const float *>(a.Q)[i];
    }
    for (long long w = threadIdx.x; w < a.words; w += blockDim.x) {
        const long long b0 = w << 5;
        const long long n = a.n_s - b0;
        const unsigned mask = n >= 32 ? FULL : (n <= 0 ? 0u : ((1u << n) - 1u));
        a.M[((long long)t * a.words + w) * a.G + g] = mask;
        if (g == 0) a.U[(long long)t * a.words + w] = mask;
    }
    if (threadIdx.x == 0) {
        a.n_par[walk] = 0;
        if (a.stats) {
            zha_stats *s = a.stats + walk;
            s->start_level = a.start_level;
            for (int l = 0; l <= ZHA_MAX_DEPTH; ++l) s->frontier[l] = s->opened[l] = 0;
            s->keys_read = 0;
            s->work = 0;
        }
    }
    chain_done();
}

// ---------------------------------------------------------------------------
struct ScoreArgs {
    const float *nodes;
    long long node_tree;  // floats per tree in the level array
    int NF, R, G, T;
    float beta;
    const unsigned *U, *M;
    long long words, n_level;
    const float *qf;
    float *S;
    long long Sstride;
    int npi;  // node ids per work item: 4, or 1 for small levels
};

template <int D, int RP>
__device__ __forceinline__ void load_node(const float *node, int R, int lane, float (&kr)[RP][D / 32]) {
    constexpr int EPL = D / 32;
#pragma unroll
    for (int r = 0; r < RP; ++r) {
        if (r < R) {
            load_f32<EPL>(node + r * D + lane * EPL, kr[r]);
        } else {
#pragma unroll
            for (int e = 0; e < EPL; ++e) kr[r][e] = 0.f;
        }
    }
}

// Scores one node (rows in kr) against every walk of tree t whose frontier
// holds node j.
template <int D, int RP>
__device__ __forceinline__ void score_node(const ScoreArgs &a, int t, long long j, const float (&kr)[RP][D / 32],
                                           float bias, int lane) {
    constexpr int EPL = D / 32;
    constexpr int LG = ilog2(RP);
    const int rr = lane >> (5 - LG);  // row whose full dot product this lane ends with
    const unsigned *Mrow = a.M + ((long long)t * a.words + (j >> 5)) * a.G;
    const int bit = (int)(j & 31);
    for (int g0 = 0; g0 < a.G; g0 += 32) {
        const unsigned mw = (g0 + lane < a.G) ? __ldg(Mrow + g0 + lane) : 0u;
        unsigned members = __ballot_sync(FULL, (mw >> bit) & 1u);
        while (members) {
            const int gl = __ffs(members) - 1;
            members &= members - 1;
            const long long walk = (long long)t * a.G + g0 + gl;
            float q[EPL];
            load_q<EPL>(a.qf + walk * D + lane * EPL, q);
            float part[RP];
#pragma unroll
            for (int r = 0; r < RP; ++r) {
                float s = 0.f;
#pragma unroll
                for (int e = 0; e < EPL; ++e) s = fmaf(kr[r][e], q[e], s);
                part[r] = s;
            }
            const float dot = transpose_reduce<RP>(part, lane);
            float sc = rr < a.R ? fmaf(a.beta, dot, bias) : -INFINITY;
#pragma unroll
            for (int off = 16; off >= (32 >> LG) && LG > 0; off >>= 1) sc = fmaxf(sc, __shfl_xor_sync(FULL, sc, off));
            if (lane == 0) a.S[walk * a.Sstride + j] = sc;
        }
    }
}

// Scores one node (rows in kr) against the walks of tree t whose frontier holds
// node j, for trees of at most GQ walks whose queries (q[g], this lane's columns)
// were loaded together with the node: no query load waits on the membership.
template <int D, int RP, int GQ>
__device__ __forceinline__ void score_node_q(const ScoreArgs &a, int t, long long j, const float (&kr)[RP][D / 32],
                                             const float (&q)[GQ][D / 32], float bias, int lane, unsigned mw) {
    constexpr int EPL = D / 32;
    constexpr int LG = ilog2(RP);
    const int rr = lane >> (5 - LG);
    const unsigned members = __ballot_sync(FULL, (mw >> (j & 31)) & 1u);
#pragma unroll
    for (int g = 0; g < GQ; ++g) {
        if (!((members >> g) & 1u)) continue;
        float part[RP];
#pragma unroll
        for (int r = 0; r < RP; ++r) {
            float s = 0.f;
#pragma unroll
            for (int e = 0; e < EPL; ++e) s = fmaf(kr[r][e], q[g][e], s);
            part[r] = s;
        }
        const float dot = transpose_reduce<RP>(part, lane);
        float sc = rr < a.R ? fmaf(a.beta, dot, bias) : -INFINITY;
#pragma unroll
        for (int off = 16; off >= (32 >> LG) && LG > 0; off >>= 1) sc = fmaxf(sc, __shfl_xor_sync(FULL, sc, off));
        if (lane == 0) a.S[((long long)t * a.G + g) * a.Sstride + j] = sc;
    }
}

// Grid-stride over (tree, group of npi node ids) items of the level's union
// bitmap (npi = 4, or 1 for levels too small to give every warp several items).
// Each lane fetches the union bits of one of the warp's next 32 items in a single
// load, so walking the items costs no memory round trip of its own; every set
// node is then loaded (R rows of 16-byte lanes) and scored.
template <int D, int RP>
__global__ void __launch_bounds__(256, 3) score_level_kernel(ScoreArgs a) {
    chain_start();
    constexpr int LG = ilog2(RP);
    const int lane = threadIdx.x & 31;
    const int rr = lane >> (5 - LG);
    const long long gw = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const long long nw = ((long long)gridDim.x * blockDim.x) >> 5;
    const int npi = a.npi;
    const unsigned nmask = (1u << npi) - 1u;
    const long long groups = (a.n_level + npi - 1) / npi;
    const long long items = groups * a.T;

    for (long long base = gw; base < items; base += 32 * nw) {
        const long long mine = base + (long long)lane * nw;
        unsigned my_bits = 0;
        if (mine < items) {
            const int t = (int)(mine / groups);
            const long long j0 = (mine - (long long)t * groups) * npi;
            my_bits = (__ldg(a.U + (long long)t * a.words + (j0 >> 5)) >> (j0 & 31)) & nmask;
        }
        unsigned any = __ballot_sync(FULL, my_bits != 0);
        while (any) {
            const int li = __ffs(any) - 1;
            any &= any - 1;
            unsigned bits = __shfl_sync(FULL, my_bits, li);
            const long long it = base + (long long)li * nw;
            const int t = (int)(it / groups);
            const long long j0 = (it - (long long)t * groups) * npi;
            const float *tree_nodes = a.nodes + (long long)t * a.node_tree;
            while (bits) {
                const long long j = j0 + __ffs(bits) - 1;
                bits &= bits - 1;
                const float *node = tree_nodes + j * a.NF;
                float kr[RP][D / 32];
                load_node<D, RP>(node, a.R, lane, kr);
                const float bias = rr < a.R ? __ldg(node + a.R * D + rr) : 0.f;
                if (a.G <= 4) {
                    // the tree's queries and membership words, issued with the node
                    constexpr int EPL = D / 32;
                    float q[4][EPL];
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        if (g < a.G) {
                            load_q<EPL>(a.qf + ((long long)t * a.G + g) * D + lane * EPL, q[g]);
                        } else {
#pragma unroll
                            for (int e = 0; e < EPL; ++e) q[g][e] = 0.f;
                        }
                    }
                    const unsigned mw =
                        lane < a.G ? __ldg(a.M + ((long long)t * a.words + (j >> 5)) * a.G + lane) : 0u;
                    score_node_q<D, RP, 4>(a, t, j, kr, q, bias, lane, mw);
                } else {
                    score_node<D, RP>(a, t, j, kr, bias, lane);
                }
            }
        }
    }
    chain_done();
}

// ---------------------------------------------------------------------------
struct SelectArgs {
    int level, C, R, G;
    int c_shift;             // log2(C) when C is a power of two, else -1
    int start;               // 1 when this level is the start level (frontier = all nodes)
    long long n_level;       // nodes at this level
    long long n_orph;        // orphans at this level (nodes past C * n_{level+1}); 0 at start
    long long n_orph_next;   // orphans at level - 1
    long long n_level_next;  // nodes at level - 1 (for orphan ids)
    const float *S;
    long long Sstride;
    const int *par_in;       // opened parents (level + 1), ascending
    int *par_out;            // opened nodes of this level (when level > 1)
    long long Lstride;
    const int *n_par_in;
    int *n_par_out;
    unsigned *M_next, *U_next;
    long long words_next;
    int mode;
    float p;
    int k;
    int *sel;
    int max_sel;
    int *sel_count;
    zha_stats *stats;
    long long tail;
    int *status;
    long long smem_keys;     // frontiers up to this size are staged in shared memory
    uint32_t *gkey;          // [W][Sstride] staging for larger frontiers
    // explicit frontiers (the context-parallel walk): per walk, list_count[w]
    // (node id, score) pairs at list_ids / list_scores + w * list_stride, ids
    // ascending; S, par_in and the orphan counts are then unused
    const int *list_ids;
    const float *list_scores;
    const int *list_count;
    long long list_stride;
    long long n_walks;       // walks of the call (select_warp_kernel)
};

// frontier position -> node id (positions and ids fit in 32 bits); lid: the
// walk's explicit list, if any
__device__ __forceinline__ long long frontier_id(const SelectArgs &a, const int *lid, const int *par, long long npar,
                                                 long long i) {
    if (lid) return lid[i];
    if (a.start) return i;
    const int ii = (int)i, C = a.C;
    const int kids = (int)npar * C;
    if (ii < kids) {
        const int pi = a.c_shift >= 0 ? ii >> a.c_shift : ii / C;
        return (long long)par[pi] * C + (ii - pi * C);
    }
    return (a.n_level - a.n_orph) + (ii - kids);
}

template <int NT>
__device__ __forceinline__ uint32_t block_max_u32(uint32_t x, unsigned *sh) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) x = max(x, __shfl_xor_sync(FULL, x, o));
    if (lane == 0) sh[w] = x;
    __syncthreads();
    uint32_t r = sh[0];
#pragma unroll
    for (int i = 1; i < NT / 32; ++i) r = max(r, sh[i]);
    __syncthreads();
    return r;
}

// Each walk's frontier keys are staged once, in shared memory when they fit
// (smem_keys), else in the walk's row of a global key array. The cutoff is found
// with at most three kinds of histogram pass, each over 256 buckets that keep
// count and fixed-point mass (HCOPIES copies, shared by groups of warps):
//   1. coarse: 1/8 nat per bucket below the frontier's highest score (keys
//      spread over many buckets, so the atomics rarely collide; this pass also
//      yields the total mass);
//   2. fine: 1/2048 nat inside the crossing coarse bucket;
//   3. radix on the raw score bits inside the crossing fine bucket, a byte at a
//      time.
// Bucket orders agree with the score order, so the crossing bucket of each pass
// holds the cutoff. As soon as it holds at most CAND_MAX keys, they are listed
// and one warp ranks them directly (mass strictly above each, mass of its equal
// keys), which ends the search.
constexpr int HCOPIES = 8;
constexpr float COARSE_PER_NAT = 8.f;
constexpr int CAND_MAX = 32;  // a crossing bucket this small is resolved by one warp

// Adds a fixed-point mass to a bucket kept as two 32-bit words, with native 32-bit
// shared atomics: the low word takes the low 32 bits, and the add that wraps it
// (old + l < old, seen in the value the atomic returns) carries one into the high
// word, so high * 2^32 + low is the exact sum. The high word stays below 2^32 for
// fewer than 2^24 keys (masses are at most 2^40).
__device__ __forceinline__ void add_mass(unsigned *lo, unsigned *hi, unsigned long long v) {
    const unsigned l = (unsigned)v;
    unsigned h = (unsigned)(v >> 32);
    if (l) {
        const unsigned old = atomicAdd(lo, l);
        h += old + l < old ? 1u : 0u;
    }
    if (h) atomicAdd(hi, h);
}

__device__ __forceinline__ int coarse_bucket(float s, float m) {
    const float x = (m - s) * COARSE_PER_NAT;
    return x >= 255.f ? 255 : (x > 0.f ? (int)x : 0);
}
__device__ __forceinline__ int fine_bucket(float s, float m, int cb) {
    const float y = ((m - s) * COARSE_PER_NAT - (float)cb) * 256.f;
    return y >= 255.f ? 255 : (y > 0.f ? (int)y : 0);
}

// KB: keys loaded together per thread in the passes over the frontier: 8 for the
// full scan, whose frontier (every key of the tree) is staged in global memory,
// so that a pass does not wait one round trip per position; 1 for the tree
// walk, whose frontiers sit in shared memory, which keeps the registers for the
// rest (batched loads made those selections slower).
template <int NT, int KB>
__global__ void __launch_bounds__(NT) select_level_kernel(SelectArgs a) {
    chain_start();
    extern __shared__ uint32_t skey_s[];
    // bucket masses as two 32-bit words (low word, then high word plus carries)
    __shared__ unsigned h_mlo[HCOPIES][256], h_mhi[HCOPIES][256];
    __shared__ unsigned h_cnt[HCOPIES][256];
    __shared__ unsigned long long sh_u64[NT / 32];
    __shared__ unsigned sh_u32[NT / 32];
    __shared__ uint32_t s_cand[CAND_MAX];
    __shared__ unsigned long long s_candm[CAND_MAX];
    __shared__ int s_bucket;
    __shared__ uint32_t s_key;
    __shared__ unsigned long long s_trem;
    __shared__ unsigned s_krem, s_count, s_ncand;

    const long long walk = blockIdx.x;
    const int tid = threadIdx.x;
    const int t = (int)(walk / a.G), g = (int)(walk % a.G);
    const int *lid = a.list_ids ? a.list_ids + walk * a.list_stride : nullptr;
    const float *lsc = a.list_scores ? a.list_scores + walk * a.list_stride : nullptr;
    const long long npar = a.start || lid ? 0 : a.n_par_in[walk];
    const int *par = lid ? nullptr : a.par_in + walk * a.Lstride;
    const long long F = lid ? a.list_count[walk] : (a.start ? a.n_level : npar * a.C + a.n_orph);
    const float *S = a.S + walk * a.Sstride;
    uint32_t *skey = F <= a.smem_keys ? skey_s : a.gkey + walk * a.Sstride;
    auto key_at = [&](long long i) -> uint32_t { return skey[i]; };

    // stage the frontier's keys (coalesced, strided) and find the largest
    // (batches of 8 strided positions, the last one predicated, so a thread's
    // parent and score loads are all in flight together)
    uint32_t kmax = 0;
    for (long long i = tid; i < F; i += 8 * NT) {
        long long id[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) id[u] = i + u * NT < F ? frontier_id(a, lid, par, npar, i + u * NT) : -1;
        float v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) v[u] = id[u] >= 0 ? (lsc ? lsc[i + u * NT] : S[id[u]]) : 0.f;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            if (id[u] >= 0) {
                const uint32_t k = order_key(v[u]);
                skey[i + u * NT] = k;
                kmax = max(kmax, k);
            }
        }
    }
    kmax = block_max_u32<NT>(kmax, sh_u32);
    const float m = key_to_float(kmax);
    auto mass = [&](float s) { return mass_fixed(expf(s - m)); };

    const bool open_all = (a.mode == ZHA_TOP_P && a.p >= 1.f) || (a.mode == ZHA_TOP_K && (long long)a.k >= F);
    const bool top_p = a.mode == ZHA_TOP_P;
    uint32_t kstar = 0;
    unsigned long long cstar = 0;
    unsigned eq_count = 0;  // keys equal to kstar
    if (F > 0 && !open_all) {
        unsigned long long trem = 0;
        unsigned krem = (unsigned)a.k;
        const int wcopy = (tid >> 5) & (HCOPIES - 1);
        // stage 0: coarse, 1: fine, 2..5: raw bytes 24, 16, 8, 0
        int cb = -1, fb = -1;
        uint32_t prefix = 0, pmask = 0;
        // keys still in play after `narrowed` stages: the crossing buckets so far
        auto in_play = [&](uint32_t k, int narrowed) -> bool {
            if (narrowed == 0) return true;
            const float s = key_to_float(k);
            if (coarse_bucket(s, m) != cb) return false;
            if (narrowed == 1) return true;
            return fine_bucket(s, m, cb) == fb && (k & pmask) == prefix;
        };
        bool done = false;
        for (int stage = 0; stage < 6 && !done; ++stage) {
            for (int j = tid; j < HCOPIES * 256; j += NT) {
                (&h_mlo[0][0])[j] = 0;
                (&h_mhi[0][0])[j] = 0;
                (&h_cnt[0][0])[j] = 0;
            }
            if (tid == 0) s_ncand = 0;
            __syncthreads();
            const int shift = 24 - 8 * (stage - 2);
            // keys in batches of KB strided positions, loaded before any is used
            for (long long i0 = tid; i0 < F; i0 += KB * NT) {
              uint32_t kk[KB];
#pragma unroll
              for (int u = 0; u < KB; ++u) kk[u] = i0 + u * NT < F ? key_at(i0 + u * NT) : 0u;
#pragma unroll
              for (int u = 0; u < KB; ++u) {
                if (i0 + u * NT >= F) break;
                const uint32_t k = kk[u];
                if (!in_play(k, stage)) continue;
                const float s = key_to_float(k);
                const int b = stage == 0 ? coarse_bucket(s, m)
                                         : (stage == 1 ? fine_bucket(s, m, cb) : (int)((k >> shift) & 255));
                atomicAdd(&h_cnt[wcopy][b], 1u);
                if (top_p) add_mass(&h_mlo[wcopy][b], &h_mhi[wcopy][b], mass(s));
              }
            }
            __syncthreads();
            // threads 0..255 own one bucket each: buckets ascend from the highest
            // scores (stages 0, 1) or descend (raw bytes), so raw stages read them
            // in reverse; threads past 255 add nothing to the scans
            const bool own = tid < 256;
            const int b = own ? (stage >= 2 ? 255 - tid : tid) : 0;
            unsigned long long vm = 0;
            unsigned vc = 0;
            if (own) {
#pragma unroll
                for (int c = 0; c < HCOPIES; ++c) {
                    vm += ((unsigned long long)h_mhi[c][b] << 32) + h_mlo[c][b];
                    vc += h_cnt[c][b];
                }
            }
            unsigned long long total_m;
            unsigned long long incl_m = vm;
            unsigned incl_c = vc;
            block_incl_scan_mc<NT>(incl_m, incl_c, sh_u64, sh_u32, &total_m);
            if (stage == 0 && top_p) {
                trem = (unsigned long long)ceil((double)a.p * (double)total_m);
                if (trem < 1) trem = 1;
                if (trem > total_m) trem = total_m;
            }
            const bool hit = own && (top_p ? (incl_m - vm < trem && trem <= incl_m)
                                           : (incl_c - vc < krem && krem <= incl_c));
            if (hit) {
                s_bucket = b;
                s_trem = trem - (incl_m - vm);
                s_krem = krem - (incl_c - vc);
                s_count = vc;
            }
            __syncthreads();
            const int hb = s_bucket;
            trem = s_trem;
            krem = s_krem;
            const unsigned cnt = s_count;
            if (stage == 0) {
                cb = hb;
            } else if (stage == 1) {
                fb = hb;
            } else {
                prefix |= (uint32_t)hb << shift;
                pmask |= 255u << shift;
            }
            if (cnt <= CAND_MAX) {
                // few keys left: list them and let one warp rank them directly
                for (long long i0 = tid; i0 < F; i0 += KB * NT) {
                    uint32_t kk[KB];
#pragma unroll
                    for (int u = 0; u < KB; ++u) kk[u] = i0 + u * NT < F ? key_at(i0 + u * NT) : 0u;
#pragma unroll
                    for (int u = 0; u < KB; ++u) {
                        if (i0 + u * NT < F && in_play(kk[u], stage + 1)) {
                            const unsigned slot = atomicAdd(&s_ncand, 1u);
                            if (slot < CAND_MAX) s_cand[slot] = kk[u];
                        }
                    }
                }
                __syncthreads();
                if (tid < 32) {
                    const int lane = tid;
                    const int n = min(s_ncand, (unsigned)CAND_MAX);
                    const bool v = lane < n;
                    const uint32_t kj = v ? s_cand[lane] : 0u;
                    const unsigned long long uj = v ? (top_p ? mass(key_to_float(kj)) : 1ull) : 0ull;
                    s_candm[lane] = uj;
                    __syncwarp();
                    // every lane reads every candidate (broadcast loads, independent
                    // of one another, so they overlap)
                    unsigned long long above = 0, same = 0;
                    unsigned same_n = 0;
#pragma unroll 8
                    for (int i = 0; i < n; ++i) {
                        const uint32_t ki = s_cand[i];
                        const unsigned long long ui = s_candm[i];
                        if (ki > kj) above += ui;
                        else if (ki == kj) {
                            same += ui;
                            ++same_n;
                        }
                    }
                    const unsigned long long target = top_p ? trem : (unsigned long long)krem;
                    unsigned bal = __ballot_sync(FULL, v && above < target && target <= above + same);
                    if (!bal) {  // cannot happen while the sums agree; then open the whole bucket
                        uint32_t kmin = v ? kj : 0xffffffffu;
#pragma unroll
                        for (int o = 16; o >= 1; o >>= 1) kmin = min(kmin, __shfl_xor_sync(FULL, kmin, o));
                        bal = __ballot_sync(FULL, v && kj == kmin);
                    }
                    const int src = bal ? __ffs(bal) - 1 : 0;
                    if (lane == src) {
                        s_key = kj;
                        s_trem = trem - above;
                        s_krem = krem - (unsigned)above;
                        s_count = same_n;
                    }
                }
                __syncthreads();
                kstar = s_key;
                trem = s_trem;
                krem = s_krem;
                eq_count = s_count;
                done = true;
            } else if (stage == 5) {
                kstar = prefix;  // every key left equals prefix
                eq_count = cnt;
                done = true;
            }
            __syncthreads();
        }
        if (top_p) {
            const unsigned long long u = mass(key_to_float(kstar));
            cstar = u > 0 ? (trem + u - 1) / u : 1;
        } else {
            cstar = krem;
        }
    }

    // opened = key above kstar, or equal to it and among the first cstar (by id).
    // Each warp owns a contiguous region of positions and reads it 32 at a time
    // (coalesced); ballots give the ranks inside a group of 32, one block scan
    // over the warps' counts the rest, so ranks follow ids.
    constexpr int NW = NT / 32;
    const int lane = tid & 31, wid = tid >> 5;
    const long long region = ((F + NW - 1) / NW + 31) & ~31LL;
    const long long rbeg = min(F, (long long)wid * region), rend = min(F, rbeg + region);
    const unsigned below = (1u << lane) - 1u;
    // ranks among keys equal to kstar matter only when some of them stay closed
    const bool split_tie = !open_all && cstar < eq_count;
    unsigned eq_base = 0;
    if (split_tie) {
        unsigned eq_w = 0;
        for (long long i0 = rbeg; i0 < rend; i0 += 32) {
            const long long i = i0 + lane;
            eq_w += __popc(__ballot_sync(FULL, i < rend && key_at(i) == kstar));
        }
        const unsigned v = lane == 0 ? eq_w : 0u;
        eq_base = block_incl_scan<NT, unsigned>(v, sh_u32, nullptr) - v;
        eq_base = __shfl_sync(FULL, eq_base, 0);
    }
    // is position i opened? `eq` is the number of keys equal to kstar before this group
    // (key: the key at i, loaded by the caller)
    auto opened = [&](long long i, uint32_t key, unsigned eq, unsigned &eq_in_group) -> bool {
        const bool in = i < rend;
        if (open_all) {
            eq_in_group = 0;
            return in;
        }
        const bool is_eq = in && key == kstar;
        const unsigned eqm = __ballot_sync(FULL, is_eq);
        eq_in_group = __popc(eqm);
        return in && (key > kstar || (is_eq && eq + __popc(eqm & below) < cstar));
    };
    unsigned open_w = 0;
    {
        unsigned eq = eq_base, eqg;
        // keys of KB groups of 32 positions are loaded before any is used
        for (long long i00 = rbeg; i00 < rend; i00 += 32 * KB) {
            uint32_t kk[KB];
#pragma unroll
            for (int u = 0; u < KB; ++u) {
                const long long i = i00 + 32 * u + lane;
                kk[u] = i < rend && !open_all ? key_at(i) : 0u;
            }
#pragma unroll
            for (int u = 0; u < KB; ++u) {
                const long long i0 = i00 + 32 * u;
                if (i0 >= rend) break;
                const bool o = opened(i0 + lane, kk[u], eq, eqg);
                open_w += __popc(__ballot_sync(FULL, o));
                eq += eqg;
            }
        }
    }
    unsigned n_open;
    const unsigned v_open = lane == 0 ? open_w : 0u;
    unsigned open_base = block_incl_scan<NT, unsigned>(v_open, sh_u32, &n_open) - v_open;
    open_base = __shfl_sync(FULL, open_base, 0);

    // write the opened ids (ascending, since frontier positions ascend in id)
    {
        unsigned *M_tree = a.M_next ? a.M_next + (long long)t * a.words_next * a.G : nullptr;
        unsigned *U_tree = a.U_next ? a.U_next + (long long)t * a.words_next : nullptr;
        unsigned eq = eq_base, eqg, rank = open_base;
        // node ids of 8 groups of 32 positions are loaded before any is used
        for (long long i00 = rbeg; i00 < rend; i00 += 32 * 8) {
            long long idv[8];
            uint32_t kk[KB > 1 ? 8 : 1];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const long long i = i00 + 32 * u + lane;
                idv[u] = i < rend ? frontier_id(a, lid, par, npar, i) : 0;
                if constexpr (KB > 1) kk[u] = i < rend && !open_all ? key_at(i) : 0u;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const long long i0 = i00 + 32 * u;
                if (i0 >= rend) break;
                const long long i = i0 + lane;
                uint32_t key;
                if constexpr (KB > 1) key = kk[u];
                else key = i < rend && !open_all ? key_at(i) : 0u;
                const bool o = opened(i, key, eq, eqg);
                const unsigned om = __ballot_sync(FULL, o);
                if (o) {
                    const unsigned r = rank + __popc(om & below);
                    const long long id = idv[u];
                    if (a.level == 1) {
                        if (r < (unsigned)a.max_sel) a.sel[walk * a.max_sel + r] = (int)id;
                    } else {
                        a.par_out[walk * a.Lstride + r] = (int)id;
                        if (M_tree) set_bits(M_tree, U_tree, a.G, g, id * a.C, id * a.C + a.C);
                    }
                }
                rank += __popc(om);
                eq += eqg;
            }
        }
        if (a.level > 1 && a.n_orph_next > 0) {
            const long long lo = a.n_level_next - a.n_orph_next, hi = a.n_level_next;
            for (long long w = (lo >> 5) + tid; w <= (hi - 1) >> 5; w += NT) {
                const long long wlo = lo > (w << 5) ? lo : (w << 5);
                const long long whi = hi < ((w + 1) << 5) ? hi : ((w + 1) << 5);
                set_bits(M_tree, U_tree, a.G, g, wlo, whi);
            }
        }
    }
    if (tid == 0) {
        if (a.level > 1) {
            a.n_par_out[walk] = (int)n_open;
        } else {
            a.sel_count[walk] = (int)min(n_open, (unsigned)a.max_sel);
            if (n_open > (unsigned)a.max_sel) report(a.status, DEV_CAPACITY);
        }
        if (a.stats) {
            zha_stats *s = a.stats + walk;
            s->frontier[a.level] = (int)F;
            s->opened[a.level] = (int)n_open;
            if (a.level == 1) {
                long long sum = 0;
                for (int l = 1; l <= ZHA_MAX_DEPTH; ++l) sum += s->frontier[l];
                s->keys_read = (long long)a.C * n_open + a.tail;
                s->work = (long long)a.R * sum + s->keys_read;
            }
        }
    }
    chain_done();
}

// Sorts the 32 * E keys of a warp in descending order (lane l holds positions
// l * E .. l * E + E - 1): a bitonic network, exchanges across lanes by shuffle
// and inside a lane in registers.
template <int E>
__device__ __forceinline__ void warp_sort_desc(uint32_t (&v)[E], int lane) {
    constexpr int N = 32 * E;
#pragma unroll
    for (int k = 2; k <= N; k <<= 1) {
#pragma unroll
        for (int j = k >> 1; j >= 1; j >>= 1) {
            if (j >= E) {
                const int lj = j / E;  // partner lane distance
                const bool lower = (lane & lj) == 0;
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    const bool desc = ((lane * E + e) & k) == 0;  // this run sorts descending
                    const uint32_t o = __shfl_xor_sync(FULL, v[e], lj);
                    v[e] = lower == desc ? max(v[e], o) : min(v[e], o);
                }
            } else {
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    if ((e & j) == 0) {
                        const bool desc = ((lane * E + e) & k) == 0;
                        const uint32_t x = v[e], y = v[e | j];
                        v[e] = desc ? max(x, y) : min(x, y);
                        v[e | j] = desc ? min(x, y) : max(x, y);
                    }
                }
            }
        }
    }
}

__device__ __forceinline__ unsigned long long warp_sum_u64(unsigned long long x) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) x += __shfl_xor_sync(FULL, x, o);
    return x;
}

// One warp per walk, for levels whose frontiers hold at most 32 * E nodes (the
// host bounds them): the frontier's keys sit in registers (E per lane, in
// position order), a sorted copy gives the cutoff key kstar as the first key at
// which the prefix of the fixed-point masses (counts for top-K) reaches the
// target, and the opened nodes follow the rule of select_level_kernel: keys above
// kstar, then the first cstar keys equal to it by position. Masses, target and
// rule are those of the block path, so both choose the same nodes; this one needs
// no block barrier, and many walks share an SM.
template <int E>
__global__ void __launch_bounds__(256) select_warp_kernel(SelectArgs a) {
    chain_start();
    const int lane = threadIdx.x & 31;
    const long long walk = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (walk < a.n_walks) {
        const int t = (int)(walk / a.G), g = (int)(walk % a.G);
        const long long npar = a.start ? 0 : a.n_par_in[walk];
        const int *par = a.start ? nullptr : a.par_in + walk * a.Lstride;
        long long F = a.start ? a.n_level : npar * a.C + a.n_orph;
        if (F > 32 * E) {  // outside the host's bound: report, open nothing
            if (lane == 0) report(a.status, DEV_BAD_INDEX);
            F = 0;
        }
        const float *S = a.S + walk * a.Sstride;
        // keys in position order (0 past the frontier: below every score's key).
        // Every load is issued unconditionally at a clamped index, so all E of a
        // lane are in flight together; positions past the frontier are masked.
        uint32_t key[E];
        int id[E];
        if (a.start) {
#pragma unroll
            for (int e = 0; e < E; ++e) id[e] = lane * E + e;
        } else {
            const int kids = (int)npar * a.C, C = a.C;
            const int orph0 = (int)(a.n_level - a.n_orph) - kids;  // id of position i >= kids: orph0 + i
            int pv[E];
#pragma unroll
            for (int e = 0; e < E; ++e) {
                const int i = lane * E + e;
                const int pi = i < kids ? (a.c_shift >= 0 ? i >> a.c_shift : i / C) : 0;
                pv[e] = par[pi];  // par holds at least one entry per walk
            }
#pragma unroll
            for (int e = 0; e < E; ++e) {
                const int i = lane * E + e;
                const int pi = a.c_shift >= 0 ? i >> a.c_shift : i / C;
                id[e] = i < kids ? pv[e] * C + (i - pi * C) : orph0 + i;
            }
        }
        float sv[E];
#pragma unroll
        for (int e = 0; e < E; ++e) sv[e] = S[lane * E + e < F ? id[e] : 0];
#pragma unroll
        for (int e = 0; e < E; ++e) key[e] = lane * E + e < F ? order_key(sv[e]) : 0u;
        uint32_t kmax = 0;
#pragma unroll
        for (int e = 0; e < E; ++e) kmax = max(kmax, key[e]);
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) kmax = max(kmax, __shfl_xor_sync(FULL, kmax, o));
        const float m = key_to_float(kmax);
        const bool top_p = a.mode == ZHA_TOP_P;
        const bool open_all = (top_p && a.p >= 1.f) || (!top_p && (long long)a.k >= F);
        auto weight = [&](uint32_t k) -> unsigned long long {
            return k == 0u ? 0ull : (top_p ? mass_fixed(expf(key_to_float(k) - m)) : 1ull);
        };

        uint32_t kstar = 0;
        unsigned long long cstar = 0;
        if (F > 0 && !open_all) {
            uint32_t sk[E];
#pragma unroll
            for (int e = 0; e < E; ++e) sk[e] = key[e];
            warp_sort_desc<E>(sk, lane);
            unsigned long long w[E], lane_tot = 0;
#pragma unroll
            for (int e = 0; e < E; ++e) {
                w[e] = weight(sk[e]);
                lane_tot += w[e];
            }
            // exclusive prefix of the lanes' totals
            unsigned long long incl = lane_tot;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const unsigned long long y = __shfl_up_sync(FULL, incl, o);
                if (lane >= o) incl += y;
            }
            const unsigned long long total = __shfl_sync(FULL, incl, 31);
            unsigned long long target;
            if (top_p) {
                target = (unsigned long long)ceil((double)a.p * (double)total);
                if (target < 1) target = 1;
                if (target > total) target = total;
            } else {
                target = (unsigned long long)a.k;
            }
            // the cutoff: the sorted key whose weight takes the prefix to the target
            unsigned long long pre = incl - lane_tot;
            uint32_t mine = 0;
            bool hit = false;
#pragma unroll
            for (int e = 0; e < E; ++e) {
                if (!hit && pre < target && target <= pre + w[e]) {
                    hit = true;
                    mine = sk[e];
                }
                pre += w[e];
            }
            const unsigned hb = __ballot_sync(FULL, hit);
            kstar = __shfl_sync(FULL, mine, hb ? __ffs(hb) - 1 : 0);
            // weight strictly above kstar, then how many of its equal keys to open
            unsigned long long above = 0;
#pragma unroll
            for (int e = 0; e < E; ++e) above += sk[e] > kstar ? w[e] : 0ull;
            above = warp_sum_u64(above);
            const unsigned long long u = weight(kstar);
            const unsigned long long rem = target > above ? target - above : 0ull;
            cstar = top_p ? (u > 0 ? (rem + u - 1) / u : 1ull) : rem;
        }

        // opened positions, in position order: rank among the keys equal to kstar
        // by a scan of per-lane counts, then compaction by a scan of opened counts
        bool open[E];
        {
            unsigned eq_l = 0;
#pragma unroll
            for (int e = 0; e < E; ++e) eq_l += (key[e] == kstar && key[e] != 0u) ? 1u : 0u;
            unsigned eq_incl = eq_l;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const unsigned y = __shfl_up_sync(FULL, eq_incl, o);
                if (lane >= o) eq_incl += y;
            }
            unsigned eq = eq_incl - eq_l;
#pragma unroll
            for (int e = 0; e < E; ++e) {
                const bool in = lane * E + e < F;
                if (open_all) {
                    open[e] = in;
                } else {
                    const bool is_eq = in && key[e] == kstar;
                    open[e] = in && (key[e] > kstar || (is_eq && (unsigned long long)eq < cstar));
                    eq += is_eq ? 1u : 0u;
                }
            }
        }
        unsigned n_l = 0;
#pragma unroll
        for (int e = 0; e < E; ++e) n_l += open[e] ? 1u : 0u;
        unsigned n_incl = n_l;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const unsigned y = __shfl_up_sync(FULL, n_incl, o);
            if (lane >= o) n_incl += y;
        }
        const unsigned n_open = __shfl_sync(FULL, n_incl, 31);
        unsigned r = n_incl - n_l;
        unsigned *M_tree = a.M_next ? a.M_next + (long long)t * a.words_next * a.G : nullptr;
        unsigned *U_tree = a.U_next ? a.U_next + (long long)t * a.words_next : nullptr;
#pragma unroll
        for (int e = 0; e < E; ++e) {
            if (!open[e]) continue;
            const long long nid = id[e];
            if (a.level == 1) {
                if (r < (unsigned)a.max_sel) a.sel[walk * a.max_sel + r] = (int)nid;
            } else {
                a.par_out[walk * a.Lstride + r] = (int)nid;
                if (M_tree) set_bits(M_tree, U_tree, a.G, g, nid * a.C, nid * a.C + a.C);
            }
            ++r;
        }
        if (a.level > 1 && a.n_orph_next > 0 && M_tree) {
            const long long lo = a.n_level_next - a.n_orph_next, hi = a.n_level_next;
            for (long long wd = (lo >> 5) + lane; wd <= (hi - 1) >> 5; wd += 32) {
                const long long wlo = lo > (wd << 5) ? lo : (wd << 5);
                const long long whi = hi < ((wd + 1) << 5) ? hi : ((wd + 1) << 5);
                set_bits(M_tree, U_tree, a.G, g, wlo, whi);
            }
        }
        if (lane == 0) {
            if (a.level > 1) {
                a.n_par_out[walk] = (int)n_open;
            } else {
                a.sel_count[walk] = (int)min(n_open, (unsigned)a.max_sel);
                if (n_open > (unsigned)a.max_sel) report(a.status, DEV_CAPACITY);
            }
            if (a.stats) {
                zha_stats *st = a.stats + walk;
                st->frontier[a.level] = (int)F;
                st->opened[a.level] = (int)n_open;
                if (a.level == 1) {
                    long long sum = 0;
                    for (int l = 1; l <= ZHA_MAX_DEPTH; ++l) sum += st->frontier[l];
                    st->keys_read = (long long)a.C * n_open + a.tail;
                    st->work = (long long)a.R * sum + st->keys_read;
                }
            }
        }
    }
    chain_done();
}

template <int E>
cudaError_t launch_select_warp(const SelectArgs &se, long long W, cudaStream_t st) {
    SelectArgs a = se;
    a.n_walks = W;
    return launch_chained(select_warp_kernel<E>, dim3((unsigned)((W + 7) / 8)), dim3(256), 0, st, a);
}

template <int NT, int KB = 1>
cudaError_t launch_select(const SelectArgs &se, long long W, cudaStream_t st) {
    static bool smem_set = false;
    if (!smem_set) {
        cudaError_t e = cudaFuncSetAttribute(select_level_kernel<NT, KB>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, 16384 * (int)sizeof(uint32_t));
        if (e != cudaSuccess) return e;
        smem_set = true;
    }
    return launch_chained(select_level_kernel<NT, KB>, dim3((unsigned)W), dim3(NT),
                          (size_t)se.smem_keys * sizeof(uint32_t), st, se);
}

template <int D, int RP>
cudaError_t launch_score(const zha_tree *t, ScoreArgs a, cudaStream_t st) {
    static int per_sm = 0;
    if (!per_sm) {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, score_level_kernel<D, RP>, 256, 0) != cudaSuccess ||
            per_sm < 1)
            per_sm = 1;
    }
    const long long resident_warps = (long long)num_sms() * per_sm * 8;
    if (a.T * ((a.n_level + 3) / 4) < 4 * resident_warps) a.npi = 1;
    const long long items = (long long)a.T * ((a.n_level + a.npi - 1) / a.npi);
    long long blocks = (items + 7) / 8;
    const long long cap = (long long)num_sms() * per_sm;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) return cudaSuccess;
    Probe pr(t, ZHA_K_SCORE, st);
    // The scorer of a very large level (more than 2^22 node slots, a multi-ms
    // launch) is launched in plain stream order: measured on B200, chaining it
    // made it about 15% slower, while chaining every smaller launch saves the
    // launch gap.
    if ((long long)a.T * a.n_level > (1LL << 22)) {
        score_level_kernel<D, RP><<<(unsigned)blocks, 256, 0, st>>>(a);
        return cudaGetLastError();
    }
    return launch_chained(score_level_kernel<D, RP>, dim3((unsigned)blocks), dim3(256), 0, st, a);
}

template <int D>
cudaError_t launch_score_d(const zha_tree *t, const ScoreArgs &a, cudaStream_t st) {
    if (a.R <= 1) return launch_score<D, 1>(t, a, st);
    if (a.R <= 2) return launch_score<D, 2>(t, a, st);
    if (a.R <= 4) return launch_score<D, 4>(t, a, st);
    if (a.R <= 8) return launch_score<D, 8>(t, a, st);
    return launch_score<D, 16>(t, a, st);
}

}  // namespace

cudaError_t launch_select_all(const zha_tree *t, const float *S, uint32_t *gkey, long long N, long long W, int G,
                              int mode, float p, int k, int *sel, int *sel_count, int max_sel, cudaStream_t st) {
    // every one of the N candidates (keys) is in the frontier: the start-level path
    SelectArgs se{};
    se.level = 1;
    se.C = 1;
    se.c_shift = 0;
    se.R = t->cfg.R;
    se.G = G;
    se.start = 1;
    se.n_level = N;
    se.n_orph = 0;
    se.n_orph_next = 0;
    se.n_level_next = 0;
    se.S = S;
    se.Sstride = N;
    se.par_in = nullptr;
    se.par_out = nullptr;
    se.Lstride = 0;
    se.n_par_in = nullptr;
    se.n_par_out = nullptr;
    se.M_next = nullptr;
    se.U_next = nullptr;
    se.words_next = 0;
    se.mode = mode;
    se.p = p;
    se.k = k;
    se.sel = sel;
    se.max_sel = max_sel;
    se.sel_count = sel_count;
    se.stats = nullptr;
    se.tail = 0;
    se.status = t->d_status;
    se.gkey = gkey;
    Probe pr(t, ZHA_K_SELECT, st);
    if (N > 8192) {
        se.smem_keys = std::min<long long>(N, 16384);
        return N > 16384 ? launch_select<1024, 8>(se, W, st) : launch_select<1024>(se, W, st);
    }
    se.smem_keys = N;
    return launch_select<256>(se, W, st);
}

cudaError_t launch_search_init(const zha_tree *t, const Scratch &s, const void *Q, zha_dtype q_dtype, int G,
                               long long W, zha_stats *stats, int start_level, cudaStream_t st) {
    auto words = [&](int l) { return (t->cap_nodes[l] + 31) / 32; };
    InitArgs ia{};
    ia.Q = Q;
    ia.q_bf16 = q_dtype == ZHA_BF16;
    ia.D = t->cfg.d;
    ia.W = W;
    ia.qf = s.qf;
    ia.n_par = s.cnt[0];
    ia.M = s.M[start_level];
    ia.U = s.U[start_level];
    ia.words = words(start_level);
    ia.G = G;
    ia.n_s = t->n_nodes[start_level];
    ia.stats = stats;
    ia.start_level = start_level;
    ia.M_all = s.M_base;
    ia.U_all = s.U_base;
    ia.M_all_words = (long long)(s.M_bytes / sizeof(unsigned));
    ia.U_all_words = (long long)(s.U_bytes / sizeof(unsigned));
    Probe pr(t, ZHA_K_SEARCH_INIT, st);
    return launch_chained(search_init_kernel, dim3((unsigned)W), dim3(128), 0, st, ia);
}

cudaError_t launch_score_level(const zha_tree *t, const Scratch &s, int l, int G, cudaStream_t st) {
    const zha_config &c = t->cfg;
    ScoreArgs sa{};
    sa.nodes = t->nodes[l];
    sa.node_tree = t->cap_nodes[l] * t->NF;
    sa.NF = t->NF;
    sa.R = c.R;
    sa.G = G;
    sa.T = t->T;
    sa.beta = c.sharpness;
    sa.U = s.U[l];
    sa.M = s.M[l];
    sa.words = (t->cap_nodes[l] + 31) / 32;
    sa.n_level = t->n_nodes[l];
    sa.qf = s.qf;
    sa.S = s.S;
    sa.Sstride = s.Sstride;
    sa.npi = 4;
    switch (c.d) {
        case 64: return launch_score_d<64>(t, sa, st);
        case 128: return launch_score_d<128>(t, sa, st);
        default: return launch_score_d<256>(t, sa, st);
    }
}

cudaError_t launch_search(const zha_tree *t, const Scratch &s, const void *Q, zha_dtype q_dtype, int G,
                          long long W, int mode, float p, int k, int *sel, int *sel_count, int max_sel,
                          zha_stats *stats, int start_level, cudaStream_t st) {
    const zha_config &c = t->cfg;
    const int C = c.chunk;
    cudaError_t e;
    auto words = [&](int l) { return (t->cap_nodes[l] + 31) / 32; };
    if ((e = launch_search_init(t, s, Q, q_dtype, G, W, stats, start_level, st)) != cudaSuccess) return e;

    // trees walked by many bf16 queries score whole small levels on the tensor cores
    bool tc_any = false;
    if (s.tc)
        for (int l = start_level; l >= 1; --l) tc_any = tc_any || tc_applicable(t, G, Q, q_dtype, l);
    if (tc_any) {
        e = launch_score_tc_queries(t, Q, G, s.tc, st);
        if (e != cudaSuccess) return e;
    }

    int cur = 0;
    for (int l = start_level; l >= 1; --l) {
        if (tc_any && tc_applicable(t, G, Q, q_dtype, l)) {
            e = launch_score_tc(t, l, G, s.tc, s.tc_b, s.S, s.Sstride, st);
            if (e != cudaSuccess) return e;
        } else if (s.tc_lists && tc_sparse_applicable(t, G, Q, q_dtype, l)) {
            e = launch_score_tc_sparse(t, l, G, Q, s.M[l], words(l), s.tc_counts, s.tc_lists, s.S, s.Sstride,
                                       st);
            if (e != cudaSuccess) return e;
        } else {
            if ((e = launch_score_level(t, s, l, G, st)) != cudaSuccess) return e;
        }

        SelectArgs se{};
        se.level = l;
        se.C = C;
        se.c_shift = (C & (C - 1)) == 0 ? __builtin_ctz((unsigned)C) : -1;
        se.R = c.R;
        se.G = G;
        se.start = l == start_level;
        se.n_level = t->n_nodes[l];
        se.n_orph = l == start_level ? 0 : t->n_nodes[l] - (long long)C * t->n_nodes[l + 1];
        se.n_level_next = l > 1 ? t->n_nodes[l - 1] : 0;
        se.n_orph_next = l > 1 ? t->n_nodes[l - 1] - (long long)C * t->n_nodes[l] : 0;
        se.S = s.S;
        se.Sstride = s.Sstride;
        se.par_in = s.L[cur];
        se.par_out = s.L[cur ^ 1];
        se.Lstride = s.Lstride;
        se.n_par_in = s.cnt[cur];
        se.n_par_out = s.cnt[cur ^ 1];
        se.M_next = l > 1 ? s.M[l - 1] : nullptr;
        se.U_next = l > 1 ? s.U[l - 1] : nullptr;
        se.words_next = l > 1 ? words(l - 1) : 0;
        se.mode = mode;
        se.p = p;
        se.k = k;
        se.sel = sel;
        se.max_sel = max_sel;
        se.sel_count = sel_count;
        se.stats = stats;
        se.tail = t->n - (long long)C * t->n_nodes[1];
        se.status = t->d_status;
        se.gkey = s.gkey;
        {
            // the widest frontier a walk can have at this level: the whole level, or
            // for top-K below the start level the children of K nodes and the orphans
            long long fmax = t->n_nodes[l];
            if (mode == ZHA_TOP_K && l != start_level)
                fmax = std::min<long long>(fmax, (long long)k * C + se.n_orph);
            Probe pr(t, ZHA_K_SELECT, st);
            if (fmax <= 64) {
                // frontiers of at most 64 nodes: one warp per walk
                e = launch_select_warp<2>(se, W, st);
            } else if (fmax <= 512 && W >= 8192) {
                // many walks (prefill) over frontiers of at most 512 nodes: one
                // warp per walk as well (with few walks the block path's shorter
                // per-walk latency wins)
                e = fmax <= 128   ? launch_select_warp<4>(se, W, st)
                    : fmax <= 256 ? launch_select_warp<8>(se, W, st)
                                  : launch_select_warp<16>(se, W, st);
            } else if (fmax > 8192 && W > 2LL * num_sms()) {
                // many walks (prefill) over a wide level: most frontiers are far
                // smaller than the level, so 256 threads and 4,096 keys of shared
                // staging per CTA (wider frontiers stage in global memory) let more
                // walks' CTAs share an SM (measured on B200: 7.31 -> 6.68 ms for the
                // prefill workload's search)
                se.smem_keys = 4096;
                e = launch_select<256>(se, W, st);
            } else if (fmax > 8192) {
                // few walks: the widest frontier sets the time, give it 1,024 threads
                se.smem_keys = std::min<long long>(fmax, 16384);
                e = launch_select<1024>(se, W, st);
            } else if (fmax > 2048 && W <= 2LL * num_sms()) {
                // few walks over a level of thousands of nodes: frontiers of a few
                // thousand keys, 512 threads
                se.smem_keys = fmax;
                e = launch_select<512>(se, W, st);
            } else {
                se.smem_keys = fmax;
                e = launch_select<256>(se, W, st);
            }
            if (e != cudaSuccess) return e;
        }
        cur ^= 1;
    }
    return cudaSuccess;
}


// ---------------------------------------------------------------------------
// Context-parallel walk: this process holds a shard of every tree (keys
// key_begin .. of the whole sequence, whole top-level nodes, so its level-l
// nodes are the whole tree's nodes off_l = key_begin / C^l onward). A level
// step is: score the shard's frontier (the CUDA-core scorer, as a search
// does), export each walk's (global id, score) list, let the caller gather the
// lists of every process (process order = id order), then pack them per walk,
// choose over them with the selector's list mode (the same passes, so the
// same choice as one search over the whole tree), and keep the opened nodes
// the shard holds: their children, and the orphans of the level below (only on
// the last process), are the shard's next frontier.
namespace {

struct CpExportArgs {
    int C, start;
    long long n_level, n_orph, off;
    const int *par;
    long long Lstride;
    const int *npar;
    const float *S;
    long long Sstride;
    int *ids;
    float *scores;
    int *counts;
    long long stride;
    int *status;
};

// one CTA per walk: the shard's frontier in position (= id) order, ids made global
__global__ void cp_export_kernel(CpExportArgs a) {
    const long long w = blockIdx.x;
    const long long npar = a.start ? 0 : a.npar[w];
    const long long kids = npar * a.C;
    const long long F = a.start ? a.n_level : kids + a.n_orph;
    const long long n = F < a.stride ? F : a.stride;
    if (threadIdx.x == 0) {
        a.counts[w] = (int)n;
        if (F > a.stride) report(a.status, DEV_CAPACITY);
    }
    const int *par = a.par + w * a.Lstride;
    for (long long i = threadIdx.x; i < n; i += blockDim.x) {
        long long id;
        if (a.start) id = i;
        else if (i < kids) id = (long long)par[i / a.C] * a.C + i % a.C;
        else id = (a.n_level - a.n_orph) + (i - kids);
        a.ids[w * a.stride + i] = (int)(id + a.off);
        a.scores[w * a.stride + i] = a.S[w * a.Sstride + id];
    }
}

// one CTA per walk: the gathered lists of the n_parts processes, concatenated
__global__ void cp_pack_kernel(int n_parts, const int *ids, const float *scores, const int *counts, long long stride,
                               long long W, int *pids, float *pscores, int *pcount, long long P) {
    const long long w = blockIdx.x;
    long long base = 0;
    for (int r = 0; r < n_parts; ++r) {
        long long c = counts[(long long)r * W + w];
        c = c < 0 ? 0 : (c > stride ? stride : c);
        const long long src = ((long long)r * W + w) * stride;
        for (long long i = threadIdx.x; i < c; i += blockDim.x) {
            pids[w * P + base + i] = ids[src + i];
            pscores[w * P + base + i] = scores[src + i];
        }
        base += c;
    }
    if (threadIdx.x == 0) pcount[w] = (int)base;
}

struct CpLocalArgs {
    int level, C, G;
    const int *opened;
    const int *ocount;
    long long P;
    long long lo, n_local;  // the shard's ids at this level: [lo, lo + n_local)
    // level > 1: the shard's opened nodes (local ids) and the next level's membership bits
    int *par_out;
    int *npar_out;
    long long Lstride;
    unsigned *M_next, *U_next;
    long long words_next, n_next_local, n_orph_next;
    // level 1: the shard's chosen chunks (local ids)
    int *sel;
    int *sel_count;
    int max_sel;
    int *status;
};

// one CTA per walk: the opened ids (ascending) that fall in the shard
__global__ void cp_localize_kernel(CpLocalArgs a) {
    __shared__ long long s_b0, s_b1;
    const long long w = blockIdx.x;
    const int t = (int)(w / a.G), g = (int)(w % a.G);
    const int *op = a.opened + w * a.P;
    const long long n = a.ocount[w];
    if (threadIdx.x == 0) {
        // first position with id >= lo, first with id >= lo + n_local
        long long lo = 0, hi = n;
        while (lo < hi) {
            const long long mid = (lo + hi) >> 1;
            if (op[mid] < a.lo) lo = mid + 1;
            else hi = mid;
        }
        s_b0 = lo;
        hi = n;
        while (lo < hi) {
            const long long mid = (lo + hi) >> 1;
            if (op[mid] < a.lo + a.n_local) lo = mid + 1;
            else hi = mid;
        }
        s_b1 = lo;
    }
    __syncthreads();
    const long long b0 = s_b0, b1 = s_b1;
    if (a.level > 1) {
        unsigned *M_tree = a.M_next + (long long)t * a.words_next * a.G;
        unsigned *U_tree = a.U_next + (long long)t * a.words_next;
        for (long long i = b0 + threadIdx.x; i < b1; i += blockDim.x) {
            const long long local = op[i] - a.lo;
            a.par_out[w * a.Lstride + (i - b0)] = (int)local;
            set_bits(M_tree, U_tree, a.G, g, local * a.C, local * a.C + a.C);
        }
        if (a.n_orph_next > 0) {
            const long long lo = a.n_next_local - a.n_orph_next, hi = a.n_next_local;
            for (long long wd = (lo >> 5) + threadIdx.x; wd <= (hi - 1) >> 5; wd += blockDim.x) {
                const long long wlo = lo > (wd << 5) ? lo : (wd << 5);
                const long long whi = hi < ((wd + 1) << 5) ? hi : ((wd + 1) << 5);
                set_bits(M_tree, U_tree, a.G, g, wlo, whi);
            }
        }
        if (threadIdx.x == 0) a.npar_out[w] = (int)(b1 - b0);
    } else {
        for (long long i = b0 + threadIdx.x; i < b1 && i - b0 < a.max_sel; i += blockDim.x)
            a.sel[w * a.max_sel + (i - b0)] = op[i] - (int)a.lo;
        if (threadIdx.x == 0) {
            a.sel_count[w] = (int)(b1 - b0 < a.max_sel ? b1 - b0 : a.max_sel);
            if (b1 - b0 > a.max_sel) report(a.status, DEV_CAPACITY);
        }
    }
}

__global__ void lse_combine_kernel(int n_parts, long long W, int D, const float *outs, const float *lses, void *out,
                                   int out_bf16, float *lse) {
    const long long w = blockIdx.x;
    float m = -INFINITY;
    for (int r = 0; r < n_parts; ++r) m = fmaxf(m, lses[(long long)r * W + w]);
    float l = 0.f;
    for (int r = 0; r < n_parts; ++r) {
        const float x = lses[(long long)r * W + w];
        l += x == -INFINITY ? 0.f : expf(x - m);
    }
    for (int e = threadIdx.x; e < D; e += blockDim.x) {
        float acc = 0.f;
        for (int r = 0; r < n_parts; ++r) {
            const float x = lses[(long long)r * W + w];
            if (x != -INFINITY) acc = fmaf(expf(x - m), outs[((long long)r * W + w) * D + e], acc);
        }
        const float v = l > 0.f ? acc / l : 0.f;
        if (out_bf16) static_cast<__nv_bfloat16 *>(out)[w * D + e] = __float2bfloat16_rn(v);
        else static_cast<float *>(out)[w * D + e] = v;
    }
    if (threadIdx.x == 0 && lse) lse[w] = l > 0.f ? m + logf(l) : -INFINITY;
}

}  // namespace

cudaError_t launch_cp_export(const zha_tree *t, const Scratch &s, int cur, int level, bool start, long long off,
                             long long W, int *ids, float *scores, int *counts, long long stride, cudaStream_t st) {
    CpExportArgs a{};
    a.C = t->cfg.chunk;
    a.start = start ? 1 : 0;
    a.n_level = t->n_nodes[level];
    a.n_orph = start ? 0 : t->n_nodes[level] - (long long)a.C * t->n_nodes[level + 1];
    a.off = off;
    a.par = s.L[cur];
    a.Lstride = s.Lstride;
    a.npar = s.cnt[cur];
    a.S = s.S;
    a.Sstride = s.Sstride;
    a.ids = ids;
    a.scores = scores;
    a.counts = counts;
    a.stride = stride;
    a.status = t->d_status;
    Probe pr(t, ZHA_K_SELECT, st);
    cp_export_kernel<<<(unsigned)W, 256, 0, st>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_cp_select(const zha_tree *t, const Scratch &s, int cur, int level, int G, long long W, int n_parts,
                             const int *ids, const float *scores, const int *counts, long long stride, int mode,
                             float p, int k, const CpScratch &cs, long long lo, int *sel, int *sel_count,
                             int max_sel, cudaStream_t st) {
    const zha_config &c = t->cfg;
    const long long P = cs.P;
    cudaError_t e;
    {
        Probe pr(t, ZHA_K_SELECT, st);
        cp_pack_kernel<<<(unsigned)W, 256, 0, st>>>(n_parts, ids, scores, counts, stride, W, cs.pids, cs.pscores,
                                                     cs.pcount, P);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    SelectArgs se{};
    se.level = level;
    se.C = c.chunk;
    se.c_shift = (c.chunk & (c.chunk - 1)) == 0 ? __builtin_ctz((unsigned)c.chunk) : -1;
    se.R = c.R;
    se.G = G;
    se.start = 0;
    se.list_ids = cs.pids;
    se.list_scores = cs.pscores;
    se.list_count = cs.pcount;
    se.list_stride = P;
    se.Sstride = P;  // the global staging rows are P keys long
    se.gkey = cs.stage;
    se.mode = mode;
    se.p = p;
    se.k = k;
    if (level > 1) {
        se.par_out = cs.opened;
        se.Lstride = P;
        se.n_par_out = cs.ocount;
    } else {
        se.sel = cs.opened;
        se.max_sel = (int)P;
        se.sel_count = cs.ocount;
    }
    se.status = t->d_status;
    {
        Probe pr(t, ZHA_K_SELECT, st);
        if (P > 8192) {
            se.smem_keys = std::min<long long>(P, 16384);
            e = launch_select<1024>(se, W, st);
        } else if (P > 2048) {
            se.smem_keys = P;
            e = launch_select<512>(se, W, st);
        } else {
            se.smem_keys = P;
            e = launch_select<256>(se, W, st);
        }
        if (e != cudaSuccess) return e;
    }
    CpLocalArgs la{};
    la.level = level;
    la.C = c.chunk;
    la.G = G;
    la.opened = cs.opened;
    la.ocount = cs.ocount;
    la.P = P;
    la.lo = lo;
    la.n_local = t->n_nodes[level];
    if (level > 1) {
        la.par_out = s.L[cur ^ 1];
        la.npar_out = s.cnt[cur ^ 1];
        la.Lstride = s.Lstride;
        la.M_next = s.M[level - 1];
        la.U_next = s.U[level - 1];
        la.words_next = (t->cap_nodes[level - 1] + 31) / 32;
        la.n_next_local = t->n_nodes[level - 1];
        la.n_orph_next = t->n_nodes[level - 1] - (long long)c.chunk * t->n_nodes[level];
    } else {
        la.sel = sel;
        la.sel_count = sel_count;
        la.max_sel = max_sel;
    }
    la.status = t->d_status;
    Probe pr(t, ZHA_K_SELECT, st);
    cp_localize_kernel<<<(unsigned)W, 256, 0, st>>>(la);
    return cudaGetLastError();
}

cudaError_t launch_lse_combine(int n_parts, long long W, int D, const float *outs, const float *lses, void *out,
                               zha_dtype out_dtype, float *lse, cudaStream_t st) {
    lse_combine_kernel<<<(unsigned)W, D < 256 ? D : 256, 0, st>>>(n_parts, W, D, outs, lses, out,
                                                                  out_dtype == ZHA_BF16, lse);
    return cudaGetLastError();
}

}  // namespace zha
