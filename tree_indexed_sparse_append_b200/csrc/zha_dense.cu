// Full-scan indexer: the comparison point for the tree walk.
//
// Page "Zyphra AI Introduces ZHA, a Path to True Subquadratic Attention": sparse
// attention methods such as DeepSeek Sparse Attention pick their keys with an
// indexer that scores every token in the context. Here every key of a walk's
// tree is scored, s_j = beta <q, k_j>, and the same selection rule as one level
// of the tree walk is applied to the keys themselves: the softmax over all keys,
// then the shortest mass-ordered prefix reaching p (top-p) or the K largest
// (top-K), ties to the lower key index.
//
// dense_score  tree-major, one pass over each tree's keys for all the walks of
//              the tree (the GQA heads and queries that share it): lane l owns
//              d/32 columns of U consecutive keys, computes U x GP partial dot
//              products (GP = walks per tree, padded to a power of two,
//              U * GP = 32), and one warp transpose-reduce leaves every lane
//              with one (key, walk) score.
// select       the tree walk's selector with every key in the frontier.
//
// Chunk-mass profile (same page set, "How does top-p differ from top-K?": how
// many 16-key chunks hold 90% of a query's attention varies a lot by task): the
// dense scores above, reduced per run of `group` keys to the chunk's
// log-sum-exp, so that the softmax over chunk scores is the chunk's share of the
// dense attention; the selector then opens the fewest chunks reaching p.
#include <algorithm>

#include "zha_internal.cuh"

namespace zha {
namespace {

struct DenseArgs {
    const void *K;
    long long cap, N;
    int T, G;
    float beta;
    const float *qf;  // [W][D]
    float *S;         // [W][N]
};

__global__ void convert_queries_kernel(const void *Q, int q_bf16, long long n, float *qf) {
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
        qf[i] = q_bf16 ? __bfloat162float(static_cast<const __nv_bfloat16 *>(Q)[i]) : static_cast<const float *>(Q)[i];
}

// EPL consecutive elements of T as floats (one vector load)
template <typename T, int EPL>
__device__ __forceinline__ void load_slice(const T *p, float (&v)[EPL]) {
    if constexpr (sizeof(T) == 2) {
        load_cached<EPL>(reinterpret_cast<const __nv_bfloat16 *>(p), v);
    } else {
        if constexpr (EPL == 2) {
            const float2 x = __ldg(reinterpret_cast<const float2 *>(p));
            v[0] = x.x;
            v[1] = x.y;
        } else {
#pragma unroll
            for (int i = 0; i < EPL; i += 4) {
                const float4 x = __ldg(reinterpret_cast<const float4 *>(p) + i / 4);
                v[i] = x.x;
                v[i + 1] = x.y;
                v[i + 2] = x.z;
                v[i + 3] = x.w;
            }
        }
    }
}

constexpr int DENSE_STEPS = 8;  // key steps per work item

template <typename T, int D, int GP>
__global__ void __launch_bounds__(256) dense_score_kernel(DenseArgs a) {
    constexpr int EPL = D / 32;
    constexpr int U = 32 / GP;  // keys per step
    const int lane = threadIdx.x & 31;
    const int my_u = lane / GP, my_g = lane % GP;  // the (key, walk) this lane ends with
    const long long gw = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const long long nw = ((long long)gridDim.x * blockDim.x) >> 5;
    const long long keys_per_item = (long long)U * DENSE_STEPS;
    const long long per_tree = (a.N + keys_per_item - 1) / keys_per_item;
    const long long items = per_tree * a.T;
    const T *Kb = static_cast<const T *>(a.K);
    for (long long it = gw; it < items; it += nw) {
        const int t = (int)(it / per_tree);
        const long long k0 = (it - (long long)t * per_tree) * keys_per_item;
        float q[GP][EPL];
#pragma unroll
        for (int g = 0; g < GP; ++g)
#pragma unroll
            for (int e = 0; e < EPL; ++e)
                q[g][e] = g < a.G ? __ldg(a.qf + ((long long)t * a.G + g) * D + lane * EPL + e) : 0.f;
        const T *Kt = Kb + (long long)t * a.cap * D + lane * EPL;
#pragma unroll 2
        for (int st = 0; st < DENSE_STEPS; ++st) {
            const long long kb = k0 + (long long)st * U;
            if (kb >= a.N) break;
            float part[32];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const long long key = kb + u < a.N ? kb + u : a.N - 1;
                float k[EPL];
                load_slice<T, EPL>(Kt + key * D, k);
#pragma unroll
                for (int g = 0; g < GP; ++g) {
                    float s = 0.f;
#pragma unroll
                    for (int e = 0; e < EPL; ++e) s = fmaf(k[e], q[g][e], s);
                    part[u * GP + g] = s;
                }
            }
            const float dot = transpose_reduce<32>(part, lane);
            const long long key = kb + my_u;
            if (my_g < a.G && key < a.N) a.S[((long long)t * a.G + my_g) * a.N + key] = a.beta * dot;
        }
    }
}

template <typename T, int D, int GP>
cudaError_t launch_dense_score(const zha_tree *t, const DenseArgs &a, cudaStream_t st) {
    static int per_sm = 0;
    if (!per_sm) {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, dense_score_kernel<T, D, GP>, 256, 0) != cudaSuccess ||
            per_sm < 1)
            per_sm = 1;
    }
    const long long keys_per_item = (32 / GP) * DENSE_STEPS;
    const long long items = (long long)a.T * ((a.N + keys_per_item - 1) / keys_per_item);
    long long blocks = (items + 7) / 8;
    const long long cap = (long long)num_sms() * per_sm;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) return cudaSuccess;
    Probe pr(t, ZHA_K_SCORE, st);
    dense_score_kernel<T, D, GP><<<(unsigned)blocks, 256, 0, st>>>(a);
    return cudaGetLastError();
}

template <typename T, int D>
cudaError_t dense_score_g(const zha_tree *t, const DenseArgs &a, cudaStream_t st) {
    if (a.G <= 1) return launch_dense_score<T, D, 1>(t, a, st);
    if (a.G <= 2) return launch_dense_score<T, D, 2>(t, a, st);
    if (a.G <= 4) return launch_dense_score<T, D, 4>(t, a, st);
    if (a.G <= 8) return launch_dense_score<T, D, 8>(t, a, st);
    if (a.G <= 16) return launch_dense_score<T, D, 16>(t, a, st);
    return launch_dense_score<T, D, 32>(t, a, st);
}

// S[w][c] of the chunk-mass profile: log sum_j exp(s_j) over the keys
// c*group .. min(c*group + group, N) - 1 of the walk's dense scores (fp32).
__global__ void chunk_lse_kernel(const float *S, long long N, int group, long long nch, long long W, float *Sc) {
    chain_start();
    const long long total = W * nch;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const long long w = i / nch, c = i - w * nch;
        const float *row = S + w * N + c * group;
        const int cnt = (int)(N - c * group < group ? N - c * group : group);
        float m = -INFINITY;
        for (int j = 0; j < cnt; ++j) m = fmaxf(m, row[j]);
        float sum = 0.f;
        for (int j = 0; j < cnt; ++j) sum += expf(row[j] - m);
        Sc[i] = m + logf(sum);
    }
    chain_done();
}

// Queries to fp32, then every key's score for every walk of its tree into S.
cudaError_t dense_scores(const zha_tree *t, const void *Q, zha_dtype q_dtype, int G, long long W, float *qf,
                         float *S, cudaStream_t st) {
    const zha_config &c = t->cfg;
    const long long nq = W * c.d;
    {
        Probe pr(t, ZHA_K_SEARCH_INIT, st);
        convert_queries_kernel<<<(unsigned)std::min<long long>((nq + 255) / 256, 4096), 256, 0, st>>>(
            Q, q_dtype == ZHA_BF16, nq, qf);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    DenseArgs a{};
    a.K = t->K;
    a.cap = c.capacity;
    a.N = t->n;
    a.T = t->T;
    a.G = G;
    a.beta = c.sharpness;
    a.qf = qf;
    a.S = S;
    if (a.N <= 0) return cudaSuccess;
    const bool bf = c.kv_dtype == ZHA_BF16;
    switch (c.d) {
        case 64: return bf ? dense_score_g<__nv_bfloat16, 64>(t, a, st) : dense_score_g<float, 64>(t, a, st);
        case 128: return bf ? dense_score_g<__nv_bfloat16, 128>(t, a, st) : dense_score_g<float, 128>(t, a, st);
        default: return bf ? dense_score_g<__nv_bfloat16, 256>(t, a, st) : dense_score_g<float, 256>(t, a, st);
    }
}

}  // namespace

cudaError_t launch_dense_scores(const zha_tree *t, const void *Q, zha_dtype q_dtype, int G, long long W, float *qf,
                                float *S, cudaStream_t st) {
    return dense_scores(t, Q, q_dtype, G, W, qf, S, st);
}

cudaError_t launch_chunk_lse(const zha_tree *t, const float *S, long long N, int group, long long nch, long long W,
                             float *Sc, cudaStream_t st) {
    if (nch <= 0 || W <= 0) return cudaSuccess;
    Probe pr(t, ZHA_K_SCORE, st);
    const long long total = W * nch;
    const long long blocks = std::min<long long>((total + 255) / 256, 8LL * num_sms());
    launch_chained(chunk_lse_kernel, dim3((unsigned)blocks), dim3(256), 0, st, S, N, group, nch, W, Sc);
    return cudaGetLastError();
}

cudaError_t launch_chunk_mass(const zha_tree *t, const void *Q, zha_dtype q_dtype, int G, long long W, int group,
                              float p, int *sel, int *count, int max_sel, float *qf, float *S, float *Sc,
                              uint32_t *gkey, cudaStream_t st) {
    cudaError_t e = dense_scores(t, Q, q_dtype, G, W, qf, S, st);
    if (e != cudaSuccess) return e;
    const long long N = t->n;
    const long long nch = (N + group - 1) / group;
    if (nch > 0) {
        Probe pr(t, ZHA_K_SCORE, st);
        const long long total = W * nch;
        const long long blocks = std::min<long long>((total + 255) / 256, 8LL * num_sms());
        launch_chained(chunk_lse_kernel, dim3((unsigned)blocks), dim3(256), 0, st, (const float *)S, N, group,
                       nch, W, Sc);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return launch_select_all(t, Sc, gkey, nch, W, G, ZHA_TOP_P, p, 0, sel, count, max_sel, st);
}

cudaError_t launch_dense_scan(const zha_tree *t, const void *Q, zha_dtype q_dtype, int G, long long W, int mode,
                              float p, int k, int *sel, int *sel_count, int max_sel, float *qf, float *S,
                              uint32_t *gkey, cudaStream_t st) {
    cudaError_t e = dense_scores(t, Q, q_dtype, G, W, qf, S, st);
    if (e != cudaSuccess) return e;
    return launch_select_all(t, S, gkey, t->n, W, G, mode, p, k, sel, sel_count, max_sel, st);
}

}  // namespace zha
