// Tree construction: node summaries and the append path.
//
// Page "How does a tree of summaries search a context? How ZHA works",
// section "What does a node summarize?": for every reference query q_r a node
// keeps one tangent of its region's log-sum-exp attention. With child scores
// s_i = beta * <key_{i,r}, q_r> + bias_{i,r} (bias 0 and key_{i,r} = k_i for
// keys), the node stores key_r = sum_i softmax(s)_i key_{i,r} and
// bias_r = logsumexp(s) - beta * <key_r, q_r>. Section "How is the tree built?":
// node j of level l covers nodes C*j .. C*j+C-1 of level l-1, and a node is made
// when its chunk fills.
//
// Mapping: one warp per (node, reference); a block holds the R warps of one
// node, so the level-1 children (the keys, shared by every reference) are read
// from HBM once and then from L1. Lane l owns D/32 consecutive columns. The
// per-child partial dot products are exchanged through shared memory (a
// [child][lane] tile), summed by the lane that owns the child, and the softmax
// weights are broadcast back for the weighted key sum. All arithmetic is fp32.
#include "zha_internal.cuh"

namespace zha {
namespace {

struct BuildArgs {
    const void *child;        // level 1: K; else the level-(l-1) nodes
    long long child_tree;     // elements per tree in `child`
    long long child_stride;   // elements between consecutive children
    long long child_ref;      // elements between the rows of two references (0 for keys)
    long long child_bias;     // offset of the bias of reference 0 inside a child (-1: none)
    const float *refs;        // [H_kv][R][D]
    float *out;               // level-l nodes
    long long out_tree;       // floats per tree in `out`
    int NF, R, C, H_kv;
    float beta;
    long long j0, per_tree;   // nodes [j0, j0 + per_tree) of every tree
    long long items;          // T * per_tree
};

template <typename CT, int D>
__global__ void __launch_bounds__(512) build_nodes_kernel(BuildArgs a) {
    chain_start();
    constexpr int EPL = D / 32;
    extern __shared__ float smem[];
    const int lane = threadIdx.x & 31;
    const int r = threadIdx.x >> 5;  // reference handled by this warp
    float *part = smem + r * (a.C * 33 + a.C);  // [C][33] partial dots
    float *wts = part + a.C * 33;                 // [C] scores, then weights
    const CT *child_base = static_cast<const CT *>(a.child);

    for (long long item = blockIdx.x; item < a.items; item += gridDim.x) {
        const long long t = item / a.per_tree;
        const long long j = a.j0 + item % a.per_tree;
        const int h = (int)(t % a.H_kv);

        float q[EPL];
        load_cached<EPL>(a.refs + ((long long)h * a.R + r) * D + lane * EPL, q);

        // child i's row for this reference: first + i * child_stride
        const CT *children = child_base + t * a.child_tree + j * a.C * a.child_stride;
        const CT *first = children + r * a.child_ref;

        // child scores: lane-local partial dots, exchanged through shared memory
        for (int i = 0; i < a.C; ++i) {
            float c[EPL];
            load_cached<EPL>(first + i * a.child_stride + lane * EPL, c);
            float p = 0.f;
#pragma unroll
            for (int e = 0; e < EPL; ++e) p = fmaf(c[e], q[e], p);
            part[i * 33 + lane] = p;
        }
        __syncwarp();
        for (int i = lane; i < a.C; i += 32) {
            float s = 0.f;
#pragma unroll 8
            for (int l = 0; l < 32; ++l) s += part[i * 33 + l];
            float b = 0.f;
            if (a.child_bias >= 0) b = to_float(children[i * a.child_stride + a.child_bias + r]);
            wts[i] = a.beta * s + b;
        }
        __syncwarp();

        // softmax over the children and the log-sum-exp
        float m = -INFINITY;
        for (int i = lane; i < a.C; i += 32) m = fmaxf(m, wts[i]);
        m = warp_max(m);
        float z = 0.f;
        for (int i = lane; i < a.C; i += 32) z += expf(wts[i] - m);
        z = warp_sum(z);
        const float lse = m + logf(z);
        __syncwarp();
        for (int i = lane; i < a.C; i += 32) wts[i] = expf(wts[i] - m) / z;
        __syncwarp();

        // key_r = sum_i w_i key_{i,r}
        float acc[EPL];
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc[e] = 0.f;
        for (int i = 0; i < a.C; ++i) {
            const float w = wts[i];
            float c[EPL];
            load_cached<EPL>(first + i * a.child_stride + lane * EPL, c);
#pragma unroll
            for (int e = 0; e < EPL; ++e) acc[e] = fmaf(w, c[e], acc[e]);
        }
        float *node = a.out + t * a.out_tree + j * a.NF;
        float dq = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e) {
            node[r * D + lane * EPL + e] = acc[e];
            dq = fmaf(acc[e], q[e], dq);
        }
        dq = warp_sum(dq);
        if (lane == 0) node[a.R * D + r] = lse - a.beta * dq;
        __syncwarp();
    }
    chain_done();
}

template <typename CT, int D>
cudaError_t launch_build_typed(const zha_tree *t, const BuildArgs &a, cudaStream_t st) {
    const int threads = 32 * a.R;
    const size_t smem = (size_t)a.R * (a.C * 33 + a.C) * sizeof(float);
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(build_nodes_kernel<CT, D>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    long long blocks = a.items;
    const long long cap = (long long)num_sms() * 16;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) return cudaSuccess;
    Probe pr(t, ZHA_K_BUILD, st);
    return launch_chained(build_nodes_kernel<CT, D>, dim3((unsigned)blocks), dim3(threads), smem, st, a);
}

template <typename T, int D>
__global__ void append_kv_kernel(T *K, T *V, const T *k_new, const T *v_new, long long cap,
                                 long long n) {
    chain_start();
    const int t = blockIdx.x;
    for (int e = threadIdx.x; e < D; e += blockDim.x) {
        K[((long long)t * cap + n) * D + e] = k_new[(long long)t * D + e];
        V[((long long)t * cap + n) * D + e] = v_new[(long long)t * D + e];
    }
    chain_done();
}

}  // namespace

cudaError_t launch_build_level(const zha_tree *t, int level, long long j0, long long j1,
                               cudaStream_t st) {
    if (j1 <= j0) return cudaSuccess;
    const zha_config &c = t->cfg;
    BuildArgs a{};
    a.refs = t->refs;
    a.out = t->nodes[level];
    a.out_tree = t->cap_nodes[level] * t->NF;
    a.NF = t->NF;
    a.R = c.R;
    a.C = c.chunk;
    a.H_kv = c.n_kv_heads;
    a.beta = c.sharpness;
    a.j0 = j0;
    a.per_tree = j1 - j0;
    a.items = (long long)t->T * a.per_tree;
    const bool keys = level == 1;
    if (keys) {
        a.child = t->K;
        a.child_tree = c.capacity * c.d;
        a.child_stride = c.d;
        a.child_ref = 0;
        a.child_bias = -1;
    } else {
        a.child = t->nodes[level - 1];
        a.child_tree = t->cap_nodes[level - 1] * t->NF;
        a.child_stride = t->NF;
        a.child_ref = c.d;
        a.child_bias = (long long)c.R * c.d;
    }
    const bool bf = keys && c.kv_dtype == ZHA_BF16;
    switch (c.d) {
        case 64:
            return bf ? launch_build_typed<__nv_bfloat16, 64>(t, a, st) : launch_build_typed<float, 64>(t, a, st);
        case 128:
            return bf ? launch_build_typed<__nv_bfloat16, 128>(t, a, st) : launch_build_typed<float, 128>(t, a, st);
        case 256:
            return bf ? launch_build_typed<__nv_bfloat16, 256>(t, a, st) : launch_build_typed<float, 256>(t, a, st);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_append_kv(const zha_tree *t, const void *k_new, const void *v_new, cudaStream_t st) {
    const zha_config &c = t->cfg;
    const int threads = c.d < 256 ? c.d : 256;
    Probe pr(t, ZHA_K_APPEND, st);
    cudaError_t e = cudaSuccess;
#define ZHA_APPEND(TY, DD)                                                                              \
    e = launch_chained(append_kv_kernel<TY, DD>, dim3(t->T), dim3(threads), 0, st, (TY *)t->K, (TY *)t->V, \
                       (const TY *)k_new, (const TY *)v_new, c.capacity, t->n)
    if (c.kv_dtype == ZHA_BF16) {
        if (c.d == 64) ZHA_APPEND(__nv_bfloat16, 64);
        else if (c.d == 128) ZHA_APPEND(__nv_bfloat16, 128);
        else ZHA_APPEND(__nv_bfloat16, 256);
    } else {
        if (c.d == 64) ZHA_APPEND(float, 64);
        else if (c.d == 128) ZHA_APPEND(float, 128);
        else ZHA_APPEND(float, 256);
    }
#undef ZHA_APPEND
    return e;
}

}  // namespace zha
