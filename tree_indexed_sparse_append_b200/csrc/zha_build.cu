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
// Mapping (all arithmetic fp32; the softmax is taken online over batches of
// children, so a node's children are read once):
//   build_leaf_batch_kernel  level 1 (C a power of two up to 32, R <= 8): a warp
//                       per batch of 32 keys, lane i scoring key i whole against
//                       references broadcast from shared memory, then lanes
//                       summing column slices of the weighted keys (described
//                       at the kernel).
//   build_leaf_kernel   level 1 otherwise: a warp per node (a contiguous run of
//                       nodes per warp), its references RPW at a time (4 at
//                       D = 128). Lane
//                       l owns D/32 consecutive columns of each key; the node's
//                       keys are loaded together (all loads in flight at once)
//                       and kept for every reference group, each key's RPW dot
//                       products are summed across the warp by one
//                       transpose-reduce, and every lane then takes the weights
//                       of the group's references by shuffles to accumulate
//                       their weighted keys in registers.
//   build_upper_kernel  levels >= 2: one warp per (node, reference), reading
//                       row r of each child (consecutive warps take the rows of
//                       one node, so the node is written row after row); the
//                       batch's child rows are loaded together, their dot
//                       products summed by one transpose-reduce and shuffled to
//                       every lane.
//   build_nodes_kernel  the earlier general kernel, kept as a fallback for an
//                       unexpected head dimension: a block of R warps per node,
//                       partial dot products exchanged through shared memory.
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

// D/32 consecutive fp32 reference columns of one lane (16-byte or 8-byte loads,
// through L1: every warp of a head reads the same rows).
template <int EPL>
__device__ __forceinline__ void load_ref(const float *p, float (&v)[EPL]) {
    if constexpr (EPL == 2) {
        const float2 x = __ldg(reinterpret_cast<const float2 *>(p));
        v[0] = x.x;
        v[1] = x.y;
    } else {
#pragma unroll
        for (int e = 0; e < EPL; e += 4) {
            const float4 x = __ldg(reinterpret_cast<const float4 *>(p + e));
            v[e] = x.x;
            v[e + 1] = x.y;
            v[e + 2] = x.z;
            v[e + 3] = x.w;
        }
    }
}

// The summaries of references r0 .. r0 + RPW - 1 of one level-1 node (keys at
// `keys`, this lane's columns). With have_keys the node's C <= KB keys are in kf
// already; otherwise they are loaded KB at a time into kf and the softmax is
// taken online over the batches.
template <typename KT, int D, int RPW, int KB>
__device__ __forceinline__ void leaf_group(const BuildArgs &a, const KT *keys, const float *refs_h, int r0,
                                           float *node, int lane, float (&kf)[KB][D / 32], bool have_keys) {
    constexpr int EPL = D / 32;
    constexpr int LG = ilog2(RPW);
    const int rr = lane >> (5 - LG);  // reference (of this group) whose sums this lane ends with
    float q[RPW][EPL];
#pragma unroll
    for (int r = 0; r < RPW; ++r) {
        if (r0 + r < a.R) {
            load_ref<EPL>(refs_h + (long long)(r0 + r) * D + lane * EPL, q[r]);
        } else {
#pragma unroll
            for (int e = 0; e < EPL; ++e) q[r][e] = 0.f;
        }
    }
    float m = -INFINITY, z = 0.f;  // running max and sum of exp, of reference r0 + rr
    float acc[RPW][EPL];
#pragma unroll
    for (int r = 0; r < RPW; ++r)
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc[r][e] = 0.f;

    for (int i0 = 0; i0 < a.C; i0 += KB) {
        if (!have_keys) {
#pragma unroll
            for (int i = 0; i < KB; ++i) {
                if (i0 + i < a.C) {
                    load_cached<EPL>(keys + (long long)(i0 + i) * D, kf[i]);
                } else {
#pragma unroll
                    for (int e = 0; e < EPL; ++e) kf[i][e] = 0.f;
                }
            }
        }
        // s[i]: beta <k_i, q_rr> (lanes of reference rr)
        float s[KB];
#pragma unroll
        for (int i = 0; i < KB; ++i) {
            float part[RPW];
#pragma unroll
            for (int r = 0; r < RPW; ++r) {
                float x = 0.f;
#pragma unroll
                for (int e = 0; e < EPL; ++e) x = fmaf(kf[i][e], q[r][e], x);
                part[r] = x;
            }
            const float dot = transpose_reduce<RPW>(part, lane);
            s[i] = i0 + i < a.C ? a.beta * dot : -INFINITY;
        }
        float bm = m;
#pragma unroll
        for (int i = 0; i < KB; ++i) bm = fmaxf(bm, s[i]);
        const float scale = expf(m - bm);  // 0 on the first batch (m = -inf)
        z *= scale;
        float wt[KB];
#pragma unroll
        for (int i = 0; i < KB; ++i) {
            wt[i] = expf(s[i] - bm);
            z += wt[i];
        }
        m = bm;
        // every lane takes each reference's scale and weights from that
        // reference's lanes and accumulates its columns of the RPW sums
#pragma unroll
        for (int r = 0; r < RPW; ++r) {
            const int src = r << (5 - LG);
            const float sc = __shfl_sync(FULL, scale, src);
#pragma unroll
            for (int e = 0; e < EPL; ++e) acc[r][e] *= sc;
#pragma unroll
            for (int i = 0; i < KB; ++i) {
                const float w = __shfl_sync(FULL, wt[i], src);
#pragma unroll
                for (int e = 0; e < EPL; ++e) acc[r][e] = fmaf(w, kf[i][e], acc[r][e]);
            }
        }
    }
    // key_r = acc_r / z_r; bias_r = m_r + log z_r - beta <key_r, q_r>
    float part[RPW];
#pragma unroll
    for (int r = 0; r < RPW; ++r) {
        const float inv = 1.f / __shfl_sync(FULL, z, r << (5 - LG));
        float x = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e) {
            acc[r][e] *= inv;
            x = fmaf(acc[r][e], q[r][e], x);
        }
        part[r] = x;
        if (r0 + r < a.R) {
            float *row = node + (r0 + r) * D + lane * EPL;
            if constexpr (EPL % 4 == 0) {
#pragma unroll
                for (int e = 0; e < EPL; e += 4)
                    *reinterpret_cast<float4 *>(row + e) = make_float4(acc[r][e], acc[r][e + 1], acc[r][e + 2],
                                                                       acc[r][e + 3]);
            } else {
                *reinterpret_cast<float2 *>(row) = make_float2(acc[r][0], acc[r][1]);
            }
        }
    }
    const float dq = transpose_reduce<RPW>(part, lane);
    if (r0 + rr < a.R && (lane & ((32 >> LG) - 1)) == 0) node[a.R * D + r0 + rr] = m + logf(z) - a.beta * dq;
}

// Level-1 nodes, one warp per node: each warp takes a contiguous run of the
// nodes (tree-major), and for each one the R references RPW at a time (RPW a
// power of two; rows past R are zero and unused). A node of C <= KB keys loads
// them once for all its reference groups (KB * D / 32 registers of keys per
// lane: 32, or 16 at D = 64); larger chunks load them KB at a time per group.
template <typename KT, int D, int RPW>
__global__ void __launch_bounds__(256, 2) build_leaf_kernel(BuildArgs a) {
    chain_start();
    constexpr int EPL = D / 32;
    constexpr int KB = 32 / EPL < 8 ? 32 / EPL : 8;  // keys per batch
    const int lane = threadIdx.x & 31;
    const long long gw = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const long long nw = ((long long)gridDim.x * blockDim.x) >> 5;
    const KT *K = static_cast<const KT *>(a.child);
    const long long per_warp = (a.items + nw - 1) / nw;
    long long item = gw * per_warp;
    const long long item_end = item + per_warp < a.items ? item + per_warp : a.items;
    if (item < item_end) {
        long long t = item / a.per_tree;
        long long jj = item - t * a.per_tree;  // node of tree t, counted from j0
        int h = (int)(t % a.H_kv);
        const bool have_keys = a.C <= KB;
        for (; item < item_end; ++item) {
            const long long j = a.j0 + jj;
            const KT *keys = K + t * a.child_tree + j * a.C * (long long)D + lane * EPL;
            const float *refs_h = a.refs + (long long)h * a.R * D;
            float *node = a.out + t * a.out_tree + j * a.NF;
            float kf[KB][EPL];
            if (have_keys) {
#pragma unroll
                for (int i = 0; i < KB; ++i) {
                    if (i < a.C) {
                        load_cached<EPL>(keys + (long long)i * D, kf[i]);
                    } else {
#pragma unroll
                        for (int e = 0; e < EPL; ++e) kf[i][e] = 0.f;
                    }
                }
            }
            for (int r0 = 0; r0 < a.R; r0 += RPW)
                leaf_group<KT, D, RPW, KB>(a, keys, refs_h, r0, node, lane, kf, have_keys);
            if (++jj == a.per_tree) {
                jj = 0;
                ++t;
                h = h + 1 == a.H_kv ? 0 : h + 1;
            }
        }
    }
    chain_done();
}

// Eight consecutive key elements from shared memory as floats (one 16-byte load
// for bf16, two for fp32).
template <typename KT>
__device__ __forceinline__ void lds8(const char *p, float (&v)[8]);
template <>
__device__ __forceinline__ void lds8<__nv_bfloat16>(const char *p, float (&v)[8]) {
    const uint4 u = *reinterpret_cast<const uint4 *>(p);
    const unsigned w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}
template <>
__device__ __forceinline__ void lds8<float>(const char *p, float (&v)[8]) {
    const float4 a = *reinterpret_cast<const float4 *>(p);
    const float4 b = *reinterpret_cast<const float4 *>(p + 16);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

constexpr int LEAF_RP = 8;  // references per pass of the batch kernel (R <= 8)

// Shared memory of one warp of build_leaf_batch_kernel: the batch's 32 key rows
// (padded by 16 bytes), the references transposed ([D][8] fp32) and the weights
// ([32 keys][8] fp32).
template <typename KT, int D>
struct LeafSmem {
    static constexpr int ROW = D * (int)sizeof(KT) + 16;
    static constexpr int KEYS = 32 * ROW;
    static constexpr int REFS = D * LEAF_RP * 4;
    static constexpr int WTS = 32 * LEAF_RP * 4;
    static constexpr int BYTES = KEYS + REFS + WTS;
};

// Level-1 nodes, one warp per batch of 32 consecutive keys: 32 / C nodes of one
// tree (C a power of two, 2..32; R <= 8). Each warp takes a contiguous run of the
// batches (tree-major).
//   1. The batch's keys are copied to the warp's shared memory with coalesced
//      16-byte loads (rows padded by 16 bytes, so lanes reading different rows
//      use different banks).
//   2. Lane i takes key i whole: its 8 dot products with the references (kept
//      transposed in shared memory and read by broadcast) need no reduction across
//      lanes. The softmax and log-sum-exp over a node's children are taken across
//      the C lanes of its keys (xor shuffles inside the group).
//   3. Lane l then takes 8 columns of one node (D / 8 lanes per node) and sums the
//      node's weighted keys for all 8 references from the staged rows.
// With key_r = sum_i w_i k_i, beta <key_r, q_r> = sum_i w_i s_i, so
// bias_r = lse_r - sum_i w_i s_i = sum_i w_i (log z_r - (s_i - m_r)) (m_r the
// largest score, z_r the sum of exp(s_i - m_r)): no second dot product, and no
// difference of two large terms.
template <typename KT, int D>
__global__ void __launch_bounds__(256) build_leaf_batch_kernel(BuildArgs a) {
    chain_start();
    using SM = LeafSmem<KT, D>;
    constexpr int PPR = D * (int)sizeof(KT) / 16;  // 16-byte pieces per key row
    constexpr int LPN = D / 8;                      // lanes per node in step 3
    constexpr int NPP = 32 / LPN > 0 ? 32 / LPN : 1;
    static_assert(LPN <= 32, "D <= 256");
    extern __shared__ __align__(16) char leaf_smem[];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    char *s_keys = leaf_smem + (size_t)wid * SM::BYTES;
    float *s_ref = reinterpret_cast<float *>(s_keys + SM::KEYS);
    float *s_w = s_ref + D * LEAF_RP;

    const int C = a.C, NPW = 32 / a.C;
    const long long bpt = (a.per_tree + NPW - 1) / NPW;  // batches per tree
    const long long batches = (a.items / a.per_tree) * bpt;
    const long long gw = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const long long nw = ((long long)gridDim.x * blockDim.x) >> 5;
    const long long per_warp = (batches + nw - 1) / nw;
    long long b = gw * per_warp;
    const long long b_end = b + per_warp < batches ? b + per_warp : batches;
    const KT *K = static_cast<const KT *>(a.child);
    int cur_h = -1;
    for (; b < b_end; ++b) {
        const long long t = b / bpt, bj = b - t * bpt;
        const int h = (int)(t % a.H_kv);
        const long long j = a.j0 + bj * NPW;  // first node of the batch
        const long long left = a.per_tree - bj * NPW;
        const int nb = left < NPW ? (int)left : NPW;  // nodes in the batch
        const int nk = nb * C;

        __syncwarp();  // the previous batch's rows and weights are no longer read
        if (h != cur_h) {
            const float *q = a.refs + (long long)h * a.R * D;
            for (int idx = lane; idx < LEAF_RP * D; idx += 32) {
                const int r = idx / D, c = idx - r * D;
                s_ref[c * LEAF_RP + r] = r < a.R ? __ldg(q + idx) : 0.f;
            }
            cur_h = h;
        }
        // 1. the batch's keys, coalesced
        {
            const char *src = reinterpret_cast<const char *>(K + t * a.child_tree + j * C * (long long)D);
#pragma unroll 4
            for (int p = lane; p < 32 * PPR; p += 32) {
                const int key = p / PPR, col = p - key * PPR;
                if (key < nk) {
                    const uint4 v = ld_stream_u4(src + (size_t)p * 16);
                    *reinterpret_cast<uint4 *>(s_keys + key * SM::ROW + col * 16) = v;
                }
            }
        }
        __syncwarp();

        // 2. lane i: key i's scores against the 8 references
        float s[LEAF_RP];
#pragma unroll
        for (int r = 0; r < LEAF_RP; ++r) s[r] = 0.f;
        {
            const char *row = s_keys + lane * SM::ROW;
#pragma unroll 2
            for (int c = 0; c < D; c += 8) {
                float kf[8];
                lds8<KT>(row + c * (int)sizeof(KT), kf);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float4 q0 = *reinterpret_cast<const float4 *>(s_ref + (c + e) * LEAF_RP);
                    const float4 q1 = *reinterpret_cast<const float4 *>(s_ref + (c + e) * LEAF_RP + 4);
                    s[0] = fmaf(kf[e], q0.x, s[0]);
                    s[1] = fmaf(kf[e], q0.y, s[1]);
                    s[2] = fmaf(kf[e], q0.z, s[2]);
                    s[3] = fmaf(kf[e], q0.w, s[3]);
                    s[4] = fmaf(kf[e], q1.x, s[4]);
                    s[5] = fmaf(kf[e], q1.y, s[5]);
                    s[6] = fmaf(kf[e], q1.z, s[6]);
                    s[7] = fmaf(kf[e], q1.w, s[7]);
                }
            }
        }
        // softmax and log-sum-exp over the node's C lanes (lanes of keys past the
        // batch compute values that are never stored)
        float w[LEAF_RP], bias[LEAF_RP];
#pragma unroll
        for (int r = 0; r < LEAF_RP; ++r) {
            const float sr = a.beta * s[r];
            float m = sr;
            for (int o = C >> 1; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(FULL, m, o));
            const float e = expf(sr - m);
            float z = e;
            for (int o = C >> 1; o >= 1; o >>= 1) z += __shfl_xor_sync(FULL, z, o);
            w[r] = e / z;
            float ent = w[r] * (logf(z) - (sr - m));
            for (int o = C >> 1; o >= 1; o >>= 1) ent += __shfl_xor_sync(FULL, ent, o);
            bias[r] = ent;
        }
        *reinterpret_cast<float4 *>(s_w + lane * LEAF_RP) = make_float4(w[0], w[1], w[2], w[3]);
        *reinterpret_cast<float4 *>(s_w + lane * LEAF_RP + 4) = make_float4(w[4], w[5], w[6], w[7]);
        if ((lane & (C - 1)) == 0 && lane < nk) {
            float *node = a.out + t * a.out_tree + (j + lane / C) * a.NF;
#pragma unroll
            for (int r = 0; r < LEAF_RP; ++r)
                if (r < a.R) node[(long long)a.R * D + r] = bias[r];
        }
        __syncwarp();

        // 3. lane l: columns cs .. cs + 7 of node n, all references
        const int cs = (lane % LPN) * 8;
        for (int n = lane / LPN; n < nb; n += NPP) {
            float o[LEAF_RP][8];
#pragma unroll
            for (int r = 0; r < LEAF_RP; ++r)
#pragma unroll
                for (int e = 0; e < 8; ++e) o[r][e] = 0.f;
#pragma unroll 2
            for (int i = 0; i < C; ++i) {
                const int key = n * C + i;
                float kf[8];
                lds8<KT>(s_keys + key * SM::ROW + cs * (int)sizeof(KT), kf);
                const float4 w0 = *reinterpret_cast<const float4 *>(s_w + key * LEAF_RP);
                const float4 w1 = *reinterpret_cast<const float4 *>(s_w + key * LEAF_RP + 4);
                const float wr[LEAF_RP] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
                for (int r = 0; r < LEAF_RP; ++r)
#pragma unroll
                    for (int e = 0; e < 8; ++e) o[r][e] = fmaf(wr[r], kf[e], o[r][e]);
            }
            float *node = a.out + t * a.out_tree + (j + n) * a.NF + cs;
#pragma unroll
            for (int r = 0; r < LEAF_RP; ++r) {
                if (r < a.R) {
                    *reinterpret_cast<float4 *>(node + r * D) = make_float4(o[r][0], o[r][1], o[r][2], o[r][3]);
                    *reinterpret_cast<float4 *>(node + r * D + 4) = make_float4(o[r][4], o[r][5], o[r][6], o[r][7]);
                }
            }
        }
    }
    chain_done();
}

// Levels >= 2, one warp per (node, reference r): row r of each child, CB at a
// time (CB * D / 32 registers of rows per lane).
template <int D>
__global__ void __launch_bounds__(256, 3) build_upper_kernel(BuildArgs a) {
    chain_start();
    constexpr int EPL = D / 32;
    constexpr int CB = 32 / EPL;  // children per batch
    constexpr int LG = ilog2(CB);
    const int lane = threadIdx.x & 31;
    const long long gw = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const long long nw = ((long long)gridDim.x * blockDim.x) >> 5;
    const float *nodes = static_cast<const float *>(a.child);
    const long long witems = a.items * a.R;
    // a contiguous run of (node, reference) pairs per warp, indices advanced in step
    const long long per_warp = (witems + nw - 1) / nw;
    long long wi = gw * per_warp;
    const long long wi_end = wi + per_warp < witems ? wi + per_warp : witems;
    if (wi >= wi_end) {
        chain_done();
        return;
    }
    long long item = wi / a.R;
    int r = (int)(wi - item * a.R);
    long long t = item / a.per_tree;
    long long jj = item - t * a.per_tree;
    int h = (int)(t % a.H_kv);
    for (; wi < wi_end; ++wi) {
        const long long j = a.j0 + jj;
        float q[EPL];
        load_ref<EPL>(a.refs + ((long long)h * a.R + r) * D + lane * EPL, q);
        const float *children = nodes + t * a.child_tree + j * a.C * a.child_stride;
        float m = -INFINITY, z = 0.f, acc[EPL];
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc[e] = 0.f;
        for (int i0 = 0; i0 < a.C; i0 += CB) {
            float kf[CB][EPL];
#pragma unroll
            for (int i = 0; i < CB; ++i) {
                if (i0 + i < a.C) {
                    load_f32<EPL>(children + (long long)(i0 + i) * a.child_stride + r * D + lane * EPL, kf[i]);
                } else {
#pragma unroll
                    for (int e = 0; e < EPL; ++e) kf[i][e] = 0.f;
                }
            }
            // lane i (< CB) fetches child i's bias for reference r
            const float cb = lane < CB && i0 + lane < a.C
                                 ? __ldg(children + (long long)(i0 + lane) * a.child_stride + a.child_bias + r)
                                 : 0.f;
            float part[CB];
#pragma unroll
            for (int i = 0; i < CB; ++i) {
                float x = 0.f;
#pragma unroll
                for (int e = 0; e < EPL; ++e) x = fmaf(kf[i][e], q[e], x);
                part[i] = x;
            }
            // lane group c = lane >> (5 - LG) ends with child c's dot product
            const float dot = transpose_reduce<CB>(part, lane);
            const int c = lane >> (5 - LG);
            const float cbias = __shfl_sync(FULL, cb, c);  // every lane takes part in the shuffle
            const float sc_own = i0 + c < a.C ? fmaf(a.beta, dot, cbias) : -INFINITY;
            float s[CB];
#pragma unroll
            for (int i = 0; i < CB; ++i) s[i] = __shfl_sync(FULL, sc_own, i << (5 - LG));
            float bm = m;
#pragma unroll
            for (int i = 0; i < CB; ++i) bm = fmaxf(bm, s[i]);
            const float scale = expf(m - bm);
            z *= scale;
#pragma unroll
            for (int e = 0; e < EPL; ++e) acc[e] *= scale;
#pragma unroll
            for (int i = 0; i < CB; ++i) {
                const float w = expf(s[i] - bm);
                z += w;
#pragma unroll
                for (int e = 0; e < EPL; ++e) acc[e] = fmaf(w, kf[i][e], acc[e]);
            }
            m = bm;
        }
        float *row = a.out + t * a.out_tree + j * a.NF + r * D + lane * EPL;
        const float inv = 1.f / z;
        float x = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e) {
            acc[e] *= inv;
            x = fmaf(acc[e], q[e], x);
        }
        if constexpr (EPL % 4 == 0) {
#pragma unroll
            for (int e = 0; e < EPL; e += 4)
                *reinterpret_cast<float4 *>(row + e) = make_float4(acc[e], acc[e + 1], acc[e + 2], acc[e + 3]);
        } else {
            *reinterpret_cast<float2 *>(row) = make_float2(acc[0], acc[1]);
        }
        const float dq = warp_sum(x);
        if (lane == 0) a.out[t * a.out_tree + j * a.NF + (long long)a.R * D + r] = m + logf(z) - a.beta * dq;
        if (++r == a.R) {
            r = 0;
            if (++jj == a.per_tree) {
                jj = 0;
                ++t;
                h = h + 1 == a.H_kv ? 0 : h + 1;
            }
        }
    }
    chain_done();
}

// Blocks of the one-warp-per-item kernels: enough to give every warp several
// items, at most 16 resident blocks' worth per SM.
inline long long warp_blocks(long long warp_items) {
    long long blocks = (warp_items + 31) / 32;
    const long long cap = (long long)num_sms() * 16;
    return blocks < 1 ? 1 : (blocks > cap ? cap : blocks);
}

// Warps per block of the batch kernel, and its resident blocks per SM (computed once).
template <typename KT, int D>
struct LeafLaunch {
    int warps = 0, per_sm = 0;
    cudaError_t err = cudaSuccess;
    LeafLaunch() {
        constexpr int per_warp = LeafSmem<KT, D>::BYTES;
        warps = 8 * per_warp <= 112 * 1024 ? 8 : 4;
        const int smem = warps * per_warp;
        err = cudaFuncSetAttribute(build_leaf_batch_kernel<KT, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (err == cudaSuccess)
            err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, build_leaf_batch_kernel<KT, D>, 32 * warps,
                                                                smem);
        if (per_sm < 1) per_sm = 1;
    }
};

template <typename KT, int D>
cudaError_t launch_leaf(const zha_tree *t, const BuildArgs &a, cudaStream_t st) {
    if (a.R <= LEAF_RP && a.C >= 2 && a.C <= 32 && (a.C & (a.C - 1)) == 0) {
        static const LeafLaunch<KT, D> L;
        if (L.err != cudaSuccess) return L.err;
        const int npw = 32 / a.C;
        const long long batches = (a.items / a.per_tree) * ((a.per_tree + npw - 1) / npw);
        long long blocks = (batches + L.warps - 1) / L.warps;
        const long long cap = (long long)num_sms() * L.per_sm;
        if (blocks > cap) blocks = cap;
        if (blocks < 1) blocks = 1;
        Probe pr(t, ZHA_K_BUILD, st);
        return launch_chained(build_leaf_batch_kernel<KT, D>, dim3((unsigned)blocks), dim3(32 * L.warps),
                              (size_t)L.warps * LeafSmem<KT, D>::BYTES, st, a);
    }
    // RPW references at a time: RPW * D / 32 = 16 registers of references (fewer when R is small)
    constexpr int RPW = 16 / (D / 32);
    const dim3 grid((unsigned)warp_blocks(a.items));
    Probe pr(t, ZHA_K_BUILD, st);
    if (a.R <= 1) return launch_chained(build_leaf_kernel<KT, D, 1>, grid, dim3(256), 0, st, a);
    if (a.R <= 2 && RPW >= 4) return launch_chained(build_leaf_kernel<KT, D, 2>, grid, dim3(256), 0, st, a);
    if constexpr (RPW >= 8) {
        if (a.R <= 4) return launch_chained(build_leaf_kernel<KT, D, 4>, grid, dim3(256), 0, st, a);
    }
    return launch_chained(build_leaf_kernel<KT, D, RPW>, grid, dim3(256), 0, st, a);
}

template <int D>
cudaError_t launch_upper(const zha_tree *t, const BuildArgs &a, cudaStream_t st) {
    Probe pr(t, ZHA_K_BUILD, st);
    return launch_chained(build_upper_kernel<D>, dim3((unsigned)warp_blocks(a.items * a.R)), dim3(256), 0, st, a);
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
    if (!keys) {
        switch (c.d) {
            case 64: return launch_upper<64>(t, a, st);
            case 128: return launch_upper<128>(t, a, st);
            case 256: return launch_upper<256>(t, a, st);
        }
    } else {
        switch (c.d) {
            case 64: return bf ? launch_leaf<__nv_bfloat16, 64>(t, a, st) : launch_leaf<float, 64>(t, a, st);
            case 128: return bf ? launch_leaf<__nv_bfloat16, 128>(t, a, st) : launch_leaf<float, 128>(t, a, st);
            case 256: return bf ? launch_leaf<__nv_bfloat16, 256>(t, a, st) : launch_leaf<float, 256>(t, a, st);
        }
    }
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
