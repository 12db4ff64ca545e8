// Gradient of the split loss with respect to the reference queries.
//
// Page "How does a tree of summaries search a context? How ZHA works", section
// "Does the model have to be retrained?": the model stays frozen and only the
// reference queries are learned, by comparing how the tree splits attention with
// how the model does (KL distillation). Reading taken: at every level l the tree
// splits a query's attention as softmax_j(score_j), score_j = max_r (beta *
// <key_{j,r}, q> + bias_{j,r}); the teacher splits it as the dense attention mass
// under each node, over the keys the level covers; the loss is KL(teacher || tree)
// summed over the levels and averaged over the walks.
//
// The gradient, per level, top level first (each level's node gradients hold
// what its parents passed on before its own loss term is added):
//   teacher       the full-scan scores, then each node's log-mass (chunk
//                 log-sum-exp over its C^l keys)
//   node_scores   one warp per (tree, node): every walk's score and best reference
//   split_kl      one CTA per walk: the level's loss term and the score gradient
//                 g = (tree split - teacher split) / walks
//   node_grads    one warp per (tree, node): g to the best reference's key
//                 (g * beta * q) and bias (g)
//   build_back    one warp per (tree, node, reference), back through the node's
//                 build (s_i = beta <c_i, q_r> + b_i, w = softmax(s),
//                 key = sum_i w_i c_i, bias = logsumexp(s) - beta <key, q_r>):
//                 with Gk = G_key - beta G_bias q_r and
//                 G_s_i = w_i (<Gk, c_i> - <Gk, key> + G_bias), the reference
//                 gets beta (sum_i G_s_i c_i - G_bias key) (atomics into the
//                 [H_kv][R][d] gradient) and child i gets w_i Gk + beta G_s_i q_r
//                 on its key and G_s_i on its bias (each child has one parent,
//                 so no atomics).
// All arithmetic is fp32.
#include <algorithm>
#include <cmath>

#include "zha_internal.cuh"

namespace zha {
namespace {

template <int D>
__global__ void __launch_bounds__(256) node_scores_kernel(const float *nodes, long long cap_l, long long n_l, int T,
                                                          int G, int R, int NF, float beta, const float *qf,
                                                          float *score, unsigned char *best) {
    constexpr int EPL = D / 32;
    const int lane = threadIdx.x & 31;
    const long long gw = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const long long nw = ((long long)gridDim.x * blockDim.x) >> 5;
    for (long long it = gw; it < (long long)T * n_l; it += nw) {
        const long long t = it / n_l, j = it - t * n_l;
        const float *node = nodes + (t * cap_l + j) * NF;
        for (int g = 0; g < G; ++g) {
            const long long w = t * G + g;
            float q[EPL];
#pragma unroll
            for (int e = 0; e < EPL; ++e) q[e] = qf[w * D + lane * EPL + e];
            float bv = -INFINITY;
            int br = 0;
            for (int r = 0; r < R; ++r) {
                float s = 0.f;
#pragma unroll
                for (int e = 0; e < EPL; ++e) s = fmaf(node[r * D + lane * EPL + e], q[e], s);
                s = warp_sum(s);
                const float v = fmaf(beta, s, node[R * D + r]);
                if (v > bv) {
                    bv = v;
                    br = r;
                }
            }
            if (lane == 0) {
                score[w * n_l + j] = bv;
                best[w * n_l + j] = (unsigned char)br;
            }
        }
    }
}

__device__ __forceinline__ float block_reduce(float v, float *sh, bool is_max) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        const float y = __shfl_xor_sync(FULL, v, o);
        v = is_max ? fmaxf(v, y) : v + y;
    }
    if (lane == 0) sh[wid] = v;
    __syncthreads();
    float r = sh[0];
    for (int i = 1; i < nw; ++i) r = is_max ? fmaxf(r, sh[i]) : r + sh[i];
    __syncthreads();
    return r;
}

// One CTA per walk: logP = teacher log-masses normalised over the level, logT =
// log_softmax of the tree's scores; the loss term sum_j P (logP - logT) / W goes
// to *loss and g = (T - P) / W to grad_score.
__global__ void __launch_bounds__(256) split_kl_kernel(const float *teacher, const float *score, long long n_l,
                                                       long long W, float *grad_score, float *loss) {
    __shared__ float sh[32];
    const long long w = blockIdx.x;
    const float *tp = teacher + w * n_l;
    const float *ts = score + w * n_l;
    float mp = -INFINITY, mt = -INFINITY;
    for (long long j = threadIdx.x; j < n_l; j += blockDim.x) {
        mp = fmaxf(mp, tp[j]);
        mt = fmaxf(mt, ts[j]);
    }
    mp = block_reduce(mp, sh, true);
    mt = block_reduce(mt, sh, true);
    float sp = 0.f, st = 0.f;
    for (long long j = threadIdx.x; j < n_l; j += blockDim.x) {
        sp += expf(tp[j] - mp);
        st += expf(ts[j] - mt);
    }
    sp = block_reduce(sp, sh, false);
    st = block_reduce(st, sh, false);
    const float lp = mp + logf(sp), lt = mt + logf(st);
    float kl = 0.f;
    for (long long j = threadIdx.x; j < n_l; j += blockDim.x) {
        const float logP = tp[j] - lp, logT = ts[j] - lt;
        const float P = expf(logP), Tm = expf(logT);
        kl += P * (logP - logT);
        grad_score[w * n_l + j] = (Tm - P) / (float)W;
    }
    kl = block_reduce(kl, sh, false);
    if (threadIdx.x == 0) atomicAdd(loss, kl / (float)W);
}

// One warp per (tree, node): every walk's score gradient to the key and bias of
// its best reference (the warp owns the node's gradient rows).
template <int D>
__global__ void __launch_bounds__(256) node_grads_kernel(const float *grad_score, const unsigned char *best,
                                                         const float *qf, long long n_l, int T, int G, int R,
                                                         float beta, float *G_key, float *G_bias) {
    constexpr int EPL = D / 32;
    const int lane = threadIdx.x & 31;
    const long long gw = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const long long nw = ((long long)gridDim.x * blockDim.x) >> 5;
    for (long long it = gw; it < (long long)T * n_l; it += nw) {
        const long long t = it / n_l, j = it - t * n_l;
        for (int g = 0; g < G; ++g) {
            const long long w = t * G + g;
            const float gv = grad_score[w * n_l + j];
            const int r = best[w * n_l + j];
            float *gk = G_key + ((t * n_l + j) * R + r) * D + lane * EPL;
#pragma unroll
            for (int e = 0; e < EPL; ++e) gk[e] += beta * gv * qf[w * D + lane * EPL + e];
            if (lane == 0) G_bias[(t * n_l + j) * R + r] += gv;
            __syncwarp();
        }
    }
}

struct BackArgs {
    const void *child;       // level 1: K; else the level-(l-1) nodes
    long long child_tree;    // elements per tree in `child`
    long long child_stride;  // elements between consecutive children
    long long child_ref;     // elements between the rows of two references (0 for keys)
    long long child_bias;    // offset of the bias of reference 0 inside a child (-1: none)
    const float *nodes;      // level-l nodes [T][cap_l][NF]
    long long cap_l, n_l, n_child;
    int T, C, R, H, NF;
    float beta;
    const float *refs;       // [H][R][D]
    const float *G_key;      // [T][n_l][R][D]
    const float *G_bias;     // [T][n_l][R]
    float *Gc_key;           // [T][n_child][R][D] (level > 1), else null
    float *Gc_bias;          // [T][n_child][R]
    float *grad;             // [H][R][D]
};

template <typename CT, int D>
__global__ void __launch_bounds__(256) build_back_kernel(BackArgs a) {
    constexpr int EPL = D / 32;
    const int lane = threadIdx.x & 31;
    const long long gw = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const long long nw = ((long long)gridDim.x * blockDim.x) >> 5;
    const CT *cbase = static_cast<const CT *>(a.child);
    const long long items = (long long)a.T * a.n_l * a.R;
    for (long long it = gw; it < items; it += nw) {
        const int r = (int)(it % a.R);
        const long long tj = it / a.R;
        const long long t = tj / a.n_l, j = tj - t * a.n_l;
        const int h = (int)(t % a.H);
        float q[EPL], key[EPL], gk[EPL];
        const float *node = a.nodes + (t * a.cap_l + j) * a.NF;
        const float gb = a.G_bias[tj * a.R + r];
#pragma unroll
        for (int e = 0; e < EPL; ++e) {
            q[e] = a.refs[((long long)h * a.R + r) * D + lane * EPL + e];
            key[e] = node[r * D + lane * EPL + e];
            gk[e] = a.G_key[(tj * a.R + r) * D + lane * EPL + e] - a.beta * gb * q[e];
        }
        float dk = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e) dk = fmaf(gk[e], key[e], dk);
        dk = warp_sum(dk);
        const CT *children = cbase + t * a.child_tree + j * a.C * a.child_stride;
        // pass 1: the child scores' maximum and sum of exponentials
        float m = -INFINITY, z = 0.f;
        for (int i = 0; i < a.C; ++i) {
            const CT *c = children + i * a.child_stride + r * a.child_ref;
            float s = 0.f;
#pragma unroll
            for (int e = 0; e < EPL; ++e) s = fmaf(to_float(c[lane * EPL + e]), q[e], s);
            s = a.beta * warp_sum(s);
            if (a.child_bias >= 0)
                s += to_float(children[i * a.child_stride + a.child_bias + r]);
            const float mn = fmaxf(m, s);
            z = z * expf(m - mn) + expf(s - mn);
            m = mn;
        }
        // pass 2: weights, gradients to the reference and to the children
        float gr[EPL];
#pragma unroll
        for (int e = 0; e < EPL; ++e) gr[e] = 0.f;
        for (int i = 0; i < a.C; ++i) {
            const CT *c = children + i * a.child_stride + r * a.child_ref;
            float cv[EPL], s = 0.f, dc = 0.f;
#pragma unroll
            for (int e = 0; e < EPL; ++e) {
                cv[e] = to_float(c[lane * EPL + e]);
                s = fmaf(cv[e], q[e], s);
                dc = fmaf(gk[e], cv[e], dc);
            }
            s = a.beta * warp_sum(s);
            dc = warp_sum(dc);
            if (a.child_bias >= 0)
                s += to_float(children[i * a.child_stride + a.child_bias + r]);
            const float wi = expf(s - m) / z;
            const float gs = wi * (dc - dk + gb);
#pragma unroll
            for (int e = 0; e < EPL; ++e) gr[e] = fmaf(gs, cv[e], gr[e]);
            if (a.Gc_key) {
                const long long ci = t * a.n_child + j * a.C + i;
                float *gck = a.Gc_key + (ci * a.R + r) * D + lane * EPL;
#pragma unroll
                for (int e = 0; e < EPL; ++e) gck[e] += wi * gk[e] + a.beta * gs * q[e];
                if (lane == 0) a.Gc_bias[ci * a.R + r] += gs;
            }
        }
        float *gout = a.grad + ((long long)h * a.R + r) * D + lane * EPL;
#pragma unroll
        for (int e = 0; e < EPL; ++e) atomicAdd(gout + e, a.beta * (gr[e] - gb * key[e]));
    }
}

long long warps_grid(long long items) {
    long long blocks = (items + 7) / 8;
    const long long cap = 8LL * num_sms();
    if (blocks > cap) blocks = cap;
    return blocks < 1 ? 1 : blocks;
}

template <int D>
cudaError_t learn_d(const zha_tree *t, const void *Q, zha_dtype q_dtype, int G, long long W, float *loss, float *grad,
                    char *ws, const size_t *off, cudaStream_t st) {
    const zha_config &c = t->cfg;
    const int T = t->T, R = c.R, C = c.chunk, depth = c.depth;
    float *qf = reinterpret_cast<float *>(ws + off[0]);
    float *S = reinterpret_cast<float *>(ws + off[1]);
    float *teacher = reinterpret_cast<float *>(ws + off[2]);
    float *score = reinterpret_cast<float *>(ws + off[3]);
    unsigned char *best = reinterpret_cast<unsigned char *>(ws + off[4]);
    float *gscore = reinterpret_cast<float *>(ws + off[5]);
    float *Gk[ZHA_MAX_DEPTH + 2] = {nullptr}, *Gb[ZHA_MAX_DEPTH + 2] = {nullptr};
    size_t o = off[6];
    for (int l = 1; l <= depth; ++l) {
        Gk[l] = reinterpret_cast<float *>(ws + o);
        o += sizeof(float) * (size_t)T * t->n_nodes[l] * R * c.d;
        Gb[l] = reinterpret_cast<float *>(ws + o);
        o += sizeof(float) * (size_t)T * t->n_nodes[l] * R;
    }
    cudaError_t e = launch_dense_scores(t, Q, q_dtype, G, W, qf, S, st);
    if (e != cudaSuccess) return e;
    long long span = 1;
    for (int l = 1; l <= depth; ++l) span *= C;
    for (int l = depth; l >= 1; --l, span /= C) {
        const long long n_l = t->n_nodes[l];
        if (n_l <= 0) continue;
        e = launch_chunk_lse(t, S, t->n, (int)span, n_l, W, teacher, st);
        if (e != cudaSuccess) return e;
        node_scores_kernel<D><<<(unsigned)warps_grid((long long)T * n_l), 256, 0, st>>>(
            t->nodes[l], t->cap_nodes[l], n_l, T, G, R, t->NF, c.sharpness, qf, score, best);
        split_kl_kernel<<<(unsigned)W, 256, 0, st>>>(teacher, score, n_l, W, gscore, loss);
        node_grads_kernel<D><<<(unsigned)warps_grid((long long)T * n_l), 256, 0, st>>>(
            gscore, best, qf, n_l, T, G, R, c.sharpness, Gk[l], Gb[l]);
        BackArgs b{};
        if (l == 1) {
            b.child = t->K;
            b.child_tree = c.capacity * c.d;
            b.child_stride = c.d;
            b.child_ref = 0;
            b.child_bias = -1;
        } else {
            b.child = t->nodes[l - 1];
            b.child_tree = t->cap_nodes[l - 1] * t->NF;
            b.child_stride = t->NF;
            b.child_ref = c.d;
            b.child_bias = (long long)R * c.d;
            b.Gc_key = Gk[l - 1];
            b.Gc_bias = Gb[l - 1];
            b.n_child = t->n_nodes[l - 1];
        }
        b.nodes = t->nodes[l];
        b.cap_l = t->cap_nodes[l];
        b.n_l = n_l;
        b.T = T;
        b.C = C;
        b.R = R;
        b.H = c.n_kv_heads;
        b.NF = t->NF;
        b.beta = c.sharpness;
        b.refs = t->refs;
        b.G_key = Gk[l];
        b.G_bias = Gb[l];
        b.grad = grad;
        const unsigned blocks = (unsigned)warps_grid((long long)T * n_l * R);
        if (l == 1 && c.kv_dtype == ZHA_BF16)
            build_back_kernel<__nv_bfloat16, D><<<blocks, 256, 0, st>>>(b);
        else if (l == 1)
            build_back_kernel<float, D><<<blocks, 256, 0, st>>>(b);
        else
            build_back_kernel<float, D><<<blocks, 256, 0, st>>>(b);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace
}  // namespace zha

using zha::set_error;

extern "C" int zha_ref_grad(zha_tree *t, const void *Q, zha_dtype q_dtype, int n_q_heads, int n_q, float *loss,
                            float *grad, void *stream) {
    if (!t || !Q || !loss || !grad) return set_error(ZHA_ERR_INVALID, "tree, Q, loss and grad must not be NULL");
    if (q_dtype != ZHA_F32 && q_dtype != ZHA_BF16) return set_error(ZHA_ERR_INVALID, "q_dtype must be ZHA_F32 or ZHA_BF16");
    const zha_config &c = t->cfg;
    if (n_q_heads < 1 || n_q < 1 || n_q_heads % c.n_kv_heads)
        return set_error(ZHA_ERR_INVALID, "n_q_heads must be a positive multiple of n_kv_heads and n_q >= 1");
    const long long G = (long long)(n_q_heads / c.n_kv_heads) * n_q;
    if (G > 32) return set_error(ZHA_ERR_INVALID, "the split-loss gradient takes at most 32 walks per tree");
    const long long W = (long long)t->T * G;
    const long long N = t->n > 0 ? t->n : 1;
    const long long n1 = t->n_nodes[1] > 0 ? t->n_nodes[1] : 1;
    auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
    size_t off[7];
    size_t o = 0;
    off[0] = o; o += al(sizeof(float) * W * c.d);
    off[1] = o; o += al(sizeof(float) * W * N);
    off[2] = o; o += al(sizeof(float) * W * n1);
    off[3] = o; o += al(sizeof(float) * W * n1);
    off[4] = o; o += al((size_t)W * n1);
    off[5] = o; o += al(sizeof(float) * W * n1);
    off[6] = o;
    for (int l = 1; l <= c.depth; ++l) o += sizeof(float) * (size_t)t->T * t->n_nodes[l] * c.R * (c.d + 1);
    const size_t gbytes = o - off[6];
    o = al(o);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // the tree's second scratch block, shared with the full-scan indexer (grown
    // when too small, then reused by later calls)
    const int rc = zha::grow_dense_scratch(t, o);
    if (rc) return rc;
    char *b = static_cast<char *>(t->dws);
    cudaError_t e = cudaMemsetAsync(b + off[6], 0, gbytes, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(loss, 0, sizeof(float), st);
    if (e == cudaSuccess) e = cudaMemsetAsync(grad, 0, sizeof(float) * (size_t)c.n_kv_heads * c.R * c.d, st);
    if (e == cudaSuccess && t->n > 0) {
        switch (c.d) {
            case 64: e = zha::learn_d<64>(t, Q, q_dtype, (int)G, W, loss, grad, b, off, st); break;
            case 128: e = zha::learn_d<128>(t, Q, q_dtype, (int)G, W, loss, grad, b, off, st); break;
            default: e = zha::learn_d<256>(t, Q, q_dtype, (int)G, W, loss, grad, b, off, st); break;
        }
    }
    if (e != cudaSuccess) return set_error(ZHA_ERR_CUDA, cudaGetErrorString(e));
    return ZHA_OK;
}
