// Final sparse attention over exactly the keys a walk chose.
//
// Page "How does a tree of summaries search a context? How ZHA works",
// sections "How is the tree built?" and "Common misunderstandings": the tree
// only finds the way; ordinary attention then runs over the original keys and
// values that the walk selected. Here those are the C keys of every opened
// level-1 node plus the tail (keys not yet covered by a level-1 node), scored
// with the same scale beta as the summaries.
//
// Design (split-K decode attention, fp32 accumulation):
//   attend_plan     one CTA scans the walks' key counts into item offsets and an
//                   item -> walk map; a walk's key list is cut into at most
//                   MAX_SPLIT items of at least SEG keys.
//   attend_partial  grid-stride over items, one warp per item. The item's chunk
//                   ids are loaded once (one per lane) and broadcast by shuffle.
//                   A row of K or V is read with 16-byte loads by LPR lanes (16
//                   for d = 128 bf16), so a warp step covers 32/LPR keys, and
//                   UNROLL steps of rows are in flight before any is used; keys
//                   of one chunk are contiguous in the cache. Online softmax per
//                   lane group, merged across groups at the end; fp32 caches
//                   take their dot products in fp64.
//   attend_combine  one warp per walk merges its items by log-sum-exp.
#include <cmath>
#include <type_traits>

#include "zha_internal.cuh"

namespace zha {
namespace {

constexpr int SEG = 64;         // keys per work item, at least
constexpr int MAX_SPLIT = 128;  // work items per walk, at most
constexpr int UNROLL = 4;       // key groups whose rows are in flight together

__device__ __forceinline__ long long walk_keys(const int *sel_count, long long w, int max_sel, int C,
                                               long long tail) {
    int c = sel_count[w];
    c = c < 0 ? 0 : (c > max_sel ? max_sel : c);
    return (long long)C * c + tail;
}

__device__ __forceinline__ long long seg_len(long long L) {
    long long s = (L + MAX_SPLIT - 1) / MAX_SPLIT;
    return s > SEG ? s : SEG;
}

struct PlanArgs {
    const int *sel_count;
    int max_sel, C;
    long long tail, W;
    int *item_off;
    int *item_walk;
};

__global__ void __launch_bounds__(1024) attend_plan_kernel(PlanArgs a) {
    __shared__ long long sh[32];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    long long carry = 0;
    for (long long base = 0; base < a.W; base += blockDim.x) {
        const long long w = base + threadIdx.x;
        long long items = 0;
        if (w < a.W) {
            const long long L = walk_keys(a.sel_count, w, a.max_sel, a.C, a.tail);
            items = L > 0 ? (L + seg_len(L) - 1) / seg_len(L) : 0;
        }
        long long inc = items;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            long long y = __shfl_up_sync(FULL, inc, o);
            if (lane >= o) inc += y;
        }
        if (lane == 31) sh[wid] = inc;
        __syncthreads();
        if (wid == 0) {
            long long s = lane < (int)(blockDim.x >> 5) ? sh[lane] : 0;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                long long y = __shfl_up_sync(FULL, s, o);
                if (lane >= o) s += y;
            }
            sh[lane] = s;
        }
        __syncthreads();
        const long long excl = carry + (wid > 0 ? sh[wid - 1] : 0) + inc - items;
        if (w < a.W) {
            a.item_off[w] = (int)excl;
            for (long long i = 0; i < items; ++i) a.item_walk[excl + i] = (int)w;
        }
        carry += sh[(blockDim.x >> 5) - 1];
        __syncthreads();
    }
    if (threadIdx.x == 0) a.item_off[a.W] = (int)carry;
}

struct PartialArgs {
    const void *K, *V, *Q;
    int q_bf16;
    const int *sel, *sel_count, *item_off, *item_walk;
    int max_sel, C, G;
    long long W, cap, n1, tail;
    float beta;
    float *partial;  // [items][D + 2]: acc[D], m, l
    int *status;
};

template <typename T>
struct Row;
template <>
struct Row<__nv_bfloat16> {
    static constexpr int EPL = 8;  // elements per 16-byte load
    __device__ static void load(const __nv_bfloat16 *p, float *v) {
        uint4 u = ld_stream_u4(p);
        const unsigned w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[2 * i] = __uint_as_float(w[i] << 16);
            v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
};
template <>
struct Row<float> {
    static constexpr int EPL = 4;
    __device__ static void load(const float *p, float *v) {
        float4 u = ld_stream4(p);
        v[0] = u.x;
        v[1] = u.y;
        v[2] = u.z;
        v[3] = u.w;
    }
};

template <typename T, int D>
__global__ void __launch_bounds__(256) attend_partial_kernel(PartialArgs a) {
    constexpr int EPL = Row<T>::EPL;
    constexpr int LPR0 = D / EPL;
    constexpr int LPR = LPR0 < 32 ? LPR0 : 32;  // lanes per row
    constexpr int VPL = LPR0 / LPR;              // 16-byte loads per lane per row
    constexpr int KPW = 32 / LPR;                // keys per warp step
    constexpr int COLS = EPL * VPL;
    using Dot = typename std::conditional<sizeof(T) == 4, double, float>::type;

    const int lane = threadIdx.x & 31;
    const int grp = lane / LPR, gl = lane % LPR;
    const long long gw = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const long long nw = ((long long)gridDim.x * blockDim.x) >> 5;
    const long long total = a.item_off[a.W];
    const T *Kb = static_cast<const T *>(a.K);
    const T *Vb = static_cast<const T *>(a.V);

    for (long long item = gw; item < total; item += nw) {
        const long long walk = a.item_walk[item];
        const long long tree = walk / a.G;
        const long long L = walk_keys(a.sel_count, walk, a.max_sel, a.C, a.tail);
        const long long seg = seg_len(L);
        const long long k0 = (item - a.item_off[walk]) * seg;
        const long long k1 = k0 + seg < L ? k0 + seg : L;
        const long long nsel = L - a.tail;  // keys coming from selected chunks
        const int *wsel = a.sel + walk * a.max_sel;

        // the segment's chunk ids, one per lane, when they fit in a warp
        const long long c0 = k0 / a.C;
        const long long c1 = (k1 < nsel ? k1 : nsel) > k0 ? ((k1 < nsel ? k1 : nsel) - 1) / a.C + 1 : c0;
        const bool pre = c1 - c0 <= 32;
        int my_chunk = 0;
        if (pre && c0 + lane < c1) my_chunk = __ldg(wsel + c0 + lane);

        float q[COLS];
#pragma unroll
        for (int v = 0; v < VPL; ++v)
#pragma unroll
            for (int e = 0; e < EPL; ++e) {
                const long long idx = walk * D + (v * LPR + gl) * EPL + e;
                q[v * EPL + e] = a.q_bf16 ? __bfloat162float(static_cast<const __nv_bfloat16 *>(a.Q)[idx])
                                          : static_cast<const float *>(a.Q)[idx];
            }

        float m = -INFINITY, l = 0.f, acc[COLS];
#pragma unroll
        for (int c = 0; c < COLS; ++c) acc[c] = 0.f;

        for (long long kb = k0; kb < k1; kb += KPW * UNROLL) {
            bool valid[UNROLL];
            long long kid[UNROLL];
#pragma unroll
            for (int u = 0; u < UNROLL; ++u) {
                const long long kk = kb + u * KPW + grp;
                valid[u] = kk < k1;
                kid[u] = 0;
                int c = 0;
                if (pre) {
                    const long long src = kk < nsel ? kk / a.C - c0 : 0;
                    c = __shfl_sync(FULL, my_chunk, (int)(src & 31));
                } else if (valid[u] && kk < nsel) {
                    c = __ldg(wsel + kk / a.C);
                }
                if (valid[u]) {
                    if (kk < nsel) {
                        if (c < 0 || c >= a.n1) {
                            valid[u] = false;
                            if (gl == 0) report(a.status, DEV_BAD_INDEX);
                        } else {
                            kid[u] = (long long)c * a.C + kk % a.C;
                        }
                    } else {
                        kid[u] = a.n1 * a.C + (kk - nsel);
                    }
                }
            }
            float kf[UNROLL][COLS], vf[UNROLL][COLS];
#pragma unroll
            for (int u = 0; u < UNROLL; ++u) {
                const long long row = (tree * a.cap + kid[u]) * D;
#pragma unroll
                for (int v = 0; v < VPL; ++v) {
                    Row<T>::load(Kb + row + (v * LPR + gl) * EPL, kf[u] + v * EPL);
                    Row<T>::load(Vb + row + (v * LPR + gl) * EPL, vf[u] + v * EPL);
                }
            }
#pragma unroll
            for (int u = 0; u < UNROLL; ++u) {
                Dot d = 0;
#pragma unroll
                for (int c = 0; c < COLS; ++c) d += (Dot)kf[u][c] * (Dot)q[c];
#pragma unroll
                for (int o = LPR / 2; o >= 1; o >>= 1) d += __shfl_xor_sync(FULL, d, o);
                const float s = (float)((Dot)a.beta * d);
                if (valid[u]) {
                    const float mn = fmaxf(m, s);
                    const float scale = expf(m - mn);
                    const float pw = expf(s - mn);
                    l = l * scale + pw;
#pragma unroll
                    for (int c = 0; c < COLS; ++c) acc[c] = fmaf(pw, vf[u][c], acc[c] * scale);
                    m = mn;
                }
            }
        }
        // merge the KPW lane groups
#pragma unroll
        for (int o = LPR; o < 32; o <<= 1) {
            const float m2 = __shfl_xor_sync(FULL, m, o);
            const float l2 = __shfl_xor_sync(FULL, l, o);
            const float mn = fmaxf(m, m2);
            const float s1 = mn == -INFINITY ? 0.f : expf(m - mn);
            const float s2 = mn == -INFINITY ? 0.f : expf(m2 - mn);
#pragma unroll
            for (int c = 0; c < COLS; ++c) {
                const float a2 = __shfl_xor_sync(FULL, acc[c], o);
                acc[c] = acc[c] * s1 + a2 * s2;
            }
            l = l * s1 + l2 * s2;
            m = mn;
        }
        if (grp == 0) {
            float *out = a.partial + item * (D + 2);
#pragma unroll
            for (int v = 0; v < VPL; ++v)
#pragma unroll
                for (int e = 0; e < EPL; ++e) out[(v * LPR + gl) * EPL + e] = acc[v * EPL + e];
            if (gl == 0) {
                out[D] = m;
                out[D + 1] = l;
            }
        }
    }
}

struct CombineArgs {
    const int *item_off;
    const float *partial;
    long long W;
    void *out;
    float *lse;
};

template <typename OT, int D>
__global__ void __launch_bounds__(256) attend_combine_kernel(CombineArgs a) {
    constexpr int CPL = D / 32;
    const int lane = threadIdx.x & 31;
    const long long walk = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (walk >= a.W) return;
    const long long i0 = a.item_off[walk], i1 = a.item_off[walk + 1];
    float m = -INFINITY;
    for (long long i = i0 + lane; i < i1; i += 32) m = fmaxf(m, a.partial[i * (D + 2) + D]);
    m = warp_max(m);
    float l = 0.f;
    for (long long i = i0 + lane; i < i1; i += 32) {
        const float mi = a.partial[i * (D + 2) + D];
        if (mi != -INFINITY) l += a.partial[i * (D + 2) + D + 1] * expf(mi - m);
    }
    l = warp_sum(l);
    float o[CPL];
#pragma unroll
    for (int c = 0; c < CPL; ++c) o[c] = 0.f;
    for (long long i = i0; i < i1; ++i) {
        const float mi = a.partial[i * (D + 2) + D];
        if (mi == -INFINITY) continue;
        const float w = expf(mi - m);
#pragma unroll
        for (int c = 0; c < CPL; ++c) o[c] = fmaf(w, a.partial[i * (D + 2) + lane * CPL + c], o[c]);
    }
    const bool empty = !(l > 0.f);
    OT *out = static_cast<OT *>(a.out) + walk * D + lane * CPL;
#pragma unroll
    for (int c = 0; c < CPL; ++c) from_float(empty ? 0.f : o[c] / l, out + c);
    if (lane == 0 && a.lse) a.lse[walk] = empty ? -INFINITY : m + logf(l);
}

template <typename T, int D>
cudaError_t launch_attend_typed(const zha_tree *t, const PartialArgs &pa, const CombineArgs &ca,
                                long long max_items, bool out_bf16, cudaStream_t st) {
    long long blocks = (max_items + 7) / 8;
    const long long cap = (long long)num_sms() * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    {
        Probe pr(t, ZHA_K_ATTEND_PARTIAL, st);
        attend_partial_kernel<T, D><<<(unsigned)blocks, 256, 0, st>>>(pa);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    Probe pr(t, ZHA_K_ATTEND_COMBINE, st);
    if (out_bf16)
        attend_combine_kernel<__nv_bfloat16, D><<<(unsigned)((ca.W + 7) / 8), 256, 0, st>>>(ca);
    else
        attend_combine_kernel<float, D><<<(unsigned)((ca.W + 7) / 8), 256, 0, st>>>(ca);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attend(const zha_tree *t, const Scratch &s, const void *Q, zha_dtype q_dtype, int G,
                          long long W, const int *sel, const int *sel_count, int max_sel, void *out,
                          zha_dtype out_dtype, float *lse, cudaStream_t st) {
    const zha_config &c = t->cfg;
    PlanArgs pl{};
    pl.sel_count = sel_count;
    pl.max_sel = max_sel;
    pl.C = c.chunk;
    pl.tail = t->n - (long long)c.chunk * t->n_nodes[1];
    pl.W = W;
    pl.item_off = s.item_off;
    pl.item_walk = s.item_walk;
    {
        Probe pr(t, ZHA_K_ATTEND_PLAN, st);
        attend_plan_kernel<<<1, 1024, 0, st>>>(pl);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }

    PartialArgs pa{};
    pa.K = t->K;
    pa.V = t->V;
    pa.Q = Q;
    pa.q_bf16 = q_dtype == ZHA_BF16;
    pa.sel = sel;
    pa.sel_count = sel_count;
    pa.item_off = s.item_off;
    pa.item_walk = s.item_walk;
    pa.max_sel = max_sel;
    pa.C = c.chunk;
    pa.G = G;
    pa.W = W;
    pa.cap = c.capacity;
    pa.n1 = t->n_nodes[1];
    pa.tail = pl.tail;
    pa.beta = c.sharpness;
    pa.partial = s.partial;
    pa.status = t->d_status;
    CombineArgs ca{};
    ca.item_off = s.item_off;
    ca.partial = s.partial;
    ca.W = W;
    ca.out = out;
    ca.lse = lse;
    const bool bf = c.kv_dtype == ZHA_BF16;
    const bool ob = out_dtype == ZHA_BF16;
    switch (c.d) {
        case 64:
            return bf ? launch_attend_typed<__nv_bfloat16, 64>(t, pa, ca, s.max_items, ob, st)
                      : launch_attend_typed<float, 64>(t, pa, ca, s.max_items, ob, st);
        case 128:
            return bf ? launch_attend_typed<__nv_bfloat16, 128>(t, pa, ca, s.max_items, ob, st)
                      : launch_attend_typed<float, 128>(t, pa, ca, s.max_items, ob, st);
        default:
            return bf ? launch_attend_typed<__nv_bfloat16, 256>(t, pa, ca, s.max_items, ob, st)
                      : launch_attend_typed<float, 256>(t, pa, ca, s.max_items, ob, st);
    }
}

}  // namespace zha
