// Final sparse attention over exactly the keys a walk chose.
//
// Page "How does a tree of summaries search a context? How ZHA works",
// sections "How is the tree built?" and "Common misunderstandings": the tree
// only finds the way; ordinary attention then runs over the original keys and
// values that the walk selected. Here those are the C keys of every opened
// level-1 node plus the tail (keys not yet covered by a level-1 node), scored
// with the same scale beta as the summaries:
//   out = sum_i softmax_i(beta <q, k_i>) v_i,   lse = logsumexp_i(beta <q, k_i>).
//
// Design (split-K decode attention, fp32 accumulation, two launches):
//   attend_plan   one CTA scans the walks' key counts into item offsets and an
//                 item -> walk map; a walk's key list is cut into at most
//                 MAX_SPLIT items of at least SEG keys. Walks without keys get
//                 out = 0, lse = -inf here.
//   attend_items  grid-stride over items, one warp per item. The item's chunk
//                 ids are loaded once (one per lane) and broadcast by shuffle.
//                 A row of K or V is read with 16-byte loads by LPR lanes (16 for
//                 d = 128 bf16), so a warp step covers KPW = 32/LPR keys; U steps
//                 of K and V rows are issued before any is used, their U dot
//                 products are independent, and the online softmax takes them in
//                 one update. The warp that finishes a walk's last item (an
//                 atomic ticket after a fence; nobody waits) merges the walk's
//                 partial results by log-sum-exp and writes out and lse.
// fp32 caches take their dot products in fp64.
#include <cmath>
#include <type_traits>

#include "zha_internal.cuh"

namespace zha {
namespace {

constexpr int SEG = 128;        // keys per work item, at least
constexpr int MAX_SPLIT = 128;  // work items per walk, at most

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

template <typename OT>
__device__ __forceinline__ void store_out(OT *p, float v) {
    from_float(v, p);
}

struct PlanArgs {
    const int *sel_count;
    int max_sel, C, D, out_bf16;
    long long tail, W;
    int *item_off;
    int *item_walk;
    int *walk_done;
    void *out;
    float *lse;
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
            a.walk_done[w] = 0;
            for (long long i = 0; i < items; ++i) a.item_walk[excl + i] = (int)w;
            if (items == 0) {  // no key at all: out = 0, lse = -inf
                for (int e = 0; e < a.D; ++e) {
                    if (a.out_bf16) store_out(static_cast<__nv_bfloat16 *>(a.out) + w * a.D + e, 0.f);
                    else store_out(static_cast<float *>(a.out) + w * a.D + e, 0.f);
                }
                if (a.lse) a.lse[w] = -INFINITY;
            }
        }
        carry += sh[(blockDim.x >> 5) - 1];
        __syncthreads();
    }
    if (threadIdx.x == 0) a.item_off[a.W] = (int)carry;
}

struct ItemArgs {
    const void *K, *V, *Q;
    int q_bf16, out_bf16;
    const int *sel, *sel_count, *item_off, *item_walk;
    int *walk_done;
    int max_sel, C, G;
    int c_shift;  // log2(C) when C is a power of two, else -1
    long long W, cap, n1, tail;
    float beta;
    float *partial;  // [items][D + 2]: acc[D], m, l
    void *out;
    float *lse;
    int *status;
};

template <typename T>
struct Row;
template <>
struct Row<__nv_bfloat16> {
    static constexpr int EPL = 8;  // elements per 16-byte load
    using Raw = uint4;
    __device__ static Raw load(const __nv_bfloat16 *p) { return ld_stream_u4(p); }
    __device__ static void unpack(const Raw &u, float *v) {
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
    using Raw = float4;
    __device__ static Raw load(const float *p) { return ld_stream4(p); }
    __device__ static void unpack(const Raw &u, float *v) {
        v[0] = u.x;
        v[1] = u.y;
        v[2] = u.z;
        v[3] = u.w;
    }
};

// Merges the partial results of one walk (one warp) and writes out / lse.
template <int D>
__device__ void combine_walk(const ItemArgs &a, long long walk, int lane) {
    constexpr int CPL = D / 32;
    const long long i0 = a.item_off[walk], i1 = a.item_off[walk + 1];
    float m = -INFINITY;
    for (long long i = i0 + lane; i < i1; i += 32) m = fmaxf(m, __ldcg(a.partial + i * (D + 2) + D));
    m = warp_max(m);
    float l = 0.f;
    for (long long i = i0 + lane; i < i1; i += 32) {
        const float mi = __ldcg(a.partial + i * (D + 2) + D);
        if (mi != -INFINITY) l += __ldcg(a.partial + i * (D + 2) + D + 1) * expf(mi - m);
    }
    l = warp_sum(l);
    float o[CPL];
#pragma unroll
    for (int c = 0; c < CPL; ++c) o[c] = 0.f;
#pragma unroll 4
    for (long long i = i0; i < i1; ++i) {
        const float *pi = a.partial + i * (D + 2);
        const float mi = __ldcg(pi + D);
        float x[CPL];
#pragma unroll
        for (int c = 0; c < CPL; ++c) x[c] = __ldcg(pi + lane * CPL + c);
        const float w = mi == -INFINITY ? 0.f : expf(mi - m);
#pragma unroll
        for (int c = 0; c < CPL; ++c) o[c] = fmaf(w, x[c], o[c]);
    }
    const bool empty = !(l > 0.f);
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
        const float v = empty ? 0.f : o[c] / l;
        if (a.out_bf16) store_out(static_cast<__nv_bfloat16 *>(a.out) + walk * D + lane * CPL + c, v);
        else store_out(static_cast<float *>(a.out) + walk * D + lane * CPL + c, v);
    }
    if (lane == 0 && a.lse) a.lse[walk] = empty ? -INFINITY : m + logf(l);
}

template <typename T, int D>
__global__ void __launch_bounds__(256) attend_items_kernel(ItemArgs a) {
    constexpr int EPL = Row<T>::EPL;
    constexpr int LPR0 = D / EPL;
    constexpr int LPR = LPR0 < 32 ? LPR0 : 32;  // lanes per row
    constexpr int VPL = LPR0 / LPR;              // 16-byte loads per lane per row
    constexpr int KPW = 32 / LPR;                // keys per warp step
    constexpr int COLS = EPL * VPL;
    constexpr int U = VPL == 1 ? 8 : 4;          // steps whose rows are in flight together
    using Dot = typename std::conditional<sizeof(T) == 4, double, float>::type;
    using Raw = typename Row<T>::Raw;

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
        const long long ke = k1 < nsel ? k1 : nsel;
        const long long c0 = k0 / a.C;
        const long long c1 = ke > k0 ? (ke - 1) / a.C + 1 : c0;
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

        // key positions fit in 32 bits (at most C * (max_sel + 1) per walk)
        const T *Kt = Kb + tree * a.cap * D;
        const T *Vt = Vb + tree * a.cap * D;
        const int nsel32 = (int)nsel, k1_32 = (int)k1, c0_32 = (int)c0, C = a.C;
        const int tail0 = (int)(a.n1 * a.C);
        for (int kb = (int)k0; kb < k1_32; kb += KPW * U) {
            bool valid[U];
            int kid[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int kk = kb + u * KPW + grp;
                valid[u] = kk < k1_32;
                kid[u] = 0;
                const int ci = a.c_shift >= 0 ? kk >> a.c_shift : kk / C;
                const int co = a.c_shift >= 0 ? kk & (C - 1) : kk - ci * C;
                int c = 0;
                if (pre) {
                    c = __shfl_sync(FULL, my_chunk, (ci - c0_32) & 31);
                } else if (valid[u] && kk < nsel32) {
                    c = __ldg(wsel + ci);
                }
                if (valid[u]) {
                    if (kk < nsel32) {
                        if (c < 0 || c >= a.n1) {
                            valid[u] = false;
                            if (gl == 0) report(a.status, DEV_BAD_INDEX);
                        } else {
                            kid[u] = c * C + co;
                        }
                    } else {
                        kid[u] = tail0 + (kk - nsel32);
                    }
                }
            }
            Raw kr[U][VPL], vr[U][VPL];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const long long row = (long long)kid[u] * D;
#pragma unroll
                for (int v = 0; v < VPL; ++v) kr[u][v] = Row<T>::load(Kt + row + (v * LPR + gl) * EPL);
#pragma unroll
                for (int v = 0; v < VPL; ++v) vr[u][v] = Row<T>::load(Vt + row + (v * LPR + gl) * EPL);
            }
            float s[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                float kf[COLS];
#pragma unroll
                for (int v = 0; v < VPL; ++v) Row<T>::unpack(kr[u][v], kf + v * EPL);
                Dot d = 0;
#pragma unroll
                for (int c = 0; c < COLS; ++c) d += (Dot)kf[c] * (Dot)q[c];
#pragma unroll
                for (int o = LPR / 2; o >= 1; o >>= 1) d += __shfl_xor_sync(FULL, d, o);
                s[u] = valid[u] ? (float)((Dot)a.beta * d) : -INFINITY;
            }
            float mx = m;
#pragma unroll
            for (int u = 0; u < U; ++u) mx = fmaxf(mx, s[u]);
            if (mx != -INFINITY) {
                const float scale = expf(m - mx);
                l *= scale;
#pragma unroll
                for (int c = 0; c < COLS; ++c) acc[c] *= scale;
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const float pw = valid[u] ? expf(s[u] - mx) : 0.f;
                    float vf[COLS];
#pragma unroll
                    for (int v = 0; v < VPL; ++v) Row<T>::unpack(vr[u][v], vf + v * EPL);
                    l += pw;
#pragma unroll
                    for (int c = 0; c < COLS; ++c) acc[c] = fmaf(pw, vf[c], acc[c]);
                }
                m = mx;
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
        // the warp that completes a walk's last item merges the walk
        __threadfence();
        __syncwarp();
        int ticket = 0;
        if (lane == 0) ticket = atomicAdd(a.walk_done + walk, 1) + 1;
        ticket = __shfl_sync(FULL, ticket, 0);
        if (ticket == a.item_off[walk + 1] - a.item_off[walk]) {
            __threadfence();
            combine_walk<D>(a, walk, lane);
        }
    }
}

template <typename T, int D>
cudaError_t launch_items(const zha_tree *t, const ItemArgs &ia, long long max_items, cudaStream_t st) {
    static int per_sm = 0;
    if (!per_sm) {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, attend_items_kernel<T, D>, 256, 0) != cudaSuccess ||
            per_sm < 1)
            per_sm = 1;
    }
    long long blocks = (max_items + 7) / 8;
    const long long cap = (long long)num_sms() * per_sm;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    Probe pr(t, ZHA_K_ATTEND_PARTIAL, st);
    attend_items_kernel<T, D><<<(unsigned)blocks, 256, 0, st>>>(ia);
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
    pl.D = c.d;
    pl.out_bf16 = out_dtype == ZHA_BF16;
    pl.tail = t->n - (long long)c.chunk * t->n_nodes[1];
    pl.W = W;
    pl.item_off = s.item_off;
    pl.item_walk = s.item_walk;
    pl.walk_done = s.walk_done;
    pl.out = out;
    pl.lse = lse;
    {
        Probe pr(t, ZHA_K_ATTEND_PLAN, st);
        attend_plan_kernel<<<1, 1024, 0, st>>>(pl);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }

    ItemArgs ia{};
    ia.K = t->K;
    ia.V = t->V;
    ia.Q = Q;
    ia.q_bf16 = q_dtype == ZHA_BF16;
    ia.out_bf16 = out_dtype == ZHA_BF16;
    ia.sel = sel;
    ia.sel_count = sel_count;
    ia.item_off = s.item_off;
    ia.item_walk = s.item_walk;
    ia.walk_done = s.walk_done;
    ia.max_sel = max_sel;
    ia.C = c.chunk;
    ia.c_shift = (c.chunk & (c.chunk - 1)) == 0 ? __builtin_ctz((unsigned)c.chunk) : -1;
    ia.G = G;
    ia.W = W;
    ia.cap = c.capacity;
    ia.n1 = t->n_nodes[1];
    ia.tail = pl.tail;
    ia.beta = c.sharpness;
    ia.partial = s.partial;
    ia.out = out;
    ia.lse = lse;
    ia.status = t->d_status;
    const bool bf = c.kv_dtype == ZHA_BF16;
    switch (c.d) {
        case 64:
            return bf ? launch_items<__nv_bfloat16, 64>(t, ia, s.max_items, st)
                      : launch_items<float, 64>(t, ia, s.max_items, st);
        case 128:
            return bf ? launch_items<__nv_bfloat16, 128>(t, ia, s.max_items, st)
                      : launch_items<float, 128>(t, ia, s.max_items, st);
        default:
            return bf ? launch_items<__nv_bfloat16, 256>(t, ia, s.max_items, st)
                      : launch_items<float, 256>(t, ia, s.max_items, st);
    }
}

}  // namespace zha
