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
// Design (split-K decode attention, fp32 accumulation):
//   plan          sum the walks' key counts and set the item length from that
//                 total: small calls get about as many items as the item kernel
//                 has resident warps beyond one per walk (the per-walk rounding),
//                 so every item starts at once, with SEG_MIN..SEG_MAX keys each;
//                 no call has more than ITEM_BUDGET items (before per-walk
//                 rounding) or a walk more than MAX_SPLIT; then scan the walks'
//                 item and group counts into offsets. Walks without keys get
//                 out = 0, lse = -inf here. Calls of up to LOCAL_MAX_W walks plan
//                 inside every CTA of attend_items (shared memory; a warp finds
//                 its item's walk by binary search) after a small clear kernel
//                 zeroes the completion counters;
//                 larger calls run attend_plan (one CTA) first, which also writes
//                 an item -> walk map and clears the counters.
//   attend_items  grid-stride over items, one warp per item. The item's chunk
//                 ids come through a two-window register prefetch (32 ids per
//                 window, one per lane) and are broadcast by shuffle. A row of K
//                 or V is read with 16-byte loads by LPR lanes (16 for d = 128
//                 bf16), so a warp step covers KPW = 32/LPR keys; U steps of K
//                 and V rows are issued before any is used, their U dot products
//                 are independent, and the online softmax takes them in one
//                 update. A walk's items form groups of GROUP: the warp that
//                 finishes a group's last item (an atomic ticket after a fence;
//                 nobody waits) merges the group by log-sum-exp, and the warp
//                 that finishes a walk's last group merges the groups and writes
//                 out and lse. Merges read their rows in one or two round trips.
// fp32 caches take their dot products in fp64.
#include <cmath>
#include <type_traits>

#include "zha_internal.cuh"

namespace zha {
namespace {

constexpr int SEG_MIN = 32;          // keys per work item, at least
constexpr int SEG_MAX = 128;         // keys per item that small calls aim at, at most
constexpr int MAX_SPLIT = 512;       // work items per walk, at most
constexpr int ITEM_BUDGET = 16384;   // work items per call (before per-walk rounding)
constexpr int GROUP = 16;            // items merged together first
constexpr int LOCAL_MAX_W = 2048;    // calls of at most this many walks plan inside the item kernel

__device__ __forceinline__ long long walk_keys(const int *sel_count, long long w, int max_sel, int C,
                                               long long tail) {
    int c = sel_count[w];
    c = c < 0 ? 0 : (c > max_sel ? max_sel : c);
    return (long long)C * c + tail;
}

// Keys per item of a call of `keys` keys in all: enough items to fill `target`
// warps (SEG_MIN..SEG_MAX keys each; SEG_MAX when there is no target), and never
// more than ITEM_BUDGET items.
__device__ __forceinline__ long long item_length(long long keys, long long target) {
    long long seg = target > 0 ? (keys + target - 1) / target : SEG_MAX;
    seg = seg < SEG_MIN ? SEG_MIN : (seg > SEG_MAX ? SEG_MAX : seg);
    const long long floor_len = (keys + ITEM_BUDGET - 1) / ITEM_BUDGET;
    return seg > floor_len ? seg : floor_len;
}

// Keys per item of a walk of L keys, given the call's item length.
__device__ __forceinline__ long long seg_len(long long L, long long seg) {
    const long long s = (L + MAX_SPLIT - 1) / MAX_SPLIT;
    return s > seg ? s : seg;
}

template <typename OT>
__device__ __forceinline__ void store_out(OT *p, float v) {
    from_float(v, p);
}

struct PlanArgs {
    const int *sel_count;
    int max_sel, C, D, out_bf16;
    long long tail, W;
    long long target_items;  // resident item warps beyond one per walk (0: none)
    int *item_off;    // [W + 1]
    int *group_off;   // [W + 1]
    int *seg;         // [1] keys per item of the call (before the per-walk cap)
    int *item_walk;   // [items]
    int *walk_done;   // [W]
    int *group_done;  // [groups]
    void *out;
    float *lse;
};

// Block-wide inclusive scan of two counts (1024 threads); returns the totals.
__device__ __forceinline__ void block_scan2(long long &a, long long &b, long long *sh, long long &ta,
                                            long long &tb) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const long long ya = __shfl_up_sync(FULL, a, o), yb = __shfl_up_sync(FULL, b, o);
        if (lane >= o) {
            a += ya;
            b += yb;
        }
    }
    if (lane == 31) {
        sh[wid] = a;
        sh[32 + wid] = b;
    }
    __syncthreads();
    if (wid == 0) {
        long long x = lane < nw ? sh[lane] : 0, y = lane < nw ? sh[32 + lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const long long yx = __shfl_up_sync(FULL, x, o), yy = __shfl_up_sync(FULL, y, o);
            if (lane >= o) {
                x += yx;
                y += yy;
            }
        }
        sh[lane] = x;
        sh[32 + lane] = y;
    }
    __syncthreads();
    if (wid > 0) {
        a += sh[wid - 1];
        b += sh[32 + wid - 1];
    }
    ta = sh[nw - 1];
    tb = sh[32 + nw - 1];
    __syncthreads();
}

__global__ void __launch_bounds__(1024) attend_plan_kernel(PlanArgs a) {
    chain_start();
    __shared__ long long sh[64];
    // 1. the call's total key count sets the item length
    long long keys = 0;
    for (long long w = threadIdx.x; w < a.W; w += blockDim.x)
        keys += walk_keys(a.sel_count, w, a.max_sel, a.C, a.tail);
    {
        long long zero = 0, total = 0, unused = 0;
        block_scan2(keys, zero, sh, total, unused);
        keys = total;
    }
    long long seg = item_length(keys, a.target_items);
    if (seg > (1LL << 30)) seg = 1LL << 30;
    if (threadIdx.x == 0) a.seg[0] = (int)seg;

    // 2. items and groups per walk, scanned into offsets
    long long icarry = 0, gcarry = 0;
    for (long long base = 0; base < a.W; base += blockDim.x) {
        const long long w = base + threadIdx.x;
        long long items = 0, groups = 0;
        if (w < a.W) {
            const long long L = walk_keys(a.sel_count, w, a.max_sel, a.C, a.tail);
            const long long sw = seg_len(L, seg);
            items = L > 0 ? (L + sw - 1) / sw : 0;
            groups = (items + GROUP - 1) / GROUP;
        }
        long long iinc = items, ginc = groups, itot, gtot;
        block_scan2(iinc, ginc, sh, itot, gtot);
        if (w < a.W) {
            const long long i0 = icarry + iinc - items, g0 = gcarry + ginc - groups;
            a.item_off[w] = (int)i0;
            a.group_off[w] = (int)g0;
            a.walk_done[w] = 0;
            for (long long i = 0; i < items; ++i) a.item_walk[i0 + i] = (int)w;
            for (long long g = 0; g < groups; ++g) a.group_done[g0 + g] = 0;
            if (items == 0) {  // no key at all: out = 0, lse = -inf
                for (int e = 0; e < a.D; ++e) {
                    if (a.out_bf16) store_out(static_cast<__nv_bfloat16 *>(a.out) + w * a.D + e, 0.f);
                    else store_out(static_cast<float *>(a.out) + w * a.D + e, 0.f);
                }
                if (a.lse) a.lse[w] = -INFINITY;
            }
        }
        icarry += itot;
        gcarry += gtot;
    }
    if (threadIdx.x == 0) {
        a.item_off[a.W] = (int)icarry;
        a.group_off[a.W] = (int)gcarry;
    }
    chain_done();
}

struct ItemArgs {
    const void *K, *V, *Q;
    int q_bf16, out_bf16;
    const int *sel, *sel_count, *item_off, *group_off, *seg, *item_walk;
    int *walk_done, *group_done;
    int max_sel, C, G, D;
    int c_shift;  // log2(C) when C is a power of two, else -1
    long long W, cap, n1, tail;
    long long target_items;  // as in PlanArgs
    float beta;
    float *partial;   // [items][D + 4]: acc[D], m, l (rows 16-byte aligned)
    float *gpartial;  // [groups][D + 4]: the same, per group
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

// Loads the CPL consecutive floats of a partial row that one lane holds.
template <int CPL>
__device__ __forceinline__ void ld_cols(const float *p, float (&x)[CPL]) {
    if constexpr (CPL == 2) {
        const float2 v = __ldcg(reinterpret_cast<const float2 *>(p));
        x[0] = v.x;
        x[1] = v.y;
    } else {
#pragma unroll
        for (int c = 0; c < CPL; c += 4) {
            const float4 v = __ldcg(reinterpret_cast<const float4 *>(p + c));
            x[c] = v.x;
            x[c + 1] = v.y;
            x[c + 2] = v.z;
            x[c + 3] = v.w;
        }
    }
}

// Merges n <= 32 partial rows (acc[D], m, l; stride D + 4) by log-sum-exp, in row
// order. Lane i reads row i's (m, l); every row's acc is read before any is used
// (RB rows at a time). The merged acc columns lane*CPL .. lane*CPL + CPL - 1 come
// back in o.
template <int D>
__device__ __forceinline__ void merge_rows(const float *rows, int n, int lane, float &m, float &l,
                                           float (&o)[D / 32]) {
    constexpr int CPL = D / 32, PS = D + 4, RB = D >= 256 ? 8 : 16;
    float mi = -INFINITY, li = 0.f;
    if (lane < n) {
        mi = __ldcg(rows + lane * PS + D);
        li = __ldcg(rows + lane * PS + D + 1);
    }
    m = warp_max(mi);
    const float wi = mi == -INFINITY ? 0.f : expf(mi - m);
    l = warp_sum(wi * li);
#pragma unroll
    for (int c = 0; c < CPL; ++c) o[c] = 0.f;
    for (int i0 = 0; i0 < n; i0 += RB) {
        float x[RB][CPL];
#pragma unroll
        for (int j = 0; j < RB; ++j) {
            if (i0 + j < n) {
                ld_cols<CPL>(rows + (i0 + j) * PS + lane * CPL, x[j]);
            } else {
#pragma unroll
                for (int c = 0; c < CPL; ++c) x[j][c] = 0.f;
            }
        }
#pragma unroll
        for (int j = 0; j < RB; ++j) {
            const float w = __shfl_sync(FULL, wi, (i0 + j) & 31);
#pragma unroll
            for (int c = 0; c < CPL; ++c) o[c] = fmaf(w, x[j][c], o[c]);
        }
    }
}

// Writes a walk's normalised output (lane's columns lane*CPL ..) and lse.
template <int D>
__device__ __forceinline__ void write_out(const ItemArgs &a, long long walk, int lane, float m, float l,
                                          const float (&o)[D / 32]) {
    constexpr int CPL = D / 32;
    const bool empty = !(l > 0.f);
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
        const float v = empty ? 0.f : o[c] / l;
        if (a.out_bf16) store_out(static_cast<__nv_bfloat16 *>(a.out) + walk * D + lane * CPL + c, v);
        else store_out(static_cast<float *>(a.out) + walk * D + lane * CPL + c, v);
    }
    if (lane == 0 && a.lse) a.lse[walk] = empty ? -INFINITY : m + logf(l);
}

// The plan of attend_plan_kernel, computed by one CTA into shared memory: item
// offsets s_io[W + 1], group offsets s_go[W + 1] and key counts s_L[W] of every
// walk; returns the call's item length. Walks without keys get out = 0,
// lse = -inf from CTA 0. Used when the walks are few enough for every CTA to
// plan for itself (the counts are a few KB, read from L2).
__device__ long long local_plan(const ItemArgs &a, int *s_io, int *s_go, int *s_L) {
    __shared__ long long sh[64];
    const int W = (int)a.W, tid = threadIdx.x, nt = blockDim.x;
    const int per = (W + nt - 1) / nt, w0 = min(W, tid * per), w1 = min(W, w0 + per);
    long long keys = 0;
    for (int w = w0; w < w1; ++w) {
        const long long L = walk_keys(a.sel_count, w, a.max_sel, a.C, a.tail);
        s_L[w] = (int)L;
        keys += L;
    }
    long long zero = 0, total_keys, unused;
    block_scan2(keys, zero, sh, total_keys, unused);
    long long seg = item_length(total_keys, a.target_items);
    if (seg > (1LL << 30)) seg = 1LL << 30;
    long long ni = 0, ng = 0;
    for (int w = w0; w < w1; ++w) {
        const long long L = s_L[w], sw = seg_len(L, seg);
        const long long items = L > 0 ? (L + sw - 1) / sw : 0;
        ni += items;
        ng += (items + GROUP - 1) / GROUP;
    }
    long long ii = ni, gi = ng, ti, tg;
    block_scan2(ii, gi, sh, ti, tg);
    ii -= ni;
    gi -= ng;
    for (int w = w0; w < w1; ++w) {
        const long long L = s_L[w], sw = seg_len(L, seg);
        const long long items = L > 0 ? (L + sw - 1) / sw : 0;
        s_io[w] = (int)ii;
        s_go[w] = (int)gi;
        ii += items;
        gi += (items + GROUP - 1) / GROUP;
        if (items == 0 && blockIdx.x == 0) {
            for (int e = 0; e < a.D; ++e) {
                if (a.out_bf16) store_out(static_cast<__nv_bfloat16 *>(a.out) + (long long)w * a.D + e, 0.f);
                else store_out(static_cast<float *>(a.out) + (long long)w * a.D + e, 0.f);
            }
            if (a.lse) a.lse[w] = -INFINITY;
        }
    }
    if (tid == 0) {
        s_io[W] = (int)ti;
        s_go[W] = (int)tg;
    }
    __syncthreads();
    return seg;
}

// Walk owning `item`: the last w with s_io[w] <= item (s_io[0] = 0 <= item < s_io[W]).
__device__ __forceinline__ int find_walk(const int *s_io, int W, long long item) {
    int lo = 0, hi = W;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (s_io[mid] <= item) lo = mid;
        else hi = mid;
    }
    return lo;
}

template <typename T, int D, bool LOCAL>
__global__ void __launch_bounds__(256) attend_items_kernel(ItemArgs a) {
    chain_start();
    constexpr int EPL = Row<T>::EPL;
    constexpr int LPR0 = D / EPL;
    constexpr int LPR = LPR0 < 32 ? LPR0 : 32;  // lanes per row
    constexpr int VPL = LPR0 / LPR;              // 16-byte loads per lane per row
    constexpr int KPW = 32 / LPR;                // keys per warp step
    constexpr int COLS = EPL * VPL;
    constexpr int U = VPL == 1 ? 8 : 4;          // steps whose rows are in flight together
    constexpr int CPL = D / 32, PS = D + 4;
    static_assert(KPW * U <= 32, "one step must span fewer than 32 chunks of C >= 2 keys");
    using Dot = typename std::conditional<sizeof(T) == 4, double, float>::type;
    using Raw = typename Row<T>::Raw;

    const int lane = threadIdx.x & 31;
    const int grp = lane / LPR, gl = lane % LPR;
    const long long gw = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const long long nw = ((long long)gridDim.x * blockDim.x) >> 5;
    extern __shared__ int s_plan[];  // LOCAL: item offsets [W + 1], group offsets [W + 1], keys [W]
    const int *item_off = a.item_off, *group_off = a.group_off;
    const int *s_L = s_plan + 2 * (a.W + 1);
    long long seg;
    if constexpr (LOCAL) {
        seg = local_plan(a, s_plan, s_plan + (a.W + 1), s_plan + 2 * (a.W + 1));
        item_off = s_plan;
        group_off = s_plan + (a.W + 1);
    } else {
        seg = a.seg[0];
    }
    const long long total = item_off[a.W];
    const T *Kb = static_cast<const T *>(a.K);
    const T *Vb = static_cast<const T *>(a.V);

    for (long long item = gw; item < total; item += nw) {
        const long long walk = LOCAL ? find_walk(item_off, (int)a.W, item) : a.item_walk[item];
        const long long tree = walk / a.G;
        const long long L = LOCAL ? (long long)s_L[walk] : walk_keys(a.sel_count, walk, a.max_sel, a.C, a.tail);
        const long long i_first = item_off[walk];
        const int nitems = item_off[walk + 1] - (int)i_first;
        const long long sw = seg_len(L, seg);
        const long long k0 = (item - i_first) * sw;
        const long long k1 = k0 + sw < L ? k0 + sw : L;
        const long long nsel = L - a.tail;  // keys coming from selected chunks
        const int *wsel = a.sel + walk * a.max_sel;

        // chunk ids of the item, 32 per window, one per lane; the next window is
        // loaded while the current one is used
        const long long ke = k1 < nsel ? k1 : nsel;
        const int c0 = (int)(k0 / a.C);
        const int c1 = ke > k0 ? (int)((ke - 1) / a.C) + 1 : c0;
        int wb = c0;
        int cur = wb + lane < c1 ? __ldg(wsel + wb + lane) : 0;
        int nxt = wb + 32 + lane < c1 ? __ldg(wsel + wb + 32 + lane) : 0;

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
        const int nsel32 = (int)nsel, k1_32 = (int)k1, C = a.C;
        const int tail0 = (int)(a.n1 * a.C);
        for (int kb = (int)k0; kb < k1_32; kb += KPW * U) {
            // a step spans fewer than 32 chunks, so one shift keeps it inside cur + nxt
            const int cfirst = a.c_shift >= 0 ? kb >> a.c_shift : kb / C;
            if (cfirst - wb >= 32) {
                wb += 32;
                cur = nxt;
                nxt = wb + 32 + lane < c1 ? __ldg(wsel + wb + 32 + lane) : 0;
            }
            bool valid[U];
            int kid[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int kk = kb + u * KPW + grp;
                valid[u] = kk < k1_32;
                kid[u] = 0;
                const int ci = a.c_shift >= 0 ? kk >> a.c_shift : kk / C;
                const int co = a.c_shift >= 0 ? kk & (C - 1) : kk - ci * C;
                const int rel = ci - wb;
                const int from_cur = __shfl_sync(FULL, cur, rel & 31);
                const int from_nxt = __shfl_sync(FULL, nxt, rel & 31);
                const int c = rel < 32 ? from_cur : from_nxt;
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

        if (nitems == 1) {  // the walk is this item: write the result directly
            if (grp == 0) {
                const bool empty = !(l > 0.f);
#pragma unroll
                for (int v = 0; v < VPL; ++v)
#pragma unroll
                    for (int e = 0; e < EPL; ++e) {
                        const long long col = walk * D + (v * LPR + gl) * EPL + e;
                        const float r = empty ? 0.f : acc[v * EPL + e] / l;
                        if (a.out_bf16) store_out(static_cast<__nv_bfloat16 *>(a.out) + col, r);
                        else store_out(static_cast<float *>(a.out) + col, r);
                    }
                if (gl == 0 && a.lse) a.lse[walk] = empty ? -INFINITY : m + logf(l);
            }
            continue;
        }

        if (grp == 0) {
            float *out = a.partial + item * PS;
#pragma unroll
            for (int v = 0; v < VPL; ++v)
#pragma unroll
                for (int e = 0; e < EPL; ++e) out[(v * LPR + gl) * EPL + e] = acc[v * EPL + e];
            if (gl == 0) {
                out[D] = m;
                out[D + 1] = l;
            }
        }
        // the warp that completes a group merges it; the one that completes the
        // walk's last group merges the groups
        __threadfence();
        __syncwarp();
        const int j = (int)(item - i_first), g = j / GROUP;
        const int gsize = nitems - g * GROUP < GROUP ? nitems - g * GROUP : GROUP;
        const long long g_first = group_off[walk];
        const int ngroups = group_off[walk + 1] - (int)g_first;
        int ticket = 0;
        if (lane == 0) ticket = atomicAdd(a.group_done + g_first + g, 1) + 1;
        ticket = __shfl_sync(FULL, ticket, 0);
        if (ticket != gsize) continue;
        __threadfence();
        float gm, gsum, o[CPL];
        merge_rows<D>(a.partial + (i_first + (long long)g * GROUP) * PS, gsize, lane, gm, gsum, o);
        if (ngroups == 1) {
            write_out<D>(a, walk, lane, gm, gsum, o);
            continue;
        }
        float *gp = a.gpartial + (g_first + g) * PS;
#pragma unroll
        for (int c = 0; c < CPL; ++c) gp[lane * CPL + c] = o[c];
        if (lane == 0) {
            gp[D] = gm;
            gp[D + 1] = gsum;
        }
        __threadfence();
        __syncwarp();
        if (lane == 0) ticket = atomicAdd(a.walk_done + walk, 1) + 1;
        ticket = __shfl_sync(FULL, ticket, 0);
        if (ticket != ngroups) continue;
        __threadfence();
        merge_rows<D>(a.gpartial + g_first * PS, ngroups, lane, gm, gsum, o);
        write_out<D>(a, walk, lane, gm, gsum, o);
    }
    chain_done();
}

// Resident CTAs of the item kernel per SM (computed once).
template <typename T, int D, bool LOCAL>
int items_per_sm() {
    static int per_sm = 0;
    if (!per_sm) {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, attend_items_kernel<T, D, LOCAL>, 256,
                                                          sizeof(int) * (3 * LOCAL_MAX_W + 2)) != cudaSuccess ||
            per_sm < 1)
            per_sm = 1;
    }
    return per_sm;
}

template <typename T, int D, bool LOCAL>
cudaError_t launch_items(const zha_tree *t, const ItemArgs &ia, long long max_items, cudaStream_t st) {
    const int per_sm = items_per_sm<T, D, LOCAL>();
    const size_t smem = LOCAL ? sizeof(int) * (3 * (size_t)ia.W + 2) : 0;
    long long blocks = (max_items + 7) / 8;
    const long long cap = (long long)num_sms() * per_sm;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    Probe pr(t, ZHA_K_ATTEND_PARTIAL, st);
    return launch_chained(attend_items_kernel<T, D, LOCAL>, dim3((unsigned)blocks), dim3(256), smem, st, ia);
}

template <typename T, int D>
cudaError_t launch_items_any(const zha_tree *t, const ItemArgs &ia, long long max_items, cudaStream_t st) {
    return ia.W <= LOCAL_MAX_W ? launch_items<T, D, true>(t, ia, max_items, st)
                               : launch_items<T, D, false>(t, ia, max_items, st);
}

// Warps of the item kernel resident at once (its grid never exceeds them).
template <typename T, int D>
long long resident_item_warps(long long W) {
    const int per_sm = W <= LOCAL_MAX_W ? items_per_sm<T, D, true>() : items_per_sm<T, D, false>();
    return (long long)num_sms() * per_sm * 8;
}
long long resident_item_warps(zha_dtype kv, int D, long long W) {
    const bool bf = kv == ZHA_BF16;
    switch (D) {
        case 64: return bf ? resident_item_warps<__nv_bfloat16, 64>(W) : resident_item_warps<float, 64>(W);
        case 128: return bf ? resident_item_warps<__nv_bfloat16, 128>(W) : resident_item_warps<float, 128>(W);
        default: return bf ? resident_item_warps<__nv_bfloat16, 256>(W) : resident_item_warps<float, 256>(W);
    }
}

}  // namespace

namespace {
__global__ void clear_kernel(int *p, long long n) {
    chain_start();
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
        p[i] = 0;
    chain_done();
}
}  // namespace

cudaError_t launch_clear(const zha_tree *t, int *p, long long n, cudaStream_t st) {
    if (n <= 0) return cudaSuccess;
    long long blocks = (n + 255) / 256;
    if (blocks > 4LL * num_sms()) blocks = 4LL * num_sms();
    Probe pr(t, ZHA_K_ATTEND_PLAN, st);
    return launch_chained(clear_kernel, dim3((unsigned)blocks), dim3(256), 0, st, p, n);
}

AttendLayout attend_layout(long long W, int D) {
    AttendLayout L{};
    const long long w = W < 1 ? 1 : W;
    L.max_items = ITEM_BUDGET + w;
    L.max_groups = L.max_items / GROUP + w;
    const long long ps = D + 4;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = (off + bytes + 255) & ~size_t(255);
        return o;
    };
    L.item_off = take(sizeof(int) * (w + 1));
    L.group_off = take(sizeof(int) * (w + 1));
    L.seg = take(sizeof(int));
    L.item_walk = take(sizeof(int) * L.max_items);
    L.walk_done = take(sizeof(int) * w);
    L.group_done = take(sizeof(int) * L.max_groups);
    L.partial = take(sizeof(float) * L.max_items * ps);
    L.gpartial = take(sizeof(float) * L.max_groups * ps);
    L.bytes = off;
    return L;
}

void attend_carve(const AttendLayout &L, void *base, Scratch *s) {
    char *b = static_cast<char *>(base);
    s->item_off = reinterpret_cast<int *>(b + L.item_off);
    s->group_off = reinterpret_cast<int *>(b + L.group_off);
    s->seg = reinterpret_cast<int *>(b + L.seg);
    s->item_walk = reinterpret_cast<int *>(b + L.item_walk);
    s->walk_done = reinterpret_cast<int *>(b + L.walk_done);
    s->group_done = reinterpret_cast<int *>(b + L.group_done);
    s->partial = reinterpret_cast<float *>(b + L.partial);
    s->gpartial = reinterpret_cast<float *>(b + L.gpartial);
    s->max_items = L.max_items;
    s->max_groups = L.max_groups;
}

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
    pl.group_off = s.group_off;
    pl.seg = s.seg;
    pl.item_walk = s.item_walk;
    pl.walk_done = s.walk_done;
    pl.group_done = s.group_done;
    pl.out = out;
    pl.lse = lse;
    // small calls: one item per resident warp, less one per walk for the rounding
    // of each walk's keys into items
    {
        const long long target = resident_item_warps(c.kv_dtype, c.d, W) - W;
        pl.target_items = target > 0 ? target : 0;
    }
    if (W <= LOCAL_MAX_W) {
        // the item kernel plans for itself; only the completion counters (walk
        // and group tickets, adjacent in the scratch) must start at zero
        const long long words = reinterpret_cast<const int *>(s.group_done + s.max_groups) - s.walk_done;
        cudaError_t e = launch_clear(t, s.walk_done, words, st);
        if (e != cudaSuccess) return e;
    } else {
        Probe pr(t, ZHA_K_ATTEND_PLAN, st);
        cudaError_t e = launch_chained(attend_plan_kernel, dim3(1), dim3(1024), 0, st, pl);
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
    ia.group_off = s.group_off;
    ia.seg = s.seg;
    ia.item_walk = s.item_walk;
    ia.walk_done = s.walk_done;
    ia.group_done = s.group_done;
    ia.max_sel = max_sel;
    ia.C = c.chunk;
    ia.D = c.d;
    ia.c_shift = (c.chunk & (c.chunk - 1)) == 0 ? __builtin_ctz((unsigned)c.chunk) : -1;
    ia.G = G;
    ia.W = W;
    ia.cap = c.capacity;
    ia.n1 = t->n_nodes[1];
    ia.tail = pl.tail;
    ia.target_items = pl.target_items;
    ia.beta = c.sharpness;
    ia.partial = s.partial;
    ia.gpartial = s.gpartial;
    ia.out = out;
    ia.lse = lse;
    ia.status = t->d_status;
    const bool bf = c.kv_dtype == ZHA_BF16;
    switch (c.d) {
        case 64:
            return bf ? launch_items_any<__nv_bfloat16, 64>(t, ia, s.max_items, st)
                      : launch_items_any<float, 64>(t, ia, s.max_items, st);
        case 128:
            return bf ? launch_items_any<__nv_bfloat16, 128>(t, ia, s.max_items, st)
                      : launch_items_any<float, 128>(t, ia, s.max_items, st);
        default:
            return bf ? launch_items_any<__nv_bfloat16, 256>(t, ia, s.max_items, st)
                      : launch_items_any<float, 256>(t, ia, s.max_items, st);
    }
}

}  // namespace zha
