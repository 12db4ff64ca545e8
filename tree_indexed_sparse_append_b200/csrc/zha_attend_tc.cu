// Final attention on the tensor cores, for trees walked by many queries at once
// (prefill).
//
// Page "How does a tree of summaries search a context? How ZHA works", sections
// "How is the tree built?" and "Common misunderstandings": ordinary attention
// over exactly the original keys a walk chose (its level-1 chunks and the tail):
//   out = sum_i softmax_i(beta <q, k_i>) v_i,   lse = logsumexp_i(beta <q, k_i>).
//
// When thousands of walks share a tree, many of them read the same keys. Here
// the keys of a tree are cut into tiles of 128 consecutive keys (128 / C chunks),
// and each tile is read from HBM once and multiplied by the queries of the walks
// that chose one of its chunks (or, for the tile holding the tail, by every
// walk), 128 walks at a time, on tcgen05 (M = walks, N = 128, K = 128, bf16 in,
// fp32 accumulators in TMEM):
//   atc_clear      zero the selection bitmap and the per-walk accumulators
//   atc_scatter    one warp per walk: its chosen chunks -> bitmap bits
//                  [T][chunk words][G] (the walks of a tree side by side)
//   atc_members    per (tree, tile): the walks touching the tile, each with the
//                  mask of its chosen chunks there (warp ballots, compacted)
//   atc_prep_v     per touched tile: V transposed into the MMA's operand order
//                  (d rows x 128 keys, K-major), so one bulk copy brings it in
//   atc_max        per touched tile: S = Q K^T for its walks; each walk's masked
//                  maximum of beta * S goes to a per-walk atomic maximum
//   atc_accum      per touched tile: S again; P = exp(beta * S - m_walk) on the
//                  chosen keys (0 elsewhere), split into bf16 hi + lo parts;
//                  O = P_hi V + P_lo V; the walk's sum of P and its O row are added
//                  to its fp32 accumulators (vector atomics)
//   atc_finish     per walk: out = acc / l, lse = m + log l
// The per-walk maximum is final before any exponential is taken, so every
// partial sum is on the same scale and atomics add them in any order; memory is
// bounded by the tree's tiles and walks (no per-pair partial rows).
//
// Precision: queries and keys are bf16 and their products are exact in the fp32
// accumulators; p in [0, 1] is kept to 16 bits of mantissa by the hi + lo split
// (relative 2^-16); V is bf16; all sums are fp32.
//
// Every wait is bounded (the tree's tensor-core wait limit, 1 s by default): on
// timeout a CTA records DEV_TIMEOUT, waits (bounded) for its copies and MMAs,
// frees its TMEM and returns.
#include <cmath>

#include "zha_internal.cuh"
#include "zha_tc.cuh"

namespace zha {
namespace {

constexpr int AT_KEYS = TC_N;  // keys per tile
constexpr int AT_THREADS = 128;
// max pass: K tile, queries; accumulate pass: V^T tile, K tile (then P's lo
// part), queries (then P's hi part), so that two CTAs fit on an SM; then
// barriers, the TMEM address and a flag
constexpr int AT_SMEM_MAX = TC_PART + TC_ATILE + 64;
constexpr int AT_SMEM_ACC = 2 * TC_PART + TC_ATILE + 64;

struct AtcArgs {
    const __nv_bfloat16 *K, *V, *Q;  // cache [T][cap][128], queries [W][128]
    long long cap, n, n1;            // keys per tree (capacity, live), level-1 nodes
    int C, c_shift, CPT, G;          // chunk (a power of two), log2 C, chunks per tile, walks per tree
    long long ntiles, words1;        // tiles per tree, chunk words per tree
    float beta;
    unsigned *bits;                  // [T][words1][G] chosen chunks
    int *counts;                     // [T][ntiles] walks touching a tile
    unsigned *lists;                 // [T][ntiles][G] walk | chunk mask << 16
    unsigned char *vt;               // [T][ntiles][TC_PART] V^T tiles
    unsigned *mkey;                  // [W] order_key of the walk's maximum
    float *lsum;                     // [W]
    float *acc;                      // [W][128]
    unsigned long long wait_ns;
    int *status;
};

__global__ void atc_clear_kernel(unsigned *bits, long long nbits, unsigned *mkey, float *lsum, float *acc, long long W) {
    const long long stride = (long long)gridDim.x * blockDim.x;
    const long long i0 = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    for (long long i = i0; i < nbits; i += stride) bits[i] = 0u;
    for (long long i = i0; i < W; i += stride) {
        mkey[i] = 0u;  // below the key of every finite score
        lsum[i] = 0.f;
    }
    for (long long i = i0; i < W * TC_K; i += stride) acc[i] = 0.f;
}

// one warp per walk
__global__ void atc_scatter_kernel(AtcArgs a, const int *sel, const int *sel_count, int max_sel, long long W) {
    const long long w = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (w >= W) return;
    const long long t = w / a.G, g = w - t * a.G;
    int n = sel_count[w];
    n = n < 0 ? 0 : (n > max_sel ? max_sel : n);
    for (int i = lane; i < n; i += 32) {
        const int c = sel[w * max_sel + i];
        if (c < 0 || c >= a.n1) {
            report(a.status, DEV_BAD_INDEX);
            continue;
        }
        // a reduction without a returned value: nothing waits for it
        asm volatile("red.relaxed.gpu.global.or.b32 [%0], %1;" ::"l"(&a.bits[(t * a.words1 + (c >> 5)) * a.G + g]),
                     "r"(1u << (c & 31))
                     : "memory");
    }
}

// does tile tau hold tail keys (keys [C * n1, n), read by every walk)?
__device__ __forceinline__ bool tile_has_tail(const AtcArgs &a, long long tau) {
    const long long lo = tau * AT_KEYS, hi = lo + AT_KEYS, t0 = (long long)a.C * a.n1;
    return a.n > t0 && lo < a.n && hi > t0;
}

// grid (tiles, trees), 256 threads
__global__ void __launch_bounds__(256) atc_members_kernel(AtcArgs a) {
    __shared__ int s_warp[8];
    const long long tau = blockIdx.x, t = blockIdx.y;
    const long long c0 = tau * a.CPT;  // first chunk of the tile
    const bool has_chunks = c0 < a.n1;
    const bool tail = tile_has_tail(a, tau);
    const unsigned cmask = a.CPT >= 32 ? 0xffffffffu : (1u << a.CPT) - 1u;
    const int shift = (int)(c0 & 31);
    const unsigned *row = a.bits + (t * a.words1 + (has_chunks ? c0 >> 5 : 0)) * a.G;
    unsigned *list = a.lists + (t * a.ntiles + tau) * a.G;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    int base = 0;
    for (int g0 = 0; g0 < a.G; g0 += 256) {
        const int g = g0 + threadIdx.x;
        const unsigned m = g < a.G && has_chunks ? (row[g] >> shift) & cmask : 0u;
        const bool member = g < a.G && (m != 0u || tail);
        const unsigned bal = __ballot_sync(FULL, member);
        if (lane == 0) s_warp[wid] = __popc(bal);
        __syncthreads();
        int before = 0, total = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int c = s_warp[i];
            before += i < wid ? c : 0;
            total += c;
        }
        if (member) list[base + before + __popc(bal & ((1u << lane) - 1u))] = (unsigned)g | (m << 16);
        base += total;
        __syncthreads();
    }
    if (threadIdx.x == 0) a.counts[t * a.ntiles + tau] = base;
}

// one thread per (tree, tile, d row, 8 keys): 16 bytes of the V^T operand tile
__global__ void atc_prep_v_kernel(AtcArgs a, long long total) {
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= total) return;
    const int kc = (int)(idx & 15);              // 8-key chunk
    const int row = (int)((idx >> 4) & 127);     // dimension
    const long long tt = idx >> 11;              // tree * ntiles + tile
    const long long t = tt / a.ntiles, tau = tt - t * a.ntiles;
    if (a.counts[tt] <= 0) return;
    const long long key0 = tau * AT_KEYS + kc * 8;
    unsigned w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const long long k0 = key0 + 2 * i, k1 = k0 + 1;
        const unsigned short lo = k0 < a.n ? __bfloat16_as_ushort(a.V[(t * a.cap + k0) * TC_K + row]) : 0;
        const unsigned short hi = k1 < a.n ? __bfloat16_as_ushort(a.V[(t * a.cap + k1) * TC_K + row]) : 0;
        w[i] = (unsigned)lo | ((unsigned)hi << 16);
    }
    *reinterpret_cast<uint4 *>(a.vt + tt * TC_PART + core_offset(row, kc * 8)) = make_uint4(w[0], w[1], w[2], w[3]);
}

// Is key j of tile tau chosen by a walk whose chunk mask there is m?
__device__ __forceinline__ bool key_chosen(const AtcArgs &a, long long tau, int j, unsigned m) {
    const long long id = tau * AT_KEYS + j;
    if (id < (long long)a.C * a.n1) return (m >> (j >> a.c_shift)) & 1u;
    return id < a.n;
}

// Gathers the tile's 128 keys (rows, K-major; zeros past n) into sK.
__device__ __forceinline__ void gather_keys(const AtcArgs &a, long long t, long long tau, unsigned char *sK) {
    const long long id = tau * AT_KEYS + threadIdx.x;
    const __nv_bfloat16 *src = a.K + (t * a.cap + (id < a.n ? id : 0)) * TC_K;
    const uint32_t dst = smem_u32(sK);
#pragma unroll
    for (int kc = 0; kc < TC_K / 8; ++kc)
        cp_async16(dst + core_offset(threadIdx.x, kc * 8), src + kc * 8, id < a.n ? 16u : 0u);
}

// Gathers the queries of members c0 .. c0 + 127 of a tile (zeros past the list).
__device__ __forceinline__ unsigned gather_queries(const AtcArgs &a, long long t, const unsigned *list, int c0,
                                                   int count, unsigned char *sA) {
    const int i = c0 + threadIdx.x;
    const unsigned e = i < count ? list[i] : 0xffffffffu;
    const int g = e == 0xffffffffu ? -1 : (int)(e & 0xffffu);
    const __nv_bfloat16 *src = a.Q + (t * a.G + (g >= 0 ? g : 0)) * TC_K;
    const uint32_t dst = smem_u32(sA);
#pragma unroll
    for (int kc = 0; kc < TC_K / 8; ++kc) cp_async16(dst + core_offset(threadIdx.x, kc * 8), src + kc * 8, g >= 0 ? 16u : 0u);
    return e;
}

__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.commit_group;" ::: "memory");
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // generic-proxy writes -> MMA reads
}

// S = A B^T over K = 128 into TMEM columns [col, col + 128)
__device__ __forceinline__ void mma_128(uint32_t tmem_col, uint32_t a0, uint32_t b0, bool accumulate_first) {
#pragma unroll
    for (int ks = 0; ks < TC_K / 16; ++ks)
        tc_mma(tmem_col, smem_desc(a0 + ks * 256), smem_desc(b0 + ks * 256), (ks || accumulate_first) ? 1u : 0u);
}

// this thread's TMEM row (lane = thread) of 128 fp32 columns starting at col
__device__ __forceinline__ void ld_row(uint32_t tmem, int col, float (&v)[TC_N]) {
    const int warp = threadIdx.x >> 5;
#pragma unroll
    for (int cc = 0; cc < TC_N; cc += 16) {
        float x[16];
        tc_ld16(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)(col + cc), x);
#pragma unroll
        for (int i = 0; i < 16; ++i) v[cc + i] = x[i];
    }
    tc_wait_ld();
    tc_fence_before();
}

// Pass 1: each member walk's maximum of beta * <q, k> over its chosen keys of the tile.
__global__ void __launch_bounds__(AT_THREADS, 1) atc_max_kernel(AtcArgs a) {
    extern __shared__ __align__(16) unsigned char smem[];
    unsigned char *sK = smem, *sA = smem + TC_PART;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + TC_PART + TC_ATILE);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 1);
    volatile int *s_ok = reinterpret_cast<volatile int *>(bars + 2);
    const long long tau = blockIdx.x, t = blockIdx.y;
    const int count = a.counts[t * a.ntiles + tau];
    if (count <= 0) return;  // uniform over the CTA; nothing allocated yet
    const unsigned *list = a.lists + (t * a.ntiles + tau) * a.G;
    const int tid = threadIdx.x, warp = tid >> 5;
    const uint32_t barS = smem_u32(bars);
    const unsigned long long lim = a.wait_ns;
    if (tid == 0) {
        mbar_init(barS, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(TC_N)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    gather_keys(a, t, tau, sK);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    uint32_t phase = 0;
    bool ok = true, pending = false;
    for (int c0 = 0; c0 < count; c0 += TC_M) {
        const unsigned e = gather_queries(a, t, list, c0, count, sA);
        cp_async_wait_all();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            mma_128(tmem, smem_u32(sA), smem_u32(sK), false);
            tc_commit(barS);
            *s_ok = mbar_wait(barS, phase, lim) ? 1 : 0;
        }
        __syncthreads();
        if (!*s_ok) {
            ok = false;
            pending = true;
            break;
        }
        phase ^= 1u;
        tc_fence_after();
        float s[TC_N];
        ld_row(tmem, 0, s);
        if (e != 0xffffffffu) {
            const unsigned m = e >> 16;
            float mx = -INFINITY;
#pragma unroll
            for (int j = 0; j < TC_N; ++j)
                if (key_chosen(a, tau, j, m)) mx = fmaxf(mx, a.beta * s[j]);
            if (mx > -INFINITY) atomicMax(a.mkey + t * a.G + (e & 0xffffu), order_key(mx));
        }
        __syncthreads();  // sA is refilled next
    }
    if (!ok) {
        if (tid == 0) report(a.status, DEV_TIMEOUT);
        if (pending && tid == 0) (void)mbar_wait(barS, phase, lim);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TC_N) : "memory");
}

// Pass 2: each member walk's sum of exp(beta * s - m) and its weighted sum of the
// values over its chosen keys of the tile, added to its accumulators.
__global__ void __launch_bounds__(AT_THREADS, 1) atc_accum_kernel(AtcArgs a) {
    extern __shared__ __align__(16) unsigned char smem[];
    // the K tile and the queries are read only by the S MMA: once it has completed,
    // their buffers take P's lo and hi parts; K is gathered again for each batch
    // (the tile is in L2 by then)
    unsigned char *sV = smem, *sK = smem + TC_PART, *sA = smem + 2 * TC_PART;
    unsigned char *sPl = sK, *sPh = sA;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + 2 * TC_PART + TC_ATILE);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 3);
    volatile int *s_ok = reinterpret_cast<volatile int *>(bars + 4);
    const long long tau = blockIdx.x, t = blockIdx.y;
    const long long tt = t * a.ntiles + tau;
    const int count = a.counts[tt];
    if (count <= 0) return;
    const unsigned *list = a.lists + tt * a.G;
    const int tid = threadIdx.x, warp = tid >> 5;
    const uint32_t barV = smem_u32(bars), barS = smem_u32(bars + 1), barO = smem_u32(bars + 2);
    const unsigned long long lim = a.wait_ns;
    if (tid == 0) {
        mbar_init(barV, 1);
        mbar_init(barS, 1);
        mbar_init(barO, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(2 * TC_N)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if (tid == 0) {
        mbar_expect_tx(barV, TC_PART);
        bulk_g2s(smem_u32(sV), a.vt + tt * TC_PART, TC_PART, barV);
    }
    bool ok = true, v_done = false, s_pending = false, o_pending = false;
    uint32_t phase = 0;
    for (int c0 = 0; c0 < count; c0 += TC_M) {
        gather_keys(a, t, tau, sK);
        const unsigned e = gather_queries(a, t, list, c0, count, sA);
        cp_async_wait_all();
        __syncthreads();
        // 2: S is in TMEM; 1: its MMAs were issued and the wait ran out; 0: the V
        // copy's wait ran out, nothing issued
        if (tid == 0) {
            int good = 2;
            if (!v_done && !mbar_wait(barV, 0, lim)) good = 0;
            if (good) {
                tc_fence_after();
                mma_128(tmem, smem_u32(sA), smem_u32(sK), false);
                tc_commit(barS);
                if (!mbar_wait(barS, phase, lim)) good = 1;
            }
            *s_ok = good;
        }
        __syncthreads();
        v_done = v_done || *s_ok != 0;
        if (*s_ok != 2) {
            ok = false;
            s_pending = *s_ok == 1;
            break;
        }
        tc_fence_after();
        float s[TC_N];
        ld_row(tmem, 0, s);
        const bool valid = e != 0xffffffffu;
        const long long w = t * a.G + (valid ? (long long)(e & 0xffffu) : 0);
        const unsigned m = valid ? e >> 16 : 0u;
        const float mw = valid ? key_to_float(a.mkey[w]) : 0.f;
        float l = 0.f;
        // P = exp(beta * s - m_walk) on the chosen keys, as bf16 hi + lo, row tid
#pragma unroll
        for (int j0 = 0; j0 < TC_N; j0 += 8) {
            unsigned hw[4], lw[4];
#pragma unroll
            for (int i = 0; i < 8; i += 2) {
                float p2[2];
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int j = j0 + i + u;
                    p2[u] = valid && key_chosen(a, tau, j, m) ? expf(a.beta * s[j] - mw) : 0.f;
                    l += p2[u];
                }
                const __nv_bfloat16 h0 = __float2bfloat16_rn(p2[0]), h1 = __float2bfloat16_rn(p2[1]);
                const __nv_bfloat16 l0 = __float2bfloat16_rn(p2[0] - __bfloat162float(h0));
                const __nv_bfloat16 l1 = __float2bfloat16_rn(p2[1] - __bfloat162float(h1));
                hw[i / 2] = (unsigned)__bfloat16_as_ushort(h0) | ((unsigned)__bfloat16_as_ushort(h1) << 16);
                lw[i / 2] = (unsigned)__bfloat16_as_ushort(l0) | ((unsigned)__bfloat16_as_ushort(l1) << 16);
            }
            const int off = core_offset(tid, j0);
            *reinterpret_cast<uint4 *>(sPh + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
            *reinterpret_cast<uint4 *>(sPl + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            // O = P_hi V + P_lo V: A = P (walks x keys), B = V^T (d x keys), both K-major
            mma_128(tmem + TC_N, smem_u32(sPh), smem_u32(sV), false);
            mma_128(tmem + TC_N, smem_u32(sPl), smem_u32(sV), true);
            tc_commit(barO);
            *s_ok = mbar_wait(barO, phase, lim) ? 1 : 0;
        }
        __syncthreads();
        if (!*s_ok) {
            ok = false;
            o_pending = true;
            break;
        }
        phase ^= 1u;
        tc_fence_after();
        float o[TC_N];
        ld_row(tmem, TC_N, o);
        if (valid && l > 0.f) {
            atomicAdd(a.lsum + w, l);
            float4 *dst = reinterpret_cast<float4 *>(a.acc + w * TC_K);
#pragma unroll
            for (int c = 0; c < TC_K; c += 4) atomicAdd(dst + c / 4, make_float4(o[c], o[c + 1], o[c + 2], o[c + 3]));
        }
        __syncthreads();  // sA, sP and the TMEM columns are reused next
    }
    if (!ok) {
        if (tid == 0) {
            report(a.status, DEV_TIMEOUT);
            if (!v_done) (void)mbar_wait(barV, 0, lim);
            if (s_pending) (void)mbar_wait(barS, phase, lim);
            if (o_pending) (void)mbar_wait(barO, phase, lim);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(2 * TC_N)
                     : "memory");
}

// one CTA of 128 threads per walk: out = acc / l, lse = m + log l
__global__ void atc_finish_kernel(const unsigned *mkey, const float *lsum, const float *acc, void *out, int out_bf16,
                                  float *lse) {
    const long long w = blockIdx.x;
    const float l = lsum[w];
    const bool empty = !(l > 0.f);
    const float v = empty ? 0.f : acc[w * TC_K + threadIdx.x] / l;
    if (out_bf16) static_cast<__nv_bfloat16 *>(out)[w * TC_K + threadIdx.x] = __float2bfloat16_rn(v);
    else static_cast<float *>(out)[w * TC_K + threadIdx.x] = v;
    if (threadIdx.x == 0 && lse) lse[w] = empty ? -INFINITY : key_to_float(mkey[w]) + logf(l);
}

}  // namespace

bool attend_tc_applicable(const zha_tree *t, int G, zha_dtype q_dtype) {
    const zha_config &c = t->cfg;
    // chunks of 8 to 64 keys (powers of two): a tile's chunk mask fits in 16 bits
    return c.d == TC_K && c.kv_dtype == ZHA_BF16 && q_dtype == ZHA_BF16 && G >= TC_MIN_G && G <= 65535 &&
           c.chunk >= 8 && c.chunk <= 64 && (c.chunk & (c.chunk - 1)) == 0 && t->n > 0;
}

size_t attend_tc_scratch(const zha_tree *t, int G, long long W) {
    const long long ntiles = (t->n + AT_KEYS - 1) / AT_KEYS;
    const long long words1 = t->n_nodes[1] > 0 ? (t->n_nodes[1] + 31) / 32 : 1;
    auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
    return al(sizeof(unsigned) * t->T * words1 * G) + al(sizeof(int) * t->T * ntiles) +
           al(sizeof(unsigned) * t->T * ntiles * G) + al((size_t)t->T * ntiles * TC_PART) + al(sizeof(unsigned) * W) +
           al(sizeof(float) * W) + al(sizeof(float) * W * TC_K);
}

cudaError_t launch_attend_tc(const zha_tree *t, int G, long long W, const void *Q, const int *sel,
                             const int *sel_count, int max_sel, void *out, zha_dtype out_dtype, float *lse,
                             void *ws, cudaStream_t st) {
    const zha_config &c = t->cfg;
    AtcArgs a{};
    a.K = static_cast<const __nv_bfloat16 *>(t->K);
    a.V = static_cast<const __nv_bfloat16 *>(t->V);
    a.Q = static_cast<const __nv_bfloat16 *>(Q);
    a.cap = c.capacity;
    a.n = t->n;
    a.n1 = t->n_nodes[1];
    a.C = c.chunk;
    a.c_shift = __builtin_ctz((unsigned)c.chunk);
    a.CPT = AT_KEYS / c.chunk;
    a.G = G;
    a.ntiles = (t->n + AT_KEYS - 1) / AT_KEYS;
    a.words1 = a.n1 > 0 ? (a.n1 + 31) / 32 : 1;
    a.beta = c.sharpness;
    a.wait_ns = t->tc_wait_ns ? t->tc_wait_ns : TC_WAIT_NS;
    a.status = t->d_status;
    auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
    char *b = static_cast<char *>(ws);
    const long long nbits = (long long)t->T * a.words1 * G;
    a.bits = reinterpret_cast<unsigned *>(b);
    b += al(sizeof(unsigned) * nbits);
    a.counts = reinterpret_cast<int *>(b);
    b += al(sizeof(int) * t->T * a.ntiles);
    a.lists = reinterpret_cast<unsigned *>(b);
    b += al(sizeof(unsigned) * t->T * a.ntiles * G);
    a.vt = reinterpret_cast<unsigned char *>(b);
    b += al((size_t)t->T * a.ntiles * TC_PART);
    a.mkey = reinterpret_cast<unsigned *>(b);
    b += al(sizeof(unsigned) * W);
    a.lsum = reinterpret_cast<float *>(b);
    b += al(sizeof(float) * W);
    a.acc = reinterpret_cast<float *>(b);

    static bool attr = false;
    if (!attr) {
        cudaError_t e = cudaFuncSetAttribute(atc_max_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, AT_SMEM_MAX);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(atc_accum_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, AT_SMEM_ACC);
        if (e != cudaSuccess) return e;
        attr = true;
    }
    cudaError_t e;
    const dim3 tiles((unsigned)a.ntiles, (unsigned)t->T);
    {
        Probe pr(t, ZHA_K_ATTEND_PLAN, st);
        long long blocks = (nbits + 255) / 256;
        blocks = blocks < 1 ? 1 : (blocks > 8LL * num_sms() ? 8LL * num_sms() : blocks);
        atc_clear_kernel<<<(unsigned)blocks, 256, 0, st>>>(a.bits, nbits, a.mkey, a.lsum, a.acc, W);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        atc_scatter_kernel<<<(unsigned)((W * 32 + 255) / 256), 256, 0, st>>>(a, sel, sel_count, max_sel, W);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        atc_members_kernel<<<tiles, 256, 0, st>>>(a);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        const long long total = (long long)t->T * a.ntiles * 2048;
        atc_prep_v_kernel<<<(unsigned)((total + 255) / 256), 256, 0, st>>>(a, total);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    {
        Probe pr(t, ZHA_K_ATTEND_PARTIAL, st);
        atc_max_kernel<<<tiles, AT_THREADS, AT_SMEM_MAX, st>>>(a);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        atc_accum_kernel<<<tiles, AT_THREADS, AT_SMEM_ACC, st>>>(a);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    Probe pr(t, ZHA_K_ATTEND_COMBINE, st);
    atc_finish_kernel<<<(unsigned)W, TC_K, 0, st>>>(a.mkey, a.lsum, a.acc, out, out_dtype == ZHA_BF16, lse);
    return cudaGetLastError();
}

}  // namespace zha
