// Frontier scoring on the tensor cores, for trees walked by many queries at once
// (prefill).
//
// Page "How does a tree of summaries search a context? How ZHA works", section
// "What does a node summarize?": a node scores max_r (beta <key_r, q> + bias_r).
// When thousands of walks share a tree, the scores of one level are a dense
// contraction: per tree, S[g][j] = max_r (beta * (Q K^T)[g][j*RP + r] + bias[j][r])
// with Q the tree's G queries (bf16, d = 128) and K the level's node keys (fp32,
// one row per node and reference). This file computes it for every node of the
// level and every walk of the tree; the selector then reads the frontier entries.
//
// Precision: the queries are bf16, exact in bf16. Each fp32 key is split into
// three bf16 parts, hi = bf16(k), mid = bf16(k - hi), lo = bf16(k - hi - mid),
// which keep 24 bits of its mantissa; bf16 x bf16 products are exact and the
// tensor cores accumulate them in fp32, so D = Q.hi + Q.mid + Q.lo matches an
// fp32 dot product up to the order of the fp32 additions.
//
// Kernels:
//   tc_prep_keys     level keys -> B tiles: per tree and tile of 128 columns
//                    (node, reference), the hi, mid and lo parts as 128 x 128 bf16
//                    in the tensor cores' K-major core-matrix order (8 rows x 16 B
//                    blocks), then the 128 biases (-inf for padding).
//   tc_prep_queries  the tree's queries -> A tiles of 128 walks, same order.
//   score_tc_kernel  one CTA per two A tiles (256 walks): both stay in shared
//                    memory while the B tiles stream through a ring of four
//                    32 KB part slots filled by bulk copies (cp.async.bulk, no
//                    multicast), each slot refilled as soon as the MMAs reading it
//                    complete. A producer warp issues the copies and the
//                    tcgen05.mma (M = N = 128, K = 16, bf16 -> fp32 in TMEM), each
//                    B part feeding both A tiles, into accumulators used in turn
//                    (2 tiles x 2 buffers = all 512 TMEM columns); eight epilogue
//                    warps read a finished accumulator back (tcgen05.ld), free it,
//                    take the max over references and store the scores.
//   Levels of more than 8,192 nodes are not computed whole (the walks' frontiers
//   cover a small part of them):
//   tc_members       per tree and tile of 16 nodes (one word of the membership
//                    bitmap), the list of walks whose frontier holds one of them.
//   score_tc_sparse_kernel  persistent, one CTA per SM over the tiles with
//                    members: the tile's fp32 node rows in one bulk copy (issued
//                    while the previous tile is multiplied), split into the three
//                    parts in shared memory; the member walks' queries gathered 128
//                    at a time (cp.async, zero-filled past the end) into two
//                    alternating buffers; the same MMAs into two alternating TMEM
//                    accumulators, so a batch's MMAs overlap the previous batch's
//                    epilogue; scores stored for the member walks only.
// Every wait is bounded: on timeout the kernel records DEV_TIMEOUT, waits (also
// bounded) for its own copies and MMAs, frees its TMEM and returns.
#include <cstdint>

#include "zha_internal.cuh"
#include "zha_tc.cuh"

namespace zha {
namespace {



// ---------------------------------------------------------------------------
struct PrepKeysArgs {
    const float *nodes;      // level array [T][cap][NF]
    long long node_tree;     // floats per tree
    int NF, R, RP, D;
    long long n_level, ntiles;
    unsigned char *tiles;    // [T][ntiles][TC_BTILE]
};

// one thread per (tree, tile, column, 8-element chunk of K)
__global__ void tc_prep_keys_kernel(PrepKeysArgs a, long long total) {
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= total) return;
    const int kc = (int)(idx & 15);
    const int c = (int)((idx >> 4) & (TC_N - 1));
    const long long tn = idx >> 11;  // tree * ntiles + tile
    const long long tile = tn % a.ntiles, t = tn / a.ntiles;
    const int npt = TC_N / a.RP;
    const long long node = tile * npt + c / a.RP;
    const int r = c % a.RP;
    const bool real = node < a.n_level && r < a.R;
    unsigned char *base = a.tiles + tn * TC_BTILE;
    uint32_t hw[4], mw[4], lw[4];
    if (real) {
        const float *src = a.nodes + t * a.node_tree + node * a.NF + (long long)r * a.D + kc * 8;
        const float4 x0 = *reinterpret_cast<const float4 *>(src);
        const float4 x1 = *reinterpret_cast<const float4 *>(src + 4);
        const float x[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            uint32_t h2 = 0, m2 = 0, l2 = 0;
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const float v = x[2 * i + j];
                const __nv_bfloat16 h = __float2bfloat16_rn(v);
                const float r1 = v - __bfloat162float(h);
                const __nv_bfloat16 m = __float2bfloat16_rn(r1);
                const float r2 = r1 - __bfloat162float(m);
                const __nv_bfloat16 l = __float2bfloat16_rn(r2);
                h2 |= (uint32_t)__bfloat16_as_ushort(h) << (16 * j);
                m2 |= (uint32_t)__bfloat16_as_ushort(m) << (16 * j);
                l2 |= (uint32_t)__bfloat16_as_ushort(l) << (16 * j);
            }
            hw[i] = h2;
            mw[i] = m2;
            lw[i] = l2;
        }
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) hw[i] = mw[i] = lw[i] = 0u;
    }
    const int off = core_offset(c, kc * 8);
    *reinterpret_cast<uint4 *>(base + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    *reinterpret_cast<uint4 *>(base + TC_PART + off) = make_uint4(mw[0], mw[1], mw[2], mw[3]);
    *reinterpret_cast<uint4 *>(base + 2 * TC_PART + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    if (kc == 0) {
        float b = -INFINITY;
        if (real) b = a.nodes[t * a.node_tree + node * a.NF + (long long)a.R * a.D + r];
        reinterpret_cast<float *>(base + 3 * TC_PART)[c] = b;
    }
}

struct PrepQArgs {
    const __nv_bfloat16 *Q;  // [W][128]
    int G;
    long long mtiles;
    unsigned char *tiles;    // [T][mtiles][TC_ATILE]
};

// one thread per (tree, tile, row, 8-element chunk)
__global__ void tc_prep_queries_kernel(PrepQArgs a, long long total) {
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= total) return;
    const int kc = (int)(idx & 15);
    const int row = (int)((idx >> 4) & (TC_M - 1));
    const long long tm = idx >> 11;
    const long long mt = tm % a.mtiles, t = tm / a.mtiles;
    const long long g = mt * TC_M + row;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (g < a.G) v = *reinterpret_cast<const uint4 *>(a.Q + (t * a.G + g) * TC_K + kc * 8);
    *reinterpret_cast<uint4 *>(a.tiles + tm * TC_ATILE + core_offset(row, kc * 8)) = v;
}

struct ScoreTcArgs {
    const unsigned char *atiles, *btiles;
    long long mtiles, ntiles, n_level;  // mtiles: A tiles per tree, a multiple of TC_MT
    int G;
    float beta;
    float *S;
    long long Sstride;
    int *status;
    unsigned long long wait_ns;  // limit of every wait
    int stall;                   // test hook: the producer first waits on a barrier nothing arrives at
};


// RP: columns per node (R rounded up to a power of two; padded references have
// zero keys and bias -inf)
template <int RP>
__global__ void __launch_bounds__(TC_THREADS, 1) score_tc_kernel(ScoreTcArgs a) {
    constexpr int NPT = TC_N / RP;  // nodes per B tile
    extern __shared__ __align__(16) unsigned char smem[];  // no static shared memory: all of it is here
    unsigned char *sA = smem;                              // TC_MT A tiles
    unsigned char *sB = smem + TC_MT * TC_ATILE;           // TC_SLOTS B part slots
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + TC_MT * TC_ATILE + TC_SLOTS * TC_PART);
    // bars 0-3: slot filled; 4-7: slot's MMAs done; 8-9: accumulator buffer written
    // (MMA commit); 10-11: accumulator buffer read back (8 warps); 12: A tiles
    // filled; 13: all MMAs done (cleanup); 16: the test hook's barrier, which
    // nothing arrives at
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 14);
    volatile int *fail = reinterpret_cast<volatile int *>(bars + 15);
    const unsigned long long lim = a.wait_ns;
    auto mbar_wait = [lim](uint32_t bar, uint32_t phase) { return zha::mbar_wait(bar, phase, lim); };

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const long long ct = blockIdx.x, t = blockIdx.y;
    const long long ntiles = a.ntiles, nparts = 3 * ntiles;
    const unsigned char *btree = a.btiles + t * ntiles * TC_BTILE;
    auto full = [&](int s) { return smem_u32(bars + s); };
    auto empty = [&](int s) { return smem_u32(bars + 4 + s); };
    auto accf = [&](int b) { return smem_u32(bars + 8 + b); };
    auto accfree = [&](int b) { return smem_u32(bars + 10 + b); };
    const uint32_t barA = smem_u32(bars + 12), barEnd = smem_u32(bars + 13), barStall = smem_u32(bars + 16);

    if (tid == 0) {
        *fail = 0;
        mbar_init(barStall, 1);
        for (int i = 0; i < TC_SLOTS; ++i) {
            mbar_init(full(i), 1);
            mbar_init(empty(i), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(accf(b), 1);
            mbar_init(accfree(b), 8);
        }
        mbar_init(barA, 1);
        mbar_init(barEnd, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(TC_TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 8) {
        // producer: one thread issues every copy and MMA
        if (lane == 0) {
            // the test hook: a wait that runs out before any copy or MMA is issued
            bool ok = !a.stall || mbar_wait(barStall, 0);
            long long fills[TC_SLOTS] = {0, 0, 0, 0}, waited[TC_SLOTS] = {0, 0, 0, 0};
            bool a_issued = false, a_waited = false, any_mma = false;
            auto fill = [&](long long j) {  // B part j -> slot j % 4
                const int s = (int)(j & (TC_SLOTS - 1));
                mbar_expect_tx(full(s), TC_PART);
                bulk_g2s(smem_u32(sB + s * TC_PART), btree + (j / 3) * TC_BTILE + (j % 3) * TC_PART, TC_PART, full(s));
                ++fills[s];
            };
            if (ok) {
                mbar_expect_tx(barA, TC_MT * TC_ATILE);
                bulk_g2s(smem_u32(sA), a.atiles + (t * a.mtiles + TC_MT * ct) * TC_ATILE, TC_MT * TC_ATILE, barA);
                a_issued = true;
                for (long long j = 0; j < TC_SLOTS && j < nparts; ++j) fill(j);
                if (mbar_wait(barA, 0)) a_waited = true;
                else ok = false;
            }
            for (long long n = 0; ok && n < ntiles; ++n) {
                const int b = (int)(n & 1);
                // accumulator buffer b is free once the epilogue of tile n - 2 read it
                if (n >= 2 && !mbar_wait(accfree(b), (uint32_t)(((n - 2) >> 1) & 1))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                for (int p = 0; p < 3; ++p) {
                    const long long j = 3 * n + p;
                    const int s = (int)(j & (TC_SLOTS - 1));
                    if (!mbar_wait(full(s), (uint32_t)((j >> 2) & 1))) {
                        ok = false;
                        break;
                    }
                    ++waited[s];
                    tc_fence_after();
                    const uint32_t b0 = smem_u32(sB + s * TC_PART);
#pragma unroll
                    for (int m = 0; m < TC_MT; ++m) {
                        const uint32_t a0 = smem_u32(sA + m * TC_ATILE);
                        const uint32_t d = tmem + (uint32_t)((2 * m + b) * TC_N);
#pragma unroll
                        for (int ks = 0; ks < TC_K / 16; ++ks)
                            tc_mma(d, smem_desc(a0 + ks * 256), smem_desc(b0 + ks * 256), (p | ks) ? 1u : 0u);
                    }
                    any_mma = true;
                    tc_commit(empty(s));
                    if (p == 2) tc_commit(accf(b));
                    // the slot of part j - 1 is free once its MMAs complete (part j's
                    // are queued behind them): refill it with part j + 3
                    if (j >= 1 && j + 3 < nparts) {
                        const int s1 = (int)((j - 1) & (TC_SLOTS - 1));
                        if (!mbar_wait(empty(s1), (uint32_t)(((j - 1) >> 2) & 1))) {
                            ok = false;
                            break;
                        }
                        fill(j + 3);
                    }
                }
            }
            if (!ok) {
                *fail = 1;
                report(a.status, DEV_TIMEOUT);
                // let the copies and MMAs in flight finish (bounded waits)
                if (a_issued && !a_waited) (void)mbar_wait(barA, 0);
                for (int s = 0; s < TC_SLOTS; ++s)
                    if (fills[s] > waited[s]) (void)mbar_wait(full(s), (uint32_t)((fills[s] - 1) & 1));
                if (any_mma) {
                    tc_commit(barEnd);
                    (void)mbar_wait(barEnd, 0);
                }
            }
        }
    } else {
        // epilogue: warps 0-3 read A tile 0's accumulators, warps 4-7 A tile 1's;
        // a warp reads TMEM lanes 32 * (warp % 4) .. + 31 (one walk per lane)
        const int m = warp >> 2, wq = warp & 3;
        const long long g = (TC_MT * ct + m) * TC_M + wq * 32 + lane;
        const bool row_ok = g < a.G;
        float *Srow = a.S + (t * a.G + (row_ok ? g : 0)) * a.Sstride;
        const bool vec_ok = (a.Sstride & 3) == 0;
        for (long long n = 0; n < ntiles; ++n) {
            const int b = (int)(n & 1);
            if (!mbar_wait(accf(b), (uint32_t)((n >> 1) & 1)) || *fail) break;
            tc_fence_after();
            const uint32_t base = tmem + ((uint32_t)(wq * 32) << 16) + (uint32_t)((2 * m + b) * TC_N);
            float sc[TC_N];
#pragma unroll
            for (int c0 = 0; c0 < TC_N; c0 += 16) {
                float v[16];
                tc_ld16(base + c0, v);
#pragma unroll
                for (int i = 0; i < 16; ++i) sc[c0 + i] = v[i];
            }
            tc_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(accfree(b));
            const float4 *bias4 = reinterpret_cast<const float4 *>(btree + n * TC_BTILE + 3 * TC_PART);
            // node q's score goes to sc[q] (q <= q * RP, so no later read is overwritten)
#pragma unroll
            for (int q = 0; q < NPT; ++q) {
                float mx = -INFINITY;
#pragma unroll
                for (int r4 = 0; r4 < RP; r4 += 4) {
                    const int c = q * RP + r4;
                    float bb[4];
                    if (RP >= 4) {
                        const float4 v = __ldg(bias4 + c / 4);
                        bb[0] = v.x, bb[1] = v.y, bb[2] = v.z, bb[3] = v.w;
                    } else {
                        const float *bias = reinterpret_cast<const float *>(bias4);
#pragma unroll
                        for (int r = 0; r < 4; ++r) bb[r] = r < RP ? __ldg(bias + c + r) : 0.f;
                    }
#pragma unroll
                    for (int r = 0; r < 4 && r < RP; ++r) mx = fmaxf(mx, fmaf(a.beta, sc[c + r], bb[r]));
                }
                sc[q] = mx;
            }
            if (row_ok) {
                const long long j0 = n * NPT;
#pragma unroll
                for (int q = 0; q < NPT; q += 4) {
                    if (NPT >= 4 && vec_ok && j0 + q + 3 < a.n_level) {
                        *reinterpret_cast<float4 *>(Srow + j0 + q) = make_float4(sc[q], sc[q + 1], sc[q + 2], sc[q + 3]);
                    } else {
#pragma unroll
                        for (int u = 0; u < 4; ++u)
                            if (q + u < NPT && j0 + q + u < a.n_level) Srow[j0 + q + u] = sc[q + u];
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TC_TMEM_COLS)
                     : "memory");
}

}  // namespace

namespace {

// level keys -> B tiles (ntiles per tree)
cudaError_t launch_prep_keys(const zha_tree *t, int level, int RP, long long ntiles, unsigned char *btiles,
                             cudaStream_t st) {
    const zha_config &c = t->cfg;
    PrepKeysArgs k{};
    k.nodes = t->nodes[level];
    k.node_tree = t->cap_nodes[level] * t->NF;
    k.NF = t->NF;
    k.R = c.R;
    k.RP = RP;
    k.D = c.d;
    k.n_level = t->n_nodes[level];
    k.ntiles = ntiles;
    k.tiles = btiles;
    const long long total = (long long)t->T * ntiles * TC_N * 16;
    Probe pr(t, ZHA_K_SCORE_TC, st);
    tc_prep_keys_kernel<<<(unsigned)((total + 255) / 256), 256, 0, st>>>(k, total);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Sparse levels: per B tile (NPT consecutive nodes, which share one membership
// word), the walks of the tree whose frontier holds one of its nodes, in
// ascending order; then one CTA per B tile multiplies the tile by those walks'
// queries, 128 at a time, gathered into shared memory.
struct MembersArgs {
    const unsigned *M;  // level membership bits [T][words][G]
    long long words, ntiles;
    int G, NPT;
    int *counts, *lists;  // [T][ntiles], [T][ntiles][G]
};

__global__ void __launch_bounds__(256) tc_members_kernel(MembersArgs a) {
    __shared__ int s_warp[8];
    const long long nt = blockIdx.x, t = blockIdx.y;
    const long long n0 = nt * a.NPT;
    const unsigned mask = a.NPT >= 32 ? 0xffffffffu : (((1u << a.NPT) - 1u) << (int)(n0 & 31));
    const unsigned *Mrow = a.M + ((long long)t * a.words + (n0 >> 5)) * a.G;
    int *list = a.lists + (t * a.ntiles + nt) * a.G;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    int base = 0;
    for (int g0 = 0; g0 < a.G; g0 += 256) {
        const int g = g0 + threadIdx.x;
        const bool member = g < a.G && (Mrow[g] & mask) != 0u;
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
        if (member) list[base + before + __popc(bal & ((1u << lane) - 1u))] = g;
        base += total;
        __syncthreads();
    }
    if (threadIdx.x == 0) a.counts[t * a.ntiles + nt] = base;
}

struct SparseArgs {
    const float *nodes;           // the level's nodes [T][cap][NF] (fp32 keys [R][D], then biases)
    long long node_tree;          // floats per tree
    int NF, R, T;
    const __nv_bfloat16 *Q;       // [T * G][128]
    const int *counts, *lists;
    long long ntiles, n_level;
    int G;
    float beta;
    float *S;
    long long Sstride;
    int *status;
    unsigned long long wait_ns;  // limit of every wait
};

// Shared memory of the sparse kernel: a tile's fp32 node rows (one bulk copy),
// two buffers of gathered queries, the three bf16 key parts, the biases, barriers
// (230,976 bytes in all).
constexpr int TS_X = TC_N * (TC_K + 1) * 4;  // 128 columns of 128 keys and a bias, at most
constexpr int TS_A_OFF = (TS_X + 1023) & ~1023;
constexpr int TS_P_OFF = TS_A_OFF + 2 * TC_ATILE;
constexpr int TS_BIAS_OFF = TS_P_OFF + 3 * TC_PART;
constexpr int TS_BAR_OFF = TS_BIAS_OFF + TC_N * 4;
constexpr int TS_SMEM = TS_BAR_OFF + 64;

// Persistent: one CTA per SM takes the B tiles with members (NPT consecutive
// nodes x RP references = 128 columns) in turn. A tile's fp32 rows arrive in one
// bulk copy, issued while the previous tile is still being multiplied, and are
// split into the hi, mid and lo parts in shared memory (no preparation pass, 4
// bytes read per key element). The member walks' queries are gathered 128 at a
// time into two alternating buffers (the first batch's while the rows arrive),
// and the MMAs of a batch write one of two TMEM accumulators: while the epilogue
// reads batch b, the MMAs of batch b + 1 run and the queries of batch b + 2 are
// gathered.
template <int RP>
__global__ void __launch_bounds__(128, 1) score_tc_sparse_kernel(SparseArgs a) {
    constexpr int NPT = TC_N / RP;
    extern __shared__ __align__(16) unsigned char smem[];  // no static shared memory: all of it is here
    unsigned char *sX = smem;                               // node rows of the next tile to split
    unsigned char *sA = smem + TS_A_OFF;                    // query buffers 0 and 1
    unsigned char *sP = smem + TS_P_OFF;                    // the tile's three key parts
    float *sBias = reinterpret_cast<float *>(smem + TS_BIAS_OFF);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + TS_BAR_OFF);  // rows copy, MMAs of buffer 0, of buffer 1
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 3);
    volatile int *s_ok = reinterpret_cast<volatile int *>(bars + 4);

    const int tid = threadIdx.x, warp = tid >> 5;
    const long long n_tiles = (long long)a.T * a.ntiles;
    // the next tile with members from `from` on, in this CTA's stride (-1: none)
    auto next_tile = [&](long long from) -> long long {
        for (long long i = from; i < n_tiles; i += gridDim.x)
            if (a.counts[i] > 0) return i;
        return -1;
    };
    long long cur = next_tile(blockIdx.x);
    if (cur < 0) return;  // the same for the whole CTA; nothing allocated yet

    const uint32_t barX = smem_u32(bars);
    const uint32_t barM0 = smem_u32(bars + 1), barM1 = smem_u32(bars + 2);
    auto barM = [&](int buf) { return buf ? barM1 : barM0; };
    const unsigned long long lim = a.wait_ns;
    auto mbar_wait = [lim](uint32_t bar, uint32_t phase) { return zha::mbar_wait(bar, phase, lim); };

    if (tid == 0) {
        mbar_init(barX, 1);
        mbar_init(barM0, 1);
        mbar_init(barM1, 1);
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

    auto tile_nodes = [&](long long tile) {  // nodes of the tile that exist
        const long long n0 = (tile % a.ntiles) * NPT;
        return (int)(a.n_level - n0 < NPT ? a.n_level - n0 : NPT);
    };
    auto copy_rows = [&](long long tile) {  // one thread
        const long long tt = tile / a.ntiles, n0 = (tile % a.ntiles) * NPT;
        const uint32_t bytes = (uint32_t)tile_nodes(tile) * (uint32_t)a.NF * 4u;  // NF * 4 is a multiple of 16
        mbar_expect_tx(barX, bytes);
        bulk_g2s(smem_u32(sX), a.nodes + tt * a.node_tree + n0 * a.NF, bytes, barX);
    };
    // thread i brings walk list[b * 128 + i]'s query into buffer buf (zeros past
    // the list); returns the walk (-1 past the list)
    auto gather = [&](long long tt, const int *list, int count, int b, int buf) -> int {
        const int c0 = b * TC_M;
        const int rows = min(TC_M, count - c0);
        const int g = tid < rows ? list[c0 + tid] : -1;
        const __nv_bfloat16 *src = a.Q + (tt * a.G + (g >= 0 ? g : 0)) * TC_K;
        const uint32_t dst = smem_u32(sA + buf * TC_ATILE);
#pragma unroll
        for (int kc = 0; kc < TC_K / 8; ++kc) cp_async16(dst + core_offset(tid, kc * 8), src + kc * 8, g >= 0 ? 16u : 0u);
        asm volatile("cp.async.commit_group;" ::: "memory");
        return g;
    };
    auto issue = [&](int buf) {  // one thread: the batch in buffer buf against the three parts
        tc_fence_after();
        const uint32_t a0 = smem_u32(sA + buf * TC_ATILE), b0 = smem_u32(sP);
#pragma unroll
        for (int part = 0; part < 3; ++part)
#pragma unroll
            for (int ks = 0; ks < TC_K / 16; ++ks)
                tc_mma(tmem + buf * TC_N, smem_desc(a0 + ks * 256), smem_desc(b0 + part * TC_PART + ks * 256),
                       (part | ks) ? 1u : 0u);
        tc_commit(barM(buf));
    };

    // waits outstanding, and the phase of each barrier
    bool pendX = false, pend0 = false, pend1 = false;
    uint32_t phX = 0u, ph0 = 0u, ph1 = 0u;
    if (tid == 0) copy_rows(cur);
    pendX = true;
    bool ok = true;
    while (ok && cur >= 0) {
        const long long tt = cur / a.ntiles;
        const long long n0 = (cur % a.ntiles) * NPT;
        const int nv = tile_nodes(cur);
        const int count = a.counts[cur];
        const int *list = a.lists + cur * a.G;
        const int nb = (count + TC_M - 1) / TC_M;
        // the first batch's queries while the rows arrive (every MMA of the
        // previous tile is complete, so both buffers are free)
        int g_cur = gather(tt, list, count, 0, 0);
        ok = __syncthreads_and(mbar_wait(barX, phX));
        if (!ok) break;
        pendX = false;
        phX ^= 1u;
        {
            // split: item -> column c (8 consecutive columns per 8 threads, so a
            // quarter warp's 16-byte part stores are contiguous) and 8-key chunk kc,
            // rotated by the column so that the row reads spread over the banks
            const float *X = reinterpret_cast<const float *>(sX);
            for (int item = tid; item < TC_N * (TC_K / 8); item += 128) {
                const int c = ((item >> 7) << 3) | (item & 7);
                const int kc = (((item >> 3) & 15) + (item & 7)) & 15;
                const int q = c / RP, r = c % RP;
                uint32_t hw[4] = {0u, 0u, 0u, 0u}, mw[4] = {0u, 0u, 0u, 0u}, lw[4] = {0u, 0u, 0u, 0u};
                if (q < nv && r < a.R) {
                    const float *src = X + (long long)q * a.NF + r * TC_K + kc * 8;
                    const float4 x0 = *reinterpret_cast<const float4 *>(src);
                    const float4 x1 = *reinterpret_cast<const float4 *>(src + 4);
                    const float x[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
#pragma unroll
                        for (int jj = 0; jj < 2; ++jj) {
                            const float v = x[2 * i + jj];
                            const __nv_bfloat16 h = __float2bfloat16_rn(v);
                            const float r1 = v - __bfloat162float(h);
                            const __nv_bfloat16 m = __float2bfloat16_rn(r1);
                            const __nv_bfloat16 l = __float2bfloat16_rn(r1 - __bfloat162float(m));
                            hw[i] |= (uint32_t)__bfloat16_as_ushort(h) << (16 * jj);
                            mw[i] |= (uint32_t)__bfloat16_as_ushort(m) << (16 * jj);
                            lw[i] |= (uint32_t)__bfloat16_as_ushort(l) << (16 * jj);
                        }
                    }
                }
                const int off = core_offset(c, kc * 8);
                *reinterpret_cast<uint4 *>(sP + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                *reinterpret_cast<uint4 *>(sP + TC_PART + off) = make_uint4(mw[0], mw[1], mw[2], mw[3]);
                *reinterpret_cast<uint4 *>(sP + 2 * TC_PART + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
            }
            const int c = tid, q = c / RP, r = c % RP;  // 128 threads, 128 columns
            sBias[c] = (q < nv && r < a.R) ? X[(long long)q * a.NF + (long long)a.R * TC_K + r] : -INFINITY;
        }
        // the parts (generic-proxy writes) are read by the MMAs; every row is read
        // before the next tile's copy overwrites them
        asm volatile("cp.async.wait_group 0;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncthreads();
        const long long nxt = next_tile(cur + gridDim.x);
        if (nxt >= 0) {
            if (tid == 0) copy_rows(nxt);
            pendX = true;
        }
        if (tid == 0) issue(0);
        pend0 = true;
        for (int b = 0; b < nb; ++b) {
            const int buf = b & 1;
            int g_next = -1;
            if (b + 1 < nb) g_next = gather(tt, list, count, b + 1, buf ^ 1);  // batch b - 1's MMAs are complete
            // one thread waits for batch b's MMAs and tells the others, so that every
            // warp takes the same branch before the warp-collective TMEM loads
            if (tid == 0) *s_ok = mbar_wait(barM(buf), buf ? ph1 : ph0) ? 1 : 0;
            __syncthreads();
            if (!*s_ok) {
                ok = false;
                break;
            }
            if (buf) {
                pend1 = false;
                ph1 ^= 1u;
            } else {
                pend0 = false;
                ph0 ^= 1u;
            }
            if (b + 1 < nb) {
                asm volatile("cp.async.wait_group 0;" ::: "memory");
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                __syncthreads();  // also: batch b - 1's TMEM reads (buffer buf ^ 1) are done
                if (tid == 0) issue(buf ^ 1);
                if (buf) pend0 = true;
                else pend1 = true;
            }
            tc_fence_after();
            float sc[TC_N];
#pragma unroll
            for (int cc = 0; cc < TC_N; cc += 16) {
                float v[16];
                tc_ld16(tmem + buf * TC_N + ((uint32_t)(warp * 32) << 16) + (uint32_t)cc, v);
#pragma unroll
                for (int i = 0; i < 16; ++i) sc[cc + i] = v[i];
            }
            tc_wait_ld();
            tc_fence_before();
#pragma unroll
            for (int q = 0; q < NPT; ++q) {
                float mx = -INFINITY;
#pragma unroll
                for (int r = 0; r < RP; ++r) mx = fmaxf(mx, fmaf(a.beta, sc[q * RP + r], sBias[q * RP + r]));
                sc[q] = mx;
            }
            if (g_cur >= 0) {
                float *Srow = a.S + (tt * a.G + g_cur) * a.Sstride + n0;
#pragma unroll
                for (int q = 0; q < NPT; ++q)
                    if (q < nv) Srow[q] = sc[q];
            }
            g_cur = g_next;
        }
        __syncthreads();  // every TMEM read and bias read of this tile is done
        cur = nxt;
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");  // no gather lands after the CTA
    if (!ok && tid == 0) {
        report(a.status, DEV_TIMEOUT);
        // the copy and MMAs still in flight finish before the memory goes away
        if (pendX) (void)mbar_wait(barX, phX);
        if (pend0) (void)mbar_wait(barM0, ph0);
        if (pend1) (void)mbar_wait(barM1, ph1);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(2 * TC_N) : "memory");
}

template <int RP>
cudaError_t launch_sparse_rp(const zha_tree *t, const SparseArgs &sa, cudaStream_t st) {
    static bool attr = false;
    if (!attr) {
        cudaError_t e =
            cudaFuncSetAttribute(score_tc_sparse_kernel<RP>, cudaFuncAttributeMaxDynamicSharedMemorySize, TS_SMEM);
        if (e != cudaSuccess) return e;
        attr = true;
    }
    Probe pr(t, ZHA_K_SCORE_TC, st);
    long long grid = sa.ntiles * t->T;  // persistent: one CTA per SM at most
    if (grid > num_sms()) grid = num_sms();
    score_tc_sparse_kernel<RP><<<(unsigned)grid, 128, TS_SMEM, st>>>(sa);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_score_tc_sparse(const zha_tree *t, int level, int G, const void *Q, const unsigned *M,
                                   long long words, int *counts, int *lists, float *S, long long Sstride,
                                   cudaStream_t st) {
    const zha_config &c = t->cfg;
    int RP = 1;
    while (RP < c.R) RP <<= 1;
    const long long n_level = t->n_nodes[level];
    const long long ntiles = (n_level * RP + TC_N - 1) / TC_N;
    cudaError_t e = cudaSuccess;
    MembersArgs m{};
    m.M = M;
    m.words = words;
    m.ntiles = ntiles;
    m.G = G;
    m.NPT = TC_N / RP;
    m.counts = counts;
    m.lists = lists;
    {
        Probe pr(t, ZHA_K_SCORE_TC, st);
        tc_members_kernel<<<dim3((unsigned)ntiles, (unsigned)t->T), 256, 0, st>>>(m);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    SparseArgs sa{};
    sa.nodes = t->nodes[level];
    sa.node_tree = t->cap_nodes[level] * t->NF;
    sa.NF = t->NF;
    sa.R = c.R;
    sa.T = t->T;
    sa.Q = static_cast<const __nv_bfloat16 *>(Q);
    sa.counts = counts;
    sa.lists = lists;
    sa.ntiles = ntiles;
    sa.n_level = n_level;
    sa.G = G;
    sa.beta = c.sharpness;
    sa.S = S;
    sa.Sstride = Sstride;
    sa.status = t->d_status;
    sa.wait_ns = t->tc_wait_ns ? t->tc_wait_ns : TC_WAIT_NS;
    switch (RP) {
        case 4: return launch_sparse_rp<4>(t, sa, st);
        case 8: return launch_sparse_rp<8>(t, sa, st);
        default: return launch_sparse_rp<16>(t, sa, st);
    }
}

TcLayout tc_layout(int T, long long G, long long maxn_b, long long maxn_sparse, int R) {
    int RP = 1;
    while (RP < R) RP <<= 1;
    const long long mtiles = (G + TC_M * TC_MT - 1) / (TC_M * TC_MT) * TC_MT;
    const long long ntiles_b = (maxn_b * RP + TC_N - 1) / TC_N;
    const long long ntiles_s = (maxn_sparse * RP + TC_N - 1) / TC_N;
    auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
    TcLayout L{};
    L.a_off = 0;
    L.b_off = up((size_t)T * mtiles * TC_ATILE);
    L.counts_off = up(L.b_off + (size_t)T * ntiles_b * TC_BTILE);
    L.lists_off = up(L.counts_off + (size_t)T * ntiles_s * sizeof(int));
    L.bytes = up(L.lists_off + (size_t)T * ntiles_s * G * sizeof(int));
    return L;
}

bool tc_applicable(const zha_tree *t, int G, const void *Q, zha_dtype q_dtype, int level) {
    return t->cfg.d == TC_K && q_dtype == ZHA_BF16 && (reinterpret_cast<uintptr_t>(Q) & 15) == 0 &&
           G >= TC_MIN_G && t->n_nodes[level] > 0 && t->n_nodes[level] <= TC_MAX_NODES;
}

bool tc_sparse_applicable(const zha_tree *t, int G, const void *Q, zha_dtype q_dtype, int level) {
    // a B tile's nodes must lie in one 32-bit membership word: at least 4 columns per node
    return t->cfg.d == TC_K && q_dtype == ZHA_BF16 && (reinterpret_cast<uintptr_t>(Q) & 15) == 0 &&
           G >= TC_MIN_G && t->n_nodes[level] > TC_MAX_NODES && t->cfg.R > 2;
}

namespace {
template <int RP>
cudaError_t launch_score_tc_rp(const zha_tree *t, const ScoreTcArgs &sa, cudaStream_t st) {
    static bool attr = false;
    if (!attr) {
        cudaError_t e =
            cudaFuncSetAttribute(score_tc_kernel<RP>, cudaFuncAttributeMaxDynamicSharedMemorySize, TC_SMEM);
        if (e != cudaSuccess) return e;
        attr = true;
    }
    Probe pr(t, ZHA_K_SCORE_TC, st);
    score_tc_kernel<RP><<<dim3((unsigned)(sa.mtiles / TC_MT), (unsigned)t->T), TC_THREADS, TC_SMEM, st>>>(sa);
    return cudaGetLastError();
}
}  // namespace

cudaError_t launch_score_tc_queries(const zha_tree *t, const void *Q, int G, unsigned char *ws, cudaStream_t st) {
    PrepQArgs q{};
    q.Q = static_cast<const __nv_bfloat16 *>(Q);
    q.G = G;
    q.mtiles = (G + TC_M * TC_MT - 1) / (TC_M * TC_MT) * TC_MT;
    q.tiles = ws;
    const long long total = (long long)t->T * q.mtiles * TC_M * 16;
    Probe pr(t, ZHA_K_SCORE_TC, st);
    tc_prep_queries_kernel<<<(unsigned)((total + 255) / 256), 256, 0, st>>>(q, total);
    return cudaGetLastError();
}

cudaError_t launch_score_tc(const zha_tree *t, int level, int G, unsigned char *atiles, unsigned char *btiles,
                            float *S, long long Sstride, cudaStream_t st) {
    const zha_config &c = t->cfg;
    int RP = 1;
    while (RP < c.R) RP <<= 1;
    const long long mtiles = (G + TC_M * TC_MT - 1) / (TC_M * TC_MT) * TC_MT;
    const long long n_level = t->n_nodes[level];
    const long long ntiles = (n_level * RP + TC_N - 1) / TC_N;
    {
        cudaError_t e = launch_prep_keys(t, level, RP, ntiles, btiles, st);
        if (e != cudaSuccess) return e;
    }

    ScoreTcArgs sa{};
    sa.atiles = atiles;
    sa.btiles = btiles;
    sa.mtiles = mtiles;
    sa.ntiles = ntiles;
    sa.n_level = n_level;
    sa.G = G;
    sa.beta = c.sharpness;
    sa.S = S;
    sa.Sstride = Sstride;
    sa.status = t->d_status;
    sa.wait_ns = t->tc_wait_ns ? t->tc_wait_ns : TC_WAIT_NS;
    sa.stall = t->tc_stall;
    switch (RP) {
        case 1: return launch_score_tc_rp<1>(t, sa, st);
        case 2: return launch_score_tc_rp<2>(t, sa, st);
        case 4: return launch_score_tc_rp<4>(t, sa, st);
        case 8: return launch_score_tc_rp<8>(t, sa, st);
        default: return launch_score_tc_rp<16>(t, sa, st);
    }
}

}  // namespace zha
