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
//   score_tc_kernel  one CTA per A tile: the A tile stays in shared memory, the B
//                    tiles stream through a two-stage ring filled by bulk copies
//                    (cp.async.bulk, no multicast; a stage is refilled as soon as
//                    the MMAs reading it complete, the biases go to a ring of
//                    their own), one thread issues the tcgen05.mma (M = N = 128,
//                    K = 16, bf16 -> fp32 in TMEM) into two accumulators used in
//                    turn, and four warps read a finished accumulator back
//                    (tcgen05.ld), take the max over references and store the
//                    scores.
// Every wait is bounded: on timeout the kernel records DEV_TIMEOUT, waits (also
// bounded) for its own copies and MMAs, frees its TMEM and returns.
#include <cstdint>

#include "zha_internal.cuh"

namespace zha {
namespace {

constexpr int TC_M = 128;                            // walks per A tile
constexpr int TC_N = 128;                            // columns (node x reference) per B tile
constexpr int TC_K = 128;                            // head dimension
constexpr int TC_PART = TC_N * TC_K * 2;             // bytes of one bf16 part of a B tile
constexpr int TC_BTILE = 3 * TC_PART + TC_N * 4;     // hi, mid, lo, biases
constexpr int TC_ATILE = TC_M * TC_K * 2;
constexpr int TC_STAGES = 2;
constexpr int TC_BIAS_SLOTS = 4;                     // a tile's biases outlive its B stage
constexpr int TC_STAGE = 3 * TC_PART;                // shared memory of one B stage (the three parts)
constexpr int TC_SMEM = TC_ATILE + TC_STAGES * TC_STAGE + TC_BIAS_SLOTS * TC_N * 4 + 128;  // + barriers, TMEM address
constexpr int TC_TMEM_COLS = 2 * TC_N;               // two fp32 accumulators of 128 columns
constexpr unsigned long long TC_WAIT_NS = 1000000000ull;  // a wait gives up after 1 s

// byte offset of element (row, k) in a 128-row K-major tile without swizzle:
// 8-row x 16-byte core matrices, consecutive along K (128 B apart), 8-row groups
// 2 KB apart
__host__ __device__ __forceinline__ int core_offset(int row, int k) {
    return (row >> 3) * 2048 + (k >> 3) * 128 + (row & 7) * 16 + (k & 7) * 2;
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// shared memory matrix descriptor: K-major, no swizzle, LBO = 128 B (between the
// two K halves of an MMA's 16-element slice), SBO = 2 KB (between 8-row groups),
// descriptor version 1
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr) {
    return (uint64_t)((addr >> 4) & 0x3FFF) | ((uint64_t)(128 >> 4) << 16) | ((uint64_t)(2048 >> 4) << 32) |
           ((uint64_t)1 << 46);
}

// instruction descriptor: D fp32, A and B bf16, both K-major, N = 128, M = 128
constexpr uint32_t TC_IDESC = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(TC_N >> 3) << 17) |
                              ((uint32_t)(TC_M >> 4) << 24);

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t phase) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(phase)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ unsigned long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// bounded wait; false when it gave up
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t phase) {
    if (mbar_try_wait(bar, phase)) return true;
    const unsigned long long t0 = global_ns();
    while (global_ns() - t0 < TC_WAIT_NS)
        if (mbar_try_wait(bar, phase)) return true;
    return false;
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}

__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(TC_IDESC), "r"(accumulate), "r"(0), "r"(0), "r"(0), "r"(0));
}

__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tc_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

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
    long long mtiles, ntiles, n_level;
    int G;
    float beta;
    float *S;
    long long Sstride;
    int *status;
};

// RP: columns per node (R rounded up to a power of two; padded references have
// zero keys and bias -inf)
template <int RP>
__global__ void __launch_bounds__(128, 1) score_tc_kernel(ScoreTcArgs a) {
    constexpr int NPT = TC_N / RP;  // nodes per B tile
    extern __shared__ __align__(16) unsigned char smem[];  // no static shared memory: all of it is here
    unsigned char *sA = smem;
    unsigned char *sB = smem + TC_ATILE;
    float *sBias = reinterpret_cast<float *>(smem + TC_ATILE + TC_STAGES * TC_STAGE);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + TC_ATILE + TC_STAGES * TC_STAGE + TC_BIAS_SLOTS * TC_N * 4);
    // bars[0..1]: B stage s filled (bulk copies); bars[2..3]: accumulator s written
    // (MMA commit); bars[4]: A tile filled
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 6);
    int &s_fail = *reinterpret_cast<int *>(bars + 7);

    const int tid = threadIdx.x, warp = tid >> 5;
    const long long mt = blockIdx.x, t = blockIdx.y;
    const long long ntiles = a.ntiles;
    const unsigned char *btree = a.btiles + t * ntiles * TC_BTILE;
    const uint32_t barA = smem_u32(bars + 4);
    auto bar_full = [&](int s) { return smem_u32(bars + s); };
    auto bar_mma = [&](int s) { return smem_u32(bars + 2 + s); };

    if (tid == 0) {
        s_fail = 0;
        for (int i = 0; i < 5; ++i) mbar_init(smem_u32(bars + i), 1);
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

    // thread 0 issues every copy and MMA and remembers which are still in flight:
    // bit 0: A copy; bits 1..2: B stage copies; bits 3..4: MMA groups
    unsigned pending = 0;
    long long issued_full[TC_STAGES] = {0, 0}, issued_mma[TC_STAGES] = {0, 0};  // uses so far, per barrier
    // B tile n -> stage s: its three parts into the stage, its biases into slot n % 4
    auto fill = [&](long long n, int s) {
        const unsigned char *src = btree + n * TC_BTILE;
        mbar_expect_tx(bar_full(s), TC_BTILE);
        bulk_g2s(smem_u32(sB + s * TC_STAGE), src, TC_STAGE, bar_full(s));
        bulk_g2s(smem_u32(sBias + (n & (TC_BIAS_SLOTS - 1)) * TC_N), src + TC_STAGE, TC_N * 4, bar_full(s));
        pending |= 2u << s;
        ++issued_full[s];
    };
    if (tid == 0) {
        mbar_expect_tx(barA, TC_ATILE);
        bulk_g2s(smem_u32(sA), a.atiles + (t * a.mtiles + mt) * TC_ATILE, TC_ATILE, barA);
        pending |= 1u;
        for (int s = 0; s < TC_STAGES && s < ntiles; ++s) fill(s, s);
    }

    const long long g = mt * TC_M + tid;  // this thread's walk within the tree (row of the tile)
    const bool row_ok = g < a.G;
    float *Srow = a.S + (t * a.G + (row_ok ? g : 0)) * a.Sstride;
    const bool vec_ok = (a.Sstride & 3) == 0;
    bool ok = true;

    // reads accumulator (n & 1) of tile n and writes its scores
    auto epilogue = [&](long long n) {
        const int s = (int)(n & 1);
        if (ok) {
            if (mbar_wait(bar_mma(s), (uint32_t)((n >> 1) & 1))) {
                if (tid == 0) pending &= ~(8u << s);
            } else {
                ok = false;
            }
        }
        tc_fence_after();
        const float *bias = sBias + (n & (TC_BIAS_SLOTS - 1)) * TC_N;
        const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)(s * TC_N);
        float sc[TC_N];
#pragma unroll
        for (int c0 = 0; c0 < TC_N; c0 += 16) {
            float v[16];
            tc_ld16(lane_base + c0, v);
#pragma unroll
            for (int i = 0; i < 16; ++i) sc[c0 + i] = v[i];
        }
        tc_wait_ld();
        // node q's score goes to sc[q] (q <= q * RP, so no later read is overwritten)
#pragma unroll
        for (int q = 0; q < NPT; ++q) {
            float m = -INFINITY;
#pragma unroll
            for (int r = 0; r < RP; ++r) m = fmaxf(m, fmaf(a.beta, sc[q * RP + r], bias[q * RP + r]));
            sc[q] = m;
        }
        if (ok && row_ok) {
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
        tc_fence_before();
    };

    if (tid == 0) {
        if (mbar_wait(barA, 0)) pending &= ~1u;
        else ok = false;
    }
    for (long long n = 0; n < ntiles; ++n) {
        const int s = (int)(n & 1);
        // MMA for tile n into accumulator s (free: the epilogue of its previous tile
        // ended before the last block barrier)
        if (tid == 0 && ok) {
            if (!mbar_wait(bar_full(s), (uint32_t)((n >> 1) & 1))) {
                ok = false;
            } else {
                pending &= ~(2u << s);
                tc_fence_after();
                const uint32_t a0 = smem_u32(sA), b0 = smem_u32(sB + s * TC_STAGE);
                const uint32_t d = tmem + (uint32_t)(s * TC_N);
#pragma unroll
                for (int part = 0; part < 3; ++part)
#pragma unroll
                    for (int ks = 0; ks < TC_K / 16; ++ks)
                        tc_mma(d, smem_desc(a0 + ks * 256), smem_desc(b0 + part * TC_PART + ks * 256),
                               (part | ks) ? 1u : 0u);
                tc_commit(bar_mma(s));
                pending |= 8u << s;
                ++issued_mma[s];
                // the stage of tile n - 1 is free once its MMAs complete: refill it
                // with tile n + 1 while tile n multiplies
                if (n >= 1 && n + 1 < ntiles) {
                    const int s1 = (int)((n + 1) & 1);
                    if (mbar_wait(bar_mma(s1), (uint32_t)(((n - 1) >> 1) & 1))) {
                        pending &= ~(8u << s1);
                        fill(n + 1, s1);
                    } else {
                        ok = false;
                    }
                }
            }
        }
        // scores of tile n - 1 while tile n multiplies
        if (n >= 1) epilogue(n - 1);
        if (!ok) s_fail = 1;
        __syncthreads();
        if (s_fail) {
            ok = false;
            break;
        }
    }
    if (ok && ntiles >= 1) epilogue(ntiles - 1);
    if (!ok) s_fail = 1;
    __syncthreads();
    if (s_fail) {
        // let the copies and MMAs still in flight finish before the memory they
        // write is released (each wait bounded as well)
        if (tid == 0) {
            report(a.status, DEV_TIMEOUT);
            if (pending & 1u) (void)mbar_wait(barA, 0);
            for (int s = 0; s < TC_STAGES; ++s) {
                if (pending & (2u << s)) (void)mbar_wait(bar_full(s), (uint32_t)((issued_full[s] - 1) & 1));
                if (pending & (8u << s)) (void)mbar_wait(bar_mma(s), (uint32_t)((issued_mma[s] - 1) & 1));
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

size_t tc_scratch_bytes(int T, long long G, long long max_level_nodes, int R) {
    int RP = 1;
    while (RP < R) RP <<= 1;
    const long long mtiles = (G + TC_M - 1) / TC_M;
    const long long ntiles = (max_level_nodes * RP + TC_N - 1) / TC_N;
    return (size_t)T * mtiles * TC_ATILE + (size_t)T * ntiles * TC_BTILE;
}

bool tc_applicable(const zha_tree *t, int G, const void *Q, zha_dtype q_dtype, int level) {
    return t->cfg.d == TC_K && q_dtype == ZHA_BF16 && (reinterpret_cast<uintptr_t>(Q) & 15) == 0 &&
           G >= TC_MIN_G && t->n_nodes[level] > 0 && t->n_nodes[level] <= TC_MAX_NODES;
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
    Probe pr(t, ZHA_K_SCORE, st);
    score_tc_kernel<RP><<<dim3((unsigned)sa.mtiles, (unsigned)t->T), 128, TC_SMEM, st>>>(sa);
    return cudaGetLastError();
}
}  // namespace

cudaError_t launch_score_tc_queries(const zha_tree *t, const void *Q, int G, unsigned char *ws, cudaStream_t st) {
    PrepQArgs q{};
    q.Q = static_cast<const __nv_bfloat16 *>(Q);
    q.G = G;
    q.mtiles = (G + TC_M - 1) / TC_M;
    q.tiles = ws;
    const long long total = (long long)t->T * q.mtiles * TC_M * 16;
    Probe pr(t, ZHA_K_SCORE, st);
    tc_prep_queries_kernel<<<(unsigned)((total + 255) / 256), 256, 0, st>>>(q, total);
    return cudaGetLastError();
}

cudaError_t launch_score_tc(const zha_tree *t, int level, int G, unsigned char *ws, float *S, long long Sstride,
                            cudaStream_t st) {
    const zha_config &c = t->cfg;
    int RP = 1;
    while (RP < c.R) RP <<= 1;
    const long long mtiles = (G + TC_M - 1) / TC_M;
    const long long n_level = t->n_nodes[level];
    const long long ntiles = (n_level * RP + TC_N - 1) / TC_N;
    unsigned char *atiles = ws;
    unsigned char *btiles = ws + (size_t)t->T * mtiles * TC_ATILE;

    PrepKeysArgs k{};
    k.nodes = t->nodes[level];
    k.node_tree = t->cap_nodes[level] * t->NF;
    k.NF = t->NF;
    k.R = c.R;
    k.RP = RP;
    k.D = c.d;
    k.n_level = n_level;
    k.ntiles = ntiles;
    k.tiles = btiles;
    const long long total = (long long)t->T * ntiles * TC_N * 16;
    {
        Probe pr(t, ZHA_K_SCORE, st);
        tc_prep_keys_kernel<<<(unsigned)((total + 255) / 256), 256, 0, st>>>(k, total);
        cudaError_t e = cudaGetLastError();
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
    switch (RP) {
        case 1: return launch_score_tc_rp<1>(t, sa, st);
        case 2: return launch_score_tc_rp<2>(t, sa, st);
        case 4: return launch_score_tc_rp<4>(t, sa, st);
        case 8: return launch_score_tc_rp<8>(t, sa, st);
        default: return launch_score_tc_rp<16>(t, sa, st);
    }
}

}  // namespace zha
