// C ABI of libzha (include/zha.h): argument checks, tree storage, scratch
// layout, and the launch sequences of build / append / search / attend.
#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <atomic>
#include <mutex>
#include <new>
#include <string>
#include <vector>

#include "zha_internal.cuh"

namespace {

thread_local std::string g_error;

int fail(int code, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_error = buf;
    return code;
}

int cuda_fail(cudaError_t e, const char *what) {
    return fail(e == cudaErrorMemoryAllocation ? ZHA_ERR_OOM : ZHA_ERR_CUDA, "%s: %s (%s)", what,
                cudaGetErrorString(e), cudaGetErrorName(e));
}

#define ZHA_CUDA(call, what)                          \
    do {                                              \
        cudaError_t e_ = (call);                      \
        if (e_ != cudaSuccess) return cuda_fail(e_, what); \
    } while (0)

int check_config(const zha_config *c) {
    if (!c) return fail(ZHA_ERR_INVALID, "config is NULL");
    if (c->batch < 1 || c->n_kv_heads < 1) return fail(ZHA_ERR_INVALID, "batch and n_kv_heads must be >= 1");
    if (c->d != 64 && c->d != 128 && c->d != 256) return fail(ZHA_ERR_INVALID, "d must be 64, 128 or 256 (got %d)", c->d);
    if (c->R < 1 || c->R > 16) return fail(ZHA_ERR_INVALID, "R must be in 1..16 (got %d)", c->R);
    if (c->chunk < 2 || c->chunk > 64) return fail(ZHA_ERR_INVALID, "chunk must be in 2..64 (got %d)", c->chunk);
    if (c->depth < 0 || c->depth > ZHA_MAX_DEPTH)
        return fail(ZHA_ERR_INVALID, "depth must be in 1..%d, or 0 to grow with the keys", ZHA_MAX_DEPTH);
    if (c->top_width < 1) return fail(ZHA_ERR_INVALID, "top_width must be >= 1");
    if (c->capacity < 1) return fail(ZHA_ERR_INVALID, "capacity must be >= 1");
    if (c->capacity > (1LL << 31) - 1) return fail(ZHA_ERR_INVALID, "capacity must fit in int32 key ids");
    if (!(c->sharpness > 0.f) || !std::isfinite(c->sharpness)) return fail(ZHA_ERR_INVALID, "sharpness must be finite and > 0");
    if (c->kv_dtype != ZHA_F32 && c->kv_dtype != ZHA_BF16) return fail(ZHA_ERR_INVALID, "kv_dtype must be ZHA_F32 or ZHA_BF16");
    return ZHA_OK;
}

int start_level(const zha_tree *t) {
    for (int l = 1; l <= t->cfg.depth; ++l)
        if (t->n_nodes[l] <= t->cfg.top_width) return l;
    return t->cfg.depth;
}

// Live node counts of every level with storage; a growing tree's depth is then
// its deepest level holding a node (at least 1).
void set_counts(zha_tree *t) {
    long long n = t->n;
    for (int l = 1; l <= t->max_depth; ++l) {
        n /= t->cfg.chunk;
        t->n_nodes[l] = n;
    }
    if (t->grow) {
        int d = 1;
        for (int l = 2; l <= t->max_depth; ++l)
            if (t->n_nodes[l] > 0) d = l;
        t->cfg.depth = d;
    }
}

size_t align_up(size_t x) { return (x + 255) & ~size_t(255); }

std::atomic<long long> g_launches{0};

// Counts the set bits of the frontier bitmaps of every level of the last search.
__global__ void count_bits_kernel(const unsigned *bits, long long words, unsigned long long *out) {
    unsigned long long c = 0;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < words; i += (long long)gridDim.x * blockDim.x)
        c += __popc(bits[i]);
    for (int o = 16; o >= 1; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
    if ((threadIdx.x & 31) == 0 && c) atomicAdd(out, c);
}

}  // namespace

// CUDA event pairs recorded around launches while a tree is profiled.
struct zha_profiler {
    struct Rec {
        int kind;
        cudaEvent_t a, b;
    };
    std::vector<Rec> live;   // recorded, not read yet
    std::vector<Rec> spare;  // reusable event pairs
    int open_kind = -1;
    cudaEvent_t open_a = nullptr;
    bool on = false;
};

namespace zha {

int num_sms() {
    static int sms = 0;
    if (!sms) {
        int dev = 0;
        cudaGetDevice(&dev);
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1) sms = 132;
    }
    return sms;
}

void probe_begin(const zha_tree *t, int kind, cudaStream_t st) {
    zha_profiler *p = t ? t->prof : nullptr;
    if (!p || !p->on) return;
    zha_profiler::Rec r;
    if (!p->spare.empty()) {
        r = p->spare.back();
        p->spare.pop_back();
    } else {
        r.a = r.b = nullptr;
        if (cudaEventCreate(&r.a) != cudaSuccess || cudaEventCreate(&r.b) != cudaSuccess) {
            cudaGetLastError();
            return;
        }
    }
    r.kind = kind;
    cudaEventRecord(r.a, st);
    p->live.push_back(r);
}

void probe_end(const zha_tree *t, int kind, cudaStream_t st) {
    g_launches.fetch_add(1, std::memory_order_relaxed);
    zha_profiler *p = t ? t->prof : nullptr;
    if (!p || !p->on || p->live.empty() || p->live.back().kind != kind) return;
    cudaEventRecord(p->live.back().b, st);
}

// Carves the scratch of one search/attend of `walks` walks out of one device
// allocation (grown when too small).
int reserve(zha_tree *t, long long walks, int max_sel, Scratch *s) {
    const zha_config &c = t->cfg;
    const long long W = walks < 1 ? 1 : walks;
    (void)max_sel;  // the layout depends on the walks and the tree only
    const long long cap1 = t->cap_nodes[1] > 0 ? t->cap_nodes[1] : 1;
    const long long cap2 = t->max_depth >= 2 && t->cap_nodes[2] > 0 ? t->cap_nodes[2] : 1;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        size_t o = off;
        off = align_up(off + bytes);
        return o;
    };
    const size_t o_qf = take(sizeof(float) * W * c.d);
    const size_t o_S = take(sizeof(float) * W * cap1);
    const size_t o_gk = take(sizeof(uint32_t) * W * cap1);
    const size_t o_L0 = take(sizeof(int) * W * cap2);
    const size_t o_L1 = take(sizeof(int) * W * cap2);
    const size_t o_c0 = take(sizeof(int) * W);
    const size_t o_c1 = take(sizeof(int) * W);
    size_t o_M[ZHA_MAX_DEPTH + 1] = {0}, o_U[ZHA_MAX_DEPTH + 1] = {0};
    // membership bits: per level, [T][words][G] with T * G = W
    const size_t M_start = off;
    // (every level with storage: a growing tree may deepen after this reservation)
    for (int l = 1; l <= t->max_depth; ++l) o_M[l] = take(sizeof(unsigned) * W * ((t->cap_nodes[l] + 31) / 32));
    const size_t M_bytes = off - M_start;
    const size_t U_start = off;
    for (int l = 1; l <= t->max_depth; ++l) o_U[l] = take(sizeof(unsigned) * t->T * ((t->cap_nodes[l] + 31) / 32));
    const size_t U_bytes = off - U_start;
    const AttendLayout att = attend_layout(W, c.d);
    const size_t o_att = take(att.bytes);
    // tensor-core scoring tiles, for trees walked by many queries
    const long long Gw = W / t->T;
    TcLayout tcl{};
    if (c.d == 128 && Gw >= TC_MIN_G) {
        long long maxn_b = 0, maxn_sparse = 0;
        for (int l = 1; l <= t->max_depth; ++l) {
            // prepared B tiles serve the dense levels only (at most TC_MAX_NODES
            // nodes scored); the sparse kernel splits its tiles itself
            maxn_b = std::max(maxn_b, std::min(t->cap_nodes[l], TC_MAX_NODES));
            if (t->cap_nodes[l] > TC_MAX_NODES) maxn_sparse = std::max(maxn_sparse, t->cap_nodes[l]);
        }
        if (maxn_b > 0) tcl = tc_layout(t->T, Gw, maxn_b, maxn_sparse, c.R);
    }
    const size_t o_tc = take(tcl.bytes);
    const size_t need = off;

    if (need > t->ws_bytes) {
        if (t->ws) cudaFree(t->ws);
        t->ws = nullptr;
        t->ws_bytes = 0;
        cudaError_t e = cudaMalloc(&t->ws, need);
        if (e != cudaSuccess) {
            cudaGetLastError();
            return cuda_fail(e, "allocating search scratch");
        }
        t->ws_bytes = need;
    }
    char *b = static_cast<char *>(t->ws);
    s->qf = reinterpret_cast<float *>(b + o_qf);
    s->S = reinterpret_cast<float *>(b + o_S);
    s->gkey = reinterpret_cast<uint32_t *>(b + o_gk);
    s->L[0] = reinterpret_cast<int *>(b + o_L0);
    s->L[1] = reinterpret_cast<int *>(b + o_L1);
    s->cnt[0] = reinterpret_cast<int *>(b + o_c0);
    s->cnt[1] = reinterpret_cast<int *>(b + o_c1);
    for (int l = 0; l <= ZHA_MAX_DEPTH; ++l) {
        s->M[l] = l >= 1 && l <= t->max_depth ? reinterpret_cast<unsigned *>(b + o_M[l]) : nullptr;
        s->U[l] = l >= 1 && l <= t->max_depth ? reinterpret_cast<unsigned *>(b + o_U[l]) : nullptr;
    }
    s->M_base = reinterpret_cast<unsigned *>(b + M_start);
    s->U_base = reinterpret_cast<unsigned *>(b + U_start);
    s->M_bytes = M_bytes;
    s->U_bytes = U_bytes;
    attend_carve(att, b + o_att, s);
    s->tc = tcl.bytes ? reinterpret_cast<unsigned char *>(b + o_tc + tcl.a_off) : nullptr;
    s->tc_b = tcl.bytes ? reinterpret_cast<unsigned char *>(b + o_tc + tcl.b_off) : nullptr;
    s->tc_counts = tcl.bytes && tcl.lists_off > tcl.counts_off ? reinterpret_cast<int *>(b + o_tc + tcl.counts_off)
                                                                : nullptr;
    s->tc_lists = tcl.bytes && tcl.bytes > tcl.lists_off ? reinterpret_cast<int *>(b + o_tc + tcl.lists_off) : nullptr;
    s->Sstride = cap1;
    s->Lstride = cap2;
    return ZHA_OK;
}

// Records `msg` as the message zha_last_error returns on this host thread.
int set_error(int code, const char *msg) {
    g_error = msg;
    return code;
}

}  // namespace zha

extern "C" {

const char *zha_last_error(void) { return g_error.c_str(); }

const char *zha_version(void) { return "zha-b200 0.1 (sm_100a)"; }

int zha_build(const zha_config *cfg, void *K, void *V, const float *refs, long long n_keys, void *stream,
              zha_tree **out) {
    if (!out) return fail(ZHA_ERR_INVALID, "out is NULL");
    *out = nullptr;
    int rc = check_config(cfg);
    if (rc) return rc;
    if (!K || !V || !refs) return fail(ZHA_ERR_INVALID, "K, V and refs must not be NULL");
    if (n_keys < 0 || n_keys > cfg->capacity) return fail(ZHA_ERR_INVALID, "n_keys must be in 0..capacity");
    const size_t elt = cfg->kv_dtype == ZHA_BF16 ? 2 : 4;
    if ((reinterpret_cast<uintptr_t>(K) | reinterpret_cast<uintptr_t>(V)) % 16 ||
        reinterpret_cast<uintptr_t>(refs) % 16)
        return fail(ZHA_ERR_INVALID, "K, V and refs must be 16-byte aligned");
    (void)elt;

    zha_tree *t = new (std::nothrow) zha_tree;
    if (!t) return fail(ZHA_ERR_OOM, "host allocation failed");
    memset(t, 0, sizeof *t);
    t->cfg = *cfg;
    t->T = cfg->batch * cfg->n_kv_heads;
    t->NF = cfg->R * cfg->d + ((cfg->R + 3) & ~3);
    t->K = K;
    t->V = V;
    t->refs = refs;
    t->n = n_keys;
    cudaGetDevice(&t->device);
    // a growing tree gets storage for every level its capacity can fill
    t->grow = cfg->depth == 0;
    t->max_depth = cfg->depth;
    if (t->grow) {
        long long c = cfg->capacity;
        t->max_depth = 1;
        for (int l = 1; l <= ZHA_MAX_DEPTH; ++l) {
            c /= cfg->chunk;
            if (c < 1) break;
            t->max_depth = l;
        }
    }
    long long cap = cfg->capacity;
    for (int l = 1; l <= t->max_depth; ++l) {
        cap /= cfg->chunk;
        t->cap_nodes[l] = cap;
        if (cap > 0) {
            cudaError_t e = cudaMalloc(&t->nodes[l], sizeof(float) * (size_t)t->T * cap * t->NF);
            if (e != cudaSuccess) {
                cudaGetLastError();
                zha_destroy(t);
                return cuda_fail(e, "allocating tree levels");
            }
        }
    }
    cudaError_t e = cudaMalloc(&t->d_status, sizeof(int));
    if (e != cudaSuccess) {
        cudaGetLastError();
        zha_destroy(t);
        return cuda_fail(e, "allocating the status word");
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    e = cudaMemsetAsync(t->d_status, 0, sizeof(int), st);
    set_counts(t);
    for (int l = 1; l <= t->max_depth && e == cudaSuccess; ++l)
        e = zha::launch_build_level(t, l, 0, t->n_nodes[l], st);
    if (e != cudaSuccess) {
        zha_destroy(t);
        return cuda_fail(e, "launching the tree build");
    }
    *out = t;
    return ZHA_OK;
}

int zha_append(zha_tree *t, const void *k_new, const void *v_new, void *stream) {
    if (!t || !k_new || !v_new) return fail(ZHA_ERR_INVALID, "tree, k_new and v_new must not be NULL");
    if (t->n >= t->cfg.capacity) return fail(ZHA_ERR_CAPACITY, "append past capacity (%lld keys)", t->cfg.capacity);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    ZHA_CUDA(zha::launch_append_kv(t, k_new, v_new, st), "launching the append");
    t->n += 1;
    long long below = t->n;
    for (int l = 1; l <= t->max_depth; ++l) {
        if (below % t->cfg.chunk != 0) break;
        const long long j = below / t->cfg.chunk - 1;
        ZHA_CUDA(zha::launch_build_level(t, l, j, j + 1, st), "launching a node build");
        t->n_nodes[l] = j + 1;
        if (l > t->cfg.depth) t->cfg.depth = l;  // a growing tree's first node of a new level
        below = j + 1;
    }
    return ZHA_OK;
}

int zha_rebuild(zha_tree *t, void *stream) {
    if (!t) return fail(ZHA_ERR_INVALID, "tree is NULL");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    for (int l = 1; l <= t->max_depth; ++l)
        ZHA_CUDA(zha::launch_build_level(t, l, 0, t->n_nodes[l], st), "launching the rebuild");
    return ZHA_OK;
}

static int check_queries(const zha_tree *t, const void *Q, zha_dtype q_dtype, int n_q_heads, int n_q,
                         long long *W, int *G) {
    if (!t) return fail(ZHA_ERR_INVALID, "tree is NULL");
    if (!Q) return fail(ZHA_ERR_INVALID, "Q is NULL");
    if (q_dtype != ZHA_F32 && q_dtype != ZHA_BF16) return fail(ZHA_ERR_INVALID, "q_dtype must be ZHA_F32 or ZHA_BF16");
    if (n_q_heads < 1 || n_q < 1 || n_q_heads % t->cfg.n_kv_heads)
        return fail(ZHA_ERR_INVALID, "n_q_heads must be a positive multiple of n_kv_heads and n_q >= 1");
    const long long g = (long long)(n_q_heads / t->cfg.n_kv_heads) * n_q;
    const long long w = (long long)t->cfg.batch * n_q_heads * n_q;
    if (w > (1LL << 31) - 1 || g > (1LL << 30)) return fail(ZHA_ERR_INVALID, "too many walks");
    *W = w;
    *G = (int)g;
    return ZHA_OK;
}

int zha_search(zha_tree *t, const void *Q, zha_dtype q_dtype, int n_q_heads, int n_q, zha_mode mode, float p,
               int k, int *sel, int *sel_count, int max_sel, zha_stats *stats, void *stream) {
    long long W;
    int G;
    int rc = check_queries(t, Q, q_dtype, n_q_heads, n_q, &W, &G);
    if (rc) return rc;
    if (!sel || !sel_count) return fail(ZHA_ERR_INVALID, "sel and sel_count must not be NULL");
    if (max_sel < 1) return fail(ZHA_ERR_INVALID, "max_sel must be >= 1");
    if (mode == ZHA_TOP_P) {
        if (!(p > 0.f) || std::isnan(p)) return fail(ZHA_ERR_INVALID, "top-p needs p > 0 (got %g)", (double)p);
    } else if (mode == ZHA_TOP_K) {
        if (k < 1) return fail(ZHA_ERR_INVALID, "top-K needs k >= 1 (got %d)", k);
    } else {
        return fail(ZHA_ERR_INVALID, "mode must be ZHA_TOP_P or ZHA_TOP_K");
    }
    zha::Scratch s;
    rc = zha::reserve(t, W, max_sel, &s);
    if (rc) return rc;
    ZHA_CUDA(zha::launch_search(t, s, Q, q_dtype, G, W, mode, p, k, sel, sel_count, max_sel, stats, start_level(t),
                                static_cast<cudaStream_t>(stream)),
             "launching the search");
    t->last_W = W;
    t->last_G = G;
    t->last_start = start_level(t);
    t->last_max_sel = max_sel;
    return ZHA_OK;
}

int zha_cp_begin(zha_tree *t, const void *Q, zha_dtype q_dtype, int n_q_heads, int n_q, long long key_begin,
                 const long long *global_counts, int n_counts, int *start_level, void *stream) {
    long long W;
    int G;
    int rc = check_queries(t, Q, q_dtype, n_q_heads, n_q, &W, &G);
    if (rc) return rc;
    if (!global_counts || !start_level) return fail(ZHA_ERR_INVALID, "global_counts and start_level must not be NULL");
    if (t->grow) return fail(ZHA_ERR_INVALID, "the context-parallel walk needs a tree of fixed depth");
    const int depth = t->cfg.depth, C = t->cfg.chunk;
    if (n_counts != depth + 1) return fail(ZHA_ERR_INVALID, "global_counts must hold depth + 1 = %d counts", depth + 1);
    long long span = 1;
    for (int l = 0; l < depth; ++l) span *= C;
    if (key_begin < 0 || key_begin % span)
        return fail(ZHA_ERR_INVALID, "key_begin must be a multiple of C^depth = %lld", span);
    long long div = 1;
    for (int l = 0; l <= depth; ++l) {
        const long long off = key_begin / div;
        const long long mine = l == 0 ? t->n : t->n_nodes[l];
        if (global_counts[l] < off + mine)
            return fail(ZHA_ERR_INVALID, "global count of level %d (%lld) is below this shard's end (%lld)", l,
                        global_counts[l], off + mine);
        t->cp_off[l] = off;
        div *= C;
    }
    int s0 = depth;
    for (int l = 1; l <= depth; ++l)
        if (global_counts[l] <= t->cfg.top_width) {
            s0 = l;
            break;
        }
    zha::Scratch s;
    rc = zha::reserve(t, W, 1, &s);
    if (rc) return rc;
    ZHA_CUDA(zha::launch_search_init(t, s, Q, q_dtype, G, W, nullptr, s0, static_cast<cudaStream_t>(stream)),
             "launching the walk set-up");
    t->cp_active = 1;
    t->cp_level = s0;
    t->cp_start = s0;
    t->cp_cur = 0;
    t->cp_W = W;
    t->cp_G = G;
    *start_level = s0;
    return ZHA_OK;
}

int zha_cp_export(zha_tree *t, int *ids, float *scores, int *counts, long long list_stride, int *level,
                  void *stream) {
    if (!t || !ids || !scores || !counts || !level) return fail(ZHA_ERR_INVALID, "NULL argument");
    if (!t->cp_active) return fail(ZHA_ERR_INVALID, "no context-parallel walk is in progress (zha_cp_begin)");
    if (list_stride < 1) return fail(ZHA_ERR_INVALID, "list_stride must be >= 1");
    zha::Scratch s;
    int rc = zha::reserve(t, t->cp_W, 1, &s);
    if (rc) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int l = t->cp_level;
    ZHA_CUDA(zha::launch_score_level(t, s, l, t->cp_G, st), "launching the shard's scoring");
    ZHA_CUDA(zha::launch_cp_export(t, s, t->cp_cur, l, l == t->cp_start, t->cp_off[l], t->cp_W, ids, scores, counts,
                                   list_stride, st),
             "launching the frontier export");
    *level = l;
    return ZHA_OK;
}

int zha_cp_select(zha_tree *t, int n_parts, const int *ids, const float *scores, const int *counts,
                  long long list_stride, zha_mode mode, float p, int k, int *sel, int *sel_count, int max_sel,
                  int *level, void *stream) {
    if (!t || !ids || !scores || !counts || !sel || !sel_count || !level) return fail(ZHA_ERR_INVALID, "NULL argument");
    if (!t->cp_active) return fail(ZHA_ERR_INVALID, "no context-parallel walk is in progress (zha_cp_begin)");
    if (n_parts < 1 || list_stride < 1 || max_sel < 1)
        return fail(ZHA_ERR_INVALID, "n_parts, list_stride and max_sel must be >= 1");
    if (mode == ZHA_TOP_P) {
        if (!(p > 0.f) || std::isnan(p)) return fail(ZHA_ERR_INVALID, "top-p needs p > 0 (got %g)", (double)p);
    } else if (mode == ZHA_TOP_K) {
        if (k < 1) return fail(ZHA_ERR_INVALID, "top-K needs k >= 1 (got %d)", k);
    } else {
        return fail(ZHA_ERR_INVALID, "mode must be ZHA_TOP_P or ZHA_TOP_K");
    }
    const long long W = t->cp_W, P = (long long)n_parts * list_stride;
    if (P > (1LL << 30)) return fail(ZHA_ERR_INVALID, "n_parts * list_stride too large");
    zha::Scratch s;
    int rc = zha::reserve(t, W, 1, &s);
    if (rc) return rc;
    // packed lists, chosen ids and the selector's staging, per walk P slots each
    const size_t o_ps = align_up(sizeof(int) * W * P), o_pc = o_ps + align_up(sizeof(float) * W * P);
    const size_t o_op = o_pc + align_up(sizeof(int) * W), o_oc = o_op + align_up(sizeof(int) * W * P);
    const size_t o_st = o_oc + align_up(sizeof(int) * W);
    rc = zha::grow_dense_scratch(t, o_st + align_up(sizeof(uint32_t) * W * P));
    if (rc) return rc;
    char *b = static_cast<char *>(t->dws);
    zha::CpScratch cs{reinterpret_cast<int *>(b), reinterpret_cast<float *>(b + o_ps), reinterpret_cast<int *>(b + o_pc),
                      reinterpret_cast<int *>(b + o_op), reinterpret_cast<int *>(b + o_oc),
                      reinterpret_cast<uint32_t *>(b + o_st), P};
    const int l = t->cp_level;
    ZHA_CUDA(zha::launch_cp_select(t, s, t->cp_cur, l, t->cp_G, W, n_parts, ids, scores, counts, list_stride, mode, p,
                                   k, cs, t->cp_off[l], sel, sel_count, max_sel, static_cast<cudaStream_t>(stream)),
             "launching the context-parallel choice");
    if (l == 1) {
        t->cp_active = 0;
        *level = 0;
    } else {
        t->cp_cur ^= 1;
        t->cp_level = l - 1;
        *level = l - 1;
    }
    return ZHA_OK;
}

int zha_lse_combine(int n_parts, long long walks, int d, const float *outs, const float *lses, void *out,
                    zha_dtype out_dtype, float *lse, void *stream) {
    if (n_parts < 1 || walks < 1 || d < 1) return fail(ZHA_ERR_INVALID, "n_parts, walks and d must be >= 1");
    if (!outs || !lses || !out) return fail(ZHA_ERR_INVALID, "outs, lses and out must not be NULL");
    if (out_dtype != ZHA_F32 && out_dtype != ZHA_BF16) return fail(ZHA_ERR_INVALID, "out_dtype must be ZHA_F32 or ZHA_BF16");
    if (walks > (1LL << 31) - 1) return fail(ZHA_ERR_INVALID, "too many walks");
    ZHA_CUDA(zha::launch_lse_combine(n_parts, walks, d, outs, lses, out, out_dtype, lse,
                                     static_cast<cudaStream_t>(stream)),
             "launching the log-sum-exp combine");
    return ZHA_OK;
}

int zha_attend(zha_tree *t, const void *Q, zha_dtype q_dtype, int n_q_heads, int n_q, const int *sel,
               const int *sel_count, int max_sel, void *out, zha_dtype out_dtype, float *lse, void *stream) {
    long long W;
    int G;
    int rc = check_queries(t, Q, q_dtype, n_q_heads, n_q, &W, &G);
    if (rc) return rc;
    if (!sel || !sel_count || !out) return fail(ZHA_ERR_INVALID, "sel, sel_count and out must not be NULL");
    if (out_dtype != ZHA_F32 && out_dtype != ZHA_BF16) return fail(ZHA_ERR_INVALID, "out_dtype must be ZHA_F32 or ZHA_BF16");
    if (max_sel < 1) return fail(ZHA_ERR_INVALID, "max_sel must be >= 1");
    zha::Scratch s;
    rc = zha::reserve(t, W, max_sel, &s);
    if (rc) return rc;
    if (t->cfg.d == 128 && zha::attend_tc_applicable(t, G, q_dtype)) {
        // many bf16 walks per tree: tree-major attention on the tensor cores, its
        // scratch from the tree's second block
        rc = zha::grow_dense_scratch(t, zha::attend_tc_scratch(t, G, W));
        if (rc) return rc;
        ZHA_CUDA(zha::launch_attend_tc(t, G, W, Q, sel, sel_count, max_sel, out, out_dtype, lse, t->dws,
                                       static_cast<cudaStream_t>(stream)),
                 "launching the tensor-core attention");
        return ZHA_OK;
    }
    ZHA_CUDA(zha::launch_attend(t, s, Q, q_dtype, G, W, sel, sel_count, max_sel, out, out_dtype, lse,
                                static_cast<cudaStream_t>(stream)),
             "launching the attention");
    return ZHA_OK;
}

}  // extern "C"

// Grows the tree's full-scan scratch to at least `need` bytes.
int zha::grow_dense_scratch(zha_tree *t, size_t need) {
    if (need <= t->dws_bytes) return ZHA_OK;
    if (t->dws) cudaFree(t->dws);
    t->dws = nullptr;
    t->dws_bytes = 0;
    cudaError_t e = cudaMalloc(&t->dws, need);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return cuda_fail(e, "allocating full-scan scratch");
    }
    t->dws_bytes = need;
    return ZHA_OK;
}

extern "C" {

int zha_chunk_mass(zha_tree *t, const void *Q, zha_dtype q_dtype, int n_q_heads, int n_q, int group, float p,
                   int *sel, int *count, int max_sel, void *stream) {
    long long W;
    int G;
    int rc = check_queries(t, Q, q_dtype, n_q_heads, n_q, &W, &G);
    if (rc) return rc;
    if (G > 32) return fail(ZHA_ERR_INVALID, "the chunk-mass profile takes at most 32 walks per tree (got %d)", G);
    if (group < 1) return fail(ZHA_ERR_INVALID, "group must be >= 1 (got %d)", group);
    if (!(p > 0.f) || std::isnan(p)) return fail(ZHA_ERR_INVALID, "p must be > 0 (got %g)", (double)p);
    if (!sel || !count) return fail(ZHA_ERR_INVALID, "sel and count must not be NULL");
    if (max_sel < 1) return fail(ZHA_ERR_INVALID, "max_sel must be >= 1");
    const long long N = t->n > 0 ? t->n : 1;
    const long long nch = (N + group - 1) / group;
    const size_t o_S = align_up(sizeof(float) * W * t->cfg.d);
    const size_t o_Sc = o_S + align_up(sizeof(float) * W * N);
    const size_t o_gk = o_Sc + align_up(sizeof(float) * W * nch);
    rc = zha::grow_dense_scratch(t, o_gk + align_up(sizeof(uint32_t) * W * nch));
    if (rc) return rc;
    char *b = static_cast<char *>(t->dws);
    ZHA_CUDA(zha::launch_chunk_mass(t, Q, q_dtype, G, W, group, p, sel, count, max_sel, reinterpret_cast<float *>(b),
                                    reinterpret_cast<float *>(b + o_S), reinterpret_cast<float *>(b + o_Sc),
                                    reinterpret_cast<uint32_t *>(b + o_gk), static_cast<cudaStream_t>(stream)),
             "launching the chunk-mass profile");
    return ZHA_OK;
}

int zha_dense_scan(zha_tree *t, const void *Q, zha_dtype q_dtype, int n_q_heads, int n_q, zha_mode mode, float p,
                   int k, int *sel, int *sel_count, int max_sel, void *stream) {
    long long W;
    int G;
    int rc = check_queries(t, Q, q_dtype, n_q_heads, n_q, &W, &G);
    if (rc) return rc;
    if (G > 32) return fail(ZHA_ERR_INVALID, "the full-scan indexer takes at most 32 walks per tree (got %d)", G);
    if (!sel || !sel_count) return fail(ZHA_ERR_INVALID, "sel and sel_count must not be NULL");
    if (max_sel < 1) return fail(ZHA_ERR_INVALID, "max_sel must be >= 1");
    if (mode == ZHA_TOP_P) {
        if (!(p > 0.f) || std::isnan(p)) return fail(ZHA_ERR_INVALID, "top-p needs p > 0 (got %g)", (double)p);
    } else if (mode == ZHA_TOP_K) {
        if (k < 1) return fail(ZHA_ERR_INVALID, "top-K needs k >= 1 (got %d)", k);
    } else {
        return fail(ZHA_ERR_INVALID, "mode must be ZHA_TOP_P or ZHA_TOP_K");
    }
    const long long N = t->n > 0 ? t->n : 1;
    const size_t need = align_up(sizeof(float) * W * t->cfg.d) + align_up(sizeof(float) * W * N) +
                        align_up(sizeof(uint32_t) * W * N);
    rc = zha::grow_dense_scratch(t, need);
    if (rc) return rc;
    char *b = static_cast<char *>(t->dws);
    float *qf = reinterpret_cast<float *>(b);
    float *S = reinterpret_cast<float *>(b + align_up(sizeof(float) * W * t->cfg.d));
    uint32_t *gkey = reinterpret_cast<uint32_t *>(b + align_up(sizeof(float) * W * t->cfg.d) +
                                                  align_up(sizeof(float) * W * N));
    ZHA_CUDA(zha::launch_dense_scan(t, Q, q_dtype, G, W, mode, p, k, sel, sel_count, max_sel, qf, S, gkey,
                                    static_cast<cudaStream_t>(stream)),
             "launching the full-scan indexer");
    return ZHA_OK;
}

int zha_reserve(zha_tree *t, long long max_walks, int max_sel) {
    if (!t) return fail(ZHA_ERR_INVALID, "tree is NULL");
    if (max_walks < 1 || max_sel < 1) return fail(ZHA_ERR_INVALID, "max_walks and max_sel must be >= 1");
    zha::Scratch s;
    return zha::reserve(t, max_walks, max_sel, &s);
}

int zha_level(const zha_tree *t, int level, const float **nodes, long long *n_nodes, long long *level_capacity,
              int *node_floats) {
    if (!t || !nodes || !n_nodes || !level_capacity || !node_floats) return fail(ZHA_ERR_INVALID, "NULL argument");
    if (level < 1 || level > t->cfg.depth) return fail(ZHA_ERR_INVALID, "level must be in 1..depth");
    *nodes = t->nodes[level];
    *n_nodes = t->n_nodes[level];
    *level_capacity = t->cap_nodes[level];
    *node_floats = t->NF;
    return ZHA_OK;
}

long long zha_num_keys(const zha_tree *t) { return t ? t->n : -1; }

int zha_depth(const zha_tree *t) { return t ? t->cfg.depth : -1; }

int zha_sync_status(zha_tree *t, void *stream) {
    if (!t) return fail(ZHA_ERR_INVALID, "tree is NULL");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    ZHA_CUDA(cudaStreamSynchronize(st), "synchronising the stream");
    int code = 0;
    ZHA_CUDA(cudaMemcpy(&code, t->d_status, sizeof(int), cudaMemcpyDeviceToHost), "reading the status word");
    ZHA_CUDA(cudaMemset(t->d_status, 0, sizeof(int)), "clearing the status word");
    if (code == zha::DEV_CAPACITY) return fail(ZHA_ERR_CAPACITY, "a walk opened more level-1 nodes than max_sel");
    if (code == zha::DEV_BAD_INDEX) return fail(ZHA_ERR_INTERNAL, "a selected chunk id was out of range");
    if (code == zha::DEV_TIMEOUT) return fail(ZHA_ERR_TIMEOUT, "a bounded wait inside a kernel gave up");
    if (code) return fail(ZHA_ERR_INTERNAL, "device status %d", code);
    return ZHA_OK;
}

int zha_profile(zha_tree *t, int enable) {
    if (!t) return fail(ZHA_ERR_INVALID, "tree is NULL");
    if (!t->prof) {
        t->prof = new (std::nothrow) zha_profiler;
        if (!t->prof) return fail(ZHA_ERR_OOM, "host allocation failed");
    }
    t->prof->on = enable != 0;
    return ZHA_OK;
}

int zha_profile_read(zha_tree *t, zha_kernel_time *out, void *stream) {
    if (!t || !out) return fail(ZHA_ERR_INVALID, "NULL argument");
    for (int k = 0; k < ZHA_K_KINDS; ++k) out[k].launches = 0, out[k].ms = 0.0;
    if (!t->prof) return ZHA_OK;
    ZHA_CUDA(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)), "synchronising the stream");
    for (auto &r : t->prof->live) {
        float ms = 0.f;
        if (cudaEventElapsedTime(&ms, r.a, r.b) == cudaSuccess && r.kind >= 0 && r.kind < ZHA_K_KINDS) {
            out[r.kind].launches += 1;
            out[r.kind].ms += ms;
        } else {
            cudaGetLastError();
        }
        t->prof->spare.push_back(r);
    }
    t->prof->live.clear();
    return ZHA_OK;
}

long long zha_kernel_launches(void) { return g_launches.load(); }

int zha_test_wait_limit(zha_tree *t, long long wait_ns, int stall) {
    if (!t) return fail(ZHA_ERR_INVALID, "tree is NULL");
    if (wait_ns < 0) return fail(ZHA_ERR_INVALID, "wait_ns must be >= 0");
    t->tc_wait_ns = (unsigned long long)wait_ns;
    t->tc_stall = stall ? 1 : 0;
    return ZHA_OK;
}

int zha_last_search_info(zha_tree *t, zha_search_info *out, void *stream) {
    if (!t || !out) return fail(ZHA_ERR_INVALID, "NULL argument");
    memset(out, 0, sizeof *out);
    if (t->last_W < 1) return fail(ZHA_ERR_INVALID, "no search has run on this tree");
    zha::Scratch s;
    int rc = zha::reserve(t, t->last_W, t->last_max_sel, &s);
    if (rc) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    unsigned long long *d = nullptr;
    ZHA_CUDA(cudaMalloc(&d, sizeof(unsigned long long) * 2 * (ZHA_MAX_DEPTH + 1)), "allocating counters");
    cudaMemsetAsync(d, 0, sizeof(unsigned long long) * 2 * (ZHA_MAX_DEPTH + 1), st);
    for (int l = 1; l <= t->last_start; ++l) {
        const long long words = (t->cap_nodes[l] + 31) / 32;
        const long long uw = (long long)t->T * words, mw = t->last_W * words;
        if (uw > 0) count_bits_kernel<<<(unsigned)std::min<long long>((uw + 255) / 256, 1024), 256, 0, st>>>(s.U[l], uw, d + l);
        if (mw > 0) count_bits_kernel<<<(unsigned)std::min<long long>((mw + 255) / 256, 1024), 256, 0, st>>>(s.M[l], mw, d + ZHA_MAX_DEPTH + 1 + l);
    }
    unsigned long long h[2 * (ZHA_MAX_DEPTH + 1)];
    cudaError_t e = cudaMemcpyAsync(h, d, sizeof h, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    cudaFree(d);
    if (e != cudaSuccess) return cuda_fail(e, "counting frontier bits");
    out->start_level = t->last_start;
    for (int l = 0; l <= ZHA_MAX_DEPTH; ++l) {
        out->union_nodes[l] = (long long)h[l];
        out->walk_nodes[l] = (long long)h[ZHA_MAX_DEPTH + 1 + l];
    }
    return ZHA_OK;
}

void zha_destroy(zha_tree *t) {
    if (!t) return;
    if (t->prof) {
        for (auto &r : t->prof->live) cudaEventDestroy(r.a), cudaEventDestroy(r.b);
        for (auto &r : t->prof->spare) cudaEventDestroy(r.a), cudaEventDestroy(r.b);
        delete t->prof;
    }
    for (int l = 1; l <= ZHA_MAX_DEPTH; ++l)
        if (t->nodes[l]) cudaFree(t->nodes[l]);
    if (t->d_status) cudaFree(t->d_status);
    if (t->ws) cudaFree(t->ws);
    if (t->dws) cudaFree(t->dws);
    delete t;
}

}  // extern "C"
