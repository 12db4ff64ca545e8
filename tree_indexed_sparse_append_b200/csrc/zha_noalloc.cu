// zha_attend_noalloc: the final attention of zha_attend, with its scratch in a
// fixed device array instead of memory the library allocates.
//
// zha_attend keeps its working memory in the tree and grows it with cudaMalloc
// when a call needs more. Some callers cannot have a library allocate once they
// are running: a serving process that hands all device memory to its own pool at
// start-up, a caller whose allocator is the only one allowed to touch the device,
// or a latency-critical loop that cannot afford the implicit synchronisation that
// cudaMalloc and cudaFree can bring. This entry point takes its scratch from
// one `static __device__` array of ZHA_NOALLOC_SCRATCH_BYTES instead; every GPU
// that loads the library holds that array until the process exits.
//
// In host code the array's name is only a host-side stand-in, not a device
// address, so the address is looked up with cudaGetSymbolAddress, once per
// device with that device current, and that address is what the kernels get.
// The kernels themselves are zha_attend's; only where their scratch lives differs.
#include <cstdio>
#include <mutex>

#include "zha_internal.cuh"

namespace {

constexpr size_t ZHA_NOALLOC_SCRATCH_BYTES = size_t(32) << 20;  // 32 MiB per device
constexpr int MAX_DEVICES = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[ZHA_NOALLOC_SCRATCH_BYTES];

std::mutex g_addr_mu;
void *g_addr[MAX_DEVICES];  // device address of g_noalloc_scratch, per device

// Device address of the array on the current device; looked up on the first call.
int scratch_address(int dev, void **out) {
    std::lock_guard<std::mutex> lock(g_addr_mu);
    if (!g_addr[dev]) {
        void *p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || !p) {
            char msg[256];
            snprintf(msg, sizeof msg, "cudaGetSymbolAddress of the static scratch: %s", cudaGetErrorString(e));
            cudaGetLastError();
            return zha::set_error(ZHA_ERR_CUDA, msg);
        }
        g_addr[dev] = p;
    }
    *out = g_addr[dev];
    return ZHA_OK;
}

}  // namespace

extern "C" int zha_attend_noalloc(zha_tree *t, const void *Q, zha_dtype q_dtype, int n_q_heads, int n_q,
                                  const int *sel, const int *sel_count, int max_sel, void *out,
                                  zha_dtype out_dtype, float *lse, void *stream) {
    if (!t) return zha::set_error(ZHA_ERR_INVALID, "tree is NULL");
    if (!Q || !sel || !sel_count || !out) return zha::set_error(ZHA_ERR_INVALID, "Q, sel, sel_count and out must not be NULL");
    if (q_dtype != ZHA_F32 && q_dtype != ZHA_BF16) return zha::set_error(ZHA_ERR_INVALID, "q_dtype must be ZHA_F32 or ZHA_BF16");
    if (out_dtype != ZHA_F32 && out_dtype != ZHA_BF16)
        return zha::set_error(ZHA_ERR_INVALID, "out_dtype must be ZHA_F32 or ZHA_BF16");
    if (n_q_heads < 1 || n_q < 1 || n_q_heads % t->cfg.n_kv_heads)
        return zha::set_error(ZHA_ERR_INVALID, "n_q_heads must be a positive multiple of n_kv_heads and n_q >= 1");
    if (max_sel < 1) return zha::set_error(ZHA_ERR_INVALID, "max_sel must be >= 1");
    const long long G = (long long)(n_q_heads / t->cfg.n_kv_heads) * n_q;
    const long long W = (long long)t->cfg.batch * n_q_heads * n_q;
    if (W > (1LL << 31) - 1 || G > (1LL << 30)) return zha::set_error(ZHA_ERR_INVALID, "too many walks");

    // the attention's scratch, laid out as zha_attend lays it out
    const zha::AttendLayout layout = zha::attend_layout(W, t->cfg.d);
    if (layout.bytes > ZHA_NOALLOC_SCRATCH_BYTES) {
        char msg[320];
        snprintf(msg, sizeof msg,
                 "zha_attend_noalloc: %lld walks need %zu bytes of scratch, more than the %zu of its "
                 "static array; use zha_attend or fewer walks per call",
                 W, layout.bytes, ZHA_NOALLOC_SCRATCH_BYTES);
        return zha::set_error(ZHA_ERR_CAPACITY, msg);
    }

    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return zha::set_error(ZHA_ERR_CUDA, "cudaGetDevice failed");
    }
    if (dev != t->device) return zha::set_error(ZHA_ERR_INVALID, "the current device is not the tree's device");
    if (dev < 0 || dev >= MAX_DEVICES) return zha::set_error(ZHA_ERR_INVALID, "device index beyond 63");
    void *base = nullptr;
    int rc = scratch_address(dev, &base);
    if (rc) return rc;

    zha::Scratch s{};
    zha::attend_carve(layout, base, &s);
    // The attention clears its completion counters itself (a clear kernel, or the
    // plan kernel for large calls) and computes every offset and item length it
    // reads, so what an earlier call left in the array needs no clearing here.

    // The profiler's CUDA events are created on demand; keep it out of this call.
    zha_profiler *prof = t->prof;
    t->prof = nullptr;
    e = zha::launch_attend(t, s, Q, q_dtype, (int)G, W, sel, sel_count, max_sel, out, out_dtype, lse,
                           static_cast<cudaStream_t>(stream));
    t->prof = prof;
    if (e != cudaSuccess) {
        char msg[256];
        snprintf(msg, sizeof msg, "launching the attention: %s", cudaGetErrorString(e));
        return zha::set_error(ZHA_ERR_CUDA, msg);
    }
    return ZHA_OK;
}
