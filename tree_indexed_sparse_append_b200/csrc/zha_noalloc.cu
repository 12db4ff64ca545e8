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
// address, so the address is looked up with cudaGetSymbolAddress, with the
// tree's device current, and that address is what the kernels get. The lookup
// runs on every call (it allocates nothing): a cached address would go stale if
// the device's primary context were torn down and made again (cudaDeviceReset),
// which loads the module, and the array, at a new address.
// The kernels themselves are zha_attend's; only where their scratch lives differs.
#include <cstdio>

#include "zha_internal.cuh"

namespace {

constexpr size_t ZHA_NOALLOC_SCRATCH_BYTES = size_t(32) << 20;  // 32 MiB per device

static __device__ __align__(256) unsigned char g_noalloc_scratch[ZHA_NOALLOC_SCRATCH_BYTES];

// Device address of the array on the current device.
int scratch_address(void **out) {
    void *p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) {
        char msg[256];
        snprintf(msg, sizeof msg, "cudaGetSymbolAddress of the static scratch: %s", cudaGetErrorString(e));
        cudaGetLastError();
        return zha::set_error(ZHA_ERR_CUDA, msg);
    }
    *out = p;
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
    void *base = nullptr;
    int rc = scratch_address(&base);
    if (rc) return rc;

    zha::Scratch s{};
    zha::attend_carve(layout, base, &s);
    // The attention clears its completion counters itself (a clear kernel, or the
    // plan kernel for large calls) and computes every offset and item length it
    // reads, so what an earlier call left in the array needs no clearing here.

    // The profiler's CUDA events are created on demand, so this call is not
    // profiled: the launches get a copy of the handle without its profiler, and
    // the caller's tree is never modified (other host threads may be using it).
    zha_tree unprofiled = *t;
    unprofiled.prof = nullptr;
    e = zha::launch_attend(&unprofiled, s, Q, q_dtype, (int)G, W, sel, sel_count, max_sel, out, out_dtype, lse,
                           static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) {
        char msg[256];
        snprintf(msg, sizeof msg, "launching the attention: %s", cudaGetErrorString(e));
        return zha::set_error(ZHA_ERR_CUDA, msg);
    }
    return ZHA_OK;
}
