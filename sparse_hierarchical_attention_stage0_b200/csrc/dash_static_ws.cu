// dash_static_ws.cu -- dash_prefill_static_ws: the prefill path for callers that cannot
// allocate device memory.
//
// Some callers cannot call cudaMalloc themselves.  One example is a plugin inside a host
// application that owns all device memory through its own pool and forbids allocations
// from outside it.  Another is a loop on a latency budget that cannot afford the blocking
// and device-wide synchronisation that cudaMalloc/cudaFree may bring.  Such a caller still
// owns its inputs and outputs, but cannot hand over a workspace.
//
// For them the workspace lives in one file-scope device array of DASH_STATIC_WS_BYTES
// (16 MiB).  The array is reserved on every GPU that loads this library and held until the
// process exits.
//
// On the first call on a device, with that device current, this file looks up the array's
// device address once (cudaGetSymbolAddress) and caches it for that device.  In host code
// the array's name is only a host-side stand-in, never a device address.  That first call
// on each device should come before any stream capture.
//
// Every call shares the one array, and each call leaves its scratch contents behind.  The
// status word is cleared at the start of every call.  tau, the chunk summaries and the mask
// words are fully written by the kernels before they are read, so nothing else needs to
// start at zero.  Calls whose work overlaps on the GPU (different streams, or different host
// threads) race on the array: callers must order them.
#include <mutex>

#include "kernels.cuh"

namespace {

static __device__ __align__(256) unsigned char g_static_ws[DASH_STATIC_WS_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_addr[kMaxDevices] = {};

// Device address of g_static_ws on the current device (looked up once per device).
dash_status_t static_ws_address(void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DASH_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_ws) != cudaSuccess || !p) return DASH_ERR_CUDA;
        g_addr[dev] = p;
    }
    *out = g_addr[dev];
    return DASH_OK;
}

size_t round256(size_t x) { return (x + 255) & ~(size_t)255; }

}  // namespace

extern "C" dash_status_t dash_prefill_static_ws(const dash_params_t *p, const void *q,
                                                const void *k, const void *v,
                                                const float *head_cls, void *out,
                                                float *summary_k, float *prob,
                                                uint64_t *active_blocks, void *stream) {
    if (!p) return DASH_ERR_INVALID_ARGUMENT;
    // The scratch this call needs, as dash_prefill carves it: status word, tau, and the
    // summaries / mask words the caller did not supply.  Sizes beyond the array are refused
    // before anything runs.
    if (dash_prefill_workspace_size(p) == 0) return DASH_ERR_INVALID_ARGUMENT;
    const bool dense = (p->flags & DASH_FLAG_DENSE) != 0;
    const size_t B = (size_t)p->batch, Hkv = (size_t)p->heads_kv, T = (size_t)p->seq_len;
    const size_t D = (size_t)p->head_dim, Bc = (size_t)p->chunk_size;
    const size_t C = (T + Bc - 1) / Bc, W = (C + 63) / 64;
    size_t need = 256 + round256(B * Hkv * T * 4);
    if (!dense && !summary_k) need += round256(B * Hkv * (T / Bc) * D * 4);
    if (!dense && !active_blocks) need += round256(B * Hkv * T * W * 8);
    if (need > (size_t)DASH_STATIC_WS_BYTES) return DASH_ERR_WORKSPACE_TOO_SMALL;
    void *ws = nullptr;
    dash_status_t rc = static_ws_address(&ws);
    if (rc != DASH_OK) return rc;
    return dash_prefill(p, q, k, v, head_cls, out, summary_k, prob, active_blocks, ws,
                        (size_t)DASH_STATIC_WS_BYTES, stream);
}
