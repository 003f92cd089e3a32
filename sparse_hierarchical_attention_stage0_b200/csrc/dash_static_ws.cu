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
// On every call made outside a stream capture, with the call's device current, this file
// looks up the array's device address (cudaGetSymbolAddress) and caches it for that device;
// in host code the array's name is only a host-side stand-in, never a device address.  A
// call made while its stream is being captured uses the cached address, so the first call on
// each device must come before any stream capture (a captured first call returns
// DASH_ERR_CUDA).  Looking the address up again outside capture keeps it right after the
// device's primary context has been reset.
//
// Every call shares the one array, and each call leaves its scratch contents behind.  The
// status word is cleared at the start of every call and read back (and cleared) with
// dash_static_ws_read_status.  tau, the chunk summaries and the mask words are fully written
// by the kernels before they are read, so nothing else needs to start at zero.  Calls whose
// work overlaps on the GPU (different streams, or different host threads) race on the array:
// callers must order them.
#include <mutex>

#include "kernels.cuh"

namespace {

static __device__ __align__(256) unsigned char g_static_ws[DASH_STATIC_WS_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_addr[kMaxDevices] = {};

// Device address of g_static_ws on the current device: looked up again when `st` is not
// being captured, taken from the per-device cache while it is.
dash_status_t static_ws_address(cudaStream_t st, void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DASH_ERR_CUDA;
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cap) != cudaSuccess) return DASH_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    if (cap == cudaStreamCaptureStatusNone) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_ws) != cudaSuccess || !p) return DASH_ERR_CUDA;
        g_addr[dev] = p;
    }
    if (!g_addr[dev]) return DASH_ERR_CUDA;
    *out = g_addr[dev];
    return DASH_OK;
}

}  // namespace

extern "C" dash_status_t dash_prefill_static_ws(const dash_params_t *p, const void *q,
                                                const void *k, const void *v,
                                                const float *head_cls, void *out,
                                                float *summary_k, float *prob,
                                                uint64_t *active_blocks, void *stream) {
    // The scratch this call needs, as dash_prefill carves it (one helper sizes both):
    // status word, tau, and the summaries / mask words the caller did not supply.  Sizes
    // beyond the array are refused before anything runs.
    const size_t need = dash::prefill_scratch_bytes(p, summary_k != nullptr, active_blocks != nullptr);
    if (need == 0)   // bad parameters: dash_prefill returns their status before any launch
        return dash_prefill(p, q, k, v, head_cls, out, summary_k, prob, active_blocks, nullptr, 0, stream);
    if (need > (size_t)DASH_STATIC_WS_BYTES) return DASH_ERR_WORKSPACE_TOO_SMALL;
    void *ws = nullptr;
    dash_status_t rc = static_ws_address(static_cast<cudaStream_t>(stream), &ws);
    if (rc != DASH_OK) return rc;
    return dash_prefill(p, q, k, v, head_cls, out, summary_k, prob, active_blocks, ws,
                        (size_t)DASH_STATIC_WS_BYTES, stream);
}

extern "C" dash_status_t dash_static_ws_read_status(void *stream) {
    void *ws = nullptr;
    dash_status_t rc = static_ws_address(static_cast<cudaStream_t>(stream), &ws);
    if (rc != DASH_OK) return rc;
    return dash_read_device_status(ws, stream);
}
