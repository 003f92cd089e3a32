// dash_api.cu -- the C ABI declared in include/dash.h: host-side argument checks, workspace
// carving and stream-ordered launches.  Nothing here allocates device memory or keeps
// global state; every failure is reported before the first launch of a call.
#include <algorithm>
#include <cmath>
#include <cstdint>

#include "kernels.cuh"

using namespace dash;

namespace {

constexpr size_t kStatusBytes = 256;

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }
bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Shape {
    int B, Hq, Hkv, T, D, Bc, G, C, Cf, W;
};

// Whether the caller asked for the routing inside the Stage 2 kernel (DASH_FLAG_FUSE_ROUTE).
bool fuse_requested(const dash_params_t *p) { return (p->flags & DASH_FLAG_FUSE_ROUTE) != 0; }

// Checks shared by every entry point.  `decode`: seq_len is a cache capacity.
dash_status_t check_params(const dash_params_t *p, Shape *s) {
    if (!p) return DASH_ERR_INVALID_ARGUMENT;
    if (p->batch < 1 || p->heads_q < 1 || p->heads_kv < 1 || p->seq_len < 1 ||
        p->head_dim < 1 || p->chunk_size < 1)
        return DASH_ERR_INVALID_ARGUMENT;
    if (p->heads_q % p->heads_kv != 0) return DASH_ERR_INVALID_ARGUMENT;
    if (!p->enable_gqa && p->heads_q != p->heads_kv) return DASH_ERR_INVALID_ARGUMENT;
    if (!std::isfinite(p->alpha) || p->alpha < 1.f) return DASH_ERR_INVALID_ARGUMENT;
    if (!std::isfinite(p->gamma) || !(p->gamma > 0.f)) return DASH_ERR_INVALID_ARGUMENT;
    if (!std::isfinite(p->sigma) || p->sigma < 0.f) return DASH_ERR_INVALID_ARGUMENT;
    if (p->flags & ~63u) return DASH_ERR_INVALID_ARGUMENT;
    if (p->topk < 0) return DASH_ERR_INVALID_ARGUMENT;
    if (p->topk > 0 && (p->flags & DASH_FLAG_ESTIMATE_DIAGONAL)) return DASH_ERR_UNSUPPORTED;
    if (p->head_dim != 64 && p->head_dim != 128) return DASH_ERR_UNSUPPORTED;
    if (p->chunk_size != 64 && p->chunk_size != 128) return DASH_ERR_UNSUPPORTED;
    const int G = p->heads_q / p->heads_kv;
    if (!(G >= 16 ? G % 16 == 0 : 16 % G == 0)) return DASH_ERR_UNSUPPORTED;
    // Element counts must stay well inside 64-bit indexing and grid limits.
    const double elems = (double)p->batch * p->heads_q * p->seq_len * p->head_dim;
    if (elems > 4e15 || (double)p->batch * p->heads_kv > 65535.0) return DASH_ERR_UNSUPPORTED;
    s->B = p->batch;
    s->Hq = p->heads_q;
    s->Hkv = p->heads_kv;
    s->T = p->seq_len;
    s->D = p->head_dim;
    s->Bc = p->chunk_size;
    s->G = G;
    s->C = (p->seq_len + p->chunk_size - 1) / p->chunk_size;
    s->Cf = p->seq_len / p->chunk_size;
    s->W = (s->C + 63) / 64;
    return DASH_OK;
}

RouteConsts route_consts(const dash_params_t *p) {
    RouteConsts rc = {};
    const double a = p->alpha, g = p->gamma, sg = p->sigma, sd = std::sqrt((double)p->head_dim);
    rc.alpha = p->alpha;
    rc.sscale = (float)(g / sd);
    if (a == 1.0) {
        rc.kind = 0;
        rc.xscale = 0.f;
        rc.beta = 0.f;
        rc.bscale2 = 0.f;
    } else {
        rc.kind = a == 1.5 ? 1 : a == 2.0 ? 2 : 3;
        rc.xscale = (float)((a - 1.0) * g / sd);
        rc.beta = (float)(1.0 / (a - 1.0));
        rc.bscale2 = (float)(sg / (a - 1.0));
        const double b = 1.0 / (a - 1.0), br = std::round(b);
        rc.beta_int = (rc.kind == 3 && br >= 3.0 && br <= 8.0 && std::fabs(b - br) < 1e-9) ? (int)br : 0;
    }
    rc.sigma2 = (float)(sg * 1.4426950408889634);
    rc.newton_cap = (p->flags & DASH_FLAG_TEST_NEWTON_CAP) ? 1 : kNewtonCap;
    rc.est_diag = (p->flags & DASH_FLAG_ESTIMATE_DIAGONAL) ? 1 : 0;
    rc.topk = p->topk;
    if (p->topk > 0) {                     // scores as for softmax routing, uniform prior
        rc.kind = kKindTopk;
        rc.xscale = rc.sscale;
        rc.bscale2 = 0.f;
        rc.sigma2 = 0.f;
    }
    rc.inv_sqrt_d = (float)(1.0 / sd);
    return rc;
}

StageArgs stage_args(const dash_params_t *p, const Shape &s) {
    StageArgs a = {};
    a.B = s.B;
    a.Hq = s.Hq;
    a.Hkv = s.Hkv;
    a.T = s.T;
    a.D = s.D;
    a.Bc = s.Bc;
    a.G = s.G;
    a.C = s.C;
    a.Cf = s.Cf;
    a.W = s.W;
    a.rc = route_consts(p);
    a.qk_scale2 = (float)(1.4426950408889634 / std::sqrt((double)s.D));
    a.ignore_routing = (p->flags & (DASH_FLAG_DENSE | DASH_FLAG_FORCE_ALL_ACTIVE)) ? 1 : 0;
    a.t_begin = 0;
    a.t_end = s.T;
    a.vt_ready = 0;
    a.test_stall = (p->flags & DASH_FLAG_TEST_STALL_WAIT) ? 1 : 0;
    return a;
}

size_t bytes_tau(const Shape &s) { return align256((size_t)s.B * s.Hkv * s.T * 4); }
size_t bytes_summary(const Shape &s) { return align256((size_t)s.B * s.Hkv * s.Cf * s.D * 4); }
size_t bytes_mask(const Shape &s) { return align256((size_t)s.B * s.Hkv * s.T * s.W * 8); }

// V^T scratch of the 128-key-block Stage 2 kernels; 0 when none of them applies (the routed
// kernel, or with `dense` the one on pairs of SMs, which also serves fewer query heads per KV
// head).
size_t bytes_vt(const Shape &s, bool dense) {
    StageArgs a = {};
    a.D = s.D;
    a.G = s.G;
    a.Bc = s.Bc;
    a.C = s.C;
    if (!attend_fa_supported(a) && !(dense && attend_pair_supported(a))) return 0;
    return align256(attend_fa_vt_bytes(s.B, s.Hkv, s.T, s.D));
}
bool dense_flags(const dash_params_t *p) {
    return (p->flags & (DASH_FLAG_DENSE | DASH_FLAG_FORCE_ALL_ACTIVE)) != 0;
}

// The status word and the record of a run-time Stage 2 choice (bytes 0-31 of the block).
dash_status_t clear_status(void *ws, cudaStream_t st) {
    return cudaMemsetAsync(ws, 0, 32, st) == cudaSuccess ? DASH_OK : DASH_ERR_CUDA;
}

dash_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? DASH_OK : DASH_ERR_CUDA; }

}  // namespace

namespace dash {

// Workspace bytes dash_prefill carves for its scratch: the status word, tau, and the
// summaries and mask words the caller does not supply (the V^T scratch is optional and not
// counted).  0 on bad parameters.
size_t prefill_scratch_bytes(const dash_params_t *p, bool has_summary, bool has_mask) {
    Shape s;
    if (check_params(p, &s) != DASH_OK) return 0;
    const bool dense = (p->flags & DASH_FLAG_DENSE) != 0;
    size_t need = kStatusBytes + bytes_tau(s);
    if (!dense && !has_summary) need += bytes_summary(s);
    if (!dense && !has_mask) need += bytes_mask(s);
    return need;
}

}  // namespace dash

namespace {

// One decode step on a contiguous cache (block_table null) or a paged one.
dash_status_t decode_common(const dash_params_t *p, const void *q, const void *k_cache,
                            const void *v_cache, const int32_t *block_table, int max_blocks,
                            int n_pages, const int32_t *seq_lens, const float *summary_cache,
                            const float *head_cls, void *out, float *prob,
                            uint64_t *active_blocks, void *ws, size_t ws_bytes, void *stream,
                            const void *k_new = nullptr, const void *v_new = nullptr,
                            int32_t *seq_inout = nullptr, float *summary_out = nullptr) {
    Shape s;
    dash_status_t rc = check_params(p, &s);
    if (rc != DASH_OK) return rc;
    if (p->flags & (DASH_FLAG_DENSE | DASH_FLAG_FORCE_ALL_ACTIVE)) return DASH_ERR_UNSUPPORTED;
    const bool step = k_new != nullptr;
    if (step && (!v_new || !seq_inout || !summary_out || !head_cls || !aligned16(k_new) ||
                 !aligned16(v_new)))
        return DASH_ERR_INVALID_ARGUMENT;
    if (step && ws_bytes < kStatusBytes + align256((size_t)s.B * 4)) return DASH_ERR_WORKSPACE_TOO_SMALL;
    if (!q || !k_cache || !v_cache || !seq_lens || !summary_cache || !out || !ws)
        return DASH_ERR_INVALID_ARGUMENT;
    if ((p->flags & DASH_FLAG_ESTIMATE_DIAGONAL) && !head_cls) return DASH_ERR_INVALID_ARGUMENT;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(summary_cache) ||
        !aligned16(head_cls) ||
        !aligned16(out) || !aligned16(prob) || !aligned16(active_blocks) ||
        (reinterpret_cast<uintptr_t>(seq_lens) & 3u) || (reinterpret_cast<uintptr_t>(ws) & 255u))
        return DASH_ERR_INVALID_ARGUMENT;
    if (!decode_supported(s.G, s.C, s.D)) return DASH_ERR_UNSUPPORTED;
    if (ws_bytes < kStatusBytes) return DASH_ERR_WORKSPACE_TOO_SMALL;
    DecodeArgs a = {};
    a.q = q;
    a.k = k_cache;
    a.v = v_cache;
    a.seq_lens = seq_lens;
    a.summary = summary_cache;
    a.head_cls = head_cls;
    a.block_table = block_table;
    a.max_blocks = max_blocks;
    a.n_pages = n_pages;
    a.out = out;
    a.p = prob;
    a.mask = active_blocks;
    a.B = s.B;
    a.Hq = s.Hq;
    a.Hkv = s.Hkv;
    a.cap = s.T;
    a.D = s.D;
    a.Bc = s.Bc;
    a.G = s.G;
    a.Ccap = s.C;
    a.Cf = s.Cf;
    a.Wcap = s.W;
    a.rc = route_consts(p);
    a.qk_scale2 = (float)(1.4426950408889634 / std::sqrt((double)s.D));
    a.status = static_cast<uint32_t *>(ws);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (step) {
        a.k_new = k_new;
        a.v_new = v_new;
        a.seq_out = seq_inout;
        a.summary_out = summary_out;
        // Per-sequence arrival counters: in the status block's free bytes (32..255) for up to
        // 56 sequences, else after the block.  The workspace starts zeroed and every step
        // leaves the counters at zero (the last arrival resets its own), and the status word
        // is not cleared: a step is one launch with no memset node between the steps of a
        // captured loop (a memset per step cost 4 us of a 29 us step at 16 x 64K).
        unsigned char *w = static_cast<unsigned char *>(ws);
        a.arrive = reinterpret_cast<int *>(w + (s.B <= (int)((kStatusBytes - 32) / 4) ? 32 : kStatusBytes));
        return from_cuda(launch_decode(a, st));
    }
    if ((rc = clear_status(ws, st)) != DASH_OK) return rc;
    return from_cuda(launch_decode(a, st));
}

}  // namespace

extern "C" {

const char *dash_status_string(dash_status_t s) {
    switch (s) {
        case DASH_OK: return "DASH_OK";
        case DASH_ERR_INVALID_ARGUMENT: return "DASH_ERR_INVALID_ARGUMENT";
        case DASH_ERR_UNSUPPORTED: return "DASH_ERR_UNSUPPORTED";
        case DASH_ERR_WORKSPACE_TOO_SMALL: return "DASH_ERR_WORKSPACE_TOO_SMALL";
        case DASH_ERR_CUDA: return "DASH_ERR_CUDA";
        case DASH_ERR_DEVICE_TIMEOUT: return "DASH_ERR_DEVICE_TIMEOUT";
        case DASH_ERR_RANGE_CLAMPED: return "DASH_ERR_RANGE_CLAMPED";
        case DASH_ERR_BOUNDS: return "DASH_ERR_BOUNDS";
    }
    return "DASH_ERR_UNKNOWN";
}

size_t dash_prefill_workspace_size(const dash_params_t *p) {
    Shape s;
    if (check_params(p, &s) != DASH_OK) return 0;
    return kStatusBytes + bytes_tau(s) + bytes_summary(s) + bytes_mask(s) + bytes_vt(s, dense_flags(p));
}

size_t dash_attend_workspace_size(const dash_params_t *p) {
    Shape s;
    if (check_params(p, &s) != DASH_OK) return 0;
    return kStatusBytes + bytes_vt(s, dense_flags(p));
}

dash_status_t dash_prefill(const dash_params_t *p, const void *q, const void *k, const void *v,
                           const float *head_cls, void *out, float *summary_k, float *prob,
                           uint64_t *active_blocks, void *ws, size_t ws_bytes, void *stream) {
    Shape s;
    dash_status_t rc = check_params(p, &s);
    if (rc != DASH_OK) return rc;
    const bool dense = (p->flags & DASH_FLAG_DENSE) != 0;
    if (!q || !k || !v || !out || !ws) return DASH_ERR_INVALID_ARGUMENT;
    if (!dense && !head_cls) return DASH_ERR_INVALID_ARGUMENT;
    if (dense && (summary_k || prob || active_blocks)) return DASH_ERR_INVALID_ARGUMENT;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
        !aligned16(head_cls) || !aligned16(summary_k) || !aligned16(prob) ||
        !aligned16(active_blocks) || (reinterpret_cast<uintptr_t>(ws) & 255u))
        return DASH_ERR_INVALID_ARGUMENT;
    if (!dense && route_rows_per_cta(s.C, s.D) == 0) return DASH_ERR_UNSUPPORTED;
    if (ws_bytes < prefill_scratch_bytes(p, summary_k != nullptr, active_blocks != nullptr))
        return DASH_ERR_WORKSPACE_TOO_SMALL;

    unsigned char *w = static_cast<unsigned char *>(ws);
    StageArgs a = stage_args(p, s);
    a.q = q;
    a.k = k;
    a.v = v;
    a.head_cls = head_cls;
    a.out = out;
    a.p = prob;
    a.status = reinterpret_cast<uint32_t *>(w);
    size_t off = kStatusBytes;
    a.tau = reinterpret_cast<float *>(w + off);
    off += bytes_tau(s);
    if (!dense) {
        if (summary_k) {
            a.summary = summary_k;
        } else {
            a.summary = reinterpret_cast<float *>(w + off);
            off += bytes_summary(s);
        }
        if (active_blocks) {
            a.mask = active_blocks;
        } else {
            a.mask = reinterpret_cast<uint64_t *>(w + off);
            off += bytes_mask(s);
        }
    }
    const size_t vt = bytes_vt(s, dense_flags(p));
    if (vt && ws_bytes >= off + vt) a.vt = w + off;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if ((rc = clear_status(ws, st)) != DASH_OK) return rc;
    // Fused route-and-attend on request, where the 128-key-block kernel takes it: Stage 2 runs
    // Stage 1 for its own tiles (liuzhao09.github.io "DashAttention 精读", section 2: fused
    // kernels), so q is read once and the routing never makes a round trip through memory.
    a.fuse_route = fuse_requested(p) && !dense && attend_kernel(a) == AttendKernel::kFa &&
                   attend_fa_fuse_supported(a);
    if (!dense) {
        if ((rc = from_cuda(launch_stage0(a, nullptr, 0, st))) != DASH_OK) return rc;
        if (!a.fuse_route && (rc = from_cuda(launch_route(a, st))) != DASH_OK) return rc;
    }
    return from_cuda(launch_attend(a, st));
}

// Keys go up in pieces that double in slices: slice 0, slices 1-2, slices 3-6, ... (a piece
// starts at slice 2^j - 1). The first slice's computation starts after a small copy, and the
// number of copies and of Stage 0 / transpose launches stays logarithmic in the slices.
// Returns the slice after the piece that starts at slice i, or 0 when no piece starts there.
static int kv_piece_end(int i, int n) {
    return ((i + 1) & i) == 0 ? std::min(n, 2 * i + 1) : 0;
}

dash_status_t dash_prefill_host(const dash_params_t *p, const void *q_host, const void *k_host,
                                const void *v_host, const float *head_cls_host, void *out_host,
                                void *q, void *k, void *v, float *head_cls, void *out, void *ws,
                                size_t ws_bytes, int n_slices, void *stream, void *h2d_stream,
                                void *d2h_stream) {
    Shape s;
    dash_status_t rc = check_params(p, &s);
    if (rc != DASH_OK) return rc;
    const bool dense = (p->flags & DASH_FLAG_DENSE) != 0;
    if (!q_host || !k_host || !v_host || !out_host || (!dense && !head_cls_host) || !q || !k ||
        !v || !out || (!dense && !head_cls) || !ws || n_slices < 1)
        return DASH_ERR_INVALID_ARGUMENT;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(head_cls) ||
        (reinterpret_cast<uintptr_t>(ws) & 255u))
        return DASH_ERR_INVALID_ARGUMENT;
    if (!dense && route_rows_per_cta(s.C, s.D) == 0) return DASH_ERR_UNSUPPORTED;
    if (ws_bytes < dash_prefill_workspace_size(p)) return DASH_ERR_WORKSPACE_TOO_SMALL;

    unsigned char *w = static_cast<unsigned char *>(ws);
    StageArgs a = stage_args(p, s);
    a.q = q;
    a.k = k;
    a.v = v;
    a.head_cls = head_cls;
    a.out = out;
    a.status = reinterpret_cast<uint32_t *>(w);
    size_t off = kStatusBytes;
    a.tau = reinterpret_cast<float *>(w + off);
    off += bytes_tau(s);
    if (!dense) {
        a.summary = reinterpret_cast<float *>(w + off);
        off += bytes_summary(s);
        a.mask = reinterpret_cast<uint64_t *>(w + off);
        off += bytes_mask(s);
    }
    const size_t vt = bytes_vt(s, dense_flags(p));
    if (vt) a.vt = w + off;
    // Row slices only where the Stage 2 kernel takes a row range; each slice a multiple of
    // 128 rows (the last one ragged).
    const bool sliceable = a.vt && (a.ignore_routing ? (attend_pair_supported(a) || attend_fa_supported(a))
                                                     : attend_fa_supported(a));
    constexpr int kMaxSlices = 64;
    const int want = std::min(n_slices, kMaxSlices);
    int rows = s.T;
    if (sliceable && want > 1) rows = ((s.T + want - 1) / want + 127) / 128 * 128;
    const int n = (s.T + rows - 1) / rows;                  // <= want

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaStream_t hs = static_cast<cudaStream_t>(h2d_stream);
    cudaStream_t ds = static_cast<cudaStream_t>(d2h_stream);
    const size_t row_bytes = (size_t)s.D * 2;
    const size_t plane = (size_t)s.T * row_bytes;          // one (b, h) plane of q or out
    const int n_ev = 3 * n + 2;
    cudaEvent_t ev[3 * kMaxSlices + 2];
    int made = 0;
    cudaError_t e = cudaSuccess;
    for (; made < n_ev && e == cudaSuccess; ++made) e = cudaEventCreateWithFlags(&ev[made], cudaEventDisableTiming);
    if (e != cudaSuccess) --made;
    cudaEvent_t &e_done = ev[0], &e_start = ev[1];
    auto e_kv = [&](int i) -> cudaEvent_t & { return ev[2 + i]; };
    auto e_q = [&](int i) -> cudaEvent_t & { return ev[2 + n + i]; };
    auto e_o = [&](int i) -> cudaEvent_t & { return ev[2 + 2 * n + i]; };
    auto ok = [&](cudaError_t r) { if (e == cudaSuccess) e = r; return e == cudaSuccess; };
    // Rows [t0, t1) of every (b, h) plane of a [B, H, T, D] tensor in one strided copy.
    auto rows_copy = [&](void *dst, const void *src, int planes, size_t t0, size_t t1,
                         cudaMemcpyKind kind, cudaStream_t cs) {
        return cudaMemcpy2DAsync(static_cast<unsigned char *>(dst) + t0 * row_bytes, plane,
                                 static_cast<const unsigned char *>(src) + t0 * row_bytes, plane,
                                 (t1 - t0) * row_bytes, (size_t)planes, kind, cs);
    };
    // Causal attention and routing of the rows below t1 read only keys below t1 and the
    // summaries of the chunks that end at or before t1. So slice i uploads its own rows of
    // K, V and q; the compute stream summarises the chunks completed by the new keys,
    // transposes the new rows of V, then routes and attends the slice.
    // Host -> device: head_cls, then per slice K, V rows and q rows.
    // Compute: per slice Stage 0 on the new chunks once K has landed, Stages 1-2 once q has.
    // Device -> host: out of slice i once it is computed.
    if (e == cudaSuccess) {
        // Both copy streams start after the work already queued on the compute stream (which
        // may still use these buffers).
        ok(cudaEventRecord(e_start, st));
        ok(cudaStreamWaitEvent(hs, e_start, 0));
        ok(cudaStreamWaitEvent(ds, e_start, 0));
        if (!dense) ok(cudaMemcpyAsync(head_cls, head_cls_host, (size_t)s.Hkv * s.D * 4, cudaMemcpyHostToDevice, hs));
        for (int i = 0; i < n; ++i) {
            const size_t t0 = (size_t)i * rows, t1 = (size_t)std::min(s.T, (i + 1) * rows);
            if (const int pe = kv_piece_end(i, n)) {
                const size_t k1 = (size_t)std::min(s.T, pe * rows);
                ok(rows_copy(k, k_host, s.B * s.Hkv, t0, k1, cudaMemcpyHostToDevice, hs));
                ok(rows_copy(v, v_host, s.B * s.Hkv, t0, k1, cudaMemcpyHostToDevice, hs));
                ok(cudaEventRecord(e_kv(i), hs));
            }
            ok(rows_copy(q, q_host, s.B * s.Hq, t0, t1, cudaMemcpyHostToDevice, hs));
            ok(cudaEventRecord(e_q(i), hs));
        }
        ok(cudaMemsetAsync(ws, 0, sizeof(uint32_t), st));
        for (int i = 0; i < n && e == cudaSuccess; ++i) {
            a.t_begin = i * rows;
            a.t_end = std::min(s.T, (i + 1) * rows);
            a.fuse_route = fuse_requested(p) && !dense && attend_kernel(a) == AttendKernel::kFa &&
                           attend_fa_fuse_supported(a);
            a.vt_ready = 1;
            if (const int pe = kv_piece_end(i, n)) {
                // A new piece of keys: summarise the chunks it completes, transpose its V rows
                // (one piece: every chunk and every key, ranges 0 meaning "all").
                const int k1 = std::min(s.T, pe * rows);
                a.s0_begin = n > 1 ? a.t_begin / s.Bc : 0;
                a.s0_end = n > 1 ? k1 / s.Bc : 0;
                a.vt_begin = n > 1 ? a.t_begin : 0;
                a.vt_end = n > 1 ? k1 : 0;
                a.vt_ready = 0;
                ok(cudaStreamWaitEvent(st, e_kv(i), 0));
                if (!dense && (n == 1 || a.s0_end > a.s0_begin)) ok(launch_stage0(a, nullptr, 0, st));
            }
            ok(cudaStreamWaitEvent(st, e_q(i), 0));
            if (!dense && !a.fuse_route) ok(launch_route(a, st));
            ok(launch_attend(a, st));
            ok(cudaEventRecord(e_o(i), st));
        }
        for (int i = 0; i < n && e == cudaSuccess; ++i) {
            ok(cudaStreamWaitEvent(ds, e_o(i), 0));
            ok(rows_copy(out_host, out, s.B * s.Hq, (size_t)i * rows, (size_t)std::min(s.T, (i + 1) * rows),
                         cudaMemcpyDeviceToHost, ds));
        }
        // The compute stream ends after the last copy back, so synchronising it covers the call.
        ok(cudaEventRecord(e_done, ds));
        ok(cudaStreamWaitEvent(st, e_done, 0));
    }
    for (int i = 0; i < made; ++i) cudaEventDestroy(ev[i]);   // released once complete
    return from_cuda(e);
}

dash_status_t dash_stage0(const dash_params_t *p, const void *k, const float *head_cls,
                          float *summary_k, void *ws, size_t ws_bytes, void *stream) {
    Shape s;
    dash_status_t rc = check_params(p, &s);
    if (rc != DASH_OK) return rc;
    if (!k || !head_cls || (!summary_k && s.Cf > 0) || !ws) return DASH_ERR_INVALID_ARGUMENT;
    if (!aligned16(k) || !aligned16(head_cls) || !aligned16(summary_k) ||
        (reinterpret_cast<uintptr_t>(ws) & 255u))
        return DASH_ERR_INVALID_ARGUMENT;
    if (ws_bytes < kStatusBytes) return DASH_ERR_WORKSPACE_TOO_SMALL;
    StageArgs a = stage_args(p, s);
    a.k = k;
    a.head_cls = head_cls;
    a.summary = summary_k;
    a.status = static_cast<uint32_t *>(ws);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if ((rc = clear_status(ws, st)) != DASH_OK) return rc;
    return from_cuda(launch_stage0(a, nullptr, 0, st));
}

dash_status_t dash_route(const dash_params_t *p, const void *q, const float *summary_k,
                         float *tau, float *prob, uint64_t *active_blocks, void *ws,
                         size_t ws_bytes, void *stream) {
    Shape s;
    dash_status_t rc = check_params(p, &s);
    if (rc != DASH_OK) return rc;
    if (!q || (!summary_k && s.Cf > 0) || !tau || !active_blocks || !ws)
        return DASH_ERR_INVALID_ARGUMENT;
    // The estimated diagonal needs the keys and head_cls, which this entry point does not take.
    if (p->flags & DASH_FLAG_ESTIMATE_DIAGONAL) return DASH_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(summary_k) || !aligned16(tau) || !aligned16(prob) ||
        !aligned16(active_blocks) || (reinterpret_cast<uintptr_t>(ws) & 255u))
        return DASH_ERR_INVALID_ARGUMENT;
    if (route_rows_per_cta(s.C, s.D) == 0) return DASH_ERR_UNSUPPORTED;
    if (ws_bytes < kStatusBytes) return DASH_ERR_WORKSPACE_TOO_SMALL;
    StageArgs a = stage_args(p, s);
    a.q = q;
    a.summary = const_cast<float *>(summary_k);
    a.tau = tau;
    a.p = prob;
    a.mask = active_blocks;
    a.status = static_cast<uint32_t *>(ws);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if ((rc = clear_status(ws, st)) != DASH_OK) return rc;
    return from_cuda(launch_route(a, st));
}

dash_status_t dash_attend(const dash_params_t *p, const void *q, const void *k, const void *v,
                          const float *summary_k, const float *tau,
                          const uint64_t *active_blocks, void *out, void *ws, size_t ws_bytes,
                          void *stream) {
    Shape s;
    dash_status_t rc = check_params(p, &s);
    if (rc != DASH_OK) return rc;
    const bool ignore = (p->flags & (DASH_FLAG_DENSE | DASH_FLAG_FORCE_ALL_ACTIVE)) != 0;
    if (!q || !k || !v || !out || !ws) return DASH_ERR_INVALID_ARGUMENT;
    if (!ignore && ((!summary_k && s.Cf > 0) || !tau || !active_blocks))
        return DASH_ERR_INVALID_ARGUMENT;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
        !aligned16(summary_k) || !aligned16(tau) || !aligned16(active_blocks) ||
        (reinterpret_cast<uintptr_t>(ws) & 255u))
        return DASH_ERR_INVALID_ARGUMENT;
    if (ws_bytes < kStatusBytes) return DASH_ERR_WORKSPACE_TOO_SMALL;
    StageArgs a = stage_args(p, s);
    a.q = q;
    a.k = k;
    a.v = v;
    a.out = out;
    a.summary = const_cast<float *>(summary_k);
    a.tau = const_cast<float *>(tau);
    a.mask = const_cast<uint64_t *>(active_blocks);
    a.status = static_cast<uint32_t *>(ws);
    const size_t vt = bytes_vt(s, dense_flags(p));
    if (vt && ws_bytes >= kStatusBytes + vt) a.vt = static_cast<unsigned char *>(ws) + kStatusBytes;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if ((rc = clear_status(ws, st)) != DASH_OK) return rc;
    return from_cuda(launch_attend(a, st));
}

dash_status_t dash_update_chunk_cache(const dash_params_t *p, const void *k_cache,
                                      const float *head_cls, const int32_t *seq_lens,
                                      int n_recent, float *summary_cache, void *ws,
                                      size_t ws_bytes, void *stream) {
    Shape s;
    dash_status_t rc = check_params(p, &s);
    if (rc != DASH_OK) return rc;
    if (!k_cache || !head_cls || !seq_lens || !summary_cache || !ws || n_recent < 1)
        return DASH_ERR_INVALID_ARGUMENT;
    if (!aligned16(k_cache) || !aligned16(head_cls) || !aligned16(summary_cache) ||
        (reinterpret_cast<uintptr_t>(seq_lens) & 3u) || (reinterpret_cast<uintptr_t>(ws) & 255u))
        return DASH_ERR_INVALID_ARGUMENT;
    if (ws_bytes < kStatusBytes) return DASH_ERR_WORKSPACE_TOO_SMALL;
    StageArgs a = stage_args(p, s);
    a.k = k_cache;
    a.head_cls = head_cls;
    a.summary = summary_cache;
    a.status = static_cast<uint32_t *>(ws);
    if (n_recent > s.Cf) n_recent = s.Cf > 0 ? s.Cf : 1;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if ((rc = clear_status(ws, st)) != DASH_OK) return rc;
    if (s.Cf == 0) return DASH_OK;
    return from_cuda(launch_stage0(a, seq_lens, n_recent, st));
}

size_t dash_decode_workspace_size(const dash_params_t *p) {
    Shape s;
    if (check_params(p, &s) != DASH_OK) return 0;
    return kStatusBytes;
}

dash_status_t dash_decode(const dash_params_t *p, const void *q, const void *k_cache,
                          const void *v_cache, const int32_t *seq_lens,
                          const float *summary_cache, const float *head_cls, void *out,
                          float *prob, uint64_t *active_blocks, void *ws, size_t ws_bytes,
                          void *stream) {
    return decode_common(p, q, k_cache, v_cache, nullptr, 0, 0, seq_lens, summary_cache,
                         head_cls, out, prob, active_blocks, ws, ws_bytes, stream);
}

dash_status_t dash_decode_paged(const dash_params_t *p, const void *q, const void *k_pool,
                                const void *v_pool, const int32_t *block_table, int max_blocks,
                                int n_pages, const int32_t *seq_lens, const float *summary_pool,
                                const float *head_cls, void *out, float *prob,
                                uint64_t *active_blocks, void *ws, size_t ws_bytes,
                                void *stream) {
    if (!p || !block_table || max_blocks < 1 || n_pages < 1 ||
        (reinterpret_cast<uintptr_t>(block_table) & 3u))
        return DASH_ERR_INVALID_ARGUMENT;
    if ((long long)max_blocks * p->chunk_size != (long long)p->seq_len) return DASH_ERR_INVALID_ARGUMENT;
    return decode_common(p, q, k_pool, v_pool, block_table, max_blocks, n_pages, seq_lens,
                         summary_pool, head_cls, out, prob, active_blocks, ws, ws_bytes, stream);
}

size_t dash_decode_step_workspace_size(const dash_params_t *p) {
    Shape s;
    if (check_params(p, &s) != DASH_OK) return 0;
    return kStatusBytes + align256((size_t)s.B * 4);
}

dash_status_t dash_decode_step(const dash_params_t *p, const void *q, const void *k_new,
                               const void *v_new, void *k_cache, void *v_cache, int32_t *seq_lens,
                               float *summary_cache, const float *head_cls, void *out,
                               float *prob, uint64_t *active_blocks, void *ws, size_t ws_bytes,
                               void *stream) {
    if (!k_new) return DASH_ERR_INVALID_ARGUMENT;
    return decode_common(p, q, k_cache, v_cache, nullptr, 0, 0, seq_lens, summary_cache,
                         head_cls, out, prob, active_blocks, ws, ws_bytes, stream, k_new, v_new,
                         seq_lens, summary_cache);
}

dash_status_t dash_decode_step_paged(const dash_params_t *p, const void *q, const void *k_new,
                                     const void *v_new, void *k_pool, void *v_pool,
                                     const int32_t *block_table, int max_blocks, int n_pages,
                                     int32_t *seq_lens, float *summary_pool, const float *head_cls,
                                     void *out, float *prob, uint64_t *active_blocks, void *ws,
                                     size_t ws_bytes, void *stream) {
    if (!p || !k_new || !block_table || max_blocks < 1 || n_pages < 1 ||
        (reinterpret_cast<uintptr_t>(block_table) & 3u))
        return DASH_ERR_INVALID_ARGUMENT;
    if ((long long)max_blocks * p->chunk_size != (long long)p->seq_len) return DASH_ERR_INVALID_ARGUMENT;
    return decode_common(p, q, k_pool, v_pool, block_table, max_blocks, n_pages, seq_lens,
                         summary_pool, head_cls, out, prob, active_blocks, ws, ws_bytes, stream,
                         k_new, v_new, seq_lens, summary_pool);
}

dash_status_t dash_update_chunk_cache_paged(const dash_params_t *p, const void *k_pool,
                                            const float *head_cls, const int32_t *block_table,
                                            int max_blocks, int n_pages, const int32_t *seq_lens,
                                            int n_recent, float *summary_pool, void *ws,
                                            size_t ws_bytes, void *stream) {
    Shape s;
    dash_status_t rc = check_params(p, &s);
    if (rc != DASH_OK) return rc;
    if (!k_pool || !head_cls || !block_table || !seq_lens || !summary_pool || !ws || n_recent < 1 ||
        max_blocks < 1 || n_pages < 1 || (long long)max_blocks * s.Bc != (long long)s.T)
        return DASH_ERR_INVALID_ARGUMENT;
    if (!aligned16(k_pool) || !aligned16(head_cls) || !aligned16(summary_pool) ||
        (reinterpret_cast<uintptr_t>(seq_lens) & 3u) || (reinterpret_cast<uintptr_t>(block_table) & 3u) ||
        (reinterpret_cast<uintptr_t>(ws) & 255u))
        return DASH_ERR_INVALID_ARGUMENT;
    if (ws_bytes < kStatusBytes) return DASH_ERR_WORKSPACE_TOO_SMALL;
    StageArgs a = stage_args(p, s);
    a.k = k_pool;
    a.head_cls = head_cls;
    a.summary = summary_pool;
    a.status = static_cast<uint32_t *>(ws);
    if (n_recent > s.Cf) n_recent = s.Cf;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if ((rc = clear_status(ws, st)) != DASH_OK) return rc;
    return from_cuda(launch_stage0_paged(a, seq_lens, n_recent, block_table, max_blocks, n_pages, st));
}

size_t dash_backward_workspace_size(const dash_params_t *p) {
    Shape s;
    if (check_params(p, &s) != DASH_OK) return 0;
    const size_t bhkv = (size_t)s.B * s.Hkv;
    size_t n = kStatusBytes + bytes_tau(s) + bytes_summary(s) + bytes_mask(s);
    n += 2 * align256(bhkv * s.T * s.C * 4);                     // p, d log p
    n += 3 * align256((size_t)s.B * s.Hq * s.T * 4);             // row max, sum, delta
    n += align256(bhkv * s.T * s.D * 4);                         // qbar
    n += align256(bhkv * s.C * 4) + align256(bhkv * (s.C + 1) * 8);   // list counts, offsets
    const size_t nblk = (size_t)backward_list_blocks(s.T);
    n += align256(bhkv * s.C * nblk * 4) + align256(bhkv * s.C * nblk * 8);   // per token block
    n += align256(bhkv * (size_t)backward_nnz_max(s.T, s.Bc) * 4);     // lists
    n += align256(bytes_summary(s));                             // d summaries
    return n;
}

dash_status_t dash_backward(const dash_params_t *p, const void *q, const void *k, const void *v,
                            const float *head_cls, const void *out, const void *dout, float *dq,
                            float *dk, float *dv, float *dhc, void *ws, size_t ws_bytes,
                            void *stream) {
    Shape s;
    dash_status_t rc = check_params(p, &s);
    if (rc != DASH_OK) return rc;
    if (p->flags & (DASH_FLAG_DENSE | DASH_FLAG_FORCE_ALL_ACTIVE | DASH_FLAG_ESTIMATE_DIAGONAL) ||
        p->topk > 0)
        return DASH_ERR_UNSUPPORTED;
    if (!q || !k || !v || !head_cls || !out || !dout || !dq || !dk || !dv || !dhc || !ws)
        return DASH_ERR_INVALID_ARGUMENT;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(head_cls) || !aligned16(out) ||
        !aligned16(dout) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || !aligned16(dhc) ||
        (reinterpret_cast<uintptr_t>(ws) & 255u))
        return DASH_ERR_INVALID_ARGUMENT;
    if (route_rows_per_cta(s.C, s.D) == 0) return DASH_ERR_UNSUPPORTED;
    if (ws_bytes < dash_backward_workspace_size(p)) return DASH_ERR_WORKSPACE_TOO_SMALL;
    unsigned char *w = static_cast<unsigned char *>(ws);
    const size_t bhkv = (size_t)s.B * s.Hkv;
    StageArgs a = stage_args(p, s);
    a.q = q;
    a.k = k;
    a.v = v;
    a.head_cls = head_cls;
    a.status = reinterpret_cast<uint32_t *>(w);
    size_t off = kStatusBytes;
    auto take = [&](size_t bytes) { unsigned char *r = w + off; off += align256(bytes); return r; };
    a.tau = reinterpret_cast<float *>(take((size_t)s.B * s.Hkv * s.T * 4));
    a.summary = reinterpret_cast<float *>(take((size_t)s.B * s.Hkv * s.Cf * s.D * 4));
    a.mask = reinterpret_cast<uint64_t *>(take((size_t)s.B * s.Hkv * s.T * s.W * 8));
    a.p = reinterpret_cast<float *>(take(bhkv * s.T * s.C * 4));
    BackwardBuffers bb;
    bb.dout = dout;
    bb.out = out;
    bb.dq = dq;
    bb.dk = dk;
    bb.dv = dv;
    bb.dhc = dhc;
    bb.dlogp = reinterpret_cast<float *>(take(bhkv * s.T * s.C * 4));
    bb.row_m = reinterpret_cast<float *>(take((size_t)s.B * s.Hq * s.T * 4));
    bb.row_l = reinterpret_cast<float *>(take((size_t)s.B * s.Hq * s.T * 4));
    bb.row_delta = reinterpret_cast<float *>(take((size_t)s.B * s.Hq * s.T * 4));
    bb.qbar = reinterpret_cast<float *>(take(bhkv * s.T * s.D * 4));
    bb.list_cnt = reinterpret_cast<int *>(take(bhkv * s.C * 4));
    bb.list_off = reinterpret_cast<long long *>(take(bhkv * (s.C + 1) * 8));
    const size_t nblk = (size_t)backward_list_blocks(s.T);
    bb.blk_cnt = reinterpret_cast<int *>(take(bhkv * s.C * nblk * 4));
    bb.blk_off = reinterpret_cast<long long *>(take(bhkv * s.C * nblk * 8));
    bb.list = reinterpret_cast<int *>(take(bhkv * (size_t)backward_nnz_max(s.T, s.Bc) * 4));
    bb.dsum = reinterpret_cast<float *>(take((size_t)s.B * s.Hkv * s.Cf * s.D * 4));
    bb.sigma = p->sigma;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if ((rc = clear_status(ws, st)) != DASH_OK) return rc;
    if ((rc = from_cuda(cudaMemsetAsync(bb.dlogp, 0, bhkv * s.T * s.C * 4, st))) != DASH_OK) return rc;
    if ((rc = from_cuda(cudaMemsetAsync(dhc, 0, (size_t)s.Hkv * s.D * 4, st))) != DASH_OK) return rc;
    // dk and dv are summed over the key-side kernel's slices
    const size_t kv_bytes = (size_t)s.B * s.Hkv * s.T * s.D * 4;
    if ((rc = from_cuda(cudaMemsetAsync(dk, 0, kv_bytes, st))) != DASH_OK) return rc;
    if ((rc = from_cuda(cudaMemsetAsync(dv, 0, kv_bytes, st))) != DASH_OK) return rc;
    // The forward's routing (with p), then the backward kernels.
    if ((rc = from_cuda(launch_stage0(a, nullptr, 0, st))) != DASH_OK) return rc;
    if ((rc = from_cuda(launch_route(a, st))) != DASH_OK) return rc;
    return from_cuda(launch_backward(a, bb, st));
}

const char *dash_attend_kernel_name(const dash_params_t *p, size_t ws_bytes) {
    Shape s;
    if (check_params(p, &s) != DASH_OK || ws_bytes < kStatusBytes) return "";
    StageArgs a = stage_args(p, s);
    const size_t vt = bytes_vt(s, dense_flags(p));
    // Only whether the V^T scratch fits matters for the choice, not where it is.
    static unsigned char probe;
    if (vt && ws_bytes >= kStatusBytes + vt) a.vt = &probe;
    return attend_kernel_name(attend_kernel(a));
}

int dash_prefill_kernel_count(const dash_params_t *p, size_t ws_bytes) {
    Shape s;
    if (check_params(p, &s) != DASH_OK) return 0;
    const bool dense = (p->flags & DASH_FLAG_DENSE) != 0;
    StageArgs a = stage_args(p, s);
    size_t off = kStatusBytes + bytes_tau(s);
    if (!dense) off += bytes_summary(s) + bytes_mask(s);
    const size_t vt = bytes_vt(s, dense_flags(p));
    static unsigned char probe;               // only whether V^T fits matters, as in dash_prefill
    if (vt && ws_bytes >= off + vt) a.vt = &probe;
    const AttendKernel kern = attend_kernel(a);
    if (kern == AttendKernel::kNone) return 0;
    const bool fused = fuse_requested(p) && !dense && kern == AttendKernel::kFa && attend_fa_fuse_supported(a);
    const bool with_vt = kern == AttendKernel::kFa || kern == AttendKernel::kPair || kern == AttendKernel::kFaOrWarp;
    // a run-time choice adds the cost kernel and launches both Stage 2 kernels
    const int extra = kern == AttendKernel::kFaOrWarp ? 2 : 0;
    return (dense ? 0 : 1) + (dense || fused ? 0 : 1) + (with_vt ? 1 : 0) + 1 + extra;
}

const char *dash_stage2_kernel_ran(void *ws, void *stream) {
    if (!ws) return "";
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return "";
    unsigned char id = 0;
    if (cudaMemcpy(&id, static_cast<unsigned char *>(ws) + kStatusRanOff, 1, cudaMemcpyDeviceToHost) != cudaSuccess)
        return "";
    return id == 1 ? "k_attend_fa" : id == 2 ? "k_attend" : "";
}

dash_status_t dash_read_device_status(void *ws, void *stream) {
    if (!ws) return DASH_ERR_INVALID_ARGUMENT;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return DASH_ERR_CUDA;
    uint32_t v = 0;
    if (cudaMemcpy(&v, ws, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return DASH_ERR_CUDA;
    if (v != 0 && cudaMemset(ws, 0, sizeof(uint32_t)) != cudaSuccess) return DASH_ERR_CUDA;
    return static_cast<dash_status_t>(v);
}

}  // extern "C"
