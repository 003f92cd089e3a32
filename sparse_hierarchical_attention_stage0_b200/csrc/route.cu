// route.cu -- Stage 1: alpha-entmax chunk routing for prefill.
//
// gist.science "DashAttention: Differentiable and Adaptive Sparse Hierarchical Attention",
// Technische Zusammenfassung, "Stufe 1: Entmax-Chunk-Routing": each query scores the chunk
// summaries, and w = alpha-entmax(gamma z) replaces top-k; query heads sharing a KV head
// share one sparse support.  aixai.ru "DashAttention ...", "Трёхстадийная архитектура": the
// result is handed to Stage 2 as a bit-packed active-block mask (64-bit words).
//
// CTA = (b, g, RT consecutive rows of one query chunk), 256 threads:
//   1. qbar[r] = mean of the G query heads of group g at row t0 + r     (shared memory)
//   2. x[r][c] = (qbar[r] . summary[c]) * (alpha-1) gamma / sqrt(D) for every routable
//      chunk c < c_t: 4 lanes per chunk, each owning an interleaved quarter of d (coalesced
//      64-byte reads per chunk), two chunks per lane, RT row accumulators per chunk in
//      registers, qbar from shared memory (each load feeds both chunks), slices combined with
//      route_dot's fixed order
//   3. with estimate_diagonal, one warp per row adds the diagonal chunk's score against its
//      estimated summary (diag_dot) as one more candidate;
//   4. one warp per row solves tau (warp_entmax_tau) and emits the mask words by ballot,
//      tau, and optionally the dense p row.
// No top-k list and no per-row index list is ever written.
#include "dash_common.cuh"
#include "kernels.cuh"

namespace dash {

int route_rows_per_cta(int C, int D) {
    // Rows per CTA: as many as keep about three CTAs resident per SM (24 warps to hide the
    // shared-memory and FMA latencies of the score loop), within 200 KB for one CTA when C is
    // too large for that.
    const size_t xstride = (size_t)((C + 3) & ~3);
    for (int rt : {16, 8, 4})
        if ((size_t)rt * D * 4 + (size_t)rt * xstride * 4 <= 72 * 1024) return rt;
    for (int rt : {16, 8, 4})
        if ((size_t)rt * D * 4 + (size_t)rt * xstride * 4 <= 200 * 1024) return rt;
    return 0;
}

template <int D, int RT>
__global__ void __launch_bounds__(kRouteThreads) k_route(StageArgs a) {
    extern __shared__ __align__(16) float sm[];
    const int xstride = (a.C + 3) & ~3;
    float *qbar = sm;               // [RT][D]
    float *xs = sm + RT * D;        // [RT][xstride]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bg = blockIdx.y, b = bg / a.Hkv, g = bg % a.Hkv;
    const int t0 = a.t_begin + blockIdx.x * RT;
    const int ct = t0 / a.Bc;                     // every row of the tile shares c_t
    const int n = dash_check(ct <= a.Cf, a.status) ? ct : a.Cf;   // routable chunks
    const __nv_bfloat16 *q = reinterpret_cast<const __nv_bfloat16 *>(a.q);
    const long long hstride = (long long)a.T * D;

    for (int idx = threadIdx.x; idx < RT * (D / 8); idx += kRouteThreads) {
        const int r = idx / (D / 8), d8 = (idx % (D / 8)) * 8, t = t0 + r;
        float m[8];
        if (t < a.t_end) {
            group_mean8(q + ((long long)(b * a.Hq + g * a.G) * a.T + t) * D + d8, hstride, a.G, m);
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) m[e] = 0.f;
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) qbar[r * D + d8 + e] = m[e];
    }
    __syncthreads();

    // Scores: 4 lanes per chunk (lane = 4*cc + k owns float4 groups k, k+4, ... of chunk cc),
    // two chunks per lane (cc and cc + 8), 16 chunks per warp and step; the RT rows' partial
    // dots stay in registers, and every query float4 loaded from shared memory feeds both
    // chunks (8 FMAs per load: the score loop is bound by the load/store pipe).  The slice sums
    // are combined with the order of route_dot: (p0 + p1) + (p2 + p3).
    const float scale = a.rc.kind == 0 ? a.rc.sscale : a.rc.xscale;
    const float *sumg = a.summary + (long long)bg * a.Cf * D;
    const int kslice = lane & 3, cc = lane >> 2;
    constexpr int kStep = (kRouteThreads / 32) * 16;      // chunks per CTA-wide step
    for (int cbase = warp * 16; cbase < n; cbase += kStep) {
        const int c = cbase + cc, c2 = c + 8;
        float4 cur[D / 16], cur2[D / 16];         // all loads of both slices in flight at once
        {
            const float4 *s4 = reinterpret_cast<const float4 *>(sumg + (long long)min(c, n - 1) * D);
            const float4 *t4 = reinterpret_cast<const float4 *>(sumg + (long long)min(c2, n - 1) * D);
#pragma unroll
            for (int i = 0; i < D / 16; ++i) {
                cur[i] = __ldg(s4 + 4 * i + kslice);
                cur2[i] = __ldg(t4 + 4 * i + kslice);
            }
        }
        float acc[RT], acc2[RT];
#pragma unroll
        for (int r = 0; r < RT; ++r) acc[r] = acc2[r] = 0.f;
#pragma unroll
        for (int i = 0; i < D / 16; ++i) {
            const float4 sv = cur[i], tv = cur2[i];
#pragma unroll
            for (int r = 0; r < RT; ++r) {
                const float4 qq = reinterpret_cast<const float4 *>(qbar + r * D)[4 * i + kslice];
                acc[r] = fmaf(qq.x, sv.x, acc[r]);
                acc2[r] = fmaf(qq.x, tv.x, acc2[r]);
                acc[r] = fmaf(qq.y, sv.y, acc[r]);
                acc2[r] = fmaf(qq.y, tv.y, acc2[r]);
                acc[r] = fmaf(qq.z, sv.z, acc[r]);
                acc2[r] = fmaf(qq.z, tv.z, acc2[r]);
                acc[r] = fmaf(qq.w, sv.w, acc[r]);
                acc2[r] = fmaf(qq.w, tv.w, acc2[r]);
            }
        }
#pragma unroll
        for (int r = 0; r < RT; ++r) {
            float v = acc[r], w = acc2[r];
            v = v + __shfl_xor_sync(kFull, v, 1);
            w = w + __shfl_xor_sync(kFull, w, 1);
            v = v + __shfl_xor_sync(kFull, v, 2);
            w = w + __shfl_xor_sync(kFull, w, 2);
            acc[r] = v;
            acc2[r] = w;
        }
        if (kslice == 0) {
#pragma unroll
            for (int r = 0; r < RT; ++r) {
                if (c < n) xs[r * xstride + c] = __fmul_rn(acc[r], scale);
                if (c2 < n) xs[r * xstride + c2] = __fmul_rn(acc2[r], scale);
            }
        }
    }
    __syncthreads();

    // estimate_diagonal: the diagonal chunk's score joins each row's candidates as entry n.
    const int n_eff = n + (a.rc.est_diag ? 1 : 0);
    if (a.rc.est_diag) {
        const __nv_bfloat16 *kd = reinterpret_cast<const __nv_bfloat16 *>(a.k) +
                                  ((long long)bg * a.T + (long long)ct * a.Bc) * D;
        for (int r = warp; r < RT; r += kRouteThreads / 32) {
            const int t = t0 + r;
            if (t >= a.t_end) break;
            const float dd = diag_dot<D>(kd, t - ct * a.Bc + 1, a.head_cls + (long long)g * D,
                                         qbar + r * D, a.rc.inv_sqrt_d);
            if (lane == 0) xs[r * xstride + n] = __fmul_rn(dd, scale);
        }
        __syncthreads();
    }

    for (int r = warp; r < RT; r += kRouteThreads / 32) {
        const int t = t0 + r;
        if (t >= a.t_end) break;
        const long long row = (long long)bg * a.T + t;
        const float *x = xs + r * xstride;
        if (a.rc.kind == kKindTopk) {
            // Top-k: the topk highest scores (all of them when there are no more), lower
            // index first on ties; p uniform over the selection; tau = the lowest selected.
            const bool all = n <= a.rc.topk;
            int need = 0;
            uint32_t key = 0;
            if (!all) key = warp_topk_key(x, n, a.rc.topk, need);
            float tau = __int_as_float(0x7fc00000);
            if (n > 0 && all) {
                float mn = INFINITY;
                for (int c = lane; c < n; c += 32) mn = fminf(mn, x[c]);
                tau = -warp_max(-mn);
            } else if (n > 0) {
                tau = key_f32(key);
            }
            if (lane == 0) a.tau[row] = tau;
            const float pv = n > 0 ? 1.f / (float)min(n, a.rc.topk) : 0.f;
            uint64_t *mrow = a.mask + row * a.W;
            float *prow = a.p ? a.p + row * a.C : nullptr;
            int run = 0;
            for (int w = 0; w < a.W; ++w) {
                const int c0 = w * 64 + lane, c1 = c0 + 32;
                const bool s0 = topk_selected(x, c0, n, all, key, need, run);
                const bool s1 = topk_selected(x, c1, n, all, key, need, run);
                const unsigned lo = __ballot_sync(kFull, c0 == ct || s0);
                const unsigned hi = __ballot_sync(kFull, c1 == ct || s1);
                if (lane == (w & 31)) mrow[w] = ((uint64_t)hi << 32) | lo;
                if (prow) {
                    if (c0 < a.C) prow[c0] = s0 ? pv : 0.f;
                    if (c1 < a.C) prow[c1] = s1 ? pv : 0.f;
                }
            }
            continue;
        }
        float tau = n_eff > 0 ? warp_entmax_tau(x, n_eff, a.rc, a.status) : __int_as_float(0x7fc00000);
        if (lane == 0) a.tau[row] = tau;
        uint64_t *mrow = a.mask + row * a.W;
        for (int w = 0; w < a.W; ++w) {
            const int c0 = w * 64 + lane, c1 = c0 + 32;
            bool p0 = c0 == ct || (c0 < n && (a.rc.kind == 0 || __fsub_rn(x[c0], tau) > 0.f));
            bool p1 = c1 == ct || (c1 < n && (a.rc.kind == 0 || __fsub_rn(x[c1], tau) > 0.f));
            unsigned lo = __ballot_sync(kFull, p0), hi = __ballot_sync(kFull, p1);
            if (lane == (w & 31)) mrow[w] = ((uint64_t)hi << 32) | lo;
        }
        if (a.p) {
            float *prow = a.p + row * a.C;
            for (int c = lane; c < a.C; c += 32) {
                float val = 0.f;
                if (c < n_eff) {
                    if (a.rc.kind == 0) {
                        val = expf(x[c] - tau);
                    } else {
                        float m = __fsub_rn(x[c], tau);
                        val = m > 0.f ? pow_beta(m, a.rc) : 0.f;
                    }
                }
                prow[c] = val;
            }
        }
    }
}

template <int D, int RT>
static cudaError_t launch_route_t(const StageArgs &a, cudaStream_t st) {
    const int xstride = (a.C + 3) & ~3;
    size_t smem = ((size_t)RT * D + (size_t)RT * xstride) * sizeof(float);
    auto kern = k_route<D, RT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((a.t_end - a.t_begin + RT - 1) / RT, a.B * a.Hkv);
    kern<<<grid, kRouteThreads, smem, st>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_route(const StageArgs &a, cudaStream_t st) {
    const int rt = route_rows_per_cta(a.C, a.D);
    if (a.D == 128) {
        if (rt == 16) return launch_route_t<128, 16>(a, st);
        if (rt == 8) return launch_route_t<128, 8>(a, st);
        if (rt == 4) return launch_route_t<128, 4>(a, st);
    } else if (a.D == 64) {
        if (rt == 16) return launch_route_t<64, 16>(a, st);
        if (rt == 8) return launch_route_t<64, 8>(a, st);
        if (rt == 4) return launch_route_t<64, 4>(a, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace dash
