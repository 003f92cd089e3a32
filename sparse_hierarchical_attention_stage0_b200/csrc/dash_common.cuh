// dash_common.cuh -- device helpers shared by the libdash kernels (sm_100a).
//
// The routing arithmetic (group-mean query, routing dot product, entmax threshold) lives
// here once, so that Stage 1 (dash_route), Stage 2 (dash_attend, which recomputes the bias
// of each active chunk) and decode produce bit-identical values: every dot product is the
// same sequential chain of fmaf over d = 0..D-1, every mean the same ordered sum.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/dash.h"

namespace dash {

constexpr float kLog2e = 1.4426950408889634f;
constexpr unsigned kFull = 0xffffffffu;
// Time limit of every bounded device wait (measured on %globaltimer, so the bound holds
// whatever time each try_wait spends suspended), and iteration cap of the entmax Newton solve.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;
constexpr int kNewtonCap = 96;

// ---------------------------------------------------------------- status word
// The first 4 bytes of every workspace; the first error code written wins.
__device__ __forceinline__ void report(uint32_t *status, uint32_t code) {
    if (status) atomicCAS(status, 0u, code);
}

// Device-side bounds checks of the DASH_DEBUG build (build.py --debug -> libdash_debug.so):
// dash_check(ok, status) returns ok; a false check is reported as DASH_ERR_BOUNDS through the
// status word, and the caller then skips (or clamps) the access it guards.  In the release
// build it returns true and compiles away.
__device__ __forceinline__ bool dash_check(bool ok, uint32_t *status) {
#ifdef DASH_DEBUG
    if (!ok) report(status, DASH_ERR_BOUNDS);
    return ok;
#else
    (void)ok;
    (void)status;
    return true;
#endif
}

// ---------------------------------------------------------------- warp reductions
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
    return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, o));
    return v;
}
__device__ __forceinline__ int warp_sum_i(int v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
    return v;
}

// ---------------------------------------------------------------- smem / async copies
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16-byte cp.async (L2 only); src_bytes = 0 fills zeros without reading global memory.
__device__ __forceinline__ void cp_async16(void *smem, const void *gmem, int src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_u32(smem)),
                 "l"(gmem), "r"(src_bytes)
                 : "memory");
}
// 4-byte cp.async (through L1), for scattered scalars.
__device__ __forceinline__ void cp_async4(void *smem, const void *gmem) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(smem_u32(smem)), "l"(gmem)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;\n" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// mbarrier + bulk (TMA engine) copy global -> shared.
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_g2s(void *smem, const void *gmem, uint32_t bytes,
                                         uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, "
        "[%3];\n" ::"r"(smem_u32(smem)),
        "l"(gmem), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ unsigned long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
// Bounded wait on an mbarrier phase; false once kWaitLimitNs has elapsed without it.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = global_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (global_ns() - t0 > kWaitLimitNs) return false;
    }
}

// ---------------------------------------------------------------- ldmatrix / mma.sync
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void *smem) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_u32(smem)));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const void *smem) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_u32(smem)));
}
// D += A(16x16 bf16, row) * B(16x8 bf16, col), fp32 accumulate.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4],
                                               uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, "
        "{%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}
__device__ __forceinline__ float bf16_round(float x) {
    return __bfloat162float(__float2bfloat16_rn(x));
}
// 2^x on the SFU (used only for attention probabilities, which are rounded to bf16).
__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
    return y;
}

// ---------------------------------------------------------------- routing arithmetic
// Group-mean query element: (sum_{h<G} q_h) / G, summed in head order.
__device__ __forceinline__ float group_mean_elem(const __nv_bfloat16 *q0, long long head_stride,
                                                 int G) {
    float s = 0.f;
    for (int h = 0; h < G; ++h) s += __bfloat162float(q0[h * head_stride]);
    return s / (float)G;
}
// The same for 8 consecutive dims (q0 16-byte aligned): one 16-byte load per head, all loads
// issued before the ordered sums; element-wise bit-identical to group_mean_elem.
__device__ __forceinline__ void group_mean8(const __nv_bfloat16 *q0, long long head_stride, int G,
                                            float (&out)[8]) {
#pragma unroll
    for (int e = 0; e < 8; ++e) out[e] = 0.f;
    int h = 0;
    for (; h + 4 <= G; h += 4) {
        uint4 v[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) v[j] = __ldg(reinterpret_cast<const uint4 *>(q0 + (h + j) * head_stride));
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const __nv_bfloat162 *b2 = reinterpret_cast<const __nv_bfloat162 *>(&v[j]);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(b2[e]);
                out[2 * e] += f.x;
                out[2 * e + 1] += f.y;
            }
        }
    }
    for (; h < G; ++h) {
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(q0 + h * head_stride));
        const __nv_bfloat162 *b2 = reinterpret_cast<const __nv_bfloat162 *>(&v);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(b2[e]);
            out[2 * e] += f.x;
            out[2 * e + 1] += f.y;
        }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) out[e] = out[e] / (float)G;
}

// Routing dot product qbar . S_c with one fixed summation order, shared by every kernel that
// needs it: d is split into 4 interleaved slices of float4 groups (slice k = groups k, k+4,
// k+8, ...), each slice is one sequential fmaf chain in increasing d, and the slice sums are
// combined as (p0 + p1) + (p2 + p3).  The routing kernel computes the slices in 4 lanes and
// combines them with two xor-shuffles, which yields exactly these bits.
template <int D>
__device__ __forceinline__ float route_dot(const float *qbar, const float *srow) {
    const float4 *s4 = reinterpret_cast<const float4 *>(srow);
    const float4 *q4 = reinterpret_cast<const float4 *>(qbar);
    float p[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        float acc = 0.f;
#pragma unroll
        for (int i = 0; i < D / 16; ++i) {
            const float4 sv = __ldg(s4 + 4 * i + k);
            const float4 qv = q4[4 * i + k];
            acc = fmaf(qv.x, sv.x, acc);
            acc = fmaf(qv.y, sv.y, acc);
            acc = fmaf(qv.z, sv.z, acc);
            acc = fmaf(qv.w, sv.w, acc);
        }
        p[k] = acc;
    }
    return (p[0] + p[1]) + (p[2] + p[3]);
}

// RouteConsts::kind of top-k routing (the k highest scores, uniform prior in Stage 2).
constexpr int kKindTopk = 4;

// Routing scores of RT query rows against chunks [0, n) into xs[r * xstride + c], computed
// by n_warps warps (this one is warp_idx of them): 4 lanes per chunk, each an interleaved
// quarter of d as one sequential fmaf chain, two chunks (c, c + 8) per lane, slices combined
// as (p0 + p1) + (p2 + p3) -- route_dot's order, so every score has route_dot's bits.  The
// summary rows are loaded one float4 group at a time (few registers: usable inside a kernel
// with a tight register budget).  qbar: RT rows of D in shared memory, qstride floats apart.
template <int D, int RT>
__device__ __forceinline__ void route_scores_lean(float *xs, int xstride, const float *qbar,
                                                  int qstride, const float *sumg, int n,
                                                  int warp_idx, int n_warps, float scale) {
    const int lane = threadIdx.x & 31;
    const int kslice = lane & 3, cc = lane >> 2;
    for (int cbase = warp_idx * 16; cbase < n; cbase += n_warps * 16) {
        const int c = cbase + cc, c2 = c + 8;
        const float4 *s4 = reinterpret_cast<const float4 *>(sumg + (long long)min(c, n - 1) * D);
        const float4 *t4 = reinterpret_cast<const float4 *>(sumg + (long long)min(c2, n - 1) * D);
        float acc[RT], acc2[RT];
#pragma unroll
        for (int r = 0; r < RT; ++r) acc[r] = acc2[r] = 0.f;
#pragma unroll 2
        for (int i = 0; i < D / 16; ++i) {
            const float4 sv = __ldg(s4 + 4 * i + kslice), tv = __ldg(t4 + 4 * i + kslice);
#pragma unroll
            for (int r = 0; r < RT; ++r) {
                const float4 qq = reinterpret_cast<const float4 *>(qbar + r * qstride)[4 * i + kslice];
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
            if (kslice == 0) {
                if (c < n) xs[r * xstride + c] = __fmul_rn(v, scale);
                if (c2 < n) xs[r * xstride + c2] = __fmul_rn(w, scale);
            }
        }
    }
}

// Constants of the routing, computed once on the host.
struct RouteConsts {
    float xscale;     // (alpha-1) * gamma / sqrt(D): x_c = dot * xscale (alpha > 1)
    float sscale;     // gamma / sqrt(D): s_c = dot * sscale (alpha = 1)
    float alpha;
    float beta;       // 1 / (alpha-1)  (alpha > 1)
    float bscale2;    // log2 of the prior: bias2 = bscale2 * log2(m) with bscale2 = sigma*beta
    float sigma2;     // sigma * log2(e) (alpha = 1: bias2 = sigma2 * (s - lse))
    int kind;         // 0: softmax (alpha = 1), 1: alpha = 1.5, 2: alpha = 2, 3: other alpha,
                      // kKindTopk: top-k routing
    int topk;         // k of top-k routing
    int newton_cap;   // iteration cap of the Newton solve (kNewtonCap; 1 under the test hook)
    int est_diag;     // estimate_diagonal: the diagonal chunk joins the entmax (diag_dot)
    float inv_sqrt_d; // 1 / sqrt(D): Stage 0's logit scale
    int beta_int;     // kind 3: beta when it is an integer 3..8 (alpha = 1 + 1/beta), else 0;
                      // the powers m^beta, m^(beta-1) are then products, not powf
};

// m^e for a small integer e >= 0 (products, left to right).
__device__ __forceinline__ float ipow(float m, int e) {
    float r = 1.f;
    for (int i = 0; i < e; ++i) r = __fmul_rn(r, m);
    return r;
}
// The same product chain with the exponent known at compile time (E >= 1): bit-identical to
// ipow(m, E), and ipow_c<E - 1>(m) * m is ipow(m, E).
template <int E>
__device__ __forceinline__ float ipow_c(float m) {
    float r = m;
#pragma unroll
    for (int i = 1; i < E; ++i) r = __fmul_rn(r, m);
    return r;
}

// Stage 0 summary of one chunk by one warp: l_j = head_cls . k_j / sqrt(D),
// summary = sum_j exp(l_j - max) k_j / sum_j exp(l_j - max); ks: the chunk's BC keys
// ([BC][D] bf16, shared or global memory), out: D floats.  The prefill / cache-update kernel
// and the decode step both call it, so a chunk's summary has the same bits either way.
template <int D, int BC>
__device__ __forceinline__ void summarize_chunk_warp(const __nv_bfloat16 *ks, const float *hc,
                                                     float *out) {
    constexpr int PER = D / 32;          // dims per lane
    constexpr int SLOTS = BC / 32;       // logits kept per lane
    const int lane = threadIdx.x & 31;
    float h[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) h[i] = hc[lane * PER + i];
    const float inv_sqrt_d = rsqrtf((float)D);
    float logit[SLOTS];
#pragma unroll
    for (int i = 0; i < SLOTS; ++i) logit[i] = 0.f;
#pragma unroll
    for (int sl = 0; sl < SLOTS; ++sl) {
#pragma unroll 4
        for (int jj = 0; jj < 32; ++jj) {
            const __nv_bfloat16 *kr = ks + (sl * 32 + jj) * D + lane * PER;
            float part = 0.f;
#pragma unroll
            for (int i = 0; i < PER; ++i) part = fmaf(h[i], __bfloat162float(kr[i]), part);
            part = warp_sum(part);
            if (jj == lane) logit[sl] = part * inv_sqrt_d;
        }
    }
    float mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < SLOTS; ++i) mx = fmaxf(mx, logit[i]);
    mx = warp_max(mx);
    float den = 0.f;
#pragma unroll
    for (int i = 0; i < SLOTS; ++i) { logit[i] = expf(logit[i] - mx); den += logit[i]; }
    den = warp_sum(den);
    float acc[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) acc[i] = 0.f;
#pragma unroll
    for (int sl = 0; sl < SLOTS; ++sl) {
#pragma unroll 4
        for (int jj = 0; jj < 32; ++jj) {
            float w = __shfl_sync(kFull, logit[sl], jj);
            const __nv_bfloat16 *kr = ks + (sl * 32 + jj) * D + lane * PER;
#pragma unroll
            for (int i = 0; i < PER; ++i) acc[i] = fmaf(w, __bfloat162float(kr[i]), acc[i]);
        }
    }
#pragma unroll
    for (int i = 0; i < PER; ++i) out[lane * PER + i] = acc[i] / den;
}

// estimate_diagonal: the routing dot qbar . dsum of the diagonal chunk of one row, where dsum
// is Stage 0's summary taken over the n_vis keys of that chunk the row can see:
// dsum = sum_j w_j k_j, w = softmax_j(hc . k_j / sqrt(D)), so qbar . dsum = sum_j w_j (qbar . k_j).
// keys: the chunk's first key, bf16 rows of D (16-byte aligned); 1 <= n_vis <= 128; all 32
// lanes of one warp call it and get the same value.
// kCoherent: the keys may have been written earlier in the same kernel (plain loads instead
// of the read-only path).
template <int D, bool kCoherent = false>
__device__ __forceinline__ float diag_dot(const __nv_bfloat16 *keys, int n_vis, const float *hc,
                                          const float *qbar, float inv_sqrt_d) {
    const int lane = threadIdx.x & 31;
    float l[4], kq[4];
    float mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int j = lane + 32 * i;
        l[i] = -INFINITY;
        kq[i] = 0.f;
        if (j < n_vis) {
            const uint4 *kr = reinterpret_cast<const uint4 *>(keys + (long long)j * D);
            float a = 0.f, b = 0.f;
#pragma unroll 4
            for (int d8 = 0; d8 < D / 8; ++d8) {
                const uint4 v = kCoherent ? kr[d8] : __ldg(kr + d8);
                const __nv_bfloat162 *b2 = reinterpret_cast<const __nv_bfloat162 *>(&v);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 f = __bfloat1622float2(b2[e]);
                    a = fmaf(__ldg(hc + 8 * d8 + 2 * e), f.x, a);
                    a = fmaf(__ldg(hc + 8 * d8 + 2 * e + 1), f.y, a);
                    b = fmaf(qbar[8 * d8 + 2 * e], f.x, b);
                    b = fmaf(qbar[8 * d8 + 2 * e + 1], f.y, b);
                }
            }
            l[i] = a * inv_sqrt_d;
            kq[i] = b;
            mx = fmaxf(mx, l[i]);
        }
    }
    mx = warp_max(mx);
    float den = 0.f, num = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float e = lane + 32 * i < n_vis ? expf(l[i] - mx) : 0.f;
        den += e;
        num = fmaf(e, kq[i], num);
    }
    return warp_sum(num) / warp_sum(den);
}

// Order-preserving map of fp32 to uint32: a > b as floats iff key(a) > key(b) (no NaN).
__device__ __forceinline__ uint32_t f32_key(float x) {
    const uint32_t u = __float_as_uint(x);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_f32(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Top-k threshold of one row xs[0..n) (all 32 lanes of a warp, 1 <= k < n): the key of the
// k-th largest score, built bit by bit from the most significant one, and in `need` how many
// scores equal to it are selected (the lowest indices first: the row's selection is every
// score above the threshold plus the first `need` equal to it).
__device__ __forceinline__ uint32_t warp_topk_key(const float *xs, int n, int k, int &need) {
    const int lane = threadIdx.x & 31;
    uint32_t ans = 0;
    for (int b = 31; b >= 0; --b) {
        const uint32_t t = ans | (1u << b);
        int cnt = 0;
        for (int c = lane; c < n; c += 32) cnt += f32_key(xs[c]) >= t ? 1 : 0;
        if (warp_sum_i(cnt) >= k) ans = t;
    }
    int gt = 0;
    for (int c = lane; c < n; c += 32) gt += f32_key(xs[c]) > ans ? 1 : 0;
    need = k - warp_sum_i(gt);
    return ans;
}

// Walks a top-k selection in index order, 32 entries per call and warp: entry c (= 32 i + lane
// of the i-th call) is selected if it is one of the n scores and either all of them are
// selected (sel_all), or its key is above `key`, or it equals `key` and fewer than `need`
// equal keys came before it (`run` counts those, and is updated).
__device__ __forceinline__ bool topk_selected(const float *xs, int c, int n, bool sel_all,
                                              uint32_t key, int need, int &run) {
    const int lane = threadIdx.x & 31;
    const bool in = c < n;
    const uint32_t kc = in ? f32_key(xs[c]) : 0u;
    const bool eq = in && !sel_all && kc == key;
    const unsigned bal = __ballot_sync(kFull, eq);
    const bool sel = in && (sel_all || kc > key || (eq && run + __popc(bal & ((1u << lane) - 1u)) < need));
    run += __popc(bal);
    return sel;
}

// m^beta for the entmax probability of margin m > 0.
__device__ __forceinline__ float pow_beta(float m, const RouteConsts &rc) {
    if (rc.kind == 1) return m * m;
    if (rc.kind == 2) return m;
    return rc.beta_int ? ipow(m, rc.beta_int) : powf(m, rc.beta);
}
// m^(beta-1), the derivative's power.
__device__ __forceinline__ float pow_beta_m1(float m, const RouteConsts &rc) {
    if (rc.kind == 1) return m;
    if (rc.kind == 2) return 1.f;
    return rc.beta_int ? ipow(m, rc.beta_int - 1) : powf(m, rc.beta - 1.f);
}

// One lane-strided pass over xs[0..n): lane l visits l, l+32, l+64, l+96, l+128, ..., with
// four independent accumulators (one per offset mod 128, for instruction-level parallelism)
// combined as (a0 + a1) + (a2 + a3): a fixed summation order.  The adds are explicit (never
// contracted into a product of the term), so every source of the row gives the same bits.
template <typename Term>
__device__ __forceinline__ float lane_pass(const float *xs, int n, int lane, Term term) {
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
    int c = lane;
    for (; c + 96 < n; c += 128) {
        a0 = __fadd_rn(a0, term(xs[c]));
        a1 = __fadd_rn(a1, term(xs[c + 32]));
        a2 = __fadd_rn(a2, term(xs[c + 64]));
        a3 = __fadd_rn(a3, term(xs[c + 96]));
    }
    if (c < n) a0 = __fadd_rn(a0, term(xs[c]));
    if (c + 32 < n) a1 = __fadd_rn(a1, term(xs[c + 32]));
    if (c + 64 < n) a2 = __fadd_rn(a2, term(xs[c + 64]));
    return (a0 + a1) + (a2 + a3);
}

// Two sums in one lane-strided pass: each with lane_pass's order, so each has lane_pass's
// bits; xs is read once for both.
template <typename Term1, typename Term2>
__device__ __forceinline__ void lane_pass2(const float *xs, int n, int lane, Term1 t1, Term2 t2,
                                           float &s1, float &s2) {
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f, b0 = 0.f, b1 = 0.f, b2 = 0.f, b3 = 0.f;
    int c = lane;
    for (; c + 96 < n; c += 128) {
        const float x0 = xs[c], x1 = xs[c + 32], x2 = xs[c + 64], x3 = xs[c + 96];
        a0 = __fadd_rn(a0, t1(x0));
        b0 = __fadd_rn(b0, t2(x0));
        a1 = __fadd_rn(a1, t1(x1));
        b1 = __fadd_rn(b1, t2(x1));
        a2 = __fadd_rn(a2, t1(x2));
        b2 = __fadd_rn(b2, t2(x2));
        a3 = __fadd_rn(a3, t1(x3));
        b3 = __fadd_rn(b3, t2(x3));
    }
    if (c < n) { const float x = xs[c]; a0 = __fadd_rn(a0, t1(x)); b0 = __fadd_rn(b0, t2(x)); }
    if (c + 32 < n) { const float x = xs[c + 32]; a1 = __fadd_rn(a1, t1(x)); b1 = __fadd_rn(b1, t2(x)); }
    if (c + 64 < n) { const float x = xs[c + 64]; a2 = __fadd_rn(a2, t1(x)); b2 = __fadd_rn(b2, t2(x)); }
    s1 = (a0 + a1) + (a2 + a3);
    s2 = (b0 + b1) + (b2 + b3);
}

// A row of n scores as seen by one warp: lane l owns the values c = l + 32 k, k = 0, 1, ...
// Two sources with the same summation order, so the same bits: the row in (shared) memory,
// or the lane's values in registers (n <= 32 NV).
struct RowInMemory {
    const float *xs;
    int n, lane;
    __device__ float max() const {
        float mx = -INFINITY;
        for (int c = lane; c < n; c += 32) mx = fmaxf(mx, xs[c]);
        return mx;
    }
    template <typename T>
    __device__ float pass(T term) const { return lane_pass(xs, n, lane, term); }
    template <typename T1, typename T2>
    __device__ void pass2(T1 t1, T2 t2, float &s1, float &s2) const { lane_pass2(xs, n, lane, t1, t2, s1, s2); }
    // Does any value lie on different sides of t and nt?
    __device__ int moved(float t, float nt) const {
        int m = 0;
        for (int c = lane; c < n; c += 32) m |= ((xs[c] > t) != (xs[c] > nt));
        return m;
    }
};
template <int NV>
struct RowInRegisters {
    const float (&v)[NV];                // v[k] = score l + 32 k of lane l (valid for k < nk)
    int nk;
    __device__ float max() const {
        float mx = -INFINITY;
#pragma unroll
        for (int k = 0; k < NV; ++k)
            if (k < nk) mx = fmaxf(mx, v[k]);
        return mx;
    }
    // lane_pass's order: accumulator k % 4 takes the values k, k + 4, ... in turn.
    template <typename T>
    __device__ float pass(T term) const {
        float a[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int k = 0; k < NV; ++k)
            if (k < nk) a[k & 3] = __fadd_rn(a[k & 3], term(v[k]));
        return (a[0] + a[1]) + (a[2] + a[3]);
    }
    template <typename T1, typename T2>
    __device__ void pass2(T1 t1, T2 t2, float &s1, float &s2) const {
        float a[4] = {0.f, 0.f, 0.f, 0.f}, b[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int k = 0; k < NV; ++k)
            if (k < nk) {
                a[k & 3] = __fadd_rn(a[k & 3], t1(v[k]));
                b[k & 3] = __fadd_rn(b[k & 3], t2(v[k]));
            }
        s1 = (a[0] + a[1]) + (a[2] + a[3]);
        s2 = (b[0] + b[1]) + (b[2] + b[3]);
    }
    __device__ int moved(float t, float nt) const {
        int m = 0;
#pragma unroll
        for (int k = 0; k < NV; ++k)
            if (k < nk) m |= ((v[k] > t) != (v[k] > nt));
        return m;
    }
};

// Newton's method on f^(1/beta) = 1, f(tau) = sum_c [x_c - tau]_+^beta, from tau0 = max x - 1
// (beta >= 1).  f^(1/beta) is a beta-norm of the margins, nearly linear in tau, so it takes
// far fewer steps than Newton on f = 1 when the support is large; it is convex and decreasing
// too, so the steps rise monotonically to the root.  Step = (f - f^(1 - 1/beta)) / sum m^(beta-1).
// BI > 0: beta = BI, the powers as ipow's product chain unrolled (m^BI = m^(BI-1) * m, the
// same bits as ipow(m, BI)); BI = 0 with KIND 3: powf.
template <int KIND, int BI, typename Row>
__device__ __forceinline__ float newton_tau(const Row &row, float mx, const RouteConsts &rc,
                                            uint32_t *status) {
    const float beta = rc.beta;
    float tau = mx - 1.f;
    int it = 0;
    for (; it < rc.newton_cap; ++it) {
        const float t = tau;
        float f, df;
        row.pass2(
            [t, beta](float x) {
                const float m = x - t;
                if (!(m > 0.f)) return 0.f;
                if constexpr (KIND == 1) return __fmul_rn(m, m);
                else if constexpr (KIND == 2) return m;
                else if constexpr (BI > 0) return __fmul_rn(ipow_c<BI - 1>(m), m);
                else return powf(m, beta);
            },
            [t, beta](float x) {
                const float m = x - t;
                if (!(m > 0.f)) return 0.f;
                if constexpr (KIND == 1) return m;
                else if constexpr (KIND == 2) return 1.f;
                else if constexpr (BI > 0) return ipow_c<BI - 1>(m);
                else return powf(m, beta - 1.f);
            },
            f, df);
        f = warp_sum(f);
        df = warp_sum(df);
        const float step = KIND == 2 ? (f - 1.f) / df
                         : KIND == 1 ? (f - sqrtf(f)) / df
                                     : (f - powf(f, 1.f - 1.f / beta)) / df;
        if (!(step > 0.f)) break;                 // at (or rounded past) the root
        const float nt = tau + step;
        if (nt == tau) break;
        tau = nt;
        if (step <= 1e-7f * fmaxf(1.f, fabsf(tau))) break;
    }
    if (it == rc.newton_cap) report(status, DASH_ERR_DEVICE_TIMEOUT);
    return tau;
}

// Entmax threshold of one row (n >= 1 scores, all 32 lanes of the warp calling), specialised
// on the kind of alpha (0 softmax, 1 alpha = 1.5, 2 alpha = 2, 3 any other alpha).  For
// alpha = 1 returns the log-sum-exp of the scores.  Otherwise x are the scaled scores
// (alpha-1) s and the return value is tau with sum_c [x_c - tau]_+^beta = 1.  For beta >= 1
// (alpha <= 2) Newton's method on f^(1/beta) = 1 from tau0 = max x - 1 increases
// monotonically to the root (the function is convex and decreasing); the support it settles
// on is then fed to the exact closed form for alpha = 1.5 and 2.  For alpha > 2, bisection on [max - 1, max - n^(1-alpha)].  The
// fixed lane-strided sums and butterfly reductions give every caller the same bits.
template <int KIND, typename Row>
__device__ __forceinline__ float entmax_tau_row(const Row &row, int n, const RouteConsts &rc,
                                                uint32_t *status) {
    const float mx = warp_max(row.max());
    if (KIND == 0) {
        const float s = warp_sum(row.pass([mx](float x) { return expf(x - mx); }));
        return mx + logf(s);
    }
    float tau;
    if (KIND != 3 || rc.beta >= 1.f) {
        if (KIND != 3) {
            tau = newton_tau<KIND, 0>(row, mx, rc, status);
        } else {
            switch (rc.beta_int) {              // integer beta: the power chain unrolled
                case 3: tau = newton_tau<3, 3>(row, mx, rc, status); break;
                case 4: tau = newton_tau<3, 4>(row, mx, rc, status); break;
                case 5: tau = newton_tau<3, 5>(row, mx, rc, status); break;
                case 6: tau = newton_tau<3, 6>(row, mx, rc, status); break;
                case 7: tau = newton_tau<3, 7>(row, mx, rc, status); break;
                case 8: tau = newton_tau<3, 8>(row, mx, rc, status); break;
                default: tau = newton_tau<3, 0>(row, mx, rc, status); break;
            }
        }
    } else {
        const float beta = rc.beta;
        float lo = mx - 1.f, hi = mx - powf((float)n, 1.f - rc.alpha);
        for (int it = 0; it < 40; ++it) {
            const float mid = 0.5f * (lo + hi);
            const float f = warp_sum(row.pass([mid, beta](float x) {
                const float m = x - mid;
                return m > 0.f ? powf(m, beta) : 0.f;
            }));
            if (f >= 1.f) lo = mid; else hi = mid;
        }
        tau = 0.5f * (lo + hi);
    }
    if (KIND == 1 || KIND == 2) {
        // Exact closed form on the support {x > tau}; repeat while the support moves.
        for (int rep = 0; rep < 4; ++rep) {
            const float t = tau;
            float sx, kf;
            row.pass2([t](float x) { return x > t ? x : 0.f; }, [t](float x) { return x > t ? 1.f : 0.f; },
                      sx, kf);
            sx = warp_sum(sx);
            const int k = (int)warp_sum(kf);
            if (k == 0) break;
            float nt;
            if (KIND == 2) {
                nt = (sx - 1.f) / (float)k;
            } else {
                const float mean = sx / (float)k;
                const float m2 = warp_sum(row.pass([t, mean](float x) {
                    const float d = x - mean;
                    return x > t ? __fmul_rn(d, d) : 0.f;
                }));
                nt = mean - sqrtf(fmaxf(1.f - m2, 0.f) / (float)k);
            }
            // Same support under the new threshold?  Then it is the fixed point.
            const int moved = __any_sync(kFull, row.moved(tau, nt));
            tau = nt;
            if (!moved) break;
        }
    }
    return tau;
}

// The row in (shared) memory xs[0..n); kept out of line (its callers' register budgets).
template <int KIND>
static __device__ __noinline__ float entmax_tau_k(const float *xs, int n, const RouteConsts rc,
                                                  uint32_t *status) {
    const RowInMemory row{xs, n, (int)(threadIdx.x & 31)};
    return entmax_tau_row<KIND>(row, n, rc, status);
}

__device__ __forceinline__ float warp_entmax_tau(const float *xs, int n, const RouteConsts &rc,
                                                 uint32_t *status) {
    switch (rc.kind) {
        case 0: return entmax_tau_k<0>(xs, n, rc, status);
        case 1: return entmax_tau_k<1>(xs, n, rc, status);
        case 2: return entmax_tau_k<2>(xs, n, rc, status);
        default: return entmax_tau_k<3>(xs, n, rc, status);
    }
}

// The same threshold from the lane's values in registers: v[k] = xs[lane + 32 k], k < NV,
// n <= 32 NV.  Same bits as warp_entmax_tau on the row in memory.
template <int NV>
__device__ __forceinline__ float warp_entmax_tau_regs(const float (&v)[NV], int n,
                                                      const RouteConsts &rc, uint32_t *status) {
    const int lane = threadIdx.x & 31;
    const RowInRegisters<NV> row{v, n > lane ? (n - lane + 31) / 32 : 0};
    switch (rc.kind) {
        case 0: return entmax_tau_row<0>(row, n, rc, status);
        case 1: return entmax_tau_row<1>(row, n, rc, status);
        case 2: return entmax_tau_row<2>(row, n, rc, status);
        default: return entmax_tau_row<3>(row, n, rc, status);
    }
}

}  // namespace dash
