// attend_fa.cu -- Stage 2 on the 5th-generation tensor cores with 128-key blocks, D = 128.
//
// gist.science "DashAttention: Differentiable and Adaptive Sparse Hierarchical Attention",
// Technische Zusammenfassung, "Stufe 2: Prior-induzierte spaerliche Softmax": a
// FlashAttention-style kernel iterates the active chunks given by the bit-packed mask and
// adds the routing bias (log of the prior) to the logits before the softmax; chunks with
// zero probability are masked; the diagonal chunk keeps its own branch.
//
// One CTA per SM, one tile of 128 query rows of one (b, g): 128/G consecutive tokens x G
// heads (G >= 8), which share one diagonal chunk.  The tile walks the union of its tokens'
// active chunks (the OR of their mask words, which carry each token's diagonal bit): the
// diagonal chunk first, then the others in ascending order, two 64-key chunks (or one
// 128-key chunk) per 128-key block.  A row whose token did not route to a chunk gets bias
// -inf there; keys above the row's position are masked.  Per block j:
//   S_j[128 x 128] = Q K^T     tcgen05.mma, A = Q (TMEM), B = K (smem, TMA), N = 128
//   softmax        four threads per row (16 warps, 32 keys each), fp32; each thread writes
//                  its bf16 P over its own S columns
//   O[128 x 128]  += P V       tcgen05.mma, A = P (TMEM), B = V^T (smem, TMA; K-major: keys
//                              contiguous per head dim), K = 128 keys
// S is double-buffered, so Q K^T of block j+1 runs while the softmax works on block j; the
// Q K^T and P V instructions come from two issuer warps.  Measured on B200: an N = 128
// tcgen05.mma with a K-major B and a precomputed descriptor issues in ~66 cycles (its tensor
// time), with an MN-major B (V as stored) in ~108, hence V^T (one transpose pass per call,
// vtranspose.cu) and descriptors built once per ring stage.
// Softmax reference: the first block holds the diagonal chunk, whose causally visible keys
// (at least one per row) give each row its exact maximum m; every probability is 2^(s - m)
// against that fixed reference, so O is never rescaled.  A logit so far above the reference
// that the row's fp32 sum overflows (beyond about 2^110 with 2^17 keys) leaves a non-finite
// row sum; such rows are reported as DASH_ERR_RANGE_CLAMPED.  Row sums add the bf16 weights
// the MMA multiplies, computed by the tensor core: V^T carries 16 extra rows of ones, so
// P V (N = 144) leaves sum_k P[r, k] in O column 128.  Off the diagonal the exponent
// arguments run on packed fp32 pairs (fma.rn.f32x2): about 2.5 instructions per score.
// Warp roles: 0 K producer (3-stage ring, 128B-swizzled), 1 Q K^T issuer
// and TMEM owner, 2 and 21 routing-bias producers (recompute qbar.summary with Stage 1's exact
// arithmetic for the active (token, chunk) pairs, 32 chunks per batch, half a batch each,
// double-buffered; at G <= 4 the batch's summary rows are staged in shared memory), 3 P V
// issuer, 4-19 softmax + epilogue, 20 V^T producer (warp 0 then streams K only).
// TMEM: Q 64 columns | S0 128 | S1 128 | O 144 (128 dims + row sums).  Every wait is bounded; on timeout the CTA
// records DASH_ERR_DEVICE_TIMEOUT and drains.
#include "kernels.cuh"
#include "tc_common.cuh"

namespace dash {
using namespace tcx;
namespace {

constexpr int kSmWarps = 16;
constexpr int kSmThreads = kSmWarps * 32;
constexpr int kFaThreads = 4 * 32 + kSmThreads + 64;
constexpr int kStages = 3;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColQ = 0, kColS = 64, kColO = 320;     // S buffer b at kColS + 128 b
constexpr int kBiasBatch = 32;
// Row stride (floats) of the tile's group-mean queries in shared memory: 4 floats of padding
// put consecutive rows 4 banks apart, so the routing-bias warp, whose lanes read different
// rows at the same column, loads them without bank conflicts (a stride of 128 floats made
// every 16-byte load a 32-way conflict with 32 tokens per tile).
constexpr int kQs = 128 + 4;
constexpr int kWarpTma = 0, kWarpQk = 1, kWarpBias = 2, kWarpPv = 3, kWarpSm0 = 4,
              kWarpTmaV = kWarpSm0 + kSmWarps, kWarpBias2 = kWarpTmaV + 1;
constexpr int kBiasThreads = 64;           // the two routing-bias warps
constexpr uint32_t kBlkBytes = 32768;      // K stage: 2 d-panels x [128 keys][128 B]
constexpr int kNv = 144;                   // P V columns: 128 dims of V, then 16 columns of ones
constexpr uint32_t kVHalf = kNv * 128;     // V^T key-half: [144 rows][64 keys x 2 B] (rows >= 128: ones)
constexpr uint32_t kVStage = 2 * kVHalf;
// K/V ring of NST stages (3, or 2 where larger tiles of tokens need the shared memory).
constexpr uint32_t ring_offv(int nst) { return (uint32_t)nst * kBlkBytes; }
constexpr uint32_t ring_bytes(int nst) { return ring_offv(nst) + (uint32_t)nst * kVStage; }

struct FaShared {
    uint64_t k_full[kStages], k_empty[kStages], v_full[kStages], v_empty[kStages];
    uint64_t s_full[2], p_full[2], pv_done[2];  // per S buffer: never more than one phase ahead
    uint64_t o_full, qk_done;
    uint64_t sum_full[2];                  // a routing-bias batch's summary rows have landed
    float mpart[4][128];                   // partial row maxima of the first block
    float tau[64];                         // fused routing: tau of the tile's tokens
    uint32_t tmem_base;
    int n_chunks;
    int failed;
};

// Packed fp32 pairs (sm_100): {lo, hi} in one 64-bit register.
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float &lo, float &hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

}  // namespace

// Fused routing of one tile (see the kernel): scores of the RT tokens over chunks [0, n) into
// xs (stride roundup(C, 4)), then per token tau, the mask words (maskw [RT][W], and mem_mask /
// mem_tau / mem_p in memory when given).  Every thread of the CTA calls it.
template <int D>
__device__ __noinline__ void fa_route_tile(const float *sumg, int C, int W, float *mem_tau,
                                           uint64_t *mem_mask, float *mem_p, const RouteConsts rc,
                                           uint32_t *status, long long row0, int t0, int t_end,
                                           int RT, int n, float *xs, const float *qbar,
                                           uint64_t *maskw, float *tau_s, int warp, int lane) {
    const int xstride = (C + 3) & ~3;
    const float scale = rc.kind == 0 ? rc.sscale : rc.xscale;
    if (warp >= kWarpSm0 && warp < kWarpTmaV) {
        const int wi = warp - kWarpSm0;
        if (RT >= 16) {
            // Rows in groups of 16 (register budget); each row's arithmetic is unchanged.
            for (int r0 = 0; r0 < RT; r0 += 16)
                route_scores_lean<D, 16>(xs + r0 * xstride, xstride, qbar + r0 * kQs, kQs, sumg, n, wi, kSmWarps, scale);
        } else if (RT == 8) {
            route_scores_lean<D, 8>(xs, xstride, qbar, kQs, sumg, n, wi, kSmWarps, scale);
        } else if (RT == 4) {
            route_scores_lean<D, 4>(xs, xstride, qbar, kQs, sumg, n, wi, kSmWarps, scale);
        } else if (RT == 2) {
            route_scores_lean<D, 2>(xs, xstride, qbar, kQs, sumg, n, wi, kSmWarps, scale);
        } else {
            route_scores_lean<D, 1>(xs, xstride, qbar, kQs, sumg, n, wi, kSmWarps, scale);
        }
    }
    __syncthreads();
    for (int u = warp - kWarpSm0; u >= 0 && u < RT && warp < kWarpTmaV; u += kSmWarps) {
        const int t = t0 + u;
        const bool live = t < t_end;
        const float *x = xs + u * xstride;
        const float tau = live && n > 0 ? warp_entmax_tau(x, n, rc, status) : __int_as_float(0x7fc00000);
        const long long rowi = row0 + t;
        if (lane == 0) {
            tau_s[u] = tau;
            if (live && mem_tau) mem_tau[rowi] = tau;
        }
        for (int w = 0; w < W; ++w) {
            const int c0 = w * 64 + lane, c1 = c0 + 32;
            const bool p0 = c0 == n || (c0 < n && (rc.kind == 0 || __fsub_rn(x[c0], tau) > 0.f));
            const bool p1 = c1 == n || (c1 < n && (rc.kind == 0 || __fsub_rn(x[c1], tau) > 0.f));
            const unsigned lo = __ballot_sync(kFull, p0), hi = __ballot_sync(kFull, p1);
            const uint64_t word = live ? ((uint64_t)hi << 32) | lo : 0ull;
            if (lane == (w & 31)) {
                maskw[u * W + w] = word;
                if (live && mem_mask) mem_mask[rowi * W + w] = word;
            }
        }
        if (live && mem_p) {
            float *prow = mem_p + rowi * C;
            for (int c = lane; c < C; c += 32) {
                float val = 0.f;
                if (c < n) {
                    if (rc.kind == 0) {
                        val = expf(x[c] - tau);
                    } else {
                        const float m = __fsub_rn(x[c], tau);
                        val = m > 0.f ? pow_beta(m, rc) : 0.f;
                    }
                }
                prow[c] = val;
            }
        }
    }
}

// Two dot products qa . sa and qb . sb, each with route_dot's slices and order (the same
// bits), their loads and multiply-adds interleaved.  kLdg: sa, sb in global memory (read-only
// path); otherwise in shared memory.
template <int D, bool kLdg>
__device__ __forceinline__ void route_dot2(const float *qa, const float *sa, const float *qb,
                                           const float *sb, float &da, float &db) {
    const float4 *qa4 = reinterpret_cast<const float4 *>(qa), *sa4 = reinterpret_cast<const float4 *>(sa);
    const float4 *qb4 = reinterpret_cast<const float4 *>(qb), *sb4 = reinterpret_cast<const float4 *>(sb);
    float pa[4], pb[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        float x = 0.f, y = 0.f;
#pragma unroll
        for (int i = 0; i < D / 16; ++i) {
            const float4 s1 = kLdg ? __ldg(sa4 + 4 * i + k) : sa4[4 * i + k];
            const float4 s2 = kLdg ? __ldg(sb4 + 4 * i + k) : sb4[4 * i + k];
            const float4 q1 = qa4[4 * i + k], q2 = qb4[4 * i + k];
            x = fmaf(q1.x, s1.x, x);
            y = fmaf(q2.x, s2.x, y);
            x = fmaf(q1.y, s1.y, x);
            y = fmaf(q2.y, s2.y, y);
            x = fmaf(q1.z, s1.z, x);
            y = fmaf(q2.z, s2.z, y);
            x = fmaf(q1.w, s1.w, x);
            y = fmaf(q2.w, s2.w, y);
        }
        pa[k] = x;
        pb[k] = y;
    }
    da = (pa[0] + pa[1]) + (pa[2] + pa[3]);
    db = (pb[0] + pb[1]) + (pb[2] + pb[3]);
}

struct FaArgs {
    StageArgs s;
    int RT;              // tokens per tile (128 / G)
    int tile0, n_tiles_bg;  // first token tile and token tiles per (b, g) of the row range
    size_t off_bias, off_qbar, off_list, off_mask, off_blist, off_sum;  // dynamic smem offsets (aligned base)
    int mask_smem;       // the tile's mask words are copied to shared memory (always when fused)
    int sum_smem;        // the bias batches' summary rows are staged in shared memory
};

template <int BC, int NST>
__global__ void __launch_bounds__(kFaThreads, 1)
k_attend_fa(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmK128,
            const __grid_constant__ CUtensorMap tmVt, const FaArgs ta) {
    extern __shared__ unsigned char smem_dyn[];
    __shared__ FaShared sh;
    constexpr uint32_t kOffVn = ring_offv(NST);
    const StageArgs &a = ta.s;
    constexpr int D = 128;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    unsigned char *base = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~(uintptr_t)1023);
    float *bias_s = reinterpret_cast<float *>(base + ta.off_bias);      // [2][kBiasBatch][RT]
    float *qbar = reinterpret_cast<float *>(base + ta.off_qbar);        // [RT][kQs]
    int16_t *list = reinterpret_cast<int16_t *>(base + ta.off_list);    // [C]

    if (a.cost) {                           // run-time choice against the warp-MMA kernel
        if (!attend_fa_chosen(a)) return;
        attend_record_ran(a, 1);
    }
    const int RT = ta.RT, G = a.G;
    // (b, g)-major, longest tiles first: the CTAs in flight share one (b, g)'s K and V^T in L2
    // (67 MB at T = 128K; both planes at once overflow the 126 MB L2: 3% slower, measured).
    const int tile_rev = blockIdx.x % ta.n_tiles_bg, bgi = blockIdx.x / ta.n_tiles_bg;
    const int tt = ta.tile0 + ta.n_tiles_bg - 1 - tile_rev;
    const int b = bgi / a.Hkv, g = bgi % a.Hkv;
    const long long bg = bgi;
    const int t0 = tt * RT;
    const int t_last = min(t0 + RT, a.t_end) - 1;
    const int ct_max = t_last / BC;                                     // the tile's diagonal chunk

    // ---------------------------------------------------------------- setup
    if (warp == kWarpQk) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&sh.tmem_base)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < NST; ++s) {
            mbar_init(&sh.k_full[s], 1);
            mbar_init(&sh.k_empty[s], 1);
            mbar_init(&sh.v_full[s], 1);
            mbar_init(&sh.v_empty[s], 1);
        }
        for (int bb = 0; bb < 2; ++bb) {
            mbar_init(&sh.s_full[bb], 1);
            mbar_init(&sh.p_full[bb], kSmWarps);
            mbar_init(&sh.pv_done[bb], 1);
        }
        mbar_init(&sh.o_full, 1);
        mbar_init(&sh.qk_done, 1);
        mbar_init(&sh.sum_full[0], 1);
        mbar_init(&sh.sum_full[1], 1);
        sh.failed = 0;
        fence_mbar_init();
    }
    const bool fuse = a.fuse_route != 0;
    uint64_t *maskw = reinterpret_cast<uint64_t *>(base + ta.off_mask);  // [RT][W] (routed)
    int16_t *blist = reinterpret_cast<int16_t *>(base + ta.off_blist);  // [kBiasBatch * RT]
    // Union of the tile's tokens' mask words (each carries its token's diagonal bit): from the
    // routing in memory, or from this kernel's own routing (maskw) when it is fused.
    auto build_list = [&](bool from_smem) {
        const int W = a.W, wlim = ct_max / 64;
        int pos = 0;
        for (int w0 = 0; w0 <= wlim; w0 += 32) {
            const int w = w0 + lane;
            uint64_t word = 0;
            if (w <= wlim) {
                if (a.ignore_routing) {
                    word = ~0ull;
                } else {
                    for (int u = 0; u < RT; ++u) {
                        const int t = t0 + u;
                        if (t < a.t_end) word |= from_smem ? maskw[u * W + w] : a.mask[(bg * a.T + t) * W + w];
                    }
                }
                const int lim = ct_max + 1 - 64 * w;          // bits [0, lim) can be attended
                if (lim < 64) word &= (1ull << lim) - 1ull;
            }
            const int cnt = __popcll(word);
            int incl = cnt;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(kFull, incl, o);
                if (lane >= o) incl += v;
            }
            int p = pos + incl - cnt;
            while (word) {
                const int bit = __ffsll((long long)word) - 1;
                word &= word - 1ull;
                const int cl = w * 64 + bit;
                list[p++] = (int16_t)(dash_check(cl <= ct_max && cl < a.C, a.status) ? cl : ct_max);
            }
            pos += __shfl_sync(kFull, incl, 31);
        }
        if (lane == 0) sh.n_chunks = pos;
    };
    if (warp >= kWarpSm0 && warp < kWarpTmaV) {
        // The tile's setup, spread over the 16 softmax warps (idle until the first block).
        const int st = threadIdx.x - kWarpSm0 * 32;
        if (!fuse && !a.ignore_routing) {
            // tau and, where they fit, the tile's mask words (up to its diagonal chunk) into
            // shared memory, as the fused routing leaves them: the bias loop then reads no
            // memory but the summaries.
            if (ta.mask_smem) {
                const int W = a.W, nw = ct_max / 64 + 1;
                for (int idx = st; idx < RT * nw; idx += kSmThreads) {
                    const int u = idx / nw, w = idx % nw, t = t0 + u;
                    maskw[u * W + w] = t < a.t_end ? a.mask[(bg * a.T + t) * W + w] : 0ull;
                }
            }
            for (int u = st; u < RT; u += kSmThreads) sh.tau[u] = t0 + u < a.t_end ? a.tau[bg * a.T + t0 + u] : 0.f;
        }
        // Group-mean queries of the tile's tokens (Stage 1's exact arithmetic).
        if (!a.ignore_routing) {
            const __nv_bfloat16 *q = reinterpret_cast<const __nv_bfloat16 *>(a.q);
            for (int idx = st; idx < RT * (D / 8); idx += kSmThreads) {
                const int u = idx / (D / 8), d8 = (idx % (D / 8)) * 8, t = t0 + u;
                float m[8];
                if (t < a.t_end) {
                    group_mean8(q + (((long long)b * a.Hq + g * G) * a.T + t) * D + d8,
                                (long long)a.T * D, G, m);
                } else {
#pragma unroll
                    for (int e = 0; e < 8; ++e) m[e] = 0.f;
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) qbar[u * kQs + d8 + e] = m[e];
            }
        }
    }
    // Rows 128-143 of every V^T key-half stage are ones (bf16 1.0 = 0x3f80): P V then also
    // yields the row sums of P in O columns 128-143.  TMA never writes these rows.  (With the
    // routing fused, the ring holds the routing scores first; the ones are written after.)
    auto write_ones = [&]() {
        const uint4 ones = make_uint4(0x3f803f80u, 0x3f803f80u, 0x3f803f80u, 0x3f803f80u);
        for (int i = lane; i < NST * 2 * 16 * 8; i += 32) {
            const int half = i / (16 * 8), r = (i / 8) % 16, c = i % 8;
            *reinterpret_cast<uint4 *>(base + kOffVn + (size_t)half * kVHalf + (128 + r) * 128 + c * 16) = ones;
        }
        fence_proxy_async();
    };
    if (warp == kWarpTma && !fuse) write_ones();
    // Softmax warps: quadrant sp (TMEM lanes 32 sp ..), key quarter kq of every block.
    const int sp = warp & 3;
    const int kq = (warp - kWarpSm0) >> 2;
    const int row = 32 * sp + lane;
    const int u_row = row / G;
    const int t_row = t0 + u_row;
    const int h_row = g * G + row % G;
    const bool row_ok = t_row < a.t_end && dash_check(t_row < a.T && h_row < a.Hq, a.status);
    __syncthreads();
    const uint32_t tb = sh.tmem_base;
    if (warp >= kWarpSm0 && warp < kWarpTmaV) {
        // Q row -> TMEM columns [0, 64): this warp's quarter of the dims (32 dims, 16 columns).
        const __nv_bfloat16 *qr = reinterpret_cast<const __nv_bfloat16 *>(a.q) +
                                  (((long long)b * a.Hq + h_row) * a.T + (row_ok ? t_row : 0)) * D +
                                  32 * kq;
        uint32_t r[16];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint4 v = row_ok ? *reinterpret_cast<const uint4 *>(qr + 8 * j) : make_uint4(0, 0, 0, 0);
            r[4 * j] = v.x;
            r[4 * j + 1] = v.y;
            r[4 * j + 2] = v.z;
            r[4 * j + 3] = v.w;
        }
        tmem_st16(tb + ((uint32_t)(32 * sp) << 16) + kColQ + 16 * kq, r);
        tmem_wait_st();
    }
    // The union list (from the mask words staged above, or from memory), beside the Q stores.
    if (warp == kWarpBias && !fuse) build_list(ta.mask_smem != 0);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    if (fuse) {
        // Stage 1 inside the tile (fused route-and-attend): every token of the tile has its
        // diagonal chunk ct_max, so all route over chunks [0, ct_max).  The 16 softmax warps
        // score them with Stage 1's arithmetic into the K/V ring (free until the copies
        // start), one warp per token solves tau and emits its mask words (to shared memory,
        // and to memory for the caller), then the union list is built as usual.  Kept out of
        // line so that its registers do not press on the attention loop's.
        fa_route_tile<D>(a.summary + bg * a.Cf * D, a.C, a.W, a.tau, a.mask, a.p, a.rc, a.status,
                         bg * a.T, t0, a.t_end, RT, ct_max, reinterpret_cast<float *>(base), qbar,
                         maskw, sh.tau, warp, lane);
        // The scores went through the generic proxy; the copies that reuse the ring next go
        // through the async proxy.
        fence_proxy_async();
        __syncthreads();
        if (warp == kWarpBias) build_list(true);
        if (warp == kWarpTma) write_ones();
        __syncthreads();
    }
    const int n_chunks = sh.n_chunks;
    const int n_blocks = BC == 64 ? (n_chunks + 1) / 2 : n_chunks;
    bool failed = false;
    // Walk order: the diagonal chunk (the largest, last entry of the ascending list) first.
    auto chunk_at = [&](int e) -> int { return (int)list[e == 0 ? n_chunks - 1 : e - 1]; };
    // List entry of half h (keys 64h .. 64h+63) of block j; -1 if that half is empty.
    auto entry_of = [&](int j, int h) -> int {
        if (BC == 64) return 2 * j + h < n_chunks ? 2 * j + h : -1;
        return j;
    };
    auto key0_of = [&](int j, int h) -> int {
        return BC == 64 ? chunk_at(2 * j + h) * 64 : chunk_at(j) * 128 + 64 * h;
    };

    if (warp == kWarpTma || warp == kWarpTmaV) {
        // ------------------------------------------------------------ TMA producer
        // K runs one block ahead of V^T (Q K^T needs it first).  K: a block's two 64-key
        // halves land at rows 0-63 and 64-127 of each 16 KB d-panel, as one 128-key box per
        // panel when the halves are adjacent keys (always for 128-key chunks, mostly in dense
        // unions): TMA throughput per SM grows with the request size (measured on B200: about
        // 35, 44 and 53 bytes per cycle for 8, 16 and 32 KB boxes).  V^T: key-half h is one
        // [128 d][64 keys] box at 16 KB * h.  An empty second half is not loaded (its MMAs are
        // not issued either).
        int k_issued = 0, v_issued = 0;
        auto issue = [&](bool is_v, int j) -> bool {
            const int s = j % NST;
            const uint32_t ph = (uint32_t)(j / NST) & 1u;
            uint64_t *empty = is_v ? &sh.v_empty[s] : &sh.k_empty[s];
            uint64_t *full = is_v ? &sh.v_full[s] : &sh.k_full[s];
            if (!wait_or_fail(empty, ph ^ 1u, a.status, failed)) return false;
            if (lane == 0) {
                unsigned char *st = base + (is_v ? kOffVn + (size_t)s * kVStage : (size_t)s * kBlkBytes);
                const int nh = entry_of(j, 1) >= 0 ? 2 : 1;
                mbar_arrive_expect_tx(full, 16384u * nh);
                for (int h = 0; h < nh; ++h) {
                    const int key0 = key0_of(j, h);
                    if (is_v) {
                        tma_load_3d(st + kVHalf * h, &tmVt, key0, 0, (int)bg, full);
                    } else if (nh == 2 && h == 0 && key0_of(j, 1) == key0 + 64) {
                        tma_load_3d(st, &tmK128, 0, key0, (int)bg, full);
                        tma_load_3d(st + 16384, &tmK128, 64, key0, (int)bg, full);
                        break;
                    } else {
                        tma_load_3d(st + 8192 * h, &tmK, 0, key0, (int)bg, full);
                        tma_load_3d(st + 16384 + 8192 * h, &tmK, 64, key0, (int)bg, full);
                    }
                }
            }
            __syncwarp();
            if (is_v) v_issued = j + 1; else k_issued = j + 1;
            return true;
        };
        // Warp 0 streams K, warp 20 streams V^T: neither ring waits behind the other.
        const bool is_v = warp == kWarpTmaV;
        for (int j = 0; j < n_blocks && !failed; ++j)
            if (!issue(is_v, j)) break;
        if (failed) {
            // Bounded wait for the copies still in flight (the last ones per ring).
            for (int i = max(0, k_issued - NST); i < k_issued; ++i)
                mbar_wait_bounded(&sh.k_full[i % NST], (uint32_t)(i / NST) & 1u);
            for (int i = max(0, v_issued - NST); i < v_issued; ++i)
                mbar_wait_bounded(&sh.v_full[i % NST], (uint32_t)(i / NST) & 1u);
            __syncwarp();
        }
    } else if (warp == kWarpQk) {
        // ------------------------------------------------------------ Q K^T issuer
        // S buffer j & 1 is free once P V of block j-2 (which read P from it) has completed.
        constexpr uint32_t id_qk128 = idesc_bf16(128, 128, 0);
        constexpr uint32_t id_qk64 = idesc_bf16(128, 64, 0);
        uint64_t kdesc[NST];
#pragma unroll
        for (int s = 0; s < NST; ++s) kdesc[s] = smem_desc_sw128(smem_u32(base + (size_t)s * kBlkBytes), 16, 1024);
        for (int j = 0; j < n_blocks; ++j) {
            const int s = j % NST, sb = j & 1;
            if (!wait_or_fail(&sh.k_full[s], (uint32_t)(j / NST) & 1u, a.status, failed)) break;
            if (j >= 2 && !wait_or_fail(&sh.pv_done[sb], (uint32_t)((j - 2) >> 1) & 1u, a.status, failed)) break;
            tc_fence_after();
            if (lane == 0) {
                const uint32_t id = entry_of(j, 1) >= 0 ? id_qk128 : id_qk64;
                uint64_t bd0 = 0;
#pragma unroll
                for (int q = 0; q < NST; ++q) bd0 = q == s ? kdesc[q] : bd0;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    // descriptor start address advances in 16-byte units: d-panel kk/4, 32 B per 16 dims
                    const uint64_t bd = bd0 + (uint64_t)(((kk / 4) * 16384 + (kk % 4) * 32) >> 4);
                    mma_ts(tb + kColS + 128u * sb, tb + kColQ + 8u * kk, bd, id, kk > 0 ? 1u : 0u);
                }
                mma_commit(&sh.s_full[sb]);
                mma_commit(&sh.k_empty[s]);
            }
            __syncwarp();
        }
        if (lane == 0) mma_commit(&sh.qk_done);       // tracks every MMA issued above
        __syncwarp();
    } else if (warp == kWarpPv) {
        // ------------------------------------------------------------ P V issuer
        // P of keys 32q .. 32q+31 sits in the first 16 columns of S quarter q; B = V^T, K-major.
        constexpr uint32_t id_pv = idesc_bf16(128, kNv, 0);
        uint64_t vdesc[NST];
#pragma unroll
        for (int s = 0; s < NST; ++s) vdesc[s] = smem_desc_sw128(smem_u32(base + kOffVn + (size_t)s * kVStage), 16, 1024);
        for (int j = 0; j < n_blocks; ++j) {
            const int s = j % NST, sb = j & 1;
            if (!wait_or_fail(&sh.v_full[s], (uint32_t)(j / NST) & 1u, a.status, failed)) break;
            if (!wait_or_fail(&sh.p_full[sb], (uint32_t)(j >> 1) & 1u, a.status, failed)) break;
            tc_fence_after();
            if (lane == 0) {
                const uint32_t pb = tb + kColS + 128u * sb;
                const bool full_blk = entry_of(j, 1) >= 0;
                uint64_t bd0 = 0;
#pragma unroll
                for (int q = 0; q < NST; ++q) bd0 = q == s ? vdesc[q] : bd0;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    if (kk >= 4 && !full_blk) break;
                    // key-half kk/4 of V^T (144 rows), 32 B per 16 keys
                    const uint64_t bd = bd0 + (uint64_t)(((kk / 4) * kVHalf + (kk % 4) * 32) >> 4);
                    mma_ts(tb + kColO, pb + 32u * (kk / 2) + 8u * (kk % 2), bd, id_pv,
                           (j > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(&sh.pv_done[sb]);
                mma_commit(&sh.v_empty[s]);
            }
            __syncwarp();
        }
        if (lane == 0) mma_commit(&sh.o_full);        // tracks every MMA issued above
        __syncwarp();
    } else if (warp == kWarpBias || warp == kWarpBias2) {
        // ------------------------------------------------------------ routing biases
        // Two warps; each takes half of every batch of kBiasBatch list entries (bw: which
        // half).  Per half: first the entries that need no dot product (invisible or inactive:
        // -inf; the diagonal chunk and top-k: 0) and the list of the others; then those, two
        // per lane and step with their dot products interleaved (each with route_dot's order,
        // so the same bits).
        const int bw = warp == kWarpBias ? 0 : 1;
        const int half_n = kBiasBatch * RT / 2;   // entries per warp and batch (RT even)
        int16_t *my_list = blist + bw * half_n;
        auto bias_of = [&](float dot, float tau) -> float {
            if (a.rc.kind == 0) return a.rc.sigma2 * (__fmul_rn(dot, a.rc.sscale) - tau);
            const float m = __fsub_rn(__fmul_rn(dot, a.rc.xscale), tau);
            return a.rc.bscale2 * log2f(fmaxf(m, 1e-37f));
        };
        const float *sumg = a.summary + bg * a.Cf * D;
        const bool msm = fuse || ta.mask_smem;
        const int n_batches = (n_chunks + kBiasBatch - 1) / kBiasBatch;
        // Staged summaries: the rows of a batch's chunks below the diagonal one (the only ones
        // with a dot product) are copied by the TMA engine into sum_s[bt & 1][k] (rows of kQs
        // floats: lanes reading different rows at the same column hit different banks), two
        // batches in flight, so the dot products read shared memory instead of waiting on L2.
        float *sum_s = reinterpret_cast<float *>(base + ta.off_sum);     // [2][kBiasBatch][kQs]
        const bool stage = ta.sum_smem && !a.ignore_routing;
        int last_issued = -1;
        auto issue_batch = [&](int bt2) {       // the first bias warp issues the copies
            if (bt2 >= n_batches) return;
            last_issued = bt2;
            const int ci = bt2 * kBiasBatch + lane;
            const int c = ci < n_chunks ? chunk_at(ci) : ct_max;
            const bool row = c < ct_max && c < a.Cf;
            const unsigned bal = __ballot_sync(kFull, row);
            if (lane == 0) mbar_arrive_expect_tx(&sh.sum_full[bt2 & 1], (uint32_t)__popc(bal) * D * 4);
            __syncwarp();
            if (row)
                bulk_g2s(sum_s + ((bt2 & 1) * kBiasBatch + lane) * kQs, sumg + (long long)c * D, D * 4,
                         &sh.sum_full[bt2 & 1]);
        };
        if (stage && bw == 0) {
            issue_batch(0);
            issue_batch(1);
        }
        bool sum_failed = false;
        for (int bt = 0; bt < n_batches; ++bt) {
            float *buf = bias_s + (bt & 1) * kBiasBatch * RT;
            // A timed-out copy leaves the biases of this and later batches unset (the status
            // word reports it); the batches' barriers are still passed.
            const bool ready = !stage || wait_or_fail(&sh.sum_full[bt & 1], (uint32_t)(bt >> 1) & 1u, a.status, sum_failed);
            int nact = 0;
            for (int e0 = bw * half_n; e0 < (bw + 1) * half_n && ready; e0 += 32) {
                const int e = e0 + lane;
                const bool mine = e < (bw + 1) * half_n;   // (a half holds 16 entries at RT = 1)
                const int k = e / RT, u = e % RT, ci = bt * kBiasBatch + k;
                float v = 0.f;
                bool need = false;
                if (mine && ci < n_chunks && !a.ignore_routing) {
                    const int c = chunk_at(ci), t = t0 + u;
                    const int ctu = t / BC;
                    if (t >= a.t_end || c > ctu) {
                        v = -INFINITY;
                    } else if (c < ctu) {
                        const uint64_t word = msm ? maskw[u * a.W + (c >> 6)]
                                                  : a.mask[(bg * a.T + t) * a.W + (c >> 6)];
                        const bool act = dash_check(t < a.T && c < a.Cf, a.status) && ((word >> (c & 63)) & 1ull);
                        if (!act) v = -INFINITY;
                        else if (a.rc.kind != kKindTopk) need = true;   // top-k: uniform prior, 0
                    }
                }
                if (mine) buf[e] = v;
                const unsigned bal = __ballot_sync(kFull, need);
                if (need) my_list[nact + __popc(bal & ((1u << lane) - 1u))] = (int16_t)e;
                nact += __popc(bal);
            }
            __syncwarp();
            for (int j = lane; j < nact; j += 64) {
                const bool two = j + 32 < nact;
                const int ea = my_list[j], eb = two ? my_list[j + 32] : ea;
                const int ua = ea % RT, ub = eb % RT;
                const int ca = chunk_at(bt * kBiasBatch + ea / RT), cb = chunk_at(bt * kBiasBatch + eb / RT);
                float da, db;
                if (stage) {
                    const float *sb0 = sum_s + (bt & 1) * kBiasBatch * kQs;
                    route_dot2<D, false>(qbar + ua * kQs, sb0 + (ea / RT) * kQs, qbar + ub * kQs,
                                         sb0 + (eb / RT) * kQs, da, db);
                } else {
                    route_dot2<D, true>(qbar + ua * kQs, sumg + (long long)ca * D, qbar + ub * kQs,
                                        sumg + (long long)cb * D, da, db);
                }
                buf[ea] = bias_of(da, sh.tau[ua]);
                if (two) buf[eb] = bias_of(db, sh.tau[ub]);
            }
            __syncwarp();
            if (stage) {
                // This batch's rows are read by both warps: order those reads before the
                // copies that refill the buffer.
                fence_proxy_async();
                named_sync(3, kBiasThreads);
                if (bw == 0 && !sum_failed) issue_batch(bt + 2);
            }
            named_sync(1, kBiasThreads + kSmThreads);
        }
        if (sum_failed) {
            // Copies issued after the timeout may still be in flight: the issuing warp waits
            // for them (bounded) before the CTA can exit.
            failed = true;
            if (bw == 0)
                for (int bb = max(last_issued - 1, 0); bb <= last_issued; ++bb)
                    mbar_wait_bounded(&sh.sum_full[bb & 1], (uint32_t)(bb >> 1) & 1u);
        }
    } else if (warp >= kWarpSm0 && warp < kWarpTmaV) {
        // ------------------------------------------------------------ softmax
        // Four threads per row: warp (sp, kq) owns keys 32 kq .. 32 kq + 31 of every block for
        // the rows of TMEM quadrant sp.  Every named barrier is passed by all softmax warps,
        // failure or not.
        const uint32_t lane_base = tb + ((uint32_t)(32 * sp) << 16);
        const int half = kq >> 1;
        float m_ref = 0.f;
        const uint64_t scale2 = f2_pack(a.qk_scale2, a.qk_scale2);
        for (int j = 0; j < n_blocks; ++j) {
            const int sb = j & 1;
            const int e0 = BC == 64 ? 2 * j : j;              // first list entry of the block
            if (e0 % kBiasBatch == 0) named_sync(1, kBiasThreads + kSmThreads);
            const bool ok = wait_or_fail(&sh.s_full[sb], (uint32_t)(j >> 1) & 1u, a.status, failed);
            if (ok) tc_fence_after();
            const int e = entry_of(j, half);
            int key0 = 0;
            float bias2 = -INFINITY;
            bool diag = false;
            if (e >= 0 && row_ok) {
                const int c = chunk_at(e);
                key0 = key0_of(j, half) + 32 * (kq & 1);
                if (c == ct_max) {
                    bias2 = 0.f;
                    diag = true;
                } else {
                    bias2 = a.ignore_routing ? 0.f
                                             : bias_s[((e / kBiasBatch) & 1) * kBiasBatch * RT +
                                                      (e % kBiasBatch) * RT + u_row];
                }
            }
            const bool dead = __all_sync(kFull, bias2 == -INFINITY);
            uint32_t sv[32];
            if (ok && (j == 0 || !dead)) {
                tmem_ld32(lane_base + kColS + 128u * sb + 32u * kq, sv);
                tmem_wait_ld();
            }
            if (j == 0) {
                // Exact row maximum over the diagonal chunk's causally visible keys (the first
                // block holds them), shared by the row's four threads: the fixed reference.
                float mx = -INFINITY;
                if (ok && diag) {
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (key0 + i <= t_row) mx = fmaxf(mx, __uint_as_float(sv[i]) * a.qk_scale2);
                }
                sh.mpart[kq][row] = mx;
                named_sync(2, kSmThreads);
                const float m4 = fmaxf(fmaxf(sh.mpart[0][row], sh.mpart[1][row]),
                                       fmaxf(sh.mpart[2][row], sh.mpart[3][row]));
                m_ref = m4 == -INFINITY ? 0.f : m4;
            }
            if (!ok) continue;
            const float c2 = bias2 - m_ref;                  // -inf for rows that do not attend
            uint32_t pw[16];
            if (dead) {
                // None of the warp's 32 rows attends these keys: P = 0, no exponentials.
#pragma unroll
                for (int i = 0; i < 16; ++i) pw[i] = 0u;
            } else if (diag) {
                const int lim = t_row - key0;                // keys i > lim are in the future
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float x0 = 2 * i <= lim ? fmaf(__uint_as_float(sv[2 * i]), a.qk_scale2, c2) : -INFINITY;
                    const float x1 = 2 * i + 1 <= lim ? fmaf(__uint_as_float(sv[2 * i + 1]), a.qk_scale2, c2) : -INFINITY;
                    pw[i] = pack_bf16x2(fast_exp2(x0), fast_exp2(x1));
                }
            } else {
                const uint64_t cc = f2_pack(c2, c2);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    float x0, x1;
                    f2_unpack(f2_fma(f2_pack(__uint_as_float(sv[2 * i]), __uint_as_float(sv[2 * i + 1])), scale2, cc), x0, x1);
                    pw[i] = pack_bf16x2(fast_exp2(x0), fast_exp2(x1));
                }
            }
            // P over this warp's own S columns (the other quarters may still be loading).
            tmem_st16(lane_base + kColS + 128u * sb + 32u * kq, pw);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh.p_full[sb]);
        }
        // Epilogue: l = O column 128 (P times the ones rows of V^T: the sum of the bf16
        // weights the MMA multiplied), O / l -> bf16 (each warp 32 of the dims).
        const bool ok_o = wait_or_fail(&sh.o_full, 0, a.status, failed);
        if (ok_o) {
            tc_fence_after();
            uint32_t lw[1];
            asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];"
                         : "=r"(lw[0]) : "r"(lane_base + kColO + 128u));
            tmem_wait_ld();
            const float l = __uint_as_float(lw[0]);
            if (__any_sync(kFull, row_ok && !isfinite(l)) && lane == 0 && kq == 0) report(a.status, DASH_ERR_RANGE_CLAMPED);
            const float inv = l > 0.f ? 1.f / l : 0.f;
            uint32_t o[32];
            tmem_ld32(lane_base + kColO + 32u * kq, o);
            tmem_wait_ld();
            if (row_ok) {
                __nv_bfloat16 *orow = reinterpret_cast<__nv_bfloat16 *>(a.out) +
                                      (((long long)b * a.Hq + h_row) * a.T + t_row) * D + 32 * kq;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    uint4 v;
                    v.x = pack_bf16x2(__uint_as_float(o[8 * i]) * inv, __uint_as_float(o[8 * i + 1]) * inv);
                    v.y = pack_bf16x2(__uint_as_float(o[8 * i + 2]) * inv, __uint_as_float(o[8 * i + 3]) * inv);
                    v.z = pack_bf16x2(__uint_as_float(o[8 * i + 4]) * inv, __uint_as_float(o[8 * i + 5]) * inv);
                    v.w = pack_bf16x2(__uint_as_float(o[8 * i + 6]) * inv, __uint_as_float(o[8 * i + 7]) * inv);
                    *reinterpret_cast<uint4 *>(orow + 8 * i) = v;
                }
            }
        }
    }

    // ---------------------------------------------------------------- teardown
    if (failed) sh.failed = 1;
    tc_fence_before();
    __syncthreads();
    if (sh.failed && lane == 0) {
        // Each issuer committed after its last MMA, failure or not: wait (bounded) for the
        // MMAs in flight before the tensor memory is released.
        if (warp == kWarpQk) mbar_wait_bounded(&sh.qk_done, 0);
        if (warp == kWarpPv) mbar_wait_bounded(&sh.o_full, 0);
    }
    __syncthreads();
    tc_fence_after();
    if (warp == kWarpQk) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tb), "r"(kTmemCols));
    }
}

// ---------------------------------------------------------------- host side
namespace {

using EncodeFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                              const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                              const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                              CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn fa_encode() {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
        return nullptr;
    return reinterpret_cast<EncodeFn>(fn);
}

// 3-D map over a [B*Hkv][T][128] bf16 plane set: box (64 d, `keys` keys, 1), 128B swizzle,
// zero fill out of bounds (keys >= T of the last chunk).
bool fa_map(EncodeFn enc, CUtensorMap *m, const void *ptr, int T, int BHkv, int keys) {
    cuuint64_t dims[3] = {128, (cuuint64_t)T, (cuuint64_t)BHkv};
    cuuint64_t strides[2] = {128 * 2, (cuuint64_t)T * 128 * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)keys, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t fa_smem_bytes(int RT, int C, bool mask_words, int nst, bool sum_rows) {
    size_t off = ring_bytes(nst);
    off += (size_t)2 * kBiasBatch * RT * 4;      // bias batches
    off += (size_t)RT * kQs * 4;                 // qbar
    off += (size_t)((C + 7) & ~7) * 2;           // chunk list
    off = (off + 7) & ~(size_t)7;
    if (mask_words) off += (size_t)RT * ((C + 63) / 64) * 8;   // the tile's mask words
    off += (size_t)kBiasBatch * RT * 2;          // a batch's entries that need a dot product
    off = (off + 15) & ~(size_t)15;
    if (sum_rows) off += (size_t)2 * kBiasBatch * kQs * 4;     // two batches' summary rows
    return off + 1024;                           // room to align the base to 1024 bytes
}

}  // namespace

size_t attend_fa_vt_bytes(int B, int Hkv, int T, int D) {
    const size_t T8 = (size_t)((T + 7) & ~7);
    return (size_t)B * Hkv * D * T8 * 2;
}

// Ring stages for these arguments (3, or 2 when 3 do not fit; 0: neither fits), whether the
// tile's mask words go to shared memory and whether the bias batches' summary rows are staged
// there: the deepest ring first, with the mask words and then the staged rows where they fit
// beside it (the fused routing needs the mask words there).
struct FaPlan {
    int nst;
    bool mask_smem, sum_smem;
};
static FaPlan fa_plan(const StageArgs &a, bool fuse) {
    if (!(a.D == 128 && a.G >= 2 && a.G <= 128 && 128 % a.G == 0 && (a.Bc == 64 || a.Bc == 128) &&
          128 / a.G <= a.Bc))                  // a tile's tokens share one diagonal chunk
        return {0, false, false};
    const int RT = 128 / a.G;
    for (int nst : {3, 2}) {
        if (fuse && (size_t)RT * ((a.C + 3) & ~3) * 4 > ring_bytes(nst)) continue;   // scores fit the ring
        for (int v = 0; v < 3; ++v) {
            const bool ms = v < 2, ss = v == 0;   // mask and rows, mask only, neither
            if (!ms && fuse) continue;
            // (bulk copies need 16-byte aligned summary rows)
            const bool m = ms && !a.ignore_routing,
                       sr = ss && !a.ignore_routing && (reinterpret_cast<uintptr_t>(a.summary) & 15) == 0;
            if (fa_smem_bytes(RT, a.C, m, nst, sr) + sizeof(FaShared) <= 227 * 1024) return {nst, m, sr};
        }
    }
    return {0, false, false};
}

bool attend_fa_supported(const StageArgs &a) { return fa_plan(a, false).nst != 0; }

bool attend_fa_fuse_supported(const StageArgs &a) {
    if (a.ignore_routing || a.rc.kind > 3 || a.rc.est_diag) return false;
    return fa_plan(a, true).nst != 0;
}

template <int BC, int NST>
static cudaError_t launch_fa_t(const StageArgs &a, bool mask_smem, bool sum_smem, cudaStream_t st) {
    static EncodeFn enc = fa_encode();
    if (!enc || !a.vt) return cudaErrorNotSupported;
    const int BHkv = a.B * a.Hkv;
    cudaError_t e = a.vt_ready ? cudaSuccess
                               : launch_vtranspose(a.v, a.vt, BHkv, a.T, 128, st, a.vt_begin, a.vt_end);
    if (e != cudaSuccess) return e;
    CUtensorMap mk, mk128, mvt;
    if (!fa_map(enc, &mk, a.k, a.T, BHkv, 64) || !fa_map(enc, &mk128, a.k, a.T, BHkv, 128))
        return cudaErrorInvalidValue;
    {
        // V^T [B*Hkv][128][T8]: box (64 keys, 128 dims, 1), 128B swizzle.
        const int T8 = (a.T + 7) & ~7;
        cuuint64_t dims[3] = {(cuuint64_t)T8, 128, (cuuint64_t)BHkv};
        cuuint64_t strides[2] = {(cuuint64_t)T8 * 2, (cuuint64_t)T8 * 2 * 128};
        cuuint32_t box[3] = {64, 128, 1};
        cuuint32_t estr[3] = {1, 1, 1};
        if (enc(&mvt, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, a.vt, dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    FaArgs ta;
    ta.s = a;
    ta.RT = 128 / a.G;
    ta.tile0 = a.t_begin / ta.RT;
    ta.n_tiles_bg = (a.t_end + ta.RT - 1) / ta.RT - ta.tile0;
    size_t off = ring_bytes(NST);
    ta.off_bias = off;
    off += (size_t)2 * kBiasBatch * ta.RT * 4;
    ta.off_qbar = off;
    off += (size_t)ta.RT * kQs * 4;
    ta.off_list = off;
    off += (size_t)((a.C + 7) & ~7) * 2;
    ta.off_mask = (off + 7) & ~(size_t)7;
    ta.mask_smem = mask_smem ? 1 : 0;
    ta.off_blist = ta.off_mask + (mask_smem ? (size_t)ta.RT * ((a.C + 63) / 64) * 8 : 0);
    ta.sum_smem = sum_smem ? 1 : 0;
    ta.off_sum = (ta.off_blist + (size_t)kBiasBatch * ta.RT * 2 + 15) & ~(size_t)15;
    const size_t smem = fa_smem_bytes(ta.RT, a.C, mask_smem, NST, sum_smem);
    auto kern = k_attend_fa<BC, NST>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const long long grid = (long long)ta.n_tiles_bg * BHkv;
    if (grid == 0) return cudaSuccess;
    kern<<<(unsigned)grid, kFaThreads, smem, st>>>(mk, mk128, mvt, ta);
    return cudaGetLastError();
}

cudaError_t launch_attend_fa(const StageArgs &a, cudaStream_t st) {
    const FaPlan pl = fa_plan(a, a.fuse_route != 0);
    if (a.Bc == 64 && pl.nst == 3) return launch_fa_t<64, 3>(a, pl.mask_smem, pl.sum_smem, st);
    if (a.Bc == 64 && pl.nst == 2) return launch_fa_t<64, 2>(a, pl.mask_smem, pl.sum_smem, st);
    if (a.Bc == 128 && pl.nst == 3) return launch_fa_t<128, 3>(a, pl.mask_smem, pl.sum_smem, st);
    if (a.Bc == 128 && pl.nst == 2) return launch_fa_t<128, 2>(a, pl.mask_smem, pl.sum_smem, st);
    return cudaErrorInvalidValue;
}

}  // namespace dash
