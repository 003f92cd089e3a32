// attend_pp.cu -- Stage 2 on the 5th-generation tensor cores with two ping-ponged query tiles
// per CTA, 128-key blocks, D = 128.
//
// gist.science "DashAttention: Differentiable and Adaptive Sparse Hierarchical Attention",
// Technische Zusammenfassung, "Stufe 2: Prior-induzierte spaerliche Softmax": a
// FlashAttention-style kernel walks the active chunks given by the bit-packed mask and adds
// the routing bias (log of the prior) to the logits before the softmax; zero-probability
// chunks are masked; the diagonal chunk keeps its own branch.
//
// Two tiles of 128 query rows of one (b, g) (2 x 128/G consecutive tokens, one diagonal chunk)
// share every K/V block of the union of their tokens' chunks.  Tensor memory holds one S
// buffer and one O accumulator per tile (S_A | S_B | O_A | O_B, 128 columns each); each tile's
// P is written over its own S.  Q_A and Q_B sit in shared memory (Q K^T is an SS MMA).  One
// thread issues, per block i, in this order:
//   Q K^T_A(i)   (after P V_A(i-1), issued just before it: the MMAs of one thread run in issue
//                 order, so S_A is overwritten only after P V_A(i-1) has read P_A)
//   P V_B(i-1)   (needs tile B's softmax of block i-1)
//   Q K^T_B(i)   (after P V_B(i-1))
//   P V_A(i)     (needs tile A's softmax of block i)
// so while tile A's softmax runs, the tensor pipe has tile B's two GEMMs queued, and the
// other way round.  Two softmax groups of 8 warps (one per tile), two threads per row (one
// 64-key half each, so one bias value per thread), row sums of the bf16 weights in the
// softmax threads.  The fixed softmax reference from the diagonal chunk, the biases
// recomputed with Stage 1's arithmetic, the skipped exponentials of warps none of whose rows
// attend a half, and the bounded waits follow the single-tile kernel (attend_fa.cu).
#include "kernels.cuh"
#include "tc_common.cuh"

namespace dash {
using namespace tcx;
namespace {

constexpr int kGrpWarps = 8;                  // softmax warps per tile
constexpr int kSmWarps = 2 * kGrpWarps;
constexpr int kSmThreads = kSmWarps * 32;
constexpr int kPpThreads = 4 * 32 + kSmThreads + 32;   // 21 warps
constexpr int kStagesK = 2, kStagesV = 2;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColO = 256;    // tile t: S at kColS + 128 t, O at kColO + 128 t
constexpr int kBiasBatch = 32;
constexpr int kWarpTma = 0, kWarpMma = 1, kWarpBias = 2, kWarpSm0 = 4,
              kWarpTmaV = kWarpSm0 + kSmWarps;
constexpr uint32_t kQBytes = 32768;           // one Q tile: 2 d-panels x [128 rows][128 B]
constexpr uint32_t kBlkBytes = 32768;         // K stage: 2 d-panels x [128 keys][128 B]
constexpr uint32_t kVHalf = 128 * 128;        // V^T key-half: [128 dims][64 keys x 2 B]
constexpr uint32_t kVStage = 2 * kVHalf;
constexpr uint32_t kOffK = 2 * kQBytes, kOffV = kOffK + kStagesK * kBlkBytes,
                   kRingBytes = kOffV + kStagesV * kVStage;

struct PpShared {
    uint64_t k_full[kStagesK], k_empty[kStagesK], v_full[kStagesV], v_empty[kStagesV];
    uint64_t s_full[2], p_full[2];            // per tile; at most one phase ahead (see issuer)
    uint64_t o_full;
    float mpart[2][2][128];                   // [tile][thread of the row] row maxima, block 0
    float lpart[2][2][128];                   // [tile][thread of the row] row sums
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
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

}  // namespace

struct PpArgs {
    StageArgs s;
    int RT;              // tokens per tile (128 / G)
    int pair0, n_pairs_bg;  // first tile pair and tile pairs per (b, g) of the row range
    size_t off_bias, off_qbar, off_list;
};

template <int BC>
__global__ void __launch_bounds__(kPpThreads, 1)
k_attend_pp(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmK128,
            const __grid_constant__ CUtensorMap tmVt, const PpArgs ta) {
    extern __shared__ unsigned char smem_dyn[];
    __shared__ PpShared sh;
    const StageArgs &a = ta.s;
    constexpr int D = 128;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    unsigned char *base = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~(uintptr_t)1023);
    float *bias_s = reinterpret_cast<float *>(base + ta.off_bias);      // [2][kBiasBatch][2 RT]
    float *qbar = reinterpret_cast<float *>(base + ta.off_qbar);        // [2 RT][D]
    int16_t *list = reinterpret_cast<int16_t *>(base + ta.off_list);    // [C]

    const int RT = ta.RT, RT2 = 2 * ta.RT, G = a.G;
    // (b, g)-major, longest pairs first.
    const int pair_rev = blockIdx.x % ta.n_pairs_bg, bgi = blockIdx.x / ta.n_pairs_bg;
    const int pp = ta.pair0 + ta.n_pairs_bg - 1 - pair_rev;
    const int b = bgi / a.Hkv, g = bgi % a.Hkv;
    const long long bg = bgi;
    const int tp0 = pp * RT2;                                           // the pair's first token
    const int t_last = min(tp0 + RT2, a.t_end) - 1;
    const int ct_max = t_last / BC;                                     // the pair's diagonal chunk

    // ---------------------------------------------------------------- setup
    if (warp == kWarpMma) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&sh.tmem_base)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStagesK; ++s) {
            mbar_init(&sh.k_full[s], 1);
            mbar_init(&sh.k_empty[s], 1);
        }
        for (int s = 0; s < kStagesV; ++s) {
            mbar_init(&sh.v_full[s], 1);
            mbar_init(&sh.v_empty[s], 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(&sh.s_full[t], 1);
            mbar_init(&sh.p_full[t], kGrpWarps);
        }
        mbar_init(&sh.o_full, 1);
        sh.failed = 0;
        fence_mbar_init();
    }
    if (warp == kWarpBias) {
        // Union of the pair's tokens' mask words (each carries its token's diagonal bit).
        const int W = a.W, wlim = ct_max / 64;
        int pos = 0;
        for (int w0 = 0; w0 <= wlim; w0 += 32) {
            const int w = w0 + lane;
            uint64_t word = 0;
            if (w <= wlim) {
                if (a.ignore_routing) {
                    word = ~0ull;
                } else {
                    for (int u = 0; u < RT2; ++u) {
                        const int t = tp0 + u;
                        if (t < a.t_end) word |= a.mask[(bg * a.T + t) * W + w];
                    }
                }
                const int lim = ct_max + 1 - 64 * w;
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
        if (!a.ignore_routing) {
            const __nv_bfloat16 *q = reinterpret_cast<const __nv_bfloat16 *>(a.q);
            for (int idx = lane; idx < RT2 * (D / 8); idx += 32) {
                const int u = idx / (D / 8), d8 = (idx % (D / 8)) * 8, t = tp0 + u;
                float m[8];
                if (t < a.t_end) {
                    group_mean8(q + (((long long)b * a.Hq + g * G) * a.T + t) * D + d8,
                                (long long)a.T * D, G, m);
                } else {
#pragma unroll
                    for (int e = 0; e < 8; ++e) m[e] = 0.f;
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) qbar[u * D + d8 + e] = m[e];
            }
        }
    }
    // Softmax warps: tile grp (warps 4-11: A, 12-19: B), TMEM lane quadrant sp, key half kq.
    const int grp = (warp - kWarpSm0) / kGrpWarps;
    const int sp = warp & 3;
    const int kq = ((warp - kWarpSm0) % kGrpWarps) >> 2;
    const int row = 32 * sp + lane;                                     // row of the tile
    const int u_row = row / G;
    const int t_row = tp0 + grp * RT + u_row;
    const int h_row = g * G + row % G;
    const bool row_ok = t_row < a.t_end && dash_check(t_row < a.T && h_row < a.Hq, a.status);
    const bool is_sm = warp >= kWarpSm0 && warp < kWarpTmaV;
    if (is_sm) {
        // Q row -> shared memory (the A operand of Q K^T): this thread's 64 dims are d-panel
        // kq of the tile, 16-byte chunks 0-7 of the row, 128B-swizzled (chunk XOR row % 8).
        const __nv_bfloat16 *qr = reinterpret_cast<const __nv_bfloat16 *>(a.q) +
                                  (((long long)b * a.Hq + h_row) * a.T + (row_ok ? t_row : 0)) * D +
                                  64 * kq;
        unsigned char *qrow = base + (size_t)grp * kQBytes + (size_t)kq * (kQBytes / 2) +
                              (row >> 3) * 1024 + (row & 7) * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const uint4 v = row_ok ? *reinterpret_cast<const uint4 *>(qr + 8 * c) : make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4 *>(qrow + ((c ^ (row & 7)) << 4)) = v;
        }
        fence_proxy_async();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tb = sh.tmem_base;

    const int n_chunks = sh.n_chunks;
    const int n_blocks = BC == 64 ? (n_chunks + 1) / 2 : n_chunks;
    bool failed = false;
    auto chunk_at = [&](int e) -> int { return (int)list[e == 0 ? n_chunks - 1 : e - 1]; };
    auto entry_of = [&](int j, int h) -> int {
        if (BC == 64) return 2 * j + h < n_chunks ? 2 * j + h : -1;
        return j;
    };
    auto key0_of = [&](int j, int h) -> int {
        return BC == 64 ? chunk_at(2 * j + h) * 64 : chunk_at(j) * 128 + 64 * h;
    };

    if (warp == kWarpTma || warp == kWarpTmaV) {
        // ------------------------------------------------------------ TMA producers
        // Warp 0: K (2 stages; one 128-key box per d-panel when the block's halves are adjacent
        // keys, else 64-key boxes); warp 20: V^T (2 stages, one [128 d][64 keys] box per half).
        const bool is_v = warp == kWarpTmaV;
        const int ns = is_v ? kStagesV : kStagesK;
        int issued = 0;
        for (int j = 0; j < n_blocks && !failed; ++j) {
            const int s = j % ns;
            const uint32_t ph = (uint32_t)(j / ns) & 1u;
            uint64_t *empty = is_v ? &sh.v_empty[s] : &sh.k_empty[s];
            uint64_t *full = is_v ? &sh.v_full[s] : &sh.k_full[s];
            if (!wait_or_fail(empty, ph ^ 1u, a.status, failed)) break;
            if (lane == 0) {
                unsigned char *st = base + (is_v ? kOffV + (size_t)s * kVStage : kOffK + (size_t)s * kBlkBytes);
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
            issued = j + 1;
        }
        if (failed) {
            for (int i = max(0, issued - ns); i < issued; ++i)
                mbar_wait_bounded(is_v ? &sh.v_full[i % ns] : &sh.k_full[i % ns], (uint32_t)(i / ns) & 1u);
            __syncwarp();
        }
    } else if (warp == kWarpMma) {
        // ------------------------------------------------------------ MMA issuer
        // Per block i: Q K^T_A(i), P V_B(i-1), Q K^T_B(i), P V_A(i).  MMAs from this thread run
        // in issue order, so Q K^T_t(i) follows the P V_t(i-1) that read P_t out of S_t.
        constexpr uint32_t id_qk128 = idesc_bf16(128, 128, 0), id_qk64 = idesc_bf16(128, 64, 0);
        constexpr uint32_t id_pv = idesc_bf16(128, 128, 0);
        uint64_t kdesc[kStagesK], vdesc[kStagesV];
#pragma unroll
        for (int s = 0; s < kStagesK; ++s) kdesc[s] = smem_desc_sw128(smem_u32(base + kOffK + (size_t)s * kBlkBytes), 16, 1024);
#pragma unroll
        for (int s = 0; s < kStagesV; ++s) vdesc[s] = smem_desc_sw128(smem_u32(base + kOffV + (size_t)s * kVStage), 16, 1024);
        const uint64_t qdesc[2] = {smem_desc_sw128(smem_u32(base), 16, 1024),
                                   smem_desc_sw128(smem_u32(base + kQBytes), 16, 1024)};
        auto qk = [&](int t, int j) {                     // lane 0 only
            const int s = j % kStagesK;
            const uint32_t id = entry_of(j, 1) >= 0 ? id_qk128 : id_qk64;
            uint64_t bd0 = 0;
#pragma unroll
            for (int q = 0; q < kStagesK; ++q) bd0 = q == s ? kdesc[q] : bd0;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint64_t off = (uint64_t)(((kk / 4) * 16384 + (kk % 4) * 32) >> 4);
                mma_ss(tb + kColS + 128u * t, qdesc[t] + off, bd0 + off, id, kk > 0 ? 1u : 0u);
            }
            mma_commit(&sh.s_full[t]);
        };
        auto pv = [&](int t, int j) {                     // lane 0 only
            const int s = j % kStagesV;
            const bool full_blk = entry_of(j, 1) >= 0;
            uint64_t bd0 = 0;
#pragma unroll
            for (int q = 0; q < kStagesV; ++q) bd0 = q == s ? vdesc[q] : bd0;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                if (kk >= 4 && !full_blk) break;
                // P of keys 16 kk .. 16 kk + 15: columns 64 (kk / 4) + 8 (kk % 4) of S_t
                const uint64_t bd = bd0 + (uint64_t)(((kk / 4) * kVHalf + (kk % 4) * 32) >> 4);
                mma_ts(tb + kColO + 128u * t, tb + kColS + 128u * t + 64u * (kk / 4) + 8u * (kk % 4),
                       bd, id_pv, (j > 0 || kk > 0) ? 1u : 0u);
            }
        };
        for (int i = 0; i < n_blocks; ++i) {
            const int sk = i % kStagesK, sv = i % kStagesV;
            if (!wait_or_fail(&sh.k_full[sk], (uint32_t)(i / kStagesK) & 1u, a.status, failed)) break;
            tc_fence_after();
            if (lane == 0) qk(0, i);
            __syncwarp();
            if (i > 0) {
                if (!wait_or_fail(&sh.p_full[1], (uint32_t)(i - 1) & 1u, a.status, failed)) break;
                tc_fence_after();
                if (lane == 0) {
                    pv(1, i - 1);
                    mma_commit(&sh.v_empty[(i - 1) % kStagesV]);   // both P V of block i-1 issued
                }
                __syncwarp();
            }
            if (lane == 0) {
                qk(1, i);
                mma_commit(&sh.k_empty[sk]);                    // both Q K^T of block i issued
            }
            __syncwarp();
            if (!wait_or_fail(&sh.v_full[sv], (uint32_t)(i / kStagesV) & 1u, a.status, failed)) break;
            if (!wait_or_fail(&sh.p_full[0], (uint32_t)i & 1u, a.status, failed)) break;
            tc_fence_after();
            if (lane == 0) pv(0, i);
            __syncwarp();
        }
        if (!failed && n_blocks > 0 &&
            wait_or_fail(&sh.p_full[1], (uint32_t)(n_blocks - 1) & 1u, a.status, failed)) {
            tc_fence_after();
            if (lane == 0) {
                pv(1, n_blocks - 1);
                mma_commit(&sh.v_empty[(n_blocks - 1) % kStagesV]);
            }
            __syncwarp();
        }
        if (lane == 0) mma_commit(&sh.o_full);          // tracks every MMA issued above
        __syncwarp();
    } else if (warp == kWarpBias) {
        // ------------------------------------------------------------ routing biases
        const int n_batches = (n_chunks + kBiasBatch - 1) / kBiasBatch;
        for (int bt = 0; bt < n_batches; ++bt) {
            float *buf = bias_s + (bt & 1) * kBiasBatch * RT2;
            for (int e = lane; e < kBiasBatch * RT2; e += 32) {
                const int k = e / RT2, u = e % RT2, ci = bt * kBiasBatch + k;
                float v = 0.f;
                if (ci < n_chunks && !a.ignore_routing) {
                    const int c = chunk_at(ci), t = tp0 + u;
                    const int ctu = t / BC;
                    if (t >= a.t_end || c > ctu) {
                        v = -INFINITY;
                    } else if (c < ctu) {
                        const long long rowi = bg * a.T + t;
                        const bool act = dash_check(t < a.T && c < a.Cf, a.status) &&
                                         ((a.mask[rowi * a.W + (c >> 6)] >> (c & 63)) & 1ull);
                        if (!act) {
                            v = -INFINITY;
                        } else {
                            const float dot = route_dot<D>(qbar + u * D, a.summary + (bg * a.Cf + c) * D);
                            const float tau = a.tau[rowi];
                            if (a.rc.kind == kKindTopk) {
                                v = 0.f;                        // top-k: uniform prior
                            } else if (a.rc.kind == 0) {
                                v = a.rc.sigma2 * (__fmul_rn(dot, a.rc.sscale) - tau);
                            } else {
                                const float m = __fsub_rn(__fmul_rn(dot, a.rc.xscale), tau);
                                v = a.rc.bscale2 * log2f(fmaxf(m, 1e-37f));
                            }
                        }
                    }
                }
                buf[e] = v;
            }
            __syncwarp();
            named_sync(1, 32 + kSmThreads);
        }
    } else if (is_sm) {
        // ------------------------------------------------------------ softmax (tile grp)
        // Two threads per row: warp (sp, kq) owns keys 64 kq .. 64 kq + 63 of every block (one
        // chunk half, one bias), in two passes of 32 columns; P of its keys goes to columns
        // 64 kq .. 64 kq + 31 of S_grp.  Named barrier 2 + grp joins the tile's 8 warps.
        const uint32_t s_base = tb + ((uint32_t)(32 * sp) << 16) + kColS + 128u * grp + 64u * kq;
        const int u_bias = grp * RT + u_row;                  // token index in the bias batch
        float m_ref = 0.f;
        const uint64_t scale2 = f2_pack(a.qk_scale2, a.qk_scale2);
        uint64_t lsum = f2_pack(0.f, 0.f);
        for (int j = 0; j < n_blocks; ++j) {
            const int e0 = BC == 64 ? 2 * j : j;
            if (e0 % kBiasBatch == 0) named_sync(1, 32 + kSmThreads);
            const bool ok = wait_or_fail(&sh.s_full[grp], (uint32_t)j & 1u, a.status, failed);
            if (ok) tc_fence_after();
            const int e = entry_of(j, kq);
            int key0 = 0;
            float bias2 = -INFINITY;
            bool diag = false;
            if (e >= 0 && row_ok) {
                const int c = chunk_at(e);
                key0 = key0_of(j, kq);
                if (c == ct_max) {
                    bias2 = 0.f;
                    diag = true;
                } else {
                    bias2 = a.ignore_routing ? 0.f
                                             : bias_s[((e / kBiasBatch) & 1) * kBiasBatch * RT2 +
                                                      (e % kBiasBatch) * RT2 + u_bias];
                }
            }
            const bool dead = __all_sync(kFull, bias2 == -INFINITY);
            if (j == 0) {
                // Exact row maximum over the diagonal chunk's causally visible keys (block 0
                // holds them), shared by the row's two threads: the fixed reference.
                float mx = -INFINITY;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    uint32_t sv[32];
                    if (ok) {
                        tmem_ld32(s_base + 32u * hh, sv);
                        tmem_wait_ld();
                    }
                    if (ok && diag) {
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            if (key0 + 32 * hh + i <= t_row) mx = fmaxf(mx, __uint_as_float(sv[i]) * a.qk_scale2);
                    }
                }
                sh.mpart[grp][kq][row] = mx;
                named_sync(2 + grp, kGrpWarps * 32);
                const float m2 = fmaxf(sh.mpart[grp][0][row], sh.mpart[grp][1][row]);
                m_ref = m2 == -INFINITY ? 0.f : m2;
            }
            if (!ok) continue;
            const float c2 = bias2 - m_ref;
            const uint64_t cc = f2_pack(c2, c2);
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                uint32_t pw[16];
                if (dead) {
#pragma unroll
                    for (int i = 0; i < 16; ++i) pw[i] = 0u;
                } else {
                    uint32_t sv[32];
                    tmem_ld32(s_base + 32u * hh, sv);
                    tmem_wait_ld();
                    if (diag) {
                        const int lim = t_row - key0 - 32 * hh;      // keys i > lim are in the future
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const float x0 = 2 * i <= lim ? fmaf(__uint_as_float(sv[2 * i]), a.qk_scale2, c2) : -INFINITY;
                            const float x1 = 2 * i + 1 <= lim ? fmaf(__uint_as_float(sv[2 * i + 1]), a.qk_scale2, c2) : -INFINITY;
                            pw[i] = pack_bf16x2(fast_exp2(x0), fast_exp2(x1));
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            float x0, x1;
                            f2_unpack(f2_fma(f2_pack(__uint_as_float(sv[2 * i]), __uint_as_float(sv[2 * i + 1])), scale2, cc), x0, x1);
                            pw[i] = pack_bf16x2(fast_exp2(x0), fast_exp2(x1));
                        }
                    }
#pragma unroll
                    for (int i = 0; i < 16; ++i)     // row sums of the bf16 weights (reading C19)
                        lsum = f2_add(lsum, f2_pack(__uint_as_float(pw[i] << 16), __uint_as_float(pw[i] & 0xffff0000u)));
                }
                // P of keys 64 kq + 32 hh .. + 31 -> columns 64 kq + 16 hh .. + 15 (S of those
                // columns was loaded in pass 0).
                tmem_st16(s_base + 16u * hh, pw);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh.p_full[grp]);
        }
        // Epilogue: l = the row's two partial sums; O / l -> bf16, each thread 64 dims.
        {
            float l0, l1;
            f2_unpack(lsum, l0, l1);
            sh.lpart[grp][kq][row] = l0 + l1;
        }
        named_sync(2 + grp, kGrpWarps * 32);
        const float l = sh.lpart[grp][0][row] + sh.lpart[grp][1][row];
        const bool ok_o = wait_or_fail(&sh.o_full, 0, a.status, failed);
        if (ok_o) {
            tc_fence_after();
            if (__any_sync(kFull, row_ok && !isfinite(l)) && lane == 0 && kq == 0) report(a.status, DASH_ERR_RANGE_CLAMPED);
            const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                uint32_t o[32];
                tmem_ld32(tb + ((uint32_t)(32 * sp) << 16) + kColO + 128u * grp + 64u * kq + 32u * hh, o);
                tmem_wait_ld();
                if (row_ok) {
                    __nv_bfloat16 *orow = reinterpret_cast<__nv_bfloat16 *>(a.out) +
                                          (((long long)b * a.Hq + h_row) * a.T + t_row) * D + 64 * kq + 32 * hh;
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
    }

    // ---------------------------------------------------------------- teardown
    if (failed) sh.failed = 1;
    tc_fence_before();
    __syncthreads();
    if (sh.failed && lane == 0 && warp == kWarpMma) mbar_wait_bounded(&sh.o_full, 0);
    __syncthreads();
    tc_fence_after();
    if (warp == kWarpMma) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tb), "r"(kTmemCols));
    }
}

// ---------------------------------------------------------------- host side
namespace {

using EncodeFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                              const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                              const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                              CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn pp_encode() {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
        return nullptr;
    return reinterpret_cast<EncodeFn>(fn);
}

// 3-D bf16 map, 128-byte swizzle: dims (inner, rows, planes), box (64, box_rows, 1).
bool pp_map(EncodeFn enc, CUtensorMap *m, const void *ptr, cuuint64_t inner, cuuint64_t rows,
            cuuint64_t planes, cuuint32_t box_rows) {
    cuuint64_t dims[3] = {inner, rows, planes};
    cuuint64_t strides[2] = {inner * 2, inner * 2 * rows};
    cuuint32_t box[3] = {64, box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t pp_smem_bytes(int RT, int C) {
    size_t off = kRingBytes;
    off += (size_t)2 * kBiasBatch * 2 * RT * 4;  // bias batches of the pair's tokens
    off += (size_t)2 * RT * 128 * 4;             // qbar
    off += (size_t)((C + 7) & ~7) * 2;           // chunk list
    return off + 1024;
}

template <int BC>
cudaError_t launch_pp_t(const StageArgs &a, cudaStream_t st) {
    static EncodeFn enc = pp_encode();
    if (!enc || !a.vt) return cudaErrorNotSupported;
    const int BHkv = a.B * a.Hkv;
    cudaError_t e = a.vt_ready ? cudaSuccess : launch_vtranspose(a.v, a.vt, BHkv, a.T, 128, st);
    if (e != cudaSuccess) return e;
    const cuuint64_t T8 = (cuuint64_t)((a.T + 7) & ~7);
    CUtensorMap mk, mk128, mvt;
    if (!pp_map(enc, &mk, a.k, 128, (cuuint64_t)a.T, (cuuint64_t)BHkv, 64) ||
        !pp_map(enc, &mk128, a.k, 128, (cuuint64_t)a.T, (cuuint64_t)BHkv, 128) ||
        !pp_map(enc, &mvt, a.vt, T8, 128, (cuuint64_t)BHkv, 128))
        return cudaErrorInvalidValue;
    PpArgs ta;
    ta.s = a;
    ta.RT = 128 / a.G;
    ta.pair0 = a.t_begin / (2 * ta.RT);
    ta.n_pairs_bg = ((a.t_end + ta.RT - 1) / ta.RT + 1) / 2 - ta.pair0;
    size_t off = kRingBytes;
    ta.off_bias = off;
    off += (size_t)2 * kBiasBatch * 2 * ta.RT * 4;
    ta.off_qbar = off;
    off += (size_t)2 * ta.RT * 128 * 4;
    ta.off_list = off;
    const size_t smem = pp_smem_bytes(ta.RT, a.C);
    auto kern = k_attend_pp<BC>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const long long grid = (long long)ta.n_pairs_bg * BHkv;
    if (grid == 0) return cudaSuccess;
    kern<<<(unsigned)grid, kPpThreads, smem, st>>>(mk, mk128, mvt, ta);
    return cudaGetLastError();
}

}  // namespace

bool attend_pp_supported(const StageArgs &a) {
    if (!(a.D == 128 && a.G >= 8 && a.G <= 128 && 128 % a.G == 0 && (a.Bc == 64 || a.Bc == 128)))
        return false;
    return pp_smem_bytes(128 / a.G, a.C) + sizeof(PpShared) <= 227 * 1024;
}

cudaError_t launch_attend_pp(const StageArgs &a, cudaStream_t st) {
    if (a.Bc == 64) return launch_pp_t<64>(a, st);
    if (a.Bc == 128) return launch_pp_t<128>(a, st);
    return cudaErrorInvalidValue;
}

}  // namespace dash
