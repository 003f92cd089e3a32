// attend_tok.cu -- Stage 2 per token on the 5th-generation tensor cores (D = 128, G = 16,
// chunk 64): no query tile ever walks the union of several tokens' routed chunks.
//
// gist.science "DashAttention: Differentiable and Adaptive Sparse Hierarchical Attention",
// Technische Zusammenfassung, "Stufe 2: Prior-induzierte spaerliche Softmax": the kernel
// walks the active chunks of the bit-packed mask, adds the routing bias log p to the logits
// of an active chunk, skips zero-probability chunks, and keeps the diagonal chunk as its own
// (causal, bias 0) branch.
//
// Shapes.  The 16 heads of one token share one routing, so they are the N = 16 columns of the
// MMAs, and keys (QK) or head dims (PV) are the M = 128 rows:
//   S^T[128 keys x 16] = [K_a; K_b] Q_t^T   A = a chunk pair in tensor memory, B = Q_t (smem)
//   O_t^T[128 x 16]   += V_c^T P_t^T         A = V_c^T in tensor memory, B = P_t (smem)
// One CTA owns a window of 16 consecutive tokens of one (b, g); they share the diagonal
// chunk.  It streams the diagonal chunk and then the union of the window's routed chunks in
// pairs (pair 0 = diagonal + first routed chunk, pair p = list entries 2p and 2p+1).  A
// pair's K and V^T are staged by TMA and copied into tensor memory once (tcgen05.cp), then
// reused by every window token that routed to either chunk.  A token that routed to one chunk
// of a pair still issues the whole M = 128 QK (an M = 64 MMA costs the same issue time) but
// only that chunk's exponentials and PV.
//
// Pipelines.  Four independent pipelines own 4 tokens each (u = L + 4m): one MMA-issuing
// warp and four softmax warps, one per tensor-memory sub-partition (warps 0-1 of a pipeline
// hold chunk a's 64 keys, warps 2-3 chunk b's).  The softmax releases the S slot as soon as
// it has loaded it, so the QK of the next item overlaps the exponentials of the current one;
// P is double-buffered in shared memory.
//
// Softmax reference.  The diagonal chunk (chunk a of pair 0) gives every token its exact
// per-head maximum m_h, the fixed reference of all its chunks (p = 2^(s - m_h)), so O needs
// no running rescale.  Routed logits can exceed m_h; excesses above 100 (log2 units) are
// clamped there, so neither bf16 P nor the fp32 sums over up to 2^17 keys can overflow, and
// reported as DASH_ERR_RANGE_CLAMPED through the status word.
//
// Ordering.  K pairs are double-buffered in tensor memory, the V^T pair single-buffered.
// Each pipeline closes the K and V phases of every pair in order (one arrival per pair, items
// or not), and before it blocks on a resource of pair r it has closed all phases of pairs
// below r, so the pipeline waiting on the lowest pair can always proceed.  Every wait is
// bounded and warp-uniform.
//
// Warps: 0 K producer (TMA + tensor-memory copy), 1 and 3 routing-bias producers, 2 tensor
// memory owner and chunk list, then V producer, 4-7 MMA issuers (pipeline L), 8-23 softmax
// (pipeline L: warps 8+4L .. 11+4L).  Tensor memory (512 columns): O 16x16 | K pairs 2x64 |
// V^T pair 64 | S 4x16.
#include "kernels.cuh"
#include "tc_common.cuh"

namespace dash {
using namespace tcx;
namespace {

constexpr int kW = 16;                            // tokens per window
constexpr int kLanes = 4;                         // pipelines
constexpr int kTpl = kW / kLanes;                 // tokens per pipeline
constexpr uint32_t kKStage = 32768;               // K pair: 2 panels x 128 rows x 128 B
constexpr uint32_t kVStage = 32768;               // V^T pair: 2 chunks x 128 dims x 128 B
constexpr int kBatch = 32;                        // list entries per routing-bias batch
constexpr int kPairsPerBatch = kBatch / 2;
constexpr int kNBias = 4;                         // bias ring slots
constexpr int kWarpK = 0, kWarpBias0 = 1, kWarpAdmin = 2, kWarpBias1 = 3, kWarpMma0 = 4,
              kWarpSm0 = 8;
constexpr int kThreads = 24 * 32;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0, kColK = 256, kColV = 384, kColS = 448;
constexpr int kQbarStride = 132;                  // padded row of the query means (floats)
constexpr float kMaxExcess = 100.f;               // log2 units above the reference
constexpr int kMaxChunks = 4096;

struct TokShared {
    uint64_t k_full[2], k_empty[2], k_ready[2], k_free[2];
    uint64_t v_full, v_empty, v_ready, v_free;
    uint64_t bias_full[kNBias], bias_empty[kNBias];
    uint64_t s_full[kLanes], s_free[kLanes], p_full[kLanes][2], o_done[kLanes], x_bar[kLanes];
    uint64_t q_full;
    uint32_t tmem_base;
    int n_ch;
    int failed;
    int abort;
};

__device__ __forceinline__ bool wait_u(uint64_t *bar, uint32_t parity, uint32_t *status, bool &failed) {
    if (failed) return false;
    const bool ok = __all_sync(kFull, mbar_wait_bounded(bar, parity));
    if (!ok) {
        if ((threadIdx.x & 31) == 0) report(status, DASH_ERR_DEVICE_TIMEOUT);
        failed = true;
    }
    return ok;
}
// Non-blocking, warp-uniform test of an mbarrier phase (test_wait never suspends, unlike
// try_wait, which may sleep for a hardware-defined window before it reports "not yet").
__device__ __forceinline__ bool test_u(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return __all_sync(kFull, ok != 0);
}

// 16 per-head values spread over a warp's 32 key lanes -> lane l holds the reduction for head
// l >> 1 in v[0] (reduce-scatter over lane bits 4..1, then an all-reduce over bit 0).
template <bool kMax>
__device__ __forceinline__ float head_reduce(float (&v)[16], int lane) {
#pragma unroll
    for (int o = 16, n = 8; o >= 2; o >>= 1, n >>= 1) {
        const bool upper = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < n; ++i) {
            const float send = upper ? v[i] : v[i + n];
            const float keep = upper ? v[i + n] : v[i];
            const float got = __shfl_xor_sync(kFull, send, o);
            v[i] = kMax ? fmaxf(keep, got) : keep + got;
        }
    }
    const float got = __shfl_xor_sync(kFull, v[0], 1);
    return kMax ? fmaxf(v[0], got) : v[0] + got;
}

}  // namespace

struct TokArgs {
    StageArgs s;
    int n_win;             // windows per (b, g)
    size_t off_q, off_k, off_v, off_p, off_bias, off_qbar, off_mref, off_mpart, off_lpart, off_list;
};

__global__ void __launch_bounds__(kThreads, 1)
k_attend_tok(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmVt,
             const __grid_constant__ CUtensorMap tmQ, const TokArgs ta) {
    constexpr int D = 128, BC = 64, G = 16;
    extern __shared__ unsigned char smem_dyn[];
    __shared__ TokShared sh;
    const StageArgs &a = ta.s;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    unsigned char *base = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~(uintptr_t)1023);
    unsigned char *qwin = base + ta.off_q;       // [2 panels][16 tokens][16 heads][128 B]
    unsigned char *kst = base + ta.off_k;        // [2 stages][2 panels][128 rows][128 B]
    unsigned char *vst = base + ta.off_v;        // [2 chunks][128 dims][128 B]
    unsigned char *pbuf = base + ta.off_p;       // [4 pipelines][2 buffers][4 KB]
    float *bias_ring = reinterpret_cast<float *>(base + ta.off_bias);  // [kNBias][kBatch][16]
    float *qbar = reinterpret_cast<float *>(base + ta.off_qbar);       // [16][kQbarStride]
    float *mref = reinterpret_cast<float *>(base + ta.off_mref);       // [16 tokens][16 heads]
    float *mpart = reinterpret_cast<float *>(base + ta.off_mpart);     // [16][2 warps][16]
    float *lpart = reinterpret_cast<float *>(base + ta.off_lpart);     // [16][4 warps][16]
    int16_t *list = reinterpret_cast<int16_t *>(base + ta.off_list);

    const int BHkv = a.B * a.Hkv;
    const int wrev = blockIdx.x / BHkv, bgi = blockIdx.x % BHkv;
    const int win = ta.n_win - 1 - wrev;          // longest windows first
    const int b = bgi / a.Hkv, g = bgi % a.Hkv;
    const long long bg = bgi;
    const int t0 = win * kW;
    const int cd = t0 / BC;                       // the window's diagonal chunk
    bool failed = false;

    // ------------------------------------------------------------------ setup
    if (warp == kWarpAdmin) tmem_alloc(&sh.tmem_base, kTmemCols);
    if (threadIdx.x == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&sh.k_full[s], 1);
            mbar_init(&sh.k_empty[s], 1);
            mbar_init(&sh.k_ready[s], 1);
            mbar_init(&sh.k_free[s], kLanes);
        }
        mbar_init(&sh.v_full, 1);
        mbar_init(&sh.v_empty, 1);
        mbar_init(&sh.v_ready, 1);
        mbar_init(&sh.v_free, kLanes);
        for (int k = 0; k < kNBias; ++k) {
            mbar_init(&sh.bias_full[k], 1);
            mbar_init(&sh.bias_empty[k], kLanes + 4 * kLanes);
        }
        for (int L = 0; L < kLanes; ++L) {
            mbar_init(&sh.s_full[L], 1);
            mbar_init(&sh.s_free[L], 4);
            mbar_init(&sh.p_full[L][0], 4);
            mbar_init(&sh.p_full[L][1], 4);
            mbar_init(&sh.o_done[L], 1);
            mbar_init(&sh.x_bar[L], 4);
        }
        mbar_init(&sh.q_full, 1);
        sh.failed = 0;
        // A CTA that starts after another one timed out does no work, so a failing launch
        // ends within about one wave of bounded waits.
        sh.abort = *reinterpret_cast<volatile uint32_t *>(a.status) == DASH_ERR_DEVICE_TIMEOUT;
        fence_mbar_init();
    }
    if (warp == kWarpAdmin) {
        // Chunk list: the diagonal chunk first, then the union of the window's routed chunks.
        const int W = a.W, wlim = cd > 0 ? (cd - 1) / 64 : -1;
        int pos = 1;
        if (lane == 0) list[0] = (int16_t)cd;
        for (int w0 = 0; w0 <= wlim; w0 += 32) {
            const int w = w0 + lane;
            uint64_t word = 0;
            if (w <= wlim) {
                if (a.ignore_routing) {
                    word = ~0ull;
                } else {
                    for (int u = 0; u < kW; ++u) {
                        const int t = t0 + u;
                        if (t < a.T) word |= __ldg(a.mask + (bg * a.T + t) * W + w);
                    }
                }
                const int lim = cd - 64 * w;                  // routed bits are < cd
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
                list[p++] = (int16_t)(w * 64 + bit);
            }
            pos += __shfl_sync(kFull, incl, 31);
        }
        if (lane == 0) sh.n_ch = pos;
    }
    if ((warp == kWarpBias0 || warp == kWarpBias1) && !a.ignore_routing) {
        // Group-mean queries of the window's tokens (the routing arithmetic of Stage 1).
        const __nv_bfloat16 *q = reinterpret_cast<const __nv_bfloat16 *>(a.q);
        const int l64 = lane + (warp == kWarpBias1 ? 32 : 0);
        for (int idx = l64; idx < kW * (D / 8); idx += 64) {
            const int u = idx / (D / 8), d8 = (idx % (D / 8)) * 8, t = t0 + u;
            float m[8];
            if (t < a.T) {
                group_mean8(q + (((long long)b * a.Hq + g * G) * a.T + t) * D + d8,
                            (long long)a.T * D, G, m);
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) m[e] = 0.f;
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) qbar[u * kQbarStride + d8 + e] = m[e];
        }
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tb = sh.tmem_base;
    if (sh.abort) {
        if (warp == kWarpAdmin) tmem_dealloc(tb, kTmemCols);
        return;
    }
    const int n_ch = sh.n_ch;
    const int n_pairs = (n_ch + 1) / 2;
    const int n_batches = (n_ch + kBatch - 1) / kBatch;

    if (warp == kWarpK) {
        // ---------------------------------------------------------------- K producer
        auto issue_k = [&](int p) {              // lane 0: TMA of pair p into stage p & 1
            unsigned char *stg = kst + (size_t)(p & 1) * kKStage;
            const bool hb = 2 * p + 1 < n_ch;
            uint64_t *bar = &sh.k_full[p & 1];
            mbar_arrive_expect_tx(bar, hb ? kKStage : kKStage / 2);
            const int ca = list[2 * p];
            tma_load_3d(stg, &tmK, 0, ca * BC, (int)bg, bar);
            tma_load_3d(stg + 16384, &tmK, 64, ca * BC, (int)bg, bar);
            if (hb) {
                const int cb = list[2 * p + 1];
                tma_load_3d(stg + 8192, &tmK, 0, cb * BC, (int)bg, bar);
                tma_load_3d(stg + 24576, &tmK, 64, cb * BC, (int)bg, bar);
            }
        };
        if (lane == 0) {
            mbar_arrive_expect_tx(&sh.q_full, kW * 4096);
            for (int u = 0; u < kW; ++u)
                for (int h = 0; h < 2; ++h)
                    tma_load_4d(qwin + h * 32768 + u * 2048, &tmQ, 64 * h, t0 + u, g * G, b, &sh.q_full);
            issue_k(0);
            if (n_pairs > 1) issue_k(1);
        }
        __syncwarp();
        int issued = min(2, n_pairs), landed = 0, copied = 0;
        for (int p = 0; p < n_pairs; ++p) {
            const int st = p & 1;
            const uint32_t ph = (uint32_t)(p >> 1) & 1u;
            if (!wait_u(&sh.k_full[st], ph, a.status, failed)) break;
            landed = p + 1;
            if (!wait_u(&sh.k_free[st], ph ^ 1u, a.status, failed)) break;   // pair p-2 done
            tc_fence_after();
            if (lane == 0) {
                const uint32_t src = smem_u32(kst + (size_t)st * kKStage);
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    tmem_cp_128x256b(tb + kColK + 64u * st + 8u * k,
                                     smem_desc_sw128(src + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024));
                mma_commit(&sh.k_ready[st]);
                mma_commit(&sh.k_empty[st]);
            }
            __syncwarp();
            copied = p + 1;
            if (p + 2 < n_pairs) {
                if (!wait_u(&sh.k_empty[st], ph, a.status, failed)) break;  // copy read the stage
                if (lane == 0) issue_k(p + 2);
                __syncwarp();
                issued = p + 3;
            }
        }
        if (failed && lane == 0) {
            // Let the bulk copies and tensor-memory copies in flight land before exit.
            mbar_wait_bounded(&sh.q_full, 0);
            for (int j = landed; j < issued; ++j) mbar_wait_bounded(&sh.k_full[j & 1], (uint32_t)(j >> 1) & 1u);
            if (copied > 0) mbar_wait_bounded(&sh.k_empty[(copied - 1) & 1], (uint32_t)((copied - 1) >> 1) & 1u);
        }
        __syncwarp();
    } else if (warp == kWarpAdmin) {
        // ---------------------------------------------------------------- V^T producer
        auto issue_v = [&](int p) {
            const bool hb = 2 * p + 1 < n_ch;
            mbar_arrive_expect_tx(&sh.v_full, hb ? kVStage : kVStage / 2);
            tma_load_3d(vst, &tmVt, list[2 * p] * BC, 0, (int)bg, &sh.v_full);
            if (hb) tma_load_3d(vst + 16384, &tmVt, list[2 * p + 1] * BC, 0, (int)bg, &sh.v_full);
        };
        if (lane == 0 && n_pairs > 0) issue_v(0);
        __syncwarp();
        int issued = min(1, n_pairs), landed = 0, copied = 0;
        for (int p = 0; p < n_pairs; ++p) {
            const uint32_t ph = (uint32_t)p & 1u;
            if (!wait_u(&sh.v_full, ph, a.status, failed)) break;
            landed = p + 1;
            if (!wait_u(&sh.v_free, ph ^ 1u, a.status, failed)) break;       // PV of pair p-1 done
            tc_fence_after();
            if (lane == 0) {
                const uint32_t src = smem_u32(vst);
                const int nchunk = 2 * p + 1 < n_ch ? 2 : 1;
                for (int c = 0; c < nchunk; ++c)
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        tmem_cp_128x256b(tb + kColV + 32u * c + 8u * k,
                                         smem_desc_sw128(src + c * 16384 + k * 32, 16, 1024));
                mma_commit(&sh.v_ready);
                mma_commit(&sh.v_empty);
            }
            __syncwarp();
            copied = p + 1;
            if (p + 1 < n_pairs) {
                if (!wait_u(&sh.v_empty, ph, a.status, failed)) break;
                if (lane == 0) issue_v(p + 1);
                __syncwarp();
                issued = p + 2;
            }
        }
        if (failed && lane == 0) {
            for (int j = landed; j < issued; ++j) mbar_wait_bounded(&sh.v_full, (uint32_t)j & 1u);
            if (copied > 0) mbar_wait_bounded(&sh.v_empty, (uint32_t)(copied - 1) & 1u);
        }
        __syncwarp();
    } else if (warp == kWarpBias0 || warp == kWarpBias1) {
        // ---------------------------------------------------------------- routing biases
        // Batch k (list entries 32k .. 32k+31) is produced by warp k % 2 into ring slot k % 4.
        for (int k = (warp == kWarpBias0 ? 0 : 1); k < n_batches; k += 2) {
            const int slot = k % kNBias;
            if (!wait_u(&sh.bias_empty[slot], ((uint32_t)(k / kNBias) & 1u) ^ 1u, a.status, failed)) break;
            float *ring = bias_ring + slot * kBatch * kW;
            // Entry e = lane + 32 i: list entry j = 32k + e / 16, token u = e % 16.  Mask bits first
            // (independent loads), then the biases of the routed entries.
            uint32_t routed = 0;
#pragma unroll
            for (int i = 0; i < (kBatch * kW) / 32; ++i) {
                const int e = lane + 32 * i, j = k * kBatch + (e >> 4), t = t0 + (e & 15);
                if (j >= 1 && j < n_ch && t < a.T && !a.ignore_routing) {
                    const int c = list[j];
                    const uint64_t w = __ldg(a.mask + (bg * a.T + t) * a.W + (c >> 6));
                    if ((w >> (c & 63)) & 1ull) routed |= 1u << i;
                }
            }
#pragma unroll 1
            for (int i = 0; i < (kBatch * kW) / 32; ++i) {
                const int e = lane + 32 * i, j = k * kBatch + (e >> 4), u = e & 15, t = t0 + u;
                float v = -INFINITY;
                if (j < n_ch && t < a.T) {
                    if (j == 0 || a.ignore_routing) {
                        v = 0.f;
                    } else if ((routed >> i) & 1u) {
                        const int c = list[j];
                        const long long rowi = bg * a.T + t;
                        const float dot = route_dot<D>(qbar + u * kQbarStride, a.summary + (bg * a.Cf + c) * D);
                        const float tau = __ldg(a.tau + rowi);
                        if (a.rc.kind == 0) {
                            v = a.rc.sigma2 * (__fmul_rn(dot, a.rc.sscale) - tau);
                        } else {
                            const float m = __fsub_rn(__fmul_rn(dot, a.rc.xscale), tau);
                            v = a.rc.bscale2 * log2f(fmaxf(m, 1e-37f));
                        }
                    }
                }
                ring[e] = v;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh.bias_full[slot]);
        }
    } else if (warp >= kWarpMma0 && warp < kWarpMma0 + kLanes) {
        // ---------------------------------------------------------------- MMA issuer, pipeline L
        const int L = warp - kWarpMma0;
        constexpr uint32_t id_qk = idesc_bf16(128, 16, 0);
        constexpr uint32_t id_pv = idesc_bf16(128, 16, 1);
        const uint32_t d_s = tb + kColS + 16u * L;
        const uint32_t p_base = smem_u32(pbuf + L * 8192);
        // Phase bookkeeping: kw / vw = last pair whose k_ready / v_ready phase was waited,
        // kq / vq = next pair whose k_free / v_free arrival is still owed.
        int kw = -1, kq = 0, vw = -1, vq = 0;
        int pend_u = -1, pend_p = 0, pend_i = 0;       // the item whose PV is still to issue
        bool pend_a = false, pend_b = false;
        int it = 0;
        auto ensure_k = [&](int p) -> bool {
            while (kw < p) {
                const int r = kw + 1;
                if (!wait_u(&sh.k_ready[r & 1], (uint32_t)(r >> 1) & 1u, a.status, failed)) return false;
                kw = r;
            }
            return true;
        };
        auto try_k = [&](int p) -> bool {
            while (kw < p) {
                const int r = kw + 1;
                if (!test_u(&sh.k_ready[r & 1], (uint32_t)(r >> 1) & 1u)) return false;
                kw = r;
            }
            return true;
        };
        auto close_k = [&](int p) -> bool {           // arrive k_free for every pair < p
            while (kq < p) {
                if (!ensure_k(kq)) return false;
                if (lane == 0) mma_commit(&sh.k_free[kq & 1]);
                __syncwarp();
                ++kq;
            }
            return true;
        };
        auto ensure_v = [&](int q) -> bool {
            while (vw < q) {
                const int r = vw + 1;
                if (!wait_u(&sh.v_ready, (uint32_t)r & 1u, a.status, failed)) return false;
                vw = r;
            }
            return true;
        };
        auto close_v = [&](int q) -> bool {           // arrive v_free for every pair < q
            while (vq < q) {
                if (!ensure_v(vq)) return false;
                if (lane == 0) mma_commit(&sh.v_free);
                __syncwarp();
                ++vq;
            }
            return true;
        };
        auto do_pv = [&]() -> bool {
            if (!close_v(pend_p) || !ensure_v(pend_p)) return false;
            // One barrier per P buffer: the softmax can run at most one phase ahead of it.
            if (!wait_u(&sh.p_full[L][pend_i & 1], (uint32_t)(pend_i >> 1) & 1u, a.status, failed)) return false;
            tc_fence_after();
            if (lane == 0) {
                const uint32_t pb = p_base + (uint32_t)(pend_i & 1) * 4096u;
                const uint32_t d_o = tb + kColO + 16u * pend_u;
                if (pend_a) {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_ts(d_o, tb + kColV + 8u * kk, smem_desc_noswz(pb + 256u * kk, 128, 2048), id_pv,
                               (pend_p > 0 || kk > 0) ? 1u : 0u);
                }
                if (pend_b) {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_ts(d_o, tb + kColV + 32u + 8u * kk,
                               smem_desc_noswz(pb + 1024u + 256u * kk, 128, 2048), id_pv, 1u);
                }
            }
            __syncwarp();
            pend_u = -1;
            return true;
        };
        // Close the K and V phases of every pair below p in pair order, so that each blocking
        // wait on a pair-r resource happens with all phases below r already closed.
        auto close_all = [&](int p) -> bool {
            while (kq < p || vq < p) {
                const int r = min(kq, vq);
                if (kq == r && !close_k(r + 1)) return false;
                if (vq == r && r < p && !close_v(r + 1)) return false;
            }
            return true;
        };
        // Before blocking on a resource of pair p: issue the pending PV and close every phase
        // of the pairs below p.
        auto flush_below = [&](int p) -> bool {
            if (pend_u >= 0 && pend_p < p && !do_pv()) return false;
            return close_all(p);
        };
        bool ok = wait_u(&sh.q_full, 0, a.status, failed);
        for (int p = 0; p < n_pairs && ok; ++p) {
            const int k = p / kPairsPerBatch, slot = k % kNBias;
            if (p % kPairsPerBatch == 0) {
                const uint32_t par = (uint32_t)(k / kNBias) & 1u;
                if (!test_u(&sh.bias_full[slot], par)) {
                    if (!flush_below(p) || !wait_u(&sh.bias_full[slot], par, a.status, failed)) { ok = false; break; }
                }
            }
            const float *ring = bias_ring + slot * kBatch * kW + (2 * p - k * kBatch) * kW;
            const bool hb = 2 * p + 1 < n_ch;
            for (int m = 0; m < kTpl; ++m) {
                const int u = L + kLanes * m;
                const bool ra = ring[u] != -INFINITY;
                const bool rb = hb && ring[kW + u] != -INFINITY;
                if (!ra && !rb) continue;
                if (!try_k(p)) {
                    if (!flush_below(p) || !ensure_k(p)) { ok = false; break; }
                }
                if (!close_k(p)) { ok = false; break; }
                if (it > 0 && !wait_u(&sh.s_free[L], (uint32_t)(it - 1) & 1u, a.status, failed)) { ok = false; break; }
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t kslot = tb + kColK + 64u * (uint32_t)(p & 1);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t qa = smem_u32(qwin + (kk >> 2) * 32768 + u * 2048) + (uint32_t)(kk & 3) * 32u;
                        mma_ts(d_s, kslot + 8u * kk, smem_desc_sw128(qa, 16, 1024), id_qk, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(&sh.s_full[L]);
                }
                __syncwarp();
                if (pend_u >= 0 && !do_pv()) { ok = false; break; }
                pend_u = u;
                pend_p = p;
                pend_i = it;
                pend_a = ra;
                pend_b = rb;
                ++it;
            }
            if (!ok) break;
            if (p % kPairsPerBatch == kPairsPerBatch - 1 || p == n_pairs - 1) {
                if (lane == 0) mbar_arrive(&sh.bias_empty[slot]);
                __syncwarp();
            }
        }
        if (ok && pend_u >= 0) ok = do_pv();
        if (ok) ok = close_all(n_pairs);
        if (lane == 0) mma_commit(&sh.o_done[L]);    // after the last MMA, failure or not
        __syncwarp();
    } else if (warp >= kWarpSm0) {
        // ---------------------------------------------------------------- softmax, pipeline L
        const int L = (warp - kWarpSm0) >> 2, sp = warp & 3;
        const int half = sp >> 1;                         // 0: chunk a keys, 1: chunk b keys
        const int kp = 32 * sp + lane;                    // key row of S^T within the pair
        const uint32_t s_addr = tb + ((uint32_t)(32 * sp) << 16) + kColS + 16u * L;
        unsigned char *pb0 = pbuf + L * 8192;
        float lsum[kTpl];
#pragma unroll
        for (int m = 0; m < kTpl; ++m) lsum[m] = 0.f;
        int it = 0, xph = 0;
        for (int p = 0; p < n_pairs; ++p) {
            const int k = p / kPairsPerBatch, slot = k % kNBias;
            if (p % kPairsPerBatch == 0)
                wait_u(&sh.bias_full[slot], (uint32_t)(k / kNBias) & 1u, a.status, failed);
            const float *ring = bias_ring + slot * kBatch * kW + (2 * p - k * kBatch) * kW;
            const bool hb = 2 * p + 1 < n_ch;
#pragma unroll 1
            for (int m = 0; m < kTpl; ++m) {
                const int u = L + kLanes * m, t = t0 + u;
                const float ba = ring[u];
                const float bb = hb ? ring[kW + u] : -INFINITY;
                if (ba == -INFINITY && bb == -INFINITY) continue;
                const float bias2 = half ? bb : ba;
                const bool mine = bias2 != -INFINITY;
                const bool ok = wait_u(&sh.s_full[L], (uint32_t)it & 1u, a.status, failed);
                uint32_t sr[16];
                if (ok && mine) {
                    tc_fence_after();
                    tmem_ld16(s_addr, sr);
                    tmem_wait_ld();
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sh.s_free[L]);       // S slot free for the next QK
                // Keys of the diagonal chunk are causal; all keys of routed chunks are < t.
                const bool valid = ok && mine && (p > 0 || half == 1 || cd * BC + kp <= t);
                float mh[16];
                if (p == 0) {
                    // Exact per-head maximum over the diagonal chunk (warps 0-1), shared with
                    // the pipeline's 4 warps through an mbarrier exchange.
                    if (half == 0) {
                        float w[16];
#pragma unroll
                        for (int h = 0; h < 16; ++h) w[h] = valid ? __uint_as_float(sr[h]) * a.qk_scale2 : -INFINITY;
                        const float mx = head_reduce<true>(w, lane);
                        if ((lane & 1) == 0) mpart[(u * 2 + sp) * 16 + (lane >> 1)] = mx;
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sh.x_bar[L]);
                    wait_u(&sh.x_bar[L], (uint32_t)xph & 1u, a.status, failed);
                    ++xph;
#pragma unroll
                    for (int h = 0; h < 16; ++h) {
                        const float x = fmaxf(mpart[(u * 2) * 16 + h], mpart[(u * 2 + 1) * 16 + h]);
                        mh[h] = x == -INFINITY ? 0.f : x;
                    }
                    if (lane < 16) mref[u * 16 + lane] = mh[lane];   // same values from every warp
                } else {
#pragma unroll
                    for (int h = 0; h < 16; h += 4) {
                        const float4 x = *reinterpret_cast<const float4 *>(mref + u * 16 + h);
                        mh[h] = x.x;
                        mh[h + 1] = x.y;
                        mh[h + 2] = x.z;
                        mh[h + 3] = x.w;
                    }
                }
                if (mine) {
                    float pr[16];
                    float emax = -INFINITY;
#pragma unroll
                    for (int h = 0; h < 16; ++h) {
                        const float e = valid ? fmaf(__uint_as_float(sr[h]), a.qk_scale2, bias2 - mh[h]) : -INFINITY;
                        emax = fmaxf(emax, e);
                        pr[h] = fast_exp2(fminf(e, kMaxExcess));
                    }
                    if (__any_sync(kFull, emax > kMaxExcess) && lane == 0) report(a.status, DASH_ERR_RANGE_CLAMPED);
                    uint4 lo, hi;
                    lo.x = pack_bf16x2(pr[0], pr[1]);
                    lo.y = pack_bf16x2(pr[2], pr[3]);
                    lo.z = pack_bf16x2(pr[4], pr[5]);
                    lo.w = pack_bf16x2(pr[6], pr[7]);
                    hi.x = pack_bf16x2(pr[8], pr[9]);
                    hi.y = pack_bf16x2(pr[10], pr[11]);
                    hi.z = pack_bf16x2(pr[12], pr[13]);
                    hi.w = pack_bf16x2(pr[14], pr[15]);
                    unsigned char *pb = pb0 + (it & 1) * 4096 + (kp & 7) * 16 + (kp >> 3) * 128;
                    *reinterpret_cast<uint4 *>(pb) = lo;
                    *reinterpret_cast<uint4 *>(pb + 2048) = hi;
                    fence_proxy_async();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sh.p_full[L][it & 1]);
                    // Row sums of the bf16 weights the PV MMA multiplies (exact normalisation).
#pragma unroll
                    for (int h = 0; h < 16; ++h) pr[h] = __bfloat162float(__float2bfloat16_rn(pr[h]));
                    const float ls = head_reduce<false>(pr, lane);
                    if ((lane & 1) == 0) lsum[m] += ls;
                } else {
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sh.p_full[L][it & 1]);
                }
                ++it;
            }
            if (p % kPairsPerBatch == kPairsPerBatch - 1 || p == n_pairs - 1) {
                __syncwarp();
                if (lane == 0) mbar_arrive(&sh.bias_empty[slot]);
            }
        }
        // ------------------------------------------------------------ epilogue
#pragma unroll
        for (int m = 0; m < kTpl; ++m)
            if ((lane & 1) == 0) lpart[((L + kLanes * m) * 4 + sp) * 16 + (lane >> 1)] = lsum[m];
        const bool ok = wait_u(&sh.o_done[L], 0, a.status, failed);
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.x_bar[L]);
        const bool ok2 = wait_u(&sh.x_bar[L], (uint32_t)xph & 1u, a.status, failed);
        if (ok && ok2) {
            tc_fence_after();
            __nv_bfloat16 *out = reinterpret_cast<__nv_bfloat16 *>(a.out);
            const int dd = 32 * sp + lane;
#pragma unroll 1
            for (int m = 0; m < kTpl; ++m) {
                const int u = L + kLanes * m, t = t0 + u;
                uint32_t orow[16];
                tmem_ld16(tb + ((uint32_t)(32 * sp) << 16) + kColO + 16u * u, orow);
                tmem_wait_ld();
                if (t < a.T) {
#pragma unroll
                    for (int h = 0; h < 16; ++h) {
                        const float *lp = lpart + (u * 4) * 16 + h;
                        const float l = (lp[0] + lp[16]) + (lp[32] + lp[48]);
                        const float val = l > 0.f ? __uint_as_float(orow[h]) / l : 0.f;
                        out[(((long long)b * a.Hq + g * G + h) * a.T + t) * D + dd] = __float2bfloat16_rn(val);
                    }
                }
            }
        }
    }

    // ------------------------------------------------------------------ teardown
    if (failed) sh.failed = 1;
    tc_fence_before();
    __syncthreads();
    // Each MMA warp committed o_done[L] after its last MMA, failure or not: wait (bounded)
    // for the MMAs in flight before the tensor memory is released.
    if (sh.failed && warp >= kWarpMma0 && warp < kWarpMma0 + kLanes && lane == 0)
        mbar_wait_bounded(&sh.o_done[warp - kWarpMma0], 0);
    __syncthreads();
    tc_fence_after();
    if (warp == kWarpAdmin) tmem_dealloc(tb, kTmemCols);
}

// ---------------------------------------------------------------- host side
namespace {

using EncodeFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                              const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                              const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                              CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn tok_encode() {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
        return nullptr;
    return reinterpret_cast<EncodeFn>(fn);
}

bool encode(EncodeFn enc, CUtensorMap *m, const void *ptr, int rank, const cuuint64_t *dims,
            const cuuint64_t *strides, const cuuint32_t *box) {
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void *>(ptr), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

size_t attend_tok_vt_bytes(int B, int Hkv, int T, int D) {
    const size_t T8 = (size_t)((T + 7) & ~7);
    return (size_t)B * Hkv * D * T8 * 2;
}

bool attend_tok_supported(const StageArgs &a) {
    return a.D == 128 && a.G == 16 && a.Bc == 64 && a.C <= kMaxChunks;
}

cudaError_t launch_attend_tok(const StageArgs &a, cudaStream_t st) {
    static EncodeFn enc = tok_encode();
    if (!enc || !a.vt) return cudaErrorNotSupported;
    cudaError_t e = launch_vtranspose(a.v, a.vt, a.B * a.Hkv, a.T, 128, st);
    if (e != cudaSuccess) return e;
    const int BHkv = a.B * a.Hkv;
    const int T8 = (a.T + 7) & ~7;
    CUtensorMap mk, mvt, mq;
    {
        cuuint64_t dims[3] = {128, (cuuint64_t)a.T, (cuuint64_t)BHkv};
        cuuint64_t str[2] = {256, (cuuint64_t)a.T * 256};
        cuuint32_t box[3] = {64, 64, 1};
        if (!encode(enc, &mk, a.k, 3, dims, str, box)) return cudaErrorInvalidValue;
    }
    {
        cuuint64_t dims[3] = {(cuuint64_t)T8, 128, (cuuint64_t)BHkv};
        cuuint64_t str[2] = {(cuuint64_t)T8 * 2, (cuuint64_t)T8 * 2 * 128};
        cuuint32_t box[3] = {64, 128, 1};
        if (!encode(enc, &mvt, a.vt, 3, dims, str, box)) return cudaErrorInvalidValue;
    }
    {
        cuuint64_t dims[4] = {128, (cuuint64_t)a.T, (cuuint64_t)a.Hq, (cuuint64_t)a.B};
        cuuint64_t str[3] = {256, (cuuint64_t)a.T * 256, (cuuint64_t)a.Hq * a.T * 256};
        cuuint32_t box[4] = {64, 1, 16, 1};
        if (!encode(enc, &mq, a.q, 4, dims, str, box)) return cudaErrorInvalidValue;
    }
    TokArgs ta;
    ta.s = a;
    ta.n_win = (a.T + kW - 1) / kW;
    size_t off = 0;
    ta.off_q = off;      off += (size_t)2 * kW * 2048;
    ta.off_k = off;      off += (size_t)2 * kKStage;
    ta.off_v = off;      off += kVStage;
    ta.off_p = off;      off += (size_t)kLanes * 2 * 4096;
    ta.off_bias = off;   off += (size_t)kNBias * kBatch * kW * 4;
    ta.off_qbar = off;   off += (size_t)kW * kQbarStride * 4;
    ta.off_mref = off;   off += (size_t)kW * 16 * 4;
    ta.off_mpart = off;  off += (size_t)kW * 2 * 16 * 4;
    ta.off_lpart = off;  off += (size_t)kW * 4 * 16 * 4;
    ta.off_list = off;   off += ((size_t)(a.C + 2) * 2 + 15) & ~(size_t)15;
    const size_t smem = off + 1024;
    e = cudaFuncSetAttribute(k_attend_tok, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const long long grid = (long long)ta.n_win * BHkv;
    if (grid == 0) return cudaSuccess;
    k_attend_tok<<<(unsigned)grid, kThreads, smem, st>>>(mk, mvt, mq, ta);
    return cudaGetLastError();
}

}  // namespace dash
