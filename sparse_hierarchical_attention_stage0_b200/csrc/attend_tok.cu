// attend_tok.cu -- Stage 2 per token on the 5th-generation tensor cores (D = 128, G = 16,
// chunk 64): no query tile ever walks the union of several tokens' routed chunks.
//
// gist.science "DashAttention: Differentiable and Adaptive Sparse Hierarchical Attention",
// Technische Zusammenfassung, "Stufe 2: Prior-induzierte spaerliche Softmax": the kernel
// walks the active chunks of the bit-packed mask, adds the routing bias log p to the logits
// of an active chunk, masks zero-probability chunks, and keeps the diagonal chunk as its own
// (causal, bias 0) branch.
//
// The 16 heads of one token share one routing, so they are the N = 16 columns of the MMAs,
// and keys (QK) or head dims (PV) are the rows:
//   S^T[64 keys x 16] = K_c Q_t^T      A = K_c in tensor memory (M = 64), B = Q_t (smem)
//   O_t^T[128 x 16]  += V_c^T P_t^T    A = V_c^T in tensor memory (M = 128), B = P_t (smem)
// One CTA owns a window of 16 consecutive tokens of one (b, g) (they share the diagonal
// chunk).  It streams the diagonal chunk first, then the union of the window's routed
// chunks; each chunk's K and V^T are staged by TMA and copied into tensor memory once, then
// reused by every window token that routed to it (about 16 x (1 - sparsity) of them).  Four
// independent pipelines ("lanes") own 4 tokens each: one MMA-issuing warp and four softmax
// warps per lane, so per-token MMAs of different lanes overlap.
//
// Softmax reference: the first item of every token is its diagonal chunk, whose exact
// per-head maximum m_h becomes the fixed reference of all later chunks of that token
// (p = 2^(s - m_h)); no running rescale of O is needed.  Logits of routed chunks can exceed
// m_h; fp32 and bf16 hold 2^(s - m_h) exactly up to s - m_h < 127 (log2 units); larger
// excesses are clamped and reported as DASH_ERR_RANGE_CLAMPED through the status word.
// The lane's 4 softmax warps exchange the diagonal maxima and the row sums through an
// mbarrier, so every wait in the kernel is bounded.
//
// Warps: 0 TMA producer, 1 routing-bias producer, 2 TMEM owner / chunk list, 4-7 fill
// (shared memory -> tensor memory), 8-11 MMA issuers (lane L), 12-27 softmax (lane L: warps
// 12+4L .. 15+4L, one per TMEM sub-partition).  Tensor memory: K slots 2x64, V^T slots 2x32,
// S slots 4x16, O 16x16 = 512 columns.  Every wait is bounded and warp-uniform.
#include "kernels.cuh"
#include "tc_common.cuh"

namespace dash {
using namespace tcx;
namespace {

constexpr int kW = 16;
constexpr int kLanes = 4;
constexpr int kTpl = kW / kLanes;                 // tokens per lane
constexpr int kNst = 2;                           // TMA stages
constexpr uint32_t kStage = 32768;                // K panels 2 x 8 KB + V^T 16 KB
constexpr int kBatch = 32;                        // chunk entries per bias batch
constexpr int kNBias = 4;                         // bias ring slots
constexpr int kWarpTma = 0, kWarpBias = 1, kWarpAdmin = 2, kWarpFill0 = 4, kWarpMma0 = 8,
              kWarpSm0 = 12;
constexpr int kThreads = 28 * 32;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColK = 0, kColV = 128, kColS = 192, kColO = 256;
constexpr float kMaxExcess = 126.f;               // log2 units above the reference

struct TokShared {
    uint64_t tma_full[kNst], tma_empty[kNst];
    uint64_t kv_ready[2], kv_free[2];
    uint64_t bias_full[kNBias], bias_empty[kNBias];
    uint64_t s_full[kLanes], p_full[kLanes], o_done[kLanes], x_bar[kLanes];
    uint64_t q_full;
    uint32_t tmem_base;
    int n_ch;
    int failed;
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

}  // namespace

struct TokArgs {
    StageArgs s;
    int n_win;             // windows per (b, g)
    size_t off_q, off_p, off_bias, off_qbar, off_mref, off_mpart, off_lpart, off_list;
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
    unsigned char *qwin = base + ta.off_q;                               // [16 tok][2 panels][16][128B]
    unsigned char *pbuf = base + ta.off_p;                               // [lanes][2 KB]
    float *bias_ring = reinterpret_cast<float *>(base + ta.off_bias);    // [kNBias][kBatch][16]
    float *qbar = reinterpret_cast<float *>(base + ta.off_qbar);         // [16][D]
    float *mref = reinterpret_cast<float *>(base + ta.off_mref);         // [16 tok][4 warps][16]
    float *mpart = reinterpret_cast<float *>(base + ta.off_mpart);       // [16 tok][4 warps][16]
    float *lpart = reinterpret_cast<float *>(base + ta.off_lpart);       // [16 tok][4 warps][16]
    int16_t *list = reinterpret_cast<int16_t *>(base + ta.off_list);

    const int BHkv = a.B * a.Hkv;
    const int wrev = blockIdx.x / BHkv, bgi = blockIdx.x % BHkv;
    const int win = ta.n_win - 1 - wrev;
    const int b = bgi / a.Hkv, g = bgi % a.Hkv;
    const long long bg = bgi;
    const int t0 = win * kW;
    const int cd = t0 / BC;                       // the window's diagonal chunk
    bool failed = false;

    // ------------------------------------------------------------------ setup
    if (warp == kWarpAdmin) tmem_alloc(&sh.tmem_base, kTmemCols);
    if (threadIdx.x == 0) {
        for (int s = 0; s < kNst; ++s) {
            mbar_init(&sh.tma_full[s], 1);
            mbar_init(&sh.tma_empty[s], 4);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&sh.kv_ready[s], 4);
            mbar_init(&sh.kv_free[s], kLanes);
        }
        for (int k = 0; k < kNBias; ++k) {
            mbar_init(&sh.bias_full[k], 1);
            mbar_init(&sh.bias_empty[k], kLanes + 4 * kLanes);
        }
        for (int L = 0; L < kLanes; ++L) {
            mbar_init(&sh.s_full[L], 1);
            mbar_init(&sh.p_full[L], 4);
            mbar_init(&sh.o_done[L], 1);
            mbar_init(&sh.x_bar[L], 4);
        }
        mbar_init(&sh.q_full, 1);
        sh.failed = 0;
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
                        if (t < a.T) word |= a.mask[(bg * a.T + t) * W + w];
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
    if (warp == kWarpBias && !a.ignore_routing) {
        const __nv_bfloat16 *q = reinterpret_cast<const __nv_bfloat16 *>(a.q);
        for (int idx = lane; idx < kW * (D / 8); idx += 32) {
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
            for (int e = 0; e < 8; ++e) qbar[u * D + d8 + e] = m[e];
        }
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tb = sh.tmem_base;
    const int n_ch = sh.n_ch;
    const int n_batches = (n_ch + kBatch - 1) / kBatch;

    if (warp == kWarpTma) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0) {
            mbar_arrive_expect_tx(&sh.q_full, kW * 4096);
            for (int u = 0; u < kW; ++u)
                for (int h = 0; h < 2; ++h)
                    tma_load_4d(qwin + u * 4096 + h * 2048, &tmQ, 64 * h, t0 + u, g * G, b, &sh.q_full);
        }
        __syncwarp();
        int issued = 0;
        for (int j = 0; j < n_ch; ++j) {
            const int st = j % kNst;
            if (!wait_u(&sh.tma_empty[st], ((uint32_t)(j / kNst) & 1u) ^ 1u, a.status, failed)) break;
            issued = j + 1;
            if (lane == 0) {
                const int c = list[j];
                unsigned char *stage = base + (size_t)st * kStage;
                mbar_arrive_expect_tx(&sh.tma_full[st], kStage);
                tma_load_3d(stage, &tmK, 0, c * BC, (int)bg, &sh.tma_full[st]);
                tma_load_3d(stage + 8192, &tmK, 64, c * BC, (int)bg, &sh.tma_full[st]);
                tma_load_3d(stage + 16384, &tmVt, c * BC, 0, (int)bg, &sh.tma_full[st]);
            }
            __syncwarp();
        }
        if (failed) {
            mbar_wait_bounded(&sh.q_full, 0);
            for (int j = max(0, issued - kNst); j < issued; ++j)
                mbar_wait_bounded(&sh.tma_full[j % kNst], (uint32_t)(j / kNst) & 1u);
            __syncwarp();
        }
    } else if (warp == kWarpBias) {
        // ---------------------------------------------------------------- routing biases
        for (int k = 0; k < n_batches; ++k) {
            const int slot = k % kNBias;
            if (!wait_u(&sh.bias_empty[slot], ((uint32_t)(k / kNBias) & 1u) ^ 1u, a.status, failed)) break;
            float *ring = bias_ring + slot * kBatch * kW;
            for (int e = lane; e < kBatch * kW; e += 32) {
                const int jj = e / kW, u = e % kW, j = k * kBatch + jj, t = t0 + u;
                float v = -INFINITY;
                if (j < n_ch && t < a.T) {
                    if (j == 0 || a.ignore_routing) {
                        v = 0.f;
                    } else {
                        const int c = list[j];
                        const long long rowi = bg * a.T + t;
                        if ((a.mask[rowi * a.W + (c >> 6)] >> (c & 63)) & 1ull) {
                            const float dot = route_dot<D>(qbar + u * D, a.summary + (bg * a.Cf + c) * D);
                            const float tau = a.tau[rowi];
                            if (a.rc.kind == 0) {
                                v = a.rc.sigma2 * (__fmul_rn(dot, a.rc.sscale) - tau);
                            } else {
                                const float m = __fsub_rn(__fmul_rn(dot, a.rc.xscale), tau);
                                v = a.rc.bscale2 * log2f(fmaxf(m, 1e-37f));
                            }
                        }
                    }
                }
                ring[e] = v;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh.bias_full[slot]);
        }
    } else if (warp >= kWarpFill0 && warp < kWarpFill0 + 4) {
        // ---------------------------------------------------------------- smem -> TMEM
        const int sp = warp & 3;
        const uint32_t lane_addr = tb + ((uint32_t)(32 * sp) << 16);
        const int key = 16 * sp + (lane & 15);        // M = 64 layout: lanes 0-15 of each quarter
        const int d = 32 * sp + lane;
        for (int j = 0; j < n_ch; ++j) {
            const int st = j % kNst, s = j & 1;
            if (!wait_u(&sh.tma_full[st], (uint32_t)(j / kNst) & 1u, a.status, failed)) break;
            if (!wait_u(&sh.kv_free[s], ((uint32_t)(j / 2) & 1u) ^ 1u, a.status, failed)) break;
            const unsigned char *stage = base + (size_t)st * kStage;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t r[32];
                const unsigned char *row = stage + h * 8192 + key * 128;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint4 v = *reinterpret_cast<const uint4 *>(row + ((c ^ (key & 7)) << 4));
                    r[4 * c] = v.x;
                    r[4 * c + 1] = v.y;
                    r[4 * c + 2] = v.z;
                    r[4 * c + 3] = v.w;
                }
                tmem_st32(lane_addr + kColK + 64u * s + 32u * h, r);
            }
            {
                uint32_t r[32];
                const unsigned char *row = stage + 16384 + d * 128;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint4 v = *reinterpret_cast<const uint4 *>(row + ((c ^ (d & 7)) << 4));
                    r[4 * c] = v.x;
                    r[4 * c + 1] = v.y;
                    r[4 * c + 2] = v.z;
                    r[4 * c + 3] = v.w;
                }
                tmem_st32(lane_addr + kColV + 32u * s, r);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&sh.kv_ready[s]);
                mbar_arrive(&sh.tma_empty[st]);
            }
        }
    } else if (warp >= kWarpMma0 && warp < kWarpMma0 + kLanes) {
        // ---------------------------------------------------------------- MMA issuer, lane L
        const int L = warp - kWarpMma0;
        constexpr uint32_t id_qk = idesc_bf16(64, 16, 0);
        constexpr uint32_t id_pv = idesc_bf16(128, 16, 1);
        const uint32_t d_s = tb + kColS + 16u * L;
        const uint32_t p_addr = smem_u32(pbuf + L * 2048);
        int it = 0;
        wait_u(&sh.q_full, 0, a.status, failed);
        for (int j = 0; j < n_ch && !failed; ++j) {
            const int s = j & 1, k = j / kBatch, slot = k % kNBias;
            if (j % kBatch == 0 && !wait_u(&sh.bias_full[slot], (uint32_t)(k / kNBias) & 1u, a.status, failed)) break;
            if (!wait_u(&sh.kv_ready[s], (uint32_t)(j / 2) & 1u, a.status, failed)) break;
            tc_fence_after();
            const float *ring = bias_ring + slot * kBatch * kW + (j % kBatch) * kW;
            for (int m = 0; m < kTpl; ++m) {
                const int u = L + kLanes * m;
                if (ring[u] == -INFINITY) continue;                 // token did not route here
                if (lane == 0) {
                    const uint32_t qa = smem_u32(qwin + u * 4096);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint64_t bd = smem_desc_sw128(qa + (uint32_t)(kk / 4) * 2048u + (uint32_t)(kk % 4) * 32u, 16, 1024);
                        mma_ts(d_s, tb + kColK + 64u * s + 8u * kk, bd, id_qk, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(&sh.s_full[L]);
                }
                __syncwarp();
                if (!wait_u(&sh.p_full[L], (uint32_t)it & 1u, a.status, failed)) break;
                tc_fence_after();
                if (lane == 0) {
#pragma unroll
                    for (int kk = 0; kk < BC / 16; ++kk) {
                        const uint64_t bd = smem_desc_noswz(p_addr + 256u * kk, 128, 1024);
                        mma_ts(tb + kColO + 16u * u, tb + kColV + 32u * s + 8u * kk, bd, id_pv,
                               (j > 0 || kk > 0) ? 1u : 0u);
                    }
                }
                __syncwarp();
                ++it;
            }
            if (lane == 0) mma_commit(&sh.kv_free[s]);
            __syncwarp();
            if ((j % kBatch == kBatch - 1 || j == n_ch - 1) && lane == 0) mbar_arrive(&sh.bias_empty[slot]);
            __syncwarp();
        }
        if (lane == 0) mma_commit(&sh.o_done[L]);
        __syncwarp();
    } else if (warp >= kWarpSm0 && warp < kWarpSm0 + 4 * kLanes) {
        // ---------------------------------------------------------------- softmax, lane L
        const int L = (warp - kWarpSm0) / 4, sp = warp & 3;
        const bool kl = lane < 16;                       // lanes 0-15 hold keys (M = 64 layout)
        const int key_in = 16 * sp + (lane & 15);
        const uint32_t s_addr = tb + ((uint32_t)(32 * sp) << 16) + kColS + 16u * L;
        unsigned char *pb = pbuf + L * 2048;
        float lsum[kTpl];
#pragma unroll
        for (int m = 0; m < kTpl; ++m) lsum[m] = 0.f;
        int it = 0, xph = 0;
        for (int j = 0; j < n_ch; ++j) {
            const int k = j / kBatch, slot = k % kNBias;
            if (j % kBatch == 0) wait_u(&sh.bias_full[slot], (uint32_t)(k / kNBias) & 1u, a.status, failed);
            const float *ring = bias_ring + slot * kBatch * kW + (j % kBatch) * kW;
            const int c = list[j];
#pragma unroll 1
            for (int m = 0; m < kTpl; ++m) {
                const int u = L + kLanes * m, t = t0 + u;
                const float bias2 = ring[u];
                if (bias2 == -INFINITY) continue;
                const bool ok = wait_u(&sh.s_full[L], (uint32_t)it & 1u, a.status, failed);
                ++it;
                float v[16];
                if (ok) {
                    tc_fence_after();
                    uint32_t sr[16];
                    tmem_ld16(s_addr, sr);
                    tmem_wait_ld();
                    const int kidx = c * BC + key_in;
                    const bool valid = kl && (j > 0 || kidx <= t);
#pragma unroll
                    for (int h = 0; h < 16; ++h)
                        v[h] = valid ? fmaf(__uint_as_float(sr[h]), a.qk_scale2, bias2) : -INFINITY;
                } else {
#pragma unroll
                    for (int h = 0; h < 16; ++h) v[h] = -INFINITY;
                }
                float* mrow = mref + (u * 4 + sp) * 16;
                float mh[16];
                if (j == 0) {
                    // Exact per-head maximum over the diagonal chunk: reduce-scatter over the
                    // 16 key lanes, then across the lane's 4 warps.
                    float w[16];
#pragma unroll
                    for (int h = 0; h < 16; ++h) w[h] = v[h];
#pragma unroll
                    for (int o = 8, n = 8; o >= 1; o >>= 1, n >>= 1) {
                        const bool upper = (lane & o) != 0;
#pragma unroll
                        for (int i = 0; i < n; ++i) {
                            const float send = upper ? w[i] : w[i + n];
                            const float keep = upper ? w[i + n] : w[i];
                            w[i] = fmaxf(keep, __shfl_xor_sync(kFull, send, o));
                        }
                    }
                    if (kl) mpart[(u * 4 + sp) * 16 + lane] = w[0];
                    // Exchange across the lane's 4 warps through an mbarrier (bounded wait).
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sh.x_bar[L]);
                    wait_u(&sh.x_bar[L], (uint32_t)xph & 1u, a.status, failed);
                    ++xph;
#pragma unroll
                    for (int h = 0; h < 16; ++h) {
                        float x = mpart[(u * 4 + 0) * 16 + h];
                        x = fmaxf(x, mpart[(u * 4 + 1) * 16 + h]);
                        x = fmaxf(x, mpart[(u * 4 + 2) * 16 + h]);
                        x = fmaxf(x, mpart[(u * 4 + 3) * 16 + h]);
                        mh[h] = x == -INFINITY ? 0.f : x;
                    }
                    if (kl) mrow[lane] = mh[lane & 15];
                    __syncwarp();
                } else {
#pragma unroll
                    for (int h = 0; h < 16; ++h) mh[h] = mrow[h];
                }
                if (ok) {
                    float p[16];
                    bool clamped = false;
#pragma unroll
                    for (int h = 0; h < 16; ++h) {
                        float e = v[h] - mh[h];
                        if (e > kMaxExcess) { e = kMaxExcess; clamped = true; }
                        p[h] = fast_exp2(e);
                    }
                    if (__any_sync(kFull, clamped) && lane == 0) report(a.status, DASH_ERR_RANGE_CLAMPED);
                    if (kl) {
                        uint4 lo, hi;
                        lo.x = pack_bf16x2(p[0], p[1]);
                        lo.y = pack_bf16x2(p[2], p[3]);
                        lo.z = pack_bf16x2(p[4], p[5]);
                        lo.w = pack_bf16x2(p[6], p[7]);
                        hi.x = pack_bf16x2(p[8], p[9]);
                        hi.y = pack_bf16x2(p[10], p[11]);
                        hi.z = pack_bf16x2(p[12], p[13]);
                        hi.w = pack_bf16x2(p[14], p[15]);
                        const int kq = key_in;
                        *reinterpret_cast<uint4 *>(pb + (kq & 7) * 16 + (kq >> 3) * 128) = lo;
                        *reinterpret_cast<uint4 *>(pb + 1024 + (kq & 7) * 16 + (kq >> 3) * 128) = hi;
                    }
                    fence_proxy_async();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sh.p_full[L]);
                    // Row sums: reduce-scatter the 16 head values over the 16 key lanes.
#pragma unroll
                    for (int o = 8, n = 8; o >= 1; o >>= 1, n >>= 1) {
                        const bool upper = (lane & o) != 0;
#pragma unroll
                        for (int i = 0; i < n; ++i) {
                            const float send = upper ? p[i] : p[i + n];
                            const float keep = upper ? p[i + n] : p[i];
                            p[i] = keep + __shfl_xor_sync(kFull, send, o);
                        }
                    }
                    lsum[m] += kl ? p[0] : 0.f;
                }
            }
            if (j % kBatch == kBatch - 1 || j == n_ch - 1) {
                __syncwarp();
                if (lane == 0) mbar_arrive(&sh.bias_empty[slot]);
            }
        }
        // ------------------------------------------------------------ epilogue
#pragma unroll
        for (int m = 0; m < kTpl; ++m)
            if (kl) lpart[((L + kLanes * m) * 4 + sp) * 16 + lane] = lsum[m];
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
                        const float* lp = lpart + (u * 4) * 16 + h;
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
    return a.D == 128 && a.G == 16 && a.Bc == 64 && a.C <= 8192;
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
    size_t off = (size_t)kNst * kStage;
    ta.off_q = off;      off += (size_t)kW * 4096;
    ta.off_p = off;      off += (size_t)kLanes * 2048;
    ta.off_bias = off;   off += (size_t)kNBias * kBatch * kW * 4;
    ta.off_qbar = off;   off += (size_t)kW * 128 * 4;
    ta.off_mref = off;   off += (size_t)kW * 4 * 16 * 4;
    ta.off_mpart = off;  off += (size_t)kW * 4 * 16 * 4;
    ta.off_lpart = off;  off += (size_t)kW * 4 * 16 * 4;
    ta.off_list = off;   off += (size_t)((a.C + 8) & ~7) * 2;
    const size_t smem = off + 1024;
    e = cudaFuncSetAttribute(k_attend_tok, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const long long grid = (long long)ta.n_win * BHkv;
    if (grid == 0) return cudaSuccess;
    k_attend_tok<<<(unsigned)grid, kThreads, smem, st>>>(mk, mvt, mq, ta);
    return cudaGetLastError();
}

}  // namespace dash
