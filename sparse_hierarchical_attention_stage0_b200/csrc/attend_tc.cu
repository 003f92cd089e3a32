// attend_tc.cu -- Stage 2 on the 5th-generation tensor cores (tcgen05, TMEM, TMA), D = 128.
//
// gist.science "DashAttention: Differentiable and Adaptive Sparse Hierarchical Attention",
// Technische Zusammenfassung, "Stufe 2: Prior-induzierte spaerliche Softmax": a
// FlashAttention-style kernel iterates the active chunks given by the bit-packed mask and
// adds the routing bias (log of the prior) to the logits before the softmax; chunks with
// zero probability are masked; the diagonal chunk keeps its own branch.
//
// One CTA = one tile of 128 query rows of one (b, g): 128/G consecutive tokens x G heads
// (G >= 8); the tile's tokens share one diagonal chunk.  The tile walks the UNION of its
// tokens' active chunks (the OR of their mask words, which carry each token's diagonal bit),
// 64 keys per pipeline block: the diagonal chunk first, then the others in ascending order.
// A row whose token did not route to a chunk gets bias -inf there; keys above the row's
// position are masked.  Per block:
//   S[128 x 64]  = Q K^T      tcgen05.mma kind::f16, A = Q from TMEM, B = K (smem, TMA)
//   softmax      two threads per row (8 warps, 32 keys each), fp32; releases S as soon as
//                it has loaded it, so the next block's Q K^T overlaps these exponentials
//   O[128 x 128] += P V       tcgen05.mma, A = P (bf16, smem, 128B-swizzled, double-buffered),
//                            B = V (smem, TMA)
// Softmax reference: the first block (the diagonal chunk's first 64 keys, which hold at least
// one causally visible key of every row) gives each row its exact maximum m over that block;
// every later probability is 2^(s - m) against that fixed reference, so O is never rescaled
// and the two threads of a row exchange nothing but their partial sums.  A logit more than
// 2^100 above the reference (log2 units) is clamped there (no fp32 overflow for up to 2^17
// keys) and reported as DASH_ERR_RANGE_CLAMPED.
// Warp roles: 0 TMA producer (K and V rings, 128B-swizzled, 2 stages each), 1 MMA issuer and TMEM
// owner, 2 routing-bias producer (recomputes qbar.summary with Stage 1's exact arithmetic,
// 32 chunks per batch, double-buffered), 4-11 softmax + epilogue.  TMEM: Q 64 columns,
// S 64, O 128 = 256 columns, so two CTAs share an SM.  Every wait is bounded; on timeout
// the CTA records DASH_ERR_DEVICE_TIMEOUT and drains.
#include "kernels.cuh"
#include "tc_common.cuh"

namespace dash {
using namespace tcx;
namespace {

constexpr int kTcThreads = 384;
constexpr int kSmThreads = 256;          // softmax warps 4-11
constexpr int kBlk = 64;                 // keys per pipeline block
constexpr int kStages = 2;
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColQ = 0, kColS = 64, kColO = 128;
constexpr int kBiasBatch = 32;
constexpr int kWarpTma = 0, kWarpMma = 1, kWarpBias = 2, kWarpSm0 = 4;
constexpr uint32_t kKBytes = 2 * 8192;      // K block: panels d 0-63, 64-127 (64 keys x 128 B)
constexpr uint32_t kVBytes = 2 * 8192;      // V block, same layout
constexpr uint32_t kPBytes = 128 * 128;     // P block: 128 rows x 64 keys bf16
constexpr uint32_t kOffV = kStages * kKBytes, kOffP = kOffV + kStages * kVBytes,
                   kRingBytes = kOffP + 2 * kPBytes;
constexpr float kMaxExcess = 100.f;         // log2 units above the row reference

struct TcShared {
    uint64_t k_full[kStages], k_empty[kStages], v_full[kStages], v_empty[kStages];
    uint64_t s_full, s_free, p_full[2], o_full;   // p_full per P buffer: at most one phase ahead
    float mpair[2][128];                 // partial row maxima of the first block
    float lpair[2][128];                 // partial row sums
    uint32_t tmem_base;
    int n_chunks;
    int failed;
};

}  // namespace

struct TcArgs {
    StageArgs s;
    int RT;              // tokens per tile (128 / G)
    int n_tiles_bg;      // token tiles per (b, g)
    size_t off_bias, off_qbar, off_list;  // dynamic smem offsets (bytes, from the aligned base)
};

template <int BC>
__global__ void __launch_bounds__(kTcThreads, 2)
k_attend_tc(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
            const TcArgs ta) {
    extern __shared__ unsigned char smem_dyn[];
    __shared__ TcShared sh;
    const StageArgs &a = ta.s;
    constexpr int D = 128;
    constexpr int NSUB = BC / kBlk;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    unsigned char *base = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~(uintptr_t)1023);
    float *bias_s = reinterpret_cast<float *>(base + ta.off_bias);      // [2][kBiasBatch][RT]
    float *qbar = reinterpret_cast<float *>(base + ta.off_qbar);        // [RT][D]
    int16_t *list = reinterpret_cast<int16_t *>(base + ta.off_list);    // [C]

    const int RT = ta.RT, G = a.G;
    const int BHkv = a.B * a.Hkv;
    const int tile_rev = blockIdx.x / BHkv, bgi = blockIdx.x % BHkv;
    const int tt = ta.n_tiles_bg - 1 - tile_rev;
    const int b = bgi / a.Hkv, g = bgi % a.Hkv;
    const long long bg = bgi;
    const int t0 = tt * RT;
    const int t_last = min(t0 + RT, a.T) - 1;
    const int ct_max = t_last / BC;

    // ---------------------------------------------------------------- setup
    if (warp == kWarpMma) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&sh.tmem_base)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sh.k_full[s], 1);
            mbar_init(&sh.k_empty[s], 1);
            mbar_init(&sh.v_full[s], 1);
            mbar_init(&sh.v_empty[s], 1);
        }
        mbar_init(&sh.s_full, 1);
        mbar_init(&sh.s_free, kSmThreads / 32);
        mbar_init(&sh.p_full[0], kSmThreads / 32);
        mbar_init(&sh.p_full[1], kSmThreads / 32);
        mbar_init(&sh.o_full, 1);
        sh.failed = 0;
        fence_mbar_init();
    }
    if (warp == kWarpBias) {
        // Union of the tile's tokens' mask words (each carries its token's diagonal bit).
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
                        if (t < a.T) word |= a.mask[(bg * a.T + t) * W + w];
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
        // Group-mean queries of the tile's tokens (Stage 1's exact arithmetic).
        if (!a.ignore_routing) {
            const __nv_bfloat16 *q = reinterpret_cast<const __nv_bfloat16 *>(a.q);
            for (int idx = lane; idx < RT * (D / 8); idx += 32) {
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
    }
    // Softmax warps: this thread's row, its token and head; Q row into TMEM columns [0, 64)
    // (warps 4-7 the first 64 dims, warps 8-11 the rest).
    const int sp = warp & 3;                     // TMEM sub-partition of this warp
    const int khalf = (warp - kWarpSm0) >> 2;    // softmax warps: which 32 keys of a block
    const int row = 32 * sp + lane;              // valid for the softmax warps
    const int u_row = row / G;                   // token of the row within the tile
    const int t_row = t0 + u_row;
    const int h_row = g * G + row % G;
    const bool row_ok = t_row < a.T;
    __syncthreads();
    const uint32_t tb = sh.tmem_base;
    if (warp >= kWarpSm0) {
        const __nv_bfloat16 *qr = reinterpret_cast<const __nv_bfloat16 *>(a.q) +
                                  (((long long)b * a.Hq + h_row) * a.T + (row_ok ? t_row : 0)) * D;
        uint32_t r[32];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            uint4 v = row_ok ? *reinterpret_cast<const uint4 *>(qr + khalf * 64 + 8 * j)
                             : make_uint4(0, 0, 0, 0);
            r[4 * j] = v.x;
            r[4 * j + 1] = v.y;
            r[4 * j + 2] = v.z;
            r[4 * j + 3] = v.w;
        }
        tmem_st32(tb + ((uint32_t)(32 * sp) << 16) + kColQ + 32 * khalf, r);
        tmem_wait_st();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const int n_chunks = sh.n_chunks;
    const int n_blocks = n_chunks * NSUB;
    bool failed = false;
    // Walk order: the diagonal chunk (the largest, last entry of the ascending list) first.
    auto chunk_at = [&](int ci) -> int { return (int)list[ci == 0 ? n_chunks - 1 : ci - 1]; };

    if (warp == kWarpTma) {
        // ------------------------------------------------------------ TMA producer
        // The whole warp runs the loop (converged); lane 0 issues the copies.  K runs one
        // block ahead of V: the K stage frees when Q K^T completes, the V stage after P V.
        int k_issued = 0, v_issued = 0;
        auto key0_of = [&](int i) { return chunk_at(i / NSUB) * BC + (i % NSUB) * kBlk; };
        auto issue = [&](bool is_v, int i) -> bool {
            const int s = i % kStages;
            const uint32_t ph = (uint32_t)(i / kStages) & 1u;
            uint64_t *empty = is_v ? &sh.v_empty[s] : &sh.k_empty[s];
            uint64_t *full = is_v ? &sh.v_full[s] : &sh.k_full[s];
            if (!wait_or_fail(empty, ph ^ 1u, a.status, failed)) return false;
            if (lane == 0) {
                const CUtensorMap *map = is_v ? &tmV : &tmK;
                unsigned char *st = base + (is_v ? kOffV + (size_t)s * kVBytes : (size_t)s * kKBytes);
                mbar_arrive_expect_tx(full, kKBytes);
                tma_load_3d(st, map, 0, key0_of(i), (int)bg, full);
                tma_load_3d(st + 8192, map, 64, key0_of(i), (int)bg, full);
            }
            __syncwarp();
            if (is_v) v_issued = i + 1; else k_issued = i + 1;
            return true;
        };
        if (n_blocks > 0) issue(false, 0);
        for (int i = 0; i < n_blocks && !failed; ++i) {
            if (i + 1 < n_blocks && !issue(false, i + 1)) break;
            if (!issue(true, i)) break;
        }
        if (failed) {
            // Bounded wait for the copies still in flight (the last ones per ring).
            for (int j = max(0, k_issued - kStages); j < k_issued; ++j)
                mbar_wait_bounded(&sh.k_full[j % kStages], (uint32_t)(j / kStages) & 1u);
            for (int j = max(0, v_issued - kStages); j < v_issued; ++j)
                mbar_wait_bounded(&sh.v_full[j % kStages], (uint32_t)(j / kStages) & 1u);
            __syncwarp();
        }
    } else if (warp == kWarpMma) {
        // ------------------------------------------------------------ MMA issuer
        // The whole warp runs the loop (converged); lane 0 issues the MMAs and commits.  Block
        // i's Q K^T is issued as soon as the softmax has loaded S(i-1); P(i-1) V follows once
        // the softmax has written P(i-1).
        constexpr uint32_t id_qk = idesc_bf16(128, kBlk, 0);
        constexpr uint32_t id_pv = idesc_bf16(128, D, 1);
        for (int i = 0; i <= n_blocks; ++i) {
            if (i < n_blocks) {
                const int s = i % kStages;
                if (!wait_or_fail(&sh.k_full[s], (uint32_t)(i / kStages) & 1u, a.status, failed)) break;
                if (i > 0 && !wait_or_fail(&sh.s_free, (uint32_t)(i - 1) & 1u, a.status, failed)) break;
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t kst = smem_u32(base + (size_t)s * kKBytes);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint64_t bd = smem_desc_sw128(kst + (uint32_t)(kk / 4) * 8192u +
                                                                (uint32_t)(kk % 4) * 32u,
                                                            16, 1024);
                        mma_ts(tb + kColS, tb + kColQ + 8u * kk, bd, id_qk, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(&sh.s_full);
                    mma_commit(&sh.k_empty[s]);
                }
                __syncwarp();
            }
            if (i > 0) {
                const int j = i - 1, s = j % kStages;
                if (!wait_or_fail(&sh.v_full[s], (uint32_t)(j / kStages) & 1u, a.status, failed)) break;
                if (!wait_or_fail(&sh.p_full[j & 1], (uint32_t)(j >> 1) & 1u, a.status, failed)) break;
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t vst = smem_u32(base + kOffV + (size_t)s * kVBytes);
                    const uint32_t pst = smem_u32(base + kOffP + (size_t)(j & 1) * kPBytes);
#pragma unroll
                    for (int kk = 0; kk < kBlk / 16; ++kk) {
                        const uint64_t ad = smem_desc_sw128(pst + (uint32_t)kk * 32u, 16, 1024);
                        const uint64_t bd = smem_desc_sw128(vst + (uint32_t)kk * 2048u, 8192, 1024);
                        mma_ss(tb + kColO, ad, bd, id_pv, (j > 0 || kk > 0) ? 1u : 0u);
                    }
                    mma_commit(&sh.v_empty[s]);
                }
                __syncwarp();
            }
        }
        if (lane == 0) mma_commit(&sh.o_full);          // tracks every MMA issued above
        __syncwarp();
    } else if (warp == kWarpBias) {
        // ------------------------------------------------------------ routing biases
        const int n_batches = (n_chunks + kBiasBatch - 1) / kBiasBatch;
        for (int bt = 0; bt < n_batches; ++bt) {
            float *buf = bias_s + (bt & 1) * kBiasBatch * RT;
            for (int e = lane; e < kBiasBatch * RT; e += 32) {
                const int k = e / RT, u = e % RT, ci = bt * kBiasBatch + k;
                float v = 0.f;
                if (ci < n_chunks && !a.ignore_routing) {
                    const int c = chunk_at(ci), t = t0 + u;
                    const int ctu = t / BC;
                    if (t >= a.T || c > ctu) {
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
    } else if (warp >= kWarpSm0) {
        // ------------------------------------------------------------ softmax
        // Two threads per row: warps 4-7 take keys [0, 32) of every block, warps 8-11 keys
        // [32, 64).  Every named barrier below is passed by all softmax warps, failure or not.
        const uint32_t lane_base = tb + ((uint32_t)(32 * sp) << 16);
        const int ct_row = t_row / BC;
        float m_ref = 0.f, l_sum = 0.f, emax_all = -INFINITY;
        for (int i = 0; i < n_blocks; ++i) {
            const int ci = i / NSUB;
            if (ci % kBiasBatch == 0 && i % NSUB == 0) named_sync(1, 32 + kSmThreads);
            const bool ok = wait_or_fail(&sh.s_full, (uint32_t)i & 1u, a.status, failed);
            if (ok) tc_fence_after();
            const int c = chunk_at(ci);
            const int key0 = c * BC + (i % NSUB) * kBlk + 32 * khalf;
            float bias2;
            bool diag = false;
            if (!row_ok || c > ct_row) {
                bias2 = -INFINITY;
            } else if (c == ct_row) {
                bias2 = 0.f;
                diag = true;
            } else {
                bias2 = a.ignore_routing ? 0.f
                                         : bias_s[((ci / kBiasBatch) & 1) * kBiasBatch * RT +
                                                  (ci % kBiasBatch) * RT + u_row];
            }
            // The diagonal chunk is the tile's last one (every token of the tile shares it).
            const bool dead = __all_sync(kFull, bias2 == -INFINITY);
            uint32_t sv[32];
            if (ok && (i == 0 || !dead)) {
                tmem_ld32(lane_base + kColS + 32 * khalf, sv);
                tmem_wait_ld();
            }
            // S is in registers: the next block's Q K^T may overwrite it.
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh.s_free);
            if (i == 0) {
                // First block: exact row maximum over the diagonal chunk's first 64 keys, the
                // fixed reference of every later block.
                float mx = -INFINITY;
                if (ok) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const float v = (row_ok && key0 + j <= t_row)
                                            ? __uint_as_float(sv[j]) * a.qk_scale2 : -INFINITY;
                        mx = fmaxf(mx, v);
                    }
                }
                sh.mpair[khalf][row] = mx;
                named_sync(2, kSmThreads);
                const float m2 = fmaxf(sh.mpair[0][row], sh.mpair[1][row]);
                m_ref = m2 == -INFINITY ? 0.f : m2;
            }
            if (!ok) continue;
            const float c2 = bias2 - m_ref;              // -inf for rows that do not attend
            uint32_t pw[16];
            if (dead) {
                // None of the warp's 32 rows attends this chunk: P = 0, no exponentials.
#pragma unroll
                for (int j = 0; j < 16; ++j) pw[j] = 0u;
            } else {
                float psum = 0.f, emax = -INFINITY;
                if (c == ct_max) {
                    const int lim = t_row - key0;            // keys j > lim are in the future
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const float e0 = 2 * j <= lim ? fmaf(__uint_as_float(sv[2 * j]), a.qk_scale2, c2) : -INFINITY;
                        const float e1 = 2 * j + 1 <= lim ? fmaf(__uint_as_float(sv[2 * j + 1]), a.qk_scale2, c2) : -INFINITY;
                        emax = fmaxf(emax, fmaxf(e0, e1));
                        const uint32_t pk = pack_bf16x2(fast_exp2(fminf(e0, kMaxExcess)),
                                                        fast_exp2(fminf(e1, kMaxExcess)));
                        // l sums the bf16 weights the PV MMA multiplies, so O / l is normalised
                        // exactly even when one key dominates the row.
                        psum += __uint_as_float(pk << 16) + __uint_as_float(pk & 0xffff0000u);
                        pw[j] = pk;
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const float e0 = fmaf(__uint_as_float(sv[2 * j]), a.qk_scale2, c2);
                        const float e1 = fmaf(__uint_as_float(sv[2 * j + 1]), a.qk_scale2, c2);
                        emax = fmaxf(emax, fmaxf(e0, e1));
                        const uint32_t pk = pack_bf16x2(fast_exp2(fminf(e0, kMaxExcess)),
                                                        fast_exp2(fminf(e1, kMaxExcess)));
                        psum += __uint_as_float(pk << 16) + __uint_as_float(pk & 0xffff0000u);
                        pw[j] = pk;
                    }
                }
                l_sum += psum;
                emax_all = fmaxf(emax_all, emax);
            }
            // P row (this thread's 32 keys = 4 16-byte chunks) into the 128B-swizzled K-major
            // P buffer of this block: row r at (r/8)*1024 + (r%8)*128, chunk c at (c ^ r%8)*16.
            {
                unsigned char *prow = base + kOffP + (size_t)(i & 1) * kPBytes + (row >> 3) * 1024 + (row & 7) * 128;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int cch = 4 * khalf + k;
                    *reinterpret_cast<uint4 *>(prow + ((cch ^ (row & 7)) << 4)) =
                        make_uint4(pw[4 * k], pw[4 * k + 1], pw[4 * k + 2], pw[4 * k + 3]);
                }
            }
            fence_proxy_async();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh.p_full[i & 1]);
        }
        if (__any_sync(kFull, emax_all > kMaxExcess) && lane == 0) report(a.status, DASH_ERR_RANGE_CLAMPED);
        // Epilogue: l = sum of the two partial sums, O / l -> bf16 (each warp 64 of the dims).
        sh.lpair[khalf][row] = l_sum;
        const bool ok_o = wait_or_fail(&sh.o_full, 0, a.status, failed);
        named_sync(2, kSmThreads);
        if (ok_o) {
            tc_fence_after();
            const float l = sh.lpair[0][row] + sh.lpair[1][row];
            const float inv = l > 0.f ? 1.f / l : 0.f;
            __nv_bfloat16 *orow = reinterpret_cast<__nv_bfloat16 *>(a.out) +
                                  (((long long)b * a.Hq + h_row) * a.T + (row_ok ? t_row : 0)) * D;
#pragma unroll 1
            for (int q2 = 0; q2 < 2; ++q2) {
                const int q4 = 2 * khalf + q2;
                uint32_t o[32];
                tmem_ld32(lane_base + kColO + 32 * q4, o);
                tmem_wait_ld();
                if (row_ok) {
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        uint4 v;
                        v.x = pack_bf16x2(__uint_as_float(o[8 * j]) * inv, __uint_as_float(o[8 * j + 1]) * inv);
                        v.y = pack_bf16x2(__uint_as_float(o[8 * j + 2]) * inv, __uint_as_float(o[8 * j + 3]) * inv);
                        v.z = pack_bf16x2(__uint_as_float(o[8 * j + 4]) * inv, __uint_as_float(o[8 * j + 5]) * inv);
                        v.w = pack_bf16x2(__uint_as_float(o[8 * j + 6]) * inv, __uint_as_float(o[8 * j + 7]) * inv);
                        *reinterpret_cast<uint4 *>(orow + 32 * q4 + 8 * j) = v;
                    }
                }
            }
        }
    }

    // ---------------------------------------------------------------- teardown
    if (failed) sh.failed = 1;
    tc_fence_before();
    __syncthreads();
    if (sh.failed && warp == kWarpMma && lane == 0) {
        // Give every MMA in flight a bounded chance to finish before TMEM is released.
        mma_commit(&sh.o_full);
        mbar_wait_bounded(&sh.o_full, 1);
    }
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

EncodeFn get_encode() {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
        return nullptr;
    return reinterpret_cast<EncodeFn>(fn);
}

// 3-D map over a [B*Hkv][T][128] bf16 plane set: box (64 d, 64 keys, 1), 128B swizzle,
// zero fill out of bounds (keys >= T of the last chunk).
bool make_map(EncodeFn enc, CUtensorMap *m, const void *ptr, int T, int BHkv) {
    cuuint64_t dims[3] = {128, (cuuint64_t)T, (cuuint64_t)BHkv};
    cuuint64_t strides[2] = {128 * 2, (cuuint64_t)T * 128 * 2};
    cuuint32_t box[3] = {64, 64, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool attend_tc_supported(const StageArgs &a) {
    return a.D == 128 && a.G >= 8 && a.G <= 128 && 128 % a.G == 0 && a.C <= 16384 &&
           (a.Bc == 64 || a.Bc == 128);
}

template <int BC>
static cudaError_t launch_tc_t(const StageArgs &a, cudaStream_t st) {
    static EncodeFn enc = get_encode();
    if (!enc) return cudaErrorNotSupported;
    CUtensorMap mk, mv;
    const int BHkv = a.B * a.Hkv;
    if (!make_map(enc, &mk, a.k, a.T, BHkv) || !make_map(enc, &mv, a.v, a.T, BHkv))
        return cudaErrorInvalidValue;
    TcArgs ta;
    ta.s = a;
    ta.RT = 128 / a.G;
    ta.n_tiles_bg = (a.T + ta.RT - 1) / ta.RT;
    size_t off = kRingBytes;
    ta.off_bias = off;
    off += (size_t)2 * kBiasBatch * ta.RT * 4;
    ta.off_qbar = off;
    off += (size_t)ta.RT * 128 * 4;
    ta.off_list = off;
    off += (size_t)((a.C + 7) & ~7) * 2;
    const size_t smem = off + 1024;              // room to align the base to 1024 bytes
    auto kern = k_attend_tc<BC>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const long long grid = (long long)ta.n_tiles_bg * BHkv;
    if (grid == 0) return cudaSuccess;
    kern<<<(unsigned)grid, kTcThreads, smem, st>>>(mk, mv, ta);
    return cudaGetLastError();
}

cudaError_t launch_attend_tc(const StageArgs &a, cudaStream_t st) {
    if (a.Bc == 64) return launch_tc_t<64>(a, st);
    if (a.Bc == 128) return launch_tc_t<128>(a, st);
    return cudaErrorInvalidValue;
}

}  // namespace dash
