// attend_pair.cu -- Stage 2 on pairs of SMs (tcgen05 cta_group::2), 128-key blocks, D = 128.
//
// gist.science "DashAttention: Differentiable and Adaptive Sparse Hierarchical Attention",
// Technische Zusammenfassung, "Stufe 2: Prior-induzierte spaerliche Softmax": a
// FlashAttention-style kernel iterates the active chunks given by the bit-packed mask and
// adds the routing bias (log of the prior) to the logits before the softmax; chunks with
// zero probability are masked; the diagonal chunk keeps its own branch.
//
// A thread-block cluster of two CTAs on two SMs takes two consecutive tiles of 128 query rows
// of one (b, g) (2 x 128/G tokens x G heads, all in one diagonal chunk) and walks the union of
// the pair's tokens' active chunks: the diagonal chunk first, then the others ascending, two
// 64-key chunks (or one 128-key chunk) per 128-key block.  Per block j, issued by one thread
// of the even CTA for both:
//   S_j[256 x 128] = Q K^T   tcgen05.mma.cta_group::2, M = 256 (each CTA's 128 rows of Q in
//                            its own TMEM), B = K: each CTA holds one 64-key half of the block
//   softmax                  in each CTA on its own rows (four threads per row, 16 warps)
//   O[256 x 144]  += P V     A = P (TMEM), B = V^T: each CTA holds 72 of its 144 rows (the
//                            even CTA dims 0-71, the odd CTA dims 72-127 and 16 rows of ones,
//                            which give the row sums of P in O column 128)
// The pair thus moves each K/V byte from L2 once for 256 rows: per SM 32 KB per block instead
// of 64 KB.  Measured on B200, the single-SM version of this loop waited on its K/V copies
// (L2 to shared memory at about 35 bytes per cycle per SM) for a third of its time.
// Softmax reference, row sums, biases and masking are those of attend_fa.cu: the first block
// holds the diagonal chunk, whose causally visible keys give each row its exact maximum m;
// every probability is 2^(s - m) against that fixed reference, so O is never rescaled.
//
// Synchronisation across the pair: each CTA's K and V^T copies complete on its own full
// barriers; the odd CTA forwards every completed phase to a peer barrier of the even CTA,
// whose issuers wait for both before an MMA reads the stage; MMA completion is committed to both
// CTAs' barriers (multicast), so each CTA's producers refill their own stages and each CTA's
// softmax sees its S; the odd CTA's softmax warps gather on a local barrier whose phases a
// forwarder warp passes to the even CTA's P barrier through the cluster's shared-memory window.  Every wait is bounded; on timeout a CTA records
// DASH_ERR_DEVICE_TIMEOUT, drains, and both CTAs meet at the final cluster barrier.
#include "kernels.cuh"
#include "tc_common.cuh"

namespace dash {
using namespace tcx;
namespace {

constexpr int kSmWarps = 16;
constexpr int kSmThreads = kSmWarps * 32;
constexpr int kPrThreads = 4 * 32 + kSmThreads + 32;       // 21 warps
constexpr int kStages = 5;
constexpr int kTmemCols = 512;
constexpr uint32_t kColQ = 0, kColS = 64, kColO = 320;     // Q 64 | S0 128 | S1 128 | O 144
constexpr int kBiasBatch = 32;
constexpr int kWarpTma = 0, kWarpQk = 1, kWarpBias = 2, kWarpPv = 3, kWarpSm0 = 4,
              kWarpTmaV = kWarpSm0 + kSmWarps;
constexpr int kNv = 144;                 // P V columns: 128 dims + 16 ones rows
constexpr int kVRows = kNv / 2;          // V^T rows held per CTA
constexpr int kVRowsOdd = 128 - kVRows;  // dims 72-127 in the odd CTA; rows 56-71 are ones
constexpr int kKStage = 16384;           // one 64-key half of K: two 8 KB d-panels
constexpr int kVPanel = kVRows * 128;    // one 64-key panel of this CTA's V^T rows (9 KB)
constexpr int kVStage = 2 * kVPanel;
constexpr int kOffV = kStages * kKStage;
constexpr int kRingBytes = kOffV + kStages * kVStage;
static_assert(kVPanel % 1024 == 0, "128B-swizzled panels start on 1 KB boundaries");
constexpr uint16_t kBoth = 3, kEven = 1;  // multicast masks of the CTA pair

struct PrShared {
    uint64_t k_full[kStages], k_empty[kStages], v_full[kStages], v_empty[kStages];
    uint64_t k_peer[kStages], v_peer[kStages];  // even CTA: the odd CTA's copies have landed
    uint64_t s_full[2], p_full[2], pv_done[2];  // per S buffer: never more than one phase ahead
    uint64_t p_part[2];                         // odd CTA: its softmax warps have written P
    uint64_t o_full, qk_done;
    float mpart[4][128];                   // partial row maxima of the first block
    uint32_t tmem_base;
    int n_chunks;
    int failed;
};

// ---------------------------------------------------------------- cluster and pair PTX
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n"
                 "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Address, in the cluster's shared-memory window, of this CTA's variable `p` in CTA `rank`.
__device__ __forceinline__ uint32_t cluster_addr(const void *p, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
    return r;
}
// Arrival on an mbarrier of the other CTA.  Relaxed: every forwarded event (copies landed,
// TMEM stores waited for) is already complete when the arrival is issued, and a cluster-scope
// release costs about 1,200 cycles here (measured on B200), on the path of every block.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t addr) {
    asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(addr) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_cl(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ bool mbar_wait_bounded_cl(uint64_t *bar, uint32_t parity) {
    if (mbar_try_wait_cl(bar, parity)) return true;
    const unsigned long long t0 = global_ns();
    while (true) {
        if (mbar_try_wait_cl(bar, parity)) return true;
        if (global_ns() - t0 > kWaitLimitNs) return false;
    }
}
// Bounded wait by a whole warp with a warp-uniform outcome (cluster-scope acquire).
__device__ __forceinline__ bool wait_or_fail_cl(uint64_t *bar, uint32_t parity, uint32_t *status,
                                                bool &failed) {
    if (failed) return false;
    const bool ok = __all_sync(kFull, mbar_wait_bounded_cl(bar, parity));
    if (!ok) {
        if ((threadIdx.x & 31) == 0) report(status, DASH_ERR_DEVICE_TIMEOUT);
        failed = true;
    }
    return ok;
}
// D (TMEM of both CTAs) (+)= A (TMEM of both CTAs) * B (shared memory of both CTAs), M = 256.
__device__ __forceinline__ void mma2_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                        uint32_t idesc, uint32_t accumulate) {
    asm volatile("{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
                 " tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
                 "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate));
}
// Arrive on `bar` (same offset) in every CTA of `mask` once the pair MMAs issued so far by
// this thread have completed.
__device__ __forceinline__ void mma2_commit(uint64_t *bar, uint16_t mask) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
        " [%0], %1;" ::"r"(smem_u32(bar)),
        "h"(mask)
        : "memory");
}
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

struct PrArgs {
    StageArgs s;
    int RT;              // tokens per tile (128 / G)
    int pair0, n_pairs_bg;  // first tile pair and tile pairs per (b, g) of the row range
    size_t off_bias, off_qbar, off_list;  // dynamic smem offsets (bytes, from the aligned base)
};

template <int BC>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPrThreads, 1)
k_attend_pair(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmVtE,
              const __grid_constant__ CUtensorMap tmVtO, const PrArgs ta) {
    extern __shared__ unsigned char smem_dyn[];
    __shared__ PrShared sh;
    const StageArgs &a = ta.s;
    constexpr int D = 128;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // Both CTAs use the same offsets: the pair MMAs address the odd CTA's operands through
    // the even CTA's descriptors.
    unsigned char *base = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~(uintptr_t)1023);
    float *bias_s = reinterpret_cast<float *>(base + ta.off_bias);      // [2][kBiasBatch][RT]
    float *qbar = reinterpret_cast<float *>(base + ta.off_qbar);        // [RT][D]
    int16_t *list = reinterpret_cast<int16_t *>(base + ta.off_list);    // [C]

    const uint32_t rank = cluster_rank();
    const bool even = rank == 0;
    const int RT = ta.RT, G = a.G;
    const int pair = blockIdx.x >> 1;
    // (b, g)-major, longest pairs first: the CTAs in flight share one (b, g)'s K and V^T in L2.
    const int pair_rev = pair % ta.n_pairs_bg, bgi = pair / ta.n_pairs_bg;
    const int pp = ta.pair0 + ta.n_pairs_bg - 1 - pair_rev;
    const int b = bgi / a.Hkv, g = bgi % a.Hkv;
    const long long bg = bgi;
    const int tp0 = pp * 2 * RT;                                        // the pair's first token
    const int t0 = tp0 + (int)rank * RT;                                // this CTA's first token
    const int t_last = min(tp0 + 2 * RT, a.t_end) - 1;
    const int ct_max = t_last / BC;                                     // the pair's diagonal chunk

    // ---------------------------------------------------------------- setup
    if (warp == kWarpQk) {
        // The same 512 columns in both CTAs of the pair.
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&sh.tmem_base)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
    }
    if (threadIdx.x == 0) {
        // Full barriers track this CTA's own copies; the even CTA's peer barriers take the odd
        // CTA's forwarded arrivals.  The even CTA's P barrier takes its own softmax warps and
        // one forwarded arrival for the odd CTA's, which gather on the odd CTA's p_part.
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sh.k_full[s], 1);
            mbar_init(&sh.k_empty[s], 1);
            mbar_init(&sh.v_full[s], 1);
            mbar_init(&sh.v_empty[s], 1);
            mbar_init(&sh.k_peer[s], 1);
            mbar_init(&sh.v_peer[s], 1);
        }
        for (int bb = 0; bb < 2; ++bb) {
            mbar_init(&sh.s_full[bb], 1);
            mbar_init(&sh.p_full[bb], kSmWarps + 1);
            mbar_init(&sh.p_part[bb], kSmWarps);
            mbar_init(&sh.pv_done[bb], 1);
        }
        mbar_init(&sh.o_full, 1);
        mbar_init(&sh.qk_done, 1);
        sh.failed = 0;
        fence_mbar_init();
    }
    if (warp == kWarpBias) {
        // Union of the pair's tokens' mask words (each carries its token's diagonal bit): both
        // CTAs build the same list.
        const int W = a.W, wlim = ct_max / 64;
        int pos = 0;
        for (int w0 = 0; w0 <= wlim; w0 += 32) {
            const int w = w0 + lane;
            uint64_t word = 0;
            if (w <= wlim) {
                if (a.ignore_routing) {
                    word = ~0ull;
                } else {
                    for (int u = 0; u < 2 * RT; ++u) {
                        const int t = tp0 + u;
                        if (t < a.t_end) word |= a.mask[(bg * a.T + t) * W + w];
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
        // Group-mean queries of this CTA's tokens (Stage 1's exact arithmetic).
        if (!a.ignore_routing) {
            const __nv_bfloat16 *q = reinterpret_cast<const __nv_bfloat16 *>(a.q);
            for (int idx = lane; idx < RT * (D / 8); idx += 32) {
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
                for (int e = 0; e < 8; ++e) qbar[u * D + d8 + e] = m[e];
            }
        }
    }
    if (warp == kWarpTma && !even) {
        // Odd CTA: rows 56-71 of every V^T panel are ones (bf16 1.0 = 0x3f80), so P V also
        // yields the row sums of P in O columns 128-143.  TMA never writes these rows.
        const uint4 ones = make_uint4(0x3f803f80u, 0x3f803f80u, 0x3f803f80u, 0x3f803f80u);
        constexpr int kOnes = kVRows - kVRowsOdd;
        for (int i = lane; i < kStages * 2 * kOnes * 8; i += 32) {
            const int panel = i / (kOnes * 8), r = (i / 8) % kOnes, c = i % 8;
            *reinterpret_cast<uint4 *>(base + kOffV + (size_t)panel * kVPanel + (kVRowsOdd + r) * 128 + c * 16) = ones;
        }
        fence_proxy_async();
    }
    // Softmax warps: quadrant sp (TMEM lanes 32 sp ..), key quarter kq of every block.
    const int sp = warp & 3;
    const int kq = (warp - kWarpSm0) >> 2;
    const int row = 32 * sp + lane;
    const int u_row = row / G;
    const int t_row = t0 + u_row;
    const int h_row = g * G + row % G;
    const bool row_ok = t_row < a.t_end;
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
    tc_fence_before();
    __syncthreads();
    // Barrier initialisation, TMEM allocation and Q of both CTAs before any cross-CTA use.
    cluster_sync_all();
    tc_fence_after();

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
        // ------------------------------------------------------------ TMA producers
        // Warp 0 streams this CTA's half of K, warp 20 its rows of V^T, each into a kStages
        // ring.  K: the even CTA loads key-half 0 of every block, the odd CTA key-half 1 (not
        // loaded when the block has a single 64-key chunk), each as two [64 keys][64 dims]
        // panels.  V^T: both key-halves of this CTA's rows (dims 0-71 in the even CTA, dims
        // 72-127 in the odd CTA), one [rows][64 keys] box per key-half.  The copies complete on
        // this CTA's full barrier; the odd CTA forwards each completed phase to the even CTA's
        // peer barrier.
        const bool is_v = warp == kWarpTmaV;
        int issued = 0;
        for (int j = 0; j < n_blocks && !failed; ++j) {
            const int s = j % kStages;
            const uint32_t ph = (uint32_t)(j / kStages) & 1u;
            uint64_t *empty = is_v ? &sh.v_empty[s] : &sh.k_empty[s];
            uint64_t *full = is_v ? &sh.v_full[s] : &sh.k_full[s];
            if (!wait_or_fail_cl(empty, ph ^ 1u, a.status, failed)) break;
            if (lane == 0) {
                const int nh = entry_of(j, 1) >= 0 ? 2 : 1;
                if (is_v) {
                    unsigned char *st = base + kOffV + (size_t)s * kVStage;
                    const uint32_t rows = even ? kVRows : kVRowsOdd;
                    mbar_arrive_expect_tx(full, rows * 128u * nh);
                    for (int h = 0; h < nh; ++h)
                        tma_load_3d(st + kVPanel * h, even ? &tmVtE : &tmVtO, key0_of(j, h),
                                    even ? 0 : kVRows, (int)bg, full);
                } else {
                    const bool mine = even || nh == 2;
                    mbar_arrive_expect_tx(full, mine ? 16384u : 0u);
                    if (mine) {
                        unsigned char *st = base + (size_t)s * kKStage;
                        const int key0 = key0_of(j, (int)rank);
                        tma_load_3d(st, &tmK, 0, key0, (int)bg, full);
                        tma_load_3d(st + 8192, &tmK, 64, key0, (int)bg, full);
                    }
                }
            }
            __syncwarp();
            issued = j + 1;
        }
        if (failed) {
            // Bounded wait for this CTA's copies still in flight (the last ones per stage).
            for (int i = max(0, issued - kStages); i < issued; ++i)
                mbar_wait_bounded_cl(is_v ? &sh.v_full[i % kStages] : &sh.k_full[i % kStages],
                                     (uint32_t)(i / kStages) & 1u);
            __syncwarp();
        }
    } else if (!even && (warp == kWarpQk || warp == kWarpPv)) {
        // ------------------------------------------------------------ odd CTA: forwarders
        // Each completed phase of this CTA's K (warp 1) or V^T (warp 3) full barrier becomes
        // one arrival on the even CTA's peer barrier of that stage.  It runs at most one phase
        // ahead: the next copy into a stage waits for the MMA that consumed it.  Warp 3 also
        // forwards each block's P (all 16 softmax warps done) to the even CTA's P barrier: one
        // cluster-scope release per block instead of one per softmax warp.  P of block j is
        // forwarded before the V^T of block j + 1, which P V of block j + 1 needs no earlier.
        const bool is_v = warp == kWarpPv;
        for (int j = 0; j < n_blocks; ++j) {
            const int s = j % kStages;
            uint64_t *full = is_v ? &sh.v_full[s] : &sh.k_full[s];
            if (!wait_or_fail_cl(full, (uint32_t)(j / kStages) & 1u, a.status, failed)) break;
            if (lane == 0) mbar_arrive_cluster(cluster_addr(is_v ? &sh.v_peer[s] : &sh.k_peer[s], 0));
            __syncwarp();
            if (is_v) {
                if (!wait_or_fail_cl(&sh.p_part[j & 1], (uint32_t)(j >> 1) & 1u, a.status, failed)) break;
                tc_fence_after();
                tc_fence_before();
                if (lane == 0) mbar_arrive_cluster(cluster_addr(&sh.p_full[j & 1], 0));
                __syncwarp();
            }
        }
    } else if (warp == kWarpQk) {
        // ------------------------------------------------------------ Q K^T issuer (even CTA)
        // S buffer j & 1 is free once P V of block j-2 (which read P from it) has completed.
        constexpr uint32_t id_qk = idesc_bf16(256, 128, 0);
        uint64_t kdesc[kStages];
#pragma unroll
        for (int s = 0; s < kStages; ++s) kdesc[s] = smem_desc_sw128(smem_u32(base + (size_t)s * kKStage), 16, 1024);
        for (int j = 0; j < n_blocks; ++j) {
            const int s = j % kStages, sb = j & 1;
            if (!wait_or_fail_cl(&sh.k_full[s], (uint32_t)(j / kStages) & 1u, a.status, failed)) break;
            if (!wait_or_fail_cl(&sh.k_peer[s], (uint32_t)(j / kStages) & 1u, a.status, failed)) break;
            if (j >= 2 && !wait_or_fail_cl(&sh.pv_done[sb], (uint32_t)((j - 2) >> 1) & 1u, a.status, failed)) break;
            tc_fence_after();
            if (lane == 0) {
                uint64_t bd0 = 0;
#pragma unroll
                for (int q = 0; q < kStages; ++q) bd0 = q == s ? kdesc[q] : bd0;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    // descriptor start address advances in 16-byte units: d-panel kk/4, 32 B per 16 dims
                    const uint64_t bd = bd0 + (uint64_t)(((kk / 4) * 8192 + (kk % 4) * 32) >> 4);
                    mma2_ts(tb + kColS + 128u * sb, tb + kColQ + 8u * kk, bd, id_qk, kk > 0 ? 1u : 0u);
                }
                mma2_commit(&sh.s_full[sb], kBoth);
                mma2_commit(&sh.k_empty[s], kBoth);
            }
            __syncwarp();
        }
        if (lane == 0) mma2_commit(&sh.qk_done, kBoth);   // tracks every MMA issued above
        __syncwarp();
    } else if (warp == kWarpPv) {
        // ------------------------------------------------------------ P V issuer (even CTA)
        // P of keys 32q .. 32q+31 sits in the first 16 columns of S quarter q; B = V^T, K-major.
        constexpr uint32_t id_pv = idesc_bf16(256, kNv, 0);
        uint64_t vdesc[kStages];
#pragma unroll
        for (int s = 0; s < kStages; ++s) vdesc[s] = smem_desc_sw128(smem_u32(base + kOffV + (size_t)s * kVStage), 16, 1024);
        for (int j = 0; j < n_blocks; ++j) {
            const int s = j % kStages, sb = j & 1;
            if (!wait_or_fail_cl(&sh.v_full[s], (uint32_t)(j / kStages) & 1u, a.status, failed)) break;
            if (!wait_or_fail_cl(&sh.v_peer[s], (uint32_t)(j / kStages) & 1u, a.status, failed)) break;
            if (!wait_or_fail_cl(&sh.p_full[sb], (uint32_t)(j >> 1) & 1u, a.status, failed)) break;
            tc_fence_after();
            if (lane == 0) {
                const uint32_t pb = tb + kColS + 128u * sb;
                const bool full_blk = entry_of(j, 1) >= 0;
                uint64_t bd0 = 0;
#pragma unroll
                for (int q = 0; q < kStages; ++q) bd0 = q == s ? vdesc[q] : bd0;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    if (kk >= 4 && !full_blk) break;
                    // key-panel kk/4 of this CTA's V^T rows, 32 B per 16 keys
                    const uint64_t bd = bd0 + (uint64_t)(((kk / 4) * kVPanel + (kk % 4) * 32) >> 4);
                    mma2_ts(tb + kColO, pb + 32u * (kk / 2) + 8u * (kk % 2), bd, id_pv,
                            (j > 0 || kk > 0) ? 1u : 0u);
                }
                mma2_commit(&sh.pv_done[sb], kEven);
                mma2_commit(&sh.v_empty[s], kBoth);
            }
            __syncwarp();
        }
        if (lane == 0) mma2_commit(&sh.o_full, kBoth);    // tracks every MMA issued above
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
            if (e0 % kBiasBatch == 0) named_sync(1, 32 + kSmThreads);
            const bool ok = wait_or_fail_cl(&sh.s_full[sb], (uint32_t)(j >> 1) & 1u, a.status, failed);
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
            // P over this warp's own S columns (the other quarters may still be loading).  The
            // odd CTA's warps gather on p_part, which its forwarder passes on.
            tmem_st16(lane_base + kColS + 128u * sb + 32u * kq, pw);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(even ? &sh.p_full[sb] : &sh.p_part[sb]);
        }
        // Epilogue: l = O column 128 (P times the ones rows of V^T: the sum of the bf16
        // weights the MMA multiplied), O / l -> bf16 (each warp 32 of the dims).
        const bool ok_o = wait_or_fail_cl(&sh.o_full, 0, a.status, failed);
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
        // Both issuers committed to both CTAs after their last MMA, failure or not: wait
        // (bounded) for the pair MMAs in flight before the tensor memory is released.
        if (warp == kWarpQk) mbar_wait_bounded_cl(&sh.qk_done, 0);
        if (warp == kWarpPv) mbar_wait_bounded_cl(&sh.o_full, 0);
    }
    __syncthreads();
    // Neither CTA releases its tensor memory or leaves while the pair's MMAs or the other
    // CTA's arrivals may still reach it.
    cluster_sync_all();
    tc_fence_after();
    if (warp == kWarpQk) {
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tb), "r"(kTmemCols));
    }
}

// ---------------------------------------------------------------- host side
namespace {

using EncodeFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                              const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                              const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                              CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn pr_encode() {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
        return nullptr;
    return reinterpret_cast<EncodeFn>(fn);
}

// 3-D bf16 map with a 128-byte swizzle: dims (inner, rows, planes), box (64, box_rows, 1),
// zero fill out of bounds.
bool pr_map(EncodeFn enc, CUtensorMap *m, const void *ptr, cuuint64_t inner, cuuint64_t rows,
            cuuint64_t planes, cuuint32_t box_rows) {
    cuuint64_t dims[3] = {inner, rows, planes};
    cuuint64_t strides[2] = {inner * 2, inner * 2 * rows};
    cuuint32_t box[3] = {64, box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t pr_smem_bytes(int RT, int C) {
    size_t off = kRingBytes;
    off += (size_t)2 * kBiasBatch * RT * 4;      // bias batches
    off += (size_t)RT * 128 * 4;                 // qbar
    off += (size_t)((C + 7) & ~7) * 2;           // chunk list
    return off + 1024;                           // room to align the base to 1024 bytes
}

template <int BC>
cudaError_t launch_pair_t(const StageArgs &a, cudaStream_t st) {
    static EncodeFn enc = pr_encode();
    if (!enc || !a.vt) return cudaErrorNotSupported;
    const int BHkv = a.B * a.Hkv;
    cudaError_t e = a.vt_ready ? cudaSuccess
                               : launch_vtranspose(a.v, a.vt, BHkv, a.T, 128, st, a.vt_begin, a.vt_end);
    if (e != cudaSuccess) return e;
    // K [B*Hkv][T][128]: box (64 dims, 64 keys).  V^T [B*Hkv][128][T8]: box (64 keys, 72 or
    // 56 dims) for the even and the odd CTA.
    const cuuint64_t T8 = (cuuint64_t)((a.T + 7) & ~7);
    CUtensorMap mk, mve, mvo;
    if (!pr_map(enc, &mk, a.k, 128, (cuuint64_t)a.T, (cuuint64_t)BHkv, 64) ||
        !pr_map(enc, &mve, a.vt, T8, 128, (cuuint64_t)BHkv, kVRows) ||
        !pr_map(enc, &mvo, a.vt, T8, 128, (cuuint64_t)BHkv, kVRowsOdd))
        return cudaErrorInvalidValue;
    PrArgs ta;
    ta.s = a;
    ta.RT = 128 / a.G;
    ta.pair0 = a.t_begin / (2 * ta.RT);
    ta.n_pairs_bg = ((a.t_end + ta.RT - 1) / ta.RT + 1) / 2 - ta.pair0;
    size_t off = kRingBytes;
    ta.off_bias = off;
    off += (size_t)2 * kBiasBatch * ta.RT * 4;
    ta.off_qbar = off;
    off += (size_t)ta.RT * 128 * 4;
    ta.off_list = off;
    const size_t smem = pr_smem_bytes(ta.RT, a.C);
    auto kern = k_attend_pair<BC>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const long long grid = 2LL * ta.n_pairs_bg * BHkv;
    if (grid == 0) return cudaSuccess;
    kern<<<(unsigned)grid, kPrThreads, smem, st>>>(mk, mve, mvo, ta);
    return cudaGetLastError();
}

}  // namespace

bool attend_pair_supported(const StageArgs &a) {
    // A pair's two tiles (2 x 128/G tokens) must share one diagonal chunk.
    if (!(a.D == 128 && a.G >= 2 && a.G <= 128 && 128 % a.G == 0 && (a.Bc == 64 || a.Bc == 128) &&
          2 * (128 / a.G) <= a.Bc))
        return false;
    return pr_smem_bytes(128 / a.G, a.C) + sizeof(PrShared) <= 227 * 1024;
}

cudaError_t launch_attend_pair(const StageArgs &a, cudaStream_t st) {
    if (a.Bc == 64) return launch_pair_t<64>(a, st);
    if (a.Bc == 128) return launch_pair_t<128>(a, st);
    return cudaErrorInvalidValue;
}

}  // namespace dash
