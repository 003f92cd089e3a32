// decode.cu -- one incremental-decode step: Stage 1 routing and Stage 2 attention for the
// newest token of every sequence, in a single launch.
//
// liuzhao09.github.io "DashAttention 精读", section 2: the three stages support incremental
// decoding with a chunk-representation cache; gist.science "DashAttention ...", Technische
// Zusammenfassung, "Stufe 0": complete chunks' summaries are frozen and cached (the cache is
// maintained by dash_update_chunk_cache).  Decode is memory-bound: the step reads the
// cached summaries and the active chunks' K/V once.  At one token per sequence the step is
// short, so the kernel is laid out to keep its memory latencies off one serial path.
//
// One thread-block cluster of kDecCluster CTAs per (b, g):
//   1. every CTA builds qbar; CTA r scores the r-th slice of the routable chunks, four lanes
//      per chunk (x_c = qbar . summary_c * (alpha-1) gamma / sqrt(D), route_dot's arithmetic
//      and summation order, so prefill and decode route alike) and stores each score into
//      every CTA's score row through distributed shared memory (st.shared::cluster); one
//      cluster barrier later every CTA holds the whole row;
//   2. warp 0 of every CTA solves the same tau (same code and data -> same bits).  Meanwhile
//      one warp attends over the diagonal chunk (always active, bias 0: it needs no tau;
//      its first K/V copies were issued at kernel entry).  (An L2 prefetch of the chunks
//      above a lower bound of tau, by the idle warps, measured slower: the bound from a few
//      Newton steps still leaves several times the support above it.);
//   3. rank 0 writes the optional p row and mask words; the routed sub-blocks (32 keys of an
//      active chunk) are dealt round-robin to the cluster's warps, which run the 16-row
//      mma.sync attention over their share (K/V double-buffered per warp);
//   4. warp partials (max, sum, O) merge inside each CTA; after a cluster barrier each CTA
//      merges one eighth of the output (row, dim) pairs across the cluster through
//      distributed shared memory and writes them in bf16.
#include "attn_warp.cuh"

namespace dash {

constexpr int kDecCluster = 8;
constexpr int kDecWarps = 4;
constexpr int kDecSlots = kDecCluster * kDecWarps;          // warps of one cluster
constexpr int kTauRegs = 33;                                // tau solved in registers up to 1056 scores

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;\n" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n"
                 "barrier.cluster.wait.acquire.aligned;\n" ::: "memory");
}
// Split cluster barrier: arrive at entry, wait before the first access to a peer's shared
// memory (a peer's shared memory may be used only once the peer has started).
__device__ __forceinline__ void cluster_arrive_relaxed() {
    asm volatile("barrier.cluster.arrive.relaxed.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
    asm volatile("barrier.cluster.wait.aligned;\n" ::: "memory");
}
// Address of the same shared-memory variable in CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t map_rank(const void *p, uint32_t rank) {
    uint32_t out;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;\n" : "=r"(out) : "r"(smem_u32(p)), "r"(rank));
    return out;
}
__device__ __forceinline__ float ld_cluster_f32(uint32_t addr) {
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];\n" : "=f"(v) : "r"(addr) : "memory");
    return v;
}
__device__ __forceinline__ void st_cluster_f32(uint32_t addr, float v) {
    asm volatile("st.shared::cluster.f32 [%0], %1;\n" ::"r"(addr), "f"(v) : "memory");
}

int decode_supported(int G, int Ccap, int D) {
    (void)D;
    return G >= 1 && G <= 16 && 16 % G == 0 && Ccap <= 8192;
}

// Shared-memory layout of one decode CTA (byte offsets).
template <int D>
struct DecLayout {
    static constexpr size_t tile = (size_t)kSub * D * 2;          // one K or V tile
    static constexpr size_t warp_tiles = 2 * tile;                 // >= a warp partial
    static constexpr size_t part = 16 * D * 4 + 2 * 16 * 4;        // O[16][D], m[16], l[16]
    static_assert(warp_tiles >= part, "warp partial must fit in the warp's tiles");
    size_t qbar, cta_part, tiles, xs, list, sel, total;
    __host__ __device__ DecLayout(int Ccap) {
        qbar = 0;
        cta_part = qbar + D * 4;
        tiles = cta_part + part;
        tiles = (tiles + 127) & ~(size_t)127;
        xs = tiles + kDecWarps * warp_tiles;
        list = xs + (size_t)((Ccap + 3) & ~3) * 4;
        sel = list + (size_t)(Ccap + 2) * 4;
        total = sel + (size_t)((Ccap + 63) / 32) * 4;
    }
};

template <int D, int BC>
__global__ void __launch_bounds__(kDecWarps * 32) k_decode(DecodeArgs a) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    __shared__ float tau_s;
    __shared__ int nact_s;
    __shared__ float wfac[kDecWarps][16], wmax[16];   // the CTA merge's per-row weights
    const DecLayout<D> L(a.Ccap);
    float *qbar = reinterpret_cast<float *>(smem_raw + L.qbar);
    float *cpart = reinterpret_cast<float *>(smem_raw + L.cta_part);   // O[16][D], m, l
    float *xs = reinterpret_cast<float *>(smem_raw + L.xs);
    int *list = reinterpret_cast<int *>(smem_raw + L.list);
    uint32_t *sel = reinterpret_cast<uint32_t *>(smem_raw + L.sel);   // top-k selection bits

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = cluster_rank();
    const int bg = blockIdx.x / kDecCluster, b = bg / a.Hkv, g = bg % a.Hkv;
    const int G = a.G;
    const bool append = a.k_new != nullptr;
    const int Lb = a.seq_lens[b] + (append ? 1 : 0);   // tokens attended, the new one included
    if (Lb < 1 || Lb > a.cap) {                 // uniform across the cluster: no barrier
        if (tid == 0 && rank == 0) report(a.status, DASH_ERR_INVALID_ARGUMENT);
        return;
    }
    const int t = Lb - 1, ct = t / BC, n = ct;
    const __nv_bfloat16 *q = reinterpret_cast<const __nv_bfloat16 *>(a.q) + (long long)b * a.Hq * D;
    // Paged cache: every page the step reads (chunks 0 .. c_t) must lie in the pools; the
    // check gives the same answer in every CTA of the cluster, so all return together.
    const int32_t *bt = a.block_table ? a.block_table + (long long)b * a.max_blocks : nullptr;
    if (bt) {
        int bad = 0;
        for (int c = tid; c <= ct; c += kDecWarps * 32) bad |= (bt[c] < 0 || bt[c] >= a.n_pages);
        if (__syncthreads_or(bad)) {
            if (tid == 0 && rank == 0) report(a.status, DASH_ERR_INVALID_ARGUMENT);
            return;
        }
    }
    cluster_arrive_relaxed();
    // Keys / values of chunk c (its first key) and the summary of chunk c.
    auto kv_base = [&](const void *pool, int c) -> const __nv_bfloat16 * {
        const __nv_bfloat16 *p0 = reinterpret_cast<const __nv_bfloat16 *>(pool);
        if (bt) return p0 + ((long long)bt[c] * a.Hkv + g) * BC * D;
        return p0 + ((long long)bg * a.cap + (long long)c * BC) * D;
    };
    // Keys of chunk c that exist in memory (a contiguous cache may end inside its last chunk).
    auto kv_rows = [&](int c) -> int { return bt ? BC : min(BC, a.cap - c * BC); };
    auto summary_of = [&](int c) -> const float * {
        if (bt) return a.summary + ((long long)bt[c] * a.Hkv + g) * D;
        return a.summary + ((long long)bg * a.Cf + c) * D;
    };

    // Per-warp attention state: 16 rows (the group's G heads), K/V tiles of kSub keys.
    unsigned char *ks = smem_raw + L.tiles + warp * L.warp_tiles;
    unsigned char *vs = ks + L.tile;
    constexpr int NSUB = BC / kSub;
    const bool diag_warp = rank == 0 && warp == 1;
    const int n_diag = (t - ct * BC) / kSub + 1;   // sub-blocks of the diagonal chunk up to t
    if (diag_warp) {
        if (append) {
            // Decode step: the new token's key and value into row t of the cache first (the
            // cluster barrier after the scores publishes them to the other CTAs).
            const long long src = ((long long)b * a.Hkv + g) * D;
            __nv_bfloat16 *kd = const_cast<__nv_bfloat16 *>(kv_base(a.k, ct)) + (long long)(t - ct * BC) * D;
            __nv_bfloat16 *vd = const_cast<__nv_bfloat16 *>(kv_base(a.v, ct)) + (long long)(t - ct * BC) * D;
            const uint2 *ksrc = reinterpret_cast<const uint2 *>(reinterpret_cast<const __nv_bfloat16 *>(a.k_new) + src);
            const uint2 *vsrc = reinterpret_cast<const uint2 *>(reinterpret_cast<const __nv_bfloat16 *>(a.v_new) + src);
            for (int i = lane; i < D / 4; i += 32) {
                reinterpret_cast<uint2 *>(kd)[i] = ksrc[i];
                reinterpret_cast<uint2 *>(vd)[i] = vsrc[i];
            }
            __threadfence();
            __syncwarp();
        }
        // The diagonal chunk is always attended: start its first copies now.
        load_sub<D>(ks, kv_base(a.k, ct), 0, kv_rows(ct));
        cp_async_commit();
        load_sub<D>(vs, kv_base(a.v, ct), 0, kv_rows(ct));
        cp_async_commit();
    }

    // 1. group-mean query and this CTA's slice of the scores, stored into every CTA's row.
    // Four lanes per chunk: lane quarter k accumulates route_dot's partial sum p_k (the float4
    // groups 4i + k, one sequential fmaf chain), combined as (p0 + p1) + (p2 + p3).  Each
    // warp scores 8 chunks per step; the summaries of its next step are loaded while this
    // one is scored (its first step's before qbar, which they do not depend on).
    const int c_lo = (int)((long long)n * rank / kDecCluster);
    const int c_hi = (int)((long long)n * (rank + 1) / kDecCluster);
    const int kslice = lane & 3, cc = lane >> 2;
    float4 sv[D / 16];
    auto load_summaries = [&](int cb) {
        const int c = cb + cc;
        const float4 *s4 = reinterpret_cast<const float4 *>(summary_of(c < c_hi ? c : cb));
#pragma unroll
        for (int i = 0; i < D / 16; ++i) sv[i] = __ldg(s4 + 4 * i + kslice);
    };
    if (c_lo + warp * 8 < c_hi) load_summaries(c_lo + warp * 8);
    for (int d8 = tid * 8; d8 < D; d8 += kDecWarps * 32 * 8) {
        float m[8];
        group_mean8(q + (long long)g * G * D + d8, D, G, m);
#pragma unroll
        for (int e = 0; e < 8; ++e) qbar[d8 + e] = m[e];
    }
    const int r_lo = lane >> 2, r_hi = r_lo + 8, qd = lane & 3;
    const bool ok_lo = r_lo < G, ok_hi = r_hi < G;
    uint32_t qf[D / 16][4];
    {
        const __nv_bfloat16 *q_lo = q + (long long)(g * G + (ok_lo ? r_lo : 0)) * D;
        const __nv_bfloat16 *q_hi = q + (long long)(g * G + (ok_hi ? r_hi : 0)) * D;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            const int d0 = 16 * kk + 2 * qd;
            qf[kk][0] = ok_lo ? *reinterpret_cast<const uint32_t *>(q_lo + d0) : 0u;
            qf[kk][1] = ok_hi ? *reinterpret_cast<const uint32_t *>(q_hi + d0) : 0u;
            qf[kk][2] = ok_lo ? *reinterpret_cast<const uint32_t *>(q_lo + d0 + 8) : 0u;
            qf[kk][3] = ok_hi ? *reinterpret_cast<const uint32_t *>(q_hi + d0 + 8) : 0u;
        }
    }
    __syncthreads();
    const float scale = a.rc.kind == 0 ? a.rc.sscale : a.rc.xscale;
    cluster_wait();                               // every peer has started
    {
        uint32_t xs_at[kDecCluster];              // the score row of every CTA
#pragma unroll
        for (int r = 0; r < kDecCluster; ++r) xs_at[r] = map_rank(xs, (uint32_t)r);
        const float4 *q4 = reinterpret_cast<const float4 *>(qbar);
        for (int cb = c_lo + warp * 8; cb < c_hi; cb += kDecWarps * 8) {
            float4 cur[D / 16];
#pragma unroll
            for (int i = 0; i < D / 16; ++i) cur[i] = sv[i];
            if (cb + kDecWarps * 8 < c_hi) load_summaries(cb + kDecWarps * 8);
            float acc = 0.f;
#pragma unroll
            for (int i = 0; i < D / 16; ++i) {
                const float4 qq = q4[4 * i + kslice];
                acc = fmaf(qq.x, cur[i].x, acc);
                acc = fmaf(qq.y, cur[i].y, acc);
                acc = fmaf(qq.z, cur[i].z, acc);
                acc = fmaf(qq.w, cur[i].w, acc);
            }
            const float pair = acc + __shfl_down_sync(kFull, acc, 1);      // p0+p1 | p2+p3
            const float dot = pair + __shfl_down_sync(kFull, pair, 2);
            const int c = cb + cc;
            if (c < c_hi && kslice == 0) {
                const float x = __fmul_rn(dot, scale);
#pragma unroll
                for (int r = 0; r < kDecCluster; ++r)
                    st_cluster_f32(xs_at[r] + 4u * (uint32_t)c, x);
            }
        }
    }
    cluster_sync_all();                           // every CTA holds the whole score row

    UnitState<D> st;
#pragma unroll
    for (int j = 0; j < D / 8; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) st.o[j][e] = 0.f;
    st.m_lo = st.m_hi = -INFINITY;
    st.l_lo = st.l_hi = 0.f;
    float tau = 0.f;
    // Attention over `cnt` sub-blocks: sub-block i is keys [sub_of(i) kSub, +kSub) of chunk
    // chunk_of(i); keys past the end of a contiguous cache are zero-filled, keys after t in the
    // diagonal chunk are masked by the softmax.  K/V double-buffered through the warp's tiles;
    // `preloaded`: the copies of sub-block 0 are already in flight.
    auto attend = [&](int cnt, auto chunk_of, auto sub_of, bool preloaded) {
        if (cnt <= 0) return;
        if (!preloaded) {
            const int c0 = chunk_of(0);
            load_sub<D>(ks, kv_base(a.k, c0), sub_of(0) * kSub, kv_rows(c0));
            cp_async_commit();
            load_sub<D>(vs, kv_base(a.v, c0), sub_of(0) * kSub, kv_rows(c0));
            cp_async_commit();
        }
        for (int s = 0; s < cnt; ++s) {
            const int c = chunk_of(s);
            const int key0 = c * BC + sub_of(s) * kSub;
            const bool diag = c == ct, more = s + 1 < cnt;
            const int c_next = more ? chunk_of(s + 1) : 0;
            const int sub_next = more ? sub_of(s + 1) * kSub : 0;
            float bias2 = 0.f;
            if (!diag)
                bias2 = a.rc.kind == kKindTopk ? 0.f                 // top-k: uniform prior
                        : a.rc.kind == 0 ? a.rc.sigma2 * (xs[c] - tau)
                                         : a.rc.bscale2 * log2f(fmaxf(__fsub_rn(xs[c], tau), 1e-37f));
            cp_async_wait<1>();
            __syncwarp();
            float acc[4][4];
            qk_sub<D>(acc, qf, ks);
            __syncwarp();
            if (more) {
                load_sub<D>(ks, kv_base(a.k, c_next), sub_next, kv_rows(c_next));
                cp_async_commit();
            }
            uint32_t pa[2][4];
            softmax_sub<D>(st, acc, pa, a.qk_scale2, ok_lo ? bias2 : -INFINITY,
                           ok_hi ? bias2 : -INFINITY, diag, key0, t, t);
            if (more) cp_async_wait<1>(); else cp_async_wait<0>();
            __syncwarp();
            pv_sub<D>(st, pa, vs);
            __syncwarp();
            if (more) {
                load_sub<D>(vs, kv_base(a.v, c_next), sub_next, kv_rows(c_next));
                cp_async_commit();
            }
        }
    };

    // 2. threshold (warp 0 of every CTA, same bits) and the diagonal chunk.  With
    // estimate_diagonal the diagonal chunk's score joins the candidates as entry n.
    const int n_eff = n + (a.rc.est_diag ? 1 : 0);
    if (warp == 0) {
        if (a.rc.est_diag) {
            // (with a decode step, row t was written in this launch: coherent loads)
            const float dd = append ? diag_dot<D, true>(kv_base(a.k, ct), t - ct * BC + 1,
                                                        a.head_cls + (long long)g * D, qbar, a.rc.inv_sqrt_d)
                                    : diag_dot<D>(kv_base(a.k, ct), t - ct * BC + 1,
                                                  a.head_cls + (long long)g * D, qbar, a.rc.inv_sqrt_d);
            if (lane == 0) xs[n] = __fmul_rn(dd, scale);
            __syncwarp();
        }
        float tw;
        if (a.rc.kind == kKindTopk) {
            // Top-k: selection bits in index order (lower index first on ties); tau = the
            // lowest selected score.
            const bool all = n <= a.rc.topk;
            int need = 0;
            uint32_t key = 0;
            if (!all) key = warp_topk_key(xs, n, a.rc.topk, need);
            int run = 0;
            for (int c0 = 0; c0 < n; c0 += 32) {
                const unsigned bal = __ballot_sync(kFull, topk_selected(xs, c0 + lane, n, all, key, need, run));
                if (lane == 0) sel[c0 >> 5] = bal;
            }
            if (n > 0 && all) {
                float mn = INFINITY;
                for (int c = lane; c < n; c += 32) mn = fminf(mn, xs[c]);
                tw = -warp_max(-mn);
            } else {
                tw = n > 0 ? key_f32(key) : __int_as_float(0x7fc00000);
            }
        } else if (n_eff > 0 && n_eff <= 32 * kTauRegs) {
            // The row in registers (same bits as the solve on the row in shared memory).
            float v[kTauRegs];
#pragma unroll
            for (int k = 0; k < kTauRegs; ++k) v[k] = lane + 32 * k < n_eff ? xs[lane + 32 * k] : 0.f;
            tw = warp_entmax_tau_regs(v, n_eff, a.rc, a.status);
        } else {
            tw = n_eff > 0 ? warp_entmax_tau(xs, n_eff, a.rc, a.status) : __int_as_float(0x7fc00000);
        }
        if (lane == 0) tau_s = tw;
    } else if (diag_warp) {
        attend(n_diag, [&](int) { return ct; }, [&](int i) { return i; }, true);
    }
    __syncthreads();
    tau = tau_s;
    auto active = [&](int c) -> bool {
        if (a.rc.kind == kKindTopk) return c < n && ((sel[c >> 5] >> (c & 31)) & 1u);
        return c < n && (a.rc.kind == 0 || __fsub_rn(xs[c], tau) > 0.f);
    };
    if (rank == 0) {
        if (a.mask) {
            for (int w = warp; w < a.Wcap; w += kDecWarps) {
                const int c0 = w * 64 + lane, c1 = c0 + 32;
                unsigned lo = __ballot_sync(kFull, c0 == ct || active(c0));
                unsigned hi = __ballot_sync(kFull, c1 == ct || active(c1));
                if (lane == 0) a.mask[(long long)bg * a.Wcap + w] = ((uint64_t)hi << 32) | lo;
            }
        }
        if (a.p) {
            for (int c = tid; c < a.Ccap; c += kDecWarps * 32) {
                float val = 0.f;
                if (a.rc.kind == kKindTopk) {
                    val = active(c) ? 1.f / (float)min(n, a.rc.topk) : 0.f;
                } else if (active(c) || (c == n && n < n_eff)) {   // routed, or the estimated diagonal
                    const float m = __fsub_rn(xs[c], tau);
                    val = a.rc.kind == 0 ? expf(xs[c] - tau) : m > 0.f ? pow_beta(m, a.rc) : 0.f;
                }
                a.p[(long long)bg * a.Ccap + c] = val;
            }
        }
    }

    // 3. active list (same on every CTA): the routed chunks (the diagonal is attended
    // separately above).
    // Lane l lists its chunks l, l + 32, ... of each block of 1024, the lanes in order.
    if (warp == 0) {
        int pos = 0;
        const int kind = a.rc.kind;
        const float tv = tau;
        for (int c0 = 0; c0 < n; c0 += 32 * 32) {
            uint32_t bits = 0;
#pragma unroll
            for (int k = 0; k < 32; ++k) {
                const int c = c0 + lane + 32 * k;
                const bool act = c < n && (kind == kKindTopk ? ((sel[c >> 5] >> (c & 31)) & 1u) != 0
                                                             : (kind == 0 || __fsub_rn(xs[c], tv) > 0.f));
                if (act && dash_check(c < a.Cf && (c + 1) * BC <= a.cap, a.status)) bits |= 1u << k;
            }
            const int cnt = __popc(bits);
            int incl = cnt;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(kFull, incl, o);
                if (lane >= o) incl += y;
            }
            int p = pos + incl - cnt;
            while (bits) {
                const int k = __ffs(bits) - 1;
                bits &= bits - 1u;
                list[p++] = c0 + lane + 32 * k;
            }
            pos += __shfl_sync(kFull, incl, 31);
        }
        if (lane == 0) nact_s = pos;
    }
    __syncthreads();
    {
        // This warp's share of the routed sub-blocks: entries e = first + i * kDecSlots.
        const int n_ent = nact_s * NSUB;
        const int first = (int)rank + kDecCluster * warp;
        const int my_n = first < n_ent ? (n_ent - first + kDecSlots - 1) / kDecSlots : 0;
        attend(my_n, [&](int i) { return list[(first + i * kDecSlots) / NSUB]; },
               [&](int i) { return (first + i * kDecSlots) % NSUB; }, false);
    }

    // 4a. warp partial -> the warp's own tile space.
    float l_lo = st.l_lo, l_hi = st.l_hi;
    l_lo += __shfl_xor_sync(kFull, l_lo, 1);
    l_lo += __shfl_xor_sync(kFull, l_lo, 2);
    l_hi += __shfl_xor_sync(kFull, l_hi, 1);
    l_hi += __shfl_xor_sync(kFull, l_hi, 2);
    float *wp = reinterpret_cast<float *>(ks);          // O[16][D], m[16], l[16]
#pragma unroll
    for (int j = 0; j < D / 8; ++j) {
        const int d0 = 8 * j + 2 * qd;
        wp[r_lo * D + d0] = st.o[j][0];
        wp[r_lo * D + d0 + 1] = st.o[j][1];
        wp[r_hi * D + d0] = st.o[j][2];
        wp[r_hi * D + d0 + 1] = st.o[j][3];
    }
    if (qd == 0) {
        wp[16 * D + r_lo] = st.m_lo;
        wp[16 * D + r_hi] = st.m_hi;
        wp[16 * D + 16 + r_lo] = l_lo;
        wp[16 * D + 16 + r_hi] = l_hi;
    }
    __syncthreads();

    // 4b. CTA merge of the warp partials into cpart: each row's warp weights 2^(m_w - m*)
    // once, then every output of the row with them.
    if (tid < 16) {
        const int r = tid;
        float mstar = -INFINITY;
        for (int w = 0; w < kDecWarps; ++w)
            mstar = fmaxf(mstar, reinterpret_cast<float *>(smem_raw + L.tiles + w * L.warp_tiles)[16 * D + r]);
        const float mu = mstar == -INFINITY ? 0.f : mstar;
        for (int w = 0; w < kDecWarps; ++w)
            wfac[w][r] = fast_exp2(reinterpret_cast<float *>(smem_raw + L.tiles + w * L.warp_tiles)[16 * D + r] - mu);
        wmax[r] = mstar;
    }
    __syncthreads();
    for (int idx = tid; idx < 16 * D + 16; idx += kDecWarps * 32) {
        const int r = idx < 16 * D ? idx / D : idx - 16 * D;
        float acc = 0.f;
        for (int w = 0; w < kDecWarps; ++w) {
            const float *pw = reinterpret_cast<float *>(smem_raw + L.tiles + w * L.warp_tiles);
            const float f = wfac[w][r];
            acc += f * (idx < 16 * D ? pw[idx] : pw[16 * D + 16 + r]);
        }
        if (idx < 16 * D) cpart[idx] = acc;
        else { cpart[16 * D + r] = wmax[r]; cpart[16 * D + 16 + r] = acc; }
    }

    // 4c. cluster merge: CTA r combines the r-th eighth of the (row, dim) outputs.
    cluster_sync_all();
    {
        __nv_bfloat16 *out = reinterpret_cast<__nv_bfloat16 *>(a.out) + ((long long)b * a.Hq + g * G) * D;
        const int total = G * D, per = (total + kDecCluster - 1) / kDecCluster;
        const int i_end = min(total, ((int)rank + 1) * per);
        for (int idx = (int)rank * per + tid; idx < i_end; idx += kDecWarps * 32) {
            const int r = idx / D;
            float mr[kDecCluster], lr[kDecCluster], orr[kDecCluster], mstar = -INFINITY;
#pragma unroll
            for (int k = 0; k < kDecCluster; ++k) {
                mr[k] = ld_cluster_f32(map_rank(&cpart[16 * D + r], k));
                lr[k] = ld_cluster_f32(map_rank(&cpart[16 * D + 16 + r], k));
                orr[k] = ld_cluster_f32(map_rank(&cpart[idx], k));
            }
#pragma unroll
            for (int k = 0; k < kDecCluster; ++k) mstar = fmaxf(mstar, mr[k]);
            const float mu = mstar == -INFINITY ? 0.f : mstar;
            float o = 0.f, l = 0.f;
#pragma unroll
            for (int k = 0; k < kDecCluster; ++k) {
                const float f = fast_exp2(mr[k] - mu);
                o += f * orr[k];
                l += f * lr[k];
            }
            out[idx] = __float2bfloat16_rn(o / l);
        }
    }
    cluster_sync_all();      // peers stay resident until every CTA has read their partials
    if (append && rank == 0) {
        // Decode step: the chunk the new token completed gets its Stage 0 summary (the same
        // function as the cache-update kernel; the keys were written by this CTA), and the
        // sequence's last cluster to finish stores the new length.
        if (warp == 2 && (t + 1) % BC == 0) {
            float *dst = bt ? a.summary_out + ((long long)bt[ct] * a.Hkv + g) * D
                            : a.summary_out + ((long long)bg * a.Cf + ct) * D;
            summarize_chunk_warp<D, BC>(kv_base(a.k, ct), a.head_cls + (long long)g * D, dst);
        }
        if (tid == 0) {
            __threadfence();
            if (atomicAdd(&a.arrive[b], 1) == a.Hkv - 1) {
                a.arrive[b] = 0;
                a.seq_out[b] = Lb;
            }
        }
    }
}

template <int D, int BC>
static cudaError_t launch_decode_t(const DecodeArgs &a, cudaStream_t st) {
    const DecLayout<D> L(a.Ccap);
    auto kern = k_decode<D, BC>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)L.total);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(a.B * a.Hkv * kDecCluster));
    cfg.blockDim = dim3(kDecWarps * 32);
    cfg.dynamicSmemBytes = L.total;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kDecCluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t st) {
    if (a.D == 128 && a.Bc == 64) return launch_decode_t<128, 64>(a, st);
    if (a.D == 128 && a.Bc == 128) return launch_decode_t<128, 128>(a, st);
    if (a.D == 64 && a.Bc == 64) return launch_decode_t<64, 64>(a, st);
    if (a.D == 64 && a.Bc == 128) return launch_decode_t<64, 128>(a, st);
    return cudaErrorInvalidValue;
}

}  // namespace dash
