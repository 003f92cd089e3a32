// attend.cu -- Stage 2: prior-induced block-sparse softmax attention (warp-MMA path).
//
// gist.science "DashAttention: Differentiable and Adaptive Sparse Hierarchical Attention",
// Technische Zusammenfassung, "Stufe 2: Prior-induzierte spaerliche Softmax": softmax with
// the reference distribution replaced by a prior g built from the routing w (g = 0 where
// w = 0, so zero-probability chunks are masked), a separate branch for the diagonal chunk,
// and a FlashAttention-style kernel that iterates the active chunks of a bit-packed mask and
// adds the routing bias to the logits before the softmax.
//
// Work unit = 16 query rows of one (b, g) that share a routing: the 16 heads of one token
// when G >= 16 (G / 16 units per token), or 16 / G tokens x G heads when G < 16 (their
// chunks are the union of the tokens' masks; a row whose own token did not route to a chunk
// gets bias -inf there).  One warp per unit, units ordered longest (largest t) first.
//
// Per unit: the active chunks are walked straight from the mask words (find-first-set),
// up to 32 at a time; lane i recomputes the bias of the i-th chunk from (qbar.summary, tau)
// with the exact arithmetic of Stage 1, so the margin m = x - tau is bit-identical and > 0.
// bias = sigma * log p_c = sigma * beta * log(m).  The diagonal chunk comes last with
// bias 0 and the causal mask.  Each 32-key sub-block: cp.async K, V into swizzled shared
// memory, S = Q K^T and O += P V with mma.sync m16n8k16 (bf16 in, fp32 accumulate), online
// softmax in the log2 domain in registers.
#include "attn_warp.cuh"

namespace dash {

template <int D, int BC>
__global__ void __launch_bounds__(kAttnWarps * 32) k_attend(StageArgs a, int TU, int UPT,
                                                            long long n_units) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (a.cost) {                           // run-time choice against the 128-key-block kernel
        if (attend_fa_chosen(a)) return;
        attend_record_ran(a, 2);
    }
    const long long unit = (long long)blockIdx.x * kAttnWarps + warp;
    if (unit >= n_units) return;

    // Per-warp shared memory: K tile, V tile, qbar[TU][D], bias[TU][32].
    const size_t tile_bytes = (size_t)kSub * D * 2;
    const size_t warp_bytes = 2 * tile_bytes + (size_t)TU * D * 4 + (size_t)TU * 32 * 4;
    unsigned char *base = smem_raw + warp * warp_bytes;
    unsigned char *ks = base, *vs = base + tile_bytes;
    float *qbar = reinterpret_cast<float *>(base + 2 * tile_bytes);
    float *bias_s = qbar + TU * D;

    const int G = a.G, Gu = G >= 16 ? 16 : G;
    const int NTG = (a.T + TU - 1) / TU;
    const int k = (int)(unit % UPT);
    long long rest = unit / UPT;
    const int g = (int)(rest % a.Hkv);
    rest /= a.Hkv;
    const int b = (int)(rest % a.B);
    const int tg = NTG - 1 - (int)(rest / a.B);
    const int t0 = tg * TU;
    const int ct = t0 / BC;

    const __nv_bfloat16 *q = reinterpret_cast<const __nv_bfloat16 *>(a.q);
    const __nv_bfloat16 *kp = reinterpret_cast<const __nv_bfloat16 *>(a.k) +
                              ((long long)b * a.Hkv + g) * a.T * D;
    const __nv_bfloat16 *vp = reinterpret_cast<const __nv_bfloat16 *>(a.v) +
                              ((long long)b * a.Hkv + g) * a.T * D;
    const long long bg = (long long)b * a.Hkv + g;

    // Rows of this thread: r_lo = lane/4, r_hi = r_lo + 8.
    const int r_lo = lane >> 2, r_hi = r_lo + 8, qd = lane & 3;
    const int tok_lo = t0 + r_lo / Gu, tok_hi = t0 + r_hi / Gu;
    const int head_lo = g * G + k * 16 + r_lo % Gu, head_hi = g * G + k * 16 + r_hi % Gu;
    const bool ok_lo = tok_lo < a.T, ok_hi = tok_hi < a.T;

    uint32_t qf[D / 16][4];
    {
        const __nv_bfloat16 *q_lo = q + (((long long)b * a.Hq + head_lo) * a.T + (ok_lo ? tok_lo : 0)) * D;
        const __nv_bfloat16 *q_hi = q + (((long long)b * a.Hq + head_hi) * a.T + (ok_hi ? tok_hi : 0)) * D;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            const int d0 = 16 * kk + 2 * qd;
            qf[kk][0] = ok_lo ? *reinterpret_cast<const uint32_t *>(q_lo + d0) : 0u;
            qf[kk][1] = ok_hi ? *reinterpret_cast<const uint32_t *>(q_hi + d0) : 0u;
            qf[kk][2] = ok_lo ? *reinterpret_cast<const uint32_t *>(q_lo + d0 + 8) : 0u;
            qf[kk][3] = ok_hi ? *reinterpret_cast<const uint32_t *>(q_hi + d0 + 8) : 0u;
        }
    }

    const bool route = !a.ignore_routing && ct > 0;
    if (route) {
        for (int idx = lane; idx < TU * (D / 8); idx += 32) {
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
    __syncwarp();

    UnitState<D> st;
#pragma unroll
    for (int j = 0; j < D / 8; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) st.o[j][e] = 0.f;
    st.m_lo = st.m_hi = -INFINITY;
    st.l_lo = st.l_hi = 0.f;

    // Iterator over the union of the unit's routed chunks (bits < c_t of the mask words).
    const int wmax = ct > 0 ? (ct - 1) >> 6 : -1;
    auto load_word = [&](int w) -> uint64_t {
        uint64_t word = 0;
        if (a.ignore_routing) {
            word = ~0ull;
        } else {
            for (int u = 0; u < TU; ++u) {
                const int t = t0 + u;
                if (t < a.T) word |= a.mask[(bg * a.T + t) * a.W + w];
            }
        }
        const int lim = ct - 64 * w;                  // bits [0, lim) are routable
        if (lim < 64) word &= (1ull << lim) - 1ull;
        return word;
    };
    int w_cur = 0;
    uint64_t bits = wmax >= 0 ? load_word(0) : 0ull;
    bool diag_pending = true;
    constexpr int NSUB = BC / kSub;

    while (true) {
        // Gather the next batch of up to 32 chunks (lane i keeps the i-th); the diagonal
        // chunk is appended once the routed chunks are exhausted.
        int nb = 0, my_c = -1;
        bool batch_has_diag = false;
        while (nb < 32) {
            while (bits == 0ull && w_cur < wmax) bits = load_word(++w_cur);
            if (bits == 0ull) {
                if (diag_pending) {
                    if (lane == nb) my_c = ct;
                    ++nb;
                    diag_pending = false;
                    batch_has_diag = true;
                }
                break;
            }
            const int c = w_cur * 64 + __ffsll((long long)bits) - 1;
            bits &= bits - 1ull;
            if (lane == nb) my_c = c;
            ++nb;
        }
        if (nb == 0) break;

        // Biases of the batch's routed chunks for each token of the unit.
        const int n_routed = batch_has_diag ? nb - 1 : nb;
        if (lane < n_routed) {
            for (int u = 0; u < TU; ++u) {
                const int t = t0 + u;
                float b2;
                if (a.ignore_routing) {
                    b2 = 0.f;
                } else if (t >= a.T) {
                    b2 = -INFINITY;
                } else {
                    const long long row = bg * a.T + t;
                    const bool act = dash_check(my_c < a.Cf, a.status) &&
                                     (TU == 1 || ((a.mask[row * a.W + (my_c >> 6)] >> (my_c & 63)) & 1ull));
                    b2 = act ? routed_bias2<D>(qbar + u * D,
                                               a.summary + (bg * a.Cf + my_c) * D, a.tau[row], a.rc)
                             : -INFINITY;
                }
                bias_s[u * 32 + lane] = b2;
            }
        }
        __syncwarp();

        // Walk the batch sub-block by sub-block: K of the next sub-block streams in while
        // this one's P V runs, V of the next while the next Q K^T runs.
        const int nsteps = nb * NSUB;
        {
            const int c0 = __shfl_sync(kFull, my_c, 0);
            load_sub<D>(ks, kp, c0 * BC, a.T);
            cp_async_commit();
            load_sub<D>(vs, vp, c0 * BC, a.T);
            cp_async_commit();
        }
        for (int s = 0; s < nsteps; ++s) {
            const int i = s / NSUB, sb = s % NSUB;
            const int c = __shfl_sync(kFull, my_c, i);
            const bool diag = c == ct;
            const int key0 = c * BC + sb * kSub;
            const bool more = s + 1 < nsteps;
            const int key_next = more ? __shfl_sync(kFull, my_c, (s + 1) / NSUB) * BC +
                                            ((s + 1) % NSUB) * kSub
                                      : 0;
            cp_async_wait<1>();
            __syncwarp();
            float acc[4][4];
            qk_sub<D>(acc, qf, ks);
            __syncwarp();
            if (more) {
                load_sub<D>(ks, kp, key_next, a.T);
                cp_async_commit();
            }
            float b_lo = 0.f, b_hi = 0.f;
            if (!diag) {
                b_lo = bias_s[((r_lo / Gu) % TU) * 32 + i];
                b_hi = bias_s[((r_hi / Gu) % TU) * 32 + i];
            }
            uint32_t pa[2][4];
            softmax_sub<D>(st, acc, pa, a.qk_scale2, b_lo, b_hi, diag, key0, tok_lo, tok_hi);
            if (more) cp_async_wait<1>(); else cp_async_wait<0>();
            __syncwarp();
            pv_sub<D>(st, pa, vs);
            __syncwarp();
            if (more) {
                load_sub<D>(vs, vp, key_next, a.T);
                cp_async_commit();
            }
        }
        __syncwarp();
    }

    // Normalise and store (bf16, round to nearest even).
    float l_lo = st.l_lo, l_hi = st.l_hi;
    l_lo += __shfl_xor_sync(kFull, l_lo, 1);
    l_lo += __shfl_xor_sync(kFull, l_lo, 2);
    l_hi += __shfl_xor_sync(kFull, l_hi, 1);
    l_hi += __shfl_xor_sync(kFull, l_hi, 2);
    const float inv_lo = 1.f / l_lo, inv_hi = 1.f / l_hi;
    __nv_bfloat16 *out = reinterpret_cast<__nv_bfloat16 *>(a.out);
    __nv_bfloat16 *o_lo = out + (((long long)b * a.Hq + head_lo) * a.T + tok_lo) * D;
    __nv_bfloat16 *o_hi = out + (((long long)b * a.Hq + head_hi) * a.T + tok_hi) * D;
#pragma unroll
    for (int j = 0; j < D / 8; ++j) {
        const int d0 = 8 * j + 2 * qd;
        if (ok_lo)
            *reinterpret_cast<uint32_t *>(o_lo + d0) =
                pack_bf16x2(st.o[j][0] * inv_lo, st.o[j][1] * inv_lo);
        if (ok_hi)
            *reinterpret_cast<uint32_t *>(o_hi + d0) =
                pack_bf16x2(st.o[j][2] * inv_hi, st.o[j][3] * inv_hi);
    }
}

template <int D, int BC>
static cudaError_t launch_attend_t(const StageArgs &a, cudaStream_t st) {
    const int G = a.G;
    const int TU = G >= 16 ? 1 : 16 / G;
    const int UPT = G >= 16 ? G / 16 : 1;
    const long long NTG = (a.T + TU - 1) / TU;
    const long long n_units = NTG * a.B * a.Hkv * UPT;
    if (n_units == 0) return cudaSuccess;
    const size_t warp_bytes = 2 * (size_t)kSub * D * 2 + (size_t)TU * D * 4 + (size_t)TU * 32 * 4;
    const size_t smem = warp_bytes * kAttnWarps;
    auto kern = k_attend<D, BC>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)((n_units + kAttnWarps - 1) / kAttnWarps);
    kern<<<grid, kAttnWarps * 32, smem, st>>>(a, TU, UPT, n_units);
    return cudaGetLastError();
}

// Token-chunk pairs the two Stage 2 kernels would execute for a routed call with G < 8: the
// 128-key-block kernel walks, per tile of 128/G tokens, the union of their chunks
// (cost[0] += |union| x 128/G), the warp-MMA kernel per unit of 16/G tokens
// (cost[1] += |union| x 16/G).  Each token's mask words carry its diagonal bit, so the
// tile's diagonal chunk counts in both.  One warp per tile, lanes over mask words.
__global__ void __launch_bounds__(128) k_union_cost(StageArgs a, unsigned long long *cost,
                                                    int n_tiles_bg) {
    const int lane = threadIdx.x & 31;
    const long long tile = (long long)blockIdx.x * 4 + (threadIdx.x >> 5);
    if (tile >= (long long)n_tiles_bg * a.B * a.Hkv) return;
    const int RT = 128 / a.G, TU = 16 / a.G;
    const long long bg = tile / n_tiles_bg;
    const int t0 = (int)(tile % n_tiles_bg) * RT;
    const int t_last = min(t0 + RT, a.T) - 1;
    const int wlim = (t_last / a.Bc) / 64;       // the last word with a bit the tile can hold
    unsigned long long cf = 0, cw = 0;
    for (int w = lane; w <= wlim; w += 32) {
        uint64_t tile_word = 0;
        for (int u0 = 0; u0 < RT; u0 += TU) {
            uint64_t unit_word = 0;
            for (int u = u0; u < u0 + TU; ++u) {
                const int t = t0 + u;
                if (t < a.T) unit_word |= a.mask[(bg * a.T + t) * a.W + w];
            }
            cw += (unsigned long long)__popcll(unit_word) * TU;
            tile_word |= unit_word;
        }
        cf += (unsigned long long)__popcll(tile_word) * RT;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        cf += __shfl_xor_sync(kFull, cf, o);
        cw += __shfl_xor_sync(kFull, cw, o);
    }
    if (lane == 0) {
        atomicAdd(&cost[0], cf);
        atomicAdd(&cost[1], cw);
    }
}

// Executed token-chunk pairs per unit of time of the two kernels for G = 4, as TFLOP/s on
// executed blocks measured on B200 over the 64K sweep cells: 128-key blocks 470-940 with
// 64-key chunks and 610-1000 with 128-key chunks (lower where more of a batch's pairs are
// active and need a routing dot product), warp MMA 128-155.  Only their ratio is used; these
// values pick the faster kernel in all six cells (the closest, alpha 1.5 and 2 with 64-key
// chunks, lie at ratios 4.5 and 5.9 on either side of 690 / 135 = 5.1).
constexpr float kRateFa64 = 690.f, kRateFa128 = 900.f, kRateWarp = 135.f;

// A run-time choice applies to full-range routed calls with fewer than 8 query heads per KV
// head: there the 128-key-block kernel's tiles (128/G tokens) walk much larger unions than
// the warp kernel's units (16/G tokens), and which costs less depends on the sparsity.
static bool attend_dynamic(const StageArgs &a) {
    return !a.ignore_routing && a.G < 8 && a.D == 128 && (a.Bc == 64 || a.Bc == 128) &&
           a.t_begin == 0 && a.t_end == a.T;
}

AttendKernel attend_kernel(const StageArgs &a) {
    if (a.t_begin != 0 || a.t_end != a.T) {
        // Row slices: only the 128-key-block kernels take a row range.
        if (a.vt && a.ignore_routing && attend_pair_supported(a)) return AttendKernel::kPair;
        if (a.vt && attend_fa_supported(a)) return AttendKernel::kFa;
        return AttendKernel::kNone;
    }
    // Pairs of SMs share each K/V block between two tiles, so they walk the union of both
    // tiles' chunks: a gain only when every visible chunk is attended anyway (dense, or every
    // chunk forced active); with routing the larger union costs more than the halved copies
    // save (measured at 128K: 128 ms against 117 ms).
    if (a.vt && a.ignore_routing && attend_pair_supported(a)) return AttendKernel::kPair;
    if (a.vt && attend_fa_supported(a)) return attend_dynamic(a) ? AttendKernel::kFaOrWarp : AttendKernel::kFa;
    if (attend_tc_supported(a)) return AttendKernel::kTc;
    if ((a.D == 128 || a.D == 64) && (a.Bc == 64 || a.Bc == 128)) return AttendKernel::kWarp;
    return AttendKernel::kNone;
}

const char *attend_kernel_name(AttendKernel k) {
    switch (k) {
        case AttendKernel::kPair: return "k_attend_pair";
        case AttendKernel::kFa: return "k_attend_fa";
        case AttendKernel::kTc: return "k_attend_tc";
        case AttendKernel::kWarp: return "k_attend";
        case AttendKernel::kFaOrWarp: return "k_attend_fa|k_attend";
        default: return "";
    }
}

static cudaError_t launch_warp(const StageArgs &a, cudaStream_t st) {
    if (a.D == 128 && a.Bc == 64) return launch_attend_t<128, 64>(a, st);
    if (a.D == 128 && a.Bc == 128) return launch_attend_t<128, 128>(a, st);
    if (a.D == 64 && a.Bc == 64) return launch_attend_t<64, 64>(a, st);
    if (a.D == 64 && a.Bc == 128) return launch_attend_t<64, 128>(a, st);
    return cudaErrorInvalidValue;
}

cudaError_t launch_attend(const StageArgs &a, cudaStream_t st) {
    switch (attend_kernel(a)) {
        case AttendKernel::kPair: return launch_attend_pair(a, st);
        case AttendKernel::kFa: return launch_attend_fa(a, st);
        case AttendKernel::kTc: return launch_attend_tc(a, st);
        case AttendKernel::kWarp: return launch_warp(a, st);
        case AttendKernel::kFaOrWarp: {
            // Costs from the mask, then both kernels; the one not chosen exits per CTA.
            unsigned char *blk = reinterpret_cast<unsigned char *>(a.status);
            unsigned long long *cost = reinterpret_cast<unsigned long long *>(blk + kStatusCostOff);
            cudaError_t e = cudaMemsetAsync(cost, 0, 2 * sizeof(unsigned long long), st);
            if (e != cudaSuccess) return e;
            const int RT = 128 / a.G;
            const int n_tiles_bg = (a.T + RT - 1) / RT;
            const long long tiles = (long long)n_tiles_bg * a.B * a.Hkv;
            if (tiles > 0) {
                k_union_cost<<<(unsigned)((tiles + 3) / 4), 128, 0, st>>>(a, cost, n_tiles_bg);
                if ((e = cudaGetLastError()) != cudaSuccess) return e;
            }
            StageArgs d = a;
            d.cost = cost;
            d.cost_ratio = (a.Bc == 64 ? kRateFa64 : kRateFa128) / kRateWarp;
            if ((e = launch_attend_fa(d, st)) != cudaSuccess) return e;
            return launch_warp(d, st);
        }
        default:
            return (a.t_begin != 0 || a.t_end != a.T) ? cudaErrorNotSupported : cudaErrorInvalidValue;
    }
}

}  // namespace dash
