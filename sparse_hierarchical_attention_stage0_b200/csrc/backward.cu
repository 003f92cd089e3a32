// backward.cu -- gradients of L = sum(O * dO) with respect to q, k, v and head_cls through
// Stages 2, 1 and 0 (dash_backward).
//
// gist.science "DashAttention: Differentiable and Adaptive Sparse Hierarchical Attention",
// Technische Zusammenfassung, "Stufe 1": alpha-entmax is differentiable, so gradients flow
// from the Stage 2 softmax through the routing decision back to the chunk summaries of
// Stage 0; liuzhao09.github.io "DashAttention 精读", section 2: the hierarchy trains end to
// end.  The chain rule, stage by stage (natural-log units; a_j the attention weights of row
// (h, t), O its output, delta = dO . O):
//   Stage 2:  dS_j = a_j (dO . v_j - delta);  dq = sum_j dS_j k_j / sqrt(D);
//             dk_j += dS_j q / sqrt(D);  dv_j += a_j dO;  d log p_c = sigma * sum_{j in c} dS_j
//             over the routed chunk's keys and the G heads of the token;
//   Stage 1:  with g_c = p_c^(2 - alpha) (p_c for alpha = 1) on the support,
//             ds_c = g_c dp_c - g_c (sum g dp) / (sum g),  dp_c = d log p_c / p_c;
//             dqbar = gamma / sqrt(D) sum_c ds_c S_c (each of the G heads gets dqbar / G);
//             dS_c = gamma / sqrt(D) sum_t ds_{t,c} qbar_t;
//   Stage 0:  w = softmax_j(hc . k_j / sqrt(D)), S_c = sum_j w_j k_j:
//             dk_j += w_j dS_c + dl_j hc / sqrt(D),  dl_j = w_j (k_j . dS_c - S_c . dS_c),
//             dhc += sum_j dl_j k_j / sqrt(D).
// Kernels (warp-level MMA, mma.sync m16n8k16, bf16 operands, fp32 accumulation):
//   k_bwd_q    query-stationary, one warp per 16 rows (a token's heads): the rows' softmax
//              statistics (pass 1), then dS, dq and d log p per routed chunk (pass 2);
//   k_bwd_lists  the routing transposed: per chunk, its routed tokens in token order;
//   k_bwd_kv   key-stationary, one CTA per chunk, one warp per 16 keys: dk and dv over the
//              chunk's diagonal tokens and its routed tokens (no atomics);
//   k_bwd_route  per row: the entmax Jacobian -> ds, dqbar added to dq;
//   k_bwd_dsum   per chunk: dS_c over its routed tokens;
//   k_bwd_stage0 per chunk: dk and dhc through the summary.
#include "attn_warp.cuh"

namespace dash {

namespace {

constexpr int kBwdWarps = 4;
constexpr int kBwdSlice = 1024;        // k_bwd_kv entries per CTA
constexpr int kListBlock = 2048;       // tokens per block of the routing transpose

struct BwdArgs {
    StageArgs s;                 // shapes, q, k, v, head_cls, summary, tau, mask, p (routing)
    const __nv_bfloat16 *dout;   // [B,Hq,T,D]
    const __nv_bfloat16 *out;    // [B,Hq,T,D] (the forward output)
    float *dq;                   // [B,Hq,T,D]
    float *dk, *dv;              // [B,Hkv,T,D]
    float *dhc;                  // [Hkv,D]
    float *dlogp;                // [B,Hkv,T,C]: d log p, then ds in place
    float *row_m, *row_l, *row_delta;   // [B,Hq,T] (row_m in log2 units)
    float *qbar;                 // [B,Hkv,T,D]
    int *list_cnt;               // [B*Hkv][C]
    long long *list_off;         // [B*Hkv][C + 1]
    int *blk_cnt;                // [B*Hkv][C][nblk]: routed tokens per (chunk, token block)
    long long *blk_off;          // [B*Hkv][C][nblk]
    int *list;                   // [B*Hkv][nnz_max]
    long long nnz_max;
    float *dsum;                 // [B,Hkv,Cf,D]
    float sigma;
};

// acc (16 x 16, two n-tiles of 8) = A (16 x D, fragments af) . Bt^T, Bt = 16 rows of a
// swizzled [rows][D] tile.
template <int D>
__device__ __forceinline__ void mm_16x16(float (&acc)[2][4], const uint32_t (&af)[D / 16][4],
                                         const unsigned char *bt) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[j][e] = 0.f;
#pragma unroll
        for (int kk = 0; kk < D / 16; kk += 2) {
            uint32_t r[4];
            ldsm_x4(r, bt + swz<D>(8 * j + (lane & 7), 2 * kk + (lane >> 3)));
            mma_bf16_16816(acc[j], af[kk], r[0], r[1]);
            mma_bf16_16816(acc[j], af[kk + 1], r[2], r[3]);
        }
    }
}

// A fragments (16 x D) of rows r0 .. r0 + 15 of a swizzled [rows][D] tile.
template <int D>
__device__ __forceinline__ void load_afrag(uint32_t (&af)[D / 16][4], const unsigned char *tile,
                                           int r0) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
        uint32_t r[4];
        // matrices: (rows 0-7, k 0-7), (rows 8-15, k 0-7), (rows 0-7, k 8-15), (rows 8-15, k 8-15)
        ldsm_x4(r, tile + swz<D>(r0 + (lane & 7) + 8 * ((lane >> 3) & 1), 2 * kk + (lane >> 4)));
        af[kk][0] = r[0];
        af[kk][1] = r[1];
        af[kk][2] = r[2];
        af[kk][3] = r[3];
    }
}

// acc[D/8][4] += A (16 x 16 bf16 fragments pa) . Btile (16 rows of k x D), Btile swizzled
// [rows][D] (row = k index).
template <int D>
__device__ __forceinline__ void mm_acc_kd(float (&acc)[D / 8][4], const uint32_t (&pa)[4],
                                          const unsigned char *bt) {
    const int lane = threadIdx.x & 31;
    const int mi = lane >> 3;
#pragma unroll
    for (int j = 0; j < D / 8; j += 2) {
        uint32_t r[4];
        ldsm_x4_t(r, bt + swz<D>((lane & 7) + 8 * (mi & 1), j + (mi >> 1)));
        mma_bf16_16816(acc[j], pa, r[0], r[1]);
        mma_bf16_16816(acc[j + 1], pa, r[2], r[3]);
    }
}

// Row-wise dot of bf16 rows a and b held at the fragment positions of this lane: the partial
// over dims {16 kk + 2 qd, +1, +8, +9}; reduced over the 4 lanes of the row.
template <int D>
__device__ __forceinline__ float row_dot_frag(const __nv_bfloat16 *a, const __nv_bfloat16 *b,
                                              bool ok) {
    const int qd = threadIdx.x & 3;
    float s = 0.f;
    if (ok) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            const int d0 = 16 * kk + 2 * qd;
            const float2 a0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(a + d0));
            const float2 b0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(b + d0));
            const float2 a1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(a + d0 + 8));
            const float2 b1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(b + d0 + 8));
            s = fmaf(a0.x, b0.x, s);
            s = fmaf(a0.y, b0.y, s);
            s = fmaf(a1.x, b1.x, s);
            s = fmaf(a1.y, b1.y, s);
        }
    }
    s += __shfl_xor_sync(kFull, s, 1);
    s += __shfl_xor_sync(kFull, s, 2);
    return s;
}

// ---------------------------------------------------------------- k_bwd_q
template <int D, int BC>
__global__ void __launch_bounds__(kBwdWarps * 32) k_bwd_q(BwdArgs ba, int TU, int UPT,
                                                          long long n_units) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    const StageArgs &a = ba.s;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long unit = (long long)blockIdx.x * kBwdWarps + warp;
    if (unit >= n_units) return;
    // Per warp: a K and a V tile, and the routing biases of the current batch of chunks.
    const size_t tile_bytes = (size_t)kSub * D * 2;
    const size_t warp_bytes = 2 * tile_bytes + (size_t)TU * 32 * 4;
    unsigned char *base = smem_raw + warp * warp_bytes;
    unsigned char *ks = base, *vs = base + tile_bytes;
    float *bias_s = reinterpret_cast<float *>(base + 2 * tile_bytes);

    const int G = a.G, Gu = G >= 16 ? 16 : G;
    const int kunit = (int)(unit % UPT);
    long long rest = unit / UPT;
    const int g = (int)(rest % a.Hkv);
    rest /= a.Hkv;
    const int b = (int)(rest % a.B);
    const int tg = (int)(rest / a.B);
    const int t0 = tg * TU;
    const int ct = t0 / BC;
    const long long bg = (long long)b * a.Hkv + g;
    const __nv_bfloat16 *q = reinterpret_cast<const __nv_bfloat16 *>(a.q);
    const __nv_bfloat16 *kp = reinterpret_cast<const __nv_bfloat16 *>(a.k) + bg * a.T * D;
    const __nv_bfloat16 *vp = reinterpret_cast<const __nv_bfloat16 *>(a.v) + bg * a.T * D;

    const int r_lo = lane >> 2, r_hi = r_lo + 8, qd = lane & 3;
    const int tok_lo = t0 + r_lo / Gu, tok_hi = t0 + r_hi / Gu;
    const int head_lo = g * G + kunit * 16 + r_lo % Gu, head_hi = g * G + kunit * 16 + r_hi % Gu;
    const bool ok_lo = tok_lo < a.T && r_lo < TU * Gu, ok_hi = tok_hi < a.T && r_hi < TU * Gu;
    const long long row_lo = ((long long)b * a.Hq + head_lo) * a.T + (ok_lo ? tok_lo : 0);
    const long long row_hi = ((long long)b * a.Hq + head_hi) * a.T + (ok_hi ? tok_hi : 0);

    uint32_t qf[D / 16][4], df[D / 16][4];
    {
        const __nv_bfloat16 *q_lo = q + row_lo * D, *q_hi = q + row_hi * D;
        const __nv_bfloat16 *d_lo = ba.dout + row_lo * D, *d_hi = ba.dout + row_hi * D;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            const int d0 = 16 * kk + 2 * qd;
            qf[kk][0] = ok_lo ? *reinterpret_cast<const uint32_t *>(q_lo + d0) : 0u;
            qf[kk][1] = ok_hi ? *reinterpret_cast<const uint32_t *>(q_hi + d0) : 0u;
            qf[kk][2] = ok_lo ? *reinterpret_cast<const uint32_t *>(q_lo + d0 + 8) : 0u;
            qf[kk][3] = ok_hi ? *reinterpret_cast<const uint32_t *>(q_hi + d0 + 8) : 0u;
            df[kk][0] = ok_lo ? *reinterpret_cast<const uint32_t *>(d_lo + d0) : 0u;
            df[kk][1] = ok_hi ? *reinterpret_cast<const uint32_t *>(d_hi + d0) : 0u;
            df[kk][2] = ok_lo ? *reinterpret_cast<const uint32_t *>(d_lo + d0 + 8) : 0u;
            df[kk][3] = ok_hi ? *reinterpret_cast<const uint32_t *>(d_hi + d0 + 8) : 0u;
        }
    }
    const float delta_lo = row_dot_frag<D>(ba.dout + row_lo * D, ba.out + row_lo * D, ok_lo);
    const float delta_hi = row_dot_frag<D>(ba.dout + row_hi * D, ba.out + row_hi * D, ok_hi);

    const bool route = ct > 0;
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
            if (kunit == 0 && t < a.T)
#pragma unroll
                for (int e = 0; e < 8; ++e) ba.qbar[(bg * a.T + t) * D + d8 + e] = m[e];
        }
    }
    __syncwarp();

    const int wmax = ct > 0 ? (ct - 1) >> 6 : -1;
    auto load_word = [&](int w) -> uint64_t {
        uint64_t word = 0;
        for (int u = 0; u < TU; ++u) {
            const int t = t0 + u;
            if (t < a.T) word |= a.mask[(bg * a.T + t) * a.W + w];
        }
        const int lim = ct - 64 * w;
        if (lim < 64) word &= (1ull << lim) - 1ull;
        return word;
    };
    constexpr int NSUB = BC / kSub;
    float m_lo = -INFINITY, m_hi = -INFINITY, l_lo = 0.f, l_hi = 0.f;
    float dqa[D / 8][4];
#pragma unroll
    for (int j = 0; j < D / 8; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) dqa[j][e] = 0.f;

    // Two passes over the unit's chunks (routed in ascending order, then the diagonal).
    for (int pass = 0; pass < 2; ++pass) {
        int w_cur = 0;
        uint64_t bits = wmax >= 0 ? load_word(0) : 0ull;
        bool diag_pending = true;
        if (pass == 1) {
            // Final statistics: the row maximum and the sum of 2^(x - m) over the row.
            l_lo += __shfl_xor_sync(kFull, l_lo, 1);
            l_lo += __shfl_xor_sync(kFull, l_lo, 2);
            l_hi += __shfl_xor_sync(kFull, l_hi, 1);
            l_hi += __shfl_xor_sync(kFull, l_hi, 2);
            if (qd == 0) {
                if (ok_lo) { ba.row_m[row_lo] = m_lo; ba.row_l[row_lo] = l_lo; ba.row_delta[row_lo] = delta_lo; }
                if (ok_hi) { ba.row_m[row_hi] = m_hi; ba.row_l[row_hi] = l_hi; ba.row_delta[row_hi] = delta_hi; }
            }
        }
        const float il_lo = l_lo > 0.f ? 1.f / l_lo : 0.f, il_hi = l_hi > 0.f ? 1.f / l_hi : 0.f;
        while (true) {
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
            const int n_routed = batch_has_diag ? nb - 1 : nb;
            if (lane < n_routed) {
                // bias = sigma log p of the token's routing (-inf where the token's p is 0:
                // a chunk of the union the token itself did not route to)
                for (int u = 0; u < TU; ++u) {
                    const int t = t0 + u;
                    bias_s[u * 32 + lane] =
                        t < a.T ? ba.sigma * log2f(a.p[(bg * a.T + t) * a.C + my_c]) : -INFINITY;
                }
            }
            __syncwarp();
            float dlp[16];                           // d log p of this batch's chunk i, per token
            for (int s = 0; s < nb * NSUB; ++s) {
                const int i = s / NSUB, sb = s % NSUB;
                const int c = __shfl_sync(kFull, my_c, i);
                const bool diag = c == ct;
                const int key0 = c * BC + sb * kSub;
                load_sub<D>(ks, kp, key0, a.T);
                if (pass == 1) load_sub<D>(vs, vp, key0, a.T);
                cp_async_commit();
                cp_async_wait<0>();
                __syncwarp();
                float b_lo = 0.f, b_hi = 0.f;
                if (!diag) {
                    b_lo = bias_s[((r_lo / Gu) % TU) * 32 + i];
                    b_hi = bias_s[((r_hi / Gu) % TU) * 32 + i];
                }
                float acc[4][4];
                qk_sub<D>(acc, qf, ks);
                // logits in log2 units, masked keys -inf
#pragma unroll
                for (int j = 0; j < 4; ++j)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const bool hi = e >= 2;
                        const int key = key0 + 8 * j + 2 * qd + (e & 1);
                        float v = fmaf(acc[j][e], a.qk_scale2, hi ? b_hi : b_lo);
                        if ((diag && key > (hi ? tok_hi : tok_lo)) || key >= a.T || !(hi ? ok_hi : ok_lo))
                            v = -INFINITY;
                        acc[j][e] = v;
                    }
                if (pass == 0) {
                    float mx_lo = -INFINITY, mx_hi = -INFINITY;
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        mx_lo = fmaxf(mx_lo, fmaxf(acc[j][0], acc[j][1]));
                        mx_hi = fmaxf(mx_hi, fmaxf(acc[j][2], acc[j][3]));
                    }
                    mx_lo = fmaxf(mx_lo, __shfl_xor_sync(kFull, mx_lo, 1));
                    mx_lo = fmaxf(mx_lo, __shfl_xor_sync(kFull, mx_lo, 2));
                    mx_hi = fmaxf(mx_hi, __shfl_xor_sync(kFull, mx_hi, 1));
                    mx_hi = fmaxf(mx_hi, __shfl_xor_sync(kFull, mx_hi, 2));
                    const float mn_lo = fmaxf(m_lo, mx_lo), mn_hi = fmaxf(m_hi, mx_hi);
                    const float mu_lo = mn_lo == -INFINITY ? 0.f : mn_lo, mu_hi = mn_hi == -INFINITY ? 0.f : mn_hi;
                    l_lo *= exp2f(m_lo - mu_lo);
                    l_hi *= exp2f(m_hi - mu_hi);
                    m_lo = mn_lo;
                    m_hi = mn_hi;
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        l_lo += exp2f(acc[j][0] - mu_lo) + exp2f(acc[j][1] - mu_lo);
                        l_hi += exp2f(acc[j][2] - mu_hi) + exp2f(acc[j][3] - mu_hi);
                    }
                    __syncwarp();
                    continue;
                }
                // pass 1: P, dP = dO V^T, dS = P (dP - delta); dq += dS K; d log p
                float dp[4][4];
                qk_sub<D>(dp, df, vs);
                float s_lo = 0.f, s_hi = 0.f;
                uint32_t dsa[2][4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    // masked keys (-inf) weigh nothing, also in rows with no key at all
                    const float p0 = acc[j][0] == -INFINITY ? 0.f : exp2f(acc[j][0] - m_lo) * il_lo;
                    const float p1 = acc[j][1] == -INFINITY ? 0.f : exp2f(acc[j][1] - m_lo) * il_lo;
                    const float p2 = acc[j][2] == -INFINITY ? 0.f : exp2f(acc[j][2] - m_hi) * il_hi;
                    const float p3 = acc[j][3] == -INFINITY ? 0.f : exp2f(acc[j][3] - m_hi) * il_hi;
                    acc[j][0] = p0 * (dp[j][0] - delta_lo);
                    acc[j][1] = p1 * (dp[j][1] - delta_lo);
                    acc[j][2] = p2 * (dp[j][2] - delta_hi);
                    acc[j][3] = p3 * (dp[j][3] - delta_hi);
                    s_lo += acc[j][0] + acc[j][1];
                    s_hi += acc[j][2] + acc[j][3];
                }
#pragma unroll
                for (int kk = 0; kk < 2; ++kk) {
                    dsa[kk][0] = pack_bf16x2(acc[2 * kk][0], acc[2 * kk][1]);
                    dsa[kk][1] = pack_bf16x2(acc[2 * kk][2], acc[2 * kk][3]);
                    dsa[kk][2] = pack_bf16x2(acc[2 * kk + 1][0], acc[2 * kk + 1][1]);
                    dsa[kk][3] = pack_bf16x2(acc[2 * kk + 1][2], acc[2 * kk + 1][3]);
                }
                // dq += dS K (K as the [keys][D] operand of the P V form)
#pragma unroll
                for (int kk = 0; kk < 2; ++kk) {
                    const int mi = lane >> 3;
#pragma unroll
                    for (int j = 0; j < D / 8; j += 2) {
                        uint32_t r[4];
                        ldsm_x4_t(r, ks + swz<D>(16 * kk + (lane & 7) + 8 * (mi & 1), j + (mi >> 1)));
                        mma_bf16_16816(dqa[j], dsa[kk], r[0], r[1]);
                        mma_bf16_16816(dqa[j + 1], dsa[kk], r[2], r[3]);
                    }
                }
                if (!diag) {
                    // d log p of chunk c per token: the sum of dS over the token's rows and keys
                    for (int u = 0; u < TU; ++u) {
                        float v = ((r_lo / Gu) == u ? s_lo : 0.f) + ((r_hi / Gu) == u ? s_hi : 0.f);
                        v = warp_sum(v);
                        if (sb == 0) dlp[u] = v; else dlp[u] += v;
                    }
                    if (sb == NSUB - 1 && lane == 0) {
                        for (int u = 0; u < TU; ++u) {
                            const int t = t0 + u;
                            if (t >= a.T) continue;
                            const long long idx = (bg * a.T + t) * a.C + c;
                            if (UPT > 1) atomicAdd(&ba.dlogp[idx], ba.sigma * dlp[u]);
                            else ba.dlogp[idx] = ba.sigma * dlp[u];
                        }
                    }
                }
                __syncwarp();
            }
            __syncwarp();
        }
    }
    // dq (natural units): sum_j dS_j k_j / sqrt(D)
    const float rs = a.qk_scale2 * 0.69314718055994531f;   // 1 / sqrt(D)
#pragma unroll
    for (int j = 0; j < D / 8; ++j) {
        const int d0 = 8 * j + 2 * qd;
        if (ok_lo) {
            ba.dq[row_lo * D + d0] = dqa[j][0] * rs;
            ba.dq[row_lo * D + d0 + 1] = dqa[j][1] * rs;
        }
        if (ok_hi) {
            ba.dq[row_hi * D + d0] = dqa[j][2] * rs;
            ba.dq[row_hi * D + d0 + 1] = dqa[j][3] * rs;
        }
    }
}

// ---------------------------------------------------------------- k_bwd_lists
// Per (b, g), mask word w and block of kListBlock tokens: the block's routed tokens of chunks
// 64 w .. 64 w + 63 (the diagonal bit excluded), in token order.  mode 0 counts them into
// blk_cnt[(bg C + c) nblk + blk]; mode 1 writes them from blk_off (the same index).  One warp
// per (b, g, w, block), 32 tokens per step; chunks of word w are routed to only by tokens from
// 64 w Bc on, so earlier blocks have nothing to do.
__global__ void k_bwd_lists(BwdArgs ba, int mode, int nblk) {
    const StageArgs &a = ba.s;
    const int lane = threadIdx.x & 31;
    const int w = blockIdx.x, bgi = blockIdx.y, blk = blockIdx.z;
    const long long bg = bgi;
    int run_lo = 0, run_hi = 0;                  // per chunk 64 w + lane and 64 w + 32 + lane
    const int c_lo = 64 * w + lane, c_hi = c_lo + 32;
    const int t_begin = max(blk * kListBlock, 64 * w * a.Bc), t_end = min(a.T, (blk + 1) * kListBlock);
    for (int t0 = t_begin; t0 < t_end; t0 += 32) {
        const int t = t0 + lane;
        uint64_t word = 0;
        if (t < t_end) {
            word = a.mask[(bg * a.T + t) * a.W + w];
            const int ct = t / a.Bc;
            if (ct / 64 == w) word &= ~(1ull << (ct & 63));
        }
        for (int bit = 0; bit < 64; ++bit) {
            const unsigned bal = __ballot_sync(kFull, (word >> bit) & 1ull);
            if (!bal) continue;
            const int c = 64 * w + bit;
            // The chunk's running count sits on lane bit % 32; every lane takes part in the
            // shuffle, whether or not its token routes to the chunk.
            const int run_c = bit < 32 ? __shfl_sync(kFull, run_lo, bit) : __shfl_sync(kFull, run_hi, bit - 32);
            if (mode == 1 && ((word >> bit) & 1ull)) {
                const int before = run_c + __popc(bal & ((1u << lane) - 1u));
                const long long pos = ba.blk_off[(bg * a.C + c) * nblk + blk] + before;
                if (pos >= 0 && pos < ba.nnz_max) ba.list[bg * ba.nnz_max + pos] = t;
                else report(a.status, DASH_ERR_BOUNDS);
            }
            if (lane == (bit & 31)) {
                if (bit < 32) run_lo += __popc(bal); else run_hi += __popc(bal);
            }
        }
    }
    if (mode == 0) {
        if (c_lo < a.C) ba.blk_cnt[(bg * a.C + c_lo) * nblk + blk] = run_lo;
        if (c_hi < a.C) ba.blk_cnt[(bg * a.C + c_hi) * nblk + blk] = run_hi;
    }
}

// Exclusive prefix sum per (b, g) over (chunk, block) in chunk-major order into blk_off, and
// per chunk its count (list_cnt) and first offset (list_off).  One warp per (b, g).
__global__ void k_bwd_scan(BwdArgs ba, int nblk) {
    const StageArgs &a = ba.s;
    const int lane = threadIdx.x & 31;
    const long long bg = blockIdx.x;
    const long long n = (long long)a.C * nblk;
    long long base = 0;
    for (long long i0 = 0; i0 < n; i0 += 32) {
        const long long i = i0 + lane;
        const int v = i < n ? ba.blk_cnt[bg * n + i] : 0;
        int incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int x = __shfl_up_sync(kFull, incl, o);
            if (lane >= o) incl += x;
        }
        if (i < n) ba.blk_off[bg * n + i] = base + incl - v;
        base += __shfl_sync(kFull, incl, 31);
    }
    __syncwarp();
    for (int c = lane; c < a.C; c += 32) {
        const long long first = ba.blk_off[bg * n + (long long)c * nblk];
        const long long next = c + 1 < a.C ? ba.blk_off[bg * n + (long long)(c + 1) * nblk] : base;
        ba.list_off[bg * (a.C + 1) + c] = first;
        ba.list_cnt[bg * a.C + c] = (int)(next - first);
    }
    if (lane == 0) ba.list_off[bg * (a.C + 1) + a.C] = base;
}

// ---------------------------------------------------------------- k_bwd_kv
// One CTA per (b, g, chunk c, slice of kBwdSlice entries), BC / 16 warps (warp w: keys
// c BC + 16 w .. + 15).  Entries are (token, group of up to 16 heads): the chunk's own tokens
// (diagonal, bias 0, causal), then its routed tokens (bias = sigma log p); the first chunks of
// a long sequence are routed to by up to a quarter of it, so each CTA takes one slice of
// the entries and adds its partial dk, dv into memory (zeroed first).  Per entry, each warp
// computes S^T = K_w Q^T, P^T, dP^T = V_w dO^T, dS^T and accumulates dv += P^T dO,
// dk += dS^T Q in registers.
template <int D, int BC>
__global__ void __launch_bounds__(BC / 16 * 32) k_bwd_kv(BwdArgs ba, int UPT) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    const StageArgs &a = ba.s;
    constexpr int NW = BC / 16;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
    const int c = blockIdx.x;
    const long long bg = blockIdx.y;
    const int b = (int)(bg / a.Hkv), g = (int)(bg % a.Hkv);
    const int G = a.G, Gu = G >= 16 ? 16 : G;
    unsigned char *kt = smem_raw;                             // [BC][D] bf16
    unsigned char *vt = kt + (size_t)BC * D * 2;              // [BC][D]
    // Two buffers per entry (the next entry's rows and statistics are copied while this one
    // is computed): q rows [16][D], dO rows [16][D], and per row m, l, delta, then the bias p.
    unsigned char *qt0 = vt + (size_t)BC * D * 2;
    unsigned char *ot0 = qt0 + (size_t)2 * 16 * D * 2;
    float *st0 = reinterpret_cast<float *>(ot0 + (size_t)2 * 16 * D * 2);   // [2][52]
    const __nv_bfloat16 *kp = reinterpret_cast<const __nv_bfloat16 *>(a.k) + bg * a.T * D;
    const __nv_bfloat16 *vp = reinterpret_cast<const __nv_bfloat16 *>(a.v) + bg * a.T * D;
    const __nv_bfloat16 *q = reinterpret_cast<const __nv_bfloat16 *>(a.q);
    const int n_diag = min(BC, a.T - c * BC);
    const long long n_routed = c < a.Cf ? ba.list_cnt[bg * a.C + c] : 0;
    const long long off = c < a.Cf ? ba.list_off[bg * (a.C + 1) + c] : 0;
    const long long n_entries = ((long long)n_diag + n_routed) * UPT;
    const long long e_begin = (long long)blockIdx.z * kBwdSlice;
    const long long e_end = min(n_entries, e_begin + kBwdSlice);
    if (e_begin >= n_entries) return;                        // the same in every thread
    constexpr int CH = D / 8;
    for (int i = tid; i < BC * CH; i += NW * 32) {
        const int row = i / CH, ch = i % CH, key = c * BC + row;
        const bool ok = key < a.T;
        cp_async16(kt + swz<D>(row, ch), kp + (long long)(ok ? key : 0) * D + ch * 8, ok ? 16 : 0);
        cp_async16(vt + swz<D>(row, ch), vp + (long long)(ok ? key : 0) * D + ch * 8, ok ? 16 : 0);
    }
    cp_async_commit();
    float dka[D / 8][4], dva[D / 8][4];
#pragma unroll
    for (int j = 0; j < D / 8; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) dka[j][e] = dva[j][e] = 0.f;
    const int r_lo = lane >> 2, qd = lane & 3;                // key rows r_lo, r_lo + 8 of the warp
    const int key_lo = c * BC + 16 * warp + r_lo, key_hi = key_lo + 8;

    // Entry e: token t (the chunk's own tokens first, then its routed ones) and head group.
    struct Ent { int t, kunit; bool diag, valid; };
    auto entry = [&](long long e) -> Ent {
        Ent en;
        const long long ti = e / UPT;
        en.kunit = (int)(e % UPT);
        en.diag = ti < n_diag;
        en.t = en.diag ? c * BC + (int)ti : ba.list[bg * ba.nnz_max + off + (ti - n_diag)];
        en.valid = en.t >= 0 && en.t < a.T;
        return en;
    };
    // Copies of an entry's rows and statistics into buffer buf; every thread commits one group.
    auto prefetch = [&](const Ent &en, int buf) {
        if (en.valid) {
            unsigned char *qt = qt0 + (size_t)buf * 16 * D * 2, *ot = ot0 + (size_t)buf * 16 * D * 2;
            float *st = st0 + buf * 52;
            for (int i = tid; i < 16 * CH; i += NW * 32) {
                const int r = i / CH, ch = i % CH;
                const bool ok = r < Gu;
                const long long row = ((long long)b * a.Hq + g * G + en.kunit * 16 + (ok ? r : 0)) * a.T + en.t;
                cp_async16(qt + swz<D>(r, ch), q + row * D + ch * 8, ok ? 16 : 0);
                cp_async16(ot + swz<D>(r, ch), ba.dout + row * D + ch * 8, ok ? 16 : 0);
            }
            if (tid < Gu) {
                const long long row = ((long long)b * a.Hq + g * G + en.kunit * 16 + tid) * a.T + en.t;
                cp_async4(st + tid, ba.row_m + row);
                cp_async4(st + 16 + tid, ba.row_l + row);
                cp_async4(st + 32 + tid, ba.row_delta + row);
            }
            // the routing bias of a routed entry is sigma log p (p > 0 on the routed chunks)
            if (tid == 0 && !en.diag) cp_async4(st + 48, a.p + (bg * a.T + en.t) * a.C + c);
        }
        cp_async_commit();
    };
    Ent cur = entry(e_begin);
    prefetch(cur, 0);
    for (long long e = e_begin; e < e_end; ++e) {
        const int buf = (int)((e - e_begin) & 1);
        const Ent nxt = e + 1 < e_end ? entry(e + 1) : Ent{0, 0, false, false};
        __syncthreads();                                     // entry e-1's buffer is read
        prefetch(nxt, buf ^ 1);
        cp_async_wait<1>();                                  // entry e's copies (and K, V)
        __syncthreads();
        if (!cur.valid) {                                    // same entry in every thread
            if (tid == 0) report(a.status, DASH_ERR_BOUNDS);
            cur = nxt;
            continue;
        }
        const int t = cur.t;
        const bool diag = cur.diag;
        const unsigned char *qt = qt0 + (size_t)buf * 16 * D * 2, *ot = ot0 + (size_t)buf * 16 * D * 2;
        const float *st = st0 + buf * 52;
        const float b2 = diag ? 0.f : ba.sigma * log2f(st[48]);
        // S^T (16 keys x 16 rows) in log2 units, P^T, dP^T, dS^T
        float sa[2][4], dpa[2][4];
        {
            uint32_t af[D / 16][4];
            load_afrag<D>(af, kt, 16 * warp);                // this warp's 16 keys
            mm_16x16<D>(sa, af, qt);
            load_afrag<D>(af, vt, 16 * warp);
            mm_16x16<D>(dpa, af, ot);
        }
        uint32_t pa[4], dsa[4];
        float pv[2][4], dsv[2][4];
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int e2 = 0; e2 < 4; ++e2) {
                const int r = 8 * j + 2 * qd + (e2 & 1);          // row (head) of the entry
                const int key = e2 >= 2 ? key_hi : key_lo;
                float x = fmaf(sa[j][e2], a.qk_scale2, b2);
                if ((diag && key > t) || key >= a.T || r >= Gu) x = -INFINITY;
                const float l = st[16 + r];
                const float p = x == -INFINITY ? 0.f : exp2f(x - st[r]) * (l > 0.f ? 1.f / l : 0.f);
                pv[j][e2] = p;
                dsv[j][e2] = p * (dpa[j][e2] - st[32 + r]);
            }
        // C fragments (rows = keys, cols = entry rows) -> A fragments of the 16 x 16 P^T, dS^T
        pa[0] = pack_bf16x2(pv[0][0], pv[0][1]);
        pa[1] = pack_bf16x2(pv[0][2], pv[0][3]);
        pa[2] = pack_bf16x2(pv[1][0], pv[1][1]);
        pa[3] = pack_bf16x2(pv[1][2], pv[1][3]);
        dsa[0] = pack_bf16x2(dsv[0][0], dsv[0][1]);
        dsa[1] = pack_bf16x2(dsv[0][2], dsv[0][3]);
        dsa[2] = pack_bf16x2(dsv[1][0], dsv[1][1]);
        dsa[3] = pack_bf16x2(dsv[1][2], dsv[1][3]);
        mm_acc_kd<D>(dva, pa, ot);
        mm_acc_kd<D>(dka, dsa, qt);
        cur = nxt;
    }
    const float rs = a.qk_scale2 * 0.69314718055994531f;
#pragma unroll
    for (int j = 0; j < D / 8; ++j) {
        const int d0 = 8 * j + 2 * qd;
        if (key_lo < a.T) {
            const long long o = (bg * a.T + key_lo) * D + d0;
            atomicAdd(&ba.dk[o], dka[j][0] * rs);
            atomicAdd(&ba.dk[o + 1], dka[j][1] * rs);
            atomicAdd(&ba.dv[o], dva[j][0]);
            atomicAdd(&ba.dv[o + 1], dva[j][1]);
        }
        if (key_hi < a.T) {
            const long long o = (bg * a.T + key_hi) * D + d0;
            atomicAdd(&ba.dk[o], dka[j][2] * rs);
            atomicAdd(&ba.dk[o + 1], dka[j][3] * rs);
            atomicAdd(&ba.dv[o], dva[j][2]);
            atomicAdd(&ba.dv[o + 1], dva[j][3]);
        }
    }
}

// ---------------------------------------------------------------- k_bwd_route
// One warp per (b, g, t) with c_t >= 1: ds = the entmax Jacobian applied to dp = d log p / p
// (in place over dlogp), dqbar = gamma / sqrt(D) sum_c ds_c S_c added (/ G) to the G heads'
// dq rows.
template <int D>
__global__ void __launch_bounds__(128) k_bwd_route(BwdArgs ba) {
    const StageArgs &a = ba.s;
    const int lane = threadIdx.x & 31;
    const long long unit = (long long)blockIdx.x * 4 + (threadIdx.x >> 5);
    if (unit >= (long long)a.B * a.Hkv * a.T) return;
    const long long bg = unit / a.T;
    const int t = (int)(unit % a.T), ct = t / a.Bc;
    const int b = (int)(bg / a.Hkv), g = (int)(bg % a.Hkv);
    if (ct == 0) return;
    const float *p = a.p + unit * a.C;
    float *dl = ba.dlogp + unit * a.C;
    const float alpha = a.rc.alpha;
    float sg = 0.f, sgdp = 0.f;
    for (int c = lane; c < ct; c += 32) {
        const float pc = p[c];
        if (pc > 0.f) {
            const float gc = a.rc.kind == 0 ? pc : a.rc.kind == 1 ? sqrtf(pc) : a.rc.kind == 2 ? 1.f : powf(pc, 2.f - alpha);
            sg += gc;
            sgdp += gc * dl[c] / pc;
        }
    }
    sg = warp_sum(sg);
    sgdp = warp_sum(sgdp);
    const float corr = sg > 0.f ? sgdp / sg : 0.f;
    for (int c = lane; c < ct; c += 32) {
        const float pc = p[c];
        float ds = 0.f;
        if (pc > 0.f) {
            const float gc = a.rc.kind == 0 ? pc : a.rc.kind == 1 ? sqrtf(pc) : a.rc.kind == 2 ? 1.f : powf(pc, 2.f - alpha);
            ds = gc * (dl[c] / pc - corr);
        }
        dl[c] = ds;
    }
    __syncwarp();
    // dqbar over the support, lanes over D
    const float sc = a.rc.sscale;                            // gamma / sqrt(D)
    float dqb[D / 32];
#pragma unroll
    for (int i = 0; i < D / 32; ++i) dqb[i] = 0.f;
    const float *sumg = a.summary + bg * a.Cf * D;
    for (int c = 0; c < ct; ++c) {
        const float ds = dl[c];
        if (ds == 0.f) continue;
#pragma unroll
        for (int i = 0; i < D / 32; ++i) dqb[i] = fmaf(ds, sumg[(long long)c * D + lane + 32 * i], dqb[i]);
    }
    for (int h = g * a.G; h < (g + 1) * a.G; ++h) {
        float *dqr = ba.dq + (((long long)b * a.Hq + h) * a.T + t) * D;
#pragma unroll
        for (int i = 0; i < D / 32; ++i) dqr[lane + 32 * i] += dqb[i] * sc / (float)a.G;
    }
}

// ---------------------------------------------------------------- k_bwd_dsum
// One warp per (b, g, c < Cf): dS_c = gamma / sqrt(D) sum over its routed tokens of ds qbar.
template <int D>
__global__ void __launch_bounds__(128) k_bwd_dsum(BwdArgs ba) {
    const StageArgs &a = ba.s;
    const int lane = threadIdx.x & 31;
    const long long unit = (long long)blockIdx.x * 4 + (threadIdx.x >> 5);
    if (unit >= (long long)a.B * a.Hkv * a.Cf) return;
    const long long bg = unit / a.Cf;
    const int c = (int)(unit % a.Cf);
    const long long n = ba.list_cnt[bg * a.C + c], off = ba.list_off[bg * (a.C + 1) + c];
    float acc[D / 32];
#pragma unroll
    for (int i = 0; i < D / 32; ++i) acc[i] = 0.f;
    for (long long e = 0; e < n; ++e) {
        const int t = ba.list[bg * ba.nnz_max + off + e];
        if (t < 0 || t >= a.T) {
            if (lane == 0) report(a.status, DASH_ERR_BOUNDS);
            continue;
        }
        const float ds = ba.dlogp[(bg * a.T + t) * a.C + c];
        const float *qb = ba.qbar + (bg * a.T + t) * D;
#pragma unroll
        for (int i = 0; i < D / 32; ++i) acc[i] = fmaf(ds, qb[lane + 32 * i], acc[i]);
    }
    float *o = ba.dsum + unit * D;
#pragma unroll
    for (int i = 0; i < D / 32; ++i) o[lane + 32 * i] = acc[i] * a.rc.sscale;
}

// ---------------------------------------------------------------- k_bwd_stage0
// One warp per (b, g, c < Cf): the summary's gradient dS_c to the chunk's keys and to head_cls.
template <int D, int BC>
__global__ void __launch_bounds__(128) k_bwd_stage0(BwdArgs ba) {
    const StageArgs &a = ba.s;
    const int lane = threadIdx.x & 31;
    const long long unit = (long long)blockIdx.x * 4 + (threadIdx.x >> 5);
    if (unit >= (long long)a.B * a.Hkv * a.Cf) return;
    const long long bg = unit / a.Cf;
    const int c = (int)(unit % a.Cf), g = (int)(bg % a.Hkv);
    const __nv_bfloat16 *kc = reinterpret_cast<const __nv_bfloat16 *>(a.k) + (bg * a.T + (long long)c * BC) * D;
    const float *hc = a.head_cls + (long long)g * D;
    const float *dS = ba.dsum + unit * D, *S = a.summary + unit * D;
    const float rs = a.rc.inv_sqrt_d;
    constexpr int KPL = BC / 32;                              // keys per lane
    float w[KPL], kd[KPL];
    float mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < KPL; ++i) {
        const __nv_bfloat16 *kr = kc + (long long)(lane + 32 * i) * D;
        float l = 0.f, x = 0.f;
        for (int d = 0; d < D; ++d) {
            const float kv = __bfloat162float(kr[d]);
            l = fmaf(hc[d], kv, l);
            x = fmaf(kv, dS[d], x);
        }
        w[i] = l * rs;
        kd[i] = x;
        mx = fmaxf(mx, w[i]);
    }
    mx = warp_max(mx);
    float den = 0.f;
#pragma unroll
    for (int i = 0; i < KPL; ++i) {
        w[i] = expf(w[i] - mx);
        den += w[i];
    }
    den = warp_sum(den);
    float sds = 0.f;
    for (int d = lane; d < D; d += 32) sds = fmaf(S[d], dS[d], sds);
    sds = warp_sum(sds);
    float dl[KPL];
#pragma unroll
    for (int i = 0; i < KPL; ++i) {
        w[i] /= den;
        dl[i] = w[i] * (kd[i] - sds);
    }
    // dk rows of this lane's keys
#pragma unroll
    for (int i = 0; i < KPL; ++i) {
        float *dkr = ba.dk + (bg * a.T + (long long)c * BC + lane + 32 * i) * D;
        for (int d = 0; d < D; ++d) dkr[d] += w[i] * dS[d] + dl[i] * hc[d] * rs;
    }
    // dhc: lanes over d, keys broadcast
    float acc[D / 32];
#pragma unroll
    for (int i = 0; i < D / 32; ++i) acc[i] = 0.f;
    for (int j = 0; j < BC; ++j) {
        const float dlj = __shfl_sync(kFull, dl[j / 32 < KPL ? j / 32 : 0], j % 32);
        const __nv_bfloat16 *kr = kc + (long long)j * D;
#pragma unroll
        for (int i = 0; i < D / 32; ++i) acc[i] = fmaf(dlj, __bfloat162float(kr[lane + 32 * i]), acc[i]);
    }
#pragma unroll
    for (int i = 0; i < D / 32; ++i) atomicAdd(&ba.dhc[(long long)g * D + lane + 32 * i], acc[i] * rs);
}

template <int D, int BC>
cudaError_t launch_bwd_t(BwdArgs ba, cudaStream_t st) {
    const StageArgs &a = ba.s;
    const int G = a.G;
    const int TU = G >= 16 ? 1 : 16 / G;
    const int UPT = G >= 16 ? G / 16 : 1;
    cudaError_t e;
    // 1. query side
    {
        const long long NTG = (a.T + TU - 1) / TU;
        const long long n_units = NTG * a.B * a.Hkv * UPT;
        const size_t warp_bytes = 2 * (size_t)kSub * D * 2 + (size_t)TU * 32 * 4;
        const size_t smem = warp_bytes * kBwdWarps;
        auto kern = k_bwd_q<D, BC>;
        if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess) return e;
        kern<<<(unsigned)((n_units + kBwdWarps - 1) / kBwdWarps), kBwdWarps * 32, smem, st>>>(ba, TU, UPT, n_units);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    // 2. the routing transposed
    {
        const int nblk = backward_list_blocks(a.T);
        dim3 grid((unsigned)a.W, (unsigned)(a.B * a.Hkv), (unsigned)nblk);
        k_bwd_lists<<<grid, 32, 0, st>>>(ba, 0, nblk);
        k_bwd_scan<<<(unsigned)(a.B * a.Hkv), 32, 0, st>>>(ba, nblk);
        k_bwd_lists<<<grid, 32, 0, st>>>(ba, 1, nblk);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    // 3. key side
    {
        const size_t smem = 2 * (size_t)BC * D * 2 + 4 * (size_t)16 * D * 2 + 2 * 52 * 4;
        auto kern = k_bwd_kv<D, BC>;
        if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess) return e;
        // slices: enough for the longest possible list (chunk 0: every token of the sequence)
        const unsigned slices = (unsigned)(((long long)a.T * UPT + kBwdSlice - 1) / kBwdSlice);
        kern<<<dim3((unsigned)a.C, (unsigned)(a.B * a.Hkv), slices), BC / 16 * 32, smem, st>>>(ba, UPT);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    // 4-6. routing, summaries, Stage 0
    {
        const long long rows = (long long)a.B * a.Hkv * a.T;
        k_bwd_route<D><<<(unsigned)((rows + 3) / 4), 128, 0, st>>>(ba);
        const long long chunks = (long long)a.B * a.Hkv * a.Cf;
        if (chunks > 0) {
            k_bwd_dsum<D><<<(unsigned)((chunks + 3) / 4), 128, 0, st>>>(ba);
            k_bwd_stage0<D, BC><<<(unsigned)((chunks + 3) / 4), 128, 0, st>>>(ba);
        }
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace

int backward_list_blocks(int T) { return (T + kListBlock - 1) / kListBlock; }

long long backward_nnz_max(int T, int Bc) {
    // routed (token, chunk) pairs of one (b, g) at most: sum over t of floor(t / Bc)
    const long long Cf = T / Bc;
    return (long long)Bc * Cf * (Cf - 1) / 2 + (long long)(T - Cf * Bc) * Cf;
}

cudaError_t launch_backward(const StageArgs &s, const BackwardBuffers &bb, cudaStream_t st) {
    BwdArgs ba;
    ba.s = s;
    ba.dout = reinterpret_cast<const __nv_bfloat16 *>(bb.dout);
    ba.out = reinterpret_cast<const __nv_bfloat16 *>(bb.out);
    ba.dq = bb.dq;
    ba.dk = bb.dk;
    ba.dv = bb.dv;
    ba.dhc = bb.dhc;
    ba.dlogp = bb.dlogp;
    ba.row_m = bb.row_m;
    ba.row_l = bb.row_l;
    ba.row_delta = bb.row_delta;
    ba.qbar = bb.qbar;
    ba.list_cnt = bb.list_cnt;
    ba.list_off = bb.list_off;
    ba.blk_cnt = bb.blk_cnt;
    ba.blk_off = bb.blk_off;
    ba.list = bb.list;
    ba.nnz_max = backward_nnz_max(s.T, s.Bc);
    ba.dsum = bb.dsum;
    ba.sigma = bb.sigma;
    if (s.D == 128 && s.Bc == 64) return launch_bwd_t<128, 64>(ba, st);
    if (s.D == 128 && s.Bc == 128) return launch_bwd_t<128, 128>(ba, st);
    if (s.D == 64 && s.Bc == 64) return launch_bwd_t<64, 64>(ba, st);
    if (s.D == 64 && s.Bc == 128) return launch_bwd_t<64, 128>(ba, st);
    return cudaErrorInvalidValue;
}

}  // namespace dash
