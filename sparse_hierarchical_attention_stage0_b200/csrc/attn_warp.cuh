// attn_warp.cuh -- warp-level pieces of the block-sparse attention (mma.sync m16n8k16):
// one warp owns 16 query rows and streams 32-key sub-blocks of K and V through swizzled
// shared memory, keeping the online-softmax state (max, sum, O) in registers.
#pragma once

#include "dash_common.cuh"
#include "kernels.cuh"

namespace dash {

// Byte offset of 16-byte chunk `ch` of row `row` in a [rows][D] bf16 tile (XOR swizzle,
// conflict-free for ldmatrix).
template <int D>
__device__ __forceinline__ uint32_t swz(int row, int ch) {
    return (uint32_t)(row * D * 2 + ((ch ^ (row & 7)) << 4));
}

// Copy keys [key0, key0 + kSub) of one (b, g) K or V plane into a swizzled tile; rows at or
// beyond T are zero-filled without a global read.
template <int D>
__device__ __forceinline__ void load_sub(unsigned char *tile, const __nv_bfloat16 *plane,
                                         int key0, int T) {
    constexpr int CH = D / 8;                     // 16-byte chunks per row
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int i = lane; i < kSub * CH; i += 32) {
        const int row = i / CH, ch = i % CH, key = key0 + row;
        const bool ok = key < T;
        const __nv_bfloat16 *src = plane + (long long)(ok ? key : 0) * D + ch * 8;
        cp_async16(tile + swz<D>(row, ch), src, ok ? 16 : 0);
    }
}

template <int D>
struct UnitState {
    float o[D / 8][4];
    float m_lo, m_hi, l_lo, l_hi;
};

// S = Q K^T for one sub-block: acc[j] is the 16x8 tile of keys 8j..8j+7.
template <int D>
__device__ __forceinline__ void qk_sub(float (&acc)[4][4], const uint32_t (&qf)[D / 16][4],
                                       const unsigned char *ks) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[j][e] = 0.f;
#pragma unroll
        for (int kk = 0; kk < D / 16; kk += 2) {
            uint32_t r[4];
            ldsm_x4(r, ks + swz<D>(8 * j + (lane & 7), 2 * kk + (lane >> 3)));
            mma_bf16_16816(acc[j], qf[kk], r[0], r[1]);
            mma_bf16_16816(acc[j], qf[kk + 1], r[2], r[3]);
        }
    }
}

// O += P V for one sub-block (P given as bf16 A fragments of the 2 key steps).
template <int D>
__device__ __forceinline__ void pv_sub(UnitState<D> &st, const uint32_t (&pa)[2][4],
                                       const unsigned char *vs) {
    const int lane = threadIdx.x & 31;
    const int mi = lane >> 3;
#pragma unroll
    for (int kk = 0; kk < 2; ++kk) {
#pragma unroll
        for (int j = 0; j < D / 8; j += 2) {
            uint32_t r[4];
            ldsm_x4_t(r, vs + swz<D>(16 * kk + (lane & 7) + 8 * (mi & 1), j + (mi >> 1)));
            mma_bf16_16816(st.o[j], pa[kk], r[0], r[1]);
            mma_bf16_16816(st.o[j + 1], pa[kk], r[2], r[3]);
        }
    }
}

// Online softmax over one sub-block of logits (log2 domain), producing P fragments.
template <int D>
__device__ __forceinline__ void softmax_sub(UnitState<D> &st, float (&acc)[4][4],
                                            uint32_t (&pa)[2][4], float qk_scale2,
                                            float bias_lo, float bias_hi, bool diag, int key0,
                                            int tok_lo, int tok_hi) {
    const int lane = threadIdx.x & 31;
    const int qd = lane & 3;
    float mx_lo = -INFINITY, mx_hi = -INFINITY;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const bool hi = e >= 2;
            const int key = key0 + 8 * j + 2 * qd + (e & 1);
            float v = fmaf(acc[j][e], qk_scale2, hi ? bias_hi : bias_lo);
            if (diag && key > (hi ? tok_hi : tok_lo)) v = -INFINITY;
            acc[j][e] = v;
            if (hi) mx_hi = fmaxf(mx_hi, v); else mx_lo = fmaxf(mx_lo, v);
        }
    }
    mx_lo = fmaxf(mx_lo, __shfl_xor_sync(kFull, mx_lo, 1));
    mx_lo = fmaxf(mx_lo, __shfl_xor_sync(kFull, mx_lo, 2));
    mx_hi = fmaxf(mx_hi, __shfl_xor_sync(kFull, mx_hi, 1));
    mx_hi = fmaxf(mx_hi, __shfl_xor_sync(kFull, mx_hi, 2));
    const float mn_lo = fmaxf(st.m_lo, mx_lo), mn_hi = fmaxf(st.m_hi, mx_hi);
    const float mu_lo = mn_lo == -INFINITY ? 0.f : mn_lo;
    const float mu_hi = mn_hi == -INFINITY ? 0.f : mn_hi;
    const float sc_lo = fast_exp2(st.m_lo - mu_lo), sc_hi = fast_exp2(st.m_hi - mu_hi);
    st.m_lo = mn_lo;
    st.m_hi = mn_hi;
    float sum_lo = 0.f, sum_hi = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        // Weights rounded to bf16 once: the row sums add exactly what the MMA multiplies.
        acc[j][0] = bf16_round(fast_exp2(acc[j][0] - mu_lo));
        acc[j][1] = bf16_round(fast_exp2(acc[j][1] - mu_lo));
        acc[j][2] = bf16_round(fast_exp2(acc[j][2] - mu_hi));
        acc[j][3] = bf16_round(fast_exp2(acc[j][3] - mu_hi));
        sum_lo += acc[j][0] + acc[j][1];
        sum_hi += acc[j][2] + acc[j][3];
    }
    st.l_lo = st.l_lo * sc_lo + sum_lo;
    st.l_hi = st.l_hi * sc_hi + sum_hi;
#pragma unroll
    for (int j = 0; j < D / 8; ++j) {
        st.o[j][0] *= sc_lo;
        st.o[j][1] *= sc_lo;
        st.o[j][2] *= sc_hi;
        st.o[j][3] *= sc_hi;
    }
#pragma unroll
    for (int kk = 0; kk < 2; ++kk) {
        pa[kk][0] = pack_bf16x2(acc[2 * kk][0], acc[2 * kk][1]);
        pa[kk][1] = pack_bf16x2(acc[2 * kk][2], acc[2 * kk][3]);
        pa[kk][2] = pack_bf16x2(acc[2 * kk + 1][0], acc[2 * kk + 1][1]);
        pa[kk][3] = pack_bf16x2(acc[2 * kk + 1][2], acc[2 * kk + 1][3]);
    }
}

// Bias (log2 domain) of routed chunk c for the token whose group-mean query is qb and whose
// threshold is tau; identical arithmetic to Stage 1's margin.
template <int D>
__device__ __forceinline__ float routed_bias2(const float *qb, const float *srow, float tau,
                                              const RouteConsts &rc) {
    if (rc.kind == kKindTopk) return 0.f;            // top-k: uniform prior
    const float dot = route_dot<D>(qb, srow);
    if (rc.kind == 0) return rc.sigma2 * (__fmul_rn(dot, rc.sscale) - tau);
    const float m = __fsub_rn(__fmul_rn(dot, rc.xscale), tau);
    return rc.bscale2 * log2f(fmaxf(m, 1e-37f));
}

}  // namespace dash
