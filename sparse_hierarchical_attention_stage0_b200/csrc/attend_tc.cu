// attend_tc.cu -- Stage 2 on the 5th-generation tensor cores (tcgen05, TMEM, TMA), D = 128.
//
// gist.science "DashAttention: Differentiable and Adaptive Sparse Hierarchical Attention",
// Technische Zusammenfassung, "Stufe 2: Prior-induzierte spaerliche Softmax": a
// FlashAttention-style kernel iterates the active chunks given by the bit-packed mask and
// adds the routing bias (log of the prior) to the logits before the softmax; chunks with
// zero probability are masked; the diagonal chunk keeps its own branch.
//
// One CTA = one tile of 128 query rows of one (b, g): 128/G consecutive tokens x G heads
// (G >= 8).  The tile walks the UNION of its tokens' active chunks (the OR of their mask
// words, which carry each token's diagonal bit), 64 keys per pipeline block, in ascending
// order.  A row whose token did not route to a chunk gets bias -inf there; keys above the
// row's position are masked.  Per block:
//   S[128 x 64]  = Q K^T      tcgen05.mma kind::f16, A = Q from TMEM, B = K (smem, TMA)
//   softmax      one thread per row (4 warps), online max with lazy rescale, fp32
//   O[128 x 128] += P V       tcgen05.mma, A = P (bf16, TMEM, aliased into S), B = V (smem)
// Warp roles: 0 TMA producer (K/V blocks, 128B-swizzled, 2 stages), 1 MMA issuer and TMEM
// owner, 2 routing-bias producer (recomputes qbar.summary with Stage 1's exact arithmetic,
// 32 chunks per batch, double-buffered), 4-7 softmax + epilogue.  TMEM: Q 64 columns,
// S/P 64, O 128 = 256 columns, so two CTAs share an SM.  Every wait is bounded; on timeout
// the CTA records DASH_ERR_DEVICE_TIMEOUT and drains.
#include "kernels.cuh"
#include "tc_common.cuh"

namespace dash {
using namespace tcx;
namespace {

constexpr int kTcThreads = 256;
constexpr int kBlk = 64;                 // keys per pipeline block
constexpr int kStages = 2;
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColQ = 0, kColS = 64, kColP = 64, kColO = 128;
constexpr int kBiasBatch = 32;
constexpr int kWarpTma = 0, kWarpMma = 1, kWarpBias = 2, kWarpSm0 = 4;
constexpr uint32_t kStageBytes = 4 * 8192;  // K panels (d 0-63, 64-127), V panels
constexpr float kRescaleThreshold = 8.f;    // log2 units, as in lazy-rescale FlashAttention

struct TcShared {
    uint64_t full[kStages], empty[kStages], s_full, p_full, o_full;
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
            mbar_init(&sh.full[s], 1);
            mbar_init(&sh.empty[s], 1);
        }
        mbar_init(&sh.s_full, 1);
        mbar_init(&sh.p_full, 4);
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
                list[p++] = (int16_t)(w * 64 + bit);
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
    // Softmax warps: this thread's row, its token and head; Q row into TMEM columns [0, 64).
    const int sp = warp & 3;                     // TMEM sub-partition of this warp
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
        for (int half = 0; half < 2; ++half) {
            uint32_t r[32];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                uint4 v = row_ok ? *reinterpret_cast<const uint4 *>(qr + half * 64 + 8 * j)
                                 : make_uint4(0, 0, 0, 0);
                r[4 * j] = v.x;
                r[4 * j + 1] = v.y;
                r[4 * j + 2] = v.z;
                r[4 * j + 3] = v.w;
            }
            tmem_st32(tb + ((uint32_t)(32 * sp) << 16) + kColQ + 32 * half, r);
        }
        tmem_wait_st();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const int n_chunks = sh.n_chunks;
    const int n_blocks = n_chunks * NSUB;
    bool failed = false;

    if (warp == kWarpTma) {
        // ------------------------------------------------------------ TMA producer
        // The whole warp runs the loop (converged); lane 0 issues the copies.
        int issued = 0;
        for (int i = 0; i < n_blocks; ++i) {
            const int s = i % kStages;
            const uint32_t ph = (uint32_t)(i / kStages) & 1u;
            if (!wait_or_fail(&sh.empty[s], ph ^ 1u, a.status, failed)) break;
            issued = i + 1;
            if (lane == 0) {
                const int key0 = (int)list[i / NSUB] * BC + (i % NSUB) * kBlk;
                unsigned char *st = base + (size_t)s * kStageBytes;
                mbar_arrive_expect_tx(&sh.full[s], kStageBytes);
                tma_load_3d(st, &tmK, 0, key0, (int)bg, &sh.full[s]);
                tma_load_3d(st + 8192, &tmK, 64, key0, (int)bg, &sh.full[s]);
                tma_load_3d(st + 16384, &tmV, 0, key0, (int)bg, &sh.full[s]);
                tma_load_3d(st + 24576, &tmV, 64, key0, (int)bg, &sh.full[s]);
            }
            __syncwarp();
        }
        if (failed) {
            // Bounded wait for the copies still in flight (the last one per stage).
            for (int j = max(0, issued - kStages); j < issued; ++j)
                mbar_wait_bounded(&sh.full[j % kStages], (uint32_t)(j / kStages) & 1u);
            __syncwarp();
        }
    } else if (warp == kWarpMma) {
        // ------------------------------------------------------------ MMA issuer
        // The whole warp runs the loop (converged); lane 0 issues the MMAs and commits.
        constexpr uint32_t id_qk = idesc_bf16(128, kBlk, 0);
        constexpr uint32_t id_pv = idesc_bf16(128, D, 1);
        for (int i = 0; i < n_blocks; ++i) {
            const int s = i % kStages;
            const uint32_t ph = (uint32_t)(i / kStages) & 1u;
            if (!wait_or_fail(&sh.full[s], ph, a.status, failed)) break;
            tc_fence_after();
            const uint32_t st = smem_u32(base + (size_t)s * kStageBytes);
            if (lane == 0) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t bd = smem_desc_sw128(st + (uint32_t)(kk / 4) * 8192u +
                                                            (uint32_t)(kk % 4) * 32u,
                                                        16, 1024);
                    mma_ts(tb + kColS, tb + kColQ + 8u * kk, bd, id_qk, kk > 0 ? 1u : 0u);
                }
                mma_commit(&sh.s_full);
            }
            __syncwarp();
            if (!wait_or_fail(&sh.p_full, (uint32_t)i & 1u, a.status, failed)) break;
            tc_fence_after();
            if (lane == 0) {
#pragma unroll
                for (int kk = 0; kk < kBlk / 16; ++kk) {
                    const uint64_t bd = smem_desc_sw128(st + 16384u + (uint32_t)kk * 2048u, 8192, 1024);
                    mma_ts(tb + kColO, tb + kColP + 8u * kk, bd, id_pv, (i > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(&sh.empty[s]);
            }
            __syncwarp();
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
                    const int c = list[ci], t = t0 + u;
                    const int ctu = t / BC;
                    if (t >= a.T || c > ctu) {
                        v = -INFINITY;
                    } else if (c < ctu) {
                        const long long rowi = bg * a.T + t;
                        const bool act = (a.mask[rowi * a.W + (c >> 6)] >> (c & 63)) & 1ull;
                        if (!act) {
                            v = -INFINITY;
                        } else {
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
                buf[e] = v;
            }
            __syncwarp();
            named_sync(1, 32 + 128);
        }
    } else if (warp >= kWarpSm0) {
        // ------------------------------------------------------------ softmax
        const uint32_t lane_base = tb + ((uint32_t)(32 * sp) << 16);
        const int ct_row = t_row / BC;
        float m_ref = -INFINITY, l_sum = 0.f;
        for (int i = 0; i < n_blocks; ++i) {
            const int ci = i / NSUB;
            // Every batch boundary is passed even after a failure: the bias warp waits there.
            if (ci % kBiasBatch == 0 && i % NSUB == 0) named_sync(1, 32 + 128);
            if (!wait_or_fail(&sh.s_full, (uint32_t)i & 1u, a.status, failed)) continue;
            tc_fence_after();
            const int c = list[ci];
            const int key0 = c * BC + (i % NSUB) * kBlk;
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
            uint32_t sv[2][32];
            tmem_ld32(lane_base + kColS, sv[0]);
            tmem_ld32(lane_base + kColS + 32, sv[1]);
            tmem_wait_ld();
            float mx = -INFINITY;
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    float v = fmaf(__uint_as_float(sv[h][j]), a.qk_scale2, bias2);
                    if (diag && key0 + 32 * h + j > t_row) v = -INFINITY;
                    sv[h][j] = __float_as_uint(v);
                    mx = fmaxf(mx, v);
                }
            // Lazy rescale: move the reference only when the block max exceeds it by more than
            // the threshold (values up to 2^threshold above the reference are exact in fp32).
            float f = 1.f;
            if (mx > m_ref + kRescaleThreshold) {
                if (m_ref != -INFINITY && l_sum > 0.f) {
                    f = fast_exp2(m_ref - mx);
                    l_sum *= f;
                }
                m_ref = mx;
            }
            // TMEM loads/stores are warp-wide: the warp rescales its O rows together whenever
            // any of them needs it (factor 1 for the others).  O is stable here: the commit
            // behind s_full also tracked the previous P V.
            if (__any_sync(kFull, f != 1.f)) {
#pragma unroll 1
                for (int q4 = 0; q4 < 4; ++q4) {
                    uint32_t o[32];
                    tmem_ld32(lane_base + kColO + 32 * q4, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * f);
                    tmem_st32(lane_base + kColO + 32 * q4, o);
                }
            }
            const float mu = m_ref == -INFINITY ? 0.f : m_ref;
            uint32_t pw[32];
            float psum = 0.f;
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const float p0 = fast_exp2(__uint_as_float(sv[h][2 * j]) - mu);
                    const float p1 = fast_exp2(__uint_as_float(sv[h][2 * j + 1]) - mu);
                    psum += p0 + p1;
                    pw[16 * h + j] = pack_bf16x2(p0, p1);
                }
            l_sum += psum;
            tmem_st32(lane_base + kColP, pw);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh.p_full);
        }
        // Epilogue: O / l -> bf16.
        if (!failed && wait_or_fail(&sh.o_full, 0, a.status, failed)) {
            tc_fence_after();
            const float inv = l_sum > 0.f ? 1.f / l_sum : 0.f;
            __nv_bfloat16 *orow = reinterpret_cast<__nv_bfloat16 *>(a.out) +
                                  (((long long)b * a.Hq + h_row) * a.T + (row_ok ? t_row : 0)) * D;
#pragma unroll 1
            for (int q4 = 0; q4 < 4; ++q4) {
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
    size_t off = (size_t)kStages * kStageBytes;
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
