// stage0.cu -- Stage 0: local chunk summarisation.
//
// gist.science "DashAttention: Differentiable and Adaptive Sparse Hierarchical Attention",
// Technische Zusammenfassung, "Stufe 0: Lokale Chunk-Zusammenfassung": a learned query
// (head_cls) attends by local scaled dot-product attention over the keys of each chunk; the
// summary of a complete chunk is frozen and cached for decoding.
//
// One warp per chunk.  The chunk's keys (Bc x D bf16, contiguous in memory) are staged into
// shared memory by one bulk copy on the TMA engine (cp.async.bulk + mbarrier), then
//   l_j = head_cls . k_j / sqrt(D)      (lane-sliced dot, butterfly-reduced)
//   summary = sum_j exp(l_j - max) k_j / sum_j exp(l_j - max)
// with each lane owning D/32 output dims (16-byte coalesced stores for D = 128).
// HBM-bound: it reads Bc*D*2 bytes and writes D*4 bytes per chunk.
#include <algorithm>

#include "dash_common.cuh"
#include "kernels.cuh"

namespace dash {

// Grid: one warp per unit.  Prefill units are (b, g, c) for every complete chunk; decode
// units (seq_lens != nullptr) are (b, g, r) = the r-th most recent complete chunk.
// Paged caches (block_table != nullptr): the keys of logical chunk c of sequence b live in
// page block_table[b * max_blocks + c] of k [n_pages, Hkv, BC, D], and its summary goes to
// summary [n_pages, Hkv, D]; a page index out of [0, n_pages) is reported and skipped.
template <int D, int BC>
__global__ void __launch_bounds__(kStage0Warps * 32)
k_stage0(const __nv_bfloat16 *__restrict__ k, const float *__restrict__ head_cls,
         float *__restrict__ summary, int B, int Hkv, int T, int Cf, const int32_t *seq_lens,
         int n_recent, uint32_t *status, int test_stall, const int32_t *block_table,
         int max_blocks, int n_pages, int c_begin, int nc) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    __shared__ __align__(8) uint64_t bars[kStage0Warps];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long unit = (long long)blockIdx.x * kStage0Warps + warp;
    int b, g, c;
    if (seq_lens == nullptr) {                    // chunks [c_begin, c_begin + nc) of every (b, g)
        if (unit >= (long long)B * Hkv * nc) return;
        c = c_begin + (int)(unit % nc);
        g = (int)((unit / nc) % Hkv);
        b = (int)(unit / ((long long)nc * Hkv));
    } else {
        if (unit >= (long long)B * Hkv * n_recent) return;
        int r = (int)(unit % n_recent);
        g = (int)((unit / n_recent) % Hkv);
        b = (int)(unit / ((long long)n_recent * Hkv));
        int L = seq_lens[b];
        if (L < 1 || L > T) {
            if (lane == 0) report(status, DASH_ERR_INVALID_ARGUMENT);
            return;
        }
        c = L / BC - 1 - r;
        if (c < 0) return;
    }
    if (!dash_check(c >= 0 && c < Cf && b < B && (long long)(c + 1) * BC <= T, status)) return;
    __nv_bfloat16 *ks = reinterpret_cast<__nv_bfloat16 *>(smem_raw) + (size_t)warp * BC * D;
    const __nv_bfloat16 *src = k + (((long long)b * Hkv + g) * T + (long long)c * BC) * D;
    float *dst = summary + (((long long)b * Hkv + g) * Cf + c) * D;
    if (block_table) {
        const int page = block_table[(long long)b * max_blocks + c];
        if (page < 0 || page >= n_pages) {
            if (lane == 0) report(status, DASH_ERR_INVALID_ARGUMENT);
            return;
        }
        src = k + ((long long)page * Hkv + g) * BC * D;
        dst = summary + ((long long)page * Hkv + g) * D;
    }
    constexpr uint32_t kBytes = BC * D * sizeof(__nv_bfloat16);
    if (lane == 0) {
        mbar_init(&bars[warp], 1);
        fence_mbar_init();
    }
    __syncwarp();
    // Test hook: with test_stall nothing arrives on the barrier (no copy is issued), so the
    // bounded wait below runs out and reports DASH_ERR_DEVICE_TIMEOUT.
    if (lane == 0 && !test_stall) {
        mbar_arrive_expect_tx(&bars[warp], kBytes);
        bulk_g2s(ks, src, kBytes, &bars[warp]);
    }
    if (!__all_sync(kFull, mbar_wait_bounded(&bars[warp], 0))) {   // warp-uniform outcome
        if (lane == 0) report(status, DASH_ERR_DEVICE_TIMEOUT);
        if (!test_stall) mbar_wait_bounded(&bars[warp], 0);   // one more bounded wait for the copy
        return;
    }
    summarize_chunk_warp<D, BC>(ks, head_cls + (size_t)g * D, dst);
}

template <int D, int BC>
static cudaError_t launch_stage0_t(const StageArgs &a, const int32_t *seq_lens, int n_recent,
                                   cudaStream_t st, const int32_t *block_table = nullptr,
                                   int max_blocks = 0, int n_pages = 0) {
    const int c_begin = seq_lens || a.s0_end <= 0 ? 0 : a.s0_begin;
    const int nc = seq_lens ? 0 : (a.s0_end <= 0 ? a.Cf : std::min(a.s0_end, a.Cf) - c_begin);
    if (!seq_lens && nc <= 0) return cudaSuccess;
    long long units = seq_lens ? (long long)a.B * a.Hkv * n_recent
                               : (long long)a.B * a.Hkv * nc;
    if (units == 0) return cudaSuccess;
    size_t smem = (size_t)kStage0Warps * BC * D * sizeof(__nv_bfloat16);
    auto kern = k_stage0<D, BC>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    unsigned grid = (unsigned)((units + kStage0Warps - 1) / kStage0Warps);
    kern<<<grid, kStage0Warps * 32, smem, st>>>(
        reinterpret_cast<const __nv_bfloat16 *>(a.k), a.head_cls, a.summary, a.B, a.Hkv, a.T,
        a.Cf, seq_lens, n_recent, a.status, a.test_stall, block_table, max_blocks, n_pages, c_begin, nc);
    return cudaGetLastError();
}

cudaError_t launch_stage0(const StageArgs &a, const int32_t *seq_lens, int n_recent,
                          cudaStream_t st) {
    if (a.D == 128 && a.Bc == 64) return launch_stage0_t<128, 64>(a, seq_lens, n_recent, st);
    if (a.D == 128 && a.Bc == 128) return launch_stage0_t<128, 128>(a, seq_lens, n_recent, st);
    if (a.D == 64 && a.Bc == 64) return launch_stage0_t<64, 64>(a, seq_lens, n_recent, st);
    if (a.D == 64 && a.Bc == 128) return launch_stage0_t<64, 128>(a, seq_lens, n_recent, st);
    return cudaErrorInvalidValue;
}

cudaError_t launch_stage0_paged(const StageArgs &a, const int32_t *seq_lens, int n_recent,
                                const int32_t *block_table, int max_blocks, int n_pages,
                                cudaStream_t st) {
    if (a.D == 128 && a.Bc == 64)
        return launch_stage0_t<128, 64>(a, seq_lens, n_recent, st, block_table, max_blocks, n_pages);
    if (a.D == 128 && a.Bc == 128)
        return launch_stage0_t<128, 128>(a, seq_lens, n_recent, st, block_table, max_blocks, n_pages);
    if (a.D == 64 && a.Bc == 64)
        return launch_stage0_t<64, 64>(a, seq_lens, n_recent, st, block_table, max_blocks, n_pages);
    if (a.D == 64 && a.Bc == 128)
        return launch_stage0_t<64, 128>(a, seq_lens, n_recent, st, block_table, max_blocks, n_pages);
    return cudaErrorInvalidValue;
}

}  // namespace dash
