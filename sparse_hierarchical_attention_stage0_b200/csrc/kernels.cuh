// kernels.cuh -- launch interfaces between the C ABI (dash_api.cu) and the kernels.
#pragma once

#include "dash_common.cuh"

namespace dash {

constexpr int kStage0Warps = 4;     // chunks summarised per CTA
constexpr int kRouteThreads = 256;  // Stage 1 CTA size
constexpr int kAttnWarps = 4;       // Stage 2 (mma.sync path) units per CTA
constexpr int kSub = 32;            // keys per Stage 2 sub-block

// Everything one prefill stage needs; pointers the stage does not use may be null.
struct StageArgs {
    const void *q, *k, *v;
    const float *head_cls;
    float *summary;           // [B,Hkv,Cf,D]
    float *tau;               // [B,Hkv,T]
    float *p;                 // [B,Hkv,T,C] or null
    uint64_t *mask;           // [B,Hkv,T,W]
    void *out;                // [B,Hq,T,D]
    void *vt;                 // [B,Hkv,D,T8] V^T scratch for the 128-key-block kernel, or null
    int B, Hq, Hkv, T, D, Bc, G, C, Cf, W;
    RouteConsts rc;
    float qk_scale2;          // log2(e) / sqrt(D)
    int ignore_routing;       // DENSE or FORCE_ALL_ACTIVE: attend every chunk, bias 0
    int t_begin, t_end;       // Stages 1-2 compute rows [t_begin, t_end) (t_begin % 128 == 0);
                              // T stays the row stride of q, tau, mask, p and out
    int vt_ready;             // V^T scratch already holds the keys this call reads
    int vt_begin, vt_end;     // keys [vt_begin, vt_end) to transpose when !vt_ready (vt_end 0: all)
    int s0_begin, s0_end;     // Stage 0 over chunks [s0_begin, s0_end) (s0_end 0: every chunk)
    int test_stall;           // test hook: Stage 0's chunk-copy wait runs out (DASH_FLAG_TEST_STALL_WAIT)
    int fuse_route;           // Stage 2 computes the routing itself (fused route-and-attend)
    // Run-time choice between the 128-key-block and the warp-MMA Stage 2 kernels (null: none):
    // cost[0] / cost[1] are the token-chunk pairs each would execute (k_union_cost), and the
    // 128-key-block kernel runs iff cost[0] <= cost[1] * cost_ratio.
    const unsigned long long *cost;
    float cost_ratio;
    uint32_t *status;
};

struct DecodeArgs {
    const void *q, *k, *v;    // q [B,Hq,D]; caches [B,Hkv,cap,D]
    const int32_t *seq_lens;  // [B]
    const float *summary;     // [B,Hkv,cap/Bc,D]
    const float *head_cls;    // [Hkv,D] (estimate_diagonal only)
    const int32_t *block_table;  // paged cache: [B, max_blocks] page of each logical chunk, or null
    int max_blocks, n_pages;  // paged cache: table row length, pages in the pools
    void *out;                // [B,Hq,D]
    float *p;                 // [B,Hkv,Ccap] or null
    uint64_t *mask;           // [B,Hkv,Wcap] or null
    int B, Hq, Hkv, cap, D, Bc, G, Ccap, Cf, Wcap;
    RouteConsts rc;
    float qk_scale2;
    // Decode step (k_new != null): the new token's k/v [B,Hkv,D] go to position seq_lens[b]
    // of the cache before the step attends over seq_lens[b] + 1 tokens; the last of the
    // sequence's Hkv clusters to finish (arrive[b] counts them) stores seq_lens[b] + 1 into
    // seq_out[b]; a chunk completed by the new token gets its summary in summary_out.
    const void *k_new, *v_new;
    int32_t *seq_out;
    int *arrive;
    float *summary_out;
    uint32_t *status;
};

// Byte offsets in the 256-byte status block at the start of every workspace: the status word
// (0), the run-time Stage 2 choice's two costs (8, 16) and the kernel that ran (24: 1 the
// 128-key-block kernel, 2 the warp-MMA kernel, 0 no run-time choice in the last call); a
// decode step keeps its per-sequence counters at 32.. when they fit.
constexpr int kStatusCostOff = 8;
constexpr int kStatusRanOff = 24;

// With a run-time Stage 2 choice: whether the 128-key-block kernel is the one that runs.
__device__ __forceinline__ bool attend_fa_chosen(const StageArgs &a) {
    return (double)a.cost[0] <= (double)a.cost[1] * (double)a.cost_ratio;
}
// Records, once per launch, which kernel a run-time choice ran (1: 128-key blocks, 2: warp MMA).
__device__ __forceinline__ void attend_record_ran(const StageArgs &a, unsigned char id) {
    if (blockIdx.x == 0 && threadIdx.x == 0)
        reinterpret_cast<volatile unsigned char *>(a.status)[kStatusRanOff] = id;
}

cudaError_t launch_stage0(const StageArgs &a, const int32_t *seq_lens, int n_recent,
                          cudaStream_t st);
// Stage 0 over the newest complete chunks of a paged cache: k_pool [n_pages, Hkv, Bc, D],
// summary_pool [n_pages, Hkv, D], block_table [B, max_blocks].
cudaError_t launch_stage0_paged(const StageArgs &a, const int32_t *seq_lens, int n_recent,
                                const int32_t *block_table, int max_blocks, int n_pages,
                                cudaStream_t st);
cudaError_t launch_route(const StageArgs &a, cudaStream_t st);
int route_rows_per_cta(int C, int D);   // 0 if C is too large for the routing kernel
cudaError_t launch_attend(const StageArgs &a, cudaStream_t st);
// The Stage 2 kernel launch_attend picks for these arguments, and its name.
// kFaOrWarp: both are launched after k_union_cost; each CTA of the one not chosen exits at
// once (see StageArgs::cost).
enum class AttendKernel { kNone, kPair, kFa, kTc, kWarp, kFaOrWarp };
AttendKernel attend_kernel(const StageArgs &a);
const char *attend_kernel_name(AttendKernel k);
bool attend_tc_supported(const StageArgs &a);
cudaError_t launch_attend_tc(const StageArgs &a, cudaStream_t st);
bool attend_fa_supported(const StageArgs &a);
// The 128-key-block kernel can run Stage 1 itself for these arguments (fused route-and-attend).
bool attend_fa_fuse_supported(const StageArgs &a);
size_t attend_fa_vt_bytes(int B, int Hkv, int T, int D);
cudaError_t launch_attend_fa(const StageArgs &a, cudaStream_t st);
bool attend_pair_supported(const StageArgs &a);
cudaError_t launch_attend_pair(const StageArgs &a, cudaStream_t st);
// Keys [k_begin, k_end) of V (k_begin a multiple of 64; k_end 0: all), the zero padding to T8
// included when the range reaches T.
cudaError_t launch_vtranspose(const void *v, void *vt, int BHkv, int T, int D, cudaStream_t st,
                              int k_begin = 0, int k_end = 0);
cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t st);

// Buffers of the backward pass (dash_backward); the StageArgs carry the forward's routing
// (summary, tau, mask, p).
struct BackwardBuffers {
    const void *dout, *out;   // [B,Hq,T,D] bf16
    float *dq;                // [B,Hq,T,D]
    float *dk, *dv;           // [B,Hkv,T,D]
    float *dhc;               // [Hkv,D]
    float *dlogp;             // [B,Hkv,T,C]
    float *row_m, *row_l, *row_delta;   // [B,Hq,T]
    float *qbar;              // [B,Hkv,T,D]
    int *list_cnt;            // [B*Hkv][C]
    long long *list_off;      // [B*Hkv][C+1]
    int *blk_cnt;             // [B*Hkv][C][backward_list_blocks(T)]
    long long *blk_off;       // [B*Hkv][C][backward_list_blocks(T)]
    int *list;                // [B*Hkv][backward_nnz_max]
    float *dsum;              // [B,Hkv,Cf,D]
    float sigma;
};
long long backward_nnz_max(int T, int Bc);
int backward_list_blocks(int T);            // token blocks of the routing transpose
cudaError_t launch_backward(const StageArgs &s, const BackwardBuffers &bb, cudaStream_t st);
int decode_supported(int G, int Ccap, int D);
// Scratch bytes dash_prefill needs in its workspace (status word, tau, and the summaries /
// mask words not supplied by the caller); 0 on bad parameters.
size_t prefill_scratch_bytes(const dash_params_t *p, bool has_summary, bool has_mask);

}  // namespace dash
