/*
 * dash.h -- C ABI of libdash: the DashAttention forward path (chunk summaries, alpha-entmax
 * block routing, prior-induced block-sparse softmax attention) for causal prefill and
 * incremental decode on NVIDIA B200 (sm_100a).
 *
 * The method (page title, section):
 *   gist.science "DashAttention: Differentiable and Adaptive Sparse Hierarchical Attention",
 *   Technische Zusammenfassung:
 *     "Stufe 0: Lokale Chunk-Zusammenfassung"   -> dash_stage0, dash_update_chunk_cache
 *     "Stufe 1: Entmax-Chunk-Routing"            -> dash_route
 *     "Stufe 2: Prior-induzierte spaerliche Softmax" -> dash_attend; its causality (row t
 *     reads keys <= t) lets dash_prefill_host overlap host copies with row slices
 *   aiexpert.news "DashAttention alcanca 75% de esparsidade ...", interface paragraph:
 *     queries, keys, values, a per-head head_cls vector, chunk_size, estimate_diagonal,
 *     enable_gqa, optional active_blocks mask -> dash_params_t, dash_prefill.
 *   aixai.ru "DashAttention ...", "Трёхстадийная архитектура": the active-block mask is
 *     bit-packed into 64-bit words and walked in one pass without explicit indices.
 *   liuzhao09.github.io "DashAttention 精读", section 2: prefill and incremental decoding
 *     with a chunk-representation cache -> dash_prefill, dash_decode.
 *
 * What is computed (notation: b batch, h query head, g = h / G its KV head with
 * G = heads_q / heads_kv, t query position, Bc = chunk_size, D = head_dim, c_t = t / Bc):
 *   Stage 0: summary[b,g,c] = sum_j softmax_j(head_cls[g].k_j / sqrt(D)) k_j over the keys j
 *            of every complete chunk c.
 *   Stage 1: for c < c_t:  s_c = gamma * qbar.summary[b,g,c] / sqrt(D), qbar = mean of the G
 *            query heads of group g at t; p = alpha-entmax(s):
 *            p_c = [(alpha-1) s_c - tau]_+^(1/(alpha-1)), sum_c p_c = 1 (alpha = 1: softmax).
 *            Chunk c < c_t is active iff p_c > 0; the diagonal chunk c_t is always active.
 *   Stage 2: O[b,h,t] = sum_j softmax_j(q.k_j / sqrt(D) + bias_j) v_j over keys j <= t in
 *            active chunks, bias_j = sigma * log p_c(j) for routed chunks and 0 on the
 *            diagonal chunk.  Zero-probability chunks are skipped.
 *
 * Conventions for every entry point:
 *   - All tensor pointers are caller-owned DEVICE memory, dense, row-major (C order), with
 *     the layouts stated per argument.  The library never allocates or frees memory and
 *     keeps no global state; calls on different streams do not interact.
 *   - Every call is asynchronous on `stream` (a cudaStream_t passed as void*; NULL = the
 *     legacy default stream).  Arguments are checked on the host before any launch; a bad
 *     argument returns DASH_ERR_INVALID_ARGUMENT / DASH_ERR_UNSUPPORTED /
 *     DASH_ERR_WORKSPACE_TOO_SMALL and launches nothing.  A launch failure returns
 *     DASH_ERR_CUDA.  Faults found on the device (a device-side bound violated, an
 *     iteration cap reached) are written to a status word in the workspace and read with
 *     dash_read_device_status; the kernels never trap.
 *   - Pointers must be 16-byte aligned; workspaces 256-byte aligned.
 *   - Supported: head_dim in {64, 128}; chunk_size in {64, 128}; heads_q % heads_kv == 0
 *     with G = heads_q / heads_kv dividing 16 or a multiple of 16; heads_q == heads_kv when
 *     enable_gqa == 0; alpha >= 1; seq_len >= 1 (seq_len % chunk_size may be non-zero: the
 *     last partial chunk is only ever a diagonal chunk).
 */
#ifndef DASH_H_
#define DASH_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    DASH_OK = 0,
    DASH_ERR_INVALID_ARGUMENT = 1,   /* a null/misaligned pointer, a bad size or value */
    DASH_ERR_UNSUPPORTED = 2,        /* valid, but outside the supported shapes/flags */
    DASH_ERR_WORKSPACE_TOO_SMALL = 3,
    DASH_ERR_CUDA = 4,               /* a CUDA runtime call or launch failed */
    DASH_ERR_DEVICE_TIMEOUT = 5,     /* a device wait or iteration cap ran out */
    DASH_ERR_RANGE_CLAMPED = 6,      /* a logit lay so far above its row's softmax reference
                                        (the maximum over the row's visible keys of the
                                        diagonal chunk) that the row's probabilities were
                                        clamped or their sum overflowed fp32; the output of
                                        that row is not exact */
    DASH_ERR_BOUNDS = 7              /* a device-side bounds check failed; the access it
                                        guarded was skipped, the output is not meaningful.
                                        Debug builds (libdash_debug.so, compiled with
                                        DASH_DEBUG) check every kernel; the release library
                                        checks only the index lists dash_backward builds. */
} dash_status_t;

enum {
    /* Dense causal attention: Stages 0-1 are skipped and every chunk c <= c_t is attended
     * with bias 0 (the uniform prior).  summary_k, p, active_blocks must be NULL. */
    DASH_FLAG_DENSE = 1,
    /* Stages 0-1 run and write their outputs, but Stage 2 attends every chunk c <= c_t with
     * bias 0 (all blocks forced active, uniform prior).  Same O as DASH_FLAG_DENSE. */
    DASH_FLAG_FORCE_ALL_ACTIVE = 2,
    /* estimate_diagonal, the diagonal correction of the alpha-entmax normalisation
     * (aiexpert.news interface paragraph; the pages give no formula, this is the reading
     * built): the diagonal chunk c_t, which has no frozen summary (gist.science "Stufe 2"),
     * joins the entmax as one more candidate, scored against an estimated summary -- Stage
     * 0's softmax-weighted key sum over the keys of chunk c_t the row can see (c_t Bc .. t).
     * The routed chunks then share 1 - p[c_t] of the mass; p[.., c_t] reports the diagonal's
     * probability; the diagonal chunk is still always attended with bias 0.  Rows t < Bc
     * route to the diagonal alone (p[.., 0] = 1).  Supported by dash_prefill,
     * dash_prefill_host and dash_decode (which then needs head_cls); dash_route returns
     * DASH_ERR_UNSUPPORTED with it (it takes no keys).  Ignored with DASH_FLAG_DENSE. */
    DASH_FLAG_ESTIMATE_DIAGONAL = 4,
    /* Test hook (fault injection without a GPU fault): caps the entmax Newton solve of the
     * routing at one iteration, so every row that needs more reports DASH_ERR_DEVICE_TIMEOUT
     * through the device status word, the way a row that hit the real cap would.  The
     * outputs of such a call are not meaningful. */
    DASH_FLAG_TEST_NEWTON_CAP = 8,
    /* Test hook (fault injection without a GPU fault): Stage 0 issues no chunk copy, so the
     * bounded wait on its barrier runs out after 2 s and reports DASH_ERR_DEVICE_TIMEOUT;
     * the CTA then returns with nothing in flight and the context stays usable.  Meant for
     * a few chunks (every CTA of the grid waits its 2 s); the outputs are not meaningful. */
    DASH_FLAG_TEST_STALL_WAIT = 16,
    /* Fused route-and-attend (dash_prefill and dash_prefill_host): where the 128-key-block
     * Stage 2 kernel applies (D = 128, G >= 8, entmax routing, no estimated diagonal), it
     * routes its own tile's tokens with Stage 1's arithmetic instead of a separate Stage 1
     * launch; q is read once and the routing makes no round trip through memory.  Mask, p,
     * tau and the output are bit-identical to the separate launches.  Off by default: on B200
     * the separate launches measured faster (32K: 3.74 against 4.04 ms per step; 128K: 124.3
     * against 126.3 ms), because the routing inside the kernel runs at one CTA per SM while
     * the tensor cores wait, and the routing kernel alone runs three. */
    DASH_FLAG_FUSE_ROUTE = 32
};

typedef struct {
    int batch;        /* B */
    int heads_q;      /* H_q */
    int heads_kv;     /* H_kv */
    int seq_len;      /* prefill: T.  decode: cache capacity (tokens per sequence). */
    int head_dim;     /* D */
    int chunk_size;   /* Bc */
    float alpha;      /* entmax alpha >= 1 (1 = softmax routing, 1.5 default, 2 = sparsemax) */
    float gamma;      /* Stage 1 score factor (1.0 default) */
    float sigma;      /* prior strength: bias = sigma * log p (1.0 default) */
    int enable_gqa;   /* nonzero: heads_q may be a multiple of heads_kv */
    unsigned flags;   /* DASH_FLAG_* */
    int topk;         /* 0: alpha-entmax routing.  k > 0: top-k routing instead -- the fixed-k
                         block selection of the hierarchical baselines the pages compare
                         against (liuzhao09.github.io "DashAttention 精读", sections 1-2): each
                         row attends the k chunks c < c_t with the highest Stage 1 scores (all
                         of them when c_t <= k; the lower index first on equal scores) and its
                         diagonal chunk, with a uniform prior (bias 0; alpha and sigma unused);
                         p is 1/min(k, c_t) on the selection, tau the lowest selected score.
                         Not combinable with DASH_FLAG_ESTIMATE_DIAGONAL. */
} dash_params_t;

/* Bytes of device workspace dash_prefill uses for these parameters (assuming summary_k and
 * active_blocks are passed as NULL; they are then kept in the workspace), including the V^T
 * scratch that dash_attend_workspace_size describes.  dash_prefill also accepts a workspace
 * without that scratch (status, tau and the NULL-passed summaries and mask only); Stage 2
 * then runs on the 64-key-block tensor-core kernel, about 10% slower.  0 on bad
 * parameters. */
size_t dash_prefill_workspace_size(const dash_params_t *params);

/* Whole causal prefill: Stage 0 -> Stage 1 -> Stage 2, stream-ordered, no host syncs.
 *   q        [B, H_q, T, D]   bf16 (in)
 *   k, v     [B, H_kv, T, D]  bf16 (in)
 *   head_cls [H_kv, D]        fp32 (in) the learned Stage 0 query of each KV head
 *   out      [B, H_q, T, D]   bf16 (out)
 *   summary_k [B, H_kv, T/Bc, D] fp32 (out, nullable) the chunk-representation cache
 *   p        [B, H_kv, T, C]  fp32 (out, nullable) routing probabilities, C = ceil(T/Bc);
 *            0 for c > c_t and for inactive chunks; p[.., c_t] = 0 (the diagonal is not
 *            routed) unless DASH_FLAG_ESTIMATE_DIAGONAL gives it its estimated probability
 *   active_blocks [B, H_kv, T, W] uint64 (out, nullable), W = ceil(C/64); bit c % 64 of word
 *            c / 64 (LSB first) is set iff chunk c is attended by row t (routed-active or
 *            the diagonal); bits above c_t are 0
 *   ws, ws_bytes: device workspace, dash_prefill_workspace_size(params) bytes for the fast path;
 *            its first 256 bytes hold the device status word (cleared by this call)
 * Returns DASH_OK when every launch was issued. */
dash_status_t dash_prefill(const dash_params_t *params, const void *q, const void *k,
                           const void *v, const float *head_cls, void *out, float *summary_k,
                           float *p, uint64_t *active_blocks, void *ws, size_t ws_bytes,
                           void *stream);

/* The same causal prefill with its inputs and output in host memory, the copies overlapped
 * with the computation (gist.science DashAttention summary, "Stufe 2": row t attends only keys
 * <= t, so rows [0, r) can finish before the queries of later rows arrive).
 *   q_host, k_host, v_host, head_cls_host, out_host: host buffers of the dash_prefill shapes;
 *            page-locked (cudaHostAlloc / cudaHostRegister) for the copies to overlap
 *   q, k, v, head_cls, out: device buffers of the same shapes, owned by the caller (the
 *            library allocates no memory); head_cls/head_cls_host may be NULL with
 *            DASH_FLAG_DENSE
 *   ws, ws_bytes: at least dash_prefill_workspace_size(params) bytes (the V^T scratch is
 *            what lets the rows be sliced)
 *   n_slices: row slices (1 = no overlap; at most 64 are used); each slice but the last is
 *            a multiple of 128 rows.  With the 128-key-block Stage 2 kernel unavailable for
 *            these parameters the call runs as one slice.
 *   stream:  computation; h2d_stream, d2h_stream: the two copy directions.  All three must
 *            be distinct streams of the current device.  Both copy streams first wait for
 *            the work already queued on stream.  Order on h2d_stream: head_cls, then per
 *            slice its q rows, preceded where one starts by a piece of k and v rows (pieces
 *            of 1, 2, 4, ... slices: rows below t route and attend only to keys below t).
 *            On stream: per piece of keys, Stage 0 on the chunks it completes and the V^T
 *            transpose of its rows; Stages 1-2 of each slice once its q has arrived.  Out of
 *            each slice back to out_host on d2h_stream once computed.  stream finally waits
 *            for the last copy, so synchronising stream covers the whole call.
 * The device output equals dash_prefill's bit for bit.  Creates and destroys its CUDA events
 * (3 * slices + 2) within the call.  Returns DASH_OK when every copy and launch was issued,
 * DASH_ERR_INVALID_ARGUMENT for a NULL buffer or n_slices < 1. */
dash_status_t dash_prefill_host(const dash_params_t *params, const void *q_host,
                                const void *k_host, const void *v_host,
                                const float *head_cls_host, void *out_host, void *q, void *k,
                                void *v, float *head_cls, void *out, void *ws, size_t ws_bytes,
                                int n_slices, void *stream, void *h2d_stream, void *d2h_stream);

/* Stage 0 alone: summary_k [B, H_kv, T/Bc, D] fp32 of every complete chunk of k
 * [B, H_kv, T, D] bf16.  Each summary is computed by one warp from a TMA (bulk-copy) staged
 * chunk in shared memory.  ws (>= 256 bytes) holds the status word.  summary_k may be NULL
 * when T < chunk_size (no complete chunk). */
dash_status_t dash_stage0(const dash_params_t *params, const void *k, const float *head_cls,
                          float *summary_k, void *ws, size_t ws_bytes, void *stream);

/* Stage 1 alone: routing of every row from q [B,H_q,T,D] bf16 and summary_k
 * [B,H_kv,T/Bc,D] fp32.  Writes tau [B,H_kv,T] fp32 (the entmax threshold of each row;
 * the log-sum-exp when alpha = 1; NaN when c_t = 0), active_blocks [B,H_kv,T,W] uint64,
 * and p [B,H_kv,T,C] fp32 when non-NULL.  ws (>= 256 bytes) holds the status word.
 * DASH_FLAG_ESTIMATE_DIAGONAL returns DASH_ERR_UNSUPPORTED here (use dash_prefill). */
dash_status_t dash_route(const dash_params_t *params, const void *q, const float *summary_k,
                         float *tau, float *p, uint64_t *active_blocks, void *ws,
                         size_t ws_bytes, void *stream);

/* Workspace bytes dash_attend uses with these params: 256 (the status word) plus, when the
 * 128-key-block tensor-core kernel applies (head_dim 128, 8 <= G <= 128 query heads per KV
 * head with 128 % G == 0, chunk_size 64 or 128), a V^T copy of v, B*H_kv*128*roundup(T,8)*2
 * bytes rounded up to 256, written by the call.  dash_attend runs correctly with any
 * ws_bytes >= 256; below this size it takes the 64-key-block kernel.  0 on bad params. */
size_t dash_attend_workspace_size(const dash_params_t *params);

/* Stage 2 alone: out [B,H_q,T,D] bf16 from q, k, v, the routing (summary_k, tau,
 * active_blocks as written by dash_stage0 / dash_route) and the flags (DASH_FLAG_DENSE and
 * DASH_FLAG_FORCE_ALL_ACTIVE ignore the routing, which may then be NULL).  The bias of an
 * active chunk is recomputed from (qbar.summary, tau) bit-identically to Stage 1. */
dash_status_t dash_attend(const dash_params_t *params, const void *q, const void *k,
                          const void *v, const float *summary_k, const float *tau,
                          const uint64_t *active_blocks, void *out, void *ws, size_t ws_bytes,
                          void *stream);

/* Name of the Stage 2 kernel dash_attend launches for these parameters with a workspace of
 * ws_bytes (dash_prefill with the same flags and a workspace that leaves ws_bytes after its
 * status word, tau, summaries and mask words picks the same one): "k_attend_pair" (dense
 * modes on pairs of SMs), "k_attend_fa" (128-key blocks), "k_attend_tc" (64-key blocks, no
 * V^T scratch), "k_attend" (warp-level MMA: head_dim 64, a single query head per KV head,
 * or tiles of 128/G tokens that would span two chunks) or "k_attend_fa|k_attend" (chosen at
 * run time, see dash_stage2_kernel_ran).  Host only, launches nothing; "" on bad parameters
 * or ws_bytes < 256.  Static storage. */
const char *dash_attend_kernel_name(const dash_params_t *params, size_t ws_bytes);

/* After a dash_prefill or dash_attend call with workspace ws, on `stream` (synchronised
 * here): the Stage 2 kernel a run-time choice ran, "k_attend_fa" or "k_attend", or "" if that
 * call made no run-time choice.  dash_attend_kernel_name reports "k_attend_fa|k_attend" for
 * calls that choose at run time: routed, full-range calls with 2 or 4 query heads per KV
 * head, where a small kernel first counts from the mask words the token-chunk pairs each
 * kernel would execute (the 128-key-block kernel walks the union of 128/G tokens' chunks,
 * the warp-MMA kernel of 16/G tokens'), both kernels are launched, and every CTA of the
 * one with the larger estimated time exits at once.  Static storage. */
const char *dash_stage2_kernel_ran(void *ws, void *stream);

/* Number of kernels one dash_prefill call with these parameters launches when its workspace
 * is ws_bytes and the caller passes neither summary_k nor active_blocks: Stage 0, Stage 1
 * (absent where the 128-key-block kernel routes its own tiles), the V^T transpose (for the
 * 128-key-block kernels) and Stage 2 (with a run-time choice: the cost kernel and both Stage 2
 * kernels).  Host only; 0 on bad parameters. */
int dash_prefill_kernel_count(const dash_params_t *params, size_t ws_bytes);

/* Chunk-representation cache update for decode: Stage 0 over each sequence's last n_recent
 * complete chunks.  Idempotent (recomputing a frozen chunk writes the same bits).
 *   k_cache       [B, H_kv, cap, D] bf16 (in), cap = params->seq_len
 *   seq_lens      [B] int32 DEVICE (in): valid tokens per sequence, 1 <= seq_lens[b] <= cap
 *   summary_cache [B, H_kv, cap/Bc, D] fp32 (in/out)
 * The summaries are bit-identical to dash_stage0's for the same keys.  A seq_lens value out
 * of range is reported through the status word in ws and that sequence is skipped. */
dash_status_t dash_update_chunk_cache(const dash_params_t *params, const void *k_cache,
                                      const float *head_cls, const int32_t *seq_lens,
                                      int n_recent, float *summary_cache, void *ws,
                                      size_t ws_bytes, void *stream);

/* Bytes of device workspace dash_decode needs (status word + split partial results). */
size_t dash_decode_workspace_size(const dash_params_t *params);

/* One incremental-decode step: for each sequence b the query row is t = seq_lens[b]-1,
 * whose K/V the caller has already written into the caches, and whose routable chunks
 * (c < t / Bc) have summaries in summary_cache (see dash_update_chunk_cache).
 *   q            [B, H_q, D] bf16 (in)
 *   k_cache, v_cache [B, H_kv, cap, D] bf16 (in)
 *   seq_lens     [B] int32 DEVICE (in)
 *   summary_cache [B, H_kv, cap/Bc, D] fp32 (in)
 *   head_cls     [H_kv, D] fp32 (in; only read with DASH_FLAG_ESTIMATE_DIAGONAL, may be NULL
 *                without it)
 *   out          [B, H_q, D] bf16 (out)
 *   p            [B, H_kv, Ccap] fp32 (out, nullable), Ccap = ceil(cap/Bc)
 *   active_blocks [B, H_kv, Wcap] uint64 (out, nullable), Wcap = ceil(Ccap/64)
 * Same arithmetic as row t of dash_prefill.  One thread-block cluster per (b, g) routes
 * and attends; no host sync, so a loop of steps can be captured in one CUDA graph. */
dash_status_t dash_decode(const dash_params_t *params, const void *q, const void *k_cache,
                          const void *v_cache, const int32_t *seq_lens,
                          const float *summary_cache, const float *head_cls, void *out,
                          float *p, uint64_t *active_blocks, void *ws, size_t ws_bytes,
                          void *stream);

/* Paged KV cache (the serving layout the pages name as the first gap of the reference kernels,
 * liuzhao09.github.io "DashAttention 精读", section 7): the cache lives in pools of pages of
 * one chunk each, and a per-sequence block table maps logical chunk c of sequence b to its page.
 *   k_pool, v_pool [n_pages, H_kv, Bc, D] bf16; summary_pool [n_pages, H_kv, D] fp32 (the
 *   summary of the chunk held by the page); block_table [B, max_blocks] int32 DEVICE, entry
 *   (b, c) the page of chunk c of sequence b (only chunks 0 .. (seq_lens[b]-1)/Bc are read);
 *   params->seq_len must equal max_blocks * chunk_size (the capacity per sequence).
 * A page index outside [0, n_pages) is reported as DASH_ERR_INVALID_ARGUMENT through the
 * status word and that sequence is skipped.  Otherwise the same arithmetic and outputs as
 * dash_update_chunk_cache / dash_decode on the gathered contiguous cache. */
dash_status_t dash_update_chunk_cache_paged(const dash_params_t *params, const void *k_pool,
                                            const float *head_cls, const int32_t *block_table,
                                            int max_blocks, int n_pages, const int32_t *seq_lens,
                                            int n_recent, float *summary_pool, void *ws,
                                            size_t ws_bytes, void *stream);
dash_status_t dash_decode_paged(const dash_params_t *params, const void *q, const void *k_pool,
                                const void *v_pool, const int32_t *block_table, int max_blocks,
                                int n_pages, const int32_t *seq_lens, const float *summary_pool,
                                const float *head_cls, void *out, float *p,
                                uint64_t *active_blocks, void *ws, size_t ws_bytes,
                                void *stream);

/* Bytes of device workspace dash_decode_step / dash_decode_step_paged need (the status word
 * and one counter per sequence).  The workspace must be zero-filled before its first step;
 * every step leaves its counters at zero again. */
size_t dash_decode_step_workspace_size(const dash_params_t *params);

/* A whole decode step in one launch (liuzhao09.github.io "DashAttention 精读", section 2:
 * incremental decoding with the chunk-representation cache): for each sequence b with
 * L = seq_lens[b] tokens in the cache,
 *   1. k_new[b], v_new[b] ([B, H_kv, D] bf16, in) are written into row L of the caches;
 *   2. the query q[b] is routed and attends exactly as dash_decode with seq_lens[b] = L + 1;
 *   3. if L + 1 is a multiple of chunk_size, the chunk it completes gets its summary in
 *      summary_cache (bit-identical to dash_update_chunk_cache's);
 *   4. seq_lens[b] (int32 DEVICE, in/out) becomes L + 1.
 * k_cache, v_cache and summary_cache are in/out; head_cls [H_kv, D] fp32 is required; L + 1
 * must not exceed the capacity (params->seq_len), else DASH_ERR_INVALID_ARGUMENT through
 * the status word and the sequence is left unchanged.  The other arguments as dash_decode.
 * The step reads seq_lens[b] before any write, so a loop of steps needs no host work between
 * them and can be captured in one CUDA graph.  ws: dash_decode_step_workspace_size bytes,
 * zero-filled before the first step.  Unlike the other entry points the step does not clear
 * the status word (it is one launch, with no memset before it): the first error of any step
 * since the last dash_read_device_status stays in it, so one read after a loop of steps (or
 * a graph replay) covers all of them. */
dash_status_t dash_decode_step(const dash_params_t *params, const void *q, const void *k_new,
                               const void *v_new, void *k_cache, void *v_cache, int32_t *seq_lens,
                               float *summary_cache, const float *head_cls, void *out, float *p,
                               uint64_t *active_blocks, void *ws, size_t ws_bytes, void *stream);
/* The same on a paged cache (pools, block table and capacity as dash_decode_paged; the page
 * of the chunk that holds row L must already be in the block table). */
dash_status_t dash_decode_step_paged(const dash_params_t *params, const void *q,
                                     const void *k_new, const void *v_new, void *k_pool,
                                     void *v_pool, const int32_t *block_table, int max_blocks,
                                     int n_pages, int32_t *seq_lens, float *summary_pool,
                                     const float *head_cls, void *out, float *p,
                                     uint64_t *active_blocks, void *ws, size_t ws_bytes,
                                     void *stream);

/* Bytes of device workspace dash_backward needs (the routing it recomputes with p, the
 * gradient into p, per-row softmax statistics, group-mean queries, the routing transposed to
 * per-chunk token lists, and the summaries' gradient).  0 on bad parameters. */
size_t dash_backward_workspace_size(const dash_params_t *params);

/* Backward pass of the causal prefill: the gradients of L = sum(out * dout) with respect to q,
 * k, v and head_cls, through Stage 2 (the attention and its prior bias sigma * log p), Stage 1
 * (the alpha-entmax routing: its Jacobian on the support) and Stage 0 (the chunk summaries).
 * gist.science "DashAttention ..." summary, "Stufe 1": alpha-entmax is differentiable, so the
 * gradient flows from the Stage 2 softmax through the routing back to the summaries of Stage 0.
 *   q, k, v, head_cls: the forward's inputs (layouts of dash_prefill); out: its output;
 *   dout [B, H_q, T, D] bf16: the gradient of L with respect to out;
 *   dq [B, H_q, T, D], dk, dv [B, H_kv, T, D], dhc [H_kv, D] fp32 (out, overwritten; dhc sums
 *   over the batch).
 * The default routing only: DASH_FLAG_DENSE, DASH_FLAG_FORCE_ALL_ACTIVE,
 * DASH_FLAG_ESTIMATE_DIAGONAL and top-k return DASH_ERR_UNSUPPORTED.  Probabilities are
 * recomputed in fp32 (not rounded to bf16 as in the forward's P V); the gradient operands of
 * the warp-level MMAs are rounded to bf16. */
dash_status_t dash_backward(const dash_params_t *params, const void *q, const void *k,
                            const void *v, const float *head_cls, const void *out,
                            const void *dout, float *dq, float *dk, float *dv, float *dhc,
                            void *ws, size_t ws_bytes, void *stream);

/* Size of the device array that dash_prefill_static_ws uses as its workspace. */
#define DASH_STATIC_WS_BYTES (16u << 20)

/* dash_prefill for callers that cannot allocate device memory.  The paper has no
 * counterpart to this entry point: it exists for callers such as a plugin inside a host
 * application that owns all device memory through its own pool, or a loop on a latency
 * budget that cannot afford cudaMalloc's blocking.  Same arguments, arithmetic and outputs as dash_prefill, but no
 * workspace: the scratch (status word, tau, and the summaries / mask words not supplied by
 * the caller) lives in one file-scope device array of DASH_STATIC_WS_BYTES, reserved on
 * every GPU that loads the library and held until exit.
 *   - Sizes whose scratch exceeds DASH_STATIC_WS_BYTES return DASH_ERR_WORKSPACE_TOO_SMALL
 *     before anything runs; passing summary_k and active_blocks shrinks the need to the
 *     status word plus tau (B*H_kv*T*4 bytes).
 *   - Every call made outside a stream capture looks up the array's device address with the
 *     call's device current (so it stays right after a reset of the device's primary
 *     context); a call made while `stream` is being captured uses the address the last
 *     uncaptured call on that device found.  Make the first call on each device before any
 *     stream capture: a captured first call returns DASH_ERR_CUDA.
 *   - Every call shares the array and leaves its contents behind; the status word is cleared
 *     per call and the rest is fully written before it is read.  Calls that overlap on the
 *     GPU race on the array: order them.
 *   - Faults found on the device go to the status word inside the array; read them with
 *     dash_static_ws_read_status.
 * Nothing here calls cudaMalloc, cudaFree or any allocating routine. */
dash_status_t dash_prefill_static_ws(const dash_params_t *params, const void *q, const void *k,
                                     const void *v, const float *head_cls, void *out,
                                     float *summary_k, float *p, uint64_t *active_blocks,
                                     void *stream);

/* The device status word of dash_prefill_static_ws: synchronises `stream` (the stream of the
 * calls to check), then returns the status the kernels wrote into the library's static array
 * (DASH_OK if none) and clears it.  Like the entry point it pairs with, it allocates nothing,
 * and the paper has no counterpart to it.  Returns DASH_ERR_CUDA if the synchronisation or
 * the copy fails (or on a device where dash_prefill_static_ws was never called outside a
 * stream capture while `stream` is being captured). */
dash_status_t dash_static_ws_read_status(void *stream);

/* Synchronises `stream`, then returns the status word the kernels wrote into ws (DASH_OK if
 * none) and clears it.  Returns DASH_ERR_CUDA if the copy itself fails. */
dash_status_t dash_read_device_status(void *ws, void *stream);

/* Human-readable name of a status code (static storage). */
const char *dash_status_string(dash_status_t status);

#ifdef __cplusplus
}
#endif

#endif /* DASH_H_ */
