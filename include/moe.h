/*
 * moe.h -- C ABI of libmoe.so: the single-GPU MoE routing hot path on B200
 * (sm_100a): top-k gate -> layout -> dispatch -> combine.
 *
 * Pages cited (title, then section):
 *   [pplx]  "Efficient and portable mixture-of-experts communication"
 *           (Perplexity Research): Introduction; Sharding and parallelism;
 *           Portable kernels; Dispatch; Combine.
 *   [EPv2]  DeepEP V2 release summary (hi.news.hada.io, "DeepSeek ने MoE
 *           training और inference के लिए open source DeepEP लाइब्रेरी जारी
 *           की"): "ElasticBuffer interface"; "training / prefill / decoding
 *           usage patterns".
 *   [EPv1]  "DeepSeek, DeepEP 오픈소스 공개" (GeekNews): Topic Body;
 *           성능 / 일반 커널 (normal kernels).
 *   [TK]    DeepSeek Tile-Kernels / DeepEP V2 news (deepinsightai.io):
 *           "Funktionen der DeepSeek-Tile-Kernel".
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Ownership: every array argument is DEVICE memory owned by the caller.
 *    The library allocates nothing, frees nothing and keeps no state between
 *    calls, so the layout outputs can be kept and reused as the "cached
 *    handle" of [EPv2] usage patterns (routing metadata reused while the
 *    gating does not change).
 *  - Streams: `stream` is a cudaStream_t passed as an opaque pointer (NULL is
 *    the legacy default stream).  Calls only enqueue work on it: they never
 *    synchronise with the host and return before the GPU work finishes.
 *  - Host-side errors: arguments are checked before anything is launched; a
 *    failed check returns MOE_ERR_INVALID_ARG (bad value, NULL pointer,
 *    misalignment) or MOE_ERR_UNSUPPORTED (beyond a documented limit) and
 *    enqueues nothing.  A launch the CUDA runtime rejects returns
 *    MOE_ERR_CUDA.
 *  - Device-side errors: an index found out of range by a kernel is skipped
 *    and, when `d_status` is not NULL, MOE_ERR_BAD_INDEX is stored to
 *    *d_status (one int32 in device memory that the caller zeroes and reads
 *    after the stream work finished).  No kernel traps or asserts.  Kernels
 *    that wait on in-flight copies bound every wait to one second; a wait
 *    that runs out stores MOE_ERR_TIMEOUT, lets the copies it issued land
 *    and returns (its output is then incomplete).
 *  - Sizes: N = num_tokens, H = hidden, E = num_experts, k = experts per
 *    token, R = logical EP ranks, S = N*k receive rows.  Row-major layouts.
 *    Byte offsets are 64-bit; S must stay below 2^31 (int32 slot ids).
 *  - Index -1 in topk_idx / token_slot marks a masked slot: it is skipped
 *    without an error.  Any other id outside range is MOE_ERR_BAD_INDEX.
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,
    MOE_ERR_UNSUPPORTED = 2,
    MOE_ERR_CUDA = 3,
    MOE_ERR_BAD_INDEX = 4,
    MOE_ERR_TIMEOUT = 5          /* a kernel's bounded wait gave up (device status only) */
} moe_status_t;

typedef enum {
    MOE_GATE_SOFTMAX = 0,        /* w_j = softmax(logits)[sel_j]                     */
    MOE_GATE_SOFTMAX_RENORM = 1, /* w_j = p_sel_j / sum_j' p_sel_j'                  */
    MOE_GATE_SIGMOID_GROUP = 2   /* DeepSeek-V3 group-limited sigmoid gating         */
} moe_gate_kind_t;

typedef enum {
    MOE_DTYPE_BF16 = 0,          /* payload copied as bf16                              */
    MOE_DTYPE_FP8_E4M3 = 1,      /* e4m3, one fp32 scale per 128 channels               */
    MOE_DTYPE_FP8_E4M3_TOKEN = 2,/* e4m3, one fp32 scale per token row                  */
    MOE_DTYPE_MXFP8_E4M3 = 3,    /* OCP MXFP8: e4m3, one E8M0 scale byte per 32 channels */
    MOE_DTYPE_NVFP4 = 4,         /* e2m1, one e4m3 scale per 16 channels + fp32 per row  */
    MOE_DTYPE_E5M6 = 5,          /* 12-bit float (FP16 minus 4 fraction bits), no scale  */
    MOE_DTYPE_FP8_E4M3_UE8M0 = 6 /* e4m3, one power-of-two (UE8M0 byte) scale per 128     */
} moe_dtype_t;

/* Where the receive scales go (moe_dispatch_ex).  Scale (s, b) is that of
 * receive row s and scale block b; a row has B blocks (H/128 per-block FP8,
 * 1 per-token FP8, H/32 MXFP8). */
typedef enum {
    MOE_SCALE_ROW_MAJOR = 0,     /* element s*B + b                                      */
    MOE_SCALE_MN_MAJOR = 1,      /* element b*ld + s, ld = S padded to 16 bytes of scales */
    MOE_SCALE_MMA_TILED = 2,     /* E8M0 only: block-scaled MMA scale-factor atoms        */
    MOE_SCALE_MN_MAJOR_PACK4 = 3 /* UE8M0 only: 4 blocks per 32-bit word, words MN-major  */
} moe_scale_layout_t;

typedef void* moe_stream_t;      /* a cudaStream_t */

#define MOE_MAX_EXPERTS 1024
#define MOE_MAX_TOPK 32
#define MOE_FP8_BLOCK 128
#define MOE_MAX_ALIGN 4096

/*
 * moe_topk_gate -- router top-k selection and weights.
 *   [pplx] Introduction: the router turns the token's logits into a
 *   probability distribution, the top-K experts are taken and their outputs
 *   are averaged with the router's weights.  [TK]: top-k selection, scoring
 *   and weight normalisation.  [EPv1] Topic Body / normal kernels: DeepSeek-V3
 *   group-limited gating with top-4 groups and top-8 experts.
 *
 *   logits   fp32 [N, E] row-major (read only).
 *   kind     MOE_GATE_SOFTMAX / _RENORM: p = softmax(logits) with
 *            e_i = exp(l_i - max l) and Z summed in ascending expert order;
 *            selection on the logits (softmax is increasing).
 *            MOE_GATE_SIGMOID_GROUP: s = sigmoid(logit); E experts in
 *            n_groups consecutive groups; group score = sum of the
 *            group_topn largest s of the group (added largest first);
 *            the topk_groups best groups are kept; the k best s among the
 *            kept experts are selected; w_j = s_j / sum of the selected s
 *            (summed in slot order).  n_groups/topk_groups/group_topn are
 *            ignored by the softmax kinds.
 *   topk_idx int32 [N, k] out: expert ids, best first.  Ties go to the
 *            lower expert (or group) index.
 *   topk_w   fp32  [N, k] out: weights in the same order.
 *   exp is one fixed fp32 routine (Cody-Waite reduction + degree-7 Taylor,
 *   input clamped to [-87, 88]), so results are reproducible bit for bit.
 *   Limits: 1 <= E <= MOE_MAX_EXPERTS, 1 <= k <= min(E, MOE_MAX_TOPK);
 *   group kind: E % n_groups == 0, 1 <= topk_groups <= n_groups,
 *   1 <= group_topn <= E/n_groups, topk_groups*(E/n_groups) >= k.
 *   Pointers 4-byte aligned.  N == 0 enqueues nothing.
 */
moe_status_t moe_topk_gate(const float* logits, int num_tokens, int num_experts, int k,
                           moe_gate_kind_t kind, int n_groups, int topk_groups,
                           int group_topn, int32_t* topk_idx, float* topk_w,
                           moe_stream_t stream);

/* Bytes of device scratch moe_get_layout needs for these sizes (>= 256). */
size_t moe_layout_workspace_bytes(int num_tokens, int k, int num_experts, int num_ranks);

/*
 * moe_get_layout -- per-expert / per-rank counts, offsets and the
 * token<->slot maps of the expert-contiguous receive buffer.
 *   [EPv2] usage patterns: the dispatch handle carries the routing metadata
 *   for combine and the per-expert received-token counts for the grouped
 *   GEMM.  [pplx] Dispatch: tokens land in one contiguous per-expert buffer
 *   and the source token of every row is kept for combine.  [pplx] Sharding:
 *   experts are sharded over EP ranks, rank r owning experts
 *   [r*E/R, (r+1)*E/R); here ranks are partitions of one buffer.
 *
 *   topk_idx      int32 [N, k] in (from moe_topk_gate or the caller).
 *   expert_count  int32 [E]    rows per expert.
 *   expert_offset int32 [E+1]  exclusive prefix sum; expert_offset[E] = valid rows.
 *   rank_count    int32 [R]    rows per logical rank.
 *   rank_offset   int32 [R+1]  = expert_offset[r*E/R]; rank_offset[R] = valid rows.
 *   rank_tokens   int32 [R]    tokens with at least one expert on rank r.
 *   token_slot    int32 [N, k] receive row of (token, j); -1 if masked/invalid.
 *   slot_token    int32 [S]    source token of every receive row; the tail rows
 *                              [expert_offset[E], S) (masked entries) hold -1.
 *   Order inside an expert is ascending token id, then slot j: the result is
 *   deterministic (the pages leave the receive order open).
 *   workspace     device scratch of moe_layout_workspace_bytes() bytes, 16-byte
 *                 aligned; contents need no initialisation and are not kept.
 *   Limits: 1 <= E <= MOE_MAX_EXPERTS, 1 <= k <= MOE_MAX_TOPK, E % R == 0.
 *   The receive buffer of this (packed) layout has S = N*k rows; pass S as
 *   num_recv_rows to the calls below.
 */
moe_status_t moe_get_layout(const int32_t* topk_idx, int num_tokens, int k,
                            int num_experts, int num_ranks, int32_t* expert_count,
                            int32_t* expert_offset, int32_t* rank_count,
                            int32_t* rank_offset, int32_t* rank_tokens,
                            int32_t* token_slot, int32_t* slot_token, void* workspace,
                            size_t workspace_bytes, int32_t* d_status, moe_stream_t stream);

/* Receive rows an aligned layout may need: N*k + E*(align - 1); 0 when an
 * argument is out of range (N < 0, k < 1, E < 1, align < 1). */
size_t moe_aligned_recv_rows(int num_tokens, int k, int num_experts, int align);

/*
 * moe_get_layout_aligned -- the layout with every expert's rows starting at a
 * multiple of `align` (1 <= align <= MOE_MAX_ALIGN), so a grouped GEMM can
 * tile each expert by align rows.  [EPv2] ElasticBuffer interface mentions a
 * new GEMM layout without defining it; this is the reading taken.
 *   expert_offset[e] = sum_{e' < e} round_up(expert_count[e'], align);
 *   rank_offset[r]   = expert_offset[r*E/R], rank_count[r] = the rows of rank
 *                      r's region (padding included);
 *   token_slot, slot_token and rank_tokens as in moe_get_layout, except that
 *   slot_token has num_recv_rows entries and is -1 on every row no token
 *   lands in (padding, masked tail, spare rows).
 *   num_recv_rows >= moe_aligned_recv_rows(N, k, E, align), else
 *   MOE_ERR_INVALID_ARG; align outside [1, MOE_MAX_ALIGN] is
 *   MOE_ERR_INVALID_ARG, and a padded layout of 2^31 rows or more
 *   MOE_ERR_UNSUPPORTED.  align = 1 is exactly moe_get_layout.
 */
moe_status_t moe_get_layout_aligned(const int32_t* topk_idx, int num_tokens, int k,
                                    int num_experts, int num_ranks, int align,
                                    int num_recv_rows, int32_t* expert_count,
                                    int32_t* expert_offset, int32_t* rank_count,
                                    int32_t* rank_offset, int32_t* rank_tokens,
                                    int32_t* token_slot, int32_t* slot_token, void* workspace,
                                    size_t workspace_bytes, int32_t* d_status,
                                    moe_stream_t stream);

/*
 * moe_get_layout_noalloc -- moe_get_layout without a caller-provided
 * workspace.  The pages have no counterpart: this is an addition for callers
 * that cannot allocate device memory, such as serving runtimes that reserve
 * all of the GPU's memory for their own pool at start-up, or deployments
 * whose memory plan is fixed before the first request; cudaMalloc there
 * fails or breaks the budget.  The scratch is a fixed array of
 * MOE_LAYOUT_NOALLOC_SCRATCH_BYTES in the library's device memory, held by
 * every GPU that loads the library until the process exits.
 *   Arguments, outputs and results are those of moe_get_layout.  The call
 *   allocates nothing.  It returns MOE_ERR_UNSUPPORTED, enqueueing nothing,
 *   when moe_layout_workspace_bytes(N, k, E, R) exceeds the array.
 *   The first call on a device looks up the array's address (once per
 *   device, with that device current); make that first call before any
 *   stream capture.  All calls share the one array and it keeps the last
 *   call's contents (nothing in it needs clearing): calls whose GPU work
 *   overlaps -- other streams, other host threads -- race on it, so
 *   serialise them.
 */
#define MOE_LAYOUT_NOALLOC_SCRATCH_BYTES (1u << 20)
moe_status_t moe_get_layout_noalloc(const int32_t* topk_idx, int num_tokens, int k,
                                    int num_experts, int num_ranks, int32_t* expert_count,
                                    int32_t* expert_offset, int32_t* rank_count,
                                    int32_t* rank_offset, int32_t* rank_tokens,
                                    int32_t* token_slot, int32_t* slot_token, int32_t* d_status,
                                    moe_stream_t stream);

/* Bytes of device workspace moe_route needs for these sizes (a multiple of
 * 256).  Its first 256 bytes must be zero before the first call (cudaMemset
 * the whole buffer once); every call leaves them zero. */
size_t moe_route_workspace_bytes(int num_tokens, int k, int num_experts, int num_ranks);

/*
 * moe_route -- moe_topk_gate and moe_get_layout_aligned in one call: the
 * routing decision and the dispatch handle come out of one enqueue.
 * [EPv2] usage patterns: build the routing handle on the GPU without a CPU
 * synchronisation and reuse it for dispatch and combine; DeepGEMM "Mega MoE"
 * news: fewer, overlapped launches (programmatic dependent launch).
 *   Arguments and outputs are exactly those of the two calls (topk_idx and
 *   topk_w as moe_topk_gate writes them, the layout arrays as
 *   moe_get_layout_aligned writes them for those ids; align = 1 and
 *   num_recv_rows = N*k give the packed layout), and so are the results, bit
 *   for bit.
 *   workspace  moe_route_workspace_bytes(N, k, E, R) bytes, 16-byte aligned.
 *              The first 256 bytes hold an arrival counter: zero before the
 *              first call, left zero by every call; the rest is scratch.  Do
 *              not share it between calls whose GPU work overlaps.
 *   How: when N*k <= 1024 and E <= 512, one launch: each CTA gates 8 tokens
 *   and the CTA that arrives last on the counter builds the layout.
 *   Otherwise the gate launch and
 *   the layout's launches follow each other with programmatic dependent
 *   launch (for large batches three overlapped launches measured faster than
 *   a gate that also counts).
 *   prefetch   optional device buffer the caller reads next -- typically x,
 *              which moe_dispatch reads right after this call -- and its size
 *              in bytes (NULL / 0: none; 16-byte aligned, a multiple of 16
 *              bytes is used; at most the first 64 MiB).  While gating and
 *              layout run (latency-bound, little traffic) the kernels ask L2
 *              to fetch it, so the next kernel reads it from L2.  A hint
 *              only: it changes no result, and the buffer must simply be
 *              readable (it is fetched after this call's predecessors
 *              finished, as any read of the call would be).
 *   Errors as in the two calls (host checks of both, then d_status).
 */
moe_status_t moe_route(const float* logits, int num_tokens, int num_experts, int k,
                       moe_gate_kind_t kind, int n_groups, int topk_groups, int group_topn,
                       int num_ranks, int align, int num_recv_rows, int32_t* topk_idx,
                       float* topk_w, int32_t* expert_count, int32_t* expert_offset,
                       int32_t* rank_count, int32_t* rank_offset, int32_t* rank_tokens,
                       int32_t* token_slot, int32_t* slot_token, void* workspace,
                       size_t workspace_bytes, const void* prefetch, size_t prefetch_bytes,
                       int32_t* d_status, moe_stream_t stream);

/* Receive-buffer payload bytes: N*k rows of H bf16 (2 B) or e4m3 (1 B). */
size_t moe_recv_bytes(int num_tokens, int hidden, int k, moe_dtype_t dtype);
/* Scale bytes for the FP8 payloads: N*k rows of H/128 fp32 (per block), of one
 * fp32 (per token) or of H/32 E8M0 bytes (MXFP8); 0 for BF16. */
size_t moe_scale_bytes(int num_tokens, int hidden, int k, moe_dtype_t dtype);

/*
 * moe_dispatch -- scatter each token's row to all of its receive rows.
 *   [pplx] Dispatch: a token's activations (plus block scaling factors when
 *   quantised) go to every expert it was routed to.  [EPv2] usage patterns:
 *   BF16 and FP8 dispatch.  [TK]: per-block FP8 quantisation.
 *
 *   x           bf16 [N, H] in.
 *   token_slot  int32 [N, k] from moe_get_layout(_aligned).
 *   num_recv_rows  rows S of the receive buffer (N*k packed, the aligned
 *               layout's num_recv_rows otherwise); slots must lie in [-1, S).
 *   BF16:  recv_x bf16 [S, H]: recv_x[token_slot[t,j]] = x[t]; recv_scale unused.
 *          H % 8 == 0; x and recv_x 16-byte aligned.
 *   FP8:   recv_x e4m3 [S, H], recv_scale fp32 [S, H/128].  Per token and
 *          128-channel block: amax = max|x|, scale = amax/448,
 *          code = e4m3_rne_satfinite(x * (448/amax)) (fp32 divisions and
 *          product, IEEE rounding); zeros keep their sign (so an all-zero
 *          block gives scale 0 and zero codes).  H % 128 == 0; x, recv_x
 *          16-byte aligned, recv_scale 4-byte aligned.
 *   FP8 per token ([TK]: "pro Token"): recv_x e4m3 [S, H], recv_scale fp32
 *          [S, 1]: amax over the whole row, then the same rule as the
 *          blocks.  H % 8 == 0 and H <= 16384.
 *   MXFP8 (OCP Microscaling, the block-scaled FP8 of Blackwell's block-scaled
 *          MMA): recv_x e4m3 [S, H], recv_scale viewed as uint8 [S, H/32].
 *          Per 32-channel block: e = floor(log2(amax)) - 8 (clamped to
 *          [-127, 127], -127 for an all-zero block), scale byte e + 127,
 *          codes e4m3_rne_satfinite(x * 2^-e) (the power-of-two scaling is
 *          exact; values up to 511.x saturate to 448).  H % 32 == 0;
 *          recv_scale 16-byte aligned.
 *   FP8 with power-of-two scales (MOE_DTYPE_FP8_E4M3_UE8M0; [TK] lists
 *          power-of-two scales, the rule is a reading): per 128-channel
 *          block e = ceil(log2(amax / 448)) of the fp32 quotient (-127 for an
 *          all-zero block, clamped to [-127, 127]), scale byte e + 127,
 *          codes e4m3_rne_satfinite(x * 2^-e); recv_scale uint8 [S, H/128].
 *          H % 128 == 0, recv_scale 16-byte aligned.
 *   E5M6 ([TK]: E5M6 conversion; the format is not defined there, reading:
 *          IEEE-style 1-5-6 bits, bias 15, i.e. FP16 with its 4 lowest
 *          fraction bits dropped; round to nearest even, saturating to
 *          +-65024): recv_x uint8 [S, 3H/2], two 12-bit codes per 3 bytes
 *          (code 2i in bits 0..11 of the little-endian 24-bit group);
 *          recv_scale unused.  H % 32 == 0.
 *   Rows no slot names are not written.  A slot outside [-1, S) is skipped
 *   and reported through d_status.
 */
moe_status_t moe_dispatch(const void* x, int num_tokens, int hidden, int k,
                          const int32_t* token_slot, int num_recv_rows, moe_dtype_t dtype,
                          void* recv_x, void* recv_scale, int32_t* d_status,
                          moe_stream_t stream);

/*
 * moe_dispatch_ex -- moe_dispatch with the receive scales laid out for the
 * grouped GEMM that consumes them.  [EPv2] ElasticBuffer interface names a
 * new GEMM layout without defining it and [TK] lists batched transposes;
 * the reading taken is one of three places for the same values:
 *   MOE_SCALE_ROW_MAJOR  as moe_dispatch.
 *   MOE_SCALE_MN_MAJOR   per-block FP8, per-token FP8 or MXFP8: scale (s, b)
 *        at element b*ld + s with ld = S rounded up to 4 (fp32) or 16 (E8M0):
 *        each block's scales are contiguous over the rows, every column
 *        16-byte aligned -- the transposed (M-major) scale operand of a
 *        grouped GEMM.
 *   MOE_SCALE_MMA_TILED  MXFP8 with H % 128 == 0: the order in which the
 *        block-scaled tensor-core MMA takes scale factors.  Rows are padded
 *        to a multiple of 128; 128-row x 4-block atoms of 512 bytes follow
 *        each other row-major over (s/128, b/4); inside an atom, row s and
 *        block b sit at byte (s%32)*16 + ((s%128)/32)*4 + b%4.  With the
 *        aligned layout at align 128 every expert's scales are a contiguous
 *        run of whole atoms.
 *   MOE_SCALE_MN_MAJOR_PACK4  FP8 with UE8M0 scales: four consecutive blocks
 *        of a row form one 32-bit word (block 4j+i in byte i; bytes of
 *        blocks past H/128 are written as 0) and the words are MN-major,
 *        word (s, j) at j*ld + s with ld = S rounded up to 4 -- the packed
 *        power-of-two scale operand of a 1x128-scaled FP8 GEMM.
 *   recv_scale holds moe_recv_scale_bytes(S, H, dtype, scale_layout) bytes,
 *   16-byte aligned for the MN-major and tiled layouts.  Only positions of
 *   rows a token lands in are written.  A layout the payload type does not
 *   have (BF16 with any but row-major, per-block FP8 tiled) is
 *   MOE_ERR_INVALID_ARG.  Everything else is as in moe_dispatch.
 */
moe_status_t moe_dispatch_ex(const void* x, int num_tokens, int hidden, int k,
                             const int32_t* token_slot, int num_recv_rows, moe_dtype_t dtype,
                             moe_scale_layout_t scale_layout, void* recv_x, void* recv_scale,
                             int32_t* d_status, moe_stream_t stream);

/* Bytes of recv_scale for S receive rows in `scale_layout`; 0 for BF16 and
 * for a layout the payload type does not have. */
size_t moe_recv_scale_bytes(int num_recv_rows, int hidden, moe_dtype_t dtype,
                            moe_scale_layout_t scale_layout);

/*
 * moe_dispatch_nvfp4 -- moe_dispatch with an NVFP4 payload, the FP4 format of
 * Blackwell's block-scaled tensor-core MMA.  [EPv2] feature list (Hybrid-EP:
 * NVFP4 support) and [TK] (FP4 conversion) name the format without a rule;
 * the reading is two-level NVFP4 scaling with the token's row in place of
 * the tensor (the per-token mode of [TK]).  Per token t:
 *   amax_t = max |x[t,:]|, row scale g_t = amax_t / 2688 (= 448 * 6),
 *   inv_t = 2688 / amax_t; per block b of 16 channels:
 *   sb = e4m3((amax_b / 6) * inv_t) (0 for an all-zero block),
 *   codes e2m1(x * (inv_t / value(sb))), round to nearest even, saturating
 *   to +-6; zeros keep their sign.  Every operation is fp32, rounded once;
 *   x ~ e2m1 * value(sb) * g_t.
 *   recv_x            uint8 [S, H/2]: two codes per byte, channel 2i in the
 *                     low nibble (the operand order of FP4 MMA).
 *   recv_block_scale  e4m3 codes, one per 16 channels, in scale_layout
 *                     (moe_recv_scale_bytes(S, H, MOE_DTYPE_NVFP4, layout)
 *                     bytes); the tiled layout is the FP4 block-scaled MMA's.
 *   recv_row_scale    fp32 [S]: g of the token in each row.
 *   Limits: H % 64 == 0, H <= 16384; x, recv_x, recv_block_scale 16-byte
 *   aligned.  Slots, masks and errors as in moe_dispatch.
 */
moe_status_t moe_dispatch_nvfp4(const void* x, int num_tokens, int hidden, int k,
                                const int32_t* token_slot, int num_recv_rows,
                                moe_scale_layout_t scale_layout, void* recv_x,
                                void* recv_block_scale, float* recv_row_scale, int32_t* d_status,
                                moe_stream_t stream);

/*
 * moe_quant_fp8_channel -- per-(expert, channel) FP8 of the receive buffer,
 * for each expert's weight-gradient GEMM.  [TK] list: FP8 quantisation "pro
 * Kanal" and batched transposes, no formula; reading: an expert's rows are
 * the contracted dimension of dW_e = X_e^T dY_e, so one scale per (expert,
 * channel) factors out of it.  Per expert e and channel c over the landed
 * rows [expert_offset[e], expert_offset[e] + expert_count[e]):
 *   amax = max |x|, scale[e*H + c] = amax / 448,
 *   code = e4m3(x * (448 / amax)) (fp32, rounded once each; zeros keep
 *   their sign) -- the per-block rule with the block = one channel of one
 *   expert.
 *   recv           bf16 [S, H] in (S = num_rows); recv and out 16-byte aligned.
 *   expert_offset  int32 [E+1], expert_count int32 [E]: device arrays, e.g.
 *                  from moe_get_layout_aligned; an expert whose range leaves
 *                  [0, S) is skipped and reported through d_status.
 *   transpose      0: out e4m3 [S, H] row-major; 1: out e4m3 [H, S]
 *                  (channel-major, the K-major operand).
 *   scale          fp32 [E, H] out (0 for an expert with no rows).
 *   workspace      device scratch of at least
 *                  moe_quant_fp8_channel_workspace_bytes(E, H) bytes,
 *                  16-byte aligned, all zero before the first call; every
 *                  call leaves it zero again, so one zeroing serves all
 *                  later calls in stream order (one workspace per stream:
 *                  calls running at the same time need their own).  It is
 *                  used when the average expert holds 256 to 1023 of the S
 *                  rows: each expert's rows are then cut into parts of at
 *                  most 256 rows (64 parts at most) and a persistent grid
 *                  takes (expert, channel slab, part) tasks from a counter
 *                  in it, so a hot expert spreads over many CTAs, whose
 *                  parts combine their amax through it.  Otherwise, and when
 *                  NULL: one CTA, or a cluster of up to 8, per (expert,
 *                  slab), sized from the average rows per expert (no
 *                  scratch).  Both give the same bits.  A wait that outlasts
 *                  1 s sets MOE_ERR_TIMEOUT.
 *   Padding rows (outside every expert's landed range) are not written.
 *   H % 128 == 0, 1 <= E <= MOE_MAX_EXPERTS.
 */
moe_status_t moe_quant_fp8_channel(const void* recv, int num_rows, int hidden, int num_experts,
                                   const int32_t* expert_offset, const int32_t* expert_count,
                                   int transpose, void* out, float* scale, void* workspace,
                                   size_t workspace_bytes, int32_t* d_status, moe_stream_t stream);

/* Bytes of moe_quant_fp8_channel's workspace for E experts of H channels
 * (0 when E or H is outside that call's limits). */
size_t moe_quant_fp8_channel_workspace_bytes(int num_experts, int hidden);

/* 1 when moe_quant_fp8_channel over num_rows receive rows and E experts
 * uses a workspace it is given (the average expert holds 256 to 1023 rows),
 * 0 when it ignores it (or the sizes are outside its limits): a caller may
 * then pass NULL and allocate nothing. */
int moe_quant_fp8_channel_takes_workspace(int num_rows, int num_experts);

/*
 * moe_swiglu_quant -- SwiGLU between an expert's two GEMMs, fused with the
 * quantisation the second GEMM reads.  [TK] list: SwiGLU combined with the
 * quantisation operations (the formula is not on the pages; reading below).
 *   h           bf16 [S, 2I] in: row s = [gate | up], the first GEMM's output
 *               for receive row s (gate half first).
 *   slot_token  int32 [S] from moe_get_layout(_aligned), or NULL: rows with
 *               slot_token < 0 (padding) are skipped and their outputs left
 *               as they were.
 *   a_c = silu(g_c) * u_c with silu(g) = g / (1 + exp(-g)), in fp32 with
 *   every operation rounded once and exp the gate's fixed routine.
 *   out / out_scale: a as bf16 [S, I] (dtype BF16, out_scale unused), or
 *   e4m3 [S, I] with scales exactly as moe_dispatch_ex produces them from a
 *   row (per-128-block FP8, per-row FP8, MXFP8) with the fp32 a in place of
 *   the bf16 input, in `scale_layout` over S rows (moe_recv_scale_bytes(S,
 *   I, dtype, scale_layout) bytes).
 *   Limits: I % 16 == 0 (BF16), % 128 (FP8 per block), % 8 and <= 16384
 *   (per row), % 32 (MXFP8; % 128 for the tiled scales); h and out 16-byte
 *   aligned; out_scale aligned as in moe_dispatch_ex.  S == 0 enqueues
 *   nothing.
 */
moe_status_t moe_swiglu_quant(const void* h, int num_rows, int inter, const int32_t* slot_token,
                              moe_dtype_t dtype, moe_scale_layout_t scale_layout, void* out,
                              void* out_scale, moe_stream_t stream);

/*
 * moe_combine -- weighted gather-reduce of each token's k expert outputs.
 *   [pplx] Introduction and Combine: the output is the average of the
 *   selected experts' outputs weighted by the router weights; [EPv2] usage
 *   patterns: combine reduces expert outputs back to the token.
 *
 *   y          bf16 [S, H] expert outputs, one row per receive slot (S =
 *              num_recv_rows, see moe_dispatch).
 *   token_slot int32 [N, k], topk_w fp32 [N, k].
 *   out        bf16 [N, H]:  acc = +0.0f; for j = 0..k-1 (slot order):
 *              acc = fmaf(topk_w[t,j], y[token_slot[t,j], c], acc);
 *              out = bf16 round-to-nearest-even(acc).  Masked slots add
 *              nothing.  H % 8 == 0; y and out 16-byte aligned.
 */
moe_status_t moe_combine(const void* y, int num_tokens, int hidden, int k,
                         const int32_t* token_slot, int num_recv_rows, const float* topk_w,
                         void* out, int32_t* d_status, moe_stream_t stream);

/*
 * moe_dispatch_backward -- gradient of dispatch: the sum of each token's
 * gradient rows.  [EPv2] usage patterns: the backward pass of dispatch is a
 * combine.  grad_recv bf16 [S, H] (one gradient row per receive slot),
 * token_slot int32 [N, k] -> grad_x bf16 [N, H]:
 *   grad_x[t, c] = bf16_rne(acc), acc = +0.0f, acc = acc + grad_recv[token_slot[t,j], c]
 *   for j = 0..k-1 in slot order (fp32; masked slots skipped).
 * (With FP8 dispatch the gradient passes the quantisation unchanged: grad_recv
 * is the gradient with respect to the dequantised rows.)
 * H % 8 == 0; grad_recv and grad_x 16-byte aligned.
 */
moe_status_t moe_dispatch_backward(const void* grad_recv, int num_tokens, int hidden, int k,
                                   const int32_t* token_slot, int num_recv_rows, void* grad_x,
                                   int32_t* d_status, moe_stream_t stream);

/*
 * moe_combine_backward -- gradients of combine with respect to the expert
 * outputs and the router weights.  [EPv2] usage patterns: the backward pass of
 * combine is a dispatch.  For every valid slot s = token_slot[t,j]:
 *   grad_y[s, c] = bf16_rne(fp32(topk_w[t,j] * grad_out[t,c]))   (grad_y bf16 [S, H])
 *   grad_w[t, j] = sum_c grad_out[t,c] * y[s,c]                   (grad_w fp32 [N, k])
 * grad_w is accumulated in fp32 in a fixed order (deterministic); its
 * rounding error is at most (H - 1) * 2^-24 * sum_c |grad_out[t,c] * y[s,c]|
 * (the products of two bf16 values are exact in fp32).  A masked slot gets
 * grad_w = 0 and writes no grad_y row; rows no slot names are not written.
 * H % 8 == 0; grad_out, y, grad_y 16-byte aligned.
 */
moe_status_t moe_combine_backward(const void* grad_out, const void* y, int num_tokens, int hidden,
                                  int k, const int32_t* token_slot, int num_recv_rows,
                                  const float* topk_w, void* grad_y, float* grad_w,
                                  int32_t* d_status, moe_stream_t stream);

/*
 * moe_e4m3_encode -- the element encoder moe_dispatch uses, exposed on its
 * own: out[i] = e4m3 code of in[i], round to nearest even, finite values and
 * infinities beyond 448 saturated to +-448, zero keeps its sign, NaN -> NaN
 * code.  (OCP 8-bit floating point, E4M3.)  n may be 0.
 */
moe_status_t moe_e4m3_encode(const float* in, size_t n, uint8_t* out, moe_stream_t stream);

/*
 * moe_gate_math -- diagnostics: the gate's exp and sigmoid, exposed on their
 * own (as moe_e4m3_encode exposes dispatch's encoder).  For i in [0, n) the
 * input x_i is the fp32 whose bit pattern is (first + i) mod 2^32, so one
 * call can cover any run of patterns without an input array:
 *   exp_out[i]     = the exp every gate kind uses (Cody-Waite reduction with
 *                    ln2 split into a 16-bit head and a tail, degree-7 Taylor
 *                    polynomial by Horner, input clamped to [-87, 88] by
 *                    comparisons, so every NaN input is taken as -87);
 *   sigmoid_out[i] = 1 / (1 + exp(-x_i)), each operation rounded once, the
 *                    score of the group-limited kind;
 *   silu_out[i]    = x_i / (1 + exp(-x_i)) as moe_swiglu_quant computes it
 *                    from a bf16 gate value: each operation rounded once, for
 *                    |x_i| <= 87 by that kernel's shortened steps (no clamp,
 *                    one corrected quotient from an approximate reciprocal),
 *                    which give the same bits on every bf16-representable
 *                    x_i and are within one unit in the last place on other
 *                    fp32 patterns.
 * "DeepSeek, DeepEP 오픈소스 공개", Topic Body: group-limited gating, whose
 * group scores are sums of these sigmoids; DeepSeek Tile-Kernels news,
 * "Funktionen der DeepSeek-Tile-Kernel": SwiGLU.  Any output may be NULL
 * (not all three); outputs are device fp32 arrays of n elements, 16-byte
 * aligned.  n may be 0.
 */
moe_status_t moe_gate_math(uint32_t first, size_t n, float* exp_out, float* sigmoid_out,
                           float* silu_out, moe_stream_t stream);

/* Human-readable name of a status code (static string). */
const char* moe_status_string(moe_status_t status);

/*
 * moe_selftest_bounded_wait -- diagnostics: runs the bounded wait that the
 * pipelined kernels (combine, combine backward, NVFP4 dispatch) use on an
 * mbarrier that nothing completes.  After about one second the wait gives up
 * and MOE_ERR_TIMEOUT is recorded in *d_status (device memory, 4-byte
 * aligned), exactly as a kernel whose copy never lands would report it; the
 * context stays usable.  No fault, trap or hang is involved.
 */
moe_status_t moe_selftest_bounded_wait(int32_t* d_status, moe_stream_t stream);

/* ABI version: bumped when a signature or a documented behaviour changes. */
int moe_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H_ */
