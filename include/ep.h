/*
 * ep.h -- C ABI of libep.so: MoE expert-parallel token dispatch and combine on
 * one B200, with the EP ranks as logical partitions of the GPU's HBM.
 *
 * The calls follow the DeepEP API as the pages state it:
 *   - ep_get_dispatch_layout  <- get_dispatch_layout(topk_idx, num_experts)
 *     ("DeepEP V1 vs V2 comparative analysis", section 2.1);
 *   - ep_dispatch             <- dispatch(x, topk_idx, topk_weights, ...) and
 *     the EPHandle it returns (same page, sections 2.1, 2.2 and 3.1), with the
 *     quantisation flags of low_latency_dispatch ("DeepEP communication
 *     library guide v2.1", sections 1.3.1 and the API listing) and the
 *     long-sequence rounds of the "DeepEP on Ascend A2" page;
 *   - ep_combine              <- combine(...) (comparative analysis, section 9.2).
 *
 * Conventions (all calls):
 *   - Every buffer is allocated and owned by the caller; the library keeps no
 *     state between calls and allocates nothing.
 *   - Pointers documented "device" must point to memory of the device that is
 *     current on the calling thread; "host" pointers to host memory.
 *   - Calls are asynchronous on `stream` (a cudaStream_t passed as void*;
 *     NULL = the legacy default stream) except where stated.
 *   - A host-side argument error returns EP_ERR_INVALID_ARG before anything
 *     is launched.  Errors the kernels detect (an expert id out of range, a
 *     receive capacity that is too small) are written to the device word
 *     `err`; read it with ep_read_error.  When *err != 0 the outputs are
 *     unspecified, but no kernel ever writes outside the buffers described
 *     here and none waits without a bound.
 *   - The routing kernel's grid barriers give up after 2 s (EP_ERR_TIMEOUT);
 *     the pack kernels of that call then write nothing.  (ep_testing.h holds
 *     test-only variants of the routing calls whose first barrier cannot be
 *     reached; no environment variable or other state changes this path.)
 *   - Sizes: T tokens (all logical ranks together), K top-k entries per
 *     token, E experts, R logical ranks, L = E / R local experts per rank,
 *     H hidden channels, A expert alignment.  Token t belongs to source rank
 *     t / (T / R); expert e lives on rank e / L.
 *   - Limits: 1 <= K <= 16, 1 <= E <= 1024, 1 <= R <= 256, E % R == 0,
 *     T % R == 0, 0 <= T <= 2^24, 8 <= H <= 65536 with H % 8 == 0, A >= 1,
 *     and T*K + E*(A-1) < 2^31 rows.
 */
#ifndef EP_B200_EP_H
#define EP_B200_EP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    EP_OK = 0,
    EP_ERR_INVALID_ARG = 1,   /* rejected on the host; nothing launched */
    EP_ERR_BAD_EXPERT_ID = 2, /* some topk_idx entry is < -1 or >= E (device) */
    EP_ERR_CAPACITY = 3,      /* recv_capacity < rows needed (device) */
    EP_ERR_CUDA = 4,          /* a CUDA runtime call failed */
    EP_ERR_TIMEOUT = 5,       /* a bounded device wait gave up (routing's grid barrier
                                 waits at most 2 s); nothing is packed after it */
    EP_ERR_NONFINITE = 6      /* a router logit is NaN or infinite (gating, device) */
} ep_status_t;

typedef enum {
    EP_QUANT_NONE = 0,     /* recv_x is the bf16 row, bit for bit */
    EP_QUANT_FP8_E4M3 = 1, /* OCP e4m3fn codes, fp32 scale per quant_size channels */
    EP_QUANT_INT8 = 2,     /* int8 codes in [-127, 127], fp32 scale per quant_size */
    EP_QUANT_MXFP4 = 3     /* OCP MXFP4: E2M1 codes, two per byte (even channel in the
                              low nibble), one UE8M0 scale byte per 32 channels
                              (use_mxfp4, guide v2.1 section 1.3.3) */
} ep_quant_t;

/* Options of ep_dispatch. */
typedef struct {
    int32_t expert_alignment; /* A >= 1: each expert's segment of received rows is
                                 padded to a multiple of A (EPHandle.expert_alignment,
                                 comparative analysis section 3.1) */
    int32_t quant;            /* ep_quant_t */
    int32_t quant_size;       /* channels per scale: 128 (group) or H (per token)
                                 (quant_size, guide v2.1 section 1.3.1); a power of
                                 two in [16, 512] dividing H, or H; 32 for MXFP4;
                                 ignored for EP_QUANT_NONE */
    int32_t round_scale;      /* nonzero: round each scale up to a power of two
                                 (round_scale / use_ue8m0); stored as fp32 */
    int32_t num_rounds;       /* >= 1, divides T / R: the rows are written in
                                 rounds of (T/R)/num_rounds tokens per rank ("ant
                                 moving home" long-sequence mode, Ascend A2 page);
                                 the result equals num_rounds == 1 */
    int32_t scale_ue8m0;      /* nonzero: store each scale as one UE8M0 byte, its
                                 biased exponent (use_ue8m0, guide v2.1); needs
                                 round_scale for FP8 / int8; always so for MXFP4.
                                 recv_scales then points to uint8 [rows, H/quant_size] */
    /* optional device [E]: the unaligned per-expert counts of this call are
     * added to it (cumulative_local_expert_recv_stats, guide v2.1) */
    int32_t* cumulative_local_expert_recv_stats;
    /* optional cudaEvent_t values (as void*) recorded on `stream` right before
     * and right after the pack kernel(s), for timing; NULL = none */
    void* event_pack_begin;
    void* event_pack_end;
    /* added to the token index written to recv_src_metadata (0 normally); a
     * GPU that holds tokens [o, o + T) of a larger batch passes o so that the
     * metadata names tokens of the whole batch */
    int32_t token_offset;
} ep_dispatch_opts_t;

/* The routing handle ep_dispatch fills and ep_combine reads (EPHandle of the
 * comparative analysis, section 3.1).  A plain struct: the caller allocates
 * every array (device memory), sets the pointers, and passes the same struct
 * to ep_combine.  ep_dispatch sets the scalar fields. */
typedef struct {
    int32_t num_tokens, num_topk, num_experts, num_ranks, hidden, expert_alignment;
    int32_t num_rounds;
    int32_t low_latency;                         /* 1: rows in the fixed-capacity layout of
                                                    ep_dispatch_low_latency (no padding rows) */
    int64_t recv_capacity;                       /* rows of recv_x / y */
    int32_t* topk_idx;                           /* [T,K] copy of the routing as int32
                                                    (-1 = masked); may be NULL */
    int32_t* psum_num_recv_tokens_per_expert;    /* [E] inclusive prefix sum of the
                                                    aligned per-expert counts */
    int32_t* num_recv_tokens_per_expert;         /* [E] unaligned counts */
    int32_t* recv_src_metadata;                  /* [recv_capacity, 2]: (t, k) of each
                                                    received row; (-1,-1) on padding */
    int32_t* dst_buffer_slot_idx;                /* [T,K]: row of (t,k), -1 if masked */
    int32_t* err;                                /* [1]: device status word */
} ep_handle_t;

/* Rows ep_dispatch may need: T*K + E*(A-1) (every entry unmasked, every
 * expert padded by A-1).  Host only. */
int64_t ep_recv_capacity_bound(int32_t T, int32_t K, int32_t E, int32_t A);

/* Bytes of device workspace the calls below need for these sizes (256-byte
 * aligned; pass at least this many).  Host only. */
size_t ep_workspace_bytes(int32_t T, int32_t K, int32_t E, int32_t R);

/*
 * Routing histogram (get_dispatch_layout, comparative analysis section 2.1;
 * the RDMA-rank output has no meaning on one GPU and is not produced).
 *   topk_idx               device int64 [T,K]; -1 = masked entry
 *   num_tokens_per_rank    device int32 [R]: tokens with >= 1 expert on rank r
 *   num_tokens_per_expert  device int32 [E]: (t,k) entries routed to expert e
 *   is_token_in_rank       device uint8 [T,R]: 1 if some expert of t is on r
 *   err                    device int32 [1]: status word (written by this call)
 *   ws, ws_bytes           device workspace of ep_workspace_bytes(T,K,E,R)
 * Any of the three outputs may be NULL to skip it.
 */
ep_status_t ep_get_dispatch_layout(const int64_t* topk_idx, int32_t T, int32_t K, int32_t E,
                                   int32_t R, int32_t* num_tokens_per_rank,
                                   int32_t* num_tokens_per_expert, uint8_t* is_token_in_rank,
                                   int32_t* err, void* ws, size_t ws_bytes, void* stream);

/*
 * Dispatch (dispatch, comparative analysis sections 2.1-3.1): one received row
 * per unmasked (t,k) ("expand" mode), rows ordered by (expert, source token, k)
 * -- the deterministic order of section 8.4 -- each expert's segment padded to
 * a multiple of A.  Padding rows hold zero bytes, scale 0, recv_topk_idx -1,
 * weight 0 and metadata (-1,-1).
 *   x                    device bf16 [T,H] (16-byte aligned rows)
 *   topk_idx             device int64 [T,K]
 *   topk_weights         device fp32 [T,K]
 *   recv_x               device [recv_capacity, H]: bf16 (NONE) or 1-byte codes
 *   recv_scales          device fp32 [recv_capacity, H/quant_size]; NULL for NONE
 *   recv_topk_idx        device int32 [recv_capacity, K]: for the row of (t,k)
 *                        with expert e on rank r, entry j is topk_idx[t,j] - r*L
 *                        if that expert is on rank r, else -1
 *   recv_topk_weights    device fp32 [recv_capacity, K]: topk_weights[t,j] where
 *                        recv_topk_idx is >= 0, else 0
 *   handle               caller-allocated arrays, see ep_handle_t; filled here
 *   num_tokens_per_rank, num_tokens_per_expert, is_token_in_rank: optional
 *                        layout outputs as in ep_get_dispatch_layout (may be NULL)
 *   ws, ws_bytes         device workspace of ep_workspace_bytes(T,K,E,R)
 * The rows needed are psum_num_recv_tokens_per_expert[E-1]; if recv_capacity is
 * smaller, *handle->err = EP_ERR_CAPACITY and no row at or past recv_capacity
 * is written.
 */
ep_status_t ep_dispatch(const void* x, int32_t T, int32_t H, const int64_t* topk_idx,
                        const float* topk_weights, int32_t K, int32_t E, int32_t R,
                        const ep_dispatch_opts_t* opts, void* recv_x, float* recv_scales,
                        int32_t* recv_topk_idx, float* recv_topk_weights,
                        int64_t recv_capacity, ep_handle_t* handle,
                        int32_t* num_tokens_per_rank, int32_t* num_tokens_per_expert,
                        uint8_t* is_token_in_rank, void* ws, size_t ws_bytes, void* stream);

/*
 * Low-latency dispatch (the decode-mode layout: low_latency_dispatch of
 * "DeepEP communication library guide v2.1", its fixed-capacity per-rank
 * buffers [num_local_experts, num_ranks * num_max_dispatch_tokens_per_rank,
 * hidden] of comparative analysis section 6.3).  On one GPU the ranks'
 * buffers stack to recv_x [E, R*M, H] (M = num_max_dispatch_tokens_per_rank):
 * the entry (t,k) for expert e from source rank r = t / (T/R) goes to row
 * e*R*M + r*M + p, p its position among rank r's entries for e in (t,k) order.
 * No global scan, no padding rows; rows past an (expert, rank) block's count
 * are left as they were.
 *   num_max_dispatch_tokens_per_rank  M >= T/R
 *   recv_x, recv_scales, recv_topk_idx, recv_topk_weights  as in ep_dispatch,
 *                        with E*R*M rows
 *   packed_recv_count    device int32 [E]: entries received per expert (may be NULL)
 *   packed_recv_layout_range  device int64 [E,R]: (r*M << 32) | entries from
 *                        rank r (may be NULL)
 *   handle               as in ep_dispatch (recv_src_metadata has E*R*M rows);
 *                        low_latency = 1, recv_capacity = E*R*M; psum holds the
 *                        inclusive prefix of the unaligned counts
 * opts->expert_alignment must be 1; opts->num_rounds must divide T/R; the
 * optional pack events bracket the pack kernel as in ep_dispatch.  More than M
 * entries of one (expert, rank) set EP_ERR_CAPACITY (they are dropped).
 * ep_combine and ep_dispatch_cached accept the handle.
 */
ep_status_t ep_dispatch_low_latency(const void* x, int32_t T, int32_t H, const int64_t* topk_idx,
                                    const float* topk_weights, int32_t K, int32_t E, int32_t R,
                                    int32_t num_max_dispatch_tokens_per_rank, const ep_dispatch_opts_t* opts,
                                    void* recv_x, float* recv_scales, int32_t* recv_topk_idx,
                                    float* recv_topk_weights, int32_t* packed_recv_count,
                                    int64_t* packed_recv_layout_range, ep_handle_t* handle, void* ws,
                                    size_t ws_bytes, void* stream);

/*
 * Cached dispatch (the cached mode of dispatch, comparative analysis sections
 * 3.2-3.3 and 8.3): re-packs new token rows x with the routing of an earlier
 * ep_dispatch whose handle is passed, skipping the layout, the slot
 * assignment and any host sync -- the decode-time case where the routing of
 * consecutive steps is unchanged.  Only recv_x (and recv_scales) are written;
 * recv_topk_idx / recv_topk_weights and the handle keep the earlier call's
 * contents.  Padding rows are zeroed again.
 *   x            device bf16 [T,H] with the handle's T and H
 *   handle       filled by ep_dispatch (read only); its err word receives
 *                device errors of this call (a handle whose err word already
 *                holds EP_ERR_TIMEOUT from its routing is not packed)
 *   opts         quant, quant_size, round_scale, num_rounds and the optional
 *                pack events are used; expert_alignment is the handle's
 *   recv_x, recv_scales  as in ep_dispatch, handle->recv_capacity rows
 */
ep_status_t ep_dispatch_cached(const void* x, const ep_handle_t* handle, const ep_dispatch_opts_t* opts,
                               void* recv_x, float* recv_scales, void* stream);

/*
 * Dispatch for callers that cannot allocate device memory.  The pages have no
 * counterpart: it is ep_dispatch with the same arguments and results, minus
 * the workspace, for code that may not call cudaMalloc (a region that must not
 * allocate, a plugin that only receives its input and output pointers, a
 * runtime without an allocator).  The routing scratch lives instead in one
 * static device array of 2 MiB per GPU, held until the process exits; sizes
 * whose scratch (ep_workspace_bytes) exceeds 2 MiB return EP_ERR_INVALID_ARG
 * with a message on stderr, before anything runs.  The first call on a device
 * looks up the array's address (make it before any stream capture); it is
 * cached per device together with the ID of the current CUDA context, and a
 * call in a new context of that device (after cudaDeviceReset) looks it up
 * again, which should likewise precede any stream capture.  All
 * calls on a device share the array: calls whose kernels overlap on the GPU
 * race, so serialise them on one stream.  Allocates nothing.
 */
ep_status_t ep_dispatch_noalloc(const void* x, int32_t T, int32_t H, const int64_t* topk_idx,
                                const float* topk_weights, int32_t K, int32_t E, int32_t R,
                                const ep_dispatch_opts_t* opts, void* recv_x, float* recv_scales,
                                int32_t* recv_topk_idx, float* recv_topk_weights,
                                int64_t recv_capacity, ep_handle_t* handle,
                                int32_t* num_tokens_per_rank, int32_t* num_tokens_per_expert,
                                uint8_t* is_token_in_rank, void* stream);

/*
 * Combine (combine, comparative analysis section 9.2): for every token t
 *   out[t] = bf16_rne( sum over k = 0..K-1 with dst_buffer_slot_idx[t,k] >= 0
 *                      of topk_weights[t,k] * y[dst_buffer_slot_idx[t,k]] ),
 * accumulated in fp32 with fused multiply-adds in k order from +0.
 *   y              device bf16 [handle->recv_capacity, H]: expert outputs, in the
 *                  received-row order of the dispatch that filled `handle`
 *   handle         as filled by ep_dispatch (num_rounds is taken from it)
 *   topk_weights   device fp32 [T,K]
 *   out            device bf16 [T,H]
 */
ep_status_t ep_combine(const void* y, const ep_handle_t* handle, const float* topk_weights,
                       void* out, void* stream);

/*
 * Combine with quantised expert outputs and / or a shared expert (the
 * combine-side int8 / fp8 of low_latency_combine, "DeepEP communication
 * library guide v2.1", section 1.3.1 and its API listing; the shared-expert
 * combine of lmdeploy PR #4783).  For every token t,
 *   out[t] = bf16_rne( fma chain in k order over the unmasked entries of
 *                      topk_weights[t,k] * value(row(t,k)) ), starting from
 *                      shared[t] (bf16) if given, else +0,
 * where value = the bf16 row (y_quant EP_QUANT_NONE) or, for FP8 e4m3 / int8
 * codes, decode(code) * scale as an fp32 product with one fp32 scale per
 * y_quant_size channels (y_scales [recv_capacity, H / y_quant_size]).
 * y_quant_size: 16..512 (a power of two) or H.  shared may be NULL.  With
 * y_quant NONE and shared NULL this is ep_combine.
 */
ep_status_t ep_combine_ex(const void* y, const float* y_scales, int32_t y_quant, int32_t y_quant_size,
                          const ep_handle_t* handle, const float* topk_weights, const void* shared, void* out,
                          void* stream);

/*
 * Group-limited gating: the routing generator whose topk_idx / topk_weights
 * feed ep_dispatch ("DeepEP V1 vs V2 comparative analysis", section 8.1,
 * DeepSeek-V3 group-limited gating: 256 experts in 32 groups of 8, each token
 * keeps its top-4 groups and the top-2 experts inside each, top-8 in all).
 * For every token t of router logits [T, E]:
 *   - the experts form n_group groups of E / n_group consecutive ids;
 *   - a group's score is the fp32 sum of its per_group largest logits, added
 *     from the largest down;
 *   - the topk_group best groups are kept, and the per_group best experts of
 *     each are the token's K = topk_group * per_group entries, listed by
 *     logit, largest first;
 *   - of two equal logits or scores, the lower expert / group id ranks first;
 *   - topk_weights[t] = softmax over the K selected logits, computed in
 *     binary64 and rounded to binary32.
 *   logits         device fp32 [T, E]
 *   topk_idx       device int64 [T, K] (output; K distinct ids in [0, E))
 *   topk_weights   device fp32 [T, K] (output)
 *   err            device int32 [1]: status word, cleared by this call;
 *                  EP_ERR_NONFINITE if a logit is NaN or infinite (the outputs
 *                  are then unspecified but still K distinct ids in range)
 * Limits: 0 <= T <= 2^24, 1 <= n_group <= 32, E % n_group == 0, E <= 1024,
 * 1 <= topk_group <= n_group, 1 <= per_group <= E / n_group, K <= 16.
 */
ep_status_t ep_group_limited_gating(const float* logits, int32_t T, int32_t E, int32_t n_group,
                                    int32_t topk_group, int32_t per_group, int64_t* topk_idx,
                                    float* topk_weights, int32_t* err, void* stream);

/*
 * Padding rows of a receive layout whose real rows were placed by another path
 * (the multi-GPU exchange writes each source GPU's rows straight into a
 * receiver's layout, and the receiver then fills the alignment padding that
 * ep_dispatch would have written; comparative analysis section 3.1, expert
 * alignment).  For each expert segment e < n_experts, the rows
 * [psum[e-1] + counts[e], psum[e]) (psum[-1] = 0) get zero bytes in recv_x,
 * zero bytes in recv_scales, recv_topk_idx -1, recv_topk_weights 0 and
 * recv_src_metadata (-1, -1) -- the padding rows of ep_dispatch.
 *   psum, counts        device int32 [n_experts]: inclusive prefix of the
 *                       aligned counts, and the unaligned counts
 *   recv_x              device, row_bytes per row (a multiple of 16, 16-byte aligned)
 *   recv_scales         device, scale_row_bytes per row, or NULL
 *   recv_topk_idx / recv_topk_weights  device [capacity, K], or NULL
 *   recv_src_metadata   device int32 [capacity, 2], or NULL
 * Rows at or past capacity are not written.  1 <= n_experts <= 1024.
 */
ep_status_t ep_write_padding_rows(const int32_t* psum, const int32_t* counts, int32_t n_experts, void* recv_x,
                                  int64_t row_bytes, void* recv_scales, int64_t scale_row_bytes,
                                  int32_t* recv_topk_idx, float* recv_topk_weights, int32_t K,
                                  int32_t* recv_src_metadata, int64_t capacity, void* stream);

/*
 * Expert parallelism over G GPUs through peer memory (one process per GPU,
 * NVLink / NVSwitch peer loads and stores; comparative analysis section 6.1,
 * the normal mode's dispatch of each rank's tokens into the receivers'
 * buffers, and section 9.2, combine).  GPU g of G holds the logical ranks
 * [g R/G, (g+1) R/G): tokens [g T/G, (g+1) T/G) of the batch and experts
 * [g E/G, (g+1) E/G).  Each GPU ends with the single-GPU result restricted to
 * itself (its experts' rows in (expert, token, k) order, padded to the
 * alignment A; its own tokens combined).
 *   1. ep_route on every GPU: routing of its own tokens with alignment 1 (its
 *      send order); handle->num_recv_tokens_per_expert is its row of the
 *      count matrix C [G, E];
 *   2. the caller all-gathers C into device memory on every GPU (NCCL);
 *   3. ep_pack_peer on every GPU: each entry's row on its receiver
 *      d = e / (E/G) is computed from C on the device, and the row (bf16 or
 *      quantised), its scales, recv_topk_idx / weights and metadata are stored
 *      straight into d's layout through the peer pointer tables;
 *   4. the caller orders the GPUs (a collective after the packs); each
 *      receiver runs ep_receiver_layout and ep_write_padding_rows;
 *   5. after the experts, ep_combine_peer on every GPU loads each of its
 *      tokens' rows from the receivers' y through peer pointers and reduces
 *      them in k order.
 * Peer pointer tables are device arrays of G pointers (entry g' = that
 * buffer on GPU g', mapped into this process; entry g = this GPU's own).
 * Nothing here waits on another GPU: the caller's collectives order the
 * steps.  Peer memory is reached with plain loads and stores only.
 */

/* Routing only (steps 1): ep_dispatch's handle, recv_topk_idx,
 * recv_topk_weights and metadata, in the same layout and with the same
 * arguments (token_offset included), but no rows: the rows are packed by
 * ep_pack_peer.  recv_capacity >= rows needed with this alignment. */
ep_status_t ep_route(const int64_t* topk_idx, const float* topk_weights, int32_t T, int32_t K, int32_t E,
                     int32_t R, int32_t expert_alignment, int32_t token_offset, int32_t* recv_topk_idx,
                     float* recv_topk_weights, int64_t recv_capacity, ep_handle_t* handle, void* ws,
                     size_t ws_bytes, void* stream);

/* Step 3.  x: this GPU's tokens [T, H]; handle from ep_route (alignment 1);
 * send_topk_idx / send_topk_weights: the recv_topk_* arrays ep_route wrote
 * (rows in send order); counts_all: device int32 [G, E]; opts: quant,
 * quant_size, round_scale and scale_ue8m0 as in ep_dispatch (FP8 / int8
 * groups of 16..512 channels, or none); A: the receivers' expert alignment;
 * peer_*: device arrays of G pointers to the receivers' recv_x, recv_scales
 * (may be NULL for bf16), recv_topk_idx, recv_topk_weights and
 * recv_src_metadata, each with peer_capacity rows.  Rows at or past
 * peer_capacity are not written (EP_ERR_CAPACITY in handle->err). */
ep_status_t ep_pack_peer(const void* x, const ep_handle_t* handle, const int32_t* send_topk_idx,
                         const float* send_topk_weights, const int32_t* counts_all, int32_t G, int32_t g,
                         int32_t A, const ep_dispatch_opts_t* opts, void* const* peer_recv_x,
                         void* const* peer_recv_scales, int32_t* const* peer_recv_topk_idx,
                         float* const* peer_recv_topk_weights, int32_t* const* peer_recv_metadata,
                         int64_t peer_capacity, void* stream);

/* Step 4: this GPU's receive layout from counts_all: psum [E/G] (inclusive
 * prefix of the aligned totals over its experts) and counts [E/G]. */
ep_status_t ep_receiver_layout(const int32_t* counts_all, int32_t G, int32_t g, int32_t E, int32_t A,
                               int32_t* psum, int32_t* counts, void* stream);

/* Step 5: for each of this GPU's tokens t, out[t] = bf16_rne(fma chain in k
 * order of topk_weights[t,k] * y_d[row]) over the unmasked entries, where
 * row on receiver d is the one ep_pack_peer wrote; peer_y: device array of G
 * pointers to the receivers' expert outputs (bf16, peer_capacity rows). */
ep_status_t ep_combine_peer(void* const* peer_y, const ep_handle_t* handle, const int32_t* counts_all, int32_t G,
                            int32_t g, int32_t A, const float* topk_weights, void* out, int64_t peer_capacity,
                            void* stream);

/* CUDA IPC for the peer pointer tables.  ep_ipc_export writes the 64-byte IPC
 * handle of the device allocation that holds ptr to handle64 and ptr's offset
 * inside that allocation to *offset; ep_ipc_import opens such a handle in
 * another process of the same machine (on the current device) and returns
 * the allocation's address there (add the offset); ep_ipc_close releases an
 * imported address.  Host calls; they allocate nothing on the device. */
ep_status_t ep_ipc_export(const void* ptr, void* handle64, int64_t* offset);
ep_status_t ep_ipc_import(const void* handle64, void** base);
ep_status_t ep_ipc_close(void* base);

/* Waits for `stream`, then copies the device status word to *host_status.
 * Returns EP_OK, or EP_ERR_CUDA if the wait or the copy failed. */
ep_status_t ep_read_error(const int32_t* err, void* stream, int32_t* host_status);

/* The host copy a "do_cpu_sync" dispatch makes (comparative analysis,
 * section 3.2): waits for `stream`, then copies the E unaligned per-expert
 * counts to host_counts[E] (may be NULL) and the number of received rows
 * (psum_num_recv_tokens_per_expert[E-1]) to *num_recv_rows (may be NULL). */
ep_status_t ep_copy_recv_counts(const ep_handle_t* handle, void* stream, int32_t* host_counts,
                                int64_t* num_recv_rows);

/* A static string naming a status code. */
const char* ep_status_string(ep_status_t status);

#ifdef __cplusplus
}
#endif

#endif /* EP_B200_EP_H */
