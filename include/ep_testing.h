/*
 * ep_testing.h -- test-only entry points of libep.so.  Not part of the
 * product API: nothing in the dispatch / combine path calls them.
 *
 * They exist so that tests can make routing's bounded grid-barrier wait run
 * out on a real GPU without a fault: each is the call of the same name in
 * ep.h, with the same arguments, validation and outputs, except that the
 * first grid barrier of the routing kernel waits for one CTA more than the
 * grid holds.  Every CTA then gives up after the barrier's 2 s limit, the
 * status word reads EP_ERR_TIMEOUT, and (for dispatch) the pack kernels write
 * nothing.  The context stays usable.
 */
#ifndef EP_B200_EP_TESTING_H
#define EP_B200_EP_TESTING_H

#include "ep.h"

#ifdef __cplusplus
extern "C" {
#endif

/* ep_get_dispatch_layout with an unreachable first grid barrier. */
ep_status_t ep_testing_get_dispatch_layout_stalled(const int64_t* topk_idx, int32_t T, int32_t K, int32_t E,
                                                   int32_t R, int32_t* num_tokens_per_rank,
                                                   int32_t* num_tokens_per_expert, uint8_t* is_token_in_rank,
                                                   int32_t* err, void* ws, size_t ws_bytes, void* stream);

/* ep_dispatch with an unreachable first grid barrier. */
ep_status_t ep_testing_dispatch_stalled(const void* x, int32_t T, int32_t H, const int64_t* topk_idx,
                                        const float* topk_weights, int32_t K, int32_t E, int32_t R,
                                        const ep_dispatch_opts_t* opts, void* recv_x, float* recv_scales,
                                        int32_t* recv_topk_idx, float* recv_topk_weights, int64_t recv_capacity,
                                        ep_handle_t* handle, int32_t* num_tokens_per_rank,
                                        int32_t* num_tokens_per_expert, uint8_t* is_token_in_rank, void* ws,
                                        size_t ws_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* EP_B200_EP_TESTING_H */
