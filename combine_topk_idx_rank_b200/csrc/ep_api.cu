// C ABI of libep.so (declared in include/ep.h): argument validation,
// workspace carving and the launch sequence of each call.  Stateless: every
// buffer belongs to the caller, nothing is allocated here.
#include <cuda.h>   // CUdeviceptr / CUresult types; driver calls are resolved at run time
#include <stdio.h>
#include <string.h>

#include "ep_internal.cuh"
#include "../../include/ep_testing.h"

namespace ep {

int device_sm_count() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (dev >= 0 && dev < 64 && cached[dev] > 0) return cached[dev];
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) n = 148;
    if (dev >= 0 && dev < 64) cached[dev] = n;
    return n;
}

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool sizes_ok(int32_t T, int32_t K, int32_t E, int32_t R) {
    if (T < 0 || T > (1 << 24)) return false;
    if (K < 1 || K > kMaxTopk) return false;
    if (E < 1 || E > kMaxExperts) return false;
    if (R < 1 || R > kMaxRanks || E % R != 0) return false;
    if (T % R != 0) return false;
    return true;
}

ep_status_t cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return EP_OK;
    fprintf(stderr, "libep: CUDA error %d (%s)\n", (int)e, cudaGetErrorString(e));
    return EP_ERR_CUDA;
}

// Routing arguments common to the layout call and dispatch.
RouteArgs route_args(void* ws, const WsLayout& L, const int64_t* topk_idx, const float* topk_weights,
                     int T, int K, int E, int R) {
    char* b = static_cast<char*>(ws);
    auto at = [&](size_t off) { return reinterpret_cast<int32_t*>(b + off); };
    RouteArgs r{};
    r.topk_idx = topk_idx;
    r.topk_weights = topk_weights;
    r.T = T; r.K = K; r.E = E; r.R = R; r.L = E / R; r.A = 1;
    r.log2_chunk = L.log2_chunk;
    r.nchunks = L.nchunks;
    r.tokens_per_rank = R > 0 ? T / R : 0;
    r.chunks_per_rank = L.chunks_per_rank;
    r.barrier = reinterpret_cast<unsigned*>(at(L.hdr));
    r.col_total = at(L.col_total);
    r.chunk_hist = at(L.chunk_hist);
    r.chunk_rcnt = at(L.chunk_rcnt);
    r.chunk_err = at(L.chunk_err);
    return r;
}

// The pack kernel(s) of a dispatch: one launch per round, each a
// programmatic dependent of the previous kernel on the stream.  Rows come
// from handle->dst_buffer_slot_idx; the padding map from the handle's psum
// and unaligned counts.  `routed`: the routing kernel was launched just
// before on the stream, so x was complete when it started and the packs may
// read x before their dependency wait.
ep_status_t launch_pack_rounds(const void* x, int T, int H, int K, int E, int R, int quant, int quant_size,
                               const ep_dispatch_opts_t* opts, void* recv_x, float* recv_scales,
                               int64_t recv_capacity, const ep_handle_t* h, cudaStream_t st, bool routed) {
    ep_status_t s;
    if (opts->event_pack_begin) {
        s = cuda_status(cudaEventRecord(static_cast<cudaEvent_t>(opts->event_pack_begin), st));
        if (s) return s;
    }
    if (T > 0) {
        const int rounds = opts->num_rounds;
        const int tpr = T / R, per_round = tpr / rounds;
        for (int j = 0; j < rounds; ++j) {
            PackArgs pa{};
            pa.x = static_cast<const uint16_t*>(x);
            pa.H = H; pa.K = K; pa.E = E;
            pa.dst_slot = h->dst_buffer_slot_idx;
            pa.recv_x = static_cast<uint8_t*>(recv_x); pa.recv_scales = recv_scales;
            pa.capacity = recv_capacity;
            pa.psum = h->psum_num_recv_tokens_per_expert; pa.cnt = h->num_recv_tokens_per_expert;
            pa.tokens_per_rank = tpr; pa.per_round = per_round; pa.round = j;
            pa.n_tok_items = R * per_round; pa.do_pad = (j == 0) && !h->low_latency && h->expert_alignment > 1;   // A = 1: no padding rows
            pa.quant_size = quant_size; pa.round_scale = opts->round_scale ? 1 : 0;
            pa.scale_bytes = (quant == EP_QUANT_MXFP4 || (quant != EP_QUANT_NONE && opts->scale_ue8m0)) ? 1 : 0;
            pa.err = h->err;
            pa.x32 = (reinterpret_cast<uintptr_t>(x) & 31u) == 0;   // rows of H % 16 == 0 channels stay aligned
            pa.early_x = routed ? 1 : 0;
            s = cuda_status(launch_pack(pa, quant, st));
            if (s) return s;
        }
    }
    if (opts->event_pack_end) {
        s = cuda_status(cudaEventRecord(static_cast<cudaEvent_t>(opts->event_pack_end), st));
        if (s) return s;
    }
    return EP_OK;
}

// Quantisation options shared by ep_dispatch and ep_dispatch_cached.
// The quantisation is a supported one for rows of H channels; the scales
// array is required as soon as there is a row to hold (rows > 0).
bool quant_ok(int quant, int quant_size, int H, const float* recv_scales, int64_t rows) {
    if (quant == EP_QUANT_NONE) return true;
    const bool scales = recv_scales != nullptr || rows == 0;
    if (quant == EP_QUANT_MXFP4) return quant_size == 32 && H % 32 == 0 && scales;
    if (quant != EP_QUANT_FP8_E4M3 && quant != EP_QUANT_INT8) return false;
    const bool group = quant_size == 16 || quant_size == 32 || quant_size == 64 || quant_size == 128 ||
                       quant_size == 256 || quant_size == 512;
    return H % 16 == 0 && (quant_size == H || group) && H % quant_size == 0 && scales;
}

}  // namespace
}  // namespace ep

using namespace ep;

extern "C" {

int64_t ep_recv_capacity_bound(int32_t T, int32_t K, int32_t E, int32_t A) {
    if (T < 0 || K < 1 || E < 1 || A < 1) return 0;
    return (int64_t)T * K + (int64_t)E * (A - 1);
}

size_t ep_workspace_bytes(int32_t T, int32_t K, int32_t E, int32_t R) {
    if (!sizes_ok(T, K, E, R)) return 0;
    return ws_layout(T, K, E, R).total;
}

const char* ep_status_string(ep_status_t s) {
    switch (s) {
        case EP_OK: return "ok";
        case EP_ERR_INVALID_ARG: return "invalid argument";
        case EP_ERR_BAD_EXPERT_ID: return "expert id out of range";
        case EP_ERR_CAPACITY: return "receive capacity too small";
        case EP_ERR_CUDA: return "CUDA error";
        case EP_ERR_TIMEOUT: return "device wait timed out";
        case EP_ERR_NONFINITE: return "router logit not finite";
    }
    return "unknown status";
}

}  // extern "C"

namespace {

// The layout call; stall > 0 only from the test entry point.
ep_status_t layout_impl(const int64_t* topk_idx, int32_t T, int32_t K, int32_t E, int32_t R,
                        int32_t* num_tokens_per_rank, int32_t* num_tokens_per_expert, uint8_t* is_token_in_rank,
                        int32_t* err, void* ws, size_t ws_bytes, void* stream, unsigned stall) {
    if (!sizes_ok(T, K, E, R) || err == nullptr || ws == nullptr) return EP_ERR_INVALID_ARG;
    if (T > 0 && topk_idx == nullptr) return EP_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(T, K, E, R);
    if (ws_bytes < L.total) return EP_ERR_INVALID_ARG;
    RouteArgs r = route_args(ws, L, topk_idx, nullptr, T, K, E, R);
    r.assign = 0;
    r.is_token_in_rank = is_token_in_rank;
    r.num_tokens_per_expert = num_tokens_per_expert;
    r.num_tokens_per_rank = num_tokens_per_rank;
    r.err_out = err;
    r.stall = stall;
    return cuda_status(launch_route(r, static_cast<cudaStream_t>(stream)));
}

// Dispatch; stall > 0 only from the test entry point.
ep_status_t dispatch_impl(const void* x, int32_t T, int32_t H, const int64_t* topk_idx, const float* topk_weights,
                          int32_t K, int32_t E, int32_t R, const ep_dispatch_opts_t* opts, void* recv_x,
                          float* recv_scales, int32_t* recv_topk_idx, float* recv_topk_weights,
                          int64_t recv_capacity, ep_handle_t* h, int32_t* num_tokens_per_rank,
                          int32_t* num_tokens_per_expert, uint8_t* is_token_in_rank, void* ws, size_t ws_bytes,
                          void* stream, unsigned stall) {
    if (!sizes_ok(T, K, E, R) || opts == nullptr || h == nullptr) return EP_ERR_INVALID_ARG;
    if (H < 8 || H > 65536 || H % 8 != 0) return EP_ERR_INVALID_ARG;
    const int A = opts->expert_alignment;
    const int quant = opts->quant;
    const int rounds = opts->num_rounds;
    if (A < 1 || rounds < 1 || (T / R) % rounds != 0) return EP_ERR_INVALID_ARG;
    if (ep_recv_capacity_bound(T, K, E, A) >= (int64_t)INT32_MAX) return EP_ERR_INVALID_ARG;
    if (recv_capacity < 0 || recv_capacity >= (int64_t)INT32_MAX) return EP_ERR_INVALID_ARG;
    const int quant_size = quant == EP_QUANT_NONE ? 0 : opts->quant_size;
    if (!quant_ok(quant, quant_size, H, recv_scales, recv_capacity)) return EP_ERR_INVALID_ARG;
    if (opts->scale_ue8m0 && (quant == EP_QUANT_FP8_E4M3 || quant == EP_QUANT_INT8) && !opts->round_scale)
        return EP_ERR_INVALID_ARG;   // UE8M0 bytes hold powers of two only
    if (h->psum_num_recv_tokens_per_expert == nullptr || h->num_recv_tokens_per_expert == nullptr ||
        h->err == nullptr)
        return EP_ERR_INVALID_ARG;
    if (T > 0 && h->dst_buffer_slot_idx == nullptr) return EP_ERR_INVALID_ARG;
    if (recv_capacity > 0 && h->recv_src_metadata == nullptr) return EP_ERR_INVALID_ARG;
    if (recv_capacity > 0 && (recv_x == nullptr || recv_topk_idx == nullptr || recv_topk_weights == nullptr))
        return EP_ERR_INVALID_ARG;
    if (T > 0 && (x == nullptr || topk_idx == nullptr || topk_weights == nullptr)) return EP_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(recv_x)) return EP_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(T, K, E, R);
    if (ws == nullptr || ws_bytes < L.total) return EP_ERR_INVALID_ARG;

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    h->num_tokens = T; h->num_topk = K; h->num_experts = E; h->num_ranks = R;
    h->hidden = H; h->expert_alignment = A; h->num_rounds = rounds; h->recv_capacity = recv_capacity;
    h->low_latency = 0;

    RouteArgs r = route_args(ws, L, topk_idx, topk_weights, T, K, E, R);
    r.A = A;
    r.capacity = recv_capacity;
    r.check_capacity = 1;
    r.assign = 1;
    r.vector_ok = aligned16(topk_idx) && aligned16(topk_weights) && aligned16(recv_topk_idx) &&
                  aligned16(recv_topk_weights);
    r.dst_slot = h->dst_buffer_slot_idx;
    r.topk_copy = h->topk_idx;
    r.recv_meta = h->recv_src_metadata;
    r.recv_topk_idx = recv_topk_idx;
    r.recv_topk_weights = recv_topk_weights;
    r.is_token_in_rank = is_token_in_rank;
    r.psum = h->psum_num_recv_tokens_per_expert;
    r.num_recv = h->num_recv_tokens_per_expert;
    r.num_tokens_per_expert = num_tokens_per_expert;
    r.num_tokens_per_rank = num_tokens_per_rank;
    r.cumulative = opts->cumulative_local_expert_recv_stats;
    r.err_out = h->err;
    r.stall = stall;
    r.token_offset = opts->token_offset;
    ep_status_t s = cuda_status(launch_route(r, st));
    if (s) return s;
    return launch_pack_rounds(x, T, H, K, E, R, quant, quant_size, opts, recv_x, recv_scales, recv_capacity, h,
                              st, true);
}

}  // namespace

extern "C" {

ep_status_t ep_get_dispatch_layout(const int64_t* topk_idx, int32_t T, int32_t K, int32_t E,
                                   int32_t R, int32_t* num_tokens_per_rank,
                                   int32_t* num_tokens_per_expert, uint8_t* is_token_in_rank,
                                   int32_t* err, void* ws, size_t ws_bytes, void* stream) {
    return layout_impl(topk_idx, T, K, E, R, num_tokens_per_rank, num_tokens_per_expert, is_token_in_rank, err,
                       ws, ws_bytes, stream, 0);
}

ep_status_t ep_dispatch(const void* x, int32_t T, int32_t H, const int64_t* topk_idx,
                        const float* topk_weights, int32_t K, int32_t E, int32_t R,
                        const ep_dispatch_opts_t* opts, void* recv_x, float* recv_scales,
                        int32_t* recv_topk_idx, float* recv_topk_weights,
                        int64_t recv_capacity, ep_handle_t* h,
                        int32_t* num_tokens_per_rank, int32_t* num_tokens_per_expert,
                        uint8_t* is_token_in_rank, void* ws, size_t ws_bytes, void* stream) {
    return dispatch_impl(x, T, H, topk_idx, topk_weights, K, E, R, opts, recv_x, recv_scales, recv_topk_idx,
                         recv_topk_weights, recv_capacity, h, num_tokens_per_rank, num_tokens_per_expert,
                         is_token_in_rank, ws, ws_bytes, stream, 0);
}

ep_status_t ep_testing_get_dispatch_layout_stalled(const int64_t* topk_idx, int32_t T, int32_t K, int32_t E,
                                                   int32_t R, int32_t* num_tokens_per_rank,
                                                   int32_t* num_tokens_per_expert, uint8_t* is_token_in_rank,
                                                   int32_t* err, void* ws, size_t ws_bytes, void* stream) {
    return layout_impl(topk_idx, T, K, E, R, num_tokens_per_rank, num_tokens_per_expert, is_token_in_rank, err,
                       ws, ws_bytes, stream, 1);
}

ep_status_t ep_testing_dispatch_stalled(const void* x, int32_t T, int32_t H, const int64_t* topk_idx,
                                        const float* topk_weights, int32_t K, int32_t E, int32_t R,
                                        const ep_dispatch_opts_t* opts, void* recv_x, float* recv_scales,
                                        int32_t* recv_topk_idx, float* recv_topk_weights, int64_t recv_capacity,
                                        ep_handle_t* h, int32_t* num_tokens_per_rank,
                                        int32_t* num_tokens_per_expert, uint8_t* is_token_in_rank, void* ws,
                                        size_t ws_bytes, void* stream) {
    return dispatch_impl(x, T, H, topk_idx, topk_weights, K, E, R, opts, recv_x, recv_scales, recv_topk_idx,
                         recv_topk_weights, recv_capacity, h, num_tokens_per_rank, num_tokens_per_expert,
                         is_token_in_rank, ws, ws_bytes, stream, 1);
}

ep_status_t ep_dispatch_low_latency(const void* x, int32_t T, int32_t H, const int64_t* topk_idx,
                                    const float* topk_weights, int32_t K, int32_t E, int32_t R, int32_t M,
                                    const ep_dispatch_opts_t* opts, void* recv_x, float* recv_scales,
                                    int32_t* recv_topk_idx, float* recv_topk_weights, int32_t* packed_recv_count,
                                    int64_t* packed_recv_layout_range, ep_handle_t* h, void* ws, size_t ws_bytes,
                                    void* stream) {
    if (!sizes_ok(T, K, E, R) || opts == nullptr || h == nullptr) return EP_ERR_INVALID_ARG;
    if (H < 8 || H > 65536 || H % 8 != 0) return EP_ERR_INVALID_ARG;
    const int rounds = opts->num_rounds;
    if (opts->expert_alignment != 1 || rounds < 1 || (T / R) % rounds != 0) return EP_ERR_INVALID_ARG;
    if (M < 1 || M < T / R) return EP_ERR_INVALID_ARG;
    const int64_t rows = (int64_t)E * R * M;
    if (rows >= (int64_t)INT32_MAX) return EP_ERR_INVALID_ARG;
    const int quant = opts->quant;
    const int quant_size = quant == EP_QUANT_NONE ? 0 : opts->quant_size;
    if (!quant_ok(quant, quant_size, H, recv_scales, rows)) return EP_ERR_INVALID_ARG;
    if (opts->scale_ue8m0 && (quant == EP_QUANT_FP8_E4M3 || quant == EP_QUANT_INT8) && !opts->round_scale)
        return EP_ERR_INVALID_ARG;   // UE8M0 bytes hold powers of two only
    if (h->psum_num_recv_tokens_per_expert == nullptr || h->num_recv_tokens_per_expert == nullptr ||
        h->err == nullptr || h->recv_src_metadata == nullptr)
        return EP_ERR_INVALID_ARG;
    if (T > 0 && h->dst_buffer_slot_idx == nullptr) return EP_ERR_INVALID_ARG;
    if (recv_x == nullptr || recv_topk_idx == nullptr || recv_topk_weights == nullptr) return EP_ERR_INVALID_ARG;
    if (T > 0 && (x == nullptr || topk_idx == nullptr || topk_weights == nullptr)) return EP_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(recv_x)) return EP_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(T, K, E, R);
    if (ws == nullptr || ws_bytes < L.total) return EP_ERR_INVALID_ARG;

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    h->num_tokens = T; h->num_topk = K; h->num_experts = E; h->num_ranks = R;
    h->hidden = H; h->expert_alignment = 1; h->num_rounds = rounds; h->recv_capacity = rows;
    h->low_latency = 1;

    RouteArgs r = route_args(ws, L, topk_idx, topk_weights, T, K, E, R);
    r.capacity = rows;
    r.check_capacity = 1;
    r.assign = 1;
    r.ll_M = M;
    r.layout_range = packed_recv_layout_range;
    r.vector_ok = aligned16(topk_idx) && aligned16(topk_weights) && aligned16(recv_topk_idx) &&
                  aligned16(recv_topk_weights);
    r.dst_slot = h->dst_buffer_slot_idx;
    r.topk_copy = h->topk_idx;
    r.recv_meta = h->recv_src_metadata;
    r.recv_topk_idx = recv_topk_idx;
    r.recv_topk_weights = recv_topk_weights;
    r.psum = h->psum_num_recv_tokens_per_expert;
    r.num_recv = h->num_recv_tokens_per_expert;
    r.num_tokens_per_expert = packed_recv_count;
    r.cumulative = opts->cumulative_local_expert_recv_stats;
    r.err_out = h->err;
    r.token_offset = opts->token_offset;
    ep_status_t s = cuda_status(launch_route(r, st));
    if (s) return s;
    return launch_pack_rounds(x, T, H, K, E, R, quant, quant_size, opts, recv_x, recv_scales, rows, h, st, true);
}

ep_status_t ep_dispatch_cached(const void* x, const ep_handle_t* h, const ep_dispatch_opts_t* opts,
                               void* recv_x, float* recv_scales, void* stream) {
    if (h == nullptr || opts == nullptr) return EP_ERR_INVALID_ARG;
    const int T = h->num_tokens, K = h->num_topk, E = h->num_experts, R = h->num_ranks, H = h->hidden;
    const int rounds = opts->num_rounds;
    if (!sizes_ok(T, K, E, R)) return EP_ERR_INVALID_ARG;
    if (H < 8 || H > 65536 || H % 8 != 0 || rounds < 1 || (T / R) % rounds != 0) return EP_ERR_INVALID_ARG;
    const int quant = opts->quant;
    const int quant_size = quant == EP_QUANT_NONE ? 0 : opts->quant_size;
    if (!quant_ok(quant, quant_size, H, recv_scales, h->recv_capacity)) return EP_ERR_INVALID_ARG;
    if (opts->scale_ue8m0 && (quant == EP_QUANT_FP8_E4M3 || quant == EP_QUANT_INT8) && !opts->round_scale)
        return EP_ERR_INVALID_ARG;   // UE8M0 bytes hold powers of two only
    if (h->psum_num_recv_tokens_per_expert == nullptr || h->num_recv_tokens_per_expert == nullptr ||
        h->err == nullptr)
        return EP_ERR_INVALID_ARG;
    if (T > 0 && (x == nullptr || h->dst_buffer_slot_idx == nullptr)) return EP_ERR_INVALID_ARG;
    if (h->recv_capacity > 0 && recv_x == nullptr) return EP_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(recv_x)) return EP_ERR_INVALID_ARG;
    return launch_pack_rounds(x, T, H, K, E, R, quant, quant_size, opts, recv_x, recv_scales, h->recv_capacity, h,
                              static_cast<cudaStream_t>(stream), false);
}

ep_status_t ep_combine_ex(const void* y, const float* y_scales, int32_t y_quant, int32_t y_quant_size,
                          const ep_handle_t* h, const float* topk_weights, const void* shared, void* out,
                          void* stream) {
    if (h == nullptr) return EP_ERR_INVALID_ARG;
    const int T = h->num_tokens, K = h->num_topk, H = h->hidden, R = h->num_ranks;
    const int rounds = h->num_rounds;
    if (!sizes_ok(T, K, h->num_experts, R)) return EP_ERR_INVALID_ARG;
    if (H < 8 || H > 65536 || H % 8 != 0 || rounds < 1 || (T / R) % rounds != 0) return EP_ERR_INVALID_ARG;
    if (h->err == nullptr) return EP_ERR_INVALID_ARG;
    if (y_quant == EP_QUANT_MXFP4) return EP_ERR_INVALID_ARG;   // combine reads FP8 / int8 codes only
    const int qs = y_quant == EP_QUANT_NONE ? 0 : y_quant_size;
    if (!quant_ok(y_quant, qs, H, y_quant == EP_QUANT_NONE ? nullptr : y_scales, h->recv_capacity))
        return EP_ERR_INVALID_ARG;
    if (T > 0 && (out == nullptr || topk_weights == nullptr || h->dst_buffer_slot_idx == nullptr))
        return EP_ERR_INVALID_ARG;
    if (h->recv_capacity > 0 && y == nullptr) return EP_ERR_INVALID_ARG;
    if (!aligned16(y) || !aligned16(out) || !aligned16(shared)) return EP_ERR_INVALID_ARG;
    if (T == 0) return EP_OK;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int tpr = T / R, per_round = tpr / rounds;
    for (int j = 0; j < rounds; ++j) {
        CombineArgs ca{};
        ca.y = y; ca.y_scales = y_scales; ca.y_quant = y_quant; ca.quant_size = qs;
        ca.shared = static_cast<const uint16_t*>(shared);
        ca.y_rows = h->recv_capacity;
        ca.H = H; ca.K = K; ca.T = T;
        ca.dst_slot = h->dst_buffer_slot_idx; ca.topk_weights = topk_weights;
        ca.out = static_cast<uint16_t*>(out);
        ca.tokens_per_rank = tpr; ca.per_round = per_round; ca.round = j; ca.n_items = R * per_round;
        ca.err = h->err;
        ep_status_t s = cuda_status(launch_combine(ca, st));
        if (s) return s;
    }
    return EP_OK;
}

ep_status_t ep_combine(const void* y, const ep_handle_t* h, const float* topk_weights, void* out,
                       void* stream) {
    return ep_combine_ex(y, nullptr, EP_QUANT_NONE, 0, h, topk_weights, nullptr, out, stream);
}

ep_status_t ep_group_limited_gating(const float* logits, int32_t T, int32_t E, int32_t n_group,
                                    int32_t topk_group, int32_t per_group, int64_t* topk_idx,
                                    float* topk_weights, int32_t* err, void* stream) {
    if (T < 0 || T > (1 << 24) || E < 1 || E > kMaxExperts) return EP_ERR_INVALID_ARG;
    if (n_group < 1 || n_group > 32 || E % n_group != 0) return EP_ERR_INVALID_ARG;
    if (topk_group < 1 || topk_group > n_group || per_group < 1 || per_group > E / n_group) return EP_ERR_INVALID_ARG;
    if (topk_group * per_group > kMaxTopk) return EP_ERR_INVALID_ARG;
    if (err == nullptr) return EP_ERR_INVALID_ARG;
    if (T > 0 && (logits == nullptr || topk_idx == nullptr || topk_weights == nullptr)) return EP_ERR_INVALID_ARG;
    GateArgs g{};
    g.logits = logits;
    g.T = T; g.E = E; g.n_group = n_group; g.topk_group = topk_group; g.per_group = per_group;
    g.vec_ok = aligned16(logits) && E % 4 == 0;
    g.vec8_ok = (reinterpret_cast<uintptr_t>(logits) & 31u) == 0 && E % 8 == 0;
    g.topk_idx = topk_idx; g.topk_weights = topk_weights;
    g.err = err;
    return cuda_status(launch_gate(g, static_cast<cudaStream_t>(stream)));
}

ep_status_t ep_write_padding_rows(const int32_t* psum, const int32_t* counts, int32_t n_experts, void* recv_x,
                                  int64_t row_bytes, void* recv_scales, int64_t scale_row_bytes,
                                  int32_t* recv_topk_idx, float* recv_topk_weights, int32_t K,
                                  int32_t* recv_src_metadata, int64_t capacity, void* stream) {
    if (n_experts < 1 || n_experts > kMaxExperts || psum == nullptr || counts == nullptr) return EP_ERR_INVALID_ARG;
    if (capacity < 0 || row_bytes < 16 || row_bytes % 16 != 0 || scale_row_bytes < 0) return EP_ERR_INVALID_ARG;
    if (K < 1 || K > kMaxTopk) return EP_ERR_INVALID_ARG;
    if (capacity > 0 && (recv_x == nullptr || !aligned16(recv_x))) return EP_ERR_INVALID_ARG;
    if (capacity == 0) return EP_OK;
    PadArgs p{};
    p.psum = psum; p.cnt = counts; p.n = n_experts;
    p.recv_x = static_cast<uint8_t*>(recv_x); p.row_bytes = row_bytes;
    p.recv_scales = static_cast<uint8_t*>(recv_scales); p.scale_row_bytes = recv_scales ? scale_row_bytes : 0;
    p.recv_topk_idx = recv_topk_idx; p.recv_topk_weights = recv_topk_weights; p.K = K;
    p.recv_meta = recv_src_metadata; p.capacity = capacity;
    return cuda_status(launch_padding(p, static_cast<cudaStream_t>(stream)));
}

ep_status_t ep_route(const int64_t* topk_idx, const float* topk_weights, int32_t T, int32_t K, int32_t E, int32_t R,
                     int32_t A, int32_t token_offset, int32_t* recv_topk_idx, float* recv_topk_weights,
                     int64_t recv_capacity, ep_handle_t* h, void* ws, size_t ws_bytes, void* stream) {
    if (!sizes_ok(T, K, E, R) || h == nullptr || A < 1) return EP_ERR_INVALID_ARG;
    if (ep_recv_capacity_bound(T, K, E, A) >= (int64_t)INT32_MAX) return EP_ERR_INVALID_ARG;
    if (recv_capacity < 0 || recv_capacity >= (int64_t)INT32_MAX) return EP_ERR_INVALID_ARG;
    if (h->psum_num_recv_tokens_per_expert == nullptr || h->num_recv_tokens_per_expert == nullptr ||
        h->err == nullptr)
        return EP_ERR_INVALID_ARG;
    if (T > 0 && (h->dst_buffer_slot_idx == nullptr || topk_idx == nullptr || topk_weights == nullptr))
        return EP_ERR_INVALID_ARG;
    if (recv_capacity > 0 && (h->recv_src_metadata == nullptr || recv_topk_idx == nullptr ||
                              recv_topk_weights == nullptr))
        return EP_ERR_INVALID_ARG;
    const WsLayout L = ws_layout(T, K, E, R);
    if (ws == nullptr || ws_bytes < L.total) return EP_ERR_INVALID_ARG;
    h->num_tokens = T; h->num_topk = K; h->num_experts = E; h->num_ranks = R;
    h->expert_alignment = A; h->num_rounds = 1; h->recv_capacity = recv_capacity; h->low_latency = 0;
    RouteArgs r = route_args(ws, L, topk_idx, topk_weights, T, K, E, R);
    r.A = A;
    r.capacity = recv_capacity;
    r.check_capacity = 1;
    r.assign = 1;
    r.vector_ok = aligned16(topk_idx) && aligned16(topk_weights) && aligned16(recv_topk_idx) &&
                  aligned16(recv_topk_weights);
    r.dst_slot = h->dst_buffer_slot_idx;
    r.topk_copy = h->topk_idx;
    r.recv_meta = h->recv_src_metadata;
    r.recv_topk_idx = recv_topk_idx;
    r.recv_topk_weights = recv_topk_weights;
    r.psum = h->psum_num_recv_tokens_per_expert;
    r.num_recv = h->num_recv_tokens_per_expert;
    r.err_out = h->err;
    r.token_offset = token_offset;
    return cuda_status(launch_route(r, static_cast<cudaStream_t>(stream)));
}

ep_status_t ep_pack_peer(const void* x, const ep_handle_t* h, const int32_t* send_topk_idx,
                         const float* send_topk_weights, const int32_t* counts_all, int32_t G, int32_t g, int32_t A,
                         const ep_dispatch_opts_t* opts, void* const* peer_recv_x, void* const* peer_recv_scales,
                         int32_t* const* peer_recv_topk_idx, float* const* peer_recv_topk_weights,
                         int32_t* const* peer_recv_metadata, int64_t peer_capacity, void* stream) {
    if (h == nullptr || opts == nullptr || counts_all == nullptr) return EP_ERR_INVALID_ARG;
    const int T = h->num_tokens, K = h->num_topk, E = h->num_experts, H = h->hidden;
    if (!sizes_ok(T, K, E, h->num_ranks) || G < 1 || g < 0 || g >= G || E % G != 0 || A < 1) return EP_ERR_INVALID_ARG;
    if (H < 16 || H > 65536 || H % 16 != 0 || peer_capacity < 0) return EP_ERR_INVALID_ARG;
    if (h->expert_alignment != 1 || h->topk_idx == nullptr || h->err == nullptr) return EP_ERR_INVALID_ARG;
    const int quant = opts->quant;
    const int qs = quant == EP_QUANT_NONE ? 16 : opts->quant_size;
    if (quant != EP_QUANT_NONE && quant != EP_QUANT_FP8_E4M3 && quant != EP_QUANT_INT8) return EP_ERR_INVALID_ARG;
    if (quant != EP_QUANT_NONE && !(qs == 16 || qs == 32 || qs == 64 || qs == 128 || qs == 256 || qs == 512))
        return EP_ERR_INVALID_ARG;
    if (quant != EP_QUANT_NONE && (H % qs != 0 || peer_recv_scales == nullptr)) return EP_ERR_INVALID_ARG;
    if (opts->scale_ue8m0 && quant != EP_QUANT_NONE && !opts->round_scale) return EP_ERR_INVALID_ARG;
    if (T > 0 && (x == nullptr || !aligned16(x) || h->dst_buffer_slot_idx == nullptr || send_topk_idx == nullptr ||
                  send_topk_weights == nullptr || h->recv_src_metadata == nullptr))
        return EP_ERR_INVALID_ARG;
    if (peer_recv_x == nullptr || peer_recv_topk_idx == nullptr || peer_recv_topk_weights == nullptr ||
        peer_recv_metadata == nullptr)
        return EP_ERR_INVALID_ARG;
    PeerPackArgs p{};
    p.x = static_cast<const uint16_t*>(x);
    p.T = T; p.H = H; p.K = K; p.E = E; p.G = G; p.g = g; p.A = A;
    p.dst_slot = h->dst_buffer_slot_idx; p.topk_copy = h->topk_idx;
    p.send_topk_idx = send_topk_idx; p.send_topk_weights = send_topk_weights; p.send_meta = h->recv_src_metadata;
    p.counts_all = counts_all;
    p.peer_x = peer_recv_x; p.peer_scales = peer_recv_scales; p.peer_topk_idx = peer_recv_topk_idx;
    p.peer_topk_weights = peer_recv_topk_weights; p.peer_meta = peer_recv_metadata;
    p.capacity = peer_capacity;
    p.quant_size = qs; p.round_scale = opts->round_scale ? 1 : 0;
    p.scale_bytes = (quant != EP_QUANT_NONE && opts->scale_ue8m0) ? 1 : 0;
    p.err = h->err;
    return cuda_status(launch_pack_peer(p, quant, static_cast<cudaStream_t>(stream)));
}

ep_status_t ep_receiver_layout(const int32_t* counts_all, int32_t G, int32_t g, int32_t E, int32_t A, int32_t* psum,
                               int32_t* counts, void* stream) {
    if (counts_all == nullptr || psum == nullptr || counts == nullptr) return EP_ERR_INVALID_ARG;
    if (G < 1 || g < 0 || g >= G || E < 1 || E > kMaxExperts || E % G != 0 || A < 1) return EP_ERR_INVALID_ARG;
    return cuda_status(launch_receiver_layout(counts_all, G, g, E, A, psum, counts, static_cast<cudaStream_t>(stream)));
}

ep_status_t ep_combine_peer(void* const* peer_y, const ep_handle_t* h, const int32_t* counts_all, int32_t G, int32_t g,
                            int32_t A, const float* topk_weights, void* out, int64_t peer_capacity, void* stream) {
    if (h == nullptr || counts_all == nullptr || peer_y == nullptr) return EP_ERR_INVALID_ARG;
    const int T = h->num_tokens, K = h->num_topk, E = h->num_experts, H = h->hidden;
    if (!sizes_ok(T, K, E, h->num_ranks) || G < 1 || g < 0 || g >= G || E % G != 0 || A < 1) return EP_ERR_INVALID_ARG;
    if (H < 8 || H > 65536 || H % 8 != 0 || peer_capacity < 0 || h->err == nullptr) return EP_ERR_INVALID_ARG;
    if (T > 0 && (out == nullptr || !aligned16(out) || topk_weights == nullptr || h->dst_buffer_slot_idx == nullptr ||
                  h->topk_idx == nullptr))
        return EP_ERR_INVALID_ARG;
    PeerCombineArgs c{};
    c.peer_y = peer_y;
    c.T = T; c.H = H; c.K = K; c.E = E; c.G = G; c.g = g; c.A = A;
    c.dst_slot = h->dst_buffer_slot_idx; c.topk_copy = h->topk_idx; c.topk_weights = topk_weights;
    c.counts_all = counts_all; c.out = static_cast<uint16_t*>(out); c.capacity = peer_capacity; c.err = h->err;
    return cuda_status(launch_combine_peer(c, static_cast<cudaStream_t>(stream)));
}

ep_status_t ep_ipc_export(const void* ptr, void* handle64, int64_t* offset) {
    if (ptr == nullptr || handle64 == nullptr || offset == nullptr) return EP_ERR_INVALID_ARG;
    static_assert(sizeof(cudaIpcMemHandle_t) == 64, "64-byte IPC handle");
    // the allocation's base (allocators hand out pieces of larger allocations):
    // cuMemGetAddressRange, resolved through the runtime
    typedef CUresult (*RangeFn)(CUdeviceptr*, size_t*, CUdeviceptr);
    static RangeFn range = nullptr;
    if (range == nullptr) {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || f == nullptr)
            return EP_ERR_CUDA;
        range = reinterpret_cast<RangeFn>(f);
    }
    CUdeviceptr base = 0;
    size_t bytes = 0;
    if (range(&base, &bytes, reinterpret_cast<CUdeviceptr>(ptr)) != CUDA_SUCCESS) return EP_ERR_CUDA;
    cudaIpcMemHandle_t h;
    ep_status_t s = cuda_status(cudaIpcGetMemHandle(&h, reinterpret_cast<void*>(base)));
    if (s) return s;
    memcpy(handle64, &h, sizeof h);
    *offset = (int64_t)(reinterpret_cast<uintptr_t>(ptr) - (uintptr_t)base);
    return EP_OK;
}

ep_status_t ep_ipc_import(const void* handle64, void** base) {
    if (handle64 == nullptr || base == nullptr) return EP_ERR_INVALID_ARG;
    cudaIpcMemHandle_t h;
    memcpy(&h, handle64, sizeof h);
    return cuda_status(cudaIpcOpenMemHandle(base, h, cudaIpcMemLazyEnablePeerAccess));
}

ep_status_t ep_ipc_close(void* base) {
    if (base == nullptr) return EP_ERR_INVALID_ARG;
    return cuda_status(cudaIpcCloseMemHandle(base));
}

ep_status_t ep_read_error(const int32_t* err, void* stream, int32_t* host_status) {
    if (err == nullptr || host_status == nullptr) return EP_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    ep_status_t s = cuda_status(cudaMemcpyAsync(host_status, err, sizeof(int32_t), cudaMemcpyDeviceToHost, st));
    if (s) return s;
    return cuda_status(cudaStreamSynchronize(st));
}

ep_status_t ep_copy_recv_counts(const ep_handle_t* h, void* stream, int32_t* host_counts,
                                int64_t* num_recv_rows) {
    if (h == nullptr || h->num_experts < 1) return EP_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int32_t last = 0;
    ep_status_t s;
    if (host_counts) {
        s = cuda_status(cudaMemcpyAsync(host_counts, h->num_recv_tokens_per_expert,
                                        sizeof(int32_t) * h->num_experts, cudaMemcpyDeviceToHost, st));
        if (s) return s;
    }
    if (num_recv_rows) {
        s = cuda_status(cudaMemcpyAsync(&last, h->psum_num_recv_tokens_per_expert + h->num_experts - 1,
                                        sizeof(int32_t), cudaMemcpyDeviceToHost, st));
        if (s) return s;
    }
    s = cuda_status(cudaStreamSynchronize(st));
    if (s) return s;
    if (num_recv_rows) *num_recv_rows = last;
    return EP_OK;
}

}  // extern "C"
