// Internal declarations shared by the kernels and the C-ABI layer of libep.so.
//
// Pipeline of one dispatch (all on the caller's stream, no host sync):
//   memset(ws counters) -> k_layout (one CTA per 128-token chunk: validated
//   routing, per-chunk expert histograms, per-entry rank inside its chunk,
//   is_token_in_rank, counters) -> k_scan (aligned expert segments, chunk
//   offsets, padding map) -> k_slots (received row of every entry, per-row
//   metadata) -> k_pack per round (persistent: TMA bulk row copies or fused
//   quantisation, zeroed padding rows).
// Combine is one persistent kernel per round: gather + k-order fp32 FMA.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/ep.h"

namespace ep {

constexpr int kChunkTokens = 128;   // tokens per layout CTA
constexpr int kLayoutThreads = 256; // 8 warps
constexpr int kLayoutWarps = kLayoutThreads / 32;
constexpr int kMaxTopk = 16;
constexpr int kMaxExperts = 1024;
constexpr int kMaxRanks = 256;
constexpr int kMaxBatches = (kChunkTokens * kMaxTopk / kLayoutWarps) / 32;  // 8

// Byte offsets of the workspace regions (each 256-byte aligned).
struct WsLayout {
    size_t hdr;          // int32[16]: [0] device error of k_layout, [1] rows, [2] padding rows
    size_t counts;       // int32[E]   per-expert counts (atomics; zeroed)
    size_t rank_counts;  // int32[R]   per-rank token counts (atomics; zeroed)
    size_t zero_bytes;   // [0, zero_bytes) is cleared at the start of each call
    size_t pad_base;     // int32[E+1] exclusive prefix sum of padding rows
    size_t pad_start;    // int32[E]   first padding row of expert e
    size_t chunk_off;    // int32[nchunks*E] chunk histogram, then row offsets
    size_t total;
    int nchunks;
};

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

inline WsLayout ws_layout(int T, int K, int E, int R) {
    (void)K;
    WsLayout w{};
    w.nchunks = (T + kChunkTokens - 1) / kChunkTokens;
    size_t o = 0;
    w.hdr = o;         o = align256(o + 16 * sizeof(int32_t));
    w.counts = o;      o = align256(o + sizeof(int32_t) * E);
    w.rank_counts = o; o = align256(o + sizeof(int32_t) * R);
    w.zero_bytes = o;
    w.pad_base = o;    o = align256(o + sizeof(int32_t) * (E + 1));
    w.pad_start = o;   o = align256(o + sizeof(int32_t) * E);
    w.chunk_off = o;   o = align256(o + sizeof(int32_t) * (size_t)w.nchunks * E);
    w.total = o;
    return w;
}

struct LayoutArgs {
    const int64_t* topk_idx;
    int T, K, E, R, L;
    int32_t* rank_in_chunk;     // [T,K] or null
    int32_t* chunk_hist;        // [nchunks,E] or null
    uint8_t* is_token_in_rank;  // [T,R] or null
    int32_t* topk_copy;         // [T,K] or null
    int32_t* counts;            // ws [E]
    int32_t* rank_counts;       // ws [R]
    int32_t* err;               // ws hdr[0]
};

struct ScanArgs {
    int E, R, A, nchunks;
    int64_t capacity;
    int check_capacity;
    const int32_t* counts;       // ws [E]
    const int32_t* rank_counts;  // ws [R]
    const int32_t* layout_err;   // ws hdr[0]
    int32_t* chunk_off;          // ws [nchunks,E]: histogram in, offsets out; null = layout only
    int32_t* pad_base;           // ws [E+1]
    int32_t* pad_start;          // ws [E]
    int32_t* hdr;                // ws hdr: [1] rows, [2] padding rows
    int32_t* psum;               // [E] or null
    int32_t* num_recv;           // [E] or null
    int32_t* num_tokens_per_expert;  // [E] or null
    int32_t* num_tokens_per_rank;    // [R] or null
    int32_t* cumulative;         // [E] or null
    int32_t* err_out;            // [1]
};

struct SlotsArgs {
    const int64_t* topk_idx;
    const float* topk_weights;
    int T, K, E, L;
    int32_t* dst_slot;          // in: rank inside chunk; out: received row (-1 = none)
    const int32_t* chunk_off;   // [nchunks,E] row offset of (chunk, expert)
    int32_t* recv_meta;
    int32_t* recv_topk_idx;
    float* recv_topk_weights;
    float* recv_scales;         // null when not quantised
    int nscales;                // scales per row (0 when not quantised)
    int64_t capacity;
    const int32_t* pad_base;
    const int32_t* pad_start;
    const int32_t* hdr;         // [2] = padding rows
    int max_pad;                // host bound on padding rows: E * (A - 1)
};

struct PackArgs {
    const uint16_t* x;
    int H, K, E;
    const int32_t* dst_slot;    // [T,K] received row of each entry (-1 = none)
    uint8_t* recv_x;
    float* recv_scales;
    int64_t capacity;
    const int32_t* pad_base;
    const int32_t* pad_start;
    const int32_t* hdr;         // [2] = padding rows
    int tokens_per_rank, per_round, round, n_tok_items, do_pad;
    int quant_size, round_scale;
    int32_t* err;
};

struct CombineArgs {
    const uint16_t* y;
    int64_t y_rows;
    int H, K, T;
    const int32_t* dst_slot;
    const float* topk_weights;
    uint16_t* out;
    int tokens_per_rank, per_round, round, n_items;
    int32_t* err;
};

// Launchers (return the CUDA error of the launch).
cudaError_t launch_layout(const LayoutArgs& a, int nchunks, cudaStream_t st);
cudaError_t launch_scan(const ScanArgs& a, cudaStream_t st);
cudaError_t launch_slots(const SlotsArgs& a, cudaStream_t st);
cudaError_t launch_pack(const PackArgs& a, int quant, cudaStream_t st);
cudaError_t launch_combine(const CombineArgs& a, cudaStream_t st);

int device_sm_count();

}  // namespace ep

// ------------------------------------------------------------ device helpers
#ifdef __CUDACC__
namespace ep {

__device__ __forceinline__ int token_of_item(int item, int tokens_per_rank, int per_round, int round) {
    const int r = item / per_round;
    return r * tokens_per_rank + round * per_round + (item - r * per_round);
}

// 16-byte load that does not allocate in L1 (each row is read once).
__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
    uint4 r;
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
        : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
        : "l"(p));
    return r;
}

__device__ __forceinline__ void st_v4(void* p, uint4 v) {
    asm volatile("st.global.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ unsigned lanemask_lt() {
    unsigned m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ void set_error(int32_t* err, int code) {
    if (err) atomicCAS(err, 0, code);
}

}  // namespace ep
#endif
