// Internal declarations shared by the kernels and the C-ABI layer of libep.so.
//
// Pipeline of one dispatch (all on the caller's stream, no host sync):
//   k_route (cooperative: chunk histograms and ranks | column prefixes |
//   segment starts, received rows, per-row metadata; two grid barriers) ->
//   k_pack per round (persistent: TMA bulk row copies or fused quantisation,
//   zeroed padding rows), launched as a programmatic dependent.
// Combine is one persistent kernel per round: gather + k-order fp32 FMA.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/ep.h"

namespace ep {

constexpr int kRouteThreads = 256;  // 8 warps
constexpr int kRouteWarps = kRouteThreads / 32;
constexpr int kMaxTopk = 16;
constexpr int kMaxExperts = 1024;
constexpr int kMaxRanks = 256;
constexpr int kMaxChunkEntries = 2048;  // tokens per chunk x K
constexpr int kMaxBatches = kMaxChunkEntries / kRouteWarps / 32;  // 8

// Tokens per routing chunk, as a power of two in [16, 256]: the largest with
// C*K <= 2048 that still gives at least 128 chunks when T allows it.
#ifndef EP_ROUTE_MIN_CHUNKS
#define EP_ROUTE_MIN_CHUNKS 128
#endif
inline int chunk_log2(int T, int K) {
    int lg = 8;
    while ((1 << lg) * K > kMaxChunkEntries) --lg;
    while (lg > 4 && ((T + (1 << lg) - 1) >> lg) < EP_ROUTE_MIN_CHUNKS) --lg;
    return lg;
}

// Byte offsets of the workspace regions (each 256-byte aligned).  Every
// region is written before it is read within one call (the barrier counter
// is cleared by the call itself), so the workspace never needs clearing.
struct WsLayout {
    size_t hdr;          // int32[16]: [0] grid-barrier counter
    size_t col_total;    // int32[E+R+1] expert counts, rank counts, error flags
    size_t chunk_hist;   // int32[nchunks*E] per-chunk expert histogram, then its prefix
    size_t chunk_rcnt;   // int32[nchunks*R] per-chunk count of tokens reaching rank r
    size_t chunk_err;    // int32[nchunks]   per-chunk status
    size_t total;
    int nchunks, log2_chunk, chunks_per_rank;
};

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

inline WsLayout ws_layout(int T, int K, int E, int R) {
    WsLayout w{};
    w.log2_chunk = chunk_log2(T, K);
    const int C = 1 << w.log2_chunk;
    const int tpr = R > 0 ? T / R : 0;
    w.chunks_per_rank = (tpr + C - 1) / C;   // chunks never straddle a source rank
    w.nchunks = R * w.chunks_per_rank;
    const size_t nc = (size_t)w.nchunks;
    size_t o = 0;
    w.hdr = o;        o = align256(o + 16 * sizeof(int32_t));
    w.col_total = o;  o = align256(o + sizeof(int32_t) * (E + R + 1));
    w.chunk_hist = o; o = align256(o + sizeof(int32_t) * nc * E);
    w.chunk_rcnt = o; o = align256(o + sizeof(int32_t) * nc * R);
    w.chunk_err = o;  o = align256(o + sizeof(int32_t) * nc);
    w.total = o;
    return w;
}

struct RouteArgs {
    const int64_t* topk_idx;
    const float* topk_weights;
    int T, K, E, R, L, A, log2_chunk, nchunks;
    int tokens_per_rank, chunks_per_rank;
    int ll_M;                   // > 0: low-latency layout with this many rows per (expert, source rank)
    int token_offset;           // added to the token index written to recv_src_metadata
    int64_t* layout_range;      // [E,R] (low-latency layout) or null
    int64_t capacity;
    int check_capacity;
    int assign;                 // 1: rows and metadata (dispatch); 0: layout outputs only
    int vector_ok;              // the four [.,K] arrays are 16-byte aligned
    // per-entry / per-row outputs (dispatch)
    int32_t* dst_slot;          // [T,K]: rank inside the chunk, then the received row
    int32_t* topk_copy;         // [T,K] or null
    int32_t* recv_meta;
    int32_t* recv_topk_idx;
    float* recv_topk_weights;
    // layout outputs (each may be null)
    uint8_t* is_token_in_rank;  // [T,R]
    int32_t* psum;
    int32_t* num_recv;
    int32_t* num_tokens_per_expert;
    int32_t* num_tokens_per_rank;
    int32_t* cumulative;
    int32_t* err_out;           // [1]
    // workspace
    unsigned* barrier;
    int32_t* col_total;
    int32_t* chunk_hist;
    int32_t* chunk_rcnt;
    int32_t* chunk_err;
    // > 0 only from the test entry points: raises the first grid barrier's
    // target past the number of CTAs, so that no CTA can pass it
    unsigned stall;
    // 1: the per-chunk tables fit in shared memory; after the first barrier
    // every CTA copies them in and sums the columns itself (no second phase)
    int fold;
};

struct PackArgs {
    const uint16_t* x;
    int H, K, E;
    const int32_t* dst_slot;    // [T,K] received row of each entry (-1 = none); a row at or
                                // past capacity is skipped and reported as EP_ERR_CAPACITY
    uint8_t* recv_x;
    float* recv_scales;
    int64_t capacity;
    const int32_t* psum;        // [E] inclusive prefix of the aligned counts (handle)
    const int32_t* cnt;         // [E] unaligned counts (handle): padding map source
    int tokens_per_rank, per_round, round, n_tok_items, do_pad;
    int quant_size, round_scale;
    int scale_bytes;            // scales stored as UE8M0 bytes (MXFP4 always)
    int x32;                    // x is 32-byte aligned: a 16-channel unit is one 32-byte load
    int early_x;                // x was complete when the kernel before this one started (the
                                // routing kernel precedes): x may be read before the wait
    int32_t* err;
};

struct CombineArgs {
    const void* y;              // bf16 rows, or 1-byte codes when y_quant != 0
    const float* y_scales;      // [rows, H / quant_size] when y_quant != 0
    int y_quant, quant_size;
    const uint16_t* shared;     // [T,H] bf16 shared-expert rows, or null
    int64_t y_rows;
    int H, K, T;
    const int32_t* dst_slot;
    const float* topk_weights;
    uint16_t* out;
    int tokens_per_rank, per_round, round, n_items;
    int32_t* err;
};

struct GateArgs {
    const float* logits;        // [T, E] router logits
    int64_t T;
    int E, n_group, topk_group, per_group;
    int vec_ok;                 // logits 16-byte aligned (rows of E % 4 == 0 floats)
    int vec8_ok;                // logits 32-byte aligned and E % 8 == 0
    int64_t* topk_idx;          // [T, K]
    float* topk_weights;        // [T, K]
    int32_t* err;               // [1] status word (cleared by the launch)
};

struct PadArgs {
    const int32_t* psum;        // [n] inclusive prefix of the aligned counts
    const int32_t* cnt;         // [n] unaligned counts
    int n;
    uint8_t* recv_x;
    int64_t row_bytes;
    uint8_t* recv_scales;       // or null
    int64_t scale_row_bytes;
    int32_t* recv_topk_idx;     // [cap, K] or null
    float* recv_topk_weights;   // [cap, K] or null
    int K;
    int32_t* recv_meta;         // [cap, 2] or null
    int64_t capacity;
};

// Multi-GPU pack and combine through peer memory (peer.cu).
struct PeerPackArgs {
    const uint16_t* x;          // this GPU's tokens [T, H]
    int T, H, K, E, G, g, A;
    const int32_t* dst_slot;    // [T, K] send rows (routing with alignment 1)
    const int32_t* topk_copy;   // [T, K] expert ids (-1 = masked)
    const int32_t* send_topk_idx;      // [rows, K] per send row
    const float* send_topk_weights;    // [rows, K]
    const int32_t* send_meta;          // [rows, 2]
    const int32_t* counts_all;  // [G, E]
    void* const* peer_x;        // [G] receivers' recv_x
    void* const* peer_scales;   // [G] or null (bf16)
    int32_t* const* peer_topk_idx;
    float* const* peer_topk_weights;
    int32_t* const* peer_meta;
    int64_t capacity;           // rows of every receiver's layout
    int quant_size, round_scale, scale_bytes;
    int32_t* err;
};

struct PeerCombineArgs {
    void* const* peer_y;        // [G] receivers' expert outputs (bf16)
    int T, H, K, E, G, g, A;
    const int32_t* dst_slot;
    const int32_t* topk_copy;
    const float* topk_weights;
    const int32_t* counts_all;
    uint16_t* out;
    int64_t capacity;
    int32_t* err;
};

// Launchers (return the CUDA error of the launch).
cudaError_t launch_route(const RouteArgs& a, cudaStream_t st);
cudaError_t launch_pack(const PackArgs& a, int quant, cudaStream_t st);
cudaError_t launch_combine(const CombineArgs& a, cudaStream_t st);
cudaError_t launch_gate(const GateArgs& a, cudaStream_t st);
cudaError_t launch_padding(const PadArgs& a, cudaStream_t st);
cudaError_t launch_pack_peer(const PeerPackArgs& a, int quant, cudaStream_t st);
cudaError_t launch_combine_peer(const PeerCombineArgs& a, cudaStream_t st);
cudaError_t launch_receiver_layout(const int32_t* C, int G, int g, int E, int A, int32_t* psum, int32_t* counts,
                                   cudaStream_t st);

int device_sm_count();

// Launches `kern` on `st` with programmatic dependent launch: the kernel may
// be scheduled while its predecessor on the stream finishes, and it waits in
// grid_dependency_wait() until the predecessor's results are visible.
template <typename... Params, typename... Args>
cudaError_t launch_dependent(void (*kern)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                             Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

}  // namespace ep

// ------------------------------------------------------------ device helpers
#ifdef __CUDACC__
namespace ep {

// Programmatic dependent launch: wait for the previous kernel's results /
// let the next kernel on the stream be scheduled.
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;"); }

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

// 32-byte load (sm_100 256-bit global load) that does not allocate in L1; p
// must be 32-byte aligned.  A warp of these reads 1 KB of whole sectors.
__device__ __forceinline__ void ld_nc_v8(const void* p, uint4& lo, uint4& hi) {
    asm("ld.global.nc.L1::no_allocate.v8.u32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
        : "=r"(lo.x), "=r"(lo.y), "=r"(lo.z), "=r"(lo.w), "=r"(hi.x), "=r"(hi.y), "=r"(hi.z), "=r"(hi.w)
        : "l"(p));
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
