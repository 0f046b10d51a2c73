// Internal declarations shared by the kernels and the C-ABI layer of libep.so.
//
// Pipeline of one dispatch (all on the caller's stream, no host sync):
//   k_layout (one CTA per chunk of 128 or 256 tokens: validated routing,
//   per-entry rank inside its chunk, per-chunk expert / rank histograms,
//   is_token_in_rank) -> k_scan (expert counts, aligned expert segments,
//   chunk row offsets, padding map, status) -> k_slots (received row of every
//   entry, per-row metadata) -> k_pack per round (persistent: TMA bulk row
//   copies or fused quantisation, zeroed padding rows).  Every kernel after
//   k_layout is launched as a programmatic dependent of its predecessor.
// Combine is one persistent kernel per round: gather + k-order fp32 FMA.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/ep.h"

namespace ep {

constexpr int kLayoutThreads = 256; // 8 warps
constexpr int kLayoutWarps = kLayoutThreads / 32;
constexpr int kMaxTopk = 16;
constexpr int kMaxExperts = 1024;
constexpr int kMaxRanks = 256;
constexpr int kMaxChunkEntries = 2048;  // tokens per chunk x K
constexpr int kMaxBatches = kMaxChunkEntries / kLayoutWarps / 32;  // 8

// Tokens per layout chunk, as a power of two: 256 (K <= 8 and R <= 64) or 128.
inline int chunk_log2(int K, int R) { return (K <= 8 && R <= 64) ? 8 : 7; }

// Byte offsets of the workspace regions (each 256-byte aligned).  Every
// region is fully written before it is read within one call, so the
// workspace never needs clearing.
struct WsLayout {
    size_t hdr;          // int32[16]: [1] received rows, [2] padding rows
    size_t pad_base;     // int32[E+1] exclusive prefix sum of padding rows
    size_t pad_start;    // int32[E]   first padding row of expert e
    size_t chunk_hist;   // int32[nchunks*E] per-chunk expert histogram
    size_t chunk_off;    // int32[nchunks*E] row offset of (chunk, expert)
    size_t chunk_rcnt;   // int32[nchunks*R] per-chunk count of tokens reaching rank r
    size_t chunk_err;    // int32[nchunks]   per-chunk status
    size_t total;
    int nchunks, log2_chunk;
};

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

inline WsLayout ws_layout(int T, int K, int E, int R) {
    WsLayout w{};
    w.log2_chunk = chunk_log2(K, R);
    const int C = 1 << w.log2_chunk;
    w.nchunks = (T + C - 1) / C;
    const size_t nc = (size_t)w.nchunks;
    size_t o = 0;
    w.hdr = o;        o = align256(o + 16 * sizeof(int32_t));
    w.pad_base = o;   o = align256(o + sizeof(int32_t) * (E + 1));
    w.pad_start = o;  o = align256(o + sizeof(int32_t) * E);
    w.chunk_hist = o; o = align256(o + sizeof(int32_t) * nc * E);
    w.chunk_off = o;  o = align256(o + sizeof(int32_t) * nc * E);
    w.chunk_rcnt = o; o = align256(o + sizeof(int32_t) * nc * R);
    w.chunk_err = o;  o = align256(o + sizeof(int32_t) * nc);
    w.total = o;
    return w;
}

struct LayoutArgs {
    const int64_t* topk_idx;
    int T, K, E, R, L, log2_chunk;
    int32_t* rank_in_chunk;     // [T,K] or null
    int32_t* chunk_hist;        // [nchunks,E]
    uint8_t* is_token_in_rank;  // [T,R] or null
    int32_t* topk_copy;         // [T,K] or null
    int32_t* chunk_rcnt;        // [nchunks,R]
    int32_t* chunk_err;         // [nchunks]
};

struct ScanArgs {
    int E, R, A, nchunks;
    int64_t capacity;
    int check_capacity;
    const int32_t* chunk_hist;   // [nchunks,E]
    const int32_t* chunk_rcnt;   // [nchunks,R]
    const int32_t* chunk_err;    // [nchunks]
    int32_t* chunk_off;          // [nchunks,E] out; null = layout outputs only
    int32_t* pad_base;           // [E+1] or null
    int32_t* pad_start;          // [E] or null
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
    int T, K, E, L, log2_chunk;
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
    int vector_ok;              // the four [.,K] arrays are 16-byte aligned
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
