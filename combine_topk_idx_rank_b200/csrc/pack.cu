// Permute / pack: every source token's row is read from HBM once and written
// to each of its received rows (one per unmasked top-k entry), as a bf16 bit
// copy or quantised once per token on the fly:
//   - FP8 e4m3 (OCP e4m3fn) or int8 with one fp32 scale per quant_size
//     channels: scale = max(amax, 1e-4) / 448 (or / 127) by IEEE division,
//     optionally rounded up to a power of two (round_scale / use_ue8m0 of
//     low_latency_dispatch, "DeepEP communication library guide v2.1"),
//     codes = RNE-saturating conversion of x / scale (IEEE division);
//   - quant_size = 128 (group) or hidden (per token) (guide v2.1, 1.3.1).
// The same persistent grid also zero-fills the padding rows that expert
// alignment adds (comparative analysis, section 3.1), and writes the
// per-row metadata (recv_src_metadata, recv_topk_idx, recv_topk_weights) and
// the final dst_buffer_slot_idx.
//
// Data movement: 16-byte vector loads that bypass L1 (x is read once) and
// 16-byte stores; every row is a whole number of 16-byte vectors and, for
// bf16 rows of 7168 channels, of 128-byte lines.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "ep_internal.cuh"

namespace ep {

namespace {

constexpr int kQuantNone = 0, kQuantFp8 = 1, kQuantInt8 = 2;

struct ItemSmem {
    int slot[kMaxTopk];
    int e[kMaxTopk];
    float w[kMaxTopk];
    float red[33];
};

// Resolves the K received rows of token t, writes dst_buffer_slot_idx and the
// per-row metadata.  Leaves the rows in s.slot (-1 = none).
__device__ __forceinline__ void token_slots(const PackArgs& a, int t, ItemSmem& s) {
    const int tid = threadIdx.x;
    const int K = a.K;
    if (tid < K) {
        const int64_t v = a.topk_idx[(int64_t)t * K + tid];
        const int e = (v >= 0 && v < a.E) ? (int)v : -1;
        int slot = -1;
        if (e >= 0) {
            const int rank = a.dst_slot[(int64_t)t * K + tid];
            const int64_t row = (int64_t)a.chunk_off[(size_t)(t / kChunkTokens) * a.E + e] + rank;
            slot = (rank >= 0 && row < a.capacity) ? (int)row : -1;
        }
        a.dst_slot[(int64_t)t * K + tid] = slot;
        s.slot[tid] = slot;
        s.e[tid] = e;
        s.w[tid] = a.topk_weights[(int64_t)t * K + tid];
    }
    __syncthreads();
    if (tid < K) {
        const int slot = s.slot[tid];
        if (slot >= 0) {
            const int rdst = s.e[tid] / a.L;
            reinterpret_cast<int2*>(a.recv_meta)[slot] = make_int2(t, tid);
            int32_t* ri = a.recv_topk_idx + (int64_t)slot * K;
            float* rw = a.recv_topk_weights + (int64_t)slot * K;
            for (int j = 0; j < K; ++j) {
                const int ej = s.e[j];
                const bool here = ej >= 0 && ej / a.L == rdst;
                ri[j] = here ? ej - rdst * a.L : -1;
                rw[j] = here ? s.w[j] : 0.0f;
            }
        }
    }
}

// Padding row number p (0-based over all experts) -> its row index.
__device__ __forceinline__ int64_t pad_row(const PackArgs& a, const int* s_pad_base, int p) {
    int lo = 0, hi = a.E;   // find the last e with pad_base[e] <= p
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (s_pad_base[mid] <= p) lo = mid; else hi = mid;
    }
    return (int64_t)a.pad_start[lo] + (p - s_pad_base[lo]);
}

__device__ __forceinline__ void pad_metadata(const PackArgs& a, int64_t row, int nscales) {
    const int tid = threadIdx.x;
    if (tid == 0) reinterpret_cast<int2*>(a.recv_meta)[row] = make_int2(-1, -1);
    for (int j = tid; j < a.K; j += blockDim.x) {
        a.recv_topk_idx[row * a.K + j] = -1;
        a.recv_topk_weights[row * a.K + j] = 0.0f;
    }
    for (int j = tid; j < nscales; j += blockDim.x) a.recv_scales[row * nscales + j] = 0.0f;
}

__device__ __forceinline__ float pow2_ceil_bits(float s) {
    // s > 0 and normal: keep the exponent if the mantissa is zero, else bump it
    const uint32_t u = __float_as_uint(s);
    const uint32_t bumped = (u & 0xff800000u) + ((u & 0x007fffffu) ? 0x00800000u : 0u);
    return __uint_as_float(bumped);
}

template <int QUANT>
__device__ __forceinline__ uint32_t quant4(float a, float b, float c, float d, float s) {
    if constexpr (QUANT == kQuantFp8) {
        const __nv_fp8x2_storage_t lo =
            __nv_cvt_float2_to_fp8x2(make_float2(__fdiv_rn(a, s), __fdiv_rn(b, s)), __NV_SATFINITE, __NV_E4M3);
        const __nv_fp8x2_storage_t hi =
            __nv_cvt_float2_to_fp8x2(make_float2(__fdiv_rn(c, s), __fdiv_rn(d, s)), __NV_SATFINITE, __NV_E4M3);
        return (uint32_t)lo | ((uint32_t)hi << 16);
    } else {
        const int qa = max(-127, min(127, __float2int_rn(__fdiv_rn(a, s))));
        const int qb = max(-127, min(127, __float2int_rn(__fdiv_rn(b, s))));
        const int qc = max(-127, min(127, __float2int_rn(__fdiv_rn(c, s))));
        const int qd = max(-127, min(127, __float2int_rn(__fdiv_rn(d, s))));
        return (uint32_t)(qa & 0xff) | ((uint32_t)(qb & 0xff) << 8) | ((uint32_t)(qc & 0xff) << 16) |
               ((uint32_t)(qd & 0xff) << 24);
    }
}

template <int QUANT>
__device__ __forceinline__ uint4 quant16(const float (&f)[16], float s) {
    uint4 q;
    q.x = quant4<QUANT>(f[0], f[1], f[2], f[3], s);
    q.y = quant4<QUANT>(f[4], f[5], f[6], f[7], s);
    q.z = quant4<QUANT>(f[8], f[9], f[10], f[11], s);
    q.w = quant4<QUANT>(f[12], f[13], f[14], f[15], s);
    return q;
}

__device__ __forceinline__ void unpack16(uint4 lo, uint4 hi, float (&f)[16]) {
    f[0] = bf16lo(lo.x); f[1] = bf16hi(lo.x); f[2] = bf16lo(lo.y); f[3] = bf16hi(lo.y);
    f[4] = bf16lo(lo.z); f[5] = bf16hi(lo.z); f[6] = bf16lo(lo.w); f[7] = bf16hi(lo.w);
    f[8] = bf16lo(hi.x); f[9] = bf16hi(hi.x); f[10] = bf16lo(hi.y); f[11] = bf16hi(hi.y);
    f[12] = bf16lo(hi.z); f[13] = bf16hi(hi.z); f[14] = bf16lo(hi.w); f[15] = bf16hi(hi.w);
}

__device__ __forceinline__ float amax16(const float (&f)[16]) {
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) m = fmaxf(m, fabsf(f[i]));
    return m;
}

__device__ __forceinline__ float finish_scale(float amax, float qmax, int round_scale) {
    float s = __fdiv_rn(fmaxf(amax, 1e-4f), qmax);
    return round_scale ? pow2_ceil_bits(s) : s;
}

}  // namespace

// ---------------------------------------------------------------- bf16 copy
template <int VPT>
__global__ void __launch_bounds__(256) k_pack_bf16(PackArgs a) {
    __shared__ ItemSmem s;
    __shared__ int s_pad_base[kMaxExperts + 1];
    const int tid = threadIdx.x;
    const int V = a.H / 8;   // 16-byte vectors per row
    const int n_pad = a.do_pad ? a.hdr[2] : 0;
    if (a.do_pad)
        for (int i = tid; i <= a.E; i += blockDim.x) s_pad_base[i] = a.pad_base[i];
    __syncthreads();
    const int n_items = a.n_tok_items + n_pad;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
        if (item < a.n_tok_items) {
            const int t = token_of_item(item, a.tokens_per_rank, a.per_round, a.round);
            token_slots(a, t, s);
            const uint4* xr = reinterpret_cast<const uint4*>(a.x + (size_t)t * a.H);
            for (int v0 = 0; v0 < V; v0 += VPT * blockDim.x) {
                uint4 r[VPT];
#pragma unroll
                for (int u = 0; u < VPT; ++u) {
                    const int v = v0 + u * blockDim.x + tid;
                    if (v < V) r[u] = ld_nc_v4(xr + v);
                }
                for (int k = 0; k < a.K; ++k) {
                    const int slot = s.slot[k];
                    if (slot < 0) continue;
                    uint4* dst = reinterpret_cast<uint4*>(a.recv_x + (size_t)slot * a.H * 2);
#pragma unroll
                    for (int u = 0; u < VPT; ++u) {
                        const int v = v0 + u * blockDim.x + tid;
                        if (v < V) st_v4(dst + v, r[u]);
                    }
                }
            }
        } else {
            const int64_t row = pad_row(a, s_pad_base, item - a.n_tok_items);
            if (row < a.capacity) {
                uint4* dst = reinterpret_cast<uint4*>(a.recv_x + (size_t)row * a.H * 2);
                for (int v = tid; v < V; v += blockDim.x) st_v4(dst + v, make_uint4(0, 0, 0, 0));
                pad_metadata(a, row, 0);
            }
        }
        __syncthreads();
    }
}

// ------------------------------------------------- group quantisation (<=512)
// A thread owns 16 consecutive channels (two 16-byte loads, one 16-byte
// store); a group of G channels is G/16 adjacent lanes, reduced by shuffles.
template <int QUANT, int G, int UPT>
__global__ void __launch_bounds__(256) k_pack_group(PackArgs a) {
    __shared__ ItemSmem s;
    __shared__ int s_pad_base[kMaxExperts + 1];
    constexpr int kLanes = G / 16;
    constexpr float kQmax = QUANT == kQuantFp8 ? 448.0f : 127.0f;
    const int tid = threadIdx.x;
    const int U = a.H / 16;
    const int nscales = a.H / G;
    const int n_pad = a.do_pad ? a.hdr[2] : 0;
    if (a.do_pad)
        for (int i = tid; i <= a.E; i += blockDim.x) s_pad_base[i] = a.pad_base[i];
    __syncthreads();
    const int n_items = a.n_tok_items + n_pad;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
        if (item < a.n_tok_items) {
            const int t = token_of_item(item, a.tokens_per_rank, a.per_round, a.round);
            token_slots(a, t, s);
            const uint4* xr = reinterpret_cast<const uint4*>(a.x + (size_t)t * a.H);
            for (int u0 = 0; u0 < U; u0 += UPT * blockDim.x) {
                uint4 q[UPT];
                float sc[UPT];
#pragma unroll
                for (int j = 0; j < UPT; ++j) {
                    const int u = u0 + j * blockDim.x + tid;
                    float f[16];
                    if (u < U) {
                        unpack16(ld_nc_v4(xr + 2 * u), ld_nc_v4(xr + 2 * u + 1), f);
                    } else {
#pragma unroll
                        for (int i = 0; i < 16; ++i) f[i] = 0.0f;
                    }
                    float m = amax16(f);
#pragma unroll
                    for (int o = kLanes / 2; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                    sc[j] = finish_scale(m, kQmax, a.round_scale);
                    q[j] = quant16<QUANT>(f, sc[j]);
                }
                for (int k = 0; k < a.K; ++k) {
                    const int slot = s.slot[k];
                    if (slot < 0) continue;
                    uint8_t* dst = a.recv_x + (size_t)slot * a.H;
#pragma unroll
                    for (int j = 0; j < UPT; ++j) {
                        const int u = u0 + j * blockDim.x + tid;
                        if (u < U) {
                            st_v4(dst + 16 * (size_t)u, q[j]);
                            if ((u % kLanes) == 0) a.recv_scales[(size_t)slot * nscales + u / kLanes] = sc[j];
                        }
                    }
                }
            }
        } else {
            const int64_t row = pad_row(a, s_pad_base, item - a.n_tok_items);
            if (row < a.capacity) {
                uint4* dst = reinterpret_cast<uint4*>(a.recv_x + (size_t)row * a.H);
                for (int v = tid; v < U; v += blockDim.x) st_v4(dst + v, make_uint4(0, 0, 0, 0));
                pad_metadata(a, row, nscales);
            }
        }
        __syncthreads();
    }
}

// ----------------------------------------------- per-token quantisation (G=H)
// The whole row stays in registers (UPT units of 16 channels per thread) while
// the block reduces its amax.
template <int QUANT, int UPT>
__global__ void __launch_bounds__(1024) k_pack_token(PackArgs a) {
    __shared__ ItemSmem s;
    __shared__ int s_pad_base[kMaxExperts + 1];
    constexpr float kQmax = QUANT == kQuantFp8 ? 448.0f : 127.0f;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nwarps = blockDim.x >> 5;
    const int U = a.H / 16;
    const int n_pad = a.do_pad ? a.hdr[2] : 0;
    if (a.do_pad)
        for (int i = tid; i <= a.E; i += blockDim.x) s_pad_base[i] = a.pad_base[i];
    __syncthreads();
    const int n_items = a.n_tok_items + n_pad;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
        if (item < a.n_tok_items) {
            const int t = token_of_item(item, a.tokens_per_rank, a.per_round, a.round);
            token_slots(a, t, s);
            const uint4* xr = reinterpret_cast<const uint4*>(a.x + (size_t)t * a.H);
            uint4 raw[UPT][2];
#pragma unroll
            for (int j = 0; j < UPT; ++j) {
                const int u = j * blockDim.x + tid;
                if (u < U) {
                    raw[j][0] = ld_nc_v4(xr + 2 * u);
                    raw[j][1] = ld_nc_v4(xr + 2 * u + 1);
                } else {
                    raw[j][0] = raw[j][1] = make_uint4(0, 0, 0, 0);
                }
            }
            float m = 0.0f;
#pragma unroll
            for (int j = 0; j < UPT; ++j) {
                float f[16];
                unpack16(raw[j][0], raw[j][1], f);
                m = fmaxf(m, amax16(f));
            }
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            if (lane == 0) s.red[warp] = m;
            __syncthreads();
            if (warp == 0) {
                float v = lane < nwarps ? s.red[lane] : 0.0f;
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
                if (lane == 0) s.red[32] = v;
            }
            __syncthreads();
            const float sc = finish_scale(s.red[32], kQmax, a.round_scale);
            uint4 q[UPT];
#pragma unroll
            for (int j = 0; j < UPT; ++j) {
                float f[16];
                unpack16(raw[j][0], raw[j][1], f);
                q[j] = quant16<QUANT>(f, sc);
            }
            for (int k = 0; k < a.K; ++k) {
                const int slot = s.slot[k];
                if (slot < 0) continue;
                uint8_t* dst = a.recv_x + (size_t)slot * a.H;
#pragma unroll
                for (int j = 0; j < UPT; ++j) {
                    const int u = j * blockDim.x + tid;
                    if (u < U) st_v4(dst + 16 * (size_t)u, q[j]);
                }
                if (tid == 0) a.recv_scales[slot] = sc;
            }
        } else {
            const int64_t row = pad_row(a, s_pad_base, item - a.n_tok_items);
            if (row < a.capacity) {
                uint4* dst = reinterpret_cast<uint4*>(a.recv_x + (size_t)row * a.H);
                for (int v = tid; v < U; v += blockDim.x) st_v4(dst + v, make_uint4(0, 0, 0, 0));
                pad_metadata(a, row, 1);
            }
        }
        __syncthreads();
    }
}

// ------------------------------------------------------------------ launch
namespace {

template <typename Kern>
int blocks_per_sm(Kern k, int threads) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k, threads, 0) != cudaSuccess || n < 1) n = 1;
    return n;
}

inline int round_up32(int x) { return (x + 31) & ~31; }

template <typename Kern>
cudaError_t run(Kern k, int threads, const PackArgs& a, cudaStream_t st) {
    const int grid = device_sm_count() * blocks_per_sm(k, threads);
    k<<<grid, threads, 0, st>>>(a);
    return cudaGetLastError();
}

template <int QUANT>
cudaError_t launch_group(const PackArgs& a, cudaStream_t st) {
    const int U = a.H / 16;
    const int threads = min(256, round_up32((U + 1) / 2));   // 2 units per thread
    switch (a.quant_size) {
        case 16: return run(k_pack_group<QUANT, 16, 2>, threads, a, st);
        case 32: return run(k_pack_group<QUANT, 32, 2>, threads, a, st);
        case 64: return run(k_pack_group<QUANT, 64, 2>, threads, a, st);
        case 128: return run(k_pack_group<QUANT, 128, 2>, threads, a, st);
        case 256: return run(k_pack_group<QUANT, 256, 2>, threads, a, st);
        case 512: return run(k_pack_group<QUANT, 512, 2>, threads, a, st);
        default: return cudaErrorInvalidValue;
    }
}

template <int QUANT>
cudaError_t launch_token(const PackArgs& a, cudaStream_t st) {
    const int U = a.H / 16;
    if (U <= 2 * 1024) {
        const int threads = min(1024, round_up32((U + 1) / 2));
        return run(k_pack_token<QUANT, 2>, threads, a, st);
    }
    const int threads = min(1024, round_up32((U + 3) / 4));
    return run(k_pack_token<QUANT, 4>, threads, a, st);
}

}  // namespace

cudaError_t launch_pack(const PackArgs& a, int quant, cudaStream_t st) {
    if (quant == EP_QUANT_NONE) {
        const int V = a.H / 8;
        // threads: a multiple of 32 that splits the row into passes of 4 vectors
        const int passes = (V + 4 * 256 - 1) / (4 * 256);
        const int threads = min(256, round_up32((V + 4 * passes - 1) / (4 * passes)));
        return run(k_pack_bf16<4>, threads, a, st);
    }
    const bool per_token = a.quant_size == a.H;
    if (quant == EP_QUANT_FP8_E4M3)
        return per_token ? launch_token<kQuantFp8>(a, st) : launch_group<kQuantFp8>(a, st);
    return per_token ? launch_token<kQuantInt8>(a, st) : launch_group<kQuantInt8>(a, st);
}

}  // namespace ep
