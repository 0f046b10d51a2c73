// Expert parallelism over several GPUs through peer memory (one process per
// GPU, NVLink / NVSwitch peer stores and loads).  GPU g of G routes its own
// tokens with alignment 1 (k_route, its send order); with the all-gathered
// count matrix C [G, E] on the device, every CTA derives where each expert's
// rows of this GPU land:
//   send_off[e]  = sum of C[g][e'] over e' < e        (this GPU's send rows)
//   before[e]    = sum of C[g'][e] over g' < g        (earlier GPUs' rows of e)
//   aligned[e]   = ceil(sum_g' C[g'][e] / A) * A
//   seg_start[e] = sum of aligned[e'] over e' < e in the receiver's block
//                  [d E/G, e), d = e / (E/G)
// so the row of send row s of expert e on receiver d is
//   s - send_off[e] + before[e] + seg_start[e]
// ("DeepEP V1 vs V2 comparative analysis", section 6.1: the normal mode's
// dispatch of each rank's tokens into the receivers' buffers; expert
// alignment, section 3.1; the deterministic order, section 8.4).
//
// k_pack_peer stores each token's row (bf16, or FP8 / int8 codes with their
// scales, quantised once) and each entry's recv_topk_idx / weights / metadata
// row straight into the receiver's layout; k_combine_peer loads each token's
// rows from the receivers' expert outputs and reduces them in k order.  Plain
// peer loads and stores only, and no waits on other GPUs (the
// caller's collectives order the steps).
#include "ep_internal.cuh"
#include "quant.cuh"

namespace ep {

namespace {

constexpr int kPeerThreads = 256;

// Exclusive prefix, in place, of n <= kMaxExperts values in shared memory
// (every thread of the block calls it); returns the total.
__device__ int block_exclusive_scan(int* v, int n, int* s_warp) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
    const int per = (n + blockDim.x - 1) / blockDim.x;
    const int e0 = min(tid * per, n), e1 = min(e0 + per, n);
    int sum = 0;
    for (int e = e0; e < e1; ++e) sum += v[e];
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int x = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += x;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int w = lane < nwarps ? s_warp[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int x = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += x;
        }
        if (lane < nwarps) s_warp[lane] = w;
    }
    __syncthreads();
    int run = incl - sum + (warp > 0 ? s_warp[warp - 1] : 0);
    for (int e = e0; e < e1; ++e) {
        const int x = v[e];
        v[e] = run;
        run += x;
    }
    const int total = s_warp[nwarps - 1];
    __syncthreads();
    return total;
}

// s_delta[e] = (row on e's receiver) - (send row) for this GPU's rows of e.
__device__ void peer_deltas(const int32_t* C, int G, int g, int E, int A, int* s_delta, int* s_a, int* s_b,
                            int* s_warp) {
    const int Eg = E / G;
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int tot = 0, bef = 0;
        for (int q = 0; q < G; ++q) {
            const int c = C[(size_t)q * E + e];
            tot += c;
            if (q < g) bef += c;
        }
        s_a[e] = C[(size_t)g * E + e];                     // -> send_off
        s_b[e] = (int)(((int64_t)tot + A - 1) / A * A);    // -> prefix of the aligned totals
        s_delta[e] = bef;
    }
    __syncthreads();
    block_exclusive_scan(s_a, E, s_warp);
    block_exclusive_scan(s_b, E, s_warp);
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        const int seg = s_b[e] - s_b[(e / Eg) * Eg];
        s_delta[e] += seg - s_a[e];
    }
    __syncthreads();
}

// FP8 / int8 groups of G2 channels (QUANT 0: bf16 rows); a thread owns
// 16-channel units tid, tid + blockDim, ...
template <int QUANT, int G2>
__global__ void __launch_bounds__(kPeerThreads) k_pack_peer(PeerPackArgs a) {
    grid_dependency_wait();
    grid_launch_dependents();
    __shared__ int s_delta[kMaxExperts], s_a[kMaxExperts], s_b[kMaxExperts], s_warp[32];
    __shared__ int s_row[kMaxTopk], s_dst[kMaxTopk];
    constexpr int kLanes = G2 / 16;
    const int tid = threadIdx.x, K = a.K;
    const int U = a.H / 16;
    const int Eg = a.E / a.G;
    const int64_t row_bytes = QUANT == 0 ? (int64_t)a.H * 2 : (int64_t)a.H;
    const int nscales = QUANT == 0 ? 0 : a.H / G2;
    const int srb = nscales * (a.scale_bytes ? 1 : 4);
    peer_deltas(a.counts_all, a.G, a.g, a.E, a.A, s_delta, s_a, s_b, s_warp);
    for (int t = blockIdx.x; t < a.T; t += gridDim.x) {
        if (tid < K) {
            const int slot = a.dst_slot[(int64_t)t * K + tid];
            const int e = a.topk_copy[(int64_t)t * K + tid];
            int row = -1, d = 0;
            if (slot >= 0 && e >= 0) {
                d = e / Eg;
                const int64_t r = (int64_t)slot + s_delta[e];
                if (r < a.capacity) {
                    row = (int)r;
                    // the entry's per-row metadata, from its send row
                    int32_t* ri = a.peer_topk_idx[d] + (int64_t)row * K;
                    float* rw = a.peer_topk_weights[d] + (int64_t)row * K;
                    for (int j = 0; j < K; ++j) {
                        ri[j] = a.send_topk_idx[(int64_t)slot * K + j];
                        rw[j] = a.send_topk_weights[(int64_t)slot * K + j];
                    }
                    reinterpret_cast<int2*>(a.peer_meta[d])[row] = reinterpret_cast<const int2*>(a.send_meta)[slot];
                } else {
                    set_error(a.err, EP_ERR_CAPACITY);
                }
            }
            s_row[tid] = row;
            s_dst[tid] = d;
        }
        __syncthreads();
        const uint4* xr = reinterpret_cast<const uint4*>(a.x + (size_t)t * a.H);
        for (int u = tid; u < (U + 31) / 32 * 32; u += blockDim.x) {   // whole warps (group shuffles)
            uint4 lo = make_uint4(0, 0, 0, 0), hi = lo;
            if (u < U) {
                lo = ld_nc_v4(xr + 2 * u);
                hi = ld_nc_v4(xr + 2 * u + 1);
            }
            if constexpr (QUANT == 0) {
                if (u < U)
                    for (int k = 0; k < K; ++k) {
                        const int row = s_row[k];
                        if (row < 0) continue;
                        uint4* dst = reinterpret_cast<uint4*>(static_cast<uint8_t*>(a.peer_x[s_dst[k]]) +
                                                              (int64_t)row * row_bytes) + 2 * u;
                        st_v4(dst, lo);
                        st_v4(dst + 1, hi);
                    }
            } else {
                float f[16];
                unpack16(lo, hi, f);
                float m = amax16(f);
#pragma unroll
                for (int o = kLanes / 2; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                const float sc = finish_scale(m, QUANT == kQuantFp8 ? 448.0f : 127.0f, a.round_scale);
                const uint4 q = quant16<QUANT>(f, sc);
                if (u < U)
                    for (int k = 0; k < K; ++k) {
                        const int row = s_row[k];
                        if (row < 0) continue;
                        uint8_t* base = static_cast<uint8_t*>(a.peer_x[s_dst[k]]) + (int64_t)row * row_bytes;
                        st_v4(base + 16 * (size_t)u, q);
                        if ((u % kLanes) == 0) {
                            uint8_t* sb = static_cast<uint8_t*>(a.peer_scales[s_dst[k]]) + (int64_t)row * srb;
                            if (a.scale_bytes) sb[u / kLanes] = ue8m0_of(sc);
                            else reinterpret_cast<float*>(sb)[u / kLanes] = sc;
                        }
                    }
            }
        }
        __syncthreads();
    }
    __threadfence_system();   // the peer stores are visible to the receivers once this grid completes
}

template <int KMAX>
__global__ void __launch_bounds__(kPeerThreads) k_combine_peer(PeerCombineArgs a) {
    grid_dependency_wait();
    grid_launch_dependents();
    __shared__ int s_delta[kMaxExperts], s_a[kMaxExperts], s_b[kMaxExperts], s_warp[32];
    __shared__ const uint4* s_ptr[kMaxTopk];
    __shared__ float s_w[kMaxTopk];
    __shared__ int s_n;
    const int tid = threadIdx.x, lane = tid & 31;
    const int V = a.H / 8;
    const int Eg = a.E / a.G;
    peer_deltas(a.counts_all, a.G, a.g, a.E, a.A, s_delta, s_a, s_b, s_warp);
    for (int t = blockIdx.x; t < a.T; t += gridDim.x) {
        if (tid < 32) {
            const uint4* p = nullptr;
            float w = 0.0f;
            if (lane < a.K) {
                const int slot = a.dst_slot[(int64_t)t * a.K + lane];
                const int e = a.topk_copy[(int64_t)t * a.K + lane];
                w = a.topk_weights[(int64_t)t * a.K + lane];
                if (slot >= 0 && e >= 0) {
                    const int64_t row = (int64_t)slot + s_delta[e];
                    if (row < a.capacity)
                        p = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(a.peer_y[e / Eg]) +
                                                           row * a.H);
                    else
                        set_error(a.err, EP_ERR_CAPACITY);
                }
            }
            const unsigned m = __ballot_sync(0xffffffffu, p != nullptr);
            if (p != nullptr) {
                const int pos = __popc(m & lanemask_lt());
                s_ptr[pos] = p;
                s_w[pos] = w;
            }
            if (lane == 0) s_n = __popc(m);
        }
        __syncthreads();
        const int n = s_n;
        uint16_t* orow = a.out + (size_t)t * a.H;
        for (int v = tid; v < V; v += blockDim.x) {
            uint4 r[KMAX];
#pragma unroll
            for (int j = 0; j < KMAX; ++j)
                if (j < n) r[j] = ld_nc_v4(s_ptr[j] + v);
            float acc[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
#pragma unroll
            for (int j = 0; j < KMAX; ++j) {
                if (j < n) {
                    const float w = s_w[j];
                    const uint4 b = r[j];
                    const float y[8] = {bf16lo(b.x), bf16hi(b.x), bf16lo(b.y), bf16hi(b.y),
                                        bf16lo(b.z), bf16hi(b.z), bf16lo(b.w), bf16hi(b.w)};
#pragma unroll
                    for (int i = 0; i < 8; ++i) acc[i] = __fmaf_rn(w, y[i], acc[i]);
                }
            }
            uint32_t o[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
                o[i] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(acc[2 * i])) |
                       ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(acc[2 * i + 1])) << 16);
            st_v4(reinterpret_cast<uint4*>(orow) + v, make_uint4(o[0], o[1], o[2], o[3]));
        }
        __syncthreads();
    }
}

__global__ void k_receiver_layout(const int32_t* C, int G, int g, int E, int A, int32_t* psum, int32_t* counts) {
    __shared__ int s_v[kMaxExperts], s_warp[32];
    const int Eg = E / G;
    for (int j = threadIdx.x; j < Eg; j += blockDim.x) {
        int tot = 0;
        for (int q = 0; q < G; ++q) tot += C[(size_t)q * E + g * Eg + j];
        counts[j] = tot;
        s_v[j] = (int)(((int64_t)tot + A - 1) / A * A);
    }
    __syncthreads();
    block_exclusive_scan(s_v, Eg, s_warp);
    for (int j = threadIdx.x; j < Eg; j += blockDim.x) {
        int tot = 0;
        for (int q = 0; q < G; ++q) tot += C[(size_t)q * E + g * Eg + j];
        psum[j] = s_v[j] + (int)(((int64_t)tot + A - 1) / A * A);
    }
}

template <int QUANT, int G2>
cudaError_t run_pack_peer(const PeerPackArgs& a, cudaStream_t st) {
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_pack_peer<QUANT, G2>, kPeerThreads, 0) !=
            cudaSuccess || per_sm < 1)
        per_sm = 1;
    const int grid = max(1, min(a.T, device_sm_count() * per_sm));
    return launch_dependent(k_pack_peer<QUANT, G2>, dim3(grid), dim3(kPeerThreads), 0, st, a);
}

template <int QUANT>
cudaError_t pack_peer_q(const PeerPackArgs& a, cudaStream_t st) {
    switch (a.quant_size) {
        case 16: return run_pack_peer<QUANT, 16>(a, st);
        case 32: return run_pack_peer<QUANT, 32>(a, st);
        case 64: return run_pack_peer<QUANT, 64>(a, st);
        case 128: return run_pack_peer<QUANT, 128>(a, st);
        case 256: return run_pack_peer<QUANT, 256>(a, st);
        case 512: return run_pack_peer<QUANT, 512>(a, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_pack_peer(const PeerPackArgs& a, int quant, cudaStream_t st) {
    if (a.T == 0) return cudaSuccess;
    if (quant == EP_QUANT_NONE) return run_pack_peer<0, 16>(a, st);
    if (quant == EP_QUANT_FP8_E4M3) return pack_peer_q<kQuantFp8>(a, st);
    if (quant == EP_QUANT_INT8) return pack_peer_q<kQuantInt8>(a, st);
    return cudaErrorInvalidValue;
}

cudaError_t launch_combine_peer(const PeerCombineArgs& a, cudaStream_t st) {
    if (a.T == 0) return cudaSuccess;
    int per_sm = 0;
    auto kern = a.K <= 8 ? k_combine_peer<8> : k_combine_peer<16>;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kPeerThreads, 0) != cudaSuccess || per_sm < 1)
        per_sm = 1;
    const int grid = max(1, min(a.T, device_sm_count() * per_sm));
    return launch_dependent(kern, dim3(grid), dim3(kPeerThreads), 0, st, a);
}

cudaError_t launch_receiver_layout(const int32_t* C, int G, int g, int E, int A, int32_t* psum, int32_t* counts,
                                   cudaStream_t st) {
    k_receiver_layout<<<1, kPeerThreads, 0, st>>>(C, G, g, E, A, psum, counts);
    return cudaGetLastError();
}

}  // namespace ep
