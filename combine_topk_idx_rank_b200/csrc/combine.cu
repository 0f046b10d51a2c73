// Combine: the reverse of dispatch ("DeepEP V1 vs V2 comparative analysis",
// section 9.2).  For every token t,
//   out[t] = bf16_rne( sum_k  topk_weights[t,k] * y[dst_buffer_slot_idx[t,k]] )
// over the unmasked k in ascending order, accumulated in fp32 with fused
// multiply-adds starting from +0.
//
// Persistent grid, one token per CTA iteration.  The K row addresses are
// resolved once per token (lanes 0..K-1 load them, a ballot compacts the
// unmasked ones in k order), then every thread issues the loads of all K
// rows for its vectors before the first FMA, so each thread keeps K x VPT
// 16-byte loads in flight.
#include <cuda_bf16.h>

#include "ep_internal.cuh"

#ifndef EP_COMBINE_VPT
#define EP_COMBINE_VPT 2   // 16-byte vectors per thread per pass (x K loads in flight)
#endif
#ifndef EP_COMBINE_MIN_BLOCKS
#define EP_COMBINE_MIN_BLOCKS 3   // caps registers at 80: 3 CTAs of 224 threads per SM
#endif

namespace ep {

template <int KMAX, int VPT>
__global__ void __launch_bounds__(256, EP_COMBINE_MIN_BLOCKS) k_combine(CombineArgs a) {
    grid_dependency_wait();
    grid_launch_dependents();
    __shared__ int s_slot[kMaxTopk];
    __shared__ float s_w[kMaxTopk];
    __shared__ int s_n;
    const int tid = threadIdx.x, lane = tid & 31;
    const int V = a.H / 8;
    for (int item = blockIdx.x; item < a.n_items; item += gridDim.x) {
        const int t = token_of_item(item, a.tokens_per_rank, a.per_round, a.round);
        if (tid < 32) {
            int slot = -1;
            float w = 0.0f;
            if (lane < a.K) {
                slot = a.dst_slot[(int64_t)t * a.K + lane];
                w = a.topk_weights[(int64_t)t * a.K + lane];
                if (slot >= a.y_rows) {
                    set_error(a.err, EP_ERR_CAPACITY);
                    slot = -1;
                }
            }
            const unsigned m = __ballot_sync(0xffffffffu, slot >= 0);
            if (slot >= 0) {
                const int pos = __popc(m & lanemask_lt());
                s_slot[pos] = slot;
                s_w[pos] = w;
            }
            if (lane == 0) s_n = __popc(m);
        }
        __syncthreads();
        const int n = s_n;
        uint16_t* orow = a.out + (size_t)t * a.H;
        for (int v0 = 0; v0 < V; v0 += VPT * blockDim.x) {
            uint4 r[VPT][KMAX];
#pragma unroll
            for (int j = 0; j < KMAX; ++j) {
                if (j < n) {
                    const uint4* yr = reinterpret_cast<const uint4*>(a.y + (size_t)s_slot[j] * a.H);
#pragma unroll
                    for (int u = 0; u < VPT; ++u) {
                        const int v = v0 + u * blockDim.x + tid;
                        if (v < V) r[u][j] = ld_nc_v4(yr + v);
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < VPT; ++u) {
                const int v = v0 + u * blockDim.x + tid;
                float acc[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
#pragma unroll
                for (int j = 0; j < KMAX; ++j) {
                    if (j < n) {
                        const float w = s_w[j];
                        const uint4 q = r[u][j];
                        acc[0] = __fmaf_rn(w, bf16lo(q.x), acc[0]);
                        acc[1] = __fmaf_rn(w, bf16hi(q.x), acc[1]);
                        acc[2] = __fmaf_rn(w, bf16lo(q.y), acc[2]);
                        acc[3] = __fmaf_rn(w, bf16hi(q.y), acc[3]);
                        acc[4] = __fmaf_rn(w, bf16lo(q.z), acc[4]);
                        acc[5] = __fmaf_rn(w, bf16hi(q.z), acc[5]);
                        acc[6] = __fmaf_rn(w, bf16lo(q.w), acc[6]);
                        acc[7] = __fmaf_rn(w, bf16hi(q.w), acc[7]);
                    }
                }
                if (v < V) {
                    uint4 o;
                    o.x = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(acc[0])) |
                          ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(acc[1])) << 16);
                    o.y = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(acc[2])) |
                          ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(acc[3])) << 16);
                    o.z = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(acc[4])) |
                          ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(acc[5])) << 16);
                    o.w = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(acc[6])) |
                          ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(acc[7])) << 16);
                    st_v4(reinterpret_cast<uint4*>(orow) + v, o);
                }
            }
        }
        __syncthreads();
    }
}

namespace {

template <typename Kern>
cudaError_t run(Kern k, int threads, const CombineArgs& a, cudaStream_t st) {
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, threads, 0) != cudaSuccess || per_sm < 1)
        per_sm = 1;
    const int grid = min(a.n_items, device_sm_count() * per_sm);
    if (grid <= 0) return cudaSuccess;
    return launch_dependent(k, dim3(grid), dim3(threads), 0, st, a);
}

}  // namespace

cudaError_t launch_combine(const CombineArgs& a, cudaStream_t st) {
    const int V = a.H / 8;
    // 2 vectors per thread per pass; split the row into equal passes
    const int passes = (V + 2 * 256 - 1) / (2 * 256);
    const int threads = min(256, ((V + 2 * passes - 1) / (2 * passes) + 31) & ~31);
    if (a.K <= 2) return run(k_combine<2, 2>, threads, a, st);
    if (a.K <= 4) return run(k_combine<4, 2>, threads, a, st);
    if (a.K <= 8) return run(k_combine<8, EP_COMBINE_VPT>, threads, a, st);
    return run(k_combine<16, 1>, threads, a, st);
}

}  // namespace ep
