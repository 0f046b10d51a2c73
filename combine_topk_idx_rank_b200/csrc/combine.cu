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
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "ep_internal.cuh"

#ifndef EP_COMBINE_VPT
#define EP_COMBINE_VPT 2   // 16-byte vectors per thread per pass (x K loads in flight)
#endif
#ifndef EP_COMBINE_MIN_BLOCKS
#define EP_COMBINE_MIN_BLOCKS 3   // caps registers at 80: 3 CTAs of 224 threads per SM
#endif

namespace ep {

// Packed fp32 pairs (sm_100): each half is the same correctly rounded
// operation as its scalar form, so results are bit-identical.
//   (r0, r1) = (a0 * b, a1 * b)          (d0, d1) = (w * a0 + d0, w * a1 + d1)
__device__ __forceinline__ void mul2_rn(float& r0, float& r1, float a0, float a1, float b) {
    uint64_t x, y, r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(x) : "f"(a0), "f"(a1));
    asm("mov.b64 %0, {%1, %1};" : "=l"(y) : "f"(b));
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(x), "l"(y));
    asm("mov.b64 {%0, %1}, %2;" : "=f"(r0), "=f"(r1) : "l"(r));
}
__device__ __forceinline__ void fma2_rn(float& d0, float& d1, float w, float a0, float a1) {
    uint64_t ww, x, d;
    asm("mov.b64 %0, {%1, %1};" : "=l"(ww) : "f"(w));
    asm("mov.b64 %0, {%1, %2};" : "=l"(x) : "f"(a0), "f"(a1));
    asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(d0), "f"(d1));
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(ww), "l"(x), "l"(d));
    asm("mov.b64 {%0, %1}, %2;" : "=f"(d0), "=f"(d1) : "l"(d));
}

// Eight codes -> decode(code) * scale (fp32 product).  YQ 1 = FP8 e4m3
// (decoded exactly through fp16), 2 = int8.
template <int YQ>
__device__ __forceinline__ void dequant8(uint2 c, float s, float (&v)[8]) {
    const uint32_t w[2] = {c.x, c.y};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        if constexpr (YQ == 1) {
            const __half2_raw lo = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w[h] & 0xffffu), __NV_E4M3);
            const __half2_raw hi = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w[h] >> 16), __NV_E4M3);
            v[4 * h + 0] = __half2float(__ushort_as_half(lo.x));
            v[4 * h + 1] = __half2float(__ushort_as_half(lo.y));
            v[4 * h + 2] = __half2float(__ushort_as_half(hi.x));
            v[4 * h + 3] = __half2float(__ushort_as_half(hi.y));
        } else {
            v[4 * h + 0] = (float)(int8_t)(w[h] & 0xff);
            v[4 * h + 1] = (float)(int8_t)((w[h] >> 8) & 0xff);
            v[4 * h + 2] = (float)(int8_t)((w[h] >> 16) & 0xff);
            v[4 * h + 3] = (float)(int8_t)(w[h] >> 24);
        }
    }
#pragma unroll
    for (int i = 0; i < 8; i += 2) mul2_rn(v[i], v[i + 1], v[i], v[i + 1], s);
}

template <int KMAX, int VPT>
__global__ void __launch_bounds__(256, EP_COMBINE_MIN_BLOCKS) k_combine(CombineArgs a) {
    grid_dependency_wait();
    grid_launch_dependents();
    __shared__ int s_slot[kMaxTopk];
    __shared__ float s_w[kMaxTopk];
    __shared__ int s_n;
    const int tid = threadIdx.x, lane = tid & 31;
    const int V = a.H / 8;                              // slots of 8 channels per row
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
            // every load of the pass is issued before the first FMA
            uint4 r[VPT][KMAX];
#pragma unroll
            for (int j = 0; j < KMAX; ++j) {
                if (j < n) {
                    const uint16_t* yr = reinterpret_cast<const uint16_t*>(a.y) + (size_t)s_slot[j] * a.H;
#pragma unroll
                    for (int u = 0; u < VPT; ++u) {
                        const int v = v0 + u * blockDim.x + tid;
                        if (v < V) r[u][j] = ld_nc_v4(reinterpret_cast<const uint4*>(yr) + v);
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < VPT; ++u) {
                const int v = v0 + u * blockDim.x + tid;
                float acc[8];
                if (a.shared != nullptr && v < V) {
                    const uint4 b = ld_nc_v4(reinterpret_cast<const uint4*>(a.shared + (size_t)t * a.H) + v);
                    acc[0] = bf16lo(b.x); acc[1] = bf16hi(b.x); acc[2] = bf16lo(b.y); acc[3] = bf16hi(b.y);
                    acc[4] = bf16lo(b.z); acc[5] = bf16hi(b.z); acc[6] = bf16lo(b.w); acc[7] = bf16hi(b.w);
                } else {
#pragma unroll
                    for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
                }
#pragma unroll
                for (int j = 0; j < KMAX; ++j) {
                    if (j < n) {
                        const float w = s_w[j];
                        float y[8];
                        const uint4 b = r[u][j];
                        y[0] = bf16lo(b.x); y[1] = bf16hi(b.x); y[2] = bf16lo(b.y); y[3] = bf16hi(b.y);
                        y[4] = bf16lo(b.z); y[5] = bf16hi(b.z); y[6] = bf16lo(b.w); y[7] = bf16hi(b.w);
#pragma unroll
                        for (int i = 0; i < 8; i += 2) fma2_rn(acc[i], acc[i + 1], w, y[i], y[i + 1]);
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

// Combine of quantised expert outputs: a thread slot covers 16 channels, so
// each (row, slot) is one 16-byte load of codes and one scale load; all K
// loads of a slot are issued before the first FMA.
template <int KMAX, int YQ>
__global__ void __launch_bounds__(256, EP_COMBINE_MIN_BLOCKS) k_combine_q(CombineArgs a) {
    grid_dependency_wait();
    grid_launch_dependents();
    __shared__ int s_slot[kMaxTopk];
    __shared__ float s_w[kMaxTopk];
    __shared__ int s_n;
    const int tid = threadIdx.x, lane = tid & 31;
    const int V = a.H / 16;                             // slots of 16 channels per row
    const int nscales = a.H / a.quant_size;
    const uint8_t* ybase = reinterpret_cast<const uint8_t*>(a.y);
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
        for (int v = tid; v < V; v += blockDim.x) {
            uint4 q[KMAX];
            float sc[KMAX];
            const int g = (v * 16) / a.quant_size;
#pragma unroll
            for (int j = 0; j < KMAX; ++j) {
                if (j < n) {
                    q[j] = ld_nc_v4(ybase + (size_t)s_slot[j] * a.H + 16 * (size_t)v);
                    sc[j] = __ldg(a.y_scales + (size_t)s_slot[j] * nscales + g);
                }
            }
            float acc[16];
            if (a.shared != nullptr) {
                const uint4* sh = reinterpret_cast<const uint4*>(a.shared + (size_t)t * a.H + 16 * (size_t)v);
                const uint4 b0 = ld_nc_v4(sh), b1 = ld_nc_v4(sh + 1);
                const uint32_t w[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    acc[2 * i] = bf16lo(w[i]);
                    acc[2 * i + 1] = bf16hi(w[i]);
                }
            } else {
#pragma unroll
                for (int i = 0; i < 16; ++i) acc[i] = 0.0f;
            }
#pragma unroll
            for (int j = 0; j < KMAX; ++j) {
                if (j < n) {
                    const float w = s_w[j];
                    float lo[8], hi[8];
                    dequant8<YQ>(make_uint2(q[j].x, q[j].y), sc[j], lo);
                    dequant8<YQ>(make_uint2(q[j].z, q[j].w), sc[j], hi);
#pragma unroll
                    for (int i = 0; i < 8; i += 2) {
                        fma2_rn(acc[i], acc[i + 1], w, lo[i], lo[i + 1]);
                        fma2_rn(acc[8 + i], acc[8 + i + 1], w, hi[i], hi[i + 1]);
                    }
                }
            }
            uint32_t o[8];
#pragma unroll
            for (int i = 0; i < 8; ++i)
                o[i] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(acc[2 * i])) |
                       ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(acc[2 * i + 1])) << 16);
            uint4* dst = reinterpret_cast<uint4*>(orow + 16 * (size_t)v);
            st_v4(dst, make_uint4(o[0], o[1], o[2], o[3]));
            st_v4(dst + 1, make_uint4(o[4], o[5], o[6], o[7]));
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
    if (a.y_quant != EP_QUANT_NONE) {
        // one 16-channel slot per thread per pass; split the row into equal passes
        const int V16 = a.H / 16;
        const int p16 = (V16 + 255) / 256;
        const int th16 = min(256, ((V16 + p16 - 1) / p16 + 31) & ~31);
        if (a.y_quant == EP_QUANT_FP8_E4M3)
            return a.K <= 8 ? run(k_combine_q<8, 1>, th16, a, st) : run(k_combine_q<16, 1>, th16, a, st);
        return a.K <= 8 ? run(k_combine_q<8, 2>, th16, a, st) : run(k_combine_q<16, 2>, th16, a, st);
    }
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
