// Padding rows of a receive layout whose real rows were written by another
// path (the multi-GPU exchange): expert alignment ("DeepEP V1 vs V2
// comparative analysis", section 3.1) pads each expert's segment to a
// multiple of expert_alignment, and the padding rows hold zero bytes, scale 0,
// recv_topk_idx -1, weight 0 and metadata (-1, -1), as ep_dispatch writes
// them.
//
// Persistent grid: every CTA numbers the padding rows over the segments from
// the psum / counts arrays (a block scan), then takes rows p = b, b + grid, ...
// and finds each row's segment by binary search.  Rows are zeroed with 16-byte
// stores by all threads of the CTA.
#include "ep_internal.cuh"

namespace ep {

namespace {

constexpr int kPadThreads = 256;

__global__ void __launch_bounds__(kPadThreads) k_padding(PadArgs a) {
    __shared__ int s_base[kMaxExperts + 1];   // padding rows before segment e
    __shared__ int s_start[kMaxExperts];      // first padding row of segment e
    __shared__ int s_warp[kPadThreads / 32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int n = a.n;
    const int per = (n + kPadThreads - 1) / kPadThreads;
    const int e0 = min(tid * per, n), e1 = min(e0 + per, n);
    int sum = 0;
    for (int e = e0; e < e1; ++e) sum += (a.psum[e] - (e ? a.psum[e - 1] : 0)) - a.cnt[e];
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int w = lane < kPadThreads / 32 ? s_warp[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += v;
        }
        if (lane < kPadThreads / 32) s_warp[lane] = w;
    }
    __syncthreads();
    int run = incl - sum + (warp > 0 ? s_warp[warp - 1] : 0);
    for (int e = e0; e < e1; ++e) {
        const int lo = e ? a.psum[e - 1] : 0;
        s_base[e] = run;
        s_start[e] = lo + a.cnt[e];
        run += (a.psum[e] - lo) - a.cnt[e];
    }
    const int total = s_warp[kPadThreads / 32 - 1];
    __syncthreads();

    for (int p = blockIdx.x; p < total; p += gridDim.x) {
        int lo = 0, hi = n;   // the last segment whose base <= p
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (s_base[mid] <= p) lo = mid; else hi = mid;
        }
        const int64_t row = (int64_t)s_start[lo] + (p - s_base[lo]);
        if (row < 0 || row >= a.capacity) continue;
        uint4* dst = reinterpret_cast<uint4*>(a.recv_x + row * a.row_bytes);
        for (int64_t v = tid; v < a.row_bytes / 16; v += kPadThreads) st_v4(dst + v, make_uint4(0, 0, 0, 0));
        if (a.recv_scales)
            for (int64_t b = tid; b < a.scale_row_bytes; b += kPadThreads) a.recv_scales[row * a.scale_row_bytes + b] = 0;
        if (tid < a.K) {
            if (a.recv_topk_idx) a.recv_topk_idx[row * a.K + tid] = -1;
            if (a.recv_topk_weights) a.recv_topk_weights[row * a.K + tid] = 0.0f;
        }
        if (tid == 0 && a.recv_meta) reinterpret_cast<int2*>(a.recv_meta)[row] = make_int2(-1, -1);
    }
}

}  // namespace

cudaError_t launch_padding(const PadArgs& a, cudaStream_t st) {
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_padding, kPadThreads, 0) != cudaSuccess || per_sm < 1)
        per_sm = 1;
    k_padding<<<device_sm_count() * per_sm, kPadThreads, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace ep
