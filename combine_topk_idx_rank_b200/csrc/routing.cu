// Routing histogram (get_dispatch_layout) and the prefix scan that assigns
// every (token, k) entry its received row in the deterministic
// (expert, token, k) order ("DeepEP V1 vs V2 comparative analysis",
// sections 2.1, 3.1 and 8.4), with expert segments padded to
// expert_alignment.
//
// The order needs no sort: k_layout gives each entry its rank among the
// entries of its chunk of tokens that go to the same expert (in (t,k)
// order) and writes the chunk's histograms; k_scan reduces the histograms
// and turns them into the row offset of every (chunk, expert) pair;
// k_slots sets row = offset[chunk][e] + rank.  No CTA ever waits on another,
// nothing is accumulated with global atomics, and no buffer needs clearing
// before a call.
#include "ep_internal.cuh"

namespace ep {

// One CTA per chunk of C = 2^log2_chunk tokens (C*K <= 2048 entries).  Warp w
// owns a contiguous range of the chunk's entries and walks it 32 at a time;
// lanes holding the same expert find each other with __match_any_sync, so an
// entry's rank within its warp's range is the warp's running count for that
// expert plus the number of lower lanes holding the same expert.  A scan over
// the 8 per-warp histograms then makes the ranks chunk-wide.
__global__ void __launch_bounds__(kLayoutThreads) k_layout(LayoutArgs a) {
    grid_launch_dependents();
    extern __shared__ int32_t smem[];
    const int E = a.E, K = a.K, R = a.R;
    const int C = 1 << a.log2_chunk;
    int32_t* wh = smem;                               // [8][E] per-warp running counts
    int32_t* s_idx = wh + kLayoutWarps * E;           // [C*K] validated expert ids
    int32_t* s_rcnt = s_idx + C * K;                  // [R]
    int32_t* s_err = s_rcnt + R;                      // [1]
    uint8_t* s_inr = reinterpret_cast<uint8_t*>(s_err + 1);  // [C][R]

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int c = blockIdx.x;
    const int t0 = c * C;
    const int nt = min(C, a.T - t0);
    const int ne = nt * K;
    const int64_t e0 = (int64_t)t0 * K;

    for (int i = tid; i < kLayoutWarps * E; i += kLayoutThreads) wh[i] = 0;
    for (int i = tid; i < R; i += kLayoutThreads) s_rcnt[i] = 0;
    for (int i = tid; i < nt * R; i += kLayoutThreads) s_inr[i] = 0;
    if (tid == 0) *s_err = 0;
    __syncthreads();

    const int per_warp = ((C * K / kLayoutWarps) + 31) & ~31;   // a multiple of 32
    const int nb = per_warp / 32;
    int my_e[kMaxBatches], my_r[kMaxBatches];
    const unsigned lt = lanemask_lt();
#pragma unroll
    for (int b = 0; b < kMaxBatches; ++b) {
        my_e[b] = -1;
        my_r[b] = 0;
        if (b < nb) {
            const int i = warp * per_warp + b * 32 + lane;
            int e = -1;
            if (i < ne) {
                const int64_t v = a.topk_idx[e0 + i];
                if (v < -1 || v >= E) *s_err = EP_ERR_BAD_EXPERT_ID;
                else e = (int)v;
                s_idx[i] = e;
            }
            const unsigned m = __match_any_sync(0xffffffffu, e);
            int r = 0;
            if (e >= 0) r = wh[warp * E + e] + __popc(m & lt);
            __syncwarp();
            if (e >= 0 && lane == __ffs(m) - 1) wh[warp * E + e] += __popc(m);
            __syncwarp();
            my_e[b] = e;
            my_r[b] = r;
        }
    }
    __syncthreads();

    // per-expert scan over the warps -> chunk-wide base of each warp's range
    for (int e = tid; e < E; e += kLayoutThreads) {
        int run = 0;
#pragma unroll
        for (int w = 0; w < kLayoutWarps; ++w) {
            const int v = wh[w * E + e];
            wh[w * E + e] = run;
            run += v;
        }
        a.chunk_hist[(size_t)c * E + e] = run;
    }
    __syncthreads();

#pragma unroll
    for (int b = 0; b < kMaxBatches; ++b) {
        if (b < nb) {
            const int i = warp * per_warp + b * 32 + lane;
            if (i < ne) {
                const int e = my_e[b];
                if (a.rank_in_chunk) a.rank_in_chunk[e0 + i] = e >= 0 ? wh[warp * E + e] + my_r[b] : -1;
                if (a.topk_copy) a.topk_copy[e0 + i] = e;
            }
        }
    }

    // which ranks each token reaches
    for (int tl = tid; tl < nt; tl += kLayoutThreads) {
        for (int k = 0; k < K; ++k) {
            const int e = s_idx[tl * K + k];
            if (e >= 0) s_inr[tl * R + e / a.L] = 1;
        }
    }
    __syncthreads();
    for (int i = tid; i < nt * R; i += kLayoutThreads) {
        const uint8_t v = s_inr[i];
        if (v) atomicAdd(&s_rcnt[i % R], 1);
        if (a.is_token_in_rank) a.is_token_in_rank[(size_t)t0 * R + i] = v;
    }
    __syncthreads();
    for (int r = tid; r < R; r += kLayoutThreads) a.chunk_rcnt[(size_t)c * R + r] = s_rcnt[r];
    if (tid == 0) a.chunk_err[c] = *s_err;
}

// Inclusive scan of one value per thread over a block of 1024 threads.
__device__ __forceinline__ int block_inclusive_scan_1024(int v, int* s_warp) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    if (lane == 31) s_warp[warp] = v;
    __syncthreads();
    if (warp == 0) {
        int w = s_warp[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += n;
        }
        s_warp[lane] = w;
    }
    __syncthreads();
    const int add = warp > 0 ? s_warp[warp - 1] : 0;
    __syncthreads();   // s_warp may be reused by the caller
    return v + add;
}

// Column sums of a [rows, ncols] int32 table (ncols <= 1024) into out[ncols]:
// each column is split into 1024 / roundup32(ncols) contiguous row ranges,
// one thread per (column, range); the ranges are then added in shared memory.
__device__ void column_sums(const int32_t* tab, int rows, int ncols, int* s_tmp, int* out) {
    const int cw = (ncols + 31) & ~31;
    const int parts = 1024 / cw;
    const int col = threadIdx.x % cw, part = threadIdx.x / cw;
    int sum = 0;
    if (col < ncols && part < parts) {
        const int per = (rows + parts - 1) / parts;
        const int r0 = min(part * per, rows), r1 = min(r0 + per, rows);
        int r = r0;
        for (; r + 4 <= r1; r += 4) {
            const int v0 = tab[(size_t)r * ncols + col], v1 = tab[(size_t)(r + 1) * ncols + col];
            const int v2 = tab[(size_t)(r + 2) * ncols + col], v3 = tab[(size_t)(r + 3) * ncols + col];
            sum += (v0 + v1) + (v2 + v3);
        }
        for (; r < r1; ++r) sum += tab[(size_t)r * ncols + col];
    }
    s_tmp[threadIdx.x] = sum;
    __syncthreads();
    if (threadIdx.x < ncols) {
        int s = 0;
        for (int p = 0; p < parts; ++p) s += s_tmp[p * cw + threadIdx.x];
        out[threadIdx.x] = s;
    }
    __syncthreads();
}

// Grid: ceil(E/32) CTAs of 1024 threads.  Every CTA reduces the chunk
// histograms to the E expert counts and scans the aligned counts for the
// segment starts; CTA g then turns the column of chunk histograms of experts
// [32g, 32g+32) into row offsets (lane = expert, warp = one of 32 contiguous
// ranges of chunks).  CTA 0 writes the per-expert and per-rank outputs, the
// padding map and the status word.
__global__ void __launch_bounds__(1024) k_scan(ScanArgs a) {
    grid_dependency_wait();
    grid_launch_dependents();
    __shared__ int s_warp[32];
    __shared__ int s_tmp[1024];
    __shared__ int s_cnt[kMaxExperts];
    __shared__ int s_seg[kMaxExperts];
    __shared__ int s_part[32][33];
    __shared__ int s_total[2];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int E = a.E;

    column_sums(a.chunk_hist, a.nchunks, E, s_tmp, s_cnt);
    const int cnt = tid < E ? s_cnt[tid] : 0;
    const int aligned = (int)(((int64_t)cnt + a.A - 1) / a.A * a.A);
    const int incl = block_inclusive_scan_1024(aligned, s_warp);
    const int seg = incl - aligned;
    if (tid < E) s_seg[tid] = seg;
    const int pad = aligned - cnt;
    const int pad_incl = block_inclusive_scan_1024(pad, s_warp);

    if (blockIdx.x == 0) {
        if (tid == E - 1) {
            s_total[0] = incl;
            s_total[1] = pad_incl;
        }
        if (tid < E) {
            if (a.psum) a.psum[tid] = incl;
            if (a.num_recv) a.num_recv[tid] = cnt;
            if (a.num_tokens_per_expert) a.num_tokens_per_expert[tid] = cnt;
            if (a.cumulative) a.cumulative[tid] += cnt;
            if (a.pad_base) a.pad_base[tid] = pad_incl - pad;
            if (a.pad_start) a.pad_start[tid] = seg + cnt;
        }
        // per-rank token counts and the layout's error flags
        column_sums(a.chunk_rcnt, a.nchunks, a.R, s_tmp, s_cnt);
        if (tid < a.R && a.num_tokens_per_rank) a.num_tokens_per_rank[tid] = s_cnt[tid];
        column_sums(a.chunk_err, a.nchunks, 1, s_tmp, s_cnt);
        if (tid == 0) {
            const int rows = s_total[0], pads = s_total[1];
            if (a.pad_base) a.pad_base[E] = pads;
            a.hdr[1] = rows;
            a.hdr[2] = pads;
            int status = s_cnt[0] ? EP_ERR_BAD_EXPERT_ID : 0;
            if (status == 0 && a.check_capacity && (int64_t)rows > a.capacity) status = EP_ERR_CAPACITY;
            *a.err_out = status;
        }
    }
    if (a.chunk_off == nullptr) return;
    __syncthreads();

    const int e = blockIdx.x * 32 + lane;
    const int per = (a.nchunks + 31) / 32;
    const int c0 = min(warp * per, a.nchunks), c1 = min(c0 + per, a.nchunks);
    int sum = 0;
    if (e < E)
        for (int c = c0; c < c1; ++c) sum += a.chunk_hist[(size_t)c * E + e];
    s_part[warp][lane] = sum;
    __syncthreads();
    {   // warp w scans column w of s_part across the 32 chunk ranges
        const int v = s_part[lane][warp];
        int s = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += n;
        }
        __syncthreads();
        s_part[lane][warp] = s - v;
    }
    __syncthreads();
    if (e < E) {
        int run = s_seg[e] + s_part[warp][lane];
        for (int c = c0; c < c1; ++c) {
            const int h = a.chunk_hist[(size_t)c * E + e];
            a.chunk_off[(size_t)c * E + e] = run;
            run += h;
        }
    }
}

// Turns every entry's rank inside its chunk into its received row,
// row = offset[chunk][e] + rank, writes dst_buffer_slot_idx and the per-row
// metadata of the receiving side: recv_src_metadata = (t, k), and for
// recv_topk_idx / recv_topk_weights the token's top-k entries whose experts
// live on the receiving rank (local ids), -1 / 0 elsewhere.  The threads past
// the T*K entries fill the padding rows' metadata: (-1, -1), -1, 0, scale 0.
// KT = K for the vectorised forms (K in {4, 8, 16}); KT = 0 for any K.
template <int KT>
__global__ void __launch_bounds__(256) k_slots(SlotsArgs a) {
    grid_dependency_wait();
    grid_launch_dependents();
    __shared__ int s_pad_base[kMaxExperts + 1];
    const int K = KT > 0 ? KT : a.K;
    const int E = a.E;
    const int64_t n_ent = (int64_t)a.T * K;
    const int n_pad = a.hdr[2];
    if (a.max_pad > 0)
        for (int i = threadIdx.x; i <= E; i += blockDim.x) s_pad_base[i] = a.pad_base[i];
    __syncthreads();
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_ent + a.max_pad; i += stride) {
        if (i < n_ent) {
            const int t = (int)(i / K), k = (int)(i - (int64_t)t * K);
            const int64_t v = a.topk_idx[i];
            const int e = (v >= 0 && v < E) ? (int)v : -1;
            int slot = -1;
            if (e >= 0) {
                const int rank = a.dst_slot[i];
                const int64_t row = (int64_t)a.chunk_off[(size_t)(t >> a.log2_chunk) * E + e] + rank;
                slot = (rank >= 0 && row < a.capacity) ? (int)row : -1;
            }
            a.dst_slot[i] = slot;
            if (slot < 0) continue;
            reinterpret_cast<int2*>(a.recv_meta)[slot] = make_int2(t, k);
            const int rdst = e / a.L;
            const int64_t* row_ids = a.topk_idx + (int64_t)t * K;
            const float* row_w = a.topk_weights + (int64_t)t * K;
            if constexpr (KT > 0) {
                // the token's K ids and weights as 16-byte loads, the row as 16-byte stores
                int ids[KT];
                float ws[KT];
#pragma unroll
                for (int j = 0; j < KT; j += 2) {
                    const longlong2 p = __ldg(reinterpret_cast<const longlong2*>(row_ids) + j / 2);
                    ids[j] = (int)p.x;
                    ids[j + 1] = (int)p.y;
                    const bool ok0 = p.x >= 0 && p.x < E, ok1 = p.y >= 0 && p.y < E;
                    if (!ok0) ids[j] = -1;
                    if (!ok1) ids[j + 1] = -1;
                }
#pragma unroll
                for (int j = 0; j < KT; j += 4) {
                    const float4 q = __ldg(reinterpret_cast<const float4*>(row_w) + j / 4);
                    ws[j] = q.x; ws[j + 1] = q.y; ws[j + 2] = q.z; ws[j + 3] = q.w;
                }
                int4* ri = reinterpret_cast<int4*>(a.recv_topk_idx + (int64_t)slot * KT);
                float4* rw = reinterpret_cast<float4*>(a.recv_topk_weights + (int64_t)slot * KT);
#pragma unroll
                for (int j = 0; j < KT; j += 4) {
                    int o[4];
                    float w[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int ej = ids[j + u];
                        const bool here = ej >= 0 && ej / a.L == rdst;
                        o[u] = here ? ej - rdst * a.L : -1;
                        w[u] = here ? ws[j + u] : 0.0f;
                    }
                    ri[j / 4] = make_int4(o[0], o[1], o[2], o[3]);
                    rw[j / 4] = make_float4(w[0], w[1], w[2], w[3]);
                }
            } else {
                int32_t* ri = a.recv_topk_idx + (int64_t)slot * K;
                float* rw = a.recv_topk_weights + (int64_t)slot * K;
                for (int j = 0; j < K; ++j) {
                    const int64_t ej = __ldg(row_ids + j);
                    const bool here = ej >= 0 && ej < E && (int)ej / a.L == rdst;
                    ri[j] = here ? (int)ej - rdst * a.L : -1;
                    rw[j] = here ? __ldg(row_w + j) : 0.0f;
                }
            }
        } else {
            const int p = (int)(i - n_ent);
            if (p < n_pad) {
                int lo = 0, hi = E;   // last expert with pad_base <= p
                while (hi - lo > 1) {
                    const int mid = (lo + hi) >> 1;
                    if (s_pad_base[mid] <= p) lo = mid; else hi = mid;
                }
                const int64_t row = (int64_t)a.pad_start[lo] + (p - s_pad_base[lo]);
                if (row < a.capacity) {
                    reinterpret_cast<int2*>(a.recv_meta)[row] = make_int2(-1, -1);
                    for (int j = 0; j < K; ++j) {
                        a.recv_topk_idx[row * K + j] = -1;
                        a.recv_topk_weights[row * K + j] = 0.0f;
                    }
                    for (int j = 0; j < a.nscales; ++j) a.recv_scales[row * a.nscales + j] = 0.0f;
                }
            }
        }
    }
}

cudaError_t launch_layout(const LayoutArgs& a, int nchunks, cudaStream_t st) {
    const int C = 1 << a.log2_chunk;
    const size_t smem = sizeof(int32_t) * (kLayoutWarps * a.E + C * a.K + a.R + 1) + (size_t)C * a.R;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(k_layout, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    k_layout<<<nchunks, kLayoutThreads, smem, st>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_scan(const ScanArgs& a, cudaStream_t st) {
    const int grid = a.chunk_off ? (a.E + 31) / 32 : 1;
    return launch_dependent(k_scan, dim3(grid), dim3(1024), 0, st, a);
}

cudaError_t launch_slots(const SlotsArgs& a, cudaStream_t st) {
    const int64_t work = (int64_t)a.T * a.K + a.max_pad;
    if (work <= 0) return cudaSuccess;
    const int64_t blocks = (work + 255) / 256;
    const int64_t cap = (int64_t)device_sm_count() * 8;
    const int grid = (int)(blocks < cap ? blocks : cap);
    switch (a.vector_ok ? a.K : 0) {
        case 4: return launch_dependent(k_slots<4>, dim3(grid), dim3(256), 0, st, a);
        case 8: return launch_dependent(k_slots<8>, dim3(grid), dim3(256), 0, st, a);
        case 16: return launch_dependent(k_slots<16>, dim3(grid), dim3(256), 0, st, a);
        default: return launch_dependent(k_slots<0>, dim3(grid), dim3(256), 0, st, a);
    }
}

}  // namespace ep
