// Routing: the histogram of get_dispatch_layout and the assignment of every
// (token, k) entry to its received row in the deterministic (expert, token, k)
// order ("DeepEP V1 vs V2 comparative analysis", sections 2.1, 3.1 and 8.4),
// expert segments padded to expert_alignment.
//
// One cooperative kernel, k_route, in three phases separated by grid-wide
// barriers (all CTAs are co-resident by construction of a cooperative
// launch; every wait is bounded and reports EP_ERR_TIMEOUT):
//   1. per chunk of 2^log2_chunk tokens (one CTA per chunk): validate ids,
//      rank every entry among the chunk's entries of the same expert
//      (warp-aggregated with __match_any_sync, then across the 8 warps),
//      write the chunk's expert and rank histograms and is_token_in_rank;
//   2. one warp per column of the [chunk, expert] histogram: exclusive prefix
//      over the chunks (in place) and the column total = expert count;
//      likewise the per-rank and error columns.  When the tables fit in
//      shared memory (a.fold) this phase and its barrier are skipped: every
//      CTA copies the whole [chunk, expert] table in with cp.async and sums
//      the columns it needs (expert totals, its chunk's prefix) itself;
//   3. every CTA scans the aligned expert counts for the segment starts;
//      row = segment start + chunk prefix + rank inside the chunk; write
//      dst_buffer_slot_idx, recv_src_metadata, recv_topk_idx/weights and the
//      padding rows' metadata (their bytes and scales are zeroed by the pack
//      kernel).  CTA 0 writes the per-expert / per-rank
//      outputs and the status word.
// No sort, no global atomics except the barrier counter.
#include "ep_internal.cuh"

#ifndef EP_ROUTE_FOLD
#define EP_ROUTE_FOLD 1   // 0: always the three-phase form
#endif

namespace ep {

namespace {

constexpr unsigned long long kBarrierTimeoutNs = 2000000000ull;   // a grid barrier gives up after 2 s
constexpr size_t kRouteFoldSmem = 200 * 1024;   // shared memory the folded routing kernel may take

__device__ __forceinline__ unsigned long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// 16-byte asynchronous copy global -> shared (L2 only), and the wait for all
// of this thread's copies.
__device__ __forceinline__ void cp_async16(void* sdst, const void* gsrc) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                     static_cast<uint32_t>(__cvta_generic_to_shared(sdst))),
                 "l"(gsrc)
                 : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Grid-wide barrier over a counter that was zero at launch; `target` is
// gridDim.x times the barrier's ordinal.  False if the wait gave up (after
// kBarrierTimeoutNs of the global timer).  Thread 0 arrives with a release
// reduction (after the block barrier it covers the whole CTA's writes) and
// polls with acquire loads; the closing block barrier hands the acquire on.
__device__ bool grid_barrier(unsigned* counter, unsigned target, int* s_flag) {
    __syncthreads();
    if (threadIdx.x == 0) {
        asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(counter) : "memory");
        int ok = 1;
        const unsigned long long t0 = global_ns();
        for (;;) {
            unsigned v;
            asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(counter) : "memory");
            if (v >= target) break;
            if (global_ns() - t0 > kBarrierTimeoutNs) {
                ok = 0;
                break;
            }
            __nanosleep(32);
        }
        *s_flag = ok;
    }
    __syncthreads();
    return *s_flag != 0;
}

// Rank of expert e (e / L): a shift when L is a power of two (sh >= 0).
__device__ __forceinline__ int rank_of(int e, int L, int sh) { return sh >= 0 ? e >> sh : e / L; }

// Inclusive scan of one value per thread over the block (blockDim.x = 256).
__device__ __forceinline__ int block_inclusive_scan(int v, int* s_warp) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    if (lane == 31) s_warp[warp] = v;
    __syncthreads();
    if (warp == 0) {
        int w = lane < kRouteWarps ? s_warp[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += n;
        }
        if (lane < kRouteWarps) s_warp[lane] = w;
    }
    __syncthreads();
    const int add = warp > 0 ? s_warp[warp - 1] : 0;
    __syncthreads();
    return v + add;
}

// Exclusive scan over E values held in smem (E <= 1024, 4 per thread):
// out[e] = sum of in[0..e-1]; returns the total.
__device__ int block_exclusive_scan_E(const int* in, int* out, int E, int* s_warp) {
    const int base = threadIdx.x * 4;
    int v[4], sum = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        v[j] = base + j < E ? in[base + j] : 0;
        sum += v[j];
    }
    const int incl = block_inclusive_scan(sum, s_warp);
    int run = incl - sum;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        if (base + j < E) out[base + j] = run;
        run += v[j];
    }
    __shared__ int s_tot;
    if (threadIdx.x == kRouteThreads - 1) s_tot = incl;
    __syncthreads();
    const int tot = s_tot;
    __syncthreads();
    return tot;
}

// Shared memory of the routing kernel without the folded tables, and the
// (16-byte aligned) offset of the tables after it.
__host__ __device__ size_t route_smem_bytes(int E, int K, int R, int log2_chunk) {
    const int C = 1 << log2_chunk;
    return sizeof(int32_t) * ((size_t)kRouteWarps * E + 3 * (size_t)C * K + R + 3 * (size_t)E + 1 + 40) +
           (size_t)C * R;
}
__host__ __device__ size_t route_table_offset(int E, int K, int R, int log2_chunk) {
    return (route_smem_bytes(E, K, R, log2_chunk) + 15) & ~size_t(15);
}
// Folded tables: [nchunks][E] + [nchunks][R] int32, then [2][threads] int4
// partial column sums.
size_t route_fold_bytes(const RouteArgs& a) {
    return sizeof(int32_t) * (size_t)a.nchunks * (a.E + a.R) + 2 * sizeof(int4) * kRouteThreads;
}

}  // namespace

template <int KT>
__global__ void __launch_bounds__(kRouteThreads) k_route(RouteArgs a) {
    grid_launch_dependents();   // the pack kernel may be scheduled; it waits for our results
    extern __shared__ int32_t smem[];
    const int E = a.E, K = KT > 0 ? KT : a.K, R = a.R, L = a.L;
    const int C = 1 << a.log2_chunk;
    int32_t* wh = smem;                               // [8][E] per-warp running counts
    int32_t* s_idx = wh + kRouteWarps * E;            // [C*K] validated expert ids
    int32_t* s_rank = s_idx + C * K;                  // [C*K] rank inside the chunk
    float* s_w = reinterpret_cast<float*>(s_rank + C * K);   // [C*K] top-k weights
    int32_t* s_rcnt = reinterpret_cast<int32_t*>(s_w + C * K);   // [R]
    int32_t* s_seg = s_rcnt + R;                      // [E] segment starts
    int32_t* s_al = s_seg + E;                        // [E] aligned counts, then padding prefix
    int32_t* s_pad = s_al + E;                        // [E+1] padding prefix
    int32_t* s_misc = s_pad + E + 1;                  // [40]: warp sums, flags
    uint8_t* s_inr = reinterpret_cast<uint8_t*>(s_misc + 40);   // [C][R]
    // folded routing: [nchunks][E] expert histogram, then [nchunks][R] rank counts
    int32_t* s_tab = reinterpret_cast<int32_t*>(reinterpret_cast<char*>(smem) +
                                                 route_table_offset(E, a.K, R, a.log2_chunk));
    int32_t* s_rtab = s_tab + (size_t)a.nchunks * E;
    int32_t* s_fpre = wh + E;  // [E] folded: this chunk's prefix (wh[0, E) holds the expert counts)
    int* s_warp = s_misc;
    int* s_flag = s_misc + 32;
    int* s_err = s_misc + 33;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int G = gridDim.x;
    const int shL = (L & (L - 1)) == 0 ? __ffs(L) - 1 : -1;
    const unsigned lt = lanemask_lt();
    const int per_warp = ((C * K / kRouteWarps) + 31) & ~31;   // entries per warp, a multiple of 32
    const int nb = per_warp / 32;
    // with one chunk per CTA its ids, weights and ranks stay in shared memory
    // from phase 1 to phase 3; otherwise phase 3 reloads them
    const bool resident = a.nchunks <= G;

    // ---------------------------------------------------------------- phase 1
    // the status word of this call starts clear; every later error is first-wins
    if (blockIdx.x == 0 && tid == 0) *a.err_out = 0;
    for (int c = blockIdx.x; c < a.nchunks; c += G) {
        // chunks never straddle a source rank: chunk c is piece c % cpr of rank c / cpr
        const int t0 = (c / a.chunks_per_rank) * a.tokens_per_rank + (c % a.chunks_per_rank) * C;
        const int nt = min(C, a.tokens_per_rank - (c % a.chunks_per_rank) * C);
        const int ne = nt * K;
        const int64_t e0 = (int64_t)t0 * K;
        // this warp's entries (and, for dispatch, the chunk's weights): every
        // load is issued first, the shared tables are cleared while they fly
        int64_t ld[kMaxBatches];
#pragma unroll
        for (int b = 0; b < kMaxBatches; ++b) {
            const int i = warp * per_warp + b * 32 + lane;
            ld[b] = (b < nb && i < ne) ? a.topk_idx[e0 + i] : -1;
        }
        constexpr int kW = kMaxChunkEntries / kRouteThreads;   // weights per thread
        float wv[kW];
        if (a.assign) {
#pragma unroll
            for (int j = 0; j < kW; ++j) {
                const int i = tid + j * kRouteThreads;
                wv[j] = i < ne ? a.topk_weights[e0 + i] : 0.0f;
            }
        }
        for (int i = tid; i < kRouteWarps * E; i += kRouteThreads) wh[i] = 0;
        for (int i = tid; i < R; i += kRouteThreads) s_rcnt[i] = 0;
        for (int i = tid; i < nt * R; i += kRouteThreads) s_inr[i] = 0;
        if (tid == 0) *s_err = 0;
        if (a.assign) {
#pragma unroll
            for (int j = 0; j < kW; ++j) {
                const int i = tid + j * kRouteThreads;
                if (i < ne) s_w[i] = wv[j];
            }
        }
        __syncthreads();
        int my_e[kMaxBatches], my_r[kMaxBatches];
#pragma unroll
        for (int b = 0; b < kMaxBatches; ++b) {
            my_e[b] = -1;
            my_r[b] = 0;
            if (b < nb) {
                const int i = warp * per_warp + b * 32 + lane;
                int e = -1;
                if (i < ne) {
                    const int64_t v = ld[b];
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
        for (int e = tid; e < E; e += kRouteThreads) {
            int run = 0;
#pragma unroll
            for (int w = 0; w < kRouteWarps; ++w) {
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
                    const int rank = e >= 0 ? wh[warp * E + e] + my_r[b] : -1;
                    s_rank[i] = rank;
                    if (a.dst_slot && !resident) a.dst_slot[e0 + i] = rank;
                    if (a.topk_copy) a.topk_copy[e0 + i] = e;
                }
            }
        }
        for (int tl = tid; tl < nt; tl += kRouteThreads) {
            for (int k = 0; k < K; ++k) {
                const int e = s_idx[tl * K + k];
                if (e >= 0) s_inr[tl * R + rank_of(e, L, shL)] = 1;
            }
        }
        __syncthreads();
        for (int i = tid; i < nt * R; i += kRouteThreads) {
            const uint8_t v = s_inr[i];
            if (v) atomicAdd(&s_rcnt[i % R], 1);
            if (a.is_token_in_rank) a.is_token_in_rank[(size_t)t0 * R + i] = v;
        }
        __syncthreads();
        for (int r = tid; r < R; r += kRouteThreads) a.chunk_rcnt[(size_t)c * R + r] = s_rcnt[r];
        if (tid == 0) a.chunk_err[c] = *s_err;
        __syncthreads();
    }
    if (!grid_barrier(a.barrier, (unsigned)G + a.stall, s_flag)) {
        if (tid == 0) set_error(a.err_out, EP_ERR_TIMEOUT);
        return;
    }

    int* s_cnt = wh;   // [E] expert counts (the per-warp table is free now)
    if (a.fold) {
        // the tables into shared memory (CTA 0 also takes the rank counts), then
        // the expert totals; chunk prefixes are summed per chunk below
        const int n16 = a.nchunks * E / 4;
        for (int i = tid; i < n16; i += kRouteThreads) cp_async16(s_tab + 4 * i, a.chunk_hist + 4 * i);
        if (blockIdx.x == 0) {
            const int r16 = a.nchunks * R / 4;
            for (int i = tid; i < r16; i += kRouteThreads) cp_async16(s_rtab + 4 * i, a.chunk_rcnt + 4 * i);
        }
        cp_async_wait_all();
        __syncthreads();
        // one pass over the table: thread (q, g) sums columns 4q..4q+3 over
        // rows g, g + RG, ... into the total and into this CTA's chunk prefix
        // (rows [cfirst, c): from the source rank's first chunk in the
        // low-latency layout); the RG partial sums of a column meet in s_part
        const int c = blockIdx.x;   // folded: one chunk per CTA
        const int cfirst = a.ll_M && a.chunks_per_rank > 0 ? (c / a.chunks_per_rank) * a.chunks_per_rank : 0;
        const int QE = E / 4, RG = kRouteThreads / QE;
        const int q = tid % QE, g = tid / QE;
        int4 tot = make_int4(0, 0, 0, 0), pre = make_int4(0, 0, 0, 0);
        if (g < RG) {
            const int4* t4 = reinterpret_cast<const int4*>(s_tab);
            for (int r = g; r < a.nchunks; r += RG) {
                const int4 v = t4[(size_t)r * QE + q];
                tot.x += v.x; tot.y += v.y; tot.z += v.z; tot.w += v.w;
                if (r >= cfirst && r < c) { pre.x += v.x; pre.y += v.y; pre.z += v.z; pre.w += v.w; }
            }
        }
        int4* s_part = reinterpret_cast<int4*>(s_rtab + (size_t)a.nchunks * R);   // [2][kRouteThreads]
        s_part[tid] = tot;
        s_part[kRouteThreads + tid] = pre;
        __syncthreads();
        const int* pt = reinterpret_cast<const int*>(s_part);
        for (int e = tid; e < E; e += kRouteThreads) {
            int cnt = 0, p = 0;
            for (int j = 0; j < RG; ++j) {
                cnt += pt[j * E + e];
                p += pt[4 * kRouteThreads + j * E + e];
            }
            s_cnt[e] = cnt;
            s_al[e] = (int)(((int64_t)cnt + a.A - 1) / a.A * a.A);
            s_fpre[e] = p;
        }
    } else {
        // ---------------------------------------------------------------- phase 2
        // column col: [0,E) experts (prefix written in place), [E,E+R) ranks, E+R errors
        {
            const int ncol = E + R + 1;
            for (int col = blockIdx.x * kRouteWarps + warp; col < ncol; col += G * kRouteWarps) {
                int32_t* tab;
                int stride, idx;
                if (col < E) { tab = a.chunk_hist; stride = E; idx = col; }
                else if (col < E + R) { tab = a.chunk_rcnt; stride = R; idx = col - E; }
                else { tab = a.chunk_err; stride = 1; idx = 0; }
                int carry = 0;
                for (int c0 = 0; c0 < a.nchunks; c0 += 32 * 8) {
                    int v[8];
#pragma unroll
                    for (int s = 0; s < 8; ++s) {
                        const int c = c0 + s * 32 + lane;
                        v[s] = c < a.nchunks ? __ldcg(tab + (size_t)c * stride + idx) : 0;
                    }
#pragma unroll
                    for (int s = 0; s < 8; ++s) {
                        int incl = v[s];
#pragma unroll
                        for (int o = 1; o < 32; o <<= 1) {
                            const int n = __shfl_up_sync(0xffffffffu, incl, o);
                            if (lane >= o) incl += n;
                        }
                        const int c = c0 + s * 32 + lane;
                        if (col < E && c < a.nchunks) tab[(size_t)c * stride + idx] = carry + incl - v[s];
                        carry += __shfl_sync(0xffffffffu, incl, 31);
                    }
                }
                if (lane == 0) a.col_total[col] = carry;
            }
        }
        if (!grid_barrier(a.barrier, 2u * G, s_flag)) {
            if (tid == 0) set_error(a.err_out, EP_ERR_TIMEOUT);
            return;
        }

        // the expert counts = the column totals
        for (int e = tid; e < E; e += kRouteThreads) {
            const int cnt = __ldcg(a.col_total + e);
            s_cnt[e] = cnt;
            s_al[e] = (int)(((int64_t)cnt + a.A - 1) / a.A * a.A);
        }
    }

    // ---------------------------------------------------------------- phase 3
    // a bad expert id in any chunk (only CTA 0 reports it)
    int bad_ids = 0;
    if (blockIdx.x == 0) {
        if (a.fold) {
            for (int c = tid; c < a.nchunks; c += kRouteThreads) bad_ids |= __ldcg(a.chunk_err + c);
        } else if (tid == 0) {
            bad_ids = __ldcg(a.col_total + E + R);
        }
    }
    bad_ids = __syncthreads_or(bad_ids);
    const int rows = block_exclusive_scan_E(s_al, s_seg, E, s_warp);
    for (int e = tid; e < E; e += kRouteThreads) s_al[e] -= s_cnt[e];   // padding rows of e
    int pads = 0;
    if (a.A > 1) {   // with expert_alignment 1 there are no padding rows to number
        __syncthreads();
        pads = block_exclusive_scan_E(s_al, s_pad, E, s_warp);
    }
    if (tid == 0) s_pad[E] = pads;
    __syncthreads();

    if (blockIdx.x == 0) {
        for (int e = tid; e < E; e += kRouteThreads) {
            const int cnt = s_cnt[e];
            if (a.psum) a.psum[e] = s_seg[e] + cnt + s_al[e];
            if (a.num_recv) a.num_recv[e] = cnt;
            if (a.num_tokens_per_expert) a.num_tokens_per_expert[e] = cnt;
            if (a.cumulative) a.cumulative[e] += cnt;
        }
        for (int r = tid; r < R; r += kRouteThreads) {
            if (!a.num_tokens_per_rank) break;
            int n = 0;
            if (a.fold) {
                for (int c = 0; c < a.nchunks; ++c) n += s_rtab[(size_t)c * R + r];
            } else {
                n = __ldcg(a.col_total + E + r);
            }
            a.num_tokens_per_rank[r] = n;
        }
        if (tid == 0) {
            int status = bad_ids ? EP_ERR_BAD_EXPERT_ID : 0;
            if (status == 0 && a.check_capacity && a.ll_M == 0 && (int64_t)rows > a.capacity)
                status = EP_ERR_CAPACITY;
            if (status) set_error(a.err_out, status);
        }
    }
    if (!a.assign) return;

    // received row of every entry, and the per-row metadata
    int32_t* s_pre = s_al;   // [E] the chunk's column prefixes (padding counts live in s_pad now)
    for (int c = blockIdx.x; c < a.nchunks; c += G) {
        const int r_src = c / a.chunks_per_rank;
        const int t0 = r_src * a.tokens_per_rank + (c % a.chunks_per_rank) * C;
        const int ne = min(C, a.tokens_per_rank - (c % a.chunks_per_rank) * C) * K;
        const int64_t e0 = (int64_t)t0 * K;
        __syncthreads();
        if (a.fold) {
            // the chunk's prefix, summed with the totals
            for (int e = tid; e < E; e += kRouteThreads) s_pre[e] = s_fpre[e];
        } else if (a.ll_M) {
            // position inside (expert, source rank) = prefix from the rank's first chunk
            const size_t c0 = (size_t)r_src * a.chunks_per_rank;
            for (int e = tid; e < E; e += kRouteThreads)
                s_pre[e] = __ldcg(a.chunk_hist + (size_t)c * E + e) - __ldcg(a.chunk_hist + c0 * E + e);
        } else {
            for (int e = tid; e < E; e += kRouteThreads) s_pre[e] = __ldcg(a.chunk_hist + (size_t)c * E + e);
        }
        if (!resident) {
            for (int i = tid; i < ne; i += kRouteThreads) {
                const int64_t v = a.topk_idx[e0 + i];
                s_idx[i] = (v >= 0 && v < E) ? (int)v : -1;
                s_rank[i] = a.dst_slot[e0 + i];
                s_w[i] = a.topk_weights[e0 + i];
            }
        }
        __syncthreads();
        for (int i = tid; i < ne; i += kRouteThreads) {
            const int tl = i / K, k = i - tl * K;
            const int e = s_idx[i];
            int slot = -1;
            if (e >= 0) {
                if (a.ll_M) {
                    const int pos = s_pre[e] + s_rank[i];
                    if (pos < a.ll_M) {
                        slot = (int)(((int64_t)e * R + r_src) * a.ll_M + pos);
                    } else {
                        set_error(a.err_out, EP_ERR_CAPACITY);
                    }
                } else {
                    const int64_t row = (int64_t)s_seg[e] + s_pre[e] + s_rank[i];
                    slot = row < a.capacity ? (int)row : -1;
                }
            }
            a.dst_slot[e0 + i] = slot;
            if (slot < 0) continue;
            reinterpret_cast<int2*>(a.recv_meta)[slot] = make_int2(a.token_offset + t0 + tl, k);
            const int rdst = rank_of(e, L, shL);
            const int lo = rdst * L;   // local ids of the receiving rank: [lo, lo + L)
            const int* ids = s_idx + tl * K;
            const float* ws = s_w + tl * K;
            if constexpr (KT > 0) {
                int4* ri = reinterpret_cast<int4*>(a.recv_topk_idx + (int64_t)slot * KT);
                float4* rw = reinterpret_cast<float4*>(a.recv_topk_weights + (int64_t)slot * KT);
#pragma unroll
                for (int j = 0; j < KT; j += 4) {
                    int o[4];
                    float w[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int ej = ids[j + u];
                        const bool here = (unsigned)(ej - lo) < (unsigned)L;
                        o[u] = here ? ej - lo : -1;
                        w[u] = here ? ws[j + u] : 0.0f;
                    }
                    ri[j / 4] = make_int4(o[0], o[1], o[2], o[3]);
                    rw[j / 4] = make_float4(w[0], w[1], w[2], w[3]);
                }
            } else {
                int32_t* ri = a.recv_topk_idx + (int64_t)slot * K;
                float* rw = a.recv_topk_weights + (int64_t)slot * K;
                for (int j = 0; j < K; ++j) {
                    const int ej = ids[j];
                    const bool here = (unsigned)(ej - lo) < (unsigned)L;
                    ri[j] = here ? ej - lo : -1;
                    rw[j] = here ? ws[j] : 0.0f;
                }
            }
        }
    }
    if (a.ll_M) {
        // per (expert, source rank): (first row of the rank's block << 32) | entries
        for (int i = blockIdx.x * kRouteThreads + tid; i < E * R; i += G * kRouteThreads) {
            const int e = i / R, r = i - e * R;
            int n = 0;
            if (a.fold) {
                for (int c = r * a.chunks_per_rank; c < (r + 1) * a.chunks_per_rank; ++c)
                    n += s_tab[(size_t)c * E + e];
            } else {
                const bool any = a.chunks_per_rank > 0;
                const int lo = any ? __ldcg(a.chunk_hist + (size_t)r * a.chunks_per_rank * E + e) : 0;
                const int hi = !any ? 0
                               : r + 1 < R ? __ldcg(a.chunk_hist + (size_t)(r + 1) * a.chunks_per_rank * E + e)
                                           : s_cnt[e];
                n = hi - lo;
            }
            if (a.layout_range) a.layout_range[i] = ((int64_t)r * a.ll_M << 32) | (int64_t)n;
        }
        return;   // no padding rows in the fixed-capacity layout
    }
    // padding rows: metadata (-1, -1), recv_topk_idx -1, weight 0
    for (int p = blockIdx.x * kRouteThreads + tid; p < pads; p += G * kRouteThreads) {
        int lo = 0, hi = E;   // the last expert with padding prefix <= p
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (s_pad[mid] <= p) lo = mid; else hi = mid;
        }
        const int64_t row = (int64_t)s_seg[lo] + s_cnt[lo] + (p - s_pad[lo]);
        if (row >= a.capacity) continue;
        reinterpret_cast<int2*>(a.recv_meta)[row] = make_int2(-1, -1);
        for (int j = 0; j < K; ++j) {
            a.recv_topk_idx[row * K + j] = -1;
            a.recv_topk_weights[row * K + j] = 0.0f;
        }
    }
}




namespace {

template <int KT>
cudaError_t launch_route_k(const RouteArgs& a, cudaStream_t st) {
    const size_t smem = a.fold ? route_table_offset(a.E, a.K, a.R, a.log2_chunk) + route_fold_bytes(a)
                               : route_smem_bytes(a.E, a.K, a.R, a.log2_chunk);
    cudaError_t e = cudaFuncSetAttribute(k_route<KT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_route<KT>, kRouteThreads, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const int resident = per_sm * device_sm_count();
    const int grid = max(1, min(a.nchunks, resident));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kRouteThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_route<KT>, a);
}

}  // namespace

cudaError_t launch_route(const RouteArgs& args, cudaStream_t st) {
    cudaError_t e = cudaMemsetAsync(args.barrier, 0, sizeof(unsigned), st);
    if (e != cudaSuccess) return e;
    RouteArgs a = args;
    // fold the column phase when both tables fit in shared memory with the rest
    // (whole 16-byte pieces at 16-byte aligned addresses, rows of whole
    // 16-byte column groups), and every chunk has its own CTA at one CTA per SM
    a.fold = EP_ROUTE_FOLD && a.E % 4 == 0 && ((size_t)a.nchunks * a.R) % 4 == 0 &&
             (reinterpret_cast<uintptr_t>(a.chunk_hist) & 15u) == 0 &&
             (reinterpret_cast<uintptr_t>(a.chunk_rcnt) & 15u) == 0 && a.nchunks <= device_sm_count() &&
             route_table_offset(a.E, a.K, a.R, a.log2_chunk) + route_fold_bytes(a) <= kRouteFoldSmem;
    switch (a.vector_ok ? a.K : 0) {
        case 4: return launch_route_k<4>(a, st);
        case 8: return launch_route_k<8>(a, st);
        case 16: return launch_route_k<16>(a, st);
        default: return launch_route_k<0>(a, st);
    }
}

}  // namespace ep
