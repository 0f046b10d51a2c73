// Permute / pack: every source token's row is read from HBM once and written
// to each of its received rows (one per unmasked top-k entry, rows already
// resolved by k_route into dst_buffer_slot_idx), as a bf16 bit copy or
// quantised once per token on the fly:
//   - FP8 e4m3 (OCP e4m3fn) or int8 with one fp32 scale per quant_size
//     channels: scale = max(amax, 1e-4) / 448 (or / 127) by IEEE division,
//     optionally rounded up to a power of two (round_scale / use_ue8m0 of
//     low_latency_dispatch, "DeepEP communication library guide v2.1") and
//     then optionally stored as its UE8M0 byte; codes = RNE-saturating
//     conversion of the IEEE quotient x / scale;
//   - MXFP4 (use_mxfp4, groups of 32): E2M1 codes of x / 2^(floor(log2 amax) - 2)
//     with the scale stored as its UE8M0 byte (the OCP MX conversion);
//   - quant_size = 16..512 (group) or hidden (per token) (guide v2.1, 1.3.1).
// The same persistent grid zero-fills the padding rows that expert alignment
// adds (comparative analysis, section 3.1).
//
// bf16 rows move entirely on the TMA engine: one warp per CTA runs an S-stage
// ring in shared memory; lane 0 streams row chunks in with cp.async.bulk
// (completion on an mbarrier) and, once a chunk has landed, issues one
// cp.async.bulk store per destination row from the same shared-memory stage.
// No register ever holds row data; every bulk copy fills or drains this
// CTA's own shared memory.
// Quantised rows are computed by threads from 16-byte vector loads and
// written with 16-byte vector stores.
#include <cuda_bf16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>

#include "ep_internal.cuh"
#include "quant.cuh"
#include "tma.cuh"

#ifndef EP_PACK_STAGES
#define EP_PACK_STAGES 4
#endif
#ifndef EP_PACK_GROUP_UPT
#define EP_PACK_GROUP_UPT 1          // 16-channel units per thread per pass of the group kernel
#endif
#ifndef EP_PACK_GROUP_MIN_BLOCKS
#define EP_PACK_GROUP_MIN_BLOCKS 2   // resident CTAs per SM the group kernel's registers must allow
#endif

namespace ep {

namespace {

constexpr int kBulkChunk = 16384;          // max bytes per pipeline stage

// 16 bytes of quantised codes to a received row, with the L2 policy `pol`
// (evict-first: the row is read once, by the experts, long after).
__device__ __forceinline__ void st_code_v4(void* p, uint4 v, uint64_t pol) {
    asm volatile("st.global.L2::cache_hint.v4.u32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(p), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w), "l"(pol)
                 : "memory");
}

// Padding map from the handle: expert e's padding rows are
// [psum[e-1] + cnt[e], psum[e]), numbered consecutively over the experts by
// base[e] (base[E] = all padding rows).  Any blockDim that is a multiple of
// 32; every thread returns the number of padding rows.
__device__ int build_pad_map(const PackArgs& a, int* s_base, int* s_start, int* s_warp) {
    const int E = a.E, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nwarps = blockDim.x >> 5;
    const int per = (E + blockDim.x - 1) / blockDim.x;
    const int e0 = min(tid * per, E), e1 = min(e0 + per, E);
    int sum = 0;
    for (int e = e0; e < e1; ++e) sum += (a.psum[e] - (e ? a.psum[e - 1] : 0)) - a.cnt[e];
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int w = lane < nwarps ? s_warp[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += n;
        }
        if (lane < nwarps) s_warp[lane] = w;
    }
    __syncthreads();
    int run = incl - sum + (warp > 0 ? s_warp[warp - 1] : 0);
    for (int e = e0; e < e1; ++e) {
        const int lo = e ? a.psum[e - 1] : 0;
        s_base[e] = run;
        s_start[e] = lo + a.cnt[e];
        run += (a.psum[e] - lo) - a.cnt[e];
    }
    const int total = s_warp[nwarps - 1];
    if (tid == 0) s_base[E] = total;
    __syncthreads();
    return total;
}

// Padding row number p (0-based over all experts) -> its row index.
__device__ __forceinline__ int64_t pad_row(int E, const int* s_base, const int* s_start, int p) {
    int lo = 0, hi = E;   // the last expert with base <= p
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (s_base[mid] <= p) lo = mid; else hi = mid;
    }
    return (int64_t)s_start[lo] + (p - s_base[lo]);
}

__device__ __forceinline__ void store_scale(const PackArgs& a, size_t idx, float s) {
    if (a.scale_bytes) reinterpret_cast<uint8_t*>(a.recv_scales)[idx] = ue8m0_of(s);
    else a.recv_scales[idx] = s;
}

__device__ __forceinline__ void zero_scales(const PackArgs& a, int64_t row, int nscales) {
    for (int j = threadIdx.x; j < nscales; j += blockDim.x) {
        if (a.scale_bytes) reinterpret_cast<uint8_t*>(a.recv_scales)[row * nscales + j] = 0;
        else a.recv_scales[row * nscales + j] = 0.0f;
    }
}

// The routing kernel that this pack depends on stopped on its bounded wait:
// the handle's rows and counts were not written, so nothing is packed (the
// status word already holds EP_ERR_TIMEOUT).
__device__ __forceinline__ bool routing_gave_up(const PackArgs& a) {
    return *reinterpret_cast<const volatile int32_t*>(a.err) == EP_ERR_TIMEOUT;
}

// A destination row as the pack kernels use it: rows at or past the receive
// capacity (a handle with foreign rows, or slots left stale by routing that
// stopped on an error) are reported as EP_ERR_CAPACITY and dropped (-1).
__device__ __forceinline__ int checked_row(const PackArgs& a, int slot) {
    if (slot >= a.capacity) {
        set_error(a.err, EP_ERR_CAPACITY);
        return -1;
    }
    return slot;
}

// Loads the K received rows of token t into s_slot (threads 0..K-1).
__device__ __forceinline__ void load_slots(const PackArgs& a, int t, int* s_slot) {
    if (threadIdx.x < a.K) s_slot[threadIdx.x] = checked_row(a, a.dst_slot[(int64_t)t * a.K + threadIdx.x]);
}

}  // namespace

// ----------------------------------------------------- bf16: TMA bulk copy
// Work unit = (token, chunk of its row); CTA b takes units b, b + grid, ...
// Stage of the i-th own unit: i % S.  Lane 0 issues every bulk copy; lanes
// 0..K-1 fetch the unit's destination rows one iteration ahead of use.
template <int S>
__global__ void __launch_bounds__(32) k_pack_bulk(PackArgs a, int chunk_bytes) {
    extern __shared__ __align__(128) uint8_t smem[];
    uint8_t* stage = smem;
    uint64_t* mbar = reinterpret_cast<uint64_t*>(smem + (size_t)S * chunk_bytes);
    int* sslot = reinterpret_cast<int*>(mbar + S);                 // [S][kMaxTopk]
    int* s_pad_base = sslot + S * kMaxTopk;                          // [E+1]
    int* s_pad_start = s_pad_base + a.E + 1;                         // [E]
    int* s_warp = s_pad_start + a.E;                                 // [32]
    const int lane = threadIdx.x;
    const int K = a.K;
    const int64_t row_bytes = (int64_t)a.H * 2;
    const int nch = (int)((row_bytes + chunk_bytes - 1) / chunk_bytes);
    const int n_units = a.n_tok_items * nch;
    const int n_mine = n_units > (int)blockIdx.x ? (n_units - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
    const uint8_t* xb = reinterpret_cast<const uint8_t*>(a.x);

    if (lane == 0) {
        for (int s = 0; s < S; ++s) mbar_init(&mbar[s], 1);
        fence_mbar_init();
    }

    auto unit = [&](int j, int& t, int& c) {
        const int u = (int)blockIdx.x + j * (int)gridDim.x;
        const int item = u / nch;
        c = u - item * nch;
        t = token_of_item(item, a.tokens_per_rank, a.per_round, a.round);
    };
    auto issue_load = [&](int j, int t, int c) {
        const int64_t off = (int64_t)c * chunk_bytes;
        const uint32_t bytes = (uint32_t)min((int64_t)chunk_bytes, row_bytes - off);
        uint64_t* bar = &mbar[j % S];
        mbar_expect_tx(bar, bytes);
        bulk_load(stage + (size_t)(j % S) * chunk_bytes, xb + (int64_t)t * row_bytes + off, bytes, bar);
    };

    // prologue: units 0 .. S-2.  With routing just ahead on the stream (x
    // complete before it started) their x chunks are requested before the
    // wait for the routing results, while routing runs
    const int pro = min(S - 1, n_mine);
    const bool early = a.early_x != 0;
    if (early && lane == 0) {
        for (int j = 0; j < pro; ++j) {
            int t, c;
            unit(j, t, c);
            issue_load(j, t, c);
        }
    }
    grid_dependency_wait();
    grid_launch_dependents();
    if (routing_gave_up(a)) {
        // the chunks requested early land before the CTA releases its smem
        if (early && lane == 0)
            for (int j = 0; j < pro; ++j) mbar_wait(&mbar[j % S], (uint32_t)((j / S) & 1));
        __syncwarp();
        return;
    }
    const int n_pad = a.do_pad ? build_pad_map(a, s_pad_base, s_pad_start, s_warp) : 0;
    __syncwarp();
    for (int j = 0; j < pro; ++j) {
        int t, c;
        unit(j, t, c);
        if (!early && lane == 0) issue_load(j, t, c);
        if (lane < K) sslot[(j % S) * kMaxTopk + lane] = checked_row(a, a.dst_slot[(int64_t)t * K + lane]);
    }
    __syncwarp();

    bool ok = true;
    int pending = -1;
    int i = 0;
    for (; i < n_mine; ++i) {
        const int s = i % S;
        // slots fetched last iteration belong to unit i + S - 2
        if (i >= 1 && i + S - 2 < n_mine && lane < K) sslot[((i + S - 2) % S) * kMaxTopk + lane] = checked_row(a, pending);
        // lane 0 waits for the stage; the outcome is broadcast so the warp stays converged
        int landed = lane == 0 ? (int)mbar_wait(&mbar[s], (uint32_t)((i / S) & 1)) : 0;
        landed = __shfl_sync(0xffffffffu, landed, 0);
        if (!landed) {
            ok = false;
            break;
        }
        int t, c;
        unit(i, t, c);
        if (lane == 0) {
            const int64_t off = (int64_t)c * chunk_bytes;
            const uint32_t bytes = (uint32_t)min((int64_t)chunk_bytes, row_bytes - off);
            fence_proxy_async_smem();
            for (int k = 0; k < K; ++k) {
                const int slot = sslot[s * kMaxTopk + k];
                if (slot >= 0)
                    bulk_store(a.recv_x + (int64_t)slot * row_bytes + off, stage + (size_t)s * chunk_bytes, bytes);
            }
            bulk_commit();
            bulk_wait_read<1>();   // the stores of unit i-1 have read their stage
        }
        __syncwarp();
        const int nxt = i + S - 1;
        if (nxt < n_mine) {
            int tn, cn;
            unit(nxt, tn, cn);
            if (lane == 0) issue_load(nxt, tn, cn);
            if (lane < K) pending = a.dst_slot[(int64_t)tn * K + lane];
        }
    }
    if (!ok) {
        set_error(a.err, EP_ERR_TIMEOUT);
        // let every load still in flight land before the CTA releases its smem
        if (lane == 0) {
            for (int j = i; j < min(n_mine, i + S - 1); ++j) mbar_wait(&mbar[j % S], (uint32_t)((j / S) & 1));
            bulk_wait_all();
        }
        __syncwarp();
        return;
    }
    if (lane == 0) bulk_wait_read<0>();
    __syncwarp();

    // padding rows: bulk stores from a zeroed stage
    const int pad_units = n_pad * nch;
    if ((int)blockIdx.x < pad_units) {
        for (int b = lane * 16; b < chunk_bytes; b += 32 * 16)
            *reinterpret_cast<uint4*>(stage + b) = make_uint4(0, 0, 0, 0);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
            for (int u = blockIdx.x; u < pad_units; u += gridDim.x) {
                const int p = u / nch, c = u - p * nch;
                const int64_t row = pad_row(a.E, s_pad_base, s_pad_start, p);
                const int64_t off = (int64_t)c * chunk_bytes;
                const uint32_t bytes = (uint32_t)min((int64_t)chunk_bytes, row_bytes - off);
                if (row >= 0 && row < a.capacity) bulk_store(a.recv_x + row * row_bytes + off, stage, bytes);
            }
            bulk_commit();
        }
    }
    if (lane == 0) bulk_wait_all();
}

// ----------------------------------------------- bf16: vector loads/stores
// Alternative data path (16-byte ld/st through registers), kept for
// comparison with the bulk-copy path.
template <int VPT>
__global__ void __launch_bounds__(256) k_pack_bf16(PackArgs a) {
    grid_dependency_wait();
    grid_launch_dependents();
    if (routing_gave_up(a)) return;
    __shared__ int s_slot[kMaxTopk];
    __shared__ int s_pad_base[kMaxExperts + 1], s_pad_start[kMaxExperts], s_warp[32];
    const int tid = threadIdx.x;
    const int V = a.H / 8;   // 16-byte vectors per row
    const int n_pad = a.do_pad ? build_pad_map(a, s_pad_base, s_pad_start, s_warp) : 0;
    const int n_items = a.n_tok_items + n_pad;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
        if (item < a.n_tok_items) {
            const int t = token_of_item(item, a.tokens_per_rank, a.per_round, a.round);
            load_slots(a, t, s_slot);
            __syncthreads();
            const uint4* xr = reinterpret_cast<const uint4*>(a.x + (size_t)t * a.H);
            for (int v0 = 0; v0 < V; v0 += VPT * blockDim.x) {
                uint4 r[VPT];
#pragma unroll
                for (int u = 0; u < VPT; ++u) {
                    const int v = v0 + u * blockDim.x + tid;
                    if (v < V) r[u] = ld_nc_v4(xr + v);
                }
                for (int k = 0; k < a.K; ++k) {
                    const int slot = s_slot[k];
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
            const int64_t row = pad_row(a.E, s_pad_base, s_pad_start, item - a.n_tok_items);
            if (row >= 0 && row < a.capacity) {
                uint4* dst = reinterpret_cast<uint4*>(a.recv_x + (size_t)row * a.H * 2);
                for (int v = tid; v < V; v += blockDim.x) st_v4(dst + v, make_uint4(0, 0, 0, 0));
            }
        }
        __syncthreads();
    }
}

// ------------------------------------------------- group quantisation (<=512)
// A thread owns 16 consecutive channels per unit (two 16-byte loads; one
// 16-byte store of FP8 / int8 codes, or one 8-byte store of 16 E2M1 codes); a
// group of G channels is G/16 adjacent lanes, reduced by shuffles.  A work
// item is one pass (UPT x blockDim units) over one token's row, or one padding
// row.  The CTA's next item is fetched (its x units into registers, its
// destination rows into the other half of s_slot) before the current item is
// quantised and stored, so its loads are in flight during that work.  A
// warp's units cover whole groups; the K x (groups of the warp) scale stores
// of an item are spread over the warp's lanes, one or a few per lane, instead
// of one lane of each group storing K scales.
// With a.early_x (the routing kernel runs just before, so x was complete
// before it started), the CTA's first item is loaded and quantised before the
// wait for the routing results, while routing runs.
template <int QUANT, int G, int UPT>
__global__ void __launch_bounds__(512 / UPT, EP_PACK_GROUP_MIN_BLOCKS) k_pack_group(PackArgs a) {
    __shared__ int s_slot[2][kMaxTopk];
    __shared__ int s_pad_base[kMaxExperts + 1], s_pad_start[kMaxExperts], s_warp[32];
    constexpr int kLanes = G / 16;
    constexpr int kGroupsPerWarp = 32 / kLanes;
    constexpr float kQmax = QUANT == kQuantFp8 ? 448.0f : 127.0f;
    constexpr int kUnitBytes = QUANT == kQuantMxfp4 ? 8 : 16;   // code bytes of 16 channels
    const int tid = threadIdx.x, lane = tid & 31;
    const int U = a.H / 16;
    const int per_pass = UPT * blockDim.x;
    const int passes = (U + per_pass - 1) / per_pass;
    const size_t row_bytes = (size_t)U * kUnitBytes;
    const int nscales = a.H / G;
    const int n_tok = a.n_tok_items * passes;

    // item -> token, and the first unit of its pass; with one pass per row and
    // one round (every workload but the longest rows and rounds) the item is
    // the token, with no division
    const bool direct = passes == 1 && a.per_round == a.tokens_per_rank;
    auto locate = [&](int item, int& t, int& u0) {
        if (direct) {
            t = item;
            u0 = 0;
            return;
        }
        const int ti = item / passes;
        u0 = (item - ti * passes) * per_pass;
        t = token_of_item(ti, a.tokens_per_rank, a.per_round, a.round);
    };
    // issues the loads of a token item's units into r
    auto fetch_x = [&](int item, uint4 (&r)[UPT][2]) {
        int t, u0;
        locate(item, t, u0);
        const uint4* xr = reinterpret_cast<const uint4*>(a.x + (size_t)t * a.H);
#pragma unroll
        for (int j = 0; j < UPT; ++j) {
            const int u = u0 + j * blockDim.x + tid;
            if (u < U) {
                if (a.x32) {
                    ld_nc_v8(xr + 2 * u, r[j][0], r[j][1]);
                } else {
                    r[j][0] = ld_nc_v4(xr + 2 * u);
                    r[j][1] = ld_nc_v4(xr + 2 * u + 1);
                }
            } else {
                r[j][0] = r[j][1] = make_uint4(0, 0, 0, 0);
            }
        }
    };
    // threads 0..K-1: the received row of entry tid of a token item
    auto fetch_slot = [&](int item) {
        int t, u0;
        locate(item, t, u0);
        return tid < a.K ? a.dst_slot[(int64_t)t * a.K + tid] : -1;
    };
    auto quantize = [&](const uint4 (&r)[UPT][2], uint4 (&q)[UPT], float (&sc)[UPT]) {
#pragma unroll
        for (int j = 0; j < UPT; ++j) {
            float f[16];
            unpack16(r[j][0], r[j][1], f);
            float m = amax16(f);
#pragma unroll
            for (int o = kLanes / 2; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            if constexpr (QUANT == kQuantMxfp4) {
                sc[j] = mx_scale(m);
                const uint2 c = quant16_fp4(f, sc[j]);
                q[j] = make_uint4(c.x, c.y, 0, 0);
            } else {
                sc[j] = finish_scale(m, kQmax, a.round_scale);
                q[j] = quant16<QUANT>(f, sc[j]);
            }
        }
    };
    // the codes and scales of a token item to its received rows s_slot[b]
    auto store_item = [&](int item, const uint4 (&q)[UPT], const float (&sc)[UPT], int b) {
        int t, u0;
        locate(item, t, u0);
        // codes: per received row one 32 x 32 -> 64-bit multiply-add and
        // one store per unit (a row is at most 64 KB of codes)
        uint8_t* const xb = a.recv_x + (size_t)(u0 + tid) * kUnitBytes;
        const int rb = (int)row_bytes;
        for (int k = 0; k < a.K; ++k) {
            const int slot = s_slot[b][k];
            if (slot < 0) continue;
            uint8_t* const dst = xb + (long long)slot * rb;
#pragma unroll
            for (int j = 0; j < UPT; ++j) {
                if (u0 + j * (int)blockDim.x + tid < U) {
                    uint8_t* const p = dst + j * (int)blockDim.x * kUnitBytes;
                    if constexpr (QUANT == kQuantMxfp4) {
                        *reinterpret_cast<uint2*>(p) = make_uint2(q[j].x, q[j].y);
                    } else {
                        st_code_v4(p, q[j], l2_evict_first());
                    }
                }
            }
        }
        // scales: entry i of the warp's K x kGroupsPerWarp stores of pass
        // slice j is (row i / kGroupsPerWarp, group i % kGroupsPerWarp of
        // the warp); lane i % 32 stores it, with the scale of the group's
        // first lane
#pragma unroll
        for (int j = 0; j < UPT; ++j) {
            const int wu = u0 + j * (int)blockDim.x + (tid & ~31);   // the warp's first unit
            const int n = a.K * kGroupsPerWarp;
            for (int i0 = 0; i0 < n; i0 += 32) {
                const int i = i0 + lane;
                const int g = i % kGroupsPerWarp;
                const float s = __shfl_sync(0xffffffffu, sc[j], g * kLanes);
                const int ug = wu + g * kLanes;
                if (i < n && ug < U) {
                    const int row = s_slot[b][i / kGroupsPerWarp];
                    if (row >= 0) store_scale(a, (size_t)row * nscales + ug / kLanes, s);
                }
            }
        }
    };

    int item = blockIdx.x;
    const bool early = a.early_x != 0 && item < n_tok;
    uint4 q0[UPT];
    float sc0[UPT];
    if (early) {
        uint4 r0[UPT][2];
        fetch_x(item, r0);
        quantize(r0, q0, sc0);
    }
    grid_dependency_wait();
    grid_launch_dependents();
    if (routing_gave_up(a)) return;
    const int n_pad = a.do_pad ? build_pad_map(a, s_pad_base, s_pad_start, s_warp) : 0;
    const int n_items = n_tok + n_pad;
    if (early) {
        // the first item, quantised during routing: its rows, then its stores
        const int slot = fetch_slot(item);
        if (tid < a.K) s_slot[1][tid] = checked_row(a, slot);
        __syncthreads();
        store_item(item, q0, sc0, 1);
        item += gridDim.x;
    }

    uint4 raw[UPT][2];
    int slot_next = -1;
    if (item < n_tok) {
        fetch_x(item, raw);
        slot_next = fetch_slot(item);
    }
    if (tid < a.K) s_slot[0][tid] = checked_row(a, slot_next);
    __syncthreads();
    int buf = 0;
    for (; item < n_items; item += gridDim.x) {
        const int nxt = item + gridDim.x;
        uint4 nraw[UPT][2];
        slot_next = -1;
        if (nxt < n_tok) {
            fetch_x(nxt, nraw);
            slot_next = fetch_slot(nxt);
        } else {
#pragma unroll
            for (int j = 0; j < UPT; ++j) nraw[j][0] = nraw[j][1] = make_uint4(0, 0, 0, 0);
        }
        if (item < n_tok) {
            uint4 q[UPT];
            float sc[UPT];
            quantize(raw, q, sc);
            store_item(item, q, sc, buf);
        } else {
            const int64_t row = pad_row(a.E, s_pad_base, s_pad_start, item - n_tok);
            if (row >= 0 && row < a.capacity) {
                uint4* dst = reinterpret_cast<uint4*>(a.recv_x + (size_t)row * row_bytes);
                for (size_t v = tid; v < row_bytes / 16; v += blockDim.x) st_v4(dst + v, make_uint4(0, 0, 0, 0));
                zero_scales(a, row, nscales);
            }
        }
        if (tid < a.K) s_slot[buf ^ 1][tid] = checked_row(a, slot_next);
#pragma unroll
        for (int j = 0; j < UPT; ++j) {
            raw[j][0] = nraw[j][0];
            raw[j][1] = nraw[j][1];
        }
        buf ^= 1;
        __syncthreads();
    }
}


// ----------------------------------------------- per-token quantisation (G=H)
// The whole row stays in registers (UPT units of 16 channels per thread) while
// the block reduces its amax.
template <int QUANT, int UPT>
__global__ void __launch_bounds__(1024) k_pack_token(PackArgs a) {
    grid_dependency_wait();
    grid_launch_dependents();
    if (routing_gave_up(a)) return;
    __shared__ int s_slot[kMaxTopk];
    __shared__ float s_red[33];
    __shared__ int s_pad_base[kMaxExperts + 1], s_pad_start[kMaxExperts], s_warp[32];
    constexpr float kQmax = QUANT == kQuantFp8 ? 448.0f : 127.0f;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nwarps = blockDim.x >> 5;
    const int U = a.H / 16;
    const int n_pad = a.do_pad ? build_pad_map(a, s_pad_base, s_pad_start, s_warp) : 0;
    const int n_items = a.n_tok_items + n_pad;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
        if (item < a.n_tok_items) {
            const int t = token_of_item(item, a.tokens_per_rank, a.per_round, a.round);
            load_slots(a, t, s_slot);
            const uint4* xr = reinterpret_cast<const uint4*>(a.x + (size_t)t * a.H);
            uint4 raw[UPT][2];
#pragma unroll
            for (int j = 0; j < UPT; ++j) {
                const int u = j * blockDim.x + tid;
                if (u < U) {
                    if (a.x32) {
                        ld_nc_v8(xr + 2 * u, raw[j][0], raw[j][1]);
                    } else {
                        raw[j][0] = ld_nc_v4(xr + 2 * u);
                        raw[j][1] = ld_nc_v4(xr + 2 * u + 1);
                    }
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
            if (lane == 0) s_red[warp] = m;
            __syncthreads();
            if (warp == 0) {
                float v = lane < nwarps ? s_red[lane] : 0.0f;
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
                if (lane == 0) s_red[32] = v;
            }
            __syncthreads();
            const float sc = finish_scale(s_red[32], kQmax, a.round_scale);
            // quantise once; raw[j][0] is reused to hold the 16 codes of unit j
#pragma unroll
            for (int j = 0; j < UPT; ++j) {
                float f[16];
                unpack16(raw[j][0], raw[j][1], f);
                raw[j][0] = quant16<QUANT, false>(f, sc);
            }
            for (int k = 0; k < a.K; ++k) {
                const int slot = s_slot[k];
                if (slot < 0) continue;
                uint8_t* dst = a.recv_x + (size_t)slot * a.H;
#pragma unroll
                for (int j = 0; j < UPT; ++j) {
                    const int u = j * blockDim.x + tid;
                    if (u < U) st_v4(dst + 16 * (size_t)u, raw[j][0]);
                }
                if (tid == 0) store_scale(a, (size_t)slot, sc);
            }
        } else {
            const int64_t row = pad_row(a.E, s_pad_base, s_pad_start, item - a.n_tok_items);
            if (row >= 0 && row < a.capacity) {
                uint4* dst = reinterpret_cast<uint4*>(a.recv_x + (size_t)row * a.H);
                for (int v = tid; v < U; v += blockDim.x) st_v4(dst + v, make_uint4(0, 0, 0, 0));
                if (tid == 0) zero_scales(a, row, 1);
            }
        }
        __syncthreads();
    }
}

// ------------------------------------------------------------------ launch
namespace {

template <typename Kern>
int blocks_per_sm(Kern k, int threads, size_t smem) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k, threads, smem) != cudaSuccess || n < 1) n = 1;
    return n;
}

inline int round_up32(int x) { return (x + 31) & ~31; }

template <typename Kern>
cudaError_t run(Kern k, int threads, const PackArgs& a, cudaStream_t st) {
    const int grid = device_sm_count() * blocks_per_sm(k, threads, 0);
    return launch_dependent(k, dim3(grid), dim3(threads), 0, st, a);
}

template <int QUANT>
cudaError_t launch_group(const PackArgs& a, cudaStream_t st) {
    constexpr int P = EP_PACK_GROUP_UPT;
    const int U = a.H / 16;
    const int threads = min(512 / P, round_up32((U + P - 1) / P));   // P units per thread
    if constexpr (QUANT == kQuantMxfp4) {
        if (a.quant_size != 32) return cudaErrorInvalidValue;
        return run(k_pack_group<kQuantMxfp4, 32, P>, threads, a, st);
    } else {
        switch (a.quant_size) {
            case 16: return run(k_pack_group<QUANT, 16, P>, threads, a, st);
            case 32: return run(k_pack_group<QUANT, 32, P>, threads, a, st);
            case 64: return run(k_pack_group<QUANT, 64, P>, threads, a, st);
            case 128: return run(k_pack_group<QUANT, 128, P>, threads, a, st);
            case 256: return run(k_pack_group<QUANT, 256, P>, threads, a, st);
            case 512: return run(k_pack_group<QUANT, 512, P>, threads, a, st);
            default: return cudaErrorInvalidValue;
        }
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

cudaError_t launch_bulk(const PackArgs& a, cudaStream_t st) {
    constexpr int S = EP_PACK_STAGES;
    const int64_t row_bytes = (int64_t)a.H * 2;
    // equal chunks of at most kBulkChunk bytes, each a multiple of 16
    const int nch = (int)((row_bytes + kBulkChunk - 1) / kBulkChunk);
    const int chunk = (int)(((row_bytes + nch - 1) / nch + 15) / 16 * 16);
    const size_t smem = (size_t)S * chunk + S * sizeof(uint64_t) + S * kMaxTopk * sizeof(int) +
                        (2 * (size_t)a.E + 1 + 32) * sizeof(int);
    cudaError_t e = cudaFuncSetAttribute(k_pack_bulk<S>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int grid = device_sm_count() * blocks_per_sm(k_pack_bulk<S>, 32, smem);
    return launch_dependent(k_pack_bulk<S>, dim3(grid), dim3(32), smem, st, a, chunk);
}

}  // namespace

cudaError_t launch_pack(const PackArgs& a, int quant, cudaStream_t st) {
    if (quant == EP_QUANT_NONE) {
#ifdef EP_PACK_VECTOR
        const int V = a.H / 8;
        const int passes = (V + 4 * 256 - 1) / (4 * 256);
        const int threads = min(256, round_up32((V + 4 * passes - 1) / (4 * passes)));
        return run(k_pack_bf16<4>, threads, a, st);
#else
        return launch_bulk(a, st);
#endif
    }
    if (quant == EP_QUANT_MXFP4) return launch_group<kQuantMxfp4>(a, st);
    const bool per_token = a.quant_size == a.H;
    if (quant == EP_QUANT_FP8_E4M3)
        return per_token ? launch_token<kQuantFp8>(a, st) : launch_group<kQuantFp8>(a, st);
    return per_token ? launch_token<kQuantInt8>(a, st) : launch_group<kQuantInt8>(a, st);
}

}  // namespace ep
