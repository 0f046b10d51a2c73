// Group-limited gating: the routing generator upstream of dispatch
// ("DeepEP V1 vs V2 comparative analysis", section 8.1, DeepSeek-V3
// group-limited gating: 256 experts in 32 groups of 8, each token keeps its
// top-4 groups, then the top-2 experts inside each kept group, top-8 in all).
//
// For every token t, from router logits [T, E] (fp32):
//   - the experts form n_group groups of S = E / n_group consecutive ids;
//   - a group's score is the fp32 sum of its per_group largest logits, added
//     from the largest down; of two equal logits (or scores) the lower id ranks
//     first;
//   - the topk_group best groups are kept, and the per_group best experts of
//     each kept group are the token's K = topk_group * per_group entries,
//     listed by logit, largest first (equal logits: lower id first);
//   - topk_weights[t] = softmax over the K selected logits, computed in
//     binary64 and rounded to binary32.
//
// One warp per token.  Lane g owns group g: it streams the group's S logits
// (16-byte loads when S % 4 == 0) through a sorted per_group-entry insertion
// list, then sums the list for the group's score.  The topk_group best groups
// are taken one at a time by a warp max-reduction of order-preserving keys of
// the scores (ties: the lowest lane, i.e. the lower group id); their lanes
// write their entries to shared memory, and lanes 0..K-1 each take one entry,
// count the entries ahead of it (its output position), and compute its weight.
// Non-finite logits set EP_ERR_NONFINITE; they are then ordered as -inf (NaN)
// or +-inf so that the outputs stay K distinct in-range ids.
#include <math.h>

#include <algorithm>

#include "ep_internal.cuh"

namespace ep {

namespace {

constexpr int kGateWarps = 8;   // tokens per CTA

// True if (v, e) ranks ahead of (w, f): larger value, then lower id.
__device__ __forceinline__ bool ahead(float v, int e, float w, int f) { return v > w || (v == w && e < f); }

// An unsigned key with the order of the (non-NaN) floats, -0 and +0 equal:
// every key is above 0, which the group selection uses for "no candidate".
__device__ __forceinline__ uint32_t order_key(float x) {
    const uint32_t u = __float_as_uint(x == 0.0f ? 0.0f : x);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float sanitize(float x, int& bad) {
    if (!isfinite(x)) bad = 1;
    return x != x ? -INFINITY : x;   // NaN ranks last
}

template <int P>
__device__ __forceinline__ void insert(float x, int e, float (&v)[P], int (&id)[P]) {
    // carry (x, e) down the list, kept in (larger value, lower id) order; an
    // empty slot (id < 0) takes it.  A displaced entry carried further down
    // may tie with a later entry by value, so the comparison includes the id.
#pragma unroll
    for (int j = 0; j < P; ++j) {
        if (id[j] < 0 || ahead(x, e, v[j], id[j])) {
            const float tv = v[j];
            const int te = id[j];
            v[j] = x;
            id[j] = e;
            x = tv;
            e = te;
        }
    }
}

template <int P>
__global__ void __launch_bounds__(kGateWarps * 32) k_gate(GateArgs a) {
    __shared__ float s_v[kGateWarps][kMaxTopk];
    __shared__ int s_e[kGateWarps][kMaxTopk];
    __shared__ double s_d[kGateWarps][kMaxTopk];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int S = a.E / a.n_group;
    const int K = a.topk_group * P;
    const bool vec = (S & 3) == 0 && a.vec_ok;
    const bool vec8 = (S & 7) == 0 && a.vec8_ok;
    for (int64_t t = (int64_t)blockIdx.x * kGateWarps + warp; t < a.T; t += (int64_t)gridDim.x * kGateWarps) {
        const float* row = a.logits + t * a.E;
        // 1. the group's per_group best experts and its score (lane g = group g)
        float v[P];
        int id[P];
#pragma unroll
        for (int j = 0; j < P; ++j) {
            v[j] = -INFINITY;
            id[j] = -1;
        }
        int bad = 0;
        const bool owner = lane < a.n_group;
        if (owner) {
            const int e0 = lane * S;
            if (vec8) {   // 32-byte loads: a warp reads whole sectors
                for (int i = 0; i < S / 8; ++i) {
                    uint4 lo, hi;
                    ld_nc_v8(row + e0 + 8 * i, lo, hi);
                    const float q[8] = {__uint_as_float(lo.x), __uint_as_float(lo.y), __uint_as_float(lo.z),
                                        __uint_as_float(lo.w), __uint_as_float(hi.x), __uint_as_float(hi.y),
                                        __uint_as_float(hi.z), __uint_as_float(hi.w)};
#pragma unroll
                    for (int c = 0; c < 8; ++c) insert<P>(sanitize(q[c], bad), e0 + 8 * i + c, v, id);
                }
            } else if (vec) {
                const float4* p = reinterpret_cast<const float4*>(row + e0);
#pragma unroll 2
                for (int i = 0; i < S / 4; ++i) {
                    const float4 q = __ldg(p + i);
                    insert<P>(sanitize(q.x, bad), e0 + 4 * i + 0, v, id);
                    insert<P>(sanitize(q.y, bad), e0 + 4 * i + 1, v, id);
                    insert<P>(sanitize(q.z, bad), e0 + 4 * i + 2, v, id);
                    insert<P>(sanitize(q.w, bad), e0 + 4 * i + 3, v, id);
                }
            } else {
                for (int i = 0; i < S; ++i) insert<P>(sanitize(__ldg(row + e0 + i), bad), e0 + i, v, id);
            }
        }
        if (__any_sync(0xffffffffu, bad) && lane == 0) set_error(a.err, EP_ERR_NONFINITE);
        float score = v[0];
#pragma unroll
        for (int j = 1; j < P; ++j) score = score + v[j];
        if (score != score) score = -INFINITY;   // +inf + -inf
        // 2. the topk_group best groups, one warp max-reduction each: the
        //    largest score's order key, then the lowest lane holding it (equal
        //    scores: the lower group id); 3. the kept groups write their entries
        bool taken = false;
        const uint32_t key = order_key(score);
        for (int j = 0; j < a.topk_group; ++j) {
            const bool cand = owner && !taken;
            const uint32_t best = __reduce_max_sync(0xffffffffu, cand ? key : 0u);
            const int win = __ffs(__ballot_sync(0xffffffffu, cand && key == best)) - 1;
            if (lane == win) {
                taken = true;
#pragma unroll
                for (int i = 0; i < P; ++i) {
                    s_v[warp][j * P + i] = v[i];
                    s_e[warp][j * P + i] = id[i];
                }
            }
        }
        __syncwarp();
        // 4. output position of entry `lane` = entries ahead of it
        float mv = 0.0f;
        int me = 0, pos = 0;
        if (lane < K) {
            mv = s_v[warp][lane];
            me = s_e[warp][lane];
            for (int i = 0; i < K; ++i) pos += ahead(s_v[warp][i], s_e[warp][i], mv, me) ? 1 : 0;
        }
        // the largest selected logit (position 0)
        const unsigned first = __ballot_sync(0xffffffffu, lane < K && pos == 0);
        const float m = __shfl_sync(0xffffffffu, mv, __ffs(first) - 1);
        // 5. softmax in binary64 over the K selected logits, summed in output order
        double d = 0.0;
        if (lane < K) {
            d = exp((double)mv - (double)m);
            s_d[warp][pos] = d;
        }
        __syncwarp();
        if (lane < K) {
            double sum = 0.0;
            for (int i = 0; i < K; ++i) sum += s_d[warp][i];
            a.topk_idx[t * K + pos] = me;
            a.topk_weights[t * K + pos] = (float)(d / sum);
        }
        __syncwarp();
    }
}

template <int P>
cudaError_t launch_gate_p(const GateArgs& a, cudaStream_t st) {
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_gate<P>, kGateWarps * 32, 0) != cudaSuccess ||
        per_sm < 1)
        per_sm = 1;
    const int64_t blocks = (a.T + kGateWarps - 1) / kGateWarps;
    const int grid = (int)std::min<int64_t>(blocks, (int64_t)device_sm_count() * per_sm);
    k_gate<P><<<grid, kGateWarps * 32, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gate(const GateArgs& a, cudaStream_t st) {
    cudaError_t e = cudaMemsetAsync(a.err, 0, sizeof(int32_t), st);
    if (e != cudaSuccess || a.T == 0) return e;
    switch (a.per_group) {
#define EP_GATE_CASE(P) \
    case P: return launch_gate_p<P>(a, st);
        EP_GATE_CASE(1) EP_GATE_CASE(2) EP_GATE_CASE(3) EP_GATE_CASE(4)
        EP_GATE_CASE(5) EP_GATE_CASE(6) EP_GATE_CASE(7) EP_GATE_CASE(8)
        EP_GATE_CASE(9) EP_GATE_CASE(10) EP_GATE_CASE(11) EP_GATE_CASE(12)
        EP_GATE_CASE(13) EP_GATE_CASE(14) EP_GATE_CASE(15) EP_GATE_CASE(16)
#undef EP_GATE_CASE
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace ep
