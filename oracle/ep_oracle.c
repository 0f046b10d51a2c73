/*
 * ep_oracle.c -- CPU oracle for MoE expert-parallel dispatch / combine.
 *
 * TEST INFRASTRUCTURE ONLY.  This is a plain, slow, single-threaded reference
 * that the parity tests, the smoke check and the benchmark's CPU-baseline leg
 * compare the CUDA path against.  It shares no code, header, table or helper
 * with the CUDA library, and the product path never calls it.
 *
 * The same source also builds with OpenMP (liboracle_omp.so): the loops over
 * independent tokens in the row functions are then split across threads.
 * Every token's arithmetic is the one written here either way; only which
 * thread computes it changes.  The row functions report the largest status
 * code that any token met.
 *
 * What it computes, and where the pages define it:
 *
 *  - get_dispatch_layout: num_tokens_per_rank, num_tokens_per_expert and
 *    is_token_in_rank from topk_idx ("DeepEP V1 vs V2 comparative analysis",
 *    section 2.1, the V1 normal-mode API).  Expert e lives on rank e / L with
 *    L = num_local_experts = num_experts / ep_world_size ("DeepEP on Ascend A2"
 *    page, Usage, the HCCL_BUFFSIZE note).  Entries equal to -1 are masked.
 *  - dispatch slots: one received row per unmasked (token, expert) pair
 *    (expand mode, do_expand in the EPHandle fields of section 3.1 of the
 *    comparative analysis), rows ordered by (expert, source token, k) -- the
 *    deterministic order of section 8.4 -- and every expert segment rounded up
 *    to expert_alignment (section 3.1).  psum_num_recv_tokens_per_expert is the
 *    inclusive prefix sum of the aligned counts; the unaligned counts are
 *    returned beside it (section 3.1; the A2 page's MOE_EXPERT_TOKEN_NUMS_TYPE
 *    switch between counts and prefix sums).  recv_src_metadata and
 *    dst_buffer_slot_idx are the two directions of the row <-> (token, k) map.
 *  - recv_x: the bf16 row of the source token, or its quantisation:
 *    FP8 e4m3 with one fp32 scale per 128 channels, optionally rounded up to a
 *    power of two (use_fp8 / round_scale / use_ue8m0 of low_latency_dispatch in
 *    "DeepEP communication library guide v2.1"; float8_e4m3fn storage in
 *    section 7.4 of the comparative analysis), or int8 with quant_size 128
 *    (group) or hidden (per token) (guide v2.1, section 1.3.1; the A2 page's
 *    DEEP_NORMAL_MODE_USE_INT8_QUANT).
 *  - combine: out[t] = bf16( sum over unmasked k, in k order, of
 *    topk_weights[t,k] * y[dst_buffer_slot_idx[t,k]] ), accumulated in fp32
 *    with fused multiply-add (the reverse of dispatch, combine in section 9.2
 *    of the comparative analysis).
 *  - long-sequence rounds: the A2 page's "ant moving home" feature processes
 *    each rank's tokens in rounds of PER_ROUND_TOKENS; the API is unchanged, so
 *    the result equals the one-shot result (see oracle_dispatch_rows with a
 *    round token list).
 *
 * Readings where the pages are silent (each also listed in the design notes):
 * padding rows hold zero bytes, scale 0, metadata (-1, -1), recv_topk_idx -1
 * and weight 0; the FP8/int8 amax is floored at 1e-4; scale = amax / 448 (or
 * / 127) by IEEE fp32 division; x / scale by IEEE fp32 division; FP8 encoding
 * rounds to nearest even and saturates to +-448; int8 rounds to nearest even
 * and clamps to [-127, 127]; recv_topk_idx holds the receiving rank's local
 * expert id of every top-k entry that lives on that rank, else -1.
 *
 * Status codes are this file's own (0 ok, 1 invalid argument, 2 expert id out
 * of range, 3 receive capacity too small, 4 a non-finite router logit).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OR_OK 0
#define OR_INVALID_ARG 1
#define OR_BAD_EXPERT_ID 2
#define OR_CAPACITY 3

#define OR_QUANT_NONE 0
#define OR_QUANT_FP8 1
#define OR_QUANT_INT8 2

/* ---------------------------------------------------------------- numbers */

/* bf16 is the upper half of an IEEE-754 binary32. */
float oracle_bf16_to_f32(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Round a binary32 to the nearest bf16, ties to even (NaN stays NaN). */
uint16_t oracle_f32_to_bf16(float f) {
    if (isnan(f)) return 0x7fc0;
    double v = (double)f;                  /* exact */
    if (v == 0.0 || isinf(v)) {
        uint32_t u;
        memcpy(&u, &f, sizeof u);
        return (uint16_t)(u >> 16);
    }
    /* bf16 keeps 8 significant bits: quantum of the binade of |v| is
     * 2^(floor(log2|v|) - 7), or 2^-133 below the smallest normal 2^-126. */
    int ex;
    frexp(fabs(v), &ex);                   /* |v| = m * 2^ex, m in [0.5, 1) */
    int e2 = ex - 1;
    if (e2 < -126) e2 = -126;
    double q = ldexp(1.0, e2 - 7);
    double n = nearbyint(fabs(v) / q);     /* exact quotient; ties to even */
    double r = n * q;
    float rf = (float)r;                   /* exact unless it overflows to inf */
    uint32_t u;
    memcpy(&u, &rf, sizeof u);
    uint16_t bits = (uint16_t)(u >> 16);
    return v < 0 ? (uint16_t)(bits | 0x8000) : bits;
}

/* OCP 8-bit floating point, E4M3 ("fn": finite values and NaN only):
 * 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits; exponent field 0
 * is subnormal (m * 2^-9); S.1111.111 is NaN; the largest finite value is
 * 1.75 * 2^8 = 448. */
double oracle_e4m3_to_f64(uint8_t c) {
    int s = c >> 7, e = (c >> 3) & 15, m = c & 7;
    if (e == 15 && m == 7) return NAN;
    double v = (e == 0) ? ldexp((double)m, -9) : ldexp(8.0 + m, e - 10);
    return s ? -v : v;
}

/* binary32 -> E4M3, round to nearest even, saturating to +-448 (NaN -> NaN). */
uint8_t oracle_f32_to_e4m3(float x) {
    uint32_t u;
    memcpy(&u, &x, sizeof u);
    uint8_t sign = (uint8_t)((u >> 24) & 0x80);
    if (isnan(x)) return (uint8_t)(sign | 0x7f);
    double a = fabs((double)x);
    if (a >= 448.0) return (uint8_t)(sign | 0x7e);
    if (a == 0.0) return sign;
    int ex;
    frexp(a, &ex);
    int e2 = ex - 1;                                   /* 2^e2 <= a < 2^(e2+1) */
    double q = (e2 < -6) ? ldexp(1.0, -9) : ldexp(1.0, e2 - 3); /* spacing */
    double v = nearbyint(a / q) * q;                   /* nearest, ties even */
    if (v == 0.0) return sign;
    if (v < ldexp(1.0, -6)) return (uint8_t)(sign | (uint8_t)(v / ldexp(1.0, -9)));
    frexp(v, &ex);
    e2 = ex - 1;
    int m = (int)(v / ldexp(1.0, e2 - 3)) - 8;         /* 0..7 */
    return (uint8_t)(sign | ((e2 + 7) << 3) | m);
}

/* 2^ceil(log2 s) for a positive normal s (the ue8m0 power-of-two scale). */
float oracle_pow2_ceil(float s) {
    int ex;
    double m = frexp((double)s, &ex);                  /* s = m * 2^ex */
    if (m == 0.5) return s;                            /* already 2^(ex-1) */
    return (float)ldexp(1.0, ex);
}

/* ---------------------------------------------------------------- layout */

static int check_ids(const int64_t* topk_idx, int T, int K, int E) {
    for (int64_t i = 0; i < (int64_t)T * K; ++i)
        if (topk_idx[i] < -1 || topk_idx[i] >= E) return OR_BAD_EXPERT_ID;
    return OR_OK;
}

/* get_dispatch_layout on one GPU (the RDMA-rank output has no meaning here).
 * num_tokens_per_expert[e] = #{(t,k) : topk_idx[t,k] == e};
 * is_token_in_rank[t,r]   = some unmasked k of token t has expert on rank r;
 * num_tokens_per_rank[r]  = #{t : is_token_in_rank[t,r]}. */
int oracle_layout(const int64_t* topk_idx, int T, int K, int E, int R,
                  int32_t* num_tokens_per_rank, int32_t* num_tokens_per_expert,
                  uint8_t* is_token_in_rank) {
    if (T < 0 || K < 1 || E < 1 || R < 1 || E % R != 0) return OR_INVALID_ARG;
    int st = check_ids(topk_idx, T, K, E);
    if (st) return st;
    int L = E / R;
    memset(num_tokens_per_rank, 0, sizeof(int32_t) * R);
    memset(num_tokens_per_expert, 0, sizeof(int32_t) * E);
    memset(is_token_in_rank, 0, (size_t)T * R);
    for (int t = 0; t < T; ++t)
        for (int k = 0; k < K; ++k) {
            int64_t e = topk_idx[(int64_t)t * K + k];
            if (e < 0) continue;
            num_tokens_per_expert[e] += 1;
            is_token_in_rank[(int64_t)t * R + e / L] = 1;
        }
    for (int t = 0; t < T; ++t)
        for (int r = 0; r < R; ++r) num_tokens_per_rank[r] += is_token_in_rank[(int64_t)t * R + r];
    return OR_OK;
}

/* ------------------------------------------------------------ slot order */

/* Assigns every unmasked (t,k) its received row.  Experts are visited in
 * order e = 0..E-1 (so ranks too, experts being rank-contiguous); within an
 * expert, tokens in ascending t (= source rank, then its local index), then
 * ascending k.  Each expert's segment is padded to a multiple of A.
 * Rows [0, n_al) of the per-row outputs are written; capacity rows are
 * needed (else OR_CAPACITY and nothing is written). */
int oracle_slots(const int64_t* topk_idx, const float* topk_weights, int T, int K, int E, int R,
                 int A, int64_t capacity,
                 int32_t* psum_num_recv_tokens_per_expert,   /* [E] inclusive, aligned */
                 int32_t* num_recv_tokens_per_expert,        /* [E] unaligned */
                 int32_t* dst_buffer_slot_idx,               /* [T,K] */
                 int32_t* recv_src_metadata,                 /* [cap,2] (t,k) */
                 int32_t* recv_topk_idx,                     /* [cap,K] */
                 float* recv_topk_weights,                   /* [cap,K] */
                 int64_t* num_recv_rows) {
    if (T < 0 || K < 1 || E < 1 || R < 1 || E % R != 0 || A < 1) return OR_INVALID_ARG;
    int st = check_ids(topk_idx, T, K, E);
    if (st) return st;
    int L = E / R;
    int64_t* count = calloc((size_t)E, sizeof(int64_t));
    for (int64_t i = 0; i < (int64_t)T * K; ++i)
        if (topk_idx[i] >= 0) count[topk_idx[i]] += 1;
    int64_t total = 0;
    for (int e = 0; e < E; ++e) {
        int64_t aligned = (count[e] + A - 1) / A * A;
        total += aligned;
        psum_num_recv_tokens_per_expert[e] = (int32_t)total;
        num_recv_tokens_per_expert[e] = (int32_t)count[e];
    }
    *num_recv_rows = total;
    free(count);
    if (total > capacity) return OR_CAPACITY;

    for (int64_t i = 0; i < (int64_t)T * K; ++i) dst_buffer_slot_idx[i] = -1;
    for (int64_t row = 0; row < total; ++row) {
        recv_src_metadata[2 * row] = -1;
        recv_src_metadata[2 * row + 1] = -1;
        for (int j = 0; j < K; ++j) {
            recv_topk_idx[row * K + j] = -1;
            recv_topk_weights[row * K + j] = 0.0f;
        }
    }
    int64_t seg_start = 0;
    for (int e = 0; e < E; ++e) {
        int64_t row = seg_start;
        int r_dst = e / L;
        for (int t = 0; t < T; ++t)
            for (int k = 0; k < K; ++k) {
                if (topk_idx[(int64_t)t * K + k] != e) continue;
                dst_buffer_slot_idx[(int64_t)t * K + k] = (int32_t)row;
                recv_src_metadata[2 * row] = t;
                recv_src_metadata[2 * row + 1] = k;
                for (int j = 0; j < K; ++j) {
                    int64_t ej = topk_idx[(int64_t)t * K + j];
                    if (ej >= 0 && ej / L == r_dst) {
                        recv_topk_idx[row * K + j] = (int32_t)(ej - (int64_t)r_dst * L);
                        recv_topk_weights[row * K + j] = topk_weights[(int64_t)t * K + j];
                    }
                }
                row += 1;
            }
        seg_start = psum_num_recv_tokens_per_expert[e];   /* padding rows stay (-1,...) */
    }
    return OR_OK;
}

/* --------------------------------------------------------- quantisation */

/* Quantises one bf16 row of H channels.  quant: OR_QUANT_FP8 or OR_QUANT_INT8;
 * quant_size: channels per scale (128, or H for one scale per token).
 * q receives H bytes (e4m3 codes or int8), scales H / quant_size floats. */
int oracle_quantize_row(const uint16_t* x, int H, int quant, int quant_size, int round_scale,
                        uint8_t* q, float* scales) {
    if (quant != OR_QUANT_FP8 && quant != OR_QUANT_INT8) return OR_INVALID_ARG;
    if (quant_size < 1 || H % quant_size != 0) return OR_INVALID_ARG;
    const float qmax = (quant == OR_QUANT_FP8) ? 448.0f : 127.0f;
    for (int g = 0; g < H / quant_size; ++g) {
        float amax = 0.0f;
        for (int i = 0; i < quant_size; ++i) {
            float v = fabsf(oracle_bf16_to_f32(x[g * quant_size + i]));
            if (v > amax) amax = v;
        }
        if (amax < 1e-4f) amax = 1e-4f;
        float s = amax / qmax;
        if (round_scale) s = oracle_pow2_ceil(s);
        scales[g] = s;
        for (int i = 0; i < quant_size; ++i) {
            float v = oracle_bf16_to_f32(x[g * quant_size + i]) / s;
            /* A group whose maximum is infinite has an infinite scale, and an
             * infinite x then gives inf / inf, a NaN whose sign IEEE 754 leaves
             * open.  Reading: that NaN encodes as the positive FP8 NaN code
             * S.1111.111 with S = 0, and as int8 0. */
            if (isnan(v)) {
                q[g * quant_size + i] = (quant == OR_QUANT_FP8) ? 0x7f : 0;
                continue;
            }
            if (quant == OR_QUANT_FP8) {
                q[g * quant_size + i] = oracle_f32_to_e4m3(v);
            } else {
                float r = nearbyintf(v);
                if (r > 127.0f) r = 127.0f;
                if (r < -127.0f) r = -127.0f;
                q[g * quant_size + i] = (uint8_t)(int8_t)r;
            }
        }
    }
    return OR_OK;
}

/* ------------------------------------------------------------- dispatch */

/* Writes the received rows of the listed tokens: recv_x[dst_buffer_slot_idx[t,k]]
 * = x[t] (bf16 bits) or its quantisation, computed once per source token and
 * copied to each of its rows.  recv_x rows are H*esize bytes (esize 2 for bf16,
 * 1 for fp8/int8); recv_scales rows are H/quant_size floats (quantised only). */
static int dispatch_token(const uint16_t* x, int T, int H, int K, const int32_t* dst_buffer_slot_idx,
                          int quant, int quant_size, int round_scale, int t, uint8_t* recv_x,
                          float* recv_scales, int64_t capacity, uint8_t* q, float* sc) {
    int esize = (quant == OR_QUANT_NONE) ? 2 : 1;
    int ns = (quant == OR_QUANT_NONE) ? 0 : H / quant_size;
    if (t < 0 || t >= T) return OR_INVALID_ARG;
    const uint16_t* xr = x + (int64_t)t * H;
    if (quant != OR_QUANT_NONE) {
        int st = oracle_quantize_row(xr, H, quant, quant_size, round_scale, q, sc);
        if (st) return st;
    }
    for (int k = 0; k < K; ++k) {
        int64_t row = dst_buffer_slot_idx[(int64_t)t * K + k];
        if (row < 0) continue;
        if (row >= capacity) return OR_CAPACITY;
        uint8_t* dst = recv_x + row * H * esize;
        if (quant == OR_QUANT_NONE) {
            memcpy(dst, xr, (size_t)H * 2);
        } else {
            memcpy(dst, q, (size_t)H);
            memcpy(recv_scales + row * ns, sc, sizeof(float) * ns);
        }
    }
    return OR_OK;
}

int oracle_dispatch_rows(const uint16_t* x, int T, int H, int K, const int32_t* dst_buffer_slot_idx,
                         int quant, int quant_size, int round_scale,
                         const int32_t* tokens, int64_t n_tokens,
                         uint8_t* recv_x, float* recv_scales, int64_t capacity) {
    if (H < 1) return OR_INVALID_ARG;
    int ns = (quant == OR_QUANT_NONE) ? 0 : H / quant_size;
    int st = OR_OK;
#pragma omp parallel reduction(max : st)
    {
        uint8_t* q = malloc((size_t)H);
        float* sc = malloc(sizeof(float) * (size_t)(ns > 0 ? ns : 1));
#pragma omp for schedule(dynamic, 4)
        for (int64_t i = 0; i < n_tokens; ++i) {
            int s = dispatch_token(x, T, H, K, dst_buffer_slot_idx, quant, quant_size, round_scale, tokens[i],
                                   recv_x, recv_scales, capacity, q, sc);
            if (s > st) st = s;
        }
        free(q);
        free(sc);
    }
    return st;
}

/* -------------------------------------------------------------- combine */

/* out[i] = bf16( fma chain over k = 0..K-1 with dst_buffer_slot_idx[t,k] >= 0 of
 * topk_weights[t,k] * y[slot] ), starting from +0.0f, for t = tokens[i].
 * out is [n_tokens, H] (compact, in list order). */
static int combine_token(const uint16_t* y, int64_t y_rows, int H, int T, int K,
                         const int32_t* dst_buffer_slot_idx, const float* topk_weights, int t, uint16_t* out_row) {
    if (t < 0 || t >= T) return OR_INVALID_ARG;
    for (int h = 0; h < H; ++h) {
        float acc = 0.0f;
        for (int k = 0; k < K; ++k) {
            int64_t row = dst_buffer_slot_idx[(int64_t)t * K + k];
            if (row < 0) continue;
            if (row >= y_rows) return OR_CAPACITY;
            acc = fmaf(topk_weights[(int64_t)t * K + k], oracle_bf16_to_f32(y[row * H + h]), acc);
        }
        out_row[h] = oracle_f32_to_bf16(acc);
    }
    return OR_OK;
}

int oracle_combine_rows(const uint16_t* y, int64_t y_rows, int H, int T, int K,
                        const int32_t* dst_buffer_slot_idx, const float* topk_weights,
                        const int32_t* tokens, int64_t n_tokens, uint16_t* out) {
    int st = OR_OK;
#pragma omp parallel for schedule(dynamic, 4) reduction(max : st)
    for (int64_t i = 0; i < n_tokens; ++i) {
        int s = combine_token(y, y_rows, H, T, K, dst_buffer_slot_idx, topk_weights, tokens[i], out + i * H);
        if (s > st) st = s;
    }
    return st;
}

/* ------------------------------------------------------- long sequences */

/* Token list of round j of the "ant moving home" schedule: each of the R
 * source ranks owns T/R consecutive tokens and sends its j-th block of
 * (T/R)/rounds tokens in round j.  Returns the number of tokens written. */
int64_t oracle_round_tokens(int T, int R, int rounds, int j, int32_t* tokens) {
    if (R < 1 || rounds < 1 || T % R != 0 || (T / R) % rounds != 0 || j < 0 || j >= rounds)
        return -1;
    int tpr = T / R, per_round = tpr / rounds;
    int64_t n = 0;
    for (int r = 0; r < R; ++r)
        for (int i = 0; i < per_round; ++i) tokens[n++] = r * tpr + j * per_round + i;
    return n;
}

/* ------------------------------------------------- array forms (for tests) */

void oracle_f32_to_e4m3_n(const float* x, int64_t n, uint8_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_f32_to_e4m3(x[i]);
}

void oracle_f32_to_bf16_n(const float* x, int64_t n, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_f32_to_bf16(x[i]);
}

void oracle_e4m3_to_f64_n(const uint8_t* c, int64_t n, double* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_e4m3_to_f64(c[i]);
}

/* -------------------------------------------- low-latency (fixed capacity) */

/* The low-latency receive layout of the decode path (comparative analysis,
 * section 6.3: a buffer of [num_local_experts, num_ranks *
 * num_max_dispatch_tokens_per_rank, hidden] per rank; on one GPU the ranks'
 * buffers stack to [E, R*M, H]).  The entry (t,k) routed to expert e from
 * source rank r = t / (T/R) goes to row e*R*M + r*M + p, where p counts the
 * earlier entries (t', k') of the same source rank and expert in (t, k) order.
 * recv_count[e] = entries of expert e; layout_range[e*R + r] = (r*M << 32) |
 * (entries of expert e from rank r).  Rows not used keep their content.
 * Returns OR_CAPACITY if some (expert, source rank) has more than M entries. */
int oracle_ll_slots(const int64_t* topk_idx, const float* topk_weights, int T, int K, int E, int R, int M,
                    int32_t* dst_buffer_slot_idx, int32_t* recv_count, int64_t* layout_range,
                    int32_t* recv_src_metadata, int32_t* recv_topk_idx, float* recv_topk_weights) {
    if (T < 0 || K < 1 || E < 1 || R < 1 || E % R != 0 || T % R != 0 || M < 1) return OR_INVALID_ARG;
    int st = check_ids(topk_idx, T, K, E);
    if (st) return st;
    int L = E / R, tpr = T / R;
    for (int64_t i = 0; i < (int64_t)T * K; ++i) dst_buffer_slot_idx[i] = -1;
    for (int e = 0; e < E; ++e) recv_count[e] = 0;
    for (int e = 0; e < E; ++e) {
        int r_dst = e / L;
        for (int r = 0; r < R; ++r) {
            int64_t p = 0;
            for (int t = r * tpr; t < (r + 1) * tpr; ++t)
                for (int k = 0; k < K; ++k) {
                    if (topk_idx[(int64_t)t * K + k] != e) continue;
                    if (p >= M) return OR_CAPACITY;
                    int64_t row = ((int64_t)e * R + r) * M + p;
                    dst_buffer_slot_idx[(int64_t)t * K + k] = (int32_t)row;
                    recv_src_metadata[2 * row] = t;
                    recv_src_metadata[2 * row + 1] = k;
                    for (int j = 0; j < K; ++j) {
                        int64_t ej = topk_idx[(int64_t)t * K + j];
                        int here = ej >= 0 && ej / L == r_dst;
                        recv_topk_idx[row * K + j] = here ? (int32_t)(ej - (int64_t)r_dst * L) : -1;
                        recv_topk_weights[row * K + j] = here ? topk_weights[(int64_t)t * K + j] : 0.0f;
                    }
                    p += 1;
                }
            layout_range[(int64_t)e * R + r] = ((int64_t)r * M << 32) | p;
            recv_count[e] += (int32_t)p;
        }
    }
    return OR_OK;
}

/* ------------------------------------------ combine of quantised outputs */

/* As oracle_combine_rows, for expert outputs given as FP8 e4m3 / int8 codes
 * with one fp32 scale per quant_size channels (the combine-side quantisation
 * of guide v2.1): each value is decode(code) * scale (fp32 product) before the
 * fma chain.  quant OR_QUANT_NONE reads bf16 y.  If `shared` is given (bf16
 * [T,H], a shared expert's output), the accumulator starts from shared[t]
 * instead of +0. */
static int combine_token_q(const void* y, const float* y_scales, int quant, int quant_size, int64_t y_rows,
                           int H, int T, int K, const int32_t* dst_buffer_slot_idx, const float* topk_weights,
                           const uint16_t* shared, int t, uint16_t* out_row) {
    int ns = quant == OR_QUANT_NONE ? 0 : H / quant_size;
    if (t < 0 || t >= T) return OR_INVALID_ARG;
    for (int h = 0; h < H; ++h) {
        float acc = shared ? oracle_bf16_to_f32(shared[(int64_t)t * H + h]) : 0.0f;
        for (int k = 0; k < K; ++k) {
            int64_t row = dst_buffer_slot_idx[(int64_t)t * K + k];
            if (row < 0) continue;
            if (row >= y_rows) return OR_CAPACITY;
            float v;
            if (quant == OR_QUANT_NONE) {
                v = oracle_bf16_to_f32(((const uint16_t*)y)[row * H + h]);
            } else {
                uint8_t c = ((const uint8_t*)y)[row * H + h];
                float d = quant == OR_QUANT_FP8 ? (float)oracle_e4m3_to_f64(c) : (float)(int8_t)c;
                v = d * y_scales[row * ns + h / quant_size];
            }
            acc = fmaf(topk_weights[(int64_t)t * K + k], v, acc);
        }
        out_row[h] = oracle_f32_to_bf16(acc);
    }
    return OR_OK;
}

int oracle_combine_rows_q(const void* y, const float* y_scales, int quant, int quant_size, int64_t y_rows,
                          int H, int T, int K, const int32_t* dst_buffer_slot_idx, const float* topk_weights,
                          const uint16_t* shared, const int32_t* tokens, int64_t n_tokens, uint16_t* out) {
    if (quant != OR_QUANT_NONE && (quant_size < 1 || H % quant_size != 0)) return OR_INVALID_ARG;
    int st = OR_OK;
#pragma omp parallel for schedule(dynamic, 4) reduction(max : st)
    for (int64_t i = 0; i < n_tokens; ++i) {
        int s = combine_token_q(y, y_scales, quant, quant_size, y_rows, H, T, K, dst_buffer_slot_idx,
                                topk_weights, shared, tokens[i], out + i * H);
        if (s > st) st = s;
    }
    return st;
}

/* ------------------------------------------------ MXFP4 and UE8M0 scales */

#define OR_QUANT_MXFP4 3

/* OCP FP4 E2M1: 1 sign, 2 exponent bits (bias 1), 1 mantissa bit; exponent
 * field 0 is subnormal (m * 0.5); no infinities or NaN; the largest value is
 * 1.5 * 2^2 = 6. */
double oracle_e2m1_to_f64(uint8_t c) {
    int s = (c >> 3) & 1, e = (c >> 1) & 3, m = c & 1;
    double v = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -v : v;
}

/* binary32 -> E2M1, round to nearest even, saturating to +-6 (finite input). */
uint8_t oracle_f32_to_e2m1(float x) {
    uint8_t sign = signbit(x) ? 8 : 0;
    double a = fabs((double)x);
    if (a >= 6.0) return (uint8_t)(sign | 7);
    if (a == 0.0) return sign;
    int ex;
    frexp(a, &ex);
    int e2 = ex - 1;                                   /* 2^e2 <= a < 2^(e2+1) */
    double q = (e2 < 0) ? 0.5 : ldexp(1.0, e2 - 1);    /* spacing in the binade */
    double v = nearbyint(a / q) * q;                   /* nearest, ties even */
    if (v == 0.0) return sign;
    if (v < 1.0) return (uint8_t)(sign | 1);           /* 0.5: subnormal */
    frexp(v, &ex);
    e2 = ex - 1;
    int m = (int)((v / ldexp(1.0, e2) - 1.0) * 2.0);   /* 0 or 1 */
    return (uint8_t)(sign | ((e2 + 1) << 1) | m);
}

/* Quantises one bf16 row with the scale encodings of the low-latency API:
 *  - OR_QUANT_FP8 / OR_QUANT_INT8 as oracle_quantize_row; with scale_ue8m0 the
 *    (power-of-two, round_scale required) scales are stored as one UE8M0 byte
 *    each: the biased exponent 127 + log2(s) (use_ue8m0 of guide v2.1);
 *  - OR_QUANT_MXFP4 (quant_size 32, guide v2.1 section 1.3.3): per group of 32
 *    the OCP MX shared scale X = 2^(floor(log2 amax) - 2) (2 = the largest
 *    exponent of E2M1; amax floored at 1e-4), elements E2M1(x / X), two per
 *    byte (even element in the low nibble), scale stored as a UE8M0 byte.
 * q receives the row's code bytes (H, or H/2 for MXFP4); scales receives
 * H/quant_size floats or bytes. */
int oracle_quantize_row_mx(const uint16_t* x, int H, int quant, int quant_size, int round_scale,
                           int scale_ue8m0, uint8_t* q, void* scales) {
    if (quant == OR_QUANT_MXFP4) {
        if (quant_size != 32 || H % 32 != 0) return OR_INVALID_ARG;
        for (int g = 0; g < H / 32; ++g) {
            float amax = 0.0f;
            for (int i = 0; i < 32; ++i) {
                float v = fabsf(oracle_bf16_to_f32(x[g * 32 + i]));
                if (v > amax) amax = v;
            }
            if (amax < 1e-4f) amax = 1e-4f;
            int ex;
            frexp((double)amax, &ex);
            int E = (ex - 1) - 2;                        /* floor(log2 amax) - 2 */
            float s = (float)ldexp(1.0, E);
            ((uint8_t*)scales)[g] = (uint8_t)(E + 127);
            for (int i = 0; i < 32; i += 2) {
                uint8_t lo = oracle_f32_to_e2m1(oracle_bf16_to_f32(x[g * 32 + i]) / s);
                uint8_t hi = oracle_f32_to_e2m1(oracle_bf16_to_f32(x[g * 32 + i + 1]) / s);
                q[(g * 32 + i) / 2] = (uint8_t)(lo | (hi << 4));
            }
        }
        return OR_OK;
    }
    if (!scale_ue8m0) return oracle_quantize_row(x, H, quant, quant_size, round_scale, q, (float*)scales);
    if (!round_scale) return OR_INVALID_ARG;             /* bytes hold powers of two only */
    if (quant_size < 1 || H % quant_size != 0) return OR_INVALID_ARG;
    float* f = malloc(sizeof(float) * (size_t)(H / quant_size));
    int st = oracle_quantize_row(x, H, quant, quant_size, round_scale, q, f);
    for (int g = 0; st == OR_OK && g < H / quant_size; ++g) {
        int ex;
        double m = frexp((double)f[g], &ex);              /* f = 0.5 * 2^ex exactly */
        if (m != 0.5) { st = OR_INVALID_ARG; break; }
        ((uint8_t*)scales)[g] = (uint8_t)((ex - 1) + 127);
    }
    free(f);
    return st;
}

/* oracle_dispatch_rows for every quantisation, including MXFP4 and UE8M0
 * scale bytes.  Row bytes: 2H (bf16), H (FP8 / int8), H/2 (MXFP4); scale
 * bytes per row: H/quant_size times 4 (fp32) or 1 (UE8M0, always for MXFP4). */
static int dispatch_token_mx(const uint16_t* x, int T, int H, int K, const int32_t* dst_buffer_slot_idx,
                             int quant, int quant_size, int round_scale, int scale_ue8m0, int t, uint8_t* recv_x,
                             uint8_t* recv_scales, int64_t capacity, uint8_t* q, uint8_t* sc) {
    int ue8 = (quant == OR_QUANT_MXFP4) || scale_ue8m0;
    int64_t row_bytes = quant == OR_QUANT_NONE ? 2 * (int64_t)H : quant == OR_QUANT_MXFP4 ? H / 2 : H;
    int ns = quant == OR_QUANT_NONE ? 0 : H / quant_size;
    int64_t scale_bytes = (int64_t)ns * (ue8 ? 1 : 4);
    if (t < 0 || t >= T) return OR_INVALID_ARG;
    const uint16_t* xr = x + (int64_t)t * H;
    if (quant != OR_QUANT_NONE) {
        int st = oracle_quantize_row_mx(xr, H, quant, quant_size, round_scale, scale_ue8m0, q, sc);
        if (st) return st;
    }
    for (int k = 0; k < K; ++k) {
        int64_t row = dst_buffer_slot_idx[(int64_t)t * K + k];
        if (row < 0) continue;
        if (row >= capacity) return OR_CAPACITY;
        if (quant == OR_QUANT_NONE) {
            memcpy(recv_x + row * row_bytes, xr, (size_t)row_bytes);
        } else {
            memcpy(recv_x + row * row_bytes, q, (size_t)row_bytes);
            memcpy(recv_scales + row * scale_bytes, sc, (size_t)scale_bytes);
        }
    }
    return OR_OK;
}

int oracle_dispatch_rows_mx(const uint16_t* x, int T, int H, int K, const int32_t* dst_buffer_slot_idx,
                            int quant, int quant_size, int round_scale, int scale_ue8m0,
                            const int32_t* tokens, int64_t n_tokens, uint8_t* recv_x, uint8_t* recv_scales,
                            int64_t capacity) {
    if (H < 1) return OR_INVALID_ARG;
    int ue8 = (quant == OR_QUANT_MXFP4) || scale_ue8m0;
    int ns = quant == OR_QUANT_NONE ? 0 : H / quant_size;
    int64_t scale_bytes = (int64_t)ns * (ue8 ? 1 : 4);
    int st = OR_OK;
#pragma omp parallel reduction(max : st)
    {
        uint8_t* q = malloc((size_t)H);
        uint8_t* sc = malloc((size_t)(scale_bytes > 0 ? scale_bytes : 1));
#pragma omp for schedule(dynamic, 4)
        for (int64_t i = 0; i < n_tokens; ++i) {
            int s = dispatch_token_mx(x, T, H, K, dst_buffer_slot_idx, quant, quant_size, round_scale, scale_ue8m0,
                                      tokens[i], recv_x, recv_scales, capacity, q, sc);
            if (s > st) st = s;
        }
        free(q);
        free(sc);
    }
    return st;
}

/* ---------------------------------------------- group-limited gating */

#define OR_NONFINITE 4

/* Group-limited gating, the routing that produces topk_idx / topk_weights
 * upstream of dispatch ("DeepEP V1 vs V2 comparative analysis", section 8.1,
 * DeepSeek-V3 group-limited gating: 256 experts in 32 groups of 8, each token
 * keeps its top-4 groups, then the top-2 experts inside each kept group, top-8
 * experts in all).  logits: fp32 [T, E]; the E experts form n_group groups of
 * E / n_group consecutive ids; K = topk_group * per_group entries per token.
 *
 * Readings where the page is silent (one each):
 *  - an expert's affinity is its router logit; of two experts the one with
 *    the larger logit ranks first, and of two equal logits the lower id;
 *  - a group's score is the fp32 sum of its per_group largest logits, added
 *    from the largest down (so the kept groups are those whose picks add up
 *    highest); of two equal scores the lower group id ranks first;
 *  - the K entries of a token are listed by logit, largest first, equal
 *    logits by lower id;
 *  - topk_weights[t] is the softmax over the K selected logits, computed in
 *    binary64 and rounded to binary32.
 * Logits must be finite: a NaN or infinite logit returns OR_NONFINITE.
 * Steps, in the page's order: per group its best experts and score; the
 * topk_group best groups; the per_group best experts of each kept group;
 * order and weights. */
int oracle_group_limited_gating(const float* logits, int T, int E, int n_group, int topk_group, int per_group,
                                int64_t* topk_idx, float* topk_weights) {
    if (T < 0 || E < 1 || n_group < 1 || E % n_group != 0) return OR_INVALID_ARG;
    const int S = E / n_group;
    if (topk_group < 1 || topk_group > n_group || per_group < 1 || per_group > S) return OR_INVALID_ARG;
    const int K = topk_group * per_group;
    int* pick = malloc(sizeof(int) * (size_t)E);         /* [n_group][per_group] best experts per group */
    float* score = malloc(sizeof(float) * (size_t)n_group);
    char* taken = malloc((size_t)(E > n_group ? E : n_group));
    int* sel = malloc(sizeof(int) * (size_t)K);
    int status = OR_OK;
    for (int t = 0; t < T && status == OR_OK; ++t) {
        const float* l = logits + (int64_t)t * E;
        for (int e = 0; e < E; ++e)
            if (!isfinite(l[e])) status = OR_NONFINITE;
        if (status) break;
        /* 1. every group's per_group best experts, and its score */
        memset(taken, 0, (size_t)E);
        for (int g = 0; g < n_group; ++g) {
            for (int j = 0; j < per_group; ++j) {
                int best = -1;
                for (int e = g * S; e < (g + 1) * S; ++e)
                    if (!taken[e] && (best < 0 || l[e] > l[best])) best = e;
                taken[best] = 1;
                pick[g * per_group + j] = best;
            }
            float sc = l[pick[g * per_group]];
            for (int j = 1; j < per_group; ++j) sc = sc + l[pick[g * per_group + j]];
            score[g] = sc;
        }
        /* 2. the topk_group best groups; 3. their picks */
        memset(taken, 0, (size_t)n_group);
        int n = 0;
        for (int j = 0; j < topk_group; ++j) {
            int best = -1;
            for (int g = 0; g < n_group; ++g)
                if (!taken[g] && (best < 0 || score[g] > score[best])) best = g;
            taken[best] = 1;
            for (int i = 0; i < per_group; ++i) sel[n++] = pick[best * per_group + i];
        }
        /* 4. order: larger logit first, equal logits by lower id (insertion sort) */
        for (int i = 1; i < K; ++i) {
            int v = sel[i], j = i - 1;
            while (j >= 0 && (l[sel[j]] < l[v] || (l[sel[j]] == l[v] && sel[j] > v))) {
                sel[j + 1] = sel[j];
                --j;
            }
            sel[j + 1] = v;
        }
        /* 5. softmax over the K selected logits in binary64, rounded to binary32 */
        const double m = (double)l[sel[0]];
        double sum = 0.0;
        for (int k = 0; k < K; ++k) sum += exp((double)l[sel[k]] - m);
        for (int k = 0; k < K; ++k) {
            topk_idx[(int64_t)t * K + k] = sel[k];
            topk_weights[(int64_t)t * K + k] = (float)(exp((double)l[sel[k]] - m) / sum);
        }
    }
    free(pick);
    free(score);
    free(taken);
    free(sel);
    return status;
}

/* ------------------------------------------------------------- threads */

#ifdef _OPENMP
#include <omp.h>
#endif

/* Threads the row functions use: 1 in the plain build; in the OpenMP build,
 * n > 0 sets the count and the current count is returned. */
int oracle_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
    return omp_get_max_threads();
#else
    (void)n;
    return 1;
#endif
}
