/*
 * CPU oracle for MoE layout, FP8 / BF16 dispatch and BF16 combine.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the package smoke check and the
 * benchmark's CPU-baseline leg load this file's library.  It shares no code,
 * header, table or constant with the CUDA path, and the CUDA path never calls it.
 *
 * What is computed, and where the DeepEP pages fix it:
 *   - dispatch sends each token to its gated experts and combine merges the
 *     experts' outputs back, accumulating (DeepEP GitHub-issue mirror,
 *     "Technical Overview"; brainleap "Day2 DeepEP", "DeepEP是什么" and the
 *     combine paragraph of "All-to-All通信");
 *   - FP8 dispatch, BF16 combine (same pages, benchmark settings);
 *   - the host reads a GPU-made receive count (brainleap "Day2 DeepEP", section
 *     "All-to-All通信", the figure caption on the host waiting for receive counts).
 * Everything finer (1x128 scale blocks, amax/448 scales, RNE + saturation,
 * ascending-token stable order, fixed-order fp32 combine) is this library's
 * reading of the benchmark spec; each function states the reading it takes.
 *
 * Parity status: the layout is pinned by brute force and invariants, the
 * e4m3 encoder/decoder by torch's float8_e4m3fn and the OCP FP8 definition,
 * dispatch by per-block closed forms, combine by closed forms and an exact
 * fp64 error bound.  No function here is "parity unpinned".
 *
 * Build: gcc -O2 -ffp-contract=off -fopenmp -shared -fPIC (x86-64 SSE floats,
 * so every float operation below is one IEEE binary32 operation, round to
 * nearest even, and no multiply-add is fused).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Error flags returned by the oracle (its own numbering). */
#define ORACLE_FLAG_RANGE 1    /* an expert id < -1 or >= E was seen; treated as masked */
#define ORACLE_FLAG_CAPACITY 2 /* a padded expert received more than `capacity` copies */

/* ---------------------------------------------------------------- threads */

int oracle_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
    return omp_get_max_threads();
#else
    (void)n;
    return 1;
#endif
}

/* ------------------------------------------------------------ BF16 <-> fp32 */

/* BF16 is the top half of a binary32; widening is exact. */
static float bf16_to_f32(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* Round a binary32 to BF16, nearest with ties to even.  Written from the
 * definition: keep the top 16 bits, look at the 16 dropped bits, round up if
 * they exceed half an ulp, or equal half and the kept value is odd. */
uint16_t oracle_bf16_from_f32(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu) != 0)
        return (uint16_t)((u >> 16) | 0x0040u); /* quiet NaN */
    uint32_t kept = u >> 16;
    uint32_t dropped = u & 0xFFFFu;
    if (dropped > 0x8000u || (dropped == 0x8000u && (kept & 1u))) kept += 1u;
    return (uint16_t)kept;
}

float oracle_bf16_to_f32(uint16_t b) { return bf16_to_f32(b); }

/* ------------------------------------------------------------- FP8 e4m3 */

/* Decode an OCP FP8 E4M3 ("fn" variant) code: sign, 4-bit exponent with bias 7,
 * 3-bit mantissa; exponent field 0 is subnormal (m * 2^-9); S.1111.111 is NaN;
 * there is no infinity. */
float oracle_e4m3_decode(uint8_t c) {
    int s = c >> 7, ex = (c >> 3) & 0xF, m = c & 7;
    double v;
    if (ex == 15 && m == 7) return s ? -NAN : NAN;
    if (ex == 0) v = ldexp((double)m, -9);
    else v = ldexp(1.0 + m / 8.0, ex - 7);
    return (float)(s ? -v : v);
}

/* Encode a binary32 as E4M3, rounding to nearest (ties to even) and saturating
 * finite overflow (and infinities) to +-448; NaN -> S.1111.111; the sign of
 * zero is kept.  The value is scaled by a power of two into the integer grid
 * of its binade and rounded there with rint() under the default
 * round-to-nearest-even mode; all steps are exact in double. */
uint8_t oracle_e4m3_encode(float f) {
    uint8_t sign = signbit(f) ? 0x80 : 0x00;
    if (isnan(f)) return sign | 0x7F;
    double a = fabs((double)f);
    if (a >= 448.0) return sign | 0x7E; /* includes +inf: saturate */
    if (a < ldexp(1.0, -6)) {
        /* subnormal grid: steps of 2^-9; 8 steps is the smallest normal */
        double q = rint(ldexp(a, 9));
        return sign | (uint8_t)q; /* q == 8 encodes 2^-6 as exponent 1, mantissa 0 */
    }
    int e2;
    frexp(a, &e2);      /* a = fr * 2^e2, fr in [0.5, 1) */
    int ex = e2 - 1;    /* a in [2^ex, 2^(ex+1)) */
    double q = rint(ldexp(a, 3 - ex)); /* in [8, 16] */
    if (q == 16.0) { q = 8.0; ex += 1; }
    int field = ex + 7;
    if (field > 15 || (field == 15 && q - 8.0 > 6.0)) return sign | 0x7E;
    return sign | (uint8_t)((field << 3) | (int)(q - 8.0));
}

/* Element-wise encode / decode over arrays (used by the codec sweeps). */
void oracle_e4m3_encode_array(const float *v, int64_t n, uint8_t *out) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_e4m3_encode(v[i]);
}

void oracle_e4m3_decode_array(const uint8_t *c, int64_t n, float *out) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_e4m3_decode(c[i]);
}

void oracle_bf16_from_f32_array(const float *v, int64_t n, uint16_t *out) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_bf16_from_f32(v[i]);
}

/* ---------------------------------------------------------------- layout */

/*
 * The layout: per-expert counts, their exclusive prefix sum, and the stable
 * receive position of every (token, slot) pair.  Reading: positions are
 * assigned by one walk over t = 0..N-1, j = 0..k-1, so copies of an expert are
 * in ascending token order (ascending slot for a duplicated expert).  A rank
 * owns experts [r*E/R, (r+1)*E/R).  Id -1 means "no copy"; other ids outside
 * [0, E) are flagged and also make no copy.  capacity == 0: compact receive
 * rows, base(e) = expert_offset[e], recv_src has N*k entries.  capacity > 0:
 * padded rows, base(e) = e*capacity, recv_src has E*capacity entries, and
 * copies past the capacity are dropped (dst_pos = -1) and flagged.
 * recv_src[row] = t*k + j of the copy in that row, -1 for an unused row.
 * tokens_per_expert and max_count count every routed copy, dropped or not.
 */
int oracle_get_layout(const int32_t *topk_idx, int64_t N, int k, int E, int R, int capacity,
                      int32_t *tokens_per_expert, int32_t *tokens_per_rank,
                      uint8_t *is_token_in_rank, int32_t *expert_offset, int32_t *max_count,
                      int32_t *dst_pos, int32_t *recv_src) {
    int flags = 0;
    int per_rank = E / R;
    for (int e = 0; e < E; ++e) tokens_per_expert[e] = 0;
    for (int r = 0; r < R; ++r) tokens_per_rank[r] = 0;
    memset(is_token_in_rank, 0, (size_t)N * (size_t)R);

    /* counts */
    for (int64_t t = 0; t < N; ++t)
        for (int j = 0; j < k; ++j) {
            int32_t e = topk_idx[t * k + j];
            if (e == -1) continue;
            if (e < -1 || e >= E) { flags |= ORACLE_FLAG_RANGE; continue; }
            tokens_per_expert[e] += 1;
            is_token_in_rank[t * R + e / per_rank] = 1;
        }
    for (int64_t t = 0; t < N; ++t)
        for (int r = 0; r < R; ++r) tokens_per_rank[r] += is_token_in_rank[t * R + r];

    /* exclusive prefix sum in expert order, and the largest count */
    expert_offset[0] = 0;
    int32_t mx = 0;
    for (int e = 0; e < E; ++e) {
        expert_offset[e + 1] = expert_offset[e] + tokens_per_expert[e];
        if (tokens_per_expert[e] > mx) mx = tokens_per_expert[e];
    }
    *max_count = mx;

    /* stable positions */
    int64_t rows = capacity > 0 ? (int64_t)E * capacity : N * k;
    for (int64_t i = 0; i < rows; ++i) recv_src[i] = -1;
    int32_t seen[E > 0 ? E : 1];
    for (int e = 0; e < E; ++e) seen[e] = 0;
    for (int64_t t = 0; t < N; ++t)
        for (int j = 0; j < k; ++j) {
            int32_t e = topk_idx[t * k + j];
            int64_t p = t * k + j;
            if (e < 0 || e >= E) { dst_pos[p] = -1; continue; }
            int32_t slot = seen[e]++;
            int64_t row;
            if (capacity > 0) {
                if (slot >= capacity) { dst_pos[p] = -1; flags |= ORACLE_FLAG_CAPACITY; continue; }
                row = (int64_t)e * capacity + slot;
            } else {
                row = expert_offset[e] + slot;
            }
            dst_pos[p] = (int32_t)row;
            recv_src[row] = (int32_t)p;
        }
    return flags;
}

/*
 * The per-rank (deduplicated) layout: a token sends one copy to each logical
 * rank that hosts at least one of its experts, instead of one per expert.
 * Reading: this is the DeepEP normal-mode behaviour behind "is_token_in_rank"
 * (one transfer per token and destination rank, the rank then serves its
 * local experts); the pages only name dispatch to experts and the host
 * waiting on receive counts.  Rows of rank r hold its tokens in ascending
 * token order.  rank_dst[t, j] = that row for the FIRST slot j of token t
 * whose expert lies on rank r = e / (E/R); later slots on the same rank, and
 * masked or out-of-range slots, get -1.  recv_token[row] = t (or -1).
 * capacity == 0: compact rows, rank r at [rank_offset[r], rank_offset[r+1]);
 * capacity > 0: rows [r*capacity, ...), copies past the capacity dropped and
 * flagged.  tokens_per_rank[r] = distinct tokens reaching rank r.
 */
int oracle_get_rank_layout(const int32_t *topk_idx, int64_t N, int k, int E, int R, int capacity,
                           int32_t *tokens_per_rank, int32_t *rank_offset, int32_t *max_count,
                           int32_t *rank_dst, int32_t *recv_token) {
    int flags = 0;
    int per_rank = E / R;
    int32_t first[R > 0 ? R : 1];   /* per rank: slot of its first copy in the current token */
    for (int r = 0; r < R; ++r) tokens_per_rank[r] = 0;

    /* counts: one per (token, rank) */
    for (int64_t t = 0; t < N; ++t) {
        for (int r = 0; r < R; ++r) first[r] = -1;
        for (int j = 0; j < k; ++j) {
            int32_t e = topk_idx[t * k + j];
            if (e == -1) continue;
            if (e < -1 || e >= E) { flags |= ORACLE_FLAG_RANGE; continue; }
            int r = e / per_rank;
            if (first[r] >= 0) continue;
            first[r] = j;
            tokens_per_rank[r] += 1;
        }
    }
    rank_offset[0] = 0;
    int32_t mx = 0;
    for (int r = 0; r < R; ++r) {
        rank_offset[r + 1] = rank_offset[r] + tokens_per_rank[r];
        if (tokens_per_rank[r] > mx) mx = tokens_per_rank[r];
    }
    *max_count = mx;

    /* rows, in token order */
    int64_t rows = capacity > 0 ? (int64_t)R * capacity : N * k;
    for (int64_t i = 0; i < rows; ++i) recv_token[i] = -1;
    int32_t seen[R > 0 ? R : 1];
    for (int r = 0; r < R; ++r) seen[r] = 0;
    for (int64_t t = 0; t < N; ++t) {
        for (int r = 0; r < R; ++r) first[r] = -1;
        for (int j = 0; j < k; ++j) {
            int32_t e = topk_idx[t * k + j];
            int64_t p = t * k + j;
            rank_dst[p] = -1;
            if (e < 0 || e >= E) continue;
            int r = e / per_rank;
            if (first[r] >= 0) continue;
            first[r] = j;
            int32_t slot = seen[r]++;
            int64_t row;
            if (capacity > 0) {
                if (slot >= capacity) { flags |= ORACLE_FLAG_CAPACITY; continue; }
                row = (int64_t)r * capacity + slot;
            } else {
                row = rank_offset[r] + slot;
            }
            rank_dst[p] = (int32_t)row;
            recv_token[row] = (int32_t)t;
        }
    }
    return flags;
}

/* -------------------------------------------------------------- dispatch */

/*
 * FP8 dispatch.  Reading: per token and per block of 128 consecutive hidden
 * values, amax = max |x|, amax_c = max(amax, 1e-4), scale = amax_c / 448 and
 * inv = 448 / amax_c (each one correctly rounded binary32 division),
 * q = e4m3(x * inv) (one binary32 product, then the encoder above).  The same
 * codes and scale go to each of the token's k receive rows dst_pos[t, j]
 * (rows with dst_pos < 0 are skipped).  recv_scale is [rows, H/128].
 */
void oracle_dispatch_fp8(const uint16_t *x, int64_t N, int H, int k, const int32_t *dst_pos,
                         uint8_t *recv_x, float *recv_scale) {
    int nb = H / 128;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < N; ++t) {
        uint8_t q[H > 0 ? H : 1];
        float sc[nb > 0 ? nb : 1];
        for (int b = 0; b < nb; ++b) {
            float amax = 0.0f;
            for (int i = 0; i < 128; ++i) {
                float v = fabsf(bf16_to_f32(x[t * H + b * 128 + i]));
                if (v > amax) amax = v;
            }
            float amax_c = amax > 1e-4f ? amax : 1e-4f;
            float scale = amax_c / 448.0f;
            float inv = 448.0f / amax_c;
            for (int i = 0; i < 128; ++i) {
                float v = bf16_to_f32(x[t * H + b * 128 + i]);
                float prod = v * inv;
                q[b * 128 + i] = oracle_e4m3_encode(prod);
            }
            sc[b] = scale;
        }
        for (int j = 0; j < k; ++j) {
            int32_t row = dst_pos[t * k + j];
            if (row < 0) continue;
            memcpy(recv_x + (int64_t)row * H, q, (size_t)H);
            memcpy(recv_scale + (int64_t)row * nb, sc, sizeof(float) * (size_t)nb);
        }
    }
}

/*
 * FP8 dispatch with power-of-two (UE8M0) scales.  Reading: the variant of the
 * dispatch above whose per-block scale is restricted to a power of two, as an
 * 8-bit exponent-only (UE8M0) scale format can hold: scale = 2^e for the
 * smallest integer e with 448 * 2^e >= amax_c (the block's largest value then
 * maps to at most 448, so nothing saturates), inv = 2^-e, q = e4m3(x * inv).
 * The scale is stored as the binary32 value 2^e (its biased exponent field is
 * the UE8M0 code).  e is found by the plain search below: 448 * 2^e is exact
 * in binary32 over the range searched, so each comparison is exact.
 */
static float pow2_scale_exponent_search(float amax_c, int *e_out) {
    int e = -40;                          /* 448 * 2^-40 < 1e-4 <= amax_c */
    while (ldexpf(448.0f, e) < amax_c) ++e;
    *e_out = e;
    return ldexpf(1.0f, e);
}

void oracle_dispatch_fp8_pow2(const uint16_t *x, int64_t N, int H, int k, const int32_t *dst_pos,
                              uint8_t *recv_x, float *recv_scale) {
    int nb = H / 128;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < N; ++t) {
        uint8_t q[H > 0 ? H : 1];
        float sc[nb > 0 ? nb : 1];
        for (int b = 0; b < nb; ++b) {
            float amax = 0.0f;
            for (int i = 0; i < 128; ++i) {
                float v = fabsf(bf16_to_f32(x[t * H + b * 128 + i]));
                if (v > amax) amax = v;
            }
            float amax_c = amax > 1e-4f ? amax : 1e-4f;
            int e;
            float scale = pow2_scale_exponent_search(amax_c, &e);
            float inv = ldexpf(1.0f, -e);
            for (int i = 0; i < 128; ++i) {
                float v = bf16_to_f32(x[t * H + b * 128 + i]);
                float prod = v * inv;
                q[b * 128 + i] = oracle_e4m3_encode(prod);
            }
            sc[b] = scale;
        }
        for (int j = 0; j < k; ++j) {
            int32_t row = dst_pos[t * k + j];
            if (row < 0) continue;
            memcpy(recv_x + (int64_t)row * H, q, (size_t)H);
            memcpy(recv_scale + (int64_t)row * nb, sc, sizeof(float) * (size_t)nb);
        }
    }
}

/* BF16 dispatch (and the combine-backward re-dispatch of gradient rows):
 * row t is copied bit for bit to each receive row dst_pos[t, j] >= 0. */
void oracle_dispatch_bf16(const uint16_t *x, int64_t N, int H, int k, const int32_t *dst_pos,
                          uint16_t *recv) {
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < N; ++t)
        for (int j = 0; j < k; ++j) {
            int32_t row = dst_pos[t * k + j];
            if (row < 0) continue;
            memcpy(recv + (int64_t)row * H, x + t * H, sizeof(uint16_t) * (size_t)H);
        }
}

/* --------------------------------------------------------------- combine */

/*
 * Combine: out[t, h] = bf16( (((0 + w0*y0) + w1*y1) + ...) + w_{k-1}*y_{k-1} )
 * with y_j = y[dst_pos[t, j], h] widened to binary32, every product and every
 * sum one binary32 operation in slot order, starting from +0, and slots with
 * dst_pos < 0 skipped.  Reading: the pages say only that combine accumulates;
 * the fixed order and fp32 accumulator are this library's contract.
 */
void oracle_combine(const uint16_t *y, const int32_t *dst_pos, const float *topk_w, int64_t N,
                    int H, int k, uint16_t *out) {
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < N; ++t)
        for (int h = 0; h < H; ++h) {
            float acc = 0.0f;
            for (int j = 0; j < k; ++j) {
                int32_t row = dst_pos[t * k + j];
                if (row < 0) continue;
                float prod = topk_w[t * k + j] * bf16_to_f32(y[(int64_t)row * H + h]);
                acc = acc + prod;
            }
            out[t * H + h] = oracle_bf16_from_f32(acc);
        }
}

/* ------------------------------------------------------- combine backward */

/*
 * Backward of combine (out[t] = sum_j w[t,j] * y[dst_pos[t,j]]) for an output
 * gradient g = dL/dout, BF16 [N, H]:
 *   grad_y[dst_pos[t,j], h] = bf16( w[t,j] * g[t,h] )   (one binary32 product, RNE)
 *   grad_w[t, j] = sum_h g[t,h] * y[dst_pos[t,j], h]     (accumulated in double, then
 *                                                          rounded once to binary32)
 * Slots with dst_pos < 0 write no row and get grad_w = 0.  Reading: the pages
 * only say that combine accumulates; this is its derivative, with the weight
 * gradient's reduction order left free (hence the double accumulation here:
 * the exact value up to one final rounding).
 */
void oracle_combine_backward(const uint16_t *g, const uint16_t *y, const int32_t *dst_pos,
                             const float *topk_w, int64_t N, int H, int k, uint16_t *grad_y,
                             float *grad_w) {
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < N; ++t)
        for (int j = 0; j < k; ++j) {
            int32_t row = dst_pos[t * k + j];
            if (row < 0) { grad_w[t * k + j] = 0.0f; continue; }
            float w = topk_w[t * k + j];
            double dot = 0.0;
            for (int h = 0; h < H; ++h) {
                float gv = bf16_to_f32(g[t * H + h]);
                float prod = w * gv;
                grad_y[(int64_t)row * H + h] = oracle_bf16_from_f32(prod);
                dot += (double)gv * (double)bf16_to_f32(y[(int64_t)row * H + h]);
            }
            grad_w[t * k + j] = (float)dot;
        }
}
