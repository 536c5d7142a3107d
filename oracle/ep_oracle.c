/*
 * CPU oracle for MoE expert-parallel dispatch / combine on one device.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  The product path
 * (the CUDA library and its Python binding) never calls it, and the two
 * share no code: no headers, helpers, tables or constants.
 *
 * Plain, slow, single-threaded C written straight from the definitions.
 * Build: gcc -O2 -std=c11 -ffp-contract=off (no fast-math), so every
 * float operation below is one IEEE-754 binary32 operation rounded to
 * nearest-even, in the order written.  The only fused operation is the
 * explicit fmaf() of the combine sum.
 *
 * What is computed, and where it is stated (page titles are those of the
 * DeepEP V2 README, section "Interfaces and examples"):
 *   - layout: per-expert receive counts and the expert-major receive
 *     layout behind the dispatch handle ("handle contains routing metadata",
 *     "num_recv_tokens_per_expert_list provides per-expert token counts for
 *     GEMM"), padded per expert to a multiple of expert_alignment;
 *   - dispatch: every token row copied to each of its top-k experts
 *     (dispatch_forward), either as bf16, as a caller-quantised
 *     (data, scale_factors) FP8 tuple, or quantised here to FP8 e4m3 with
 *     one fp32 scale per 1x128 block;
 *   - combine: the k expert outputs of each token gathered back and summed
 *     (combine_forward), weighted by topk_weights; with no weights it is
 *     the adjoint of dispatch (dispatch_backward), optionally gathering the
 *     per-row weight gradient back to [T, k];
 *   - the backward of the weighted combine (combine_backward, which the
 *     page runs as a dispatch of the output gradient): each receive row gets
 *     its slot's weight times the token's output gradient, and each slot's
 *     weight gradient is the dot product of the token's output gradient with
 *     the row's expert output.
 *
 * Readings taken where the pages are silent (each is a definition here):
 *   - rows of one expert are ordered by flat slot s = t*k + j, ascending;
 *     experts are laid out in ascending id order;
 *   - expert e gets A(c_e) = ceil(c_e / align) * align rows, A(0) = 0; its
 *     padding rows come after its c_e real rows and hold zero data, zero
 *     scales, recv_src = recv_topk_idx = -1 and weight 0;
 *   - a topk_idx value of -1 drops the slot; any other value outside
 *     [0, E) is an error, flagged and then treated as dropped;
 *   - segment s (a logical "rank") owns experts [s*E/S, (s+1)*E/S); its
 *     token count counts a token once if any of its valid slots land there;
 *   - FP8 block scale: amax = max |x| over the 128 values, floored at 1e-4,
 *     scale = amax / 448, inv = 448 / amax (two IEEE divisions),
 *     q = e4m3(x * inv) rounded to nearest-even with saturation to +-448;
 *   - combine: acc = +0.0f, then for j = 0..k-1 over valid slots
 *     acc = fmaf(w[t,j], y[row], acc), and one bf16 rounding at the end;
 *   - NVFP4 dispatch (the Hybrid-EP branch of the DeepEP V2 README lists the
 *     NVFP4 data type; nothing more is stated): E2M1 values in 1x16 blocks,
 *     one E4M3 scale per block, no per-tensor scale: amax = max |x| floored
 *     at 6 * 2^-9, scale = e4m3(amax / 6) (nearest-even, saturating),
 *     inv = 1 / scale (one IEEE division), q = e2m1(x * inv) rounded to
 *     nearest-even and saturating at +-6; two codes per byte, the even
 *     element in the low nibble;
 *   - FP8 combine (the README's introduction says the kernels support low
 *     precision, FP8 included; nothing fixes the combine's arithmetic):
 *     expert outputs as e4m3 codes with one f32 scale per 1x128 block, the
 *     same layout as the FP8 dispatch's output; v = e4m3_decode(q) * scale
 *     (one binary32 multiply), then the combine sum above;
 *   - combine backward: grad_y[row] = bf16(w * g) with the product taken in
 *     binary32 (one multiply, one bf16 rounding); padding rows of grad_y are
 *     zero; grad_w is the exact dot product, accumulated here in binary64
 *     (the GPU accumulates in binary32; tests bound the difference by the
 *     binary32 summation error bound).
 *
 * Parity pins: every function here is checked against brute force,
 * independent library routines, exact rational arithmetic or invariants
 * in tests/test_oracle.py.  None is "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define EXPORT __attribute__((visibility("default")))

/* ---------------------------------------------------------------- formats */

static float f32_from_bits(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t bits_from_f32(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

/* bfloat16 is the upper half of a binary32: widening is exact. */
EXPORT float oracle_bf16_to_f32(uint16_t b) { return f32_from_bits((uint32_t)b << 16); }

/* binary32 -> bfloat16, round to nearest, ties to even.  bfloat16 keeps the
 * binary32 exponent range and 8 significand bits, so rounding is done on
 * the 16 low bits that are dropped; a carry out of the mantissa moves into
 * the exponent, which is the correct next binade (or infinity).  NaN stays
 * NaN with its sign (quiet bit set). */
EXPORT uint16_t oracle_f32_to_bf16(float v) {
    uint32_t u = bits_from_f32(v);
    if (isnan(v)) return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t keep = u >> 16, dropped = u & 0xFFFFu;
    if (dropped > 0x8000u || (dropped == 0x8000u && (keep & 1u))) keep += 1u;
    return (uint16_t)keep;
}

/* OCP 8-bit float, E4M3 variant: sign, 4 exponent bits (bias 7), 3 mantissa
 * bits, no infinities; S.1111.111 is NaN, so the largest finite magnitude is
 * S.1111.110 = 1.75 * 2^8 = 448.  Exponent field 0 holds subnormals
 * m * 2^-9; the smallest normal is 2^-6.  Every binade [2^b, 2^(b+1)) holds 8
 * values spaced 2^(b-3); the subnormals share the spacing of the first
 * normal binade (2^-9).
 *
 * Encoding: round to nearest, ties to even mantissa, and saturate: every
 * magnitude at or above 448 (infinity included) encodes as 448. */
EXPORT uint8_t oracle_e4m3_encode(float v) {
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    if (isnan(v)) return (uint8_t)(sign | 0x7F);
    float a = fabsf(v);
    if (a >= 448.0f) return (uint8_t)(sign | 0x7E);
    if (a == 0.0f) return sign;
    int e;
    frexpf(a, &e);             /* a = f * 2^e with f in [0.5, 1): binade e-1 */
    int binade = e - 1;
    if (binade < -6) binade = -6;               /* subnormal spacing 2^-9 */
    float quantum = ldexpf(1.0f, binade - 3);
    float n = rintf(a / quantum);  /* exact scaling; rintf: nearest, ties even */
    int m = (int)n;                /* value = m * quantum, 0 <= m <= 16 */
    if (a < 0.015625f)             /* below 2^-6: subnormal code m (m = 8 is 2^-6) */
        return (uint8_t)(sign | m);
    if (m == 16) { m = 8; binade += 1; }        /* rounded up into the next binade */
    return (uint8_t)(sign | ((binade + 7) << 3) | (m - 8));
}

EXPORT float oracle_e4m3_decode(uint8_t c) {
    int ef = (c >> 3) & 0xF, mant = c & 7;
    float mag;
    if (ef == 0xF && mant == 7) mag = NAN;
    else if (ef == 0) mag = ldexpf((float)mant, -9);
    else mag = ldexpf((float)(8 + mant), ef - 7 - 3);
    return (c & 0x80) ? -mag : mag;
}

/* Array forms, so that tests can sweep millions of values. */
EXPORT void oracle_f32_to_bf16_n(const float* v, uint16_t* out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_f32_to_bf16(v[i]);
}
EXPORT void oracle_e4m3_encode_n(const float* v, uint8_t* out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_e4m3_encode(v[i]);
}

/* ------------------------------------------------------- FP8 1x128 blocks */

#define QBLOCK 128
static const float E4M3_MAX = 448.0f;
static const float AMAX_FLOOR = 1e-4f;

/* One 1x128 block of bf16 values -> 128 e4m3 codes and one fp32 scale such
 * that x ~= decode(q) * scale. */
static void quantize_block(const uint16_t* x, uint8_t* q, float* scale) {
    float amax = 0.0f;
    for (int i = 0; i < QBLOCK; ++i) amax = fmaxf(amax, fabsf(oracle_bf16_to_f32(x[i])));
    if (amax < AMAX_FLOOR) amax = AMAX_FLOOR;
    *scale = amax / E4M3_MAX;
    float inv = E4M3_MAX / amax;
    for (int i = 0; i < QBLOCK; ++i) q[i] = oracle_e4m3_encode(oracle_bf16_to_f32(x[i]) * inv);
}

/* A [rows, H] bf16 matrix -> e4m3 [rows, H] and scales [rows, H/128]. */
EXPORT void oracle_quantize_rows(int64_t rows, int32_t H, const uint16_t* x, uint8_t* q,
                                 float* scales) {
    int32_t nb = H / QBLOCK;
    for (int64_t r = 0; r < rows; ++r)
        for (int32_t b = 0; b < nb; ++b)
            quantize_block(x + r * H + (int64_t)b * QBLOCK, q + r * H + (int64_t)b * QBLOCK,
                           scales + r * nb + b);
}

/* ---------------------------------------------------- NVFP4 (E2M1, 1x16) */

/* 4-bit float E2M1: sign, 2 exponent bits (bias 1), 1 mantissa bit, no
 * infinities or NaN.  Magnitudes: exponent field 0 holds 0 and 0.5 (m * 0.5);
 * field f >= 1 holds (1 + m/2) * 2^(f-1): 1, 1.5, 2, 3, 4, 6.  Encoding:
 * nearest, ties to even mantissa, saturating at 6. */
EXPORT uint8_t oracle_e2m1_encode(float v) {
    uint8_t sign = signbit(v) ? 0x8 : 0x0;
    float a = fabsf(v);
    if (isnan(v)) return sign | 0x7;          /* unspecified; never produced by finite inputs */
    if (a >= 6.0f) return sign | 0x7;
    float quantum;                            /* spacing of the grid at a's magnitude */
    int field;
    if (a < 2.0f) { quantum = 0.5f; field = 0; }
    else if (a < 4.0f) { quantum = 1.0f; field = 2; }
    else { quantum = 2.0f; field = 3; }
    int n = (int)rintf(a / quantum);          /* exact scaling, nearest-even */
    if (field == 0) {                         /* [0, 2): 0, 0.5, 1, 1.5 -> codes 0..3; 2 -> code 4 */
        return sign | (uint8_t)n;
    }
    if (field == 2) {                         /* [2, 4): n in {2, 3, 4}: 2 -> 0x4, 3 -> 0x5, 4 -> 0x6 */
        return sign | (uint8_t)(n + 2);
    }
    return sign | (uint8_t)(n == 2 ? 0x6 : 0x7); /* [4, 6): n in {2, 3}: 4 -> 0x6, 6 -> 0x7 */
}

EXPORT float oracle_e2m1_decode(uint8_t c) {
    static const float mag[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};
    return (c & 0x8) ? -mag[c & 7] : mag[c & 7];
}

EXPORT void oracle_e2m1_encode_n(const float* v, uint8_t* out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_e2m1_encode(v[i]);
}

#define FP4BLOCK 16
static const float E2M1_MAX = 6.0f;
static const float FP4_AMAX_FLOOR = 6.0f / 512.0f;   /* 6 * 2^-9: smallest e4m3 scale */

/* One 1x16 block of bf16 -> 8 bytes of E2M1 pairs and one E4M3 scale byte. */
static void nvfp4_block(const uint16_t* x, uint8_t* q, uint8_t* scale) {
    float amax = 0.0f;
    for (int i = 0; i < FP4BLOCK; ++i) amax = fmaxf(amax, fabsf(oracle_bf16_to_f32(x[i])));
    if (amax < FP4_AMAX_FLOOR) amax = FP4_AMAX_FLOOR;
    *scale = oracle_e4m3_encode(amax / E2M1_MAX);
    float inv = 1.0f / oracle_e4m3_decode(*scale);
    for (int i = 0; i < FP4BLOCK; i += 2)
        q[i / 2] = (uint8_t)(oracle_e2m1_encode(oracle_bf16_to_f32(x[i]) * inv) |
                             (oracle_e2m1_encode(oracle_bf16_to_f32(x[i + 1]) * inv) << 4));
}

/* A [rows, H] bf16 matrix -> packed E2M1 [rows, H/2] and scales [rows, H/16]. */
EXPORT void oracle_nvfp4_rows(int64_t rows, int32_t H, const uint16_t* x, uint8_t* q, uint8_t* scales) {
    int32_t nb = H / FP4BLOCK;
    for (int64_t r = 0; r < rows; ++r)
        for (int32_t b = 0; b < nb; ++b)
            nvfp4_block(x + r * H + (int64_t)b * FP4BLOCK, q + r * (H / 2) + (int64_t)b * (FP4BLOCK / 2),
                        scales + r * nb + b);
}

/* ---------------------------------------------------------------- layout */

EXPORT int32_t oracle_max_recv_rows(int32_t T, int32_t k, int32_t E, int32_t align) {
    return T * k + E * (align - 1);
}

/* Returns 1 if some topk_idx value was outside [-1, E) (treated as dropped),
 * 2 if the layout would need more than max_recv_rows rows (nothing written
 * past the capacity), 0 otherwise. */
EXPORT uint32_t oracle_layout(int32_t T, int32_t k, int32_t E, int32_t S, int32_t align,
                              const int64_t* topk_idx, const float* topk_weights,
                              int32_t max_recv_rows, int32_t* counts, int32_t* offsets,
                              int32_t* seg_tokens, int32_t* slot_map, int32_t* recv_src,
                              int32_t* recv_topk_idx, float* recv_topk_weights) {
    uint32_t flags = 0;
    int64_t n = (int64_t)T * k;
    int32_t per_seg = E / S;

    /* Expert of each slot, -1 when dropped. */
    int32_t* expert = (int32_t*)malloc(sizeof(int32_t) * (n > 0 ? n : 1));
    for (int64_t s = 0; s < n; ++s) {
        int64_t e = topk_idx[s];
        if (e < -1 || e >= E) { flags |= 1u; e = -1; }
        expert[s] = (int32_t)e;
    }

    /* Raw per-expert counts. */
    for (int32_t e = 0; e < E; ++e) counts[e] = 0;
    for (int64_t s = 0; s < n; ++s)
        if (expert[s] >= 0) counts[expert[s]] += 1;

    /* Expert-major offsets: expert e starts after all lower experts' padded
     * blocks; offsets[E] is the total row count R. */
    offsets[0] = 0;
    for (int32_t e = 0; e < E; ++e) {
        int32_t padded = (counts[e] + align - 1) / align * align;
        offsets[e + 1] = offsets[e] + padded;
    }
    if (offsets[E] > max_recv_rows) flags |= 2u;

    /* Slot map: walk the slots in flat order, each expert handing out its
     * rows from the front of its block. */
    int32_t* cursor = (int32_t*)malloc(sizeof(int32_t) * E);
    for (int32_t e = 0; e < E; ++e) cursor[e] = offsets[e];
    for (int64_t s = 0; s < n; ++s) {
        int32_t e = expert[s];
        if (e < 0) { slot_map[s] = -1; continue; }
        int32_t row = cursor[e]++;
        if (row >= max_recv_rows) { slot_map[s] = -1; continue; }
        slot_map[s] = row;
        recv_src[row] = (int32_t)s;
        recv_topk_idx[row] = e;
        recv_topk_weights[row] = topk_weights ? topk_weights[s] : 0.0f;
    }
    /* Padding rows of each expert: after its real rows, up to the next block. */
    for (int32_t e = 0; e < E; ++e)
        for (int32_t row = offsets[e] + counts[e]; row < offsets[e + 1] && row < max_recv_rows;
             ++row) {
            recv_src[row] = -1;
            recv_topk_idx[row] = -1;
            recv_topk_weights[row] = 0.0f;
        }

    /* Tokens per segment: a token counts once per segment it sends to. */
    for (int32_t g = 0; g < S; ++g) seg_tokens[g] = 0;
    for (int32_t t = 0; t < T; ++t)
        for (int32_t g = 0; g < S; ++g) {
            int hit = 0;
            for (int32_t j = 0; j < k; ++j) {
                int32_t e = expert[(int64_t)t * k + j];
                if (e >= 0 && e / per_seg == g) hit = 1;
            }
            seg_tokens[g] += hit;
        }

    free(cursor);
    free(expert);
    return flags;
}

/* -------------------------------------------------------------- dispatch */

enum { ORACLE_X_BF16 = 0, ORACLE_X_FP8_PREQUANT = 1, ORACLE_X_BF16_QUANT_FP8 = 2, ORACLE_X_BF16_QUANT_NVFP4 = 3 };

/* Copies token t's row into row slot_map[t*k+j] for every valid j, and zeroes
 * the padding rows (rows r < R with recv_src[r] < 0).
 *   mode 0: x bf16 [T,H]                  -> recv_x bf16 [*,H]
 *   mode 1: x e4m3 [T,H], x_scales [T,H/128] -> recv_x e4m3, recv_scales f32
 *   mode 2: x bf16 [T,H], quantised here   -> recv_x e4m3, recv_scales f32 [*,H/128]
 *   mode 3: x bf16 [T,H], NVFP4 here       -> recv_x [*,H/2] bytes, recv_scales e4m3 bytes [*,H/16] */
EXPORT void oracle_dispatch(int32_t mode, int32_t T, int32_t k, int32_t H, int32_t R,
                            const int32_t* slot_map, const int32_t* recv_src, const void* x,
                            const float* x_scales, void* recv_x, void* recv_scales) {
    const int fp4 = mode == ORACLE_X_BF16_QUANT_NVFP4;
    int32_t nb = fp4 ? H / FP4BLOCK : H / QBLOCK;
    size_t row_bytes = mode == ORACLE_X_BF16 ? (size_t)H * 2 : fp4 ? (size_t)H / 2 : (size_t)H;
    size_t scale_bytes = fp4 ? (size_t)nb : sizeof(float) * (size_t)nb;
    uint8_t* qrow = (uint8_t*)malloc((size_t)H);
    uint8_t* srow = (uint8_t*)malloc(scale_bytes > 0 ? scale_bytes : 1);

    for (int32_t t = 0; t < T; ++t) {
        const uint8_t* src;
        const float* src_scales = NULL;
        if (mode == ORACLE_X_BF16) {
            src = (const uint8_t*)x + (size_t)t * row_bytes;
        } else if (mode == ORACLE_X_FP8_PREQUANT) {
            src = (const uint8_t*)x + (size_t)t * row_bytes;
            src_scales = x_scales + (size_t)t * nb;
        } else if (fp4) {
            const uint16_t* xt = (const uint16_t*)x + (size_t)t * H;
            for (int32_t b = 0; b < nb; ++b)
                nvfp4_block(xt + b * FP4BLOCK, qrow + b * (FP4BLOCK / 2), srow + b);
            src = qrow;
            src_scales = (const float*)srow;
        } else {
            const uint16_t* xt = (const uint16_t*)x + (size_t)t * H;
            for (int32_t b = 0; b < nb; ++b)
                quantize_block(xt + b * QBLOCK, qrow + b * QBLOCK, (float*)srow + b);
            src = qrow;
            src_scales = (const float*)srow;
        }
        for (int32_t j = 0; j < k; ++j) {
            int32_t row = slot_map[(int64_t)t * k + j];
            if (row < 0) continue;
            memcpy((uint8_t*)recv_x + (size_t)row * row_bytes, src, row_bytes);
            if (mode != ORACLE_X_BF16)
                memcpy((uint8_t*)recv_scales + (size_t)row * scale_bytes, src_scales, scale_bytes);
        }
    }
    for (int32_t row = 0; row < R; ++row) {
        if (recv_src[row] >= 0) continue;
        memset((uint8_t*)recv_x + (size_t)row * row_bytes, 0, row_bytes);
        if (mode != ORACLE_X_BF16) memset((uint8_t*)recv_scales + (size_t)row * scale_bytes, 0, scale_bytes);
    }
    free(srow);
    free(qrow);
}

/* --------------------------------------------------------------- combine */

/* out[t,h] = bf16( sum over valid j, in ascending j, of w[t,j] * y[slot_map[t,j], h] ),
 * accumulated as acc = fmaf(w, y, acc) from acc = +0.0f.  With weights NULL
 * every w is 1 (the unweighted sum: dispatch's adjoint).  If out_weights is
 * given, out_weights[t,j] = recv_weights_in[slot_map[t,j]] (0 when dropped). */
EXPORT void oracle_combine(int32_t T, int32_t k, int32_t H, const int32_t* slot_map,
                           const uint16_t* y, const float* weights,
                           const float* recv_weights_in, float* out_weights, uint16_t* out) {
    for (int32_t t = 0; t < T; ++t) {
        const int32_t* sm = slot_map + (int64_t)t * k;
        for (int32_t h = 0; h < H; ++h) {
            float acc = 0.0f;
            for (int32_t j = 0; j < k; ++j) {
                if (sm[j] < 0) continue;
                float w = weights ? weights[(int64_t)t * k + j] : 1.0f;
                acc = fmaf(w, oracle_bf16_to_f32(y[(size_t)sm[j] * H + h]), acc);
            }
            out[(size_t)t * H + h] = oracle_f32_to_bf16(acc);
        }
        if (out_weights)
            for (int32_t j = 0; j < k; ++j)
                out_weights[(int64_t)t * k + j] =
                    (sm[j] >= 0 && recv_weights_in) ? recv_weights_in[sm[j]] : 0.0f;
    }
}

/* Combine of FP8 expert outputs (the low-precision combine: DeepEP V2
 * README, introduction -- the kernels support low precision, FP8 included).
 * Row r of y holds e4m3 codes yq[r, :] and one f32 scale per 1x128 block,
 * ys[r, b].  Each value is decoded and multiplied by its block's scale in
 * binary32 (one rounding), then accumulated as in oracle_combine:
 *   v = e4m3_decode(yq[r,h]) * ys[r, h/128]
 *   out[t,h] = bf16( acc ),  acc = fmaf(w[t,j], v, acc) from +0 over valid j ascending.
 * With weights NULL every w is 1. */
EXPORT void oracle_combine_fp8(int32_t T, int32_t k, int32_t H, const int32_t* slot_map, const uint8_t* yq,
                               const float* ys, const float* weights, uint16_t* out) {
    const int32_t B = H / 128;
    for (int32_t t = 0; t < T; ++t) {
        for (int32_t h = 0; h < H; ++h) {
            float sum = 0.0f;
            for (int32_t j = 0; j < k; ++j) {
                const int32_t r = slot_map[(int64_t)t * k + j];
                if (r < 0) continue;
                const float wj = weights ? weights[(int64_t)t * k + j] : 1.0f;
                const float v = oracle_e4m3_decode(yq[(size_t)r * H + h]) * ys[(size_t)r * B + h / 128];
                sum = fmaf(wj, v, sum);
            }
            out[(size_t)t * H + h] = oracle_f32_to_bf16(sum);
        }
    }
}

/* ------------------------------------------------------- combine backward */

/* Backward of the weighted combine, for the output gradient g [T,H] bf16:
 *   grad_y[slot_map[t*k+j], h] = bf16(w[t,j] * g[t,h])   (binary32 product)
 *   grad_w[t,j] = sum_h g[t,h] * y[slot_map[t*k+j], h]   (binary64; 0 when dropped)
 * and grad_y rows r < R with recv_src[r] < 0 (padding) are zero. */
EXPORT void oracle_combine_backward(int32_t T, int32_t k, int32_t H, int32_t R, const int32_t* slot_map,
                                    const int32_t* recv_src, const uint16_t* g, const uint16_t* y,
                                    const float* weights, uint16_t* grad_y, double* grad_w) {
    for (int32_t t = 0; t < T; ++t)
        for (int32_t j = 0; j < k; ++j) {
            int32_t row = slot_map[(int64_t)t * k + j];
            if (row < 0) {
                grad_w[(int64_t)t * k + j] = 0.0;
                continue;
            }
            float w = weights[(int64_t)t * k + j];
            double dot = 0.0;
            for (int32_t h = 0; h < H; ++h) {
                float gv = oracle_bf16_to_f32(g[(size_t)t * H + h]);
                grad_y[(size_t)row * H + h] = oracle_f32_to_bf16(w * gv);
                dot += (double)gv * (double)oracle_bf16_to_f32(y[(size_t)row * H + h]);
            }
            grad_w[(int64_t)t * k + j] = dot;
        }
    for (int32_t row = 0; row < R; ++row)
        if (recv_src[row] < 0) memset(grad_y + (size_t)row * H, 0, sizeof(uint16_t) * H);
}
