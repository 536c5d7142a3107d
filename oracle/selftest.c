/*
 * Self-test of the CPU oracle as a C program: hand-derived values only.
 *
 * TEST INFRASTRUCTURE.  Built with the oracle's own flags as one
 * translation unit with ep_oracle.c and run by the test suite; exit status
 * 0 means every check held.  Every expected value below is derived by hand
 * from a format's definition or from the hand-worked layout example in
 * tests/golden/layout_hand_example.json (the pages print no worked
 * example).
 */
#include "ep_oracle.c"

#include <stdio.h>

static int failures = 0;

#define CHECK(cond, ...)                     \
    do {                                     \
        if (!(cond)) {                       \
            fprintf(stderr, "FAIL: ");       \
            fprintf(stderr, __VA_ARGS__);    \
            fprintf(stderr, "\n");           \
            ++failures;                      \
        }                                    \
    } while (0)

static float f32_of(uint32_t u) { return f32_from_bits(u); }

static void formats(void) {
    /* bf16: nearest, ties to the even upper half */
    CHECK(oracle_f32_to_bf16(1.0f) == 0x3F80, "bf16(1)");
    CHECK(oracle_f32_to_bf16(f32_of(0x3F808000u)) == 0x3F80, "bf16 tie to even (down)");
    CHECK(oracle_f32_to_bf16(f32_of(0x3F818000u)) == 0x3F82, "bf16 tie to even (up)");
    CHECK(oracle_f32_to_bf16(f32_of(0x3F808001u)) == 0x3F81, "bf16 above the tie");
    CHECK(oracle_bf16_to_f32(0xC040) == -3.0f, "bf16 -> f32");
    /* e4m3 (bias 7, 3 mantissa bits, max 448, saturating) */
    CHECK(oracle_e4m3_encode(1.0f) == 0x38, "e4m3(1)");
    CHECK(oracle_e4m3_encode(-2.0f) == 0xC0, "e4m3(-2)");
    CHECK(oracle_e4m3_encode(448.0f) == 0x7E, "e4m3(448)");
    CHECK(oracle_e4m3_encode(1000.0f) == 0x7E, "e4m3 saturates");
    CHECK(oracle_e4m3_encode(0.001953125f) == 0x01, "e4m3(2^-9), smallest subnormal");
    CHECK(oracle_e4m3_encode(1.0625f) == 0x38, "e4m3 tie 1.0625 -> even mantissa 1.0");
    CHECK(oracle_e4m3_encode(1.1875f) == 0x3A, "e4m3 tie 1.1875 -> even mantissa 1.25");
    CHECK(oracle_e4m3_decode(0x7E) == 448.0f && oracle_e4m3_decode(0x01) == 0.001953125f, "e4m3 decode");
    /* e2m1 (magnitudes 0 0.5 1 1.5 2 3 4 6, saturating, ties to the even code) */
    CHECK(oracle_e2m1_encode(1.5f) == 0x3, "e2m1(1.5)");
    CHECK(oracle_e2m1_encode(-6.0f) == 0xF, "e2m1(-6)");
    CHECK(oracle_e2m1_encode(7.0f) == 0x7, "e2m1 saturates");
    CHECK(oracle_e2m1_encode(0.25f) == 0x0, "e2m1 tie 0.25 -> 0");
    CHECK(oracle_e2m1_encode(2.5f) == 0x4, "e2m1 tie 2.5 -> 2");
    CHECK(oracle_e2m1_encode(5.0f) == 0x6, "e2m1 tie 5 -> 4");
    CHECK(oracle_e2m1_decode(0xD) == -3.0f, "e2m1 decode");
}

static void layout_and_combine(void) {
    /* the hand-worked example: T=3, k=2, E=4, S=2, alignment 2 */
    const int64_t idx[6] = {2, 0, 0, -1, 3, 0};
    const float w[6] = {0.75f, 0.25f, 1.0f, 0.5f, 0.5f, 0.5f};
    int32_t counts[4], offsets[5], seg[2], slot_map[6], recv_src[10], recv_idx[10];
    float recv_w[10];
    const uint32_t flags = oracle_layout(3, 2, 4, 2, 2, idx, w, 10, counts, offsets, seg, slot_map, recv_src,
                                         recv_idx, recv_w);
    const int32_t e_counts[4] = {3, 0, 1, 1}, e_off[5] = {0, 4, 4, 6, 8}, e_seg[2] = {3, 2};
    const int32_t e_slot[6] = {4, 0, 1, -1, 6, 2}, e_src[8] = {1, 2, 5, -1, 0, -1, 4, -1};
    const int32_t e_ridx[8] = {0, 0, 0, -1, 2, -1, 3, -1};
    const float e_rw[8] = {0.25f, 1.0f, 0.5f, 0.0f, 0.75f, 0.0f, 0.5f, 0.0f};
    CHECK(flags == 0, "layout flags");
    for (int i = 0; i < 4; ++i) CHECK(counts[i] == e_counts[i], "counts[%d]", i);
    for (int i = 0; i < 5; ++i) CHECK(offsets[i] == e_off[i], "offsets[%d]", i);
    for (int i = 0; i < 2; ++i) CHECK(seg[i] == e_seg[i], "seg_tokens[%d]", i);
    for (int i = 0; i < 6; ++i) CHECK(slot_map[i] == e_slot[i], "slot_map[%d]", i);
    for (int i = 0; i < 8; ++i) CHECK(recv_src[i] == e_src[i], "recv_src[%d]", i);
    for (int i = 0; i < 8; ++i) CHECK(recv_idx[i] == e_ridx[i], "recv_topk_idx[%d]", i);
    for (int i = 0; i < 8; ++i) CHECK(recv_w[i] == e_rw[i], "recv_topk_weights[%d]", i);

    /* combine over y rows of the example (all values exact in bf16 and every partial sum exact in fp32) */
    const float yf[16] = {1, 2, 3, -4, 0.5f, 8, 99, 99, 10, 1, 99, 99, -2, 0.25f, 99, 99};
    uint16_t y[16], out[6];
    for (int i = 0; i < 16; ++i) y[i] = oracle_f32_to_bf16(yf[i]);
    oracle_combine(3, 2, 2, slot_map, y, w, NULL, NULL, out);
    const float e_out[6] = {7.75f, 1.25f, 3.0f, -4.0f, -0.75f, 4.125f};
    for (int i = 0; i < 6; ++i) CHECK(oracle_bf16_to_f32(out[i]) == e_out[i], "combine[%d]", i);
    oracle_combine(3, 2, 2, slot_map, y, NULL, NULL, NULL, out);
    const float e_unw[6] = {11.0f, 3.0f, 3.0f, -4.0f, -1.5f, 8.25f};
    for (int i = 0; i < 6; ++i) CHECK(oracle_bf16_to_f32(out[i]) == e_unw[i], "unweighted combine[%d]", i);
}

static void combine_fp8(void) {
    /* codes 0x38 (1.0) and 0x40 (2.0), block scale 0.75 -> v = 0.75, 1.5;
     * 0.5 * 0.75 + 0.25 * 1.5 = 0.75 -> bf16 0x3F40 */
    uint8_t q[2 * 128] = {0};
    q[0] = 0x38;
    q[128] = 0x40;
    const float s[2] = {0.75f, 0.75f}, w[2] = {0.5f, 0.25f};
    const int32_t sm[2] = {0, 1};
    uint16_t out[128];
    oracle_combine_fp8(1, 2, 128, sm, q, s, w, out);
    CHECK(out[0] == 0x3F40, "fp8 combine");
    CHECK(out[1] == 0x0000, "fp8 combine of zero codes");
}

int main(void) {
    formats();
    layout_and_combine();
    combine_fp8();
    if (failures) {
        fprintf(stderr, "%d check(s) failed\n", failures);
        return 1;
    }
    printf("oracle self-test: all checks hold\n");
    return 0;
}
