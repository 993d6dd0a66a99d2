// Host check of the table-free ternary decode (ternary_weight_moe_b200/csrc/decode.cuh):
// for every byte value in every byte position of a word, and every code position j, the
// int8 lane produced for (byte, j) must equal 64 * w with w the weight of that code
// (00 -> 0, 01 -> +1, 10 -> -1, 11 -> 0), and other bytes must not leak into it.  Then the
// 64-weight segment dot product written with these lanes must equal the plain sum for
// random words and limbs.  Prints "decode ok" and exits 0, or reports the first mismatch.
#include <cstdio>
#include <cstdint>
#include <cstdlib>

#include "../ternary_weight_moe_b200/csrc/decode.cuh"

static int weight_of(unsigned code) { return code == 1 ? 1 : (code == 2 ? -1 : 0); }

int main() {
    using namespace tern;
    for (int bytepos = 0; bytepos < 4; bytepos++) {
        for (unsigned v = 0; v < 256; v++) {
            // fill the other bytes with a pattern that must not leak
            const uint32_t other = 0xB7u * 0x01010101u;
            uint32_t w = (other & ~(0xFFu << (8 * bytepos))) | (v << (8 * bytepos));
            const uint32_t s = tern_signed_fields(w);
            for (int j = 0; j < 4; j++) {
                const uint32_t lanes = tern_position_lanes(s, j);
                const int8_t got = (int8_t)((lanes >> (8 * bytepos)) & 0xFFu);
                const int want = 64 * weight_of((v >> (2 * j)) & 3u);
                if (got != want) {
                    printf("mismatch byte %u pos %d j %d: got %d want %d\n", v, bytepos, j, got, want);
                    return 1;
                }
            }
        }
    }
    // segment dot: 4 words x 16 weights against signed 8-bit activations
    srand(12345);
    for (int trial = 0; trial < 20000; trial++) {
        uint32_t words[4];
        int8_t act[64];
        for (int q = 0; q < 4; q++) words[q] = ((uint32_t)rand() << 16) ^ (uint32_t)rand();
        for (int i = 0; i < 64; i++) act[i] = (int8_t)((rand() % 255) - 127);
        long plain = 0;
        for (int i = 0; i < 64; i++) {
            const unsigned code = (words[i / 16] >> (2 * (i % 16))) & 3u;
            plain += (long)weight_of(code) * act[i];
        }
        long lanes_sum = 0;
        for (int q = 0; q < 4; q++) {
            const uint32_t s = tern_signed_fields(words[q]);
            for (int j = 0; j < 4; j++) {
                const uint32_t m = tern_position_lanes(s, j);
                for (int b = 0; b < 4; b++)
                    lanes_sum += (long)(int8_t)((m >> (8 * b)) & 0xFFu) * act[tern_position_activation(q, j, b)];
            }
        }
        if (lanes_sum % 64 != 0 || lanes_sum / 64 != plain) {
            printf("segment mismatch trial %d: %ld vs %ld\n", trial, lanes_sum, plain);
            return 1;
        }
    }
    printf("decode ok\n");
    return 0;
}
