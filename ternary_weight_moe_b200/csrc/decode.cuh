// decode.cuh -- ternary decode by integer logic, without a lookup table.
//
// A packed 32-bit word holds 16 ternary weights: byte b (0..3) holds weights 4b..4b+3, weight
// 4b+j in bits 8b+2j (low, "l") and 8b+2j+1 (high, "h") with codes 00 -> 0, 01 -> +1,
// 10 -> -1 and 11 read as 0.  The weight is w = l - h when the code is valid, and the dot
// product with activations needs only adds and subtracts of the activations ("A 20B AI Model
// Trained in Ternary Just Hit 218 Tokens/Second on a $599 Mac Mini", "What Ternary Actually
// Means"); here the four weights of one code position j in the four bytes become four signed
// int8 lanes, and one dp4a per activation limb adds or subtracts the four activations.
//
//  1. tern_signed_fields: every 2-bit field (h, l) becomes the 2-bit two's complement of its
//     weight, (h & ~l, h ^ l): 00 -> 00, 01 -> 01, 10 -> 11 (-1), 11 -> 00.
//  2. tern_position_lanes: field j of every byte moved to bits 7..6 of that byte and the other
//     bits cleared, so the byte read as int8 is 64 * w (0x40 = +64, 0xC0 = -64, 0).
// A dot product accumulated over such lanes is 64 times the weight sum; it is a multiple of
// 64, so an arithmetic shift right by 6 recovers it exactly.
//
// The activations meet these lanes in a position-major order: for the 16 weights of packed
// word q of a 16-byte segment, the limb word for position j holds the activations of weights
// 16q + j, 16q + 4 + j, 16q + 8 + j, 16q + 12 + j (one byte each, in that order).
#pragma once

#include <stdint.h>

#ifndef __CUDACC__
#define __host__
#define __device__
#define __forceinline__ inline
#endif

namespace tern {

__host__ __device__ __forceinline__ uint32_t tern_signed_fields(uint32_t w) {
    const uint32_t h = (w >> 1) & 0x55555555u;      // high bit of each field, at the low position
    const uint32_t hl = w & h;                      // h & l, at the low position
    return w ^ h ^ (hl << 1);                       // low bit l ^ h, high bit h ^ (h & l) = h & ~l
}

// lanes of position j (0..3) of a word returned by tern_signed_fields: int8 value 64 * w
__host__ __device__ __forceinline__ uint32_t tern_position_lanes(uint32_t s, int j) {
    return (s << (6 - 2 * j)) & 0xC0C0C0C0u;
}

// index of the activation met by lane b of position j of packed word q (0..63 in a segment)
__host__ __device__ __forceinline__ int tern_position_activation(int q, int j, int b) { return 16 * q + 4 * b + j; }

}  // namespace tern
