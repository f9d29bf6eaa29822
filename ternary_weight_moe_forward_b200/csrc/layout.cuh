// Internal weight layouts of the ternary MoE layer (library-owned copies).
//
// Interchange format (input of create): a row of n ternary values is n/16
// uint32 words, value j in word j/16 at bits 2*(j%16)..+1, code 0 = 0,
// 1 = +1, 2 = -1 (3 reads as 0).
//
// GEMV layout (weight streaming, T <= decode_max_tokens).  The codes of 32
// rows are interleaved in 16-byte chunks so that one warp-wide 128-bit load
// fetches chunk c of 32 different rows (512 contiguous bytes, lane l = row l):
//   gate/up  [E][F/16 groups][D/64 chunks][32 lanes][4 words]
//            lane l < 16: gate row 16*g + l;  lane l >= 16: up row 16*g + l - 16
//   down     [E][D/32 groups][F/64 chunks][32 lanes][4 words], lane l: row 32*g + l
// Word w of chunk c holds values j = 64*c + 16*w + 4*k + b (k, b = 0..3) as
// offset codes t + 1 in {0, 1, 2} at bits 8*b + 2*k.  Then (word >> 2k) &
// 0x03030303 is four bytes, one per value j = 64c+16w+4k+0..3, and dp4a with
// the four int8 activations x_j gives sum (t_j + 1) x_j; subtracting the
// token's sum of codes sum_j x_j leaves the exact ternary dot product.
//
// GEMM layout (tcgen05 int8 grouped GEMM, T > decode_max_tokens): see
// tc_gemm.cuh.
#pragma once

#include <stdint.h>

namespace maple {

__host__ __device__ constexpr int64_t gu_bytes_per_expert(int D, int F) { return (int64_t)F * D / 2; }
__host__ __device__ constexpr int64_t dn_bytes_per_expert(int D, int F) { return (int64_t)D * F / 4; }

// map an interchange code to the offset code t + 1 (invalid 3 -> value 0 -> 1)
__host__ __device__ inline uint32_t offset_code(uint32_t code)
{
    return code == 1u ? 2u : (code == 2u ? 0u : 1u);
}

// re-order the 16 codes of one interchange word into the GEMV word
__host__ __device__ inline uint32_t gemv_word(uint32_t canon)
{
    uint32_t out = 0;
#pragma unroll
    for (int i = 0; i < 16; i++) {
        uint32_t oc = offset_code((canon >> (2 * i)) & 3u);
        int k = i >> 2, b = i & 3;
        out |= oc << (8 * b + 2 * k);
    }
    return out;
}

}  // namespace maple
