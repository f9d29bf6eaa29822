// Internal weight layouts of the ternary MoE layer (library-owned copies).
//
// Interchange format (input of create): a row of n ternary values is n/16
// uint32 words, value j in word j/16 at bits 2*(j%16)..+1, code 0 = 0,
// 1 = +1, 2 = -1 (3 reads as 0).
//
// GEMM layout (tcgen05 int8 grouped GEMM, T > decode_max_tokens): see
// tc_gemm.cuh.
//
// MMA-tile layout (the decode kernels, warp-level int8 MMA m16n8k32 with
// the weights as the 16 x 32 A operand).  A tile is 16 rows over the whole K,
// stored as K/128 blocks of 512 bytes (32 lanes x 4 words).  Tiles are grouped
// into items, the unit of the kernels' weight stream, each followed by the
// row scales it needs, so that one copy brings both:
//   gate/up  [E][F/8 items]  item t = one tile (rows 0..7 = gate rows 8t..8t+7,
//            rows 8..15 = the up rows of the same outputs) over D/128 blocks,
//            then alpha_gate[8t..8t+7], alpha_up[8t..8t+7]   (4D + 64 bytes)
//   down     [E][F/16 items] item t = S2 = D/F consecutive tiles (tile 16c +
//            r = channel of row r) over F/128 blocks each, then alpha_down of
//            its 16*S2 channels                               (4D + 64*S2 bytes)
// Consecutive items of one expert are contiguous, so a run of them is one copy.
// Lane l (g = l/4, c = l%4), word i, byte j, plane q (bits 8j + 2q) holds the
// offset code t + 1 of row g + 8*(i%2), column 128*kb + 32q + 16*(i/2) + 4c + j.
// So w_i & (0x03030303 << 2q) is A-fragment register i of the MMA over
// columns 128kb + 32q .. +31, with every value scaled by 4^q: one logic
// operation per register, one accumulator per plane, combined exactly as
// acc_0 + acc_1/4 + acc_2/16 + acc_3/64 (each acc_q a multiple of 4^q).
//
// The matching B operand (activations, 8 tokens per MMA) wants, from token
// g's 128 columns of block kb, the four bytes at 32q + 16h + 4c (h = 0, 1)
// in lane 4g + c.  frag_word_pos(w) is where 4-byte word w (columns 4w ..
// 4w+3) of a 128-column block goes so that lane c of a token reads its eight
// words (q = 0..3, h = 0..1) as 32 contiguous bytes at 32c.
#pragma once

#include <stdint.h>

namespace maple {

// bytes of one item of the MMA-tile layout (codes and scales) and items per expert
__host__ __device__ constexpr int64_t mma_gu_item_bytes(int D) { return 4 * (int64_t)D + 64; }
__host__ __device__ constexpr int64_t mma_dn_item_bytes(int D, int F) { return 4 * (int64_t)D + 64 * (int64_t)(D / F); }
__host__ __device__ constexpr int mma_gu_items(int F) { return F / 8; }
__host__ __device__ constexpr int mma_dn_items(int F) { return F / 16; }

// map an interchange code to the offset code t + 1 (invalid 3 -> value 0 -> 1)
__host__ __device__ inline uint32_t offset_code(uint32_t code)
{
    return code == 1u ? 2u : (code == 2u ? 0u : 1u);
}

// word position of 4-byte word w (0..31) of a 128-column block in the fragment order
__host__ __device__ inline int frag_word_pos(int w)
{
    const int q = w >> 3, h = (w >> 2) & 1, c = w & 3;
    return c * 8 + q * 2 + h;
}

// tile row (0..15) whose codes sit in word i of lane `lane`
__host__ __device__ inline int mma_word_row(int lane, int i) { return (lane >> 2) + 8 * (i & 1); }

// the MMA-tile word (lane, word i) of k-block kb from the interchange words of
// its row (src = that row's words, mma_word_row(lane, i) of the tile)
__host__ __device__ inline uint32_t mma_word(const uint32_t *src, int lane, int i, int kb)
{
    const int c = lane & 3;
    uint32_t out = 0;
    for (int q = 0; q < 4; q++) {
        // columns 128kb + 32q + 16(i/2) + 4c + j (j = 0..3): one interchange word,
        // positions 4c + j
        const uint32_t w = src[kb * 8 + q * 2 + (i >> 1)];
        for (int j = 0; j < 4; j++)
            out |= offset_code((w >> (2 * (4 * c + j))) & 3u) << (8 * j + 2 * q);
    }
    return out;
}

}  // namespace maple
