// 2-bit ternary packer, the re-layout of packed weights into the decode
// kernel's MMA-tile layout (run once, at create), and the stack's RMSNorm.
#pragma once

#include "common.cuh"
#include "layout.cuh"

namespace maple {

// values [rows][cols] int8 in {-1,0,1} -> packed [rows][cols/16]; one thread per word
__global__ void pack_ternary_kernel(const int8_t *values, int64_t n_words, uint32_t *packed, int *bad_count)
{
    for (int64_t w = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; w < n_words; w += (int64_t)gridDim.x * blockDim.x) {
        const uint4 v = reinterpret_cast<const uint4 *>(values)[w];
        const uint32_t b[4] = {v.x, v.y, v.z, v.w};
        uint32_t word = 0;
        int bad = 0;
#pragma unroll
        for (int i = 0; i < 16; i++) {
            const int8_t t = (int8_t)((b[i >> 2] >> (8 * (i & 3))) & 0xffu);
            uint32_t code = 0;
            if (t == 1) code = 1;
            else if (t == -1) code = 2;
            else if (t != 0) bad++;
            word |= code << (2 * i);
        }
        packed[w] = word;
        if (bad && bad_count) atomicAdd(bad_count, bad);
    }
}

// gate/up interchange -> MMA-tile layout (layout.cuh); one thread per code word
__global__ void repack_mma_gu_kernel(const uint32_t *gate, const uint32_t *up, int E, int D, int F, uint32_t *out)
{
    const int KB = D / 128, NT = mma_gu_items(F);
    const int64_t item_words = mma_gu_item_bytes(D) / 4;
    const int64_t n = (int64_t)E * NT * KB * 128;
    for (int64_t o = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; o < n; o += (int64_t)gridDim.x * blockDim.x) {
        int64_t q = o;
        const int i = q % 4; q /= 4;
        const int lane = q % 32; q /= 32;
        const int kb = q % KB; q /= KB;
        const int t = q % NT; q /= NT;
        const int e = (int)q;
        const int r = mma_word_row(lane, i);   // rows 0..7 gate, 8..15 up, outputs 8t .. 8t+7
        const uint32_t *src = (r < 8 ? gate : up) + ((int64_t)e * F + 8 * t + (r & 7)) * (D / 16);
        out[((int64_t)e * NT + t) * item_words + (kb * 32 + lane) * 4 + i] = mma_word(src, lane, i, kb);
    }
}

// down interchange -> MMA-tile layout; one thread per code word
__global__ void repack_mma_dn_kernel(const uint32_t *down, int E, int D, int F, uint32_t *out)
{
    const int KB = F / 128, NT = D / 16, S2 = D / F, NI = mma_dn_items(F);
    const int64_t item_words = mma_dn_item_bytes(D, F) / 4;
    const int64_t n = (int64_t)E * NT * KB * 128;
    for (int64_t o = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; o < n; o += (int64_t)gridDim.x * blockDim.x) {
        int64_t q = o;
        const int i = q % 4; q /= 4;
        const int lane = q % 32; q /= 32;
        const int kb = q % KB; q /= KB;
        const int t = q % NT; q /= NT;
        const int e = (int)q;
        const uint32_t *src = down + ((int64_t)e * D + 16 * t + mma_word_row(lane, i)) * (F / 16);
        out[((int64_t)e * NI + t / S2) * item_words + (int64_t)(t % S2) * F + (kb * 32 + lane) * 4 + i] =
            mma_word(src, lane, i, kb);
    }
}

// the row scales behind the codes of every MMA-tile item: gate/up item t of
// expert e ends in alpha_gate[e][8t..8t+7], alpha_up[e][8t..8t+7]; down item t
// in alpha_down[e][16*S2*t ..] (16*S2 values); one thread per value
__global__ void mma_item_scales_kernel(const float *alpha_gate, const float *alpha_up, const float *alpha_down, int E,
                                       int D, int F, float *gu, float *dn)
{
    const int S2 = D / F;
    const int64_t gu_words = mma_gu_item_bytes(D) / 4, dn_words = mma_dn_item_bytes(D, F) / 4;
    const int64_t n_gu = (int64_t)E * F * 2, n = n_gu + (int64_t)E * D;
    for (int64_t o = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; o < n; o += (int64_t)gridDim.x * blockDim.x) {
        if (o < n_gu) {   // (e, output f, gate|up)
            const int64_t e = o / (2 * F);
            const int f = (int)(o / 2 % F), m = (int)(o & 1);
            const float v = (m ? alpha_up : alpha_gate)[e * F + f];
            gu[(e * mma_gu_items(F) + f / 8) * gu_words + D + 8 * m + (f & 7)] = v;
        } else {          // (e, channel c)
            const int64_t q = o - n_gu, e = q / D;
            const int c = (int)(q % D);
            dn[(e * mma_dn_items(F) + c / (16 * S2)) * dn_words + D + c % (16 * S2)] = alpha_down[q];
        }
    }
}

// residual stream -> bf16(RMSNorm(resid)); one warp per token.  Sum of squares
// in the router's order: lane l takes j = 256*i + 8*l + m (fmaf), xor tree.
__global__ void rmsnorm_bf16_kernel(const float *resid, int T, int D, uint16_t *out)
{
    const int t = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
    if (t >= T) return;
    rmsnorm_token_warp(resid + (size_t)t * D, D, out + (size_t)t * D);
}

}  // namespace maple
