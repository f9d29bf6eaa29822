// 2-bit ternary packer and the re-layout of packed weights into the GEMV
// layout (run once, at create).
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

// gate/up interchange [E][F][D/16] (two tensors) -> GEMV layout; one thread per output word
__global__ void repack_gu_kernel(const uint32_t *gate, const uint32_t *up, int E, int D, int F, uint32_t *out)
{
    const int C = D / 64, G = F / 16;
    const int64_t n = (int64_t)E * G * C * 32 * 4;
    for (int64_t o = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; o < n; o += (int64_t)gridDim.x * blockDim.x) {
        int64_t q = o;
        const int w = q % 4; q /= 4;
        const int lane = q % 32; q /= 32;
        const int c = q % C; q /= C;
        const int g = q % G; q /= G;
        const int e = (int)q;
        const int r = 16 * g + (lane & 15);
        const uint32_t *src = (lane < 16 ? gate : up) + ((int64_t)e * F + r) * (D / 16);
        out[o] = gemv_word(src[4 * c + w]);
    }
}

// down interchange [E][D][F/16] -> GEMV layout
__global__ void repack_dn_kernel(const uint32_t *down, int E, int D, int F, uint32_t *out)
{
    const int C = F / 64, G = D / 32;
    const int64_t n = (int64_t)E * G * C * 32 * 4;
    for (int64_t o = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; o < n; o += (int64_t)gridDim.x * blockDim.x) {
        int64_t q = o;
        const int w = q % 4; q /= 4;
        const int lane = q % 32; q /= 32;
        const int c = q % C; q /= C;
        const int g = q % G; q /= G;
        const int e = (int)q;
        const int row = 32 * g + lane;
        const uint32_t *src = down + ((int64_t)e * D + row) * (F / 16);
        out[o] = gemv_word(src[4 * c + w]);
    }
}

// residual stream -> bf16(RMSNorm(resid)); one warp per token.  Sum of squares
// in the router's order: lane l takes j = 256*i + 8*l + m (fmaf), xor tree.
__global__ void rmsnorm_bf16_kernel(const float *resid, int T, int D, uint16_t *out)
{
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
    if (t >= T) return;
    const float *r = resid + (size_t)t * D;
    float acc = 0.0f;
    for (int i = 0; i < D / 256; i++) {
        const float4 v0 = *reinterpret_cast<const float4 *>(r + 256 * i + 8 * lane);
        const float4 v1 = *reinterpret_cast<const float4 *>(r + 256 * i + 8 * lane + 4);
        const float v[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
        for (int m = 0; m < 8; m++) acc = __fmaf_rn(v[m], v[m], acc);
    }
    const float ms = __fdiv_rn(warp_tree_sum(acc), (float)D);
    const float rms = __fsqrt_rn(__fadd_rn(ms, 1e-6f));
    for (int i = 0; i < D / 256; i++) {
        const float4 v0 = *reinterpret_cast<const float4 *>(r + 256 * i + 8 * lane);
        const float4 v1 = *reinterpret_cast<const float4 *>(r + 256 * i + 8 * lane + 4);
        const float v[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
        uint32_t pk[4];
#pragma unroll
        for (int m = 0; m < 4; m++)
            pk[m] = (uint32_t)f32_to_bf16_bits(__fdiv_rn(v[2 * m], rms)) |
                    ((uint32_t)f32_to_bf16_bits(__fdiv_rn(v[2 * m + 1], rms)) << 16);
        *reinterpret_cast<uint4 *>(out + (size_t)t * D + 256 * i + 8 * lane) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    }
}

}  // namespace maple
