// Weight-streaming expert kernels (decode, small T): gate/up ternary GEMV with
// SwiGLU, per-slot requantisation, down ternary GEMV with the weighted
// combine.  One warp owns 32 weight rows of one active expert (one row per
// lane, interleaved layout, coalesced 512-byte loads) and runs them against
// up to kGemvTokens of that expert's tokens at a time.
#pragma once

#include "common.cuh"
#include "layout.cuh"

namespace maple {

constexpr int kGemvTokens = 8;      // tokens per pass over an expert's rows
constexpr int kGemvWarps = 8;       // warps per CTA

struct GemvArgs {
    int T, D, E, K, F;
    // expert list and permutation
    const int *active, *n_active, *counts, *offsets, *perm, *inv;
    const float *topk_w;
    // activations
    const int8_t *qx;
    const float *sx;
    const int *sumx;
    // weights
    const uint8_t *w_gu, *w_dn;
    const float *alpha_gate, *alpha_up, *alpha_down;
    // intermediates (perm order)
    float *h;          // [T*K][F]
    int8_t *qh;        // [T*K][F]
    float *sh;         // [T*K]
    int *sumqh;        // [T*K]
    float *ye;         // [T*K][D]
    // outputs
    float *y;            // [T][D]
    const float *resid;  // [T][D] or null: y = resid + combine
    // counters
    unsigned *exp_cnt;   // [E]
    unsigned *comb_cnt;  // [T][D/32]
    // taps (slot order, may be null)
    int *tap_acc_gate, *tap_acc_up, *tap_acc_down;
    int8_t *tap_qh;
    float *tap_sh;
};

// plane k of a GEMV word: the four offset codes of values 4k..4k+3, one per byte
__device__ __forceinline__ uint32_t plane(uint32_t w, int k) { return (w >> (2 * k)) & 0x03030303u; }

// acc += sum over the 64 values of one chunk (4 words of one row) against the
// 64 int8 activations at xp
__device__ __forceinline__ int chunk_dot(const uint32_t (&pw)[16], const int8_t *xp, int acc)
{
    const uint4 *x4 = reinterpret_cast<const uint4 *>(xp);
#pragma unroll
    for (int w = 0; w < 4; w++) {
        const uint4 xv = __ldg(x4 + w);
        acc = dp4a_us(pw[4 * w + 0], xv.x, acc);
        acc = dp4a_us(pw[4 * w + 1], xv.y, acc);
        acc = dp4a_us(pw[4 * w + 2], xv.z, acc);
        acc = dp4a_us(pw[4 * w + 3], xv.w, acc);
    }
    return acc;
}

// Run 32 rows (this lane: one row) of nchunks 64-value chunks against nb
// token rows.  wrow: this lane's chunk 0 (chunk stride 512 bytes); xrow[j]:
// token j's activation row (chunk c at xrow[j] + 64*c).
template <int U>
__device__ __forceinline__ void rows_dot(const uint8_t *wrow, int nchunks, const int8_t *const (&xrow)[kGemvTokens],
                                         int nb, int (&acc)[kGemvTokens])
{
    uint4 cur[U], nxt[U];
#pragma unroll
    for (int u = 0; u < U; u++) cur[u] = ld_stream_v4(wrow + (size_t)u * 512);
    for (int c0 = 0; c0 < nchunks; c0 += U) {
        const bool more = c0 + U < nchunks;
#pragma unroll
        for (int u = 0; u < U; u++)
            if (more) nxt[u] = ld_stream_v4(wrow + (size_t)(c0 + U + u) * 512);
#pragma unroll
        for (int u = 0; u < U; u++) {
            const uint32_t wv[4] = {cur[u].x, cur[u].y, cur[u].z, cur[u].w};
            uint32_t pw[16];
#pragma unroll
            for (int w = 0; w < 4; w++)
#pragma unroll
                for (int k = 0; k < 4; k++) pw[4 * w + k] = plane(wv[w], k);
            const int c = c0 + u;
#pragma unroll
            for (int j = 0; j < kGemvTokens; j++)
                if (j < nb) acc[j] = chunk_dot(pw, xrow[j] + 64 * c, acc[j]);
        }
#pragma unroll
        for (int u = 0; u < U; u++) cur[u] = nxt[u];
    }
}

// requantise every slot of expert e (positions [base, base+cnt)) from h; one warp
__device__ void requant_expert_warp(const GemvArgs &a, int base, int cnt)
{
    const int lane = threadIdx.x & 31;
    for (int p = base; p < base + cnt; p++) {
        const float4 *hr = reinterpret_cast<const float4 *>(a.h + (size_t)p * a.F);
        float amax = 0.0f;
        for (int i = lane; i < a.F / 4; i += 32) {
            float4 v = __ldcg(hr + i);
            amax = fmaxf(fmaxf(fmaxf(amax, fabsf(v.x)), fmaxf(fabsf(v.y), fabsf(v.z))), fabsf(v.w));
        }
        amax = warp_max(amax);
        const float inv = amax > 0.0f ? __fdiv_rn(127.0f, amax) : 0.0f;
        const int slot = a.perm[p];
        int sum = 0;
        for (int i = lane; i < a.F / 4; i += 32) {
            float4 v = __ldcg(hr + i);
            int q0 = 0, q1 = 0, q2 = 0, q3 = 0;
            if (amax > 0.0f) {
                q0 = quant_code(v.x, inv);
                q1 = quant_code(v.y, inv);
                q2 = quant_code(v.z, inv);
                q3 = quant_code(v.w, inv);
            }
            sum += q0 + q1 + q2 + q3;
            const uint32_t pk = (uint32_t)(q0 & 0xff) | ((uint32_t)(q1 & 0xff) << 8) | ((uint32_t)(q2 & 0xff) << 16) |
                                ((uint32_t)(q3 & 0xff) << 24);
            reinterpret_cast<uint32_t *>(a.qh + (size_t)p * a.F)[i] = pk;
            if (a.tap_qh) reinterpret_cast<uint32_t *>(a.tap_qh + (size_t)slot * a.F)[i] = pk;
        }
        sum = warp_sum_int(sum);
        if (lane == 0) {
            const float s = amax > 0.0f ? __fdiv_rn(amax, 127.0f) : 0.0f;
            a.sh[p] = s;
            a.sumqh[p] = sum;
            if (a.tap_sh) a.tap_sh[slot] = s;
        }
    }
}

// ---------------------------------------------------------------------------
// gate/up: warp item (active expert, group of 16 gate + 16 up rows)
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kGemvWarps * 32) gateup_gemv_kernel(GemvArgs a)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int G = a.F / 16, C = a.D / 64;
    const int n_items = __ldg(a.n_active) * G;
    const int nwarps = gridDim.x * kGemvWarps;
    for (int item = warp * gridDim.x + blockIdx.x; item < n_items; item += nwarps) {
        const int ai = item / G, g = item - ai * G;
        const int e = a.active[ai];
        const int cnt = a.counts[e], base = a.offsets[e];
        const uint8_t *wrow = a.w_gu + (size_t)e * gu_bytes_per_expert(a.D, a.F) + (size_t)g * C * 512 + lane * 16;
        const int r = g * 16 + (lane & 15);
        const bool is_up = lane >= 16;
        const float alpha = is_up ? a.alpha_up[(size_t)e * a.F + r] : a.alpha_gate[(size_t)e * a.F + r];
        for (int b0 = 0; b0 < cnt; b0 += kGemvTokens) {
            const int nb = min(kGemvTokens, cnt - b0);
            const int my_slot = lane < nb ? a.perm[base + b0 + lane] : 0;
            int slot[kGemvTokens];
            const int8_t *xrow[kGemvTokens];
            int acc[kGemvTokens];
#pragma unroll
            for (int j = 0; j < kGemvTokens; j++) {
                slot[j] = __shfl_sync(FULL, my_slot, j);
                xrow[j] = a.qx + (size_t)(slot[j] / a.K) * a.D;
                acc[j] = 0;
            }
            rows_dot<4>(wrow, C, xrow, nb, acc);
#pragma unroll
            for (int j = 0; j < kGemvTokens; j++) {
                if (j < nb) {
                    const int t = slot[j] / a.K;
                    const int av = acc[j] - a.sumx[t];
                    const float v = __fmul_rn((float)av, __fmul_rn(alpha, a.sx[t]));
                    const float u = __shfl_down_sync(FULL, v, 16);
                    if (!is_up) a.h[(size_t)(base + b0 + j) * a.F + r] = swiglu(v, u);
                    int *tap = is_up ? a.tap_acc_up : a.tap_acc_gate;
                    if (tap) tap[(size_t)slot[j] * a.F + r] = av;
                }
            }
        }
        // the last warp to finish a group of expert e requantises e's slots
        __threadfence();
        __syncwarp();
        unsigned prev = 0;
        if (lane == 0) prev = atomicAdd(a.exp_cnt + e, 1u);
        prev = __shfl_sync(FULL, prev, 0);
        if (prev == (unsigned)(G - 1)) {
            __threadfence();
            if (lane == 0) a.exp_cnt[e] = 0;
            requant_expert_warp(a, base, cnt);
        }
    }
}

// ---------------------------------------------------------------------------
// down: warp item (active expert, group of 32 output channels); the last of a
// token's K slots to arrive for a group combines that token's 32 channels
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kGemvWarps * 32) down_gemv_kernel(GemvArgs a)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int G = a.D / 32, C = a.F / 64;
    const int n_items = __ldg(a.n_active) * G;
    const int nwarps = gridDim.x * kGemvWarps;
    for (int item = warp * gridDim.x + blockIdx.x; item < n_items; item += nwarps) {
        const int ai = item / G, g = item - ai * G;
        const int e = a.active[ai];
        const int cnt = a.counts[e], base = a.offsets[e];
        const uint8_t *wrow = a.w_dn + (size_t)e * dn_bytes_per_expert(a.D, a.F) + (size_t)g * C * 512 + lane * 16;
        const int c = g * 32 + lane;
        const float alpha = a.alpha_down[(size_t)e * a.D + c];
        for (int b0 = 0; b0 < cnt; b0 += kGemvTokens) {
            const int nb = min(kGemvTokens, cnt - b0);
            const int my_slot = lane < nb ? a.perm[base + b0 + lane] : 0;
            const int8_t *xrow[kGemvTokens];
            int acc[kGemvTokens];
#pragma unroll
            for (int j = 0; j < kGemvTokens; j++) {
                xrow[j] = a.qh + (size_t)(base + b0 + j) * a.F;
                acc[j] = 0;
            }
            rows_dot<2>(wrow, C, xrow, nb, acc);
#pragma unroll
            for (int j = 0; j < kGemvTokens; j++) {
                if (j < nb) {
                    const int p = base + b0 + j;
                    const int av = acc[j] - a.sumqh[p];
                    a.ye[(size_t)p * a.D + c] = __fmul_rn((float)av, __fmul_rn(alpha, a.sh[p]));
                    if (a.tap_acc_down) a.tap_acc_down[(size_t)__shfl_sync(FULL, my_slot, j) * a.D + c] = av;
                }
            }
            // arrivals: lane j < nb counts slot j's token for this group
            __threadfence();
            __syncwarp();
            const int my_t = my_slot / a.K;
            unsigned prev = 0;
            if (lane < nb) prev = atomicAdd(a.comb_cnt + (size_t)my_t * G + g, 1u);
            unsigned done = __ballot_sync(FULL, lane < nb && prev == (unsigned)(a.K - 1));
            if (done) __threadfence();
            while (done) {
                const int j = __ffs(done) - 1;
                done &= done - 1;
                const int t = __shfl_sync(FULL, my_t, j);
                if (lane == j) a.comb_cnt[(size_t)t * G + g] = 0;
                float yv = 0.0f;
                for (int k = 0; k < a.K; k++) {
                    const int s = t * a.K + k;
                    const float ev = __ldcg(a.ye + (size_t)a.inv[s] * a.D + c);
                    yv = __fmaf_rn(a.topk_w[s], ev, yv);
                }
                const size_t o = (size_t)t * a.D + c;
                a.y[o] = a.resid ? __fadd_rn(a.resid[o], yv) : yv;
            }
        }
    }
}

}  // namespace maple
