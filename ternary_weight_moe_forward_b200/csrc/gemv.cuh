// Weight-streaming expert kernels (decode, small T): gate/up ternary GEMV with
// SwiGLU, per-slot requantisation, down ternary GEMV with the weighted
// combine.  A warp streams 32 weight rows of one active expert (one row per
// lane, interleaved layout, coalesced 512-byte loads, all of its chunks in
// flight at once) over a slice of K, and runs them against up to kGemvTokens
// of that expert's tokens at a time, whose int8 rows sit in shared memory.
// The int32 partial sums of the K slices are added in shared memory (exact in
// any order).
#pragma once

#include "common.cuh"
#include "layout.cuh"
#include "route.cuh"

namespace maple {

constexpr int kGemvTokens = 8;      // tokens per pass over an expert's rows
constexpr int kGemvWarps = 8;       // warps per CTA
#ifndef MAPLE_GEMV_MINB
#define MAPLE_GEMV_MINB 2  // resident CTAs per SM the register budget is cut for
#endif

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
    unsigned *comb_cnt;  // [T][D/128]
    // taps (slot order, may be null)
    int *tap_acc_gate, *tap_acc_up, *tap_acc_down;
    int8_t *tap_qh;
    float *tap_sh;
    unsigned *flag_dev;  // device flag word (timeouts)
};

__device__ __forceinline__ uint64_t global_timer_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// dynamic shared memory of the two kernels: activation rows + partial sums
__host__ __device__ inline size_t gemv_smem_bytes(int row_bytes)
{
    return (size_t)kGemvTokens * row_bytes + (size_t)kGemvWarps * kGemvTokens * 32 * 4;
}

// plane k of a GEMV word: the four offset codes of values 4k..4k+3, one per byte
__device__ __forceinline__ uint32_t plane(uint32_t w, int k) { return (w >> (2 * k)) & 0x03030303u; }

// acc[j] += sum over the 64 values of one chunk (this lane's row) against token
// j's 64 activations at xs + j*ld + off, for j < nb
__device__ __forceinline__ void chunk_tokens(const uint4 wv, const int8_t *xs, int ld, int off, int nb,
                                             int (&acc)[kGemvTokens])
{
    const uint32_t w4[4] = {wv.x, wv.y, wv.z, wv.w};
    uint32_t pw[16];
#pragma unroll
    for (int w = 0; w < 4; w++)
#pragma unroll
        for (int k = 0; k < 4; k++) pw[4 * w + k] = plane(w4[w], k);
#pragma unroll
    for (int j = 0; j < kGemvTokens; j++) {
        if (j < nb) {
            const uint4 *x4 = reinterpret_cast<const uint4 *>(xs + (size_t)j * ld + off);
#pragma unroll
            for (int w = 0; w < 4; w++) {
                const uint4 xv = x4[w];
                acc[j] = dp4a_us(pw[4 * w + 0], xv.x, acc[j]);
                acc[j] = dp4a_us(pw[4 * w + 1], xv.y, acc[j]);
                acc[j] = dp4a_us(pw[4 * w + 2], xv.z, acc[j]);
                acc[j] = dp4a_us(pw[4 * w + 3], xv.w, acc[j]);
            }
        }
    }
}

// Padded token count of a decode batch: the dot kernels below exist for 1, 2
// and 4 tokens (8 = two passes of 4); rows nb..nbp-1 of the batch hold zeros.
__device__ __forceinline__ int dec_pad_tokens(int nb) { return nb <= 1 ? 1 : nb <= 2 ? 2 : nb <= 4 ? 4 : 8; }

// Sum over chunks [c0, c0+nch) of this lane's row against NB token rows (16-byte
// units x[j*ld16 + 4c + w]).  Byte plane k is taken as w & (0x03030303 << 2k),
// i.e. 4^k times the offset codes, one logic op per plane, and gets its own
// accumulator; acc_k is then an exact multiple of 4^k and the row total is
// acc_0 + acc_1/4 + acc_2/16 + acc_3/64 (int32, exact).  Token j's total goes
// to out[32 j].
template <int NB>
__device__ __forceinline__ void dot_rows(const uint4 *wl, const uint4 *x, int ld16, int c0, int nch, int *out)
{
    int acc[NB][4];
#pragma unroll
    for (int j = 0; j < NB; j++)
#pragma unroll
        for (int k = 0; k < 4; k++) acc[j][k] = 0;
    const uint4 *wr = wl + 32 * c0;
    const uint4 *xr = x + 4 * c0;
#pragma unroll 1
    for (int u = 0; u < nch; u++) {
        const uint4 wv = wr[32 * u];
        const uint32_t w4[4] = {wv.x, wv.y, wv.z, wv.w};
        uint32_t pw[16];
#pragma unroll
        for (int w = 0; w < 4; w++)
#pragma unroll
            for (int k = 0; k < 4; k++) pw[4 * w + k] = w4[w] & (0x03030303u << (2 * k));
#pragma unroll
        for (int j = 0; j < NB; j++) {
#pragma unroll
            for (int w = 0; w < 4; w++) {
                const uint4 xv = xr[j * ld16 + 4 * u + w];
                acc[j][0] = dp4a_us(pw[4 * w + 0], xv.x, acc[j][0]);
                acc[j][1] = dp4a_us(pw[4 * w + 1], xv.y, acc[j][1]);
                acc[j][2] = dp4a_us(pw[4 * w + 2], xv.z, acc[j][2]);
                acc[j][3] = dp4a_us(pw[4 * w + 3], xv.w, acc[j][3]);
            }
        }
    }
#pragma unroll
    for (int j = 0; j < NB; j++) out[32 * j] = acc[j][0] + (acc[j][1] >> 2) + (acc[j][2] >> 4) + (acc[j][3] >> 6);
}

__device__ __forceinline__ void dot_rows_any(int nbp, const uint4 *wl, const uint4 *x, int ld16, int c0, int nch,
                                             int *out)
{
    switch (nbp) {
    case 1: dot_rows<1>(wl, x, ld16, c0, nch, out); break;
    case 2: dot_rows<2>(wl, x, ld16, c0, nch, out); break;
    case 4: dot_rows<4>(wl, x, ld16, c0, nch, out); break;
    default:   // two passes of four tokens keep the accumulators in registers
        dot_rows<4>(wl, x, ld16, c0, nch, out);
        dot_rows<4>(wl, x + 4 * ld16, ld16, c0, nch, out + 4 * 32);
        break;
    }
}

// requantise every slot of an expert (positions [base, base+cnt)) from h; the
// first nw warps of the CTA take one slot each
__device__ void requant_slots_warps(const GemvArgs &a, int base, int cnt, int nw)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (warp >= nw) return;
    for (int p = base + warp; p < base + cnt; p += nw) {
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
// gate/up.  CTA = (active expert, pair of row groups, each 16 gate + 16 up
// rows); warp w takes group w/4 and K quarter w%4 (NI chunks of 64 values,
// loaded up front).  The last CTA of an expert to finish requantises that
// expert's slots.
// ---------------------------------------------------------------------------
template <int NI>
__global__ void __launch_bounds__(kGemvWarps * 32, MAPLE_GEMV_MINB) gateup_gemv_kernel(GemvArgs a)
{
    extern __shared__ __align__(16) uint8_t gsm[];
    int8_t *xs = (int8_t *)gsm;                               // [kGemvTokens][D]
    int *red = (int *)(gsm + (size_t)kGemvTokens * a.D);      // [8 warps][kGemvTokens][32]
    __shared__ int s_slot[kGemvTokens];
    __shared__ unsigned s_last;

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int G = a.F / 16, pairs = G / 2, C = a.D / 64;
    const int ai = blockIdx.x / pairs;
    if (ai >= __ldg(a.n_active)) return;
    const int e = a.active[ai];
    const int g = 2 * (blockIdx.x % pairs) + (warp >> 2), kq = warp & 3;
    const int cnt = a.counts[e], base = a.offsets[e];

    const uint8_t *wrow = a.w_gu + (size_t)e * gu_bytes_per_expert(a.D, a.F) + (size_t)g * C * 512 + lane * 16;
    uint4 wv[NI];
#pragma unroll
    for (int u = 0; u < NI; u++) wv[u] = ld_stream_v4(wrow + (size_t)(kq * NI + u) * 512);

    const int r = g * 16 + (lane & 15);
    const bool is_up = lane >= 16;
    const float alpha = is_up ? a.alpha_up[(size_t)e * a.F + r] : a.alpha_gate[(size_t)e * a.F + r];

    for (int b0 = 0; b0 < cnt; b0 += kGemvTokens) {
        const int nb = min(kGemvTokens, cnt - b0);
        if (threadIdx.x < nb) s_slot[threadIdx.x] = a.perm[base + b0 + threadIdx.x];
        __syncthreads();
        const int row16 = a.D / 16;
        for (int i = threadIdx.x; i < nb * row16; i += blockDim.x) {
            const int j = i / row16, c16 = i - j * row16;
            reinterpret_cast<uint4 *>(xs + (size_t)j * a.D)[c16] =
                __ldg(reinterpret_cast<const uint4 *>(a.qx + (size_t)(s_slot[j] / a.K) * a.D) + c16);
        }
        __syncthreads();
        int acc[kGemvTokens];
#pragma unroll
        for (int j = 0; j < kGemvTokens; j++) acc[j] = 0;
#pragma unroll
        for (int u = 0; u < NI; u++) chunk_tokens(wv[u], xs, a.D, 64 * (kq * NI + u), nb, acc);
#pragma unroll
        for (int j = 0; j < kGemvTokens; j++) red[(warp * kGemvTokens + j) * 32 + lane] = acc[j];
        __syncthreads();
        if (warp < 2) {
            // warp w finalises group 2*pair + w (its K quarters are warps 4w .. 4w+3)
            const int rr = (2 * (blockIdx.x % pairs) + warp) * 16 + (lane & 15);
            const float al = is_up ? a.alpha_up[(size_t)e * a.F + rr] : a.alpha_gate[(size_t)e * a.F + rr];
            for (int j = 0; j < nb; j++) {
                int sum = 0;
#pragma unroll
                for (int q = 0; q < 4; q++) sum += red[((warp * 4 + q) * kGemvTokens + j) * 32 + lane];
                const int slot = s_slot[j], t = slot / a.K;
                const int av = sum - a.sumx[t];
                const float v = __fmul_rn((float)av, __fmul_rn(al, a.sx[t]));
                const float uu = __shfl_down_sync(FULL, v, 16);
                if (!is_up) a.h[(size_t)(base + b0 + j) * a.F + rr] = swiglu(v, uu);
                int *tap = is_up ? a.tap_acc_up : a.tap_acc_gate;
                if (tap) tap[(size_t)slot * a.F + rr] = av;
            }
        }
        __syncthreads();
    }
    (void)alpha;
    (void)r;

    // the last CTA of expert e to finish requantises e's slots
    fence_gpu();
    __syncthreads();
    if (threadIdx.x == 0) s_last = atomicAdd(a.exp_cnt + e, 1u) == (unsigned)(pairs - 1);
    __syncthreads();
    if (!s_last) return;
    fence_gpu();
    if (threadIdx.x == 0) a.exp_cnt[e] = 0;
    requant_slots_warps(a, base, cnt, blockDim.x >> 5);
}

// ---------------------------------------------------------------------------
// down.  CTA = (active expert, block of 128 output channels); warp w takes
// channel group 4*blk + w/2 and K half w%2.  The q_h rows of the expert's
// slots (consecutive positions) are staged in shared memory.  Every slot adds
// one arrival on (token, channel block); the K-th arrival combines that
// token's 128 channels in rank order.
// ---------------------------------------------------------------------------
template <int NH>
__global__ void __launch_bounds__(kGemvWarps * 32, MAPLE_GEMV_MINB) down_gemv_kernel(GemvArgs a)
{
    extern __shared__ __align__(16) uint8_t gsm[];
    int8_t *xs = (int8_t *)gsm;                               // [kGemvTokens][F]
    int *red = (int *)(gsm + (size_t)kGemvTokens * a.F);      // [8 warps][kGemvTokens][32]
    __shared__ int s_slot[kGemvTokens];
    __shared__ int s_done[kGemvTokens];

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int blocks = a.D / 128, C = a.F / 64;
    const int ai = blockIdx.x / blocks;
    if (ai >= __ldg(a.n_active)) return;
    const int e = a.active[ai];
    const int blk = blockIdx.x % blocks;
    const int g = blk * 4 + (warp >> 1), kh = warp & 1;
    const int cnt = a.counts[e], base = a.offsets[e];

    const uint8_t *wrow = a.w_dn + (size_t)e * dn_bytes_per_expert(a.D, a.F) + (size_t)g * C * 512 + lane * 16;
    uint4 wv[NH];
#pragma unroll
    for (int u = 0; u < NH; u++) wv[u] = ld_stream_v4(wrow + (size_t)(kh * NH + u) * 512);

    for (int b0 = 0; b0 < cnt; b0 += kGemvTokens) {
        const int nb = min(kGemvTokens, cnt - b0);
        if (threadIdx.x < nb) s_slot[threadIdx.x] = a.perm[base + b0 + threadIdx.x];
        const int n16 = nb * a.F / 16;
        for (int i = threadIdx.x; i < n16; i += blockDim.x)
            reinterpret_cast<uint4 *>(xs)[i] = __ldg(reinterpret_cast<const uint4 *>(a.qh + (size_t)(base + b0) * a.F) + i);
        __syncthreads();
        int acc[kGemvTokens];
#pragma unroll
        for (int j = 0; j < kGemvTokens; j++) acc[j] = 0;
#pragma unroll
        for (int u = 0; u < NH; u++) chunk_tokens(wv[u], xs, a.F, 64 * (kh * NH + u), nb, acc);
#pragma unroll
        for (int j = 0; j < kGemvTokens; j++) red[(warp * kGemvTokens + j) * 32 + lane] = acc[j];
        __syncthreads();
        if (warp < 4) {
            // warp w finalises channel group 4*blk + w (its K halves are warps 2w, 2w+1)
            const int cg = (blk * 4 + warp) * 32 + lane;
            const float al = a.alpha_down[(size_t)e * a.D + cg];
            for (int j = 0; j < nb; j++) {
                const int p = base + b0 + j;
                const int sum = red[((2 * warp) * kGemvTokens + j) * 32 + lane] +
                                red[((2 * warp + 1) * kGemvTokens + j) * 32 + lane];
                const int av = sum - a.sumqh[p];
                a.ye[(size_t)p * a.D + cg] = __fmul_rn((float)av, __fmul_rn(al, a.sh[p]));
                if (a.tap_acc_down) a.tap_acc_down[(size_t)s_slot[j] * a.D + cg] = av;
            }
        }
        // arrivals on (token, channel block)
        fence_gpu();
        __syncthreads();
        if (threadIdx.x < nb) {
            const int t = s_slot[threadIdx.x] / a.K;
            const unsigned prev = atomicAdd(a.comb_cnt + (size_t)t * blocks + blk, 1u);
            s_done[threadIdx.x] = prev == (unsigned)(a.K - 1);
        }
        __syncthreads();
        for (int j = 0; j < nb; j++) {
            if (!s_done[j]) continue;
            fence_gpu();
            const int t = s_slot[j] / a.K;
            if (threadIdx.x < 128) {
                const int cc = blk * 128 + threadIdx.x;
                float yv = 0.0f;
                for (int k = 0; k < a.K; k++) {
                    const int s = t * a.K + k;
                    yv = __fmaf_rn(a.topk_w[s], __ldcg(a.ye + (size_t)a.inv[s] * a.D + cc), yv);
                }
                const size_t o = (size_t)t * a.D + cc;
                a.y[o] = a.resid ? __fadd_rn(a.resid[o], yv) : yv;
            }
            if (threadIdx.x == 0) a.comb_cnt[(size_t)t * blocks + blk] = 0;
        }
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------
// Persistent weight-streaming kernel for the whole expert stage (decode).
//
// Grid = one CTA per SM, launched cooperatively (all CTAs resident).  Every
// CTA first builds the permutation of all T*K slots for itself from the
// router's top-k (in shared memory), so no routing step needs a grid-wide
// hand-off.  Work items: gate/up items (active expert, 32 gate + 32 up rows)
// then down items (active expert, 128 output channels); every CTA takes a
// contiguous range of each kind holding an equal share of its estimated cost
// (the cost of an item grows with its expert's token count).  Warp roles:
//   warp 0      streams the 2-bit codes and row scales of its items, in order,
//               with bulk copies into a ring of weight slots;
//   warps 1, 2  stage the activations of compute group 0 / 1 (double
//               buffered): for gate/up the int8 rows of the item's tokens, for
//               down the fp32 SwiGLU rows h of the item's slots once every
//               gate/up item of that expert has finished;
//   warps 3, 4  publish the results of group 0 / 1: make a finished gate/up
//               item visible (GPU fence, arrival counter of its expert), and for
//               a down item count each token's arrival on its channel block,
//               the last of the K arrivals combining that token's 128 channels;
//   warps 5..20 two compute groups of eight warps; group g takes items g, g+2,
//               ... of the CTA.
// Compute groups never wait on global memory: fences, atomics and the
// combine run on the publishing warps.  Down items requantise h locally (the
// same per-slot absmax int8 rule).  Every wait is bounded (2 s) and raises the
// device flag on expiry.
// ---------------------------------------------------------------------------
constexpr int kDecWSlots = 4;
constexpr int kDecGroups = 2;
constexpr int kDecGroupWarps = 8;
constexpr int kDecGroupThreads = kDecGroupWarps * 32;
constexpr int kDecRec = 4;   // completion records per group
constexpr int kDecFirstCompute = 1 + 2 * kDecGroups;
constexpr int kDecThreads = (kDecFirstCompute + kDecGroups * kDecGroupWarps) * 32;   // 672

struct DecActMeta {
    int nb, b0, base, e;
    int slot[kGemvTokens];
    float s[kGemvTokens];     // gate/up: s_x of the token
    int sum[kGemvTokens];     // gate/up: sum of the token's int8 codes
};
struct DecWMeta {
    int e, sub, kind, cnt, base;
};
struct DecRecord {            // one finished batch of a compute group
    int kind, e, sub, nb, base, last;
    int slot[kGemvTokens];
};

struct DecodeArgs {
    GemvArgs g;
    unsigned *arrive;     // [E] finished gate/up items per expert, zero at launch
    int wslot_bytes;      // codes + scales of one item
    int aslot_bytes;      // activation rows of one batch
    int nw;               // weight ring slots (2..kDecWSlots)
    const int8_t *zrow;   // D zero bytes (padding rows of a gate/up batch)
    const int *topk_idx;  // [T][K] the router's choices (distinct per token)
    const float *topk_w;  // [T][K] their softmax weights
    // outputs of the permutation, written by CTA 0 (may be null)
    int *tap_counts, *tap_offsets, *tap_perm;
};

__host__ __device__ inline int dec_wslot_bytes(int D, int F)
{
    const int g = 16 * D + 256, d = 32 * F + 512;
    return ((g > d ? g : d) + 127) & ~127;
}
__host__ __device__ inline int dec_aslot_bytes(int D, int F)
{
    const int g = kGemvTokens * D, d = kGemvTokens * F * 4;
    return ((g > d ? g : d) + 127) & ~127;
}
// routing tables every CTA builds for itself in shared memory
__host__ __device__ inline size_t dec_table_bytes(int T, int K, int E)
{
    return (size_t)4 * T * K * 4 + (size_t)(3 * E + 1) * 4 + (size_t)2 * T * 4 + 48 * 4 + 8 + (size_t)8 * E +
           (size_t)2 * (E + 1) * 4;
}
__host__ __device__ inline size_t dec_group_scratch_bytes(int F)
{
    return (size_t)kDecGroupWarps * kGemvTokens * 32 * 4 + (size_t)kGemvTokens * F + 2 * kGemvTokens * 4;
}
constexpr int kDecBars = 2 * kDecWSlots + 4 * kDecGroups + 2 * kDecRec * kDecGroups;
__host__ __device__ inline size_t decode_smem_bytes(int D, int F, int T, int K, int E, int nw)
{
    return (size_t)nw * dec_wslot_bytes(D, F) + (size_t)kDecGroups * 2 * dec_aslot_bytes(D, F) +
           kDecGroups * dec_group_scratch_bytes(F) + kDecGroups * 2 * sizeof(DecActMeta) +
           kDecWSlots * sizeof(DecWMeta) + kDecGroups * kDecRec * sizeof(DecRecord) + 8 * kDecBars + 64 +
           dec_table_bytes(T, K, E);
}

// bounded wait on an mbarrier phase (2 s); false on timeout
__device__ __forceinline__ bool dec_wait(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    const uint64_t t0 = global_timer_ns();
    while (true) {
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(bar), "r"(parity), "r"(kSuspendHintNs)
            : "memory");
        if (ok) return true;
        if (global_timer_ns() - t0 > 2000000000ull) return false;
    }
}
__device__ __forceinline__ void dec_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void dec_expect(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void dec_bulk(void *dst, const void *src, uint32_t bytes, uint32_t bar)
{
    const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst);
    for (uint32_t off = 0; off < bytes; off += 8192) {
        const uint32_t n = bytes - off < 8192 ? bytes - off : 8192;
        asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                         d + off),
                     "l"((const uint8_t *)src + off), "r"(n), "r"(bar)
                     : "memory");
    }
}

// Relative cost of one work item of an expert with c tokens (kind 0 gate/up, 1
// down): per batch of up to 8 tokens a fixed part (waits, barriers, epilogue)
// plus a part per padded token (the dot), in units of about 0.1 us measured on
// the decode-shape layer.  Only the split of the items over CTAs depends on it.
__device__ __forceinline__ int dec_item_cost(int c, int kind)
{
    int cost = 0;
    for (int b0 = 0; b0 < c; b0 += kGemvTokens) {
        const int nbp = dec_pad_tokens(min(kGemvTokens, c - b0));
        cost += kind == 0 ? 23 + 5 * nbp : 18 + 7 * nbp;
    }
    return cost;
}

// First item whose cumulative cost start is >= target; pref[ai] is the cost of
// the items of active experts before ai (per_exp items of equal cost each).
__device__ __forceinline__ int dec_item_at(const int *pref, int n_active, int per_exp, int64_t target)
{
    if (target >= pref[n_active]) return n_active * per_exp;
    int lo = 0, hi = n_active - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (pref[mid] <= target) lo = mid;
        else hi = mid - 1;
    }
    const int w = (pref[lo + 1] - pref[lo]) / per_exp;
    return lo * per_exp + (int)((target - pref[lo] + w - 1) / w);
}

__global__ void __launch_bounds__(kDecThreads, 1) decode_experts_kernel(DecodeArgs d)
{
    GemvArgs a = d.g;
    const int nw = d.nw;
    extern __shared__ __align__(1024) uint8_t dsm[];
    uint8_t *wring = dsm;
    uint8_t *aring = wring + (size_t)nw * d.wslot_bytes;                          // [group][2][aslot]
    uint8_t *gscr = aring + (size_t)kDecGroups * 2 * d.aslot_bytes;               // [group] scratch
    const size_t gscr_bytes = dec_group_scratch_bytes(a.F);
    DecActMeta *ameta = (DecActMeta *)(gscr + kDecGroups * gscr_bytes);           // [group][2]
    DecWMeta *wmeta = (DecWMeta *)(ameta + kDecGroups * 2);                       // [kDecWSlots]
    DecRecord *recs = (DecRecord *)(wmeta + kDecWSlots);                          // [group][kDecRec]
    uint64_t *bars = (uint64_t *)(((uintptr_t)(recs + kDecGroups * kDecRec) + 7) & ~(uintptr_t)7);
    // bars: wfull[W], wempty[W], afull[G][2], aempty[G][2], rfull[G][R], rempty[G][R]
    const uint32_t b_wfull = (uint32_t)__cvta_generic_to_shared(bars), b_wempty = b_wfull + 8 * kDecWSlots;
    const uint32_t b_afull = b_wempty + 8 * kDecWSlots, b_aempty = b_afull + 8 * 2 * kDecGroups;
    const uint32_t b_rfull = b_aempty + 8 * 2 * kDecGroups, b_rempty = b_rfull + 8 * kDecRec * kDecGroups;
    // routing tables
    const int T = a.T, K = a.K, E = a.E, S = a.T * a.K;
    int *t_idx = (int *)(bars + kDecBars);
    float *t_w = (float *)(t_idx + S);
    int *t_perm = (int *)(t_w + S);
    int *t_inv = t_perm + S;
    int *t_cnt = t_inv + S;
    int *t_off = t_cnt + E;
    int *t_act = t_off + E + 1;
    float *t_sx = (float *)(t_act + E);
    int *t_sumx = (int *)(t_sx + T);
    int *t_misc = t_sumx + T;   // [0] n_active, [8..40] scan scratch

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (threadIdx.x == 0) {
        for (int i = 0; i < kDecBars; i++)
            asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(b_wfull + 8 * i), "r"(1) : "memory");
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }

    // ---------------- prologue: the permutation of the T*K slots (T <= 64), from the
    // router's choices: a token bitmask per expert gives the counts, and a slot's
    // rank within its expert is the number of earlier tokens in that mask
    unsigned long long *tmask = (unsigned long long *)(((uintptr_t)(t_misc + 48) + 7) & ~(uintptr_t)7);
    const bool writer = blockIdx.x == 0;
    for (int e = threadIdx.x; e < E; e += blockDim.x) tmask[e] = 0ull;
    for (int q = threadIdx.x; q < S; q += blockDim.x) {
        t_idx[q] = __ldcg(d.topk_idx + q);
        t_w[q] = __ldcg(d.topk_w + q);
    }
    for (int t = threadIdx.x; t < T; t += blockDim.x) {
        t_sx[t] = __ldcg(a.sx + t);
        t_sumx[t] = __ldcg(a.sumx + t);
    }
    __syncthreads();
    for (int q = threadIdx.x; q < S; q += blockDim.x) {
        const int e = t_idx[q];
        if (e >= 0 && e < E)
            atomicOr(tmask + e, 1ull << (q / K));
        else if (writer)
            set_flag(a.flag_dev, MAPLE_DEVFLAG_BAD_INDEX);
    }
    __syncthreads();
    if (warp == 0) {
        const int per = (E + 31) / 32, e0 = lane * per;
        int csum = 0, asum = 0;
        for (int i = 0; i < per; i++) {
            const int e = e0 + i;
            if (e < E) {
                const int c = __popcll(tmask[e]);
                csum += c;
                asum += c > 0;
            }
        }
        int cs = csum, as = asum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(FULL, cs, o), w = __shfl_up_sync(FULL, as, o);
            if (lane >= o) {
                cs += v;
                as += w;
            }
        }
        int coff = cs - csum, aoff = as - asum;
        for (int i = 0; i < per; i++) {
            const int e = e0 + i;
            if (e < E) {
                const int c = __popcll(tmask[e]);
                t_cnt[e] = c;
                t_off[e] = coff;
                if (writer && d.tap_counts) d.tap_counts[e] = c;
                if (writer && d.tap_offsets) d.tap_offsets[e] = coff;
                coff += c;
                if (c) t_act[aoff++] = e;
            }
        }
        if (lane == 31) {
            t_off[E] = cs;
            t_misc[0] = as;
            if (writer && d.tap_offsets) d.tap_offsets[E] = cs;
        }
    }
    __syncthreads();
    for (int q = threadIdx.x; q < S; q += blockDim.x) {
        const int e = t_idx[q];
        if (e < 0 || e >= E) continue;
        const int t = q / K;
        const int p = t_off[e] + __popcll(tmask[e] & ((1ull << t) - 1ull));
        t_perm[p] = q;
        t_inv[q] = p;
        if (writer && d.tap_perm) d.tap_perm[p] = q;
    }
    __syncthreads();
    a.active = t_act;
    a.n_active = t_misc;
    a.counts = t_cnt;
    a.offsets = t_off;
    a.perm = t_perm;
    a.inv = t_inv;
    a.topk_w = t_w;
    a.sx = t_sx;
    a.sumx = t_sumx;

    const int n_active = t_misc[0];
    const int pairs = a.F / 32, blocks = a.D / 128;
    // split each kind of item over the CTAs in equal shares of estimated cost
    int *t_pg = (int *)(tmask + E), *t_pd = t_pg + E + 1;
    if (warp == 0) {
        const int per = (n_active + 31) / 32, a0 = lane * per;
        int sg = 0, sd = 0;
        for (int i = 0; i < per; i++)
            if (a0 + i < n_active) {
                const int c = t_cnt[t_act[a0 + i]];
                sg += pairs * dec_item_cost(c, 0);
                sd += blocks * dec_item_cost(c, 1);
            }
        int cg = sg, cd = sd;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(FULL, cg, o), w = __shfl_up_sync(FULL, cd, o);
            if (lane >= o) {
                cg += v;
                cd += w;
            }
        }
        int og = cg - sg, od = cd - sd;
        for (int i = 0; i < per; i++)
            if (a0 + i < n_active) {
                const int c = t_cnt[t_act[a0 + i]];
                t_pg[a0 + i] = og;
                t_pd[a0 + i] = od;
                og += pairs * dec_item_cost(c, 0);
                od += blocks * dec_item_cost(c, 1);
            }
        if (lane == 31) {
            t_pg[n_active] = cg;
            t_pd[n_active] = cd;
        }
    }
    __syncthreads();
    const int64_t WG = t_pg[n_active], WD = t_pd[n_active];
    const int g0 = dec_item_at(t_pg, n_active, pairs, WG * blockIdx.x / gridDim.x);
    const int g1 = dec_item_at(t_pg, n_active, pairs, WG * (blockIdx.x + 1) / gridDim.x);
    const int d0 = dec_item_at(t_pd, n_active, blocks, WD * blockIdx.x / gridDim.x);
    const int d1 = dec_item_at(t_pd, n_active, blocks, WD * (blockIdx.x + 1) / gridDim.x);
    const int nG = g1 - g0, n_items = nG + (d1 - d0);
    const int Cg = a.D / 64, Cd = a.F / 64;
    // item i of this CTA -> kind (0 gate/up, 1 down), active index, sub-block
    auto item_of = [&](int i, int &kind, int &ai, int &sub) {
        if (i < nG) {
            kind = 0;
            ai = (g0 + i) / pairs;
            sub = (g0 + i) % pairs;
        } else {
            kind = 1;
            ai = (d0 + i - nG) / blocks;
            sub = (d0 + i - nG) % blocks;
        }
    };

    if (warp == 0) {
        // ---------------- codes and scales of every item, in order
        if (lane == 0) {
            int issued = 0;
            for (int i = 0; i < n_items; i++) {
                const int ws = i % nw;
                if (!dec_wait(b_wempty + 8 * ws, ((i / nw) & 1) ^ 1)) {
                    set_flag(a.flag_dev, MAPLE_DEVFLAG_TIMEOUT);
                    break;
                }
                issued = i + 1;
                int kind, ai, sub;
                item_of(i, kind, ai, sub);
                const int e = a.active[ai];
                DecWMeta *m = wmeta + ws;
                m->e = e;
                m->sub = sub;
                m->kind = kind;
                m->cnt = a.counts[e];
                m->base = a.offsets[e];
                uint8_t *dst = wring + (size_t)ws * d.wslot_bytes;
                const uint32_t bar = b_wfull + 8 * ws;
                if (kind == 0) {
                    const uint32_t cb = (uint32_t)(2 * Cg * 512);
                    dec_expect(bar, cb + 256);
                    dec_bulk(dst, a.w_gu + (size_t)e * gu_bytes_per_expert(a.D, a.F) + (size_t)(2 * sub) * Cg * 512, cb, bar);
                    dec_bulk(dst + cb, a.alpha_gate + (size_t)e * a.F + 32 * sub, 128, bar);
                    dec_bulk(dst + cb + 128, a.alpha_up + (size_t)e * a.F + 32 * sub, 128, bar);
                } else {
                    const uint32_t cb = (uint32_t)(4 * Cd * 512);
                    dec_expect(bar, cb + 512);
                    dec_bulk(dst, a.w_dn + (size_t)e * dn_bytes_per_expert(a.D, a.F) + (size_t)(4 * sub) * Cd * 512, cb, bar);
                    dec_bulk(dst + cb, a.alpha_down + (size_t)e * a.D + 128 * sub, 512, bar);
                }
            }
            // no copy may still be landing when the CTA exits
            for (int j = issued > nw ? issued - nw : 0; j < issued; j++)
                (void)dec_wait(b_wfull + 8 * (j % nw), (j / nw) & 1);
        }
        return;
    }

    if (warp <= kDecGroups) {
        // ---------------- activation staging for compute group g
        const int g = warp - 1;
        if (lane == 0) {
            int k = 0;
            bool ok = true;
            int staged = 0;   // units whose copies were issued
            for (int i = g; i < n_items && ok; i += kDecGroups) {
                int kind, ai, sub;
                item_of(i, kind, ai, sub);
                const int e = a.active[ai], cnt = a.counts[e], base = a.offsets[e];
                if (kind == 1) {
                    // every gate/up item of expert e must be done before its h rows are read
                    const uint64_t t0 = global_timer_ns();
                    unsigned v = 0;
                    while (true) {
                        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(d.arrive + e) : "memory");
                        if (v >= (unsigned)pairs) break;
                        __nanosleep(128);
                        if (global_timer_ns() - t0 > 2000000000ull) {
                            set_flag(a.flag_dev, MAPLE_DEVFLAG_TIMEOUT);
                            ok = false;
                            break;
                        }
                    }
                    if (!ok) break;
                    asm volatile("fence.proxy.async.global;" ::: "memory");
                }
                for (int b0 = 0; b0 < cnt; b0 += kGemvTokens, k++) {
                    const int buf = k & 1;
                    if (!dec_wait(b_aempty + 8 * (2 * g + buf), ((k >> 1) & 1) ^ 1)) {
                        set_flag(a.flag_dev, MAPLE_DEVFLAG_TIMEOUT);
                        ok = false;
                        break;
                    }
                    const int nb = min(kGemvTokens, cnt - b0);
                    DecActMeta *m = ameta + 2 * g + buf;
                    m->nb = nb;
                    m->b0 = b0;
                    m->base = base;
                    m->e = e;
                    uint8_t *dst = aring + (size_t)(2 * g + buf) * d.aslot_bytes;
                    const uint32_t bar = b_afull + 8 * (2 * g + buf);
                    if (kind == 0) {
                        for (int j = 0; j < nb; j++) {
                            const int slot = a.perm[base + b0 + j], t = slot / a.K;
                            m->slot[j] = slot;
                            m->s[j] = a.sx[t];
                            m->sum[j] = a.sumx[t];
                        }
                        const int nbp = dec_pad_tokens(nb);
                        dec_expect(bar, (uint32_t)(nbp * a.D));
                        for (int j = 0; j < nbp; j++)
                            dec_bulk(dst + (size_t)j * a.D,
                                     j < nb ? a.qx + (size_t)(m->slot[j] / a.K) * a.D : d.zrow, (uint32_t)a.D, bar);
                    } else {
                        for (int j = 0; j < nb; j++) m->slot[j] = a.perm[base + b0 + j];
                        dec_expect(bar, (uint32_t)(nb * a.F * 4));
                        dec_bulk(dst, a.h + (size_t)(base + b0) * a.F, (uint32_t)(nb * a.F * 4), bar);
                    }
                    staged = k + 1;
                }
            }
            for (int j = staged > 2 ? staged - 2 : 0; j < staged; j++)
                (void)dec_wait(b_afull + 8 * (2 * g + (j & 1)), (j >> 1) & 1);
        }
        return;
    }

    if (warp < kDecFirstCompute) {
        // ---------------- publishing warp of group g
        const int g = warp - 1 - kDecGroups;
        int r = 0;
        for (int i = g; i < n_items; i += kDecGroups) {
            int kind, ai, sub;
            item_of(i, kind, ai, sub);
            const int cnt = a.counts[a.active[ai]];
            bool ok = true;
            for (int b0 = 0; b0 < cnt; b0 += kGemvTokens, r++) {
                const int rs = r % kDecRec;
                if (!dec_wait(b_rfull + 8 * (kDecRec * g + rs), (r / kDecRec) & 1)) {
                    if (lane == 0) set_flag(a.flag_dev, MAPLE_DEVFLAG_TIMEOUT);
                    ok = false;
                    break;
                }
                const DecRecord rec = recs[kDecRec * g + rs];
                fence_gpu();   // the group's h / yE stores, seen through the barrier chain, before what follows
                if (rec.kind == 0) {
                    if (rec.last && lane == 0)
                        asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(d.arrive + rec.e) : "memory");
                } else {
                    unsigned prev = 0;
                    int t = 0;
                    if (lane < rec.nb) {
                        t = rec.slot[lane] / a.K;
                        prev = atomicAdd(a.comb_cnt + (size_t)t * blocks + rec.sub, 1u);
                    }
                    unsigned done = __ballot_sync(FULL, lane < rec.nb && prev == (unsigned)(a.K - 1));
                    if (done) fence_gpu();
                    while (done) {
                        const int j = __ffs(done) - 1;
                        done &= done - 1;
                        const int tt = __shfl_sync(FULL, t, j);
                        // channels rec.sub*128 + 4*lane .. +3 of token tt, in rank order
                        const int cc = rec.sub * 128 + 4 * lane;
                        float4 yv = make_float4(0.f, 0.f, 0.f, 0.f);
                        for (int kk = 0; kk < a.K; kk++) {
                            const int sl = tt * a.K + kk;
                            const float wk = a.topk_w[sl];
                            const float4 ev = __ldcg(reinterpret_cast<const float4 *>(a.ye + (size_t)a.inv[sl] * a.D + cc));
                            yv.x = __fmaf_rn(wk, ev.x, yv.x);
                            yv.y = __fmaf_rn(wk, ev.y, yv.y);
                            yv.z = __fmaf_rn(wk, ev.z, yv.z);
                            yv.w = __fmaf_rn(wk, ev.w, yv.w);
                        }
                        const size_t o = (size_t)tt * a.D + cc;
                        if (a.resid) {
                            const float4 rv = *reinterpret_cast<const float4 *>(a.resid + o);
                            yv.x = __fadd_rn(rv.x, yv.x);
                            yv.y = __fadd_rn(rv.y, yv.y);
                            yv.z = __fadd_rn(rv.z, yv.z);
                            yv.w = __fadd_rn(rv.w, yv.w);
                        }
                        *reinterpret_cast<float4 *>(a.y + o) = yv;
                        if (lane == j) a.comb_cnt[(size_t)tt * blocks + rec.sub] = 0;
                    }
                }
                __syncwarp();
                if (lane == 0) dec_arrive(b_rempty + 8 * (kDecRec * g + rs));
            }
            if (!ok) break;
        }
        return;
    }

    // ---------------- compute group g: eight warps
    const int g = (warp - kDecFirstCompute) / kDecGroupWarps, gw = (warp - kDecFirstCompute) % kDecGroupWarps;
    const int gtid = gw * 32 + lane;
    const int bar_id = 1 + g;
    auto gsync = [&] { asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "n"(kDecGroupThreads) : "memory"); };
    uint8_t *scr = gscr + (size_t)g * gscr_bytes;
    int *red = (int *)scr;                                            // [8 warps][kGemvTokens][32]
    int8_t *qh = (int8_t *)(red + kDecGroupWarps * kGemvTokens * 32);  // [kGemvTokens][F]
    float *shs = (float *)(qh + (size_t)kGemvTokens * a.F);          // [kGemvTokens]
    int *sumqh = (int *)(shs + kGemvTokens);                         // [kGemvTokens]

    int k = 0, r = 0;
    for (int i = g; i < n_items; i += kDecGroups) {
        const int ws = i % nw;
        if (!dec_wait(b_wfull + 8 * ws, (i / nw) & 1)) {
            if (gtid == 0) set_flag(a.flag_dev, MAPLE_DEVFLAG_TIMEOUT);
            break;
        }
        const DecWMeta wm = wmeta[ws];
        const uint8_t *wb = wring + (size_t)ws * d.wslot_bytes;
        const int cnt = wm.cnt, base = wm.base;
        bool ok = true;
        for (int b0 = 0; b0 < cnt; b0 += kGemvTokens, k++, r++) {
            const int buf = k & 1;
            if (!dec_wait(b_afull + 8 * (2 * g + buf), (k >> 1) & 1)) {
                if (gtid == 0) set_flag(a.flag_dev, MAPLE_DEVFLAG_TIMEOUT);
                ok = false;
                break;
            }
            const DecActMeta &am = ameta[2 * g + buf];
            const uint8_t *ab = aring + (size_t)(2 * g + buf) * d.aslot_bytes;
            const int nb = am.nb;
            const int nbp = dec_pad_tokens(nb);
            int *red_w = red + gw * kGemvTokens * 32 + lane;
            if (wm.kind == 0) {
                // ---- gate/up: warp gw = row group gw/4 (of the pair), K quarter gw%4
                const int rg = gw >> 2, kq = gw & 3, quarter = Cg / 4;
                const uint4 *wl = reinterpret_cast<const uint4 *>(wb + (size_t)rg * Cg * 512) + lane;
                dot_rows_any(nbp, wl, reinterpret_cast<const uint4 *>(ab), a.D / 16, kq * quarter, quarter, red_w);
                gsync();
                if (kq == 0) {
                    const bool is_up = lane >= 16;
                    const int rr = (2 * wm.sub + rg) * 16 + (lane & 15);
                    const float al = ((const float *)(wb + 2 * Cg * 512))[(is_up ? 32 : 0) + 16 * rg + (lane & 15)];
                    for (int j = 0; j < nb; j++) {
                        int sum = 0;
#pragma unroll
                        for (int q = 0; q < 4; q++) sum += red[((gw + q) * kGemvTokens + j) * 32 + lane];
                        const int av = sum - am.sum[j];
                        const float v = __fmul_rn((float)av, __fmul_rn(al, am.s[j]));
                        const float uu = __shfl_down_sync(FULL, v, 16);
                        if (!is_up) a.h[(size_t)(base + am.b0 + j) * a.F + rr] = swiglu(v, uu);
                        int *tap = is_up ? a.tap_acc_up : a.tap_acc_gate;
                        if (tap) tap[(size_t)am.slot[j] * a.F + rr] = av;
                    }
                }
            } else {
                // ---- down: requantise the batch's h rows (one slot per warp), then warp gw =
                //      channel group 4*blk + gw/2, K half gw%2
                const float *hr = (const float *)ab;
                for (int j = nb + gw; j < nbp; j += kDecGroupWarps)
                    for (int q = lane; q < a.F / 16; q += 32)
                        reinterpret_cast<uint4 *>(qh + (size_t)j * a.F)[q] = make_uint4(0u, 0u, 0u, 0u);
                for (int j = gw; j < nb; j += kDecGroupWarps) {
                    const float4 *h4 = reinterpret_cast<const float4 *>(hr + (size_t)j * a.F);
                    float amax = 0.0f;
                    for (int q = lane; q < a.F / 4; q += 32) {
                        const float4 v = h4[q];
                        amax = fmaxf(fmaxf(fmaxf(amax, fabsf(v.x)), fmaxf(fabsf(v.y), fabsf(v.z))), fabsf(v.w));
                    }
                    amax = warp_max(amax);
                    const float inv = amax > 0.0f ? __fdiv_rn(127.0f, amax) : 0.0f;
                    int sum = 0;
                    for (int q = lane; q < a.F / 4; q += 32) {
                        const float4 v = h4[q];
                        int q0 = 0, q1 = 0, q2 = 0, q3 = 0;
                        if (amax > 0.0f) {
                            q0 = quant_code(v.x, inv);
                            q1 = quant_code(v.y, inv);
                            q2 = quant_code(v.z, inv);
                            q3 = quant_code(v.w, inv);
                        }
                        sum += q0 + q1 + q2 + q3;
                        const uint32_t pk = (uint32_t)(q0 & 0xff) | ((uint32_t)(q1 & 0xff) << 8) |
                                            ((uint32_t)(q2 & 0xff) << 16) | ((uint32_t)(q3 & 0xff) << 24);
                        reinterpret_cast<uint32_t *>(qh + (size_t)j * a.F)[q] = pk;
                        if (wm.sub == 0 && a.tap_qh) reinterpret_cast<uint32_t *>(a.tap_qh + (size_t)am.slot[j] * a.F)[q] = pk;
                    }
                    sum = warp_sum_int(sum);
                    if (lane == 0) {
                        const float sv = amax > 0.0f ? __fdiv_rn(amax, 127.0f) : 0.0f;
                        shs[j] = sv;
                        sumqh[j] = sum;
                        if (wm.sub == 0 && a.tap_sh) a.tap_sh[am.slot[j]] = sv;
                    }
                }
                gsync();
                const int cgl = gw >> 1, kh = gw & 1, half = Cd / 2;
                const uint4 *wl = reinterpret_cast<const uint4 *>(wb + (size_t)cgl * Cd * 512) + lane;
                dot_rows_any(nbp, wl, reinterpret_cast<const uint4 *>(qh), a.F / 16, kh * half, half, red_w);
                gsync();
                if (kh == 0) {
                    const int cg = (wm.sub * 4 + cgl) * 32 + lane;
                    const float al = ((const float *)(wb + 4 * Cd * 512))[cgl * 32 + lane];
                    for (int j = 0; j < nb; j++) {
                        const int p = base + am.b0 + j;
                        const int av = red[(gw * kGemvTokens + j) * 32 + lane] +
                                       red[((gw + 1) * kGemvTokens + j) * 32 + lane] - sumqh[j];
                        a.ye[(size_t)p * a.D + cg] = __fmul_rn((float)av, __fmul_rn(al, shs[j]));
                        if (a.tap_acc_down) a.tap_acc_down[(size_t)am.slot[j] * a.D + cg] = av;
                    }
                }
            }
            gsync();
            if (gtid == 0) {
                // hand the batch to the publishing warp, free the activation slot
                const int rs = r % kDecRec;
                if (!dec_wait(b_rempty + 8 * (kDecRec * g + rs), ((r / kDecRec) & 1) ^ 1))
                    set_flag(a.flag_dev, MAPLE_DEVFLAG_TIMEOUT);
                DecRecord *rec = recs + kDecRec * g + rs;
                rec->kind = wm.kind;
                rec->e = wm.e;
                rec->sub = wm.sub;
                rec->nb = nb;
                rec->base = base;
                rec->last = b0 + kGemvTokens >= cnt;
                for (int j = 0; j < nb; j++) rec->slot[j] = am.slot[j];
                dec_arrive(b_rfull + 8 * (kDecRec * g + rs));
                dec_arrive(b_aempty + 8 * (2 * g + buf));
            }
        }
        if (!ok) break;
        gsync();
        if (gtid == 0) dec_arrive(b_wempty + 8 * ws);
    }
}

}  // namespace maple
