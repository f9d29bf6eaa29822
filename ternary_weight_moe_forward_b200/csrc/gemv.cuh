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
// Grid = one CTA per SM, launched cooperatively (all CTAs resident).  Work
// items: gate/up items (active expert, 32 gate + 32 up rows = two row groups)
// then down items (active expert, 128 output channels).  Every CTA takes an
// equal contiguous range of the gate/up items and of the down items.  One
// producer thread streams the 2-bit codes of its items with bulk copies into
// a ring of shared-memory buffers (the copies do not depend on any result, so
// they run ahead into the down items while gate/up is computed); eight
// compute warps consume them.  The last CTA to finish an expert's gate/up
// items requantises that expert's slots and publishes ready[e] = epoch; a
// down item waits (bounded) for that before reading q_h.
// ---------------------------------------------------------------------------
constexpr int kDecThreads = (kGemvWarps + 1) * 32;   // + one producer warp
constexpr int kDecRingBytes = 160 * 1024;

struct DecodeArgs {
    GemvArgs g;
    unsigned *ready;     // [E]: epoch of the last requantisation
    unsigned epoch;
    int nbuf;            // ring buffers
    int buf_bytes;       // bytes per ring buffer
};

__host__ __device__ inline size_t decode_smem_bytes(int D, int F, int buf_bytes, int nbuf)
{
    const int row = D > F ? D : F;
    return (size_t)nbuf * buf_bytes + (size_t)kGemvTokens * row + (size_t)kGemvWarps * kGemvTokens * 32 * 4 +
           (size_t)2 * 8 * nbuf + 1024;
}

// bounded wait on an mbarrier phase (2 s); false on timeout
__device__ __forceinline__ bool dec_wait(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    const uint64_t t0 = global_timer_ns();
    while (true) {
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(bar), "r"(parity)
            : "memory");
        if (ok) return true;
        if (global_timer_ns() - t0 > 2000000000ull) return false;
    }
}

__global__ void __launch_bounds__(kDecThreads, 1) decode_experts_kernel(DecodeArgs d)
{
    const GemvArgs &a = d.g;
    extern __shared__ __align__(1024) uint8_t dsm[];
    uint8_t *ring = dsm;
    const int rowmax = a.D > a.F ? a.D : a.F;
    int8_t *xs = (int8_t *)(dsm + (size_t)d.nbuf * d.buf_bytes);
    int *red = (int *)(xs + (size_t)kGemvTokens * rowmax);
    uint64_t *bars = (uint64_t *)(red + kGemvWarps * kGemvTokens * 32);   // full[nbuf], empty[nbuf]
    __shared__ int s_slot[kGemvTokens];
    __shared__ int s_done[kGemvTokens];
    __shared__ unsigned s_flag;

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t b_full = (uint32_t)__cvta_generic_to_shared(bars), b_empty = b_full + 8 * d.nbuf;
    if (threadIdx.x == 0) {
        for (int i = 0; i < d.nbuf; i++) {
            asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(b_full + 8 * i), "r"(1) : "memory");
            asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(b_empty + 8 * i), "r"(1) : "memory");
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    const int n_active = __ldg(a.n_active);
    const int pairs = a.F / 32, blocks = a.D / 128;
    const int n_g = n_active * pairs, n_d = n_active * blocks;
    const int g0 = (int)((int64_t)n_g * blockIdx.x / gridDim.x), g1 = (int)((int64_t)n_g * (blockIdx.x + 1) / gridDim.x);
    const int d0 = (int)((int64_t)n_d * blockIdx.x / gridDim.x), d1 = (int)((int64_t)n_d * (blockIdx.x + 1) / gridDim.x);
    const int n_mine = (g1 - g0) + (d1 - d0);
    const int Cg = a.D / 64, Cd = a.F / 64;
    const uint32_t g_bytes = (uint32_t)(2 * Cg * 512), d_bytes = (uint32_t)(4 * Cd * 512);

    if (warp == kGemvWarps) {
        // ---------------- producer: bulk copies of the codes, in item order
        if (lane == 0) {
            for (int i = 0; i < n_mine; i++) {
                const int buf = i % d.nbuf;
                if (!dec_wait(b_empty + 8 * buf, ((i / d.nbuf) & 1) ^ 1)) {
                    set_flag(a.flag_dev, MAPLE_DEVFLAG_TIMEOUT);
                    break;
                }
                const uint8_t *src;
                uint32_t bytes;
                if (i < g1 - g0) {
                    const int it = g0 + i, e = a.active[it / pairs], pr = it % pairs;
                    src = a.w_gu + (size_t)e * gu_bytes_per_expert(a.D, a.F) + (size_t)(2 * pr) * Cg * 512;
                    bytes = g_bytes;
                } else {
                    const int it = d0 + (i - (g1 - g0)), e = a.active[it / blocks], blk = it % blocks;
                    src = a.w_dn + (size_t)e * dn_bytes_per_expert(a.D, a.F) + (size_t)(4 * blk) * Cd * 512;
                    bytes = d_bytes;
                }
                const uint32_t dst = (uint32_t)__cvta_generic_to_shared(ring + (size_t)buf * d.buf_bytes);
                asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(b_full + 8 * buf),
                             "r"(bytes)
                             : "memory");
                for (uint32_t off = 0; off < bytes; off += 8192) {
                    const uint32_t n = bytes - off < 8192 ? bytes - off : 8192;
                    asm volatile(
                        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                            dst + off),
                        "l"(src + off), "r"(n), "r"(b_full + 8 * buf)
                        : "memory");
                }
            }
        }
        return;   // the producer warp takes no part in the compute barriers below
    }

    // ---------------- compute warps (named barrier 1, kGemvWarps*32 threads)
    auto csync = [] { asm volatile("bar.sync 1, %0;" ::"n"(kGemvWarps * 32) : "memory"); };
    bool ok = true;
    int staged_e = -1, staged_b0 = -1, staged_kind = -1;
    for (int i = 0; i < n_mine && ok; i++) {
        const int buf = i % d.nbuf;
        const bool is_down = i >= g1 - g0;
        const int it = is_down ? d0 + (i - (g1 - g0)) : g0 + i;
        const int ai = is_down ? it / blocks : it / pairs;
        const int e = a.active[ai];
        const int cnt = a.counts[e], base = a.offsets[e];
        if (is_down && staged_kind != 1 + e) {
            // wait until expert e's q_h is published
            if (threadIdx.x == 0) {
                const uint64_t t0 = global_timer_ns();
                unsigned v;
                s_flag = 1;
                while (true) {
                    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(d.ready + e) : "memory");
                    if (v == d.epoch) break;
                    if (global_timer_ns() - t0 > 2000000000ull) {
                        set_flag(a.flag_dev, MAPLE_DEVFLAG_TIMEOUT);
                        s_flag = 0;
                        break;
                    }
                }
            }
            csync();
            if (!s_flag) break;
        }
        if (!dec_wait(b_full + 8 * buf, (i / d.nbuf) & 1)) {
            if (threadIdx.x == 0) set_flag(a.flag_dev, MAPLE_DEVFLAG_TIMEOUT);
            break;
        }
        const uint8_t *wb = ring + (size_t)buf * d.buf_bytes;
        if (!is_down) {
            const int pr = it % pairs;
            const int gl = warp >> 2, kq = warp & 3, NI = Cg / 4;
            for (int b0 = 0; b0 < cnt; b0 += kGemvTokens) {
                const int nb = min(kGemvTokens, cnt - b0);
                if (!(staged_kind == 0 && staged_e == e && staged_b0 == b0)) {
                    if (threadIdx.x < nb) s_slot[threadIdx.x] = a.perm[base + b0 + threadIdx.x];
                    csync();
                    const int row16 = a.D / 16;
                    for (int q = threadIdx.x; q < nb * row16; q += kGemvWarps * 32) {
                        const int j = q / row16, c16 = q - j * row16;
                        reinterpret_cast<uint4 *>(xs + (size_t)j * a.D)[c16] =
                            __ldg(reinterpret_cast<const uint4 *>(a.qx + (size_t)(s_slot[j] / a.K) * a.D) + c16);
                    }
                    staged_kind = 0;
                    staged_e = e;
                    staged_b0 = b0;
                }
                csync();
                int acc[kGemvTokens];
#pragma unroll
                for (int j = 0; j < kGemvTokens; j++) acc[j] = 0;
                const uint8_t *wl = wb + (size_t)gl * Cg * 512 + lane * 16;
                for (int u = 0; u < NI; u++) {
                    const int c = kq * NI + u;
                    chunk_tokens(*reinterpret_cast<const uint4 *>(wl + (size_t)c * 512), xs, a.D, 64 * c, nb, acc);
                }
#pragma unroll
                for (int j = 0; j < kGemvTokens; j++) red[(warp * kGemvTokens + j) * 32 + lane] = acc[j];
                csync();
                if (warp < 2) {
                    const int rr = (2 * pr + warp) * 16 + (lane & 15);
                    const bool is_up = lane >= 16;
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
                csync();
            }
            if (threadIdx.x == 0)
                asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(b_empty + 8 * buf) : "memory");
            // the last item of expert e to finish requantises e's slots and publishes them
            if (warp < 2) fence_gpu();
            csync();
            if (threadIdx.x == 0) s_flag = atomicAdd(a.exp_cnt + e, 1u) == (unsigned)(pairs - 1);
            csync();
            if (s_flag) {
                fence_gpu();
                if (threadIdx.x == 0) a.exp_cnt[e] = 0;
                requant_slots_warps(a, base, cnt, kGemvWarps);
                fence_gpu();
                csync();
                if (threadIdx.x == 0) asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(d.ready + e), "r"(d.epoch) : "memory");
            }
        } else {
            const int blk = it % blocks;
            const int gl = warp >> 1, kh = warp & 1, NH = Cd / 2;
            for (int b0 = 0; b0 < cnt; b0 += kGemvTokens) {
                const int nb = min(kGemvTokens, cnt - b0);
                if (!(staged_kind == 1 + e && staged_b0 == b0)) {
                    if (threadIdx.x < nb) s_slot[threadIdx.x] = a.perm[base + b0 + threadIdx.x];
                    const int n16 = nb * a.F / 16;
                    for (int q = threadIdx.x; q < n16; q += kGemvWarps * 32)
                        reinterpret_cast<uint4 *>(xs)[q] =
                            __ldcg(reinterpret_cast<const uint4 *>(a.qh + (size_t)(base + b0) * a.F) + q);
                    staged_kind = 1 + e;
                    staged_b0 = b0;
                }
                csync();
                int acc[kGemvTokens];
#pragma unroll
                for (int j = 0; j < kGemvTokens; j++) acc[j] = 0;
                const uint8_t *wl = wb + (size_t)gl * Cd * 512 + lane * 16;
                for (int u = 0; u < NH; u++) {
                    const int c = kh * NH + u;
                    chunk_tokens(*reinterpret_cast<const uint4 *>(wl + (size_t)c * 512), xs, a.F, 64 * c, nb, acc);
                }
#pragma unroll
                for (int j = 0; j < kGemvTokens; j++) red[(warp * kGemvTokens + j) * 32 + lane] = acc[j];
                csync();
                if (warp < 4) {
                    const int cg = (blk * 4 + warp) * 32 + lane;
                    const float al = a.alpha_down[(size_t)e * a.D + cg];
                    for (int j = 0; j < nb; j++) {
                        const int p = base + b0 + j;
                        const int sum = red[((2 * warp) * kGemvTokens + j) * 32 + lane] +
                                        red[((2 * warp + 1) * kGemvTokens + j) * 32 + lane];
                        const int av = sum - __ldcg(a.sumqh + p);
                        a.ye[(size_t)p * a.D + cg] = __fmul_rn((float)av, __fmul_rn(al, __ldcg(a.sh + p)));
                        if (a.tap_acc_down) a.tap_acc_down[(size_t)s_slot[j] * a.D + cg] = av;
                    }
                    fence_gpu();
                }
                csync();
                if (threadIdx.x < nb) {
                    const int t = s_slot[threadIdx.x] / a.K;
                    const unsigned prev = atomicAdd(a.comb_cnt + (size_t)t * blocks + blk, 1u);
                    s_done[threadIdx.x] = prev == (unsigned)(a.K - 1);
                }
                csync();
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
                csync();
            }
            if (threadIdx.x == 0)
                asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(b_empty + 8 * buf) : "memory");
        }
    }
    (void)ok;
}

}  // namespace maple
