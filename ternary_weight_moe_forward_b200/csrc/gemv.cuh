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
// Persistent expert-stage kernel for decode batches (T <= 64).
//
// Grid = one CTA per SM (a plain launch: no CTA waits on work of a CTA that
// has not started, so residency of the whole grid is not needed).  Every
// CTA first builds the permutation of all T*K slots for itself from the
// router's top-k (in shared memory), so no routing step needs a grid-wide
// hand-off.  Work items: gate/up items (active expert, 8 groups of 16 gate +
// 16 up rows) then down items (active expert, 8 groups of 32 output
// channels).  Items are handed out dynamically: compute group 0 or 1 of
// any CTA claims the next one from a global counter (gate/up items first, so
// no down item can wait on an unclaimed gate/up item), which balances the
// load whatever the tokens per expert; a small queue in shared memory passes a
// group's claims to its warps.
// Warp roles:
//   warps 0, 1  stage the activations of compute group 0 / 1 (double
//               buffered): for gate/up the int8 rows of the item's tokens; for
//               down, once every gate/up item of the expert has finished, the
//               fp32 SwiGLU rows h of the item's slots, which the warp then
//               requantises (per-slot absmax int8) into the buffer;
//   warps 2, 3  publish the results of group 0 / 1: make a finished gate/up
//               item visible (GPU fence, arrival counter of its expert), and for
//               a down item count each token's arrival on its 256-channel block,
//               the last of the K arrivals combining that token's channels;
//   warps 4..19 two compute groups of eight warps; group g takes items g, g+2,
//               ... of the CTA.  Warp w of a group owns row group w of the
//               item over all of K: it streams its own 2-bit codes (512
//               contiguous bytes per 64 columns, one 16-byte cp.async per lane,
//               kDecStages chunks in flight) and runs them against the staged
//               activations, then its own epilogue.  The last warp of a batch
//               to finish hands it on and frees the activation buffer; no
//               barrier spans the group.
// Every wait is bounded (2 s) and raises the device flag on expiry.
// ---------------------------------------------------------------------------
constexpr int kDecGroups = 2;
constexpr int kDecGroupWarps = 8;
constexpr int kDecRec = 4;   // completion records per group
constexpr int kDecFirstCompute = 2 * kDecGroups;
constexpr int kDecThreads = (kDecFirstCompute + kDecGroups * kDecGroupWarps) * 32;   // 640
constexpr int kDecStages = 12;   // 512-byte weight chunks in flight per compute warp

struct DecActMeta {
    int nb, b0, base, e;
    int slot[kGemvTokens];
    float s[kGemvTokens];     // gate/up: s_x of the token; down: s_h of the slot
    int sum[kGemvTokens];     // sum of the row's int8 codes (q_x or q_h)
    unsigned done;            // warps finished with the batch
};
constexpr int kDecQueue = 16;   // claimed items a group's queue holds
struct DecQueue {               // the items a compute group has claimed, in order
    int item[kDecQueue];        // global item id (>= total: no more work)
    int n;                      // items claimed so far
};
struct DecRecord {            // one finished batch of a compute group
    int kind, e, sub, nb, base, last;
    int slot[kGemvTokens];
};

struct DecodeArgs {
    GemvArgs g;
    unsigned *arrive;     // [E] finished gate/up items per expert, zero at launch
    int aslot_bytes;      // one activation buffer
    const int8_t *zrow;   // D zero bytes (padding rows of a gate/up batch)
    int *item_ctr;        // work items claimed so far, zero at launch
    const int *topk_idx;  // [T][K] the router's choices (distinct per token)
    const float *topk_w;  // [T][K] their softmax weights
    // outputs of the permutation, written by CTA 0 (may be null)
    int *tap_counts, *tap_offsets, *tap_perm;
};

// activation buffer: [x rows int8 | h rows fp32] [q_h rows int8]
__host__ __device__ inline int dec_qh_off(int D, int F)
{
    const int g = kGemvTokens * D, d = kGemvTokens * F * 4;
    return ((g > d ? g : d) + 127) & ~127;
}
__host__ __device__ inline int dec_aslot_bytes(int D, int F) { return dec_qh_off(D, F) + ((kGemvTokens * F + 127) & ~127); }
// routing tables every CTA builds for itself in shared memory
__host__ __device__ inline size_t dec_table_bytes(int T, int K, int E)
{
    return (size_t)4 * T * K * 4 + (size_t)(3 * E + 1) * 4 + (size_t)2 * T * 4 + 48 * 4 + 8 + (size_t)8 * E;
}
constexpr int kDecBars = 6 * kDecGroups + 2 * kDecRec * kDecGroups;
constexpr int kDecRingBytes = kDecGroups * kDecGroupWarps * kDecStages * 512;
__host__ __device__ inline size_t decode_smem_bytes(int D, int F, int T, int K, int E)
{
    return (size_t)kDecRingBytes + (size_t)kDecGroups * 2 * dec_aslot_bytes(D, F) + kDecGroups * 2 * sizeof(DecActMeta) +
           kDecGroups * sizeof(DecQueue) + kDecGroups * kDecRec * sizeof(DecRecord) + 8 * kDecBars + 64 +
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

// Padded token count of a decode batch: the dot below exists for 1, 2, 4 and 8
// tokens; rows nb..nbp-1 of a batch hold zeros.
__device__ __forceinline__ int dec_pad_tokens(int nb) { return nb <= 1 ? 1 : nb <= 2 ? 2 : nb <= 4 ? 4 : 8; }

// The weight stream of one compute warp: for every batch of every item the
// warp takes (items g, g+2, ... of the CTA; a batch is up to 8 tokens of the
// item's expert), the nch chunks of its row group, 512 contiguous bytes per 64
// columns, this lane's 16 bytes of each copied with one cp.async into a ring of
// kDecStages chunks.  The issue cursor runs kDecStages-1 chunks ahead of the
// chunk in use, across batch and item boundaries, so the pipeline never drains
// between items.  Each lane reads back only the bytes it copied itself, so no
// barrier is needed.
struct DecStream {
    uint8_t *ring;          // this lane's 16 bytes of stage 0
    const uint8_t *src;     // this lane's 16 bytes of chunk 0 of the current segment
    int nch, c, left;       // chunks in the segment, next chunk, batches left in the item
    int item, st;           // queue ordinal of the issue cursor's item, ring stage to fill next

    __device__ __forceinline__ void issue()
    {
        if (left > 0) cp_async16(ring + st * 512, src + (size_t)c * 512, true);
        cp_async_commit();
        st = st == kDecStages - 1 ? 0 : st + 1;
    }
};

// This lane's row against NB token rows over the nch chunks of the current
// batch; for every chunk used one more is issued (advance() moves the issue
// cursor).  Byte plane k is taken as w & (0x03030303 << 2k), i.e. 4^k times the
// offset codes, one logic op per plane, into its own accumulator; acc_k is an
// exact multiple of 4^k and the row total is acc_0 + acc_1/4 + acc_2/16 +
// acc_3/64 (int32, exact).  Activations: 16-byte units x[j*ld16 + 4c + w], read
// as broadcasts.
template <int NB, class Adv>
__device__ __forceinline__ void dec_stream_dot(DecStream &ws, int &cst, int nch, const uint4 *x, int ld16, Adv &advance,
                                               int (&tot)[kGemvTokens])
{
    int acc[NB][4];
#pragma unroll
    for (int j = 0; j < NB; j++)
#pragma unroll
        for (int k = 0; k < 4; k++) acc[j][k] = 0;
#pragma unroll 1
    for (int c = 0; c < nch; c++) {
        cp_async_wait<kDecStages - 2>();
        const uint4 wv = *reinterpret_cast<const uint4 *>(ws.ring + cst * 512);
        cst = cst == kDecStages - 1 ? 0 : cst + 1;
        ws.issue();
        advance();
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
                const uint4 xv = x[j * ld16 + 4 * c + w];
                acc[j][0] = dp4a_us(pw[4 * w + 0], xv.x, acc[j][0]);
                acc[j][1] = dp4a_us(pw[4 * w + 1], xv.y, acc[j][1]);
                acc[j][2] = dp4a_us(pw[4 * w + 2], xv.z, acc[j][2]);
                acc[j][3] = dp4a_us(pw[4 * w + 3], xv.w, acc[j][3]);
            }
        }
    }
#pragma unroll
    for (int j = 0; j < kGemvTokens; j++)
        tot[j] = j < NB ? acc[j < NB ? j : 0][0] + (acc[j < NB ? j : 0][1] >> 2) + (acc[j < NB ? j : 0][2] >> 4) +
                              (acc[j < NB ? j : 0][3] >> 6)
                        : 0;
}

// Eight tokens: byte planes by shift and mask (two ops for k > 0) into a single
// accumulator per token, which keeps the eight accumulators in registers.
template <class Adv>
__device__ __forceinline__ void dec_stream_dot8(DecStream &ws, int &cst, int nch, const uint4 *x, int ld16, Adv &advance,
                                                int (&tot)[kGemvTokens])
{
#pragma unroll
    for (int j = 0; j < kGemvTokens; j++) tot[j] = 0;
#pragma unroll 1
    for (int c = 0; c < nch; c++) {
        cp_async_wait<kDecStages - 2>();
        const uint4 wv = *reinterpret_cast<const uint4 *>(ws.ring + cst * 512);
        cst = cst == kDecStages - 1 ? 0 : cst + 1;
        ws.issue();
        advance();
        const uint32_t w4[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
        for (int w = 0; w < 4; w++) {
            uint32_t pw[4];
#pragma unroll
            for (int k = 0; k < 4; k++) pw[k] = plane(w4[w], k);
#pragma unroll
            for (int j = 0; j < kGemvTokens; j++) {
                const uint4 xv = x[j * ld16 + 4 * c + w];
                tot[j] = dp4a_us(pw[0], xv.x, tot[j]);
                tot[j] = dp4a_us(pw[1], xv.y, tot[j]);
                tot[j] = dp4a_us(pw[2], xv.z, tot[j]);
                tot[j] = dp4a_us(pw[3], xv.w, tot[j]);
            }
        }
    }
}

template <class Adv>
__device__ __forceinline__ void dec_stream_dot_any(int nbp, DecStream &ws, int &cst, int nch, const uint4 *x, int ld16,
                                                   Adv &advance, int (&tot)[kGemvTokens])
{
    switch (nbp) {
    case 1: dec_stream_dot<1>(ws, cst, nch, x, ld16, advance, tot); break;
    case 2: dec_stream_dot<2>(ws, cst, nch, x, ld16, advance, tot); break;
    case 4: dec_stream_dot<4>(ws, cst, nch, x, ld16, advance, tot); break;
    default: dec_stream_dot8(ws, cst, nch, x, ld16, advance, tot); break;
    }
}

// Item m of a compute group's queue (all 32 lanes of a warp call it).  With
// claim, the warp takes the next global item (lane 0, atomically; n_tot once
// all are taken) and appends it; otherwise it waits (bounded, 2 s; n_tot and
// the device flag on expiry) until the claiming warp has appended item m.
// Out of line: it runs once per item, and keeps the dot loop's registers free.
__device__ __noinline__ int dec_queue_item(DecQueue *qp, int m, bool claim, int n_tot, int *ctr, unsigned *flag)
{
    volatile DecQueue *q = qp;
    const int lane = threadIdx.x & 31;
    if (claim) {
        int x = 0;
        if (lane == 0) {
            x = min(atomicAdd(ctr, 1), n_tot);
            q->item[m & (kDecQueue - 1)] = x;
            __threadfence_block();
            q->n = m + 1;
        }
        return __shfl_sync(FULL, x, 0);
    }
    if (q->n <= m) {
        const uint64_t t0 = global_timer_ns();
        while (q->n <= m) {
            __nanosleep(64);
            if (global_timer_ns() - t0 > 2000000000ull) {
                if (lane == 0) set_flag(flag, MAPLE_DEVFLAG_TIMEOUT);
                return n_tot;
            }
        }
    }
    __threadfence_block();
    return q->item[m & (kDecQueue - 1)];
}

__global__ void __launch_bounds__(kDecThreads, 1) decode_experts_kernel(DecodeArgs d)
{
    GemvArgs a = d.g;
    extern __shared__ __align__(1024) uint8_t dsm[];
    uint8_t *wring = dsm;                                                         // [group][warp][stage][512]
    uint8_t *aring = wring + kDecRingBytes;                                       // [group][2][aslot]
    DecActMeta *ameta = (DecActMeta *)(aring + (size_t)kDecGroups * 2 * d.aslot_bytes);   // [group][2]
    DecQueue *queue = (DecQueue *)(ameta + kDecGroups * 2);                       // [group]
    DecRecord *recs = (DecRecord *)(queue + kDecGroups);                          // [group][kDecRec]
    uint64_t *bars = (uint64_t *)(((uintptr_t)(recs + kDecGroups * kDecRec) + 7) & ~(uintptr_t)7);
    // bars: afull[G][2], aempty[G][2], hfull[G][2], rfull[G][R], rempty[G][R]
    const uint32_t b_afull = (uint32_t)__cvta_generic_to_shared(bars), b_aempty = b_afull + 8 * 2 * kDecGroups;
    const uint32_t b_hfull = b_aempty + 8 * 2 * kDecGroups, b_rfull = b_hfull + 8 * 2 * kDecGroups;
    const uint32_t b_rempty = b_rfull + 8 * kDecRec * kDecGroups;
    const int qh_off = dec_qh_off(a.D, a.F);
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
    int *t_misc = t_sumx + T;   // [0] n_active
    unsigned long long *tmask = (unsigned long long *)(((uintptr_t)(t_misc + 48) + 7) & ~(uintptr_t)7);

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (threadIdx.x == 0) {
        for (int i = 0; i < kDecBars; i++)
            asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(b_afull + 8 * i), "r"(1) : "memory");
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (threadIdx.x < kDecGroups * 2) ameta[threadIdx.x].done = 0u;
    if (threadIdx.x < kDecGroups) queue[threadIdx.x].n = 0;
    // The kernel may be launched while the routing kernel still runs (programmatic
    // dependent launch): nothing it writes is read before this point.
    asm volatile("griddepcontrol.wait;" ::: "memory");

    // ---------------- prologue: the permutation of the T*K slots (T <= 64), from the
    // router's choices: a token bitmask per expert gives the counts, and a slot's
    // rank within its expert is the number of earlier tokens in that mask
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
    const int Cg = a.D / 64, Cd = a.F / 64;
    const int gitems = a.F / 128, ditems = a.D / 256;   // items per expert (8 row groups each)
    __syncthreads();
    const int n_g = n_active * gitems, n_tot = n_g + n_active * ditems;
    // global item id x -> kind (0 gate/up, 1 down), active index, sub-item
    auto item_of = [&](int x, int &kind, int &ai, int &sub) {
        if (x < n_g) {
            kind = 0;
            ai = x / gitems;
            sub = x % gitems;
        } else {
            kind = 1;
            ai = (x - n_g) / ditems;
            sub = (x - n_g) % ditems;
        }
    };
    auto q_get = [&](int g, int m) -> int {
        return dec_queue_item(queue + g, m, false, n_tot, d.item_ctr, a.flag_dev);
    };

    if (warp < kDecGroups) {
        // ---------------- activation staging for compute group g (whole warp)
        const int g = warp;
        int k = 0, kh0 = 0, kh1 = 0;   // batches staged; down batches staged per buffer
        bool ok = true;
        for (int m = 0; ok; m++) {
            const int x = q_get(g, m);
            if (x >= n_tot) break;
            int kind, ai, sub;
            item_of(x, kind, ai, sub);
            const int e = a.active[ai], cnt = a.counts[e], base = a.offsets[e];
            if (kind == 1) {
                // every gate/up item of expert e must be done before its h rows are read
                if (lane == 0) {
                    const uint64_t t0 = global_timer_ns();
                    unsigned v = 0;
                    while (true) {
                        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(d.arrive + e) : "memory");
                        if (v >= (unsigned)gitems) break;
                        __nanosleep(128);
                        if (global_timer_ns() - t0 > 2000000000ull) {
                            set_flag(a.flag_dev, MAPLE_DEVFLAG_TIMEOUT);
                            ok = false;
                            break;
                        }
                    }
                    asm volatile("fence.proxy.async.global;" ::: "memory");
                }
                ok = __shfl_sync(FULL, ok, 0);
                if (!ok) break;
            }
            for (int b0 = 0; b0 < cnt; b0 += kGemvTokens, k++) {
                const int buf = k & 1;
                if (!dec_wait(b_aempty + 8 * (2 * g + buf), ((k >> 1) & 1) ^ 1)) {
                    if (lane == 0) set_flag(a.flag_dev, MAPLE_DEVFLAG_TIMEOUT);
                    ok = false;
                    break;
                }
                const int nb = min(kGemvTokens, cnt - b0), nbp = dec_pad_tokens(nb);
                DecActMeta *m = ameta + 2 * g + buf;
                uint8_t *dst = aring + (size_t)(2 * g + buf) * d.aslot_bytes;
                if (lane < nb) {
                    const int slot = a.perm[base + b0 + lane];
                    m->slot[lane] = slot;
                    if (kind == 0) {
                        m->s[lane] = a.sx[slot / a.K];
                        m->sum[lane] = a.sumx[slot / a.K];
                    }
                }
                if (lane == 0) {
                    m->nb = nb;
                    m->b0 = b0;
                    m->base = base;
                    m->e = e;
                }
                __syncwarp();
                if (kind == 0) {
                    if (lane == 0) {
                        const uint32_t bar = b_afull + 8 * (2 * g + buf);
                        dec_expect(bar, (uint32_t)(nbp * a.D));
                        for (int j = 0; j < nbp; j++)
                            dec_bulk(dst + (size_t)j * a.D,
                                     j < nb ? a.qx + (size_t)(m->slot[j] / a.K) * a.D : d.zrow, (uint32_t)a.D, bar);
                    }
                    continue;
                }
                // down: bring the h rows in, requantise them per slot into the buffer
                const uint32_t hb = b_hfull + 8 * (2 * g + buf);
                if (lane == 0) {
                    dec_expect(hb, (uint32_t)(nb * a.F * 4));
                    dec_bulk(dst, a.h + (size_t)(base + b0) * a.F, (uint32_t)(nb * a.F * 4), hb);
                }
                const int kh = buf ? kh1++ : kh0++;
                if (!dec_wait(hb, kh & 1)) {
                    if (lane == 0) set_flag(a.flag_dev, MAPLE_DEVFLAG_TIMEOUT);
                    ok = false;
                    break;
                }
                int8_t *qh = (int8_t *)(dst + qh_off);
                for (int j = 0; j < nb; j++) {
                    const float4 *h4 = reinterpret_cast<const float4 *>(dst + (size_t)j * a.F * 4);
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
                        if (sub == 0 && a.tap_qh)
                            reinterpret_cast<uint32_t *>(a.tap_qh + (size_t)m->slot[j] * a.F)[q] = pk;
                    }
                    sum = warp_sum_int(sum);
                    if (lane == 0) {
                        const float sv = amax > 0.0f ? __fdiv_rn(amax, 127.0f) : 0.0f;
                        m->s[j] = sv;
                        m->sum[j] = sum;
                        if (sub == 0 && a.tap_sh) a.tap_sh[m->slot[j]] = sv;
                    }
                }
                for (int j = nb; j < nbp; j++)
                    for (int q = lane; q < a.F / 16; q += 32)
                        reinterpret_cast<uint4 *>(qh + (size_t)j * a.F)[q] = make_uint4(0u, 0u, 0u, 0u);
                __syncwarp();
                if (lane == 0) dec_arrive(b_afull + 8 * (2 * g + buf));
            }
        }
        // no copy may still be landing when the CTA exits
        for (int j = k > 2 ? k - 2 : 0; j < k; j++) (void)dec_wait(b_afull + 8 * (2 * g + (j & 1)), (j >> 1) & 1);
        return;
    }

    if (warp < kDecFirstCompute) {
        // ---------------- publishing warp of group g
        const int g = warp - kDecGroups;
        const int nblk = a.D / 256;
        int r = 0;
        for (int m = 0;; m++) {
            const int x = q_get(g, m);
            if (x >= n_tot) break;
            int kind, ai, sub;
            item_of(x, kind, ai, sub);
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
                        prev = atomicAdd(a.comb_cnt + (size_t)t * nblk + rec.sub, 1u);
                    }
                    unsigned done = __ballot_sync(FULL, lane < rec.nb && prev == (unsigned)(a.K - 1));
                    if (done) fence_gpu();
                    while (done) {
                        const int j = __ffs(done) - 1;
                        done &= done - 1;
                        const int tt = __shfl_sync(FULL, t, j);
                        // channels rec.sub*256 + 4*lane .. +3 and +128 of token tt, in rank order
#pragma unroll
                        for (int hlf = 0; hlf < 2; hlf++) {
                            const int cc = rec.sub * 256 + 128 * hlf + 4 * lane;
                            float4 yv = make_float4(0.f, 0.f, 0.f, 0.f);
                            for (int kk = 0; kk < a.K; kk++) {
                                const int sl = tt * a.K + kk;
                                const float wk = a.topk_w[sl];
                                const float4 ev =
                                    __ldcg(reinterpret_cast<const float4 *>(a.ye + (size_t)a.inv[sl] * a.D + cc));
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
                        }
                        if (lane == j) a.comb_cnt[(size_t)tt * nblk + rec.sub] = 0;
                    }
                }
                __syncwarp();
                if (lane == 0) dec_arrive(b_rempty + 8 * (kDecRec * g + rs));
            }
            if (!ok) break;
        }
        return;
    }

    // ---------------- compute warp gw of group g: row group gw of every item of the group
    const int g = (warp - kDecFirstCompute) / kDecGroupWarps, gw = (warp - kDecFirstCompute) % kDecGroupWarps;
    // the issue cursor: item ws.item, batches left ws.left, chunk ws.c of its row group
    DecStream ws;
    ws.ring = wring + (size_t)((g * kDecGroupWarps + gw) * kDecStages) * 512 + lane * 16;
    ws.st = 0;
    ws.c = 0;
    auto seg_of = [&](int x, const uint8_t *&src, int &nch, int &nbat) {
        int kind, ai, sub;
        item_of(x, kind, ai, sub);
        const int e = a.active[ai], grp = sub * kDecGroupWarps + gw;
        nch = kind == 0 ? Cg : Cd;
        nbat = (a.counts[e] + kGemvTokens - 1) / kGemvTokens;
        src = (kind == 0 ? a.w_gu + (size_t)e * gu_bytes_per_expert(a.D, a.F) + (size_t)grp * Cg * 512
                         : a.w_dn + (size_t)e * dn_bytes_per_expert(a.D, a.F) + (size_t)grp * Cd * 512) +
              lane * 16;
    };
    // warp 0 of the group claims the items as its issue cursor reaches them; the
    // other warps take them from the queue
    auto next_item = [&](int m) -> int {
        return dec_queue_item(queue + g, m, gw == 0, n_tot, d.item_ctr, a.flag_dev);
    };
    ws.item = 0;   // ordinal of the issue cursor's item in the group's queue
    ws.left = 0;
    {
        const int x = next_item(0);
        if (x < n_tot) seg_of(x, ws.src, ws.nch, ws.left);
    }
    auto advance = [&]() {
        if (ws.left <= 0) return;
        if (++ws.c < ws.nch) return;
        ws.c = 0;
        if (--ws.left > 0) return;   // next batch of the same item: the same chunks again
        const int x = next_item(++ws.item);
        if (x < n_tot) seg_of(x, ws.src, ws.nch, ws.left);
    };
    for (int s = 0; s < kDecStages - 1; s++) {
        ws.issue();
        advance();
    }
    int cst = 0;   // ring stage of the next chunk to use
    int k = 0;     // batches of this group (= completion record index)
    for (int m = 0;; m++) {
        const int x = q_get(g, m);   // already claimed: this warp's issue cursor is past it
        if (x >= n_tot) break;
        int kind, ai, sub;
        item_of(x, kind, ai, sub);
        const int e = a.active[ai], cnt = a.counts[e], base = a.offsets[e];
        const int grp = sub * kDecGroupWarps + gw;   // row group (32 rows) within the expert
        const int nch = kind == 0 ? Cg : Cd;
        // the row scale: gate/up lanes 0..15 gate rows grp*16+l, lanes 16..31 the up rows of
        // the same outputs; down lane l channel grp*32+l
        const float al = kind == 0 ? __ldg((lane < 16 ? a.alpha_gate : a.alpha_up) + (size_t)e * a.F + grp * 16 + (lane & 15))
                                   : __ldg(a.alpha_down + (size_t)e * a.D + grp * 32 + lane);
        for (int b0 = 0; b0 < cnt; b0 += kGemvTokens, k++) {
            const int buf = k & 1;
            if (!dec_wait(b_afull + 8 * (2 * g + buf), (k >> 1) & 1)) {
                if (lane == 0) set_flag(a.flag_dev, MAPLE_DEVFLAG_TIMEOUT);
                cp_async_wait<0>();
                return;
            }
            DecActMeta *am = ameta + 2 * g + buf;
            const uint8_t *ab = aring + (size_t)(2 * g + buf) * d.aslot_bytes;
            const int nb = am->nb;
            int tot[kGemvTokens];
            if (kind == 0)
                dec_stream_dot_any(dec_pad_tokens(nb), ws, cst, nch, reinterpret_cast<const uint4 *>(ab), a.D / 16,
                                   advance, tot);
            else
                dec_stream_dot_any(dec_pad_tokens(nb), ws, cst, nch, reinterpret_cast<const uint4 *>(ab + qh_off),
                                   a.F / 16, advance, tot);
            if (kind == 0) {
                const bool is_up = lane >= 16;
                const int rr = grp * 16 + (lane & 15);
                int *tap = is_up ? a.tap_acc_up : a.tap_acc_gate;
#pragma unroll
                for (int j = 0; j < kGemvTokens; j++) {
                    if (j < nb) {
                        const int av = tot[j] - am->sum[j];
                        const float v = __fmul_rn((float)av, __fmul_rn(al, am->s[j]));
                        const float uu = __shfl_down_sync(FULL, v, 16);
                        if (!is_up) a.h[(size_t)(base + b0 + j) * a.F + rr] = swiglu(v, uu);
                        if (tap) tap[(size_t)am->slot[j] * a.F + rr] = av;
                    }
                }
            } else {
                const int cg = grp * 32 + lane;
#pragma unroll
                for (int j = 0; j < kGemvTokens; j++) {
                    if (j < nb) {
                        const int av = tot[j] - am->sum[j];
                        a.ye[(size_t)(base + b0 + j) * a.D + cg] = __fmul_rn((float)av, __fmul_rn(al, am->s[j]));
                        if (a.tap_acc_down) a.tap_acc_down[(size_t)am->slot[j] * a.D + cg] = av;
                    }
                }
            }
            // the last warp of the batch hands it to the publishing warp and frees the buffer
            __syncwarp();
            unsigned prev = 0;
            if (lane == 0) {
                __threadfence_block();
                prev = atomicAdd(&am->done, 1u);
                __threadfence_block();
            }
            prev = __shfl_sync(FULL, prev, 0);
            if (prev != (unsigned)(kDecGroupWarps - 1)) continue;
            if (lane == 0) {
                am->done = 0u;
                const int rs = k % kDecRec;
                if (!dec_wait(b_rempty + 8 * (kDecRec * g + rs), ((k / kDecRec) & 1) ^ 1))
                    set_flag(a.flag_dev, MAPLE_DEVFLAG_TIMEOUT);
                DecRecord *rec = recs + kDecRec * g + rs;
                rec->kind = kind;
                rec->e = e;
                rec->sub = sub;
                rec->nb = nb;
                rec->base = base;
                rec->last = b0 + kGemvTokens >= cnt;
                for (int j = 0; j < nb; j++) rec->slot[j] = am->slot[j];
                dec_arrive(b_rfull + 8 * (kDecRec * g + rs));
                dec_arrive(b_aempty + 8 * (2 * g + buf));
            }
        }
    }
    cp_async_wait<0>();
}

}  // namespace maple
