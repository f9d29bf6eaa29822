// Routing stage: activation quantiser, router logits, top-k + softmax over the
// kept logits, and the token -> expert permutation.
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"
#include "layout.cuh"

namespace maple {

constexpr int kRouteTokens = 8;        // tokens per route CTA (one per warp)
constexpr int kRouteExperts = 8;       // experts per route CTA (one per warp)
constexpr int kFusedMarkBytes = 16384; // largest T*E the routing kernel builds the permutation for itself
constexpr int kPermBlockTokens = 32;   // tokens per CTA of the multi-CTA permutation
constexpr int kMaxExperts = 1024;
constexpr int kRouteSmallT = 64;       // up to this many tokens the latency-oriented router runs

struct RouteArgs {
    const uint16_t *x;
    const float *resid;   // optional (route_kernel): x = bf16(RMSNorm(resid)) computed here, x unused
    int T, D, E, K;
    const float *Wr, *bias;
    // workspace outputs
    int8_t *qx;
    int8_t *qxp;   // optional: q_x rows in the fragment order of the decode kernel (frag_word_pos)
    float *sx;
    int *sumx;
    float *logits;
    int *topk_idx;
    float *topk_w;
    // optional caller outputs (may be null)
    int8_t *tap_qx;
    float *tap_sx, *tap_logits;
    int *out_idx;
    float *out_w;
    // last-arriver counters (zero between launches)
    unsigned *tg_cnt, *glob_cnt;
    // permutation (filled by the last CTA when fuse_permute)
    int fuse_permute;
    unsigned *clear;   // [n_clear] counters of the next kernel, zeroed by CTA (0, 0) (may be null)
    int n_clear;
    int *counts, *offsets, *perm, *inv, *active, *n_active;
    int *out_counts, *tap_offsets, *tap_perm;
    int2 *units;   // optional (with fuse_permute): the decode kernels' units, {expert, first | count << 16}
    int *n_units;
    unsigned *flag;
    int group_tokens;   // route_cluster_kernel: tokens per cluster (8 or 16)
    // optional (with units, T <= 8 and K <= 8): per unit {expert, first position |
    // count << 16, its tokens 0-3 and 4-7 as bytes}, for the fused expert kernel
    int4 *funits;
};

constexpr int kUnitTokens = 16;   // slots of a decode unit (two 8-token MMA n-tiles)
constexpr int kPermCacheSlots = 512;   // route_fused_permutation: slots whose expert it keeps in shared memory
constexpr int kRcExperts = 16;    // route_cluster_kernel: experts per CTA (one per warp)
constexpr int kRcMaxExperts = 256;
constexpr int kRcMaxGroup = 16;   // route_cluster_kernel: tokens per cluster at most (one top-k warp each)

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem, bool pred)
{
    const uint32_t d = (uint32_t)__cvta_generic_to_shared(smem);
    const int n = pred ? 16 : 0;   // zero-fill when out of range
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(gmem), "r"(n) : "memory");
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// ---------------------------------------------------------------------------
// block-wide exclusive scan of one int per thread (blockDim multiple of 32)
// ---------------------------------------------------------------------------
__device__ __forceinline__ int block_excl_scan(int v, int *s_warp, int *total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int n = __shfl_up_sync(FULL, incl, o);
        if (lane >= o) incl += n;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int w = lane < nw ? s_warp[lane] : 0;
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int n = __shfl_up_sync(FULL, wi, o);
            if (lane >= o) wi += n;
        }
        if (lane < nw) s_warp[lane] = wi - w;     // exclusive prefix of warp totals
        if (lane == 31) s_warp[32] = wi;          // grand total
    }
    __syncthreads();
    int res = s_warp[warp] + incl - v;
    if (total) *total = s_warp[32];
    __syncthreads();
    return res;
}

// exclusive scan of s_cnt[0..E) into s_off[0..E] (s_off[E] = total) and the
// ascending list of experts with a nonzero count; any blockDim, E <= 1024
__device__ void scan_experts(const int *s_cnt, int *s_off, int E, int *active, int *n_active, int *s_warp)
{
    const int per = (E + blockDim.x - 1) / blockDim.x;
    const int lo = min(E, (int)threadIdx.x * per), hi = min(E, lo + per);
    int sum = 0, nz = 0;
    for (int e = lo; e < hi; e++) {
        sum += s_cnt[e];
        nz += s_cnt[e] > 0;
    }
    int tot, tot_nz;
    int base = block_excl_scan(sum, s_warp, &tot);
    int base_nz = block_excl_scan(nz, s_warp, &tot_nz);
    for (int e = lo; e < hi; e++) {
        s_off[e] = base;
        base += s_cnt[e];
        if (s_cnt[e] > 0) active[base_nz++] = e;
    }
    if (threadIdx.x == 0) {
        s_off[E] = tot;
        *n_active = tot_nz;
    }
    __syncthreads();
}

// ---------------------------------------------------------------------------
// quantise one token (one warp) from its bf16 row xr (shared memory): amax,
// codes, scale, sum of codes
// ---------------------------------------------------------------------------
template <int NI>
__device__ void quantize_token_warp(const RouteArgs &a, int t, const uint16_t *xr)
{
    const int lane = threadIdx.x & 31;
    uint4 v[NI];
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < NI; i++) {
        v[i] = *reinterpret_cast<const uint4 *>(xr + 256 * i + 8 * lane);
        const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
        for (int m = 0; m < 4; m++) {
            amax = fmaxf(amax, fabsf(bf16_bits_to_f32(w[m] & 0xffffu)));
            amax = fmaxf(amax, fabsf(bf16_bits_to_f32(w[m] >> 16)));
        }
    }
    amax = warp_max(amax);
    const float inv = amax > 0.0f ? __fdiv_rn(127.0f, amax) : 0.0f;
    int sum = 0;
#pragma unroll
    for (int i = 0; i < NI; i++) {
        const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
        uint32_t packed[2] = {0u, 0u};
#pragma unroll
        for (int m = 0; m < 8; m++) {
            uint32_t bits = (m & 1) ? (w[m >> 1] >> 16) : (w[m >> 1] & 0xffffu);
            int q = amax > 0.0f ? quant_code(bf16_bits_to_f32(bits), inv) : 0;
            sum += q;
            packed[m >> 2] |= (uint32_t)(q & 0xff) << (8 * (m & 3));
        }
        uint2 pv = make_uint2(packed[0], packed[1]);
        size_t off = (size_t)t * a.D + 256 * i + 8 * lane;
        *reinterpret_cast<uint2 *>(a.qx + off) = pv;
        if (a.tap_qx) *reinterpret_cast<uint2 *>(a.tap_qx + off) = pv;
        if (a.qxp) {
            // the two words sit at word positions 2(l%16), +1 of 128-column block 2i + l/16
            uint32_t *blk = reinterpret_cast<uint32_t *>(a.qxp + (size_t)t * a.D + 256 * i + 128 * (lane >> 4));
            blk[frag_word_pos(2 * (lane & 15))] = packed[0];
            blk[frag_word_pos(2 * (lane & 15) + 1)] = packed[1];
        }
    }
    sum = warp_sum_int(sum);
    if (lane == 0) {
        float s = amax > 0.0f ? __fdiv_rn(amax, 127.0f) : 0.0f;
        a.sx[t] = s;
        a.sumx[t] = sum;
        if (a.tap_sx) a.tap_sx[t] = s;
    }
}

// ---------------------------------------------------------------------------
// top-k (ties to the lower index) and softmax over the kept logits, one warp
// per token; NPER = logits held per lane (E <= 32*NPER)
// ---------------------------------------------------------------------------
// A logit as a 32-bit value whose unsigned order is the order of the logits:
// the float's bits made order-preserving (-0 taken as +0, which compares
// equal).  No finite or infinite logit maps to 0, which marks a taken entry.
__device__ __forceinline__ uint32_t rank_value(float v)
{
    uint32_t b = __float_as_uint(v);
    if (b == 0x80000000u) b = 0u;
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float rank_value_float(uint32_t o)
{
    return __uint_as_float((o & 0x80000000u) ? (o & 0x7fffffffu) : ~o);
}

// Top-k of one row of E logits (one warp); lane k < K ends with the k-th
// choice (my_e) and its softmax weight (my_w).  Ranking: larger logit first,
// equal logits by lower index.  A NaN logit ranks last and raises the flag.
template <int NPER, bool SMEM = false>
__device__ __forceinline__ void topk_row_warp(const float *row, int E, int K, unsigned *flag, int &my_e, float &my_w)
{
    const int lane = threadIdx.x & 31;
    uint32_t ov[NPER];
    bool nan_seen = false;
#pragma unroll
    for (int j = 0; j < NPER; j++) {
        const int e = lane + 32 * j;
        ov[j] = 0u;
        if (e < E) {
            float v = SMEM ? row[e] : __ldcg(row + e);
            if (isnan(v)) {
                nan_seen = true;
                v = -INFINITY;
            }
            ov[j] = rank_value(v);
        }
    }
    if (__any_sync(FULL, nan_seen) && lane == 0) set_flag(flag, MAPLE_DEVFLAG_NAN);
    // K rounds: the warp's largest value not yet taken (one warp reduction),
    // then the lowest index holding it (a second one); a compact loop, since
    // this runs once per token group on an SM whose instruction cache is cold
    uint32_t my_o = 0u;
    my_e = 0;
#pragma unroll 1
    for (int k = 0; k < K; k++) {
        uint32_t m = 0u;
#pragma unroll
        for (int j = 0; j < NPER; j++) m = max(m, ov[j]);
        const uint32_t best = __reduce_max_sync(FULL, m);
        uint32_t ci = 0xffffffffu;
#pragma unroll
        for (int j = NPER - 1; j >= 0; j--)
            if (ov[j] == best) ci = (uint32_t)(lane + 32 * j);
        const int be = (int)__reduce_min_sync(FULL, ci);
#pragma unroll
        for (int j = 0; j < NPER; j++)
            if (lane + 32 * j == be) ov[j] = 0u;
        if (lane == k) {
            my_o = best;
            my_e = be;
        }
    }
    // softmax over the kept logits: e_k = exp(l_k - l_0), S = e_0 + e_1 + ..., w_k = e_k / S
    const float my_v = rank_value_float(my_o);
    const float l0 = __shfl_sync(FULL, my_v, 0);
    const float ek = exp_ref(__fsub_rn(my_v, l0));
    float S = 0.0f;
    for (int k = 0; k < K; k++) S = __fadd_rn(S, __shfl_sync(FULL, ek, k));
    my_w = __fdiv_rn(ek, S);
}

// top-k of token t from its logits (global, or a row in shared memory), written
// to the routing outputs; returns the lane's choice (lanes < K)
template <int NPER, bool SMEM = false>
__device__ int topk_token_warp(const RouteArgs &a, int t, const float *row = nullptr)
{
    const int lane = threadIdx.x & 31;
    int my_e;
    float my_w;
    topk_row_warp<NPER, SMEM>(SMEM ? row : a.logits + (size_t)t * a.E, a.E, a.K, a.flag, my_e, my_w);
    if (lane < a.K) {
        const size_t o = (size_t)t * a.K + lane;
        a.topk_idx[o] = my_e;
        a.topk_w[o] = my_w;
        if (a.out_idx) a.out_idx[o] = my_e;
        if (a.out_w) a.out_w[o] = my_w;
    }
    return my_e;
}

// ---------------------------------------------------------------------------
// Stable token -> expert permutation of one block of tokens [t0, t0+nt):
// mark[t][e] = k+1 when token t's k-th choice is e (a token's choices are
// distinct), then every expert walks its column in token order.
// ---------------------------------------------------------------------------
__device__ void build_marks(uint8_t *mark, const int *idx, int t0, int nt, int K, int E, unsigned *flag)
{
    // zero ceil(nt*E/16) 16-byte words (callers size mark as a multiple of 16 bytes)
    for (int i = threadIdx.x; i < (nt * E + 15) / 16; i += blockDim.x)
        reinterpret_cast<uint4 *>(mark)[i] = make_uint4(0, 0, 0, 0);
    __syncthreads();
    for (int s = threadIdx.x; s < nt * K; s += blockDim.x) {
        int t = s / K, k = s - t * K;
        int e = __ldcg(idx + (size_t)(t0 + t) * K + k);
        if (e < 0 || e >= E) {
            set_flag(flag, MAPLE_DEVFLAG_BAD_INDEX);
            continue;
        }
        mark[t * E + e] = (uint8_t)(k + 1);
    }
    __syncthreads();
}

// place the block's slots: expert e's first slot in this block goes to base_e(e)
template <class BaseFn>
__device__ void scatter_marks(const uint8_t *mark, int t0, int nt, int K, int E, BaseFn base_e, int *perm, int *inv,
                              int *tap_perm, const float *sx = nullptr, float *pscale = nullptr)
{
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int p = base_e(e);
        for (int t = 0; t < nt; t++) {
            int m = mark[t * E + e];
            if (m) {
                int s = (t0 + t) * K + m - 1;
                perm[p] = s;
                inv[s] = p;
                if (tap_perm) tap_perm[p] = s;
                if (pscale) pscale[p] = sx[t0 + t];
                p++;
            }
        }
    }
}

// ---------------------------------------------------------------------------
// The routing kernel.  grid = (E/8, ceil(T/8)); warp w of CTA (eb, tg) scores
// expert 8*eb + w for tokens 8*tg .. 8*tg+7.  CTAs with eb == 0 also quantise
// their 8 tokens.  The last CTA of a token group to finish runs top-k for it;
// with fuse_permute the last token group to finish builds the permutation.
// Router logit order: lane l sums j = 256*i + 8*l + m (fmaf, from 0), then the
// 32 lane partials are added by the xor tree (distance 16, 8, 4, 2, 1).
// Dynamic shared memory: route_smem_bytes(D) (the bf16 rows of the 8 tokens,
// later reused for the permutation's marks).
// ---------------------------------------------------------------------------
__host__ __device__ inline size_t route_smem_bytes(int D)
{
    const size_t xb = (size_t)kRouteTokens * D * 2;
    return xb > (size_t)kFusedMarkBytes ? xb : (size_t)kFusedMarkBytes;
}

// Stage the bf16 rows of tokens t0 .. t0+nt-1 in shared memory: from x by
// asynchronous copies (all in flight at once), or, for the layer stack, as
// bf16(RMSNorm(resid)) with one warp per token.  Ends with __syncthreads.
template <int NI>
__device__ __forceinline__ void route_stage_tokens(const RouteArgs &a, uint16_t *xs, int t0, int nt)
{
    const int warp = threadIdx.x >> 5;
    if (a.resid) {
        if (warp < nt) rmsnorm_token_warp(a.resid + (size_t)(t0 + warp) * a.D, a.D, xs + (size_t)warp * a.D);
    } else {
        const int n16 = nt * (a.D / 8);
        const uint4 *src = reinterpret_cast<const uint4 *>(a.x + (size_t)t0 * a.D);
        for (int idx = threadIdx.x; idx < n16; idx += blockDim.x)
            cp_async16(reinterpret_cast<uint4 *>(xs) + idx, src + idx, true);
        cp_async_commit();
        cp_async_wait<0>();
    }
    __syncthreads();
}

// Logits of one expert (this warp's router row, in registers as w0/w1) for the
// nt staged tokens, two tokens at a time (two independent fmaf chains, each in
// the pinned order); store(t, logit) is called by lane 0 for t = 0 .. nt-1.
template <int NI, class Store>
__device__ __forceinline__ void route_logits_warp(const RouteArgs &a, const float4 (&w0)[NI], const float4 (&w1)[NI],
                                                  const uint16_t *xs, int nt, float bias_e, Store store)
{
    const int lane = threadIdx.x & 31;
    for (int tt = 0; tt < nt; tt += 2) {
        const int tb = min(tt + 1, nt - 1);   // an odd last token is computed twice, stored once
        float acc0 = 0.0f, acc1 = 0.0f;
#pragma unroll
        for (int i = 0; i < NI; i++) {
            const uint4 xa = *reinterpret_cast<const uint4 *>(xs + (size_t)tt * a.D + 256 * i + 8 * lane);
            const uint4 xb = *reinterpret_cast<const uint4 *>(xs + (size_t)tb * a.D + 256 * i + 8 * lane);
            const uint32_t wa[4] = {xa.x, xa.y, xa.z, xa.w}, wb[4] = {xb.x, xb.y, xb.z, xb.w};
            const float wv[8] = {w0[i].x, w0[i].y, w0[i].z, w0[i].w, w1[i].x, w1[i].y, w1[i].z, w1[i].w};
#pragma unroll
            for (int m = 0; m < 8; m++) {
                const uint32_t ba = (m & 1) ? (wa[m >> 1] >> 16) : (wa[m >> 1] & 0xffffu);
                const uint32_t bb = (m & 1) ? (wb[m >> 1] >> 16) : (wb[m >> 1] & 0xffffu);
                acc0 = __fmaf_rn(bf16_bits_to_f32(ba), wv[m], acc0);
                acc1 = __fmaf_rn(bf16_bits_to_f32(bb), wv[m], acc1);
            }
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {   // the pairwise tree of warp_tree_sum, two rows at once
            acc0 = __fadd_rn(acc0, __shfl_xor_sync(FULL, acc0, o));
            acc1 = __fadd_rn(acc1, __shfl_xor_sync(FULL, acc1, o));
        }
        if (a.bias) {
            acc0 = __fadd_rn(acc0, bias_e);
            acc1 = __fadd_rn(acc1, bias_e);
        }
        if (lane == 0) {
            store(tt, acc0);
            if (tb != tt) store(tb, acc1);
        }
    }
}

// The permutation of all T*K slots (T <= 64) in one CTA, from every token's
// choices (expert_of(slot)).  Per expert the mask of the tokens that chose it
// (a token's choices are distinct); a slot's position is its expert's offset
// plus the number of earlier tokens in the mask, so every step is a constant
// number of shared-memory operations per thread (no loop over tokens).  Also
// writes the decode kernels' units.  s_mask: E words of shared memory.
template <class ExpertOf>
__device__ void route_fused_permutation(const RouteArgs &a, unsigned long long *s_mask, int *s_warp, ExpertOf expert_of)
{
    __shared__ int s_cnt[kMaxExperts];
    __shared__ int s_off[kMaxExperts + 1];
    __shared__ short s_ev[kPermCacheSlots];   // the first slots' experts, read once
    for (int ee = threadIdx.x; ee < a.E; ee += blockDim.x) s_mask[ee] = 0ull;
    __syncthreads();
    for (int sl = threadIdx.x; sl < a.T * a.K; sl += blockDim.x) {
        const int ee = expert_of(sl);
        if (sl < kPermCacheSlots) s_ev[sl] = (short)(ee < 0 || ee >= a.E ? -1 : ee);
        if (ee < 0 || ee >= a.E) {
            set_flag(a.flag, MAPLE_DEVFLAG_BAD_INDEX);
            continue;
        }
        atomicOr(s_mask + ee, 1ull << (sl / a.K));
    }
    __syncthreads();
    for (int ee = threadIdx.x; ee < a.E; ee += blockDim.x) s_cnt[ee] = __popcll(s_mask[ee]);
    __syncthreads();
    scan_experts(s_cnt, s_off, a.E, a.active, a.n_active, s_warp);
    for (int ee = threadIdx.x; ee <= a.E; ee += blockDim.x) {
        a.offsets[ee] = s_off[ee];
        if (a.tap_offsets) a.tap_offsets[ee] = s_off[ee];
        if (ee < a.E) {
            a.counts[ee] = s_cnt[ee];
            if (a.out_counts) a.out_counts[ee] = s_cnt[ee];
        }
    }
    for (int sl = threadIdx.x; sl < a.T * a.K; sl += blockDim.x) {
        const int ee = sl < kPermCacheSlots ? (int)s_ev[sl] : expert_of(sl);
        if (ee < 0 || ee >= a.E) continue;
        const int t = sl / a.K;
        const int p = s_off[ee] + __popcll(s_mask[ee] & ((1ull << t) - 1ull));
        a.perm[p] = sl;
        a.inv[sl] = p;
        if (a.tap_perm) a.tap_perm[p] = sl;
    }
    if (a.units) {
        // units: every expert's slots cut into runs of at most kUnitTokens, in expert order
        const int per = (a.E + blockDim.x - 1) / blockDim.x;
        const int lo = min(a.E, (int)threadIdx.x * per), hi = min(a.E, lo + per);
        int nu = 0;
        for (int ee = lo; ee < hi; ee++) nu += (s_cnt[ee] + kUnitTokens - 1) / kUnitTokens;
        int total;
        int u = block_excl_scan(nu, s_warp, &total);
        for (int ee = lo; ee < hi; ee++)
            for (int u0 = 0; u0 < s_cnt[ee]; u0 += kUnitTokens)
                a.units[u++] = make_int2(ee, (s_off[ee] + u0) | (min(kUnitTokens, s_cnt[ee] - u0) << 16));
        if (threadIdx.x == 0) *a.n_units = total;
    }
}

template <int NI, int NPER>
__global__ void __launch_bounds__(256, 2) route_kernel(RouteArgs a)
{
    extern __shared__ __align__(16) uint8_t rsm[];
    uint16_t *xs = (uint16_t *)rsm;   // [nt][D] bf16
    __shared__ unsigned s_last;
    __shared__ int s_warp[33];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int eb = blockIdx.x, tg = blockIdx.y;
    const int t0 = tg * kRouteTokens;
    const int nt = min(kRouteTokens, a.T - t0);
    const int e = eb * kRouteExperts + warp;
    // let a kernel launched after this one as a programmatic dependent start its
    // set-up now (it waits for this grid's completion before reading any output)
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    // this lane's part of the router row, all in flight at once (the router
    // weights are not written by any kernel, so this may run before the wait)
    const float *wr = a.Wr + (size_t)e * a.D;
    float4 w0[NI], w1[NI];
#pragma unroll
    for (int i = 0; i < NI; i++) {
        w0[i] = __ldg(reinterpret_cast<const float4 *>(wr + 256 * i + 8 * lane));
        w1[i] = __ldg(reinterpret_cast<const float4 *>(wr + 256 * i + 8 * lane + 4));
    }
    // launched as a programmatic dependent (the layer stack), wait here for the
    // grid before, which wrote the input; otherwise this returns at once
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (a.clear && eb == 0 && tg == 0)
        for (int i = threadIdx.x; i < a.n_clear; i += blockDim.x) a.clear[i] = 0u;
    route_stage_tokens<NI>(a, xs, t0, nt);

    if (eb == 0 && warp < nt) quantize_token_warp<NI>(a, t0 + warp, xs + (size_t)warp * a.D);

    route_logits_warp<NI>(a, w0, w1, xs, nt, a.bias ? a.bias[e] : 0.0f, [&](int t, float v) {
        a.logits[(size_t)(t0 + t) * a.E + e] = v;
        if (a.tap_logits) a.tap_logits[(size_t)(t0 + t) * a.E + e] = v;
    });

    // ---- last CTA of this token group: top-k + softmax
    fence_gpu();
    __syncthreads();
    if (threadIdx.x == 0) {
        unsigned prev = atomicAdd(a.tg_cnt + tg, 1u);
        s_last = (prev == gridDim.x - 1);
    }
    __syncthreads();
    if (!s_last) return;
    fence_gpu();
    if (threadIdx.x == 0) a.tg_cnt[tg] = 0;
    if (warp < nt) topk_token_warp<NPER>(a, t0 + warp);
    if (!a.fuse_permute) return;

    // ---- last token group: permutation of all T*K slots in one CTA
    fence_gpu();
    __syncthreads();
    if (threadIdx.x == 0) {
        unsigned prev = atomicAdd(a.glob_cnt, 1u);
        s_last = (prev == gridDim.y - 1);
    }
    __syncthreads();
    if (!s_last) return;
    fence_gpu();
    if (threadIdx.x == 0) *a.glob_cnt = 0;

    route_fused_permutation(a, reinterpret_cast<unsigned long long *>(rsm), s_warp,
                            [&](int sl) { return __ldcg(a.topk_idx + sl); });
}

// The same permutation for T <= 8 (K <= 8, E <= 256) by one warp, from the
// choices in shared memory (ch[slot]): per expert an 8-bit token mask,
// counts, offsets and the active list by warp scans, so no block-wide barrier
// is taken.  Every active expert is one unit (at most 8 slots).
__device__ void route_perm_warp(const RouteArgs &a, const int *ch)
{
    __shared__ uint32_t s_m8[kRcMaxExperts / 4];   // 8-bit token masks, four experts a word
    __shared__ int s_off[kRcMaxExperts];
    const int lane = threadIdx.x & 31;
    const int S = a.T * a.K, per = (a.E + 31) / 32, e0 = lane * per;
    for (int w = lane; w < a.E / 4; w += 32) s_m8[w] = 0u;
    __syncwarp();
    for (int sl = lane; sl < S; sl += 32) {
        const int e = ch[sl];
        if (e < 0 || e >= a.E) {
            set_flag(a.flag, MAPLE_DEVFLAG_BAD_INDEX);
            continue;
        }
        atomicOr(s_m8 + e / 4, 1u << (8 * (e & 3) + sl / a.K));
    }
    __syncwarp();
    int cnt[8], sum = 0, nz = 0;   // this lane's experts e0 .. e0+per-1 (per <= 8)
#pragma unroll
    for (int i = 0; i < 8; i++) {
        const int e = e0 + i;
        cnt[i] = (i < per && e < a.E) ? __popc((s_m8[e / 4] >> (8 * (e & 3))) & 0xffu) : 0;
        sum += cnt[i];
        nz += cnt[i] > 0;
    }
    int off = sum, act = nz;   // inclusive warp scans, made exclusive below
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(FULL, off, o), w = __shfl_up_sync(FULL, act, o);
        if (lane >= o) {
            off += v;
            act += w;
        }
    }
    const int total = __shfl_sync(FULL, off, 31), n_act = __shfl_sync(FULL, act, 31);
    off -= sum;
    act -= nz;
#pragma unroll
    for (int i = 0; i < 8; i++) {
        const int e = e0 + i;
        if (i >= per || e >= a.E) break;
        s_off[e] = off;
        a.offsets[e] = off;
        a.counts[e] = cnt[i];
        if (a.tap_offsets) a.tap_offsets[e] = off;
        if (a.out_counts) a.out_counts[e] = cnt[i];
        if (cnt[i]) {
            a.active[act] = e;
            if (a.units) a.units[act] = make_int2(e, off | (cnt[i] << 16));
            if (a.funits) {   // its tokens in order, one byte each
                uint32_t m = (s_m8[e / 4] >> (8 * (e & 3))) & 0xffu, tk[2] = {0u, 0u};
                for (int j = 0; m; j++, m &= m - 1u) tk[j >> 2] |= (uint32_t)(__ffs(m) - 1) << (8 * (j & 3));
                a.funits[act] = make_int4(e, off | (cnt[i] << 16), (int)tk[0], (int)tk[1]);
            }
            act++;
        }
        off += cnt[i];
    }
    if (lane == 0) {
        a.offsets[a.E] = total;
        if (a.tap_offsets) a.tap_offsets[a.E] = total;
        *a.n_active = n_act;
        if (a.units) *a.n_units = n_act;
    }
    __syncwarp();
    for (int sl = lane; sl < S; sl += 32) {
        const int e = ch[sl];
        if (e < 0 || e >= a.E) continue;
        const int t = sl / a.K;
        const int p = s_off[e] + __popc((s_m8[e / 4] >> (8 * (e & 3))) & ((1u << t) - 1u));
        a.perm[p] = sl;
        a.inv[sl] = p;
        if (a.tap_perm) a.tap_perm[p] = sl;
    }
}

// ---------------------------------------------------------------------------
// The routing kernel on thread-block clusters (T <= 64, E <= 256 and a
// multiple of 16): one cluster of E/16 CTAs per group of 8 or 16 tokens (16
// when 8-token groups would need more clusters than fit at once), 16 warps per
// CTA, warp w of cluster rank r scoring expert 16r + w with the same
// arithmetic in the same order as route_kernel.  Every warp writes its logits
// straight into rank 0's shared memory (distributed shared memory); after the
// cluster barrier rank 0 runs top-k for the group's tokens from there, so no
// logit goes through global memory and no CTA waits on a counter.  With one
// token group (T <= 8) rank 0 builds the permutation at once from its own
// choices; with several, the last group to finish does (as in route_kernel).
// Dynamic shared memory: route_cluster_smem_bytes(D, E, group_tokens).
// ---------------------------------------------------------------------------
__host__ __device__ inline size_t route_cluster_rows_bytes(int D, int E, int gt)
{
    const size_t xb = (size_t)gt * D * 2, mb = (size_t)E * 8;   // token rows, later the experts' masks
    return xb > mb ? xb : mb;
}
__host__ __device__ inline size_t route_cluster_smem_bytes(int D, int E, int gt)
{
    // + the group's logits [gt][E] and its choices [gt][8]
    return route_cluster_rows_bytes(D, E, gt) + (size_t)gt * E * 4 + (size_t)gt * 8 * 4;
}

// a cluster barrier in two halves (every thread of every CTA of the cluster)
__device__ __forceinline__ void cluster_arrive() { asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory"); }
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }

template <int NI, int NPER>
__global__ void __launch_bounds__(512, 1) route_cluster_kernel(RouteArgs a)
{
    namespace cg = cooperative_groups;
    extern __shared__ __align__(16) uint8_t rsm[];
    uint16_t *xs = (uint16_t *)rsm;                                       // [nt][D] bf16
    const int gt = a.group_tokens;
    float *lg = (float *)(rsm + route_cluster_rows_bytes(a.D, a.E, gt));  // [gt][E] (rank 0)
    int *ch = (int *)(lg + gt * a.E);                                     // [gt][K] (rank 0, one group)
    __shared__ unsigned s_last;
    __shared__ int s_warp[33];
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tg = blockIdx.y, t0 = tg * gt;
    const int nt = min(gt, a.T - t0);
    const int e = rank * kRcExperts + warp;
    // first cluster barrier, split: arriving says this CTA is running; its wait
    // comes before the first write into rank 0's shared memory
    cluster_arrive();
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    const float *wr = a.Wr + (size_t)e * a.D;
    float4 w0[NI], w1[NI];
#pragma unroll
    for (int i = 0; i < NI; i++) {
        w0[i] = __ldg(reinterpret_cast<const float4 *>(wr + 256 * i + 8 * lane));
        w1[i] = __ldg(reinterpret_cast<const float4 *>(wr + 256 * i + 8 * lane + 4));
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (a.clear && rank == 0 && tg == 0)
        for (int i = threadIdx.x; i < a.n_clear; i += blockDim.x) a.clear[i] = 0u;
    route_stage_tokens<NI>(a, xs, t0, nt);

    float *lg0 = cluster.map_shared_rank(lg, 0);   // rank 0's logit rows
    cluster_wait();
    route_logits_warp<NI>(a, w0, w1, xs, nt, a.bias ? a.bias[e] : 0.0f, [&](int t, float v) {
        lg0[t * a.E + e] = v;
        if (a.tap_logits) a.tap_logits[(size_t)(t0 + t) * a.E + e] = v;
    });
    cluster.sync();   // every logit of the group is in rank 0's shared memory
    if (rank != 0) return;

    // top-k by warps 0 .. nt-1 while warps 16-nt .. 15 quantise the tokens
    // (q_x feeds the expert kernels, not the router)
    int my_e = 0;
    if (warp < nt) {
        my_e = topk_token_warp<NPER, true>(a, t0 + warp, lg + warp * a.E);
    }
    if (warp >= kRcExperts - nt) quantize_token_warp<NI>(a, t0 + warp - (kRcExperts - nt), xs + (size_t)(warp - (kRcExperts - nt)) * a.D);
    if (!a.fuse_permute) return;
    if (gridDim.y == 1) {
        // one token group: the choices are the top-k warps' own; once they are
        // all in shared memory (a barrier of those warps alone: the quantising
        // warps go on by themselves), warp 0 builds the permutation, its masks
        // over the logit rows, which are no longer read
        if (warp >= nt) return;
        if (lane < a.K) ch[warp * a.K + lane] = my_e;
        if (nt > 1) asm volatile("bar.sync 1, %0;" ::"r"(32 * nt) : "memory");
        if (warp == 0) route_perm_warp(a, ch);   // (one group of 8 tokens: T <= 8)
        return;
    }
    // several token groups: the last to finish builds the permutation
    fence_gpu();
    __syncthreads();
    if (threadIdx.x == 0) {
        unsigned prev = atomicAdd(a.glob_cnt, 1u);
        s_last = (prev == gridDim.y - 1);
    }
    __syncthreads();
    if (!s_last) return;
    fence_gpu();
    if (threadIdx.x == 0) *a.glob_cnt = 0;
    route_fused_permutation(a, reinterpret_cast<unsigned long long *>(rsm), s_warp,
                            [&](int sl) { return __ldcg(a.topk_idx + sl); });
}

// ---------------------------------------------------------------------------
// Multi-CTA permutation for large T: (1) per-block counts, (2) per-expert scan
// over blocks and over experts, (3) scatter.
// ---------------------------------------------------------------------------
struct PermArgs {
    const int *idx;
    int T, K, E;
    int *blk_cnt;  // [nblk][E]: counts, then (after pass 2) global base positions
    int *counts, *offsets, *perm, *inv, *active, *n_active;
    int *out_counts, *tap_offsets, *tap_perm;
    int4 *pieces;   // optional: expert slot ranges of at most kPieceSlots for the grouped GEMM
    int *n_pieces;
    const float *sx;   // with pscale: s_x of every token
    float *pscale;     // optional: s_x of each position's token (the tensor-core path's column scales)
    unsigned *flag;
};

constexpr int kPieceSlots = 128;

__global__ void __launch_bounds__(256) perm_count_kernel(PermArgs a)
{
    __shared__ __align__(16) uint8_t s_mark[kPermBlockTokens * kMaxExperts];
    const int t0 = blockIdx.x * kPermBlockTokens;
    const int nt = min(kPermBlockTokens, a.T - t0);
    build_marks(s_mark, a.idx, t0, nt, a.K, a.E, a.flag);
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
        int c = 0;
        for (int t = 0; t < nt; t++) c += s_mark[t * a.E + e] != 0;
        a.blk_cnt[(size_t)blockIdx.x * a.E + e] = c;
    }
}

__global__ void __launch_bounds__(1024) perm_scan_kernel(PermArgs a)
{
    __shared__ int s_cnt[kMaxExperts];
    __shared__ int s_off[kMaxExperts + 1];
    __shared__ int s_warp[33];
    constexpr int kB = 16;   // per-block counts loaded 16 at a time (independent loads in flight)
    const int nblk = (a.T + kPermBlockTokens - 1) / kPermBlockTokens;
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
        int run = 0;
        for (int b0 = 0; b0 < nblk; b0 += kB) {
            int c[kB];
#pragma unroll
            for (int j = 0; j < kB; j++) c[j] = b0 + j < nblk ? a.blk_cnt[(size_t)(b0 + j) * a.E + e] : 0;
#pragma unroll
            for (int j = 0; j < kB; j++) run += c[j];
        }
        s_cnt[e] = run;
    }
    __syncthreads();
    scan_experts(s_cnt, s_off, a.E, a.active, a.n_active, s_warp);
    for (int e = threadIdx.x; e <= a.E; e += blockDim.x) {
        a.offsets[e] = s_off[e];
        if (a.tap_offsets) a.tap_offsets[e] = s_off[e];
        if (e < a.E) {
            a.counts[e] = s_cnt[e];
            if (a.out_counts) a.out_counts[e] = s_cnt[e];
            // first position of expert e's slots in each token block
            int run = s_off[e];
            for (int b0 = 0; b0 < nblk; b0 += kB) {
                int c[kB];
#pragma unroll
                for (int j = 0; j < kB; j++) c[j] = b0 + j < nblk ? a.blk_cnt[(size_t)(b0 + j) * a.E + e] : 0;
#pragma unroll
                for (int j = 0; j < kB; j++)
                    if (b0 + j < nblk) {
                        a.blk_cnt[(size_t)(b0 + j) * a.E + e] = run;
                        run += c[j];
                    }
            }
        }
    }
    if (a.pieces) {
        // split every expert's slots into ceil(count / kPieceSlots) near-equal
        // ranges, listed by size, largest first (a counting sort over the sizes;
        // the order of equal sizes is arbitrary: every piece is computed on its
        // own, so it changes no result, only which CTA takes which piece)
        __shared__ int s_size[kPieceSlots + 1];
        for (int i = threadIdx.x; i <= kPieceSlots; i += blockDim.x) s_size[i] = 0;
        __syncthreads();
        const int e = threadIdx.x;
        const int cnt = e < a.E ? s_cnt[e] : 0;
        const int np = (cnt + kPieceSlots - 1) / kPieceSlots;
        const int q = np ? cnt / np : 0, rem = np ? cnt % np : 0;
        if (rem) atomicAdd(&s_size[q + 1], rem);
        if (np - rem) atomicAdd(&s_size[q], np - rem);
        __syncthreads();
        if (threadIdx.x == 0) {
            int run = 0;   // first list position of each size, sizes in descending order
            for (int z = kPieceSlots; z >= 1; z--) {
                const int c = s_size[z];
                s_size[z] = run;
                run += c;
            }
            *a.n_pieces = run;
        }
        __syncthreads();
        for (int i = 0; i < np; i++) {
            const int sz = q + (i < rem ? 1 : 0);
            const int start = i * q + min(i, rem);
            a.pieces[atomicAdd(&s_size[sz], 1)] = make_int4(e, s_off[e] + start, sz, 0);
        }
    }
}

__global__ void __launch_bounds__(256) perm_scatter_kernel(PermArgs a)
{
    __shared__ __align__(16) uint8_t s_mark[kPermBlockTokens * kMaxExperts];
    const int t0 = blockIdx.x * kPermBlockTokens;
    const int nt = min(kPermBlockTokens, a.T - t0);
    build_marks(s_mark, a.idx, t0, nt, a.K, a.E, nullptr);
    const int *base = a.blk_cnt + (size_t)blockIdx.x * a.E;
    scatter_marks(s_mark, t0, nt, a.K, a.E, [&](int e) { return base[e]; }, a.perm, a.inv, a.tap_perm, a.sx,
                  a.pscale);
}

// ---------------------------------------------------------------------------
// Router for many tokens (register-tiled SIMT GEMM in the same fixed order).
// CTA = 32 tokens x 16 experts, 8 warps; warp w owns tokens 8*(w/2)..+7 and
// experts 8*(w%2)..+7 and keeps, per lane, the 64 partial sums of that lane's
// part of K (lane l: j = 256*i + 8*l + m).  Per K chunk of 256 the CTA stages
// the token rows (bf16) and router rows (fp32) in shared memory.  The 32 lane
// partials of every output are then added with the same xor tree as the
// decode router, as a transposing reduction: at the level with distance o a
// lane keeps half of its outputs and sends the other half to lane l^o, so lane
// l ends with outputs 2l and 2l+1 (token 2l/8, expert 2l%8 + {0,1}).
// ---------------------------------------------------------------------------
constexpr int kRgTok = 32, kRgExp = 16;

template <int N>
__device__ __forceinline__ void tree_level(float (&v)[64], int off, bool upper)
{
#pragma unroll
    for (int j = 0; j < N / 2; j++) {
        const float send = upper ? v[j] : v[j + N / 2];
        const float keep = upper ? v[j + N / 2] : v[j];
        v[j] = __fadd_rn(keep, __shfl_xor_sync(FULL, send, off));
    }
}


// dynamic shared memory: two stages of (32 token rows x 256 bf16, 16 router rows x 256 fp32)
constexpr int kRgStage = kRgTok * 256 * 2 + kRgExp * 256 * 4;

__global__ void __launch_bounds__(256, 1) router_gemm_kernel(const uint16_t *x, int T, int D, int E, const float *Wr,
                                                             const float *bias, float *logits, float *tap_logits)
{
    extern __shared__ __align__(16) uint8_t rg_smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t0 = blockIdx.x * kRgTok, e0 = blockIdx.y * kRgExp;
    const int wt = (warp >> 1) * 8, we = (warp & 1) * 8;
    const int NI = D / 256;
    auto stage = [&](int i, int buf) {
        uint16_t *sx = (uint16_t *)(rg_smem + buf * kRgStage);
        float *sw = (float *)(rg_smem + buf * kRgStage + kRgTok * 256 * 2);
        for (int q = threadIdx.x; q < kRgTok * 32; q += 256) {
            const int tt = q >> 5, c = q & 31;
            const bool ok = t0 + tt < T;
            cp_async16(sx + tt * 256 + c * 8, x + (size_t)(ok ? t0 + tt : 0) * D + 256 * i + c * 8, ok);
        }
        for (int q = threadIdx.x; q < kRgExp * 64; q += 256) {
            const int ee = q >> 6, c = q & 63;
            cp_async16(sw + ee * 256 + c * 4, Wr + (size_t)(e0 + ee) * D + 256 * i + c * 4, true);
        }
        cp_async_commit();
    };
    float acc[64];
#pragma unroll
    for (int o = 0; o < 64; o++) acc[o] = 0.0f;
    stage(0, 0);
    for (int i = 0; i < NI; i++) {
        if (i + 1 < NI) {
            stage(i + 1, (i + 1) & 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        const uint16_t *sx = (const uint16_t *)(rg_smem + (i & 1) * kRgStage);
        const float *sw = (const float *)(rg_smem + (i & 1) * kRgStage + kRgTok * 256 * 2);
#pragma unroll
        for (int h = 0; h < 2; h++) {   // lane's 8 elements of the chunk, 4 at a time (m = 4h .. 4h+3)
            float wv[8][4];
#pragma unroll
            for (int b = 0; b < 8; b++) {
                const float4 w4 = *reinterpret_cast<const float4 *>(sw + (we + b) * 256 + 8 * lane + 4 * h);
                wv[b][0] = w4.x; wv[b][1] = w4.y; wv[b][2] = w4.z; wv[b][3] = w4.w;
            }
#pragma unroll
            for (int aa = 0; aa < 8; aa++) {
                const uint2 xv = *reinterpret_cast<const uint2 *>(sx + (wt + aa) * 256 + 8 * lane + 4 * h);
                const float xf[4] = {bf16_bits_to_f32(xv.x & 0xffffu), bf16_bits_to_f32(xv.x >> 16),
                                     bf16_bits_to_f32(xv.y & 0xffffu), bf16_bits_to_f32(xv.y >> 16)};
#pragma unroll
                for (int b = 0; b < 8; b++)
#pragma unroll
                    for (int m = 0; m < 4; m++) acc[aa * 8 + b] = __fmaf_rn(xf[m], wv[b][m], acc[aa * 8 + b]);
            }
        }
        __syncthreads();
    }
    tree_level<64>(acc, 16, lane & 16);
    tree_level<32>(acc, 8, lane & 8);
    tree_level<16>(acc, 4, lane & 4);
    tree_level<8>(acc, 2, lane & 2);
    tree_level<4>(acc, 1, lane & 1);
#pragma unroll
    for (int q = 0; q < 2; q++) {
        const int o = 2 * lane + q;
        const int t = t0 + wt + o / 8, e = e0 + we + o % 8;
        if (t < T) {
            float v = acc[q];
            if (bias) v = __fadd_rn(v, bias[e]);
            logits[(size_t)t * E + e] = v;
            if (tap_logits) tap_logits[(size_t)t * E + e] = v;
        }
    }
}

// quantise + top-k/softmax for many tokens: one warp per token
// (dynamic shared memory: 8 rows of D bf16)
template <int NI, int NPER>
__global__ void __launch_bounds__(256) quant_topk_kernel(RouteArgs a)
{
    extern __shared__ __align__(16) uint8_t qsm[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint16_t *xr = (uint16_t *)qsm + (size_t)warp * NI * 256;
    const int t = blockIdx.x * 8 + warp;
    if (t >= a.T) return;
#pragma unroll
    for (int i = 0; i < NI; i++)
        reinterpret_cast<uint4 *>(xr + 256 * i)[lane] =
            __ldg(reinterpret_cast<const uint4 *>(a.x + (size_t)t * a.D + 256 * i) + lane);
    __syncwarp();
    quantize_token_warp<NI>(a, t, xr);
    topk_token_warp<NPER>(a, t);
}

}  // namespace maple
