// Routing stage: activation quantiser, router logits, top-k + softmax over the
// kept logits, and the token -> expert permutation.
#pragma once

#include "common.cuh"

namespace maple {

constexpr int kRouteTokens = 8;        // tokens per route CTA (one per warp)
constexpr int kRouteExperts = 8;       // experts per route CTA (one per warp)
constexpr int kFusedMarkBytes = 16384; // T*E bytes the fused single-CTA permutation can hold
constexpr int kPermBlockTokens = 32;   // tokens per CTA of the multi-CTA permutation
constexpr int kMaxExperts = 1024;

struct RouteArgs {
    const uint16_t *x;
    int T, D, E, K;
    const float *Wr, *bias;
    // workspace outputs
    int8_t *qx;
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
    int *counts, *offsets, *perm, *inv, *active, *n_active;
    int *out_counts, *tap_offsets, *tap_perm;
    unsigned *flag;
};

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
// quantise one token (one warp): amax, codes, scale, sum of codes
// ---------------------------------------------------------------------------
__device__ void quantize_token_warp(const RouteArgs &a, int t)
{
    const int lane = threadIdx.x & 31;
    const uint16_t *xr = a.x + (size_t)t * a.D;
    float amax = 0.0f;
    for (int i = 0; i < a.D / 256; i++) {
        uint4 v = *reinterpret_cast<const uint4 *>(xr + 256 * i + 8 * lane);
        uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int m = 0; m < 4; m++) {
            amax = fmaxf(amax, fabsf(bf16_bits_to_f32(w[m] & 0xffffu)));
            amax = fmaxf(amax, fabsf(bf16_bits_to_f32(w[m] >> 16)));
        }
    }
    amax = warp_max(amax);
    const float inv = amax > 0.0f ? __fdiv_rn(127.0f, amax) : 0.0f;
    int sum = 0;
    for (int i = 0; i < a.D / 256; i++) {
        uint4 v = *reinterpret_cast<const uint4 *>(xr + 256 * i + 8 * lane);
        uint32_t w[4] = {v.x, v.y, v.z, v.w};
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
__device__ __forceinline__ bool ranks_before(float v, int e, float bv, int be)
{
    return v > bv || (v == bv && e < be);
}

template <int NPER>
__device__ void topk_token_warp(const RouteArgs &a, int t)
{
    const int lane = threadIdx.x & 31;
    float lv[NPER];
    bool nan_seen = false;
#pragma unroll
    for (int j = 0; j < NPER; j++) {
        int e = lane + 32 * j;
        float v = -INFINITY;
        if (e < a.E) {
            v = __ldcg(a.logits + (size_t)t * a.E + e);
            if (isnan(v)) {
                nan_seen = true;
                v = -INFINITY;
            }
        }
        lv[j] = v;
    }
    if (__any_sync(FULL, nan_seen) && lane == 0) set_flag(a.flag, MAPLE_DEVFLAG_NAN);
    uint32_t taken = 0;
    float my_v = 0.0f;
    int my_e = 0;
    for (int k = 0; k < a.K; k++) {
        float bv = -INFINITY;
        int be = 0x7fffffff;
#pragma unroll
        for (int j = 0; j < NPER; j++) {
            int e = lane + 32 * j;
            if (e < a.E && !((taken >> j) & 1u) && ranks_before(lv[j], e, bv, be)) {
                bv = lv[j];
                be = e;
            }
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            float ov = __shfl_xor_sync(FULL, bv, o);
            int oe = __shfl_xor_sync(FULL, be, o);
            if (ranks_before(ov, oe, bv, be)) {
                bv = ov;
                be = oe;
            }
        }
        if ((be & 31) == lane) taken |= 1u << (be >> 5);
        if (lane == k) {
            my_v = bv;
            my_e = be;
        }
    }
    // softmax over the kept logits: e_k = exp(l_k - l_0), S = e_0 + e_1 + ..., w_k = e_k / S
    const float l0 = __shfl_sync(FULL, my_v, 0);
    const float ek = exp_ref(__fsub_rn(my_v, l0));
    float S = 0.0f;
    for (int k = 0; k < a.K; k++) S = __fadd_rn(S, __shfl_sync(FULL, ek, k));
    if (lane < a.K) {
        const float w = __fdiv_rn(ek, S);
        const size_t o = (size_t)t * a.K + lane;
        a.topk_idx[o] = my_e;
        a.topk_w[o] = w;
        if (a.out_idx) a.out_idx[o] = my_e;
        if (a.out_w) a.out_w[o] = w;
    }
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
                              int *tap_perm)
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
// ---------------------------------------------------------------------------
template <int NPER>
__global__ void __launch_bounds__(256) route_kernel(RouteArgs a)
{
    __shared__ unsigned s_last;
    __shared__ int s_warp[33];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int eb = blockIdx.x, tg = blockIdx.y;
    const int t0 = tg * kRouteTokens;
    const int nt = min(kRouteTokens, a.T - t0);

    if (eb == 0 && warp < nt) quantize_token_warp(a, t0 + warp);

    {
        const int e = eb * kRouteExperts + warp;
        const float *wr = a.Wr + (size_t)e * a.D;
        float acc[kRouteTokens];
#pragma unroll
        for (int tt = 0; tt < kRouteTokens; tt++) acc[tt] = 0.0f;
        for (int i = 0; i < a.D / 256; i++) {
            const float4 w0 = *reinterpret_cast<const float4 *>(wr + 256 * i + 8 * lane);
            const float4 w1 = *reinterpret_cast<const float4 *>(wr + 256 * i + 8 * lane + 4);
            const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
            for (int tt = 0; tt < kRouteTokens; tt++) {
                if (tt < nt) {
                    const uint4 xv = *reinterpret_cast<const uint4 *>(a.x + (size_t)(t0 + tt) * a.D + 256 * i + 8 * lane);
                    const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
                    for (int m = 0; m < 8; m++) {
                        uint32_t bits = (m & 1) ? (xw[m >> 1] >> 16) : (xw[m >> 1] & 0xffffu);
                        acc[tt] = __fmaf_rn(bf16_bits_to_f32(bits), wv[m], acc[tt]);
                    }
                }
            }
        }
#pragma unroll
        for (int tt = 0; tt < kRouteTokens; tt++) {
            if (tt < nt) {
                float v = warp_tree_sum(acc[tt]);
                if (a.bias) v = __fadd_rn(v, a.bias[e]);
                if (lane == 0) {
                    a.logits[(size_t)(t0 + tt) * a.E + e] = v;
                    if (a.tap_logits) a.tap_logits[(size_t)(t0 + tt) * a.E + e] = v;
                }
            }
        }
    }

    // ---- last CTA of this token group: top-k + softmax
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        unsigned prev = atomicAdd(a.tg_cnt + tg, 1u);
        s_last = (prev == gridDim.x - 1);
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    if (threadIdx.x == 0) a.tg_cnt[tg] = 0;
    if (warp < nt) topk_token_warp<NPER>(a, t0 + warp);
    if (!a.fuse_permute) return;

    // ---- last token group: permutation of all T*K slots in one CTA
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        unsigned prev = atomicAdd(a.glob_cnt, 1u);
        s_last = (prev == gridDim.y - 1);
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    if (threadIdx.x == 0) *a.glob_cnt = 0;

    __shared__ __align__(16) uint8_t s_mark[kFusedMarkBytes];
    __shared__ int s_cnt[kMaxExperts];
    __shared__ int s_off[kMaxExperts + 1];
    build_marks(s_mark, a.topk_idx, 0, a.T, a.K, a.E, a.flag);
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
        int c = 0;
        for (int t = 0; t < a.T; t++) c += s_mark[t * a.E + e] != 0;
        s_cnt[e] = c;
    }
    __syncthreads();
    scan_experts(s_cnt, s_off, a.E, a.active, a.n_active, s_warp);
    for (int e = threadIdx.x; e <= a.E; e += blockDim.x) {
        a.offsets[e] = s_off[e];
        if (a.tap_offsets) a.tap_offsets[e] = s_off[e];
        if (e < a.E) {
            a.counts[e] = s_cnt[e];
            if (a.out_counts) a.out_counts[e] = s_cnt[e];
        }
    }
    scatter_marks(s_mark, 0, a.T, a.K, a.E, [&](int e) { return s_off[e]; }, a.perm, a.inv, a.tap_perm);
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
    unsigned *flag;
};

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
    const int nblk = (a.T + kPermBlockTokens - 1) / kPermBlockTokens;
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
        int run = 0;
        for (int b = 0; b < nblk; b++) {
            int c = a.blk_cnt[(size_t)b * a.E + e];
            a.blk_cnt[(size_t)b * a.E + e] = run;
            run += c;
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
            for (int b = 0; b < nblk; b++) a.blk_cnt[(size_t)b * a.E + e] += s_off[e];
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
    scatter_marks(s_mark, t0, nt, a.K, a.E, [&](int e) { return base[e]; }, a.perm, a.inv, a.tap_perm);
}

}  // namespace maple
