// Shared device helpers of the ternary MoE layer kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#define MAPLE_DEVFLAG_NAN 0x1u
#define MAPLE_DEVFLAG_BAD_INDEX 0x2u
#define MAPLE_DEVFLAG_BAD_VALUE 0x4u
#define MAPLE_DEVFLAG_TIMEOUT 0x8u

namespace maple {

constexpr unsigned FULL = 0xffffffffu;

// upper bound (ns) a thread may stay suspended in one mbarrier.try_wait; the
// hardware wakes it as soon as the phase completes, so waiting threads take no
// issue slots from the ones doing work
constexpr uint32_t kSuspendHintNs = 200000;

// default limit of every bounded wait in the kernels (2 s, far above any
// legitimate wait); a handle may set another one
constexpr uint64_t kDefaultWaitNs = 2000000000ull;

__device__ __forceinline__ uint64_t global_timer_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// ---------------------------------------------------------------------------
// exp(x), written out from the mathematics so that host and device give the
// same bits: clamp to [-87, 88]; n = rint(x*log2 e); r = x - n ln2 with ln2
// split into a 17-bit head and a tail (Cody-Waite); Taylor polynomial of
// degree 7 in r by Horner's rule with fused multiply-adds; times 2^n built
// from exponent bits.  Coefficients are 1/k! rounded once to binary32.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float exp_ref(float x)
{
    const float kLog2e = 0x1.715476p+0f;   // 1/ln 2
    const float kLn2Hi = 0x1.62e4p-1f;     // 0.693145751953125
    const float kLn2Lo = 0x1.7f7d1cp-20f;  // ln 2 - kLn2Hi
    x = fminf(fmaxf(x, -87.0f), 88.0f);
    float n = rintf(__fmul_rn(x, kLog2e));
    float r = __fmaf_rn(-n, kLn2Hi, x);
    r = __fmaf_rn(-n, kLn2Lo, r);
    float p = 0x1.a01a02p-13f;             // 1/7!
    p = __fmaf_rn(p, r, 0x1.6c16c2p-10f);  // 1/6!
    p = __fmaf_rn(p, r, 0x1.111112p-7f);   // 1/5!
    p = __fmaf_rn(p, r, 0x1.555556p-5f);   // 1/4!
    p = __fmaf_rn(p, r, 0x1.555556p-3f);   // 1/3!
    p = __fmaf_rn(p, r, 0.5f);             // 1/2!
    p = __fmaf_rn(p, r, 1.0f);             // 1/1!
    p = __fmaf_rn(p, r, 1.0f);             // 1/0!
    float scale = __int_as_float(((int)n + 127) << 23);
    return __fmul_rn(p, scale);
}

// SiLU(g) * u with every step rounded once: (g / (1 + exp(-g))) * u
__device__ __forceinline__ float swiglu(float g, float u)
{
    float den = __fadd_rn(1.0f, exp_ref(-g));
    return __fmul_rn(__fdiv_rn(g, den), u);
}

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b16) { return __uint_as_float(b16 << 16); }

// round a finite float to bf16 (nearest, ties to even); returns the 16 bits
__device__ __forceinline__ uint16_t f32_to_bf16_bits(float f)
{
    uint32_t u = __float_as_uint(f);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

// int8 absmax code of v given inv = 127/amax: clamp(rint(v*inv), -127, 127)
__device__ __forceinline__ int quant_code(float v, float inv)
{
    int q = __float2int_rn(__fmul_rn(v, inv));
    return max(-127, min(127, q));
}

__device__ __forceinline__ float warp_max(float v)
{
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(FULL, v, o));
    return v;
}

__device__ __forceinline__ int warp_sum_int(int v)
{
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(FULL, v, o);
    return v;
}

// Pairwise tree over the 32 lanes: lane l with l^16, then 8, 4, 2, 1.  Every
// lane ends with the same value (fp addition is commutative).
__device__ __forceinline__ float warp_tree_sum(float v)
{
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v = __fadd_rn(v, __shfl_xor_sync(FULL, v, o));
    return v;
}

// d = c + sum of the four byte products (a unsigned bytes, b signed bytes)
__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c)
{
    int d;
    asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// 16-byte streaming load that skips L1 (weights are read once per use)
__device__ __forceinline__ uint4 ld_stream_v4(const void *p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// GPU-scope acquire-release fence: orders this thread's earlier global writes
// before its later ones (and earlier reads before later reads) for all CTAs;
// used around the last-arriver counters
__device__ __forceinline__ void fence_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }

__device__ __forceinline__ void set_flag(unsigned *flag, unsigned bits)
{
    if (flag) atomicOr(flag, bits);
}

// One token's pre-norm input, one warp: out = bf16(r / rms) with
// rms = sqrt(sum(r^2) / D + 1e-6), norm weights 1; the sum of squares in the
// router's fixed order (lane l takes j = 256i + 8l + m with fmaf, then the
// pairwise tree).  `out` may be global or shared memory.
__device__ __forceinline__ void rmsnorm_token_warp(const float *r, int D, uint16_t *out)
{
    const int lane = threadIdx.x & 31;
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
        *reinterpret_cast<uint4 *>(out + 256 * i + 8 * lane) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    }
}

}  // namespace maple
