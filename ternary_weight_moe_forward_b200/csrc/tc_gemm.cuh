// Prefill expert stage on the 5th-generation tensor cores (tcgen05, int8).
//
// Grouped GEMM over "pieces": a piece is up to 128 consecutive slots of one
// expert in the permutation (the routing stage lists them largest first).  A
// tile is (piece, 128-row block of the weight matrix).  The MMA computes
// D[128 weight rows][N slots] (M = 128, N = the piece size rounded up to 16,
// K = 32 per instruction) with
//   A = ternary weights, expanded in shared memory from 2-bit codes to int8
//       {0, +64, -64} (64 * t: the code sits in the two top bits of the byte),
//   B = int8 activation rows of the piece's slots,
// both K-major with the 128-byte swizzle, the int32 accumulator in tensor
// memory (two accumulator buffers, so the epilogue of one tile overlaps the
// MMAs of the next).  The accumulator is 64x the ternary dot product; the
// epilogue shifts it back (exact).
//
// Warp roles (20 warps): warp 0 issues the bulk copies of the 2-bit codes,
// warp 2 the activation loads (lane 0), warp 1 the MMAs (and owns the TMEM
// allocation), warps 4..11 run the epilogue (TMEM lane quarter = warp % 4,
// two warps per quarter splitting the columns), warps 12..19 expand the codes
// into int8 tiles.  Three rings of K stages with their own lifetimes: the
// codes (small, deep: freed as soon as they are expanded), the activation
// tiles (freed by the MMAs) and the expanded weight tiles (two or three
// stages: expansion is quick and local), so that the loads run many stages
// ahead of the MMAs.  Hand-off uses mbarriers; every wait is bounded in time
// and a timeout makes the whole CTA drain and return with a device flag set.
//
// Mode 0 (gate/up): A = gate rows and up rows of one 128-row block (two MMAs
// per K step, gate and up accumulators 128 columns apart), B = the q_x rows of
// the piece's positions (gather_rows_kernel has laid out the q_x row of every
// position in position order), one 2-D TMA copy per stage.  (Fetching them
// straight from q_x by four-row TMA gathers, 32 per stage, kept the loading
// warp issuing for most of the kernel.)  A CTA takes whole pieces (all F/128 row blocks of one piece in a
// row, pieces dealt out in a snake order over the size-sorted list), so that
// it holds every h value of its slots: the epilogue writes h = SiLU(g) * u
// (fp32) to a per-CTA scratch area, stored with an L2 evict-last policy (and
// the codes copied evict-first) so that it stays in L2; after the piece's last
// row block the epilogue warps requantise the slots, a slot's row at a time
// in registers (its |h| maximum by a warp reduction, then the int8 absmax
// codes q_h and the scale s_h), so no fp32 h leaves the chip.
// Mode 1 (down): A = 128 output channels of the down matrix, B = q_h rows
// (consecutive slot positions, a plain 2-D TMA load); tiles are dealt out
// round robin.  The epilogue stores the exact int32 accumulators, which need
// 17 bits (|acc| <= 127 * 512): acc >> 1 as int16 and the lowest bit in a bit
// plane (one 32-bit word per 32 channels, by warp ballot), 2.125 bytes per
// value instead of 4 for fp32 yE; combine_kernel rebuilds acc and scales it
// exactly as the oracle does.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace maple {

constexpr int kTcThreads = 640;
constexpr int kTcEpiWarp0 = 4, kTcEpiWarps = 8;     // epilogue warps 4..11
constexpr int kTcProdWarp0 = 12, kTcProdWarps = 8;  // code-expanding warps 12..19
constexpr int kTcMaxN = 128;
constexpr int kTcBK = 128;  // K elements (bytes) per stage = one swizzle row

// 2-bit tensor-core layout, one 16-value word per (row, 16-column chunk):
//   gate/up [E][F/128][D/128][2][128][8] words, down [E][D/128][F/128][128][8]
// word w of (row, stage ks) holds columns ks*128 + 16w + 4k + b at bits
// 8b + 2k as a two's complement 2-bit code (+1 -> 01, -1 -> 11, 0 -> 00).
__host__ __device__ inline uint32_t tc_word(uint32_t canon)
{
    uint32_t out = 0;
    for (int i = 0; i < 16; i++) {
        uint32_t c = (canon >> (2 * i)) & 3u;
        uint32_t s = c == 1u ? 1u : (c == 2u ? 3u : 0u);
        out |= s << (8 * (i & 3) + 2 * (i >> 2));
    }
    return out;
}

template <int MODE>
struct TcCfg;
template <>
struct TcCfg<0> {
    static constexpr int kCS = 6, kBS = 4, kAS = 3;   // stages of the code, activation and weight rings
    static constexpr int kABytes = 2 * 128 * kTcBK;   // gate + up blocks
    static constexpr int kCodeBytes = 2 * 128 * 32;   // 8 words of 4 bytes per row
};
template <>
struct TcCfg<1> {
    static constexpr int kCS = 8, kBS = 6, kAS = 3;
    static constexpr int kABytes = 128 * kTcBK;
    static constexpr int kCodeBytes = 128 * 32;
};

template <int MODE>
struct TcSmem {
    using C = TcCfg<MODE>;
    static constexpr int kBBytes = kTcMaxN * kTcBK;
    static constexpr int kA = 0;                                   // [kAS] expanded weight tiles
    static constexpr int kB = kA + C::kAS * C::kABytes;            // [kBS] activation tiles
    static constexpr int kCodes = kB + C::kBS * kBBytes;           // [kCS] 2-bit codes
    static constexpr int kBars = kCodes + C::kCS * C::kCodeBytes;  // barriers, TMEM holder, abort word: 512 B
    static constexpr int kMeta = kBars + 512;                      // epilogue column metadata [2][2][128]
    static constexpr int kTotal = kMeta + 2 * 2 * kTcMaxN * 4;
    static constexpr int kNumBars = 2 * (C::kCS + C::kBS + C::kAS) + 5;
    static_assert(C::kABytes % 1024 == 0 && kBBytes % 1024 == 0, "tiles must keep 1024-byte alignment");
    static_assert(8 * kNumBars + 8 <= 512, "barrier area");
};

struct TcArgs {
    int D, F, K;
    const int4 *pieces;      // {expert, first position, count, 0}, largest first
    const int *n_pieces;
    const uint8_t *codes;    // tensor-core layout
    const int *perm;         // position -> slot
    float *sh;               // mode 0: written (s_h per position); mode 1: read
    const float *pscale;     // mode 0: s_x of each position's token
    const float *alpha0, *alpha1;  // mode 0: gate, up; mode 1: down, unused
    float *out;              // mode 0: per-CTA h scratch [gridDim][128][F]
    int8_t *qh;              // mode 0: q_h [S][F] (position order)
    int16_t *acc_hi;         // mode 1: down accumulators >> 1 [S][D] (position order)
    uint32_t *acc_lo;        // mode 1: their lowest bits, [S][D/32] words (bit c%32 = channel c)
    int *tap0, *tap1;        // mode 0: acc_gate, acc_up; mode 1: acc_down
    int8_t *tap_qh;          // mode 0 (slot order, may be null)
    float *tap_sh;
    unsigned *flag;
    uint64_t wait_ns;        // limit of every bounded wait
};

// ---------------------------------------------------------------------------
// PTX wrappers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_addr(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(kSuspendHintNs)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ uint64_t global_ns() { return global_timer_ns(); }

// Wait for the phase of `bar` with the given parity to complete.  Gives up
// after `limit` ns, or at once when another role of the CTA has given up;
// returns false then (and raises the CTA abort word and the device flag).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile uint32_t *abort, unsigned *flag,
                                          uint64_t limit)
{
    if (mbar_test(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    while (true) {
        if (mbar_test(bar, parity)) return true;
        if (*abort) return false;
        if (global_ns() - t0 > limit) {
            *abort = 1u;
            set_flag(flag, MAPLE_DEVFLAG_TIMEOUT);
            return false;
        }
    }
}

__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}
// L2 cache policies: the weight codes are read once (evict first), the
// gate/up kernel's h scratch is read back once by the same CTA (evict last)
__device__ __forceinline__ uint64_t l2_evict_first()
{
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t l2_evict_last()
{
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ void bulk_g2s_hint(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar, uint64_t pol)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;"
                 ::"r"(dst), "l"(src), "r"(bytes), "r"(bar), "l"(pol)
                 : "memory");
}
__device__ __forceinline__ void st_f32_hint(float *p, float v, uint64_t pol)
{
    asm volatile("st.global.L2::cache_hint.f32 [%0], %1, %2;" ::"l"(p), "f"(v), "l"(pol) : "memory");
}
// 2-D tiled TMA load (box given by the tensor map) into 128B-swizzled shared memory
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y, uint32_t bar)
{
    asm volatile("cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];"
                 ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
                 : "memory");
}
__device__ __forceinline__ void cp_async4_tc(void *smem, const void *gmem)
{
    const uint32_t d = (uint32_t)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(d), "l"(gmem) : "memory");
}
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void fence_barrier_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_alloc(uint32_t holder_smem, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(holder_smem), "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, int8 x int8 -> int32
__device__ __forceinline__ void mma_i8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t acc)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc), "r"(0), "r"(0), "r"(0), "r"(0)
        : "memory");
}
__device__ __forceinline__ void mma_commit(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, int (&v)[32])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
          "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
          "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
        : "r"(taddr)
        : "memory");
}
// 32 lanes x 16 consecutive 32-bit columns
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, int *v)
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr)
        : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// K-major operand, 128-byte swizzle: rows of 128 bytes, 8-row atoms 1024 bytes apart
__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr)
{
    uint64_t d = (uint64_t)((saddr & 0x3FFFFu) >> 4);
    d |= (uint64_t)1 << 16;             // leading byte offset (unused for swizzled K-major)
    d |= (uint64_t)(1024 >> 4) << 32;   // stride byte offset: next 8-row atom
    d |= (uint64_t)1 << 46;             // descriptor version (sm_100)
    d |= (uint64_t)2 << 61;             // 128-byte swizzle
    return d;
}

// instruction descriptor: kind::i8, s8 x s8 -> s32, both K-major, M = 128
__device__ __forceinline__ uint32_t idesc_i8(int n)
{
    return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

// byte offset of 16-byte chunk `chunk` of row `row` in a 128-byte-swizzled tile
__device__ __forceinline__ uint32_t sw128(int row, int chunk) { return row * 128 + ((chunk ^ (row & 7)) << 4); }

// four planes of a 2-bit word as int8 {0, +64, -64}, 16 consecutive columns
__device__ __forceinline__ uint4 expand_word(uint32_t w)
{
    return make_uint4((w << 6) & 0xC0C0C0C0u, (w << 4) & 0xC0C0C0C0u, (w << 2) & 0xC0C0C0C0u, w & 0xC0C0C0C0u);
}

// ---------------------------------------------------------------------------
// The CTA's u-th tile: piece (index into the size-sorted list) and row block;
// false once the CTA has no more.  Mode 0 deals out whole pieces: the j-th
// piece of CTA b is j*G + b for even j and j*G + G-1-b for odd j (a snake over
// the sorted list, which evens out the work), its R row blocks one after the
// other.  Mode 1 deals out tiles round robin over the piece-major tile list.
template <int MODE>
__device__ __forceinline__ bool tc_tile(int u, int R, int n_pc, int &pc, int &rb)
{
    const int G = gridDim.x, b = blockIdx.x;
    if (MODE == 0) {
        const int j = u / R;
        pc = j * G + ((j & 1) ? G - 1 - b : b);
        rb = u - j * R;
        return pc < n_pc;
    }
    const int t = b + u * G;
    pc = t / R;
    rb = t - pc * R;
    return pc < n_pc;
}

template <int MODE>
__global__ void __launch_bounds__(kTcThreads, 1) tc_gemm_kernel(const __grid_constant__ CUtensorMap act_map, TcArgs a)
{
    using Cfg = TcCfg<MODE>;
    using L = TcSmem<MODE>;
    constexpr int CS = Cfg::kCS, BS = Cfg::kBS, AS = Cfg::kAS;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = smem_raw;
    if (smem_addr(smem) & 1023u) {   // the 128-byte-swizzled tiles need 1024-byte alignment
        if (threadIdx.x == 0) set_flag(a.flag, MAPLE_DEVFLAG_TIMEOUT);
        return;
    }
    int *meta_slot = (int *)(smem + L::kMeta);                      // [2][kTcMaxN]
    float *meta_scale = (float *)(smem + L::kMeta + 2 * kTcMaxN * 4);
    uint64_t *bars = (uint64_t *)(smem + L::kBars);
    // bars: codes_full[CS], codes_empty[CS], act_full[BS], act_empty[BS], w_full[AS], w_empty[AS],
    // acc_full[2], acc_empty[2], drain
    uint32_t *tmem_holder = (uint32_t *)(bars + L::kNumBars);
    volatile uint32_t *abort = tmem_holder + 1;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t b_codes_full = smem_addr(bars), b_codes_empty = b_codes_full + 8 * CS;
    const uint32_t b_act_full = b_codes_empty + 8 * CS, b_act_empty = b_act_full + 8 * BS;
    const uint32_t b_w_full = b_act_empty + 8 * BS, b_w_empty = b_w_full + 8 * AS;
    const uint32_t b_acc_full = b_w_empty + 8 * AS, b_acc_empty = b_acc_full + 16, b_drain = b_acc_empty + 16;

    if (threadIdx.x == 0) {
        for (int s = 0; s < CS; s++) {
            mbar_init(b_codes_full + 8 * s, 1);                 // bulk copy
            mbar_init(b_codes_empty + 8 * s, kTcProdWarps);     // one arrival per producer warp
        }
        for (int s = 0; s < BS; s++) {
            mbar_init(b_act_full + 8 * s, 1);                   // TMA
            mbar_init(b_act_empty + 8 * s, 1);                  // MMA commit
        }
        for (int s = 0; s < AS; s++) {
            mbar_init(b_w_full + 8 * s, kTcProdWarps);          // one arrival per producer warp
            mbar_init(b_w_empty + 8 * s, 1);                    // MMA commit
        }
        for (int b = 0; b < 2; b++) {
            mbar_init(b_acc_full + 8 * b, 1);
            mbar_init(b_acc_empty + 8 * b, kTcEpiWarps);  // one arrival per epilogue warp
        }
        mbar_init(b_drain, 1);
        *abort = 0u;
        fence_barrier_init();
    }
    if (warp == 1) tmem_alloc(smem_addr(tmem_holder), 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    const int R = MODE == 0 ? a.F / 128 : a.D / 128;   // row blocks per piece
    const int KS = MODE == 0 ? a.D / kTcBK : a.F / kTcBK;
    const int n_pc = __ldg(a.n_pieces);

    if (warp == 0) {
        // ---------------- bulk copies of the 2-bit codes, up to CS stages ahead
        if (lane == 0) {
            const uint64_t pol = l2_evict_first();
            uint32_t it = 0;
            bool ok = true;
            int pc, rb;
            for (int u = 0; ok && tc_tile<MODE>(u, R, n_pc, pc, rb); u++) {
                const int4 P = a.pieces[pc];
                const uint8_t *src = a.codes + ((size_t)P.x * R + rb) * KS * Cfg::kCodeBytes;
                for (int ks = 0; ks < KS; ks++, it++) {
                    const int s = it % CS;
                    if (!mbar_wait(b_codes_empty + 8 * s, ((it / CS) & 1) ^ 1, abort, a.flag, a.wait_ns)) {
                        ok = false;
                        break;
                    }
                    mbar_expect_tx(b_codes_full + 8 * s, Cfg::kCodeBytes);
                    bulk_g2s_hint(smem_addr(smem + L::kCodes + s * Cfg::kCodeBytes), src + (size_t)ks * Cfg::kCodeBytes,
                             Cfg::kCodeBytes, b_codes_full + 8 * s, pol);
                }
            }
            if (!ok) {
                // drain: wait (bounded) for the copies still in flight, the last CS issued
                for (uint32_t j = (it > (uint32_t)CS ? it - CS : 0); j < it; j++) {
                    const uint64_t t0 = global_ns();
                    while (!mbar_test(b_codes_full + 8 * (j % CS), (j / CS) & 1) && global_ns() - t0 < a.wait_ns) {
                    }
                }
            }
        }
    } else if (warp == 2) {
        // ---------------- activation tiles, up to BS stages ahead: 128 consecutive
        // position rows (mode 0: the q_x row of every position, mode 1: q_h), one
        // 2-D copy per stage
        uint32_t it = 0;
        bool ok = true;
        int pc, rb;
        for (int u = 0; ok && tc_tile<MODE>(u, R, n_pc, pc, rb); u++) {
            const int4 P = a.pieces[pc];
            for (int ks = 0; ks < KS; ks++, it++) {
                const int s = it % BS;
                if (lane == 0) ok = mbar_wait(b_act_empty + 8 * s, ((it / BS) & 1) ^ 1, abort, a.flag, a.wait_ns);
                ok = __shfl_sync(FULL, ok, 0);
                if (!ok) break;
                const uint32_t full = b_act_full + 8 * s;
                if (lane == 0) {
                    mbar_expect_tx(full, L::kBBytes);
                    tma_load_2d(smem_addr(smem + L::kB + s * L::kBBytes), &act_map, ks * kTcBK, P.y, full);
                }
                __syncwarp();
            }
        }
        if (!ok && lane == 0) {
            for (uint32_t j = (it > (uint32_t)BS ? it - BS : 0); j < it; j++) {
                const uint64_t t0 = global_ns();
                while (!mbar_test(b_act_full + 8 * (j % BS), (j / BS) & 1) && global_ns() - t0 < a.wait_ns) {
                }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issue
        if (lane == 0) {
            uint32_t it = 0, tcount = 0;
            bool ok = true;
            int pc, rb;
            for (int u = 0; ok && tc_tile<MODE>(u, R, n_pc, pc, rb); u++, tcount++) {
                const int4 P = a.pieces[pc];
                const int npad = (P.z + 15) & ~15;
                const uint32_t idesc = idesc_i8(npad);
                const uint32_t ab = tcount & 1, dt = tmem + 256 * ab;
                if (!mbar_wait(b_acc_empty + 8 * ab, ((tcount >> 1) & 1) ^ 1, abort, a.flag, a.wait_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                for (int ks = 0; ks < KS; ks++, it++) {
                    const int sw = it % AS, sb_ = it % BS;
                    if (!mbar_wait(b_w_full + 8 * sw, (it / AS) & 1, abort, a.flag, a.wait_ns) ||
                        !mbar_wait(b_act_full + 8 * sb_, (it / BS) & 1, abort, a.flag, a.wait_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_addr(smem + L::kA + sw * Cfg::kABytes);
                    const uint32_t sb = smem_addr(smem + L::kB + sb_ * L::kBBytes);
                    const uint64_t da0 = desc_sw128(sa), db = desc_sw128(sb);
                    const uint64_t da1 = desc_sw128(sa + 128 * kTcBK);
#pragma unroll
                    for (int k = 0; k < kTcBK / 32; k++) {
                        const uint32_t acc = (ks | k) != 0;
                        mma_i8(dt, da0 + 2 * k, db + 2 * k, idesc, acc);
                        if (MODE == 0) mma_i8(dt + 128, da1 + 2 * k, db + 2 * k, idesc, acc);
                    }
                    mma_commit(b_w_empty + 8 * sw);     // both tiles are free once these MMAs are done
                    mma_commit(b_act_empty + 8 * sb_);
                }
                if (!ok) break;
                mma_commit(b_acc_full + 8 * ab);
            }
            // make sure every issued MMA has finished before TMEM is released
            mma_commit(b_drain);
            const uint64_t t0 = global_ns();
            while (!mbar_test(b_drain, 0) && global_ns() - t0 < a.wait_ns) {
            }
        }
    } else if (warp >= kTcEpiWarp0 && warp < kTcEpiWarp0 + kTcEpiWarps) {
        // ---------------- epilogue: TMEM -> registers -> global
        // Warp ew takes lane quarter q = warp % 4 (rows 32q .. 32q+31 of the
        // block) and every other chunk of 32 columns (half hf = ew / 4).  The
        // next tile's per-column metadata (slot ids and token / slot scales,
        // contiguous per piece) is copied with cp.async and its row scales loaded
        // into registers while this tile is processed.
        const int ew = warp - kTcEpiWarp0;
        const int q = warp & 3, hf = ew >> 2;
        const int r = q * 32 + lane;
        const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16);
        const int ldo = MODE == 0 ? a.F : a.D;
        const float *scale_src = MODE == 0 ? a.pscale : a.sh;
        float *hs = MODE == 0 ? a.out + (size_t)blockIdx.x * kTcMaxN * a.F : nullptr;   // [128 slots][F]
        const uint64_t pol_h = l2_evict_last();   // (the scratch is read back by this CTA)
        auto fetch = [&](int buf, const int4 &P, int rbk, float &al0, float &al1) {
            const int row = rbk * 128 + r;
            al0 = a.alpha0[(size_t)P.x * ldo + row];
            al1 = MODE == 0 ? a.alpha1[(size_t)P.x * ldo + row] : 0.0f;
            if (hf == 0 && r < P.z) {   // one slot id and one scale per column (4-byte copies: any alignment)
                cp_async4_tc(meta_slot + buf * kTcMaxN + r, a.perm + P.y + r);
                cp_async4_tc(meta_scale + buf * kTcMaxN + r, scale_src + P.y + r);
            }
            asm volatile("cp.async.commit_group;" ::: "memory");
        };
        uint32_t tcount = 0;
        bool dead = false;   // after a failed wait: keep the loop (and its named barriers) in step, do nothing
        int npc = 0, nrb = 0;
        float nal0 = 0.0f, nal1 = 0.0f;
        bool have = tc_tile<MODE>(0, R, n_pc, npc, nrb);
        int4 nP = have ? a.pieces[npc] : make_int4(0, 0, 0, 0);
        if (have) fetch(0, nP, nrb, nal0, nal1);
        while (have) {
            const int rb = nrb;
            const int4 P = nP;
            const float al0 = nal0, al1 = nal1;
            const uint32_t ab = tcount & 1, tb = tbase + 256 * ab;
            const int row = rb * 128 + r;
            const int p0 = P.y, n = P.z;
            const int *ms = meta_slot + ab * kTcMaxN;
            const float *mf = meta_scale + ab * kTcMaxN;
            asm volatile("cp.async.wait_group 0;" ::: "memory");
            asm volatile("bar.sync 2, 256;" ::: "memory");   // this tile's metadata is in place
            have = tc_tile<MODE>((int)tcount + 1, R, n_pc, npc, nrb);
            if (have) {
                nP = a.pieces[npc];
                fetch(ab ^ 1, nP, nrb, nal0, nal1);
            }
            if (!dead && !mbar_wait(b_acc_full + 8 * ab, (tcount >> 1) & 1, abort, a.flag, a.wait_ns)) dead = true;
            if (!dead) {
                tc_fence_after();
                if (MODE == 0) {
                    // h = SiLU(g) * u to the scratch; the slots' |h| maxima are taken
                    // when the piece is requantised (each slot's row is then in registers)
                    // Sixteen columns per TMEM load, eight values at a time computed with
                    // no branch between them, so that their dependency chains interleave,
                    // and stored afterwards (columns past the piece's end hold no slot:
                    // computed, never stored).
                    for (int c0 = 32 * hf; c0 < n; c0 += 64) {
#pragma unroll
                        for (int jj = 0; jj < 32; jj += 16) {
                            const int cb = c0 + jj;
                            if (cb >= n) break;
                            int g[16], u[16];
                            tmem_ld16(tb + cb, g);
                            tmem_ld16(tb + 128 + cb, u);
                            tmem_wait_ld();
                            float *hd = hs + (size_t)cb * a.F + row;
#pragma unroll
                            for (int j0 = 0; j0 < 16; j0 += 8) {   // eight chains at a time (register budget)
                                float hv[8];
#pragma unroll
                                for (int j = 0; j < 8; j++) {
                                    const float sxt = mf[cb + j0 + j];
                                    const float gv = __fmul_rn((float)(g[j0 + j] >> 6), __fmul_rn(al0, sxt));
                                    const float uv = __fmul_rn((float)(u[j0 + j] >> 6), __fmul_rn(al1, sxt));
                                    hv[j] = swiglu(gv, uv);
                                }
                                if (cb + j0 + 8 <= n) {
#pragma unroll
                                    for (int j = 0; j < 8; j++) st_f32_hint(hd + (size_t)(j0 + j) * a.F, hv[j], pol_h);
                                } else {
#pragma unroll
                                    for (int j = 0; j < 8; j++)
                                        if (cb + j0 + j < n) st_f32_hint(hd + (size_t)(j0 + j) * a.F, hv[j], pol_h);
                                }
                            }
                            if (a.tap0 || a.tap1) {
                                // the raw accumulators, loaded again (checking runs only)
                                tmem_ld16(tb + cb, g);
                                tmem_ld16(tb + 128 + cb, u);
                                tmem_wait_ld();
                                for (int j = 0; j < 16 && cb + j < n; j++) {
                                    if (a.tap0) a.tap0[(size_t)ms[cb + j] * a.F + row] = g[j] >> 6;
                                    if (a.tap1) a.tap1[(size_t)ms[cb + j] * a.F + row] = u[j] >> 6;
                                }
                            }
                        }
                    }
                } else {
                    // The warp's 32 channels x 32 slot columns: per slot the 32 lanes
                    // (consecutive channels) write acc >> 1 as one 64-byte run, and the
                    // slot's low bits (the column's ballot) go out as one word from lane j.
                    const int row0 = rb * 128 + q * 32;   // this warp's first channel
                    for (int c0 = 32 * hf; c0 < n; c0 += 64) {
                        uint32_t my_lo = 0;   // lane j: the low bits of column j
#pragma unroll
                        for (int hh = 0; hh < 32; hh += 16) {   // sixteen columns at a time (register budget)
                            const int cb = c0 + hh;
                            int dd[16];
                            tmem_ld16(tb + cb, dd);
                            tmem_wait_ld();
#pragma unroll
                            for (int j = 0; j < 16; j++) {
                                dd[j] >>= 6;
                                const uint32_t lo = __ballot_sync(FULL, dd[j] & 1);
                                my_lo = lane == hh + j ? lo : my_lo;
                            }
                            int16_t *dst = a.acc_hi + ((size_t)p0 + cb) * a.D + row0 + lane;
                            if (cb + 16 <= n) {
#pragma unroll
                                for (int j = 0; j < 16; j++) dst[(size_t)j * a.D] = (int16_t)(dd[j] >> 1);
                            } else {
#pragma unroll
                                for (int j = 0; j < 16; j++)
                                    if (cb + j < n) dst[(size_t)j * a.D] = (int16_t)(dd[j] >> 1);
                            }
                            if (a.tap0)
                                for (int j = 0; j < 16 && cb + j < n; j++) a.tap0[(size_t)ms[cb + j] * a.D + row] = dd[j];
                        }
                        if (c0 + lane < n) a.acc_lo[((size_t)p0 + c0 + lane) * (a.D / 32) + (row0 >> 5)] = my_lo;
                    }
                    (void)al0;
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(b_acc_empty + 8 * ab);
            }
            if (MODE == 0 && rb == R - 1) {
                // the piece's last row block: requantise its slots (h from the scratch
                // area, read past L1)
                __threadfence_block();
                asm volatile("bar.sync 3, 256;" ::: "memory");
                if (!dead) {
                    // two slots per round and 512 columns at a time, all eight of a
                    // lane's loads in flight together: first each slot's |h| maximum
                    // (over the lane's values, then the warp), then the codes (for
                    // d_ff <= 512 from the same registers, else from a second pass)
                    for (int i = ew; i < n; i += 2 * kTcEpiWarps) {
                        const int ib = i + kTcEpiWarps;   // the round's second slot (if any)
                        float4 hv[2][4];
                        float am[2] = {0.0f, 0.0f};
                        auto load = [&](int c0) {
#pragma unroll
                            for (int k = 0; k < 4; k++) {
                                const int c = c0 + lane + 32 * k;   // d_ff need not be a multiple of 512
                                hv[0][k] = hv[1][k] = make_float4(0.f, 0.f, 0.f, 0.f);
                                if (c < a.F / 4) {
                                    hv[0][k] = __ldcg(reinterpret_cast<const float4 *>(hs + (size_t)i * a.F) + c);
                                    if (ib < n) hv[1][k] = __ldcg(reinterpret_cast<const float4 *>(hs + (size_t)ib * a.F) + c);
                                }
                            }
                        };
                        for (int c0 = 0; c0 < a.F / 4; c0 += 128) {
                            load(c0);
#pragma unroll
                            for (int r = 0; r < 2; r++)
#pragma unroll
                                for (int k = 0; k < 4; k++)
                                    am[r] = fmaxf(fmaxf(am[r], fmaxf(fabsf(hv[r][k].x), fabsf(hv[r][k].y))),
                                                  fmaxf(fabsf(hv[r][k].z), fabsf(hv[r][k].w)));
                        }
#pragma unroll
                        for (int o = 16; o >= 1; o >>= 1) {
                            am[0] = fmaxf(am[0], __shfl_xor_sync(FULL, am[0], o));
                            am[1] = fmaxf(am[1], __shfl_xor_sync(FULL, am[1], o));
                        }
                        const float inv0 = am[0] > 0.0f ? __fdiv_rn(127.0f, am[0]) : 0.0f;
                        const float inv1 = am[1] > 0.0f ? __fdiv_rn(127.0f, am[1]) : 0.0f;
                        for (int c0 = 0; c0 < a.F / 4; c0 += 128) {
                            if (a.F / 4 > 128) load(c0);   // the registers hold only the last 512 columns
#pragma unroll
                            for (int r = 0; r < 2; r++) {
                                const int ii = r ? ib : i;
                                if (ii >= n) break;
                                const float amx = am[r], inv = r ? inv1 : inv0;
                                const int p = p0 + ii, slot = ms[ii];
#pragma unroll
                                for (int k = 0; k < 4; k++) {
                                    const int c = c0 + lane + 32 * k;
                                    if (c >= a.F / 4) break;
                                    int q0 = 0, q1 = 0, q2 = 0, q3 = 0;
                                    if (amx > 0.0f) {
                                        q0 = quant_code(hv[r][k].x, inv);
                                        q1 = quant_code(hv[r][k].y, inv);
                                        q2 = quant_code(hv[r][k].z, inv);
                                        q3 = quant_code(hv[r][k].w, inv);
                                    }
                                    const uint32_t pk = (uint32_t)(q0 & 0xff) | ((uint32_t)(q1 & 0xff) << 8) |
                                                        ((uint32_t)(q2 & 0xff) << 16) | ((uint32_t)(q3 & 0xff) << 24);
                                    reinterpret_cast<uint32_t *>(a.qh + (size_t)p * a.F)[c] = pk;
                                    if (a.tap_qh) reinterpret_cast<uint32_t *>(a.tap_qh + (size_t)slot * a.F)[c] = pk;
                                }
                            }
                        }
                        if (lane == 0) {
#pragma unroll
                            for (int r = 0; r < 2; r++) {
                                const int ii = r ? ib : i;
                                if (ii >= n) break;
                                const float sv = am[r] > 0.0f ? __fdiv_rn(am[r], 127.0f) : 0.0f;
                                a.sh[p0 + ii] = sv;
                                if (a.tap_sh) a.tap_sh[ms[ii]] = sv;
                            }
                        }
                    }
                }
                asm volatile("bar.sync 3, 256;" ::: "memory");   // every read of the scratch is done
            }
            tcount++;
        }
    } else if (warp >= kTcProdWarp0) {
        // ---------------- producers: expand the 2-bit codes into int8 A tiles
        const int pid = threadIdx.x - kTcProdWarp0 * 32;
        uint32_t it = 0;
        bool ok = true;
        int pc, rb;
        for (int u = 0; ok && tc_tile<MODE>(u, R, n_pc, pc, rb); u++) {
            for (int ks = 0; ks < KS; ks++, it++) {
                const int sc = it % CS, sw = it % AS;
                if (!mbar_wait(b_codes_full + 8 * sc, (it / CS) & 1, abort, a.flag, a.wait_ns) ||
                    !mbar_wait(b_w_empty + 8 * sw, ((it / AS) & 1) ^ 1, abort, a.flag, a.wait_ns)) {
                    ok = false;
                    break;
                }
                uint8_t *st = smem + sw * Cfg::kABytes;   // this stage's weight tile is at st + L::kA (kA = 0)
                const uint4 *codes = (const uint4 *)(smem + L::kCodes + sc * Cfg::kCodeBytes);
                constexpr int kQuads = Cfg::kCodeBytes / 16;   // four words = one row's half stage
#pragma unroll
                for (int i = 0; i < kQuads / (kTcProdWarps * 32); i++) {
                    const int qi = pid + kTcProdWarps * 32 * i;
                    const int mrow = qi >> 1, w0 = (qi & 1) * 4;  // row within gate|up (or down), first word
                    const uint4 c4 = codes[qi];
                    *(uint4 *)(st + L::kA + sw128(mrow, w0 + 0)) = expand_word(c4.x);
                    *(uint4 *)(st + L::kA + sw128(mrow, w0 + 1)) = expand_word(c4.y);
                    *(uint4 *)(st + L::kA + sw128(mrow, w0 + 2)) = expand_word(c4.z);
                    *(uint4 *)(st + L::kA + sw128(mrow, w0 + 3)) = expand_word(c4.w);
                }
                fence_async_smem();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(b_w_full + 8 * sw);
                    mbar_arrive(b_codes_empty + 8 * sc);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// The q_x row of every position (xpos[p] = q_x[perm[p] / K]), so that the gate/up
// GEMM loads 128 positions' rows with one 2-D copy; one warp per row.
__global__ void __launch_bounds__(256) gather_rows_kernel(const int8_t *qx, const int *perm, int S, int K, int D,
                                                          int8_t *xpos)
{
    const int lane = threadIdx.x & 31;
    const int64_t w0 = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5, nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t p = w0; p < S; p += nw) {
        const int t = __ldg(perm + p) / K;
        const uint4 *src = reinterpret_cast<const uint4 *>(qx + (size_t)t * D);
        uint4 *dst = reinterpret_cast<uint4 *>(xpos + (size_t)p * D);
        for (int c = lane; c < D / 16; c += 32) dst[c] = __ldg(src + c);
    }
}

// y[t][c] = (resid[t][c] +) sum_k fmaf(w[t][k], yE_k[c]) in rank order, with
// yE_k[c] = f32(acc) * (alpha_down[e_k][c] * s_h) rebuilt from the stored
// accumulator (acc = 2 * acc_hi + its bit in acc_lo); one thread per 4 channels
__global__ void combine_kernel(const int16_t *acc_hi, const uint32_t *acc_lo, const float *alpha_down, const float *sh,
                               const int *topk_idx, const int *inv, const float *topk_w, int T, int K, int D, float *y,
                               const float *resid)
{
    const int64_t n4 = (int64_t)T * D / 4;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n4; i += (int64_t)gridDim.x * blockDim.x) {
        const int t = (int)(i / (D / 4));
        const int c = 4 * (int)(i % (D / 4));
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int k = 0; k < K; k++) {
            const int sl = t * K + k, p = __ldg(inv + sl), e = __ldg(topk_idx + sl);
            const float w = __ldg(topk_w + sl), s = __ldg(sh + p);
            const uint2 hv = __ldcs(reinterpret_cast<const uint2 *>(acc_hi + (size_t)p * D + c));
            const uint32_t lo = __ldg(acc_lo + (size_t)p * (D / 32) + (c >> 5)) >> (c & 31);
            const float4 al = __ldg(reinterpret_cast<const float4 *>(alpha_down + (size_t)e * D + c));
            const int a0 = 2 * (int)(int16_t)(hv.x & 0xffffu) + (int)(lo & 1u);
            const int a1 = 2 * (int)(int16_t)(hv.x >> 16) + (int)((lo >> 1) & 1u);
            const int a2 = 2 * (int)(int16_t)(hv.y & 0xffffu) + (int)((lo >> 2) & 1u);
            const int a3 = 2 * (int)(int16_t)(hv.y >> 16) + (int)((lo >> 3) & 1u);
            acc.x = __fmaf_rn(w, __fmul_rn((float)a0, __fmul_rn(al.x, s)), acc.x);
            acc.y = __fmaf_rn(w, __fmul_rn((float)a1, __fmul_rn(al.y, s)), acc.y);
            acc.z = __fmaf_rn(w, __fmul_rn((float)a2, __fmul_rn(al.z, s)), acc.z);
            acc.w = __fmaf_rn(w, __fmul_rn((float)a3, __fmul_rn(al.w, s)), acc.w);
        }
        if (resid) {
            const float4 r = reinterpret_cast<const float4 *>(resid)[i];
            acc.x = __fadd_rn(r.x, acc.x);
            acc.y = __fadd_rn(r.y, acc.y);
            acc.z = __fadd_rn(r.z, acc.z);
            acc.w = __fadd_rn(r.w, acc.w);
        }
        reinterpret_cast<float4 *>(y)[i] = acc;
    }
}

// 2-bit interchange -> tensor-core layout (one thread per output word)
__global__ void repack_tc_gu_kernel(const uint32_t *gate, const uint32_t *up, int E, int D, int F, uint32_t *out)
{
    const int FT = F / 128, KS = D / 128;
    const int64_t n = (int64_t)E * FT * KS * 2 * 128 * 8;
    for (int64_t o = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; o < n; o += (int64_t)gridDim.x * blockDim.x) {
        int64_t q = o;
        const int w = q % 8; q /= 8;
        const int row = q % 128; q /= 128;
        const int mat = q % 2; q /= 2;
        const int ks = q % KS; q /= KS;
        const int ft = q % FT; q /= FT;
        const int e = (int)q;
        const uint32_t *src = (mat == 0 ? gate : up) + ((int64_t)e * F + ft * 128 + row) * (D / 16);
        out[o] = tc_word(src[ks * 8 + w]);
    }
}

__global__ void repack_tc_dn_kernel(const uint32_t *down, int E, int D, int F, uint32_t *out)
{
    const int CT = D / 128, KS = F / 128;
    const int64_t n = (int64_t)E * CT * KS * 128 * 8;
    for (int64_t o = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; o < n; o += (int64_t)gridDim.x * blockDim.x) {
        int64_t q = o;
        const int w = q % 8; q /= 8;
        const int row = q % 128; q /= 128;
        const int ks = q % KS; q /= KS;
        const int ct = q % CT; q /= CT;
        const int e = (int)q;
        const uint32_t *src = down + ((int64_t)e * D + ct * 128 + row) * (F / 16);
        out[o] = tc_word(src[ks * 8 + w]);
    }
}

}  // namespace maple
