// Expert stage for decode batches (T <= 64) on warp-level int8 MMA
// (mma.sync m16n8k32: A = 2-bit weight codes as unsigned byte planes,
// B = int8 activations, int32 accumulators), as two persistent streaming
// kernels, one CTA per SM, and a combine kernel:
//
//   decode_stage_kernel<1>  gate/up: h = SiLU(g) * u per (slot, output), fp32,
//                           and the per-slot |h| maxima (atomicMax);
//   decode_stage_kernel<2>  down: requantise h (int8 absmax per slot), the down
//                           contraction, yE;
//   dx_combine_kernel       y = resid + the rank-order combine of yE.
//
// Each is launched as a programmatic dependent of the kernel before it: its
// CTAs start as the previous kernel's CTAs retire (the down kernel streams its
// codes into shared memory at once) and wait for the previous grid
// (griddepcontrol.wait) before reading its outputs.  The grid boundaries are
// the only synchronisation between the phases; no CTA waits on another CTA of
// its own grid, so no grid-wide residency is assumed.
//
// Work.  The routing kernel has built the token -> expert permutation and
// cut every active expert's slots into units of at most 16 (two 8-token MMA
// n-tiles); every CTA loads those tables into shared memory.  Stage 1 has F/8
// items per unit (one 16-row tile: 8 gate rows and the up rows of the same 8
// outputs over all of K), stage 2 has F/16 items per unit (D/F consecutive
// 16-channel tiles); an item is 4*D bytes of codes followed by its row scales
// (layout.cuh).  CTA b takes the contiguous item range [N*b/G, N*(b+1)/G).
//
// Warp roles (11 warps):
//   warps 0-1  stream the range's items into a ring of shared-memory slots in
//              groups of kDxCopyItems consecutive items (one mbarrier pair per
//              group; warp p fills the groups g = p mod 2), one bulk copy per run
//              of items of one unit (consecutive in memory), as far ahead as the
//              ring allows.  Two issuing warps and large copies: one thread
//              issuing one copy per item does not keep HBM busy;
//   warp 2     builds each unit's B operand (the unit's activations in MMA
//              fragment order, 128-byte swizzled) in one of two buffers: stage 1
//              from the fragment-ordered copy of q_x by 16-byte loads; stage 2 (after
//              griddepcontrol.wait) from the unit's rows of h, brought in by one
//              bulk copy, requantised with the per-slot maxima, with each
//              slot's scale and code sum;
//   warps 3-10 compute: item j of the range goes to warp j % 8.  Per 128-column
//              block one 16-byte shared load gives the lane its four code words;
//              w & (0x03030303 << 2q) is the A fragment of the MMA over columns
//              32q.. of the block, scaled by 4^q, so four plane accumulators hold
//              exact multiples of 4^q and combine exactly; subtracting the row's
//              code sum gives the ternary dot product.  A warp hands its item back
//              as soon as its MMAs have read it.  Stage-1 epilogue: SwiGLU in the
//              lane (gate and up of one output sit in c0/c2 and c1/c3), h to global
//              memory, the slot maxima by shuffles and one atomicMax.  Stage-2
//              epilogue: yE to global memory.
// Every wait is bounded (the handle's limit) and raises the device flag on
// expiry; the CTA then drains its copies in flight and returns.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "layout.cuh"
#include "route.cuh"
#include "tc_gemm.cuh"

namespace maple {

// Twelve compute warps, claiming the CTA's items one at a time: each holds a
// ring slot only while its MMAs read it, so most of the ring's slots are
// always copies in flight, and three warps per scheduler hide the latency of
// the MMA chains and the SwiGLU epilogue.
constexpr int kDxComputeWarps = 12;
constexpr int kDxProducers = 2;                          // weight-stream warps
constexpr int kDxBuilder = kDxProducers;                 // the B-operand warp
constexpr int kDxCompute0 = kDxProducers + 1;            // first compute warp
constexpr int kDxThreads = (kDxCompute0 + kDxComputeWarps) * 32;   // 480
constexpr int kDxUnitTokens = kUnitTokens;               // tokens of a unit: two MMA n-tiles
constexpr int kDxNB = 2;                                 // B-operand buffers
constexpr int kDxMaxF = 1024;                            // largest d_ff (the shape limit)
// Items per ring group (one copy per run of an expert's items): few large copies
// stream faster than many small ones.
constexpr int kDxCopyItems = 4;

struct DxArgs {
    int T, D, E, K, F;
    const float *sx;       // [T] scale of q_x
    const int *sumx;       // [T] sum of q_x's codes
    const uint8_t *w_gu, *w_dn;   // MMA-tile layouts (codes and row scales per item)
    const int8_t *qxp;     // [T][D] q_x rows in fragment order (frag_word_pos)
    const int *perm;       // [T*K] position -> slot (the routing kernel's permutation)
    const int2 *units;     // the units: {expert, first position | count << 16}
    const int *n_units;
    float *h;              // [T*K][F] SwiGLU outputs, position order
    unsigned *amax;        // [T*K] |h| maxima (float bits), zero before stage 1
    const unsigned *never; // a word that stays 0 (the stall test hook waits for it to become 1)
    float *ye;             // [T*K][D] expert outputs, position order
    int *tap_acc_gate, *tap_acc_up, *tap_acc_down;
    int8_t *tap_qh;
    float *tap_sh;
    unsigned *flag;
    uint64_t wait_ns;
    int stall;             // test hook: stage 2 waits for `never` to become 1
    int nslot;             // ring slots (a multiple of kDxCopyItems * kDxProducers)
};

struct DxSide {                 // per-slot data of a unit, next to its B operand
    float s[kDxUnitTokens];     // stage 1: s_x of the token; stage 2: s_h of the slot
    int sum[kDxUnitTokens];     // sum of the row's int8 codes (q_x or q_h)
    int pos[kDxUnitTokens];     // position of the slot in the permutation
    int e, cnt;
};

// shared-memory layout of a decode kernel
struct DxSmem {
    int ring, bbuf, hst, side, bars, tables, total;
    int code_bytes, item_bytes, b_bytes, hst_bytes, ngroups;
    __host__ __device__ DxSmem(int stage, int D, int F, int T, int K, int E, int nslot)
    {
        code_bytes = 4 * D;
        item_bytes = stage == 1 ? (int)mma_gu_item_bytes(D) : (int)mma_dn_item_bytes(D, F);
        b_bytes = 2 * ((stage == 1 ? D : F) / 128) * 1024;            // two 8-token n-tiles
        hst_bytes = stage == 1 ? 0 : 2 * kDxUnitTokens * F * 4;      // two units' rows of h
        ngroups = nslot / kDxCopyItems;
        ring = 0;
        bbuf = (ring + nslot * item_bytes + 1023) & ~1023;
        hst = bbuf + kDxNB * b_bytes;
        side = hst + hst_bytes;
        bars = (side + kDxNB * (int)sizeof(DxSide) + 7) & ~7;
        const int n_bars = 2 * ngroups + 2 * kDxNB + 2;   // ring groups full/empty, B full/empty, h staged [2]
        // + abort word, item claim counter, copies into each h buffer; per ring group the
        // copies issued into it; per ring slot the items consumed from it
        tables = bars + 8 * n_bars + 16 + 4 * ngroups + 4 * nslot;
        const int S = T * K, units = E + (S + kDxUnitTokens - 1) / kDxUnitTokens + 1;
        // t_perm [S]; t_sx, t_sumx [T]; misc [2]; units [units] (int2, 8-byte aligned)
        int tb = S * 4 + 2 * T * 4 + 2 * 4;
        tb = (tb + 7) & ~7;
        total = tables + tb + units * 8;
    }
};

// Ring slots of a decode kernel within a shared-memory budget (0: it does not
// fit): a multiple of kDxCopyItems * kDxProducers, so that every ring group
// belongs to one producer warp.  Item j of a CTA's range goes to slot
// j % nslot, round j / nslot; the warp that claims it first waits until item
// j - nslot has been consumed (a per-slot count), so that when it tests the
// group's full barrier the barrier is in round j / nslot or later.  (A parity
// wait accepts the current phase and the one before it: without that count a
// warp could take the previous round's phase as complete.)  Otherwise the warp of item j + nslot could
// test the slot group's full barrier while item j's copy is still landing, see
// the barrier in the phase before and take it as complete (a parity wait
// accepts the current phase and the one before it).
__host__ inline int dx_ring_slots(int stage, int D, int F, int T, int K, int E, size_t budget)
{
    if (F > D || D % F) return 0;
    constexpr int step = kDxCopyItems * kDxProducers;
    for (int n = 32; n >= 2 * step; n -= step)
        if ((size_t)DxSmem(stage, D, F, T, K, E, n).total <= budget) return n;
    return 0;
}

__device__ __forceinline__ void mma_u8s8(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1)
{
    asm volatile("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%0,%1,%2,%3};"
                 : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint4 lds128(uint32_t addr)
{
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}

// One 16-row tile over nkb 128-column blocks against NT n-tiles of 8 tokens:
// acc[nt][q][i] is plane q of C-fragment register i (a multiple of 4^q).
// b_lo / b_hi: this lane's two 16-byte B chunks in the first block (the B
// operand is 128-byte swizzled, see dx_b_chunk).
template <int NT>
__device__ __forceinline__ void dx_tile(uint32_t a_addr, uint32_t b_lo, uint32_t b_hi, int nkb, int b_nt_stride,
                                        int (&acc)[2][4][4])
{
#pragma unroll
    for (int nt = 0; nt < 2; nt++)
#pragma unroll
        for (int q = 0; q < 4; q++)
#pragma unroll
            for (int i = 0; i < 4; i++) acc[nt][q][i] = 0;
#pragma unroll 2
    for (int kb = 0; kb < nkb; kb++) {
        const uint4 w = lds128(a_addr + kb * 512);
#pragma unroll
        for (int nt = 0; nt < NT; nt++) {
            const uint4 b0 = lds128(b_lo + nt * b_nt_stride + kb * 1024);
            const uint4 b1 = lds128(b_hi + nt * b_nt_stride + kb * 1024);
            const uint32_t bq[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int q = 0; q < 4; q++) {
                const uint32_t m = 0x03030303u << (2 * q);
                mma_u8s8(acc[nt][q], w.x & m, w.y & m, w.z & m, w.w & m, bq[2 * q], bq[2 * q + 1]);
            }
        }
    }
}

// B operand layout: per n-tile and 128-column block 1 KB, token g's 128 bytes
// (fragment order, frag_word_pos) in row g, its 16-byte chunk c stored at
// chunk c ^ g (the TMA's 128-byte swizzle).  Lane 4g + c2 reads chunks 2c2 and
// 2c2 + 1 of token g, which lands the eight lanes of every quarter warp on
// distinct banks.  Byte offset of chunk c of token g within a block:
__device__ __forceinline__ uint32_t dx_b_chunk(int g, int c) { return (uint32_t)(g * 128 + ((c ^ g) << 4)); }

// Four 16-row tiles (a_addr + d * tile_stride) against one n-tile at once: the
// four tiles' accumulator chains interleave, instead of four short chains one
// after another.  acc[d][q][i] as in dx_tile.
__device__ __forceinline__ void dx_tile4(uint32_t a_addr, int tile_stride, uint32_t b_lo, uint32_t b_hi, int nkb,
                                         int (&acc)[4][4][4])
{
#pragma unroll
    for (int d = 0; d < 4; d++)
#pragma unroll
        for (int q = 0; q < 4; q++)
#pragma unroll
            for (int i = 0; i < 4; i++) acc[d][q][i] = 0;
#pragma unroll 1
    for (int kb = 0; kb < nkb; kb++) {
        const uint4 b0 = lds128(b_lo + kb * 1024);
        const uint4 b1 = lds128(b_hi + kb * 1024);
        const uint32_t bq[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
        for (int d = 0; d < 4; d++) {
            const uint4 w = lds128(a_addr + d * tile_stride + kb * 512);
#pragma unroll
            for (int q = 0; q < 4; q++) {
                const uint32_t m = 0x03030303u << (2 * q);
                mma_u8s8(acc[d][q], w.x & m, w.y & m, w.z & m, w.w & m, bq[2 * q], bq[2 * q + 1]);
            }
        }
    }
}

// the exact row total of register i: acc_0 + acc_1/4 + acc_2/16 + acc_3/64
__device__ __forceinline__ int dx_total(const int (&acc)[2][4][4], int nt, int i)
{
    return acc[nt][0][i] + (acc[nt][1][i] >> 2) + (acc[nt][2][i] >> 4) + (acc[nt][3][i] >> 6);
}

template <int STAGE>
__global__ void __launch_bounds__(kDxThreads, 1)
    decode_stage_kernel(DxArgs a)
{
    extern __shared__ __align__(1024) uint8_t dsm[];
    const DxSmem L(STAGE, a.D, a.F, a.T, a.K, a.E, a.nslot);
    const int D = a.D, F = a.F, T = a.T, K = a.K, S = T * K;
    const int KB1 = D / 128, KB2 = F / 128;
    const int S2 = D / F;                                     // down tiles per stage-2 item
    const int GS = STAGE == 1 ? mma_gu_items(F) : mma_dn_items(F);   // items per unit (= per expert)
    const uint8_t *wsrc = STAGE == 1 ? a.w_gu : a.w_dn;

    uint8_t *ring = dsm + L.ring;
    uint8_t *bbuf = dsm + L.bbuf;
    uint8_t *hst = dsm + L.hst;
    DxSide *side = (DxSide *)(dsm + L.side);
    uint64_t *bars = (uint64_t *)(dsm + L.bars);
    const uint32_t b_rfull = smem_addr(bars), b_rempty = b_rfull + 8 * L.ngroups;
    const uint32_t b_bfull = b_rempty + 8 * L.ngroups, b_bempty = b_bfull + 8 * kDxNB;
    const uint32_t b_hst = b_bempty + 8 * kDxNB;   // [2]: the two h staging buffers
    volatile uint32_t *abort = (volatile uint32_t *)(bars + 2 * L.ngroups + 2 * kDxNB + 2);
    int *s_claim = (int *)(abort + 1);                    // the CTA's next unclaimed item (relative)
    volatile int *s_hgen = (volatile int *)(abort + 2);   // stage 2: [2] copies issued into each h buffer
    volatile int *s_gen = (volatile int *)(abort + 4);    // [ngroups] copies issued into each ring group
    volatile int *s_done = s_gen + L.ngroups;             // [nslot] items consumed from each ring slot
    // routing tables (loaded from the routing kernel's outputs)
    int *t_perm = (int *)(dsm + L.tables);
    float *t_sx = (float *)(t_perm + S);
    int *t_sumx = (int *)(t_sx + T);
    int *t_misc = t_sumx + T;   // [1] n_units
    int2 *t_unit = (int2 *)(((uintptr_t)(t_misc + 2) + 7) & ~(uintptr_t)7);   // {expert, first | count << 16}

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int g = 0; g < L.ngroups; g++) {
            mbar_init(b_rfull + 8 * g, 1);
            mbar_init(b_rempty + 8 * g, kDxCopyItems);
        }
        for (int b = 0; b < kDxNB; b++) {
            mbar_init(b_bfull + 8 * b, 1);
            mbar_init(b_bempty + 8 * b, kDxComputeWarps);
        }
        mbar_init(b_hst, 1);
        mbar_init(b_hst + 8, 1);
        *abort = 0u;
        *s_claim = 0;
        s_hgen[0] = s_hgen[1] = 0;
        for (int g = 0; g < L.ngroups; g++) s_gen[g] = 0;
        for (int q = 0; q < a.nslot; q++) s_done[q] = 0;
        fence_barrier_init();
    }
    if (STAGE == 1) {
        // Launched as a programmatic dependent of the routing kernel: nothing it
        // wrote is read before this wait.  Only after it may the down kernel
        // launch, so that when a down CTA runs the routing outputs are complete.
        asm volatile("griddepcontrol.wait;" ::: "memory");
    }
    // the next kernel may launch; it waits for this grid before it reads
    // anything this grid writes
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    // ---------------- prologue: the routing tables, one round of loads
    // (stage 2 reads only the routing outputs here; h and the maxima of the
    // gate/up kernel are read after its own wait, by the B-operand warp)
    const int n_units_g = __ldcg(a.n_units);
    const int unit_cap = a.E + (S + kDxUnitTokens - 1) / kDxUnitTokens + 1;   // the units array's length
    for (int q = threadIdx.x; q < S; q += blockDim.x) t_perm[q] = __ldcg(a.perm + q);
    if (STAGE == 1)
        for (int t = threadIdx.x; t < T; t += blockDim.x) {
            t_sx[t] = __ldcg(a.sx + t);
            t_sumx[t] = __ldcg(a.sumx + t);
        }
    for (int u = threadIdx.x; u < unit_cap; u += blockDim.x) t_unit[u] = __ldcg(a.units + u);   // not waiting for n_units
    if (threadIdx.x == 0) t_misc[1] = n_units_g;
    __syncthreads();
    const int n_units = t_misc[1];
    // this CTA's item range and the units it touches (unit ordinals 0 .. n_uo-1)
    const int N = n_units * GS;
    const int j0 = (int)((int64_t)N * blockIdx.x / gridDim.x), j1 = (int)((int64_t)N * (blockIdx.x + 1) / gridDim.x);
    const int u_first = j0 / GS, n_uo = j1 > j0 ? (j1 - 1) / GS - u_first + 1 : 0;

    if (warp < kDxProducers) {
        // ---------------- weight stream: group gi of the range (items j0 + M*gi ..) goes to
        // ring group gi mod ngroups; this warp takes the groups gi = warp mod kDxProducers
        bool ok = true;
        const int n_grp = (j1 - j0 + kDxCopyItems - 1) / kDxCopyItems;
        for (int gi = warp; gi < n_grp && ok; gi += kDxProducers) {
            const int sg = gi % L.ngroups;
            if (lane == 0) {
                if (!mbar_wait(b_rempty + 8 * sg, ((gi / L.ngroups) & 1) ^ 1, abort, a.flag, a.wait_ns)) {
                    ok = false;
                } else {
                    const int ja = j0 + kDxCopyItems * gi, jb = min(j1, ja + kDxCopyItems);
                    const uint32_t full = b_rfull + 8 * sg;
                    mbar_expect_tx(full, (uint32_t)((jb - ja) * L.item_bytes));
                    uint32_t dst = smem_addr(ring + (size_t)sg * kDxCopyItems * L.item_bytes);
                    for (int j = ja; j < jb;) {
                        // a run of items of one unit: consecutive in memory
                        const int u = j / GS, it = j - u * GS, e = t_unit[u].x;
                        const int n = min(jb - j, GS - it);
                        bulk_g2s(dst, wsrc + ((size_t)e * GS + it) * L.item_bytes, (uint32_t)(n * L.item_bytes), full);
                        dst += n * L.item_bytes;
                        j += n;
                    }
                    s_gen[sg] = gi / L.ngroups + 1;
                }
            }
            ok = __shfl_sync(FULL, ok, 0);
        }
    } else if (warp == kDxBuilder) {
        // ---------------- B operands, one per unit of the range
        bool ok = true;
        if (STAGE == 2) {
            // h and the maxima come from the gate/up kernel: wait for its grid
            asm volatile("griddepcontrol.wait;" ::: "memory");
            if (a.stall && lane == 0) {
                // test hook: wait for a word nothing sets, so that the bounded wait expires
                const uint64_t t0 = global_ns();
                while (true) {
                    unsigned v;
                    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(a.never) : "memory");
                    if (v == 1u) break;
                    __nanosleep(256);
                    if (*abort || global_ns() - t0 > a.wait_ns) {
                        *abort = 1u;
                        set_flag(a.flag, MAPLE_DEVFLAG_TIMEOUT);
                        ok = false;
                        break;
                    }
                }
            }
            ok = __shfl_sync(FULL, ok, 0);
        }
        for (int uo = 0; uo < n_uo && ok; uo++) {
            const int b = uo % kDxNB;
            if (uo >= kDxNB && !mbar_wait(b_bempty + 8 * b, ((uo / kDxNB) & 1) ^ 1, abort, a.flag, a.wait_ns)) break;
            const int2 un = t_unit[u_first + uo];
            const int e = un.x, p0 = un.y & 0xffff, cnt = un.y >> 16;
            DxSide *sd = side + b;
            uint8_t *bb = bbuf + (size_t)b * L.b_bytes;
            const int ntiles = (cnt + 7) / 8;
            if (STAGE == 1) {
                if (lane < kDxUnitTokens) {
                    const int n = min(lane, cnt - 1);
                    const int slot = t_perm[p0 + n], t = slot / K;
                    sd->s[lane] = t_sx[t];
                    sd->sum[lane] = t_sumx[t];
                    sd->pos[lane] = p0 + n;
                }
                if (lane == 0) {
                    sd->e = e;
                    sd->cnt = cnt;
                }
                // the unit's q_x rows (fragment order) by 16-byte asynchronous copies,
                // all in flight at once, into the B operand's swizzled positions
                // (dx_b_chunk); the padding tokens of the last n-tile are left as they
                // are (their outputs are never read)
                const int cpr = D / 16;   // 16-byte chunks per row
                for (int idx = lane; idx < cnt * cpr; idx += 32) {
                    const int n = idx / cpr, cc = idx - n * cpr;
                    const int t = t_perm[p0 + n] / K;
                    const uint32_t dst = smem_addr(bb + (n >> 3) * KB1 * 1024 + (cc >> 3) * 1024 + dx_b_chunk(n & 7, cc & 7));
                    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst),
                                 "l"(reinterpret_cast<const uint4 *>(a.qxp + (size_t)t * D) + cc)
                                 : "memory");
                }
                asm volatile("cp.async.commit_group;" ::: "memory");
                asm volatile("cp.async.wait_group 0;" ::: "memory");
                __threadfence_block();
                __syncwarp();
                if (lane == 0) mbar_arrive(b_bfull + 8 * b);
                continue;
            }
            // stage 2: the unit's rows of h (consecutive positions) came in one copy
            // (issued one unit ahead, into the other of two staging buffers), the
            // per-slot maxima by the lanes; requantise (int8 absmax per slot) into
            // fragment order, with each slot's scale and code sum (every CTA that
            // holds items of the unit does this; their q_h / s_h taps agree bitwise)
            auto stage_h = [&](int un_o) {   // copy unit un_o's rows of h into buffer un_o & 1
                const int2 uu = t_unit[u_first + un_o];
                const int q0 = uu.y & 0xffff, qc = uu.y >> 16, hb = un_o & 1;
                fence_async_smem();   // earlier reads of the buffer come first
                __syncwarp();
                if (lane == 0) {
                    mbar_expect_tx(b_hst + 8 * hb, (uint32_t)(qc * F * 4));
                    bulk_g2s(smem_addr(hst + (size_t)hb * (L.hst_bytes / 2)), a.h + (size_t)q0 * F, (uint32_t)(qc * F * 4),
                             b_hst + 8 * hb);
                    s_hgen[hb] = s_hgen[hb] + 1;
                }
            };
            if (uo == 0) stage_h(0);
            const float am_lane = lane < cnt ? __uint_as_float(__ldcg(a.amax + p0 + lane)) : 0.0f;
            if (!__all_sync(FULL, mbar_wait(b_hst + 8 * (uo & 1), (uo >> 1) & 1, abort, a.flag, a.wait_ns))) break;
            if (uo + 1 < n_uo) stage_h(uo + 1);
            const uint8_t *hsrc = hst + (size_t)(uo & 1) * (L.hst_bytes / 2);
            for (int n = 0; n < cnt; n++) {   // (padding tokens: left as they are, never read)
                const int nt = n >> 3, g = n & 7;
                uint8_t *dst = bb + nt * KB2 * 1024;   // token g's row: 128 bytes at g * 128 of each block
                const int pos = p0 + n, slot = t_perm[pos];
                const float4 *hr = reinterpret_cast<const float4 *>(hsrc + (size_t)n * F * 4);
                const float amax = __shfl_sync(FULL, am_lane, n);
                const float inv = amax > 0.0f ? __fdiv_rn(127.0f, amax) : 0.0f;
                int sum = 0;
#pragma unroll
                for (int i = 0; i < kDxMaxF / 128; i++) {
                    if (i >= F / 128) break;
                    const int w = lane + 32 * i;   // word w: columns 4w .. 4w+3
                    const float4 hv = hr[w];
                    int q0 = 0, q1 = 0, q2 = 0, q3 = 0;
                    if (amax > 0.0f) {
                        q0 = quant_code(hv.x, inv);
                        q1 = quant_code(hv.y, inv);
                        q2 = quant_code(hv.z, inv);
                        q3 = quant_code(hv.w, inv);
                    }
                    sum += q0 + q1 + q2 + q3;
                    const uint32_t pk = (uint32_t)(q0 & 0xff) | ((uint32_t)(q1 & 0xff) << 8) |
                                        ((uint32_t)(q2 & 0xff) << 16) | ((uint32_t)(q3 & 0xff) << 24);
                    const int fp = frag_word_pos(w & 31);   // word of token g's row, swizzled by chunk
                    reinterpret_cast<uint32_t *>(dst + (w >> 5) * 1024 + dx_b_chunk(g, fp >> 2))[fp & 3] = pk;
                    if (a.tap_qh) reinterpret_cast<uint32_t *>(a.tap_qh + (size_t)slot * F)[w] = pk;
                }
                sum = warp_sum_int(sum);
                if (lane == 0) {
                    const float sv = amax > 0.0f ? __fdiv_rn(amax, 127.0f) : 0.0f;
                    sd->s[n] = sv;
                    sd->sum[n] = sum;
                    sd->pos[n] = pos;
                    if (a.tap_sh) a.tap_sh[slot] = sv;
                }
            }
            if (lane == 0) {
                sd->e = e;
                sd->cnt = cnt;
            }
            __threadfence_block();
            __syncwarp();
            if (lane == 0) mbar_arrive(b_bfull + 8 * b);
        }
    } else {
        // ---------------- compute warps: claim the range's items one at a time (in
        // order), visiting every unit's B operand in turn
        const int g = lane >> 2, tig = lane & 3;
        bool ok = true;
        auto claim = [&]() {
            int c = 0;
            if (lane == 0) c = atomicAdd(s_claim, 1);
            return j0 + __shfl_sync(FULL, c, 0);
        };
        int j = claim();
        for (int uo = 0; uo < n_uo && ok; uo++) {
            const int b = uo % kDxNB;
            if (!mbar_wait(b_bfull + 8 * b, (uo / kDxNB) & 1, abort, a.flag, a.wait_ns)) break;
            const DxSide *sd = side + b;
            const int u = u_first + uo, cnt = sd->cnt;
            const int ntiles = (cnt + 7) / 8;
            const uint32_t bbase = smem_addr(bbuf + (size_t)b * L.b_bytes);
            const uint32_t bb_lo = bbase + dx_b_chunk(g, 2 * tig), bb_hi = bbase + dx_b_chunk(g, 2 * tig + 1);
            const int jb = min(j1, (u + 1) * GS);   // this unit's items end here
            for (; j < jb; j = claim()) {
                const int rel = j - j0, slot = rel % a.nslot, sg = slot / kDxCopyItems, round = rel / a.nslot;
                // item j - nslot consumed first: the group's barrier is then in this round or later
                if (lane == 0) {
                    const uint64_t t0 = global_ns();
                    while (s_done[slot] < round) {
                        if (*abort || global_ns() - t0 > a.wait_ns) {
                            *abort = 1u;
                            set_flag(a.flag, MAPLE_DEVFLAG_TIMEOUT);
                            break;
                        }
                    }
                }
                __syncwarp();
                if (!mbar_wait(b_rfull + 8 * sg, round & 1, abort, a.flag, a.wait_ns)) {
                    ok = false;
                    break;
                }
                const uint8_t *slot_p = ring + (size_t)slot * L.item_bytes;
                const float *alpha_s = reinterpret_cast<const float *>(slot_p + L.code_bytes);   // the item's scales
                const uint32_t aa = smem_addr(slot_p) + lane * 16;
                const int it = j - u * GS;
                int acc[2][4][4];
                if (STAGE == 1) {
                    // ---- gate/up tile `it`: outputs 8it .. 8it+7 (this lane: output 8it + g)
                    const int o = 8 * it + g;
                    const float ag = alpha_s[g], au = alpha_s[8 + g];
                    if (ntiles == 2)
                        dx_tile<2>(aa, bb_lo, bb_hi, KB1, KB1 * 1024, acc);
                    else
                        dx_tile<1>(aa, bb_lo, bb_hi, KB1, KB1 * 1024, acc);
                    // the codes and scales have been read: hand the item back to the weight stream
                    __syncwarp();
                    if (lane == 0) {
                        mbar_arrive(b_rempty + 8 * sg);
                        s_done[slot] = round + 1;
                    }
#pragma unroll
                    for (int nt = 0; nt < 2; nt++) {
                        if (nt >= ntiles) break;
                        // both tokens' SwiGLU chains with no branch between them (a padding
                        // token's side data repeat the unit's last token: finite, never stored)
                        float hv[2];
#pragma unroll
                        for (int h2 = 0; h2 < 2; h2++) {
                            const int n = 8 * nt + 2 * tig + h2;
                            const int gd = dx_total(acc, nt, h2) - sd->sum[n];
                            const int ud = dx_total(acc, nt, 2 + h2) - sd->sum[n];
                            hv[h2] = swiglu(__fmul_rn((float)gd, __fmul_rn(ag, sd->s[n])),
                                            __fmul_rn((float)ud, __fmul_rn(au, sd->s[n])));
                        }
                        float hm[2];
#pragma unroll
                        for (int h2 = 0; h2 < 2; h2++) {
                            const int n = 8 * nt + 2 * tig + h2;
                            hm[h2] = 0.0f;
                            if (n < cnt) {
                                const int pos = sd->pos[n];
                                a.h[(size_t)pos * F + o] = hv[h2];
                                hm[h2] = fabsf(hv[h2]);
                                if (a.tap_acc_gate || a.tap_acc_up) {
                                    const int slot_t = t_perm[pos];
                                    if (a.tap_acc_gate) a.tap_acc_gate[(size_t)slot_t * F + o] = dx_total(acc, nt, h2) - sd->sum[n];
                                    if (a.tap_acc_up) a.tap_acc_up[(size_t)slot_t * F + o] = dx_total(acc, nt, 2 + h2) - sd->sum[n];
                                }
                            }
                        }
                        // maxima over the tile's 8 outputs (lanes of equal tig), then over the unit
#pragma unroll
                        for (int o2 = 4; o2 <= 16; o2 <<= 1) {
                            hm[0] = fmaxf(hm[0], __shfl_xor_sync(FULL, hm[0], o2));
                            hm[1] = fmaxf(hm[1], __shfl_xor_sync(FULL, hm[1], o2));
                        }
                        if (g == 0) {
#pragma unroll
                            for (int h2 = 0; h2 < 2; h2++) {
                                const int n = 8 * nt + 2 * tig + h2;
                                if (n < cnt) atomicMax(a.amax + sd->pos[n], __float_as_uint(hm[h2]));
                            }
                        }
                    }
                } else {
                    // ---- down item `it`: tiles S2*it .. S2*it + S2-1, channels 16*S2*it ..
                    if (S2 == 4 && ntiles == 1) {
                        // the common decode shape (d_ff = d_model / 4, at most 8 tokens):
                        // the four tiles' chains together
                        int acc4[4][4][4];
                        dx_tile4(aa, KB2 * 512, bb_lo, bb_hi, KB2, acc4);
                        float ad[4][2];   // this lane's channel scales, read before the slot is handed back
#pragma unroll
                        for (int d = 0; d < 4; d++) {
                            ad[d][0] = alpha_s[16 * d + g];
                            ad[d][1] = alpha_s[16 * d + 8 + g];
                        }
                        __syncwarp();
                        if (lane == 0) {   // the item's codes and scales are read: hand it back
                            mbar_arrive(b_rempty + 8 * sg);
                            s_done[slot] = round + 1;
                        }
#pragma unroll
                        for (int d = 0; d < 4; d++) {
                            const int ch0 = 16 * (4 * it + d) + g;
                            const float ad0 = ad[d][0], ad1 = ad[d][1];
#pragma unroll
                            for (int h2 = 0; h2 < 2; h2++) {
                                const int n = 2 * tig + h2;
                                if (n < cnt) {
                                    const int pos = sd->pos[n];
                                    const int d0 = acc4[d][0][h2] + (acc4[d][1][h2] >> 2) + (acc4[d][2][h2] >> 4) +
                                                   (acc4[d][3][h2] >> 6) - sd->sum[n];
                                    const int d1 = acc4[d][0][2 + h2] + (acc4[d][1][2 + h2] >> 2) +
                                                   (acc4[d][2][2 + h2] >> 4) + (acc4[d][3][2 + h2] >> 6) - sd->sum[n];
                                    a.ye[(size_t)pos * D + ch0] = __fmul_rn((float)d0, __fmul_rn(ad0, sd->s[n]));
                                    a.ye[(size_t)pos * D + ch0 + 8] = __fmul_rn((float)d1, __fmul_rn(ad1, sd->s[n]));
                                    if (a.tap_acc_down) {
                                        const int slot_t = t_perm[pos];
                                        a.tap_acc_down[(size_t)slot_t * D + ch0] = d0;
                                        a.tap_acc_down[(size_t)slot_t * D + ch0 + 8] = d1;
                                    }
                                }
                            }
                        }
                        continue;
                    }
                    for (int d = 0; d < S2; d++) {
                        const int dt = S2 * it + d;
                        if (ntiles == 2)
                            dx_tile<2>(aa + d * KB2 * 512, bb_lo, bb_hi, KB2, KB2 * 1024, acc);
                        else
                            dx_tile<1>(aa + d * KB2 * 512, bb_lo, bb_hi, KB2, KB2 * 1024, acc);
                        const int ch0 = 16 * dt + g;
                        const float ad0 = alpha_s[16 * d + g], ad1 = alpha_s[16 * d + 8 + g];
                        if (d == S2 - 1) {   // the item's codes and scales are read: hand it back
                            __syncwarp();
                            if (lane == 0) {
                                mbar_arrive(b_rempty + 8 * sg);
                                s_done[slot] = round + 1;
                            }
                        }
#pragma unroll
                        for (int nt = 0; nt < 2; nt++) {
                            if (nt >= ntiles) break;
#pragma unroll
                            for (int h2 = 0; h2 < 2; h2++) {
                                const int n = 8 * nt + 2 * tig + h2;
                                if (n < cnt) {
                                    const int pos = sd->pos[n];
                                    const int d0 = dx_total(acc, nt, h2) - sd->sum[n];
                                    const int d1 = dx_total(acc, nt, 2 + h2) - sd->sum[n];
                                    a.ye[(size_t)pos * D + ch0] = __fmul_rn((float)d0, __fmul_rn(ad0, sd->s[n]));
                                    a.ye[(size_t)pos * D + ch0 + 8] = __fmul_rn((float)d1, __fmul_rn(ad1, sd->s[n]));
                                    if (a.tap_acc_down) {
                                        const int slot_t = t_perm[pos];
                                        a.tap_acc_down[(size_t)slot_t * D + ch0] = d0;
                                        a.tap_acc_down[(size_t)slot_t * D + ch0 + 8] = d1;
                                    }
                                }
                            }
                        }
                    }
                }
            }
            if (!ok) break;
            __syncwarp();
            if (lane == 0) mbar_arrive(b_bempty + 8 * b);
        }
    }

    // ---------------- common exit: no copy may still be landing when the CTA exits.
    // After a normal run every copy has been waited for; after a failed wait the
    // last copy into every ring group and into each h staging buffer is waited
    // for (bounded).
    __syncthreads();
    if (threadIdx.x == 0 && *abort) {
        for (int g = 0; g < L.ngroups; g++) {
            const int gen = s_gen[g];   // copies issued into group g; the last one has phase gen - 1
            if (!gen) continue;
            const uint64_t t0 = global_ns();
            while (!mbar_test(b_rfull + 8 * g, (gen - 1) & 1) && global_ns() - t0 < a.wait_ns) {
            }
        }
        for (int hb = 0; STAGE == 2 && hb < 2; hb++) {
            const int gen = s_hgen[hb];   // copies issued into h buffer hb; the last one has phase gen - 1
            if (!gen) continue;
            const uint64_t t0 = global_ns();
            while (!mbar_test(b_hst + 8 * hb, (gen - 1) & 1) && global_ns() - t0 < a.wait_ns) {
            }
        }
    }
}

// y[t] = resid[t] + sum over ranks k of topk_w[t][k] * yE[inv[t*K + k]]: fmaf
// from 0 in rank order, then the residual added; one thread per 4 channels.
// A programmatic dependent of the down kernel (and itself the primary of the
// next layer's routing kernel).
__global__ void __launch_bounds__(256) dx_combine_kernel(const float *ye, const int *inv, const float *topk_w, int T,
                                                         int K, int D, float *y, const float *resid)
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int d4 = D / 4;
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < T * d4; i += gridDim.x * blockDim.x) {
        const int t = i / d4, c = 4 * (i - t * d4);
        float4 yv = make_float4(0.f, 0.f, 0.f, 0.f);
        // eight ranks at a time: their positions and weights, then their yE rows, all
        // loads in flight together; the sum still runs in rank order
        for (int k0 = 0; k0 < K; k0 += 8) {
            int pk[8];
            float wk[8];
            float4 ev[8];
#pragma unroll
            for (int j = 0; j < 8; j++)
                if (k0 + j < K) {
                    pk[j] = __ldcg(inv + t * K + k0 + j);
                    wk[j] = __ldcg(topk_w + t * K + k0 + j);
                }
#pragma unroll
            for (int j = 0; j < 8; j++)
                if (k0 + j < K) ev[j] = __ldcg(reinterpret_cast<const float4 *>(ye + (size_t)pk[j] * D + c));
#pragma unroll
            for (int j = 0; j < 8; j++)
                if (k0 + j < K) {
                    yv.x = __fmaf_rn(wk[j], ev[j].x, yv.x);
                    yv.y = __fmaf_rn(wk[j], ev[j].y, yv.y);
                    yv.z = __fmaf_rn(wk[j], ev[j].z, yv.z);
                    yv.w = __fmaf_rn(wk[j], ev[j].w, yv.w);
                }
        }
        const size_t o = (size_t)t * D + c;
        if (resid) {
            const float4 rv = *reinterpret_cast<const float4 *>(resid + o);
            yv.x = __fadd_rn(rv.x, yv.x);
            yv.y = __fadd_rn(rv.y, yv.y);
            yv.z = __fadd_rn(rv.z, yv.z);
            yv.w = __fadd_rn(rv.w, yv.w);
        }
        *reinterpret_cast<float4 *>(y + o) = yv;
    }
}


// ---------------------------------------------------------------------------
// Small decode batches (T <= 8): the whole expert stage in one kernel.
// At T <= 8 an expert holds at most 8 slots, so every active expert is one
// unit and one 8-token MMA n-tile.  One thread-block cluster of C CTAs per
// unit; CTA r of the cluster takes the r-th slice of the expert's gate/up
// outputs (F/C of them: F/8/C items) and of its down channels (D/C: F/16/C
// items), so the expert's weights are in flight at once across C SMs and each
// slice fits its CTA's shared memory (no slot is reused):
//   1. each warp issues the bulk copies of its items (gate/up and down) at
//      once; the unit's q_x rows come in as the gate/up B operand;
//   2. gate/up items -> SwiGLU -> the slice of h in shared memory; each
//      token's |h| maximum over the slice goes to every CTA of the cluster
//      (distributed shared memory); cluster barrier;
//   3. the maxima of all slices give each slot's s_h; every CTA requantises
//      its slice and writes the codes into every CTA's down B operand (in
//      fragment order), with the slice's code sums; cluster barrier;
//   4. down items -> yE (position order) for the CTA's channels;
//   5. combine: per (token, channel slice) a count of the token's K slots
//      done; the CTA that completes it adds the K slots' yE in rank order
//      (fmaf from 0, then the residual) into y, and sets the count back to 0.
// The arithmetic of every value is that of the two-kernel path (the same
// MMA planes, the same fp32 operations in the same order), so both give the
// same bits.  Grid: (units at most) x C CTAs, launched as a programmatic
// dependent of the routing kernel; clusters past the routing's unit count
// return at once.  Every wait is bounded; after a failed wait the CTA still
// takes the cluster barriers (doing no work), drains its copies and returns.
// ---------------------------------------------------------------------------
constexpr int kDfWarps = 16;
constexpr int kDfThreads = kDfWarps * 32;

struct DfArgs {
    int T, D, E, K, F;
    const float *sx;
    const int *sumx;
    const int8_t *qxp;        // [T][D] q_x rows in fragment order
    const int *perm, *inv;    // position -> slot, slot -> position
    const float *topk_w;      // [T][K]
    const int4 *funits;       // {expert, first position | count << 16, tokens 0-3, tokens 4-7 (bytes)}
    const int *n_units;
    const uint8_t *w_gu, *w_dn;
    float *ye;                // [T*K][D] position order
    unsigned *ctr;            // [T][C] slots done per (token, channel slice), zero between launches
    float *y;
    const float *resid;       // optional
    int *tap_acc_gate, *tap_acc_up, *tap_acc_down;
    int8_t *tap_qh;
    float *tap_sh;
    unsigned *flag;
    const unsigned *never;
    uint64_t wait_ns;
    int stall;                // test hook: the down phase waits for `never` to become 1
};

// shared-memory layout of dx_fused_kernel for a cluster of C CTAs
struct DfSmem {
    int ig, id, gu_bytes, dn_bytes, items, b1, b2, hl, amax, sums, side, comb, bars, total;
    __host__ __device__ DfSmem(int D, int F, int C)
    {
        ig = mma_gu_items(F) / C;
        id = mma_dn_items(F) / C;
        gu_bytes = (int)mma_gu_item_bytes(D);
        dn_bytes = (int)mma_dn_item_bytes(D, F);
        items = 0;                                                   // ig gate/up items, then id down items
        b1 = (items + ig * gu_bytes + id * dn_bytes + 1023) & ~1023;  // q_x B operand: D/128 blocks of 1 KB
        b2 = b1 + (D / 128) * 1024;                                  // q_h B operand: F/128 blocks
        hl = b2 + (F / 128) * 1024;                                  // [8][F/C] h of the slice
        amax = hl + 8 * (F / C) * 4;                                 // [C][8] slice maxima (float)
        sums = amax + C * 8 * 4;                                     // [C][8] slice code sums
        side = sums + C * 8 * 4;                                     // per token: pos, slot, tok, s_x, sum_x, s_h, sum_h, last
        comb = side + 8 * 8 * 4;                                     // per token and rank: combine weight, yE position [8][8] each
        bars = (comb + 2 * 64 * 4 + 7) & ~7;                         // [ig + id] copy barriers, then the abort word
        total = bars + 8 * (ig + id) + 16;
    }
};

__global__ void __launch_bounds__(kDfThreads, 1) dx_fused_kernel(DfArgs a)
{
    namespace cg = cooperative_groups;
    extern __shared__ __align__(1024) uint8_t dsm[];
    cg::cluster_group cluster = cg::this_cluster();
    const int C = (int)cluster.num_blocks(), r = (int)cluster.block_rank();
    const int c = blockIdx.x / C;
    const int D = a.D, F = a.F, K = a.K;
    const DfSmem L(D, F, C);
    const int KB1 = D / 128, KB2 = F / 128, S2 = D / F;
    const int IG = L.ig, NI = L.ig + L.id, FS = F / C, DS = D / C;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, tig = lane & 3;
    uint8_t *b1 = dsm + L.b1;
    uint8_t *b2 = dsm + L.b2;
    float *hl = (float *)(dsm + L.hl);
    float *s_amax = (float *)(dsm + L.amax);
    int *s_sums = (int *)(dsm + L.sums);
    int *s_pos = (int *)(dsm + L.side), *s_slot = s_pos + 8, *s_tok = s_slot + 8;
    float *s_sx = (float *)(s_tok + 8);
    int *s_sumx = (int *)(s_sx + 8);
    float *s_sh = (float *)(s_sumx + 8);
    int *s_sumh = (int *)(s_sh + 8), *s_last = s_sumh + 8;
    float *s_cw = (float *)(dsm + L.comb);   // [8][8]: token n's rank-k weight
    int *s_cinv = (int *)(s_cw + 64);        // [8][8]: the position of its rank-k slot
    uint64_t *bars = (uint64_t *)(dsm + L.bars);
    volatile uint32_t *abort = (volatile uint32_t *)(bars + NI);
    const uint32_t bar0 = smem_addr(bars);
    auto item_addr = [&](int i) {
        return dsm + L.items + (i < IG ? i * L.gu_bytes : IG * L.gu_bytes + (i - IG) * L.dn_bytes);
    };

    if (threadIdx.x == 0) {
        for (int i = 0; i < NI; i++) mbar_init(bar0 + 8 * i, 1);
        *abort = 0u;
        fence_barrier_init();
    }
    __syncthreads();
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    // the routing kernel's outputs: wait for its grid
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int n_units = __ldcg(a.n_units);
    const int4 fu = __ldcg(a.funits + c);   // (read with the count: the array holds stale units past it)
    if (c >= n_units) return;   // the whole cluster: n_units is the same for all its CTAs
    // first cluster barrier, split: arriving says this CTA is running; its wait
    // comes before the first access to another CTA's shared memory
    cluster_arrive();
    const int e = fu.x, p0 = fu.y & 0xffff;
    int cnt = fu.y >> 16;
    if (cnt > 8) {   // (at most T <= 8 slots per expert by construction)
        if (threadIdx.x == 0) set_flag(a.flag, MAPLE_DEVFLAG_BAD_INDEX);
        cnt = 8;
    }

    // ---- 1. this warp's items, all copies at once (gate/up items r*IG.., down items r*ID..)
    if (lane == 0)
        for (int i = warp; i < NI; i += kDfWarps) {
            const uint32_t bytes = i < IG ? L.gu_bytes : L.dn_bytes;
            const uint8_t *src = i < IG ? a.w_gu + ((size_t)e * mma_gu_items(F) + r * IG + i) * L.gu_bytes
                                        : a.w_dn + ((size_t)e * mma_dn_items(F) + r * L.id + (i - IG)) * L.dn_bytes;
            mbar_expect_tx(bar0 + 8 * i, bytes);
            bulk_g2s(smem_addr(item_addr(i)), src, bytes, bar0 + 8 * i);
        }
    // the unit's tokens, and their q_x rows into the B operand (fragment order,
    // 128-byte swizzled); padding tokens of the n-tile are left as they are
    const bool taps = a.tap_acc_gate || a.tap_acc_up || a.tap_qh || a.tap_sh || a.tap_acc_down;
    auto tok = [&](int n) { return min((int)(((uint32_t)(n < 4 ? fu.z : fu.w) >> (8 * (n & 3))) & 0xffu), a.T - 1); };
    if (threadIdx.x < cnt) {
        const int n = threadIdx.x, t = tok(n);
        s_pos[n] = p0 + n;
        s_tok[n] = t;
        s_slot[n] = taps ? __ldcg(a.perm + p0 + n) : 0;   // (slot order: for the taps only)
        s_sx[n] = __ldcg(a.sx + t);
        s_sumx[n] = __ldcg(a.sumx + t);
    }
    if (threadIdx.x >= 32 && threadIdx.x < 32 + 8 * K) {   // the combine's weights and yE positions, early
        const int n = (threadIdx.x - 32) / K, k = threadIdx.x - 32 - n * K;
        if (n < cnt) {
            const int t = tok(n);
            s_cw[n * 8 + k] = __ldcg(a.topk_w + t * K + k);
            s_cinv[n * 8 + k] = __ldcg(a.inv + t * K + k);
        }
    }
    const int cpr = D / 16;
    for (int idx = threadIdx.x; idx < cnt * cpr; idx += kDfThreads) {
        const int n = idx / cpr, cc = idx - n * cpr;
        const int t = tok(n);
        const uint32_t dst = smem_addr(b1 + (cc >> 3) * 1024 + dx_b_chunk(n, cc & 7));
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst),
                     "l"(reinterpret_cast<const uint4 *>(a.qxp + (size_t)t * D) + cc)
                     : "memory");
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    __syncthreads();

    // ---- 2. gate/up items: item i of the slice is tile r*IG + i (outputs 8(r*IG+i) ..)
    {
        const uint32_t bb_lo = smem_addr(b1) + dx_b_chunk(g, 2 * tig), bb_hi = smem_addr(b1) + dx_b_chunk(g, 2 * tig + 1);
        for (int i = warp; i < IG; i += kDfWarps) {
            if (!mbar_wait(bar0 + 8 * i, 0, abort, a.flag, a.wait_ns)) break;
            const uint8_t *ip = item_addr(i);
            const float *alpha_s = reinterpret_cast<const float *>(ip + 4 * D);
            int acc[2][4][4];
            dx_tile<1>(smem_addr(ip) + lane * 16, bb_lo, bb_hi, KB1, 0, acc);
            const int ol = 8 * i + g, o = r * FS + ol;
            const float ag = alpha_s[g], au = alpha_s[8 + g];
#pragma unroll
            for (int h2 = 0; h2 < 2; h2++) {
                const int n = 2 * tig + h2;
                if (n < cnt) {
                    const int gd = dx_total(acc, 0, h2) - s_sumx[n];
                    const int ud = dx_total(acc, 0, 2 + h2) - s_sumx[n];
                    const float gv = __fmul_rn((float)gd, __fmul_rn(ag, s_sx[n]));
                    const float uv = __fmul_rn((float)ud, __fmul_rn(au, s_sx[n]));
                    hl[n * FS + ol] = swiglu(gv, uv);
                    if (a.tap_acc_gate) a.tap_acc_gate[(size_t)s_slot[n] * F + o] = gd;
                    if (a.tap_acc_up) a.tap_acc_up[(size_t)s_slot[n] * F + o] = ud;
                }
            }
        }
    }
    __syncthreads();
    const bool dead = *abort != 0;   // (no wait runs from here to the down phase: the same in every thread)
    cluster_wait();   // every CTA of the cluster is running: distributed shared memory may be used
    // each token's |h| maximum over the slice, to every CTA of the cluster
    if (warp < cnt && !dead) {
        float m = 0.0f;
        for (int k = lane; k < FS; k += 32) m = fmaxf(m, fabsf(hl[warp * FS + k]));
        m = warp_max(m);
        if (lane < C) cluster.map_shared_rank(s_amax, lane)[r * 8 + warp] = m;
    }
    cluster.sync();

    // ---- 3. s_h from the maxima of all slices; requantise the slice into every CTA's
    // down B operand (word w = columns 4w .. 4w+3 of the slot's row), with the code sums
    const int wps = FS / 4;              // words of the slice per token (a power of two >= C)
    const int tpt = wps < 32 ? wps : 32; // threads per token, each taking wps / tpt words
    if (threadIdx.x < cnt * tpt && !dead) {
        const int n = threadIdx.x / tpt, wl0 = threadIdx.x - n * tpt;
        float amax = 0.0f;
        for (int q = 0; q < C; q++) amax = fmaxf(amax, s_amax[q * 8 + n]);
        const float inv = amax > 0.0f ? __fdiv_rn(127.0f, amax) : 0.0f;
        int sum = 0;
        for (int wl = wl0; wl < wps; wl += tpt) {
            const int w = r * wps + wl;
            const float4 hv = *reinterpret_cast<const float4 *>(hl + n * FS + 4 * wl);
            int q0 = 0, q1 = 0, q2 = 0, q3 = 0;
            if (amax > 0.0f) {
                q0 = quant_code(hv.x, inv);
                q1 = quant_code(hv.y, inv);
                q2 = quant_code(hv.z, inv);
                q3 = quant_code(hv.w, inv);
            }
            const uint32_t pk = (uint32_t)(q0 & 0xff) | ((uint32_t)(q1 & 0xff) << 8) | ((uint32_t)(q2 & 0xff) << 16) |
                                ((uint32_t)(q3 & 0xff) << 24);
            const int fp = frag_word_pos(w & 31);
            const uint32_t off = (uint32_t)((w >> 5) * 1024) + dx_b_chunk(n, fp >> 2) + (fp & 3) * 4;
            for (int q = 0; q < C; q++) *reinterpret_cast<uint32_t *>(cluster.map_shared_rank(b2, q) + off) = pk;
            if (a.tap_qh) reinterpret_cast<uint32_t *>(a.tap_qh + (size_t)s_slot[n] * F)[w] = pk;
            sum += q0 + q1 + q2 + q3;
        }
        const int live = cnt * tpt - warp * 32;   // lanes of this warp in the mapping (whole groups of tpt)
        const unsigned mask = live >= 32 ? FULL : (1u << live) - 1u;
        for (int o2 = tpt / 2; o2 >= 1; o2 >>= 1) sum += __shfl_xor_sync(mask, sum, o2);
        if (wl0 < C) cluster.map_shared_rank(s_sums, wl0)[r * 8 + n] = sum;
    }
    cluster.sync();   // every code and sum is in place; no shared memory of another CTA is touched after this
    if (threadIdx.x < cnt) {
        const int n = threadIdx.x;
        float amax = 0.0f;
        int sum = 0;
        for (int q = 0; q < C; q++) {
            amax = fmaxf(amax, s_amax[q * 8 + n]);
            sum += s_sums[q * 8 + n];
        }
        const float sv = amax > 0.0f ? __fdiv_rn(amax, 127.0f) : 0.0f;
        s_sh[n] = sv;
        s_sumh[n] = sum;
        if (a.tap_sh && r == 0) a.tap_sh[s_slot[n]] = sv;
    }
    if (a.stall && threadIdx.x == 0) {
        // test hook: wait for a word nothing sets, so that the bounded wait expires
        const uint64_t t0 = global_ns();
        while (true) {
            unsigned v;
            asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(a.never) : "memory");
            if (v == 1u) break;
            __nanosleep(256);
            if (*abort || global_ns() - t0 > a.wait_ns) {
                *abort = 1u;
                set_flag(a.flag, MAPLE_DEVFLAG_TIMEOUT);
                break;
            }
        }
    }
    __syncthreads();

    // ---- 4. down items: item i of the slice is item r*ID + i (tiles S2*(r*ID+i) ..)
    if (!*abort) {   // (read after the barrier above: the same in every thread)
        const uint32_t bb_lo = smem_addr(b2) + dx_b_chunk(g, 2 * tig), bb_hi = smem_addr(b2) + dx_b_chunk(g, 2 * tig + 1);
        for (int i = IG + (kDfWarps - 1 - warp); i < NI; i += kDfWarps) {
            if (!mbar_wait(bar0 + 8 * i, 0, abort, a.flag, a.wait_ns)) break;
            const uint8_t *ip = item_addr(i);
            const float *alpha_s = reinterpret_cast<const float *>(ip + 4 * D);
            const int it = r * L.id + (i - IG);
            const uint32_t aa = smem_addr(ip) + lane * 16;
            auto store = [&](int dt, int dd, int d0, int d1) {   // channels 16dt + g and + 8, token dd
                const int ch0 = 16 * dt + g, pos = s_pos[dd];
                a.ye[(size_t)pos * D + ch0] = __fmul_rn((float)d0, __fmul_rn(alpha_s[16 * (dt - S2 * it) + g], s_sh[dd]));
                a.ye[(size_t)pos * D + ch0 + 8] =
                    __fmul_rn((float)d1, __fmul_rn(alpha_s[16 * (dt - S2 * it) + 8 + g], s_sh[dd]));
                if (a.tap_acc_down) {
                    a.tap_acc_down[(size_t)s_slot[dd] * D + ch0] = d0;
                    a.tap_acc_down[(size_t)s_slot[dd] * D + ch0 + 8] = d1;
                }
            };
            if (S2 == 4) {
                int acc4[4][4][4];
                dx_tile4(aa, KB2 * 512, bb_lo, bb_hi, KB2, acc4);
#pragma unroll
                for (int d = 0; d < 4; d++)
#pragma unroll
                    for (int h2 = 0; h2 < 2; h2++) {
                        const int n = 2 * tig + h2;
                        if (n < cnt)
                            store(S2 * it + d, n,
                                  acc4[d][0][h2] + (acc4[d][1][h2] >> 2) + (acc4[d][2][h2] >> 4) + (acc4[d][3][h2] >> 6) -
                                      s_sumh[n],
                                  acc4[d][0][2 + h2] + (acc4[d][1][2 + h2] >> 2) + (acc4[d][2][2 + h2] >> 4) +
                                      (acc4[d][3][2 + h2] >> 6) - s_sumh[n]);
                    }
            } else {
                for (int d = 0; d < S2; d++) {
                    int acc[2][4][4];
                    dx_tile<1>(aa + d * KB2 * 512, bb_lo, bb_hi, KB2, 0, acc);
#pragma unroll
                    for (int h2 = 0; h2 < 2; h2++) {
                        const int n = 2 * tig + h2;
                        if (n < cnt)
                            store(S2 * it + d, n, dx_total(acc, 0, h2) - s_sumh[n], dx_total(acc, 0, 2 + h2) - s_sumh[n]);
                    }
                }
            }
        }
    }

    // ---- 5. combine: count this slice of each of the unit's tokens as done.  The
    // count is an acquire-release atomic after the CTA barrier: it publishes every
    // yE store of the CTA, and the CTA that completes a count sees every other
    // CTA's (its readers are ordered after it by the next barrier).
    __syncthreads();
    if (threadIdx.x < cnt) {
        int last = 0;
        if (!*abort) {
            const int t = s_tok[threadIdx.x];
            unsigned prev;
            asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(prev) : "l"(a.ctr + t * C + r) : "memory");
            last = prev == (unsigned)(K - 1);
            if (last) a.ctr[t * C + r] = 0u;   // every slot of (t, r) has arrived: nobody else touches it
        }
        s_last[threadIdx.x] = last;
    }
    __syncthreads();
    for (int n = 0; n < cnt; n++) {
        if (!s_last[n]) continue;
        const int t = s_tok[n];
        for (int c4 = threadIdx.x; c4 < DS / 4; c4 += kDfThreads) {
            const int ch = r * DS + 4 * c4;
            float4 yv = make_float4(0.f, 0.f, 0.f, 0.f);
            float4 ev[8];   // (K <= 8) every rank's row in flight at once, summed in rank order
#pragma unroll
            for (int k = 0; k < 8; k++)
                if (k < K) ev[k] = __ldcg(reinterpret_cast<const float4 *>(a.ye + (size_t)s_cinv[n * 8 + k] * D + ch));
#pragma unroll
            for (int k = 0; k < 8; k++)
                if (k < K) {
                    const float wk = s_cw[n * 8 + k];
                    yv.x = __fmaf_rn(wk, ev[k].x, yv.x);
                    yv.y = __fmaf_rn(wk, ev[k].y, yv.y);
                    yv.z = __fmaf_rn(wk, ev[k].z, yv.z);
                    yv.w = __fmaf_rn(wk, ev[k].w, yv.w);
                }
            const size_t o = (size_t)t * D + ch;
            if (a.resid) {
                const float4 rv = *reinterpret_cast<const float4 *>(a.resid + o);
                yv.x = __fadd_rn(rv.x, yv.x);
                yv.y = __fadd_rn(rv.y, yv.y);
                yv.z = __fadd_rn(rv.z, yv.z);
                yv.w = __fadd_rn(rv.w, yv.w);
            }
            *reinterpret_cast<float4 *>(a.y + o) = yv;
        }
    }

    // ---- exit: no copy may still be landing (after a failed wait: bounded waits)
    if (threadIdx.x == 0 && *abort)
        for (int i = 0; i < NI; i++) {
            const uint64_t t0 = global_ns();
            while (!mbar_test(bar0 + 8 * i, 0) && global_ns() - t0 < a.wait_ns) {
            }
        }
}

}  // namespace maple
