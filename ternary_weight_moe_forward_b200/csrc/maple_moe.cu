// C ABI of the ternary-weight MoE FFN layer (see include/maple_moe.h).
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <mutex>
#include <new>

#include "../../include/maple_moe.h"
#include "common.cuh"
#include "decode.cuh"
#include "layout.cuh"
#include "pack.cuh"
#include "route.cuh"
#include "tc_gemm.cuh"

using namespace maple;

namespace {

constexpr uint32_t kMagic = 0x4d41504cu;  // "MAPL"

struct Arena {
    size_t size = 0;
    size_t take(size_t bytes)
    {
        size_t off = size;
        size += (bytes + 255) & ~(size_t)255;
        return off;
    }
};

}  // namespace

struct maple_moe_s {
    uint32_t magic;
    int D, E, K, F, Tm, dmax;
    uint32_t cfg_flags;
    int num_sms;
    int device;
    int optin;                     // shared memory a block may opt in to
    int route_clusters;            // decode batches route with route_cluster_kernel: clusters that fit at once (0: not used)
    int df_fit[2];                 // dx_fused_kernel: clusters of 8 / 4 CTAs that fit at once (0: not used)
    char *base;                    // one device allocation: weights + workspace
    // weights
    uint8_t *w_mma_gu, *w_mma_dn;  // decode layout (MMA tiles), null when not built
    uint8_t *w_tc_gu, *w_tc_dn;    // tensor-core layout, null when not built
    float *alpha_gate, *alpha_up, *alpha_down, *router_w, *router_bias;
    // workspace: routing
    int8_t *qx, *qxp;              // q_x rows; the decode kernel's fragment-ordered copy (T <= 64)
    int8_t *xpos;                  // tensor-core path: the q_x row of every position (position order)
    const int8_t *zrow;
    float *sx;
    int *sumx;
    float *logits;
    int *topk_idx;
    float *topk_w;
    int *counts, *offsets, *perm, *inv, *active, *n_active, *blk_cnt;
    // workspace: experts
    int4 *pieces;
    int *n_pieces;
    float *pscale;                 // s_x of each position's token (tensor-core path)
    float *hscratch;               // per-CTA h rows of the gate/up grouped GEMM [num_sms][128][F]
    float *h;                      // decode kernel: SwiGLU rows [64*K][F]
    int8_t *qh;
    float *sh;
    float *ye;                     // decode kernel: expert outputs [64*K][D]
    int16_t *acc_hi;               // tensor-core path: down accumulators >> 1 [S][D]
    uint32_t *acc_lo;              // and their lowest bits [S][D/32]
    CUtensorMap map_xpos, map_qh;   // TMA maps of the tensor-core path's activation operands
    // counters (zero between calls)
    unsigned *tg_cnt, *glob_cnt;
    unsigned *dx_clear;            // decode kernels: |h| maxima [64*K] (zeroed by the routing kernel)
    int2 *units;                   // decode kernels: units of <= 16 slots of one expert (routing kernel)
    int *n_units;
    const unsigned *dx_never;      // a word that stays 0 (the stall test hook)
    unsigned *df_ctr;              // dx_fused_kernel: slots done per (token, channel slice) [8][8]
    int4 *funits;                  // dx_fused_kernel: its units with their tokens [64]
    uint16_t *xn;                  // stack: normalised input of the current layer
    // flag word in host-mapped memory
    unsigned *flag_host;
    unsigned *flag_dev;
    // failure handling: limit of every bounded device wait, test hooks, and the
    // counters a timed-out kernel may leave non-zero (reset before the next call)
    uint64_t wait_ns;
    uint32_t debug_flags;
    bool pending_reset;
    char *ctr_base;
    size_t ctr_bytes;
    // optional stage events (profiling)
    cudaEvent_t ev[4];
    bool use_events;
};

// Stage events are recorded as external event nodes when the stream is being
// captured into a CUDA graph, so that they can still be timed after replay.
static void stage_event(maple_moe_s *h, int i, cudaStream_t st)
{
    if (!h->use_events) return;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    cudaStreamIsCapturing(st, &cs);
    if (cs == cudaStreamCaptureStatusActive)
        cudaEventRecordWithFlags(h->ev[i], st, cudaEventRecordExternal);
    else
        cudaEventRecord(h->ev[i], st);
}

static bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

static int launch_status()
{
    return cudaGetLastError() == cudaSuccess ? MAPLE_OK : MAPLE_ERR_CUDA;
}

static int grid_for(int64_t n, int block, int cap)
{
    int64_t g = (n + block - 1) / block;
    if (g < 1) g = 1;
    if (g > cap) g = cap;
    return (int)g;
}

extern "C" const char *maple_moe_status_string(int status)
{
    switch (status) {
    case MAPLE_OK: return "ok";
    case MAPLE_ERR_INVALID_ARG: return "invalid argument";
    case MAPLE_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case MAPLE_ERR_OOM: return "out of device memory";
    case MAPLE_ERR_CUDA: return "CUDA error";
    case MAPLE_ERR_TIMEOUT: return "device wait timed out";
    case MAPLE_ERR_DEVICE_FLAG: return "a kernel flagged an invalid value";
    default: return "unknown status";
    }
}

extern "C" int maple_moe_pack_ternary(const int8_t *values, int64_t rows, int32_t cols, uint32_t *packed,
                                      int32_t *bad_count, maple_stream_t stream)
{
    if (rows < 0 || cols <= 0 || cols % 16 != 0) return MAPLE_ERR_INVALID_ARG;
    if (rows == 0) return MAPLE_OK;
    if (!values || !packed || !aligned16(values) || ((uintptr_t)packed & 3u)) return MAPLE_ERR_INVALID_ARG;
    const int64_t n_words = rows * (cols / 16);
    pack_ternary_kernel<<<grid_for(n_words, 256, 148 * 16), 256, 0, (cudaStream_t)stream>>>(values, n_words, packed,
                                                                                          bad_count);
    return launch_status();
}

// TMA map over an int8 row matrix [rows][cols]: boxes of box_rows rows x 128
// bytes, with the 128-byte swizzle (the UMMA K-major operand layout) or none;
// one-row boxes serve the four-row gathers
typedef CUresult (*encode_tiled_fn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                    const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                    CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static int make_act_map(CUtensorMap *map, void *base, int64_t rows, int64_t cols, int box_rows, bool swizzle)
{
    static encode_tiled_fn encode = nullptr;
    if (!encode) {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !fn)
            return MAPLE_ERR_CUDA;
        encode = (encode_tiled_fn)fn;
    }
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols};
    cuuint32_t box[2] = {(cuuint32_t)kTcBK, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, base, dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? MAPLE_OK : MAPLE_ERR_CUDA;
}

// Raise a kernel's dynamic shared-memory limit to what the device offers.
// Returns false (with the CUDA error state cleared) when that fails.
static bool allow_max_smem(const void *fn, int device)
{
    cudaFuncAttributes fa;
    int optin = 0;
    if (cudaFuncGetAttributes(&fa, fn) != cudaSuccess ||
        cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, device) != cudaSuccess ||
        cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, optin - (int)fa.sharedSizeBytes) !=
            cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return true;
}

typedef void (*route_fn)(RouteArgs);
template <int NPER>
static route_fn pick_route_n(int ni)
{
    switch (ni) {
    case 1: return route_kernel<1, NPER>;
    case 2: return route_kernel<2, NPER>;
    case 4: return route_kernel<4, NPER>;
    case 8: return route_kernel<8, NPER>;
    case 16: return route_kernel<16, NPER>;
    default: return nullptr;
    }
}
static route_fn pick_route(int D, int E) { return E <= 256 ? pick_route_n<8>(D / 256) : pick_route_n<32>(D / 256); }

// the cluster routing kernel for d_model = 256 * ni (E <= 256): d_model <= 2048
static route_fn pick_route_cluster(int D)
{
    switch (D / 256) {
    case 1: return route_cluster_kernel<1, 8>;
    case 2: return route_cluster_kernel<2, 8>;
    case 4: return route_cluster_kernel<4, 8>;
    case 8: return route_cluster_kernel<8, 8>;
    default: return nullptr;
    }
}

template <int NPER>
static route_fn pick_qtopk_n(int ni)
{
    switch (ni) {
    case 1: return quant_topk_kernel<1, NPER>;
    case 2: return quant_topk_kernel<2, NPER>;
    case 4: return quant_topk_kernel<4, NPER>;
    case 8: return quant_topk_kernel<8, NPER>;
    case 16: return quant_topk_kernel<16, NPER>;
    default: return nullptr;
    }
}
static route_fn pick_qtopk(int D, int E) { return E <= 256 ? pick_qtopk_n<8>(D / 256) : pick_qtopk_n<32>(D / 256); }

static bool pow2_upto(int v, int hi) { return v >= 1 && v <= hi && (v & (v - 1)) == 0; }

// launch configuration of the cluster routing kernel: one cluster of E/16 CTAs
// per group of 8 tokens
static void route_cluster_config(maple_moe_t h, int T, int gt, cudaStream_t st, cudaLaunchConfig_t *lc,
                                 cudaLaunchAttribute (&attr)[2], bool pdl)
{
    memset(lc, 0, sizeof *lc);
    lc->gridDim = dim3(h->E / kRcExperts, (T + gt - 1) / gt);
    lc->blockDim = dim3(kRcExperts * 32);
    lc->dynamicSmemBytes = route_cluster_smem_bytes(h->D, h->E, gt);
    lc->stream = st;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = h->E / kRcExperts;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    lc->attrs = attr;
    lc->numAttrs = pdl ? 2 : 1;
}

// How many clusters of the cluster routing kernel run at once on this device
// and shape (E <= 256, a multiple of 16; K <= 8; d_model <= 2048), 0 when it cannot run.
// Sets the kernel's attributes; clears any CUDA error it causes.
static void fused_setup(maple_moe_t h);
static int fused_cluster(maple_moe_t h, int T);

static int cluster_route_ok(maple_moe_t h)
{
    if (h->E > kRcMaxExperts || h->E % kRcExperts || h->K > 8) return 0;   // (choices buffer: 8 per token)
    route_fn k = pick_route_cluster(h->D);
    if (!k) return 0;
    const int csize = h->E / kRcExperts;
    if (cudaFuncSetAttribute((const void *)k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)route_cluster_smem_bytes(h->D, h->E, kRcMaxGroup)) != cudaSuccess ||
        (csize > 8 &&
         cudaFuncSetAttribute((const void *)k, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess)) {
        cudaGetLastError();
        return 0;
    }
    cudaLaunchConfig_t lc;
    cudaLaunchAttribute attr[2];
    route_cluster_config(h, kRcMaxGroup, kRcMaxGroup, nullptr, &lc, attr, false);
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, (const void *)k, &lc) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    return n;
}

// tokens per cluster for a batch of T: 8 when its 8-token groups all fit at
// once, else 0 (route_kernel serves the batch: 16-token groups measured slower)
static int route_cluster_group(maple_moe_t h, int T)
{
    const int nc = h->route_clusters;
    return nc >= 1 && (T + kRouteTokens - 1) / kRouteTokens <= nc ? kRouteTokens : 0;
}

static int check_shape(const maple_moe_config *c)
{
    if (c->d_model <= 0 || c->d_model % 256 != 0 || !pow2_upto(c->d_model / 256, 16)) return MAPLE_ERR_UNSUPPORTED_SHAPE;
    if (c->d_ff <= 0 || c->d_ff % 128 != 0 || !pow2_upto(c->d_ff / 128, 8)) return MAPLE_ERR_UNSUPPORTED_SHAPE;
    if (c->n_experts < 16 || c->n_experts > kMaxExperts || c->n_experts % 16 != 0) return MAPLE_ERR_UNSUPPORTED_SHAPE;
    if (c->top_k < 1 || c->top_k > 32 || c->top_k > c->n_experts) return MAPLE_ERR_UNSUPPORTED_SHAPE;
    if (c->max_tokens < 1 || c->max_tokens > 65536) return MAPLE_ERR_UNSUPPORTED_SHAPE;
    if (c->decode_max_tokens < 0 || c->decode_max_tokens > kRouteSmallT) return MAPLE_ERR_UNSUPPORTED_SHAPE;
    return MAPLE_OK;
}

extern "C" int maple_moe_create(const maple_moe_config *config, const maple_moe_weights *w, maple_stream_t stream,
                                maple_moe_t *out)
{
    if (!config || !w || !out) return MAPLE_ERR_INVALID_ARG;
    *out = nullptr;
    int rc = check_shape(config);
    if (rc) return rc;
    const uint32_t known = MAPLE_CFG_FORCE_GEMV | MAPLE_CFG_FORCE_TC | MAPLE_CFG_DECODE_ONLY;
    if ((config->flags & ~known) || ((config->flags & MAPLE_CFG_FORCE_TC) && (config->flags & ~MAPLE_CFG_FORCE_TC)))
        return MAPLE_ERR_INVALID_ARG;
    const void *need[] = {w->w_gate, w->w_up, w->w_down, w->alpha_gate, w->alpha_up, w->alpha_down, w->router_w};
    for (const void *p : need)
        if (!p || !aligned16(p)) return MAPLE_ERR_INVALID_ARG;
    if (w->router_bias && !aligned16(w->router_bias)) return MAPLE_ERR_INVALID_ARG;

    maple_moe_s *h = new (std::nothrow) maple_moe_s();
    if (!h) return MAPLE_ERR_OOM;
    h->magic = kMagic;
    h->D = config->d_model;
    h->E = config->n_experts;
    h->K = config->top_k;
    h->F = config->d_ff;
    h->Tm = config->max_tokens;
    h->dmax = config->decode_max_tokens ? config->decode_max_tokens : kRouteSmallT;
    h->cfg_flags = config->flags;
    if (cudaGetDevice(&h->device) != cudaSuccess ||
        cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, h->device) != cudaSuccess ||
        cudaDeviceGetAttribute(&h->optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, h->device) != cudaSuccess) {
        cudaGetLastError();
        delete h;
        return MAPLE_ERR_CUDA;
    }
    const int64_t D = h->D, E = h->E, K = h->K, F = h->F, Tm = h->Tm;
    const int64_t S = Tm * K;
    const int64_t T64 = Tm < kRouteSmallT ? Tm : kRouteSmallT, S64 = T64 * K;   // decode batches
    // which weight layouts the handle needs: the decode kernel's (when it fits the
    // shape: d_ff <= d_model and its shared memory at one token) unless every T
    // goes to the tensor cores; the tensor-core one unless the handle is for
    // decode batches only
    const bool dec_fits = dx_ring_slots(1, h->D, h->F, 1, h->K, h->E, (size_t)h->optin) > 0 &&
                          dx_ring_slots(2, h->D, h->F, 1, h->K, h->E, (size_t)h->optin) > 0;
    const bool build_dec = !(h->cfg_flags & MAPLE_CFG_FORCE_TC) && dec_fits;
    const bool build_tc = !(h->cfg_flags & (MAPLE_CFG_FORCE_GEMV | MAPLE_CFG_DECODE_ONLY)) || !dec_fits;
    if (!build_dec && (h->cfg_flags & (MAPLE_CFG_FORCE_GEMV | MAPLE_CFG_DECODE_ONLY))) {
        delete h;
        return MAPLE_ERR_UNSUPPORTED_SHAPE;   // the decode kernel does not fit this shape
    }
    const int64_t nblk = (Tm + kPermBlockTokens - 1) / kPermBlockTokens;
    Arena ar;
    const size_t o_mgu = build_dec ? ar.take(E * mma_gu_items((int)F) * mma_gu_item_bytes((int)D)) : 0;
    const size_t o_mdn = build_dec ? ar.take(E * mma_dn_items((int)F) * mma_dn_item_bytes((int)D, (int)F)) : 0;
    const size_t o_tgu = build_tc ? ar.take(E * F * D / 2) : 0, o_tdn = build_tc ? ar.take(E * D * F / 4) : 0;
    const size_t o_ag = ar.take(E * F * 4), o_au = ar.take(E * F * 4), o_ad = ar.take(E * D * 4);
    const size_t o_rw = ar.take(E * D * 4), o_rb = ar.take(E * 4);
    // workspace (zeroed once below)
    const size_t o_ws = ar.take(0);
    const size_t o_qx = ar.take(Tm * D), o_qxp = ar.take(T64 * D), o_zr = ar.take(D);
    const size_t o_sx = ar.take(Tm * 4), o_sumx = ar.take(Tm * 4);
    const size_t o_lg = ar.take(Tm * E * 4), o_ti = ar.take(S * 4), o_tw = ar.take(S * 4);
    const size_t o_cnt = ar.take(E * 4), o_off = ar.take((E + 1) * 4), o_perm = ar.take(S * 4), o_inv = ar.take(S * 4);
    const size_t o_act = ar.take(E * 4), o_nact = ar.take(4), o_blk = ar.take(nblk * E * 4);
    const size_t o_pc = build_tc ? ar.take((E + S / kPieceSlots + 1) * 16) : 0, o_npc = ar.take(4);
    const size_t o_ps = build_tc ? ar.take(S * 4 + 512) : 0;
    const size_t o_hs = build_tc ? ar.take((size_t)h->num_sms * kTcMaxN * F * 4) : 0;
    const size_t o_h = build_dec ? ar.take(S64 * F * 4) : 0;
    const size_t o_qh = build_tc ? ar.take(S * F) : 0, o_sh = build_tc ? ar.take(S * 4) : 0;
    const size_t o_xpos = build_tc ? ar.take(S * D) : 0;
    const size_t o_ye = build_dec ? ar.take(S64 * D * 4) : 0;
    const size_t o_ahi = build_tc ? ar.take(S * D * 2) : 0, o_alo = build_tc ? ar.take(S * D / 8) : 0;
    const size_t o_ctr = ar.take(0);   // counters: zero between calls
    const size_t o_tg = ar.take(((Tm + kRouteTokens - 1) / kRouteTokens) * 4), o_gc = ar.take(4);
    const size_t o_dx = ar.take((S64 + 1) * 4), o_dfc = ar.take(64 * 4), o_fu = ar.take(64 * 16);
    const size_t o_un = ar.take((E + (S64 + kUnitTokens - 1) / kUnitTokens + 1) * 8), o_nun = ar.take(4);
    const size_t o_ctr_end = ar.take(0);
    const size_t o_xn = ar.take(Tm * D * 2);

    if (cudaMalloc(&h->base, ar.size) != cudaSuccess) {
        cudaGetLastError();
        delete h;
        return MAPLE_ERR_OOM;
    }
    if (cudaHostAlloc(&h->flag_host, sizeof(unsigned), cudaHostAllocMapped) != cudaSuccess ||
        cudaHostGetDevicePointer(&h->flag_dev, h->flag_host, 0) != cudaSuccess) {
        cudaGetLastError();
        cudaFree(h->base);
        delete h;
        return MAPLE_ERR_CUDA;
    }
    *h->flag_host = 0;
    char *b = h->base;
    h->w_mma_gu = build_dec ? (uint8_t *)(b + o_mgu) : nullptr;
    h->w_mma_dn = build_dec ? (uint8_t *)(b + o_mdn) : nullptr;
    h->w_tc_gu = build_tc ? (uint8_t *)(b + o_tgu) : nullptr;
    h->w_tc_dn = build_tc ? (uint8_t *)(b + o_tdn) : nullptr;
    h->alpha_gate = (float *)(b + o_ag);
    h->alpha_up = (float *)(b + o_au);
    h->alpha_down = (float *)(b + o_ad);
    h->router_w = (float *)(b + o_rw);
    h->router_bias = w->router_bias ? (float *)(b + o_rb) : nullptr;
    h->qx = (int8_t *)(b + o_qx);
    h->qxp = (int8_t *)(b + o_qxp);
    h->zrow = (const int8_t *)(b + o_zr);
    h->sx = (float *)(b + o_sx);
    h->sumx = (int *)(b + o_sumx);
    h->logits = (float *)(b + o_lg);
    h->topk_idx = (int *)(b + o_ti);
    h->topk_w = (float *)(b + o_tw);
    h->counts = (int *)(b + o_cnt);
    h->offsets = (int *)(b + o_off);
    h->perm = (int *)(b + o_perm);
    h->inv = (int *)(b + o_inv);
    h->active = (int *)(b + o_act);
    h->n_active = (int *)(b + o_nact);
    h->blk_cnt = (int *)(b + o_blk);
    h->pieces = build_tc ? (int4 *)(b + o_pc) : nullptr;
    h->n_pieces = (int *)(b + o_npc);
    h->pscale = build_tc ? (float *)(b + o_ps) : nullptr;
    h->hscratch = build_tc ? (float *)(b + o_hs) : nullptr;
    h->h = build_dec ? (float *)(b + o_h) : nullptr;
    h->qh = build_tc ? (int8_t *)(b + o_qh) : nullptr;
    h->xpos = build_tc ? (int8_t *)(b + o_xpos) : nullptr;
    h->sh = build_tc ? (float *)(b + o_sh) : nullptr;
    h->ye = build_dec ? (float *)(b + o_ye) : nullptr;
    h->acc_hi = build_tc ? (int16_t *)(b + o_ahi) : nullptr;
    h->acc_lo = build_tc ? (uint32_t *)(b + o_alo) : nullptr;
    h->tg_cnt = (unsigned *)(b + o_tg);
    h->glob_cnt = (unsigned *)(b + o_gc);
    h->dx_clear = (unsigned *)(b + o_dx);
    h->dx_never = h->dx_clear + S64;   // zeroed at create, written by nothing
    h->df_ctr = (unsigned *)(b + o_dfc);
    h->funits = (int4 *)(b + o_fu);
    h->units = (int2 *)(b + o_un);
    h->n_units = (int *)(b + o_nun);
    h->xn = (uint16_t *)(b + o_xn);
    h->wait_ns = kDefaultWaitNs;
    h->ctr_base = b + o_ctr;
    h->ctr_bytes = o_ctr_end - o_ctr;

    cudaStream_t st = (cudaStream_t)stream;
    // the whole workspace starts at zero: counters must, and every index array
    // then holds in-range values even before its first write
    cudaMemsetAsync(b + o_ws, 0, ar.size - o_ws, st);
    cudaMemcpyAsync(h->alpha_gate, w->alpha_gate, E * F * 4, cudaMemcpyDeviceToDevice, st);
    cudaMemcpyAsync(h->alpha_up, w->alpha_up, E * F * 4, cudaMemcpyDeviceToDevice, st);
    cudaMemcpyAsync(h->alpha_down, w->alpha_down, E * D * 4, cudaMemcpyDeviceToDevice, st);
    cudaMemcpyAsync(h->router_w, w->router_w, E * D * 4, cudaMemcpyDeviceToDevice, st);
    if (w->router_bias) cudaMemcpyAsync(h->router_bias, w->router_bias, E * 4, cudaMemcpyDeviceToDevice, st);
    const int cap = h->num_sms * 16;
    if (build_dec) {
        repack_mma_gu_kernel<<<grid_for(E * F * D / 8, 256, cap), 256, 0, st>>>(w->w_gate, w->w_up, h->E, h->D, h->F,
                                                                               (uint32_t *)h->w_mma_gu);
        repack_mma_dn_kernel<<<grid_for(E * D * F / 16, 256, cap), 256, 0, st>>>(w->w_down, h->E, h->D, h->F,
                                                                                (uint32_t *)h->w_mma_dn);
        mma_item_scales_kernel<<<grid_for(E * (2 * F + D), 256, cap), 256, 0, st>>>(
            h->alpha_gate, h->alpha_up, h->alpha_down, h->E, h->D, h->F, (float *)h->w_mma_gu, (float *)h->w_mma_dn);
    }
    if (build_tc) {
        repack_tc_gu_kernel<<<grid_for(E * F * D / 8, 256, cap), 256, 0, st>>>(w->w_gate, w->w_up, h->E, h->D, h->F,
                                                                              (uint32_t *)h->w_tc_gu);
        repack_tc_dn_kernel<<<grid_for(E * D * F / 16, 256, cap), 256, 0, st>>>(w->w_down, h->E, h->D, h->F,
                                                                               (uint32_t *)h->w_tc_dn);
    }
    bool maps_ok = true;
    if (build_tc)
        maps_ok = make_act_map(&h->map_xpos, h->xpos, S, D, kTcMaxN, true) == MAPLE_OK &&
                  make_act_map(&h->map_qh, h->qh, S, F, kTcMaxN, true) == MAPLE_OK;
    // allow every kernel the largest dynamic shared memory the device offers, so
    // that handles of different shapes never cap one another's launches
    const void *kernels[] = {(const void *)tc_gemm_kernel<0>,         (const void *)tc_gemm_kernel<1>,
                             (const void *)pick_route(h->D, h->E),    (const void *)pick_qtopk(h->D, h->E),
                             (const void *)router_gemm_kernel,        (const void *)decode_stage_kernel<1>,
                             (const void *)decode_stage_kernel<2>};
    bool smem_ok = true;
    for (const void *k : kernels) smem_ok = allow_max_smem(k, h->device) && smem_ok;
    h->route_clusters = cluster_route_ok(h);
    fused_setup(h);
    if (!maps_ok || !smem_ok || cudaGetLastError() != cudaSuccess) {
        cudaFree(h->base);
        cudaFreeHost(h->flag_host);
        delete h;
        return MAPLE_ERR_CUDA;
    }
    *out = h;
    return MAPLE_OK;
}

static int check_handle(maple_moe_t h)
{
    if (!h || h->magic != kMagic) return MAPLE_ERR_INVALID_ARG;
    return MAPLE_OK;
}

// Report (and clear) what kernels of earlier calls flagged.  After a timeout the
// self-resetting counters may hold stale values: zero them on this call's
// stream first, so that the next call starts from the state create left.
static int take_flag(maple_moe_t h, cudaStream_t st)
{
    const unsigned f = __atomic_exchange_n(h->flag_host, 0u, __ATOMIC_ACQ_REL);
    if ((f & MAPLE_DEVFLAG_TIMEOUT) || h->pending_reset) {
        h->pending_reset = false;
        if (cudaMemsetAsync(h->ctr_base, 0, h->ctr_bytes, st) != cudaSuccess) return MAPLE_ERR_CUDA;
        if (f & MAPLE_DEVFLAG_TIMEOUT) return MAPLE_ERR_TIMEOUT;
    }
    return f ? MAPLE_ERR_DEVICE_FLAG : MAPLE_OK;
}

// routing stage: quantise, logits, top-k (+ the permutation)
static int run_route(maple_moe_t h, const uint16_t *x, int T, const maple_moe_taps *taps, int32_t *out_idx,
                     float *out_w, int32_t *out_counts, bool permute, bool pieces, cudaStream_t st,
                     unsigned *clear = nullptr, int n_clear = 0, bool frag = false, const float *norm_resid = nullptr,
                     bool pdl = false)
{
    RouteArgs a;
    memset(&a, 0, sizeof a);
    a.x = x;
    a.resid = norm_resid;   // (T <= 64 only) x = bf16(RMSNorm(resid)), computed by the routing kernel
    a.qxp = frag ? h->qxp : nullptr;   // the decode kernels' fragment-ordered q_x
    a.units = frag ? h->units : nullptr;   // and their units (built with the fused permutation)
    a.funits = frag && fused_cluster(h, T) ? h->funits : nullptr;   // (the fused expert kernel's)
    a.n_units = h->n_units;
    a.T = T;
    a.D = h->D;
    a.E = h->E;
    a.K = h->K;
    a.Wr = h->router_w;
    a.bias = h->router_bias;
    a.qx = h->qx;
    a.sx = h->sx;
    a.sumx = h->sumx;
    a.logits = h->logits;
    a.topk_idx = h->topk_idx;
    a.topk_w = h->topk_w;
    if (taps) {
        a.tap_qx = taps->q_x;
        a.tap_sx = taps->s_x;
        a.tap_logits = taps->logits;
        a.tap_offsets = taps->expert_offsets;
        a.tap_perm = taps->perm;
    }
    a.out_idx = out_idx ? out_idx : (taps ? taps->topk_idx : nullptr);
    a.out_w = out_w ? out_w : (taps ? taps->topk_w : nullptr);
    a.out_counts = out_counts ? out_counts : (taps ? taps->expert_counts : nullptr);
    a.tg_cnt = h->tg_cnt;
    a.glob_cnt = h->glob_cnt;
    a.counts = h->counts;
    a.offsets = h->offsets;
    a.perm = h->perm;
    a.inv = h->inv;
    a.active = h->active;
    a.n_active = h->n_active;
    a.flag = h->flag_dev;
    // few tokens: one latency-oriented kernel (logits, top-k by the last CTA of
    // each token group, permutation by the last group); many tokens: a tiled
    // router GEMM, then quantise + top-k, then the multi-CTA permutation
    const bool small = T <= kRouteSmallT;
    const bool fused = small && permute && !pieces && (int64_t)T * h->E <= kFusedMarkBytes;
    a.fuse_permute = fused ? 1 : 0;
    if (clear && !small) {
        if (cudaMemsetAsync(clear, 0, (size_t)n_clear * 4, st) != cudaSuccess) return MAPLE_ERR_CUDA;
    } else {
        a.clear = clear;
        a.n_clear = n_clear;
    }
    const int gt = small ? route_cluster_group(h, T) : 0;
    if (gt) {
        // as a programmatic dependent (the layer stack) the kernel loads its router
        // rows while the previous layer finishes, then waits for it
        a.group_tokens = gt;
        cudaLaunchConfig_t lc;
        cudaLaunchAttribute attr[2];
        route_cluster_config(h, T, gt, st, &lc, attr, pdl);
        if (cudaLaunchKernelEx(&lc, pick_route_cluster(h->D), a) != cudaSuccess) return MAPLE_ERR_CUDA;
    } else if (small) {
        cudaLaunchConfig_t lc;
        memset(&lc, 0, sizeof lc);
        lc.gridDim = dim3(h->E / kRouteExperts, (T + kRouteTokens - 1) / kRouteTokens);
        lc.blockDim = dim3(256);
        lc.dynamicSmemBytes = route_smem_bytes(h->D);
        lc.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        lc.attrs = attr;
        lc.numAttrs = pdl ? 1 : 0;
        if (cudaLaunchKernelEx(&lc, pick_route(h->D, h->E), a) != cudaSuccess) return MAPLE_ERR_CUDA;
    } else {
        dim3 grid((T + kRgTok - 1) / kRgTok, h->E / kRgExp);
        router_gemm_kernel<<<grid, 256, 2 * kRgStage, st>>>(x, T, h->D, h->E, h->router_w, h->router_bias,
                                                           h->logits, a.tap_logits);
        pick_qtopk(h->D, h->E)<<<(T + 7) / 8, 256, (size_t)8 * h->D * 2, st>>>(a);
    }
    if (permute && !fused) {
        PermArgs p;
        memset(&p, 0, sizeof p);
        p.idx = h->topk_idx;
        p.T = T;
        p.K = h->K;
        p.E = h->E;
        p.blk_cnt = h->blk_cnt;
        p.counts = h->counts;
        p.offsets = h->offsets;
        p.perm = h->perm;
        p.inv = h->inv;
        p.active = h->active;
        p.n_active = h->n_active;
        p.out_counts = a.out_counts;
        p.tap_offsets = a.tap_offsets;
        p.tap_perm = a.tap_perm;
        p.pieces = pieces ? h->pieces : nullptr;
        p.n_pieces = h->n_pieces;
        p.sx = h->sx;
        p.pscale = pieces ? h->pscale : nullptr;
        p.flag = h->flag_dev;
        const int nblk = (T + kPermBlockTokens - 1) / kPermBlockTokens;
        perm_count_kernel<<<nblk, 256, 0, st>>>(p);
        perm_scan_kernel<<<1, 1024, 0, st>>>(p);
        perm_scatter_kernel<<<nblk, 256, 0, st>>>(p);
    }
    return launch_status();
}

// the decode kernels: gate/up (+ SwiGLU, per-slot maxima), down (+
// requantisation), combine; the first two persistent, one CTA per SM
// dx_fused_kernel with clusters of C CTAs: the slices must split into whole
// items, the requantisation's words of a slice (F/C/4 per token) must be a
// power of two of at least C, and the slices must fit shared memory
static bool fused_shape_ok(maple_moe_t h, int C)
{
    const int F = h->F, wps = F / C / 4;
    if (!h->w_mma_gu || h->K > 8 || h->F > h->D || h->D % h->F) return false;
    if ((F / 8) % C || (F / 16) % C || wps < C || (wps & (wps - 1))) return false;
    return DfSmem(h->D, F, C).total <= h->optin;
}

static void fused_cluster_config(int C, int n_clusters, int smem, cudaStream_t st, cudaLaunchConfig_t *lc,
                                 cudaLaunchAttribute *attr)
{
    memset(lc, 0, sizeof *lc);
    lc->gridDim = dim3((unsigned)(n_clusters * C));
    lc->blockDim = dim3(kDfThreads);
    lc->dynamicSmemBytes = (size_t)smem;
    lc->stream = st;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    lc->attrs = attr;
    lc->numAttrs = 2;
}

// at create: which cluster sizes of dx_fused_kernel serve this shape, and how
// many such clusters fit at once
static const int kDfSizes[2] = {8, 4};   // cluster sizes of dx_fused_kernel, in order of preference

static void fused_setup(maple_moe_t h)
{
    int need = 0;
    for (int i = 0; i < 2; i++) {
        h->df_fit[i] = 0;
        if (fused_shape_ok(h, kDfSizes[i]) && DfSmem(h->D, h->F, kDfSizes[i]).total > need)
            need = DfSmem(h->D, h->F, kDfSizes[i]).total;
    }
    if (!need) return;
    if (cudaFuncSetAttribute((const void *)dx_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, need) !=
        cudaSuccess) {
        cudaGetLastError();
        return;
    }
    for (int i = 0; i < 2; i++) {
        const int C = kDfSizes[i];
        if (!fused_shape_ok(h, C)) continue;
        cudaLaunchConfig_t lc;
        cudaLaunchAttribute attr[2];
        fused_cluster_config(C, 1, DfSmem(h->D, h->F, C).total, nullptr, &lc, attr);
        lc.numAttrs = 1;   // (occupancy: the cluster shape only)
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, (const void *)dx_fused_kernel, &lc) != cudaSuccess) {
            cudaGetLastError();
            n = 0;
        }
        h->df_fit[i] = n;
    }
}

// cluster size of the fused expert kernel for a batch of T tokens (0: the
// two-kernel path).  Its clusters (one per unit, at most min(T*K, E)) must all
// fit at once: a second wave of clusters costs the whole kernel's latency
// again, more than the two-kernel path takes.  The larger size (8, 4) whose
// clusters all fit.  (Two-CTA clusters with a ring of slots, so that T = 8 fits
// in one wave, measured no faster than the two-kernel path: the slowest
// cluster's combine and the weight stream of 400 KB per CTA set its pace.)
static int fused_cluster(maple_moe_t h, int T)
{
    if (T > 8 || h->K > 8 || (h->debug_flags & MAPLE_DEBUG_SPLIT_SMALL)) return 0;
    const int n = T * h->K < h->E ? T * h->K : h->E;
    for (int i = 0; i < 2; i++)
        if (h->df_fit[i] >= n) return kDfSizes[i];
    return 0;
}

static int run_experts_fused(maple_moe_t h, int T, int C, float *y, const float *resid, const maple_moe_taps *taps,
                             cudaStream_t st)
{
    DfArgs d;
    memset(&d, 0, sizeof d);
    d.T = T;
    d.D = h->D;
    d.E = h->E;
    d.K = h->K;
    d.F = h->F;
    d.sx = h->sx;
    d.sumx = h->sumx;
    d.qxp = h->qxp;
    d.perm = h->perm;
    d.inv = h->inv;
    d.topk_w = h->topk_w;
    d.funits = h->funits;
    d.n_units = h->n_units;
    d.w_gu = h->w_mma_gu;
    d.w_dn = h->w_mma_dn;
    d.ye = h->ye;
    d.ctr = h->df_ctr;
    d.y = y;
    d.resid = resid;
    if (taps) {
        d.tap_acc_gate = taps->acc_gate;
        d.tap_acc_up = taps->acc_up;
        d.tap_acc_down = taps->acc_down;
        d.tap_qh = taps->q_h;
        d.tap_sh = taps->s_h;
    }
    d.flag = h->flag_dev;
    d.never = h->dx_never;
    d.wait_ns = h->wait_ns;
    d.stall = (h->debug_flags & MAPLE_DEBUG_STALL_DOWN) ? 1 : 0;
    // one cluster per unit: at most one unit per slot and per expert
    const int n_clusters = T * h->K < h->E ? T * h->K : h->E;
    cudaLaunchConfig_t lc;
    cudaLaunchAttribute attr[2];
    fused_cluster_config(C, n_clusters, DfSmem(h->D, h->F, C).total, st, &lc, attr);
    if (cudaLaunchKernelEx(&lc, dx_fused_kernel, d) != cudaSuccess) return MAPLE_ERR_CUDA;
    stage_event(h, 2, st);
    stage_event(h, 3, st);
    return launch_status();
}

static int run_experts_dec(maple_moe_t h, int T, float *y, const float *resid, const maple_moe_taps *taps,
                           cudaStream_t st)
{
    const int C = fused_cluster(h, T);
    if (C) return run_experts_fused(h, T, C, y, resid, taps, st);
    const int n1 = dx_ring_slots(1, h->D, h->F, T, h->K, h->E, (size_t)h->optin);
    const int n2 = dx_ring_slots(2, h->D, h->F, T, h->K, h->E, (size_t)h->optin);
    if (!n1 || !n2) return MAPLE_ERR_UNSUPPORTED_SHAPE;
    DxArgs d;
    memset(&d, 0, sizeof d);
    d.T = T;
    d.D = h->D;
    d.E = h->E;
    d.K = h->K;
    d.F = h->F;
    d.sx = h->sx;
    d.sumx = h->sumx;
    d.qxp = h->qxp;
    d.perm = h->perm;
    d.units = h->units;
    d.n_units = h->n_units;
    d.w_gu = h->w_mma_gu;
    d.w_dn = h->w_mma_dn;
    d.h = h->h;
    d.amax = h->dx_clear;
    d.never = h->dx_never;
    d.ye = h->ye;
    if (taps) {
        d.tap_acc_gate = taps->acc_gate;
        d.tap_acc_up = taps->acc_up;
        d.tap_acc_down = taps->acc_down;
        d.tap_qh = taps->q_h;
        d.tap_sh = taps->s_h;
    }
    d.flag = h->flag_dev;
    d.wait_ns = h->wait_ns;
    d.stall = (h->debug_flags & MAPLE_DEBUG_STALL_DOWN) ? 1 : 0;
    // Each is a programmatic dependent of the kernel before it (the routing
    // kernel, the gate/up kernel, the down kernel): its launch and set-up
    // overlap that kernel's tail, and griddepcontrol.wait orders every read of
    // that kernel's outputs after its grid.  No CTA waits on another CTA of its
    // own grid.
    cudaLaunchConfig_t lc;
    memset(&lc, 0, sizeof lc);
    lc.gridDim = dim3(h->num_sms);
    lc.blockDim = dim3(kDxThreads);
    lc.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    lc.attrs = attr;
    lc.numAttrs = 1;
    d.nslot = n1;
    lc.dynamicSmemBytes = DxSmem(1, h->D, h->F, T, h->K, h->E, n1).total;
    if (cudaLaunchKernelEx(&lc, decode_stage_kernel<1>, d) != cudaSuccess) return MAPLE_ERR_CUDA;
    stage_event(h, 2, st);
    d.nslot = n2;
    lc.dynamicSmemBytes = DxSmem(2, h->D, h->F, T, h->K, h->E, n2).total;
    if (cudaLaunchKernelEx(&lc, decode_stage_kernel<2>, d) != cudaSuccess) return MAPLE_ERR_CUDA;
    lc.gridDim = dim3((unsigned)((T * (h->D / 4) + 255) / 256));
    lc.blockDim = dim3(256);
    lc.dynamicSmemBytes = 0;
    if (cudaLaunchKernelEx(&lc, dx_combine_kernel, (const float *)h->ye, (const int *)h->inv, (const float *)h->topk_w,
                           T, h->K, h->D, y, resid) != cudaSuccess)
        return MAPLE_ERR_CUDA;
    stage_event(h, 3, st);
    return launch_status();
}

static int check_taps(const maple_moe_taps *t)
{
    if (!t) return MAPLE_OK;
    const void *ps[] = {t->q_x, t->s_x, t->logits, t->topk_idx, t->topk_w, t->acc_gate, t->acc_up, t->q_h,
                        t->s_h, t->acc_down, t->expert_counts, t->expert_offsets, t->perm};
    for (const void *p : ps)
        if (p && !aligned16(p)) return MAPLE_ERR_INVALID_ARG;
    return MAPLE_OK;
}

extern "C" int maple_moe_route(maple_moe_t h, const uint16_t *x, int32_t T, int32_t *topk_idx, float *topk_w,
                               int32_t *expert_counts, maple_stream_t stream)
{
    int rc = check_handle(h);
    if (rc) return rc;
    if (T < 0 || T > h->Tm) return MAPLE_ERR_INVALID_ARG;
    if ((rc = take_flag(h, (cudaStream_t)stream))) return rc;
    if (T == 0) return MAPLE_OK;
    if (!x || !aligned16(x)) return MAPLE_ERR_INVALID_ARG;
    for (const void *p : {(const void *)topk_idx, (const void *)topk_w, (const void *)expert_counts})
        if (p && !aligned16(p)) return MAPLE_ERR_INVALID_ARG;
    return run_route(h, x, T, nullptr, topk_idx, topk_w, expert_counts, expert_counts != nullptr, false,
                     (cudaStream_t)stream);
}

// tensor-core expert stage: gate/up grouped GEMM (SwiGLU and the requantisation
// fused), down grouped GEMM, combine
static int run_experts_tc(maple_moe_t h, int T, float *y, const float *resid, const maple_moe_taps *taps,
                          cudaStream_t st)
{
    TcArgs g;
    memset(&g, 0, sizeof g);
    g.D = h->D;
    g.F = h->F;
    g.K = h->K;
    g.pieces = h->pieces;
    g.n_pieces = h->n_pieces;
    g.perm = h->perm;
    g.sh = h->sh;
    g.pscale = h->pscale;
    g.flag = h->flag_dev;
    g.wait_ns = h->wait_ns;
    g.codes = h->w_tc_gu;
    g.alpha0 = h->alpha_gate;
    g.alpha1 = h->alpha_up;
    g.out = h->hscratch;
    g.qh = h->qh;
    g.tap0 = taps ? taps->acc_gate : nullptr;
    g.tap1 = taps ? taps->acc_up : nullptr;
    g.tap_qh = taps ? taps->q_h : nullptr;
    g.tap_sh = taps ? taps->s_h : nullptr;
    // the q_x row of every position, so that the gate/up GEMM loads its activation
    // tiles with one 2-D copy per stage
    gather_rows_kernel<<<grid_for((int64_t)T * h->K, 8, h->num_sms * 16), 256, 0, st>>>(h->qx, h->perm, T * h->K,
                                                                                       h->K, h->D, h->xpos);
    tc_gemm_kernel<0><<<h->num_sms, kTcThreads, TcSmem<0>::kTotal, st>>>(h->map_xpos, g);
    stage_event(h, 2, st);
    g.codes = h->w_tc_dn;
    g.alpha0 = h->alpha_down;
    g.alpha1 = nullptr;
    g.out = nullptr;
    g.qh = nullptr;
    g.acc_hi = h->acc_hi;
    g.acc_lo = h->acc_lo;
    g.tap0 = taps ? taps->acc_down : nullptr;
    g.tap1 = nullptr;
    g.tap_qh = nullptr;
    g.tap_sh = nullptr;
    tc_gemm_kernel<1><<<h->num_sms, kTcThreads, TcSmem<1>::kTotal, st>>>(h->map_qh, g);
    combine_kernel<<<grid_for((int64_t)T * h->D / 4, 256, h->num_sms * 8), 256, 0, st>>>(
        h->acc_hi, h->acc_lo, h->alpha_down, h->sh, h->topk_idx, h->inv, h->topk_w, T, h->K, h->D, y, resid);
    stage_event(h, 3, st);
    return launch_status();
}

// ring slots of the decode kernel for a batch of T tokens, 0 when it does not serve it
static int dec_slots(maple_moe_t h, int T)
{
    if (!h->w_mma_gu || T > kRouteSmallT || (int64_t)T * h->E > kFusedMarkBytes) return 0;
    if (T > h->dmax && !(h->cfg_flags & MAPLE_CFG_FORCE_GEMV)) return 0;
    const int n1 = dx_ring_slots(1, h->D, h->F, T, h->K, h->E, (size_t)h->optin);
    const int n2 = dx_ring_slots(2, h->D, h->F, T, h->K, h->E, (size_t)h->optin);
    return n1 < n2 ? n1 : n2;
}

// norm_resid (decode batches only): the layer input is bf16(RMSNorm(norm_resid)),
// computed by the routing kernel, and x is unused; pdl: launch the routing
// kernel as a programmatic dependent of the kernel before it (the layer stack)
static int forward_impl(maple_moe_t h, const uint16_t *x, int32_t T, float *y, const float *resid,
                        const maple_moe_taps *taps, cudaStream_t st, const float *norm_resid = nullptr,
                        bool pdl = false)
{
    const int nslot = (h->cfg_flags & MAPLE_CFG_FORCE_TC) ? 0 : dec_slots(h, T);
    if (!nslot && !h->w_tc_gu) return MAPLE_ERR_UNSUPPORTED_SHAPE;   // decode-only handle, T too large
    if (norm_resid && !nslot) return MAPLE_ERR_INVALID_ARG;          // (callers check dec_slots first)
    stage_event(h, 0, st);
    int rc;
    if (nslot) {
        // the routing kernel also builds the permutation and the decode kernels'
        // units (its last CTA), zeroes the per-slot maxima and writes the
        // fragment-ordered q_x
        rc = run_route(h, x, T, taps, nullptr, nullptr, nullptr, true, false, st, h->dx_clear, T * h->K, true,
                       norm_resid, pdl);
    } else {
        rc = run_route(h, x, T, taps, nullptr, nullptr, nullptr, true, true, st);
    }
    if (rc) return rc;
    stage_event(h, 1, st);
    return nslot ? run_experts_dec(h, T, y, resid, taps, st) : run_experts_tc(h, T, y, resid, taps, st);
}

extern "C" int maple_moe_forward(maple_moe_t h, const uint16_t *x, int32_t T, float *y, const maple_moe_taps *taps,
                                 maple_stream_t stream)
{
    int rc = check_handle(h);
    if (rc) return rc;
    if (T < 0 || T > h->Tm) return MAPLE_ERR_INVALID_ARG;
    if ((rc = take_flag(h, (cudaStream_t)stream))) return rc;
    if (T == 0) return MAPLE_OK;
    if (!x || !y || !aligned16(x) || !aligned16(y)) return MAPLE_ERR_INVALID_ARG;
    if ((rc = check_taps(taps))) return rc;
    return forward_impl(h, x, T, y, nullptr, taps, (cudaStream_t)stream);
}

extern "C" int maple_moe_stack_forward(const maple_moe_t *layers, int32_t n_layers, float *resid, int32_t T,
                                       maple_stream_t stream)
{
    if (!layers || n_layers < 0) return MAPLE_ERR_INVALID_ARG;
    if (n_layers == 0) return MAPLE_OK;
    for (int l = 0; l < n_layers; l++) {
        int rc = check_handle(layers[l]);
        if (rc) return rc;
        const maple_moe_s *a = layers[l], *b = layers[0];
        if (a->D != b->D || a->E != b->E || a->K != b->K || a->F != b->F) return MAPLE_ERR_INVALID_ARG;
        if (T < 0 || T > a->Tm) return MAPLE_ERR_INVALID_ARG;
    }
    for (int l = 0; l < n_layers; l++) {
        int rc = take_flag(layers[l], (cudaStream_t)stream);
        if (rc) return rc;
    }
    if (T == 0) return MAPLE_OK;
    if (!resid || !aligned16(resid)) return MAPLE_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    uint16_t *xn = layers[0]->xn;
    bool chained = false;   // the previous layer ended with the decode kernel
    for (int l = 0; l < n_layers; l++) {
        maple_moe_t L = layers[l];
        int rc;
        if (!(L->cfg_flags & MAPLE_CFG_FORCE_TC) && dec_slots(L, T)) {
            // decode batch: the routing kernel normalises the residual itself, and
            // after a decode kernel it is launched as that kernel's dependent
            rc = forward_impl(L, nullptr, T, resid, resid, nullptr, st, resid, chained);
            chained = true;
        } else {
            rmsnorm_bf16_kernel<<<(T + 7) / 8, 256, 0, st>>>(resid, T, L->D, xn);
            if ((rc = launch_status())) return rc;
            rc = forward_impl(L, xn, T, resid, resid, nullptr, st);
            chained = false;
        }
        if (rc) return rc;
    }
    return MAPLE_OK;
}

extern "C" int maple_moe_set_stage_events(maple_moe_t h, void *const *events, int32_t n_events)
{
    int rc = check_handle(h);
    if (rc) return rc;
    if (!events) {
        h->use_events = false;
        return MAPLE_OK;
    }
    if (n_events != 4) return MAPLE_ERR_INVALID_ARG;
    for (int i = 0; i < 4; i++) {
        if (!events[i]) return MAPLE_ERR_INVALID_ARG;
        h->ev[i] = (cudaEvent_t)events[i];
    }
    h->use_events = true;
    return MAPLE_OK;
}

extern "C" int maple_moe_device_flags(maple_moe_t h, uint32_t *flags, int32_t clear)
{
    int rc = check_handle(h);
    if (rc) return rc;
    if (!flags) return MAPLE_ERR_INVALID_ARG;
    *flags = clear ? __atomic_exchange_n(h->flag_host, 0u, __ATOMIC_ACQ_REL)
                   : __atomic_load_n(h->flag_host, __ATOMIC_ACQUIRE);
    if (clear && (*flags & MAPLE_DEVFLAG_TIMEOUT)) h->pending_reset = true;
    return MAPLE_OK;
}

extern "C" int maple_moe_set_debug(maple_moe_t h, int32_t wait_limit_us, uint32_t debug_flags)
{
    int rc = check_handle(h);
    if (rc) return rc;
    if (wait_limit_us < 0 || wait_limit_us > 60000000 || (debug_flags & ~(MAPLE_DEBUG_STALL_DOWN | MAPLE_DEBUG_SPLIT_SMALL))) return MAPLE_ERR_INVALID_ARG;
    h->wait_ns = wait_limit_us ? (uint64_t)wait_limit_us * 1000ull : kDefaultWaitNs;
    h->debug_flags = debug_flags;
    return MAPLE_OK;
}

extern "C" int maple_moe_expert_path(maple_moe_t h, int32_t T, int32_t *path)
{
    int rc = check_handle(h);
    if (rc) return rc;
    if (!path || T < 1 || T > h->Tm) return MAPLE_ERR_INVALID_ARG;
    const int nslot = (h->cfg_flags & MAPLE_CFG_FORCE_TC) ? 0 : dec_slots(h, T);
    if (!nslot && !h->w_tc_gu) return MAPLE_ERR_UNSUPPORTED_SHAPE;
    *path = !nslot ? MAPLE_PATH_TC : (fused_cluster(h, T) ? MAPLE_PATH_DECODE_FUSED : MAPLE_PATH_DECODE);
    return MAPLE_OK;
}

extern "C" int maple_moe_destroy(maple_moe_t h)
{
    if (!h) return MAPLE_OK;
    int rc = check_handle(h);
    if (rc) return rc;
    int status = MAPLE_OK;
    if (cudaDeviceSynchronize() != cudaSuccess) status = MAPLE_ERR_CUDA;
    if (cudaFree(h->base) != cudaSuccess) status = MAPLE_ERR_CUDA;
    if (cudaFreeHost(h->flag_host) != cudaSuccess) status = MAPLE_ERR_CUDA;
    h->magic = 0;
    delete h;
    return status;
}

// ===========================================================================
// Routing that allocates nothing.
//
// Some callers cannot let a library call cudaMalloc: processes whose device
// memory is handed out by their own pool allocator (a cudaMalloc behind the
// pool's back fragments it and can synchronise the whole device), and serving
// loops that forbid any allocation once they are running.  For them,
// maple_moe_route_noalloc runs the routing kernel with its scratch (logits,
// int8 codes, counters, permutation) in the fixed array below instead of a
// handle's workspace.  The array is a file-scope device variable: every GPU
// that loads this library holds its kNoallocScratchBytes until the process
// exits.
// ===========================================================================
namespace {

constexpr size_t kNoallocScratchBytes = (size_t)1 << 20;   // 1 MiB
constexpr int kNoallocMaxDevices = 64;

static __device__ __align__(256) unsigned char g_route_scratch[kNoallocScratchBytes];

std::mutex g_noalloc_mu;
void *g_noalloc_addr[kNoallocMaxDevices];   // device address of g_route_scratch on each device

// Once per device, with that device current: look up the device address of
// the scratch array (in host code its name is only a host-side stand-in) and
// raise the routing kernels' dynamic shared-memory limit.  Both are cached for
// the life of the process; a cudaDeviceReset invalidates them (the module is
// loaded again, at a new address), so a process that resets a device must not
// call this entry point on that device afterwards.
int noalloc_scratch(void **out)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoallocMaxDevices) {
        cudaGetLastError();
        return MAPLE_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || !p) {
            cudaGetLastError();
            return MAPLE_ERR_CUDA;
        }
        bool ok = true;
        for (int ni = 1; ni <= 16; ni *= 2) {
            ok = allow_max_smem((const void *)pick_route(ni * 256, 16), dev) && ok;
            ok = allow_max_smem((const void *)pick_route(ni * 256, 1024), dev) && ok;
        }
        if (!ok) return MAPLE_ERR_CUDA;
        g_noalloc_addr[dev] = p;
    }
    *out = g_noalloc_addr[dev];
    return MAPLE_OK;
}

}  // namespace

extern "C" int maple_moe_route_noalloc(const uint16_t *x, int32_t T, int32_t d_model, int32_t n_experts,
                                       int32_t top_k, const float *router_w, const float *router_bias,
                                       int32_t *topk_idx, float *topk_w, int32_t *expert_counts,
                                       maple_stream_t stream)
{
    maple_moe_config c;
    memset(&c, 0, sizeof c);
    c.d_model = d_model;
    c.n_experts = n_experts;
    c.top_k = top_k;
    c.d_ff = 128;
    c.max_tokens = 1;
    int rc = check_shape(&c);
    if (rc) return rc;
    if (T < 0 || T > kRouteSmallT || (int64_t)T * n_experts > kFusedMarkBytes) return MAPLE_ERR_INVALID_ARG;
    if (T == 0) return MAPLE_OK;
    if (!x || !router_w || !topk_idx || !topk_w || !aligned16(x) || !aligned16(router_w) || !aligned16(topk_idx) ||
        !aligned16(topk_w) || (router_bias && !aligned16(router_bias)) || (expert_counts && !aligned16(expert_counts)))
        return MAPLE_ERR_INVALID_ARG;

    const int64_t D = d_model, E = n_experts, S = (int64_t)T * top_k;
    Arena ar;
    const size_t o_lg = ar.take(T * E * 4), o_qx = ar.take(T * D), o_sx = ar.take(T * 4), o_sumx = ar.take(T * 4);
    const size_t o_ti = ar.take(S * 4), o_tw = ar.take(S * 4), o_cnt = ar.take(E * 4), o_off = ar.take((E + 1) * 4);
    const size_t o_perm = ar.take(S * 4), o_inv = ar.take(S * 4), o_act = ar.take(E * 4), o_nact = ar.take(4);
    const size_t o_ctr = ar.take(((kRouteSmallT + kRouteTokens - 1) / kRouteTokens + 1) * 4);
    if (ar.size > kNoallocScratchBytes) return MAPLE_ERR_INVALID_ARG;

    void *scratch = nullptr;
    if ((rc = noalloc_scratch(&scratch))) return rc;
    char *b = (char *)scratch;
    cudaStream_t st = (cudaStream_t)stream;
    // the last-arriver counters must start at zero; the array keeps whatever the last call left
    const int n_tg = (T + kRouteTokens - 1) / kRouteTokens;
    if (cudaMemsetAsync(b + o_ctr, 0, (size_t)(n_tg + 1) * 4, st) != cudaSuccess) return MAPLE_ERR_CUDA;

    RouteArgs a;
    memset(&a, 0, sizeof a);
    a.x = x;
    a.T = T;
    a.D = d_model;
    a.E = n_experts;
    a.K = top_k;
    a.Wr = router_w;
    a.bias = router_bias;
    a.qx = (int8_t *)(b + o_qx);
    a.sx = (float *)(b + o_sx);
    a.sumx = (int *)(b + o_sumx);
    a.logits = (float *)(b + o_lg);
    a.topk_idx = (int *)(b + o_ti);
    a.topk_w = (float *)(b + o_tw);
    a.out_idx = topk_idx;
    a.out_w = topk_w;
    a.out_counts = expert_counts;
    a.tg_cnt = (unsigned *)(b + o_ctr);
    a.glob_cnt = (unsigned *)(b + o_ctr) + n_tg;
    a.fuse_permute = 1;
    a.counts = (int *)(b + o_cnt);
    a.offsets = (int *)(b + o_off);
    a.perm = (int *)(b + o_perm);
    a.inv = (int *)(b + o_inv);
    a.active = (int *)(b + o_act);
    a.n_active = (int *)(b + o_nact);
    a.flag = nullptr;
    dim3 grid(n_experts / kRouteExperts, n_tg);
    pick_route(d_model, n_experts)<<<grid, 256, route_smem_bytes(d_model), st>>>(a);
    return launch_status();
}
