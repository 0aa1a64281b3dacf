// moe_api.cu -- the C ABI declared in include/moe.h: argument checks, workspace carving,
// tensor-map encoding and kernel launches. Every step of the layer runs in the kernels
// included below; this file only validates and launches.
#include "moe.h"

#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <memory>
#include <mutex>

#include "backward.cuh"
#include "combine.cuh"
#include "dispatch.cuh"
#include "ep.cuh"
#include "fp8.cuh"
#include "fused.cuh"
#include "route_chain.cuh"
#include "gemm_tc.cuh"
#include "ptx.cuh"
#include "route.cuh"
#include "route_filter.cuh"
#include "gemm_narrow.cuh"

namespace {

using namespace moe;

constexpr int64_t kDefaultTimeoutNs = 2000000000LL;
std::atomic<int64_t> g_timeout_ns{kDefaultTimeoutNs};
// grouped GEMM variant: MOE_GEMM_AUTO / MOE_GEMM_SINGLE_CTA / MOE_GEMM_CTA_PAIR
std::atomic<int> g_gemm_mode{MOE_GEMM_AUTO};
// test hook: layer0 work item of the fused kernel whose ready signal is withheld (-1: none)
std::atomic<int> g_fault_skip{-1};
// router variant for many experts: MOE_ROUTER_AUTO (tensor-core filter) or sequential only
std::atomic<int> g_router_mode{MOE_ROUTER_AUTO};
// optional schedule trace of the fused launch (device buffer and its record capacity)
std::atomic<unsigned long long *> g_trace{nullptr};
std::atomic<int64_t> g_trace_cap{0};
// grouped-GEMM work order (MOE_ORDER_*; test and tuning hook)
std::atomic<int> g_order{MOE_ORDER_NARROW};
// whole-layer launch (routing and dispatch inside the persistent launch) where it applies
std::atomic<int> g_front{1};

// ---------------------------------------------------------------------------------------
// problem checks and workspace layout
// ---------------------------------------------------------------------------------------

moe_status check_problem(const moe_problem *p)
{
    if (p == nullptr) return MOE_ERR_INVALID_ARG;
    if (p->T < 0 || p->H <= 0 || p->F <= 0 || p->E <= 0 || p->top_k <= 0) return MOE_ERR_INVALID_ARG;
    if (p->top_k > p->E) return MOE_ERR_INVALID_ARG;
    if (p->act < MOE_ACT_SWIGLU || p->act > MOE_ACT_IDENTITY) return MOE_ERR_INVALID_ARG;
    if (p->gate != MOE_GATE_SOFTMAX_TOPK && p->gate != MOE_GATE_SOFTMAX_ALL &&
        p->gate != MOE_GATE_SELECT_BIAS)
        return MOE_ERR_INVALID_ARG;
    if (p->m_tile != M_TILE) return MOE_ERR_UNSUPPORTED;
    if (p->H % 64 != 0 || p->F % 64 != 0) return MOE_ERR_UNSUPPORTED;
    if (p->E > 1024) return MOE_ERR_UNSUPPORTED;
    // 32-bit row indices and element offsets inside one expert block
    const int64_t pmax = (int64_t)p->T * p->top_k + (int64_t)p->E * (M_TILE - 1);
    if (pmax >= (1LL << 31) - M_TILE) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

int64_t padded_rows_max(const moe_problem *p)
{
    const int64_t tk = (int64_t)p->T * p->top_k;
    const int64_t nonempty = tk < p->E ? tk : p->E;
    return tk + nonempty * (M_TILE - 1);
}

size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

struct Layout {
    size_t status, meta, logits, wgt, wnorm, xsq, topk_idx, topk_w, chunk,
        counts, offsets, poff, tile_off, gcount,
        tile_expert, ptile_off, ptile_expert, hot_off, hot_tile_expert, cold_tile, ready,
        gather_idx, inv_pos, row_w, x_perm, h, ys,
        x_stage, out_stage, x_stage2, out_stage2, sh_gate, sh_h, sh_ys, xq, sx, hq, sh,
        bgu, ba, bdxp, bdw, bdl, bact;
    size_t end_route, end_dispatch, end_forward, end_host, end_shared, end_fp8, end_bwd;
    int64_t pmax;
    int nchunk, max_tiles, n_ready;
};

// Tensor-core filter router (route_filter.cuh): applicable shapes and launch plan. The plan
// depends on the problem only, so the workspace size does not depend on the device.
struct FilterPlan {
    bool ok;
    int split;      // K ranges of the filter GEMM (fp32 partials [split, E, T])
    int bt;         // tokens per block of the exact kernel
    int ring_bytes; // its chunk ring
    size_t smem;    // its dynamic shared memory
    float cA;       // interval coefficient
};

FilterPlan filter_plan(const moe_problem *p)
{
    FilterPlan f{false, 1, 0, 0, 0, 0.0f};
    const int T = p->T, H = p->H, E = p->E;
    if (T <= 0 || E < 8 || E > RF_MAX_E || (E % 8) != 0 || (H % gemm::BK) != 0 ||
        p->gate == MOE_GATE_SOFTMAX_ALL || (int64_t)T * E >= (1LL << 31) / RF_SPLIT_MAX)
        return f;
    const int kb = H / gemm::BK;
    const int tiles = ((T + gemm::BM - 1) / gemm::BM) * ((E + gemm::BN - 1) / gemm::BN);
    int split = 148 / tiles; // about one wave of filter-GEMM CTAs on a 148-SM part
    const int smax = kb < RF_SPLIT_MAX ? kb : RF_SPLIT_MAX;
    if (split > smax) split = smax;
    if (split < 1) split = 1;
    // tokens per block: whole waves of RF_BLOCKS_PER_SM blocks per SM on a 148-SM part (the
    // latency-bound selection phases of one block overlap another's stream), at most
    // RF_MAX_BT tokens each
    const int slots = 148 * RF_BLOCKS_PER_SM;
    const int waves = (T + slots * RF_MAX_BT - 1) / (slots * RF_MAX_BT);
    int bt = (T + slots * waves - 1) / (slots * waves);
    if (bt < 1) bt = 1;
    // ring: as deep as the blocks that share an SM leave room for (1 KB per block is reserved)
    const int blocks = (T + bt - 1) / bt;
    int per_sm = (blocks + 147) / 148;
    if (per_sm > 4) per_sm = 4;
    int ring = 0;
    for (; per_sm >= 1; --per_sm) {
        const int budget = RF_SMEM_MAX / per_sm - 1024;
        ring = budget - (int)rf_smem_bytes(bt, E, 0);
        if (ring >= rf_ring_min(bt, E)) break;
    }
    if (per_sm < 1 || rf_smem_bytes(bt, E, ring) > (size_t)RF_SMEM_MAX) return f;
    const int hs = ((kb + split - 1) / split) * gemm::BK; // longest K range
    f.ok = true;
    f.split = split;
    f.bt = bt;
    f.ring_bytes = ring;
    f.smem = rf_smem_bytes(bt, E, ring);
    f.cA = (float)(1.25 * ((double)H + 4.0 * hs + split + 4.0) * 5.9604644775390625e-8);
    return f;
}

Layout make_layout(const moe_problem *p, int F_s = 0, bool fp8 = false, bool bwd = false,
                   bool no_rows = false)
{
    Layout L{};
    const size_t T = (size_t)p->T, H = (size_t)p->H, F = (size_t)p->F, E = (size_t)p->E,
                 K = (size_t)p->top_k;
    L.pmax = padded_rows_max(p);
    const size_t P = (size_t)L.pmax;
    L.nchunk = (int)((T + DISPATCH_CHUNK - 1) / DISPATCH_CHUNK);
    L.max_tiles = (int)(P / M_TILE) + 1;
    size_t o = 0;
    auto take = [&](size_t bytes) {
        const size_t at = o;
        o = align256(o + (bytes ? bytes : 1));
        return at;
    };
    L.status = take(256);
    L.meta = take(sizeof(DispatchMeta));
    // router logits; the filter router keeps its GEMM partials [split, T, E] here
    const FilterPlan fp = filter_plan(p);
    L.logits = take(T * E * 4 * (size_t)(fp.ok ? fp.split : 1));
    L.wgt = take(fp.ok ? E * H * 2 : 0); // filter router: W_g^T
    L.wnorm = take(fp.ok ? (H + RF_SLAB - 1) / RF_SLAB * E * 4 : 0); // W_g column sums of squares
    L.xsq = take(fp.ok ? (size_t)fp.split * T * 4 : 0);              // x row sums of squares
    L.end_route = o;
    L.topk_idx = take(T * K * 4);
    L.topk_w = take(T * K * 4);
    L.chunk = take((size_t)L.nchunk * E * 4);
    // whole-layer launch: selections per group of at least 8 tokens and expert
    L.gcount = take((T + 7) / 8 * E * 4);
    L.counts = take(E * 4);
    L.offsets = take((E + 1) * 4);
    L.poff = take((E + 1) * 4);
    L.tile_off = take((E + 1) * 4);
    L.tile_expert = take((size_t)L.max_tiles * 4);
    L.ptile_off = take((E + 1) * 4);
    L.ptile_expert = take((size_t)L.max_tiles * 4);
    L.hot_off = take((E + 1) * 4);
    L.hot_tile_expert = take((size_t)L.max_tiles * 4);
    L.cold_tile = take(E * 4);
    // fused kernel: a counter per M tile (layer0), a flag per (stripe, M tile) (layer1), the
    // count of finished layer0 items and the combine queue's next item
    L.n_ready = L.max_tiles * (1 + (int)((H + 255) / 256)) + 2;
    L.ready = take((size_t)L.n_ready * 4);
    L.gather_idx = take(P * 4);
    L.inv_pos = take(T * K * 4);
    L.row_w = take(P * 4);
    L.end_dispatch = o;
    // materialised gather (large batches, the CTA-pair GEMM variant); no_rows: the rows live
    // elsewhere (the expert-parallel layer's receive buffer) and layer1 writes no ys
    L.x_perm = take(no_rows ? 0 : P * H * 2);
    L.h = take(P * F * 2);
    L.ys = take(no_rows ? 0 : P * H * 2);
    L.end_forward = o;
    L.x_stage = take(T * H * 2);
    L.out_stage = take(T * H * 2);
    L.x_stage2 = take(T * H * 2); // second staging pair: moe_forward_host_batches
    L.out_stage2 = take(T * H * 2);
    L.end_host = o;
    // shared expert (moe_forward_shared): gate, h_s and ys_s over T rounded up to 128 rows
    const size_t Tpad = (T + M_TILE - 1) / M_TILE * M_TILE;
    L.sh_gate = take(F_s > 0 ? Tpad * 4 : 0);
    L.sh_h = take(F_s > 0 ? Tpad * (size_t)F_s * 2 : 0);
    L.sh_ys = take(F_s > 0 ? Tpad * H * 2 : 0);
    L.end_shared = o;
    // FP8 experts (moe_forward_fp8): e4m3 codes of x and h with their row scales
    L.xq = take(fp8 ? T * H : 0);
    L.sx = take(fp8 ? T * 4 : 0);
    L.hq = take(fp8 ? P * F : 0);
    L.sh = take(fp8 ? P * 4 : 0);
    L.end_fp8 = o;
    // backward (moe_backward): recomputed pre-activations, overwritten by their gradient;
    // hidden activations; the expert rows' input gradients; per-row gate and logit gradients
    const size_t w1c = p->act == MOE_ACT_SWIGLU ? 2 * F : F;
    L.bgu = take(bwd ? P * w1c * 2 : 0);
    L.ba = take(bwd ? P * F * 2 : 0);
    L.bdxp = take(bwd ? P * H * 2 : 0);
    L.bdw = take(bwd ? P * 4 : 0);
    L.bdl = take(bwd ? P * 4 : 0);
    L.bact = take(bwd ? E * 4 : 0);
    L.end_bwd = o;
    return L;
}

template <typename T> T *at(void *ws, size_t off)
{
    return reinterpret_cast<T *>(static_cast<char *>(ws) + off);
}

struct FilterBufs;
FilterBufs filter_bufs(void *ws, const Layout &L);

bool aligned16(const void *ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }
bool aligned4(const void *ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 3u) == 0; }

// ---------------------------------------------------------------------------------------
// device properties and tensor maps
// ---------------------------------------------------------------------------------------

int sm_count()
{
    static std::atomic<int> cache[64]; // per device; 0 = not yet queried (static: zeroed)
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (dev < 0 || dev >= 64) return 0;
    int n = cache[dev].load(std::memory_order_relaxed);
    if (n == 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
        cache[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault,
                                             &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

// 2D bf16 row-major [rows, cols]; box = 64 columns x box_rows rows, 128-byte swizzle.
bool make_map_2d(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols, uint32_t box_rows)
{
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2D bf16 row-major [rows, cols] without swizzle; box = box_cols x box_rows (box_cols * 2 a
// multiple of 16 bytes).
bool make_map_2d_plain(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols,
                       uint32_t box_cols, uint32_t box_rows)
{
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3D bf16 [depth, rows, cols]; box = 64 columns x box_rows rows x 1, 128-byte swizzle.
bool make_map_3d(CUtensorMap *m, const void *base, uint64_t depth, uint64_t rows, uint64_t cols,
                 uint32_t box_rows = 64)
{
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr) return false;
    cuuint64_t dims[3] = {cols, rows, depth};
    cuuint64_t strides[2] = {cols * 2, rows * cols * 2};
    cuuint32_t box[3] = {64, box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2D uint8 [rows, cols] (e4m3 codes); box = 128 bytes x box_rows rows, 128-byte swizzle.
bool make_map_2d_u8(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols, uint32_t box_rows)
{
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols};
    cuuint32_t box[2] = {128, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3D uint8 [depth, rows, cols] (per-expert e4m3 code matrices, K contiguous);
// box = 128 bytes x box_rows rows x 1, 128-byte swizzle.
bool make_map_3d_u8(CUtensorMap *m, const void *base, uint64_t depth, uint64_t rows, uint64_t cols,
                    uint32_t box_rows = gemm::B8_BOX_ROWS)
{
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr) return false;
    cuuint64_t dims[3] = {cols, rows, depth};
    cuuint64_t strides[2] = {cols, rows * cols};
    cuuint32_t box[3] = {128, box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int KIND> cudaError_t gemm_smem_attr()
{
    // set once per process and device; cheap to repeat
    return cudaFuncSetAttribute(moe_grouped_gemm_kernel<KIND>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, gemm::SMEM_BYTES);
}

// ---------------------------------------------------------------------------------------
// stage launchers (no argument checks; callers validated)
// ---------------------------------------------------------------------------------------

template <int BT, int BE, int RT, int RE, int HC, int NS>
void launch_route_logits(const __nv_bfloat16 *x, const __nv_bfloat16 *Wg, const float *bias,
                         float *logits, int T, int H, int E, int *status, cudaStream_t st)
{
    constexpr int smem = RouteSmem<BT, BE, HC, NS>::BYTES;
    auto kern = route_logits_kernel<BT, BE, RT, RE, HC, NS>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    dim3 grid((T + BT - 1) / BT, (E + BE - 1) / BE), block(BE / RE, BT / RT);
    kern<<<grid, block, smem, st>>>(x, Wg, bias, logits, T, H, E, status);
}

// Buffers of the tensor-core filter router (inside the caller's workspace).
struct FilterBufs {
    uint16_t *wgt;
    float *wnorm;
    float *xsq;
};

template <int KIND>
cudaError_t launch_gemm(const CUtensorMap &ta, const CUtensorMap &tb, const GemmArgs &args,
                        int max_work, cudaStream_t st);
bool make_map_2d(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols, uint32_t box_rows);
bool make_map_3d(CUtensorMap *m, const void *base, uint64_t depth, uint64_t rows, uint64_t cols,
                 uint32_t box_rows);

FilterBufs filter_bufs(void *ws, const Layout &L)
{
    FilterBufs f;
    f.wgt = at<uint16_t>(ws, L.wgt);
    f.wnorm = at<float>(ws, L.wnorm);
    f.xsq = at<float>(ws, L.xsq);
    return f;
}

// Exact top-k for many experts: tensor-core filter logits, rigorous intervals, exact
// sequential recomputation of the candidates only (route_filter.cuh). Three launches.
cudaError_t launch_route_filter(const moe_problem *p, const FilterPlan &fp,
                                const __nv_bfloat16 *xb, const __nv_bfloat16 *wb,
                                const float *bias, int32_t *topk_idx, float *topk_w,
                                float *parts, const FilterBufs &fb, int *status, cudaStream_t st)
{
    const int T = p->T, H = p->H, E = p->E;
    route_filter_prep_kernel<<<dim3(E / 8, (H + RF_SLAB - 1) / RF_SLAB), 256, 0, st>>>(
        wb, H, E, fb.wgt, fb.wnorm, status);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    CUtensorMap mx, mw;
    if (!make_map_2d(&mx, xb, (uint64_t)T, (uint64_t)H, gemm::BM) ||
        !make_map_3d(&mw, wb, 1, (uint64_t)H, (uint64_t)E))
        return cudaErrorInvalidValue;
    GemmArgs a{};
    a.dense_m_tiles = (T + gemm::BM - 1) / gemm::BM;
    a.dense_rows = T;
    a.k_split = fp.split;
    a.n_tiles = (E + gemm::BN - 1) / gemm::BN;
    a.n_boxes = E <= gemm::BN ? (E + 63) / 64 : 4;
    a.k_blocks = H / gemm::BK;
    a.out_f32 = parts;
    a.xsq_f32 = fb.xsq;
    a.ld_out = E;
    a.n_cols = E;
    a.status = status;
    a.timeout_ns = g_timeout_ns.load();
    err = launch_gemm<GEMM_LOGITS>(mx, mw, a, a.dense_m_tiles * a.n_tiles * fp.split, st);
    if (err != cudaSuccess) return err;
    CUtensorMap mxs, mws; // the exact kernel's streams: bt rows of x, 64 rows of W_g^T per box
    if (!make_map_2d(&mxs, xb, (uint64_t)T, (uint64_t)H, (uint32_t)fp.bt) ||
        !make_map_2d(&mws, fb.wgt, (uint64_t)E, (uint64_t)H, RF_WBOX))
        return cudaErrorInvalidValue;
    RfArgs r{};
    r.wpart = fb.wnorm;
    r.xsq = fb.xsq;
    r.bias = bias;
    r.parts = parts;
    r.topk_idx = topk_idx;
    r.topk_w = topk_w;
    r.T = T;
    r.H = H;
    r.E = E;
    r.k = p->top_k;
    r.S = fp.split;
    r.bt = fp.bt;
    r.ring_bytes = fp.ring_bytes;
    r.cA = fp.cA;
    r.gate = p->gate;
    r.status = status;
    r.timeout_ns = g_timeout_ns.load();
    const size_t smem = fp.smem;
    err = cudaFuncSetAttribute(route_filter_exact_kernel,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    route_filter_exact_kernel<<<(T + fp.bt - 1) / fp.bt, RF_THREADS, smem, st>>>(mxs, mws, r);
    return cudaGetLastError();
}

// The one-launch router for up to 32 experts (route_chain.cuh): E a multiple of 8 (whole
// 16-byte W_g rows for its TMA boxes).
bool route_uses_chain(const moe_problem *p)
{
    return p->E % 8 == 0 && p->E <= 32 && p->H % 64 == 0;
}

template <int EPT, int G>
cudaError_t launch_route_chain_t(const moe_problem *p, const __nv_bfloat16 *x,
                                 const __nv_bfloat16 *Wg, const float *bias, int32_t *topk_idx,
                                 float *topk_w, int *status, cudaStream_t st)
{
    const int T = p->T, H = p->H, E = p->E;
    const int sms = sm_count() > 0 ? sm_count() : 148;
    // about one CTA per SM: tt tokens each (at most 256 box rows, RC_MAX_CONSUMERS threads)
    int tt = (T + sms - 1) / sms;
    tt = std::max(1, std::min(tt, std::min(256, RC_MAX_CONSUMERS / G)));
    const int ncw = (tt * G + 31) / 32;
    int stages = RC_MAX_STAGES;
    RcLayout L = rc_layout(tt, E, EPT * G, stages);
    while (stages > 3 && L.total + 1024 > RC_SMEM_BUDGET) {
        --stages;
        L = rc_layout(tt, E, EPT * G, stages);
    }
    const int smem = L.total + 1024;
    if (smem > 227 * 1024) return cudaErrorInvalidValue;
    CUtensorMap mx, mw;
    if (!make_map_2d(&mx, x, (uint64_t)T, (uint64_t)H, (uint32_t)tt) ||
        !make_map_2d_plain(&mw, Wg, (uint64_t)H, (uint64_t)E, (uint32_t)E, RC_HC))
        return cudaErrorInvalidValue;
    RcArgs a{};
    a.bias = bias;
    a.topk_idx = topk_idx;
    a.topk_w = topk_w;
    a.T = T;
    a.H = H;
    a.E = E;
    a.k = p->top_k;
    a.gate = p->gate;
    a.tt = tt;
    a.stages = stages;
    a.status = status;
    a.timeout_ns = g_timeout_ns.load();
    auto kern = route_chain_kernel<EPT, G>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    kern<<<(T + tt - 1) / tt, 32 + ncw * 32, smem, st>>>(mx, mw, a);
    return cudaGetLastError();
}

cudaError_t launch_route_chain(const moe_problem *p, const __nv_bfloat16 *x, const __nv_bfloat16 *Wg,
                               const float *bias, int32_t *topk_idx, float *topk_w, int *status,
                               cudaStream_t st)
{
    if (p->E <= 8) return launch_route_chain_t<4, 2>(p, x, Wg, bias, topk_idx, topk_w, status, st);
    if (p->E <= 16) return launch_route_chain_t<4, 4>(p, x, Wg, bias, topk_idx, topk_w, status, st);
    return launch_route_chain_t<4, 8>(p, x, Wg, bias, topk_idx, topk_w, status, st);
}

// Router choice for AUTO / FILTER / SEQUENTIAL (operands assumed 16-byte aligned).
bool route_uses_filter(const moe_problem *p)
{
    const int mode = g_router_mode.load();
    // AUTO takes the filter from 16 experts and 2^16 logits on (below, its fixed costs -- the
    // W_g transpose, the GEMM and one chain of H dependent FMAs per candidate -- outweigh the
    // savings: measured slower on the Mixtral-shaped E = 8 router and the T = 64 decode one)
    const bool want = mode == MOE_ROUTER_FILTER ||
                      (mode == MOE_ROUTER_AUTO && p->E >= 16 && (int64_t)p->T * p->E >= (1 << 16));
    return want && filter_plan(p).ok;
}

cudaError_t launch_route(const moe_problem *p, const moe_bf16 *x, const moe_bf16 *Wg,
                         const float *bias, int32_t *topk_idx, float *topk_w, float *logits,
                         int *status, cudaStream_t st, const FilterBufs *filter = nullptr)
{
    const int T = p->T, H = p->H, E = p->E;
    const auto *xb = reinterpret_cast<const __nv_bfloat16 *>(x);
    const auto *wb = reinterpret_cast<const __nv_bfloat16 *>(Wg);
    // many experts: tensor-core filter plus exact recomputation of the candidates (needs the
    // workspace buffers, W_g rows that TMA can address, and the top-k renormalised gates)
    if (filter != nullptr && aligned16(x) && aligned16(Wg) && route_uses_filter(p))
        return launch_route_filter(p, filter_plan(p), xb, wb, bias, topk_idx, topk_w, logits,
                                   *filter, status, st);
    // up to 32 experts: logits and top-k in one launch, no logits buffer
    if (aligned16(x) && aligned16(Wg) && route_uses_chain(p))
        return launch_route_chain(p, xb, wb, bias, topk_idx, topk_w, status, st);
    // blocks of the large-E tile (64 tokens x 64 experts); fewer than the SMs: go narrow
    const int64_t large_blocks = (int64_t)((T + 63) / 64) * ((E + 63) / 64);
    const int sms = sm_count() > 0 ? sm_count() : 148;
    // selection bias: the logits stay without it, the top-k kernel adds it to the keys
    const float *lbias = (p->gate == MOE_GATE_SELECT_BIAS) ? nullptr : bias;
    if (E <= 8 && T >= 64 * sms / 2) {
        launch_route_logits<ROUTE_SMALL_CFG>(xb, wb, lbias, logits, T, H, E, status, st);
    } else if (E > 8 && E <= 16 && T >= 32 * sms / 2) {
        launch_route_logits<ROUTE_MID_CFG>(xb, wb, lbias, logits, T, H, E, status, st);
    } else if (E > 16 && large_blocks >= sms / 2) {
        launch_route_logits<ROUTE_LARGE_CFG>(xb, wb, lbias, logits, T, H, E, status, st);
    } else if ((int64_t)((T + 7) / 8) * ((E + 15) / 16) <= sms) {
        launch_route_logits<ROUTE_NARROW_CFG>(xb, wb, lbias, logits, T, H, E, status, st);
    } else {
        launch_route_logits<ROUTE_NARROW2_CFG>(xb, wb, lbias, logits, T, H, E, status, st);
    }
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    const size_t smem = (size_t)TOPK_WARPS * E * sizeof(float);
    route_topk_kernel<<<(T + TOPK_WARPS - 1) / TOPK_WARPS, TOPK_WARPS * 32, smem, st>>>(
        logits, topk_idx, topk_w, T, E, p->top_k, p->gate, bias);
    return cudaGetLastError();
}

struct DispatchOut {
    int32_t *counts, *offsets, *poff, *gather_idx, *inv_pos, *tile_off, *tile_expert, *chunk;
    int32_t *ptile_off, *ptile_expert;
    int32_t *hot_off, *hot_tile_expert, *cold_tile;
    int32_t *active_list = nullptr; // experts with rows, ascending (moe_backward)
    int *ready;
    int n_ready;
    float *row_w;
    DispatchMeta *meta;
};

// The scan step's outputs in the workspace.
ScanOut scan_out(const Layout &L, const DispatchOut &o)
{
    ScanOut so{};
    so.counts = o.counts;
    so.offsets = o.offsets;
    so.padded_offsets = o.poff;
    so.tile_off = o.tile_off;
    so.tile_expert = o.tile_expert;
    so.ptile_off = o.ptile_off;
    so.ptile_expert = o.ptile_expert;
    so.meta = o.meta;
    so.gather_idx = o.gather_idx;
    so.row_w = o.row_w;
    so.padded_rows_max = L.pmax;
    so.ready = o.ready;
    so.n_ready = o.ready ? o.n_ready : 0;
    so.hot_off = o.hot_off;
    so.hot_tile_expert = o.hot_tile_expert;
    so.cold_tile = o.cold_tile;
    so.active_list = o.active_list;
    return so;
}

cudaError_t launch_dispatch(const moe_problem *p, const Layout &L, const int32_t *topk_idx,
                            const float *topk_w, const DispatchOut &o, int *status, int clear_status,
                            cudaStream_t st, const int32_t *n_rows = nullptr)
{
    const int T = p->T, E = p->E, k = p->top_k;
    const int nchunk = L.nchunk;
    const ScanOut so = scan_out(L, o);
    if (nchunk == 1) { // one chunk of tokens: the three steps in one block
        dispatch_small_kernel<<<1, 1024, (size_t)E * (DISPATCH_WORDS + 1) * 4, st>>>(
            topk_idx, topk_w, T, E, k, so, o.inv_pos, status, clear_status, n_rows);
        return cudaGetLastError();
    }
    cudaError_t err = cudaSuccess;
    if (clear_status && status != nullptr && nchunk > 1) {
        // cleared before any block can record a bad id (blocks of one launch are unordered)
        err = cudaMemsetAsync(status, 0, 8, st);
        if (err != cudaSuccess) return err;
        clear_status = 0;
    }
    if (nchunk > 0) {
        dispatch_count_kernel<<<nchunk, DISPATCH_CHUNK, E * sizeof(int), st>>>(
            topk_idx, T, E, k, o.chunk, status, clear_status, n_rows);
    }
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    dispatch_scan_kernel<<<1, 1024, 0, st>>>(o.chunk, nchunk, E, so);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    if (nchunk > 0) {
        dispatch_place_kernel<<<nchunk, DISPATCH_CHUNK, (size_t)E * DISPATCH_WORDS * 4, st>>>(
            topk_idx, topk_w, T, E, k, o.chunk, o.poff, o.gather_idx, o.inv_pos, o.row_w, n_rows);
    }
    return cudaGetLastError();
}

cudaError_t launch_gather(const moe_problem *p, const moe_bf16 *x, const int32_t *gather_idx,
                          const DispatchMeta *meta, moe_bf16 *x_perm, cudaStream_t st)
{
    const int blocks = sm_count() * 8;
    gather_rows_kernel<<<blocks > 0 ? blocks : 1024, 256, 0, st>>>(
        reinterpret_cast<const __nv_bfloat16 *>(x), gather_idx, meta, p->T, p->H,
        reinterpret_cast<__nv_bfloat16 *>(x_perm));
    return cudaGetLastError();
}

cudaError_t launch_combine(const moe_problem *p, const moe_bf16 *ys, int64_t ys_rows,
                           const int32_t *inv_pos, moe_bf16 *out, int *status, int clear_status,
                           cudaStream_t st, const moe_bf16 *ys_shared = nullptr,
                           const int32_t *n_rows = nullptr)
{
    const int64_t vecs = (int64_t)p->T * (p->H / 8);
    int64_t blocks = (vecs + 255) / 256;
    const int64_t cap = (int64_t)(sm_count() > 0 ? sm_count() : 148) * 16;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    // a grid that does not fill the GPU twice over: every thread issues all k row loads at
    // once; large grids: four row loads in flight per thread for k >= 4 (Qwen2-shaped and
    // skewed layers, k = 8: 113 -> 101 us, 0.80 of the measured HBM copy bandwidth; eight
    // rows: 110 us), two for smaller k
    auto kern = (blocks < 2 * cap / 16 && p->top_k > 2) ? combine_kernel<8>
                : p->top_k >= 4                         ? combine_kernel<4>
                                                        : combine_kernel<2>;
    kern<<<(int)blocks, 256, 0, st>>>(reinterpret_cast<const __nv_bfloat16 *>(ys), ys_rows, inv_pos,
                                      p->T, p->H, p->top_k, reinterpret_cast<__nv_bfloat16 *>(out),
                                      status, clear_status,
                                      reinterpret_cast<const __nv_bfloat16 *>(ys_shared), n_rows);
    return cudaGetLastError();
}

template <int KIND>
cudaError_t launch_gemm(const CUtensorMap &ta, const CUtensorMap &tb, const GemmArgs &args,
                        int max_work, cudaStream_t st)
{
    cudaError_t err = gemm_smem_attr<KIND>();
    if (err != cudaSuccess) return err;
    int grid = sm_count();
    if (grid <= 0) grid = 148;
    if (grid > max_work) grid = max_work;
    if (grid < 1) grid = 1;
    const int threads = args.gather_idx != nullptr ? gemm::NUM_THREADS_GATHER : gemm::NUM_THREADS;
    moe_grouped_gemm_kernel<KIND><<<grid, threads, gemm::SMEM_BYTES, st>>>(ta, tb, args);
    return cudaGetLastError();
}

// e4m3 layer GEMM: one launch whose CTAs run the narrow (operand-swapped) body when every
// expert owns a single m-tile, the 128-row body otherwise (decided on the device).
template <int KIND>
cudaError_t launch_gemm_select_f8(const CUtensorMap &ta, const CUtensorMap &tb,
                                  const CUtensorMap &twn, const GemmArgs &wide,
                                  const GemmArgs &narrow, cudaStream_t st)
{
    constexpr int smem = gemm::SMEM_BYTES > gemmn::SMEM_BYTES ? gemm::SMEM_BYTES : gemmn::SMEM_BYTES;
    auto kern = moe_grouped_gemm_select_f8_kernel<KIND>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess) return err;
    int grid = sm_count();
    if (grid <= 0) grid = 148;
    const int threads = (wide.gather_idx != nullptr || wide.epi8) ? gemm::NUM_THREADS_GATHER
                                                                   : gemm::NUM_THREADS;
    kern<<<grid, threads, smem, st>>>(ta, tb, twn, wide, narrow);
    return cudaGetLastError();
}

cudaError_t launch_quant_rows(const moe_bf16 *src, int64_t rows, int cols, const DispatchMeta *meta,
                              uint8_t *dst, float *scale, cudaStream_t st)
{
    if (rows <= 0) return cudaSuccess;
    int grid = sm_count() * 8;
    if (grid <= 0) grid = 1184;
    if ((int64_t)grid > rows) grid = (int)rows;
    quant_rows_fp8_kernel<<<grid, Q_THREADS, 0, st>>>(reinterpret_cast<const __nv_bfloat16 *>(src),
                                                      rows, cols, meta, M_TILE, dst, scale);
    return cudaGetLastError();
}

// W [E, K, N] -> Wq [E, N, K] codes and per-column scales [E, N]
cudaError_t launch_quant_cols(const moe_bf16 *W, int E, int K, int N, uint8_t *Wq, float *scale,
                              cudaStream_t st)
{
    const __nv_bfloat16 *w = reinterpret_cast<const __nv_bfloat16 *>(W);
    quant_cols_amax_kernel<<<dim3((N + 127) / 128, E), 256, 0, st>>>(w, K, N, scale);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    quant_cols_codes_kernel<<<dim3(N / 64, K / 64, E), 256, 0, st>>>(w, K, N, scale, Wq);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int64_t n = (int64_t)E * N;
    quant_cols_scale_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(scale, n);
    return cudaGetLastError();
}

template <int KIND, bool F8 = false>
cudaError_t launch_gemm_pair(const CUtensorMap &ta, const CUtensorMap &tb, const GemmArgs &args,
                             int max_work, cudaStream_t st)
{
    auto kern = moe_grouped_gemm_pair_kernel<KIND, F8>;
    cudaError_t err =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, gemm2::SMEM_BYTES);
    if (err != cudaSuccess) return err;
    // persistent grid: as many CTA pairs as can be resident at once (one CTA per SM)
    // per device and kind (the e4m3 form has the same block size and shared memory); 0 = not
    // yet queried
    static std::atomic<int> cache[64][3];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    int pairs = cache[dev][KIND].load(std::memory_order_relaxed);
    if (pairs == 0) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)(2 * (sm_count() / 2)), 1, 1);
        cfg.blockDim = dim3(gemm::NUM_THREADS, 1, 1);
        cfg.dynamicSmemBytes = gemm2::SMEM_BYTES;
        int n = 0;
        err = cudaOccupancyMaxActiveClusters(&n, (const void *)kern, &cfg);
        if (err != cudaSuccess) return err;
        pairs = n > 0 ? n : 1;
        cache[dev][KIND].store(pairs, std::memory_order_relaxed);
    }
    int npairs = pairs;
    if (npairs > max_work) npairs = max_work;
    if (npairs < 1) npairs = 1;
    kern<<<2 * npairs, gemm::NUM_THREADS, gemm2::SMEM_BYTES, st>>>(ta, tb, args);
    return cudaGetLastError();
}

// One launch per layer; the device picks the narrow body when every expert owns a single
// m-tile (moe_grouped_gemm_select_kernel).
constexpr int SELECT_SMEM = gemm::SMEM_BYTES > gemmn::SMEM_BYTES ? gemm::SMEM_BYTES : gemmn::SMEM_BYTES;
template <int KIND>
cudaError_t launch_gemm_select(const CUtensorMap &ta, const CUtensorMap &tb, const GemmArgs &wide,
                               const GemmArgs &narrow, cudaStream_t st)
{
    auto kern = moe_grouped_gemm_select_kernel<KIND>;
    cudaError_t err =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SELECT_SMEM);
    if (err != cudaSuccess) return err;
    int grid = sm_count();
    if (grid <= 0) grid = 148;
    const int threads = (wide.gather_idx != nullptr || wide.epi8) ? gemm::NUM_THREADS_GATHER
                                                                   : gemm::NUM_THREADS;
    kern<<<grid, threads, SELECT_SMEM, st>>>(ta, tb, wide, narrow);
    return cudaGetLastError();
}

template <int KIND>
cudaError_t launch_gemm_any(const CUtensorMap &ta, const CUtensorMap &tb, const GemmArgs &args,
                            int max_work, cudaStream_t st)
{
    // AUTO = single CTA: under the sustained 1 kW power cap the pair variant keeps the tensor
    // pipe busier per clock but draws more power per clock, and measured ~4% slower overall
    if (g_gemm_mode.load() == MOE_GEMM_CTA_PAIR) return launch_gemm_pair<KIND>(ta, tb, args, max_work, st);
    return launch_gemm<KIND>(ta, tb, args, max_work, st);
}

template <int KIND0, bool FRONT>
cudaError_t launch_fused(const CUtensorMap &a0, const CUtensorMap &w1, const CUtensorMap &hm,
                         const CUtensorMap &w2, const CUtensorMap &rx, const CUtensorMap &rw,
                         const FusedArgs &fa, int max_work, cudaStream_t st)
{
    auto kern = moe_fused_layer_kernel<KIND0, FRONT>;
    cudaError_t err =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, gemm::SMEM_BYTES);
    if (err != cudaSuccess) return err;
    // every CTA must be resident at once (the ready-flag waits rely on it): one per SM
    int grid = sm_count();
    if (grid <= 0) grid = 148;
    if (!FRONT && grid > max_work) grid = max_work; // (the whole-layer launch: one CTA per SM)
    if (grid < 1) grid = 1;
    kern<<<grid, gemm::NUM_THREADS_GATHER, gemm::SMEM_BYTES, st>>>(a0, w1, hm, w2, rx, rw, fa);
    return cudaGetLastError();
}

// Whole-layer launch (routing and dispatch inside the persistent launch): the routing's token
// groups and ring for one CTA per SM. `ok` is false where the shape does not fit it.
struct FrontPlan {
    bool ok;
    int grid, tt, n_groups, ncw, stages;
};

FrontPlan front_plan(const moe_problem *p)
{
    FrontPlan f{};
    const int sms = sm_count() > 0 ? sm_count() : 148;
    f.grid = sms;
    // tokens per group: about one group per SM, at most 128 (two consumer threads per token
    // on the eight non-GEMM-issuing warps), at least 8 (the per-group count buffer)
    f.tt = std::max(8, std::min(128, (p->T + sms - 1) / sms));
    f.n_groups = (p->T + f.tt - 1) / f.tt;
    f.ncw = (f.tt * 2 + 31) / 32;
    const int budget = gemm::STAGES * gemm::STAGE; // the GEMM stages' shared memory
    f.stages = RC_MAX_STAGES;
    while (f.stages > 3 && rc_layout(f.tt, p->E, 8, f.stages).total > budget) --f.stages;
    f.ok = p->E == 8 && rc_layout(f.tt, p->E, 8, f.stages).total <= budget &&
           (int64_t)front_scratch_ints(f.n_groups, p->E) * 4 <= budget;
    return f;
}

moe_status to_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

// Fixed logits scratch of moe_route_noalloc: one copy per GPU that loads the library, held
// until the process exits. Only device code may name it directly; host code must use the
// address that cudaGetSymbolAddress returns for the current device.
static __device__ __align__(256) float g_route_noalloc_logits[MOE_ROUTE_NOALLOC_MAX_LOGITS];

// Device address of g_route_noalloc_logits on the current device, looked up on the first
// call for each device and cached; nullptr if the lookup fails.
float *route_noalloc_scratch()
{
    static std::mutex mu;
    static float *cache[64] = {nullptr};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (cache[dev] == nullptr) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_route_noalloc_logits) != cudaSuccess) {
            // consume the failure so that it is not reported again by the next launch check
            // of this host thread (the caller returns MOE_ERR_CUDA for it)
            (void)cudaGetLastError();
            return nullptr;
        }
        cache[dev] = static_cast<float *>(ptr);
    }
    return cache[dev];
}

cudaError_t record(void *const *events, int n, int i, cudaStream_t st)
{
    if (n == 0) return cudaSuccess;
    return cudaEventRecord(static_cast<cudaEvent_t>(events[i]), st);
}

// The shared expert's GEMMs (dense over all tokens, padded to whole 128-row tiles): the
// gate, layer0 (SwiGLU) into h_s, layer1 (gate-scaled) into ys_s; the combine adds ys_s.
cudaError_t launch_shared(const moe_problem *p, const moe_bf16 *x, const moe_shared_expert *sh,
                          float *g, moe_bf16 *hs, moe_bf16 *ys_s, int *status, int64_t timeout,
                          cudaStream_t st)
{
    const int T = p->T, H = p->H, Fs = sh->F_s;
    const int mt = (T + gemm::BM - 1) / gemm::BM, Tpad = mt * gemm::BM;
    shared_gate_kernel<<<(Tpad + 7) / 8, 256, 0, st>>>(
        reinterpret_cast<const __nv_bfloat16 *>(x),
        reinterpret_cast<const __nv_bfloat16 *>(sh->w_sg), T, H, Tpad, g);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    CUtensorMap m_x, m_w1, m_h, m_w2;
    if (!make_map_2d(&m_x, x, (uint64_t)T, (uint64_t)H, gemm::BM) ||
        !make_map_3d(&m_w1, sh->W1s, 1, (uint64_t)H, (uint64_t)(2 * Fs)) ||
        !make_map_2d(&m_h, hs, (uint64_t)Tpad, (uint64_t)Fs, gemm::BM) ||
        !make_map_3d(&m_w2, sh->W2s, 1, (uint64_t)Fs, (uint64_t)H))
        return cudaErrorInvalidValue;
    GemmArgs a0{};
    a0.dense_m_tiles = mt;
    a0.dense_rows = Tpad;
    a0.k_split = 1;
    a0.out = reinterpret_cast<__nv_bfloat16 *>(hs);
    a0.ld_out = Fs;
    a0.n_cols = Fs;
    a0.up_col = Fs;
    a0.n_tiles = (Fs + 127) / 128;
    a0.k_blocks = H / gemm::BK;
    a0.act = MOE_ACT_SWIGLU;
    a0.status = status;
    a0.timeout_ns = timeout;
    GemmArgs a1 = a0;
    a1.row_w = g;
    a1.out = reinterpret_cast<__nv_bfloat16 *>(ys_s);
    a1.ld_out = H;
    a1.n_cols = H;
    a1.n_tiles = (H + gemm::BN - 1) / gemm::BN;
    a1.k_blocks = Fs / gemm::BK;
    e = launch_gemm<GEMM_SWIGLU>(m_x, m_w1, a0, mt * a0.n_tiles, st);
    if (e != cudaSuccess) return e;
    return launch_gemm<GEMM_SCALE>(m_h, m_w2, a1, mt * a1.n_tiles, st);
}

// The dispatch outputs inside the caller's workspace.
DispatchOut dispatch_bufs(void *ws, const Layout &L)
{
    DispatchOut d;
    d.counts = at<int32_t>(ws, L.counts);
    d.offsets = at<int32_t>(ws, L.offsets);
    d.poff = at<int32_t>(ws, L.poff);
    d.gather_idx = at<int32_t>(ws, L.gather_idx);
    d.inv_pos = at<int32_t>(ws, L.inv_pos);
    d.tile_off = at<int32_t>(ws, L.tile_off);
    d.tile_expert = at<int32_t>(ws, L.tile_expert);
    d.chunk = at<int32_t>(ws, L.chunk);
    d.ptile_off = at<int32_t>(ws, L.ptile_off);
    d.ptile_expert = at<int32_t>(ws, L.ptile_expert);
    d.hot_off = at<int32_t>(ws, L.hot_off);
    d.hot_tile_expert = at<int32_t>(ws, L.hot_tile_expert);
    d.cold_tile = at<int32_t>(ws, L.cold_tile);
    d.ready = at<int>(ws, L.ready);
    d.n_ready = L.n_ready;
    d.row_w = at<float>(ws, L.row_w);
    d.meta = at<DispatchMeta>(ws, L.meta);
    return d;
}

// Materialise x_perm (one gather pass, then TMA reads in layer0) when the routed rows
// average at least one 128-row tile per expert. Measured on the bench layers: layer0 -6% to
// -15% (TMA instead of four cp.async warps per CTA, less power per FLOP under the cap)
// against +0.04 to +0.17 ms for the gather; decode-sized batches keep the in-kernel gather.
bool use_x_perm(const moe_problem *p)
{
    return (int64_t)p->T * p->top_k >= (int64_t)p->E * M_TILE;
}

// Per-shape plan of the layer's GEMM and combine work (Comet §3.2.2: the split between
// data-movement and compute work is chosen per shape). `fused`: one persistent launch in
// which each SM's four data-movement warps first serve layer0 (row gather or half of each
// epilogue) and then run the combine beside the layer1 GEMM pipeline; otherwise three
// launches (layer0, layer1, combine). `comb_tokens`: tokens per combine item.
// Why the rule: layer1 runs expert-major (each expert's h rows stay in L2 across its 256-
// column stripes), so a combine item can start only when the last expert its tokens touch
// has stored that stripe; the window in which the combine overlaps layer1 is about 1/E of
// layer1. Timed on one B200 (alternating launches, 20 layers each, under the power cap):
//   E = 8  (Mixtral-shaped): 5.19 ms persistent against 5.26 ms separate, and in one staged
//          run 4.61 against 4.73 ms for the three stages (combine 99.8% hidden);
//   E = 16 (Phi-3.5-shaped): 5.08 against 4.67 ms; E = 64 (Qwen2-shaped): 4.36 against
//          3.57 ms; E = 256 (skewed): 4.89 against 4.63 ms -- the combine waits for the last
//          experts and runs exposed on eight warps per SM, and the longer full-power launch
//          settles at a lower clock.
// So the persistent launch is taken for large batches with at most 8 experts; decode-sized
// batches (single-tile experts) keep the separate launches and their operand-swapped body.
struct FusedPlan {
    bool fused;
    int comb_tokens;
};

FusedPlan fused_plan(const moe_problem *p)
{
    FusedPlan f;
    f.fused = use_x_perm(p) && p->E <= 8;
    f.comb_tokens = p->T >= 2048 ? COMBINE_TOKENS : 64;
    return f;
}

bool run_fused(const moe_problem *p)
{
    const int mode = g_gemm_mode.load();
    return mode == MOE_GEMM_FUSED || mode == MOE_GEMM_FUSED_LAYERS ||
           (mode == MOE_GEMM_AUTO && fused_plan(p).fused);
}

// The persistent launch runs the combine too (else the combine is its own launch after it).
bool fused_combine_in_launch()
{
    return g_gemm_mode.load() != MOE_GEMM_FUSED_LAYERS;
}

// The persistent launch also routes and dispatches (a computed routing, no stage events and
// 16-byte aligned operands besides): one-launch exact router, rows read by TMA from x_perm.
bool whole_layer(const moe_problem *p)
{
    return g_front.load() != 0 && g_gemm_mode.load() != MOE_GEMM_CTA_PAIR && run_fused(p) &&
           fused_combine_in_launch() && use_x_perm(p) && route_uses_chain(p) &&
           !route_uses_filter(p) && front_plan(p).ok;
}

moe_status forward_impl(const moe_problem *p, const moe_bf16 *x, const moe_bf16 *Wg,
                        const float *bias, const moe_bf16 *W1, const moe_bf16 *W2, moe_bf16 *out,
                        int32_t *topk_idx_out, float *topk_w_out, void *ws, size_t ws_bytes,
                        cudaStream_t st, void *const *events, int n_events,
                        const moe_shared_expert *sh = nullptr,
                        const int32_t *given_idx = nullptr, const float *given_w = nullptr,
                        const int32_t *n_rows = nullptr)
{
    moe_status s = check_problem(p);
    if (s != MOE_OK) return s;
    if (n_events != 0 && (n_events != MOE_NUM_STAGE_EVENTS || events == nullptr))
        return MOE_ERR_INVALID_ARG;
    const bool given = (given_idx != nullptr); // routing supplied: no router launch, no W_g
    if (ws == nullptr || (p->T > 0 && (x == nullptr || out == nullptr)) ||
        (Wg == nullptr && !given) || W1 == nullptr || W2 == nullptr ||
        (given && p->T > 0 && given_w == nullptr))
        return MOE_ERR_INVALID_ARG;
    const Layout L = make_layout(p);
    if (ws_bytes < L.end_forward) return MOE_ERR_WORKSPACE;
    if (!aligned16(x) || !aligned16(out) || !aligned16(W1) || !aligned16(W2) || !aligned16(Wg) ||
        !aligned16(ws) || !aligned4(bias) || !aligned4(topk_idx_out) || !aligned4(topk_w_out))
        return MOE_ERR_INVALID_ARG;

    int *status = at<int>(ws, L.status);
    if (p->T == 0) {
        // nothing to compute; still clear the status word and mark the stage boundaries
        cudaError_t e = cudaMemsetAsync(status, 0, 8, st);
        for (int i = 0; i < n_events && e == cudaSuccess; ++i) e = record(events, n_events, i, st);
        return to_status(e);
    }
    int32_t *topk_idx = given ? const_cast<int32_t *>(given_idx)
                              : (topk_idx_out ? topk_idx_out : at<int32_t>(ws, L.topk_idx));
    float *topk_w = given ? const_cast<float *>(given_w)
                          : (topk_w_out ? topk_w_out : at<float>(ws, L.topk_w));
    const DispatchOut d = dispatch_bufs(ws, L);
    moe_bf16 *x_perm = at<moe_bf16>(ws, L.x_perm);
    moe_bf16 *h = at<moe_bf16>(ws, L.h);
    moe_bf16 *ys = at<moe_bf16>(ws, L.ys);

    const int F = p->F, H = p->H, E = p->E;
    const bool gated = (p->act == MOE_ACT_SWIGLU);
    CUtensorMap m_x, m_w1, m_h, m_w2;
    // layer0's A rows: a materialised x_perm read with TMA (CTA pairs, and large batches in
    // the single-CTA kernel), or gathered from x inside the kernel by cp.async warps (decode-
    // sized batches, whose padded rows would be mostly zeros, and the fused launch)
    const bool pair = (g_gemm_mode.load() == MOE_GEMM_CTA_PAIR);
    const bool fused = !pair && n_rows == nullptr && run_fused(p);
    const bool xperm = pair || use_x_perm(p);
    // the whole layer in one launch: the persistent launch routes and dispatches first (its
    // router is the one-launch exact router; stage events need the stages' own launches)
    const FrontPlan fpl = front_plan(p);
    const bool one = fused && !given && n_events == 0 && whole_layer(p);
    const bool a_ok = xperm ? make_map_2d(&m_x, x_perm, (uint64_t)L.pmax, (uint64_t)H, gemm::BM)
                            : make_map_2d(&m_x, x, (uint64_t)p->T, (uint64_t)H, 1);
    if (!a_ok ||
        !make_map_3d(&m_w1, W1, (uint64_t)E, (uint64_t)H, (uint64_t)(gated ? 2 * F : F)) ||
        !make_map_2d(&m_h, h, (uint64_t)L.pmax, (uint64_t)F, gemm::BM) ||
        !make_map_3d(&m_w2, W2, (uint64_t)E, (uint64_t)F, (uint64_t)H))
        return MOE_ERR_CUDA;

    const int64_t timeout = g_timeout_ns.load();
    const FilterBufs fb = filter_bufs(ws, L);
    cudaError_t e = record(events, n_events, 0, st);
    CUtensorMap m_rx = m_x, m_rw = m_x; // the router's maps (whole-layer launch only)
    if (one) {
        // status word and grid-barrier counter (same 256-byte block) start from zero
        if (!make_map_2d(&m_rx, x, (uint64_t)p->T, (uint64_t)H, (uint32_t)fpl.tt) ||
            !make_map_2d_plain(&m_rw, Wg, (uint64_t)H, (uint64_t)E, (uint32_t)E, RC_HC))
            return MOE_ERR_CUDA;
        if (e == cudaSuccess) e = cudaMemsetAsync(status, 0, 32, st);
    } else {
        if (e == cudaSuccess && !given)
            e = launch_route(p, x, Wg, bias, topk_idx, topk_w, at<float>(ws, L.logits), status, st,
                             &fb);
        if (e == cudaSuccess) e = record(events, n_events, 1, st);
        // with the routing supplied the dispatch clears the status word (and checks the ids)
        if (e == cudaSuccess)
            e = launch_dispatch(p, L, topk_idx, topk_w, d, status, given ? 1 : 0, st, n_rows);
        if (e == cudaSuccess && xperm) e = launch_gather(p, x, d.gather_idx, d.meta, x_perm, st);
        if (e == cudaSuccess) e = record(events, n_events, 2, st);
    }

    GemmArgs a0{};
    a0.tile_off = d.tile_off;
    a0.tile_expert = d.tile_expert;
    a0.ptile_off = d.ptile_off;
    a0.ptile_expert = d.ptile_expert;
    a0.expert_rows = d.counts;
    a0.hot_off = d.hot_off;
    a0.hot_tile_expert = d.hot_tile_expert;
    a0.cold_tile = d.cold_tile;
    a0.meta = d.meta;
    a0.row_w = nullptr;
    a0.gather_idx = xperm ? nullptr : d.gather_idx;
    a0.epi8 = xperm && !pair ? 1 : 0; // the idle gather warps join the epilogue
    a0.gather_len = L.pmax;
    a0.gather_src = reinterpret_cast<const __nv_bfloat16 *>(x);
    a0.gather_rows = p->T;
    a0.gather_ld = H;
    a0.out = reinterpret_cast<__nv_bfloat16 *>(h);
    a0.ld_out = F;
    a0.n_cols = F;
    a0.k_blocks = H / gemm::BK;
    a0.up_col = F;
    a0.act = p->act;
    a0.status = status;
    a0.timeout_ns = timeout;
    a0.n_tiles = gated ? (F + 127) / 128 : (F + gemm::BN - 1) / gemm::BN;
    GemmArgs a1 = a0;
    a1.gather_idx = nullptr; // layer1 reads h rows in place
    a1.epi8 = 0;             // four epilogue warps (eight measured slower on layer1)
    a1.row_w = d.row_w;
    a1.out = reinterpret_cast<__nv_bfloat16 *>(ys);
    a1.ld_out = H;
    a1.n_cols = H;
    a1.n_tiles = (H + gemm::BN - 1) / gemm::BN;
    a1.k_blocks = F / gemm::BK;

    // shared expert (dense over all tokens): its rows are added by the combine
    moe_bf16 *ys_s = nullptr;
    if (sh != nullptr && e == cudaSuccess) {
        const Layout LS = make_layout(p, sh->F_s);
        ys_s = at<moe_bf16>(ws, LS.sh_ys);
        e = launch_shared(p, x, sh, at<float>(ws, LS.sh_gate), at<moe_bf16>(ws, LS.sh_h), ys_s,
                          status, timeout, st);
    }

    if (fused) {
        // one persistent launch: layer0 -> layer1 -> combine, tile-level ready flags
        const FusedPlan plan = fused_plan(p);
        FusedArgs fa{};
        fa.l0 = a0;
        fa.l1 = a1;
        fa.ready0 = d.ready;
        fa.ready1 = d.ready + L.max_tiles;
        fa.done0 = d.ready + L.n_ready - 2;
        fa.comb_next = d.ready + L.n_ready - 1;
        fa.max_tiles = L.max_tiles;
        fa.inv_pos = d.inv_pos;
        fa.out = reinterpret_cast<__nv_bfloat16 *>(out);
        fa.T = p->T;
        fa.H = H;
        fa.k = p->top_k;
        fa.ys_rows = L.pmax;
        fa.ys_shared = reinterpret_cast<const __nv_bfloat16 *>(ys_s);
        fa.a_tma = xperm ? 1 : 0;
        fa.comb_tokens = plan.comb_tokens;
        fa.comb_in_launch = fused_combine_in_launch() ? 1 : 0;
        fa.fault_skip = g_fault_skip.load();
        fa.trace = g_trace.load();
        fa.trace_cap = g_trace_cap.load();
        const int max_work = L.max_tiles * (a0.n_tiles + a1.n_tiles);
        if (one) {
            FrontArgs &f = fa.front;
            f.ra.bias = bias;
            f.ra.topk_idx = topk_idx;
            f.ra.topk_w = topk_w;
            f.ra.T = p->T;
            f.ra.H = H;
            f.ra.E = E;
            f.ra.k = p->top_k;
            f.ra.gate = p->gate;
            f.ra.tt = fpl.tt;
            f.ra.stages = fpl.stages;
            f.ra.status = status;
            f.ra.timeout_ns = timeout;
            f.ra.group_counts = at<int32_t>(ws, L.gcount);
            f.ncw = fpl.ncw;
            f.n_groups = fpl.n_groups;
            FrontDispatch &fd = f.fd;
            fd.group_counts = f.ra.group_counts;
            fd.n_groups = fpl.n_groups;
            fd.tt = fpl.tt;
            fd.topk_idx = topk_idx;
            fd.topk_w = topk_w;
            fd.T = p->T;
            fd.E = E;
            fd.k = p->top_k;
            fd.H = H;
            fd.so = scan_out(L, d);
            fd.inv_pos = d.inv_pos;
            fd.x = reinterpret_cast<const __nv_bfloat16 *>(x);
            fd.x_perm = reinterpret_cast<__nv_bfloat16 *>(x_perm);
            f.gbar = status + 4;
        }
        if (e == cudaSuccess) {
            // (a0.epi8 is for the separate launches; the fused kernel splits layer0's epilogue
            // itself when its rows come by TMA)
            if (one)
                e = gated ? launch_fused<GEMM_SWIGLU, true>(m_x, m_w1, m_h, m_w2, m_rx, m_rw, fa, max_work, st)
                          : launch_fused<GEMM_ACT, true>(m_x, m_w1, m_h, m_w2, m_rx, m_rw, fa, max_work, st);
            else
                e = gated ? launch_fused<GEMM_SWIGLU, false>(m_x, m_w1, m_h, m_w2, m_rx, m_rw, fa, max_work, st)
                          : launch_fused<GEMM_ACT, false>(m_x, m_w1, m_h, m_w2, m_rx, m_rw, fa, max_work, st);
        }
        if (fa.comb_in_launch) {
            // the three stages share one launch: their boundaries coincide at its end
            for (int i = 3; i < 6 && e == cudaSuccess; ++i) e = record(events, n_events, i, st);
            return to_status(e);
        }
        // layer0 and layer1 share the launch; the combine follows as its own launch
        for (int i = 3; i < 5 && e == cudaSuccess; ++i) e = record(events, n_events, i, st);
        if (e == cudaSuccess)
            e = launch_combine(p, ys, L.pmax, d.inv_pos, out, status, 0, st, ys_s, n_rows);
        if (e == cudaSuccess) e = record(events, n_events, 5, st);
        return to_status(e);
    }

    // work order of the single-CTA launches; MOE_ORDER_NARROW lets the device run the
    // operand-swapped body (N = the experts' row counts) when every expert is single-tile
    const int order = g_order.load();
    const bool narrow = (order == MOE_ORDER_NARROW || order == MOE_ORDER_PHASED) && !pair;
    a0.order = a1.order = order == MOE_ORDER_MIXED    ? ORDER_MIXED
                          : order == MOE_ORDER_PHASED ? ORDER_HOT
                                                      : ORDER_EXPERT;
    GemmArgs n0 = a0, n1 = a1; // narrow items: column blocks of 64 (SwiGLU) or 128 columns
    n0.n_tiles = gated ? F / 64 : (F + 127) / 128;
    n1.n_tiles = (H + 127) / 128;
    if (narrow) {
        if (e == cudaSuccess)
            e = gated ? launch_gemm_select<GEMM_SWIGLU>(m_x, m_w1, a0, n0, st)
                      : launch_gemm_select<GEMM_ACT>(m_x, m_w1, a0, n0, st);
        if (e == cudaSuccess) e = record(events, n_events, 3, st);
        if (e == cudaSuccess) e = launch_gemm_select<GEMM_SCALE>(m_h, m_w2, a1, n1, st);
        if (e == cudaSuccess) e = record(events, n_events, 4, st);
    } else {
        if (gated) {
            if (e == cudaSuccess)
                e = launch_gemm_any<GEMM_SWIGLU>(m_x, m_w1, a0, L.max_tiles * a0.n_tiles, st);
        } else {
            if (e == cudaSuccess)
                e = launch_gemm_any<GEMM_ACT>(m_x, m_w1, a0, L.max_tiles * a0.n_tiles, st);
        }
        if (e == cudaSuccess) e = record(events, n_events, 3, st);
        if (e == cudaSuccess)
            e = launch_gemm_any<GEMM_SCALE>(m_h, m_w2, a1, L.max_tiles * a1.n_tiles, st);
        if (e == cudaSuccess) e = record(events, n_events, 4, st);
    }
    if (e == cudaSuccess)
        e = launch_combine(p, ys, L.pmax, d.inv_pos, out, status, 0, st, ys_s, n_rows);
    if (e == cudaSuccess) e = record(events, n_events, 5, st);
    return to_status(e);
}

template <int BMODE>
cudaError_t launch_gemm_bwd(const CUtensorMap &ta, const CUtensorMap &tb, const GemmArgs &args,
                            int max_work, cudaStream_t st)
{
    auto kern = moe_grouped_gemm_bwd_kernel<BMODE>;
    cudaError_t err =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, gemm::SMEM_BYTES);
    if (err != cudaSuccess) return err;
    int grid = sm_count();
    if (grid <= 0) grid = 148;
    if (grid > max_work) grid = max_work;
    if (grid < 1) grid = 1;
    const int threads = args.gather_idx != nullptr ? gemm::NUM_THREADS_GATHER : gemm::NUM_THREADS;
    kern<<<grid, threads, gemm::SMEM_BYTES, st>>>(ta, tb, args);
    return cudaGetLastError();
}

// Shapes the backward supports: the weight-gradient GEMMs' M (F and H) in whole 128-row
// tiles; the gates a softmax over the selected logits.
moe_status check_problem_bwd(const moe_problem *p)
{
    const moe_status s = check_problem(p);
    if (s != MOE_OK) return s;
    if (p->H % 128 != 0 || p->F % 128 != 0 || p->gate == MOE_GATE_SOFTMAX_ALL)
        return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

// The layer's gradients (see backward.cuh): route and dispatch as the forward; x rows
// gathered (x_perm); z = x W1 recomputed (identity epilogue); u = dy W2^T (dy rows gathered,
// W2 read K-major); the row pass (a, dz in place of z, gy, dw); logit gradients; dW2 = a^T gy
// and dW1 = x_perm^T dz per expert; dx_perm = dz W1^T (W1 read K-major); dx; dW_g and dbias.
moe_status backward_impl(const moe_problem *p, const moe_bf16 *x, const moe_bf16 *Wg,
                         const float *bias, const moe_bf16 *W1, const moe_bf16 *W2,
                         const moe_bf16 *dy, moe_bf16 *dx, float *dWg, float *dbias, moe_bf16 *dW1,
                         moe_bf16 *dW2, void *ws, size_t ws_bytes, cudaStream_t st)
{
    moe_status s = check_problem_bwd(p);
    if (s != MOE_OK) return s;
    if (ws == nullptr || Wg == nullptr || W1 == nullptr || W2 == nullptr || dWg == nullptr ||
        dbias == nullptr || dW1 == nullptr || dW2 == nullptr ||
        (p->T > 0 && (x == nullptr || dy == nullptr || dx == nullptr)))
        return MOE_ERR_INVALID_ARG;
    const Layout L = make_layout(p, 0, false, true);
    if (ws_bytes < L.end_bwd) return MOE_ERR_WORKSPACE;
    if (!aligned16(x) || !aligned16(Wg) || !aligned16(W1) || !aligned16(W2) || !aligned16(dy) ||
        !aligned16(dx) || !aligned16(dW1) || !aligned16(dW2) || !aligned4(dWg) || !aligned4(dbias) ||
        !aligned4(bias) || !aligned16(ws))
        return MOE_ERR_INVALID_ARG;
    const int T = p->T, H = p->H, F = p->F, E = p->E, k = p->top_k;
    const bool gated = (p->act == MOE_ACT_SWIGLU);
    const int w1c = gated ? 2 * F : F;
    int *status = at<int>(ws, L.status);
    if (T == 0) { // no rows: every gradient is zero
        cudaError_t e = cudaMemsetAsync(status, 0, 8, st);
        if (e == cudaSuccess) e = cudaMemsetAsync(dWg, 0, (size_t)H * E * 4, st);
        if (e == cudaSuccess) e = cudaMemsetAsync(dbias, 0, (size_t)E * 4, st);
        if (e == cudaSuccess) e = cudaMemsetAsync(dW1, 0, (size_t)E * H * w1c * 2, st);
        if (e == cudaSuccess) e = cudaMemsetAsync(dW2, 0, (size_t)E * F * H * 2, st);
        return to_status(e);
    }
    int32_t *topk_idx = at<int32_t>(ws, L.topk_idx);
    float *topk_w = at<float>(ws, L.topk_w);
    DispatchOut d = dispatch_bufs(ws, L);
    d.active_list = at<int32_t>(ws, L.bact);
    moe_bf16 *x_perm = at<moe_bf16>(ws, L.x_perm);
    moe_bf16 *u = at<moe_bf16>(ws, L.h);   // [P, F]
    moe_bf16 *gy = at<moe_bf16>(ws, L.ys); // [P, H]
    moe_bf16 *gu = at<moe_bf16>(ws, L.bgu), *a = at<moe_bf16>(ws, L.ba);
    moe_bf16 *dxp = at<moe_bf16>(ws, L.bdxp);
    float *dw_row = at<float>(ws, L.bdw), *dl_row = at<float>(ws, L.bdl);

    CUtensorMap m_x, m_w1, m_w2k, m_gu, m_a, m_gy, m_xp, m_dz, m_w1k;
    // z = x W1 reads the expert-sorted x_perm rows (gathered for dW1 anyway) with TMA
    if (!make_map_2d(&m_x, x_perm, (uint64_t)L.pmax, (uint64_t)H, gemm::BM) ||
        !make_map_3d(&m_w1, W1, (uint64_t)E, (uint64_t)H, (uint64_t)w1c) ||
        !make_map_3d(&m_w2k, W2, (uint64_t)E, (uint64_t)F, (uint64_t)H, 128) ||
        !make_map_2d(&m_a, a, (uint64_t)L.pmax, (uint64_t)F, 64) ||
        !make_map_3d(&m_gy, gy, 1, (uint64_t)L.pmax, (uint64_t)H) ||
        !make_map_2d(&m_xp, x_perm, (uint64_t)L.pmax, (uint64_t)H, 64) ||
        !make_map_3d(&m_dz, gu, 1, (uint64_t)L.pmax, (uint64_t)w1c) ||
        !make_map_2d(&m_gu, gu, (uint64_t)L.pmax, (uint64_t)w1c, gemm::BM) ||
        !make_map_3d(&m_w1k, W1, (uint64_t)E, (uint64_t)H, (uint64_t)w1c, 128))
        return MOE_ERR_CUDA;
    const int64_t timeout = g_timeout_ns.load();
    const FilterBufs fb = filter_bufs(ws, L);
    cudaError_t e = launch_route(p, x, Wg, bias, topk_idx, topk_w, at<float>(ws, L.logits), status,
                                 st, &fb);
    if (e == cudaSuccess) e = launch_dispatch(p, L, topk_idx, topk_w, d, status, 0, st);
    if (e == cudaSuccess) e = launch_gather(p, x, d.gather_idx, d.meta, x_perm, st);

    GemmArgs g{};
    g.tile_off = d.tile_off;
    g.tile_expert = d.tile_expert;
    g.meta = d.meta;
    g.order = ORDER_EXPERT;
    g.act = MOE_ACT_IDENTITY;
    g.status = status;
    g.timeout_ns = timeout;
    g.gather_len = L.pmax;
    g.gather_rows = T;
    g.gather_ld = H;
    // z = x W1 (recomputed pre-activations) from the sorted rows
    GemmArgs gz = g;
    gz.out = reinterpret_cast<__nv_bfloat16 *>(gu);
    gz.ld_out = gz.n_cols = w1c;
    gz.n_tiles = (w1c + gemm::BN - 1) / gemm::BN;
    gz.k_blocks = H / gemm::BK;
    if (e == cudaSuccess) e = launch_gemm<GEMM_ACT>(m_x, m_w1, gz, L.max_tiles * gz.n_tiles, st);
    // u = dy W2^T, dy rows gathered
    GemmArgs gu_ = g;
    gu_.gather_idx = d.gather_idx;
    gu_.gather_src = reinterpret_cast<const __nv_bfloat16 *>(dy);
    gu_.out = reinterpret_cast<__nv_bfloat16 *>(u);
    gu_.ld_out = gu_.n_cols = F;
    gu_.n_tiles = (F + gemm::BN - 1) / gemm::BN;
    gu_.k_blocks = H / gemm::BK;
    CUtensorMap m_dy; // unused: the dy rows are gathered in the kernel
    if (!make_map_2d(&m_dy, dy, (uint64_t)T, (uint64_t)H, 1)) return MOE_ERR_CUDA;
    if (e == cudaSuccess)
        e = launch_gemm_bwd<BMODE_KMAJOR>(m_dy, m_w2k, gu_, L.max_tiles * gu_.n_tiles, st);
    // row pass: a, dz (in place of z), gy, dw
    if (e == cudaSuccess) {
        int grid = sm_count() * 8;
        if (grid <= 0) grid = 1184;
        bwd_rows_kernel<<<grid, BWD_THREADS, 0, st>>>(
            reinterpret_cast<__nv_bfloat16 *>(gu), reinterpret_cast<const __nv_bfloat16 *>(u),
            reinterpret_cast<const __nv_bfloat16 *>(dy), d.gather_idx, d.row_w, d.meta, M_TILE, F, H,
            T, p->act, reinterpret_cast<__nv_bfloat16 *>(a), reinterpret_cast<__nv_bfloat16 *>(gy),
            dw_row);
        e = cudaGetLastError();
    }
    if (e == cudaSuccess) {
        bwd_router_kernel<<<(T * 32 + 255) / 256, 256, 0, st>>>(topk_w, d.inv_pos, dw_row, T, k, dl_row);
        e = cudaGetLastError();
    }
    // weight gradients: zero for the experts without rows; dW2[e] = a_e^T gy_e and
    // dW1[e] = x_perm_e^T dz_e for the others (the active list from the dispatch)
    if (e == cudaSuccess) {
        const int64_t v1 = (int64_t)H * w1c / 8, v2 = (int64_t)F * H / 8;
        zero_inactive_slabs_kernel<<<dim3((unsigned)((v1 + 255) / 256 < 64 ? (v1 + 255) / 256 : 64), E), 256, 0, st>>>(
            reinterpret_cast<uint4 *>(dW1), v1, d.counts);
        zero_inactive_slabs_kernel<<<dim3((unsigned)((v2 + 255) / 256 < 64 ? (v2 + 255) / 256 : 64), E), 256, 0, st>>>(
            reinterpret_cast<uint4 *>(dW2), v2, d.counts);
        e = cudaGetLastError();
    }
    GemmArgs w2 = g;
    w2.active_list = d.active_list;
    w2.wg_experts = E;
    w2.wg_mtiles = F / gemm::BM;
    w2.out = reinterpret_cast<__nv_bfloat16 *>(dW2);
    w2.ld_out = w2.n_cols = H;
    w2.n_tiles = (H + gemm::BN - 1) / gemm::BN;
    if (e == cudaSuccess)
        e = launch_gemm_bwd<BMODE_WGRAD>(m_a, m_gy, w2, E * w2.wg_mtiles * w2.n_tiles, st);
    GemmArgs w1 = g;
    w1.active_list = d.active_list;
    w1.wg_experts = E;
    w1.wg_mtiles = H / gemm::BM;
    w1.out = reinterpret_cast<__nv_bfloat16 *>(dW1);
    w1.ld_out = w1.n_cols = w1c;
    w1.n_tiles = (w1c + gemm::BN - 1) / gemm::BN;
    if (e == cudaSuccess)
        e = launch_gemm_bwd<BMODE_WGRAD>(m_xp, m_dz, w1, E * w1.wg_mtiles * w1.n_tiles, st);
    // dx_perm = dz W1^T (dz rows by TMA, W1 read K-major)
    GemmArgs gx = g;
    gx.out = reinterpret_cast<__nv_bfloat16 *>(dxp);
    gx.ld_out = gx.n_cols = H;
    gx.n_tiles = (H + gemm::BN - 1) / gemm::BN;
    gx.k_blocks = w1c / gemm::BK;
    if (e == cudaSuccess)
        e = launch_gemm_bwd<BMODE_KMAJOR>(m_gu, m_w1k, gx, L.max_tiles * gx.n_tiles, st);
    if (e == cudaSuccess) {
        int grid = sm_count() * 8;
        if (grid <= 0) grid = 1184;
        if (grid > T) grid = T;
        bwd_dx_kernel<<<grid, BWD_THREADS, 0, st>>>(reinterpret_cast<const __nv_bfloat16 *>(dxp),
                                                     d.inv_pos, topk_idx, dl_row,
                                                     reinterpret_cast<const __nv_bfloat16 *>(Wg), T,
                                                     H, E, k, reinterpret_cast<__nv_bfloat16 *>(dx));
        e = cudaGetLastError();
    }
    if (e == cudaSuccess) {
        bwd_router_weights_kernel<<<dim3(E, (H + BWD_THREADS - 1) / BWD_THREADS), BWD_THREADS, 0, st>>>(
            reinterpret_cast<const __nv_bfloat16 *>(x), d.gather_idx, d.poff, d.counts, dl_row, H, E,
            (bias != nullptr && p->gate != MOE_GATE_SELECT_BIAS) ? 1 : 0, dWg, dbias);
        e = cudaGetLastError();
    }
    return to_status(e);
}

// Shapes the FP8 expert path supports: both GEMMs' K (H and F) in whole 128-value k-blocks.
moe_status check_problem_fp8(const moe_problem *p)
{
    const moe_status s = check_problem(p);
    if (s != MOE_OK) return s;
    if (p->H % 128 != 0 || p->F % 128 != 0) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

// The layer with e4m3 experts: route and dispatch as in forward_impl (bf16 x and W_g), then
// x rows quantised, layer0 on codes (single-CTA persistent kernel, kind::f8f6f4, gathered
// rows), h rows quantised, layer1 on codes, the combine. Stage events as moe_forward_staged
// (the x quantisation falls in the dispatch stage, the h quantisation in the layer1 stage).
moe_status forward_impl_fp8(const moe_problem *p, const moe_bf16 *x, const moe_bf16 *Wg,
                            const float *bias, const moe_fp8 *W1q, const float *s1,
                            const moe_fp8 *W2q, const float *s2, moe_bf16 *out,
                            int32_t *topk_idx_out, float *topk_w_out, void *ws, size_t ws_bytes,
                            cudaStream_t st, void *const *events, int n_events)
{
    moe_status s = check_problem_fp8(p);
    if (s != MOE_OK) return s;
    if (n_events != 0 && (n_events != MOE_NUM_STAGE_EVENTS || events == nullptr))
        return MOE_ERR_INVALID_ARG;
    if (ws == nullptr || (p->T > 0 && (x == nullptr || out == nullptr)) || Wg == nullptr ||
        W1q == nullptr || W2q == nullptr || s1 == nullptr || s2 == nullptr)
        return MOE_ERR_INVALID_ARG;
    const Layout L = make_layout(p, 0, true);
    if (ws_bytes < L.end_fp8) return MOE_ERR_WORKSPACE;
    if (!aligned16(x) || !aligned16(out) || !aligned16(W1q) || !aligned16(W2q) || !aligned16(Wg) ||
        !aligned16(s1) || !aligned16(s2) || !aligned16(ws) || !aligned4(bias) ||
        !aligned4(topk_idx_out) || !aligned4(topk_w_out))
        return MOE_ERR_INVALID_ARG;
    int *status = at<int>(ws, L.status);
    if (p->T == 0) {
        cudaError_t e = cudaMemsetAsync(status, 0, 8, st);
        for (int i = 0; i < n_events && e == cudaSuccess; ++i) e = record(events, n_events, i, st);
        return to_status(e);
    }
    int32_t *topk_idx = topk_idx_out ? topk_idx_out : at<int32_t>(ws, L.topk_idx);
    float *topk_w = topk_w_out ? topk_w_out : at<float>(ws, L.topk_w);
    const DispatchOut d = dispatch_bufs(ws, L);
    moe_bf16 *h = at<moe_bf16>(ws, L.h);
    moe_bf16 *ys = at<moe_bf16>(ws, L.ys);
    uint8_t *xq = at<uint8_t>(ws, L.xq), *hq = at<uint8_t>(ws, L.hq);
    float *sx = at<float>(ws, L.sx), *sh = at<float>(ws, L.sh);

    const int F = p->F, H = p->H, E = p->E;
    const bool gated = (p->act == MOE_ACT_SWIGLU);
    const int w1_cols = gated ? 2 * F : F;
    CUtensorMap m_x, m_w1, m_h, m_w2, n_w1, n_w2;
    // large batches (single-CTA): the x codes gathered into expert-sorted rows first and read
    // with TMA, so the four gather warps can join the epilogue (which sets the pace with e4m3)
    uint8_t *xq_perm = at<uint8_t>(ws, L.x_perm); // [P_max, H] codes in the x_perm region
    const bool xperm = g_gemm_mode.load() != MOE_GEMM_CTA_PAIR && use_x_perm(p);
    if (!(xperm ? make_map_2d_u8(&m_x, xq_perm, (uint64_t)L.pmax, (uint64_t)H, gemm::BM)
                : make_map_2d_u8(&m_x, xq, (uint64_t)p->T, (uint64_t)H, 1)) ||
        !make_map_3d_u8(&m_w1, W1q, (uint64_t)E, (uint64_t)w1_cols, (uint64_t)H) ||
        !make_map_2d_u8(&m_h, hq, (uint64_t)L.pmax, (uint64_t)F, gemm::BM) ||
        !make_map_3d_u8(&m_w2, W2q, (uint64_t)E, (uint64_t)H, (uint64_t)F) ||
        // the narrow body's weight boxes: 64 rows
        !make_map_3d_u8(&n_w1, W1q, (uint64_t)E, (uint64_t)w1_cols, (uint64_t)H, 64) ||
        !make_map_3d_u8(&n_w2, W2q, (uint64_t)E, (uint64_t)H, (uint64_t)F, 64))
        return MOE_ERR_CUDA;

    const int64_t timeout = g_timeout_ns.load();
    const FilterBufs fb = filter_bufs(ws, L);
    cudaError_t e = record(events, n_events, 0, st);
    if (e == cudaSuccess)
        e = launch_route(p, x, Wg, bias, topk_idx, topk_w, at<float>(ws, L.logits), status, st,
                         &fb);
    if (e == cudaSuccess) e = record(events, n_events, 1, st);
    if (e == cudaSuccess) e = launch_dispatch(p, L, topk_idx, topk_w, d, status, 0, st);
    if (e == cudaSuccess) e = launch_quant_rows(x, p->T, H, nullptr, xq, sx, st);
    if (e == cudaSuccess && xperm) { // a row of H codes moves as H / 2 two-byte elements
        moe_problem ph = *p;
        ph.H = H / 2;
        e = launch_gather(&ph, reinterpret_cast<const moe_bf16 *>(xq), d.gather_idx, d.meta,
                          reinterpret_cast<moe_bf16 *>(xq_perm), st);
    }
    if (e == cudaSuccess) e = record(events, n_events, 2, st);

    GemmArgs a0{};
    a0.tile_off = d.tile_off;
    a0.tile_expert = d.tile_expert;
    a0.meta = d.meta;
    a0.hot_off = d.hot_off;
    a0.hot_tile_expert = d.hot_tile_expert;
    a0.cold_tile = d.cold_tile;
    // the select kernels below: MOE_ORDER_PHASED runs the cold experts' items narrow first
    a0.order = g_order.load() == MOE_ORDER_PHASED ? ORDER_HOT : ORDER_EXPERT;
    a0.gather_idx = xperm ? nullptr : d.gather_idx;
    a0.scale_idx = xperm ? d.gather_idx : nullptr; // the token of each sorted row's scale
    a0.epi8 = xperm ? 1 : 0;
    a0.gather_len = L.pmax;
    a0.gather_src = reinterpret_cast<const __nv_bfloat16 *>(xq); // bytes: the codes of x
    a0.gather_rows = p->T;
    a0.gather_ld = H;
    a0.out = reinterpret_cast<__nv_bfloat16 *>(h);
    a0.ld_out = F;
    a0.n_cols = F;
    a0.k_blocks = H / 128;
    a0.up_col = F;
    a0.act = p->act;
    a0.status = status;
    a0.timeout_ns = timeout;
    a0.n_tiles = gated ? F / 128 : (F + gemm::BN - 1) / gemm::BN;
    a0.a_scale = sx;
    a0.b_scale = s1;
    a0.b_scale_ld = w1_cols;
    GemmArgs a1 = a0;
    a1.gather_idx = nullptr; // layer1 reads the h codes in place (TMA)
    a1.row_w = d.row_w;
    a1.out = reinterpret_cast<__nv_bfloat16 *>(ys);
    a1.ld_out = H;
    a1.n_cols = H;
    a1.n_tiles = (H + gemm::BN - 1) / gemm::BN;
    a1.k_blocks = F / 128;
    a1.a_scale = sh;
    a1.scale_idx = nullptr; // h rows carry their own scales
    a1.epi8 = 0;            // four epilogue warps (eight measured slower on layer1)
    a1.b_scale = s2;
    a1.b_scale_ld = H;
    // narrow items (every expert single-tile): column blocks of 64 (SwiGLU) or 128 columns
    GemmArgs n0 = a0, n1 = a1;
    n0.expert_rows = n1.expert_rows = d.counts;
    n0.cold_tile = n1.cold_tile = d.cold_tile;
    n0.n_tiles = gated ? F / 64 : (F + 127) / 128;
    n1.n_tiles = (H + 127) / 128;

    if (g_gemm_mode.load() == MOE_GEMM_CTA_PAIR) {
        // CTA pairs: the x code rows gathered first (one byte per value: a row of H codes is
        // moved as H / 2 two-byte elements), read by TMA; the scales looked up per row
        CUtensorMap m_xp;
        if (!make_map_2d_u8(&m_xp, xq_perm, (uint64_t)L.pmax, (uint64_t)H, gemm::BM))
            return MOE_ERR_CUDA;
        moe_problem ph = *p;
        ph.H = H / 2;
        if (e == cudaSuccess)
            e = launch_gather(&ph, reinterpret_cast<const moe_bf16 *>(xq), d.gather_idx, d.meta,
                              reinterpret_cast<moe_bf16 *>(xq_perm), st);
        GemmArgs p0 = a0, p1 = a1;
        p0.ptile_off = p1.ptile_off = d.ptile_off;
        p0.ptile_expert = p1.ptile_expert = d.ptile_expert;
        p0.scale_idx = d.gather_idx;
        p0.gather_idx = nullptr;
        if (e == cudaSuccess)
            e = gated ? launch_gemm_pair<GEMM_SWIGLU, true>(m_xp, m_w1, p0, L.max_tiles * p0.n_tiles, st)
                      : launch_gemm_pair<GEMM_ACT, true>(m_xp, m_w1, p0, L.max_tiles * p0.n_tiles, st);
        if (e == cudaSuccess) e = record(events, n_events, 3, st);
        if (e == cudaSuccess) e = launch_quant_rows(h, L.pmax, F, d.meta, hq, sh, st);
        if (e == cudaSuccess)
            e = launch_gemm_pair<GEMM_SCALE, true>(m_h, m_w2, p1, L.max_tiles * p1.n_tiles, st);
    } else {
    if (e == cudaSuccess)
        e = gated ? launch_gemm_select_f8<GEMM_SWIGLU>(m_x, m_w1, n_w1, a0, n0, st)
                  : launch_gemm_select_f8<GEMM_ACT>(m_x, m_w1, n_w1, a0, n0, st);
    if (e == cudaSuccess) e = record(events, n_events, 3, st);
    if (e == cudaSuccess) e = launch_quant_rows(h, L.pmax, F, d.meta, hq, sh, st);
    if (e == cudaSuccess) e = launch_gemm_select_f8<GEMM_SCALE>(m_h, m_w2, n_w2, a1, n1, st);
    }
    if (e == cudaSuccess) e = record(events, n_events, 4, st);
    if (e == cudaSuccess) e = launch_combine(p, ys, L.pmax, d.inv_pos, out, status, 0, st, nullptr);
    if (e == cudaSuccess) e = record(events, n_events, 5, st);
    return to_status(e);
}

} // namespace

// ---------------------------------------------------------------------------------------
// expert-parallel layer, one persistent launch per GPU (fused.cuh, FUSED_EP)
// ---------------------------------------------------------------------------------------

// Workspace of one rank: the receive side is a layer of E / world experts over
// recv_cap = pmax of world * T * min(k, E / world) one-selection rows (its h, tile lists,
// ready counters; the rows themselves are in the exchange buffers), then this rank's
// routing, its group counts and its pairs' destinations.
struct EpLayout {
    moe_problem pr; // the receive side as a problem: T = rows, E = E / world, top_k = 1
    Layout L;
    int64_t recv_cap;
    size_t topk_idx, topk_w, gcount, slot, dest, end;
};

bool ep_shape_ok(const moe_problem *p, int world)
{
    return check_problem(p) == MOE_OK && world >= 1 && world <= MOE_EP_MAX_WORLD &&
           p->E % world == 0 && p->T > 0 && p->E % 8 == 0 && p->E <= 32 && p->H % 64 == 0;
}

EpLayout make_layout_ep(const moe_problem *p, int world)
{
    EpLayout X{};
    const int el = p->E / world;
    X.pr = *p;
    X.pr.T = world * p->T * std::min(p->top_k, el);
    X.pr.E = el;
    X.pr.top_k = 1;
    X.L = make_layout(&X.pr, 0, false, false, true);
    X.recv_cap = X.L.pmax;
    size_t o = X.L.end_forward;
    auto take = [&](size_t bytes) {
        const size_t at = o;
        o = align256(o + (bytes ? bytes : 1));
        return at;
    };
    const size_t TK = (size_t)p->T * p->top_k;
    X.topk_idx = take(TK * 4);
    X.topk_w = take(TK * 4);
    X.gcount = take(((size_t)p->T + 7) / 8 * p->E * 4);
    X.slot = take(TK * 4);
    X.dest = take(TK * 4);
    X.end = o;
    return X;
}

// Token groups and router ring of one rank's CTAs (ncta = SMs / n_local).
struct EpPlan {
    bool ok;
    int ncta, G, tt, n_groups, ncw, stages;
};

EpPlan ep_plan(const moe_problem *p, int world, int n_local)
{
    EpPlan f{};
    const int sms = sm_count() > 0 ? sm_count() : 148;
    f.ncta = sms / n_local;
    f.G = p->E <= 8 ? 2 : p->E <= 16 ? 4 : 8; // consumer threads per token (4 experts each)
    f.tt = std::max(8, std::min(256 / f.G, (p->T + f.ncta - 1) / f.ncta));
    f.n_groups = (p->T + f.tt - 1) / f.tt;
    f.ncw = (f.tt * f.G + 31) / 32;
    const int budget = gemm::STAGES * gemm::STAGE;
    f.stages = RC_MAX_STAGES;
    while (f.stages > 3 && rc_layout(f.tt, p->E, 4 * f.G, f.stages).total > budget) --f.stages;
    const int el = p->E / world;
    f.ok = f.ncta >= 1 && rc_layout(f.tt, p->E, 4 * f.G, f.stages).total <= budget &&
           (int64_t)ep_scratch_ints(world, p->E, el, f.n_groups) * 4 <= budget;
    return f;
}

template <int KIND0>
cudaError_t launch_ep_layer(const EpLaunch &L, int grid, cudaStream_t st)
{
    auto kern = moe_ep_layer_kernel<KIND0>;
    cudaError_t err =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, gemm::SMEM_BYTES);
    if (err != cudaSuccess) return err;
    kern<<<grid, gemm::NUM_THREADS_GATHER, gemm::SMEM_BYTES, st>>>(L);
    return cudaGetLastError();
}

moe_status ep_layer_impl(const moe_ep_rank *ranks, int n_local, cudaStream_t st)
{
    if (ranks == nullptr || n_local < 1 || n_local > MOE_EP_MAX_LOCAL) return MOE_ERR_INVALID_ARG;
    const moe_problem *p = &ranks[0].p;
    const int world = ranks[0].world;
    if (!ep_shape_ok(p, world)) return MOE_ERR_INVALID_ARG;
    const EpPlan plan = ep_plan(p, world, n_local);
    if (!plan.ok) return MOE_ERR_INVALID_ARG;
    const EpLayout X = make_layout_ep(p, world);
    const int el = p->E / world;
    const int F = p->F, H = p->H;
    const bool gated = (p->act == MOE_ACT_SWIGLU);
    static_assert(MOE_EP_MAX_LOCAL == EP_MAX_LOCAL && MOE_EP_MAX_WORLD == EP_MAX_WORLD, "limits");
    auto *Lp = new EpLaunch(); // large: kept off the stack
    std::unique_ptr<EpLaunch> hold(Lp);
    EpLaunch &L = *Lp;
    L.n_local = n_local;
    for (int i = 0; i < n_local; ++i) {
        const moe_ep_rank &R = ranks[i];
        const moe_problem &q = R.p;
        if (q.T != p->T || q.H != p->H || q.F != p->F || q.E != p->E || q.top_k != p->top_k ||
            q.act != p->act || q.gate != p->gate || R.world != world || R.rank < 0 ||
            R.rank >= world || R.epoch <= 0)
            return MOE_ERR_INVALID_ARG;
        for (int j = 0; j < i; ++j)
            if (ranks[j].rank == R.rank) return MOE_ERR_INVALID_ARG;
        if (R.ws == nullptr || R.ws_bytes < X.end) return MOE_ERR_WORKSPACE;
        if (R.x == nullptr || R.Wg == nullptr || R.W1 == nullptr || R.W2 == nullptr ||
            R.out == nullptr || !aligned16(R.x) || !aligned16(R.Wg) || !aligned16(R.W1) ||
            !aligned16(R.W2) || !aligned16(R.out) || !aligned16(R.ws) || !aligned4(R.bias) ||
            !aligned4(R.topk_idx) || !aligned4(R.topk_w))
            return MOE_ERR_INVALID_ARG;
        for (int b = 0; b < MOE_EP_NUM_BUFFERS; ++b)
            for (int d = 0; d < world; ++d)
                if (R.buf[b][d] == nullptr || !aligned16(R.buf[b][d])) return MOE_ERR_INVALID_ARG;

        void *ws = R.ws;
        const Layout &LL = X.L;
        const DispatchOut d = dispatch_bufs(ws, LL);
        int *status = at<int>(ws, LL.status);
        moe_bf16 *h = at<moe_bf16>(ws, LL.h);
        int32_t *topk_idx = R.topk_idx ? R.topk_idx : at<int32_t>(ws, X.topk_idx);
        float *topk_w = R.topk_w ? R.topk_w : at<float>(ws, X.topk_w);
        auto *recv_rows = reinterpret_cast<const moe_bf16 *>(R.buf[2][R.rank]);
        EpRankMaps &m = L.maps[i];
        if (!make_map_2d(&m.a0, recv_rows, (uint64_t)X.recv_cap, (uint64_t)H, gemm::BM) ||
            !make_map_3d(&m.w1, R.W1, (uint64_t)el, (uint64_t)H, (uint64_t)(gated ? 2 * F : F)) ||
            !make_map_2d(&m.h, h, (uint64_t)X.recv_cap, (uint64_t)F, gemm::BM) ||
            !make_map_3d(&m.w2, R.W2, (uint64_t)el, (uint64_t)F, (uint64_t)H) ||
            !make_map_2d(&m.rx, R.x, (uint64_t)p->T, (uint64_t)H, (uint32_t)plan.tt) ||
            !make_map_2d_plain(&m.rw, R.Wg, (uint64_t)H, (uint64_t)p->E, (uint32_t)p->E, RC_HC))
            return MOE_ERR_CUDA;

        GemmArgs a0{};
        a0.tile_off = d.tile_off;
        a0.tile_expert = d.tile_expert;
        a0.ptile_off = d.ptile_off;
        a0.ptile_expert = d.ptile_expert;
        a0.expert_rows = d.counts;
        a0.hot_off = d.hot_off;
        a0.hot_tile_expert = d.hot_tile_expert;
        a0.cold_tile = d.cold_tile;
        a0.meta = d.meta;
        a0.gather_len = X.recv_cap;
        a0.out = reinterpret_cast<__nv_bfloat16 *>(h);
        a0.ld_out = F;
        a0.n_cols = F;
        a0.k_blocks = H / gemm::BK;
        a0.up_col = F;
        a0.act = p->act;
        a0.status = status;
        a0.timeout_ns = g_timeout_ns.load();
        a0.n_tiles = gated ? (F + 127) / 128 : (F + gemm::BN - 1) / gemm::BN;
        GemmArgs a1 = a0;
        a1.row_w = reinterpret_cast<const float *>(R.buf[3][R.rank]);
        a1.out = reinterpret_cast<__nv_bfloat16 *>(h); // unused: every row is returned or skipped
        a1.row_dst = reinterpret_cast<const long long *>(R.buf[4][R.rank]);
        for (int dd = 0; dd < world; ++dd) a1.peer_out[dd] = reinterpret_cast<__nv_bfloat16 *>(R.buf[6][dd]);
        a1.ld_out = H;
        a1.n_cols = H;
        a1.n_tiles = (H + gemm::BN - 1) / gemm::BN;
        a1.k_blocks = F / gemm::BK;

        FusedArgs &fa = L.fa[i];
        fa = FusedArgs{};
        fa.l0 = a0;
        fa.l1 = a1;
        fa.ready0 = d.ready;
        fa.ready1 = d.ready + LL.max_tiles;
        fa.done0 = d.ready + LL.n_ready - 2;
        fa.comb_next = d.ready + LL.n_ready - 1;
        fa.max_tiles = LL.max_tiles;
        fa.inv_pos = d.inv_pos;
        fa.out = reinterpret_cast<__nv_bfloat16 *>(R.out);
        fa.T = p->T;
        fa.H = H;
        fa.k = p->top_k;
        fa.ys_rows = (int64_t)p->T * p->top_k;
        fa.a_tma = 1;
        fa.comb_tokens = fused_plan(p).comb_tokens;
        fa.comb_in_launch = 1; // the combine of the returned rows is part of the EP launch
        fa.fault_skip = -1;
        fa.trace = i == 0 ? g_trace.load() : nullptr;
        fa.trace_cap = g_trace_cap.load();
        FrontArgs &f = fa.front;
        f.ra.bias = R.bias;
        f.ra.topk_idx = topk_idx;
        f.ra.topk_w = topk_w;
        f.ra.T = p->T;
        f.ra.H = H;
        f.ra.E = p->E;
        f.ra.k = p->top_k;
        f.ra.gate = p->gate;
        f.ra.tt = plan.tt;
        f.ra.stages = plan.stages;
        f.ra.status = status;
        f.ra.timeout_ns = a0.timeout_ns;
        f.ra.group_counts = at<int32_t>(ws, X.gcount);
        f.ncw = plan.ncw;
        f.n_groups = plan.n_groups;
        f.fd.T = p->T;
        f.fd.E = el;
        f.fd.k = p->top_k;
        f.fd.H = H;
        f.fd.x = reinterpret_cast<const __nv_bfloat16 *>(R.x);
        f.fd.so = scan_out(LL, d);
        f.fd.so.row_w = reinterpret_cast<float *>(R.buf[3][R.rank]); // pad rows: gate 0
        f.gbar = status + 4;
        EpArgs &ep = fa.ep;
        ep.world = world;
        ep.rank = R.rank;
        ep.e_loc = el;
        ep.epoch = R.epoch;
        for (int dd = 0; dd < world; ++dd) {
            ep.all_counts[dd] = reinterpret_cast<int32_t *>(R.buf[0][dd]);
            ep.flags[dd] = reinterpret_cast<int *>(R.buf[1][dd]);
            ep.recv_rows[dd] = reinterpret_cast<__nv_bfloat16 *>(R.buf[2][dd]);
            ep.recv_gate[dd] = reinterpret_cast<float *>(R.buf[3][dd]);
            ep.recv_origin[dd] = reinterpret_cast<long long *>(R.buf[4][dd]);
            ep.arrive[dd] = reinterpret_cast<int *>(R.buf[5][dd]);
            ep.back[dd] = reinterpret_cast<__nv_bfloat16 *>(R.buf[6][dd]);
            ep.back_cnt[dd] = reinterpret_cast<int *>(R.buf[7][dd]);
        }
        ep.recv_cap = X.recv_cap;
        ep.max_tiles = LL.max_tiles;
        ep.slot = at<int32_t>(ws, X.slot);
        ep.dest = at<int32_t>(ws, X.dest);
        // status word and grid-barrier counter start from zero
        cudaError_t e = cudaMemsetAsync(status, 0, 32, st);
        if (e != cudaSuccess) return MOE_ERR_CUDA;
    }
    const int grid = n_local * plan.ncta;
    const cudaError_t e = gated ? launch_ep_layer<GEMM_SWIGLU>(L, grid, st)
                                : launch_ep_layer<GEMM_ACT>(L, grid, st);
    return to_status(e);
}

extern "C" {

int moe_forward_launches(const moe_problem *p)
{
    if (check_problem(p) != MOE_OK) return -1;
    if (p->T == 0) return 0;
    // filter: prep, GEMM, exact; up to 32 experts: one launch; else logits, top-k
    const int route = route_uses_filter(p) ? 3 : route_uses_chain(p) ? 1 : 2;
    // count, scan, place; one block for a single chunk of tokens
    const int dispatch = p->T <= DISPATCH_CHUNK ? 1 : 3;
    const int mode = g_gemm_mode.load();
    const bool pair = mode == MOE_GEMM_CTA_PAIR;
    // + the x_perm gather (CTA pairs, large batches); then layer0, layer1, combine, or the one
    // persistent launch
    const int gather = (pair || use_x_perm(p)) ? 1 : 0;
    const int layers = (!pair && run_fused(p)) ? (fused_combine_in_launch() ? 1 : 2) : 3;
    return whole_layer(p) ? 1 : route + dispatch + gather + layers;
}

int moe_set_whole_layer_launch(int on)
{
    return g_front.exchange(on != 0 ? 1 : 0);
}

size_t moe_workspace_size(const moe_problem *p)
{
    if (check_problem(p) != MOE_OK) return 0;
    return make_layout(p).end_host;
}

int64_t moe_padded_rows_max(const moe_problem *p)
{
    if (check_problem(p) != MOE_OK) return -1;
    return padded_rows_max(p);
}

moe_status moe_route(const moe_problem *p, const moe_bf16 *x, const moe_bf16 *Wg, const float *bias,
                     int32_t *topk_idx, float *topk_w, void *ws, size_t ws_bytes, void *stream)
{
    moe_status s = check_problem(p);
    if (s != MOE_OK) return s;
    if (ws == nullptr || Wg == nullptr) return MOE_ERR_INVALID_ARG;
    if (p->T > 0 && (x == nullptr || topk_idx == nullptr || topk_w == nullptr))
        return MOE_ERR_INVALID_ARG;
    const Layout L = make_layout(p);
    if (ws_bytes < L.end_route) return MOE_ERR_WORKSPACE;
    if (!aligned16(x) || !aligned16(Wg) || !aligned16(ws) || !aligned4(bias) || !aligned4(topk_idx) ||
        !aligned4(topk_w))
        return MOE_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int *status = at<int>(ws, L.status);
    if (p->T == 0) return to_status(cudaMemsetAsync(status, 0, 8, st));
    const FilterBufs fb = filter_bufs(ws, L);
    return to_status(
        launch_route(p, x, Wg, bias, topk_idx, topk_w, at<float>(ws, L.logits), status, st, &fb));
}

moe_status moe_route_noalloc(const moe_problem *p, const moe_bf16 *x, const moe_bf16 *Wg,
                             const float *bias, int32_t *topk_idx, float *topk_w, void *stream)
{
    moe_status s = check_problem(p);
    if (s != MOE_OK) return s;
    if (Wg == nullptr) return MOE_ERR_INVALID_ARG;
    if (p->T > 0 && (x == nullptr || topk_idx == nullptr || topk_w == nullptr))
        return MOE_ERR_INVALID_ARG;
    if ((int64_t)p->T * p->E > (int64_t)MOE_ROUTE_NOALLOC_MAX_LOGITS) return MOE_ERR_UNSUPPORTED;
    if (!aligned16(x) || !aligned16(Wg) || !aligned4(bias) || !aligned4(topk_idx) || !aligned4(topk_w))
        return MOE_ERR_INVALID_ARG;
    if (p->T == 0) return MOE_OK;
    float *logits = route_noalloc_scratch();
    if (logits == nullptr) return MOE_ERR_CUDA;
    // the router kernels overwrite every logit before reading it: nothing to clear; there is
    // no status word to report through (the router raises no device errors)
    return to_status(launch_route(p, x, Wg, bias, topk_idx, topk_w, logits, nullptr,
                                  static_cast<cudaStream_t>(stream)));
}

moe_status moe_dispatch(const moe_problem *p, const int32_t *topk_idx, int32_t *counts,
                        int32_t *offsets, int32_t *padded_offsets, int32_t *gather_idx,
                        int32_t *inv_pos, moe_bf16 *x_perm, const moe_bf16 *x, void *ws,
                        size_t ws_bytes, void *stream)
{
    moe_status s = check_problem(p);
    if (s != MOE_OK) return s;
    if (ws == nullptr || counts == nullptr || offsets == nullptr || padded_offsets == nullptr ||
        gather_idx == nullptr)
        return MOE_ERR_INVALID_ARG;
    if (p->T > 0 && (topk_idx == nullptr || inv_pos == nullptr)) return MOE_ERR_INVALID_ARG;
    if (x_perm != nullptr && x == nullptr) return MOE_ERR_INVALID_ARG;
    const Layout L = make_layout(p);
    if (ws_bytes < L.end_dispatch) return MOE_ERR_WORKSPACE;
    if (!aligned16(ws) || !aligned16(x_perm) || !aligned16(x) || !aligned4(topk_idx) ||
        !aligned4(counts) || !aligned4(offsets) || !aligned4(padded_offsets) ||
        !aligned4(gather_idx) || !aligned4(inv_pos))
        return MOE_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int *status = at<int>(ws, L.status);
    cudaError_t e = cudaSuccess;
    if (p->T == 0) e = cudaMemsetAsync(status, 0, 8, st);
    DispatchOut d;
    d.counts = counts;
    d.offsets = offsets;
    d.poff = padded_offsets;
    d.gather_idx = gather_idx;
    d.inv_pos = inv_pos;
    d.tile_off = at<int32_t>(ws, L.tile_off);
    d.tile_expert = at<int32_t>(ws, L.tile_expert);
    d.chunk = at<int32_t>(ws, L.chunk);
    d.ptile_off = at<int32_t>(ws, L.ptile_off);
    d.ptile_expert = at<int32_t>(ws, L.ptile_expert);
    d.hot_off = at<int32_t>(ws, L.hot_off);
    d.hot_tile_expert = at<int32_t>(ws, L.hot_tile_expert);
    d.cold_tile = at<int32_t>(ws, L.cold_tile);
    d.ready = nullptr;
    d.n_ready = 0;
    d.row_w = nullptr;
    d.meta = at<DispatchMeta>(ws, L.meta);
    if (e == cudaSuccess) e = launch_dispatch(p, L, topk_idx, nullptr, d, status, 1, st);
    if (e == cudaSuccess && x_perm != nullptr)
        e = launch_gather(p, x, gather_idx, d.meta, x_perm, st);
    return to_status(e);
}

moe_status moe_forward(const moe_problem *p, const moe_bf16 *x, const moe_bf16 *Wg, const float *bias,
                       const moe_bf16 *W1, const moe_bf16 *W2, moe_bf16 *out, int32_t *topk_idx_out,
                       float *topk_w_out, void *ws, size_t ws_bytes, void *stream)
{
    return forward_impl(p, x, Wg, bias, W1, W2, out, topk_idx_out, topk_w_out, ws, ws_bytes,
                        static_cast<cudaStream_t>(stream), nullptr, 0);
}

moe_status moe_forward_staged(const moe_problem *p, const moe_bf16 *x, const moe_bf16 *Wg,
                              const float *bias, const moe_bf16 *W1, const moe_bf16 *W2,
                              moe_bf16 *out, int32_t *topk_idx_out, float *topk_w_out, void *ws,
                              size_t ws_bytes, void *stream, void *const *events, int n_events)
{
    return forward_impl(p, x, Wg, bias, W1, W2, out, topk_idx_out, topk_w_out, ws, ws_bytes,
                        static_cast<cudaStream_t>(stream), events, n_events);
}

// Two copy streams and per-slot events for moe_forward_host_batches, created once per device.
struct HostPipe {
    cudaStream_t h2d = nullptr, d2h = nullptr;
    cudaEvent_t start = nullptr, h2d_done[2] = {}, comp_done[2] = {}, d2h_done[2] = {};
    bool ok = false;
};
HostPipe *host_pipe()
{
    static std::mutex mu;
    static HostPipe pipes[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    HostPipe &hp = pipes[dev];
    if (!hp.ok) {
        bool good = cudaStreamCreateWithFlags(&hp.h2d, cudaStreamNonBlocking) == cudaSuccess &&
                    cudaStreamCreateWithFlags(&hp.d2h, cudaStreamNonBlocking) == cudaSuccess &&
                    cudaEventCreateWithFlags(&hp.start, cudaEventDisableTiming) == cudaSuccess;
        for (int i = 0; i < 2 && good; ++i)
            good = cudaEventCreateWithFlags(&hp.h2d_done[i], cudaEventDisableTiming) == cudaSuccess &&
                   cudaEventCreateWithFlags(&hp.comp_done[i], cudaEventDisableTiming) == cudaSuccess &&
                   cudaEventCreateWithFlags(&hp.d2h_done[i], cudaEventDisableTiming) == cudaSuccess;
        if (!good) return nullptr;
        hp.ok = true;
    }
    return &hp;
}

moe_status moe_forward_host(const moe_problem *p, const moe_bf16 *x_host, const moe_bf16 *Wg,
                            const float *bias, const moe_bf16 *W1, const moe_bf16 *W2,
                            moe_bf16 *out_host, void *ws, size_t ws_bytes, void *stream)
{
    moe_status s = check_problem(p);
    if (s != MOE_OK) return s;
    if (ws == nullptr || (p->T > 0 && (x_host == nullptr || out_host == nullptr)))
        return MOE_ERR_INVALID_ARG;
    const Layout L = make_layout(p);
    if (ws_bytes < L.end_host) return MOE_ERR_WORKSPACE;
    if (!aligned16(ws)) return MOE_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t bytes = (size_t)p->T * p->H * 2;
    moe_bf16 *xd = at<moe_bf16>(ws, L.x_stage);
    moe_bf16 *od = at<moe_bf16>(ws, L.out_stage);
    if (bytes > 0 && cudaMemcpyAsync(xd, x_host, bytes, cudaMemcpyHostToDevice, st) != cudaSuccess)
        return MOE_ERR_CUDA;
    s = forward_impl(p, xd, Wg, bias, W1, W2, od, nullptr, nullptr, ws, ws_bytes, st, nullptr, 0);
    if (s != MOE_OK) return s;
    if (bytes > 0 && cudaMemcpyAsync(out_host, od, bytes, cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return MOE_ERR_CUDA;
    return to_status(cudaStreamSynchronize(st));
}

size_t moe_workspace_size_shared(const moe_problem *p, int32_t F_s)
{
    if (check_problem(p) != MOE_OK || F_s <= 0 || F_s % 64 != 0) return 0;
    return make_layout(p, F_s).end_shared;
}

moe_status moe_forward_shared(const moe_problem *p, const moe_bf16 *x, const moe_bf16 *Wg,
                              const float *bias, const moe_bf16 *W1, const moe_bf16 *W2,
                              const moe_shared_expert *shared, moe_bf16 *out,
                              int32_t *topk_idx_out, float *topk_w_out, void *ws,
                              size_t ws_bytes, void *stream)
{
    moe_status s = check_problem(p);
    if (s != MOE_OK) return s;
    if (shared == nullptr || shared->F_s <= 0 || shared->W1s == nullptr || shared->W2s == nullptr)
        return MOE_ERR_INVALID_ARG;
    if (shared->F_s % 64 != 0) return MOE_ERR_UNSUPPORTED;
    if (!aligned16(shared->W1s) || !aligned16(shared->W2s) ||
        (shared->w_sg != nullptr && !aligned16(shared->w_sg)))
        return MOE_ERR_INVALID_ARG;
    if (ws_bytes < make_layout(p, shared->F_s).end_shared) return MOE_ERR_WORKSPACE;
    return forward_impl(p, x, Wg, bias, W1, W2, out, topk_idx_out, topk_w_out, ws, ws_bytes,
                        static_cast<cudaStream_t>(stream), nullptr, 0, shared);
}

moe_status moe_forward_host_batches(const moe_problem *p, int n_batches,
                                    const moe_bf16 *const *x_host, const moe_bf16 *Wg,
                                    const float *bias, const moe_bf16 *W1, const moe_bf16 *W2,
                                    moe_bf16 *const *out_host, void *ws, size_t ws_bytes,
                                    void *stream)
{
    moe_status s = check_problem(p);
    if (s != MOE_OK) return s;
    if (n_batches < 0 || ws == nullptr || (n_batches > 0 && (x_host == nullptr || out_host == nullptr)))
        return MOE_ERR_INVALID_ARG;
    for (int i = 0; i < n_batches && p->T > 0; ++i)
        if (x_host[i] == nullptr || out_host[i] == nullptr) return MOE_ERR_INVALID_ARG;
    const Layout L = make_layout(p);
    if (ws_bytes < L.end_host) return MOE_ERR_WORKSPACE;
    if (!aligned16(ws)) return MOE_ERR_INVALID_ARG;
    if (n_batches == 0) return MOE_OK;
    HostPipe *hp = host_pipe();
    if (hp == nullptr) return MOE_ERR_CUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t bytes = (size_t)p->T * p->H * 2;
    moe_bf16 *xs[2] = {at<moe_bf16>(ws, L.x_stage), at<moe_bf16>(ws, L.x_stage2)};
    moe_bf16 *os[2] = {at<moe_bf16>(ws, L.out_stage), at<moe_bf16>(ws, L.out_stage2)};
    auto ok = [](cudaError_t e) { return e == cudaSuccess; };
    // the copies start after the work already queued on the caller's stream
    if (!ok(cudaEventRecord(hp->start, st)) || !ok(cudaStreamWaitEvent(hp->h2d, hp->start, 0)) ||
        !ok(cudaStreamWaitEvent(hp->d2h, hp->start, 0)))
        return MOE_ERR_CUDA;
    for (int i = 0; i < n_batches; ++i) {
        const int b = i & 1;
        // x slot b is free once batch i-2 computed; out slot b once its copy-out landed
        if (i >= 2 && !ok(cudaStreamWaitEvent(hp->h2d, hp->comp_done[b], 0))) return MOE_ERR_CUDA;
        if (bytes > 0 &&
            !ok(cudaMemcpyAsync(xs[b], x_host[i], bytes, cudaMemcpyHostToDevice, hp->h2d)))
            return MOE_ERR_CUDA;
        if (!ok(cudaEventRecord(hp->h2d_done[b], hp->h2d)) ||
            !ok(cudaStreamWaitEvent(st, hp->h2d_done[b], 0)) ||
            (i >= 2 && !ok(cudaStreamWaitEvent(st, hp->d2h_done[b], 0))))
            return MOE_ERR_CUDA;
        s = forward_impl(p, xs[b], Wg, bias, W1, W2, os[b], nullptr, nullptr, ws, ws_bytes, st,
                         nullptr, 0);
        if (s != MOE_OK) return s;
        if (!ok(cudaEventRecord(hp->comp_done[b], st)) ||
            !ok(cudaStreamWaitEvent(hp->d2h, hp->comp_done[b], 0)))
            return MOE_ERR_CUDA;
        if (bytes > 0 &&
            !ok(cudaMemcpyAsync(out_host[i], os[b], bytes, cudaMemcpyDeviceToHost, hp->d2h)))
            return MOE_ERR_CUDA;
        if (!ok(cudaEventRecord(hp->d2h_done[b], hp->d2h))) return MOE_ERR_CUDA;
    }
    // the caller's stream continues after the last copy-out; wait for it here
    if (!ok(cudaStreamWaitEvent(st, hp->d2h_done[(n_batches - 1) & 1], 0))) return MOE_ERR_CUDA;
    return to_status(cudaStreamSynchronize(st));
}

moe_status moe_combine(const moe_problem *p, const moe_bf16 *ys, int64_t ys_rows,
                       const int32_t *inv_pos, moe_bf16 *out, void *ws, size_t ws_bytes, void *stream)
{
    moe_status s = check_problem(p);
    if (s != MOE_OK) return s;
    if (p->T > 0 && (ys == nullptr || inv_pos == nullptr || out == nullptr)) return MOE_ERR_INVALID_ARG;
    if (ys_rows < 0) return MOE_ERR_INVALID_ARG;
    if (!aligned16(ys) || !aligned16(out) || !aligned4(inv_pos) || !aligned16(ws))
        return MOE_ERR_INVALID_ARG;
    int *status = nullptr;
    if (ws != nullptr) {
        if (ws_bytes < 256) return MOE_ERR_WORKSPACE;
        status = at<int>(ws, 0);
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (p->T == 0) return status ? to_status(cudaMemsetAsync(status, 0, 8, st)) : MOE_OK;
    return to_status(launch_combine(p, ys, ys_rows, inv_pos, out, status, 1, st));
}

moe_status moe_get_device_status(void *ws, void *stream)
{
    if (ws == nullptr || !aligned16(ws)) return MOE_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return MOE_ERR_CUDA;
    int host[2] = {0, 0};
    if (cudaMemcpy(host, ws, sizeof(host), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
    const int zero[2] = {0, 0};
    if (cudaMemcpy(ws, zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return MOE_ERR_CUDA;
    switch (host[0]) {
    case DEV_OK: return MOE_OK;
    case DEV_TIMEOUT: return MOE_ERR_DEVICE_TIMEOUT;
    case DEV_BAD_INDEX: return MOE_ERR_DEVICE_BAD_INDEX;
    default: return MOE_ERR_CUDA;
    }
}

const char *moe_status_string(moe_status s)
{
    switch (s) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_DEVICE_TIMEOUT: return "MOE_ERR_DEVICE_TIMEOUT";
    case MOE_ERR_DEVICE_BAD_INDEX: return "MOE_ERR_DEVICE_BAD_INDEX";
    }
    return "MOE_UNKNOWN_STATUS";
}

int64_t moe_set_wait_timeout_ns(int64_t ns)
{
    return g_timeout_ns.exchange(ns > 0 ? ns : kDefaultTimeoutNs);
}

int moe_set_gemm_mode(int mode)
{
    if (mode != MOE_GEMM_AUTO && mode != MOE_GEMM_SINGLE_CTA && mode != MOE_GEMM_CTA_PAIR &&
        mode != MOE_GEMM_FUSED && mode != MOE_GEMM_FUSED_LAYERS)
        return -1;
    return g_gemm_mode.exchange(mode);
}

int moe_set_work_order(int order)
{
    if (order != MOE_ORDER_EXPERT && order != MOE_ORDER_MIXED && order != MOE_ORDER_NARROW &&
        order != MOE_ORDER_PHASED)
        return -1;
    return g_order.exchange(order);
}

int moe_set_router_mode(int mode)
{
    if (mode != MOE_ROUTER_AUTO && mode != MOE_ROUTER_SEQUENTIAL && mode != MOE_ROUTER_FILTER)
        return -1;
    return g_router_mode.exchange(mode);
}

int moe_route_uses_filter(const moe_problem *p)
{
    if (check_problem(p) != MOE_OK) return -1;
    return route_uses_filter(p) ? 1 : 0;
}

size_t moe_workspace_size_fp8(const moe_problem *p)
{
    if (check_problem_fp8(p) != MOE_OK) return 0;
    return make_layout(p, 0, true).end_fp8;
}

moe_status moe_quantize_rows_fp8(const moe_bf16 *src, int64_t rows, int32_t cols, moe_fp8 *dst,
                                 float *scale, void *stream)
{
    if (rows < 0 || cols <= 0 || cols % 8 != 0) return MOE_ERR_INVALID_ARG;
    if (rows == 0) return MOE_OK;
    if (src == nullptr || dst == nullptr || scale == nullptr || !aligned16(src) ||
        (reinterpret_cast<uintptr_t>(dst) & 7u) != 0 || !aligned4(scale))
        return MOE_ERR_INVALID_ARG;
    return to_status(launch_quant_rows(src, rows, cols, nullptr, dst, scale,
                                       static_cast<cudaStream_t>(stream)));
}

moe_status moe_quantize_experts_fp8(const moe_problem *p, const moe_bf16 *W1, const moe_bf16 *W2,
                                    moe_fp8 *W1q, float *s1, moe_fp8 *W2q, float *s2, void *stream)
{
    moe_status s = check_problem_fp8(p);
    if (s != MOE_OK) return s;
    if (W1 == nullptr || W2 == nullptr || W1q == nullptr || W2q == nullptr || s1 == nullptr ||
        s2 == nullptr)
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(W1) || !aligned16(W2) || !aligned16(W1q) || !aligned16(W2q) || !aligned16(s1) ||
        !aligned16(s2))
        return MOE_ERR_INVALID_ARG;
    const int w1_cols = p->act == MOE_ACT_SWIGLU ? 2 * p->F : p->F;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = launch_quant_cols(W1, p->E, p->H, w1_cols, W1q, s1, st);
    if (e == cudaSuccess) e = launch_quant_cols(W2, p->E, p->F, p->H, W2q, s2, st);
    return to_status(e);
}

moe_status moe_forward_fp8(const moe_problem *p, const moe_bf16 *x, const moe_bf16 *Wg,
                           const float *bias, const moe_fp8 *W1q, const float *s1,
                           const moe_fp8 *W2q, const float *s2, moe_bf16 *out,
                           int32_t *topk_idx_out, float *topk_w_out, void *ws, size_t ws_bytes,
                           void *stream)
{
    return forward_impl_fp8(p, x, Wg, bias, W1q, s1, W2q, s2, out, topk_idx_out, topk_w_out, ws,
                            ws_bytes, static_cast<cudaStream_t>(stream), nullptr, 0);
}

moe_status moe_forward_fp8_staged(const moe_problem *p, const moe_bf16 *x, const moe_bf16 *Wg,
                                  const float *bias, const moe_fp8 *W1q, const float *s1,
                                  const moe_fp8 *W2q, const float *s2, moe_bf16 *out,
                                  int32_t *topk_idx_out, float *topk_w_out, void *ws,
                                  size_t ws_bytes, void *stream, void *const *events,
                                  int32_t n_events)
{
    return forward_impl_fp8(p, x, Wg, bias, W1q, s1, W2q, s2, out, topk_idx_out, topk_w_out, ws,
                            ws_bytes, static_cast<cudaStream_t>(stream), events, n_events);
}

moe_status moe_experts_forward(const moe_problem *p, const moe_bf16 *x, const int32_t *expert,
                               const float *gate, const moe_bf16 *W1, const moe_bf16 *W2,
                               moe_bf16 *out, void *ws, size_t ws_bytes, void *stream)
{
    if (p != nullptr && p->top_k != 1) return MOE_ERR_INVALID_ARG;
    if (p != nullptr && p->T > 0 && (expert == nullptr || gate == nullptr || !aligned4(expert) ||
                                     !aligned4(gate)))
        return MOE_ERR_INVALID_ARG;
    return forward_impl(p, x, nullptr, nullptr, W1, W2, out, nullptr, nullptr, ws, ws_bytes,
                        static_cast<cudaStream_t>(stream), nullptr, 0, nullptr,
                        p != nullptr && p->T > 0 ? expert : nullptr, gate);
}

moe_status moe_experts_forward_n(const moe_problem *p, const moe_bf16 *x, const int32_t *expert,
                                 const float *gate, const int32_t *n_rows, const moe_bf16 *W1,
                                 const moe_bf16 *W2, moe_bf16 *out, void *ws, size_t ws_bytes,
                                 void *stream)
{
    if (p != nullptr && p->top_k != 1) return MOE_ERR_INVALID_ARG;
    if (p != nullptr && p->T > 0 &&
        (expert == nullptr || gate == nullptr || n_rows == nullptr || !aligned4(expert) ||
         !aligned4(gate) || !aligned4(n_rows)))
        return MOE_ERR_INVALID_ARG;
    return forward_impl(p, x, nullptr, nullptr, W1, W2, out, nullptr, nullptr, ws, ws_bytes,
                        static_cast<cudaStream_t>(stream), nullptr, 0, nullptr,
                        p != nullptr && p->T > 0 ? expert : nullptr, gate,
                        p != nullptr && p->T > 0 ? n_rows : nullptr);
}

moe_status moe_ep_publish_counts(const moe_problem *p, int32_t world, int32_t rank,
                                 const int32_t *offsets, int32_t *const *tables, void *stream)
{
    moe_status s = check_problem(p);
    if (s != MOE_OK) return s;
    if (world < 1 || rank < 0 || rank >= world || p->E % world != 0 || offsets == nullptr ||
        tables == nullptr)
        return MOE_ERR_INVALID_ARG;
    ep_publish_counts_kernel<<<1, 256, 0, static_cast<cudaStream_t>(stream)>>>(
        offsets, p->E / world, world, rank, tables);
    return to_status(cudaGetLastError());
}

moe_status moe_ep_scatter(const moe_problem *p, int32_t world, int32_t rank, const moe_bf16 *x,
                          const int32_t *topk_idx, const float *topk_w, const int32_t *offsets,
                          const int32_t *padded_offsets, const int32_t *inv_pos,
                          const int32_t *table, moe_bf16 *const *rows, int32_t *const *ids,
                          float *const *gates, int64_t *const *origin, int64_t recv_cap,
                          int32_t *n_recv, void *ws, size_t ws_bytes, void *stream)
{
    moe_status s = check_problem(p);
    if (s != MOE_OK) return s;
    if (world < 1 || rank < 0 || rank >= world || p->E % world != 0 || recv_cap < 0 ||
        (int64_t)p->T * p->top_k >= ((int64_t)1 << 31))
        return MOE_ERR_INVALID_ARG;
    if (ws == nullptr || n_recv == nullptr || table == nullptr || rows == nullptr ||
        ids == nullptr || gates == nullptr || origin == nullptr ||
        (p->T > 0 && (x == nullptr || topk_idx == nullptr || topk_w == nullptr ||
                      offsets == nullptr || padded_offsets == nullptr || inv_pos == nullptr)))
        return MOE_ERR_INVALID_ARG;
    const Layout L = make_layout(p);
    if (ws_bytes < L.end_route) return MOE_ERR_WORKSPACE;
    if (!aligned16(x)) return MOE_ERR_INVALID_ARG;
    EpScatterArgs a{};
    a.x = reinterpret_cast<const __nv_bfloat16 *>(x);
    a.topk_idx = topk_idx;
    a.topk_w = topk_w;
    a.offsets = offsets;
    a.poff = padded_offsets;
    a.inv_pos = inv_pos;
    a.table = table;
    a.rows = reinterpret_cast<__nv_bfloat16 *const *>(rows);
    a.ids = ids;
    a.gates = gates;
    a.origin = reinterpret_cast<long long *const *>(origin);
    a.recv_cap = recv_cap;
    a.n_recv = n_recv;
    a.T = p->T;
    a.H = p->H;
    a.E = p->E;
    a.k = p->top_k;
    a.E_loc = p->E / world;
    a.world = world;
    a.rank = rank;
    a.status = at<int>(ws, L.status);
    const int64_t pairs = (int64_t)p->T * p->top_k;
    int64_t blocks = (pairs * 32 + 255) / 256;
    const int64_t cap = (int64_t)(sm_count() > 0 ? sm_count() : 148) * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    ep_scatter_kernel<<<(int)blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(a);
    return to_status(cudaGetLastError());
}

moe_status moe_ep_return(int32_t H, int32_t world, const moe_bf16 *y, const int64_t *origin,
                         const int32_t *n_recv, int64_t recv_cap, moe_bf16 *const *back,
                         int64_t back_rows, void *ws, void *stream)
{
    if (H <= 0 || H % 64 != 0 || world < 1 || y == nullptr || origin == nullptr ||
        n_recv == nullptr || back == nullptr || ws == nullptr || recv_cap < 0 || back_rows < 0 ||
        !aligned16(y) || !aligned16(ws))
        return MOE_ERR_INVALID_ARG;
    int64_t blocks = (recv_cap * 32 + 255) / 256;
    const int64_t cap = (int64_t)(sm_count() > 0 ? sm_count() : 148) * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    ep_return_kernel<<<(int)blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(
        reinterpret_cast<const __nv_bfloat16 *>(y), reinterpret_cast<const long long *>(origin),
        n_recv, H, world, back_rows, reinterpret_cast<__nv_bfloat16 *const *>(back),
        static_cast<int *>(ws));
    return to_status(cudaGetLastError());
}

moe_status moe_ep_buffer_sizes(const moe_problem *p, int32_t world, int64_t *sizes)
{
    if (sizes == nullptr || !ep_shape_ok(p, world)) return MOE_ERR_INVALID_ARG;
    const EpLayout X = make_layout_ep(p, world);
    const int64_t T = p->T, H = p->H, E = p->E, k = p->top_k;
    sizes[0] = (int64_t)world * ((T + 7) / 8) * E * 4; // counts [world][groups][E]
    sizes[1] = (int64_t)world * 4;                     // flags
    sizes[2] = X.recv_cap * H * 2;                     // recv_rows
    sizes[3] = X.recv_cap * 4;                         // recv_gate
    sizes[4] = X.recv_cap * 8;                         // recv_origin
    sizes[5] = (int64_t)X.L.max_tiles * 4;             // arrive
    sizes[6] = T * k * H * 2;                          // back
    sizes[7] = T * ((H + gemm::BN - 1) / gemm::BN) * 4; // back_cnt [T][stripes]
    return MOE_OK;
}

size_t moe_ep_workspace_size(const moe_problem *p, int32_t world)
{
    if (!ep_shape_ok(p, world)) return 0;
    return make_layout_ep(p, world).end;
}

moe_status moe_ep_layer_forward(const moe_ep_rank *ranks, int32_t n_local, void *stream)
{
    return ep_layer_impl(ranks, n_local, reinterpret_cast<cudaStream_t>(stream));
}

size_t moe_backward_workspace_size(const moe_problem *p)
{
    if (check_problem_bwd(p) != MOE_OK) return 0;
    return make_layout(p, 0, false, true).end_bwd;
}

moe_status moe_backward(const moe_problem *p, const moe_bf16 *x, const moe_bf16 *Wg,
                        const float *bias, const moe_bf16 *W1, const moe_bf16 *W2,
                        const moe_bf16 *dout, moe_bf16 *dx, float *dWg, float *dbias,
                        moe_bf16 *dW1, moe_bf16 *dW2, void *ws, size_t ws_bytes, void *stream)
{
    return backward_impl(p, x, Wg, bias, W1, W2, dout, dx, dWg, dbias, dW1, dW2, ws, ws_bytes,
                         static_cast<cudaStream_t>(stream));
}

moe_status moe_set_schedule_trace(void *records, int64_t capacity)
{
    if (capacity < 0) return MOE_ERR_INVALID_ARG;
    g_trace_cap.store(records == nullptr ? 0 : capacity);
    g_trace.store(static_cast<unsigned long long *>(records));
    return MOE_OK;
}

int moe_set_fault_injection(int layer0_item)
{
    return g_fault_skip.exchange(layer0_item < 0 ? -1 : layer0_item);
}

} // extern "C"
