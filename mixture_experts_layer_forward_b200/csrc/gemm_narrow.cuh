// gemm_narrow.cuh -- grouped GEMM for the experts that own a single m-tile, with the operands
// swapped so the MMA's N is the expert's row count instead of a padded 128.
//
// With a skewed expert prior (and in decode) many experts receive only a few token rows.
// In the 128-row tiles of gemm_tc.cuh such an expert still costs a full 128 x 256 x K MMA
// per item, almost all of it on padding rows, while its weights are streamed for that one
// tile only. Here the tensor cores compute the transposed product
//     D^T [weight columns x rows] = W^T [weight columns x K] . X^T [K x rows]
// with M = 128 weight columns (A = the weight tile, MN-major as stored) and N = the expert's
// row count rounded up to 16 (B = the token rows, K-major). The weights are still read once
// per item, but the tensor-core work and its energy shrink with the row count.
//
// Work items: (cold expert j, block of 128 weight columns), expert-major, a static
// round-robin over the CTAs of the narrow group (moe_grouped_gemm_split_kernel below runs
// this group beside the 128-row kernel's). Kinds as in gemm_tc.cuh:
//   GEMM_SWIGLU  A = [64 gate columns | the matching 64 up columns] of W1[e]; B = the
//                expert's x rows (gathered in-kernel by four cp.async warps);
//                h[row][64 cb + c] = silu(gate) * up. The epilogue warps holding the up
//                lanes hand their values to the gate lanes through shared memory.
//   GEMM_ACT     A = 128 columns of W1[e]; h = act(acc).
//   GEMM_SCALE   A = 128 columns of W2[e]; B = the expert's h rows (one TMA box);
//                ys[row][col] = row_w[row] * acc.
// Roles, barriers, bounded waits and TMEM handling follow gemm_tc.cuh: warp 0 TMA producer,
// warp 1 MMA issuer (two accumulators of up to 128 columns), warps 2-5 epilogue, warps 6-9
// layer0 row gather.
// e4m3 operands (F8): the weight codes are K-major ([E, N rows, K]), so A is two boxes of 64
// weight rows x 128 K bytes (the same 8 KB per box), both operands K-major, the MMA
// kind::f8f6f4; the epilogue multiplies each accumulator by its row's and column's scales
// first (as gemm_tc.cuh's).
#pragma once

#include "gemm_tc.cuh"

namespace moe {

namespace gemmn {
constexpr int BM = 128;                  // weight columns per item (the MMA's M)
constexpr int BK = 64;
constexpr int STAGES = 5;
constexpr int A_BOX = 64 * BK * 2;       // 8 KB: 64 weight columns x 64 K
constexpr int A_TILE = 2 * A_BOX;        // 16 KB
constexpr int B_TILE = 128 * BK * 2;     // 16 KB: up to 128 token rows x 64 K
constexpr int STAGE = A_TILE + B_TILE;   // 32 KB
constexpr int XCH_LD = 129;              // up -> gate hand-off, floats per column
constexpr int XCH_BYTES = 64 * XCH_LD * 4;
constexpr int NUM_THREADS = 192;
constexpr int GATHER_THREADS = 128;
constexpr int NUM_THREADS_GATHER = NUM_THREADS + GATHER_THREADS;
constexpr int NUM_BARS = 2 * STAGES + 5;
constexpr int SMEM_BYTES = 1024 + STAGES * STAGE + XCH_BYTES + NUM_BARS * 8 + 16;
constexpr uint32_t TMEM_COLS = 256;      // two accumulators of up to 128 columns
constexpr uint32_t A_LBO = A_BOX;        // MN-major A: next 64-column block
constexpr uint32_t A_SBO = 1024;         // 8 K rows x 128 B
constexpr uint32_t B_LBO = 16;           // K-major B (unused with the 128-byte swizzle)
constexpr uint32_t B_SBO = 1024;         // 8 rows x 128 B
} // namespace gemmn

// fp32 accumulator, bf16 A and B, A MN-major, B K-major, M x N
__host__ __device__ constexpr uint32_t idesc_bf16_f32_swapped(int M, int N)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (0u << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Work item w -> cold expert slot j, column block cb, its m-tile, expert and padded row count.
struct NarrowItem {
    int cb, mt, e, rows, n_pad;
};
__device__ __forceinline__ NarrowItem narrow_item(int w, const GemmArgs &a)
{
    NarrowItem it;
    const int j = w / a.n_tiles;
    it.cb = w - j * a.n_tiles;
    it.mt = a.cold_tile[j];
    it.e = a.tile_expert[it.mt];
    it.rows = a.expert_rows[it.e];
    int np = (it.rows + 15) & ~15;
    it.n_pad = np < 16 ? 16 : (np > 128 ? 128 : np);
    return it;
}

// The whole CTA: work items w_first, w_first + w_step, ... (smem 1024-byte aligned).
// relinquish = false keeps the CTA's TMEM allocation permit for a second body afterwards.
template <int KIND, bool F8 = false>
__device__ __forceinline__ void grouped_gemm_narrow_cta(const CUtensorMap &tmW,
                                                        const CUtensorMap &tmX,
                                                        const GemmArgs &args, uint8_t *smem,
                                                        int w_first, int w_step,
                                                        bool relinquish = true)
{
    using namespace gemmn;
    float *xch = reinterpret_cast<float *>(smem + STAGES * STAGE); // [64][XCH_LD]
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + STAGES * STAGE + XCH_BYTES);
    const uint32_t bar0 = smem_u32(bars);
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
    auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + a); };
    auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + 2 + a); };
    const uint32_t done_bar = bar0 + 8u * (2 * STAGES + 4);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + NUM_BARS);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const bool gather = (args.gather_idx != nullptr); // layer0: B rows gathered from x

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full_bar(s), gather ? 1 + GATHER_THREADS : 1);
            mbar_init(empty_bar(s), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(tfull_bar(a), 1);
            mbar_init(tempty_bar(a), 4);
        }
        mbar_init(done_bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmW);
        if (!gather) tma_prefetch_desc(&tmX);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
        if (relinquish) tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const int total = args.meta->num_cold * args.n_tiles;
    const int KB = args.k_blocks;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer ----------------
            int s = 0;
            uint32_t ph = 0;
            int armed[STAGES];
#pragma unroll
            for (int i = 0; i < STAGES; ++i) armed[i] = -1;
            bool ok = true;
            for (int w = w_first; ok && w < total; w += w_step) {
                const NarrowItem it = narrow_item(w, args);
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait_bounded(empty_bar(s), ph ^ 1u, abort_flag, args.timeout_ns,
                                           args.status, 200 + KIND)) {
                        ok = false;
                        break;
                    }
                    const uint32_t a_dst = smem_u32(smem + s * STAGE);
                    const uint32_t b_dst = a_dst + A_TILE;
                    mbar_arrive_expect_tx(full_bar(s), A_TILE + (gather ? 0 : B_TILE));
                    armed[s] = (int)ph;
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        const int col = (KIND == GEMM_SWIGLU)
                                            ? (i == 0 ? it.cb * 64 : args.up_col + it.cb * 64)
                                            : it.cb * BM + i * 64;
                        if (F8) // K-major codes: x = the k-block's byte offset, y = weight row
                            tma_load_3d(a_dst + i * A_BOX, &tmW, full_bar(s), kb * 128, col, it.e);
                        else
                            tma_load_3d(a_dst + i * A_BOX, &tmW, full_bar(s), col, kb * BK, it.e);
                    }
                    if (!gather)
                        tma_load_2d(b_dst, &tmX, full_bar(s), kb * (F8 ? 128 : BK), it.mt * 128);
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            for (int i = 0; i < STAGES; ++i)
                if (armed[i] >= 0) {
                    volatile int never = 0;
                    mbar_wait_bounded(full_bar(i), (uint32_t)armed[i], &never, args.timeout_ns,
                                      nullptr, 0);
                }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- MMA issuer ----------------
            int s = 0;
            uint32_t ph = 0;
            int it_n = 0;
            bool ok = true;
            for (int w = w_first; ok && w < total; w += w_step, ++it_n) {
                const NarrowItem it = narrow_item(w, args);
                const uint32_t idesc =
                    F8 ? idesc_e4m3_f32(BM, it.n_pad) : idesc_bf16_f32_swapped(BM, it.n_pad);
                const int acc = it_n & 1;
                const uint32_t aph = (uint32_t)(it_n >> 1) & 1u;
                if (!mbar_wait_bounded(tempty_bar(acc), aph ^ 1u, abort_flag, args.timeout_ns,
                                       args.status, 210 + KIND)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * 128);
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait_bounded(full_bar(s), ph, abort_flag, args.timeout_ns,
                                           args.status, 220 + KIND)) {
                        ok = false;
                        break;
                    }
                    if (gather) fence_proxy_async_smem(); // B rows came through cp.async
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smem + s * STAGE);
                    const uint32_t b_addr = a_addr + A_TILE;
                    const uint64_t b_desc = sw128_desc(b_addr, B_LBO, B_SBO);
                    if (F8) {
                        // both K-major: +32 B (32 e4m3 values) per MMA
                        const uint64_t a_desc = sw128_desc(a_addr, B_LBO, B_SBO);
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            umma_f8(d_tmem, a_desc + (uint64_t)((k * 32) >> 4),
                                    b_desc + (uint64_t)((k * 32) >> 4), idesc,
                                    (kb | k) != 0 ? 1u : 0u);
                    } else {
                        const uint64_t a_desc = sw128_desc(a_addr, A_LBO, A_SBO);
#pragma unroll
                        for (int k = 0; k < BK / 16; ++k) {
                            // A (MN-major): +16 K rows x 128 B per K=16 step; B (K-major): +32 B
                            umma_bf16(d_tmem, a_desc + (uint64_t)((k * 16 * 128) >> 4),
                                      b_desc + (uint64_t)((k * 32) >> 4), idesc,
                                      (kb | k) != 0 ? 1u : 0u);
                        }
                    }
                    umma_commit(empty_bar(s));
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (!ok) break;
                umma_commit(tfull_bar(acc));
            }
            umma_commit(done_bar);
            volatile int never = 0;
            mbar_wait_bounded(done_bar, 0, &never, args.timeout_ns, args.status, 230 + KIND);
        }
    } else if (warp >= 6) {
        // ---------------- B-row gather: warps 6..9 (layer0 only) ----------------
        // Thread g copies 16-byte chunk (g & 7) of rows (g >> 3) + 16 i of every K step, for
        // the expert's n_pad rows only; destinations follow the 128-byte swizzle.
        if (gather) {
            const int g = threadIdx.x - NUM_THREADS;
            const int chunk = g & 7;
            const int r0 = g >> 3;
            int s = 0;
            uint32_t ph = 0;
            for (int w = w_first; w < total; w += w_step) {
                const NarrowItem it = narrow_item(w, args);
                const uint8_t *src[8]; // byte addresses: a k-block is 128 bytes of a row
                const size_t ld_bytes = (size_t)args.gather_ld * (F8 ? 1 : 2);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int64_t r = (int64_t)it.mt * 128 + r0 + 16 * i;
                    int t = (r < args.gather_len) ? args.gather_idx[r] : -1;
                    if (t < 0 || t >= args.gather_rows) t = 0; // pad rows read token 0
                    src[i] = reinterpret_cast<const uint8_t *>(args.gather_src) + (size_t)t * ld_bytes +
                             chunk * 16;
                }
                bool ok = true;
                for (int kb = 0; kb < KB; ++kb) {
                    ok = mbar_wait_bounded(empty_bar(s), ph ^ 1u, abort_flag, args.timeout_ns,
                                           args.status, 250 + KIND);
                    if (!__all_sync(0xffffffffu, ok)) {
                        ok = false;
                        break;
                    }
                    const uint32_t b_dst = smem_u32(smem + s * STAGE) + A_TILE;
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int r = r0 + 16 * i;
                        if (r < it.n_pad) {
                            const uint32_t dst = b_dst + r * 128 + ((chunk ^ (r & 7)) << 4);
                            cp_async_16_cg(dst, src[i] + (size_t)kb * 128);
                        }
                    }
                    cp_async_arrive_noinc(full_bar(s));
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (!ok) break;
            }
            cp_async_wait_all();
        }
    } else {
        // ---------------- epilogue: warps 2..5 ----------------
        // Warp (warp & 3) = q reads TMEM lanes 32q..32q+31, i.e. weight columns 32q + lane of
        // the item; TMEM column n is the expert's row n.
        const int q = warp & 3;
        int it_n = 0;
        for (int w = w_first; w < total; w += w_step, ++it_n) {
            const NarrowItem it = narrow_item(w, args);
            const int acc = it_n & 1;
            const uint32_t aph = (uint32_t)(it_n >> 1) & 1u;
            const bool got = mbar_wait_bounded(tfull_bar(acc), aph, abort_flag, args.timeout_ns,
                                               args.status, 240 + KIND);
            // every epilogue warp continues or all stop (they meet at named barriers below)
            if (!named_bar_and(1, 128, got)) break;
            tc_fence_after();
            const uint32_t t_row = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * 128);
            const int64_t row0 = (int64_t)it.mt * 128;
            // e4m3: this lane's weight-column scale (SwiGLU: q < 2 gate, q >= 2 up columns)
            float sb = 1.0f;
            if (F8) {
                const int wcol = (KIND == GEMM_SWIGLU)
                                     ? (q < 2 ? it.cb * 64 + q * 32 + lane
                                              : args.up_col + it.cb * 64 + (q - 2) * 32 + lane)
                                     : it.cb * BM + q * 32 + lane;
                sb = wcol < args.b_scale_ld ? args.b_scale[(size_t)it.e * args.b_scale_ld + wcol] : 0.0f;
            }
#pragma unroll 1
            for (int c0 = 0; c0 < it.n_pad; c0 += 32) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(t_row + c0, r);
                tmem_ld_wait();
                const int nc = (it.n_pad - c0) < 32 ? (it.n_pad - c0) : 32;
                if (F8) { // row scale (0 for pad rows), then this lane's column scale
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        if (i < nc) {
                            const int64_t row = row0 + c0 + i;
                            float sa;
                            const int32_t *si =
                                args.scale_idx != nullptr ? args.scale_idx : args.gather_idx;
                            if (si != nullptr) {
                                const int t = row < args.gather_len ? si[row] : -1;
                                sa = (t >= 0 && t < args.gather_rows) ? args.a_scale[t] : 0.0f;
                            } else {
                                sa = args.a_scale[row];
                            }
                            r[i] = __float_as_uint((__uint_as_float(r[i]) * sa) * sb);
                        }
                    }
                }
                if (KIND == GEMM_SWIGLU) {
                    if (q >= 2) { // up columns: hand them to the gate lanes
                        float *dst = xch + (size_t)((q - 2) * 32 + lane) * XCH_LD + c0;
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            if (i < nc) dst[i] = __uint_as_float(r[i]);
                    }
                    named_bar_sync(1, 128);
                    if (q < 2) {
                        const float *up = xch + (size_t)(q * 32 + lane) * XCH_LD + c0;
                        __nv_bfloat16 *o = args.out + (size_t)(row0 + c0) * args.ld_out +
                                           it.cb * 64 + q * 32 + lane;
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            if (i < nc) {
                                const float v = silu_f(__uint_as_float(r[i])) * up[i];
                                o[(size_t)i * args.ld_out] = __float2bfloat16_rn(v);
                            }
                        }
                    }
                    named_bar_sync(1, 128); // the hand-off buffer is refilled next chunk
                } else {
                    const int col = it.cb * BM + q * 32 + lane;
                    if (col < args.n_cols) {
                        __nv_bfloat16 *o = args.out + (size_t)(row0 + c0) * args.ld_out + col;
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            if (i < nc) {
                                float v = __uint_as_float(r[i]);
                                v = (KIND == GEMM_SCALE) ? v * args.row_w[row0 + c0 + i]
                                                         : act_f(args.act, v);
                                o[(size_t)i * args.ld_out] = __float2bfloat16_rn(v);
                            }
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tempty_bar(acc));
        }
    }

    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}


} // namespace moe

namespace moe {

// Phased order (wide.order == ORDER_HOT): every CTA first runs its share of the cold
// experts' items in the narrow body (their weights streamed by all SMs at once, the MMA N
// cut to the rows), then its share of the hot experts' 128-row items. Between the bodies the
// narrow body's mbarriers are invalidated and the generic writes to shared memory ordered
// before the wide body's TMA writes; the narrow body keeps the TMEM allocation permit.
template <int KIND, bool F8>
__device__ __forceinline__ void phased_bodies(const CUtensorMap &tmA, const CUtensorMap &tmB,
                                              const CUtensorMap &tmWn, const GemmArgs &wide,
                                              const GemmArgs &narrow, uint8_t *smem)
{
    if (wide.meta->num_cold > 0) {
        grouped_gemm_narrow_cta<KIND, F8>(tmWn, tmA, narrow, smem, blockIdx.x, gridDim.x, false);
        fence_proxy_async_smem();
        if (threadIdx.x == 0) {
            const uint32_t bar0 = smem_u32(smem + gemmn::STAGES * gemmn::STAGE + gemmn::XCH_BYTES);
            for (int i = 0; i < gemmn::NUM_BARS; ++i) mbar_inval(bar0 + 8u * i);
        }
        __syncthreads();
    }
    if (wide.meta->num_cold < wide.meta->num_tiles)
        grouped_gemm_cta<KIND, F8>(tmA, tmB, wide, smem, blockIdx.x, gridDim.x);
}

// One launch per layer that picks its kernel body on the device from the dispatch counts:
// when every routed expert owns a single m-tile (decode-sized batches), all CTAs run the
// narrow items; otherwise all CTAs run the 128-row items of every expert (args.order).
//
// Measured on the skewed layer (T = 4096, E = 256, Zipf 1.2; 107 of 135 active experts own a
// single m-tile), a split of the SMs between the two kinds is slower: a narrow CTA streams
// weights at ~43 GB/s (80 KB in flight against ~2 us of HBM latency), so the single-tile
// experts cost about as much SM time in either form, while the 128-row items of the other
// experts lose the SMs given to them. With every expert single-tile (decode), the narrow
// form is 5-7% faster: the same weight bytes, far less tensor-core work under the power cap.
template <int KIND>
__global__ void __launch_bounds__(gemm::NUM_THREADS_GATHER, 1)
    moe_grouped_gemm_select_kernel(const __grid_constant__ CUtensorMap tmA,
                                   const __grid_constant__ CUtensorMap tmB, const GemmArgs wide,
                                   const GemmArgs narrow)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int num_cold = wide.meta->num_cold;
    if (wide.order == ORDER_HOT)
        phased_bodies<KIND, false>(tmA, tmB, tmB, wide, narrow, smem);
    else if (num_cold > 0 && num_cold == wide.meta->num_tiles)
        grouped_gemm_narrow_cta<KIND>(tmB, tmA, narrow, smem, blockIdx.x, gridDim.x);
    else
        grouped_gemm_cta<KIND>(tmA, tmB, wide, smem, blockIdx.x, gridDim.x);
}

// The e4m3 form of moe_grouped_gemm_select_kernel: the narrow body reads the weight codes
// through tmWn (64-row boxes), the 128-row body through tmB (128-row boxes).
template <int KIND>
__global__ void __launch_bounds__(gemm::NUM_THREADS_GATHER, 1)
    moe_grouped_gemm_select_f8_kernel(const __grid_constant__ CUtensorMap tmA,
                                      const __grid_constant__ CUtensorMap tmB,
                                      const __grid_constant__ CUtensorMap tmWn,
                                      const GemmArgs wide, const GemmArgs narrow)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int num_cold = wide.meta->num_cold;
    if (wide.order == ORDER_HOT)
        phased_bodies<KIND, true>(tmA, tmB, tmWn, wide, narrow, smem);
    else if (num_cold > 0 && num_cold == wide.meta->num_tiles)
        grouped_gemm_narrow_cta<KIND, true>(tmWn, tmA, narrow, smem, blockIdx.x, gridDim.x);
    else
        grouped_gemm_cta<KIND, true>(tmA, tmB, wide, smem, blockIdx.x, gridDim.x);
}

} // namespace moe
