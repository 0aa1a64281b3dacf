// gemm_tc.cuh -- persistent grouped GEMM over all experts on the 5th-generation tensor cores
// (tcgen05 + TMEM), fed by TMA, with the expert epilogues fused.
//
// Where it comes from (Comet: Fine-grained Computation-communication Overlapping for
// Mixture-of-Experts):
//   §3.1.1  layer0 (hidden -> FFN) is decomposed along M: its work items are 128-row tiles
//           of expert-sorted token rows; layer1 (FFN -> hidden) is decomposed along N:
//           each work item owns a 256-column stripe of the output, so the top-k reduce of
//           a stripe never depends on another stripe.
//   §3.1.2  rows are regrouped into whole GEMM tiles (128-row padded expert blocks) and the
//           GroupGEMM covers every expert in one launch.
//   §3.2.1  thread-block specialisation: inside each CTA one warp only moves data (TMA),
//           one warp only issues MMAs, four warps only run the epilogue.
//   §4      the GEMMs are expert-grouped GEMMs; row metadata is read once per tile, not
//           per K step.
//
// Design on sm_100a
//   - One CTA per SM (persistent), 192 threads:
//       warp 0  TMA producer: A tile 128 x 64 (one 2D box) and B tile 64 x 256 (four
//               3D boxes of 64 x 64 from the expert's weight matrix) per K step;
//       warp 1  allocates 512 TMEM columns (two 128 x 256 fp32 accumulators) and issues
//               tcgen05.mma (M=128, N=256, K=16) from one thread;
//       warps 2-5 epilogue: tcgen05.ld of their 32 TMEM lanes, activation or gate scale,
//               bf16 stores. The two accumulators let the epilogue of tile i overlap the
//               mainloop of tile i+1.
//   - 4-stage shared-memory ring (48 KB per stage), 128-byte swizzle; A is K-major, B is
//     the weight matrix as stored (N contiguous), read MN-major by the MMA.
//   - Work items are ordered expert-major, then N tile, then M tile, so the CTAs that run
//     together share one expert's weight stripe and its token rows in L2.
//   - Every wait is bounded: on timeout the CTA records DEV_TIMEOUT, all roles stop, the
//     producer waits (bounded) for its in-flight copies, the MMA warp waits for its
//     in-flight MMAs, and TMEM is released before exit.
//
// Kinds:
//   GEMM_SWIGLU  A = x_perm [rows, H], B = W1[e] [H, 2F]; the B tile holds gate columns
//                n*128.. and up columns F + n*128..; out h[r][n*128 + c] =
//                silu(gate) * up (bf16).
//   GEMM_ACT     A = x_perm, B = W1[e] [H, F]; out h = act(acc) (bf16), 256 columns/tile.
//   GEMM_SCALE   A = h [rows, F], B = W2[e] [F, H]; out ys[r][n*256 + c] =
//                row_w[r] * acc (bf16).
#pragma once

#include "dispatch.cuh"
#include "ptx.cuh"

namespace moe {

// ranks of the expert-parallel layer at most (pointer tables travel in kernel parameters)
constexpr int EP_MAX_WORLD = 8;

namespace gemm {
constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;
constexpr int STAGES = 4;
constexpr int A_TILE = BM * BK * 2;    // 16 KB
constexpr int B_BOX = 64 * BK * 2;     // 8 KB: 64 columns x 64 K rows
constexpr int B_TILE = BN * BK * 2;    // 32 KB
constexpr int STAGE = A_TILE + B_TILE; // 48 KB
constexpr int NUM_THREADS = 192;      // TMA warp, MMA warp, 4 epilogue warps
constexpr int GATHER_THREADS = 128;   // 4 more warps that gather layer0 A rows (cp.async)
constexpr int NUM_THREADS_GATHER = NUM_THREADS + GATHER_THREADS;
constexpr int NUM_BARS = 2 * STAGES + 5;
constexpr int SCALE_STAGE = 2 * BN * 4; // e4m3: the items' column scales, one buffer per accumulator
// the scale buffers start on a 128-byte boundary after the barriers, the TMEM slot and the
// abort flag (16-byte reads)
constexpr int SCALE_OFF = STAGES * STAGE + ((NUM_BARS * 8 + 16 + 127) & ~127);
constexpr int SMEM_BYTES = 1024 /*alignment slack*/ + SCALE_OFF + SCALE_STAGE;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t IDESC = idesc_bf16_f32(BM, BN, /*b_mn_major=*/true);
// e4m3 operands: both K-major; a K step of 128 values is the same 128-byte row as 64 bf16
// values, so the stage layout, the swizzle and the four MMAs per stage are unchanged
constexpr uint32_t IDESC_F8 = idesc_e4m3_f32(BM, BN);
constexpr int B8_BOX_ROWS = 128; // e4m3 B tile: two boxes of 128 weight rows x 128 K bytes
// descriptor strides
constexpr uint32_t A_SBO = 1024; // 8 rows x 128 B
constexpr uint32_t A_LBO = 16;   // unused for swizzled K-major
constexpr uint32_t B_SBO = 1024; // 8 K rows x 128 B
constexpr uint32_t B_LBO = B_BOX; // next 64-column block
} // namespace gemm

enum GemmKind { GEMM_SWIGLU = 0, GEMM_ACT = 1, GEMM_SCALE = 2, GEMM_LOGITS = 3 };
// Operand layouts of grouped_gemm_cta:
//   BMODE_FWD     B = the expert's weight matrix as stored [K, N] (MN-major; e4m3 codes are
//                 stored K-major instead, see F8);
//   BMODE_KMAJOR  B = the expert's matrix [N rows, K] read K-major (backward: dy . W2^T and
//                 dz . W1^T, where the forward's weight is the transposed operand);
//   BMODE_WGRAD   weight gradients: D[e] = A_e^T B_e over the expert's padded rows r (K),
//                 A [rows, M] and B [rows, N] both read MN-major.
enum GemmBMode { BMODE_FWD = 0, BMODE_KMAJOR = 1, BMODE_WGRAD = 2 };
enum GemmOrder { ORDER_EXPERT = 0, ORDER_MIXED = 1, ORDER_HOT = 2 };

struct GemmArgs {
    const int32_t *tile_off;    // [E+1] first m-tile of each expert
    const int32_t *tile_expert; // [max_tiles] expert of each m-tile
    const int32_t *ptile_off;   // [E+1] first m-tile pair of each expert (pair kernel)
    const int32_t *ptile_expert; // expert of each m-tile pair (pair kernel)
    const DispatchMeta *meta;   // num_tiles, num_cold
    // Work order over the experts' m-tiles ("cold" experts have one m-tile, so their weight
    // tiles are streamed for a single tile; the others are "hot"):
    //   ORDER_EXPERT  expert-major over all m-tiles;
    //   ORDER_MIXED   the cold experts' items spread evenly among the hot ones;
    //   ORDER_HOT     the hot experts' m-tiles only, expert-major (the cold experts' items
    //                 run in the narrow body first: moe_grouped_gemm_select_kernel).
    // hot_off [E+1] prefixes the hot experts' m-tiles, hot_tile_expert lists the expert of
    // each hot m-tile, cold_tile the m-tile of each cold expert (written by the dispatch scan).
    int order;
    const int32_t *expert_rows; // [E] routed rows of each expert (narrow kernel)
    const int32_t *hot_off;
    const int32_t *hot_tile_expert;
    const int32_t *cold_tile;
    const float *row_w;         // GEMM_SCALE: gate weight of each padded row
    const int32_t *gather_idx;  // layer0: token of each padded row (-1: pad), A rows are
                                // gathered from x with it; nullptr: A rows are contiguous
    int64_t gather_len;         // entries of gather_idx
    const __nv_bfloat16 *gather_src; // x [gather_rows, gather_ld]
    int gather_rows;
    int gather_ld;
    __nv_bfloat16 *out;         // [rows, ld_out]
    int ld_out;                 // elements per output row
    int n_cols;                 // valid output columns
    int n_tiles;                // N tiles per m-tile
    int k_blocks;               // K / 64
    int up_col;                 // GEMM_SWIGLU: first up column of W1 (= F)
    int act;                    // GEMM_ACT: 1 gelu-tanh, 2 relu, 3 identity
    int *status;
    int64_t timeout_ns;
    // GEMM_LOGITS (router filter): one dense operand A [dense_rows, K] in dense_m_tiles
    // 128-row tiles, N = 64 * n_boxes columns per tile (n_boxes <= 4); K is split into
    // k_split contiguous ranges of k-blocks and split s writes its fp32 partial product
    // column-major: out_f32[(s * n_cols + col) * dense_rows + row]
    int dense_m_tiles;
    int dense_rows;
    int k_split;
    int n_boxes;
    float *out_f32;
    float *xsq_f32; // optional: sum of squares of every A row over each split's K range,
                    // [k_split, dense_rows] (the epilogue warps read the staged A tiles)
    // e4m3 operands (moe_grouped_gemm_select_f8_kernel): the accumulator of row r, column c of
    // expert e is multiplied by a_scale[token of r] (gathered rows) or a_scale[r], then by
    // b_scale[e * b_scale_ld + c]
    const float *a_scale;
    const float *b_scale;
    int b_scale_ld;
    const int32_t *scale_idx; // a_scale index of each padded row when the rows arrive
                              // already gathered (CTA-pair layer0); else gather_idx, or none
    // BMODE_WGRAD: wg_experts experts, each an output of wg_mtiles 128-row tiles (M =
    // 128 * wg_mtiles) by n_tiles 256-column tiles; expert e's K is its padded rows
    // [128 tile_off[e], 128 tile_off[e + 1]); out[(e * M + m) * ld_out + n]
    int wg_experts;
    int wg_mtiles;
    const int32_t *active_list; // BMODE_WGRAD: only these experts (meta->num_active of them)
    int epi8; // A by TMA (no gather): warps 6..9 join the epilogue, each pair of warps on one
              // TMEM lane quarter splits the item's column chunks (launch with 320 threads)
    // Expert parallelism (GEMM_SCALE rows returned to their origin): row r's output goes to
    // row (row_dst[r] & 0xffffffff) of peer_out[row_dst[r] >> 32] (another GPU's buffer:
    // plain 16-byte stores), and is not stored at all where row_dst[r] < 0 (pad rows);
    // row_dst == nullptr: rows go to `out`.
    const long long *row_dst;
    __nv_bfloat16 *peer_out[EP_MAX_WORLD];
};

__device__ __forceinline__ void gemm_map_work(int w, const GemmArgs &a, int &e, int &mt, int &nt,
                                              int &ks)
{
    ks = 0;
    if (a.dense_m_tiles > 0) { // one operand, no expert groups; m fastest, then n, then split
        e = 0;
        mt = w % a.dense_m_tiles;
        const int r = w / a.dense_m_tiles;
        nt = r % a.n_tiles;
        ks = r / a.n_tiles;
        return;
    }
    if (a.order == ORDER_MIXED || a.order == ORDER_HOT) {
        int64_t cb = 0;
        if (a.order == ORDER_MIXED) {
            const int64_t total = (int64_t)a.meta->num_tiles * a.n_tiles;
            const int64_t cold = (int64_t)a.meta->num_cold * a.n_tiles;
            cb = (int64_t)w * cold / total;                   // cold items before slot w
            const int64_t cb1 = ((int64_t)w + 1) * cold / total;
            if (cb1 > cb) { // slot w holds cold item cb: the expert's single m-tile, n-tile cb % n
                const int j = (int)(cb / a.n_tiles);
                nt = (int)(cb - (int64_t)j * a.n_tiles);
                mt = a.cold_tile[j];
                e = a.tile_expert[mt];
                return;
            }
        }
        const int h = (int)(w - cb); // hot item h, in the hot experts' expert-major order
        e = a.hot_tile_expert[h / a.n_tiles];
        const int hb = a.hot_off[e];
        const int base = a.tile_off[e];
        const int cnt = a.tile_off[e + 1] - base;
        const int local = h - hb * a.n_tiles;
        mt = base + local % cnt;
        nt = local / cnt;
        return;
    }
    const int q = w / a.n_tiles;
    e = a.tile_expert[q];
    const int base = a.tile_off[e];
    const int cnt = a.tile_off[e + 1] - base;
    const int local = w - base * a.n_tiles;
    mt = base + local % cnt;
    nt = local / cnt;
}

__device__ __forceinline__ void gemm_map_work(int w, const GemmArgs &a, int &e, int &mt, int &nt)
{
    int ks;
    gemm_map_work(w, a, e, mt, nt, ks);
}

// silu(z) = z * sigmoid(z), with the fast exponential and an IEEE reciprocal (1 + e^-z = inf
// gives 0; NaN propagates)
__device__ __forceinline__ float silu_f(float z) { return z * __frcp_rn(1.0f + __expf(-z)); }

__device__ __forceinline__ float act_f(int act, float z)
{
    if (act == 1) {
        const float c = 0.7978845608028654f; // sqrt(2/pi)
        return 0.5f * z * (1.0f + tanhf(c * (z + 0.044715f * z * z * z)));
    }
    if (act == 2) return z > 0.0f ? z : 0.0f;
    return z;
}

// Epilogue of one accumulator tile for the 32 rows of this warp: thread `lane` owns row `row`
// and reads its TMEM lane `t_row` (already offset to the accumulator buffer). Warp-collective
// (tcgen05.ld), so the whole warp calls it.
// sbs: the item's column scales staged in shared memory (e4m3; SwiGLU: 128 gate then 128 up
// columns, else the tile's 256 columns), or nullptr to read them from global memory
// Column chunks [c_lo, c_hi) of the item (32 columns each: SwiGLU 4 gate/up pairs, else 8);
// c_hi < 0: all of them.
template <int KIND, bool F8 = false>
__device__ __forceinline__ void epilogue_rows(const GemmArgs &args, uint32_t t_row, int row, int nt,
                                              int ks = 0, int e = 0, const float *sbs = nullptr,
                                              int c_lo = 0, int c_hi = -1)
{
    using namespace gemm;
    // e4m3 operands: the row's scale (0 for pad rows, whose outputs are never read)
    float sa = 1.0f;
    if (F8) {
        const int32_t *si = args.scale_idx != nullptr ? args.scale_idx : args.gather_idx;
        if (si != nullptr) {
            const int t = row < args.gather_len ? si[row] : -1;
            sa = (t >= 0 && t < args.gather_rows) ? args.a_scale[t] : 0.0f;
        } else {
            sa = args.a_scale[row];
        }
    }
    const float *sb = F8 ? args.b_scale + (size_t)e * args.b_scale_ld : nullptr;
    if (KIND == GEMM_SWIGLU) {
        __nv_bfloat16 *orow = args.out + (size_t)row * args.ld_out + nt * 128;
#pragma unroll 1
        for (int c = c_lo; c < (c_hi < 0 ? 4 : c_hi); ++c) {
            uint32_t g[32], u[32];
            tmem_ld_32x32b_x32(t_row + c * 32, g);
            tmem_ld_32x32b_x32(t_row + 128 + c * 32, u);
            tmem_ld_wait();
            if (nt * 128 + c * 32 < args.n_cols) {
                uint4 *dst = reinterpret_cast<uint4 *>(orow + c * 32);
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    float sg[8], su[8]; // column scales of the 8 gate and 8 up columns
                    if (F8) {
                        const int c0 = nt * 128 + c * 32 + v * 8;
                        const float4 *pg = reinterpret_cast<const float4 *>(
                            sbs ? sbs + c * 32 + v * 8 : sb + c0);
                        const float4 *pu = reinterpret_cast<const float4 *>(
                            sbs ? sbs + 128 + c * 32 + v * 8 : sb + args.up_col + c0);
                        const float4 g0 = pg[0], g1 = pg[1], u0 = pu[0], u1 = pu[1];
                        sg[0] = g0.x; sg[1] = g0.y; sg[2] = g0.z; sg[3] = g0.w;
                        sg[4] = g1.x; sg[5] = g1.y; sg[6] = g1.z; sg[7] = g1.w;
                        su[0] = u0.x; su[1] = u0.y; su[2] = u0.z; su[3] = u0.w;
                        su[4] = u1.x; su[5] = u1.y; su[6] = u1.z; su[7] = u1.w;
                    }
                    uint32_t p[4];
#pragma unroll
                    for (int h2 = 0; h2 < 4; ++h2) {
                        const int i = v * 8 + h2 * 2;
                        float g0 = __uint_as_float(g[i]), g1 = __uint_as_float(g[i + 1]);
                        float u0 = __uint_as_float(u[i]), u1 = __uint_as_float(u[i + 1]);
                        if (F8) {
                            g0 = (g0 * sa) * sg[h2 * 2];
                            g1 = (g1 * sa) * sg[h2 * 2 + 1];
                            u0 = (u0 * sa) * su[h2 * 2];
                            u1 = (u1 * sa) * su[h2 * 2 + 1];
                        }
                        const float a0 = silu_f(g0) * u0;
                        const float a1 = silu_f(g1) * u1;
                        p[h2] = pack_bf16x2(a0, a1);
                    }
                    dst[v] = make_uint4(p[0], p[1], p[2], p[3]);
                }
            }
        }
    } else if (KIND == GEMM_LOGITS) {
        // column-major partials: the 32 lanes (consecutive rows) store 128 contiguous bytes
        const int nc = args.n_boxes * 2;
        float *out = args.out_f32 + (size_t)ks * args.n_cols * args.dense_rows + row;
#pragma unroll 1
        for (int c = 0; c < nc; ++c) {
            uint32_t r[32];
            tmem_ld_32x32b_x32(t_row + c * 32, r);
            tmem_ld_wait();
            if (row < args.dense_rows) {
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int col = nt * BN + c * 32 + i;
                    if (col < args.n_cols) out[(size_t)col * args.dense_rows] = __uint_as_float(r[i]);
                }
            }
        }
    } else {
        __nv_bfloat16 *orow = args.out + (size_t)row * args.ld_out + nt * BN;
        bool keep = true;
        if (KIND == GEMM_SCALE && args.row_dst != nullptr) {
            const long long o = args.row_dst[row];
            keep = o >= 0;
            if (keep)
                orow = args.peer_out[(int)(o >> 32)] + (size_t)(o & 0xffffffffll) * args.ld_out + nt * BN;
        }
        const float wt = (KIND == GEMM_SCALE) ? args.row_w[row] : 1.0f;
#pragma unroll 1
        for (int c = c_lo; c < (c_hi < 0 ? BN / 32 : c_hi); ++c) {
            uint32_t r[32];
            tmem_ld_32x32b_x32(t_row + c * 32, r);
            tmem_ld_wait();
            if (keep && nt * BN + c * 32 < args.n_cols) {
                uint4 *dst = reinterpret_cast<uint4 *>(orow + c * 32);
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    float sc[8]; // column scales of these 8 columns
                    if (F8) {
                        const float4 *pc = reinterpret_cast<const float4 *>(
                            sbs ? sbs + c * 32 + v * 8 : sb + nt * BN + c * 32 + v * 8);
                        const float4 c0 = pc[0], c1 = pc[1];
                        sc[0] = c0.x; sc[1] = c0.y; sc[2] = c0.z; sc[3] = c0.w;
                        sc[4] = c1.x; sc[5] = c1.y; sc[6] = c1.z; sc[7] = c1.w;
                    }
                    uint32_t p[4];
#pragma unroll
                    for (int h2 = 0; h2 < 4; ++h2) {
                        const int i = v * 8 + h2 * 2;
                        float a0 = __uint_as_float(r[i]);
                        float a1 = __uint_as_float(r[i + 1]);
                        if (F8) {
                            a0 = (a0 * sa) * sc[h2 * 2];
                            a1 = (a1 * sa) * sc[h2 * 2 + 1];
                        }
                        if (KIND == GEMM_SCALE) {
                            a0 *= wt;
                            a1 *= wt;
                        } else {
                            a0 = act_f(args.act, a0);
                            a1 = act_f(args.act, a1);
                        }
                        p[h2] = pack_bf16x2(a0, a1);
                    }
                    dst[v] = make_uint4(p[0], p[1], p[2], p[3]);
                }
            }
        }
    }
}

// The whole CTA: work items w_first, w_first + w_step, ... (smem 1024-byte aligned).
// BMODE_WGRAD work item w: expert-major, then N tile, then M tile; its k-blocks of 64 rows
__device__ __forceinline__ void wgrad_item(int w, const GemmArgs &a, int &e, int &mt, int &nt,
                                           int &kb0, int &kb1)
{
    const int per = a.wg_mtiles * a.n_tiles;
    const int j = w / per;
    e = a.active_list != nullptr ? a.active_list[j] : j;
    const int r = w - j * per;
    mt = r % a.wg_mtiles;
    nt = r / a.wg_mtiles;
    kb0 = a.tile_off[e] * (gemm::BM / gemm::BK);
    kb1 = a.tile_off[e + 1] * (gemm::BM / gemm::BK);
}

template <int KIND, bool F8 = false, int BMODE = BMODE_FWD>
__device__ __forceinline__ void grouped_gemm_cta(const CUtensorMap &tmA, const CUtensorMap &tmB,
                                                 const GemmArgs &args, uint8_t *smem, int w_first,
                                                 int w_step)
{
    using namespace gemm;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + STAGES * STAGE);
    const uint32_t bar0 = smem_u32(bars);
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
    auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + a); };
    auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + 2 + a); };
    const uint32_t done_bar = bar0 + 8u * (2 * STAGES + 4);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + NUM_BARS);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    float *scale_stage = reinterpret_cast<float *>(smem + SCALE_OFF);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // layer0 A rows come from the gather warps (cp.async, one arrival per gather thread);
    // otherwise A is one TMA box like B
    const bool gather = (args.gather_idx != nullptr);
    // router filter: the four epilogue warps also read every staged A tile (row norms)
    const bool row_sq = (KIND == GEMM_LOGITS) && args.xsq_f32 != nullptr;
    // eight epilogue warps (A by TMA, 320 threads); not with the row norms or weight gradients
    const bool epi8 = args.epi8 && !gather && !row_sq && BMODE != BMODE_WGRAD &&
                      blockDim.x >= NUM_THREADS_GATHER;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full_bar(s), gather ? 1 + GATHER_THREADS : 1);
            mbar_init(empty_bar(s), row_sq ? 5 : 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(tfull_bar(a), 1);
            mbar_init(tempty_bar(a), epi8 ? 8 : 4);
        }
        mbar_init(done_bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const bool wgrad = (BMODE == BMODE_WGRAD);
    const int num_tiles = wgrad ? 0
                          : args.dense_m_tiles > 0 ? args.dense_m_tiles
                          : args.order == ORDER_HOT ? args.meta->num_tiles - args.meta->num_cold
                                                    : args.meta->num_tiles;
    const int n_split = (args.dense_m_tiles > 0 && args.k_split > 1) ? args.k_split : 1;
    const int total = wgrad ? (args.active_list != nullptr ? args.meta->num_active : args.wg_experts) *
                                  args.wg_mtiles * args.n_tiles
                            : num_tiles * args.n_tiles * n_split;
    const int KB = args.k_blocks;
    // k-blocks [kb_lo(ks), kb_lo(ks + 1)) belong to split ks (n_split <= KB: none is empty)
    auto kb_lo = [&](int ks) { return (int)(((int64_t)ks * KB) / n_split); };
    // k-block range of work item w (per expert for BMODE_WGRAD, possibly empty)
    auto kb_range = [&](int w, int &e, int &mt, int &nt, int &kb0, int &kb1) {
        if (wgrad) {
            wgrad_item(w, args, e, mt, nt, kb0, kb1);
        } else {
            int ks;
            gemm_map_work(w, args, e, mt, nt, ks);
            kb0 = kb_lo(ks);
            kb1 = kb_lo(ks + 1);
        }
    };
    // B boxes of 64 columns per k-block; the router filter narrows N to what E needs
    const int nbox = (KIND == GEMM_LOGITS && args.n_boxes >= 1 && args.n_boxes < 4) ? args.n_boxes : 4;
    const uint32_t idesc = BMODE == BMODE_KMAJOR ? idesc_bf16_f32(BM, BN, /*b_mn_major=*/false)
                           : BMODE == BMODE_WGRAD ? (IDESC | (1u << 15)) // A MN-major too
                           : (nbox == 4) ? IDESC
                                         : idesc_bf16_f32(BM, nbox * 64, /*b_mn_major=*/true);

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
                int e, mt, nt, kb0, kb1;
                kb_range(w, e, mt, nt, kb0, kb1);
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!mbar_wait_bounded(empty_bar(s), ph ^ 1u, abort_flag, args.timeout_ns,
                                           args.status, 100 + KIND)) {
                        ok = false;
                        break;
                    }
                    const uint32_t a_dst = smem_u32(smem + s * STAGE);
                    const uint32_t b_dst = a_dst + A_TILE;
                    mbar_arrive_expect_tx(full_bar(s), (gather ? 0 : A_TILE) +
                                                           ((F8 || BMODE != BMODE_FWD) ? B_TILE : nbox * B_BOX));
                    armed[s] = (int)ph;
                    if (BMODE == BMODE_WGRAD) {
                        // A [rows, M] MN-major: two boxes of 64 M columns x 64 rows; B [rows, N]
                        // (a depth-1 3D map) MN-major: four boxes of 64 N columns x 64 rows
                        tma_load_2d(a_dst, &tmA, full_bar(s), mt * BM, kb * BK);
                        tma_load_2d(a_dst + B_BOX, &tmA, full_bar(s), mt * BM + 64, kb * BK);
                        for (int i = 0; i < 4; ++i)
                            tma_load_3d(b_dst + i * B_BOX, &tmB, full_bar(s), nt * BN + i * 64, kb * BK, 0);
                    } else {
                    // the x coordinate is the K offset in elements: 128 B per k-block either way
                    if (!gather) tma_load_2d(a_dst, &tmA, full_bar(s), kb * (F8 ? 128 : BK), mt * BM);
                    if (BMODE == BMODE_KMAJOR) { // bf16 [E, N rows, K]: two boxes of 128 rows
                        tma_load_3d(b_dst, &tmB, full_bar(s), kb * BK, nt * BN, e);
                        tma_load_3d(b_dst + 128 * 128, &tmB, full_bar(s), kb * BK, nt * BN + 128, e);
                    }
                    if (F8) { // K-major e4m3 weights [E, N rows, K]: two boxes of 128 rows
                        const int r0 = (KIND == GEMM_SWIGLU) ? nt * 128 : nt * BN;
                        const int r1 = (KIND == GEMM_SWIGLU) ? args.up_col + nt * 128 : nt * BN + B8_BOX_ROWS;
                        tma_load_3d(b_dst, &tmB, full_bar(s), kb * 128, r0, e);
                        tma_load_3d(b_dst + B8_BOX_ROWS * 128, &tmB, full_bar(s), kb * 128, r1, e);
                    }
                    for (int i = 0; i < ((F8 || BMODE != BMODE_FWD) ? 0 : nbox); ++i) {
                        int col;
                        if (KIND == GEMM_SWIGLU)
                            col = (i < 2 ? nt * 128 + i * 64 : args.up_col + nt * 128 + (i - 2) * 64);
                        else
                            col = nt * BN + i * 64;
                        tma_load_3d(b_dst + i * B_BOX, &tmB, full_bar(s), col, kb * BK, e);
                    }
                    }
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            // every TMA copy issued must have landed before the CTA exits (immediate when
            // the MMA warp consumed them all; bounded after an abort)
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
            int it = 0;
            bool ok = true;
            for (int w = w_first; ok && w < total; w += w_step, ++it) {
                const int acc = it & 1;
                const uint32_t aph = (uint32_t)(it >> 1) & 1u;
                if (!mbar_wait_bounded(tempty_bar(acc), aph ^ 1u, abort_flag, args.timeout_ns,
                                       args.status, 110 + KIND)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
                int kb_first = 0, kb_end = KB;
                if (n_split > 1 || wgrad) {
                    int e_, mt_, nt_;
                    kb_range(w, e_, mt_, nt_, kb_first, kb_end);
                }
                for (int kb = kb_first; kb < kb_end; ++kb) {
                    if (!mbar_wait_bounded(full_bar(s), ph, abort_flag, args.timeout_ns, args.status,
                                           120 + KIND)) {
                        ok = false;
                        break;
                    }
                    // the gathered A rows were written through the generic proxy (cp.async);
                    // order them before the tensor cores read the stage
                    if (gather) fence_proxy_async_smem();
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smem + s * STAGE);
                    const uint32_t b_addr = a_addr + A_TILE;
                    const uint64_t a_desc = sw128_desc(a_addr, A_LBO, A_SBO);
                    if (F8) {
                        // both K-major: +32 B (32 e4m3 values) per MMA inside the swizzle atom
                        const uint64_t b_desc = sw128_desc(b_addr, A_LBO, A_SBO);
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            umma_f8(d_tmem, a_desc + (uint64_t)((k * 32) >> 4),
                                    b_desc + (uint64_t)((k * 32) >> 4), IDESC_F8,
                                    (kb != kb_first || k != 0) ? 1u : 0u);
                    } else if (BMODE == BMODE_KMAJOR) {
                        // both K-major: +32 B per K=16 step
                        const uint64_t b_desc = sw128_desc(b_addr, A_LBO, A_SBO);
#pragma unroll
                        for (int k = 0; k < BK / 16; ++k)
                            umma_bf16(d_tmem, a_desc + (uint64_t)((k * 32) >> 4),
                                      b_desc + (uint64_t)((k * 32) >> 4), idesc,
                                      (kb != kb_first || k != 0) ? 1u : 0u);
                    } else {
                        // MN-major A (BMODE_WGRAD: next 64-column block one box further) and
                        // B: +16 K rows x 128 B per K=16 step
                        const uint64_t a_mn = sw128_desc(a_addr, B_LBO, B_SBO);
                        const uint64_t b_desc = sw128_desc(b_addr, B_LBO, B_SBO);
#pragma unroll
                        for (int k = 0; k < BK / 16; ++k) {
                            // A: +32 B per K=16 step inside the swizzle atom; B: +16 rows x 128 B
                            umma_bf16(d_tmem,
                                      wgrad ? a_mn + (uint64_t)((k * 16 * 128) >> 4)
                                            : a_desc + (uint64_t)((k * 32) >> 4),
                                      b_desc + (uint64_t)((k * 16 * 128) >> 4), idesc,
                                      (kb != kb_first || k != 0) ? 1u : 0u);
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
            // every MMA issued so far must finish before TMEM is released
            umma_commit(done_bar);
            volatile int never = 0;
            mbar_wait_bounded(done_bar, 0, &never, args.timeout_ns, args.status, 130 + KIND);
        }
    } else if (warp >= 6 && !epi8) {
        // ---------------- A-row gather: warps 6..9 (layer0 only) ----------------
        // Thread g copies 16-byte chunk (g & 7) of rows (g >> 3) + 16 i, i = 0..7, of every K
        // step. The 8 token ids of its rows are read once per tile and kept in registers
        // (Comet §4: row indices cached in registers instead of re-read every K step).
        // Destinations follow the 128-byte swizzle the MMA descriptor expects.
        if (gather) {
            const int g = threadIdx.x - NUM_THREADS;
            const int chunk = g & 7;
            const int r0 = g >> 3;
            int s = 0;
            uint32_t ph = 0;
            for (int w = w_first; w < total; w += w_step) {
                int e, mt, nt;
                gemm_map_work(w, args, e, mt, nt);
                // row addresses in bytes: a k-block is the next 128 bytes of every row (64
                // bf16 or 128 e4m3 values)
                const uint8_t *src[8];
                const size_t ld_bytes = (size_t)args.gather_ld * (F8 ? 1 : 2);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int64_t r = (int64_t)mt * BM + r0 + 16 * i;
                    int t = (r < args.gather_len) ? args.gather_idx[r] : -1;
                    if (t < 0 || t >= args.gather_rows) t = 0; // pad rows read token 0; never used
                    src[i] = reinterpret_cast<const uint8_t *>(args.gather_src) + (size_t)t * ld_bytes +
                             chunk * 16;
                }
                bool ok = true;
                for (int kb = 0; kb < KB; ++kb) { // layer0 only: never split
                    ok = mbar_wait_bounded(empty_bar(s), ph ^ 1u, abort_flag, args.timeout_ns,
                                           args.status, 150 + KIND);
                    if (!__all_sync(0xffffffffu, ok)) {
                        ok = false;
                        break;
                    }
                    const uint32_t a_dst = smem_u32(smem + s * STAGE);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int r = r0 + 16 * i;
                        const uint32_t dst = a_dst + r * 128 + ((chunk ^ (r & 7)) << 4);
                        cp_async_16_cg(dst, src[i] + (size_t)kb * 128);
                    }
                    cp_async_arrive_noinc(full_bar(s));
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (!ok) break;
            }
            cp_async_wait_all(); // this thread's copies land before the CTA exits
        }
    } else {
        // ---------------- epilogue: warps 2..5 (and 6..9 with epi8) ----------------
        const int q = warp & 3; // TMEM lanes 32q .. 32q+31
        // with epi8, warps 2..5 take the first half of the item's column chunks and warps
        // 6..9 the second; nep threads meet at the named barriers below
        const int half = warp >= 6 ? 1 : 0;
        const int nep = epi8 ? 256 : 128;
        const int nchunks = (KIND == GEMM_SWIGLU) ? 4 : BN / 32;
        const int c_lo = epi8 ? half * (nchunks / 2) : 0;
        const int c_hi = epi8 ? c_lo + nchunks / 2 : -1;
        int it = 0;
        int rs = 0;             // stage ring position (row_sq only)
        uint32_t rph = 0;
        for (int w = w_first; w < total; w += w_step, ++it) {
            int e, mt, nt, ks = 0, kb0 = 0, kb1 = 1;
            if (wgrad)
                wgrad_item(w, args, e, mt, nt, kb0, kb1);
            else
                gemm_map_work(w, args, e, mt, nt, ks);
            if (row_sq) {
                // sum of squares of this thread's A row over the item's k-blocks (the order of
                // the 16-byte pieces does not matter; lane-rotated reads avoid bank conflicts)
                float ss = 0.0f;
                bool ok = true;
                for (int kb = kb_lo(ks); kb < kb_lo(ks + 1); ++kb) {
                    ok = mbar_wait_bounded(full_bar(rs), rph, abort_flag, args.timeout_ns,
                                           args.status, 160 + KIND);
                    if (!__all_sync(0xffffffffu, ok)) {
                        ok = false;
                        break;
                    }
                    const uint8_t *arow = smem + rs * STAGE + (q * 32 + lane) * 128;
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const uint4 u = *reinterpret_cast<const uint4 *>(arow + (((j + lane) & 7) << 4));
                        const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            ss = fmaf(bf16_lo(w4[i]), bf16_lo(w4[i]), ss);
                            ss = fmaf(bf16_hi(w4[i]), bf16_hi(w4[i]), ss);
                        }
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(empty_bar(rs));
                    if (++rs == STAGES) {
                        rs = 0;
                        rph ^= 1u;
                    }
                }
                if (!ok) break;
                const int row = mt * BM + q * 32 + lane;
                if (nt == 0 && row < args.dense_rows)
                    args.xsq_f32[(size_t)ks * args.dense_rows + row] = ss;
            }
            const int acc = it & 1;
            const uint32_t aph = (uint32_t)(it >> 1) & 1u;
            bool ok = mbar_wait_bounded(tfull_bar(acc), aph, abort_flag, args.timeout_ns,
                                        args.status, 140 + KIND);
            // the TMEM loads below are warp-collective: the whole warp continues or stops;
            // with e4m3 the four epilogue warps also meet at a named barrier per item, so
            // they continue or stop together
            if (F8 ? !named_bar_and(1, nep, ok) : !__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            const int row = wgrad ? (e * args.wg_mtiles + mt) * BM + q * 32 + lane
                                  : mt * BM + q * 32 + lane;
            const uint32_t t_row = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN);
            if (wgrad && kb1 == kb0) { // an expert without rows: a zero gradient
                uint4 *orow = reinterpret_cast<uint4 *>(args.out + (size_t)row * args.ld_out + nt * BN);
                for (int c = 0; c < BN / 8; ++c)
                    if (nt * BN + c * 8 < args.n_cols) orow[c] = make_uint4(0u, 0u, 0u, 0u);
            } else if (F8) {
                // the item's 256 column scales into shared memory once (the four epilogue
                // warps, 2 each), then broadcast reads; one buffer per accumulator, so a
                // warp rewrites a buffer only after every warp passed the next item's barrier
                float *sbs = scale_stage + acc * BN;
                const float *sbg = args.b_scale + (size_t)e * args.b_scale_ld;
                for (int i = half * 128 + q * 32 + lane; i < BN; i += nep) {
                    const int col = (KIND == GEMM_SWIGLU)
                                        ? (i < 128 ? nt * 128 + i : args.up_col + nt * 128 + i - 128)
                                        : nt * BN + i;
                    sbs[i] = col < args.b_scale_ld ? sbg[col] : 0.0f;
                }
                named_bar_sync(1, nep);
                epilogue_rows<KIND, F8>(args, t_row, row, nt, ks, e, sbs, c_lo, c_hi);
            } else {
                epilogue_rows<KIND, F8>(args, t_row, row, nt, ks, e, nullptr, c_lo, c_hi);
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

template <int KIND>
__global__ void __launch_bounds__(gemm::NUM_THREADS_GATHER, 1)
    moe_grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                            const __grid_constant__ CUtensorMap tmB, const GemmArgs args)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    grouped_gemm_cta<KIND>(tmA, tmB, args, smem, blockIdx.x, gridDim.x);
}


// The backward GEMMs (identity epilogue, bf16 out): BMODE_KMAJOR for the data gradients
// through the transposed weights, BMODE_WGRAD for the weight gradients.
template <int BMODE>
__global__ void __launch_bounds__(gemm::NUM_THREADS_GATHER, 1)
    moe_grouped_gemm_bwd_kernel(const __grid_constant__ CUtensorMap tmA,
                                const __grid_constant__ CUtensorMap tmB, const GemmArgs args)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    grouped_gemm_cta<GEMM_ACT, false, BMODE>(tmA, tmB, args, smem, blockIdx.x, gridDim.x);
}

// ---------------------------------------------------------------------------------------
// CTA-pair variant: tcgen05.mma.cta_group::2, M = 256 (128 rows per CTA), N = 256.
// ---------------------------------------------------------------------------------------
//
// Two CTAs of a cluster work on one 256-row x 256-column tile: each CTA loads its own 128
// token rows of A and its own half (128 columns) of the B tile, so per SM the B traffic and
// the shared-memory bytes per K step drop by a third compared with the single-CTA tile.
// The leader CTA (cluster rank 0) issues the MMAs for the pair; its "full" barrier counts
// the bytes of both CTAs' copies. Its commits arrive on both CTAs' "empty" and "tmem full"
// barriers; both CTAs' epilogue warps release the leader's "tmem empty" barrier. A pair of
// m-tiles always belongs to one expert; when an expert has an odd number of m-tiles, the
// second CTA's half of its last pair is computed on rows of no use and not stored.
// For layer0 (SwiGLU) CTA 0 loads the 128 gate columns and CTA 1 the matching 128 up
// columns, so each CTA's accumulator holds [gate | up] for its own rows.

namespace gemm2 {
constexpr int STAGES = 6;
constexpr int A_TILE = 128 * gemm::BK * 2;   // 16 KB per CTA
constexpr int B_TILE = 128 * gemm::BK * 2;   // 16 KB per CTA (two 64-column boxes)
constexpr int STAGE = A_TILE + B_TILE;       // 32 KB per CTA
constexpr int NUM_BARS = 2 * STAGES + 5;
constexpr int SMEM_BYTES = 1024 + STAGES * STAGE + NUM_BARS * 8 + 16;
constexpr uint32_t IDESC = idesc_bf16_f32(256, 256, /*b_mn_major=*/true);
constexpr uint32_t IDESC_F8 = idesc_e4m3_f32(256, 256);
constexpr uint16_t PAIR_MASK = 0x3;
} // namespace gemm2

__device__ __forceinline__ void gemm_map_pair(int w, const GemmArgs &a, int &e, int &mt0, int &nt)
{
    const int q = w / a.n_tiles;
    e = a.ptile_expert[q];
    const int base = a.ptile_off[e];
    const int cnt = a.ptile_off[e + 1] - base;
    const int local = w - base * a.n_tiles;
    mt0 = a.tile_off[e] + 2 * (local % cnt);
    nt = local / cnt;
}

// F8: e4m3 operands, both K-major: each CTA loads 128 rows x 128 bytes of A (its m-tile of
// gathered x codes or h codes) and one 128-row box of the expert's K-major weight codes (its
// half of N: the gate or up rows for SwiGLU); kind::f8f6f4, the scales in the epilogue.
template <int KIND, bool F8 = false>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(gemm::NUM_THREADS, 1)
    moe_grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                                 const __grid_constant__ CUtensorMap tmB, const GemmArgs args)
{
    using gemm::BK;
    using gemm::B_BOX;
    using gemm2::STAGES;
    using gemm2::STAGE;
    using gemm2::A_TILE;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + STAGES * STAGE);
    const uint32_t bar0 = smem_u32(bars);
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
    auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + a); };
    auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + 2 + a); };
    const uint32_t done_bar = bar0 + 8u * (2 * STAGES + 4);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + gemm2::NUM_BARS);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank(); // 0: leader, 1: peer
    const int pair_id = blockIdx.x >> 1;
    const int npairs = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full_bar(s), 1);  // leader: its own arrive + both CTAs' bytes
            mbar_init(empty_bar(s), 1); // the leader's multicast commit
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(tfull_bar(a), 1);
            mbar_init(tempty_bar(a), 8); // leader: 4 epilogue warps of each CTA
        }
        mbar_init(done_bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_u32(tmem_slot), gemm::TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync_all(); // barriers of both CTAs initialised before any cross-CTA signal
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const int total = args.meta->num_ptiles * args.n_tiles;
    const int KB = args.k_blocks;

    if (warp == 0) {
        // ---------------- TMA producer (whole warp, both CTAs) ----------------
        const bool gather = (args.gather_idx != nullptr);
        int s = 0;
        uint32_t ph = 0;
        bool ok = true, issued = false;
        for (int w = pair_id; ok && w < total; w += npairs) {
            int e, mt0, nt;
            gemm_map_pair(w, args, e, mt0, nt);
            const int my_mt = mt0 + (int)rank;
            int rows[4] = {0, 0, 0, 0};
            if (gather) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int64_t r = (int64_t)my_mt * 128 + 4 * lane + i;
                    const int g = (r < args.gather_len) ? args.gather_idx[r] : -1;
                    rows[i] = g < 0 ? 0 : g;
                }
            }
            for (int kb = 0; kb < KB; ++kb) {
                ok = mbar_wait_bounded(empty_bar(s), ph ^ 1u, abort_flag, args.timeout_ns,
                                       args.status, 200 + KIND);
                if (!__all_sync(0xffffffffu, ok)) {
                    ok = false;
                    break;
                }
                if (rank == 0 && lane == 0) mbar_arrive_expect_tx(full_bar(s), 2 * STAGE);
                __syncwarp();
                const uint32_t leader_full = mapa_shared(full_bar(s), 0);
                const uint32_t a_dst = smem_u32(smem + s * STAGE);
                const uint32_t b_dst = a_dst + A_TILE;
                if (gather) {
                    tma_gather4_pair(a_dst + lane * 512, &tmA, leader_full, kb * BK, rows[0],
                                     rows[1], rows[2], rows[3]);
                } else if (lane == 0) {
                    tma_load_2d_pair(a_dst, &tmA, leader_full, kb * (F8 ? 128 : BK), my_mt * 128);
                }
                if (F8 && lane == 0) { // K-major codes: this CTA's 128 weight rows
                    const int row = (KIND == GEMM_SWIGLU) ? (rank == 0 ? 0 : args.up_col) + nt * 128
                                                          : nt * gemm::BN + (int)rank * 128;
                    tma_load_3d_pair(b_dst, &tmB, leader_full, kb * 128, row, e);
                }
                if (!F8 && lane == 0) {
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        int col;
                        if (KIND == GEMM_SWIGLU)
                            col = (rank == 0 ? 0 : args.up_col) + nt * 128 + i * 64;
                        else
                            col = nt * gemm::BN + (int)rank * 128 + i * 64;
                        tma_load_3d_pair(b_dst + i * B_BOX, &tmB, leader_full, col, kb * BK, e);
                    }
                }
                issued = true;
                if (++s == STAGES) {
                    s = 0;
                    ph ^= 1u;
                }
            }
        }
        if (!ok && issued) {
            // gave up: copies already issued complete on their own; let them land before
            // the cluster exits (about 100 us)
            for (int i = 0; i < 100; ++i) __nanosleep(1000);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            if (rank == 0) {
                // ---------------- MMA issuer (leader only) ----------------
                int s = 0;
                uint32_t ph = 0;
                int it = 0;
                bool ok = true;
                for (int w = pair_id; ok && w < total; w += npairs, ++it) {
                    const int acc = it & 1;
                    const uint32_t aph = (uint32_t)(it >> 1) & 1u;
                    if (!mbar_wait_bounded(tempty_bar(acc), aph ^ 1u, abort_flag, args.timeout_ns,
                                           args.status, 210 + KIND)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t d_tmem = tmem_base + (uint32_t)(acc * gemm::BN);
                    for (int kb = 0; kb < KB; ++kb) {
                        if (!mbar_wait_bounded(full_bar(s), ph, abort_flag, args.timeout_ns,
                                               args.status, 220 + KIND)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t a_addr = smem_u32(smem + s * STAGE);
                        const uint32_t b_addr = a_addr + A_TILE;
                        const uint64_t a_desc = sw128_desc(a_addr, gemm::A_LBO, gemm::A_SBO);
                        if (F8) { // both K-major: +32 B per MMA
                            const uint64_t b_desc = sw128_desc(b_addr, gemm::A_LBO, gemm::A_SBO);
#pragma unroll
                            for (int k = 0; k < 4; ++k)
                                umma_f8_pair(d_tmem, a_desc + (uint64_t)((k * 32) >> 4),
                                             b_desc + (uint64_t)((k * 32) >> 4), gemm2::IDESC_F8,
                                             (kb | k) != 0 ? 1u : 0u);
                        } else {
                            const uint64_t b_desc = sw128_desc(b_addr, gemm::B_LBO, gemm::B_SBO);
#pragma unroll
                            for (int k = 0; k < BK / 16; ++k) {
                                umma_bf16_pair(d_tmem, a_desc + (uint64_t)((k * 32) >> 4),
                                               b_desc + (uint64_t)((k * 16 * 128) >> 4),
                                               gemm2::IDESC, (kb | k) != 0 ? 1u : 0u);
                            }
                        }
                        umma_commit_pair(empty_bar(s), gemm2::PAIR_MASK);
                        if (++s == STAGES) {
                            s = 0;
                            ph ^= 1u;
                        }
                    }
                    if (!ok) break;
                    umma_commit_pair(tfull_bar(acc), gemm2::PAIR_MASK);
                }
                // every MMA issued so far must finish before either CTA releases TMEM
                umma_commit_pair(done_bar, gemm2::PAIR_MASK);
            }
            volatile int never = 0;
            mbar_wait_bounded(done_bar, 0, &never, args.timeout_ns, args.status, 230 + KIND);
        }
    } else {
        // ---------------- epilogue: warps 2..5 of both CTAs ----------------
        const int q = warp & 3;
        int it = 0;
        for (int w = pair_id; w < total; w += npairs, ++it) {
            int e, mt0, nt;
            gemm_map_pair(w, args, e, mt0, nt);
            const int my_mt = mt0 + (int)rank;
            const bool valid = my_mt < args.tile_off[e + 1];
            const int acc = it & 1;
            const uint32_t aph = (uint32_t)(it >> 1) & 1u;
            bool ok = mbar_wait_bounded(tfull_bar(acc), aph, abort_flag, args.timeout_ns,
                                        args.status, 240 + KIND);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            if (valid) {
                const int row = my_mt * 128 + q * 32 + lane;
                const uint32_t t_row =
                    tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * gemm::BN);
                epilogue_rows<KIND, F8>(args, t_row, row, nt, 0, e);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(mapa_shared(tempty_bar(acc), 0));
        }
    }

    __syncwarp();
    tc_fence_before();
    cluster_sync_all(); // no CTA leaves while its peer may still signal its barriers
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, gemm::TMEM_COLS);
    }
}

} // namespace moe
