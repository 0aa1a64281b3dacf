// fused.cuh -- one persistent launch for layer0, layer1 and the combine, scheduled by
// tile-level ready flags.
//
// Where it comes from (Comet: Fine-grained Computation-communication Overlapping for
// Mixture-of-Experts; and "Fine-grained Computation-Communication Overlap via Tile-level
// Signaling and Scheduling for MoE"):
//   - shared-tensor dependency resolving (Comet §3.1.1): the tensor shared by layer0 and
//     layer1 is h; layer0 produces it in 128-row M tiles, and a layer1 tile only needs the
//     h rows of its own M tile, so layer1 work starts tile by tile as layer0 finishes rows;
//   - layer1 is decomposed along N (§3.1.1, column-wise §3.1.2): a combine item reduces one
//     256-column stripe of the output, and needs only that stripe of every layer1 tile;
//   - the tile-signalling design's producer (one persistent kernel over all local experts)
//     and its consumer driven by ready flags as tiles finish: here both live in one launch,
//     the ready flags are gpu-scope counters in global memory, and every wait is bounded.
//
// Work items form one static queue in dependency order:
//   [ layer0 tiles (expert, m, n) | layer1 tiles (expert, m, n) | combine (stripe, tokens) ]
// CTA b takes items b, b + grid, b + 2 grid, ... All CTAs are resident at once (one per SM),
// every item waits only on items earlier in the queue, and a CTA finishes all its earlier
// items before waiting, so the waits always end.
//   ready0[m] counts finished layer0 column tiles of M tile m; a layer1 tile of m waits for
//             ready0[m] == layer0 N tiles before its TMA loads of h;
//   ready1[n] counts finished layer1 M tiles of column stripe n; a combine item of stripe n
//             waits for ready1[n] == number of M tiles.
// Writers publish with a gpu-scope release after their stores and a generic-to-async proxy
// fence (layer1 reads h with TMA); readers acquire, then fence again before their TMA.
#pragma once

#include "gemm_tc.cuh"

namespace moe {

constexpr int COMBINE_TOKENS = 128; // tokens per combine item

struct FusedArgs {
    GemmArgs l0;            // layer0: rows gathered from x, W1, writes h
    GemmArgs l1;            // layer1: h rows by TMA, W2, writes ys (gate-scaled)
    int *ready0;            // [max_tiles]
    int *ready1;            // [layer1 N tiles]
    const int32_t *inv_pos; // [T, k]
    __nv_bfloat16 *out;     // [T, H]
    int T, H, k;
    int64_t ys_rows;
    const __nv_bfloat16 *ys_shared; // [T, H] shared-expert rows added last, or nullptr
    int fault_skip;         // test hook: layer0 item whose ready signal is withheld (-1: none)
};

__device__ __forceinline__ int ld_acquire_gpu(const int *p)
{
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void red_release_gpu_add(int *p, int v)
{
    asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ void fence_proxy_async_global()
{
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Bounded wait for *p >= target with acquire semantics. False after an abort elsewhere in
// the CTA or after timeout_ns (then the abort flag is raised and DEV_TIMEOUT recorded).
__device__ __forceinline__ bool flag_wait_bounded(const int *p, int target, volatile int *abort_flag,
                                                  int64_t timeout_ns, int *status, int where)
{
    if (ld_acquire_gpu(p) >= target) return true;
    const uint64_t t0 = globaltimer_ns();
#pragma unroll 1
    while (true) {
        __nanosleep(128);
        if (ld_acquire_gpu(p) >= target) return true;
        if (*abort_flag) return false;
        if ((int64_t)(globaltimer_ns() - t0) > timeout_ns) {
            *abort_flag = 1;
            record_status(status, DEV_TIMEOUT, where);
            return false;
        }
    }
}

struct FusedItem {
    int phase; // 0 layer0, 1 layer1, 2 combine
    int e, mt, nt;
};

__device__ __forceinline__ FusedItem fused_item(int w, const FusedArgs &fa, int total0, int total1)
{
    FusedItem it{};
    if (w < total0) {
        it.phase = 0;
        gemm_map_work(w, fa.l0, it.e, it.mt, it.nt);
    } else if (w < total0 + total1) {
        it.phase = 1;
        gemm_map_work(w - total0, fa.l1, it.e, it.mt, it.nt);
    } else {
        const int v = w - total0 - total1;
        const int chunks = (fa.T + COMBINE_TOKENS - 1) / COMBINE_TOKENS;
        it.phase = 2;
        it.nt = v / chunks; // output column stripe
        it.mt = v % chunks; // token chunk
        it.e = 0;
    }
    return it;
}

// Combine of one item (256-column stripe x 128 tokens) by eight warps: warp wq (0..7) takes
// tokens wq, wq + 8, ... of the chunk, eight of them at a time so that eight 16-byte rows per
// lane are in flight; lane l owns columns stripe*256 + 8l .. +7. Sum over j ascending in fp32,
// one bf16 rounding.
__device__ __forceinline__ void fused_combine(const FusedArgs &fa, int stripe, int chunk, int wq,
                                              int lane, int *status)
{
    const int col = stripe * gemm::BN + lane * 8;
    if (col >= fa.H) return;
    const __nv_bfloat16 *ys = fa.l1.out;
    for (int g = 0; g < COMBINE_TOKENS / 64; ++g) {
        int t[8];
        float a[8][8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            t[i] = chunk * COMBINE_TOKENS + g * 64 + i * 8 + wq;
#pragma unroll
            for (int c = 0; c < 8; ++c) a[i][c] = 0.0f;
        }
        for (int j = 0; j < fa.k; ++j) {
            uint4 u[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                u[i] = make_uint4(0u, 0u, 0u, 0u);
                if (t[i] < fa.T) {
                    const int r = fa.inv_pos[(size_t)t[i] * fa.k + j];
                    if (r >= 0 && (int64_t)r < fa.ys_rows)
                        u[i] = *reinterpret_cast<const uint4 *>(ys + (size_t)r * fa.H + col);
                    else
                        record_status(status, DEV_BAD_INDEX, 331);
                }
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                a[i][0] += bf16_lo(u[i].x); a[i][1] += bf16_hi(u[i].x);
                a[i][2] += bf16_lo(u[i].y); a[i][3] += bf16_hi(u[i].y);
                a[i][4] += bf16_lo(u[i].z); a[i][5] += bf16_hi(u[i].z);
                a[i][6] += bf16_lo(u[i].w); a[i][7] += bf16_hi(u[i].w);
            }
        }
        if (fa.ys_shared != nullptr) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                if (t[i] >= fa.T) continue;
                const uint4 u = *reinterpret_cast<const uint4 *>(fa.ys_shared + (size_t)t[i] * fa.H + col);
                a[i][0] += bf16_lo(u.x); a[i][1] += bf16_hi(u.x);
                a[i][2] += bf16_lo(u.y); a[i][3] += bf16_hi(u.y);
                a[i][4] += bf16_lo(u.z); a[i][5] += bf16_hi(u.z);
                a[i][6] += bf16_lo(u.w); a[i][7] += bf16_hi(u.w);
            }
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            if (t[i] >= fa.T) continue;
            uint4 o;
            o.x = pack_bf16x2(a[i][0], a[i][1]);
            o.y = pack_bf16x2(a[i][2], a[i][3]);
            o.z = pack_bf16x2(a[i][4], a[i][5]);
            o.w = pack_bf16x2(a[i][6], a[i][7]);
            *reinterpret_cast<uint4 *>(fa.out + (size_t)t[i] * fa.H + col) = o;
        }
    }
}

template <int KIND0>
__global__ void __launch_bounds__(gemm::NUM_THREADS_GATHER, 1)
    moe_fused_layer_kernel(const __grid_constant__ CUtensorMap tmW1,
                           const __grid_constant__ CUtensorMap tmH,
                           const __grid_constant__ CUtensorMap tmW2, const FusedArgs fa)
{
    using namespace gemm;
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
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + NUM_BARS);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    int *warps_done = reinterpret_cast<int *>(tmem_slot + 2); // [2], per accumulator buffer

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const GemmArgs &l0 = fa.l0;
    const GemmArgs &l1 = fa.l1;
    int *status = l0.status;
    const int64_t tmo = l0.timeout_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full_bar(s), 1 + GATHER_THREADS); // TMA arrive + one per gather thread
            mbar_init(empty_bar(s), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(tfull_bar(a), 1);
            mbar_init(tempty_bar(a), 4);
        }
        mbar_init(done_bar, 1);
        *abort_flag = 0;
        warps_done[0] = 0;
        warps_done[1] = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmW1);
        tma_prefetch_desc(&tmH);
        tma_prefetch_desc(&tmW2);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const int num_tiles = l0.meta->num_tiles;
    const int total0 = num_tiles * l0.n_tiles;
    const int total1 = num_tiles * l1.n_tiles;
    const int total2 = l1.n_tiles * ((fa.T + COMBINE_TOKENS - 1) / COMBINE_TOKENS);
    const int total = total0 + total1 + total2;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer ----------------
            int s = 0;
            uint32_t ph = 0;
            int armed[STAGES];
#pragma unroll
            for (int i = 0; i < STAGES; ++i) armed[i] = -1;
            bool ok = true;
            for (int w = blockIdx.x; ok && w < total; w += gridDim.x) {
                const FusedItem it = fused_item(w, fa, total0, total1);
                if (it.phase == 2) continue;
                if (it.phase == 1) {
                    // layer1 needs every layer0 column tile of its M tile
                    if (!flag_wait_bounded(fa.ready0 + it.mt, l0.n_tiles, abort_flag, tmo, status,
                                           300)) {
                        ok = false;
                        break;
                    }
                    fence_proxy_async_global(); // h was written by generic stores
                }
                const int KB = it.phase == 0 ? l0.k_blocks : l1.k_blocks;
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait_bounded(empty_bar(s), ph ^ 1u, abort_flag, tmo, status, 301)) {
                        ok = false;
                        break;
                    }
                    const uint32_t a_dst = smem_u32(smem + s * STAGE);
                    const uint32_t b_dst = a_dst + A_TILE;
                    mbar_arrive_expect_tx(full_bar(s), it.phase == 0 ? B_TILE : STAGE);
                    armed[s] = (int)ph;
                    if (it.phase == 0) {
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            int col;
                            if (KIND0 == GEMM_SWIGLU)
                                col = (i < 2 ? it.nt * 128 + i * 64
                                             : l0.up_col + it.nt * 128 + (i - 2) * 64);
                            else
                                col = it.nt * BN + i * 64;
                            tma_load_3d(b_dst + i * B_BOX, &tmW1, full_bar(s), col, kb * BK, it.e);
                        }
                    } else {
                        tma_load_2d(a_dst, &tmH, full_bar(s), kb * BK, it.mt * BM);
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            tma_load_3d(b_dst + i * B_BOX, &tmW2, full_bar(s), it.nt * BN + i * 64,
                                        kb * BK, it.e);
                    }
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            for (int i = 0; i < STAGES; ++i)
                if (armed[i] >= 0) {
                    volatile int never = 0;
                    mbar_wait_bounded(full_bar(i), (uint32_t)armed[i], &never, tmo, nullptr, 0);
                }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- MMA issuer ----------------
            int s = 0;
            uint32_t ph = 0;
            int n = 0; // accumulator tiles issued
            bool ok = true;
            for (int w = blockIdx.x; ok && w < total; w += gridDim.x) {
                const FusedItem it = fused_item(w, fa, total0, total1);
                if (it.phase == 2) continue;
                const int acc = n & 1;
                const uint32_t aph = (uint32_t)(n >> 1) & 1u;
                if (!mbar_wait_bounded(tempty_bar(acc), aph ^ 1u, abort_flag, tmo, status, 310)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
                const int KB = it.phase == 0 ? l0.k_blocks : l1.k_blocks;
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait_bounded(full_bar(s), ph, abort_flag, tmo, status, 311)) {
                        ok = false;
                        break;
                    }
                    fence_proxy_async_smem(); // gathered rows arrive through the generic proxy
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smem + s * STAGE);
                    const uint32_t b_addr = a_addr + A_TILE;
                    const uint64_t a_desc = sw128_desc(a_addr, A_LBO, A_SBO);
                    const uint64_t b_desc = sw128_desc(b_addr, B_LBO, B_SBO);
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k)
                        umma_bf16(d_tmem, a_desc + (uint64_t)((k * 32) >> 4),
                                  b_desc + (uint64_t)((k * 16 * 128) >> 4), IDESC,
                                  (kb | k) != 0 ? 1u : 0u);
                    umma_commit(empty_bar(s));
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (!ok) break;
                umma_commit(tfull_bar(acc));
                ++n;
            }
            umma_commit(done_bar);
            volatile int never = 0;
            mbar_wait_bounded(done_bar, 0, &never, tmo, status, 312);
        }
    } else if (warp >= 6) {
        // ---------------- layer0 A-row gather (cp.async), warps 6..9 ----------------
        const int g = threadIdx.x - NUM_THREADS;
        const int chunk = g & 7;
        const int r0 = g >> 3;
        int s = 0;
        uint32_t ph = 0;
        bool ok = true;
        for (int w = blockIdx.x; ok && w < total; w += gridDim.x) {
            const FusedItem it = fused_item(w, fa, total0, total1);
            if (it.phase == 2) {
                // the gather warps help with the combine (warps 4..7 of its eight)
                ok = flag_wait_bounded(fa.ready1 + it.nt, num_tiles, abort_flag, tmo, status, 332);
                if (!__all_sync(0xffffffffu, ok)) {
                    ok = false;
                    break;
                }
                fused_combine(fa, it.nt, it.mt, 4 + (warp - 6), lane, status);
                continue;
            }
            const __nv_bfloat16 *src[8];
            if (it.phase == 0) {
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int64_t r = (int64_t)it.mt * BM + r0 + 16 * i;
                    int t = (r < l0.gather_len) ? l0.gather_idx[r] : -1;
                    if (t < 0 || t >= l0.gather_rows) t = 0;
                    src[i] = l0.gather_src + (size_t)t * l0.gather_ld + chunk * 8;
                }
            }
            const int KB = it.phase == 0 ? l0.k_blocks : l1.k_blocks;
            for (int kb = 0; kb < KB; ++kb) {
                ok = mbar_wait_bounded(empty_bar(s), ph ^ 1u, abort_flag, tmo, status, 320);
                if (!__all_sync(0xffffffffu, ok)) {
                    ok = false;
                    break;
                }
                if (it.phase == 0) {
                    const uint32_t a_dst = smem_u32(smem + s * STAGE);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int r = r0 + 16 * i;
                        cp_async_16_cg(a_dst + r * 128 + ((chunk ^ (r & 7)) << 4), src[i] + kb * BK);
                    }
                }
                // layer1 stages carry no gathered rows: the arrival is immediate
                cp_async_arrive_noinc(full_bar(s));
                if (++s == STAGES) {
                    s = 0;
                    ph ^= 1u;
                }
            }
        }
        cp_async_wait_all();
    } else {
        // ---------------- epilogue + combine: warps 2..5 ----------------
        const int q = warp & 3;
        int n = 0;
        for (int w = blockIdx.x; w < total; w += gridDim.x) {
            const FusedItem it = fused_item(w, fa, total0, total1);
            if (it.phase == 2) {
                // combine stripe it.nt for tokens it.mt*128 .. +127: out = sum_j ys[inv_pos]
                bool ok = flag_wait_bounded(fa.ready1 + it.nt, num_tiles, abort_flag, tmo, status,
                                            330);
                if (!__all_sync(0xffffffffu, ok)) break;
                fused_combine(fa, it.nt, it.mt, q, lane, status);
                continue;
            }
            const int acc = n & 1;
            const uint32_t aph = (uint32_t)(n >> 1) & 1u;
            bool ok = mbar_wait_bounded(tfull_bar(acc), aph, abort_flag, tmo, status, 340);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            const int row = it.mt * BM + q * 32 + lane;
            const uint32_t t_row = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN);
            if (it.phase == 0)
                epilogue_rows<KIND0>(l0, t_row, row, it.nt);
            else
                epilogue_rows<GEMM_SCALE>(l1, t_row, row, it.nt);
            // Ready signal: the last of the four epilogue warps to finish this tile publishes
            // it (before releasing the accumulator, so a buffer's counter is never reused
            // while a slower warp still holds the previous tile).
            __threadfence();
            __syncwarp();
            if (lane == 0) {
                const int prev = atomicAdd(&warps_done[acc], 1);
                if (prev == 3) {
                    warps_done[acc] = 0;
                    __threadfence();
                    const bool withhold = (it.phase == 0 && w == fa.fault_skip);
                    if (!withhold) {
                        fence_proxy_async_global();
                        red_release_gpu_add(it.phase == 0 ? fa.ready0 + it.mt : fa.ready1 + it.nt, 1);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tempty_bar(acc));
            ++n;
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
