// route_chain.cuh -- the router for up to 32 experts in one launch: exact sequential fp32
// logits and the top-k with its gate weights (Comet: Fine-grained Computation-communication
// Overlapping for Mixture-of-Experts, §2.1 "MoE Structure": each token is routed to its
// selected experts).
//
// What it computes (the same as route_logits_kernel followed by route_topk_kernel, bit for
// bit): for token t and expert e one fp32 accumulator walks h upward,
// l[t][e] = fma(x[t][h], W_g[h][e], l[t][e]) from 0, then + b[e]; the top-k and the gates
// are those of topk_row_warp, bit for bit (topk_seg).
//
// Design for sm_100a. The order of the sum is part of the contract, so the parallelism is the
// T*E chains themselves; the kernel feeds them at the issue rate of one warp per SM
// sub-partition:
//   - one CTA per group of `tt` tokens (about one group per SM), G consumer threads per
//     token, each owning EPT experts of its token (EPT*G >= E);
//   - x arrives by TMA: per chunk of 128 h, two 64-column boxes of the CTA's tt token rows
//     (128-byte swizzle, so the 16-byte reads of 8+ consecutive rows are conflict-free);
//   - W_g arrives by TMA as stored (bf16 [128 h, E] per chunk) and one producer warp widens
//     it to fp32 in shared memory, so a consumer reads the EPT weights of one h with one
//     16-byte broadcast load (all threads of a warp sit at the same h);
//   - a consumer widens each x value once and feeds it to the EPT fused multiply-adds of its
//     experts (measured on B200: packed fma.rn.f32x2 occupies the FMA pipe for two cycles and
//     saved nothing here; the chains are bound by shared-memory delivery and load latency);
//   - stages are counted by mbarriers (x landed, W_g landed, W_g widened, stage free); every
//     wait is bounded;
//   - a consumer loads the operands of the next 8 h values into registers while it consumes
//     the current ones (software pipelining: its warp is alone on its scheduler);
//   - after the last chunk each consumer writes its logits to shared memory and the consumer
//     warps run the top-k on segments of 8, 16 or 32 lanes, several tokens per warp.
#pragma once

#include "route.cuh"

namespace moe {

constexpr int RC_HC = 128;                // h values per chunk (two 64-column x boxes)
constexpr int RC_MAX_STAGES = 6;
constexpr int RC_SMEM_BUDGET = 200 * 1024;
constexpr int RC_MAX_CONSUMERS = 512;     // consumer threads per CTA at most

struct RcArgs {
    const float *bias;  // [E] or nullptr
    int32_t *topk_idx;  // [T, k]
    float *topk_w;      // [T, k]
    int T, H, E, k, gate;
    int tt;             // tokens per CTA (rows of the x box), 1..256
    int stages;         // ring stages, 3..RC_MAX_STAGES
    int *status;        // device status word or nullptr
    int64_t timeout_ns;
};

// Shared-memory layout (offsets from the 1024-byte aligned base). Stage s holds the two x
// boxes [tt_pad rows][128 B] (swizzled), W_g as stored [128][E] bf16 and widened [128][EP]
// fp32; after the stages: the logits [tt][EP] and the barriers.
struct RcLayout {
    int tt_pad, x_box, x_bytes, wraw_bytes, wf_bytes, stage_bytes;
    int lg_off, bar_off, total;
};

__host__ __device__ inline RcLayout rc_layout(int tt, int E, int EP, int stages)
{
    RcLayout L;
    L.tt_pad = (tt + 7) & ~7;
    L.x_box = L.tt_pad * 128;          // a multiple of 1024: every box starts swizzle-aligned
    L.x_bytes = 2 * L.x_box;
    L.wraw_bytes = ((RC_HC * E * 2) + 1023) & ~1023;
    L.wf_bytes = ((RC_HC * EP * 4) + 1023) & ~1023;
    L.stage_bytes = L.x_bytes + L.wraw_bytes + L.wf_bytes;
    L.lg_off = stages * L.stage_bytes;
    L.bar_off = L.lg_off + ((tt * EP * 4 + 127) & ~127);
    L.total = L.bar_off + (4 * RC_MAX_STAGES + 2) * 8;
    return L;
}

// 16-byte shared-memory load that the compiler keeps in program order (issued early on purpose)
__device__ __forceinline__ uint4 lds_v4(uint32_t addr)
{
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr));
    return v;
}

// The top-k and gates of one token on a segment of `seg` lanes (a power of two >= E, <= 32;
// lane sl of the segment holds expert sl): the same selections and the same fp32 gate
// arithmetic as topk_row_warp on a whole warp. The warp's butterflies there add exact zeros
// (or take maxima with -inf) from the lanes past the segment, so reducing over the segment
// alone gives bitwise the same values; the argmax order (logit desc, id asc) is total.
// All lanes of the warp call it; `has` is false for a segment without a token.
__device__ __forceinline__ void topk_seg(const float *lg, int E, int k, int gate,
                                         const float *__restrict__ bias, int32_t *__restrict__ idx_out,
                                         float *__restrict__ w_out, int sl, int seg, bool has)
{
    const bool in = has && sl < E;
    const float l = in ? lg[sl] : 0.0f;
    float key = in ? ((gate == 2 && bias != nullptr) ? l + bias[sl] : l) : -INFINITY;
    float sel_val = 0.0f, top = 0.0f;
    for (int j = 0; j < k; ++j) {
        float bv = key;
        int bi = in ? sl : 0x7fffffff;
        for (int off = seg >> 1; off > 0; off >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
            if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
        }
        if (bi < 0 || bi >= E) bi = 0;
        const float gv = (gate == 2) ? __shfl_sync(0xffffffffu, l, (threadIdx.x & 31 & ~(seg - 1)) + bi) : bv;
        if (j == 0) top = gv;
        if (has && sl == 0) idx_out[j] = bi;
        if (sl == bi) key = -INFINITY; // removed from later rounds (logits are finite)
        if (j == sl) sel_val = gv;
    }
    if (gate == 2) { // the largest selected logit
        float m = sl < k ? sel_val : -INFINITY;
        for (int off = seg >> 1; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
        top = m;
    }
    float denom = 0.0f;
    if (gate == 1) {
        if (in) denom = expf(l - top);
    } else if (sl < k) {
        denom = expf(sel_val - top);
    }
    for (int off = seg >> 1; off > 0; off >>= 1) denom += __shfl_xor_sync(0xffffffffu, denom, off);
    if (has && sl < k) w_out[sl] = expf(sel_val - top) / denom;
}

template <int EPT, int G>
__global__ void __launch_bounds__(32 + RC_MAX_CONSUMERS, 1)
    route_chain_kernel(const __grid_constant__ CUtensorMap tmX,
                       const __grid_constant__ CUtensorMap tmW, const RcArgs a)
{
    static_assert(EPT == 4 || EPT == 8, "experts per thread");
    constexpr int EP = EPT * G;
    extern __shared__ uint8_t rc_smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(rc_smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int ncw = (blockDim.x >> 5) - 1; // consumer warps
    const int S = a.stages;
    const RcLayout L = rc_layout(a.tt, a.E, EP, S);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L.bar_off);
    const uint32_t bar0 = smem_u32(bars);
    auto xb_bar = [&](int s) { return bar0 + 8u * s; };                      // x landed
    auto raw_bar = [&](int s) { return bar0 + 8u * (RC_MAX_STAGES + s); };   // W_g landed
    auto wf_bar = [&](int s) { return bar0 + 8u * (2 * RC_MAX_STAGES + s); }; // W_g widened
    auto empty_bar = [&](int s) { return bar0 + 8u * (3 * RC_MAX_STAGES + s); };
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + 4 * RC_MAX_STAGES);
    auto stage = [&](int s) { return sm + (size_t)s * L.stage_bytes; };

    if (a.status != nullptr && blockIdx.x == 0 && threadIdx.x == 0) {
        a.status[0] = DEV_OK; // a new call starts with a clean status word
        a.status[1] = 0;
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(xb_bar(s), 1);
            mbar_init(raw_bar(s), 1);
            mbar_init(wf_bar(s), 32);
            mbar_init(empty_bar(s), ncw);
        }
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmX);
        tma_prefetch_desc(&tmW);
    }
    __syncthreads();

    const int t0 = blockIdx.x * a.tt;
    const int nchunk = (a.H + RC_HC - 1) / RC_HC; // a short last chunk reads zeros past H
    const uint32_t x_tx = 2u * (uint32_t)a.tt * 128u;
    const uint32_t w_tx = (uint32_t)(RC_HC * a.E * 2);

    if (warp == 0) {
        // ---------------- producer: TMA issue and W_g widening ----------------
        const int D = S - 2; // chunks of TMA lead over the widening
        int armed_ph[RC_MAX_STAGES];
#pragma unroll
        for (int i = 0; i < RC_MAX_STAGES; ++i) armed_ph[i] = -1;
        bool ok = true;
        // chunk c goes to stage c % S once the consumers have finished chunk c - S
        auto issue = [&](int c) -> bool {
            const int s = c % S;
            if (c >= S && !mbar_wait_bounded(empty_bar(s), (uint32_t)((c / S - 1) & 1), abort_flag,
                                             a.timeout_ns, a.status, 701))
                return false;
            const uint32_t xd = smem_u32(stage(s));
            mbar_arrive_expect_tx(raw_bar(s), w_tx);
            tma_load_2d(xd + L.x_bytes, &tmW, raw_bar(s), 0, c * RC_HC);
            mbar_arrive_expect_tx(xb_bar(s), x_tx);
            tma_load_2d(xd, &tmX, xb_bar(s), c * RC_HC, t0);
            tma_load_2d(xd + L.x_box, &tmX, xb_bar(s), c * RC_HC + 64, t0);
            armed_ph[s] = (c / S) & 1;
            return true;
        };
        if (lane == 0)
            for (int c = 0; c < D && c < nchunk && ok; ++c) ok = issue(c);
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        const int n8 = a.E / 8; // 16-byte pieces of one W_g row
        for (int c = 0; ok && c < nchunk; ++c) {
            const int s = c % S;
            ok = mbar_wait_bounded(raw_bar(s), (uint32_t)((c / S) & 1), abort_flag, a.timeout_ns,
                                   a.status, 702);
            if (!__all_sync(0xffffffffu, ok)) {
                ok = false;
                break;
            }
            const uint4 *wr = reinterpret_cast<const uint4 *>(stage(s) + L.x_bytes);
            float *wf = reinterpret_cast<float *>(stage(s) + L.x_bytes + L.wraw_bytes);
            for (int i = lane; i < RC_HC * n8; i += 32) {
                const int h = i / n8, g = i - h * n8;
                const uint4 u = wr[i];
                float4 *d = reinterpret_cast<float4 *>(wf + h * EP + g * 8);
                d[0] = make_float4(bf16_lo(u.x), bf16_hi(u.x), bf16_lo(u.y), bf16_hi(u.y));
                d[1] = make_float4(bf16_lo(u.z), bf16_hi(u.z), bf16_lo(u.w), bf16_hi(u.w));
            }
            mbar_arrive(wf_bar(s)); // every lane: its own widened pieces are published
            if (lane == 0 && c + D < nchunk) ok = issue(c + D);
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        }
        // every copy issued has landed before the CTA exits (immediate in a normal run)
        if (lane == 0) {
            volatile int never = 0;
            for (int s = 0; s < S; ++s)
                if (armed_ph[s] >= 0) {
                    mbar_wait_bounded(xb_bar(s), (uint32_t)armed_ph[s], &never, a.timeout_ns, nullptr, 0);
                    mbar_wait_bounded(raw_bar(s), (uint32_t)armed_ph[s], &never, a.timeout_ns, nullptr, 0);
                }
        }
    } else {
        // ---------------- consumers: the fp32 chains ----------------
        const int cid = threadIdx.x - 32;
        int r = cid / G;
        const int grp = cid - r * G;
        const bool live = r < a.tt;
        if (!live) r = 0; // lanes past the CTA's tokens compute on row 0 and store nothing
        float acc[EPT];
#pragma unroll
        for (int i = 0; i < EPT; ++i) acc[i] = 0.0f;
        bool ok = true;
        const int rsw = r & 7;
        // Operands of one group of 8 h values: the 16-byte x piece and the 8 weight rows of
        // this thread's experts. The next group's shared-memory loads are issued (volatile, so
        // they stay ahead of the arithmetic) before the current group's FMAs: a consumer warp is
        // alone on its scheduler, so the load latency must be covered by its own arithmetic.
        const uint32_t xrow0 = smem_u32(stage(0)) + (uint32_t)(r * 128);
        const uint32_t wrow0 = smem_u32(stage(0)) + (uint32_t)(L.x_bytes + L.wraw_bytes + grp * EPT * 4);
        struct Grp {
            uint4 x;
            uint4 w[8][EPT / 4];
        };
        auto load_grp = [&](Grp &gq, int s, int g) {
            const uint32_t so = (uint32_t)(s * L.stage_bytes);
            gq.x = lds_v4(xrow0 + so + (uint32_t)((g >> 3) * L.x_box + (((g & 7) ^ rsw) << 4)));
#pragma unroll
            for (int q = 0; q < 8; ++q)
#pragma unroll
                for (int v = 0; v < EPT / 4; ++v)
                    gq.w[q][v] = lds_v4(wrow0 + so + (uint32_t)((g * 8 + q) * EP * 4 + v * 16));
        };
        auto fma_grp = [&](const Grp &gq) {
            const uint32_t xw[4] = {gq.x.x, gq.x.y, gq.x.z, gq.x.w};
#pragma unroll
            for (int q = 0; q < 8; ++q) { // h ascending within every chain
                const float xf = __uint_as_float((q & 1) ? (xw[q >> 1] & 0xFFFF0000u) : (xw[q >> 1] << 16));
#pragma unroll
                for (int v = 0; v < EPT / 4; ++v) {
                    acc[4 * v + 0] = fmaf(xf, __uint_as_float(gq.w[q][v].x), acc[4 * v + 0]);
                    acc[4 * v + 1] = fmaf(xf, __uint_as_float(gq.w[q][v].y), acc[4 * v + 1]);
                    acc[4 * v + 2] = fmaf(xf, __uint_as_float(gq.w[q][v].z), acc[4 * v + 2]);
                    acc[4 * v + 3] = fmaf(xf, __uint_as_float(gq.w[q][v].w), acc[4 * v + 3]);
                }
            }
        };
        for (int c = 0; c < nchunk; ++c) {
            const int s = c % S;
            const uint32_t ph = (uint32_t)((c / S) & 1);
            ok = mbar_wait_bounded(xb_bar(s), ph, abort_flag, a.timeout_ns, a.status, 711) &&
                 mbar_wait_bounded(wf_bar(s), ph, abort_flag, a.timeout_ns, a.status, 712);
            if (!__all_sync(0xffffffffu, ok)) {
                ok = false;
                break;
            }
            Grp g0, g1;
            load_grp(g0, s, 0);
#pragma unroll
            for (int g = 0; g < RC_HC / 8; g += 2) {
                load_grp(g1, s, g + 1);
                fma_grp(g0);
                if (g + 2 < RC_HC / 8) load_grp(g0, s, g + 2);
                fma_grp(g1);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(empty_bar(s));
        }
        // logits of this thread's experts (+ b[e], except with the selection-only bias)
        float *lg = reinterpret_cast<float *>(sm + L.lg_off);
        const float *lbias = (a.gate == 2) ? nullptr : a.bias;
        if (ok && live) {
#pragma unroll
            for (int i = 0; i < EPT; ++i) {
                const int e = grp * EPT + i;
                float v = acc[i];
                if (e < a.E) {
                    if (lbias != nullptr) v = v + lbias[e];
                    lg[r * EP + e] = v;
                }
            }
        }
        // every consumer thread has stored its logits (or every warp has given up)
        ok = named_bar_and(1, ncw * 32, ok);
        if (ok) {
            // top-k: SEG lanes per token (the experts' count rounded up to a power of two),
            // 32 / SEG tokens per warp at a time
            const int cw = warp - 1;
            const int seg = a.E <= 8 ? 8 : a.E <= 16 ? 16 : 32;
            const int per = 32 / seg;
            const int sl = lane & (seg - 1);
            const int sub = lane / seg;
            for (int rr0 = cw * per; rr0 < a.tt; rr0 += ncw * per) {
                const int rr = rr0 + sub;
                const int t = t0 + rr;
                const bool has = rr < a.tt && t < a.T;
                topk_seg(lg + (has ? rr : 0) * EP, a.E, a.k, a.gate, a.bias,
                         a.topk_idx + (size_t)t * a.k, a.topk_w + (size_t)t * a.k, sl, seg, has);
            }
        }
    }
    __syncthreads();
}

} // namespace moe
