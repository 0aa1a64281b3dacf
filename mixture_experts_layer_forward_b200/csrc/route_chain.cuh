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
//   - W_g arrives by TMA as stored (bf16 [128 h, E] per chunk); a consumer reads the EPT
//     weights of one h with one 8-byte load that all threads of a warp share (they sit at
//     the same h);
//   - neither operand is widened: the mixed-precision fused multiply-add of sm_100
//     (bf16 x bf16 + fp32, rounded once to fp32) takes the bf16 halves of the packed words.
//     A bf16 product is exact in fp32, so each step is bitwise fmaf on the widened values.
//     Against widening W_g to fp32 in shared memory and x in registers it measured 49.3 ->
//     36.8 us on the Mixtral-shaped router (T=8192, H=4096, E=8) and 139 -> 86 us on
//     T=16384, E=16 (half the shared-memory bytes per step, no widening pass);
//   - stages are counted by mbarriers (x landed, W_g landed, stage free); every wait is
//     bounded; the producer warp only keeps the ring of stages full;
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
    int tt;             // tokens per group (rows of the x box), 1..256
    int stages;         // ring stages, 3..RC_MAX_STAGES
    int *status;        // device status word or nullptr
    int64_t timeout_ns;
    int32_t *group_counts; // [ceil(T / tt)][E] selections per group and expert, or nullptr
};

// Shared-memory layout (offsets from the 1024-byte aligned base). Stage s holds the two x
// boxes [tt_pad rows][128 B] (swizzled) and W_g as stored [128][E] bf16; after the stages:
// the logits [tt][EP] and the barriers. Consumers of experts past E (E = 24: the last group
// of 4) read up to 16 bytes past a stage's W_g rows, inside the next region, and store
// nothing from those chains.
struct RcLayout {
    int tt_pad, x_box, x_bytes, w_bytes, stage_bytes;
    int lg_off, bar_off, cnt_off, total;
};

__host__ __device__ inline RcLayout rc_layout(int tt, int E, int EP, int stages)
{
    RcLayout L;
    L.tt_pad = (tt + 7) & ~7;
    L.x_box = L.tt_pad * 128;          // a multiple of 1024: every box starts swizzle-aligned
    L.x_bytes = 2 * L.x_box;
    L.w_bytes = ((RC_HC * E * 2) + 1023) & ~1023;
    L.stage_bytes = L.x_bytes + L.w_bytes;
    L.lg_off = stages * L.stage_bytes;
    L.bar_off = L.lg_off + ((tt * EP * 4 + 127) & ~127);
    L.cnt_off = L.bar_off + (3 * RC_MAX_STAGES + 2) * 8;
    L.total = L.cnt_off + 32 * 4;      // per-expert selection counts of a group (E <= 32)
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

// 8-byte shared-memory load, kept in program order like lds_v4
__device__ __forceinline__ uint2 lds_v2(uint32_t addr)
{
    uint2 v;
    asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
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
                                         float *__restrict__ w_out, int sl, int seg, bool has,
                                         int *cnt = nullptr)
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
        if (has && sl == 0) {
            idx_out[j] = bi;
            if (cnt != nullptr) atomicAdd(&cnt[bi], 1); // shared-memory count of the group
        }
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

// Barriers of the ring, from one thread before the CTA's first barrier sync: `ncw` consumer
// warps release each stage.
__device__ __forceinline__ void rc_init(uint8_t *sm, const RcLayout &L, int S, int ncw)
{
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L.bar_off);
    const uint32_t bar0 = smem_u32(bars);
    for (int s = 0; s < S; ++s) {
        mbar_init(bar0 + 8u * s, 1);                           // x landed
        mbar_init(bar0 + 8u * (RC_MAX_STAGES + s), 1);         // W_g landed
        mbar_init(bar0 + 8u * (2 * RC_MAX_STAGES + s), ncw);   // stage free
    }
    *reinterpret_cast<volatile int *>(bars + 3 * RC_MAX_STAGES) = 0; // abort flag
    int *cnt = reinterpret_cast<int *>(sm + L.cnt_off);
    for (int e = 0; e < 32; ++e) cnt[e] = 0;
    fence_mbar_init();
}

// Invalidates the ring's barriers (one thread, after a CTA barrier sync that follows rc_run),
// so that the shared memory can be used for something else.
__device__ __forceinline__ void rc_fini(uint8_t *sm, const RcLayout &L, int S)
{
    const uint32_t bar0 = smem_u32(sm + L.bar_off);
    for (int s = 0; s < S; ++s)
        for (int b = 0; b < 3; ++b) mbar_inval(bar0 + 8u * (b * RC_MAX_STAGES + s));
}

// Routes the token groups g_first, g_first + g_step, ... < n_groups (group g: tokens
// g * tt .. g * tt + tt - 1) with the ring at `sm` (1024-byte aligned, initialised by
// rc_init): warp `pw` issues the TMA copies, warps cw0 .. cw0 + ncw - 1 are the consumers
// (G threads per token). Chunk numbering runs on across the groups, so the ring never
// drains between them. After each group's top-k, with a.group_counts set, the consumers write
// the group's selections per expert. Returns false when a wait gave up.
template <int EPT, int G>
__device__ __forceinline__ bool rc_run(const CUtensorMap *tmX, const CUtensorMap *tmW, const RcArgs &a,
                                       uint8_t *sm, int pw, int cw0, int ncw, int g_first, int g_step,
                                       int n_groups, int bar_id)
{
    static_assert(EPT == 4 || EPT == 8, "experts per thread");
    constexpr int EP = EPT * G;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int S = a.stages;
    const RcLayout L = rc_layout(a.tt, a.E, EP, S);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L.bar_off);
    const uint32_t bar0 = smem_u32(bars);
    auto xb_bar = [&](int s) { return bar0 + 8u * s; };
    auto raw_bar = [&](int s) { return bar0 + 8u * (RC_MAX_STAGES + s); };
    auto empty_bar = [&](int s) { return bar0 + 8u * (2 * RC_MAX_STAGES + s); };
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + 3 * RC_MAX_STAGES);
    int *cnt = reinterpret_cast<int *>(sm + L.cnt_off);
    auto stage = [&](int s) { return sm + (size_t)s * L.stage_bytes; };

    const int nchunk = (a.H + RC_HC - 1) / RC_HC; // a short last chunk reads zeros past H
    const int my_groups = g_first < n_groups ? (n_groups - 1 - g_first) / g_step + 1 : 0;
    const int total = my_groups * nchunk;
    const uint32_t x_tx = 2u * (uint32_t)a.tt * 128u;
    const uint32_t w_tx = (uint32_t)(RC_HC * a.E * 2);
    bool ok = true;

    if (warp == pw) {
        // ---------------- producer: keeps the ring of stages full ----------------
        int armed_ph[RC_MAX_STAGES];
#pragma unroll
        for (int i = 0; i < RC_MAX_STAGES; ++i) armed_ph[i] = -1;
        if (lane == 0) {
            // chunk c goes to stage c % S once the consumers have finished chunk c - S
            for (int c = 0; c < total; ++c) {
                const int s = c % S;
                if (c >= S && !mbar_wait_bounded(empty_bar(s), (uint32_t)((c / S - 1) & 1), abort_flag,
                                                 a.timeout_ns, a.status, 701)) {
                    ok = false;
                    break;
                }
                const int t0 = (g_first + (c / nchunk) * g_step) * a.tt;
                const int h0 = (c % nchunk) * RC_HC;
                const uint32_t xd = smem_u32(stage(s));
                mbar_arrive_expect_tx(raw_bar(s), w_tx);
                tma_load_2d(xd + L.x_bytes, tmW, raw_bar(s), 0, h0);
                mbar_arrive_expect_tx(xb_bar(s), x_tx);
                tma_load_2d(xd, tmX, xb_bar(s), h0, t0);
                tma_load_2d(xd + L.x_box, tmX, xb_bar(s), h0 + 64, t0);
                armed_ph[s] = (c / S) & 1;
            }
            // every copy issued has landed before the ring is left (immediate in a normal run)
            volatile int never = 0;
            for (int s = 0; s < S; ++s)
                if (armed_ph[s] >= 0) {
                    mbar_wait_bounded(xb_bar(s), (uint32_t)armed_ph[s], &never, a.timeout_ns, nullptr, 0);
                    mbar_wait_bounded(raw_bar(s), (uint32_t)armed_ph[s], &never, a.timeout_ns, nullptr, 0);
                }
        }
        return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    }
    if (warp < cw0 || warp >= cw0 + ncw) return true;

    // ---------------- consumers: the fp32 chains ----------------
    const int cid = threadIdx.x - 32 * cw0;
    int r = cid / G;
    const int grp = cid - r * G;
    const bool live = r < a.tt;
    if (!live) r = 0; // lanes past the group's tokens compute on row 0 and store nothing
    const int rsw = r & 7;
    // Operands of one group of 8 h values: the 16-byte x piece and the 8 weight rows of this
    // thread's experts. The next group's shared-memory loads are issued (volatile, so they
    // stay ahead of the arithmetic) before the current group's FMAs: a consumer warp is alone
    // on its scheduler, so the load latency must be covered by its own arithmetic.
    const uint32_t xrow0 = smem_u32(stage(0)) + (uint32_t)(r * 128);
    // W_g rows as landed, [128][E] bf16: this thread's EPT experts of one h are 8*EPT/4 bytes
    const uint32_t wrow0 = smem_u32(stage(0)) + (uint32_t)(L.x_bytes + grp * EPT * 2);
    const int wstride = a.E * 2;
    float acc[EPT];
    struct Grp {
        uint4 x;
        uint32_t w[8][EPT / 2]; // bf16 weight pairs (experts 2v, 2v + 1) of 8 h values
    };
    auto load_grp = [&](Grp &gq, int s, int g) {
        const uint32_t so = (uint32_t)(s * L.stage_bytes);
        gq.x = lds_v4(xrow0 + so + (uint32_t)((g >> 3) * L.x_box + (((g & 7) ^ rsw) << 4)));
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const uint32_t wa = wrow0 + so + (uint32_t)((g * 8 + q) * wstride);
#pragma unroll
            for (int v = 0; v < EPT / 4; ++v) {
                const uint2 u = lds_v2(wa + v * 8);
                gq.w[q][2 * v] = u.x;
                gq.w[q][2 * v + 1] = u.y;
            }
        }
    };
    auto fma_grp = [&](const Grp &gq) {
        const uint32_t xw[4] = {gq.x.x, gq.x.y, gq.x.z, gq.x.w};
#pragma unroll
        for (int q = 0; q < 8; ++q) { // h ascending within every chain
#pragma unroll
            for (int v = 0; v < EPT / 2; ++v) {
                if (q & 1) {
                    acc[2 * v] = fma_bf16h<1, 0>(acc[2 * v], xw[q >> 1], gq.w[q][v]);
                    acc[2 * v + 1] = fma_bf16h<1, 1>(acc[2 * v + 1], xw[q >> 1], gq.w[q][v]);
                } else {
                    acc[2 * v] = fma_bf16h<0, 0>(acc[2 * v], xw[q >> 1], gq.w[q][v]);
                    acc[2 * v + 1] = fma_bf16h<0, 1>(acc[2 * v + 1], xw[q >> 1], gq.w[q][v]);
                }
            }
        }
    };
    float *lg = reinterpret_cast<float *>(sm + L.lg_off);
    const float *lbias = (a.gate == 2) ? nullptr : a.bias;
    const bool counting = a.group_counts != nullptr;
    for (int gi = 0; ok && gi < my_groups; ++gi) {
        const int grp_id = g_first + gi * g_step;
        const int t0 = grp_id * a.tt;
#pragma unroll
        for (int i = 0; i < EPT; ++i) acc[i] = 0.0f;
        for (int cc = 0; cc < nchunk; ++cc) {
            const int c = gi * nchunk + cc;
            const int s = c % S;
            const uint32_t ph = (uint32_t)((c / S) & 1);
            ok = mbar_wait_bounded(xb_bar(s), ph, abort_flag, a.timeout_ns, a.status, 711) &&
                 mbar_wait_bounded(raw_bar(s), ph, abort_flag, a.timeout_ns, a.status, 712);
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
        ok = named_bar_and(bar_id, ncw * 32, ok);
        if (!ok) break;
        // top-k: SEG lanes per token (the experts' count rounded up to a power of two),
        // 32 / SEG tokens per warp at a time
        const int cw = warp - cw0;
        const int seg = a.E <= 8 ? 8 : a.E <= 16 ? 16 : 32;
        const int per = 32 / seg;
        const int sl = lane & (seg - 1);
        const int sub = lane / seg;
        for (int rr0 = cw * per; rr0 < a.tt; rr0 += ncw * per) {
            const int rr = rr0 + sub;
            const int t = t0 + rr;
            const bool has = rr < a.tt && t < a.T;
            topk_seg(lg + (has ? rr : 0) * EP, a.E, a.k, a.gate, a.bias,
                     a.topk_idx + (size_t)t * a.k, a.topk_w + (size_t)t * a.k, sl, seg, has,
                     counting ? cnt : nullptr);
        }
        if (counting || gi + 1 < my_groups) {
            // the group's top-k is complete (its counts and logits may be reused)
            named_bar_sync(bar_id, ncw * 32);
            if (counting && cid < a.E) {
                a.group_counts[(size_t)grp_id * a.E + cid] = cnt[cid];
                cnt[cid] = 0;
            }
        }
    }
    return ok;
}

template <int EPT, int G>
__global__ void __launch_bounds__(32 + RC_MAX_CONSUMERS, 1)
    route_chain_kernel(const __grid_constant__ CUtensorMap tmX,
                       const __grid_constant__ CUtensorMap tmW, const RcArgs a)
{
    extern __shared__ uint8_t rc_smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(rc_smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int ncw = (blockDim.x >> 5) - 1; // consumer warps
    if (a.status != nullptr && blockIdx.x == 0 && threadIdx.x == 0) {
        a.status[0] = DEV_OK; // a new call starts with a clean status word
        a.status[1] = 0;
    }
    if (threadIdx.x == 0) {
        rc_init(sm, rc_layout(a.tt, a.E, EPT * G, a.stages), a.stages, ncw);
        tma_prefetch_desc(&tmX);
        tma_prefetch_desc(&tmW);
    }
    __syncthreads();
    // one group of tt tokens per CTA
    rc_run<EPT, G>(&tmX, &tmW, a, sm, 0, 1, ncw, blockIdx.x, gridDim.x, gridDim.x, 1);
    __syncthreads();
}

} // namespace moe
