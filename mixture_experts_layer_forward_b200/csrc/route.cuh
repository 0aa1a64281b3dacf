// route.cuh -- router kernels (Comet: Fine-grained Computation-communication Overlapping for
// Mixture-of-Experts, §2.1 "MoE Structure": each token is routed to its selected experts).
//
// 1. route_logits_kernel: logits[t][e] = sum_h x[t][h] * Wg[h][e] (+ bias[e]) in fp32.
//    Each output is owned by one thread, which walks h upward with one accumulator, so the
//    result is bit-identical to a plain sequential fp32 loop. Each step is the mixed-precision
//    fused multiply-add of sm_100 on the bf16 operands as stored (a bf16 x bf16 product is
//    exact in fp32, so it rounds exactly like add-after-multiply on widened values). The tile
//    is staged through shared memory; h is consumed 8 values (one 16-byte load of each
//    operand) at a time, in order.
//    That order caps the parallelism at T*E independent chains, and each chain needs two
//    shared-memory operands per 8 steps unless a thread owns several tokens and experts; the
//    kernel is bound by shared-memory delivery and latency for small T*E and by FMA issue
//    for large E.
// 2. route_topk_kernel: one warp per token; k rounds of a warp argmax (ties to the lower
//    expert id), then the gate weights.
#pragma once

#include "ptx.cuh"

namespace moe {

__device__ __forceinline__ void cp_async_16(uint32_t dst, const void *src, bool valid)
{
    // src-size 0 zero-fills the 16 destination bytes (rows past T, columns past H or E)
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
                 "r"(valid ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N> __device__ __forceinline__ void cp_async_wait()
{
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

template <int BT, int BE, int HC, int NS> struct RouteSmem {
    static constexpr int LDB = HC + 8;                     // bf16 gate row (odd 16-byte count)
    static constexpr int XLD = HC * 2 + 16;                // ring row of x in bytes (likewise)
    static constexpr int X_RING = BT * XLD;                // bf16 x chunk [t][h]
    static constexpr int W_RING = HC * BE * 2;             // bf16 gate chunk [h][e]
    static constexpr int RING = NS * (X_RING + W_RING);
    static constexpr int WT = 2 * BE * LDB * 2;            // bf16 gate, [e][h], double buffered
    static constexpr int BYTES = RING + WT;
};

// acc + x * w for one bf16 half of each of two packed words (XH, WH: 0 = low half, 1 = high),
// rounded once to fp32. A bf16 product is exact in fp32, so this is bitwise
// fmaf(float(x), float(w), acc), without widening either operand first.
template <int XH, int WH>
__device__ __forceinline__ float fma_bf16h(float acc, uint32_t xw, uint32_t ww)
{
    float d;
    if constexpr (XH == 0 && WH == 0)
        asm("{.reg .b16 a0, a1, b0, b1;\n\tmov.b32 {a0, a1}, %1;\n\tmov.b32 {b0, b1}, %2;\n\t"
            "fma.rn.f32.bf16 %0, a0, b0, %3;}" : "=f"(d) : "r"(xw), "r"(ww), "f"(acc));
    else if constexpr (XH == 0 && WH == 1)
        asm("{.reg .b16 a0, a1, b0, b1;\n\tmov.b32 {a0, a1}, %1;\n\tmov.b32 {b0, b1}, %2;\n\t"
            "fma.rn.f32.bf16 %0, a0, b1, %3;}" : "=f"(d) : "r"(xw), "r"(ww), "f"(acc));
    else if constexpr (XH == 1 && WH == 0)
        asm("{.reg .b16 a0, a1, b0, b1;\n\tmov.b32 {a0, a1}, %1;\n\tmov.b32 {b0, b1}, %2;\n\t"
            "fma.rn.f32.bf16 %0, a1, b0, %3;}" : "=f"(d) : "r"(xw), "r"(ww), "f"(acc));
    else
        asm("{.reg .b16 a0, a1, b0, b1;\n\tmov.b32 {a0, a1}, %1;\n\tmov.b32 {b0, b1}, %2;\n\t"
            "fma.rn.f32.bf16 %0, a1, b1, %3;}" : "=f"(d) : "r"(xw), "r"(ww), "f"(acc));
    return d;
}

// Block = (BE/RE) x (BT/RT) threads. Thread (tx, ty) owns tokens ty + (BT/RT)*i and experts
// tx + (BE/RE)*j; the strided ownership keeps the 16-byte shared-memory reads free of bank
// conflicts. The h axis is streamed in chunks of HC through an NS-stage cp.async ring (bf16,
// exactly as stored; x rows padded to an odd count of 16-byte units). The threads read x
// straight from the ring; each thread transposes the gate pieces it copied itself (two h
// values of 8 experts) into a bf16 [expert][h] buffer, so one barrier per chunk suffices and
// NS-1 chunks are in flight while the current one is consumed. Every accumulator still walks
// h upward, one fused multiply-add per h. Against widening both operands to fp32 buffers
// first, this measured 53 -> 41 us on T=64, E=256, H=7168 and 491 -> 414 us on T=4096.
template <int BT, int BE, int RT, int RE, int HC, int NS>
__global__ void __launch_bounds__((BT / RT) * (BE / RE))
    route_logits_kernel(const __nv_bfloat16 *__restrict__ x, const __nv_bfloat16 *__restrict__ Wg,
                        const float *__restrict__ bias, float *__restrict__ logits, int T, int H,
                        int E, int *status)
{
    using S = RouteSmem<BT, BE, HC, NS>;
    constexpr int TX = BE / RE;
    constexpr int TY = BT / RT;
    constexpr int NT = TX * TY;
    constexpr int LDB = S::LDB;
    constexpr int XLD = S::XLD;
    constexpr int XV = BT * HC / 8; // 16-byte x pieces per chunk
    constexpr int XPT = (XV + NT - 1) / NT;
    constexpr int WP = HC * BE / 16; // pairs of 16-byte gate pieces (h even, h odd; 8 experts)
    constexpr int WPP = (WP + NT - 1) / NT;
    static_assert(BE % 8 == 0 && HC % 16 == 0, "tile shape");
    extern __shared__ __align__(16) uint8_t rsmem[];
    uint16_t *wt = reinterpret_cast<uint16_t *>(rsmem + S::RING); // [2][BE][LDB]

    if (status != nullptr && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0 &&
        threadIdx.y == 0) {
        status[0] = DEV_OK; // a new call starts with a clean status word
        status[1] = 0;
    }

    const int tid = threadIdx.y * TX + threadIdx.x;
    const int t0 = blockIdx.x * BT;
    const int e0 = blockIdx.y * BE;
    const int nchunk = (H + HC - 1) / HC;
    // rows of a vectorised gate copy must be whole 8-expert groups inside the row
    const bool wvec = (E % 8) == 0;

    auto ring_x = [&](int slot) { return rsmem + slot * (S::X_RING + S::W_RING); };
    auto ring_w = [&](int slot) { return rsmem + slot * (S::X_RING + S::W_RING) + S::X_RING; };

    auto issue = [&](int c) {
        const int slot = c % NS;
        const int h0 = c * HC;
        const uint32_t xs = smem_u32(ring_x(slot));
        const uint32_t wsr = smem_u32(ring_w(slot));
#pragma unroll
        for (int i = 0; i < XPT; ++i) {
            const int v = tid + i * NT;
            if (v < XV) {
                const int r = v / (HC / 8), q = v % (HC / 8);
                const int t = t0 + r, h = h0 + q * 8;
                const bool ok = (t < T) && (h < H);
                cp_async_16(xs + r * XLD + q * 16, ok ? (const void *)(x + (size_t)t * H + h) : (const void *)x, ok);
            }
        }
        if (wvec) {
            // piece (g, h) = experts e0 + 8g .. +7 of one h, at ring index g * HC + (h - h0);
            // one thread copies the pieces of h and h + 1 (it later transposes both)
#pragma unroll
            for (int i = 0; i < WPP; ++i) {
                const int pv = tid + i * NT;
                if (pv < WP) {
                    const int hh = 2 * (pv % (HC / 2)), g = pv / (HC / 2);
                    const int e = e0 + g * 8;
#pragma unroll
                    for (int o = 0; o < 2; ++o) {
                        const int h = h0 + hh + o;
                        const bool ok = (h < H) && (e < E);
                        cp_async_16(wsr + (g * HC + hh + o) * 16,
                                    ok ? (const void *)(Wg + (size_t)h * E + e) : (const void *)Wg, ok);
                    }
                }
            }
        }
        cp_async_commit();
    };
    // transpose the gate pieces this thread copied for chunk c into the bf16 [e][h] buffer of
    // parity c&1 (x is read from the ring as it landed)
    auto transpose = [&](int c) {
        const int slot = c % NS;
        const int h0 = c * HC;
        uint16_t *wd = wt + (c & 1) * BE * LDB;
        if (wvec) {
            const uint4 *wsrc = reinterpret_cast<const uint4 *>(ring_w(slot));
#pragma unroll
            for (int i = 0; i < WPP; ++i) {
                const int pv = tid + i * NT;
                if (pv < WP) {
                    const int hh = 2 * (pv % (HC / 2)), g = pv / (HC / 2);
                    const uint4 u0 = wsrc[g * HC + hh], u1 = wsrc[g * HC + hh + 1];
                    const uint32_t a0[4] = {u0.x, u0.y, u0.z, u0.w};
                    const uint32_t a1[4] = {u1.x, u1.y, u1.z, u1.w};
                    // word of expert e: (h, h + 1) in its (low, high) half
                    uint32_t *d = reinterpret_cast<uint32_t *>(wd + (g * 8) * LDB + hh);
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        d[(2 * m) * (LDB / 2)] = __byte_perm(a0[m], a1[m], 0x5410);
                        d[(2 * m + 1) * (LDB / 2)] = __byte_perm(a0[m], a1[m], 0x7632);
                    }
                }
            }
        } else {
            // expert counts that are not a multiple of 8: plain loads (small problems only)
            const uint16_t *wraw = reinterpret_cast<const uint16_t *>(Wg);
            for (int v = tid; v < HC * BE; v += NT) {
                const int hh = v / BE, ee = v % BE;
                const int h = h0 + hh, e = e0 + ee;
                wd[ee * LDB + hh] = (h < H && e < E) ? wraw[(size_t)h * E + e] : (uint16_t)0;
            }
        }
    };

    float acc[RT][RE];
#pragma unroll
    for (int i = 0; i < RT; ++i)
#pragma unroll
        for (int j = 0; j < RE; ++j) acc[i][j] = 0.0f;

    // prologue: NS-1 chunks in flight, chunk 0 transposed
#pragma unroll
    for (int c = 0; c < NS - 1; ++c) {
        if (c < nchunk) issue(c);
        else cp_async_commit();
    }
    cp_async_wait<NS - 2>();
    transpose(0);

    for (int c = 0; c < nchunk; ++c) {
        __syncthreads(); // chunk c landed and transposed by everyone; chunk c-1's buffers are free
        if (c + NS - 1 < nchunk) issue(c + NS - 1);
        else cp_async_commit(); // keep one group per iteration
        // the last chunk may run past H: its x and gate values are zero there, and an exact
        // zero product leaves each accumulator's value unchanged.
        // Operands of the next 8 h values are loaded into registers before the FMAs of the
        // current ones, so the dependent FMA chains never wait on a shared-memory load.
        const uint8_t *xc = ring_x(c % NS) + threadIdx.y * XLD;
        const uint16_t *wc = wt + (c & 1) * BE * LDB + threadIdx.x * LDB;
        uint4 xa[RT], wa[RE], xb[RT], wb[RE];
        auto ld = [&](uint4 (&xv)[RT], uint4 (&wv)[RE], int hh) {
#pragma unroll
            for (int i = 0; i < RT; ++i)
                xv[i] = *reinterpret_cast<const uint4 *>(xc + TY * i * XLD + hh * 2);
#pragma unroll
            for (int j = 0; j < RE; ++j)
                wv[j] = *reinterpret_cast<const uint4 *>(wc + TX * j * LDB + hh);
        };
        // h ascending: the low half of each word is the lower h
        auto fma8 = [&](const uint4 (&xv)[RT], const uint4 (&wv)[RE]) {
#pragma unroll
            for (int i = 0; i < RT; ++i)
#pragma unroll
                for (int j = 0; j < RE; ++j) {
                    const uint32_t xw[4] = {xv[i].x, xv[i].y, xv[i].z, xv[i].w};
                    const uint32_t ww[4] = {wv[j].x, wv[j].y, wv[j].z, wv[j].w};
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        acc[i][j] = fma_bf16h<0, 0>(acc[i][j], xw[m], ww[m]);
                        acc[i][j] = fma_bf16h<1, 1>(acc[i][j], xw[m], ww[m]);
                    }
                }
        };
        ld(xa, wa, 0);
#pragma unroll
        for (int hh = 0; hh < HC; hh += 16) {
            ld(xb, wb, hh + 8);
            fma8(xa, wa);
            if (hh + 16 < HC) ld(xa, wa, hh + 16);
            fma8(xb, wb);
        }
        if (c + 1 < nchunk) {
            cp_async_wait<NS - 2>(); // this thread's copies of chunk c+1 have landed
            transpose(c + 1);
        }
    }
    cp_async_wait<0>();
#pragma unroll
    for (int i = 0; i < RT; ++i) {
        const int t = t0 + threadIdx.y + TY * i;
        if (t >= T) continue;
#pragma unroll
        for (int j = 0; j < RE; ++j) {
            const int e = e0 + threadIdx.x + TX * j;
            if (e >= E) continue;
            float v = acc[i][j];
            if (bias != nullptr) v = v + bias[e];
            logits[(size_t)t * E + e] = v;
        }
    }
}

// Tile shapes per expert-count class: BT, BE, RT, RE, HC, NS.
// Measured on B200 (router alone, before the mixed-precision steps): E=8, T=8192, H=4096:
// 75 us; E=16, T=16384: 162 us; E=64, T=8192, H=3584: 169 us; E=256, T=4096, H=7168: 518 us
// (491 us with the filter off since; 414 us with the mixed-precision steps).
#ifndef ROUTE_SMALL_CFG
#define ROUTE_SMALL_CFG 64, 8, 2, 2, 64, 4    // E <= 8
#endif
#ifndef ROUTE_MID_CFG
#define ROUTE_MID_CFG 32, 16, 2, 2, 64, 4     // 8 < E <= 16
#endif
#ifndef ROUTE_LARGE_CFG
#define ROUTE_LARGE_CFG 64, 64, 4, 4, 32, 4   // E > 16
#endif
// Small batches (decode): one output per thread, so that T*E outputs still spread over
// every SM: 8 x 16 tiles while they make at most one block per SM (T=64, E=256: 128 blocks;
// with fp32-widened operands 53 us against 86 us with 16 x 16 tiles and 64-value chunks, and
// against 65-115 us for six other token x expert shapes; 41 us with the mixed-precision
// steps), else 16 x 16 tiles (T=128, E=256: 72 us widened); long chunks halve the per-chunk
// barriers and transposes.
#ifndef ROUTE_NARROW_CFG
#define ROUTE_NARROW_CFG 8, 16, 1, 1, 128, 4
#endif
#ifndef ROUTE_NARROW2_CFG
#define ROUTE_NARROW2_CFG 16, 16, 1, 1, 256, 4
#endif

constexpr int TOPK_WARPS = 8; // tokens per block

// One warp selects the k largest keys of one token's E logits and writes the token's expert
// ids and gate weights. `lg` holds the logits (without the bias in gate mode 2), `row` is a
// scratch row of E floats in shared memory owned by this warp.
// Keys: the logits, or in gate mode 2 (selection bias) logits[e] + bias[e] (the same fp32
// addition the logits kernels make in the other modes); the gates use the logits without the
// bias, shifted by their maximum. k rounds of a warp argmax, ties to the lower expert id.
__device__ __forceinline__ void topk_row_warp(const float *lg, float *row, int E, int k, int gate,
                                              const float *__restrict__ bias,
                                              int32_t *__restrict__ idx_out,
                                              float *__restrict__ w_out, int lane)
{
    const bool sel_bias = (gate == 2) && bias != nullptr;
    for (int e = lane; e < E; e += 32) row[e] = sel_bias ? lg[e] + bias[e] : lg[e];
    __syncwarp();

    float sel_val = 0.0f; // lane j keeps the j-th selected logit (j < k <= 32 covered below)
    float top = 0.0f;
    for (int j = 0; j < k; ++j) {
        float bv = -INFINITY;
        int bi = 0x7fffffff;
        for (int e = lane; e < E; e += 32) {
            const float v = row[e];
            if (v > bv) { bv = v; bi = e; } // e ascending within a lane: strict > keeps the lower id
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
            if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
        }
        // every lane now holds the winner (bv, bi); a non-finite row (unsupported input)
        // must still not index outside the row
        if (bi < 0 || bi >= E) bi = 0;
        const float gv = (gate == 2) ? lg[bi] : bv; // the gate's logit (no bias in mode 2)
        if (j == 0) top = gv;
        if (lane == 0) {
            idx_out[j] = bi;
            row[bi] = -INFINITY; // removed from later rounds (logits are finite)
        }
        if (j < 32 && j == lane) sel_val = gv;
        if (j >= 32 && lane == 0) w_out[j] = gv; // stash; rescaled below
        __syncwarp();
    }
    if (gate == 2) { // the largest selected logit (the first selected one need not be)
        float m = -INFINITY;
        for (int j = lane; j < k; j += 32) m = fmaxf(m, (j < 32) ? sel_val : w_out[j]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
        top = m;
    }

    // gate weights: w_j = exp(l_j - l_0) / denom
    float denom = 0.0f;
    if (gate == 1) { // SOFTMAX_ALL: sum over every expert's logit
        for (int e = lane; e < E; e += 32) denom += expf(lg[e] - top);
    } else {
        for (int j = lane; j < k; j += 32) {
            const float v = (j < 32) ? sel_val : w_out[j];
            denom += expf(v - top);
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) denom += __shfl_xor_sync(0xffffffffu, denom, off);
    __syncwarp();
    for (int j = lane; j < k; j += 32) {
        const float v = (j < 32) ? sel_val : w_out[j];
        w_out[j] = expf(v - top) / denom;
    }
}

// One warp per token. Dynamic shared memory: TOPK_WARPS * E floats.
__global__ void __launch_bounds__(TOPK_WARPS * 32)
    route_topk_kernel(const float *__restrict__ logits, int32_t *__restrict__ topk_idx,
                      float *__restrict__ topk_w, int T, int E, int k, int gate,
                      const float *__restrict__ bias)
{
    extern __shared__ float srow[];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * TOPK_WARPS + warp;
    if (t >= T) return;
    topk_row_warp(logits + (size_t)t * E, srow + (size_t)warp * E, E, k, gate, bias,
                  topk_idx + (size_t)t * k, topk_w + (size_t)t * k, lane);
}

} // namespace moe
