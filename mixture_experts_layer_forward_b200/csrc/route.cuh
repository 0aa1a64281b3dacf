// route.cuh -- router kernels (Comet: Fine-grained Computation-communication Overlapping for
// Mixture-of-Experts, §2.1 "MoE Structure": each token is routed to its selected experts).
//
// 1. route_logits_kernel: logits[t][e] = sum_h x[t][h] * Wg[h][e] (+ bias[e]) in fp32.
//    Each output is owned by one thread, which walks h upward with one accumulator, so the
//    result is bit-identical to a plain sequential fp32 loop (a bf16 x bf16 product is exact
//    in fp32, so the fused multiply-add rounds exactly like add-after-multiply). The tile
//    is staged through shared memory; h is consumed in float4 steps, in order.
// 2. route_topk_kernel: one warp per token; k rounds of a warp argmax (ties to the lower
//    expert id), then the gate weights.
#pragma once

#include "ptx.cuh"

namespace moe {

constexpr int ROUTE_HC = 32; // h values staged per shared-memory step

// Block = (BE/RE) x (BT/RT) threads; thread (tx, ty) owns tokens ty*RT.. and experts tx*RE..
template <int BT, int BE, int RT, int RE>
__global__ void __launch_bounds__((BT / RT) * (BE / RE))
    route_logits_kernel(const __nv_bfloat16 *__restrict__ x, const __nv_bfloat16 *__restrict__ Wg,
                        const float *__restrict__ bias, float *__restrict__ logits, int T, int H,
                        int E, int *status)
{
    constexpr int TX = BE / RE;
    constexpr int TY = BT / RT;
    constexpr int NT = TX * TY;
    constexpr int LD = ROUTE_HC + 4; // row stride in floats (keeps float4 alignment)
    __shared__ __align__(16) float xs[BT][LD];
    __shared__ __align__(16) float ws[BE][LD];

    if (status != nullptr && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0 &&
        threadIdx.y == 0) {
        status[0] = DEV_OK; // a new call starts with a clean status word
        status[1] = 0;
    }

    const int tid = threadIdx.y * TX + threadIdx.x;
    const int t0 = blockIdx.x * BT;
    const int e0 = blockIdx.y * BE;

    float acc[RT][RE];
#pragma unroll
    for (int i = 0; i < RT; ++i)
#pragma unroll
        for (int j = 0; j < RE; ++j) acc[i][j] = 0.0f;

    for (int h0 = 0; h0 < H; h0 += ROUTE_HC) {
        // x tile: BT rows x 32 bf16, 16-byte chunks
        for (int c = tid; c < BT * (ROUTE_HC / 8); c += NT) {
            const int r = c / (ROUTE_HC / 8);
            const int q = c % (ROUTE_HC / 8);
            const int t = t0 + r;
            float v[8];
            if (t < T) {
                const uint4 u = *reinterpret_cast<const uint4 *>(x + (size_t)t * H + h0 + q * 8);
                v[0] = bf16_lo(u.x); v[1] = bf16_hi(u.x);
                v[2] = bf16_lo(u.y); v[3] = bf16_hi(u.y);
                v[4] = bf16_lo(u.z); v[5] = bf16_hi(u.z);
                v[6] = bf16_lo(u.w); v[7] = bf16_hi(u.w);
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) v[i] = 0.0f;
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) xs[r][q * 8 + i] = v[i];
        }
        // gate tile, transposed to [expert][h]
        for (int c = tid; c < BE * ROUTE_HC; c += NT) {
            const int hh = c / BE;
            const int ee = c % BE;
            const int e = e0 + ee;
            ws[ee][hh] = (e < E) ? __bfloat162float(Wg[(size_t)(h0 + hh) * E + e]) : 0.0f;
        }
        __syncthreads();
#pragma unroll 2
        for (int hh = 0; hh < ROUTE_HC; hh += 4) {
            float4 xv[RT], wv[RE];
#pragma unroll
            for (int i = 0; i < RT; ++i)
                xv[i] = *reinterpret_cast<const float4 *>(&xs[threadIdx.y * RT + i][hh]);
#pragma unroll
            for (int j = 0; j < RE; ++j)
                wv[j] = *reinterpret_cast<const float4 *>(&ws[threadIdx.x * RE + j][hh]);
#pragma unroll
            for (int i = 0; i < RT; ++i)
#pragma unroll
                for (int j = 0; j < RE; ++j) {
                    acc[i][j] = fmaf(xv[i].x, wv[j].x, acc[i][j]);
                    acc[i][j] = fmaf(xv[i].y, wv[j].y, acc[i][j]);
                    acc[i][j] = fmaf(xv[i].z, wv[j].z, acc[i][j]);
                    acc[i][j] = fmaf(xv[i].w, wv[j].w, acc[i][j]);
                }
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < RT; ++i) {
        const int t = t0 + threadIdx.y * RT + i;
        if (t >= T) continue;
#pragma unroll
        for (int j = 0; j < RE; ++j) {
            const int e = e0 + threadIdx.x * RE + j;
            if (e >= E) continue;
            float v = acc[i][j];
            if (bias != nullptr) v = v + bias[e];
            logits[(size_t)t * E + e] = v;
        }
    }
}

constexpr int TOPK_WARPS = 8; // tokens per block

// One warp per token. Dynamic shared memory: TOPK_WARPS * E floats.
__global__ void __launch_bounds__(TOPK_WARPS * 32)
    route_topk_kernel(const float *__restrict__ logits, int32_t *__restrict__ topk_idx,
                      float *__restrict__ topk_w, int T, int E, int k, int gate)
{
    extern __shared__ float srow[];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * TOPK_WARPS + warp;
    if (t >= T) return;
    float *row = srow + (size_t)warp * E;
    const float *lg = logits + (size_t)t * E;
    for (int e = lane; e < E; e += 32) row[e] = lg[e];
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
        if (j == 0) top = bv;
        if (lane == 0) {
            topk_idx[(size_t)t * k + j] = bi;
            row[bi] = -INFINITY; // removed from later rounds (logits are finite)
        }
        if (j < 32 && j == lane) sel_val = bv;
        if (j >= 32 && lane == 0) topk_w[(size_t)t * k + j] = bv; // stash; rescaled below
        __syncwarp();
    }

    // gate weights: w_j = exp(l_j - l_0) / denom
    float denom = 0.0f;
    if (gate == 1) { // SOFTMAX_ALL: sum over every expert's logit
        for (int e = lane; e < E; e += 32) denom += expf(lg[e] - top);
    } else {
        for (int j = lane; j < k; j += 32) {
            const float v = (j < 32) ? sel_val : topk_w[(size_t)t * k + j];
            denom += expf(v - top);
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) denom += __shfl_xor_sync(0xffffffffu, denom, off);
    __syncwarp();
    for (int j = lane; j < k; j += 32) {
        const float v = (j < 32) ? sel_val : topk_w[(size_t)t * k + j];
        topk_w[(size_t)t * k + j] = expf(v - top) / denom;
    }
}

} // namespace moe
