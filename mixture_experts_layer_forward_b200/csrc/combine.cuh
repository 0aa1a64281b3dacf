// combine.cuh -- top-k gather-reduce (Comet: Fine-grained Computation-communication
// Overlapping for Mixture-of-Experts, §2.1 "MoE Structure": gather and reduce the top-k
// expert outputs of each token).
//
//   out[t][n] = bf16_rne( sum_{j=0..k-1} ys[inv_pos[t][j]][n]  (+ ys_shared[t][n]) )
// The sum runs in fp32 with j ascending (the shared expert's row, when there is one, last),
// so the result does not depend on scheduling.
// Each thread owns 8 consecutive columns (one 16-byte vector) of one token; the grid
// strides over T * H/8 vectors. HBM-bound: k*T*H*2 bytes read, T*H*2 bytes written.
#pragma once

#include "ptx.cuh"

namespace moe {

// BATCH = top-k rows whose loads one thread issues together: on large grids 2 for k <= 3 and
// 4 for k >= 4 (more rows in flight per thread costs occupancy there: 8 was slower at both
// k = 2 and k = 8), 8 when the grid is smaller than the GPU and latency, not occupancy,
// sets the time.
template <int BATCH>
__global__ void __launch_bounds__(256)
    combine_kernel(const __nv_bfloat16 *__restrict__ ys, int64_t ys_rows,
                   const int32_t *__restrict__ inv_pos, int T, int H, int k,
                   __nv_bfloat16 *__restrict__ out, int *status, int clear_status,
                   const __nv_bfloat16 *__restrict__ ys_shared, const int *__restrict__ n_rows)
{
    if (clear_status && status != nullptr && blockIdx.x == 0 && threadIdx.x == 0) {
        status[0] = DEV_OK;
        status[1] = 0;
    }
    if (n_rows != nullptr) T = min(T, *n_rows); // output rows past *n_rows are left untouched
    const int vec_per_row = H / 8;
    const int64_t total = (int64_t)T * vec_per_row;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += stride) {
        const int t = (int)(i / vec_per_row);
        const int v = (int)(i - (int64_t)t * vec_per_row);
        float acc[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[q] = 0.0f;
        // up to BATCH rows per round: all their indices, then all their loads, are
        // issued before the first add, so a thread keeps several loads in flight; the adds
        // still run with j ascending
        for (int j0 = 0; j0 < k; j0 += BATCH) {
            int rr[BATCH];
#pragma unroll
            for (int q = 0; q < BATCH; ++q)
                rr[q] = (j0 + q < k) ? inv_pos[(size_t)t * k + j0 + q] : 0;
            uint4 uu[BATCH];
#pragma unroll
            for (int q = 0; q < BATCH; ++q) {
                const bool ok = (j0 + q < k) && rr[q] >= 0 && (int64_t)rr[q] < ys_rows;
                uu[q] = ok ? *reinterpret_cast<const uint4 *>(ys + (size_t)rr[q] * H + (size_t)v * 8)
                           : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int q = 0; q < BATCH; ++q) {
                if (j0 + q >= k) break;
                if (rr[q] < 0 || (int64_t)rr[q] >= ys_rows) {
                    record_status(status, DEV_BAD_INDEX, 3);
                    continue;
                }
                const uint4 u = uu[q];
                acc[0] += bf16_lo(u.x); acc[1] += bf16_hi(u.x);
                acc[2] += bf16_lo(u.y); acc[3] += bf16_hi(u.y);
                acc[4] += bf16_lo(u.z); acc[5] += bf16_hi(u.z);
                acc[6] += bf16_lo(u.w); acc[7] += bf16_hi(u.w);
            }
        }
        if (ys_shared != nullptr) {
            const uint4 u = *reinterpret_cast<const uint4 *>(ys_shared + (size_t)t * H + (size_t)v * 8);
            acc[0] += bf16_lo(u.x); acc[1] += bf16_hi(u.x);
            acc[2] += bf16_lo(u.y); acc[3] += bf16_hi(u.y);
            acc[4] += bf16_lo(u.z); acc[5] += bf16_hi(u.z);
            acc[6] += bf16_lo(u.w); acc[7] += bf16_hi(u.w);
        }
        uint4 o;
        o.x = pack_bf16x2(acc[0], acc[1]);
        o.y = pack_bf16x2(acc[2], acc[3]);
        o.z = pack_bf16x2(acc[4], acc[5]);
        o.w = pack_bf16x2(acc[6], acc[7]);
        *reinterpret_cast<uint4 *>(out + (size_t)t * H + (size_t)v * 8) = o;
    }
}

// Shared expert gate (Qwen2-MoE style): g[t] = 1 / (1 + exp(-x_t . w_sg)) in fp32, or 1
// without w_sg, for t < T; 0 for the pad rows T <= t < Tpad. One warp per token.
__global__ void __launch_bounds__(256)
    shared_gate_kernel(const __nv_bfloat16 *__restrict__ x, const __nv_bfloat16 *__restrict__ w_sg,
                       int T, int H, int Tpad, float *__restrict__ g)
{
    const int t = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (t >= Tpad) return;
    if (t >= T || w_sg == nullptr) {
        if (lane == 0) g[t] = t < T ? 1.0f : 0.0f;
        return;
    }
    const uint4 *xr = reinterpret_cast<const uint4 *>(x + (size_t)t * H);
    const uint4 *wr = reinterpret_cast<const uint4 *>(w_sg);
    float z = 0.0f;
    for (int v = lane; v < H / 8; v += 32) {
        const uint4 a = xr[v], b = wr[v];
        z = fmaf(bf16_lo(a.x), bf16_lo(b.x), z); z = fmaf(bf16_hi(a.x), bf16_hi(b.x), z);
        z = fmaf(bf16_lo(a.y), bf16_lo(b.y), z); z = fmaf(bf16_hi(a.y), bf16_hi(b.y), z);
        z = fmaf(bf16_lo(a.z), bf16_lo(b.z), z); z = fmaf(bf16_hi(a.z), bf16_hi(b.z), z);
        z = fmaf(bf16_lo(a.w), bf16_lo(b.w), z); z = fmaf(bf16_hi(a.w), bf16_hi(b.w), z);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
    if (lane == 0) g[t] = 1.0f / (1.0f + expf(-z));
}

} // namespace moe
