// backward.cuh -- the row-wise and router parts of the layer's backward pass (training; a
// next-work item beyond the pages, which describe the forward). The GEMMs of the backward
// run in gemm_tc.cuh (BMODE_KMAJOR, BMODE_WGRAD).
//
// With the selection fixed and w the gates (softmax over the selected logits), for a padded
// expert row r = (token t, selection j) of expert e:
//   z_r   = x_t W1[e]                     (recomputed: gu, bf16)
//   u_r   = dy_t W2[e]^T                  (the gradient at the hidden activation, before w)
//   a_r   = silu(g) * up  (or act(z))     (the hidden activation)
//   dw_r  = a_r . u_r                     (= dy_t . y_e(x_t), the gate's gradient)
//   dz_r  = w_r u_r * [up silu'(g), silu(g)]   (or w_r u_r act'(z))
//   gy_r  = w_r dy_t                      (the gradient at the expert output)
// then dl (the logits' gradient) per token from the dw of its k rows, dx_t from the k rows'
// dz W1^T plus the router term, dW_g and the bias gradient per expert over its rows.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "dispatch.cuh"

namespace moe {

constexpr int BWD_THREADS = 256;

__device__ __forceinline__ float bwd_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bwd_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
__device__ __forceinline__ uint32_t bwd_pack(float a, float b)
{
    const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t *>(&v);
}

__device__ __forceinline__ float bwd_act(int act, float z)
{
    if (act == 1) {
        const float c = 0.7978845608028654f;
        return 0.5f * z * (1.0f + tanhf(c * (z + 0.044715f * z * z * z)));
    }
    if (act == 2) return z > 0.0f ? z : 0.0f;
    return z;
}

__device__ __forceinline__ float bwd_act_grad(int act, float z)
{
    if (act == 1) {
        const float c = 0.7978845608028654f;
        const float th = tanhf(c * (z + 0.044715f * z * z * z));
        return 0.5f * (1.0f + th) + 0.5f * z * (1.0f - th * th) * c * (1.0f + 3.0f * 0.044715f * z * z);
    }
    if (act == 2) return z > 0.0f ? 1.0f : 0.0f;
    return 1.0f;
}

// One block per live padded row (grid-stride over num_tiles * m_tile rows). gu [P, w1c] is
// overwritten in place by dz; writes a [P, F], gy [P, H], dw_row [P]. F, H % 8 == 0.
__global__ void __launch_bounds__(BWD_THREADS)
    bwd_rows_kernel(__nv_bfloat16 *gu_dz, const __nv_bfloat16 *__restrict__ u,
                    const __nv_bfloat16 *__restrict__ dy, const int32_t *__restrict__ gather_idx,
                    const float *__restrict__ row_w, const DispatchMeta *meta, int m_tile, int F,
                    int H, int T, int act, __nv_bfloat16 *__restrict__ a_out,
                    __nv_bfloat16 *__restrict__ gy, float *__restrict__ dw_row)
{
    __shared__ float red[BWD_THREADS / 32];
    const int64_t rows = (int64_t)meta->num_tiles * m_tile;
    const bool gated = (act == 0);
    const int w1c = gated ? 2 * F : F;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
        const int t = gather_idx[r];
        const float w = (t >= 0 && t < T) ? row_w[r] : 0.0f;
        uint4 *zr = reinterpret_cast<uint4 *>(gu_dz + r * w1c);
        const uint4 *ur = reinterpret_cast<const uint4 *>(u + r * F);
        uint4 *ar = reinterpret_cast<uint4 *>(a_out + r * F);
        float dw = 0.0f;
        for (int i = threadIdx.x; i < F / 8; i += BWD_THREADS) {
            const uint4 uv = ur[i];
            const uint4 gv = zr[i];
            const uint32_t uw[4] = {uv.x, uv.y, uv.z, uv.w};
            const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
            uint32_t aw[4], dgw[4], duw[4];
            if (gated) {
                const uint4 pv = zr[F / 8 + i]; // the up half
                const uint32_t pw[4] = {pv.x, pv.y, pv.z, pv.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    float av[2], dg[2], du[2];
                    const float gg[2] = {bwd_lo(gw[j]), bwd_hi(gw[j])};
                    const float pp[2] = {bwd_lo(pw[j]), bwd_hi(pw[j])};
                    const float uu[2] = {bwd_lo(uw[j]), bwd_hi(uw[j])};
#pragma unroll
                    for (int h2 = 0; h2 < 2; ++h2) {
                        const float s = 1.0f / (1.0f + expf(-gg[h2]));
                        const float silu = gg[h2] * s;
                        av[h2] = silu * pp[h2];
                        dw = fmaf(av[h2], uu[h2], dw);
                        const float da = w * uu[h2];
                        dg[h2] = da * pp[h2] * s * (1.0f + gg[h2] * (1.0f - s));
                        du[h2] = da * silu;
                    }
                    aw[j] = bwd_pack(av[0], av[1]);
                    dgw[j] = bwd_pack(dg[0], dg[1]);
                    duw[j] = bwd_pack(du[0], du[1]);
                }
                zr[i] = make_uint4(dgw[0], dgw[1], dgw[2], dgw[3]);
                zr[F / 8 + i] = make_uint4(duw[0], duw[1], duw[2], duw[3]);
            } else {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float zz[2] = {bwd_lo(gw[j]), bwd_hi(gw[j])};
                    const float uu[2] = {bwd_lo(uw[j]), bwd_hi(uw[j])};
                    float av[2], dz[2];
#pragma unroll
                    for (int h2 = 0; h2 < 2; ++h2) {
                        av[h2] = bwd_act(act, zz[h2]);
                        dw = fmaf(av[h2], uu[h2], dw);
                        dz[h2] = w * uu[h2] * bwd_act_grad(act, zz[h2]);
                    }
                    aw[j] = bwd_pack(av[0], av[1]);
                    dgw[j] = bwd_pack(dz[0], dz[1]);
                }
                zr[i] = make_uint4(dgw[0], dgw[1], dgw[2], dgw[3]);
            }
            ar[i] = make_uint4(aw[0], aw[1], aw[2], aw[3]);
        }
        // gy = w * dy[t] (0 for pad rows)
        const uint4 *dyr = reinterpret_cast<const uint4 *>(dy + (size_t)(t >= 0 && t < T ? t : 0) * H);
        uint4 *gyr = reinterpret_cast<uint4 *>(gy + r * H);
        for (int i = threadIdx.x; i < H / 8; i += BWD_THREADS) {
            const uint4 v = dyr[i];
            const uint32_t vw[4] = {v.x, v.y, v.z, v.w};
            uint32_t o[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) o[j] = bwd_pack(w * bwd_lo(vw[j]), w * bwd_hi(vw[j]));
            gyr[i] = make_uint4(o[0], o[1], o[2], o[3]);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) dw += __shfl_xor_sync(0xffffffffu, dw, off);
        if (lane == 0) red[warp] = dw;
        __syncthreads();
        if (threadIdx.x == 0) {
            float s = 0.0f;
            for (int i = 0; i < BWD_THREADS / 32; ++i) s += red[i];
            dw_row[r] = (t >= 0 && t < T) ? s : 0.0f;
        }
        __syncthreads();
    }
}

// Logit gradients, one warp per token: dl_j = w_j (dw_j - sum_i w_i dw_i), written per row.
__global__ void bwd_router_kernel(const float *__restrict__ topk_w, const int32_t *__restrict__ inv_pos,
                                  const float *__restrict__ dw_row, int T, int k,
                                  float *__restrict__ dl_row)
{
    const int t = (int)(((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5);
    const int lane = threadIdx.x & 31;
    if (t >= T) return;
    float s = 0.0f;
    for (int j = lane; j < k; j += 32) s += topk_w[(size_t)t * k + j] * dw_row[inv_pos[(size_t)t * k + j]];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    for (int j = lane; j < k; j += 32) {
        const int r = inv_pos[(size_t)t * k + j];
        dl_row[r] = topk_w[(size_t)t * k + j] * (dw_row[r] - s);
    }
}

// dx[t] = sum_j dx_perm[inv_pos[t][j]] + sum_j dl_j W_g[:, e_j], fp32 sum, one bf16 rounding.
// One block per token (grid-stride), eight h per thread.
__global__ void __launch_bounds__(BWD_THREADS)
    bwd_dx_kernel(const __nv_bfloat16 *__restrict__ dx_perm, const int32_t *__restrict__ inv_pos,
                  const int32_t *__restrict__ topk_idx, const float *__restrict__ dl_row,
                  const __nv_bfloat16 *__restrict__ Wg, int T, int H, int E, int k,
                  __nv_bfloat16 *__restrict__ dx)
{
    for (int t = blockIdx.x; t < T; t += gridDim.x) {
        for (int i = threadIdx.x; i < H / 8; i += BWD_THREADS) {
            float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
            for (int j = 0; j < k; ++j) {
                const int r = inv_pos[(size_t)t * k + j];
                const int e = topk_idx[(size_t)t * k + j];
                const uint4 v = reinterpret_cast<const uint4 *>(dx_perm + (size_t)r * H)[i];
                const uint32_t vw[4] = {v.x, v.y, v.z, v.w};
                const float dl = dl_row[r];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    acc[2 * q] += bwd_lo(vw[q]);
                    acc[2 * q + 1] += bwd_hi(vw[q]);
                }
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    acc[q] = fmaf(dl, __bfloat162float(Wg[(size_t)(i * 8 + q) * E + e]), acc[q]);
            }
            uint32_t o[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) o[q] = bwd_pack(acc[2 * q], acc[2 * q + 1]);
            reinterpret_cast<uint4 *>(dx + (size_t)t * H)[i] = make_uint4(o[0], o[1], o[2], o[3]);
        }
    }
}

// dW_g[h][e] = sum over expert e's routed rows r of x[t_r][h] dl_r, and dbias[e] = sum dl_r
// (with_bias == 0: the bias does not reach the gates, dbias = 0). Rows of expert e are
// poff[e] .. poff[e] + counts[e] - 1 (routed rows first in each padded block), summed in
// that order. Grid (E, ceil(H / BWD_THREADS)).
__global__ void __launch_bounds__(BWD_THREADS)
    bwd_router_weights_kernel(const __nv_bfloat16 *__restrict__ x, const int32_t *__restrict__ gather_idx,
                              const int32_t *__restrict__ poff, const int32_t *__restrict__ counts,
                              const float *__restrict__ dl_row, int H, int E, int with_bias,
                              float *__restrict__ dWg, float *__restrict__ dbias)
{
    const int e = blockIdx.x;
    const int h = blockIdx.y * BWD_THREADS + threadIdx.x;
    const int r0 = poff[e], n = counts[e];
    if (h < H) {
        float s = 0.0f;
        for (int i = 0; i < n; ++i) {
            const int t = gather_idx[r0 + i];
            s = fmaf(__bfloat162float(x[(size_t)t * H + h]), dl_row[r0 + i], s);
        }
        dWg[(size_t)h * E + e] = s;
    }
    if (blockIdx.y == 0 && threadIdx.x == 0) {
        float s = 0.0f;
        if (with_bias)
            for (int i = 0; i < n; ++i) s += dl_row[r0 + i];
        dbias[e] = s;
    }
}

// Zero the per-expert slabs (slab_vec 16-byte vectors each) of the experts without routed
// rows; the weight-gradient GEMMs write the others. Grid (chunks, E).
__global__ void zero_inactive_slabs_kernel(uint4 *__restrict__ dst, int64_t slab_vec,
                                           const int32_t *__restrict__ counts)
{
    const int e = blockIdx.y;
    if (counts[e] > 0) return;
    uint4 *slab = dst + (size_t)e * slab_vec;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < slab_vec;
         i += (int64_t)gridDim.x * blockDim.x)
        slab[i] = make_uint4(0u, 0u, 0u, 0u);
}

} // namespace moe
