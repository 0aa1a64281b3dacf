// fp8.cuh -- e4m3 quantisation for the FP8 expert path (a precision variant; the pages fix
// no precision).
//
// Format: e4m3 of the OCP 8-bit floating-point formats (1 sign, 4 exponent bits with bias 7,
// 3 mantissa bits, largest finite magnitude 448). Scaling, for one vector (a token row of x
// or h, or an output column of W1 or W2 over its K values):
//   r = 448 / amax, s = amax / 448 (both rounded to fp32; r = s = 1 when r is not finite),
//   code = e4m3(v * r), the product rounded to fp32, the conversion to the nearest e4m3
//   value with ties to even and saturation at 448 (cvt.rn.satfinite);
//   v ~ decode(code) * s.
// Weights are stored transposed, K contiguous ([E, N rows, K]), so both MMA operands are
// K-major and a 128-value k-block is one 128-byte row segment, as for 64 bf16 values.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "dispatch.cuh"

namespace moe {

constexpr int Q_THREADS = 256;

__device__ __forceinline__ void fp8_scales(float amax, float &r, float &s)
{
    r = __fdiv_rn(448.0f, amax);
    s = __fdiv_rn(amax, 448.0f);
    if (!isfinite(r)) {
        r = 1.0f;
        s = 1.0f;
    }
}

// e4m3 codes of a and b (nearest, ties to even, saturating); a in the low byte
__device__ __forceinline__ uint32_t e4m3x2(float a, float b)
{
    return (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
}

__device__ __forceinline__ float bf16_lo_f(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi_f(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Row quantisation of src [rows, cols] bf16 (cols % 8 == 0) into dst [rows, cols] codes and
// scale [rows]. One block per row, grid-stride over the rows. With meta != nullptr only the
// first meta->num_tiles * m_tile rows are live (the padded expert rows of h).
__global__ void __launch_bounds__(Q_THREADS)
    quant_rows_fp8_kernel(const __nv_bfloat16 *__restrict__ src, int64_t rows, int cols,
                          const DispatchMeta *meta, int m_tile, uint8_t *__restrict__ dst,
                          float *__restrict__ scale)
{
    __shared__ float red[Q_THREADS / 32];
    __shared__ float row_r;
    int64_t nrows = rows;
    if (meta != nullptr) {
        const int64_t live = (int64_t)meta->num_tiles * m_tile;
        if (live < nrows) nrows = live;
    }
    const int nvec = cols / 8;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int64_t row = blockIdx.x; row < nrows; row += gridDim.x) {
        const uint4 *sv = reinterpret_cast<const uint4 *>(src + row * cols);
        float amax = 0.0f;
        for (int i = threadIdx.x; i < nvec; i += Q_THREADS) {
            const uint4 u = sv[i];
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int j = 0; j < 4; ++j)
                amax = fmaxf(amax, fmaxf(fabsf(bf16_lo_f(w[j])), fabsf(bf16_hi_f(w[j]))));
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
        if (lane == 0) red[warp] = amax;
        __syncthreads();
        if (threadIdx.x == 0) {
            float m = red[0];
            for (int i = 1; i < Q_THREADS / 32; ++i) m = fmaxf(m, red[i]);
            float r, s;
            fp8_scales(m, r, s);
            row_r = r;
            scale[row] = s;
        }
        __syncthreads();
        const float r = row_r;
        uint2 *dv = reinterpret_cast<uint2 *>(dst + row * cols);
        for (int i = threadIdx.x; i < nvec; i += Q_THREADS) {
            const uint4 u = sv[i];
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
            uint32_t c[4];
#pragma unroll
            for (int j = 0; j < 4; ++j)
                c[j] = e4m3x2(__fmul_rn(bf16_lo_f(w[j]), r), __fmul_rn(bf16_hi_f(w[j]), r));
            dv[i] = make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
        }
        __syncthreads(); // red and row_r are reused by the next row
    }
}

// Column maxima of expert weights W [E, K, N] bf16 -> amax [E, N]. Grid (ceil(N/128), E);
// thread c of each half-block walks column n0 + c over every other K row.
__global__ void __launch_bounds__(256)
    quant_cols_amax_kernel(const __nv_bfloat16 *__restrict__ W, int K, int N, float *__restrict__ amax)
{
    __shared__ float part[128];
    const int e = blockIdx.y, c = threadIdx.x & 127, half = threadIdx.x >> 7;
    const int n = blockIdx.x * 128 + c;
    float m = 0.0f;
    if (n < N) {
        const __nv_bfloat16 *col = W + (size_t)e * K * N + n;
        for (int k = half; k < K; k += 2) m = fmaxf(m, fabsf(__bfloat162float(col[(size_t)k * N])));
    }
    if (half == 1) part[c] = m;
    __syncthreads();
    if (half == 0 && n < N) amax[(size_t)e * N + n] = fmaxf(m, part[c]);
}

// Codes of W [E, K, N] (K % 64 == 0, N % 64 == 0) written transposed into Wq [E, N, K], using
// the column maxima in amax [E, N]. Grid (N/64, K/64, E): one 64 x 64 tile through shared
// memory per block.
__global__ void __launch_bounds__(256)
    quant_cols_codes_kernel(const __nv_bfloat16 *__restrict__ W, int K, int N,
                            const float *__restrict__ amax, uint8_t *__restrict__ Wq)
{
    __shared__ float tile[64][65];
    __shared__ float col_r[64];
    const int n0 = blockIdx.x * 64, k0 = blockIdx.y * 64, e = blockIdx.z;
    const __nv_bfloat16 *We = W + (size_t)e * K * N;
    for (int i = threadIdx.x; i < 64 * 8; i += 256) {
        const int k = i >> 3, nv = i & 7;
        const uint4 u = *reinterpret_cast<const uint4 *>(We + (size_t)(k0 + k) * N + n0 + nv * 8);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            tile[k][nv * 8 + 2 * j] = bf16_lo_f(w[j]);
            tile[k][nv * 8 + 2 * j + 1] = bf16_hi_f(w[j]);
        }
    }
    if (threadIdx.x < 64) {
        float r, s;
        fp8_scales(amax[(size_t)e * N + n0 + threadIdx.x], r, s);
        col_r[threadIdx.x] = r;
    }
    __syncthreads();
    uint8_t *Wqe = Wq + (size_t)e * N * K;
    for (int i = threadIdx.x; i < 64 * 8; i += 256) {
        const int n = i >> 3, kc = i & 7;
        const float r = col_r[n];
        uint32_t c[4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
            c[j] = e4m3x2(__fmul_rn(tile[kc * 8 + 2 * j][n], r), __fmul_rn(tile[kc * 8 + 2 * j + 1][n], r));
        *reinterpret_cast<uint2 *>(Wqe + (size_t)(n0 + n) * K + k0 + kc * 8) =
            make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
    }
}

// amax [n] -> dequantisation scale s [n], in place
__global__ void quant_cols_scale_kernel(float *__restrict__ amax_to_scale, int64_t n)
{
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) {
        float r, s;
        fp8_scales(amax_to_scale[i], r, s);
        amax_to_scale[i] = s;
    }
}

} // namespace moe
