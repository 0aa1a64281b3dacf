// dispatch.cuh -- token dispatch into expert-contiguous, tile-padded rows
// (Comet: Fine-grained Computation-communication Overlapping for Mixture-of-Experts,
// §2.2.1: expose to each computation tile only the rows it needs; §3.1.2: regroup the
// decomposed rows into whole GEMM tiles).
//
// A deterministic counting sort of the T*k routed pairs by expert, stable in token id:
//   dispatch_count_kernel   per token chunk, per-expert pair counts           [nchunk][E]
//   dispatch_scan_kernel    per-expert scan over chunks, expert counts, offsets, padded
//                           offsets, the m-tile list, pad-row markers         (one block)
//   dispatch_place_kernel   each pair's row = padded_offset[e] + chunk base + rank of the
//                           token among the chunk's tokens routed to e (a popcount over a
//                           per-expert token bitmap, so no ordering depends on atomics)
//   gather_rows_kernel      optional materialised x_perm[r] = x[gather_idx[r]]
// Batches of at most one chunk (T <= 256: decode-sized) take dispatch_small_kernel instead,
// the three steps in one block, with the same outputs.
// Counts and bitmaps are built with shared-memory atomics whose result does not depend on
// their order, so every output is bit-reproducible.
#pragma once

#include "ptx.cuh"

namespace moe {

constexpr int DISPATCH_CHUNK = 256; // tokens per chunk (one thread per token)
constexpr int DISPATCH_WORDS = DISPATCH_CHUNK / 32;
constexpr int M_TILE = 128;

// Workspace-resident bookkeeping written by the scan and read by the GEMMs.
struct DispatchMeta {
    int num_tiles;   // sum_e ceil(c_e / M_TILE)
    int padded_rows; // P_pad = num_tiles * M_TILE
    int num_ptiles;  // sum_e ceil(ceil(c_e / M_TILE) / 2): pairs of m-tiles of one expert
    int num_cold;    // experts with exactly one m-tile (their weights are read for one tile)
    int num_active;  // experts with at least one routed row
};

__global__ void __launch_bounds__(DISPATCH_CHUNK)
    dispatch_count_kernel(const int32_t *__restrict__ topk_idx, int T, int E, int k,
                          int32_t *__restrict__ chunk_counts, int *status, int clear_status,
                          const int *__restrict__ n_rows)
{
    extern __shared__ int cnt[];
    if (clear_status && status != nullptr && blockIdx.x == 0 && threadIdx.x == 0) {
        status[0] = DEV_OK;
        status[1] = 0;
    }
    for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
    __syncthreads();
    const int t = blockIdx.x * DISPATCH_CHUNK + threadIdx.x;
    // n_rows (optional, device): only tokens t < *n_rows are routed
    const int Tn = n_rows != nullptr ? min(T, *n_rows) : T;
    if (t < Tn) {
        for (int j = 0; j < k; ++j) {
            const int e = topk_idx[(size_t)t * k + j];
            if (e >= 0 && e < E) {
                atomicAdd(&cnt[e], 1);
            } else {
                record_status(status, DEV_BAD_INDEX, 1);
            }
            // a token's experts must be distinct (checked for the usual small k)
            if (k <= 16) {
                for (int j2 = 0; j2 < j; ++j2)
                    if (topk_idx[(size_t)t * k + j2] == e) record_status(status, DEV_BAD_INDEX, 2);
            }
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x)
        chunk_counts[(size_t)blockIdx.x * E + e] = cnt[e];
}

// Inclusive block scan of one int per thread (blockDim.x == 1024).
__device__ __forceinline__ int block_inclusive_scan_1024(int v, int *warp_sums)
{
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, v, off);
        if (lane >= off) v += o;
    }
    if (lane == 31) warp_sums[warp] = v;
    __syncthreads();
    if (warp == 0) {
        int s = warp_sums[lane];
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int o = __shfl_up_sync(0xffffffffu, s, off);
            if (lane >= off) s += o;
        }
        warp_sums[lane] = s;
    }
    __syncthreads();
    if (warp > 0) v += warp_sums[warp - 1];
    __syncthreads();
    return v;
}

// Outputs of the scan step (all device pointers; the optional ones may be null).
struct ScanOut {
    int32_t *counts, *offsets, *padded_offsets, *tile_off, *tile_expert;
    int32_t *ptile_off, *ptile_expert;
    DispatchMeta *meta;
    int32_t *gather_idx;
    float *row_w;
    int64_t padded_rows_max;
    int *ready;
    int n_ready;
    int32_t *hot_off, *hot_tile_expert, *cold_tile, *active_list;
};

// Everything derived from the per-expert row counts, by one block of 1024 threads in which
// thread e owns expert e (c = its routed rows; E <= 1024). s_poff[0..E] receives the padded
// row offsets, s_cnt[0..E-1] the counts. Ends with a block barrier.
__device__ __forceinline__ void dispatch_scan_body(int c, int E, const ScanOut &o, int *warp_sums,
                                                   int *s_poff, int *s_cnt)
{
    // the fused layer kernel's tile-level ready counters start from zero on every call
    for (int i = threadIdx.x; i < o.n_ready; i += blockDim.x) o.ready[i] = 0;
    const int e = threadIdx.x;
    int32_t *const counts = o.counts, *const offsets = o.offsets;
    int32_t *const padded_offsets = o.padded_offsets, *const tile_off = o.tile_off;
    int32_t *const tile_expert = o.tile_expert, *const ptile_off = o.ptile_off;
    int32_t *const ptile_expert = o.ptile_expert, *const hot_off = o.hot_off;
    int32_t *const hot_tile_expert = o.hot_tile_expert, *const cold_tile = o.cold_tile;
    int32_t *const active_list = o.active_list, *const gather_idx = o.gather_idx;
    float *const row_w = o.row_w;
    DispatchMeta *const meta = o.meta;
    if (e < E && counts != nullptr) counts[e] = c;
    const int ntile = (c + M_TILE - 1) / M_TILE;
    const int inc_c = block_inclusive_scan_1024(c, warp_sums);
    const int inc_t = block_inclusive_scan_1024(ntile, warp_sums);
    const int nptile = (ntile + 1) / 2;
    const int inc_p = block_inclusive_scan_1024(nptile, warp_sums);
    // work classes of the grouped GEMMs: "cold" experts (one m-tile) stream their weights for
    // a single tile; the rest ("hot") reuse each weight tile across their m-tiles
    const int hot_t = ntile >= 2 ? ntile : 0;
    const int inc_h = block_inclusive_scan_1024(hot_t, warp_sums);
    const int inc_1 = block_inclusive_scan_1024(ntile == 1 ? 1 : 0, warp_sums);
    const int inc_a = block_inclusive_scan_1024(c > 0 ? 1 : 0, warp_sums);
    if (e < E) {
        if (offsets != nullptr) {
            offsets[e + 1] = inc_c;
            if (e == 0) offsets[0] = 0;
        }
        const int poff_next = inc_t * M_TILE;
        const int tile_first = inc_t - ntile;
        padded_offsets[e + 1] = poff_next;
        tile_off[e + 1] = inc_t;
        if (e == 0) {
            padded_offsets[0] = 0;
            tile_off[0] = 0;
        }
        s_poff[e] = tile_first * M_TILE;
        for (int i = 0; i < ntile; ++i) tile_expert[tile_first + i] = e;
        if (ptile_off != nullptr) {
            ptile_off[e + 1] = inc_p;
            if (e == 0) ptile_off[0] = 0;
            for (int i = 0; i < nptile; ++i) ptile_expert[inc_p - nptile + i] = e;
        }
        if (hot_off != nullptr) {
            hot_off[e + 1] = inc_h;
            if (e == 0) hot_off[0] = 0;
            for (int i = 0; i < hot_t; ++i) hot_tile_expert[inc_h - hot_t + i] = e;
            if (ntile == 1) cold_tile[inc_1 - 1] = tile_first;
        }
        if (active_list != nullptr && c > 0) active_list[inc_a - 1] = e; // ascending ids
        if (e == E - 1) {
            meta->num_tiles = inc_t;
            meta->padded_rows = poff_next;
            meta->num_ptiles = inc_p;
            meta->num_cold = inc_1;
            meta->num_active = inc_a;
            s_poff[E] = poff_next;
        }
    }
    if (e < E) s_cnt[e] = c;
    __syncthreads();
    // pad rows of each expert (one warp per expert, lanes on consecutive rows), then
    // everything past P_pad: gather_idx = -1, weight 0
    for (int ex = threadIdx.x >> 5; ex < E; ex += blockDim.x >> 5) {
        const int end = s_poff[ex + 1];
        for (int r = s_poff[ex] + s_cnt[ex] + (threadIdx.x & 31); r < end; r += 32) {
            gather_idx[r] = -1;
            if (row_w != nullptr) row_w[r] = 0.0f;
        }
    }
    for (int64_t r = (int64_t)s_poff[E] + threadIdx.x; r < o.padded_rows_max; r += blockDim.x) {
        gather_idx[r] = -1;
        if (row_w != nullptr) row_w[r] = 0.0f;
    }
    __syncthreads();
}

// One block of 1024 threads; thread e owns expert e (E <= 1024).
//   chunk_counts [nchunk][E] is rewritten in place into each chunk's base row within e.
__global__ void __launch_bounds__(1024)
    dispatch_scan_kernel(int32_t *__restrict__ chunk_counts, int nchunk, int E, ScanOut o)
{
    __shared__ int warp_sums[32];
    __shared__ int s_poff[1025];
    __shared__ int s_cnt[1024];
    const int e = threadIdx.x;
    int c = 0;
    if (e < E) {
        int run = 0;
        // eight chunks' counts loaded before any is rewritten: eight loads in flight
        for (int ch0 = 0; ch0 < nchunk; ch0 += 8) {
            int v[8];
#pragma unroll
            for (int q = 0; q < 8; ++q)
                v[q] = (ch0 + q < nchunk) ? chunk_counts[(size_t)(ch0 + q) * E + e] : 0;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                if (ch0 + q < nchunk) chunk_counts[(size_t)(ch0 + q) * E + e] = run;
                run += v[q];
            }
        }
        c = run;
    }
    dispatch_scan_body(c, E, o, warp_sums, s_poff, s_cnt);
}

// Rows of token t's k pairs: padded_offsets[e] + chunk_base[e] (null: 0) + the rank of t
// among its chunk's tokens routed to e (tl = t's position in the chunk; bits = the chunk's
// token bitmap per expert).
__device__ __forceinline__ void dispatch_place_token(
    const int32_t *__restrict__ topk_idx, const float *__restrict__ topk_w, int t, int tl, int E,
    int k, const uint32_t *bits, const int32_t *padded_offsets, const int32_t *chunk_base,
    int32_t *__restrict__ gather_idx, int32_t *__restrict__ inv_pos, float *__restrict__ row_w)
{
    const int word = tl >> 5;
    const uint32_t bit = 1u << (tl & 31);
    for (int j = 0; j < k; ++j) {
        const int e = topk_idx[(size_t)t * k + j];
        if (e < 0 || e >= E) {
            inv_pos[(size_t)t * k + j] = -1;
            continue;
        }
        const uint32_t *b = bits + e * DISPATCH_WORDS;
        int rank = __popc(b[word] & (bit - 1u));
        for (int w = 0; w < word; ++w) rank += __popc(b[w]);
        const int r = padded_offsets[e] + (chunk_base != nullptr ? chunk_base[e] : 0) + rank;
        gather_idx[r] = t;
        inv_pos[(size_t)t * k + j] = r;
        if (row_w != nullptr) row_w[r] = topk_w[(size_t)t * k + j];
    }
}

// Dynamic shared memory: E * DISPATCH_WORDS uint32 (token bitmap per expert).
__global__ void __launch_bounds__(DISPATCH_CHUNK)
    dispatch_place_kernel(const int32_t *__restrict__ topk_idx, const float *__restrict__ topk_w,
                          int T, int E, int k, const int32_t *__restrict__ chunk_base,
                          const int32_t *__restrict__ padded_offsets,
                          int32_t *__restrict__ gather_idx, int32_t *__restrict__ inv_pos,
                          float *__restrict__ row_w, const int *__restrict__ n_rows)
{
    extern __shared__ uint32_t bits[];
    for (int i = threadIdx.x; i < E * DISPATCH_WORDS; i += blockDim.x) bits[i] = 0u;
    __syncthreads();
    const int tl = threadIdx.x;
    const int t = blockIdx.x * DISPATCH_CHUNK + tl;
    const int word = tl >> 5;
    const uint32_t bit = 1u << (tl & 31);
    T = n_rows != nullptr ? min(T, *n_rows) : T; // tokens past *n_rows are not routed
    if (t < T) {
        for (int j = 0; j < k; ++j) {
            const int e = topk_idx[(size_t)t * k + j];
            if (e >= 0 && e < E) atomicOr(&bits[e * DISPATCH_WORDS + word], bit);
        }
    }
    __syncthreads();
    if (t >= T) return;
    dispatch_place_token(topk_idx, topk_w, t, tl, E, k, bits, padded_offsets,
                         chunk_base + (size_t)blockIdx.x * E, gather_idx, inv_pos, row_w);
}

// T <= DISPATCH_CHUNK: count, scan and place in one block of 1024 threads (the threads stride
// over the T * k (token, selection) pairs in the count and place steps; thread e owns expert
// e in the scan), with the outputs of the three-kernel path. Dynamic shared memory: E * (DISPATCH_WORDS + 1) uint32.
__global__ void __launch_bounds__(1024)
    dispatch_small_kernel(const int32_t *__restrict__ topk_idx, const float *__restrict__ topk_w,
                          int T, int E, int k, ScanOut o, int32_t *__restrict__ inv_pos,
                          int *status, int clear_status, const int *__restrict__ n_rows)
{
    extern __shared__ uint32_t sm_words[];
    uint32_t *bits = sm_words;                                        // [E][DISPATCH_WORDS]
    int *cnt = reinterpret_cast<int *>(sm_words + E * DISPATCH_WORDS); // [E]
    __shared__ int warp_sums[32];
    __shared__ int s_poff[1025];
    __shared__ int s_cnt[1024];
    if (clear_status && status != nullptr && threadIdx.x == 0) {
        status[0] = DEV_OK;
        status[1] = 0;
    }
    for (int i = threadIdx.x; i < E * DISPATCH_WORDS; i += blockDim.x) bits[i] = 0u;
    for (int i = threadIdx.x; i < E; i += blockDim.x) cnt[i] = 0;
    __syncthreads();
    // One (token, selection) pair per thread and step, so that the pairs' loads are
    // independent. A token's experts must be distinct: a pair that finds its (expert, token)
    // bit already set is a repeat.
    const int P = (n_rows != nullptr ? min(T, *n_rows) : T) * k; // tokens past *n_rows: not routed
    for (int q = threadIdx.x; q < P; q += blockDim.x) {
        const int t = q / k;
        const int e = topk_idx[q];
        if (e >= 0 && e < E) {
            atomicAdd(&cnt[e], 1);
            const uint32_t bit = 1u << (t & 31);
            if (atomicOr(&bits[e * DISPATCH_WORDS + (t >> 5)], bit) & bit)
                record_status(status, DEV_BAD_INDEX, 2);
        } else {
            record_status(status, DEV_BAD_INDEX, 1);
        }
    }
    __syncthreads();
    dispatch_scan_body(threadIdx.x < E ? cnt[threadIdx.x] : 0, E, o, warp_sums, s_poff, s_cnt);
    // placement of each pair: its row is the expert's padded offset plus the number of
    // earlier tokens of the expert (ascending token order within the expert)
    for (int q = threadIdx.x; q < P; q += blockDim.x) {
        const int t = q / k;
        const int e = topk_idx[q];
        if (e < 0 || e >= E) {
            inv_pos[q] = -1;
            continue;
        }
        const uint32_t *b = bits + e * DISPATCH_WORDS;
        const int word = t >> 5;
        int rank = __popc(b[word] & ((1u << (t & 31)) - 1u));
        for (int w = 0; w < word; ++w) rank += __popc(b[w]);
        const int r = s_poff[e] + rank;
        o.gather_idx[r] = t;
        inv_pos[q] = r;
        if (o.row_w != nullptr) o.row_w[r] = topk_w[q];
    }
}

// x_perm[r][:] = x[gather_idx[r]][:] (zeros on pad rows), for r < P_pad. One warp per row.
__global__ void __launch_bounds__(256)
    gather_rows_kernel(const __nv_bfloat16 *__restrict__ x, const int32_t *__restrict__ gather_idx,
                       const DispatchMeta *meta, int T, int H, __nv_bfloat16 *__restrict__ x_perm)
{
    const int rows = meta->padded_rows;
    const int lane = threadIdx.x & 31;
    const int nw = (gridDim.x * blockDim.x) >> 5;
    const int chunks = H / 8;
    for (int r = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < rows; r += nw) {
        const int t = gather_idx[r];
        uint4 *dst = reinterpret_cast<uint4 *>(x_perm + (size_t)r * H);
        if (t >= 0 && t < T) {
            const uint4 *src = reinterpret_cast<const uint4 *>(x + (size_t)t * H);
            for (int c = lane; c < chunks; c += 32) dst[c] = src[c];
        } else {
            for (int c = lane; c < chunks; c += 32) dst[c] = make_uint4(0u, 0u, 0u, 0u);
        }
    }
}

} // namespace moe
