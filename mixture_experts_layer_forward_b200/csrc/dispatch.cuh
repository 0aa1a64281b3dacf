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

// Outputs of expert e (< E) from its routed rows c and the inclusive scans over experts of:
// c, its m-tiles, its m-tile pairs, its m-tiles if it has two or more ("hot"), 1 if it has
// exactly one ("cold"), 1 if it has rows. s_poff[e] receives the expert's padded row offset
// and, from the last expert, s_poff[E] = P_pad.
__device__ __forceinline__ void scan_write_expert(int e, int E, int c, int inc_c, int inc_t,
                                                  int inc_p, int inc_h, int inc_1, int inc_a,
                                                  const ScanOut &o, int *s_poff)
{
    const int ntile = (c + M_TILE - 1) / M_TILE;
    const int nptile = (ntile + 1) / 2;
    const int hot_t = ntile >= 2 ? ntile : 0;
    if (o.counts != nullptr) o.counts[e] = c;
    if (o.offsets != nullptr) {
        o.offsets[e + 1] = inc_c;
        if (e == 0) o.offsets[0] = 0;
    }
    const int poff_next = inc_t * M_TILE;
    const int tile_first = inc_t - ntile;
    o.padded_offsets[e + 1] = poff_next;
    o.tile_off[e + 1] = inc_t;
    if (e == 0) {
        o.padded_offsets[0] = 0;
        o.tile_off[0] = 0;
    }
    s_poff[e] = tile_first * M_TILE;
    for (int i = 0; i < ntile; ++i) o.tile_expert[tile_first + i] = e;
    if (o.ptile_off != nullptr) {
        o.ptile_off[e + 1] = inc_p;
        if (e == 0) o.ptile_off[0] = 0;
        for (int i = 0; i < nptile; ++i) o.ptile_expert[inc_p - nptile + i] = e;
    }
    if (o.hot_off != nullptr) {
        o.hot_off[e + 1] = inc_h;
        if (e == 0) o.hot_off[0] = 0;
        for (int i = 0; i < hot_t; ++i) o.hot_tile_expert[inc_h - hot_t + i] = e;
        if (ntile == 1) o.cold_tile[inc_1 - 1] = tile_first;
    }
    if (o.active_list != nullptr && c > 0) o.active_list[inc_a - 1] = e; // ascending ids
    if (e == E - 1) {
        o.meta->num_tiles = inc_t;
        o.meta->padded_rows = poff_next;
        o.meta->num_ptiles = inc_p;
        o.meta->num_cold = inc_1;
        o.meta->num_active = inc_a;
        s_poff[E] = poff_next;
    }
}

// Pad rows of each expert (rows s_poff[e] + s_cnt[e] .. s_poff[e + 1]) and every row past
// P_pad = s_poff[E]: gather_idx = -1, weight 0. Thread `tid` of `nt` (a multiple of 32): one
// warp per expert, lanes on consecutive rows.
__device__ __forceinline__ void scan_write_pads(int E, const ScanOut &o, const int *s_poff,
                                                const int *s_cnt, int tid, int nt)
{
    for (int ex = tid >> 5; ex < E; ex += nt >> 5) {
        const int end = s_poff[ex + 1];
        for (int r = s_poff[ex] + s_cnt[ex] + (tid & 31); r < end; r += 32) {
            o.gather_idx[r] = -1;
            if (o.row_w != nullptr) o.row_w[r] = 0.0f;
        }
    }
    for (int64_t r = (int64_t)s_poff[E] + tid; r < o.padded_rows_max; r += nt) {
        o.gather_idx[r] = -1;
        if (o.row_w != nullptr) o.row_w[r] = 0.0f;
    }
}

// Everything derived from the per-expert row counts, by one block of 1024 threads in which
// thread e owns expert e (c = its routed rows; E <= 1024). s_poff[0..E] receives the padded
// row offsets, s_cnt[0..E-1] the counts. Ends with a block barrier.
__device__ __forceinline__ void dispatch_scan_body(int c, int E, const ScanOut &o, int *warp_sums,
                                                   int *s_poff, int *s_cnt)
{
    // the fused layer kernel's tile-level ready counters start from zero on every call
    for (int i = threadIdx.x; i < o.n_ready; i += blockDim.x) o.ready[i] = 0;
    const int e = threadIdx.x;
    const int ntile = (c + M_TILE - 1) / M_TILE;
    const int inc_c = block_inclusive_scan_1024(c, warp_sums);
    const int inc_t = block_inclusive_scan_1024(ntile, warp_sums);
    const int inc_p = block_inclusive_scan_1024((ntile + 1) / 2, warp_sums);
    // work classes of the grouped GEMMs: "cold" experts (one m-tile) stream their weights for
    // a single tile; the rest ("hot") reuse each weight tile across their m-tiles
    const int inc_h = block_inclusive_scan_1024(ntile >= 2 ? ntile : 0, warp_sums);
    const int inc_1 = block_inclusive_scan_1024(ntile == 1 ? 1 : 0, warp_sums);
    const int inc_a = block_inclusive_scan_1024(c > 0 ? 1 : 0, warp_sums);
    if (e < E) {
        scan_write_expert(e, E, c, inc_c, inc_t, inc_p, inc_h, inc_1, inc_a, o, s_poff);
        s_cnt[e] = c;
    }
    __syncthreads();
    scan_write_pads(E, o, s_poff, s_cnt, threadIdx.x, blockDim.x);
    __syncthreads();
}

// Inclusive scan over the lanes of one warp.
__device__ __forceinline__ int warp_inclusive_scan(int v, int lane)
{
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, v, off);
        if (lane >= off) v += o;
    }
    return v;
}

// The scan outputs for E <= 32 experts by one warp (lane e owns expert e, c = its rows):
// the same values as dispatch_scan_body. s_poff[0..E] receives the padded row offsets.
__device__ __forceinline__ void dispatch_scan_warp(int c, int E, const ScanOut &o, int *s_poff,
                                                   int lane)
{
    if (lane >= E) c = 0;
    const int ntile = (c + M_TILE - 1) / M_TILE;
    const int inc_c = warp_inclusive_scan(c, lane);
    const int inc_t = warp_inclusive_scan(ntile, lane);
    const int inc_p = warp_inclusive_scan((ntile + 1) / 2, lane);
    const int inc_h = warp_inclusive_scan(ntile >= 2 ? ntile : 0, lane);
    const int inc_1 = warp_inclusive_scan(ntile == 1 ? 1 : 0, lane);
    const int inc_a = warp_inclusive_scan(c > 0 ? 1 : 0, lane);
    if (lane < E) scan_write_expert(lane, E, c, inc_c, inc_t, inc_p, inc_h, inc_1, inc_a, o, s_poff);
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

// In-launch dispatch of the whole-layer launch (routing, dispatch, the expert GEMMs and the
// combine in one persistent launch). The routing left, per group g of tt tokens (tokens
// g * tt .. g * tt + tt - 1), its selections per expert in group_counts[g][e]; after a
// grid-wide barrier every CTA runs dispatch_front for the groups it routed. The outputs are
// those of the three dispatch kernels and the gather, except that x_perm's pad rows are not
// written (their layer0 and layer1 rows are never combined).
struct FrontDispatch {
    const int32_t *group_counts; // [n_groups][E]
    int n_groups, tt;
    const int32_t *topk_idx;     // [T, k]
    const float *topk_w;         // [T, k]
    int T, E, k, H;
    ScanOut so;                  // CTA 0 writes the scan outputs and clears so.ready
    int32_t *inv_pos;            // [T, k]
    const __nv_bfloat16 *x;      // [T, H]
    __nv_bfloat16 *x_perm;       // [P_pad, H]
};

// Shared-memory scratch of dispatch_front, in ints (E <= 32, tt <= 128).
__host__ __device__ inline int front_scratch_ints(int n_groups, int E)
{
    return (n_groups + 1) * E + (E + 1) + 4 * E;
}

// All threads of the CTA; groups g_first, g_first + g_step, ... are this CTA's; the lead CTA
// writes the scan outputs. Every thread has fenced its x_perm stores for the async proxy
// (TMA readers) at the end.
__device__ __forceinline__ void dispatch_front(const FrontDispatch &d, int g_first, int g_step,
                                               bool lead, int *scratch)
{
    const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31, warp = tid >> 5, nw = nt >> 5;
    const int E = d.E, G = d.n_groups, k = d.k;
    int *pref = scratch;                                              // [G + 1][E]
    int *s_poff = pref + (size_t)(G + 1) * E;                          // [E + 1]
    uint32_t *bits = reinterpret_cast<uint32_t *>(s_poff + E + 1);     // [E][4]
    // 1. per expert, the exclusive prefix of the selections over the groups (the rows of
    //    lower token ids come first within an expert), one warp per expert; row G: totals
    for (int e = warp; e < E; e += nw) {
        int run = 0;
        for (int g0 = 0; g0 < G; g0 += 32) {
            const int g = g0 + lane;
            const int v = g < G ? d.group_counts[(size_t)g * E + e] : 0;
            const int inc = warp_inclusive_scan(v, lane);
            if (g < G) pref[(size_t)g * E + e] = run + inc - v;
            run += __shfl_sync(0xffffffffu, inc, 31);
        }
        if (lane == 0) pref[(size_t)G * E + e] = run;
    }
    __syncthreads();
    const int *total = pref + (size_t)G * E;
    // 2. padded offsets (every CTA); CTA 0 also writes the scan outputs, the pad markers and
    //    clears the ready counters of the GEMM phases
    if (warp == 0) {
        const int c = lane < E ? total[lane] : 0;
        if (lead) {
            dispatch_scan_warp(c, E, d.so, s_poff, lane);
        } else {
            const int ntile = (c + M_TILE - 1) / M_TILE;
            const int inc_t = warp_inclusive_scan(ntile, lane);
            if (lane < E) s_poff[lane] = (inc_t - ntile) * M_TILE;
            if (lane == E - 1) s_poff[E] = inc_t * M_TILE;
        }
    }
    if (lead)
        for (int i = tid; i < d.so.n_ready; i += nt) d.so.ready[i] = 0;
    __syncthreads();
    if (lead) scan_write_pads(E, d.so, s_poff, total, tid, nt);
    // 3. rows of this CTA's pairs (expert, then token order), and their x rows
    const int chunks = d.H / 8;
    for (int g = g_first; g < G; g += g_step) {
        const int t0 = g * d.tt;
        const int ntg = min(d.tt, d.T - t0);
        for (int i = tid; i < 4 * E; i += nt) bits[i] = 0u;
        __syncthreads();
        const int P = ntg * k;
        const size_t q0 = (size_t)t0 * k;
        for (int q = tid; q < P; q += nt) {
            const int tl = q / k;
            const int e = d.topk_idx[q0 + q];
            if (e >= 0 && e < E) atomicOr(&bits[e * 4 + (tl >> 5)], 1u << (tl & 31));
        }
        __syncthreads();
        // one warp per pair: lane 0 writes the indices, the warp copies the row
        for (int q = warp; q < P; q += nw) {
            const int tl = q / k;
            const int t = t0 + tl;
            const int e = d.topk_idx[q0 + q];
            if (e < 0 || e >= E) continue;
            const uint32_t *b = bits + e * 4;
            const int wd = tl >> 5;
            int rank = __popc(b[wd] & ((1u << (tl & 31)) - 1u));
            for (int w = 0; w < wd; ++w) rank += __popc(b[w]);
            const int r = s_poff[e] + pref[(size_t)g * E + e] + rank;
            if (lane == 0) {
                d.so.gather_idx[r] = t;
                d.inv_pos[q0 + q] = r;
                if (d.so.row_w != nullptr) d.so.row_w[r] = d.topk_w[q0 + q];
            }
            const uint4 *src = reinterpret_cast<const uint4 *>(d.x + (size_t)t * d.H);
            uint4 *dst = reinterpret_cast<uint4 *>(d.x_perm + (size_t)r * d.H);
            // a lane's 16-byte pieces of the row, 16 loads in flight before the stores (ten
            // warps per SM copy: memory parallelism has to come from each lane)
            int c = lane;
            for (; c + 15 * 32 < chunks; c += 16 * 32) {
                uint4 v[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) v[i] = src[c + i * 32];
#pragma unroll
                for (int i = 0; i < 16; ++i) dst[c + i * 32] = v[i];
            }
            for (; c < chunks; c += 32) dst[c] = src[c];
        }
        __syncthreads(); // the bitmaps are reused by the next group
    }
    asm volatile("fence.proxy.async.global;" ::: "memory");
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
