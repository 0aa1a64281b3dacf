// ep.cuh -- the expert-parallel exchange driven by the device: the routed rows travel to the
// rank that holds their expert and the expert outputs travel back by plain stores into the
// other ranks' buffers (peer memory over NVLink), with no host read of the routing.
//
// Where it comes from (Comet: Fine-grained Computation-communication Overlapping for
// Mixture-of-Experts, §2.1 and §3.1: experts are placed on different GPUs, the routed tokens
// travel to their experts' GPU before layer0 and the outputs travel back after layer1; §4:
// the transfers are issued from the GPU, not by a host-driven collective).
//
// Rank r holds experts [r * E_loc, (r + 1) * E_loc). Every rank owns, in memory that every
// other rank can address (symmetric allocations), a counts table [world, world], receive
// buffers for rows, local expert ids, gates and origins, and a return buffer [T * k, H]:
//   1. publish: this rank's rows for destination d (from its dispatch offsets) are written
//      into row `rank` of every rank's table;               -- then a barrier of all ranks
//   2. scatter: every routed pair (t, j) of this rank goes to slot
//      base(rank, d) + (its position among this rank's rows for d) of destination d's
//      buffers, base(rank, d) = rows that lower ranks send to d; the slot also records the
//      pair's origin (rank, t * k + j);                      -- then a barrier
//   3. the receiver runs its experts on its first n_recv = sum_s table[s][rank] rows
//      (moe_experts_forward_n: the row count stays on the device);
//   4. return: received row i goes to row (t * k + j) of its origin rank's return buffer;
//                                                             -- then a barrier
//   5. every rank combines its return buffer (j ascending, fp32, one bf16 rounding).
// The positions keep the order of the single-GPU dispatch (expert, then token), so every
// gated row is bitwise the row moe_forward computes. Loads read this GPU's own memory only;
// the stores to other GPUs are plain 16-byte stores.
#pragma once

#include "ptx.cuh"

namespace moe {

// tables[r][rank * world + d] = rows this rank sends to d, for every rank r (thread d owns d)
__global__ void ep_publish_counts_kernel(const int32_t *__restrict__ offsets, int E_loc, int world,
                                         int rank, int32_t *const *tables)
{
    for (int d = threadIdx.x; d < world; d += blockDim.x) {
        const int c = offsets[(d + 1) * E_loc] - offsets[d * E_loc];
        for (int r = 0; r < world; ++r) tables[r][rank * world + d] = c;
    }
}

struct EpScatterArgs {
    const __nv_bfloat16 *x;       // [T, H]
    const int32_t *topk_idx;      // [T, k], global expert ids
    const float *topk_w;          // [T, k]
    const int32_t *offsets;       // [E + 1] this rank's rows per expert (exclusive scan)
    const int32_t *poff;          // [E + 1] the same, padded to 128-row tiles
    const int32_t *inv_pos;       // [T, k] padded row of each pair
    const int32_t *table;         // [world, world] this rank's copy of the counts table
    __nv_bfloat16 *const *rows;   // [world] -> [recv_cap, H]
    int32_t *const *ids;          // [world] -> [recv_cap] expert id local to the receiver
    float *const *gates;          // [world] -> [recv_cap]
    long long *const *origin;     // [world] -> [recv_cap] (rank << 32) | pair
    int64_t recv_cap;
    int32_t *n_recv;              // [1] rows this rank receives
    int T, H, E, k, E_loc, world, rank;
    int *status;
};

// One warp per routed pair of this rank: its row, expert id, gate and origin into the
// destination's buffers. Block 0 also writes n_recv.
__global__ void __launch_bounds__(256) ep_scatter_kernel(const EpScatterArgs a)
{
    const int lane = threadIdx.x & 31;
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        int n = 0;
        for (int s = 0; s < a.world; ++s) n += a.table[s * a.world + a.rank];
        *a.n_recv = n;
    }
    const int64_t P = (int64_t)a.T * a.k;
    const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t q = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; q < P; q += nw) {
        const int e = a.topk_idx[q];
        if (e < 0 || e >= a.E) {
            if (lane == 0) record_status(a.status, DEV_BAD_INDEX, 401);
            continue;
        }
        const int d = e / a.E_loc;
        const int u = a.inv_pos[q] - a.poff[e] + a.offsets[e]; // unpadded (expert, token) order
        int base = 0;
        for (int s = 0; s < a.rank; ++s) base += a.table[s * a.world + d];
        const int64_t slot = (int64_t)base + (u - a.offsets[d * a.E_loc]);
        if (slot < 0 || slot >= a.recv_cap) {
            if (lane == 0) record_status(a.status, DEV_BAD_INDEX, 402);
            continue;
        }
        const int t = (int)(q / a.k);
        const uint4 *src = reinterpret_cast<const uint4 *>(a.x + (size_t)t * a.H);
        uint4 *dst = reinterpret_cast<uint4 *>(a.rows[d] + (size_t)slot * a.H);
        for (int v = lane; v < a.H / 8; v += 32) dst[v] = src[v];
        if (lane == 0) {
            a.ids[d][slot] = e - d * a.E_loc;
            a.gates[d][slot] = a.topk_w[q];
            a.origin[d][slot] = ((long long)a.rank << 32) | (long long)q;
        }
    }
}

// One warp per received row i < n_recv: the expert output y[i] goes to row `pair` of the
// return buffer of rank `origin >> 32`.
__global__ void __launch_bounds__(256)
    ep_return_kernel(const __nv_bfloat16 *__restrict__ y, const long long *__restrict__ origin,
                     const int32_t *__restrict__ n_recv, int H, int world, int64_t back_rows,
                     __nv_bfloat16 *const *back, int *status)
{
    const int lane = threadIdx.x & 31;
    const int64_t n = *n_recv;
    const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; i < n; i += nw) {
        const long long o = origin[i];
        const int s = (int)(o >> 32);
        const int64_t q = (int64_t)(o & 0xffffffffll);
        if (s < 0 || s >= world || q >= back_rows) {
            if (lane == 0) record_status(status, DEV_BAD_INDEX, 403);
            continue;
        }
        const uint4 *src = reinterpret_cast<const uint4 *>(y + (size_t)i * H);
        uint4 *dst = reinterpret_cast<uint4 *>(back[s] + (size_t)q * H);
        for (int v = lane; v < H / 8; v += 32) dst[v] = src[v];
    }
}

} // namespace moe
