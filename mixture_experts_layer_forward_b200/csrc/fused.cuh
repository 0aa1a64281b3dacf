// fused.cuh -- one persistent launch for layer0, layer1 and the combine, scheduled by
// tile-level ready flags; optionally with the routing and dispatch in front of them (the
// whole layer in one launch), or as one rank of the expert-parallel layer (rows exchanged
// with the other ranks inside the launch). The body is fused_layer_body<KIND0, MODE>:
//   FUSED_LAYERS  layer0 -> layer1 -> combine (route and dispatch ran before the launch);
//   FUSED_WHOLE   fused_front (routing of the CTA's token groups, grid barrier, in-launch
//                 dispatch and row copy, grid barrier), then the same GEMM phases;
//   FUSED_EP      ep_front (routing, counts to every rank, a flag barrier of all ranks,
//                 destinations), ep_scatter by the eight non-GEMM-issuing warps while layer0
//                 tiles wait for their rows' arrival counts, layer1 rows stored back into
//                 their origins' buffers with per-(token, stripe) counts, and the combine of
//                 the rows that came back.
//
// Where it comes from (Comet: Fine-grained Computation-communication Overlapping for
// Mixture-of-Experts; and "Fine-grained Computation-Communication Overlap via Tile-level
// Signaling and Scheduling for MoE"):
//   - shared-tensor dependency resolving (Comet §3.1.1): the tensor shared by layer0 and
//     layer1 is h; layer0 produces it in 128-row M tiles, and a layer1 tile only needs the
//     h rows of its own M tile, so layer1 work starts tile by tile as layer0 finishes rows;
//   - layer1 is decomposed along N (§3.1.1): a combine item reduces one 256-column stripe of
//     the output for a block of tokens, and needs only that stripe of the layer1 tiles that
//     hold its tokens' rows;
//   - thread-block specialisation (§3.2.1) at warp granularity: in every CTA one warp moves
//     the GEMM operands (TMA), one issues the MMAs, four drain the accumulators, and four
//     more are the data-movement warps: during layer0 they gather token rows (small batches)
//     or take half of each tile's epilogue (rows arrive by TMA from the expert-sorted copy),
//     and during layer1 they run the combine, concurrently with the GEMM pipeline of their
//     own SM; the per-shape choice of this arrangement is fused_plan() in the host code
//     (§3.2.2 adaptive workload assignment);
//   - the tile-signalling design's producer (one persistent kernel over all local experts)
//     and its consumer driven by ready flags as tiles finish: here both live in one launch,
//     the flags are in global memory, and every wait is bounded.
//
// Work:
//   GEMM queue [ layer0 tiles (expert, m, n) | layer1 tiles (expert, m, n) ], both expert-
//   major (an expert's weight stripe and its rows stay in L2 across its tiles); CTA b takes
//   items b, b + grid, ... All CTAs are resident at once (one per SM), every item waits only
//   on items earlier in the queue, and a CTA finishes its earlier items before waiting.
//   Combine queue: (stripe, token block) items, stripe-major; CTA b's data-movement warps
//   take items b, b + grid, ... after their layer0 duties; they wait only on layer1 tiles,
//   and layer1 never waits on them.
//   ready0[m]             counts finished layer0 column tiles of M tile m; a layer1 tile of m
//                         waits for ready0[m] == layer0 N tiles before its TMA loads of h;
//   ready1[n * tiles + m] is set to 1 once layer1 tile (m, stripe n) is stored; a combine
//                         item waits, row by row, for the flag of the tile holding the row.
// Writers publish with a gpu-scope release after their stores (plus a generic-to-async proxy
// fence before ready0, since layer1 reads h with TMA); readers acquire.
#pragma once

#include "gemm_tc.cuh"
#include "route_chain.cuh"

namespace moe {

// The front of the whole-layer launch: routing (route_chain.cuh, with warp 0 issuing its TMA
// copies and warps 2 .. 2 + ncw - 1 walking the chains) of the token groups b, b + grid, ...,
// a grid-wide barrier, the in-launch dispatch (dispatch.cuh), and a second barrier after
// which every CTA sees the dispatch outputs and every x_perm row.
struct FrontArgs {
    RcArgs ra;        // router; ra.group_counts receives the per-group selections
    int ncw;          // consumer warps of the router (1..8)
    int n_groups;     // ceil(T / ra.tt)
    FrontDispatch fd; // in-launch dispatch
    int *gbar;        // grid-barrier counter, zero when the launch starts
};

// Expert parallelism inside the persistent launch (Comet §3.1.2 and §4; the tile-signalling
// abstract): rank r holds experts [r * e_loc, (r + 1) * e_loc). Every rank owns the buffers
// below (every rank can address every rank's copy: [world] arrays of pointers, plain
// loads and stores over NVLink); a rank's copy of the receive buffers holds the rows routed
// to its experts in its own expert-sorted, 128-row padded order (expert, then source rank,
// then source token), so that its layer0 reads them with TMA from its own memory.
struct EpArgs {
    int world, rank, e_loc;
    int epoch;                                // this call's number (> 0): barrier flags reach it
    int32_t *all_counts[EP_MAX_WORLD];        // [world][n_groups][E] every source's group counts
    int *flags[EP_MAX_WORLD];                 // [world] barrier flags, one per source rank
    __nv_bfloat16 *recv_rows[EP_MAX_WORLD];   // [recv_cap][H] rows routed to the rank's experts
    float *recv_gate[EP_MAX_WORLD];           // [recv_cap] their gate weights (0 on pad rows)
    long long *recv_origin[EP_MAX_WORLD];     // [recv_cap] (source rank << 32) | (t * k + j); -1 pads
    int *arrive[EP_MAX_WORLD];                // [max_tiles] rows arrived per local M tile
    __nv_bfloat16 *back[EP_MAX_WORLD];        // [T * k][H] gated rows returned to their origin
    int *back_cnt[EP_MAX_WORLD];              // [T][H / 256] rows returned per token and stripe
    int64_t recv_cap;
    int max_tiles;
    int32_t *slot;                            // [T * k] this rank's pairs: destination row
    int32_t *dest;                            // [T * k] this rank's pairs: destination rank
};

enum : int { FUSED_LAYERS = 0, FUSED_WHOLE = 1, FUSED_EP = 2 };

constexpr int COMBINE_TOKENS = 128; // tokens per combine item unless fused_plan() says otherwise

struct FusedArgs {
    GemmArgs l0;            // layer0: A = x_perm by TMA (a_tma) or rows gathered from x
    GemmArgs l1;            // layer1: h rows by TMA, W2, writes ys (gate-scaled)
    int *ready0;            // [max_tiles]
    int *done0;             // finished layer0 items (all of them: every M tile is ready)
    int *comb_next;         // next unclaimed combine item
    int *ready1;            // [l1.n_tiles, max_tiles]
    int max_tiles;
    const int32_t *inv_pos; // [T, k]
    __nv_bfloat16 *out;     // [T, H]
    int T, H, k;
    int64_t ys_rows;
    const __nv_bfloat16 *ys_shared; // [T, H] shared-expert rows added last, or nullptr
    int a_tma;              // 1: layer0 A rows by TMA (expert-sorted copy of x)
    int comb_tokens;        // tokens per combine item, a multiple of 32
    int comb_in_launch;     // 0: no combine in this launch (it runs as its own launch after)
    int fault_skip;         // test hook: layer0 item whose ready signal is withheld (-1: none)
    // optional schedule trace: records of 4 x uint64 {kind << 32 | item, smid, t_begin_ns,
    // t_end_ns}; trace[0] is the record counter, records start at trace[4]; nullptr: off
    unsigned long long *trace;
    int64_t trace_cap;      // records that fit after the counter
    FrontArgs front;        // whole-layer and expert-parallel launches
    EpArgs ep;              // expert-parallel launch (world > 0)
};

// TRACE_FRONT: a CTA's routing and dispatch (launch start to the GEMM phases); TRACE_SCATTER:
// a CTA's row sends of the expert-parallel launch (item = the CTA)
enum : int { TRACE_L0 = 0, TRACE_L1 = 1, TRACE_COMBINE = 2, TRACE_FRONT = 3, TRACE_SCATTER = 4 };

__device__ __forceinline__ int ld_acquire_gpu(const int *p)
{
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void red_release_gpu_add(int *p, int v)
{
    asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ void st_release_gpu(int *p, int v)
{
    asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// system scope (flags and counters that other GPUs write or read over NVLink)
__device__ __forceinline__ int ld_acquire_sys(const int *p)
{
    int v;
    asm volatile("ld.acquire.sys.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void red_release_sys_add(int *p, int v)
{
    asm volatile("red.release.sys.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ void st_release_sys(int *p, int v)
{
    asm volatile("st.release.sys.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// relaxed add at system scope: the release comes from a system-scope fence issued before
// it by the same thread (fence + strong write is a release pattern)
__device__ __forceinline__ void red_relaxed_sys_add(int *p, int v)
{
    asm volatile("red.relaxed.sys.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ void fence_proxy_async_global()
{
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

// arrive on an mbarrier with an arrival count (the phase expects that many more arrivals)
__device__ __forceinline__ void mbar_arrive_cnt(uint32_t bar, uint32_t cnt)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(cnt) : "memory");
}

__device__ __forceinline__ uint32_t smid_u32()
{
    uint32_t v;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(v));
    return v;
}

__device__ __forceinline__ void trace_record(const FusedArgs &fa, int kind, int item, uint64_t t0,
                                             uint64_t t1)
{
    if (fa.trace == nullptr) return;
    const unsigned long long i = atomicAdd(fa.trace, 1ull);
    if ((int64_t)i >= fa.trace_cap) return;
    unsigned long long *r = fa.trace + 4 + 4 * i;
    r[0] = ((unsigned long long)kind << 32) | (unsigned)item;
    r[1] = smid_u32();
    r[2] = t0;
    r[3] = t1;
}

// Bounded wait for *p >= target with acquire semantics (gpu scope, or system scope for
// values that other GPUs write). False after an abort elsewhere in the CTA or after
// timeout_ns (then the abort flag is raised and DEV_TIMEOUT recorded).
template <bool SYS = false>
__device__ __forceinline__ bool flag_wait_bounded(const int *p, int target, volatile int *abort_flag,
                                                  int64_t timeout_ns, int *status, int where)
{
    auto ld = [](const int *q) { return SYS ? ld_acquire_sys(q) : ld_acquire_gpu(q); };
    if (ld(p) >= target) return true;
    const uint64_t t0 = globaltimer_ns();
    uint32_t nap = 64; // exponential backoff up to 2 us: pollers stay off the L2 meanwhile
#pragma unroll 1
    while (true) {
        __nanosleep(nap);
        if (nap < 2048) nap <<= 1;
        if (ld(p) >= target) return true;
        if (*abort_flag) return false;
        if ((int64_t)(globaltimer_ns() - t0) > timeout_ns) {
            *abort_flag = 1;
            record_status(status, DEV_TIMEOUT, where);
            return false;
        }
    }
}

// Grid-wide barrier of a persistent launch (every CTA resident): the CTA's threads meet, thread
// 0 publishes the CTA's writes and waits, bounded, until `target` CTA arrivals have been
// counted on `ctr` (a launch-wide counter: the n-th barrier of the launch waits for n * grid).
// sys: the CTAs' earlier stores also went to other GPUs, and are made visible at system
// scope before the arrival.
__device__ __forceinline__ bool grid_barrier(int *ctr, int target, volatile int *abort_flag,
                                             int64_t timeout_ns, int *status, int where,
                                             bool sys = false)
{
    __syncthreads();
    int ok = 1;
    if (threadIdx.x == 0) {
        if (sys) __threadfence_system();
        else __threadfence();
        red_release_gpu_add(ctr, 1);
        ok = flag_wait_bounded(ctr, target, abort_flag, timeout_ns, status, where) ? 1 : 0;
    }
    return __syncthreads_and(ok) != 0;
}

// Routing, dispatch and the row copy of the whole-layer launch, in the GEMM stages' shared
// memory (free until the GEMM phases start). False when a wait gave up.
// Routing of the CTA's token groups (cta, cta + ncta, ...) in the GEMM stages' shared memory.
template <int G>
__device__ __forceinline__ bool front_route(const CUtensorMap *tmRX, const CUtensorMap *tmRW,
                                            const FrontArgs &f, uint8_t *smem,
                                            volatile int *abort_flag, int cta, int ncta)
{
    const RcLayout L = rc_layout(f.ra.tt, f.ra.E, 4 * G, f.ra.stages);
    if (threadIdx.x == 0) {
        rc_init(smem, L, f.ra.stages, f.ncw);
        tma_prefetch_desc(tmRX);
        tma_prefetch_desc(tmRW);
    }
    __syncthreads();
    bool ok = rc_run<4, G>(tmRX, tmRW, f.ra, smem, 0, 2, f.ncw, cta, ncta, f.n_groups, 1);
    ok = __syncthreads_and(ok ? 1 : 0) != 0;
    if (threadIdx.x == 0) rc_fini(smem, L, f.ra.stages);
    if (!ok) *abort_flag = 1;
    return ok;
}

__device__ __forceinline__ bool front_route_any(const CUtensorMap *tmRX, const CUtensorMap *tmRW,
                                                const FrontArgs &f, uint8_t *smem,
                                                volatile int *abort_flag, int cta, int ncta)
{
    // consumer threads per token: 4 experts each
    if (f.ra.E <= 8) return front_route<2>(tmRX, tmRW, f, smem, abort_flag, cta, ncta);
    if (f.ra.E <= 16) return front_route<4>(tmRX, tmRW, f, smem, abort_flag, cta, ncta);
    return front_route<8>(tmRX, tmRW, f, smem, abort_flag, cta, ncta);
}

// Routing, dispatch and the row copy of the whole-layer launch (E == 8). False when a wait
// gave up.
__device__ __forceinline__ bool fused_front(const CUtensorMap *tmRX, const CUtensorMap *tmRW,
                                            const FusedArgs &fa, uint8_t *smem,
                                            volatile int *abort_flag, int *status, int64_t tmo,
                                            int cta, int ncta)
{
    const FrontArgs &f = fa.front;
    if (!front_route<2>(tmRX, tmRW, f, smem, abort_flag, cta, ncta)) return false;
    // every CTA's routing (top-k and per-group counts) is complete
    if (!grid_barrier(f.gbar, ncta, abort_flag, tmo, status, 350)) return false;
    dispatch_front(f.fd, cta, ncta, cta == 0, reinterpret_cast<int *>(smem));
    // every CTA's rows, indices and (CTA 0) the dispatch outputs are in place
    if (!grid_barrier(f.gbar, 2 * ncta, abort_flag, tmo, status, 351)) return false;
    fence_proxy_async_global(); // x_perm was written by generic stores; layer0 reads it by TMA
    return true;
}

// Offsets of the expert-parallel launch, after every rank's group counts have arrived
// (all CTAs; scratch in shared memory): where each of this rank's pairs goes (destination
// rank and row, into ep.dest / ep.slot), and on CTA 0 this rank's receive-side dispatch
// outputs for its e_loc experts (the tile list of its GEMMs, pad markers) and the cleared
// ready counters of its GEMM phases.
__device__ __forceinline__ void ep_offsets(const FusedArgs &fa, int cta, int ncta, int *scratch)
{
    const EpArgs &ep = fa.ep;
    const FrontArgs &f = fa.front;
    const ScanOut &so = f.fd.so;
    const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31, warp = tid >> 5, nw = nt >> 5;
    const int W = ep.world, E = f.ra.E, EL = ep.e_loc, G = f.n_groups, k = f.ra.k;
    int *tot = scratch;                         // [W][E] rows per source rank and expert
    int *pref = tot + W * E;                    // [G][E] this rank's prefix over its groups
    int *poffD = pref + (size_t)G * E;          // [W][EL + 1] padded offsets of every rank
    int *cntL = poffD + W * (EL + 1);           // [EL] rows of this rank's experts
    int *base = cntL + EL;                      // [E] rows of lower source ranks per expert
    uint32_t *bits = reinterpret_cast<uint32_t *>(base + E); // [E][4] group token bitmap
    const int32_t *ac = ep.all_counts[ep.rank];  // this rank's copy: [W][G][E]
    // 1. totals per source and expert; this rank's exclusive prefix over its groups
    for (int i = warp; i < W * E; i += nw) {
        const int sr = i / E, e = i - sr * E;
        const int32_t *c = ac + (size_t)sr * G * E + e;
        int run = 0;
        for (int g0 = 0; g0 < G; g0 += 32) {
            const int g = g0 + lane;
            const int v = g < G ? c[(size_t)g * E] : 0;
            const int inc = warp_inclusive_scan(v, lane);
            if (sr == ep.rank && g < G) pref[(size_t)g * E + e] = run + inc - v;
            run += __shfl_sync(0xffffffffu, inc, 31);
        }
        if (lane == 0) tot[sr * E + e] = run;
    }
    __syncthreads();
    // 2. every rank's padded offsets (warp d: rank d's experts), the bases, and (CTA 0) the
    //    scan outputs of this rank's experts
    for (int d = warp; d < W; d += nw) {
        int c = 0;
        if (lane < EL)
            for (int sr = 0; sr < W; ++sr) c += tot[sr * E + d * EL + lane];
        if (d == ep.rank && cta == 0) {
            dispatch_scan_warp(c, EL, so, poffD + d * (EL + 1), lane);
        } else {
            const int ntile = (c + M_TILE - 1) / M_TILE;
            const int inc_t = warp_inclusive_scan(ntile, lane);
            if (lane < EL) poffD[d * (EL + 1) + lane] = (inc_t - ntile) * M_TILE;
            if (lane == EL - 1) poffD[d * (EL + 1) + EL] = inc_t * M_TILE;
        }
        if (d == ep.rank && lane < EL) cntL[lane] = c;
    }
    for (int e = tid; e < E; e += nt) {
        int b = 0;
        for (int sr = 0; sr < ep.rank; ++sr) b += tot[sr * E + e];
        base[e] = b;
    }
    if (cta == 0)
        for (int i = tid; i < so.n_ready; i += nt) so.ready[i] = 0;
    __syncthreads();
    if (cta == 0) {
        // pad rows: no token (-1), gate 0, no origin (their layer1 rows are not returned)
        const int *pl = poffD + ep.rank * (EL + 1);
        scan_write_pads(EL, so, pl, cntL, tid, nt);
        long long *org = ep.recv_origin[ep.rank];
        for (int ex = warp; ex < EL; ex += nw)
            for (int r = pl[ex] + cntL[ex] + lane; r < pl[ex + 1]; r += 32) org[r] = -1;
    }
    // 3. destinations of this rank's pairs: rank d = e / e_loc, row = d's padded offset of
    //    the expert + rows of lower source ranks + this rank's earlier groups + the token's
    //    rank in its group
    for (int g = cta; g < G; g += ncta) {
        const int t0 = g * f.ra.tt;
        const int ntg = min(f.ra.tt, f.ra.T - t0);
        for (int i = tid; i < 4 * E; i += nt) bits[i] = 0u;
        __syncthreads();
        const int P = ntg * k;
        const size_t q0 = (size_t)t0 * k;
        for (int q = tid; q < P; q += nt) {
            const int tl = q / k;
            const int e = f.ra.topk_idx[q0 + q];
            if (e >= 0 && e < E) atomicOr(&bits[e * 4 + (tl >> 5)], 1u << (tl & 31));
        }
        __syncthreads();
        for (int q = tid; q < P; q += nt) {
            const int tl = q / k;
            const int e = f.ra.topk_idx[q0 + q];
            if (e < 0 || e >= E) {
                ep.dest[q0 + q] = -1;
                continue;
            }
            const uint32_t *b = bits + e * 4;
            const int wd = tl >> 5;
            int rk = __popc(b[wd] & ((1u << (tl & 31)) - 1u));
            for (int w = 0; w < wd; ++w) rk += __popc(b[w]);
            const int d = e / EL;
            ep.dest[q0 + q] = d;
            ep.slot[q0 + q] = poffD[d * (EL + 1) + (e - d * EL)] + base[e] + pref[(size_t)g * E + e] + rk;
        }
        __syncthreads();
    }
}

// Shared-memory scratch of ep_offsets, in ints.
__host__ __device__ inline int ep_scratch_ints(int world, int E, int e_loc, int n_groups)
{
    return world * E + n_groups * E + world * (e_loc + 1) + e_loc + E + 4 * E;
}

// The front of the expert-parallel launch: routing of this rank's tokens, their group
// counts published to every rank, a barrier of all ranks (each rank's flag in every rank's
// memory), the offsets, and a barrier of this rank's CTAs.
__device__ __forceinline__ bool ep_front(const CUtensorMap *tmRX, const CUtensorMap *tmRW,
                                         const FusedArgs &fa, uint8_t *smem,
                                         volatile int *abort_flag, int *status, int64_t tmo,
                                         int cta, int ncta)
{
    const FrontArgs &f = fa.front;
    const EpArgs &ep = fa.ep;
    const int E = f.ra.E, G = f.n_groups;
    if (!front_route_any(tmRX, tmRW, f, smem, abort_flag, cta, ncta)) return false;
    // this CTA's groups' counts into every rank's copy; CTA 0 clears this rank's receive
    // counters (no rank writes them before this rank's flag is up)
    for (int g = cta; g < G; g += ncta)
        for (int i = threadIdx.x; i < ep.world * E; i += blockDim.x) {
            const int d = i / E, e = i - d * E;
            ep.all_counts[d][((size_t)ep.rank * G + g) * E + e] = f.ra.group_counts[(size_t)g * E + e];
        }
    if (cta == 0)
        for (int i = threadIdx.x; i < ep.max_tiles; i += blockDim.x) ep.arrive[ep.rank][i] = 0;
    {
        const int64_t n = (int64_t)fa.T * fa.l1.n_tiles;
        for (int64_t i = (int64_t)cta * blockDim.x + threadIdx.x; i < n; i += (int64_t)ncta * blockDim.x)
            ep.back_cnt[ep.rank][i] = 0;
    }
    if (!grid_barrier(f.gbar, ncta, abort_flag, tmo, status, 360, true)) return false;
    // every rank: its counts are everywhere and its receive counters are clear
    if (cta == 0 && threadIdx.x == 0) {
        __threadfence_system();
        for (int d = 0; d < ep.world; ++d) st_release_sys(ep.flags[d] + ep.rank, ep.epoch);
    }
    int ok = 1;
    if (threadIdx.x == 0)
        for (int sr = 0; sr < ep.world && ok; ++sr)
            ok = flag_wait_bounded<true>(ep.flags[ep.rank] + sr, ep.epoch, abort_flag, tmo, status, 361) ? 1 : 0;
    if (!__syncthreads_and(ok)) return false;
    ep_offsets(fa, cta, ncta, reinterpret_cast<int *>(smem));
    return grid_barrier(f.gbar, 2 * ncta, abort_flag, tmo, status, 362);
}

// The scatter of the expert-parallel launch (after ep_front), by the CTA's eight epilogue and
// data-movement warps (`dw` 0..7, meeting at named barrier `bar`; no layer0 tile can start
// before the rows arrive, so the epilogue warps are free): every pair of this CTA's groups
// sends its token's x row, gate and origin to its destination row; after all of them (the
// barrier), warp 0 of the eight fences at system scope once -- the barrier puts every lane's
// stores before that fence -- and adds each pair to its destination tile's arrival count, so
// the destination's layer0 may read a tile once its count is complete.
__device__ __forceinline__ void ep_scatter(const FusedArgs &fa, int cta, int ncta, int dw, int lane,
                                           int bar)
{
    constexpr int NW = 8;
    const EpArgs &ep = fa.ep;
    const FrontArgs &f = fa.front;
    const int k = f.ra.k, H = f.fd.H, G = f.n_groups;
    const int chunks = H / 8;
    auto valid = [&](size_t q, int &d, int &slot) {
        d = ep.dest[q];
        slot = ep.slot[q];
        return d >= 0 && d < ep.world && slot >= 0 && (int64_t)slot < ep.recv_cap;
    };
    for (int g = cta; g < G; g += ncta) {
        const int t0 = g * f.ra.tt;
        const int P = min(f.ra.tt, f.ra.T - t0) * k;
        const size_t q0 = (size_t)t0 * k;
        for (int qq = dw; qq < P; qq += NW) {
            const size_t q = q0 + qq;
            int d, slot;
            if (!valid(q, d, slot)) continue;
            const int t = (int)(q / k);
            const uint4 *src = reinterpret_cast<const uint4 *>(f.fd.x + (size_t)t * H);
            uint4 *dst = reinterpret_cast<uint4 *>(ep.recv_rows[d] + (size_t)slot * H);
            // a lane's 16-byte pieces of the row, 16 loads in flight before the stores
            int c = lane;
            for (; c + 15 * 32 < chunks; c += 16 * 32) {
                uint4 v[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) v[i] = src[c + i * 32];
#pragma unroll
                for (int i = 0; i < 16; ++i) dst[c + i * 32] = v[i];
            }
            for (; c < chunks; c += 32) dst[c] = src[c];
            if (lane == 0) {
                ep.recv_gate[d][slot] = f.ra.topk_w[q];
                ep.recv_origin[d][slot] = ((long long)ep.rank << 32) | (long long)q;
            }
        }
    }
    named_bar_sync(bar, NW * 32);
    if (dw != 0) return;
    __threadfence_system();
    for (int g = cta; g < G; g += ncta) {
        const int t0 = g * f.ra.tt;
        const int P = min(f.ra.tt, f.ra.T - t0) * k;
        const size_t q0 = (size_t)t0 * k;
        for (int qq = lane; qq < P; qq += 32) {
            int d, slot;
            if (valid(q0 + qq, d, slot)) red_relaxed_sys_add(ep.arrive[d] + (slot >> 7), 1);
        }
    }
}

struct FusedItem {
    int phase; // 0 layer0, 1 layer1
    int e, mt, nt;
};

__device__ __forceinline__ FusedItem fused_item(int w, const FusedArgs &fa, int total0)
{
    FusedItem it{};
    if (w < total0) {
        it.phase = 0;
        gemm_map_work(w, fa.l0, it.e, it.mt, it.nt);
    } else {
        it.phase = 1;
        gemm_map_work(w - total0, fa.l1, it.e, it.mt, it.nt);
    }
    return it;
}

// Bounded wait until the layer1 tiles (stripe `stripe`) that hold the k rows of eight tokens
// t[0..7] are all stored: lane q checks row (token q & 7, selection q >> 3) and the warp votes,
// so one round of loads covers all 8 k flags. The rows are the same for every lane; the warp
// barrier after the vote orders every lane's later loads after the lanes' acquires.
__device__ __forceinline__ bool combine_rows_ready(const FusedArgs &fa, const int *flags, const int (&t)[8],
                                                   int stripe, int lane, volatile int *abort_flag,
                                                   int *status)
{
    const uint64_t t_start = globaltimer_ns();
    uint32_t nap = 64;
    const bool ep = fa.ep.world > 0;
#pragma unroll 1
    while (true) {
        bool ready = true;
        if (ep) {
            // expert parallelism: this stripe of the token's k rows has come back
            if (lane < 8) {
                const int tok = t[0] + lane * 4;
                if (tok < fa.T &&
                    ld_acquire_sys(fa.ep.back_cnt[fa.ep.rank] + (size_t)tok * fa.l1.n_tiles + stripe) < fa.k)
                    ready = false;
            }
        } else {
            for (int q = lane; q < 8 * fa.k; q += 32) {
                const int tok = t[0] + (q & 7) * 4; // t[i] = t[0] + 4 i
                if (tok >= fa.T) continue;
                const int rr = fa.inv_pos[(size_t)tok * fa.k + (q >> 3)];
                if (rr < 0 || (int64_t)rr >= fa.ys_rows || (rr >> 7) >= fa.max_tiles) continue;
                if (ld_acquire_gpu(flags + (rr >> 7)) == 0) ready = false;
            }
        }
        if (__all_sync(0xffffffffu, ready)) break;
        if (*abort_flag) return false;
        if ((int64_t)(globaltimer_ns() - t_start) > fa.l0.timeout_ns) {
            *abort_flag = 1;
            record_status(status, DEV_TIMEOUT, 332);
            return false;
        }
        __nanosleep(nap);
        if (nap < 1024) nap <<= 1;
    }
    __syncwarp();
    return true;
}

// Combine of one item (256-column stripe x comb_tokens tokens) by a group of four warps:
// warp wq (0..3) takes tokens wq, wq + 4, ... of the block, eight at a time; lane l owns
// columns stripe*256 + 8l .. +7. For each group of eight tokens it waits until the layer1
// tiles holding their rows are stored, then loads the rows two selections at a time (16
// loads in flight per lane) and sums over j ascending in fp32 with one bf16 rounding.
// Returns false when a wait gave up (timeout or abort).
__device__ __forceinline__ bool fused_combine(const FusedArgs &fa, int stripe, int chunk, int wq,
                                              int lane, volatile int *abort_flag, int *status)
{
    const int col = stripe * gemm::BN + lane * 8;
    const bool have_col = col < fa.H;
    const bool ep = fa.ep.world > 0;
    // expert parallelism: the returned rows, row t * k + j of the rank's own buffer
    const __nv_bfloat16 *ys = ep ? fa.ep.back[fa.ep.rank] : fa.l1.out;
    const int *flags = fa.ready1 + (size_t)stripe * fa.max_tiles;
    for (int g = 0; g < fa.comb_tokens / 32; ++g) {
        int t[8];
        float a[8][8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            t[i] = chunk * fa.comb_tokens + g * 32 + i * 4 + wq;
#pragma unroll
            for (int c = 0; c < 8; ++c) a[i][c] = 0.0f;
        }
        if (t[0] >= fa.T) break; // the block's remaining groups are past the batch
        if (!combine_rows_ready(fa, flags, t, stripe, lane, abort_flag, status)) return false;
        for (int j0 = 0; j0 < fa.k; j0 += 2) {
            uint4 u[2][8];
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) {
                const int j = j0 + jj;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    u[jj][i] = make_uint4(0u, 0u, 0u, 0u);
                    if (j < fa.k && t[i] < fa.T) {
                        const int r = ep ? t[i] * fa.k + j : fa.inv_pos[(size_t)t[i] * fa.k + j];
                        if (ep || (r >= 0 && (int64_t)r < fa.ys_rows && (r >> 7) < fa.max_tiles)) {
                            if (have_col)
                                u[jj][i] = *reinterpret_cast<const uint4 *>(ys + (size_t)r * fa.H + col);
                        } else if (lane == 0) {
                            record_status(status, DEV_BAD_INDEX, 331);
                        }
                    }
                }
            }
            // j ascending: the first selection of the pair, then the second
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) {
                if (j0 + jj >= fa.k) break;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    a[i][0] += bf16_lo(u[jj][i].x); a[i][1] += bf16_hi(u[jj][i].x);
                    a[i][2] += bf16_lo(u[jj][i].y); a[i][3] += bf16_hi(u[jj][i].y);
                    a[i][4] += bf16_lo(u[jj][i].z); a[i][5] += bf16_hi(u[jj][i].z);
                    a[i][6] += bf16_lo(u[jj][i].w); a[i][7] += bf16_hi(u[jj][i].w);
                }
            }
        }
        if (!have_col) continue;
        if (fa.ys_shared != nullptr) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                if (t[i] >= fa.T) continue;
                const uint4 u = *reinterpret_cast<const uint4 *>(fa.ys_shared + (size_t)t[i] * fa.H + col);
                a[i][0] += bf16_lo(u.x); a[i][1] += bf16_hi(u.x);
                a[i][2] += bf16_lo(u.y); a[i][3] += bf16_hi(u.y);
                a[i][4] += bf16_lo(u.z); a[i][5] += bf16_hi(u.z);
                a[i][6] += bf16_lo(u.w); a[i][7] += bf16_hi(u.w);
            }
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            if (t[i] >= fa.T) continue;
            uint4 o;
            o.x = pack_bf16x2(a[i][0], a[i][1]);
            o.y = pack_bf16x2(a[i][2], a[i][3]);
            o.z = pack_bf16x2(a[i][4], a[i][5]);
            o.w = pack_bf16x2(a[i][6], a[i][7]);
            *reinterpret_cast<uint4 *>(fa.out + (size_t)t[i] * fa.H + col) = o;
        }
    }
    return true;
}

// Combine items from the launch-wide queue (stripe-major), taken one at a time by a group of
// four warps (128 threads meeting at named barrier `bar`): the group's first thread claims
// the next item with an atomic and shares it through shared memory. Returns false on abort.
__device__ __forceinline__ bool combine_queue(const FusedArgs &fa, int group_warp, int lane, int bar,
                                              volatile int *slot, volatile int *abort_flag,
                                              int *status)
{
    const int nchunk = (fa.T + fa.comb_tokens - 1) / fa.comb_tokens;
    const int total2 = fa.l1.n_tiles * nchunk;
    bool ok = true;
    while (true) {
        if (group_warp == 0 && lane == 0) *slot = atomicAdd(fa.comb_next, 1);
        named_bar_sync(bar, 128);
        const int j = *slot;
        named_bar_sync(bar, 128); // everyone has read the slot before it is overwritten
        if (j >= total2 || !ok) break;
        const uint64_t t_begin = globaltimer_ns();
        ok = fused_combine(fa, j / nchunk, j % nchunk, group_warp, lane, abort_flag, status);
        // a group stops only together: vote at the next claim
        ok = named_bar_and(bar, 128, ok);
        if (ok && group_warp == 0 && lane == 0) trace_record(fa, TRACE_COMBINE, j, t_begin, globaltimer_ns());
        if (!ok) break;
    }
    return ok;
}

// The persistent layer launch on CTAs cta = 0 .. ncta - 1 (one per SM, all resident).
// MODE: FUSED_LAYERS layer0 -> layer1 -> combine; FUSED_WHOLE routes and dispatches the
// tokens first (router maps tmRX, tmRW); FUSED_EP is the expert-parallel layer of one rank
// (ep_front, then the data-movement warps scatter the rank's rows to their experts' ranks
// while the GEMM pipeline runs the rank's experts on the rows that have arrived, layer1
// returns each gated row to its origin, and the combine sums the rows that came back).
template <int KIND0, int MODE>
__device__ __forceinline__ void fused_layer_body(const CUtensorMap &tmA0, const CUtensorMap &tmW1,
                                                 const CUtensorMap &tmH, const CUtensorMap &tmW2,
                                                 const CUtensorMap &tmRX, const CUtensorMap &tmRW,
                                                 const FusedArgs &fa, int cta, int ncta)
{
    using namespace gemm;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + STAGES * STAGE);
    const uint32_t bar0 = smem_u32(bars);
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
    auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + a); };
    auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + 2 + a); };
    const uint32_t done_bar = bar0 + 8u * (2 * STAGES + 4);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + NUM_BARS);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    // [4] ring of part counters, then the two combine groups' claimed-item slots (inside the
    // shared-memory allocation: the GEMM's column-scale buffers, unused here, follow)
    int *warps_done = reinterpret_cast<int *>(tmem_slot + 2);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const GemmArgs &l0 = fa.l0;
    const GemmArgs &l1 = fa.l1;
    int *status = l0.status;
    const int64_t tmo = l0.timeout_ns;
    const bool a_tma = fa.a_tma != 0;
    // layer0 epilogue parts: warps 2..5, and with A by TMA also warps 6..9 (half the chunks
    // each; not in the expert-parallel launch, whose data-movement warps scatter rows then)
    const bool split0 = a_tma && MODE != FUSED_EP;
    const int parts0 = split0 ? 8 : 4;
    const int nch0 = (KIND0 == GEMM_SWIGLU) ? 4 : BN / 32;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            // TMA arrive (+ one per gather thread when layer0 rows are gathered in the kernel;
            // the producer adds those arrivals itself for layer1 stages)
            mbar_init(full_bar(s), a_tma ? 1 : 1 + GATHER_THREADS);
            mbar_init(empty_bar(s), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(tfull_bar(a), 1);
            mbar_init(tempty_bar(a), parts0);
        }
        mbar_init(done_bar, 1);
        *abort_flag = 0;
        for (int i = 0; i < 4; ++i) warps_done[i] = 0;
        fence_mbar_init();
        if (a_tma) tma_prefetch_desc(&tmA0);
        tma_prefetch_desc(&tmW1);
        tma_prefetch_desc(&tmH);
        tma_prefetch_desc(&tmW2);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    bool front_ok = true;
    const uint64_t t_launch = globaltimer_ns();
    if constexpr (MODE == FUSED_WHOLE)
        front_ok = fused_front(&tmRX, &tmRW, fa, smem, abort_flag, status, tmo, cta, ncta);
    if constexpr (MODE == FUSED_EP)
        front_ok = ep_front(&tmRX, &tmRW, fa, smem, abort_flag, status, tmo, cta, ncta);
    if (MODE != FUSED_LAYERS && front_ok && threadIdx.x == 0)
        trace_record(fa, TRACE_FRONT, cta, t_launch, globaltimer_ns());

    const int num_tiles = front_ok ? l0.meta->num_tiles : 0;
    const int total0 = num_tiles * l0.n_tiles;
    const int total = total0 + num_tiles * l1.n_tiles;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer ----------------
            int s = 0;
            uint32_t ph = 0;
            int armed[STAGES];
#pragma unroll
            for (int i = 0; i < STAGES; ++i) armed[i] = -1;
            bool ok = true;
            bool all0 = false; // every layer0 item finished: no more per-tile waits
            for (int w = cta; ok && w < total; w += ncta) {
                const FusedItem it = fused_item(w, fa, total0);
                if (MODE == FUSED_EP && it.phase == 0) {
                    // the tile's rows have arrived from their source ranks (count per M tile)
                    const int first = l0.tile_off[it.e];
                    const int need = min(BM, l0.expert_rows[it.e] - (it.mt - first) * BM);
                    if (!flag_wait_bounded<true>(fa.ep.arrive[fa.ep.rank] + it.mt, need, abort_flag, tmo,
                                                 status, 363)) {
                        ok = false;
                        break;
                    }
                    fence_proxy_async_global(); // rows written by generic stores, read by TMA
                }
                if (it.phase == 1) {
                    // layer1 needs every layer0 column tile of its M tile
                    if (!all0) all0 = ld_acquire_gpu(fa.done0) >= total0;
                    if (!all0 && !flag_wait_bounded(fa.ready0 + it.mt, l0.n_tiles, abort_flag, tmo,
                                                    status, 300)) {
                        ok = false;
                        break;
                    }
                    fence_proxy_async_global(); // h was written by generic stores
                }
                const int KB = it.phase == 0 ? l0.k_blocks : l1.k_blocks;
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait_bounded(empty_bar(s), ph ^ 1u, abort_flag, tmo, status, 301)) {
                        ok = false;
                        break;
                    }
                    const uint32_t a_dst = smem_u32(smem + s * STAGE);
                    const uint32_t b_dst = a_dst + A_TILE;
                    const bool a_here = it.phase == 1 || a_tma;
                    mbar_arrive_expect_tx(full_bar(s), a_here ? STAGE : B_TILE);
                    // layer1 stages when layer0 gathers: the gather warps do not arrive
                    if (it.phase == 1 && !a_tma) mbar_arrive_cnt(full_bar(s), GATHER_THREADS);
                    armed[s] = (int)ph;
                    if (it.phase == 0) {
                        if (a_tma) tma_load_2d(a_dst, &tmA0, full_bar(s), kb * BK, it.mt * BM);
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            int col;
                            if (KIND0 == GEMM_SWIGLU)
                                col = (i < 2 ? it.nt * 128 + i * 64
                                             : l0.up_col + it.nt * 128 + (i - 2) * 64);
                            else
                                col = it.nt * BN + i * 64;
                            tma_load_3d(b_dst + i * B_BOX, &tmW1, full_bar(s), col, kb * BK, it.e);
                        }
                    } else {
                        tma_load_2d(a_dst, &tmH, full_bar(s), kb * BK, it.mt * BM);
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            tma_load_3d(b_dst + i * B_BOX, &tmW2, full_bar(s), it.nt * BN + i * 64,
                                        kb * BK, it.e);
                    }
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            for (int i = 0; i < STAGES; ++i)
                if (armed[i] >= 0) {
                    volatile int never = 0;
                    mbar_wait_bounded(full_bar(i), (uint32_t)armed[i], &never, tmo, nullptr, 0);
                }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- MMA issuer ----------------
            int s = 0;
            uint32_t ph = 0;
            int n = 0; // accumulator tiles issued
            bool ok = true;
            for (int w = cta; ok && w < total; w += ncta) {
                const FusedItem it = fused_item(w, fa, total0);
                const int acc = n & 1;
                const uint32_t aph = (uint32_t)(n >> 1) & 1u;
                if (!mbar_wait_bounded(tempty_bar(acc), aph ^ 1u, abort_flag, tmo, status, 310)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
                const int KB = it.phase == 0 ? l0.k_blocks : l1.k_blocks;
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait_bounded(full_bar(s), ph, abort_flag, tmo, status, 311)) {
                        ok = false;
                        break;
                    }
                    // gathered rows arrive through the generic proxy
                    if (it.phase == 0 && !a_tma) fence_proxy_async_smem();
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smem + s * STAGE);
                    const uint32_t b_addr = a_addr + A_TILE;
                    const uint64_t a_desc = sw128_desc(a_addr, A_LBO, A_SBO);
                    const uint64_t b_desc = sw128_desc(b_addr, B_LBO, B_SBO);
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k)
                        umma_bf16(d_tmem, a_desc + (uint64_t)((k * 32) >> 4),
                                  b_desc + (uint64_t)((k * 16 * 128) >> 4), IDESC,
                                  (kb | k) != 0 ? 1u : 0u);
                    umma_commit(empty_bar(s));
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (!ok) break;
                umma_commit(tfull_bar(acc));
                ++n;
            }
            umma_commit(done_bar);
            volatile int never = 0;
            mbar_wait_bounded(done_bar, 0, &never, tmo, status, 312);
        }
    } else {
        // ---------------- epilogue warps 2..5 and data-movement warps 6..9 ----------------
        const bool dm = warp >= 6;
        if (MODE == FUSED_EP && front_ok) {
            // expert parallelism: all eight send this rank's rows out first (named barrier 4)
            const uint64_t t_sc = globaltimer_ns();
            ep_scatter(fa, cta, ncta, warp - 2, lane, 4);
            if (warp == 2 && lane == 0) trace_record(fa, TRACE_SCATTER, cta, t_sc, globaltimer_ns());
        }
        const int q = warp & 3; // TMEM lanes 32q .. 32q+31
        int n = 0;
        bool ok = true;
        // gather mode: ring position of the data-movement warps (layer0 stages only)
        int gs = 0;
        uint32_t gph = 0;
        const int g = threadIdx.x - NUM_THREADS;
        for (int w = cta; ok && w < total; w += ncta) {
            const FusedItem it = fused_item(w, fa, total0);
            // the data-movement warps serve layer0 items only (none in the expert-parallel launch)
            if (dm && (it.phase == 1 || MODE == FUSED_EP)) break;
            if (dm && !a_tma) {
                // ---- A-row gather for a layer0 item (cp.async): thread g copies 16-byte chunk
                // (g & 7) of rows (g >> 3) + 16 i; its 8 token ids are read once per tile and
                // kept in registers (Comet §4: row indices cached in registers)
                const int chunk = g & 7;
                const int r0 = g >> 3;
                const __nv_bfloat16 *src[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int64_t r = (int64_t)it.mt * BM + r0 + 16 * i;
                    int t = (r < l0.gather_len) ? l0.gather_idx[r] : -1;
                    if (t < 0 || t >= l0.gather_rows) t = 0;
                    src[i] = l0.gather_src + (size_t)t * l0.gather_ld + chunk * 8;
                }
                for (int kb = 0; kb < l0.k_blocks; ++kb) {
                    ok = mbar_wait_bounded(empty_bar(gs), gph ^ 1u, abort_flag, tmo, status, 320);
                    if (!__all_sync(0xffffffffu, ok)) {
                        ok = false;
                        break;
                    }
                    const uint32_t a_dst = smem_u32(smem + gs * STAGE);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int r = r0 + 16 * i;
                        cp_async_16_cg(a_dst + r * 128 + ((chunk ^ (r & 7)) << 4), src[i] + kb * BK);
                    }
                    cp_async_arrive_noinc(full_bar(gs));
                    if (++gs == STAGES) {
                        gs = 0;
                        gph ^= 1u;
                    }
                }
                continue;
            }
            // ---- epilogue of a GEMM item (warps 2..5; warps 6..9 for the second half of a
            // layer0 tile when its A rows came by TMA)
            const int acc = n & 1;
            const uint32_t aph = (uint32_t)(n >> 1) & 1u;
            ok = mbar_wait_bounded(tfull_bar(acc), aph, abort_flag, tmo, status, 340);
            if (!__all_sync(0xffffffffu, ok)) {
                ok = false;
                break;
            }
            const uint64_t t_begin = globaltimer_ns();
            tc_fence_after();
            const int row = it.mt * BM + q * 32 + lane;
            const uint32_t t_row = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN);
            if (it.phase == 0) {
                const int c_lo = (split0 && dm) ? nch0 / 2 : 0;
                const int c_hi = split0 ? c_lo + nch0 / 2 : -1;
                epilogue_rows<KIND0>(l0, t_row, row, it.nt, 0, 0, nullptr, c_lo, c_hi);
            } else {
                epilogue_rows<GEMM_SCALE>(l1, t_row, row, it.nt);
            }
            // The accumulator is free as soon as its TMEM reads are done (layer1 items with
            // eight epilogue parts configured: warps 2..5 stand for 6..9).
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive_cnt(tempty_bar(acc), (it.phase == 1 && split0) ? 2u : 1u);
            if (MODE == FUSED_EP && it.phase == 1) {
                // the row's stripe went to its origin: count it there once it is visible
                // (after the accumulator is released, so the MMA warp does not wait for it)
                const long long o = l1.row_dst[row];
                if (o >= 0) {
                    __threadfence_system();
                    const int q = (int)(o & 0xffffffffll);
                    red_relaxed_sys_add(fa.ep.back_cnt[(int)(o >> 32)] + (size_t)(q / fa.k) * l1.n_tiles + it.nt, 1);
                }
            }
            // Ready signal: every part makes its stores visible, then the last of the item's
            // parts publishes it. The part counters form a ring of 4 indexed by the CTA's item
            // count: slot n & 3 is reused by item n + 4, whose parts can only arrive after
            // every warp (this one included) has finished item n + 2.
            __threadfence();
            __syncwarp();
            if (lane == 0) {
                const int parts = it.phase == 0 ? parts0 : 4;
                const int prev = atomicAdd(&warps_done[n & 3], 1);
                if (prev == parts - 1) {
                    warps_done[n & 3] = 0;
                    __threadfence();
                    if (it.phase == 0) {
                        if (w != fa.fault_skip) {
                            fence_proxy_async_global();
                            red_release_gpu_add(fa.ready0 + it.mt, 1);
                            red_release_gpu_add(fa.done0, 1);
                        }
                    } else {
                        st_release_gpu(fa.ready1 + (size_t)it.nt * fa.max_tiles + it.mt, 1);
                    }
                    trace_record(fa, it.phase == 0 ? TRACE_L0 : TRACE_L1, w, t_begin, globaltimer_ns());
                }
            }
            ++n;
        }
        if (dm && !a_tma) cp_async_wait_all(); // this thread's copies land first
        // expert parallelism: the data-movement warps send this rank's rows out first

        // combine: the data-movement warps from the end of their layer0 duties (beside the
        // layer1 GEMM pipeline), the epilogue warps once this CTA's GEMM items are done
        // (each group of four warps decides together whether to go on: named barrier 2 for
        // the data-movement warps, 3 for the epilogue warps)
        volatile int *slots = reinterpret_cast<volatile int *>(warps_done + 4);
        const int bar = dm ? 2 : 3;
        if (named_bar_and(bar, 128, ok && front_ok) && fa.comb_in_launch)
            combine_queue(fa, dm ? warp - 6 : warp - 2, lane, bar, slots + (dm ? 0 : 1), abort_flag,
                          status);
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

// FRONT: the launch also routes and dispatches the tokens first (the whole layer in one
// launch; its router tensor maps tmRX, tmRW are used only then).
template <int KIND0, bool FRONT>
__global__ void __launch_bounds__(gemm::NUM_THREADS_GATHER, 1)
    moe_fused_layer_kernel(const __grid_constant__ CUtensorMap tmA0,
                           const __grid_constant__ CUtensorMap tmW1,
                           const __grid_constant__ CUtensorMap tmH,
                           const __grid_constant__ CUtensorMap tmW2,
                           const __grid_constant__ CUtensorMap tmRX,
                           const __grid_constant__ CUtensorMap tmRW, const FusedArgs fa)
{
    fused_layer_body<KIND0, FRONT ? FUSED_WHOLE : FUSED_LAYERS>(tmA0, tmW1, tmH, tmW2, tmRX, tmRW, fa,
                                                               blockIdx.x, gridDim.x);
}

// The expert-parallel layer: one launch per GPU, each GPU a rank; or, to exercise several
// ranks on one GPU, one launch holding n_local ranks (CTA b plays rank b % n_local; the
// ranks' buffers all live on this GPU, and their waits on one another stay inside the
// launch, whose CTAs are all resident).
constexpr int EP_MAX_LOCAL = 4;
struct EpRankMaps {
    CUtensorMap a0, w1, h, w2, rx, rw;
};
struct EpLaunch {
    EpRankMaps maps[EP_MAX_LOCAL];
    FusedArgs fa[EP_MAX_LOCAL];
    int n_local;
};

template <int KIND0>
__global__ void __launch_bounds__(gemm::NUM_THREADS_GATHER, 1)
    moe_ep_layer_kernel(const __grid_constant__ EpLaunch L)
{
    const int nl = L.n_local;
    const int r = (int)(blockIdx.x % (unsigned)nl);
    const EpRankMaps &m = L.maps[r];
    fused_layer_body<KIND0, FUSED_EP>(m.a0, m.w1, m.h, m.w2, m.rx, m.rw, L.fa[r],
                                      (int)(blockIdx.x / (unsigned)nl), (int)(gridDim.x / (unsigned)nl));
}

} // namespace moe
