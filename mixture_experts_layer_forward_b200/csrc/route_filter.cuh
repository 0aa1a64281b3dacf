// route_filter.cuh -- exact top-k routing for many experts with a tensor-core filter.
//
// The routing decision is defined on the sequential fp32 logits l[t][e] (one accumulator,
// h ascending, then + bias; see route.cuh). For large E computing all T*E of them that way
// costs T*E*H dependent FMAs. Instead:
//   1. route_filter_prep_kernel: W_g^T (expert rows, for streaming) and partial sums of
//      squares of every W_g column;
//   2. m = x . W_g on the tensor cores (GEMM_LOGITS in gemm_tc.cuh), K split into S ranges
//      of at most hs values; the S fp32 partial products are summed here in fixed order;
//   3. route_filter_exact_kernel, per block of bt tokens:
//      a. an interval [m - eta, m + eta] (m including the bias) that holds l, with
//           eta = cA ||x_t|| ||w_e|| + 4 u (|m| + 1),  u = 2^-24,
//           cA  = 1.25 (H + 4 hs + S + 4) u.
//         ||x_t|| ||w_e|| bounds A = sum_h |x_h w_he| (Cauchy-Schwarz; both norms rounded
//         up). The sequential fp32 chain is within 1.01 H u A of the exact dot product (every
//         product of two bf16 values is exact in fp32, one rounding per step); the tensor-core
//         partial of a K range of n values is assumed within 4 n u A_range of it (an adder
//         that aligns to the largest addend with a 24-bit window and truncates stays near
//         2.3 n u), and the S partials are summed with S u A; the last term covers the bias
//         additions and the rounding of the interval ends; 1.25 is margin;
//      b. an expert whose upper end is below the k-th largest lower end L cannot be in the
//         top k: the k experts holding the k largest lower ends have exact logits >= L, all
//         strictly above the excluded one's. The rest are the candidates;
//      c. every candidate (token, expert) pair gets its exact sequential logit. A producer
//         thread streams 64-value chunks through a ring: per chunk one 2D TMA box of the
//         block's x rows and the W_g^T rows of the candidates' id range (64-row boxes),
//         128-byte swizzled, completion counted on mbarriers; in eight consumer warps a
//         thread owns two candidates of one token, so one x load serves two chains;
//      d. top k among the candidates' exact logits, ties to the lower expert id, and the gates
//         from those exact logits, in the same arithmetic as route_topk_kernel.
// Hence the selection, its order and the gates equal those of the full sequential router.
#pragma once

#include "ptx.cuh"
#include "route.cuh"

namespace moe {

constexpr int RF_CWARPS = 8;                 // consumer warps (pair chains)
constexpr int RF_CTHREADS = RF_CWARPS * 32;
constexpr int RF_WARPS = RF_CWARPS + 1;      // + one producer warp (TMA, one thread)
constexpr int RF_THREADS = RF_WARPS * 32;
constexpr int RF_HC = 64;                    // h values per streamed chunk: 128-byte rows,
                                             // 16-byte column v of row r at (v ^ (r & 7))
constexpr int RF_WBOX = 64;                  // W_g^T rows per TMA box (8 KB)
constexpr int RF_NS_MAX = 16;                // deepest chunk ring
constexpr int RF_MAX_BT = 32;                // tokens per block
constexpr int RF_BLOCKS_PER_SM = 2;          // blocks the token split aims to co-schedule
constexpr int RF_MAX_E = 512;
constexpr int RF_SPLIT_MAX = 16;
constexpr int RF_SLAB = 256;                 // h values per partial sum of squares of W_g
constexpr int RF_SMEM_MAX = 232448;

__device__ __forceinline__ float rf_norm_up(float ss, int n)
{
    // sqrt of an fp32 sum of n squares, scaled up past its rounding error
    return sqrtf(ss) * (1.0f + (float)(n + 2) * 5.9604645e-8f);
}

// order-preserving int key of a float (for warp max/min reductions), and back
__device__ __forceinline__ int rf_key(float f)
{
    const int i = __float_as_int(f);
    return i >= 0 ? i : (i ^ 0x7fffffff);
}
__device__ __forceinline__ float rf_unkey(int k) { return __int_as_float(k >= 0 ? k : (k ^ 0x7fffffff)); }

// Two chains that share the x word: acc0 += x.lo * a.lo, then x.hi * a.hi; acc1 likewise with
// b. bf16 halves of 32-bit words; each product is exact and each addition is rounded once to
// fp32 (the arithmetic of fmaf on the widened values).
__device__ __forceinline__ void fma2x2_bf16(uint32_t x, uint32_t a, uint32_t b, float &acc0,
                                            float &acc1)
{
    asm("{\n\t.reg .b16 xl, xh, al, ah, bl, bh;\n\t"
        "mov.b32 {xl, xh}, %2;\n\t"
        "mov.b32 {al, ah}, %3;\n\t"
        "mov.b32 {bl, bh}, %4;\n\t"
        "fma.rn.f32.bf16 %0, xl, al, %0;\n\t"
        "fma.rn.f32.bf16 %1, xl, bl, %1;\n\t"
        "fma.rn.f32.bf16 %0, xh, ah, %0;\n\t"
        "fma.rn.f32.bf16 %1, xh, bh, %1;\n\t}"
        : "+f"(acc0), "+f"(acc1)
        : "r"(x), "r"(a), "r"(b));
}

// Grid (E/8, ceil(H/RF_SLAB)): W_g^T[e][h] = W_g[h][e] and, per slab of RF_SLAB rows,
// wpart[slab][e] = sum of W_g[h][e]^2 over the slab. Also clears the status word of the call.
__global__ void __launch_bounds__(256)
    route_filter_prep_kernel(const __nv_bfloat16 *__restrict__ Wg, int H, int E,
                             uint16_t *__restrict__ WgT, float *__restrict__ wpart, int *status)
{
    __shared__ float red[8][8];
    if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0 && status != nullptr) {
        status[0] = DEV_OK; // a new call starts with a clean status word
        status[1] = 0;
    }
    const int e0 = blockIdx.x * 8;
    const int h = blockIdx.y * RF_SLAB + threadIdx.x;
    float ss[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) ss[j] = 0.0f;
    if (h < H) {
        const uint4 u = *reinterpret_cast<const uint4 *>(Wg + (size_t)h * E + e0);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint32_t b = (j & 1) ? (w[j >> 1] >> 16) : (w[j >> 1] & 0xffffu);
            const float v = __uint_as_float(b << 16);
            ss[j] = v * v;
            WgT[(size_t)(e0 + j) * H + h] = (uint16_t)b;
        }
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        float v = ss[j];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        if (lane == 0) red[warp][j] = v;
    }
    __syncthreads();
    if (threadIdx.x < 8) {
        float v = 0.0f;
        for (int w = 0; w < 8; ++w) v += red[w][threadIdx.x];
        wpart[(size_t)blockIdx.y * E + e0 + threadIdx.x] = v;
    }
}

// The exact kernel also takes two tensor maps: x [T, H] with bt-row boxes and W_g^T [E, H]
// with RF_WBOX-row boxes, both 64 columns wide, 128-byte swizzle.
struct RfArgs {
    const float *wpart;       // [ceil(H / RF_SLAB), E] partial sums of squares of W_g
    const float *xsq;         // [S, T] partial sums of squares of the x rows
    const float *bias;        // [E] or nullptr
    const float *parts;       // [S, E, T] tensor-core partials (column-major)
    int32_t *topk_idx;        // [T, k]
    float *topk_w;            // [T, k]
    int T, H, E, k, S, bt;
    int ring_bytes;           // bytes of the chunk ring (region 0)
    float cA;                 // interval coefficient of ||x|| ||w||
    int gate;                 // MOE_GATE_SOFTMAX_TOPK, or 2: the bias steers the selection only
    int *status;
    int64_t timeout_ns;
};

// Shared memory of route_filter_exact_kernel (from a 1024-byte aligned base). Region 0 holds
// the filter logits [bt][E + 1], then the chunk ring; the exact logits of the candidates
// have their own [bt][E].
__host__ __device__ inline size_t rf_region0_bytes(int bt, int E, int ring_bytes)
{
    const size_t mrow = (size_t)bt * (E + 1) * 4;
    const size_t r = (size_t)ring_bytes > mrow ? (size_t)ring_bytes : mrow;
    return (r + 1023) & ~(size_t)1023;
}
__host__ __device__ inline size_t rf_smem_bytes(int bt, int E, int ring_bytes)
{
    const int ew = (E + 31) / 32;
    return 1024 /*alignment slack*/ + rf_region0_bytes(bt, E, ring_bytes) +
           (size_t)bt * E * 4 /*exact*/ + 2 * RF_NS_MAX * 8 /*mbarriers*/ +
           (size_t)E * 4 /*wn*/ + (size_t)bt * ew * 4 /*cand*/ +
           (size_t)(RF_MAX_BT + 1) * 4 * 2 /*tok_off, unit_off*/ + 16 /*range, abort*/;
}
// Bytes of one ring stage: the x box (bt rows, padded to 1024 bytes for the swizzle) and
// nbw W_g^T boxes.
__host__ __device__ inline int rf_stage_bytes(int bt, int nbw)
{
    return ((bt * 128 + 1023) & ~1023) + nbw * RF_WBOX * 128;
}
// Smallest ring that holds two chunks when the candidates span every expert.
__host__ __device__ inline int rf_ring_min(int bt, int E)
{
    return 2 * rf_stage_bytes(bt, (E + RF_WBOX - 1) / RF_WBOX);
}

// r-th set bit (r >= 0) of the candidate words of one token; E when there is none
__device__ __forceinline__ int rf_nth_bit(const uint32_t *words, int ew, int r, int E)
{
    for (int w0 = 0; w0 < ew; ++w0) {
        uint32_t bits = words[w0];
        const int pc = __popc(bits);
        if (r < pc) {
            for (int i = 0; i < r; ++i) bits &= bits - 1u;
            return w0 * 32 + __ffs(bits) - 1;
        }
        r -= pc;
    }
    return E;
}

// Key of the k-th largest lower interval end of one token (one warp), counted with
// multiplicity: per round the warp maximum of the remaining lower ends and how many experts
// hold it. Lane owns e = lane + 32 i (i < NS, NS * 32 >= E); its keys stay in registers and
// a taken one becomes INT_MIN.
template <int NS>
__device__ __forceinline__ int rf_kth_lower(const float *mr, const float *wn, float cx, int E,
                                            int k, int lane)
{
    int lk[NS];
#pragma unroll
    for (int i = 0; i < NS; ++i) {
        const int e = lane + 32 * i;
        lk[i] = (int)0x80000000;
        if (e < E) {
            const float m = mr[e];
            lk[i] = rf_key(m - (cx * wn[e] + 2.3841858e-7f * (fabsf(m) + 1.0f)));
        }
    }
    int taken = 0, Lk = (int)0x80000000;
    while (taken < k) {
        int best = (int)0x80000000;
#pragma unroll
        for (int i = 0; i < NS; ++i) best = lk[i] > best ? lk[i] : best;
        const int mx = __reduce_max_sync(0xffffffffu, best);
        Lk = mx;
        if (mx == (int)0x80000000) break; // nothing left (non-finite input)
        int mine = 0;
#pragma unroll
        for (int i = 0; i < NS; ++i)
            if (lk[i] == mx) {
                lk[i] = (int)0x80000000;
                ++mine;
            }
        taken += (int)__reduce_add_sync(0xffffffffu, (unsigned)mine);
    }
    return Lk;
}

// Top k of one token's candidates (one warp), ties to the lower expert id: writes
// idx_t[j] and returns, in lane j (j < 32), the gate value of the j-th selection (the
// selection key, or with the selection bias the logit without it); selections j >= 32 go to
// w_t[j] for the caller's softmax. *top receives the first selected value.
template <int NS>
__device__ __forceinline__ float rf_topk_token(const float *row, const uint32_t *cw,
                                               const float *bias, int E, int k, int gate,
                                               int32_t *idx_t, float *w_t, int lane, float *top)
{
    int fk[NS]; // selection keys of the lane's candidates, INT_MIN otherwise or once selected
#pragma unroll
    for (int i = 0; i < NS; ++i) {
        const int e = lane + 32 * i;
        fk[i] = (int)0x80000000;
        if (e < E && ((cw[i] >> lane) & 1u))
            fk[i] = rf_key((bias != nullptr) ? row[e] + bias[e] : row[e]);
    }
    float sel_val = 0.0f;
    for (int j = 0; j < k; ++j) {
        int best = (int)0x80000000, bi = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < NS; ++i)
            if (fk[i] > best) { // i ascending: keeps the lower id
                best = fk[i];
                bi = lane + 32 * i;
            }
        const int mx = __reduce_max_sync(0xffffffffu, best);
        int w = (int)__reduce_min_sync(0xffffffffu, (unsigned)(best == mx ? bi : 0x7fffffff));
        if (w < 0 || w >= E) w = 0; // unsupported non-finite rows still index the row
        const float bv = (gate == 2) ? row[w] : rf_unkey(mx);
#pragma unroll
        for (int i = 0; i < NS; ++i)
            if (lane + 32 * i == w) fk[i] = (int)0x80000000;
        if (j == 0) *top = bv;
        if (lane == 0) idx_t[j] = w;
        if (j < 32 && j == lane) sel_val = bv;
        if (j >= 32 && lane == 0) w_t[j] = bv;
    }
    return sel_val;
}

__global__ void __launch_bounds__(RF_THREADS)
    route_filter_exact_kernel(const __grid_constant__ CUtensorMap tmx,
                              const __grid_constant__ CUtensorMap tmw, const RfArgs a)
{
    extern __shared__ uint8_t rf_smem_raw[];
    uint8_t *rf_smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(rf_smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int E = a.E, H = a.H, T = a.T, k = a.k, bt = a.bt;
    const int ew = (E + 31) / 32;
    const int nslot = ew <= 1 ? 1 : ew <= 2 ? 2 : ew <= 4 ? 4 : ew <= 8 ? 8 : RF_MAX_E / 32;
    const int ME = E + 1; // padded filter-logit row
    const size_t r0 = rf_region0_bytes(bt, E, a.ring_bytes);
    float *mrow = reinterpret_cast<float *>(rf_smem);                // a/b: [bt][E + 1]
    float *exact = reinterpret_cast<float *>(rf_smem + r0);          // [bt][E] exact logits
    uint64_t *bars = reinterpret_cast<uint64_t *>(exact + (size_t)bt * E); // full, empty
    float *wn = reinterpret_cast<float *>(bars + 2 * RF_NS_MAX);     // [E] >= ||w_e||
    uint32_t *cand = reinterpret_cast<uint32_t *>(wn + E);          // [bt][ew]
    int *tok_off = reinterpret_cast<int *>(cand + (size_t)bt * ew); // [bt + 1] candidates
    int *unit_off = tok_off + RF_MAX_BT + 1;                         // [bt + 1] pair units
    int *e_range = unit_off + RF_MAX_BT + 1;                         // lowest, highest candidate
    volatile int *abort_flag = e_range + 2;
    const uint32_t bar0 = smem_u32(bars);
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (RF_NS_MAX + s); };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
    const int t0 = blockIdx.x * bt;
    const int nt = (T - t0) < bt ? (T - t0) : bt; // tokens of this block
    const size_t ET = (size_t)E * T;

    if (tid == 0) {
        for (int i = 0; i < RF_NS_MAX; ++i) {
            mbar_init(full_bar(i), 1);
            mbar_init(empty_bar(i), RF_CWARPS);
        }
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmx);
        tma_prefetch_desc(&tmw);
    }

    // ---- column norms and filter logits (summed over the splits, + bias) ----
    const int nslab = (H + RF_SLAB - 1) / RF_SLAB;
    for (int e = tid; e < E; e += RF_THREADS) {
        float s = 0.0f;
        for (int j0 = 0; j0 < nslab; j0 += 16) { // sixteen independent loads in flight
#pragma unroll
            for (int j = 0; j < 16; ++j)
                if (j0 + j < nslab) s += a.wpart[(size_t)(j0 + j) * E + e];
        }
        wn[e] = rf_norm_up(s, H);
    }
#pragma unroll 4
    for (int q = tid; q < E * bt; q += RF_THREADS) {
        const int e = q / bt, tl = q - e * bt; // consecutive threads: consecutive tokens
        if (tl < nt) {
            const float *pp = a.parts + (size_t)e * T + t0 + tl;
            float s = pp[0];
#pragma unroll
            for (int j = 1; j < RF_SPLIT_MAX; ++j) // splits in order; the loads are independent
                if (j < a.S) s += pp[(size_t)j * ET];
            if (a.bias != nullptr) s = s + a.bias[e];
            mrow[tl * ME + e] = s;
        }
    }
    __syncthreads();

    // ---- a/b. intervals and candidates, one warp per token ----
    for (int tl = warp; tl < bt; tl += RF_WARPS) {
        if (tl >= nt) {
            for (int w0 = lane; w0 < ew; w0 += 32) cand[tl * ew + w0] = 0u;
            continue;
        }
        const float *mr = mrow + tl * ME;
        float ss = 0.0f; // ||x_t||^2 from the filter GEMM's per-split partial sums
        for (int j = 0; j < a.S; ++j) ss += a.xsq[(size_t)j * T + t0 + tl];
        const float cx = a.cA * rf_norm_up(ss, H);
        // L = k-th largest lower end, counted with multiplicity
        int Lk;
        switch (nslot) {
        case 1: Lk = rf_kth_lower<1>(mr, wn, cx, E, k, lane); break;
        case 2: Lk = rf_kth_lower<2>(mr, wn, cx, E, k, lane); break;
        case 4: Lk = rf_kth_lower<4>(mr, wn, cx, E, k, lane); break;
        case 8: Lk = rf_kth_lower<8>(mr, wn, cx, E, k, lane); break;
        default: Lk = rf_kth_lower<RF_MAX_E / 32>(mr, wn, cx, E, k, lane); break;
        }
        const float L = rf_unkey(Lk);
        for (int w0 = 0; w0 < ew; ++w0) {
            const int e = w0 * 32 + lane;
            bool c = false;
            if (e < E) {
                const float m = mr[e];
                c = (m + (cx * wn[e] + 2.3841858e-7f * (fabsf(m) + 1.0f)) >= L);
            }
            const uint32_t bits = __ballot_sync(0xffffffffu, c);
            if (lane == 0) cand[tl * ew + w0] = bits;
        }
    }
    __syncthreads();

    // ---- candidate and unit offsets per token, union of the candidate experts ----
    if (warp == 0) {
        int cnt = 0;
        if (lane < bt)
            for (int w0 = 0; w0 < ew; ++w0) cnt += __popc(cand[lane * ew + w0]);
        const int units = (cnt + 1) >> 1; // two candidates of one token per thread
        int inc = cnt, uinc = units;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int o = __shfl_up_sync(0xffffffffu, inc, off);
            const int uo = __shfl_up_sync(0xffffffffu, uinc, off);
            if (lane >= off) {
                inc += o;
                uinc += uo;
            }
        }
        if (lane < bt) {
            tok_off[lane] = inc - cnt;
            unit_off[lane] = uinc - units;
        }
        if (lane == 31) { // lanes >= bt add 0
            tok_off[bt] = inc;
            unit_off[bt] = uinc;
        }
    } else if (warp == 1) {
        // id range of the candidate experts of the block's tokens (streamed as W_g^T rows)
        uint32_t uw = 0u; // union word `lane` (ew <= 16)
        if (lane < ew)
            for (int tl = 0; tl < bt; ++tl) uw |= cand[tl * ew + lane];
        const int lo = uw ? lane * 32 + __ffs(uw) - 1 : 0x7fffffff;
        const int hi = uw ? lane * 32 + 31 - __clz(uw) : -1;
        const int lo_all = __reduce_min_sync(0xffffffffu, lo);
        const int hi_all = __reduce_max_sync(0xffffffffu, hi);
        if (lane == 0) {
            e_range[0] = hi_all >= 0 ? lo_all : 0;
            e_range[1] = hi_all >= 0 ? hi_all : -1;
        }
    }
    __syncthreads();

    // ---- c. exact sequential logits of the candidate pairs ----
    // One producer thread streams chunk g of every pass into ring slot g % ns: a 2D TMA box
    // of the block's x rows and nbw boxes of the W_g^T rows e_lo.. (the candidates' id range),
    // counted on full[slot]; the consumer warps release the slot on empty[slot]. In a slot,
    // row r of a box holds its 16-byte column v at (v ^ (r & 7)) (128-byte swizzle).
    const int e_lo = e_range[0];
    const int n_rows_w = e_range[1] - e_lo + 1; // 0 when the block has no candidate
    const int nbw = (n_rows_w + RF_WBOX - 1) / RF_WBOX;
    const int NU = unit_off[bt];
    const uint32_t xs_bytes = (uint32_t)((bt * 128 + 1023) & ~1023);
    const uint32_t stage_bytes = (uint32_t)rf_stage_bytes(bt, nbw);
    int ns = a.ring_bytes / (int)stage_bytes;
    if (ns > RF_NS_MAX) ns = RF_NS_MAX;
    if (ns < 2) ns = 2; // the host sizes the ring for two chunks of every expert's rows
    const int nchunk = H / RF_HC;
    const int npass = (NU + RF_CTHREADS - 1) / RF_CTHREADS;
    const int total = npass * nchunk;

    if (warp >= RF_CWARPS) {
        // ---------------- producer ----------------
        if (lane == 0) {
            fence_proxy_async_smem(); // the filter logits written here before are dead
            const uint32_t ring0 = smem_u32(rf_smem);
            const uint32_t tx = (uint32_t)bt * 128 + (uint32_t)nbw * RF_WBOX * 128;
            int issued = 0;
            for (int g = 0; g < total; ++g) {
                const int slot = g % ns;
                if (g >= ns && !mbar_wait_bounded(empty_bar(slot), (uint32_t)((g / ns - 1) & 1),
                                                  abort_flag, a.timeout_ns, a.status, 180))
                    break;
                const int h0 = (g % nchunk) * RF_HC;
                const uint32_t base = ring0 + (uint32_t)slot * stage_bytes;
                mbar_arrive_expect_tx(full_bar(slot), tx);
                tma_load_2d(base, &tmx, full_bar(slot), h0, t0);
                for (int b = 0; b < nbw; ++b)
                    tma_load_2d(base + xs_bytes + (uint32_t)b * RF_WBOX * 128, &tmw, full_bar(slot),
                                h0, e_lo + b * RF_WBOX);
                issued = g + 1;
            }
            // every box issued has landed before the block moves on (immediate unless aborted)
            volatile int never = 0;
            for (int g = issued - 1; g >= 0 && g >= issued - ns; --g)
                mbar_wait_bounded(full_bar(g % ns), (uint32_t)((g / ns) & 1), &never, a.timeout_ns,
                                  nullptr, 0);
        }
        __syncwarp();
    } else {
        // ---------------- consumers ----------------
        bool ok = true;
        for (int pass = 0; ok && pass < npass; ++pass) {
            const int u = pass * RF_CTHREADS + tid;
            const bool active = u < NU;
            int tl = 0, e0 = 0, e1 = E;
            if (active) {
                while (tl + 1 < bt && unit_off[tl + 1] <= u) ++tl;
                const int r = 2 * (u - unit_off[tl]);
                e0 = rf_nth_bit(cand + tl * ew, ew, r, E);
                e1 = rf_nth_bit(cand + tl * ew, ew, r + 1, E); // E: this unit has one chain
            }
            const int r0w = active ? e0 - e_lo : 0;
            const int r1w = (e1 < E) ? e1 - e_lo : r0w;
            const uint32_t xo = (uint32_t)tl * 128, xk = (uint32_t)(tl & 7) << 4;
            const uint32_t wo0 = xs_bytes + (uint32_t)r0w * 128, wk0 = (uint32_t)(r0w & 7) << 4;
            const uint32_t wo1 = xs_bytes + (uint32_t)r1w * 128, wk1 = (uint32_t)(r1w & 7) << 4;
            float acc0 = 0.0f, acc1 = 0.0f;
            for (int c = 0; c < nchunk; ++c) {
                const int g = pass * nchunk + c;
                const int slot = g % ns;
                const bool got = mbar_wait_bounded(full_bar(slot), (uint32_t)((g / ns) & 1),
                                                   abort_flag, a.timeout_ns, a.status, 181);
                if (!__all_sync(0xffffffffu, got)) {
                    ok = false;
                    break;
                }
                if (active) {
                    const uint8_t *st = rf_smem + (size_t)slot * stage_bytes;
#pragma unroll
                    for (int vv = 0; vv < RF_HC / 8; ++vv) { // h ascending: storage order
                        const uint32_t v16 = (uint32_t)vv << 4;
                        const uint4 p = *reinterpret_cast<const uint4 *>(st + xo + (v16 ^ xk));
                        const uint4 q0 = *reinterpret_cast<const uint4 *>(st + wo0 + (v16 ^ wk0));
                        const uint4 q1 = *reinterpret_cast<const uint4 *>(st + wo1 + (v16 ^ wk1));
                        fma2x2_bf16(p.x, q0.x, q1.x, acc0, acc1);
                        fma2x2_bf16(p.y, q0.y, q1.y, acc0, acc1);
                        fma2x2_bf16(p.z, q0.z, q1.z, acc0, acc1);
                        fma2x2_bf16(p.w, q0.w, q1.w, acc0, acc1);
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(empty_bar(slot));
            }
            if (ok && active) { // the sequential logits without the bias
                exact[tl * E + e0] = acc0;
                if (e1 < E) exact[tl * E + e1] = acc1;
            }
        }
    }
    __syncthreads(); // exact logits complete

    // ---- d. top k of the candidates' exact logits (ties to the lower id) and the gates ----
    // Selection key: logit + bias (one fp32 addition, as the sequential router's logits);
    // gate value: the key, or with the selection bias (gate 2) the logit without the bias.
    for (int tl = warp; tl < nt; tl += RF_WARPS) {
        const int t = t0 + tl;
        const float *row = exact + tl * E;
        const uint32_t *cw = cand + tl * ew;
        float top = 0.0f, sel_val;
        int32_t *idx_t = a.topk_idx + (size_t)t * k;
        float *w_t = a.topk_w + (size_t)t * k;
        switch (nslot) {
        case 1: sel_val = rf_topk_token<1>(row, cw, a.bias, E, k, a.gate, idx_t, w_t, lane, &top); break;
        case 2: sel_val = rf_topk_token<2>(row, cw, a.bias, E, k, a.gate, idx_t, w_t, lane, &top); break;
        case 4: sel_val = rf_topk_token<4>(row, cw, a.bias, E, k, a.gate, idx_t, w_t, lane, &top); break;
        case 8: sel_val = rf_topk_token<8>(row, cw, a.bias, E, k, a.gate, idx_t, w_t, lane, &top); break;
        default:
            sel_val = rf_topk_token<RF_MAX_E / 32>(row, cw, a.bias, E, k, a.gate, idx_t, w_t, lane, &top);
            break;
        }
        __syncwarp();
        if (a.gate == 2) { // the largest selected logit (the first selected one need not be)
            float m = -INFINITY;
            for (int j = lane; j < k; j += 32)
                m = fmaxf(m, (j < 32) ? sel_val : a.topk_w[(size_t)t * k + j]);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
            top = m;
        }
        float denom = 0.0f;
        for (int j = lane; j < k; j += 32) {
            const float v = (j < 32) ? sel_val : a.topk_w[(size_t)t * k + j];
            denom += expf(v - top);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) denom += __shfl_xor_sync(0xffffffffu, denom, off);
        __syncwarp();
        for (int j = lane; j < k; j += 32) {
            const float v = (j < 32) ? sel_val : a.topk_w[(size_t)t * k + j];
            a.topk_w[(size_t)t * k + j] = expf(v - top) / denom;
        }
    }
}

} // namespace moe
