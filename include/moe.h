/*
 * moe.h -- C ABI of the B200 (sm_100a) forward pass of one mixture-of-experts layer.
 *
 * The layer is the one described in "Comet: Fine-grained Computation-communication
 * Overlapping for Mixture-of-Experts", §2.1 "MoE Structure": every token is routed to
 * its top-k experts, each selected expert applies its feed-forward network to the token,
 * and the k expert outputs are gathered back and reduced with the gate weights. The
 * dispatch step reorganises the routed tokens into expert-contiguous, tile-aligned rows
 * (§2.2.1 and §3.1.2, "How to reschedule the decomposed shared tensor?"); layer0 is
 * decomposed along M (token rows) and layer1 along N (output columns) (§3.1.1).
 *
 * Conventions shared by every entry point
 *   - Every tensor pointer is a DEVICE pointer owned by the caller, unless the entry point
 *     says HOST. The library never allocates device memory: scratch space comes from the
 *     caller's workspace (moe_workspace_size()).
 *   - bf16 tensors are passed as moe_bf16 (the raw 16-bit pattern), row-major, 16-byte
 *     aligned. int32/fp32 tensors are 4-byte aligned.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream). All work is enqueued
 *     asynchronously on it; no entry point synchronises except moe_get_device_status,
 *     moe_forward_host and moe_forward_host_batches (which wait for their own
 *     device-to-host copies).
 *   - Host-detectable errors (NULL pointers, unsupported sizes, a short workspace) are
 *     returned at once and nothing is launched. Errors found on the device (an expert id
 *     out of range, a bounded wait that ran out) are written to a status word in the
 *     workspace and returned by moe_get_device_status().
 *   - No C++ exception crosses this boundary.
 *   - The caller's buffers may not overlap each other or the workspace.
 *   - Concurrent calls that share one workspace race; give each stream its own.
 *   - The whole-layer launch and the expert-parallel launch are persistent, one CTA per SM,
 *     and their CTAs meet at grid-wide barriers: they expect the whole GPU. Kernels that
 *     run at the same time on other streams can keep some CTAs from starting; the waiting
 *     CTAs then give up after the wait timeout (moe_set_wait_timeout_ns) and the call
 *     reports MOE_ERR_DEVICE_TIMEOUT through the status word instead of hanging.
 *
 * Supported problem sizes: T >= 0, H % 64 == 0, F % 64 == 0, 1 <= top_k <= E <= 1024,
 * m_tile == 128; anything else returns MOE_ERR_UNSUPPORTED.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* bfloat16 bit pattern (sign, 8 exponent bits, 7 mantissa bits). */
typedef uint16_t moe_bf16;

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = -1,    /* NULL pointer, negative size, top_k > E, ... */
    MOE_ERR_UNSUPPORTED = -2,    /* legal but not supported by these kernels (see above) */
    MOE_ERR_WORKSPACE = -3,      /* ws_bytes smaller than moe_workspace_size() */
    MOE_ERR_CUDA = -4,           /* a CUDA runtime call failed (launch, copy, attribute) */
    MOE_ERR_DEVICE_TIMEOUT = -5, /* a bounded device wait ran out (status word) */
    MOE_ERR_DEVICE_BAD_INDEX = -6 /* an expert id or row index out of range (status word) */
} moe_status;

/* Expert activation. SWIGLU uses W1 [E, H, 2F]: columns [0, F) are the gate projection
 * (through silu), columns [F, 2F) the up projection; h = silu(x W_gate) * (x W_up).
 * The other three use W1 [E, H, F] and h = act(x W1). */
typedef enum {
    MOE_ACT_SWIGLU = 0,
    MOE_ACT_GELU_TANH = 1,
    MOE_ACT_RELU = 2,
    MOE_ACT_IDENTITY = 3
} moe_act;

/* Gate weights of the k selected experts (selection is always the k largest logits,
 * ties broken toward the lower expert id).
 * SOFTMAX_TOPK: softmax over the k selected logits. In exact arithmetic this equals a
 *   softmax over all E logits renormalised over the selected k (Mixtral's "softmax over
 *   the top-k logits" and Qwen2's "renormalised top-k gates" are the same function).
 * SOFTMAX_ALL: the full-E softmax values of the selected experts, not renormalised.
 * SELECT_BIAS: the bias steers the selection only (load balancing by a per-expert bias
 *   instead of an auxiliary loss): experts are selected by the logit plus bias[e] (the
 *   same fp32 sum as in the other modes), and the gates are the softmax over the k selected
 *   experts' logits without the bias. With a NULL bias it equals SOFTMAX_TOPK. */
typedef enum {
    MOE_GATE_SOFTMAX_TOPK = 0,
    MOE_GATE_SOFTMAX_ALL = 1,
    MOE_GATE_SELECT_BIAS = 2
} moe_gate;

typedef struct {
    int32_t T;      /* tokens */
    int32_t H;      /* hidden size (model dimension) */
    int32_t F;      /* expert FFN size */
    int32_t E;      /* number of experts */
    int32_t top_k;  /* experts per token */
    int32_t act;    /* moe_act */
    int32_t gate;   /* moe_gate */
    int32_t m_tile; /* row-tile height of the grouped GEMMs; must be 128 */
} moe_problem;

/* Number of stage boundaries recorded by moe_forward_staged: before routing, after
 * routing, after dispatch, after layer0, after layer1, after combine. */
#define MOE_NUM_STAGE_EVENTS 6

/* Bytes of workspace that is enough for every entry point on problem *p (moe_forward_host
 * uses all of it; moe_route, moe_dispatch and moe_forward use a prefix of it and accept a
 * buffer of this size). The caller allocates it, 256-byte aligned, and may reuse it across
 * calls on one stream. 0 if *p is invalid. */
MOE_API size_t moe_workspace_size(const moe_problem *p);

/* Number of kernels one moe_forward call on *p launches under the current GEMM and router
 * modes, assuming 16-byte aligned operands: 1 for the whole-layer launch
 * (moe_set_whole_layer_launch); otherwise the router (1 for up to 32 experts when E is a
 * multiple of 8, 3 with the tensor-core filter, else 2), the dispatch (3; 1 for T <= 256),
 * the gather of x into expert-sorted rows (1 when T * top_k >= E * 128, and always for the
 * CTA-pair GEMM) and the layers (layer0, layer1 and the combine: 3; or 1 for the persistent
 * launch that MOE_GEMM_FUSED forces and MOE_GEMM_AUTO picks for T * top_k >= E * 128 with
 * E <= 8). moe_forward_staged never takes the whole-layer launch (its stage events need the
 * stages' own launches). 0 for T == 0; -1 if *p is invalid. */
MOE_API int moe_forward_launches(const moe_problem *p);

/* Upper bound on the padded row count P_pad = sum_e ceil(c_e / m_tile) * m_tile, namely
 * T*top_k + min(E, T*top_k) * (m_tile - 1). gather_idx and ys buffers are sized with it,
 * so no host read of the expert counts is ever needed. -1 if *p is invalid. */
MOE_API int64_t moe_padded_rows_max(const moe_problem *p);

/* Router (§2.1: tokens are routed to selected experts at run time; §2.2.2: the
 * resulting expert loads vary).
 *   logits[t][e] = sum_h x[t][h] * Wg[h][e] (+ bias[e]), fp32, one accumulator per
 *   (t, e) walking h upward (this order is part of the contract: the selection below
 *   is bit-exact against a CPU reference that sums the same way);
 *   topk_idx[t][0..k-1] = the k largest logits, descending, ties to the lower id;
 *   topk_w[t][j] = gate weight per moe_gate.
 * x [T, H] bf16; Wg [H, E] bf16 (E contiguous); bias [E] fp32 or NULL;
 * topk_idx [T, k] int32 (out); topk_w [T, k] fp32 (out); ws/ws_bytes: workspace. */
MOE_API moe_status moe_route(const moe_problem *p, const moe_bf16 *x, const moe_bf16 *Wg,
                     const float *bias, int32_t *topk_idx, float *topk_w, void *ws,
                     size_t ws_bytes, void *stream);

/* Dispatch (§2.2.1 and §3.1.2: expose to each computation tile only the rows it needs;
 * regroup the routed rows into whole GEMM tiles). A counting sort of the T*k routed
 * pairs by expert, stable in token id, with each expert's rows padded to a multiple of
 * m_tile:
 *   counts[e]         pairs routed to expert e                                  [E]
 *   offsets[e]        exclusive prefix sum of counts                            [E+1]
 *   padded_offsets[e] exclusive prefix sum of ceil(counts/m_tile)*m_tile        [E+1]
 *   gather_idx[r]     token held by padded row r, -1 for a pad row   [moe_padded_rows_max]
 *   inv_pos[t][j]     padded row that holds pair (t, j)                         [T, k]
 *   x_perm (optional, may be NULL): x_perm[r] = x[gather_idx[r]], zeros on pad rows,
 *                     [moe_padded_rows_max, H] bf16; needs x.
 * topk_idx [T, k] int32 must hold distinct experts per token; an id outside [0, E) is
 * skipped and reported as MOE_ERR_DEVICE_BAD_INDEX by moe_get_device_status. */
MOE_API moe_status moe_dispatch(const moe_problem *p, const int32_t *topk_idx, int32_t *counts,
                        int32_t *offsets, int32_t *padded_offsets, int32_t *gather_idx,
                        int32_t *inv_pos, moe_bf16 *x_perm, const moe_bf16 *x, void *ws,
                        size_t ws_bytes, void *stream);

/* The whole layer: route -> dispatch -> layer0 grouped GEMM with the activation fused
 * in its epilogue (decomposed along M, §3.1.1) -> layer1 grouped GEMM with the gate
 * weight fused in its epilogue (decomposed along N, §3.1.1, column-wise §3.1.2) ->
 * deterministic top-k reduce (j ascending, fp32, rounded once to bf16).
 *   x [T, H] bf16; Wg [H, E] bf16; bias [E] fp32 or NULL;
 *   W1 [E, H, 2F] bf16 for SWIGLU, [E, H, F] otherwise; W2 [E, F, H] bf16;
 *   out [T, H] bf16 (out);
 *   topk_idx_out [T, k] int32 and topk_w_out [T, k] fp32: optional copies of the routing
 *   (NULL to keep them in the workspace only). */
MOE_API moe_status moe_forward(const moe_problem *p, const moe_bf16 *x, const moe_bf16 *Wg,
                       const float *bias, const moe_bf16 *W1, const moe_bf16 *W2, moe_bf16 *out,
                       int32_t *topk_idx_out, float *topk_w_out, void *ws, size_t ws_bytes,
                       void *stream);

/* moe_forward, plus cudaEventRecord of events[i] (cudaEvent_t handles owned by the
 * caller) at the MOE_NUM_STAGE_EVENTS stage boundaries, for per-stage timing.
 * n_events must be 0 (no events) or MOE_NUM_STAGE_EVENTS. */
MOE_API moe_status moe_forward_staged(const moe_problem *p, const moe_bf16 *x, const moe_bf16 *Wg,
                              const float *bias, const moe_bf16 *W1, const moe_bf16 *W2,
                              moe_bf16 *out, int32_t *topk_idx_out, float *topk_w_out, void *ws,
                              size_t ws_bytes, void *stream, void *const *events, int n_events);

/* moe_forward with HOST activations: x_host [T, H] and out_host [T, H] are host buffers
 * (pinned for asynchronous copies); the weights stay on the device. The call copies x
 * into the workspace, runs the layer, copies out back and waits for that copy, so
 * out_host is valid on return. */
MOE_API moe_status moe_forward_host(const moe_problem *p, const moe_bf16 *x_host, const moe_bf16 *Wg,
                            const float *bias, const moe_bf16 *W1, const moe_bf16 *W2,
                            moe_bf16 *out_host, void *ws, size_t ws_bytes, void *stream);

/* moe_forward on a stream of n_batches host batches: batch i reads x_host[i] and writes
 * out_host[i] (each [T, H] bf16, pinned host memory for overlap; arrays of n_batches
 * pointers; the same buffer may appear several times). Batch i+1's host-to-device copy and
 * batch i-1's device-to-host copy run on two library-owned copy streams while batch i
 * computes on `stream`; the x and out staging buffers in the workspace are double-buffered
 * (moe_workspace_size covers them). Every batch still copies its own input in and its own
 * output out. Returns after the last output has landed in host memory. The copy streams
 * and their events are created on the first call on a device and kept for the process. */
MOE_API moe_status moe_forward_host_batches(const moe_problem *p, int n_batches,
                                            const moe_bf16 *const *x_host, const moe_bf16 *Wg,
                                            const float *bias, const moe_bf16 *W1,
                                            const moe_bf16 *W2, moe_bf16 *const *out_host,
                                            void *ws, size_t ws_bytes, void *stream);

/* Shared expert (Qwen2-MoE style; a model feature beyond the pages): a SwiGLU FFN that
 * every token passes through, added to the routed experts' output with a per-token gate:
 *   out[t] = sum_j w_j FFN_{e_j}(x_t) + g_t FFN_s(x_t),   g_t = sigmoid(x_t . w_sg)
 * (g_t = 1 when w_sg is NULL). W1s [H, 2 F_s] bf16 (columns [0, F_s) gate, [F_s, 2 F_s)
 * up), W2s [F_s, H] bf16, w_sg [H] bf16; F_s % 64 == 0; device pointers, 16-byte aligned.
 * Precision as the routed experts: bf16 h_s and gated rows, the final sum in fp32 (the
 * shared row after the k routed ones), one bf16 rounding. */
typedef struct {
    int32_t F_s;
    const moe_bf16 *W1s;
    const moe_bf16 *W2s;
    const moe_bf16 *w_sg;
} moe_shared_expert;

/* Workspace bytes for moe_forward_shared on *p with a shared expert of width F_s (it also
 * covers every other entry point); 0 if invalid. */
MOE_API size_t moe_workspace_size_shared(const moe_problem *p, int32_t F_s);

/* moe_forward plus the shared expert. Its three kernels (the gate, then the dense SwiGLU
 * and gate-scaled GEMMs over all T tokens rounded up to 128 rows) run after the dispatch;
 * the combine adds its rows. moe_forward_launches(p) + 3 kernels. */
MOE_API moe_status moe_forward_shared(const moe_problem *p, const moe_bf16 *x,
                                      const moe_bf16 *Wg, const float *bias, const moe_bf16 *W1,
                                      const moe_bf16 *W2, const moe_shared_expert *shared,
                                      moe_bf16 *out, int32_t *topk_idx_out, float *topk_w_out,
                                      void *ws, size_t ws_bytes, void *stream);

/* FP8 experts (a precision variant beyond the pages, which fix no precision).
 * Element format e4m3 (OCP 8-bit floating point: 1 sign, 4 exponent bits with bias 7,
 * 3 mantissa bits, largest finite magnitude 448), stored as one byte per value.
 * Scaling of one vector v (a token row of x or of h over its K values, or one output column
 * of W1 or W2 over its K values): r = 448 / max|v|, s = max|v| / 448, both rounded to fp32
 * (r = s = 1 when r is not finite); code = e4m3(v * r), the product rounded to fp32, then
 * the nearest e4m3 value, ties to even, saturating at 448; v ~ decode(code) * s.
 * Weights are stored transposed, K contiguous: W1q [E, w1_cols, H] with s1 [E, w1_cols]
 * (w1_cols = 2F for SwiGLU, columns [0,F) gate and [F,2F) up, else F), W2q [E, H, F] with
 * s2 [E, H]. The FP8 path needs H % 128 == 0 and F % 128 == 0 (MOE_ERR_UNSUPPORTED
 * otherwise). All pointers are device pointers, 16-byte aligned. */
typedef uint8_t moe_fp8;

/* One-off preparation: the e4m3 codes and per-column scales of W1 [E, H, w1_cols] and
 * W2 [E, F, H] (bf16, as moe_forward takes them). Asynchronous on `stream`. */
MOE_API moe_status moe_quantize_experts_fp8(const moe_problem *p, const moe_bf16 *W1,
                                            const moe_bf16 *W2, moe_fp8 *W1q, float *s1,
                                            moe_fp8 *W2q, float *s2, void *stream);

/* Per-row quantisation of src [rows, cols] bf16 (cols % 8 == 0; src 16-byte and dst 8-byte
 * aligned) into dst [rows, cols] codes and scale [rows]: the step moe_forward_fp8 applies
 * to x and to h. */
MOE_API moe_status moe_quantize_rows_fp8(const moe_bf16 *src, int64_t rows, int32_t cols,
                                         moe_fp8 *dst, float *scale, void *stream);

/* Workspace bytes for moe_forward_fp8 on *p (it covers every bf16 entry point as well);
 * 0 if *p is invalid or unsupported on the FP8 path. */
MOE_API size_t moe_workspace_size_fp8(const moe_problem *p);

/* The layer with e4m3 experts. Routing and dispatch are the bf16 path's (x and W_g in bf16,
 * fp32 logits, bit-identical selection). Then: x rows quantised; layer0 on codes
 * (tcgen05 kind::f8f6f4, fp32 accumulation), each accumulator times s_x[token] * s1[column],
 * the activation, h stored bf16; h rows quantised; layer1 on codes, times
 * s_h[row] * s2[column] * the gate weight, stored bf16; the combine as moe_forward.
 * moe_forward_launches(p) counts the same route and dispatch kernels; this path launches
 * 3 + 1 + 1 + 1 + 1 + 1 kernels after the router (dispatch, x quantisation, layer0,
 * h quantisation, layer1, combine), plus one that gathers the x codes into expert-sorted
 * rows when T * top_k >= 128 * E (layer0 then reads them with TMA). */
MOE_API moe_status moe_forward_fp8(const moe_problem *p, const moe_bf16 *x, const moe_bf16 *Wg,
                                   const float *bias, const moe_fp8 *W1q, const float *s1,
                                   const moe_fp8 *W2q, const float *s2, moe_bf16 *out,
                                   int32_t *topk_idx_out, float *topk_w_out, void *ws,
                                   size_t ws_bytes, void *stream);

/* moe_forward_fp8 with caller events recorded at the MOE_NUM_STAGE_EVENTS stage boundaries
 * (as moe_forward_staged; the x quantisation is in the dispatch stage, the h quantisation
 * in the layer1 stage). */
MOE_API moe_status moe_forward_fp8_staged(const moe_problem *p, const moe_bf16 *x,
                                          const moe_bf16 *Wg, const float *bias,
                                          const moe_fp8 *W1q, const float *s1,
                                          const moe_fp8 *W2q, const float *s2, moe_bf16 *out,
                                          int32_t *topk_idx_out, float *topk_w_out, void *ws,
                                          size_t ws_bytes, void *stream, void *const *events,
                                          int32_t n_events);

/* The experts alone, for rows whose expert and gate are already known: the step each rank
 * runs on the rows it received under expert parallelism (the pages' multi-GPU layout, §2.1
 * and §3.1: experts sharded across GPUs, tokens exchanged all-to-all), or a caller's own
 * router. With p->top_k == 1 and p->E the experts held here, for each row r < p->T:
 *   out[r] = bf16(gate[r] * FFN_{expert[r]}(x[r]))
 * computed exactly as moe_forward computes a routed row (dispatch into 128-row expert tiles,
 * the same GEMMs and epilogues, one bf16 rounding of the gated row). expert [T] int32 in
 * [0, E) (an id outside it is reported as MOE_ERR_DEVICE_BAD_INDEX through
 * moe_get_device_status), gate [T] fp32. Workspace: moe_workspace_size(p). */
MOE_API moe_status moe_experts_forward(const moe_problem *p, const moe_bf16 *x,
                                       const int32_t *expert, const float *gate,
                                       const moe_bf16 *W1, const moe_bf16 *W2, moe_bf16 *out,
                                       void *ws, size_t ws_bytes, void *stream);

/* moe_experts_forward on the first *n_rows of its T rows, where n_rows is a device int32
 * read by the kernels (the host never reads it): the count of rows a rank received in the
 * device-driven expert-parallel exchange. Rows t >= *n_rows are not routed and their output
 * rows are left untouched; p->T is the capacity (sizes the workspace and the launches).
 * Always the separate launches (layer0, layer1, a k = 1 combine). Otherwise as
 * moe_experts_forward. */
MOE_API moe_status moe_experts_forward_n(const moe_problem *p, const moe_bf16 *x,
                                         const int32_t *expert, const float *gate,
                                         const int32_t *n_rows, const moe_bf16 *W1,
                                         const moe_bf16 *W2, moe_bf16 *out, void *ws,
                                         size_t ws_bytes, void *stream);

/* Expert parallelism with the exchange driven by the device (Comet: Fine-grained
 * Computation-communication Overlapping for Mixture-of-Experts, §2.1, §3.1: the routed
 * tokens travel to their experts' GPU and the outputs back; §4: the GPU issues the
 * transfers). Rank r of `world` holds experts [r * E / world, (r + 1) * E / world). Every
 * rank owns buffers that every rank can address (symmetric allocations): a counts table
 * [world, world] int32, receive buffers rows [recv_cap, H] bf16, ids [recv_cap] int32,
 * gates [recv_cap] fp32, origins [recv_cap] int64, and a return buffer [T * k, H] bf16. The
 * pointer arguments `tables`, `rows`, `ids`, `gates`, `origin`, `back` are DEVICE arrays of
 * `world` pointers (entry r: rank r's buffer as this GPU addresses it). The host never reads
 * the routing. The caller synchronises the ranks between the steps (a barrier of all ranks
 * on the stream, e.g. the symmetric-memory barrier):
 *   1. moe_route and moe_dispatch on this rank's tokens (all E experts);
 *   2. moe_ep_publish_counts: this rank's rows per destination (from `offsets`, the
 *      dispatch's [E+1] unpadded offsets) into row `rank` of every rank's table;  -- barrier
 *   3. moe_ep_scatter: every routed pair (t, j) goes, by stores into the destination's
 *      buffers, to slot (rows lower ranks send there) + (its position among this rank's rows
 *      for that destination, in the dispatch's expert-then-token order), with its local
 *      expert id, gate and origin (rank << 32 | t * k + j); writes n_recv[0] = the rows this
 *      rank receives (a device int);                                               -- barrier
 *   4. moe_experts_forward_n on the receive buffers (E / world experts, k = 1, T = recv_cap,
 *      n_rows = n_recv);
 *   5. moe_ep_return: received row i goes to row (origin & 0xffffffff) of rank
 *      (origin >> 32)'s return buffer;                                             -- barrier
 *   6. moe_combine of the return buffer with inv_pos[t][j] = t * k + j.
 * Every gated row is bitwise the row moe_forward computes on one GPU. Errors (an expert id
 * outside [0, E), a slot past recv_cap, a bad origin) go to the status word of `ws`
 * (moe_workspace_size of the scatter's problem; for moe_ep_return the workspace of the
 * step-4 call) as MOE_ERR_DEVICE_BAD_INDEX. recv_cap >= world * T * min(k, E / world) holds
 * every routing. The stores to other GPUs are plain stores; nothing loads another GPU's
 * memory. */
MOE_API moe_status moe_ep_publish_counts(const moe_problem *p, int32_t world, int32_t rank,
                                         const int32_t *offsets, int32_t *const *tables,
                                         void *stream);
MOE_API moe_status moe_ep_scatter(const moe_problem *p, int32_t world, int32_t rank,
                                  const moe_bf16 *x, const int32_t *topk_idx,
                                  const float *topk_w, const int32_t *offsets,
                                  const int32_t *padded_offsets, const int32_t *inv_pos,
                                  const int32_t *table, moe_bf16 *const *rows,
                                  int32_t *const *ids, float *const *gates,
                                  int64_t *const *origin, int64_t recv_cap, int32_t *n_recv,
                                  void *ws, size_t ws_bytes, void *stream);
MOE_API moe_status moe_ep_return(int32_t H, int32_t world, const moe_bf16 *y,
                                 const int64_t *origin, const int32_t *n_recv, int64_t recv_cap,
                                 moe_bf16 *const *back, int64_t back_rows, void *ws,
                                 void *stream);

/* Expert-parallel layer with the exchange overlapped with the expert GEMMs, one persistent
 * launch per GPU (Comet §3.1.2: layer0 tiles start as their rows arrive, layer1 rows return
 * as their tiles finish; §4: the GPU issues fine-grained transfers; the tile-signalling
 * abstract: transfers fired and awaited per tile through ready flags). Rank r of `world`
 * (1 <= world <= MOE_EP_MAX_WORLD, world dividing E) holds experts [r * E / world,
 * (r + 1) * E / world) and its own T tokens; the router (E a multiple of 8, E <= 32, H a
 * multiple of 64) is replicated. In the launch, every CTA of rank r:
 *   1. routes a group of r's tokens (the exact router), and writes the group's selections per
 *      expert into every rank's counts buffer; a barrier of r's CTAs; r raises its flag in
 *      every rank's flags buffer (value `epoch`) and waits for every rank's flag in its own;
 *   2. derives, from every rank's counts, where each of r's pairs goes -- row = destination
 *      d's padded offset of the expert + the rows of lower source ranks + r's earlier tokens
 *      (d's receive buffer is expert-sorted, 128-row padded, source rank then token within an
 *      expert); CTA 0 writes r's receive-side tile list; a barrier of r's CTAs;
 *   3. four data-movement warps per CTA store each of r's pairs' x row, gate and origin into
 *      the destination's receive buffers and then add 1 to the destination's arrival count
 *      of that 128-row tile; meanwhile the GEMM pipeline runs r's experts: a layer0 tile
 *      waits only until its rows have arrived; a layer1 tile waits for its layer0 rows (the
 *      tile-level counters of the persistent launch) and its epilogue stores each gated row
 *      straight into row t * k + j of the origin's return buffer and adds 1 to the origin's
 *      count of that token and 256-column stripe;
 *   4. the combine sums the k returned rows of each of r's tokens (j ascending, fp32, one
 *      bf16 rounding), a 256-column stripe as soon as that stripe of the k rows is back.
 * Stores to other GPUs are plain 16-byte stores followed by a system-scope fence before the
 * count; nothing loads another GPU's memory, no TMA reads another GPU's memory, and every
 * wait is bounded (MOE_ERR_DEVICE_TIMEOUT in the status word of the rank's workspace). Every
 * gated row is bitwise the row moe_forward computes on one GPU, so `out` is bitwise
 * moe_forward's output for r's tokens with all E experts.
 * Buffers: each rank owns the eight exchange buffers of moe_ep_buffer_sizes, addressable by
 * every rank (symmetric allocations; zero-filled once before the first call); entry d of
 * each pointer table of moe_ep_rank is rank d's buffer as this GPU addresses it. Calls on
 * the same buffers pass epoch 1, 2, 3, ... (the same on every rank for one layer call).
 * n_local: ranks this launch carries -- 1 on a GPU per rank; up to MOE_EP_MAX_LOCAL to run
 * several ranks on one GPU (all their buffers on this GPU; each rank gets 1/n_local of the
 * SMs), which is how the ranks' interplay is tested with one GPU. All ranks of a layer call
 * must launch (their waits on one another are bounded, not avoided), with the same problem
 * (T, H, F, E, top_k, act, gate), the same n_local and the same number of SMs: the layout
 * of the counts buffers follows the token groups, which these fix. A call that reported an
 * error may leave other ranks' stores in flight into these buffers: zero-fill every rank's
 * buffers again (and synchronise the ranks) before the next call. */
#define MOE_EP_MAX_WORLD 8
#define MOE_EP_MAX_LOCAL 4
#define MOE_EP_NUM_BUFFERS 8
typedef struct {
    moe_problem p;           /* this rank's tokens T; all E experts; top_k, act, gate */
    int32_t world, rank;
    int32_t epoch;           /* > 0, increasing call to call on the same buffers */
    const moe_bf16 *x;       /* [T, H] this rank's tokens */
    const moe_bf16 *Wg;      /* [H, E] router (the same on every rank) */
    const float *bias;       /* [E] or NULL */
    const moe_bf16 *W1;      /* [E / world, H, 2F] (SwiGLU) or [E / world, H, F]: r's experts */
    const moe_bf16 *W2;      /* [E / world, F, H] */
    moe_bf16 *out;           /* [T, H] */
    int32_t *topk_idx;       /* [T, top_k] or NULL (kept in the workspace) */
    float *topk_w;           /* [T, top_k] or NULL */
    void *ws;                /* moe_ep_workspace_size bytes, 256-byte aligned */
    size_t ws_bytes;
    /* every rank's exchange buffers (index d: rank d's), in the order of moe_ep_buffer_sizes:
     * counts, flags, recv_rows, recv_gate, recv_origin, arrive, back, back_cnt */
    void *buf[MOE_EP_NUM_BUFFERS][MOE_EP_MAX_WORLD];
} moe_ep_rank;

/* Bytes of each exchange buffer of one rank for ranks of T tokens (*p) in a world of
 * `world`: sizes[0..7] = counts, flags, recv_rows, recv_gate, recv_origin, arrive, back,
 * back_cnt (each to be 256-byte aligned, zero-filled once). MOE_OK or an error code. */
MOE_API moe_status moe_ep_buffer_sizes(const moe_problem *p, int32_t world, int64_t *sizes);
/* Workspace bytes of one rank (0 if *p or world is invalid). */
MOE_API size_t moe_ep_workspace_size(const moe_problem *p, int32_t world);
/* The layer for the n_local ranks ranks[0 .. n_local - 1] on this GPU, one launch on
 * `stream` (after a 32-byte memset per rank). MOE_OK, MOE_ERR_INVALID_ARG (shapes, world,
 * alignment, router not applicable), MOE_ERR_WORKSPACE or MOE_ERR_CUDA. */
MOE_API moe_status moe_ep_layer_forward(const moe_ep_rank *ranks, int32_t n_local, void *stream);

/* Backward pass (training; beyond the pages, which describe the forward).
 * Given dout = dL/dout [T, H] bf16, the gradients of the layer moe_forward computes, with the
 * selection held fixed (it is piecewise constant) and the gates the softmax over the
 * selected logits:
 *   dx [T, H] bf16, dWg [H, E] fp32, dbias [E] fp32 (zero with MOE_GATE_SELECT_BIAS, or
 *   without a bias), dW1 [E, H, w1_cols] bf16, dW2 [E, F, H] bf16.
 * Per routed row (token t, selection j, expert e): dw_j = dout_t . y_e(x_t),
 * dl_j = w_j (dw_j - sum_i w_i dw_i), gy = w_j dout_t, dW2[e] += a^T gy, da = gy W2[e]^T,
 * dz = da * act'(z) (SwiGLU: [da up silu'(g), da silu(g)]), dW1[e] += x_t^T dz,
 * dx_t += dz W1[e]^T + dl_j W_g[:, e], dW_g[:, e] += x_t dl_j, dbias[e] += dl_j.
 * The call recomputes the routing, the dispatch and z = x W1 (it needs no state from a
 * forward call). bf16 intermediates with fp32 accumulation; sums over tokens in the
 * experts' row order. Needs H % 128 == 0, F % 128 == 0 and a gate mode other than
 * MOE_GATE_SOFTMAX_ALL (MOE_ERR_UNSUPPORTED otherwise). Device pointers, 16-byte aligned
 * (4-byte for the fp32 ones). */
MOE_API size_t moe_backward_workspace_size(const moe_problem *p);
MOE_API moe_status moe_backward(const moe_problem *p, const moe_bf16 *x, const moe_bf16 *Wg,
                                const float *bias, const moe_bf16 *W1, const moe_bf16 *W2,
                                const moe_bf16 *dout, moe_bf16 *dx, float *dWg, float *dbias,
                                moe_bf16 *dW1, moe_bf16 *dW2, void *ws, size_t ws_bytes,
                                void *stream);

/* Combine (§2.1: gather and reduce the top-k outputs).
 *   out[t][n] = bf16_rne( sum_{j=0..k-1} ys[inv_pos[t][j]][n] ), fp32 sum, j ascending.
 * ys [ys_rows, H] bf16 holds expert-sorted rows that already carry their gate weight;
 * inv_pos [T, k] int32 as produced by moe_dispatch. A row index outside [0, ys_rows)
 * contributes nothing; if ws is not NULL it is also reported as MOE_ERR_DEVICE_BAD_INDEX
 * through moe_get_device_status (ws may be NULL, then ws_bytes is ignored). */
MOE_API moe_status moe_combine(const moe_problem *p, const moe_bf16 *ys, int64_t ys_rows,
                       const int32_t *inv_pos, moe_bf16 *out, void *ws, size_t ws_bytes,
                       void *stream);

/* Synchronises `stream`, then reads and clears the device status word in ws.
 * Returns MOE_OK, MOE_ERR_DEVICE_TIMEOUT, MOE_ERR_DEVICE_BAD_INDEX or MOE_ERR_CUDA.
 * Every other entry point clears the word when its first kernel starts. */
MOE_API moe_status moe_get_device_status(void *ws, void *stream);

/* Human-readable name of a status code (static storage). */
MOE_API const char *moe_status_string(moe_status s);

/* Largest T * E that moe_route_noalloc accepts: its logits scratch is a fixed array of
 * this many floats (4 MiB) inside the library. */
#define MOE_ROUTE_NOALLOC_MAX_LOGITS (1 << 20)

/* moe_route without a workspace, for callers that cannot allocate device memory: code that
 * is handed only its input and output buffers by a host framework that owns the device
 * heap (a plugin inside an inference engine, for example), and serving loops that must not
 * call cudaMalloc/cudaFree after start-up because those calls can synchronise the device
 * and stall every other stream. The pages have no counterpart of this entry point.
 *   Same arguments and results as moe_route, minus ws/ws_bytes. The router's fp32 logits
 *   [T, E] go to a fixed scratch array that the library holds in device memory on every GPU
 *   that loads it, until the process exits; T * E above MOE_ROUTE_NOALLOC_MAX_LOGITS
 *   returns MOE_ERR_UNSUPPORTED and launches nothing.
 *   The first call on a device looks up that array's device address (once per device,
 *   with the device current); make that first call before any stream capture. Later calls
 *   do no set-up. The call allocates nothing and frees nothing.
 *   All calls share the one array and every call overwrites the logits it reads, so nothing
 *   has to be cleared between calls; but two calls whose kernels overlap on the GPU (on
 *   different streams, or from different host threads) race on the array and may return
 *   each other's routing. The current device must be the device of `stream`. */
MOE_API moe_status moe_route_noalloc(const moe_problem *p, const moe_bf16 *x, const moe_bf16 *Wg,
                                     const float *bias, int32_t *topk_idx, float *topk_w,
                                     void *stream);

/* Test hook for the bounded device waits: the timeout, in nanoseconds, that every
 * bounded wait of later launches uses (default 2e9; values <= 0 restore the default).
 * Returns the previous value. Not thread-safe; meant for tests. */
MOE_API int64_t moe_set_wait_timeout_ns(int64_t ns);

/* Grouped-GEMM variant used by later launches (a tuning and test hook; not thread-safe):
 * MOE_GEMM_SINGLE_CTA runs one 128 x 256 tile per SM; MOE_GEMM_CTA_PAIR runs one
 * 256 x 256 tile per pair of SMs (tcgen05 cta_group::2: each SM loads half of the weight
 * tile); MOE_GEMM_AUTO (the default) picks the single-CTA variant, the faster one under the
 * sustained power cap. Both compute the same layer. Returns the previous mode, or -1 for an
 * unknown mode. */
#define MOE_GEMM_AUTO 0
#define MOE_GEMM_SINGLE_CTA 1
#define MOE_GEMM_CTA_PAIR 2
/* MOE_GEMM_FUSED: layer0, layer1 and the combine in one persistent launch, scheduled by
 * tile-level ready flags (a layer1 tile starts when layer0 has finished its 128 h rows; a
 * combine item -- a 256-column stripe of a block of tokens -- reads each of its rows as
 * soon as layer1 has stored that stripe of the row's tile). In every CTA four warps move
 * data: during layer0 they gather token rows or take half of each tile's epilogue, during
 * layer1 they run the combine beside the GEMM pipeline. MOE_GEMM_AUTO takes this launch
 * when T * top_k >= E * 128 (every expert averages a full 128-row tile) and E <= 8: layer1
 * runs expert-major, so the combine's window beside it is about 1/E of layer1, and with
 * more experts the separate launches measured faster. Otherwise the separate launches. Stage events 3..5 of moe_forward_staged then all mark the end of that one
 * launch. */
#define MOE_GEMM_FUSED 3
/* MOE_GEMM_FUSED_LAYERS: layer0 and layer1 in the persistent launch (layer1 tiles start as
 * their M tile's h rows are done, no launch boundary between the layers), the combine as
 * its own launch after it (full occupancy); stage event 5 then marks the combine's end. */
#define MOE_GEMM_FUSED_LAYERS 4
MOE_API int moe_set_gemm_mode(int mode);

/* Whole-layer launch (Comet §5.3: the small-batch gains come from taking the host-driven
 * steps out of the layer; here the route and dispatch steps join the persistent launch).
 * On by default. It applies when the persistent launch runs (MOE_GEMM_FUSED, or
 * MOE_GEMM_AUTO's choice), E == 8, the layer's routing is computed (not supplied), the
 * router is the one-launch exact router (not the tensor-core filter), no stage events are
 * requested and x, W_g are 16-byte aligned. Every CTA of the persistent launch (one per SM)
 * then first routes about T / SMs tokens and counts its selections per expert; the CTAs
 * meet at a grid-wide barrier (a counter in the workspace's status block); each derives the
 * experts' offsets, CTA 0 writes the dispatch outputs, and each places its own pairs
 * (expert-major, ascending token order within an expert -- the rows of the separate
 * dispatch) and copies their x rows into the expert-sorted buffer; after a second barrier
 * the GEMM phases begin. moe_forward is then one kernel launch after one 32-byte memset of
 * the status block. The outputs equal those of the separate launches bit for bit, except
 * that pad rows of the expert-sorted copy of x are not written. on = 0 turns it off
 * (routing and dispatch as their own launches). Returns the previous setting. */
MOE_API int moe_set_whole_layer_launch(int on);

/* Work order of the single-CTA grouped-GEMM launches (a tuning and test hook; not
 * thread-safe). An expert with a single m-tile ("cold": at most m_tile routed rows) has its
 * weights streamed for that one tile.
 * MOE_ORDER_EXPERT: one launch per layer, expert-major (expert, then N tile, then M tile);
 * MOE_ORDER_MIXED: the same launch with the cold experts' work items spread evenly among
 *   the others' (measured no gain: the GEMMs are power-bound under the 1 kW cap);
 * MOE_ORDER_NARROW (default): as MOE_ORDER_EXPERT, except that when every routed expert is
 *   cold (decode-sized batches) the device runs the layer with the operands swapped (the
 *   weight tile is the MMA's M = 128, the expert's rows rounded up to 16 its N): the same
 *   weight bytes with far less tensor-core work (measured 5-7% faster per GEMM there);
 * MOE_ORDER_PHASED: in each launch every CTA first runs its share of the cold experts'
 *   items in that operand-swapped form (all SMs streaming cold weights at once), then its
 *   share of the other experts' 128-row items (as MOE_ORDER_NARROW when all are cold or
 *   none is). Also used by moe_forward_fp8.
 * The layer outputs agree within the parity tolerance in every order; MOE_ORDER_EXPERT and
 * MOE_ORDER_MIXED are bitwise identical. Returns the previous order, or -1. */
#define MOE_ORDER_EXPERT 0
#define MOE_ORDER_MIXED 1
#define MOE_ORDER_NARROW 2
#define MOE_ORDER_PHASED 3
MOE_API int moe_set_work_order(int order);

/* Router variant (a tuning and test hook; not thread-safe). All give the same routing and
 * gates (the selection is always made on the sequential fp32 logits, see moe_route):
 * MOE_ROUTER_FILTER: for 8 <= E <= 512 with E % 8 == 0, a gate other than SOFTMAX_ALL and 16-byte
 *   aligned x and Wg, the logits are first computed on the tensor cores; every expert whose
 *   logit interval (a rigorous bound on the difference between the two fp32 sums) cannot
 *   reach the top k is dropped, and only the rest get the sequential fp32 logit (other
 *   problems use the sequential router);
 * MOE_ROUTER_SEQUENTIAL: every (token, expert) logit is computed sequentially;
 * MOE_ROUTER_AUTO (default): the filter where it applies, E >= 16 and T * E >= 2^16, else
 *   sequential.
 * moe_route_noalloc always uses the sequential router.
 * Returns the previous mode, or -1 for an unknown mode. */
#define MOE_ROUTER_AUTO 0
#define MOE_ROUTER_SEQUENTIAL 1
#define MOE_ROUTER_FILTER 2
MOE_API int moe_set_router_mode(int mode);

/* 1 if moe_route / moe_forward on *p take the filter router under the current router mode,
 * 0 if the sequential one, -1 if *p is invalid. */
MOE_API int moe_route_uses_filter(const moe_problem *p);

/* Test hook for the bounded ready-flag waits of MOE_GEMM_FUSED: the layer0 work item with
 * this index (in the kernel's static work queue) withholds its ready signal, so the layer1
 * tiles that need it wait until the timeout (moe_set_wait_timeout_ns) and the call reports
 * MOE_ERR_DEVICE_TIMEOUT through moe_get_device_status. Nothing faults or hangs: every CTA
 * leaves within a few timeouts and the context stays usable. -1 switches it off (default).
 * Returns the previous value. Not thread-safe; meant for tests. */
MOE_API int moe_set_fault_injection(int layer0_item);

/* Schedule trace of the persistent (fused) launch, for profiling; off by default.
 * `records` is a device buffer of 4 + 4 * capacity uint64 values owned by the caller; pass
 * nullptr to switch the trace off. The caller zeroes records[0] (the record counter) before
 * a traced call. Each finished work item appends {kind << 32 | item, SM id, begin ns, end ns}
 * at records[4 + 4 i] (globaltimer nanoseconds; kind 0 = a layer0 tile's epilogue, 1 = a
 * layer1 tile's epilogue, 2 = a combine item); items past `capacity` are counted but not
 * stored. Not thread-safe; meant for profiling runs (it adds one atomic per work item).
 * Returns MOE_OK, or MOE_ERR_INVALID_ARG for a negative capacity. */
MOE_API moe_status moe_set_schedule_trace(void *records, int64_t capacity);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
