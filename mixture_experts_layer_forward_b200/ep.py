"""Expert parallelism: the layer with its experts sharded across GPUs.

This is the pages' multi-GPU layout (Comet: Fine-grained Computation-communication
Overlapping for Mixture-of-Experts, §2.1 "MoE Structure" and §3.1: experts are placed on
different GPUs, the routed tokens travel to their experts' GPU before layer0 and the expert
outputs travel back after layer1, by all-to-all). Each rank holds E / world experts
(experts r * E_local .. (r + 1) * E_local - 1 on rank r), a replicated router, and its own
tokens:

1. route its tokens (moe_route on the full W_g);
2. order its T * k routed pairs by destination rank, stable in (token, selection) order;
3. all-to-all the row counts, then the x rows, the local expert ids and the gates;
4. run its experts on the rows it received (moe_experts_forward: the same per-row
   arithmetic as moe_forward, so every gated row is bitwise the row moe_forward computes);
5. all-to-all the gated rows back, in the order they were sent;
6. combine: out[t] = bf16(sum over j ascending of row (t, j)), fp32 sum (moe_combine).

bf16 rows cross the collectives as int32 words (the same bytes, two values per word, a
dtype every backend carries). The exchange runs on NCCL between GPUs; the expert and combine
steps are pluggable, so the plan is also exercised on CPU (gloo) by the tests. NCCL's
all-to-all needs the split sizes on the host, so step 3 reads the counts back (one device
synchronisation per layer).

ep_moe_forward_device is the same layer with the exchange driven by the device instead
(csrc/ep.cuh): the counts, the row positions and the transfers stay on the GPU, the rows are
stored straight into the destination's receive buffers (symmetric memory every rank can
address), and the host never reads the routing; the ranks meet at device barriers between
the steps. Not measured on several GPUs here (one GPU per run); its one-rank form is tested
against moe_forward.

EpLayer is the layer with the exchange overlapped with the expert GEMMs, one persistent launch
per GPU (moe_ep_layer_forward, csrc/fused.cuh): the rows are stored into the experts' ranks'
expert-sorted receive buffers by four warps per SM while the same SMs run the rank's experts,
a layer0 tile starting as soon as its rows have arrived (an arrival count per tile, Comet
§3.1.2 and §4; the tile-signalling abstract); layer1 stores every gated row straight into its
origin's return buffer and counts it there, and the origin's combine sums a token's rows as
soon as they are all back. ep_layer_forward_local runs several ranks in one launch on one
GPU (each rank a share of the SMs, all buffers on this GPU): the same kernels and waits as
one GPU per rank, which is how the ranks' interplay is tested here.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def experts_per_rank(E: int, world: int) -> int:
    if E % world != 0:
        raise ValueError(f"E = {E} experts do not shard evenly over {world} ranks")
    return E // world


def dispatch_plan(topk_idx: torch.Tensor, E: int, world: int):
    """For the [T, k] routing of this rank: the stable order of its T * k pairs by
    destination rank, the number of pairs sent to each rank, and each sent pair's expert id
    local to its destination."""
    e_loc = experts_per_rank(E, world)
    flat = topk_idx.reshape(-1).long()
    dest = torch.div(flat, e_loc, rounding_mode="floor")
    order = torch.argsort(dest, stable=True)
    send_counts = torch.bincount(dest, minlength=world)
    local_ids = (flat - dest * e_loc)[order]
    return order, send_counts, local_ids


def _exchange(send: torch.Tensor, send_counts, recv_counts, group):
    """all-to-all of the rows of `send` (already in destination order). bf16 rows travel as
    int32 words (two values each, H even)."""
    bf = send.dtype == torch.bfloat16
    bits = send.contiguous().view(torch.int32) if bf else send.contiguous()
    shape = (int(sum(recv_counts)),) + tuple(bits.shape[1:])
    recv = torch.empty(shape, dtype=bits.dtype, device=send.device)
    dist.all_to_all_single(recv, bits, output_split_sizes=list(recv_counts),
                           input_split_sizes=list(send_counts), group=group)
    return recv.view(torch.bfloat16) if bf else recv


def ep_forward(x: torch.Tensor, topk_idx: torch.Tensor, topk_w: torch.Tensor, E: int,
               expert_fn, combine_fn, group=None) -> torch.Tensor:
    """Steps 2-6 above for this rank's tokens x [T, H] (bf16) routed to topk_idx / topk_w
    [T, k]. expert_fn(rows [R, H], local ids [R] int32, gates [R] fp32) -> gated rows [R, H]
    bf16 for this rank's experts; combine_fn(rows [T * k, H], inv_pos [T, k] int32) -> out."""
    world = dist.get_world_size(group)
    T, k = topk_idx.shape
    order, send_counts, local_ids = dispatch_plan(topk_idx, E, world)
    send_counts = send_counts.to(device=x.device, dtype=torch.int64)
    recv_counts = torch.empty_like(send_counts)
    dist.all_to_all_single(recv_counts, send_counts, group=group)
    sc, rc = send_counts.tolist(), recv_counts.tolist() # split sizes on the host
    tok = torch.div(order, k, rounding_mode="floor").to(x.device)
    rows = _exchange(x.index_select(0, tok), sc, rc, group)
    ids = _exchange(local_ids.to(device=x.device, dtype=torch.int32), sc, rc, group)
    gates = _exchange(topk_w.reshape(-1)[order.to(topk_w.device)].float(), sc, rc, group)
    y = expert_fn(rows, ids, gates)
    back = _exchange(y, rc, sc, group)                # row i of `back` is pair order[i]
    inv = torch.empty_like(order)
    inv[order] = torch.arange(order.numel(), device=order.device)
    return combine_fn(back, inv.view(T, k).to(device=x.device, dtype=torch.int32))


def gpu_expert_fn(H: int, F: int, E_local: int, W1_local, W2_local, act: int = 0):
    """expert_fn running moe_experts_forward on this GPU's expert weights."""
    from . import _native as moe

    def fn(rows, ids, gates):
        R = rows.shape[0]
        p = moe.Problem.make(R, H, F, E_local, 1, act)
        out = torch.empty(R, H, dtype=torch.bfloat16, device=rows.device)
        ws = torch.empty(max(moe.moe_workspace_size(p), 1), dtype=torch.uint8, device=rows.device)
        moe.moe_experts_forward(p, rows, ids, gates, W1_local, W2_local, out, ws)
        if moe.moe_get_device_status(ws) != 0:
            raise RuntimeError("moe_experts_forward reported a device error")
        return out

    return fn


def gpu_combine_fn(H: int, F: int, E: int, k: int):
    """combine_fn running moe_combine (fp32 sum over j ascending, one bf16 rounding)."""
    from . import _native as moe

    def fn(back, inv_pos):
        T = inv_pos.shape[0]
        p = moe.Problem.make(T, H, F, E, k)
        out = torch.empty(T, H, dtype=torch.bfloat16, device=back.device)
        moe.moe_combine(p, back, inv_pos, out)
        return out

    return fn


def ep_moe_forward(p, x, Wg, bias, W1_local, W2_local, group=None):
    """The whole layer under expert parallelism on this rank's GPU: route (replicated W_g,
    all E experts), exchange, local experts, exchange back, combine. p is the full layer's
    problem (all E experts, this rank's T tokens); W1_local / W2_local hold this rank's
    E / world experts."""
    from . import _native as moe

    world = dist.get_world_size(group)
    e_loc = experts_per_rank(p.E, world)
    idx = torch.empty(p.T, p.top_k, dtype=torch.int32, device=x.device)
    w = torch.empty(p.T, p.top_k, dtype=torch.float32, device=x.device)
    ws = torch.empty(moe.moe_workspace_size(p), dtype=torch.uint8, device=x.device)
    moe.moe_route(p, x, Wg, bias, idx, w, ws)
    return ep_forward(x, idx, w, p.E, gpu_expert_fn(p.H, p.F, e_loc, W1_local, W2_local, p.act),
                      gpu_combine_fn(p.H, p.F, p.E, p.top_k), group)


class DeviceExchange:
    """Buffers of ep_moe_forward_device in symmetric memory (every rank can address every
    rank's copy) and the device arrays of their per-rank addresses. One instance per layer
    shape and process group; the ranks must create it in the same order (a collective)."""

    def __init__(self, p, group=None, device=None):
        import torch.distributed._symmetric_memory as symm_mem

        from . import _native as moe

        self.group = group if group is not None else dist.group.WORLD
        self.world = dist.get_world_size(self.group)
        self.rank = dist.get_rank(self.group)
        dev = device if device is not None else torch.device("cuda", torch.cuda.current_device())
        e_loc = experts_per_rank(p.E, self.world)
        self.p = p
        self.e_loc = e_loc
        # every rank sends each destination at most min(k, E_loc) rows per token
        self.recv_cap = self.world * p.T * min(p.top_k, e_loc)
        self.bufs = {}
        self.handles = {}
        self.addr = {}
        for name, shape, dtype in (("table", (self.world * self.world,), torch.int32),
                                   ("rows", (self.recv_cap, p.H), torch.bfloat16),
                                   ("ids", (self.recv_cap,), torch.int32),
                                   ("gates", (self.recv_cap,), torch.float32),
                                   ("origin", (self.recv_cap,), torch.int64),
                                   ("back", (p.T * p.top_k, p.H), torch.bfloat16)):
            t = symm_mem.empty(*shape, dtype=dtype, device=dev)
            h = symm_mem.rendezvous(t, self.group)
            base = h.buffer_ptrs[self.rank]
            off = t.data_ptr() - base
            self.bufs[name] = t
            self.handles[name] = h
            self.addr[name] = torch.tensor([b + off for b in h.buffer_ptrs], dtype=torch.int64,
                                           device=dev)
        self.n_recv = torch.zeros(1, dtype=torch.int32, device=dev)
        self.recv_problem = moe.Problem.make(self.recv_cap, p.H, p.F, e_loc, 1, p.act)
        self.ws_route = torch.empty(moe.moe_workspace_size(p), dtype=torch.uint8, device=dev)
        self.ws_recv = torch.empty(moe.moe_workspace_size(self.recv_problem), dtype=torch.uint8,
                                   device=dev)
        self.y = torch.empty(self.recv_cap, p.H, dtype=torch.bfloat16, device=dev)
        k = p.top_k
        self.identity = torch.arange(p.T * k, dtype=torch.int32, device=dev).view(p.T, k)

    def barrier(self, channel):
        self.handles["table"].barrier(channel=channel)


def ep_moe_forward_device(xch: DeviceExchange, x, Wg, bias, W1_local, W2_local):
    """The whole layer under expert parallelism, exchange driven by the device (csrc/ep.cuh):
    route and dispatch this rank's tokens, publish the counts, barrier, store the rows into
    their destinations' buffers, barrier, run this rank's experts on the rows it received
    (row count on the device), store the outputs back into their origins' return buffers,
    barrier, combine. Returns out [T, H] bf16; no host read of the routing."""
    from . import _native as moe

    p = xch.p
    dev = x.device
    T, k, E = p.T, p.top_k, p.E
    idx = torch.empty(T, k, dtype=torch.int32, device=dev)
    w = torch.empty(T, k, dtype=torch.float32, device=dev)
    moe.moe_route(p, x, Wg, bias, idx, w, xch.ws_route)
    pmax = moe.moe_padded_rows_max(p)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    poff = torch.empty(E + 1, dtype=torch.int32, device=dev)
    gather_idx = torch.empty(pmax, dtype=torch.int32, device=dev)
    inv_pos = torch.empty(T, k, dtype=torch.int32, device=dev)
    moe.moe_dispatch(p, idx, counts, offsets, poff, gather_idx, inv_pos, xch.ws_route)
    moe.moe_ep_publish_counts(p, xch.world, xch.rank, offsets, xch.addr["table"])
    xch.barrier(0)
    a = xch.addr
    moe.moe_ep_scatter(p, xch.world, xch.rank, x, idx, w, offsets, poff, inv_pos,
                       xch.bufs["table"], a["rows"], a["ids"], a["gates"], a["origin"],
                       xch.recv_cap, xch.n_recv, xch.ws_route)
    xch.barrier(1)
    moe.moe_experts_forward_n(xch.recv_problem, xch.bufs["rows"], xch.bufs["ids"],
                              xch.bufs["gates"], xch.n_recv, W1_local, W2_local, xch.y,
                              xch.ws_recv)
    moe.moe_ep_return(p.H, xch.world, xch.y, xch.bufs["origin"], xch.n_recv, xch.recv_cap,
                      a["back"], T * k, xch.ws_recv)
    xch.barrier(2)
    out = torch.empty(T, p.H, dtype=torch.bfloat16, device=dev)
    moe.moe_combine(p, xch.bufs["back"], xch.identity, out)
    return out


def ep_layer_buffers(p, world: int, device=None):
    """One rank's exchange buffers for moe_ep_layer_forward, zero-filled (plain device
    tensors: for several ranks on one GPU)."""
    from . import _native as moe

    dev = device if device is not None else torch.device("cuda", torch.cuda.current_device())
    return [torch.zeros(max(n, 16), dtype=torch.uint8, device=dev)
            for n in moe.moe_ep_buffer_sizes(p, world)]


def ep_layer_forward_local(p, xs, Wg, bias, W1s, W2s, outs, bufs, wss, epoch: int,
                           stream=None):
    """The expert-parallel layer for world = len(xs) ranks in one launch on this GPU: rank r's
    tokens xs[r] [T, H], its experts W1s[r] [E/world, H, 2F], W2s[r] [E/world, F, H], its
    output outs[r] [T, H], its buffers bufs[r] (ep_layer_buffers) and workspace wss[r]
    (moe_ep_workspace_size bytes). epoch: 1, 2, ... on successive calls with these buffers."""
    from . import _native as moe

    world = len(xs)
    if world > moe.EP_MAX_LOCAL:
        raise ValueError(f"at most {moe.EP_MAX_LOCAL} ranks in one launch")
    table = [[bufs[d][b] for d in range(world)] for b in range(len(moe.EP_BUFFERS))]
    ranks = [moe.ep_rank(p, world, r, epoch, xs[r], Wg, bias, W1s[r], W2s[r], outs[r], wss[r],
                         table) for r in range(world)]
    moe.moe_ep_layer_forward(ranks, stream)


class EpLayer:
    """The expert-parallel layer, one GPU per rank (moe_ep_layer_forward with one rank per
    launch). The exchange buffers are symmetric allocations (every rank addresses every
    rank's copy); the ranks must create it together (a collective) and then call forward
    together, once per layer call."""

    def __init__(self, p, group=None, device=None):
        import torch.distributed._symmetric_memory as symm_mem

        from . import _native as moe

        self.group = group if group is not None else dist.group.WORLD
        self.world = dist.get_world_size(self.group)
        self.rank = dist.get_rank(self.group)
        dev = device if device is not None else torch.device("cuda", torch.cuda.current_device())
        experts_per_rank(p.E, self.world)
        self.p = p
        self.epoch = 0
        self.bufs, self.handles, self.table = [], [], []
        for n in moe.moe_ep_buffer_sizes(p, self.world):
            t = symm_mem.empty(max(n, 16), dtype=torch.uint8, device=dev)
            t.zero_()
            h = symm_mem.rendezvous(t, self.group)
            off = t.data_ptr() - h.buffer_ptrs[self.rank]
            self.bufs.append(t)
            self.handles.append(h)
            self.table.append([int(b) + off for b in h.buffer_ptrs])
        self.ws = torch.empty(moe.moe_ep_workspace_size(p, self.world), dtype=torch.uint8,
                              device=dev)
        torch.cuda.synchronize(dev)
        self.handles[0].barrier(channel=0) # every rank's buffers are zero

    def forward(self, x, Wg, bias, W1_local, W2_local, out=None):
        from . import _native as moe

        self.epoch += 1
        if out is None:
            out = torch.empty(self.p.T, self.p.H, dtype=torch.bfloat16, device=x.device)
        r = moe.ep_rank(self.p, self.world, self.rank, self.epoch, x, Wg, bias, W1_local,
                        W2_local, out, self.ws, self.table)
        moe.moe_ep_layer_forward([r])
        return out
