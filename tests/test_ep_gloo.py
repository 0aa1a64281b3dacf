"""Expert parallelism on CPU (gloo, world sizes 2 and 4): the exchange plan of ep.ep_forward.

Each rank routes its own tokens with the oracle's router, keeps E / world of the experts, and
runs the same row function on the rows it receives; the result must equal, bit for bit,
the same row function applied to its own routed pairs with all experts at hand and combined
in the same order: the exchange only moves rows. The GPU form of the two steps
(moe_experts_forward, moe_combine over NCCL) is covered by tests/test_gpu_ep.py."""
import os

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from mixture_experts_layer_forward_b200 import ep


def _row_fn(W1, W2, F, id_offset=0):
    """gate * FFN_e(x) per row in fp64 (SwiGLU), rounded once to bf16."""
    def fn(rows, ids, gates):
        out = torch.empty(rows.shape, dtype=torch.bfloat16)
        for r in range(rows.shape[0]):
            e = int(ids[r]) + id_offset
            z = rows[r].double() @ W1[e].double()
            a = torch.nn.functional.silu(z[:F]) * z[F:]
            out[r] = (float(gates[r]) * (a @ W2[e].double())).to(torch.bfloat16)
        return out
    return fn


def _combine(back, inv_pos):
    T, k = inv_pos.shape
    out = torch.empty(T, back.shape[1], dtype=torch.bfloat16)
    for t in range(T):
        s = torch.zeros(back.shape[1], dtype=torch.float32)
        for j in range(k):
            s = s + back[int(inv_pos[t, j])].float()
        out[t] = s.to(torch.bfloat16)
    return out


def _worker(rank, world, port, tmpdir, skewed):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        from mixture_experts_layer_forward_b200 import synth

        cfg = synth.LayerConfig("ep", T=37 + 5 * rank, H=32, F=16, E=4, k=2)
        inp = synth.make_inputs(cfg, seed=3, x_seed=100 + rank)
        bias = None
        if skewed:  # every token picks experts 0 and 1: rank 1 receives no rows
            bias = np.array([50.0, 40.0, 0.0, 0.0], np.float32)
        logits = oracle.router_logits(synth.bf16_bits(inp["x"]), synth.bf16_bits(inp["Wg"]), bias)
        idx, w = oracle.topk_gates(logits, cfg.k)
        idx = torch.from_numpy(idx.astype(np.int32))
        w = torch.from_numpy(w.astype(np.float32))
        e_loc = ep.experts_per_rank(cfg.E, world)
        mine = slice(rank * e_loc, (rank + 1) * e_loc)
        got = ep.ep_forward(inp["x"], idx, w, cfg.E,
                            _row_fn(inp["W1"][mine], inp["W2"][mine], cfg.F), _combine)
        # the same rows with every expert at hand, in (token, selection) order
        pairs = torch.arange(cfg.T * cfg.k)
        rows = inp["x"][pairs // cfg.k]
        ref_rows = _row_fn(inp["W1"], inp["W2"], cfg.F)(rows, idx.reshape(-1), w.reshape(-1))
        ref = _combine(ref_rows, pairs.view(cfg.T, cfg.k).int())
        assert torch.equal(got.view(torch.int16), ref.view(torch.int16))
        order, counts, _ = ep.dispatch_plan(idx, cfg.E, world)
        assert int(counts.sum()) == cfg.T * cfg.k
        if skewed:
            assert int(counts[1]) == 0
        open(os.path.join(tmpdir, f"ok{rank}"), "w").write("ok")
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,skewed", [(2, False), (2, True), (4, False)],
                         ids=["balanced", "one_rank_idle", "four_ranks"])
def test_ep_exchange_matches_local_compute(tmp_path, world, skewed):
    port = 29600 + (11 if skewed else 0) + (23 if world == 4 else 0) + os.getpid() % 97
    mp.spawn(_worker, args=(world, port, str(tmp_path), skewed), nprocs=world, join=True)
    assert all(os.path.exists(tmp_path / f"ok{r}") for r in range(world))


def test_dispatch_plan_is_stable_and_local():
    idx = torch.tensor([[3, 0], [1, 2], [0, 3], [2, 1]], dtype=torch.int32)
    order, counts, local = ep.dispatch_plan(idx, 4, 2)
    # pairs to rank 0 (experts 0, 1) first, each group in (token, selection) order
    assert order.tolist() == [1, 2, 4, 7, 0, 3, 5, 6]
    assert counts.tolist() == [4, 4]
    assert local.tolist() == [0, 1, 0, 1, 1, 0, 1, 0]
    with pytest.raises(ValueError):
        ep.experts_per_rank(6, 4)
