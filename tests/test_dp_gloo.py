"""Multi-process (gloo, world size 2, CPU) checks of the data-parallel host logic.

The layer is independent per token, so replicas need no collective on the data path: the
oracle output of a batch equals the concatenation of the outputs of its token shards. The
only cross-rank operations are barriers and the max-over-ranks timing reduction."""
import os

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from mixture_experts_layer_forward_b200 import dp


def _worker(rank, world, port, tmpdir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        from mixture_experts_layer_forward_b200 import synth

        r, lr, w = dp.env_rank()
        assert (r, lr, w) == (rank, rank, world)
        cfg = synth.LayerConfig("dp", T=50, H=64, F=64, E=6, k=2)
        inp = synth.make_inputs(cfg, seed=4)
        bits = {k: synth.bf16_bits(v) for k, v in inp.items() if v is not None}
        start, count = dp.shard_tokens(cfg.T, rank, world)
        toks = np.arange(start, start + count, dtype=np.int32)
        out, _, _ = oracle.moe_tokens(bits["x"], bits["Wg"], None, bits["W1"], bits["W2"], cfg.k, toks)
        # gather shards only to check them (a replica run never needs this)
        sizes = [None] * world
        dist.all_gather_object(sizes, (start, out))
        got = dp.max_over_ranks(float(rank) * 10.0 + 1.0)
        dp.barrier()
        if rank == 0:
            full, _, _ = oracle.moe_forward(bits["x"], bits["Wg"], None, bits["W1"], bits["W2"], cfg.k)
            parts = sorted(sizes, key=lambda s: s[0])
            cat = np.concatenate([p[1] for p in parts], axis=0)
            np.testing.assert_allclose(cat, full, rtol=1e-12, atol=1e-14)
            assert got == 10.0 * (world - 1) + 1.0
            open(os.path.join(tmpdir, "ok"), "w").write("ok")
    finally:
        dist.destroy_process_group()


def test_token_shards_partition_the_batch():
    for T in (0, 1, 7, 50, 8192):
        for world in (1, 2, 3, 8):
            spans = [dp.shard_tokens(T, r, world) for r in range(world)]
            assert sum(c for _, c in spans) == T
            pos = 0
            for s, c in spans:
                assert s == pos
                pos += c


def test_replica_seeds_are_distinct():
    seeds = {dp.replica_x_seed(0, r) for r in range(8)}
    assert len(seeds) == 8


def test_two_rank_gloo_shards_equal_whole_batch(tmp_path):
    port = 29500 + (os.getpid() % 2000)
    mp.start_processes(_worker, args=(2, port, str(tmp_path)), nprocs=2, join=True, start_method="spawn")
    assert (tmp_path / "ok").exists()
