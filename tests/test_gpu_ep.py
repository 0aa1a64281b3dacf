"""The expert-parallel building blocks on one GPU: moe_experts_forward reproduces the routed
rows of moe_forward bit for bit, ep.ep_moe_forward over a one-rank NCCL group equals
moe_forward, and so does the device-driven exchange (ep.ep_moe_forward_device: counts,
positions and row transfers on the GPU, symmetric-memory buffers, device barriers) run by
one rank, twice in a row on the same buffers. The multi-rank NCCL exchange plan is tested on
CPU (tests/test_ep_gloo.py); several GPUs are not available to these tests."""
import os

import numpy as np
import pytest
import torch
import torch.distributed as dist

import mixture_experts_layer_forward_b200 as moe
from mixture_experts_layer_forward_b200 import ep, synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)


def _forward(cfg, inp):
    p = moe.Problem.from_config(cfg)
    ws = torch.empty(moe.moe_workspace_size(p), dtype=torch.uint8, device="cuda")
    out = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device="cuda")
    idx = torch.empty(cfg.T, cfg.k, dtype=torch.int32, device="cuda")
    w = torch.empty(cfg.T, cfg.k, dtype=torch.float32, device="cuda")
    moe.moe_forward(p, inp["x"], inp["Wg"], inp["bias"], inp["W1"], inp["W2"], out, ws, idx, w)
    assert moe.moe_get_device_status(ws) == 0
    return p, out, idx, w


@pytest.mark.parametrize("name,T,E,k,zipf", [("mixed", 700, 16, 2, 1.2), ("cold", 40, 32, 4, 0.0)])
def test_experts_forward_rows_equal_forward(name, T, E, k, zipf):
    cfg = synth.LayerConfig(name, T=T, H=256, F=256, E=E, k=k, zipf_s=zipf)
    inp = synth.make_inputs(cfg, seed=9, device="cuda")
    p, out, idx, w = _forward(cfg, inp)
    pairs = torch.arange(T * k, device="cuda")
    rows = inp["x"].index_select(0, pairs // k)
    pr = moe.Problem.make(T * k, cfg.H, cfg.F, E, 1)
    ws = torch.empty(moe.moe_workspace_size(pr), dtype=torch.uint8, device="cuda")
    y = torch.empty(T * k, cfg.H, dtype=torch.bfloat16, device="cuda")
    moe.moe_experts_forward(pr, rows, idx.reshape(-1).contiguous(), w.reshape(-1).contiguous(),
                            inp["W1"], inp["W2"], y, ws)
    assert moe.moe_get_device_status(ws) == 0
    comb = y.float().view(T, k, cfg.H)
    s = comb[:, 0]
    for j in range(1, k):
        s = s + comb[:, j]
    assert torch.equal(s.to(torch.bfloat16).view(torch.int16), out.view(torch.int16))


def test_experts_forward_reports_bad_expert_id():
    cfg = synth.LayerConfig("bad", T=64, H=128, F=128, E=4, k=1)
    inp = synth.make_inputs(cfg, seed=2, device="cuda")
    p = moe.Problem.from_config(cfg)
    ids = torch.zeros(64, dtype=torch.int32, device="cuda")
    ids[5] = 4                                             # one past the last expert
    gates = torch.ones(64, dtype=torch.float32, device="cuda")
    ws = torch.empty(moe.moe_workspace_size(p), dtype=torch.uint8, device="cuda")
    y = torch.empty(64, 128, dtype=torch.bfloat16, device="cuda")
    moe.moe_experts_forward(p, inp["x"], ids, gates, inp["W1"], inp["W2"], y, ws)
    assert moe.moe_get_device_status(ws) == -6              # MOE_ERR_DEVICE_BAD_INDEX


def test_ep_single_rank_equals_forward():
    cfg = synth.LayerConfig("ep1", T=500, H=256, F=256, E=8, k=2, zipf_s=1.2)
    inp = synth.make_inputs(cfg, seed=4, device="cuda")
    p, out, _, _ = _forward(cfg, inp)
    port = 29700 + os.getpid() % 97
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            device_id=torch.device("cuda", 0))
    try:
        got = ep.ep_moe_forward(p, inp["x"], inp["Wg"], inp["bias"], inp["W1"], inp["W2"])
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    assert torch.equal(got.view(torch.int16), out.view(torch.int16))


def test_experts_forward_n_computes_only_the_counted_rows():
    """moe_experts_forward_n with a device row count: the first n rows equal
    moe_experts_forward on those rows, the rows past n are left untouched."""
    T, n = 300, 173
    cfg = synth.LayerConfig("rows_n", T=T, H=256, F=256, E=4, k=1)
    inp = synth.make_inputs(cfg, seed=31, device="cuda")
    g = torch.Generator(device="cuda").manual_seed(5)
    ids = torch.randint(0, 4, (T,), generator=g, device="cuda", dtype=torch.int32)
    gates = torch.rand(T, generator=g, device="cuda")
    p = moe.Problem.make(T, 256, 256, 4, 1)
    ws = torch.empty(moe.moe_workspace_size(p), dtype=torch.uint8, device="cuda")
    y = torch.full((T, 256), 7.0, dtype=torch.bfloat16, device="cuda")
    n_rows = torch.tensor([n], dtype=torch.int32, device="cuda")
    moe.moe_experts_forward_n(p, inp["x"], ids, gates, n_rows, inp["W1"], inp["W2"], y, ws)
    assert moe.moe_get_device_status(ws) == 0
    pn = moe.Problem.make(n, 256, 256, 4, 1)
    wsn = torch.empty(moe.moe_workspace_size(pn), dtype=torch.uint8, device="cuda")
    yn = torch.empty(n, 256, dtype=torch.bfloat16, device="cuda")
    moe.moe_experts_forward(pn, inp["x"][:n].contiguous(), ids[:n].contiguous(),
                            gates[:n].contiguous(), inp["W1"], inp["W2"], yn, wsn)
    assert moe.moe_get_device_status(wsn) == 0
    assert torch.equal(y[:n].view(torch.int16), yn.view(torch.int16))
    assert bool(torch.all(y[n:] == 7.0))


@pytest.mark.parametrize("T,E,k,zipf", [(500, 8, 2, 1.2), (96, 16, 4, 0.0)])
def test_device_exchange_single_rank_equals_forward(T, E, k, zipf):
    cfg = synth.LayerConfig("epd", T=T, H=256, F=256, E=E, k=k, zipf_s=zipf)
    inp = synth.make_inputs(cfg, seed=6, device="cuda")
    p, out, _, _ = _forward(cfg, inp)
    port = 29800 + os.getpid() % 97
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            device_id=torch.device("cuda", 0))
    try:
        xch = ep.DeviceExchange(p)
        got = [ep.ep_moe_forward_device(xch, inp["x"], inp["Wg"], inp["bias"], inp["W1"],
                                        inp["W2"]) for _ in range(2)]
        torch.cuda.synchronize()
        st = (moe.moe_get_device_status(xch.ws_route), moe.moe_get_device_status(xch.ws_recv))
        del xch
    finally:
        dist.destroy_process_group()
    assert st == (0, 0)
    for g in got:
        assert torch.equal(g.view(torch.int16), out.view(torch.int16))
