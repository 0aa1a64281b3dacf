"""The expert-parallel building blocks on one GPU: moe_experts_forward reproduces the routed
rows of moe_forward bit for bit, and ep.ep_moe_forward over a one-rank NCCL group equals
moe_forward. The multi-rank exchange itself is tested on CPU (tests/test_ep_gloo.py)."""
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
