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


# ---------------------------------------------------------------------------------------
# the expert-parallel layer with the exchange overlapped with the GEMMs (one persistent launch
# per rank; here every rank of the world in one launch on this GPU)
# ---------------------------------------------------------------------------------------

EP_LAYER_CASES = [
    # name, world, T per rank, H, F, E, k, zipf, gate
    ("w1_e8", 1, 600, 256, 256, 8, 2, 0.0, 0),
    ("w2_e8", 2, 700, 256, 320, 8, 2, 0.8, 0),
    ("w4_e8", 4, 500, 192, 256, 8, 2, 0.0, 0),
    ("w2_e16_k4", 2, 300, 256, 256, 16, 4, 1.2, 0),
    ("w4_e32_k4", 4, 257, 128, 192, 32, 4, 1.2, 0),
    ("w2_e8_selbias", 2, 400, 256, 256, 8, 3, 1.5, 2),
]


def _ep_layer_inputs(world, T, H, F, E, k, zipf, gate, seed):
    cfg = synth.LayerConfig("ep_layer", T=T * world, H=H, F=F, E=E, k=k, zipf_s=zipf, gate=gate)
    inp = synth.make_inputs(cfg, seed=seed, device="cuda")
    xs = [inp["x"][r * T:(r + 1) * T].contiguous() for r in range(world)]
    el = E // world
    W1s = [inp["W1"][r * el:(r + 1) * el].contiguous() for r in range(world)]
    W2s = [inp["W2"][r * el:(r + 1) * el].contiguous() for r in range(world)]
    return inp, xs, W1s, W2s


@pytest.mark.parametrize("name,world,T,H,F,E,k,zipf,gate", EP_LAYER_CASES,
                         ids=[c[0] for c in EP_LAYER_CASES])
def test_ep_layer_ranks_equal_forward(name, world, T, H, F, E, k, zipf, gate):
    """Every rank's output of the overlapped expert-parallel layer is bitwise moe_forward's
    on the rank's tokens with all E experts; a second call on the same buffers (next epoch)
    gives the same."""
    inp, xs, W1s, W2s = _ep_layer_inputs(world, T, H, F, E, k, zipf, gate, seed=31)
    p = moe.Problem.make(T, H, F, E, k, gate=gate)
    bufs = [ep.ep_layer_buffers(p, world) for _ in range(world)]
    wss = [torch.empty(moe.moe_ep_workspace_size(p, world), dtype=torch.uint8, device="cuda")
           for _ in range(world)]
    outs = [torch.empty(T, H, dtype=torch.bfloat16, device="cuda") for _ in range(world)]
    ep.ep_layer_forward_local(p, xs, inp["Wg"], inp["bias"], W1s, W2s, outs, bufs, wss, epoch=1)
    torch.cuda.synchronize()
    for r in range(world):
        assert moe.moe_get_device_status(wss[r]) == 0, r
    cfg_r = synth.LayerConfig("rank", T=T, H=H, F=F, E=E, k=k, gate=gate)
    for r in range(world):
        ref = {"x": xs[r], "Wg": inp["Wg"], "bias": inp["bias"], "W1": inp["W1"], "W2": inp["W2"]}
        _, out_ref, _, _ = _forward(cfg_r, ref)
        assert torch.equal(outs[r], out_ref), (name, r)
    first = [o.clone() for o in outs]
    ep.ep_layer_forward_local(p, xs, inp["Wg"], inp["bias"], W1s, W2s, outs, bufs, wss, epoch=2)
    torch.cuda.synchronize()
    for r in range(world):
        assert moe.moe_get_device_status(wss[r]) == 0
        assert torch.equal(outs[r], first[r])


def test_ep_layer_matches_oracle():
    """Two ranks in one launch against the oracle on all their tokens."""
    import oracle

    world, T, H, F, E, k = 2, 300, 256, 192, 8, 2
    inp, xs, W1s, W2s = _ep_layer_inputs(world, T, H, F, E, k, 0.0, 0, seed=32)
    p = moe.Problem.make(T, H, F, E, k)
    bufs = [ep.ep_layer_buffers(p, world) for _ in range(world)]
    wss = [torch.empty(moe.moe_ep_workspace_size(p, world), dtype=torch.uint8, device="cuda")
           for _ in range(world)]
    outs = [torch.empty(T, H, dtype=torch.bfloat16, device="cuda") for _ in range(world)]
    ep.ep_layer_forward_local(p, xs, inp["Wg"], None, W1s, W2s, outs, bufs, wss, epoch=1)
    torch.cuda.synchronize()
    got = torch.cat(outs).float().cpu().numpy().astype(np.float64)
    ref, _, _ = oracle.moe_forward(synth.bf16_bits(inp["x"].cpu()), synth.bf16_bits(inp["Wg"].cpu()),
                                   None, synth.bf16_bits(inp["W1"].cpu()),
                                   synth.bf16_bits(inp["W2"].cpu()), k)
    assert np.all(np.abs(got - ref) <= 2e-2 + 2e-2 * np.abs(ref))


def test_ep_layer_timeout_when_a_rank_never_comes():
    """The ranks' waits on one another are bounded: two ranks' buffers, but only rank 0 is
    launched; its flag wait gives up, the status word says MOE_ERR_DEVICE_TIMEOUT, and the
    context stays usable."""
    world, T, H, F, E, k = 2, 256, 128, 128, 8, 2
    inp, xs, W1s, W2s = _ep_layer_inputs(world, T, H, F, E, k, 0.0, 0, seed=33)
    p = moe.Problem.make(T, H, F, E, k)
    bufs = [ep.ep_layer_buffers(p, world) for _ in range(world)]
    wss = [torch.empty(moe.moe_ep_workspace_size(p, world), dtype=torch.uint8, device="cuda")
           for _ in range(world)]
    outs = [torch.empty(T, H, dtype=torch.bfloat16, device="cuda") for _ in range(world)]
    table = [[bufs[d][b] for d in range(world)] for b in range(len(moe.EP_BUFFERS))]
    r0 = moe.ep_rank(p, world, 0, 1, xs[0], inp["Wg"], None, W1s[0], W2s[0], outs[0], wss[0], table)
    prev = moe.moe_set_wait_timeout_ns(50_000_000)
    try:
        moe.moe_ep_layer_forward([r0])
        torch.cuda.synchronize()
        assert moe.moe_get_device_status(wss[0]) == -5
    finally:
        moe.moe_set_wait_timeout_ns(prev)
    # the same context: a complete call (both ranks, next epoch) succeeds
    ep.ep_layer_forward_local(p, xs, inp["Wg"], None, W1s, W2s, outs, bufs, wss, epoch=2)
    torch.cuda.synchronize()
    assert all(moe.moe_get_device_status(w) == 0 for w in wss)


@pytest.mark.parametrize("world", [2, 4])
def test_ep_layer_full_size_mixtral(world):
    """The Mixtral-shaped layer (8192 tokens, H 4096, F 14336, 8 experts, top-2) split over
    `world` ranks in one launch: every rank's output is bitwise moe_forward's on its tokens."""
    cfg = synth.CONFIGS["mixtral"]
    inp = synth.make_inputs(cfg, seed=34, device="cuda")
    T, el = cfg.T // world, cfg.E // world
    xs = [inp["x"][r * T:(r + 1) * T].contiguous() for r in range(world)]
    W1s = [inp["W1"][r * el:(r + 1) * el].contiguous() for r in range(world)]
    W2s = [inp["W2"][r * el:(r + 1) * el].contiguous() for r in range(world)]
    p = moe.Problem.make(T, cfg.H, cfg.F, cfg.E, cfg.k)
    bufs = [ep.ep_layer_buffers(p, world) for _ in range(world)]
    wss = [torch.empty(moe.moe_ep_workspace_size(p, world), dtype=torch.uint8, device="cuda")
           for _ in range(world)]
    outs = [torch.empty(T, cfg.H, dtype=torch.bfloat16, device="cuda") for _ in range(world)]
    ep.ep_layer_forward_local(p, xs, inp["Wg"], inp["bias"], W1s, W2s, outs, bufs, wss, epoch=1)
    torch.cuda.synchronize()
    del bufs, W1s, W2s
    cfg_r = synth.LayerConfig("rank", T=T, H=cfg.H, F=cfg.F, E=cfg.E, k=cfg.k)
    for r in range(world):
        assert moe.moe_get_device_status(wss[r]) == 0
        ref = {"x": xs[r], "Wg": inp["Wg"], "bias": inp["bias"], "W1": inp["W1"], "W2": inp["W2"]}
        _, out_ref, _, _ = _forward(cfg_r, ref)
        assert torch.equal(outs[r], out_ref), r
