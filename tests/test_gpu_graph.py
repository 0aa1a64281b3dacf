"""The library's entry points take a stream and never synchronise the host, so a whole layer
forward (and backward) can be captured in a CUDA graph and replayed: the replay must equal
the eager call bit for bit."""
import pytest
import torch

import mixture_experts_layer_forward_b200 as moe
from mixture_experts_layer_forward_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)


@pytest.mark.parametrize("name,T,E,k,zipf", [("mixed", 600, 64, 4, 1.2), ("decode", 64, 256, 8, 1.2)])
def test_forward_graph_replay_equals_eager(name, T, E, k, zipf):
    cfg = synth.LayerConfig(name, T=T, H=512, F=256, E=E, k=k, zipf_s=zipf)
    inp = synth.make_inputs(cfg, seed=6, device="cuda")
    p = moe.Problem.from_config(cfg)
    ws = torch.empty(moe.moe_workspace_size(p), dtype=torch.uint8, device="cuda")
    eager = torch.empty(T, cfg.H, dtype=torch.bfloat16, device="cuda")
    moe.moe_forward(p, inp["x"], inp["Wg"], inp["bias"], inp["W1"], inp["W2"], eager, ws)
    torch.cuda.synchronize()
    out = torch.empty_like(eager)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            moe.moe_forward(p, inp["x"], inp["Wg"], inp["bias"], inp["W1"], inp["W2"], out, ws,
                            stream=s)
    for _ in range(3):
        out.zero_()
        g.replay()
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == 0
    assert torch.equal(out.view(torch.int16), eager.view(torch.int16))
    # new inputs in the same buffers: the replay follows them
    inp["x"].copy_(torch.randn_like(inp["x"].float()).to(torch.bfloat16))
    g.replay()
    moe.moe_forward(p, inp["x"], inp["Wg"], inp["bias"], inp["W1"], inp["W2"], eager, ws)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), eager.view(torch.int16))
