"""Backward pass on the GPU against the CPU oracle's gradients (fp64, hand-derived and
pinned against autograd). The GPU keeps the intermediates (z, u, a, dz, gy, the rows' input
gradients) in bf16 with fp32 accumulation, so the bar is scale-relative: every element
within 2% of the tensor's largest magnitude plus 3% of its own."""
import math

import numpy as np
import pytest
import torch

import mixture_experts_layer_forward_b200 as moe
import oracle
from mixture_experts_layer_forward_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)


def bits(t):
    return synth.bf16_bits(t)


def assert_grad_close(got, ref, what):
    got = np.asarray(got, np.float64)
    scale = np.abs(ref).max()
    if scale == 0:  # e.g. the router gradients with k = 1 (every gate is 1)
        assert np.all(got == 0), what
        return
    err = np.abs(got - ref)
    bad = err > 2e-2 * scale + 3e-2 * np.abs(ref)
    assert not bad.any(), (f"{what}: {bad.sum()} of {bad.size} out of tolerance; max |err| "
                           f"{err.max():.3e}, scale {scale:.3e}")


def run_backward(p, inp, dy):
    d = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    w1c = 2 * p.F if p.act == moe.ACT_SWIGLU else p.F
    dx = torch.empty(p.T, p.H, dtype=torch.bfloat16, device="cuda")
    dWg = torch.empty(p.H, p.E, dtype=torch.float32, device="cuda")
    dbias = torch.empty(p.E, dtype=torch.float32, device="cuda")
    dW1 = torch.empty(p.E, p.H, w1c, dtype=torch.bfloat16, device="cuda")
    dW2 = torch.empty(p.E, p.F, p.H, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(moe.moe_backward_workspace_size(p), dtype=torch.uint8, device="cuda")
    moe.moe_backward(p, d["x"], d["Wg"], d["bias"], d["W1"], d["W2"], dy.cuda(), dx, dWg, dbias,
                     dW1, dW2, ws)
    assert moe.moe_get_device_status(ws) == 0
    f = lambda t: t.float().cpu().numpy()
    return dict(dx=f(dx), dWg=f(dWg), dbias=f(dbias), dW1=f(dW1), dW2=f(dW2))


def make_dy(T, H, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(T, H, generator=g).to(torch.bfloat16)


BWD_CASES = [
    # name, T, H, F, E, k, act, gate, zipf
    ("swiglu_bias", 300, 256, 256, 8, 2, 0, 0, 1.2),
    ("relu_k4", 200, 128, 384, 16, 4, 2, 0, 0.0),
    ("gelu", 130, 256, 128, 4, 1, 1, 0, 0.0),
    ("select_bias", 150, 128, 256, 8, 2, 0, 2, 1.2),
    ("empty_experts", 40, 128, 128, 64, 2, 0, 0, 0.0),
    ("several_tiles", 700, 256, 256, 4, 2, 0, 0, 0.0),
]


@pytest.mark.parametrize("case", BWD_CASES, ids=[c[0] for c in BWD_CASES])
def test_backward_matches_oracle(case):
    name, T, H, F, E, k, act, gate, zipf = case
    cfg = synth.LayerConfig(name, T=T, H=H, F=F, E=E, k=k, act=act, gate=gate, zipf_s=zipf)
    inp = synth.make_inputs(cfg, seed=17)
    dy = make_dy(T, H, 18)
    p = moe.Problem.from_config(cfg)
    got = run_backward(p, inp, dy)
    b = None if inp["bias"] is None else inp["bias"].numpy()
    ref = oracle.moe_backward(bits(inp["x"]), bits(inp["Wg"]), b, bits(inp["W1"]), bits(inp["W2"]),
                              bits(dy), k, act=act, gate=gate)
    for key in ("dx", "dW1", "dW2", "dWg"):
        assert_grad_close(got[key], ref[key], f"{name} {key}")
    if b is None or gate == 2:
        assert np.all(got["dbias"] == 0)
    else:
        assert_grad_close(got["dbias"], ref["dbias"], f"{name} dbias")
    if name == "empty_experts":  # experts without rows get exactly zero weight gradients
        used = np.unique(oracle.topk_gates(oracle.router_logits(bits(inp["x"]), bits(inp["Wg"])), k)[0])
        unused = np.setdiff1d(np.arange(E), used)
        assert unused.size > 0
        assert np.all(got["dW1"][unused] == 0) and np.all(got["dW2"][unused] == 0)


def test_backward_rejects_unsupported():
    assert moe.moe_backward_workspace_size(moe.Problem.make(64, 192, 256, 8, 2)) == 0   # H % 128
    p = moe.Problem.make(64, 256, 256, 8, 2, gate=moe.GATE_SOFTMAX_ALL)
    assert moe.moe_backward_workspace_size(p) == 0


@pytest.mark.parametrize("name", ["qwen2", "mixtral"])
def test_backward_full_size_dx_sample(name):
    """Bench-sized layers: dx of a token sample against the oracle's per-token gradient; the
    weight gradients are checked for finiteness and for the experts without rows."""
    cfg = synth.CONFIGS[name]
    inp = synth.make_inputs(cfg, seed=0, device="cuda")
    dy = make_dy(cfg.T, cfg.H, 5)
    p = moe.Problem.from_config(cfg)
    got = run_backward(p, inp, dy)
    toks = np.random.default_rng(2).choice(cfg.T, size=6, replace=False).astype(np.int32)
    host = {k: (bits(v) if v is not None and v.dtype == torch.bfloat16 else v) for k, v in inp.items()}
    b = None if inp["bias"] is None else inp["bias"].cpu().numpy()
    ref = oracle.moe_backward_dx_tokens(host["x"], host["Wg"], b, host["W1"], host["W2"], bits(dy),
                                        cfg.k, toks, act=cfg.act, gate=cfg.gate)
    assert_grad_close(got["dx"][toks], ref, f"{name} dx")
    for key in ("dW1", "dW2", "dWg"):
        assert np.isfinite(got[key]).all(), key
