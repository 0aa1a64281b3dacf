"""moe_route_noalloc: the router entry point that allocates nothing.

It exists for callers that cannot allocate device memory -- code that a host framework
hands only its input and output buffers (a plugin inside an inference engine that owns the
device heap), or a serving loop that must not call cudaMalloc/cudaFree after start-up
because those calls can synchronise the device and stall other streams. Its logits scratch
is a fixed array inside the library instead of a caller-provided workspace.

The file name sorts last, so pytest collects these tests after every other file. That is
only about reporting: if a test here fails, a run that stops at its first failure (-x) has
already run and reported the rest of the suite. Nothing here depends on what ran before:
the tests pass alone in a fresh process and after the whole suite.

The routing is checked against the CPU oracle (indices bit-exact, gates within 1e-6
relative) and against moe_route with a caller workspace.
"""
import ctypes

import numpy as np
import pytest
import torch

import mixture_experts_layer_forward_b200 as moe
import oracle
from mixture_experts_layer_forward_b200 import synth

pytestmark = pytest.mark.gpu

MAX_LOGITS = 1 << 20   # MOE_ROUTE_NOALLOC_MAX_LOGITS in include/moe.h


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)


def _route_with_workspace(cfg, inp):
    p = moe.Problem.from_config(cfg)
    ws = torch.empty(moe.moe_workspace_size(p), dtype=torch.uint8, device="cuda")
    idx = torch.empty(cfg.T, cfg.k, dtype=torch.int32, device="cuda")
    w = torch.empty(cfg.T, cfg.k, dtype=torch.float32, device="cuda")
    bias = None if inp["bias"] is None else inp["bias"].cuda()
    moe.moe_route(p, inp["x"].cuda(), inp["Wg"].cuda(), bias, idx, w, ws)
    return idx, w


def _route_noalloc_c_abi(cfg, inp):
    """Call the C entry point directly through ctypes (no workspace argument exists)."""
    lib = moe.library()
    p = moe.Problem.from_config(cfg)
    idx = torch.full((cfg.T, cfg.k), -1, dtype=torch.int32, device="cuda")
    w = torch.full((cfg.T, cfg.k), -1.0, dtype=torch.float32, device="cuda")
    x, Wg = inp["x"].cuda(), inp["Wg"].cuda()
    bias = None if inp["bias"] is None else inp["bias"].cuda()
    vp = ctypes.c_void_p
    rc = lib.moe_route_noalloc(ctypes.byref(p), vp(x.data_ptr()), vp(Wg.data_ptr()),
                               None if bias is None else vp(bias.data_ptr()),
                               vp(idx.data_ptr()), vp(w.data_ptr()),
                               vp(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, rc
    torch.cuda.synchronize()
    return idx, w


def _oracle_route(cfg, inp):
    b = None if inp["bias"] is None else inp["bias"].numpy()
    # with the selection-only bias the logits exclude it and the top-k adds it to the keys
    logits = oracle.router_logits(synth.bf16_bits(inp["x"]), synth.bf16_bits(inp["Wg"]),
                                  None if cfg.gate == moe.GATE_SELECT_BIAS else b)
    return oracle.topk_gates(logits, cfg.k, gate=cfg.gate, bias=b)


def test_noalloc_route_matches_oracle_on_two_calls_in_a_row():
    # different layers back to back: a later call must not see an earlier call's logits
    cases = [synth.LayerConfig("a", T=4096, H=512, F=64, E=256, k=8, zipf_s=1.2),
             synth.LayerConfig("b", T=3000, H=1024, F=64, E=8, k=2),
             synth.LayerConfig("c", T=1000, H=256, F=64, E=64, k=4, zipf_s=1.2,
                               gate=moe.GATE_SELECT_BIAS)]
    for i, cfg in enumerate(cases):
        inp = synth.make_inputs(cfg, seed=20 + i)
        ref_idx, ref_w = _oracle_route(cfg, inp)
        idx_ws, w_ws = _route_with_workspace(cfg, inp)
        idx, w = _route_noalloc_c_abi(cfg, inp)
        assert np.array_equal(idx.cpu().numpy(), ref_idx), cfg.name
        np.testing.assert_allclose(w.cpu().numpy(), ref_w, rtol=1e-6, atol=1e-7)
        assert torch.equal(idx, idx_ws), cfg.name
        np.testing.assert_allclose(w.cpu().numpy(), w_ws.cpu().numpy(), rtol=1e-6, atol=1e-7)


def test_noalloc_route_rejects_sizes_beyond_its_scratch():
    lib = moe.library()
    p = moe.Problem.make(MAX_LOGITS // 256 + 1, 64, 64, 256, 8)   # T * E just above the limit
    x = torch.zeros(p.T, 64, dtype=torch.bfloat16, device="cuda")
    Wg = torch.zeros(64, 256, dtype=torch.bfloat16, device="cuda")
    idx = torch.empty(p.T, 8, dtype=torch.int32, device="cuda")
    w = torch.empty(p.T, 8, dtype=torch.float32, device="cuda")
    vp = ctypes.c_void_p
    rc = lib.moe_route_noalloc(ctypes.byref(p), vp(x.data_ptr()), vp(Wg.data_ptr()), None,
                               vp(idx.data_ptr()), vp(w.data_ptr()), None)
    assert rc == -2   # MOE_ERR_UNSUPPORTED
