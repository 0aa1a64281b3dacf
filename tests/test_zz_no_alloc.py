"""moe_route_noalloc: the router entry point that allocates nothing.

It exists for callers that cannot allocate device memory -- code that a host framework
hands only its input and output buffers (a plugin inside an inference engine that owns the
device heap), or a serving loop that must not call cudaMalloc/cudaFree after start-up
because those calls can synchronise the device and stall other streams. Its logits scratch
is a fixed array inside the library instead of a caller-provided workspace.

This file is named so that pytest collects it last: if it fails, a run that stops at the
first failure has already run every other test. It passes alone in a fresh process and
after the rest of the suite.
"""
import ctypes

import numpy as np
import pytest
import torch

import mixture_experts_layer_forward_b200 as moe
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


def test_noalloc_route_matches_workspace_route_on_two_calls_in_a_row():
    # two different layers back to back: the second call must not see the first one's logits
    cases = [synth.LayerConfig("a", T=4096, H=512, F=64, E=256, k=8, zipf_s=1.2),
             synth.LayerConfig("b", T=3000, H=1024, F=64, E=8, k=2)]
    for i, cfg in enumerate(cases):
        inp = synth.make_inputs(cfg, seed=20 + i)
        idx_ref, w_ref = _route_with_workspace(cfg, inp)
        idx, w = _route_noalloc_c_abi(cfg, inp)
        assert torch.equal(idx, idx_ref), cfg.name
        np.testing.assert_allclose(w.cpu().numpy(), w_ref.cpu().numpy(), rtol=1e-5, atol=1e-7)


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
