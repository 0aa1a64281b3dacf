"""Failure detection on the GPU without a fault: the fused kernel's tile-level ready-flag
waits are bounded. A test hook withholds one ready signal (a flag that nothing then sets);
the waits run out, the kernel records MOE_ERR_DEVICE_TIMEOUT in the workspace status word
and returns, and the next call on the same context succeeds. Nothing traps or hangs."""
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


def _forward(cfg, d, ws):
    p = moe.Problem.from_config(cfg)
    out = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device="cuda")
    moe.moe_forward(p, d["x"], d["Wg"], d["bias"], d["W1"], d["W2"], out, ws)
    return out, moe.moe_get_device_status(ws)


# T*k < 128 E: layer0 rows gathered in the kernel; T*k >= 128 E: sorted rows by TMA, and the
# data-movement warps take half of each layer0 epilogue before the combine; E = 8 with sorted
# rows: the whole layer in one launch (routing and dispatch first, then the same GEMM phases)
@pytest.mark.parametrize("T,E", [(300, 8), (700, 4), (1100, 8)],
                         ids=["gathered_rows", "sorted_rows", "whole_layer"])
def test_withheld_ready_signal_times_out_and_context_recovers(T, E):
    cfg = synth.LayerConfig("fault", T=T, H=256, F=256, E=E, k=2)
    inp = synth.make_inputs(cfg, seed=21)
    d = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    ws = torch.empty(moe.moe_workspace_size(moe.Problem.from_config(cfg)), dtype=torch.uint8,
                     device="cuda")
    prev_mode = moe.moe_set_gemm_mode(moe.GEMM_FUSED)
    prev_tmo = moe.moe_set_wait_timeout_ns(50_000_000)  # 50 ms
    try:
        moe.moe_set_fault_injection(0)               # layer0 item 0 never signals
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record()
        _, status = _forward(cfg, d, ws)
        t1.record()
        torch.cuda.synchronize()
        assert status == -5                          # MOE_ERR_DEVICE_TIMEOUT
        assert t0.elapsed_time(t1) < 2000.0          # ended by the bounded waits
        moe.moe_set_fault_injection(-1)
        out, status = _forward(cfg, d, ws)           # same context, next call is clean
        assert status == 0
        ref, _, _ = oracle.moe_forward(synth.bf16_bits(inp["x"]), synth.bf16_bits(inp["Wg"]), None,
                                       synth.bf16_bits(inp["W1"]), synth.bf16_bits(inp["W2"]), cfg.k)
        got = out.float().cpu().numpy().astype(np.float64)
        assert np.all(np.abs(got - ref) <= 2e-2 + 2e-2 * np.abs(ref))
    finally:
        moe.moe_set_fault_injection(-1)
        moe.moe_set_wait_timeout_ns(prev_tmo)
        moe.moe_set_gemm_mode(prev_mode)
