"""FP8 (e4m3) expert path against the CPU oracle: the quantisers bit for bit, the layer
within the bf16 path's tolerance (the codes are the same on both sides; the GPU sums the
code products in fp32 on the tensor cores and rounds h and ys to bf16)."""
import math

import numpy as np
import pytest
import torch

import mixture_experts_layer_forward_b200 as moe
import oracle
from mixture_experts_layer_forward_b200 import synth

pytestmark = pytest.mark.gpu

ATOL, RTOL = 2e-2, 2e-2


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)


def bits(t):
    return synth.bf16_bits(t)


def quantize_on_gpu(p, inp):
    E, H, F = p.E, p.H, p.F
    w1c = 2 * F if p.act == moe.ACT_SWIGLU else F
    W1q = torch.empty(E, w1c, H, dtype=torch.uint8, device="cuda")
    W2q = torch.empty(E, H, F, dtype=torch.uint8, device="cuda")
    s1 = torch.empty(E, w1c, dtype=torch.float32, device="cuda")
    s2 = torch.empty(E, H, dtype=torch.float32, device="cuda")
    moe.moe_quantize_experts_fp8(p, inp["W1"].cuda(), inp["W2"].cuda(), W1q, s1, W2q, s2)
    return W1q, s1, W2q, s2


def forward_fp8(p, inp, q):
    ws = torch.empty(moe.moe_workspace_size_fp8(p), dtype=torch.uint8, device="cuda")
    d = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    out = torch.empty(p.T, p.H, dtype=torch.bfloat16, device="cuda")
    idx = torch.empty(p.T, p.top_k, dtype=torch.int32, device="cuda")
    moe.moe_forward_fp8(p, d["x"], d["Wg"], d["bias"], *q, out, ws, topk_idx_out=idx)
    assert moe.moe_get_device_status(ws) == 0
    return out, idx


def assert_close(got_bf16, ref, what):
    got = got_bf16.float().cpu().numpy().astype(np.float64)
    err = np.abs(got - ref)
    bad = err > ATOL + RTOL * np.abs(ref)
    assert not bad.any(), f"{what}: {bad.sum()} elements out of tolerance; max |err| {err.max():.3e}"


def test_quantize_rows_bit_exact():
    g = torch.Generator().manual_seed(1)
    x = torch.randn(300, 512, generator=g)
    x[3] = 0.0                                  # zero row: scale 1, codes 0
    x[4] *= 1e-30                               # tiny row: 448 / amax overflows, scale 1
    x[5] *= 3e4                                 # large values
    x[6, ::7] = 0.0
    x[7] = torch.linspace(-2, 2, 512)           # many values near code boundaries
    xb = x.to(torch.bfloat16)
    q = torch.empty(300, 512, dtype=torch.uint8, device="cuda")
    s = torch.empty(300, dtype=torch.float32, device="cuda")
    moe.moe_quantize_rows_fp8(xb.cuda(), q, s)
    rq, rs = oracle.quant_rows_fp8(bits(xb))
    np.testing.assert_array_equal(q.cpu().numpy(), rq)
    np.testing.assert_array_equal(s.cpu().numpy().view(np.uint32), rs.view(np.uint32))


@pytest.mark.parametrize("act", [moe.ACT_SWIGLU, moe.ACT_GELU_TANH])
def test_quantize_experts_bit_exact(act):
    cfg = synth.LayerConfig("q", T=8, H=384, F=256, E=3, k=1, act=act)
    inp = synth.make_inputs(cfg, seed=4)
    p = moe.Problem.from_config(cfg)
    W1q, s1, W2q, s2 = quantize_on_gpu(p, inp)
    r1q, r1s = oracle.quant_cols_fp8(bits(inp["W1"]))
    r2q, r2s = oracle.quant_cols_fp8(bits(inp["W2"]))
    np.testing.assert_array_equal(W1q.cpu().numpy(), r1q)
    np.testing.assert_array_equal(W2q.cpu().numpy(), r2q)
    np.testing.assert_array_equal(s1.cpu().numpy().view(np.uint32), r1s.view(np.uint32))
    np.testing.assert_array_equal(s2.cpu().numpy().view(np.uint32), r2s.view(np.uint32))


FP8_CASES = [
    # name, T, H, F, E, k, act, zipf
    ("ragged", 300, 256, 256, 16, 2, 0, 1.2),
    ("several_tiles", 1000, 512, 384, 8, 2, 0, 0.0),
    ("many_experts", 77, 128, 128, 64, 8, 0, 0.0),
    ("relu", 260, 256, 384, 4, 2, 2, 0.0),
    ("gelu_odd_n_tiles", 150, 384, 128, 4, 1, 1, 0.0),
    # every expert single-tile: the operand-swapped narrow body
    ("narrow_swiglu", 16, 256, 384, 32, 4, 0, 1.2),
    ("narrow_relu", 40, 384, 256, 16, 2, 2, 0.0),
]


@pytest.fixture(params=[moe.GEMM_SINGLE_CTA, moe.GEMM_CTA_PAIR], ids=["single_cta", "cta_pair"])
def fp8_gemm_mode(request):
    prev = moe.moe_set_gemm_mode(request.param)
    yield request.param
    moe.moe_set_gemm_mode(prev)


@pytest.mark.parametrize("case", FP8_CASES, ids=[c[0] for c in FP8_CASES])
def test_forward_fp8_matches_oracle(case, fp8_gemm_mode):
    name, T, H, F, E, k, act, zipf = case
    cfg = synth.LayerConfig(name, T=T, H=H, F=F, E=E, k=k, act=act, zipf_s=zipf)
    inp = synth.make_inputs(cfg, seed=13)
    p = moe.Problem.from_config(cfg)
    out, idx = forward_fp8(p, inp, quantize_on_gpu(p, inp))
    r1q, r1s = oracle.quant_cols_fp8(bits(inp["W1"]))
    r2q, r2s = oracle.quant_cols_fp8(bits(inp["W2"]))
    b = None if inp["bias"] is None else inp["bias"].numpy()
    ref, ridx, _ = oracle.moe_tokens_fp8(bits(inp["x"]), bits(inp["Wg"]), b, r1q, r1s, r2q, r2s,
                                         k, np.arange(T), act=act)
    np.testing.assert_array_equal(idx.cpu().numpy(), ridx)
    assert_close(out, ref, name)


@pytest.mark.parametrize("case", FP8_CASES[:2], ids=[c[0] for c in FP8_CASES[:2]])
def test_forward_fp8_phased_order_matches_oracle(case):
    """The phased order (single-tile experts in the narrow body first) on the FP8 path."""
    name, T, H, F, E, k, act, zipf = case
    cfg = synth.LayerConfig(name, T=T, H=H, F=F, E=E, k=k, act=act, zipf_s=zipf)
    inp = synth.make_inputs(cfg, seed=13)
    p = moe.Problem.from_config(cfg)
    prev = moe.moe_set_work_order(moe.ORDER_PHASED)
    try:
        out, idx = forward_fp8(p, inp, quantize_on_gpu(p, inp))
    finally:
        moe.moe_set_work_order(prev)
    r1q, r1s = oracle.quant_cols_fp8(bits(inp["W1"]))
    r2q, r2s = oracle.quant_cols_fp8(bits(inp["W2"]))
    b = None if inp["bias"] is None else inp["bias"].numpy()
    ref, ridx, _ = oracle.moe_tokens_fp8(bits(inp["x"]), bits(inp["Wg"]), b, r1q, r1s, r2q, r2s,
                                         k, np.arange(T), act=act)
    np.testing.assert_array_equal(idx.cpu().numpy(), ridx)
    assert_close(out, ref, name)


def test_forward_fp8_close_to_bf16_path():
    """The FP8 layer stays within its quantisation error of the bf16 layer on the GPU."""
    cfg = synth.LayerConfig("cmp", T=512, H=512, F=256, E=8, k=2)
    inp = synth.make_inputs(cfg, seed=2, device="cuda")
    p = moe.Problem.from_config(cfg)
    out8, _ = forward_fp8(p, inp, quantize_on_gpu(p, inp))
    ws = torch.empty(moe.moe_workspace_size(p), dtype=torch.uint8, device="cuda")
    out16 = torch.empty_like(out8)
    moe.moe_forward(p, inp["x"], inp["Wg"], inp["bias"], inp["W1"], inp["W2"], out16, ws)
    rel = (torch.linalg.norm((out8 - out16).float()) / torch.linalg.norm(out16.float())).item()
    assert rel < 0.08, rel


def test_forward_fp8_rejects_unsupported_shapes():
    p = moe.Problem.make(64, 192, 256, 8, 2)           # H % 128 != 0
    assert moe.moe_workspace_size_fp8(p) == 0


@pytest.mark.parametrize("name", ["mixtral", "skew_decode", "qwen2"])
def test_forward_fp8_full_size(name):
    """Bench-sized layers: the GPU quantiser against the oracle's in full, the layer on a
    token sample (the rarest experts' tokens and seeded random ones)."""
    cfg = synth.CONFIGS[name]
    inp = synth.make_inputs(cfg, seed=0, device="cuda")
    p = moe.Problem.from_config(cfg)
    q = quantize_on_gpu(p, inp)
    r1q, r1s = oracle.quant_cols_fp8(bits(inp["W1"]))
    r2q, r2s = oracle.quant_cols_fp8(bits(inp["W2"]))
    assert np.array_equal(q[0].cpu().numpy(), r1q) and np.array_equal(q[2].cpu().numpy(), r2q)
    assert np.array_equal(q[1].cpu().numpy(), r1s) and np.array_equal(q[3].cpu().numpy(), r2s)
    out, idx = forward_fp8(p, inp, q)
    gidx = idx.cpu().numpy()
    counts = np.bincount(gidx.reshape(-1), minlength=cfg.E)
    active = np.nonzero(counts)[0]
    rare = active[np.argsort(counts[active], kind="stable")][:3]
    toks = []
    for e in rare:
        toks += list(np.nonzero((gidx == e).any(axis=1))[0][:2])
    toks += list(np.random.default_rng(1).choice(cfg.T, size=min(cfg.T, 6), replace=False))
    toks = np.unique(np.array(toks, dtype=np.int32))
    b = None if inp["bias"] is None else inp["bias"].cpu().numpy()
    ref, ridx, _ = oracle.moe_tokens_fp8(bits(inp["x"]), bits(inp["Wg"]), b, r1q, r1s, r2q, r2s,
                                         cfg.k, toks, act=cfg.act, gate=cfg.gate)
    np.testing.assert_array_equal(gidx[toks], ridx)
    assert_close(out[torch.from_numpy(toks).long().cuda()], ref, name)
